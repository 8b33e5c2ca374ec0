// Internal host interface between the C API (fa_api.cu) and the launchers.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "fa.h"

namespace fa {

struct AttnArgs {
  int dtype;  // 0 fp16, 1 bf16
  const void* q;
  const void* k;
  const void* v;
  const void* o;  // forward: output
  float* lse;     // forward: output; backward: input
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  void* workspace;
  int B, H, N, d;  // N: query rows
  int Nk = 0;      // key / value rows (0: equal to N)
  float scale;
  int causal;
  const uint8_t* block_mask;
  int32_t* trace;
  int* status;
  int phases = 7;  // backward launches to run: bit 0 prep, bit 1 main
  uint64_t timeout_ns = 2000000000ull;  // limit of every device-side wait
  int withhold = 0;  // debug (forward): the producer issues no load, so the first wait runs out
  // 8-bit forward: per-tensor scales of the e4m3 q, k, v
  float q_scale = 1.0f, k_scale = 1.0f, v_scale = 1.0f;
  // dropout on P: threshold t (drop iff draw < t; 0 = no dropout) and seed
  int drop_t = 0;
  uint64_t drop_seed = 0;
  // split-KV forward: partial results per key range (see launch_splitkv_merge)
  int n_splits = 1;
  float* o_part = nullptr;    // fp32 [n_splits][B*H][N][d]
  float* lse_part = nullptr;  // fp32 [n_splits][B*H][N]
};

// Return 0 on success, a cudaError_t value otherwise.
int launch_fwd(const AttnArgs& a, cudaStream_t stream);
// The 8-bit forward (a.q, a.k, a.v e4m3; a.o bf16; d = 128).
int launch_fwd_fp8(const AttnArgs& a, cudaStream_t stream);
// Merge of the split-KV partials (a.o_part, a.lse_part, a.n_splits) into a.o, a.lse.
int launch_splitkv_merge(const AttnArgs& a, cudaStream_t stream);
// Split-KV step 1 on the CUDA cores for at most kDecodeMaxRows query rows (fa_decode.cu).
constexpr int kDecodeMaxRows = 4;
int launch_decode_splitkv(const AttnArgs& a, cudaStream_t stream);

// Debug: the dropout draws of every (head, query row, key), through the
// row-major and the column-major generator paths of the attention kernels.
int launch_dropout_draws(int BH, int Nq, int Nk, uint64_t seed, uint8_t* row_major, uint8_t* col_major,
                         cudaStream_t stream);

// Workspace of the split-KV forward: partial O then partial lse, in bytes.
struct SplitWorkspace {
  size_t o_part;
  size_t lse_part;
  size_t total;
};
SplitWorkspace splitkv_workspace_layout(int B, int H, int Nq, int d, int n_splits);
int launch_bwd(const AttnArgs& a, cudaStream_t stream);

// Workspace layout of the backward, in bytes from the workspace base.
struct BwdWorkspace {
  size_t delta;     // fp32 [BH][Npad]  D = rowsum(dO o O)
  size_t lse2;      // fp32 [BH][Npad]  lse * log2(e), +inf on padding rows
  size_t total;
};
BwdWorkspace bwd_workspace_layout(int B, int H, int N, int d);
int bwd_row_tile(int d);

// Device address of the per-device status word (nullptr on failure).
int* device_status_word();

// Head dimensions the forward takes: 64, 128 and 256 natively, 32 and 96 inside
// the 64 and 128 kernels with the missing columns zero-filled by TMA. The
// backward takes all but 256.
bool head_dim_supported(int d);
bool bwd_head_dim_supported(int d);

// Limits every entry point applies to the element type and sizes of a square
// (N queries, N keys) problem: FA_OK, FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED.
fa_status check_common(fa_dtype dtype, int B, int H, int N, int d);

}  // namespace fa
