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
};

// Return 0 on success, a cudaError_t value otherwise.
int launch_fwd(const AttnArgs& a, cudaStream_t stream);
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

// Limits every entry point applies to the element type and sizes of a square
// (N queries, N keys) problem: FA_OK, FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED.
fa_status check_common(fa_dtype dtype, int B, int H, int N, int d);

}  // namespace fa
