// C ABI of the attention library: argument checks, the device status word and
// dispatch to the launchers. Declarations and contracts are in include/fa.h.
#include "fa.h"

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa_internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace {

// Status word written by kernels whose waits time out; one per device, in the
// library's static device memory, so no allocation is needed.
__device__ int g_fa_status;

__global__ void timeout_probe_kernel(int* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    fa::sm100::mbar_init(fa::sm100::smem_u32(&bar), 1);
    fa::sm100::fence_barrier_init();
  }
  __syncthreads();
  fa::sm100::WaitCtx ctx{&abort_flag, status, timeout_ns};
  // Nothing ever arrives on this barrier: the wait runs out and records the time-out.
  fa::sm100::mbar_wait(fa::sm100::smem_u32(&bar), 0, ctx);
}

int* status_word() {
  static std::mutex mu;
  static int* ptrs[128] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using fa::check_common;

// Dropout threshold t of probability p (drop iff draw < t): t = floor(256 p + 1/2),
// p in [0, 1); -1 if p is outside it.
int drop_threshold(float p_drop) {
  if (!(p_drop >= 0.0f && p_drop < 1.0f)) return -1;
  const int t = static_cast<int>(p_drop * 256.0f + 0.5f);
  return t > 255 ? 255 : t;
}

// The same limits for a problem with Nq query rows and Nk key rows (the
// backward grid holds batch*heads*(Tq + Tk) CTAs).
fa_status check_qk(fa_dtype dtype, int B, int H, int Nq, int Nk, int d) {
  fa_status s = check_common(dtype, B, H, Nq, d);
  if (s != FA_OK) return s;
  s = check_common(dtype, B, H, Nk, d);
  if (s != FA_OK) return s;
  const long long bh = static_cast<long long>(B) * H;
  const long long tiles = (static_cast<long long>(Nq) + 127) / 128 + (static_cast<long long>(Nk) + 127) / 128;
  if (bh * tiles > 0x7FFFFFFFLL) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status check_mask_qk(int Nq, int Nk) {
  if (Nq % 128 != 0 || Nk % 128 != 0 || Nq / 128 > 2048 || Nk / 128 > 2048) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status check_mask(int N, int d, const uint8_t* block_mask) {
  (void)d;
  if (block_mask == nullptr) return FA_ERR_INVALID_ARG;
  if (N % 128 != 0 || N / 128 > 2048) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status fwd_impl(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float scale, int causal, const uint8_t* mask, int32_t* trace,
                   cudaStream_t stream, int Nk = 0, uint64_t withhold_timeout_ns = 0, int drop_t = 0,
                   uint64_t drop_seed = 0) {
  fa_status s = Nk > 0 ? check_qk(dtype, B, H, N, Nk, d) : check_common(dtype, B, H, N, d);
  if (s != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  fa::AttnArgs a{};
  a.dtype = dtype;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = N;
  a.Nk = Nk;
  a.d = d;
  a.scale = scale;
  a.causal = causal ? 1 : 0;
  a.block_mask = mask;
  a.trace = trace;
  if (withhold_timeout_ns != 0) {
    a.withhold = 1;
    a.timeout_ns = withhold_timeout_ns;
  }
  a.drop_t = drop_t;
  a.drop_seed = drop_seed;
  a.status = status_word();
  if (!a.status) return FA_ERR_CUDA;
  return fa::launch_fwd(a, stream) == 0 ? FA_OK : FA_ERR_CUDA;
}

fa_status bwd_impl(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int N, int d,
                   float scale, int causal, const uint8_t* mask, int32_t* trace, cudaStream_t stream,
                   int phases = 7, int Nk = 0, uint64_t withhold_timeout_ns = 0, int drop_t = 0,
                   uint64_t drop_seed = 0) {
  fa_status s = Nk > 0 ? check_qk(dtype, B, H, N, Nk, d) : check_common(dtype, B, H, N, d);
  if (s != FA_OK) return s;
  if (!fa::bwd_head_dim_supported(d)) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  fa::AttnArgs a{};
  a.dtype = dtype;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = const_cast<float*>(lse);
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.workspace = workspace;
  a.B = B;
  a.H = H;
  a.N = N;
  a.Nk = Nk;
  a.d = d;
  a.scale = scale;
  a.causal = causal ? 1 : 0;
  a.block_mask = mask;
  a.trace = trace;
  a.phases = phases;
  if (withhold_timeout_ns != 0) {
    a.withhold = 1;
    a.timeout_ns = withhold_timeout_ns;
  }
  a.drop_t = drop_t;
  a.drop_seed = drop_seed;
  a.status = status_word();
  if (!a.status) return FA_ERR_CUDA;
  return fa::launch_bwd(a, stream) == 0 ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

int* fa::device_status_word() { return status_word(); }

bool fa::head_dim_supported(int d) { return d == 32 || d == 64 || d == 96 || d == 128 || d == 256; }

bool fa::bwd_head_dim_supported(int d) { return d == 32 || d == 64 || d == 96 || d == 128; }

fa_status fa::check_common(fa_dtype dtype, int B, int H, int N, int d) {
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (!fa::head_dim_supported(d)) return FA_ERR_UNSUPPORTED;
  const long long bh = static_cast<long long>(B) * H;
  const long long tiles = (static_cast<long long>(N) + 127) / 128;
  // Grids are 1-D over batch*heads*(2*tiles) CTAs (< 2^31); key-tile indices fit 16 bits.
  if (bh > 65535 || tiles > 32767 || bh * 2 * tiles > 0x7FFFFFFFLL) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status fa_fwd(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float softmax_scale, int causal, cudaStream_t stream) {
  return fwd_impl(dtype, q, k, v, o, lse, B, H, N, d, softmax_scale, causal, nullptr, nullptr, stream);
}

fa_status fa_blocksparse_fwd(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, cudaStream_t stream) {
  fa_status s = check_mask(N, d, block_mask);
  if (s != FA_OK) return s;
  return fwd_impl(dtype, q, k, v, o, lse, B, H, N, d, softmax_scale, causal, block_mask, nullptr, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || !fa::bwd_head_dim_supported(d)) return 0;
  return fa::bwd_workspace_layout(B, H, N, d).total;
}

int fa_bwd_row_tile(int d) { return fa::bwd_row_tile(d); }

fa_status fa_bwd(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int N, int d,
                 float softmax_scale, int causal, cudaStream_t stream) {
  return bwd_impl(dtype, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, N, d, softmax_scale, causal, nullptr,
                  nullptr, stream);
}

fa_status fa_blocksparse_bwd(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, cudaStream_t stream) {
  fa_status s = check_mask(N, d, block_mask);
  if (s != FA_OK) return s;
  return bwd_impl(dtype, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, N, d, softmax_scale, causal,
                  block_mask, nullptr, stream);
}

fa_status fa_fwd_qk(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int Nq, int Nk, int d, float softmax_scale, int causal, const uint8_t* block_mask,
                    cudaStream_t stream) {
  if (Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  if (block_mask != nullptr) {
    fa_status s = check_mask_qk(Nq, Nk);
    if (s != FA_OK) return s;
  }
  return fwd_impl(dtype, q, k, v, o, lse, B, H, Nq, d, softmax_scale, causal, block_mask, nullptr, stream, Nk);
}

fa_status fa_bwd_qk(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk,
                    int d, float softmax_scale, int causal, const uint8_t* block_mask, cudaStream_t stream) {
  if (Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  if (block_mask != nullptr) {
    fa_status s = check_mask_qk(Nq, Nk);
    if (s != FA_OK) return s;
  }
  return bwd_impl(dtype, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, d, softmax_scale, causal,
                  block_mask, nullptr, stream, 7, Nk);
}

size_t fa_fwd_trace_size(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  const size_t tiles = (static_cast<size_t>(N) + 127) / 128;
  const size_t pairs = (tiles + 1) / 2;
  return static_cast<size_t>(B) * H * pairs * (tiles + 1);
}

size_t fa_bwd_trace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || !fa::bwd_head_dim_supported(d)) return 0;
  const size_t t = (static_cast<size_t>(N) + 127) / 128;
  const size_t br = static_cast<size_t>(fa::bwd_row_tile(d));
  const size_t tq = (static_cast<size_t>(N) + br - 1) / br;
  return static_cast<size_t>(B) * H * t * ((tq + 1) + (t + 1));
}

fa_status fa_debug_fwd_trace(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, int32_t* trace, cudaStream_t stream) {
  if (trace == nullptr) return FA_ERR_INVALID_ARG;
  if (d == 256) return FA_ERR_UNSUPPORTED;  // the trace records pairs of query tiles
  if (block_mask) {
    fa_status s = check_mask(N, d, block_mask);
    if (s != FA_OK) return s;
  }
  return fwd_impl(dtype, q, k, v, o, lse, B, H, N, d, softmax_scale, causal, block_mask, trace, stream);
}

fa_status fa_debug_bwd_trace(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, int32_t* trace, cudaStream_t stream) {
  if (trace == nullptr) return FA_ERR_INVALID_ARG;
  if (block_mask) {
    fa_status s = check_mask(N, d, block_mask);
    if (s != FA_OK) return s;
  }
  return bwd_impl(dtype, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, N, d, softmax_scale, causal,
                  block_mask, trace, stream);
}

fa_status fa_debug_bwd_phase(int phase, fa_dtype dtype, const void* q, const void* k, const void* v,
                             const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             void* workspace, int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, cudaStream_t stream) {
  if (phase < 0 || phase > 1) return FA_ERR_INVALID_ARG;
  if (block_mask) {
    fa_status s = check_mask(N, d, block_mask);
    if (s != FA_OK) return s;
  }
  return bwd_impl(dtype, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, N, d, softmax_scale, causal,
                  block_mask, nullptr, stream, 1 << phase);
}

fa_status fa_device_status(cudaStream_t stream) {
  int* w = status_word();
  if (!w) return FA_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyAsync(&h, w, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaMemsetAsync(w, 0, sizeof(int), stream) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
  return static_cast<fa_status>(h);
}

size_t fa_fwd_splitkv_workspace_size(int B, int H, int Nq, int d, int n_splits) {
  if (B < 1 || H < 1 || Nq < 1 || n_splits < 1 || !fa::head_dim_supported(d)) return 0;
  return fa::splitkv_workspace_layout(B, H, Nq, d, n_splits).total;
}

int fa_fwd_splitkv_splits(int B, int H, int Nq, int Nk) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return 0;
  const int sms = fa::host::sm_count();
  if (sms < 1) return 1;
  const long long tq = (static_cast<long long>(Nq) + 127) / 128;
  const long long base = static_cast<long long>(B) * H * ((tq + 1) / 2);  // CTAs without splitting
  const long long tk = (static_cast<long long>(Nk) + 127) / 128;
  long long ns = base >= sms ? 1 : sms / base;  // one wave of CTAs
  if (tq == 1) ns *= 2;  // one query tile: a CTA takes two consecutive ranges
  if (Nq <= fa::kDecodeMaxRows) {
    // CUDA-core decoding: one range per CTA, two CTAs per SM, one wave.
    const long long heads = static_cast<long long>(B) * H;
    ns = heads >= 2LL * sms ? 1 : (2LL * sms) / heads;
  }
  if (ns > tk) ns = tk;
  return static_cast<int>(ns < 1 ? 1 : ns);
}

fa_status fa_fwd_splitkv(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Nq, int Nk, int d, float softmax_scale, int causal, const uint8_t* block_mask,
                         int n_splits, void* workspace, cudaStream_t stream) {
  if (Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  fa_status s = check_qk(dtype, B, H, Nq, Nk, d);
  if (s != FA_OK) return s;
  if (block_mask != nullptr) {
    s = check_mask_qk(Nq, Nk);
    if (s != FA_OK) return s;
  }
  const long long tk = (static_cast<long long>(Nk) + 127) / 128;
  if (n_splits < 1 || n_splits > tk) return FA_ERR_INVALID_ARG;
  const long long pairs = ((static_cast<long long>(Nq) + 127) / 128 + 1) / 2;
  if (static_cast<long long>(B) * H * pairs * n_splits > 0x7FFFFFFFLL) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  const fa::SplitWorkspace ws = fa::splitkv_workspace_layout(B, H, Nq, d, n_splits);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  fa::AttnArgs a{};
  a.dtype = dtype;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = Nq;
  a.Nk = Nk;
  a.d = d;
  a.scale = softmax_scale;
  a.causal = causal ? 1 : 0;
  a.block_mask = block_mask;
  a.trace = nullptr;
  a.n_splits = n_splits;
  a.o_part = reinterpret_cast<float*>(base + ws.o_part);
  a.lse_part = reinterpret_cast<float*>(base + ws.lse_part);
  a.status = status_word();
  if (!a.status) return FA_ERR_CUDA;
  // A few query rows (decoding): the ranges' partials on the CUDA cores, which
  // stream K and V once; otherwise the tensor-core forward's split-KV instance.
  const int st = Nq <= fa::kDecodeMaxRows ? fa::launch_decode_splitkv(a, stream) : fa::launch_fwd(a, stream);
  if (st != 0) return FA_ERR_CUDA;
  return fa::launch_splitkv_merge(a, stream) == 0 ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_dropout(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Nq, int Nk, int d, float softmax_scale, int causal, const uint8_t* block_mask,
                         float p_drop, unsigned long long seed, cudaStream_t stream) {
  if (Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  const int t = drop_threshold(p_drop);
  if (t < 0) return FA_ERR_INVALID_ARG;
  if (d == 256 && t > 0) return FA_ERR_UNSUPPORTED;  // dropout has a backward; d = 256 is forward-only
  if (block_mask != nullptr) {
    fa_status s = check_mask_qk(Nq, Nk);
    if (s != FA_OK) return s;
  }
  return fwd_impl(dtype, q, k, v, o, lse, B, H, Nq, d, softmax_scale, causal, block_mask, nullptr, stream, Nk, 0, t,
                  seed);
}

fa_status fa_bwd_dropout(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk,
                         int d, float softmax_scale, int causal, const uint8_t* block_mask, float p_drop,
                         unsigned long long seed, cudaStream_t stream) {
  if (Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  const int t = drop_threshold(p_drop);
  if (t < 0) return FA_ERR_INVALID_ARG;
  if (block_mask != nullptr) {
    fa_status s = check_mask_qk(Nq, Nk);
    if (s != FA_OK) return s;
  }
  return bwd_impl(dtype, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, d, softmax_scale, causal, block_mask,
                  nullptr, stream, 7, Nk, 0, t, seed);
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_scale, float k_scale, float v_scale,
                     void* o, float* lse, int B, int H, int Nq, int Nk, int d, float softmax_scale, int causal,
                     const uint8_t* block_mask, cudaStream_t stream) {
  if (Nq < 1 || Nk < 1 || B < 1 || H < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  fa_status s = check_qk(FA_BF16, B, H, Nq, Nk, d);
  if (s != FA_OK) return s;
  if (block_mask != nullptr) {
    s = check_mask_qk(Nq, Nk);
    if (s != FA_OK) return s;
  }
  if (!(q_scale > 0.0f) || !(k_scale > 0.0f) || !(v_scale > 0.0f) || !std::isfinite(q_scale) ||
      !std::isfinite(k_scale) || !std::isfinite(v_scale))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  fa::AttnArgs a{};
  a.dtype = FA_BF16;
  a.q = q8;
  a.k = k8;
  a.v = v8;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = Nq;
  a.Nk = Nk;
  a.d = d;
  a.scale = softmax_scale;
  a.causal = causal ? 1 : 0;
  a.block_mask = block_mask;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.status = status_word();
  if (!a.status) return FA_ERR_CUDA;
  return fa::launch_fwd_fp8(a, stream) == 0 ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_debug_dropout_draws(int B, int H, int Nq, int Nk, unsigned long long seed, uint8_t* row_major,
                                 uint8_t* col_major, cudaStream_t stream) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || row_major == nullptr || col_major == nullptr) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return FA_ERR_UNSUPPORTED;
  return fa::launch_dropout_draws(B * H, Nq, Nk, seed, row_major, col_major, stream) == 0 ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_debug_fwd_withhold(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int N, int d, float softmax_scale, int causal, int timeout_ms,
                                cudaStream_t stream) {
  if (timeout_ms < 1 || timeout_ms > 5000) return FA_ERR_INVALID_ARG;
  return fwd_impl(dtype, q, k, v, o, lse, B, H, N, d, softmax_scale, causal, nullptr, nullptr, stream, 0,
                  static_cast<uint64_t>(timeout_ms) * 1000000ull);
}

fa_status fa_debug_bwd_withhold(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                                int B, int H, int N, int d, float softmax_scale, int causal, int timeout_ms,
                                cudaStream_t stream) {
  if (timeout_ms < 1 || timeout_ms > 5000) return FA_ERR_INVALID_ARG;
  return bwd_impl(dtype, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, N, d, softmax_scale, causal, nullptr,
                  nullptr, stream, 7, 0, static_cast<uint64_t>(timeout_ms) * 1000000ull);
}

fa_status fa_debug_timeout_probe(int timeout_ms, cudaStream_t stream) {
  if (timeout_ms < 1 || timeout_ms > 5000) return FA_ERR_INVALID_ARG;
  int* w = status_word();
  if (!w) return FA_ERR_CUDA;
  timeout_probe_kernel<<<1, 32, 0, stream>>>(w, static_cast<uint64_t>(timeout_ms) * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
