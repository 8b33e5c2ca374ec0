// fa_bwd_noalloc: the backward for callers that cannot allocate device memory.
//
// fa_bwd needs a device workspace (two fp32 row vectors: D = rowsum(dO o O) and
// lse in log2 units). Some callers have no way to provide one: a host
// application that plans every byte of device memory up front and gives plugins
// no allocator, or a latency-critical loop in which cudaMalloc (which may
// synchronise the device and may fail) is not allowed. For them this entry point
// keeps that workspace in a fixed array in the library's own static device
// memory, so no call allocates anything.
//
// Limits and sharing:
//   * The array holds FA_BWD_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads
//     the library, for the life of the process. Problems whose workspace
//     (fa_bwd_workspace_size) is larger are rejected with FA_ERR_UNSUPPORTED
//     before anything is launched; every other limit is that of fa_bwd.
//   * Every call on a device uses the same array. Calls whose kernels overlap
//     on the GPU (different streams without ordering between them) race on it
//     and give wrong gradients; callers must order such calls. Nothing in the
//     array has to start at zero: each call's first kernel rewrites every entry
//     its second kernel reads, so what the previous call left does not matter.
//   * The first call on a device looks up the array's device address with
//     cudaGetSymbolAddress (a host-side stand-in name is not a device address)
//     and caches it; that first call should come before any stream capture.
#include "fa.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fa_internal.h"

namespace {

static __device__ __align__(256) uint8_t g_bwd_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device (set up once per device).
uint8_t* scratch_on_current_device(cudaError_t* err) {
  static std::mutex mu;
  static uint8_t* ptrs[128] = {nullptr};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 128) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<uint8_t*>(p);
  }
  return ptrs[dev];
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" fa_status fa_bwd_noalloc(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                                    const float* lse, const void* dout, void* dq, void* dk, void* dv, int B, int H,
                                    int N, int d, float softmax_scale, int causal, cudaStream_t stream) {
  // The same limits as fa_bwd, then the size of the static array.
  const fa_status st = fa::check_common(dtype, B, H, N, d);
  if (st != FA_OK) return st;
  if (!fa::bwd_head_dim_supported(d)) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  const fa::BwdWorkspace ws = fa::bwd_workspace_layout(B, H, N, d);
  if (ws.total > static_cast<size_t>(FA_BWD_NOALLOC_SCRATCH_BYTES)) return FA_ERR_UNSUPPORTED;

  cudaError_t err = cudaSuccess;
  uint8_t* scratch = scratch_on_current_device(&err);
  if (scratch == nullptr || err != cudaSuccess) return FA_ERR_CUDA;

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
  a.workspace = scratch;
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.scale = softmax_scale;
  a.causal = causal ? 1 : 0;
  a.block_mask = nullptr;
  a.trace = nullptr;
  a.status = fa::device_status_word();
  if (a.status == nullptr) return FA_ERR_CUDA;
  return fa::launch_bwd(a, stream) == 0 ? FA_OK : FA_ERR_CUDA;
}
