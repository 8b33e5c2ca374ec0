// Split-KV forward, second step: merge the partial results of the key ranges.
//
// The forward kernel, run with n_splits key ranges, leaves for every query row
// and range s an fp32 O_s (the softmax-weighted mean of that range's values) and
// lse_s (the log of that range's exp-sum). The whole row is
//   lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) * O_s,
// the online-softmax update ("FlashAttention" interview explainer,
// mstx.cn/posts/485, section 3.2) applied to whole ranges at once, as
// FlashDecoding does (the "FlashAttention" concept card's lineage table). A
// range without an allowed key for the row has lse_s = -inf and weight 0.
//
// HBM bound: one warp per row reads its n_splits lse values and partial rows
// (coalesced 128-byte loads) and writes the row once in the tensor's type.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kMergeThreads = 256;

template <bool BF16>
__global__ void __launch_bounds__(kMergeThreads) fa_splitkv_merge_kernel(const float* __restrict__ o_part,
                                                                        const float* __restrict__ lse_part,
                                                                        void* __restrict__ o, float* __restrict__ lse,
                                                                        long long rows, int d, int n_splits) {
  const long long row = (static_cast<long long>(blockIdx.x) * kMergeThreads + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  // Largest partial lse, then the sum of exp(lse_s - max): lanes over ranges.
  float m = -INFINITY;
  for (int s = lane; s < n_splits; s += 32) m = fmaxf(m, lse_part[s * rows + row]);
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
  float z = 0.0f;
  if (m != -INFINITY) {
    for (int s = lane; s < n_splits; s += 32) {
      const float l = lse_part[s * rows + row];
      if (l != -INFINITY) z += expf(l - m);
    }
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) z += __shfl_xor_sync(0xffffffffu, z, k);
  // Weighted sum of the partial rows: lanes over columns (d <= 256).
  float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  if (z > 0.0f) {
    const float inv_z = 1.0f / z;
    for (int s = 0; s < n_splits; ++s) {
      const float l = lse_part[s * rows + row];
      if (l == -INFINITY) continue;
      const float w = expf(l - m) * inv_z;
      const float* src = o_part + (s * rows + row) * d;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int c = lane + 32 * k;
        if (c < d) acc[k] = fmaf(w, src[c], acc[k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int c = lane + 32 * k;
    if (c < d) {
      if constexpr (BF16) {
        reinterpret_cast<__nv_bfloat16*>(o)[row * d + c] = __float2bfloat16_rn(acc[k]);
      } else {
        reinterpret_cast<__half*>(o)[row * d + c] = __float2half_rn(acc[k]);
      }
    }
  }
  if (lane == 0) lse[row] = z > 0.0f ? m + logf(z) : -INFINITY;
}

}  // namespace

SplitWorkspace splitkv_workspace_layout(int B, int H, int Nq, int d, int n_splits) {
  SplitWorkspace w{};
  const size_t rows = static_cast<size_t>(B) * H * Nq;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  w.o_part = 0;
  w.lse_part = up(static_cast<size_t>(n_splits) * rows * d * 4);
  w.total = w.lse_part + up(static_cast<size_t>(n_splits) * rows * 4);
  return w;
}

int launch_splitkv_merge(const AttnArgs& a, cudaStream_t stream) {
  const long long rows = static_cast<long long>(a.B) * a.H * a.N;
  const long long blocks = (rows * 32 + kMergeThreads - 1) / kMergeThreads;
  void* o = const_cast<void*>(a.o);
  if (a.dtype == 1)
    fa_splitkv_merge_kernel<true><<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(
        a.o_part, a.lse_part, o, a.lse, rows, a.d, a.n_splits);
  else
    fa_splitkv_merge_kernel<false><<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(
        a.o_part, a.lse_part, o, a.lse, rows, a.d, a.n_splits);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace fa
