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
// HBM bound: one block per row reads its n_splits lse values and partial rows
// (each range's row in coalesced loads) and writes the row once in the tensor's
// type.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kMergeThreads = 256;

// One block per row. Step 1, threads over ranges: the largest partial lse m
// and z = sum_s exp(lse_s - m). Step 2, thread t takes column t % d of ranges
// s = t / d, t / d + G, ... (G = 256 / d groups), so the loads of different
// ranges are in flight together; the groups' sums meet in shared memory.
template <bool BF16>
__global__ void __launch_bounds__(kMergeThreads) fa_splitkv_merge_kernel(const float* __restrict__ o_part,
                                                                        const float* __restrict__ lse_part,
                                                                        void* __restrict__ o, float* __restrict__ lse,
                                                                        long long rows, int d, int n_splits) {
  __shared__ float red[kMergeThreads];
  __shared__ float stat[2];
  const long long row = blockIdx.x;
  const int t = threadIdx.x, lane = t % 32, warp = t / 32;
  float m = -INFINITY;
  for (int s = t; s < n_splits; s += kMergeThreads) m = fmaxf(m, lse_part[s * rows + row]);
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (t == 0) {
    float mm = red[0];
    for (int w = 1; w < kMergeThreads / 32; ++w) mm = fmaxf(mm, red[w]);
    stat[0] = mm;
  }
  __syncthreads();
  m = stat[0];
  float z = 0.0f;
  if (m != -INFINITY) {
    for (int s = t; s < n_splits; s += kMergeThreads) {
      const float l = lse_part[s * rows + row];
      if (l != -INFINITY) z += expf(l - m);
    }
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) z += __shfl_xor_sync(0xffffffffu, z, k);
  __syncthreads();
  if (lane == 0) red[warp] = z;
  __syncthreads();
  if (t == 0) {
    float zz = 0.0f;
    for (int w = 0; w < kMergeThreads / 32; ++w) zz += red[w];
    stat[1] = zz;
  }
  __syncthreads();
  z = stat[1];
  const int groups = kMergeThreads / d;  // d <= 256
  const int c = t % d, g = t / d;
  float acc = 0.0f;
  if (g < groups && z > 0.0f) {
#pragma unroll 4
    for (int s = g; s < n_splits; s += groups) {
      const float l = lse_part[s * rows + row];
      const float x = o_part[(s * rows + row) * d + c];
      if (l != -INFINITY) acc = fmaf(expf(l - m), x, acc);
    }
  }
  red[t] = acc;
  __syncthreads();
  if (t < d) {
    float sum = 0.0f;
    for (int k = 0; k < groups; ++k) sum += red[k * d + t];
    const float out = z > 0.0f ? sum / z : 0.0f;
    if constexpr (BF16) {
      reinterpret_cast<__nv_bfloat16*>(o)[row * d + t] = __float2bfloat16_rn(out);
    } else {
      reinterpret_cast<__half*>(o)[row * d + t] = __float2half_rn(out);
    }
  }
  if (t == 0) lse[row] = z > 0.0f ? m + logf(z) : -INFINITY;
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
  const long long blocks = rows;  // one block per row
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
