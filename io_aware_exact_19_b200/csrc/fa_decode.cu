// Split-KV step 1 for decoding (a few query rows against a long key sequence) on
// the CUDA cores. With N_q <= 4 the scores of a key range are a matrix-vector
// product: the work is bound by reading K and V from HBM once, and a 128-row
// tensor-core tile would be almost all padding. Each CTA takes one key range of
// one head (the same ranges of whole 128-key tiles as the tensor-core path) and
// writes that range's partial (O_s, lse_s); the merge kernel combines the ranges
// ("FlashAttention" concept card, lineage table, FlashDecoding; the update of the
// interview explainer, section 3.2, applied to groups of keys and to ranges).
//
// Threads: d/8 per key row (16 bytes = 8 elements of K and of V each), so a CTA
// of 256 threads works on G = 2048/d keys at a time; thread group g takes keys
// g, g + G, g + 2G, ... of the range and keeps its own running maximum, sum and
// O (its 8 columns) for each query row, rescaled only when the maximum grows by
// more than 2^8 (exact in exact arithmetic). The groups are merged once, at the
// end, through shared memory. Each thread streams its own pieces of K and V
// through a private three-stage ring in shared memory with cp.async (zero-filled
// past the range), so 96 KB per CTA are in flight without holding registers and
// no thread waits for another until the merge.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "fa_internal.h"
#include "tma_host.h"

namespace fa {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecUnroll = 4;  // keys per thread group and ring stage
constexpr int kDecStages = 3;  // ring stages of cp.async copies in flight
constexpr int kDecSmem = kDecStages * kDecUnroll * 2 * kDecThreads * 16;  // 96 KB
constexpr float kDecRescale = 8.0f;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, uint32_t bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

struct DecodeParams {
  const uint16_t* q;  // [BH][Nq][d]
  const uint16_t* k;  // [BH][Nk][d]
  const uint16_t* v;
  float* o_part;      // [n_splits][BH][Nq][d]
  float* lse_part;    // [n_splits][BH][Nq]
  int BH, Nq, Nk, d, Tc, n_splits, causal;
  float scale_log2;
};

template <bool BF16>
__device__ __forceinline__ void widen8(const uint4& w, float (&x)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (BF16) {
      x[2 * i] = __uint_as_float(u[i] << 16);
      x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
}

template <int D, bool BF16, int NQ>
__global__ void __launch_bounds__(kDecThreads, 2) fa_decode_split_kernel(const DecodeParams p) {
  constexpr int kTpr = D / 8;                  // threads per key row
  constexpr int kG = kDecThreads / kTpr;       // key groups per CTA
  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int ci = tid % kTpr;                   // columns 8ci .. 8ci + 7
  const int g = tid / kTpr;
  const bool cols = 8 * ci < p.d;              // a padded head dimension's columns are not loaded
  const int t0 = static_cast<int>(static_cast<long long>(split) * p.Tc / p.n_splits);
  const int t1 = static_cast<int>(static_cast<long long>(split + 1) * p.Tc / p.n_splits);

  // Query rows, pre-scaled by scale * log2(e), in registers (8 columns each).
  float qv[NQ][8];
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    uint4 w = make_uint4(0, 0, 0, 0);
    if (i < p.Nq && cols) w = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(bh) * p.Nq + i) * p.d + 8 * ci);
    widen8<BF16>(w, qv[i]);
#pragma unroll
    for (int c = 0; c < 8; ++c) qv[i][c] *= p.scale_log2;
  }
  float m[NQ], l[NQ], acc[NQ][8];
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.0f;
  }
  const size_t kv_head = static_cast<size_t>(bh) * p.Nk;
  const int shift = p.Nk - p.Nq;  // bottom-right causal: row i sees keys <= i + shift

  // Keys [kbeg, kend) of this range in chunks of kG * kDecUnroll; chunk c, key u
  // of thread group g is key kbeg + c * kChunk + u * kG + g. (Block masks need
  // N_q to be a multiple of 128, so they never reach this kernel.)
  extern __shared__ uint4 ring[];  // [stage][u][K, V][thread]
  constexpr int kChunk = kG * kDecUnroll;
  const int kbeg = 128 * t0;
  const int kend = min(128 * t1, p.Nk);
  const int nc = kend > kbeg ? (kend - kbeg + kChunk - 1) / kChunk : 0;
  auto issue = [&](int c) {
    const int stage = c % kDecStages;
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
      const int key = kbeg + c * kChunk + u * kG + g;
      const bool valid = key < kend && cols;
      const size_t off = valid ? (kv_head + key) * p.d + 8 * ci : 0;
      uint4* slot = ring + ((stage * kDecUnroll + u) * 2) * kDecThreads + tid;
      cp_async16(slot, p.k + off, valid ? 16u : 0u);
      cp_async16(slot + kDecThreads, p.v + off, valid ? 16u : 0u);
    }
  };
#pragma unroll
  for (int c = 0; c < kDecStages - 1; ++c) {
    if (c < nc) issue(c);
    cp_async_commit();
  }
  for (int c = 0; c < nc; ++c) {
    if (c + kDecStages - 1 < nc) issue(c + kDecStages - 1);
    cp_async_commit();
    cp_async_wait<kDecStages - 1>();  // this thread's copies of chunk c have landed
    const int stage = c % kDecStages;
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
      const int key = kbeg + c * kChunk + u * kG + g;
      const uint4* slot = ring + ((stage * kDecUnroll + u) * 2) * kDecThreads + tid;
      float kx[8], vx[8];
      widen8<BF16>(slot[0], kx);
      widen8<BF16>(slot[kDecThreads], vx);
#pragma unroll
      for (int i = 0; i < NQ; ++i) {
        float s = 0.0f;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) s = fmaf(qv[i][cc], kx[cc], s);
        // Every thread runs the same iterations: the shuffles take the whole warp,
        // which holds several key groups; keys past the range are masked below.
#pragma unroll
        for (int o = kTpr / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const bool allowed = key < kend && i < p.Nq && (!p.causal || key <= i + shift);
        if (!allowed) continue;
        if (s > m[i] + kDecRescale || m[i] == -INFINITY) {
          const float alpha = (m[i] == -INFINITY) ? 0.0f : exp2f(m[i] - s);
          l[i] *= alpha;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) acc[i][cc] *= alpha;
          m[i] = s;
        }
        const float pr = exp2f(s - m[i]);
        l[i] += pr;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) acc[i][cc] = fmaf(pr, vx[cc], acc[i][cc]);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();  // the ring is reused for the merge below

  // Merge the kG groups: the largest maximum per row, then the rescaled sums.
  float(*sm_m)[kG] = reinterpret_cast<float(*)[kG]>(ring);
  float(*sm_l)[kG] = sm_m + NQ;
  float(*sm_o)[kG][D] = reinterpret_cast<float(*)[kG][D]>(sm_l + NQ);
  float* sm_mx = reinterpret_cast<float*>(sm_o + NQ);
  if (ci == 0) {
#pragma unroll
    for (int i = 0; i < NQ; ++i) sm_m[i][g] = m[i];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    float mx = -INFINITY;
    for (int gg = 0; gg < kG; ++gg) mx = fmaxf(mx, sm_m[i][gg]);
    const float w = (m[i] == -INFINITY) ? 0.0f : exp2f(m[i] - mx);
    if (ci == 0) sm_l[i][g] = l[i] * w;
#pragma unroll
    for (int c = 0; c < 8; ++c) sm_o[i][g][8 * ci + c] = acc[i][c] * w;
    if (tid == 0) sm_mx[i] = mx;
  }
  __syncthreads();
  // 256 threads over NQ x D outputs.
  for (int idx = tid; idx < NQ * D; idx += kDecThreads) {
    const int i = idx / D, c = idx % D;
    if (i >= p.Nq || c >= p.d) continue;
    float ls = 0.0f, os = 0.0f;
    for (int gg = 0; gg < kG; ++gg) {
      ls += sm_l[i][gg];
      os += sm_o[i][gg][c];
    }
    const size_t row = (static_cast<size_t>(split) * p.BH + bh) * p.Nq + i;
    p.o_part[row * p.d + c] = ls > 0.0f ? os / ls : 0.0f;
    if (c == 0) p.lse_part[row] = ls > 0.0f ? (sm_mx[i] + log2f(ls)) * 0.6931471805599453f : -INFINITY;
  }
}

template <int D, bool BF16, int NQ>
int launch_decode_q(const DecodeParams& p, cudaStream_t stream) {
  // The merge arrays reuse the ring; both fit in kDecSmem.
  static_assert((2 * NQ * (kDecThreads / (D / 8)) + NQ * (kDecThreads / (D / 8)) * D + NQ) * 4 <= kDecSmem,
                "merge arrays exceed the ring");
  auto kern = fa_decode_split_kernel<D, BF16, NQ>;
  const cudaError_t e = host::ensure_dynamic_smem(reinterpret_cast<const void*>(kern), kDecSmem);
  if (e != cudaSuccess) return static_cast<int>(e);
  dim3 grid(static_cast<unsigned>(p.n_splits), static_cast<unsigned>(p.BH));
  kern<<<grid, kDecThreads, kDecSmem, stream>>>(p);
  return static_cast<int>(cudaGetLastError());
}

template <int D, bool BF16>
int launch_decode_t(const DecodeParams& p, cudaStream_t stream) {
  if (p.Nq == 1) return launch_decode_q<D, BF16, 1>(p, stream);
  if (p.Nq == 2) return launch_decode_q<D, BF16, 2>(p, stream);
  return launch_decode_q<D, BF16, 4>(p, stream);
}

}  // namespace

int launch_decode_splitkv(const AttnArgs& a, cudaStream_t stream) {
  DecodeParams p{};
  p.q = static_cast<const uint16_t*>(a.q);
  p.k = static_cast<const uint16_t*>(a.k);
  p.v = static_cast<const uint16_t*>(a.v);
  p.o_part = a.o_part;
  p.lse_part = a.lse_part;
  p.BH = a.B * a.H;
  p.Nq = a.N;
  p.Nk = a.Nk;
  p.d = a.d;
  p.Tc = (a.Nk + 127) / 128;
  p.n_splits = a.n_splits;
  p.causal = a.causal;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const bool bf16 = a.dtype == 1;
  if (a.d <= 64) return bf16 ? launch_decode_t<64, true>(p, stream) : launch_decode_t<64, false>(p, stream);
  if (a.d <= 128) return bf16 ? launch_decode_t<128, true>(p, stream) : launch_decode_t<128, false>(p, stream);
  return bf16 ? launch_decode_t<256, true>(p, stream) : launch_decode_t<256, false>(p, stream);
}

}  // namespace fa
