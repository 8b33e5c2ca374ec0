// Attention backward for sm_100a: recompute P from Q, K and the saved lse
// instead of storing it ("FlashAttention" concept card, lukebest.github.io,
// "反向：重算而非存储"; interview explainer mstx.cn/posts/485, section 3.3).
//
// Three kernels:
//   prep     D_i = rowsum(dO_i o O_i), lse2_i = lse_i * log2(e) (+inf on padding
//            rows and rows without keys, so their P is 0), dQacc = 0.
//   main     one CTA per 128-key tile j of one (batch, head); it loops over the
//            query tiles i that reach j (B_r rows each) and, per tile:
//              S^T  = K_j Q_i^T           P^T = exp2(S^T * scale*log2e - lse2_i)
//              dP^T = V_j dO_i^T          dS^T = P^T o (dP^T - D_i)
//              dV_j += P^T dO_i           dK_j += dS^T Q_i
//              dQ_i (+)= dS K_j           added to fp32 dQacc by a TMA reduce
//            then writes dV_j and scale * dK_j.
//   finish   dQ = scale * dQacc in the input dtype.
//
// Main-kernel roles (512 threads, one CTA per SM):
//   warp 0      TMA producer: K_j, V_j once; Q_i, dO_i, lse2_i, D_i into a 2-stage ring
//   warp 1      MMA issuer and TMEM owner
//   warp 2      builds the query-tile list of a block-sparse CTA
//   warps 4-7   elementwise, query columns [0, B_r/2)   (thread = key row)
//   warps 8-11  elementwise, query columns [B_r/2, B_r)
//   warps 12-15 dQ drain: TMEM -> shared -> cp.reduce.async.bulk.tensor (add) into dQacc
//
// Tile shapes: B_c = 128 keys per CTA. B_r = 128 query rows for d = 64 and 64
// for d = 128, so that the five accumulators fit the 512 TMEM columns:
//   d=64:  S^T 0..127, dP^T 128..255, P^T 256..319, dV 320..383, dK 384..447, dQ 448..511
//   d=128: S^T 0..63,  dP^T 64..127,  P^T 128..159, dV 160..287, dK 288..415, dQ^T 416..479
// For d=128 dQ is produced transposed (dQ^T = K_j^T dS^T, M = d = 128), which
// keeps every MMA at M = 128.
//
// MMA order per tile n (all tcgen05 MMAs of a CTA execute in issue order):
//   wait elementwise(n) -> S^T, dP^T of n+1 -> dV(n), dK(n) -> dQ(n)
// so the elementwise work of tile n+1 overlaps dV, dK, dQ of tile n.
#pragma once

#include <cuda_fp16.h>

#include "sm100.cuh"

namespace fa {
namespace bwd {

using namespace fa::sm100;

constexpr int kBlockN = 128;  // keys per CTA
constexpr int kThreads = 512;
constexpr int kMaxSparseTiles = 4096;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int BR = (D == 64) ? 128 : 64;  // query rows per step
  static constexpr int kColS = 0;
  static constexpr int kColDP = BR;
  static constexpr int kColP = 2 * BR;
  static constexpr int kColDV = 2 * BR + BR / 2;
  static constexpr int kColDK = kColDV + D;
  static constexpr int kColDQ = kColDK + D;
  static_assert(kColDQ + (D == 64 ? D : BR) <= 512, "TMEM budget");

  static constexpr int kKVBytes = kBlockN * D * 2;  // K_j or V_j
  static constexpr int kQBytes = BR * D * 2;        // Q_i or dO_i
  static constexpr int kDSBytes = kBlockN * BR * 2; // dS^T (bf16/fp16)
  static constexpr int kStageVec = BR * 4;          // lse2 or D of one tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffQ = kOffV + kKVBytes;             // [2 stages]
  static constexpr int kOffDO = kOffQ + 2 * kQBytes;         // [2 stages]
  static constexpr int kOffDS = kOffDO + 2 * kQBytes;        // [2 buffers]
  static constexpr int kOffDQ = kOffDS + 2 * kDSBytes;       // fp32 staging BR x D
  static constexpr int kOffL = kOffDQ + BR * D * 4;          // lse2 [2][BR]
  static constexpr int kOffDv = kOffL + 2 * kStageVec;       // D [2][BR]
  static constexpr int kOffBar = kOffDv + 2 * kStageVec;
  // bars: kv_full, qdo_full[2], qdo_empty[2], s_full, p_full, p_free, ds_empty[2], dq_full, dq_empty, all_done
  static constexpr int kNumBars = 13;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;    // tmem slot, abort flag, list length
  static constexpr int kOffList = kOffMisc + 16;
  static constexpr int kBytes = kOffList + 4 * kMaxSparseTiles;
  static constexpr int kAlloc = kBytes + 1024;
};

struct Params {
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* dq_acc;   // [BH][N][d]
  float* delta;    // [BH][Npad]
  float* lse2;     // [BH][Npad]
  const uint8_t* block_mask;
  int32_t* trace;
  int* status;
  int N;
  int Npad;
  int BH;
  int Tq;  // query tiles of B_r rows
  int Tc;  // key tiles of 128
  int causal;
  float scale;
  float scale_log2;
};

// --------------------------------------------------------------------------- prep

// One group of D/8 threads per row: 16-byte loads of O and dO, fp32 dot product.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(Params p) {
  constexpr int kTPR = D / 8;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gt / kTPR;  // over BH * Npad
  const int part = static_cast<int>(gt % kTPR);
  const long long total = static_cast<long long>(p.BH) * p.Npad;
  if (row >= total) return;
  const int bh = static_cast<int>(row / p.Npad);
  const int r = static_cast<int>(row % p.Npad);
  float acc = 0.0f;
  const bool valid = r < p.N;
  if (valid) {
    const size_t off = (static_cast<size_t>(bh) * p.N + r) * D + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.o) + off);
    const uint4 b = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + off);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a0, a1, b0, b1;
      if constexpr (BF16) {
        a0 = __uint_as_float(aw[i] << 16);
        a1 = __uint_as_float(aw[i] & 0xFFFF0000u);
        b0 = __uint_as_float(bw[i] << 16);
        b1 = __uint_as_float(bw[i] & 0xFFFF0000u);
      } else {
        const __half2 ha = *reinterpret_cast<const __half2*>(&aw[i]);
        const __half2 hb = *reinterpret_cast<const __half2*>(&bw[i]);
        const float2 fa = __half22float2(ha);
        const float2 fb = __half22float2(hb);
        a0 = fa.x; a1 = fa.y; b0 = fb.x; b1 = fb.y;
      }
      acc = fmaf(a0, b0, acc);
      acc = fmaf(a1, b1, acc);
    }
    float4* z = reinterpret_cast<float4*>(p.dq_acc + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int m = kTPR / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (part == 0) {
    const size_t vo = static_cast<size_t>(bh) * p.Npad + r;
    float l2 = INFINITY;
    if (valid) {
      const float l = p.lse[static_cast<size_t>(bh) * p.N + r];
      if (l != -INFINITY) l2 = l * kLog2e;
    }
    p.delta[vo] = valid ? acc : 0.0f;
    p.lse2[vo] = l2;
  }
}

// --------------------------------------------------------------------------- finish

template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_finish_kernel(Params p) {
  const long long total4 = static_cast<long long>(p.BH) * p.N * D / 4;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total4;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(p.dq_acc)[t];
    uint2 w;
    w.x = pack2<BF16>(a.x * p.scale, a.y * p.scale);
    w.y = pack2<BF16>(a.z * p.scale, a.w * p.scale);
    reinterpret_cast<uint2*>(p.dq)[t] = w;
  }
}

// --------------------------------------------------------------------------- main

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Query-tile iteration of one key tile: entry n is query tile i(n).
struct QList {
  int len;
  int mode;  // 0 dense, 1 causal (range from start), 2 smem list
  int start;
  const uint32_t* list;
  __device__ __forceinline__ int at(int n) const { return mode == 2 ? static_cast<int>(list[n]) : start + n; }
};

template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_do,
                       const __grid_constant__ CUtensorMap tmap_dq, const Params p) {
  using C = Cfg<D>;
  constexpr int BR = C::BR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* list_len = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::kOffList);
  float* sL = reinterpret_cast<float*>(smem + C::kOffL);
  float* sDv = reinterpret_cast<float*>(smem + C::kOffDv);

  const uint32_t bar_kv_full = smem_u32(&bars[0]);
  auto bar_qdo_full = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto bar_qdo_empty = [&](int s) { return smem_u32(&bars[3 + s]); };
  const uint32_t bar_s_full = smem_u32(&bars[5]);
  const uint32_t bar_p_full = smem_u32(&bars[6]);
  const uint32_t bar_p_free = smem_u32(&bars[7]);
  auto bar_ds_empty = [&](int b) { return smem_u32(&bars[8 + b]); };
  const uint32_t bar_dq_full = smem_u32(&bars[10]);
  const uint32_t bar_dq_empty = smem_u32(&bars[11]);
  const uint32_t bar_all_done = smem_u32(&bars[12]);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // x runs over the key tiles of one head, so the CTAs that share a head's Q, dO
  // and dQ accumulator in L2 run together; small j (most query tiles under a
  // causal mask) goes first.
  const int bh = blockIdx.y;
  const int j = blockIdx.x;
  const int cta = bh * p.Tc + j;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar_kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_qdo_full(s), 1);
      mbar_init(bar_qdo_empty(s), 1);
      mbar_init(bar_ds_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_p_full, 256);
    mbar_init(bar_p_free, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 128);
    mbar_init(bar_all_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 2 && p.block_mask != nullptr) {
    // Query tiles i whose mask row (i*B_r/128) has column j set, with the causal
    // valid-tile rule j*128 <= i*B_r + B_r - 1 applied by AND; ascending i.
    int count = 0;
    for (int base = 0; base < p.Tq; base += 32) {
      const int i = base + lane;
      bool use = false;
      if (i < p.Tq) {
        use = p.block_mask[static_cast<size_t>((i * BR) / 128) * p.Tc + j] != 0;
        if (p.causal && j * kBlockN > i * BR + BR - 1) use = false;
      }
      const uint32_t ballot = __ballot_sync(0xffffffffu, use);
      if (use) {
        const int pos = count + __popc(ballot & ((1u << lane) - 1u));
        if (pos < kMaxSparseTiles) list[pos] = static_cast<uint32_t>(i);
      }
      count += __popc(ballot);
    }
    if (lane == 0) *list_len = count < kMaxSparseTiles ? count : kMaxSparseTiles;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = *tmem_slot;
  WaitCtx ctx{abort_flag, p.status};

  QList ql;
  ql.list = list;
  if (p.block_mask != nullptr) {
    ql.mode = 2;
    ql.start = 0;
    ql.len = *list_len;
  } else if (p.causal) {
    ql.mode = 1;
    ql.start = (j * kBlockN) / BR;
    ql.len = p.Tq > ql.start ? p.Tq - ql.start : 0;
  } else {
    ql.mode = 0;
    ql.start = 0;
    ql.len = p.Tq;
  }

  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sDS = smem + C::kOffDS;
  float* sDQ = reinterpret_cast<float*>(smem + C::kOffDQ);
  constexpr int kKVChunk = kBlockN * 128;  // 64 columns x 128 key rows
  constexpr int kQChunk = BR * 128;        // 64 columns x B_r query rows

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      if (p.trace) {
        int32_t* t = p.trace + static_cast<size_t>(cta) * (p.Tq + 1);
        t[0] = ql.len;
        for (int n = 0; n < ql.len; ++n) t[1 + n] = ql.at(n) | (1 << 16);
      }
      if (ql.len > 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        prefetch_tmap(&tmap_do);
        mbar_arrive_expect_tx(bar_kv_full, 2 * C::kKVBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem_u32(sK + c * kKVChunk), &tmap_k, bar_kv_full, c * 64, j * kBlockN, bh);
          tma_load_3d(smem_u32(sV + c * kKVChunk), &tmap_v, bar_kv_full, c * 64, j * kBlockN, bh);
        }
        for (int n = 0; n < ql.len; ++n) {
          const int i = ql.at(n);
          const int s = n & 1;
          if (!mbar_wait(bar_qdo_empty(s), ((n >> 1) & 1) ^ 1, ctx)) break;
          const uint32_t bar = bar_qdo_full(s);
          mbar_arrive_expect_tx(bar, 2 * C::kQBytes + 2 * C::kStageVec);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(smem_u32(sQ + s * C::kQBytes + c * kQChunk), &tmap_q, bar, c * 64, i * BR, bh);
            tma_load_3d(smem_u32(sDO + s * C::kQBytes + c * kQChunk), &tmap_do, bar, c * 64, i * BR, bh);
          }
          const size_t vo = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(i) * BR;
          bulk_load(smem_u32(sL + s * BR), p.lse2 + vo, C::kStageVec, bar);
          bulk_load(smem_u32(sDv + s * BR), p.delta + vo, C::kStageVec, bar);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ql.len > 0) {
      constexpr uint32_t idesc_sp = idesc_f16(BF16, 128, BR, false, false);  // S^T, dP^T
      constexpr uint32_t idesc_kv = idesc_f16(BF16, 128, D, false, true);    // dV, dK
      constexpr uint32_t idesc_q = idesc_f16(BF16, 128, D == 64 ? D : BR, true, true);  // dQ / dQ^T

      auto issue_sdp = [&](int n) {
        const int s = n & 1;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int kk = k * 16;
          const uint32_t okv = (kk / 64) * kKVChunk + (kk % 64) * 2;
          const uint32_t oq = (kk / 64) * kQChunk + (kk % 64) * 2;
          umma_ss(tmem + C::kColS, sdesc_sw128(smem_u32(sK + okv), 16, 1024),
                  sdesc_sw128(smem_u32(sQ + s * C::kQBytes + oq), 16, 1024), idesc_sp, k > 0);
        }
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int kk = k * 16;
          const uint32_t okv = (kk / 64) * kKVChunk + (kk % 64) * 2;
          const uint32_t oq = (kk / 64) * kQChunk + (kk % 64) * 2;
          umma_ss(tmem + C::kColDP, sdesc_sw128(smem_u32(sV + okv), 16, 1024),
                  sdesc_sw128(smem_u32(sDO + s * C::kQBytes + oq), 16, 1024), idesc_sp, k > 0);
        }
        umma_commit(bar_s_full);
      };

      bool ok = mbar_wait(bar_kv_full, 0, ctx) && mbar_wait(bar_qdo_full(0), 0, ctx);
      if (ok) {
        tc_fence_after();
        issue_sdp(0);
      }
      for (int n = 0; ok && n < ql.len; ++n) {
        const int s = n & 1;
        const int b = n & 1;
        if (!(ok = mbar_wait(bar_p_full, n & 1, ctx))) break;
        tc_fence_after();
        if (n + 1 < ql.len) {
          if (!(ok = mbar_wait(bar_qdo_full((n + 1) & 1), ((n + 1) >> 1) & 1, ctx))) break;
          tc_fence_after();
          issue_sdp(n + 1);
        }
        const uint32_t acc = n > 0 ? 1u : 0u;
        // dV += P^T dO_i   (A: P^T in TMEM; B: dO_i, d contiguous)
#pragma unroll
        for (int k = 0; k < BR / 16; ++k) {
          const int kk = k * 16;
          umma_ts(tmem + C::kColDV, tmem + C::kColP + kk / 2,
                  sdesc_sw128(smem_u32(sDO + s * C::kQBytes + kk * 128), kQChunk, 1024), idesc_kv,
                  acc | static_cast<uint32_t>(k > 0));
        }
        umma_commit(bar_p_free);
        // dK += dS^T Q_i   (A: dS^T in smem, query columns contiguous; B: Q_i, d contiguous)
#pragma unroll
        for (int k = 0; k < BR / 16; ++k) {
          const int kk = k * 16;
          const uint32_t oa = (kk / 64) * (kBlockN * 128) + (kk % 64) * 2;
          umma_ss(tmem + C::kColDK, sdesc_sw128(smem_u32(sDS + b * C::kDSBytes + oa), 16, 1024),
                  sdesc_sw128(smem_u32(sQ + s * C::kQBytes + kk * 128), kQChunk, 1024), idesc_kv,
                  acc | static_cast<uint32_t>(k > 0));
        }
        if (!(ok = mbar_wait(bar_dq_empty, (n & 1) ^ 1, ctx))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kBlockN / 16; ++k) {
          const int kk = k * 16;
          if constexpr (D == 64) {
            // dQ = dS K_j: A = dS (query rows contiguous in smem), B = K_j (d contiguous)
            umma_ss(tmem + C::kColDQ, sdesc_sw128(smem_u32(sDS + b * C::kDSBytes + kk * 128), kBlockN * 128, 1024),
                    sdesc_sw128(smem_u32(sK + kk * 128), kKVChunk, 1024), idesc_q, k > 0);
          } else {
            // dQ^T = K_j^T dS^T: A = K_j^T (d contiguous), B = dS^T (query columns contiguous)
            umma_ss(tmem + C::kColDQ, sdesc_sw128(smem_u32(sK + kk * 128), kKVChunk, 1024),
                    sdesc_sw128(smem_u32(sDS + b * C::kDSBytes + kk * 128), kBlockN * 128, 1024), idesc_q,
                    k > 0);
          }
        }
        umma_commit(bar_dq_full);
        umma_commit(bar_ds_empty(b));
        umma_commit(bar_qdo_empty(s));
      }
      if (ok) umma_commit(bar_all_done);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ elementwise (thread = key row)
    const int half = (warp - 4) / 4;  // which half of the query columns
    const int wq = warp % 4;
    const int r = wq * 32 + lane;      // key row within the tile
    const int key = j * kBlockN + r;
    const bool key_valid = key < p.N;  // rows past N were zero-filled; keep their P at 0
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int n = 0; ok && n < ql.len; ++n) {
      const int i = ql.at(n);
      const int s = n & 1;
      const int b = n & 1;
      if (!(ok = mbar_wait_warp(bar_s_full, n & 1, ctx))) break;
      // lse2 and D of this tile arrived with Q_i (same barrier phase as the S^T inputs).
      if (!(ok = mbar_wait_warp(bar_qdo_full(s), (n >> 1) & 1, ctx))) break;
      tc_fence_after();
      const bool diag = p.causal && (j * kBlockN + kBlockN - 1 > i * BR);
      const uint32_t aL = smem_u32(sL + s * BR);
      const uint32_t aD = smem_u32(sDv + s * BR);
#pragma unroll
      for (int cc = 0; cc < BR / 64; ++cc) {
        const int qo = half * (BR / 2) + cc * 32;  // first query column of this chunk
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_off + C::kColS + qo, sr);
        tmem_ld32(tmem + lane_off + C::kColDP + qo, dr);
        tmem_ld_wait();
        // Columns x < lim are masked (causal: key > query; or the key row is past N).
        int lim = 0;
        if (!key_valid) lim = 32;
        else if (diag) lim = min(32, max(0, key - (i * BR + qo)));
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const float4 l4 = lds128(aL + (qo + x) * 4);
          const float4 d4 = lds128(aD + (qo + x) * 4);
          float p0 = ex2(fmaf(__uint_as_float(sr[x]), sl2, -l4.x));
          float p1 = ex2(fmaf(__uint_as_float(sr[x + 1]), sl2, -l4.y));
          float p2 = ex2(fmaf(__uint_as_float(sr[x + 2]), sl2, -l4.z));
          float p3 = ex2(fmaf(__uint_as_float(sr[x + 3]), sl2, -l4.w));
          if (lim > 0) {
            if (x < lim) p0 = 0.0f;
            if (x + 1 < lim) p1 = 0.0f;
            if (x + 2 < lim) p2 = 0.0f;
            if (x + 3 < lim) p3 = 0.0f;
          }
          pk[x / 2] = pack2<BF16>(p0, p1);
          pk[x / 2 + 1] = pack2<BF16>(p2, p3);
          dk[x / 2] = pack2<BF16>(p0 * (__uint_as_float(dr[x]) - d4.x), p1 * (__uint_as_float(dr[x + 1]) - d4.y));
          dk[x / 2 + 1] = pack2<BF16>(p2 * (__uint_as_float(dr[x + 2]) - d4.z), p3 * (__uint_as_float(dr[x + 3]) - d4.w));
        }
        if (cc == 0 && n > 0) {
          // P^T of the previous tile must have been consumed by its dV MMA.
          if (!(ok = mbar_wait_warp(bar_p_free, (n - 1) & 1, ctx))) break;
        }
        tmem_st16(tmem + lane_off + C::kColP + qo / 2, pk);
        if (cc == 0 && n >= 2) {
          if (!(ok = mbar_wait_warp(bar_ds_empty(b), ((n - 2) >> 1) & 1, ctx))) break;
        }
        // dS^T row r, query columns qo..qo+31 -> four 16-byte pieces of the swizzled row.
        const uint32_t rowa = smem_u32(sDS + b * C::kDSBytes + (qo / 64) * (kBlockN * 128) + r * 128);
        const int p0i = (qo % 64) / 8;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int phys = (p0i + t) ^ (r & 7);
          sts128(rowa + phys * 16, dk[4 * t], dk[4 * t + 1], dk[4 * t + 2], dk[4 * t + 3]);
        }
      }
      if (!ok) break;
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p_full);
    }
    // Epilogue: half 0 writes dV_j, half 1 writes scale * dK_j.
    bool have = false;
    if (ok && ql.len > 0) {
      ok = mbar_wait_warp(bar_all_done, 0, ctx);
      have = ok;
    }
    tc_fence_after();
    if (ok) {
      const uint32_t col = half == 0 ? C::kColDV : C::kColDK;
      const float mul = half == 0 ? 1.0f : p.scale;
      uint16_t* dst = reinterpret_cast<uint16_t*>(half == 0 ? p.dv : p.dk);
      const bool valid = key < p.N;
      uint16_t* rowp = dst + (static_cast<size_t>(bh) * p.N + (valid ? key : 0)) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t v[32];
        if (have) {
          tmem_ld32(tmem + lane_off + col + c, v);
          tmem_ld_wait();
        }
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x)
          w[x] = have ? pack2<BF16>(__uint_as_float(v[2 * x]) * mul, __uint_as_float(v[2 * x + 1]) * mul) : 0u;
        if (valid) {
          uint4* o4 = reinterpret_cast<uint4*>(rowp + c);
          o4[0] = make_uint4(w[0], w[1], w[2], w[3]);
          o4[1] = make_uint4(w[4], w[5], w[6], w[7]);
          o4[2] = make_uint4(w[8], w[9], w[10], w[11]);
          o4[3] = make_uint4(w[12], w[13], w[14], w[15]);
        }
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ dQ drain
    const int wq = warp % 4;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const bool leader = (warp == 12 && lane == 0);
    bool ok = true;
    for (int n = 0; ok && n < ql.len; ++n) {
      const int i = ql.at(n);
      if (!(ok = mbar_wait_warp(bar_dq_full, n & 1, ctx))) break;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld32(tmem + lane_off + C::kColDQ, v0);
      tmem_ld32(tmem + lane_off + C::kColDQ + 32, v1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar_dq_empty);
      if (leader) bulk_wait_group_read<0>();  // the previous reduce has read the staging tile
      named_barrier(1, 128);
      const int t = wq * 32 + lane;  // TMEM lane
      if constexpr (D == 64) {
        // lane = query row. Staging is two [128 rows][32] fp32 boxes in the TMA
        // 128-byte swizzle: 16-byte piece x of row t sits at piece x ^ (t & 7).
        const uint32_t row0 = smem_u32(sDQ) + t * 128;
        const uint32_t row1 = row0 + 128 * 128;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const int phys = (x ^ (t & 7)) * 16;
          sts128(row0 + phys, v0[4 * x], v0[4 * x + 1], v0[4 * x + 2], v0[4 * x + 3]);
          sts128(row1 + phys, v1[4 * x], v1[4 * x + 1], v1[4 * x + 2], v1[4 * x + 3]);
        }
      } else {
        // lane = d index; columns are the 64 query rows; staging is [64 rows][128] fp32.
        const uint32_t base = smem_u32(sDQ) + t * 4;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          sts32(base + x * D * 4, v0[x]);
          sts32(base + (x + 32) * D * 4, v1[x]);
        }
      }
      fence_proxy_async_smem();
      named_barrier(1, 128);
      if (leader) {
        if constexpr (D == 64) {
          tma_reduce_add_3d(&tmap_dq, smem_u32(sDQ), 0, i * BR, bh);
          tma_reduce_add_3d(&tmap_dq, smem_u32(sDQ) + 128 * 128, 32, i * BR, bh);
        } else {
          tma_reduce_add_3d(&tmap_dq, smem_u32(sDQ), 0, i * BR, bh);
        }
        bulk_commit_group();
      }
    }
    if (leader) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd
}  // namespace fa
