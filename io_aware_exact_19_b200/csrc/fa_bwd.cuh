// Attention backward for sm_100a: recompute P from Q, K and the saved lse
// instead of storing it ("FlashAttention" concept card, lukebest.github.io,
// "反向：重算而非存储"; interview explainer mstx.cn/posts/485, section 3.3).
//
// Two kernels:
//   prep   D_i = rowsum(dO_i o O_i) and lse2_i = lse_i * log2(e) (+inf on padding
//          rows and rows without keys, so their P is 0).
//   main   one launch with two kinds of CTA, interleaved heaviest first:
//     key-stationary (one 128-key tile j of one head; dK_j and dV_j stay in TMEM)
//       for each 128-row query tile i that reaches j:
//         S^T  = K_j Q_i^T,  dP^T = V_j dO_i^T
//         P^T  = exp2(S^T * scale*log2e - lse2_i),  dS^T = P^T o (dP^T - D_i)
//         dV_j += P^T dO_i,  dK_j += dS^T Q_i         (P^T, dS^T read from TMEM)
//       then dV_j and scale * dK_j are written once.
//     query-stationary (one 128-row query tile i of one head; dQ_i stays in TMEM)
//       for each 128-key tile j that i reaches:
//         S = Q_i K_j^T,  dP = dO_i V_j^T               (Q_i, dO_i read from TMEM)
//         P = exp2(S*scale*log2e - lse2),  dS = P o (dP - D)
//         dQ_i += dS K_j                                (dS read from TMEM)
//       then scale * dQ_i is written once.
// dQ is thus produced without atomics or an fp32 accumulator in global memory,
// at the price of recomputing S and dP once more (7 MMAs per 128x128 block of
// scores instead of 5). Every MMA is 128 x 128 (x d) or 128 x d (x 128), and
// operands that would be re-read from shared memory every step (Q_i, dO_i in
// the query-stationary CTA; P^T, dS^T, dS) are kept in TMEM, which keeps the
// shared-memory port (128 bytes per clock) below the tensor core's demand.
//
// In both kinds the elementwise warps signal as soon as they have copied S^T
// (or S) into registers, so the MMA for the next tile's S^T (S) overlaps their
// work on the current tile; dP^T (dP) shares its TMEM columns with the P^T and
// dS^T (dS) written back from it, so the next dP^T waits for the dV/dK (dQ)
// MMAs that read them, which run in issue order. At d = 64 the TMEM columns
// 384-511 are free in both kinds and hold a second dP^T (dP) buffer: tile n
// uses buffer n % 2, so the next tile's dP^T (dP) runs before this tile's
// dV/dK (dQ).
//
// Roles (384 threads, one CTA per SM, both kinds):
//   warp 0      TMA producer          warp 1      MMA issuer, TMEM owner
//   warp 2      counts the tiles of a block-sparse CTA
//   warps 4-7   elementwise, columns [0, 64) of each tile (thread = TMEM lane = row)
//   warps 8-11  elementwise, columns [64, 128)
//
// TMEM (512 columns):
//   key-stationary:   S^T at 0; dP^T at 128, where warpgroup h later writes its
//                     P^T (32 columns) at 128+64h and dS^T at 128+64h+32;
//                     dV at 256, dK at 256+d; at d = 64 odd tiles use 384 for dP^T.
//   query-stationary: Q_i at 0 and dO_i at d/2 (bf16 pairs), S at d, dP at
//                     d+128 (warpgroup h writes its dS at d+128+64h), dQ at d+256;
//                     at d = 64 odd tiles use 384 for dP.
#pragma once

#include <cuda_fp16.h>

#include "philox.cuh"
#include "sm100.cuh"

namespace fa {
namespace bwd {

using namespace fa::sm100;

constexpr int kThreads = 384;
constexpr int kBlockN = 128;  // keys per key-stationary CTA and per query-stationary step
constexpr int kBlockQ = 128;  // queries per query-stationary CTA
constexpr int kBR = 128;      // queries per key-stationary step
constexpr int kRegsLaunch = 168;
constexpr int kRegsLow = 88;
constexpr int kRegsHigh = 208;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kTile = 128 * D * 2;  // one 128-row tile of Q, dO, K or V
  static constexpr int kChunk = 128 * 128;   // 64 columns x 128 rows, 128-byte swizzle
  // key-stationary layout: K_j, V_j, then a ring of (Q_i, dO_i, lse2_i, D_i)
  static constexpr int kS1 = (D == 128) ? 2 : 3;
  static constexpr int k1K = 0;
  static constexpr int k1V = k1K + kTile;
  static constexpr int k1Q = k1V + kTile;
  static constexpr int k1DO = k1Q + kS1 * kTile;
  static constexpr int k1L = k1DO + kS1 * kTile;
  static constexpr int k1Dv = k1L + kS1 * kBR * 4;
  static constexpr int k1End = k1Dv + kS1 * kBR * 4;
  // query-stationary layout: rings of K_j and V_j (Q_i, dO_i live in TMEM)
  static constexpr int kS2 = 3;
  static constexpr int k2K = 0;
  static constexpr int k2V = k2K + kS2 * kTile;
  static constexpr int k2End = k2V + kS2 * kTile;
  static constexpr int kOffBar = ((k1End > k2End ? k1End : k2End) + 15) / 16 * 16;
  static constexpr int kNumBars = 21;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;  // tmem slot, abort flag, tile count
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= 512 && 2 * D + 256 <= 512, "TMEM budget");
  // TMEM columns
  static constexpr int kColQ = 0, kColDO = D / 2, kColS2 = D, kColDP2 = D + 128, kColDQ = D + 256;
};

// Barrier slots of the two CTA kinds (they share the same shared-memory words).
// `drain` (both kinds) lets the MMA issuer wait for its own MMAs on the abort path.
struct KeyBars {
  static constexpr int kv_full = 0, qdo_full = 1, qdo_empty = 4, s_full = 7, s_free = 8, dp_full = 9,
                       p_full = 10, all_done = 11, dp_full1 = 12, drain = 19;
};
struct QueryBars {
  static constexpr int q_ready = 0, k_full = 1, k_empty = 4, v_full = 7, v_empty = 10, s_full = 13,
                       s_free = 14, dp_full = 15, ds_full = 16, all_done = 17, qdo_in = 18, drain = 19,
                       dp_full1 = 20;
};

// Abort path of a producer: wait (bounded, whatever the abort flag says) for the
// last load issued into each of the S stages of a ring whose full barriers start
// at `bar0`, `issued` loads in all, so no copy still writes shared memory when
// the CTA exits.
__device__ __forceinline__ void drain_ring(const uint64_t* bars, int bar0, int S, int issued, uint64_t timeout_ns) {
  for (int s = 0; s < S; ++s) {
    if (issued > s) {
      const int last = issued - 1 - ((issued - 1 - s) % S);
      mbar_wait_bounded(smem_u32(&bars[bar0 + s]), (last / S) & 1, timeout_ns);
    }
  }
}

// Walks the tiles one CTA visits, in ascending order. Dense and causal ranges
// are arithmetic; a block mask is read from global memory (a few cached bytes
// per step): key-stationary CTAs scan mask column j, query-stationary CTAs scan
// mask row i, both with the causal valid-tile rule applied by AND.
// The causal valid-tile rule ("当算力不再是瓶颈" essay, section 三.1) with the
// diagonal shifted by off = Nk - N (the N queries are the last N of Nk positions):
// query tile x and key tile y share an allowed pair iff y*128 <= (x's last row,
// at most N - 1) + off. `first`/`last` below solve it for x and for y.
struct TileCursor {
  const uint8_t* mask;  // [Tq][Tk]
  int kind;  // 0 key-stationary (walks query tiles), 1 query-stationary (walks key tiles)
  int tile, Tq, Tk, N, off, causal, pos;
  __device__ __forceinline__ bool causal_ok(int x) const {
    if (!causal) return true;
    const int qt = kind == 0 ? x : tile, kt = kind == 0 ? tile : x;
    return kt * 128 <= min(qt * 128 + 127, N - 1) + off;
  }
  __device__ __forceinline__ bool allowed(int x) const {
    if (!causal_ok(x)) return false;
    const size_t e = kind == 0 ? static_cast<size_t>(x) * Tk + tile : static_cast<size_t>(tile) * Tk + x;
    return mask[e] != 0;
  }
  // Key-stationary: first query tile reaching this key tile (the last query tile
  // always does: its last row N - 1 reaches key Nk - 1).
  __device__ __forceinline__ int first() const {
    if (mask != nullptr || kind != 0 || !causal) return 0;
    const int y = tile * 128 - off - 127;
    return y <= 0 ? 0 : (y + 127) / 128;
  }
  // Query-stationary: one past the last key tile this query tile reaches.
  __device__ __forceinline__ int end() const {
    if (!causal) return Tk;
    const int last_key = min(tile * 128 + 127, N - 1) + off;
    return last_key < 0 ? 0 : min(Tk, last_key / 128 + 1);
  }
  // Next visited tile (call exactly `len` times).
  __device__ __forceinline__ int next() {
    if (mask == nullptr) return pos++;
    while (!allowed(pos)) ++pos;
    return pos++;
  }
};

struct Params {
  const void* q;
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* delta;  // [BH][Npad]
  float* lse2;   // [BH][Npad]
  const uint8_t* block_mask;  // [Tq][Tk] or null
  int32_t* trace;
  int* status;
  uint64_t timeout_ns;  // limit of every wait
  int withhold;         // debug: the producers issue no load, so the first waits run out
  // Dropout (kDropout instances, see philox.cuh): an element is dropped iff its
  // draw is below drop_t; kept ones are scaled by drop_scale = 256 / (256 - drop_t).
  uint32_t drop_t;
  float drop_scale;
  philox::Keys drop_keys;  // round keys of the dropout seed
  int N;     // query rows
  int Nk;    // key / value rows
  int d;     // head dimension of the tensors (<= D; columns d..D-1 are zero in the kernel)
  int Npad;  // query rows rounded up to 128
  int BH;
  int Tq;    // ceil(N / 128) query tiles
  int Tk;    // ceil(Nk / 128) key tiles
  int head_group;  // heads walked together (CTA order)
  int causal;
  float scale;
  float scale_log2;
};

// --------------------------------------------------------------------------- prep

// HBM bound. A group of D/8 threads per row, each with one 16-byte piece of O
// and of dO; every thread covers kPrepRounds rows and issues all its loads
// before the first product, so each warp keeps 2 x kPrepRounds x 512 bytes in
// flight. A block covers kPrepRows(D) consecutive padded rows (a divisor of 128).
constexpr int kPrepThreads = 256;
constexpr int kPrepRounds = 2;
template <int D>
constexpr int kPrepRows = kPrepThreads / (D / 8) * kPrepRounds;

template <int D, bool BF16>
__global__ void __launch_bounds__(kPrepThreads) fa_bwd_prep_kernel(Params p) {
  constexpr int kTPR = D / 8;
  constexpr int kRowsPerRound = kPrepThreads / kTPR;
  const int part = static_cast<int>(threadIdx.x % kTPR);
  // The block's rows lie in one head (kPrepRows divides Npad).
  const long long block_row = static_cast<long long>(blockIdx.x) * kPrepRows<D>;
  const int bh = static_cast<int>(block_row / p.Npad);
  const int r_first = static_cast<int>(block_row - static_cast<long long>(bh) * p.Npad) +
                      static_cast<int>(threadIdx.x / kTPR);
  uint4 a[kPrepRounds], b[kPrepRounds];
#pragma unroll
  for (int k = 0; k < kPrepRounds; ++k) {
    const int r = r_first + k * kRowsPerRound;
    a[k] = make_uint4(0, 0, 0, 0);
    b[k] = make_uint4(0, 0, 0, 0);
    if (r < p.N && part * 8 < p.d) {
      const size_t off = (static_cast<size_t>(bh) * p.N + r) * p.d + part * 8;
      a[k] = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.o) + off);
      b[k] = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + off);
    }
  }
#pragma unroll
  for (int k = 0; k < kPrepRounds; ++k) {
    const int r = r_first + k * kRowsPerRound;
    const uint32_t aw[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
    const uint32_t bw[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a0, a1, b0, b1;
      if constexpr (BF16) {
        a0 = __uint_as_float(aw[i] << 16);
        a1 = __uint_as_float(aw[i] & 0xFFFF0000u);
        b0 = __uint_as_float(bw[i] << 16);
        b1 = __uint_as_float(bw[i] & 0xFFFF0000u);
      } else {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&aw[i]));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&bw[i]));
        a0 = fa.x;
        a1 = fa.y;
        b0 = fb.x;
        b1 = fb.y;
      }
      acc = fmaf(a0, b0, acc);
      acc = fmaf(a1, b1, acc);
    }
#pragma unroll
    for (int m = kTPR / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (part == 0) {
      const bool valid = r < p.N;
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
}

// --------------------------------------------------------------------------- shared state

struct Ctx {
  uint8_t* smem;
  uint64_t* bars;
  TileCursor cursor;  // positioned at the first candidate tile
  int len;
  uint32_t tmem;
  WaitCtx wait;
  int warp, lane, bh;
  __device__ __forceinline__ uint32_t bar(int i) const { return smem_u32(&bars[i]); }
};

// Round NCOLS fp32 TMEM columns of this thread's lane, times `mul`, to 16-bit
// values (zeros if `have` is false) and write the warp's 32 rows with TMA through
// shared memory: boxes of 64 columns x 32 rows in the 128-byte-swizzled layout
// (NCOLS = 64 or 128), or one unswizzled box of 32 columns (NCOLS = 32). `stage`
// is the warp's own staging area (32 * NCOLS * 2 bytes, 1024-byte aligned). The
// rows go to columns [col0, col0 + NCOLS) of rows [row0, row0 + 32) of head
// `bh`; the store clips rows past N. Lane 0 commits one bulk group, which the
// caller waits for before the CTA exits.
template <bool BF16, int NCOLS>
__device__ __forceinline__ void store_rows_tma(uint32_t taddr, float mul, bool have, uint32_t stage,
                                               const CUtensorMap* map, int col0, int row0, int bh, int N,
                                               int ncols_tensor) {
  const uint32_t lane = threadIdx.x & 31u;
  constexpr int kBoxCols = NCOLS >= 64 ? 64 : NCOLS;
  constexpr uint32_t kRowBytes = kBoxCols * 2;
  constexpr uint32_t kBoxBytes = 32 * kRowBytes;
  constexpr bool kSwizzle = kBoxCols == 64;
#pragma unroll
  for (int c = 0; c < NCOLS; c += 32) {
    uint32_t v[32];
    if (have) {
      tmem_ld32(taddr + c, v);
      tmem_ld_wait();
    }
    uint32_t w[16];
#pragma unroll
    for (int x = 0; x < 16; ++x)
      w[x] = have ? pack2<BF16>(__uint_as_float(v[2 * x]) * mul, __uint_as_float(v[2 * x + 1]) * mul) : 0u;
    const uint32_t row_addr = stage + static_cast<uint32_t>(c / kBoxCols) * kBoxBytes + lane * kRowBytes;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t chunk = static_cast<uint32_t>((c % kBoxCols) / 8 + k);
      if (kSwizzle) chunk ^= lane & 7u;
      sts128(row_addr + chunk * 16, w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && row0 < N) {
    // Boxes that start past the tensor's last column (a padded head dimension)
    // are not stored; a box that straddles it is clipped by the store.
#pragma unroll
    for (int b = 0; b < NCOLS / kBoxCols; ++b)
      if (col0 + b * kBoxCols < ncols_tensor)
        tma_store_3d(map, stage + static_cast<uint32_t>(b) * kBoxBytes, col0 + b * kBoxCols, row0, bh);
    bulk_commit_group();
  }
}

// --------------------------------------------------------------------------- key-stationary CTA

template <int D, bool BF16, bool kDropout>
__device__ __forceinline__ void key_cta(const Ctx& c, const Params& p, const CUtensorMap* tq, const CUtensorMap* tk,
                                        const CUtensorMap* tv, const CUtensorMap* tdo, const CUtensorMap* tdk,
                                        const CUtensorMap* tdv, int j) {
  using C = Cfg<D>;
  using B = KeyBars;
  constexpr int S = C::kS1;
  constexpr int kChunk = C::kChunk;
  uint8_t* sK = c.smem + C::k1K;
  uint8_t* sV = c.smem + C::k1V;
  uint8_t* sQ = c.smem + C::k1Q;
  uint8_t* sDO = c.smem + C::k1DO;
  float* sL = reinterpret_cast<float*>(c.smem + C::k1L);
  float* sDv = reinterpret_cast<float*>(c.smem + C::k1Dv);
  const int len = c.len;
  // TMEM: S^T at columns 0-127, dP^T (then P^T and dS^T over it) at 128-255, dV and dK
  // from 256. At d = 64 columns 384-511 are free and hold a second dP^T buffer: tile
  // n uses buffer n % 2, so dP^T of tile n + 1 is computed before dV and dK of tile n.
  constexpr bool kTwoDP = D == 64;
  auto dp_col = [&](int n) -> uint32_t { return (kTwoDP && (n & 1)) ? 384u : 128u; };
  auto dp_bar = [&](int n) { return (kTwoDP && (n & 1)) ? B::dp_full1 : B::dp_full; };

  if (c.warp < 4) {
    reg_dealloc<kRegsLow>();
    if (c.warp == 0 && c.lane == 0) {
      // ---------------------------------------------------------- producer
      TileCursor cur = c.cursor;
      int32_t* tr = p.trace ? p.trace + (static_cast<size_t>(c.bh) * p.Tk + j) * (p.Tq + 1) : nullptr;
      if (tr) tr[0] = len;
      if (len > 0 && !p.withhold) {
        mbar_arrive_expect_tx(c.bar(B::kv_full), 2 * C::kTile);
        for (int ch = 0; ch < D / 64; ++ch) {
          tma_load_3d(smem_u32(sK + ch * kChunk), tk, c.bar(B::kv_full), ch * 64, j * kBlockN, c.bh);
          tma_load_3d(smem_u32(sV + ch * kChunk), tv, c.bar(B::kv_full), ch * 64, j * kBlockN, c.bh);
        }
      }
      int issued = 0;
      for (int n = 0; n < len && !p.withhold; ++n) {
        const int i = cur.next();
        if (tr) tr[1 + n] = i | (1 << 16);
        const int s = n % S;
        if (!mbar_wait(c.bar(B::qdo_empty + s), ((n / S) & 1) ^ 1, c.wait)) break;
        ++issued;
        const uint32_t bar = c.bar(B::qdo_full + s);
        mbar_arrive_expect_tx(bar, 2 * C::kTile + 2 * kBR * 4);
        // The Q and dO maps have 64-row boxes: two boxes fill one 128-row chunk.
        for (int ch = 0; ch < D / 64; ++ch) {
          for (int hr = 0; hr < 2; ++hr) {
            const uint32_t off = s * C::kTile + ch * kChunk + hr * 64 * 128;
            tma_load_3d(smem_u32(sQ + off), tq, bar, ch * 64, i * kBR + hr * 64, c.bh);
            tma_load_3d(smem_u32(sDO + off), tdo, bar, ch * 64, i * kBR + hr * 64, c.bh);
          }
        }
        const size_t vo = static_cast<size_t>(c.bh) * p.Npad + static_cast<size_t>(i) * kBR;
        bulk_load(smem_u32(sL + s * kBR), p.lse2 + vo, kBR * 4, bar);
        bulk_load(smem_u32(sDv + s * kBR), p.delta + vo, kBR * 4, bar);
      }
      if (*c.wait.abort_flag) {
        if (len > 0 && !p.withhold) mbar_wait_bounded(c.bar(B::kv_full), 0, c.wait.timeout_ns);
        drain_ring(c.bars, B::qdo_full, S, issued, c.wait.timeout_ns);
      }
    } else if (c.warp == 1 && c.lane == 0 && len > 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_sp = idesc_f16(BF16, 128, kBR, false, false);  // S^T, dP^T
      constexpr uint32_t idesc_kv = idesc_f16(BF16, 128, D, false, true);     // dV, dK
      const uint32_t t = c.tmem;
      // Base descriptors; every MMA below adds a compile-time offset to them.
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);          // K-major A of S^T
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 16, 1024);          // K-major A of dP^T
      const uint64_t dQk = sdesc_sw128(smem_u32(sQ), 16, 1024);         // K-major B of S^T
      const uint64_t dDOk = sdesc_sw128(smem_u32(sDO), 16, 1024);       // K-major B of dP^T
      const uint64_t dQm = sdesc_sw128(smem_u32(sQ), kChunk, 1024);     // MN-major B of dK
      const uint64_t dDOm = sdesc_sw128(smem_u32(sDO), kChunk, 1024);   // MN-major B of dV
      auto issue_s = [&](int n) {  // S^T_n (stage resident)
        const uint64_t bq = sdesc_add(dQk, static_cast<uint32_t>(n % S) * C::kTile);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k * 16) / 64) * kChunk + ((k * 16) % 64) * 2;
          umma_ss(t, sdesc_add(dK, off), sdesc_add(bq, off), idesc_sp, k > 0);
        }
        umma_commit(c.bar(B::s_full));
      };
      auto issue_dp = [&](int n) {  // dP^T_n (stage resident), into dP^T buffer n % 2 at d = 64
        const uint64_t bdo = sdesc_add(dDOk, static_cast<uint32_t>(n % S) * C::kTile);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k * 16) / 64) * kChunk + ((k * 16) % 64) * 2;
          umma_ss(t + dp_col(n), sdesc_add(dV, off), sdesc_add(bdo, off), idesc_sp, k > 0);
        }
        umma_commit(c.bar(dp_bar(n)));
      };
      bool ok = mbar_wait(c.bar(B::kv_full), 0, c.wait) && mbar_wait(c.bar(B::qdo_full), 0, c.wait);
      const bool issued = ok;  // MMAs are issued from here on
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int n = 0; ok && n < len; ++n) {
        const int s = n % S;
        if (n + 1 < len) {
          // S^T_{n+1} overwrites S^T_n once the elementwise warps hold it in registers.
          if (!(ok = mbar_wait(c.bar(B::s_free), n & 1, c.wait))) break;
          if (!(ok = mbar_wait(c.bar(B::qdo_full + (n + 1) % S), ((n + 1) / S) & 1, c.wait))) break;
          tc_fence_after();
          issue_s(n + 1);
          // dP^T_{n+1} into the other buffer, last read by dV_{n-1} and dK_{n-1} (issued earlier).
          if (kTwoDP) issue_dp(n + 1);
        }
        if (!(ok = mbar_wait(c.bar(B::p_full), n & 1, c.wait))) break;
        tc_fence_after();
        const uint32_t acc = n > 0 ? 1u : 0u;
        const uint64_t bdo = sdesc_add(dDOm, static_cast<uint32_t>(s) * C::kTile);
        const uint64_t bq = sdesc_add(dQm, static_cast<uint32_t>(s) * C::kTile);
#pragma unroll
        for (int k = 0; k < kBR / 16; ++k) {
          // P^T columns of query rows 16k..16k+15: warpgroup h = k/4 wrote them at 128 + 64h.
          umma_ts(t + 256, t + dp_col(n) + 64 * (k / 4) + 8 * (k % 4), sdesc_add(bdo, k * 16 * 128), idesc_kv,
                  acc | static_cast<uint32_t>(k > 0));
        }
#pragma unroll
        for (int k = 0; k < kBR / 16; ++k) {
          umma_ts(t + 256 + D, t + dp_col(n) + 64 * (k / 4) + 32 + 8 * (k % 4), sdesc_add(bq, k * 16 * 128), idesc_kv,
                  acc | static_cast<uint32_t>(k > 0));
        }
        umma_commit(c.bar(B::qdo_empty + s));
        if (!kTwoDP && n + 1 < len) issue_dp(n + 1);  // dP^T columns: ordered after dV, dK read P^T, dS^T
      }
      if (ok) {
        umma_commit(c.bar(B::all_done));
      } else if (issued) {
        // Aborting: let every MMA this thread issued complete before TMEM and the
        // shared-memory operands are released.
        umma_commit(c.bar(B::drain));
        mbar_wait_bounded(c.bar(B::drain), 0, c.wait.timeout_ns);
      }
    }
  } else {
    reg_alloc<kRegsHigh>();
    // ------------------------------------------------------------ elementwise (thread = key row)
    TileCursor cur = c.cursor;
    const int h = (c.warp - 4) / 4;  // query columns [64h, 64h + 64) of each tile
    const int wq = c.warp % 4;
    const int r = wq * 32 + c.lane;
    const int key = j * kBlockN + r;
    const bool key_valid = key < p.Nk;
    const uint32_t tl = c.tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint32_t drop_c7 = philox::keep_bias(p.drop_t);
    const int qo = 64 * h;
    bool ok = true;
    for (int n = 0; n < len; ++n) {
      const int i = cur.next();
      const int s = n % S;
      // Dropout: keep flags of this key against query rows i*128 + qo .. +63
      // (group g: rows 4g .. 4g + 3), drawn while S^T is computed.
      uint32_t kb[kDropout ? 2 : 1] = {};
      if constexpr (kDropout) {
        const uint32_t rg_first = static_cast<uint32_t>(i * kBR + qo) / 4;
#pragma unroll
        for (int g = 0; g < 16; g += 4) {
          const uint4 w = philox::draws_col(rg_first + g, static_cast<uint32_t>(key), static_cast<uint32_t>(c.bh),
                                            p.drop_keys);
          philox::add_keep_flags(kb, g, w.x, drop_c7);
          philox::add_keep_flags(kb, g + 1, w.y, drop_c7);
          philox::add_keep_flags(kb, g + 2, w.z, drop_c7);
          philox::add_keep_flags(kb, g + 3, w.w, drop_c7);
        }
      }
      if (!(ok = mbar_wait_warp(c.bar(B::s_full), n & 1, c.wait))) break;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tl + qo, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + qo + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(c.bar(B::s_free));
      if (!(ok = mbar_wait_warp(c.bar(B::qdo_full + s), (n / S) & 1, c.wait))) break;  // lse2, D of tile i
      // Columns x < lim are masked (causal: key > query + Nk - N; or the key row
      // lies past Nk).
      int lim = 0;
      if (!key_valid) {
        lim = 64;
      } else if (p.causal) {
        lim = min(64, max(0, key - (p.Nk - p.N) - (i * kBR + qo)));
      }
      const uint32_t aL = smem_u32(sL + s * kBR + qo);
      float pv[64];
#pragma unroll
      for (int x = 0; x < 64; x += 4) {
        const float4 l4 = lds128(aL + x * 4);
        pv[x] = ex2(fmaf(__uint_as_float(sr[x]), sl2, -l4.x));
        pv[x + 1] = ex2(fmaf(__uint_as_float(sr[x + 1]), sl2, -l4.y));
        pv[x + 2] = ex2(fmaf(__uint_as_float(sr[x + 2]), sl2, -l4.z));
        pv[x + 3] = ex2(fmaf(__uint_as_float(sr[x + 3]), sl2, -l4.w));
      }
      if (lim > 0) {
#pragma unroll
        for (int x = 0; x < 64; ++x)
          if (x < lim) pv[x] = 0.0f;
      }
      if (!(ok = mbar_wait_warp(c.bar(dp_bar(n)), kTwoDP ? ((n >> 1) & 1) : (n & 1), c.wait))) break;
      tc_fence_after();
      uint32_t dr[64];
      tmem_ld32(tl + dp_col(n) + qo, *reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
      tmem_ld32(tl + dp_col(n) + qo + 32, *reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
      tmem_ld_wait();
      const uint32_t aD = smem_u32(sDv + s * kBR + qo);
      uint32_t pk[32], dk[32];
      if constexpr (kDropout) {
        // dV takes (P o M)^T (the factor 256 / (256 - t) of Z = M * 256 / (256 - t)
        // is applied in the dV epilogue); dS^T = P^T o (dP^T o Z - D).
        const uint32_t zs = __float_as_uint(p.drop_scale);
#pragma unroll
        for (int x = 0; x < 64; x += 4) {
          const float4 d4 = lds128(aD + x * 4);
          const uint32_t f = philox::group_flags(kb, x / 4);
          uint32_t m01, m23;
          philox::pair_masks(f, m01, m23);
          const float z0 = __uint_as_float(philox::elem_mask<0>(f) & zs);
          const float z1 = __uint_as_float(philox::elem_mask<1>(f) & zs);
          const float z2 = __uint_as_float(philox::elem_mask<2>(f) & zs);
          const float z3 = __uint_as_float(philox::elem_mask<3>(f) & zs);
          pk[x / 2] = pack2<BF16>(pv[x], pv[x + 1]) & m01;
          pk[x / 2 + 1] = pack2<BF16>(pv[x + 2], pv[x + 3]) & m23;
          dk[x / 2] = pack2<BF16>(pv[x] * fmaf(__uint_as_float(dr[x]), z0, -d4.x),
                                  pv[x + 1] * fmaf(__uint_as_float(dr[x + 1]), z1, -d4.y));
          dk[x / 2 + 1] = pack2<BF16>(pv[x + 2] * fmaf(__uint_as_float(dr[x + 2]), z2, -d4.z),
                                      pv[x + 3] * fmaf(__uint_as_float(dr[x + 3]), z3, -d4.w));
        }
      } else {
#pragma unroll
        for (int x = 0; x < 64; x += 4) {
          const float4 d4 = lds128(aD + x * 4);
          pk[x / 2] = pack2<BF16>(pv[x], pv[x + 1]);
          pk[x / 2 + 1] = pack2<BF16>(pv[x + 2], pv[x + 3]);
          dk[x / 2] =
              pack2<BF16>(pv[x] * (__uint_as_float(dr[x]) - d4.x), pv[x + 1] * (__uint_as_float(dr[x + 1]) - d4.y));
          dk[x / 2 + 1] = pack2<BF16>(pv[x + 2] * (__uint_as_float(dr[x + 2]) - d4.z),
                                      pv[x + 3] * (__uint_as_float(dr[x + 3]) - d4.w));
        }
      }
      tmem_st32(tl + dp_col(n) + qo, pk);
      tmem_st32(tl + dp_col(n) + qo + 32, dk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(c.bar(B::p_full));
    }
    // Epilogue: warpgroup 0 writes dV_j, warpgroup 1 writes scale * dK_j, staged in
    // the Q/dO ring (free once the last MMA, which read the last stage, completed).
    bool have = false;
    if (ok && len > 0) {
      ok = mbar_wait_warp(c.bar(B::all_done), 0, c.wait);
      have = ok;
    }
    tc_fence_after();
    if (ok) {
      const uint32_t stage = smem_u32(sQ) + static_cast<uint32_t>(c.warp - 4) * (32 * D * 2);
      const float dv_scale = kDropout ? p.drop_scale : 1.0f;
      store_rows_tma<BF16, D>(tl + 256 + h * D, h == 0 ? dv_scale : p.scale, have, stage, h == 0 ? tdv : tdk, 0,
                              j * kBlockN + wq * 32, c.bh, p.Nk, p.d);
    }
    if (c.lane == 0) bulk_wait_group_read<0>();  // shared memory read; the writes complete on their own
  }
}

// --------------------------------------------------------------------------- query-stationary CTA

template <int D, bool BF16, bool kDropout>
__device__ __forceinline__ void query_cta(const Ctx& c, const Params& p, const CUtensorMap* tq,
                                          const CUtensorMap* tk, const CUtensorMap* tv, const CUtensorMap* tdo,
                                          const CUtensorMap* tdq, int i) {
  using C = Cfg<D>;
  using B = QueryBars;
  constexpr int S = C::kS2;
  constexpr int kChunk = C::kChunk;
  uint8_t* sK = c.smem + C::k2K;
  uint8_t* sV = c.smem + C::k2V;
  const int len = c.len;
  // At d = 128, Q_i and dO_i (256-byte rows) are staged through shared memory by
  // TMA: per-thread row loads from global memory would touch 32 rows per warp
  // instruction. At d = 64 the rows are read directly (measured faster there).
  constexpr bool kStageQdo = D == 128;
  // At d = 64 TMEM columns 384-511 are free and hold a second dP buffer: tile n uses
  // buffer n % 2, so dP of tile n + 1 is computed before dQ of tile n.
  constexpr bool kTwoDP = D == 64;
  auto dp_col = [&](int n) -> uint32_t { return (kTwoDP && (n & 1)) ? 384u : static_cast<uint32_t>(C::kColDP2); };
  auto dp_bar = [&](int n) { return (kTwoDP && (n & 1)) ? B::dp_full1 : B::dp_full; };

  if (c.warp < 4) {
    reg_dealloc<kRegsLow>();
    if (c.warp == 0 && c.lane == 0) {
      // ---------------------------------------------------------- producer
      TileCursor cur = c.cursor;
      int32_t* tr = p.trace ? p.trace + static_cast<size_t>(p.BH) * p.Tk * (p.Tq + 1) +
                                  (static_cast<size_t>(c.bh) * p.Tq + i) * (p.Tk + 1)
                            : nullptr;
      if (tr) tr[0] = len;
      if (kStageQdo && !p.withhold) {
        // Q_i and dO_i land in the last K and V stages, which the elementwise warps
        // copy into TMEM before those stages first take K and V.
        mbar_arrive_expect_tx(c.bar(B::qdo_in), 2 * C::kTile);
        for (int ch = 0; ch < D / 64; ++ch)
          for (int hr = 0; hr < 2; ++hr) {
            const uint32_t off = (S - 1) * C::kTile + ch * kChunk + hr * 64 * 128;
            tma_load_3d(smem_u32(sK + off), tq, c.bar(B::qdo_in), ch * 64, i * kBlockQ + hr * 64, c.bh);
            tma_load_3d(smem_u32(sV + off), tdo, c.bar(B::qdo_in), ch * 64, i * kBlockQ + hr * 64, c.bh);
          }
      }
      int k_issued = 0, v_issued = 0;
      for (int n = 0; n < len && !p.withhold; ++n) {
        const int jt = cur.next();
        if (tr) tr[1 + n] = jt | (1 << 16);
        const int s = n % S;
        if (kStageQdo && n == S - 1 && !mbar_wait(c.bar(B::q_ready), 0, c.wait)) break;
        if (!mbar_wait(c.bar(B::k_empty + s), ((n / S) & 1) ^ 1, c.wait)) break;
        mbar_arrive_expect_tx(c.bar(B::k_full + s), C::kTile);
        for (int ch = 0; ch < D / 64; ++ch)
          tma_load_3d(smem_u32(sK + s * C::kTile + ch * kChunk), tk, c.bar(B::k_full + s), ch * 64,
                      jt * kBlockN, c.bh);
        ++k_issued;
        if (!mbar_wait(c.bar(B::v_empty + s), ((n / S) & 1) ^ 1, c.wait)) break;
        mbar_arrive_expect_tx(c.bar(B::v_full + s), C::kTile);
        for (int ch = 0; ch < D / 64; ++ch)
          tma_load_3d(smem_u32(sV + s * C::kTile + ch * kChunk), tv, c.bar(B::v_full + s), ch * 64,
                      jt * kBlockN, c.bh);
        ++v_issued;
      }
      if (*c.wait.abort_flag) {
        if (kStageQdo && !p.withhold) mbar_wait_bounded(c.bar(B::qdo_in), 0, c.wait.timeout_ns);
        drain_ring(c.bars, B::k_full, S, k_issued, c.wait.timeout_ns);
        drain_ring(c.bars, B::v_full, S, v_issued, c.wait.timeout_ns);
      }
    } else if (c.warp == 1 && c.lane == 0 && len > 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_sp = idesc_f16(BF16, 128, kBlockN, false, false);  // S, dP
      constexpr uint32_t idesc_q = idesc_f16(BF16, 128, D, false, true);          // dQ
      const uint32_t t = c.tmem;
      const uint64_t dKk = sdesc_sw128(smem_u32(sK), 16, 1024);       // K-major B of S
      const uint64_t dVk = sdesc_sw128(smem_u32(sV), 16, 1024);       // K-major B of dP
      const uint64_t dKm = sdesc_sw128(smem_u32(sK), kChunk, 1024);   // MN-major B of dQ
      auto issue_s = [&](int n) -> bool {  // S_n = Q K_n^T (A: Q in TMEM)
        const int s = n % S;
        if (!mbar_wait(c.bar(B::k_full + s), (n / S) & 1, c.wait)) return false;
        tc_fence_after();
        const uint64_t bk = sdesc_add(dKk, static_cast<uint32_t>(s) * C::kTile);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k * 16) / 64) * kChunk + ((k * 16) % 64) * 2;
          umma_ts(t + C::kColS2, t + C::kColQ + 8 * k, sdesc_add(bk, off), idesc_sp, k > 0);
        }
        umma_commit(c.bar(B::s_full));
        return true;
      };
      auto issue_dp = [&](int n) -> bool {  // dP_n = dO V_n^T (A: dO in TMEM); V_n released after
        const int s = n % S;
        if (!mbar_wait(c.bar(B::v_full + s), (n / S) & 1, c.wait)) return false;
        tc_fence_after();
        const uint64_t bv = sdesc_add(dVk, static_cast<uint32_t>(s) * C::kTile);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k * 16) / 64) * kChunk + ((k * 16) % 64) * 2;
          umma_ts(t + dp_col(n), t + C::kColDO + 8 * k, sdesc_add(bv, off), idesc_sp, k > 0);
        }
        umma_commit(c.bar(dp_bar(n)));
        umma_commit(c.bar(B::v_empty + s));
        return true;
      };
      bool ok = mbar_wait(c.bar(B::q_ready), 0, c.wait);
      const bool issued = ok;  // MMAs may be issued from here on
      if (ok) {
        tc_fence_after();
        ok = issue_s(0) && issue_dp(0);
      }
      for (int n = 0; ok && n < len; ++n) {
        const int s = n % S;
        if (n + 1 < len) {
          // S_{n+1} overwrites S_n once the elementwise warps hold it in registers.
          if (!(ok = mbar_wait(c.bar(B::s_free), n & 1, c.wait))) break;
          if (!(ok = issue_s(n + 1))) break;
          // dP_{n+1} into the other buffer, last read by dQ_{n-1} (issued earlier).
          if (kTwoDP && !(ok = issue_dp(n + 1))) break;
        }
        if (!(ok = mbar_wait(c.bar(B::ds_full), n & 1, c.wait))) break;  // dS_n written over dP_n
        tc_fence_after();
        const uint64_t bk = sdesc_add(dKm, static_cast<uint32_t>(s) * C::kTile);
#pragma unroll
        for (int k = 0; k < kBlockN / 16; ++k) {
          // dS columns of keys 16k..16k+15: warpgroup h = k/4 wrote them at dP + 64h.
          umma_ts(t + C::kColDQ, t + dp_col(n) + 64 * (k / 4) + 8 * (k % 4), sdesc_add(bk, k * 16 * 128),
                  idesc_q, (n > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(c.bar(B::k_empty + s));               // K_n free once dQ_n is done
        if (!kTwoDP && n + 1 < len && !(ok = issue_dp(n + 1))) break;  // dP columns: after dQ_n read dS_n
      }
      if (ok) {
        umma_commit(c.bar(B::all_done));
      } else if (issued) {
        // Aborting: let every MMA this thread issued complete before TMEM and the
        // shared-memory operands are released.
        umma_commit(c.bar(B::drain));
        mbar_wait_bounded(c.bar(B::drain), 0, c.wait.timeout_ns);
      }
    }
  } else {
    reg_alloc<kRegsHigh>();
    // ------------------------------------------------------------ elementwise (thread = query row)
    TileCursor cur = c.cursor;
    const int h = (c.warp - 4) / 4;  // key columns [64h, 64h + 64) of each tile
    const int wq = c.warp % 4;
    const int r = wq * 32 + c.lane;
    const int qrow = i * kBlockQ + r;
    const bool row_valid = qrow < p.N;
    const uint32_t tl = c.tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint32_t drop_c7 = philox::keep_bias(p.drop_t);
    const size_t vo = static_cast<size_t>(c.bh) * p.Npad + static_cast<size_t>(i) * kBlockQ + r;
    const float l2 = p.lse2[vo];  // +inf on padding rows: P = 0
    const float dd = p.delta[vo];
    // Q_i and dO_i rows into TMEM as the A operands of S and dP: warpgroup h
    // copies its half of the 32-bit words (pairs of 16-bit values) of this row.
    {
      constexpr int kWords = D / 4;  // this warpgroup's 32-bit words per row
      uint32_t a[kWords], b[kWords];
      if constexpr (kStageQdo) {
        // From the staged tiles (128-byte swizzle: 16-byte piece x of row r sits at
        // x ^ (r % 8)); rows past N arrive as zeros.
        const bool ok_in = mbar_wait_warp(c.bar(B::qdo_in), 0, c.wait);
        const uint32_t q_base = smem_u32(sK) + (S - 1) * C::kTile;
        const uint32_t do_base = smem_u32(sV) + (S - 1) * C::kTile;
#pragma unroll
        for (int v = 0; v < kWords / 4; ++v) {
          const int col = h * (D / 2) + 8 * v;  // first of the 8 columns of this 16-byte piece
          const uint32_t off = static_cast<uint32_t>((col / 64) * kChunk + r * 128 +
                                                     ((((col % 64) / 8) ^ (r & 7)) * 16));
          const float4 x = ok_in ? lds128(q_base + off) : make_float4(0.f, 0.f, 0.f, 0.f);
          const float4 y = ok_in ? lds128(do_base + off) : make_float4(0.f, 0.f, 0.f, 0.f);
          a[4 * v] = __float_as_uint(x.x); a[4 * v + 1] = __float_as_uint(x.y);
          a[4 * v + 2] = __float_as_uint(x.z); a[4 * v + 3] = __float_as_uint(x.w);
          b[4 * v] = __float_as_uint(y.x); b[4 * v + 1] = __float_as_uint(y.y);
          b[4 * v + 2] = __float_as_uint(y.z); b[4 * v + 3] = __float_as_uint(y.w);
        }
      } else {
        // Straight from global memory (row stride d; columns past d are zero); all
        // loads first, then the TMEM stores.
        const size_t roff = (static_cast<size_t>(c.bh) * p.N + (row_valid ? qrow : 0)) * p.d;
        const uint4* gq = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.q) + roff);
        const uint4* gdo = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + roff);
#pragma unroll
        for (int v = 0; v < kWords / 4; ++v) {
          const bool in = row_valid && (h * (D / 2) + 8 * v) < p.d;
          const uint4 x = in ? gq[h * kWords / 4 + v] : make_uint4(0, 0, 0, 0);
          const uint4 y = in ? gdo[h * kWords / 4 + v] : make_uint4(0, 0, 0, 0);
          a[4 * v] = x.x; a[4 * v + 1] = x.y; a[4 * v + 2] = x.z; a[4 * v + 3] = x.w;
          b[4 * v] = y.x; b[4 * v + 1] = y.y; b[4 * v + 2] = y.z; b[4 * v + 3] = y.w;
        }
      }
#pragma unroll
      for (int w0 = 0; w0 < kWords; w0 += 16) {
        tmem_st16(tl + C::kColQ + h * kWords + w0, *reinterpret_cast<uint32_t(*)[16]>(&a[w0]));
        tmem_st16(tl + C::kColDO + h * kWords + w0, *reinterpret_cast<uint32_t(*)[16]>(&b[w0]));
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(c.bar(B::q_ready));
    }
    bool ok = true;
    for (int n = 0; n < len; ++n) {
      const int jt = cur.next();
      // Dropout: keep flags of this query row against keys jt*128 + 64h .. +63
      // (group g: keys 4g .. 4g + 3), drawn while S is computed.
      uint32_t kb[kDropout ? 2 : 1] = {};
      if constexpr (kDropout) {
        const uint32_t cg_first = static_cast<uint32_t>(jt * kBlockN + 64 * h) / 4;
#pragma unroll
        for (int g = 0; g < 16; g += 4) {
          const uint4 w = philox::draws_row(cg_first + g, static_cast<uint32_t>(qrow), static_cast<uint32_t>(c.bh),
                                            p.drop_keys);
          philox::add_keep_flags(kb, g, w.x, drop_c7);
          philox::add_keep_flags(kb, g + 1, w.y, drop_c7);
          philox::add_keep_flags(kb, g + 2, w.z, drop_c7);
          philox::add_keep_flags(kb, g + 3, w.w, drop_c7);
        }
      }
      if (!(ok = mbar_wait_warp(c.bar(B::s_full), n & 1, c.wait))) break;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tl + C::kColS2 + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tl + C::kColS2 + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(c.bar(B::s_free));
      // Mask columns x > lim: causal (key > query) and keys past N.
      int lim = 63;
      if (p.causal) lim = min(lim, qrow + (p.Nk - p.N) - jt * kBlockN - 64 * h);
      const int kv_left = p.Nk - jt * kBlockN - 64 * h - 1;
      if (kv_left < lim) lim = kv_left;
      float pv[64];
#pragma unroll
      for (int x = 0; x < 64; ++x) pv[x] = ex2(fmaf(__uint_as_float(sr[x]), sl2, -l2));
      if (lim < 63) {
#pragma unroll
        for (int x = 0; x < 64; ++x)
          if (x > lim) pv[x] = 0.0f;
      }
      if (!(ok = mbar_wait_warp(c.bar(dp_bar(n)), kTwoDP ? ((n >> 1) & 1) : (n & 1), c.wait))) break;  // dP_n
      tc_fence_after();
      uint32_t dr[64];
      tmem_ld32(tl + dp_col(n) + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
      tmem_ld32(tl + dp_col(n) + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
      tmem_ld_wait();
      uint32_t dk[32];
      if constexpr (kDropout) {
        // dS = P o (dP o Z - D), Z = M * drop_scale.
        const uint32_t zs = __float_as_uint(p.drop_scale);
#pragma unroll
        for (int x = 0; x < 64; x += 4) {
          const uint32_t f = philox::group_flags(kb, x / 4);
          const float z0 = __uint_as_float(philox::elem_mask<0>(f) & zs);
          const float z1 = __uint_as_float(philox::elem_mask<1>(f) & zs);
          const float z2 = __uint_as_float(philox::elem_mask<2>(f) & zs);
          const float z3 = __uint_as_float(philox::elem_mask<3>(f) & zs);
          dk[x / 2] = pack2<BF16>(pv[x] * fmaf(__uint_as_float(dr[x]), z0, -dd),
                                  pv[x + 1] * fmaf(__uint_as_float(dr[x + 1]), z1, -dd));
          dk[x / 2 + 1] = pack2<BF16>(pv[x + 2] * fmaf(__uint_as_float(dr[x + 2]), z2, -dd),
                                      pv[x + 3] * fmaf(__uint_as_float(dr[x + 3]), z3, -dd));
        }
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          dk[x] = pack2<BF16>(pv[2 * x] * (__uint_as_float(dr[2 * x]) - dd),
                              pv[2 * x + 1] * (__uint_as_float(dr[2 * x + 1]) - dd));
      }
      tmem_st32(tl + dp_col(n) + 64 * h, dk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(c.bar(B::ds_full));
    }
    // Epilogue: warpgroup h writes columns [h*D/2, (h+1)*D/2) of scale * dQ_i,
    // staged in the K ring (free once the last dQ MMA, which read it, completed).
    bool have = false;
    if (ok && len > 0) {
      ok = mbar_wait_warp(c.bar(B::all_done), 0, c.wait);
      have = ok;
    }
    tc_fence_after();
    if (ok) {
      const uint32_t stage = smem_u32(sK) + static_cast<uint32_t>(c.warp - 4) * (32 * (D / 2) * 2);
      store_rows_tma<BF16, D / 2>(tl + C::kColDQ + h * (D / 2), p.scale, have, stage, tdq, h * (D / 2),
                                  i * kBlockQ + wq * 32, c.bh, p.N, p.d);
    }
    if (c.lane == 0) bulk_wait_group_read<0>();  // shared memory read; the writes complete on their own
  }
}

// --------------------------------------------------------------------------- main

// 1-D grid of batch*heads*2T CTAs walked in groups of heads (grouped_order).
// Rank 2t: key-stationary CTA for key tile t; rank 2t+1: query-stationary CTA
// for query tile T-1-t. Under a causal mask small key tiles and large query
// tiles carry the most work, so the heaviest CTAs of both kinds start first.
template <int D, bool BF16, bool kDropout>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_do,
                       const __grid_constant__ CUtensorMap tmap_dq, const __grid_constant__ CUtensorMap tmap_dk,
                       const __grid_constant__ CUtensorMap tmap_dv, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctx c;
  c.smem = smem;
  c.bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* tile_count = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
  c.warp = threadIdx.x / 32;
  c.lane = threadIdx.x % 32;
  int rank = 0;
  grouped_order(static_cast<int>(blockIdx.x), p.BH, p.Tk + p.Tq, p.head_group, c.bh, rank);
  // Ranks alternate key / query CTAs while both kinds remain, then the rest of
  // the longer kind; small key tiles and large query tiles (the heaviest under a
  // causal mask) come first.
  const int both = 2 * min(p.Tk, p.Tq);
  const bool keys = rank < both ? (rank & 1) == 0 : p.Tk > p.Tq;
  const int t = rank < both ? (rank >> 1) : (both >> 1) + (rank - both);
  const int tile = keys ? t : p.Tq - 1 - t;

  c.cursor.mask = p.block_mask;
  c.cursor.kind = keys ? 0 : 1;
  c.cursor.tile = tile;
  c.cursor.Tq = p.Tq;
  c.cursor.Tk = p.Tk;
  c.cursor.N = p.N;
  c.cursor.off = p.Nk - p.N;
  c.cursor.causal = p.causal;
  c.cursor.pos = c.cursor.first();

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    if (keys) {
      using B = KeyBars;
      mbar_init(c.bar(B::kv_full), 1);
      for (int s = 0; s < 3; ++s) {
        mbar_init(c.bar(B::qdo_full + s), 1);
        mbar_init(c.bar(B::qdo_empty + s), 1);
      }
      mbar_init(c.bar(B::s_full), 1);
      mbar_init(c.bar(B::s_free), 256);
      mbar_init(c.bar(B::dp_full), 1);
      mbar_init(c.bar(B::p_full), 256);
      mbar_init(c.bar(B::dp_full1), 1);
      mbar_init(c.bar(B::all_done), 1);
      mbar_init(c.bar(B::drain), 1);
    } else {
      using B = QueryBars;
      mbar_init(c.bar(B::q_ready), 256);
      for (int s = 0; s < 3; ++s) {
        mbar_init(c.bar(B::k_full + s), 1);
        mbar_init(c.bar(B::k_empty + s), 1);
        mbar_init(c.bar(B::v_full + s), 1);
        mbar_init(c.bar(B::v_empty + s), 1);
      }
      mbar_init(c.bar(B::s_full), 1);
      mbar_init(c.bar(B::s_free), 256);
      mbar_init(c.bar(B::dp_full), 1);
      mbar_init(c.bar(B::ds_full), 256);
      mbar_init(c.bar(B::dp_full1), 1);
      mbar_init(c.bar(B::all_done), 1);
      mbar_init(c.bar(B::qdo_in), 1);
      mbar_init(c.bar(B::drain), 1);
    }
    fence_barrier_init();
  }
  if (c.warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (c.warp == 2) {
    // Number of tiles this CTA visits.
    int count = 0;
    const int range = keys ? p.Tq : p.Tk;  // candidate tiles of the other kind
    if (p.block_mask != nullptr) {
      for (int base = 0; base < range; base += 32) {
        const int x = base + c.lane;
        const bool use = x < range && c.cursor.allowed(x);
        count += __popc(__ballot_sync(0xffffffffu, use));
      }
    } else if (keys) {
      count = p.Tq - c.cursor.first();
    } else {
      count = c.cursor.end();
    }
    if (c.lane == 0) *tile_count = count;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = *tmem_slot;
  c.len = *tile_count;
  c.wait = WaitCtx{abort_flag, p.status, p.timeout_ns};

  if (keys) {
    key_cta<D, BF16, kDropout>(c, p, &tmap_q, &tmap_k, &tmap_v, &tmap_do, &tmap_dk, &tmap_dv, tile);
  } else {
    query_cta<D, BF16, kDropout>(c, p, &tmap_q, &tmap_k, &tmap_v, &tmap_do, &tmap_dq, tile);
  }

  tc_fence_before();
  __syncthreads();
  if (c.warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(c.tmem, 512);
  }
}

}  // namespace bwd
}  // namespace fa
