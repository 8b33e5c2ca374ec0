// Fused exact attention forward for sm_100a.
//
// One CTA owns two 128-row query tiles (2p, 2p+1) of one (batch, head) and
// streams the 128-key tiles of K and V past them, as in FlashAttention's
// tiling ("FlashAttention" interview explainer, mstx.cn/posts/485, section 3.1)
// with the loop nest inverted so that the running statistics of a query tile
// stay on chip for its whole pass. Per key tile j and query tile q:
//   S = Q_q K_j^T                       tcgen05.mma, fp32 accumulator in TMEM
//   online softmax on S (running max m, sum l)   -- same explainer, section 3.2
//   O_q = alpha * O_q + P V_j           tcgen05.mma, P read from TMEM
// and only O = O_q / l and lse = (m + log2 l) * ln 2 are written to HBM.
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0      TMA producer: Q once, then K_j and V_j into two smem rings
//   warp 1      MMA issuer (one lane) and TMEM owner
//   warp 2      builds the key-tile list of a block-sparse CTA
//   warps 4-7   softmax for query tile 0 (thread = row, lane of TMEM)
//   warps 8-11  softmax for query tile 1
// The two softmax warpgroups alternate with the tensor core: while one turns
// its S into P, the tensor core runs the other tile's P V and next Q K^T.
//
// TMEM (512 columns): S/P of tile q at columns 128q .. 128q+127 (P is written
// over the first 64 columns as packed 16-bit pairs), O of tile q at 256 + q*D.
//
// Softmax detail: scores are used in the log2 domain, s2 = S * scale * log2(e),
// so exp is one FFMA plus ex2. The running max used for exponentiation is only
// moved when the new row max exceeds it by more than 8 (a factor 256), which
// leaves P <= 256 and keeps O and l consistent; the final O / l and lse are the
// same quantities in exact arithmetic, and the rescale of O (read, scale, write
// back in TMEM) is skipped for almost every tile.
#pragma once

#include "philox.cuh"
#include "sm100.cuh"

namespace fa {
namespace fwd {

using namespace fa::sm100;

constexpr int kBlockM = 128;  // query rows per tile
constexpr int kBlockN = 128;  // keys per tile
constexpr int kThreads = 384;
constexpr int kMaxSparseTiles = 2048;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kRegsLaunch = 168;  // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsLow = 64;
constexpr int kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split exceeds the launch allocation");

struct Params {
  void* o;
  float* lse;
  const uint8_t* block_mask;  // null unless block-sparse: [ceil(N/128)][Tc]
  int32_t* trace;             // null unless tracing
  int* status;
  uint64_t timeout_ns;        // limit of every wait
  int N;        // query rows
  int Nk;       // key / value rows
  int d;        // head dimension of the tensors (<= D; columns d..D-1 are zero in the kernel)
  int withhold;  // debug: the producer issues no load, so the first wait runs out
  // Split-KV: the key tiles are cut into n_splits consecutive ranges, one CTA per
  // (query-tile pair, range); each writes its partial O (fp32, normalised by its
  // own exp-sum) to o_part [n_splits][BH][N][d] and its lse to lse_part
  // [n_splits][BH][N] instead of o / lse. n_splits = 1 and o_part = null otherwise.
  int n_splits;
  float* o_part;
  float* lse_part;
  // Split-KV with one query tile per head (decoding): a CTA takes two
  // consecutive key ranges, one per softmax warpgroup ("slot"), both against
  // that query tile, so two dependency chains share the tensor core. No block mask.
  int dual;
  // Dropout (kDropout instances): an element is dropped iff its draw is below
  // drop_t; kept ones are scaled by drop_scale = 256 / (256 - drop_t).
  uint32_t drop_t;
  float drop_scale;
  philox::Keys drop_keys;  // round keys of the dropout seed
  float v_scale;  // kFp8: per-tensor scale of V (those of Q and K are in scale_log2)
  int BH;
  int n_pairs;  // ceil(T_q / 2)
  int Tc;       // ceil(Nk / 128)
  int head_group;  // heads walked together (CTA order)
  int causal;
  float scale_log2;  // softmax scale * log2(e)
};

// Shared memory. kF8: Q and K are e4m3 (one byte per element, so a 128 x 128 tile
// is one 128-byte-swizzled chunk), V arrives as e4m3 in a staging ring and is
// widened to 16 bits into the V ring. The V ring follows the K ring, so the
// epilogue's staging (64 KB at d = 128, from the K ring on) stays inside both.
// D = 256: one query tile per CTA (two S buffers of 128 + O 256 TMEM columns) and
// single K and V stages (64 KB tiles). kDeep (split-KV at D = 64, i.e. decoding, which streams
// K and V from HBM once): five stages, so more bytes are in flight per SM.
template <int D, bool kF8 = false, bool kDeep = false>
struct Smem {
  static constexpr int kStages = D == 256 ? 1 : (D == 128 ? 2 : (kDeep ? 5 : 3));
  static constexpr int kQTiles = D == 256 ? 1 : 2;  // query tiles per CTA
  static constexpr int kTileBytes = kBlockN * D * 2;           // one 16-bit V tile
  static constexpr int kQKBytes = kF8 ? kBlockN * D : kTileBytes;  // one Q or K tile
  static constexpr int kV8Bytes = kBlockN * D;                  // one e4m3 V tile (kF8)
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQTiles * kQKBytes;
  static constexpr int kVOff = kKOff + kStages * kQKBytes;
  static constexpr int kV8Off = kVOff + kStages * kTileBytes;
  static constexpr int kBarOff = kV8Off + (kF8 ? kStages * kV8Bytes : 0);
  // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2], o_full[2], drain,
  // for kF8 v8_full[S], v8_empty[S], and last pv_done (D = 256: P V of a key tile completed)
  static constexpr int kNumBars = 1 + 4 * kStages + 7 + (kF8 ? 2 * kStages : 0) + 1;
  static constexpr int kListOff = kBarOff + 8 * kNumBars + 16;  // + tmem slot, abort flag, list length
  static constexpr int kBytes = kListOff + 4 * kMaxSparseTiles;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

// Key-tile iteration shared by every role: entry n of the CTA's list is key
// tile j(n) with flags f(n) (bit q set: query tile 2p+q uses it). The tiles are
// those of the CTA's key range [lo, hi) (all of them unless split-KV).
struct TileList {
  int len;
  int mode;        // 0 dense, 1 causal, 2 list in shared memory, 3 two key ranges (dual)
  int lo;          // first key tile of the range (mode 3: of slot 0's range)
  int lim0, lim1;  // last key tile query tile 0 / 1 uses (-1: none, e.g. no tile 1)
  const uint32_t* list;
  int lo1, len0, len1;  // mode 3: slot 1's first key tile; tiles of each slot

  __device__ __forceinline__ uint32_t entry(int n) const {
    if (mode == 2) return list[n];
    if (mode == 3) {
      // The two slots' tiles alternate while both have some, then the longer one's rest.
      const int both = 2 * min(len0, len1);
      int slot, idx;
      if (n < both) {
        slot = n & 1;
        idx = n >> 1;
      } else {
        slot = len0 > len1 ? 0 : 1;
        idx = both / 2 + (n - both);
      }
      return static_cast<uint32_t>((slot ? lo1 : lo) + idx) | ((1u << slot) << 16);
    }
    const int j = lo + n;
    const uint32_t f = (j <= lim0 ? 1u : 0u) | (j <= lim1 ? 2u : 0u);
    return static_cast<uint32_t>(j) | (f << 16);
  }
};

// Causal valid-tile rule ("当算力不再是瓶颈" essay, section 三.1, with the diagonal
// shifted by Nk - N when the N queries are the last N of Nk positions): query
// tile qt reaches key tile j iff j*128 <= (its last row, at most N - 1) + Nk - N.
// Returns the last such j, or -1 if the tile reaches no key.
__device__ __forceinline__ int causal_last_key_tile(int qt, int N, int Nk) {
  const int last_row = min(qt * kBlockM + kBlockM - 1, N - 1);
  const int last_key = last_row + (Nk - N);
  return last_key < 0 ? -1 : last_key / kBlockN;
}

// Kernel variants, separate instances so the plain forward compiles without the
// others' bookkeeping: kPlain; kSplitKV (key ranges, fp32 partials); kDropout
// (P scaled by the dropout keep decisions before P V, see philox.cuh); kFp8
// (e4m3 Q, K, V with per-tensor scales: S = Q K^T by kind::f8f6f4 MMAs, V
// widened to 16 bits in shared memory by warps 2-3 for the 16-bit P V; d = 128).
enum Mode : int { kPlain = 0, kSplitKV = 1, kDropout = 2, kFp8 = 3 };

template <int D, bool BF16, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
                  const Params p) {
  constexpr bool kF8 = kMode == kFp8;
  using L = Smem<D, kF8, kMode == kSplitKV>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOff + 8 * L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBarOff + 8 * L::kNumBars + 4);
  int* list_len = reinterpret_cast<int*>(smem + L::kBarOff + 8 * L::kNumBars + 8);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + L::kListOff);

  const uint32_t bar_q_full = smem_u32(&bars[0]);
  auto bar_k_full = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto bar_k_empty = [&](int s) { return smem_u32(&bars[1 + S + s]); };
  auto bar_v_full = [&](int s) { return smem_u32(&bars[1 + 2 * S + s]); };
  auto bar_v_empty = [&](int s) { return smem_u32(&bars[1 + 3 * S + s]); };
  auto bar_s_full = [&](int q) { return smem_u32(&bars[1 + 4 * S + q]); };
  auto bar_p_full = [&](int q) { return smem_u32(&bars[1 + 4 * S + 2 + q]); };
  auto bar_o_full = [&](int q) { return smem_u32(&bars[1 + 4 * S + 4 + q]); };
  const uint32_t bar_drain = smem_u32(&bars[1 + 4 * S + 6]);
  auto bar_v8_full = [&](int s) { return smem_u32(&bars[1 + 4 * S + 7 + s]); };
  auto bar_v8_empty = [&](int s) { return smem_u32(&bars[1 + 4 * S + 7 + S + s]); };
  const uint32_t bar_pv_done = smem_u32(&bars[L::kNumBars - 1]);
  // D = 256 (one query tile per CTA): key tile n's S goes to TMEM columns
  // 128 * (n % 2), so S of tile n + 1 is computed while the softmax warps work on
  // tile n; otherwise query tile q's S is at columns 128 * q.
  constexpr bool kTwoS = D == 256;
  // D = 256 (single-stage K and V rings): warp 3 loads V, so the load of the next
  // K tile never waits in one thread's program order behind a V slot that the
  // current P V still reads. At smaller D (deeper rings) one producer is faster.
  constexpr bool kSplitV = D == 256 && !kF8;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // Heads in groups of p.head_group (their K/V stay in L2); inside a group the
  // heaviest query-tile pairs (the last ones, under a causal mask) start first.
  constexpr bool kSplit = kMode == kSplitKV;
  const int n_splits = kSplit ? p.n_splits : 1;
  const bool dual = kSplit && p.dual != 0;
  const int split_items = dual ? (n_splits + 1) / 2 : n_splits;  // CTAs per query-tile pair
  int bh, rank;
  grouped_order(static_cast<int>(blockIdx.x), p.BH, p.n_pairs * split_items, p.head_group, bh, rank);
  const int pair = p.n_pairs - 1 - rank / split_items;
  // Key range(s): split (slot 0) and, in dual mode, split + 1 (slot 1).
  const int split = kSplit ? (dual ? 2 : 1) * (rank % split_items) : 0;
  auto range_lo = [&](int sp) { return static_cast<int>(static_cast<long long>(sp) * p.Tc / n_splits); };
  const int key_lo = kSplit ? range_lo(split) : 0;
  const int key_hi = kSplit ? range_lo(split + 1) : p.Tc;
  const int q0 = L::kQTiles * pair;  // an item's query tiles: q0 and (a pair) q0 + 1
  const int Tq = (p.N + kBlockM - 1) / kBlockM;
  // Slot 1 holds query tile q0 + 1, or in dual mode key range split + 1 of q0.
  const int q1_active = dual ? (split + 1 < n_splits) : (L::kQTiles == 2 && (q0 + 1) < Tq);
  // Dual mode with at most 96 query rows: slot 1 takes the rows 32 TMEM lanes
  // lower (its Q is loaded from row -32), so the two slots' valid rows are worked
  // on by warps of different SM sub-partitions (a warp may only reach the 32
  // lanes of its own quarter).
  const int shift1 = (dual && p.N <= 96) ? 32 : 0;
  const int cta = bh * p.n_pairs + pair;  // trace record (never split)

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_k_full(s), 1);
      mbar_init(bar_k_empty(s), 1);
      mbar_init(bar_v_full(s), kF8 ? 2 : 1);  // kF8: one arrival per widening warp
      mbar_init(bar_v_empty(s), 1);
      if (kF8) {
        mbar_init(bar_v8_full(s), 1);
        mbar_init(bar_v8_empty(s), 2);
      }
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(bar_s_full(q), 1);
      mbar_init(bar_p_full(q), 128);
      mbar_init(bar_o_full(q), 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_pv_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // Causal reach of the two query tiles (every key tile when not causal). Each
  // role derives it where it needs it, so it is not live across the register split.
  auto reach = [&](int qi) {
    if (qi == 1 && !q1_active) return -1;
    return p.causal ? causal_last_key_tile(q0 + (dual ? 0 : qi), p.N, p.Nk) : p.Tc - 1;
  };
  if (warp == 2) {
    const int lim0 = reach(0), lim1 = reach(1);
    if (p.block_mask != nullptr) {
      // Union of the non-zero key tiles of mask rows q0 and q0+1, in order, with
      // the causal valid-tile rule applied by AND.
      const uint8_t* row0 = p.block_mask + static_cast<size_t>(q0) * p.Tc;
      const uint8_t* row1 = row0 + p.Tc;
      int count = 0;
      for (int base = key_lo; base < key_hi; base += 32) {
        const int j = base + lane;
        uint32_t f = 0;
        if (j < key_hi) {
          if (row0[j] && j <= lim0) f |= 1u;
          if (q1_active && row1[j] && j <= lim1) f |= 2u;
        }
        const uint32_t ballot = __ballot_sync(0xffffffffu, f != 0);
        if (f != 0) {
          const int pos = count + __popc(ballot & ((1u << lane) - 1u));
          if (pos < kMaxSparseTiles) list[pos] = static_cast<uint32_t>(j) | (f << 16);
        }
        count += __popc(ballot);
      }
      if (lane == 0) *list_len = count < kMaxSparseTiles ? count : kMaxSparseTiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = *tmem_slot;
  WaitCtx ctx{abort_flag, p.status, p.timeout_ns};

  auto make_tiles = [&]() {
    TileList tl;
    tl.lim0 = reach(0);
    tl.lim1 = reach(1);
    tl.list = list;
    tl.lo = key_lo;
    if (dual) {
      // Slot s covers key range split + s, clipped at the causal reach.
      tl.mode = 3;
      tl.lo1 = key_hi;
      const int hi1 = q1_active ? range_lo(split + 2) : key_hi;
      tl.len0 = max(0, min(key_hi, tl.lim0 + 1) - key_lo);
      tl.len1 = q1_active ? max(0, min(hi1, tl.lim1 + 1) - key_hi) : 0;
      tl.len = tl.len0 + tl.len1;
    } else if (p.block_mask != nullptr) {
      tl.mode = 2;
      tl.len = *list_len;
    } else if (p.causal) {
      tl.mode = 1;
      tl.len = max(0, min(key_hi, max(tl.lim0, tl.lim1) + 1) - key_lo);
    } else {
      tl.mode = 0;
      tl.len = key_hi - key_lo;
    }
    return tl;
  };

  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sK = smem + L::kKOff;
  uint8_t* sV = smem + L::kVOff;
  constexpr int kChunkBytes = 128 * 128;  // one 128-row x 64-column swizzled chunk

  // Register split: warpgroup 0 (producer, MMA, list builder, idle) needs few
  // registers; the two softmax warpgroups hold a 128-column row of S each.
  // 128 x kRegsLow + 256 x kRegsHigh <= 384 x 168, the launch allocation. Each
  // setmaxnreg sits inside the branch of the roles it serves, so the compiler
  // sees the budget of every code path.
  if (warp < 4) {
   reg_dealloc<kRegsLow>();
   const TileList tl = make_tiles();
   if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && tl.len > 0 && !p.withhold) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      int k_issued = 0, v_issued = 0;  // K and V loads issued (for the abort drain)
      // Dual mode: slot 1 reads query tile q0 too, from slot 0's buffer or, when its
      // rows are shifted, from its own copy loaded from row -32 (zero-filled there).
      const int nq = dual ? (shift1 ? 2 : 1) : 1 + q1_active;
      mbar_arrive_expect_tx(bar_q_full, nq * L::kQKBytes);
      for (int q = 0; q < nq; ++q) {
        const int qrow = dual ? q0 * kBlockM - q * shift1 : (q0 + q) * kBlockM;
        if constexpr (kF8) {
          tma_load_3d(smem_u32(sQ + q * L::kQKBytes), &tmap_q, bar_q_full, 0, qrow, bh);
        } else {
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem_u32(sQ + q * L::kQKBytes + c * kChunkBytes), &tmap_q, bar_q_full, c * 64, qrow, bh);
        }
      }
      if (p.trace) p.trace[static_cast<size_t>(cta) * (p.Tc + 1)] = tl.len;
      for (int n = 0; n < tl.len; ++n) {
        const uint32_t e = tl.entry(n);
        const int j = static_cast<int>(e & 0xFFFFu);
        if (p.trace) p.trace[static_cast<size_t>(cta) * (p.Tc + 1) + 1 + n] = static_cast<int32_t>(e);
        const int s = n % S;
        const uint32_t ph = ((n / S) & 1) ^ 1;
        if (!mbar_wait(bar_k_empty(s), ph, ctx)) break;
        mbar_arrive_expect_tx(bar_k_full(s), L::kQKBytes);
        if constexpr (kF8) {
          tma_load_3d(smem_u32(sK + s * L::kQKBytes), &tmap_k, bar_k_full(s), 0, j * kBlockN, bh);
        } else {
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem_u32(sK + s * L::kQKBytes + c * kChunkBytes), &tmap_k, bar_k_full(s), c * 64,
                        j * kBlockN, bh);
        }
        ++k_issued;
        if constexpr (kF8) {
          // e4m3 V into the staging ring; warps 2-3 widen it into the V ring.
          if (!mbar_wait(bar_v8_empty(s), ph, ctx)) break;
          mbar_arrive_expect_tx(bar_v8_full(s), L::kV8Bytes);
          tma_load_3d(smem_u32(smem + L::kV8Off + s * L::kV8Bytes), &tmap_v, bar_v8_full(s), 0, j * kBlockN, bh);
          ++v_issued;
        } else if (!kSplitV) {
          if (!mbar_wait(bar_v_empty(s), ph, ctx)) break;
          mbar_arrive_expect_tx(bar_v_full(s), L::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem_u32(sV + s * L::kTileBytes + c * kChunkBytes), &tmap_v, bar_v_full(s), c * 64,
                        j * kBlockN, bh);
          ++v_issued;
        }
      }
      if (*abort_flag) {
        // Aborting: wait (bounded, whatever the flag says) for every load this
        // thread issued, so no copy still writes shared memory when the CTA exits.
        // The last load into stage s completes that stage's barrier phase.
        for (int s = 0; s < S; ++s) {
          if (k_issued > s) {
            const int last = k_issued - 1 - ((k_issued - 1 - s) % S);
            mbar_wait_bounded(bar_k_full(s), (last / S) & 1, p.timeout_ns);
          }
          if (v_issued > s) {
            const int last = v_issued - 1 - ((v_issued - 1 - s) % S);
            mbar_wait_bounded(kF8 ? bar_v8_full(s) : bar_v_full(s), (last / S) & 1, p.timeout_ns);
          }
        }
        mbar_wait_bounded(bar_q_full, 0, p.timeout_ns);
      }
    }
  } else if (kSplitV && warp == 3) {
    // ------------------------------------------------------------ V producer (D = 256)
    if (lane == 0 && tl.len > 0 && !p.withhold) {
      prefetch_tmap(&tmap_v);
      int v_issued = 0;
      for (int n = 0; n < tl.len; ++n) {
        const int j = static_cast<int>(tl.entry(n) & 0xFFFFu);
        const int s = n % S;
        if (!mbar_wait(bar_v_empty(s), ((n / S) & 1) ^ 1, ctx)) break;
        mbar_arrive_expect_tx(bar_v_full(s), L::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem_u32(sV + s * L::kTileBytes + c * kChunkBytes), &tmap_v, bar_v_full(s), c * 64,
                      j * kBlockN, bh);
        ++v_issued;
      }
      if (*abort_flag) {
        // Aborting: wait (bounded) for the last load into each stage.
        for (int s = 0; s < S; ++s) {
          if (v_issued > s) {
            const int last = v_issued - 1 - ((v_issued - 1 - s) % S);
            mbar_wait_bounded(bar_v_full(s), (last / S) & 1, p.timeout_ns);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && tl.len > 0) {
      constexpr uint32_t idesc_s = idesc_f16(BF16, kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_pv = idesc_f16(BF16, kBlockM, D, false, true);
      uint32_t p_count[2] = {0, 0};
      uint32_t started[2] = {0, 0};
      bool ok = mbar_wait(bar_q_full, 0, ctx);

      // Base descriptors; every MMA below adds a compile-time offset to them.
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);             // K-major A of S
      const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);             // K-major B of S
      const uint64_t dV = sdesc_sw128(smem_u32(sV), kChunkBytes, 1024);    // MN-major B of P V
      auto issue_s = [&](int q, int n) {
        const int s = n % S;
        const int region = kTwoS ? (n & 1) : q;
        const uint32_t d_tmem = tmem + region * 128;
        const uint64_t bq = sdesc_add(dQ, static_cast<uint32_t>(dual && !shift1 ? 0 : q) * L::kQKBytes);
        const uint64_t bk = sdesc_add(dK, static_cast<uint32_t>(s) * L::kQKBytes);
        if constexpr (kF8) {
          // e4m3: K = 32 per MMA, 32 bytes along the 128-byte swizzled rows.
          constexpr uint32_t idesc_s8 = idesc_e4m3(kBlockM, kBlockN);
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            umma_ss_f8(d_tmem, sdesc_add(bq, 32 * k), sdesc_add(bk, 32 * k), idesc_s8, k > 0);
        } else {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int kk = k * 16;
            const uint32_t off = (kk / 64) * kChunkBytes + (kk % 64) * 2;
            umma_ss(d_tmem, sdesc_add(bq, off), sdesc_add(bk, off), idesc_s, k > 0);
          }
        }
        umma_commit(bar_s_full(region));
      };
      auto issue_pv = [&](int q, int n) {
        const int s = n % S;
        const uint32_t d_tmem = tmem + 256 + q * D;
        const uint32_t a_tmem = tmem + (kTwoS ? (n & 1) : q) * 128;
        const uint64_t bv = sdesc_add(dV, static_cast<uint32_t>(s) * L::kTileBytes);
#pragma unroll
        for (int k = 0; k < kBlockN / 16; ++k) {
          umma_ts(d_tmem, a_tmem + 8 * k, sdesc_add(bv, k * 16 * 128), idesc_pv,
                  (started[q] | static_cast<uint32_t>(k > 0)));
        }
        started[q] = 1;
      };

      // Prologue: S of the first key tile for each query tile that uses it.
      if (ok) ok = mbar_wait(bar_k_full(0), 0, ctx);
      bool issued = ok;  // an MMA has been issued (from here on)
      if (ok) {
        tc_fence_after();
        const uint32_t f0 = tl.entry(0) >> 16;
        for (int q = 0; q < 2; ++q)
          if (f0 & (1u << q)) issue_s(q, 0);
        umma_commit(bar_k_empty(0));
      }
      for (int n = 0; ok && n < tl.len; ++n) {
        const uint32_t f = tl.entry(n) >> 16;
        const bool has_next = (n + 1) < tl.len;
        const uint32_t fn = has_next ? (tl.entry(n + 1) >> 16) : 0u;
        if (has_next) {
          if (!(ok = mbar_wait(bar_k_full((n + 1) % S), ((n + 1) / S) & 1, ctx))) break;
          // A slot the next tile uses but this one does not gets its S first: its
          // S/P columns were last read by a P V issued in an earlier step, so its
          // softmax can run while this step waits for V and the other slot's P.
          if (kTwoS) {
            // The other S buffer was last read by P V of tile n - 1, issued earlier.
            tc_fence_after();
            issue_s(0, n + 1);
            umma_commit(bar_k_empty((n + 1) % S));
          } else if (fn & ~f) {
            tc_fence_after();
            for (int q = 0; q < 2; ++q)
              if ((fn & ~f) & (1u << q)) issue_s(q, n + 1);
          }
        }
        if (!(ok = mbar_wait(bar_v_full(n % S), (n / S) & 1, ctx))) break;
        tc_fence_after();
        for (int q = 0; q < 2; ++q) {
          if (f & (1u << q)) {
            const int pr = kTwoS ? (n & 1) : q;
            if (!(ok = mbar_wait(bar_p_full(pr), p_count[pr] & 1, ctx))) break;
            ++p_count[pr];
            tc_fence_after();
            issue_pv(q, n);
            if (kTwoS) umma_commit(bar_pv_done);
            else if (fn & (1u << q)) issue_s(q, n + 1);
          }
        }
        if (!ok) break;
        umma_commit(bar_v_empty(n % S));
        if (has_next && !kTwoS) umma_commit(bar_k_empty((n + 1) % S));
      }
      if (ok) {
        for (int q = 0; q < 2; ++q)
          if (started[q]) umma_commit(bar_o_full(q));
      } else if (issued) {
        // Aborting: let every MMA this thread issued complete before TMEM and the
        // shared-memory operands are released.
        umma_commit(bar_drain);
        mbar_wait_bounded(bar_drain, 0, p.timeout_ns);
      }
    }
  } else if (kF8 && !p.withhold) {
    // ------------------------------------------------------------ V widening (kFp8, warps 2-3)
    // Warp 2 + h widens key rows [64h, 64h + 64) of each e4m3 V tile into the
    // 16-bit V ring, in the layout TMA gives a 16-bit tile (64-column chunks,
    // 128-byte swizzle: 16-byte piece x of row r at x ^ (r % 8)). Four lanes per
    // row... a warp covers 4 rows x 128 columns per iteration, 16 columns a lane.
    const int h = warp - 2;
    bool ok = true;
    for (int n = 0; n < tl.len; ++n) {
      const int s = n % S;
      const uint32_t ph = (n / S) & 1;
      if (!(ok = mbar_wait_warp(bar_v8_full(s), ph, ctx))) break;
      if (!(ok = mbar_wait_warp(bar_v_empty(s), ph ^ 1, ctx))) break;
      const uint32_t src = smem_u32(smem + L::kV8Off + s * L::kV8Bytes);
      const uint32_t dst = smem_u32(sV + s * L::kTileBytes);
      const int c = lane % 8;  // columns 16c .. 16c + 15
#pragma unroll 4
      for (int it = 0; it < 16; ++it) {
        const int r = 64 * h + 4 * it + lane / 8;
        const float4 x4 = lds128(src + r * 128 + c * 16);
        const uint32_t xw[4] = {__float_as_uint(x4.x), __float_as_uint(x4.y), __float_as_uint(x4.z),
                                __float_as_uint(x4.w)};
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          w[2 * i] = e4m3x2_to_bf16x2(xw[i] & 0xFFFFu);
          w[2 * i + 1] = e4m3x2_to_bf16x2(xw[i] >> 16);
        }
        const uint32_t chunk = dst + static_cast<uint32_t>(c / 4) * kChunkBytes + static_cast<uint32_t>(r) * 128;
        const uint32_t p0 = static_cast<uint32_t>(2 * (c % 4));
        sts128(chunk + ((p0 ^ (r & 7)) * 16), w[0], w[1], w[2], w[3]);
        sts128(chunk + (((p0 + 1) ^ (r & 7)) * 16), w[4], w[5], w[6], w[7]);
      }
      // The MMA reads the ring through the async proxy.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar_v_full(s));
        mbar_arrive(bar_v8_empty(s));
      }
    }
  }
  } else {
    reg_alloc<kRegsHigh>();
    const TileList tl = make_tiles();
    // ------------------------------------------------------------ softmax
    const int q = (warp - 4) / 4;  // query tile within the pair
    const int wq = warp % 4;       // TMEM lane quarter
    const int qt = q0 + (dual ? 0 : q);
    const int row_local = wq * 32 + lane;
    const int row = qt * kBlockM + row_local - (q == 1 ? shift1 : 0);  // query row of this TMEM lane
    // A warp whose 32 rows are all outside [0, N) (padding of a short last tile, or
    // the shifted slot) keeps the barrier protocol but skips the arithmetic: rows
    // of P V are independent, and such rows are never stored.
    const int warp_row0 = row - lane;
    const bool warp_rows = warp_row0 + 31 >= 0 && warp_row0 < p.N;
    const bool tile_active = (q == 0) || q1_active;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_o = tmem + lane_off + 256 + q * D;
    const float sl2 = p.scale_log2;
    const uint32_t drop_c7 = philox::keep_bias(p.drop_t);

    float m_ref = -INFINITY;  // log2-domain reference max
    float l_sum = 0.0f;
    int count = 0;
    bool ok = true;

    if (tile_active && !p.withhold) {
      for (int n = 0; n < tl.len; ++n) {
        const uint32_t e = tl.entry(n);
        if (!((e >> 16) & (1u << q))) continue;
        const int j = static_cast<int>(e & 0xFFFFu);
        // Dropout keep decisions of this row's 128 keys, 16 draws per generator
        // block, made while S is still being computed. Key group w (keys 4w ..
        // 4w + 3) is bit 7 - w % 8 of the bytes of word w / 8, byte k for key 4w + k.
        uint32_t kb[kMode == kDropout ? 4 : 1] = {};
        if constexpr (kMode == kDropout) {
          if (warp_rows) {
            const uint32_t cg_tile = static_cast<uint32_t>(j) * (kBlockN / 4);
#pragma unroll
            for (int g = 0; g < kBlockN / 4; g += 4) {
              const uint4 w = philox::draws_row(cg_tile + g, static_cast<uint32_t>(row), static_cast<uint32_t>(bh),
                                                p.drop_keys);
              philox::add_keep_flags(kb, g, w.x, drop_c7);
              philox::add_keep_flags(kb, g + 1, w.y, drop_c7);
              philox::add_keep_flags(kb, g + 2, w.z, drop_c7);
              philox::add_keep_flags(kb, g + 3, w.w, drop_c7);
            }
          }
        }
        const int region = kTwoS ? (count & 1) : q;
        const uint32_t t_s = tmem + lane_off + region * 128;
        const uint32_t s_parity = kTwoS ? ((count >> 1) & 1) : (count & 1);
        if (!(ok = mbar_wait_warp(bar_s_full(region), s_parity, ctx))) break;
        tc_fence_after();
        if (!warp_rows) {
          tc_fence_before();
          mbar_arrive(bar_p_full(region));
          ++count;
          continue;
        }
        uint32_t sr[128];
        tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_ld_wait();
        float* s = reinterpret_cast<float*>(sr);

        // Element mask: causal (key > row + Nk - N) and keys past Nk.
        int limit = kBlockN - 1;
        if (p.causal) limit = min(limit, row + (p.Nk - p.N) - j * kBlockN);
        const int kv_left = p.Nk - j * kBlockN - 1;
        if (kv_left < limit) limit = kv_left;
        if (limit < kBlockN - 1) {
#pragma unroll
          for (int c = 0; c < kBlockN; ++c)
            if (c > limit) s[c] = -INFINITY;
        }

        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < kBlockN; c += 4) {
          mx0 = fmaxf(mx0, s[c]);
          mx1 = fmaxf(mx1, s[c + 1]);
          mx2 = fmaxf(mx2, s[c + 2]);
          mx3 = fmaxf(mx3, s[c + 3]);
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;

        if (count == 0) {
          m_ref = mx;
        } else {
          const bool need = mx > m_ref + kRescaleThreshold;
          if (__any_sync(0xffffffffu, need)) {
            if (kTwoS) {
              // P V of the previous tile may still be accumulating into O.
              if (!(ok = mbar_wait_warp(bar_pv_done, (count - 1) & 1, ctx))) break;
              tc_fence_after();
            }
            const float alpha = need ? ex2(m_ref - mx) : 1.0f;
            if (need) {
              l_sum *= alpha;
              m_ref = mx;
            }
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              uint32_t o[32];
              tmem_ld32(t_o + c, o);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(t_o + c, o);
            }
            tmem_st_wait();
          }
        }
        const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;

        float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
#pragma unroll
        for (int c = 0; c < kBlockN; c += 4) {
          s[c] = ex2(fmaf(s[c], sl2, -m_use));
          s[c + 1] = ex2(fmaf(s[c + 1], sl2, -m_use));
          s[c + 2] = ex2(fmaf(s[c + 2], sl2, -m_use));
          s[c + 3] = ex2(fmaf(s[c + 3], sl2, -m_use));
          ls0 += s[c];
          ls1 += s[c + 1];
          ls2 += s[c + 2];
          ls3 += s[c + 3];
        }
        l_sum += (ls0 + ls1) + (ls2 + ls3);

        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) pk[i] = pack2<BF16>(s[2 * i], s[2 * i + 1]);
        if constexpr (kMode == kDropout) {
          // P V uses P o M, M the keep decisions (the sum l above is of the
          // undropped P); the factor 256 / (256 - t) of Z = M * 256 / (256 - t) is
          // applied with 1 / l in the epilogue.
#pragma unroll
          for (int w = 0; w < kBlockN / 4; ++w) {
            uint32_t m01, m23;
            philox::pair_masks(philox::group_flags(kb, w), m01, m23);
            pk[2 * w] &= m01;
            pk[2 * w + 1] &= m23;
          }
        }
        tmem_st32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p_full(region));
        ++count;
      }

      // Epilogue: O / l and lse for the rows of this tile that exist. Each warp
      // rounds its 32 rows into shared memory, in the 128-byte-swizzled layout of a
      // 64-column x 32-row TMA box, and writes them with one TMA store per box;
      // rows past N are clipped by the store. The K/V ring is free by now: every
      // load has landed and the last P V MMA, which read the last V, has completed.
      bool have_o = false;
      if (ok && count > 0) {
        ok = mbar_wait_warp(bar_o_full(q), 0, ctx);
        have_o = ok;
      } else if (ok && tl.len > 0) {
        // No key tile for this query tile (block-sparse): the other tile used them
        // all; its completion frees the K/V ring used for staging.
        ok = mbar_wait_warp(bar_o_full(1 - q), 0, ctx);
      }
      tc_fence_after();
      const size_t row_base = static_cast<size_t>(bh) * p.N;
      const bool row_valid = row >= 0 && row < p.N;
      const float o_scale = kF8 ? p.v_scale : (kMode == kDropout ? p.drop_scale : 1.0f);
      const float inv_l = (l_sum > 0.0f) ? o_scale / l_sum : 0.0f;
      if (kSplit && ok) {
        // Split-KV partial: fp32 O / l of this key range (0 if it has no key for
        // the row) and its lse (-inf then), stored straight from the row's thread.
        const size_t prow = (static_cast<size_t>(split + (dual ? q : 0)) * p.BH + bh) * p.N + row;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          if (have_o) {
            tmem_ld32(t_o + c, o);
            tmem_ld_wait();
          }
          if (row_valid && c < p.d) {
            float4* dst = reinterpret_cast<float4*>(p.o_part + prow * p.d + c);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              float4 v;
              v.x = have_o ? __uint_as_float(o[4 * k]) * inv_l : 0.0f;
              v.y = have_o ? __uint_as_float(o[4 * k + 1]) * inv_l : 0.0f;
              v.z = have_o ? __uint_as_float(o[4 * k + 2]) * inv_l : 0.0f;
              v.w = have_o ? __uint_as_float(o[4 * k + 3]) * inv_l : 0.0f;
              dst[k] = v;
            }
          }
        }
        if (row_valid)
          p.lse_part[prow] = (l_sum > 0.0f) ? (m_ref + lg2(l_sum)) * 0.6931471805599453f : -INFINITY;
      } else if (ok) {
        constexpr uint32_t kBoxBytes = 32 * 128;  // 32 rows x 64 columns x 2 bytes
        const uint32_t stage = smem_u32(sK) + static_cast<uint32_t>(warp - 4) * (D / 64) * kBoxBytes;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          if (have_o) {
            tmem_ld32(t_o + c, o);
            tmem_ld_wait();
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = have_o ? __uint_as_float(o[2 * i]) * inv_l : 0.0f;
            const float b = have_o ? __uint_as_float(o[2 * i + 1]) * inv_l : 0.0f;
            w[i] = pack2<BF16>(a, b);
          }
          // Columns c..c+31 are 16-byte chunks 4*((c/32)%2) .. +3 of the row in box c/64.
          const uint32_t row_addr = stage + static_cast<uint32_t>(c / 64) * kBoxBytes + lane * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t chunk = static_cast<uint32_t>(((c % 64) / 8 + k) ^ (lane & 7));
            sts128(row_addr + chunk * 16, w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int row0 = qt * kBlockM + wq * 32;
        if (lane == 0 && row0 < p.N) {
          // Boxes past the tensor's last column (a padded head dimension) are not
          // stored; a box that straddles it is clipped by the store.
#pragma unroll
          for (int b = 0; b < D / 64; ++b)
            if (b * 64 < p.d) tma_store_3d(&tmap_o, stage + b * kBoxBytes, b * 64, row0, bh);
          bulk_commit_group();
        }
        if (row_valid) {
          const float lse = (l_sum > 0.0f) ? (m_ref + lg2(l_sum)) * 0.6931471805599453f : -INFINITY;
          p.lse[row_base + row] = lse;
        }
      }
    }
    // The stores read shared memory asynchronously: the CTA may exit once they have
    // read it; their global writes complete by themselves before the grid does.
    if (lane == 0) bulk_wait_group_read<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fwd
}  // namespace fa
