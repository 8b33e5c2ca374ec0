// Host launcher of the fused forward kernel.
#include "fa_fwd.cuh"
#include "fa_internal.h"
#include "tma_host.h"

namespace fa {

namespace {

template <int D, bool BF16>
int launch_fwd_t(const AttnArgs& a, cudaStream_t stream) {
  using L = fwd::Smem<D>;
  const int BH = a.B * a.H;
  const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const int Nk = a.Nk > 0 ? a.Nk : a.N;
  CUtensorMap tq, tk, tv, to;
  // O is written by 64-column x 32-row boxes, one per warp and 64 columns.
  bool ok = host::make_map_3d(&tq, dt, 2, a.q, a.d, a.N, BH, 64, fwd::kBlockM, CU_TENSOR_MAP_SWIZZLE_128B) &&
            host::make_map_3d(&tk, dt, 2, a.k, a.d, Nk, BH, 64, fwd::kBlockN, CU_TENSOR_MAP_SWIZZLE_128B) &&
            host::make_map_3d(&tv, dt, 2, a.v, a.d, Nk, BH, 64, fwd::kBlockN, CU_TENSOR_MAP_SWIZZLE_128B) &&
            host::make_map_3d(&to, dt, 2, a.o, a.d, a.N, BH, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return static_cast<int>(cudaErrorInvalidValue);
  fwd::Params p;
  p.o = const_cast<void*>(a.o);
  p.lse = a.lse;
  p.block_mask = a.block_mask;
  p.trace = a.trace;
  p.status = a.status;
  p.N = a.N;
  p.Nk = Nk;
  p.d = a.d;
  p.timeout_ns = a.timeout_ns;
  p.withhold = a.withhold;
  p.n_splits = a.n_splits > 1 || a.o_part != nullptr ? a.n_splits : 1;
  p.o_part = a.o_part;
  p.lse_part = a.lse_part;
  {
    const int tq = (a.N + fwd::kBlockM - 1) / fwd::kBlockM;
    p.dual = (a.o_part != nullptr && tq == 1 && p.n_splits >= 2 && a.block_mask == nullptr && D <= 128) ? 1 : 0;
  }
  p.BH = BH;
  const int Tq = (a.N + fwd::kBlockM - 1) / fwd::kBlockM;
  p.n_pairs = (Tq + L::kQTiles - 1) / L::kQTiles;  // work items per head
  p.Tc = (Nk + fwd::kBlockN - 1) / fwd::kBlockN;
  p.causal = a.causal;
  // Heads per CTA-order group: their K and V (2*N*d*2 bytes each) fit ~48 MB of L2.
  {
    const long long per_head = 4LL * Nk * D;
    long long g = (48LL << 20) / (per_head > 0 ? per_head : 1);
    p.head_group = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
  }
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.drop_t = static_cast<uint32_t>(a.drop_t);
  p.drop_scale = 256.0f / static_cast<float>(256 - a.drop_t);
  p.drop_keys = philox::round_keys(a.drop_seed);
  // d = 256 (a forward-only head dimension) has the plain and split-KV variants.
  constexpr int kDropMode = D == 256 ? fwd::kPlain : fwd::kDropout;
  if (D == 256 && a.drop_t > 0) return static_cast<int>(cudaErrorInvalidValue);
  auto kern = p.o_part != nullptr ? fwd::fa_fwd_kernel<D, BF16, fwd::kSplitKV>
              : a.drop_t > 0      ? fwd::fa_fwd_kernel<D, BF16, kDropMode>
                                  : fwd::fa_fwd_kernel<D, BF16, fwd::kPlain>;
  const int smem_bytes = p.o_part != nullptr ? fwd::Smem<D, false, true>::kAlloc : L::kAlloc;
  cudaError_t e = host::ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem_bytes);
  if (e != cudaSuccess) return static_cast<int>(e);
  const int split_items = p.dual ? (p.n_splits + 1) / 2 : p.n_splits;
  dim3 grid(static_cast<unsigned>(static_cast<long long>(BH) * p.n_pairs * split_items));
  kern<<<grid, fwd::kThreads, smem_bytes, stream>>>(tq, tk, tv, to, p);
  return static_cast<int>(cudaGetLastError());
}

// The 8-bit forward: e4m3 Q, K, V (one byte per element) with per-tensor scales,
// 16-bit (bf16) O; d = 128.
int launch_fwd_fp8_t(const AttnArgs& a, cudaStream_t stream) {
  constexpr int D = 128;
  using L = fwd::Smem<D, true>;
  const int BH = a.B * a.H;
  const int Nk = a.Nk > 0 ? a.Nk : a.N;
  CUtensorMap tq, tk, tv, to;
  // Q and K: one 128-byte-swizzled 128 x 128 box per tile; V: unswizzled rows for
  // the widening warps; O: 16-bit, 64-column x 32-row boxes.
  bool ok = host::make_map_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.q, D, a.N, BH, 128, fwd::kBlockM,
                              CU_TENSOR_MAP_SWIZZLE_128B) &&
            host::make_map_3d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.k, D, Nk, BH, 128, fwd::kBlockN,
                              CU_TENSOR_MAP_SWIZZLE_128B) &&
            host::make_map_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.v, D, Nk, BH, 128, fwd::kBlockN,
                              CU_TENSOR_MAP_SWIZZLE_NONE) &&
            host::make_map_3d(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.o, D, a.N, BH, 64, 32,
                              CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return static_cast<int>(cudaErrorInvalidValue);
  fwd::Params p{};
  p.o = const_cast<void*>(a.o);
  p.lse = a.lse;
  p.block_mask = a.block_mask;
  p.trace = nullptr;
  p.status = a.status;
  p.N = a.N;
  p.Nk = Nk;
  p.d = D;
  p.timeout_ns = a.timeout_ns;
  p.withhold = 0;
  p.n_splits = 1;
  p.BH = BH;
  const int Tq = (a.N + fwd::kBlockM - 1) / fwd::kBlockM;
  p.n_pairs = (Tq + 1) / 2;
  p.Tc = (Nk + fwd::kBlockN - 1) / fwd::kBlockN;
  p.causal = a.causal;
  {
    const long long per_head = 2LL * Nk * D;  // K and V, one byte per element
    long long g = (48LL << 20) / (per_head > 0 ? per_head : 1);
    p.head_group = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
  }
  // S is computed on the stored e4m3 values: the Q and K scales join the softmax
  // scale in the exponent; the V scale multiplies O with 1 / l.
  p.scale_log2 = a.scale * a.q_scale * a.k_scale * 1.4426950408889634f;
  p.v_scale = a.v_scale;
  auto kern = fwd::fa_fwd_kernel<D, true, fwd::kFp8>;
  cudaError_t e = host::ensure_dynamic_smem(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (e != cudaSuccess) return static_cast<int>(e);
  dim3 grid(static_cast<unsigned>(static_cast<long long>(BH) * p.n_pairs));
  kern<<<grid, fwd::kThreads, L::kAlloc, stream>>>(tq, tk, tv, to, p);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_fwd_fp8(const AttnArgs& a, cudaStream_t stream) { return launch_fwd_fp8_t(a, stream); }

// Head dimensions 32 and 96 run in the 64 and 128 kernels: the tensor maps have
// the tensors' d columns, so TMA loads fill columns d..D-1 with zeros (which add
// nothing to S or to P V) and the O stores skip or clip them.
int launch_fwd(const AttnArgs& a, cudaStream_t stream) {
  if (a.d <= 64) return a.dtype == 1 ? launch_fwd_t<64, true>(a, stream) : launch_fwd_t<64, false>(a, stream);
  if (a.d == 256) return a.dtype == 1 ? launch_fwd_t<256, true>(a, stream) : launch_fwd_t<256, false>(a, stream);
  return a.dtype == 1 ? launch_fwd_t<128, true>(a, stream) : launch_fwd_t<128, false>(a, stream);
}

}  // namespace fa
