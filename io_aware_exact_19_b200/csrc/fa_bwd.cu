// Host launchers of the backward: prep (D and lse in log2 units) and the main
// kernel (key-stationary dK/dV CTAs and query-stationary dQ CTAs in one grid).
#include "fa_bwd.cuh"
#include "fa_internal.h"
#include "tma_host.h"

namespace fa {

int bwd_row_tile(int) { return bwd::kBR; }

BwdWorkspace bwd_workspace_layout(int B, int H, int N, int) {
  BwdWorkspace w{};
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  w.delta = 0;
  w.lse2 = up(bh * npad * 4);
  w.total = w.lse2 + up(bh * npad * 4);
  return w;
}

namespace {

template <int D, bool BF16>
int launch_bwd_t(const AttnArgs& a, cudaStream_t stream) {
  using C = bwd::Cfg<D>;
  const int BH = a.B * a.H;
  const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const BwdWorkspace ws = bwd_workspace_layout(a.B, a.H, a.N, D);
  uint8_t* base = static_cast<uint8_t*>(a.workspace);

  bwd::Params p;
  p.q = a.q;
  p.o = a.o;
  p.dout = a.dout;
  p.lse = a.lse;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.delta = reinterpret_cast<float*>(base + ws.delta);
  p.lse2 = reinterpret_cast<float*>(base + ws.lse2);
  p.block_mask = a.block_mask;
  p.trace = a.trace;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.withhold = a.withhold;
  p.drop_t = static_cast<uint32_t>(a.drop_t);
  p.drop_scale = 256.0f / static_cast<float>(256 - a.drop_t);
  p.drop_keys = philox::round_keys(a.drop_seed);
  const int Nk = a.Nk > 0 ? a.Nk : a.N;
  p.N = a.N;
  p.Nk = Nk;
  p.d = a.d;
  p.Npad = (a.N + 127) / 128 * 128;
  p.BH = BH;
  p.Tq = (a.N + 127) / 128;
  p.Tk = (Nk + 127) / 128;
  p.causal = a.causal;
  p.scale = a.scale;
  // Heads per CTA-order group: their Q, dO (N*d*2 bytes each) and K, V (Nk*d*2
  // bytes each) fit ~48 MB of L2.
  {
    const long long per_head = 4LL * (a.N + Nk) * D;
    long long g = (48LL << 20) / (per_head > 0 ? per_head : 1);
    p.head_group = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
  }
  p.scale_log2 = a.scale * 1.4426950408889634f;

  // prep: blocks of kPrepRows<D> padded rows (a divisor of 128, so of Npad).
  if (a.phases & 1) {
    static_assert(128 % bwd::kPrepRows<D> == 0, "prep rows per block must divide the row padding");
    const long long blocks = static_cast<long long>(BH) * p.Npad / bwd::kPrepRows<D>;
    bwd::fa_bwd_prep_kernel<D, BF16><<<static_cast<unsigned>(blocks), bwd::kPrepThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  // main
  if (a.phases & 2) {
    CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
    // Q and dO are read by key-stationary CTAs in 128-row tiles, loaded as two
    // 64-row boxes per 64-column chunk. dK, dV and dQ are written by each warp in
    // 32-row boxes: 64 columns with the 128-byte swizzle, or (dQ at d = 64, where
    // a warpgroup owns 32 columns) 32 columns unswizzled.
    const bool dq64 = D / 2 >= 64;
    bool ok = host::make_map_3d(&tq, dt, 2, a.q, a.d, a.N, BH, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              host::make_map_3d(&tdo, dt, 2, a.dout, a.d, a.N, BH, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              host::make_map_3d(&tk, dt, 2, a.k, a.d, Nk, BH, 64, bwd::kBlockN, CU_TENSOR_MAP_SWIZZLE_128B) &&
              host::make_map_3d(&tv, dt, 2, a.v, a.d, Nk, BH, 64, bwd::kBlockN, CU_TENSOR_MAP_SWIZZLE_128B) &&
              host::make_map_3d(&tdk, dt, 2, a.dk, a.d, Nk, BH, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B) &&
              host::make_map_3d(&tdv, dt, 2, a.dv, a.d, Nk, BH, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B) &&
              host::make_map_3d(&tdq, dt, 2, a.dq, a.d, a.N, BH, dq64 ? 64 : 32, 32,
                                dq64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return static_cast<int>(cudaErrorInvalidValue);
    auto kern = a.drop_t > 0 ? bwd::fa_bwd_main_kernel<D, BF16, true> : bwd::fa_bwd_main_kernel<D, BF16, false>;
    cudaError_t e = host::ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::kAlloc);
    if (e != cudaSuccess) return static_cast<int>(e);
    dim3 grid(static_cast<unsigned>(BH) * static_cast<unsigned>(p.Tq + p.Tk));
    kern<<<grid, bwd::kThreads, C::kAlloc, stream>>>(tq, tk, tv, tdo, tdq, tdk, tdv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  return 0;
}

}  // namespace

// Head dimensions 32 and 96 run in the 64 and 128 kernels: the tensor maps have
// the tensors' d columns, so TMA loads fill columns d..D-1 with zeros (which add
// nothing to any product) and stores clip them.
int launch_bwd(const AttnArgs& a, cudaStream_t stream) {
  if (a.d <= 64) return a.dtype == 1 ? launch_bwd_t<64, true>(a, stream) : launch_bwd_t<64, false>(a, stream);
  return a.dtype == 1 ? launch_bwd_t<128, true>(a, stream) : launch_bwd_t<128, false>(a, stream);
}

}  // namespace fa
