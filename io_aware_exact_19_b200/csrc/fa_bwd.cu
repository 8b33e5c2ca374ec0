// Host launcher of the backward kernels (placeholder until the kernels land).
#include "fa_internal.h"

namespace fa {

int bwd_row_tile(int d) { return d == 128 ? 64 : 128; }

BwdWorkspace bwd_workspace_layout(int B, int H, int N, int d) {
  BwdWorkspace w{};
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  w.dq_acc = 0;
  w.delta = up(bh * N * d * 4);
  w.lse2 = w.delta + up(bh * npad * 4);
  w.total = w.lse2 + up(bh * npad * 4);
  return w;
}

int launch_bwd(const AttnArgs&, cudaStream_t) { return static_cast<int>(cudaErrorNotSupported); }

}  // namespace fa
