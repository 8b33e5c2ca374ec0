// Debug launch that writes the dropout draws exactly as the attention kernels
// generate them, in both of their access patterns: row-major (a thread per query
// row: forward and query-stationary backward) and column-major (a thread per
// key: key-stationary backward). Tests compare both with the oracle's draws.
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_internal.h"
#include "philox.cuh"

namespace fa {
namespace {

// Block (jt, it, bh), 128 threads: the 128 x 128 tile of draws at query rows
// 128*it.., keys 128*jt.. of head bh, once through each pattern.
__global__ void __launch_bounds__(128) dropout_draws_kernel(uint8_t* row_major, uint8_t* col_major, int Nq, int Nk,
                                                            const philox::Keys key) {
  const uint32_t bh = blockIdx.z, it = blockIdx.y, jt = blockIdx.x, t = threadIdx.x;
  const size_t head = static_cast<size_t>(bh) * Nq * Nk;
  // Row-major: thread t holds query row 128*it + t.
  const uint32_t row = it * 128 + t;
#pragma unroll 1
  for (uint32_t cg = 0; cg < 32; cg += 4) {
    const uint4 w = philox::draws_row(jt * 32 + cg, row, bh, key);
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t col = jt * 128 + 4 * (cg + k) + b;
        if (row < static_cast<uint32_t>(Nq) && col < static_cast<uint32_t>(Nk))
          row_major[head + static_cast<size_t>(row) * Nk + col] = static_cast<uint8_t>(philox::draw_byte(w, k, b));
      }
  }
  // Column-major: thread t holds key 128*jt + t.
  const uint32_t kc = jt * 128 + t;
#pragma unroll 1
  for (uint32_t rg = 0; rg < 32; rg += 4) {
    const uint4 w = philox::draws_col(it * 32 + rg, kc, bh, key);
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t r = it * 128 + 4 * (rg + k) + b;
        if (r < static_cast<uint32_t>(Nq) && kc < static_cast<uint32_t>(Nk))
          col_major[head + static_cast<size_t>(r) * Nk + kc] = static_cast<uint8_t>(philox::draw_byte(w, k, b));
      }
  }
}

}  // namespace

int launch_dropout_draws(int BH, int Nq, int Nk, uint64_t seed, uint8_t* row_major, uint8_t* col_major,
                         cudaStream_t stream) {
  dim3 grid((Nk + 127) / 128, (Nq + 127) / 128, BH);
  dropout_draws_kernel<<<grid, 128, 0, stream>>>(row_major, col_major, Nq, Nk, philox::round_keys(seed));
  return static_cast<int>(cudaGetLastError());
}

}  // namespace fa
