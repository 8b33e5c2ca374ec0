// Dropout keep decisions for the attention kernels, drawn from the counter-based
// generator Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
// as easy as 1, 2, 3", SC'11), written here from its definition.
//
// Draw layout (the same in the forward and in both backward CTA kinds, so the
// backward regenerates exactly the forward's decisions): one generator block
// covers a 4 x 4 block of (query row i, key column j) of head bh. Its counter
// is (j >> 2, i >> 2, bh, 0), its key (seed low word, seed high word); output
// word (i & 3) holds row i's four draws, byte (j & 3) of it (least significant
// first) is element (i, j)'s draw u in [0, 255]. The element is kept iff
// u >= t, t = round(256 p), and a kept entry of P is scaled by 256 / (256 - t).
//
// The four lanes of a warp that hold four consecutive rows (or keys) all need
// the same blocks. Each of them computes a different one and the words are
// exchanged with four shuffles, so a lane pays one generator block per 16 of
// its elements.
#pragma once

#include <cstdint>

namespace fa {
namespace philox {

__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                               uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

__device__ __forceinline__ uint32_t pick4(const uint4& v, uint32_t k) {
  const uint32_t a = (k & 1u) ? v.y : v.x;
  const uint32_t b = (k & 1u) ? v.w : v.z;
  return (k & 2u) ? b : a;
}

__device__ __forceinline__ void place4(uint4& v, uint32_t k, uint32_t x) {
  v.x = k == 0 ? x : v.x;
  v.y = k == 1 ? x : v.y;
  v.z = k == 2 ? x : v.z;
  v.w = k == 3 ? x : v.w;
}

// Four rounds of exchange inside each group of four lanes: lane a holds `mine`,
// four words meant for lanes 0..3 of its group (word r for lane r); afterwards
// word s of the result is what lane s of the group held for this lane.
__device__ __forceinline__ uint4 exchange4(const uint4& mine) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t a = lane & 3u;
  uint4 out = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (uint32_t k = 0; k < 4; ++k) {
    // Round k: lane a sends its word for lane (a + k) & 3 and receives from lane (a - k) & 3.
    const uint32_t send = pick4(mine, (a + k) & 3u);
    const uint32_t src = (a - k) & 3u;
    const uint32_t got = __shfl_sync(0xffffffffu, send, static_cast<int>((lane & ~3u) | src));
    place4(out, src, got);
  }
  return out;
}

// Row-major use (forward, query-stationary backward): this lane holds query row
// `row`; the four lanes of its group hold rows 4*(row>>2) .. +3. Returns the
// draws of 16 columns, column groups cg0 .. cg0+3 (4 columns each): word k,
// byte b = draw of column 4*(cg0+k)+b in this row.
__device__ __forceinline__ uint4 draws_row(uint32_t cg0, uint32_t row, uint32_t bh, uint32_t k0, uint32_t k1) {
  const uint32_t a = threadIdx.x & 3u;
  // This lane's block: column group cg0 + a, its word r belongs to row 4*(row>>2) + r.
  const uint4 blk = philox4x32_10(cg0 + a, row >> 2, bh, 0u, k0, k1);
  return exchange4(blk);
}

// Column-major use (key-stationary backward): this lane holds key `key`; the
// four lanes of its group hold keys 4*(key>>2) .. +3. Returns the draws of 16
// query rows, row groups rg0 .. rg0+3: word k, byte b = draw of element
// (query row 4*(rg0+k)+b, this key).
__device__ __forceinline__ uint4 draws_col(uint32_t rg0, uint32_t key, uint32_t bh, uint32_t k0, uint32_t k1) {
  const uint32_t a = threadIdx.x & 3u;
  // This lane's block: row group rg0 + a; its word w is query row 4*(rg0+a) + w,
  // byte c of that word is key 4*(key>>2) + c. Lane c of the group needs byte c
  // of each word: transpose the 4 x 4 bytes so word c gathers them.
  const uint4 blk = philox4x32_10(key >> 2, rg0 + a, bh, 0u, k0, k1);
  const uint32_t t01lo = __byte_perm(blk.x, blk.y, 0x5140), t01hi = __byte_perm(blk.x, blk.y, 0x7362);
  const uint32_t t23lo = __byte_perm(blk.z, blk.w, 0x5140), t23hi = __byte_perm(blk.z, blk.w, 0x7362);
  uint4 tr;
  tr.x = __byte_perm(t01lo, t23lo, 0x5410);
  tr.y = __byte_perm(t01lo, t23lo, 0x7632);
  tr.z = __byte_perm(t01hi, t23hi, 0x5410);
  tr.w = __byte_perm(t01hi, t23hi, 0x7632);
  return exchange4(tr);
}

// Byte b of word k of a draws_* result.
__device__ __forceinline__ uint32_t draw_byte(const uint4& w, int k, int b) {
  const uint32_t x = k == 0 ? w.x : (k == 1 ? w.y : (k == 2 ? w.z : w.w));
  return (x >> (8 * b)) & 0xFFu;
}

}  // namespace philox
}  // namespace fa
