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
// its elements. The round keys come from the host (round_keys).
#pragma once

#include <cstdint>

namespace fa {
namespace philox {

// The key words of the ten rounds: round r uses (seed low + r * 0x9E3779B9,
// seed high + r * 0xBB67AE85) mod 2^32. They are computed once on the host and
// read from the kernel parameters, so the rounds spend no instructions on them.
struct Keys {
  uint32_t k[20];  // k[2r], k[2r + 1]: round r
};

__host__ __device__ inline Keys round_keys(uint64_t seed) {
  Keys r;
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int i = 0; i < 10; ++i) {
    r.k[2 * i] = k0;
    r.k[2 * i + 1] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return r;
}

__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, const Keys& key) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ key.k[2 * r];
    const uint32_t n2 = hi0 ^ c3 ^ key.k[2 * r + 1];
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// A 4 x 4 transpose across each group of four lanes: lane a holds `mine`, four
// words meant for lanes 0..3 of its group (word r for lane r); afterwards word s
// of the result is what lane s of the group held for this lane. Two butterfly
// rounds: lanes a and a^1 swap the 2 x 2 blocks' off-diagonal words, then lanes
// a and a^2 swap the off-diagonal 2 x 2 blocks.
__device__ __forceinline__ uint4 exchange4(const uint4& mine) {
  const bool b0 = (threadIdx.x & 1u) != 0;
  const bool b1 = (threadIdx.x & 2u) != 0;
  uint32_t w0 = mine.x, w1 = mine.y, w2 = mine.z, w3 = mine.w;
  // First butterfly step: send word (b0 ^ 1) of each column pair; the partner's arrives in its place.
  uint32_t r0 = __shfl_xor_sync(0xffffffffu, b0 ? w0 : w1, 1);
  uint32_t r1 = __shfl_xor_sync(0xffffffffu, b0 ? w2 : w3, 1);
  w0 = b0 ? r0 : w0;
  w1 = b0 ? w1 : r0;
  w2 = b0 ? r1 : w2;
  w3 = b0 ? w3 : r1;
  // Second butterfly step: send the column pair (b1 ^ 1); the partner's arrives in its place.
  r0 = __shfl_xor_sync(0xffffffffu, b1 ? w0 : w2, 2);
  r1 = __shfl_xor_sync(0xffffffffu, b1 ? w1 : w3, 2);
  w0 = b1 ? r0 : w0;
  w1 = b1 ? r1 : w1;
  w2 = b1 ? w2 : r0;
  w3 = b1 ? w3 : r1;
  return make_uint4(w0, w1, w2, w3);
}

// Row-major use (forward, query-stationary backward): this lane holds query row
// `row`; the four lanes of its group hold rows 4*(row>>2) .. +3. Returns the
// draws of 16 columns, column groups cg0 .. cg0+3 (4 columns each): word k,
// byte b = draw of column 4*(cg0+k)+b in this row.
__device__ __forceinline__ uint4 draws_row(uint32_t cg0, uint32_t row, uint32_t bh, const Keys& key) {
  const uint32_t a = threadIdx.x & 3u;
  // This lane's block: column group cg0 + a, its word r belongs to row 4*(row>>2) + r.
  const uint4 blk = philox4x32_10(cg0 + a, row >> 2, bh, 0u, key);
  return exchange4(blk);
}

// Column-major use (key-stationary backward): this lane holds key `col`; the
// four lanes of its group hold keys 4*(col>>2) .. +3. Returns the draws of 16
// query rows, row groups rg0 .. rg0+3: word k, byte b = draw of element
// (query row 4*(rg0+k)+b, this key).
__device__ __forceinline__ uint4 draws_col(uint32_t rg0, uint32_t col, uint32_t bh, const Keys& key) {
  const uint32_t a = threadIdx.x & 3u;
  // This lane's block: row group rg0 + a; its word w is query row 4*(rg0+a) + w,
  // byte c of that word is key 4*(col>>2) + c. Lane c of the group needs byte c
  // of each word: transpose the 4 x 4 bytes so word c gathers them.
  const uint4 blk = philox4x32_10(col >> 2, rg0 + a, bh, 0u, key);
  const uint32_t t01lo = __byte_perm(blk.x, blk.y, 0x5140), t01hi = __byte_perm(blk.x, blk.y, 0x7362);
  const uint32_t t23lo = __byte_perm(blk.z, blk.w, 0x5140), t23hi = __byte_perm(blk.z, blk.w, 0x7362);
  uint4 tr;
  tr.x = __byte_perm(t01lo, t23lo, 0x5410);
  tr.y = __byte_perm(t01lo, t23lo, 0x7632);
  tr.z = __byte_perm(t01hi, t23hi, 0x5410);
  tr.w = __byte_perm(t01hi, t23hi, 0x7632);
  return exchange4(tr);
}

// Keep decisions of four draws (bytes 0..3 of x, four consecutive keys of a row):
// byte k of the result is 0xFF where draw k >= t (kept) and 0 where it is below
// (dropped). c7 = keep_bias(t).
//
// Byte u >= t exactly when u + 256 - t reaches 256: the even bytes, then the odd
// ones, are spread to the top of 16-bit lanes (u << 7) and added to (256 - t) << 7,
// which sets bit 15 of the lane exactly for kept bytes (no carry crosses a lane:
// u + 256 - t < 512). prmt's sign-replicating selectors (nibble 8 | i: the sign
// bit of input byte i over the whole result byte) gather the four bits.
__host__ __device__ __forceinline__ uint32_t keep_bias(uint32_t t) { return ((256u - t) << 7) * 0x10001u; }

__device__ __forceinline__ uint32_t keep_bytes(uint32_t x, uint32_t c7) {
  const uint32_t even = ((x & 0x00FF00FFu) << 7) + c7;  // keys 0, 2 -> bits 15, 31
  const uint32_t odd = ((x >> 1) & 0x7F807F80u) + c7;   // keys 1, 3 -> bits 15, 31
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, 0xFBD9;" : "=r"(r) : "r"(even), "r"(odd));
  return r;
}

// Keep flags of a row (or key) against 4G consecutive keys (or rows), G groups of
// four: group g is bit 7 - g % 8 of the four bytes of word g / 8, byte k for its
// element k. add_keep_flags puts the flags of group g, from its draws word x, in.
__device__ __forceinline__ void add_keep_flags(uint32_t* kb, int g, uint32_t x, uint32_t c7) {
  kb[g / 8] |= keep_bytes(x, c7) & (0x80808080u >> (g % 8));
}

// Group g's flags with the bit of each byte moved to its top.
__device__ __forceinline__ uint32_t group_flags(const uint32_t* kb, int g) { return kb[g / 8] << (g % 8); }

// All ones where element b of a group is kept, zero where it is dropped (flags
// from group_flags).
template <int b>
__device__ __forceinline__ uint32_t elem_mask(uint32_t flags) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %1, %2;" : "=r"(r) : "r"(flags), "n"((8 | b) * 0x1111));
  return r;
}

// Masks for two packed 16-bit pairs from a word whose byte k has keep(key k) in
// its top bit: m01 covers keys 0 and 1, m23 keys 2 and 3; each half is 0xFFFF for
// a kept key and 0 for a dropped one, so a pair is dropped with one AND.
__device__ __forceinline__ void pair_masks(uint32_t flags, uint32_t& m01, uint32_t& m23) {
  asm("prmt.b32 %0, %1, %1, 0x9988;" : "=r"(m01) : "r"(flags));
  asm("prmt.b32 %0, %1, %1, 0xBBAA;" : "=r"(m23) : "r"(flags));
}

// Byte b of word k of a draws_* result.
__device__ __forceinline__ uint32_t draw_byte(const uint4& w, int k, int b) {
  const uint32_t x = k == 0 ? w.x : (k == 1 ? w.y : (k == 2 ? w.z : w.w));
  return (x >> (8 * b)) & 0xFFu;
}

}  // namespace philox
}  // namespace fa
