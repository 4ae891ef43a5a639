// fa_dropout.cuh - keep masks for dropout on the attention probabilities.
//
// The mask is a pure function of (batch*head, query row, key column, seed, offset),
// so the forward and both backward kernels regenerate the same bits instead of
// storing them. Generator: Philox4x32 with 10 rounds (Salmon, Moraes, Dror and
// Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011). One call covers a
// 4 x 4 block of the score matrix:
//   counter (key column / 4, query row / 4, b * H + h, offset), key (seed low, high);
//   output word w belongs to query row 4 (i / 4) + w, its byte e (least significant
//   first) to key column 4 (j / 4) + e; the element is kept iff that byte is below
//   the keep threshold t (1..256), and kept probabilities are scaled by 256 / t.
//
// A warp's 32 threads hold 32 consecutive rows of a tile (query rows in the forward
// and dQ kernels, key rows in the dK/dV kernel), so each aligned group of four lanes
// shares the 4 x 4 blocks of its four rows: each lane computes a quarter of the
// group's calls and a 4 x 4 exchange of words through shuffles hands every lane the
// bytes of its own row.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

struct DropParams {
  uint32_t seed_lo, seed_hi;  // Philox key
  uint32_t offset;            // fourth counter word (e.g. a step number)
  uint32_t tm1;               // keep threshold minus one: keep iff byte <= tm1
  float rs;                   // 256 / t: scale of the kept probabilities
};

// Ten Philox4x32 rounds on counter c with key (k0, k1); c receives the output.
__device__ __forceinline__ void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c[0]), lo0 = 0xD2511F53u * c[0];
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c[2]), lo1 = 0xCD9E8D57u * c[2];
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
  }
}

// Bit e (0..3) set iff byte e of `word` is kept (<= tm1, replicated in tm1x4).
__device__ __forceinline__ uint32_t keep_nibble(uint32_t word, uint32_t tm1x4) {
  const uint32_t m = __vcmpleu4(word, tm1x4) & 0x01010101u;  // bit 8e = keep byte e
  return ((m * 0x00204081u) >> 21) & 0xFu;                   // gathers bits 0, 8, 16, 24 at 21..24
}

__device__ __forceinline__ uint32_t pick4(const uint32_t (&c)[4], uint32_t idx) {
  return idx == 0 ? c[0] : idx == 1 ? c[1] : idx == 2 ? c[2] : c[3];
}

// Keep bits of the calling thread's QUERY row over 4 NB consecutive key columns,
// which start at key block kb0 (column 4 kb0): bit c of bits[c / 32]. qblk is the
// row's query block (row / 4); the row's index within it must be lane % 4.
template <int NB>
__device__ __forceinline__ void drop_bits_rows(uint32_t (&bits)[NB / 8], uint32_t qblk, uint32_t kb0, uint32_t bh,
                                               const DropParams& dp) {
  const uint32_t lane = lane_id();
  const uint32_t s = lane & 3u;
  const uint32_t tm1x4 = dp.tm1 * 0x01010101u;
#pragma unroll
  for (int x = 0; x < NB / 8; ++x) bits[x] = 0u;
#pragma unroll
  for (int u = 0; u < NB / 4; ++u) {
    uint32_t c[4] = {kb0 + 4u * u + s, qblk, bh, dp.offset};
    philox4x32_10(c, dp.seed_lo, dp.seed_hi);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // Round k: lane s reads lane (s + k) % 4 of its group, which sends the word of
      // the reader's row, (sender - k) % 4, from its block kb0 + 4u + sender.
      const uint32_t send = pick4(c, (s - k) & 3u);
      const uint32_t from = (s + k) & 3u;
      const uint32_t w = k == 0 ? send : __shfl_sync(0xffffffffu, send, (lane & ~3u) | from);
      bits[u >> 1] |= keep_nibble(w, tm1x4) << (16u * (u & 1) + 4u * from);
    }
  }
}

// Keep bits of the calling thread's KEY row over 4 NB consecutive query columns,
// which start at query block qb0 (query 4 qb0): bit c of bits[c / 32]. kblk is the
// key's block (key / 4); the key's index within it must be lane % 4.
template <int NB>
__device__ __forceinline__ void drop_bits_cols(uint32_t (&bits)[NB / 8], uint32_t kblk, uint32_t qb0, uint32_t bh,
                                               const DropParams& dp) {
  const uint32_t lane = lane_id();
  const uint32_t s = lane & 3u;
  const uint32_t tm1x4 = dp.tm1 * 0x01010101u;
#pragma unroll
  for (int x = 0; x < NB / 8; ++x) bits[x] = 0u;
#pragma unroll
  for (int u = 0; u < NB / 4; ++u) {
    uint32_t c[4] = {kblk, qb0 + 4u * u + s, bh, dp.offset};
    philox4x32_10(c, dp.seed_lo, dp.seed_hi);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // The reader's key is byte e = (sender - k) % 4 of every word: gather byte e of
      // words 0..3 (query rows 0..3 of the block) into one word.
      const uint32_t e = (s - k) & 3u;
      const uint32_t sel = e | ((e + 4u) << 4);
      const uint32_t send = __byte_perm(__byte_perm(c[0], c[1], sel), __byte_perm(c[2], c[3], sel), 0x5410u);
      const uint32_t from = (s + k) & 3u;
      const uint32_t w = k == 0 ? send : __shfl_sync(0xffffffffu, send, (lane & ~3u) | from);
      bits[u >> 1] |= keep_nibble(w, tm1x4) << (16u * (u & 1) + 4u * from);
    }
  }
}

// Probabilities pair (x, y) at columns c, c + 1 (c even) after dropout.
__device__ __forceinline__ float2 drop_pair(float x, float y, uint32_t bits_at_c, float rs) {
  return make_float2((bits_at_c & 1u) ? x * rs : 0.f, (bits_at_c & 2u) ? y * rs : 0.f);
}

}  // namespace fa
