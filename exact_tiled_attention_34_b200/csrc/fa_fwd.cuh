// fa_fwd.cuh - forward kernel: exact attention with online softmax on sm_100a.
//
// Method: "FlashAttention-2: Faster Attention with Better Parallelism and Work
// Partitioning" (paper review), "Proposed method": online-softmax tiling, fewer
// non-matmul FLOPs, parallelism over sequence length, work split between warps,
// causal masking by skipping tiles; "Researchers at Stanford University Propose
// FlashAttention ..." (summary), method paragraph: blocks of Q, K, V processed in
// on-chip memory with the softmax reduced progressively, the normalisation factor
// saved for the backward.
//
// The kernel is persistent: one CTA per SM walks a static list of work items, each a
// block of 2 x 128 query rows (two Q tiles) of one (batch, head), streaming the
// 128-key K/V tiles the block needs through a shared-memory ring that runs on
// across items (as do the barrier phases), so that the next item's Q load and first
// S products overlap the previous item's last products and epilogue:
//   warp 0      TMA producer (one elected thread): Q once, then K_j, V_j per tile
//   warp 1      MMA issuer (one thread) + TMEM allocator (whole warp)
//   warps 4-7   softmax warpgroup for Q tile 0 (thread = query row = TMEM lane)
//   warps 8-11  softmax warpgroup for Q tile 1
// Tensor memory (512 columns): S0 | S1 | O0 | O1 (fp32), with the bf16 P_i written
// over S_i (head dim 128) or into spare columns (head dim 64). The MMA warp
// alternates between the two tiles so that the softmax of one tile overlaps the
// matrix products of the other.
//
// Online softmax per row (base-2, scale folded into c = scale * log2 e):
//   m' = max(m, c * max_j s_j); P_j = 2^(c s_j - m'); l = l 2^(m - m') + sum P_j;
//   O = O 2^(m - m') + P V;  at the end O /= l, lse = (m + log2 l) ln 2.
// The rescale of O in TMEM is skipped unless some row of the warp raised its max by
// more than 8 (P then stays <= 2^8): the final O / l and lse use the same reference
// max, so skipping is exact (a deferred normalisation).
#pragma once

#include <type_traits>

#include "fa_dropout.cuh"
#include "fa_ptx.cuh"

namespace fa {

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  const uint8_t* tile_mask;  // [nT, nT] or nullptr
  int* status;               // library status word (global)
  unsigned long long timeout_ns;
  int stall;                 // test hook: 1 = the producer issues no copies, so every wait runs out
  int N;                     // query rows N_q (any N >= 1)
  int Nk;                    // key rows N_k (any N_k >= 1)
  int BH;                    // B * H
  int H;                     // heads (item bh = b * H + h)
  int bnhd;                  // 1: q, k, v, o are [B, N, H, d]; 0: [B, H, N, d] (lse is [B, H, N] either way)
  int v8;                    // 1: o is 32-byte aligned (32-byte row stores)
  int n_tiles;               // query tiles ceil(N_q / 128); the last may be partial
  int n_ktiles;              // key tiles ceil(N_k / 128)
  int off;                   // N_k - N_q: with the causal mask key j is visible to query i iff j <= i + off
  int n_qblocks;             // ceil(n_tiles / 2)
  int n_items;               // n_qblocks * BH work items (query block, batch*head)
  float c_log2;              // scale * log2(e)
  // Merging kernels (MERGE): the running result of earlier key blocks, updated in place
  // (fp32 [BH, N, D] and [BH, N]); o and lse above are then not written.
  float* o_acc;
  float* lse_acc;
};

// The dropout kernels' parameters (the others keep the plain block unchanged).
struct FwdParamsDrop : FwdParams {
  DropParams drop;
};
template <bool DROP>
using FwdParamsT = std::conditional_t<DROP, FwdParamsDrop, FwdParams>;

template <int D>
struct FwdCfg {
  static constexpr int kRows = 128;                   // rows per Q tile and per K/V tile
  static constexpr int kColBlocks = D / 64;           // 128-byte column blocks per row
  static constexpr int kBlockBytes = kRows * 128;     // one column block of a tile
  static constexpr int kTileBytes = kRows * D * 2;    // one bf16 tile
  static constexpr int kStages = (D == 64) ? 3 : 2;   // K/V ring depth
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  // Head dim 128: each softmax warp stages its O rows (4 KB per warp) so that the
  // epilogue writes whole 128-byte lines (measured 2-4% faster there; no gain at 64).
  static constexpr bool kStageO = (D == 128);
  static constexpr int kOffStage = kOffV + kStages * kTileBytes;
  static constexpr int kOffBar = kOffStage + (kStageO ? 8 * 4096 : 0);
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // barriers + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "forward shared memory above the per-block limit");
  static constexpr int kThreads = 384;
  // TMEM columns
  __host__ __device__ static constexpr uint32_t tm_s(int i) { return i ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t tm_o(int i) { return 256u + (i ? uint32_t(D) : 0u); }
  __host__ __device__ static constexpr uint32_t tm_p(int i) {
    return D == 64 ? (i ? 448u : 384u) : tm_s(i);  // spare columns, or over S_i
  }
  static constexpr uint32_t kTmCols = 512;
};

// Barrier block in shared memory.
template <int S>
struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[S];
  uint64_t v_full[S];
  uint64_t kv_empty[S];
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t o_full[2];
  uint64_t o_empty[2];   // the softmax warpgroup has read O_i (the next item may overwrite it)
  uint64_t q_empty;      // the item's S products are done with the Q tiles
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// Persistent schedule: the k-th work item of this CTA, or false when it has none.
// Without the causal mask all items cost the same and go head-major (the query blocks
// of one head together, sharing its K/V tiles through L2). With it, a block's cost
// grows with its index, and items go longest first across all heads (block-major),
// which with the alternating deal of item_position balances the CTAs' work.
struct FwdItem {
  int bh, qb;
};
template <bool CAUSAL>
__device__ __forceinline__ bool fwd_item(int n_items, int n_qblocks, int BH, int k, FwdItem& it) {
  const long long pos = item_position(n_items, k);
  if (pos < 0) return false;
  if (CAUSAL) {
    it.qb = n_qblocks - 1 - static_cast<int>(pos / BH);
    it.bh = static_cast<int>(pos % BH);
  } else {
    it.bh = static_cast<int>(pos / n_qblocks);
    it.qb = n_qblocks - 1 - static_cast<int>(pos % n_qblocks);
  }
  return true;
}

// Last key tile that query tile t sees with the causal mask (key j visible to query i
// iff j <= i + off), clamped to the key tiles; -1 when the tile sees no key.
__device__ __forceinline__ int causal_klast(int t, int off, int n_ktiles) {
  const long long x = 128LL * t + 127 + off;  // last key the tile's last row sees
  const long long l = x < 0 ? -1 : (x >> 7);
  return static_cast<int>(l < n_ktiles - 1 ? l : n_ktiles - 1);
}

// Which of the CTA's two Q tiles need K/V tile j (bit 0: tile 0, bit 1: tile 1); the
// K/V tiles are visited in increasing order. (Visiting the causal tiles diagonal-first,
// or tile 1's extra diagonal tile earlier, was measured: up to 6% faster at N = 2048 but
// 1-2% slower at N >= 8192, so the plain order stays.)
template <bool CAUSAL, bool SPARSE, bool XQK>
struct FwdSched {
  int t0, t1;
  bool valid1;
  int n_ktiles;
  int klast0, klast1;  // causal with N_q != N_k (XQK): last key tile of Q tile 0 / 1
  const uint8_t* mask;
  // With N_q = N_k the causal limit of Q tile t is key tile t (its diagonal).
  __device__ __forceinline__ int kl0() const { return XQK ? klast0 : t0; }
  __device__ __forceinline__ int kl1() const { return XQK ? klast1 : t1; }
  __device__ __forceinline__ int last() const { return CAUSAL ? (valid1 ? kl1() : kl0()) : n_ktiles - 1; }
  __device__ __forceinline__ uint32_t bits(int j) const {
    bool k0 = CAUSAL ? (j <= kl0()) : true;
    bool k1 = valid1 && (CAUSAL ? (j <= kl1()) : true);
    if (SPARSE) {
      k0 = k0 && (mask[size_t(t0) * n_ktiles + j] != 0);
      k1 = k1 && (mask[size_t(t1) * n_ktiles + j] != 0);
    }
    return (k0 ? 1u : 0u) | (k1 ? 2u : 0u);
  }
  // The K/V tile visited after j0 with a non-empty bit set (or -1).
  __device__ __forceinline__ int next(int j0, uint32_t& b) const {
    const int jl = last();
    for (int j = j0 + 1; j <= jl; ++j) {
      b = bits(j);
      if (b) return j;
    }
    b = 0;
    return -1;
  }
  __device__ __forceinline__ int first(uint32_t& b) const { return next(-1, b); }
};

// Wait-site codes reported through the status word (detail field).
enum FwdSite : int {
  kSiteFwdQ = 101, kSiteFwdKvEmpty, kSiteFwdKFull, kSiteFwdVFull, kSiteFwdPReady, kSiteFwdSFull,
  kSiteFwdOFull, kSiteFwdDrain, kSiteFwdQEmpty, kSiteFwdOEmpty
};

// One softmax step for the calling thread's row: s[0..127] are the raw scores of
// the current K/V tile; m is the running (base-2, scaled) reference max. Writes the
// bf16 probabilities into TMEM at tp (64 columns of packed pairs), returns the row
// sum of this tile, the factor alpha = 2^(m - m_use) for the old O and l, and the new
// reference max m_use. The rescale decision is warp-uniform (see the file header).
// Pairs of columns go through packed f32x2 arithmetic; the exponentials are split
// between the special-function unit and a polynomial on the FMA pipe.
// MASK: only columns t < lim are visible, for the tile on the causal diagonal
// (lim = r + 1) or the last K/V tile of a sequence whose length is not a multiple of
// 128 (lim = number of keys in it).
// DROP: the probabilities written for P V are dropped where bit t of kb is clear and
// scaled by rs where it is set; the returned sum is that of the undropped row.
template <bool MASK, int POLY8, bool DROP = false>
__device__ __forceinline__ void softmax_row(float (&s)[128], int lim, float c, float m, uint32_t tp, float& sum,
                                            float& alpha, float& m_use, const uint32_t (&kb)[4], float rs) {
  // Four independent accumulators keep the reduction chains short.
  float mx;
  if (c >= 0.f) {
    float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int t = 0; t < 128; t += 2)
      a[(t >> 1) & 3] = max3f(a[(t >> 1) & 3], (MASK && t >= lim) ? -INFINITY : s[t],
                              (MASK && t + 1 >= lim) ? -INFINITY : s[t + 1]);
    mx = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])) * c;
  } else {
    float a[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll
    for (int t = 0; t < 128; t += 2)
      a[(t >> 1) & 3] = min3f(a[(t >> 1) & 3], (MASK && t >= lim) ? INFINITY : s[t],
                              (MASK && t + 1 >= lim) ? INFINITY : s[t + 1]);
    mx = fminf(fminf(a[0], a[1]), fminf(a[2], a[3])) * c;
  }
  const float m_new = fmaxf(m, mx);
  const bool rescale = __any_sync(0xffffffffu, m_new > m + 8.f);
  m_use = rescale ? m_new : m;
  const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
  alpha = ex2(m - m_sub);  // 0 on the first tile (m = -inf), 1 when the max is kept
  const uint64_t c2 = f2(c, c), nm2 = f2(-m_sub, -m_sub);
  uint64_t acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const int c0 = h * 64 + 2 * t;
      const uint64_t x = f2_fma(f2(s[c0], s[c0 + 1]), c2, nm2);
      uint64_t pv = ex2_split_x2<POLY8>(x, t);
      if (MASK) {
        const float2 v = f2_split(pv);
        pv = f2((c0 >= lim) ? 0.f : v.x, (c0 + 1 >= lim) ? 0.f : v.y);
      }
      acc[t & 3] = f2_add(acc[t & 3], pv);
      const float2 v = f2_split(pv);
      if constexpr (DROP) {
        const float2 w = drop_pair(v.x, v.y, kb[c0 >> 5] >> (c0 & 31), rs);
        pk[t] = pack_bf16(w.x, w.y);
      } else {
        pk[t] = pack_bf16(v.x, v.y);
      }
    }
    tmem_st32(tp + h * 32, pk);
  }
  const float2 a = f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])));
  sum = a.x + a.y;
}

// Register split of the 384-thread forward block (launched with 168 per thread,
// 64,512 in all): the producer/MMA warpgroup drops to 88, the two softmax
// warpgroups rise to 208 -> 128 * (88 + 2 * 208) = 64,512. Only the softmax
// warpgroups increase, once, by what the first warpgroup releases.
constexpr int kFwdRegsCtl = 88;
constexpr int kFwdRegsSoftmax = 208;
constexpr int kFwdRegsNeeded = 128 * (kFwdRegsCtl + 2 * kFwdRegsSoftmax);

// DS: the head dim as stored (row length of q, k, v, o): D, or 96 on the D = 128 kernels
// (the loads read zeros for columns 96..127; only DS columns of O are written).
// DROP: dropout on the probabilities that multiply V (keep masks regenerated per tile).
// MERGE: this call's keys are one block of a longer key sequence: the epilogue merges the
// block's result into a running fp32 (O_acc, lse_acc) through their log-sum-exp, with no
// bf16 rounding of the block's partial O (the online softmax's combination, one level up).
template <int D, bool CAUSAL, bool SPARSE, bool XQK, int DS, bool DROP = false, bool MERGE = false>
__global__ void __launch_bounds__(384, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdParamsT<DROP> p) {
  using Cfg = FwdCfg<D>;
  constexpr int S = Cfg::kStages;
  // Causal offset N_k - N_q: a compile-time 0 in the N_q = N_k kernels (XQK false).
  const int off_ = XQK ? p.off : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  FwdBars<S>* bars = reinterpret_cast<FwdBars<S>*>(smem + Cfg::kOffBar);
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sK = smem + Cfg::kOffK;
  uint8_t* sV = smem + Cfg::kOffV;
  uint32_t* sStage = reinterpret_cast<uint32_t*>(smem + Cfg::kOffStage);

  const int warp = warp_id();
  const int lane = lane_id();
  auto sched_of = [&](const FwdItem& item) {
    FwdSched<CAUSAL, SPARSE, XQK> sch;
    sch.t0 = 2 * item.qb;
    sch.t1 = 2 * item.qb + 1;
    sch.valid1 = sch.t1 < p.n_tiles;
    sch.n_ktiles = p.n_ktiles;
    sch.klast0 = XQK ? causal_klast(sch.t0, off_, p.n_ktiles) : 0;
    sch.klast1 = XQK ? causal_klast(sch.t1, off_, p.n_ktiles) : 0;
    sch.mask = p.tile_mask;
    return sch;
  };

  WaitCtl wc{&bars->abort, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_ready[i], 128);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_empty[i], 128);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, Cfg::kTmCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    regs_dec<kFwdRegsCtl>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t keep = policy_evict_last();
      int it = 0;   // K/V tiles loaded so far (ring position, continues across items)
      int nq = 0;   // Q blocks loaded so far
      bool ok = p.stall == 0;
      FwdItem item;
      for (int k = 0; ok && fwd_item<CAUSAL>(p.n_items, p.n_qblocks, p.BH, k, item); ++k) {
        const auto sch = sched_of(item);
        const int ib = item.bh / p.H, ih = item.bh - ib * p.H;  // batch, head (tensor-map coordinates)
        // The previous item's S products must be done with the Q buffer.
        if (k > 0 && !mbar_wait(&bars->q_empty, (k - 1) & 1, wc, kSiteFwdQEmpty)) break;
        mbar_arrive_expect_tx(&bars->q_full, Cfg::kTileBytes * (sch.valid1 ? 2 : 1));
        for (int cb = 0; cb < Cfg::kColBlocks; ++cb)
          tma_load_4d(sQ + cb * Cfg::kBlockBytes, &tm_q, &bars->q_full, cb * 64, sch.t0 * 128, ih, ib);
        if (sch.valid1)
          for (int cb = 0; cb < Cfg::kColBlocks; ++cb)
            tma_load_4d(sQ + Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_q, &bars->q_full, cb * 64,
                        sch.t1 * 128, ih, ib);
        ++nq;
        uint32_t b;
        for (int j = sch.first(b); j >= 0; j = sch.next(j, b), ++it) {
          const int st = it % S;
          const int n = it / S;
          if (n > 0 && !mbar_wait(&bars->kv_empty[st], (n - 1) & 1, wc, kSiteFwdKvEmpty)) {
            ok = false;
            break;
          }
          uint8_t* dk = sK + st * Cfg::kTileBytes;
          uint8_t* dv = sV + st * Cfg::kTileBytes;
          mbar_arrive_expect_tx(&bars->k_full[st], Cfg::kTileBytes);
          for (int cb = 0; cb < Cfg::kColBlocks; ++cb)
            tma_load_4d_hint(dk + cb * Cfg::kBlockBytes, &tm_k, &bars->k_full[st], cb * 64, j * 128, ih, ib,
                             keep);
          mbar_arrive_expect_tx(&bars->v_full[st], Cfg::kTileBytes);
          for (int cb = 0; cb < Cfg::kColBlocks; ++cb)
            tma_load_4d_hint(dv + cb * Cfg::kBlockBytes, &tm_v, &bars->v_full[st], cb * 64, j * 128, ih, ib,
                             keep);
        }
      }
      // On abort, wait (bounded) for this thread's own copies still in flight.
      if (bars->abort) {
        if (nq > 0) mbar_wait_drain(&bars->q_full, (nq - 1) & 1, wc, kSiteFwdDrain);
        for (int x = (it > S ? it - S : 0); x < it; ++x) {
          mbar_wait_drain(&bars->k_full[x % S], (x / S) & 1, wc, kSiteFwdDrain);
          mbar_wait_drain(&bars->v_full[x % S], (x / S) & 1, wc, kSiteFwdDrain);
        }
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kFwdRegsCtl>();
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);  // S = Q K^T, both K-major
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);    // O += P V, V is N-major
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      auto issue_s = [&](int i, int st) {
        const uint32_t qa = sQa + i * Cfg::kTileBytes;
        const uint32_t ka = sKa + st * Cfg::kTileBytes;
#pragma unroll
        for (int k = 0; k < DS / 16; ++k) {  // head dim 96: columns 96..127 of the tiles are zeros
          const uint32_t off = (k >> 2) * Cfg::kBlockBytes + (k & 3) * 32;
          mma_ss(tmem + Cfg::tm_s(i), sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), idS,
                 k > 0);
        }
      };
      auto issue_pv = [&](int i, int st, bool acc) {
        const uint32_t va = sVa + st * Cfg::kTileBytes;
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k) {
          mma_ts(tmem + Cfg::tm_o(i), tmem + Cfg::tm_p(i) + k * 8,
                 sdesc_sw128(va + k * 16 * 128, Cfg::kBlockBytes, 1024), idO, (acc || k > 0) ? 1u : 0u);
        }
      };
      bool ok = true;
      int it = 0;               // K/V ring position (continues across items)
      int cnt[2] = {0, 0};      // S_i / P_i handshakes so far (continue across items)
      FwdItem item;
      for (int kk = 0; ok && fwd_item<CAUSAL>(p.n_items, p.n_qblocks, p.BH, kk, item); ++kk) {
        const auto sch = sched_of(item);
        if (!mbar_wait(&bars->q_full, kk & 1, wc, kSiteFwdQ)) { ok = false; break; }
        tc_fence_after();
        uint32_t issued = 0;
        bool first_pv[2] = {true, true};
        uint32_t b = 0, bn = 0;
        int j = sch.first(b);
        if (j < 0) mma_commit(&bars->q_empty);  // nothing to do for this block
        while (j >= 0) {
          const int st = it % S;
          const uint32_t ph = (it / S) & 1;
          const int jn = sch.next(j, bn);
          const int stn = (it + 1) % S;
          const uint32_t phn = ((it + 1) / S) & 1;
          const uint32_t need = b & ~issued;
          if (need) {
            if (!mbar_wait(&bars->k_full[st], ph, wc, kSiteFwdKFull)) { ok = false; break; }
            tc_fence_after();
            for (int i = 0; i < 2; ++i)
              if (need & (1u << i)) {
                issue_s(i, st);
                mma_commit(&bars->s_full[i]);
              }
          }
          // With a block mask the two Q tiles often need different K/V tiles: a tile with
          // no work on this K/V tile but some on the next one gets its next S now, so
          // that its softmax overlaps the other tile's (measured +17% at 25% density).
          // Without a mask both tiles need every K/V tile, and with the causal mask only
          // the last K/V tile of a block is for one tile alone.
          const uint32_t ahead = (SPARSE && jn >= 0) ? (bn & ~b) : 0u;
          if (ahead) {
            if (!mbar_wait(&bars->k_full[stn], phn, wc, kSiteFwdKFull)) { ok = false; break; }
            tc_fence_after();
            for (int i = 0; i < 2; ++i)
              if (ahead & (1u << i)) {
                issue_s(i, stn);
                mma_commit(&bars->s_full[i]);
              }
          }
          // Every S product of this item has now been issued: release Q when they finish.
          if (jn < 0) mma_commit(&bars->q_empty);
          if (!mbar_wait(&bars->v_full[st], ph, wc, kSiteFwdVFull)) { ok = false; break; }
          tc_fence_after();
          uint32_t next_issued = 0;
          for (int i = 0; i < 2; ++i) {
            if (!(b & (1u << i))) continue;
            if (!mbar_wait(&bars->p_ready[i], cnt[i] & 1, wc, kSiteFwdPReady)) { ok = false; break; }
            // The first P.V of an item overwrites O_i: the previous item's epilogue must
            // have read it.
            if (first_pv[i] && kk > 0 && !mbar_wait(&bars->o_empty[i], (kk - 1) & 1, wc, kSiteFwdOEmpty)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(i, st, !first_pv[i]);
            first_pv[i] = false;
            ++cnt[i];
            if (jn >= 0 && (bn & (1u << i))) {
              if (!mbar_wait(&bars->k_full[stn], phn, wc, kSiteFwdKFull)) { ok = false; break; }
              tc_fence_after();
              issue_s(i, stn);
              mma_commit(&bars->s_full[i]);
              next_issued |= 1u << i;
            }
          }
          if (!ok) break;
          mma_commit(&bars->kv_empty[st]);
          issued = next_issued | ahead;
          b = bn;
          j = jn;
          ++it;
        }
        if (!ok) break;
        mma_commit(&bars->o_full[0]);
        mma_commit(&bars->o_full[1]);
      }
      // Every MMA issued by this thread must finish before TMEM is released.
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, wc, kSiteFwdDrain);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmCols);
  } else if (warp < 4) {
    // idle warps of the first warpgroup: they take part in its register hand-over
    regs_dec<kFwdRegsCtl>();
    __syncthreads();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    regs_inc<kFwdRegsSoftmax>();
    const int i = (warp - 4) >> 2;  // Q tile of this warpgroup
    const int quarter = warp & 3;   // TMEM lane quarter
    const int r = quarter * 32 + lane;
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    const float c = p.c_log2;
    float drop_rs = 1.f;  // scale of the kept probabilities
    if constexpr (DROP) drop_rs = p.drop.rs;
    int cnt = 0;  // S_i tiles consumed so far (continues across items)
    bool ok = true;
    FwdItem item;
    for (int kk = 0; ok && fwd_item<CAUSAL>(p.n_items, p.n_qblocks, p.BH, kk, item); ++kk) {
      const auto sch = sched_of(item);
      const int tile = i == 0 ? sch.t0 : sch.t1;
      const bool active = (i == 0) || sch.valid1;
      float m = -INFINITY, l = 0.f;
      int local = 0;  // tiles of this item
      if (active) {
        uint32_t b;
        for (int j = sch.first(b); j >= 0; j = sch.next(j, b)) {
          if (!(b & (1u << i))) continue;
          // Keep bits of this row over key tile j, drawn while S is being computed.
          uint32_t kb[4] = {0u, 0u, 0u, 0u};
          if constexpr (DROP)
            drop_bits_rows<32>(kb, uint32_t(tile * 32 + quarter * 8 + (lane >> 2)), uint32_t(j * 32),
                               uint32_t(item.bh), p.drop);
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[i], cnt & 1, wc, kSiteFwdSFull))) {
            ok = false;
            break;
          }
          tc_fence_after();
          float s[128];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t raw[32];
            tmem_ld32(trow + Cfg::tm_s(i) + q4 * 32, raw);
#pragma unroll
            for (int t = 0; t < 32; ++t) s[q4 * 32 + t] = __uint_as_float(raw[t]);
          }
          tmem_wait_ld();
          float sum, alpha, m_use;
          // Masked columns: keys past the causal limit (key 128 j + t is visible to
          // row 128 tile + r iff t < r + 1 + 128 (tile - j) + off), and keys past N_k in
          // the last K/V tile. The choice of variant is per tile, so warp-uniform.
          // Row r sees t < r + 1 + dbase; dbase is clamped to [-256, 256], beyond which
          // a tile is fully hidden or fully visible for every row.
          int dbase = 0;  // N_q = N_k: only the diagonal tile (j == tile) is partial, with dbase 0
          if constexpr (XQK) {
            const long long db64 = 128LL * (tile - j) + off_;
            dbase = static_cast<int>(db64 < -256 ? -256 : (db64 > 256 ? 256 : db64));
          }
          const bool diag = CAUSAL && (XQK ? dbase < 127 : j == tile);
          // (With the causal mask, keys past N_k are past every existing row's limit.)
          const int nk_last = p.Nk - 128 * (p.n_ktiles - 1);  // keys in the last K/V tile
          const bool tail = !CAUSAL && j == p.n_ktiles - 1 && nk_last != 128;
          if (diag || tail) {
            int lim = diag ? r + 1 + dbase : nk_last;
            if (XQK && lim < 0) lim = 0;  // (only an offset makes a row see none of a scheduled tile)
            softmax_row<true, PolyShare<D>::kFwd, DROP>(s, lim, c, m, trow + Cfg::tm_p(i), sum, alpha, m_use, kb,
                                                        drop_rs);
          } else {
            softmax_row<false, PolyShare<D>::kFwd, DROP>(s, 128, c, m, trow + Cfg::tm_p(i), sum, alpha, m_use, kb,
                                                         drop_rs);
          }
          const bool rescale = m_use != m;
          l = l * alpha + sum;
          if (__any_sync(0xffffffffu, rescale) && local > 0) {
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t ov[32];
              tmem_ld32(trow + Cfg::tm_o(i) + cc * 32, ov);
              tmem_wait_ld();
#pragma unroll
              for (int t = 0; t < 32; ++t) ov[t] = __float_as_uint(__uint_as_float(ov[t]) * alpha);
              tmem_st32(trow + Cfg::tm_o(i) + cc * 32, ov);
            }
          }
          m = m_use;
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars->p_ready[i]);
          ++cnt;
          ++local;
        }
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      // Every item ends with one o_full phase per tile and one o_empty arrival per
      // thread, whether or not this tile had work, so the phases stay in step.
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_full[i], kk & 1, wc, kSiteFwdOFull))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const size_t row = size_t(item.bh) * p.N + size_t(tile) * 128 + r;  // lse index
      const int ib = item.bh / p.H, ih = item.bh - ib * p.H;
      __nv_bfloat16* orow = p.o + seq_row_offset(ib, ih, tile * 128 + r, p.N, p.H, DS, p.bnhd != 0);
      const bool row_ok = tile * 128 + r < p.N;  // rows past N (last tile) do not exist
      if (MERGE && active && local > 0) {
        // lse' = ln(e^lse_acc + e^lse_b), O_acc' = O_acc e^(lse_acc - lse') + (O / l) e^(lse_b - lse'),
        // 32 columns of O at a time (then O_i is released).
        float wa = 0.f, wb = 0.f, lnew = 0.f;
        if (row_ok) {
          const float lb = (m + __log2f(l)) * 0.69314718055994531f;  // this block's lse (l > 0 here)
          const float la = p.lse_acc[row];
          const float mx = fmaxf(la, lb);
          wa = expf(la - mx);
          wb = expf(lb - mx);
          const float ssum = wa + wb;
          lnew = mx + logf(ssum);
          wa /= ssum;
          wb /= ssum * l;  // with the 1 / l of this block's O
        }
        float4* oa = reinterpret_cast<float4*>(p.o_acc + row * D);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(trow + Cfg::tm_o(i) + cc * 32, ov);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 a = oa[cc * 8 + c];
              oa[cc * 8 + c] =
                  make_float4(a.x * wa + __uint_as_float(ov[4 * c]) * wb, a.y * wa + __uint_as_float(ov[4 * c + 1]) * wb,
                              a.z * wa + __uint_as_float(ov[4 * c + 2]) * wb,
                              a.w * wa + __uint_as_float(ov[4 * c + 3]) * wb);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->o_empty[i]);
        if (row_ok) p.lse_acc[row] = lnew;
      } else if (MERGE) {
        mbar_arrive(&bars->o_empty[i]);  // the row saw no key of this block: nothing to merge
      } else if (active && local > 0) {
        // l = 0: the row saw no key (causal with N_q > N_k): O = 0, lse = -inf.
        const float inv_l = (!XQK || l > 0.f) ? 1.f / l : 0.f;
        uint32_t ov[D];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc)
          tmem_ld32(trow + Cfg::tm_o(i) + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[cc * 32]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->o_empty[i]);
        if constexpr (Cfg::kStageO) {
          // O rows of this warp, 64 columns at a time, through the warp's stage (the
          // second block has 32 columns when the stored head dim is 96).
          __nv_bfloat16* row0 = p.o + seq_row_offset(ib, ih, tile * 128 + r - lane, p.N, p.H, DS, p.bnhd != 0);
          const size_t ld = p.bnhd ? size_t(p.H) * DS : size_t(DS);  // elements between rows
          const int nrows = p.N - (tile * 128 + r - lane);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            uint32_t w[32];
#pragma unroll
            for (int t = 0; t < 32; ++t)
              w[t] = pack_bf16(__uint_as_float(ov[cb * 64 + 2 * t]) * inv_l,
                               __uint_as_float(ov[cb * 64 + 2 * t + 1]) * inv_l);
            if constexpr (DS == D) {
              warp_store_rows<32>(sStage + (warp - 4) * 1024, w, row0 + cb * 64, ld, nrows);
            } else if (cb * 64 + 64 <= DS) {
              warp_store_rows<32>(sStage + (warp - 4) * 1024, w, row0 + cb * 64, ld, nrows);
            } else if (cb * 64 + 32 == DS) {
              uint32_t w16[16];
#pragma unroll
              for (int t = 0; t < 16; ++t) w16[t] = w[t];
              warp_store_rows<16>(sStage + (warp - 4) * 1024, w16, row0 + cb * 64, ld, nrows);
            }
          }
        } else if (row_ok) {
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            if (cc * 32 >= DS) break;
            uint32_t pw[16];
#pragma unroll
            for (int t = 0; t < 16; ++t)
              pw[t] = pack_bf16(__uint_as_float(ov[cc * 32 + 2 * t]) * inv_l,
                                __uint_as_float(ov[cc * 32 + 2 * t + 1]) * inv_l);
            store_row64(orow + cc * 32, pw, p.v8 != 0);
          }
        }
        if (row_ok) p.lse[row] = (!XQK || l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      } else {
        mbar_arrive(&bars->o_empty[i]);
        if (active && row_ok) {
          // No visible key for this row (a block mask, or causal with N_q > N_k).
          const uint4 z = make_uint4(0, 0, 0, 0);
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int t = 0; t < D / 8; ++t)
            if (t * 8 < DS) dst[t] = z;
          p.lse[row] = -INFINITY;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  // Every role ends with its own CTA barrier (no common tail, so each warpgroup
  // keeps its register budget to the end); warp 1 then frees TMEM.
}

}  // namespace fa
