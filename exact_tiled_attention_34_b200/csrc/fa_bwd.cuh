// fa_bwd.cuh - backward kernels: attention recomputed tile by tile from the saved
// log-sum-exp ("Researchers at Stanford University Propose FlashAttention ..."
// summary, method paragraph: the forward's normalisation factor is saved so the
// backward recomputes attention on chip instead of storing it).
//
// Gradients of L = sum(O * dO):
//   D_i  = sum_c dO_ic O_ic                     (pre-processing kernel)
//   P    = exp(scale q_i.k_j - lse_i)           (recomputed, base 2)
//   dV_j = sum_i P_ij dO_i,   dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - D_i)
//   dK_j = scale sum_i dS_ij q_i,   dQ_i = scale sum_j dS_ij k_j
// (P enters dV and dS rounded to bf16, as it enters the tensor-core products.)
//
// Three launches, all deterministic (no atomics):
//  1. fa_bwd_pre_kernel: D and -lse * log2(e) into the workspace.
//  2. fa_bwd_dkdv_kernel: work item = (128-key tile j, batch*head), looping over the
//     query tiles i that see tile j (causal: i >= j; block-sparse: mask[i][j] = 1).
//     The transposed products put key rows on TMEM lanes:
//       S^T  = K_j Q_i^T   (SS, both K-major)       dP^T = V_j dO_i^T  (SS)
//       dV  += P^T dO_i    (TS: P^T from TMEM, dO_i N-major)
//       dK  += dS^T Q_i    (TS: dS^T from TMEM, Q_i N-major)
//     so the TMA-loaded Q/dO tiles serve as K-major and N-major operands alike.
//  3. fa_bwd_dq_kernel: work item = (128-query tile i, batch*head), looping over the
//     key tiles j that tile i sees; it recomputes S = Q_i K_j^T and dP = dO_i V_j^T,
//     forms dS and accumulates dQ_i += dS K_j in TMEM (TS: dS from TMEM, K_j N-major),
//     then writes dQ_i once. Recomputing S and dP (2 of its 3 products) costs tensor
//     time but removes the fp32 atomic accumulation of dQ, whose L2 traffic bounded a
//     single fused kernel.
//
// Both main kernels are persistent (one CTA per SM walking a static list of items;
// ring positions and barrier phases run on across items so loads and first products
// of the next item overlap the previous epilogue). 384 threads; warp 0 TMA producer, warp 1 MMA issuer + TMEM
// owner, warps 4-11 two "compute" warpgroups (thread = TMEM lane; warpgroup h takes
// the tile columns [64h, 64h+64)). A packed bf16 result for column c goes to TMEM
// column c/2, so warpgroup 1 writes columns that warpgroup 0 reads as fp32: both
// first finish reading (bounded mbarrier handshake).
#pragma once

#include <type_traits>

#include "fa_dropout.cuh"
#include "fa_ptx.cuh"

namespace fa {

// ---------------------------------------------------------------- pre-processing

// D[row] = sum_c dO[row, c] O[row, c] and nl2[row] = -lse[row] log2(e) (fp32), so
// that the exponent of the recomputed P is one fused multiply-add: s c + nl2. The two
// row arrays hold Npad = 128 * ceil(N / 128) rows per (batch, head): a tile's rows are
// one 512-byte run. The pad rows of the last tile (n >= N, when N % 128 != 0) get
// D = 0 and nl2 = -inf, so their recomputed P is 0 and they add nothing to dK or dV.
// A row that sees no key (lse = -inf: an empty tile row of a block mask, or the causal
// mask with N_q > N_k) also gets nl2 = -inf rather than +inf, so its exponents are
// never +inf (2^(+inf) is not finite on either exponential path); its P is then 0
// without relying on the element mask of the tiles it meets.
// D / 8 threads per row, 16 bytes each; rows hold ds <= D columns (96 with D = 128).
// dqacc (or nullptr): an fp32 [rows_pad, D] accumulator that the fused backward adds
// dQ into; it is zeroed here (pad rows included), each thread 8 columns of its row.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse, float* __restrict__ Drow,
                                                         float* __restrict__ lse2, int N, int Npad, int ds,
                                                         int H, int bnhd, long long rows_pad,
                                                         float* __restrict__ dqacc) {
  constexpr int TPR = D / 8;
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long prow = g / TPR;  // padded row index: bh * Npad + n
  const int part = static_cast<int>(g % TPR);
  const bool inrange = prow < rows_pad;
  // rows_pad <= INT_MAX (checked on the host), so 32-bit unsigned division suffices.
  const unsigned pr = static_cast<unsigned>(inrange ? prow : 0);
  const unsigned bh = pr / static_cast<unsigned>(Npad);
  const int n = static_cast<int>(pr - bh * static_cast<unsigned>(Npad));
  const bool valid = inrange && n < N;
  const long long row = static_cast<long long>(bh) * N + n;  // row of lse
  float s = 0.f;
  if (valid && part * 8 < ds) {
    const int b_ = static_cast<int>(bh / static_cast<unsigned>(H)), h_ = static_cast<int>(bh) - b_ * H;
    const size_t off = seq_row_offset(b_, h_, n, N, H, ds, bnhd != 0) + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + off);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 x = __bfloat1622float2(pa[t]);
      const float2 y = __bfloat1622float2(pb[t]);
      s = fmaf(x.x, y.x, s);
      s = fmaf(x.y, y.y, s);
    }
  }
  if (dqacc != nullptr && inrange) {
    float4* z = reinterpret_cast<float4*>(dqacc + static_cast<size_t>(prow) * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int w = TPR / 2; w > 0; w >>= 1) s += __shfl_xor_sync(0xffffffffu, s, w);
  if (inrange && part == 0) {
    Drow[prow] = s;
    const float l = valid ? lse[row] : -INFINITY;
    lse2[prow] = l > -INFINITY ? -l * 1.4426950408889634f : -INFINITY;
  }
}

// ---------------------------------------------------------------- common

struct BwdParams {
  const float* lse2;    // [BH, Npad] -lse * log2(e) (Npad = 128 * n_tiles; pad rows -inf)
  const float* Drow;    // [BH, Npad]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dk32;          // fused backward with fp32 outputs: dK, dV written as fp32 (dk, dv unused)
  float* dv32;
  const uint8_t* tile_mask;  // [nT, nT] or nullptr
  int* status;
  unsigned long long timeout_ns;
  int stall;            // test hook: 1 = the producer issues no copies, so every wait runs out
  int N;                // query rows N_q (any N >= 1)
  int Nk;               // key rows N_k
  int BH;
  int H;                // heads (item bh = b * H + h)
  int bnhd;             // 1: q, k, v, dO, dq, dk, dv are [B, N, H, d]; 0: [B, H, N, d]
  int n_tiles;          // query tiles ceil(N_q / 128)
  int n_ktiles;         // key tiles ceil(N_k / 128)
  int off;              // N_k - N_q: with the causal mask key j is visible to query i iff j <= i + off
  int ds;               // head dim as stored (row length of q, k, v, dO, dq, dk, dv): D, or 96 with D = 128
  int v8;               // 1: the gradient outputs are 32-byte aligned (32-byte row stores)
  int paired = 0;       // fused backward, causal: key tiles dealt in pairs (set by the launcher)
  float scale;          // softmax scale
};

// The dropout kernels' parameters (the others keep the plain block unchanged).
struct BwdParamsDrop : BwdParams {
  DropParams drop;
};
template <bool DROP>
using BwdParamsT = std::conditional_t<DROP, BwdParamsDrop, BwdParams>;

// Register split of both 384-thread kernels: the producer/MMA warpgroup drops to 80,
// the two compute warpgroups rise to 200 -> 128 * (80 + 2 * 200) = 61,440 registers,
// which the launch must provide (checked by the host: registers per thread x 384).
// Only the compute warpgroups increase, once, by less than the first warpgroup
// releases, so no increase can wait forever.
constexpr int kBwdThreads = 384;
constexpr int kBwdRegsCtl = 80;
constexpr int kBwdRegsCompute = 200;
constexpr int kBwdRegsNeeded = 128 * (kBwdRegsCtl + 2 * kBwdRegsCompute);

template <int D>
struct BwdCfg {
  static constexpr int kColBlocks = D / 64;
  static constexpr int kBlockBytes = 128 * 128;  // one 64-column block of a 128-row tile
  static constexpr int kTileBytes = 128 * D * 2;
  // dK/dV kernel: K, V resident; Q, dO in 2 stages; lse2 and D rows in 2 stages.
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;
  static constexpr int kOffDO = kOffQ + 2 * kTileBytes;
  static constexpr int kOffL = kOffDO + 2 * kTileBytes;
  static constexpr int kOffDr = kOffL + 1024;
  static constexpr int kOffBar = kOffDr + 1024;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  // dQ kernel: Q, dO resident; K, V in 2 stages.
  static constexpr int kQOffQ = 0;
  static constexpr int kQOffDO = kQOffQ + kTileBytes;
  static constexpr int kQOffK = kQOffDO + kTileBytes;
  static constexpr int kQOffV = kQOffK + 2 * kTileBytes;
  static constexpr int kQOffBar = kQOffV + 2 * kTileBytes;
  static constexpr int kQSmemBytes = kQOffBar + 256 + 1024;
  // TMEM columns. dK/dV kernel: dK | dV | S^T | dP^T. dQ kernel: S | dP | dQ.
  static constexpr uint32_t kTmDK = 0;
  static constexpr uint32_t kTmDV = D;
  static constexpr uint32_t kTmS = 2 * D;
  static constexpr uint32_t kTmDP = 2 * D + 128;
  static constexpr uint32_t kQTmS = 0;
  static constexpr uint32_t kQTmDP = 128;
  static constexpr uint32_t kQTmDQ = 256;
  static constexpr uint32_t kTmCols = 512;
};

enum BwdSite : int {
  kSiteBwdKV = 201, kSiteBwdTEmpty, kSiteBwdTFull, kSiteBwdPReady, kSiteBwdDsReady, kSiteBwdSFull,
  kSiteBwdDpFull, kSiteBwdAcc, kSiteBwdDrain, kSiteBwdRead, kSiteBwdSRead
};

// Causal limits between tiles (key j visible to query i iff j <= i + off):
// the first query tile that sees key tile j, and the last key tile query tile i sees
// (clamped to the key tiles; -1 for none).
__device__ __forceinline__ int causal_qfirst(int j, int off) {
  const long long x = 128LL * j - 127 - off;  // query tile t sees key tile j iff 128 t >= x
  return x <= 0 ? 0 : static_cast<int>((x + 127) >> 7);
}
__device__ __forceinline__ int causal_klast_b(int i, int off, int n_ktiles) {
  const long long x = 128LL * i + 127 + off;
  const long long l = x < 0 ? -1 : (x >> 7);
  return static_cast<int>(l < n_ktiles - 1 ? l : n_ktiles - 1);
}

// Query tiles that see key tile j (dK/dV kernel). The block mask is [n_tiles, n_ktiles].
// i_first: the first query tile that can see tile j (0 without the causal mask).
template <bool CAUSAL, bool SPARSE, bool XQK>
struct KeySched {
  int j, n_tiles, n_ktiles, i_first;
  const uint8_t* mask;
  __device__ __forceinline__ KeySched(int j_, int n_tiles_, int n_ktiles_, int off, const uint8_t* mask_)
      : j(j_), n_tiles(n_tiles_), n_ktiles(n_ktiles_),
        i_first(CAUSAL ? (XQK ? causal_qfirst(j_, off) : j_) : 0), mask(mask_) {}
  __device__ __forceinline__ int next(int i0) const {
    for (int i = (i0 + 1 > i_first ? i0 + 1 : i_first); i < n_tiles; ++i) {
      if (!SPARSE || mask[size_t(i) * n_ktiles + j] != 0) return i;
    }
    return -1;
  }
  __device__ __forceinline__ int first() const { return next(-1); }
};

// Key tiles that query tile i sees (dQ kernel). j_last: the last key tile tile i can
// see (-1 for none).
template <bool CAUSAL, bool SPARSE, bool XQK>
struct QuerySched {
  int i, n_ktiles, j_last;
  const uint8_t* mask;
  __device__ __forceinline__ QuerySched(int i_, int n_ktiles_, int off, const uint8_t* mask_)
      : i(i_), n_ktiles(n_ktiles_),
        j_last(CAUSAL ? (XQK ? causal_klast_b(i_, off, n_ktiles_) : i_) : n_ktiles_ - 1), mask(mask_) {}
  __device__ __forceinline__ int next(int j0) const {
    for (int j = j0 + 1; j <= j_last; ++j) {
      if (!SPARSE || mask[size_t(i) * n_ktiles + j] != 0) return j;
    }
    return -1;
  }
  __device__ __forceinline__ int first() const { return next(-1); }
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// X[tm] = A[128 x D] * B[128 x D]^T, both K-major 128-byte-swizzled tiles.
template <int D>
__device__ __forceinline__ void mma_tile_nt(uint32_t tm, uint32_t a, uint32_t b) {
  constexpr uint32_t id = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint32_t off = (k >> 2) * BwdCfg<D>::kBlockBytes + (k & 3) * 32;
    mma_ss(tm, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(b + off, 16, 1024), id, k > 0);
  }
}

// G[tm] (+)= A_tmem[128 x 128] * B[128 x D], A packed bf16 in TMEM, B N-major tile.
template <int D>
__device__ __forceinline__ void mma_tile_tn(uint32_t tm, uint32_t a_tm, uint32_t b, bool acc) {
  constexpr uint32_t id = idesc_bf16_f32(128, D, 0, 1);
  // Compute warpgroup h leaves its 64 queries' (or keys') packed values, 32 columns, at
  // the start of its own 64-column half of the operand region: k-steps 0..3 read
  // a_tm + 0..31, k-steps 4..7 read a_tm + 64..95.
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mma_ts(tm, a_tm + (k >> 2) * 64 + (k & 3) * 8, sdesc_sw128(b + k * 2048, BwdCfg<D>::kBlockBytes, 1024), id,
           (acc || k > 0) ? 1u : 0u);
}

// 64 columns of one thread's row, fp32 from TMEM, as 2 x 32.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}

// The first ncols (a multiple of 32, at most NCOL) of NCOL fp32 values of the thread's
// row (in registers), times mul, as bf16 to dst.
// v8: dst is 32-byte aligned (then 32-byte stores).
template <int NCOL>
__device__ __forceinline__ void store_regs_bf16(__nv_bfloat16* dst, const uint32_t (&v)[NCOL], float mul,
                                                int ncols, bool v8) {
#pragma unroll
  for (int cc = 0; cc < NCOL / 32; ++cc) {
    if (cc * 32 >= ncols) break;
    uint32_t w[16];
#pragma unroll
    for (int t = 0; t < 16; ++t)
      w[t] = pack_bf16(__uint_as_float(v[cc * 32 + 2 * t]) * mul, __uint_as_float(v[cc * 32 + 2 * t + 1]) * mul);
    store_row64(dst + cc * 32, w, v8);
  }
}

// The first ncols (a multiple of 32) of NCOL fp32 values of the thread's row, times mul,
// as fp32 to dst (16-byte aligned).
template <int NCOL>
__device__ __forceinline__ void store_regs_f32(float* dst, const uint32_t (&v)[NCOL], float mul, int ncols) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int c = 0; c < NCOL / 4; ++c) {
    if (c * 4 >= ncols) break;
    d4[c] = make_float4(__uint_as_float(v[4 * c]) * mul, __uint_as_float(v[4 * c + 1]) * mul,
                        __uint_as_float(v[4 * c + 2]) * mul, __uint_as_float(v[4 * c + 3]) * mul);
  }
}

// ---------------------------------------------------------------- persistent schedule

// The k-th work item (tile index, batch*head) of this CTA, or false when it has none.
// Without the causal mask all items cost the same and go head-major (the tiles of one
// head together, sharing its other operand tiles through L2); with it, an item's cost
// grows as its tile index falls (key tiles, dK/dV kernel) or rises (query tiles, dQ
// kernel), and items go costliest first across all heads, which with the alternating
// deal of item_position balances the CTAs' work.
struct BwdItem {
  int bh, tile;
};
template <bool CAUSAL, bool HEAVY_LOW>
__device__ __forceinline__ bool bwd_item(int n_tiles, int BH, int k, BwdItem& it) {
  const long long pos = item_position(static_cast<long long>(n_tiles) * BH, k);
  if (pos < 0) return false;
  if (CAUSAL) {
    const int rank = static_cast<int>(pos / BH);  // 0 = most work
    it.tile = HEAVY_LOW ? rank : n_tiles - 1 - rank;
    it.bh = static_cast<int>(pos % BH);
  } else {
    it.bh = static_cast<int>(pos / n_tiles);
    it.tile = static_cast<int>(pos % n_tiles);
  }
  return true;
}

// ---------------------------------------------------------------- dK / dV kernel

struct DkdvBars {
  uint64_t kv_full;
  uint64_t kv_empty;  // the item's S^T and dP^T products are done with K_j, V_j
  uint64_t t_full[2];
  uint64_t t_empty[2];
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t p_ready;
  uint64_t ds_ready;
  uint64_t acc_done;
  uint64_t acc_empty;  // the epilogue has read dK and dV (the next item may overwrite them)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// DROP: dropout on P (dV takes the dropped P^T, dS the kept part of dP^T).
template <int D, bool CAUSAL, bool SPARSE, bool XQK, bool DROP = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const BwdParamsT<DROP> p) {
  using Cfg = BwdCfg<D>;
  // Causal offset N_k - N_q: a compile-time 0 in the N_q = N_k kernels (XQK false).
  const int off_ = XQK ? p.off : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  DkdvBars* bars = reinterpret_cast<DkdvBars*>(smem + Cfg::kOffBar);
  uint8_t* sK = smem + Cfg::kOffK;
  uint8_t* sV = smem + Cfg::kOffV;
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sDO = smem + Cfg::kOffDO;
  float* sL = reinterpret_cast<float*>(smem + Cfg::kOffL);
  float* sDr = reinterpret_cast<float*>(smem + Cfg::kOffDr);

  const int warp = warp_id();
  const int lane = lane_id();
  WaitCtl wc{&bars->abort, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->t_full[s], 1);
      mbar_init(&bars->t_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_ready, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->acc_empty, 256);
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
  constexpr uint32_t kTileTx = 2 * Cfg::kTileBytes + 2 * 512;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    regs_dec<kBwdRegsCtl>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint64_t keep = policy_evict_last();
      int it = 0;  // Q/dO tiles loaded so far (ring position, continues across items)
      int nkv = 0;
      bool ok = p.stall == 0;
      BwdItem item;
      for (int kk = 0; ok && bwd_item<CAUSAL, true>(p.n_ktiles, p.BH, kk, item); ++kk) {
        const int j = item.tile, bh = item.bh;
        const int ib = bh / p.H, ih = bh - ib * p.H;  // batch, head (tensor-map coordinates)
        KeySched<CAUSAL, SPARSE, XQK> sch{j, p.n_tiles, p.n_ktiles, off_, p.tile_mask};
        if (kk > 0 && !mbar_wait(&bars->kv_empty, (kk - 1) & 1, wc, kSiteBwdTEmpty)) break;
        mbar_arrive_expect_tx(&bars->kv_full, 2 * Cfg::kTileBytes);
        for (int cb = 0; cb < Cfg::kColBlocks; ++cb) {
          tma_load_4d(sK + cb * Cfg::kBlockBytes, &tm_k, &bars->kv_full, cb * 64, j * 128, ih, ib);
          tma_load_4d(sV + cb * Cfg::kBlockBytes, &tm_v, &bars->kv_full, cb * 64, j * 128, ih, ib);
        }
        ++nkv;
        for (int i = sch.first(); i >= 0; i = sch.next(i), ++it) {
          const int st = it & 1;
          const int n = it >> 1;
          if (n > 0 && !mbar_wait(&bars->t_empty[st], (n - 1) & 1, wc, kSiteBwdTEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->t_full[st], kTileTx);
          for (int cb = 0; cb < Cfg::kColBlocks; ++cb) {
            tma_load_4d_hint(sQ + st * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_q, &bars->t_full[st],
                             cb * 64, i * 128, ih, ib, keep);
            tma_load_4d_hint(sDO + st * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_do, &bars->t_full[st],
                             cb * 64, i * 128, ih, ib, keep);
          }
          const size_t roff = (size_t(bh) * p.n_tiles + size_t(i)) * 128;  // padded row arrays
          bulk_load(sL + st * 128, p.lse2 + roff, 512, &bars->t_full[st]);
          bulk_load(sDr + st * 128, p.Drow + roff, 512, &bars->t_full[st]);
        }
      }
      if (bars->abort) {
        if (nkv > 0) mbar_wait_drain(&bars->kv_full, (nkv - 1) & 1, wc, kSiteBwdDrain);
        for (int x = (it > 2 ? it - 2 : 0); x < it; ++x)
          mbar_wait_drain(&bars->t_full[x & 1], (x >> 1) & 1, wc, kSiteBwdDrain);
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kBwdRegsCtl>();
    if (lane == 0) {
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO);
      bool ok = true;
      int it = 0;  // query tiles processed so far (continues across items)
      BwdItem item;
      for (int kk = 0; ok && bwd_item<CAUSAL, true>(p.n_ktiles, p.BH, kk, item); ++kk) {
        KeySched<CAUSAL, SPARSE, XQK> sch{item.tile, p.n_tiles, p.n_ktiles, off_, p.tile_mask};
        if (!mbar_wait(&bars->kv_full, kk & 1, wc, kSiteBwdKV)) { ok = false; break; }
        tc_fence_after();
        int i = sch.first();
        if (i < 0) mma_commit(&bars->kv_empty);
        if (i >= 0) {
          if (!mbar_wait(&bars->t_full[it & 1], (it >> 1) & 1, wc, kSiteBwdTFull)) { ok = false; break; }
          tc_fence_after();
          mma_tile_nt<D>(tmem + Cfg::kTmS, aK, aQ + (it & 1) * Cfg::kTileBytes);
          mma_commit(&bars->s_full);
          mma_tile_nt<D>(tmem + Cfg::kTmDP, aV, aDO + (it & 1) * Cfg::kTileBytes);
          mma_commit(&bars->dp_full);
        }
        bool first = true;
        while (i >= 0) {
          const int st = it & 1;
          const int in = sch.next(i);
          const int stn = (it + 1) & 1;
          const uint32_t phn = ((it + 1) >> 1) & 1;
          // All S^T / dP^T products of this item are issued: K_j, V_j free when done.
          if (in < 0) mma_commit(&bars->kv_empty);
          // dV += P^T dO_i, then the next S^T (it overwrites P^T only after this dV
          // product has read it: products execute in issue order).
          if (!mbar_wait(&bars->p_ready, it & 1, wc, kSiteBwdPReady)) { ok = false; break; }
          // The first dV/dK products of an item overwrite the accumulators: the
          // previous item's epilogue must have read them.
          if (first && kk > 0 && !mbar_wait(&bars->acc_empty, (kk - 1) & 1, wc, kSiteBwdAcc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_tn<D>(tmem + Cfg::kTmDV, tmem + Cfg::kTmS, aDO + st * Cfg::kTileBytes, !first);
          if (in >= 0) {
            if (!mbar_wait(&bars->t_full[stn], phn, wc, kSiteBwdTFull)) { ok = false; break; }
            tc_fence_after();
            mma_tile_nt<D>(tmem + Cfg::kTmS, aK, aQ + stn * Cfg::kTileBytes);
            mma_commit(&bars->s_full);
          }
          // dK += dS^T Q_i, then the next dP^T (over dS^T, in issue order).
          if (!mbar_wait(&bars->ds_ready, it & 1, wc, kSiteBwdDsReady)) { ok = false; break; }
          tc_fence_after();
          mma_tile_tn<D>(tmem + Cfg::kTmDK, tmem + Cfg::kTmDP, aQ + st * Cfg::kTileBytes, !first);
          mma_commit(&bars->t_empty[st]);
          if (in >= 0) {
            mma_tile_nt<D>(tmem + Cfg::kTmDP, aV, aDO + stn * Cfg::kTileBytes);
            mma_commit(&bars->dp_full);
          }
          first = false;
          i = in;
          ++it;
        }
        if (!ok) break;
        mma_commit(&bars->acc_done);
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, wc, kSiteBwdDrain);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmCols);
  } else if (warp < 4) {
    // idle warps of the first warpgroup: they take part in its register hand-over
    regs_dec<kBwdRegsCtl>();
    __syncthreads();
  } else {
    // ------------------------------------------------------------ compute warpgroups
    // Warpgroup h handles query columns [64h, 64h + 64) of the 128 key rows.
    regs_inc<kBwdRegsCompute>();
    const int h = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row within tile j
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    const float c2 = p.scale * 1.4426950408889634f;
    bool ok = true;
    int it = 0;  // query tiles processed so far (continues across items)
    BwdItem item;
    for (int kk = 0; ok && bwd_item<CAUSAL, true>(p.n_ktiles, p.BH, kk, item); ++kk) {
      const int j = item.tile;
      KeySched<CAUSAL, SPARSE, XQK> sch{j, p.n_tiles, p.n_ktiles, off_, p.tile_mask};
      int local = 0;
      for (int i = sch.first(); i >= 0; i = sch.next(i), ++it, ++local) {
        const int st = it & 1;
        // Keep bits of this key over query columns [64h, 64h + 64) of tile i.
        uint32_t kb[2] = {0u, 0u};
        if constexpr (DROP)
          drop_bits_cols<16>(kb, uint32_t(j * 32 + quarter * 8 + (lane >> 2)), uint32_t(i * 32 + h * 16),
                             uint32_t(item.bh), p.drop);
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->t_full[st], (it >> 1) & 1, wc, kSiteBwdTFull)) ||
            !__all_sync(0xffffffffu, mbar_wait(&bars->s_full, it & 1, wc, kSiteBwdSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* lse2 = sL + st * 128 + h * 64;
        const float* Dr = sDr + st * 128 + h * 64;
        // Query 128 i + c sees key 128 j + r iff c >= r + cbase; the tile is partial
        // (element mask) iff some (r, c) fails, i.e. cbase + 127 > 0.
        int cbase = 0;  // N_q = N_k: only the diagonal tile (i == j) is partial, with cbase 0
        if constexpr (XQK) {
          const long long cb64 = 128LL * (j - i) - off_;  // clamped: beyond +-256 no row is partial
          cbase = static_cast<int>(cb64 < -256 ? -256 : (cb64 > 256 ? 256 : cb64));
        }
        const bool diag = CAUSAL && (XQK ? cbase > -127 : i == j);
        const int cmin = cbase + r;
        // ---- P^T row r, query columns 64h + (0..63), packed bf16 pairs
        uint32_t pk[32];
        {
          uint32_t raw[64];
          tmem_ld64(trow + Cfg::kTmS + h * 64, raw);
          tmem_wait_ld();
          // The packed P^T of this warpgroup's 64 queries goes to the first 32 of its own 64
          // score columns: this thread has read its row of them, and no other thread reads
          // this row.
          const uint64_t c2v = f2(c2, c2);
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int c0 = 2 * t;
            const float2 nl = *reinterpret_cast<const float2*>(lse2 + c0);  // -lse log2 e
            uint64_t pv = ex2_split_x2<PolyShare<D>::kDkdv>(
                f2_fma(f2(__uint_as_float(raw[c0]), __uint_as_float(raw[c0 + 1])), c2v, f2(nl.x, nl.y)), t);
            if (diag) {
              const float2 v = f2_split(pv);
              pv = f2((h * 64 + c0 < cmin) ? 0.f : v.x, (h * 64 + c0 + 1 < cmin) ? 0.f : v.y);
            }
            const float2 v = f2_split(pv);
            pk[t] = pack_bf16(v.x, v.y);
          }
        }
        if constexpr (DROP) {
          // dV = P~^T dO takes the dropped probabilities; dS below the undropped ones.
          uint32_t pd[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float2 pp = unpack_bf16(pk[t]);
            const float2 w = drop_pair(pp.x, pp.y, kb[t >> 4] >> ((2 * t) & 31), p.drop.rs);
            pd[t] = pack_bf16(w.x, w.y);
          }
          tmem_st32(trow + Cfg::kTmS + h * 64, pd);
        } else {
          tmem_st32(trow + Cfg::kTmS + h * 64, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_ready);
        // ---- dS^T = P^T * (dP^T - D) into TMEM (A operand of dK)
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full, it & 1, wc, kSiteBwdDpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          uint32_t dpr[64];
          tmem_ld64(trow + Cfg::kTmDP + h * 64, dpr);
          tmem_wait_ld();
          uint32_t ds[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float2 pp = unpack_bf16(pk[t]);
            const float2 dd = *reinterpret_cast<const float2*>(Dr + 2 * t);
            uint64_t diff;
            if constexpr (DROP) {
              const float2 dpv = drop_pair(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1]),
                                           kb[t >> 4] >> ((2 * t) & 31), p.drop.rs);
              diff = f2_sub(f2(dpv.x, dpv.y), f2(dd.x, dd.y));
            } else {
              diff = f2_sub(f2(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1])), f2(dd.x, dd.y));
            }
            const float2 v = f2_split(f2_mul(f2(pp.x, pp.y), diff));
            ds[t] = pack_bf16(v.x, v.y);
          }
          tmem_st32(trow + Cfg::kTmDP + h * 64, ds);  // over this warpgroup's own dP^T columns
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready);
      }
      if (!ok) break;
      // -------------------------------------------------------- epilogue: dK (h = 0), dV (h = 1)
      // One acc_done phase and one acc_empty arrival per thread for every item.
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, kk & 1, wc, kSiteBwdAcc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int ib = item.bh / p.H, ih = item.bh - ib * p.H;
      const size_t row = seq_row_offset(ib, ih, j * 128 + r, p.Nk, p.H, p.ds, p.bnhd != 0);  // key row (elements)
      uint32_t acc[D];
      if (local > 0) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc)
          tmem_ld32(trow + (h == 0 ? Cfg::kTmDK : Cfg::kTmDV) + cc * 32,
                    *reinterpret_cast<uint32_t(*)[32]>(&acc[cc * 32]));
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int t = 0; t < D; ++t) acc[t] = 0u;
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
      if (j * 128 + r < p.Nk)  // key rows past N_k (last tile, N_k % 128 != 0) do not exist
        store_regs_bf16<D>((h == 0 ? p.dk : p.dv) + row, acc, h == 0 ? p.scale : 1.f, p.ds, p.v8 != 0);
    }
    tc_fence_before();
    __syncthreads();
  }
  // Every role ends with its own CTA barrier (no common tail, so each warpgroup
  // keeps its register budget to the end); warp 1 then frees TMEM.
}

// ---------------------------------------------------------------- dQ kernel

struct DqBars {
  uint64_t q_full;
  uint64_t q_empty;   // the item's S and dP products are done with Q_i, dO_i
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t s_read;    // both compute warpgroups have read S (the next S may start)
  uint64_t ds_ready;
  uint64_t acc_done;
  uint64_t acc_empty;  // the epilogue has read dQ (the next item may overwrite it)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// DROP: dropout on P (dS takes the kept part of dP).
template <int D, bool CAUSAL, bool SPARSE, bool XQK, bool DROP = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const BwdParamsT<DROP> p) {
  using Cfg = BwdCfg<D>;
  // Causal offset N_k - N_q: a compile-time 0 in the N_q = N_k kernels (XQK false).
  const int off_ = XQK ? p.off : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  DqBars* bars = reinterpret_cast<DqBars*>(smem + Cfg::kQOffBar);
  uint8_t* sQ = smem + Cfg::kQOffQ;
  uint8_t* sDO = smem + Cfg::kQOffDO;
  uint8_t* sK = smem + Cfg::kQOffK;
  uint8_t* sV = smem + Cfg::kQOffV;

  const int warp = warp_id();
  const int lane = lane_id();
  WaitCtl wc{&bars->abort, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->s_read, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->acc_empty, 256);
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
    regs_dec<kBwdRegsCtl>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint64_t keep = policy_evict_last();
      int it = 0;  // K/V tiles loaded so far (ring position, continues across items)
      int nq = 0;
      bool ok = p.stall == 0;
      BwdItem item;
      for (int kk = 0; ok && bwd_item<CAUSAL, false>(p.n_tiles, p.BH, kk, item); ++kk) {
        const int i = item.tile, bh = item.bh;
        const int ib = bh / p.H, ih = bh - ib * p.H;  // batch, head (tensor-map coordinates)
        QuerySched<CAUSAL, SPARSE, XQK> sch{i, p.n_ktiles, off_, p.tile_mask};
        if (kk > 0 && !mbar_wait(&bars->q_empty, (kk - 1) & 1, wc, kSiteBwdTEmpty)) break;
        mbar_arrive_expect_tx(&bars->q_full, 2 * Cfg::kTileBytes);
        for (int cb = 0; cb < Cfg::kColBlocks; ++cb) {
          tma_load_4d(sQ + cb * Cfg::kBlockBytes, &tm_q, &bars->q_full, cb * 64, i * 128, ih, ib);
          tma_load_4d(sDO + cb * Cfg::kBlockBytes, &tm_do, &bars->q_full, cb * 64, i * 128, ih, ib);
        }
        ++nq;
        for (int jj = sch.first(); jj >= 0; jj = sch.next(jj), ++it) {
          const int st = it & 1;
          const int n = it >> 1;
          if (n > 0 && !mbar_wait(&bars->kv_empty[st], (n - 1) & 1, wc, kSiteBwdTEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->kv_full[st], 2 * Cfg::kTileBytes);
          for (int cb = 0; cb < Cfg::kColBlocks; ++cb) {
            tma_load_4d_hint(sK + st * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_k, &bars->kv_full[st],
                             cb * 64, jj * 128, ih, ib, keep);
            tma_load_4d_hint(sV + st * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_v, &bars->kv_full[st],
                             cb * 64, jj * 128, ih, ib, keep);
          }
        }
      }
      if (bars->abort) {
        if (nq > 0) mbar_wait_drain(&bars->q_full, (nq - 1) & 1, wc, kSiteBwdDrain);
        for (int x = (it > 2 ? it - 2 : 0); x < it; ++x)
          mbar_wait_drain(&bars->kv_full[x & 1], (x >> 1) & 1, wc, kSiteBwdDrain);
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kBwdRegsCtl>();
    if (lane == 0) {
      const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = true;
      int it = 0;  // key tiles processed so far (continues across items)
      BwdItem item;
      for (int kk = 0; ok && bwd_item<CAUSAL, false>(p.n_tiles, p.BH, kk, item); ++kk) {
        QuerySched<CAUSAL, SPARSE, XQK> sch{item.tile, p.n_ktiles, off_, p.tile_mask};
        if (!mbar_wait(&bars->q_full, kk & 1, wc, kSiteBwdKV)) { ok = false; break; }
        tc_fence_after();
        int jj = sch.first();
        if (jj < 0) mma_commit(&bars->q_empty);
        if (jj >= 0) {
          if (!mbar_wait(&bars->kv_full[it & 1], (it >> 1) & 1, wc, kSiteBwdTFull)) { ok = false; break; }
          tc_fence_after();
          mma_tile_nt<D>(tmem + Cfg::kQTmS, aQ, aK + (it & 1) * Cfg::kTileBytes);
          mma_commit(&bars->s_full);
          mma_tile_nt<D>(tmem + Cfg::kQTmDP, aDO, aV + (it & 1) * Cfg::kTileBytes);
          mma_commit(&bars->dp_full);
        }
        bool first = true;
        while (jj >= 0) {
          const int st = it & 1;
          const int jn = sch.next(jj);
          const int stn = (it + 1) & 1;
          const uint32_t phn = ((it + 1) >> 1) & 1;
          // All S and dP products of this item are issued: Q_i, dO_i free when done.
          if (jn < 0) mma_commit(&bars->q_empty);
          // Next S as soon as both warpgroups have read this one.
          if (jn >= 0) {
            if (!mbar_wait(&bars->s_read, it & 1, wc, kSiteBwdSRead)) { ok = false; break; }
            if (!mbar_wait(&bars->kv_full[stn], phn, wc, kSiteBwdTFull)) { ok = false; break; }
            tc_fence_after();
            mma_tile_nt<D>(tmem + Cfg::kQTmS, aQ, aK + stn * Cfg::kTileBytes);
            mma_commit(&bars->s_full);
          }
          // dQ += dS K_j, then the next dP (over dS, in issue order). The first dQ
          // product of an item overwrites the accumulator: the previous item's
          // epilogue must have read it.
          if (!mbar_wait(&bars->ds_ready, it & 1, wc, kSiteBwdDsReady)) { ok = false; break; }
          if (first && kk > 0 && !mbar_wait(&bars->acc_empty, (kk - 1) & 1, wc, kSiteBwdAcc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_tn<D>(tmem + Cfg::kQTmDQ, tmem + Cfg::kQTmDP, aK + st * Cfg::kTileBytes, !first);
          mma_commit(&bars->kv_empty[st]);
          if (jn >= 0) {
            mma_tile_nt<D>(tmem + Cfg::kQTmDP, aDO, aV + stn * Cfg::kTileBytes);
            mma_commit(&bars->dp_full);
          }
          first = false;
          jj = jn;
          ++it;
        }
        if (!ok) break;
        mma_commit(&bars->acc_done);
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, wc, kSiteBwdDrain);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmCols);
  } else if (warp < 4) {
    regs_dec<kBwdRegsCtl>();
    __syncthreads();
  } else {
    // ------------------------------------------------------------ compute warpgroups
    // Warpgroup h handles key columns [64h, 64h + 64) of the 128 query rows.
    regs_inc<kBwdRegsCompute>();
    const int h = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within tile i
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    const float c2 = p.scale * 1.4426950408889634f;
    bool ok = true;
    int it = 0;  // key tiles processed so far (continues across items)
    // The row values of an item (-lse log2 e and D) are loaded ahead, during the previous
    // item's epilogue, so that they do not queue behind its row stores.
    auto row_vals = [&](const BwdItem& x, float& l2_, float& dv_) {
      const size_t prow = (size_t(x.bh) * p.n_tiles + size_t(x.tile)) * 128 + r;  // padded row arrays
      l2_ = p.lse2[prow];
      dv_ = p.Drow[prow];
    };
    BwdItem item;
    bool have = bwd_item<CAUSAL, false>(p.n_tiles, p.BH, 0, item);
    float l2_next = 0.f, dv_next = 0.f;
    if (have) row_vals(item, l2_next, dv_next);
    for (int kk = 0; ok && have; ++kk) {
      const int i = item.tile;
      QuerySched<CAUSAL, SPARSE, XQK> sch{i, p.n_ktiles, off_, p.tile_mask};
      const int ib = item.bh / p.H, ih = item.bh - ib * p.H;
      const size_t row = seq_row_offset(ib, ih, i * 128 + r, p.N, p.H, p.ds, p.bnhd != 0);  // query row (elements)
      const float l2 = l2_next;
      const float Dv = dv_next;
      int local = 0;
      for (int jj = sch.first(); jj >= 0; jj = sch.next(jj), ++it, ++local) {
        // Keep bits of this query row over key columns [64h, 64h + 64) of tile jj.
        uint32_t kb[2] = {0u, 0u};
        if constexpr (DROP)
          drop_bits_rows<16>(kb, uint32_t(i * 32 + quarter * 8 + (lane >> 2)), uint32_t(jj * 32 + h * 16),
                             uint32_t(item.bh), p.drop);
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, it & 1, wc, kSiteBwdSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Key 128 jj + c is visible to query 128 i + r iff c <= r + cbase; the tile is
        // partial (element mask) iff cbase < 127.
        int cbase = 0;  // N_q = N_k: only the diagonal tile (jj == i) is partial, with cbase 0
        if constexpr (XQK) {
          const long long cb64 = 128LL * (i - jj) + off_;  // clamped: beyond +-256 no row is partial
          cbase = static_cast<int>(cb64 < -256 ? -256 : (cb64 > 256 ? 256 : cb64));
        }
        const bool diag = CAUSAL && (XQK ? cbase < 127 : jj == i);
        const int cmax = cbase + r;
        uint32_t pk[32];
        {
          uint32_t raw[64];
          tmem_ld64(trow + Cfg::kQTmS + h * 64, raw);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&bars->s_read);
          const uint64_t c2v = f2(c2, c2), nl2 = f2(l2, l2);  // l2 = -lse log2 e
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            uint64_t pv = ex2_split_x2<PolyShare<D>::kDq>(
                f2_fma(f2(__uint_as_float(raw[2 * t]), __uint_as_float(raw[2 * t + 1])), c2v, nl2), t);
            if (diag) {
              const float2 v = f2_split(pv);
              pv = f2((h * 64 + 2 * t > cmax) ? 0.f : v.x, (h * 64 + 2 * t + 1 > cmax) ? 0.f : v.y);
            }
            const float2 v = f2_split(pv);
            pk[t] = pack_bf16(v.x, v.y);
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full, it & 1, wc, kSiteBwdDpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          uint32_t dpr[64];
          tmem_ld64(trow + Cfg::kQTmDP + h * 64, dpr);
          tmem_wait_ld();
          const uint64_t dv2 = f2(Dv, Dv);
          uint32_t ds[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float2 pp = unpack_bf16(pk[t]);
            uint64_t diff;
            if constexpr (DROP) {
              const float2 dpv = drop_pair(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1]),
                                           kb[t >> 4] >> ((2 * t) & 31), p.drop.rs);
              diff = f2_sub(f2(dpv.x, dpv.y), dv2);
            } else {
              diff = f2_sub(f2(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1])), dv2);
            }
            const float2 v = f2_split(f2_mul(f2(pp.x, pp.y), diff));
            ds[t] = pack_bf16(v.x, v.y);
          }
          tmem_st32(trow + Cfg::kQTmDP + h * 64, ds);  // over this warpgroup's own dP columns
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready);
      }
      if (!ok) break;
      // -------------------------------------------------------- epilogue: dQ columns [h D/2, (h+1) D/2)
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, kk & 1, wc, kSiteBwdAcc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t acc[D / 2];
      if (local > 0) {
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc)
          tmem_ld32(trow + Cfg::kQTmDQ + h * (D / 2) + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&acc[cc * 32]));
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int t = 0; t < D / 2; ++t) acc[t] = 0u;
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
      const bool row_ok = i * 128 + r < p.N;  // query rows past N (last tile, N % 128 != 0) do not exist
      have = bwd_item<CAUSAL, false>(p.n_tiles, p.BH, kk + 1, item);
      if (have) row_vals(item, l2_next, dv_next);
      if (row_ok) store_regs_bf16<D / 2>(p.dq + row + h * (D / 2), acc, p.scale, p.ds - h * (D / 2), p.v8 != 0);
    }
    tc_fence_before();
    __syncthreads();
  }
}

}  // namespace fa
