// fa_fwd256.cuh - forward kernel for head dim 256: exact attention with online
// softmax, one 128-row Q tile per work item.
//
// Same method as fa_fwd.cuh ("FlashAttention-2 ..." review, "Proposed method":
// online-softmax tiling, parallelism over sequence length, causal tile skipping;
// the Stanford summary's saved normalisation factor). At head dim 256 a Q tile's
// fp32 O accumulator alone takes 256 of the 512 tensor-memory columns, so an item holds
// ONE Q tile (not two as at 64/128) and the overlap of softmax and matrix products comes
// from double-buffered scores instead: S_{j+1} = Q K_{j+1}^T runs while the softmax of
// tile j does, then O += P_j V_j.
//   warp 0      TMA producer of Q and K (one elected thread)
//   warp 1      MMA issuer + TMEM owner
//   warp 2      TMA producer of V (its own thread, so that a K load never waits
//               behind a V load that waits for the previous P V product)
//   warps 4-7   softmax warpgroup (thread = query row = TMEM lane)
// Shared memory: Q, K, V one 64 KB tile each (192 KB). Tensor memory: S0 | S1 | O.
// Order of products: S_0, S_1, P_0 V_0, S_2, P_1 V_1, ...; so the softmax of tile j+1
// may start while P_j V_j is still running, and a rescale of O (only when a row's max
// rose by more than 2^8) first waits for that product (pv_done).
#pragma once

#include "fa_fwd.cuh"

namespace fa {

struct Fwd256Cfg {
  static constexpr int kTileBytes = 128 * 256 * 2;  // 64 KB: four 64-column blocks of 16 KB
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kTileBytes;
  static constexpr int kOffV = 2 * kTileBytes;
  static constexpr int kOffBar = 3 * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "forward (head dim 256) shared memory above the per-block limit");
  static constexpr int kThreads = 256;
  static constexpr uint32_t kTmO = 256;
  static constexpr uint32_t kTmCols = 512;
  __host__ __device__ static constexpr uint32_t tm_s(int b) { return b ? 128u : 0u; }
};

struct Fwd256Bars {
  uint64_t q_full, q_empty;  // q_empty: every S product of the item is done
  uint64_t k_full, k_empty;
  uint64_t v_full, v_empty;
  uint64_t s_full[2];
  uint64_t p_ready[2];       // 128 arrivals
  uint64_t pv_done;          // one phase per P V product
  uint64_t o_full, o_empty;  // o_empty: 128 arrivals (the epilogue has read O)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

enum Fwd256Site : int {
  kSite256Q = 401, kSite256QEmpty, kSite256KFull, kSite256KEmpty, kSite256VFull, kSite256VEmpty, kSite256SFull,
  kSite256PReady, kSite256PvDone, kSite256OFull, kSite256OEmpty, kSite256Drain
};

// K/V tiles that query tile t visits, in increasing order.
template <bool CAUSAL, bool SPARSE, bool XQK>
struct Sched256 {
  int t, n_ktiles, jlast;
  const uint8_t* mask;
  __device__ __forceinline__ Sched256(int t_, int n_ktiles_, int off, const uint8_t* mask_)
      : t(t_), n_ktiles(n_ktiles_),
        jlast(CAUSAL ? (XQK ? causal_klast(t_, off, n_ktiles_) : t_) : n_ktiles_ - 1), mask(mask_) {}
  __device__ __forceinline__ int next(int j0) const {
    for (int j = j0 + 1; j <= jlast; ++j)
      if (!SPARSE || mask[size_t(t) * n_ktiles + j] != 0) return j;
    return -1;
  }
  __device__ __forceinline__ int first() const { return next(-1); }
};

template <bool CAUSAL, bool SPARSE, bool XQK>
__global__ void __launch_bounds__(256, 1)
fa_fwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Cfg = Fwd256Cfg;
  constexpr int D = 256;
  const int off_ = XQK ? p.off : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  Fwd256Bars* bars = reinterpret_cast<Fwd256Bars*>(smem + Cfg::kOffBar);
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sK = smem + Cfg::kOffK;
  uint8_t* sV = smem + Cfg::kOffV;
  const int warp = warp_id();
  const int lane = lane_id();
  WaitCtl wc{&bars->abort, p.status, p.timeout_ns};
  auto sched_of = [&](const FwdItem& it) { return Sched256<CAUSAL, SPARSE, XQK>(it.qb, p.n_ktiles, off_, p.tile_mask); };

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->k_full, 1);
    mbar_init(&bars->k_empty, 1);
    mbar_init(&bars->v_full, 1);
    mbar_init(&bars->v_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_ready[b], 128);
    }
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->o_empty, 128);
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

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool qk = warp == 0;  // warp 0: Q and K; warp 2: V
      tma_prefetch_desc(qk ? &tm_k : &tm_v);
      if (qk) tma_prefetch_desc(&tm_q);
      const uint64_t keep = policy_evict_last();
      int n = 0, nq = 0;  // K (or V) tiles and Q tiles loaded so far
      bool ok = p.stall == 0;
      FwdItem item;
      for (int kk = 0; ok && fwd_item<CAUSAL>(p.n_items, p.n_qblocks, p.BH, kk, item); ++kk) {
        const auto sch = sched_of(item);
        const int ib = item.bh / p.H, ih = item.bh - ib * p.H;
        if (qk) {
          if (kk > 0 && !mbar_wait(&bars->q_empty, (kk - 1) & 1, wc, kSite256QEmpty)) break;
          mbar_arrive_expect_tx(&bars->q_full, Cfg::kTileBytes);
          for (int cb = 0; cb < 4; ++cb)
            tma_load_4d(sQ + cb * Cfg::kBlockBytes, &tm_q, &bars->q_full, cb * 64, item.qb * 128, ih, ib);
          ++nq;
        }
        for (int j = sch.first(); j >= 0; j = sch.next(j)) {
          uint64_t* full = qk ? &bars->k_full : &bars->v_full;
          uint64_t* empty = qk ? &bars->k_empty : &bars->v_empty;
          if (n > 0 && !mbar_wait(empty, (n - 1) & 1, wc, qk ? kSite256KEmpty : kSite256VEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full, Cfg::kTileBytes);
          uint8_t* dst = qk ? sK : sV;
          for (int cb = 0; cb < 4; ++cb)
            tma_load_4d_hint(dst + cb * Cfg::kBlockBytes, qk ? &tm_k : &tm_v, full, cb * 64, j * 128, ih, ib, keep);
          ++n;
        }
      }
      // On abort, wait (bounded) for this thread's own copies still in flight.
      if (bars->abort) {
        if (qk && nq > 0) mbar_wait_drain(&bars->q_full, (nq - 1) & 1, wc, kSite256Drain);
        if (n > 0) mbar_wait_drain(qk ? &bars->k_full : &bars->v_full, (n - 1) & 1, wc, kSite256Drain);
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);  // S = Q K^T, both K-major
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);    // O += P V, V N-major (N = 256)
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      auto issue_s = [&](int b) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t o = (k >> 2) * Cfg::kBlockBytes + (k & 3) * 32;
          mma_ss(tmem + Cfg::tm_s(b), sdesc_sw128(sQa + o, 16, 1024), sdesc_sw128(sKa + o, 16, 1024), idS, k > 0);
        }
      };
      auto issue_pv = [&](int b, bool acc) {
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k)
          mma_ts(tmem + Cfg::kTmO, tmem + Cfg::tm_s(b) + k * 8, sdesc_sw128(sVa + k * 2048, Cfg::kBlockBytes, 1024),
                 idO, (acc || k > 0) ? 1u : 0u);
      };
      bool ok = true;
      int g = 0;       // score tiles issued so far (buffer g & 1; continues across items)
      int nk = 0, nv = 0;
      FwdItem item;
      for (int kk = 0; ok && fwd_item<CAUSAL>(p.n_items, p.n_qblocks, p.BH, kk, item); ++kk) {
        const auto sch = sched_of(item);
        if (!mbar_wait(&bars->q_full, kk & 1, wc, kSite256Q)) { ok = false; break; }
        tc_fence_after();
        int j = sch.first();
        if (j >= 0) {
          if (!mbar_wait(&bars->k_full, nk & 1, wc, kSite256KFull)) { ok = false; break; }
          tc_fence_after();
          issue_s(g & 1);
          mma_commit(&bars->k_empty);
          mma_commit(&bars->s_full[g & 1]);
          ++nk;
        } else {
          mma_commit(&bars->q_empty);  // nothing to do for this tile
        }
        bool first_pv = true;
        while (j >= 0) {
          const int jn = sch.next(j);
          const int b = g & 1;
          if (jn >= 0) {
            // The next scores into the other buffer (its P was consumed by the previous
            // P V, issued before this in order).
            if (!mbar_wait(&bars->k_full, nk & 1, wc, kSite256KFull)) { ok = false; break; }
            tc_fence_after();
            issue_s(b ^ 1);
            mma_commit(&bars->k_empty);
            mma_commit(&bars->s_full[b ^ 1]);
            ++nk;
          } else {
            mma_commit(&bars->q_empty);  // every S product of the item is issued
          }
          if (!mbar_wait(&bars->p_ready[b], (g >> 1) & 1, wc, kSite256PReady)) { ok = false; break; }
          if (first_pv && kk > 0 && !mbar_wait(&bars->o_empty, (kk - 1) & 1, wc, kSite256OEmpty)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&bars->v_full, nv & 1, wc, kSite256VFull)) { ok = false; break; }
          tc_fence_after();
          issue_pv(b, !first_pv);
          mma_commit(&bars->v_empty);
          mma_commit(&bars->pv_done);
          ++nv;
          first_pv = false;
          ++g;
          j = jn;
        }
        if (!ok) break;
        mma_commit(&bars->o_full);
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, wc, kSite256Drain);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmCols);
  } else if (warp == 3) {
    __syncthreads();
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    const float c = p.c_log2;
    const uint32_t kb0[4] = {0u, 0u, 0u, 0u};
    bool ok = true;
    int g = 0;   // score tiles consumed so far
    FwdItem item;
    for (int kk = 0; ok && fwd_item<CAUSAL>(p.n_items, p.n_qblocks, p.BH, kk, item); ++kk) {
      const auto sch = sched_of(item);
      const int tile = item.qb;
      float m = -INFINITY, l = 0.f;
      int local = 0;
      for (int j = sch.first(); j >= 0; j = sch.next(j), ++g, ++local) {
        const int b = g & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[b], (g >> 1) & 1, wc, kSite256SFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[128];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t raw[32];
          tmem_ld32(trow + Cfg::tm_s(b) + q4 * 32, raw);
#pragma unroll
          for (int t = 0; t < 32; ++t) s[q4 * 32 + t] = __uint_as_float(raw[t]);
        }
        tmem_wait_ld();
        float sum, alpha, m_use;
        int dbase = 0;
        if constexpr (XQK) {
          const long long db64 = 128LL * (tile - j) + off_;
          dbase = static_cast<int>(db64 < -256 ? -256 : (db64 > 256 ? 256 : db64));
        }
        const bool diag = CAUSAL && (XQK ? dbase < 127 : j == tile);
        const int nk_last = p.Nk - 128 * (p.n_ktiles - 1);
        const bool tail = !CAUSAL && j == p.n_ktiles - 1 && nk_last != 128;
        if (diag || tail) {
          int lim = diag ? r + 1 + dbase : nk_last;
          if (XQK && lim < 0) lim = 0;
          softmax_row<true, PolyShare<D>::kFwd>(s, lim, c, m, trow + Cfg::tm_s(b), sum, alpha, m_use, kb0, 1.f);
        } else {
          softmax_row<false, PolyShare<D>::kFwd>(s, 128, c, m, trow + Cfg::tm_s(b), sum, alpha, m_use, kb0, 1.f);
        }
        l = l * alpha + sum;
        if (__any_sync(0xffffffffu, m_use != m) && local > 0) {
          // O is rescaled in place: the previous tile's P V product must be complete (the
          // scores of this tile may have finished before it).
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (g - 1) & 1, wc, kSite256PvDone))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t ov[32];
            tmem_ld32(trow + Cfg::kTmO + cc * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) ov[t] = __float_as_uint(__uint_as_float(ov[t]) * alpha);
            tmem_st32(trow + Cfg::kTmO + cc * 32, ov);
          }
        }
        m = m_use;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_ready[b]);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_full, kk & 1, wc, kSite256OFull))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const size_t row = size_t(item.bh) * p.N + size_t(tile) * 128 + r;  // lse index
      const int ib = item.bh / p.H, ih = item.bh - ib * p.H;
      __nv_bfloat16* orow = p.o + seq_row_offset(ib, ih, tile * 128 + r, p.N, p.H, D, p.bnhd != 0);
      const bool row_ok = tile * 128 + r < p.N;
      if (local > 0) {
        const float inv_l = (!XQK || l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(trow + Cfg::kTmO + cc * 32, ov);
          tmem_wait_ld();
          uint32_t pw[16];
#pragma unroll
          for (int t = 0; t < 16; ++t)
            pw[t] = pack_bf16(__uint_as_float(ov[2 * t]) * inv_l, __uint_as_float(ov[2 * t + 1]) * inv_l);
          if (row_ok) store_row64(orow + cc * 32, pw, p.v8 != 0);
        }
        tc_fence_before();
        mbar_arrive(&bars->o_empty);
        if (row_ok) p.lse[row] = (!XQK || l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      } else {
        mbar_arrive(&bars->o_empty);
        if (row_ok) {
          const uint4 z = make_uint4(0, 0, 0, 0);
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int t = 0; t < D / 8; ++t) dst[t] = z;
          p.lse[row] = -INFINITY;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
}

}  // namespace fa
