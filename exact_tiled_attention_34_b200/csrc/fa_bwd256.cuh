// fa_bwd256.cuh - backward for head dim 256: dK, dV and dQ from one kernel, with dQ
// reduced in fp32 into the workspace by TMA reduce-add (as fa_bwd_fused.cuh).
//
// The recomputation scheme is the same ("Researchers at Stanford University Propose
// FlashAttention ..." summary, method paragraph): per (key tile j, query tile),
//   S^T = K_j Q^T, dP^T = V_j dO^T, dV_j += P^T dO, dK_j += dS^T Q, dQ += dS K_j.
// At head dim 256 the fp32 dK_j and dV_j alone would fill the 512 tensor-memory
// columns, and K_j, V_j, Q and dO tiles of 128 rows would need 256 KB of shared memory.
// So a work item is (key tile j, batch*head, column half c): it accumulates dK_j and
// dV_j for head-dim columns [128c, 128c + 128) only and adds dQ's share of the same
// columns; S^T and dP^T (reductions over all 256 columns) are formed by both halves' items.
// Query rows are visited in sub-tiles of 64 (Q and dO 32 KB each, single-buffered), and
// dQ's share is formed transposed, dQ^T = K_j[:, c]^T dS^T (M = 128 head-dim rows, N =
// 64 queries), so every product keeps M = 128.
//   warp 0      TMA producer: K_j, V_j per item; Q and dO (+ row arrays) per sub-tile
//   warp 1      MMA issuer + TMEM owner
//   warps 4-11  compute warpgroups (thread = key row; warpgroup h takes query columns
//               [32h, 32h + 32) of S^T and dP^T; in the dQ drain, thread = head-dim row)
// Tensor memory: dK_c | dV_c | X (S^T, then P^T packed) | Y (dP^T) | Z (dQ^T).
// Shared memory: K 64 KB | V 64 KB | Q 32 KB | dO 32 KB | dS^T 16 KB (key rows of 128 B;
// K-major A operand of dK, N-major B operand of dQ^T; then the dQ staging area) | rows.
#pragma once

#include "fa_bwd_fused.cuh"

namespace fa {

struct Bwd256Cfg {
  static constexpr int kKvBlock = 128 * 128;   // one 64-column block of a 128-row tile
  static constexpr int kSubBlock = 64 * 128;   // one 64-column block of a 64-row sub-tile
  static constexpr int kKvBytes = 4 * kKvBlock;
  static constexpr int kSubBytes = 4 * kSubBlock;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKvBytes;
  static constexpr int kOffQ = kOffV + kKvBytes;
  static constexpr int kOffDO = kOffQ + kSubBytes;
  static constexpr int kOffDS = kOffDO + kSubBytes;   // 128 key rows x 128 bytes
  static constexpr int kOffL = kOffDS + 16384;        // -lse log2 e of the sub-tile's 64 rows
  static constexpr int kOffDr = kOffL + 256;          // D of the sub-tile's 64 rows
  static constexpr int kOffBar = kOffDr + 256;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "backward (head dim 256) shared memory above the per-block limit");
  static constexpr uint32_t kTmDK = 0, kTmDV = 128, kTmX = 256, kTmY = 320, kTmZ = 384, kTmCols = 512;
};

struct Bwd256Bars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full, q_empty;    // Q sub-tile + row arrays; empty: S^T and dK done with it
  uint64_t do_full, do_empty;  // empty: dP^T and dV done with it
  uint64_t s_full, dp_full, dq_full;
  uint64_t p_ready, ds_ready, dq_taken;  // 256 arrivals
  uint64_t acc_done, acc_empty;                // acc_empty: 256
  uint64_t pair[4];   // 64 arrivals: both warps of a lane quarter are done with their dQ staging
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

enum Bwd256Site : int {
  kSiteB256KV = 501, kSiteB256KvEmpty, kSiteB256QEmpty, kSiteB256DoEmpty, kSiteB256QFull, kSiteB256DoFull,
  kSiteB256PReady, kSiteB256DsReady, kSiteB256Acc, kSiteB256SFull, kSiteB256DpFull, kSiteB256DqFull,
  kSiteB256Read, kSiteB256Drain
};

// 64-row query sub-tiles that see key tile j (key j' visible to query i iff j' <= i + off).
template <bool CAUSAL, bool SPARSE, bool XQK>
struct SubSched256 {
  int j, n_sub, n_ktiles, u_first;
  const uint8_t* mask;  // [n_tiles, n_ktiles] at 128-row granularity
  __device__ __forceinline__ SubSched256(int j_, int n_sub_, int n_ktiles_, int off, const uint8_t* mask_)
      : j(j_), n_sub(n_sub_), n_ktiles(n_ktiles_), mask(mask_) {
    int f = 0;
    if (CAUSAL) {
      // sub-tile u (rows 64u .. 64u + 63) sees some of key tile j iff 64u + 63 + off >= 128j
      const long long x = 128LL * j_ - 63 - (XQK ? off : 0);
      f = x <= 0 ? 0 : static_cast<int>((x + 63) >> 6);
    }
    u_first = f;
  }
  __device__ __forceinline__ int next(int u0) const {
    for (int u = (u0 + 1 > u_first ? u0 + 1 : u_first); u < n_sub; ++u)
      if (!SPARSE || mask[size_t(u >> 1) * n_ktiles + j] != 0) return u;
    return -1;
  }
  __device__ __forceinline__ int first() const { return next(-1); }
};

// Register split of the 384-thread block (launched with 168 per thread, 64,512 in all):
// the producer/MMA warpgroup drops to 120, the compute warpgroups rise to 192:
// 128 * (120 + 2 * 192) = 64,512. Only the compute warpgroups increase, once, by what
// the first releases.
constexpr int kBwd256RegsCtl = 120;
constexpr int kBwd256RegsCompute = 192;
constexpr int kBwd256RegsNeeded = 128 * (kBwd256RegsCtl + 2 * kBwd256RegsCompute);

template <bool CAUSAL, bool SPARSE, bool XQK>
__global__ void __launch_bounds__(kBwdThreads, 1)
fa_bwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using Cfg = Bwd256Cfg;
  const int off_ = XQK ? p.off : 0;
  const int n_sub = (p.N + 63) / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  Bwd256Bars* bars = reinterpret_cast<Bwd256Bars*>(smem + Cfg::kOffBar);
  uint8_t* sK = smem + Cfg::kOffK;
  uint8_t* sV = smem + Cfg::kOffV;
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sDO = smem + Cfg::kOffDO;
  uint8_t* sDS = smem + Cfg::kOffDS;
  float* sL = reinterpret_cast<float*>(smem + Cfg::kOffL);
  float* sDr = reinterpret_cast<float*>(smem + Cfg::kOffDr);
  const int warp = warp_id();
  const int lane = lane_id();
  WaitCtl wc{&bars->abort, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->do_full, 1);
    mbar_init(&bars->do_empty, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->p_ready, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->dq_taken, 256);
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->acc_empty, 256);
    for (int q = 0; q < 4; ++q) mbar_init(&bars->pair[q], 64);
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

  // Work item k of this CTA: key tile j, column half c, batch*head.
  auto item_of = [&](int k, int& j, int& c, int& bh) -> bool {
    BwdItem it;
    if (!bwd_item<CAUSAL, true>(2 * p.n_ktiles, p.BH, k, it)) return false;
    j = it.tile >> 1;
    c = it.tile & 1;
    bh = it.bh;
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    regs_dec<kBwd256RegsCtl>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint64_t keep = policy_evict_last();
      int n = 0, nkv = 0, nq = 0, ndo = 0;
      bool ok = p.stall == 0;
      int j, c, bh;
      for (int kk = 0; ok && item_of(kk, j, c, bh); ++kk) {
        const int ib = bh / p.H, ih = bh - ib * p.H;
        SubSched256<CAUSAL, SPARSE, XQK> sch{j, n_sub, p.n_ktiles, off_, p.tile_mask};
        if (kk > 0 && !mbar_wait(&bars->kv_empty, (kk - 1) & 1, wc, kSiteB256KvEmpty)) break;
        mbar_arrive_expect_tx(&bars->kv_full, 2 * Cfg::kKvBytes);
        for (int cb = 0; cb < 4; ++cb) {
          tma_load_4d(sK + cb * Cfg::kKvBlock, &tm_k, &bars->kv_full, cb * 64, j * 128, ih, ib);
          tma_load_4d(sV + cb * Cfg::kKvBlock, &tm_v, &bars->kv_full, cb * 64, j * 128, ih, ib);
        }
        ++nkv;
        for (int u = sch.first(); u >= 0; u = sch.next(u), ++n) {
          // dO is released (after dV) before Q (after dK and dQ^T): load it first.
          if (n > 0 && !mbar_wait(&bars->do_empty, (n - 1) & 1, wc, kSiteB256DoEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->do_full, Cfg::kSubBytes);
          for (int cb = 0; cb < 4; ++cb)
            tma_load_4d_hint(sDO + cb * Cfg::kSubBlock, &tm_do, &bars->do_full, cb * 64, u * 64, ih, ib, keep);
          ++ndo;
          if (n > 0 && !mbar_wait(&bars->q_empty, (n - 1) & 1, wc, kSiteB256QEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->q_full, Cfg::kSubBytes + 512);
          for (int cb = 0; cb < 4; ++cb)
            tma_load_4d_hint(sQ + cb * Cfg::kSubBlock, &tm_q, &bars->q_full, cb * 64, u * 64, ih, ib, keep);
          const size_t roff = size_t(bh) * p.n_tiles * 128 + size_t(u) * 64;  // padded row arrays
          bulk_load(sL, p.lse2 + roff, 256, &bars->q_full);
          bulk_load(sDr, p.Drow + roff, 256, &bars->q_full);
          ++nq;
        }
      }
      if (bars->abort) {
        if (nkv > 0) mbar_wait_drain(&bars->kv_full, (nkv - 1) & 1, wc, kSiteB256Drain);
        if (nq > 0) mbar_wait_drain(&bars->q_full, (nq - 1) & 1, wc, kSiteB256Drain);
        if (ndo > 0) mbar_wait_drain(&bars->do_full, (ndo - 1) & 1, wc, kSiteB256Drain);
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kBwd256RegsCtl>();
    if (lane == 0) {
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO);
      const uint32_t aDS = smem_u32(sDS);
      constexpr uint32_t idNT = idesc_bf16_f32(128, 64, 0, 0);   // S^T, dP^T: 128 keys x 64 queries
      constexpr uint32_t idTN = idesc_bf16_f32(128, 128, 0, 1);  // dV_c, dK_c: 128 keys x 128 columns
      constexpr uint32_t idQT = idesc_bf16_f32(128, 64, 1, 1);   // dQ^T: 128 columns x 64 queries
      // X[128 x 64] = A[128 x 256] B[64 x 256]^T, both K-major (A: 128-row blocks, B: 64-row blocks)
      auto nt = [&](uint32_t tm, uint32_t a, uint32_t b) {
#pragma unroll
        for (int k = 0; k < 16; ++k)
          mma_ss(tm, sdesc_sw128(a + (k >> 2) * Cfg::kKvBlock + (k & 3) * 32, 16, 1024),
                 sdesc_sw128(b + (k >> 2) * Cfg::kSubBlock + (k & 3) * 32, 16, 1024), idNT, k > 0);
      };
      bool ok = true;
      int n = 0;  // sub-tiles processed so far (continues across items)
      int j, c, bh;
      for (int kk = 0; ok && item_of(kk, j, c, bh); ++kk) {
        SubSched256<CAUSAL, SPARSE, XQK> sch{j, n_sub, p.n_ktiles, off_, p.tile_mask};
        if (!mbar_wait(&bars->kv_full, kk & 1, wc, kSiteB256KV)) { ok = false; break; }
        tc_fence_after();
        int u = sch.first();
        if (u < 0) mma_commit(&bars->kv_empty);
        if (u >= 0) {
          if (!mbar_wait(&bars->q_full, n & 1, wc, kSiteB256QFull)) { ok = false; break; }
          tc_fence_after();
          nt(tmem + Cfg::kTmX, aK, aQ);
          mma_commit(&bars->s_full);
          if (!mbar_wait(&bars->do_full, n & 1, wc, kSiteB256DoFull)) { ok = false; break; }
          tc_fence_after();
          nt(tmem + Cfg::kTmY, aV, aDO);
          mma_commit(&bars->dp_full);
        }
        bool first = true;
        while (u >= 0) {
          const int un = sch.next(u);
          if (!mbar_wait(&bars->p_ready, n & 1, wc, kSiteB256PReady)) { ok = false; break; }
          if (first && kk > 0 && !mbar_wait(&bars->acc_empty, (kk - 1) & 1, wc, kSiteB256Acc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dV_c += P^T dO[:, c]   (P^T packed in X; dO column blocks 2c, 2c + 1)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts(tmem + Cfg::kTmDV, tmem + Cfg::kTmX + (k >> 1) * 32 + (k & 1) * 8,  // P^T of warpgroup k / 2
                   sdesc_sw128(aDO + 2 * c * Cfg::kSubBlock + k * 2048, Cfg::kSubBlock, 1024), idTN,
                   (!first || k > 0) ? 1u : 0u);
          mma_commit(&bars->do_empty);
          if (!mbar_wait(&bars->ds_ready, n & 1, wc, kSiteB256DsReady)) { ok = false; break; }
          tc_fence_after();
          // dK_c += dS^T Q[:, c]   (dS^T K-major in shared memory: 128 keys x 64 queries)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss(tmem + Cfg::kTmDK, sdesc_sw128(aDS + k * 32, 16, 1024),
                   sdesc_sw128(aQ + 2 * c * Cfg::kSubBlock + k * 2048, Cfg::kSubBlock, 1024), idTN,
                   (!first || k > 0) ? 1u : 0u);
          mma_commit(&bars->q_empty);  // dK's product is the last to read this Q sub-tile
          // dQ^T = K[:, c]^T dS^T   (K read MN-major: head-dim rows; dS^T N-major: query columns)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tmem + Cfg::kTmZ, sdesc_sw128(aK + 2 * c * Cfg::kKvBlock + k * 2048, Cfg::kKvBlock, 1024),
                   sdesc_sw128(aDS + k * 2048, 16, 1024), idQT, k > 0 ? 1u : 0u);
          mma_commit(&bars->dq_full);
          if (un < 0) mma_commit(&bars->kv_empty);
          if (un >= 0) {
            if (!mbar_wait(&bars->q_full, (n + 1) & 1, wc, kSiteB256QFull)) { ok = false; break; }
            tc_fence_after();
            nt(tmem + Cfg::kTmX, aK, aQ);
            mma_commit(&bars->s_full);
            if (!mbar_wait(&bars->do_full, (n + 1) & 1, wc, kSiteB256DoFull)) { ok = false; break; }
            tc_fence_after();
            nt(tmem + Cfg::kTmY, aV, aDO);
            mma_commit(&bars->dp_full);
          }
          first = false;
          u = un;
          ++n;
        }
        if (!ok) break;
        mma_commit(&bars->acc_done);
      }
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, wc, kSiteB256Drain);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmCols);
  } else if (warp < 4) {
    regs_dec<kBwd256RegsCtl>();
    __syncthreads();
  } else {
    // ------------------------------------------------------------ compute warpgroups
    regs_inc<kBwd256RegsCompute>();
    const int h = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row (S^T, dP^T, dK, dV) / head-dim row (dQ^T)
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    const float c2 = p.scale * 1.4426950408889634f;
    // dQ staging: 2 KB (16 query rows x 32 fp32 columns) per warp, inside the key rows
    // 32 quarter .. +31 of the dS^T buffer, which this warp and its partner in the other
    // warpgroup (same quarter) write: the pair synchronises (pair[quarter]) before
    // writing dS^T again.
    uint8_t* my_stage = sDS + quarter * 4096 + h * 2048;
    uint8_t* my_ds = sDS + r * 128;
    bool ok = true;
    int n = 0;
    // dQ^T of sub-tile t (rows 64 ut ..) out of tensor memory into dQacc rows
    // [64 ut + 32h, +32), columns [128c + 32 quarter, +32), as two 16-row boxes.
    auto drain = [&](int t, int ut, int c, int bh) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->dq_full, t & 1, wc, kSiteB256DqFull))) return false;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(trow + Cfg::kTmZ + h * 32, v);  // this thread's head-dim row, 32 queries
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->dq_taken);
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        if (b > 0) {
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
        }
        uint32_t* s32 = reinterpret_cast<uint32_t*>(my_stage);
#pragma unroll
        for (int i = 0; i < 16; ++i)  // query row i of the box, column = lane
          s32[i * 32 + ((((lane >> 2) ^ (i & 7)) << 2) | (lane & 3))] = v[b * 16 + i];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tm_dqacc, my_stage, c * 128 + quarter * 32, ut * 64 + h * 32 + b * 16, bh);
          bulk_commit();
        }
      }
      return true;
    };
    int j, c, bh;
    for (int kk = 0; ok && item_of(kk, j, c, bh); ++kk) {
      SubSched256<CAUSAL, SPARSE, XQK> sch{j, n_sub, p.n_ktiles, off_, p.tile_mask};
      const bool kvalid = j * 128 + r < p.Nk;
      int local = 0, prev_u = -1;
      for (int u = sch.first(); u >= 0; u = sch.next(u), ++n, ++local) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->q_full, n & 1, wc, kSiteB256QFull)) ||
            !__all_sync(0xffffffffu, mbar_wait(&bars->s_full, n & 1, wc, kSiteB256SFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // query 64u + cq sees key 128j + r iff cq >= r + cbase
        int cbase = 0;
        bool diag = false;
        if constexpr (CAUSAL) {
          const long long cb64 = 128LL * j - 64LL * u - off_;
          cbase = static_cast<int>(cb64 < -256 ? -256 : (cb64 > 256 ? 256 : cb64));
          diag = cbase > -127;
        }
        const int cmin = cbase + r;
        uint32_t pk[16];
        {
          uint32_t raw[32];
          tmem_ld32(trow + Cfg::kTmX + h * 32, raw);
          tmem_wait_ld();
          const uint64_t c2v = f2(c2, c2);
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int c0 = 2 * t;
            const float2 nl = *reinterpret_cast<const float2*>(sL + h * 32 + c0);
            uint64_t pv = ex2_mufu_x2(
                f2_fma(f2(__uint_as_float(raw[c0]), __uint_as_float(raw[c0 + 1])), c2v, f2(nl.x, nl.y)));
            if (diag) {
              const float2 x = f2_split(pv);
              pv = f2((h * 32 + c0 < cmin) ? 0.f : x.x, (h * 32 + c0 + 1 < cmin) ? 0.f : x.y);
            }
            const float2 x = f2_split(pv);
            pk[t] = kvalid ? pack_bf16(x.x, x.y) : 0u;
          }
        }
        // P^T over the first half of this warpgroup's own 32 score columns: this thread has
        // read its row of them, and no other thread reads this row.
        tmem_st16(trow + Cfg::kTmX + h * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_ready);
        if (local > 0 && !drain(n - 1, prev_u, c, bh)) {
          ok = false;
          break;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full, n & 1, wc, kSiteB256DpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t ds[16];
        {
          uint32_t dpr[32];
          tmem_ld32(trow + Cfg::kTmY + h * 32, dpr);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const float2 pp = unpack_bf16(pk[t]);
            const float2 dd = *reinterpret_cast<const float2*>(sDr + h * 32 + 2 * t);
            const uint64_t diff =
                f2_sub(f2(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1])), f2(dd.x, dd.y));
            const float2 x = f2_split(f2_mul(f2(pp.x, pp.y), diff));
            ds[t] = pack_bf16(x.x, x.y);
          }
        }
        // This pair's staging copies must have left the buffer before dS^T overwrites it
        // (a bounded mbarrier wait, so that a partner that gave up cannot strand this warp).
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        mbar_arrive(&bars->pair[quarter]);
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->pair[quarter], n & 1, wc, kSiteB256Read))) {
          ok = false;
          break;
        }
        {
          uint4* d4 = reinterpret_cast<uint4*>(my_ds);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            d4[(4 * h + cc) ^ (r & 7)] = make_uint4(ds[4 * cc], ds[4 * cc + 1], ds[4 * cc + 2], ds[4 * cc + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready);
        prev_u = u;
      }
      if (!ok) break;
      if (local > 0 && !drain(n - 1, prev_u, c, bh)) {
        ok = false;
        break;
      }
      // -------------------------------------------------------- epilogue: dK_c (h = 0), dV_c (h = 1)
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, kk & 1, wc, kSiteB256Acc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int ib = bh / p.H, ih = bh - ib * p.H;
      __nv_bfloat16* dst = (h == 0 ? p.dk : p.dv) + seq_row_offset(ib, ih, j * 128 + r, p.Nk, p.H, 256, p.bnhd != 0) +
                           c * 128;
      const float mul = h == 0 ? p.scale : 1.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t acc[32];
        if (local > 0) {
          tmem_ld32(trow + (h == 0 ? Cfg::kTmDK : Cfg::kTmDV) + cc * 32, acc);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) acc[t] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int t = 0; t < 16; ++t)
          w[t] = pack_bf16(__uint_as_float(acc[2 * t]) * mul, __uint_as_float(acc[2 * t + 1]) * mul);
        if (kvalid) store_row64(dst + cc * 32, w, p.v8 != 0);
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  }
}

}  // namespace fa
