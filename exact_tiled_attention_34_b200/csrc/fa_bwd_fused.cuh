// fa_bwd_fused.cuh - single-kernel backward: dK, dV and dQ from one pass over the
// (key tile, query tile) pairs, with dQ reduced into an fp32 accumulator in global
// memory by tensor-memory-accelerator reduce-add copies.
//
// The pages' recomputation scheme ("Researchers at Stanford University Propose
// FlashAttention ..." summary, method paragraph: the backward recomputes attention on
// chip from the saved normalisation factor) gives, for each pair (key tile j, query
// tile i), the five products
//   S^T = K_j Q_i^T,  dP^T = V_j dO_i^T,  dV_j += P^T dO_i,  dK_j += dS^T Q_i,
//   dQ_i += dS K_j.
// The deterministic path (fa_bwd.cuh) runs the first four in a key-tile-parallel
// kernel and recomputes S and dP in a second, query-tile-parallel kernel for dQ
// (seven products). Here all five run once: dQ_i's share from key tile j is written
// to tensor memory and added into fp32 dQacc[b, h, i] with cp.reduce.async.bulk.tensor
// (whole 128-byte lines reduced in L2). The order in which key tiles add into a dQ
// row varies from run to run, so dQ is not bit-reproducible (dK and dV are).
//
// Work item = (128-key tile j, batch*head) as in the dK/dV kernel; 512 threads:
//   warp 0       TMA producer: K_j, V_j per item; Q_i (+ row arrays) and dO_i per tile
//   warp 1       MMA issuer + TMEM owner
//   warps 4-11   two compute warpgroups (thread = key row = TMEM lane; warpgroup h
//                takes query columns [64h, 64h + 64) of S^T and dP^T)
//   warps 12-15  dQ warpgroup (thread = query row = TMEM lane): dQ_i out of tensor
//                memory, through shared memory, into dQacc by reduce-add copies
// dS leaves the compute warps through shared memory (bf16, 128 x 128, 128-byte
// swizzle, [query block of 64][key row][128 B]); that one buffer is the K-major A
// operand of dK += dS^T Q and the MN-major A operand of dQ = dS K. Each dQ warp stages
// its 32 dQ rows (fp32, 32 x 32 boxes, 4 KB each) for the reduce-add in a stage area of
// its own (8 KB per warp, two boxes); at head dim 128 a warp's other two boxes wait in
// registers until the first two copies have read the area. With the drain in warps of
// its own, the compute warps go from one tile's dS straight to the next tile's
// exponentials, and at head dim 128 dQ's product goes before dK's so that dQ's columns
// (which the next dP^T reuses) are read out while dK's product runs.
//
// Tensor memory (512 columns): dK | dV | X (S^T, then P^T as packed bf16) |
// Y (dP^T; at head dim 128 also dQ) | Z (dQ at head dim 64). At head dim 128 the five
// buffers do not fit, so dQ_i shares Y with dP^T: dP^T of the next tile is issued once
// the dQ warps have read dQ_i out (while the compute warps run the next tile's
// exponentials). At head dim 64 the next dQ product waits for the same read.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

template <int D>
struct FusedCfg {
  static constexpr int kBlockBytes = 128 * 128;  // one 64-column block of a 128-row bf16 tile
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kDoStages = (D == 128) ? 1 : 2;  // dO ring depth (shared memory is short at 128)
  // K_j, V_j per item: at head dim 64 two stages, so that the next item's tiles load while
  // this item's last query tiles run (the item boundary then costs little more than the
  // dK/dV epilogue); at 128 one.
  static constexpr int kKvStages = (D == 128) ? 1 : 2;
  static constexpr int kOffK = 0;                                   // kKvStages stages
  static constexpr int kOffV = kOffK + kKvStages * kTileBytes;      // kKvStages stages
  static constexpr int kOffQ = kOffV + kKvStages * kTileBytes;      // 2 stages
  static constexpr int kOffDO = kOffQ + 2 * kTileBytes;             // kDoStages stages
  static constexpr int kOffDS = kOffDO + kDoStages * kTileBytes;    // dS bf16 128 x 128 / dQ stages
  static constexpr int kOffL = kOffDS + 32768;                      // -lse log2 e rows, 2 stages
  static constexpr int kOffDr = kOffL + 1024;                       // D rows, 2 stages
  // dQ stage area, 8 KB per dQ warp (two 4 KB boxes at a time).
  static constexpr int kOffStage = kOffDr + 1024;
  static constexpr int kOffBar = kOffStage + 32768;
  // Barriers (well under 256 bytes), plus 1 KB of alignment slack at head dim 64. At head
  // dim 128 there is no room for the slack: the kernel then requires the dynamic
  // shared-memory base to be 1024-byte aligned (it is when, as here, the kernel declares
  // no static shared memory) and returns with an error status if it is not.
  static constexpr bool kAlignedBase = (D == 128);
  static constexpr int kSmemBytes = kOffBar + 256 + (kAlignedBase ? 0 : 1024);
  static_assert(kSmemBytes <= 227 * 1024, "fused backward shared memory above the per-block limit");
  static constexpr uint32_t kTmDK = 0;
  static constexpr uint32_t kTmDV = D;
  static constexpr uint32_t kTmX = 2 * D;
  static constexpr uint32_t kTmY = 2 * D + 128;
  static constexpr bool kDqInY = (D == 128);
  static constexpr uint32_t kTmDQ = kDqInY ? kTmY : 2 * D + 256;
  static_assert(kTmDQ + D <= 512, "fused backward tensor memory above 512 columns");
  static constexpr uint32_t kTmCols = 512;
};

struct FusedBars {
  uint64_t kv_full[2];
  uint64_t kv_empty[2];  // every product of the item that reads K_j or V_j is done
  uint64_t q_full[2];    // Q_i and the row arrays of tile i
  uint64_t q_empty[2];
  uint64_t do_full[2];
  uint64_t do_empty[2];
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t dq_full;      // dQ_i's product is done
  uint64_t p_ready;      // 256 arrivals: P^T is in tensor memory
  uint64_t ds_ready;     // 256: dS is in shared memory and dP^T has been read
  uint64_t dq_taken;     // 128: dQ_i has been read out of tensor memory
  uint64_t acc_done;
  uint64_t acc_empty;    // 256: the epilogue has read dK and dV
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

enum FusedSite : int {
  kSiteFuKV = 301, kSiteFuQEmpty, kSiteFuDoEmpty, kSiteFuKvEmpty, kSiteFuQFull, kSiteFuDoFull, kSiteFuPReady,
  kSiteFuDsReady, kSiteFuDqTaken, kSiteFuAcc, kSiteFuSFull, kSiteFuDpFull, kSiteFuDqFull,
  kSiteFuDrain,
  kSiteFuSmemAlign = 399  // reported with kStatusUnsupported: dynamic shared memory not 1024-aligned
};
constexpr int kStatusUnsupported = 2;  // == FA_ERR_UNSUPPORTED

// dK += dS^T Q_i: A = dS^T from shared memory (K-major: key rows, query columns in
// 64-wide blocks), B = Q_i (N-major), 8 steps of 16 queries.
template <int D>
__device__ __forceinline__ void mma_dk_ss(uint32_t tm, uint32_t a_ds, uint32_t b_q, bool acc) {
  constexpr uint32_t id = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t aoff = (k >> 2) * 16384 + (k & 3) * 32;
    mma_ss(tm, sdesc_sw128(a_ds + aoff, 16, 1024), sdesc_sw128(b_q + k * 2048, 16384, 1024), id,
           (acc || k > 0) ? 1u : 0u);
  }
}

// dV += P^T dO_i: A = P^T packed bf16 in tensor memory, where compute warpgroup h left
// its 64 queries in the first 32 of its own 64 score columns (X + 64h), so that no
// warpgroup overwrites scores the other has yet to read; B = dO_i (N-major), 8 steps of
// 16 queries.
template <int D>
__device__ __forceinline__ void mma_dv_ts(uint32_t tm, uint32_t a_tm, uint32_t b, bool acc) {
  constexpr uint32_t id = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mma_ts(tm, a_tm + (k >> 2) * 64 + (k & 3) * 8, sdesc_sw128(b + k * 2048, FusedCfg<D>::kBlockBytes, 1024), id,
           (acc || k > 0) ? 1u : 0u);
}

// dQ = dS K_j: A = dS from the same buffer read MN-major (query rows contiguous in
// 64-wide blocks, 16384 bytes apart; key = reduction index, 128 bytes per key),
// B = K_j (N-major: key rows, head-dim columns), 8 steps of 16 keys. Overwrites tm.
template <int D>
__device__ __forceinline__ void mma_dq_ss(uint32_t tm, uint32_t a_ds, uint32_t b_k) {
  constexpr uint32_t id = idesc_bf16_f32(128, D, 1, 1);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mma_ss(tm, sdesc_sw128(a_ds + k * 2048, 16384, 1024), sdesc_sw128(b_k + k * 2048, 16384, 1024), id,
           k > 0 ? 1u : 0u);
}

// The items one CTA visits, in order. Causal and `paired`: key tiles j and n - 1 - j of
// one head form a pair that costs n + 1 query tiles in all, so pairs are uniform and
// need no costliest-first order; pairs are dealt head-major by item_position's
// alternating deal, so the CTAs at work at any time hold the pairs of a few heads, and
// those heads' Q, dO and dQ accumulator rows stay in L2 while all their key tiles add
// into them (dealing single items costliest first spreads every head over the whole
// run). A middle tile (n odd) is a pair of one item. The launcher pairs only when the
// pairs fill the last round of CTAs well; otherwise (and when not causal) bwd_item's
// order.
template <bool CAUSAL>
struct FusedWalk {
  int n, BH, paired;
  int k = 0;         // pair (or item) position of this CTA
  bool second = false;
  __device__ __forceinline__ bool next(BwdItem& it) {
    if (!CAUSAL || !paired) return bwd_item<CAUSAL, true>(n, BH, k++, it);
    const int n_pairs = (n + 1) >> 1;
    const long long pos = item_position(static_cast<long long>(n_pairs) * BH, k);
    if (pos < 0) return false;
    const int pr = static_cast<int>(pos % n_pairs);
    it.bh = static_cast<int>(pos / n_pairs);
    if (second) {
      it.tile = n - 1 - pr;
      second = false;
      ++k;
    } else {
      it.tile = pr;
      second = n - 1 - pr != pr;
      if (!second) ++k;
    }
    return true;
  }
};

// Register split of the 512-thread block (launched with 128 per thread, 65,536 in all):
// the producer/MMA warpgroup drops to 96 (the issuer keeps the descriptors of five
// products in registers), the dQ warpgroup keeps 96 (64 hold two boxes of dQ), the
// compute warpgroups rise to 160: 128 * (96 + 96 + 2 * 160) = 65,536. Only the compute
// warpgroups increase, once, by what the first releases.
constexpr int kFusedThreads = 512;
constexpr int kFusedRegsCtl = 96;
constexpr int kFusedRegsDrain = 96;
constexpr int kFusedRegsCompute = 160;
constexpr int kFusedRegsNeeded = 128 * (kFusedRegsCtl + kFusedRegsDrain + 2 * kFusedRegsCompute);
static_assert(kFusedRegsNeeded <= 65536, "fused backward register split above the register file");

template <int D, bool CAUSAL, bool SPARSE, bool XQK>
__global__ void __launch_bounds__(kFusedThreads, 1)
fa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using Cfg = FusedCfg<D>;
  constexpr int SD = Cfg::kDoStages;
  constexpr int SKV = Cfg::kKvStages;
  const int off_ = XQK ? p.off : 0;
  extern __shared__ uint8_t smem_raw[];
  if (Cfg::kAlignedBase && (smem_u32(smem_raw) & 1023u) != 0) {
    // Every thread leaves before any barrier, copy or tensor-memory allocation.
    if (threadIdx.x == 0 && atomicCAS(p.status, 0, kStatusUnsupported) == 0) atomicExch(p.status + 1, kSiteFuSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
  FusedBars* bars = reinterpret_cast<FusedBars*>(smem + Cfg::kOffBar);
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
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->do_full[s], 1);
      mbar_init(&bars->do_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->p_ready, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->dq_taken, 128);
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
    regs_dec<kFusedRegsCtl>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const uint64_t keep = policy_evict_last();
      int it = 0;   // query tiles loaded so far (continues across items)
      int nkv = 0;  // K/V tiles loaded so far
      int nq = 0, ndo = 0;  // Q and dO loads issued (for the drain on abort)
      bool ok = p.stall == 0;
      BwdItem item;
      FusedWalk<CAUSAL> walk{p.n_ktiles, p.BH, p.paired};
      for (int kk = 0; ok && walk.next(item); ++kk) {
        const int j = item.tile, bh = item.bh;
        const int ib = bh / p.H, ih = bh - ib * p.H;
        KeySched<CAUSAL, SPARSE, XQK> sch{j, p.n_tiles, p.n_ktiles, off_, p.tile_mask};
        const int kvs = kk % SKV;
        if (kk >= SKV && !mbar_wait(&bars->kv_empty[kvs], ((kk / SKV) - 1) & 1, wc, kSiteFuKvEmpty)) break;
        mbar_arrive_expect_tx(&bars->kv_full[kvs], 2 * Cfg::kTileBytes);
        for (int cb = 0; cb < D / 64; ++cb) {
          tma_load_4d(sK + kvs * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_k, &bars->kv_full[kvs], cb * 64,
                      j * 128, ih, ib);
          tma_load_4d(sV + kvs * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_v, &bars->kv_full[kvs], cb * 64,
                      j * 128, ih, ib);
        }
        ++nkv;
        for (int i = sch.first(); i >= 0; i = sch.next(i), ++it) {
          const int st = it & 1;
          if (it >= 2 && !mbar_wait(&bars->q_empty[st], ((it >> 1) - 1) & 1, wc, kSiteFuQEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->q_full[st], Cfg::kTileBytes + 1024);
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_4d_hint(sQ + st * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_q, &bars->q_full[st], cb * 64,
                             i * 128, ih, ib, keep);
          const size_t roff = (size_t(bh) * p.n_tiles + size_t(i)) * 128;  // padded row arrays
          bulk_load(sL + st * 128, p.lse2 + roff, 512, &bars->q_full[st]);
          bulk_load(sDr + st * 128, p.Drow + roff, 512, &bars->q_full[st]);
          ++nq;
          const int ds_ = it % SD;
          if (it >= SD && !mbar_wait(&bars->do_empty[ds_], ((it / SD) - 1) & 1, wc, kSiteFuDoEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->do_full[ds_], Cfg::kTileBytes);
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_4d_hint(sDO + ds_ * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_do, &bars->do_full[ds_],
                             cb * 64, i * 128, ih, ib, keep);
          ++ndo;
        }
      }
      // On abort, wait (bounded) for this thread's own copies still in flight.
      if (bars->abort) {
        for (int x = (nkv > SKV ? nkv - SKV : 0); x < nkv; ++x)
          mbar_wait_drain(&bars->kv_full[x % SKV], (x / SKV) & 1, wc, kSiteFuDrain);
        for (int x = (nq > 2 ? nq - 2 : 0); x < nq; ++x)
          mbar_wait_drain(&bars->q_full[x & 1], (x >> 1) & 1, wc, kSiteFuDrain);
        for (int x = (ndo > SD ? ndo - SD : 0); x < ndo; ++x)
          mbar_wait_drain(&bars->do_full[x % SD], (x / SD) & 1, wc, kSiteFuDrain);
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kFusedRegsCtl>();
    if (lane == 0) {
      const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO);
      const uint32_t aDS = smem_u32(sDS);
      bool ok = true;
      int it = 0;  // query tiles processed so far (continues across items)
      BwdItem item;
      FusedWalk<CAUSAL> walk{p.n_ktiles, p.BH, p.paired};
      for (int kk = 0; ok && walk.next(item); ++kk) {
        KeySched<CAUSAL, SPARSE, XQK> sch{item.tile, p.n_tiles, p.n_ktiles, off_, p.tile_mask};
        const int kvs = kk % SKV;
        const uint32_t aK = smem_u32(sK) + kvs * Cfg::kTileBytes, aV = smem_u32(sV) + kvs * Cfg::kTileBytes;
        if (!mbar_wait(&bars->kv_full[kvs], (kk / SKV) & 1, wc, kSiteFuKV)) { ok = false; break; }
        tc_fence_after();
        int i = sch.first();
        if (i < 0) mma_commit(&bars->kv_empty[kvs]);
        if (i >= 0) {
          // The item's first S^T and dP^T.
          if (!mbar_wait(&bars->q_full[it & 1], (it >> 1) & 1, wc, kSiteFuQFull)) { ok = false; break; }
          tc_fence_after();
          mma_tile_nt<D>(tmem + Cfg::kTmX, aK, aQ + (it & 1) * Cfg::kTileBytes);
          mma_commit(&bars->s_full);
          // Y may still hold the previous tile's dQ (head dim 128): wait until it is read.
          if (Cfg::kDqInY && it > 0 && !mbar_wait(&bars->dq_taken, (it - 1) & 1, wc, kSiteFuDqTaken)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&bars->do_full[it % SD], (it / SD) & 1, wc, kSiteFuDoFull)) { ok = false; break; }
          tc_fence_after();
          mma_tile_nt<D>(tmem + Cfg::kTmY, aV, aDO + (it % SD) * Cfg::kTileBytes);
          mma_commit(&bars->dp_full);
        }
        bool first = true;
        while (i >= 0) {
          const int in = sch.next(i);
          const int st = it & 1, ds_ = it % SD;
          // dV += P^T dO_i, then the next S^T into X (it overwrites P^T only after this
          // product has read it: products execute in issue order).
          if (!mbar_wait(&bars->p_ready, it & 1, wc, kSiteFuPReady)) { ok = false; break; }
          if (first && kk > 0 && !mbar_wait(&bars->acc_empty, (kk - 1) & 1, wc, kSiteFuAcc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_dv_ts<D>(tmem + Cfg::kTmDV, tmem + Cfg::kTmX, aDO + ds_ * Cfg::kTileBytes, !first);
          mma_commit(&bars->do_empty[ds_]);
          if (in >= 0) {
            if (!mbar_wait(&bars->q_full[(it + 1) & 1], ((it + 1) >> 1) & 1, wc, kSiteFuQFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma_tile_nt<D>(tmem + Cfg::kTmX, aK, aQ + ((it + 1) & 1) * Cfg::kTileBytes);
            mma_commit(&bars->s_full);
          }
          // dK += dS^T Q_i and dQ_i = dS K_j, both reading dS from shared memory (dQ first
          // at head dim 128, where the next dP^T waits for dQ's columns to be read out).
          if (!mbar_wait(&bars->ds_ready, it & 1, wc, kSiteFuDsReady)) { ok = false; break; }
          // Head dim 64: Z may still hold the previous tile's dQ.
          if (!Cfg::kDqInY && it > 0 && !mbar_wait(&bars->dq_taken, (it - 1) & 1, wc, kSiteFuDqTaken)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if constexpr (Cfg::kDqInY) {
            mma_dq_ss<D>(tmem + Cfg::kTmDQ, aDS, aK);
            mma_commit(&bars->dq_full);
            mma_dk_ss<D>(tmem + Cfg::kTmDK, aDS, aQ + st * Cfg::kTileBytes, !first);
          } else {
            mma_dk_ss<D>(tmem + Cfg::kTmDK, aDS, aQ + st * Cfg::kTileBytes, !first);
            mma_dq_ss<D>(tmem + Cfg::kTmDQ, aDS, aK);
            mma_commit(&bars->dq_full);
          }
          mma_commit(&bars->q_empty[st]);
          if (in < 0) mma_commit(&bars->kv_empty[kvs]);  // every product reading K_j, V_j is issued
          if (in >= 0) {
            if (Cfg::kDqInY && !mbar_wait(&bars->dq_taken, it & 1, wc, kSiteFuDqTaken)) { ok = false; break; }
            const int dn = (it + 1) % SD;
            if (!mbar_wait(&bars->do_full[dn], ((it + 1) / SD) & 1, wc, kSiteFuDoFull)) { ok = false; break; }
            tc_fence_after();
            mma_tile_nt<D>(tmem + Cfg::kTmY, aV, aDO + dn * Cfg::kTileBytes);
            mma_commit(&bars->dp_full);
          }
          first = false;
          i = in;
          ++it;
        }
        if (!ok) break;
        mma_commit(&bars->acc_done);
      }
      // Every MMA issued by this thread must finish before TMEM is released.
      mma_commit(&bars->mma_done);
      mbar_wait_drain(&bars->mma_done, 0, wc, kSiteFuDrain);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmCols);
  } else if (warp < 4) {
    // idle warps of the first warpgroup: they take part in its register hand-over
    regs_dec<kFusedRegsCtl>();
    __syncthreads();
  } else if (warp >= 12) {
    // ------------------------------------------------------------ dQ warpgroup
    // dQ_t out of tensor memory (thread = query row 32 quarter + lane of tile t) into
    // global dQacc rows [128 t + 32 quarter, +32), in 32 x 32 fp32 boxes through this
    // warp's stages, each box added by one reduce-add copy as soon as it is staged.
    regs_dec<kFusedRegsDrain>();
    const int quarter = warp & 3;
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    bool ok = true;
    int it = 0;
    BwdItem item;
    FusedWalk<CAUSAL> walk{p.n_ktiles, p.BH, p.paired};
    for (int kk = 0; ok && walk.next(item); ++kk) {
      KeySched<CAUSAL, SPARSE, XQK> sch{item.tile, p.n_tiles, p.n_ktiles, off_, p.tile_mask};
      for (int i = sch.first(); i >= 0; i = sch.next(i), ++it) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->dq_full, it & 1, wc, kSiteFuDqFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int y0 = i * 128 + quarter * 32;
        // Two 32-column boxes leave tensor memory in one load (64 registers); each is
        // staged and reduce-added by lane 0 as one copy.
        uint32_t v[64];
        auto stage_box = [&](int b, int half, uint8_t* stage) {
          uint4* s4 = reinterpret_cast<uint4*>(stage);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int o = half * 32 + 4 * c;
            s4[lane * 8 + (c ^ (lane & 7))] = make_uint4(v[o], v[o + 1], v[o + 2], v[o + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) tma_reduce_add_3d(&tm_dqacc, stage, b * 32, y0, item.bh);
        };
        uint8_t* area = smem + Cfg::kOffStage + quarter * 8192;
        if constexpr (D == 128) {
          // Boxes 0 and 1 through the stage area; boxes 2 and 3 stay in registers (dQ's
          // columns are released as soon as they are loaded) until those copies have read
          // the area.
          tmem_ld64(trow + Cfg::kTmDQ, v);
          tmem_wait_ld();
          stage_box(0, 0, area);
          stage_box(1, 1, area + 4096);
          if (lane == 0) bulk_commit();
          tmem_ld64(trow + Cfg::kTmDQ + 64, v);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&bars->dq_taken);
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
          stage_box(2, 0, area);
          stage_box(3, 1, area + 4096);
          if (lane == 0) {
            bulk_commit();
            bulk_wait_read0();  // this warp's stage area may be overwritten by the next tile
          }
        } else {
          tmem_ld64(trow + Cfg::kTmDQ, v);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&bars->dq_taken);
          stage_box(0, 0, area);
          stage_box(1, 1, area + 4096);
          if (lane == 0) {
            bulk_commit();
            bulk_wait_read0();
          }
        }
        __syncwarp();
      }
    }
    // Every reduce-add copy of this warp must be complete (its source is this CTA's
    // shared memory and its target the caller's workspace) before the kernel ends; a
    // copy issued before an abort may not be committed yet, hence the commit.
    if (lane == 0) {
      bulk_commit();
      bulk_wait0();
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
  } else {
    // ------------------------------------------------------------ compute warpgroups
    regs_inc<kFusedRegsCompute>();
    const int h = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row within tile j (TMEM lane of S^T, dP^T, dK, dV)
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    const float c2 = p.scale * 1.4426950408889634f;
    uint8_t* my_ds = sDS + h * 16384 + r * 128;  // this thread's dS row (key row r, query block h)
    bool ok = true;
    int it = 0;
    BwdItem item;
    FusedWalk<CAUSAL> walk{p.n_ktiles, p.BH, p.paired};
    for (int kk = 0; ok && walk.next(item); ++kk) {
      const int j = item.tile;
      KeySched<CAUSAL, SPARSE, XQK> sch{j, p.n_tiles, p.n_ktiles, off_, p.tile_mask};
      const bool kvalid = j * 128 + r < p.Nk;  // key rows past N_k (last tile) contribute nothing
      int local = 0;
      for (int i = sch.first(); i >= 0; i = sch.next(i), ++it, ++local) {
        const int st = it & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->q_full[st], (it >> 1) & 1, wc, kSiteFuQFull)) ||
            !__all_sync(0xffffffffu, mbar_wait(&bars->s_full, it & 1, wc, kSiteFuSFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* lse2 = sL + st * 128 + h * 64;
        const float* Dr = sDr + st * 128 + h * 64;
        int cbase = 0;
        if constexpr (XQK) {
          const long long cb64 = 128LL * (j - i) - off_;
          cbase = static_cast<int>(cb64 < -256 ? -256 : (cb64 > 256 ? 256 : cb64));
        }
        const bool diag = CAUSAL && (XQK ? cbase > -127 : i == j);
        const int cmin = cbase + r;
        // ---- P^T row r, query columns 64h + (0..63), packed bf16 pairs
        uint32_t pk[32];
        {
          uint32_t raw[64];
          tmem_ld64(trow + Cfg::kTmX + h * 64, raw);
          tmem_wait_ld();
          const uint64_t c2v = f2(c2, c2);
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int c0 = 2 * t;
            const float4 n4 = *reinterpret_cast<const float4*>(lse2 + (c0 & ~3));
            const float2 nl = (t & 1) ? make_float2(n4.z, n4.w) : make_float2(n4.x, n4.y);
            uint64_t pv = ex2_split_x2<PolyShare<D>::kDkdv>(
                f2_fma(f2(__uint_as_float(raw[c0]), __uint_as_float(raw[c0 + 1])), c2v, f2(nl.x, nl.y)), t);
            if (diag) {
              const float2 v = f2_split(pv);
              pv = f2((h * 64 + c0 < cmin) ? 0.f : v.x, (h * 64 + c0 + 1 < cmin) ? 0.f : v.y);
            }
            const float2 v = f2_split(pv);
            pk[t] = kvalid ? pack_bf16(v.x, v.y) : 0u;
          }
        }
        // P^T over the first half of this warpgroup's own score columns: this thread has read
        // its row of them, and no other thread reads this row.
        tmem_st32(trow + Cfg::kTmX + h * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_ready);
        // ---- dS = P (dP - D) into shared memory
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full, it & 1, wc, kSiteFuDpFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t ds[32];
        {
          uint32_t dpr[64];
          tmem_ld64(trow + Cfg::kTmY + h * 64, dpr);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float2 pp = unpack_bf16(pk[t]);
            const float4 d4 = *reinterpret_cast<const float4*>(Dr + ((2 * t) & ~3));
            const float2 dd = (t & 1) ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
            const uint64_t diff =
                f2_sub(f2(__uint_as_float(dpr[2 * t]), __uint_as_float(dpr[2 * t + 1])), f2(dd.x, dd.y));
            const float2 v = f2_split(f2_mul(f2(pp.x, pp.y), diff));
            ds[t] = pack_bf16(v.x, v.y);
          }
        }
        {
          uint4* d4 = reinterpret_cast<uint4*>(my_ds);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            d4[c ^ (r & 7)] = make_uint4(ds[4 * c], ds[4 * c + 1], ds[4 * c + 2], ds[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready);
      }
      if (!ok) break;
      // -------------------------------------------------------- epilogue: dK (h = 0), dV (h = 1)
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_done, kk & 1, wc, kSiteFuAcc))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int ib = item.bh / p.H, ih = item.bh - ib * p.H;
      const size_t row = seq_row_offset(ib, ih, j * 128 + r, p.Nk, p.H, p.ds, p.bnhd != 0);
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
      if (kvalid) {
        if (p.dk32 != nullptr)  // fp32 outputs (a key block's share of a longer sequence's gradients)
          store_regs_f32<D>((h == 0 ? p.dk32 : p.dv32) + row, acc, h == 0 ? p.scale : 1.f, p.ds);
        else
          store_regs_bf16<D>((h == 0 ? p.dk : p.dv) + row, acc, h == 0 ? p.scale : 1.f, p.ds, p.v8 != 0);
      }
    }
    tc_fence_before();
    __syncthreads();
  }
}

// ---------------------------------------------------------------- dQ conversion

// dq[b, h, n, :ds] = bf16(scale * dqacc[bh, n, :ds]) for the rows n < N (dqacc rows
// are Npad apart per (batch, head) and D wide). D / 8 threads per row, 8 columns each.
template <int D>
__global__ void __launch_bounds__(256) fa_dq_convert_kernel(const float* __restrict__ dqacc,
                                                            __nv_bfloat16* __restrict__ dq, int N, int Npad, int ds,
                                                            int H, int bnhd, long long rows, float scale) {
  constexpr int TPR = D / 8;
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = g / TPR;  // bh * N + n
  const int part = static_cast<int>(g % TPR);
  if (row >= rows || part * 8 >= ds) return;
  const unsigned bh = static_cast<unsigned>(row / N);
  const int n = static_cast<int>(row - static_cast<long long>(bh) * N);
  const float4* src = reinterpret_cast<const float4*>(dqacc + (static_cast<size_t>(bh) * Npad + n) * D + part * 8);
  const float4 a = src[0], b = src[1];
  const int b_ = static_cast<int>(bh / static_cast<unsigned>(H)), h_ = static_cast<int>(bh) - b_ * H;
  uint4 w;
  w.x = pack_bf16(a.x * scale, a.y * scale);
  w.y = pack_bf16(a.z * scale, a.w * scale);
  w.z = pack_bf16(b.x * scale, b.y * scale);
  w.w = pack_bf16(b.z * scale, b.w * scale);
  *reinterpret_cast<uint4*>(dq + seq_row_offset(b_, h_, n, N, H, ds, bnhd != 0) + part * 8) = w;
}

}  // namespace fa
