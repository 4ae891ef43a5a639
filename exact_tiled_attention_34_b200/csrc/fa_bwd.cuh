// fa_bwd.cuh - backward kernels: attention recomputed tile by tile from the saved
// log-sum-exp ("Researchers at Stanford University Propose FlashAttention ..."
// summary, method paragraph: the forward's normalisation factor is saved so the
// backward recomputes attention on chip instead of storing it).
//
// Gradients of L = sum(O * dO):
//   D_i  = sum_c dO_ic O_ic                     (pre-processing kernel)
//   P    = exp(scale q_i.k_j - lse_i)           (recomputed)
//   dV_j = sum_i P_ij dO_i,   dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - D_i)
//   dK_j = scale sum_i dS_ij q_i,   dQ_i = scale sum_j dS_ij k_j
//
// Main kernel: one CTA per (128-key tile j, batch*head), looping over the query
// tiles i that see tile j (causal: i >= j; block-sparse: mask[i][j] = 1). The
// transposed products are formed directly so key rows sit on TMEM lanes:
//   S^T  = K_j Q_i^T      (SS MMA, both K-major)          -> TMEM
//   dP^T = V_j dO_i^T     (SS MMA, both K-major)          -> TMEM
//   dV  += P^T dO_i       (TS MMA: P^T from TMEM, dO_i N-major)
//   dK  += dS^T Q_i       (TS MMA: dS^T from TMEM, Q_i N-major)
//   dQ_i = dS K_j         (SS MMA: dS from shared memory M-major, K_j N-major)
// so the TMA-loaded tiles serve both as K-major and as N-major operands and no
// transposed copy is made. dQ_i is added into an fp32 accumulator in global memory
// with vector atomics (order of the additions not fixed); dK and dV stay in TMEM
// until the end. A final kernel converts the fp32 dQ accumulator to bf16.
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 MMA issuer + TMEM owner,
// warps 4-11 two "compute" warpgroups (thread = key row; warpgroup h takes query
// columns [64h, 64h+64): P^T, dS^T; epilogue dK (h = 0) / dV (h = 1)),
// warps 12-15 "dQ" (thread = query row: TMEM -> atomics).
// TMEM columns, head dim 64:  dK 0 | dV 64 | S^T 128 | dP^T 256 | dQ 384
//               head dim 128: dK 0 | dV 128 | S^T 256 | dP^T 384; dQ_i is formed in
// two 64-column parts, one after the other, in the dP^T columns that dS^T (bf16,
// 64 columns) leaves free. The next S^T is issued right after dV (it overwrites
// P^T, which dV has read: products execute in issue order); the next dP^T waits
// until the last dQ part has been read out.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

// ---------------------------------------------------------------- pre-processing

// D[row] = sum_c dO[row, c] * O[row, c] (fp32), and dQacc[row, :] = 0.
// D / 8 threads per row, 16 bytes each.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         float* __restrict__ Drow, float* __restrict__ dqacc,
                                                         long long rows) {
  constexpr int TPR = D / 8;
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = g / TPR;
  const int part = static_cast<int>(g % TPR);
  const bool valid = row < rows;
  float s = 0.f;
  if (valid) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + row * D + part * 8);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 x = __bfloat1622float2(pa[t]);
      const float2 y = __bfloat1622float2(pb[t]);
      s = fmaf(x.x, y.x, s);
      s = fmaf(x.y, y.y, s);
    }
    float4* z = reinterpret_cast<float4*>(dqacc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int w = TPR / 2; w > 0; w >>= 1) s += __shfl_xor_sync(0xffffffffu, s, w);
  if (valid && part == 0) Drow[row] = s;
}

// dq = bf16(scale * dQacc), 4 elements per thread per step.
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float4* __restrict__ acc,
                                                                uint2* __restrict__ dq, float scale,
                                                                long long n4) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = acc[i];
    uint2 r;
    r.x = pack_bf16(v.x * scale, v.y * scale);
    r.y = pack_bf16(v.z * scale, v.w * scale);
    dq[i] = r;
  }
}

// ---------------------------------------------------------------- main kernel

struct BwdParams {
  const float* lse;     // [BH, N]
  const float* Drow;    // [BH, N]
  float* dqacc;         // [BH, N, D]
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const uint8_t* tile_mask;  // [nT, nT] or nullptr
  int* status;
  unsigned long long timeout_ns;
  int N;
  int BH;
  int n_tiles;
  float scale;          // softmax scale (dK is scaled in the epilogue)
};

template <int D>
struct BwdCfg {
  static constexpr int kColBlocks = D / 64;
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;       // 2 stages
  static constexpr int kOffDO = kOffQ + 2 * kTileBytes;  // 2 stages
  static constexpr int kOffDS = kOffDO + 2 * kTileBytes; // dS, 128 x 128 bf16 (32 KiB)
  static constexpr int kOffL = kOffDS + 32768;           // lse, 2 stages x 128 fp32
  static constexpr int kOffDr = kOffL + 1024;            // D rows, 2 stages x 128 fp32
  static constexpr int kOffBar = kOffDr + 1024;
  // Head dim 128 fills shared memory to the limit: no alignment slack (the kernel
  // checks that the dynamic shared memory base is 1024-byte aligned).
  static constexpr int kSlack = (D == 64) ? 1024 : 0;
  static constexpr int kSmemBytes = kOffBar + 256 + kSlack;
  static constexpr bool kAlias = (D == 128);
  static constexpr uint32_t kTmDK = 0;
  static constexpr uint32_t kTmDV = D;
  static constexpr uint32_t kTmS = 2 * D;
  static constexpr uint32_t kTmDP = 2 * D + 128;
  static constexpr uint32_t kTmDQ = 2 * D + 256;  // head dim 64 only
  static constexpr uint32_t kTmCols = 512;
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t t_full[2];
  uint64_t t_empty[2];
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t p_ready;
  uint64_t ds_ready;
  uint64_t dq_full;
  uint64_t dq_empty;
  uint64_t acc_done;
  uint64_t mma_done;
  uint64_t rd_s;   // both compute warpgroups have read S^T of this tile
  uint64_t rd_dp;  // ... and dP^T
  uint32_t tmem_base;
  int abort;
};

// Register split of the 512-thread backward block launched with 128 registers per
// thread (65,536 in all): producer/MMA warpgroup 80, the two compute warpgroups 160
// each, the dQ warpgroup 112 -> 128 * (80 + 160 + 160 + 112) = 65,536. The two
// decreases happen first thing and are never undone; the compute warpgroups' single
// increase needs exactly what they release.
constexpr int kBwdLaunchRegs = 128;
constexpr int kBwdRegsCtl = 80;
constexpr int kBwdRegsCompute = 160;
constexpr int kBwdRegsDq = 112;
static_assert(128 * (kBwdRegsCtl + 2 * kBwdRegsCompute + kBwdRegsDq) <= 512 * kBwdLaunchRegs,
              "register split exceeds the block's register pool");

enum BwdSite : int {
  kSiteBwdKV = 201, kSiteBwdTEmpty, kSiteBwdTFull, kSiteBwdPReady, kSiteBwdDsReady, kSiteBwdDqEmpty,
  kSiteBwdSFull, kSiteBwdDpFull, kSiteBwdDqFull, kSiteBwdAcc, kSiteBwdDrain, kSiteBwdAlign, kSiteBwdRead
};

// Query tiles that see key tile j.
template <bool CAUSAL, bool SPARSE>
struct BwdSched {
  int j, n_tiles;
  const uint8_t* mask;
  __device__ __forceinline__ int next(int i0) const {
    for (int i = (CAUSAL ? (i0 < j ? j : i0 + 1) : i0 + 1); i < n_tiles; ++i) {
      if (!SPARSE || mask[size_t(i) * n_tiles + j] != 0) return i;
    }
    return -1;
  }
  __device__ __forceinline__ int first() const { return next(CAUSAL ? j - 1 : -1); }
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

template <int D, bool CAUSAL, bool SPARSE>
__global__ void __launch_bounds__(512, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const BwdParams p) {
  using Cfg = BwdCfg<D>;
  constexpr int kDqParts = Cfg::kAlias ? 2 : 1;  // dQ_i products (and read-outs) per query tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_off = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((base_off + 1023u) & ~1023u) - base_off);
  if (Cfg::kSlack == 0 && (base_off & 1023u) != 0) {
    // Cannot happen with the launch configuration used here; refuse rather than
    // overrun shared memory.
    if (threadIdx.x == 0 && atomicCAS(p.status, 0, 2) == 0) atomicExch(p.status + 1, kSiteBwdAlign);
    return;
  }
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + Cfg::kOffBar);
  uint8_t* sK = smem + Cfg::kOffK;
  uint8_t* sV = smem + Cfg::kOffV;
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sDO = smem + Cfg::kOffDO;
  uint8_t* sDS = smem + Cfg::kOffDS;
  float* sL = reinterpret_cast<float*>(smem + Cfg::kOffL);
  float* sDr = reinterpret_cast<float*>(smem + Cfg::kOffDr);

  const int warp = warp_id();
  const int lane = lane_id();
  // Head-major order (the key tiles of one head run together and share its Q/dO
  // tiles through L2), small j first within a head (most query tiles when causal).
  const int lin = blockIdx.x;
  const int bh = lin / p.n_tiles;
  const int j = lin % p.n_tiles;
  BwdSched<CAUSAL, SPARSE> sch{j, p.n_tiles, p.tile_mask};
  WaitCtl wc{&bars->abort, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->t_full[s], 1);
      mbar_init(&bars->t_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_ready, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_empty, 128);
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->rd_s, 256);
    mbar_init(&bars->rd_dp, 256);
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
      mbar_arrive_expect_tx(&bars->kv_full, 2 * Cfg::kTileBytes);
      for (int cb = 0; cb < Cfg::kColBlocks; ++cb) {
        tma_load_3d(sK + cb * Cfg::kBlockBytes, &tm_k, &bars->kv_full, cb * 64, j * 128, bh);
        tma_load_3d(sV + cb * Cfg::kBlockBytes, &tm_v, &bars->kv_full, cb * 64, j * 128, bh);
      }
      const uint64_t keep = policy_evict_last();
      int it = 0;
      for (int i = sch.first(); i >= 0; i = sch.next(i), ++it) {
        const int st = it & 1;
        const int n = it >> 1;
        if (n > 0 && !mbar_wait(&bars->t_empty[st], (n - 1) & 1, wc, kSiteBwdTEmpty)) break;
        mbar_arrive_expect_tx(&bars->t_full[st], kTileTx);
        for (int cb = 0; cb < Cfg::kColBlocks; ++cb) {
          tma_load_3d_hint(sQ + st * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_q, &bars->t_full[st], cb * 64,
                           i * 128, bh, keep);
          tma_load_3d_hint(sDO + st * Cfg::kTileBytes + cb * Cfg::kBlockBytes, &tm_do, &bars->t_full[st],
                           cb * 64, i * 128, bh, keep);
        }
        const size_t roff = size_t(bh) * p.N + size_t(i) * 128;
        bulk_load(sL + st * 128, p.lse + roff, 512, &bars->t_full[st]);
        bulk_load(sDr + st * 128, p.Drow + roff, 512, &bars->t_full[st]);
      }
      if (bars->abort) {
        mbar_wait_drain(&bars->kv_full, 0, wc, kSiteBwdDrain);
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
      constexpr uint32_t idT = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t idG = idesc_bf16_f32(128, D, 0, 1);    // dV, dK (A in TMEM, B N-major)
      constexpr uint32_t idQ = idesc_bf16_f32(128, 64, 1, 1);   // dQ (part): A M-major, B N-major
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO),
                     aDS = smem_u32(sDS);
      // X[tm] = A[128 x D] * B[128 x D]^T with both operands K-major (A: key rows, B: query rows)
      auto issue_t = [&](uint32_t tm, uint32_t a, uint32_t b) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * Cfg::kBlockBytes + (k & 3) * 32;
          mma_ss(tmem + tm, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(b + off, 16, 1024), idT, k > 0);
        }
      };
      // G[tm] (+)= A_tmem[128 x 128 q] * B[q x D] with B N-major in shared memory
      auto issue_g = [&](uint32_t tm, uint32_t a_tm, uint32_t b, bool acc) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tmem + tm, tmem + a_tm + k * 8, sdesc_sw128(b + k * 2048, Cfg::kBlockBytes, 1024), idG,
                 (acc || k > 0) ? 1u : 0u);
      };
      // 64 columns [64h, 64h+64) of dQ_i = dS[q x kv] * K_j[kv x D] into TMEM column tm
      auto issue_dq = [&](uint32_t tm, int h) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + tm, sdesc_sw128(aDS + k * 2048, Cfg::kBlockBytes, 1024),
                 sdesc_sw128(aK + h * Cfg::kBlockBytes + k * 2048, Cfg::kBlockBytes, 1024), idQ, k > 0);
      };
      constexpr uint32_t kTmDqPart = Cfg::kAlias ? Cfg::kTmDP + 64 : Cfg::kTmDQ;
      bool ok = mbar_wait(&bars->kv_full, 0, wc, kSiteBwdKV);
      tc_fence_after();
      int i = ok ? sch.first() : -1;
      int it = 0;
      if (i >= 0) {
        if (!mbar_wait(&bars->t_full[0], 0, wc, kSiteBwdTFull)) {
          ok = false;
          i = -1;
        } else {
          tc_fence_after();
          issue_t(Cfg::kTmS, aK, aQ);
          mma_commit(&bars->s_full);
          issue_t(Cfg::kTmDP, aV, aDO);
          mma_commit(&bars->dp_full);
        }
      }
      while (i >= 0) {
        const int st = it & 1;
        const int in = sch.next(i);
        const int stn = (it + 1) & 1;
        const uint32_t phn = ((it + 1) >> 1) & 1;
        // dV += P^T dO_i, then at once S^T for the next query tile (it overwrites P^T
        // only after this dV product has read it: products run in issue order).
        if (!mbar_wait(&bars->p_ready, it & 1, wc, kSiteBwdPReady)) { ok = false; break; }
        tc_fence_after();
        issue_g(Cfg::kTmDV, Cfg::kTmS, aDO + st * Cfg::kTileBytes, it > 0);
        if (in >= 0) {
          if (!mbar_wait(&bars->t_full[stn], phn, wc, kSiteBwdTFull)) { ok = false; break; }
          tc_fence_after();
          issue_t(Cfg::kTmS, aK, aQ + stn * Cfg::kTileBytes);
          mma_commit(&bars->s_full);
        }
        // dK += dS^T Q_i ; dQ_i = dS K_j (in kDqParts column parts of 64)
        if (!mbar_wait(&bars->ds_ready, it & 1, wc, kSiteBwdDsReady)) { ok = false; break; }
        tc_fence_after();
        issue_g(Cfg::kTmDK, Cfg::kTmDP, aQ + st * Cfg::kTileBytes, it > 0);
        for (int h = 0; h < kDqParts && ok; ++h) {
          const int hc = it * kDqParts + h;  // dQ product counter
          if (hc > 0 && !mbar_wait(&bars->dq_empty, (hc - 1) & 1, wc, kSiteBwdDqEmpty)) { ok = false; break; }
          tc_fence_after();
          issue_dq(kTmDqPart, h);
          mma_commit(&bars->dq_full);
        }
        if (!ok) break;
        mma_commit(&bars->t_empty[st]);
        if (in >= 0) {
          // dP^T for the next tile overwrites dS^T (read by dK above, in issue order)
          // and, at head dim 128, the dQ part columns: wait until they are read out.
          if (Cfg::kAlias) {
            const int hc = it * kDqParts + kDqParts - 1;
            if (!mbar_wait(&bars->dq_empty, hc & 1, wc, kSiteBwdDqEmpty)) { ok = false; break; }
            tc_fence_after();
          }
          issue_t(Cfg::kTmDP, aV, aDO + stn * Cfg::kTileBytes);
          mma_commit(&bars->dp_full);
        }
        i = in;
        ++it;
      }
      if (ok) mma_commit(&bars->acc_done);
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
  } else if (warp < 12) {
    // ------------------------------------------------------------ compute warpgroups
    regs_inc<kBwdRegsCompute>();
    // Warpgroup h (0 or 1) handles query columns [64h, 64h + 64) of the key rows.
    const int h = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row within tile j
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    const float sc = p.scale;
    constexpr float kLog2e = 1.4426950408889634f;
    bool ok = true;
    int it = 0;
    for (int i = sch.first(); i >= 0; i = sch.next(i), ++it) {
      const int st = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->t_full[st], (it >> 1) & 1, wc, kSiteBwdTFull))) {
        ok = false;
        break;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, it & 1, wc, kSiteBwdSFull))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* lse = sL + st * 128 + h * 64;
      const float* Dr = sDr + st * 128 + h * 64;
      const bool diag = CAUSAL && (i == j);  // query c visible to key r iff c >= r
      // ---- P^T row r, query columns 64h + (0..63), packed bf16 pairs
      uint32_t pk[32];
      {
        uint32_t raw[64];
        tmem_ld32(trow + Cfg::kTmS + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&raw[0]));
        tmem_ld32(trow + Cfg::kTmS + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&raw[32]));
        tmem_wait_ld();
        // The packed P^T of query q goes to column q / 2: warpgroup 1 writes columns
        // 32..63, which hold scores warpgroup 0 reads. Both finish reading first.
        mbar_arrive(&bars->rd_s);
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->rd_s, it & 1, wc, kSiteBwdRead))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int t4 = 0; t4 < 16; ++t4) {
          const int c0 = 4 * t4;
          const float4 l4 = *reinterpret_cast<const float4*>(lse + c0);
          float pv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float lu = u == 0 ? l4.x : u == 1 ? l4.y : u == 2 ? l4.z : l4.w;
            pv[u] = ex2(fmaf(__uint_as_float(raw[c0 + u]), sc, -lu) * kLog2e);
            if (diag) pv[u] = (h * 64 + c0 + u < r) ? 0.f : pv[u];
          }
          pk[2 * t4] = pack_bf16(pv[0], pv[1]);
          pk[2 * t4 + 1] = pack_bf16(pv[2], pv[3]);
        }
      }
      tmem_st32(trow + Cfg::kTmS + h * 32, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_ready);
      // ---- dS^T = P^T * (dP^T - D), to TMEM (A of dK) and to shared memory (A of dQ)
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full, it & 1, wc, kSiteBwdDpFull))) {
        ok = false;
        break;
      }
      // The previous tile's dQ products read the shared dS buffer: wait for the last.
      if (it > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->dq_full, (it * kDqParts - 1) & 1, wc,
                                                       kSiteBwdDqFull))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t dpr[64];
      tmem_ld32(trow + Cfg::kTmDP + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&dpr[0]));
      tmem_ld32(trow + Cfg::kTmDP + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dpr[32]));
      tmem_wait_ld();
      // dS^T (packed) overwrites dP^T columns that the other warpgroup reads.
      mbar_arrive(&bars->rd_dp);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->rd_dp, it & 1, wc, kSiteBwdRead))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t ds[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int c0 = q2 * 32 + 2 * t;
          const float2 pp = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[q2 * 16 + t]));
          const float2 dd = *reinterpret_cast<const float2*>(Dr + c0);
          ds[t] = pack_bf16(pp.x * (__uint_as_float(dpr[c0]) - dd.x), pp.y * (__uint_as_float(dpr[c0 + 1]) - dd.y));
        }
        tmem_st16(trow + Cfg::kTmDP + h * 32 + q2 * 16, ds);
        // Shared memory, M-major 128-byte swizzle: [q block h][key row][64 q].
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int cq = q2 * 4 + ch;  // 16-byte chunk index (8 q values) within the block
          uint8_t* dst = sDS + h * Cfg::kBlockBytes + r * 128 + ((cq ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(ds[4 * ch], ds[4 * ch + 1], ds[4 * ch + 2], ds[4 * ch + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready);
    }
    // ---------------------------------------------------------- epilogue: dK (h = 0), dV (h = 1)
    const size_t row = size_t(bh) * p.N + size_t(j) * 128 + r;
    if (ok) {
      const bool any = it > 0;
      if (any) ok = __all_sync(0xffffffffu, mbar_wait(&bars->acc_done, 0, wc, kSiteBwdAcc));
      if (ok) {
        tc_fence_after();
        __nv_bfloat16* dst = (h == 0 ? p.dk : p.dv) + row * D;
        const float mul = h == 0 ? sc : 1.f;
        const uint32_t col = h == 0 ? Cfg::kTmDK : Cfg::kTmDV;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          if (any) {
            tmem_ld32(trow + col + cc * 32, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] = 0u;
          }
          uint4 o4[4];
          uint32_t* w = reinterpret_cast<uint32_t*>(o4);
#pragma unroll
          for (int t = 0; t < 16; ++t)
            w[t] = pack_bf16(__uint_as_float(v[2 * t]) * mul, __uint_as_float(v[2 * t + 1]) * mul);
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
          for (int t = 0; t < 4; ++t) d4[t] = o4[t];
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  } else {
    // ------------------------------------------------------------ dQ warpgroup
    regs_dec<kBwdRegsDq>();
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within tile i
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    constexpr uint32_t kTmDqPart = Cfg::kAlias ? Cfg::kTmDP + 64 : Cfg::kTmDQ;
    int it = 0;
    bool ok = true;
    for (int i = sch.first(); i >= 0 && ok; i = sch.next(i), ++it) {
      float4* dst = reinterpret_cast<float4*>(p.dqacc + (size_t(bh) * p.N + size_t(i) * 128 + r) * D);
      for (int h = 0; h < kDqParts; ++h) {
        const int hc = it * kDqParts + h;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->dq_full, hc & 1, wc, kSiteBwdDqFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t a[32], b[32];
        tmem_ld32(trow + kTmDqPart, a);
        tmem_ld32(trow + kTmDqPart + 32, b);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->dq_empty);
#pragma unroll
        for (int t = 0; t < 8; ++t)
          atomicAdd(dst + h * 16 + t, make_float4(__uint_as_float(a[4 * t]), __uint_as_float(a[4 * t + 1]),
                                                  __uint_as_float(a[4 * t + 2]), __uint_as_float(a[4 * t + 3])));
#pragma unroll
        for (int t = 0; t < 8; ++t)
          atomicAdd(dst + h * 16 + 8 + t, make_float4(__uint_as_float(b[4 * t]), __uint_as_float(b[4 * t + 1]),
                                                      __uint_as_float(b[4 * t + 2]), __uint_as_float(b[4 * t + 3])));
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  // Teardown: every role ends with its own CTA barrier (there is no common tail,
  // so the warpgroups keep their register budgets to the end); warp 1 then frees
  // TMEM. Only the compute warpgroups ever raise their budget, and only once, by
  // exactly what the other two warpgroups released: no increase can be starved.
}

}  // namespace fa
