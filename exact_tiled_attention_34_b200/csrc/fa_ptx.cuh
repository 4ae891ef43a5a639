// fa_ptx.cuh - thin inline-PTX layer for sm_100a: mbarriers with bounded waits,
// TMA tensor loads (no multicast), and the tcgen05 tensor-memory / MMA family.
//
// Every wait in this library goes through mbar_wait(), which gives up after a time
// limit, records FA_ERR_DEVICE_TIMEOUT plus a site code in the library status word,
// raises a CTA-wide abort flag and returns false; callers then leave their loops
// and tear down (drain their own copies, wait for their own MMAs, free TMEM).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace fa {

constexpr int kStatusTimeout = 6;  // == FA_ERR_DEVICE_TIMEOUT

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared control block for bounded waits.
struct WaitCtl {
  volatile int* abort;   // CTA-wide flag in shared memory
  int* status;           // library status word in global memory: [0] code, [1] site
  uint64_t timeout_ns;   // per-wait limit
};

__device__ __forceinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, const WaitCtl& c, int site,
                                            bool honour_abort) {
  const uint64_t t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_test(bar, parity)) return true;
    if (honour_abort && *c.abort) return false;
    if (global_ns() - t0 > c.timeout_ns) {
      *c.abort = 1;
      if (atomicCAS(c.status, 0, kStatusTimeout) == 0) atomicExch(c.status + 1, site);
      return false;
    }
  }
}

// Wait for the phase with the given parity to complete; false on timeout/abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl& c, int site) {
  if (mbar_test(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, c, site, true);
}

// Same, but keeps waiting after another role raised the abort flag (used to drain
// this thread's own copies / MMAs before teardown). Still bounded by the time limit.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, const WaitCtl& c, int site) {
  if (mbar_test(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, c, site, false);
}

// ------------------------------------------------------------------ TMA (no multicast)

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load of one box into shared memory; completion is signalled on `bar`
// as transaction bytes. Coordinates are element indices (x innermost).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Same with an L2 eviction-priority hint (a policy from createpolicy).
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z),
      "l"(policy)
      : "memory");
}

// 4-D tiled load (coordinates x innermost, then y, z, w); completion as for tma_load_3d.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                            int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 int z, int w, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z),
      "r"(w), "l"(policy)
      : "memory");
}

// Element offset of row n of sequence (b, h) in a [B, H, N, ds] (bnhd = false) or
// [B, N, H, ds] (bnhd = true) tensor.
__device__ __forceinline__ size_t seq_row_offset(int b, int h, int n, int N, int H, int ds, bool bnhd) {
  return bnhd ? ((size_t(b) * N + n) * H + h) * ds : ((size_t(b) * H + h) * N + n) * ds;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// fp32 reduce-add of one box from shared memory into global memory through a tensor
// map (coordinates x innermost); tracked by the calling thread's bulk async groups.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// Close the calling thread's current bulk async group.
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every bulk group of the calling thread has finished READING its source.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Same, for every bulk group but the most recently committed one.
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Wait until every bulk group of the calling thread is complete.
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Generic-proxy writes to shared memory -> visible to the async proxy (MMA, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05: TMEM

// Warp-wide: allocate `ncols` (power of two >= 32) TMEM columns; the address is
// written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMEM address: lane in bits 31..16, column in bits 15..0.
__device__ __forceinline__ uint32_t tmem_at(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// Warp-wide 32 lanes x 32 columns of 32-bit: thread t gets lane (base lane + t),
// columns col..col+31 into r[0..31].
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// ------------------------------------------------------------------ tcgen05: MMA

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
// a_mn / b_mn: 1 = operand is MN-major (M resp. N contiguous), 0 = K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                               // D format: f32
         | (1u << 7)                             // A format: bf16
         | (1u << 10)                            // B format: bf16
         | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17)                // N / 8
         | (uint32_t(M >> 4) << 24);             // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle.
//   lbo / sbo: leading / stride byte offsets (multiples of 16).
// For K-major tiles stored as 8-row x 128-byte swizzle atoms stacked along M/N,
// sbo = 1024 (next 8 rows) and lbo is unused. For MN-major tiles, lbo is the
// distance between 64-element (128-byte) atoms along M/N and sbo the distance
// between 8-row groups along K.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr >> 4) & 0x3FFF) | (uint64_t((lbo >> 4) & 0x3FFF) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46)  // descriptor version (sm_100)
         | (2ull << 61);                                          // 128-byte swizzle
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Per-warpgroup register budget (all warps of the warpgroup execute the same one).
// The increases must fit in what the decreases of other warpgroups release: the
// pool is the launch register count times the block size.
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------ row stores

// 32 bytes to global memory in one instruction (sm_100); p must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// 16 packed words (32 bf16 columns, 64 bytes) of one row: two 32-byte stores when the
// destination is 32-byte aligned (v8), else four 16-byte stores.
__device__ __forceinline__ void store_row64(void* dst, const uint32_t (&w)[16], bool v8) {
  if (v8) {
    st_global_v8(dst, &w[0]);
    st_global_v8(static_cast<uint8_t*>(dst) + 32, &w[8]);
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int t = 0; t < 4; ++t) d4[t] = make_uint4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
  }
}

// Stores the calling warp's 32 rows (lane = row) of 2 * NW bf16 values, given as NW
// packed words per lane, to global rows row0 + lane * ld (ld in elements); rows at or
// past `nrows` are not written (the tail of the last tile). Each lane's
// words go through `stage` (32 * NW words of this warp's shared memory, 16-byte
// aligned) so that every global store instruction writes 32 / (NW / 4) whole rows of
// NW * 4 bytes instead of 32 scattered 16-byte pieces. The 16-byte chunks of a row are
// rotated by the row index in the stage, which keeps both passes free of bank
// conflicts. NW is 16 or 32.
template <int NW>
__device__ __forceinline__ void warp_store_rows(uint32_t* stage, const uint32_t (&w)[NW], __nv_bfloat16* row0,
                                                size_t ld, int nrows) {
  constexpr int kCpr = NW / 4;       // 16-byte chunks per row
  constexpr int kRpi = 32 / kCpr;    // rows per store instruction
  const int lane = static_cast<int>(lane_id());
  uint4* st4 = reinterpret_cast<uint4*>(stage);
#pragma unroll
  for (int c = 0; c < kCpr; ++c)
    st4[lane * kCpr + (c ^ (lane & (kCpr - 1)))] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
  __syncwarp();
  const int c = lane & (kCpr - 1);
#pragma unroll
  for (int k = 0; k < kCpr; ++k) {
    const int row = k * kRpi + lane / kCpr;
    const uint4 v = st4[row * kCpr + (c ^ (row & (kCpr - 1)))];
    if (row < nrows) *reinterpret_cast<uint4*>(row0 + size_t(row) * ld + c * 8) = v;
  }
  __syncwarp();  // the stage may be rewritten after this
}

// ------------------------------------------------------------------ persistent schedules

// Position of this CTA's k-th work item in the global item order, or -1 when it has
// none: rounds of gridDim.x positions are dealt alternately forwards and backwards,
// so a CTA that drew a costly item in one round draws a cheap one in the next.
__device__ __forceinline__ long long item_position(long long n_items, int k) {
  const int G = gridDim.x, c = blockIdx.x;
  const long long pos = static_cast<long long>(k) * G + ((k & 1) ? (G - 1 - c) : c);
  return pos < n_items ? pos : -1;
}

// ------------------------------------------------------------------ math helpers

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t v) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
}

// ---- packed pairs of fp32 (one f32x2 instruction works on both halves; low half first)

__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_split(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Three-input maximum / minimum (one instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair of values without the special-function unit, so that part of a
// tile's exponentials can run on the FMA and integer pipes next to the MUFU ones.
// x = n + f with n = round(x) (adding 1.5 * 2^23 rounds to an integer in the low
// mantissa bits) and f in [-1/2, 1/2]; 2^f ~ 1 + f (c1 + f (c2 + f c3)), a cubic
// fitted here to minimise the relative error on [-1/2, 1/2] with the constant term
// fixed at 1 (csrc/fit_exp2_poly.py: max relative error 1.02e-4, 2^0 exact); 2^n is
// then added into the exponent field. Inputs below -126 are clamped (result about
// 1e-38), so the exponent never underflows; inputs must stay below 2^22.
__device__ __forceinline__ uint64_t ex2_poly_x2(uint64_t x) {
  constexpr float kC1 = 6.932800412e-01f, kC2 = 2.422109395e-01f, kC3 = 5.502312258e-02f;
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float2 xv = f2_split(x);
  const uint64_t xc = f2(fmaxf(xv.x, -126.f), fmaxf(xv.y, -126.f));
  const uint64_t rnd = f2(kRound, kRound);
  const uint64_t t = f2_add(xc, rnd);            // round(x) in the low mantissa bits
  const uint64_t f = f2_sub(xc, f2_sub(t, rnd));  // x - round(x)
  uint64_t p = f2_fma(f, f2(kC3, kC3), f2(kC2, kC2));
  p = f2_fma(p, f, f2(kC1, kC1));
  p = f2_fma(p, f, f2(1.f, 1.f));
  const float2 pv = f2_split(p), tv = f2_split(t);
  const uint32_t y0 = __float_as_uint(pv.x) + (__float_as_uint(tv.x) << 23);
  const uint32_t y1 = __float_as_uint(pv.y) + (__float_as_uint(tv.y) << 23);
  return f2(__uint_as_float(y0), __uint_as_float(y1));
}

// 2^x for a pair on the special-function unit.
__device__ __forceinline__ uint64_t ex2_mufu_x2(uint64_t x) {
  const float2 v = f2_split(x);
  return f2(ex2(v.x), ex2(v.y));
}

// Which column pairs use the polynomial: pairs t with (t mod 8) < POLY8. Called from
// fully unrolled loops, so the choice is made at compile time. The shares were chosen
// by timing every value from 0 to 5 of 8 on B200 (same GPU, same run): the polynomial
// pays only where MUFU limits the softmax (forward at head dim 64); elsewhere its
// extra instructions cost more than the MUFU time they save.
template <int D>
struct PolyShare {
  static constexpr int kFwd = (D == 64) ? 2 : 0;
  static constexpr int kDkdv = 1;
  static constexpr int kDq = 0;
};
template <int POLY8>
__device__ __forceinline__ uint64_t ex2_split_x2(uint64_t x, int t) {
  return ((t & 7) < POLY8) ? ex2_poly_x2(x) : ex2_mufu_x2(x);
}

}  // namespace fa
