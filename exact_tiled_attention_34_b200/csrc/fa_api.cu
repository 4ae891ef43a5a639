// fa_api.cu - the C ABI of libfa.so (declared in include/fa.h): argument checks,
// TMA tensor-map encoding, kernel selection and launch. No allocation on any call
// path; every buffer is the caller's.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_bwd_fused.cuh"
#include "fa_bwd256.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd256.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kTimeoutNs = 4000000000ull;  // 4 s per device-side wait

// Library status word, one per device (module globals are per device).
__device__ int g_fa_status[2];

// Test hook set by fa_debug_stall_producer: attention launches made while it is on run
// with an idle TMA producer and this wait limit instead of kTimeoutNs.
std::atomic<int> g_stall{0};
std::atomic<unsigned long long> g_stall_limit_ns{kTimeoutNs};

void set_wait_limit(unsigned long long* timeout_ns, int* stall) {
  const int on = g_stall.load(std::memory_order_acquire);
  *stall = on;
  *timeout_ns = on ? g_stall_limit_ns.load(std::memory_order_relaxed) : kTimeoutNs;
}

// ------------------------------------------------------------------ argument checks

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_sizes(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 96 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  // Padded rows (N rounded up to whole 128-row tiles) index the backward's row arrays.
  const long long rows = static_cast<long long>(B) * H * ((static_cast<long long>(N) + 127) / 128 * 128);
  if (rows > INT_MAX || static_cast<long long>(B) * H > INT_MAX / 2) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs)
    if (p == nullptr) return FA_ERR_INVALID_ARG;
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_ALIGNMENT;
  return FA_OK;
}

fa_status check_scale(float scale) { return std::isfinite(scale) ? FA_OK : FA_ERR_INVALID_ARG; }

// Dropout settings: keep threshold t = round(256 (1 - p)) in 1..256 (computed in double
// from the float argument), kept probabilities scaled by 256 / t.
fa_status make_drop(float p_drop, uint64_t seed, uint32_t offset, fa::DropParams* dp) {
  if (!std::isfinite(p_drop) || p_drop < 0.f || p_drop >= 1.f) return FA_ERR_INVALID_ARG;
  const double t = std::nearbyint(256.0 * (1.0 - static_cast<double>(p_drop)));
  if (t < 1.0) return FA_ERR_INVALID_ARG;
  dp->seed_lo = static_cast<uint32_t>(seed);
  dp->seed_hi = static_cast<uint32_t>(seed >> 32);
  dp->offset = offset;
  dp->tm1 = static_cast<uint32_t>(t) - 1u;
  dp->rs = static_cast<float>(256.0 / t);
  return FA_OK;
}

// ------------------------------------------------------------------ per-device state

struct DeviceState {
  std::once_flag once;
  int* status = nullptr;  // device address of g_fa_status
  cudaError_t err = cudaSuccess;
};
DeviceState g_dev[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

fa_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return FA_ERR_CUDA;
  return FA_OK;
}

// Device address of the status word for the current device (set up once).
fa_status device_status_ptr(int** out) {
  int dev;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  DeviceState& st = g_dev[dev];
  std::call_once(st.once, [&] {
    void* ptr = nullptr;
    st.err = cudaGetSymbolAddress(&ptr, g_fa_status);
    if (st.err == cudaSuccess) {
      st.status = static_cast<int*>(ptr);
      st.err = cudaMemset(st.status, 0, sizeof(int) * 2);
    }
  });
  if (st.err != cudaSuccess || st.status == nullptr) return FA_ERR_CUDA;
  *out = st.status;
  return FA_OK;
}

fa_status encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? FA_OK : FA_ERR_CUDA;
}

// [BH, N, d] bf16 viewed as a 3-D tensor (d innermost); boxes of 64 columns x
// `box_rows` rows with 128-byte swizzle, matching the MMA operand layout.
fa_status make_map(CUtensorMap* m, const void* base, int B, int H, int N, int d, bool bnhd, int box_rows) {
  // Coordinates (column, row, head, batch) for both layouts; only the strides differ:
  // [B, H, N, d] rows are d apart and heads N*d; [B, N, H, d] rows are H*d apart and heads d.
  const cuuint64_t e = 2;  // bytes per element
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(H), cuuint64_t(B)};
  cuuint64_t strides[3];
  if (bnhd) {
    strides[0] = cuuint64_t(H) * d * e;
    strides[1] = cuuint64_t(d) * e;
  } else {
    strides[0] = cuuint64_t(d) * e;
    strides[1] = cuuint64_t(N) * d * e;
  }
  strides[2] = cuuint64_t(N) * H * d * e;
  cuuint32_t box[4] = {64, cuuint32_t(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename K>
fa_status set_smem(K kernel, int bytes, std::once_flag (&flags)[kMaxDevices], cudaError_t (&errs)[kMaxDevices]) {
  int dev;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  std::call_once(flags[dev], [&] {
    errs[dev] = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
  return errs[dev] == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}


template <int D, bool CAUSAL, bool SPARSE, bool XQK = false, int DS = D, bool DROP = false, bool MERGE = false>
fa_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const fa::FwdParamsT<DROP>& p, cudaStream_t stream) {
  static std::once_flag flags[kMaxDevices];
  static cudaError_t errs[kMaxDevices];
  static int regs[kMaxDevices];
  auto kernel = fa::fa_fwd_kernel<D, CAUSAL, SPARSE, XQK, DS, DROP, MERGE>;
  constexpr int smem = fa::FwdCfg<D>::kSmemBytes;
  if (set_smem(kernel, smem, flags, errs) != FA_OK) return FA_ERR_CUDA;
  // The kernel re-divides its register pool between warpgroups: refuse to launch a
  // build that gave it fewer registers per thread than the split needs.
  int dev;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  if (regs[dev] == 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FA_ERR_CUDA;
    regs[dev] = attr.numRegs;
  }
  if (regs[dev] * fa::FwdCfg<D>::kThreads < fa::kFwdRegsNeeded) return FA_ERR_UNSUPPORTED;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return FA_ERR_CUDA;
  const unsigned grid = unsigned(p.n_items < sms ? p.n_items : sms);  // persistent: one CTA per SM
  kernel<<<grid, fa::FwdCfg<D>::kThreads, smem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool CAUSAL, bool SPARSE, bool XQK = false>
fa_status launch_fwd256(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdParams& p,
                        cudaStream_t stream) {
  static std::once_flag flags[kMaxDevices];
  static cudaError_t errs[kMaxDevices];
  auto kernel = fa::fa_fwd256_kernel<CAUSAL, SPARSE, XQK>;
  constexpr int smem = fa::Fwd256Cfg::kSmemBytes;
  if (set_smem(kernel, smem, flags, errs) != FA_OK) return FA_ERR_CUDA;
  int dev, sms = 0;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return FA_ERR_CUDA;
  const unsigned grid = unsigned(p.n_items < sms ? p.n_items : sms);  // persistent: one CTA per SM
  kernel<<<grid, fa::Fwd256Cfg::kThreads, smem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// drop: dropout settings, or nullptr (dropout needs d 64 or 128, N_q = N_k and no tile mask).
// o_acc, lse_acc: the merging forward (fp32 running result updated in place; then o and
// lse are not used): N_q = N_k, [B, H, N, d] layout, d 64 or 128, no mask or dropout.
fa_status fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, const uint8_t* mask,
                     int B, int H, int N, int Nk, int d, int layout, int causal, float scale, void* stream,
                     const fa::DropParams* drop = nullptr, float* o_acc = nullptr, float* lse_acc = nullptr) {
  fa_status s;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID_ARG;
  const bool bnhd = layout == FA_LAYOUT_BNHD;
  const bool merge = o_acc != nullptr;
  if ((s = check_ptrs({q, k, v, merge ? static_cast<const void*>(o_acc) : o,
                       merge ? static_cast<const void*>(lse_acc) : lse})) != FA_OK)
    return s;
  if ((s = check_sizes(B, H, N, d)) != FA_OK) return s;
  if ((s = check_sizes(B, H, Nk, d)) != FA_OK) return s;
  if (mask != nullptr && Nk != N) return FA_ERR_UNSUPPORTED;
  if (merge && (mask != nullptr || drop != nullptr || Nk != N || bnhd || (d != 64 && d != 128)))
    return FA_ERR_UNSUPPORTED;
  if (drop != nullptr && (mask != nullptr || Nk != N || d == 96 || d == 256)) return FA_ERR_UNSUPPORTED;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if ((s = encoder()) != FA_OK) return s;
  int* status;
  if ((s = device_status_ptr(&status)) != FA_OK) return s;
  const int BH = B * H;
  CUtensorMap mq, mk, mv;
  if ((s = make_map(&mq, q, B, H, N, d, bnhd, 128)) != FA_OK) return s;
  if ((s = make_map(&mk, k, B, H, Nk, d, bnhd, 128)) != FA_OK) return s;
  if ((s = make_map(&mv, v, B, H, Nk, d, bnhd, 128)) != FA_OK) return s;
  fa::FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.tile_mask = mask;
  p.status = status;
  set_wait_limit(&p.timeout_ns, &p.stall);
  p.N = N;
  p.Nk = Nk;
  p.BH = BH;
  p.H = H;
  p.bnhd = bnhd ? 1 : 0;
  p.v8 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;  // rows are 128/192/256 B: all aligned alike
  p.n_tiles = (N + 127) / 128;
  p.n_ktiles = (Nk + 127) / 128;
  p.off = Nk - N;
  p.n_qblocks = (p.n_tiles + 1) / 2;
  p.n_items = p.n_qblocks * BH;
  p.c_log2 = scale * 1.4426950408889634f;
  p.o_acc = o_acc;
  p.lse_acc = lse_acc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (merge) {
    if (causal)
      return d == 64 ? launch_fwd<64, true, false, false, 64, false, true>(mq, mk, mv, p, st)
                     : launch_fwd<128, true, false, false, 128, false, true>(mq, mk, mv, p, st);
    return d == 64 ? launch_fwd<64, false, false, false, 64, false, true>(mq, mk, mv, p, st)
                   : launch_fwd<128, false, false, false, 128, false, true>(mq, mk, mv, p, st);
  }
  if (d == 256) {  // one Q tile per work item
    p.n_qblocks = p.n_tiles;
    p.n_items = p.n_tiles * BH;
    if (mask) return launch_fwd256<false, true>(mq, mk, mv, p, st);
    if (causal && Nk != N) return launch_fwd256<true, false, true>(mq, mk, mv, p, st);
    if (causal) return launch_fwd256<true, false>(mq, mk, mv, p, st);
    return launch_fwd256<false, false>(mq, mk, mv, p, st);
  }
  if (drop) {
    fa::FwdParamsDrop pd;
    static_cast<fa::FwdParams&>(pd) = p;
    pd.drop = *drop;
    if (causal)
      return d == 64 ? launch_fwd<64, true, false, false, 64, true>(mq, mk, mv, pd, st)
                     : launch_fwd<128, true, false, false, 128, true>(mq, mk, mv, pd, st);
    return d == 64 ? launch_fwd<64, false, false, false, 64, true>(mq, mk, mv, pd, st)
                   : launch_fwd<128, false, false, false, 128, true>(mq, mk, mv, pd, st);
  }
  if (d == 96) {  // the 128-wide kernels with 96 stored columns
    if (mask) return launch_fwd<128, false, true, false, 96>(mq, mk, mv, p, st);
    if (causal && Nk != N) return launch_fwd<128, true, false, true, 96>(mq, mk, mv, p, st);
    if (causal) return launch_fwd<128, true, false, false, 96>(mq, mk, mv, p, st);
    return launch_fwd<128, false, false, false, 96>(mq, mk, mv, p, st);
  }
  if (mask) {
    return d == 64 ? launch_fwd<64, false, true>(mq, mk, mv, p, st) : launch_fwd<128, false, true>(mq, mk, mv, p, st);
  }
  if (causal && Nk != N)  // causal mask with an offset (N_q != N_k)
    return d == 64 ? launch_fwd<64, true, false, true>(mq, mk, mv, p, st)
                   : launch_fwd<128, true, false, true>(mq, mk, mv, p, st);
  if (causal) {
    return d == 64 ? launch_fwd<64, true, false>(mq, mk, mv, p, st) : launch_fwd<128, true, false>(mq, mk, mv, p, st);
  }
  return d == 64 ? launch_fwd<64, false, false>(mq, mk, mv, p, st) : launch_fwd<128, false, false>(mq, mk, mv, p, st);
}


size_t round256(size_t x) { return (x + 255) & ~size_t(255); }


// Workspace: fp32 D rows, then fp32 -lse*log2(e) rows, each [BH * Npad] (Npad = N
// rounded up to a multiple of 128) and 256-aligned.
size_t bwd_ws_bytes(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  const size_t rows = size_t(B) * H * ((size_t(N) + 127) / 128 * 128);
  return 2 * round256(rows * 4);
}

// Launch one of the two 384-thread backward kernels. They re-divide their register
// pool between warpgroups; refuse to launch if the build gave them fewer registers
// per thread than that split needs.
template <typename K, typename P>
fa_status launch_bwd_kernel(K kernel, int smem, unsigned grid /* work items */, const CUtensorMap& mq, const CUtensorMap& mk,
                            const CUtensorMap& mv, const CUtensorMap& mdo, const P& p,
                            cudaStream_t stream, std::once_flag (&flags)[kMaxDevices],
                            cudaError_t (&errs)[kMaxDevices], int (&regs)[kMaxDevices]) {
  if (set_smem(kernel, smem, flags, errs) != FA_OK) return FA_ERR_CUDA;
  int dev;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  if (regs[dev] == 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FA_ERR_CUDA;
    regs[dev] = attr.numRegs;
  }
  if (regs[dev] * fa::kBwdThreads < fa::kBwdRegsNeeded) return FA_ERR_UNSUPPORTED;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return FA_ERR_CUDA;
  if (grid > unsigned(sms)) grid = unsigned(sms);  // persistent: at most one CTA per SM
  kernel<<<grid, fa::kBwdThreads, smem, stream>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool CAUSAL, bool SPARSE, bool XQK = false, bool DROP = false>
fa_status launch_dkdv(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                      const fa::BwdParamsT<DROP>& p, cudaStream_t stream) {
  static std::once_flag flags[kMaxDevices];
  static cudaError_t errs[kMaxDevices];
  static int regs[kMaxDevices];
  return launch_bwd_kernel(fa::fa_bwd_dkdv_kernel<D, CAUSAL, SPARSE, XQK, DROP>, fa::BwdCfg<D>::kSmemBytes,
                           unsigned(p.n_ktiles) * unsigned(p.BH), mq, mk, mv, mdo, p, stream, flags, errs, regs);
}

template <int D, bool CAUSAL, bool SPARSE, bool XQK = false, bool DROP = false>
fa_status launch_dq(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                    const fa::BwdParamsT<DROP>& p, cudaStream_t stream) {
  static std::once_flag flags[kMaxDevices];
  static cudaError_t errs[kMaxDevices];
  static int regs[kMaxDevices];
  return launch_bwd_kernel(fa::fa_bwd_dq_kernel<D, CAUSAL, SPARSE, XQK, DROP>, fa::BwdCfg<D>::kQSmemBytes,
                           unsigned(p.n_tiles) * unsigned(p.BH), mq, mk, mv, mdo, p, stream, flags, errs, regs);
}

struct BwdArgs {
  int BH;
  int Npad;     // N rounded up to a multiple of 128
  size_t rows;  // BH * Npad
  float* Drow;
  float* lse2;
};

// Checks shared by the backward stages; fills the workspace views.
// allow256: head dim 256 has only the fused backward (fa_bwd_fused*).
fa_status bwd_check(const void* ws, size_t ws_bytes, int B, int H, int N, int d, BwdArgs* a, bool allow256 = false) {
  fa_status s;
  if (ws == nullptr) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FA_ERR_ALIGNMENT;
  if ((s = check_sizes(B, H, N, d)) != FA_OK) return s;
  if (d == 256 && !allow256) return FA_ERR_UNSUPPORTED;
  if (ws_bytes < bwd_ws_bytes(B, H, N, d)) return FA_ERR_WORKSPACE;
  a->BH = B * H;
  a->Npad = (N + 127) / 128 * 128;
  a->rows = size_t(a->BH) * a->Npad;
  a->Drow = static_cast<float*>(const_cast<void*>(ws));
  a->lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(const_cast<void*>(ws)) + round256(a->rows * 4));
  return FA_OK;
}

fa_status bwd_pre(const void* o, const void* dO, const float* lse, void* ws, size_t ws_bytes, int B, int H, int N,
                  int d, int layout, void* stream, float* dqacc = nullptr) {
  fa_status s;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID_ARG;
  const int bnhd = layout == FA_LAYOUT_BNHD ? 1 : 0;
  if ((s = check_ptrs({o, dO, lse})) != FA_OK) return s;
  BwdArgs a;
  if ((s = bwd_check(ws, ws_bytes, B, H, N, d, &a, dqacc != nullptr)) != FA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long threads = static_cast<long long>(a.rows) * (d == 64 ? 8 : (d == 256 ? 32 : 16));  // D / 8 per row
  const unsigned grid = unsigned((threads + 255) / 256);
  const auto* ob = static_cast<const __nv_bfloat16*>(o);
  const auto* db = static_cast<const __nv_bfloat16*>(dO);
  const long long rows = static_cast<long long>(a.rows);
  if (d == 64)
    fa::fa_bwd_pre_kernel<64><<<grid, 256, 0, st>>>(ob, db, lse, a.Drow, a.lse2, N, a.Npad, d, H, bnhd, rows, dqacc);
  else if (d == 256)
    fa::fa_bwd_pre_kernel<256><<<grid, 256, 0, st>>>(ob, db, lse, a.Drow, a.lse2, N, a.Npad, d, H, bnhd, rows,
                                                     dqacc);
  else  // 96 or 128 (16 threads per row)
    fa::fa_bwd_pre_kernel<128><<<grid, 256, 0, st>>>(ob, db, lse, a.Drow, a.lse2, N, a.Npad, d, H, bnhd, rows,
                                                     dqacc);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

enum class BwdStage { kDkdv, kDq };

// dK/dV (stage kDkdv: dk, dv written) or dQ (stage kDq: dq written).
// N: query rows (the workspace's rows), Nk: key rows.
fa_status bwd_stage(BwdStage stage, const void* q, const void* k, const void* v, const void* dO, void* out0,
                    void* out1, const void* ws, size_t ws_bytes, const uint8_t* mask, int mask_block, int B, int H,
                    int N, int Nk, int d, int layout, int causal, float scale, void* stream,
                    const fa::DropParams* drop = nullptr) {
  fa_status s;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID_ARG;
  const bool bnhd = layout == FA_LAYOUT_BNHD;
  if ((s = check_ptrs({q, k, v, dO, out0})) != FA_OK) return s;
  if (stage == BwdStage::kDkdv && (s = check_ptrs({out1})) != FA_OK) return s;
  if (mask != nullptr && (mask_block != 128 || causal || Nk != N)) return FA_ERR_UNSUPPORTED;
  BwdArgs a;
  if ((s = bwd_check(ws, ws_bytes, B, H, N, d, &a)) != FA_OK) return s;
  if ((s = check_sizes(B, H, Nk, d)) != FA_OK) return s;
  if (drop != nullptr && (mask != nullptr || Nk != N || d == 96)) return FA_ERR_UNSUPPORTED;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if ((s = encoder()) != FA_OK) return s;
  int* status;
  if ((s = device_status_ptr(&status)) != FA_OK) return s;
  CUtensorMap mq, mk, mv, mdo;
  if ((s = make_map(&mq, q, B, H, N, d, bnhd, 128)) != FA_OK) return s;
  if ((s = make_map(&mk, k, B, H, Nk, d, bnhd, 128)) != FA_OK) return s;
  if ((s = make_map(&mv, v, B, H, Nk, d, bnhd, 128)) != FA_OK) return s;
  if ((s = make_map(&mdo, dO, B, H, N, d, bnhd, 128)) != FA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fa::BwdParams p;
  p.lse2 = a.lse2;
  p.Drow = a.Drow;
  p.dq = stage == BwdStage::kDq ? static_cast<__nv_bfloat16*>(out0) : nullptr;
  p.dk = stage == BwdStage::kDkdv ? static_cast<__nv_bfloat16*>(out0) : nullptr;
  p.dv = stage == BwdStage::kDkdv ? static_cast<__nv_bfloat16*>(out1) : nullptr;
  p.dk32 = nullptr;
  p.dv32 = nullptr;
  p.tile_mask = mask;
  p.status = status;
  set_wait_limit(&p.timeout_ns, &p.stall);
  p.N = N;
  p.Nk = Nk;
  p.BH = a.BH;
  p.H = H;
  p.bnhd = bnhd ? 1 : 0;
  // Rows are 128, 192 or 256 bytes, so every row of a 32-byte aligned output is aligned.
  p.v8 = ((reinterpret_cast<uintptr_t>(out0) | (out1 ? reinterpret_cast<uintptr_t>(out1) : 0)) & 31u) == 0 ? 1 : 0;
  p.n_tiles = (N + 127) / 128;
  p.n_ktiles = (Nk + 127) / 128;
  p.off = Nk - N;
  p.ds = d;
  p.scale = scale;
  fa::BwdParamsDrop pd;  // the dropout kernels' parameter block
  if (drop) {
    static_cast<fa::BwdParams&>(pd) = p;
    pd.drop = *drop;
  }
#define FA_BWD_DISPATCH(LAUNCH)                                                                  \
  if (drop)                                                                                      \
    return causal ? (d == 64 ? LAUNCH<64, true, false, false, true>(mq, mk, mv, mdo, pd, st)     \
                             : LAUNCH<128, true, false, false, true>(mq, mk, mv, mdo, pd, st))   \
                  : (d == 64 ? LAUNCH<64, false, false, false, true>(mq, mk, mv, mdo, pd, st)    \
                             : LAUNCH<128, false, false, false, true>(mq, mk, mv, mdo, pd, st)); \
  if (mask)                                                                                      \
    return d == 64 ? LAUNCH<64, false, true>(mq, mk, mv, mdo, p, st)                             \
                   : LAUNCH<128, false, true>(mq, mk, mv, mdo, p, st);                           \
  if (causal && Nk != N)                                                                         \
    return d == 64 ? LAUNCH<64, true, false, true>(mq, mk, mv, mdo, p, st)                       \
                   : LAUNCH<128, true, false, true>(mq, mk, mv, mdo, p, st);                     \
  if (causal)                                                                                    \
    return d == 64 ? LAUNCH<64, true, false>(mq, mk, mv, mdo, p, st)                             \
                   : LAUNCH<128, true, false>(mq, mk, mv, mdo, p, st);                           \
  return d == 64 ? LAUNCH<64, false, false>(mq, mk, mv, mdo, p, st)                              \
                 : LAUNCH<128, false, false>(mq, mk, mv, mdo, p, st);
  if (stage == BwdStage::kDkdv) {
    FA_BWD_DISPATCH(launch_dkdv)
  }
  FA_BWD_DISPATCH(launch_dq)
#undef FA_BWD_DISPATCH
}

fa_status bwd_common(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, const uint8_t* mask, int B, int H,
                     int N, int Nk, int d, int layout, int causal, float scale, void* stream,
                     const fa::DropParams* drop = nullptr) {
  fa_status s;
  // Validate everything before the first launch so that an error writes nothing.
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({q, k, v, o, lse, dO, dq, dk, dv})) != FA_OK) return s;
  BwdArgs a;
  if ((s = bwd_check(ws, ws_bytes, B, H, N, d, &a)) != FA_OK) return s;
  if ((s = check_sizes(B, H, Nk, d)) != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if (mask != nullptr && Nk != N) return FA_ERR_UNSUPPORTED;
  if (drop != nullptr && (mask != nullptr || Nk != N || d == 96)) return FA_ERR_UNSUPPORTED;
  if ((s = bwd_pre(o, dO, lse, ws, ws_bytes, B, H, N, d, layout, stream)) != FA_OK) return s;
  if ((s = bwd_stage(BwdStage::kDkdv, q, k, v, dO, dk, dv, ws, ws_bytes, mask, 128, B, H, N, Nk, d, layout, causal,
                     scale, stream, drop)) != FA_OK)
    return s;
  return bwd_stage(BwdStage::kDq, q, k, v, dO, dq, nullptr, ws, ws_bytes, mask, 128, B, H, N, Nk, d, layout, causal,
                   scale, stream, drop);
}

__global__ void fa_debug_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n, int mode) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  const uint64_t v = fa::f2(a, b);
  const float2 r = fa::f2_split(mode == 1 ? fa::ex2_poly_x2(v) : fa::ex2_mufu_x2(v));
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

// Self-test of the bounded waits: warp w waits on barrier w, which nothing ever
// completes. Warp 0 has the short limit and so records the timeout (site
// kSiteDebugWait) and raises the abort flag; warp 1 has a limit 64 times longer and
// honours the flag, as the kernels' other roles do. No copy, MMA or tensor memory
// is involved, so nothing is left to drain.
constexpr int kSiteDebugWait = 901;

__global__ void fa_debug_wait_kernel(unsigned long long timeout_ns, int* status, int* out) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_flag;
  const int w = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    fa::mbar_init(&bar[0], 1);
    fa::mbar_init(&bar[1], 1);
    abort_flag = 0;
    fa::fence_mbar_init();
  }
  __syncthreads();
  const unsigned long long limit = w == 0 ? timeout_ns : 64ull * timeout_ns;
  const fa::WaitCtl wc{&abort_flag, status, limit};
  const uint64_t t0 = fa::global_ns();
  const bool done = __any_sync(0xffffffffu, fa::mbar_wait(&bar[w], 0, wc, kSiteDebugWait + w));
  const uint64_t dt = fa::global_ns() - t0;
  if ((threadIdx.x & 31) == 0 && out != nullptr) {
    if (w == 0) {
      out[0] = (!done && dt >= limit) ? 1 : 0;
      out[2] = static_cast<int>(dt / 1000 < INT_MAX ? dt / 1000 : INT_MAX);
    } else {
      out[1] = (!done && dt < limit) ? 1 : 0;
    }
  }
}

}  // namespace

extern "C" {

fa_status fa_debug_exp2(const float* x, float* y, int n, int mode, void* stream) {
  if (n < 0 || (mode != 0 && mode != 1)) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (x == nullptr || y == nullptr) return FA_ERR_INVALID_ARG;
  const int pairs = (n + 1) / 2;
  fa_debug_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, mode);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_debug_wait_timeout(int timeout_us, int* out, void* stream) {
  if (timeout_us < 1 || timeout_us > 100000) return FA_ERR_INVALID_ARG;
  if (out != nullptr && (reinterpret_cast<uintptr_t>(out) & 3u) != 0) return FA_ERR_ALIGNMENT;
  int* status;
  if (device_status_ptr(&status) != FA_OK) return FA_ERR_CUDA;
  fa_debug_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * timeout_us, status, out);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_debug_stall_producer(int mode, int timeout_us) {
  if (mode == 0) {
    g_stall.store(0, std::memory_order_release);
    return FA_OK;
  }
  if (mode != 1 || timeout_us < 1 || timeout_us > 100000) return FA_ERR_INVALID_ARG;
  g_stall_limit_ns.store(1000ull * timeout_us, std::memory_order_relaxed);
  g_stall.store(1, std::memory_order_release);
  return FA_OK;
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

int fa_version(void) { return 100; }

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 int causal, float scale, void* stream) {
  return fwd_common(q, k, v, o, lse, nullptr, B, H, N, N, d, FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                    int d, int causal, float scale, void* stream) {
  return fwd_common(q, k, v, o, lse, nullptr, B, H, Nq, Nk, d, FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                    int d, int layout, int causal, float scale, void* stream) {
  return fwd_common(q, k, v, o, lse, nullptr, B, H, Nq, Nk, d, layout, causal != 0, scale, stream);
}

fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                             const uint8_t* tile_mask, int mask_block, int B, int H, int N, int d, float scale,
                             void* stream) {
  if (tile_mask == nullptr) return FA_ERR_INVALID_ARG;
  if (mask_block != 128) return FA_ERR_UNSUPPORTED;
  return fwd_common(q, k, v, o, lse, tile_mask, B, H, N, N, d, FA_LAYOUT_BHND, 0, scale, stream);
}

fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                         int d, int causal, float scale, float p_drop, uint64_t seed, uint32_t offset, void* stream) {
  fa::DropParams dp;
  const fa_status s = make_drop(p_drop, seed, offset, &dp);
  if (s != FA_OK) return s;
  return fwd_common(q, k, v, o, lse, nullptr, B, H, N, N, d, FA_LAYOUT_BHND, causal != 0, scale, stream, &dp);
}

fa_status fa_fwd_merge(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc, int B, int H,
                       int N, int d, int causal, float scale, void* stream) {
  if (o_acc == nullptr || lse_acc == nullptr) return FA_ERR_INVALID_ARG;
  // o and lse are not written by the merging kernels; the running result stands in for them.
  return fwd_common(q, k, v, o_acc, lse_acc, nullptr, B, H, N, N, d, FA_LAYOUT_BHND, causal != 0, scale, stream,
                    nullptr, o_acc, lse_acc);
}

fa_status fa_device_status(void* stream, int* detail) {
  int* status;
  if (detail) *detail = 0;
  if (device_status_ptr(&status) != FA_OK) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpy(h, status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaMemset(status, 0, sizeof(h)) != cudaSuccess) return FA_ERR_CUDA;
  if (detail) *detail = h[1];
  return h[0] == 0 ? FA_OK : static_cast<fa_status>(h[0]);
}

}  // extern "C"


extern "C" {

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) { return bwd_ws_bytes(B, H, N, d); }

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                 int causal, float scale, void* stream) {
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, nullptr, B, H, N, N, d,
                    FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                         int H, int N, int d, int causal, float scale, float p_drop, uint64_t seed, uint32_t offset,
                         void* stream) {
  fa::DropParams dp;
  const fa_status s = make_drop(p_drop, seed, offset, &dp);
  if (s != FA_OK) return s;
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, nullptr, B, H, N, N, d,
                    FA_LAYOUT_BHND, causal != 0, scale, stream, &dp);
}

fa_status fa_bwd_qk(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int Nq,
                    int Nk, int d, int causal, float scale, void* stream) {
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, nullptr, B, H, Nq, Nk, d,
                    FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int Nq,
                    int Nk, int d, int layout, int causal, float scale, void* stream) {
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, nullptr, B, H, Nq, Nk, d, layout,
                    causal != 0, scale, stream);
}

fa_status fa_bwd_preprocess(const void* o, const void* dO, const float* lse, void* workspace,
                            size_t workspace_bytes, int B, int H, int N, int d, void* stream) {
  return bwd_pre(o, dO, lse, workspace, workspace_bytes, B, H, N, d, FA_LAYOUT_BHND, stream);
}

fa_status fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                      const void* workspace, size_t workspace_bytes, const uint8_t* tile_mask, int mask_block, int B,
                      int H, int N, int d, int causal, float scale, void* stream) {
  return bwd_stage(BwdStage::kDkdv, q, k, v, dO, dk, dv, workspace, workspace_bytes, tile_mask, mask_block, B, H, N,
                   N, d, FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_bwd_dq(const void* q, const void* k, const void* v, const void* dO, void* dq, const void* workspace,
                    size_t workspace_bytes, const uint8_t* tile_mask, int mask_block, int B, int H, int N, int d,
                    int causal, float scale, void* stream) {
  return bwd_stage(BwdStage::kDq, q, k, v, dO, dq, nullptr, workspace, workspace_bytes, tile_mask, mask_block, B, H,
                   N, N, d, FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                             const uint8_t* tile_mask, int mask_block, int B, int H, int N, int d, float scale,
                             void* stream) {
  if (tile_mask == nullptr) return FA_ERR_INVALID_ARG;
  if (mask_block != 128) return FA_ERR_UNSUPPORTED;
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, tile_mask, B, H, N, N, d,
                    FA_LAYOUT_BHND, 0, scale, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------- fused backward
// One kernel for dK, dV and dQ (five products per tile pair instead of seven), with
// dQ reduced in fp32 into the workspace and converted to bf16 by a last launch.
namespace {

int dq_width(int d) { return d == 64 ? 64 : (d == 256 ? 256 : 128); }  // columns of the fp32 dQ accumulator

// Workspace: the two row arrays of the deterministic backward, then the fp32 dQ
// accumulator [B*H, Npad, 64 or 128], 256-byte aligned.
size_t fused_ws_bytes(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  const size_t rows = size_t(B) * H * ((size_t(N) + 127) / 128 * 128);
  return bwd_ws_bytes(B, H, N, d) + round256(rows * size_t(dq_width(d)) * 4);
}

float* fused_dqacc(const void* ws, int B, int H, int N, int d) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(const_cast<void*>(ws)) + bwd_ws_bytes(B, H, N, d));
}

fa_status fused_check(const void* ws, size_t ws_bytes, int B, int H, int N, int d, BwdArgs* a) {
  fa_status s;
  if ((s = bwd_check(ws, ws_bytes, B, H, N, d, a, true)) != FA_OK) return s;
  return ws_bytes < fused_ws_bytes(B, H, N, d) ? FA_ERR_WORKSPACE : FA_OK;
}

// The fp32 accumulator [BH, Npad, Dk] as a 3-D tensor (column, row, batch*head) for
// 32 x 32 reduce-add boxes with 128-byte swizzle (a box row is 32 fp32 = 128 bytes).
fa_status make_acc_map(CUtensorMap* m, const float* base, int BH, int Npad, int Dk, int box_rows = 32) {
  cuuint64_t dims[3] = {cuuint64_t(Dk), cuuint64_t(Npad), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(Dk) * 4, cuuint64_t(Npad) * cuuint64_t(Dk) * 4};
  cuuint32_t box[3] = {32, cuuint32_t(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool CAUSAL, bool SPARSE, bool XQK = false>
fa_status launch_fused(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                       const CUtensorMap& macc, const fa::BwdParams& p, cudaStream_t stream) {
  static std::once_flag flags[kMaxDevices];
  static cudaError_t errs[kMaxDevices];
  static int regs[kMaxDevices];
  auto kernel = fa::fa_bwd_fused_kernel<D, CAUSAL, SPARSE, XQK>;
  constexpr int smem = fa::FusedCfg<D>::kSmemBytes;
  if (set_smem(kernel, smem, flags, errs) != FA_OK) return FA_ERR_CUDA;
  int dev;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  if (regs[dev] == 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FA_ERR_CUDA;
    regs[dev] = attr.numRegs;
  }
  // The kernel re-divides its register pool between warpgroups.
  if (regs[dev] * fa::kFusedThreads < fa::kFusedRegsNeeded) return FA_ERR_UNSUPPORTED;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return FA_ERR_CUDA;
  // Causal: deal key tiles in pairs (j, n - 1 - j), one position per pair, when the
  // pairs leave at most 5% of the CTA rounds idle (they are of equal cost, so the last
  // round's empty slots are the whole imbalance); else single items, costliest first.
  fa::BwdParams q = p;
  long long npos = static_cast<long long>(p.n_ktiles) * p.BH;
  if (CAUSAL) {
    const long long pairs = static_cast<long long>((p.n_ktiles + 1) / 2) * p.BH;
    const long long slots = (pairs + sms - 1) / sms * sms;
    if (20 * (slots - pairs) <= slots) {
      q.paired = 1;
      npos = pairs;
    }
  }
  const unsigned grid = unsigned(npos < sms ? npos : sms);  // persistent: at most one CTA per SM
  kernel<<<grid, fa::kFusedThreads, smem, stream>>>(mq, mk, mv, mdo, macc, q);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool CAUSAL, bool SPARSE, bool XQK = false>
fa_status launch_bwd256(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                        const CUtensorMap& macc, const fa::BwdParams& p, cudaStream_t stream) {
  static std::once_flag flags[kMaxDevices];
  static cudaError_t errs[kMaxDevices];
  static int regs[kMaxDevices];
  auto kernel = fa::fa_bwd256_kernel<CAUSAL, SPARSE, XQK>;
  constexpr int smem = fa::Bwd256Cfg::kSmemBytes;
  if (set_smem(kernel, smem, flags, errs) != FA_OK) return FA_ERR_CUDA;
  int dev;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  if (regs[dev] == 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FA_ERR_CUDA;
    regs[dev] = attr.numRegs;
  }
  if (regs[dev] * fa::kBwdThreads < fa::kBwd256RegsNeeded) return FA_ERR_UNSUPPORTED;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return FA_ERR_CUDA;
  unsigned grid = 2u * unsigned(p.n_ktiles) * unsigned(p.BH);  // (key tile, column half, batch*head) items
  if (grid > unsigned(sms)) grid = unsigned(sms);
  kernel<<<grid, fa::kBwdThreads, smem, stream>>>(mq, mk, mv, mdo, macc, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// D and -lse log2 e rows, and the zeroed dQ accumulator.
fa_status fused_pre(const void* o, const void* dO, const float* lse, void* ws, size_t ws_bytes, int B, int H, int N,
                    int d, int layout, void* stream) {
  BwdArgs a;
  fa_status s;
  if (ws == nullptr) return FA_ERR_INVALID_ARG;
  if ((s = fused_check(ws, ws_bytes, B, H, N, d, &a)) != FA_OK) return s;
  return bwd_pre(o, dO, lse, ws, ws_bytes, B, H, N, d, layout, stream, fused_dqacc(ws, B, H, N, d));
}

// The fused kernel: dk, dv written, dQ added into the accumulator (which the
// pre-pass must have zeroed).
// f32: dk and dv are fp32 outputs (float*), else bf16.
fa_status fused_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, const void* ws,
                     size_t ws_bytes, const uint8_t* mask, int mask_block, int B, int H, int N, int Nk, int d,
                     int layout, int causal, float scale, void* stream, bool f32 = false) {
  fa_status s;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID_ARG;
  const bool bnhd = layout == FA_LAYOUT_BNHD;
  if ((s = check_ptrs({q, k, v, dO, dk, dv})) != FA_OK) return s;
  if (mask != nullptr && (mask_block != 128 || causal || Nk != N)) return FA_ERR_UNSUPPORTED;
  if (ws == nullptr) return FA_ERR_INVALID_ARG;
  BwdArgs a;
  if ((s = fused_check(ws, ws_bytes, B, H, N, d, &a)) != FA_OK) return s;
  if ((s = check_sizes(B, H, Nk, d)) != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if ((s = encoder()) != FA_OK) return s;
  int* status;
  if ((s = device_status_ptr(&status)) != FA_OK) return s;
  CUtensorMap mq, mk, mv, mdo, macc;
  // Head dim 256 visits queries in 64-row sub-tiles and reduces dQ in 32 x 16 boxes.
  const int qrows = d == 256 ? 64 : 128;
  if ((s = make_map(&mq, q, B, H, N, d, bnhd, qrows)) != FA_OK) return s;
  if ((s = make_map(&mk, k, B, H, Nk, d, bnhd, 128)) != FA_OK) return s;
  if ((s = make_map(&mv, v, B, H, Nk, d, bnhd, 128)) != FA_OK) return s;
  if ((s = make_map(&mdo, dO, B, H, N, d, bnhd, qrows)) != FA_OK) return s;
  if ((s = make_acc_map(&macc, fused_dqacc(ws, B, H, N, d), a.BH, a.Npad, dq_width(d), d == 256 ? 16 : 32)) !=
      FA_OK)
    return s;
  fa::BwdParams p;
  p.lse2 = a.lse2;
  p.Drow = a.Drow;
  p.dq = nullptr;
  p.dk = f32 ? nullptr : static_cast<__nv_bfloat16*>(dk);
  p.dv = f32 ? nullptr : static_cast<__nv_bfloat16*>(dv);
  p.dk32 = f32 ? static_cast<float*>(dk) : nullptr;
  p.dv32 = f32 ? static_cast<float*>(dv) : nullptr;
  p.tile_mask = mask;
  p.status = status;
  set_wait_limit(&p.timeout_ns, &p.stall);
  p.N = N;
  p.Nk = Nk;
  p.BH = a.BH;
  p.H = H;
  p.bnhd = bnhd ? 1 : 0;
  p.v8 = ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 31u) == 0 ? 1 : 0;
  p.n_tiles = (N + 127) / 128;
  p.n_ktiles = (Nk + 127) / 128;
  p.off = Nk - N;
  p.ds = d;
  p.scale = scale;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 256) {
    if (mask) return launch_bwd256<false, true>(mq, mk, mv, mdo, macc, p, st);
    if (causal && Nk != N) return launch_bwd256<true, false, true>(mq, mk, mv, mdo, macc, p, st);
    if (causal) return launch_bwd256<true, false>(mq, mk, mv, mdo, macc, p, st);
    return launch_bwd256<false, false>(mq, mk, mv, mdo, macc, p, st);
  }
  if (mask)
    return d == 64 ? launch_fused<64, false, true>(mq, mk, mv, mdo, macc, p, st)
                   : launch_fused<128, false, true>(mq, mk, mv, mdo, macc, p, st);
  if (causal && Nk != N)
    return d == 64 ? launch_fused<64, true, false, true>(mq, mk, mv, mdo, macc, p, st)
                   : launch_fused<128, true, false, true>(mq, mk, mv, mdo, macc, p, st);
  if (causal)
    return d == 64 ? launch_fused<64, true, false>(mq, mk, mv, mdo, macc, p, st)
                   : launch_fused<128, true, false>(mq, mk, mv, mdo, macc, p, st);
  return d == 64 ? launch_fused<64, false, false>(mq, mk, mv, mdo, macc, p, st)
                 : launch_fused<128, false, false>(mq, mk, mv, mdo, macc, p, st);
}

// dq = bf16(scale * accumulator) for the N real rows of every (batch, head).
fa_status fused_dq(void* dq, const void* ws, size_t ws_bytes, int B, int H, int N, int d, int layout, float scale,
                   void* stream) {
  fa_status s;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({dq})) != FA_OK) return s;
  if (ws == nullptr) return FA_ERR_INVALID_ARG;
  BwdArgs a;
  if ((s = fused_check(ws, ws_bytes, B, H, N, d, &a)) != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  const long long rows = static_cast<long long>(a.BH) * N;
  const int Dk = dq_width(d);
  const long long threads = rows * (Dk / 8);
  const unsigned grid = unsigned((threads + 255) / 256);
  const float* acc = fused_dqacc(ws, B, H, N, d);
  auto* out = static_cast<__nv_bfloat16*>(dq);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bnhd = layout == FA_LAYOUT_BNHD ? 1 : 0;
  if (Dk == 64)
    fa::fa_dq_convert_kernel<64><<<grid, 256, 0, st>>>(acc, out, N, a.Npad, d, H, bnhd, rows, scale);
  else if (Dk == 256)
    fa::fa_dq_convert_kernel<256><<<grid, 256, 0, st>>>(acc, out, N, a.Npad, d, H, bnhd, rows, scale);
  else
    fa::fa_dq_convert_kernel<128><<<grid, 256, 0, st>>>(acc, out, N, a.Npad, d, H, bnhd, rows, scale);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fused_common(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                       void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, const uint8_t* mask, int mask_block,
                       int B, int H, int N, int Nk, int d, int layout, int causal, float scale, void* stream) {
  fa_status s;
  // Validate everything before the first launch so that an error writes nothing.
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BNHD) return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({q, k, v, o, lse, dO, dq, dk, dv})) != FA_OK) return s;
  if (ws == nullptr) return FA_ERR_INVALID_ARG;
  BwdArgs a;
  if ((s = fused_check(ws, ws_bytes, B, H, N, d, &a)) != FA_OK) return s;
  if ((s = check_sizes(B, H, Nk, d)) != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if (mask != nullptr && (mask_block != 128 || causal || Nk != N)) return FA_ERR_UNSUPPORTED;
  if ((s = fused_pre(o, dO, lse, ws, ws_bytes, B, H, N, d, layout, stream)) != FA_OK) return s;
  if ((s = fused_main(q, k, v, dO, dk, dv, ws, ws_bytes, mask, mask_block, B, H, N, Nk, d, layout, causal, scale,
                      stream)) != FA_OK)
    return s;
  return fused_dq(dq, ws, ws_bytes, B, H, N, d, layout, scale, stream);
}

}  // namespace

extern "C" {

size_t fa_bwd_fused_workspace_bytes(int B, int H, int N, int d) { return fused_ws_bytes(B, H, N, d); }

fa_status fa_bwd_fused(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                       void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N,
                       int d, int causal, float scale, void* stream) {
  return fused_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, nullptr, 128, B, H, N, N, d,
                      FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_bwd_fused_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                          const uint8_t* tile_mask, int mask_block, int B, int H, int Nq, int Nk, int d, int layout,
                          int causal, float scale, void* stream) {
  return fused_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, tile_mask, mask_block, B, H, Nq,
                      Nk, d, layout, causal != 0, scale, stream);
}

fa_status fa_bwd_fused_preprocess(const void* o, const void* dO, const float* lse, void* workspace,
                                  size_t workspace_bytes, int B, int H, int N, int d, void* stream) {
  return fused_pre(o, dO, lse, workspace, workspace_bytes, B, H, N, d, FA_LAYOUT_BHND, stream);
}

fa_status fa_bwd_fused_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, const uint8_t* tile_mask, int mask_block, int B,
                            int H, int N, int d, int causal, float scale, void* stream) {
  return fused_main(q, k, v, dO, dk, dv, workspace, workspace_bytes, tile_mask, mask_block, B, H, N, N, d,
                    FA_LAYOUT_BHND, causal != 0, scale, stream);
}

fa_status fa_bwd_fused_main_f32(const void* q, const void* k, const void* v, const void* dO, float* dk, float* dv,
                                void* workspace, size_t workspace_bytes, int B, int H, int N, int d, int causal,
                                float scale, void* stream) {
  if (d == 256) return FA_ERR_UNSUPPORTED;  // the head-dim-256 kernel writes bf16 only
  return fused_main(q, k, v, dO, dk, dv, workspace, workspace_bytes, nullptr, 128, B, H, N, N, d, FA_LAYOUT_BHND,
                    causal != 0, scale, stream, true);
}

fa_status fa_bwd_fused_dq(void* dq, const void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                          float scale, void* stream) {
  return fused_dq(dq, workspace, workspace_bytes, B, H, N, d, FA_LAYOUT_BHND, scale, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------- no-allocation backward
// Scratch for fa_bwd_noalloc: a fixed array compiled into the library, so callers
// that may not allocate device memory can still run the backward. Every device
// that loads the library holds it until exit. In host code `g_noalloc_scratch`
// only names the symbol; its device address comes from cudaGetSymbolAddress,
// looked up once per device in noalloc_scratch() below.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

struct NoallocState {
  std::once_flag once;
  void* ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
NoallocState g_noalloc[kMaxDevices];

// Device address of the scratch array on the current device (first call: lookup).
fa_status noalloc_scratch(void** out) {
  int dev;
  if (current_device(&dev) != FA_OK) return FA_ERR_CUDA;
  NoallocState& st = g_noalloc[dev];
  std::call_once(st.once, [&] {
    void* ptr = nullptr;
    st.err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    st.ptr = (st.err == cudaSuccess) ? ptr : nullptr;
  });
  if (st.err != cudaSuccess || st.ptr == nullptr) return FA_ERR_CUDA;
  *out = st.ptr;
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                    const void* dO, void* dq, void* dk, void* dv, const uint8_t* tile_mask,
                                    int mask_block, int B, int H, int N, int d, int causal, float scale,
                                    void* stream) {
  fa_status s;
  if ((s = check_ptrs({q, k, v, o, lse, dO, dq, dk, dv})) != FA_OK) return s;
  if ((s = check_sizes(B, H, N, d)) != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if (tile_mask != nullptr && (mask_block != 128 || causal)) return FA_ERR_UNSUPPORTED;
  const size_t need = bwd_ws_bytes(B, H, N, d);
  if (need > size_t(FA_BWD_NOALLOC_SCRATCH_BYTES)) return FA_ERR_WORKSPACE;
  void* scratch;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  // The pre-pass rewrites every row the other two launches read, so whatever an
  // earlier call left in the array does not matter.
  const size_t bytes = size_t(FA_BWD_NOALLOC_SCRATCH_BYTES);
  if ((s = bwd_pre(o, dO, lse, scratch, bytes, B, H, N, d, FA_LAYOUT_BHND, stream)) != FA_OK) return s;
  if ((s = bwd_stage(BwdStage::kDkdv, q, k, v, dO, dk, dv, scratch, bytes, tile_mask, mask_block, B, H, N, N, d,
                     FA_LAYOUT_BHND, causal, scale, stream)) != FA_OK)
    return s;
  return bwd_stage(BwdStage::kDq, q, k, v, dO, dq, nullptr, scratch, bytes, tile_mask, mask_block, B, H, N, N, d,
                   FA_LAYOUT_BHND, causal, scale, stream);
}
