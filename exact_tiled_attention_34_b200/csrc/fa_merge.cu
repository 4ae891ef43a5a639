// fa_merge.cu - element-wise kernels for attention split over key blocks (the
// sequence-parallel ring): merging partial outputs through their log-sum-exp, and
// fp32 accumulation of partial gradients. All are HBM-bound: one pass over their
// operands, 16-byte vector accesses, grids sized in whole rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>

#include "fa.h"

namespace {

// Threads of one row: d / 8 (8 or 16), each owning 8 consecutive columns; a row's
// threads sit in one warp, so a warp-level barrier orders the log-sum-exp update.
__global__ void fa_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                const __nv_bfloat16* __restrict__ o_part, const float* __restrict__ lse_part,
                                long long rows, int tpr) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = t / tpr;
  const int chunk = static_cast<int>(t - row * tpr);
  const bool live = row < rows;
  float a = -INFINITY, b = -INFINITY;
  if (live) {
    a = lse_acc[row];
    b = lse_part[row];
  }
  __syncwarp();  // every thread of the row has read lse_acc before it is overwritten
  if (!live) return;
  const float m = fmaxf(a, b);
  float wa = 0.f, wb = 0.f, lse = -INFINITY;
  if (m != -INFINITY) {  // some key of either part visible: weights relative to the larger
    wa = expf(a - m);
    wb = expf(b - m);
    const float s = wa + wb;
    lse = m + logf(s);
    wa /= s;
    wb /= s;
  }
  const size_t base = static_cast<size_t>(row) * (tpr * 8) + chunk * 8;
  float4* acc = reinterpret_cast<float4*>(o_acc + base);
  const uint4 pv = *reinterpret_cast<const uint4*>(o_part + base);
  const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
  float x[8];
  const float4 a0 = acc[0], a1 = acc[1];
  const float ao[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[e]));
    x[2 * e] = ao[2 * e] * wa + f.x * wb;
    x[2 * e + 1] = ao[2 * e + 1] * wa + f.y * wb;
  }
  acc[0] = make_float4(x[0], x[1], x[2], x[3]);
  acc[1] = make_float4(x[4], x[5], x[6], x[7]);
  if (chunk == 0) lse_acc[row] = lse;
}

// acc[i] (+)= x[i] for 8 elements per thread.
__global__ void fa_accumulate_kernel(float* __restrict__ acc, const __nv_bfloat16* __restrict__ x, long long n8,
                                     int overwrite) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n8) return;
  const uint4 xv = reinterpret_cast<const uint4*>(x)[t];
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  float4* a = reinterpret_cast<float4*>(acc) + 2 * t;
  float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
  if (!overwrite) {
    a0 = a[0];
    a1 = a[1];
  }
  const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[0]));
  const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[1]));
  const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[2]));
  const float2 f3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[3]));
  a[0] = make_float4(a0.x + f0.x, a0.y + f0.y, a0.z + f1.x, a0.w + f1.y);
  a[1] = make_float4(a1.x + f2.x, a1.y + f2.y, a1.z + f3.x, a1.w + f3.y);
}

// acc[i] += x[i] (fp32), 8 elements per thread.
__global__ void fa_accumulate_f32_kernel(float* __restrict__ acc, const float* __restrict__ x, long long n8) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n8) return;
  float4* a = reinterpret_cast<float4*>(acc) + 2 * t;
  const float4* b = reinterpret_cast<const float4*>(x) + 2 * t;
  const float4 a0 = a[0], a1 = a[1], b0 = b[0], b1 = b[1];
  a[0] = make_float4(a0.x + b0.x, a0.y + b0.y, a0.z + b0.z, a0.w + b0.w);
  a[1] = make_float4(a1.x + b1.x, a1.y + b1.y, a1.z + b1.z, a1.w + b1.w);
}

// out[i] = bf16(in[i]) (round to nearest even), 8 elements per thread.
__global__ void fa_to_bf16_kernel(__nv_bfloat16* __restrict__ out, const float* __restrict__ in, long long n8) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n8) return;
  const float4* s = reinterpret_cast<const float4*>(in) + 2 * t;
  const float4 a0 = s[0], a1 = s[1];
  __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a0.x, a0.y), __floats2bfloat162_rn(a0.z, a0.w),
                         __floats2bfloat162_rn(a1.x, a1.y), __floats2bfloat162_rn(a1.z, a1.w)};
  reinterpret_cast<uint4*>(out)[t] = *reinterpret_cast<const uint4*>(h);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

unsigned blocks_for(long long threads) { return static_cast<unsigned>((threads + 255) / 256); }

// Launches of 256 threads cover at most INT_MAX blocks (the grid's x limit).
bool grid_fits(long long threads) { return threads <= static_cast<long long>(INT_MAX) * 256; }

}  // namespace

extern "C" {

fa_status fa_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, long long rows,
                           int d, void* stream) {
  if (rows < 0 || (d != 64 && d != 128)) return rows < 0 ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  if (rows == 0) return FA_OK;
  if (!o_acc || !lse_acc || !o_part || !lse_part) return FA_ERR_INVALID_ARG;
  if (!aligned(o_acc, 16) || !aligned(o_part, 16) || !aligned(lse_acc, 4) || !aligned(lse_part, 4))
    return FA_ERR_ALIGNMENT;
  const int tpr = d / 8;
  if (rows > (1LL << 40) || !grid_fits(rows * tpr)) return FA_ERR_UNSUPPORTED;
  fa_merge_kernel<<<blocks_for(rows * tpr), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      o_acc, lse_acc, static_cast<const __nv_bfloat16*>(o_part), lse_part, rows, tpr);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_accumulate_bf16(float* acc, const void* x, long long n, int overwrite, void* stream) {
  if (n < 0 || n % 8 != 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!acc || !x) return FA_ERR_INVALID_ARG;
  if (!aligned(acc, 16) || !aligned(x, 16)) return FA_ERR_ALIGNMENT;
  if (!grid_fits(n / 8)) return FA_ERR_UNSUPPORTED;
  fa_accumulate_kernel<<<blocks_for(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      acc, static_cast<const __nv_bfloat16*>(x), n / 8, overwrite != 0);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_accumulate_f32(float* acc, const float* x, long long n, void* stream) {
  if (n < 0 || n % 8 != 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!acc || !x) return FA_ERR_INVALID_ARG;
  if (!aligned(acc, 16) || !aligned(x, 16)) return FA_ERR_ALIGNMENT;
  if (!grid_fits(n / 8)) return FA_ERR_UNSUPPORTED;
  fa_accumulate_f32_kernel<<<blocks_for(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(acc, x, n / 8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_to_bf16(void* out, const float* in, long long n, void* stream) {
  if (n < 0 || n % 8 != 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!out || !in) return FA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(in, 16)) return FA_ERR_ALIGNMENT;
  if (!grid_fits(n / 8)) return FA_ERR_UNSUPPORTED;
  fa_to_bf16_kernel<<<blocks_for(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<__nv_bfloat16*>(out), in, n / 8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
