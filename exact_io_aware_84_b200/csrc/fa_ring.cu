// Ring-attention helpers: merging partial (O, LSE) results over disjoint key
// sets, accumulating 16-bit gradient partials into fp32, and writing fp32
// results out in 16 bits.  All three are memory-bound streams: each element is read once and written once, with
// 16-byte vector accesses and a grid-stride loop over a grid sized to the SMs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int kThreads = 256;

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if constexpr (BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
  if constexpr (BF16) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
}

// One row of D floats is handled by D/4 consecutive threads (a float4 each).
// (o, lse) <- merge((o, lse), (o_part, lse_part)):
//   m = max(LSE_a, LSE_b), w = e^{LSE - m}, LSE = m + ln(w_a + w_b),
//   O = (w_a O_a + w_b O_b) / (w_a + w_b); both -inf: O = 0, LSE = -inf.
// When `out` is set, O is also written there in the 16-bit type (OUT = 1 bf16,
// 2 fp16).
template <int D, int OUT>
__global__ void __launch_bounds__(kThreads) fa_merge_kernel(float* __restrict__ o, float* __restrict__ lse,
                                                            const float* __restrict__ o_part,
                                                            const float* __restrict__ lse_part,
                                                            void* __restrict__ out, long long rows) {
  constexpr int TPR = D / 4;                 // threads per row
  constexpr int RPB = kThreads / TPR;        // rows per block pass
  const int sub = threadIdx.x % TPR;
  for (long long row = (long long)blockIdx.x * RPB + threadIdx.x / TPR; row < rows;
       row += (long long)gridDim.x * RPB) {
    const float la = lse[row], lb = lse_part[row];
    const float m = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, l_new = -INFINITY;
    if (m != -INFINITY) {
      wa = expf(la - m);                     // 0 when la = -inf
      wb = expf(lb - m);
      const float tot = wa + wb;
      l_new = m + logf(tot);
      wa /= tot;
      wb /= tot;
    }
    const size_t off = (size_t)row * D + 4 * sub;
    const float4 a = *reinterpret_cast<const float4*>(o + off);
    const float4 b = *reinterpret_cast<const float4*>(o_part + off);
    float4 r;
    r.x = wa * a.x + wb * b.x;
    r.y = wa * a.y + wb * b.y;
    r.z = wa * a.z + wb * b.z;
    r.w = wa * a.w + wb * b.w;
    if (m == -INFINITY) r = make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(o + off) = r;
    if constexpr (OUT != 0) {
      uint2 h = make_uint2(pack2<OUT == 1>(r.x, r.y), pack2<OUT == 1>(r.z, r.w));
      *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + off) = h;
    }
    if (sub == 0) lse[row] = l_new;
  }
}

// acc[i] += float(src[i]); eight elements per thread per pass (16 bytes of
// 16-bit input), the ragged tail element by element.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) fa_accumulate_kernel(float* __restrict__ acc,
                                                                 const void* __restrict__ src, long long n) {
  const long long n8 = n / 8;
  const uint4* s8 = reinterpret_cast<const uint4*>(src);
  float4* a4 = reinterpret_cast<float4*>(acc);
  for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < n8; i += (long long)gridDim.x * kThreads) {
    const uint4 u = s8[i];
    const float2 f0 = unpack2<BF16>(u.x), f1 = unpack2<BF16>(u.y), f2 = unpack2<BF16>(u.z), f3 = unpack2<BF16>(u.w);
    float4 x = a4[2 * i], y = a4[2 * i + 1];
    x.x += f0.x; x.y += f0.y; x.z += f1.x; x.w += f1.y;
    y.x += f2.x; y.y += f2.y; y.z += f3.x; y.w += f3.y;
    a4[2 * i] = x;
    a4[2 * i + 1] = y;
  }
  const long long t = 8 * n8 + (long long)blockIdx.x * kThreads + threadIdx.x;
  if (t < n && t < 8 * n8 + 8) {
    const uint16_t* s = reinterpret_cast<const uint16_t*>(src);
    uint32_t u = s[t];
    acc[t] += unpack2<BF16>(u).x;
  }
}

// dst[i] = 16-bit(src[i]) (round to nearest even); four elements per thread
// per pass, the ragged tail element by element.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) fa_convert_kernel(void* __restrict__ dst, const float* __restrict__ src,
                                                              long long n) {
  const long long n4 = n / 4;
  for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < n4; i += (long long)gridDim.x * kThreads) {
    const float4 f = reinterpret_cast<const float4*>(src)[i];
    reinterpret_cast<uint2*>(dst)[i] = make_uint2(pack2<BF16>(f.x, f.y), pack2<BF16>(f.z, f.w));
  }
  const long long t = 4 * n4 + (long long)blockIdx.x * kThreads + threadIdx.x;
  if (t < n && t < 4 * n4 + 4) reinterpret_cast<uint16_t*>(dst)[t] = (uint16_t)(pack2<BF16>(src[t], 0.f) & 0xffffu);
}

int grid_for(long long items, int per_block, int sms) {
  long long g = (items + per_block - 1) / per_block;
  const long long cap = (long long)sms * 8;  // 8 resident 256-thread blocks per SM
  if (g > cap) g = cap;
  return g < 1 ? 1 : (int)g;
}

}  // namespace

cudaError_t launch_merge(int d, int out_kind, float* o, float* lse, const float* o_part, const float* lse_part,
                         void* out, long long rows, int sms, cudaStream_t st) {
  const int rpb = kThreads / (d / 4);
  const int grid = grid_for(rows, rpb, sms);
#define FA_MERGE_LAUNCH(DD, OO) \
  fa_merge_kernel<DD, OO><<<grid, kThreads, 0, st>>>(o, lse, o_part, lse_part, out, rows)
  if (d == 64) {
    if (out_kind == 0) FA_MERGE_LAUNCH(64, 0);
    else if (out_kind == 1) FA_MERGE_LAUNCH(64, 1);
    else FA_MERGE_LAUNCH(64, 2);
  } else {
    if (out_kind == 0) FA_MERGE_LAUNCH(128, 0);
    else if (out_kind == 1) FA_MERGE_LAUNCH(128, 1);
    else FA_MERGE_LAUNCH(128, 2);
  }
#undef FA_MERGE_LAUNCH
  return cudaGetLastError();
}

cudaError_t launch_accumulate(bool bf16, float* acc, const void* src, long long n, int sms, cudaStream_t st) {
  const int grid = grid_for((n + 7) / 8, kThreads, sms);
  if (bf16)
    fa_accumulate_kernel<true><<<grid, kThreads, 0, st>>>(acc, src, n);
  else
    fa_accumulate_kernel<false><<<grid, kThreads, 0, st>>>(acc, src, n);
  return cudaGetLastError();
}

cudaError_t launch_convert(bool bf16, void* dst, const float* src, long long n, int sms, cudaStream_t st) {
  const int grid = grid_for((n + 3) / 4, kThreads, sms);
  if (bf16)
    fa_convert_kernel<true><<<grid, kThreads, 0, st>>>(dst, src, n);
  else
    fa_convert_kernel<false><<<grid, kThreads, 0, st>>>(dst, src, n);
  return cudaGetLastError();
}

}  // namespace fa
