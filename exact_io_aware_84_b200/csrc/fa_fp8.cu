// FP8 operand preparation for the FP8 forward (head dim 128).
//
// Incoherent processing (marketmaker.cc "Flash Attention and the
// sequence-length problem", section "FA3: Hopper mechanics", item 3): Q and K
// are multiplied by a random orthogonal matrix R = diag(s) H / sqrt(d) (H the
// Sylvester Hadamard matrix, s random signs supplied by the caller), which
// leaves Q K^T unchanged and spreads outlier channels over all coordinates,
// then quantised to float8 e4m3 block by block:
//   Q, K : one scale per (head, 128-row block), scale = amax / 448
//   V    : one scale per (head, channel), stored transposed [head][dim][key]
//          so that it is the K-major operand of the P V product.
// code = e4m3(x / scale) rounded to nearest even with saturation; scale = 1
// when amax = 0.  The rotation is the fast Walsh-Hadamard transform in fp32:
// signs, butterflies of span 1, 2, ..., 64, then the factor 1/sqrt(128).
//
// All three kernels are memory-bound streams (read 2 B, write 1 B per
// element; V is read twice, once for its channel maxima).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_kernels.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kD = 128;
constexpr float kE4m3Max = 448.0f;
constexpr float kRsqrt128 = 0.0883883476483184405501f;  // 1 / sqrt(128), rounded to fp32

template <bool BF16>
__device__ __forceinline__ void load8(const void* src, float* f) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t;
    if constexpr (BF16) {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
      t = __bfloat1622float2(h);
    } else {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      t = __half22float2(h);
    }
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f; }

// Q and K: one CTA per (128-row block, head, tensor), one thread per row.
template <bool BF16>
__global__ void __launch_bounds__(128) fa_fp8_rows_kernel(const void* __restrict__ q, const void* __restrict__ k,
                                                          const float* __restrict__ signs, uint8_t* __restrict__ q8,
                                                          uint8_t* __restrict__ k8, float* __restrict__ sq,
                                                          float* __restrict__ sk, int N, int n_pad, int nb) {
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const void* src = which ? k : q;
  uint8_t* dst = which ? k8 : q8;
  float* sc = which ? sk : sq;
  const int row = blk * 128 + threadIdx.x;
  float v[kD];
  if (row < N) {
    const uint8_t* r = reinterpret_cast<const uint8_t*>(src) + ((size_t)bh * N + row) * kD * 2;
#pragma unroll
    for (int c = 0; c < kD / 8; ++c) load8<BF16>(r + 16 * c, v + 8 * c);
  } else {
#pragma unroll
    for (int c = 0; c < kD; ++c) v[c] = 0.f;
  }
  if (signs != nullptr) {
#pragma unroll
    for (int c = 0; c < kD; ++c) v[c] *= signs[c];
#pragma unroll
    for (int h = 1; h < kD; h <<= 1) {
#pragma unroll
      for (int i = 0; i < kD; ++i) {
        if ((i & h) == 0) {
          const float a = v[i], b = v[i + h];
          v[i] = a + b;
          v[i + h] = a - b;
        }
      }
    }
#pragma unroll
    for (int c = 0; c < kD; ++c) v[c] *= kRsqrt128;
  }
  float m = 0.f;
#pragma unroll
  for (int c = 0; c < kD; ++c) m = fmaxf(m, fabsf(v[c]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[4];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  const float amax = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
  const float s = scale_of(amax);
  if (threadIdx.x == 0) sc[(size_t)bh * nb + blk] = s;
  if (row < n_pad) {
    uint4* out = reinterpret_cast<uint4*>(dst + ((size_t)bh * n_pad + row) * kD);
#pragma unroll
    for (int c = 0; c < kD / 16; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float* x = v + 16 * c + 4 * e;
        w[e] = pack_e4m3x4(__fdiv_rn(x[0], s), __fdiv_rn(x[1], s), __fdiv_rn(x[2], s), __fdiv_rn(x[3], s));
      }
      out[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// V channel maxima: one CTA per (256-row chunk, head); 16 threads per row, 8
// channels each; the chunk's maxima are merged with an integer atomic max on
// the (non-negative) float bits.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_fp8_vamax_kernel(const void* __restrict__ v, unsigned* __restrict__ vamax,
                                                           int N) {
  const int bh = blockIdx.y;
  const int c8 = threadIdx.x & 15, r16 = threadIdx.x >> 4;
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int r_end = min(N, (int)(blockIdx.x + 1) * 256);
  for (int r = blockIdx.x * 256 + r16; r < r_end; r += 16) {
    float f[8];
    load8<BF16>(reinterpret_cast<const uint8_t*>(v) + (((size_t)bh * N + r) * kD + 8 * c8) * 2, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
  }
  __shared__ float part[16][kD];
#pragma unroll
  for (int e = 0; e < 8; ++e) part[r16][8 * c8 + e] = m[e];
  __syncthreads();
  if (threadIdx.x < kD) {
    float x = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) x = fmaxf(x, part[i][threadIdx.x]);
    atomicMax(vamax + (size_t)bh * kD + threadIdx.x, __float_as_uint(x));
  }
}

// V codes, transposed: one CTA per (128-key block, head).  Codes are gathered
// in shared memory as [dim][key] and written out as 128-byte rows.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_fp8_vt_kernel(const void* __restrict__ v,
                                                        const unsigned* __restrict__ vamax,
                                                        uint8_t* __restrict__ v8t, float* __restrict__ sv, int N,
                                                        int n_pad) {
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int c8 = threadIdx.x & 15, r16 = threadIdx.x >> 4;
  __shared__ __align__(16) uint8_t tile[kD][128];
  float s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) s[e] = scale_of(__uint_as_float(vamax[(size_t)bh * kD + 8 * c8 + e]));
  if (blk == 0 && r16 == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) sv[(size_t)bh * kD + 8 * c8 + e] = s[e];
  }
#pragma unroll
  for (int pass = 0; pass < 8; ++pass) {
    const int key = pass * 16 + r16;
    const int r = blk * 128 + key;
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < N) load8<BF16>(reinterpret_cast<const uint8_t*>(v) + (((size_t)bh * N + r) * kD + 8 * c8) * 2, f);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const uint32_t two = pack_e4m3x2(__fdiv_rn(f[e], s[e]), __fdiv_rn(f[e + 1], s[e + 1]));
      tile[8 * c8 + e][key] = (uint8_t)(two & 0xffu);
      tile[8 * c8 + e + 1][key] = (uint8_t)(two >> 8);
    }
  }
  __syncthreads();
  // 128 dims x 128 keys = 1024 16-byte chunks, four per thread
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int chunk = threadIdx.x + 256 * i;
    const int dim = chunk >> 3, part8 = chunk & 7;
    const uint4 val = *reinterpret_cast<const uint4*>(&tile[dim][16 * part8]);
    *reinterpret_cast<uint4*>(v8t + ((size_t)bh * kD + dim) * n_pad + (size_t)blk * 128 + 16 * part8) = val;
  }
}

}  // namespace

cudaError_t launch_fp8_prep(bool bf16, const void* q, const void* k, const void* v, const float* signs,
                            const Fp8Buffers& b, int bh, int N, cudaStream_t st) {
  const int nb = (N + 127) / 128;
  const int n_pad = nb * 128;
  cudaError_t e = cudaMemsetAsync(b.vamax, 0, (size_t)bh * kD * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  const dim3 g_rows(nb, bh, 2), g_vamax((N + 255) / 256, bh), g_vt(nb, bh);
  if (bf16) {
    fa_fp8_rows_kernel<true><<<g_rows, 128, 0, st>>>(q, k, signs, b.q8, b.k8, b.sq, b.sk, N, n_pad, nb);
    fa_fp8_vamax_kernel<true><<<g_vamax, 256, 0, st>>>(v, b.vamax, N);
    fa_fp8_vt_kernel<true><<<g_vt, 256, 0, st>>>(v, b.vamax, b.v8t, b.sv, N, n_pad);
  } else {
    fa_fp8_rows_kernel<false><<<g_rows, 128, 0, st>>>(q, k, signs, b.q8, b.k8, b.sq, b.sk, N, n_pad, nb);
    fa_fp8_vamax_kernel<false><<<g_vamax, 256, 0, st>>>(v, b.vamax, N);
    fa_fp8_vt_kernel<false><<<g_vt, 256, 0, st>>>(v, b.vamax, b.v8t, b.sv, N, n_pad);
  }
  return cudaGetLastError();
}

}  // namespace fa
