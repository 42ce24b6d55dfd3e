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

// Two 16-bit values (low half first) to floats, without taking addresses.
template <bool BF16>
__device__ __forceinline__ float2 unpack16x2(uint32_t x) {
  if constexpr (BF16) {
    return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
  } else {
    return make_float2(__half2float(__ushort_as_half((unsigned short)(x & 0xffffu))),
                       __half2float(__ushort_as_half((unsigned short)(x >> 16))));
  }
}

template <bool BF16>
__device__ __forceinline__ void load8(const void* src, float* f) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const float2 a = unpack16x2<BF16>(u.x), b = unpack16x2<BF16>(u.y), c = unpack16x2<BF16>(u.z),
               d = unpack16x2<BF16>(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f; }

// Q and K: one CTA per (128-row block, head, tensor); each warp takes 16 rows,
// lane l holding elements 4l..4l+3 of every row (coalesced 256-byte row
// loads and 128-byte code stores).  The transform's spans 1 and 2 stay in a
// lane, spans 4..64 pair lane l with lane l ^ (span / 4); at every stage the
// lower element of a pair becomes a + b and the upper a - b.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_fp8_rows_kernel(const void* __restrict__ q, const void* __restrict__ k,
                                                          const float* __restrict__ signs, uint8_t* __restrict__ q8,
                                                          uint8_t* __restrict__ k8, float* __restrict__ sq,
                                                          float* __restrict__ sk, int N, int n_pad, int nb) {
  constexpr int kRows = 16;  // rows per warp
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const void* src = which ? k : q;
  uint8_t* dst = which ? k8 : q8;
  float* sc = which ? sk : sq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blk * 128 + warp * kRows;
  float v[kRows][4];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int row = row0 + r;
    if (row < N) {
      const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(src) +
                                                      (((size_t)bh * N + row) * kD + 4 * lane) * 2);
      const float2 a = unpack16x2<BF16>(u.x), b = unpack16x2<BF16>(u.y);
      v[r][0] = a.x;
      v[r][1] = a.y;
      v[r][2] = b.x;
      v[r][3] = b.y;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[r][c] = 0.f;
    }
  }
  if (signs != nullptr) {
    float sg[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) sg[c] = signs[4 * lane + c];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[r][c] *= sg[c];
      // spans 1 and 2, inside the lane
#pragma unroll
      for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if ((c & h) == 0) {
            const float a = v[r][c], b = v[r][c + h];
            v[r][c] = a + b;
            v[r][c + h] = a - b;
          }
        }
      }
      // spans 4 .. 64, across lanes
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float other = __shfl_xor_sync(0xffffffffu, v[r][c], m);
          v[r][c] = upper ? other - v[r][c] : v[r][c] + other;
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) v[r][c] *= kRsqrt128;
    }
  }
  float m = 0.f;
#pragma unroll
  for (int r = 0; r < kRows; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) m = fmaxf(m, fabsf(v[r][c]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[8];
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  float amax = wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, wmax[i]);
  const float s = scale_of(amax);
  if (threadIdx.x == 0) sc[(size_t)bh * nb + blk] = s;
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int row = row0 + r;  // < n_pad: the block lies inside the padded rows
    const uint32_t w = pack_e4m3x4(__fdiv_rn(v[r][0], s), __fdiv_rn(v[r][1], s), __fdiv_rn(v[r][2], s),
                                   __fdiv_rn(v[r][3], s));
    *reinterpret_cast<uint32_t*>(dst + ((size_t)bh * n_pad + row) * kD + 4 * lane) = w;
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

// V codes, transposed: one CTA per (128-key block, head); each warp takes 16
// keys, lane l the channels 4l..4l+3 of each.  Four keys' codes (one 32-bit
// word per key, a byte per channel) are byte-transposed into one word per
// channel, so each lane ends with 16 consecutive keys of each of its four
// channels: one 16-byte store per channel row of V^T, no shared memory.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_fp8_vt_kernel(const void* __restrict__ v,
                                                        const unsigned* __restrict__ vamax,
                                                        uint8_t* __restrict__ v8t, float* __restrict__ sv, int N,
                                                        int n_pad) {
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float s[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) s[c] = scale_of(__uint_as_float(vamax[(size_t)bh * kD + 4 * lane + c]));
  if (blk == 0 && warp == 0) {
#pragma unroll
    for (int c = 0; c < 4; ++c) sv[(size_t)bh * kD + 4 * lane + c] = s[c];
  }
  const int key0 = blk * 128 + warp * 16;
  uint32_t out[4][4];  // [channel c][group of four keys]
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t w[4];  // key key0 + 4g + i: codes of channels 4l..4l+3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int key = key0 + 4 * g + i;
      float f[4] = {0.f, 0.f, 0.f, 0.f};
      if (key < N) {
        const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(v) +
                                                        (((size_t)bh * N + key) * kD + 4 * lane) * 2);
        const float2 a = unpack16x2<BF16>(u.x), b = unpack16x2<BF16>(u.y);
        f[0] = a.x;
        f[1] = a.y;
        f[2] = b.x;
        f[3] = b.y;
      }
      w[i] = pack_e4m3x4(__fdiv_rn(f[0], s[0]), __fdiv_rn(f[1], s[1]), __fdiv_rn(f[2], s[2]),
                         __fdiv_rn(f[3], s[3]));
    }
    // 4 x 4 byte transpose: out[c][g] byte i = w[i] byte c
    const uint32_t t0 = __byte_perm(w[0], w[1], 0x5140), t1 = __byte_perm(w[2], w[3], 0x5140);
    const uint32_t t2 = __byte_perm(w[0], w[1], 0x7362), t3 = __byte_perm(w[2], w[3], 0x7362);
    out[0][g] = __byte_perm(t0, t1, 0x5410);
    out[1][g] = __byte_perm(t0, t1, 0x7632);
    out[2][g] = __byte_perm(t2, t3, 0x5410);
    out[3][g] = __byte_perm(t2, t3, 0x7632);
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(v8t + ((size_t)bh * kD + 4 * lane + c) * n_pad + key0) =
        make_uint4(out[c][0], out[c][1], out[c][2], out[c][3]);
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
    fa_fp8_rows_kernel<true><<<g_rows, 256, 0, st>>>(q, k, signs, b.q8, b.k8, b.sq, b.sk, N, n_pad, nb);
    fa_fp8_vamax_kernel<true><<<g_vamax, 256, 0, st>>>(v, b.vamax, N);
    fa_fp8_vt_kernel<true><<<g_vt, 256, 0, st>>>(v, b.vamax, b.v8t, b.sv, N, n_pad);
  } else {
    fa_fp8_rows_kernel<false><<<g_rows, 256, 0, st>>>(q, k, signs, b.q8, b.k8, b.sq, b.sk, N, n_pad, nb);
    fa_fp8_vamax_kernel<false><<<g_vamax, 256, 0, st>>>(v, b.vamax, N);
    fa_fp8_vt_kernel<false><<<g_vt, 256, 0, st>>>(v, b.vamax, b.v8t, b.sv, N, n_pad);
  }
  return cudaGetLastError();
}

}  // namespace fa
