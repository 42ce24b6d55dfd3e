// C-ABI front end of libfa.so: argument checks, TMA descriptor encoding and
// kernel dispatch.  See include/fa.h for the contract of every entry point.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "fa.h"
#include "fa_kernels.h"
#include "sm100_ptx.cuh"

namespace fa {

// Host-side NVTX range around each entry point (visible in timeline
// profilers; a no-op when none is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Device status word: 0 = OK, else the fa_status of a kernel that gave up.
__device__ int g_device_status = 0;

namespace {

int* status_ptr() {
  int* ptr = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_device_status) != cudaSuccess) return nullptr;
  return ptr;
}

std::atomic<int> g_wait_limit_ms{1000};
std::atomic<int> g_debug_flags{0};
// Events recorded around the backward's main kernel (fa_debug_set_timing_events).
std::atomic<void*> g_ev_main_before{nullptr};
std::atomic<void*> g_ev_main_after{nullptr};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [bh, n, d] 16-bit tensor, tile box = 64 columns x `rows` rows, 128-byte
// swizzle; rows past n (and columns past d) read as zero.
int encode_tile_map(CUtensorMap* m, const void* ptr, int bh, int n, int d, bool bf16, int rows) {
  auto fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

struct DeviceInfo {
  int sms = 0;
  bool sm100 = false;
};

int device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  static DeviceInfo cache[64];
  static std::once_flag flags[64];
  if (dev < 0 || dev >= 64) return FA_ERR_NO_DEVICE;
  std::call_once(flags[dev], [dev] {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cache[dev].sms = sms;
    cache[dev].sm100 = (major == 10 && minor == 0);
  });
  *out = cache[dev];
  return out->sm100 ? FA_OK : FA_ERR_NO_DEVICE;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 8-bit [outer][rows][inner] tensor, box = 128 inner x 128 rows, 128-byte
// swizzle (the FP8 operands: inner = 128 bytes of a row).
int encode_u8_map(CUtensorMap* m, const void* ptr, int outer, int rows, int inner) {
  auto fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)inner, (cuuint64_t)rows * inner};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Layout of the FP8 forward's workspace (each part 256-byte aligned).
struct Fp8Layout {
  size_t q8, k8, v8t, sq, sk, sv, vamax, total;
};
Fp8Layout fp8_layout(int B, int H, int N) {
  const size_t bh = (size_t)B * H;
  const size_t nb = ((size_t)N + 127) / 128, n_pad = nb * 128;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  Fp8Layout l;
  l.q8 = 0;
  l.k8 = l.q8 + up(bh * n_pad * 128);
  l.v8t = l.k8 + up(bh * n_pad * 128);
  l.sq = l.v8t + up(bh * n_pad * 128);
  l.sk = l.sq + up(bh * nb * 4);
  l.sv = l.sk + up(bh * nb * 4);
  l.vamax = l.sv + up(bh * 128 * 4);
  l.total = l.vamax + up(bh * 128 * 4);
  return l;
}

Fp8Buffers fp8_buffers(void* ws, int B, int H, int N) {
  const Fp8Layout l = fp8_layout(B, H, N);
  uint8_t* b = static_cast<uint8_t*>(ws);
  Fp8Buffers f;
  f.q8 = b + l.q8;
  f.k8 = b + l.k8;
  f.v8t = b + l.v8t;
  f.sq = reinterpret_cast<float*>(b + l.sq);
  f.sk = reinterpret_cast<float*>(b + l.sk);
  f.sv = reinterpret_cast<float*>(b + l.sv);
  f.vamax = reinterpret_cast<unsigned*>(b + l.vamax);
  return f;
}

int check_common(int B, int H, int N, int d, float scale, int dtype) {
  if (B <= 0 || H <= 0 || N <= 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale > 3.0e38f) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (dtype != FA_BF16 && dtype != FA_FP16 && dtype != FA_BF16_O_F32 && dtype != FA_FP16_O_F32)
    return FA_ERR_UNSUPPORTED;
  const long long total = (long long)B * H * ((long long)N + 255) * d;
  if (total >= (1ll << 31)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

uint64_t wait_limit_ns() { return (uint64_t)g_wait_limit_ms.load() * 1000000ull; }

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_version(void) { return "fa-sm100 0.1"; }

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_NO_DEVICE: return "FA_ERR_NO_DEVICE";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_debug_set_wait_limit_ms(int ms) {
  if (ms < 1) return FA_ERR_INVALID_ARG;
  g_wait_limit_ms.store(ms);
  return FA_OK;
}

int fa_debug_set_flags(int flags) {
  if (flags < 0) return FA_ERR_INVALID_ARG;
  g_debug_flags.store(flags);
  return FA_OK;
}

int fa_debug_set_timing_events(void* before_main, void* after_main) {
  g_ev_main_before.store(before_main);
  g_ev_main_after.store(after_main);
  return FA_OK;
}

int fa_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  return v;
}

static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                    int N, int d, float scale, int causal, int dtype, void* stream,
                    const unsigned char* bmask = nullptr, long long bmask_stride = 0) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (bmask_stride < 0) return FA_ERR_INVALID_ARG;
  int st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  if (Hkv <= 0 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((st = device_info(&di)) != FA_OK) return st;
  const bool bf16 = dtype == FA_BF16 || dtype == FA_BF16_O_F32;
  const bool o32 = dtype == FA_BF16_O_F32 || dtype == FA_FP16_O_F32;
  const int bh = B * H;
  CUtensorMap tq, tk, tv;
  if (encode_tile_map(&tq, q, bh, N, d, bf16, kBlockM) != FA_OK ||
      encode_tile_map(&tk, k, B * Hkv, N, d, bf16, kBlockN) != FA_OK ||
      encode_tile_map(&tv, v, B * Hkv, N, d, bf16, kBlockN) != FA_OK)
    return FA_ERR_CUDA;
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.N = N;
  p.bh = bh;
  p.H = H;
  p.group = H / Hkv;
  p.n_kv = (N + kBlockN - 1) / kBlockN;
  p.n_pairs = (N + 2 * kBlockM - 1) / (2 * kBlockM);
  p.n_units = bh * p.n_pairs;
  p.scale_log2 = scale * kLog2e;
  p.wait_limit_ns = wait_limit_ns();
  p.debug_flags = g_debug_flags.load();
  p.bmask = bmask;
  p.bmask_stride = bmask_stride;
  if (!(p.status = status_ptr())) return FA_ERR_CUDA;
  const int grid = p.n_units < di.sms ? p.n_units : di.sms;
  cudaError_t e = launch_fwd(d, bf16, o32, causal != 0, tq, tk, tv, p, grid, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, int dtype, void* stream) {
  NvtxRange nvtx_range("fa_fwd");
  return fwd_impl(q, k, v, o, lse, B, H, H, N, d, scale, causal, dtype, stream);
}

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
               int d, float scale, int causal, int dtype, void* stream) {
  NvtxRange nvtx_range("fa_fwd_gqa");
  return fwd_impl(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, dtype, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.0f, FA_BF16) != FA_OK) return 0;
  const size_t n_pad = ((size_t)N + kBlockN - 1) / kBlockN * kBlockN;
  const size_t bh = (size_t)B * H;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  return up(bh * n_pad * d * sizeof(float)) + 2 * up(bh * n_pad * sizeof(float));
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                    int H, int Hkv, int N, int d, float scale, int causal, int dtype, void* stream,
                    const unsigned char* bmask = nullptr, long long bmask_stride = 0) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (bmask_stride < 0) return FA_ERR_INVALID_ARG;
  int st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  if (Hkv <= 0 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  if ((st = device_info(&di)) != FA_OK) return st;
  const bool bf16 = dtype == FA_BF16 || dtype == FA_BF16_O_F32;
  const bool o32 = dtype == FA_BF16_O_F32 || dtype == FA_FP16_O_F32;
  const int bh = B * H;
  BwdParams p{};
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.N = N;
  p.n_kv = (N + kBlockN - 1) / kBlockN;
  p.n_pad = p.n_kv * kBlockN;
  p.bh = bh;
  p.group = H / Hkv;
  p.n_units = B * Hkv * p.n_kv;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.wait_limit_ns = wait_limit_ns();
  p.debug_flags = g_debug_flags.load();
  p.bmask = bmask;
  p.bmask_stride = bmask_stride;
  if (!(p.status = status_ptr())) return FA_ERR_CUDA;
  const size_t acc_bytes = ((size_t)bh * p.n_pad * d * sizeof(float) + 255) / 256 * 256;
  const size_t vec_bytes = ((size_t)bh * p.n_pad * sizeof(float) + 255) / 256 * 256;
  p.dq_acc = static_cast<float*>(workspace);
  p.dvec = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + acc_bytes);
  p.nlse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + acc_bytes + vec_bytes);
  CUtensorMap tq, tk, tv, tdo;
  const int q_rows = (d == 64) ? 128 : 64;  // backward query tile (see fa_bwd_sm100.cu)
  if (encode_tile_map(&tq, q, bh, N, d, bf16, q_rows) != FA_OK ||
      encode_tile_map(&tk, k, B * Hkv, N, d, bf16, kBlockN) != FA_OK ||
      encode_tile_map(&tv, v, B * Hkv, N, d, bf16, kBlockN) != FA_OK ||
      encode_tile_map(&tdo, dout, bh, N, d, bf16, q_rows) != FA_OK)
    return FA_ERR_CUDA;
  const int grid = p.n_units < di.sms ? p.n_units : di.sms;
  const cudaEvent_t ev_main[2] = {static_cast<cudaEvent_t>(g_ev_main_before.load()),
                                  static_cast<cudaEvent_t>(g_ev_main_after.load())};
  cudaError_t e = launch_bwd(d, bf16, o32, causal != 0, tq, tk, tv, tdo, p, grid, static_cast<cudaStream_t>(stream),
                             ev_main);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
           float scale, int causal, int dtype, void* stream) {
  NvtxRange nvtx_range("fa_bwd");
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, H, N, d, scale, causal,
                  dtype, stream);
}

int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int Hkv, int N,
               int d, float scale, int causal, int dtype, void* stream) {
  NvtxRange nvtx_range("fa_bwd_gqa");
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, N, d, scale, causal,
                  dtype, stream);
}

int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                       const unsigned char* block_mask, long long mask_head_stride, int B, int H, int N, int d,
                       float scale, int causal, int dtype, void* stream) {
  NvtxRange nvtx_range("fa_fwd_blocksparse");
  if (!block_mask) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, B, H, H, N, d, scale, causal, dtype, stream, block_mask, mask_head_stride);
}

int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, const unsigned char* block_mask, long long mask_head_stride, void* dq,
                       void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                       float scale, int causal, int dtype, void* stream) {
  NvtxRange nvtx_range("fa_bwd_blocksparse");
  if (!block_mask) return FA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, H, N, d, scale, causal,
                  dtype, stream, block_mask, mask_head_stride);
}

size_t fa_fwd_fp8_workspace_size(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.0f, FA_BF16) != FA_OK || d != 128) return 0;
  return fp8_layout(B, H, N).total;
}

static int fp8_prep(const void* q, const void* k, const void* v, const float* signs, void* workspace,
                    size_t workspace_bytes, int B, int H, int N, int d, int dtype, void* stream) {
  if (!q || !k || !v) return FA_ERR_INVALID_ARG;
  int st = check_common(B, H, N, d, 1.0f, dtype);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(workspace)) return FA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < fp8_layout(B, H, N).total) return FA_ERR_WORKSPACE;
  DeviceInfo di;
  if ((st = device_info(&di)) != FA_OK) return st;
  const bool bf16 = dtype == FA_BF16 || dtype == FA_BF16_O_F32;
  cudaError_t e = launch_fp8_prep(bf16, q, k, v, signs, fp8_buffers(workspace, B, H, N), B * H, N,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fp8_quantize(const void* q, const void* k, const void* v, const float* signs, void* workspace,
                    size_t workspace_bytes, int B, int H, int N, int d, int dtype, void* stream) {
  NvtxRange nvtx_range("fa_fp8_quantize");
  return fp8_prep(q, k, v, signs, workspace, workspace_bytes, B, H, N, d, dtype, stream);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, const float* signs,
               void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
               int dtype, void* stream) {
  NvtxRange nvtx_range("fa_fwd_fp8");
  if (!o || !lse) return FA_ERR_INVALID_ARG;
  int st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  if ((st = fp8_prep(q, k, v, signs, workspace, workspace_bytes, B, H, N, d, dtype, stream)) != FA_OK) return st;
  DeviceInfo di;
  if ((st = device_info(&di)) != FA_OK) return st;
  const bool bf16 = dtype == FA_BF16 || dtype == FA_BF16_O_F32;
  const bool o32 = dtype == FA_BF16_O_F32 || dtype == FA_FP16_O_F32;
  const int bh = B * H;
  const int n_pad = (N + 127) / 128 * 128;
  const Fp8Buffers fb = fp8_buffers(workspace, B, H, N);
  CUtensorMap tq, tk, tvt;
  if (encode_u8_map(&tq, fb.q8, bh, n_pad, 128) != FA_OK || encode_u8_map(&tk, fb.k8, bh, n_pad, 128) != FA_OK ||
      encode_u8_map(&tvt, fb.v8t, bh, 128, n_pad) != FA_OK)
    return FA_ERR_CUDA;
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.N = N;
  p.bh = bh;
  p.H = H;
  p.group = 1;
  p.n_kv = (N + kBlockN - 1) / kBlockN;
  p.n_pairs = (N + 2 * kBlockM - 1) / (2 * kBlockM);
  p.n_units = bh * p.n_pairs;
  p.scale_log2 = scale * kLog2e;
  p.wait_limit_ns = wait_limit_ns();
  p.debug_flags = g_debug_flags.load();
  p.fp8_sq = fb.sq;
  p.fp8_sk = fb.sk;
  p.fp8_sv = fb.sv;
  if (!(p.status = status_ptr())) return FA_ERR_CUDA;
  const int grid = p.n_units < di.sms ? p.n_units : di.sms;
  cudaError_t e = launch_fwd_fp8(bf16, o32, causal != 0, tq, tk, tvt, p, grid, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_merge(float* o, float* lse, const float* o_part, const float* lse_part, void* out, int out_dtype,
             long long rows, int d, void* stream) {
  NvtxRange nvtx_range("fa_merge");
  if (rows < 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (out_dtype < -1 || out_dtype > FA_FP16) return FA_ERR_UNSUPPORTED;
  if (rows == 0) return FA_OK;
  if (!o || !lse || !o_part || !lse_part || (out_dtype >= 0 && !out)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(o_part)) % 16 != 0 ||
      (out_dtype >= 0 && reinterpret_cast<uintptr_t>(out) % 8 != 0))
    return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int st;
  if ((st = device_info(&di)) != FA_OK) return st;
  const int kind = out_dtype < 0 ? 0 : (out_dtype == FA_BF16 ? 1 : 2);
  cudaError_t e = launch_merge(d, kind, o, lse, o_part, lse_part, out_dtype < 0 ? nullptr : out, rows, di.sms,
                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_grad_accumulate(float* acc, const void* src, long long n, int src_dtype, void* stream) {
  NvtxRange nvtx_range("fa_grad_accumulate");
  if (n < 0) return FA_ERR_INVALID_ARG;
  if (src_dtype != FA_BF16 && src_dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
  if (n == 0) return FA_OK;
  if (!acc || !src) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(acc) | reinterpret_cast<uintptr_t>(src)) % 16 != 0) return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int st;
  if ((st = device_info(&di)) != FA_OK) return st;
  cudaError_t e = launch_accumulate(src_dtype == FA_BF16, acc, src, n, di.sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_convert(void* dst, const float* src, long long n, int dst_dtype, void* stream) {
  NvtxRange nvtx_range("fa_convert");
  if (n < 0) return FA_ERR_INVALID_ARG;
  if (dst_dtype != FA_BF16 && dst_dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
  if (n == 0) return FA_OK;
  if (!dst || !src) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(src) % 16 != 0 || reinterpret_cast<uintptr_t>(dst) % 8 != 0)
    return FA_ERR_MISALIGNED;
  DeviceInfo di;
  int st;
  if ((st = device_info(&di)) != FA_OK) return st;
  cudaError_t e = launch_convert(dst_dtype == FA_BF16, dst, src, n, di.sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
