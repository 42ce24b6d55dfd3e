// Parameter blocks and launch entry points shared by the C-ABI front end
// (fa_api.cu) and the kernel translation units.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

namespace fa {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream is finishing, so that its launch
// and prologue (barrier setup, tensor-memory allocation) overlap that tail.
// Every kernel launched this way executes griddepcontrol.wait before its
// first access to global memory, which returns once the previous grid has
// completed and its writes are visible.
template <typename... Params, typename... Args>
inline cudaError_t launch_chained(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

constexpr int kBlockM = 128;  // query rows per Q tile (tcgen05 M)
constexpr int kBlockN = 128;  // keys per K/V tile

struct FwdParams {
  void* o;             // [B*H, N, D] 16-bit, or fp32 when the O32 variant runs
  float* lse;          // [B*H, N] fp32
  int N;               // sequence length
  int bh;              // B*H (query heads)
  int H;               // query heads per batch entry
  int group;           // query heads per key/value head (H / Hkv)
  int n_kv;            // ceil(N / 128): key/value tiles per head
  int n_pairs;         // ceil(N / 256): pairs of 128-row Q tiles per head
  int n_units;         // bh * n_pairs
  float scale_log2;    // scale * log2(e)
  uint64_t wait_limit_ns;
  int* status;         // device status word
  int debug_flags;
  // Block sparsity (nullptr = dense): uint8 [n_kv][n_kv] tile mask per query
  // head, head h at bmask + h * bmask_stride (stride 0 = one mask for all).
  const uint8_t* bmask;
  long long bmask_stride;
  // FP8 variant only (d = 128): dequantisation scales, e4m3 codes in the
  // tensor maps.  Q: [B*H][n_kv] per 128-row block; K: [B*Hkv][n_kv];
  // V: [B*Hkv][128] per channel.
  const float* fp8_sq;
  const float* fp8_sk;
  const float* fp8_sv;
};

// Device buffers of the FP8 forward's quantised operands (see fa_fp8.cu).
struct Fp8Buffers {
  uint8_t* q8;     // [B*H][n_pad][128] e4m3
  uint8_t* k8;     // [B*H][n_pad][128] e4m3
  uint8_t* v8t;    // [B*H][128][n_pad] e4m3 (transposed)
  float* sq;       // [B*H][n_kv]
  float* sk;       // [B*H][n_kv]
  float* sv;       // [B*H][128]
  unsigned* vamax; // [B*H][128] scratch: channel maxima (float bits)
};

struct BwdParams {
  const void* o;       // forward output, [B*H, N, D] (16-bit, or fp32 for O32)
  // q, o, dout, dq are [B*H, N, D]; k, v, dk, dv are [B*Hkv, N, D]
  const void* dout;    // dO, [B*H, N, D]
  const float* lse;    // [B*H, N]
  void* dq;            // [B*H, N, D]
  void* dk;            // [B*H, N, D]
  void* dv;            // [B*H, N, D]
  float* dq_acc;       // [B*H, n_pad, D] fp32 workspace
  float* dvec;         // [B*H, n_pad] fp32 workspace (D_i)
  float* nlse2;        // [B*H, n_pad] fp32 workspace (-LSE_i * log2 e; -inf on padding)
  int N;
  int n_pad;           // ceil(N / 128) * 128
  int bh;              // B*H (query heads)
  int group;           // query heads per key/value head (H / Hkv)
  int n_kv;            // ceil(N / 128)
  int n_units;         // B * Hkv * n_kv
  float scale;         // softmax scale
  float scale_log2;    // scale * log2(e)
  uint64_t wait_limit_ns;
  int* status;         // device status word
  int debug_flags;     // bit 1: withhold one arrival (timeout test)
  const uint8_t* bmask;  // block sparsity as in FwdParams (nullptr = dense)
  long long bmask_stride;
};

// The k-th work unit of this CTA in a persistent kernel: consecutive rounds
// of gridDim.x units, taken in alternating directions (CTA c gets c, then
// 2G-1-c, then 2G+c, ...).  Causal units are numbered longest first, so a CTA
// that drew a long unit in one round draws a short one in the next; with a
// plain round-robin the same CTAs would draw the longest unit of every round.
__device__ __forceinline__ int unit_of(int k) {
  const int g = (int)gridDim.x, c = (int)blockIdx.x;
  return k * g + ((k & 1) ? g - 1 - c : c);
}

// Launchers (return cudaError_t of the launch).
cudaError_t launch_fwd(int d, bool bf16, bool o32, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const FwdParams& p, int grid, cudaStream_t st);
// FP8 forward (d = 128): e4m3 Q, K (K-major) and V^T tensor maps; `bf16`
// selects the output type.
cudaError_t launch_fwd_fp8(bool bf16, bool o32, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tvt, const FwdParams& p, int grid, cudaStream_t st);
cudaError_t launch_fp8_prep(bool bf16, const void* q, const void* k, const void* v, const float* signs,
                            const Fp8Buffers& b, int bh, int N, cudaStream_t st);
int fwd_fp8_smem();

// ev_main[0] / ev_main[1] (may be null): events recorded on `st` right
// before and right after the launch of the main backward kernel.
cudaError_t launch_bwd(int d, bool bf16, bool o32, bool causal, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const CUtensorMap& tdo, const BwdParams& p, int grid,
                       cudaStream_t st, cudaEvent_t const* ev_main);

// Ring-attention helpers (fa_ring.cu).  out_kind: 0 none, 1 bf16, 2 fp16.
cudaError_t launch_merge(int d, int out_kind, float* o, float* lse, const float* o_part, const float* lse_part,
                         void* out, long long rows, int sms, cudaStream_t st);
cudaError_t launch_accumulate(bool bf16, float* acc, const void* src, long long n, int sms, cudaStream_t st);
cudaError_t launch_convert(bool bf16, void* dst, const float* src, long long n, int sms, cudaStream_t st);

int fwd_threads();
int bwd_threads();

}  // namespace fa
