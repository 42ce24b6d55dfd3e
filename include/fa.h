/*
 * fa.h -- C ABI of libfa.so: exact, IO-aware scaled-dot-product attention
 * (forward and backward) for NVIDIA B200 (sm_100a).
 *
 * What it computes.  For every batch b and head h, with S = scale * Q K^T
 * (entries with key j > query i set to -inf when `causal` is non-zero):
 *     LSE_i = ln sum_j exp(S_ij),   P = exp(S - LSE),   O = P V.
 * The N x N matrices S and P are never written to device memory: the forward
 * streams key/value tiles through on-chip memory with the online-softmax
 * recurrence and writes only O and the per-row log-sum-exp; the backward
 * recomputes P from Q, K and the stored LSE.  Sources (page title, section):
 *   - marketmaker.cc, "Flash Attention and the sequence-length problem":
 *     "Why attention is memory-bound" (the definition), "The Flash Attention
 *     algorithm" (tiling over query and key/value blocks), "Online softmax
 *     recurrence", "Backward pass: recompute instead of store", "Causal
 *     masking" (future tiles skipped), "Integration is eight lines" (the
 *     (batch, heads, seq, head_dim) layout and the is_causal flag);
 *   - ultralytics.com glossary "Flash Attention", "How Flash Attention works"
 *     (only the output and two numbers per row go back to HBM).
 * Results are exact in exact arithmetic, not bitwise: the fp32 accumulation
 * order and the rounding of P to the input type differ from a two-pass
 * evaluation (delect.ru glossary "FlashAttention", "What is confirmed").
 *
 * Layout.  q, k, v, o, dout, dq, dk, dv: [B, H, N, d] contiguous, row stride d
 * elements, element type given by `dtype`: FA_BF16 / FA_FP16 = all of them
 * bf16 / fp16; FA_BF16_O_F32 / FA_FP16_O_F32 = the same except that o (the
 * forward's output and the backward's input) is float32.  lse: [B, H, N]
 * contiguous float32, natural log.  Every pointer is a device pointer
 * aligned to 16 bytes.  Supported: d in {64, 128}; N >= 1 (any N: the last
 * tile may be ragged); B >= 1, H >= 1; B*H*N*d < 2^31.
 *
 * Ownership.  The caller allocates and owns every buffer.  The library never
 * allocates device memory and keeps no per-call state.  All calls are
 * asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 * stream).  Outputs are overwritten, never accumulated into.
 *
 * Errors.  Every entry point returns an fa_status.  Argument errors are
 * detected on the host before anything is launched.  A kernel whose internal
 * pipeline wait exceeds the wait limit (default 1000 ms, see
 * fa_debug_set_wait_limit_ms) abandons its work, records FA_ERR_TIMEOUT in a
 * device status word and returns; fa_last_device_status() reports it.
 * Nothing in the library traps or asserts on the device.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, size overflow */
  FA_ERR_UNSUPPORTED = 2, /* head dim other than 64/128, unknown dtype */
  FA_ERR_MISALIGNED = 3,  /* a pointer not 16-byte aligned */
  FA_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  FA_ERR_TIMEOUT = 5,     /* a kernel gave up on a pipeline wait */
  FA_ERR_WORKSPACE = 6,   /* workspace missing or smaller than required */
  FA_ERR_NO_DEVICE = 7    /* no sm_100 device is current */
} fa_status;

/*
 * Storage types.  With O stored in 16 bits, the backward's row term
 * D_i = sum_c dO_ic O_ic inherits O's rounding (2^-9 relative for bf16); on
 * sharply peaked softmax rows dP - D cancels and that rounding reaches dQ at
 * about 1e-2 relative.  The *_O_F32 codes keep O in float32 (the forward's
 * own accumulator, normalised) so that D carries only the forward's
 * arithmetic error; they cost 2 extra bytes per element of O traffic.
 * A caller that runs the backward (training) should store O this way: on
 * the one-trading-day workload (N = 23400, peaked rows) bf16 storage of O
 * alone puts dQ at 1.03e-2 - 1.16e-2 relative error, with every other step
 * exact, while float32 storage leaves about 2e-7.
 */
typedef enum { FA_BF16 = 0, FA_FP16 = 1, FA_BF16_O_F32 = 2, FA_FP16_O_F32 = 3 } fa_dtype;

/*
 * Forward: O = softmax(scale * Q K^T [causal]) V and LSE.
 *   q, k, v : inputs, [B,H,N,d], dtype.
 *   o       : output, [B,H,N,d], dtype's O type (16-bit: round-to-nearest-
 *             even of O; float32 for the *_O_F32 codes).
 *   lse     : output, [B,H,N] float32, LSE_i = ln sum_j exp(S_ij).
 *   scale   : score multiplier (1/sqrt(d) for standard attention).
 *   causal  : non-zero => key j attends to query i only if j <= i
 *             (top-left aligned; key blocks entirely in the future are
 *             skipped).
 * One kernel launch.  Source: marketmaker.cc "The Flash Attention
 * algorithm" and "Online softmax recurrence"; ultralytics.com glossary
 * "How Flash Attention works".
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, int dtype, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: a float32 dQ
 * accumulator of B*H*ceil(N/128)*128*d elements, then two float32 row
 * vectors of B*H*ceil(N/128)*128 elements (D_i = sum_c dO_ic O_ic, and
 * -LSE_i * log2(e)), each section rounded up to 256 bytes.  Returns 0 for
 * invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward: given dO = dL/dO, computes dQ, dK, dV by recomputing P from Q, K
 * and the forward's LSE (never storing P):
 *   D_i = sum_c dO_ic O_ic;  dV = P^T dO;  dP = dO V^T;  dS = P o (dP - D);
 *   dQ = scale dS K;  dK = scale dS^T Q.
 *   q, k, v, dout    : inputs, [B,H,N,d], dtype.
 *   o                : input, the forward's output in dtype's O type.
 *   lse              : input, [B,H,N] float32 from fa_fwd.
 *   dq, dk, dv       : outputs, [B,H,N,d], dtype.
 *   workspace        : device buffer of at least fa_bwd_workspace_size()
 *                      bytes, 256-byte aligned; contents on entry ignored.
 * Three kernel launches on `stream` (D and dQ-accumulator zeroing; dK/dV with
 * dQ accumulation; dQ conversion).  Source: marketmaker.cc "Backward pass:
 * recompute instead of store"; delect.ru glossary, the backward-recomputation
 * claim.  The gradient formulas are the softmax Jacobian (the pages do not
 * print them).
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
           float scale, int causal, int dtype, void* stream);

/*
 * Backward without caller-provided workspace, for callers that cannot
 * allocate device memory (for example an operator inside a framework whose
 * allocator owns every device allocation, or a host loop that must not call
 * cudaMalloc after start-up).  The pages have no counterpart: this is a
 * library convenience, not part of the method.
 *   Same arguments and results as fa_bwd, minus workspace/workspace_bytes.
 *   The scratch fa_bwd needs is taken from a fixed array of 32 MiB
 *   (33554432 bytes) inside the library's device memory, present on every GPU
 *   that loads the library until the process exits.  Problems whose
 *   fa_bwd_workspace_size exceeds it return FA_ERR_WORKSPACE before anything
 *   runs.  The call allocates nothing.
 *   Invalid arguments are reported (as by fa_bwd) without touching the
 *   array.  The first successful call on each device looks up the array's
 *   device address (with that device current) and keeps it; a lookup that
 *   fails returns FA_ERR_CUDA and is retried by the next call.  Make the
 *   first call on a device before any stream capture.
 *   All calls on a device share the array: calls that overlap on the GPU
 *   (other streams, other host threads) race and must be serialised by the
 *   caller.  The array keeps the last call's contents; fa_bwd rewrites every
 *   part of it that it reads, so no clearing is needed between calls.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                   int causal, int dtype, void* stream);

/*
 * Grouped-query attention (GQA / MQA): H query heads share Hkv key/value
 * heads; query head h reads key/value head h / (H / Hkv).  H must be a
 * multiple of Hkv (Hkv = 1: multi-query; Hkv = H: same as fa_fwd / fa_bwd).
 *   q, o, lse, dout, dq : [B, H, N, d] (lse [B, H, N]), as in fa_fwd / fa_bwd.
 *   k, v, dk, dv        : [B, Hkv, N, d]; dk, dv are the gradients summed over
 *                         the query heads of each group.
 *   workspace           : fa_bwd_workspace_size(B, H, N, d) bytes (per query head).
 * Everything else as fa_fwd / fa_bwd; Hkv <= 0 or H % Hkv != 0 returns
 * FA_ERR_INVALID_ARG.  The backward keeps each key/value head's dK and dV in
 * tensor memory while it walks every query head of its group.  Source:
 * delect.ru glossary "FlashAttention", "What is confirmed" (the attention
 * computation does not change the number of key/value heads, so grouping is
 * independent of it).
 */
int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
               int d, float scale, int causal, int dtype, void* stream);
int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int Hkv, int N,
               int d, float scale, int causal, int dtype, void* stream);

/*
 * Block-sparse attention: whole 128 x 128 (query block, key block) tiles are
 * skipped, never loaded nor computed, where the mask is 0 (on top of the
 * causal mask when `causal` is set).  This approximates full attention; it
 * equals it when every tile is kept.  Source: ultralytics.com glossary
 * "Flash Attention", "Flash Attention and related terms" (the block-sparse
 * variant skips empty tiles); delect.ru glossary "FlashAttention", "What is
 * confirmed" (described separately as an approximation).
 *   block_mask       : device uint8 [nb][nb] per query head, nb = ceil(N/128),
 *                      row = query block, column = key block, non-zero = keep;
 *                      head b*H + h starts at block_mask + (b*H + h) *
 *                      mask_head_stride (0 = one mask for every head).
 *   Other arguments as fa_fwd / fa_bwd.  A query row with no kept key gets
 *   O = 0, LSE = -inf and zero gradients; a key with no query attending it
 *   gets dK = dV = 0.  NULL mask or negative stride: FA_ERR_INVALID_ARG.
 */
int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                       const unsigned char* block_mask, long long mask_head_stride, int B, int H, int N, int d,
                       float scale, int causal, int dtype, void* stream);
int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, const unsigned char* block_mask, long long mask_head_stride, void* dq,
                       void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                       float scale, int causal, int dtype, void* stream);

/*
 * Ring attention (context parallelism) splits the sequence into one chunk per
 * device; each device keeps its query chunk and computes attention block by
 * block against the key/value chunks as they pass around a ring (ultralytics
 * glossary "Flash Attention", "Flash Attention and related terms", ring
 * attention).  The per-chunk attention is fa_fwd / fa_bwd on the chunk pair
 * (fp32-O dtype codes for the partial forward; the merged O and LSE for the
 * backward); the two calls below are the steps between chunks.  The ring
 * schedule and the exchange live in the Python package (exact_io_aware_84_b200.ring).
 *
 * fa_merge: (o, lse) <- the combination of two partial results of the same
 * rows over disjoint key sets:
 *   LSE = ln(e^{LSE_a} + e^{LSE_b}),  O = e^{LSE_a - LSE} O_a + e^{LSE_b - LSE} O_b
 * (the online-softmax recurrence of marketmaker.cc "Online softmax
 * recurrence", one whole chunk at a time).  Rows where both LSEs are -inf
 * give O = 0, LSE = -inf.
 *   o, o_part     : device fp32 [rows][d], 16-byte aligned; o updated in place
 *   lse, lse_part : device fp32 [rows]; lse updated in place
 *   out           : optional device [rows][d] 16-bit copy of the merged O
 *                   (8-byte aligned), written when out_dtype is FA_BF16 or
 *                   FA_FP16; out_dtype = -1 writes none (out may be NULL)
 *   rows          : number of rows (B*H*n for a [B,H,n,d] chunk); 0 is a no-op
 *   d             : 64 or 128
 * Errors: FA_ERR_INVALID_ARG (NULL pointer, rows < 0), FA_ERR_UNSUPPORTED (d,
 * out_dtype), FA_ERR_MISALIGNED, FA_ERR_CUDA (launch).
 *
 * fa_grad_accumulate: acc[i] += src[i] for i < n, src 16-bit (FA_BF16 or
 * FA_FP16), acc fp32; both device pointers 16-byte aligned.  Used to sum the
 * per-chunk gradients of the ring backward in fp32.  Errors as fa_merge.
 *
 * fa_convert: dst[i] = src[i] rounded to nearest even in the 16-bit type
 * dst_dtype (FA_BF16 or FA_FP16), i < n; src fp32 16-byte aligned, dst 8-byte
 * aligned.  Writes the ring's fp32 results (O, dQ, dK, dV) out in the input
 * type.  Errors as fa_merge.
 */
int fa_merge(float* o, float* lse, const float* o_part, const float* lse_part, void* out, int out_dtype,
             long long rows, int d, void* stream);
int fa_grad_accumulate(float* acc, const void* src, long long n, int src_dtype, void* stream);
int fa_convert(void* dst, const float* src, long long n, int dst_dtype, void* stream);

/*
 * FP8 forward with incoherent processing (head dim 128).  FP8 attention is
 * hurt by outliers; multiplying the vectors by a random orthogonal matrix
 * before the block-wise quantisation spreads an outlier over all coordinates
 * (marketmaker.cc "Flash Attention and the sequence-length problem", section
 * "FA3: Hopper mechanics", item 3).  Here:
 *   rotation  R = diag(signs) H / sqrt(128), H the Sylvester Hadamard matrix,
 *             applied to Q and K only ((Q R)(K R)^T = Q K^T); signs = NULL
 *             skips it (plain FP8);
 *   format    float8 e4m3, round to nearest even, saturating at +-448;
 *   scales    Q and K one per (head, 128-row block), V one per (head,
 *             channel): scale = amax / 448 (1 if amax = 0), code = e4m3(x / scale);
 *   products  S = Q8 K8^T and O = P8 V8 on the tensor cores in FP8 with fp32
 *             accumulation; S is dequantised through the exponent's factor,
 *             P rounded to e4m3 (l sums the unrounded P), O times V's channel
 *             scales in the epilogue.
 * This approximates attention; the error is that of the e4m3 rounding of Q,
 * K, V (after the rotation) and of P.
 *
 * fa_fwd_fp8_workspace_size(B, H, N, 128): bytes of the caller-owned scratch
 *   (0 for an unsupported d): Q8, K8 [B*H][n_pad][128] and V8^T
 *   [B*H][128][n_pad] e4m3 (n_pad = ceil(N/128)*128), then the fp32 scales
 *   sq, sk [B*H][ceil(N/128)] and sv [B*H][128], then [B*H][128] words of
 *   scratch; each part starts on a 256-byte boundary, in that order.
 * fa_fp8_quantize: only the preparation (rotation, scales, codes) into the
 *   workspace; exposed so that the codes can be checked.
 * fa_fwd_fp8: preparation + attention.  q, k, v: [B,H,N,128] 16-bit (dtype
 *   FA_BF16 / FA_FP16, or the _O_F32 codes for a float32 O); o, lse as in
 *   fa_fwd; signs: device float[128] of +-1 or NULL.  Errors: as fa_fwd, plus
 *   FA_ERR_UNSUPPORTED for d != 128 and FA_ERR_WORKSPACE for a missing or
 *   short workspace.
 */
size_t fa_fwd_fp8_workspace_size(int B, int H, int N, int d);
int fa_fp8_quantize(const void* q, const void* k, const void* v, const float* signs, void* workspace,
                    size_t workspace_bytes, int B, int H, int N, int d, int dtype, void* stream);
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, const float* signs,
               void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
               int dtype, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/*
 * Synchronises `stream`, then returns FA_ERR_TIMEOUT if any kernel of this
 * library on the current device gave up on a pipeline wait since the last
 * call (FA_OK otherwise), and clears that record.  Returns FA_ERR_CUDA if
 * the synchronisation itself fails.
 */
int fa_last_device_status(void* stream);

/*
 * Diagnostics.  fa_debug_set_wait_limit_ms sets the per-wait limit used by
 * later launches (process-wide; ms >= 1).  fa_debug_set_flags sets
 * process-wide debug flags: bit 0 makes the forward kernel, bit 1 the
 * backward's main kernel, withhold one pipeline arrival on its first tile,
 * so that its bounded waits run out and the launch ends with FA_ERR_TIMEOUT
 * (used by the timeout tests); 0 restores normal operation.  Both return FA_OK or FA_ERR_INVALID_ARG.
 */
int fa_debug_set_wait_limit_ms(int ms);
int fa_debug_set_flags(int flags);

/*
 * Diagnostics: kernel timing.  While set (non-NULL), every backward call
 * records `before_main` on its stream right before it launches its main
 * kernel (the dK/dV/dQ kernel) and `after_main` right after, so that the
 * elapsed time between the two events is that kernel's duration.  Both are
 * cudaEvent_t handles created by the caller with timing enabled; the caller
 * owns them and must clear the setting (NULL, NULL) before destroying them.
 * Process-wide; a recorded event changes the chaining of the backward's
 * launches (the main kernel then starts after the event, not overlapped with
 * the end of the preprocessing kernel).  Returns FA_OK.
 */
int fa_debug_set_timing_events(void* before_main, void* after_main);

/* Version string of the library build. */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
