/*
 * sage_attn.h -- C ABI of the B200 (sm_100a) SageAttention-style 8-bit attention library.
 *
 * The operation follows "SageAttention: Accurate 8-Bit Attention for Plug-and-play
 * Inference Acceleration" (research.elamur.ai summary page):
 *   O = softmax(Q K^T * sm_scale) V, where
 *   - K is first smoothed by subtracting its per-channel mean over tokens
 *     (Summary, first bullet; Interesting idea I1: a component shared by all tokens of K
 *     can be removed without changing the softmax);
 *   - Q and K are quantized to INT8 with absmax scales (Summary, first bullet;
 *     Key points: per-token granularity), here per token or per block of tokens;
 *   - Q K^T runs as an INT8 matrix product with INT32 accumulation and is dequantized by
 *     scale_q * scale_k * sm_scale;
 *   - softmax runs online over key/value tiles, FlashAttention-style (Summary: the kernels
 *     follow FlashAttention-style tiling);
 *   - P V runs on 16-bit floating-point operands (Summary, second bullet), P rounded to fp16.
 *
 * Conventions shared by every entry point
 *   - Tensors are device memory owned by the caller, dense and contiguous in the order
 *     [B][H][N][d] ("BHND").  Q, K, V and O are IEEE fp16.  q8/k8 are int8 with the same
 *     layout.  km is fp32 [B][H][d].  Scales are fp32 [B][H][G] with
 *     G = sage_scale_count(N, granularity, is_q).
 *   - granularity SAGE_PER_TOKEN: one scale per token (G = N);
 *     SAGE_PER_BLOCK: one scale per 128 consecutive Q tokens / 64 consecutive K tokens
 *     (groups start at token 0 of each (b,h); the last group holds the remaining tokens).
 *   - d must be 64 or 128; N >= 1 (any value; sage_debug_qk_int32 alone needs a multiple of
 *     128); B, H >= 1;
 *     B*H*N*d must stay below 2^31.  sm_scale must be finite and > 0.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Calls only enqueue work:
 *     they never synchronize the host.  Arguments are validated before anything is
 *     enqueued; an invalid call returns an error and launches nothing.
 *   - Return value: SAGE_OK (0) or a negative sage_status.  A kernel whose bounded
 *     internal wait gave up leaves a code readable with sage_last_device_error().
 *   - Inputs must not alias outputs.  Non-finite inputs give unspecified (but bounded,
 *     non-faulting) results.
 */
#ifndef SAGE_ATTN_H
#define SAGE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID = -1,     /* null pointer, bad size, bad sm_scale, bad granularity */
  SAGE_ERR_UNSUPPORTED = -2, /* valid request outside what the kernels implement (d, N) */
  SAGE_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
  SAGE_ERR_TIMEOUT = -4,     /* a kernel's bounded wait gave up (sage_last_device_error) */
  SAGE_ERR_NOMEM = -5,       /* workspace allocation failed */
  SAGE_ERR_TOO_LARGE = -6    /* problem needs more than the fixed no-alloc scratch */
} sage_status;

enum { SAGE_PER_TOKEN = 0, SAGE_PER_BLOCK = 1 };

/* Human-readable name of a status code (static string, never NULL). */
const char* sage_status_string(int status);

/* Number of scales per (b,h): N for per-token; ceil(N/128) for Q and ceil(N/64) for K
 * per-block.  Returns 0 for an unknown granularity or N <= 0. */
size_t sage_scale_count(int N, int granularity, int is_q);

/* K smoothing (Summary, first bullet; idea I1).
 * km[b,h,c] = mean over the N tokens of K[b,h,:,c], computed from the exact sum
 * (fixed point, order independent) as fl32(fl32(sum) / N).
 * k: fp16 [B,H,N,d] (in); km: fp32 [B,H,d] (out). */
int sage_smooth_k(const void* k, float* km, int B, int H, int N, int d, void* stream);

/* INT8 quantization of Q and K (Summary, first bullet; Key points: per-token).
 * For every group (one token, or 128 Q / 64 K consecutive tokens, all d channels):
 *   x = Q, or x = fl32(K - km) when km != NULL (no smoothing when km == NULL);
 *   a = max|x|; scale = fl32(a/127); code = clamp(round_half_even(fl32(x * fl32(127/a))), +-127)
 *   (a == 0: scale 0, codes 0).
 * q, k: fp16 [B,H,N,d] (in); km: fp32 [B,H,d] or NULL (in);
 * q8, k8: int8 [B,H,N,d] (out); sq: fp32 [B,H,Gq], sk: fp32 [B,H,Gk] (out). */
int sage_quant_qk(const void* q, const void* k, const float* km, int8_t* q8, int8_t* k8, float* sq,
                  float* sk, int B, int H, int N, int d, int granularity, void* stream);

/* sage_smooth_k followed by sage_quant_qk (with the mean) in ONE launch and one pass over the
 * tokens of each head (K smoothing fused with the quantization): one cluster
 * of CTAs per head sums K exactly over its token slices and shares the sums through distributed
 * shared memory, then quantizes the slices' K groups (K minus the mean) and Q groups.  Outputs,
 * bit for bit, those of the two calls: km fp32 [B,H,d]; q8, k8 int8 [B,H,N,d]; sq, sk fp32 scales
 * of the granularity.  q, k: fp16 [B,H,N,d] (in). */
int sage_prep_qk(const void* q, const void* k, float* km, int8_t* q8, int8_t* k8, float* sq, float* sk, int B, int H,
                 int N, int d, int granularity, void* stream);

/* The whole forward pass as a user calls it: smooth K, quantize Q and K, fused attention.
 * q, k, v: fp16 [B,H,N,d] (in); o: fp16 [B,H,N,d] (out).  causal: keys j > i masked
 * (top-left aligned).  Workspace (int8 Q/K, scales, km: 2*B*H*N*d bytes plus scales) is
 * allocated and freed stream-ordered inside the call, from a memory pool the library owns
 * (one per device) that keeps freed memory reserved for the next call: the largest workspace
 * used so far stays reserved until the process exits. */
int sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                  int causal, float sm_scale, int granularity, void* stream);

/* The fused attention kernel alone, on already-quantized inputs (Summary bullets 1-2):
 * S = (q8 k8^T) * sq * sk * sm_scale with INT32 accumulation on the tensor cores, online
 * softmax in fp32 with exp2, P rounded to fp16, O = P V with fp16 operands and fp32
 * accumulation, O stored as fp16.  q8, k8: int8 [B,H,N,d]; sq, sk: fp32 scales of the
 * given granularity; v: fp16 [B,H,N,d] (in); o: fp16 [B,H,N,d] (out). */
int sage_attn_fwd_quantized(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk,
                            const void* v, void* o, int B, int H, int N, int d, int causal,
                            float sm_scale, int granularity, void* stream);

/* ---------------------------------------------------------------------------------------
 * FP8 P.V variant, following the SageAttention2 abstract (author pages of Jia Wei and Haofeng
 * Huang): the matrices (P~, V) are quantized to FP8, V is smoothed, and P~V is
 * accumulated in an FP32 buffer.  Q.K^T stays the INT8 product above (the abstract's INT4 Q.K^T
 * is not part of this variant).  FP8 is E4M3 (bias 7, largest finite 448), round to nearest
 * even, saturating.  Head dimension 128 only (d = 64 returns SAGE_ERR_UNSUPPORTED).
 *
 * V to FP8, per (b,h) and channel c: vm = channel mean over the N tokens (exact sum, as the K
 * mean) when vm != NULL, else 0; x = fl32(V - vm); a = max_t |x|; sv = fl32(a/448);
 * v8 = e4m3(fl32(x * fl32(448/a))) (a == 0: sv = 0, codes 0).  One scale per channel: it is
 * constant along the P.V contraction (the tokens).
 * v: fp16 [B,H,N,d] (in); v8: E4M3 codes [B,H,N,d] (out); sv: fp32 [B,H,d] (out);
 * vm: fp32 [B,H,d] (out) or NULL (no smoothing). */
int sage_quant_v_fp8(const void* v, uint8_t* v8, float* sv, float* vm, int B, int H, int N, int d, void* stream);

/* The fused kernel of the FP8 P.V variant on quantized inputs: S and the online softmax as in
 * sage_attn_fwd_quantized, except that the row offsets are integers in log2 units and
 * P~ = e4m3(2^(s*log2(e) - offset + 8)) (the row's largest weight near 2^8, every weight rounded on
 * the E4M3 grid of a power-of-two scaling of exp(s - max s)); O^T += V8^T . P~^T on tcgen05
 * kind::f8f6f4 with fp32 accumulation in tensor memory; O = acc / l * sv + vm stored as fp16.
 * The row sum l uses the unrounded weights.  q8, k8, sq, sk as for sage_attn_fwd_quantized;
 * v8, sv, vm from sage_quant_v_fp8 (vm may be NULL); o: fp16 [B,H,N,d] (out). */
int sage_attn_fwd_fp8pv_quantized(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk,
                                  const uint8_t* v8, const float* sv, const float* vm, void* o, int B, int H, int N,
                                  int d, int causal, float sm_scale, int granularity, void* stream);

/* The whole FP8 P.V variant as a user calls it: smooth K, INT8 Q and K, V to FP8 with
 * smoothing, the fused kernel above.  Arguments, validation and workspace as sage_attn_fwd (the
 * workspace also holds the E4M3 V: 3*B*H*N*d bytes plus scales and means). */
int sage_attn_fwd_fp8pv(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                        int causal, float sm_scale, int granularity, void* stream);

/* ---------------------------------------------------------------------------------------
 * Block-sparse variant, following the SpargeAttn abstract (author pages of Jia Wei and Haofeng
 * Huang): a sparse and quantized attention with a two-stage online filter.
 * Stage 1 predicts the attention map at block level and skips the products of the blocks it
 * drops; stage 2, inside the online softmax, skips the P.V product (and the exp2 work) of a block
 * whose scores all lie far below the running row maximum.  Head dimension 64 or 128 and
 * N <= 65536 (SAGE_ERR_UNSUPPORTED otherwise); P.V in fp16 as in sage_attn_fwd.
 *
 * Stage 1 (sage_sparse_predict): query blocks of 256 tokens (QB = ceil(N/256) per (b,h)) and key
 * blocks of 128 tokens (KB = ceil(N/128)).  Each block is represented by the mean of its tokens;
 * the predicted map of a query block is softmax_j(q_mean . k_mean_j * sm_scale) over the key
 * blocks it may see (causal: those starting at or before its last query).  Kept: the fewest key
 * blocks, in decreasing predicted probability (ties: lower index first), whose probabilities sum
 * to at least tau (0 < tau <= 1); every visible key block when the query block's self-
 * similarity (the mean cosine over ordered pairs of its tokens) is below theta; every key block
 * whose self-similarity is below theta; causal: the blocks holding the query block's own keys.
 * q, k: fp16 [B,H,N,d] (in); kv_count: int [B,H,QB] (out, the number of kept key blocks);
 * kv_index: int16 [B,H,QB,KB] (out, the kept key blocks in increasing order, entries past the
 * count left unchanged).  Allocates a small stream-ordered workspace (block means). */
int sage_sparse_predict(const void* q, const void* k, int B, int H, int N, int d, int causal, float sm_scale,
                        float tau, float theta, int* kv_count, int16_t* kv_index, void* stream);

/* The fused kernel of the block-sparse variant on quantized inputs: as sage_attn_fwd_quantized
 * over the kept key blocks of kv_count / kv_index (any ascending lists; causal lists must hold
 * the blocks with each query's own key), plus stage 2: a query tile of 128 rows drops key block
 * j when, for each of its rows below N, the block's largest score (log2 units) lies more than
 * skip_lambda below the row's largest score over the blocks it visited before (its first block
 * is never dropped).  skip_lambda > 0; +INFINITY turns stage 2 off.  A query block whose count
 * is 0 (or whose list lacks the blocks its causal rows need) gets unspecified output; counts
 * and entries out of range are clamped, so no access ever leaves the tensors. */
int sage_attn_fwd_sparse_quantized(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk,
                                   const void* v, void* o, int B, int H, int N, int d, int causal, float sm_scale,
                                   int granularity, const int* kv_count, const int16_t* kv_index, float skip_lambda,
                                   void* stream);

/* The whole block-sparse variant as a user calls it: stage-1 prediction, smooth K, INT8 Q and K,
 * the fused kernel with stage 2.  Workspace as sage_attn_fwd plus the block lists. */
int sage_attn_fwd_sparse(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                         int causal, float sm_scale, int granularity, float tau, float theta, float skip_lambda,
                         void* stream);

/* ---------------------------------------------------------------------------------------
 * Microscaling FP4 variant, following the SageAttention3 abstract (author pages of Jia Wei and
 * Haofeng Huang): both products of the attention run on Blackwell's FP4 tensor
 * cores (tcgen05 kind::mxf4nvf4, block16) with microscaling.  Head dimension d = 64 or 128.
 * Formats: E2M1 codes (0, 0.5, 1, 1.5, 2, 3, 4, 6 and their
 * negatives), two per byte with the even element in the low nibble; one UE4M3 scale per 16
 * elements along the contraction dimension, e4m3(fl32(max|z| / 6)), codes
 * e2m1(fl32(z * fl32(1 / scale))); scales stored as the tensor cores' scale atoms: for every 128
 * rows and 64 elements of the contraction, 512 bytes with row r's four scales at byte
 * (r % 32) * 16 + (r / 32) * 4.  A second, fp32 scale lifts the range: per 128-token tile of Q
 * and of smoothed K, g = fl32(a / 2688) with a = the tile's largest |x|, z = fl32(x * fl32(2688 /
 * a)); per channel of smoothed V the same over all tokens.  P~ = 2^(u - m + 10) in the online
 * softmax's integer frame m (the ceil of the running row maximum, log2 units), microscaled along
 * the keys; the row sum uses P~ before rounding.  tiles = ceil(N/128); A = d / 64, the scale
 * atoms per row group of Q and K (one per 64 channels). */

/* Q and K (minus km, the channel means of sage_smooth_k, when km is not null) to FP4.
 * q, k: fp16 [B,H,N,d] (in); q4, k4: uint8 [B,H,N,d/2] (out, codes); sfq: uint8
 * [B,H,tiles,A,512] (out, scale atoms of Q, the 128 tokens of a tile as rows); sfk: uint8
 * [B,H,ceil(N/64),A,512] (out, scale atoms of K, the 64 tokens of each half tile as the first 64
 * rows, the other rows zero); rows past N get zero scales; gq, gk: fp32 [B,H,tiles] (out, tile
 * scales).  No workspace. */
int sage_quant_qk_fp4(const void* q, const void* k, const float* km, uint8_t* q4, uint8_t* sfq, float* gq,
                      uint8_t* k4, uint8_t* sfk, float* gk, int B, int H, int N, int d, void* stream);

/* V to FP4 along the tokens (the P.V contraction), smoothed by its exact channel mean when vm is
 * not null.  v: fp16 [B,H,N,d] (in); v4t: uint8 [B,H,d,tiles*64] (out, codes transposed:
 * row c holds channel c's codes of keys 0 .. tiles*128-1, keys past N zero); sfv: uint8
 * [B,H,tiles,2,512] (out, scale atoms of keys 0-63 and 64-127 of a tile with the channels as
 * rows; d = 64: rows 64-127 zero); gv: fp32 [B,H,d] (out, channel scales); vm: fp32 [B,H,d] (out,
 * channel means) or null.  Allocates a small stream-ordered
 * workspace (the inverse channel scales). */
int sage_quant_v_fp4(const void* v, uint8_t* v4t, uint8_t* sfv, float* gv, float* vm, int B, int H, int N, int d,
                     void* stream);

/* The fused FP4 kernel on quantized inputs (layouts above; vm may be null).  o: fp16
 * [B,H,N,d] (out).  All pointers 16-byte aligned.  No workspace. */
int sage_attn_fwd_fp4_quantized(const uint8_t* q4, const uint8_t* sfq, const float* gq, const uint8_t* k4,
                                const uint8_t* sfk, const float* gk, const uint8_t* v4t, const uint8_t* sfv,
                                const float* gv, const float* vm, void* o, int B, int H, int N, int d, int causal,
                                float sm_scale, void* stream);

/* The whole FP4 variant as a user calls it: smooth K, Q and K to FP4, V to FP4 (smoothed), the
 * fused kernel.  Allocates its workspace stream-ordered. */
int sage_attn_fwd_fp4(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, int causal,
                      float sm_scale, void* stream);

/* Debug: the full integer product s[b,h,i,j] = sum_c q8[b,h,i,c] * k8[b,h,j,c] as int32
 * (exact: |s| <= 128*127*127 < 2^31), computed with the same tensor-core path as the fused
 * kernel.  s: int32 [B,H,N,N] (out); needs B*H*N*N < 2^31. */
int sage_debug_qk_int32(const int8_t* q8, const int8_t* k8, int32_t* s, int B, int H, int N, int d,
                        void* stream);

/* Debug / tracing: sage_attn_fwd_quantized (per-block granularity and N a multiple of 128
 * only, else SAGE_ERR_UNSUPPORTED) built with SM clock
 * stamps (clock64) of its pipeline events, for the first trace_ctas CTAs.  Output equals the
 * untraced kernel's.  trace: int64 [trace_ctas][2 + 10*T] with T = ceil(N/128) key tiles, zeroed by
 * the caller; per CTA: [0] start, [1] end, then for key tile j:
 *   [2 + (3t+e)*T + j]   softmax warpgroup of query tile t (0/1), event e: 0 = S ready,
 *                        1 = row max and offset done, 2 = P~ written and signalled;
 *   [2 + (6+2t+e)*T + j] MMA thread, tile t, event e: 0 = P.V issued, 1 = next Q.K^T issued.
 * Slots of events that do not happen (causal tiles, a missing second query tile) stay 0.
 * CTA c works on head c / ceil(N/256) and query tiles 2p, 2p+1 with p = ceil(N/256)-1 - c % ceil(N/256). */
int sage_debug_attn_trace(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk,
                          const void* v, void* o, int B, int H, int N, int d, int causal,
                          float sm_scale, int granularity, long long* trace, int trace_ctas,
                          void* stream);

/* Debug / measurement: the dense tensor-core rate of this GPU per MMA kind, for the roofline's
 * denominators (not an operation of the pages).  Launches `ctas` CTAs (use the SM count: one per
 * SM); in each, two warps issue `iters` (a multiple of 8, 8 .. 2^24) back-to-back tcgen05 MMAs of
 * shape M=128, N=256 with loop-invariant operands (zero-filled shared memory) into their own
 * accumulators.  kind 0 = kind::i8 (K = 32), 1 = kind::f16 (K = 16), 2 = kind::f8f6f4 with E4M3
 * operands (K = 32); every instruction is 128*256*K multiply-accumulates.  cycles: int64 [ctas]
 * device memory, receives each CTA's SM cycles from its first issue to the completion of both
 * warps' products.  status: device int (caller-zeroed), set to 1 if a bounded wait gave up.
 * SAGE_ERR_INVALID for a bad kind, iters or pointer; SAGE_ERR_CUDA if the launch failed. */
int sage_debug_mma_peak(int kind, int iters, int ctas, long long* cycles, int* status, void* stream);

/* Debug / failure detection: launches one warp that waits on an mbarrier nothing ever arrives
 * on, with the same bounded wait (about 0.5 s of SM clocks) that every pipeline role of the
 * attention kernels uses.  The wait gives up, records status 1 for sage_last_device_error()
 * and the kernel returns: no trap, no fault, the context stays usable.  gave_up: device int,
 * written 0 when the wait gave up (1 would mean it completed).  Returns SAGE_ERR_INVALID for a
 * null pointer, SAGE_ERR_CUDA if the launch failed.  (Not an operation of the pages: a check of
 * the library's own failure detection.) */
int sage_debug_wait_timeout(int* gave_up, void* stream);

/* Waits for all work on stream, then returns and clears the device status word written by
 * kernels whose bounded waits gave up (0 = none; 1 = an mbarrier wait timed out; 2, from
 * sage_debug_attn_trace only: a CTA barrier let a thread through before every thread had
 * arrived).  Returns
 * SAGE_ERR_CUDA (negative) if the synchronization itself failed. */
int sage_last_device_error(void* stream);

/* ---------------------------------------------------------------------------------------
 * Allocation-free variant of sage_attn_fwd.  The SageAttention page has no counterpart of
 * this entry point: it exists for callers that cannot allocate device memory while they
 * run -- hosts whose device-memory budget is fixed at start-up (embedded and real-time
 * services), and plugins of frameworks that own every device allocation themselves and
 * forbid a library from calling the CUDA allocator -- and so cannot use the stream-ordered
 * workspace of sage_attn_fwd.
 *
 * Same arguments, results and validation as sage_attn_fwd (bit-identical output), but the
 * workspace (INT8 Q/K, scales, K mean) lives in a scratch array compiled into the library:
 * SAGE_NOALLOC_SCRATCH_BYTES of device memory that every GPU which loads the library holds
 * until the process exits.  The call allocates nothing (no cudaMalloc / cudaFree, no
 * library allocator).  Problems whose workspace, sage_noalloc_scratch_bytes(), exceeds the
 * scratch size return SAGE_ERR_TOO_LARGE without launching anything.
 *
 * The first call on each device looks up the scratch array's device address with
 * cudaGetSymbolAddress (with that device current) and caches it; make that first call
 * before any stream capture.  All calls share the one scratch array and nothing in it needs
 * clearing (every value is rewritten before it is read), but two calls whose work overlaps
 * on the GPU (different streams, or different host threads on one device) race on it:
 * serialize them on one stream. */
#define SAGE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* Scratch bytes a problem needs: 2*B*H*N*d (INT8 Q, K) plus the scales and the K mean,
 * each rounded up to 256 bytes.  0 for invalid sizes or granularity. */
size_t sage_noalloc_scratch_bytes(int B, int H, int N, int d, int granularity);

int sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                          int causal, float sm_scale, int granularity, void* stream);

/* The whole forward pass with Q, K, V and O in HOST memory: the host->device copies of the
 * inputs and the device->host copy of O overlap the compute.  (Not an operation of the
 * pages: a serving convenience built from the three steps above.)
 *
 * The B*H heads are processed in chunks of heads_per_chunk consecutive heads (0 = automatic,
 * about sixteen chunks).  For chunk c, its slice of Q, K, V is copied in on an internal
 * stream, the three steps run on `stream`, and its slice of O is copied out on a second
 * internal stream, while chunk c+1 is copied in and chunk c-1 copied out; events order every
 * reuse of the two sets of device buffers.  The output is bit-identical to sage_attn_fwd on
 * the same tensors (every head is an independent problem and runs the same kernels).
 *
 * q, k, v: fp16 [B][H][N][d] host memory, read; o: fp16 [B][H][N][d] host memory, written.
 * Any host allocation works; page-locked memory (cudaMallocHost / cudaHostRegister) is
 * needed for the copies to overlap.  The caller keeps all four buffers alive and unchanged
 * (o unread) until `stream` has passed the call: like every entry point here, the call only
 * enqueues work (with pageable memory the runtime may block the host during a copy).  The
 * device workspace (2 x chunk slices of Q, K, V, O plus INT8 copies and scales) is
 * allocated and freed stream-ordered on `stream`.  Same size, scale and granularity rules
 * and statuses as sage_attn_fwd; heads_per_chunk < 0 gives SAGE_ERR_INVALID; a failed
 * workspace allocation SAGE_ERR_NOMEM. */
int sage_attn_fwd_host(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                       int causal, float sm_scale, int granularity, int heads_per_chunk, void* stream);

/* Variants for sage_attn_fwd_host_variant. */
enum { SAGE_VARIANT_FP16PV = 0, SAGE_VARIANT_FP8PV = 1, SAGE_VARIANT_FP4 = 2 };

/* sage_attn_fwd_host for the method or one of its variants: each chunk of heads runs
 * sage_attn_fwd (SAGE_VARIANT_FP16PV, identical to sage_attn_fwd_host), sage_attn_fwd_fp8pv
 * (SAGE_VARIANT_FP8PV, d = 128) or sage_attn_fwd_fp4 (SAGE_VARIANT_FP4, d = 64 or 128;
 * granularity must still be a valid value and is not used) on its device copies.  The output
 * is bit-identical to that entry point on the whole tensors.  An unknown variant gives
 * SAGE_ERR_INVALID, SAGE_VARIANT_FP8PV with d = 64 SAGE_ERR_UNSUPPORTED, both before any copy
 * is enqueued; otherwise as sage_attn_fwd_host. */
int sage_attn_fwd_host_variant(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                               int causal, float sm_scale, int granularity, int heads_per_chunk, int variant,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_ATTN_H */
