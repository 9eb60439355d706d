/*
 * sage.h - C ABI of the B200 (sm_100a) SageAttention forward pass (libsage.so).
 *
 * The method ("SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
 * Acceleration", and the follow-up article on SageAttention2) computes attention
 * O = softmax(sm_scale * Q K^T) V with:
 *   1. smooth K: K <- K - mean(K), the mean per channel over the tokens of one head
 *      (「SageAttention：低比特量化Attention，实现推理加速」, section 技术方案, paragraph on smoothing K; softmax is
 *      unchanged because q.mean(K) is constant along a row);
 *   2. per-block INT8 quantization of Q and K with one fp32 scale per block
 *      (scale = amax/127), blocks of FlashAttention size: 128 Q tokens, 64 K tokens
 *      (same section, paragraph on per-block INT8 of Q, K);
 *   3. a fused FlashAttention-style pass: S = Q_i8 K_i8^T with INT32 accumulation,
 *      dequantized by q_scale*k_scale*sm_scale, online softmax over 128-key tiles, and
 *      P.V either in FP16 (SAGE_PV_FP16; same section, paragraph on the FP16 PV
 *      accumulator) or with P and V in FP8 E4M3 (SAGE_PV_FP8; "SageAttention2"
 *      article, 技术方案 items (3) and (4)), each tile's P.V summed into fp32 registers.
 *
 * Conventions for every entry point:
 *   - fp16 tensors are IEEE binary16, passed as `const void*`/`void*`.
 *   - Dense layout [B, H, N, d] row-major (the layout of the scaled_dot_product_attention
 *     call the method replaces). Packed varlen layout [T, H, d] with int32 cu_seqlens
 *     [nseq+1] ON THE DEVICE: sequence s owns tokens cu_seqlens[s] .. cu_seqlens[s+1]-1;
 *     every per-head quantity (K mean, blocks, causal mask, V scale) is per sequence.
 *   - Scales: q_scale [nseq, H, ceil(maxlen/128)], k_scale [nseq, H, ceil(maxlen/64)],
 *     k_mean and v_scale [nseq, H, d] (dense: nseq = B, maxlen = N).
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library never
 *     frees or retains them. Tensor pointers must be 16-byte aligned.
 *   - Head dim d is 64 or 128. sm_scale <= 0 selects 1/sqrt(d). causal is the square
 *     mask j <= i within each sequence.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - "Stream-ordered allocation": scratch taken with cudaMallocFromPoolAsync from a
 *     memory pool the library creates once per device and never trims (it keeps the
 *     largest working set it has seen), released with cudaFreeAsync on the same stream.
 *     Callers that must not allocate use the *_ws entry points or sage_attn_fwd_noalloc.
 *     Nothing synchronizes except sage_get_device_status().
 *   - Host-detectable argument errors return before anything is enqueued. Errors that
 *     only the device can see (a bounded wait that timed out, malformed cu_seqlens) set
 *     a device status word, read and cleared by sage_get_device_status(); the output is
 *     then undefined. No kernel traps or spins without bound.
 */
#ifndef SAGE_H
#define SAGE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAGE_API __attribute__((visibility("default")))
#else
#define SAGE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARG = 1,   /* bad size, null pointer, unknown mode */
    SAGE_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement (e.g. d) */
    SAGE_ERR_MISALIGNED = 3,    /* a tensor pointer is not 16-byte aligned */
    SAGE_ERR_WORKSPACE = 4,     /* workspace missing or smaller than sage_workspace_size() */
    SAGE_ERR_CUDA = 5,          /* a CUDA runtime call failed (see sage_last_cuda_error) */
    SAGE_ERR_TIMEOUT = 6,       /* device: a bounded wait inside a kernel gave up */
    SAGE_ERR_BAD_SEQLENS = 7    /* device: cu_seqlens not monotonic / out of range */
} sage_status_t;

enum { SAGE_PV_FP16 = 0, SAGE_PV_FP8 = 1 };

/*
 * Option flags, passed in the `smooth_k` argument of the fused entry points
 * (sage_attn_fwd, sage_attn_fwd_ws, sage_attn_varlen_fwd, sage_attn_fwd_noalloc and the
 * *_kv forms) and of the Q/K quantization entry points:
 *   SAGE_SMOOTH_K (1): step 1 above. 0 and 1 keep their plain boolean meaning.
 *   SAGE_SMOOTH_V (2): smooth V in FP8 mode (「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案,
 *     the paragraph after item (4)): V <- V - mean(V), the mean per channel over the
 *     tokens of one head (per sequence in varlen, summed in fp64 and rounded once to
 *     fp32), the E4M3 codes and per-channel scales taken of the smoothed V, and mean(V)
 *     added to every output row. Softmax rows sum to one, so the exact result is
 *     unchanged; the E4M3 range is no longer spent on a channel offset.
 *   SAGE_SMOOTH_Q (4): smooth Q ("SageAttention2" article, 技术方案 (1)): Q <- Q - mean(Q),
 *     the mean per channel over the query tokens of one head (fp64 sum, rounded once),
 *     and the vector-matrix product mean(Q) K^T (with K as it is quantized, i.e.
 *     smoothed) added back to every score row: comp[j] = sum_c mean(Q)[c] K'[j,c] in
 *     fp32, and the base-2 logit is (S q_scale k_scale + comp[j]) sm_scale log2(e). The
 *     compensation varies along a row, so the kernel takes the exact row max of the
 *     dequantized scores instead of the integer max; it costs some throughput.
 *   SAGE_QK_FINE (8): finer quantization groups ("SageAttention2" article, 技术方案 (2),
 *     which groups tokens by the threads that hold them in the tensor-core layout): here
 *     every query row is held by one thread, so Q gets one scale per token, and K one
 *     scale per 32 tokens (the tensor-memory load width). q_scale is then
 *     [nseq, H, maxlen_q] and k_scale [nseq, H, ceil(maxlen_k / 32)].
 * Other bits give SAGE_ERR_INVALID_ARG (sage_quant_qk, _ws and _varlen accept only
 * SAGE_SMOOTH_K and SAGE_QK_FINE; sage_quant_qk_kv also SAGE_SMOOTH_Q); SAGE_SMOOTH_V
 * with SAGE_PV_FP16 gives SAGE_ERR_UNSUPPORTED (fp16 V is not quantized, so there is
 * nothing to smooth for).
 */
enum { SAGE_SMOOTH_K = 1, SAGE_SMOOTH_V = 2, SAGE_SMOOTH_Q = 4, SAGE_QK_FINE = 8 };

/* Opaque CUDA stream (binary-compatible with cudaStream_t). */
typedef struct CUstream_st *sage_stream_t;

/*
 * Bytes of scratch the fused entry points need for one call: INT8 codes of Q and K,
 * their block scales, the K mean (and its fp64 column sums), and in FP8 mode the E4M3
 * codes of V with their per-channel scales and the V column statistics (sum, max,
 * min) smooth V needs. Dense: nseq = B, max_seqlen = N, total_tokens = B*N. The size
 * does not depend on the smoothing flags.
 */
SAGE_API size_t sage_workspace_size(int nseq, int H, int max_seqlen, int total_tokens, int d,
                           int pv_mode);

/* sage_workspace_size for the dense layout: the scratch sage_attn_fwd_ws needs for
 * [B,H,N,d] inputs (= sage_workspace_size(B, H, N, B*N, d, pv_mode); 0 for a negative
 * size, or when B*N overflows int). */
SAGE_API size_t sage_attn_workspace_size(int B, int H, int N, int d, int pv_mode);

/* sage_workspace_size for queries and keys of different lengths (the *_kv entry points):
 * max_seqlen_q / total_q for Q and the output, max_seqlen_k / total_k for K and V. */
SAGE_API size_t sage_workspace_size_kv(int nseq, int H, int max_seqlen_q, int max_seqlen_k,
                                       int total_q, int total_k, int d, int pv_mode);

/*
 * Steps 1-2 on their own (dense): k_mean[b,h,c] = mean over tokens of K[b,h,:,c]
 * (zeros when smooth_k == 0), q_i8/q_scale = per-128-token INT8 of Q, k_i8/k_scale =
 * per-64-token INT8 of fp32(K) - k_mean. The K-mean sum is accumulated in fp64 (exact
 * for |K| N < 2^29) and rounded once to fp32; codes are round-half-even of the fp32
 * quotient x/scale clamped to [-127, 127]; an all-zero block has scale 0 and codes 0.
 * Outputs are caller-owned device buffers of the shapes in the conventions above.
 * Uses a small stream-ordered allocation for the fp64 sums.
 */
SAGE_API sage_status_t sage_quant_qk(const void *q, const void *k, int8_t *q_i8, float *q_scale,
                            int8_t *k_i8, float *k_scale, float *k_mean, int B, int H, int N,
                            int d, int smooth_k, sage_stream_t stream);

/* sage_quant_qk with caller-owned scratch for the fp64 K column sums: at least
 * B*H*d*8 bytes, 16-byte aligned (unused when smooth_k == 0). Allocates nothing. */
SAGE_API sage_status_t sage_quant_qk_ws(const void *q, const void *k, int8_t *q_i8,
                                        float *q_scale, int8_t *k_i8, float *k_scale,
                                        float *k_mean, int B, int H, int N, int d, int smooth_k,
                                        void *workspace, size_t ws_bytes, sage_stream_t stream);

/* sage_quant_qk for the packed varlen layout (cu_seqlens on the device; NULL reads the
 * buffers as dense [nseq, H, max_seqlen, d]). */
SAGE_API sage_status_t sage_quant_qk_varlen(const void *q, const void *k, const int32_t *cu_seqlens,
                                   int nseq, int total_tokens, int max_seqlen, int H, int d,
                                   int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                                   float *k_mean, int smooth_k, sage_stream_t stream);

/* Steps 1-2 in general form: Q [B,H,Nq,d] and K [B,H,Nk,d] (Nq may differ from Nk; the
 * K mean is taken over the Nk keys), flags = SAGE_SMOOTH_K | SAGE_SMOOTH_Q |
 * SAGE_QK_FINE. Scales: q_scale [B,H,ceil(Nq/128)] and k_scale [B,H,ceil(Nk/64)], or
 * with SAGE_QK_FINE [B,H,Nq] and [B,H,ceil(Nk/32)]. With SAGE_SMOOTH_Q the Q codes are
 * those of Q - q_mean, q_mean [B,H,d] and the score compensation q_comp
 * [B,H,ceil(Nk/128)*128] (entries past Nk are 0) are written; otherwise both may be
 * NULL. workspace: NULL (a stream-ordered allocation for the fp64 column sums) or caller
 * scratch of at least B*H*d*8 bytes (B*H*d*16 with SAGE_SMOOTH_Q), 16-byte aligned. */
SAGE_API sage_status_t sage_quant_qk_kv(const void *q, const void *k, int8_t *q_i8,
                                        float *q_scale, int8_t *k_i8, float *k_scale,
                                        float *k_mean, float *q_mean, float *q_comp, int B,
                                        int H, int Nq, int Nk, int d, int flags,
                                        void *workspace, size_t ws_bytes, sage_stream_t stream);

/*
 * V to FP8 E4M3 (「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案 (4)) with one fp32 scale per
 * channel over all tokens of a head: v_scale = amax/448, v_e4m3 = round-to-nearest-even
 * saturating E4M3 of the fp32 quotient V/v_scale (same [B,H,N,d] layout, one byte each).
 */
SAGE_API sage_status_t sage_quant_v_fp8(const void *v, uint8_t *v_e4m3, float *v_scale, int B, int H,
                               int N, int d, sage_stream_t stream);
SAGE_API sage_status_t sage_quant_v_fp8_varlen(const void *v, const int32_t *cu_seqlens, int nseq,
                                      int total_tokens, int max_seqlen, int H, int d,
                                      uint8_t *v_e4m3, float *v_scale, sage_stream_t stream);

/* sage_quant_v_fp8 (v_mean == NULL) or sage_quant_v_fp8_smooth (v_mean != NULL) with
 * caller-owned scratch for the column statistics: at least B*H*d*16 bytes, 16-byte
 * aligned. Allocates nothing. */
SAGE_API sage_status_t sage_quant_v_fp8_ws(const void *v, uint8_t *v_e4m3, float *v_scale,
                                           float *v_mean, int B, int H, int N, int d,
                                           void *workspace, size_t ws_bytes,
                                           sage_stream_t stream);

/*
 * Smooth V, then V to E4M3 (the SAGE_SMOOTH_V step on its own): v_mean [B,H,d] fp32 =
 * mean over tokens of V[b,h,:,c] (fp64 sum, rounded once); x = fp32(V) - v_mean (one
 * fp32 subtraction); v_scale = amax|x|/448 per channel; v_e4m3 = E4M3 of fp32 x/v_scale
 * as in sage_quant_v_fp8. A channel with x all zero (a constant channel) has scale 0
 * and codes 0. Uses a small stream-ordered allocation for the column statistics.
 */
SAGE_API sage_status_t sage_quant_v_fp8_smooth(const void *v, uint8_t *v_e4m3, float *v_scale,
                                               float *v_mean, int B, int H, int N, int d,
                                               sage_stream_t stream);
SAGE_API sage_status_t sage_quant_v_fp8_smooth_varlen(const void *v, const int32_t *cu_seqlens,
                                                      int nseq, int total_tokens,
                                                      int max_seqlen, int H, int d,
                                                      uint8_t *v_e4m3, float *v_scale,
                                                      float *v_mean, sage_stream_t stream);

/*
 * The whole forward pass (steps 1-3), dense layout: out[B,H,N,d] fp16. pv_mode selects
 * SAGE_PV_FP16 or SAGE_PV_FP8. Scratch comes from stream-ordered allocation on `stream`.
 */
SAGE_API sage_status_t sage_attn_fwd(const void *q, const void *k, const void *v, void *out, int B,
                            int H, int N, int d, int causal, int smooth_k, int pv_mode,
                            float sm_scale, sage_stream_t stream);

/* sage_attn_fwd with caller-owned scratch of at least sage_workspace_size() bytes
 * (256-byte aligned); allocates nothing. */
SAGE_API sage_status_t sage_attn_fwd_ws(const void *q, const void *k, const void *v, void *out, int B,
                               int H, int N, int d, int causal, int smooth_k, int pv_mode,
                               float sm_scale, void *workspace, size_t ws_bytes,
                               sage_stream_t stream);

/*
 * The whole forward pass on packed sequences: q, k, v, out are [total_tokens, H, d];
 * cu_seqlens is int32 [nseq+1] on the device with cu_seqlens[0] = 0 and
 * cu_seqlens[nseq] = total_tokens; max_seqlen (host) must bound every length (it sizes
 * the grid, so no device-to-host copy is made). workspace may be NULL (stream-ordered
 * allocation) or caller-owned scratch of sage_workspace_size() bytes.
 */
SAGE_API sage_status_t sage_attn_varlen_fwd(const void *q, const void *k, const void *v, void *out,
                                   const int32_t *cu_seqlens, int nseq, int total_tokens,
                                   int max_seqlen, int H, int d, int causal, int smooth_k,
                                   int pv_mode, float sm_scale, void *workspace,
                                   size_t ws_bytes, sage_stream_t stream);

/*
 * Queries and keys of different lengths (dense): q and out are [B,H,Nq,d], k and v are
 * [B,H,Nk,d], e.g. the last Nq tokens of a sequence attending to all Nk = past + Nq of
 * its keys (prefill against cached keys; Nq = 1 is a decode step). With causal, query i
 * sees keys j <= i + (Nk - Nq): the mask is aligned at the bottom-right corner and is
 * the square mask when Nq = Nk. A query that sees no key (only if Nq > Nk) gets a zero
 * output row, and Nk = 0 gives a zero output. workspace may be NULL (stream-ordered
 * allocation) or caller scratch of sage_workspace_size_kv(B, H, Nq, Nk, B*Nq, B*Nk, d,
 * pv_mode) bytes, 256-byte aligned. The pages only recommend the causal mode for the
 * decoding stage of language models (「如何将SageAttention量化注意力机制集成到你的AI项目中获得2-5倍速度提升」, section
 * 语言模型推理加速); queries fewer than keys and the bottom-right alignment are the
 * usual reading of that use.
 */
SAGE_API sage_status_t sage_attn_fwd_kv(const void *q, const void *k, const void *v, void *out,
                                        int B, int H, int Nq, int Nk, int d, int causal,
                                        int smooth_k, int pv_mode, float sm_scale,
                                        void *workspace, size_t ws_bytes, sage_stream_t stream);

/* sage_attn_fwd_kv on packed sequences: q/out [total_q,H,d] with cu_seqlens_q, k/v
 * [total_k,H,d] with cu_seqlens_k (both int32 [nseq+1] on the device); sequence s has
 * cu_seqlens_q[s+1]-cu_seqlens_q[s] queries and cu_seqlens_k[s+1]-cu_seqlens_k[s] keys,
 * bounded by max_seqlen_q and max_seqlen_k. */
SAGE_API sage_status_t sage_attn_varlen_fwd_kv(const void *q, const void *k, const void *v,
                                               void *out, const int32_t *cu_seqlens_q,
                                               const int32_t *cu_seqlens_k, int nseq,
                                               int total_q, int total_k, int max_seqlen_q,
                                               int max_seqlen_k, int H, int d, int causal,
                                               int smooth_k, int pv_mode, float sm_scale,
                                               void *workspace, size_t ws_bytes,
                                               sage_stream_t stream);

/*
 * Step 3 alone on pre-quantized operands (dense): q_i8/q_scale and k_i8/k_scale as
 * produced by sage_quant_qk; v is fp16 V (SAGE_PV_FP16, v_scale ignored) or E4M3 codes
 * with per-channel v_scale (SAGE_PV_FP8). Allocates nothing.
 */
SAGE_API sage_status_t sage_attn_fwd_quantized(const int8_t *q_i8, const float *q_scale,
                                      const int8_t *k_i8, const float *k_scale, const void *v,
                                      const float *v_scale, void *out, int B, int H, int N,
                                      int d, int causal, int pv_mode, float sm_scale,
                                      sage_stream_t stream);

/* Step 3 alone in FP8 mode with smoothed V: v_e4m3, v_scale and v_mean [B,H,d] as
 * produced by sage_quant_v_fp8_smooth; out = O v_scale / (448 l) + v_mean per channel.
 * Allocates nothing. */
SAGE_API sage_status_t sage_attn_fwd_quantized_smooth_v(const int8_t *q_i8, const float *q_scale,
                                                        const int8_t *k_i8, const float *k_scale,
                                                        const uint8_t *v_e4m3,
                                                        const float *v_scale, const float *v_mean,
                                                        void *out, int B, int H, int N, int d,
                                                        int causal, float sm_scale,
                                                        sage_stream_t stream);

/* Step 3 alone with Nq queries and Nk keys (codes and scales from sage_quant_qk_kv; V
 * codes from sage_quant_v_fp8[_smooth] with N = Nk); v_mean selects the smooth-V
 * epilogue (FP8 only) or is NULL; q_comp (16-byte aligned) is the smooth-Q compensation
 * of sage_quant_qk_kv or NULL; flags is 0 or SAGE_QK_FINE (the scale layout the codes
 * were made with). */
SAGE_API sage_status_t sage_attn_fwd_quantized_kv(const int8_t *q_i8, const float *q_scale,
                                                  const int8_t *k_i8, const float *k_scale,
                                                  const void *v, const float *v_scale,
                                                  const float *v_mean, const float *q_comp,
                                                  void *out, int B, int H, int Nq, int Nk, int d,
                                                  int causal, int pv_mode, float sm_scale,
                                                  int flags, sage_stream_t stream);

/*
 * Decode: steps 2-3 for a few queries (1 <= Nq <= SAGE_DECODE_MAX_Q) against many keys,
 * FP16 P.V mode, dense layout: q_i8 [B,H,Nq,d], k_i8 [B,H,Nk,d] and the scales as
 * produced by sage_quant_qk_kv (flags 0: q_scale [B,H,1], k_scale [B,H,ceil(Nk/64)];
 * flags SAGE_QK_FINE: q_scale [B,H,Nq], k_scale [B,H,ceil(Nk/32)]), v fp16 [B,H,Nk,d],
 * out fp16 [B,H,Nq,d]. The method is that of sage_attn_fwd_quantized_kv
 * (「SageAttention：低比特量化Attention，实现推理加速」, 技术方案: INT8 scores dequantized by
 * the two scales, online softmax, FP16 P times FP16 V): causal masks bottom-right (query
 * i sees keys j <= i + Nk - Nq; the decode step of 「如何将SageAttention量化注意力机制集成到
 * 你的AI项目中获得2-5倍速度提升」, 语言模型推理加速). The keys are split over many CTAs and
 * the splits' partial softmax results merged, so P is taken relative to each split's
 * maximum; the result agrees with the tile walk of sage_attn_fwd_quantized_kv to FP16
 * rounding. A query that sees no key is written as zeros.
 *
 * workspace: device memory of at least sage_attn_decode_workspace_size(B, H, Nq, Nk, d)
 * bytes, 16-byte aligned, owned by the caller (nothing is allocated). Returns
 * SAGE_ERR_UNSUPPORTED for Nq > SAGE_DECODE_MAX_Q, SAGE_ERR_WORKSPACE for a short
 * workspace, SAGE_ERR_INVALID_ARG / SAGE_ERR_MISALIGNED as the other entry points;
 * every check happens before anything is enqueued. sm_scale <= 0 means 1/sqrt(d).
 */
#define SAGE_DECODE_MAX_Q 16
SAGE_API size_t sage_attn_decode_workspace_size(int B, int H, int Nq, int Nk, int d);
SAGE_API sage_status_t sage_attn_decode_quantized(const int8_t *q_i8, const float *q_scale,
                                                  const int8_t *k_i8, const float *k_scale,
                                                  const void *v, void *out, int B, int H,
                                                  int Nq, int Nk, int d, int causal,
                                                  float sm_scale, int flags, void *workspace,
                                                  size_t ws_bytes, sage_stream_t stream);

/*
 * Debug: the integer score tiles S = q_i8 k_i8^T (int32, [B,H,N,N]) exactly as the
 * attention kernel's tensor-core pass produces them, dumped from tensor memory. Meant
 * for small N (the output is N^2 per head). Uses stream-ordered scratch for a dummy
 * pass over V.
 */
SAGE_API sage_status_t sage_debug_qk_int32(const int8_t *q_i8, const int8_t *k_i8, int32_t *s_out,
                                  int B, int H, int N, int d, sage_stream_t stream);

/*
 * sage_attn_fwd without any allocation, for callers that cannot allocate device memory
 * while they run (for instance a serving process whose own allocator owns all GPU
 * memory after start-up, or a latency-critical loop that must not risk an allocation
 * stalling or failing) and have no scratch buffer to pass to sage_attn_fwd_ws. The
 * paper has no counterpart; this is an interface convenience of this library.
 *
 * Scratch comes from a static device array of SAGE_NOALLOC_SCRATCH_BYTES (64 MiB) that
 * every GPU which loads this library holds until the process exits. A call whose
 * sage_workspace_size(B, H, N, B*N, d, pv_mode) exceeds that returns SAGE_ERR_WORKSPACE
 * before anything is enqueued (set SAGE_LOG=1 for the byte counts). Arguments, layout
 * and results are those of sage_attn_fwd.
 *
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current) and caches it; make that first call before any stream
 * capture. All calls share the one array and it keeps the previous call's contents (the
 * parts that must start at zero are cleared on every call): calls that can overlap on
 * the GPU, on different streams of one device, race and must be serialized by the caller.
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define SAGE_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
SAGE_API sage_status_t sage_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                             void *out, int B, int H, int N, int d, int causal,
                                             int smooth_k, int pv_mode, float sm_scale,
                                             sage_stream_t stream);

/*
 * Debug: exercises the bounded-wait path every kernel uses. One thread waits on a
 * barrier that nothing arrives on; after timeout_ns (1 us .. 1 s) the wait gives up,
 * SAGE_ERR_TIMEOUT is recorded in the device status word and the kernel returns, so the
 * context stays usable. Read the result with sage_get_device_status().
 */
SAGE_API sage_status_t sage_debug_wait_timeout(unsigned long long timeout_ns,
                                               sage_stream_t stream);

/* Synchronizes `stream`, returns the device status word (SAGE_OK if clean) and clears
 * it. SAGE_ERR_CUDA if the synchronization itself failed. */
SAGE_API sage_status_t sage_get_device_status(sage_stream_t stream);

/* Human-readable name of a status code (static storage). */
SAGE_API const char *sage_status_string(sage_status_t status);

/* cudaError_t value of the last failed CUDA runtime call made by this library. */
SAGE_API int sage_last_cuda_error(void);

/* ABI version (major*100 + minor). */
SAGE_API int sage_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_H */
