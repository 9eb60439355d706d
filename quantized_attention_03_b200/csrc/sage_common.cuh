// Shared definitions of the CUDA library: sequence layouts, status codes, launch helpers.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/sage.h"

namespace sage {

constexpr int kQBlock = 128;   // Q tokens per INT8 scale block (= the attention Q tile)
constexpr int kKBlock = 64;    // K tokens per INT8 scale block
constexpr int kKvTile = 128;   // keys per attention KV tile (two K blocks)

// Where the tokens of one (sequence, head) live. Dense [B,H,N,d]: cu == nullptr,
// nseq = B, maxlen = N. Packed [T,H,d]: cu = device cu_seqlens, maxlen bounds lengths.
struct SeqLayout {
    const int32_t *cu;
    int nseq, H, d;
    int maxlen;
    int total;          // total tokens (dense: B*N)
    int64_t tok_stride; // elements between consecutive tokens of one head
    int64_t head_stride;

    __host__ static SeqLayout dense(int B, int H, int N, int d)
    {
        return SeqLayout{nullptr, B, H, d, N, B * N, (int64_t)d, (int64_t)N * d};
    }
    __host__ static SeqLayout packed(const int32_t *cu, int nseq, int total, int maxlen, int H,
                                     int d)
    {
        return SeqLayout{cu, nseq, H, d, maxlen, total, (int64_t)H * d, (int64_t)d};
    }

    // Token range of sequence s; false (and a status bit) if cu_seqlens is malformed.
    __device__ bool range(int s, int &start, int &len, int *status) const
    {
        if (cu == nullptr) {
            start = s * maxlen;
            len = maxlen;
            return true;
        }
        const int a = __ldg(cu + s), b = __ldg(cu + s + 1);
        if (a < 0 || b < a || b > total || b - a > maxlen || (s == 0 && a != 0)) {
            atomicOr(status, 1 << SAGE_ERR_BAD_SEQLENS);
            start = 0;
            len = 0;
            return false;
        }
        start = a;
        len = b - a;
        return true;
    }

    // Element offset of token `row` of head h of the sequence starting at token `start`.
    __device__ __host__ int64_t offset(int s, int start, int h, int64_t row) const
    {
        if (cu == nullptr)
            return ((int64_t)s * H + h) * maxlen * d + row * d;
        return ((int64_t)start + row) * H * d + (int64_t)h * d;
    }
};

// Device status bits are 1 << sage_status_t; the host reports the lowest set.
__host__ __device__ constexpr int status_bit(sage_status_t s) { return 1 << (int)s; }

// Per-(sequence, head, channel) reductions over tokens, each [nseq, H, d], zeroed by the
// caller before colstats accumulates into them. A null member is not computed.
//   ksum, vsum: fp64 sums of K and V (exact, so the means are order-independent);
//   vhi, vneg:  max V and max -V as order-preserving keys (float_key) for atomicMax.
struct ColStats {
    double *ksum = nullptr;
    double *qsum = nullptr;   // Q column sums, [nseq, H, d] of the query layout (smooth Q)
    double *vsum = nullptr;
    uint32_t *vhi = nullptr;
    uint32_t *vneg = nullptr;
};

// Unsigned key whose integer order is the float order (for atomicMax on floats of any
// sign); key 0 is below every float.
__host__ __device__ inline uint32_t float_key(uint32_t bits)
{
    return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}
__host__ __device__ inline uint32_t key_bits(uint32_t key)
{
    return (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
}

// Launchers (quant.cu, attn_sm100.cu). All return cudaSuccess or the launch error.
// launch_colstats sets *launched (when given) if it launched a kernel.
cudaError_t launch_colstats(const __half *k, const __half *v, const ColStats &cs,
                            const SeqLayout &L, int *status, cudaStream_t st,
                            bool *launched = nullptr);
// Quantizes Q (q_i8 != nullptr), K (k_i8 != nullptr) and/or V (v_e4m3 != nullptr). K is
// smoothed when cs.ksum is set, V when cs.vsum is set (its mean goes to v_mean if that
// is set), Q when cs.qsum is set (its mean goes to q_mean if that is set, and the
// compensation mean(Q) K^T of every key to q_comp, [nseq, H, comp_stride(maxk)]). Q
// lives in layout Lq, K and V in Lk (the same layout for self-attention). fine: one Q
// scale per token and one K scale per 32 tokens (q_scale [nseq,H,maxq], k_scale
// [nseq,H,ceil(maxk/32)]); else per-block scales (128 Q tokens, 64 K tokens).
// after_colstats: the previous launch on the stream is launch_colstats (the one that
// produced cs); this launch may then overlap its tail.
cudaError_t launch_quant(const __half *q, const __half *k, const __half *v, const ColStats &cs,
                         int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                         float *k_mean, uint8_t *v_e4m3, float *v_scale, float *v_mean,
                         float *q_mean, float *q_comp, const SeqLayout &Lq,
                         const SeqLayout &Lk, bool fine, bool after_colstats, int *status,
                         cudaStream_t st);

// Row stride of the smooth-Q compensation array: the key count rounded up to whole
// 128-key tiles, so that every tile's 512 bytes start 16-byte aligned.
__host__ __device__ constexpr int comp_stride(int maxlen_k) { return (maxlen_k + 127) / 128 * 128; }

struct AttnArgs {
    const int8_t *q_i8;
    const float *q_scale;
    const int8_t *k_i8;
    const float *k_scale;
    const void *v;        // fp16 V or E4M3 codes
    const float *v_scale; // FP8 mode
    const float *v_mean;  // FP8 mode with smooth V, else nullptr
    const float *q_comp;  // smooth Q: mean(Q) K^T per key, [nseq, H, comp_stride]; or nullptr
    __half *out;
    int32_t *s_dump;      // debug: int32 scores [nseq,H,maxlen,maxlen] or nullptr
    int causal;
    int pv_mode;
    float sm_scale;
    int fine;             // scales per Q token and per 32 K tokens (else per block)
    // fp16 Q quantized by the attention kernel itself (each CTA its own query tiles, with
    // the codes and scales the quantization kernel would give); q_i8 and q_scale are then
    // unused. With smooth Q, qsum holds Q's fp64 column sums [nseq, H, d]. Else nullptr.
    const __half *q16 = nullptr;
    const double *qsum = nullptr;
};
// Queries in layout Lq, keys and values in Lk (the same layout for self-attention; with
// different lengths the causal mask aligns at the bottom right).
cudaError_t launch_attention(const AttnArgs &a, const SeqLayout &Lq, const SeqLayout &Lk,
                             int *status, cudaStream_t st, sage_status_t *host_err);
cudaError_t launch_wait_selftest(int *status, uint64_t timeout_ns, cudaStream_t st);

}  // namespace sage
