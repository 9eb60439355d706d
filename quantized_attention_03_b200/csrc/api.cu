// C-ABI entry points of libsage.so: argument validation, workspace carving and the
// launch sequence colstats -> quant -> attention on the caller's stream.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "decode.cuh"
#include "sage_common.cuh"

namespace sage {
namespace {

__device__ int g_status;   // device status word: OR of 1 << sage_status_t

int g_last_cuda_error = 0;
std::mutex g_mu;
int *g_status_ptr[64] = {};

sage_status_t cuda_fail(cudaError_t e)
{
    g_last_cuda_error = (int)e;
    if (std::getenv("SAGE_LOG"))
        std::fprintf(stderr, "sage: CUDA error %d (%s)\n", (int)e, cudaGetErrorString(e));
    return SAGE_ERR_CUDA;
}

// Device address of this device's status word (looked up once per device).
int *status_ptr(sage_status_t *err)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *err = cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e);
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_status_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_status);
        if (e != cudaSuccess) {
            *err = cuda_fail(e);
            return nullptr;
        }
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    *err = SAGE_OK;
    return g_status_ptr[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Stream-ordered scratch comes from one memory pool per device that the library creates
// and never trims (release threshold = all), so that after the first calls an
// allocation is bookkeeping only and never waits for memory to be mapped again.
cudaMemPool_t g_pool[64] = {};

cudaError_t scratch_alloc(void **p, size_t bytes, cudaStream_t st)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_pool[dev] == nullptr) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.handleTypes = cudaMemHandleTypeNone;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t pool = nullptr;
            if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess)
                return e;
            uint64_t keep = ~0ull;
            if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) !=
                cudaSuccess) {
                cudaMemPoolDestroy(pool);
                return e;
            }
            g_pool[dev] = pool;
        }
    }
    return cudaMallocFromPoolAsync(p, bytes ? bytes : 256, g_pool[dev], st);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch carved from one buffer, every part 256-byte aligned.
struct Workspace {
    int8_t *q_i8 = nullptr, *k_i8 = nullptr;
    float *q_scale = nullptr, *k_scale = nullptr, *k_mean = nullptr;
    ColStats cs;                 // contiguous: one memset clears all of it
    uint8_t *v8 = nullptr;
    float *v_scale = nullptr, *v_mean = nullptr;
    float *q_comp = nullptr;     // smooth Q: mean(Q) K^T per key, [nseq, H, comp_stride(maxk)]
    size_t stats_bytes = 0;      // bytes of the column statistics
    size_t total = 0;
};

// Queries: max_q / total_q tokens per (sequence) / in all; keys and values: max_k / total_k.
Workspace carve(char *base, int nseq, int H, int max_q, int max_k, int total_q, int total_k,
                int d, int pv_mode)
{
    Workspace w;
    const size_t qcodes = (size_t)total_q * H * d, kcodes = (size_t)total_k * H * d;
    // scale rows sized for the finer groups (one Q scale per token, one K scale per 32
    // tokens), which also hold the per-block scales
    const size_t nqb = (size_t)max_q, nkb = (max_k + 31) / 32;
    const size_t heads = (size_t)nseq * H;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base ? base + off : nullptr;
        off += align256(bytes);
        return p;
    };
    w.q_i8 = reinterpret_cast<int8_t *>(take(qcodes));
    w.k_i8 = reinterpret_cast<int8_t *>(take(kcodes));
    w.q_scale = reinterpret_cast<float *>(take(heads * nqb * 4));
    w.k_scale = reinterpret_cast<float *>(take(heads * nkb * 4));
    w.k_mean = reinterpret_cast<float *>(take(heads * d * 4));
    w.q_comp = reinterpret_cast<float *>(take(heads * (size_t)comp_stride(max_k) * 4));
    const size_t stats0 = off;
    w.cs.ksum = reinterpret_cast<double *>(take(heads * d * 8));
    w.cs.qsum = reinterpret_cast<double *>(take(heads * d * 8));
    if (pv_mode == SAGE_PV_FP8) {
        w.cs.vsum = reinterpret_cast<double *>(take(heads * d * 8));
        w.cs.vhi = reinterpret_cast<uint32_t *>(take(heads * d * 4));
        w.cs.vneg = reinterpret_cast<uint32_t *>(take(heads * d * 4));
        w.stats_bytes = off - stats0;
        w.v8 = reinterpret_cast<uint8_t *>(take(kcodes));
        w.v_scale = reinterpret_cast<float *>(take(heads * d * 4));
        w.v_mean = reinterpret_cast<float *>(take(heads * d * 4));
    } else {
        w.stats_bytes = off - stats0;
    }
    w.total = off;
    return w;
}

sage_status_t check_shape(int nseq, int H, int maxlen, int d)
{
    if (nseq < 0 || H < 0 || maxlen < 0)
        return SAGE_ERR_INVALID_ARG;
    if (d != 64 && d != 128)
        return SAGE_ERR_UNSUPPORTED;
    if (H > 65535 || nseq > 65535)
        return SAGE_ERR_UNSUPPORTED;    // grid y/z limits
    return SAGE_OK;
}

// The option flags of the fused entry points.
sage_status_t check_smooth(int smooth, int pv_mode)
{
    if (smooth & ~(SAGE_SMOOTH_K | SAGE_SMOOTH_V | SAGE_SMOOTH_Q | SAGE_QK_FINE))
        return SAGE_ERR_INVALID_ARG;
    if ((smooth & SAGE_SMOOTH_V) && pv_mode != SAGE_PV_FP8)
        return SAGE_ERR_UNSUPPORTED;
    return SAGE_OK;
}

float resolve_scale(float sm_scale, int d)
{
    return sm_scale > 0.0f ? sm_scale : 1.0f / std::sqrt((float)d);
}

// Steps 1-3 with the given scratch; q/k/v/out and the smoothing flags already validated.
// Queries in layout L, keys and values in LK (the same layout for self-attention).
sage_status_t forward(const void *q, const void *k, const void *v, void *out, const SeqLayout &L,
                      const SeqLayout &LK, int causal, int smooth, int pv_mode, float sm_scale,
                      char *ws, cudaStream_t st)
{
    sage_status_t err;
    int *status = status_ptr(&err);
    if (!status)
        return err;
    Workspace w = carve(ws, L.nseq, L.H, L.maxlen, LK.maxlen, L.total, LK.total, L.d, pv_mode);
    const bool fp8 = pv_mode == SAGE_PV_FP8;
    const bool sk = (smooth & SAGE_SMOOTH_K) != 0, sv = (smooth & SAGE_SMOOTH_V) != 0;
    const bool fine = (smooth & SAGE_QK_FINE) != 0, sq = (smooth & SAGE_SMOOTH_Q) != 0;
    cudaError_t e = cudaMemsetAsync(w.cs.ksum, 0, w.stats_bytes, st);
    if (e != cudaSuccess)
        return cuda_fail(e);
    const __half *qh = static_cast<const __half *>(q);
    const __half *kh = static_cast<const __half *>(k);
    const __half *vh = static_cast<const __half *>(v);
    ColStats cs = w.cs;
    if (!sk)
        cs.ksum = nullptr;
    if (!sv)
        cs.vsum = nullptr;
    if (!sq)
        cs.qsum = nullptr;
    bool stats = false;
    if ((e = launch_colstats(kh, vh, cs, LK, status, st, &stats)) != cudaSuccess)
        return cuda_fail(e);
    if (sq) {                                  // Q column sums (the K-sum path over Q)
        ColStats qs;
        qs.ksum = cs.qsum;
        if ((e = launch_colstats(qh, nullptr, qs, L, status, st, &stats)) != cudaSuccess)
            return cuda_fail(e);
    }
    // With smooth Q the attention kernel quantizes its own Q tiles from fp16 (measured
    // faster there); otherwise Q's codes come from this pass with K's.
    const bool q_in_kernel = sq;
    if ((e = launch_quant(qh, kh, vh, cs, q_in_kernel ? nullptr : w.q_i8,
                          q_in_kernel ? nullptr : w.q_scale, w.k_i8, w.k_scale, w.k_mean,
                          fp8 ? w.v8 : nullptr, w.v_scale, sv ? w.v_mean : nullptr, nullptr,
                          sq ? w.q_comp : nullptr, L, LK, fine, stats, status, st)) !=
        cudaSuccess)
        return cuda_fail(e);
    AttnArgs a{w.q_i8,     w.q_scale, w.k_i8, w.k_scale, fp8 ? (const void *)w.v8 : v,
               w.v_scale,  sv ? w.v_mean : nullptr,     sq ? w.q_comp : nullptr,
               static_cast<__half *>(out), nullptr, causal, pv_mode,
               resolve_scale(sm_scale, L.d), fine ? 1 : 0};
    if (q_in_kernel) {
        a.q16 = qh;
        a.qsum = cs.qsum;
    }
    sage_status_t herr;
    if ((e = launch_attention(a, L, LK, status, st, &herr)) != cudaSuccess)
        return herr != SAGE_OK ? herr : cuda_fail(e);
    return SAGE_OK;
}

sage_status_t alloc_ws(size_t bytes, cudaStream_t st, char **p)
{
    void *ptr = nullptr;
    cudaError_t e = scratch_alloc(&ptr, bytes, st);
    if (e != cudaSuccess)
        return cuda_fail(e);
    *p = static_cast<char *>(ptr);
    return SAGE_OK;
}

// Shapes of one call: nseq sequences (dense: B), H heads, head dim d; queries have
// max_q tokens per sequence and total_q in all, keys and values max_k and total_k;
// cu_q / cu_k are the device cu_seqlens of a packed layout, or nullptr for dense.
struct Shape {
    const int32_t *cu_q, *cu_k;
    int nseq, H, d, max_q, max_k, total_q, total_k;
    SeqLayout lq() const
    {
        return cu_q ? SeqLayout::packed(cu_q, nseq, total_q, max_q, H, d)
                    : SeqLayout::dense(nseq, H, max_q, d);
    }
    SeqLayout lk() const
    {
        return cu_k ? SeqLayout::packed(cu_k, nseq, total_k, max_k, H, d)
                    : SeqLayout::dense(nseq, H, max_k, d);
    }
    bool empty() const { return nseq == 0 || H == 0 || max_q == 0 || total_q == 0; }
};

Shape dense_shape(int B, int H, int Nq, int Nk, int d)
{
    return Shape{nullptr, nullptr, B, H, d, Nq, Nk, B * Nq, B * Nk};
}

// Host-side checks shared by the entry points: sizes, the head dim and the grid limits.
sage_status_t check_shape2(const Shape &sh)
{
    sage_status_t r = check_shape(sh.nseq, sh.H, sh.max_q, sh.d);
    if (r != SAGE_OK)
        return r;
    if (sh.max_k < 0 || sh.total_q < 0 || sh.total_k < 0)
        return SAGE_ERR_INVALID_ARG;
    return SAGE_OK;
}

// B*N fits the int32 token counts of the dense layout.
bool dense_fits(int B, int N) { return !(B > 0 && N > 0 && (int64_t)B * N > INT32_MAX); }

sage_status_t quant_qk_entry(const void *q, const void *k, const Shape &sh, int8_t *q_i8,
                             float *q_scale, int8_t *k_i8, float *k_scale, float *k_mean,
                             float *q_mean, float *q_comp, int flags, void *workspace,
                             size_t ws_bytes, cudaStream_t st);
sage_status_t quant_v_entry(const void *v, const int32_t *cu_seqlens, int nseq, int total_tokens,
                            int max_seqlen, int H, int d, uint8_t *v_e4m3, float *v_scale,
                            float *v_mean, bool smooth, void *workspace, size_t ws_bytes,
                            cudaStream_t st);

// Step 3 alone on pre-quantized operands (dense; Nq queries, Nk keys).
sage_status_t quantized_entry(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                              const float *k_scale, const void *v, const float *v_scale,
                              const float *v_mean, const float *q_comp, void *out, int B,
                              int H, int Nq, int Nk, int d, int causal, int pv_mode,
                              float sm_scale, bool fine, cudaStream_t st)
{
    sage_status_t r = check_shape(B, H, Nq, d);
    if (r != SAGE_OK)
        return r;
    if (Nk < 0)
        return SAGE_ERR_INVALID_ARG;
    if (pv_mode != SAGE_PV_FP16 && pv_mode != SAGE_PV_FP8)
        return SAGE_ERR_INVALID_ARG;
    if (B == 0 || H == 0 || Nq == 0)
        return SAGE_OK;
    if (!q_i8 || !q_scale || !out || (Nk > 0 && (!k_i8 || !k_scale || !v)) ||
        (pv_mode == SAGE_PV_FP8 && Nk > 0 && !v_scale))
        return SAGE_ERR_INVALID_ARG;
    if (!dense_fits(B, Nq) || !dense_fits(B, Nk))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v) || !aligned16(out) ||
        !aligned16(q_comp))
        return SAGE_ERR_MISALIGNED;
    int *status = status_ptr(&r);
    if (!status)
        return r;
    const Shape sh = dense_shape(B, H, Nq, Nk, d);
    AttnArgs a{q_i8,   q_scale, k_i8,   k_scale,
               v,      v_scale, v_mean, q_comp,
               static_cast<__half *>(out), nullptr, causal, pv_mode,
               resolve_scale(sm_scale, d), fine ? 1 : 0};
    sage_status_t herr;
    cudaError_t e = launch_attention(a, sh.lq(), sh.lk(), status, st, &herr);
    if (e != cudaSuccess)
        return herr != SAGE_OK ? herr : cuda_fail(e);
    return SAGE_OK;
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" {

size_t sage_workspace_size(int nseq, int H, int max_seqlen, int total_tokens, int d, int pv_mode)
{
    return sage_workspace_size_kv(nseq, H, max_seqlen, max_seqlen, total_tokens, total_tokens, d,
                                  pv_mode);
}

size_t sage_attn_workspace_size(int B, int H, int N, int d, int pv_mode)
{
    const int64_t total = (int64_t)B * N;
    if (B < 0 || N < 0 || total > INT_MAX)
        return 0;
    return sage_workspace_size(B, H, N, (int)total, d, pv_mode);
}

size_t sage_workspace_size_kv(int nseq, int H, int max_seqlen_q, int max_seqlen_k,
                              int total_q, int total_k, int d, int pv_mode)
{
    if (nseq < 0 || H < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || total_q < 0 || total_k < 0)
        return 0;
    return carve(nullptr, nseq, H, max_seqlen_q, max_seqlen_k, total_q, total_k, d, pv_mode)
        .total;
}

sage_status_t sage_quant_qk(const void *q, const void *k, int8_t *q_i8, float *q_scale,
                            int8_t *k_i8, float *k_scale, float *k_mean, int B, int H, int N,
                            int d, int smooth_k, sage_stream_t stream)
{
    if (!dense_fits(B, N))
        return SAGE_ERR_UNSUPPORTED;
    if (smooth_k & ~(SAGE_SMOOTH_K | SAGE_QK_FINE))
        return SAGE_ERR_INVALID_ARG;
    return quant_qk_entry(q, k, dense_shape(B, H, N, N, d), q_i8, q_scale, k_i8, k_scale, k_mean,
                          nullptr, nullptr, smooth_k, nullptr, 0,
                          reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_qk_kv(const void *q, const void *k, int8_t *q_i8, float *q_scale,
                               int8_t *k_i8, float *k_scale, float *k_mean, float *q_mean,
                               float *q_comp, int B, int H, int Nq, int Nk, int d, int flags,
                               void *workspace, size_t ws_bytes, sage_stream_t stream)
{
    if (!dense_fits(B, Nq) || !dense_fits(B, Nk))
        return SAGE_ERR_UNSUPPORTED;
    return quant_qk_entry(q, k, dense_shape(B, H, Nq, Nk, d), q_i8, q_scale, k_i8, k_scale,
                          k_mean, q_mean, q_comp, flags, workspace, ws_bytes,
                          reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace sage {
namespace {
// Steps 1-2 with optional caller scratch for the fp64 column sums of K (and of Q with
// smooth Q); nullptr: a stream-ordered allocation is made and released.
sage_status_t quant_qk_entry(const void *q, const void *k, const Shape &sh, int8_t *q_i8,
                             float *q_scale, int8_t *k_i8, float *k_scale, float *k_mean,
                             float *q_mean, float *q_comp, int flags, void *workspace,
                             size_t ws_bytes, cudaStream_t st)
{
    sage_status_t r = check_shape2(sh);
    if (r != SAGE_OK)
        return r;
    // the flags word: SAGE_SMOOTH_K (1, the original boolean), SAGE_SMOOTH_Q, SAGE_QK_FINE
    if (flags & ~(SAGE_SMOOTH_K | SAGE_SMOOTH_Q | SAGE_QK_FINE))
        return SAGE_ERR_INVALID_ARG;
    const bool fine = (flags & SAGE_QK_FINE) != 0;
    const bool sk = (flags & SAGE_SMOOTH_K) != 0, sq = (flags & SAGE_SMOOTH_Q) != 0;
    const bool has_q = sh.max_q > 0 && sh.total_q > 0, has_k = sh.max_k > 0 && sh.total_k > 0;
    if (sh.nseq == 0 || sh.H == 0 || (!has_q && !has_k))
        return SAGE_OK;
    if ((has_q && (!q || !q_i8 || !q_scale)) || (has_k && (!k || !k_i8 || !k_scale || !k_mean)) ||
        (sq && (!q_mean || !q_comp)))
        return SAGE_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_i8) || !aligned16(k_i8))
        return SAGE_ERR_MISALIGNED;
    const size_t sum_bytes = (size_t)sh.nseq * sh.H * sh.d * 8;
    const size_t need = (sk || sq) ? (sq ? 2 : 1) * sum_bytes : 0;   // [K sums | Q sums]
    if (workspace != nullptr && need) {
        if (ws_bytes < need)
            return SAGE_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
            return SAGE_ERR_MISALIGNED;
    }
    int *status = status_ptr(&r);
    if (!status)
        return r;
    const SeqLayout Lq = sh.lq(), Lk = sh.lk();
    char *sums = nullptr;
    bool owned = false;
    cudaError_t e = cudaSuccess;
    if (need) {
        if (workspace != nullptr) {
            sums = static_cast<char *>(workspace);
        } else {
            void *p = nullptr;
            if ((e = scratch_alloc(&p, need, st)) != cudaSuccess)
                return cuda_fail(e);
            sums = static_cast<char *>(p);
            owned = true;
        }
    }
    ColStats cs;
    if (sk && has_k)
        cs.ksum = reinterpret_cast<double *>(sums);
    if (sq)
        cs.qsum = reinterpret_cast<double *>(sums + sum_bytes);
    if (need)
        e = cudaMemsetAsync(sums, 0, need, st);
    bool stats = false;
    if (e == cudaSuccess && cs.ksum != nullptr) {
        ColStats kc;
        kc.ksum = cs.ksum;
        e = launch_colstats(static_cast<const __half *>(k), nullptr, kc, Lk, status, st, &stats);
    }
    if (e == cudaSuccess && cs.qsum != nullptr) {
        ColStats qc;
        qc.ksum = cs.qsum;
        e = launch_colstats(static_cast<const __half *>(q), nullptr, qc, Lq, status, st, &stats);
    }
    if (e == cudaSuccess)
        e = launch_quant(static_cast<const __half *>(q), static_cast<const __half *>(k), nullptr,
                         cs, q_i8, q_scale, k_i8, k_scale, k_mean, nullptr, nullptr, nullptr,
                         sq ? q_mean : nullptr, sq ? q_comp : nullptr, Lq, Lk, fine, stats,
                         status, st);
    if (owned)
        cudaFreeAsync(sums, st);
    return e == cudaSuccess ? SAGE_OK : cuda_fail(e);
}

// V to E4M3 (smooth: V - mean(V) first, the mean written to v_mean), dense or packed,
// with caller scratch for the column statistics or (workspace == nullptr) a
// stream-ordered allocation.
sage_status_t quant_v_entry(const void *v, const int32_t *cu_seqlens, int nseq, int total_tokens,
                            int max_seqlen, int H, int d, uint8_t *v_e4m3, float *v_scale,
                            float *v_mean, bool smooth, void *workspace, size_t ws_bytes,
                            cudaStream_t st)
{
    sage_status_t r = check_shape(nseq, H, max_seqlen, d);
    if (r != SAGE_OK)
        return r;
    if (nseq == 0 || H == 0 || max_seqlen == 0 || total_tokens == 0)
        return SAGE_OK;
    if (!v || !v_e4m3 || !v_scale || (smooth && !v_mean) || total_tokens < 0)
        return SAGE_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(v_e4m3))
        return SAGE_ERR_MISALIGNED;
    // [vsum (fp64) | vhi | vneg] per (sequence, head, channel)
    const size_t n = (size_t)nseq * H * d;
    const size_t bytes = n * (8 + 4 + 4);
    if (workspace != nullptr) {
        if (ws_bytes < bytes)
            return SAGE_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
            return SAGE_ERR_MISALIGNED;
    }
    int *status = status_ptr(&r);
    if (!status)
        return r;
    const SeqLayout L = cu_seqlens ? SeqLayout::packed(cu_seqlens, nseq, total_tokens, max_seqlen, H, d)
                                   : SeqLayout::dense(nseq, H, max_seqlen, d);
    void *p = workspace;
    cudaError_t e;
    if (p == nullptr && (e = scratch_alloc(&p, bytes, st)) != cudaSuccess)
        return cuda_fail(e);
    ColStats cs;
    cs.vsum = smooth ? static_cast<double *>(p) : nullptr;
    cs.vhi = reinterpret_cast<uint32_t *>(static_cast<char *>(p) + n * 8);
    cs.vneg = cs.vhi + n;
    bool stats = false;
    if ((e = cudaMemsetAsync(p, 0, bytes, st)) == cudaSuccess &&
        (e = launch_colstats(nullptr, static_cast<const __half *>(v), cs, L, status, st,
                             &stats)) == cudaSuccess)
        e = launch_quant(nullptr, nullptr, static_cast<const __half *>(v), cs, nullptr, nullptr,
                         nullptr, nullptr, nullptr, v_e4m3, v_scale, smooth ? v_mean : nullptr,
                         nullptr, nullptr, L, L, false, stats, status, st);
    if (workspace == nullptr)
        cudaFreeAsync(p, st);
    return e == cudaSuccess ? SAGE_OK : cuda_fail(e);
}
}  // namespace
}  // namespace sage

extern "C" {

sage_status_t sage_quant_qk_varlen(const void *q, const void *k, const int32_t *cu_seqlens,
                                   int nseq, int total_tokens, int max_seqlen, int H, int d,
                                   int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                                   float *k_mean, int smooth_k, sage_stream_t stream)
{
    const Shape sh{cu_seqlens, cu_seqlens, nseq, H, d, max_seqlen, max_seqlen, total_tokens,
                   total_tokens};
    if (smooth_k & ~(SAGE_SMOOTH_K | SAGE_QK_FINE))
        return SAGE_ERR_INVALID_ARG;
    return quant_qk_entry(q, k, sh, q_i8, q_scale, k_i8, k_scale, k_mean, nullptr, nullptr,
                          smooth_k, nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_qk_ws(const void *q, const void *k, int8_t *q_i8, float *q_scale,
                               int8_t *k_i8, float *k_scale, float *k_mean, int B, int H, int N,
                               int d, int smooth_k, void *workspace, size_t ws_bytes,
                               sage_stream_t stream)
{
    if (workspace == nullptr && (smooth_k & SAGE_SMOOTH_K) && !(B == 0 || H == 0 || N == 0))
        return SAGE_ERR_WORKSPACE;
    if (!dense_fits(B, N))
        return SAGE_ERR_UNSUPPORTED;
    if (smooth_k & ~(SAGE_SMOOTH_K | SAGE_QK_FINE))
        return SAGE_ERR_INVALID_ARG;
    return quant_qk_entry(q, k, dense_shape(B, H, N, N, d), q_i8, q_scale, k_i8, k_scale, k_mean,
                          nullptr, nullptr, smooth_k, workspace, ws_bytes,
                          reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_v_fp8_smooth_varlen(const void *v, const int32_t *cu_seqlens, int nseq,
                                             int total_tokens, int max_seqlen, int H, int d,
                                             uint8_t *v_e4m3, float *v_scale, float *v_mean,
                                             sage_stream_t stream)
{
    return quant_v_entry(v, cu_seqlens, nseq, total_tokens, max_seqlen, H, d, v_e4m3, v_scale,
                         v_mean, true, nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_v_fp8_smooth(const void *v, uint8_t *v_e4m3, float *v_scale,
                                      float *v_mean, int B, int H, int N, int d,
                                      sage_stream_t stream)
{
    if (B > 0 && N > 0 && (int64_t)B * N > INT32_MAX)
        return SAGE_ERR_UNSUPPORTED;
    return quant_v_entry(v, nullptr, B, B * N, N, H, d, v_e4m3, v_scale, v_mean, true, nullptr,
                         0, reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_v_fp8_varlen(const void *v, const int32_t *cu_seqlens, int nseq,
                                      int total_tokens, int max_seqlen, int H, int d,
                                      uint8_t *v_e4m3, float *v_scale, sage_stream_t stream)
{
    return quant_v_entry(v, cu_seqlens, nseq, total_tokens, max_seqlen, H, d, v_e4m3, v_scale,
                         nullptr, false, nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_v_fp8(const void *v, uint8_t *v_e4m3, float *v_scale, int B, int H,
                               int N, int d, sage_stream_t stream)
{
    if (B > 0 && N > 0 && (int64_t)B * N > INT32_MAX)
        return SAGE_ERR_UNSUPPORTED;
    return quant_v_entry(v, nullptr, B, B * N, N, H, d, v_e4m3, v_scale, nullptr, false, nullptr,
                         0, reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_quant_v_fp8_ws(const void *v, uint8_t *v_e4m3, float *v_scale, float *v_mean,
                                  int B, int H, int N, int d, void *workspace, size_t ws_bytes,
                                  sage_stream_t stream)
{
    if (workspace == nullptr && !(B == 0 || H == 0 || N == 0))
        return SAGE_ERR_WORKSPACE;
    if (!dense_fits(B, N))
        return SAGE_ERR_UNSUPPORTED;
    return quant_v_entry(v, nullptr, B, B * N, N, H, d, v_e4m3, v_scale, v_mean,
                         v_mean != nullptr, workspace, ws_bytes,
                         reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace sage {
namespace {
// Dense or packed forward pass with optional caller scratch.
sage_status_t attn_entry(const void *q, const void *k, const void *v, void *out, const Shape &sh,
                         int causal, int smooth_k, int pv_mode, float sm_scale, void *workspace,
                         size_t ws_bytes, sage_stream_t stream)
{
    sage_status_t r = check_shape2(sh);
    if (r != SAGE_OK)
        return r;
    if (pv_mode != SAGE_PV_FP16 && pv_mode != SAGE_PV_FP8)
        return SAGE_ERR_INVALID_ARG;
    if ((r = check_smooth(smooth_k, pv_mode)) != SAGE_OK)
        return r;
    if (sh.empty())
        return SAGE_OK;
    const bool no_keys = sh.max_k == 0 || sh.total_k == 0;
    if (!q || !out || (!no_keys && (!k || !v)))
        return SAGE_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return SAGE_ERR_MISALIGNED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (no_keys) {   // no query sees a key: the output is zero
        cudaError_t e = cudaMemsetAsync(out, 0, (size_t)sh.total_q * sh.H * sh.d * 2, st);
        return e == cudaSuccess ? SAGE_OK : cuda_fail(e);
    }
    const size_t need = sage_workspace_size_kv(sh.nseq, sh.H, sh.max_q, sh.max_k, sh.total_q,
                                               sh.total_k, sh.d, pv_mode);
    if (workspace != nullptr) {
        if (ws_bytes < need)
            return SAGE_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return SAGE_ERR_MISALIGNED;
        return forward(q, k, v, out, sh.lq(), sh.lk(), causal, smooth_k, pv_mode, sm_scale,
                       static_cast<char *>(workspace), st);
    }
    char *ws = nullptr;
    if ((r = alloc_ws(need, st, &ws)) != SAGE_OK)
        return r;
    r = forward(q, k, v, out, sh.lq(), sh.lk(), causal, smooth_k, pv_mode, sm_scale, ws, st);
    cudaFreeAsync(ws, st);
    return r;
}
}  // namespace
}  // namespace sage

extern "C" {

sage_status_t sage_attn_varlen_fwd(const void *q, const void *k, const void *v, void *out,
                                   const int32_t *cu_seqlens, int nseq, int total_tokens,
                                   int max_seqlen, int H, int d, int causal, int smooth_k,
                                   int pv_mode, float sm_scale, void *workspace,
                                   size_t ws_bytes, sage_stream_t stream)
{
    if (cu_seqlens == nullptr && nseq > 0 && total_tokens > 0)
        return SAGE_ERR_INVALID_ARG;
    const Shape sh{cu_seqlens, cu_seqlens, nseq, H, d, max_seqlen, max_seqlen, total_tokens,
                   total_tokens};
    return attn_entry(q, k, v, out, sh, causal, smooth_k, pv_mode, sm_scale, workspace,
                      ws_bytes, stream);
}

sage_status_t sage_attn_varlen_fwd_kv(const void *q, const void *k, const void *v, void *out,
                                      const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                      int nseq, int total_q, int total_k, int max_seqlen_q,
                                      int max_seqlen_k, int H, int d, int causal, int smooth_k,
                                      int pv_mode, float sm_scale, void *workspace,
                                      size_t ws_bytes, sage_stream_t stream)
{
    if (nseq > 0 && ((cu_seqlens_q == nullptr && total_q > 0) ||
                     (cu_seqlens_k == nullptr && total_k > 0)))
        return SAGE_ERR_INVALID_ARG;
    const Shape sh{cu_seqlens_q, cu_seqlens_k, nseq, H, d, max_seqlen_q, max_seqlen_k, total_q,
                   total_k};
    return attn_entry(q, k, v, out, sh, causal, smooth_k, pv_mode, sm_scale, workspace,
                      ws_bytes, stream);
}

sage_status_t sage_attn_fwd_ws(const void *q, const void *k, const void *v, void *out, int B,
                               int H, int N, int d, int causal, int smooth_k, int pv_mode,
                               float sm_scale, void *workspace, size_t ws_bytes,
                               sage_stream_t stream)
{
    if (workspace == nullptr && !(B == 0 || H == 0 || N == 0))
        return SAGE_ERR_WORKSPACE;
    if (!dense_fits(B, N))
        return SAGE_ERR_UNSUPPORTED;
    return attn_entry(q, k, v, out, dense_shape(B, H, N, N, d), causal, smooth_k, pv_mode,
                      sm_scale, workspace, ws_bytes, stream);
}

sage_status_t sage_attn_fwd(const void *q, const void *k, const void *v, void *out, int B, int H,
                            int N, int d, int causal, int smooth_k, int pv_mode, float sm_scale,
                            sage_stream_t stream)
{
    if (!dense_fits(B, N))
        return SAGE_ERR_UNSUPPORTED;
    return attn_entry(q, k, v, out, dense_shape(B, H, N, N, d), causal, smooth_k, pv_mode,
                      sm_scale, nullptr, 0, stream);
}

sage_status_t sage_attn_fwd_kv(const void *q, const void *k, const void *v, void *out, int B,
                               int H, int Nq, int Nk, int d, int causal, int smooth_k,
                               int pv_mode, float sm_scale, void *workspace, size_t ws_bytes,
                               sage_stream_t stream)
{
    if (!dense_fits(B, Nq) || !dense_fits(B, Nk))
        return SAGE_ERR_UNSUPPORTED;
    return attn_entry(q, k, v, out, dense_shape(B, H, Nq, Nk, d), causal, smooth_k, pv_mode,
                      sm_scale, workspace, ws_bytes, stream);
}

sage_status_t sage_attn_fwd_quantized(const int8_t *q_i8, const float *q_scale,
                                      const int8_t *k_i8, const float *k_scale, const void *v,
                                      const float *v_scale, void *out, int B, int H, int N,
                                      int d, int causal, int pv_mode, float sm_scale,
                                      sage_stream_t stream)
{
    return quantized_entry(q_i8, q_scale, k_i8, k_scale, v, v_scale, nullptr, nullptr, out, B, H,
                           N, N, d, causal, pv_mode, sm_scale, false,
                           reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_attn_fwd_quantized_kv(const int8_t *q_i8, const float *q_scale,
                                         const int8_t *k_i8, const float *k_scale, const void *v,
                                         const float *v_scale, const float *v_mean,
                                         const float *q_comp, void *out, int B, int H, int Nq,
                                         int Nk, int d, int causal, int pv_mode, float sm_scale,
                                         int flags, sage_stream_t stream)
{
    if (flags & ~SAGE_QK_FINE)
        return SAGE_ERR_INVALID_ARG;
    if (v_mean != nullptr && pv_mode != SAGE_PV_FP8)
        return SAGE_ERR_UNSUPPORTED;
    return quantized_entry(q_i8, q_scale, k_i8, k_scale, v, v_scale, v_mean, q_comp, out, B, H,
                           Nq, Nk, d, causal, pv_mode, sm_scale, (flags & SAGE_QK_FINE) != 0,
                           reinterpret_cast<cudaStream_t>(stream));
}

size_t sage_attn_decode_workspace_size(int B, int H, int Nq, int Nk, int d)
{
    if (B <= 0 || H <= 0 || Nq <= 0 || Nq > kDecodeMaxQ || Nk <= 0 || (d != 64 && d != 128))
        return 0;
    return decode_partial_floats(B, H, Nq, Nk, d) * sizeof(float);
}

sage_status_t sage_attn_decode_quantized(const int8_t *q_i8, const float *q_scale,
                                         const int8_t *k_i8, const float *k_scale, const void *v,
                                         void *out, int B, int H, int Nq, int Nk, int d,
                                         int causal, float sm_scale, int flags, void *workspace,
                                         size_t ws_bytes, sage_stream_t stream)
{
    sage_status_t r = check_shape(B, H, Nq, d);
    if (r != SAGE_OK)
        return r;
    if (Nk < 0 || (flags & ~SAGE_QK_FINE))
        return SAGE_ERR_INVALID_ARG;
    if (Nq > kDecodeMaxQ)
        return SAGE_ERR_UNSUPPORTED;
    if (B == 0 || H == 0 || Nq == 0)
        return SAGE_OK;
    if (!q_i8 || !q_scale || !out || (Nk > 0 && (!k_i8 || !k_scale || !v || !workspace)))
        return SAGE_ERR_INVALID_ARG;
    if (!dense_fits(B, Nq) || !dense_fits(B, Nk))
        return SAGE_ERR_UNSUPPORTED;
    if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v) || !aligned16(out) ||
        !aligned16(workspace))
        return SAGE_ERR_MISALIGNED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (Nk == 0) {   // no keys: every query sees none
        cudaError_t e = cudaMemsetAsync(out, 0, (size_t)B * H * Nq * d * 2, st);
        return e == cudaSuccess ? SAGE_OK : cuda_fail(e);
    }
    if (ws_bytes < sage_attn_decode_workspace_size(B, H, Nq, Nk, d))
        return SAGE_ERR_WORKSPACE;
    DecodeArgs a{q_i8, q_scale, k_i8, k_scale, static_cast<const __half *>(v),
                 static_cast<__half *>(out), static_cast<float *>(workspace), B, H, Nq, Nk, d,
                 causal ? 1 : 0, (flags & SAGE_QK_FINE) ? 1 : 0, resolve_scale(sm_scale, d)};
    cudaError_t e = launch_decode(a, st);
    return e == cudaSuccess ? SAGE_OK : cuda_fail(e);
}

sage_status_t sage_attn_fwd_quantized_smooth_v(const int8_t *q_i8, const float *q_scale,
                                               const int8_t *k_i8, const float *k_scale,
                                               const uint8_t *v_e4m3, const float *v_scale,
                                               const float *v_mean, void *out, int B, int H,
                                               int N, int d, int causal, float sm_scale,
                                               sage_stream_t stream)
{
    if (v_mean == nullptr && B > 0 && H > 0 && N > 0)
        return SAGE_ERR_INVALID_ARG;
    return quantized_entry(q_i8, q_scale, k_i8, k_scale, v_e4m3, v_scale, v_mean, nullptr, out,
                           B, H, N, N, d, causal, SAGE_PV_FP8, sm_scale, false,
                           reinterpret_cast<cudaStream_t>(stream));
}

sage_status_t sage_debug_qk_int32(const int8_t *q_i8, const int8_t *k_i8, int32_t *s_out, int B,
                                  int H, int N, int d, sage_stream_t stream)
{
    sage_status_t r = check_shape(B, H, N, d);
    if (r != SAGE_OK)
        return r;
    if (B == 0 || H == 0 || N == 0)
        return SAGE_OK;
    if (!q_i8 || !k_i8 || !s_out)
        return SAGE_ERR_INVALID_ARG;
    if (!aligned16(q_i8) || !aligned16(k_i8))
        return SAGE_ERR_MISALIGNED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int *status = status_ptr(&r);
    if (!status)
        return r;
    const size_t elems = (size_t)B * H * N * d;
    const size_t nqb = (N + kQBlock - 1) / kQBlock, nkb = (N + kKBlock - 1) / kKBlock;
    const size_t sc_bytes = align256((size_t)B * H * (nqb + nkb) * 4);
    const size_t bytes = sc_bytes + 2 * align256(elems * 2);
    char *ws = nullptr;
    if ((r = alloc_ws(bytes, st, &ws)) != SAGE_OK)
        return r;
    cudaError_t e = cudaMemsetAsync(ws, 0, bytes, st);   // zero scales and V: P V stays finite
    if (e == cudaSuccess) {
        const float *qs = reinterpret_cast<float *>(ws);
        const float *ks = qs + (size_t)B * H * nqb;
        const void *vz = ws + sc_bytes;
        __half *o = reinterpret_cast<__half *>(ws + sc_bytes + align256(elems * 2));
        AttnArgs a{q_i8, qs, k_i8, ks, vz, nullptr, nullptr, nullptr, o, s_out, 0, SAGE_PV_FP16,
                   1.0f, 0};
        sage_status_t herr;
        const SeqLayout L = SeqLayout::dense(B, H, N, d);
        e = launch_attention(a, L, L, status, st, &herr);
        if (e != cudaSuccess && herr != SAGE_OK) {
            cudaFreeAsync(ws, st);
            return herr;
        }
    }
    cudaFreeAsync(ws, st);
    return e == cudaSuccess ? SAGE_OK : cuda_fail(e);
}

sage_status_t sage_debug_wait_timeout(unsigned long long timeout_ns, sage_stream_t stream)
{
    if (timeout_ns < 1000ull || timeout_ns > 1000000000ull)
        return SAGE_ERR_INVALID_ARG;
    sage_status_t r;
    int *status = status_ptr(&r);
    if (!status)
        return r;
    cudaError_t e =
        launch_wait_selftest(status, timeout_ns, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SAGE_OK : cuda_fail(e);
}

sage_status_t sage_get_device_status(sage_stream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e);
    int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int))) != cudaSuccess)
        return cuda_fail(e);
    if (v != 0) {
        const int zero = 0;
        if ((e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int))) != cudaSuccess)
            return cuda_fail(e);
        for (int b = 1; b < 31; b++)
            if (v & (1 << b))
                return static_cast<sage_status_t>(b);
    }
    return SAGE_OK;
}

const char *sage_status_string(sage_status_t s)
{
    switch (s) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_MISALIGNED: return "SAGE_ERR_MISALIGNED";
    case SAGE_ERR_WORKSPACE: return "SAGE_ERR_WORKSPACE";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
    case SAGE_ERR_BAD_SEQLENS: return "SAGE_ERR_BAD_SEQLENS";
    }
    return "SAGE_ERR_UNKNOWN";
}

int sage_last_cuda_error(void) { return g_last_cuda_error; }

int sage_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------------
// Allocation-free variant of sage_attn_fwd.
//
// Some callers cannot allocate device memory once they are running: a serving process
// that hands all GPU memory to its own allocator at start-up and forbids further driver
// allocations, or a latency-critical loop that must not risk an allocation stalling or
// failing. If such a caller also has no scratch buffer of its own to pass to
// sage_attn_fwd_ws, it uses this entry point: its scratch is a fixed array in device
// memory that belongs to this library (every GPU that loads the library holds it until
// the process exits).
namespace sage {
namespace {

// Host code may not use the array's name as a device address: on the host it is only a
// stand-in symbol. Its device address is looked up once per device with
// cudaGetSymbolAddress and cached here.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SAGE_NOALLOC_SCRATCH_BYTES];
char *g_noalloc_ptr[64] = {};

sage_status_t noalloc_scratch(char **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64)
        return cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // with `dev` current
        if (e != cudaSuccess)
            return cuda_fail(e);
        g_noalloc_ptr[dev] = static_cast<char *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return SAGE_OK;
}

}  // namespace
}  // namespace sage

extern "C" sage_status_t sage_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                               void *out, int B, int H, int N, int d, int causal,
                                               int smooth_k, int pv_mode, float sm_scale,
                                               sage_stream_t stream)
{
    sage_status_t r = check_shape(B, H, N, d);
    if (r != SAGE_OK)
        return r;
    if (pv_mode != SAGE_PV_FP16 && pv_mode != SAGE_PV_FP8)
        return SAGE_ERR_INVALID_ARG;
    if ((r = check_smooth(smooth_k, pv_mode)) != SAGE_OK)
        return r;
    if (B == 0 || H == 0 || N == 0)
        return SAGE_OK;
    if ((int64_t)B * N > INT32_MAX)
        return SAGE_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out)
        return SAGE_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return SAGE_ERR_MISALIGNED;
    const size_t need = sage_workspace_size(B, H, N, B * N, d, pv_mode);
    if (need > (size_t)SAGE_NOALLOC_SCRATCH_BYTES) {
        if (std::getenv("SAGE_LOG"))
            std::fprintf(stderr,
                         "sage_attn_fwd_noalloc: this call needs %zu bytes of scratch, more than "
                         "the %zu-byte static buffer; use sage_attn_fwd or sage_attn_fwd_ws\n",
                         need, (size_t)SAGE_NOALLOC_SCRATCH_BYTES);
        return SAGE_ERR_WORKSPACE;
    }
    char *ws = nullptr;
    if ((r = noalloc_scratch(&ws)) != SAGE_OK)
        return r;
    // forward() zeroes the only scratch that must start at zero (the K and V column
    // statistics) before its kernels run; everything else is written before it is read.
    const SeqLayout L = SeqLayout::dense(B, H, N, d);
    return forward(q, k, v, out, L, L, causal, smooth_k, pv_mode,
                   sm_scale, ws, reinterpret_cast<cudaStream_t>(stream));
}
