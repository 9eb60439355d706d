// K-ATTN for a handful of queries against many keys (decode): a split-K pass on the CUDA
// cores, for the FP16 P.V mode.
//
// Method (「SageAttention：低比特量化Attention，实现推理加速」, section 技术方案;
// 「如何将SageAttention量化注意力机制集成到你的AI项目中获得2-5倍速度提升」, section
// 语言模型推理加速, the causal mode used while decoding): the scores are the INT8 products
// q_i8 . k_i8 dequantized by q_scale * k_scale * sm_scale (base-2 logits), the softmax
// probabilities are rounded to FP16 and multiply the FP16 V with fp32 accumulation, and the
// output is O / l rounded to FP16, exactly as in the tensor-core kernel. What changes is
// the order: with Nq <= 16 queries a 128-row tensor-core tile is almost empty and one CTA
// per (sequence, head) leaves most SMs idle, so the keys are cut into splits, each split
// is one CTA, and a second kernel merges the splits' partial results
// (m_s, l_s, O_s) -> O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s.
// P is taken relative to its split's maximum instead of the running maximum of a tile
// walk; binary16 rounds with the same relative bound at every scale P takes, so the
// result carries the same rounding error as the tile walk's.
//
// The pass is bound by HBM: every K code (1 byte) and every V element (2 bytes) is read
// once, and at one query the arithmetic (Nq dp4a per 4 key bytes, Nq FMA pairs per V
// pair) is small: B8 H32 Nk32768 d128 reads at the copy bandwidth, 1.8x the tensor-core
// kernel. The arithmetic grows with Nq; from about 8 queries the tensor-core kernel,
// whose tile holds them all, is the faster one.
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>

#include "decode.cuh"
#include "sage_common.cuh"
#include "sm100_ptx.cuh"

namespace sage {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kDecThreads = 256;
constexpr int kDecTile = 128;    // keys per shared-memory tile
constexpr int kDecMaxQ = kDecodeMaxQ;

struct DecodeParams {
    const int8_t *q;      // [B, H, Nq, D]
    const float *qs;      // [B, H, nqb]
    const int8_t *k;      // [B, H, Nk, D]
    const float *ks;      // [B, H, nkb]
    const __half *v;      // [B, H, Nk, D]
    float *pm;            // [B*H, nsplit, Nq]   split maxima (base-2 logits)
    float *pl;            // [B*H, nsplit, Nq]   split sums of p
    float *po;            // [B*H, nsplit, Nq, D] split sums of f16(p) * V
    __half *out;          // [B, H, Nq, D]
    int H, Nq, Nk, nqb, nkb, split_keys, nsplit, causal, fine;
    float sc_log2;        // sm_scale * log2 e
};

// 16-byte asynchronous copy global -> shared (zero-filled when `valid` is false; the source
// address is then not read), grouped with commit / wait.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared memory: the Q codes, a double-buffered tile region (two K tiles, then two V
// tiles, then the key groups' partial outputs) and the split's scores.
template <int D>
constexpr int dec_smem_fixed()
{
    return kDecMaxQ * D + 2 * kDecTile * D * 2;
}

// One CTA: queries 0..Nq-1 of one (sequence, head) against keys [k0, k0 + split_keys).
// NQ: Nq rounded up to a power of two, so that the per-query loops have their exact trip
// count (a loop over all 16 query slots with a predicate each was 5x slower at Nq = 1).
template <int D, int NQ>
__global__ void __launch_bounds__(kDecThreads) decode_partial(const DecodeParams p)
{
    constexpr int kChunks = D / 16;                   // 16-byte chunks of a K row
    constexpr int kCp = D / 2;                        // column pairs of a V row
    constexpr int kKG = kDecThreads / kCp;            // key groups in the P.V pass
    constexpr int kKBytes = kDecTile * D;             // one K tile
    constexpr int kVBytes = kDecTile * D * 2;         // one V tile
    extern __shared__ __align__(16) uint8_t dsm[];
    int8_t *sq = reinterpret_cast<int8_t *>(dsm);                 // Nq rows of Q codes
    uint8_t *tiles = dsm + kDecMaxQ * D;                           // 2 x kVBytes
    float *st = reinterpret_cast<float *>(tiles + 2 * kVBytes);   // [Nq][split_keys]
    __shared__ float s_red[kDecThreads / 32][kDecMaxQ];
    __shared__ float s_m[kDecMaxQ], s_l[kDecMaxQ], s_qsc[kDecMaxQ];

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * p.H + h;
    const int Nq = p.Nq, SK = p.split_keys;
    const int k0 = split * SK;
    const int nk = min(p.Nk - k0, SK);                // >= 1: nsplit = ceil(Nk / SK)
    const int ntile = (nk + kDecTile - 1) / kDecTile;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int8_t *kg0 = p.k + (bh * p.Nk + k0) * D;
    const __half *vg0 = p.v + (bh * p.Nk + k0) * D;

    // K tile t into buffer t % 2, 16-byte chunk ch of row r at chunk ch ^ (r % kChunks)
    // (conflict-free reads by one thread per row); rows past the split are zeros
    auto issue_k = [&](int t) {
        int8_t *dst = reinterpret_cast<int8_t *>(tiles + (t & 1) * kKBytes);
#pragma unroll
        for (int i = 0; i < kDecTile * kChunks / kDecThreads; i++) {
            const int c = tid + i * kDecThreads;
            const int row = c / kChunks, ch = c % kChunks;
            const bool ok = t * kDecTile + row < nk;
            cp_async16(dst + row * D + ((ch ^ (row % kChunks)) * 16),
                       kg0 + (ok ? (int64_t)(t * kDecTile + row) * D + ch * 16 : 0), ok);
        }
        cp_async_commit();
    };
    // V tile t into buffer t % 2, row-major
    auto issue_v = [&](int t) {
        uint8_t *dst = tiles + (t & 1) * kVBytes;
#pragma unroll
        for (int i = 0; i < kVBytes / 16 / kDecThreads; i++) {
            const int c = tid + i * kDecThreads;
            const int row = c / (D / 8);
            const bool ok = t * kDecTile + row < nk;
            cp_async16(dst + c * 16, vg0 + (ok ? (int64_t)t * kDecTile * D + c * 8 : 0), ok);
        }
        cp_async_commit();
    };

    issue_k(0);
    // the queries' codes and their dequantization factors (Nq <= 16: one Q block)
    for (int c = tid; c < Nq * kChunks; c += kDecThreads)
        reinterpret_cast<uint4 *>(sq)[c] =
            __ldg(reinterpret_cast<const uint4 *>(p.q + bh * Nq * D) + c);
    if (tid < Nq)
        s_qsc[tid] = __ldg(p.qs + bh * p.nqb + (p.fine ? tid : 0)) * p.sc_log2;

    // ---- scores: thread = one key of the tile and every other query
    const int jt = tid % kDecTile, qg = tid / kDecTile;   // qg in {0, 1}
    const int kgrp = p.fine ? 32 : kKBlock;
    constexpr int kQHalf = (NQ + 1) / 2;              // queries per thread in the score pass
    float mx[kQHalf];
#pragma unroll
    for (int i = 0; i < kQHalf; i++)
        mx[i] = -INFINITY;
    for (int t = 0; t < ntile; t++) {
        if (t + 1 < ntile) {
            issue_k(t + 1);
            cp_async_wait<1>();                       // tile t has landed (this thread's part)
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();                              // ... and every thread's part
        const int to = t * kDecTile;
        if (to + jt < nk) {
            const int8_t *sk = reinterpret_cast<const int8_t *>(tiles + (t & 1) * kKBytes);
            const int gk = k0 + to + jt;              // key index
            const float ksc = __ldg(p.ks + bh * p.nkb + gk / kgrp);
            uint4 kr[kChunks];
#pragma unroll
            for (int ch = 0; ch < kChunks; ch++)
                kr[ch] = reinterpret_cast<const uint4 *>(sk + jt * D)[ch ^ (jt % kChunks)];
#pragma unroll
            for (int i = 0; i < kQHalf; i++) {
                const int q = qg + 2 * i;
                if (q < Nq) {
                    int acc = 0;
#pragma unroll
                    for (int ch = 0; ch < kChunks; ch++) {
                        const uint4 qv = reinterpret_cast<const uint4 *>(sq + q * D)[ch];
                        acc = __dp4a((int)kr[ch].x, (int)qv.x, acc);
                        acc = __dp4a((int)kr[ch].y, (int)qv.y, acc);
                        acc = __dp4a((int)kr[ch].z, (int)qv.z, acc);
                        acc = __dp4a((int)kr[ch].w, (int)qv.w, acc);
                    }
                    // causal, bottom-right aligned: query q sees keys <= q + Nk - Nq
                    const bool vis = !p.causal || gk <= q + p.Nk - Nq;
                    const float tv = vis ? (float)acc * (s_qsc[q] * ksc) : -INFINITY;
                    st[q * SK + to + jt] = tv;
                    mx[i] = fmaxf(mx[i], tv);
                }
            }
        }
        __syncthreads();                              // buffer t % 2 is free again
    }
    issue_v(0);                                       // lands during the exponentials
    // split maximum per query: over the lanes, then over the 4 warps of the query group
#pragma unroll
    for (int i = 0; i < kQHalf; i++) {
        float m = mx[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0)
            s_red[warp][i] = m;
    }
    __syncthreads();
    if (tid < Nq) {
        const int g = tid % 2, i = tid / 2;           // query tid = g + 2 i
        float m = -INFINITY;
        for (int w = g * 4; w < g * 4 + 4; w++)
            m = fmaxf(m, s_red[w][i]);
        s_m[tid] = m;
    }
    __syncthreads();

    // ---- p = 2^(t - m): l sums p, P.V takes f16(p) (stored back as float); a warp per query
    for (int q = warp; q < Nq; q += kDecThreads / 32) {
        const float m = s_m[q];
        float l = 0.0f;
        for (int j = lane; j < nk; j += 32) {
            const float tv = st[q * SK + j];
            const float pv = m == -INFINITY ? 0.0f : ex2_approx(tv - m);
            l += pv;
            st[q * SK + j] = __half2float(__float2half_rn(pv));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0)
            s_l[q] = l;
    }

    // ---- O_s = sum_j f16(p_j) V_j: thread = one column pair and one key group (keys
    // j = kg, kg + kKG, ...), every query; the key groups are summed at the end
    const int cp = tid % kCp, kg = tid / kCp;
    float2 acc[NQ];
#pragma unroll
    for (int q = 0; q < NQ; q++)
        acc[q] = make_float2(0.0f, 0.0f);
    for (int t = 0; t < ntile; t++) {
        if (t + 1 < ntile) {
            issue_v(t + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();                              // tile t landed; P written (t = 0)
        const __half2 *sv = reinterpret_cast<const __half2 *>(tiles + (t & 1) * kVBytes);
        const int to = t * kDecTile;
        const int nrows = min(kDecTile, nk - to);
        for (int j = kg; j < nrows; j += kKG) {
            const float2 vv = __half22float2(sv[j * kCp + cp]);
#pragma unroll
            for (int q = 0; q < NQ; q++) {
                if (q < Nq) {
                    const float pj = st[q * SK + to + j];
                    acc[q].x = fmaf(pj, vv.x, acc[q].x);
                    acc[q].y = fmaf(pj, vv.y, acc[q].y);
                }
            }
        }
        __syncthreads();                              // buffer t % 2 is free again
    }
    // the key groups' partial sums through shared memory (the tile region is idle now)
    float2 *red = reinterpret_cast<float2 *>(tiles);  // [kKG][Nq][kCp]
#pragma unroll
    for (int q = 0; q < NQ; q++)
        if (q < Nq)
            red[(kg * Nq + q) * kCp + cp] = acc[q];
    __syncthreads();
    const int64_t part = bh * p.nsplit + split;
    for (int e = tid; e < Nq * kCp; e += kDecThreads) {
        const int q = e / kCp, c2 = e % kCp;
        float2 o = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int g = 0; g < kKG; g++) {
            const float2 r = red[(g * Nq + q) * kCp + c2];
            o.x += r.x;
            o.y += r.y;
        }
        reinterpret_cast<float2 *>(p.po + (part * Nq + q) * D)[c2] = o;
    }
    if (tid < Nq) {
        p.pm[part * Nq + tid] = s_m[tid];
        p.pl[part * Nq + tid] = s_l[tid];
    }
}

// One CTA per (sequence, head), one thread per channel: merge the splits of every query.
template <int D>
__global__ void __launch_bounds__(D) decode_combine(const DecodeParams p)
{
    const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
    const int64_t bh = (int64_t)b * p.H + h;
    for (int q = 0; q < p.Nq; q++) {
        float M = -INFINITY;
        for (int s = 0; s < p.nsplit; s++)
            M = fmaxf(M, p.pm[(bh * p.nsplit + s) * p.Nq + q]);
        float l = 0.0f, o = 0.0f;
        if (M != -INFINITY) {
            for (int s = 0; s < p.nsplit; s++) {
                const int64_t part = (bh * p.nsplit + s) * p.Nq + q;
                const float ms = p.pm[part];
                if (ms == -INFINITY)
                    continue;                         // the query sees no key of this split
                const float w = ex2_approx(ms - M);
                l = fmaf(w, p.pl[part], l);
                o = fmaf(w, p.po[part * D + c], o);
            }
        }
        // a query that sees no key at all (more queries than keys, causal) is zero
        p.out[(bh * p.Nq + q) * D + c] = __float2half_rn(l > 0.0f ? o / l : 0.0f);
    }
}

}  // namespace

DecodePlan decode_plan(int B, int H, int Nq, int Nk)
{
    DecodePlan pl{0, 0};
    if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0)
        return pl;
    // about 4 CTAs per SM over the whole grid, whole 128-key tiles per split, and the
    // split's scores (Nq x split_keys fp32) within 32 KB of shared memory
    const int64_t heads = (int64_t)B * H;
    const int64_t want = std::max<int64_t>(1, (4 * 148 + heads - 1) / heads);
    const int cap = std::max(kDecTile, std::min(1024, 8192 / Nq / kDecTile * kDecTile));
    int64_t sk = (Nk + want - 1) / want;
    sk = (sk + kDecTile - 1) / kDecTile * kDecTile;
    pl.split_keys = (int)std::max<int64_t>(kDecTile, std::min<int64_t>(cap, sk));
    pl.nsplit = (Nk + pl.split_keys - 1) / pl.split_keys;
    return pl;
}

size_t decode_partial_floats(int B, int H, int Nq, int Nk, int d)
{
    const DecodePlan pl = decode_plan(B, H, Nq, Nk);
    return (size_t)B * H * pl.nsplit * Nq * (2 + (size_t)d);
}

namespace {
template <int D, int NQ>
cudaError_t launch_partial_nq(dim3 grid, size_t smem, const DecodeParams &p, cudaStream_t st)
{
    cudaError_t e = cudaFuncSetAttribute(decode_partial<D, NQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    decode_partial<D, NQ><<<grid, kDecThreads, smem, st>>>(p);
    return cudaGetLastError();
}
template <int D>
cudaError_t launch_partial(int nq2, dim3 grid, size_t smem, const DecodeParams &p, cudaStream_t st)
{
    switch (nq2) {
    case 1: return launch_partial_nq<D, 1>(grid, smem, p, st);
    case 2: return launch_partial_nq<D, 2>(grid, smem, p, st);
    case 4: return launch_partial_nq<D, 4>(grid, smem, p, st);
    case 8: return launch_partial_nq<D, 8>(grid, smem, p, st);
    default: return launch_partial_nq<D, 16>(grid, smem, p, st);
    }
}
}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st)
{
    DecodeParams p;
    p.q = a.q_i8;
    p.qs = a.q_scale;
    p.k = a.k_i8;
    p.ks = a.k_scale;
    p.v = a.v;
    p.out = a.out;
    p.H = a.H;
    p.Nq = a.Nq;
    p.Nk = a.Nk;
    p.fine = a.fine;
    p.causal = a.causal;
    p.nqb = a.fine ? a.Nq : (a.Nq + kQBlock - 1) / kQBlock;
    p.nkb = a.fine ? (a.Nk + 31) / 32 : (a.Nk + kKBlock - 1) / kKBlock;
    p.sc_log2 = a.sm_scale * kLog2e;
    const DecodePlan pl = decode_plan(a.B, a.H, a.Nq, a.Nk);
    p.split_keys = pl.split_keys;
    p.nsplit = pl.nsplit;
    const size_t np = (size_t)a.B * a.H * pl.nsplit * a.Nq;
    p.pm = a.workspace;
    p.pl = p.pm + np;
    p.po = p.pl + np;
    const size_t smem =
        (a.d == 128 ? dec_smem_fixed<128>() : dec_smem_fixed<64>()) + (size_t)a.Nq * pl.split_keys * 4;
    dim3 grid(pl.nsplit, a.H, a.B);
    const int nq2 = a.Nq <= 1 ? 1 : a.Nq <= 2 ? 2 : a.Nq <= 4 ? 4 : a.Nq <= 8 ? 8 : 16;
    cudaError_t e = a.d == 128 ? launch_partial<128>(nq2, grid, smem, p, st)
                               : launch_partial<64>(nq2, grid, smem, p, st);
    if (e != cudaSuccess)
        return e;
    if (a.d == 128)
        decode_combine<128><<<dim3(a.H, a.B), 128, 0, st>>>(p);
    else
        decode_combine<64><<<dim3(a.H, a.B), 64, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sage
