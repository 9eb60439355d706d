// K-QUANT: smooth K and per-block INT8 quantization of Q and K; E4M3 quantization of V.
//
// 「SageAttention：低比特量化Attention，实现推理加速」, section 技术方案: K <- K - mean(K) with the mean per channel
// over tokens; Q and K quantized to INT8 per block of FlashAttention size (Q: 128
// tokens, K: 64 tokens) with one fp32 scale amax/127 per block. "SageAttention2"
// article, 技术方案 (4): V in E4M3, here with one fp32 scale (amax/448) per channel;
// the paragraph after (4): optionally V <- V - mean(V) first (smooth V).
//
// Two HBM-bound passes:
//   colstats: per-(sequence, head, channel) reductions over tokens: fp64 sums of K and
//             V (exact for |x| N < 2^29, so the means do not depend on summation
//             order) and the max and min of V. Row chunks of 512 tokens, atomics.
//             amax |fl(V - mean)| = max(fl(max V - mean), fl(mean - min V)) exactly,
//             because fp32 rounding is monotonic, so V needs no third pass.
//   quant:    one CTA per 128-token chunk of Q (one Q block), K (two K blocks) or V,
//             staged in shared memory by bulk copies; warp-shuffle amax. Codes are the
//             rounding of the IEEE fp32 quotient x / scale, computed as x * (1 / scale)
//             with an exact division only where the two could round differently, so
//             they match the definition bit for bit without a division per element.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "quant_codes.cuh"
#include "sage_common.cuh"
#include "sm100_ptx.cuh"

namespace sage {

namespace {

constexpr int kColChunk = 512;   // tokens per colstats CTA
constexpr int kThreads = 256;
constexpr uint64_t kWaitNs = 2000000000ull;   // bound on the wait for a chunk's bulk copy

// DO_K: fp64 sums of K; DO_V: max and max of -V, plus fp64 sums of V when cs.vsum is set.
template <int D, bool DO_K, bool DO_V>
__global__ void __launch_bounds__(kThreads) colstats_kernel(const __half *__restrict__ k,
                                                            const __half *__restrict__ v,
                                                            ColStats cs, SeqLayout L, int *status)
{
    constexpr int kGroups = D / 8;              // 16-byte column groups per row
    constexpr int kRowsPerPass = kThreads / kGroups;
    constexpr int kWarps = kThreads / 32;
    // the quantization kernel that follows may start its Q blocks now (they do not read
    // the sums; its K and V blocks wait for this grid to complete)
    griddep_launch_dependents();
    const int s = blockIdx.z, h = blockIdx.y;
    int start, len;
    if (!L.range(s, start, len, status))
        return;
    const int r_begin = blockIdx.x * kColChunk;
    if (r_begin >= len)
        return;
    const int r_end = min(len, r_begin + kColChunk);
    const int g = threadIdx.x % kGroups, r0 = threadIdx.x / kGroups;
    constexpr bool do_k = DO_K, do_v = DO_V;
    const bool do_vsum = DO_V && cs.vsum != nullptr;

    double ks[8], vs[8];
    float hi[8], ng[8];                          // max V and max -V
#pragma unroll
    for (int i = 0; i < 8; i++) {
        ks[i] = vs[i] = 0.0;
        hi[i] = ng[i] = -INFINITY;
    }
    auto add_k = [&](const uint4 &u) {
        float f[8];
        unpack8(u, f);
#pragma unroll
        for (int i = 0; i < 8; i++)
            ks[i] += (double)f[i];
    };
    auto add_v = [&](const uint4 &u) {
        float f[8];
        unpack8(u, f);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            hi[i] = fmaxf(hi[i], f[i]);
            ng[i] = fmaxf(ng[i], -f[i]);
            if (do_vsum)
                vs[i] += (double)f[i];
        }
    };
    // eight rows per iteration, so that eight 16-byte loads per tensor are in flight (the
    // pass is bound by memory latency: four measured 2% slower)
    constexpr int kUnroll = 8;
    int r = r_begin + r0;
    for (; r + (kUnroll - 1) * kRowsPerPass < r_end; r += kUnroll * kRowsPerPass) {
        uint4 uk[kUnroll], uv[kUnroll];
#pragma unroll
        for (int j = 0; j < kUnroll; j++) {
            const int64_t off = L.offset(s, start, h, r + j * kRowsPerPass) + g * 8;
            if (do_k)
                uk[j] = __ldg(reinterpret_cast<const uint4 *>(k + off));
            if (do_v)
                uv[j] = __ldg(reinterpret_cast<const uint4 *>(v + off));
        }
#pragma unroll
        for (int j = 0; j < kUnroll; j++) {
            if (do_k)
                add_k(uk[j]);
            if (do_v)
                add_v(uv[j]);
        }
    }
    for (; r < r_end; r += kRowsPerPass) {
        const int64_t off = L.offset(s, start, h, r) + g * 8;
        if (do_k)
            add_k(__ldg(reinterpret_cast<const uint4 *>(k + off)));
        if (do_v)
            add_v(__ldg(reinterpret_cast<const uint4 *>(v + off)));
    }

    // lanes kGroups apart hold the same columns: fold them, then one row per warp
#pragma unroll
    for (int o = kGroups; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < 8; i++) {
            ks[i] += __shfl_xor_sync(0xffffffffu, ks[i], o);
            vs[i] += __shfl_xor_sync(0xffffffffu, vs[i], o);
            hi[i] = fmaxf(hi[i], __shfl_xor_sync(0xffffffffu, hi[i], o));
            ng[i] = fmaxf(ng[i], __shfl_xor_sync(0xffffffffu, ng[i], o));
        }
    __shared__ double s_ks[kWarps][D], s_vs[kWarps][D];
    __shared__ float s_hi[kWarps][D], s_ng[kWarps][D];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane < kGroups) {
#pragma unroll
        for (int i = 0; i < 8; i++) {
            s_ks[warp][g * 8 + i] = ks[i];
            s_vs[warp][g * 8 + i] = vs[i];
            s_hi[warp][g * 8 + i] = hi[i];
            s_ng[warp][g * 8 + i] = ng[i];
        }
    }
    __syncthreads();
    if (threadIdx.x < D) {
        const int c = threadIdx.x;
        double tk = 0.0, tv = 0.0;
        float mh = -INFINITY, mn = -INFINITY;
        for (int w = 0; w < kWarps; w++) {
            tk += s_ks[w][c];
            tv += s_vs[w][c];
            mh = fmaxf(mh, s_hi[w][c]);
            mn = fmaxf(mn, s_ng[w][c]);
        }
        const int64_t o = ((int64_t)s * L.H + h) * D + c;
        if (do_k)
            atomicAdd(cs.ksum + o, tk);
        if (do_v) {
            if (do_vsum)
                atomicAdd(cs.vsum + o, tv);
            atomicMax(cs.vhi + o, float_key(__float_as_uint(mh)));
            atomicMax(cs.vneg + o, float_key(__float_as_uint(mn)));
        }
    }
}

// fl(x / s) for the E4M3 encoder, with r = fl(1 / s): the product x * r differs from the
// IEEE quotient by at most a few ulps, which changes the E4M3 rounding only next to a
// rounding midpoint of a normal E4M3 binade (low 20 mantissa bits near 1 << 19) or in the
// E4M3 subnormal range; there the exact division is used.
__device__ __forceinline__ float e4m3_quotient(float x, float s, float r)
{
    const float q = x * r;
    const uint32_t m = __float_as_uint(q) & 0xFFFFFu;
    const bool near_mid = (m > 0x80000u - 16u) && (m < 0x80000u + 16u);
    if (near_mid || fabsf(q) < 0.015625f)          // 2^-6: E4M3 subnormals below this
        return __fdiv_rn(x, s);
    return q;
}

// Codes of one 128-token chunk of Q or K (already in shared memory) with one scale per G
// rows: G = 128 (a Q block), 64 (a K block), 32 (finer K groups) or 1 (one scale per
// token). Thread (cg, r_in) owns the 16-byte column group cg of rows r_in + i * kRowStep;
// mu holds its 8 channels' means (0 for Q), scale_out the head's scale row of nsc
// entries.
template <int D, int G>
__device__ __forceinline__ void qk_chunk(const uint4 *__restrict__ s_x, const float (&mu)[8],
                                         int cg, int r_in, int nrows, int row0, int chunk,
                                         float *__restrict__ scale_out, int nsc,
                                         int8_t *__restrict__ dst, const SeqLayout &L, int s,
                                         int start, int h, float (*s_red)[kThreads / 32])
{
    constexpr int kGpr = D / 8;
    constexpr int kRowStep = kThreads / kGpr;
    constexpr int kSteps = kQBlock / kRowStep;
    constexpr int kWarps = kThreads / 32;
    const int c0 = cg * 8;
    float sc[kSteps], rc[kSteps];
    if constexpr (G == 1) {
        // one scale per row: the row's kGpr 16-byte groups sit in consecutive lanes
#pragma unroll
        for (int i = 0; i < kSteps; i++) {
            const int row = i * kRowStep + r_in;
            float m = 0.0f;
            if (row < nrows) {
                float f[8];
                unpack8(s_x[row * kGpr + cg], f);
#pragma unroll
                for (int e = 0; e < 8; e++)
                    m = fmaxf(m, fabsf(__fsub_rn(f[e], mu[e])));
            }
#pragma unroll
            for (int o = 1; o < kGpr; o <<= 1)
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            sc[i] = __fdiv_rn(m, 127.0f);
            rc[i] = sc[i] != 0.0f ? __fdiv_rn(1.0f, sc[i]) : 0.0f;
            if (cg == 0 && row0 + row < nsc)
                scale_out[row0 + row] = sc[i];          // rows past the sequence: 0
        }
    } else {
        // one scale per G rows. fp32 rounding is monotonic, so the largest |fl(x - mu)| of a
        // group is max(fl(max x - mu), fl(mu - min x)) over its channels: pass 1 keeps
        // per-channel fp16 extrema only (Q: mu = 0, i.e. max |x|)
        constexpr int kGroups = kQBlock / G;
        constexpr int kStepsPerGroup = G / kRowStep;
        static_assert(G % kRowStep == 0, "a group spans whole row steps");
        const __half2 kNegInf =
            __halves2half2(__ushort_as_half(0xFC00), __ushort_as_half(0xFC00));
        const __half2 kPosInf =
            __halves2half2(__ushort_as_half(0x7C00), __ushort_as_half(0x7C00));
        __half2 hi[kGroups][4], lo[kGroups][4];
#pragma unroll
        for (int g = 0; g < kGroups; g++)
#pragma unroll
            for (int j = 0; j < 4; j++) {
                hi[g][j] = kNegInf;
                lo[g][j] = kPosInf;
            }
#pragma unroll
        for (int i = 0; i < kSteps; i++) {
            const int row = i * kRowStep + r_in;
            const int g = i / kStepsPerGroup;
            if (row < nrows) {
                const uint4 u = s_x[row * kGpr + cg];
                const __half2 *x2 = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    hi[g][j] = __hmax2(hi[g][j], x2[j]);
                    lo[g][j] = __hmin2(lo[g][j], x2[j]);
                }
            }
        }
        float am[kGroups];
#pragma unroll
        for (int g = 0; g < kGroups; g++) {
            am[g] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const float2 hf = __half22float2(hi[g][j]), lf = __half22float2(lo[g][j]);
                am[g] = fmaxf(am[g],
                              fmaxf(__fsub_rn(hf.x, mu[2 * j]), __fsub_rn(mu[2 * j], lf.x)));
                am[g] = fmaxf(am[g], fmaxf(__fsub_rn(hf.y, mu[2 * j + 1]),
                                           __fsub_rn(mu[2 * j + 1], lf.y)));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                am[g] = fmaxf(am[g], __shfl_xor_sync(0xffffffffu, am[g], o));
        }
        const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
        if (lane == 0)
#pragma unroll
            for (int g = 0; g < kGroups; g++)
                s_red[g][warp] = am[g];
        __syncthreads();
        float sg[kGroups], rg[kGroups];
#pragma unroll
        for (int g = 0; g < kGroups; g++) {
            float A = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; w++)
                A = fmaxf(A, s_red[g][w]);
            sg[g] = __fdiv_rn(A, 127.0f);
            rg[g] = sg[g] != 0.0f ? __fdiv_rn(1.0f, sg[g]) : 0.0f;
            if (threadIdx.x == 0 && chunk * kGroups + g < nsc)
                scale_out[chunk * kGroups + g] = sg[g];
        }
#pragma unroll
        for (int i = 0; i < kSteps; i++) {
            sc[i] = sg[i / kStepsPerGroup];
            rc[i] = rg[i / kStepsPerGroup];
        }
    }
    float2 nmu[4];                        // -mu (Q: -0, so that x + nmu = x exactly)
#pragma unroll
    for (int j = 0; j < 4; j++)
        nmu[j] = make_float2(-mu[2 * j], -mu[2 * j + 1]);
#pragma unroll
    for (int i = 0; i < kSteps; i++) {
        const int row = i * kRowStep + r_in;
        if (row >= nrows)
            break;
        float f[8];
        unpack8(s_x[row * kGpr + cg], f);
        float2 x[4];
#pragma unroll
        for (int j = 0; j < 4; j++)
            x[j] = add2(make_float2(f[2 * j], f[2 * j + 1]), nmu[j]);
        const uint2 w = int8_codes8(x, sc[i], rc[i]);
        *reinterpret_cast<uint2 *>(dst + L.offset(s, start, h, row0 + row) + c0) = w;
    }
}

// Codes of one 128-token chunk with per-block scales: one 128-row Q block (is_q) or two
// 64-row K blocks, the chunk already in shared memory (s_x), thread (cg, r_in) owning the
// 16-byte column group cg of rows r_in + i * kRowStep, mu its 8 channels' means (0 for
// Q). scale_row is the head's row of nsc scales. Every thread of the CTA calls it (it
// holds a CTA barrier).
template <int D>
__device__ __forceinline__ void block_codes(const uint4 *__restrict__ s_x, const float (&mu)[8],
                                            bool is_q, int cg, int r_in, int nrows, int row0,
                                            int chunk, float *__restrict__ scale_row, int nsc,
                                            int8_t *__restrict__ dst, const SeqLayout &L, int s,
                                            int start, int h, float (*s_red)[kThreads / 32])
{
    constexpr int kGpr = D / 8;
    constexpr int kRowStep = kThreads / kGpr;
    constexpr int kSteps = kQBlock / kRowStep;
    constexpr int kWarps = kThreads / 32;
    constexpr int kHalfSteps = kKBlock / kRowStep;   // steps in the first K block
    const int c0 = cg * 8;
    // Block amax (K: one per 64-row half), then codes. Pass 1 keeps per-channel fp16
    // extrema only: fp32 rounding is monotonic, so the largest |fl(x - mu)| of a block is
    // max(fl(max x - mu), fl(mu - min x)) over its channels (Q: mu = 0, i.e. max |x|).
    const __half2 kNegInf = __halves2half2(__ushort_as_half(0xFC00), __ushort_as_half(0xFC00));
    const __half2 kPosInf = __halves2half2(__ushort_as_half(0x7C00), __ushort_as_half(0x7C00));
    __half2 hi[2][4], lo[2][4];
#pragma unroll
    for (int b = 0; b < 2; b++)
#pragma unroll
        for (int j = 0; j < 4; j++) {
            hi[b][j] = kNegInf;
            lo[b][j] = kPosInf;
        }
#pragma unroll
    for (int i = 0; i < kSteps; i++) {
        const int row = i * kRowStep + r_in;
        const int b = i < kHalfSteps ? 0 : 1;
        if (row < nrows) {
            const uint4 u = s_x[row * kGpr + cg];
            const __half2 *x2 = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                hi[b][j] = __hmax2(hi[b][j], x2[j]);
                lo[b][j] = __hmin2(lo[b][j], x2[j]);
            }
        }
    }
    float am[2] = {0.0f, 0.0f};
#pragma unroll
    for (int b = 0; b < 2; b++)
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float2 hf = __half22float2(hi[b][j]), lf = __half22float2(lo[b][j]);
            am[b] = fmaxf(am[b], fmaxf(__fsub_rn(hf.x, mu[2 * j]), __fsub_rn(mu[2 * j], lf.x)));
            am[b] = fmaxf(am[b],
                          fmaxf(__fsub_rn(hf.y, mu[2 * j + 1]), __fsub_rn(mu[2 * j + 1], lf.y)));
        }
    float a0 = am[0], a1 = am[1];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, o));
        a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, o));
    }
    const int warp = (int)threadIdx.x / 32, lane = (int)threadIdx.x % 32;
    if (lane == 0) {
        s_red[0][warp] = a0;
        s_red[1][warp] = a1;
    }
    __syncthreads();
    float A0 = 0.0f, A1 = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
        A0 = fmaxf(A0, s_red[0][w]);
        A1 = fmaxf(A1, s_red[1][w]);
    }
    float sc0, sc1;
    if (is_q) {
        sc0 = sc1 = __fdiv_rn(fmaxf(A0, A1), 127.0f);
        if ((int)threadIdx.x == 0)
            scale_row[chunk] = sc0;
    } else {
        sc0 = __fdiv_rn(A0, 127.0f);
        sc1 = __fdiv_rn(A1, 127.0f);
        if ((int)threadIdx.x == 0) {
            if (2 * chunk < nsc)
                scale_row[2 * chunk] = sc0;
            if (2 * chunk + 1 < nsc)
                scale_row[2 * chunk + 1] = sc1;
        }
    }
    const float rc0 = sc0 != 0.0f ? __fdiv_rn(1.0f, sc0) : 0.0f;
    const float rc1 = sc1 != 0.0f ? __fdiv_rn(1.0f, sc1) : 0.0f;
    float2 nmu[4];                        // -mu (Q: -0, so that x + nmu = x exactly)
#pragma unroll
    for (int j = 0; j < 4; j++)
        nmu[j] = make_float2(-mu[2 * j], -mu[2 * j + 1]);
    // (unrolled by 2, not fully: the quantization kernel is sensitive to its code size;
    // full unrolling measured 0.29 ms against 0.24 ms at B2 H32 N16384 d128)
#pragma unroll 2
    for (int i = 0; i < kSteps; i++) {
        const int row = i * kRowStep + r_in;
        if (row >= nrows)
            break;
        const float scale = i < kHalfSteps ? sc0 : sc1;
        const float rcp = i < kHalfSteps ? rc0 : rc1;
        float f[8];
        unpack8(s_x[row * kGpr + cg], f);
        float2 x[4];
#pragma unroll
        for (int j = 0; j < 4; j++)
            x[j] = add2(make_float2(f[2 * j], f[2 * j + 1]), nmu[j]);
        const uint2 w = int8_codes8(x, scale, rcp);
        *reinterpret_cast<uint2 *>(dst + L.offset(s, start, h, row0 + row) + c0) = w;
    }
}

// One CTA per 128-token chunk of one (sequence, head): a Q block, a pair of K blocks or
// a V chunk. The chunk (128 rows x D fp16, 32 KB at D = 128) comes into shared memory
// with bulk copies (one for the dense layout, one per row for the packed layout) issued
// at CTA start, so every resident CTA keeps its whole chunk in flight. Thread t then
// owns the 16-byte column group t % (D/8) of rows t / (D/8) + i (256 / (D/8)), which
// makes the shared-memory reads conflict-free and fixes the thread's 8 channels.
// FINE: one Q scale per token and one K scale per 32 tokens; else per-block scales (Q:
// 128 tokens, K: 64 tokens).
// QK_ONLY: a launch without V and without the smooth-Q compensation; the V and
// compensation code is left out of it (the kernel is sensitive to its code size).
template <int D, bool FINE, bool QK_ONLY>
__global__ void __launch_bounds__(kThreads, 4) quant_kernel(
    const __half *__restrict__ q, const __half *__restrict__ k, const __half *__restrict__ v,
    ColStats cs, int8_t *__restrict__ q_i8, float *__restrict__ q_scale,
    int8_t *__restrict__ k_i8, float *__restrict__ k_scale, float *__restrict__ k_mean,
    uint8_t *__restrict__ v_e4m3, float *__restrict__ v_scale, float *__restrict__ v_mean,
    float *__restrict__ q_mean, float *__restrict__ q_comp, SeqLayout Lq, SeqLayout Lk,
    int nqc, int nkc, int *status)
{
    constexpr int kGpr = D / 8;                      // 16-byte groups per row
    constexpr int kRowStep = kThreads / kGpr;        // rows between a thread's groups
    constexpr int kSteps = kQBlock / kRowStep;       // groups per thread
    constexpr int kWarps = kThreads / 32;
    constexpr int kQG = FINE ? 1 : kQBlock;          // tokens per Q scale
    constexpr int kKG = FINE ? 32 : kKBlock;         // tokens per K scale
    __shared__ __align__(128) uint4 s_x[kQBlock * kGpr];
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ float s_red[4][kWarps];
    __shared__ float s_mu[D];             // K mean or V mean per channel
    __shared__ float s_sc[D];             // V scale per channel
    __shared__ float s_rc[D];             // fl(1 / V scale) per channel
    __shared__ float s_muq[D];            // Q mean per channel (smooth Q, K chunks)

    // 0: Q block, 1: K pair of blocks, 2: V chunk. grid.x spans the parts in order:
    // [nqc Q chunks of Lq | nkc K chunks of Lk | V chunks of Lk]; nqc or nkc is 0 when
    // that part is not quantized here.
    const int nqb = (Lq.maxlen + kQG - 1) / kQG;           // Q scales per head
    const int nkb = (Lk.maxlen + kKG - 1) / kKG;           // K scales per head
    int kind, chunk = (int)blockIdx.x;
    if (chunk < nqc) {
        kind = 0;
    } else {
        chunk -= nqc;
        kind = chunk < nkc ? 1 : 2;
        if (kind == 2)
            chunk -= nkc;
    }
    const SeqLayout &L = kind == 0 ? Lq : Lk;
    const int s = blockIdx.z, h = blockIdx.y;
    int start, len;
    if (!L.range(s, start, len, status))
        return;
    const int64_t sh = (int64_t)s * L.H + h;
    const int row0 = chunk * kQBlock;
    const int ncomp = comp_stride(Lk.maxlen);
    const bool comp = !QK_ONLY && kind == 1 && q_comp != nullptr;   // smooth-Q compensation

    if (row0 >= len) {                    // padding block of a short sequence
        if (comp && (int)threadIdx.x < kQBlock)
            q_comp[sh * ncomp + row0 + threadIdx.x] = 0.0f;
        if (kind == 0 && chunk == 0 && q_mean != nullptr && threadIdx.x < D)
            q_mean[sh * D + threadIdx.x] = 0.0f;
        if (kind == 1 && chunk == 0 && threadIdx.x < D)
            k_mean[sh * D + threadIdx.x] = 0.0f;
        if (kind == 2 && chunk == 0 && threadIdx.x < D) {   // empty sequence
            v_scale[sh * D + threadIdx.x] = 0.0f;
            if (v_mean != nullptr)
                v_mean[sh * D + threadIdx.x] = 0.0f;
        }
        if (kind != 2) {                  // the chunk's scale entries are 0
            const int G = kind == 0 ? kQG : kKG, nsc = kind == 0 ? nqb : nkb;
            float *so = (kind == 0 ? q_scale : k_scale) + sh * nsc;
            const int e = row0 / G + (int)threadIdx.x;
            if ((int)threadIdx.x < kQBlock / G && e < nsc)
                so[e] = 0.0f;
        }
        return;
    }
    const int nrows = min(kQBlock, len - row0);
    const __half *src = kind == 0 ? q : (kind == 1 ? k : v);

    // ---- the chunk into shared memory
    if (threadIdx.x == 0) {
        mbar_init(&s_bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&s_bar, (uint32_t)(nrows * D * 2));
        if (L.cu == nullptr)       // rows of one head are contiguous
            bulk_load_g2s(s_x, src + L.offset(s, start, h, row0), (uint32_t)(nrows * D * 2),
                          &s_bar);
    }
    if (L.cu != nullptr && (int)threadIdx.x < nrows)
        bulk_load_g2s(s_x + threadIdx.x * kGpr, src + L.offset(s, start, h, row0 + threadIdx.x),
                      D * 2, &s_bar);

    // ---- per-channel statistics while the copy is in flight
    // The sums come from the column-statistics kernel just before this one, which this
    // launch may overlap (programmatic dependent launch): every block that reads them
    // waits for that grid first. Plain Q blocks need nothing from it.
    if (kind != 0 || cs.qsum != nullptr)
        griddep_wait();
    if (kind == 1 && threadIdx.x < D) {
        const int c = threadIdx.x;
        const float mu = cs.ksum ? (float)(cs.ksum[sh * D + c] / (double)len) : 0.0f;
        s_mu[c] = mu;
        if (chunk == 0)
            k_mean[sh * D + c] = mu;
    }
    if (!QK_ONLY && kind == 2 && threadIdx.x < D) {
        const int c = threadIdx.x;
        const int64_t o = sh * D + c;
        const float mu = cs.vsum ? (float)(cs.vsum[o] / (double)len) : 0.0f;
        const float vmax = __uint_as_float(key_bits(cs.vhi[o]));
        const float vnegmax = __uint_as_float(key_bits(cs.vneg[o]));   // -min V
        // the largest |fl(V - mu)|: rounding is monotonic, so it is at max V or min V
        const float amax = fmaxf(__fsub_rn(vmax, mu), __fadd_rn(vnegmax, mu));
        const float sv = __fdiv_rn(amax, 448.0f);
        s_sc[c] = sv;
        s_rc[c] = sv != 0.0f ? __fdiv_rn(1.0f, sv) : 0.0f;
        s_mu[c] = mu;
        if (chunk == 0) {
            v_scale[o] = sv;
            if (v_mean != nullptr)
                v_mean[o] = mu;
        }
    }
    if (kind == 0 && threadIdx.x < D) {
        const int c = threadIdx.x;
        const float mu = cs.qsum ? (float)(cs.qsum[sh * D + c] / (double)len) : 0.0f;
        s_mu[c] = mu;
        if (chunk == 0 && q_mean != nullptr)
            q_mean[sh * D + c] = mu;
    }
    if (comp && threadIdx.x < D) {        // the Q mean of this sequence and head
        int qstart, qlen;
        float mu = 0.0f;
        if (Lq.range(s, qstart, qlen, status) && qlen > 0)
            mu = (float)(cs.qsum[sh * D + threadIdx.x] / (double)qlen);
        s_muq[threadIdx.x] = mu;
    }
    __syncthreads();

    const int cg = threadIdx.x % kGpr, r_in = threadIdx.x / kGpr;
    const int c0 = cg * 8;
    float mu[8];
#pragma unroll
    for (int e = 0; e < 8; e++)
        mu[e] = s_mu[c0 + e];

    if (!mbar_wait(&s_bar, 0, nullptr, status, status_bit(SAGE_ERR_TIMEOUT), kWaitNs))
        return;

    if (!QK_ONLY && kind == 2) {
        float sc[8], rc[8];
#pragma unroll
        for (int e = 0; e < 8; e++) {
            sc[e] = s_sc[c0 + e];
            rc[e] = s_rc[c0 + e];
        }
#pragma unroll
        for (int i = 0; i < kSteps; i++) {
            const int row = i * kRowStep + r_in;
            if (row >= nrows)
                break;
            float f[8];
            unpack8(s_x[row * kGpr + cg], f);
            float qv[8];
#pragma unroll
            for (int e = 0; e < 8; e++) {
                const float xs = __fsub_rn(f[e], mu[e]);
                qv[e] = sc[e] != 0.0f ? e4m3_quotient(xs, sc[e], rc[e]) : 0.0f;
            }
            uint2 w;
            w.x = (uint32_t)pack_e4m3x2(qv[0], qv[1]) | ((uint32_t)pack_e4m3x2(qv[2], qv[3]) << 16);
            w.y = (uint32_t)pack_e4m3x2(qv[4], qv[5]) | ((uint32_t)pack_e4m3x2(qv[6], qv[7]) << 16);
            *reinterpret_cast<uint2 *>(v_e4m3 + L.offset(s, start, h, row0 + row) + c0) = w;
        }
        return;
    }

    // ---- Q / K codes
    if constexpr (FINE) {
        if (kind == 0)
            qk_chunk<D, kQG>(s_x, mu, cg, r_in, nrows, row0, chunk, q_scale + sh * nqb, nqb, q_i8,
                             L, s, start, h, s_red);
        else
            qk_chunk<D, kKG>(s_x, mu, cg, r_in, nrows, row0, chunk, k_scale + sh * nkb, nkb, k_i8,
                             L, s, start, h, s_red);
    } else {
        // per-block scales, written out for this case (the generic qk_chunk form of it
        // measured 30% slower): one Q block, or two 64-row K blocks, per chunk
        if (kind == 0)
            block_codes<D>(s_x, mu, true, cg, r_in, nrows, row0, chunk, q_scale + sh * nqb, nqb,
                           q_i8, L, s, start, h, s_red);
        else
            block_codes<D>(s_x, mu, false, cg, r_in, nrows, row0, chunk, k_scale + sh * nkb, nkb,
                           k_i8, L, s, start, h, s_red);
    }

    // ---- smooth Q: comp[j] = mean(Q) . (K[j] - mean(K)), the smoothed K as quantized
    if (comp) {
        float muq[8];
#pragma unroll
        for (int e = 0; e < 8; e++)
            muq[e] = s_muq[c0 + e];
#pragma unroll
        for (int i = 0; i < kSteps; i++) {
            const int row = i * kRowStep + r_in;
            float dot = 0.0f;
            if (row < nrows) {
                float f[8];
                unpack8(s_x[row * kGpr + cg], f);
#pragma unroll
                for (int e = 0; e < 8; e++)
                    dot = fmaf(muq[e], __fsub_rn(f[e], mu[e]), dot);
            }
#pragma unroll
            for (int o = 1; o < kGpr; o <<= 1)   // the row's kGpr column groups
                dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (cg == 0)
                q_comp[sh * ncomp + row0 + row] = dot;   // rows past the sequence: 0
        }
    }
}


}  // namespace

cudaError_t launch_colstats(const __half *k, const __half *v, const ColStats &cs,
                            const SeqLayout &L, int *status, cudaStream_t st, bool *launched)
{
    if ((cs.ksum == nullptr && cs.vhi == nullptr) || L.maxlen == 0 || L.H == 0 || L.nseq == 0)
        return cudaSuccess;
    if (launched != nullptr)
        *launched = true;
    dim3 grid((L.maxlen + kColChunk - 1) / kColChunk, L.H, L.nseq);
    const bool dk = cs.ksum != nullptr, dv = cs.vhi != nullptr;
    if (L.d == 128) {
        if (dk && dv)
            colstats_kernel<128, true, true><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
        else if (dk)
            colstats_kernel<128, true, false><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
        else
            colstats_kernel<128, false, true><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
    } else {
        if (dk && dv)
            colstats_kernel<64, true, true><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
        else if (dk)
            colstats_kernel<64, true, false><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
        else
            colstats_kernel<64, false, true><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
    }
    return cudaGetLastError();
}


// Quantizes Q (q_i8 != nullptr), K (k_i8 != nullptr) and/or V (v_e4m3 != nullptr) in
// one launch.
cudaError_t launch_quant(const __half *q, const __half *k, const __half *v, const ColStats &cs,
                         int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                         float *k_mean, uint8_t *v_e4m3, float *v_scale, float *v_mean,
                         float *q_mean, float *q_comp, const SeqLayout &Lq,
                         const SeqLayout &Lk, bool fine, bool after_colstats, int *status,
                         cudaStream_t st)
{
    const bool with_q = q_i8 != nullptr, with_k = k_i8 != nullptr;
    const bool with_v = v_e4m3 != nullptr;
    const int nqc = with_q ? (Lq.maxlen + kQBlock - 1) / kQBlock : 0;   // 128-token chunks
    const int nkc = with_k ? (Lk.maxlen + kQBlock - 1) / kQBlock : 0;
    const int nvc = with_v ? (Lk.maxlen + kQBlock - 1) / kQBlock : 0;
    const int nx = nqc + nkc + nvc;
    if (nx == 0 || Lk.H == 0 || Lk.nseq == 0)
        return cudaSuccess;
    if (with_q && (Lq.nseq != Lk.nseq || Lq.H != Lk.H || Lq.d != Lk.d))
        return cudaErrorInvalidValue;
    dim3 grid(nx, Lk.H, Lk.nseq);
    const bool qk_only = !with_v && q_comp == nullptr;
    auto kern = Lk.d == 128
                    ? (fine ? (qk_only ? quant_kernel<128, true, true> : quant_kernel<128, true, false>)
                            : (qk_only ? quant_kernel<128, false, true> : quant_kernel<128, false, false>))
                    : (fine ? (qk_only ? quant_kernel<64, true, true> : quant_kernel<64, true, false>)
                            : (qk_only ? quant_kernel<64, false, true> : quant_kernel<64, false, false>));
    // Right after a column-statistics launch, this one may overlap its tail: the blocks
    // that read the statistics wait for it in the kernel. Anything else launched before
    // has completed by then, because the statistics kernel itself started after it.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = after_colstats ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, q, k, v, cs, q_i8, q_scale, k_i8, k_scale, k_mean,
                              v_e4m3, v_scale, v_mean, q_mean, q_comp, Lq, Lk, nqc, nkc, status);
}

}  // namespace sage
