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
//   quant:    one CTA per 128-token chunk of Q (one Q block), K (two K blocks) or V;
//             16-byte vector loads/stores, warp-shuffle amax. Codes are the rounding of
//             the IEEE fp32 quotient x / scale, computed as x * (1 / scale) with an exact
//             division only where the two could round differently, so they match the
//             definition bit for bit without a division per element.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "sage_common.cuh"
#include "sm100_ptx.cuh"

namespace sage {

namespace {

constexpr int kColChunk = 512;   // tokens per colstats CTA
constexpr int kThreads = 256;

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8])
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 t = __half22float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads) colstats_kernel(const __half *__restrict__ k,
                                                            const __half *__restrict__ v,
                                                            ColStats cs, SeqLayout L, int *status)
{
    constexpr int kGroups = D / 8;              // 16-byte column groups per row
    constexpr int kRowsPerPass = kThreads / kGroups;
    constexpr int kWarps = kThreads / 32;
    const int s = blockIdx.z, h = blockIdx.y;
    int start, len;
    if (!L.range(s, start, len, status))
        return;
    const int r_begin = blockIdx.x * kColChunk;
    if (r_begin >= len)
        return;
    const int r_end = min(len, r_begin + kColChunk);
    const int g = threadIdx.x % kGroups, r0 = threadIdx.x / kGroups;
    const bool do_k = cs.ksum != nullptr, do_v = cs.vhi != nullptr, do_vsum = cs.vsum != nullptr;

    double ks[8], vs[8];
    float hi[8], ng[8];                          // max V and max -V
#pragma unroll
    for (int i = 0; i < 8; i++) {
        ks[i] = vs[i] = 0.0;
        hi[i] = ng[i] = -INFINITY;
    }
    for (int r = r_begin + r0; r < r_end; r += kRowsPerPass) {
        const int64_t off = L.offset(s, start, h, r) + g * 8;
        float f[8];
        if (do_k) {
            unpack8(__ldg(reinterpret_cast<const uint4 *>(k + off)), f);
#pragma unroll
            for (int i = 0; i < 8; i++)
                ks[i] += (double)f[i];
        }
        if (do_v) {
            unpack8(__ldg(reinterpret_cast<const uint4 *>(v + off)), f);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                hi[i] = fmaxf(hi[i], f[i]);
                ng[i] = fmaxf(ng[i], -f[i]);
                if (do_vsum)
                    vs[i] += (double)f[i];
            }
        }
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

// Block-wide max over `nthreads` consecutive threads starting at warp `w0`.
template <int NWARPS>
__device__ __forceinline__ float group_max(float x, float *s_red, int w0)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0)
        s_red[warp] = x;
    __syncthreads();
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < NWARPS; i++)
        m = fmaxf(m, s_red[w0 + i]);
    return m;
}

constexpr float kRound = 12582912.0f;            // 1.5 * 2^23: adding it rounds to an integer
constexpr int kRoundBits = 0x4B400000;

// round-half-even(fl(x / s)) clamped to [-127, 127], where fl(x / s) is the IEEE fp32
// quotient and r = fl(1 / s). The product x * r is within 2^-15 of fl(x / s) (|x / s| <=
// 127.5 keeps every ulp <= 2^-17), so both round to the same integer unless the product
// lies within 2^-15 of a half-integer; those rare elements take the exact division.
__device__ __forceinline__ int8_t int8_code(float x, float s, float r)
{
    if (s == 0.0f)
        return 0;
    const float q = x * r;
    const float b = q + kRound;                    // RNE integer in the low mantissa bits
    const float d = fabsf(q - (b - kRound));       // distance to that integer, <= 1/2
    int c = __float_as_int(b) - kRoundBits;
    if (d > 0.5f - 3.0517578125e-05f)              // near a tie: exact IEEE quotient
        c = __float2int_rn(__fdiv_rn(x, s));
    c = max(-127, min(127, c));
    return (int8_t)c;
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

template <int D>
__global__ void __launch_bounds__(kThreads) quant_kernel(
    const __half *__restrict__ q, const __half *__restrict__ k, const __half *__restrict__ v,
    ColStats cs, int8_t *__restrict__ q_i8, float *__restrict__ q_scale,
    int8_t *__restrict__ k_i8, float *__restrict__ k_scale, float *__restrict__ k_mean,
    uint8_t *__restrict__ v_e4m3, float *__restrict__ v_scale, float *__restrict__ v_mean,
    SeqLayout L, int nqb, int nkb, int part0, int *status)
{
    constexpr int kHalf = D / 2;          // elements per thread (two threads per token)
    constexpr int kVec = kHalf / 8;       // 16-byte loads per thread
    __shared__ float s_red[8];
    __shared__ float s_aux[D];            // K mean or V scale per channel
    __shared__ float s_rcp[D];            // fl(1 / V scale) per channel
    __shared__ float s_vmu[D];            // V mean per channel (0 without smooth V)
    const double *ksum = cs.ksum;

    const int s = blockIdx.z, h = blockIdx.y;
    int start, len;
    if (!L.range(s, start, len, status))
        return;
    const int64_t sh = (int64_t)s * L.H + h;
    // 0: Q block, 1: K pair of blocks, 2: V chunk; grid.x spans consecutive parts
    const int kind = part0 + (int)blockIdx.x / nqb;
    const int chunk = (int)blockIdx.x % nqb;
    const int row0 = chunk * kQBlock;
    const int row = row0 + threadIdx.x / 2;
    const int col0 = (threadIdx.x & 1) * kHalf;
    const bool valid = row < len;

    if (row0 >= len) {                    // padding block of a short sequence
        if (kind == 1 && chunk == 0 && threadIdx.x < D)
            k_mean[sh * D + threadIdx.x] = 0.0f;
        if (kind == 2 && chunk == 0 && threadIdx.x < D) {   // empty sequence
            v_scale[sh * D + threadIdx.x] = 0.0f;
            if (v_mean != nullptr)
                v_mean[sh * D + threadIdx.x] = 0.0f;
        }
        if (threadIdx.x == 0) {
            if (kind == 0)
                q_scale[sh * nqb + chunk] = 0.0f;
            if (kind == 1) {
                if (2 * chunk < nkb)
                    k_scale[sh * nkb + 2 * chunk] = 0.0f;
                if (2 * chunk + 1 < nkb)
                    k_scale[sh * nkb + 2 * chunk + 1] = 0.0f;
            }
        }
        return;
    }

    if (kind == 1 && threadIdx.x < D) {
        const int c = threadIdx.x;
        const float mu = ksum ? (float)(ksum[sh * D + c] / (double)len) : 0.0f;
        s_aux[c] = mu;
        if (chunk == 0)
            k_mean[sh * D + c] = mu;
    }
    if (kind == 2 && threadIdx.x < D) {
        const int c = threadIdx.x;
        const int64_t o = sh * D + c;
        const float mu = cs.vsum ? (float)(cs.vsum[o] / (double)len) : 0.0f;
        const float vmax = __uint_as_float(key_bits(cs.vhi[o]));
        const float vnegmax = __uint_as_float(key_bits(cs.vneg[o]));   // -min V
        // the largest |fl(V - mu)|: rounding is monotonic, so it is at max V or min V
        const float amax = fmaxf(__fsub_rn(vmax, mu), __fadd_rn(vnegmax, mu));
        const float sv = __fdiv_rn(amax, 448.0f);
        s_aux[c] = sv;
        s_rcp[c] = sv != 0.0f ? __fdiv_rn(1.0f, sv) : 0.0f;
        s_vmu[c] = mu;
        if (chunk == 0) {
            v_scale[o] = sv;
            if (v_mean != nullptr)
                v_mean[o] = mu;
        }
    }
    __syncthreads();

    const int64_t off = L.offset(s, start, h, row) + col0;
    const __half *src = kind == 0 ? q : (kind == 1 ? k : v);
    float x[kHalf];
#pragma unroll
    for (int i = 0; i < kVec; i++) {
        float f[8];
        if (valid)
            unpack8(__ldg(reinterpret_cast<const uint4 *>(src + off) + i), f);
        else
#pragma unroll
            for (int e = 0; e < 8; e++)
                f[e] = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; e++)
            x[i * 8 + e] = f[e];
    }

    if (kind == 2) {
        // E4M3 codes with the per-channel scale
        if (!valid)
            return;
        uint32_t w[kHalf / 4];
#pragma unroll
        for (int i = 0; i < kHalf; i += 4) {
            float qv[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int c = col0 + i + e;
                const float sv = s_aux[c];
                const float xs = __fsub_rn(x[i + e], s_vmu[c]);
                qv[e] = sv != 0.0f ? e4m3_quotient(xs, sv, s_rcp[c]) : 0.0f;
            }
            const uint32_t lo = pack_e4m3x2(qv[0], qv[1]);
            const uint32_t hi = pack_e4m3x2(qv[2], qv[3]);
            w[i / 4] = lo | (hi << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(v_e4m3 + off);
#pragma unroll
        for (int i = 0; i < kHalf / 16; i++)
            dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        return;
    }

    float amax = 0.0f;
    if (kind == 1) {
#pragma unroll
        for (int i = 0; i < kHalf; i++)
            x[i] = __fsub_rn(x[i], s_aux[col0 + i]);
    }
    if (valid) {
#pragma unroll
        for (int i = 0; i < kHalf; i++)
            amax = fmaxf(amax, fabsf(x[i]));
    }

    float scale;
    if (kind == 0) {
        scale = __fdiv_rn(group_max<8>(amax, s_red, 0), 127.0f);
        if (threadIdx.x == 0)
            q_scale[sh * nqb + chunk] = scale;
    } else {
        const int half_blk = threadIdx.x / 128;    // 64-token K block within the chunk
        scale = __fdiv_rn(group_max<4>(amax, s_red, half_blk * 4), 127.0f);
        const int kb = 2 * chunk + half_blk;
        if ((threadIdx.x & 127) == 0 && kb < nkb)
            k_scale[sh * nkb + kb] = scale;
    }
    if (!valid)
        return;

    const float rcp = scale != 0.0f ? __fdiv_rn(1.0f, scale) : 0.0f;
    uint32_t w[kHalf / 4];
#pragma unroll
    for (int i = 0; i < kHalf; i += 4) {
        const uint32_t b0 = (uint8_t)int8_code(x[i], scale, rcp);
        const uint32_t b1 = (uint8_t)int8_code(x[i + 1], scale, rcp);
        const uint32_t b2 = (uint8_t)int8_code(x[i + 2], scale, rcp);
        const uint32_t b3 = (uint8_t)int8_code(x[i + 3], scale, rcp);
        w[i / 4] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
    int8_t *dst8 = (kind == 0 ? q_i8 : k_i8) + off;
    uint4 *dst = reinterpret_cast<uint4 *>(dst8);
#pragma unroll
    for (int i = 0; i < kHalf / 16; i++)
        dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

}  // namespace

cudaError_t launch_colstats(const __half *k, const __half *v, const ColStats &cs,
                            const SeqLayout &L, int *status, cudaStream_t st)
{
    if (cs.ksum == nullptr && cs.vhi == nullptr)
        return cudaSuccess;
    dim3 grid((L.maxlen + kColChunk - 1) / kColChunk, L.H, L.nseq);
    if (L.d == 128)
        colstats_kernel<128><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
    else
        colstats_kernel<64><<<grid, kThreads, 0, st>>>(k, v, cs, L, status);
    return cudaGetLastError();
}

cudaError_t launch_quant(const __half *q, const __half *k, const __half *v, const ColStats &cs,
                         int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                         float *k_mean, uint8_t *v_e4m3, float *v_scale, float *v_mean,
                         const SeqLayout &L, int *status, cudaStream_t st)
{
    const int nqb = (L.maxlen + kQBlock - 1) / kQBlock;
    const int nkb = (L.maxlen + kKBlock - 1) / kKBlock;
    const int part0 = q_i8 != nullptr ? 0 : 2;
    const int part1 = v_e4m3 != nullptr ? 3 : 2;
    if (part1 <= part0)
        return cudaSuccess;
    dim3 grid(nqb * (part1 - part0), L.H, L.nseq);
    if (L.d == 128)
        quant_kernel<128><<<grid, kThreads, 0, st>>>(q, k, v, cs, q_i8, q_scale, k_i8, k_scale,
                                                     k_mean, v_e4m3, v_scale, v_mean, L, nqb,
                                                     nkb, part0, status);
    else
        quant_kernel<64><<<grid, kThreads, 0, st>>>(q, k, v, cs, q_i8, q_scale, k_i8, k_scale,
                                                    k_mean, v_e4m3, v_scale, v_mean, L, nqb,
                                                    nkb, part0, status);
    return cudaGetLastError();
}

}  // namespace sage
