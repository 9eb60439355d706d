// K-ATTN: the fused quantized attention pass for sm_100a.
//
// Method (「SageAttention：低比特量化Attention，实现推理加速」, section 技术方案;
// 「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案 (3)-(4)):
// S = Q_i8 K_i8^T with INT32 accumulation, dequantized by q_scale * k_scale * sm_scale,
// FlashAttention online softmax over 128-key tiles, and P.V with P, V in FP16 (FP16
// mode) or both in E4M3 (FP8 mode); each tile's P.V is a fresh tensor-core product
// added into an fp32 accumulator across tiles.
//
// B200 design. One CTA owns NQT = 2 query tiles of 128 rows of one (sequence, head) and
// walks the KV tiles once for both, so each K/V tile read from L2 feeds 256 rows:
//   warps 0-3 / 4-7   softmax warpgroups, one per query tile; thread t owns row t
//                     (TMEM lane t)
//   warp 8            TMA producer: Q tiles once, then K/V tiles into a STAGES-deep
//                     shared-memory ring (mbarrier full/empty pairs); the whole warp
//                     runs the loop, one elected lane issues each copy
//   warp 9            MMA issuer and TMEM owner (the whole warp runs the issue loop,
//                     one elected lane issues each MMA):
//                       S_i  = Q_i K^T    tcgen05.mma kind::i8, smem x smem -> TMEM s32
//                       O_i += P_i V      tcgen05.mma kind::f16 | kind::f8f6f4, P from
//                                         TMEM, V from shared memory (MN-major) -> f32
//   warps 10-11       idle (complete the warpgroup for the register split)
// TMEM columns: [S | O_0 | O_1 | P_0 | P_1] = 128 + 2d + 2 * (64 | 32) <= 512: the two
// query tiles take turns in one S region (S_1(j) is computed once S_0(j) has been read,
// S_0(j+1) once S_1(j) has); P is 64 columns per tile in FP16 mode, 32 in FP8 mode.
//
// Per tile, a softmax thread reads its 128 scores from TMEM into registers once and
// releases S at once, so the tensor core computes the next scores while the
// exponentials of this tile run. It takes the integer max of each K scale group (each
// has its own scale), converts S to fp32 exactly with a magic-number bias, forms
// p = 2^(S*sc - m) with one packed FFMA + ex2, and writes P (f16, or E4M3 of 448 p)
// into TMEM, where the P.V MMA reads it as its A operand. O lives in TMEM; a row's O is
// rescaled in place only when its reference max m moves (in FP16 mode only when the
// max grows by more than 2^8, so P <= 256; in FP8 mode on every increase, so 448 P fits
// E4M3).
//
// Every wait is bounded (global timer); a timeout sets the device status word, all
// roles drain and the CTA releases TMEM and exits. Nothing traps.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <type_traits>
#include <cstdio>
#include <mutex>

#include "quant_codes.cuh"
#include "sage_common.cuh"
#include "sm100_ptx.cuh"

namespace sage {

namespace {

constexpr uint64_t kTimeoutNs = 2000000000ull;   // 2 s: far above any legitimate wait
// The producer and MMA warps poll with a 1 us suspend hint: they share SM sub-partitions
// 0 and 1 with softmax warps, whose issue slots a hot poll takes (same-box A/B: FP16
// +1.5%, FP8 +0.9% at the headline; 100 us measured no better).
constexpr uint32_t kPollSleepNs = 1000;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448): E4M3 P = e4m3(448 p)


template <int D, bool FP8, int NQT, bool SQ = false>
struct Cfg {
    static constexpr int BM = 128, BN = 128;
    static constexpr int kQBytes = BM * D;                   // int8 Q tile
    static constexpr int kKBytes = BN * D;                   // int8 K tile
    static constexpr int kVBytes = BN * D * (FP8 ? 1 : 2);   // V tile
    // P lives in TMEM and P.V takes its A operand from there, so P.V reads only V from
    // shared memory and P never enters it (P in shared memory measured 6% slower in FP16
    // mode and 13% in FP8 mode at d = 128). To make room for P at d = 128, the two query
    // tiles' scores share one S region: S_1(j) is computed once S_0(j) has been read,
    // S_0(j+1) once S_1(j) has. That also keeps the two softmax warpgroups half a tile
    // apart, so it is used at d = 64 as well (1-5% faster there than an S region each).
    static_assert(NQT == 2, "two query tiles per CTA");
    static constexpr int kSCols = BN;                             // TMEM columns of S
    static constexpr int kPCols = BN * (FP8 ? 1 : 2) / 4;        // TMEM columns of a P tile
    // smooth Q: each stage also holds the 128 fp32 score compensations of its keys
    static constexpr int kCompBytes = SQ ? BN * 4 : 0;
    static constexpr int kStageBytes = kKBytes + kVBytes + kCompBytes;
    static constexpr int kBudget = 220 * 1024;
    static constexpr int kStagesFit = (kBudget - NQT * kQBytes) / kStageBytes;
    static constexpr int STAGES = kStagesFit > 4 ? 4 : kStagesFit;
    static_assert(STAGES >= 2, "shared-memory ring too shallow");
    static constexpr int kSoftmaxWarps = 4 * NQT;
    static constexpr int kProducerWarp = kSoftmaxWarps;
    static constexpr int kMmaWarp = kSoftmaxWarps + 1;
    static constexpr int kThreads = (kSoftmaxWarps + 4) * 32;
    static constexpr int kTmemNeed = kSCols + NQT * (D + kPCols);
    static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
    static_assert(kTmemNeed <= 512, "TMEM budget exceeded");
    // Registers: the kernel launches with kLaunchRegs per thread (65536 / 384, rounded
    // down to a multiple of 8); setmaxnreg then moves them from the producer, MMA and idle
    // warps to the softmax warps. The split draws only on the block's own registers, so
    // the totals must match (the host checks kLaunchRegs against the compiled kernel).
    static constexpr int kLaunchRegs = 168;
    static constexpr int kRegSoftmax = FP8 ? 208 : 216;   // measured best per P.V mode
    static constexpr int kRegOther = FP8 ? 88 : 72;
    static_assert((kSoftmaxWarps * kRegSoftmax + 4 * kRegOther) * 32 <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
    // shared memory map (offsets from a 1024-byte aligned base)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + NQT * kQBytes;
    static constexpr int kOffV = kOffK + STAGES * kKBytes;
    static constexpr int kOffB = kOffV + STAGES * kVBytes;
    // in-kernel Q quantization: per warpgroup 4 warp maxima + D channel means (fp32)
    static constexpr int kOffScr = kOffB + STAGES * kCompBytes;
    static constexpr int kOffBar = kOffScr + NQT * (4 + D) * 4;
    // barriers: q, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[NQT],
    //           p_full[NQT], pv_full[NQT], s_free, drain
    static constexpr int kNumBars = 1 + 4 * STAGES + 3 * NQT + 2;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    // V operand geometry (MN-major): bytes per token row inside one swizzle chunk
    static constexpr int kVElem = FP8 ? 1 : 2;
    static constexpr int kVRowBytes = (D * kVElem) >= 128 ? 128 : D * kVElem;
    static constexpr int kVChunks = (D * kVElem) / kVRowBytes;          // boxes per V tile
    static constexpr int kVBoxBytes = BN * kVRowBytes;
    static constexpr int kPvK = FP8 ? 32 : 16;                          // K per PV MMA
    // Q/K operand geometry (K-major, one swizzle atom wide)
    static constexpr int kQkSwizzle = D == 128 ? 2 : 4;                 // 128B / 64B
    static constexpr int kQkSbo = 8 * D;                                 // 8 rows
    static constexpr int kVSwizzle = kVRowBytes == 128 ? 2 : 4;
    static constexpr int kVSbo = 8 * kVRowBytes;
    // The reference max of a row is refreshed only when the row max exceeds it by more
    // than this (log2 units): FP16 P then stays <= 2^8, far inside fp16. FP8 mode keeps
    // P <= 1 so that 448 P fits E4M3.
    static constexpr float kRescaleSlack = FP8 ? 0.0f : 8.0f;
};

struct KParams {
    const float *q_scale;
    const float *k_scale;
    const float *v_scale;
    const float *v_mean;   // FP8 with smooth V: added to every output row; else nullptr
    const float *q_comp;   // smooth Q: score compensation per key; else nullptr
    int ncomp;             // row stride of q_comp (whole 128-key tiles)
    __half *out;
    int32_t *s_dump;
    SeqLayout L;         // queries (and the output)
    SeqLayout LK;        // keys and values (L again for self-attention)
    int nqb, nkb;        // scales per (sequence, head) row of the scale arrays
    int causal;
    float sc_log2;       // sm_scale * log2(e)
    int *status;
    const __half *q16;   // QIN: fp16 Q, quantized in the prologue
    const double *qsum;  // QIN with smooth Q: fp64 column sums of Q
};

__device__ __forceinline__ void tma_coords(const SeqLayout &L, int s, int start, int h, int row,
                                           int &c1, int &c2)
{
    if (L.cu == nullptr) {
        c1 = row;
        c2 = s * L.H + h;
    } else {
        c1 = h;
        c2 = start + row;
    }
}

// Bit e set iff key e of a 32-key chunk is visible, given `n` visible keys from the
// chunk start.
__device__ __forceinline__ uint32_t chunk_mask(int n)
{
    return n >= 32 ? ~0u : (n <= 0 ? 0u : (1u << n) - 1u);
}

// Every lane polls the barrier (the warp stays converged, as the .sync.aligned tcgen05
// operations that follow require) and a vote makes a timeout seen by any lane the whole
// warp's outcome. Polling from lane 0 alone and broadcasting the result with a shuffle
// measured 3-6% slower over the whole kernel.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          int *status)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status,
                                             status_bit(SAGE_ERR_TIMEOUT), kTimeoutNs));
}

// A softmax warp's arrival on a barrier (after __syncwarp): one elected lane in FP16 mode;
// lane 0 under a branch in FP8 mode (same-box A/B: FP16 +1.5-2.5%, FP8 -4% with elect).
template <bool FP8>
__device__ __forceinline__ void warp_arrive(uint64_t *bar)
{
    if constexpr (FP8) {
        if ((threadIdx.x & 31) == 0)
            mbar_arrive(bar);
    } else {
        mbar_arrive_w(bar);
    }
}

// The INT8 codes and the scale of this thread's query row (QIN): Q is read as fp16, made
// smooth (x - mean(Q), SQ), and quantized with one scale per 128-row tile (the
// warpgroup's amax) or per row (FINE) exactly as the quantization kernel does it; the
// codes go to the Q tile in shared memory in the layout its TMA copy would give (rows of
// D bytes, 16-byte chunks XOR-swizzled by the row: 128-byte swizzle for D = 128, 64-byte
// for D = 64). scratch: this warpgroup's 4 + D floats of shared memory. Returns the
// row's scale (0 for rows past the sequence, and for a tile with no row in it).
template <int D, bool FINE, bool SQ>
__device__ __forceinline__ float quantize_q_row(const __half *__restrict__ src, bool valid,
                                                const double *__restrict__ qsum, int len,
                                                uint8_t *tile, int row, int i, float *scratch)
{
    const int quarter = row / 32, lane = row % 32;
    float *s_amax = scratch;          // one per warp
    float *s_mu = scratch + 4;        // mean(Q) per channel
    if constexpr (SQ) {
        for (int c = row; c < D; c += 128)
            s_mu[c] = (float)(qsum[c] / (double)len);
        named_bar_sync(1 + i, 128);
    }
    uint4 raw[D / 8];
#pragma unroll
    for (int g = 0; g < D / 8; g++)
        raw[g] = valid ? __ldg(reinterpret_cast<const uint4 *>(src) + g) : make_uint4(0, 0, 0, 0);
    // amax |fl(x - mu)| over the row (mu = 0 without smooth Q: max |x|, exact)
    float amax = 0.0f;
#pragma unroll
    for (int g = 0; g < D / 8; g++) {
        float f[8];
        unpack8(raw[g], f);
#pragma unroll
        for (int e = 0; e < 8; e++)
            amax = fmaxf(amax, fabsf(SQ ? __fsub_rn(f[e], s_mu[g * 8 + e]) : f[e]));
    }
    if (!valid)
        amax = 0.0f;
    if constexpr (!FINE) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0)
            s_amax[quarter] = amax;
        named_bar_sync(1 + i, 128);
        amax = fmaxf(fmaxf(s_amax[0], s_amax[1]), fmaxf(s_amax[2], s_amax[3]));
    }
    const float scale = __fdiv_rn(amax, 127.0f);
    const float rcp = scale != 0.0f ? __fdiv_rn(1.0f, scale) : 0.0f;
    const uint32_t base = smem_u32(tile) + row * D;
#pragma unroll
    for (int c = 0; c < D / 16; c++) {      // 16 codes = one 16-byte chunk
        uint2 w[2];
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
            const int g = 2 * c + hh;
            float f[8];
            unpack8(raw[g], f);
            float2 x[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                x[e] = make_float2(f[2 * e], f[2 * e + 1]);
                if constexpr (SQ)
                    x[e] = make_float2(__fsub_rn(x[e].x, s_mu[g * 8 + 2 * e]),
                                       __fsub_rn(x[e].y, s_mu[g * 8 + 2 * e + 1]));
            }
            w[hh] = valid ? int8_codes8(x, scale, rcp) : make_uint2(0u, 0u);
        }
        const int sw = D == 128 ? (row & 7) : ((row >> 1) & 3);
        st_shared_v4(base + ((c ^ sw) << 4), w[0].x, w[0].y, w[1].x, w[1].y);
    }
    return valid || !FINE ? scale : 0.0f;
}

// FINE: one Q scale per query row and one K scale per 32 keys; else one Q scale per
// 128-row tile and one K scale per 64 keys. SQ: smooth Q, the score of key j gets the
// compensation mean(Q) K_j^T (p.q_comp), loaded with V into each stage. QIN: the CTA
// quantizes its own Q tiles from fp16 (p.q16) instead of loading INT8 codes.
template <int D, bool FP8, int NQT, bool DUMP, bool FINE, bool SQ, bool QIN>
__global__ void __launch_bounds__(Cfg<D, FP8, NQT, SQ>::kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const KParams p)
{
    using C = Cfg<D, FP8, NQT, SQ>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);

    const SeqLayout &L = p.L;
    const SeqLayout &LK = p.LK;
    const int s = blockIdx.z, h = blockIdx.y;
    int start, len, kstart, klen;
    if (!L.range(s, start, len, p.status) || !LK.range(s, kstart, klen, p.status))
        return;
    const int cta_x = p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
    const int qt0 = cta_x * NQT;
    if (qt0 * C::BM >= len)
        return;                                    // whole CTA beyond this sequence
    const int last_row = min(len, (qt0 + NQT) * C::BM) - 1;
    // causal: query i sees keys j <= i + koff (bottom-right aligned; koff = 0 when the
    // queries and keys are the same sequence)
    const int koff = klen - len;
    const int nkt = (klen + C::BN - 1) / C::BN;
    const int nkv = !p.causal ? nkt : (last_row + koff < 0 ? 0 : min(nkt, (last_row + koff) / C::BN + 1));
    if (nkv == 0) {
        // no query row of this CTA sees a key: its output rows are zero
        const int r0 = qt0 * C::BM, nrow = last_row + 1 - r0;
        for (int idx = threadIdx.x; idx < nrow * (D / 8); idx += blockDim.x) {
            const int r = r0 + idx / (D / 8);
            *reinterpret_cast<uint4 *>(p.out + L.offset(s, start, h, r) + (idx % (D / 8)) * 8) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        return;
    }

    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;
    [[maybe_unused]] const float *sB = reinterpret_cast<const float *>(smem + C::kOffB);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *bar_q = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *k_empty = k_full + C::STAGES;
    uint64_t *v_full = k_empty + C::STAGES;
    uint64_t *v_empty = v_full + C::STAGES;
    uint64_t *s_full = v_empty + C::STAGES;
    uint64_t *p_full = s_full + NQT;
    uint64_t *pv_full = p_full + NQT;
    uint64_t *s_free = pv_full + NQT;      // S read into registers: the S region is free
    uint64_t *bar_drain = s_free + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        mbar_init(bar_q, QIN ? C::kSoftmaxWarps : 1);
        for (int i = 0; i < C::STAGES; i++) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < NQT; i++) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_full[i], 1);
        }
        mbar_init(s_free, 4);   // the 4 warps of the warpgroup that read S
        mbar_init(bar_drain, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == C::kMmaWarp)
        tmem_alloc(tmem_slot, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < C::kSoftmaxWarps) {
        // ------------------------------------------------------------ softmax warps
        if constexpr (NQT == 2)
            asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(C::kRegSoftmax) : "memory");
        const int i = warp / 4;                    // query tile within the CTA
        const int quarter = warp % 4;              // TMEM lane quarter of this warp
        const int qt = qt0 + i;
        const int row_in_tile = quarter * 32 + lane;
        const int qrow = qt * C::BM + row_in_tile;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem_base + lane_off;   // the shared S region
        const uint32_t tO = tmem_base + lane_off + C::kSCols + i * D;
        [[maybe_unused]] const uint32_t tP =
            tmem_base + lane_off + C::kSCols + NQT * D + i * C::kPCols;
        const int64_t sh = (int64_t)s * L.H + h;
        // this row's Q scale (one per query tile, or one per token)
        float qsc;
        if constexpr (QIN) {
            // quantize this row into Q tile i, then tell the MMA issuer (bar_q counts the
            // softmax warps)
            qsc = quantize_q_row<D, FINE, SQ>(
                      p.q16 + L.offset(s, start, h, qrow < len ? qrow : 0), qrow < len,
                      SQ ? p.qsum + sh * D : nullptr, len, smem + C::kOffQ + i * C::kQBytes,
                      row_in_tile, i,
                      reinterpret_cast<float *>(smem + C::kOffScr + i * (4 + D) * 4)) *
                  p.sc_log2;
            fence_proxy_async_smem();
            __syncwarp();
            warp_arrive<FP8>(bar_q);
        } else {
            const int qidx = FINE ? qrow : qt;
            const bool q_valid = (FINE ? qrow : qt * C::BM) < len;
            qsc = (q_valid ? __ldg(p.q_scale + sh * p.nqb + qidx) : 0.0f) * p.sc_log2;
        }
        constexpr int kKGroups = FINE ? 4 : 2;        // K scales per 128-key tile
        const int kb_valid = (klen + C::BN / kKGroups - 1) / (C::BN / kKGroups);

        // m_ref: the max that P is taken relative to; it moves only when the row max
        // exceeds it by more than kRescaleSlack (0 in FP8 mode, so P <= 1 and 448 P fits E4M3)
        float m_ref = -INFINITY, l = 0.0f;
        bool ok = true;

        for (int j = 0; j < nkv && ok; j++) {
            if (!(ok = warp_wait(&s_full[i], j & 1, abort, p.status)))
                break;
            tc_fence_after();
            // dequantization factor of each K scale group of the tile
            float sck[kKGroups];
#pragma unroll
            for (int c = 0; c < kKGroups; c++) {
                const int kb = kKGroups * j + c;
                sck[c] = qsc * (kb < kb_valid ? __ldg(p.k_scale + sh * p.nkb + kb) : 0.0f);
            }
            const int kcol0 = j * C::BN;
            const bool need_mask =
                (kcol0 + C::BN > klen) || (p.causal && kcol0 + C::BN - 1 > qt * C::BM + koff);
            // keys < col_lim are visible to this row
            const int col_lim = p.causal ? min(klen, qrow + 1 + koff) : klen;

            // the whole 128-key score row into registers (one TMEM pass)
            uint32_t sreg[4][32];
#pragma unroll
            for (int ch = 0; ch < 4; ch++)
                tmem_ld32_async(tS + ch * 32, sreg[ch]);
#pragma unroll
            for (int ch = 0; ch < 4; ch++)
                tmem_ld_wait(sreg[ch]);
            if constexpr (DUMP) {
                if (qrow < len) {
                    int32_t *drow = p.s_dump + (sh * L.maxlen + qrow) * LK.maxlen;
                    for (int e = 0; e < C::BN; e++)
                        if (kcol0 + e < klen)
                            drow[kcol0 + e] = static_cast<int>(sreg[e / 32][e % 32]);
                }
            }
            // S_i is in registers: the tensor core may write the other tile's scores now
            tc_fence_before();
            __syncwarp();
            warp_arrive<FP8>(s_free);
            // smooth Q: this tile's score compensations arrive with V(j); the stage is not
            // refilled before P.V(j), which needs this tile's P first
            [[maybe_unused]] const float *bt = sB + (j % C::STAGES) * C::BN;
            if constexpr (SQ) {
                if (!(ok = warp_wait(&v_full[j % C::STAGES], (j / C::STAGES) & 1, abort,
                                     p.status)))
                    break;
            }

            // Score math of one tile, in two steps around the wait for the previous P.V.
            // Only the diagonal (causal) and the ragged last tile need the per-key
            // visibility mask; every other tile takes the MASKED = false instantiation.
            float alpha = 1.0f, bias = 0.0f;
            auto tile_max = [&](auto masked) {
                constexpr bool MASKED = decltype(masked)::value;
                float tmax = -INFINITY;
                if constexpr (SQ) {
                    // u = S sc + comp c, in place of S; its exact max (the compensation
                    // varies along the row, so the integer max no longer orders it)
                    const float cq = p.sc_log2;
#pragma unroll
                    for (int ch = 0; ch < 4; ch++) {
                        const uint32_t keep =
                            MASKED ? chunk_mask(col_lim - kcol0 - ch * 32) : ~0u;
                        const float sc = sck[ch * kKGroups / 4];
                        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 b4 = *reinterpret_cast<const float4 *>(bt + ch * 32 + e);
#pragma unroll
                            for (int hh = 0; hh < 2; hh++) {
                                float2 x = make_float2(magic_biased(sreg[ch][e + 2 * hh]),
                                                       magic_biased(sreg[ch][e + 2 * hh + 1]));
                                x = add2(x, make_float2(-kMagic, -kMagic));      // exact S
                                const float2 bc = mul2(hh ? make_float2(b4.z, b4.w)
                                                          : make_float2(b4.x, b4.y),
                                                       make_float2(cq, cq));
                                float2 u = fma2(x, make_float2(sc, sc), bc);
                                if constexpr (MASKED) {
                                    u.x = ((keep >> (e + 2 * hh)) & 1u) ? u.x : -INFINITY;
                                    u.y = ((keep >> (e + 2 * hh + 1)) & 1u) ? u.y : -INFINITY;
                                }
                                sreg[ch][e + 2 * hh] = __float_as_uint(u.x);
                                sreg[ch][e + 2 * hh + 1] = __float_as_uint(u.y);
                                mx[hh] = fmaxf(mx[hh], fmaxf(u.x, u.y));
                            }
                        }
                        tmax = fmaxf(tmax, fmaxf(mx[0], mx[1]));
                    }
                } else {
                // integer maxima of the K scale groups (each has its own scale)
                int im[kKGroups];
#pragma unroll
                for (int c = 0; c < kKGroups; c++)
                    im[c] = INT_MIN;
#pragma unroll
                for (int ch = 0; ch < 4; ch++) {
                    const uint32_t keep = MASKED ? chunk_mask(col_lim - kcol0 - ch * 32) : ~0u;
                    int mx[4] = {INT_MIN, INT_MIN, INT_MIN, INT_MIN};
#pragma unroll
                    for (int e = 0; e < 32; e++) {
                        const int v = static_cast<int>(sreg[ch][e]);
                        if constexpr (MASKED)
                            mx[e & 3] = ((keep >> e) & 1u) ? max(mx[e & 3], v) : mx[e & 3];
                        else
                            mx[e & 3] = max(mx[e & 3], v);
                    }
                    const int g = ch * kKGroups / 4;      // the 32 columns' K group
                    im[g] = max(im[g], max(max(mx[0], mx[1]), max(mx[2], mx[3])));
                }
#pragma unroll
                for (int c = 0; c < kKGroups; c++)
                    if (im[c] != INT_MIN)
                        tmax = fmaxf(tmax, static_cast<float>(im[c]) * sck[c]);
                }
                const float m_new = tmax > m_ref + C::kRescaleSlack ? tmax : m_ref;
                alpha = m_new == m_ref ? 1.0f : ex2_approx(m_ref - m_new);
                bias = FP8 ? m_new - kLog2_448 : m_new;
                m_ref = m_new;
            };
            if (need_mask)
                tile_max(std::true_type{});
            else
                tile_max(std::false_type{});

            // PV_i(j-1) must be complete before P_i is rewritten in TMEM, and O is
            // rescaled in TMEM before this tile's P.V lands on it (the whole warp takes
            // part if any of its rows moved its reference max)
            auto await_pv_and_rescale = [&]() -> bool {
                if (j == 0)
                    return true;
                if (!warp_wait(&pv_full[i], (j - 1) & 1, abort, p.status))
                    return false;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
                    for (int ch = 0; ch < D / 32; ch++) {
                        uint32_t orow[32];
                        tmem_ld32_async(tO + ch * 32, orow);
                        tmem_ld_wait(orow);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 ov = fma2(make_float2(__uint_as_float(orow[e]),
                                                               __uint_as_float(orow[e + 1])),
                                                   make_float2(alpha, alpha),
                                                   make_float2(0.0f, 0.0f));
                            orow[e] = __float_as_uint(ov.x);
                            orow[e + 1] = __float_as_uint(ov.y);
                        }
                        tmem_st32(tO + ch * 32, orow);
                    }
                    tmem_st_wait();
                }
                return true;
            };
            // FP16 mode at d = 128 streams each 32-key chunk of P into TMEM as it is
            // produced (the P.V wait comes first). FP8 mode (a P row of 32 words) and FP16
            // mode at d = 64 (64 words) pack the row in registers and store it after the
            // wait. Same-box A/B: streaming FP8 P is slower (into shared memory and into
            // TMEM alike); packing FP16 P is 2% faster at d = 64 and 1.5% slower at d = 128.
            constexpr bool kStreamP = !FP8 && D != 64;
            if constexpr (kStreamP) {
                if (!(ok = await_pv_and_rescale()))
                    break;
            }
            constexpr int kWords = FP8 ? C::BN / 4 : (kStreamP ? 1 : C::BN / 2);
            uint32_t pw[kWords];

            // p = 2^(S sc - m): S to fp32 exactly through the magic bias
            // (|S| <= 127^2 d < 2^22), one packed FFMA, ex2; each 32-key chunk is packed to
            // f16 / E4M3. P_i goes to TMEM: row = lane, keys along the columns (two f16 or
            // four E4M3 per column), the layout of an A operand in TMEM.
            auto tile_exp = [&](auto masked) {
                constexpr bool MASKED = decltype(masked)::value;
                float2 lsum2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
                for (int cq = 0; cq < 4; cq++) {   // 32 keys: one TMEM load's worth
                    [[maybe_unused]] const float sc = sck[cq * kKGroups / 4];
                    const uint32_t keep = MASKED ? chunk_mask(col_lim - kcol0 - cq * 32) : ~0u;
                    float pe[32];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float2 t;
                        if constexpr (SQ) {   // u = S sc + comp c is already in sreg
                            t = add2(make_float2(__uint_as_float(sreg[cq][e]),
                                                 __uint_as_float(sreg[cq][e + 1])),
                                     make_float2(-bias, -bias));
                        } else {
                            float2 x = make_float2(magic_biased(sreg[cq][e]),
                                                   magic_biased(sreg[cq][e + 1]));
                            x = add2(x, make_float2(-kMagic, -kMagic));      // exact S
                            t = fma2(x, make_float2(sc, sc), make_float2(-bias, -bias));
                        }
                        float2 pv = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                        if constexpr (MASKED) {
                            pv.x = ((keep >> e) & 1u) ? pv.x : 0.0f;
                            pv.y = ((keep >> (e + 1)) & 1u) ? pv.y : 0.0f;
                        }
                        pe[e] = pv.x;
                        pe[e + 1] = pv.y;
                        lsum2[(e >> 1) & 1] = add2(lsum2[(e >> 1) & 1], pv);
                    }
                    if constexpr (!FP8) {
                        // 32 keys = 16 columns of P_i (two f16 per column)
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 16; e++)
                            w[e] = pack_half2(pe[2 * e], pe[2 * e + 1]);
                        tmem_st16(tP + cq * 16, w);
                    } else {
                        // 32 keys = 8 words of four E4M3 codes, kept for the store after
                        // the wait for the previous P.V
#pragma unroll
                        for (int e = 0; e < 8; e++)
                            pw[cq * 8 + e] =
                                static_cast<uint32_t>(pack_e4m3x2(pe[4 * e], pe[4 * e + 1])) |
                                (static_cast<uint32_t>(pack_e4m3x2(pe[4 * e + 2], pe[4 * e + 3]))
                                 << 16);
                    }
                }
                l = alpha * l + (lsum2[0].x + lsum2[0].y + lsum2[1].x + lsum2[1].y);
            };
            auto tile_exp_il = [&](auto masked) {
                constexpr bool MASKED = decltype(masked)::value;
                float2 lsum2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
                // Row kept in registers (FP8; FP16 at d = 64): two 32-key chunks at a time,
                // their element pairs interleaved, so that two independent dependency chains
                // are in flight (FP8 +1.5%; FP16 at d = 128, which streams each chunk of P to
                // TMEM as it is produced, measured 1% slower this way)
#pragma unroll
                for (int cp = 0; cp < 4; cp += 2) {
                    float pe[2][32];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
#pragma unroll
                        for (int h2 = 0; h2 < 2; h2++) {
                            const int cq = cp + h2;
                            [[maybe_unused]] const float sc = sck[cq * kKGroups / 4];
                            float2 t;
                            if constexpr (SQ) {
                                t = add2(make_float2(__uint_as_float(sreg[cq][e]),
                                                     __uint_as_float(sreg[cq][e + 1])),
                                         make_float2(-bias, -bias));
                            } else {
                                float2 x = make_float2(magic_biased(sreg[cq][e]),
                                                       magic_biased(sreg[cq][e + 1]));
                                x = add2(x, make_float2(-kMagic, -kMagic));      // exact S
                                t = fma2(x, make_float2(sc, sc), make_float2(-bias, -bias));
                            }
                            float2 pv = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                            if constexpr (MASKED) {
                                const uint32_t keep = chunk_mask(col_lim - kcol0 - cq * 32);
                                pv.x = ((keep >> e) & 1u) ? pv.x : 0.0f;
                                pv.y = ((keep >> (e + 1)) & 1u) ? pv.y : 0.0f;
                            }
                            pe[h2][e] = pv.x;
                            pe[h2][e + 1] = pv.y;
                            lsum2[h2] = add2(lsum2[h2], pv);
                        }
                    }
#pragma unroll
                    for (int h2 = 0; h2 < 2; h2++) {
                        const int cq = cp + h2;
                        if constexpr (!FP8) {
                            // 32 keys = 16 words of two f16, kept for the store after the
                            // wait for the previous P.V
#pragma unroll
                            for (int e = 0; e < 16; e++)
                                pw[cq * 16 + e] = pack_half2(pe[h2][2 * e], pe[h2][2 * e + 1]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; e++)
                                pw[cq * 8 + e] =
                                    static_cast<uint32_t>(pack_e4m3x2(pe[h2][4 * e], pe[h2][4 * e + 1])) |
                                    (static_cast<uint32_t>(pack_e4m3x2(pe[h2][4 * e + 2], pe[h2][4 * e + 3]))
                                     << 16);
                        }
                    }
                }
                l = alpha * l + (lsum2[0].x + lsum2[0].y + lsum2[1].x + lsum2[1].y);
            };
            if constexpr (!kStreamP) {
                if (need_mask)
                    tile_exp_il(std::true_type{});
                else
                    tile_exp_il(std::false_type{});
            } else {
                if (need_mask)
                    tile_exp(std::true_type{});
                else
                    tile_exp(std::false_type{});
            }
            if constexpr (!kStreamP) {
                if (!(ok = await_pv_and_rescale()))
                    break;
                // 4 E4M3 keys or 2 f16 keys per column
#pragma unroll
                for (int c = 0; c < kWords; c += 32)
                    tmem_st32(tP + c, *reinterpret_cast<uint32_t(*)[32]>(pw + c));
            }
            tmem_st_wait();   // P in TMEM before the MMA issuer is told
            tc_fence_before();
            __syncwarp();
            warp_arrive<FP8>(&p_full[i]);
        }
        // epilogue: the last P.V, normalize, round to fp16, store the row
        if (ok && (ok = warp_wait(&pv_full[i], (nkv - 1) & 1, abort, p.status))) {
            tc_fence_after();
            // a row that sees no key (only when there are more queries than keys) has
            // l = 0 and P = 0: it is written as zeros
            const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            __half *dst = p.out + L.offset(s, start, h, qrow);
            uint32_t orow[D / 32][32];
#pragma unroll
            for (int ch = 0; ch < D / 32; ch++)
                tmem_ld32_async(tO + ch * 32, orow[ch]);
#pragma unroll
            for (int ch = 0; ch < D / 32; ch++) {
                uint32_t(&r)[32] = orow[ch];
                tmem_ld_wait(r);
                if (qrow < len) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) {
                            float sc = inv_l;
                            if constexpr (FP8)
                                sc = __ldg(p.v_scale + sh * D + ch * 32 + c + e) * inv_l;
                            f[e] = __uint_as_float(r[c + e]) * sc;
                            if constexpr (FP8)
                                if (p.v_mean != nullptr && l > 0.0f)
                                    f[e] += __ldg(p.v_mean + sh * D + ch * 32 + c + e);
                        }
                        uint4 u;
                        u.x = pack_half2(f[0], f[1]);
                        u.y = pack_half2(f[2], f[3]);
                        u.z = pack_half2(f[4], f[5]);
                        u.w = pack_half2(f[6], f[7]);
                        *reinterpret_cast<uint4 *>(dst + ch * 32 + c) = u;
                    }
                }
            }
        }
    } else if (warp == C::kProducerWarp) {
        // ----------------------------------------------------------------- producer
        // (like the MMA warp, the whole warp runs the loop and one elected lane issues each
        // copy: 0.5-1.5% faster than a lane-0 loop, and the warp no longer spills)
        if constexpr (NQT == 2)
            asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::kRegOther) : "memory");
        {
            if constexpr (!QIN)
                tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int c1, c2;
            if constexpr (!QIN) {   // (QIN: the softmax warps write the Q tiles)
                mbar_arrive_expect_tx_w(bar_q, NQT * C::kQBytes);
                for (int i = 0; i < NQT; i++) {
                    tma_coords(L, s, start, h, (qt0 + i) * C::BM, c1, c2);
                    tma_load_3d_w(sQ + i * C::kQBytes, &tmQ, bar_q, 0, c1, c2);
                }
            }
            int issued = 0;
            for (int j = 0; j < nkv; j++) {
                const int stg = j % C::STAGES;
                const uint32_t ph = (j / C::STAGES) & 1;
                tma_coords(LK, s, kstart, h, j * C::BN, c1, c2);
                if (!__all_sync(0xffffffffu, mbar_wait(&k_empty[stg], ph ^ 1, abort, p.status,
                                                       status_bit(SAGE_ERR_TIMEOUT), kTimeoutNs,
                                                       kPollSleepNs)))
                    break;
                mbar_arrive_expect_tx_w(&k_full[stg], C::kKBytes);
                tma_load_3d_w(sK + stg * C::kKBytes, &tmK, &k_full[stg], 0, c1, c2);
                if (!__all_sync(0xffffffffu, mbar_wait(&v_empty[stg], ph ^ 1, abort, p.status,
                                                       status_bit(SAGE_ERR_TIMEOUT), kTimeoutNs,
                                                       kPollSleepNs))) {
                    issued = j + 1;   // the K load of this tile is in flight
                    break;
                }
                mbar_arrive_expect_tx_w(&v_full[stg], C::kVBytes + C::kCompBytes);
                if constexpr (SQ)   // the stride is whole 128-key tiles: 16-byte aligned
                    bulk_load_g2s_w(smem + C::kOffB + stg * C::kCompBytes,
                                    p.q_comp + ((int64_t)s * L.H + h) * p.ncomp + j * C::BN,
                                    C::kCompBytes, &v_full[stg]);
#pragma unroll
                for (int cb = 0; cb < C::kVChunks; cb++)
                    tma_load_3d_w(sV + stg * C::kVBytes + cb * C::kVBoxBytes, &tmV,
                                  &v_full[stg], cb * (C::kVRowBytes / C::kVElem), c1, c2);
                issued = j + 1;
            }
            // drain: make sure no copy is still landing in shared memory when we leave
            if (lane == 0) {
                if constexpr (!QIN)
                    mbar_wait(bar_q, 0, nullptr, p.status, status_bit(SAGE_ERR_TIMEOUT),
                              kTimeoutNs);
                for (int j = max(0, issued - C::STAGES); j < issued; j++) {
                    const int stg = j % C::STAGES;
                    const uint32_t ph = (j / C::STAGES) & 1;
                    mbar_wait(&k_full[stg], ph, nullptr, p.status, status_bit(SAGE_ERR_TIMEOUT),
                              kTimeoutNs);
                    mbar_wait(&v_full[stg], ph, nullptr, p.status, status_bit(SAGE_ERR_TIMEOUT),
                              kTimeoutNs);
                }
            }
            __syncwarp();
        }
    } else if (warp == C::kMmaWarp) {
        // ---------------------------------------------------------------- MMA issuer
        if constexpr (NQT == 2)
            asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::kRegOther) : "memory");
        {
            constexpr uint32_t idesc_qk = instr_desc(2 /*s32*/, 1 /*s8*/, 1 /*s8*/, 0, 0, 128, 128);
            constexpr uint32_t idesc_pv = instr_desc(1 /*f32*/, 0 /*f16|e4m3*/, 0, 0,
                                                     1 /*V MN-major*/, 128, D);
            // descriptors are built once; a tile/k-step offset is added to the start
            // address field (bits 0-13, 16-byte units; shared addresses stay < 2^18)
            const uint64_t dQ0 = smem_desc(smem_u32(sQ), 16, C::kQkSbo, C::kQkSwizzle);
            const uint64_t dK0 = smem_desc(smem_u32(sK), 16, C::kQkSbo, C::kQkSwizzle);
            const uint64_t dV0 = smem_desc(smem_u32(sV), C::kVBoxBytes, C::kVSbo, C::kVSwizzle);
            auto issue_s = [&](int i, int stg) {
                const uint32_t dS = tmem_base;   // the shared S region
#pragma unroll
                for (int kk = 0; kk < D / 32; kk++) {
                    const uint64_t a = dQ0 + ((i * C::kQBytes + kk * 32) >> 4);
                    const uint64_t b = dK0 + ((stg * C::kKBytes + kk * 32) >> 4);
                    mma_i8_ss(dS, a, b, idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[i]);
            };
            auto issue_pv = [&](int i, int stg, int j) {
                const uint32_t dO = tmem_base + C::kSCols + i * D;
#pragma unroll
                for (int kk = 0; kk < C::BN / C::kPvK; kk++) {
                    const int key0 = kk * C::kPvK;            // first key of this k-step
                    const uint64_t b =
                        dV0 + ((stg * C::kVBytes + key0 * C::kVRowBytes) >> 4);
                    const uint32_t acc = (kk > 0 || j > 0) ? 1u : 0u;
                    // P_i in TMEM: 8 columns (16 f16 or 32 E4M3 keys) per k-step
                    const uint32_t ta = tmem_base + C::kSCols + NQT * D + i * C::kPCols + kk * 8;
                    if constexpr (FP8)
                        mma_f8_ts(dO, ta, b, idesc_pv, acc);
                    else
                        mma_f16_ts(dO, ta, b, idesc_pv, acc);
                }
                mma_commit(&pv_full[i]);
            };
            // every lane polls (the warp stays converged); the vote makes a timeout seen
            // by any lane the whole warp's outcome
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, p.status,
                                                         status_bit(SAGE_ERR_TIMEOUT),
                                                         kTimeoutNs, kPollSleepNs));
            };
            // One S region for both query tiles. s_free completes once per read of S,
            // in the order S_0(0), S_1(0), S_0(1), ...: completion 2j + i is query
            // tile i's read of S_i(j). Per KV tile: S_0(j+1) once S_1(j) has been
            // read, P.V_0(j), S_1(j+1) once S_0(j+1) has been read, P.V_1(j).
            bool ok = wait(bar_q, 0) && wait(&k_full[0], 0);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
            }
            if (ok && (ok = wait(s_free, 0))) {
                tc_fence_after();
                issue_s(1, 0);
                mma_commit(&k_empty[0]);
            }
            for (int j = 0; j < nkv && ok; j++) {
                const int stg = j % C::STAGES;
                const uint32_t ph = (j / C::STAGES) & 1;
                const bool more = j + 1 < nkv;
                const int stg1 = (j + 1) % C::STAGES;
                const uint32_t ph1 = ((j + 1) / C::STAGES) & 1;
                if (more) {
                    if (!(ok = wait(&k_full[stg1], ph1) && wait(s_free, 1)))
                        break;
                    tc_fence_after();
                    issue_s(0, stg1);
                }
                if (!(ok = wait(&v_full[stg], ph) && wait(&p_full[0], j & 1)))
                    break;
                tc_fence_after();
                issue_pv(0, stg, j);
                if (more) {
                    if (!(ok = wait(s_free, 0)))
                        break;
                    tc_fence_after();
                    issue_s(1, stg1);
                    mma_commit(&k_empty[stg1]);
                }
                if (!(ok = wait(&p_full[1], j & 1)))
                    break;
                tc_fence_after();
                issue_pv(1, stg, j);
                mma_commit(&v_empty[stg]);
            }
            // drain: every MMA issued above has completed before TMEM is released
            mma_commit(bar_drain);
            if (lane == 0)
                mbar_wait(bar_drain, 0, nullptr, p.status, status_bit(SAGE_ERR_TIMEOUT), kTimeoutNs);
            __syncwarp();
        }
    } else {
        if constexpr (NQT == 2)
            asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(C::kRegOther) : "memory");
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::kMmaWarp) {
        __syncwarp();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ----------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D map over the tensor [.., .., d] seen as (d, rows, heads) for the dense layout or
// (d, H, T) for the packed layout; a box is one tile of `box_rows` tokens of one head.
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes,
              const SeqLayout &L, int box_inner, int box_rows, CUtensorMapSwizzle swz)
{
    auto enc = get_encode();
    if (!enc)
        return false;
    cuuint64_t dims[3];
    cuuint64_t strides[2];
    cuuint32_t box[3];
    const cuuint32_t estr[3] = {1, 1, 1};
    if (L.cu == nullptr) {
        dims[0] = L.d;
        dims[1] = L.maxlen;
        dims[2] = (cuuint64_t)L.nseq * L.H;
        strides[0] = (cuuint64_t)L.d * elem_bytes;
        strides[1] = (cuuint64_t)L.maxlen * L.d * elem_bytes;
        box[0] = box_inner;
        box[1] = box_rows;
        box[2] = 1;
    } else {
        dims[0] = L.d;
        dims[1] = L.H;
        dims[2] = L.total;
        strides[0] = (cuuint64_t)L.d * elem_bytes;
        strides[1] = (cuuint64_t)L.H * L.d * elem_bytes;
        box[0] = box_inner;
        box[1] = 1;
        box[2] = box_rows;
    }
    CUresult r = enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, bool FP8, int NQT, bool DUMP, bool FINE, bool SQ, bool QIN>
cudaError_t run(const AttnArgs &a, const SeqLayout &L, const SeqLayout &LK, int *status,
                cudaStream_t st, sage_status_t *host_err)
{
    using C = Cfg<D, FP8, NQT, SQ>;
    CUtensorMap mq, mk, mv;
    const CUtensorMapSwizzle qk_swz =
        D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapSwizzle v_swz =
        C::kVRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    // (QIN: no Q map; the K map stands in for the unused parameter)
    bool ok = make_map(&mk, a.k_i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, LK, D, C::BN, qk_swz) &&
              (QIN ? (mq = mk, true)
                   : make_map(&mq, a.q_i8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L, D, C::BM,
                              qk_swz)) &&
              make_map(&mv, a.v,
                       FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                       C::kVElem, LK, C::kVRowBytes / C::kVElem, C::BN, v_swz);
    if (!ok) {
        *host_err = SAGE_ERR_CUDA;
        return cudaErrorInvalidValue;
    }
    KParams p;
    p.q_scale = a.q_scale;
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.v_mean = a.v_mean;
    p.q_comp = a.q_comp;
    p.ncomp = comp_stride(LK.maxlen);
    p.out = a.out;
    p.s_dump = a.s_dump;
    p.L = L;
    p.LK = LK;
    const int q_grp = FINE ? 1 : kQBlock, k_grp = FINE ? 32 : kKBlock;
    p.nqb = (L.maxlen + q_grp - 1) / q_grp;
    p.nkb = (LK.maxlen + k_grp - 1) / k_grp;
    p.causal = a.causal;
    p.sc_log2 = a.sm_scale * kLog2e;
    p.status = status;
    p.q16 = a.q16;
    p.qsum = a.qsum;

    auto kern = attn_kernel<D, FP8, NQT, DUMP, FINE, SQ, QIN>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess)
        return e;
    // the kernel must launch with the registers the setmaxnreg split assumes (with fewer,
    // the softmax warps' increase could never be granted); read once per instantiation
    static std::once_flag once;
    static int regs = 0;
    std::call_once(once, [&] {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess)
            regs = fa.numRegs;
    });
    if (regs != C::kLaunchRegs) {
        *host_err = SAGE_ERR_UNSUPPORTED;
        return cudaErrorInvalidConfiguration;
    }
    const int nqt = (L.maxlen + C::BM - 1) / C::BM;
    dim3 grid((nqt + NQT - 1) / NQT, L.H, L.nseq);
    kern<<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

// The instantiation for the P.V mode, the scale groups, smooth Q and where Q's codes
// come from. In-kernel Q quantization is built for smooth Q only, where it measures
// faster than the separate pass (with plain Q the per-CTA prologue costs more than the
// pass it saves, most on short causal sequences).
template <int D>
cudaError_t dispatch_d(const AttnArgs &a, const SeqLayout &L, const SeqLayout &LK, int *status,
                       cudaStream_t st, sage_status_t *host_err)
{
    const bool fp8 = a.pv_mode == SAGE_PV_FP8, fine = a.fine != 0, sq = a.q_comp != nullptr;
    auto pick = [&](auto f8, auto fn, auto q) {
        return run<D, decltype(f8)::value, 2, false, decltype(fn)::value, decltype(q)::value,
                   false>(a, L, LK, status, st, host_err);
    };
    auto pick_qin = [&](auto f8, auto fn) {
        return run<D, decltype(f8)::value, 2, false, decltype(fn)::value, true, true>(
            a, L, LK, status, st, host_err);
    };
    using T = std::true_type;
    using F = std::false_type;
    if (a.q16 != nullptr) {
        if (!sq || a.qsum == nullptr) {
            *host_err = SAGE_ERR_INVALID_ARG;
            return cudaErrorInvalidValue;
        }
        if (fp8)
            return fine ? pick_qin(T{}, T{}) : pick_qin(T{}, F{});
        return fine ? pick_qin(F{}, T{}) : pick_qin(F{}, F{});
    }
    if (fp8) {
        if (fine)
            return sq ? pick(T{}, T{}, T{}) : pick(T{}, T{}, F{});
        return sq ? pick(T{}, F{}, T{}) : pick(T{}, F{}, F{});
    }
    if (fine)
        return sq ? pick(F{}, T{}, T{}) : pick(F{}, T{}, F{});
    return sq ? pick(F{}, F{}, T{}) : pick(F{}, F{}, F{});
}

}  // namespace

cudaError_t launch_attention(const AttnArgs &a, const SeqLayout &L, const SeqLayout &LK,
                             int *status, cudaStream_t st, sage_status_t *host_err)
{
    *host_err = SAGE_OK;
    if (L.nseq != LK.nseq || L.H != LK.H || L.d != LK.d) {
        *host_err = SAGE_ERR_INVALID_ARG;
        return cudaErrorInvalidValue;
    }
    if (a.s_dump != nullptr) {
        if (L.d == 128)
            return run<128, false, 2, true, false, false, false>(a, L, LK, status, st, host_err);
        return run<64, false, 2, true, false, false, false>(a, L, LK, status, st, host_err);
    }
    return L.d == 128 ? dispatch_d<128>(a, L, LK, status, st, host_err)
                      : dispatch_d<64>(a, L, LK, status, st, host_err);
}

}  // namespace sage
