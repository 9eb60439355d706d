// Declarations of the decode path (decode.cu), used by the C-ABI layer.
#pragma once

#include "sage_common.cuh"

namespace sage {

// Decode (decode.cu): Nq <= kDecodeMaxQ queries against Nk keys, dense [B, H, N, d], FP16
// P.V, split over the keys. The plan is a function of the shape only, so the workspace
// size and the launch agree.
constexpr int kDecodeMaxQ = 16;
struct DecodePlan {
    int split_keys;   // keys per split (whole 128-key tiles)
    int nsplit;       // splits per (sequence, head)
};
DecodePlan decode_plan(int B, int H, int Nq, int Nk);
// fp32 words of the splits' partial results: per (sequence, head, split, query) its
// maximum, its sum and d output sums
size_t decode_partial_floats(int B, int H, int Nq, int Nk, int d);
struct DecodeArgs {
    const int8_t *q_i8;
    const float *q_scale;   // [B,H,1] per block, [B,H,Nq] with fine groups
    const int8_t *k_i8;
    const float *k_scale;   // [B,H,ceil(Nk/64)] per block, [B,H,ceil(Nk/32)] fine
    const __half *v;
    __half *out;
    float *workspace;       // decode_partial_floats(...) floats
    int B, H, Nq, Nk, d;
    int causal;
    int fine;
    float sm_scale;
};
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);

}  // namespace sage
