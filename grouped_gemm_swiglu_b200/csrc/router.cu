// router.cu -- gate epilogue: top-k selection and routing weights, one warp per token.
//
// Follows sglang PR #36385 "Enable and fuse the Inkling MoE gate epilogue on Intel XPU":
//  * item 3: top-k by k masked-max passes (not a sort); ties go to the lower column id
//    (the ~index half of the packed sort key); a column is selected at most once
//    (the "remaining" mask); the raw logit, not an activated score, is carried out;
//  * item 2: weights exp(lp - logsumexp(lp)) with lp = logsigmoid(x), which stays
//    finite when every logit is below -104;
//  * trailing shared-sink columns never enter the top-k but join the normaliser.
// The softmax epilogue renormalises over the k selected logits.
#include <cfloat>
#include <climits>

#include "internal.h"

namespace moe {

// CPL = columns per lane (N <= 32*CPL). Lane l holds columns c*32 + l, c < CPL.
template <int CPL>
__global__ void __launch_bounds__(256) router_kernel(const float* __restrict__ logits, int T, int N, int S, int k,
                                                     int score, float route_scale, int32_t* __restrict__ ids,
                                                     float* __restrict__ w, float* __restrict__ sw) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + (size_t)t * (size_t)(N + S);

    float v[CPL];
    uint32_t live = 0;  // bit c set: column c*32 + lane is still a candidate
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int col = c * 32 + lane;
        if (col < N) {
            v[c] = __ldg(row + col);
            live |= 1u << c;
        } else {
            v[c] = -FLT_MAX;
        }
    }

    float my_v = 0.f;  // lane j < k keeps the j-th winner
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        // Best remaining column of this lane: largest value, lowest id among equals
        // (ids grow with c, so a strict comparison keeps the first).
        float bv = -FLT_MAX;
        int bi = INT_MAX;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            if ((live >> c) & 1u) {
                if (bi == INT_MAX || v[c] > bv) {
                    bv = v[c];
                    bi = c * 32 + lane;
                }
            }
        }
        // Warp-wide maximum of (value, -id).
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (oi != INT_MAX && (bi == INT_MAX || ov > bv || (ov == bv && oi < bi))) {
                bv = ov;
                bi = oi;
            }
        }
        if (bi != INT_MAX && (bi & 31) == lane) live &= ~(1u << (bi >> 5));
        if (lane == j) {
            my_v = bv;
            my_id = bi;
        }
    }

    // Epilogue: lanes [0, k) hold the selected logits, lanes [k, k+S) the sink logits.
    const bool active = lane < k + S;
    float x = 0.f;
    if (lane < k) x = my_v;
    else if (lane < k + S) x = __ldg(row + N + (lane - k));
    float lp = x;
    if (score == MOE_SCORE_SIGMOID) lp = fminf(x, 0.f) - log1pf(expf(-fabsf(x)));  // logsigmoid
    float m = active ? lp : -FLT_MAX;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    // exp(lp - logsumexp(lp)) evaluated as exp(lp - m) / sum exp(lp - m): the same
    // value, without the rounding of a large log-sum-exp (|lp| ~ 200) in fp32.
    const float e = active ? expf(lp - m) : 0.f;
    float sum = e;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float wt = (e / sum) * route_scale;  // sum >= 1: the maximum contributes exp(0)
    if (lane < k) {
        ids[(size_t)t * k + lane] = my_id;
        w[(size_t)t * k + lane] = wt;
    } else if (lane < k + S) {
        sw[(size_t)t * S + (lane - k)] = wt;
    }
}

cudaError_t launch_router(const float* logits, int T, int N, int S, int k, int score, float route_scale,
                          int32_t* ids, float* w, float* sw, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps), block(32 * warps);
    if (N <= 32) router_kernel<1><<<grid, block, 0, stream>>>(logits, T, N, S, k, score, route_scale, ids, w, sw);
    else if (N <= 64) router_kernel<2><<<grid, block, 0, stream>>>(logits, T, N, S, k, score, route_scale, ids, w, sw);
    else if (N <= 128) router_kernel<4><<<grid, block, 0, stream>>>(logits, T, N, S, k, score, route_scale, ids, w, sw);
    else if (N <= 256) router_kernel<8><<<grid, block, 0, stream>>>(logits, T, N, S, k, score, route_scale, ids, w, sw);
    else if (N <= 512) router_kernel<16><<<grid, block, 0, stream>>>(logits, T, N, S, k, score, route_scale, ids, w, sw);
    else router_kernel<32><<<grid, block, 0, stream>>>(logits, T, N, S, k, score, route_scale, ids, w, sw);
    return cudaGetLastError();
}

}  // namespace moe
