// router.cu -- gate epilogue: top-k selection and routing weights, one warp per token.
//
// Follows sglang PR #36385 "Enable and fuse the Inkling MoE gate epilogue on Intel XPU":
//  * item 3: top-k by k masked-max passes (not a sort); ties go to the lower column id
//    (the ~index half of the packed sort key); a column is selected at most once
//    (the "remaining" mask); the raw logit, not an activated score, is carried out;
//  * item 2: weights exp(lp - logsumexp(lp)) with lp = logsigmoid(x), which stays
//    finite when every logit is below -104;
//  * trailing shared-sink columns never enter the top-k but join the normaliser;
//  * an optional correction bias [N] (routed columns only) changes the ranking key to
//    sigmoid(logit) + bias in fp32 while the weights still come from the raw logits;
//  * optional packed output (id << 16 | bf16 weight), the form a fused consumer reads.
// The softmax epilogue renormalises over the k selected logits.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>

#include "internal.h"

namespace moe {

// CPL = columns per lane (N <= 32*CPL). Lane l holds columns c*32 + l, c < CPL.
// BIAS: rank on sigmoid(logit) + bias instead of the raw logit (a separate instance, so
// the unbiased router keeps one value per column in registers).
template <int CPL, bool BIAS>
__global__ void __launch_bounds__(256) router_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                                     int T, int N, int S, int k, int score, float route_scale,
                                                     int32_t* __restrict__ ids, float* __restrict__ w,
                                                     float* __restrict__ sw, uint32_t* __restrict__ packed) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + (size_t)t * (size_t)(N + S);

    float v[CPL];                 // raw logits: the value carried out of the selection
    float key[BIAS ? CPL : 1];    // BIAS: sigmoid(logit) + bias; else the key is v itself
    uint32_t live = 0;  // bit c set: column c*32 + lane is still a candidate
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int col = c * 32 + lane;
        if (col < N) {
            v[c] = __ldg(row + col);
            if constexpr (BIAS) key[c] = __fadd_rn(__fdiv_rn(1.f, 1.f + expf(-v[c])), __ldg(bias + col));
            live |= 1u << c;
        } else {
            v[c] = -FLT_MAX;
            if constexpr (BIAS) key[c] = -FLT_MAX;
        }
    }

    float my_v = 0.f;  // lane j < k keeps the j-th winner
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        // Best remaining column of this lane: largest key, lowest id among equals
        // (ids grow with c, so a strict comparison keeps the first).
        float bk = -FLT_MAX, bv = 0.f;
        int bi = INT_MAX;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            if ((live >> c) & 1u) {
                const float kc = BIAS ? key[BIAS ? c : 0] : v[c];
                if (bi == INT_MAX || kc > bk) {
                    bk = kc;
                    bv = v[c];
                    bi = c * 32 + lane;
                }
            }
        }
        // Warp-wide maximum of (key, -id), carrying the winner's raw logit.
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
            const float ov = BIAS ? __shfl_xor_sync(0xffffffffu, bv, off) : ok;
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (oi != INT_MAX && (bi == INT_MAX || ok > bk || (ok == bk && oi < bi))) {
                bk = ok;
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
        if (packed)
            packed[(size_t)t * k + lane] =
                ((uint32_t)my_id << 16) | (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(wt));
    } else if (lane < k + S) {
        sw[(size_t)t * S + (lane - k)] = wt;
    }
}

cudaError_t launch_router(const float* logits, const float* bias, int T, int N, int S, int k, int score,
                          float route_scale, int32_t* ids, float* w, float* sw, uint32_t* packed, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps), block(32 * warps);
#define MOE_ROUTER(CPL)                                                                                        \
    (bias ? router_kernel<CPL, true><<<grid, block, 0, stream>>>(logits, bias, T, N, S, k, score, route_scale, ids, \
                                                                  w, sw, packed)                                  \
          : router_kernel<CPL, false><<<grid, block, 0, stream>>>(logits, bias, T, N, S, k, score, route_scale,   \
                                                                   ids, w, sw, packed))
    if (N <= 32) MOE_ROUTER(1);
    else if (N <= 64) MOE_ROUTER(2);
    else if (N <= 128) MOE_ROUTER(4);
    else if (N <= 256) MOE_ROUTER(8);
    else if (N <= 512) MOE_ROUTER(16);
    else MOE_ROUTER(32);
#undef MOE_ROUTER
    return cudaGetLastError();
}

}  // namespace moe
