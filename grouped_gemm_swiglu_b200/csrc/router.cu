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

// Logit loads: through the read-only path when the logits are an input of the launch,
// through L2 when other CTAs of the same launch wrote them (the fused gate GEMV).
template <bool COHERENT>
__device__ __forceinline__ float load_logit(const float* p) {
    if constexpr (COHERENT) return __ldcg(p);
    else return __ldg(p);
}

// Routes token t with one warp (all 32 lanes must call it).
// CPL = columns per lane (N <= 32*CPL). Lane l holds columns c*32 + l, c < CPL.
// BIAS: rank on sigmoid(logit) + bias instead of the raw logit (a separate instance, so
// the unbiased router keeps one value per column in registers).
template <int CPL, bool BIAS, bool COHERENT>
__device__ __forceinline__ void route_token(const float* __restrict__ row, const float* __restrict__ bias, int t,
                                            int N, int S, int k, int score, float route_scale,
                                            int32_t* __restrict__ ids, float* __restrict__ w,
                                            float* __restrict__ sw, uint32_t* __restrict__ packed) {
    const int lane = threadIdx.x & 31;

    float v[CPL];                 // raw logits: the value carried out of the selection
    float key[BIAS ? CPL : 1];    // BIAS: sigmoid(logit) + bias; else the key is v itself
    uint32_t live = 0;  // bit c set: column c*32 + lane is still a candidate
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const int col = c * 32 + lane;
        if (col < N) {
            v[c] = load_logit<COHERENT>(row + col);
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
    else if (lane < k + S) x = load_logit<COHERENT>(row + N + (lane - k));
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

template <int CPL, bool BIAS>
__global__ void __launch_bounds__(256) router_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                                     int T, int N, int S, int k, int score, float route_scale,
                                                     int32_t* __restrict__ ids, float* __restrict__ w,
                                                     float* __restrict__ sw, uint32_t* __restrict__ packed) {
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    route_token<CPL, BIAS, false>(logits + (size_t)t * (size_t)(N + S), bias, t, N, S, k, score, route_scale, ids, w,
                                  sw, packed);
}

// ---------------------------------------------------------------- fused gate GEMV + router
// The 258-column gate GEMM and its epilogue in one launch for decode-sized batches
// (sglang PR #36385: the fused gate GEMV path taken at <= 4 tokens; the op is
// submission-bound there). logits[t][c] = sum_h x[t][h] * wg[c][h], fp32 accumulation
// of the bf16 products. Each CTA computes kGateCols columns for every token, a column
// split over kGateSplit warps (H/kGateSplit elements each, 16-byte loads), the partial
// sums added in a fixed order. The CTA that finishes last (an atomic counter, then
// reset to zero) routes every token from the finished logits. XSMEM: the CTA first copies
// x into shared memory (one coalesced pass), so the dot products read every token's row
// from there instead of from L2 once per 8-element chunk.
constexpr int kGateCols = 2;
constexpr int kGateSplit = 4;  // warps per column: 8 warps = kGateCols * kGateSplit
constexpr size_t kGateXSmemMax = 96 * 1024;

template <int TMAX, int CPL, bool BIAS, bool XSMEM>
__global__ void __launch_bounds__(256) gate_route_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ wg,
                                                         const float* __restrict__ bias, int T, int H, int N, int S,
                                                         int k, int score, float route_scale, float* logits,
                                                         int32_t* __restrict__ ids, float* __restrict__ w,
                                                         float* __restrict__ sw, uint32_t* __restrict__ packed,
                                                         unsigned int* counter) {
    __shared__ float part[kGateCols][kGateSplit][TMAX];
    __shared__ int s_last;
    extern __shared__ __align__(16) uint8_t gate_sm[];
    const int C = N + S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();
    const __nv_bfloat16* xs = x;
    if constexpr (XSMEM) {
        uint4* dst = reinterpret_cast<uint4*>(gate_sm);
        const int nvec = T * H / 8;
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) dst[v] = __ldg(reinterpret_cast<const uint4*>(x) + v);
        __syncthreads();
        xs = reinterpret_cast<const __nv_bfloat16*>(gate_sm);
    }
    const int col_local = warp / kGateSplit, piece = warp % kGateSplit;
    const int col = blockIdx.x * kGateCols + col_local;
    const int len = H / kGateSplit;  // a multiple of 32 (H is a multiple of 128)
    float acc[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) acc[t] = 0.f;
    if (col < C) {
        const __nv_bfloat16* wr = wg + (size_t)col * H + (size_t)piece * len;
#pragma unroll 4
        for (int i = lane * 8; i < len; i += 32 * 8) {
            const uint4 wv = __ldg(reinterpret_cast<const uint4*>(wr + i));
            const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&wv);
            float wf[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(w2[j]);
                wf[2 * j] = f.x;
                wf[2 * j + 1] = f.y;
            }
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t < T) {
                    const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)t * H + (size_t)piece * len + i);
                    const uint4 xv = XSMEM ? *xp : __ldg(xp);
                    const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = __bfloat1622float2(x2[j]);
                        acc[t] = fmaf(f.x, wf[2 * j], acc[t]);
                        acc[t] = fmaf(f.y, wf[2 * j + 1], acc[t]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < TMAX; ++t) part[col_local][piece][t] = acc[t];
    }
    __syncthreads();
    if (threadIdx.x < kGateCols * TMAX) {
        const int cl = threadIdx.x / TMAX, t = threadIdx.x % TMAX;
        const int c = blockIdx.x * kGateCols + cl;
        if (c < C && t < T) {
            float v = 0.f;
#pragma unroll
            for (int q = 0; q < kGateSplit; ++q) v += part[cl][q][t];
            logits[(size_t)t * C + c] = v;
        }
    }
    // Publish this CTA's logits (fence before the count), and let the last CTA route.
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned int done = atomicAdd(counter, 1u);
        s_last = done == gridDim.x - 1;
        if (s_last) {
            __threadfence();
            atomicExch(counter, 0u);
        }
    }
    __syncthreads();
    if (!s_last) return;
    for (int t = warp; t < T; t += blockDim.x >> 5)
        route_token<CPL, BIAS, true>(logits + (size_t)t * C, bias, t, N, S, k, score, route_scale, ids, w, sw, packed);
}

cudaError_t launch_router(const float* logits, const float* bias, int T, int N, int S, int k, int score,
                          float route_scale, int32_t* ids, float* w, float* sw, uint32_t* packed, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps), block(32 * warps);
#define MOE_ROUTER(CPL)                                                                                          \
    return launch_pdl(bias ? router_kernel<CPL, true> : router_kernel<CPL, false>, grid, block, 0, stream, logits, \
                      bias, T, N, S, k, score, route_scale, ids, w, sw, packed)
    if (N <= 32) MOE_ROUTER(1);
    if (N <= 64) MOE_ROUTER(2);
    if (N <= 128) MOE_ROUTER(4);
    if (N <= 256) MOE_ROUTER(8);
    if (N <= 512) MOE_ROUTER(16);
    MOE_ROUTER(32);
#undef MOE_ROUTER
}

template <int TMAX>
static cudaError_t launch_gate_t(const void* x, const void* wg, const float* bias, int T, int H, int N, int S, int k,
                                 int score, float route_scale, float* logits, int32_t* ids, float* w, float* sw,
                                 uint32_t* packed, unsigned int* counter, cudaStream_t stream) {
    const int C = N + S;
    dim3 grid((C + kGateCols - 1) / kGateCols), block(256);
    auto xb = static_cast<const __nv_bfloat16*>(x);
    auto wb = static_cast<const __nv_bfloat16*>(wg);
    const size_t xbytes = (size_t)T * H * 2;
    const bool xsmem = T >= 2 && xbytes <= kGateXSmemMax;  // one token: nothing to share, skip the copy
#define MOE_GATE(CPL)                                                                                                \
    {                                                                                                                \
        auto kern = xsmem ? (bias ? gate_route_kernel<TMAX, CPL, true, true> : gate_route_kernel<TMAX, CPL, false, true>) \
                          : (bias ? gate_route_kernel<TMAX, CPL, true, false>                                        \
                                  : gate_route_kernel<TMAX, CPL, false, false>);                                     \
        if (xsmem && xbytes > 48 * 1024) {                                                                           \
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGateXSmemMax); \
            if (e != cudaSuccess) return e;                                                                          \
        }                                                                                                            \
        return launch_pdl(kern, grid, block, xsmem ? xbytes : (size_t)0, stream, xb, wb, bias, T, H, N, S, k, score,  \
                          route_scale, logits, ids, w, sw, packed, counter);                                         \
    }
    if (N <= 32) MOE_GATE(1);
    if (N <= 64) MOE_GATE(2);
    if (N <= 128) MOE_GATE(4);
    if (N <= 256) MOE_GATE(8);
    if (N <= 512) MOE_GATE(16);
    MOE_GATE(32);
#undef MOE_GATE
}

cudaError_t launch_gate_route(const void* x, const void* wg, const float* bias, int T, int H, int N, int S, int k,
                              int score, float route_scale, float* logits, int32_t* ids, float* w, float* sw,
                              uint32_t* packed, unsigned int* counter, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    if (T <= 1) return launch_gate_t<1>(x, wg, bias, T, H, N, S, k, score, route_scale, logits, ids, w, sw, packed,
                                        counter, stream);
    if (T <= 4) return launch_gate_t<4>(x, wg, bias, T, H, N, S, k, score, route_scale, logits, ids, w, sw, packed,
                                        counter, stream);
    if (T <= 8) return launch_gate_t<8>(x, wg, bias, T, H, N, S, k, score, route_scale, logits, ids, w, sw, packed,
                                        counter, stream);
    return launch_gate_t<kGateMaxTokens>(x, wg, bias, T, H, N, S, k, score, route_scale, logits, ids, w, sw, packed,
                                         counter, stream);
}

}  // namespace moe
