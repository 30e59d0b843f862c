// permute.cu -- expert histogram, prefix scan and the stable gather of activation
// rows by expert (per-expert sorted-token dispatch, batchgen PR #239 commit notes),
// with the 1x128 E4M3 activation quantisation fused into the copy (the "fused
// act-quant" activation kernel of the xorl-wheels FlashInfer 0.6.18 release notes).
//
// Order inside a group is (token, slot), fixed by construction, so the result does not
// depend on scheduling: every 256-token chunk builds one membership bitmap per warp
// and expert (atomicOr is order-free), ranks come from popcounts, and chunk bases from
// a prefix over chunks.
#include <cuda_fp8.h>

#include "internal.h"
#include "status.cuh"

namespace moe {

constexpr int kChunk = 256;  // tokens per counting chunk (8 warps x 32 lanes)

size_t permute_scratch_bytes(int T, int k, int E) {
    const size_t nchunk = (size_t)(T + kChunk - 1) / kChunk;
    auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
    return al(nchunk * E * sizeof(int32_t)) + al((size_t)T * k * sizeof(int32_t));
}

// One CTA per 256-token chunk. Writes cnt[chunk][e] (tokens of the chunk routed to e)
// and rank[t][j] (position of (t, j) among the chunk's rows of its expert).
__global__ void __launch_bounds__(256) permute_count_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                            int32_t* __restrict__ cnt, int32_t* __restrict__ rank,
                                                            int* status) {
    extern __shared__ uint32_t sm[];
    uint32_t* flags = sm;                                      // [8][E] membership bitmaps
    uint16_t* pre = reinterpret_cast<uint16_t*>(sm + 8 * E);  // [8][E] rows of earlier warps
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) flags[i] = 0;
    __syncthreads();
    const int t = blockIdx.x * kChunk + threadIdx.x;
    uint32_t* f = flags + warp * E;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = ids[(size_t)t * k + j];
            if (e < 0 || e >= E) {
                set_status(status, MOE_ERR_EXPERT_ID);
            } else {
                const uint32_t old = atomicOr(&f[e], 1u << lane);
                if (old & (1u << lane)) set_status(status, MOE_ERR_EXPERT_ID);  // repeated within a token
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            pre[w * E + e] = (uint16_t)run;
            run += __popc(flags[w * E + e]);
        }
        cnt[(size_t)blockIdx.x * E + e] = (int32_t)run;
    }
    __syncthreads();
    if (t < T) {
        const uint32_t lt = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int e = ids[(size_t)t * k + j];
            rank[(size_t)t * k + j] = (e >= 0 && e < E) ? (int32_t)pre[warp * E + e] + __popc(f[e] & lt) : -1;
        }
    }
}

// Single CTA. Turns cnt[chunk][e] into exclusive chunk bases (in place), and writes
// offsets[0..G] = exclusive scan of the group sizes (shared groups hold T rows).
__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t* __restrict__ cnt, int nchunk, int E,
                                                            int n_shared, int T, int32_t* __restrict__ offsets) {
    extern __shared__ int32_t tot[];  // [G]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int G = E + n_shared;
    const int cpl = (nchunk + 31) / 32;  // chunks per lane
    for (int e = warp; e < E; e += nwarps) {
        const int c0 = min(lane * cpl, nchunk), c1 = min(c0 + cpl, nchunk);
        int s = 0;
        for (int c = c0; c < c1; ++c) s += cnt[(size_t)c * E + e];
        int incl = s;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += n;
        }
        int run = incl - s;
        for (int c = c0; c < c1; ++c) {
            const int v = cnt[(size_t)c * E + e];
            cnt[(size_t)c * E + e] = run;
            run += v;
        }
        if (lane == 31) tot[e] = incl;
    }
    for (int s = threadIdx.x; s < n_shared; s += blockDim.x) tot[E + s] = T;
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < G; base += 32) {
            const int g = base + lane;
            const int v = g < G ? tot[g] : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += n;
            }
            if (g < G) offsets[g] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) offsets[G] = carry;
    }
}

// One warp per token: destinations of its k routed slots and n_shared shared rows,
// perm / inv_perm, and the copy (bf16) or quantised copy (E4M3 + scales) of x[t].
template <bool FP8>
__global__ void __launch_bounds__(256) permute_scatter_kernel(
    const int32_t* __restrict__ ids, const int32_t* __restrict__ rank, const int32_t* __restrict__ base,
    const int32_t* __restrict__ offsets, const uint16_t* __restrict__ x, int T, int H, int k, int E, int n_shared,
    int64_t A, int32_t* __restrict__ perm, int32_t* __restrict__ inv, void* __restrict__ x_perm,
    float* __restrict__ x_scale) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    int dst = -1;
    if (lane < k) {
        const int e = ids[(size_t)t * k + lane];
        const int r = rank[(size_t)t * k + lane];
        if (e >= 0 && e < E && r >= 0) dst = offsets[e] + base[(size_t)(t / kChunk) * E + e] + r;
        inv[(size_t)t * k + lane] = dst;
    } else if (lane < k + n_shared) {
        dst = offsets[E + (lane - k)] + t;
    }
    if (dst >= 0) perm[dst] = t;
    const int nd = k + n_shared;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    const int nvec = H / 8;
    // Warp-uniform trip count: every lane takes part in the shuffles below.
    for (int v0 = 0; v0 < nvec; v0 += 32) {
        const int v = v0 + lane;
        const bool act = v < nvec;
        const uint4 xv = act ? __ldg(xr + v) : make_uint4(0, 0, 0, 0);
        if constexpr (!FP8) {
            for (int d = 0; d < nd; ++d) {
                const int D = __shfl_sync(0xffffffffu, dst, d);
                if (D >= 0 && act) reinterpret_cast<uint4*>(static_cast<uint16_t*>(x_perm) + (size_t)D * H)[v] = xv;
            }
        } else {
            // 16 lanes x 8 values = one 128-wide block; amax, s = amax/448 (1 if 0),
            // code = E4M3(x/s) with round-to-nearest-even and saturation, in fp32.
            float f[8];
            const uint32_t wv[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                f[2 * i] = __uint_as_float(wv[i] << 16);
                f[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
            }
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t q = (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(f[i], s), __NV_SATFINITE, __NV_E4M3);
                if (i < 4) lo |= q << (8 * i);
                else hi |= q << (8 * (i - 4));
            }
            const int blk = v / 16;
            for (int d = 0; d < nd; ++d) {
                const int D = __shfl_sync(0xffffffffu, dst, d);
                if (D >= 0 && act) {
                    reinterpret_cast<uint2*>(static_cast<uint8_t*>(x_perm) + (size_t)D * H)[v] = make_uint2(lo, hi);
                    if ((lane & 15) == 0) x_scale[(size_t)blk * A + D] = s;
                }
            }
        }
    }
}

cudaError_t launch_permute(const int32_t* ids, const void* x, int T, int H, int k, int E, int n_shared, bool fp8,
                           int32_t* offsets, int32_t* perm, int32_t* inv, void* x_perm, float* x_scale,
                           void* scratch, int* status, cudaStream_t stream) {
    const int G = E + n_shared;
    if (T == 0) return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (G + 1), stream);
    const int nchunk = (T + kChunk - 1) / kChunk;
    int32_t* cnt = static_cast<int32_t*>(scratch);
    int32_t* rank = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) +
                                               (((size_t)nchunk * E * sizeof(int32_t) + 255) & ~size_t(255)));
    const size_t sm1 = (size_t)8 * E * sizeof(uint32_t) + (size_t)8 * E * sizeof(uint16_t);
    cudaError_t err;
    if (sm1 > 48 * 1024) {
        err = cudaFuncSetAttribute(permute_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
        if (err != cudaSuccess) return err;
    }
    permute_count_kernel<<<nchunk, 256, sm1, stream>>>(ids, T, k, E, cnt, rank, status);
    permute_scan_kernel<<<1, 1024, (size_t)G * sizeof(int32_t), stream>>>(cnt, nchunk, E, n_shared, T, offsets);
    const int64_t A = (int64_t)T * (k + n_shared);
    dim3 grid((T + 7) / 8);
    if (fp8)
        permute_scatter_kernel<true><<<grid, 256, 0, stream>>>(ids, rank, cnt, offsets,
                                                               static_cast<const uint16_t*>(x), T, H, k, E,
                                                               n_shared, A, perm, inv, x_perm, x_scale);
    else
        permute_scatter_kernel<false><<<grid, 256, 0, stream>>>(ids, rank, cnt, offsets,
                                                                static_cast<const uint16_t*>(x), T, H, k, E,
                                                                n_shared, A, perm, inv, x_perm, x_scale);
    return cudaGetLastError();
}

}  // namespace moe
