// permute.cu -- expert histogram, prefix scan and the stable gather of activation
// rows by expert (per-expert sorted-token dispatch, batchgen PR #239 commit notes),
// with the 1x128 E4M3 activation quantisation fused into the copy (the "fused
// act-quant" activation kernel of the xorl-wheels FlashInfer 0.6.18 release notes).
//
// Order inside a group is (token, slot), fixed by construction, so the result does not
// depend on scheduling: every 256-token chunk builds one membership bitmap per warp
// and expert (atomicOr is order-free), ranks come from popcounts, and chunk bases from
// a prefix over chunks. Two launches: count (+ scan in the CTA that finishes last), and
// the scatter/copy.
#include <cuda_fp8.h>

#include "internal.h"
#include "status.cuh"

namespace moe {

constexpr int kChunk = 256;          // tokens per counting chunk (8 warps x 32 lanes)
constexpr int kMaxGroups = 1024 + 32;
constexpr int kScatterThreads = 256;

size_t permute_scratch_bytes(int T, int k, int E) {
    const size_t nchunk = (size_t)(T + kChunk - 1) / kChunk;
    auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
    return al(nchunk * E * sizeof(int32_t)) + al((size_t)T * k * sizeof(int32_t));
}

// Exclusive scan of v[0..n) (n <= kMaxGroups) into out[0..n], out[n] = total; 256 threads.
__device__ void block_exclusive_scan_256(const int32_t* v, int n, int32_t* out) {
    __shared__ int32_t warp_tot[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + 255) / 256;
    const int b = min(tid * per, n), e = min(b + per, n);
    int local = 0;
    for (int i = b; i < e; ++i) local += v[i];
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    int run = before + incl - local;
    for (int i = b; i < e; ++i) {
        out[i] = run;
        run += v[i];
    }
    if (tid == 255) out[n] = before + incl;
}

// One CTA per 256-token chunk. Writes cnt[chunk][e] (tokens of the chunk routed to e)
// and rank[t][j] (position of (t, j) among the chunk's rows of its expert). The CTA
// that finishes last turns cnt into exclusive chunk bases (in place) and writes
// offsets[0..G] (shared groups hold T rows each), then resets the counter to zero.
__global__ void __launch_bounds__(256) permute_count_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                            int n_shared, int32_t* __restrict__ cnt,
                                                            int32_t* __restrict__ rank, int32_t* __restrict__ offsets,
                                                            unsigned int* counter, int* status, int* zero,
                                                            size_t zero_words) {
    extern __shared__ uint32_t sm[];
    __shared__ int32_t tot[kMaxGroups];
    __shared__ bool s_last;
    uint32_t* flags = sm;                                      // [8][E] membership bitmaps
    uint16_t* pre = reinterpret_cast<uint16_t*>(sm + 8 * E);  // [8][E] rows of earlier warps
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) flags[i] = 0;
    pdl_wait();
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < zero_words; i += (size_t)gridDim.x * blockDim.x)
        zero[i] = 0;
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

    // ---- the last CTA to get here scans
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(counter, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int nchunk = gridDim.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int c0 = 0; c0 < nchunk; c0 += 8) {
            int v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = (c0 + i < nchunk) ? __ldcg(cnt + (size_t)(c0 + i) * E + e) : 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (c0 + i < nchunk) {
                    cnt[(size_t)(c0 + i) * E + e] = run;
                    run += v[i];
                }
        }
        tot[e] = run;
    }
    for (int s = threadIdx.x; s < n_shared; s += blockDim.x) tot[E + s] = T;
    __syncthreads();
    block_exclusive_scan_256(tot, E + n_shared, offsets);
    if (threadIdx.x == 0) *counter = 0u;
}

// Token t's row of x to its nd destination rows s_dst[] (-1: none) of x_perm, by the
// whole CTA in 16-byte vectors: a copy (bf16) or a quantised copy (E4M3 + scales).
template <bool FP8>
__device__ __forceinline__ void scatter_row(const uint16_t* __restrict__ x, int t, int H, int nd, const int* s_dst,
                                            void* __restrict__ x_perm, float* __restrict__ x_scale, int64_t A) {
    const int nvec = H / 8;
    for (int v0 = 0; v0 < nvec; v0 += blockDim.x) {
        const int v = v0 + threadIdx.x;
        const bool act = v < nvec;  // nvec is a multiple of 16: a 128-wide block is all in or all out
        const uint4 xv = act ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H) + v) : make_uint4(0, 0, 0, 0);
        if constexpr (!FP8) {
            if (!act) break;
            for (int d = 0; d < nd; ++d) {
                const int D = s_dst[d];
                if (D >= 0) reinterpret_cast<uint4*>(static_cast<uint16_t*>(x_perm) + (size_t)D * H)[v] = xv;
            }
        } else {
            // 16 threads x 8 values = one 128-wide block: amax, s = amax/448 (1 if 0),
            // code = E4M3(x/s) with round-to-nearest-even and saturation, all in fp32.
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
            if (!act) break;
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
                const int D = s_dst[d];
                if (D >= 0) {
                    reinterpret_cast<uint2*>(static_cast<uint8_t*>(x_perm) + (size_t)D * H)[v] = make_uint2(lo, hi);
                    if ((threadIdx.x & 15) == 0) x_scale[(size_t)blk * A + D] = s;
                }
            }
        }
    }
}

// blockIdx.x = token: the destinations of its k routed slots and n_shared shared rows
// are looked up once, perm / inv_perm written, then the CTA streams the row in 16-byte
// vectors (kScatterThreads at a time): a copy (bf16) or a quantised copy (E4M3 + scales).
template <bool FP8>
__global__ void __launch_bounds__(kScatterThreads) permute_scatter_kernel(
    const int32_t* __restrict__ ids, const int32_t* __restrict__ rank, const int32_t* __restrict__ base,
    const int32_t* __restrict__ offsets, const uint16_t* __restrict__ x, int T, int H, int k, int E, int n_shared,
    int64_t A, int32_t* __restrict__ perm, int32_t* __restrict__ inv, void* __restrict__ x_perm,
    float* __restrict__ x_scale, int* status) {
    __shared__ int s_dst[32];
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x;
    const int nd = k + n_shared;
    if (threadIdx.x < nd) {
        const int d = threadIdx.x;
        int64_t dst = -1;
        if (d < k) {
            const int e = ids[(size_t)t * k + d];
            const int r = rank[(size_t)t * k + d];
            if (e >= 0 && e < E && r >= 0) dst = (int64_t)offsets[e] + base[(size_t)(t / kChunk) * E + e] + r;
        } else {
            dst = (int64_t)offsets[E + (d - k)] + t;
        }
        if (dst >= A) {
            set_status(status, MOE_ERR_EXPERT_ID);
            dst = -1;
        }
        s_dst[d] = (int)dst;
        if (d < k) inv[(size_t)t * k + d] = (int)dst;
        if (dst >= 0) perm[dst] = t;
    }
    __syncthreads();
    scatter_row<FP8>(x, t, H, nd, s_dst, x_perm, x_scale, A);
}

// Batches of at most one counting chunk (T <= 256) in one launch: CTA t stages all T*k
// ids in shared memory, counts the rows of every group and scans them (every CTA does the
// same; CTA 0 writes offsets), ranks its own slots among earlier tokens' rows of the same
// expert (the stable (expert, token, slot) order), and scatters its row. Ids outside
// [0, E) or repeated within a token are flagged by the CTA of that token.
template <bool FP8>
__global__ void __launch_bounds__(kScatterThreads) permute_small_kernel(
    const int32_t* __restrict__ ids, const uint16_t* __restrict__ x, int T, int H, int k, int E, int n_shared,
    int64_t A, int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    void* __restrict__ x_perm, float* __restrict__ x_scale, int* status, int* zero, size_t zero_words) {
    extern __shared__ int32_t sm_small[];
    const int G = E + n_shared;
    int32_t* s_ids = sm_small;             // [T*k]
    int32_t* s_cnt = s_ids + T * k;        // [G]
    int32_t* s_off = s_cnt + G;            // [G+1]
    int32_t* s_mark = s_off + G + 1;       // [E]: 1 + slot of this token routed to e, else 0
    __shared__ int s_dst[32];
    __shared__ int s_rank[32];
    pdl_trigger();
    for (int g = threadIdx.x; g < G; g += blockDim.x) s_cnt[g] = g < E ? 0 : T;
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_mark[e] = 0;
    if (threadIdx.x < 32) s_rank[threadIdx.x] = 0;
    pdl_wait();
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < zero_words; i += (size_t)gridDim.x * blockDim.x)
        zero[i] = 0;
    const int t = blockIdx.x;
    __syncthreads();
    for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
        const int e = ids[i];
        s_ids[i] = e;
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    if (threadIdx.x < k) {  // this token's slots: valid and distinct
        const int j = threadIdx.x, e = s_ids[t * k + j];
        bool good = e >= 0 && e < E;
        for (int j2 = 0; j2 < j && good; ++j2) good = s_ids[t * k + j2] != e;
        if (!good) set_status(status, MOE_ERR_EXPERT_ID);
        else s_mark[e] = j + 1;  // distinct valid ids: one writer per expert
    }
    block_exclusive_scan_256(s_cnt, G, s_off);
    __syncthreads();
    for (int i = threadIdx.x; i < t * k; i += blockDim.x) {  // earlier tokens' rows of this token's experts
        const int e = s_ids[i];
        if (e >= 0 && e < E) {
            const int m = s_mark[e];
            if (m) atomicAdd(&s_rank[m - 1], 1);
        }
    }
    if (t == 0)
        for (int g = threadIdx.x; g <= G; g += blockDim.x) offsets[g] = s_off[g];
    __syncthreads();
    const int nd = k + n_shared;
    if (threadIdx.x < nd) {
        const int d = threadIdx.x;
        int64_t dst = -1;
        if (d < k) {
            const int e = s_ids[t * k + d];
            if (e >= 0 && e < E && s_mark[e] == d + 1) dst = (int64_t)s_off[e] + s_rank[d];
        } else {
            dst = (int64_t)s_off[E + (d - k)] + t;
        }
        if (dst >= A) {
            set_status(status, MOE_ERR_EXPERT_ID);
            dst = -1;
        }
        s_dst[d] = (int)dst;
        if (d < k) inv[(size_t)t * k + d] = (int)dst;
        if (dst >= 0) perm[dst] = t;
    }
    __syncthreads();
    scatter_row<FP8>(x, t, H, nd, s_dst, x_perm, x_scale, A);
}

cudaError_t launch_permute(const int32_t* ids, const void* x, int T, int H, int k, int E, int n_shared, bool fp8,
                           int32_t* offsets, int32_t* perm, int32_t* inv, void* x_perm, float* x_scale,
                           void* scratch, unsigned int* counter, int* status, cudaStream_t stream, int* zero,
                           size_t zero_words) {
    const int G = E + n_shared;
    if (T == 0) return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (G + 1), stream);
    if (G > kMaxGroups) return cudaErrorInvalidValue;
    const int nchunk = (T + kChunk - 1) / kChunk;
    const int64_t A = (int64_t)T * (k + n_shared);
    if (nchunk == 1) {  // one launch: counting, scan and scatter per token
        const size_t sm = sizeof(int32_t) * ((size_t)T * k + 2 * (size_t)G + 1 + (size_t)E);
        if (sm > 48 * 1024) {
            cudaError_t e2 = cudaFuncSetAttribute(fp8 ? permute_small_kernel<true> : permute_small_kernel<false>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            if (e2 != cudaSuccess) return e2;
        }
        return launch_pdl(fp8 ? permute_small_kernel<true> : permute_small_kernel<false>, dim3(T), dim3(kScatterThreads),
                          sm, stream, ids, static_cast<const uint16_t*>(x), T, H, k, E, n_shared, A, offsets, perm,
                          inv, x_perm, x_scale, status, zero, zero ? zero_words : (size_t)0);
    }
    int32_t* cnt = static_cast<int32_t*>(scratch);
    int32_t* rank = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) +
                                               (((size_t)nchunk * E * sizeof(int32_t) + 255) & ~size_t(255)));
    const size_t sm1 = (size_t)8 * E * sizeof(uint32_t) + (size_t)8 * E * sizeof(uint16_t);
    cudaError_t err;
    if (sm1 > 40 * 1024) {
        err = cudaFuncSetAttribute(permute_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
        if (err != cudaSuccess) return err;
    }
    err = launch_pdl(permute_count_kernel, dim3(nchunk), dim3(256), sm1, stream, ids, T, k, E, n_shared, cnt, rank,
                     offsets, counter, status, zero, zero ? zero_words : (size_t)0);
    if (err != cudaSuccess) return err;
    return launch_pdl(fp8 ? permute_scatter_kernel<true> : permute_scatter_kernel<false>, dim3(T), dim3(kScatterThreads),
                      0, stream, ids, static_cast<const int32_t*>(rank), static_cast<const int32_t*>(cnt), offsets,
                      static_cast<const uint16_t*>(x), T, H, k, E, n_shared, A, perm, inv, x_perm, x_scale, status);
}

}  // namespace moe
