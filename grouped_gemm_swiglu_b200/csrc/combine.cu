// combine.cu -- routing-weighted unpermute: out[t] = sum_j w[t,j] * y[inv[t,j]] +
// sum_s gamma[t,s] * y[shared row of t], in fp32 in that fixed slot order, rounded once
// to bf16 (slot-specific routing-weight reduction with fp32 accumulation, batchgen
// PR #239 commit notes; shared-sink weights gamma from sglang PR #36385 item 3).
//
// One CTA per token, one thread per 8 output columns (16 bytes) at a time: the token's
// source rows and weights are looked up once, and each thread issues the loads of eight
// rows back to back (predicated, no branch) before it accumulates them in slot order, so
// the kernel runs at the memory system's rate instead of one dependent chain per row.
#include <cuda_bf16.h>

#include "internal.h"
#include "status.cuh"

namespace moe {

constexpr int kCombineThreads = 256;
constexpr int kCombineBatch = 8;  // row loads in flight per thread

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const uint16_t* __restrict__ y, const int32_t* __restrict__ offsets, const int32_t* __restrict__ inv,
    const float* __restrict__ topk_w, const float* __restrict__ shared_w, int T, int H, int k, int E, int n_shared,
    int n_sink, int64_t A, uint16_t* __restrict__ out, int* status) {
    __shared__ int s_row[32];
    __shared__ float s_w[32];
    pdl_trigger();
    pdl_wait();
    const int t = blockIdx.x;
    const int nd = k + n_shared;
    if (threadIdx.x < nd) {
        const int d = threadIdx.x;
        int64_t r;
        float wt;
        if (d < k) {
            r = inv[(size_t)t * k + d];
            wt = topk_w[(size_t)t * k + d];
        } else {
            r = (int64_t)offsets[E + (d - k)] + t;
            wt = n_sink > 0 ? shared_w[(size_t)t * n_sink + (d - k)] : 1.f;
        }
        if (r >= A) {  // never read past the intermediate, whatever the routing data says
            set_status(status, MOE_ERR_EXPERT_ID);
            r = -1;
        }
        s_row[d] = (int)r;
        s_w[d] = wt;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < H / 8; v += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int d0 = 0; d0 < nd; d0 += kCombineBatch) {
            uint4 yv[kCombineBatch];
#pragma unroll
            for (int b = 0; b < kCombineBatch; ++b) {  // all loads first; missing rows read as zero
                const int d = d0 + b;
                const int R = d < nd ? s_row[d] : -1;
                yv[b] = R >= 0 ? __ldg(reinterpret_cast<const uint4*>(y + (size_t)R * H) + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int b = 0; b < kCombineBatch; ++b) {  // then the sums, in slot order
                const int d = d0 + b;
                const float W = (d < nd && s_row[d] >= 0) ? s_w[d] : 0.f;
                const uint32_t wv[4] = {yv[b].x, yv[b].y, yv[b].z, yv[b].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] = fmaf(W, __uint_as_float(wv[i] << 16), acc[2 * i]);
                    acc[2 * i + 1] = fmaf(W, __uint_as_float(wv[i] & 0xFFFF0000u), acc[2 * i + 1]);
                }
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            o[i] = *reinterpret_cast<const uint32_t*>(&p);
        }
        reinterpret_cast<uint4*>(out + (size_t)t * H)[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

cudaError_t launch_combine(const void* y, const int32_t* offsets, const int32_t* inv, const float* topk_w,
                           const float* shared_w, int T, int H, int k, int E, int n_shared, int n_sink, int64_t A,
                           void* out, int* status, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    return launch_pdl(combine_kernel, dim3(T), dim3(kCombineThreads), 0, stream, static_cast<const uint16_t*>(y), offsets,
                      inv, topk_w, shared_w, T, H, k, E, n_shared, n_sink, A, static_cast<uint16_t*>(out), status);
}

}  // namespace moe
