// combine.cu -- routing-weighted unpermute: out[t] = sum_j w[t,j] * y[inv[t,j]] +
// sum_s gamma[t,s] * y[shared row of t], in fp32 in that fixed slot order, rounded once
// to bf16 (slot-specific routing-weight reduction with fp32 accumulation, batchgen
// PR #239 commit notes; shared-sink weights gamma from sglang PR #36385 item 3).
#include <cuda_bf16.h>

#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y, const int32_t* __restrict__ offsets,
                                                      const int32_t* __restrict__ inv, const float* __restrict__ topk_w,
                                                      const float* __restrict__ shared_w, int T, int H, int k, int E,
                                                      int n_shared, int n_sink, uint16_t* __restrict__ out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    int r = -1;
    float wt = 0.f;
    if (lane < k) {
        r = inv[(size_t)t * k + lane];
        wt = topk_w[(size_t)t * k + lane];
    } else if (lane < k + n_shared) {
        r = offsets[E + (lane - k)] + t;
        wt = n_sink > 0 ? shared_w[(size_t)t * n_sink + (lane - k)] : 1.f;
    }
    const int nd = k + n_shared;
    const int nvec = H / 8;
    // Warp-uniform trip count: every lane takes part in the shuffles below.
    for (int v0 = 0; v0 < nvec; v0 += 32) {
        const int v = v0 + lane;
        const bool act = v < nvec;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int d = 0; d < nd; ++d) {
            const int R = __shfl_sync(0xffffffffu, r, d);
            const float W = __shfl_sync(0xffffffffu, wt, d);
            if (R < 0 || !act) continue;
            const uint4 yv = __ldg(reinterpret_cast<const uint4*>(y + (size_t)R * H) + v);
            const uint32_t wv[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = fmaf(W, __uint_as_float(wv[i] << 16), acc[2 * i]);
                acc[2 * i + 1] = fmaf(W, __uint_as_float(wv[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            o[i] = *reinterpret_cast<const uint32_t*>(&p);
        }
        if (act) reinterpret_cast<uint4*>(out + (size_t)t * H)[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

cudaError_t launch_combine(const void* y, const int32_t* offsets, const int32_t* inv, const float* topk_w,
                           const float* shared_w, int T, int H, int k, int E, int n_shared, int n_sink, void* out,
                           cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    combine_kernel<<<(T + 7) / 8, 256, 0, stream>>>(static_cast<const uint16_t*>(y), offsets, inv, topk_w, shared_w,
                                                    T, H, k, E, n_shared, n_sink, static_cast<uint16_t*>(out));
    return cudaGetLastError();
}

}  // namespace moe
