// internal.h -- launchers shared between the translation units of the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "moe_b200.h"

namespace moe {

cudaError_t launch_router(const float* logits, int T, int N, int S, int k, int score, float route_scale,
                          int32_t* ids, float* w, float* sw, cudaStream_t stream);

// Scratch of the permutation: per 256-token chunk counts/bases [nchunk][E] and the
// in-chunk rank of every (token, slot) [T][k].
size_t permute_scratch_bytes(int T, int k, int E);
cudaError_t launch_permute(const int32_t* ids, const void* x, int T, int H, int k, int E, int n_shared, bool fp8,
                           int32_t* offsets, int32_t* perm, int32_t* inv, void* x_perm, float* x_scale,
                           void* scratch, int* status, cudaStream_t stream);

cudaError_t launch_combine(const void* y, const int32_t* offsets, const int32_t* inv, const float* topk_w,
                           const float* shared_w, int T, int H, int k, int E, int n_shared, int n_sink, void* out,
                           cudaStream_t stream);

// Grouped GEMM over the groups described by offsets. Weights are the MMA's M side
// (128 rows per tile), permuted activation rows the N side (BN rows per tile).
struct GemmArgs {
    const int32_t* offsets;  // [G+1]
    int G;
    int64_t A;               // rows of the activation matrix (tensor-map extent)
    int K;                   // reduction depth (H for GEMM1, I for GEMM2)
    int wrows;               // weight rows per group (2I for GEMM1, H for GEMM2)
    int n_chunks;            // 128-row output chunks per group (I/128 or H/128)
    int up_off;              // GEMM1: row offset of the up half inside a group (I)
    const void* act;         // activation matrix [A][K]
    const float* act_scale;  // FP8: [K/128][A]
    const void* w;           // weights [G][wrows][K]
    const float* w_scale;    // FP8: [G][wrows/128][K/128]
    void* out;               // GEMM1: h [A][I]; GEMM2: y [A][H] bf16
    float* out_scale;        // GEMM1 FP8: [I/128][A]
    int out_ld;              // I or H
    const float* gate_scale; // [G] or NULL
    const float* up_scale;   // [G] or NULL
    float alpha, beta, limit;
    int* status;
};

// Picks the token-tile width from the expected rows per group.
int gemm_pick_bn(int64_t A, int G, bool gated, bool fp8);
cudaError_t launch_gemm(const GemmArgs& a, bool gated, bool fp8, int bn, cudaStream_t stream);

int num_sms();

}  // namespace moe
