// internal.h -- launchers shared between the translation units of the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "moe_b200.h"

namespace moe {

// Programmatic dependent launch. Every kernel of the library is launched with
// launch_pdl, so it may start while the previous kernel on the stream is finishing; each
// kernel calls pdl_wait() before it touches global memory (which waits for the previous
// grid to complete and its writes to be visible), so the order of completion stays that
// of the stream and only launch latency and prologues overlap. pdl_trigger() lets the
// next kernel launch: the small kernels call it on entry, the grouped-GEMM kernel when a
// CTA runs out of tiles. A dependent grid starts only after every CTA of its predecessor
// has triggered or exited, so it never takes resources that a pending predecessor CTA
// needs. Without the launch attribute (or with a plain predecessor) both are no-ops.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
#endif

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// bias [N] or NULL (rank on the raw logit); packed [T][k] or NULL.
cudaError_t launch_router(const float* logits, const float* bias, int T, int N, int S, int k, int score,
                          float route_scale, int32_t* ids, float* w, float* sw, uint32_t* packed, cudaStream_t stream);

// Fused gate GEMV + router for T <= kGateMaxTokens: logits[T][N+S] = x[T][H] . wg[N+S][H]^T
// (bf16 in, fp32 accumulation), then the router. `counter`: one word, zero when idle,
// left at zero.
constexpr int kGateMaxTokens = 16;
cudaError_t launch_gate_route(const void* x, const void* wg, const float* bias, int T, int H, int N, int S, int k,
                              int score, float route_scale, float* logits, int32_t* ids, float* w, float* sw,
                              uint32_t* packed, unsigned int* counter, cudaStream_t stream);

// Scratch of the permutation: per 256-token chunk counts/bases [nchunk][E] and the
// in-chunk rank of every (token, slot) [T][k]. `counter` is one word that must be zero
// before the first call; every call leaves it at zero.
size_t permute_scratch_bytes(int T, int k, int E);
// `zero`/`zero_words`: an optional buffer the counting kernel clears on the way (the
// GEMM's per-block flags of the same layer pass).
cudaError_t launch_permute(const int32_t* ids, const void* x, int T, int H, int k, int E, int n_shared, bool fp8,
                           int32_t* offsets, int32_t* perm, int32_t* inv, void* x_perm, float* x_scale,
                           void* scratch, unsigned int* counter, int* status, cudaStream_t stream,
                           int* zero = nullptr, size_t zero_words = 0);

cudaError_t launch_combine(const void* y, const int32_t* offsets, const int32_t* inv, const float* topk_w,
                           const float* shared_w, int T, int H, int k, int E, int n_shared, int n_sink, int64_t A,
                           void* out, int* status, cudaStream_t stream);

// Grouped GEMM1 (+ SwiGLU) and/or GEMM2 over the groups described by offsets, in one
// persistent launch. Weights are the MMA's M side (128 rows per tile), permuted token
// rows the N side. With both phases, GEMM2 tiles of a token block start once the
// block's GEMM1 tiles have published h (done1 counters, zero at launch).
struct MoeGemmArgs {
    const int32_t* offsets;  // [G+1]
    int G;
    int64_t A;               // rows of x_perm / h / y
    int H, I;
    bool fp8;
    bool int4;               // 4-bit weights, INT4 group-32 or NVFP4 (bf16 activations)
    bool fp4;                // the 4-bit weights are NVFP4 (E2M1, E4M3 scale per 16 K)
    bool run_gemm1, run_gemm2;
    const void* x_perm;      // [A][H]
    const float* x_scale;    // FP8: [H/128][A]
    const void* w1;          // [G][2I][H]
    const void* w1_scale;    // FP8: fp32 [G][2I/128][H/128]; INT4: bf16 [G][2I][H/32]; NVFP4: E4M3 [G][2I][H/16]
    const float* gate_scale; // [G] or NULL
    const float* up_scale;   // [G] or NULL
    float alpha, beta, limit;
    const float* limits;     // [G] per-group clamp (replaces limit) or NULL
    void* h;                 // [A][I]
    float* h_scale;          // FP8: [I/128][A]
    const void* w2;          // [G][H][I]
    const void* w2_scale;    // FP8: fp32 [G][H/128][I/128]; INT4: bf16 [G][H][I/32]; NVFP4: E4M3 [G][H][I/16]
    void* y;                 // [A][H] bf16
    unsigned int* tile_ctr;  // zero when idle; left at zero
    unsigned int* exit_ctr;  // zero when idle; left at zero
    int* done1;              // gemm_block_flags_bytes(A, G), zeroed before a two-phase launch
    float* part;             // split-K partials of GEMM1 (gemm_split_scratch_bytes), or NULL
    int* split_cnt;          // per GEMM1 tile: splits finished (zero when idle), or NULL
    int* status;
};

int gemm_pick_bn(int64_t A, int G, int wdtype);
// Process-wide choice of the FP8 CTA-pair layout (moe_set_option): returns the old value.
int gemm_set_fp8_pair(int enable);
// The same for bf16 layers with 256-row token blocks (MOE_OPT_BF16_CTA_PAIR).
int gemm_set_bf16_pair(int enable);
// Upper bound on token blocks: every non-empty group adds at most one partial block.
int64_t gemm_max_blocks(int64_t A, int G, int bn);
size_t gemm_block_flags_bytes(int64_t A, int G);
// Tile width, GEMM1 split-K factor (1, 2 or 4) for these sizes and weight format (moe_wdtype), and the scratch it needs: fp32
// partials [tiles][splits][2][BN][128] plus one counter per GEMM1 tile.
int gemm_split_factor(int64_t A, int G, int H, int I, int wdtype);
size_t gemm_split_scratch_bytes(int64_t A, int G, int H, int I, int wdtype);
size_t gemm_split_counter_bytes(int64_t A, int G, int H, int I, int wdtype);
cudaError_t launch_moe_gemm(const MoeGemmArgs& a, cudaStream_t stream);
cudaError_t launch_ep_row_ids(const int32_t* offsets, int G, int A, int32_t* row_ids, cudaStream_t stream);
cudaError_t launch_ep_rebase(const int32_t* ids, int64_t n, int E, int n_shared, int local_offset, int n_local,
                             int32_t* out, cudaStream_t stream);

int num_sms();

}  // namespace moe
