/*
 * moe_b200.h -- C ABI of the routed mixture-of-experts expert layer for NVIDIA B200
 * (sm_100a). The layer runs, per call and entirely on the GPU:
 *
 *   router / gate epilogue  ->  permute by expert  ->  grouped GEMM1 (gate|up) with a
 *   clamped, parameterised SwiGLU epilogue  ->  grouped GEMM2 (down)  ->  routing-
 *   weighted combine.
 *
 * Sources of the operations (web pages, cited by title and section):
 *   [P2] sglang PR #39920 "Fix flashinfer_trtllm silently dropping swiglu_limit",
 *        "Modifications": gate = clamp(gate, max=L), up = clamp(up, -L, L),
 *        out = gate * sigmoid(alpha * gate) * (up + beta); "Motivation": GLM FP8
 *        blockwise 128x128, 288 routed experts, top-8, 1 shared expert, L = 10.
 *   [P3] sglang PR #36385 "Enable and fuse the Inkling MoE gate epilogue on Intel XPU",
 *        items 2-3: masked-max top-k, ties to the lower expert id, weights
 *        exp(lp - logsumexp(lp)) with lp = logsigmoid(x), shared-sink columns that
 *        join the normaliser but never the top-k, a scalar routing scale, ranking on
 *        sigmoid(logit) + bias with the raw logit carried out, the packed
 *        (id << 16 | bf16 weight) output.
 *   [P2'] the same sglang PR #39920, "Speed Tests and Profiling": the clamp limit as one
 *        fp32 value per expert.
 *   [P4] DeepGEMM PR #445 "fix(sm90): support parameterized SwiGLU in FP8 MegaMoE",
 *        "Summary"/"Compatibility": alpha, up_bias (beta) and clamp as explicit
 *        parameters; alpha = 1, beta = 0, no clamp is the standard SwiGLU.
 *   [P1] xorl-wheels "FlashInfer 0.6.18 SM100a+SM103a MoE-LoRA AOT", "Changes":
 *        activation quantisation fused into the activation kernel; gate and up halves
 *        carry separate scales that apply before the activation; routing ids outside
 *        the expert range are an error.
 *   [P5] batchgen PR #239 "sm100: Fused INT4 grouped + SiLU Triton kernel": per-expert
 *        sorted-token dispatch, fp32 accumulation, slot-specific weighted reduction.
 *   [P1'] the same xorl-wheels release, "Changes": expert-parallel lookups are rank-local;
 *        routing ids stay global, each rank rebases them by its local expert offset and
 *        bounds-checks them against its local expert count, and ids outside that range
 *        are an error.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer on the current CUDA device unless
 *     stated otherwise; the caller owns (allocates and frees) every buffer. The
 *     library never allocates, frees or synchronises on the hot path.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream) and returns before it runs. Calls are capturable in a CUDA graph.
 *   - Arguments are checked on the host first. A bad argument returns a negative
 *     moe_status and enqueues nothing. A kernel launch failure returns MOE_ERR_CUDA.
 *   - Errors found while the kernels run (an expert id outside [0, E) or repeated
 *     within a token, offsets or inverse-permutation entries outside [0, A], a pipeline
 *     wait that exceeded its time limit) are written to a status word at the start of
 *     the workspace `ws`; read it with moe_read_status(). It is sticky until
 *     moe_clear_status(). Offending entries are dropped or clamped, never used to read
 *     or write out of bounds. No kernel traps.
 *   - Row-major layouts throughout. bf16 is stored as 16-bit words, E4M3 as bytes.
 *   - Calls that share a workspace or outputs must not overlap on the GPU.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 7

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,  /* a size, pointer or parameter outside the documented range */
    MOE_ERR_UNSUPPORTED = -2,  /* a valid combination this library does not implement */
    MOE_ERR_ARCH = -3,         /* the current device is not compute capability 10.x */
    MOE_ERR_WORKSPACE = -4,    /* ws is NULL, misaligned (256 B) or smaller than required */
    MOE_ERR_EXPERT_ID = -5,    /* (device) routing data out of range: an id outside [0, E) or
                                  repeated in a token, offsets / inv_perm outside [0, A] */
    MOE_ERR_TIMEOUT = -6,      /* (device) a pipeline wait exceeded its limit; outputs invalid */
    MOE_ERR_CUDA = -7          /* a CUDA runtime/driver call failed */
} moe_status;

typedef enum moe_score_fn {
    MOE_SCORE_SOFTMAX = 0,     /* weights = softmax over the k selected logits          */
    MOE_SCORE_SIGMOID = 1      /* weights = exp(lp - logsumexp(lp)), lp = logsigmoid(x),
                                  over the k selected columns plus the sink columns      */
} moe_score_fn;

typedef enum moe_wdtype {
    MOE_WDTYPE_BF16 = 0,             /* bf16 weights and activations                       */
    MOE_WDTYPE_FP8_E4M3_BLOCK128 = 1, /* E4M3 weights with one fp32 scale per 128x128 block;
                                        E4M3 activations with one fp32 scale per 1x128 block */
    MOE_WDTYPE_INT4_G32 = 2,         /* [P5] INT4 weights, two per byte (low nibble = even K),
                                        one bf16 scale per 32 K per row, value
                                        bf16((nibble - 8) * scale); bf16 activations       */
    MOE_WDTYPE_NVFP4 = 3             /* [P1] NVFP4 weights: E2M1 values (1 sign, 2 exponent
                                        bits with bias 1, 1 mantissa bit), two per byte (low
                                        nibble = even K), one E4M3 scale per 16 K per row,
                                        value E2M1 * E4M3 (exact in bf16); the checkpoint's
                                        per-expert gate / up global scales are gate_scale /
                                        up_scale; bf16 activations                          */
} moe_wdtype;

/* Problem statement. All fields are read on every call.
 *   T        tokens (>= 0; T = 0 is a no-op that still writes empty offsets)
 *   H        hidden size (multiple of 128)
 *   I        intermediate size per expert (multiple of 128)
 *   E        routed experts (1 .. 1024)
 *   k        experts per token (1 .. min(E, 32))
 *   n_sink   shared-sink columns after the E routed logits (0 .. 32-k; sigmoid only)
 *   n_shared always-on shared experts, stored after the routed ones in the weights;
 *            shared expert s is weighted by sink s when n_sink > 0 (then
 *            n_shared == n_sink), else by 1
 *   wdtype   moe_wdtype;  score  moe_score_fn
 *   alpha, beta  SwiGLU sigmoid slope and up bias ([P4] "Summary")
 *   limit    clamp L > 0; +INFINITY disables the clamp
 *   route_scale  scalar multiplying every routing weight (routed and sink), usually 1
 * Derived: G = E + n_shared weight groups; A = T*k + T*n_shared permuted rows. */
typedef struct moe_dims {
    int32_t T, H, I, E, k, n_sink, n_shared;
    int32_t wdtype;
    int32_t score;
    float alpha, beta, limit, route_scale;
} moe_dims;

/* Which call a workspace is sized for (moe_workspace_size). */
typedef enum moe_ws_kind {
    MOE_WS_PERMUTE = 0,
    MOE_WS_GEMM1 = 1,
    MOE_WS_GEMM2_COMBINE = 2,
    MOE_WS_FORWARD = 3,
    MOE_WS_EXPERTS = 4,
    MOE_WS_COMBINE = 5,
    MOE_WS_GATE_ROUTE = 6
} moe_ws_kind;

/* ABI version compiled into the library (MOE_ABI_VERSION). */
int moe_abi_version(void);

/* Process-wide options (moe_set_option). No counterpart on the pages: a choice between
 * two kernel layouts that compute the same thing.
 *   MOE_OPT_FP8_CTA_PAIR: FP8 layers whose groups average more than 128 rows.
 *     0 (default): one CTA per 128-token tile, both weight blocks of a tile loaded by it.
 *     1: two CTAs of a cluster share each tensor-core MMA (tcgen05 cta_group::2) over a
 *        256-token tile, each loading its own 128 token rows and one of the two weight
 *        blocks, so each SM moves a third fewer bytes from L2. Measured on the GLM-shaped
 *        FP8 prefill it runs at the same speed as the default (2.67 against 2.61 ms).
 *     Results agree to the FP8 tolerance, not necessarily bit for bit (the tensor core's
 *     summation order within a K block may differ between the two layouts).
 *   MOE_OPT_BF16_CTA_PAIR: bf16 layers whose groups average more than 128 rows (256-row
 *     token blocks).
 *     0 (default): one CTA per 256-token tile with the weight rows as the MMA's M side;
 *        the tile's gate and up sums fill all of tensor memory, so the tensor core waits
 *        while the epilogue drains them.
 *     1: a CTA pair per 256-token tile with the token rows as M (128 per CTA) and each CTA
 *        loading one of the two 128-row weight blocks: the same bytes per SM from L2, and
 *        two accumulator buffers, so one tile's drain overlaps the next tile's MMAs.
 *        Measured on the Qwen3-shaped bf16 prefill it is slower than the default (417
 *        against 349 us for the grouped GEMMs: each stage waits for both CTAs' copies).
 *     Results agree to the bf16 tolerance (the summation order may differ). */
typedef enum moe_option {
    MOE_OPT_FP8_CTA_PAIR = 1,
    MOE_OPT_BF16_CTA_PAIR = 2
} moe_option;

/* Sets a process-wide option for calls made after it returns (a CUDA graph keeps the
 * layout chosen when it was captured). Thread-safe. Returns the previous value, or
 * MOE_ERR_INVALID_ARG for an unknown option or value (nothing changes then). */
int moe_set_option(int option, int value);

/* Static string for a moe_status value. Never NULL. */
const char* moe_status_string(int status);

/* Bytes of device workspace the given call needs for these dims (written to *bytes).
 * The workspace must be 256-byte aligned. Its first 256 bytes hold the status word and
 * a completion counter of the permutation; zero them once (moe_clear_status) before
 * first use. Every call leaves the counter at zero again. */
int moe_workspace_size(const moe_dims* dims, int kind, size_t* bytes);

/* Copies the workspace's device status word to *status (host). Synchronises `stream`.
 * Not for the hot path. */
int moe_read_status(const void* ws, int32_t* status, void* stream);

/* Zeroes the workspace's status word (asynchronous, on `stream`). */
int moe_clear_status(void* ws, void* stream);

/* Router / gate epilogue ([P3] items 2 and 3).
 *   logits   [T][E + n_sink] fp32, read only. Finite values required.
 *   bias     [E] fp32 correction bias of the routed columns, or NULL. With NULL the ranking
 *            key is the raw logit (which orders like sigmoid(logit)); with a bias it is
 *            sigmoid(logit) + bias[e], both evaluated in fp32 (sigmoid saturates there:
 *            ties are then broken by the bias, then by the lower id). Sink columns take no
 *            bias. Sigmoid scoring only (else MOE_ERR_UNSUPPORTED).
 *   topk_ids [T][k] int32 out: per token, the k routed columns with the largest key,
 *            in descending order; equal keys go to the lower id.
 *   topk_w   [T][k] fp32 out: routing weights in the same order, times route_scale.
 *            softmax: exp(l_j - logsumexp(l_sel)); sigmoid: exp(lp_j - logsumexp(lp over
 *            the selected and the sink columns)), lp = logsigmoid(l) of the RAW logit
 *            (never the biased key) -- finite even when every logit is below -104.
 *   shared_w [T][n_sink] fp32 out (NULL iff n_sink == 0): the sink columns' weights.
 *   packed   [T][k] uint32 out, or NULL: (topk_ids << 16) | bf16 bits of topk_w
 *            (round to nearest even). Ids fit 16 bits (E <= 1024).
 * Errors: INVALID_ARG (sizes, NULL pointers, n_sink > 0 with softmax), UNSUPPORTED (bias
 * with softmax), ARCH, CUDA. */
int moe_route_topk(const float* logits, const moe_dims* dims, const float* bias, int32_t* topk_ids,
                   float* topk_w, float* shared_w, uint32_t* packed, void* stream);

/* Gate GEMV fused with the router, for decode-sized batches ([P3]: the gate's fused GEMV
 * path taken at <= 4 tokens, where the op is submission-bound; item 3 for the epilogue).
 * One launch computes
 *   logits[t][c] = sum_h x[t][h] * w_gate[c][h]     (bf16 products, fp32 accumulation;
 *                                                    per column, per-warp partial sums over
 *                                                    H/4 elements added in a fixed order)
 * for the E routed and n_sink sink columns, then routes every token exactly as
 * moe_route_topk does on those logits.
 *   x        [T][H] bf16, 16-byte aligned; T <= 16 (larger T: a GEMM, then moe_route_topk;
 *            UNSUPPORTED here).
 *   w_gate   [E + n_sink][H] bf16, 16-byte aligned (row c = gate column c).
 *   bias, topk_ids, topk_w, shared_w, packed   as moe_route_topk.
 *   logits   [T][E + n_sink] fp32 out, or NULL to keep them in the workspace.
 *   ws       moe_workspace_size(MOE_WS_GATE_ROUTE): the header (a completion counter that
 *            every call leaves at zero) and room for the logits.
 * Errors: INVALID_ARG, UNSUPPORTED (T > 16, bias with softmax), WORKSPACE, ARCH, CUDA. */
int moe_gate_route(const void* x, const void* w_gate, const moe_dims* dims, const float* bias,
                   float* logits, int32_t* topk_ids, float* topk_w, float* shared_w,
                   uint32_t* packed, void* ws, size_t ws_bytes, void* stream);

/* Permute by expert ([P5]: per-expert sorted-token dispatch; [P1]: fused act-quant).
 *   topk_ids [T][k] int32 in: expert ids in [0, E), distinct within a token.
 *            Ids outside the range set MOE_ERR_EXPERT_ID in the status word; those
 *            entries are dropped (never read out of bounds).
 *   x        [T][H] bf16 in.
 *   offsets  [G+1] int32 out: group g occupies rows [offsets[g], offsets[g+1]); groups
 *            0..E-1 are the routed experts, E..G-1 the shared experts (T rows each).
 *   perm     [A] int32 out: source token of each permuted row. Within a group rows are
 *            ordered by token, then slot (deterministic).
 *   inv_perm [T][k] int32 out: the row that holds slot j of token t.
 *   x_perm   [A][H] out: x[perm[r]] as bf16 (wdtype BF16) or as E4M3 codes (FP8), where
 *            each 1x128 block is quantised with s = amax/448 (1 if amax = 0), code =
 *            E4M3 round-to-nearest-even, saturating, of x/s (fp32 arithmetic).
 *   x_scale  [H/128][A] fp32 out (FP8 only, else may be NULL): s per block, block-major.
 *   ws       workspace of moe_workspace_size(MOE_WS_PERMUTE) bytes.
 * Errors: INVALID_ARG, WORKSPACE, ARCH, CUDA. */
int moe_permute(const int32_t* topk_ids, const void* x, const moe_dims* dims,
                int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                void* x_perm, float* x_scale, void* ws, size_t ws_bytes, void* stream);

/* moe_permute_noalloc -- the same permutation as moe_permute for callers that cannot
 * allocate device memory: no workspace argument, and the library allocates nothing.
 * (The pages have no counterpart; this is a deployment convenience.)
 * Which callers: those whose device memory is laid out in advance by a host framework
 * (a serving engine that reserves the whole GPU, a static memory planner, a plugin
 * interface that passes only inputs and outputs), and latency-critical code where
 * cudaMalloc and the synchronisation it may cause are not allowed.
 *   Arguments as moe_permute, except: no ws/ws_bytes; `status` is an optional device
 *   int32 (NULL = not reported) where a routing id outside [0, E) or repeated within a
 *   token is recorded (first error wins, the caller zeroes it).
 *   Weight types: all four (BF16, FP8, INT4_G32, NVFP4), as moe_permute; only FP8
 *   quantises x_perm, the others copy it in bf16.
 *   Scratch: a 1 MiB array compiled into the library, one per GPU that loads it, held
 *   until the process exits. Calls needing more -- 256-byte-rounded
 *   ceil(T/256)*E*4 + T*k*4 bytes above 1 MiB - 256 (at k = 8, E = 288: T >= 28689)
 *   -- return MOE_ERR_WORKSPACE and enqueue nothing.
 *   The array's device address is looked up (cudaGetSymbolAddress) in the current
 *   context on every call made outside stream capture, so a context created after
 *   cudaDeviceReset is served correctly. Under capture the address of the last
 *   uncaptured call on the device is used: make one uncaptured call on each device
 *   (and again after a reset) before capturing; a captured call with none before it
 *   returns MOE_ERR_UNSUPPORTED.
 *   Every call shares the array: calls that overlap on the GPU (two streams, or two
 *   host threads) race and corrupt each other's results. Its first word counts the
 *   CTAs of a call that have finished counting; every call first clears it on its own
 *   stream (cudaMemsetAsync of 4 bytes), so a race damages only the calls that raced.
 *   The rest of the array is written by each call before it is read.
 * Errors: INVALID_ARG, WORKSPACE (too large), ARCH, CUDA. */
int moe_permute_noalloc(const int32_t* topk_ids, const void* x, const moe_dims* dims,
                        int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* x_perm,
                        float* x_scale, int32_t* status, void* stream);

/* Grouped GEMM1 with the SwiGLU epilogue ([P2] "Modifications", [P4] "Summary",
 * [P1] "Changes"). For every row r of group g:
 *   gate = s_g[g] * sum_c x_perm[r][c] * W1[g][i][c]       (i < I)
 *   up   = s_u[g] * sum_c x_perm[r][c] * W1[g][I + i][c]
 *   h[r][i] = min(gate, L) * sigmoid(alpha * min(gate, L)) * (clamp(up, -L, L) + beta)
 * accumulated in fp32 (FP8: per 128-deep K block, times x_scale * w1_scale).
 *   x_perm, x_scale, offsets   as written by moe_permute (A = offsets[G]).
 *   w1        [G][2I][H]: rows [0, I) gate, [I, 2I) up; bf16 or E4M3, or for INT4 and NVFP4
 *             [G][2I][H/2] packed bytes (16-byte aligned).
 *   w1_scale  FP8: fp32 [G][2I/128][H/128]; INT4: bf16 [G][2I][H/32]; NVFP4: E4M3 codes
 *             [G][2I][H/16] (both 4-byte aligned); else NULL.
 *   gate_scale, up_scale  [G] fp32 per-group scales, or NULL for 1.0.
 *   limits    [G] fp32 clamp L per group ([P2'] one value per expert), or NULL for
 *             dims->limit. Each value > 0; +INFINITY disables that group's clamp.
 *   h         [A][I] out: bf16, or E4M3 codes quantised per 1x128 block like x_perm.
 *   h_scale   [I/128][A] fp32 out (FP8 only, else NULL).
 * Errors: INVALID_ARG, WORKSPACE, ARCH, CUDA; TIMEOUT in the status word. */
int moe_gemm1_swiglu(const void* x_perm, const float* x_scale, const int32_t* offsets,
                     const void* w1, const void* w1_scale, const float* gate_scale,
                     const float* up_scale, const float* limits, const moe_dims* dims, void* h,
                     float* h_scale, void* ws, size_t ws_bytes, void* stream);

/* Grouped GEMM2 and the routing-weighted combine ([P5]: slot-specific weighted
 * reduction in fp32). y[r] = h[r] . W2[g]^T for each row r of group g (fp32
 * accumulation, stored as bf16 in the workspace), then for every token t
 *   out[t] = sum_{j<k} topk_w[t][j] * y[inv_perm[t][j]]
 *          + sum_{s<n_shared} gamma[t][s] * y[offsets[E+s] + t],
 *   gamma = shared_w[t][s] when n_sink > 0, else 1,
 * summed in fp32 in that fixed order and rounded once to bf16.
 *   h, h_scale, offsets  as written by moe_gemm1_swiglu / moe_permute.
 *   inv_perm [T][k], topk_w [T][k], shared_w [T][n_sink] (NULL iff n_sink == 0).
 *   w2       [G][H][I] bf16 or E4M3, or INT4 / NVFP4 [G][H][I/2] packed bytes; w2_scale FP8:
 *            fp32 [G][H/128][I/128], INT4: bf16 [G][H][I/32], NVFP4: E4M3 codes [G][H][I/16];
 *            else NULL.
 *   out      [T][H] bf16 out.
 * Errors: INVALID_ARG, WORKSPACE, ARCH, CUDA; TIMEOUT in the status word. */
int moe_gemm2_combine(const void* h, const float* h_scale, const int32_t* offsets,
                      const int32_t* inv_perm, const float* topk_w, const float* shared_w,
                      const void* w2, const void* w2_scale, const moe_dims* dims,
                      void* out, void* ws, size_t ws_bytes, void* stream);

/* Both grouped GEMMs in one persistent launch (the expert MLPs of every group):
 * h = SwiGLU(GEMM1) exactly as moe_gemm1_swiglu, then y[r] = h[r] . W2[g]^T (fp32
 * accumulation, bf16 out, unweighted) as the first half of moe_gemm2_combine. GEMM2 work
 * on a block of rows starts as soon as that block's h is complete, so the two GEMMs
 * overlap. ([P2] "Modifications", [P4] "Summary", [P5] per-expert dispatch.)
 *   Inputs as moe_gemm1_swiglu (limits included) plus w2 / w2_scale as moe_gemm2_combine.
 *   h [A][I] (+ h_scale [I/128][A] for FP8) and y [A][H] bf16 are outputs.
 *   ws: moe_workspace_size(MOE_WS_EXPERTS); besides the header it holds per-block
 *   completion flags that must be zero when a call starts: zero the whole workspace once
 *   after allocating it; every call leaves the flags at zero.
 * Errors: INVALID_ARG, WORKSPACE, ARCH, CUDA; TIMEOUT / EXPERT_ID in the status word. */
int moe_experts(const void* x_perm, const float* x_scale, const int32_t* offsets, const void* w1,
                const void* w1_scale, const float* gate_scale, const float* up_scale,
                const float* limits, const void* w2, const void* w2_scale, const moe_dims* dims,
                void* h, float* h_scale, void* y, void* ws, size_t ws_bytes, void* stream);

/* The routing-weighted combine alone ([P5] slot-specific weighted reduction):
 *   out[t] = sum_{j<k} topk_w[t][j] * y[inv_perm[t][j]]
 *          + sum_{s<n_shared} gamma[t][s] * y[offsets[E+s] + t]
 * in fp32 in that order, one rounding to bf16; gamma as in moe_gemm2_combine.
 *   y [A][H] bf16 (as written by moe_experts), offsets, inv_perm [T][k], topk_w [T][k],
 *   shared_w [T][n_sink] (NULL iff n_sink == 0); out [T][H] bf16.
 *   ws: moe_workspace_size(MOE_WS_COMBINE) (the status header).
 * Errors: INVALID_ARG, WORKSPACE, ARCH, CUDA; EXPERT_ID in the status word. */
int moe_combine(const void* y, const int32_t* offsets, const int32_t* inv_perm,
                const float* topk_w, const float* shared_w, const moe_dims* dims, void* out,
                void* ws, size_t ws_bytes, void* stream);

/* The whole layer: moe_route_topk, moe_permute, moe_experts and moe_combine in sequence
 * on `stream`, with every intermediate in the workspace
 * (moe_workspace_size(MOE_WS_FORWARD)).
 *   logits [T][E+n_sink] fp32, bias [E] or NULL, x [T][H] bf16, weights, scales and
 *   limits as above.
 *   out [T][H] bf16 out.
 *   topk_ids / topk_w / shared_w / packed: optional outputs ([T][k], [T][k], [T][n_sink],
 *   [T][k]); pass NULL to keep the first three in the workspace and skip `packed`.
 * Errors: as the four calls. */
int moe_forward(const float* logits, const float* bias, const void* x, const void* w1,
                const void* w1_scale, const float* gate_scale, const float* up_scale,
                const float* limits, const void* w2, const void* w2_scale, const moe_dims* dims,
                void* out, int32_t* topk_ids, float* topk_w, float* shared_w, uint32_t* packed,
                void* ws, size_t ws_bytes, void* stream);

/* ---- Expert parallelism [P1']: experts partitioned over ranks ----------------------
 * Rank r of R holds routed experts [r*E/R, (r+1)*E/R) and every shared expert. A rank
 * permutes its own tokens as usual (the routed rows are then already in order of the
 * rank that owns their expert), sends each routed row with its global group id to that
 * rank, rebases the ids it receives (moe_ep_rebase), runs moe_permute / moe_experts /
 * moe_combine (k = 1, unit weights) over its local groups, sends the rows back and
 * combines them as in the one-rank layer. The exchange itself is the caller's (NCCL). */

/* moe_ep_row_ids -- the weight group of every permuted row.
 *   offsets [G+1] as written by moe_permute (G = E + n_shared; entries are clamped into
 *   [0, A] before use), A = T*(k + n_shared) from dims.
 *   row_ids [A] int32 out: row_ids[r] = g with offsets[g] <= r < offsets[g+1], i.e. the
 *   global routed expert id (< E) or E + s for shared expert s.
 * Errors: INVALID_ARG (dims, NULL pointers), ARCH, CUDA. */
int moe_ep_row_ids(const int32_t* offsets, const moe_dims* dims, int32_t* row_ids, void* stream);

/* moe_ep_rebase -- global group ids to this rank's local group ids.
 *   ids [n] int32: global ids as written by moe_ep_row_ids on any rank.
 *   E, n_shared: the global routed expert count and shared expert count;
 *   local_offset, n_local: this rank's routed experts are [local_offset,
 *   local_offset + n_local) (0 <= local_offset, local_offset + n_local <= E).
 *   out [n] int32: id - local_offset for a local routed expert, n_local + s for shared
 *   expert s (replicated on every rank), -1 for anything else: an id of another rank or
 *   out of range. moe_permute over these local ids (E = n_local + n_shared, k = 1)
 *   records MOE_ERR_EXPERT_ID for a -1 and drops that row. out may alias ids.
 * Errors: INVALID_ARG (sizes, NULL pointers), ARCH, CUDA. */
int moe_ep_rebase(const int32_t* ids, int64_t n, int32_t E, int32_t n_shared, int32_t local_offset,
                  int32_t n_local, int32_t* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
