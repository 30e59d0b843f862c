// gemm.cu -- grouped GEMMs of the expert layer on the 5th-generation tensor cores.
//
// Orientation: the expert's weight rows are the MMA's M side (128 rows per tile, TMEM
// lanes) and the permuted token rows of the group are the N side (up to BN per tile,
// TMEM columns), so a group with n rows costs ceil(n/16)*16 MMA columns, not a 128-row
// tile, and decode-sized groups stream weights with N = 16.
//
// GEMM1 (gated): each tile covers 128 gate rows and the matching 128 up rows of W1[g]
// (two MMAs per K step into two TMEM column ranges), so one thread holds gate and up
// of the same intermediate index and the clamped, parameterised SwiGLU (sglang PR
// #39920 "Modifications"; DeepGEMM PR #445 "Summary") runs in the epilogue, with the
// per-group gate/up scales applied to the accumulators first (xorl-wheels FlashInfer
// 0.6.18 release notes, "Changes"). The intermediate never leaves the SM unactivated.
// GEMM2: one MMA per K step; the epilogue stores y in bf16.
//
// FP8 (E4M3, 128x128 weight blocks, 1x128 activation blocks; GLM FP8 blockwise, sglang
// PR #39920 "Motivation"): every 128-deep K block is one pipeline stage; its product
// goes to one of two TMEM partial buffers and the epilogue warps promote it into fp32
// registers with the product of the two block scales, while the tensor core fills the
// other buffer. GEMM1's epilogue then quantises h per 1x128 block (fused act-quant).
//
// Roles (320 threads): warp 0 lane 0 issues TMA loads into a STAGES-deep ring; warp 1
// owns TMEM and lane 0 issues tcgen05.mma; warps 2..9 are the epilogue (warp w reads
// TMEM lanes 32*(w%4).., and columns of half (w-2)/4 of the tile). Tiles are scheduled
// persistently: tile L = (token block, chunk), CTA b takes L = b, b + grid, ...
// Every wait is bounded (ptx.cuh): on timeout the CTA sets MOE_ERR_TIMEOUT, drains its
// outstanding copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block

constexpr int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

template <int BN_, bool GATED_, bool FP8_>
struct Cfg {
    static constexpr int BN = BN_;
    static constexpr bool GATED = GATED_;
    static constexpr bool FP8 = FP8_;
    static constexpr int BK = FP8 ? 128 : 64;  // K elements per stage: one 128-byte row
    static constexpr int NUM_A = GATED ? 2 : 1;
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    static constexpr int STAGES_RAW = (196 * 1024) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int ACC_COLS = NUM_A * BN;  // one TMEM buffer
    static constexpr int TMEM_COLS = pow2_at_least(2 * ACC_COLS);
    static constexpr int HALF = BN / 2;           // columns per epilogue warp
    static constexpr int CW = HALF < 16 ? HALF : 16;
    static constexpr int RED_FLOATS = (FP8 && GATED) ? 2 * 4 * HALF : 4;
    static_assert(STAGE_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned");
    static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
    static_assert(HALF % CW == 0, "column share must be a multiple of the load width");

    static constexpr size_t ctrl_bytes() { return 8 * (2 * STAGES + 6) + 16 + 4 * RED_FLOATS; }
    static size_t smem_bytes(int G) {
        return 1024 + (size_t)STAGES * STAGE_BYTES + ctrl_bytes() + 4 * (size_t)(G + 1) + 16;
    }
};

struct DevArgs {
    const int32_t* offsets;
    int G;
    int num_kb;       // K / BK
    int wrows;        // weight rows per group
    int n_chunks;     // 128-row chunks per group
    int up_off;       // gate->up row offset (GEMM1)
    int kblocks;      // K / 128 (FP8 scale columns)
    int64_t A;
    const float* act_scale;
    const float* w_scale;
    void* out;
    float* out_scale;
    int out_ld;
    const float* gate_scale;
    const float* up_scale;
    float alpha, beta, limit;
    int* status;
};

struct Tile {
    int g, c, row0, nrows;
};

template <int BN>
__device__ __forceinline__ Tile decode_tile(int L, const int32_t* blk_start, const DevArgs& p) {
    const int blk = L / p.n_chunks;
    Tile t;
    t.c = L - blk * p.n_chunks;
    int lo = 0, hi = p.G - 1;  // largest g with blk_start[g] <= blk
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (blk_start[mid] <= blk) lo = mid;
        else hi = mid - 1;
    }
    t.g = lo;
    const int end = __ldg(p.offsets + lo + 1);
    t.row0 = __ldg(p.offsets + lo) + (blk - blk_start[lo]) * BN;
    t.nrows = min(BN, end - t.row0);
    return t;
}

__device__ __forceinline__ float swiglu_dev(float gate, float up, float alpha, float beta, float limit) {
    const float g = fminf(gate, limit);
    const float u = fminf(fmaxf(up, -limit), limit);
    const float sig = 1.f / (1.f + __expf(-alpha * g));
    return g * sig * (u + beta);
}

// Warp-collective bounded wait: lane 0 waits, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, PipeAbort* ab, int* status) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, ab, status);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const DevArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* epibar = drain + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 1);
    PipeAbort* ab = reinterpret_cast<PipeAbort*>(tmem_slot + 1);
    float* red = reinterpret_cast<float*>(tmem_slot + 4);
    int32_t* blk_start = reinterpret_cast<int32_t*>(red + C::RED_FLOATS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(epibar, kEpiWarps);
        ab->flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    // Token blocks per group and their running start: blk_start[g] = sum_{g'<g} ceil(n_g'/BN).
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int n = __ldg(p.offsets + g + 1) - __ldg(p.offsets + g);
        blk_start[g + 1] = n > 0 ? (n + C::BN - 1) / C::BN : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int b0 = 1; b0 <= G; b0 += 32) {
            const int g = b0 + lane;
            const int v = g <= G ? blk_start[g] : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += n;
            }
            if (g <= G) blk_start[g] = carry + incl;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) blk_start[0] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = blk_start[G] * p.n_chunks;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            uint32_t stage = 0, phase = 0, pend_mask = 0, pend_phase = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                const Tile tl = decode_tile<C::BN>(L, blk_start, p);
                const int arow = tl.g * p.wrows + tl.c * 128;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + (size_t)stage * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
                    tma_load_2d(st, &tmA, &full[stage], kb * C::BK, arow);
                    if constexpr (C::GATED)
                        tma_load_2d(st + C::A_BYTES, &tmA, &full[stage], kb * C::BK, arow + p.up_off);
                    tma_load_2d(st + C::NUM_A * C::A_BYTES, &tmB, &full[stage], kb * C::BK, tl.row0);
                    pend_mask |= 1u << stage;
                    pend_phase = (pend_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == (uint32_t)C::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Never leave with a copy in flight: wait for the last fill of every stage.
            for (int s = 0; s < C::STAGES; ++s)
                if ((pend_mask >> s) & 1u) mbar_wait_drain(&full[s], (pend_phase >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, it = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                const Tile tl = decode_tile<C::BN>(L, blk_start, p);
                const int n_mma = max(16, (tl.nrows + 15) & ~15);
                const uint32_t idesc = idesc_m128(n_mma, C::FP8);
                if constexpr (!C::FP8) {
                    const uint32_t buf = it & 1, bph = (it >> 1) & 1;
                    if (!mbar_wait(&tempty[buf], bph ^ 1, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d0 = tmem_base + buf * C::ACC_COLS;
                    for (int kb = 0; kb < p.num_kb; ++kb) {
                        if (!mbar_wait(&full[stage], phase, ab, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(smem + (size_t)stage * C::STAGE_BYTES);
                        const uint32_t b0 = a0 + C::NUM_A * C::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bd = smem_desc_sw128(b0 + kk * 32);
                            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                            mma_bf16(d0, smem_desc_sw128(a0 + kk * 32), bd, idesc, acc);
                            if constexpr (C::GATED)
                                mma_bf16(d0 + C::BN, smem_desc_sw128(a0 + C::A_BYTES + kk * 32), bd, idesc, acc);
                        }
                        tc_commit(&empty[stage]);
                        if (++stage == (uint32_t)C::STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (!ok) break;
                    tc_commit(&tfull[buf]);
                    ++it;
                } else {
                    for (int kb = 0; kb < p.num_kb; ++kb) {
                        const uint32_t buf = it & 1, bph = (it >> 1) & 1;
                        if (!mbar_wait(&tempty[buf], bph ^ 1, ab, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        if (!mbar_wait(&full[stage], phase, ab, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d0 = tmem_base + buf * C::ACC_COLS;
                        const uint32_t a0 = smem_u32(smem + (size_t)stage * C::STAGE_BYTES);
                        const uint32_t b0 = a0 + C::NUM_A * C::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bd = smem_desc_sw128(b0 + kk * 32);
                            const uint32_t acc = kk > 0 ? 1u : 0u;
                            mma_fp8(d0, smem_desc_sw128(a0 + kk * 32), bd, idesc, acc);
                            if constexpr (C::GATED)
                                mma_fp8(d0 + C::BN, smem_desc_sw128(a0 + C::A_BYTES + kk * 32), bd, idesc, acc);
                        }
                        tc_commit(&empty[stage]);
                        tc_commit(&tfull[buf]);
                        ++it;
                        if (++stage == (uint32_t)C::STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
            }
            // All MMAs issued by this thread complete before TMEM is released.
            tc_commit(drain);
            mbar_wait_drain(drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int q = warp & 3;        // TMEM lane quarter this warp may access
        const int hc = ew >> 2;        // which half of the tile's columns
        const int c0 = hc * C::HALF;
        const int row_local = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        uint32_t it = 0, ephase = 0;
        bool ok = true;
        for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
            const Tile tl = decode_tile<C::BN>(L, blk_start, p);
            const int n_mma = max(16, (tl.nrows + 15) & ~15);
            const int col = tl.c * 128 + row_local;  // output column (intermediate or hidden index)
            if constexpr (!C::FP8) {
                const uint32_t buf = it & 1, bph = (it >> 1) & 1;
                if (!warp_wait(&tfull[buf], bph, ab, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tb = tmem_base + lane_off + buf * C::ACC_COLS;
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
                if constexpr (C::GATED) {
                    const float sg = p.gate_scale ? __ldg(p.gate_scale + tl.g) : 1.f;
                    const float su = p.up_scale ? __ldg(p.up_scale + tl.g) : 1.f;
#pragma unroll 1
                    for (int cc = c0; cc < c0 + C::HALF && cc < n_mma; cc += C::CW) {
                        float gv[C::CW], uv[C::CW];
                        if constexpr (C::CW == 16) tmem_ld16x2(tb + cc, tb + C::BN + cc, gv, uv);
                        else tmem_ld8x2(tb + cc, tb + C::BN + cc, gv, uv);
#pragma unroll
                        for (int j = 0; j < C::CW; ++j) {
                            const int n = cc + j;
                            if (n < tl.nrows) {
                                const float h = swiglu_dev(sg * gv[j], su * uv[j], p.alpha, p.beta, p.limit);
                                out[(size_t)(tl.row0 + n) * p.out_ld + col] = __float2bfloat16_rn(h);
                            }
                        }
                    }
                } else {
#pragma unroll 1
                    for (int cc = c0; cc < c0 + C::HALF && cc < n_mma; cc += C::CW) {
                        float v[C::CW];
                        if constexpr (C::CW == 16) tmem_ld16(tb + cc, v);
                        else tmem_ld8(tb + cc, v);
#pragma unroll
                        for (int j = 0; j < C::CW; ++j) {
                            const int n = cc + j;
                            if (n < tl.nrows) out[(size_t)(tl.row0 + n) * p.out_ld + col] = __float2bfloat16_rn(v[j]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
                ++it;
            } else {
                float acc_g[C::HALF];
                float acc_u[C::GATED ? C::HALF : 1];
#pragma unroll
                for (int j = 0; j < C::HALF; ++j) acc_g[j] = 0.f;
#pragma unroll
                for (int j = 0; j < (C::GATED ? C::HALF : 1); ++j) acc_u[j] = 0.f;
                const float* wsg = p.w_scale + ((size_t)tl.g * (p.wrows / 128) + tl.c) * p.kblocks;
                const float* wsu = p.w_scale + ((size_t)tl.g * (p.wrows / 128) + p.up_off / 128 + tl.c) * p.kblocks;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    const uint32_t buf = it & 1, bph = (it >> 1) & 1;
                    // Per-column activation scales of this K block (one lane per column).
                    float sb0 = 0.f, sb1 = 0.f;
                    {
                        const int n = c0 + lane;
                        if (n < tl.nrows) sb0 = __ldg(p.act_scale + (size_t)kb * p.A + tl.row0 + n);
                        if constexpr (C::HALF > 32) {
                            const int n2 = c0 + 32 + lane;
                            if (n2 < tl.nrows) sb1 = __ldg(p.act_scale + (size_t)kb * p.A + tl.row0 + n2);
                        }
                    }
                    const float sa_g = __ldg(wsg + kb);
                    const float sa_u = C::GATED ? __ldg(wsu + kb) : 0.f;
                    if (!warp_wait(&tfull[buf], bph, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tb = tmem_base + lane_off + buf * C::ACC_COLS;
#pragma unroll
                    for (int ch = 0; ch < C::HALF / C::CW; ++ch) {
                        const int cc = c0 + ch * C::CW;
                        if (cc < n_mma) {
                            float pg[C::CW], pu[C::CW];
                            if constexpr (C::GATED) {
                                if constexpr (C::CW == 16) tmem_ld16x2(tb + cc, tb + C::BN + cc, pg, pu);
                                else tmem_ld8x2(tb + cc, tb + C::BN + cc, pg, pu);
                            } else {
                                if constexpr (C::CW == 16) tmem_ld16(tb + cc, pg);
                                else tmem_ld8(tb + cc, pg);
                            }
#pragma unroll
                            for (int j = 0; j < C::CW; ++j) {
                                const int jj = ch * C::CW + j;
                                const float sb = __shfl_sync(0xffffffffu, jj < 32 ? sb0 : sb1, jj & 31);
                                acc_g[jj] = fmaf(pg[j], sa_g * sb, acc_g[jj]);
                                if constexpr (C::GATED) acc_u[jj] = fmaf(pu[j], sa_u * sb, acc_u[jj]);
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[buf]);
                    ++it;
                }
                if (!ok) break;
                if constexpr (C::GATED) {
                    // SwiGLU, then 1x128 E4M3 quantisation of h: the block of row r is
                    // the 128 intermediate indices of this chunk = the 4 lane quarters.
                    const float sg = p.gate_scale ? __ldg(p.gate_scale + tl.g) : 1.f;
                    const float su = p.up_scale ? __ldg(p.up_scale + tl.g) : 1.f;
#pragma unroll
                    for (int j = 0; j < C::HALF; ++j) {
                        acc_g[j] = swiglu_dev(sg * acc_g[j], su * acc_u[j], p.alpha, p.beta, p.limit);
                        float m = fabsf(acc_g[j]);
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                        if (lane == 0) red[(hc * 4 + q) * C::HALF + j] = m;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(epibar);
                    if (!warp_wait(epibar, ephase, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    ephase ^= 1;
                    uint8_t* out = static_cast<uint8_t*>(p.out);
#pragma unroll
                    for (int j = 0; j < C::HALF; ++j) {
                        const int n = c0 + j;
                        float amax = red[(hc * 4 + 0) * C::HALF + j];
                        amax = fmaxf(amax, red[(hc * 4 + 1) * C::HALF + j]);
                        amax = fmaxf(amax, red[(hc * 4 + 2) * C::HALF + j]);
                        amax = fmaxf(amax, red[(hc * 4 + 3) * C::HALF + j]);
                        const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
                        if (n < tl.nrows) {
                            out[(size_t)(tl.row0 + n) * p.out_ld + col] = (uint8_t)__nv_cvt_float_to_fp8(
                                __fdiv_rn(acc_g[j], s), __NV_SATFINITE, __NV_E4M3);
                            if (q == 0 && lane == 0) p.out_scale[(size_t)tl.c * p.A + tl.row0 + n] = s;
                        }
                    }
                    // red is rewritten by the next tile: everyone must have read it.
                    __syncwarp();
                    if (lane == 0) mbar_arrive(epibar);
                    if (!warp_wait(epibar, ephase, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    ephase ^= 1;
                } else {
                    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
                    for (int j = 0; j < C::HALF; ++j) {
                        const int n = c0 + j;
                        if (n < tl.nrows) out[(size_t)(tl.row0 + n) * p.out_ld + col] = __float2bfloat16_rn(acc_g[j]);
                    }
                }
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2D K-major tensor map: rows x K elements, box = box_rows x 128 bytes, 128B swizzle.
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K, bool fp8, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const uint32_t elt = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {K, rows};
    cuuint64_t strides[1] = {K * elt};
    cuuint32_t box[2] = {128 / elt, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 64 && cache[dev]) return cache[dev];
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev < 64) cache[dev] = n;
    return n;
}

template <class C>
static cudaError_t launch_cfg(const GemmArgs& a, cudaStream_t stream) {
    CUtensorMap tmA, tmB;
    if (!make_map(&tmA, a.w, (uint64_t)a.G * a.wrows, a.K, C::FP8, 128)) return cudaErrorInvalidValue;
    if (!make_map(&tmB, a.act, (uint64_t)a.A, a.K, C::FP8, C::BN)) return cudaErrorInvalidValue;
    DevArgs p;
    p.offsets = a.offsets;
    p.G = a.G;
    p.num_kb = a.K / C::BK;
    p.wrows = a.wrows;
    p.n_chunks = a.n_chunks;
    p.up_off = a.up_off;
    p.kblocks = a.K / 128;
    p.A = a.A;
    p.act_scale = a.act_scale;
    p.w_scale = a.w_scale;
    p.out = a.out;
    p.out_scale = a.out_scale;
    p.out_ld = a.out_ld;
    p.gate_scale = a.gate_scale;
    p.up_scale = a.up_scale;
    p.alpha = a.alpha;
    p.beta = a.beta;
    p.limit = a.limit;
    p.status = a.status;
    const size_t smem = C::smem_bytes(a.G);
    if (smem > (size_t)kSmemLimit) return cudaErrorInvalidValue;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(grouped_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kSmemLimit);
    });
    if (attr_err != cudaSuccess) return attr_err;
    grouped_gemm_kernel<C><<<num_sms(), kThreads, smem, stream>>>(tmA, tmB, p);
    return cudaGetLastError();
}

int gemm_pick_bn(int64_t A, int G, bool gated, bool fp8) {
    const double avg = G > 0 ? (double)A / (double)G : 0.0;
    int bn = 16;
    while (bn < 128 && bn < 1.5 * avg) bn <<= 1;
    if (gated && fp8 && bn > 64) bn = 64;
    return bn;
}

template <int BN>
static cudaError_t launch_bn(const GemmArgs& a, bool gated, bool fp8, cudaStream_t s) {
    if (gated) {
        if (fp8) {
            if constexpr (BN <= 64) return launch_cfg<Cfg<BN, true, true>>(a, s);
            else return cudaErrorInvalidValue;
        }
        return launch_cfg<Cfg<BN, true, false>>(a, s);
    }
    if (fp8) return launch_cfg<Cfg<BN, false, true>>(a, s);
    return launch_cfg<Cfg<BN, false, false>>(a, s);
}

cudaError_t launch_gemm(const GemmArgs& a, bool gated, bool fp8, int bn, cudaStream_t stream) {
    if (a.A == 0 || a.G == 0) return cudaSuccess;
    switch (bn) {
        case 16: return launch_bn<16>(a, gated, fp8, stream);
        case 32: return launch_bn<32>(a, gated, fp8, stream);
        case 64: return launch_bn<64>(a, gated, fp8, stream);
        case 128: return launch_bn<128>(a, gated, fp8, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
