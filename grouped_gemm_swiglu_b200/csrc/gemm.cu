// gemm.cu -- grouped GEMMs of the expert layer on the 5th-generation tensor cores, as
// one persistent kernel that can run GEMM1 (+ SwiGLU), GEMM2, or both in one launch.
//
// Orientation: the expert's weight rows are the MMA's M side (128 rows per tile, TMEM
// lanes) and the permuted token rows of the group are the N side (up to BN per tile,
// TMEM columns), so a group with n rows costs ceil(n/16)*16 MMA columns, not a 128-row
// tile, and decode-sized groups stream weights with N = 16.
//
// Phase 1, GEMM1 (gated): a tile covers 128 gate rows and the matching 128 up rows of
// W1[g] (two MMAs per K step into two TMEM column ranges), so one thread holds gate and
// up of the same intermediate index and the clamped, parameterised SwiGLU (sglang PR
// #39920 "Modifications"; DeepGEMM PR #445 "Summary") runs in the epilogue, with the
// per-group gate/up scales applied to the accumulators first (xorl-wheels FlashInfer
// 0.6.18 release notes, "Changes"). The intermediate never leaves the SM unactivated.
// Phase 2, GEMM2: a tile covers two 128-row chunks of H (the last one alone when H/128
// is odd), two MMAs per K step; the epilogue stores y in bf16.
//
// FP8 (E4M3, 128x128 weight blocks, 1x128 activation blocks; GLM FP8 blockwise, sglang
// PR #39920 "Motivation"): every 128-deep K block is one pipeline stage; its product
// goes to one of two TMEM partial buffers and the epilogue warps promote it into fp32
// registers with the product of the two block scales, while the tensor core fills the
// other buffer. GEMM1's epilogue then quantises h per 1x128 block (fused act-quant).
//
// 4-bit weights (INT4 group-32, NVFP4): TMA brings the packed bytes and the token rows;
// dequantisation warps convert each 64-deep stage of the weight rows to bf16 and store
// it into tensor memory, which the MMA reads as its A operand.
//
// Scheduling: tiles are numbered GEMM1 first -- (token block, 128-row chunk of I, K
// split) -- then GEMM2 -- (token block, pair of 128-row chunks of H). The producer warp claims the next
// tile from a global counter and hands its number to the MMA and epilogue warps through
// a two-slot ring in shared memory. When both phases run, a GEMM2 tile of token block b
// first loads its weights, then waits until all GEMM1 tiles of b have published their h
// rows (a per-block release counter); a tile only ever waits for tiles claimed before
// it, which never wait themselves, so the schedule cannot deadlock.
//
// Roles: warp 0 lane 0 issues TMA loads into a STAGES-deep ring; warp 1 owns TMEM and
// lane 0 issues tcgen05.mma; the next EPI warps are the epilogue (warp w reads TMEM lanes
// 32*(w%4).., and its group's share of the tile's columns): 8 warps (320 threads), 16 at
// 256 token columns, 4 for 4-bit decode tiles, which add their DQ dequantisation warps
// after the epilogue. FP8 tiles of 128 tokens are token-major (tokens = M = TMEM lanes)
// and launch 384 threads: warp 2 releases GEMM1 tiles' h to GEMM2, warp 3 only lends its
// registers, and warps 4..11 are the epilogue. Every wait is bounded
// (ptx.cuh): on timeout the CTA sets MOE_ERR_TIMEOUT, drains its outstanding copies and
// MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

constexpr int kSmemLimit = 232448;  // 227 KB opt-in per block
constexpr int kRing = 2;            // tile-number ring depth
constexpr int kMaxGroupsGemm = 1024 + 32;

constexpr int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

template <int BN_, bool FP8_, bool INT4_ = false, bool PAIR_ = false>
struct Cfg {
    static constexpr int BN = BN_;
    static constexpr bool FP8 = FP8_;
    // Two CTAs of a cluster share each MMA (cta_group::2, M = 256 token rows): each CTA
    // loads its own 128 token rows and half of the 256 weight rows (the gate rows in the
    // even CTA, the up rows in the odd one; GEMM2: one 128-row chunk of H each), so a CTA
    // pulls 32 KB through L2 per 128-byte K step instead of 48 KB. A token block is then
    // TB = 256 rows of a group. FP8 or bf16 (for bf16 the tile's partial sums stay in
    // TMEM over the whole K range, so each tile drains one of two TMEM buffers while the
    // tensor core fills the other).
    static constexpr bool PAIR = PAIR_;
    static constexpr int TB = PAIR ? 2 * BN : BN;  // token rows per block
    // INT4 group-32 weights: TMA brings the packed bytes (RAW_BYTES per 128x64 block) and
    // dequantisation warps write the bf16 weight tiles into tensor memory, where the MMA
    // takes its A operand; shared memory then holds only the token tile and packed bytes.
    static constexpr bool INT4 = INT4_;
    static constexpr int BK = FP8 ? 128 : 64;  // K elements per stage: one 128-byte row
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int RAW_BYTES = INT4 ? 128 * 32 : 0;
    static constexpr int B_OFF = INT4 ? 0 : (PAIR ? A_BYTES : 2 * A_BYTES);  // token tile within a stage
    static constexpr int RAW_OFF = B_OFF + B_BYTES;        // INT4: packed A0, A1 after the token tile
    static constexpr int STAGE_BYTES =
        INT4 ? B_BYTES + 2 * RAW_BYTES : (PAIR ? A_BYTES + B_BYTES : 2 * A_BYTES + B_BYTES);  // GEMM1-sized
    static constexpr int A_TMEM_COLS = 64;  // INT4: one stage's bf16 A0 | A1 (128 x 64 K, two K per column)
    // Dequantisation warps, in sets of four (a warp may only touch its TMEM lane quarter,
    // warp % 4, so a set covers the 128 rows of a tile). For decode-sized tiles (the
    // epilogue then has 4 warps) 8 warps in two stage groups of one set each: a group
    // converts every other stage, so one stage's fixed latency (barrier wait, shared-memory
    // load, tensor-memory store and its wait, fence, arrive) overlaps the other's work.
    // Otherwise one group of 4. A thread converts its row of both tiles of a stage.
    // (Measured at decode sizes: one group of 8 and of 16 warps splitting each stage's
    // tiles or K range, two groups of 8, four of 4 were all slower.)
    static constexpr int DQ = INT4 ? (BN <= 32 ? 8 : 4) : 0;
    static constexpr int NGRP = (INT4 && BN <= 32) ? 2 : 1;  // stage groups (alternate stages)
    static constexpr int DQG = DQ / NGRP;                    // warps per stage: one set of 4
    // Token rows arrive in boxes of up to 64 rows, and only the boxes a tile's rows reach
    // are loaded, so a short token block does not pull a full BN-row tile through L2.
    static constexpr int BOX_ROWS = BN < 64 ? BN : 64;
    static constexpr int BOX_BYTES = BOX_ROWS * 128;
    // as many stages as fit next to the control block and the largest group table
    // wide FP8 tile (FP8 at 128 tokens): 2 KB per epilogue warp to turn its token rows into
    // row-contiguous stores (16 rows x 128 bytes at a time)
    static constexpr int XPOSE_BYTES = ((FP8_ && BN_ >= 128) || PAIR_) ? 8 * 2048 : 0;
    static constexpr int STAGE_BUDGET =
        kSmemLimit - 1024 - 8 * (kMaxGroupsGemm + 1) - 1024 - 4 * 16 * 16 * 3 - XPOSE_BYTES;
    static constexpr int ACC_COLS = 2 * BN;  // one TMEM buffer: gate | up (GEMM2 uses the first BN)
    // bf16 hands one buffer per tile to the epilogue, FP8 one per 128-deep K block, so
    // FP8 keeps up to four partial buffers in flight.
    // At 256 token columns gate | up fill all 512 TMEM columns: one buffer, and the TMA
    // ring keeps streaming the next tile while the epilogue drains it.
    static constexpr int NBUF = (FP8 && 4 * ACC_COLS <= 512) ? 4 : (2 * ACC_COLS <= 512 ? 2 : 1);
    static constexpr int STAGES_SMEM = STAGE_BUDGET / STAGE_BYTES;
    static constexpr int STAGES_TMEM = INT4 ? (512 - NBUF * ACC_COLS) / A_TMEM_COLS : 8;  // INT4: A tiles in TMEM
    static constexpr int STAGES_RAW = STAGES_SMEM < STAGES_TMEM ? STAGES_SMEM : STAGES_TMEM;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int A_TMEM = NBUF * ACC_COLS;  // INT4: first TMEM column of the A tiles
    static constexpr int TMEM_COLS = pow2_at_least(NBUF * ACC_COLS + (INT4 ? STAGES * A_TMEM_COLS : 0));
    // Epilogue warps: groups of four (one warp per TMEM lane quarter), each group owning
    // an equal share of the tile's columns; four groups at 256 columns, whose single
    // accumulator buffer makes the drain time part of the tile time.
    // FP8 at 128 token columns: the promoted gate and up sums of a 128 x 128 tile fill half
    // the register file. Two more warps make warps 0-3 (producer, MMA, the publisher of
    // GEMM1 tiles, an idle warp) one warpgroup, which gives registers back (setmaxnreg) to
    // the epilogue warpgroups: the launch's threads x registers cover 4 warps at REG_LOW
    // and WEPI epilogue warps at REG_HIGH.
    static constexpr bool WIDE = (FP8 && BN >= 128) || PAIR;  // token-major (FP8 at 128 tokens, or a pair)
    static constexpr int WEPI = 8;  // wide FP8 epilogue warps: 8 (128 sums each) or 16 (64)
    static constexpr int EPI = WIDE ? WEPI : (BN >= 256 ? 16 : ((INT4 && BN <= 32) ? 4 : 8));
    static constexpr int EPI0 = WIDE ? 4 : 2;  // first epilogue warp
    static constexpr int REG_LAUNCH = WIDE ? (65536 / (32 * (4 + WEPI))) / 8 * 8 : 0;
    // (the bf16 pair's epilogue holds no promotion sums: its producer and MMA loops get more)
    static constexpr int REG_LOW = (PAIR && !FP8) ? 88 : 56;
    static constexpr int REG_HIGH = WEPI == 8 ? ((PAIR && !FP8) ? 208 : 224) : 104;
    static constexpr int WCH = 16;  // wide FP8: TMEM columns per load of each half
    static constexpr int THREADS = 32 * EPI0 + 32 * EPI + 32 * DQ;
    static constexpr int GROUPS = EPI / 4;
    static constexpr int COLS = BN / GROUPS;  // columns per epilogue warp
    static constexpr int CW = COLS < 16 ? COLS : 16;  // TMEM load width (columns)
    static constexpr int RED_FLOATS = WIDE ? 2 * GROUPS * 128 : (FP8 ? EPI * COLS : 4);
    // FP8: per epilogue warp, the two rows of scale products (A0, A1) of its columns
    static constexpr int SCT_FLOATS = (FP8 && !WIDE) ? EPI * 2 * COLS : 4;
    static_assert(STAGE_BYTES % 1024 == 0, "stage tiles must stay 1024-byte aligned");
    static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
    static_assert(COLS % CW == 0 && CW >= 4, "column share must be a multiple of the load width");
    static_assert(!FP8 || WIDE || COLS <= 32, "FP8 loads a warp's whole column share at once");
    static_assert(!WIDE || XPOSE_BYTES == EPI * 2048, "one 2 KB row-staging buffer per epilogue warp");
    static_assert(!WIDE || (BN == 128 && (EPI == 8 || EPI == 16) && COLS % 16 == 0 &&
                            128 * REG_LOW + 32 * EPI * REG_HIGH <= THREADS * REG_LAUNCH &&
                            REG_LOW + (EPI / 4) * REG_HIGH <= 512),
                  "register split of the wide FP8 tile (whole CTA and per SM sub-partition)");
    static_assert(BN % BOX_ROWS == 0 && BN <= 256, "token tile = whole boxes, at most the MMA's N limit");
    static_assert(STAGES >= 2, "at least two pipeline stages");
    static_assert(!(INT4 && FP8), "INT4 weights take bf16 activations");
    static_assert(!PAIR || (WIDE && BN == 128 && !INT4), "the CTA pair is a token-major tile of 2 x 128 rows");
    static_assert(!INT4 || BN <= 64, "INT4 keeps its A tiles next to the accumulators in TMEM");
    static_assert(!INT4 || (DQG == 4 && DQG * NGRP == DQ), "dequantisation warps: stage groups of 4");
    static_assert(COLS % 8 == 0, "split-K merges columns in chunks of 8");
    // Split-K of GEMM1 is compiled in where it can be chosen (see gemm_split_factor):
    // every tile width except FP8 from 64 columns, whose promotion registers are full,
    // and 256 columns, whose merge path alone would push the kernel past its register
    // cap (a 256-column tile means large groups, which never need a split).
    static constexpr bool SPLIT_OK = !(FP8 && BN >= 64) && BN < 256 && !PAIR;

    // full/empty per stage, tfull/tempty per TMEM buffer, ring_full/ring_empty x kRing, drain,
    // epibar, and for INT4 raw_full per stage (packed bytes and token rows landed)
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + 2 * kRing + 2 + (INT4 ? STAGES : 0) + (WIDE ? 1 : 0);
    static constexpr size_t ctrl_bytes() {
        return 8 * NUM_BARS + 16 + 4 * kRing + 16 + 4 * RED_FLOATS + 16 + 4 * SCT_FLOATS + 16 + XPOSE_BYTES;
    }
    static size_t smem_bytes(int G) {  // + block table and clamped offsets, G+1 ints each
        return 1024 + (size_t)STAGES * STAGE_BYTES + ctrl_bytes() + 8 * (size_t)(G + 1) + 16;
    }
};

struct DevArgs {
    const int32_t* offsets;
    int G, A, H, I;
    int c1;      // GEMM1 tiles per token block: I/128 (0 = phase absent)
    int c2;      // GEMM2 tiles per token block: ceil(H/256), each two 128-row chunks of H (0 = absent)
    const float* x_scale;   // FP8: [H/128][A]
    const void* w1_scale;   // FP8: fp32 [G][2I/128][H/128]; INT4: bf16 [G][2I][H/32]; NVFP4: E4M3 [G][2I][H/16]
    const void* w2_scale;   // FP8: fp32 [G][H/128][I/128]; INT4: bf16 [G][H][I/32]; NVFP4: E4M3 [G][H][I/16]
    int fp4;                // 4-bit weights are NVFP4 (else INT4 group-32)
    const float* gate_scale;
    const float* up_scale;
    float alpha, beta, limit;
    const float* limits;    // [G] per-group clamp, or NULL for `limit`
    void* h;                // GEMM1 out / GEMM2 in: [A][I]
    float* h_scale;         // FP8: [I/128][A]
    void* y;                // GEMM2 out: [A][H] bf16
    unsigned int* tile_ctr;  // next tile to claim (zero when idle)
    unsigned int* exit_ctr;  // CTAs finished (zero when idle)
    int* done1;              // per token block: GEMM1 chunks published (zero at launch; both phases only)
    int s1;                  // GEMM1 split-K factor
    float* part;             // split-K partials [tile1][s1][2][BN][128]
    int* split_cnt;          // per GEMM1 tile: splits finished
    int* status;
};

// A tile is one or two 128-row weight blocks (A0, A1) against BN token rows: GEMM1 =
// gate rows and the matching up rows; GEMM2 = two consecutive 128-row chunks of H (the
// second absent when H/128 is odd and this is the last pair).
struct Tile {
    int phase;  // 1 = GEMM1 + SwiGLU, 2 = GEMM2
    int blk, g, c, row0, nrows;
    int ks;           // GEMM1 split index (0 .. s1-1)
    bool dual;        // A1 present
    int a0row, a1row; // first weight row of A0 / A1 in the [G*rows][K] weight matrix
    int col0, col1;   // first output column of A0 / A1 (intermediate or hidden index)
};

// blk_start: first token block of each group; s_off: group bounds clamped into [0, A].
// All GEMM1 units are claimed before any GEMM2 tile (interleaving the GEMM2 tiles of a
// block one or two waves after its GEMM1 units measured slower: they hold their SM while
// waiting for inputs still in flight).
template <int TB>
__device__ __forceinline__ Tile decode_tile(int L, int T1, const int32_t* blk_start, const int32_t* s_off,
                                            const DevArgs& p) {
    Tile t;
    if (L < T1) {
        t.phase = 1;
        const int tile1 = L / p.s1;  // the splits of one GEMM1 tile are consecutive
        t.ks = L - tile1 * p.s1;
        t.blk = tile1 / p.c1;
        t.c = tile1 - t.blk * p.c1;
    } else {
        t.ks = 0;
        t.phase = 2;
        const int L2 = L - T1;
        t.blk = L2 / p.c2;
        t.c = L2 - t.blk * p.c2;
    }
    int lo = 0, hi = p.G - 1;  // largest g with blk_start[g] <= blk
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (blk_start[mid] <= t.blk) lo = mid;
        else hi = mid - 1;
    }
    t.g = lo;
    const int g0 = s_off[lo];
    const int g1 = max(s_off[lo + 1], g0);
    t.row0 = g0 + (t.blk - blk_start[lo]) * TB;
    t.nrows = min(TB, g1 - t.row0);
    if (t.phase == 1) {
        t.dual = true;
        t.a0row = t.g * 2 * p.I + t.c * 128;
        t.a1row = t.a0row + p.I;
        t.col0 = t.col1 = t.c * 128;
    } else {
        t.dual = 2 * t.c + 1 < p.H / 128;
        t.a0row = t.g * p.H + 2 * t.c * 128;
        t.a1row = t.a0row + 128;
        t.col0 = 2 * t.c * 128;
        t.col1 = t.col0 + 128;
    }
    return t;
}

// The rows of a CTA-pair tile that CTA `rank` holds: 128 from row0 + 128 * rank (none
// when the block's group ends before them).
__device__ __forceinline__ void pair_rows(Tile& t, uint32_t rank) {
    const int skip = 128 * (int)rank;
    t.row0 += skip;
    t.nrows = max(0, min(128, t.nrows - skip));
}

// g * sigmoid(alpha*g) * (u + beta) written as g*(u+beta) / (1 + exp(-alpha*g)): one
// exponential and one fast reciprocal-multiply. A huge negative g sends the denominator
// to +inf and the quotient to the limit value 0.
__device__ __forceinline__ float swiglu_dev(float gate, float up, float alpha, float beta, float limit) {
    const float g = fminf(gate, limit);
    const float u = fminf(fmaxf(up, -limit), limit);
    return __fdividef(g * (u + beta), 1.f + __expf(-alpha * g));
}

// a0 += p0 * s0, a1 += p1 * s1 as one packed fp32x2 fused multiply-add.
__device__ __forceinline__ void ffma2(float& a0, float& a1, float p0, float p1, float s0, float s1) {
    asm("{\n\t.reg .b64 d, x, y, z;\n\t"
        "mov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %5};\n\tmov.b64 z, {%0, %1};\n\t"
        "fma.rn.f32x2 d, x, y, z;\n\tmov.b64 {%0, %1}, d;\n\t}\n"
        : "+f"(a0), "+f"(a1)
        : "f"(p0), "f"(p1), "f"(s0), "f"(s1));
}

// Split-K merge: the sums over splits 0..s1-1 of the gate and up partials of CH
// consecutive columns from `col`, this thread's row. part_tile is the tile's partials,
// laid out [split][gate, up][bn][128 rows]. Splits are read four at a time with every
// load of a group issued before its first add: one L2 round trip per four splits.
template <int CH>
__device__ __forceinline__ void sum_split_partials(const float* part_tile, int s1, int bn, int col, int row, float* g,
                                                   float* u) {
#pragma unroll
    for (int j = 0; j < CH; ++j) g[j] = u[j] = 0.f;
#pragma unroll 1
    for (int k0 = 0; k0 < s1; k0 += 4) {
        float pg[4][CH], pu[4][CH];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int j = 0; j < CH; ++j) {
                const float* q = part_tile + ((size_t)(2 * (k0 + kk)) * bn + col + j) * 128 + row;
                pg[kk][j] = k0 + kk < s1 ? __ldcg(q) : 0.f;
                pu[kk][j] = k0 + kk < s1 ? __ldcg(q + (size_t)bn * 128) : 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < CH; ++j) {
            g[j] += (pg[0][j] + pg[1][j]) + (pg[2][j] + pg[3][j]);
            u[j] += (pu[0][j] + pu[1][j]) + (pu[2][j] + pu[3][j]);
        }
    }
}

// Packed 4-bit weights: the 8 words (8 K each) of a row's 64-deep stage segment (16-byte aligned).
__device__ __forceinline__ void load_words(const uint8_t* raw, uint32_t* qw) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 q = *reinterpret_cast<const uint4*>(raw + 16 * i);
        qw[4 * i] = q.x;
        qw[4 * i + 1] = q.y;
        qw[4 * i + 2] = q.z;
        qw[4 * i + 3] = q.w;
    }
}

// INT4 group-32 dequantisation of a weight row segment into the bf16 pairs the MMA reads
// from tensor memory (batchgen PR #239 commit notes: low nibble = even K, value
// (nibble - 8) * scale with one bf16 scale per 32 K, taken in bf16).
// Each byte becomes one bf16x2 pair: the bf16 with bits 0x4300 | n is exactly 128 + n, so
// subtracting 136 gives n - 8 exactly, and one packed bf16 multiply (round to nearest
// even) gives the weight. lo / hi hold the low / high nibbles of the word's four bytes
// (one per byte); a byte permute puts byte j's pair in bytes 0 and 2 of one word.
__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t int4_pair_bf16(uint32_t lo, uint32_t hi, int byte, __nv_bfloat162 s) {
    // selector: result byte 0 = byte `byte` of lo, byte 2 = byte `byte` of hi (index 4 + byte)
    const uint32_t u = (byte_perm(lo, hi, (uint32_t)byte | ((uint32_t)(4 + byte) << 8)) & 0x00FF00FFu) | 0x43004300u;
    __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&u);
    v = __hmul2(__hsub2(v, __float2bfloat162_rn(136.f)), s);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// out[j] = the bf16 pair (K 2j, 2j+1) of a row's 64-deep segment, j < 32; `sc` holds its
// two group scales (bf16 bits, K 0-31 in the low half).
__device__ __forceinline__ void dequant_int4_row(const uint8_t* raw, uint32_t sc, uint32_t* out) {
    uint32_t qw[8];
    load_words(raw, qw);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const unsigned short sb = (unsigned short)((sc >> (16 * (w >> 2))) & 0xFFFFu);  // 4 words per group
        const __nv_bfloat162 s = __halves2bfloat162(__ushort_as_bfloat16(sb), __ushort_as_bfloat16(sb));
        const uint32_t lo = qw[w] & 0x0F0F0F0Fu, hi = (qw[w] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int b = 0; b < 4; ++b) out[4 * w + b] = int4_pair_bf16(lo, hi, b, s);
    }
}

// Row-contiguous stores of a warp's 32 token rows: lane i holds NV 16-byte pieces of row
// i (its row = base + (row0 + i) * ld, pieces consecutive). Sixteen rows at a time go
// through the warp's 2 KB buffer (16 rows x 128 bytes, the piece index XOR-swizzled by the
// row so neither the writes nor the reads conflict), and come back out with 128 / (16 NV)
// rows per store instruction and each row's bytes from consecutive lanes. Rows at or past
// `nrows` (relative to row0) are not stored. NV is 4 or 8.
template <int NV>
__device__ __forceinline__ void store_rows(uint8_t* buf, const uint4 (&v)[NV], uint8_t* base, size_t ld, int row0,
                                           int nrows, int lane) {
    static_assert(NV == 4 || NV == 8, "a row is 64 or 128 bytes");
    constexpr int RPI = 32 / NV;  // rows per store instruction
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        __syncwarp();
        if ((lane >> 4) == pass) {
            const int r = lane & 15;
#pragma unroll
            for (int c = 0; c < NV; ++c)
                *reinterpret_cast<uint4*>(buf + r * (NV * 16) + ((c ^ (r & (NV - 1))) * 16)) = v[c];
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 16 / RPI; ++it) {
            const int r = it * RPI + lane / NV, c = lane % NV;
            const int row = pass * 16 + r;
            if (row < nrows) {
                const uint4 val = *reinterpret_cast<const uint4*>(buf + r * (NV * 16) + ((c ^ (r & (NV - 1))) * 16));
                *reinterpret_cast<uint4*>(base + (size_t)(row0 + row) * ld + c * 16) = val;
            }
        }
    }
    __syncwarp();
}

// NVFP4 dequantisation of one 64-deep weight row segment: 32 packed bytes (low nibble =
// even K) of E2M1 values (1 sign, 2 exponent bits with bias 1, 1 mantissa bit), one E4M3
// scale per 16 K (`sc` holds the segment's four scale bytes, K 0-15 in the low byte). The
// E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are bf16 values whose high and low bytes are
// two 8-entry byte tables: one byte permute looks up four values' high (or low) bytes at
// once, two more interleave them into bf16 pairs, and a fourth gathers the pair's two sign
// bits into bits 15 and 31. The product with the bf16 scale is exact (at most 6
// significant bits), so the tile holds exactly E2M1 * E4M3.
//   q: one packed word (K 8w .. 8w+7); out[b]: the bf16 pair of its byte b.
__device__ __forceinline__ void fp4_word_bf16(uint32_t q, __nv_bfloat162 s, uint32_t* out) {
    // bf16 bits of the magnitudes, split into high and low bytes (entries 0-3, 4-7)
    constexpr uint32_t kHi03 = 0x3F3F3F00u, kHi47 = 0x40404040u;
    constexpr uint32_t kLo03 = 0xC0800000u, kLo47 = 0xC0804000u;
    const uint32_t m = q & 0x77777777u;  // magnitude codes, one per nibble
    const uint32_t t = q << 4;           // bit 7 of byte b: the sign of byte b's even-K value
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // values 0-3, then 4-7 (the selector takes 4 nibbles)
        const uint32_t sel = h ? (m >> 16) : m;
        const uint32_t hi = byte_perm(kHi03, kHi47, sel);
        const uint32_t lo = byte_perm(kLo03, kLo47, sel);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t b = 2 * h + j;  // the packed byte this pair comes from
            uint32_t u = byte_perm(lo, hi, j ? 0x7362u : 0x5140u);  // lo hi lo hi: two bf16
            // bytes 1 and 3 of the sign word: byte b of t (even value), byte b of q (odd value)
            const uint32_t sg = byte_perm(t, q, b * 0x111u | ((4u + b) << 12));
            u |= sg & 0x80008000u;
            __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&u);
            v = __hmul2(v, s);
            out[b] = *reinterpret_cast<const uint32_t*>(&v);
        }
    }
}

// out[j] = the bf16 pair (K 2j, 2j+1) of a row's 64-deep segment, j < 32; `sc` holds its
// four E4M3 scale bytes (K 0-15 in the low byte).
__device__ __forceinline__ void dequant_fp4_row(const uint8_t* raw, uint32_t sc, uint32_t* out) {
    // the four scales to bf16, two per conversion (every E4M3 value is exact in f16 and in bf16)
    __nv_bfloat162 sb[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const __half2 h2 = __half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)((sc >> (16 * i)) & 0xFFFFu),
                                                              __NV_E4M3));
        sb[i] = __float22bfloat162_rn(__half22float2(h2));
    }
    uint32_t qw[8];
    load_words(raw, qw);
#pragma unroll
    for (int w = 0; w < 8; ++w) {  // two words per scale
        const __nv_bfloat16 s1 = (w & 2) ? sb[w >> 2].y : sb[w >> 2].x;
        fp4_word_bf16(qw[w], __halves2bfloat162(s1, s1), out + 4 * w);
    }
}

// One tile row of a stage into the 32 TMEM columns from `at`.
__device__ __forceinline__ void dequant_store(bool fp4, const uint8_t* raw, uint32_t sc, uint32_t at) {
    uint32_t w[32];
    if (fp4) dequant_fp4_row(raw, sc, w);
    else dequant_int4_row(raw, sc, w);
    tmem_st32(at, w);
}

// Warp-collective bounded wait: lane 0 waits, the verdict is broadcast. CL: the barrier
// has arrivals from the other CTA of a pair (acquire at cluster scope).
template <bool CL = false>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, PipeAbort* ab, int* status) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = CL ? mbar_wait_cl(bar, parity, ab, status) : mbar_wait(bar, parity, ab, status);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmH,
                    const DevArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + C::NBUF;
    uint64_t* ring_full = tempty + C::NBUF;
    uint64_t* ring_empty = ring_full + kRing;
    uint64_t* drain = ring_empty + kRing;
    uint64_t* epibar = drain + 1;
    uint64_t* raw_full = epibar + 1;  // INT4 only: [STAGES]
    uint64_t* pubbar = raw_full + (C::INT4 ? C::STAGES : 0);  // wide FP8 only: a GEMM1 tile's h is stored
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pubbar + (C::WIDE ? 1 : 0));
    PipeAbort* ab = reinterpret_cast<PipeAbort*>(tmem_slot + 1);
    int* ring = reinterpret_cast<int*>(tmem_slot + 4);
    float* red = reinterpret_cast<float*>(ring + kRing + 4);
    float* sct = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(red + C::RED_FLOATS) + 15) & ~uintptr_t(15));
    uint8_t* xpose = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sct + C::SCT_FLOATS) + 15) & ~uintptr_t(15));
    int32_t* blk_start = reinterpret_cast<int32_t*>(xpose + C::XPOSE_BYTES);
    int32_t* s_off = blk_start + (p.G + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;
    // CTA pair: rank 1 mirrors rank 0's barriers but only rank 0's full, tempty and
    // ring_empty count anything: the MMA (issued by rank 0) waits for both CTAs' copies
    // (rank 0 arms the stage with both CTAs' byte counts; rank 1's copies complete their
    // bytes on rank 0's barrier) and both CTAs' epilogues, and rank 0's producer, which
    // claims the tiles and writes them into both CTAs' rings, waits for both CTAs'
    // readers. `lead` maps a barrier to its copy in rank 0.
    const uint32_t rank = C::PAIR ? cluster_ctarank() : 0u;
    auto lead = [&](uint64_t* b) -> uint32_t { return mapa_shared(smem_u32(b), 0); };
    auto peer = [&](const void* v) -> uint32_t { return mapa_shared(smem_u32(v), 1); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], C::INT4 ? C::DQG : 1);  // INT4: the dequantisation warps complete it
            if (C::INT4) mbar_init(&raw_full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < C::NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], (C::PAIR ? 2 : 1) * C::EPI);
        }
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&ring_full[r], 1);
            // readers per CTA: MMA (rank 0) or producer (rank 1), the epilogue, the publisher
            mbar_init(&ring_empty[r], C::PAIR ? 2 * (1 + C::EPI + 1) : 1 + C::EPI + C::DQ + (C::WIDE ? 1 : 0));
        }
        mbar_init(drain, 1);
        mbar_init(epibar, C::EPI);
        if (C::WIDE) mbar_init(pubbar, C::EPI);
        ab->flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        if constexpr (C::PAIR) {  // the same warp in both CTAs: one allocation at one address in both
            tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    // Everything above is private to the SM; the offsets (and all other global data) come
    // from the previous kernels on the stream.
    pdl_wait();
    // Token blocks per group and their running start: blk_start[g] = sum_{g'<g} ceil(n_g'/TB).
    // The offsets may come from the caller: group bounds are clamped into [0, A] (and a
    // bad array is flagged), so no tile ever reads or writes a row outside the matrices.
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int o0 = __ldg(p.offsets + g), o1 = __ldg(p.offsets + g + 1);
        const int lo = min(max(o0, 0), p.A), hi = min(max(o1, lo), p.A);
        if (o0 != lo || o1 != hi) set_status(p.status, MOE_ERR_EXPERT_ID);
        blk_start[g + 1] = (hi - lo + C::TB - 1) / C::TB;
        s_off[g] = lo;
        if (g == G - 1) s_off[G] = min(max(o1, 0), p.A);
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
    // pair: neither CTA signals the other's barriers before both have initialised them
    if constexpr (C::PAIR) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int nblk = blk_start[G];
    const int T1 = nblk * p.c1 * p.s1;
    const int total = T1 + nblk * p.c2;
    const bool chained = p.done1 != nullptr && p.c1 > 0 && p.c2 > 0;

    // Register split of the wide FP8 tile (warpgroup-uniform, at the top of each role so
    // the compiler allocates each role within its own limit): warps 0-3 (producer, MMA,
    // spares) give, the epilogue warps take.
    if (warp < C::EPI0) {
        if constexpr (C::WIDE) setmaxnreg_dec<C::REG_LOW>();
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                tma_prefetch_desc(&tmW1);
                tma_prefetch_desc(&tmX);
                tma_prefetch_desc(&tmW2);
                tma_prefetch_desc(&tmH);
                uint32_t stage = 0, phase = 0, pend_mask = 0, pend_phase = 0;
                bool ok = true;
                // Tiles are claimed one ahead, so the atomic's latency overlaps the current tile.
                // In a CTA pair rank 0 claims and hands every tile number to rank 1 as well.
                const bool claims = !C::PAIR || rank == 0;
                auto claim = [&](int i) -> int {
                    return p.tile_ctr ? (int)atomicAdd(p.tile_ctr, 1u) : (int)(blockIdx.x / (C::PAIR ? 2 : 1)) +
                                                                          i * (int)(gridDim.x / (C::PAIR ? 2 : 1));
                };
                int next_L = claims ? claim(0) : 0;
                // Completion of a stage's copies: this CTA's full barrier, or rank 0's for a pair.
                auto land = [&](uint32_t st) -> uint64_t* { return C::INT4 ? &raw_full[st] : &full[st]; };
                auto load = [&](uint8_t* dst, const CUtensorMap* map, uint32_t st, int x, int y) {
                    if constexpr (C::PAIR) tma_load_2d_pair(dst, map, lead(&full[st]), x, y);
                    else tma_load_2d(dst, map, land(st), x, y);
                };
                for (int i = 0; ok; ++i) {
                    const int slot = i % kRing;
                    int L;
                    if (claims) {
                        L = next_L;
                        if (L >= total) L = -1;
                        else next_L = claim(i + 1);
                        const bool free_slot = C::PAIR ? mbar_wait_cl(&ring_empty[slot], ((i / kRing) & 1) ^ 1, ab, p.status)
                                                       : mbar_wait(&ring_empty[slot], ((i / kRing) & 1) ^ 1, ab, p.status);
                        if (!free_slot) break;
                        ring[slot] = L;
                        if constexpr (C::PAIR) {  // rank 1's copy of the slot, then its ring_full
                            st_cluster_u32(peer(&ring[slot]), (uint32_t)L);
                            mbar_arrive_cluster(peer(&ring_full[slot]));
                        }
                        mbar_arrive(&ring_full[slot]);
                    } else {  // pair rank 1: the tile number comes from rank 0
                        if (!mbar_wait_cl(&ring_full[slot], (i / kRing) & 1, ab, p.status)) break;
                        L = *reinterpret_cast<volatile int*>(&ring[slot]);
                        mbar_arrive_cluster(lead(&ring_empty[slot]));
                    }
                    if (L < 0) break;
                    Tile tl = decode_tile<C::TB>(L, T1, blk_start, s_off, p);
                    const int blk_rows = tl.nrows;  // pair: rows of the whole 256-row block
                    if constexpr (C::PAIR) pair_rows(tl, rank);
                    const bool g1 = tl.phase == 1;
                    const CUtensorMap* tw = g1 ? &tmW1 : &tmW2;
                    const CUtensorMap* ta = g1 ? &tmX : &tmH;
                    const int all_kb = (g1 ? p.H : p.I) / C::BK;
                    const int kbase = g1 ? tl.ks * all_kb / p.s1 : 0;  // this tile's K blocks
                    const int num_kb = g1 ? (tl.ks + 1) * all_kb / p.s1 - kbase : all_kb;
                    // token boxes for `rows` rows (pair: a CTA with no rows of the block loads
                    // none; the MMA's rows from it are never stored)
                    auto boxes = [&](int rows) {
                        return (C::PAIR && rows <= 0) ? 0 : (max(16, (rows + 15) & ~15) + C::BOX_ROWS - 1) / C::BOX_ROWS;
                    };
                    const int n_box = boxes(tl.nrows);
                    // pair: one 128-row weight block per CTA (rank 1 takes A1; without A1 it
                    // loads A0 again, and those accumulator columns are not stored)
                    const int wrow = (C::PAIR && rank == 1 && tl.dual) ? tl.a1row : tl.a0row;
                    // bytes that complete a stage: this CTA's copies, or for a pair both CTAs'
                    // (rank 0 arms the barrier for the pair)
                    const uint32_t tx = C::PAIR ? 2 * C::A_BYTES + (boxes(min(128, blk_rows)) +
                                                                    boxes(min(128, blk_rows - 128))) * C::BOX_BYTES
                                                : (tl.dual ? 2 : 1) * (C::INT4 ? C::RAW_BYTES : C::A_BYTES) +
                                                      n_box * C::BOX_BYTES;
                    auto load_act = [&](uint8_t* st, uint32_t s_idx, int kx) {
                        for (int r = 0; r < n_box; ++r)
                            load(st + C::B_OFF + r * C::BOX_BYTES, ta, s_idx, kx, tl.row0 + r * C::BOX_ROWS);
                    };
                    // GEMM2 after GEMM1 in the same launch: weights of the first stages go out
                    // before waiting for the block's h rows.
                    const bool dep = chained && !g1;
                    const int pre = dep ? min(num_kb, C::STAGES) : 0;
                    const uint32_t st0 = stage;
                    // Wait for the block's h rows (pair: this CTA's half of the block), then
                    // load the activation rows of the prefetched stages. They are loaded even
                    // when the wait gave up (the rows are in bounds; the results are
                    // discarded), so every armed stage completes.
                    auto release_prefetched = [&]() -> bool {
                        const int ctr = C::PAIR ? 2 * tl.blk + (int)rank : tl.blk;
                        const bool dep_ok = wait_counter_geq(p.done1 + ctr, p.c1, ab, p.status);
                        uint32_t s2 = st0;
                        for (int k2 = 0; k2 < pre; ++k2) {
                            load_act(smem + (size_t)s2 * C::STAGE_BYTES, s2, (kbase + k2) * C::BK);
                            if (++s2 == (uint32_t)C::STAGES) s2 = 0;
                        }
                        return dep_ok;
                    };
                    for (int kb = 0; kb < num_kb && ok; ++kb) {
                        if (kb == pre && dep && !release_prefetched()) {
                            ok = false;
                            break;
                        }
                        const bool free_stage = C::PAIR ? mbar_wait_cl(&empty[stage], phase ^ 1, ab, p.status)
                                                        : mbar_wait(&empty[stage], phase ^ 1, ab, p.status);
                        if (!free_stage) {
                            ok = false;
                            break;
                        }
                        uint8_t* st = smem + (size_t)stage * C::STAGE_BYTES;
                        if constexpr (C::PAIR) {
                            if (rank == 0) mbar_arrive_expect_tx(&full[stage], tx);
                        } else {
                            mbar_arrive_expect_tx(land(stage), tx);
                        }
                        const int kx = (kbase + kb) * C::BK;
                        if constexpr (C::INT4) {  // packed weight bytes: x is a byte offset (2 K per byte)
                            load(st + C::RAW_OFF, tw, stage, kx / 2, tl.a0row);
                            if (tl.dual) load(st + C::RAW_OFF + C::RAW_BYTES, tw, stage, kx / 2, tl.a1row);
                        } else if constexpr (C::PAIR) {
                            load(st, tw, stage, kx, wrow);
                        } else {
                            load(st, tw, stage, kx, tl.a0row);
                            if (tl.dual) load(st + C::A_BYTES, tw, stage, kx, tl.a1row);
                        }
                        if (kb >= pre) load_act(st, stage, kx);
                        pend_mask |= 1u << stage;
                        pend_phase = (pend_phase & ~(1u << stage)) | (phase << stage);
                        if (++stage == (uint32_t)C::STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (ok && dep && pre == num_kb && !release_prefetched()) ok = false;  // whole K prefetched
                }
                // Never leave with a copy in flight: wait for the last fill of every stage.
                // (pair: rank 0's full barrier counts both CTAs' copies; rank 1 is held at
                // the kernel's final cluster barrier until rank 0 has drained)
                if (!C::PAIR || rank == 0)
                    for (int s = 0; s < C::STAGES; ++s)
                        if ((pend_mask >> s) & 1u) {
                            if constexpr (C::PAIR) mbar_wait_drain_cl(&full[s], (pend_phase >> s) & 1u);
                            else mbar_wait_drain(land(s), (pend_phase >> s) & 1u);
                        }
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            // (pair: rank 0 issues for both CTAs; rank 1's warp only owns its TMEM share)
            if (lane == 0 && (!C::PAIR || rank == 0)) {
                uint32_t stage = 0, phase = 0, it = 0;
                bool ok = true;
                for (int i = 0; ok; ++i) {
                    const int slot = i % kRing;
                    if (!mbar_wait(&ring_full[slot], (i / kRing) & 1, ab, p.status)) break;
                    const int L = ring[slot];
                    mbar_arrive(&ring_empty[slot]);
                    if (L < 0) break;
                    const Tile tl = decode_tile<C::TB>(L, T1, blk_start, s_off, p);
                    const bool g1 = tl.phase == 1;
                    const int all_kb = (g1 ? p.H : p.I) / C::BK;
                    const int kbase = g1 ? tl.ks * all_kb / p.s1 : 0;
                    const int num_kb = g1 ? (tl.ks + 1) * all_kb / p.s1 - kbase : all_kb;
                    const int n_mma = max(16, (tl.nrows + 15) & ~15);
                    // wide FP8: M = the 128 token rows, N = the 256 (or 128) weight rows
                    // pair: M = 2 x 128 token rows, N = 2 x 128 weight rows (one block from each CTA)
                    const uint32_t idesc = C::PAIR ? idesc_m256(256, C::FP8)
                                                   : (C::WIDE ? idesc_m128(tl.dual ? 256 : 128, true)
                                                              : idesc_m128(n_mma, C::FP8));
                    // bf16: one TMEM buffer per tile; FP8: one per 128-deep K block
                    const int units = C::FP8 ? num_kb : 1;
                    const int kb_per_unit = C::FP8 ? 1 : num_kb;
                    int kb = 0;
                    for (int u = 0; u < units && ok; ++u) {
                        const uint32_t buf = it % C::NBUF, bph = (it / C::NBUF) & 1;
                        const bool drained = C::PAIR ? mbar_wait_cl(&tempty[buf], bph ^ 1, ab, p.status)
                                                     : mbar_wait(&tempty[buf], bph ^ 1, ab, p.status);
                        if (!drained) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d0 = tmem_base + buf * C::ACC_COLS;
                        for (int j = 0; j < kb_per_unit; ++j, ++kb) {
                            const bool landed = C::PAIR ? mbar_wait_cl(&full[stage], phase, ab, p.status)
                                                        : mbar_wait(&full[stage], phase, ab, p.status);
                            if (!landed) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t a0 = smem_u32(smem + (size_t)stage * C::STAGE_BYTES);
                            const uint32_t b0 = a0 + C::B_OFF;
                            const uint32_t at = tmem_base + C::A_TMEM + stage * C::A_TMEM_COLS;  // INT4 A tiles
    #pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t bd = smem_desc_sw128(b0 + kk * 32);
                                const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                                if constexpr (C::INT4) {
                                    mma_bf16_tmem_a(d0, at + kk * 8, bd, idesc, acc);
                                    if (tl.dual) mma_bf16_tmem_a(d0 + C::BN, at + 32 + kk * 8, bd, idesc, acc);
                                } else if constexpr (C::PAIR) {
                                    // token tiles (A, 128 rows per CTA) x weight blocks (B, 128 rows per CTA)
                                    if constexpr (C::FP8) mma_fp8_pair(d0, bd, smem_desc_sw128(a0 + kk * 32), idesc, acc);
                                    else mma_bf16_pair(d0, bd, smem_desc_sw128(a0 + kk * 32), idesc, acc);
                                } else if constexpr (C::WIDE) {
                                    // the token tile is the A operand; A0 | A1 (contiguous) the B operand
                                    mma_fp8(d0, bd, smem_desc_sw128(a0 + kk * 32), idesc, acc);
                                } else if constexpr (C::FP8) {
                                    mma_fp8(d0, smem_desc_sw128(a0 + kk * 32), bd, idesc, acc);
                                    if (tl.dual)
                                        mma_fp8(d0 + C::BN, smem_desc_sw128(a0 + C::A_BYTES + kk * 32), bd, idesc, acc);
                                } else {
                                    mma_bf16(d0, smem_desc_sw128(a0 + kk * 32), bd, idesc, acc);
                                    if (tl.dual)
                                        mma_bf16(d0 + C::BN, smem_desc_sw128(a0 + C::A_BYTES + kk * 32), bd, idesc, acc);
                                }
                            }
                            // the stage is free in both CTAs once these MMAs have read it
                            if constexpr (C::PAIR) tc_commit_pair_both(&empty[stage]);
                            else tc_commit(&empty[stage]);
                            if (++stage == (uint32_t)C::STAGES) {
                                stage = 0;
                                phase ^= 1;
                            }
                        }
                        if (!ok) break;
                        if constexpr (C::PAIR) tc_commit_pair_both(&tfull[buf]);
                        else tc_commit(&tfull[buf]);
                        ++it;
                    }
                }
                // All MMAs issued by this thread complete before TMEM is released.
                if constexpr (C::PAIR) tc_commit_pair(drain);
                else tc_commit(drain);
                mbar_wait_drain(drain, 0);
            }
            __syncwarp();
        } else if (C::WIDE && warp == 2) {
            // -------------------------------------------------------- publisher (wide FP8)
            // Releases each GEMM1 tile's h rows to the GEMM2 tiles of its block once every
            // epilogue warp has stored its share (pubbar: arrive = release, wait = acquire at
            // CTA scope, then a GPU-scope fence and a release add), so that fence, which can
            // take microseconds under a saturated memory system, stays off the epilogue.
            if (lane == 0) {
                uint32_t pph = 0;
                for (int i = 0;; ++i) {
                    const int slot = i % kRing;
                    const bool got = C::PAIR ? mbar_wait_cl(&ring_full[slot], (i / kRing) & 1, ab, p.status)
                                             : mbar_wait(&ring_full[slot], (i / kRing) & 1, ab, p.status);
                    if (!got) break;
                    const int L = *reinterpret_cast<volatile int*>(&ring[slot]);
                    if constexpr (C::PAIR) mbar_arrive_cluster(lead(&ring_empty[slot]));
                    else mbar_arrive(&ring_empty[slot]);
                    if (L < 0) break;
                    if (!chained || L >= T1) continue;  // GEMM1 tiles of a two-phase launch only
                    if (!mbar_wait(pubbar, pph, ab, p.status)) break;
                    pph ^= 1;
                    __threadfence();
                    fence_proxy_async_global();
                    // pair: one counter per 128-row half of the block, completed by this CTA's tiles
                    const int blk = (L / p.s1) / p.c1;
                    red_release_add_gpu(p.done1 + (C::PAIR ? 2 * blk + (int)rank : blk), 1);
                }
            }
            __syncwarp();
        }
    } else if (C::INT4 && warp >= C::EPI0 + C::EPI) {
        // ------------------------------------------------------------ INT4 dequantisation
        // Each warp converts the 32 weight rows of its TMEM lane quarter (warp % 4) of both
        // tiles (A0, A1) of every stage of its stage group, in the same order as the MMA,
        // stores them into the stage's TMEM A columns and completes `full`.
        const int r = (warp & 3) * 32 + lane;
        const int grp = (warp - C::EPI0 - C::EPI) / C::DQG;  // this warp's stage group
        const uint32_t lane_sel = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t stage = 0, phase = 0, n_run = 0;  // n_run: stages of earlier tiles
        bool ok = true;
        for (int i = 0; ok; ++i) {
            const int slot = i % kRing;
            if (!warp_wait(&ring_full[slot], (i / kRing) & 1, ab, p.status)) break;
            const int L = ring[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&ring_empty[slot]);
            if (L < 0) break;
            const Tile tl = decode_tile<C::TB>(L, T1, blk_start, s_off, p);
            const bool g1 = tl.phase == 1;
            const int K = g1 ? p.H : p.I;
            const int all_kb = K / C::BK;
            const int kbase = g1 ? tl.ks * all_kb / p.s1 : 0;
            const int num_kb = g1 ? (tl.ks + 1) * all_kb / p.s1 - kbase : all_kb;
            // this thread's row of tile A0 and, for a tile pair, of A1; the row's scales are
            // one 32-bit word per 64-deep stage: INT4 two bf16 group scales ([rows][K/32]),
            // NVFP4 four E4M3 block scales ([rows][K/16])
            const bool both = tl.dual;
            const uint32_t* sc = static_cast<const uint32_t*>(g1 ? p.w1_scale : p.w2_scale);
            const uint32_t* sc0 = sc + (size_t)(tl.a0row + r) * (K / 64) + kbase;
            const uint32_t* sc1 = sc + (size_t)(tl.a1row + r) * (K / 64) + kbase;
            // this group's stages of the tile: kb = kb_first, kb_first + NGRP, ...
            const int kb_first = (int)((uint32_t)(grp - (int)(n_run % C::NGRP) + C::NGRP) % C::NGRP);
            const bool any = kb_first < num_kb;
            uint32_t s0 = any ? __ldg(sc0 + kb_first) : 0u, s1 = (any && both) ? __ldg(sc1 + kb_first) : 0u;
            for (int kb = 0; kb < num_kb; ++kb) {
                if ((int)((n_run + kb) % C::NGRP) != grp) {  // another group's stage
                    if (++stage == (uint32_t)C::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                    continue;
                }
                // the next stage's scales are loaded before this stage's bytes are awaited
                const bool more = kb + C::NGRP < num_kb;
                const uint32_t n0 = more ? __ldg(sc0 + kb + C::NGRP) : 0u;
                const uint32_t n1 = (more && both) ? __ldg(sc1 + kb + C::NGRP) : 0u;
                if (!warp_wait(&raw_full[stage], phase, ab, p.status)) {
                    ok = false;
                    break;
                }
                const uint8_t* raw = smem + (size_t)stage * C::STAGE_BYTES + C::RAW_OFF + r * 32;
                const uint32_t at = tmem_base + lane_sel + C::A_TMEM + stage * C::A_TMEM_COLS;
                dequant_store(p.fp4, raw, s0, at);
                if (both) dequant_store(p.fp4, raw + C::RAW_BYTES, s1, at + 32);  // warp-uniform
                tc_fence_before();  // the tensor-memory stores happen before the MMA that reads them
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[stage]);
                if (++stage == (uint32_t)C::STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
                s0 = n0;
                s1 = n1;
            }
            n_run += (uint32_t)num_kb;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        if constexpr (C::WIDE) setmaxnreg_inc<C::REG_HIGH>();
        const int ew = warp - C::EPI0;
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int cg = ew >> 2;  // which group of the tile's columns
        const int c0 = cg * C::COLS;
        const int row_local = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        uint32_t it = 0, ephase = 0;
        uint32_t g1_tiles = 0;  // wide FP8: GEMM1 tiles done (parity picks the amax buffer)
        bool ok = true;
        int* merge_flag = ring + kRing + 1;
        // Split-K of GEMM1: this split's partials are in memory. Returns 1 when this CTA
        // holds the last split of the tile (and merges), 0 when another split merges, -1
        // when the CTA aborted. The counter goes back to zero in the merging CTA.
        // Ordering: the warps' partial stores reach the counting thread through the CTA
        // barrier (mbarrier arrive = release, wait = acquire, CTA scope); its GPU-scope fence
        // before the counter increment publishes them, and the merging CTA's fence after
        // reading the counter orders its loads of the other splits' partials.
        auto split_arrive = [&](int tile1) -> int {
            __syncwarp();
            if (lane == 0) mbar_arrive(epibar);
            if (!warp_wait(epibar, ephase, ab, p.status)) return -1;
            ephase ^= 1;
            if (ew == 0 && lane == 0) {
                __threadfence();
                const int old = atomicAdd(p.split_cnt + tile1, 1);
                const int last = old == p.s1 - 1;
                if (last) {
                    __threadfence();
                    p.split_cnt[tile1] = 0;
                }
                *merge_flag = last;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(epibar);
            if (!warp_wait(epibar, ephase, ab, p.status)) return -1;
            ephase ^= 1;
            return *reinterpret_cast<volatile int*>(merge_flag);
        };
        // partial of split ks, half (0 gate, 1 up), column n, this thread's row
        auto part_at = [&](int tile1, int ks, int half, int n) -> float* {
            return p.part + (((size_t)(tile1 * p.s1 + ks) * 2 + half) * C::BN + n) * 128 + row_local;
        };
        for (int i = 0; ok; ++i) {
            const int slot = i % kRing;
            if (!warp_wait<C::PAIR>(&ring_full[slot], (i / kRing) & 1, ab, p.status)) break;
            const int L = *reinterpret_cast<volatile int*>(&ring[slot]);
            __syncwarp();
            if (lane == 0) {
                if constexpr (C::PAIR) mbar_arrive_cluster(lead(&ring_empty[slot]));
                else mbar_arrive(&ring_empty[slot]);
            }
            if (L < 0) break;
            Tile tl = decode_tile<C::TB>(L, T1, blk_start, s_off, p);
            if constexpr (C::PAIR) pair_rows(tl, rank);
            const bool g1 = tl.phase == 1;
            const int n_mma = max(16, (tl.nrows + 15) & ~15);
            // output columns of this thread: A0's and A1's row (intermediate or hidden index)
            const int col = tl.col0 + row_local, col_b = tl.col1 + row_local;
            const int out_ld = g1 ? p.I : p.H;
            const float sg = (g1 && p.gate_scale) ? __ldg(p.gate_scale + tl.g) : 1.f;
            const float su = (g1 && p.up_scale) ? __ldg(p.up_scale + tl.g) : 1.f;
            const float lim = (g1 && p.limits) ? __ldg(p.limits + tl.g) : p.limit;  // this expert's clamp
            if constexpr (!C::FP8 && !C::WIDE) {
                const uint32_t buf = it % C::NBUF, bph = (it / C::NBUF) & 1;
                if (!warp_wait(&tfull[buf], bph, ab, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tb = tmem_base + lane_off + buf * C::ACC_COLS;
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g1 ? p.h : p.y);
                const int tile1 = tl.blk * p.c1 + tl.c;
                if (C::SPLIT_OK && g1 && p.s1 > 1) {
                    // split-K: store this split's fp32 gate/up sums; the last split merges
#pragma unroll 1
                    for (int cc = c0; cc < c0 + C::COLS && cc < n_mma; cc += C::CW) {
                        float gv[C::CW], uv[C::CW];
                        tmem_ld_x2<C::CW>(tb + cc, tb + C::BN + cc, gv, uv);
#pragma unroll
                        for (int j = 0; j < C::CW; ++j) {
                            *part_at(tile1, tl.ks, 0, cc + j) = gv[j];
                            *part_at(tile1, tl.ks, 1, cc + j) = uv[j];
                        }
                    }
                } else if (g1) {
#pragma unroll 1
                    for (int cc = c0; cc < c0 + C::COLS && cc < n_mma; cc += C::CW) {
                        float gv[C::CW], uv[C::CW];
                        tmem_ld_x2<C::CW>(tb + cc, tb + C::BN + cc, gv, uv);
#pragma unroll
                        for (int j = 0; j < C::CW; ++j) {
                            const int n = cc + j;
                            if (n < tl.nrows) {
                                const float h = swiglu_dev(sg * gv[j], su * uv[j], p.alpha, p.beta, lim);
                                out[(size_t)(tl.row0 + n) * out_ld + col] = __float2bfloat16_rn(h);
                            }
                        }
                    }
                } else if (tl.dual) {
#pragma unroll 1
                    for (int cc = c0; cc < c0 + C::COLS && cc < n_mma; cc += C::CW) {
                        float v[C::CW], v2[C::CW];
                        tmem_ld_x2<C::CW>(tb + cc, tb + C::BN + cc, v, v2);
#pragma unroll
                        for (int j = 0; j < C::CW; ++j) {
                            const int n = cc + j;
                            if (n < tl.nrows) {
                                __nv_bfloat16* row = out + (size_t)(tl.row0 + n) * out_ld;
                                row[col] = __float2bfloat16_rn(v[j]);
                                row[col_b] = __float2bfloat16_rn(v2[j]);
                            }
                        }
                    }
                } else {
#pragma unroll 1
                    for (int cc = c0; cc < c0 + C::COLS && cc < n_mma; cc += C::CW) {
                        float v[C::CW];
                        tmem_ld_x1<C::CW>(tb + cc, v);
#pragma unroll
                        for (int j = 0; j < C::CW; ++j) {
                            const int n = cc + j;
                            if (n < tl.nrows) out[(size_t)(tl.row0 + n) * out_ld + col] = __float2bfloat16_rn(v[j]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
                ++it;
                if (C::SPLIT_OK && g1 && p.s1 > 1) {
                    const int r = split_arrive(tile1);
                    if (r < 0) {
                        ok = false;
                        break;
                    }
                    if (r == 0) continue;  // another split of this tile writes h
                    const float* ptile = part_at(tile1, 0, 0, 0) - row_local;
#pragma unroll 1
                    for (int j0 = 0; j0 < C::COLS && c0 + j0 < tl.nrows; j0 += 8) {
                        float gs[8], us[8];
                        sum_split_partials<8>(ptile, p.s1, C::BN, c0 + j0, row_local, gs, us);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int n = c0 + j0 + j;
                            if (n < tl.nrows) {
                                const float hv = swiglu_dev(sg * gs[j], su * us[j], p.alpha, p.beta, lim);
                                out[(size_t)(tl.row0 + n) * out_ld + col] = __float2bfloat16_rn(hv);
                            }
                        }
                    }
                }
            } else if constexpr (C::WIDE && !C::FP8) {
                // Token-major bf16 tile (CTA pair): TMEM lane = token row, columns = this
                // tile's 256 weight rows (gate | up, or two 128-row chunks of H), summed over
                // the whole K range in one buffer. This warp takes columns cg*CC .. +CC of
                // each half and writes its token's row piece of h (SwiGLU of the per-group
                // scaled gate and up) or of y, 16 bytes at a time, row-contiguously.
                constexpr int CC = C::COLS;
                constexpr int W = 16;
                const bool quarter_live = q * 32 < tl.nrows;  // warp-uniform
                const uint32_t buf = it % C::NBUF, bph = (it / C::NBUF) & 1;
                if (!warp_wait<C::PAIR>(&tfull[buf], bph, ab, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tb = tmem_base + lane_off + buf * C::ACC_COLS + cg * CC;
                auto release = [&]() {  // the buffer goes back to the MMA (pair: to rank 0)
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (C::PAIR) mbar_arrive_remote(lead(&tempty[buf]));
                        else mbar_arrive(&tempty[buf]);
                    }
                };
                if (!quarter_live) {
                    release();  // no token of this lane quarter in the tile
                } else if (g1) {
                    uint4 hv[CC / 8];  // this token's CC values of h, 8 bf16 per piece
#pragma unroll
                    for (int ch = 0; ch < CC / W; ++ch) {
                        float gv[W], uv[W];
                        tmem_ld_x2<W>(tb + ch * W, tb + C::BN + ch * W, gv, uv);
                        if (ch == CC / W - 1) release();  // before the arithmetic
#pragma unroll
                        for (int v = 0; v < W / 8; ++v) {
                            uint32_t w[4];
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const int j = v * 8 + 2 * t;
                                const float h0 = swiglu_dev(sg * gv[j], su * uv[j], p.alpha, p.beta, lim);
                                const float h1 = swiglu_dev(sg * gv[j + 1], su * uv[j + 1], p.alpha, p.beta, lim);
                                const __nv_bfloat162 b = __floats2bfloat162_rn(h0, h1);
                                w[t] = *reinterpret_cast<const uint32_t*>(&b);
                            }
                            hv[ch * (W / 8) + v] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    store_rows<CC / 8>(xpose + ew * 2048, hv,
                                       static_cast<uint8_t*>(p.h) + 2 * (size_t)(tl.col0 + cg * CC), 2 * (size_t)p.I,
                                       tl.row0 + q * 32, tl.nrows - q * 32, lane);
                } else {
                    // y rows (H % 128 == 0, y 16-byte aligned): this token's CC bf16 of each half
                    uint8_t* ybase = static_cast<uint8_t*>(p.y);
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        if (half == 1 && !tl.dual) break;  // the second block's columns are not stored
                        uint4 yv[CC / 8];
#pragma unroll
                        for (int ch = 0; ch < CC / W; ++ch) {
                            float v[W];
                            tmem_ld_x1<W>(tb + half * C::BN + ch * W, v);
#pragma unroll
                            for (int u = 0; u < W / 8; ++u) {
                                uint32_t w[4];
#pragma unroll
                                for (int t = 0; t < 4; ++t) {
                                    const __nv_bfloat162 b =
                                        __floats2bfloat162_rn(v[u * 8 + 2 * t], v[u * 8 + 2 * t + 1]);
                                    w[t] = *reinterpret_cast<const uint32_t*>(&b);
                                }
                                yv[ch * (W / 8) + u] = make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                        if (half == 1 || !tl.dual) release();  // after the tile's last TMEM load
                        const int colb = (half ? tl.col1 : tl.col0) + cg * CC;  // first bf16 column
                        store_rows<CC / 8>(xpose + ew * 2048, yv, ybase + 2 * (size_t)colb, 2 * (size_t)p.H,
                                           tl.row0 + q * 32, tl.nrows - q * 32, lane);
                    }
                }
                ++it;
            } else if constexpr (C::WIDE) {
                // Token-major FP8 tile: TMEM lane = token row of the block, columns = weight
                // rows (gate | up, or two 128-row chunks of H). This warp takes columns
                // cg*CC .. +CC of each half, so a thread holds gate and up of CC intermediate
                // indices of its own token, and a K block's scale product is one scalar per
                // half: no per-column scale table, a thread-local amax for h's 1x128 block
                // (plus the other column group's, through shared memory), and whole 16-byte
                // stores of h and y rows.
                constexpr int CC = C::COLS;  // columns of each half per warp
                const int tok = row_local;
                const bool has_tok = tok < tl.nrows;
                const bool quarter_live = q * 32 < tl.nrows;  // warp-uniform
                const int num_kb = (g1 ? p.H : p.I) / C::BK;   // no split-K at this width
                const float* act_scale = g1 ? p.x_scale : p.h_scale;
                const float* wscale = static_cast<const float*>(g1 ? p.w1_scale : p.w2_scale);
                const float* wsg = wscale + (size_t)(tl.a0row / 128) * num_kb;
                const float* wsu = wscale + (size_t)(tl.a1row / 128) * num_kb;
                if (!g1 && chained) {  // h_scale comes from GEMM1 tiles of this block (see below)
                    bool dep_ok = true;
                    const int ctr = C::PAIR ? 2 * tl.blk + (int)rank : tl.blk;
                    if (lane == 0) dep_ok = wait_counter_geq(p.done1 + ctr, p.c1, ab, p.status);
                    dep_ok = __shfl_sync(0xffffffffu, dep_ok ? 1 : 0, 0) != 0;
                    __syncwarp();
                    if (!dep_ok) {
                        ok = false;
                        break;
                    }
                }
                float acc0[CC], acc1[CC];
#pragma unroll
                for (int j = 0; j < CC; ++j) acc0[j] = acc1[j] = 0.f;
                constexpr int kPF = 4;  // K blocks of scales loaded ahead
                const float* sb_ptr = act_scale + tl.row0 + tok;
                float q_sb[kPF], q_s0[kPF], q_s1[kPF];
#pragma unroll
                for (int i = 0; i < kPF; ++i) {
                    const bool in = i < num_kb;
                    q_sb[i] = (in && has_tok) ? __ldcg(sb_ptr + (size_t)i * p.A) : 0.f;
                    q_s0[i] = in ? __ldg(wsg + i) : 0.f;
                    q_s1[i] = (in && tl.dual) ? __ldg(wsu + i) : 0.f;
                }
                for (int kb = 0; kb < num_kb; ++kb) {
                    const uint32_t buf = it % C::NBUF, bph = (it / C::NBUF) & 1;
                    const float f0 = q_s0[0] * q_sb[0], f1 = q_s1[0] * q_sb[0];
#pragma unroll
                    for (int i = 0; i + 1 < kPF; ++i) {
                        q_sb[i] = q_sb[i + 1];
                        q_s0[i] = q_s0[i + 1];
                        q_s1[i] = q_s1[i + 1];
                    }
                    {
                        const int kn = kb + kPF;
                        const bool in = kn < num_kb;
                        q_sb[kPF - 1] = (in && has_tok) ? __ldcg(sb_ptr + (size_t)kn * p.A) : 0.f;
                        q_s0[kPF - 1] = in ? __ldg(wsg + kn) : 0.f;
                        q_s1[kPF - 1] = (in && tl.dual) ? __ldg(wsu + kn) : 0.f;
                    }
                    if (!warp_wait<C::PAIR>(&tfull[buf], bph, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tb = tmem_base + lane_off + buf * C::ACC_COLS + cg * CC;
                    // the buffer goes back to the MMA (pair: to rank 0, which issues it)
                    auto release = [&]() {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (C::PAIR) mbar_arrive_remote(lead(&tempty[buf]));  // per K block: no store wait
                            else mbar_arrive(&tempty[buf]);
                        }
                    };
                    if (!quarter_live) release();  // no token of this lane quarter in the tile
                    constexpr int W = C::WCH;
#pragma unroll
                    for (int ch = 0; ch < CC / W; ++ch) {
                        if (!quarter_live) break;
                        float p0[W], p1[W];
                        if (tl.dual) tmem_ld_x2<W>(tb + ch * W, tb + C::BN + ch * W, p0, p1);
                        else tmem_ld_x1<W>(tb + ch * W, p0);
                        if (ch == CC / W - 1) release();  // before the arithmetic
#pragma unroll
                        for (int j = 0; j < W; j += 2) {
                            ffma2(acc0[ch * W + j], acc0[ch * W + j + 1], p0[j], p0[j + 1], f0, f0);
                            if (tl.dual) ffma2(acc1[ch * W + j], acc1[ch * W + j + 1], p1[j], p1[j + 1], f1, f1);
                        }
                    }
                    ++it;
                }
                if (!ok) break;
                if (g1) {
                    float amax = 0.f;
#pragma unroll
                    for (int j = 0; j < CC; ++j) {
                        acc0[j] = swiglu_dev(sg * acc0[j], su * acc1[j], p.alpha, p.beta, lim);
                        amax = fmaxf(amax, fabsf(acc0[j]));
                    }
                    float* rb = red + (g1_tiles++ & 1) * (C::GROUPS * 128);  // two tiles' worth: no second meeting
                    rb[cg * 128 + tok] = amax;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(epibar);
                    if (!warp_wait(epibar, ephase, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    ephase ^= 1;
#pragma unroll
                    for (int g = 0; g < C::GROUPS; ++g) amax = fmaxf(amax, rb[g * 128 + tok]);  // the 1x128 block
                    const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
                    const float inv_s = amax == 0.f ? 1.f : __fdividef(448.f, amax);
                    {
                        uint4 hv[CC / 16];  // this token's CC codes
#pragma unroll
                        for (int v = 0; v < CC / 16; ++v) {
                            uint32_t w[4];
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const int j = v * 16 + t * 4;
                                const uint32_t lo = __nv_cvt_float2_to_fp8x2(
                                    make_float2(acc0[j] * inv_s, acc0[j + 1] * inv_s), __NV_SATFINITE, __NV_E4M3);
                                const uint32_t hi = __nv_cvt_float2_to_fp8x2(
                                    make_float2(acc0[j + 2] * inv_s, acc0[j + 3] * inv_s), __NV_SATFINITE, __NV_E4M3);
                                w[t] = lo | (hi << 16);
                            }
                            hv[v] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                        store_rows<CC / 16>(xpose + ew * 2048, hv, static_cast<uint8_t*>(p.h) + tl.col0 + cg * CC,
                                            (size_t)p.I, tl.row0 + q * 32, tl.nrows - q * 32, lane);
                        if (has_tok && cg == 0) p.h_scale[(size_t)tl.c * p.A + tl.row0 + tok] = s;
                    }
                } else {
                    // y rows (H % 128 == 0, y 16-byte aligned): this token's CC bf16 of each half
                    uint8_t* ybase = static_cast<uint8_t*>(p.y);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        if (half == 1 && !tl.dual) break;
                        const float* a = half ? acc1 : acc0;
                        uint4 yv[CC / 8];
#pragma unroll
                        for (int v = 0; v < CC / 8; ++v) {
                            uint32_t w[4];
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const __nv_bfloat162 b = __floats2bfloat162_rn(a[v * 8 + 2 * t], a[v * 8 + 2 * t + 1]);
                                w[t] = *reinterpret_cast<const uint32_t*>(&b);
                            }
                            yv[v] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                        const int colb = (half ? tl.col1 : tl.col0) + cg * CC;  // first bf16 column
                        store_rows<CC / 8>(xpose + ew * 2048, yv, ybase + 2 * (size_t)colb, 2 * (size_t)p.H,
                                           tl.row0 + q * 32, tl.nrows - q * 32, lane);
                    }
                }
            } else {
                const int kblocks = (g1 ? p.H : p.I) / C::BK;  // BK = 128 for FP8: one scale per K block
                const int kbase = g1 ? tl.ks * kblocks / p.s1 : 0;
                const int num_kb = g1 ? (tl.ks + 1) * kblocks / p.s1 - kbase : kblocks;
                const float* act_scale = g1 ? p.x_scale : p.h_scale;
                // block scales of A0 and A1: weight row block a_row / 128 of the [G*rows/128][K/128] grid
                const float* wscale = static_cast<const float*>(g1 ? p.w1_scale : p.w2_scale);
                const float* wsg = wscale + (size_t)(tl.a0row / 128) * kblocks + kbase;
                const float* wsu = wscale + (size_t)(tl.a1row / 128) * kblocks + kbase;
                float acc_g[C::COLS], acc_u[C::COLS];
#pragma unroll
                for (int j = 0; j < C::COLS; ++j) acc_g[j] = acc_u[j] = 0.f;
                // h_scale of a GEMM2 tile is written by the GEMM1 tiles of its block, in
                // other CTAs of this launch and possibly still running: this warp waits for
                // the block's counter itself (acquire) before its first scale load, and
                // reads the scales through L2.
                if (!g1 && chained) {
                    bool dep_ok = true;
                    if (lane == 0) dep_ok = wait_counter_geq(p.done1 + tl.blk, p.c1, ab, p.status);
                    dep_ok = __shfl_sync(0xffffffffu, dep_ok ? 1 : 0, 0) != 0;
                    __syncwarp();  // orders lane 0's acquire before every lane's scale loads
                    if (!dep_ok) {
                        ok = false;
                        break;
                    }
                }
                // This warp's scale products: tab[j] = sa0 * sb[c0+j], tab[COLS+j] = sa1 * sb[c0+j].
                // The scales of block kb are loaded kPF blocks ahead (a register ring), so the
                // L2 latency of those loads stays off the tensor core's critical path.
                float* tab = sct + ew * 2 * C::COLS;
                constexpr int kPF = C::BN >= 64 ? 2 : 4;
                const bool has_col = lane < C::COLS && c0 + lane < tl.nrows;
                const float* sb_ptr = act_scale + (size_t)kbase * p.A + tl.row0 + c0 + lane;
                float q_sb[kPF], q_s0[kPF], q_s1[kPF];
#pragma unroll
                for (int i = 0; i < kPF; ++i) {
                    const bool in = i < num_kb;
                    q_sb[i] = (in && has_col) ? __ldcg(sb_ptr + (size_t)i * p.A) : 0.f;
                    q_s0[i] = in ? __ldg(wsg + i) : 0.f;
                    q_s1[i] = (in && tl.dual) ? __ldg(wsu + i) : 0.f;
                }
                for (int kb = 0; kb < num_kb; ++kb) {
                    const uint32_t buf = it % C::NBUF, bph = (it / C::NBUF) & 1;
                    {
                        const float sb = q_sb[0], sa0 = q_s0[0], sa1 = q_s1[0];
#pragma unroll
                        for (int i = 0; i + 1 < kPF; ++i) {
                            q_sb[i] = q_sb[i + 1];
                            q_s0[i] = q_s0[i + 1];
                            q_s1[i] = q_s1[i + 1];
                        }
                        const int kn = kb + kPF;
                        const bool in = kn < num_kb;
                        q_sb[kPF - 1] = (in && has_col) ? __ldcg(sb_ptr + (size_t)kn * p.A) : 0.f;
                        q_s0[kPF - 1] = in ? __ldg(wsg + kn) : 0.f;
                        q_s1[kPF - 1] = (in && tl.dual) ? __ldg(wsu + kn) : 0.f;
                        __syncwarp();  // the previous block's reads of tab are done
                        if (lane < C::COLS) {
                            tab[lane] = sa0 * sb;
                            tab[C::COLS + lane] = sa1 * sb;
                        }
                        __syncwarp();
                    }
                    if (!warp_wait(&tfull[buf], bph, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tb = tmem_base + lane_off + buf * C::ACC_COLS;
                    // Partials in chunks of 16 columns; the TMEM buffer goes back to the MMA as
                    // soon as the last chunk is in registers, before its arithmetic runs.
                    const bool live = c0 < n_mma;  // warp-uniform
                    if (!live) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty[buf]);
                    }
#pragma unroll
                    for (int ch = 0; ch < C::COLS / C::CW; ++ch) {
                        if (!live) break;
                        const int cc = c0 + ch * C::CW;
                        float pg[C::CW], pu[C::CW];
                        if (tl.dual) tmem_ld_x2<C::CW>(tb + cc, tb + C::BN + cc, pg, pu);
                        else tmem_ld_x1<C::CW>(tb + cc, pg);
                        if (ch == C::COLS / C::CW - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&tempty[buf]);
                        }
#pragma unroll
                        for (int j = 0; j < C::CW; j += 4) {
                            const int jj = ch * C::CW + j;
                            const float4 s0 = *reinterpret_cast<const float4*>(tab + jj);
                            ffma2(acc_g[jj], acc_g[jj + 1], pg[j], pg[j + 1], s0.x, s0.y);
                            ffma2(acc_g[jj + 2], acc_g[jj + 3], pg[j + 2], pg[j + 3], s0.z, s0.w);
                            if (tl.dual) {
                                const float4 s1 = *reinterpret_cast<const float4*>(tab + C::COLS + jj);
                                ffma2(acc_u[jj], acc_u[jj + 1], pu[j], pu[j + 1], s1.x, s1.y);
                                ffma2(acc_u[jj + 2], acc_u[jj + 3], pu[j + 2], pu[j + 3], s1.z, s1.w);
                            }
                        }
                    }
                    ++it;
                }
                if (!ok) break;
                if (C::SPLIT_OK && g1 && p.s1 > 1) {
                    // split-K: store this split's promoted sums; the last split merges
                    const int tile1 = tl.blk * p.c1 + tl.c;
#pragma unroll
                    for (int j = 0; j < C::COLS; ++j) {
                        *part_at(tile1, tl.ks, 0, c0 + j) = acc_g[j];
                        *part_at(tile1, tl.ks, 1, c0 + j) = acc_u[j];
                    }
                    const int r = split_arrive(tile1);
                    if (r < 0) {
                        ok = false;
                        break;
                    }
                    if (r == 0) continue;  // another split of this tile writes h
                    const float* ptile = part_at(tile1, 0, 0, 0) - row_local;
#pragma unroll
                    for (int j0 = 0; j0 < C::COLS; j0 += 8)
                        sum_split_partials<8>(ptile, p.s1, C::BN, c0 + j0, row_local, acc_g + j0, acc_u + j0);
                }
                if (g1) {
                    // SwiGLU, then 1x128 E4M3 quantisation of h: the block of row r is the
                    // 128 intermediate indices of this chunk = the 4 lane quarters.
#pragma unroll
                    for (int j = 0; j < C::COLS; ++j) {
                        acc_g[j] = swiglu_dev(sg * acc_g[j], su * acc_u[j], p.alpha, p.beta, lim);
                        float m = fabsf(acc_g[j]);
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                        if (lane == 0) red[(cg * 4 + q) * C::COLS + j] = m;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(epibar);
                    if (!warp_wait(epibar, ephase, ab, p.status)) {
                        ok = false;
                        break;
                    }
                    ephase ^= 1;
                    uint8_t* out = static_cast<uint8_t*>(p.h);
#pragma unroll
                    for (int j = 0; j < C::COLS; ++j) {
                        const int n = c0 + j;
                        float amax = red[(cg * 4 + 0) * C::COLS + j];
                        amax = fmaxf(amax, red[(cg * 4 + 1) * C::COLS + j]);
                        amax = fmaxf(amax, red[(cg * 4 + 2) * C::COLS + j]);
                        amax = fmaxf(amax, red[(cg * 4 + 3) * C::COLS + j]);
                        const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
                        const float inv_s = amax == 0.f ? 1.f : __fdividef(448.f, amax);
                        if (n < tl.nrows) {
                            out[(size_t)(tl.row0 + n) * p.I + col] =
                                (uint8_t)__nv_cvt_float_to_fp8(acc_g[j] * inv_s, __NV_SATFINITE, __NV_E4M3);
                            if (q == 0 && lane == 0) p.h_scale[(size_t)tl.c * p.A + tl.row0 + n] = s;
                        }
                    }
                } else {
                    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.y);
#pragma unroll
                    for (int j = 0; j < C::COLS; ++j) {
                        const int n = c0 + j;
                        if (n < tl.nrows) {
                            __nv_bfloat16* row = out + (size_t)(tl.row0 + n) * p.H;
                            row[col] = __float2bfloat16_rn(acc_g[j]);
                            if (tl.dual) row[col_b] = __float2bfloat16_rn(acc_u[j]);
                        }
                    }
                }
            }
            // GEMM1 tile done: publish its h rows (and scales) to GEMM2 tiles of this block.
            // The epilogue warps meet (their stores reach the meeting thread through the
            // CTA-scope mbarrier: arrive = release, wait = acquire), and one thread fences at
            // GPU scope and for the async proxy and releases the block counter; a reader
            // acquires the counter and fences the async proxy before its TMA loads. One
            // fencing thread instead of every thread: under a saturated memory system each
            // fence waits microseconds for its stores to be acknowledged. In FP8 mode the
            // meeting also keeps `red` from being rewritten while read.
            if constexpr (C::WIDE) {
                if (g1 && chained) {  // the publisher warp releases the block counter
                    __syncwarp();
                    if (lane == 0) mbar_arrive(pubbar);
                }
            } else if (g1 && (chained || C::FP8)) {
                __syncwarp();
                if (lane == 0) mbar_arrive(epibar);
                if (!warp_wait(epibar, ephase, ab, p.status)) {
                    ok = false;
                    break;
                }
                ephase ^= 1;
                if (chained && ew == 0 && lane == 0) {
                    __threadfence();
                    fence_proxy_async_global();
                    red_release_add_gpu(p.done1 + tl.blk, 1);
                }
            }
        }
    }

    pdl_trigger();  // this CTA has no tiles left: the next kernel may launch
    __syncthreads();
    // pair: rank 0 has drained its MMAs (which write rank 1's TMEM and read rank 1's
    // shared memory) and its copies before either CTA frees TMEM or exits
    if constexpr (C::PAIR) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (C::PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
    // The CTA that finishes last leaves the tile counter, the exit counter and the block
    // flags at zero for the next launch.
    // (the flag lives in dynamic shared memory: the kernel has no static shared memory,
    // so the whole 227 KB can be requested dynamically)
    int* s_last = ring + kRing;
    if (threadIdx.x == 0) {
        *s_last = 0;
        if (p.tile_ctr) {
            __threadfence();
            *s_last = atomicAdd(p.exit_ctr, 1u) == gridDim.x - 1;
        }
    }
    __syncthreads();
    if (*s_last) {
        if (chained)  // pair: two counters per block
            for (int b = threadIdx.x; b < (C::PAIR ? 2 : 1) * nblk; b += blockDim.x) p.done1[b] = 0;
        if (p.s1 > 1)
            for (int t = threadIdx.x; t < nblk * p.c1; t += blockDim.x) p.split_cnt[t] = 0;
        if (threadIdx.x == 0) {
            atomicExch(p.tile_ctr, 0u);
            atomicExch(p.exit_ctr, 0u);
        }
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

// INT4 weights: rows x K/2 packed bytes, box = 128 rows x 32 bytes (64 K), no swizzle: the
// dequantisation warps read each row's 32 bytes and write the swizzled bf16 tile.
static bool make_map_int4(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {K / 2, rows};
    cuuint64_t strides[1] = {K / 2};
    cuuint32_t box[2] = {32, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
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

// Launch as clusters of two CTAs (the CTA-pair tile), with programmatic dependent launch.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pair_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                   Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// CTAs of a persistent pair launch: two per cluster that can be resident at once (one
// CTA per SM; a GPC with an odd number of free SMs leaves one idle).
template <class C>
static int pair_grid(size_t smem) {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && cache[dev]) return cache[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, moe_gemm_kernel<C>, &cfg) != cudaSuccess) return 0;
    const int g = std::min(2 * n, 2 * (num_sms() / 2));
    if (dev < 64) cache[dev] = g;
    return g;
}

template <class C>
static cudaError_t launch_cfg(const MoeGemmArgs& a, cudaStream_t stream) {
    // Unused maps of an absent phase point at the present phase's buffers (never read).
    CUtensorMap tmW1, tmX, tmW2, tmH;
    const bool p1 = a.run_gemm1, p2 = a.run_gemm2;
    const void* w1 = p1 ? a.w1 : a.w2;
    const void* x = p1 ? a.x_perm : a.h;
    const void* w2 = p2 ? a.w2 : a.w1;
    const void* hh = p2 ? a.h : a.x_perm;
    const uint64_t k1 = p1 ? a.H : a.I, k2 = p2 ? a.I : a.H;
    const uint64_t r1 = p1 ? (uint64_t)a.G * 2 * a.I : (uint64_t)a.G * a.H;
    const uint64_t r2 = p2 ? (uint64_t)a.G * a.H : (uint64_t)a.G * 2 * a.I;
    auto wmap = [&](CUtensorMap* m, const void* base, uint64_t rows, uint64_t K) {
        return C::INT4 ? make_map_int4(m, base, rows, K) : make_map(m, base, rows, K, C::FP8, 128);
    };
    if (!wmap(&tmW1, w1, r1, k1) || !make_map(&tmX, x, (uint64_t)a.A, k1, C::FP8, C::BOX_ROWS) ||
        !wmap(&tmW2, w2, r2, k2) || !make_map(&tmH, hh, (uint64_t)a.A, k2, C::FP8, C::BOX_ROWS))
        return cudaErrorInvalidValue;
    DevArgs p;
    p.offsets = a.offsets;
    p.G = a.G;
    p.A = (int)a.A;
    p.H = a.H;
    p.I = a.I;
    p.c1 = p1 ? a.I / 128 : 0;
    p.c2 = p2 ? (a.H / 128 + 1) / 2 : 0;
    p.x_scale = a.x_scale;
    p.w1_scale = a.w1_scale;
    p.w2_scale = a.w2_scale;
    p.fp4 = a.fp4 ? 1 : 0;
    p.gate_scale = a.gate_scale;
    p.up_scale = a.up_scale;
    p.alpha = a.alpha;
    p.beta = a.beta;
    p.limit = a.limit;
    p.limits = a.limits;
    p.h = a.h;
    p.h_scale = a.h_scale;
    p.y = a.y;
    p.tile_ctr = a.tile_ctr;
    p.exit_ctr = a.exit_ctr;
    p.done1 = (p1 && p2) ? a.done1 : nullptr;
    p.s1 = p1 ? gemm_split_factor(a.A, a.G, a.H, a.I,
                                  a.fp4 ? MOE_WDTYPE_NVFP4
                                        : (C::INT4 ? MOE_WDTYPE_INT4_G32
                                                   : (C::FP8 ? MOE_WDTYPE_FP8_E4M3_BLOCK128 : MOE_WDTYPE_BF16)))
              : 1;
    p.part = a.part;
    p.split_cnt = a.split_cnt;
    if (p.s1 > 1 && (!p.part || !p.split_cnt)) return cudaErrorInvalidValue;
    p.status = a.status;
    const size_t smem = C::smem_bytes(a.G);
    static std::mutex mu;
    static int max_dyn[64] = {0};  // per device: dynamic shared memory the kernel may request
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    int limit = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 64 || !max_dyn[dev]) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, moe_gemm_kernel<C>);
            if (e != cudaSuccess) return e;
            // The register split must fit what the launch brings, else setmaxnreg.inc would
            // wait for registers that never come: refuse to launch instead.
            if (C::WIDE && fa.numRegs * C::THREADS < 128 * C::REG_LOW + 32 * C::EPI * C::REG_HIGH)
                return cudaErrorInvalidConfiguration;
            limit = kSmemLimit - (int)fa.sharedSizeBytes;
            e = cudaFuncSetAttribute(moe_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
            if (e != cudaSuccess) return e;
            if (dev < 64) max_dyn[dev] = limit;
        } else {
            limit = max_dyn[dev];
        }
    }
    if (smem > (size_t)limit) return cudaErrorInvalidValue;
    if constexpr (C::PAIR) {
        // the occupancy query is taken at the largest dynamic shared memory the kernel may use
        const int grid = pair_grid<C>((size_t)limit);
        if (grid < 2) return cudaErrorInvalidConfiguration;
        return launch_pair_pdl(moe_gemm_kernel<C>, dim3(grid), dim3(C::THREADS), smem, stream, tmW1, tmX, tmW2, tmH,
                               p);
    } else {
        return launch_pdl(moe_gemm_kernel<C>, dim3(num_sms()), dim3(C::THREADS), smem, stream, tmW1, tmX, tmW2, tmH,
                          p);
    }
}

static std::atomic<int> g_fp8_pair{0};   // MOE_OPT_FP8_CTA_PAIR
static std::atomic<int> g_bf16_pair{0};  // MOE_OPT_BF16_CTA_PAIR

int gemm_set_fp8_pair(int enable) { return g_fp8_pair.exchange(enable ? 1 : 0); }
int gemm_set_bf16_pair(int enable) { return g_bf16_pair.exchange(enable ? 1 : 0); }

// A pair needs two GEMM1 completion counters per 256-row block within the workspace's
// block flags (true whenever groups average more than 128 rows).
static bool pair_flags_fit(int64_t A, int G) {
    return 2 * gemm_max_blocks(A, G, 256) + 1 <= gemm_max_blocks(A, G, 16) + 1;
}

int gemm_pick_bn(int64_t A, int G, int wdtype) {
    const double avg = G > 0 ? (double)A / (double)G : 0.0;
    int bn = 16;
    while (bn < 256 && bn < avg) bn <<= 1;  // smallest tile holding an average group
    // FP8 above 128 rows: the 128-token tile, or (when chosen) the CTA pair at "256" (2 x
    // 128 token rows)
    if (wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128 && bn > 128 && (!g_fp8_pair.load() || !pair_flags_fit(A, G)))
        bn = 128;
    if ((wdtype == MOE_WDTYPE_INT4_G32 || wdtype == MOE_WDTYPE_NVFP4) && bn > 64)
        bn = 64;  // 4-bit weights: A tiles share TMEM with the accumulators
    return bn;
}

int64_t gemm_max_blocks(int64_t A, int G, int bn) {
    return (A < G ? A : (int64_t)G) + A / bn;
}

size_t gemm_block_flags_bytes(int64_t A, int G) {
    return sizeof(int) * (size_t)(gemm_max_blocks(A, G, 16) + 1);
}

// Split GEMM1's K range when its tiles cannot fill two waves of the 148 SMs (decode-sized
// batches), keeping at least two K blocks per split.
int gemm_split_factor(int64_t A, int G, int H, int I, int wdtype) {
    constexpr int64_t kTarget = 2 * 148;
    const bool fp8 = wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128;
    const int bn = gemm_pick_bn(A, G, wdtype);
    const int64_t tiles = gemm_max_blocks(A, G, bn) * (I / 128);
    const int kb = H / (fp8 ? 128 : 64);
    if ((fp8 && bn >= 64) || bn >= 256) return 1;  // the kernel variant has no split-K path
    int s = 1;
    while (s < 4 && tiles * s < kTarget && kb >= 4 * s) s *= 2;
    return s;
}

size_t gemm_split_scratch_bytes(int64_t A, int G, int H, int I, int wdtype) {
    const int s = gemm_split_factor(A, G, H, I, wdtype);
    if (s == 1) return 0;
    const int bn = gemm_pick_bn(A, G, wdtype);
    return (size_t)gemm_max_blocks(A, G, bn) * (I / 128) * s * 2 * bn * 128 * sizeof(float);
}

size_t gemm_split_counter_bytes(int64_t A, int G, int H, int I, int wdtype) {
    if (gemm_split_factor(A, G, H, I, wdtype) == 1) return 0;
    const int bn = gemm_pick_bn(A, G, wdtype);
    return (size_t)gemm_max_blocks(A, G, bn) * (I / 128) * sizeof(int);
}

cudaError_t launch_moe_gemm(const MoeGemmArgs& a, cudaStream_t stream) {
    if (a.A == 0 || a.G == 0 || (!a.run_gemm1 && !a.run_gemm2)) return cudaSuccess;
    const int wdtype = a.fp4 ? MOE_WDTYPE_NVFP4
                             : (a.int4 ? MOE_WDTYPE_INT4_G32 : (a.fp8 ? MOE_WDTYPE_FP8_E4M3_BLOCK128 : MOE_WDTYPE_BF16));
    const int bn = gemm_pick_bn(a.A, a.G, wdtype);
    if (a.int4) {
        switch (bn) {
            case 16: return launch_cfg<Cfg<16, false, true>>(a, stream);
            case 32: return launch_cfg<Cfg<32, false, true>>(a, stream);
            case 64: return launch_cfg<Cfg<64, false, true>>(a, stream);
            default: return cudaErrorInvalidValue;
        }
    }
    if (a.fp8) {
        switch (bn) {
            case 16: return launch_cfg<Cfg<16, true>>(a, stream);
            case 32: return launch_cfg<Cfg<32, true>>(a, stream);
            case 64: return launch_cfg<Cfg<64, true>>(a, stream);
            case 128: return launch_cfg<Cfg<128, true>>(a, stream);
            case 256: return launch_cfg<Cfg<128, true, false, true>>(a, stream);  // CTA pair
            default: return cudaErrorInvalidValue;
        }
    }
    switch (bn) {
        case 16: return launch_cfg<Cfg<16, false>>(a, stream);
        case 32: return launch_cfg<Cfg<32, false>>(a, stream);
        case 64: return launch_cfg<Cfg<64, false>>(a, stream);
        case 128: return launch_cfg<Cfg<128, false>>(a, stream);
        case 256:  // 256-row token blocks: one CTA, or (when chosen) the token-major CTA pair
            if (g_bf16_pair.load() && pair_flags_fit(a.A, a.G)) return launch_cfg<Cfg<128, false, false, true>>(a, stream);
            return launch_cfg<Cfg<256, false>>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
