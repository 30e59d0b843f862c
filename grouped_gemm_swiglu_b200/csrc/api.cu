// api.cu -- the C ABI declared in include/moe_b200.h: argument checks, workspace
// layout and the launch sequence of the expert layer. Host code only.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "internal.h"
#include "status.cuh"

using namespace moe;

namespace {

constexpr int kMaxE = 1024;
constexpr int kMaxSlots = 32;  // k + n_sink and k + n_shared share one warp

inline size_t al256(size_t b) { return (b + 255) & ~size_t(255); }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_dims(const moe_dims* d) {
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->H <= 0 || d->I <= 0 || d->H % 128 || d->I % 128) return MOE_ERR_INVALID_ARG;
    if (d->E < 1 || d->E > kMaxE) return MOE_ERR_INVALID_ARG;
    if (d->k < 1 || d->k > d->E || d->k > kMaxSlots) return MOE_ERR_INVALID_ARG;
    if (d->n_sink < 0 || d->k + d->n_sink > kMaxSlots) return MOE_ERR_INVALID_ARG;
    if (d->n_shared < 0 || d->k + d->n_shared > kMaxSlots) return MOE_ERR_INVALID_ARG;
    if (d->score != MOE_SCORE_SOFTMAX && d->score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (d->wdtype != MOE_WDTYPE_BF16 && d->wdtype != MOE_WDTYPE_FP8_E4M3_BLOCK128 && d->wdtype != MOE_WDTYPE_INT4_G32 &&
        d->wdtype != MOE_WDTYPE_NVFP4)
        return MOE_ERR_INVALID_ARG;
    if (d->n_sink > 0 && d->score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (d->n_sink > 0 && d->n_shared > 0 && d->n_shared != d->n_sink) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(d->alpha) || !std::isfinite(d->beta) || !std::isfinite(d->route_scale))
        return MOE_ERR_INVALID_ARG;
    if (!(d->limit > 0.f)) return MOE_ERR_INVALID_ARG;  // rejects NaN too; +inf = no clamp
    const int64_t A = (int64_t)d->T * (d->k + d->n_shared);
    if (A > INT32_MAX / 2) return MOE_ERR_INVALID_ARG;
    const int64_t G = (int64_t)d->E + d->n_shared;
    if (G * 2 * d->I > INT32_MAX / 2 || G * d->H > INT32_MAX / 2) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

int check_arch() {
    static int verdict[64] = {0};  // 0 unknown, 1 ok, -1 wrong arch
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev >= 0 && dev < 64 && verdict[dev]) return verdict[dev] > 0 ? MOE_OK : MOE_ERR_ARCH;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MOE_ERR_CUDA;
    const int ok = (major == 10) ? 1 : -1;
    if (dev >= 0 && dev < 64) verdict[dev] = ok;
    return ok > 0 ? MOE_OK : MOE_ERR_ARCH;
}

int64_t rows_A(const moe_dims* d) { return (int64_t)d->T * (d->k + d->n_shared); }
int groups(const moe_dims* d) { return d->E + d->n_shared; }
size_t act_elt(const moe_dims* d) { return d->wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128 ? 1 : 2; }
bool is_fp8(const moe_dims* d) { return d->wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128; }
// 4-bit weights (INT4 group-32 or NVFP4): packed bytes, per-row scales read one 32-bit
// word per 64-deep K step, bf16 activations
bool is_int4(const moe_dims* d) { return d->wdtype == MOE_WDTYPE_INT4_G32 || d->wdtype == MOE_WDTYPE_NVFP4; }

// Sub-buffers of a workspace, as byte offsets from its start.
struct Layout {
    size_t ids = 0, w = 0, sw = 0, offsets = 0, perm = 0, inv = 0, xperm = 0, xscale = 0, h = 0, hscale = 0,
           flags = 0, splitcnt = 0, part = 0, pscratch = 0, y = 0, logits = 0, total = 0;
};

Layout layout(const moe_dims* d, int kind) {
    Layout L;
    const size_t T = d->T, k = d->k, A = rows_A(d), H = d->H, I = d->I, G = groups(d);
    size_t off = kWsHeader;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += al256(bytes);
        return at;
    };
    if (kind == MOE_WS_FORWARD) {
        L.ids = take(T * k * 4);
        L.w = take(T * k * 4);
        L.sw = take(T * (size_t)d->n_sink * 4);
        L.offsets = take((G + 1) * 4);
        L.perm = take(A * 4);
        L.inv = take(T * k * 4);
        L.xperm = take(A * H * act_elt(d));
        L.xscale = take(is_fp8(d) ? (H / 128) * A * 4 : 0);
        L.h = take(A * I * act_elt(d));
        L.hscale = take(is_fp8(d) ? (I / 128) * A * 4 : 0);
    }
    // block flags and split-K counters are adjacent so one clear covers both
    if (kind == MOE_WS_FORWARD || kind == MOE_WS_EXPERTS) L.flags = take(gemm_block_flags_bytes(A, G));
    if (kind == MOE_WS_FORWARD || kind == MOE_WS_EXPERTS || kind == MOE_WS_GEMM1) {
        L.splitcnt = take(gemm_split_counter_bytes(A, G, H, I, d->wdtype));
        L.part = take(gemm_split_scratch_bytes(A, G, H, I, d->wdtype));
    }
    if (kind == MOE_WS_FORWARD || kind == MOE_WS_PERMUTE) L.pscratch = take(permute_scratch_bytes(d->T, d->k, d->E));
    if (kind == MOE_WS_FORWARD || kind == MOE_WS_GEMM2_COMBINE) L.y = take(A * H * 2);
    if (kind == MOE_WS_GATE_ROUTE) L.logits = take(T * (size_t)(d->E + d->n_sink) * 4);
    L.total = off;
    return L;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int check_ws(const void* ws, size_t ws_bytes, const moe_dims* d, int kind) {
    if (!ws || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
    if (ws_bytes < layout(d, kind).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

template <class P>
P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

// The individual steps, after every check has passed.
int do_route(const float* logits, const float* bias, const moe_dims* d, int32_t* ids, float* w, float* sw,
             uint32_t* packed, cudaStream_t s) {
    return cuda_status(launch_router(logits, bias, d->T, d->E, d->n_sink, d->k, d->score, d->route_scale, ids, w, sw,
                                     packed, s));
}

// A correction bias is defined for the sigmoid ranking only.
int check_bias(const moe_dims* d, const float* bias) {
    return (bias && d->score != MOE_SCORE_SIGMOID) ? MOE_ERR_UNSUPPORTED : MOE_OK;
}

int do_permute(const int32_t* ids, const void* x, const moe_dims* d, int32_t* offsets, int32_t* perm, int32_t* inv,
               void* xperm, float* xscale, void* scratch, int* status, cudaStream_t s, int* zero = nullptr,
               size_t zero_words = 0) {
    unsigned int* counter = reinterpret_cast<unsigned int*>(reinterpret_cast<char*>(status) + kWsCounterOffset);
    return cuda_status(launch_permute(ids, x, d->T, d->H, d->k, d->E, d->n_shared, is_fp8(d), offsets, perm, inv,
                                      xperm, xscale, scratch, counter, status, s, zero, zero_words));
}

MoeGemmArgs gemm_args(const moe_dims* d, const int32_t* offsets, int* status) {
    MoeGemmArgs a{};
    a.offsets = offsets;
    a.G = groups(d);
    a.A = rows_A(d);
    a.H = d->H;
    a.I = d->I;
    a.fp8 = is_fp8(d);
    a.int4 = is_int4(d);
    a.fp4 = d->wdtype == MOE_WDTYPE_NVFP4;
    a.alpha = d->alpha;
    a.beta = d->beta;
    a.limit = d->limit;
    a.status = status;
    a.tile_ctr = reinterpret_cast<unsigned int*>(reinterpret_cast<char*>(status) + kWsTileCtrOffset);
    a.exit_ctr = a.tile_ctr + 1;
    return a;
}

int do_gemm1(const void* xperm, const float* xscale, const int32_t* offsets, const void* w1, const void* w1s,
             const float* gs, const float* us, const float* limits, const moe_dims* d, void* h, float* hs, void* ws,
             cudaStream_t s) {
    const Layout L = layout(d, MOE_WS_GEMM1);
    MoeGemmArgs a = gemm_args(d, offsets, at<int>(ws, 0));
    a.split_cnt = L.part ? at<int>(ws, L.splitcnt) : nullptr;
    a.part = L.part ? at<float>(ws, L.part) : nullptr;
    a.run_gemm1 = true;
    a.x_perm = xperm;
    a.x_scale = xscale;
    a.w1 = w1;
    a.w1_scale = w1s;
    a.gate_scale = gs;
    a.up_scale = us;
    a.limits = limits;
    a.h = h;
    a.h_scale = hs;
    return cuda_status(launch_moe_gemm(a, s));
}

int do_combine(const void* y, const int32_t* offsets, const int32_t* inv, const float* topk_w,
               const float* shared_w, const moe_dims* d, void* out, int* status, cudaStream_t s) {
    return cuda_status(launch_combine(y, offsets, inv, topk_w, shared_w, d->T, d->H, d->k, d->E, d->n_shared,
                                      d->n_sink, rows_A(d), out, status, s));
}

int do_gemm2_combine(const void* h, const float* hs, const int32_t* offsets, const int32_t* inv, const float* topk_w,
                     const float* shared_w, const void* w2, const void* w2s, const moe_dims* d, void* out, void* y,
                     int* status, cudaStream_t s) {
    MoeGemmArgs a = gemm_args(d, offsets, status);
    a.run_gemm2 = true;
    a.h = const_cast<void*>(h);
    a.h_scale = const_cast<float*>(hs);
    a.w2 = w2;
    a.w2_scale = w2s;
    a.y = y;
    int rc = cuda_status(launch_moe_gemm(a, s));
    if (rc != MOE_OK) return rc;
    return do_combine(y, offsets, inv, topk_w, shared_w, d, out, status, s);
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

int moe_set_option(int option, int value) {
    if (option == MOE_OPT_FP8_CTA_PAIR && (value == 0 || value == 1)) return gemm_set_fp8_pair(value);
    if (option == MOE_OPT_BF16_CTA_PAIR && (value == 0 || value == 1)) return gemm_set_bf16_pair(value);
    return MOE_ERR_INVALID_ARG;
}

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported combination";
        case MOE_ERR_ARCH: return "device is not compute capability 10.x (sm_100a)";
        case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MOE_ERR_EXPERT_ID: return "routing id outside [0, E) or repeated within a token";
        case MOE_ERR_TIMEOUT: return "a pipeline wait exceeded its time limit";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        default: return "unknown status";
    }
}

int moe_workspace_size(const moe_dims* dims, int kind, size_t* bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    int rc = check_dims(dims);
    if (rc != MOE_OK) return rc;
    if (kind < MOE_WS_PERMUTE || kind > MOE_WS_GATE_ROUTE) return MOE_ERR_INVALID_ARG;
    *bytes = layout(dims, kind).total;
    return MOE_OK;
}

int moe_read_status(const void* ws, int32_t* status, void* stream) {
    if (!ws || !status) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    *status = v;
    return MOE_OK;
}

int moe_clear_status(void* ws, void* stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, kWsHeader, static_cast<cudaStream_t>(stream)));
}

int moe_route_topk(const float* logits, const moe_dims* d, const float* bias, int32_t* topk_ids, float* topk_w,
                   float* shared_w, uint32_t* packed, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T > 0 && (!logits || !topk_ids || !topk_w)) return MOE_ERR_INVALID_ARG;
    if (d->T > 0 && (d->n_sink > 0) != (shared_w != nullptr)) return MOE_ERR_INVALID_ARG;
    if ((rc = check_bias(d, bias)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    return do_route(logits, bias, d, topk_ids, topk_w, shared_w, packed, static_cast<cudaStream_t>(stream));
}

int moe_gate_route(const void* x, const void* w_gate, const moe_dims* d, const float* bias, float* logits,
                   int32_t* topk_ids, float* topk_w, float* shared_w, uint32_t* packed, void* ws, size_t ws_bytes,
                   void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T > 0) {
        if (!x || !w_gate || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
        if ((d->n_sink > 0) != (shared_w != nullptr)) return MOE_ERR_INVALID_ARG;
        if (!aligned(x, 16) || !aligned(w_gate, 16)) return MOE_ERR_INVALID_ARG;
    }
    if ((rc = check_bias(d, bias)) != MOE_OK) return rc;
    if (d->T > kGateMaxTokens) return MOE_ERR_UNSUPPORTED;
    if ((rc = check_ws(ws, ws_bytes, d, MOE_WS_GATE_ROUTE)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    const Layout L = layout(d, MOE_WS_GATE_ROUTE);
    float* lg = logits ? logits : at<float>(ws, L.logits);
    unsigned int* counter = at<unsigned int>(ws, kWsGateCtrOffset);
    return cuda_status(launch_gate_route(x, w_gate, bias, d->T, d->H, d->E, d->n_sink, d->k, d->score,
                                         d->route_scale, lg, topk_ids, topk_w, shared_w, packed, counter,
                                         static_cast<cudaStream_t>(stream)));
}

int moe_permute(const int32_t* topk_ids, const void* x, const moe_dims* d, int32_t* offsets, int32_t* perm,
                int32_t* inv_perm, void* x_perm, float* x_scale, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (!offsets) return MOE_ERR_INVALID_ARG;
    if (d->T > 0) {
        if (!topk_ids || !x || !perm || !inv_perm || !x_perm) return MOE_ERR_INVALID_ARG;
        if (is_fp8(d) && !x_scale) return MOE_ERR_INVALID_ARG;
        if (!aligned(x, 16) || !aligned(x_perm, 16)) return MOE_ERR_INVALID_ARG;
    }
    if ((rc = check_ws(ws, ws_bytes, d, MOE_WS_PERMUTE)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    const Layout L = layout(d, MOE_WS_PERMUTE);
    return do_permute(topk_ids, x, d, offsets, perm, inv_perm, x_perm, x_scale, at<void>(ws, L.pscratch),
                      at<int>(ws, 0), static_cast<cudaStream_t>(stream));
}

int moe_gemm1_swiglu(const void* x_perm, const float* x_scale, const int32_t* offsets, const void* w1,
                     const void* w1_scale, const float* gate_scale, const float* up_scale, const float* limits,
                     const moe_dims* d, void* h, float* h_scale, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T > 0) {
        if (!x_perm || !offsets || !w1 || !h) return MOE_ERR_INVALID_ARG;
        if (is_fp8(d) && (!x_scale || !w1_scale || !h_scale)) return MOE_ERR_INVALID_ARG;
        if (is_int4(d) && (!w1_scale || !aligned(w1_scale, 4))) return MOE_ERR_INVALID_ARG;
        if (!aligned(x_perm, 16) || !aligned(w1, 16) || !aligned(h, 16)) return MOE_ERR_INVALID_ARG;
    }
    if ((rc = check_ws(ws, ws_bytes, d, MOE_WS_GEMM1)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    return do_gemm1(x_perm, x_scale, offsets, w1, w1_scale, gate_scale, up_scale, limits, d, h, h_scale, ws,
                    static_cast<cudaStream_t>(stream));
}

int moe_gemm2_combine(const void* h, const float* h_scale, const int32_t* offsets, const int32_t* inv_perm,
                      const float* topk_w, const float* shared_w, const void* w2, const void* w2_scale,
                      const moe_dims* d, void* out, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T > 0) {
        if (!h || !offsets || !inv_perm || !topk_w || !w2 || !out) return MOE_ERR_INVALID_ARG;
        if ((d->n_sink > 0) != (shared_w != nullptr)) return MOE_ERR_INVALID_ARG;
        if (is_fp8(d) && (!h_scale || !w2_scale)) return MOE_ERR_INVALID_ARG;
        if (is_int4(d) && (!w2_scale || !aligned(w2_scale, 4))) return MOE_ERR_INVALID_ARG;
        if (!aligned(h, 16) || !aligned(w2, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
    }
    if ((rc = check_ws(ws, ws_bytes, d, MOE_WS_GEMM2_COMBINE)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    const Layout L = layout(d, MOE_WS_GEMM2_COMBINE);
    return do_gemm2_combine(h, h_scale, offsets, inv_perm, topk_w, shared_w, w2, w2_scale, d, out, at<void>(ws, L.y),
                            at<int>(ws, 0), static_cast<cudaStream_t>(stream));
}

int moe_experts(const void* x_perm, const float* x_scale, const int32_t* offsets, const void* w1,
                const void* w1_scale, const float* gate_scale, const float* up_scale, const float* limits,
                const void* w2, const void* w2_scale, const moe_dims* d, void* h, float* h_scale, void* y, void* ws,
                size_t ws_bytes, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T > 0) {
        if (!x_perm || !offsets || !w1 || !w2 || !h || !y) return MOE_ERR_INVALID_ARG;
        if (is_fp8(d) && (!x_scale || !w1_scale || !w2_scale || !h_scale)) return MOE_ERR_INVALID_ARG;
        if (is_int4(d) && (!w1_scale || !w2_scale || !aligned(w1_scale, 4) || !aligned(w2_scale, 4)))
            return MOE_ERR_INVALID_ARG;
        if (!aligned(x_perm, 16) || !aligned(w1, 16) || !aligned(w2, 16) || !aligned(h, 16) || !aligned(y, 16))
            return MOE_ERR_INVALID_ARG;
    }
    if ((rc = check_ws(ws, ws_bytes, d, MOE_WS_EXPERTS)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    const Layout L = layout(d, MOE_WS_EXPERTS);
    MoeGemmArgs a = gemm_args(d, offsets, at<int>(ws, 0));
    a.run_gemm1 = a.run_gemm2 = true;
    a.x_perm = x_perm;
    a.x_scale = x_scale;
    a.w1 = w1;
    a.w1_scale = w1_scale;
    a.gate_scale = gate_scale;
    a.up_scale = up_scale;
    a.limits = limits;
    a.h = h;
    a.h_scale = h_scale;
    a.w2 = w2;
    a.w2_scale = w2_scale;
    a.y = y;
    a.done1 = at<int>(ws, L.flags);
    a.split_cnt = L.part ? at<int>(ws, L.splitcnt) : nullptr;
    a.part = L.part ? at<float>(ws, L.part) : nullptr;
    return cuda_status(launch_moe_gemm(a, static_cast<cudaStream_t>(stream)));
}

int moe_combine(const void* y, const int32_t* offsets, const int32_t* inv_perm, const float* topk_w,
                const float* shared_w, const moe_dims* d, void* out, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T > 0) {
        if (!y || !offsets || !inv_perm || !topk_w || !out) return MOE_ERR_INVALID_ARG;
        if ((d->n_sink > 0) != (shared_w != nullptr)) return MOE_ERR_INVALID_ARG;
        if (!aligned(y, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
    }
    if ((rc = check_ws(ws, ws_bytes, d, MOE_WS_COMBINE)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    return do_combine(y, offsets, inv_perm, topk_w, shared_w, d, out, at<int>(ws, 0),
                      static_cast<cudaStream_t>(stream));
}

int moe_forward(const float* logits, const float* bias, const void* x, const void* w1, const void* w1_scale,
                const float* gate_scale, const float* up_scale, const float* limits, const void* w2,
                const void* w2_scale, const moe_dims* d, void* out, int32_t* topk_ids, float* topk_w,
                float* shared_w, uint32_t* packed, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if ((rc = check_bias(d, bias)) != MOE_OK) return rc;
    if (d->T > 0) {
        if (!logits || !x || !w1 || !w2 || !out) return MOE_ERR_INVALID_ARG;
        if (is_fp8(d) && (!w1_scale || !w2_scale)) return MOE_ERR_INVALID_ARG;
        if (is_int4(d) && (!w1_scale || !w2_scale || !aligned(w1_scale, 4) || !aligned(w2_scale, 4)))
            return MOE_ERR_INVALID_ARG;
        if (!aligned(x, 16) || !aligned(w1, 16) || !aligned(w2, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
        if (shared_w && d->n_sink == 0) return MOE_ERR_INVALID_ARG;
    }
    if ((rc = check_ws(ws, ws_bytes, d, MOE_WS_FORWARD)) != MOE_OK) return rc;
    if ((rc = check_arch()) != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Layout L = layout(d, MOE_WS_FORWARD);
    int* status = at<int>(ws, 0);
    int32_t* ids = topk_ids ? topk_ids : at<int32_t>(ws, L.ids);
    float* w = topk_w ? topk_w : at<float>(ws, L.w);
    float* sw = d->n_sink > 0 ? (shared_w ? shared_w : at<float>(ws, L.sw)) : nullptr;
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    if (d->T == 0) return cuda_status(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (groups(d) + 1), s));
    float* xscale = is_fp8(d) ? at<float>(ws, L.xscale) : nullptr;
    float* hscale = is_fp8(d) ? at<float>(ws, L.hscale) : nullptr;
    if ((rc = do_route(logits, bias, d, ids, w, sw, packed, s)) != MOE_OK) return rc;
    // The counting kernel also clears the GEMM's per-block completion flags.
    int* flags = at<int>(ws, L.flags);
    const size_t clear_words =
        (L.splitcnt + gemm_split_counter_bytes(rows_A(d), groups(d), d->H, d->I, d->wdtype) - L.flags) / sizeof(int);
    if ((rc = do_permute(ids, x, d, offsets, at<int32_t>(ws, L.perm), at<int32_t>(ws, L.inv), at<void>(ws, L.xperm),
                         xscale, at<void>(ws, L.pscratch), status, s, flags, clear_words)) != MOE_OK)
        return rc;
    // GEMM1 + SwiGLU and GEMM2 in one persistent launch, then the combine.
    MoeGemmArgs a = gemm_args(d, offsets, status);
    a.run_gemm1 = a.run_gemm2 = true;
    a.x_perm = at<void>(ws, L.xperm);
    a.x_scale = xscale;
    a.w1 = w1;
    a.w1_scale = w1_scale;
    a.gate_scale = gate_scale;
    a.up_scale = up_scale;
    a.limits = limits;
    a.h = at<void>(ws, L.h);
    a.h_scale = hscale;
    a.w2 = w2;
    a.w2_scale = w2_scale;
    a.y = at<void>(ws, L.y);
    a.done1 = flags;
    a.split_cnt = L.part ? at<int>(ws, L.splitcnt) : nullptr;
    a.part = L.part ? at<float>(ws, L.part) : nullptr;
    if ((rc = cuda_status(launch_moe_gemm(a, s))) != MOE_OK) return rc;
    return do_combine(at<void>(ws, L.y), offsets, at<int32_t>(ws, L.inv), w, sw, d, out, status, s);
}

int moe_ep_row_ids(const int32_t* offsets, const moe_dims* d, int32_t* row_ids, void* stream) {
    int rc = check_dims(d);
    if (rc != MOE_OK) return rc;
    if (d->T > 0 && (!offsets || !row_ids)) return MOE_ERR_INVALID_ARG;
    if ((rc = check_arch()) != MOE_OK) return rc;
    if (d->T == 0) return MOE_OK;
    return cuda_status(launch_ep_row_ids(offsets, groups(d), (int)rows_A(d), row_ids, static_cast<cudaStream_t>(stream)));
}

int moe_ep_rebase(const int32_t* ids, int64_t n, int32_t E, int32_t n_shared, int32_t local_offset, int32_t n_local,
                  int32_t* out, void* stream) {
    if (n < 0 || n > INT32_MAX || E < 1 || E > kMaxE || n_shared < 0 || n_shared > kMaxSlots || n_local < 1 ||
        local_offset < 0 || (int64_t)local_offset + n_local > E)
        return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!ids || !out)) return MOE_ERR_INVALID_ARG;
    int rc = check_arch();
    if (rc != MOE_OK) return rc;
    return cuda_status(
        launch_ep_rebase(ids, n, E, n_shared, local_offset, n_local, out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
