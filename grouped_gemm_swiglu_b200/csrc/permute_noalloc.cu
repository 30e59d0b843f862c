// permute_noalloc.cu -- moe_permute_noalloc: the expert permutation without a
// caller-provided workspace, for callers that cannot allocate device memory.
//
// Who needs it: code whose device memory is planned entirely ahead of time by someone
// else -- a serving engine or framework that reserves the whole GPU up front and hands
// an operator only its input and output buffers, a plugin interface with a fixed
// signature and no workspace query, or a latency-critical path where a cudaMalloc (and
// the device-wide synchronisation it can cause) is not acceptable. Such a caller can
// still pass the inputs and outputs it owns; the scratch the permutation needs (per
// chunk counts and per slot ranks) comes from a fixed array compiled into this library.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// kNoAllocScratchBytes of it until the process exits, and every call on that GPU shares
// it. Host code must not pass the array's name to a kernel (on the host it is only a
// stand-in symbol); the device address is fetched with cudaGetSymbolAddress, with the
// device current: on every call that is not being captured into a CUDA graph (so a
// context created after cudaDeviceReset, or another context current on the device, gets
// its own address), and from the last such lookup on that device while the stream is
// capturing.
#include <mutex>

#include "internal.h"
#include "status.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB per device

static __device__ __align__(256) unsigned char g_permute_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the static scratch in the current context. Looked up on each call
// (a cheap host call once the module is loaded), except while `stream` is capturing,
// where the address of the last uncaptured call on this device is reused.
int scratch_address(cudaStream_t stream, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (cap == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    } else if (!g_scratch_addr[dev]) {
        return MOE_ERR_UNSUPPORTED;  // the look-up itself may not run under capture
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

bool valid_dims(const moe_dims* d) {
    if (!d) return false;
    if (d->T < 0 || d->H <= 0 || d->I <= 0 || d->H % 128 || d->I % 128) return false;
    if (d->E < 1 || d->E > 1024 || d->k < 1 || d->k > d->E || d->k > 32) return false;
    if (d->n_shared < 0 || d->k + d->n_shared > 32) return false;
    if (d->wdtype != MOE_WDTYPE_BF16 && d->wdtype != MOE_WDTYPE_FP8_E4M3_BLOCK128 && d->wdtype != MOE_WDTYPE_INT4_G32 &&
        d->wdtype != MOE_WDTYPE_NVFP4)
        return false;  // 4-bit weights take bf16 activations: a bf16 permutation
    return (int64_t)d->T * (d->k + d->n_shared) <= INT32_MAX / 2;
}

}  // namespace

extern "C" int moe_permute_noalloc(const int32_t* topk_ids, const void* x, const moe_dims* d, int32_t* offsets,
                                   int32_t* perm, int32_t* inv_perm, void* x_perm, float* x_scale, int32_t* status,
                                   void* stream) {
    if (!valid_dims(d) || !offsets) return MOE_ERR_INVALID_ARG;
    const bool fp8 = d->wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128;
    if (d->T > 0) {
        if (!topk_ids || !x || !perm || !inv_perm || !x_perm || (fp8 && !x_scale)) return MOE_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(x_perm) % 16)
            return MOE_ERR_INVALID_ARG;
    }
    // Sizes beyond the static scratch (after its 256-byte counter header) are refused up front.
    if (moe::permute_scratch_bytes(d->T, d->k, d->E) > kNoAllocScratchBytes - 256) return MOE_ERR_WORKSPACE;
    int major = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (major != 10) return MOE_ERR_ARCH;
    void* scratch = nullptr;
    int rc = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (rc != MOE_OK) return rc;
    // The first word of the array counts finished CTAs of the counting kernel and must be
    // zero when the counting kernel starts. A clean call leaves it at zero, but two calls
    // that overlapped can leave it anywhere, so every call clears it on its stream first
    // (a memset, no allocation): one race then corrupts only the calls that raced. The
    // rest of the array is written before it is read. The status word is the caller's.
    unsigned int* counter = static_cast<unsigned int*>(scratch);
    if (d->T > 0 && cudaMemsetAsync(counter, 0, sizeof(unsigned int), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    cudaError_t e = moe::launch_permute(topk_ids, x, d->T, d->H, d->k, d->E, d->n_shared, fp8, offsets, perm,
                                        inv_perm, x_perm, x_scale, static_cast<char*>(scratch) + 256, counter, status,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
