// ep.cu -- the two index steps of expert parallelism (experts partitioned over ranks).
//
// Routing ids are global expert ids; an expert-parallel rank holds the weights of its
// local experts only, so ids that reach it are rebased by its local expert offset and
// checked against its local expert count, and an id outside that range is an error,
// never an index into another rank's tables (xorl-wheels "FlashInfer 0.6.18
// SM100a+SM103a MoE-LoRA AOT", "Changes": expert-parallel lookups are rank-local).
//
//   ep_row_ids_kernel: the weight group of every permuted row, read off the group
//     offsets (rows of group g are offsets[g] .. offsets[g+1]-1): what travels with a
//     row to the rank that owns its expert.
//   ep_rebase_kernel: global group id -> local group id on this rank (routed experts
//     [off, off + n_local) -> [0, n_local); shared experts, replicated on every rank,
//     E + s -> n_local + s); anything else -> -1, which the local permutation reports
//     as MOE_ERR_EXPERT_ID and drops.
#include "internal.h"

namespace moe {

constexpr int kEpThreads = 256;

// One thread per row; a binary search over the G + 1 offsets (clamped into [0, A], so a
// bad offsets array cannot make the search leave it).
__global__ void __launch_bounds__(kEpThreads) ep_row_ids_kernel(const int32_t* __restrict__ offsets, int G, int A,
                                                               int32_t* __restrict__ row_ids) {
    const int r = blockIdx.x * kEpThreads + threadIdx.x;
    if (r >= A) return;
    int lo = 0, hi = G;  // find the last g in [0, G) with offsets[g] <= r
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (min(max(__ldg(offsets + mid), 0), A) <= r) lo = mid;
        else hi = mid;
    }
    row_ids[r] = lo;
}

__global__ void __launch_bounds__(kEpThreads) ep_rebase_kernel(const int32_t* __restrict__ ids, int64_t n, int E,
                                                              int n_shared, int local_offset, int n_local,
                                                              int32_t* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * kEpThreads + threadIdx.x;
    if (i >= n) return;
    const int g = __ldg(ids + i);
    int l = -1;
    if (g >= local_offset && g < local_offset + n_local) l = g - local_offset;
    else if (g >= E && g < E + n_shared) l = n_local + (g - E);
    out[i] = l;
}

cudaError_t launch_ep_row_ids(const int32_t* offsets, int G, int A, int32_t* row_ids, cudaStream_t stream) {
    if (A <= 0) return cudaSuccess;
    ep_row_ids_kernel<<<(A + kEpThreads - 1) / kEpThreads, kEpThreads, 0, stream>>>(offsets, G, A, row_ids);
    return cudaGetLastError();
}

cudaError_t launch_ep_rebase(const int32_t* ids, int64_t n, int E, int n_shared, int local_offset, int n_local,
                             int32_t* out, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = (n + kEpThreads - 1) / kEpThreads;
    ep_rebase_kernel<<<(unsigned)blocks, kEpThreads, 0, stream>>>(ids, n, E, n_shared, local_offset, n_local, out);
    return cudaGetLastError();
}

}  // namespace moe
