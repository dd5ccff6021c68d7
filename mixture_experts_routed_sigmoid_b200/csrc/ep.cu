// Expert-parallel dispatch and combine kernels.
//
// With G ranks each owning n_experts / G consecutive experts, the routed
// layer becomes: sort this rank's routed rows by owner rank, pack their input
// rows, exchange them (all-to-all), run the owner's experts on the rows it
// received, send the unweighted per-slot rows back, and combine them on the
// token's home rank.  The combine is the routed FFN's own definition
// [cortiq-engine 0.7.7, src/mimo_moe.rs tests::exact_moe: y = sum_j w_j *
// down_e(silu(gate_e x) * up_e x); hf2q qwen35/dense_ffn_arena.rs MoeFfnArena:
// the weighted reduce over the top-k slots], with the weight applied to each
// returned row (one f32 multiply) and the slots added in slot order, so the
// bits equal those of the single-rank layer whenever the owners run the same
// kernels on each row.
//
// Kernels here:
//   ep_owner_kernel    owner rank of every routed row (and the id check)
//   ep_pack_kernel     send-ordered input rows and local expert ids
//   ep_combine_kernel  y[t] = sum_j fl(w[t,j] * d_back[pos(t,j)]), slot order
// The owner-sorted order itself is the expert map over owner ranks.
#include "device_common.cuh"
#include "launch.h"

namespace moe {

__global__ void __launch_bounds__(256) ep_owner_kernel(const int* __restrict__ ids, long long rows,
                                                       int n_experts, int experts_per_rank,
                                                       int* __restrict__ owner,
                                                       int* __restrict__ status) {
    for (long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; r < rows;
         r += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int e = ids[r];
        if (e < 0 || e >= n_experts) {
            set_status(status, kDevBadId);
            owner[r] = 0;  // keeps the map in range; the status stops every later kernel
        } else {
            owner[r] = e / experts_per_rank;
        }
    }
}

// One warp per send position p: routed row r = perm[p], its input row
// (x[t] shared per token, x[t, j] slotted) copied with 16-byte loads.
__global__ void __launch_bounds__(256) ep_pack_kernel(
    const uint4* __restrict__ x, const int* __restrict__ ids, const int* __restrict__ perm,
    long long rows, int row_vec, int top_k, int layout, int experts_per_rank,
    uint4* __restrict__ send_x, int* __restrict__ send_expert, const int* __restrict__ status) {
    if (*status != 0) return;
    const int lane = threadIdx.x & 31;
    const long long warp0 = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
    const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long p = warp0; p < rows; p += n_warps) {
        const int r = perm[p];
        if (r < 0 || r >= rows) continue;  // never reached with a valid map
        const long long src = layout ? r : r / top_k;
        const uint4* s = x + src * row_vec;
        uint4* d = send_x + p * row_vec;
        for (int i = lane; i < row_vec; i += 32) d[i] = __ldg(s + i);
        if (lane == 0) {
            const int e = ids[r];
            send_expert[p] = e - (e / experts_per_rank) * experts_per_rank;
        }
    }
}

// y[t, :] = sum_{j < top_k} fl(w[t, j] * d_back[inv[t*top_k + j], :]), added in
// slot order with the first product initialising the sum; explicit
// round-to-nearest multiply and add keep the compiler from fusing them.
__global__ void __launch_bounds__(256) ep_combine_kernel(const float4* __restrict__ d_back,
                                                         const int* __restrict__ inv,
                                                         const float* __restrict__ weights,
                                                         float4* __restrict__ y, long long m,
                                                         int hidden4, int top_k,
                                                         long long rows,
                                                         const int* __restrict__ status) {
    if (*status != 0) return;
    const long long total = m * hidden4;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long t = i / hidden4;
        const int h = static_cast<int>(i - t * hidden4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < top_k; ++j) {
            const long long r = t * top_k + j;
            long long p = inv[r];
            if (p < 0 || p >= rows) p = 0;  // never reached with a valid map
            const float w = weights[r];
            const float4 v = __ldcs(d_back + p * hidden4 + h);
            const float4 q = make_float4(__fmul_rn(w, v.x), __fmul_rn(w, v.y), __fmul_rn(w, v.z),
                                         __fmul_rn(w, v.w));
            if (j == 0) {
                acc = q;
            } else {
                acc.x = __fadd_rn(acc.x, q.x);
                acc.y = __fadd_rn(acc.y, q.y);
                acc.z = __fadd_rn(acc.z, q.z);
                acc.w = __fadd_rn(acc.w, q.w);
            }
        }
        __stcs(y + i, acc);
    }
}

namespace {
int device_sms() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}
}  // namespace

cudaError_t launch_ep_owner(const int* ids, long long rows, int n_experts, int experts_per_rank,
                            int* owner, int* status, cudaStream_t stream) {
    long long blocks = (rows + 255) / 256;
    const long long cap = 4LL * device_sms();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    ep_owner_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(ids, rows, n_experts,
                                                                  experts_per_rank, owner, status);
    return cudaGetLastError();
}

cudaError_t launch_ep_pack(const __nv_bfloat16* x, const int* ids, const int* perm, long long rows,
                           int hidden, int top_k, int layout, int experts_per_rank,
                           __nv_bfloat16* send_x, int* send_expert, const int* status,
                           cudaStream_t stream) {
    long long blocks = (rows + 7) / 8;  // 8 warps per block, one row per warp
    const long long cap = 8LL * device_sms();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    ep_pack_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), ids, perm, rows, hidden / 8, top_k, layout,
        experts_per_rank, reinterpret_cast<uint4*>(send_x), send_expert, status);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const float* d_back, const int* inv, const float* weights, float* y,
                              int m, int hidden, int top_k, const int* status,
                              cudaStream_t stream) {
    const long long total = static_cast<long long>(m) * (hidden / 4);
    long long blocks = (total + 255) / 256;
    const long long cap = 8LL * device_sms();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    ep_combine_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(d_back), inv, weights, reinterpret_cast<float4*>(y), m,
        hidden / 4, top_k, static_cast<long long>(m) * top_k, status);
    return cudaGetLastError();
}

}  // namespace moe
