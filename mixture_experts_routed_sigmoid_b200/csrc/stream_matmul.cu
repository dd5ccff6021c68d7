// Small-m matmul by expert id: stream each chosen expert's weights once.
//
// Definition [mlx-native 0.13.0, src/ops/dense_matmul_id_auto.rs,
// DenseMatmulIdShape and the Direct route of expected_dispatches]:
//   y[t, j, c] = sum_i W[ids[t,j], c, i] * x_row(t, j)[i]
//
// At decode sizes (m*top_k <= 256) the work is bound by reading the weights
// of the distinct chosen experts.  The expert map groups routed rows by
// expert; persistent blocks walk the work items (active expert, 32 weight
// rows), and every weight row is read exactly once with 16-byte
// non-allocating loads (4 k-steps per lane in flight), then applied to all
// (up to 8 per pass) routed rows of that expert, whose x rows stay in L1/L2.
// Lanes split K in 8-element pieces; a fixed xor-butterfly reduces the
// lanes, so results are deterministic.
#include "device_common.cuh"
#include "launch.h"

namespace moe {

constexpr int kStreamWarps = 8;
constexpr int kStreamRowsPerWarp = 4;
constexpr int kStreamRowsPerBlock = kStreamWarps * kStreamRowsPerWarp;
constexpr int kStreamBatch = 8;  // routed rows applied per pass over the weights

// Dot products of one k-step (8 elements per lane) for NB routed rows.  The
// weights are widened per row inside the loop to keep register use low.
template <int NB>
__device__ __forceinline__ void stream_accumulate(const uint4 (&wraw)[kStreamRowsPerWarp],
                                                  const __nv_bfloat16* const (&xrow)[NB], int nb,
                                                  int kk, float (&acc)[NB][kStreamRowsPerWarp]) {
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        if (q < nb) {
            float xf[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(xrow[q] + kk), xf);
#pragma unroll
            for (int j = 0; j < kStreamRowsPerWarp; ++j) {
                float wf[8];
                bf16x8_to_f32(wraw[j], wf);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[q][j] = fmaf(wf[i], xf[i], acc[q][j]);
            }
        }
    }
}

// One pass over a warp's 4 weight rows for nb <= NB routed rows of the
// expert (sorted positions first..first+nb-1).  U k-steps of 16-byte weight
// loads are issued before any arithmetic.
template <int NB, int U>
__device__ __forceinline__ void stream_pass(const __nv_bfloat16* const (&wrow)[kStreamRowsPerWarp],
                                            const __nv_bfloat16* __restrict__ x,
                                            float* __restrict__ y, const int* __restrict__ perm,
                                            int first, int nb, int c0, int n, int k, int top_k,
                                            int layout, long long rows, int lane) {
    const __nv_bfloat16* xrow[NB];
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        int r = q < nb ? perm[first + q] : 0;
        if (r < 0 || r >= rows) r = 0;  // never reached with a valid map
        const long long xr = layout ? r : r / top_k;
        xrow[q] = x + static_cast<size_t>(xr) * k;
    }
    float acc[NB][kStreamRowsPerWarp];
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
        for (int j = 0; j < kStreamRowsPerWarp; ++j) acc[q][j] = 0.0f;

    int kk = lane * 8;
    for (; kk + 256 * (U - 1) < k; kk += 256 * U) {
        uint4 wraw[U][kStreamRowsPerWarp];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int j = 0; j < kStreamRowsPerWarp; ++j)
                wraw[u][j] = ld_stream_u4(wrow[j] + kk + 256 * u);
#pragma unroll
        for (int u = 0; u < U; ++u) stream_accumulate<NB>(wraw[u], xrow, nb, kk + 256 * u, acc);
    }
    for (; kk < k; kk += 256) {
        uint4 wraw[kStreamRowsPerWarp];
#pragma unroll
        for (int j = 0; j < kStreamRowsPerWarp; ++j) wraw[j] = ld_stream_u4(wrow[j] + kk);
        stream_accumulate<NB>(wraw, xrow, nb, kk, acc);
    }
#pragma unroll
    for (int q = 0; q < NB; ++q) {
#pragma unroll
        for (int j = 0; j < kStreamRowsPerWarp; ++j) {
            float v = acc[q][j];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            acc[q][j] = v;
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            if (q < nb) {
                int r = perm[first + q];
                if (r < 0 || r >= rows) continue;
#pragma unroll
                for (int j = 0; j < kStreamRowsPerWarp; ++j)
                    if (c0 + j < n) y[static_cast<size_t>(r) * n + c0 + j] = acc[q][j];
            }
        }
    }
}

// Persistent: work item = (active expert a, chunk of 32 weight rows), chunk
// fastest so consecutive blocks stream consecutive rows of one expert.
__global__ void __launch_bounds__(kStreamWarps * 32, 2) stream_matmul_id_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W,
    float* __restrict__ y, int n, int k, int top_k, int layout, const int* __restrict__ perm,
    const int* __restrict__ counts, const int* __restrict__ offsets,
    const int* __restrict__ active, const int* __restrict__ n_active, long long rows,
    size_t w_stride) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_chunks = (n + kStreamRowsPerBlock - 1) / kStreamRowsPerBlock;
    const int items = *n_active * n_chunks;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int a = item / n_chunks, chunk = item - a * n_chunks;
        const int e = active[a];
        const int first = offsets[e], cnt = counts[e];
        const int c0 = chunk * kStreamRowsPerBlock + warp * kStreamRowsPerWarp;
        if (c0 >= n) continue;  // warp-uniform
        const __nv_bfloat16* We = W + static_cast<size_t>(e) * w_stride;
        const __nv_bfloat16* wrow[kStreamRowsPerWarp];
#pragma unroll
        for (int j = 0; j < kStreamRowsPerWarp; ++j)
            wrow[j] = We + static_cast<size_t>(min(c0 + j, n - 1)) * k;
        // The batch size is a function of the count only; every routed row's
        // K order and reduction tree are the same whichever batch it is in.
        for (int b0 = 0; b0 < cnt; b0 += kStreamBatch) {
            const int nb = min(kStreamBatch, cnt - b0);
            if (nb == 1)
                stream_pass<1, 4>(wrow, x, y, perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
            else if (nb == 2)
                stream_pass<2, 2>(wrow, x, y, perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
            else if (nb <= 4)
                stream_pass<4, 2>(wrow, x, y, perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
            else
                stream_pass<8, 1>(wrow, x, y, perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
        }
    }
}

// The same matmul with the expert map built inside the kernel, for up to
// kStreamMaxRows routed rows: every block ranks the routed rows in shared
// memory -- the stable order by (expert id, routed row) that the expert map
// gives, so each row meets the same batches and arithmetic as above -- groups
// them by expert and walks the same work items.  Block 0 writes the call's
// status word (MOE_ERR_DEVICE_BAD_ID when an id is out of range, else 0); a
// call with a bad id writes no output.  One launch replaces the status reset,
// the map kernel and the streaming kernel.
__global__ void __launch_bounds__(kStreamWarps * 32, 2) stream_matmul_id_fused_kernel(
    const __nv_bfloat16* __restrict__ x, const int* __restrict__ ids,
    const __nv_bfloat16* __restrict__ W, float* __restrict__ y, int n, int k, int top_k,
    int n_experts, int layout, int rows, size_t w_stride, int* __restrict__ status) {
    __shared__ int s_id[kStreamMaxRows];
    __shared__ int s_perm[kStreamMaxRows];
    __shared__ int s_gexp[kStreamMaxRows], s_gfirst[kStreamMaxRows], s_gcnt[kStreamMaxRows];
    __shared__ int s_warp[kStreamWarps];
    __shared__ int s_flag;
    static_assert(kStreamWarps * 32 >= kStreamMaxRows, "one thread per routed row");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int n_groups = 0;
    const bool ok = block_small_map(ids, rows, n_experts, s_id, s_perm, s_gexp, s_gfirst, s_gcnt,
                                    s_warp, &s_flag, &n_groups);
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = ok ? kDevOk : kDevBadId;
    if (!ok) return;

    const int n_chunks = (n + kStreamRowsPerBlock - 1) / kStreamRowsPerBlock;
    const int items = n_groups * n_chunks;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int g = item / n_chunks, chunk = item - g * n_chunks;
        const int e = s_gexp[g], first = s_gfirst[g], cnt = s_gcnt[g];
        const int c0 = chunk * kStreamRowsPerBlock + warp * kStreamRowsPerWarp;
        if (c0 >= n) continue;  // warp-uniform
        const __nv_bfloat16* We = W + static_cast<size_t>(e) * w_stride;
        const __nv_bfloat16* wrow[kStreamRowsPerWarp];
#pragma unroll
        for (int j = 0; j < kStreamRowsPerWarp; ++j)
            wrow[j] = We + static_cast<size_t>(min(c0 + j, n - 1)) * k;
        for (int b0 = 0; b0 < cnt; b0 += kStreamBatch) {
            const int nb = min(kStreamBatch, cnt - b0);
            if (nb == 1)
                stream_pass<1, 4>(wrow, x, y, s_perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
            else if (nb == 2)
                stream_pass<2, 2>(wrow, x, y, s_perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
            else if (nb <= 4)
                stream_pass<4, 2>(wrow, x, y, s_perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
            else
                stream_pass<8, 1>(wrow, x, y, s_perm, first + b0, nb, c0, n, k, top_k, layout, rows, lane);
        }
    }
}

cudaError_t launch_stream_matmul_id_fused(const __nv_bfloat16* x, const int* ids,
                                          const __nv_bfloat16* W, float* y, int m, int n, int k,
                                          int top_k, int n_experts, int layout, size_t w_stride,
                                          int* status, cudaStream_t stream) {
    const int rows = m * top_k;  // <= kStreamMaxRows, checked by the caller
    const long long max_active = rows < n_experts ? rows : n_experts;
    const long long max_items = max_active * ((n + kStreamRowsPerBlock - 1) / kStreamRowsPerBlock);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long grid = max_items < 2LL * sms ? max_items : 2LL * sms;
    if (grid < 1) grid = 1;  // block 0 always writes the status word
    stream_matmul_id_fused_kernel<<<static_cast<int>(grid), kStreamWarps * 32, 0, stream>>>(
        x, ids, W, y, n, k, top_k, n_experts, layout, rows, w_stride, status);
    return cudaGetLastError();
}

cudaError_t launch_stream_matmul_id(const __nv_bfloat16* x, const __nv_bfloat16* W, float* y,
                                    int m, int n, int k, int top_k, int n_experts, int layout,
                                    size_t w_stride, const MapBuffers& b, cudaStream_t stream) {
    const long long rows = static_cast<long long>(m) * top_k;
    const long long max_active = rows < n_experts ? rows : n_experts;
    const long long max_items = max_active * ((n + kStreamRowsPerBlock - 1) / kStreamRowsPerBlock);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long grid = max_items < 2LL * sms ? max_items : 2LL * sms;
    stream_matmul_id_kernel<<<static_cast<int>(grid), kStreamWarps * 32, 0, stream>>>(
        x, W, y, n, k, top_k, layout, b.perm, b.counts, b.offsets, b.active, b.n_active, rows,
        w_stride);
    return cudaGetLastError();
}

}  // namespace moe
