// Small-m matmul by expert id: stream each chosen expert's weights once.
//
// Definition [mlx-native 0.13.0, src/ops/dense_matmul_id_auto.rs,
// DenseMatmulIdShape and the Direct route of expected_dispatches]:
//   y[t, j, c] = sum_i W[ids[t,j], c, i] * x_row(t, j)[i]
//
// At decode sizes (m*top_k <= 256) the work is bound by reading the weights
// of the distinct chosen experts.  The expert map groups routed rows by
// expert; block (chunk, a) takes active expert a and 32 output rows of its
// weight matrix, and every weight row is read exactly once with 16-byte
// non-allocating loads, then applied to all (up to 8 per pass) routed rows of
// that expert, whose x rows stay in L1/L2.  Lanes split K in 8-element
// pieces; a fixed xor-butterfly reduces the lanes, so results are
// deterministic.
#include "device_common.cuh"
#include "launch.h"

namespace moe {

constexpr int kStreamWarps = 8;
constexpr int kStreamRowsPerWarp = 4;
constexpr int kStreamRowsPerBlock = kStreamWarps * kStreamRowsPerWarp;
constexpr int kStreamBatch = 8;  // routed rows applied per pass over the weights

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__global__ void __launch_bounds__(kStreamWarps * 32) stream_matmul_id_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W,
    float* __restrict__ y, int n, int k, int top_k, int layout, const int* __restrict__ perm,
    const int* __restrict__ counts, const int* __restrict__ offsets,
    const int* __restrict__ active, const int* __restrict__ n_active, long long rows) {
    const int a = blockIdx.y;
    if (a >= *n_active) return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = active[a];
    const int first = offsets[e], cnt = counts[e];
    const int c0 = blockIdx.x * kStreamRowsPerBlock + warp * kStreamRowsPerWarp;
    if (c0 >= n) return;
    const __nv_bfloat16* We = W + static_cast<size_t>(e) * n * k;

    for (int b0 = 0; b0 < cnt; b0 += kStreamBatch) {
        const int nb = min(kStreamBatch, cnt - b0);
        const __nv_bfloat16* xrow[kStreamBatch];
        int rrow[kStreamBatch];
#pragma unroll
        for (int q = 0; q < kStreamBatch; ++q) {
            int r = q < nb ? perm[first + b0 + q] : 0;
            if (r < 0 || r >= rows) r = 0;  // never reached with a valid map
            rrow[q] = r;
            const long long xr = layout ? r : r / top_k;
            xrow[q] = x + static_cast<size_t>(xr) * k;
        }
        float acc[kStreamBatch][kStreamRowsPerWarp];
#pragma unroll
        for (int q = 0; q < kStreamBatch; ++q)
#pragma unroll
            for (int j = 0; j < kStreamRowsPerWarp; ++j) acc[q][j] = 0.0f;

#pragma unroll 2
        for (int kk = lane * 8; kk < k; kk += 256) {
            float wf[kStreamRowsPerWarp][8];
#pragma unroll
            for (int j = 0; j < kStreamRowsPerWarp; ++j) {
                const int c = min(c0 + j, n - 1);
                bf16x8_to_f32(ld_stream_u4(We + static_cast<size_t>(c) * k + kk), wf[j]);
            }
#pragma unroll
            for (int q = 0; q < kStreamBatch; ++q) {
                if (q < nb) {
                    float xf[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4*>(xrow[q] + kk), xf);
#pragma unroll
                    for (int j = 0; j < kStreamRowsPerWarp; ++j)
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[q][j] = fmaf(wf[j][i], xf[i], acc[q][j]);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kStreamBatch; ++q) {
#pragma unroll
            for (int j = 0; j < kStreamRowsPerWarp; ++j) {
                float v = acc[q][j];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                acc[q][j] = v;
            }
        }
        if (lane == 0) {
            for (int q = 0; q < nb; ++q)
#pragma unroll
                for (int j = 0; j < kStreamRowsPerWarp; ++j)
                    if (c0 + j < n) y[static_cast<size_t>(rrow[q]) * n + c0 + j] = acc[q][j];
        }
    }
}

cudaError_t launch_stream_matmul_id(const __nv_bfloat16* x, const __nv_bfloat16* W, float* y,
                                    int m, int n, int k, int top_k, int n_experts, int layout,
                                    const MapBuffers& b, cudaStream_t stream) {
    const long long rows = static_cast<long long>(m) * top_k;
    const int max_active = static_cast<int>(rows < n_experts ? rows : n_experts);
    const dim3 grid((n + kStreamRowsPerBlock - 1) / kStreamRowsPerBlock, max_active);
    stream_matmul_id_kernel<<<grid, kStreamWarps * 32, 0, stream>>>(
        x, W, y, n, k, top_k, layout, b.perm, b.counts, b.offsets, b.active, b.n_active, rows);
    return cudaGetLastError();
}

}  // namespace moe
