// Decode-size routed SwiGLU FFN: stream each chosen expert's weights once.
//
// Definition [cortiq-engine 0.7.7, src/mimo_moe.rs tests::exact_moe;
// hf2q 0.1.1 eagle3/forward.rs "Phase E4b.8" SwiGLU MLP]:
//   a = silu(W_gate[e] . x_row) * (W_up[e] . x_row);  d = W_down[e] . a;
//   y[t] = sum_j w[t, j] * d_j   (in slot order, by the ordered combine)
//
// For m*top_k <= 128 routed rows the layer is bound by reading the weights of
// the distinct chosen experts (the decode regime the pages' bank frames
// serve); the routed call builds its expert map inside the first kernel.  Two persistent kernels walk warp-sized work items over the expert
// map, reading every weight row once with 16-byte non-allocating loads:
//   gate/up: item = (active expert, two intermediate rows i): the warp streams
//            W_gate[e, i, :] and W_up[e, i, :], dots them with the expert's
//            x rows and writes a = silu(g)*u in f32 (no rounding of a).
//   down:    item = (active expert, 4 hidden rows): streams W_down rows, dots
//            them with the expert's f32 activation rows and writes the
//            combine-weighted rows to their (token, slot) places.
// The ordered combine then sums the slots.  Lanes split K in 8-element
// pieces and a fixed xor-butterfly reduces them, so every routed row has the
// same arithmetic whichever batch or routing it arrives in.
#include "device_common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kBatch = 4;      // routed rows per pass over a gate/up weight row
constexpr int kDownRows = 4;   // W_down rows per warp item
constexpr int kDownBatch = 4;  // routed rows per pass over W_down rows

__device__ __forceinline__ float silu_mul_f(float g, float u) { return g / (1.0f + expf(-g)) * u; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// --------------------------------------------------------------- gate / up
constexpr int kGuRows = 2;  // intermediate rows per warp item (gate + up each)

template <int NB, int U>
__device__ __forceinline__ void gate_up_pass(const __nv_bfloat16* const (&wg)[kGuRows],
                                             const __nv_bfloat16* const (&wu)[kGuRows],
                                             const __nv_bfloat16* __restrict__ x,
                                             float* __restrict__ act, const int* __restrict__ perm,
                                             int first, int nb, int i0, int inter, int hidden,
                                             int top_k, int layout, long long rows, int lane) {
    const __nv_bfloat16* xrow[NB];
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        int r = q < nb ? perm[first + q] : 0;
        if (r < 0 || r >= rows) r = 0;  // never reached with a valid map
        xrow[q] = x + static_cast<size_t>(layout ? r : r / top_k) * hidden;
    }
    float ag[NB][kGuRows], au[NB][kGuRows];
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
        for (int j = 0; j < kGuRows; ++j) ag[q][j] = au[q][j] = 0.0f;
    int kk = lane * 8;
    for (; kk + 256 * (U - 1) < hidden; kk += 256 * U) {
        uint4 rg[U][kGuRows], ru[U][kGuRows];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int j = 0; j < kGuRows; ++j) {
                rg[u][j] = ld_stream_u4(wg[j] + kk + 256 * u);
                ru[u][j] = ld_stream_u4(wu[j] + kk + 256 * u);
            }
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                if (q < nb) {
                    float xf[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4*>(xrow[q] + kk + 256 * u), xf);
#pragma unroll
                    for (int j = 0; j < kGuRows; ++j) {
                        float fg[8], fu[8];
                        bf16x8_to_f32(rg[u][j], fg);
                        bf16x8_to_f32(ru[u][j], fu);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            ag[q][j] = fmaf(fg[e], xf[e], ag[q][j]);
                            au[q][j] = fmaf(fu[e], xf[e], au[q][j]);
                        }
                    }
                }
            }
        }
    }
    for (; kk < hidden; kk += 256) {
#pragma unroll
        for (int j = 0; j < kGuRows; ++j) {
            float fg[8], fu[8];
            bf16x8_to_f32(ld_stream_u4(wg[j] + kk), fg);
            bf16x8_to_f32(ld_stream_u4(wu[j] + kk), fu);
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                if (q < nb) {
                    float xf[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4*>(xrow[q] + kk), xf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        ag[q][j] = fmaf(fg[e], xf[e], ag[q][j]);
                        au[q][j] = fmaf(fu[e], xf[e], au[q][j]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < NB; ++q) {
#pragma unroll
        for (int j = 0; j < kGuRows; ++j) {
            const float g = warp_sum(ag[q][j]);
            const float u = warp_sum(au[q][j]);
            if (lane == 0 && q < nb && i0 + j < inter)
                act[static_cast<size_t>(first + q) * inter + i0 + j] = silu_mul_f(g, u);
        }
    }
}

__global__ void __launch_bounds__(kWarps * 32, 2) stream_gate_up_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W_gate,
    const __nv_bfloat16* __restrict__ W_up, float* __restrict__ act, int hidden, int inter,
    int top_k, int layout, const int* __restrict__ perm, const int* __restrict__ counts,
    const int* __restrict__ offsets, const int* __restrict__ active,
    const int* __restrict__ n_active, long long rows) {
    const int lane = threadIdx.x & 31;
    const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int i_items = (inter + kGuRows - 1) / kGuRows;
    const long long items = static_cast<long long>(*n_active) * i_items;
    for (long long item = warp_id; item < items; item += n_warps) {
        const int a = static_cast<int>(item / i_items);
        const int i0 = static_cast<int>(item - static_cast<long long>(a) * i_items) * kGuRows;
        const int e = active[a];
        const int first = offsets[e], cnt = counts[e];
        const __nv_bfloat16* wg[kGuRows];
        const __nv_bfloat16* wu[kGuRows];
#pragma unroll
        for (int j = 0; j < kGuRows; ++j) {
            const size_t roff = (static_cast<size_t>(e) * inter + min(i0 + j, inter - 1)) * hidden;
            wg[j] = W_gate + roff;
            wu[j] = W_up + roff;
        }
        for (int b0 = 0; b0 < cnt; b0 += kBatch) {
            const int nb = min(kBatch, cnt - b0);
            if (nb == 1)
                gate_up_pass<1, 4>(wg, wu, x, act, perm, first + b0, nb, i0, inter, hidden, top_k,
                                   layout, rows, lane);
            else if (nb == 2)
                gate_up_pass<2, 2>(wg, wu, x, act, perm, first + b0, nb, i0, inter, hidden, top_k,
                                   layout, rows, lane);
            else
                gate_up_pass<4, 2>(wg, wu, x, act, perm, first + b0, nb, i0, inter, hidden, top_k,
                                   layout, rows, lane);
        }
    }
}

// The gate/up kernel with the expert map built inside it (routed FFN calls of
// at most kStreamFfnMaxRows rows): every block ranks the routed rows in
// shared memory (the stable (expert id, routed row) order of the expert map,
// so each row meets the same batches as above); block 0 also publishes the
// map the down kernel reads (perm, counts and offsets of the active experts,
// the active list) and the call's status word (MOE_ERR_DEVICE_BAD_ID for an
// id out of range, which leaves no active expert, else 0).  One launch
// replaces the status reset and the map kernel.
__global__ void __launch_bounds__(kWarps * 32, 2) stream_gate_up_fused_kernel(
    const __nv_bfloat16* __restrict__ x, const int* __restrict__ ids, int n_experts,
    const __nv_bfloat16* __restrict__ W_gate, const __nv_bfloat16* __restrict__ W_up,
    float* __restrict__ act, int hidden, int inter, int top_k, int layout, int rows,
    int* __restrict__ perm, int* __restrict__ counts, int* __restrict__ offsets,
    int* __restrict__ active, int* __restrict__ n_active, int* __restrict__ status) {
    __shared__ int s_id[kStreamFfnMaxRows];
    __shared__ int s_perm[kStreamFfnMaxRows];
    __shared__ int s_gexp[kStreamFfnMaxRows], s_gfirst[kStreamFfnMaxRows], s_gcnt[kStreamFfnMaxRows];
    __shared__ int s_warp[kWarps];
    __shared__ int s_flag;
    static_assert(kWarps * 32 >= kStreamFfnMaxRows, "one thread per routed row");
    const int lane = threadIdx.x & 31;
    int n_groups = 0;
    const bool ok = block_small_map(ids, rows, n_experts, s_id, s_perm, s_gexp, s_gfirst, s_gcnt,
                                    s_warp, &s_flag, &n_groups);
    if (blockIdx.x == 0) {
        if (ok) {
            for (int p = threadIdx.x; p < rows; p += blockDim.x) perm[p] = s_perm[p];
            for (int g = threadIdx.x; g < n_groups; g += blockDim.x) {
                const int e = s_gexp[g];
                active[g] = e;
                offsets[e] = s_gfirst[g];
                counts[e] = s_gcnt[g];
            }
        }
        if (threadIdx.x == 0) {
            *n_active = ok ? n_groups : 0;
            *status = ok ? kDevOk : kDevBadId;
        }
    }
    if (!ok) return;
    const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int i_items = (inter + kGuRows - 1) / kGuRows;
    const long long items = static_cast<long long>(n_groups) * i_items;
    for (long long item = warp_id; item < items; item += n_warps) {
        const int g = static_cast<int>(item / i_items);
        const int i0 = static_cast<int>(item - static_cast<long long>(g) * i_items) * kGuRows;
        const int e = s_gexp[g];
        const int first = s_gfirst[g], cnt = s_gcnt[g];
        const __nv_bfloat16* wg[kGuRows];
        const __nv_bfloat16* wu[kGuRows];
#pragma unroll
        for (int j = 0; j < kGuRows; ++j) {
            const size_t roff = (static_cast<size_t>(e) * inter + min(i0 + j, inter - 1)) * hidden;
            wg[j] = W_gate + roff;
            wu[j] = W_up + roff;
        }
        for (int b0 = 0; b0 < cnt; b0 += kBatch) {
            const int nb = min(kBatch, cnt - b0);
            if (nb == 1)
                gate_up_pass<1, 4>(wg, wu, x, act, s_perm, first + b0, nb, i0, inter, hidden, top_k,
                                   layout, rows, lane);
            else if (nb == 2)
                gate_up_pass<2, 2>(wg, wu, x, act, s_perm, first + b0, nb, i0, inter, hidden, top_k,
                                   layout, rows, lane);
            else
                gate_up_pass<4, 2>(wg, wu, x, act, s_perm, first + b0, nb, i0, inter, hidden, top_k,
                                   layout, rows, lane);
        }
    }
}

// --------------------------------------------------------------- down
template <int NB>
__device__ __forceinline__ void down_pass(const __nv_bfloat16* const (&wrow)[kDownRows],
                                          const float* __restrict__ act,
                                          float* __restrict__ y_slots,
                                          const float* __restrict__ weights,
                                          const int* __restrict__ perm, int first, int nb, int h0,
                                          int hidden, int inter, long long rows, int lane) {
    float acc[NB][kDownRows];
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
        for (int j = 0; j < kDownRows; ++j) acc[q][j] = 0.0f;
    for (int kk = lane * 8; kk < inter; kk += 256) {
        uint4 raw[kDownRows];
#pragma unroll
        for (int j = 0; j < kDownRows; ++j) raw[j] = ld_stream_u4(wrow[j] + kk);
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            if (q < nb) {
                const float4* ap = reinterpret_cast<const float4*>(act + static_cast<size_t>(first + q) * inter + kk);
                const float4 a0 = ap[0], a1 = ap[1];
                const float af[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                for (int j = 0; j < kDownRows; ++j) {
                    float wf[8];
                    bf16x8_to_f32(raw[j], wf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[q][j] = fmaf(wf[e], af[e], acc[q][j]);
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < NB; ++q) {
#pragma unroll
        for (int j = 0; j < kDownRows; ++j) acc[q][j] = warp_sum(acc[q][j]);
    }
    if (lane == 0) {
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            if (q < nb) {
                const int r = perm[first + q];
                if (r < 0 || r >= rows) continue;  // never reached with a valid map
                const float w = weights ? weights[r] : 1.0f;  // null: unweighted rows
#pragma unroll
                for (int j = 0; j < kDownRows; ++j)
                    if (h0 + j < hidden) y_slots[static_cast<size_t>(r) * hidden + h0 + j] = w * acc[q][j];
            }
        }
    }
}

__global__ void __launch_bounds__(kWarps * 32, 2) stream_down_kernel(
    const float* __restrict__ act, const __nv_bfloat16* __restrict__ W_down,
    const float* __restrict__ weights, float* __restrict__ y_slots, int hidden, int inter,
    const int* __restrict__ perm, const int* __restrict__ counts, const int* __restrict__ offsets,
    const int* __restrict__ active, const int* __restrict__ n_active, long long rows) {
    const int lane = threadIdx.x & 31;
    const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int h_items = (hidden + kDownRows - 1) / kDownRows;
    const long long items = static_cast<long long>(*n_active) * h_items;
    for (long long item = warp_id; item < items; item += n_warps) {
        const int a = static_cast<int>(item / h_items);
        const int h0 = static_cast<int>(item - static_cast<long long>(a) * h_items) * kDownRows;
        const int e = active[a];
        const int first = offsets[e], cnt = counts[e];
        const __nv_bfloat16* wrow[kDownRows];
#pragma unroll
        for (int j = 0; j < kDownRows; ++j)
            wrow[j] = W_down + (static_cast<size_t>(e) * hidden + min(h0 + j, hidden - 1)) * inter;
        for (int b0 = 0; b0 < cnt; b0 += kDownBatch) {
            const int nb = min(kDownBatch, cnt - b0);
            if (nb == 1)
                down_pass<1>(wrow, act, y_slots, weights, perm, first + b0, nb, h0, hidden, inter, rows, lane);
            else if (nb == 2)
                down_pass<2>(wrow, act, y_slots, weights, perm, first + b0, nb, h0, hidden, inter, rows, lane);
            else
                down_pass<4>(wrow, act, y_slots, weights, perm, first + b0, nb, h0, hidden, inter, rows, lane);
        }
    }
}

}  // namespace

cudaError_t launch_stream_ffn(const __nv_bfloat16* x, const float* weights,
                              const __nv_bfloat16* W_gate, const __nv_bfloat16* W_up,
                              const __nv_bfloat16* W_down, float* act, float* y_slots, int m,
                              int hidden, int inter, int top_k, int layout, const MapBuffers& b,
                              cudaStream_t stream, const int* ids, int n_experts) {
    const long long rows = static_cast<long long>(m) * top_k;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = 2 * sms;
    if (ids)
        stream_gate_up_fused_kernel<<<grid, kWarps * 32, 0, stream>>>(
            x, ids, n_experts, W_gate, W_up, act, hidden, inter, top_k, layout,
            static_cast<int>(rows), b.perm, b.counts, b.offsets, b.active, b.n_active, b.status);
    else
        stream_gate_up_kernel<<<grid, kWarps * 32, 0, stream>>>(x, W_gate, W_up, act, hidden,
                                                                inter, top_k, layout, b.perm,
                                                                b.counts, b.offsets, b.active,
                                                                b.n_active, rows);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    stream_down_kernel<<<grid, kWarps * 32, 0, stream>>>(act, W_down, weights, y_slots, hidden,
                                                         inter, b.perm, b.counts, b.offsets,
                                                         b.active, b.n_active, rows);
    return cudaGetLastError();
}

}  // namespace moe
