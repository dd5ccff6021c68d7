// Expert map: a deterministic, stable counting sort of routed rows by expert.
//
// Definition [mlx-native 0.13.0, src/ops/dense_matmul_id_auto.rs,
// expected_dispatches: the Grouped route first runs a map pass over the
// expert ids, then the grouped kernel walks rows expert by expert]:
//   counts[e], offsets = exclusive scan of counts, perm = routed rows
//   r = t*top_k + j sorted by (ids[r], r), inv_perm[perm[p]] = p.
//
// Up to 2048 rows: one fused block (map_fused_kernel).  Above that, three
// launches, all free of global atomics:
//   1. map_count:   per 2048-row chunk, a shared-memory histogram.
//   2. map_scan:    one block: per-expert totals, the exclusive scan, each
//                   chunk's starting position per expert, the list of
//                   128-row tiles (expert, first sorted row, rows) consumed by
//                   the grouped GEMM, and the list of experts with rows.
//   3. map_scatter: per chunk, 8 warps of 256 rows; per-warp histograms give
//                   each warp its start, and __match_any_sync ranks equal ids
//                   inside a 32-row step so rows keep ascending r.
#include "device_common.cuh"
#include "launch.h"

namespace moe {

constexpr int kMapThreads = 256;
constexpr int kMapWarpRows = 256;  // rows per warp in map_scatter
constexpr int kMapScanThreads = 1024;

__global__ void __launch_bounds__(kMapThreads) map_count_kernel(const int* __restrict__ ids,
                                                                int rows, int n_experts,
                                                                int* __restrict__ chunk_hist,
                                                                int* __restrict__ status) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < n_experts; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int begin = blockIdx.x * kMapChunkRows;
    const int end = min(rows, begin + kMapChunkRows);
    bool bad = false;
    for (int r = begin + threadIdx.x; r < end; r += blockDim.x) {
        const int e = ids[r];
        if (e >= 0 && e < n_experts) atomicAdd(&hist[e], 1);
        else bad = true;
    }
    if (bad) set_status(status, kDevBadId);
    __syncthreads();
    int* out = chunk_hist + static_cast<size_t>(blockIdx.x) * n_experts;
    for (int e = threadIdx.x; e < n_experts; e += blockDim.x) out[e] = hist[e];
}

// Exclusive block scan of three int values at once (blockDim.x == 1024).
__device__ __forceinline__ int3 block_exclusive_scan3(int3 v, int3* total) {
    __shared__ int3 warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int3 inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, inc.x, off);
        const int b = __shfl_up_sync(0xffffffffu, inc.y, off);
        const int c = __shfl_up_sync(0xffffffffu, inc.z, off);
        if (lane >= off) {
            inc.x += a;
            inc.y += b;
            inc.z += c;
        }
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int3 s = warp_sums[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, s.x, off);
            const int b = __shfl_up_sync(0xffffffffu, s.y, off);
            const int c = __shfl_up_sync(0xffffffffu, s.z, off);
            if (lane >= off) {
                s.x += a;
                s.y += b;
                s.z += c;
            }
        }
        warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int3 before = warp > 0 ? warp_sums[warp - 1] : make_int3(0, 0, 0);
    *total = warp_sums[31];
    return make_int3(before.x + inc.x - v.x, before.y + inc.y - v.y, before.z + inc.z - v.z);
}

__global__ void __launch_bounds__(kMapScanThreads) map_scan_kernel(
    const int* __restrict__ chunk_hist, int n_chunks, int n_experts, int tile_rows,
    int* __restrict__ counts, int* __restrict__ offsets, int* __restrict__ chunk_base,
    int4* __restrict__ tiles, int* __restrict__ n_tiles, int* __restrict__ active,
    int* __restrict__ n_active, const int* __restrict__ status) {
    const int e = threadIdx.x;
    int cnt = 0;
    if (e < n_experts)
        for (int c = 0; c < n_chunks; ++c) cnt += chunk_hist[static_cast<size_t>(c) * n_experts + e];
    const int ntile = (cnt + tile_rows - 1) / tile_rows;
    int3 total;
    const int3 ex = block_exclusive_scan3(make_int3(cnt, ntile, cnt > 0 ? 1 : 0), &total);
    const bool failed = *status != 0;
    if (e < n_experts) {
        counts[e] = cnt;
        offsets[e] = ex.x;
        int run = ex.x;
        for (int c = 0; c < n_chunks; ++c) {
            const size_t i = static_cast<size_t>(c) * n_experts + e;
            const int h = chunk_hist[i];
            chunk_base[i] = run;
            run += h;
        }
        for (int i = 0; i < ntile; ++i)
            tiles[ex.y + i] = make_int4(e, ex.x + i * tile_rows, min(tile_rows, cnt - i * tile_rows), 0);
        if (cnt > 0) active[ex.z] = e;
    }
    if (threadIdx.x == 0) {
        offsets[n_experts] = total.x;
        // A failed call hands the consumers no work at all.
        *n_tiles = failed ? 0 : total.y;
        *n_active = failed ? 0 : total.z;
    }
}

__global__ void __launch_bounds__(kMapThreads) map_scatter_kernel(
    const int* __restrict__ ids, int rows, int n_experts, const int* __restrict__ chunk_base,
    int* __restrict__ perm, int* __restrict__ inv_perm) {
    extern __shared__ int warp_hist[];  // [8][n_experts]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kMapThreads / 32;
    for (int i = threadIdx.x; i < kWarps * n_experts; i += blockDim.x) warp_hist[i] = 0;
    __syncthreads();
    const int base_r = blockIdx.x * kMapChunkRows + warp * kMapWarpRows;
    int* my_hist = warp_hist + warp * n_experts;
    for (int s = 0; s < kMapWarpRows; s += 32) {
        const int r = base_r + s + lane;
        if (r < rows) {
            const int e = ids[r];
            if (e >= 0 && e < n_experts) atomicAdd(&my_hist[e], 1);
        }
    }
    __syncthreads();
    const int* cb = chunk_base + static_cast<size_t>(blockIdx.x) * n_experts;
    for (int e = threadIdx.x; e < n_experts; e += blockDim.x) {
        int run = cb[e];
        for (int w = 0; w < kWarps; ++w) {
            const int h = warp_hist[w * n_experts + e];
            warp_hist[w * n_experts + e] = run;
            run += h;
        }
    }
    __syncthreads();
    const uint32_t lt = lanemask_lt();
    for (int s = 0; s < kMapWarpRows; s += 32) {
        const int r = base_r + s + lane;
        int e = -1;
        if (r < rows) e = ids[r];
        const bool ok = r < rows && e >= 0 && e < n_experts;
        if (!ok) e = -1;
        const uint32_t valid = __ballot_sync(0xffffffffu, ok);
        const uint32_t peers = __match_any_sync(0xffffffffu, e) & valid;
        int base = 0, rank = 0;
        if (ok) {
            base = my_hist[e];
            rank = __popc(peers & lt);
            const int pos = base + rank;
            perm[pos] = r;
            inv_perm[r] = pos;
        }
        __syncwarp();
        if (ok && rank == 0) my_hist[e] = base + __popc(peers);
        __syncwarp();
    }
}

// Whole map in one block for up to kMapChunkRows rows (decode sizes): the
// three passes above with one chunk, fused so a small call pays one launch.
// Phases: per-expert counts (shared atomics) -> block scan (offsets, tile
// and active-expert lists) -> stable scatter by 8 warps of 256 rows each.
__global__ void __launch_bounds__(kMapScanThreads) map_fused_kernel(
    const int* __restrict__ ids, int rows, int n_experts, int tile_rows, int* __restrict__ counts,
    int* __restrict__ offsets, int* __restrict__ perm, int* __restrict__ inv_perm,
    int4* __restrict__ tiles, int* __restrict__ n_tiles, int* __restrict__ active,
    int* __restrict__ n_active, int* __restrict__ status) {
    extern __shared__ int sm[];
    int* hist = sm;                    // [E]
    int* warp_hist = sm + n_experts;   // [8][E]
    __shared__ int bad;
    constexpr int kScatterWarps = kMapThreads / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (1 + kScatterWarps) * n_experts; i += blockDim.x) sm[i] = 0;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    for (int r = threadIdx.x; r < rows; r += blockDim.x) {
        const int e = ids[r];
        if (e >= 0 && e < n_experts) {
            atomicAdd(&hist[e], 1);
            atomicAdd(&warp_hist[(r / kMapWarpRows) * n_experts + e], 1);
        } else {
            bad = 1;
        }
    }
    __syncthreads();
    const bool failed = bad != 0;
    if (failed && threadIdx.x == 0) set_status(status, kDevBadId);
    const int e = threadIdx.x;
    const int cnt = e < n_experts ? hist[e] : 0;
    const int ntile = (cnt + tile_rows - 1) / tile_rows;
    int3 total;
    const int3 ex = block_exclusive_scan3(make_int3(cnt, ntile, cnt > 0 ? 1 : 0), &total);
    if (e < n_experts) {
        counts[e] = cnt;
        offsets[e] = ex.x;
        for (int i = 0; i < ntile; ++i)
            tiles[ex.y + i] = make_int4(e, ex.x + i * tile_rows, min(tile_rows, cnt - i * tile_rows), 0);
        if (cnt > 0) active[ex.z] = e;
        int run = ex.x;  // each scatter warp's first position for expert e
        for (int w = 0; w < kScatterWarps; ++w) {
            const int h = warp_hist[w * n_experts + e];
            warp_hist[w * n_experts + e] = run;
            run += h;
        }
    }
    if (threadIdx.x == 0) {
        offsets[n_experts] = total.x;
        *n_tiles = failed ? 0 : total.y;
        *n_active = failed ? 0 : total.z;
    }
    __syncthreads();
    if (warp < kScatterWarps) {
        int* my_hist = warp_hist + warp * n_experts;
        const uint32_t lt = lanemask_lt();
        const int base_r = warp * kMapWarpRows;
        for (int s = 0; s < kMapWarpRows; s += 32) {
            const int r = base_r + s + lane;
            int ev = -1;
            if (r < rows) ev = ids[r];
            const bool ok = r < rows && ev >= 0 && ev < n_experts;
            if (!ok) ev = -1;
            const uint32_t valid = __ballot_sync(0xffffffffu, ok);
            const uint32_t peers = __match_any_sync(0xffffffffu, ev) & valid;
            int base = 0, rank = 0;
            if (ok) {
                base = my_hist[ev];
                rank = __popc(peers & lt);
                const int pos = base + rank;
                perm[pos] = r;
                inv_perm[r] = pos;
            }
            __syncwarp();
            if (ok && rank == 0) my_hist[ev] = base + __popc(peers);
            __syncwarp();
        }
    }
}

cudaError_t launch_expert_map(const int* ids, int rows, int n_experts, int tile_rows,
                              const MapBuffers& b, cudaStream_t stream) {
    if (rows <= kMapChunkRows) {
        const size_t smem = (1 + kMapThreads / 32) * static_cast<size_t>(n_experts) * sizeof(int);
        map_fused_kernel<<<1, kMapScanThreads, smem, stream>>>(
            ids, rows, n_experts, tile_rows, b.counts, b.offsets, b.perm, b.inv_perm, b.tiles,
            b.n_tiles, b.active, b.n_active, b.status);
        return cudaGetLastError();
    }
    const int n_chunks = (rows + kMapChunkRows - 1) / kMapChunkRows;
    map_count_kernel<<<n_chunks, kMapThreads, n_experts * sizeof(int), stream>>>(
        ids, rows, n_experts, b.chunk_hist, b.status);
    map_scan_kernel<<<1, kMapScanThreads, 0, stream>>>(b.chunk_hist, n_chunks, n_experts,
                                                       tile_rows, b.counts, b.offsets,
                                                       b.chunk_base, b.tiles, b.n_tiles, b.active,
                                                       b.n_active, b.status);
    map_scatter_kernel<<<n_chunks, kMapThreads, (kMapThreads / 32) * n_experts * sizeof(int),
                         stream>>>(ids, rows, n_experts, b.chunk_base, b.perm, b.inv_perm);
    return cudaGetLastError();
}

// One expert takes every row: perm and inv_perm are the identity and the
// tiles cut rows 0..rows-1 in tile_rows pieces.  Grid-stride over rows.
__global__ void __launch_bounds__(kMapThreads) map_dense_kernel(
    int rows, int tile_rows, int* __restrict__ counts, int* __restrict__ offsets,
    int* __restrict__ perm, int* __restrict__ inv_perm, int4* __restrict__ tiles,
    int* __restrict__ n_tiles, int* __restrict__ active, int* __restrict__ n_active) {
    const int stride = gridDim.x * blockDim.x;
    const int first = blockIdx.x * blockDim.x + threadIdx.x;
    for (int r = first; r < rows; r += stride) {
        perm[r] = r;
        inv_perm[r] = r;
    }
    const int nt = (rows + tile_rows - 1) / tile_rows;
    for (int i = first; i < nt; i += stride)
        tiles[i] = make_int4(0, i * tile_rows, min(tile_rows, rows - i * tile_rows), 0);
    if (first == 0) {
        counts[0] = rows;
        offsets[0] = 0;
        offsets[1] = rows;
        *n_tiles = nt;
        active[0] = 0;
        *n_active = rows > 0 ? 1 : 0;
    }
}

cudaError_t launch_dense_map(int rows, int tile_rows, const MapBuffers& b, cudaStream_t stream) {
    int blocks = (rows + kMapThreads - 1) / kMapThreads;
    if (blocks > 256) blocks = 256;
    if (blocks < 1) blocks = 1;
    map_dense_kernel<<<blocks, kMapThreads, 0, stream>>>(rows, tile_rows, b.counts, b.offsets,
                                                         b.perm, b.inv_perm, b.tiles, b.n_tiles,
                                                         b.active, b.n_active);
    return cudaGetLastError();
}

}  // namespace moe
