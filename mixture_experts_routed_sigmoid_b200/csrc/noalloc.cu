// moe_matmul_id_noalloc: the decode-size matmul by expert id for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand this library a workspace: a
// plugin inside a host runtime that owns every device allocation, or a decode
// loop that must never enter the driver's allocator (which can block or
// synchronise).  This entry point keeps its scratch -- the expert map: status
// word, counts, offsets, permutation, per-chunk histograms, tile and expert
// lists -- in one static device array of this file, so the caller passes only
// inputs and outputs.
//
// Rules of the static scratch:
//  * It holds kNoallocScratchBytes (64 KiB) per device, reserved on every
//    GPU that loads the library until the process exits.
//  * Its address is looked up once per device, by the first call made with
//    that device current; make that first call before any stream capture.
//  * Every call on a device shares it and leaves the last call's contents.
//    Each call clears the status word itself; the other fields are fully
//    rewritten by the map kernels.  Calls that overlap on the GPU (different
//    streams, or different host threads, without ordering between them) race
//    on it and give wrong results.
//  * A context reset after the first call on a device (cudaDeviceReset, or
//    anything else that destroys the primary context) is not supported: the
//    cached address would name memory of the destroyed context.
//  * Errors found on the device (an expert id outside [0, n_experts)) land in
//    the scratch's status word; moe_matmul_id_noalloc_status() reads it.
//  * No call allocates: no cudaMalloc, no cudaFree, no allocating library.
#include <mutex>

#include "device_common.cuh"
#include "launch.h"
#include "moe_b200.h"

namespace {

constexpr size_t kNoallocScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
// Up to kMapChunkRows routed rows the expert map runs as one fused block that
// needs no per-chunk histograms, so the carve below leaves them out.
static_assert(MOE_NOALLOC_MAX_ROUTED_ROWS <= moe::kMapChunkRows,
              "the static scratch holds no per-chunk map buffers");
// The status word sits at offset 0 of the scratch.
constexpr size_t kStatusOffset = 0;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

moe_status_t noalloc_fail(moe_status_t code, const char* msg) {
    moe::set_last_error(msg);
    return code;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Device address of the static scratch on the current device (set up once).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

MOE_API moe_status_t moe_matmul_id_noalloc(const moe_bf16_t* x, const int32_t* ids,
                                           const moe_bf16_t* W, float* y, int32_t m, int32_t n,
                                           int32_t k, int32_t top_k, int32_t n_experts,
                                           int32_t layout, void* stream) {
    moe::set_last_error("");
    if (m < 0) return noalloc_fail(MOE_ERR_INVALID_ARGUMENT, "m must be >= 0");
    if (n_experts < 1 || n_experts > MOE_MAX_EXPERTS)
        return noalloc_fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_experts must be in [1, 1024]");
    if (top_k < 1 || top_k > n_experts || top_k > MOE_MAX_TOP_K)
        return noalloc_fail(MOE_ERR_UNSUPPORTED_SHAPE, "top_k must be in [1, min(n_experts, 32)]");
    if (layout != MOE_LAYOUT_SHARED_PER_TOKEN && layout != MOE_LAYOUT_SLOTTED)
        return noalloc_fail(MOE_ERR_INVALID_ARGUMENT, "layout must be 0 or 1");
    if (n < 1 || n > (1 << 20)) return noalloc_fail(MOE_ERR_UNSUPPORTED_SHAPE, "n must be in [1, 2^20]");
    if (k < 8 || k % 8 || k > (1 << 20))
        return noalloc_fail(MOE_ERR_UNSUPPORTED_SHAPE, "k must be a positive multiple of 8");
    const long long rows = static_cast<long long>(m) * top_k;
    if (rows > MOE_NOALLOC_MAX_ROUTED_ROWS)
        return noalloc_fail(MOE_ERR_UNSUPPORTED_SHAPE,
                            "m*top_k exceeds the static-scratch limit of 256 routed rows; "
                            "use moe_matmul_id with a workspace");
    if (m == 0) return MOE_OK;
    for (const void* p : {static_cast<const void*>(x), static_cast<const void*>(W),
                          static_cast<const void*>(y)})
        if (!p || reinterpret_cast<uintptr_t>(p) % 16)
            return noalloc_fail(MOE_ERR_INVALID_ARGUMENT, "x, W and y must be 16-byte aligned, non-NULL");
    if (!ids || reinterpret_cast<uintptr_t>(ids) % 4)
        return noalloc_fail(MOE_ERR_INVALID_ARGUMENT, "ids must be 4-byte aligned, non-NULL");

    // Carve the expert map out of the static scratch.
    const long long max_tiles = rows / moe::kTileRows + 1 + (rows < n_experts ? rows : n_experts);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t o_status = take(sizeof(int));  // the first carve: kStatusOffset
    const size_t o_counts = take(sizeof(int) * n_experts);
    const size_t o_offsets = take(sizeof(int) * (n_experts + 1));
    const size_t o_perm = take(sizeof(int) * rows);
    const size_t o_inv = take(sizeof(int) * rows);
    const size_t o_tiles = take(sizeof(int4) * max_tiles);
    const size_t o_ntiles = take(sizeof(int));
    const size_t o_active = take(sizeof(int) * n_experts);
    const size_t o_nactive = take(sizeof(int));
    if (off > kNoallocScratchBytes)
        return noalloc_fail(MOE_ERR_UNSUPPORTED_SHAPE, "shape needs more than the 64 KiB static scratch");

    void* base = nullptr;
    cudaError_t err = scratch_address(&base);
    if (err != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, cudaGetErrorString(err));
    char* b = static_cast<char*>(base);
    moe::MapBuffers mb;
    mb.status = reinterpret_cast<int*>(b + o_status);
    mb.counts = reinterpret_cast<int*>(b + o_counts);
    mb.offsets = reinterpret_cast<int*>(b + o_offsets);
    mb.perm = reinterpret_cast<int*>(b + o_perm);
    mb.inv_perm = reinterpret_cast<int*>(b + o_inv);
    mb.chunk_hist = nullptr;  // not used by the fused single-block map
    mb.chunk_base = nullptr;
    mb.tiles = reinterpret_cast<int4*>(b + o_tiles);
    mb.n_tiles = reinterpret_cast<int*>(b + o_ntiles);
    mb.active = reinterpret_cast<int*>(b + o_active);
    mb.n_active = reinterpret_cast<int*>(b + o_nactive);

    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The status word must start at zero; it keeps the previous call's value.
    err = cudaMemsetAsync(mb.status, 0, sizeof(int), s);
    if (err != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, cudaGetErrorString(err));
    err = moe::launch_expert_map(ids, static_cast<int>(rows), n_experts, moe::kTileRows, mb, s);
    if (err != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, cudaGetErrorString(err));
    err = moe::launch_stream_matmul_id(reinterpret_cast<const __nv_bfloat16*>(x),
                                       reinterpret_cast<const __nv_bfloat16*>(W), y, m, n, k,
                                       top_k, n_experts, layout,
                                       static_cast<size_t>(n) * k, mb, s);
    if (err != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, cudaGetErrorString(err));
    return MOE_OK;
}

MOE_API moe_status_t moe_matmul_id_noalloc_status(void* stream) {
    moe::set_last_error("");
    void* base = nullptr;
    cudaError_t err = scratch_address(&base);
    if (err != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, cudaGetErrorString(err));
    int v = 0;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    err = cudaMemcpyAsync(&v, static_cast<char*>(base) + kStatusOffset, sizeof v,
                          cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return noalloc_fail(MOE_ERR_CUDA, cudaGetErrorString(err));
    if (v == MOE_OK) return MOE_OK;
    if (v == MOE_ERR_DEVICE_BAD_ID)
        return noalloc_fail(v, "an expert id was outside [0, n_experts)");
    if (v == MOE_ERR_DEVICE_TIMEOUT) return noalloc_fail(v, "a kernel wait exceeded its time limit");
    return noalloc_fail(MOE_ERR_CUDA, "unknown device status");
}

}  // extern "C"
