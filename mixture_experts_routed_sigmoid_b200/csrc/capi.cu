// C ABI of the library: host-side validation, workspace layout, tensor-map
// encoding and the launch sequence of each entry point.  Never allocates,
// never synchronises the host (except moe_check_status), launches only on
// the caller's stream.
//
// Argument conventions follow the pages' boundary checks: fail closed before
// any GPU work, checked size products, dtype/shape/zero-size rejection
// [mlx-native 0.13.0, src/ops/dense_matmul_id_auto.rs: validate_cases,
// checked_product; hf2q 0.1.1 eagle3/forward.rs projection boundary checks],
// and caller-owned scratch sized once [hf2q qwen35/dense_ffn_arena.rs,
// MoeFfnArena lifetime contract].
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "device_common.cuh"
#include "launch.h"
#include "moe_b200.h"

namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_stage_events[8] = {};
thread_local int g_n_stage_events = 0;

// Records stage event i on the stream when the caller registered events.
void stage_mark(int i, cudaStream_t stream) {
    if (i < g_n_stage_events && g_stage_events[i]) cudaEventRecord(g_stage_events[i], stream);
}

moe_status_t fail(moe_status_t code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

moe_status_t ok() {
    g_last_error.clear();
    return MOE_OK;
}

moe_status_t cuda_fail(cudaError_t err, const char* what) {
    return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

constexpr size_t kAlign = 256;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Carver {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t o = off;
        off += round_up(bytes, kAlign);
        return o;
    }
};

// Offsets of the expert map's buffers inside a workspace.
struct MapLayout {
    size_t status, counts, offsets, perm, inv_perm, chunk_hist, chunk_base, tiles, n_tiles, active,
        n_active, end;
};

long long max_tiles(long long rows, int n_experts) {
    return rows / moe::kTileRows + 1 + (rows < n_experts ? rows : n_experts);
}

MapLayout map_layout(long long rows, int n_experts, bool own_outputs, Carver& c) {
    MapLayout L{};
    const long long n_chunks = (rows + moe::kMapChunkRows - 1) / moe::kMapChunkRows;
    L.status = c.take(sizeof(int));
    if (own_outputs) {
        L.counts = c.take(sizeof(int) * n_experts);
        L.offsets = c.take(sizeof(int) * (n_experts + 1));
        L.perm = c.take(sizeof(int) * rows);
        L.inv_perm = c.take(sizeof(int) * rows);
    }
    L.chunk_hist = c.take(sizeof(int) * n_chunks * n_experts);
    L.chunk_base = c.take(sizeof(int) * n_chunks * n_experts);
    L.tiles = c.take(sizeof(int4) * max_tiles(rows, n_experts));
    L.n_tiles = c.take(sizeof(int));
    L.active = c.take(sizeof(int) * n_experts);
    L.n_active = c.take(sizeof(int));
    L.end = c.off;
    return L;
}

moe::MapBuffers map_buffers(void* ws, const MapLayout& L, int* counts, int* offsets, int* perm,
                            int* inv_perm) {
    char* b = static_cast<char*>(ws);
    moe::MapBuffers m;
    m.status = reinterpret_cast<int*>(b + L.status);
    m.counts = counts ? counts : reinterpret_cast<int*>(b + L.counts);
    m.offsets = offsets ? offsets : reinterpret_cast<int*>(b + L.offsets);
    m.perm = perm ? perm : reinterpret_cast<int*>(b + L.perm);
    m.inv_perm = inv_perm ? inv_perm : reinterpret_cast<int*>(b + L.inv_perm);
    m.chunk_hist = reinterpret_cast<int*>(b + L.chunk_hist);
    m.chunk_base = reinterpret_cast<int*>(b + L.chunk_base);
    m.tiles = reinterpret_cast<int4*>(b + L.tiles);
    m.n_tiles = reinterpret_cast<int*>(b + L.n_tiles);
    m.active = reinterpret_cast<int*>(b + L.active);
    m.n_active = reinterpret_cast<int*>(b + L.n_active);
    return m;
}

struct FfnLayout {
    MapLayout map;
    size_t act, y_slots, conv_slot, w16, end;
    int n_slots;  // experts whose W_down the grouped path converts to fp16 up front
};

// An expert pass's buffers after its map: the activation (fp16 [rows, inter]
// on the grouped path, f32 on the streaming path), the per-slot rows
// [rows, hidden] f32 and, on the grouped path, the slots of the up-front
// fp16 W_down copies (conv_slot [E] and w16 [n_slots, hidden, inter]).
void carve_ffn_buffers(FfnLayout& L, Carver& c, long long rows, int hidden, int inter,
                       int n_experts) {
    L.act = c.take(sizeof(float) * rows * inter);
    L.y_slots = c.take(sizeof(float) * rows * hidden);
    const long long fit = rows / moe::kPreconvMinRows;
    L.n_slots = rows > moe::kStreamFfnMaxRows ? static_cast<int>(fit < n_experts ? fit : n_experts) : 0;
    L.conv_slot = L.n_slots ? c.take(sizeof(int) * n_experts) : 0;
    L.w16 = L.n_slots ? c.take(sizeof(uint16_t) * static_cast<size_t>(L.n_slots) * hidden * inter) : 0;
    L.end = c.off;
}

FfnLayout ffn_layout(long long rows, int hidden, int inter, int n_experts) {
    Carver c;
    FfnLayout L;
    L.map = map_layout(rows, n_experts, true, c);
    carve_ffn_buffers(L, c, rows, hidden, inter, n_experts);
    return L;
}

// ---------------------------------------------------------------- validation
moe_status_t check_routing_shape(long long m, int n_experts, int top_k) {
    if (m < 0) return fail(MOE_ERR_INVALID_ARGUMENT, "m must be >= 0 (got %lld)", m);
    if (n_experts < 1 || n_experts > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_experts must be in [1, %d] (got %d)",
                    MOE_MAX_EXPERTS, n_experts);
    if (top_k < 1 || top_k > n_experts || top_k > MOE_MAX_TOP_K)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "top_k must be in [1, min(n_experts, %d)] (got %d)",
                    MOE_MAX_TOP_K, top_k);
    if (m * top_k > MOE_MAX_ROUTED_ROWS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "m*top_k must be <= %d (got %lld)",
                    MOE_MAX_ROUTED_ROWS, m * top_k);
    return MOE_OK;
}

moe_status_t check_ptr(const void* p, const char* name, size_t align) {
    if (!p) return fail(MOE_ERR_INVALID_ARGUMENT, "%s must not be NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % align)
        return fail(MOE_ERR_INVALID_ARGUMENT, "%s must be %zu-byte aligned", name, align);
    return MOE_OK;
}

moe_status_t check_k(long long k, const char* name) {
    if (k < 8 || k % 8)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s must be a positive multiple of 8 (got %lld)",
                    name, k);
    if (k > (1 << 20)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s too large (got %lld)", name, k);
    return MOE_OK;
}

moe_status_t check_ws(const void* ws, size_t ws_bytes, size_t need) {
    moe_status_t s = check_ptr(ws, "ws", kAlign);
    if (s) return s;
    if (ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", ws_bytes,
                    need);
    return MOE_OK;
}

#define MOE_TRY(expr)                 \
    do {                              \
        moe_status_t _s = (expr);     \
        if (_s != MOE_OK) return _s;  \
    } while (0)

// ---------------------------------------------------------------- device info
int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        cache[dev] = v;
    }
    return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D 16-bit tensor [outer, inner] (inner contiguous; bf16 unless `dtype`
// says fp16) copied in boxes of box_outer rows x 64 columns with the 128-byte
// swizzle.
moe_status_t make_map(CUtensorMap* map, const void* base, unsigned long long inner,
                      unsigned long long outer, unsigned box_outer, const char* name,
                      CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    auto fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {64, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", name,
                    static_cast<int>(r));
    return MOE_OK;
}

// 3-D bf16 tensor [outer, mid, inner] whose outer index steps by
// outer_stride_bytes (a padded expert stride), copied in boxes of one outer
// slice x box_mid rows x 64 columns with the 128-byte swizzle.  Rows past
// `mid` inside a slice read as zeros, so a box never reaches into padding.
moe_status_t make_map_3d(CUtensorMap* map, const void* base, unsigned long long inner,
                         unsigned long long mid, unsigned long long outer,
                         unsigned long long outer_stride_bytes, unsigned box_mid,
                         const char* name) {
    auto fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[3] = {inner, mid, outer};
    const cuuint64_t strides[2] = {inner * 2, outer_stride_bytes};
    const cuuint32_t box[3] = {64, box_mid, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", name,
                    static_cast<int>(r));
    return MOE_OK;
}

moe_status_t run_map(const int32_t* ids, long long rows, int n_experts,
                     const moe::MapBuffers& b, cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(b.status, 0, sizeof(int), stream);
    if (err != cudaSuccess) return cuda_fail(err, "status reset");
    err = moe::launch_expert_map(ids, static_cast<int>(rows), n_experts, moe::kTileRows, b, stream);
    if (err != cudaSuccess) return cuda_fail(err, "expert map launch");
    return MOE_OK;
}

}  // namespace

namespace moe {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace moe

extern "C" {

MOE_API const char* moe_last_error(void) { return g_last_error.c_str(); }

MOE_API const char* moe_version(void) { return "moe_b200 0.1.0 (sm_100a)"; }

MOE_API moe_status_t moe_route_topk(const float* logits, const float* bias, int32_t m,
                                    int32_t n_experts, int32_t top_k, int32_t* ids,
                                    float* weights, float* scores, void* stream) {
    MOE_TRY(check_routing_shape(m, n_experts, top_k));
    if (m == 0) return ok();
    MOE_TRY(check_ptr(logits, "logits", 4));
    MOE_TRY(check_ptr(ids, "ids", 4));
    MOE_TRY(check_ptr(weights, "weights", 4));
    if (bias) MOE_TRY(check_ptr(bias, "bias", 4));
    if (scores) MOE_TRY(check_ptr(scores, "scores", 4));
    const cudaError_t err = moe::launch_route_topk(logits, bias, m, n_experts, top_k, ids, weights,
                                                   scores, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "route launch");
    return ok();
}

MOE_API moe_status_t moe_route_weights(const float* logits, const int32_t* ids, int32_t m,
                                       int32_t n_experts, int32_t top_k, float* weights,
                                       void* stream) {
    MOE_TRY(check_routing_shape(m, n_experts, top_k));
    if (m == 0) return ok();
    MOE_TRY(check_ptr(logits, "logits", 4));
    MOE_TRY(check_ptr(ids, "ids", 4));
    MOE_TRY(check_ptr(weights, "weights", 4));
    const cudaError_t err = moe::launch_route_weights(logits, ids, m, n_experts, top_k, weights,
                                                      static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "route weights launch");
    return ok();
}

// K ranges of the router projection: enough 256-column output tiles x K
// ranges to cover a B200's 148 SMs, at least 4 k-blocks (256 columns of K)
// per range, at most 8 ranges.  A function of the shape alone, so the
// partial sums, and with them the logits' bits, do not depend on the device.
int router_k_splits(long long m, int hidden, int n_experts) {
    const long long tiles = ((m + moe::kTileRows - 1) / moe::kTileRows) * ((n_experts + 255) / 256);
    const long long by_sms = tiles > 0 ? 148 / tiles : 1;
    const long long by_k = (hidden + 63) / 64 / 4;
    long long s = by_sms < by_k ? by_sms : by_k;
    if (s > 8) s = 8;
    return s < 1 ? 1 : static_cast<int>(s);
}

MOE_API size_t moe_router_workspace(int32_t m, int32_t hidden, int32_t n_experts) {
    if (m < 0 || hidden < 0 || n_experts < 1) return kAlign;
    const int s = router_k_splits(m, hidden, n_experts);
    // the status word, then the partial slabs [s, m, n_experts] f32 when split
    return kAlign + (s > 1 ? round_up(sizeof(float) * s * static_cast<size_t>(m) * n_experts, kAlign)
                           : 0);
}

MOE_API moe_status_t moe_router_topk(const moe_bf16_t* x, const moe_bf16_t* W_router,
                                     const float* bias, int32_t m, int32_t hidden,
                                     int32_t n_experts, int32_t top_k, float* logits,
                                     int32_t* ids, float* weights, void* ws, size_t ws_bytes,
                                     void* stream) {
    MOE_TRY(check_routing_shape(m, n_experts, top_k));
    MOE_TRY(check_k(hidden, "hidden"));
    if (m == 0) return ok();
    MOE_TRY(check_ptr(x, "x", 16));
    MOE_TRY(check_ptr(W_router, "W_router", 16));
    MOE_TRY(check_ptr(logits, "logits", 16));
    MOE_TRY(check_ptr(ids, "ids", 4));
    MOE_TRY(check_ptr(weights, "weights", 4));
    if (bias) MOE_TRY(check_ptr(bias, "bias", 4));
    MOE_TRY(check_ws(ws, ws_bytes, moe_router_workspace(m, hidden, n_experts)));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = static_cast<int*>(ws);
    cudaError_t err = cudaMemsetAsync(status, 0, sizeof(int), s);
    if (err != cudaSuccess) return cuda_fail(err, "status reset");
    const int splits = router_k_splits(m, hidden, n_experts);
    float* parts = splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + kAlign) : logits;
    CUtensorMap map_x, map_w;
    MOE_TRY(make_map(&map_x, x, hidden, m, 128, "x"));
    MOE_TRY(make_map(&map_w, W_router, hidden, n_experts, 256, "W_router"));
    moe::GroupedGemmArgs a{};
    a.out = parts;
    a.status = status;
    a.status_out = status;
    a.rows = m;
    a.n = n_experts;
    a.k = hidden;
    a.n_col_tiles = (n_experts + 255) / 256;  // 256-column tiles
    a.dense_m_tiles = (m + moe::kTileRows - 1) / moe::kTileRows;
    a.k_splits = splits;
    a.wait_limit_ns = moe::kDefaultWaitLimitNs;
    err = moe::launch_grouped_gemm(4, map_x, map_w, map_w, a, num_sms(), s);
    if (err != cudaSuccess) return cuda_fail(err, "router projection launch");
    err = moe::launch_route_topk(parts, bias, m, n_experts, top_k, ids, weights, nullptr, s, splits,
                                 logits);
    if (err != cudaSuccess) return cuda_fail(err, "route launch");
    return ok();
}

MOE_API size_t moe_expert_map_workspace(int32_t m, int32_t top_k, int32_t n_experts) {
    if (check_routing_shape(m, n_experts, top_k) != MOE_OK) return 0;
    Carver c;
    return map_layout(static_cast<long long>(m) * top_k, n_experts, false, c).end;
}

MOE_API moe_status_t moe_expert_map(const int32_t* ids, int32_t m, int32_t top_k,
                                    int32_t n_experts, int32_t* counts, int32_t* offsets,
                                    int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes,
                                    void* stream) {
    MOE_TRY(check_routing_shape(m, n_experts, top_k));
    if (m == 0) return ok();
    MOE_TRY(check_ptr(ids, "ids", 4));
    MOE_TRY(check_ptr(counts, "counts", 4));
    MOE_TRY(check_ptr(offsets, "offsets", 4));
    MOE_TRY(check_ptr(perm, "perm", 4));
    MOE_TRY(check_ptr(inv_perm, "inv_perm", 4));
    const long long rows = static_cast<long long>(m) * top_k;
    Carver c;
    const MapLayout L = map_layout(rows, n_experts, false, c);
    MOE_TRY(check_ws(ws, ws_bytes, L.end));
    const moe::MapBuffers b = map_buffers(ws, L, counts, offsets, perm, inv_perm);
    MOE_TRY(run_map(ids, rows, n_experts, b, static_cast<cudaStream_t>(stream)));
    return ok();
}

MOE_API size_t moe_matmul_id_workspace(int32_t m, int32_t n, int32_t k, int32_t top_k,
                                       int32_t n_experts, int32_t layout) {
    (void)n;
    (void)k;
    (void)layout;
    if (check_routing_shape(m, n_experts, top_k) != MOE_OK) return 0;
    Carver c;
    return map_layout(static_cast<long long>(m) * top_k, n_experts, true, c).end;
}

}  // extern "C"

namespace {

// Shared body of moe_matmul_id and moe_matmul_id_strided; stride_bytes = 0
// means the dense stack (expert e at W + e * n * k).
moe_status_t matmul_id_impl(const moe_bf16_t* x, const int32_t* ids, const moe_bf16_t* W, float* y,
                            int32_t m, int32_t n, int32_t k, int32_t top_k, int32_t n_experts,
                            int32_t layout, unsigned long long stride_bytes, void* ws,
                            size_t ws_bytes, void* stream) {
    MOE_TRY(check_routing_shape(m, n_experts, top_k));
    if (layout != MOE_LAYOUT_SHARED_PER_TOKEN && layout != MOE_LAYOUT_SLOTTED)
        return fail(MOE_ERR_INVALID_ARGUMENT, "layout must be 0 or 1 (got %d)", layout);
    if (n < 1 || n > (1 << 20)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n must be in [1, 2^20] (got %d)", n);
    MOE_TRY(check_k(k, "k"));
    const unsigned long long dense_bytes = 2ull * static_cast<unsigned long long>(n) * k;
    if (stride_bytes) {
        if (stride_bytes < dense_bytes)
            return fail(MOE_ERR_INVALID_ARGUMENT,
                        "expert_stride_bytes %llu is below one expert's n*k*2 = %llu bytes",
                        stride_bytes, dense_bytes);
        if (stride_bytes % 16)
            return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                        "expert_stride_bytes must be a multiple of 16 (got %llu)", stride_bytes);
        if (stride_bytes >= (1ull << 40))
            return fail(MOE_ERR_UNSUPPORTED_SHAPE, "expert_stride_bytes too large (got %llu)",
                        stride_bytes);
    }
    if (m == 0) return ok();
    MOE_TRY(check_ptr(x, "x", 16));
    MOE_TRY(check_ptr(ids, "ids", 4));
    MOE_TRY(check_ptr(W, "W", 16));
    MOE_TRY(check_ptr(y, "y", 16));
    const long long rows = static_cast<long long>(m) * top_k;
    Carver c;
    const MapLayout L = map_layout(rows, n_experts, true, c);
    MOE_TRY(check_ws(ws, ws_bytes, L.end));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const moe::MapBuffers b = map_buffers(ws, L, nullptr, nullptr, nullptr, nullptr);
    const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    const auto* Wb = reinterpret_cast<const __nv_bfloat16*>(W);
    if (rows <= moe::kStreamMaxRows) {
        // one launch: the kernel builds the expert map itself and writes the
        // status word
        const size_t w_stride = stride_bytes ? static_cast<size_t>(stride_bytes / 2)
                                             : static_cast<size_t>(dense_bytes / 2);
        stage_mark(0, s);
        stage_mark(1, s);
        const cudaError_t err = moe::launch_stream_matmul_id_fused(
            xb, ids, Wb, y, m, n, k, top_k, n_experts, layout, w_stride, b.status, s);
        if (err != cudaSuccess) return cuda_fail(err, "streaming matmul_id launch");
        stage_mark(2, s);
        return ok();
    }
    stage_mark(0, s);
    MOE_TRY(run_map(ids, rows, n_experts, b, s));
    stage_mark(1, s);
    CUtensorMap map_w;
    if (stride_bytes)
        MOE_TRY(make_map_3d(&map_w, W, k, n, n_experts, stride_bytes, 256, "W"));
    else
        MOE_TRY(make_map(&map_w, W, k, static_cast<unsigned long long>(n_experts) * n, 256, "W"));
    moe::GroupedGemmArgs a{};
    a.a_ptr = xb;
    a.perm = b.perm;
    a.tiles = b.tiles;
    a.n_tiles = b.n_tiles;
    a.weights = nullptr;
    a.out = y;
    a.status = b.status;
    a.status_out = b.status;
    a.rows = rows;
    a.n = n;
    a.k = k;
    a.n_col_tiles = (n + 255) / 256;
    a.top_k = top_k;
    a.layout = layout;
    a.b_rows_per_expert = n;
    a.b_3d = stride_bytes ? 1 : 0;
    a.zero_fill_dead = rows <= moe::kZeroFillMaxRowsPerExpert * n_experts;
    a.wait_limit_ns = moe::kDefaultWaitLimitNs;
    const cudaError_t err = moe::launch_grouped_gemm(2, map_w, map_w, map_w, a, num_sms(), s);
    if (err != cudaSuccess) return cuda_fail(err, "grouped matmul_id launch");
    stage_mark(2, s);
    return ok();
}

}  // namespace

extern "C" {

MOE_API moe_status_t moe_matmul_id(const moe_bf16_t* x, const int32_t* ids, const moe_bf16_t* W,
                                   float* y, int32_t m, int32_t n, int32_t k, int32_t top_k,
                                   int32_t n_experts, int32_t layout, void* ws, size_t ws_bytes,
                                   void* stream) {
    return matmul_id_impl(x, ids, W, y, m, n, k, top_k, n_experts, layout, 0, ws, ws_bytes,
                          stream);
}

MOE_API moe_status_t moe_matmul_id_strided(const moe_bf16_t* x, const int32_t* ids,
                                           const moe_bf16_t* W, uint64_t expert_stride_bytes,
                                           float* y, int32_t m, int32_t n, int32_t k,
                                           int32_t top_k, int32_t n_experts, int32_t layout,
                                           void* ws, size_t ws_bytes, void* stream) {
    if (expert_stride_bytes == 0)
        return fail(MOE_ERR_INVALID_ARGUMENT, "expert_stride_bytes must be nonzero");
    return matmul_id_impl(x, ids, W, y, m, n, k, top_k, n_experts, layout, expert_stride_bytes,
                          ws, ws_bytes, stream);
}

MOE_API size_t moe_ffn_workspace(int32_t m, int32_t hidden, int32_t inter, int32_t top_k,
                                 int32_t n_experts, int32_t layout) {
    (void)layout;
    if (check_routing_shape(m, n_experts, top_k) != MOE_OK || hidden < 1 || inter < 1) return 0;
    return ffn_layout(static_cast<long long>(m) * top_k, hidden, inter, n_experts).end;
}

}  // extern "C"

namespace {

// One expert pass of the FFN: the map (from ids, or the one-expert map when
// ids is null), gate/up with SwiGLU, then down scaled by the row's weight
// into y_slots [rows, hidden].  `status` replaces the map's own status word
// when given (the shared expert reports into the routed call's word).
struct ExpertPass {
    const moe_bf16_t* x;
    const int32_t* ids;
    const float* weights;
    const moe_bf16_t* W_gate;
    const moe_bf16_t* W_up;
    const moe_bf16_t* W_down;
    int32_t m, hidden, inter, top_k, n_experts, layout;
};

moe_status_t run_expert_pass(const ExpertPass& f, char* wsb, const FfnLayout& L, int* status,
                             bool marks, cudaStream_t s, float* slots_out = nullptr) {
    const long long rows = static_cast<long long>(f.m) * f.top_k;
    moe::MapBuffers b = map_buffers(wsb, L.map, nullptr, nullptr, nullptr, nullptr);
    if (status) b.status = status;
    void* act = wsb + L.act;
    float* y_slots = slots_out ? slots_out : reinterpret_cast<float*>(wsb + L.y_slots);
    const auto mark = [&](int i) {
        if (marks) stage_mark(i, s);
    };
    const auto run_pass_map = [&]() -> moe_status_t {
        if (f.ids) return run_map(f.ids, rows, f.n_experts, b, s);
        const cudaError_t err = moe::launch_dense_map(static_cast<int>(rows), moe::kTileRows, b, s);
        if (err != cudaSuccess) return cuda_fail(err, "dense map launch");
        return MOE_OK;
    };

    if (rows <= moe::kStreamFfnMaxRows) {
        // Decode sizes: weight-streaming kernels (the act region holds the
        // f32 activation [rows, inter]; the grouped path uses half of it).
        // A routed pass builds its expert map inside the gate/up kernel.
        mark(0);
        if (!f.ids) MOE_TRY(run_pass_map());
        mark(1);
        const cudaError_t err = moe::launch_stream_ffn(
            reinterpret_cast<const __nv_bfloat16*>(f.x), f.weights,
            reinterpret_cast<const __nv_bfloat16*>(f.W_gate),
            reinterpret_cast<const __nv_bfloat16*>(f.W_up),
            reinterpret_cast<const __nv_bfloat16*>(f.W_down), static_cast<float*>(act), y_slots,
            f.m, f.hidden, f.inter, f.top_k, f.layout, b, s, f.ids, f.n_experts);
        if (err != cudaSuccess) return cuda_fail(err, "streaming FFN launch");
        mark(2);
        mark(3);
        return MOE_OK;
    }

    const unsigned long long E = static_cast<unsigned long long>(f.n_experts);
    CUtensorMap map_g, map_u, map_act, map_act64, map_d;
    MOE_TRY(make_map(&map_g, f.W_gate, f.hidden, E * f.inter, 128, "W_gate"));
    MOE_TRY(make_map(&map_u, f.W_up, f.hidden, E * f.inter, 128, "W_up"));
    // the fp16 activation [rows, inter] (expert-sorted rows)
    MOE_TRY(make_map(&map_act, act, f.inter, rows, 128, "act", CU_TENSOR_MAP_DATA_TYPE_FLOAT16));
    MOE_TRY(make_map(&map_act64, act, f.inter, rows, 64, "act",  // tiles of <= 64 rows
                     CU_TENSOR_MAP_DATA_TYPE_FLOAT16));
    MOE_TRY(make_map(&map_d, f.W_down, f.inter, E * f.hidden, 256, "W_down"));

    mark(0);
    MOE_TRY(run_pass_map());
    mark(1);

    moe::GroupedGemmArgs a{};
    a.a_ptr = reinterpret_cast<const __nv_bfloat16*>(f.x);
    a.perm = b.perm;
    a.tiles = b.tiles;
    a.n_tiles = b.n_tiles;
    a.status = b.status;
    a.status_out = b.status;
    a.rows = rows;
    a.top_k = f.top_k;
    a.layout = f.layout;
    a.wait_limit_ns = moe::kDefaultWaitLimitNs;
    a.zero_fill_dead = rows <= moe::kZeroFillMaxRowsPerExpert * f.n_experts;
    a.swap_small = 1;

    // gate/up + SwiGLU -> act (expert-sorted rows)
    a.out = act;
    a.n = f.inter;
    a.k = f.hidden;
    a.n_col_tiles = (f.inter + 127) / 128;
    a.b_rows_per_expert = f.inter;
    cudaError_t err = moe::launch_grouped_gemm(0, map_g, map_g, map_u, a, num_sms(), s);
    if (err != cudaSuccess) return cuda_fail(err, "gate/up launch");
    mark(2);

    // W_down of the experts with kPreconvMinRows or more rows -> fp16, once
    CUtensorMap map_w16;
    if (L.n_slots > 0) {
        int* conv_slot = reinterpret_cast<int*>(wsb + L.conv_slot);
        __half* w16 = reinterpret_cast<__half*>(wsb + L.w16);
        MOE_TRY(make_map(&map_w16, w16, f.inter,
                         static_cast<unsigned long long>(L.n_slots) * f.hidden, 256, "W_down fp16",
                         CU_TENSOR_MAP_DATA_TYPE_FLOAT16));
        err = moe::launch_w_down_fp16(reinterpret_cast<const __nv_bfloat16*>(f.W_down), b.counts,
                                      f.n_experts, static_cast<long long>(f.hidden) * f.inter,
                                      moe::kPreconvMinRows, L.n_slots, conv_slot, w16, b.status, s);
        if (err != cudaSuccess) return cuda_fail(err, "W_down fp16 launch");
        a.conv_slot = conv_slot;
    }

    // down + combine weight -> y_slots[t, j]
    a.out = y_slots;
    a.weights = f.weights;
    a.n = f.hidden;
    a.k = f.inter;
    a.n_col_tiles = (f.hidden + 255) / 256;
    a.b_rows_per_expert = f.hidden;
    err = moe::launch_grouped_gemm(1, map_act, map_d, map_act64, a, num_sms(), s,
                                   L.n_slots > 0 ? &map_w16 : nullptr);
    if (err != cudaSuccess) return cuda_fail(err, "down launch");
    mark(3);
    return MOE_OK;
}

moe_status_t check_ffn_args(const moe_bf16_t* x, const int32_t* ids, const float* weights,
                            const moe_bf16_t* W_gate, const moe_bf16_t* W_up,
                            const moe_bf16_t* W_down, const float* y, int32_t m, int32_t hidden,
                            int32_t inter, int32_t top_k, int32_t n_experts, int32_t layout,
                            bool with_weights = true) {
    MOE_TRY(check_routing_shape(m, n_experts, top_k));
    if (layout != MOE_LAYOUT_SHARED_PER_TOKEN && layout != MOE_LAYOUT_SLOTTED)
        return fail(MOE_ERR_INVALID_ARGUMENT, "layout must be 0 or 1 (got %d)", layout);
    MOE_TRY(check_k(hidden, "hidden"));
    MOE_TRY(check_k(inter, "inter"));
    if (m == 0) return MOE_OK;
    MOE_TRY(check_ptr(x, "x", 16));
    MOE_TRY(check_ptr(ids, "ids", 4));
    if (with_weights) MOE_TRY(check_ptr(weights, "weights", 4));
    MOE_TRY(check_ptr(W_gate, "W_gate", 16));
    MOE_TRY(check_ptr(W_up, "W_up", 16));
    MOE_TRY(check_ptr(W_down, "W_down", 16));
    MOE_TRY(check_ptr(y, "y", 16));
    return MOE_OK;
}

// The routed layer's workspace, then the shared expert's: its one-expert map,
// gate [m] f32, then its activation, gated rows [m, hidden] f32 and (for
// m >= 512 on the grouped path) the slot of its fp16 W_sh_down copy.
struct SharedFfnLayout {
    FfnLayout routed, shared;
    size_t gate, end;
};

SharedFfnLayout shared_ffn_layout(long long m, int top_k, int hidden, int inter, int inter_sh,
                                  int n_experts) {
    SharedFfnLayout L;
    L.routed = ffn_layout(m * top_k, hidden, inter, n_experts);
    Carver c;
    c.off = L.routed.end;
    L.shared.map = map_layout(m, 1, true, c);
    L.gate = c.take(sizeof(float) * m);
    carve_ffn_buffers(L.shared, c, m, hidden, inter_sh, 1);
    L.end = c.off;
    return L;
}

}  // namespace

extern "C" {

MOE_API moe_status_t moe_ffn_forward(const moe_bf16_t* x, const int32_t* ids,
                                     const float* weights, const moe_bf16_t* W_gate,
                                     const moe_bf16_t* W_up, const moe_bf16_t* W_down, float* y,
                                     int32_t m, int32_t hidden, int32_t inter, int32_t top_k,
                                     int32_t n_experts, int32_t layout, void* ws,
                                     size_t ws_bytes, void* stream) {
    MOE_TRY(check_ffn_args(x, ids, weights, W_gate, W_up, W_down, y, m, hidden, inter, top_k,
                           n_experts, layout));
    if (m == 0) return ok();
    const FfnLayout L = ffn_layout(static_cast<long long>(m) * top_k, hidden, inter, n_experts);
    MOE_TRY(check_ws(ws, ws_bytes, L.end));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* wsb = static_cast<char*>(ws);
    const ExpertPass f{x, ids, weights, W_gate, W_up, W_down, m, hidden, inter, top_k, n_experts,
                       layout};
    MOE_TRY(run_expert_pass(f, wsb, L, nullptr, true, s));
    const int* status = reinterpret_cast<const int*>(wsb + L.map.status);
    const cudaError_t err = moe::launch_combine(reinterpret_cast<const float*>(wsb + L.y_slots), y,
                                                m, hidden, top_k, nullptr, status, s);
    if (err != cudaSuccess) return cuda_fail(err, "combine launch");
    stage_mark(4, s);
    return ok();
}

MOE_API moe_status_t moe_ffn_slots(const moe_bf16_t* x, const int32_t* ids,
                                   const moe_bf16_t* W_gate, const moe_bf16_t* W_up,
                                   const moe_bf16_t* W_down, float* d_slots, int32_t m,
                                   int32_t hidden, int32_t inter, int32_t top_k,
                                   int32_t n_experts, int32_t layout, void* ws, size_t ws_bytes,
                                   void* stream) {
    MOE_TRY(check_ffn_args(x, ids, nullptr, W_gate, W_up, W_down, d_slots, m, hidden, inter,
                           top_k, n_experts, layout, false));
    if (m == 0) return ok();
    const FfnLayout L = ffn_layout(static_cast<long long>(m) * top_k, hidden, inter, n_experts);
    MOE_TRY(check_ws(ws, ws_bytes, L.end));
    const ExpertPass f{x, ids, nullptr, W_gate, W_up, W_down, m, hidden, inter, top_k, n_experts,
                       layout};
    MOE_TRY(run_expert_pass(f, static_cast<char*>(ws), L, nullptr, false,
                            static_cast<cudaStream_t>(stream), d_slots));
    return ok();
}

MOE_API size_t moe_ffn_shared_workspace(int32_t m, int32_t hidden, int32_t inter,
                                        int32_t inter_sh, int32_t top_k, int32_t n_experts) {
    if (check_routing_shape(m, n_experts, top_k) != MOE_OK || hidden < 1 || inter < 1 ||
        inter_sh < 1)
        return 0;
    return shared_ffn_layout(m, top_k, hidden, inter, inter_sh, n_experts).end;
}

MOE_API moe_status_t moe_ffn_forward_shared(
    const moe_bf16_t* x, const int32_t* ids, const float* weights, const moe_bf16_t* W_gate,
    const moe_bf16_t* W_up, const moe_bf16_t* W_down, const moe_bf16_t* w_sh,
    const moe_bf16_t* W_sh_gate, const moe_bf16_t* W_sh_up, const moe_bf16_t* W_sh_down, float* y,
    int32_t m, int32_t hidden, int32_t inter, int32_t inter_sh, int32_t top_k, int32_t n_experts,
    void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_ffn_args(x, ids, weights, W_gate, W_up, W_down, y, m, hidden, inter, top_k,
                           n_experts, MOE_LAYOUT_SHARED_PER_TOKEN));
    MOE_TRY(check_k(inter_sh, "inter_sh"));
    if (m == 0) return ok();
    MOE_TRY(check_ptr(w_sh, "w_sh", 16));
    MOE_TRY(check_ptr(W_sh_gate, "W_sh_gate", 16));
    MOE_TRY(check_ptr(W_sh_up, "W_sh_up", 16));
    MOE_TRY(check_ptr(W_sh_down, "W_sh_down", 16));
    const SharedFfnLayout L = shared_ffn_layout(m, top_k, hidden, inter, inter_sh, n_experts);
    MOE_TRY(check_ws(ws, ws_bytes, L.end));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* wsb = static_cast<char*>(ws);
    int* status = reinterpret_cast<int*>(wsb + L.routed.map.status);
    float* gate = reinterpret_cast<float*>(wsb + L.gate);

    // routed experts (the map resets the status word first)
    const ExpertPass routed{x, ids, weights, W_gate, W_up, W_down, m, hidden, inter, top_k,
                            n_experts, MOE_LAYOUT_SHARED_PER_TOKEN};
    MOE_TRY(run_expert_pass(routed, wsb, L.routed, nullptr, false, s));

    // shared expert gate: sigmoid(x . w_sh) per token
    CUtensorMap map_x, map_w;
    MOE_TRY(make_map(&map_x, x, hidden, m, 128, "x"));
    MOE_TRY(make_map(&map_w, w_sh, hidden, 1, 64, "w_sh"));
    moe::GroupedGemmArgs a{};
    a.out = gate;
    a.status = status;
    a.status_out = status;
    a.rows = m;
    a.n = 1;
    a.k = hidden;
    a.n_col_tiles = 1;
    a.dense_m_tiles = (m + moe::kTileRows - 1) / moe::kTileRows;
    a.out_sigmoid = 1;
    a.wait_limit_ns = moe::kDefaultWaitLimitNs;
    cudaError_t err = moe::launch_grouped_gemm(3, map_x, map_w, map_w, a, num_sms(), s);
    if (err != cudaSuccess) return cuda_fail(err, "shared gate launch");

    // shared expert: every token, weight = its gate
    const ExpertPass shared{x, nullptr, gate, W_sh_gate, W_sh_up, W_sh_down, m, hidden, inter_sh,
                            1, 1, MOE_LAYOUT_SHARED_PER_TOKEN};
    MOE_TRY(run_expert_pass(shared, wsb, L.shared, status, false, s));

    err = moe::launch_combine(reinterpret_cast<const float*>(wsb + L.routed.y_slots), y, m, hidden,
                              top_k, reinterpret_cast<const float*>(wsb + L.shared.y_slots),
                              status, s);
    if (err != cudaSuccess) return cuda_fail(err, "combine launch");
    return ok();
}

}  // extern "C"

namespace {

// Dispatch workspace: the expert map over owner ranks (status word first),
// then the owner rank of every routed row.
struct EpLayout {
    MapLayout map;
    size_t owner, end;
};

EpLayout ep_layout(long long rows, int n_ranks) {
    Carver c;
    EpLayout L;
    L.map = map_layout(rows, n_ranks, true, c);
    L.owner = c.take(sizeof(int) * rows);
    L.end = c.off;
    return L;
}

moe_status_t check_ep_shape(long long m, int hidden, int top_k, int n_experts, int n_ranks) {
    MOE_TRY(check_routing_shape(m, n_experts, top_k));
    MOE_TRY(check_k(hidden, "hidden"));
    if (n_ranks < 1 || n_ranks > n_experts)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_ranks must be in [1, n_experts] (got %d)", n_ranks);
    if (n_experts % n_ranks)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "n_experts (%d) must be a multiple of n_ranks (%d)", n_experts, n_ranks);
    return MOE_OK;
}

}  // namespace

extern "C" {

MOE_API size_t moe_ep_dispatch_workspace(int32_t m, int32_t top_k, int32_t n_ranks) {
    if (m < 0 || top_k < 1 || top_k > MOE_MAX_TOP_K || n_ranks < 1 || n_ranks > MOE_MAX_EXPERTS ||
        static_cast<long long>(m) * top_k > MOE_MAX_ROUTED_ROWS)
        return 0;
    return ep_layout(static_cast<long long>(m) * top_k, n_ranks).end;
}

MOE_API moe_status_t moe_ep_dispatch(const moe_bf16_t* x, const int32_t* ids, int32_t m,
                                     int32_t hidden, int32_t top_k, int32_t n_experts,
                                     int32_t n_ranks, int32_t layout, moe_bf16_t* send_x,
                                     int32_t* send_expert, int32_t* send_counts, void* ws,
                                     size_t ws_bytes, void* stream) {
    MOE_TRY(check_ep_shape(m, hidden, top_k, n_experts, n_ranks));
    if (layout != MOE_LAYOUT_SHARED_PER_TOKEN && layout != MOE_LAYOUT_SLOTTED)
        return fail(MOE_ERR_INVALID_ARGUMENT, "layout must be 0 or 1 (got %d)", layout);
    MOE_TRY(check_ptr(send_counts, "send_counts", 4));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (m == 0) {
        // nothing to send: the counts are all zero
        const cudaError_t err = cudaMemsetAsync(send_counts, 0, sizeof(int32_t) * n_ranks, s);
        if (err != cudaSuccess) return cuda_fail(err, "send_counts reset");
        return ok();
    }
    MOE_TRY(check_ptr(x, "x", 16));
    MOE_TRY(check_ptr(ids, "ids", 4));
    MOE_TRY(check_ptr(send_x, "send_x", 16));
    MOE_TRY(check_ptr(send_expert, "send_expert", 4));
    const long long rows = static_cast<long long>(m) * top_k;
    const EpLayout L = ep_layout(rows, n_ranks);
    MOE_TRY(check_ws(ws, ws_bytes, L.end));
    char* wsb = static_cast<char*>(ws);
    moe::MapBuffers b = map_buffers(ws, L.map, send_counts, nullptr, nullptr, nullptr);
    int* owner = reinterpret_cast<int*>(wsb + L.owner);
    cudaError_t err = cudaMemsetAsync(b.status, 0, sizeof(int), s);
    if (err != cudaSuccess) return cuda_fail(err, "status reset");
    const int per_rank = n_experts / n_ranks;
    err = moe::launch_ep_owner(ids, rows, n_experts, per_rank, owner, b.status, s);
    if (err != cudaSuccess) return cuda_fail(err, "owner launch");
    // The map's own status reset would clear a bad-id flag: launch its kernels directly.
    err = moe::launch_expert_map(owner, static_cast<int>(rows), n_ranks, moe::kTileRows, b, s);
    if (err != cudaSuccess) return cuda_fail(err, "owner map launch");
    err = moe::launch_ep_pack(reinterpret_cast<const __nv_bfloat16*>(x), ids, b.perm, rows, hidden,
                              top_k, layout, per_rank, reinterpret_cast<__nv_bfloat16*>(send_x),
                              send_expert, b.status, s);
    if (err != cudaSuccess) return cuda_fail(err, "pack launch");
    return ok();
}

MOE_API moe_status_t moe_ep_combine(const float* d_back, const float* weights, float* y, int32_t m,
                                    int32_t hidden, int32_t top_k, int32_t n_ranks,
                                    const void* ws, size_t ws_bytes, void* stream) {
    if (m < 0) return fail(MOE_ERR_INVALID_ARGUMENT, "m must be >= 0 (got %d)", m);
    if (top_k < 1 || top_k > MOE_MAX_TOP_K)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "top_k must be in [1, %d] (got %d)", MOE_MAX_TOP_K,
                    top_k);
    if (n_ranks < 1 || n_ranks > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_ranks must be in [1, %d] (got %d)",
                    MOE_MAX_EXPERTS, n_ranks);
    MOE_TRY(check_k(hidden, "hidden"));
    if (static_cast<long long>(m) * top_k > MOE_MAX_ROUTED_ROWS)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "m*top_k must be <= %d", MOE_MAX_ROUTED_ROWS);
    if (m == 0) return ok();
    MOE_TRY(check_ptr(d_back, "d_back", 16));
    MOE_TRY(check_ptr(weights, "weights", 4));
    MOE_TRY(check_ptr(y, "y", 16));
    const long long rows = static_cast<long long>(m) * top_k;
    const EpLayout L = ep_layout(rows, n_ranks);
    MOE_TRY(check_ws(ws, ws_bytes, L.end));
    const char* wsb = static_cast<const char*>(ws);
    const cudaError_t err = moe::launch_ep_combine(
        d_back, reinterpret_cast<const int*>(wsb + L.map.inv_perm), weights, y, m, hidden, top_k,
        reinterpret_cast<const int*>(wsb + L.map.status), static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "combine launch");
    return ok();
}

MOE_API moe_status_t moe_set_stage_events(void* const* events, int32_t n_events) {
    if (!events) {
        g_n_stage_events = 0;
        return ok();
    }
    if (n_events < 5 || n_events > 8)
        return fail(MOE_ERR_INVALID_ARGUMENT, "n_events must be in [5, 8] (got %d)", n_events);
    for (int i = 0; i < n_events; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_n_stage_events = n_events;
    return ok();
}

MOE_API moe_status_t moe_check_status(const void* ws, void* stream) {
    MOE_TRY(check_ptr(ws, "ws", kAlign));
    int v = 0;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The status word is the first field of every workspace layout.
    cudaError_t err = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return cuda_fail(err, "status read");
    if (v == MOE_OK) return ok();
    if (v == MOE_ERR_DEVICE_BAD_ID) return fail(v, "an expert id was outside [0, n_experts)");
    if (v == MOE_ERR_DEVICE_TIMEOUT) return fail(v, "a kernel wait exceeded its time limit");
    if (v == MOE_ERR_DEVICE_RANGE)
        return fail(v, "the fp16 down projection gave a non-finite value: an activation above "
                       "65504 * 16, a W_down entry of 65536 or more, or a non-finite input");
    return fail(MOE_ERR_CUDA, "unknown device status %d", v);
}

MOE_API moe_status_t moe_clock_probe(uint64_t* out, int32_t n_blocks, void* stream) {
    MOE_TRY(check_ptr(out, "out", 8));
    if (n_blocks < 1 || n_blocks > 4096)
        return fail(MOE_ERR_INVALID_ARGUMENT, "n_blocks must be in [1, 4096] (got %d)", n_blocks);
    const cudaError_t err = moe::launch_clock_probe(reinterpret_cast<unsigned long long*>(out),
                                                    n_blocks, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "clock probe launch");
    return ok();
}

MOE_API moe_status_t moe_selftest_wait_timeout(int32_t* status_word, int64_t limit_ns,
                                               void* stream) {
    MOE_TRY(check_ptr(status_word, "status_word", 4));
    if (limit_ns < 1 || limit_ns > 1000000000LL)
        return fail(MOE_ERR_INVALID_ARGUMENT, "limit_ns must be in [1, 1e9]");
    const cudaError_t err = moe::launch_wait_timeout_selftest(
        status_word, static_cast<unsigned long long>(limit_ns), static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "self-test launch");
    return ok();
}

}  // extern "C"
