// Device helpers for sm_100a: mbarriers with bounded waits, TMA tensor
// tile copies, cp.async gathers, tcgen05 tensor-memory allocation, MMA,
// commit and loads.  Inline PTX only; no library templates.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

// Status word values written by kernels (same numbers as the C ABI).
constexpr int kDevOk = MOE_OK;
constexpr int kDevTimeout = MOE_ERR_DEVICE_TIMEOUT;
constexpr int kDevBadId = MOE_ERR_DEVICE_BAD_ID;
constexpr int kDevRange = MOE_ERR_DEVICE_RANGE;

// Default limit of one barrier wait: long enough for any legitimate wait on a
// loaded GPU, short enough that a broken pipeline returns instead of hanging.
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s
// Second, clock-independent bound on the number of polls of one wait.
constexpr uint64_t kMaxWaitPolls = 1ull << 28;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Records the first error of a call; later errors keep the first one.
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Suspend-time hint of one poll: a waiting thread sleeps until the phase
// completes or this many nanoseconds pass, instead of spinning (fewer issued
// instructions, less power on a power-capped part; no added wake-up latency).
constexpr uint32_t kPollSuspendNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kPollSuspendNs)
        : "memory");
    return done != 0;
}

// Shared state of one CTA's bounded waits: the first wait that gives up sets
// `abort`, records MOE_ERR_DEVICE_TIMEOUT, and every other wait in the CTA
// then returns false at its next poll, so all roles leave their loops.
struct WaitCtl {
    volatile int* abort;  // in shared memory
    int* status;          // global status word (may be null)
    uint64_t limit_ns;
};

// Waits until the phase with the given parity has completed.  Returns false
// (without completing) if the CTA aborted or the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t start = global_timer_ns();
    for (uint64_t polls = 1;; ++polls) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*ctl.abort) return false;
        if ((polls & 63) == 0) {
            if (global_timer_ns() - start > ctl.limit_ns || polls > kMaxWaitPolls) {
                *ctl.abort = 1;
                set_status(ctl.status, kDevTimeout);
                return false;
            }
        }
    }
}

// Wait used only while tearing down after an abort: bounded, never flags.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t start = global_timer_ns();
    for (uint64_t polls = 0; polls < kMaxWaitPolls; ++polls) {
        if (mbar_try_wait(bar, parity)) return;
        if ((polls & 63) == 0 && global_timer_ns() - start > limit_ns) return;
    }
}

// ----------------------------------------------------------------- TMA
// 2-D tiled bulk tensor copy global -> shared, completion on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// 3-D tiled bulk tensor copy global -> shared (e.g. a [E, n, k] weight stack
// whose experts sit at a padded stride).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// ----------------------------------------------------------------- cp.async
// 16-byte global -> shared copy through the load/store unit; src_bytes < 16
// zero-fills the rest (0 reads nothing).
__device__ __forceinline__ void cp_async_16(uint32_t dst_smem, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// Arrives on `bar` once every cp.async this thread issued so far has landed.
// The barrier's expected count must include this arrival (.noinc).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Orders this thread's view of generic-proxy shared-memory writes before its
// later async-proxy (tensor core, TMA) accesses.
// bf16 x 8 -> fp16 x 8, round to nearest even, element order kept (the
// down projection's weight conversion: in shared memory by the down kernel,
// or once per expert by w_down_fp16_kernel; both give the same values).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 v) {
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __half2 h = __floats2half2_rn(__uint_as_float(in[q] << 16),
                                            __uint_as_float(in[q] & 0xffff0000u));
        out[q] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------- streaming
// 16-byte read-only load that does not allocate in L1 (weights streamed once).
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 8 packed bf16 -> 8 f32 (exact).
__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, f32 accumulator.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on `bar` when every MMA this thread issued so far has finished.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 consecutive f32 columns from tensor memory (one row per lane).
__device__ __forceinline__ void tmem_load_32cols(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_load_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major bf16 tile stored as rows of
// 128 bytes (64 elements) with the 128-byte swizzle; 8-row groups are 1024 B
// apart.  The tile base must be 1024-byte aligned; advancing K by 16 elements
// inside the 128-byte row adds 32 bytes to the start address.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address >> 4
    d |= static_cast<uint64_t>(1) << 16;                       // leading offset (unused here)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride offset: 8 rows
    d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16 with bf16 A/B, f32 D, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(uint32_t M, uint32_t N) {
    return (1u << 4)            // D format f32
           | (1u << 7)          // A format bf16
           | (1u << 10)         // B format bf16
           | ((N >> 3) << 17)   // N / 8
           | ((M >> 4) << 24);  // M / 16
}

// Instruction descriptor: kind::f16 with fp16 A/B, f32 D, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_f16_f32(uint32_t M, uint32_t N) {
    return (1u << 4)            // D format f32 (A and B formats 0: fp16)
           | ((N >> 3) << 17)   // N / 8
           | ((M >> 4) << 24);  // M / 16
}

// Expert map of a few routed rows (rows <= blockDim.x) built by one block in
// shared memory: s_perm lists the routed rows in the stable order by
// (expert id, routed row); group g (g < *n_groups) holds the rows of expert
// s_gexp[g] at sorted positions s_gfirst[g] .. + s_gcnt[g].  s_warp has one
// int per warp of the block.  Returns false (and builds nothing) when an id
// lies outside [0, n_experts).  Every thread of the block must call it.
__device__ __forceinline__ bool block_small_map(const int* __restrict__ ids, int rows,
                                                int n_experts, int* s_id, int* s_perm,
                                                int* s_gexp, int* s_gfirst, int* s_gcnt,
                                                int* s_warp, int* s_flag, int* n_groups) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, n_warps = blockDim.x >> 5;
    if (tid == 0) *s_flag = 0;
    __syncthreads();
    int my_id = 0;
    if (tid < rows) {
        my_id = ids[tid];
        if (my_id < 0 || my_id >= n_experts) *s_flag = 1;
        s_id[tid] = my_id;
    }
    __syncthreads();
    if (*s_flag) return false;  // block-uniform
    if (tid < rows) {
        int rank = 0;
        for (int r2 = 0; r2 < rows; ++r2) {
            const int v = s_id[r2];
            rank += (v < my_id) || (v == my_id && r2 < tid);
        }
        s_perm[rank] = tid;
    }
    __syncthreads();
    int start = 0, e_here = 0;
    if (tid < rows) {
        e_here = s_id[s_perm[tid]];
        start = (tid == 0 || s_id[s_perm[tid - 1]] != e_here) ? 1 : 0;
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, start);
    if (lane == 0) s_warp[warp] = __popc(ballot);
    __syncthreads();
    int base = 0, total = 0;
    for (int w = 0; w < n_warps; ++w) {
        if (w < warp) base += s_warp[w];
        total += s_warp[w];
    }
    if (start) {
        const int g = base + __popc(ballot & ((1u << lane) - 1u));
        s_gexp[g] = e_here;
        s_gfirst[g] = tid;
    }
    __syncthreads();
    if (tid < total) s_gcnt[tid] = (tid + 1 < total ? s_gfirst[tid + 1] : rows) - s_gfirst[tid];
    *n_groups = total;
    __syncthreads();
    return true;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace moe
