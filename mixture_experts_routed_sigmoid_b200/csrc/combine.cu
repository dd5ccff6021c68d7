// Ordered, atomic-free combine of the weighted per-slot rows, the clock
// probe used to measure the SM clock over a timed region, and the
// bounded-wait self-test kernel.
//
// Combine [hf2q, qwen35/dense_ffn_arena.rs: MoeFfnArena holds y_all
// [seq*topk, h] and the layer ends with a weighted reduce over the top-k
// slots; cortiq-engine src/mimo_moe.rs tests::exact_moe sums w*down(...) over
// the picks]:  y[t, h] = sum_{j=0..top_k-1} y_slots[t, j, h], added in slot
// order in f32, so the result is deterministic and independent of which CTA
// produced which slot.  A shared expert's gated rows [hf2q qwen35
// MoeFfnArena: sh_logit, h_s], when present, are added after the last slot.
// Streaming, 16-byte loads and stores.
#include <atomic>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y_slots,
                                                      float4* __restrict__ y, long long m,
                                                      int hidden4, int top_k,
                                                      const float4* __restrict__ y_extra,
                                                      const int* __restrict__ status) {
    if (*status != 0) return;
    const long long total = m * hidden4;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long t = i / hidden4;
        const int h = static_cast<int>(i - t * hidden4);
        const float4* src = y_slots + (t * top_k) * hidden4 + h;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        // Up to 8 slots' loads in flight at once, then added in slot order
        // (the first slot initialises the sum, so the order of additions is
        // exactly ((s0 + s1) + s2) + ...).
        for (int j0 = 0; j0 < top_k; j0 += 8) {
            float4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (j0 + q < top_k) v[q] = __ldcs(src + static_cast<long long>(j0 + q) * hidden4);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (j0 + q >= top_k) break;
                if (j0 + q == 0) {
                    acc = v[0];
                } else {
                    acc.x += v[q].x;
                    acc.y += v[q].y;
                    acc.z += v[q].z;
                    acc.w += v[q].w;
                }
            }
        }
        if (y_extra) {
            const float4 v = __ldcs(y_extra + i);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        __stcs(y + i, acc);
    }
}

cudaError_t launch_combine(const float* y_slots, float* y, int m, int hidden, int top_k,
                           const float* y_extra, const int* status, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int hidden4 = hidden / 4;
    const long long total = static_cast<long long>(m) * hidden4;
    long long blocks = (total + 255) / 256;
    // resident blocks per SM (queried once per device): the grid-stride loop
    // covers the rest
    static std::atomic<int> per_sm_cache[64];
    int per_sm = dev >= 0 && dev < 64 ? per_sm_cache[dev].load(std::memory_order_relaxed) : 0;
    if (per_sm < 1) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_kernel, 256, 0) !=
                cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        else if (dev >= 0 && dev < 64)
            per_sm_cache[dev].store(per_sm, std::memory_order_relaxed);
    }
    const long long cap = static_cast<long long>(sms) * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    combine_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(y_slots), reinterpret_cast<float4*>(y), m, hidden4, top_k,
        reinterpret_cast<const float4*>(y_extra), status);
    return cudaGetLastError();
}

// Clock probe: each block's first thread records (SM id, SM cycle counter,
// global nanosecond timer).  Two probes around a timed region give the
// average SM clock over it: (cycles_end - cycles_start) / (ns_end - ns_start)
// on any SM present in both.
__global__ void clock_probe_kernel(unsigned long long* out) {
    if (threadIdx.x != 0) return;
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    const unsigned long long cycles = clock64();
    const unsigned long long ns = global_timer_ns();
    out[3 * blockIdx.x] = smid;
    out[3 * blockIdx.x + 1] = cycles;
    out[3 * blockIdx.x + 2] = ns;
}

cudaError_t launch_clock_probe(unsigned long long* out, int n_blocks, cudaStream_t stream) {
    clock_probe_kernel<<<n_blocks, 32, 0, stream>>>(out);
    return cudaGetLastError();
}

// One thread waits, with the library's bounded wait, on an mbarrier whose
// phase nothing completes (its one expected arrival never comes).
__global__ void wait_timeout_selftest_kernel(int* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitCtl ctl{&abort_flag, status, limit_ns};
        mbar_wait(&bar, 0, ctl);
    }
    __syncthreads();
}

cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns,
                                         cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(status, 0, sizeof(int), stream);
    if (err != cudaSuccess) return err;
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace moe
