// Down-projection weights in fp16, converted once per heavily routed expert.
//
// [hf2q, qwen35/dense_ffn_arena.rs: MoeFfnArena's down projection reads the
// W_down rows of each chosen expert; this library multiplies them in fp16 on
// the tensor cores.]  The grouped down kernel converts every W_down tile it
// loads in shared memory, so an expert with many 128-row tiles would convert
// the same weights once per row tile.  For the experts with at least
// min_rows routed rows this kernel writes fp16(W_down[e]) once into the
// workspace, and the down kernel loads those tiles as they are.  Streaming
// 16-byte loads and stores: HBM-bound, 4 bytes moved per weight (2 read,
// 2 written), and the copy stays in L2 for the down kernel when it fits.
#include "device_common.cuh"
#include "launch.h"

namespace moe {

constexpr int kConvBlock = 512;

__global__ void __launch_bounds__(kConvBlock) w_down_fp16_kernel(
    const uint4* __restrict__ W_down, const int* __restrict__ counts, int n_experts,
    long long pieces_per_expert, long long min_rows, int max_slots, int* __restrict__ conv_slot,
    uint4* __restrict__ w16, const int* __restrict__ status) {
    __shared__ int slot_expert[MOE_MAX_EXPERTS];
    __shared__ int n_slots;
    if (*status != 0) return;
    // Slots: the qualifying experts in id order (one warp, 32 experts a step).
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int base = 0;
        for (int e0 = 0; e0 < n_experts; e0 += 32) {
            const int e = e0 + lane;
            const bool q = e < n_experts && counts[e] >= min_rows;
            const unsigned ball = __ballot_sync(0xffffffffu, q);
            const int rank = base + __popc(ball & ((1u << lane) - 1u));
            const bool kept = q && rank < max_slots;
            if (kept) slot_expert[rank] = e;
            if (blockIdx.x == 0 && e < n_experts) conv_slot[e] = kept ? rank : -1;
            base += __popc(ball);
        }
        if (lane == 0) n_slots = base < max_slots ? base : max_slots;
    }
    __syncthreads();
    // Piece p of the copy is piece p - s * pieces_per_expert of slot s's
    // expert; four loads in flight per thread.
    const long long total = static_cast<long long>(n_slots) * pieces_per_expert;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < total; i += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const long long p = i + q * stride;
            const int s = static_cast<int>(p / pieces_per_expert);
            v[q] = ld_stream_u4(W_down + static_cast<long long>(slot_expert[s]) * pieces_per_expert +
                                (p - s * pieces_per_expert));
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) w16[i + q * stride] = bf16x8_to_f16x8(v[q]);
    }
    for (; i < total; i += stride) {
        const int s = static_cast<int>(i / pieces_per_expert);
        const uint4 v = ld_stream_u4(W_down + static_cast<long long>(slot_expert[s]) * pieces_per_expert +
                                     (i - s * pieces_per_expert));
        w16[i] = bf16x8_to_f16x8(v);
    }
}

cudaError_t launch_w_down_fp16(const __nv_bfloat16* W_down, const int* counts, int n_experts,
                               long long expert_elems, long long min_rows, int max_slots,
                               int* conv_slot, __half* w16, const int* status,
                               cudaStream_t stream) {
    if (n_experts < 1 || n_experts > MOE_MAX_EXPERTS || expert_elems % 8 != 0 || max_slots < 1)
        return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    w_down_fp16_kernel<<<2 * sms, kConvBlock, 0, stream>>>(
        reinterpret_cast<const uint4*>(W_down), counts, n_experts, expert_elems / 8, min_rows,
        max_slots, conv_slot, reinterpret_cast<uint4*>(w16), status);
    return cudaGetLastError();
}

}  // namespace moe
