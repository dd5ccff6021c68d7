// Sigmoid + selection-bias top-k routing, one warp per token.
//
// Definition [cortiq-engine 0.7.7, src/mimo_moe.rs: module doc "top-8,
// sigmoid + selection-bias routing"; Dynamic::run combine weight p[e]/wsum;
// test config "router_sigmoid", "norm_topk_prob", tensor mlp.expert_bias]:
//   s[e]   = sigmoid(logit[e])   computed in double, rounded once to f32
//   key[e] = s[e] + bias[e]      f32 add; NaN ranks as -inf, -0 as +0
//   ids    = top_k experts by (key descending, index ascending)
//   w[j]   = s[ids[j]] / sum_j s[ids[j]]   (double sum in slot order)
//
// Each lane owns experts e = lane + 32*i and sorts its (key, e) pairs once in
// the total order (key desc, index asc) with a bitonic network.  Round j then
// needs only the lanes' first pairs: one warp max-reduction over their keys
// (as order-preserving unsigned integers) finds the best key, one
// min-reduction over the indices of the lanes holding it breaks the tie, and
// the winning lane drops its first pair, so every lane ends with the same
// sequence of winners as a full sort of all experts would give.
#include <climits>
#include <float.h>
#include <math.h>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

__device__ __forceinline__ float routing_score(float logit) {
    return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(logit))));
}

__device__ __forceinline__ float canonical_key(float k) {
    if (isnan(k)) return -INFINITY;
    return k == 0.0f ? 0.0f : k;
}

// (ka, ia) ranks before (kb, ib)?
__device__ __forceinline__ bool ranks_before(float ka, int ia, float kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// Order-preserving map of a canonical key (no NaN, no -0) to an unsigned
// integer, and back: a > b as floats iff key_bits(a) > key_bits(b).
__device__ __forceinline__ unsigned key_bits(float k) {
    const unsigned b = __float_as_uint(k);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_from_bits(unsigned u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// With n_parts > 1, `logits` holds n_parts partial slabs [m, n_experts] of a
// projection split along K; each logit is their f32 sum in slab order, which
// the kernel also stores to logits_out.
template <int NPL>  // experts per lane: ceil(n_experts / 32) rounded up to a power of two
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         const float* __restrict__ bias, int m,
                                                         int n_experts, int top_k,
                                                         int* __restrict__ ids,
                                                         float* __restrict__ weights,
                                                         float* __restrict__ scores, int n_parts,
                                                         float* __restrict__ logits_out) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= m) return;
    const float* lg = logits + static_cast<size_t>(t) * n_experts;
    const size_t slab = static_cast<size_t>(m) * n_experts;

    float key[NPL], lv[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        lv[i] = e < n_experts ? lg[e] : 0.0f;
    }
    if (n_parts > 1) {
        // slab q for all of the lane's experts at once, slabs added in order
        for (int q = 1; q < n_parts; ++q) {
            float pv[NPL];
#pragma unroll
            for (int i = 0; i < NPL; ++i) {
                const int e = lane + 32 * i;
                pv[i] = e < n_experts ? lg[q * slab + e] : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < NPL; ++i) lv[i] += pv[i];
        }
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < n_experts) logits_out[static_cast<size_t>(t) * n_experts + e] = lv[i];
        }
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        key[i] = -INFINITY;
        if (e < n_experts) {
            const float l = lv[i];
            const float s = routing_score(l);
            key[i] = canonical_key(s + (bias ? bias[e] : 0.0f));
            if (scores) scores[static_cast<size_t>(t) * n_experts + e] = s;
        }
    }

    // the lane's pairs in the total order; experts past n_experts (key -inf,
    // index INT_MAX) rank after every real expert
    int idx[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        idx[i] = e < n_experts ? e : INT_MAX;
    }
#pragma unroll
    for (int k = 2; k <= NPL; k <<= 1) {
#pragma unroll
        for (int h = k >> 1; h > 0; h >>= 1) {
#pragma unroll
            for (int i = 0; i < NPL; ++i) {
                const int l = i ^ h;
                if (l > i) {
                    // blocks with (i & k) == 0 end in order, the others reversed
                    const bool out_of_order = (i & k) == 0
                                                  ? ranks_before(key[l], idx[l], key[i], idx[i])
                                                  : ranks_before(key[i], idx[i], key[l], idx[l]);
                    if (out_of_order) {
                        const float tk = key[i];
                        key[i] = key[l];
                        key[l] = tk;
                        const int ti = idx[i];
                        idx[i] = idx[l];
                        idx[l] = ti;
                    }
                }
            }
        }
    }
    int my_id = 0;
    for (int j = 0; j < top_k; ++j) {
        const unsigned u = key_bits(key[0]);
        const unsigned best = __reduce_max_sync(0xffffffffu, u);
        const int win = static_cast<int>(__reduce_min_sync(
            0xffffffffu, u == best ? static_cast<unsigned>(idx[0]) : 0xffffffffu));
        if (idx[0] == win) {  // the winning lane drops its first pair
#pragma unroll
            for (int i = 0; i + 1 < NPL; ++i) {
                key[i] = key[i + 1];
                idx[i] = idx[i + 1];
            }
            key[NPL - 1] = -INFINITY;
            idx[NPL - 1] = INT_MAX;
        }
        if (lane == j) my_id = win;
    }
    // the winner's score, recomputed from its logit (the same rounding as s)
    float my_lv = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const float v = __shfl_sync(0xffffffffu, lv[i], my_id & 31);
        if ((my_id >> 5) == i) my_lv = v;
    }
    const float my_s = lane < top_k ? routing_score(my_lv) : 0.0f;
    double wsum = 0.0;
    for (int j = 0; j < top_k; ++j) wsum += static_cast<double>(__shfl_sync(0xffffffffu, my_s, j));
    if (lane < top_k) {
        ids[static_cast<size_t>(t) * top_k + lane] = my_id;
        weights[static_cast<size_t>(t) * top_k + lane] =
            static_cast<float>(static_cast<double>(my_s) / wsum);
    }
}

// One thread per token: weights of caller-fixed ids.
__global__ void route_weights_kernel(const float* __restrict__ logits,
                                     const int* __restrict__ ids, int m, int n_experts, int top_k,
                                     float* __restrict__ weights) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= m) return;
    const float* lg = logits + static_cast<size_t>(t) * n_experts;
    const int* id = ids + static_cast<size_t>(t) * top_k;
    double wsum = 0.0;
    bool ok = true;
    for (int j = 0; j < top_k; ++j) {
        const int e = id[j];
        if (e < 0 || e >= n_experts) {
            ok = false;
            break;
        }
        wsum += static_cast<double>(routing_score(lg[e]));
    }
    for (int j = 0; j < top_k; ++j) {
        float w = NAN;
        if (ok) w = static_cast<float>(static_cast<double>(routing_score(lg[id[j]])) / wsum);
        weights[static_cast<size_t>(t) * top_k + j] = w;
    }
}

cudaError_t launch_route_topk(const float* logits, const float* bias, int m, int n_experts,
                              int top_k, int* ids, float* weights, float* scores,
                              cudaStream_t stream, int n_parts, float* logits_out) {
    const int warps = 8;
    const dim3 grid((m + warps - 1) / warps), block(32 * warps);
    const int npl = (n_experts + 31) / 32;
#define MOE_ROUTE_CASE(N)                                                                      \
    route_topk_kernel<N><<<grid, block, 0, stream>>>(logits, bias, m, n_experts, top_k, ids, \
                                                     weights, scores, n_parts, logits_out)
    if (npl <= 1) MOE_ROUTE_CASE(1);
    else if (npl <= 2) MOE_ROUTE_CASE(2);
    else if (npl <= 4) MOE_ROUTE_CASE(4);
    else if (npl <= 8) MOE_ROUTE_CASE(8);
    else if (npl <= 16) MOE_ROUTE_CASE(16);
    else MOE_ROUTE_CASE(32);
#undef MOE_ROUTE_CASE
    return cudaGetLastError();
}

cudaError_t launch_route_weights(const float* logits, const int* ids, int m, int n_experts,
                                 int top_k, float* weights, cudaStream_t stream) {
    const int threads = 128;
    route_weights_kernel<<<(m + threads - 1) / threads, threads, 0, stream>>>(
        logits, ids, m, n_experts, top_k, weights);
    return cudaGetLastError();
}

}  // namespace moe
