// Grouped GEMM over experts on the 5th-generation tensor cores (tcgen05).
//
// Definitions:
//  * matmul by expert id [mlx-native 0.13.0, src/ops/dense_matmul_id_auto.rs:
//    the Grouped route reorders routed rows by expert and multiplies each
//    expert's rows by its weight matrix]: y[r] = W[ids[r]] . x_row(r).
//  * SwiGLU expert FFN [hf2q 0.1.1, eagle3/forward.rs "Phase E4b.8":
//    down(silu(gate(x)) * up(x)); cortiq-engine src/mimo_moe.rs
//    tests::exact_moe: sum_j w_j * down_e(silu(gate_e x) * up_e x)].
//
// One persistent kernel per GEMM, one CTA per SM (288 threads; 448 for down):
//   warps 0-3   producers.  In the gathered modes the 128 threads copy the A
//               rows picked by the expert permutation with 16-byte cp.async
//               straight into the 128-byte-swizzled K-major layout (8 threads
//               per 128-byte row piece, coalesced), and each thread's copies
//               arrive on the stage's mbarrier when they land.  Thread 0 also
//               streams B (the expert's weights) with 2-D TMA tile copies.  A
//               4-stage shared-memory ring decouples them from the MMA.
//               (A per-row TMA gather, tile::gather4, was measured at ~78 SM
//               cycles per 4-row copy, too slow to keep up with the weights.)
//   warp 4      TMEM allocation; one thread issues tcgen05.mma (M=128, N=256,
//               K=16, bf16 -> f32) and commits each stage back to the
//               producers and each finished accumulator to the epilogue.
//   warps 5-8   epilogue: tcgen05.ld of their 32-lane quarter, fused math,
//               32x32 chunks staged through padded shared memory so that
//               each store instruction writes whole row pieces.
//   warps 9-13  (down only) W_down converters, with producer warps 1-3.
// Two 256-column TMEM accumulators let the epilogue of tile i overlap the
// mainloop of tile i+1.  Tiles are (expert m-tile, column tile) with the
// column tile fastest, so CTAs in flight share A rows and expert weights in L2.
//
// Modes:
//   0 gate/up: B = [128 gate rows ; 128 up rows] of one expert, so one N=256
//     MMA produces both; epilogue a = silu(g)*u, written in expert-sorted row
//     order as fp16(a * kActScale): 11 significant bits of a.
//   1 down: A = fp16 activation tiles, B = the W_down tile, which 256
//     converter threads rewrite in shared memory from bf16 to fp16 once its
//     copy has landed (exact for bf16 |w| in [2^-17, 65280]), or which
//     arrives as fp16 when the expert's W_down was converted before the launch
//     (experts with at least 512 routed rows); one f16 MMA per k-step, f32
//     accumulate; the epilogue multiplies by the routed row's combine weight
//     times 1 / kActScale, checks that the accumulator is finite, and stores
//     the row to its (token, slot) place.  A tile of at
//     most 64 routed rows (its activation arrives as 64-row boxes) swaps the
//     operands: the two 128-row halves of the W_down tile are A (M=128) and
//     the 64 token rows B (N=64), half the MMA work of the M=128 x N=256
//     form; the tensor cores give the same bits either way.
//   2 matmul by id: A gathered from x, epilogue stores rows to (token, slot).
//   3 dense (the shared expert's gate logit): A is plain 128-row TMA tiles of
//     x, 64-column B tiles, the output rows stay in place; no expert map.
//   4 dense split along K (router projection [cortiq-engine src/mimo_moe.rs
//     test model, tensor mlp.gate.weight]: logits = x . W_router^T): 256-column
//     tiles, each output tile's K split into k_splits ranges on separate CTAs,
//     each range storing its partial sums to its own slab; the routing kernel
//     adds the slabs in range order.
//
// Determinism: tile shape, K order and per-row epilogue math are fixed by the
// shape alone, so a row's bits do not depend on which other rows share its
// expert (balanced and skewed routings give identical rows).
//
// Every barrier wait is bounded (device_common.cuh); on a timeout the CTA
// records MOE_ERR_DEVICE_TIMEOUT, all roles leave their loops, in-flight copies
// and MMAs are drained with bounded waits, and TMEM is freed before exit.
#include <atomic>
#include <cfloat>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

constexpr int kProducerWarps = 4;                 // warps 0-3
constexpr int kMmaWarp = 4;                       // warp 4
constexpr int kEpilogueWarp0 = 5;                 // warps 5-8
constexpr int kBaseWarps = 9;
constexpr int kConvWarp0 = 9;                     // down only: warps 9-13 convert W_down
constexpr int kConvExtraWarps = 5;
constexpr int kGatherThreads = kProducerWarps * 32;
// tcgen05.ld lets warp w read TMEM lanes [32*(w%4), +32): four consecutive
// epilogue warps cover all 128 accumulator rows.
static_assert(kBaseWarps - kEpilogueWarp0 == 4, "epilogue must be 4 warps");
template <int MODE>
constexpr int gemm_threads() {
    return (MODE == 1 ? kBaseWarps + kConvExtraWarps : kBaseWarps) * 32;
}
constexpr int kBK = 64;                 // k-block: 64 bf16 = one 128-byte swizzle row
constexpr int kTileA = 128 * 128;       // bytes of a 128-row x 64-col bf16 tile
constexpr int kTmemCols = 512;          // two 256-column f32 accumulators

template <int MODE>
struct GemmCfg;
template <>
struct GemmCfg<0> {  // gate/up + SwiGLU
    static constexpr int kStages = 4, kABytes = kTileA, kBBytes = 2 * kTileA, kOutCols = 128;
    static constexpr int kMmaN = 256;
};
template <>
struct GemmCfg<1> {  // down (fp16 activation x fp16-converted W_down) + weighted scatter
    static constexpr int kStages = 4, kABytes = kTileA, kBBytes = 2 * kTileA, kOutCols = 256;
    static constexpr int kMmaN = 256;
};

// The down projection multiplies in fp16: the gate/up epilogue stores the
// activation a as fp16(a * kActScale) (|a| up to 65504 / kActScale), each
// W_down tile is converted in shared memory to fp16(w) (exact for bf16 w with
// 2^-17 <= |w| <= 65280; 65536 and above become infinite), and the down
// epilogue multiplies the f32 accumulator by 1 / kActScale, a power of two,
// so every product and partial sum is the unscaled one.  A non-finite
// accumulator (an out-of-range value, or a non-finite input) sets
// MOE_ERR_DEVICE_RANGE.
constexpr float kActScale = 0.0625f;
// W_down converter threads of the down kernel: producer warps 1-3 (warp 0's
// first lane issues the tile copies) and warps 9-13.
constexpr int kConvThreads = (kProducerWarps - 1 + kConvExtraWarps) * 32;
template <>
struct GemmCfg<2> {  // matmul by expert id
    static constexpr int kStages = 4, kABytes = kTileA, kBBytes = 2 * kTileA, kOutCols = 256;
    static constexpr int kMmaN = 256;
};
template <>
struct GemmCfg<3> {  // dense rows x W^T (the shared expert's gate): 64-column tiles
    static constexpr int kStages = 8, kABytes = kTileA, kBBytes = kTileA / 2, kOutCols = 64;
    static constexpr int kMmaN = 64;
};
template <>
struct GemmCfg<4> {  // dense rows x W^T split along K (router projection): 256-column
                     // tiles, so each x row is read once per K range, and K ranges
                     // spread the few row tiles over the SMs
    static constexpr int kStages = 4, kABytes = kTileA, kBBytes = 2 * kTileA, kOutCols = 256;
    static constexpr int kMmaN = 256;
};

template <int MODE>
constexpr int stage_bytes() {
    return GemmCfg<MODE>::kABytes + GemmCfg<MODE>::kBBytes;
}

// Epilogue staging: per epilogue warp 32 rows x 32 f32, rows padded to 33
// words so that both the row-wise writes and the column-wise reads are free
// of bank conflicts.
constexpr int kStagePitch = 33;
constexpr int kEpiStageBytes = 4 * 32 * kStagePitch * 4;

template <int MODE>
constexpr size_t smem_bytes() {
    // ring + barriers/flags + epilogue staging + slack to align the ring
    return static_cast<size_t>(GemmCfg<MODE>::kStages) * stage_bytes<MODE>() + 256 +
           kEpiStageBytes + 1024;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// Gate of a shared expert (mode 3 with out_sigmoid): f64 math, one rounding.
__device__ __forceinline__ float sigmoid_f64_to_f32(float v) {
    return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(v))));
}

// (expert, first row, rows, -) of m-tile mt: from the expert map's tile list,
// or, for the dense mode, the 128-row blocks of the rows themselves.
template <int MODE>
__device__ __forceinline__ int4 tile_rows_of(const GroupedGemmArgs& args, int mt) {
    if (MODE == 3 || MODE == 4) {
        const long long first = static_cast<long long>(mt) * kTileRows;
        const long long left = args.rows - first;
        return make_int4(0, static_cast<int>(first), static_cast<int>(left < kTileRows ? left : kTileRows), 0);
    }
    return args.tiles[mt];
}

// Tile t -> (m-tile, column tile, K range): the column tile runs fastest; the
// split-K mode puts the K ranges of one output tile on consecutive tiles.
struct TileCoord {
    int mt, nt, ks;
};
template <int MODE>
__device__ __forceinline__ TileCoord tile_coord(const GroupedGemmArgs& args, int tile) {
    int ks = 0;
    if (MODE == 4) {
        ks = tile % args.k_splits;
        tile /= args.k_splits;
    }
    const int mt = tile / args.n_col_tiles;
    return TileCoord{mt, tile - mt * args.n_col_tiles, ks};
}

// W_down converters of the down kernel: once a stage's W_down tile has landed
// (wload), rewrite it in place as fp16 (an element-wise map, so the 128-byte
// swizzle is untouched), order the writes for the tensor core and release
// the stage to the MMA (full).  Thread ct converts 16-byte pieces ct,
// ct + kConvThreads, ...: a warp covers 512 contiguous bytes per access, and
// all of a thread's loads are in flight before its first conversion.  A tile
// of an expert whose weights were converted before the launch (conv_slot)
// landed as fp16 and is only passed on.
template <int MODE>
__device__ __forceinline__ void convert_w_down(uint8_t* smem, uint64_t* wload, uint64_t* full,
                                               int ct, int total, int nk, const GroupedGemmArgs& args,
                                               const WaitCtl& ctl) {
    using C = GemmCfg<MODE>;
    constexpr int kStage = stage_bytes<MODE>();
    constexpr int kPer = C::kBBytes / 16 / kConvThreads;
    static_assert(C::kBBytes / 16 == kPer * kConvThreads, "whole pieces per converter");
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const bool converted =
            args.conv_slot != nullptr &&
            args.conv_slot[tile_rows_of<MODE>(args, tile / args.n_col_tiles).x] >= 0;
        for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(&wload[stage], phase, ctl)) return;
            if (!converted) {
                uint4* w4 = reinterpret_cast<uint4*>(smem + stage * kStage + C::kABytes) + ct;
                uint4 v[kPer];
#pragma unroll
                for (int i = 0; i < kPer; ++i) v[i] = w4[i * kConvThreads];
#pragma unroll
                for (int i = 0; i < kPer; ++i) w4[i * kConvThreads] = bf16x8_to_f16x8(v[i]);
                fence_proxy_async_smem();  // generic writes -> tensor core reads
            }
            mbar_arrive(&full[stage]);
            if (++stage == C::kStages) {
                stage = 0;
                phase ^= 1;
            }
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(gemm_threads<MODE>(), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_b0,
                        const __grid_constant__ CUtensorMap map_b1,
                        const __grid_constant__ CUtensorMap map_c, const GroupedGemmArgs args) {
    using C = GemmCfg<MODE>;
    constexpr int kStage = stage_bytes<MODE>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * kStage);
    uint64_t* empty = full + C::kStages;
    uint64_t* acc_full = empty + C::kStages;  // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2]
    uint64_t* drain_bar = acc_empty + 2;      // [1]
    uint64_t* wload = drain_bar + 1;          // [kStages] mode 1: W_down tile landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wload + C::kStages);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* epi_stage = reinterpret_cast<float*>(smem + C::kStages * kStage + 256);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool kGather = MODE == 0 || MODE == 2;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // gathered modes: 128 cp.async arrivals + the B copy's expect_tx
            // arrival; down: the converters' arrivals + the A copy's
            mbar_init(&full[s], kGather ? kGatherThreads + 1 : MODE == 1 ? kConvThreads + 1 : 1);
            mbar_init(&empty[s], 1);
            mbar_init(&wload[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 0) {
        if (!kGather) prefetch_tensormap(&map_a);
        prefetch_tensormap(&map_b0);
        if (MODE == 0 || MODE == 1) prefetch_tensormap(&map_b1);
        if (MODE == 1 && args.conv_slot) prefetch_tensormap(&map_c);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    const WaitCtl ctl{abort_flag, args.status_out, args.wait_limit_ns};
    const bool failed = args.status != nullptr && *args.status != 0;
    const int n_mtiles = MODE == 3 || MODE == 4 ? args.dense_m_tiles : *args.n_tiles;
    const int n_split = MODE == 4 ? args.k_splits : 1;
    const int total = failed ? 0 : n_mtiles * args.n_col_tiles * n_split;
    // k-blocks per tile (split-K: per K range; the last range may run past K,
    // where the tile copies read zeros)
    const int nk = ((args.k + kBK - 1) / kBK + n_split - 1) / n_split;
    const long long R = args.rows;

    if (warp < kProducerWarps) {
        // ------------------------------------------------------------ producers
        const int pt = threadIdx.x;        // 0..127
        const int prow0 = pt >> 3;         // first tile row of this thread (0..15)
        const int pchunk = pt & 7;         // 16-byte piece of the 128-byte row
        // 128-byte swizzle: piece c of row r sits at piece (c ^ (r & 7)); the
        // thread's rows prow0 + 16 i all share r & 7.
        const uint32_t swz = static_cast<uint32_t>((pchunk ^ (prow0 & 7)) << 4);
        int stage = 0;
        uint32_t phase = 0, armed = 0, armed_parity = 0;
        if (kGather || pt == 0) {
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
                const TileCoord tc = tile_coord<MODE>(args, tile);
                const int mt = tc.mt, nt = tc.nt;
                const int4 d = tile_rows_of<MODE>(args, mt);  // (expert, first row, rows, -)
                const __nv_bfloat16* src[8];
                uint32_t live = 0;  // bit i: tile row prow0 + 16 i holds a routed row
                if (kGather) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int row = prow0 + 16 * i;
                        long long r = args.perm[d.y + (row < d.z ? row : 0)];
                        live |= static_cast<uint32_t>(row < d.z) << i;
                        if (r < 0 || r >= R) r = 0;  // never reached with a valid map
                        const long long xr = args.layout ? r : r / args.top_k;
                        src[i] = args.a_ptr + xr * args.k + pchunk * 8;
                    }
                }
                const int b_row = d.x * args.b_rows_per_expert + nt * (MODE == 0 ? 128 : C::kMmaN);
                // down: the expert's W_down converted before the launch, if any
                const int slot = MODE == 1 && pt == 0 && args.conv_slot ? args.conv_slot[d.x] : -1;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, ctl)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * kStage;
                    uint8_t* sb = sa + C::kABytes;
                    const int kc = (tc.ks * nk + kb) * kBK;
                    if (pt == 0) {
                        if (MODE == 1) {
                            // the fp16 activation: a 64-row box (map_b1) when
                            // the tile holds at most 64 routed rows, else 128
                            // rows (rows past them are never stored); the
                            // W_down tile lands on wload for the converters
                            const bool half = d.z <= 64;
                            mbar_arrive_expect_tx(&full[stage], half ? kTileA / 2 : kTileA);
                            tma_load_2d(sa, half ? &map_b1 : &map_a, &full[stage], kc, d.y);
                            mbar_arrive_expect_tx(&wload[stage], C::kBBytes);
                            if (slot >= 0)
                                tma_load_2d(sb, &map_c, &wload[stage], kc,
                                            slot * args.b_rows_per_expert + nt * C::kMmaN);
                            else
                                tma_load_2d(sb, &map_b0, &wload[stage], kc, b_row);
                        } else if (MODE == 0) {
                            mbar_arrive_expect_tx(&full[stage], C::kBBytes);
                            tma_load_2d(sb, &map_b0, &full[stage], kc, b_row);
                            tma_load_2d(sb + kTileA, &map_b1, &full[stage], kc, b_row);
                        } else if (MODE == 3 || MODE == 4) {
                            mbar_arrive_expect_tx(&full[stage], kStage);
                            tma_load_2d(sa, &map_a, &full[stage], kc, d.y);
                            tma_load_2d(sb, &map_b0, &full[stage], kc, b_row);
                        } else {
                            mbar_arrive_expect_tx(&full[stage], C::kBBytes);
                            if (args.b_3d)
                                tma_load_3d(sb, &map_b0, &full[stage], kc, nt * 256, d.x);
                            else
                                tma_load_2d(sb, &map_b0, &full[stage], kc, b_row);
                        }
                        armed |= 1u << stage;
                        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    }
                    if (kGather) {
                        const uint32_t a0 = smem_u32(sa) + static_cast<uint32_t>(prow0 * 128) + swz;
                        // past K (last k-block): zero-fill, and point at the row
                        // start.  Rows past the tile's routed rows either copy
                        // the tile's first row again or, with zero_fill_dead,
                        // are zero-filled without a read (never stored either way)
                        const bool in_k = kc + pchunk * 8 < args.k;
                        const int koff = in_k ? kc : 0;
                        if (args.zero_fill_dead && d.z < 128) {
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                cp_async_16(a0 + static_cast<uint32_t>(i * 16 * 128), src[i] + koff,
                                            in_k && (live >> i & 1) ? 16u : 0u);
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                cp_async_16(a0 + static_cast<uint32_t>(i * 16 * 128), src[i] + koff,
                                            in_k ? 16u : 0u);
                        }
                        cp_async_arrive_noinc(&full[stage]);
                    }
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
            }
        }
        if (MODE == 1 && warp >= 1)  // pieces 0..95 of each piece group
            convert_w_down<MODE>(smem, wload, full, threadIdx.x - 32, total, nk, args, ctl);
        // Every copy this CTA started has landed before it can exit.
        if (kGather) cp_async_wait_all();
        if (pt == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (armed >> s & 1) {
                    if (MODE == 1) mbar_drain(&wload[s], armed_parity >> s & 1, 100000000ull);
                    mbar_drain(&full[s], armed_parity >> s & 1, 100000000ull);
                }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
                // down: a tile of at most 64 routed rows runs with the operands
                // swapped (the weights as M, its tokens as N = 64)
                const bool swp = MODE == 1 && args.swap_small &&
                                 tile_rows_of<MODE>(args, tile / args.n_col_tiles).z <= 64;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, ctl)) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&full[stage], phase, ctl)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    if (kGather) fence_proxy_async_smem();  // cp.async rows -> tensor core
                    const uint32_t a_addr = smem_u32(smem + stage * kStage);
                    const uint32_t b_addr = a_addr + C::kABytes;
                    constexpr uint32_t idesc = umma_idesc_bf16_f32(128, C::kMmaN);
                    if (MODE == 1 && swp) {
                        // D^T[h, token] for the W_down rows of both 128-row
                        // halves (A) against the tile's 64 token rows (B)
                        constexpr uint32_t idesc_s = umma_idesc_f16_f32(128, 64);
#pragma unroll
                        for (int k4 = 0; k4 < kBK / 16; ++k4) {
                            const uint64_t act_d = sw128_kmajor_desc(a_addr + k4 * 32);
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh)
                                umma_bf16(d_tmem + hh * 64,
                                          sw128_kmajor_desc(b_addr + hh * kTileA + k4 * 32), act_d,
                                          idesc_s, (kb | k4) != 0);
                        }
                    } else {
                        // modes 0/2/3: bf16 operands; mode 1: fp16 operands
                        constexpr uint32_t idesc_mode =
                            MODE == 1 ? umma_idesc_f16_f32(128, C::kMmaN) : idesc;
#pragma unroll
                        for (int k4 = 0; k4 < kBK / 16; ++k4)
                            umma_bf16(d_tmem, sw128_kmajor_desc(a_addr + k4 * 32),
                                      sw128_kmajor_desc(b_addr + k4 * 32), idesc_mode,
                                      (kb | k4) != 0);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit(&acc_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            // All MMAs issued by this thread have finished before TMEM is freed.
            umma_commit(drain_bar);
            mbar_drain(drain_bar, 0, 100000000ull);
        }
        __syncwarp();
    } else if (warp < kBaseWarps) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
        const int row = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const TileCoord tc = tile_coord<MODE>(args, tile);
            const int mt = tc.mt, nt = tc.nt;
            const int4 d = tile_rows_of<MODE>(args, mt);
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase, ctl))) break;
            tc_fence_after_sync();
            const uint32_t t_row =
                tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * 256);
            bool valid = row < d.z;
            const long long p = static_cast<long long>(d.y) + row;  // expert-sorted position
            if (MODE == 0) {
                // silu(g)*u per element (lane = row), staged through shared
                // memory, then written as fp16(a * kActScale) with each lane
                // storing 8 consecutive columns of one row: 8 rows x 16 bytes
                // per store instruction.
                __half* act = static_cast<__half*>(args.out);
                bool range_ok = true;
                float* buf = epi_stage + (warp - kEpilogueWarp0) * 32 * kStagePitch;
                const int n0 = nt * 128;
                const int sub_row = lane >> 2;       // 0..7
                const int sub_col = (lane & 3) * 8;  // 8 of the 32 columns
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t g[32], u[32];
                    tmem_load_32cols(t_row + c * 32, g);
                    tmem_load_32cols(t_row + 128 + c * 32, u);
                    tmem_load_wait();
                    const int col0 = n0 + c * 32;
                    if (col0 >= args.n) break;  // warp-uniform
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        buf[lane * kStagePitch + j] =
                            silu_mul(__uint_as_float(g[j]), __uint_as_float(u[j]));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = i * 8 + sub_row;           // row within the warp's 32
                        const int trow = quarter * 32 + rr;       // row within the tile
                        const int col = col0 + sub_col;
                        if (trow < d.z && col < args.n) {
                            const float* a = buf + rr * kStagePitch + sub_col;
                            uint32_t h[4];
#pragma unroll
                            for (int q = 0; q < 8; q += 2) {
                                const float v0 = a[q] * kActScale, v1 = a[q + 1] * kActScale;
                                range_ok &= !(fabsf(v0) > 65504.0f) && !(fabsf(v1) > 65504.0f);
                                const __half2 hv = __floats2half2_rn(v0, v1);
                                h[q / 2] = *reinterpret_cast<const uint32_t*>(&hv);
                            }
                            const long long pr = static_cast<long long>(d.y) + trow;
                            *reinterpret_cast<uint4*>(act + pr * args.n + col) =
                                make_uint4(h[0], h[1], h[2], h[3]);
                        }
                    }
                    __syncwarp();
                }
                if (!range_ok) set_status(args.status_out, kDevRange);
            } else if (MODE == 1 && args.swap_small && d.z <= 64) {
                // Swapped tile: TMEM lane = output column h (hidden), column =
                // the tile's token c.  For each token the warp's 32 lanes
                // store 32 consecutive f32 of its (token, slot) row.
                float* out = static_cast<float*>(args.out);
                const int n0 = nt * C::kMmaN;
                int r0 = -1, r1 = -1;
                // the combine weight times the activation's unscale (exact)
                float w0 = 1.0f / kActScale, w1 = 1.0f / kActScale;
                bool finite = true;
                if (lane < d.z) {
                    r0 = args.perm[d.y + lane];
                    if (r0 < 0 || r0 >= R) r0 = -1;  // never reached with a valid map
                    else if (args.weights) w0 = args.weights[r0] * (1.0f / kActScale);
                }
                if (32 + lane < d.z) {
                    r1 = args.perm[d.y + 32 + lane];
                    if (r1 < 0 || r1 >= R) r1 = -1;
                    else if (args.weights) w1 = args.weights[r1] * (1.0f / kActScale);
                }
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t v0[32], v1[32];
                    tmem_load_32cols(t_row + hh * 64, v0);
                    tmem_load_32cols(t_row + hh * 64 + 32, v1);
                    tmem_load_wait();
                    const int h = n0 + hh * 128 + quarter * 32 + lane;
                    const bool h_ok = h < args.n;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        if (c >= d.z) break;  // warp-uniform
                        const int rr = __shfl_sync(0xffffffffu, r0, c);
                        const float ww = __shfl_sync(0xffffffffu, w0, c);
                        const float acc_v = __uint_as_float(v0[c]);
                        if (h_ok && rr >= 0) {
                            finite &= fabsf(acc_v) <= FLT_MAX;
                            out[static_cast<long long>(rr) * args.n + h] = ww * acc_v;
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        if (32 + c >= d.z) break;  // warp-uniform
                        const int rr = __shfl_sync(0xffffffffu, r1, c);
                        const float ww = __shfl_sync(0xffffffffu, w1, c);
                        const float acc_v = __uint_as_float(v1[c]);
                        if (h_ok && rr >= 0) {
                            finite &= fabsf(acc_v) <= FLT_MAX;
                            out[static_cast<long long>(rr) * args.n + h] = ww * acc_v;
                        }
                    }
                }
                if (!finite) set_status(args.status_out, kDevRange);
            } else {
                // Each lane owns one tile row; rows go to scattered (token, slot)
                // places.  A 32x32 chunk is staged through padded shared memory
                // so that every store instruction writes 4 rows x 128
                // contiguous bytes instead of 32 rows x 16 bytes.
                // split-K: each K range writes its own partial slab [rows, n]
                float* out = static_cast<float*>(args.out) +
                             (MODE == 4 ? static_cast<long long>(tc.ks) * R * args.n : 0);
                float* buf = epi_stage + (warp - kEpilogueWarp0) * 32 * kStagePitch;
                const int n0 = nt * C::kMmaN;
                int r = 0;
                // down: the combine weight (null: unweighted) times the
                // activation's unscale, a power of two
                float w = 1.0f / kActScale;
                bool finite = true;
                if (valid) {
                    const int rv = MODE == 3 || MODE == 4 ? static_cast<int>(p) : args.perm[p];
                    if (rv < 0 || rv >= R) valid = false;  // never reached with a valid map
                    else {
                        r = rv;
                        if (MODE == 1 && args.weights) w = args.weights[r] * (1.0f / kActScale);
                    }
                }
                const bool vec4 = (args.n & 3) == 0;
                const int sub_row = lane >> 3;        // 0..3: row of a store instruction
                const int sub_col = (lane & 7) * 4;   // 4 columns of the 32
#pragma unroll 1
                for (int c = 0; c < C::kMmaN / 32; ++c) {
                    uint32_t v[32];
                    tmem_load_32cols(t_row + c * 32, v);
                    tmem_load_wait();
                    const int col0 = n0 + c * 32;
                    if (col0 >= args.n) break;  // warp-uniform
                    const int n_here = args.n - col0;  // columns of this chunk inside n
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float acc_v = __uint_as_float(v[j]);
                        if (MODE == 1) finite &= !valid || j >= n_here || fabsf(acc_v) <= FLT_MAX;
                        buf[lane * kStagePitch + j] = MODE == 1 ? w * acc_v : acc_v;
                    }
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = i * 4 + sub_row;
                        const int dst_row = __shfl_sync(0xffffffffu, r, rr);
                        const bool dst_ok = __shfl_sync(0xffffffffu, valid ? 1 : 0, rr) != 0;
                        const float* srow = buf + rr * kStagePitch + sub_col;
                        const int col = col0 + sub_col;
                        float* dst = out + static_cast<long long>(dst_row) * args.n + col;
                        if (dst_ok && col < args.n) {
                            float o[4] = {srow[0], srow[1], srow[2], srow[3]};
                            if (MODE == 3 && args.out_sigmoid) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) o[q] = sigmoid_f64_to_f32(o[q]);
                            }
                            if (vec4) {
                                *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
                            } else {
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    if (col + q < args.n) dst[q] = o[q];
                            }
                        }
                    }
                    __syncwarp();
                }
                if (MODE == 1 && !finite) set_status(args.status_out, kDevRange);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    } else if (MODE == 1) {
        // ------------------------------------------------------------ converters
        // warps 9-13: pieces 96..255 of each piece group
        convert_w_down<MODE>(smem, wload, full,
                             (kProducerWarps - 1) * 32 + threadIdx.x - kConvWarp0 * 32, total, nk,
                             args, ctl);
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

size_t grouped_gemm_smem_bytes(int mode) {
    switch (mode) {
        case 0: return smem_bytes<0>();
        case 1: return smem_bytes<1>();
        case 2: return smem_bytes<2>();
        case 3: return smem_bytes<3>();
        default: return smem_bytes<4>();
    }
}

template <int MODE>
static cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                               const CUtensorMap& c, const GroupedGemmArgs& args, int grid,
                               cudaStream_t stream) {
    const size_t smem = smem_bytes<MODE>();
    // The shared-memory opt-in is set once per device (a device reset after
    // the first call would need it again; the library does not support that).
    static std::atomic<unsigned long long> opted_in{0};  // bit d: device d
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0;
    if (!bit || !(opted_in.load(std::memory_order_acquire) & bit)) {
        err = cudaFuncSetAttribute(grouped_gemm_kernel<MODE>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem));
        if (err != cudaSuccess) return err;
        opted_in.fetch_or(bit, std::memory_order_release);
    }
    grouped_gemm_kernel<MODE><<<grid, gemm_threads<MODE>(), smem, stream>>>(a, b0, b1, c, args);
    return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(int mode, const CUtensorMap& map_a, const CUtensorMap& map_b0,
                                const CUtensorMap& map_b1, const GroupedGemmArgs& args,
                                int num_sms, cudaStream_t stream, const CUtensorMap* map_c) {
    if (mode == 1 && args.conv_slot && !map_c) return cudaErrorInvalidValue;
    const CUtensorMap& c = map_c ? *map_c : map_b0;
    // Upper bound of tiles: every expert with rows adds at most one partial tile.
    const long long max_mtiles =
        mode >= 3 ? args.dense_m_tiles
                  : args.rows / kTileRows + 1 + (args.rows < MOE_MAX_EXPERTS ? args.rows : MOE_MAX_EXPERTS);
    if (mode == 4 && args.k_splits < 1) return cudaErrorInvalidValue;
    const long long max_tiles = max_mtiles * args.n_col_tiles * (mode == 4 ? args.k_splits : 1);
    const int grid = static_cast<int>(max_tiles < num_sms ? max_tiles : num_sms);
    switch (mode) {
        case 0: return launch_mode<0>(map_a, map_b0, map_b1, c, args, grid, stream);
        case 1: return launch_mode<1>(map_a, map_b0, map_b1, c, args, grid, stream);
        case 2: return launch_mode<2>(map_a, map_b0, map_b1, c, args, grid, stream);
        case 3: return launch_mode<3>(map_a, map_b0, map_b1, c, args, grid, stream);
        default: return launch_mode<4>(map_a, map_b0, map_b1, c, args, grid, stream);
    }
}

}  // namespace moe
