// Host-side launchers shared between the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Routed rows per block of the expert-map count/scatter passes.
constexpr int kMapChunkRows = 2048;
// Rows of one grouped-GEMM tile (the tcgen05 MMA M).
constexpr int kTileRows = 128;
// Largest m*top_k handled by the weight-streaming matmul_id kernel.
constexpr int kStreamMaxRows = 256;
// Largest m*top_k handled by the weight-streaming FFN kernels (measured on
// B200: the grouped GEMMs overtake them between 160 and 192 routed rows).
constexpr int kStreamFfnMaxRows = 128;
// Gathered GEMMs zero-fill a partial tile's unused A rows when the average
// routed rows per expert are at most this (measured on B200: saves 10% of
// gate/up at 128 rows per expert, costs ~20% at 1024, where partial tiles are
// rare; the choice depends on the shape only and never changes a result).
constexpr long long kZeroFillMaxRowsPerExpert = 256;
// The grouped FFN converts an expert's W_down to fp16 once, before the down
// GEMM, when the expert has at least this many routed rows (4 row tiles, each
// of which would otherwise convert the weights again in shared memory;
// measured on B200: the in-kernel conversion of a weight tile costs more than
// the tile's MMAs when the tensor pipe is busy).  At most
// min(E, rows / kPreconvMinRows) experts qualify, which sizes the workspace.
// The fp16 weights are the same either way, so results never depend on it.
constexpr long long kPreconvMinRows = 512;

// Device buffers of one expert map (all inside the caller's workspace).
struct MapBuffers {
    int* status;      // [1] first error code of the call
    int* counts;      // [E]
    int* offsets;     // [E + 1]
    int* perm;        // [R]
    int* inv_perm;    // [R]
    int* chunk_hist;  // [n_chunks, E]
    int* chunk_base;  // [n_chunks, E]
    int4* tiles;      // [max tiles]: (expert, first sorted row, rows, 0)
    int* n_tiles;     // [1]
    int* active;      // [E] experts with at least one row, ascending
    int* n_active;    // [1]
};

// n_parts > 1: `logits` is n_parts partial slabs [m, n_experts] (a projection
// split along K), summed in slab order into logits_out before the routing.
cudaError_t launch_route_topk(const float* logits, const float* bias, int m, int n_experts,
                              int top_k, int* ids, float* weights, float* scores,
                              cudaStream_t stream, int n_parts = 1, float* logits_out = nullptr);
cudaError_t launch_route_weights(const float* logits, const int* ids, int m, int n_experts,
                                 int top_k, float* weights, cudaStream_t stream);
cudaError_t launch_expert_map(const int* ids, int rows, int n_experts, int tile_rows,
                              const MapBuffers& b, cudaStream_t stream);

// The map of `rows` rows that all go to one expert (0): identity perm, one
// expert, ceil(rows / tile_rows) tiles.  Writes no status.
cudaError_t launch_dense_map(int rows, int tile_rows, const MapBuffers& b, cudaStream_t stream);

// Weight-streaming matmul by expert id (small m).
// W_e = W + e * w_stride (elements; n * k for a dense stack).
cudaError_t launch_stream_matmul_id(const __nv_bfloat16* x, const __nv_bfloat16* W, float* y,
                                    int m, int n, int k, int top_k, int n_experts, int layout,
                                    size_t w_stride, const MapBuffers& b, cudaStream_t stream);

// The same for m*top_k <= kStreamMaxRows with the expert map built inside the
// kernel (one launch; writes the status word itself).
cudaError_t launch_stream_matmul_id_fused(const __nv_bfloat16* x, const int* ids,
                                          const __nv_bfloat16* W, float* y, int m, int n, int k,
                                          int top_k, int n_experts, int layout, size_t w_stride,
                                          int* status, cudaStream_t stream);

// Grouped tcgen05 GEMMs.
struct GroupedGemmArgs {
    const __nv_bfloat16* a_ptr;  // gathered modes: x, rows of length k
    const int* perm;
    const int4* tiles;
    const int* n_tiles;
    const float* weights;  // DOWN: per routed row
    void* out;
    const int* status;
    int* status_out;
    long long rows;   // R = m * top_k
    int n;            // output columns (inter for gate/up)
    int k;            // reduction length
    int n_col_tiles;  // ceil(n / output columns per tile)
    int top_k;
    int layout;
    int b_rows_per_expert;  // rows of B per expert in its 2-D view
    int dense_m_tiles;      // modes 3/4: ceil(rows / 128)
    int k_splits;           // mode 4: K ranges per output tile (partial slabs in out)
    int b_3d;               // mode 2: B map is 3-D [E, n, k] (padded expert stride)
    int out_sigmoid;        // mode 3: store sigmoid(acc) (f64 math, rounded to f32)
    int zero_fill_dead;     // modes 0/2: zero-fill (no read) a partial tile's unused rows
    int swap_small;         // mode 1: tiles of <= 64 rows run with the operands swapped
    const int* conv_slot;   // mode 1: [E] slot of the expert's fp16 W_down in map_c, or -1
                            // (null: every tile converts its W_down in shared memory)
    unsigned long long wait_limit_ns;
};

// mode 0: gate/up + SwiGLU -> fp16 act (scaled by 2^-4); 1: fp16 down +
// weighted scatter; 2: matmul_id scatter; 3: dense rows x W^T (status
// pointers may be null); 4: dense rows x W^T in 256-column tiles split into
// k_splits K ranges, range s writing its partial sums to out + s * rows * n.
// map_c (mode 1 with conv_slot): the pre-converted fp16 W_down
// [slots * hidden, inter].
cudaError_t launch_grouped_gemm(int mode, const CUtensorMap& map_a, const CUtensorMap& map_b0,
                                const CUtensorMap& map_b1, const GroupedGemmArgs& args,
                                int num_sms, cudaStream_t stream,
                                const CUtensorMap* map_c = nullptr);

// fp16 copies of W_down for the experts with at least min_rows routed rows
// (counts from the expert map): conv_slot[e] = the expert's slot (its rank
// among those experts, in id order; -1 for the others, and for every expert
// past max_slots), w16[slot] = fp16(W_down[e]) [hidden * inter], rounded to
// nearest.  Does nothing once the status word is set.
cudaError_t launch_w_down_fp16(const __nv_bfloat16* W_down, const int* counts, int n_experts,
                               long long expert_elems, long long min_rows, int max_slots,
                               int* conv_slot, __half* w16, const int* status,
                               cudaStream_t stream);
size_t grouped_gemm_smem_bytes(int mode);

// Decode-size FFN (m*top_k <= kStreamFfnMaxRows): weight-streaming gate/up with
// SwiGLU into f32 act [rows, inter], then down with the combine weight into
// y_slots [rows, hidden].  With ids, the gate/up kernel builds the expert map
// itself (and writes it to b, with the status word, for the kernels after
// it); without ids, b must already hold a map.
cudaError_t launch_stream_ffn(const __nv_bfloat16* x, const float* weights,
                              const __nv_bfloat16* W_gate, const __nv_bfloat16* W_up,
                              const __nv_bfloat16* W_down, float* act, float* y_slots, int m,
                              int hidden, int inter, int top_k, int layout, const MapBuffers& b,
                              cudaStream_t stream, const int* ids = nullptr, int n_experts = 0);

// y[t] = sum_j y_slots[t, j] (slot order), then + y_extra[t] when given.
cudaError_t launch_combine(const float* y_slots, float* y, int m, int hidden, int top_k,
                           const float* y_extra, const int* status, cudaStream_t stream);

// Expert parallelism: owner rank of each routed row (ids / experts_per_rank;
// an id outside [0, n_experts) sets MOE_ERR_DEVICE_BAD_ID), the send-ordered
// input rows and local expert ids, and the weighted slot-order combine of
// the returned rows (d_back in send order, inv = send position of routed row).
cudaError_t launch_ep_owner(const int* ids, long long rows, int n_experts, int experts_per_rank,
                            int* owner, int* status, cudaStream_t stream);
cudaError_t launch_ep_pack(const __nv_bfloat16* x, const int* ids, const int* perm, long long rows,
                           int hidden, int top_k, int layout, int experts_per_rank,
                           __nv_bfloat16* send_x, int* send_expert, const int* status,
                           cudaStream_t stream);
cudaError_t launch_ep_combine(const float* d_back, const int* inv, const float* weights, float* y,
                              int m, int hidden, int top_k, const int* status,
                              cudaStream_t stream);

// Sets the calling thread's moe_last_error() message.
void set_last_error(const char* msg);

cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns,
                                         cudaStream_t stream);
cudaError_t launch_clock_probe(unsigned long long* out, int n_blocks, cudaStream_t stream);

}  // namespace moe
