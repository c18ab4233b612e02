// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "switch_moe.h"

namespace switchmoe {

// Tokens per routing tile: the granularity of the per-tile expert histograms,
// of the probability partial sums and of the slot-assignment blocks.
constexpr int kTileT = 64;

// Kernel ids reported by the tracer.
enum KernelId : int32_t {
    K_ROUTER_WARP = 1,
    K_ROUTER_TILED = 2,
    K_SCAN = 3,
    K_ASSIGN = 4,
    K_DISPATCH = 5,
    K_FFN_TC_GEMM1 = 6,
    K_FFN_TC_GEMM2 = 7,
    K_FFN_SIMT_GEMM1 = 8,
    K_FFN_SIMT_GEMM2 = 9,
    K_COMBINE = 10,
    K_FFN_TC_GEMM2_GATED = 11,
    K_ASSIGN_SCATTER = 12,
    K_ROUTER_STAGED = 13,
    K_ROUTER_TC = 14,
    K_ROUTER_SPLIT = 15,
    K_SELFTEST_WAIT = 16,
    K_FFN_TC_FUSED = 17,
    K_COMBINE_TOP2 = 18,
    K_BWD_TOKEN = 19,
    K_BWD_GEMM_DZ = 21,
    K_BWD_GEMM_DX = 22,
    K_BWD_GEMM_DW = 23,
    K_BWD_ROUTER_DX = 24,
    K_BWD_ROUTER_DW = 25,
    K_BWD_REDUCE = 26,
    K_ROUTER_STATS = 27,
    K_SMALL_LAYER = 28,
    K_BWD_ROUTER_SPLIT = 29,
    K_BWD_ROUTER_TC_DX = 30,
    K_BWD_ROUTER_TC_DW = 31,
    K_BWD_ZERO_TAILS = 32,
};

struct Workspace {
    void *status;        // DeviceStatus
    uint32_t *ticket;    // last-block ticket of the scan kernel
    int32_t *hist;       // [N][tiles] tokens of each expert in each tile
    float *psum;         // [N][tiles] sum of p_i over each tile
    int32_t *tile_off;   // [N][tiles] exclusive prefix of hist over tiles
    double *prob_total;  // [N] sum of p_i over all tokens
    void *w_split;       // [3][N][d] bf16 terms of W_r (tensor-core router)
    int32_t *slot_token; // [N*C] (layer_fwd only)
    void *xbuf;          // [N][C][d] (layer_fwd only)
    float *ybuf;         // [N][C][d] float32 (layer_fwd only)
    void *hidden;        // [N][C][F] expert hidden activations
    int32_t *done;       // fused FFN: [N][ceil(C/256)] GEMM1 completion counters, the tile claim counter,
                         // [N][ceil(C/256)][ceil(d/256)] GEMM2 first-half counters (fused_counter_ints)
    int32_t *hist2;      // top-2: [N][tiles] second choices of each expert in each tile
    int32_t *tile_off2;  // top-2: [N][tiles] first slot of each tile's second choices
    int32_t *counts_first;  // top-2: [N] first choices per expert (the aux loss's f)
    float *ent;          // with SWITCH_FLAG_ROUTER_STATS: [tiles] per-tile sums of the router entropy (else null)
    float *probs;        // training: [T][N] router probabilities kept for the backward pass (else null)
    // training only (SWITCH_FLAG_TRAINING): backward-pass buffers
    float *dh;           // [T][N] gradient of the router logits
    void *grad_e;        // [N][C][d] bf16 gate * dy in expert order
    void *grad_z;        // [N][C][F] bf16 gradient of the pre-activations
    float *dw_part;      // [chunks][N][d] partial sums of dW_r
    float *db_part;      // [chunks][N] partial sums of d bias
    void *rdx_a;         // [T][6 Np] bf16 split dh terms (tensor-core router dx)
    void *rdx_b;         // [d][6 Np] bf16 split W_r terms (tensor-core router dx)
    void *rdw_a;         // [chunks][3N][Tc] bf16 split dh terms, token-contiguous (tensor-core dW_r)
    int32_t *chunk_counts;  // [chunks + 1] tokens of each dW_r chunk, then a 1
    int64_t tiles;
};

size_t workspace_bytes(const switch_dims_t &dims);
// int32 counters the fused expert FFN keeps in Workspace::done (GEMM2 counters
// for its narrower 128-column tiles, the larger count).
inline int64_t fused_counter_ints(int64_t N, int64_t C, int64_t d) {
    const int64_t MT = (C + 255) / 256;
    return N * MT + 1 + N * MT * ((d + 127) / 128);
}
// Bytes at the start of the workspace layout that the routing step uses
// (status word, ticket, per-tile counts / sums / offsets, probability totals).
size_t route_scratch_bytes(const switch_dims_t &dims);
Workspace carve_workspace(const switch_dims_t &dims, void *base);

// Launch bookkeeping (tracing + launch counter).
void launch_begin(int32_t kernel_id, cudaStream_t stream);
void launch_end(cudaStream_t stream);

// Launchers.  Each returns the cudaError_t of its launch.
// With `x_scatter` set, the slot assignment also copies every kept token's
// row of x into xbuf[expert, slot] (scatter form of the dispatch) and, with
// `y_zero` set, writes the zero output row of every dropped token.
// With `top2`, expert, gate and slot are [T][2] (first and second choice of
// each token) and the scan always runs as its own kernel.
cudaError_t launch_route(const switch_dims_t &dims, const void *x, const float *w_r, const float *bias,
                         int32_t *expert, float *gate, int32_t *slot, int32_t *counts, int32_t *slot_token,
                         float *aux, const Workspace &ws, cudaStream_t stream, void *xbuf_scatter = nullptr,
                         float *y_zero = nullptr, int32_t *done_zero = nullptr, int64_t n_done = 0,
                         bool top2 = false);
cudaError_t launch_dispatch(const switch_dims_t &dims, const void *x, const int32_t *slot_token,
                            const int32_t *counts, void *xbuf, cudaStream_t stream);
cudaError_t launch_combine(const switch_dims_t &dims, const float *ybuf, const int32_t *expert,
                           const int32_t *slot, const float *gate, float *y, cudaStream_t stream);
// Top-2 combine: y[t] = gate[2t] ybuf[expert[2t], slot[2t]] + gate[2t+1] ybuf[expert[2t+1], slot[2t+1]]
// over the kept choices (0 when both were dropped).
cudaError_t launch_combine_top2(const switch_dims_t &dims, const float *ybuf, const int32_t *expert,
                                const int32_t *slot, const float *gate, float *y, cudaStream_t stream);
// Tensor-core router (bf16 x, N <= 128): writes expert, gate and the
// per-tile counts / probability sums like the CUDA-core routers.
bool router_tc_supported(const switch_dims_t &dims);
cudaError_t launch_router_tc(const switch_dims_t &dims, const void *x, const float *w_r, const float *bias,
                             int32_t *expert, float *gate, const Workspace &ws, cudaStream_t stream,
                             bool top2 = false);
// Expert FFN; ybuf is float32 [N][C][d].
cudaError_t launch_ffn_simt(const switch_dims_t &dims, const void *xbuf, const void *w_in, const void *w_out,
                            const int32_t *counts, float *ybuf, const Workspace &ws, cudaStream_t stream);
// Tensor-core expert FFN.  With `y` set, GEMM2 writes y[t] = gate[t] * acc
// straight to token order (t = slot_token[i*C+s]) instead of ybuf.
cudaError_t launch_ffn_tc(const switch_dims_t &dims, const void *xbuf, const void *w_in, const void *w_out,
                          const int32_t *counts, void *ybuf, const int32_t *slot_token, const float *gate, float *y,
                          const Workspace &ws, cudaStream_t stream);

// The whole layer in one block for small float32 layers (switch_layer_fwd's default there).
bool small_layer_supported(const switch_dims_t &dims);
cudaError_t launch_small_layer(const switch_dims_t &dims, const void *x, const float *w_r, const float *bias,
                               const void *w_in, const void *w_out, float *y, int32_t *expert, float *gate,
                               int32_t *slot, int32_t *counts, float *aux, const Workspace &ws, cudaStream_t stream);

// Router statistics from the per-tile entropy sums a routing call left in the workspace.
cudaError_t launch_router_stats(const switch_dims_t &dims, const int32_t *counts, const Workspace &ws, float *stats,
                                cudaStream_t stream);

// Backward pass (bfloat16 experts; the workspace of a SWITCH_FLAG_TRAINING forward).
int64_t router_dw_chunks(int64_t T);
int64_t router_tc_chunk_tokens(int64_t T);
int64_t router_tc_chunks(int64_t T);
int router_tc_np(int N);
cudaError_t launch_router_tc_bwd_dx(const void *a, const void *b, const int32_t *one, int64_t T, int d, int K,
                                    float *dx, DeviceStatus *st, cudaStream_t stream);
cudaError_t launch_router_tc_bwd_dw(const void *a, const void *b, const int32_t *chunk_counts, int chunks, int rows,
                                    int chunk_tokens, int d, int64_t T, float *part, DeviceStatus *st,
                                    cudaStream_t stream);
cudaError_t launch_layer_bwd(const switch_dims_t &dims, const void *x, const float *w_r, const void *w_in,
                             const void *w_out, const int32_t *expert, const float *gate, const int32_t *slot,
                             const int32_t *counts, const float *dy, float g_aux, float *dx, float *dw_r, float *dbias,
                             float *dw_in, float *dw_out, const Workspace &ws, cudaStream_t stream);
cudaError_t launch_ffn_tc_bwd_dz(const switch_dims_t &dims, const void *grad_e, const void *w_out,
                                 const int32_t *counts, void *grad_z, const void *hidden, DeviceStatus *st,
                                 cudaStream_t stream);
cudaError_t launch_ffn_tc_bwd_dx(const switch_dims_t &dims, const void *grad_z, const void *w_in,
                                 const int32_t *counts, const int32_t *slot_token, float *dx, DeviceStatus *st,
                                 cudaStream_t stream);
cudaError_t launch_ffn_tc_bwd_dw(const switch_dims_t &dims, const void *a, const void *b, const int32_t *counts,
                                 int rows, int nout, float *out, DeviceStatus *st, cudaStream_t stream);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Kernel launch; with `pdl` the kernel may begin while its predecessor on the
// stream finishes (it must pdl_wait() before using the predecessor's data).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                          Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace switchmoe
