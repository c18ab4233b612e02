/*
 * switch_moe.h -- C ABI of the B200 (sm_100a) Switch Transformer sparse FFN
 * layer forward pass.
 *
 * The layer (Switch routing, top-1): for every token x of a group of T tokens
 *   h = W_r . x (+ b)             router logits, float32
 *   p_i = softmax(h)_i            gate probabilities
 *   i* = argmax_i p_i             one expert per token, lowest index on ties
 *   C  = ceil(T / N * c)          expert capacity (slots per expert)
 *   the first C tokens of each expert, in token order, are kept; the others
 *   are dropped and get a zero layer output (they pass on through the
 *   residual connection, which is the caller's)
 *   y  = p_i*(x) * W_out[i*] . ReLU(W_in[i*] . x)
 *   aux = N * sum_i f_i * P_i     load-balancing loss without its alpha weight
 * Sources: llm-papers-study "精读 06 | Switch Transformers" §3.1 (router
 * logits and softmax), §3.2 (top-1 routing, y = p_i* E_i*), §3.3 (load
 * balancing loss), §3.4 (expert capacity, dropped tokens); Incredible.AI
 * "Switch Transformer - Scaling to Trillion Parameter Models with Simple and
 * Efficient Sparsity", sections "Router Implementation" and "MoE Layer";
 * kasblo "Switch Transformerとは？" section "Routerだけfloat32で計算する
 * Selective Precision" (router in float32, experts in bfloat16).
 *
 * Conventions shared by every entry point:
 *  - Ownership: the caller allocates and frees every buffer.  All array
 *    arguments are DEVICE pointers to contiguous row-major memory, 16-byte
 *    aligned, unless marked otherwise.  The library never allocates, frees or
 *    synchronises, except switch_check() (which synchronises the stream).
 *  - Streams: every compute call is asynchronous on `stream` (a cudaStream_t;
 *    NULL means the legacy default stream) and enqueues only kernels of this
 *    library, plus a few small cudaMemsetAsync calls on the workspace, on it.
 *  - Errors: argument errors are detected on the host before anything is
 *    launched and leave every output untouched.  A failed launch returns
 *    SWITCH_ERR_CUDA.  A kernel that gives up a bounded wait records
 *    SWITCH_ERR_DEVICE_TIMEOUT in the workspace status word, which
 *    switch_check() reports.
 *  - Token order: token t is row t of x (a [batch, seq, d] tensor flattened
 *    row-major, t = b * seq + s).
 */
#ifndef SWITCH_MOE_H
#define SWITCH_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* Same type as cudaStream_t. */
typedef struct CUstream_st *switch_stream_t;

typedef enum {
    SWITCH_OK = 0,
    SWITCH_ERR_NULL = 1,           /* a required pointer is NULL */
    SWITCH_ERR_SHAPE = 2,          /* a size is out of range or violates a divisibility rule */
    SWITCH_ERR_DTYPE = 3,          /* unknown dtype code */
    SWITCH_ERR_ALIGN = 4,          /* a pointer is not 16-byte aligned */
    SWITCH_ERR_WORKSPACE = 5,      /* workspace smaller than switch_workspace_size() */
    SWITCH_ERR_UNSUPPORTED = 6,    /* valid request the library cannot run (e.g. no sm_100 device) */
    SWITCH_ERR_CUDA = 7,           /* a CUDA runtime call or kernel launch failed */
    SWITCH_ERR_DEVICE_TIMEOUT = 8, /* a kernel gave up a bounded wait (reported by switch_check) */
    SWITCH_ERR_TOO_LARGE = 9       /* switch_route_noalloc: the group needs more scratch than its static buffer */
} switch_status_t;

/* Storage type of the input activations (x, xbuf) and of the expert weights
 * (W_in, W_out).  The router weight, the logit bias, the gates, the expert
 * outputs (ybuf) and the layer output (y) are always float32: the expert
 * output stays in the float32 accumulator precision until it is scaled by
 * its gate, and the result is rounded once. */
typedef enum {
    SWITCH_F32 = 0,  /* IEEE binary32 */
    SWITCH_BF16 = 1  /* bfloat16 */
} switch_dtype_t;

/* Diagnostic switches for switch_dims_t.flags. */
enum {
    SWITCH_FLAG_NONE = 0,
    /* Run the expert FFN on CUDA cores instead of tcgen05 tensor cores (bf16). */
    SWITCH_FLAG_SIMT_FFN = 1,
    /* Compute router logits on CUDA cores (FFMA) even where a tensor-core
     * router exists. */
    SWITCH_FLAG_SIMT_ROUTER = 2,
    /* Run each expert GEMM tile on one SM (cta_group::1, 128-row tiles)
     * instead of on a pair of SMs (cta_group::2, 256-row tiles). */
    SWITCH_FLAG_GEMM_1CTA = 4,
    /* In switch_layer_fwd, launch the two expert GEMMs one after the other
     * instead of as one persistent kernel. */
    SWITCH_FLAG_FFN_TWO_LAUNCHES = 8,
    /* Always run the capacity scan as its own kernel.  By default, when the
     * per-tile expert histogram is small, each slot-assignment block sums the
     * counts it needs itself and the scan kernel is skipped; both give the
     * same slots and counts (aux may differ in the last bits: its fp64 sums
     * run in another fixed order). */
    SWITCH_FLAG_SEPARATE_SCAN = 16,
    /* Training: switch_layer_fwd keeps what the backward pass needs in the
     * workspace (the router probabilities, the dispatched tokens, the hidden
     * activations and the ungated expert outputs) and runs the two expert
     * GEMMs and the combine as separate launches; switch_workspace_size grows
     * accordingly.  switch_layer_bwd requires it.  bfloat16 experts only. */
    SWITCH_FLAG_TRAINING = 32,
    /* The routing step also sums the entropy of every token's router
     * distribution per 64-token tile into the workspace, for
     * switch_router_stats. */
    SWITCH_FLAG_ROUTER_STATS = 64,
    /* In switch_layer_fwd, run the layer as its separate kernels even where
     * the single-block path for small float32 layers (T <= 256, N <= 32,
     * inputs and weights within 160 KB of shared memory) would apply. */
    SWITCH_FLAG_MULTI_KERNEL = 128,
    /* switch_dispatch and switch_combine move rows of up to ~6 KB through
     * shared memory by bulk copies (the TMA engine) instead of vector loads
     * and stores; the results are identical. */
    SWITCH_FLAG_STAGED_MOVES = 256
};

typedef struct {
    int64_t T;            /* tokens in the group; 0 <= T < 2^31 */
    int32_t d_model;      /* d, 1..8192 */
    int32_t d_ff;         /* F, 1..32768 */
    int32_t num_experts;  /* N, 1..256 */
    int32_t capacity;     /* C, slots per expert, >= 1 (see switch_capacity) */
    int32_t dtype;        /* switch_dtype_t */
    int32_t flags;        /* SWITCH_FLAG_* (0 for the default path) */
} switch_dims_t;
/* Shape rules: bfloat16 requires d_model % 64 == 0 and d_ff % 64 == 0;
 * float32 accepts any d_model, d_ff >= 1.  N * C must fit in int32. */

/* Expert capacity C = ceil(T / N * c), at least 1 (llm-papers-study §3.4,
 * expert capacity = tokens per batch / number of experts x capacity factor;
 * the sources leave the rounding open and this library rounds up).  A
 * product within 1e-9 of an integer counts as that integer.  Host only.
 * Returns -1 if T < 0, N < 1 or c is not a positive finite number. */
int64_t switch_capacity(int64_t T, int32_t num_experts, double capacity_factor);

/* Bytes of device workspace that every entry point below needs for `dims`
 * (scan state, per-tile partial sums, the hidden activations H[N, C, F], the
 * layer's internal [N, C, d] buffers and the status word).  Host only.
 * Errors: SWITCH_ERR_NULL, SWITCH_ERR_SHAPE, SWITCH_ERR_DTYPE. */
switch_status_t switch_workspace_size(const switch_dims_t *dims, size_t *bytes);

/* Router, top-1, capacity assignment, per-expert counts and the aux loss
 * (llm-papers-study §3.1-§3.4; Incredible.AI "Router Implementation").
 *   x          [T, d]   activation dtype
 *   w_r        [N, d]   float32 router weight (row i produces logit i)
 *   logit_bias [N]      float32 added to the logits, or NULL for none
 * Outputs (all written):
 *   expert     [T]      int32, argmax expert of each token (lowest index on ties)
 *   gate       [T]      float32, p_expert(x) = softmax(h)[expert]
 *   slot       [T]      int32, position of the token in its expert's buffer,
 *                       in token order, or -1 when it overflowed capacity
 *   counts     [N]      int32, tokens routed to each expert BEFORE capacity
 *   slot_token [N * C]  int32, token held by slot s of expert i at [i*C+s],
 *                       -1 for an empty slot
 *   aux        [1]      float32, N * sum_i (counts_i / T) * (mean_t p_i);
 *                       0 when T == 0
 * Deterministic: identical inputs give identical bytes. */
switch_status_t switch_route(const switch_dims_t *dims, const void *x, const float *w_r,
                             const float *logit_bias, int32_t *expert, float *gate, int32_t *slot,
                             int32_t *counts, int32_t *slot_token, float *aux, void *workspace,
                             size_t workspace_bytes, switch_stream_t stream);

/* Dispatch: gather the kept tokens into per-expert buffers
 * (Incredible.AI "MoE Layer", x_flat[expert_indices]; kasblo "tokenを
 * Expertへ送って戻すforward pass", single-device gather).
 *   xbuf[i, s, :] = x[slot_token[i*C+s], :]   for s < min(counts[i], C)
 *   x [T, d], slot_token [N*C], counts [N]  ->  xbuf [N, C, d] (activation dtype)
 * Rows s >= min(counts[i], C) of xbuf are not written. */
switch_status_t switch_dispatch(const switch_dims_t *dims, const void *x, const int32_t *slot_token,
                                const int32_t *counts, void *xbuf, switch_stream_t stream);

/* Expert FFN on the kept rows of every expert:
 *   ybuf[i, s, :] = W_out[i] . ReLU(W_in[i] . xbuf[i, s, :])   for s < min(counts[i], C)
 *   xbuf  [N, C, d]   activation dtype
 *   w_in  [N, F, d]   expert dtype (nn.Linear layout: row j feeds hidden unit j)
 *   w_out [N, d, F]   expert dtype
 *   ybuf  [N, C, d]   float32; other rows are not written
 * bfloat16: tcgen05 tensor cores, float32 accumulation, the hidden
 * activations rounded to bfloat16 in the workspace.  float32: CUDA cores.
 * (Switch FFN experts: llm-papers-study §3.2; two-layer ReLU experts without
 * biases, the sources leave the body open.) */
switch_status_t switch_expert_ffn(const switch_dims_t *dims, const void *xbuf, const void *w_in,
                                  const void *w_out, const int32_t *counts, void *ybuf, void *workspace,
                                  size_t workspace_bytes, switch_stream_t stream);

/* Combine: scatter back to token order, scaled by the gate
 * (llm-papers-study §3.2, y = p_i*(x) E_i*(x); §3.4, dropped tokens skip the
 * expert):
 *   y[t, :] = gate[t] * ybuf[expert[t], slot[t], :]   if slot[t] >= 0
 *   y[t, :] = 0                                       if slot[t] == -1
 * The product is formed in float32.
 *   ybuf [N, C, d] float32, expert [T], slot [T], gate [T]  ->  y [T, d] float32 */
switch_status_t switch_combine(const switch_dims_t *dims, const void *ybuf, const int32_t *expert,
                               const int32_t *slot, const float *gate, void *y, switch_stream_t stream);

/* The whole layer: switch_route, then dispatch, expert FFN and combine, with
 * the [N, C, d] buffers and slot_token kept in the workspace.  Arguments as
 * above; y [T, d] float32 is the layer output WITHOUT the residual.  On the
 * bfloat16 tensor-core path the dispatch is fused into the slot assignment
 * and both expert GEMMs run in one persistent kernel with the combine in the
 * second GEMM's epilogue; when the second GEMM may have many tiles (12 waves
 * of 256 x 256 tiles over the SM pairs or more, an upper bound from T, N and
 * C), the first GEMM also gets its own launch, and the device counts decide
 * which of the two launches runs it.  With SWITCH_FLAG_FFN_TWO_LAUNCHES the
 * result is bit-identical to calling the four steps one by one, and so is the
 * default wherever the second GEMM is not split.  By default, when the second
 * GEMM has few tiles, its tiles are split along d_ff and their parts added
 * into y in a fixed order: routing, counts and aux are unchanged and y differs
 * from the four-step result by float32 rounding only.  Small float32 layers
 * (T <= 256, N <= 32, everything within 160 KB of shared memory) run in one
 * thread block instead (SWITCH_FLAG_MULTI_KERNEL keeps the separate steps);
 * there y differs from the four-step result by float32 rounding only.  Either
 * way identical inputs give identical bytes. */
switch_status_t switch_layer_fwd(const switch_dims_t *dims, const void *x, const float *w_r,
                                 const float *logit_bias, const void *w_in, const void *w_out, void *y,
                                 int32_t *expert, float *gate, int32_t *slot, int32_t *counts, float *aux,
                                 void *workspace, size_t workspace_bytes, switch_stream_t stream);

/* ---- top-2 routing ------------------------------------------------------
 * The classic mixture-of-experts layer that Switch routing simplifies
 * (Incredible.AI "Switch Transformer - Scaling to Trillion Parameter Models",
 * section "Mixture of Experts Routing"; llm-papers-study "精读 06 | Switch
 * Transformers" §3.1, y = sum over the top-K experts of p_i(x) E_i(x), with
 * K = 2): the two largest softmax probabilities select two experts, and each
 * selected expert's output is weighted by its own probability (no
 * renormalisation over the pair).  Requires N >= 2.  Readings where the
 * sources are silent:
 *  - the first choice is the lowest index of the largest logit, the second
 *    the lowest index of the largest logit among the other experts;
 *  - capacity C applies to (token, choice) assignments; every first choice
 *    (in token order) ranks before every second choice (in token order), so
 *    first choices get exactly the slots of top-1 routing;
 *  - the aux loss keeps its definition: f_i counts first choices only.
 * Per-token arrays are [T][2]: element 2t is the first choice of token t,
 * element 2t + 1 its second choice.  The workspace is the one of
 * switch_workspace_size(dims). */

/* Router, top-2, capacity assignment, counts and aux.
 *   expert [T][2] int32, gate [T][2] float32 (p of each choice),
 *   slot [T][2] int32 (-1 = that choice was dropped),
 *   counts [N] int32: (token, choice) assignments per expert over both
 *   choices, before capacity; slot_token [N * C] int32 (-1 = empty);
 *   aux [1] float32 = N * sum_i (first choices of i / T) * (mean_t p_i).
 * Errors as switch_route, plus SWITCH_ERR_SHAPE when N < 2.  Deterministic. */
switch_status_t switch_route_top2(const switch_dims_t *dims, const void *x, const float *w_r,
                                  const float *logit_bias, int32_t *expert, float *gate, int32_t *slot,
                                  int32_t *counts, int32_t *slot_token, float *aux, void *workspace,
                                  size_t workspace_bytes, switch_stream_t stream);

/* Top-2 combine:  y[t, :] = sum over the kept choices c of token t of
 *   gate[2t+c] * ybuf[expert[2t+c], slot[2t+c], :]
 * in float32, the first choice's product first, then the second's added
 * (each product and the sum rounded to float32); an all-zero row when both
 * choices were dropped.  ybuf [N, C, d] float32 -> y [T, d] float32.
 * (switch_dispatch and switch_expert_ffn serve top-2 routing unchanged: they
 * work from slot_token and counts.) */
switch_status_t switch_combine_top2(const switch_dims_t *dims, const void *ybuf, const int32_t *expert,
                                    const int32_t *slot, const float *gate, void *y, switch_stream_t stream);

/* The whole top-2 layer: switch_route_top2 (with both choices' rows of x
 * copied into the workspace's per-expert buffers by the slot assignment), the
 * expert FFN into the workspace's float32 ybuf, then switch_combine_top2.
 * Arguments as switch_layer_fwd, with expert, gate and slot of shape [T][2].
 * Identical inputs give identical bytes. */
switch_status_t switch_layer_fwd_top2(const switch_dims_t *dims, const void *x, const float *w_r,
                                      const float *logit_bias, const void *w_in, const void *w_out, void *y,
                                      int32_t *expert, float *gate, int32_t *slot, int32_t *counts, float *aux,
                                      void *workspace, size_t workspace_bytes, switch_stream_t stream);

/* Router statistics that the sources list for monitoring a Switch layer next
 * to its loss (kasblo "Switch Transformerとは？", end of section "補助負荷分散
 * lossは何を均等にするのか": tokens per expert, use of capacity, the overflow /
 * dropped-token rate, the entropy of the router probabilities), for the last
 * switch_route / switch_layer_fwd (or top-2) call made with the same dims and
 * workspace.  stats [4] float32 (device):
 *   stats[0] mean over tokens of -sum_i p_i ln p_i  (NaN unless that call had
 *            SWITCH_FLAG_ROUTER_STATS in its dims flags, as these dims must)
 *   stats[1] dropped fraction  sum_i max(0, counts_i - C) / T
 *   stats[2] capacity utilisation  sum_i min(counts_i, C) / (N C)
 *   stats[3] busiest expert's load over the uniform load  max_i counts_i N / T
 * counts [N] as that call wrote them (after a top-2 call: assignments; the
 * dropped fraction is then per (token, choice) over T).  All 0 when T == 0. */
switch_status_t switch_router_stats(const switch_dims_t *dims, const int32_t *counts, const void *workspace,
                                    size_t workspace_bytes, float *stats, switch_stream_t stream);

/* Backward pass of the layer (top-1), after a switch_layer_fwd call made with
 * SWITCH_FLAG_TRAINING in the same dims and the same workspace (whose
 * contents that call left behind are its input here).  The loss is
 * L = sum(y * dy) + g_aux * aux; the argmax and the capacity assignment pass no
 * gradient: the router learns through the selected probability p_i*(x) that
 * scales the expert output (kasblo "Switch Transformerとは？", section
 * "argmaxは離散なのに、Routerはなぜ学習できるのか") and, for the aux loss,
 * through P_i only, f_i being a count (llm-papers-study §3.3).
 *   x, w_r, w_in, w_out       the forward's inputs; expert, gate, slot, counts
 *                             the forward's outputs (as it wrote them)
 *   dy [T, d] float32         upstream gradient of y
 *   g_aux                     upstream gradient of aux (the loss weight alpha)
 * Outputs (float32, all written): dx [T, d]; dw_r [N, d]; dbias [N] (the
 * gradient of the logit bias; NULL to skip); dw_in [N, F, d]; dw_out [N, d, F]
 * (zero for experts without kept tokens).  A dropped token's dx is the router
 * part only.  The expert GEMMs run on tcgen05 tensor cores with bfloat16
 * operands (gate * dy and the pre-activation gradient rounded to bfloat16) and
 * float32 accumulation.  The router products (dh W_r into dx, dh^T x into
 * dw_r) run on the tensor cores too, over exact three-term bfloat16 splits of
 * their float32 operands with float32 accumulation (the three smallest term
 * pairs of dh W_r, below 2^-23 of |dh| |W_r| together, are left out); with
 * SWITCH_FLAG_SIMT_ROUTER in dims.flags (for the forward too) they run as
 * float32 FMA kernels instead.  Deterministic.
 * Errors: SWITCH_ERR_UNSUPPORTED without SWITCH_FLAG_TRAINING, for float32
 * experts or with SWITCH_FLAG_SIMT_FFN / SWITCH_FLAG_GEMM_1CTA; SWITCH_ERR_SHAPE
 * for a non-finite g_aux; otherwise as switch_layer_fwd. */
switch_status_t switch_layer_bwd(const switch_dims_t *dims, const void *x, const float *w_r, const void *w_in,
                                 const void *w_out, const int32_t *expert, const float *gate, const int32_t *slot,
                                 const int32_t *counts, const float *dy, float g_aux, float *dx, float *dw_r,
                                 float *dbias, float *dw_in, float *dw_out, void *workspace, size_t workspace_bytes,
                                 switch_stream_t stream);

/* Routing without a workspace, for callers that cannot allocate device
 * memory at the point where they route tokens: code running under a host
 * framework that owns every device allocation and forbids new ones while it
 * executes (an inference engine's plugin, a server that reserves all of its
 * device memory up front), or code with no allocator at hand.  The sources
 * have no counterpart of this entry point; it exists for those callers only.
 *
 * Same arguments (minus the workspace) and the same outputs, bit for bit, as
 * switch_route.  Its scratch is one static device array of
 * SWITCH_NOALLOC_SCRATCH_BYTES inside this library, which every GPU that
 * loads the library holds until the process exits; it allocates and frees
 * nothing.  A call needs about 12 * N * ceil(T / 64) + 8 * N + 6 * N * d
 * bytes of it (plus under 2 KiB of alignment padding), so the 4 MiB array
 * holds, for example, T = 131072 tokens with 128 experts and d_model = 1024;
 * a larger group returns SWITCH_ERR_TOO_LARGE before anything runs.
 *
 * Every call looks up the array's device address (cudaGetSymbolAddress, which
 * allocates nothing) with the calling device current; on the first call on a
 * device this may load the library's device code, so make that first call
 * before any stream capture.
 * Every call shares the one array and leaves its contents behind (the next
 * call clears what must start at zero), so calls whose kernels may overlap
 * on the GPU (on different streams, or from several host threads) race and
 * must not be issued; calls on one stream are fine.  The device status word
 * lives in the array too: switch_check_noalloc reads it. */
#define SWITCH_NOALLOC_SCRATCH_BYTES (4u << 20)
switch_status_t switch_route_noalloc(const switch_dims_t *dims, const void *x, const float *w_r,
                                     const float *logit_bias, int32_t *expert, float *gate, int32_t *slot,
                                     int32_t *counts, int32_t *slot_token, float *aux, switch_stream_t stream);

/* switch_check for switch_route_noalloc: synchronise `stream`, then read and
 * clear the status word kept in the library's static routing array on the
 * current device (a bounded wait of the router that gave up leaves
 * SWITCH_ERR_DEVICE_TIMEOUT there).  Allocates nothing. */
switch_status_t switch_check_noalloc(switch_stream_t stream);

/* switch_selftest_wait_timeout on the static routing array's status word
 * (for testing switch_check_noalloc); allocates nothing. */
switch_status_t switch_selftest_wait_timeout_noalloc(switch_stream_t stream);

/* Synchronise `stream`, then read and clear the device status word kept in
 * `workspace`.  switch_route, switch_expert_ffn and switch_layer_fwd clear
 * that word before their first kernel runs, so the workspace needs no
 * initialisation; switch_check reports the first failure recorded since.
 * Returns SWITCH_OK, SWITCH_ERR_DEVICE_TIMEOUT, or SWITCH_ERR_CUDA if the
 * stream reports an error. */
switch_status_t switch_check(void *workspace, size_t workspace_bytes, switch_stream_t stream);

/* Self-test of the device-side failure detection.  Launches one block that
 * waits, with the same bounded wait the library's kernels use, on an mbarrier
 * that nothing completes.  After about one second the wait gives up, records
 * SWITCH_ERR_DEVICE_TIMEOUT in the workspace status word and the kernel exits
 * normally (no trap, no fault): switch_check() then returns
 * SWITCH_ERR_DEVICE_TIMEOUT and the CUDA context stays usable.  Needs at
 * least 16 bytes of workspace. */
switch_status_t switch_selftest_wait_timeout(void *workspace, size_t workspace_bytes, switch_stream_t stream);

/* Static description of a status code. */
const char *switch_status_string(switch_status_t status);

/* ---- instrumentation -------------------------------------------------- */

/* Number of kernels this library has launched in this process. */
int64_t switch_launch_count(void);

/* Per-launch tracing.  While tracing is on, every kernel launch is bracketed
 * by two CUDA events recorded on its stream; at most `max_launches` launches
 * are kept.  switch_trace_read() synchronises those events and fills
 * kernel_id[k] and ms[k] (elapsed milliseconds of launch k), returning the
 * number of launches traced.  Host only; not thread-safe. */
switch_status_t switch_trace_start(int32_t max_launches);
int32_t switch_trace_read(int32_t *kernel_id, float *ms, int32_t capacity);
void switch_trace_stop(void);
/* Name of a traced kernel id, or "?" if unknown. */
const char *switch_kernel_name(int32_t kernel_id);

#ifdef __cplusplus
}
#endif

#endif /* SWITCH_MOE_H */
