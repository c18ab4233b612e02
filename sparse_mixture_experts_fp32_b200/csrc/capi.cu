// C ABI of the Switch layer library: argument checks, workspace layout,
// launch bookkeeping and the extern "C" entry points declared in
// include/switch_moe.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace switchmoe {

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

size_t elem_size(const switch_dims_t &d) { return d.dtype == SWITCH_BF16 ? 2 : 4; }

int64_t tiles_of(const switch_dims_t &d) { return (d.T + kTileT - 1) / kTileT; }

struct Sections {
    size_t status, ticket, hist, psum, tile_off, prob_total, w_split, slot_token, xbuf, ybuf, hidden, done, hist2,
        tile_off2, counts_first, ent, probs, dh, grad_e, grad_z,
        dw_part, db_part, rdx_a, rdx_b, rdw_a, chunk_counts, total;
};

Sections layout(const switch_dims_t &d) {
    Sections s{};
    const size_t N = (size_t)d.num_experts, C = (size_t)d.capacity, tiles = (size_t)tiles_of(d);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align_up(bytes);
        return at;
    };
    s.status = take(sizeof(DeviceStatus));
    s.ticket = take(sizeof(uint32_t));
    s.hist = take(N * tiles * 4);
    s.psum = take(N * tiles * 4);
    s.tile_off = take(N * tiles * 4);
    s.prob_total = take(N * 8);
    s.w_split = take(3 * N * (size_t)d.d_model * 2);
    s.slot_token = take(N * C * 4);
    s.xbuf = take(N * C * (size_t)d.d_model * elem_size(d));
    s.ybuf = take(N * C * (size_t)d.d_model * sizeof(float));
    s.hidden = take(N * C * (size_t)d.d_ff * elem_size(d));
    s.done = take(fused_counter_ints(N, C, d.d_model) * sizeof(int32_t));  // the fused FFN's counters
    // top-2 routing only; after everything top-1 routing uses
    s.hist2 = take(N * tiles * 4);
    s.tile_off2 = take(N * tiles * 4);
    s.counts_first = take(N * 4);
    s.ent = take(tiles * 4);
    if (d.flags & SWITCH_FLAG_TRAINING) {  // kept by the training forward, used by the backward pass
        const size_t T = (size_t)d.T, dm = (size_t)d.d_model, F = (size_t)d.d_ff, es = elem_size(d);
        const size_t chunks = (size_t)router_dw_chunks(d.T);
        s.probs = take(T * N * 4);
        s.dh = take(T * N * 4);
        s.grad_e = take(N * C * dm * es);
        s.grad_z = take(N * C * F * es);
        if (d.flags & SWITCH_FLAG_SIMT_ROUTER) {  // float32 FMA router products
            s.dw_part = take(chunks * N * dm * 4);
            s.db_part = take(chunks * N * 4);
        } else {  // tensor-core router products on split operands
            const size_t Np = (size_t)router_tc_np((int)N), Tc = (size_t)router_tc_chunk_tokens(d.T),
                         ch = (size_t)router_tc_chunks(d.T);
            s.dw_part = take(ch * 3 * N * dm * 4);
            s.db_part = take(ch * N * 4);
            s.rdx_a = take(T * 6 * Np * 2);
            s.rdx_b = take(dm * 6 * Np * 2);
            s.rdw_a = take(ch * 3 * N * Tc * 2);
            s.chunk_counts = take((ch + 1) * 4);
        }
    }
    s.total = off;
    return s;
}

// ---- launch bookkeeping ----------------------------------------------------
std::atomic<int64_t> g_launches{0};

struct Tracer {
    std::mutex mu;
    bool on = false;
    int32_t max = 0;
    int32_t n = 0;
    std::vector<cudaEvent_t> events;  // 2 per launch
    std::vector<int32_t> ids;
};
Tracer &tracer() {
    static Tracer t;
    return t;
}

// ---- device properties ------------------------------------------------------
struct DeviceInfo {
    int sm_count = 0;
    bool sm100 = false;
    bool known = false;
};
DeviceInfo g_devices[64];
std::mutex g_dev_mu;

const DeviceInfo *current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo &info = g_devices[dev];
    if (!info.known) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return nullptr;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
        info.sm100 = major == 10;
        info.sm_count = sms;
        info.known = true;
    }
    return &info;
}

// ---- argument checks --------------------------------------------------------
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

switch_status_t check_dims(const switch_dims_t *d) {
    if (!d) return SWITCH_ERR_NULL;
    if (d->dtype != SWITCH_F32 && d->dtype != SWITCH_BF16) return SWITCH_ERR_DTYPE;
    if (d->T < 0 || d->T > INT32_MAX) return SWITCH_ERR_SHAPE;
    if (d->d_model < 1 || d->d_model > 8192) return SWITCH_ERR_SHAPE;
    if (d->d_ff < 1 || d->d_ff > 32768) return SWITCH_ERR_SHAPE;
    if (d->num_experts < 1 || d->num_experts > 256) return SWITCH_ERR_SHAPE;
    if (d->capacity < 1) return SWITCH_ERR_SHAPE;
    if ((int64_t)d->num_experts * d->capacity > INT32_MAX) return SWITCH_ERR_SHAPE;
    if (d->dtype == SWITCH_BF16 && (d->d_model % 64 != 0 || d->d_ff % 64 != 0)) return SWITCH_ERR_SHAPE;
    return SWITCH_OK;
}

// Pointers that must be present; all of them must also be 16-byte aligned.
switch_status_t check_ptrs(std::initializer_list<const void *> required, std::initializer_list<const void *> optional) {
    for (const void *p : required)
        if (!p) return SWITCH_ERR_NULL;
    for (const void *p : required)
        if (!aligned16(p)) return SWITCH_ERR_ALIGN;
    for (const void *p : optional)
        if (p && !aligned16(p)) return SWITCH_ERR_ALIGN;
    return SWITCH_OK;
}

switch_status_t check_device() {
    const DeviceInfo *info = current_device();
    if (!info) return SWITCH_ERR_CUDA;
    if (!info->sm100) return SWITCH_ERR_UNSUPPORTED;
    return SWITCH_OK;
}

switch_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? SWITCH_OK : SWITCH_ERR_CUDA; }

// One thread waits on an mbarrier whose phase never completes; the bounded
// wait gives up and records the timeout (tag 99), then the block exits.
__global__ void selftest_wait_kernel(DeviceStatus *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        status->code = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, status, 99);
}

}  // namespace

size_t workspace_bytes(const switch_dims_t &dims) { return layout(dims).total; }

size_t route_scratch_bytes(const switch_dims_t &dims) { return layout(dims).slot_token; }

Workspace carve_workspace(const switch_dims_t &dims, void *base) {
    const Sections s = layout(dims);
    uint8_t *b = static_cast<uint8_t *>(base);
    Workspace w;
    w.status = b + s.status;
    w.ticket = reinterpret_cast<uint32_t *>(b + s.ticket);
    w.hist = reinterpret_cast<int32_t *>(b + s.hist);
    w.psum = reinterpret_cast<float *>(b + s.psum);
    w.tile_off = reinterpret_cast<int32_t *>(b + s.tile_off);
    w.prob_total = reinterpret_cast<double *>(b + s.prob_total);
    w.w_split = b + s.w_split;
    w.slot_token = reinterpret_cast<int32_t *>(b + s.slot_token);
    w.xbuf = b + s.xbuf;
    w.ybuf = reinterpret_cast<float *>(b + s.ybuf);
    w.hidden = b + s.hidden;
    w.done = reinterpret_cast<int32_t *>(b + s.done);
    w.hist2 = reinterpret_cast<int32_t *>(b + s.hist2);
    w.tile_off2 = reinterpret_cast<int32_t *>(b + s.tile_off2);
    w.counts_first = reinterpret_cast<int32_t *>(b + s.counts_first);
    w.ent = (dims.flags & SWITCH_FLAG_ROUTER_STATS) ? reinterpret_cast<float *>(b + s.ent) : nullptr;
    const bool training = (dims.flags & SWITCH_FLAG_TRAINING) != 0;
    auto at = [&](size_t o) -> void * { return training ? (void *)(b + o) : nullptr; };
    w.probs = static_cast<float *>(at(s.probs));
    w.dh = static_cast<float *>(at(s.dh));
    w.grad_e = at(s.grad_e);
    w.grad_z = at(s.grad_z);
    w.dw_part = static_cast<float *>(at(s.dw_part));
    w.db_part = static_cast<float *>(at(s.db_part));
    w.rdx_a = at(s.rdx_a);
    w.rdx_b = at(s.rdx_b);
    w.rdw_a = at(s.rdw_a);
    w.chunk_counts = static_cast<int32_t *>(at(s.chunk_counts));
    w.tiles = tiles_of(dims);
    return w;
}

void launch_begin(int32_t kernel_id, cudaStream_t stream) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    Tracer &t = tracer();
    if (t.on && t.n < t.max) {
        t.ids[t.n] = kernel_id;
        cudaEventRecord(t.events[2 * t.n], stream);
    }
}

void launch_end(cudaStream_t stream) {
    Tracer &t = tracer();
    if (t.on && t.n < t.max) {
        cudaEventRecord(t.events[2 * t.n + 1], stream);
        ++t.n;
    }
}

int device_sm_count() {
    const DeviceInfo *info = current_device();
    return info ? info->sm_count : 148;
}

}  // namespace switchmoe

using namespace switchmoe;

extern "C" {

int64_t switch_capacity(int64_t T, int32_t num_experts, double c) {
    if (T < 0 || num_experts < 1 || !(c > 0.0) || !std::isfinite(c)) return -1;
    const double exact = (double)T / (double)num_experts * c;
    const double nearest = std::floor(exact + 0.5);
    double cap = std::fabs(exact - nearest) <= 1e-9 ? nearest : std::ceil(exact);
    if (cap < 1.0) cap = 1.0;
    return (int64_t)cap;
}

switch_status_t switch_workspace_size(const switch_dims_t *dims, size_t *bytes) {
    if (!bytes) return SWITCH_ERR_NULL;
    const switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    *bytes = workspace_bytes(*dims);
    return SWITCH_OK;
}

switch_status_t switch_route(const switch_dims_t *dims, const void *x, const float *w_r, const float *logit_bias,
                             int32_t *expert, float *gate, int32_t *slot, int32_t *counts, int32_t *slot_token,
                             float *aux, void *workspace, size_t workspace_bytes_given, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    const bool has_tokens = dims->T > 0;
    s = check_ptrs({w_r, counts, slot_token, aux, workspace,
                    has_tokens ? x : w_r, has_tokens ? (const void *)expert : w_r,
                    has_tokens ? (const void *)gate : w_r, has_tokens ? (const void *)slot : w_r},
                   {logit_bias, x, expert, gate, slot});
    if (s != SWITCH_OK) return s;
    if (workspace_bytes_given < workspace_bytes(*dims)) return SWITCH_ERR_WORKSPACE;
    if ((s = check_device()) != SWITCH_OK) return s;
    const Workspace ws = carve_workspace(*dims, workspace);
    return from_cuda(launch_route(*dims, x, w_r, logit_bias, expert, gate, slot, counts, slot_token, aux, ws,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

switch_status_t switch_dispatch(const switch_dims_t *dims, const void *x, const int32_t *slot_token,
                                const int32_t *counts, void *xbuf, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    s = check_ptrs({slot_token, counts, xbuf, dims->T > 0 ? x : xbuf}, {x});
    if (s != SWITCH_OK) return s;
    if ((s = check_device()) != SWITCH_OK) return s;
    return from_cuda(launch_dispatch(*dims, x, slot_token, counts, xbuf, reinterpret_cast<cudaStream_t>(stream)));
}

switch_status_t switch_expert_ffn(const switch_dims_t *dims, const void *xbuf, const void *w_in, const void *w_out,
                                  const int32_t *counts, void *ybuf, void *workspace, size_t workspace_bytes_given,
                                  switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    s = check_ptrs({xbuf, w_in, w_out, counts, ybuf, workspace}, {});
    if (s != SWITCH_OK) return s;
    if (workspace_bytes_given < workspace_bytes(*dims)) return SWITCH_ERR_WORKSPACE;
    if ((s = check_device()) != SWITCH_OK) return s;
    const Workspace ws = carve_workspace(*dims, workspace);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool tensor_cores = dims->dtype == SWITCH_BF16 && !(dims->flags & SWITCH_FLAG_SIMT_FFN);
    float *yb = static_cast<float *>(ybuf);
    if (cudaMemsetAsync(ws.status, 0, sizeof(DeviceStatus), st) != cudaSuccess) return SWITCH_ERR_CUDA;
    return from_cuda(tensor_cores ? launch_ffn_tc(*dims, xbuf, w_in, w_out, counts, yb, nullptr, nullptr, nullptr, ws, st)
                                  : launch_ffn_simt(*dims, xbuf, w_in, w_out, counts, yb, ws, st));
}

switch_status_t switch_combine(const switch_dims_t *dims, const void *ybuf, const int32_t *expert,
                               const int32_t *slot, const float *gate, void *y, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    if (dims->T > 0) {
        s = check_ptrs({ybuf, expert, slot, gate, y}, {});
        if (s != SWITCH_OK) return s;
    }
    if ((s = check_device()) != SWITCH_OK) return s;
    return from_cuda(launch_combine(*dims, static_cast<const float *>(ybuf), expert, slot, gate,
                                    static_cast<float *>(y), reinterpret_cast<cudaStream_t>(stream)));
}

switch_status_t switch_layer_fwd(const switch_dims_t *dims, const void *x, const float *w_r, const float *logit_bias,
                                 const void *w_in, const void *w_out, void *y, int32_t *expert, float *gate,
                                 int32_t *slot, int32_t *counts, float *aux, void *workspace,
                                 size_t workspace_bytes_given, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    const bool has_tokens = dims->T > 0;
    s = check_ptrs({w_r, w_in, w_out, counts, aux, workspace, has_tokens ? x : w_r, has_tokens ? y : w_r,
                    has_tokens ? (const void *)expert : w_r, has_tokens ? (const void *)gate : w_r,
                    has_tokens ? (const void *)slot : w_r},
                   {logit_bias, x, y, expert, gate, slot});
    if (s != SWITCH_OK) return s;
    if (workspace_bytes_given < workspace_bytes(*dims)) return SWITCH_ERR_WORKSPACE;
    if ((s = check_device()) != SWITCH_OK) return s;
    const Workspace ws = carve_workspace(*dims, workspace);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *yf = static_cast<float *>(y);
    const bool tensor_cores = dims->dtype == SWITCH_BF16 && !(dims->flags & SWITCH_FLAG_SIMT_FFN);
    const bool rows16 = ((int64_t)dims->d_model * (int64_t)elem_size(*dims)) % 16 == 0;
    cudaError_t err;
    if (small_layer_supported(*dims)) {
        err = launch_small_layer(*dims, x, w_r, logit_bias, w_in, w_out, yf, expert, gate, slot, counts, aux, ws, st);
    } else if (dims->flags & SWITCH_FLAG_TRAINING) {
        // training forward: keeps the router probabilities, xbuf, H and the ungated
        // expert output ybuf in the workspace for switch_layer_bwd
        if (!tensor_cores) return SWITCH_ERR_UNSUPPORTED;
        err = launch_route(*dims, x, w_r, logit_bias, expert, gate, slot, counts, ws.slot_token, aux, ws, st,
                           ws.xbuf, nullptr);
        if (err == cudaSuccess)
            err = launch_ffn_tc(*dims, ws.xbuf, w_in, w_out, counts, ws.ybuf, nullptr, nullptr, nullptr, ws, st);
        if (err == cudaSuccess) err = launch_combine(*dims, ws.ybuf, expert, slot, gate, yf, st);
    } else if (tensor_cores) {
        // route + scatter-dispatch (zeroing dropped rows of y), GEMM1, GEMM2 with
        // the gate and the token-order scatter fused into its epilogue
        err = launch_route(*dims, x, w_r, logit_bias, expert, gate, slot, counts, ws.slot_token, aux, ws, st,
                           ws.xbuf, yf, ws.done, fused_counter_ints(dims->num_experts, dims->capacity, dims->d_model));
        if (err == cudaSuccess)
            err = launch_ffn_tc(*dims, ws.xbuf, w_in, w_out, counts, nullptr, ws.slot_token, gate, yf, ws, st);
    } else {
        err = launch_route(*dims, x, w_r, logit_bias, expert, gate, slot, counts, ws.slot_token, aux, ws, st,
                           rows16 ? ws.xbuf : nullptr, nullptr);
        if (err == cudaSuccess && !rows16) err = launch_dispatch(*dims, x, ws.slot_token, counts, ws.xbuf, st);
        if (err == cudaSuccess) err = launch_ffn_simt(*dims, ws.xbuf, w_in, w_out, counts, ws.ybuf, ws, st);
        if (err == cudaSuccess) err = launch_combine(*dims, ws.ybuf, expert, slot, gate, yf, st);
    }
    return from_cuda(err);
}

switch_status_t switch_route_top2(const switch_dims_t *dims, const void *x, const float *w_r,
                                  const float *logit_bias, int32_t *expert, float *gate, int32_t *slot,
                                  int32_t *counts, int32_t *slot_token, float *aux, void *workspace,
                                  size_t workspace_bytes_given, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    if (dims->num_experts < 2) return SWITCH_ERR_SHAPE;
    const bool has_tokens = dims->T > 0;
    s = check_ptrs({w_r, counts, slot_token, aux, workspace,
                    has_tokens ? x : w_r, has_tokens ? (const void *)expert : w_r,
                    has_tokens ? (const void *)gate : w_r, has_tokens ? (const void *)slot : w_r},
                   {logit_bias, x, expert, gate, slot});
    if (s != SWITCH_OK) return s;
    if (workspace_bytes_given < workspace_bytes(*dims)) return SWITCH_ERR_WORKSPACE;
    if ((s = check_device()) != SWITCH_OK) return s;
    const Workspace ws = carve_workspace(*dims, workspace);
    return from_cuda(launch_route(*dims, x, w_r, logit_bias, expert, gate, slot, counts, slot_token, aux, ws,
                                  reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, 0, true));
}

switch_status_t switch_combine_top2(const switch_dims_t *dims, const void *ybuf, const int32_t *expert,
                                    const int32_t *slot, const float *gate, void *y, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    if (dims->num_experts < 2) return SWITCH_ERR_SHAPE;
    if (dims->T > 0) {
        s = check_ptrs({ybuf, expert, slot, gate, y}, {});
        if (s != SWITCH_OK) return s;
    }
    if ((s = check_device()) != SWITCH_OK) return s;
    return from_cuda(launch_combine_top2(*dims, static_cast<const float *>(ybuf), expert, slot, gate,
                                         static_cast<float *>(y), reinterpret_cast<cudaStream_t>(stream)));
}

switch_status_t switch_layer_fwd_top2(const switch_dims_t *dims, const void *x, const float *w_r,
                                      const float *logit_bias, const void *w_in, const void *w_out, void *y,
                                      int32_t *expert, float *gate, int32_t *slot, int32_t *counts, float *aux,
                                      void *workspace, size_t workspace_bytes_given, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    if (dims->num_experts < 2) return SWITCH_ERR_SHAPE;
    const bool has_tokens = dims->T > 0;
    s = check_ptrs({w_r, w_in, w_out, counts, aux, workspace, has_tokens ? x : w_r, has_tokens ? y : w_r,
                    has_tokens ? (const void *)expert : w_r, has_tokens ? (const void *)gate : w_r,
                    has_tokens ? (const void *)slot : w_r},
                   {logit_bias, x, y, expert, gate, slot});
    if (s != SWITCH_OK) return s;
    if (workspace_bytes_given < workspace_bytes(*dims)) return SWITCH_ERR_WORKSPACE;
    if ((s = check_device()) != SWITCH_OK) return s;
    const Workspace ws = carve_workspace(*dims, workspace);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool tensor_cores = dims->dtype == SWITCH_BF16 && !(dims->flags & SWITCH_FLAG_SIMT_FFN);
    const bool rows16 = ((int64_t)dims->d_model * (int64_t)elem_size(*dims)) % 16 == 0;
    // route (+ scatter-dispatch of both choices), expert FFN into ybuf, top-2 combine
    cudaError_t err = launch_route(*dims, x, w_r, logit_bias, expert, gate, slot, counts, ws.slot_token, aux, ws, st,
                                   rows16 ? ws.xbuf : nullptr, nullptr, nullptr, 0, true);
    if (err == cudaSuccess && !rows16) err = launch_dispatch(*dims, x, ws.slot_token, counts, ws.xbuf, st);
    // the expert GEMMs see up to 2T kept rows (their grid is sized from that bound)
    switch_dims_t rows = *dims;
    rows.T = 2 * dims->T;
    // (two launches: with ~2T rows both GEMMs have many tiles, and the persistent
    // fused kernel measured slower here: 2.13 against 2.04 ms on the Switch-Large shape)
    if (err == cudaSuccess)
        err = tensor_cores ? launch_ffn_tc(rows, ws.xbuf, w_in, w_out, counts, ws.ybuf, nullptr, nullptr, nullptr, ws,
                                           st)
                           : launch_ffn_simt(rows, ws.xbuf, w_in, w_out, counts, ws.ybuf, ws, st);
    if (err == cudaSuccess) err = launch_combine_top2(*dims, ws.ybuf, expert, slot, gate, static_cast<float *>(y), st);
    return from_cuda(err);
}

switch_status_t switch_router_stats(const switch_dims_t *dims, const int32_t *counts, const void *workspace,
                                    size_t workspace_bytes_given, float *stats, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    s = check_ptrs({counts, workspace, stats}, {});
    if (s != SWITCH_OK) return s;
    if (workspace_bytes_given < workspace_bytes(*dims)) return SWITCH_ERR_WORKSPACE;
    if ((s = check_device()) != SWITCH_OK) return s;
    const Workspace ws = carve_workspace(*dims, const_cast<void *>(workspace));
    return from_cuda(launch_router_stats(*dims, counts, ws, stats, reinterpret_cast<cudaStream_t>(stream)));
}

switch_status_t switch_layer_bwd(const switch_dims_t *dims, const void *x, const float *w_r, const void *w_in,
                                 const void *w_out, const int32_t *expert, const float *gate, const int32_t *slot,
                                 const int32_t *counts, const float *dy, float g_aux, float *dx, float *dw_r,
                                 float *dbias, float *dw_in, float *dw_out, void *workspace,
                                 size_t workspace_bytes_given, switch_stream_t stream) {
    switch_status_t s = check_dims(dims);
    if (s != SWITCH_OK) return s;
    if (!(dims->flags & SWITCH_FLAG_TRAINING)) return SWITCH_ERR_UNSUPPORTED;
    if (dims->dtype != SWITCH_BF16 || (dims->flags & (SWITCH_FLAG_SIMT_FFN | SWITCH_FLAG_GEMM_1CTA)))
        return SWITCH_ERR_UNSUPPORTED;
    const bool has_tokens = dims->T > 0;
    s = check_ptrs({w_r, w_in, w_out, counts, dw_r, dw_in, dw_out, workspace, has_tokens ? x : w_r,
                    has_tokens ? (const void *)expert : w_r, has_tokens ? (const void *)gate : w_r,
                    has_tokens ? (const void *)slot : w_r, has_tokens ? (const void *)dy : w_r,
                    has_tokens ? (const void *)dx : w_r},
                   {x, expert, gate, slot, dy, dx, dbias});
    if (s != SWITCH_OK) return s;
    if (!std::isfinite(g_aux)) return SWITCH_ERR_SHAPE;
    if (workspace_bytes_given < workspace_bytes(*dims)) return SWITCH_ERR_WORKSPACE;
    if ((s = check_device()) != SWITCH_OK) return s;
    const Workspace ws = carve_workspace(*dims, workspace);
    return from_cuda(launch_layer_bwd(*dims, x, w_r, w_in, w_out, expert, gate, slot, counts, dy, g_aux, dx, dw_r,
                                      dbias, dw_in, dw_out, ws, reinterpret_cast<cudaStream_t>(stream)));
}

switch_status_t switch_check(void *workspace, size_t workspace_bytes_given, switch_stream_t stream) {
    if (!workspace) return SWITCH_ERR_NULL;
    if (workspace_bytes_given < sizeof(DeviceStatus)) return SWITCH_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    DeviceStatus host{};
    if (cudaStreamSynchronize(st) != cudaSuccess) return SWITCH_ERR_CUDA;
    if (cudaMemcpyAsync(&host, workspace, sizeof host, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return SWITCH_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof host, st) != cudaSuccess) return SWITCH_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SWITCH_ERR_CUDA;
    return host.code == 0 ? SWITCH_OK : (switch_status_t)host.code;
}

switch_status_t switch_selftest_wait_timeout(void *workspace, size_t workspace_bytes_given, switch_stream_t stream) {
    if (!workspace) return SWITCH_ERR_NULL;
    if (!aligned16(workspace)) return SWITCH_ERR_ALIGN;
    if (workspace_bytes_given < sizeof(DeviceStatus)) return SWITCH_ERR_WORKSPACE;
    switch_status_t s = check_device();
    if (s != SWITCH_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    launch_begin(K_SELFTEST_WAIT, st);
    selftest_wait_kernel<<<1, 32, 0, st>>>(static_cast<DeviceStatus *>(workspace));
    const cudaError_t err = cudaGetLastError();
    launch_end(st);
    return from_cuda(err);
}

const char *switch_status_string(switch_status_t status) {
    switch (status) {
        case SWITCH_OK: return "ok";
        case SWITCH_ERR_NULL: return "a required pointer is NULL";
        case SWITCH_ERR_SHAPE: return "a size is out of range or breaks a divisibility rule";
        case SWITCH_ERR_DTYPE: return "unknown dtype";
        case SWITCH_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case SWITCH_ERR_WORKSPACE: return "workspace too small";
        case SWITCH_ERR_UNSUPPORTED: return "unsupported on this device (needs sm_100)";
        case SWITCH_ERR_CUDA: return "CUDA error";
        case SWITCH_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
        case SWITCH_ERR_TOO_LARGE: return "needs more scratch than the library's static buffer holds";
    }
    return "unknown status";
}

int64_t switch_launch_count(void) { return g_launches.load(); }

switch_status_t switch_trace_start(int32_t max_launches) {
    if (max_launches < 1) return SWITCH_ERR_SHAPE;
    Tracer &t = tracer();
    std::lock_guard<std::mutex> lock(t.mu);
    for (cudaEvent_t e : t.events) cudaEventDestroy(e);
    t.events.assign(2 * (size_t)max_launches, nullptr);
    t.ids.assign((size_t)max_launches, 0);
    for (auto &e : t.events)
        if (cudaEventCreate(&e) != cudaSuccess) return SWITCH_ERR_CUDA;
    t.max = max_launches;
    t.n = 0;
    t.on = true;
    return SWITCH_OK;
}

int32_t switch_trace_read(int32_t *kernel_id, float *ms, int32_t capacity) {
    Tracer &t = tracer();
    std::lock_guard<std::mutex> lock(t.mu);
    const int32_t n = std::min(t.n, capacity);
    for (int32_t k = 0; k < n; ++k) {
        float v = -1.f;
        if (cudaEventSynchronize(t.events[2 * k + 1]) == cudaSuccess)
            cudaEventElapsedTime(&v, t.events[2 * k], t.events[2 * k + 1]);
        if (kernel_id) kernel_id[k] = t.ids[k];
        if (ms) ms[k] = v;
    }
    return n;
}

void switch_trace_stop(void) {
    Tracer &t = tracer();
    std::lock_guard<std::mutex> lock(t.mu);
    t.on = false;
    t.n = 0;
    for (cudaEvent_t e : t.events) cudaEventDestroy(e);
    t.events.clear();
    t.ids.clear();
    t.max = 0;
}

const char *switch_kernel_name(int32_t id) {
    switch (id) {
        case K_ROUTER_WARP: return "router_warp";
        case K_ROUTER_TILED: return "router_tiled";
        case K_SCAN: return "capacity_scan";
        case K_ASSIGN: return "slot_assign";
        case K_DISPATCH: return "dispatch";
        case K_FFN_TC_GEMM1: return "ffn_tc_gemm1_relu";
        case K_FFN_TC_GEMM2: return "ffn_tc_gemm2";
        case K_FFN_SIMT_GEMM1: return "ffn_simt_gemm1_relu";
        case K_FFN_SIMT_GEMM2: return "ffn_simt_gemm2";
        case K_COMBINE: return "combine";
        case K_FFN_TC_GEMM2_GATED: return "ffn_tc_gemm2_gated_scatter";
        case K_ASSIGN_SCATTER: return "slot_assign_scatter";
        case K_ROUTER_STAGED: return "router_staged";
        case K_ROUTER_TC: return "router_tc";
        case K_ROUTER_SPLIT: return "router_weight_split";
        case K_SELFTEST_WAIT: return "selftest_wait_timeout";
        case K_FFN_TC_FUSED: return "ffn_tc_fused";
        case K_COMBINE_TOP2: return "combine_top2";
        case K_BWD_TOKEN: return "bwd_gate_softmax";
        case K_BWD_GEMM_DZ: return "bwd_tc_gemm_dz";
        case K_BWD_GEMM_DX: return "bwd_tc_gemm_dx";
        case K_BWD_GEMM_DW: return "bwd_tc_gemm_dw";
        case K_BWD_ROUTER_DX: return "bwd_router_dx";
        case K_BWD_ROUTER_DW: return "bwd_router_dw";
        case K_BWD_REDUCE: return "bwd_reduce";
        case K_ROUTER_STATS: return "router_stats";
        case K_SMALL_LAYER: return "small_layer";
        case K_BWD_ROUTER_SPLIT: return "bwd_router_split";
        case K_BWD_ROUTER_TC_DX: return "bwd_router_tc_dx";
        case K_BWD_ROUTER_TC_DW: return "bwd_router_tc_dw";
        case K_BWD_ZERO_TAILS: return "bwd_zero_tails";
    }
    return "?";
}

}  // extern "C"
