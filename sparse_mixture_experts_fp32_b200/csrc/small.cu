// The whole layer in one thread block, for small float32 layers (T <= 256
// tokens, N <= 32 experts, x, W_r and all expert weights together in shared
// memory): router logits, softmax, top-1 (lowest index on ties), gate,
// capacity assignment in token order, aux loss, the expert FFN of every kept
// token with its hidden activations in shared memory, and the gated combine
// (zero rows for dropped tokens), in one launch instead of five
// (llm-papers-study "精读 06 | Switch Transformers" §3.1-§3.4; the expert body
// d -> d_ff -> ReLU -> d as in the multi-kernel path).
#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr int kSmallThreads = 256;
constexpr int kSmallMaxT = 256;
constexpr int kSmallMaxN = 32;

// Rows in shared memory have odd pitches (d | 1, F | 1 floats), so that the 32
// lanes of a warp reading one element of 32 different rows hit 32 different
// banks (with a pitch of 32 or 64 floats they all hit one bank, and the layer
// ran about 10x slower).
struct SmallLayout {
    int pd, pf;  // row pitches (floats) of x / W_r / W_in rows and of W_out rows
    int64_t x, wr, win, wout, h, logit, gate_s, expert_s, slot_s, total;  // float offsets
};
__host__ __device__ inline SmallLayout small_layout(int T, int d, int F, int N) {
    SmallLayout L{};
    L.pd = d | 1;
    L.pf = F | 1;
    int64_t o = 0;
    auto take = [&](int64_t n) { const int64_t at = o; o += (n + 3) / 4 * 4; return at; };
    L.x = take((int64_t)T * L.pd);
    L.wr = take((int64_t)N * L.pd);
    L.win = take((int64_t)N * F * L.pd);
    L.wout = take((int64_t)N * d * L.pf);
    L.h = take((int64_t)(kSmallThreads / 32) * F);  // one hidden row per warp
    L.logit = take((int64_t)T * N);                  // logits, then probabilities
    L.gate_s = take(T);
    L.expert_s = take(T);
    L.slot_s = take(T);
    L.total = o;
    return L;
}

// Copies an [n / cols][cols] float32 matrix into shared-memory rows of `pitch`
// floats.  Each thread keeps eight 16-byte loads in flight before it stores
// them (a load-then-store loop left every load's latency exposed).
// (The layer's arrays hold at most 160 KB here, so 32-bit indices suffice: a
// 64-bit division per element cost more than the loads.)
__device__ __forceinline__ void load_rows(float *dst, const float *__restrict__ src, int n, int cols, int pitch) {
    const bool vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    const int n4 = vec ? n / 4 : 0;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    for (int base = threadIdx.x; base < n4; base += 8 * kSmallThreads) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * kSmallThreads;
            if (i < n4) v[u] = __ldg(s4 + i);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * kSmallThreads;
            if (i < n4) {
                const float c[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                int row = (4 * i) / cols, col = 4 * i - row * cols;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    dst[row * pitch + col] = c[q];
                    if (++col == cols) {
                        col = 0;
                        ++row;
                    }
                }
            }
        }
    }
    for (int k = 4 * n4 + threadIdx.x; k < n; k += kSmallThreads) dst[k / cols * pitch + k % cols] = src[k];
}

// sum_k a[k] b[k] over k < n, in four interleaved partial sums (k mod 4) added
// as (s0 + s1) + (s2 + s3): four independent FMA chains instead of one.
__device__ __forceinline__ float dot4(const float *a, const float *b, int n) {
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int k = 0;
#pragma unroll 4
    for (; k + 4 <= n; k += 4) {
        s0 = fmaf(a[k], b[k], s0);
        s1 = fmaf(a[k + 1], b[k + 1], s1);
        s2 = fmaf(a[k + 2], b[k + 2], s2);
        s3 = fmaf(a[k + 3], b[k + 3], s3);
    }
    for (; k < n; ++k) s0 = fmaf(a[k], b[k], s0);
    return (s0 + s1) + (s2 + s3);
}

__global__ void __launch_bounds__(kSmallThreads, 1)
    small_layer_kernel(const float *__restrict__ x, const float *__restrict__ w_r, const float *__restrict__ bias,
                       const float *__restrict__ w_in, const float *__restrict__ w_out, int T, int d, int F, int N,
                       int C, float *__restrict__ y, int32_t *__restrict__ expert, float *__restrict__ gate,
                       int32_t *__restrict__ slot, int32_t *__restrict__ counts, float *__restrict__ aux,
                       DeviceStatus *status) {
    extern __shared__ __align__(16) float sm[];
    const SmallLayout L = small_layout(T, d, F, N);
    float *xs = sm + L.x, *wrs = sm + L.wr, *wis = sm + L.win, *wos = sm + L.wout, *hs = sm + L.h;
    float *lg = sm + L.logit, *gs = sm + L.gate_s;
    int32_t *es = reinterpret_cast<int32_t *>(sm + L.expert_s);
    int32_t *ss = reinterpret_cast<int32_t *>(sm + L.slot_s);
    __shared__ double psum_s[kSmallMaxN];
    __shared__ int32_t cnt_s[kSmallMaxN];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        status->code = 0;
        status->where = 0;
        status->block = 0;
        status->reserved = 0;
    }
    const int pd = L.pd, pf = L.pf;
    // All four arrays start on their way to L2 at once; then they are staged one after the other.
    if (tid < 4) {
        const float *src = tid == 0 ? x : tid == 1 ? w_r : tid == 2 ? w_in : w_out;
        const int n = tid == 0 ? T * d : tid == 1 ? N * d : N * F * d;
        const uint32_t bytes = (uint32_t)n * 4u & ~15u;
        if (bytes > 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
    }
    load_rows(xs, x, T * d, d, pd);
    load_rows(wrs, w_r, N * d, d, pd);
    load_rows(wis, w_in, N * F * d, d, pd);   // rows (e, j) of W_in
    load_rows(wos, w_out, N * d * F, F, pf);  // rows (e, k) of W_out
    __syncthreads();
    // router logits, one (token, expert) pair per thread at a time
    for (int q = tid; q < T * N; q += kSmallThreads) {
        const int t = q / N, i = q % N;
        lg[q] = dot4(xs + t * pd, wrs + i * pd, d) + (bias ? bias[i] : 0.f);
    }
    __syncthreads();
    // softmax, argmax (lowest index on ties), gate: one thread per token
    for (int t = tid; t < T; t += kSmallThreads) {
        float *row = lg + t * N;
        float m = row[0];
        int arg = 0;
        for (int i = 1; i < N; ++i)
            if (row[i] > m) {
                m = row[i];
                arg = i;
            }
        float s = 0.f;
        for (int i = 0; i < N; ++i) {
            row[i] = expf(row[i] - m);
            s += row[i];
        }
        for (int i = 0; i < N; ++i) row[i] = row[i] / s;
        es[t] = arg;
        gs[t] = 1.0f / s;
        expert[t] = arg;
        gate[t] = 1.0f / s;
    }
    __syncthreads();
    // capacity: the slot of token t is the number of earlier tokens of its expert
    for (int t = tid; t < T; t += kSmallThreads) {
        const int e = es[t];
        int before = 0;
        for (int u = 0; u < t; ++u) before += es[u] == e;
        const int s_ = before < C ? before : -1;
        ss[t] = s_;
        slot[t] = s_;
    }
    // counts and the probability sums per expert (fp64), then aux
    // (a warp per expert: lane-strided partial sums, then a fixed xor tree)
    for (int i = warp; i < N; i += kSmallThreads / 32) {
        int c = 0;
        double p = 0.0;
        for (int t = lane; t < T; t += 32) {
            c += es[t] == i;
            p += (double)lg[t * N + i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            c += __shfl_xor_sync(0xffffffffu, c, off);
            p += __shfl_xor_sync(0xffffffffu, p, off);
        }
        if (lane == 0) {
            cnt_s[i] = c;
            psum_s[i] = p;
            counts[i] = c;
        }
    }
    __syncthreads();
    if (tid == 0) {
        double total = 0.0;
        for (int i = 0; i < N; ++i) total += ((double)cnt_s[i] / (double)T) * (psum_s[i] / (double)T);
        *aux = T > 0 ? (float)((double)N * total) : 0.f;
    }
    // expert FFN + gated combine: one warp per token, its hidden row in shared memory
    float *hrow = hs + warp * F;
    for (int t = warp; t < T; t += kSmallThreads / 32) {
        float *yt = y + (int64_t)t * d;
        const int s_ = ss[t];
        if (s_ < 0) {
            for (int k = lane; k < d; k += 32) yt[k] = 0.f;
            continue;
        }
        const int e = es[t];
        const float *wi = wis + (int64_t)e * F * pd, *wo = wos + (int64_t)e * d * pf, *xt = xs + t * pd;
        for (int j = lane; j < F; j += 32) hrow[j] = fmaxf(dot4(wi + j * pd, xt, d), 0.f);
        __syncwarp();
        const float g = gs[t];
        for (int k = lane; k < d; k += 32) yt[k] = g * dot4(wo + k * pf, hrow, F);
        __syncwarp();
    }
}

}  // namespace

bool small_layer_supported(const switch_dims_t &dims) {
    if (dims.dtype != SWITCH_F32 || dims.T < 1 || dims.T > kSmallMaxT || dims.num_experts > kSmallMaxN) return false;
    if (dims.flags & (SWITCH_FLAG_MULTI_KERNEL | SWITCH_FLAG_TRAINING | SWITCH_FLAG_ROUTER_STATS)) return false;
    const SmallLayout L = small_layout((int)dims.T, dims.d_model, dims.d_ff, dims.num_experts);
    return (size_t)L.total * sizeof(float) <= 160 * 1024;
}

cudaError_t launch_small_layer(const switch_dims_t &dims, const void *x, const float *w_r, const float *bias,
                               const void *w_in, const void *w_out, float *y, int32_t *expert, float *gate,
                               int32_t *slot, int32_t *counts, float *aux, const Workspace &ws, cudaStream_t stream) {
    const int T = (int)dims.T, d = dims.d_model, F = dims.d_ff, N = dims.num_experts;
    const size_t smem = (size_t)small_layout(T, d, F, N).total * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(small_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    launch_begin(K_SMALL_LAYER, stream);
    small_layer_kernel<<<1, kSmallThreads, smem, stream>>>(
        static_cast<const float *>(x), w_r, bias, static_cast<const float *>(w_in), static_cast<const float *>(w_out),
        T, d, F, N, dims.capacity, y, expert, gate, slot, counts, aux, static_cast<DeviceStatus *>(ws.status));
    err = cudaGetLastError();
    launch_end(stream);
    return err;
}

}  // namespace switchmoe
