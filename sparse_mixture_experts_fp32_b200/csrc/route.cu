// Router, top-1, capacity scan and slot assignment (sm_100a).
//
//   router  h = W_r . x (+ b) in float32; p = softmax(h); expert = argmax
//           (lowest index on ties); gate = p[expert]; per 64-token tile:
//           tokens per expert and sum of p_i.
//           (llm-papers-study "精读 06 | Switch Transformers" §3.1-§3.2;
//           kasblo "Switch Transformerとは？" section "Routerだけfloat32で
//           計算するSelective Precision": router arithmetic in float32.)
//   scan    per expert, exclusive prefix of the tile counts -> each tile's
//           first slot; totals -> counts; fp64 sum of p_i -> aux loss
//           N * sum_i (counts_i / T) * (P_i / T)   (llm-papers-study §3.3).
//   assign  slot of a token = its tile's first slot for its expert + its
//           rank among the tile's tokens of that expert; kept iff slot < C
//           (llm-papers-study §3.4; Incredible.AI "MoE Layer": the first C
//           tokens of each expert in token order are kept).
#include <float.h>

#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ int lanemask_lt() {
    int m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Per-token softmax / top-1 (or top-2) bookkeeping, done by one warp.  Each
// lane holds up to J logits: value v[j] for expert idx[j] (idx < 0: not held).
// Every expert is held by exactly one "owner" lane (own[j] true); other lanes
// may hold copies, which take part in the max but not in the sums.  With
// TOP2 the warp also finds the second choice (the largest logit among the
// other experts, lowest index on ties) and writes both choices of token t to
// expert[2t], expert[2t+1] and their probabilities to gate[2t], gate[2t+1].
__device__ __forceinline__ bool better(float v, int i, float m, int a) { return v > m || (v == m && i < a); }

template <int J, bool TOP2>
__device__ __forceinline__ void token_epilogue(const float (&v)[J], const int (&idx)[J], const bool (&own)[J],
                                               int64_t t, float *warp_psum, int32_t *warp_hist,
                                               int32_t *warp_hist2, int32_t *expert, float *gate, float *probs,
                                               int N, float *warp_ent) {
    const int lane = threadIdx.x & 31;
    float m = -FLT_MAX;
    int arg = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        if (idx[j] >= 0 && better(v[j], idx[j], m, arg)) {
            m = v[j];
            arg = idx[j];
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, m, off);
        const int oa = __shfl_xor_sync(0xffffffffu, arg, off);
        if (better(om, oa, m, arg)) {
            m = om;
            arg = oa;
        }
    }
    if (arg == 0x7fffffff) arg = 0;  // no comparable logit (NaN inputs): keep every index in range
    float m2 = -FLT_MAX;
    int arg2 = 0x7fffffff;
    if (TOP2) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            if (idx[j] >= 0 && idx[j] != arg && better(v[j], idx[j], m2, arg2)) {
                m2 = v[j];
                arg2 = idx[j];
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, m2, off);
            const int oa = __shfl_xor_sync(0xffffffffu, arg2, off);
            if (better(om, oa, m2, arg2)) {
                m2 = om;
                arg2 = oa;
            }
        }
        if (arg2 == 0x7fffffff) arg2 = arg == 0 ? 1 : 0;
    }
    float ex[J];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        ex[j] = (idx[j] >= 0 && own[j]) ? expf(v[j] - m) : 0.f;
        s += ex[j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (warp_ent) {  // entropy -sum p ln p = ln s - sum e (v - m) / s
        float sv = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j)
            if (idx[j] >= 0 && own[j]) sv += ex[j] * (v[j] - m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sv += __shfl_xor_sync(0xffffffffu, sv, off);
        if (lane == 0) *warp_ent += logf(s) - sv / s;
    }
#pragma unroll
    for (int j = 0; j < J; ++j)
        if (idx[j] >= 0 && own[j]) {
            warp_psum[idx[j]] += ex[j] / s;
            if (probs) probs[t * N + idx[j]] = ex[j] / s;  // kept for the backward pass
        }
    if (lane == 0) {
        warp_hist[arg] += 1;
        if (TOP2) {
            warp_hist2[arg2] += 1;
            expert[2 * t] = arg;
            expert[2 * t + 1] = arg2;
            gate[2 * t] = 1.0f / s;  // p at the argmax: exp(0) / s
            gate[2 * t + 1] = expf(m2 - m) / s;
        } else {
            expert[t] = arg;
            gate[t] = 1.0f / s;  // p at the argmax: exp(0) / s
        }
    }
}

// Sum the per-warp partials of a tile in fixed warp order and publish them
// expert-major ([N][tiles]) for the scan (with hist2: second-choice counts too).
__device__ __forceinline__ void publish_tile(const float *psum_w, const int32_t *hist_w, const int32_t *hist2_w,
                                             int N, int tiles, int tile, int32_t *hist, int32_t *hist2,
                                             float *psum, const float *ent_w, float *ent) {
    if (ent && threadIdx.x == 0) {  // the tile's entropy sum, warps in fixed order
        float e = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) e += ent_w[w];
        ent[tile] = e;
    }
    for (int i = threadIdx.x; i < N; i += kThreads) {
        int32_t c = 0, c2 = 0;
        float p = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            c += hist_w[w * N + i];
            if (hist2) c2 += hist2_w[w * N + i];
            p += psum_w[w * N + i];
        }
        hist[(int64_t)i * tiles + tile] = c;
        if (hist2) hist2[(int64_t)i * tiles + tile] = c2;
        psum[(int64_t)i * tiles + tile] = p;
    }
}

// The first block of a routing call resets the scan ticket and the status
// word of the workspace (which the caller may hand over uninitialised).
__device__ __forceinline__ void reset_call_state(uint32_t *ticket, DeviceStatus *status) {
    *ticket = 0u;
    status->code = 0;
    status->where = 0;
    status->block = 0;
    status->reserved = 0;
}

template <typename XT>
struct XLoad;
template <>
struct XLoad<__nv_bfloat16> {
    static constexpr int V = 8;  // elements per 16-byte vector
    static __device__ __forceinline__ void vec(const __nv_bfloat16 *p, float (&o)[V]) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ float one(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    // the same 16-byte vector read through a generic pointer (shared memory)
    static __device__ __forceinline__ void vec_generic(const __nv_bfloat16 *p, float (&o)[V]) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <>
struct XLoad<float> {
    static constexpr int V = 4;
    static __device__ __forceinline__ void vec(const float *p, float (&o)[V]) {
        const float4 raw = __ldg(reinterpret_cast<const float4 *>(p));
        o[0] = raw.x;
        o[1] = raw.y;
        o[2] = raw.z;
        o[3] = raw.w;
    }
    static __device__ __forceinline__ float one(const float *p) { return *p; }
    static __device__ __forceinline__ void vec_generic(const float *p, float (&o)[V]) {
        const float4 raw = *reinterpret_cast<const float4 *>(p);
        o[0] = raw.x;
        o[1] = raw.y;
        o[2] = raw.z;
        o[3] = raw.w;
    }
};

// ---------------------------------------------------------------------------
// Router for N <= 32: one warp per token, W_r resident in shared memory as
// [d][NP] (NP = N rounded up to a power of two >= 8).  Each lane accumulates
// NP partial dot products over its share of d; a halving exchange then
// leaves lane L with the full logit of expert L >> (5 - log2 NP).
// ---------------------------------------------------------------------------
template <typename XT, int NP, bool TOP2>
__global__ void __launch_bounds__(kThreads) router_warp_kernel(const XT *__restrict__ x, const float *__restrict__ w_r,
                                                               const float *__restrict__ bias, int64_t T, int d,
                                                               int N, int tiles, int32_t *__restrict__ expert,
                                                               float *__restrict__ gate, int32_t *__restrict__ hist,
                                                               int32_t *__restrict__ hist2,
                                                               float *__restrict__ psum, float *__restrict__ probs,
                                                               float *__restrict__ ent, uint32_t *ticket,
                                                               DeviceStatus *status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *wsm = reinterpret_cast<float *>(smem_raw);  // [d][NP]
    float *psum_w = wsm + (size_t)d * NP;               // [kWarps][N]
    int32_t *hist_w = reinterpret_cast<int32_t *>(psum_w + kWarps * N);
    int32_t *hist2_w = hist_w + kWarps * N;             // [kWarps][N] second choices (TOP2)
    float *ent_w = reinterpret_cast<float *>(hist2_w + kWarps * N);  // [kWarps] entropy sums
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x;

    if (tile == 0 && tid == 0) reset_call_state(ticket, status);
    if (tid < kWarps) ent_w[tid] = 0.f;
    for (int i = tid; i < d * NP; i += kThreads) {
        const int k = i / NP, e = i % NP;
        wsm[i] = e < N ? w_r[(int64_t)e * d + k] : 0.f;
    }
    for (int i = tid; i < kWarps * N; i += kThreads) {
        psum_w[i] = 0.f;
        hist_w[i] = 0;
        if (TOP2) hist2_w[i] = 0;
    }
    __syncthreads();

    constexpr int LOG_NP = NP == 8 ? 3 : NP == 16 ? 4 : 5;
    constexpr int SHIFT = 5 - LOG_NP;
    const int my_e = lane >> SHIFT;
    const bool valid_e = my_e < N;
    const float my_bias = (bias && valid_e) ? bias[my_e] : 0.f;
    constexpr int V = XLoad<XT>::V;
    const bool vec_ok = (d % V) == 0;

    for (int r = warp; r < kTileT; r += kWarps) {
        const int64_t t = (int64_t)tile * kTileT + r;
        if (t >= T) break;
        const XT *xr = x + t * d;
        float acc[NP];
#pragma unroll
        for (int e = 0; e < NP; ++e) acc[e] = 0.f;
        if (vec_ok) {
            for (int k = lane * V; k < d; k += 32 * V) {
                float xv[V];
                XLoad<XT>::vec(xr + k, xv);
#pragma unroll
                for (int u = 0; u < V; ++u) {
                    const float4 *wrow = reinterpret_cast<const float4 *>(wsm + (size_t)(k + u) * NP);
#pragma unroll
                    for (int q = 0; q < NP / 4; ++q) {
                        const float4 w4 = wrow[q];
                        acc[4 * q + 0] = fmaf(xv[u], w4.x, acc[4 * q + 0]);
                        acc[4 * q + 1] = fmaf(xv[u], w4.y, acc[4 * q + 1]);
                        acc[4 * q + 2] = fmaf(xv[u], w4.z, acc[4 * q + 2]);
                        acc[4 * q + 3] = fmaf(xv[u], w4.w, acc[4 * q + 3]);
                    }
                }
            }
        } else {
            for (int k = lane; k < d; k += 32) {
                const float xv = XLoad<XT>::one(xr + k);
#pragma unroll
                for (int e = 0; e < NP; ++e) acc[e] = fmaf(xv, wsm[(size_t)k * NP + e], acc[e]);
            }
        }
        // Halving exchange: after step s, a lane keeps the half of its
        // remaining values selected by lane bit (4 - s) and adds the
        // partner's copy of that half.
#pragma unroll
        for (int step = 0; step < 5; ++step) {
            const int off = 16 >> step;
            const int n = NP >> step;  // values still held per lane
            if (n > 1) {
                const bool upper = (lane & off) != 0;
                const int half = n / 2;
#pragma unroll
                for (int i = 0; i < NP / 2; ++i) {
                    if (i < half) {
                        const float send = upper ? acc[i] : acc[i + half];
                        const float keep = upper ? acc[i + half] : acc[i];
                        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                    }
                }
            } else {
                acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], off);
            }
        }
        float v[1] = {acc[0] + my_bias};
        int idx[1] = {valid_e ? my_e : -1};
        bool own[1] = {(lane & ((1 << SHIFT) - 1)) == 0};
        token_epilogue<1, TOP2>(v, idx, own, t, psum_w + warp * N, hist_w + warp * N, hist2_w + warp * N, expert,
                                gate, probs, N, ent ? ent_w + warp : nullptr);
    }
    __syncthreads();
    publish_tile(psum_w, hist_w, hist2_w, N, tiles, tile, hist, TOP2 ? hist2 : nullptr, psum, ent_w, ent);
}

// ---------------------------------------------------------------------------
// Router for N <= 32 with the whole 64-token tile of x staged in shared
// memory.  One bulk copy per 16-token chunk (the rows are contiguous) completes
// on the chunk's mbarrier, so the first warps start while later rows still land;
// W_r is loaded meanwhile as [d/V][V][NP] (+4 floats of padding per j).
// A register-blocked skinny GEMM: thread (group, part) accumulates 4 tokens
// x NP experts over the 16-byte x vectors j = part, part + 16, ..., so each
// W_r value read from shared memory serves four tokens; four shuffles sum the
// 16 parts.  Softmax, argmax and gate per token in registers; the tile's sum
// of p is formed in fixed token order (deterministic).
// ---------------------------------------------------------------------------
// Threads of the staged router: 16 groups of 4 tokens of a 64-token tile,
// each group one warp (NP <= 16) or half a warp (NP = 32: 4 x 32 accumulators
// per thread, which 512 threads' register budget cannot hold).
__host__ __device__ constexpr int staged_threads(int NP) { return NP <= 16 ? 512 : 256; }

template <typename XT>
struct Staged {
    static constexpr int V = XLoad<XT>::V;
    static __host__ __device__ int64_t xpitch(int d) { return (int64_t)d * sizeof(XT); }
    static __host__ __device__ int64_t wpitch(int NP) { return (int64_t)V * NP + 4; }  // floats per 16-byte x vector of W_r
    // The x tile region is reused for the per-token probabilities at the end.
    static __host__ __device__ int64_t x_region(int d, int NP) {
        const int64_t a = kTileT * xpitch(d), b = (int64_t)kTileT * NP * 4;
        return ((a > b ? a : b) + 15) / 16 * 16;
    }
    // smem layout: x tile | W_r as [d/V][V][NP] | counts | second-choice counts |
    // per-token entropies [64] | 5 mbarriers | raw W_r (optional)
    static size_t smem_base(int d, int NP) {
        return (size_t)x_region(d, NP) + (size_t)((d / V) * wpitch(NP)) * 4 +
               2 * (size_t)NP * 4 + kTileT * 4 + 5 * 8 + 16;
    }
    static size_t smem(int d, int NP, int N, bool raw) {
        return smem_base(d, NP) + (raw ? (size_t)N * d * 4 + 16 : 0);
    }
};

template <typename XT, int NP, bool TOP2>
__global__ void __launch_bounds__(staged_threads(NP), 1)
    router_staged_kernel(const XT *__restrict__ x, const float *__restrict__ w_r, const float *__restrict__ bias,
                         int64_t T, int d, int N, int tiles, int32_t *__restrict__ expert, float *__restrict__ gate,
                         int32_t *__restrict__ hist, int32_t *__restrict__ hist2, float *__restrict__ psum,
                         float *__restrict__ probs, float *__restrict__ ent, uint32_t *ticket, DeviceStatus *status,
                         int raw_w) {
    using S = Staged<XT>;
    constexpr int V = S::V;
    constexpr int kST = staged_threads(NP);
    if (blockDim.x != (unsigned)kST) {  // launched with another block size: report it, write nothing
        if (threadIdx.x == 0) report_status(status, SWITCH_ERR_CUDA, 62);
        return;
    }
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int64_t xpitch = S::xpitch(d);
    const int64_t wpitch = S::wpitch(NP);
    unsigned char *xs = smem_raw;
    float *wsm = reinterpret_cast<float *>(smem_raw + S::x_region(d, NP));
    int32_t *hist_s = reinterpret_cast<int32_t *>(wsm + (d / V) * wpitch);
    int32_t *hist2_s = hist_s + NP;  // second choices (TOP2)
    float *ent_tok = reinterpret_cast<float *>(hist2_s + NP);  // [64] per-token entropy (with ent)
    uint64_t *bar = reinterpret_cast<uint64_t *>((reinterpret_cast<uintptr_t>(ent_tok + kTileT) + 15) & ~uintptr_t(15));
    float *w_raw = reinterpret_cast<float *>(bar + 5) + 2;  // 16-byte aligned: bar is, and 5 * 8 + 8 = 48
    const int tid = threadIdx.x;
    const int tile = blockIdx.x;
    const int64_t t0 = (int64_t)tile * kTileT;
    const int n_tok = (int)(T - t0 < kTileT ? T - t0 : kTileT);
    const uint32_t row_bytes = (uint32_t)(d * sizeof(XT));

    pdl_launch_dependents();
    const uint32_t w_bytes = (uint32_t)(N * d * 4);
    if (tid == 0) {
        if (tile == 0) reset_call_state(ticket, status);
        for (int c = 0; c < 5; ++c) mbar_init(&bar[c], 1);
        fence_barrier_init();
        for (int c = 0; c < 4; ++c) {
            const int rows = max(0, min(16, n_tok - 16 * c));
            if (rows > 0) mbar_arrive_expect_tx(&bar[c], (uint32_t)rows * row_bytes);
        }
        if (raw_w) mbar_arrive_expect_tx(&bar[4], w_bytes);
    }
    __syncthreads();  // barriers initialised before any copy signals them
    if (tid < 32) {  // warp 0: W_r first (every thread needs it), then one bulk copy per row of x
        if (tid == 0 && raw_w) bulk_load(w_raw, w_r, w_bytes, &bar[4]);  // W_r [N][d] as stored
        __syncwarp();
        for (int r = tid; r < n_tok; r += 32)
            bulk_load(xs + r * xpitch, x + (t0 + r) * d, row_bytes, &bar[r >> 4]);
    }
    // W_r -> [d/V][V][NP] with padding, while the rows of x are on their way
    if (raw_w) {
        mbar_wait(&bar[4], 0, status, 11);
        for (int i = tid; i < NP * d; i += kST) {
            const int e = i / d, k = i - e * d;
            float v = 0.f;
            if (e < N) v = w_raw[i];  // padding experts e >= N read nothing
            wsm[(k / V) * wpitch + (k % V) * NP + e] = v;
        }
    } else {
        for (int k0 = 0; k0 < d; k0 += kST) {
            const int k = k0 + tid;
#pragma unroll
            for (int e0 = 0; e0 < NP; e0 += 8) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = (k < d && e0 + u < N) ? w_r[(int64_t)(e0 + u) * d + k] : 0.f;
                if (k < d) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) wsm[(k / V) * wpitch + (k % V) * NP + e0 + u] = v[u];
                }
            }
        }
    }
    for (int i = tid; i < NP; i += kST) {
        hist_s[i] = 0;
        hist2_s[i] = 0;
    }
    __syncthreads();

    // Thread (group g, part p of PARTS = 32 or 16 lanes): tokens 4g .. 4g+3 of
    // the tile, 16-byte x vectors j = p, p + PARTS, ... of their rows; 4 x NP
    // accumulators.  Each W_r value read from shared memory feeds four tokens.
    constexpr int TM = 4, PARTS = kST / 16;
    static_assert(kST / PARTS * TM == kTileT, "16 groups of 4 tokens");
    const int part = tid & (PARTS - 1), group = tid / PARTS;  // 16 groups x 4 tokens = 64 tokens
    float acc[TM][NP];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int e = 0; e < NP; ++e) acc[i][e] = 0.f;
    const int tok0 = group * TM;
    bool ready = tok0 < n_tok;
    if (ready) ready = mbar_wait(&bar[tok0 >> 4], 0, status, 10);  // the 4 tokens share one 16-row chunk
    if (ready) {
        for (int j = part; j < d / V; j += PARTS) {
            float xv[TM][V];
#pragma unroll
            for (int i = 0; i < TM; ++i)
                XLoad<XT>::vec_generic(reinterpret_cast<const XT *>(xs + (tok0 + i) * xpitch + (int64_t)j * 16),
                                       xv[i]);  // shared memory (rows past n_tok hold stale data, never used)
            const float *wj = wsm + j * wpitch;
#pragma unroll
            for (int u = 0; u < V; ++u) {
#pragma unroll
                for (int q = 0; q < NP / 4; ++q) {
                    const float4 w4 = *reinterpret_cast<const float4 *>(wj + u * NP + 4 * q);
#pragma unroll
                    for (int i = 0; i < TM; ++i) {
                        acc[i][4 * q + 0] = fmaf(xv[i][u], w4.x, acc[i][4 * q + 0]);
                        acc[i][4 * q + 1] = fmaf(xv[i][u], w4.y, acc[i][4 * q + 1]);
                        acc[i][4 * q + 2] = fmaf(xv[i][u], w4.z, acc[i][4 * q + 2]);
                        acc[i][4 * q + 3] = fmaf(xv[i][u], w4.w, acc[i][4 * q + 3]);
                    }
                }
            }
        }
    }
    // sum over the parts (lanes of the group): every lane of the group ends
    // with the full logits of the group's 4 tokens
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], 1);
            acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], 2);
            acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], 4);
            acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], 8);
            if (PARTS == 32) acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], 16);
        }
    // lanes with part < TM finish token tok0 + part
    float *ptile = reinterpret_cast<float *>(xs);  // [64][NP] per-token p, reusing the x tile
    __syncthreads();                               // every read of the x tile is done
    if (part < TM) {
        const int tl = tok0 + part;
        const bool valid = tl < n_tok;
        float h[NP];
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            float v = acc[0][e];
#pragma unroll
            for (int i = 1; i < TM; ++i) v = (part == i) ? acc[i][e] : v;
            h[e] = v;
        }
#pragma unroll
        for (int e = 0; e < NP; ++e)
            if (e < N) h[e] += bias ? bias[e] : 0.f;
        float m = h[0], m2 = -FLT_MAX;
        int arg = 0, arg2 = -1;
#pragma unroll
        for (int e = 1; e < NP; ++e) {
            if (e < N) {
                if (h[e] > m) {  // strict: the lowest index wins a tie
                    if (TOP2) {  // the previous leader is now the best of the others
                        m2 = m;
                        arg2 = arg;
                    }
                    m = h[e];
                    arg = e;
                } else if (TOP2 && (arg2 < 0 || h[e] > m2)) {  // strict: lowest index among the others
                    m2 = h[e];
                    arg2 = e;
                }
            }
        }
        if (TOP2 && arg2 < 0) arg2 = arg == 0 ? 1 : 0;  // N == 1 only, which top-2 routing rejects
        float s = 0.f, sv = 0.f;
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            const float z = h[e] - m;
            h[e] = e < N ? expf(z) : 0.f;
            s += h[e];
            if (e < N) sv += h[e] * z;
        }
        if (ent) ent_tok[tl] = valid ? logf(s) - sv / s : 0.f;  // -sum p ln p
#pragma unroll
        for (int e = 0; e < NP; ++e) ptile[tl * NP + e] = valid ? h[e] / s : 0.f;  // p_e
        if (probs && valid) {  // kept for the backward pass
#pragma unroll
            for (int e = 0; e < NP; ++e)
                if (e < N) probs[(t0 + tl) * N + e] = h[e] / s;
        }
        if (valid) {
            const int64_t t = t0 + tl;
            if (TOP2) {
                expert[2 * t] = arg;
                expert[2 * t + 1] = arg2;
                gate[2 * t] = 1.0f / s;
                gate[2 * t + 1] = expf(m2 - m) / s;
                atomicAdd(&hist2_s[arg2], 1);
            } else {
                expert[t] = arg;
                gate[t] = 1.0f / s;  // p at the argmax: exp(0) / s
            }
            atomicAdd(&hist_s[arg], 1);
        }
    }
    __syncthreads();
    if (ent && tid == 0) {  // the tile's entropy sum in token order
        float e = 0.f;
        for (int tl = 0; tl < kTileT; ++tl) e += ent_tok[tl];
        ent[tile] = e;
    }
    // tile sums of p: four interleaved partial sums, combined in fixed order (deterministic)
    for (int i = tid; i < N; i += kST) {
        float p4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int tl = 0; tl < kTileT; tl += 4) {
#pragma unroll
            for (int u = 0; u < 4; ++u) p4[u] += ptile[(tl + u) * NP + i];
        }
        hist[(int64_t)i * tiles + tile] = hist_s[i];
        if (TOP2) hist2[(int64_t)i * tiles + tile] = hist2_s[i];
        psum[(int64_t)i * tiles + tile] = (p4[0] + p4[1]) + (p4[2] + p4[3]);
    }
}

// ---------------------------------------------------------------------------
// Router for any N <= 256: a 64-token x EC-expert SIMT tile GEMM over
// 32-wide chunks of d, logits collected in shared memory, then one warp per
// token for the softmax / top-1.
// ---------------------------------------------------------------------------
constexpr int kKC = 32;

template <typename XT, int EC, bool TOP2>
__global__ void __launch_bounds__(kThreads) router_tiled_kernel(const XT *__restrict__ x, const float *__restrict__ w_r,
                                                                const float *__restrict__ bias, int64_t T, int d,
                                                                int N, int tiles, int32_t *__restrict__ expert,
                                                                float *__restrict__ gate, int32_t *__restrict__ hist,
                                                                int32_t *__restrict__ hist2,
                                                                float *__restrict__ psum, float *__restrict__ probs,
                                                                float *__restrict__ ent, uint32_t *ticket,
                                                                DeviceStatus *status) {
    constexpr int TE = EC / 16;  // experts per thread
    constexpr int TT = 4;        // tokens per thread
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int NL = N + 1;
    float *xs = reinterpret_cast<float *>(smem_raw);  // [kKC][kTileT]
    float *ws = xs + kKC * kTileT;                     // [kKC][EC]
    float *logits = ws + kKC * EC;                     // [kTileT][NL]
    float *psum_w = logits + kTileT * NL;              // [kWarps][N]
    int32_t *hist_w = reinterpret_cast<int32_t *>(psum_w + kWarps * N);
    int32_t *hist2_w = hist_w + kWarps * N;            // [kWarps][N] second choices (TOP2)
    float *ent_w = reinterpret_cast<float *>(hist2_w + kWarps * N);  // [kWarps] entropy sums
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tx = tid % 16, ty = tid / 16;
    const int tile = blockIdx.x;
    const int64_t t0 = (int64_t)tile * kTileT;

    if (tile == 0 && tid == 0) reset_call_state(ticket, status);
    if (tid < kWarps) ent_w[tid] = 0.f;
    for (int i = tid; i < kWarps * N; i += kThreads) {
        psum_w[i] = 0.f;
        hist_w[i] = 0;
        if (TOP2) hist2_w[i] = 0;
    }

    for (int e0 = 0; e0 < N; e0 += EC) {
        float acc[TT][TE];
#pragma unroll
        for (int i = 0; i < TT; ++i)
#pragma unroll
            for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;
        for (int k0 = 0; k0 < d; k0 += kKC) {
            __syncthreads();
            for (int i = tid; i < kTileT * kKC; i += kThreads) {
                const int r = i / kKC, kk = i % kKC;
                const int64_t t = t0 + r;
                const int k = k0 + kk;
                xs[kk * kTileT + r] = (t < T && k < d) ? XLoad<XT>::one(x + t * d + k) : 0.f;
            }
            for (int i = tid; i < EC * kKC; i += kThreads) {
                const int e = i / kKC, kk = i % kKC;
                const int k = k0 + kk;
                ws[kk * EC + e] = (e0 + e < N && k < d) ? w_r[(int64_t)(e0 + e) * d + k] : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int kk = 0; kk < kKC; ++kk) {
                float a[TT], b[TE];
#pragma unroll
                for (int i = 0; i < TT; ++i) a[i] = xs[kk * kTileT + ty + 16 * i];
#pragma unroll
                for (int j = 0; j < TE; ++j) b[j] = ws[kk * EC + tx + 16 * j];
#pragma unroll
                for (int i = 0; i < TT; ++i)
#pragma unroll
                    for (int j = 0; j < TE; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
        }
#pragma unroll
        for (int i = 0; i < TT; ++i)
#pragma unroll
            for (int j = 0; j < TE; ++j) {
                const int e = e0 + tx + 16 * j;
                if (e < N) logits[(ty + 16 * i) * NL + e] = acc[i][j];
            }
    }
    __syncthreads();

    constexpr int J = 8;  // up to 256 experts, 8 per lane
    for (int r = warp; r < kTileT; r += kWarps) {
        const int64_t t = t0 + r;
        if (t >= T) break;
        float v[J];
        int idx[J];
        bool own[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int e = lane + 32 * j;
            idx[j] = e < N ? e : -1;
            own[j] = true;
            v[j] = e < N ? logits[r * NL + e] + (bias ? bias[e] : 0.f) : 0.f;
        }
        token_epilogue<J, TOP2>(v, idx, own, t, psum_w + warp * N, hist_w + warp * N, hist2_w + warp * N, expert,
                                gate, probs, N, ent ? ent_w + warp : nullptr);
    }
    __syncthreads();
    publish_tile(psum_w, hist_w, hist2_w, N, tiles, tile, hist, TOP2 ? hist2 : nullptr, psum, ent_w, ent);
}

// ---------------------------------------------------------------------------
// Scan: one block per expert.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;

// Exclusive prefix over tiles of one expert's row of tile counts, starting at
// `base`: thread tid owns tiles [begin, end).  Returns the row total.
__device__ __forceinline__ int32_t scan_row(const int32_t *__restrict__ h, int tiles, int32_t base,
                                            int32_t *__restrict__ off, int32_t *warp_cnt) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = (tiles + kScanThreads - 1) / kScanThreads;
    const int begin = min(tiles, tid * chunk), end = min(tiles, begin + chunk);
    int32_t mine = 0;
    for (int i = begin; i < end; ++i) mine += h[i];
    int32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    __syncthreads();  // warp_cnt may still be read from a previous row
    if (lane == 31) warp_cnt[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int32_t c = warp_cnt[lane];
        int32_t ci = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, ci, o);
            if (lane >= o) ci += u;
        }
        warp_cnt[lane] = ci - c;  // exclusive prefix of warp totals
        if (lane == 31) warp_cnt[32] = ci;
    }
    __syncthreads();
    int32_t run = base + warp_cnt[warp] + incl - mine;
    for (int i = begin; i < end; ++i) {
        off[i] = run;
        run += h[i];
    }
    return warp_cnt[32];
}

// Scan: one block per expert.  Top-1: tile_off = exclusive prefix of the tile
// counts.  Top-2 (hist2 set): first choices take the slots first, so
// tile_off = prefix of the first-choice counts and tile_off2 = (all first
// choices of the expert) + prefix of the second-choice counts; counts = both
// totals, counts_first = the first-choice total (the aux loss counts argmax
// choices only).
template <bool TOP2>
__global__ void __launch_bounds__(kScanThreads) scan_kernel(const int32_t *__restrict__ hist,
                                                            const int32_t *__restrict__ hist2,
                                                            const float *__restrict__ psum, int tiles, int N,
                                                            int64_t T, int32_t *__restrict__ tile_off,
                                                            int32_t *__restrict__ tile_off2,
                                                            int32_t *__restrict__ counts,
                                                            int32_t *__restrict__ counts_first, double *prob_total,
                                                            float *aux, uint32_t *ticket) {
    __shared__ int32_t warp_cnt[33];
    __shared__ double warp_p[kScanThreads / 32];
    __shared__ bool is_last;
    pdl_wait();
    pdl_launch_dependents();
    const int e = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = (tiles + kScanThreads - 1) / kScanThreads;
    const int begin = min(tiles, tid * chunk), end = min(tiles, begin + chunk);
    const float *ps = psum + (int64_t)e * tiles;

    double pmine = 0.0;
    for (int i = begin; i < end; ++i) pmine += (double)ps[i];
    double pw = pmine;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) pw += __shfl_xor_sync(0xffffffffu, pw, off);
    if (lane == 0) warp_p[warp] = pw;
    const int32_t total1 = scan_row(hist + (int64_t)e * tiles, tiles, 0, tile_off + (int64_t)e * tiles, warp_cnt);
    int32_t total = total1;
    if (TOP2)
        total += scan_row(hist2 + (int64_t)e * tiles, tiles, total1, tile_off2 + (int64_t)e * tiles, warp_cnt);
    if (tid == 0) {
        counts[e] = total;
        if (TOP2) counts_first[e] = total1;
        double p = 0.0;
        for (int w = 0; w < kScanThreads / 32; ++w) p += warp_p[w];
        prob_total[e] = p;
    }

    // The last expert block to finish forms the aux loss: one f_i * P_i per
    // thread (all loads in parallel), then a fixed-order tree over threads.
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = atomicAdd(ticket, 1u) == (uint32_t)(N - 1);
    __syncthreads();
    if (is_last) {
        __threadfence();
        double term = 0.0;
        if (T > 0 && tid < N) {
            const double f = (double)__ldcg((TOP2 ? counts_first : counts) + tid) / (double)T;
            const double P = __ldcg(prob_total + tid) / (double)T;
            term = f * P;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) term += __shfl_xor_sync(0xffffffffu, term, off);
        __syncthreads();  // every warp has read warp_p above
        if (lane == 0) warp_p[warp] = term;
        __syncthreads();
        if (tid == 0) {
            double total_aux = 0.0;
            for (int w = 0; w < kScanThreads / 32; ++w) total_aux += warp_p[w];
            *aux = (float)((double)N * total_aux);
            *ticket = 0u;
        }
    }
}

// ---------------------------------------------------------------------------
// Assignment: blocks [0, tiles) take one 64-token tile each; warps 0 and 1
// rank the tile's tokens within their experts, and with SCATTER all eight
// warps then move rows: a kept token's row of x goes to xbuf[expert, slot]
// (the dispatch, in scatter form), a dropped token's output row is zeroed.
// Every block also clears a share of the empty slots of slot_token.
// ---------------------------------------------------------------------------
constexpr int kAssignThreads = 256;
constexpr int64_t kFusedScanLoads = int64_t(1) << 22;  // histogram loads of all assignment blocks together

// Per-expert sums over the tile histograms for one block: the tiles before
// `tile` (the block's first slot per expert) and all tiles (the counts).
// Integer sums: exact in any order.  Used when the whole histogram is small,
// in place of the separate scan kernel.
__device__ __forceinline__ void block_tile_sums(const int32_t *__restrict__ hist, int tiles, int N, int tile,
                                                int32_t *s_off, int32_t *s_cnt) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = warp; e < N; e += kAssignThreads / 32) {
        int32_t pre = 0, tot = 0;
        for (int i = lane; i < tiles; i += 32) {
            const int32_t h = hist[(int64_t)e * tiles + i];
            tot += h;
            pre += i < tile ? h : 0;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            pre += __shfl_xor_sync(0xffffffffu, pre, off);
            tot += __shfl_xor_sync(0xffffffffu, tot, off);
        }
        if (lane == 0) {
            s_off[e] = pre;
            s_cnt[e] = tot;
        }
    }
}

// SCAN: the block forms its own first slots and the counts from the tile
// histograms (small histograms only), and block 0 writes counts, the Σp
// totals and aux; otherwise they come from scan_kernel.
template <bool SCATTER, bool SCAN>
__global__ void __launch_bounds__(kAssignThreads) assign_kernel(
    const int32_t *__restrict__ expert, const int32_t *__restrict__ tile_off, int32_t *__restrict__ counts,
    int64_t T, int N, int C, int tiles, int32_t *__restrict__ slot, int32_t *__restrict__ slot_token,
    const uint4 *__restrict__ x, uint4 *__restrict__ xbuf, int x_words, float4 *__restrict__ y_zero, int y_words,
    int32_t *__restrict__ done_zero, int64_t n_done, const int32_t *__restrict__ hist, const float *__restrict__ psum,
    double *__restrict__ prob_total, float *__restrict__ aux, DeviceStatus *status) {
    static_assert(kTileT == 64, "assignment assumes two ranking warps per tile");
    __shared__ int32_t first_warp_count[256];
    __shared__ int32_t tile_slot[kTileT];
    __shared__ int32_t tile_expert[kTileT];
    __shared__ int32_t s_off[SCAN ? 256 : 1], s_cnt[SCAN ? 256 : 1];
    __shared__ double s_p[SCAN ? 256 : 1];
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x;
    if (SCAN) {
        block_tile_sums(hist, tiles, N, tile, s_off, s_cnt);
        if (blockIdx.x == 0) {
            // Σp per expert (fp64, lane-strided partial sums, then a fixed xor tree)
            for (int e = warp; e < N; e += kAssignThreads / 32) {
                double p = 0.0;
                for (int i = lane; i < tiles; i += 32) p += (double)psum[(int64_t)e * tiles + i];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
                if (lane == 0) s_p[e] = p;
            }
        }
        __syncthreads();
        if (blockIdx.x == 0) {
            for (int e = tid; e < N; e += kAssignThreads) {
                counts[e] = s_cnt[e];
                prob_total[e] = s_p[e];
            }
            if (warp == 0) {  // aux = N * sum_i f_i P_i, one term per lane, then a fixed xor tree
                double term = 0.0;
                if (T > 0)
                    for (int e = lane; e < N; e += 32) term += ((double)s_cnt[e] / (double)T) * (s_p[e] / (double)T);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) term += __shfl_xor_sync(0xffffffffu, term, off);
                if (lane == 0) *aux = (float)((double)N * term);
            }
        }
    }
    if (tile < tiles) {
        for (int i = tid; i < N; i += kAssignThreads) first_warp_count[i] = 0;
        __syncthreads();
        int e = -1, rank = 0;
        bool valid = false, rejected = false;
        int64_t t = 0;
        unsigned same = 0;
        if (warp < 2) {
            t = (int64_t)tile * kTileT + tid;
            valid = t < T;
            e = valid ? expert[t] : -1 - lane;  // distinct keys for absent tokens
            if (valid && (unsigned)e >= (unsigned)N) {  // an id no router writes: report it, index
                report_status(status, SWITCH_ERR_SHAPE, 60);  // nothing, and drop the token
                valid = false;
                rejected = true;
                e = -1 - lane;
            }
            same = __match_any_sync(0xffffffffu, e);
            rank = __popc(same & (unsigned)lanemask_lt());
            if (warp == 0 && valid && rank == 0) first_warp_count[e] = __popc(same);
        }
        __syncthreads();
        if (warp < 2) {
            int s_out = rejected ? -1 : -2;  // -2: no token here; -1: dropped
            if (rejected) slot[t] = -1;
            if (valid) {
                if (warp == 1) rank += first_warp_count[e];
                const int s = (SCAN ? s_off[e] : tile_off[(int64_t)e * tiles + tile]) + rank;
                if (s < C) {
                    slot[t] = s;
                    slot_token[(int64_t)e * C + s] = (int32_t)t;
                    s_out = s;
                } else {
                    slot[t] = -1;
                    s_out = -1;
                }
            }
            tile_slot[tid] = s_out;
            tile_expert[tid] = e;
        }
        if (SCATTER) {
            __syncthreads();
            // Each warp moves rows warp, warp + 8, ...: all loads of a group of
            // four rows are in flight before the first store.
            constexpr int kRows = 4, kWords = 4;  // per lane: 4 rows x 4 x 16 bytes
            for (int r0 = warp; r0 < kTileT; r0 += (kAssignThreads / 32) * kRows) {
                for (int w0 = 0; w0 < x_words; w0 += 32 * kWords) {
                    uint4 v[kRows][kWords];
#pragma unroll
                    for (int i = 0; i < kRows; ++i) {
                        const int r = r0 + i * (kAssignThreads / 32);
                        const int s = r < kTileT ? tile_slot[r] : -2;
                        const uint4 *src = x + ((int64_t)tile * kTileT + r) * x_words;
#pragma unroll
                        for (int u = 0; u < kWords; ++u) {
                            const int w = w0 + lane + 32 * u;
                            if (s >= 0 && w < x_words) v[i][u] = __ldcs(src + w);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < kRows; ++i) {
                        const int r = r0 + i * (kAssignThreads / 32);
                        const int s = r < kTileT ? tile_slot[r] : -2;
                        if (s < 0) continue;
                        uint4 *dst = xbuf + ((int64_t)tile_expert[r] * C + s) * x_words;
#pragma unroll
                        for (int u = 0; u < kWords; ++u) {
                            const int w = w0 + lane + 32 * u;
                            if (w < x_words) dst[w] = v[i][u];
                        }
                    }
                }
                if (y_zero) {
                    for (int i = 0; i < kRows; ++i) {
                        const int r = r0 + i * (kAssignThreads / 32);
                        if (r >= kTileT || tile_slot[r] != -1) continue;
                        float4 *dst = y_zero + ((int64_t)tile * kTileT + r) * y_words;
                        for (int w = lane; w < y_words; w += 32) __stcs(dst + w, make_float4(0.f, 0.f, 0.f, 0.f));
                    }
                }
            }
        }
    }
    for (int64_t i = (int64_t)blockIdx.x * kAssignThreads + tid; i < n_done; i += (int64_t)gridDim.x * kAssignThreads)
        done_zero[i] = 0;  // completion counters of the fused expert FFN that follows
    const int64_t total = (int64_t)N * C;
    for (int64_t i = (int64_t)blockIdx.x * kAssignThreads + tid; i < total; i += (int64_t)gridDim.x * kAssignThreads) {
        const int e = (int)(i / C);
        const int s = (int)(i % C);
        if (s >= min(SCAN ? s_cnt[e] : counts[e], C)) slot_token[i] = -1;
    }
}

// Top-2 assignment: block `tile` ranks the tile's first choices (warps 0-1)
// and second choices (warps 2-3) within their experts, in token order.  A
// first choice takes slot tile_off[e][tile] + rank, a second choice
// tile_off2[e][tile] + rank (tile_off2 starts after all first choices of the
// expert); kept iff the slot is below C.  With SCATTER all eight warps then
// copy x[t] to xbuf[e, slot] for every kept (token, choice).  Every block
// also clears a share of the empty slots of slot_token.
template <bool SCATTER>
__global__ void __launch_bounds__(kAssignThreads) assign_top2_kernel(
    const int32_t *__restrict__ expert2, const int32_t *__restrict__ tile_off, const int32_t *__restrict__ tile_off2,
    const int32_t *__restrict__ counts, int64_t T, int N, int C, int tiles, int32_t *__restrict__ slot2,
    int32_t *__restrict__ slot_token, const uint4 *__restrict__ x, uint4 *__restrict__ xbuf, int x_words,
    DeviceStatus *status) {
    static_assert(kTileT == 64, "top-2 assignment assumes 64-token tiles");
    __shared__ int32_t first_warp_count[2][256];
    __shared__ int32_t tile_slot[2 * kTileT];    // [choice][token of the tile]
    __shared__ int32_t tile_expert[2 * kTileT];
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile = blockIdx.x;
    if (tile < tiles) {
        for (int i = tid; i < 2 * 256; i += kAssignThreads) (&first_warp_count[0][0])[i] = 0;
        __syncthreads();
        const int c = warp >> 1;         // warps 0-1: first choices, 2-3: second choices
        const int half = warp & 1;       // tokens 0-31 or 32-63 of the tile
        int e = -1, rank = 0;
        bool valid = false, rejected = false;
        int64_t t = 0;
        unsigned same = 0;
        if (warp < 4) {
            t = (int64_t)tile * kTileT + half * 32 + lane;
            valid = t < T;
            e = valid ? expert2[2 * t + c] : -1 - lane;  // distinct keys for absent tokens
            if (valid && (unsigned)e >= (unsigned)N) {  // an id no router writes: report it, index
                report_status(status, SWITCH_ERR_SHAPE, 61);  // nothing, and drop the choice
                valid = false;
                rejected = true;
                e = -1 - lane;
            }
            same = __match_any_sync(0xffffffffu, e);
            rank = __popc(same & (unsigned)lanemask_lt());
            if (half == 0 && valid && rank == 0) first_warp_count[c][e] = __popc(same);
        }
        __syncthreads();
        if (warp < 4) {
            int s_out = rejected ? -1 : -2;  // -2: no token here; -1: dropped
            if (rejected) slot2[2 * t + c] = -1;
            if (valid) {
                if (half == 1) rank += first_warp_count[c][e];
                const int s = (c == 0 ? tile_off : tile_off2)[(int64_t)e * tiles + tile] + rank;
                if (s < C) {
                    slot2[2 * t + c] = s;
                    slot_token[(int64_t)e * C + s] = (int32_t)t;
                    s_out = s;
                } else {
                    slot2[2 * t + c] = -1;
                    s_out = -1;
                }
            }
            tile_slot[c * kTileT + half * 32 + lane] = s_out;
            tile_expert[c * kTileT + half * 32 + lane] = e;
        }
        if (SCATTER) {
            __syncthreads();
            // 128 (token, choice) entries; warp w copies entries w, w + 8, ...
            for (int j = warp; j < 2 * kTileT; j += kAssignThreads / 32) {
                const int s = tile_slot[j];
                if (s < 0) continue;
                const int r = j & (kTileT - 1);
                const uint4 *src = x + ((int64_t)tile * kTileT + r) * x_words;
                uint4 *dst = xbuf + ((int64_t)tile_expert[j] * C + s) * x_words;
                for (int w = lane; w < x_words; w += 32) dst[w] = __ldg(src + w);
            }
        }
    }
    const int64_t total = (int64_t)N * C;
    for (int64_t i = (int64_t)blockIdx.x * kAssignThreads + tid; i < total; i += (int64_t)gridDim.x * kAssignThreads) {
        const int e = (int)(i / C);
        const int s = (int)(i % C);
        if (s >= min(counts[e], C)) slot_token[i] = -1;
    }
}

template <typename XT, int NP, bool TOP2>
cudaError_t launch_router_warp(const switch_dims_t &dims, const XT *x, const float *w_r, const float *bias,
                               int32_t *expert, float *gate, const Workspace &ws, cudaStream_t stream) {
    const int N = dims.num_experts, d = dims.d_model;
    const size_t smem = (size_t)d * NP * sizeof(float) + (size_t)kWarps * N * (sizeof(float) + 2 * sizeof(int32_t)) +
                        kWarps * sizeof(float);
    auto kern = router_warp_kernel<XT, NP, TOP2>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    launch_begin(K_ROUTER_WARP, stream);
    kern<<<(unsigned)ws.tiles, kThreads, smem, stream>>>(x, w_r, bias, dims.T, d, N, (int)ws.tiles, expert, gate,
                                                         ws.hist, ws.hist2, ws.psum, ws.probs, ws.ent, ws.ticket,
                                                         static_cast<DeviceStatus *>(ws.status));
    err = cudaGetLastError();
    launch_end(stream);
    return err;
}

// Shared memory the staged router may use (x tile + W_r + partials).
constexpr size_t kStagedSmemLimit = 200 * 1024;

template <typename XT, int NP, bool TOP2>
cudaError_t launch_router_staged(const switch_dims_t &dims, const XT *x, const float *w_r, const float *bias,
                                 int32_t *expert, float *gate, const Workspace &ws, cudaStream_t stream) {
    const int N = dims.num_experts, d = dims.d_model;
    const bool raw = ((int64_t)N * d * 4) % 16 == 0 && Staged<XT>::smem(d, NP, N, true) <= kStagedSmemLimit;
    const size_t smem = Staged<XT>::smem(d, NP, N, raw);
    auto kern = router_staged_kernel<XT, NP, TOP2>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    launch_begin(K_ROUTER_STAGED, stream);
    kern<<<(unsigned)ws.tiles, staged_threads(NP), smem, stream>>>(x, w_r, bias, dims.T, d, N, (int)ws.tiles, expert, gate,
                                                         ws.hist, ws.hist2, ws.psum, ws.probs, ws.ent, ws.ticket,
                                                         static_cast<DeviceStatus *>(ws.status), raw ? 1 : 0);
    err = cudaGetLastError();
    launch_end(stream);
    return err;
}

template <typename XT, int EC, bool TOP2>
cudaError_t launch_router_tiled(const switch_dims_t &dims, const XT *x, const float *w_r, const float *bias,
                                int32_t *expert, float *gate, const Workspace &ws, cudaStream_t stream) {
    const int N = dims.num_experts, d = dims.d_model;
    const size_t smem = (size_t)(kKC * kTileT + kKC * EC + kTileT * (N + 1)) * sizeof(float) +
                        (size_t)kWarps * N * (sizeof(float) + 2 * sizeof(int32_t)) + kWarps * sizeof(float);
    auto kern = router_tiled_kernel<XT, EC, TOP2>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    launch_begin(K_ROUTER_TILED, stream);
    kern<<<(unsigned)ws.tiles, kThreads, smem, stream>>>(x, w_r, bias, dims.T, d, N, (int)ws.tiles, expert, gate,
                                                         ws.hist, ws.hist2, ws.psum, ws.probs, ws.ent, ws.ticket,
                                                         static_cast<DeviceStatus *>(ws.status));
    err = cudaGetLastError();
    launch_end(stream);
    return err;
}

// Largest d for which the warp router keeps W_r in shared memory.
constexpr size_t kWarpRouterSmemLimit = 160 * 1024;
template <typename XT, bool TOP2>
cudaError_t launch_router(const switch_dims_t &dims, const XT *x, const float *w_r, const float *bias,
                          int32_t *expert, float *gate, const Workspace &ws, cudaStream_t stream) {
    const int N = dims.num_experts;
    const int NP = N <= 8 ? 8 : N <= 16 ? 16 : 32;
    const bool staged = N <= 32 && ((int64_t)dims.d_model * (int64_t)sizeof(XT)) % 16 == 0 &&
                        Staged<XT>::smem(dims.d_model, NP, N, false) <= kStagedSmemLimit;
    if (staged) {
        if (NP == 8) return launch_router_staged<XT, 8, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
        if (NP == 16) return launch_router_staged<XT, 16, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
        return launch_router_staged<XT, 32, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
    }
    const bool fits = N <= 32 && (size_t)dims.d_model * NP * sizeof(float) + 2048 * 8 <= kWarpRouterSmemLimit;
    if (fits) {
        if (NP == 8) return launch_router_warp<XT, 8, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
        if (NP == 16) return launch_router_warp<XT, 16, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
        return launch_router_warp<XT, 32, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
    }
    if (N <= 32) return launch_router_tiled<XT, 32, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
    if (N <= 64) return launch_router_tiled<XT, 64, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
    return launch_router_tiled<XT, 128, TOP2>(dims, x, w_r, bias, expert, gate, ws, stream);
}

template <bool TOP2>
cudaError_t launch_any_router(const switch_dims_t &dims, const void *x, const float *w_r, const float *bias,
                              int32_t *expert, float *gate, const Workspace &ws, cudaStream_t stream) {
    return dims.dtype == SWITCH_BF16
               ? launch_router<__nv_bfloat16, TOP2>(dims, static_cast<const __nv_bfloat16 *>(x), w_r, bias, expert,
                                                    gate, ws, stream)
               : launch_router<float, TOP2>(dims, static_cast<const float *>(x), w_r, bias, expert, gate, ws, stream);
}

// Router statistics from a routing call's per-tile entropy sums and counts:
// stats = {mean entropy, dropped fraction, capacity utilisation, busiest load
// over the uniform load}; fp64 sums in a fixed order.  One block.
__global__ void __launch_bounds__(256) router_stats_kernel(const float *__restrict__ ent, int tiles,
                                                          const int32_t *__restrict__ counts, int N, int C,
                                                          int64_t T, float *__restrict__ stats) {
    __shared__ double s_ent[kWarps];
    __shared__ long long s_drop[kWarps], s_kept[kWarps], s_max[kWarps];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    double e = 0.0;
    if (ent)
        for (int i = tid; i < tiles; i += 256) e += (double)ent[i];
    long long drop = 0, kept = 0, mx = 0;
    for (int i = tid; i < N; i += 256) {
        const long long c = counts[i];
        drop += c > C ? c - C : 0;
        kept += c < C ? c : C;
        mx = c > mx ? c : mx;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        e += __shfl_xor_sync(0xffffffffu, e, off);
        drop += __shfl_xor_sync(0xffffffffu, drop, off);
        kept += __shfl_xor_sync(0xffffffffu, kept, off);
        const long long o = __shfl_xor_sync(0xffffffffu, mx, off);
        mx = o > mx ? o : mx;
    }
    if (lane == 0) {
        s_ent[warp] = e;
        s_drop[warp] = drop;
        s_kept[warp] = kept;
        s_max[warp] = mx;
    }
    __syncthreads();
    if (tid == 0) {
        double et = 0.0;
        long long dt = 0, kt = 0, mt = 0;
        for (int w = 0; w < kWarps; ++w) {
            et += s_ent[w];
            dt += s_drop[w];
            kt += s_kept[w];
            mt = s_max[w] > mt ? s_max[w] : mt;
        }
        const bool any = T > 0;
        stats[0] = !ent ? __int_as_float(0x7fc00000) : any ? (float)(et / (double)T) : 0.f;
        stats[1] = any ? (float)((double)dt / (double)T) : 0.f;
        stats[2] = any ? (float)((double)kt / ((double)N * (double)C)) : 0.f;
        stats[3] = any ? (float)((double)mt * (double)N / (double)T) : 0.f;
    }
}

}  // namespace

cudaError_t launch_router_stats(const switch_dims_t &dims, const int32_t *counts, const Workspace &ws, float *stats,
                                cudaStream_t stream) {
    launch_begin(K_ROUTER_STATS, stream);
    router_stats_kernel<<<1, 256, 0, stream>>>(ws.ent, (int)ws.tiles, counts, dims.num_experts, dims.capacity,
                                               dims.T, stats);
    const cudaError_t err = cudaGetLastError();
    launch_end(stream);
    return err;
}

cudaError_t launch_route(const switch_dims_t &dims, const void *x, const float *w_r, const float *bias,
                         int32_t *expert, float *gate, int32_t *slot, int32_t *counts, int32_t *slot_token,
                         float *aux, const Workspace &ws, cudaStream_t stream, void *xbuf_scatter, float *y_zero,
                         int32_t *done_zero, int64_t n_done, bool top2) {
    cudaError_t err = cudaSuccess;
    const int N = dims.num_experts, C = dims.capacity;
    if (ws.tiles > 0 && router_tc_supported(dims)) {
        err = launch_router_tc(dims, x, w_r, bias, expert, gate, ws, stream, top2);
        if (err != cudaSuccess) return err;
    } else if (ws.tiles > 0) {
        err = top2 ? launch_any_router<true>(dims, x, w_r, bias, expert, gate, ws, stream)
                   : launch_any_router<false>(dims, x, w_r, bias, expert, gate, ws, stream);
        if (err != cudaSuccess) return err;
    } else {
        // No router launch to reset the scan ticket and the status word.
        err = cudaMemsetAsync(ws.ticket, 0, sizeof(uint32_t), stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(ws.status, 0, sizeof(DeviceStatus), stream);
        if (err != cudaSuccess) return err;
    }
    const int64_t fill_blocks = ((int64_t)N * C + kAssignThreads * 4 - 1) / (kAssignThreads * 4);
    const int64_t grid = ws.tiles > fill_blocks ? ws.tiles : fill_blocks;
    const int x_words = (int)((int64_t)dims.d_model * (dims.dtype == SWITCH_BF16 ? 2 : 4) / 16);
    const uint4 *xs = static_cast<const uint4 *>(x);
    uint4 *xb = static_cast<uint4 *>(xbuf_scatter);
    if (top2) {
        // top-2: the scan kernel always runs (two prefixes per expert)
        launch_begin(K_SCAN, stream);
        err = launch_kernel(scan_kernel<true>, dim3(N), dim3(kScanThreads), 0, stream, ws.tiles > 0, ws.hist,
                            ws.hist2, ws.psum, (int)ws.tiles, N, dims.T, ws.tile_off, ws.tile_off2, counts,
                            ws.counts_first, ws.prob_total, aux, ws.ticket);
        launch_end(stream);
        if (err != cudaSuccess) return err;
        launch_begin(xbuf_scatter ? K_ASSIGN_SCATTER : K_ASSIGN, stream);
        if (xbuf_scatter)
            err = launch_kernel(assign_top2_kernel<true>, dim3((unsigned)grid), dim3(kAssignThreads), 0, stream, true,
                                expert, ws.tile_off, ws.tile_off2, counts, dims.T, N, C, (int)ws.tiles, slot,
                                slot_token, xs, xb, x_words, static_cast<DeviceStatus *>(ws.status));
        else
            err = launch_kernel(assign_top2_kernel<false>, dim3((unsigned)grid), dim3(kAssignThreads), 0, stream,
                                true, expert, ws.tile_off, ws.tile_off2, counts, dims.T, N, C, (int)ws.tiles, slot,
                                slot_token, (const uint4 *)nullptr, (uint4 *)nullptr, 0,
                                static_cast<DeviceStatus *>(ws.status));
        launch_end(stream);
        return err;
    }
    // Small histograms: every assignment block sums the tile counts it needs
    // itself (at most kFusedScanLoads loads over the whole grid), saving the
    // scan kernel's launch and its round trip through memory.
    const bool fused_scan = ws.tiles > 0 && (int64_t)N * ws.tiles * grid <= kFusedScanLoads &&
                            !(dims.flags & SWITCH_FLAG_SEPARATE_SCAN);
    if (!fused_scan) {
        launch_begin(K_SCAN, stream);
        err = launch_kernel(scan_kernel<false>, dim3(N), dim3(kScanThreads), 0, stream, ws.tiles > 0, ws.hist,
                            (const int32_t *)nullptr, ws.psum, (int)ws.tiles, N, dims.T, ws.tile_off,
                            (int32_t *)nullptr, counts, (int32_t *)nullptr, ws.prob_total, aux, ws.ticket);
        launch_end(stream);
        if (err != cudaSuccess) return err;
    }
    float4 *yz = reinterpret_cast<float4 *>(y_zero);
    const int y_words = dims.d_model / 4;
    const int32_t kid = xbuf_scatter ? K_ASSIGN_SCATTER : K_ASSIGN;
    launch_begin(kid, stream);
    if (xbuf_scatter && fused_scan)
        err = launch_kernel(assign_kernel<true, true>, dim3((unsigned)grid), dim3(kAssignThreads), 0, stream, true,
                            expert, ws.tile_off, counts, dims.T, N, C, (int)ws.tiles, slot, slot_token, xs, xb,
                            x_words, yz, y_words, done_zero, n_done, ws.hist, ws.psum, ws.prob_total, aux,
                            static_cast<DeviceStatus *>(ws.status));
    else if (xbuf_scatter)
        err = launch_kernel(assign_kernel<true, false>, dim3((unsigned)grid), dim3(kAssignThreads), 0, stream, true,
                            expert, ws.tile_off, counts, dims.T, N, C, (int)ws.tiles, slot, slot_token, xs, xb,
                            x_words, yz, y_words, done_zero, n_done, ws.hist, ws.psum, ws.prob_total, aux,
                            static_cast<DeviceStatus *>(ws.status));
    else if (fused_scan)
        err = launch_kernel(assign_kernel<false, true>, dim3((unsigned)grid), dim3(kAssignThreads), 0, stream, true,
                            expert, ws.tile_off, counts, dims.T, N, C, (int)ws.tiles, slot, slot_token,
                            (const uint4 *)nullptr, (uint4 *)nullptr, 0, (float4 *)nullptr, 0, done_zero, n_done,
                            ws.hist, ws.psum, ws.prob_total, aux,
                            static_cast<DeviceStatus *>(ws.status));
    else
        err = launch_kernel(assign_kernel<false, false>, dim3((unsigned)grid), dim3(kAssignThreads), 0, stream, true,
                            expert, ws.tile_off, counts, dims.T, N, C, (int)ws.tiles, slot, slot_token,
                            (const uint4 *)nullptr, (uint4 *)nullptr, 0, (float4 *)nullptr, 0, done_zero, n_done,
                            ws.hist, ws.psum, ws.prob_total, aux,
                            static_cast<DeviceStatus *>(ws.status));
    launch_end(stream);
    return err;
}

}  // namespace switchmoe
