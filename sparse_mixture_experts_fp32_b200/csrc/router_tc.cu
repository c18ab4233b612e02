// Router on tcgen05 tensor cores, for bfloat16 activations and N <= 128
// experts (sm_100a).
//
// The router computes in float32 (kasblo "Switch Transformerとは？" section
// "Routerだけfloat32で計算するSelective Precision"; logits h = W_r . x,
// llm-papers-study "精读 06 | Switch Transformers" §3.1).  x is bfloat16, so
// it is exact as an MMA operand.  W_r (float32) is split into three bfloat16
// terms, hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid), whose sum
// is w exactly for every w of normal magnitude.  Three kind::f16 MMAs per
// K-step add x . hi, x . mid and x . lo into one float32 accumulator in
// tensor memory: every product is exact, only the order of the float32
// additions differs from a CUDA-core dot product.
//
// Tile = 256 tokens (MMA M, a pair of CTAs on two SMs with
// tcgen05.mma.cta_group::2, 128 tokens each) x BN experts (the experts padded
// to 64 or 128; padding rows of W_r are zero-filled by TMA and ignored).  Per
// 16-wide K step two MMAs: one with N = 2 BN against hi and mid stacked (the
// leader's shared memory holds the hi rows, the peer's the mid rows), which
// writes x . hi to accumulator columns [0, BN) and x . mid to [BN, 2 BN), and
// one with N = BN against lo (each CTA holds half of its rows), added into
// columns [0, BN).  The epilogue adds the two column blocks.  The tensor
// work is the same as three N = BN MMAs (an N = 256 pair MMA takes 128 cycles,
// an N = 128 one 64 on B200); the MMA thread issues two instructions per K
// step instead of three.  Persistent over token tiles, one CTA per SM:
//   warp 0     TMA: 128 x 64 slice of x, this CTA's term of the stacked
//              operand and half of lo, counted on the leader's (rank 0)
//              barrier
//   warp 1     TMEM allocation; one lane of the leader issues the MMAs
//   warps 2 .. 2 + 4G - 1 (G = BN / 32)  epilogue of the CTA's 128 tokens,
//              one warp per TMEM lane quarter (warp w may only reach TMEM lanes
//              32 (w % 4) .. +31) and 32-expert column group: max and argmax
//              (lowest index on ties) and the sum of exp per group, combined
//              across the G groups through shared memory; gate = 1/sum, p_i;
//              per-64-token-tile expert counts and sums of p_i
//              (deterministic: a fixed shuffle tree, then a fixed warp order).
//              Several warps per SM sub-partition hide the latency of this
//              per-token chain.
// Barrier addresses of the other CTA come from mapa; no load is multicast.
// (An L2 prefetch of the next token tile of x, issued at the start of each
// tile, made the kernel slower on B200, as it did for the expert GEMMs.)
#include <cuda.h>

#include <algorithm>
#include <float.h>

#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr int RM = 128;  // tokens per CTA (a pair tile is 2 * RM)
constexpr int RK = 64;   // K per ring stage (one 128-byte swizzle row of bf16)
constexpr int kTerms = 3;
// Epilogue: G = BN / 32 column groups of 32 experts; four warps (one per TMEM
// lane quarter) per group.
template <int BN>
struct RouterThreads {
    static constexpr int kGroups = BN / 32;
    static constexpr int kEpi = 128 * kGroups;  // warps 2 .. 2 + 4G - 1
    static constexpr int kAll = 64 + kEpi;
};

// W_r float32 [N][d] -> three bfloat16 terms [3][N][d].
__global__ void split_router_weight(const float *__restrict__ w, __nv_bfloat16 *__restrict__ out, int64_t n) {
    pdl_launch_dependents();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = w[i];
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);
        out[i] = hi;
        out[n + i] = mid;
        out[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

template <int BN, int STAGES, bool TOP2 = false>
struct RouterLayout {
    static constexpr size_t a_bytes = (size_t)RM * RK * 2;
    static constexpr size_t b_half_bytes = (size_t)(BN / 2) * RK * 2;  // BN/2 rows of one term
    // this CTA's rows: all BN rows of its stacked term (hi or mid), then BN/2 rows of lo
    static constexpr size_t b_stack_bytes = 2 * b_half_bytes;
    static constexpr size_t b_bytes = kTerms * b_half_bytes;
    static constexpr size_t ring = STAGES * (a_bytes + b_bytes);
    static constexpr size_t barriers = (2 * STAGES + 2 + 2 + 1) * 8 + 16;
    // bias, per-quarter sums of p and per-64-token counts (both double-buffered by tile parity),
    // and the exchange of per-group max, argmax and sum between the warps of a token
    // (+ the exchange of each group's entropy partial and per-quarter entropy sums, both parities)
    static constexpr size_t epi =
        (size_t)BN * 4 + 2 * 4 * BN * 4 + 2 * 2 * BN * 4 + 3 * (BN / 32) * RM * 4 + (BN / 32) * RM * 4 + 2 * 4 * 4;
    // top-2: second-choice counts and the exchange of each group's second best
    static constexpr size_t epi2 = TOP2 ? 2 * 2 * BN * 4 + 2 * (BN / 32) * RM * 4 : 0;
    static constexpr size_t bytes = 1024 + ring + barriers + epi + epi2;
};

// Sum v[i] over the 32 lanes for every i; lane l ends with the total of index l.
__device__ __forceinline__ float reduce_scatter32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int off = 16 >> step;
        const int half = 16 >> step;
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i < half) {
                const float send = upper ? v[i] : v[i + half];
                const float keep = upper ? v[i + half] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
            }
        }
    }
    return v[0];
}

template <int NT>
__device__ __forceinline__ void named_barrier_epilogue() {
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// 2-D TMA load into this CTA's shared memory, counted on the mbarrier at
// `bar_cluster_addr` (the leader's).  No multicast load.
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const void *tmap, uint32_t bar_cluster_addr,
                                                 int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster_addr), "r"(c0), "r"(c1)
        : "memory");
}

// Top-2 bookkeeping: keep the best two (value, index) pairs, larger value
// first, lower index first among equal values, whatever the insertion order.
__device__ __forceinline__ bool better_pair(float v, int i, float m, int a) { return v > m || (v == m && i < a); }
__device__ __forceinline__ void insert_top2(float v, int i, float &m1, int &a1, float &m2, int &a2) {
    if (better_pair(v, i, m1, a1)) {
        m2 = m1;
        a2 = a1;
        m1 = v;
        a1 = i;
    } else if (better_pair(v, i, m2, a2)) {
        m2 = v;
        a2 = i;
    }
}

template <int BN, int STAGES, bool TOP2>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(RouterThreads<BN>::kAll, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const float *__restrict__ bias, int64_t T, int d, int N, int tiles64,
                     int32_t *__restrict__ expert, float *__restrict__ gate, int32_t *__restrict__ hist,
                     int32_t *__restrict__ hist2, float *__restrict__ psum, float *__restrict__ probs,
                     float *__restrict__ ent, uint32_t *ticket, DeviceStatus *status) {
    using L = RouterLayout<BN, STAGES, TOP2>;
    constexpr int PM = 2 * RM;  // tokens per pair tile
    constexpr int G = RouterThreads<BN>::kGroups;
    constexpr int kEpiThreads = RouterThreads<BN>::kEpi;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = sA + STAGES * L::a_bytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(base + L::ring);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    float *bias_s = reinterpret_cast<float *>(tmem_holder + 4);
    float *psum_w = bias_s + BN;                                     // [2 parity][4 quarters][BN]
    int32_t *hist_s = reinterpret_cast<int32_t *>(psum_w + 8 * BN);  // [2 parity][2 halves][BN]
    float *x_max = reinterpret_cast<float *>(hist_s + 4 * BN);       // [G column groups][RM]
    int32_t *x_arg = reinterpret_cast<int32_t *>(x_max + G * RM);    // [G][RM]
    float *x_sum = reinterpret_cast<float *>(x_arg + G * RM);        // [G][RM]
    float *x_ent = x_sum + G * RM;                                   // [G][RM] sum of e (h - max), with ent
    float *ent_q = x_ent + G * RM;                                   // [2 parity][4 quarters] entropy sums
    // top-2 only (inside epi2): second-choice counts and each group's second best
    int32_t *hist2_s = reinterpret_cast<int32_t *>(ent_q + 8);       // [2 parity][2 halves][BN]
    float *x_max2 = reinterpret_cast<float *>(hist2_s + 4 * BN);     // [G][RM]
    int32_t *x_arg2 = reinterpret_cast<int32_t *>(x_max2 + G * RM);  // [G][RM]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int m_tiles = (int)((T + PM - 1) / PM);
    const int k_blocks = (d + RK - 1) / RK;
    constexpr uint32_t kAccCols = 2 * BN;  // x . (hi + lo) in [0, BN), x . mid in [BN, 2 BN)
    constexpr uint32_t kTmemCols = 2 * kAccCols;

    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *ticket = 0u;
        status->code = 0;
        status->where = 0;
        status->block = 0;
        status->reserved = 0;
    }
    if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            for (int a = 0; a < 2; ++a) {
                mbar_init(&acc_full[a], 1);
                mbar_init(&acc_empty[a], 2 * kEpiThreads);
            }
            mbar_init(drain, 1);
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc_pair(tmem_holder, kTmemCols);
        tmem_relinquish_pair();
    } else if (warp >= 2) {
        const int et = threadIdx.x - 64;
        for (int i = et; i < BN; i += kEpiThreads) bias_s[i] = (bias && i < N) ? bias[i] : 0.f;
        for (int i = et; i < 4 * BN; i += kEpiThreads) {
            hist_s[i] = 0;
            if (TOP2) hist2_s[i] = 0;
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers are initialised before anyone signals them
    tc_fence_after();
    pdl_wait();  // the split terms of W_r come from the previous kernel
    pdl_launch_dependents();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmap_x);
            prefetch_tmap(&tmap_w);
            uint32_t issued = 0, parity_of = 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const int my_rows = (int)rank * RM;
            for (int tile = pair; ok && tile < m_tiles; tile += n_pairs) {
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, status, 31)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 * (L::a_bytes + L::b_bytes)));
                    const uint32_t leader_full = map_to_rank(&full[stage], 0);
                    tma_load_2d_pair(sA + stage * L::a_bytes, &tmap_x, leader_full, kb * RK, tile * PM + my_rows);
                    uint8_t *b_stage = sB + stage * L::b_bytes;
                    tma_load_3d_pair(b_stage, &tmap_w, leader_full, kb * RK, 0, (int)rank);  // hi or mid
                    tma_load_3d_pair(b_stage + L::b_half_bytes, &tmap_w, leader_full, kb * RK, BN / 2, (int)rank);
                    tma_load_3d_pair(b_stage + L::b_stack_bytes, &tmap_w, leader_full, kb * RK,
                                     (int)rank * (BN / 2), 2);  // lo
                    issued |= 1u << stage;
                    parity_of = (parity_of & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (rank == 0)
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s)) mbar_wait(&full[s], (parity_of >> s) & 1u, status, 36);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc_stack = idesc_bf16_f32(PM, 2 * BN);
            constexpr uint32_t idesc_lo = idesc_bf16_f32(PM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < m_tiles; tile += n_pairs) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, status, 32)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, status, 33)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = smem_desc_sw128(sA + stage * L::a_bytes);
                    const uint64_t b_stack = smem_desc_sw128(sB + stage * L::b_bytes);
                    const uint64_t b_lo = smem_desc_sw128(sB + stage * L::b_bytes + L::b_stack_bytes);
#pragma unroll
                    for (int k = 0; k < RK / 16; ++k) {
                        tc_mma_bf16_pair(d_tmem, a_desc + (uint64_t)(2 * k), b_stack + (uint64_t)(2 * k),
                                         idesc_stack, (kb | k) != 0 ? 1u : 0u);
                        tc_mma_bf16_pair(d_tmem, a_desc + (uint64_t)(2 * k), b_lo + (uint64_t)(2 * k), idesc_lo,
                                         1u);
                    }
                    tc_commit_both(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_both(&acc_full[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            tc_commit_pair(smem_u32(drain));
            mbar_wait(drain, 0, status, 34);
        }
    } else {
        constexpr int CW = 32;               // columns per warp
        const int q = warp & 3;              // TMEM lane quarter: tokens 32q .. 32q+31 of this CTA's rows
        const int grp = (warp - 2) >> 2;     // column group: experts 32 grp .. 32 grp + 31
        const int col0 = grp * CW;
        const int tok = q * 32 + lane;       // token within this CTA's 128 rows
        const int et = threadIdx.x - 64;
        const uint32_t acc_empty_leader0 = map_to_rank(&acc_empty[0], 0);
        const uint32_t acc_empty_leader1 = map_to_rank(&acc_empty[1], 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        int par = 0;
        for (int tile = pair; tile < m_tiles; tile += n_pairs) {
            if (!mbar_wait(&acc_full[acc], acc_phase, status, 35)) break;
            tc_fence_after();
            const int64_t row0 = (int64_t)tile * PM + (int64_t)rank * RM;  // this CTA's first token
            const int64_t t = row0 + tok;
            const bool valid = t < T;
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kAccCols + col0);
            float h[CW];
            {
                uint32_t r[32], r2[32];
                tmem_ld_32x32b_x32(t_row, r);                       // x . (hi + lo)
                tmem_ld_32x32b_x32(t_row + (uint32_t)BN, r2);       // x . mid
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) h[j] = (__uint_as_float(r[j]) + __uint_as_float(r2[j])) + bias_s[col0 + j];
            }
            tc_fence_before();
            mbar_arrive_cluster(acc ? acc_empty_leader1 : acc_empty_leader0);  // columns in registers: reusable
            float mx, mx2 = -FLT_MAX;
            int amax, amax2 = 0x7fffffff;
            if (TOP2) {
                // best two of this group's 32 columns, then of all groups
                float m1 = -FLT_MAX, m2 = -FLT_MAX;
                int a1 = 0x7fffffff, a2 = 0x7fffffff;
#pragma unroll
                for (int j = 0; j < CW; ++j)
                    if (col0 + j < N) insert_top2(h[j], col0 + j, m1, a1, m2, a2);
                x_max[grp * RM + tok] = m1;
                x_arg[grp * RM + tok] = a1;
                x_max2[grp * RM + tok] = m2;
                x_arg2[grp * RM + tok] = a2;
                named_barrier_epilogue<kEpiThreads>();
                m1 = x_max[tok];
                a1 = x_arg[tok];
                m2 = x_max2[tok];
                a2 = x_arg2[tok];
#pragma unroll
                for (int g = 1; g < G; ++g) {
                    insert_top2(x_max[g * RM + tok], x_arg[g * RM + tok], m1, a1, m2, a2);
                    insert_top2(x_max2[g * RM + tok], x_arg2[g * RM + tok], m1, a1, m2, a2);
                }
                if (a1 == 0x7fffffff) a1 = 0;  // no comparable logit (NaN inputs): keep indices in range
                if (a2 == 0x7fffffff) a2 = a1 == 0 ? 1 : 0;
                mx = m1;
                amax = a1;
                mx2 = m2;
                amax2 = a2;
            } else {
            // four interleaved max / argmax chains (j = u mod 4), then merged with
            // ties going to the lowest index, as a single left-to-right scan would
            float m4[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
            int a4[4] = {col0, col0 + 1, col0 + 2, col0 + 3};
#pragma unroll
            for (int j = 0; j < CW; j += 4) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (col0 + j + u < N && h[j + u] > m4[u]) {  // strict: the lowest index of the chain wins
                        m4[u] = h[j + u];
                        a4[u] = col0 + j + u;
                    }
                }
            }
            float m = m4[0];
            int arg = a4[0];
#pragma unroll
            for (int u = 1; u < 4; ++u) {
                if (m4[u] > m || (m4[u] == m && a4[u] < arg)) {
                    m = m4[u];
                    arg = a4[u];
                }
            }
            x_max[grp * RM + tok] = m;
            x_arg[grp * RM + tok] = arg;
            named_barrier_epilogue<kEpiThreads>();
            mx = x_max[tok];
            amax = x_arg[tok];
#pragma unroll
            for (int g = 1; g < G; ++g) {  // groups in column order; strict: ties keep the lower index
                const float v = x_max[g * RM + tok];
                if (v > mx) {
                    mx = v;
                    amax = x_arg[g * RM + tok];
                }
            }
            }
            // __expf (hardware exp2 of a scaled argument): arguments are <= 0 here
            // and its relative error, a few 1e-6 over the range that matters, moves
            // the gates by well under the 1e-5 parity bound; the full-precision
            // expf made this phase the longest of the epilogue
            float s4[4] = {0.f, 0.f, 0.f, 0.f};  // four interleaved partial sums, merged in fixed order
            float sv = 0.f;                       // with ent: sum of e (h - max) over this group
#pragma unroll
            for (int j = 0; j < CW; j += 4) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float z = h[j + u] - mx;
                    h[j + u] = col0 + j + u < N ? __expf(z) : 0.f;
                    s4[u] += h[j + u];
                    if (ent && col0 + j + u < N) sv += h[j + u] * z;
                }
            }
            x_sum[grp * RM + tok] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            if (ent) x_ent[grp * RM + tok] = sv;
            named_barrier_epilogue<kEpiThreads>();
            float s_all = x_sum[tok];
#pragma unroll
            for (int g = 1; g < G; ++g) s_all += x_sum[g * RM + tok];
            const float inv_s = 1.0f / s_all;
            if (ent && grp == 0) {  // entropy -sum p ln p = ln s - sum e (h - max) / s; summed over the warp's tokens
                float sv_all = x_ent[tok];
#pragma unroll
                for (int g = 1; g < G; ++g) sv_all += x_ent[g * RM + tok];
                float hq = valid ? __logf(s_all) - sv_all * inv_s : 0.f;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) hq += __shfl_xor_sync(0xffffffffu, hq, off);
                if (lane == 0) ent_q[par * 4 + q] = hq;
            }
            float *psum_p = psum_w + par * 4 * BN;
            int32_t *hist_p = hist_s + par * 2 * BN;
            {
                float p[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) p[j] = valid ? h[j] * inv_s : 0.f;
                if (probs && valid) {  // kept for the backward pass
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (col0 + j < N) probs[t * N + col0 + j] = p[j];
                }
                const float col_sum = reduce_scatter32(p);  // this warp's 32 tokens, column col0 + lane
                psum_p[q * BN + col0 + lane] = col_sum;
            }
            if (valid && grp == 0) {
                if (TOP2) {
                    expert[2 * t] = amax;
                    expert[2 * t + 1] = amax2;
                    gate[2 * t] = inv_s;
                    gate[2 * t + 1] = __expf(mx2 - mx) * inv_s;
                    atomicAdd(&hist2_s[par * 2 * BN + (q >> 1) * BN + amax2], 1);
                } else {
                    expert[t] = amax;
                    gate[t] = inv_s;  // p at the argmax: exp(0) / s
                }
                atomicAdd(&hist_p[(q >> 1) * BN + amax], 1);
            }
            named_barrier_epilogue<kEpiThreads>();
            // the buffers of this parity are next written two tiles later, after two more barriers
            const int t64_0 = (int)(row0 / 64);
            for (int i = et; i < N; i += kEpiThreads) {
#pragma unroll
                for (int h64 = 0; h64 < 2; ++h64) {
                    const int t64 = t64_0 + h64;
                    if (ent && i == 0 && t64 < tiles64)
                        ent[t64] = ent_q[par * 4 + 2 * h64] + ent_q[par * 4 + 2 * h64 + 1];
                    if (t64 < tiles64) {
                        hist[(int64_t)i * tiles64 + t64] = hist_p[h64 * BN + i];
                        psum[(int64_t)i * tiles64 + t64] = psum_p[(2 * h64) * BN + i] + psum_p[(2 * h64 + 1) * BN + i];
                        if (TOP2) hist2[(int64_t)i * tiles64 + t64] = hist2_s[par * 2 * BN + h64 * BN + i];
                    }
                    hist_p[h64 * BN + i] = 0;
                    if (TOP2) hist2_s[par * 2 * BN + h64 * BN + i] = 0;
                }
            }
            par ^= 1;
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int BN, int STAGES, bool TOP2>
cudaError_t launch_bn(const switch_dims_t &dims, const __nv_bfloat16 *x, const float *bias, int32_t *expert,
                      float *gate, const Workspace &ws, cudaStream_t stream) {
    const int N = dims.num_experts, d = dims.d_model;
    const int64_t T = dims.T;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    CUtensorMap tx, tw;
    const cuuint32_t estr[3] = {1, 1, 1};
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)T};
        const cuuint64_t gstr[1] = {(cuuint64_t)d * 2};
        const cuuint32_t box[2] = {(cuuint32_t)RK, (cuuint32_t)RM};
        if (fn(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(x), gdim, gstr, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t gdim[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)kTerms};
        const cuuint64_t gstr[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
        const cuuint32_t box[3] = {(cuuint32_t)RK, (cuuint32_t)(BN / 2), 1};
        if (fn(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ws.w_split, gdim, gstr, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    auto kern = router_tc_kernel<BN, STAGES, TOP2>;
    const size_t smem = RouterLayout<BN, STAGES, TOP2>::bytes;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int64_t m_tiles = (T + 2 * RM - 1) / (2 * RM);
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(device_sm_count() / 2, m_tiles));
    launch_begin(K_ROUTER_TC, stream);
    err = launch_kernel(kern, dim3(2 * pairs), dim3(RouterThreads<BN>::kAll), smem, stream, true, tx, tw, bias, T, d,
                        N, (int)ws.tiles, expert, gate, ws.hist, ws.hist2, ws.psum, ws.probs, ws.ent, ws.ticket,
                        static_cast<DeviceStatus *>(ws.status));
    launch_end(stream);
    return err;
}

}  // namespace

// For N <= 32 the CUDA-core router with the x tile staged in shared memory
// was faster on B200 (Base-8 shape: 15.6 us against 16.7 + 6.5 us).
bool router_tc_supported(const switch_dims_t &dims) {
    return dims.dtype == SWITCH_BF16 && dims.num_experts > 32 && dims.num_experts <= 128 && dims.T > 0 &&
           !(dims.flags & SWITCH_FLAG_SIMT_ROUTER);
}

cudaError_t launch_router_tc(const switch_dims_t &dims, const void *x, const float *w_r, const float *bias,
                             int32_t *expert, float *gate, const Workspace &ws, cudaStream_t stream, bool top2) {
    const int64_t n = (int64_t)dims.num_experts * dims.d_model;
    launch_begin(K_ROUTER_SPLIT, stream);
    split_router_weight<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, stream>>>(
        w_r, static_cast<__nv_bfloat16 *>(ws.w_split), n);
    cudaError_t err = cudaGetLastError();
    launch_end(stream);
    if (err != cudaSuccess) return err;
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
    if (top2) {
        if (dims.num_experts <= 64) return launch_bn<64, 7, true>(dims, xb, bias, expert, gate, ws, stream);
        return launch_bn<128, 5, true>(dims, xb, bias, expert, gate, ws, stream);
    }
    if (dims.num_experts <= 64) return launch_bn<64, 7, false>(dims, xb, bias, expert, gate, ws, stream);
    return launch_bn<128, 5, false>(dims, xb, bias, expert, gate, ws, stream);
}

}  // namespace switchmoe
