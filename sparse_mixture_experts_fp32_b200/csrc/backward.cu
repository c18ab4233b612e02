// Backward pass of the Switch layer (top-1, bfloat16 experts), sm_100a.
//
// Given the upstream gradient dy [T, d] of the layer output y and the scalar
// upstream gradient g_aux of the aux loss, computes dx, dW_r, d(logit bias),
// dW_in and dW_out.  The argmax and the capacity assignment pass no gradient:
// the router learns through the selected probability p_i*(x) that scales the
// expert output (kasblo "Switch Transformerとは？", section "argmaxは離散なの
// に、Routerはなぜ学習できるのか"), and through P_i in the aux loss, f_i being
// a count (llm-papers-study "精读 06 | Switch Transformers" §3.3).  With
// z = W_in x, u = ReLU(z), o = W_out u, y = p_i* o for a kept token:
//   g_gate = dy . o                      dE = p_i* dy          (bwd_token_kernel)
//   dp_i = [i = i*] g_gate + g_aux N f_i / T,  dh = p (dp - p . dp)
//   dZ = (dE W_out[i*]) masked by z > 0  (tcgen05 GEMM, epilogue kEpiReluGrad)
//   dx = dh W_r + dZ W_in[i*]            (tcgen05 GEMM on exact bf16 splits of dh
//                                         and W_r, then a tcgen05 GEMM whose
//                                         epilogue adds into dx rows)
//   dW_out[i] = sum over kept tokens of dE u^T   (tcgen05 GEMM over K = tokens)
//   dW_in[i]  = sum over kept tokens of dZ x^T   (tcgen05 GEMM over K = tokens)
//   dW_r = sum_t dh x^T, d bias = sum_t dh        (tcgen05 GEMM per chunk of tokens
//                                         on the split dh, + fixed-order reduce)
// With SWITCH_FLAG_SIMT_ROUTER the two router products run as float32 FMA
// kernels instead (router_dx_kernel, router_dw_kernel).
// The expert GEMMs are the forward's grouped "A . B^T" pair kernel reading
// the weights and the per-expert activation buffers where they lie, as
// MN-major operands where the contraction runs along their rows (W_out and
// W_in for dZ and dx; dE, H, dZ and xbuf along the tokens for the weight
// gradients; x along its tokens for the tensor-core dW_r), so nothing is
// transposed in HBM; rows past an expert's kept tokens up to the next
// multiple of 64 are zeroed first, so the weight-gradient GEMMs only see kept
// tokens.  Every reduction runs in a fixed order: identical inputs give
// identical bytes.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// One warp per token: the gate gradient g_gate = dy . o (o = the forward's
// ungated expert output), dE[e, s] = bf16(gate * dy) for a kept token, then
// the softmax backward over the N probabilities kept by the forward.
__global__ void __launch_bounds__(kThreads) bwd_token_kernel(const float *__restrict__ dy, const float *__restrict__ ybuf,
                                                            const int32_t *__restrict__ expert,
                                                            const int32_t *__restrict__ slot,
                                                            const float *__restrict__ gate,
                                                            const float *__restrict__ probs,
                                                            const int32_t *__restrict__ counts, int64_t T, int d,
                                                            int N, int C, float g_aux, __nv_bfloat16 *__restrict__ dE,
                                                            float *__restrict__ dh) {
    const int64_t t = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (t >= T) return;
    const int lane = threadIdx.x & 31;
    const int s = slot[t], e = expert[t];
    float g = 0.f;
    if (s >= 0) {
        const float gt = gate[t];
        const float4 *o = reinterpret_cast<const float4 *>(ybuf + ((int64_t)e * C + s) * d);
        const float4 *dyt = reinterpret_cast<const float4 *>(dy + t * d);
        uint2 *de = reinterpret_cast<uint2 *>(dE + ((int64_t)e * C + s) * d);
        float acc = 0.f;
        for (int w = lane; w < d / 4; w += 32) {
            const float4 a = __ldg(dyt + w), b = __ldg(o + w);
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
            acc = fmaf(a.z, b.z, acc);
            acc = fmaf(a.w, b.w, acc);
            de[w] = make_uint2(pack_bf16x2(gt * a.x, gt * a.y), pack_bf16x2(gt * a.z, gt * a.w));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        g = acc;
    }
    const float *pt = probs + t * N;
    const float c_aux = g_aux * (float)N / ((float)T * (float)T);
    float dot = 0.f;
    for (int i = lane; i < N; i += 32) {
        const float dp = (i == e ? g : 0.f) + c_aux * (float)counts[i];
        dot = fmaf(pt[i], dp, dot);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    for (int i = lane; i < N; i += 32) {
        const float dp = (i == e ? g : 0.f) + c_aux * (float)counts[i];
        dh[t * N + i] = pt[i] * (dp - dot);
    }
}

// dx[t, :] = sum_i dh[t, i] W_r[i, :]  (overwrites dx; the expert part is
// added afterwards).  Block: 64 tokens x 128 columns; thread: 8 tokens x 4
// columns; experts in chunks of 32 through shared memory, dh stored
// expert-major so that a thread's 8 tokens are two 16-byte reads.
constexpr int kDxTok = 64, kDxCol = 128, kDxI = 32, kDxPitch = kDxTok + 8;
__global__ void __launch_bounds__(256) router_dx_kernel(const float *__restrict__ dh, const float *__restrict__ w_r,
                                                       int64_t T, int N, int d, float *__restrict__ dx) {
    __shared__ __align__(16) float s_dh[kDxI][kDxPitch];  // [expert][token]
    __shared__ __align__(16) float s_w[kDxI][kDxCol];
    const int64_t t0 = (int64_t)blockIdx.y * kDxTok;
    const int k0 = blockIdx.x * kDxCol;
    const int tid = threadIdx.x;
    const int tc = tid & 31;   // columns k0 + 4 tc .. + 3
    const int tt = tid >> 5;   // tokens t0 + 8 tt .. + 7
    float acc[8][4] = {};
    for (int i0 = 0; i0 < N; i0 += kDxI) {
        __syncthreads();
        for (int q = tid; q < kDxI * kDxTok; q += 256) {  // coalesced along the experts of a token
            const int ii = q % kDxI, tl = q / kDxI;
            const int64_t t = t0 + tl;
            s_dh[ii][tl] = (t < T && i0 + ii < N) ? dh[t * N + i0 + ii] : 0.f;
        }
        for (int q = tid; q < kDxI * kDxCol; q += 256) {
            const int ii = q / kDxCol, kk = q % kDxCol;
            s_w[ii][kk] = (i0 + ii < N && k0 + kk < d) ? w_r[(int64_t)(i0 + ii) * d + k0 + kk] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int ii = 0; ii < kDxI; ++ii) {
            const float4 w = *reinterpret_cast<const float4 *>(&s_w[ii][4 * tc]);
            const float4 a0 = *reinterpret_cast<const float4 *>(&s_dh[ii][8 * tt]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&s_dh[ii][8 * tt + 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                acc[j][0] = fmaf(a[j], w.x, acc[j][0]);
                acc[j][1] = fmaf(a[j], w.y, acc[j][1]);
                acc[j][2] = fmaf(a[j], w.z, acc[j][2]);
                acc[j][3] = fmaf(a[j], w.w, acc[j][3]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int64_t t = t0 + 8 * tt + j;
        const int k = k0 + 4 * tc;
        if (t < T && k < d)  // d % 64 == 0 on this path: the four columns are in range together
            *reinterpret_cast<float4 *>(dx + t * d + k) = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
    }
}

// Partial sums of dW_r and d bias over chunks of tokens:
//   part_w[chunk][i][k] = sum_{t in chunk} dh[t, i] x[t, k],  part_b[chunk][i] = sum dh[t, i]
// Block: 64 experts x 128 columns of one chunk; thread: 4 consecutive experts x
// 8 columns (three 16-byte shared-memory reads per 32 FMAs).
constexpr int kDwI = 64, kDwCol = 128, kDwTok = 32, kDwPitch = kDwI + 4;
__global__ void __launch_bounds__(256) router_dw_kernel(const float *__restrict__ dh, const uint16_t *__restrict__ x,
                                                       int64_t T, int N, int d, int64_t chunk_tokens,
                                                       float *__restrict__ part_w, float *__restrict__ part_b) {
    __shared__ __align__(16) float s_dh[kDwTok][kDwPitch];  // [token][expert]
    __shared__ __align__(16) float s_x[kDwTok][kDwCol];
    const int k0 = blockIdx.x * kDwCol, i0 = blockIdx.y * kDwI;
    const int chunk = blockIdx.z;
    const int64_t tbeg = (int64_t)chunk * chunk_tokens;
    const int64_t tend = min(T, tbeg + chunk_tokens);
    const int tid = threadIdx.x;
    const int tk = tid & 15;   // columns k0 + 8 tk .. + 7
    const int ti = tid >> 4;   // experts i0 + 4 ti .. + 3
    float acc[4][8] = {};
    float accb[4] = {0.f, 0.f, 0.f, 0.f};  // d bias of the thread's four experts (written by tk == 0)
    for (int64_t tb = tbeg; tb < tend; tb += kDwTok) {
        __syncthreads();
        for (int q = tid; q < kDwTok * kDwI; q += 256) {
            const int ii = q % kDwI, tl = q / kDwI;
            const int64_t t = tb + tl;
            s_dh[tl][ii] = (t < tend && i0 + ii < N) ? dh[t * N + i0 + ii] : 0.f;
        }
        for (int q = tid; q < kDwTok * kDwCol / 2; q += 256) {
            const int tl = q / (kDwCol / 2), kk = 2 * (q % (kDwCol / 2));
            const int64_t t = tb + tl;
            uint32_t v = 0u;
            if (t < tend && k0 + kk < d) v = *reinterpret_cast<const uint32_t *>(x + t * d + k0 + kk);
            s_x[tl][kk] = __uint_as_float(v << 16);
            s_x[tl][kk + 1] = __uint_as_float(v & 0xffff0000u);
        }
        __syncthreads();
#pragma unroll 4
        for (int tl = 0; tl < kDwTok; ++tl) {
            const float4 xa = *reinterpret_cast<const float4 *>(&s_x[tl][8 * tk]);
            const float4 xb = *reinterpret_cast<const float4 *>(&s_x[tl][8 * tk + 4]);
            const float4 h4 = *reinterpret_cast<const float4 *>(&s_dh[tl][4 * ti]);
            const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            const float hv[4] = {h4.x, h4.y, h4.z, h4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[j][c] = fmaf(hv[j], xv[c], acc[j][c]);
                accb[j] += hv[j];  // every thread: no divergent branch in the inner loop
            }
        }
    }
    float *pw = part_w + (int64_t)chunk * N * d;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int i = i0 + 4 * ti + j;
        const int k = k0 + 8 * tk;
        if (i < N && k < d) {
            float4 *dst = reinterpret_cast<float4 *>(pw + (int64_t)i * d + k);
            dst[0] = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
            dst[1] = make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]);
        }
        if (tk == 0 && blockIdx.x == 0 && i < N) part_b[(int64_t)chunk * N + i] = accb[j];
    }
}

// Sum the chunk partials in chunk order: out[j] = sum_c part[c][j].
__global__ void reduce_chunks_kernel(const float *__restrict__ part, int chunks, int64_t n, float *__restrict__ out) {
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int c = 0; c < chunks; ++c) acc += part[(int64_t)c * n + j];
        out[j] = acc;
    }
}

// ---------------------------------------------------------------------------
// Router backward on the tensor cores.  Both router products are dense
// float32 contractions (dx += dh W_r over the N experts, dW_r = dh^T x over
// the tokens); they run as bf16 tcgen05 GEMMs on exact three-term splits of
// their float32 operands (split_bf16x3; x is bf16 already):
//   dx:   sum over the six term pairs (dh_a, W_b) with a + b <= 2 of
//         dh_a W_b, laid side by side along K (K = 6 Np, Np = N rounded up
//         to 64, zero columns past N).  The three dropped pairs are below
//         2^-23 of |dh| |W_r| together.
//   dW_r: the three dh terms stacked as rows (M = 3N) against x^T, per chunk
//         of Tc tokens (the chunks are the GEMM's groups, K = Tc), then a
//         fixed-order sum over terms and chunks.
// Products of bf16 terms are exact in float32; the tensor cores accumulate
// in float32.
// ---------------------------------------------------------------------------
constexpr int kDxPairs = 6;
__device__ __forceinline__ int dx_dh_term(int p) { return p < 3 ? 0 : (p < 5 ? 1 : 2); }  // 0 0 0 1 1 2
__device__ __forceinline__ int dx_w_term(int p) { return p < 3 ? p : (p < 5 ? p - 3 : 0); }  // 0 1 2 0 1 0

// A operand of the dx product: a[t][p * Np + i] = term dx_dh_term(p) of dh[t, i]
// (zero for i >= N).  One thread per 8 experts of a token.
__global__ void __launch_bounds__(256) router_dx_a_kernel(const float *__restrict__ dh, int64_t T, int N, int Np,
                                                         uint16_t *__restrict__ a) {
    const int oct = Np / 8;
    const int64_t total = T * oct;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = q / oct;
        const int i0 = (int)(q % oct) * 8;
        uint16_t sp[8][3];
#pragma unroll
        for (int j = 0; j < 8; ++j) split_bf16x3(i0 + j < N ? dh[t * N + i0 + j] : 0.f, sp[j]);
        uint16_t *row = a + t * (int64_t)(kDxPairs * Np) + i0;
#pragma unroll
        for (int p = 0; p < kDxPairs; ++p) {
            const int m = dx_dh_term(p);
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = (uint32_t)sp[2 * j][m] | ((uint32_t)sp[2 * j + 1][m] << 16);
            *reinterpret_cast<uint4 *>(row + p * Np) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// B operand of the dx product: b[k][p * Np + i] = term dx_w_term(p) of W_r[i, k]
// (zero for i >= N); also the token count of every dW_r chunk and a 1 at
// chunk_counts[chunks] (the single group of the dx GEMM).
__global__ void __launch_bounds__(256) router_dx_b_kernel(const float *__restrict__ w_r, int N, int d, int Np,
                                                         uint16_t *__restrict__ b, int64_t T, int64_t chunk_tokens,
                                                         int chunks, int32_t *__restrict__ chunk_counts) {
    const int oct = Np / 8;
    const int64_t total = (int64_t)d * oct;
    const int64_t first = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t c = first; c <= chunks; c += (int64_t)gridDim.x * blockDim.x)
        chunk_counts[c] = c < chunks ? (int32_t)min(chunk_tokens, T - c * chunk_tokens) : 1;
    for (int64_t q = first; q < total; q += (int64_t)gridDim.x * blockDim.x) {
        const int k = (int)(q / oct);
        const int i0 = (int)(q % oct) * 8;
        uint16_t sp[8][3];
#pragma unroll
        for (int j = 0; j < 8; ++j) split_bf16x3(i0 + j < N ? w_r[(int64_t)(i0 + j) * d + k] : 0.f, sp[j]);
        uint16_t *row = b + (int64_t)k * (kDxPairs * Np) + i0;
#pragma unroll
        for (int p = 0; p < kDxPairs; ++p) {
            const int m = dx_w_term(p);
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = (uint32_t)sp[2 * j][m] | ((uint32_t)sp[2 * j + 1][m] << 16);
            *reinterpret_cast<uint4 *>(row + p * Np) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// A operand of the dW_r product, transposed per chunk of Tc tokens:
// a[c][m * N + i][tl] = term m of dh[c Tc + tl, i] (zero past T), and the
// chunk's d bias partial db_part[c][i] = sum over its tokens of dh[t, i] in
// token order.  Block: one chunk x 32 experts, 128-token tiles through shared
// memory; lane = expert, each thread writes 16 tokens (32 bytes) of one term.
constexpr int kDwtTok = 128;
__global__ void __launch_bounds__(256) router_dw_a_kernel(const float *__restrict__ dh, int64_t T, int N,
                                                         int64_t chunk_tokens, uint16_t *__restrict__ a,
                                                         float *__restrict__ db_part) {
    __shared__ float s[kDwtTok][33];
    const int c = blockIdx.x, i0 = blockIdx.y * 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t tbeg = (int64_t)c * chunk_tokens;
    float acc_b = 0.f;
    for (int64_t tl0 = 0; tl0 < chunk_tokens; tl0 += kDwtTok) {
        __syncthreads();
        for (int q = tid; q < kDwtTok * 32; q += 256) {
            const int tl = q >> 5, ii = q & 31;
            const int64_t t = tbeg + tl0 + tl;
            s[tl][ii] = (t < T && tl0 + tl < chunk_tokens && i0 + ii < N) ? dh[t * N + i0 + ii] : 0.f;
        }
        __syncthreads();
        if (warp == 0)
            for (int tl = 0; tl < kDwtTok; ++tl) acc_b += s[tl][lane];
        const int i = i0 + lane;
        if (i < N) {
            for (int combo = warp; combo < 3 * (kDwtTok / 16); combo += 8) {
                const int m = combo / (kDwtTok / 16), q = combo % (kDwtTok / 16);
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint16_t lo[3], hi[3];
                    split_bf16x3(s[16 * q + 2 * j][lane], lo);
                    split_bf16x3(s[16 * q + 2 * j + 1][lane], hi);
                    w[j] = (uint32_t)lo[m] | ((uint32_t)hi[m] << 16);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(a + (((int64_t)c * 3 * N + (int64_t)m * N + i) * chunk_tokens +
                                                            tl0 + 16 * q));
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
        }
    }
    if (warp == 0 && i0 + lane < N) db_part[(int64_t)c * N + i0 + lane] = acc_b;
}

// dW_r[i][k] = sum over chunks c, in order, of (part[c][2N + i][k] + part[c][N + i][k]) + part[c][i][k].
__global__ void router_dw_reduce_kernel(const float *__restrict__ part, int chunks, int N, int d,
                                        float *__restrict__ dw_r) {
    const int64_t n = (int64_t)N * d, term = (int64_t)N * d;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int c = 0; c < chunks; ++c) {
            const float *pc = part + (int64_t)c * 3 * term;
            acc += (pc[2 * term + j] + pc[term + j]) + pc[j];
        }
        dw_r[j] = acc;
    }
}

// The weight-gradient GEMMs read the token-indexed buffers dE, H, dZ and
// xbuf along K = tokens in blocks of 64: block (expert e, row r) zeroes row
// kept_e + r of each of them when that row lies below both C and kept_e
// rounded up to 64 (those rows hold values of no token).
__global__ void __launch_bounds__(256) zero_tails_kernel(const int32_t *__restrict__ counts, int C, int d, int F,
                                                        uint16_t *__restrict__ grad_e, uint16_t *__restrict__ xbuf,
                                                        uint16_t *__restrict__ hidden, uint16_t *__restrict__ grad_z) {
    const int e = blockIdx.x;
    const int kept = min(counts[e], C);
    const int row = kept + (int)blockIdx.y;
    if (kept == 0 || row >= C || row >= (kept + 63) / 64 * 64) return;
    const int64_t r = (int64_t)e * C + row;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int w = threadIdx.x; w < d / 8; w += blockDim.x) {
        reinterpret_cast<uint4 *>(grad_e + r * d)[w] = z;
        reinterpret_cast<uint4 *>(xbuf + r * d)[w] = z;
    }
    for (int w = threadIdx.x; w < F / 8; w += blockDim.x) {
        reinterpret_cast<uint4 *>(hidden + r * F)[w] = z;
        reinterpret_cast<uint4 *>(grad_z + r * F)[w] = z;
    }
}


}  // namespace

// Chunks of tokens for the dW_r partial sums (enough blocks to fill the GPU,
// each chunk long enough that the partials stay small).
int64_t router_dw_chunks(int64_t T) {
    const int64_t c = (T + 2047) / 2048;
    return c < 1 ? 1 : (c > 64 ? 64 : c);
}

// Tokens per chunk of the tensor-core dW_r product: a multiple of 128, at
// least 256, and at most 64 chunks.
int64_t router_tc_chunk_tokens(int64_t T) {
    int64_t tc = ((T + 63) / 64 + 127) / 128 * 128;
    return tc < 256 ? 256 : tc;
}
int64_t router_tc_chunks(int64_t T) {
    const int64_t tc = router_tc_chunk_tokens(T);
    return T > 0 ? (T + tc - 1) / tc : 1;
}
int router_tc_np(int N) { return (N + 63) / 64 * 64; }

cudaError_t launch_layer_bwd(const switch_dims_t &dims, const void *x, const float *w_r, const void *w_in,
                             const void *w_out, const int32_t *expert, const float *gate, const int32_t *slot,
                             const int32_t *counts, const float *dy, float g_aux, float *dx, float *dw_r, float *dbias,
                             float *dw_in, float *dw_out, const Workspace &ws, cudaStream_t stream) {
    const int64_t T = dims.T;
    const int N = dims.num_experts, C = dims.capacity, d = dims.d_model, F = dims.d_ff;
    DeviceStatus *st = static_cast<DeviceStatus *>(ws.status);
    cudaError_t err = cudaMemsetAsync(ws.status, 0, sizeof(DeviceStatus), stream);
    // weight gradients of experts without kept tokens are zero; the GEMMs write the others
    if (err == cudaSuccess) err = cudaMemsetAsync(dw_in, 0, (size_t)N * F * d * sizeof(float), stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(dw_out, 0, (size_t)N * d * F * sizeof(float), stream);
    if (err != cudaSuccess) return err;
    if (T == 0) {
        err = cudaMemsetAsync(dw_r, 0, (size_t)N * d * sizeof(float), stream);
        if (err == cudaSuccess && dbias) err = cudaMemsetAsync(dbias, 0, (size_t)N * sizeof(float), stream);
        return err;
    }
    // 1. gate gradients, dE and the softmax backward
    launch_begin(K_BWD_TOKEN, stream);
    bwd_token_kernel<<<(unsigned)((T + kWarps - 1) / kWarps), kThreads, 0, stream>>>(
        dy, ws.ybuf, expert, slot, gate, ws.probs, counts, T, d, N, C, g_aux,
        static_cast<__nv_bfloat16 *>(ws.grad_e), ws.dh);
    err = cudaGetLastError();
    launch_end(stream);
    if (err != cudaSuccess) return err;
    // 2. dZ = (dE W_out) masked by the forward's ReLU: [N][C][F] bf16 (W_out read as it is stored)
    err = launch_ffn_tc_bwd_dz(dims, ws.grad_e, w_out, counts, ws.grad_z, ws.hidden, st, stream);
    if (err != cudaSuccess) return err;
    // 3. zero rows past each expert's kept tokens up to the next 64 (the dW GEMMs' last K block)
    launch_begin(K_BWD_ZERO_TAILS, stream);
    zero_tails_kernel<<<dim3((unsigned)N, 64), 256, 0, stream>>>(
        counts, C, d, F, static_cast<uint16_t *>(ws.grad_e), static_cast<uint16_t *>(ws.xbuf),
        static_cast<uint16_t *>(ws.hidden), static_cast<uint16_t *>(ws.grad_z));
    err = cudaGetLastError();
    launch_end(stream);
    if (err != cudaSuccess) return err;
    // 4. dx = dh W_r (all rows), then + dZ W_in for kept rows
    const bool simt_router = (dims.flags & SWITCH_FLAG_SIMT_ROUTER) != 0;
    const int Np = router_tc_np(N);
    const int64_t Tc = router_tc_chunk_tokens(T), chunks_tc = router_tc_chunks(T);
    if (simt_router) {
        const dim3 grid((unsigned)((d + kDxCol - 1) / kDxCol), (unsigned)((T + kDxTok - 1) / kDxTok));
        launch_begin(K_BWD_ROUTER_DX, stream);
        router_dx_kernel<<<grid, 256, 0, stream>>>(ws.dh, w_r, T, N, d, dx);
        err = cudaGetLastError();
        launch_end(stream);
        if (err != cudaSuccess) return err;
    } else {
        const int sms = device_sm_count();
        launch_begin(K_BWD_ROUTER_SPLIT, stream);
        router_dx_a_kernel<<<(unsigned)std::min<int64_t>((T * (Np / 8) + 255) / 256, 16 * sms), 256, 0, stream>>>(
            ws.dh, T, N, Np, static_cast<uint16_t *>(ws.rdx_a));
        err = cudaGetLastError();
        launch_end(stream);
        if (err != cudaSuccess) return err;
        launch_begin(K_BWD_ROUTER_SPLIT, stream);
        router_dx_b_kernel<<<(unsigned)(((int64_t)d * (Np / 8) + 255) / 256), 256, 0, stream>>>(
            w_r, N, d, Np, static_cast<uint16_t *>(ws.rdx_b), T, Tc, (int)chunks_tc, ws.chunk_counts);
        err = cudaGetLastError();
        launch_end(stream);
        if (err != cudaSuccess) return err;
        err = launch_router_tc_bwd_dx(ws.rdx_a, ws.rdx_b, ws.chunk_counts + chunks_tc, T, d, kDxPairs * Np, dx, st,
                                      stream);
        if (err != cudaSuccess) return err;
    }
    err = launch_ffn_tc_bwd_dx(dims, ws.grad_z, w_in, counts, ws.slot_token, dx, st, stream);
    if (err != cudaSuccess) return err;
    // 5. dW_out = dE^T H, dW_in = dZ^T x over each expert's kept tokens (token-major operands)
    err = launch_ffn_tc_bwd_dw(dims, ws.grad_e, ws.hidden, counts, d, F, dw_out, st, stream);
    if (err != cudaSuccess) return err;
    err = launch_ffn_tc_bwd_dw(dims, ws.grad_z, ws.xbuf, counts, F, d, dw_in, st, stream);
    if (err != cudaSuccess) return err;
    // 6. dW_r and d bias: chunk partials, then a fixed-order sum
    if (!simt_router) {
        launch_begin(K_BWD_ROUTER_SPLIT, stream);
        router_dw_a_kernel<<<dim3((unsigned)chunks_tc, (unsigned)((N + 31) / 32)), 256, 0, stream>>>(
            ws.dh, T, N, Tc, static_cast<uint16_t *>(ws.rdw_a), ws.db_part);
        err = cudaGetLastError();
        launch_end(stream);
        if (err != cudaSuccess) return err;
        err = launch_router_tc_bwd_dw(ws.rdw_a, x, ws.chunk_counts, (int)chunks_tc, 3 * N, (int)Tc, d, T,
                                      ws.dw_part, st, stream);
        if (err != cudaSuccess) return err;
        launch_begin(K_BWD_REDUCE, stream);
        router_dw_reduce_kernel<<<256, 256, 0, stream>>>(ws.dw_part, (int)chunks_tc, N, d, dw_r);
        err = cudaGetLastError();
        launch_end(stream);
        if (err == cudaSuccess && dbias) {
            launch_begin(K_BWD_REDUCE, stream);
            reduce_chunks_kernel<<<1, 256, 0, stream>>>(ws.db_part, (int)chunks_tc, (int64_t)N, dbias);
            err = cudaGetLastError();
            launch_end(stream);
        }
    } else {
        const int64_t chunks = router_dw_chunks(T);
        const int64_t chunk_tokens = (T + chunks - 1) / chunks;
        const dim3 grid((unsigned)((d + kDwCol - 1) / kDwCol), (unsigned)((N + kDwI - 1) / kDwI), (unsigned)chunks);
        launch_begin(K_BWD_ROUTER_DW, stream);
        router_dw_kernel<<<grid, 256, 0, stream>>>(ws.dh, static_cast<const uint16_t *>(x), T, N, d, chunk_tokens,
                                                   ws.dw_part, ws.db_part);
        err = cudaGetLastError();
        launch_end(stream);
        if (err != cudaSuccess) return err;
        launch_begin(K_BWD_REDUCE, stream);
        reduce_chunks_kernel<<<256, 256, 0, stream>>>(ws.dw_part, (int)chunks, (int64_t)N * d, dw_r);
        err = cudaGetLastError();
        launch_end(stream);
        if (err == cudaSuccess && dbias) {
            launch_begin(K_BWD_REDUCE, stream);
            reduce_chunks_kernel<<<1, 256, 0, stream>>>(ws.db_part, (int)chunks, (int64_t)N, dbias);
            err = cudaGetLastError();
            launch_end(stream);
        }
    }
    return err;
}

}  // namespace switchmoe
