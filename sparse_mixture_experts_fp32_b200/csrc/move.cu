// Dispatch (gather kept tokens into per-expert buffers) and combine (gated
// scatter back to token order), sm_100a.
//
// Dispatch: xbuf[i, s, :] = x[slot_token[i*C+s], :] for s < min(counts[i], C)
//   (Incredible.AI "MoE Layer", x_flat[expert_indices]; kasblo section
//   "tokenをExpertへ送って戻すforward pass": on one device the exchange is a
//   gather/scatter in memory).
// Combine:  y[t, :] = gate[t] * ybuf[expert[t], slot[t], :] in float32, or
//   0 for a dropped token (llm-papers-study "精读 06 | Switch Transformers" §3.2,
//   y = p_i*(x) E_i*(x); §3.4, dropped tokens skip the expert).
//
// Both are pure HBM streams: one warp per row, 16-byte vector accesses, all of
// a lane's loads issued before its stores.
#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = kThreads / 32;
constexpr int kUnroll = 4;

// Row copy of `words` 16-byte words by one warp: kUnroll loads per lane are
// in flight before the first store.
__device__ __forceinline__ void warp_copy_row16(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int words) {
    const int lane = threadIdx.x & 31;
    for (int w0 = 0; w0 < words; w0 += 32 * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int w = w0 + lane + 32 * u;
            if (w < words) v[u] = __ldcs(src + w);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int w = w0 + lane + 32 * u;
            if (w < words) dst[w] = v[u];
        }
    }
}

__global__ void __launch_bounds__(kThreads) dispatch_kernel16(const uint4 *__restrict__ x,
                                                             const int32_t *__restrict__ slot_token,
                                                             const int32_t *__restrict__ counts, int N, int C,
                                                             int words, uint4 *__restrict__ xbuf) {
    const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (row >= (int64_t)N * C) return;
    const int e = (int)(row / C), s = (int)(row % C);
    if (s >= min(counts[e], C)) return;
    const int64_t t = slot_token[row];
    warp_copy_row16(x + t * words, xbuf + row * words, words);
}

// Rows whose byte size is not a multiple of 16 (float32 with d % 4 != 0).
__global__ void __launch_bounds__(kThreads) dispatch_kernel4(const uint32_t *__restrict__ x,
                                                            const int32_t *__restrict__ slot_token,
                                                            const int32_t *__restrict__ counts, int N, int C,
                                                            int words, uint32_t *__restrict__ xbuf) {
    const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (row >= (int64_t)N * C) return;
    const int e = (int)(row / C), s = (int)(row % C);
    if (s >= min(counts[e], C)) return;
    const int64_t t = slot_token[row];
    for (int w = threadIdx.x & 31; w < words; w += 32) xbuf[row * words + w] = x[t * words + w];
}

// y[t] = gate[t] * ybuf[expert[t], slot[t]] (float32, one rounding), or 0.
__global__ void __launch_bounds__(kThreads) combine_kernel_vec(const float4 *__restrict__ ybuf,
                                                              const int32_t *__restrict__ expert,
                                                              const int32_t *__restrict__ slot,
                                                              const float *__restrict__ gate, int64_t T, int C,
                                                              int words, float4 *__restrict__ y) {
    const int64_t t = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (t >= T) return;
    const int lane = threadIdx.x & 31;
    const int s = slot[t];
    float4 *dst = y + t * words;
    if (s < 0) {
        for (int w = lane; w < words; w += 32) __stcs(dst + w, make_float4(0.f, 0.f, 0.f, 0.f));
        return;
    }
    const float g = gate[t];
    const float4 *src = ybuf + ((int64_t)expert[t] * C + s) * words;
    for (int w0 = 0; w0 < words; w0 += 32 * kUnroll) {
        float4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int w = w0 + lane + 32 * u;
            if (w < words) v[u] = __ldcs(src + w);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int w = w0 + lane + 32 * u;
            if (w < words) __stcs(dst + w, make_float4(g * v[u].x, g * v[u].y, g * v[u].z, g * v[u].w));
        }
    }
}

// Rows of d % 4 != 0 floats.
__global__ void __launch_bounds__(kThreads) combine_kernel_scalar(const float *__restrict__ ybuf,
                                                                 const int32_t *__restrict__ expert,
                                                                 const int32_t *__restrict__ slot,
                                                                 const float *__restrict__ gate, int64_t T, int C,
                                                                 int d, float *__restrict__ y) {
    const int64_t t = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (t >= T) return;
    const int lane = threadIdx.x & 31;
    const int s = slot[t];
    float *dst = y + t * d;
    if (s < 0) {
        for (int k = lane; k < d; k += 32) dst[k] = 0.f;
        return;
    }
    const float g = gate[t];
    const float *src = ybuf + ((int64_t)expert[t] * C + s) * d;
    for (int k = lane; k < d; k += 32) dst[k] = g * src[k];
}

// Top-2: y[t] = g0 * ybuf[e0, s0] + g1 * ybuf[e1, s1] over the kept choices,
// the first choice's product first (float32; 0 when both were dropped).
template <bool VEC>
__global__ void __launch_bounds__(kThreads) combine_top2_kernel(const float *__restrict__ ybuf,
                                                               const int32_t *__restrict__ expert2,
                                                               const int32_t *__restrict__ slot2,
                                                               const float *__restrict__ gate2, int64_t T, int C,
                                                               int d, float *__restrict__ y) {
    const int64_t t = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
    if (t >= T) return;
    const int lane = threadIdx.x & 31;
    const int s0 = slot2[2 * t], s1 = slot2[2 * t + 1];
    const float g0 = s0 >= 0 ? gate2[2 * t] : 0.f, g1 = s1 >= 0 ? gate2[2 * t + 1] : 0.f;
    const float *src0 = s0 >= 0 ? ybuf + ((int64_t)expert2[2 * t] * C + s0) * d : nullptr;
    const float *src1 = s1 >= 0 ? ybuf + ((int64_t)expert2[2 * t + 1] * C + s1) * d : nullptr;
    if (VEC) {
        const int words = d / 4;
        float4 *dst = reinterpret_cast<float4 *>(y + t * d);
        for (int w = lane; w < words; w += 32) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
            if (src0) a = __ldcs(reinterpret_cast<const float4 *>(src0) + w);
            if (src1) b = __ldcs(reinterpret_cast<const float4 *>(src1) + w);
            float4 o;
            o.x = __fadd_rn(__fmul_rn(g0, a.x), __fmul_rn(g1, b.x));
            o.y = __fadd_rn(__fmul_rn(g0, a.y), __fmul_rn(g1, b.y));
            o.z = __fadd_rn(__fmul_rn(g0, a.z), __fmul_rn(g1, b.z));
            o.w = __fadd_rn(__fmul_rn(g0, a.w), __fmul_rn(g1, b.w));
            __stcs(dst + w, o);
        }
    } else {
        float *dst = y + t * d;
        for (int k = lane; k < d; k += 32) {
            const float a = src0 ? src0[k] : 0.f, b = src1 ? src1[k] : 0.f;
            dst[k] = __fadd_rn(__fmul_rn(g0, a), __fmul_rn(g1, b));
        }
    }
}

}  // namespace

cudaError_t launch_combine_top2(const switch_dims_t &dims, const float *ybuf, const int32_t *expert,
                                const int32_t *slot, const float *gate, float *y, cudaStream_t stream) {
    const int64_t T = dims.T;
    if (T == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((T + kRowsPerBlock - 1) / kRowsPerBlock);
    launch_begin(K_COMBINE_TOP2, stream);
    if (dims.d_model % 4 == 0)
        combine_top2_kernel<true><<<grid, kThreads, 0, stream>>>(ybuf, expert, slot, gate, T, dims.capacity,
                                                                 dims.d_model, y);
    else
        combine_top2_kernel<false><<<grid, kThreads, 0, stream>>>(ybuf, expert, slot, gate, T, dims.capacity,
                                                                  dims.d_model, y);
    cudaError_t err = cudaGetLastError();
    launch_end(stream);
    return err;
}

cudaError_t launch_dispatch(const switch_dims_t &dims, const void *x, const int32_t *slot_token,
                            const int32_t *counts, void *xbuf, cudaStream_t stream) {
    const int N = dims.num_experts, C = dims.capacity;
    const int64_t rows = (int64_t)N * C;
    const int64_t row_bytes = (int64_t)dims.d_model * (dims.dtype == SWITCH_BF16 ? 2 : 4);
    const unsigned grid = (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
    if (dims.T == 0) return cudaSuccess;
    launch_begin(K_DISPATCH, stream);
    if (row_bytes % 16 == 0)
        dispatch_kernel16<<<grid, kThreads, 0, stream>>>(static_cast<const uint4 *>(x), slot_token, counts, N, C,
                                                         (int)(row_bytes / 16), static_cast<uint4 *>(xbuf));
    else
        dispatch_kernel4<<<grid, kThreads, 0, stream>>>(static_cast<const uint32_t *>(x), slot_token, counts, N, C,
                                                        (int)(row_bytes / 4), static_cast<uint32_t *>(xbuf));
    cudaError_t err = cudaGetLastError();
    launch_end(stream);
    return err;
}

cudaError_t launch_combine(const switch_dims_t &dims, const float *ybuf, const int32_t *expert, const int32_t *slot,
                           const float *gate, float *y, cudaStream_t stream) {
    const int64_t T = dims.T;
    if (T == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((T + kRowsPerBlock - 1) / kRowsPerBlock);
    launch_begin(K_COMBINE, stream);
    if (dims.d_model % 4 == 0)
        combine_kernel_vec<<<grid, kThreads, 0, stream>>>(reinterpret_cast<const float4 *>(ybuf), expert, slot, gate,
                                                          T, dims.capacity, dims.d_model / 4,
                                                          reinterpret_cast<float4 *>(y));
    else
        combine_kernel_scalar<<<grid, kThreads, 0, stream>>>(ybuf, expert, slot, gate, T, dims.capacity,
                                                             dims.d_model, y);
    cudaError_t err = cudaGetLastError();
    launch_end(stream);
    return err;
}

}  // namespace switchmoe
