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
// Both are pure HBM streams: by default one warp per row with 16-byte (or
// 4-byte) vector accesses, all of a lane's loads issued before its stores.
// With SWITCH_FLAG_STAGED_MOVES, rows up to ~6 KB move through shared memory
// by bulk copies (the TMA engine) instead; on B200 that measured 4-6 % slower
// on the Switch-Large shape (dispatch 98.9 against 94.7 us, combine 194.5
// against 183.3 us), so the vector kernels stay the default.
#include <algorithm>

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

// ---------------------------------------------------------------------------
// Bulk-copy (TMA engine) staged forms, for rows whose byte size is a multiple
// of 16.  Each warp streams rows through its own ring of kRing row buffers in
// shared memory, in rounds: lane 0 issues the round's cp.async.bulk row loads
// (each completing on its own mbarrier, with a per-buffer phase bit), then per
// row waits for the load, (combine: all lanes scale the row by its gate in
// shared memory, or write zeros for a dropped token), and issues one
// cp.async.bulk store of the whole row; before the next round reuses the
// buffers it waits until the stores have read them.  The waits are bounded
// (about a second); these entry points have no status word, so a wait that
// gives up ends the warp's work after a second bounded wait for its loads.
// ---------------------------------------------------------------------------
constexpr int kRingWarps = 4;
constexpr int kRing = 4;
// Shared memory of one ring block at most (rows up to ~6 KB; longer rows use the LSU kernels).
constexpr size_t kRingSmemLimit = 100 * 1024;

__host__ __device__ constexpr int ring_stage_bytes(int row_bytes) { return (row_bytes + 127) / 128 * 128; }
__host__ __device__ constexpr size_t ring_warp_bytes(int row_bytes) {
    return 128 + (size_t)kRing * ring_stage_bytes(row_bytes);  // barriers (padded to 128), then the buffers
}

__device__ __forceinline__ bool ring_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_wait(bar, parity, nullptr, 0)) return true;
    mbar_wait(bar, parity, nullptr, 0);  // the load may still land: wait once more before giving up
    return false;
}

// xbuf[e, s] = x[slot_token[e*C+s]] for the kept slots of every expert.
__global__ void __launch_bounds__(32 * kRingWarps) dispatch_bulk_kernel(const uint8_t *__restrict__ x,
                                                                       const int32_t *__restrict__ slot_token,
                                                                       const int32_t *__restrict__ counts, int N,
                                                                       int C, int row_bytes,
                                                                       uint8_t *__restrict__ xbuf) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *base = smem_raw + (size_t)warp * ring_warp_bytes(row_bytes);
    uint64_t *bar = reinterpret_cast<uint64_t *>(base);
    uint8_t *buf = base + 128;
    const int stage = ring_stage_bytes(row_bytes);
    if (lane != 0) return;  // one thread per warp drives the copy engine
    for (int k = 0; k < kRing; ++k) mbar_init(&bar[k], 1);
    fence_barrier_init();
    const int64_t rows = (int64_t)N * C;
    const int64_t nwarps = (int64_t)gridDim.x * kRingWarps;
    uint32_t phases = 0;
    bool ok = true;
    for (int64_t first = (int64_t)blockIdx.x * kRingWarps + warp; ok && first < rows; first += nwarps * kRing) {
        int64_t dst[kRing];
        for (int k = 0; k < kRing; ++k) {
            const int64_t row = first + (int64_t)k * nwarps;
            dst[k] = -1;
            if (row >= rows) continue;
            const int e = (int)(row / C), s = (int)(row % C);
            if (s >= min(counts[e], C)) continue;
            const int64_t t = slot_token[row];
            mbar_arrive_expect_tx(&bar[k], (uint32_t)row_bytes);
            bulk_load(buf + (size_t)k * stage, x + t * row_bytes, (uint32_t)row_bytes, &bar[k]);
            dst[k] = row;
        }
        for (int k = 0; k < kRing; ++k) {
            if (dst[k] < 0) continue;
            const bool landed = ring_wait(&bar[k], (phases >> k) & 1u);
            phases ^= 1u << k;
            if (!landed) {
                ok = false;
                continue;
            }
            bulk_store(xbuf + dst[k] * row_bytes, buf + (size_t)k * stage, (uint32_t)row_bytes);
            bulk_commit();
        }
        bulk_wait_read_all();  // the stores have read the buffers: the next round may refill them
    }
    bulk_wait_all();
}

// y[t] = gate[t] * ybuf[expert[t], slot[t]] (float32, one rounding), or a zero row.
__global__ void __launch_bounds__(32 * kRingWarps) combine_bulk_kernel(const float *__restrict__ ybuf,
                                                                      const int32_t *__restrict__ expert,
                                                                      const int32_t *__restrict__ slot,
                                                                      const float *__restrict__ gate, int64_t T,
                                                                      int C, int d, float *__restrict__ y) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_bytes = d * 4;
    uint8_t *base = smem_raw + (size_t)warp * ring_warp_bytes(row_bytes);
    uint64_t *bar = reinterpret_cast<uint64_t *>(base);
    uint8_t *buf = base + 128;
    const int stage = ring_stage_bytes(row_bytes);
    if (lane == 0) {
        for (int k = 0; k < kRing; ++k) mbar_init(&bar[k], 1);
        fence_barrier_init();
    }
    __syncwarp();
    const int64_t nwarps = (int64_t)gridDim.x * kRingWarps;
    const int words = d / 4;
    uint32_t phases = 0;
    bool ok = true;
    for (int64_t first = (int64_t)blockIdx.x * kRingWarps + warp; ok && first < T; first += nwarps * kRing) {
        // lane k < kRing reads row k's slot; lane 0 starts the kept rows' loads
        int my_slot = -2;  // -2: past T
        const int64_t my_t = first + (int64_t)lane * nwarps;
        if (lane < kRing && my_t < T) my_slot = slot[my_t];
        int s_of[kRing];
#pragma unroll
        for (int k = 0; k < kRing; ++k) s_of[k] = __shfl_sync(0xffffffffu, my_slot, k);
        if (lane == 0) {
#pragma unroll
            for (int k = 0; k < kRing; ++k) {
                if (s_of[k] < 0) continue;
                const int64_t t = first + (int64_t)k * nwarps;
                mbar_arrive_expect_tx(&bar[k], (uint32_t)row_bytes);
                bulk_load(buf + (size_t)k * stage, ybuf + ((int64_t)expert[t] * C + s_of[k]) * d,
                          (uint32_t)row_bytes, &bar[k]);
            }
        }
        for (int k = 0; k < kRing; ++k) {
            if (s_of[k] == -2) break;
            const int64_t t = first + (int64_t)k * nwarps;
            float4 *row = reinterpret_cast<float4 *>(buf + (size_t)k * stage);
            if (s_of[k] >= 0) {
                const bool landed = ring_wait(&bar[k], (phases >> k) & 1u);
                phases ^= 1u << k;
                if (!landed) {
                    ok = false;
                    continue;
                }
                const float g = gate[t];
                for (int w = lane; w < words; w += 32) {
                    const float4 v = row[w];
                    row[w] = make_float4(g * v.x, g * v.y, g * v.z, g * v.w);
                }
            } else {
                for (int w = lane; w < words; w += 32) row[w] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            fence_proxy_async_shared();  // the lanes' shared-memory writes, before the bulk store reads them
            __syncwarp();
            if (lane == 0) {
                bulk_store(y + t * d, row, (uint32_t)row_bytes);
                bulk_commit();
            }
        }
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
    }
    if (lane == 0) bulk_wait_all();
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
    const size_t ring_smem = kRingWarps * ring_warp_bytes((int)row_bytes);
    launch_begin(K_DISPATCH, stream);
    if ((dims.flags & SWITCH_FLAG_STAGED_MOVES) && row_bytes % 16 == 0 && ring_smem <= kRingSmemLimit) {
        cudaError_t err = cudaFuncSetAttribute(dispatch_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)ring_smem);
        if (err != cudaSuccess) {
            launch_end(stream);
            return err;
        }
        const int64_t warps = (rows + kRing - 1) / kRing;
        const unsigned g = (unsigned)std::max<int64_t>(
            1, std::min<int64_t>((warps + kRingWarps - 1) / kRingWarps, (int64_t)device_sm_count() * 8));
        dispatch_bulk_kernel<<<g, 32 * kRingWarps, ring_smem, stream>>>(static_cast<const uint8_t *>(x), slot_token,
                                                                         counts, N, C, (int)row_bytes,
                                                                         static_cast<uint8_t *>(xbuf));
    } else if (row_bytes % 16 == 0)
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
    const size_t ring_smem = kRingWarps * ring_warp_bytes(dims.d_model * 4);
    launch_begin(K_COMBINE, stream);
    if ((dims.flags & SWITCH_FLAG_STAGED_MOVES) && dims.d_model % 4 == 0 && ring_smem <= kRingSmemLimit) {
        cudaError_t err = cudaFuncSetAttribute(combine_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)ring_smem);
        if (err != cudaSuccess) {
            launch_end(stream);
            return err;
        }
        const int64_t warps = (T + kRing - 1) / kRing;
        const unsigned g = (unsigned)std::max<int64_t>(
            1, std::min<int64_t>((warps + kRingWarps - 1) / kRingWarps, (int64_t)device_sm_count() * 8));
        combine_bulk_kernel<<<g, 32 * kRingWarps, ring_smem, stream>>>(ybuf, expert, slot, gate, T, dims.capacity,
                                                                        dims.d_model, y);
    } else if (dims.d_model % 4 == 0)
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
