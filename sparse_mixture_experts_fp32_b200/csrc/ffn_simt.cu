// Expert FFN on CUDA cores: a grouped SIMT GEMM over the kept rows of every
// expert.  It is the float32 path (any d_model, d_ff) and, for bfloat16, a
// diagnostic alternative to the tensor-core kernel selected with
// SWITCH_FLAG_SIMT_FFN.
//
//   H[i, s, :]    = ReLU(xbuf[i, s, :] . W_in[i]^T)     s < min(counts[i], C)
//   ybuf[i, s, :] = H[i, s, :] . W_out[i]^T              (float32)
// H is stored in the activation type (bfloat16 rounding between the two
// products for bf16, exactly as the tensor-core path does).
#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr int BM = 64, BN = 64, KC = 16, kThreads = 256;

// D[e] (rows < kept_e) = act(A[e] . B[e]^T); A [E][C][K], B [E][Nout][K], D [E][C][Nout].
template <typename T, typename TO, bool RELU>
__global__ void __launch_bounds__(kThreads) grouped_gemm_simt(const T *__restrict__ A, const T *__restrict__ B,
                                                              TO *__restrict__ D, const int32_t *__restrict__ counts,
                                                              int C, int K, int Nout) {
    __shared__ float as[KC][BM + 4];
    __shared__ float bs[KC][BN + 4];
    const int e = blockIdx.z;
    const int kept = min(counts[e], C);
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    if (m0 >= kept) return;
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const T *Ae = A + (int64_t)e * C * K;
    const T *Be = B + (int64_t)e * Nout * K;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += KC) {
        for (int i = tid; i < BM * KC; i += kThreads) {
            const int r = i / KC, kk = i % KC;
            const int m = m0 + r, k = k0 + kk;
            as[kk][r] = (m < kept && k < K) ? Elem<T>::load(Ae, (int64_t)m * K + k) : 0.f;
        }
        for (int i = tid; i < BN * KC; i += kThreads) {
            const int r = i / KC, kk = i % KC;
            const int n = n0 + r, k = k0 + kk;
            bs[kk][r] = (n < Nout && k < K) ? Elem<T>::load(Be, (int64_t)n * K + k) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < KC; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = as[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = bs[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    TO *De = D + (int64_t)e * C * Nout;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty + 16 * i;
        if (m >= kept) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx + 16 * j;
            if (n < Nout) Elem<TO>::store(De, (int64_t)m * Nout + n, RELU ? fmaxf(acc[i][j], 0.f) : acc[i][j]);
        }
    }
}

template <typename T>
cudaError_t run(const switch_dims_t &dims, const T *xbuf, const T *w_in, const T *w_out, const int32_t *counts,
                float *ybuf, T *hidden, cudaStream_t stream) {
    const int N = dims.num_experts, C = dims.capacity, d = dims.d_model, F = dims.d_ff;
    dim3 g1((F + BN - 1) / BN, (C + BM - 1) / BM, N);
    launch_begin(K_FFN_SIMT_GEMM1, stream);
    grouped_gemm_simt<T, T, true><<<g1, kThreads, 0, stream>>>(xbuf, w_in, hidden, counts, C, d, F);
    cudaError_t err = cudaGetLastError();
    launch_end(stream);
    if (err != cudaSuccess) return err;
    dim3 g2((d + BN - 1) / BN, (C + BM - 1) / BM, N);
    launch_begin(K_FFN_SIMT_GEMM2, stream);
    grouped_gemm_simt<T, float, false><<<g2, kThreads, 0, stream>>>(hidden, w_out, ybuf, counts, C, F, d);
    err = cudaGetLastError();
    launch_end(stream);
    return err;
}

}  // namespace

cudaError_t launch_ffn_simt(const switch_dims_t &dims, const void *xbuf, const void *w_in, const void *w_out,
                            const int32_t *counts, float *ybuf, const Workspace &ws, cudaStream_t stream) {
    if (dims.dtype == SWITCH_BF16)
        return run<__nv_bfloat16>(dims, static_cast<const __nv_bfloat16 *>(xbuf),
                                  static_cast<const __nv_bfloat16 *>(w_in), static_cast<const __nv_bfloat16 *>(w_out),
                                  counts, ybuf, static_cast<__nv_bfloat16 *>(ws.hidden),
                                  stream);
    return run<float>(dims, static_cast<const float *>(xbuf), static_cast<const float *>(w_in),
                      static_cast<const float *>(w_out), counts, ybuf,
                      static_cast<float *>(ws.hidden), stream);
}

}  // namespace switchmoe
