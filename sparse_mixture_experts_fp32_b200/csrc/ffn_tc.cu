// Expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
//   GEMM1: H[i, s, :]    = ReLU(xbuf[i, s, :] . W_in[i]^T)    (K = d, Nout = F)
//   GEMM2: ybuf[i, s, :] = H[i, s, :] . W_out[i]^T            (K = F, Nout = d)
// over the kept rows s < min(counts[i], C) of every expert i.  Both GEMMs
// are the same grouped "A . B^T" kernel with both operands K-major (the
// nn.Linear weight layout), bf16 inputs and fp32 accumulation in tensor
// memory.  Epilogues (rows below the expert's kept count only):
//   kEpiHiddenRelu   ReLU, round to bf16, store H[i, s, :]
//   kEpiExpertOut    store the fp32 accumulator as ybuf[i, s, :]
//   kEpiGatedScatter y[t, :] = gate[t] * acc in fp32, t = slot_token[i*C+s]
//                    (the combine step fused into GEMM2: the expert output
//                    goes straight to token order, scaled by its gate, and
//                    is rounded once, to float32)
// (Expert FFN and y = p_i* E_i*(x): llm-papers-study "精读 06 | Switch
// Transformers" §3.2; bfloat16 experts with float32 accumulation: kasblo
// section "Routerだけfloat32で計算するSelective Precision".)
//
// Kernel structure (one CTA per SM, persistent over a tile list that every
// CTA derives on the device from `counts`, so no host synchronisation):
//   warp 0      one lane issues TMA loads of 128 x 64 A and BN x 64 B tiles
//               (128-byte swizzle) into a STAGES-deep shared-memory ring
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN,
//               K=16) into one of two TMEM accumulators and commits to
//               mbarriers that free ring slots / publish the accumulator
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes (one thread per
//               row), then one of the epilogues above with 16-byte
//               stores; then release the accumulator
// Every mbarrier wait is bounded (about 1 s); on a timeout the kernel records
// SWITCH_ERR_DEVICE_TIMEOUT in the status word, waits (bounded) for its own
// TMA loads and MMAs in flight, frees TMEM and returns.
#include <cuda.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace switchmoe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kEpilogueThreads = 128;

template <int BN, int STAGES>
struct TcLayout {
    static constexpr size_t a_bytes = (size_t)BM * BK * 2;
    static constexpr size_t b_bytes = (size_t)BN * BK * 2;
    static constexpr size_t ring = STAGES * (a_bytes + b_bytes);
    static constexpr size_t barriers = (2 * STAGES + 2 + 2 + 1) * 8 + 16;
    static size_t bytes(int experts) { return 1024 + ring + barriers + (size_t)(experts + 1) * 4; }
};

__device__ __forceinline__ void locate_tile(const int32_t *tile_start, int E, int n_tiles_n, int tile, int &e,
                                            int &m, int &n) {
    int lo = 0, hi = E - 1;  // largest e with tile_start[e] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    e = lo;
    const int local = tile - tile_start[e];
    m = local / n_tiles_n;
    n = local % n_tiles_n;
}

enum Epilogue {
    kEpiHiddenRelu = 0,    // H = bf16(ReLU(acc))
    kEpiExpertOut = 1,     // fp32 rows out[e * out_rows + row]
    kEpiGatedScatter = 2,  // y[slot_token] = gate * acc (with `add`: += )
    kEpiReluGrad = 3,      // backward: dZ = bf16(acc) where the forward's H > 0, else 0
    kEpiScatterAdd = 4,    // backward: dx[slot_token] += acc
    kEpiWeightGrad = 5     // backward weight gradients: fp32 rows out[e * out_rows + row] by TMA box stores
};

// Epilogue for one thread = one accumulator row (`row` of expert e's rows),
// BN columns starting at column tile n: tcgen05.ld 32 columns at a time, then
// the epilogue selected by EPI, for rows below the kept count only.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_rows(uint32_t t_row, int e, int row, int kept, int C, int n, int Nout,
                                              void *__restrict__ out, const int32_t *__restrict__ slot_token,
                                              const float *__restrict__ gate) {
    const bool row_ok = row < kept;
    // destination row of this thread (a token row for the gated scatter)
    int64_t out_row = (int64_t)e * C + row;
    float g = 1.f;
    if (EPI == kEpiGatedScatter && row_ok) {
        out_row = slot_token[(int64_t)e * C + row];
        g = gate[out_row];
    }
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + (uint32_t)c, r);
        tmem_ld_wait();
        const int col0 = n * BN + c;
        if (row_ok && col0 < Nout) {
            if (EPI == kEpiHiddenRelu) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + out_row * Nout + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = fmaxf(__uint_as_float(r[8 * q + i]), 0.f);
                    dst[q] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                        pack_bf16x2(v[6], v[7]));
                }
            } else {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + out_row * Nout + col0);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    dst[q] = make_float4(g * __uint_as_float(r[4 * q + 0]), g * __uint_as_float(r[4 * q + 1]),
                                         g * __uint_as_float(r[4 * q + 2]), g * __uint_as_float(r[4 * q + 3]));
            }
        }
    }
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    tc_grouped_gemm(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    void *__restrict__ out, const int32_t *__restrict__ counts, int E, int C, int K, int Nout,
                    const int32_t *__restrict__ slot_token, const float *__restrict__ gate, DeviceStatus *status) {
    using L = TcLayout<BN, STAGES>;
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
    int32_t *tile_start = reinterpret_cast<int32_t *>(tmem_holder + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles_n = (Nout + BN - 1) / BN;
    const int k_blocks = K / BK;
    constexpr uint32_t kTmemCols = 2 * BN;

    // Tile list: expert e owns tiles [tile_start[e], tile_start[e+1]), laid
    // out m-major with the BN-wide column tiles innermost.
    if (warp == 0) {
        int kept_of[8];  // E <= 256: every count is loaded before the scan starts
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = 32 * j + lane;
            kept_of[j] = e < E ? min(counts[e], C) : 0;
        }
        int running = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e0 = 32 * j;
            if (e0 >= E) break;
            const int e = e0 + lane;
            const int kept = kept_of[j];
            const int mine = (kept + BM - 1) / BM * n_tiles_n;
            int incl = mine;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += u;
            }
            if (e < E) tile_start[e] = running + incl - mine;
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) tile_start[E] = running;
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            for (int a = 0; a < 2; ++a) {
                mbar_init(&acc_full[a], 1);
                mbar_init(&acc_empty[a], kEpilogueThreads);
            }
            mbar_init(drain, 1);
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int total_tiles = tile_start[E];

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmap_a);
            prefetch_tmap(&tmap_b);
            uint32_t issued = 0, parity_of = 0;  // per ring slot: load issued, parity of its phase
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
                int e, m, n;
                locate_tile(tile_start, E, n_tiles_n, tile, e, m, n);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, status, 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)(L::a_bytes + L::b_bytes));
                    tma_load_3d(sA + stage * L::a_bytes, &tmap_a, &full[stage], kb * BK, m * BM, e);
                    tma_load_3d(sB + stage * L::b_bytes, &tmap_b, &full[stage], kb * BK, n * BN, e);
                    issued |= 1u << stage;
                    parity_of = (parity_of & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Wind-down: the last load into every slot must have landed
            // before the CTA may exit (already true unless a wait timed out).
            for (int s = 0; s < STAGES; ++s)
                if (issued & (1u << s)) mbar_wait(&full[s], (parity_of >> s) & 1u, status, 6);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, status, 2)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, status, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = smem_desc_sw128(sA + stage * L::a_bytes);
                    const uint64_t b_desc = smem_desc_sw128(sB + stage * L::b_bytes);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // advance 16 bf16 = 32 bytes along K inside the swizzled row
                        tc_mma_bf16(d_tmem, a_desc + (uint64_t)(2 * k), b_desc + (uint64_t)(2 * k), idesc,
                                    (kb | k) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&acc_full[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // Wind-down: every MMA issued above has completed once `drain` flips.
            tc_commit(drain);
            mbar_wait(drain, 0, status, 4);
        }
    } else {
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter+32) belong to this warp
        const int row_in_tile = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            int e, m, n;
            locate_tile(tile_start, E, n_tiles_n, tile, e, m, n);
            if (!mbar_wait(&acc_full[acc], acc_phase, status, 5)) break;
            tc_fence_after();
            const int row = m * BM + row_in_tile;
            epilogue_rows<BN, EPI>(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN), e, row,
                                   min(counts[e], C), C, n, Nout, out, slot_token, gate);
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Epilogue through the async proxy, one warp = 32 consecutive rows
// (row_base .. row_base + 31, thread = row), `stage` = this warp's shared
// staging buffer (4.5 KB, 1024-byte aligned):
//   kEpiHiddenRelu  64 columns at a time: ReLU + bf16 into a 32 x 128-byte
//                   box in the 128-byte swizzled layout (conflict-free
//                   writes), then one TMA tensor store of the box into H.
//                   Rows in [kept, C) receive values of rows that are never
//                   read downstream; rows >= C are clipped by the tensor map.
//   kEpiExpertOut / kEpiGatedScatter / kEpiScatterAdd  32 fp32 columns at a
//                   time: each thread writes its row (144-byte pitch:
//                   conflict-free), then the warp stores the block with
//                   row-coalesced 16-byte stores (with `add`: 16-byte fp32
//                   reductions onto the destination), no bulk-copy waits.
//   kEpiWeightGrad  32 fp32 columns at a time into a 32 x 128-byte swizzled
//                   box, one TMA tensor store per box into the fixed-row
//                   output [E][out_rows][Nout] (rows past out_rows clipped
//                   by the tensor map).
template <int BN, int EPI>
__device__ __forceinline__ int epilogue_async(uint32_t t_row, int e, int row_base, int kept, int C, int n, int Nout,
                                               void *__restrict__ out, const void *tmap_out,
                                               const int32_t *__restrict__ slot_token,
                                               const float *__restrict__ gate, uint8_t *stage, bool add = false,
                                               int out_rows = 0, const uint16_t *__restrict__ mask_h = nullptr,
                                               int cols = BN) {
    // `cols` (a multiple of 64, at most BN): the tile's width; column tile n starts at n * cols
    const int lane = threadIdx.x & 31;
    const int row = row_base + lane;
    const bool row_ok = row < kept;
    int groups = 0;  // bulk groups committed by lane 0 (the box-store epilogues)
    if (EPI == kEpiHiddenRelu || EPI == kEpiReluGrad) {
        const bool any_row = row_base < kept;
#pragma unroll 1
        for (int c = 0; c < cols; c += 64) {
            uint32_t r0[32], r1[32];
            tmem_ld_32x32b_x32(t_row + (uint32_t)c, r0);
            tmem_ld_32x32b_x32(t_row + (uint32_t)(c + 32), r1);
            tmem_ld_wait();
            if (lane == 0) bulk_wait_read_all();  // the previous box has left the buffer
            __syncwarp();
            uint8_t *rowp = stage + lane * 128;
            uint4 hm[8];  // kEpiReluGrad: the forward's H at these 64 columns (its sign is the ReLU mask)
            if (EPI == kEpiReluGrad) {
                const int col = n * cols + c;
                const bool ld = row_ok && col < Nout;
                const uint4 *hp = reinterpret_cast<const uint4 *>(mask_h + ((int64_t)e * C + row) * Nout + col);
#pragma unroll
                for (int q = 0; q < 8; ++q) hm[q] = ld ? __ldg(hp + q) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t *src = q < 4 ? &r0[8 * q] : &r1[8 * (q - 4)];
                float v[8];
                if (EPI == kEpiReluGrad) {
                    const uint32_t w[4] = {hm[q].x, hm[q].y, hm[q].z, hm[q].w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t hb = (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xffffu);
                        // H = bf16(ReLU(z)) > 0 exactly where z > 0 (but for z below the smallest bf16 subnormal)
                        const bool pos = hb != 0u && (hb & 0x8000u) == 0u;
                        v[i] = pos ? __uint_as_float(src[i]) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = fmaxf(__uint_as_float(src[i]), 0.f);
                }
                *reinterpret_cast<uint4 *>(rowp + ((q ^ (lane & 7)) << 4)) =
                    make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                               pack_bf16x2(v[6], v[7]));
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0 && any_row && n * cols + c < Nout) {
                tma_store_3d(tmap_out, stage, n * cols + c, row_base, e);
                bulk_commit();
                ++groups;
            }
        }
        if (lane == 0) bulk_wait_read_all();
    } else if (EPI == kEpiWeightGrad) {
        // the warp's 32 rows x 32 fp32 columns per step, 128-byte-swizzled in its staging buffer
        // (conflict-free writes), then one TMA tensor store of the 32 x 32 box
        const bool any_row = row_base < kept;
#pragma unroll 1
        for (int c = 0; c < cols; c += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + (uint32_t)c, r);
            tmem_ld_wait();
            if (lane == 0) bulk_wait_read_all();  // the previous box has left the buffer
            __syncwarp();
            uint8_t *rowp = stage + lane * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4 *>(rowp + ((q ^ (lane & 7)) << 4)) =
                    make_uint4(r[4 * q + 0], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0 && any_row && n * cols + c < Nout) {
                tma_store_3d(tmap_out, stage, n * cols + c, row_base, e);
                bulk_commit();
            }
        }
        if (lane == 0) bulk_wait_read_all();
    } else {
        // 32 fp32 columns at a time: each lane writes its row (scaled by its gate) into the
        // staging buffer (144-byte pitch: conflict-free), then the warp stores the 32 x 128-byte
        // block row-coalesced: 8 lanes per row, 4 rows per instruction (float4 stores, or float4
        // reductions with `add`).
        float g = 1.f;
        int32_t out_row = -1;  // this lane's destination row, -1 past the kept rows
        if (row_ok) {
            out_row = (int32_t)((int64_t)e * (out_rows > 0 ? out_rows : C) + row);
            if (EPI == kEpiGatedScatter || EPI == kEpiScatterAdd) {
                out_row = slot_token[(int64_t)e * C + row];
                if (EPI == kEpiGatedScatter) g = gate[out_row];
            }
        }
        if (EPI == kEpiScatterAdd) add = true;
        const int sub = lane >> 3, q4 = lane & 7;  // store phase: row 4 i + sub, 16-byte column q4
        int32_t dst[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = __shfl_sync(0xffffffffu, out_row, 4 * i + sub);
        float *outf = static_cast<float *>(out);
        uint8_t *rowp = stage + lane * 144;
#pragma unroll 1
        for (int c = 0; c < cols; c += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + (uint32_t)c, r);
            tmem_ld_wait();
            const int col0 = n * cols + c;
            if (col0 < Nout) {  // the same for every lane
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4 *>(rowp + 16 * q) =
                        make_float4(g * __uint_as_float(r[4 * q + 0]), g * __uint_as_float(r[4 * q + 1]),
                                    g * __uint_as_float(r[4 * q + 2]), g * __uint_as_float(r[4 * q + 3]));
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 v = *reinterpret_cast<const float4 *>(stage + (4 * i + sub) * 144 + 16 * q4);
                    if (dst[i] >= 0) {
                        float *p = outf + (int64_t)dst[i] * Nout + col0 + 4 * q4;
                        if (add) red_add_v4_f32(p, v);
                        else *reinterpret_cast<float4 *>(p) = v;
                    }
                }
                __syncwarp();
            }
        }
    }
    return groups;
}

// ---------------------------------------------------------------------------
// Pair (2-CTA) version: a cluster of two CTAs on two SMs computes 256-row x
// BN-column tiles with tcgen05.mma.cta_group::2 (M = 256).  Each CTA loads
// its own 128 rows of A and half of the BN rows of B, so a ring stage is
// (16 + BN/8) KB instead of (16 + BN/4) KB: twice the lookahead in the same
// shared memory, and a third less L2 traffic per flop.
//   both CTAs, warp 0   TMA loads into their own shared memory, counted on
//                       the leader's (rank 0) "full" barrier
//   leader, warp 1      issues the pair MMAs; commits free the ring slot in
//                       both CTAs and publish the accumulator to both
//   both CTAs, warps 2-5  epilogue of their own 128 rows, then one arrival
//                       each on the leader's "accumulator empty" barrier
// Barrier addresses of the other CTA come from mapa; no load is multicast.
// ---------------------------------------------------------------------------
template <int BN, int STAGES>
struct PairLayout {
    static constexpr size_t a_bytes = (size_t)BM * BK * 2;
    static constexpr size_t b_bytes = (size_t)(BN / 2) * BK * 2;
    static constexpr size_t ring = STAGES * (a_bytes + b_bytes);
    static constexpr size_t stage_bytes = 5120;  // per epilogue warp (4.5 KB used), keeps 1024-byte alignment
    static constexpr size_t staging = 4 * stage_bytes;
    static constexpr size_t barriers = (2 * STAGES + 2 + 2 + 1) * 8 + 16;
    static size_t bytes(int experts) { return 1024 + ring + staging + barriers + (size_t)(experts + 1) * 4; }
};

// Per-expert shape of a grouped GEMM.  Forward: the rows of expert e are its
// kept tokens (min(counts[e], C)) and K is fixed.  Weight gradients of the
// backward pass: every expert with kept tokens has `rows_fixed` output rows
// (d_model or d_ff), no rows otherwise, and K runs over its kept tokens only
// (k_per_expert: ceil(kept / 64) K blocks; the operands are zero past them).
struct GroupShape {
    int rows_fixed;    // 0: rows = kept tokens
    int k_per_expert;  // 0: K / BK blocks for every tile
    int out_rows;      // kEpiExpertOut: rows of each expert's block of `out` (0: C)
    const uint16_t *mask_h;  // kEpiReluGrad: the forward's H [E][C][Nout]
    int b_k_stride;    // MN-major B only: > 0: B is one [T][Nout] matrix and group e's K rows start at
                       // row e * b_k_stride (groups = consecutive chunks of its rows)
    int wide_min;      // > 0: run only when (256-row blocks over all groups) * wide_n2 >= wide_min
    int wide_n2;       //      (the expert FFN's GEMM2 tile count; otherwise the fused kernel runs it)
};

__device__ __forceinline__ int group_rows(const GroupShape &g, int kept) {
    return g.rows_fixed > 0 ? (kept > 0 ? g.rows_fixed : 0) : kept;
}

// Operand storage of the pair GEMM: K-major (K contiguous, the forward's
// layout) or MN-major (M resp. N contiguous: the backward reads activations
// and weights in their forward layout, no transposes).  MN-major operands
// are loaded as two 64-element-wide TMA boxes per CTA and stage.
enum OperandMajor : int { kMajK = 0, kMajAmn = 1, kMajBmn = 2 };

template <int BN, int STAGES, int EPI, int MAJ = kMajK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_grouped_gemm_pair(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_out, void *__restrict__ out,
                         const int32_t *__restrict__ counts, int E, int C, int K, int Nout,
                         const int32_t *__restrict__ slot_token, const float *__restrict__ gate,
                         DeviceStatus *status, const GroupShape shape) {
    using L = PairLayout<BN, STAGES>;
    constexpr int BMP = 2 * BM;  // rows of a pair tile
    constexpr bool kAmn = (MAJ & kMajAmn) != 0, kBmn = (MAJ & kMajBmn) != 0;
    static_assert(!kAmn || BM == 128, "MN-major A: two 64-row boxes per CTA");
    static_assert(!kBmn || BN == 256, "MN-major B: two 64-column boxes per CTA");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = sA + STAGES * L::a_bytes;
    uint8_t *staging = base + L::ring;  // 1024-aligned: the ring is a multiple of 1024 bytes
    uint64_t *full = reinterpret_cast<uint64_t *>(staging + L::staging);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    int32_t *tile_start = reinterpret_cast<int32_t *>(tmem_holder + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int n_tiles_n = (Nout + BN - 1) / BN;
    const int k_blocks = K / BK;
    constexpr uint32_t kTmemCols = 2 * BN;

    if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            for (int a = 0; a < 2; ++a) {
                mbar_init(&acc_full[a], 1);
                mbar_init(&acc_empty[a], 2 * kEpilogueThreads);
            }
            mbar_init(drain, 1);
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc_pair(tmem_holder, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers are initialised before anyone signals them
    tc_fence_after();
    pdl_wait();  // counts, the A operand and the epilogue's inputs come from earlier kernels
    pdl_launch_dependents();
    if (warp == 0) {
        int kept_of[8];  // E <= 256: every count is loaded before the scan starts
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = 32 * j + lane;
            kept_of[j] = e < E ? group_rows(shape, min(counts[e], C)) : 0;
        }
        int running = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e0 = 32 * j;
            if (e0 >= E) break;
            const int e = e0 + lane;
            const int kept = kept_of[j];
            const int mine = (kept + BMP - 1) / BMP * n_tiles_n;
            int incl = mine;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += u;
            }
            if (e < E) tile_start[e] = running + incl - mine;
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) tile_start[E] = running;
    }
    __syncthreads();
    const uint32_t tmem_base = *tmem_holder;
    int total_tiles = tile_start[E];
    if (shape.wide_min > 0 && total_tiles / n_tiles_n * shape.wide_n2 < shape.wide_min)
        total_tiles = 0;  // few tiles: the fused kernel of this call computes the FFN

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmap_a);
            prefetch_tmap(&tmap_b);
            uint32_t issued = 0, parity_of = 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
                int e, m, n;
                locate_tile(tile_start, E, n_tiles_n, tile, e, m, n);
                const int kbs = shape.k_per_expert ? (min(counts[e], C) + BK - 1) / BK : k_blocks;
                for (int kb = 0; kb < kbs; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, status, 21)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 * (L::a_bytes + L::b_bytes)));
                    const uint32_t leader_full = map_to_rank(&full[stage], 0);
                    const int a_row = m * BMP + (int)rank * BM, b_row = n * BN + (int)rank * (BN / 2);
                    if (kAmn) {  // A stored [E][K][M]: this CTA's 128 rows as two 64-row slices of 8 KB
                        tma_load_3d_pair(sA + stage * L::a_bytes, &tmap_a, leader_full, a_row, kb * BK, e);
                        tma_load_3d_pair(sA + stage * L::a_bytes + L::a_bytes / 2, &tmap_a, leader_full,
                                         a_row + 64, kb * BK, e);
                    } else {
                        tma_load_3d_pair(sA + stage * L::a_bytes, &tmap_a, leader_full, kb * BK, a_row, e);
                    }
                    if (kBmn) {  // B stored [E][K][N]: this CTA's 128 columns as two 64-column slices
                        const int bk = shape.b_k_stride > 0 ? e * shape.b_k_stride + kb * BK : kb * BK;
                        const int bz = shape.b_k_stride > 0 ? 0 : e;
                        tma_load_3d_pair(sB + stage * L::b_bytes, &tmap_b, leader_full, b_row, bk, bz);
                        tma_load_3d_pair(sB + stage * L::b_bytes + L::b_bytes / 2, &tmap_b, leader_full,
                                         b_row + 64, bk, bz);
                    } else {
                        tma_load_3d_pair(sB + stage * L::b_bytes, &tmap_b, leader_full, kb * BK, b_row, e);
                    }
                    issued |= 1u << stage;
                    parity_of = (parity_of & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Wind-down (leader): every load counted on its barriers has landed.
            if (rank == 0)
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s)) mbar_wait(&full[s], (parity_of >> s) & 1u, status, 26);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32_major(BMP, BN, kAmn, kBmn);
            // per 16-element K step: +32 bytes inside a K-major row, +2048 bytes (two 8-row
            // groups) in an MN-major slice; descriptor start addresses count 16-byte units
            constexpr uint64_t a_step = kAmn ? 128 : 2, b_step = kBmn ? 128 : 2;
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
                int kbs = k_blocks;
                if (shape.k_per_expert) {
                    int e, m, n;
                    locate_tile(tile_start, E, n_tiles_n, tile, e, m, n);
                    kbs = (min(counts[e], C) + BK - 1) / BK;
                }
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, status, 22)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < kbs; ++kb) {
                    if (!mbar_wait(&full[stage], phase, status, 23)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = kAmn ? smem_desc_sw128_mn(sA + stage * L::a_bytes, L::a_bytes / 2)
                                                 : smem_desc_sw128(sA + stage * L::a_bytes);
                    const uint64_t b_desc = kBmn ? smem_desc_sw128_mn(sB + stage * L::b_bytes, L::b_bytes / 2)
                                                 : smem_desc_sw128(sB + stage * L::b_bytes);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16_pair(d_tmem, a_desc + a_step * (uint64_t)k, b_desc + b_step * (uint64_t)k, idesc,
                                         (kb | k) != 0 ? 1u : 0u);
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
            mbar_wait(drain, 0, status, 24);
        }
    } else {
        const int quarter = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < total_tiles; tile += n_pairs) {
            int e, m, n;
            locate_tile(tile_start, E, n_tiles_n, tile, e, m, n);
            if (!mbar_wait(&acc_full[acc], acc_phase, status, 25)) break;
            tc_fence_after();
            const int row_base = m * BMP + (int)rank * BM + quarter * 32;
            epilogue_async<BN, EPI>(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN), e,
                                    row_base, group_rows(shape, min(counts[e], C)), C, n, Nout, out, &tmap_out,
                                    slot_token, gate, staging + (warp - 2) * L::stage_bytes, false, shape.out_rows,
                                    shape.mask_h);
            tc_fence_before();
            mbar_arrive_cluster(map_to_rank(&acc_empty[acc], 0));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    if (warp >= 2) bulk_wait_all();  // this thread's stores have completed
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its peer may still use its shared memory or barriers
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Both expert GEMMs in one persistent launch on SM pairs (256 x 256 tiles).
// The tile list holds every GEMM1 tile (expert e, 256-row block m, H column
// block n) and then every GEMM2 tile (e, m, y column block).  Pairs claim
// tiles in list order from a per-call counter (the leader's producer thread
// takes the next index one tile ahead and hands it, through a 4-deep queue in
// shared memory, to its MMA thread, its epilogue warps and the peer CTA); a
// pair works through its claims in claim order, and every wait below is on a
// tile of lower index, so the lowest unfinished tile can always proceed.  A GEMM2
// tile reads the H rows of its row block, written by the n1 = F / 256 GEMM1
// tiles of (e, m): each of the pair's 8 epilogue warps adds 1 to done[e, m]
// once its H boxes have fully landed (TMA store completion, then a release
// add), and both producers of the GEMM2 tile wait (bounded) for done[e, m]
// = 8 * n1 before loading H.  Every GEMM1 tile is claimed before any GEMM2
// tile, and only by a running pair whose earlier tiles are GEMM1 tiles too,
// so each wait is on work that is already in progress: no assumption about
// how many pairs are resident at once.  The tail of GEMM1 overlaps the start
// of GEMM2, and the GEMM2 tiles, too few for one even wave on their own,
// share the waves with GEMM1.
// When GEMM2 has fewer tiles than two waves, every GEMM2 tile is cut into S
// parts (S = 2 or 4) along K = F, the part count picked on the device from
// the real tile counts (fused_split).  All parts ks = 0 come first in the
// list, then all parts ks = 1, and so on.  Part 0 stores gate * acc into y;
// part ks > 0 waits until y_done[e, m, n] reaches 8 ks (parts 0 .. ks-1 are
// in y) and adds its gate * acc with 16-byte fp32 reductions, then releases 8 more.
// Every y element is ((y0 + y1) + y2) + ... in that order: deterministic.
// The short parts fill the last wave; the chain of adds costs one epilogue
// per part.
// ---------------------------------------------------------------------------
constexpr int kFusedBN = 256;
// GEMM2 tile waves (256 x 256 tiles over the SM pairs) from which a layer call
// runs GEMM1 as its own launch and the fused kernel takes GEMM2 only.
constexpr int kWideWaves = 12;

// Parts per GEMM2 tile: 1, 2 or 4, for GEMM2 with fewer tiles than two waves
// only (the adds cost y traffic).  Picks the S that minimises a rough time
// for the GEMM2 waves in K blocks: waves * (K blocks per part) plus about six
// K blocks of epilogue per extra part in the chain of adds.  Every CTA
// computes the same value from the same counts.
__device__ __forceinline__ int fused_split(int tiles2, int kb_total, int pairs) {
    if (tiles2 <= 0 || tiles2 >= 2 * pairs) return 1;
    int best = 1, best_cost = ((tiles2 + pairs - 1) / pairs) * kb_total;
    for (int s = 2; s <= 4; s *= 2) {
        if (kb_total % s != 0 || kb_total / s < 8) break;
        const int cost = ((s * tiles2 + pairs - 1) / pairs) * (kb_total / s) + 6 * (s - 1);
        if (cost < best_cost) {
            best = s;
            best_cost = cost;
        }
    }
    return best;
}
constexpr int kTileQ = 4;                // tile-index queue depth
constexpr int kTileConsumers = 1 + 1 + 8;  // leader MMA thread, peer producer, 8 epilogue warps

template <int STAGES>
struct FusedLayout {
    using L = PairLayout<kFusedBN, STAGES>;
    // PairLayout (ring, staging, barriers, start1[E+1]) + tile queue + start2[E+1]
    static size_t bytes(int experts) {
        return L::bytes(experts) + 2 * kTileQ * 8 + kTileQ * 4 + (size_t)(experts + 1) * 4;
    }
};

template <int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_ffn_fused_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w1,
                      const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w2,
                      const __grid_constant__ CUtensorMap tm_w1h, const __grid_constant__ CUtensorMap tm_w2h,
                      const __grid_constant__ CUtensorMap tm_hstore, float *__restrict__ y,
                      const int32_t *__restrict__ counts, int E, int C, int d, int F,
                      const int32_t *__restrict__ slot_token, const float *__restrict__ gate,
                      int32_t *__restrict__ done, int MT, DeviceStatus *status, int wide_min) {
    constexpr int BN = kFusedBN;
    using L = PairLayout<BN, STAGES>;
    constexpr int BMP = 2 * BM;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = sA + STAGES * L::a_bytes;
    uint8_t *staging = base + L::ring;
    uint64_t *full = reinterpret_cast<uint64_t *>(staging + L::staging);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint64_t *tq_full = drain + 1;          // [kTileQ] tile index written (both CTAs)
    uint64_t *tq_empty = tq_full + kTileQ;  // [kTileQ] tile index read by all (leader's)
    int32_t *tq = reinterpret_cast<int32_t *>(tq_empty + kTileQ);  // [kTileQ] tile index, -1 = no more
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tq + kTileQ);
    int32_t *start1 = reinterpret_cast<int32_t *>(tmem_holder + 4);  // [E+1] GEMM1 tiles per expert
    int32_t *start2 = start1 + (E + 1);                              // [E+1] GEMM2 tiles per expert
    int32_t *ticket = done + (int64_t)E * MT;                        // tile claim counter of this call
    int32_t *y_done = ticket + 1;                                    // [E][MT][n2] GEMM2 parts stored in y

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int kb1 = d / BK;  // K blocks of a GEMM1 tile
    constexpr uint32_t kTmemCols = 2 * BN;

    if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            for (int a = 0; a < 2; ++a) {
                mbar_init(&acc_full[a], 1);
                mbar_init(&acc_empty[a], 2 * kEpilogueThreads);
            }
            mbar_init(drain, 1);
            for (int j = 0; j < kTileQ; ++j) {
                mbar_init(&tq_full[j], 1);
                mbar_init(&tq_empty[j], kTileConsumers);
            }
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc_pair(tmem_holder, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    pdl_wait();
    pdl_launch_dependents();
    if (warp == 0) {
        int kept_of[8];
        int mt_all = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = 32 * j + lane;
            kept_of[j] = e < E ? min(counts[e], C) : 0;
            mt_all += (kept_of[j] + BMP - 1) / BMP;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt_all += __shfl_xor_sync(0xffffffffu, mt_all, off);
        // Tile widths, per GEMM: 256 columns, or 128 when few rows are kept (e.g.
        // a skewed routing): twice the tiles, each half as long.  GEMM1 goes
        // narrow only when 256-wide tiles would leave more than half the pairs
        // without one (a narrow tile re-reads its A rows for half the output);
        // GEMM2, whose tiles wait on H, goes narrow as soon as 256-wide tiles
        // cannot give every pair one.  Every CTA derives the same widths from
        // the same counts.
        const int pairs = (int)(gridDim.x >> 1);
        const int bw1 = 2 * mt_all * ((F + BN - 1) / BN) <= pairs ? BN / 2 : BN;
        const int bw2 = mt_all * ((d + BN - 1) / BN) < pairs ? BN / 2 : BN;
        const int n1 = (F + bw1 - 1) / bw1, n2 = (d + bw2 - 1) / bw2;
        if (lane == 0) {
            tmem_holder[1] = (uint32_t)bw1;
            tmem_holder[2] = (uint32_t)bw2;
        }
        int run1 = 0, run2 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e0 = 32 * j;
            if (e0 >= E) break;
            const int e = e0 + lane;
            const int mt = (kept_of[j] + BMP - 1) / BMP;
            int i1 = mt * n1, i2 = mt * n2;
            const int m1 = i1, m2 = i2;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int u1 = __shfl_up_sync(0xffffffffu, i1, off);
                const int u2 = __shfl_up_sync(0xffffffffu, i2, off);
                if (lane >= off) {
                    i1 += u1;
                    i2 += u2;
                }
            }
            if (e < E) {
                start1[e] = run1 + i1 - m1;
                start2[e] = run2 + i2 - m2;
            }
            run1 += __shfl_sync(0xffffffffu, i1, 31);
            run2 += __shfl_sync(0xffffffffu, i2, 31);
        }
        if (lane == 0) {
            start1[E] = run1;
            start2[E] = run2;
        }
    }
    __syncthreads();
    const uint32_t tmem_base = *tmem_holder;
    const int bw1 = (int)tmem_holder[1], bw2 = (int)tmem_holder[2];  // tile widths (columns) of GEMM1, GEMM2
    const int n1 = (F + bw1 - 1) / bw1, n2 = (d + bw2 - 1) / bw2;
    const int32_t need = 8 * n1;  // arrivals on done[e, m] once H of the row block is complete
    // Many tiles: GEMM1 ran as its own launch just before this one (measured faster there), so
    // this launch takes the GEMM2 tiles only and their H is complete before griddepcontrol.wait
    // returns; every CTA decides alike from the same counts.
    const bool wide = wide_min > 0 && start1[E] / n1 * ((d + BN - 1) / BN) >= wide_min;
    const int total1 = wide ? 0 : start1[E];
    const int total2 = start2[E];  // GEMM2 output tiles
    const int split = fused_split(total2, F / BK, (int)(gridDim.x >> 1));
    const int kb2 = F / BK / split;  // K blocks of a GEMM2 part
    const int total = total1 + split * total2;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(bw1 == BN ? &tm_w1 : &tm_w1h);
            prefetch_tmap(&tm_h);
            prefetch_tmap(bw2 == BN ? &tm_w2 : &tm_w2h);
            uint32_t issued = 0, parity_of = 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            // The leader claims one tile ahead: the claim of the next tile is in
            // flight while this tile's loads are issued, so the ring does not run
            // dry for the claim's round trip at every tile boundary.  Tiles are
            // still processed in claim order, one pair at a time.
            int pending = rank == 0 ? atomicAdd(ticket, 1) : -1;
            for (int it = 0; ok; ++it) {
                const int j = it % kTileQ;
                const uint32_t qph = (uint32_t)(it / kTileQ) & 1u;
                int tile;
                if (rank == 0) {  // hand the claimed tile's index to everyone, claim the next
                    if (!mbar_wait_cluster(&tq_empty[j], qph ^ 1u, status, 48)) break;
                    tile = pending;
                    if (tile >= total) tile = -1;
                    if (tile >= 0) pending = atomicAdd(ticket, 1);
                    tq[j] = tile;
                    st_cluster_s32(map_to_rank(&tq[j], 1), tile);
                    mbar_arrive(&tq_full[j]);
                    mbar_arrive_cluster(map_to_rank(&tq_full[j], 1));
                } else {
                    if (!mbar_wait_cluster(&tq_full[j], qph, status, 49)) break;
                    tile = tq[j];
                    mbar_arrive_cluster(map_to_rank(&tq_empty[j], 0));
                }
                if (tile < 0) break;
                const bool second = tile >= total1;
                int e, m, n, ks = 0;
                if (second) {
                    ks = (tile - total1) / total2;
                    locate_tile(start2, E, n2, tile - total1 - ks * total2, e, m, n);
                } else {
                    locate_tile(start1, E, n1, tile, e, m, n);
                }
                const int k0 = ks * kb2;  // first K block of this tile
                if (second && !wide) {
                    if (!wait_counter_geq(done + e * MT + m, need, status, 47)) break;
                    fence_proxy_async_global();  // H, written through the async proxy, before our TMA reads
                }
                const void *ta = second ? (const void *)&tm_h : (const void *)&tm_x;
                const void *tb = second ? (bw2 == BN ? (const void *)&tm_w2 : (const void *)&tm_w2h)
                                        : (bw1 == BN ? (const void *)&tm_w1 : (const void *)&tm_w1h);
                const int kbs = second ? kb2 : kb1;
                const int bw = second ? bw2 : bw1;
                const uint32_t b_bytes = (uint32_t)(bw / 2) * BK * 2;  // this CTA's rows of a B stage
                const int a_row = m * BMP + (int)rank * BM, b_row = n * bw + (int)rank * (bw / 2);
                for (int kb = 0; kb < kbs; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, status, 41)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 * (L::a_bytes + b_bytes)));
                    const uint32_t leader_full = map_to_rank(&full[stage], 0);
                    tma_load_3d_pair(sA + stage * L::a_bytes, ta, leader_full, (k0 + kb) * BK, a_row, e);
                    tma_load_3d_pair(sB + stage * L::b_bytes, tb, leader_full, (k0 + kb) * BK, b_row, e);
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
                    if (issued & (1u << s)) mbar_wait(&full[s], (parity_of >> s) & 1u, status, 46);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            const uint32_t idesc1 = idesc_bf16_f32(BMP, bw1), idesc2 = idesc_bf16_f32(BMP, bw2);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int it = 0;; ++it) {
                const int j = it % kTileQ;
                if (!mbar_wait(&tq_full[j], (uint32_t)(it / kTileQ) & 1u, status, 50)) break;
                const int tile = tq[j];
                mbar_arrive(&tq_empty[j]);
                if (tile < 0) break;
                const int kbs = tile >= total1 ? kb2 : kb1;
                const uint32_t idesc = tile >= total1 ? idesc2 : idesc1;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, status, 42)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < kbs; ++kb) {
                    if (!mbar_wait(&full[stage], phase, status, 43)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = smem_desc_sw128(sA + stage * L::a_bytes);
                    const uint64_t b_desc = smem_desc_sw128(sB + stage * L::b_bytes);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16_pair(d_tmem, a_desc + (uint64_t)(2 * k), b_desc + (uint64_t)(2 * k), idesc,
                                         (kb | k) != 0 ? 1u : 0u);
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
            mbar_wait(drain, 0, status, 44);
        }
    } else {
        const int quarter = warp & 3;
        uint8_t *my_stage = staging + (warp - 2) * L::stage_bytes;
        int acc = 0;
        uint32_t acc_phase = 0;
        // Lane 0 releases a GEMM1 tile's H counter one tile late: after the next
        // GEMM1 tile's boxes are issued it waits for all but those, so the warp
        // never idles on its own store completions between tiles.  Before a GEMM2
        // tile (whose loads may wait on that counter) or the end, it releases at once.
        int32_t *deferred = nullptr;
        for (int it = 0;; ++it) {
            const int j = it % kTileQ;
            const uint32_t qph = (uint32_t)(it / kTileQ) & 1u;
            const bool got = rank == 0 ? mbar_wait(&tq_full[j], qph, status, 51)
                                       : mbar_wait_cluster(&tq_full[j], qph, status, 52);
            if (!got) break;
            const int tile = tq[j];
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&tq_empty[j]);
                else mbar_arrive_cluster(map_to_rank(&tq_empty[j], 0));
                if (deferred && (tile < 0 || tile >= total1)) {
                    bulk_wait_all();
                    fence_proxy_async_global();
                    red_release_add_gpu(deferred, 1);
                    deferred = nullptr;
                }
            }
            if (tile < 0) break;
            const bool second = tile >= total1;
            int e, m, n, ks = 0;
            if (second) {
                ks = (tile - total1) / total2;
                locate_tile(start2, E, n2, tile - total1 - ks * total2, e, m, n);
            } else {
                locate_tile(start1, E, n1, tile, e, m, n);
            }
            int32_t *ydone = y_done + ((int64_t)e * MT + m) * n2 + n;
            if (ks > 0) {  // parts 0 .. ks-1 of this output tile are in y
                bool okw = true;
                if (lane == 0) okw = wait_counter_geq(ydone, 8 * ks, status, 53);
                __syncwarp();  // every lane's adds below come after lane 0's acquire
                if (!__shfl_sync(0xffffffffu, okw, 0)) break;
            }
            if (!mbar_wait(&acc_full[acc], acc_phase, status, 45)) break;
            tc_fence_after();
            const int row_base = m * BMP + (int)rank * BM + quarter * 32;
            const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            int groups = 0;
            if (second)
                epilogue_async<BN, kEpiGatedScatter>(t_row, e, row_base, min(counts[e], C), C, n, d, y, nullptr,
                                                     slot_token, gate, my_stage, ks > 0, 0, nullptr, bw2);
            else
                groups = epilogue_async<BN, kEpiHiddenRelu>(t_row, e, row_base, min(counts[e], C), C, n, F,
                                                            nullptr, &tm_hstore, slot_token, gate, my_stage, false, 0,
                                                            nullptr, bw1);
            tc_fence_before();
            mbar_arrive_cluster(map_to_rank(&acc_empty[acc], 0));
            if (lane == 0) {
                if (!second) {
                    if (deferred) {  // the previous GEMM1 tile's boxes, this tile's may stay in flight
                        bulk_wait_all_but(groups);
                        fence_proxy_async_global();  // ... ordered before the release below
                        red_release_add_gpu(deferred, 1);
                    }
                    deferred = done + e * MT + m;
                }
            }
            if (second && ks < split - 1) {
                __syncwarp();  // every lane's y stores / adds of this part ...
                if (lane == 0) {
                    __threadfence();  // ... are visible before the release below
                    red_release_add_gpu(ydone, 1);
                }
            }
            __syncwarp();
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    if (warp >= 2) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches
// ---------------------------------------------------------------------------
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

// 3-D bf16 tensor [E][rows][K] (K contiguous), box = box_rows x 64, 128-byte swizzle.
bool make_tmap(CUtensorMap *map, const void *ptr, int E, int rows, int K, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)E};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)rows * K * 2};
    const cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 tensor [E][rows][cols] (cols contiguous), box = 32 rows x 32 columns, 128-byte swizzle
// (the weight-gradient epilogue's store boxes).
bool make_tmap_f32_box32(CUtensorMap *map, const void *ptr, int E, int rows, int cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)E};
    const cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)rows * cols * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES, int EPI>
cudaError_t launch_gemm(int32_t kernel_id, const void *a, const void *b, void *out, const int32_t *counts, int E,
                        int C, int K, int Nout, int64_t T, const int32_t *slot_token, const float *gate,
                        DeviceStatus *status, cudaStream_t stream) {
    CUtensorMap ta, tb;
    if (!make_tmap(&ta, a, E, C, K, BM) || !make_tmap(&tb, b, E, Nout, K, BN)) return cudaErrorInvalidValue;
    const size_t smem = TcLayout<BN, STAGES>::bytes(E);
    auto kern = tc_grouped_gemm<BN, STAGES, EPI>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    // Upper bound on the number of tiles, from host-known sizes only.
    const int64_t m_tiles = std::min<int64_t>((int64_t)E * ((C + BM - 1) / BM), (T + BM - 1) / BM + E);
    const int64_t tiles = m_tiles * ((Nout + BN - 1) / BN);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(device_sm_count(), tiles));
    launch_begin(kernel_id, stream);
    kern<<<grid, kThreads, smem, stream>>>(ta, tb, out, counts, E, C, K, Nout, slot_token, gate, status);
    err = cudaGetLastError();
    launch_end(stream);
    return err;
}

// A [E][a_rows][K] and B [E][Nout][K] (bf16, K contiguous), or with MAJ
// MN-major A [E][K][a_rows] and/or B [E][K][Nout]; a_rows = C unless the shape
// has fixed rows (then A holds rows_fixed rows per expert and K is the token
// extent of the operands, read up to each expert's kept tokens).
template <int BN, int STAGES, int EPI, int MAJ = kMajK>
cudaError_t launch_gemm_pair(int32_t kernel_id, const void *a, const void *b, void *out, const int32_t *counts, int E,
                             int C, int K, int Nout, int64_t T, const int32_t *slot_token, const float *gate,
                             DeviceStatus *status, cudaStream_t stream, GroupShape shape = GroupShape{0, 0, 0, nullptr}) {
    const int a_rows = shape.rows_fixed > 0 ? shape.rows_fixed : C;
    CUtensorMap ta, tb, tout;
    const bool ok_a = (MAJ & kMajAmn) ? make_tmap(&ta, a, E, K, a_rows, 64) : make_tmap(&ta, a, E, a_rows, K, BM);
    if (shape.b_k_stride > 0 && (!(MAJ & kMajBmn) || T > INT32_MAX)) return cudaErrorInvalidValue;
    const bool ok_b = !(MAJ & kMajBmn)        ? make_tmap(&tb, b, E, Nout, K, BN / 2)
                      : shape.b_k_stride > 0 ? make_tmap(&tb, b, 1, (int)T, Nout, 64)  // one [T][Nout] matrix
                                             : make_tmap(&tb, b, E, K, Nout, 64);
    if (!ok_a || !ok_b) return cudaErrorInvalidValue;
    memset(&tout, 0, sizeof tout);
    if ((EPI == kEpiHiddenRelu || EPI == kEpiReluGrad) && !make_tmap(&tout, out, E, C, Nout, 32))
        return cudaErrorInvalidValue;
    if (EPI == kEpiWeightGrad && (shape.rows_fixed <= 0 || !make_tmap_f32_box32(&tout, out, E, shape.rows_fixed, Nout)))
        return cudaErrorInvalidValue;
    const size_t smem = PairLayout<BN, STAGES>::bytes(E);
    auto kern = tc_grouped_gemm_pair<BN, STAGES, EPI, MAJ>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int64_t m_tiles =
        shape.rows_fixed > 0
            ? (int64_t)E * ((shape.rows_fixed + 2 * BM - 1) / (2 * BM))
            : std::min<int64_t>((int64_t)E * ((C + 2 * BM - 1) / (2 * BM)), (T + 2 * BM - 1) / (2 * BM) + E);
    const int64_t tiles = m_tiles * ((Nout + BN - 1) / BN);
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(device_sm_count() / 2, tiles));
    launch_begin(kernel_id, stream);
    err = launch_kernel(kern, dim3(2 * pairs), dim3(kThreads), smem, stream, true, ta, tb, tout, out, counts, E, C, K,
                        Nout, slot_token, gate, status, shape);
    launch_end(stream);
    return err;
}

template <int STAGES>
cudaError_t launch_ffn_fused(const switch_dims_t &dims, const void *xbuf, const void *w_in, const void *w_out,
                             const int32_t *counts, const int32_t *slot_token, const float *gate, float *y,
                             const Workspace &ws, bool zero_done, int wide_min, cudaStream_t stream) {
    const int E = dims.num_experts, C = dims.capacity, d = dims.d_model, F = dims.d_ff;
    const size_t smem = FusedLayout<STAGES>::bytes(E);
    auto kern = tc_ffn_fused_pair<STAGES>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    CUtensorMap tx, tw1, th, tw2, tw1h, tw2h, ths;
    if (!make_tmap(&tx, xbuf, E, C, d, BM) || !make_tmap(&tw1, w_in, E, F, d, kFusedBN / 2) ||
        !make_tmap(&th, ws.hidden, E, C, F, BM) || !make_tmap(&tw2, w_out, E, d, F, kFusedBN / 2) ||
        !make_tmap(&tw1h, w_in, E, F, d, kFusedBN / 4) || !make_tmap(&tw2h, w_out, E, d, F, kFusedBN / 4) ||
        !make_tmap(&ths, ws.hidden, E, C, F, 32))
        return cudaErrorInvalidValue;
    const int MT = (C + 2 * BM - 1) / (2 * BM);
    const int n2 = (d + kFusedBN / 2 - 1) / (kFusedBN / 2);  // at the narrow tile width
    if (zero_done) {  // counters, the tile claim counter and the y_done counters
        err = cudaMemsetAsync(ws.done, 0, fused_counter_ints(E, C, d) * sizeof(int32_t), stream);
        if (err != cudaSuccess) return err;
    }
    const int64_t m_tiles = std::min<int64_t>((int64_t)E * MT, (dims.T + 2 * BM - 1) / (2 * BM) + E);
    const int64_t tiles2 = m_tiles * n2;
    const int max_pairs = device_sm_count() / 2;
    // upper bound on the tile count (GEMM2 tiles may be cut into up to 4 parts on the device)
    const int64_t tiles = m_tiles * ((F + kFusedBN / 2 - 1) / (kFusedBN / 2)) + 4 * tiles2;
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(max_pairs, tiles));
    launch_begin(K_FFN_TC_FUSED, stream);
    err = launch_kernel(kern, dim3(2 * pairs), dim3(kThreads), smem, stream, !zero_done, tx, tw1, th, tw2, tw1h, tw2h,
                        ths, y, counts, E, C, d, F, slot_token, gate, ws.done, MT,
                        static_cast<DeviceStatus *>(ws.status), wide_min);
    launch_end(stream);
    return err;
}

}  // namespace

// Backward GEMMs (SM pairs, 256 x 256 tiles, the forward's kernel; weights and
// activations read in their forward layout as MN-major operands).
// dZ [N][C][F] = bf16((dE W_out) where H > 0): A = dE [N][C][d] (K-major),
// B = W_out [N][d][F] (K = d rows, N = F contiguous).
cudaError_t launch_ffn_tc_bwd_dz(const switch_dims_t &dims, const void *grad_e, const void *w_out,
                                 const int32_t *counts, void *grad_z, const void *hidden, DeviceStatus *st,
                                 cudaStream_t stream) {
    return launch_gemm_pair<256, 6, kEpiReluGrad, kMajBmn>(
        K_BWD_GEMM_DZ, grad_e, w_out, grad_z, counts, dims.num_experts, dims.capacity, dims.d_model, dims.d_ff,
        dims.T, nullptr, nullptr, st, stream, GroupShape{0, 0, 0, static_cast<const uint16_t *>(hidden)});
}

// dx[slot_token] += dZ W_in: A = dZ [N][C][F] (K-major), B = W_in [N][F][d]
// (K = F rows, N = d contiguous).
cudaError_t launch_ffn_tc_bwd_dx(const switch_dims_t &dims, const void *grad_z, const void *w_in,
                                 const int32_t *counts, const int32_t *slot_token, float *dx, DeviceStatus *st,
                                 cudaStream_t stream) {
    return launch_gemm_pair<256, 6, kEpiScatterAdd, kMajBmn>(K_BWD_GEMM_DX, grad_z, w_in, dx, counts,
                                                             dims.num_experts, dims.capacity, dims.d_ff, dims.d_model,
                                                             dims.T, slot_token, nullptr, st, stream);
}

// Weight gradient out [N][rows][nout] (fp32) = sum over each expert's kept
// tokens s of a[s] b[s]^T: A [N][C][rows] and B [N][C][nout], both read
// MN-major (token rows, K = the tokens; rows from the expert's kept count up
// to the next multiple of 64 must hold zeros, rows past C read as zeros).
cudaError_t launch_ffn_tc_bwd_dw(const switch_dims_t &dims, const void *a, const void *b, const int32_t *counts,
                                 int rows, int nout, float *out, DeviceStatus *st, cudaStream_t stream) {
    return launch_gemm_pair<256, 6, kEpiWeightGrad, kMajAmn | kMajBmn>(
        K_BWD_GEMM_DW, a, b, out, counts, dims.num_experts, dims.capacity, dims.capacity, nout, dims.T, nullptr,
        nullptr, st, stream, GroupShape{rows, 1, rows, nullptr});
}

// Router part of dx (float32 [T][d], overwritten) = A . B^T with A [T][K] the
// split dh terms and B [d][K] the split W_r terms: one group of T fixed rows
// (`one` points at a device 1, the group's count).
cudaError_t launch_router_tc_bwd_dx(const void *a, const void *b, const int32_t *one, int64_t T, int d, int K,
                                    float *dx, DeviceStatus *st, cudaStream_t stream) {
    if (T > INT32_MAX) return cudaErrorInvalidValue;
    return launch_gemm_pair<256, 6, kEpiWeightGrad>(K_BWD_ROUTER_TC_DX, a, b, dx, one, 1, 1, K, d, T, nullptr,
                                                   nullptr, st, stream, GroupShape{(int)T, 0, (int)T, nullptr});
}

// dW_r partials part [chunks][rows][d] (float32): per chunk c of Tc tokens,
// A [rows][Tc] (split dh terms, token-contiguous) . x[c Tc .. c Tc + Tc)
// (x [T][d] read as an MN-major B along its token rows; rows past T read as
// zeros) over the chunk's chunk_counts[c] tokens.
cudaError_t launch_router_tc_bwd_dw(const void *a, const void *x, const int32_t *chunk_counts, int chunks, int rows,
                                    int chunk_tokens, int d, int64_t T, float *part, DeviceStatus *st,
                                    cudaStream_t stream) {
    return launch_gemm_pair<256, 6, kEpiWeightGrad, kMajBmn>(K_BWD_ROUTER_TC_DW, a, x, part, chunk_counts, chunks,
                                                            chunk_tokens, chunk_tokens, d, T, nullptr, nullptr, st,
                                                            stream, GroupShape{rows, 1, rows, nullptr, chunk_tokens});
}

cudaError_t launch_ffn_tc(const switch_dims_t &dims, const void *xbuf, const void *w_in, const void *w_out,
                          const int32_t *counts, void *ybuf, const int32_t *slot_token, const float *gate, float *y,
                          const Workspace &ws, cudaStream_t stream) {
    const int N = dims.num_experts, C = dims.capacity, d = dims.d_model, F = dims.d_ff;
    DeviceStatus *st = static_cast<DeviceStatus *>(ws.status);
    if (y && !(dims.flags & (SWITCH_FLAG_GEMM_1CTA | SWITCH_FLAG_FFN_TWO_LAUNCHES))) {
        // Both GEMMs in one launch (the dependency counters were zeroed by the
        // slot assignment of this call).  When GEMM2 may have kWideWaves waves of
        // 256-wide tiles or more, GEMM1's own launch goes first and the device
        // counts decide: with that many tiles GEMM1 runs there and the fused
        // kernel takes GEMM2 only (measured faster: 1.68 against 1.78 ms of
        // expert GEMMs on the Switch-Large shape); otherwise GEMM1's launch exits
        // at once and the fused kernel runs both.
        const int pairs = device_sm_count() / 2;
        const int n2w = (d + 255) / 256;
        const int64_t max_mt = std::min<int64_t>((int64_t)N * ((C + 255) / 256), (dims.T + 255) / 256 + N);
        const int wide_min = kWideWaves * pairs;
        if (max_mt * n2w < wide_min)
            return launch_ffn_fused<6>(dims, xbuf, w_in, w_out, counts, slot_token, gate, y, ws, false, 0, stream);
        const GroupShape gated{0, 0, 0, nullptr, 0, wide_min, n2w};
        cudaError_t err = launch_gemm_pair<256, 6, kEpiHiddenRelu>(K_FFN_TC_GEMM1, xbuf, w_in, ws.hidden, counts, N,
                                                                   C, d, F, dims.T, nullptr, nullptr, st, stream,
                                                                   gated);
        if (err != cudaSuccess) return err;
        return launch_ffn_fused<6>(dims, xbuf, w_in, w_out, counts, slot_token, gate, y, ws, false, wide_min, stream);
    }
    if (dims.flags & SWITCH_FLAG_GEMM_1CTA) {
        cudaError_t err = launch_gemm<256, 4, kEpiHiddenRelu>(K_FFN_TC_GEMM1, xbuf, w_in, ws.hidden, counts, N, C, d,
                                                              F, dims.T, nullptr, nullptr, st, stream);
        if (err != cudaSuccess) return err;
        if (y)
            return launch_gemm<128, 6, kEpiGatedScatter>(K_FFN_TC_GEMM2_GATED, ws.hidden, w_out, y, counts, N, C, F,
                                                         d, dims.T, slot_token, gate, st, stream);
        return launch_gemm<128, 6, kEpiExpertOut>(K_FFN_TC_GEMM2, ws.hidden, w_out, ybuf, counts, N, C, F, d,
                                                  dims.T, nullptr, nullptr, st, stream);
    }
    cudaError_t err = launch_gemm_pair<256, 6, kEpiHiddenRelu>(K_FFN_TC_GEMM1, xbuf, w_in, ws.hidden, counts, N, C,
                                                               d, F, dims.T, nullptr, nullptr, st, stream);
    if (err != cudaSuccess) return err;
    // 256-column tiles for both GEMMs: a 128-column GEMM2 tile re-reads its
    // A rows (H) for half the output, doubling the operand traffic per flop,
    // and ran about half as fast on B200 (the MMAs themselves take 64 cycles
    // for N = 128 against 128 for N = 256: the same rate per flop).
    if (y)
        return launch_gemm_pair<256, 6, kEpiGatedScatter>(K_FFN_TC_GEMM2_GATED, ws.hidden, w_out, y, counts, N, C,
                                                          F, d, dims.T, slot_token, gate, st, stream);
    return launch_gemm_pair<256, 6, kEpiExpertOut>(K_FFN_TC_GEMM2, ws.hidden, w_out, ybuf, counts, N, C, F, d,
                                                   dims.T, nullptr, nullptr, st, stream);
}

}  // namespace switchmoe
