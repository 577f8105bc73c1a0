// skinny_mma.cuh -- the rank-r products of the adapter on tcgen05 tensor cores.
//
//   D[i, j] = sum_t P(i, t) * Q(j, t),    i in tiles of 128 (MMA M = TMEM lanes),
//                                          j < r (MMA N = Nq, a multiple of 16 >= r),
//                                          t in stages of 128
//   out[i * ld_i + j * ld_j] += scaling * D[i, j]      (fp32 reductions)
//
// P is the streamed activation, Q the small rank-r factor; each is K-major (t
// contiguous) or MN-major (i or j contiguous) and is staged by TMA in the
// swizzled layout the MMA reads directly:
//   U  = X . A_lora^T   P = X [M, K] K-major,    Q = A [r, K] K-major,   out [M, r]
//   G  = dY . B_lora    P = dY [M, N] K-major,   Q = B [N, r] MN-major,  out [M, r]
//   dA^T = X^T . G      P = X [M, K] MN-major,   Q = G [M, r] MN-major,  out dA [r, K]
//   dB = dY^T . U       P = dY [M, N] MN-major,  Q = U [M, r] MN-major,  out dB [N, r]
// The products stream P once from HBM and are memory-bound.  Putting i on the
// TMEM lanes gives every epilogue thread one output row, so the r results of a
// row leave in a few vector reductions.
// Work split (stream-K): the (i tile, t stage) units are numbered tile-major and
// each CTA takes one contiguous range of them, so every SM streams about the
// same number of bytes; the accumulator is double-buffered in TMEM so the
// epilogue of one tile overlaps the MMAs of the next.  Two CTAs share an SM (half
// of the shared memory and of TMEM each), so that one CTA's first loads and last
// reductions overlap the other's streaming: 13-15 % faster on the 70B shapes than one
// CTA with the whole ring.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {
namespace skinny {

constexpr int BI = 128;                    // i per tile
constexpr int BT = 128;                    // t per stage
constexpr int kThreads = 192;              // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kPBytes = BI * BT * 2;       // 32 KB
constexpr int kMaxStages = 8;
constexpr int kRingBudget = 100 * 1024;    // bytes of stage buffers (two CTAs per SM)
constexpr int kTmemCols = 256;             // two accumulators of up to 128 columns

struct Params {
    int T;             // contraction length
    int I;             // rows i
    int r;             // valid columns j
    int Nq;            // MMA N: multiple of 16, r <= Nq <= 128
    int p_mn, q_mn;    // majorness (0: K-major, 1: MN-major)
    int p_3d;          // P as one 3-D box {64, 128, 2} (else two 2-D boxes of 64 x 128)
    int q_3d;          // K-major Q as one 3-D box {64, Nq, 2} (else two 2-D boxes)
    int q_atoms;       // MN-major Q: swizzle atoms per stage (1 or 2)
    int q_span;        // MN-major Q: swizzle span in bytes (32, 64 or 128) = row bytes of an atom
    int q_bytes;       // Q bytes per stage
    int stages;        // ring depth
    int64_t units;     // tiles * stages along t
    float scaling;
    float *out;
    int64_t ld_i, ld_j;
};

__host__ __device__ constexpr int stage_bytes(int q_bytes) { return kPBytes + q_bytes; }
__host__ __device__ constexpr int smem_bytes(int stages, int q_bytes) {
    return 1024 + stages * stage_bytes(q_bytes) + 256;
}

__global__ void __launch_bounds__(kThreads, 2)
    skinny_mma_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                      const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int SB = stage_bytes(p.q_bytes);
    const int S = p.stages;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * SB);
    uint64_t *full = bars, *empty = bars + kMaxStages;
    uint64_t *acc_full = bars + 2 * kMaxStages, *acc_empty = acc_full + 2, *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ST = (p.T + BT - 1) / BT;
    const int64_t u_begin = p.units * blockIdx.x / gridDim.x;
    const int64_t u_end = p.units * (blockIdx.x + 1) / gridDim.x;
    const int nu = static_cast<int>(u_end - u_begin);

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && nu > 0) {
            tma_prefetch_desc(&tmP);
            tma_prefetch_desc(&tmQ);
            const uint32_t tx = kPBytes + p.q_bytes;
            const int qw = p.q_span / 2;          // elements per MN-major Q atom row
            int issued = 0;
            for (int k = 0; k < nu; ++k) {
                const int64_t u = u_begin + k;
                const int i0 = static_cast<int>(u / ST) * BI;
                const int t0 = static_cast<int>(u % ST) * BT;
                const int sx = k % S;
                if (!mbar_wait(&empty[sx], ((k / S) & 1) ^ 1, abort_flag)) break;
                uint8_t *sp = smem + sx * SB;
                uint8_t *sq = sp + kPBytes;
                mbar_arrive_expect_tx(&full[sx], tx);
                if (!p.p_mn) {                     // [I, T]: rows i, t contiguous
                    if (p.p_3d) {
                        tma_load_3d(sp, &tmP, &full[sx], 0, i0, t0 / 64);
                    } else {
                        tma_load_2d(sp, &tmP, &full[sx], t0, i0);
                        tma_load_2d(sp + kPBytes / 2, &tmP, &full[sx], t0 + 64, i0);
                    }
                } else {                           // [T, I]: rows t, i contiguous
                    if (p.p_3d) {
                        tma_load_3d(sp, &tmP, &full[sx], 0, t0, i0 / 64);
                    } else {
                        tma_load_2d(sp, &tmP, &full[sx], i0, t0);
                        tma_load_2d(sp + kPBytes / 2, &tmP, &full[sx], i0 + 64, t0);
                    }
                }
                if (!p.q_mn) {                     // [r, T]
                    if (p.q_3d) {
                        tma_load_3d(sq, &tmQ, &full[sx], 0, 0, t0 / 64);
                    } else {
                        tma_load_2d(sq, &tmQ, &full[sx], t0, 0);
                        tma_load_2d(sq + p.Nq * 128, &tmQ, &full[sx], t0 + 64, 0);
                    }
                } else {                           // [T, r]
                    for (int a = 0; a < p.q_atoms; ++a)
                        tma_load_2d(sq + a * BT * p.q_span, &tmQ, &full[sx], a * qw, t0);
                }
                issued = k + 1;
            }
            for (int k = max(0, issued - S); k < issued; ++k) mbar_drain(&full[k % S], (k / S) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0 && nu > 0) {
            const uint32_t idesc = make_idesc_bf16(BI, p.Nq, p.p_mn, p.q_mn);
            int seg = 0, done = 0;
            for (int k = 0; k < nu; ++k) {
                const int64_t u = u_begin + k;
                const bool first = (k == 0) || (u % ST == 0);
                const bool last = (k == nu - 1) || ((u + 1) % ST == 0);
                const int buf = seg & 1;
                if (first && !mbar_wait(&acc_empty[buf], ((seg >> 1) & 1) ^ 1, abort_flag)) break;
                const int sx = k % S;
                if (!mbar_wait(&full[sx], (k / S) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t sp = smem_u32(smem + sx * SB);
                const uint32_t sq = sp + kPBytes;
#pragma unroll
                for (int kk = 0; kk < BT / 16; ++kk) {
                    const uint64_t pd = p.p_mn ? make_sdesc_sw128(sp + kk * 2048, kPBytes / 2, 1024)
                                               : make_sdesc_sw128(sp + (kk >> 2) * (kPBytes / 2) + (kk & 3) * 32,
                                                                  16, 1024);
                    const uint64_t qd =
                        p.q_mn ? make_sdesc_swz(sq + kk * 16 * p.q_span, BT * p.q_span, 8 * p.q_span, p.q_span)
                               : make_sdesc_sw128(sq + (kk >> 2) * (p.Nq * 128) + (kk & 3) * 32, 16, 1024);
                    mma_ss(tmem + buf * 128, pd, qd, idesc, (first && kk == 0) ? 0u : 1u);
                }
                tc_commit(&empty[sx]);
                if (last) {
                    tc_commit(&acc_full[buf]);
                    ++seg;
                }
                done = k + 1;
            }
            // TMEM is released only after every MMA has completed
            tc_commit(mma_done);
            mbar_drain(mma_done, 0);
            // every release commit has landed before the CTA exits, so none can reach the
            // shared memory of a CTA launched after it
            for (int k = max(0, done - S); k < done; ++k) mbar_drain(&empty[k % S], (k / S) & 1);
        }
    } else if (nu > 0) {
        // epilogue, warps 2-5: TMEM lane quadrant (warp % 4), one output row i per thread
        const int quad = warp & 3;
        const uint32_t lane_addr = uint32_t(quad * 32) << 16;
        int seg = 0;
        for (int k = 0; k < nu; ++k) {
            const int64_t u = u_begin + k;
            const bool last = (k == nu - 1) || ((u + 1) % ST == 0);
            if (!last) continue;
            const int buf = seg & 1;
            const int i = static_cast<int>(u / ST) * BI + quad * 32 + lane;
            if (!mbar_wait(&acc_full[buf], (seg >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            for (int c = 0; c < p.r; c += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + lane_addr + buf * 128 + c, v);
                tmem_wait_ld16(v);
                if (i < p.I) {
                    if (p.ld_j == 1) {             // row i holds r consecutive floats: 16-byte reductions
                        float *dst = p.out + int64_t(i) * p.ld_i + c;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (c + 4 * q < p.r)
                                red_add_v4(dst + 4 * q, p.scaling * __uint_as_float(v[4 * q]),
                                           p.scaling * __uint_as_float(v[4 * q + 1]),
                                           p.scaling * __uint_as_float(v[4 * q + 2]),
                                           p.scaling * __uint_as_float(v[4 * q + 3]));
                    } else {                       // ld_i == 1: the warp's 32 rows are contiguous
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (c + e < p.r)
                                atomicAdd(p.out + int64_t(c + e) * p.ld_j + i, p.scaling * __uint_as_float(v[e]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
            ++seg;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// [M, r] fp32 accumulator -> bf16 copy (save) and bf16 scaled copy (scaled)
__global__ void finalize_rank_kernel(const float *__restrict__ acc, int64_t n, float scaling,
                                     uint16_t *__restrict__ save, uint16_t *__restrict__ scaled) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        const float v = acc[i];
        if (save) {
            __nv_bfloat16 h = __float2bfloat16_rn(v);
            save[i] = *reinterpret_cast<uint16_t *>(&h);
        }
        if (scaled) {
            __nv_bfloat16 h = __float2bfloat16_rn(scaling * v);
            scaled[i] = *reinterpret_cast<uint16_t *>(&h);
        }
    }
}

}  // namespace skinny
}  // namespace qlora
