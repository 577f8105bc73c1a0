// skinny_mma.cuh -- the rank-r products of the adapter on tcgen05 tensor cores.
//
//   D[j, i] = sum_t Aop(j, t) * Bop(i, t),   j < r (MMA M = 128, rows past r are zero),
//                                             i in tiles of 256 (MMA N), t split across CTAs
//   out[j * ld_row + i * ld_col] += scaling * D[j, i]      (fp32 atomics)
//
// with the operand of each side either K-major (t contiguous, a [rows, t] tensor)
// or MN-major (rows contiguous, a [t, rows] tensor), both staged by TMA in the
// 128-byte-swizzled layouts the MMA reads directly:
//   U^T = A_lora . X^T     Aop = A [r, K] K-major,        Bop = X [M, K] K-major
//   G^T = B_lora^T . dY^T  Aop = B [N, r] MN-major,       Bop = dY [M, N] K-major
//   dA  = G^T . X          Aop = G [M, r] MN-major,       Bop = X [M, K] MN-major
//   dB^T = U^T . dY        Aop = U [M, r] MN-major,       Bop = dY [M, N] MN-major
// These products stream the activation once from HBM; the tensor core keeps
// them memory-bound at any adapter rank up to 128.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {
namespace skinny {

constexpr int BI = 256;                  // columns i per tile (MMA N)
constexpr int SXS = 4;                   // pipeline stages (64 t each)
constexpr int kThreads = 256;            // warp 0 TMA, 1 MMA, 2 TMEM alloc, 4-7 epilogue
constexpr int kAStage = 128 * 128;       // 128 rows x 64 t bf16
constexpr int kBStage = BI * 128;        // 256 rows x 64 t bf16
constexpr int kStage = kAStage + kBStage;

struct Params {
    int T;                 // contraction length
    int I;                 // number of columns
    int r;                 // valid rows
    int stages_per_split;  // 64-wide t stages per CTA along blockIdx.y
    int a_mn, b_mn;        // operand majorness (0: K-major, 1: MN-major)
    float scaling;
    float *out;
    int64_t ld_row, ld_col;
};

__host__ __device__ constexpr int smem_bytes() { return 1024 + SXS * kStage + 512; }

__global__ void __launch_bounds__(kThreads, 1)
    skinny_mma_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SXS * kStage);
    uint64_t *full = bars, *empty = bars + SXS, *acc_full = bars + 2 * SXS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * BI;
    const int ST = (p.T + 63) / 64;
    const int s_begin = blockIdx.y * p.stages_per_split;
    const int s_end = min(ST, s_begin + p.stages_per_split);
    const int nst = s_end - s_begin;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SXS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && nst > 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            int issued = 0;
            for (int s = 0; s < nst; ++s) {
                const int sx = s % SXS;
                if (!mbar_wait(&empty[sx], ((s / SXS) & 1) ^ 1, abort_flag)) break;
                uint8_t *sa = smem + sx * kStage;
                uint8_t *sb = sa + kAStage;
                const int t0 = (s_begin + s) * 64;
                mbar_arrive_expect_tx(&full[sx], kStage);
                if (p.a_mn) {
                    tma_load_2d(sa, &tmA, &full[sx], 0, t0);
                    tma_load_2d(sa + 8192, &tmA, &full[sx], 64, t0);
                } else {
                    tma_load_2d(sa, &tmA, &full[sx], t0, 0);
                }
                if (p.b_mn) {
#pragma unroll
                    for (int q = 0; q < BI / 64; ++q) tma_load_2d(sb + 8192 * q, &tmB, &full[sx], i0 + 64 * q, t0);
                } else {
                    tma_load_2d(sb, &tmB, &full[sx], t0, i0);
                }
                issued = s + 1;
            }
            for (int s = max(0, issued - SXS); s < issued; ++s) mbar_drain(&full[s % SXS], (s / SXS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0 && nst > 0) {
            const uint32_t idesc = make_idesc_bf16(128, BI, p.a_mn, p.b_mn);
            for (int s = 0; s < nst; ++s) {
                const int sx = s % SXS;
                if (!mbar_wait(&full[sx], (s / SXS) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + sx * kStage);
                const uint32_t sb = sa + kAStage;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = p.a_mn ? make_sdesc_sw128(sa + kk * 2048, 8192, 1024)
                                               : make_sdesc_sw128(sa + kk * 32, 16, 1024);
                    const uint64_t bd = p.b_mn ? make_sdesc_sw128(sb + kk * 2048, 8192, 1024)
                                               : make_sdesc_sw128(sb + kk * 32, 16, 1024);
                    mma_ss(tmem, ad, bd, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty[sx]);
            }
            tc_commit(acc_full);
            mbar_drain(acc_full, 0);
        }
    } else if (warp >= 4 && nst > 0) {
        const int quad = warp & 3;
        if (quad * 32 < p.r && mbar_wait(acc_full, 0, abort_flag)) {
            tc_fence_after();
            const int j = quad * 32 + lane;
            const uint32_t taddr = tmem + (uint32_t(quad * 32) << 16);
            for (int ch = 0; ch < BI / 16; ++ch) {
                if (i0 + ch * 16 >= p.I) break;   // warp-uniform
                uint32_t v[16];
                tmem_ld16(taddr + ch * 16, v);
                tmem_wait_ld16(v);
                if (j < p.r) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int i = i0 + ch * 16 + e;
                        if (i < p.I)
                            atomicAdd(p.out + int64_t(j) * p.ld_row + int64_t(i) * p.ld_col,
                                      p.scaling * __uint_as_float(v[e]));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
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
