// fused_fwd.cuh -- forward GEMM with NF4 dequant in the main loop (tcgen05, sm_100a).
//
// Computed per CTA tile (swap-AB orientation, W rows are the MMA M dimension):
//   D[n, m] = sum_k W'[n, k] X[m, k]  +  sum_j B[n, j] us[m, j]        n in 128 rows, m in BN tokens
// with us = bf16(scaling * X A^T) prepared by a side kernel, so the adapter is
// one or two extra K-chunks folded into the same TMEM accumulator.  Y = D^T.
//
// Roles (384 threads):
//   warp 0      TMA producer for the X tile ring (and the us tiles of the adapter chunk)
//   warp 1      MMA issuer (one thread): tcgen05.mma with A from TMEM, B (X) from smem
//   warp 2      TMEM allocator
//   warp 3      TMA producer for the packed-code ring
//   warps 4-11  dequant: thread = one W row; 16 code bytes -> 32 bf16 via a
//               byte->bf16x2 lookup table in shared memory, times the bf16 block
//               scale, written straight into TMEM (the MMA's A operand);
//               then the epilogue: TMEM -> registers -> bf16 Y (or fp32 atomics
//               into a split-K accumulator).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {
namespace fwd {

constexpr int BM = 128;            // W rows per tile
constexpr int SX = 4;              // X/us smem ring stages (64 K each)
constexpr int SC = 2;              // code ring stages (256 K each)
constexpr int SA = 4;              // TMEM A stages (64 K = 32 columns each)
constexpr int kDqWarps = 8;
constexpr int kThreads = 128 + 32 * kDqWarps;
constexpr int kCodeStageBytes = BM * 128;     // 128 rows x 128 bytes (256 weights)
constexpr int kLutWords = 256 * 32;           // byte -> bf16x2, replicated per lane

struct Params {
    const uint8_t *scales;
    const float *scales2;
    const uint16_t *Blora;   // [N, r] bf16 or nullptr
    uint16_t *Y;             // [M, N] bf16 (split == 1)
    float *Yacc;             // [M, N] fp32 accumulator (split > 1), zeroed by the host
    int M, N, K, r, BN;
    int kb_per_split;        // 64-wide K stages per CTA along blockIdx.z
    float level[16];
};

__host__ __device__ constexpr int x_stage_bytes(int BN) { return BN * 128; }
__host__ __device__ constexpr int smem_bytes(int BN) {
    return 1024 /*align slack*/ + SX * x_stage_bytes(BN) + SC * kCodeStageBytes + kLutWords * 4 + 256;
}
__host__ __device__ constexpr uint32_t tmem_cols(int BN) {
    // A ring at columns [0, 128), accumulator at [128, 128 + BN)
    return (128 + BN) <= 256 ? 256u : 512u;
}

__global__ void __launch_bounds__(kThreads, 1)
    fused_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmU, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int xsb = x_stage_bytes(p.BN);
    uint8_t *sX = smem;
    uint8_t *sC = sX + SX * xsb;
    uint32_t *sLut = reinterpret_cast<uint32_t *>(sC + SC * kCodeStageBytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sLut + kLutWords);
    uint64_t *x_full = bars, *x_empty = bars + SX;
    uint64_t *c_full = bars + 2 * SX, *c_empty = c_full + SC;
    uint64_t *a_full = c_empty + SC, *a_empty = a_full + SA;
    uint64_t *acc_full = a_empty + SA;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *s_level = reinterpret_cast<float *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BM;
    const int m0 = blockIdx.y * p.BN;
    const int KB = p.K / 64;
    const int kb_begin = blockIdx.z * p.kb_per_split;
    const int kb_end = min(KB, kb_begin + p.kb_per_split);
    const bool last_split = kb_end == KB;
    const int LS = (last_split && p.r > 0) ? (p.r + 63) / 64 : 0;
    const int nmain = kb_end - kb_begin;
    const int total = nmain + LS;
    const uint32_t ncols = tmem_cols(p.BN);

    if (threadIdx.x < 16) s_level[threadIdx.x] = p.level[threadIdx.x];
    if (threadIdx.x == 0) {
        for (int i = 0; i < SX; ++i) { mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], 1); }
        for (int i = 0; i < SC; ++i) { mbar_init(&c_full[i], 1); mbar_init(&c_empty[i], kDqWarps); }
        for (int i = 0; i < SA; ++i) { mbar_init(&a_full[i], kDqWarps); mbar_init(&a_empty[i], 1); }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    __syncthreads();
    // byte -> (level[lo nibble], level[hi nibble]) as bf16x2, replicated for each lane
    for (int i = threadIdx.x; i < kLutWords; i += blockDim.x) {
        const int e = i >> 5;
        __nv_bfloat162 v = __floats2bfloat162_rn(s_level[e & 15], s_level[e >> 4]);
        sLut[i] = *reinterpret_cast<uint32_t *>(&v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_a = tmem;          // A stages: columns sa*32 .. sa*32+31
    const uint32_t tmem_acc = tmem + 128;  // accumulator: columns 128 .. 128+BN-1

    if (warp == 0) {
        // ---------------- X / us producer
        if (lane == 0) {
            tma_prefetch_desc(&tmX);
            if (LS) tma_prefetch_desc(&tmU);
            int issued = 0;
            for (int s = 0; s < total; ++s) {
                const int sx = s % SX;
                if (!mbar_wait(&x_empty[sx], ((s / SX) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&x_full[sx], xsb);
                if (s < nmain)
                    tma_load_2d(sX + sx * xsb, &tmX, &x_full[sx], (kb_begin + s) * 64, m0);
                else
                    tma_load_2d(sX + sx * xsb, &tmU, &x_full[sx], (s - nmain) * 64, m0);
                issued = s + 1;
            }
            // never leave a copy in flight into this CTA's shared memory
            for (int s = max(0, issued - SX); s < issued; ++s) mbar_drain(&x_full[s % SX], (s / SX) & 1);
        }
    } else if (warp == 3) {
        // ---------------- packed-code producer (256 weights per row per stage)
        if (lane == 0) {
            tma_prefetch_desc(&tmC);
            const int c_begin = kb_begin / 4;
            const int c_end = (kb_end + 3) / 4;
            int issued = 0;
            for (int c = c_begin; c < c_end; ++c) {
                const int i = c - c_begin, sc = i % SC;
                if (!mbar_wait(&c_empty[sc], ((i / SC) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&c_full[sc], kCodeStageBytes);
                tma_load_2d(sC + sc * kCodeStageBytes, &tmC, &c_full[sc], c * 128, n0);
                issued = i + 1;
            }
            for (int i = max(0, issued - SC); i < issued; ++i) mbar_drain(&c_full[i % SC], (i / SC) & 1);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(BM, p.BN, 0, 0);
            for (int s = 0; s < total; ++s) {
                const int sx = s % SX, sa = s % SA;
                if (!mbar_wait(&x_full[sx], (s / SX) & 1, abort_flag)) break;
                if (!mbar_wait(&a_full[sa], (s / SA) & 1, abort_flag)) break;
                tc_fence_after();
                const int nk = (s < nmain) ? 4 : min(4, (p.r - (s - nmain) * 64 + 15) / 16);
                const uint32_t xbase = smem_u32(sX + sx * xsb);
                for (int kk = 0; kk < nk; ++kk) {
                    const uint64_t bdesc = make_sdesc_sw128(xbase + kk * 32, 16, 1024);
                    mma_ts(tmem_acc, tmem_a + sa * 32 + kk * 8, bdesc, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&x_empty[sx]);
                tc_commit(&a_empty[sa]);
            }
            tc_commit(acc_full);
            // the accumulator (and TMEM) must not be released while MMAs are in flight
            mbar_drain(acc_full, 0);
        }
    } else if (warp >= 4) {
        // ---------------- dequant into TMEM, then epilogue
        const int dw = warp - 4;
        const int half = dw >> 2;                 // which 32 weights of each 64-block
        const int quad = warp & 3;                // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;         // W row within the tile
        const int n = n0 + row;
        const bool valid = n < p.N;
        const uint32_t lut = smem_u32(sLut) + lane * 4;
        const uint32_t sCu = smem_u32(sC);
        const uint32_t lane_addr = uint32_t(quad * 32) << 16;
        bool ok = true;
        const int64_t row_block0 = int64_t(n) * KB;
        // block scale of the next main stage, loaded one stage ahead
        uint32_t q_next = 0;
        float d_next = 0.f;
        if (valid && nmain > 0) {
            const int64_t b = row_block0 + kb_begin;
            q_next = __ldg(p.scales + b);
            d_next = __ldg(p.scales2 + (b >> 8));
        }

        for (int s = 0; s < total && ok; ++s) {
            const int sa = s % SA;
            uint32_t out[16];
            if (s < nmain) {
                const int kb = kb_begin + s;
                const int ci = kb / 4 - kb_begin / 4;
                const int sc = ci % SC;
                if ((s == 0) || (kb % 4 == 0)) {
                    if (!mbar_wait(&c_full[sc], (ci / SC) & 1, abort_flag)) { ok = false; break; }
                }
                const float sv = __fmul_rn(static_cast<float>(q_next), d_next);
                if (valid && s + 1 < nmain) {
                    const int64_t b = row_block0 + kb + 1;
                    q_next = __ldg(p.scales + b);
                    d_next = __ldg(p.scales2 + (b >> 8));
                }
                __nv_bfloat162 s2b = __float2bfloat162_rn(sv);
                const uint32_t s2 = *reinterpret_cast<uint32_t *>(&s2b);
                const int j = 2 * (kb & 3) + half;            // 16-byte chunk within the 128-byte row
                const uint4 cw = lds128(sCu + sc * kCodeStageBytes + row * 128 + ((j ^ (row & 7)) << 4));
                const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) {
#pragma unroll
                    for (int by = 0; by < 4; ++by) {
                        const uint32_t e = (words[w4] >> (8 * by)) & 0xFFu;
                        out[w4 * 4 + by] = bf16x2_mul(lds32(lut + (e << 7)), s2);
                    }
                }
                if ((kb % 4 == 3) || (kb == kb_end - 1)) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&c_empty[sc]);
                }
            } else {
                // adapter chunk: A operand = B_lora row n, elements e0 .. e0+31 (zero past r)
                const int e0 = (s - nmain) * 64 + half * 32;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 q = make_uint4(0, 0, 0, 0);
                    if (valid && e0 + v * 8 < p.r)
                        q = __ldg(reinterpret_cast<const uint4 *>(p.Blora + int64_t(n) * p.r + e0 + v * 8));
                    out[v * 4 + 0] = q.x; out[v * 4 + 1] = q.y; out[v * 4 + 2] = q.z; out[v * 4 + 3] = q.w;
                }
            }
            if (!mbar_wait(&a_empty[sa], ((s / SA) & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            tmem_st16(tmem_a + lane_addr + sa * 32 + half * 16, out);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[sa]);
        }

        // ---------------- epilogue
        if (ok && mbar_wait(acc_full, 0, abort_flag)) {
            tc_fence_after();
            const int nchunks = p.BN / 16;
            for (int ch = half; ch < nchunks; ch += 2) {
                uint32_t v[16];
                tmem_ld16(tmem_acc + lane_addr + ch * 16, v);
                tmem_wait_ld16(v);
                if (valid) {
                    const int mb = m0 + ch * 16;
                    if (p.Yacc) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (mb + i < p.M) atomicAdd(p.Yacc + int64_t(mb + i) * p.N + n, __uint_as_float(v[i]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (mb + i < p.M) {
                                __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[i]));
                                p.Y[int64_t(mb + i) * p.N + n] = *reinterpret_cast<uint16_t *>(&h);
                            }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

}  // namespace fwd
}  // namespace qlora
