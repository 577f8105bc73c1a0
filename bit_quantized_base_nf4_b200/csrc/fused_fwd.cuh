// fused_fwd.cuh -- forward GEMM with NF4 dequant in the main loop (tcgen05, sm_100a).
//
// Computed per CTA tile (swap-AB orientation, W rows are the MMA M dimension):
//   D[n, m] = sum_k W'[n, k] X[m, k]  +  sum_j B[n, j] us[m, j]        n in 128 rows, m in BN tokens
// with us = bf16(scaling * X A^T) prepared by a side kernel, so the adapter is
// one or two extra K-chunks folded into the same TMEM accumulator.  Y = D^T.
//
// Pipeline per 64-wide K stage s:
//   producer (warp 0)   TMA load of the X tile [BN x 64] into the X ring (read by the MMA only)
//   producer (warp 3)   TMA load of the packed codes for four stages [128 rows x 128 bytes]
//                       into the code ring; every dequant group reads every chunk, in
//                       chunk order, so no barrier is waited on two phases ahead
//   dequant group s%4   (4 warps, thread = one W row, 64 weights) reads its row's 32
//                       code bytes, expands each byte through a shared-memory table
//                       byte -> (level[lo], level[hi]) as bf16x2, multiplies by the
//                       bf16 block scale and stores the 32 columns into TMEM slot s%4
//   MMA (warp 1)        four tcgen05.mma (K = 16) with A from TMEM, B (X) from smem
// Four dequant groups work on four consecutive stages at once, so the TMEM
// store and barrier latency of one stage overlaps the expansion of the next.
// Epilogue: the dequant warps read the accumulator back (tcgen05.ld) and write
// bf16 Y (or add fp32 partial sums into a split-K accumulator).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "scale_src.cuh"

namespace qlora {
namespace fwd {

constexpr int BM = 128;            // W rows per tile
constexpr int SX = 5;              // X ring stages (64 K each)
constexpr int SC = 2;              // code ring chunks (256 K each, read by all four groups)
constexpr int kGroups = 4;         // dequant groups = TMEM A slots (32 columns each)
constexpr int SA = kGroups;
constexpr int kDqWarps = 4 * kGroups;
constexpr int kThreads = 128 + 32 * kDqWarps;
constexpr int kCodeChunkBytes = BM * 128;     // 128 rows x 128 bytes (256 weights = 4 stages)
constexpr int kLutWords = 256 * 32;           // byte -> bf16x2, replicated per lane

struct Params {
    ScaleSrc sc;             // first-level scales of the weight's storage format
    const uint16_t *Blora;   // [N, r] bf16 or nullptr
    uint16_t *Y;             // [M, N] bf16 (split == 1)
    float *Yacc;             // [M, N] fp32 accumulator (split > 1), zeroed by the host
    int M, N, K, r, BN;
    int kb_per_split;        // 64-wide K stages per CTA along blockIdx.z
    float level[16];
};

__host__ __device__ constexpr int smem_bytes(int BN) {
    return 1024 /*align slack*/ + SX * BN * 128 + SC * kCodeChunkBytes + kLutWords * 4 + 512 /*barriers*/;
}
__host__ __device__ constexpr uint32_t tmem_cols(int BN) {
    // A slots at columns [0, 128), accumulator at [128, 128 + BN)
    return (128 + BN) <= 256 ? 256u : 512u;
}

__global__ void __launch_bounds__(kThreads, 1)
    fused_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmU, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int xsb = p.BN * 128;
    uint8_t *sX = smem;
    uint8_t *sC = sX + SX * xsb;
    uint32_t *sLut = reinterpret_cast<uint32_t *>(sC + SC * kCodeChunkBytes);
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

    if (threadIdx.x < 16) {
        float v = 0.f;  // constant-index reads keep the parameter block out of local memory
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (threadIdx.x == i) v = p.level[i];
        s_level[threadIdx.x] = v;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < SX; ++i) { mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], 1); }
        for (int i = 0; i < SC; ++i) { mbar_init(&c_full[i], 1); mbar_init(&c_empty[i], kDqWarps); }
        for (int i = 0; i < SA; ++i) { mbar_init(&a_full[i], 4); mbar_init(&a_empty[i], 1); }
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
    const uint32_t tmem_a = tmem;          // A slots: columns g*32 .. g*32+31
    const uint32_t tmem_acc = tmem + 128;  // accumulator: columns 128 .. 128+BN-1

    if (warp == 0) {
        // ---------------- X producer (us tiles for the adapter chunks)
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
        // ---------------- packed-code producer
        if (lane == 0) {
            tma_prefetch_desc(&tmC);
            // one 128-row x 128-byte tile (256 K, four stages) per chunk; kb_begin is a multiple of 4
            const int nchunk = (nmain + 3) / 4;
            int issued = 0;
            for (int c = 0; c < nchunk; ++c) {
                const int sc = c % SC;
                if (!mbar_wait(&c_empty[sc], ((c / SC) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&c_full[sc], kCodeChunkBytes);
                tma_load_2d(sC + sc * kCodeChunkBytes, &tmC, &c_full[sc], (kb_begin / 4 + c) * 128, n0);
                issued = c + 1;
            }
            for (int c = max(0, issued - SC); c < issued; ++c) mbar_drain(&c_full[c % SC], (c / SC) & 1);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(BM, p.BN, 0, 0);
            int done = 0;
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
                done = s + 1;
            }
            tc_commit(acc_full);
            // the accumulator (and TMEM) must not be released while MMAs are in flight
            mbar_drain(acc_full, 0);
            // every release commit has landed before the CTA exits, so none can reach the
            // shared memory of a CTA launched after it
            for (int s = max(0, done - SX); s < done; ++s) mbar_drain(&x_empty[s % SX], (s / SX) & 1);
            for (int s = max(0, done - SA); s < done; ++s) mbar_drain(&a_empty[s % SA], (s / SA) & 1);
        }
    } else if (warp >= 4) {
        // ---------------- dequant into TMEM, then epilogue
        const int dw = warp - 4;
        const int grp = dw >> 2;                  // stages s with s % kGroups == grp
        const int quad = warp & 3;                // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;         // W row within the tile
        const int n = n0 + row;
        const bool valid = n < p.N;
        const uint32_t lut = smem_u32(sLut) + lane * 4;
        const uint32_t lane_addr = uint32_t(quad * 32) << 16;
        // 32-byte code row, 32-byte swizzle: chunk c of row r sits at chunk c ^ ((r >> 2) & 1)
        const uint32_t code_row = smem_u32(sC) + row * 128;
        const uint32_t cswz = row & 7;
        bool ok = true;
        const int64_t row_block0 = int64_t(n) * KB + kb_begin;
        // the raw scale words of a 64-weight run (zero past the row end), converted only
        // when the stage is expanded
        auto load_scale = [&](int s, uint32_t &qv, float &dv) {
            qv = 0u;
            dv = 0.f;
            if (valid && s < nmain) scale_load(p.sc, row_block0 + s, qv, dv);
        };
        // block scales of this group's next three stages (12 stages of lookahead)
        uint32_t qa, qb, qc;
        float da, db, dc;
        load_scale(grp, qa, da);
        load_scale(grp + kGroups, qb, db);
        load_scale(grp + 2 * kGroups, qc, dc);

        for (int s = grp; s < total && ok; s += kGroups) {
            const int ci = s >> 2, sc = ci % SC, sa = s % SA;
            uint32_t out[32];
            if (s < nmain) {
                if (!mbar_wait(&c_full[sc], (ci / SC) & 1, abort_flag)) { ok = false; break; }
                const float sv = scale_of(p.sc, qa, da);
                qa = qb; da = db; qb = qc; db = dc;
                load_scale(s + 3 * kGroups, qc, dc);
                __nv_bfloat162 s2b = __float2bfloat162_rn(sv);
                const uint32_t s2 = *reinterpret_cast<uint32_t *>(&s2b);
                const uint32_t cbase = code_row + sc * kCodeChunkBytes;
                const uint32_t j0 = 2u * uint32_t(s & 3);
                const uint4 c0 = lds128(cbase + (((j0 + 0u) ^ cswz) << 4));
                const uint4 c1 = lds128(cbase + (((j0 + 1u) ^ cswz) << 4));
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8) {
#pragma unroll
                    for (int by = 0; by < 4; ++by) {
                        const uint32_t e = (words[w8] >> (8 * by)) & 0xFFu;
                        out[w8 * 4 + by] = bf16x2_mul(lds32_const(lut + (e << 7)), s2);
                    }
                }
                // released only once every code this thread read has been used: a release right
                // after the loads let the next copy overwrite codes still being read
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[sc]);
            } else {
                // adapter chunk: A operand = B_lora row n, elements e0 .. e0+63 (zero past r)
                const int e0 = (s - nmain) * 64;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    uint4 q = make_uint4(0, 0, 0, 0);
                    if (valid && e0 + v * 8 < p.r)
                        q = __ldg(reinterpret_cast<const uint4 *>(p.Blora + int64_t(n) * p.r + e0 + v * 8));
                    out[v * 4 + 0] = q.x; out[v * 4 + 1] = q.y; out[v * 4 + 2] = q.z; out[v * 4 + 3] = q.w;
                }
            }
            if (!mbar_wait(&a_empty[sa], ((s / SA) & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            tmem_st32_checked(tmem_a + lane_addr + sa * 32, out);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[sa]);
        }

        // ---------------- epilogue
        if (ok && mbar_wait(acc_full, 0, abort_flag)) {
            tc_fence_after();
            const int nchunks = p.BN / 16;
            for (int ch = grp; ch < nchunks; ch += kGroups) {
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
