// fused_bwd.cuh -- input-gradient GEMM with NF4 dequant in the main loop (tcgen05, sm_100a).
//
// Per CTA tile (swap-AB: rows of dX^T are the MMA M dimension):
//   D[k, m] = sum_n W'[n, k] dY[m, n]  +  sum_j A[j, k] gs[m, j]      k in 128 columns of W0, m in BN tokens
// with gs = bf16(scaling * dY B) from a side kernel; dX = D^T.  The weight is
// consumed transposed relative to the forward: its 64-blocks run along the
// MMA M dimension, so the dequant warps write each tile of W' [64 n x 128 k]
// into shared memory in the MN-major 128-byte-swizzled layout (k contiguous)
// and the MMA reads A from there.  B (dY) arrives by TMA, K-major.
//
// Roles (640 threads): warp 0 TMA producer of the dY ring (read by the MMA only),
// warp 3 TMA producer of the packed-code ring (slot s % 8 is read only by
// dequant group s % 4, in stage order), warp 1 MMA issuer, warp 2 TMEM
// allocator, warps 4-19 four dequant groups (group g takes stages s % 4 == g,
// thread = one 64-block of a contraction row), then the epilogue.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {
namespace bwd {

constexpr int BM = 128;                 // columns k of W0 per tile
constexpr int SX = 3;                   // dY ring (64 n each)
constexpr int SC = 8;                   // code ring (a multiple of kGroups)
constexpr int kGroups = 4;              // dequant groups = smem A slots
constexpr int SA = kGroups;             // A ring in smem (W'^T tiles)
constexpr int kDqWarps = 4 * kGroups;
constexpr int kThreads = 128 + 32 * kDqWarps;
constexpr int kCodeStageBytes = 64 * 64;     // 64 rows x 64 bytes
constexpr int kAStageBytes = 64 * 128 * 2;   // 64 n x 128 k bf16
constexpr int kLutWords = 256 * 32;

struct Params {
    const uint8_t *scales;
    const float *scales2;
    const uint16_t *Alora;   // [r, K] bf16 or nullptr
    uint16_t *dX;            // [M, K] bf16 (split == 1)
    float *dXacc;            // [M, K] fp32 accumulator (split > 1), zeroed by the host
    int M, N, K, r, BN;
    int nb_per_split;        // 64-wide n stages per CTA along blockIdx.z
    float level[16];
};

__host__ __device__ constexpr int smem_bytes(int BN) {
    return 1024 + SX * BN * 128 + SC * kCodeStageBytes + SA * kAStageBytes + kLutWords * 4 + 512 /*barriers*/;
}
__host__ __device__ constexpr uint32_t tmem_cols(int BN) { return BN <= 32 ? 32u : BN <= 64 ? 64u : BN <= 128 ? 128u : 256u; }

__global__ void __launch_bounds__(kThreads, 1)
    fused_bwd_dx_kernel(const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmC,
                        const __grid_constant__ CUtensorMap tmG, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int ysb = p.BN * 128;
    uint8_t *sY = smem;
    uint8_t *sA = sY + SX * ysb;
    uint8_t *sC = sA + SA * kAStageBytes;
    uint32_t *sLut = reinterpret_cast<uint32_t *>(sC + SC * kCodeStageBytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sLut + kLutWords);
    uint64_t *y_full = bars, *y_empty = bars + SX;
    uint64_t *c_full = bars + 2 * SX, *c_empty = c_full + SC;
    uint64_t *a_full = c_empty + SC, *a_empty = a_full + SA;
    uint64_t *acc_full = a_empty + SA;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *s_level = reinterpret_cast<float *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = blockIdx.x * BM;
    const int m0 = blockIdx.y * p.BN;
    const int KB = p.K / 64;
    const int NB = (p.N + 63) / 64;
    const int nb_begin = blockIdx.z * p.nb_per_split;
    const int nb_end = min(NB, nb_begin + p.nb_per_split);
    const bool last_split = nb_end == NB;
    const int LS = (last_split && p.r > 0) ? (p.r + 63) / 64 : 0;
    const int nmain = nb_end - nb_begin;
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
        for (int i = 0; i < SX; ++i) { mbar_init(&y_full[i], 1); mbar_init(&y_empty[i], 1); }
        for (int i = 0; i < SC; ++i) { mbar_init(&c_full[i], 1); mbar_init(&c_empty[i], 4); }
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
    for (int i = threadIdx.x; i < kLutWords; i += blockDim.x) {
        const int e = i >> 5;
        __nv_bfloat162 v = __floats2bfloat162_rn(s_level[e & 15], s_level[e >> 4]);
        sLut[i] = *reinterpret_cast<uint32_t *>(&v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_acc = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmY);
            if (LS) tma_prefetch_desc(&tmG);
            int issued = 0;
            for (int s = 0; s < total; ++s) {
                const int sx = s % SX;
                if (!mbar_wait(&y_empty[sx], ((s / SX) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&y_full[sx], ysb);
                if (s < nmain)
                    tma_load_2d(sY + sx * ysb, &tmY, &y_full[sx], (nb_begin + s) * 64, m0);
                else
                    tma_load_2d(sY + sx * ysb, &tmG, &y_full[sx], (s - nmain) * 64, m0);
                issued = s + 1;
            }
            for (int s = max(0, issued - SX); s < issued; ++s) mbar_drain(&y_full[s % SX], (s / SX) & 1);
        }
    } else if (warp == 3) {
        if (lane == 0) {
            tma_prefetch_desc(&tmC);
            int issued = 0;
            for (int s = 0; s < nmain; ++s) {
                const int sc = s % SC;
                if (!mbar_wait(&c_empty[sc], ((s / SC) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&c_full[sc], kCodeStageBytes);
                // rows n = 64*(nb_begin+s) .., bytes k0/2 .. k0/2+63
                tma_load_2d(sC + sc * kCodeStageBytes, &tmC, &c_full[sc], k0 / 2, (nb_begin + s) * 64);
                issued = s + 1;
            }
            for (int s = max(0, issued - SC); s < issued; ++s) mbar_drain(&c_full[s % SC], (s / SC) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(BM, p.BN, 1, 0);
            int done = 0;
            for (int s = 0; s < total; ++s) {
                const int sx = s % SX, sa = s % SA;
                if (!mbar_wait(&y_full[sx], (s / SX) & 1, abort_flag)) break;
                if (!mbar_wait(&a_full[sa], (s / SA) & 1, abort_flag)) break;
                tc_fence_after();
                const int nk = (s < nmain) ? 4 : min(4, (p.r - (s - nmain) * 64 + 15) / 16);
                const uint32_t ybase = smem_u32(sY + sx * ysb);
                const uint32_t abase = smem_u32(sA + sa * kAStageBytes);
                for (int kk = 0; kk < nk; ++kk) {
                    const uint64_t adesc = make_sdesc_sw128(abase + kk * 2048, 8192, 1024);
                    const uint64_t bdesc = make_sdesc_sw128(ybase + kk * 32, 16, 1024);
                    mma_ss(tmem_acc, adesc, bdesc, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&y_empty[sx]);
                tc_commit(&a_empty[sa]);
                done = s + 1;
            }
            tc_commit(acc_full);
            mbar_drain(acc_full, 0);
            // every release commit has landed before the CTA exits, so none can reach the
            // shared memory of a CTA launched after it
            for (int s = max(0, done - SX); s < done; ++s) mbar_drain(&y_empty[s % SX], (s / SX) & 1);
            for (int s = max(0, done - SA); s < done; ++s) mbar_drain(&a_empty[s % SA], (s / SA) & 1);
        }
    } else if (warp >= 4) {
        // thread = (contraction row nl, k half h): one 64-block of W0 row n
        const int dw = warp - 4;
        const int grp = dw >> 2;                    // stages s with s % kGroups == grp
        const int wi = dw & 3;
        const int nl = (wi & 1) * 32 + lane;        // contraction row within the stage (0..63)
        const int h = wi >> 1;                      // k half: columns k0 + 64h ..
        const int kblk = k0 / 64 + h;               // 64-block index along the row
        const bool kvalid = kblk < KB;
        const uint32_t lut = smem_u32(sLut) + lane * 4;
        const uint32_t sAu = smem_u32(sA);
        // 64-byte code rows, 64-byte swizzle: chunk c of row r sits at chunk c ^ ((r >> 1) & 3)
        const uint32_t c_row = smem_u32(sC) + nl * 64;
        const uint32_t c_swz = (nl >> 1) & 3;
        const uint32_t a_off = h * 8192 + nl * 128;
        bool ok = true;

        auto load_scale = [&](int s, uint32_t &qv, float &dv) {
            const int n = (nb_begin + s) * 64 + nl;
            qv = 0;
            dv = 0.f;
            if (kvalid && s < nmain && n < p.N) {
                const int64_t b = int64_t(n) * KB + kblk;
                qv = __ldg(p.scales + b);
                dv = __ldg(p.scales2 + (b >> 8));
            }
        };
        // block scales of this group's next three stages (12 stages of lookahead)
        uint32_t qa, qb, qc;
        float da, db, dc;
        load_scale(grp, qa, da);
        load_scale(grp + kGroups, qb, db);
        load_scale(grp + 2 * kGroups, qc, dc);

        for (int s = grp; s < total && ok; s += kGroups) {
            const int sc = s % SC, sa = s % SA;
            uint32_t out[32];
            if (s < nmain) {
                if (!mbar_wait(&c_full[sc], (s / SC) & 1, abort_flag)) { ok = false; break; }
                const float sv = __fmul_rn(static_cast<float>(qa), da);
                qa = qb; da = db; qb = qc; db = dc;
                load_scale(s + 3 * kGroups, qc, dc);
                __nv_bfloat162 s2b = __float2bfloat162_rn(sv);
                const uint32_t s2 = *reinterpret_cast<uint32_t *>(&s2b);
                const uint32_t cbase = c_row + sc * kCodeStageBytes;
                const uint4 c0 = lds128(cbase + (((2u * h + 0u) ^ c_swz) << 4));
                const uint4 c1 = lds128(cbase + (((2u * h + 1u) ^ c_swz) << 4));
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[sc]);
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8) {
#pragma unroll
                    for (int by = 0; by < 4; ++by) {
                        const uint32_t e = (words[w8] >> (8 * by)) & 0xFFu;
                        out[w8 * 4 + by] = bf16x2_mul(lds32(lut + (e << 7)), s2);
                    }
                }
            } else {
                // adapter chunk: row j of A [r, K], 64 k starting at k0 + 64h (zero past r / K)
                const int j = (s - nmain) * 64 + nl;
                const int kk0 = k0 + h * 64;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (j < p.r && kk0 < p.K)
                        w = __ldg(reinterpret_cast<const uint4 *>(p.Alora + int64_t(j) * p.K + kk0 + v * 8));
                    out[v * 4 + 0] = w.x; out[v * 4 + 1] = w.y; out[v * 4 + 2] = w.z; out[v * 4 + 3] = w.w;
                }
            }
            if (!mbar_wait(&a_empty[sa], ((s / SA) & 1) ^ 1, abort_flag)) { ok = false; break; }
            const uint32_t abase = sAu + sa * kAStageBytes + a_off;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t chunk = uint32_t(i) ^ uint32_t(nl & 7);
                sts128(abase + (chunk << 4), make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[sa]);
        }

        // epilogue: warp quadrant (warp & 3) owns TMEM lanes = k rows
        if (ok && mbar_wait(acc_full, 0, abort_flag)) {
            tc_fence_after();
            const int quad = warp & 3;
            const int row = quad * 32 + lane;
            const int k = k0 + row;
            const uint32_t lane_addr = uint32_t(quad * 32) << 16;
            const int nchunks = p.BN / 16;
            for (int ch = grp; ch < nchunks; ch += kGroups) {
                uint32_t v[16];
                tmem_ld16(tmem_acc + lane_addr + ch * 16, v);
                tmem_wait_ld16(v);
                if (k < p.K) {
                    const int mb = m0 + ch * 16;
                    if (p.dXacc) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (mb + i < p.M) atomicAdd(p.dXacc + int64_t(mb + i) * p.K + k, __uint_as_float(v[i]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (mb + i < p.M) {
                                __nv_bfloat16 hv = __float2bfloat16_rn(__uint_as_float(v[i]));
                                p.dX[int64_t(mb + i) * p.K + k] = *reinterpret_cast<uint16_t *>(&hv);
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
        tmem_dealloc(tmem_acc, ncols);
    }
}

}  // namespace bwd
}  // namespace qlora
