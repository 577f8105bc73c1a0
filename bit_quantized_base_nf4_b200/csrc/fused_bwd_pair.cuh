// fused_bwd_pair.cuh -- input-gradient GEMM with NF4 dequant, on CTA pairs (tcgen05 cta_group::2).
//
//   D[k, m] = sum_n W'[n, k] dY[m, n]  +  sum_j A[j, k] gs[m, j]     k in 256 columns of W0
//                                                                      (128 per CTA), m in BN tokens
// with gs = bf16(scaling * dY B) from the rank-r side kernel; dX = D^T.
//
// Two CTAs on two SMs form one 256-k x BN-token tile.  Each CTA dequantizes the
// weight for its own 128 k into its own shared memory, as the MN-major
// (k contiguous) 128-byte-swizzled A operand, and loads only its half of the
// token tile (BN/2 rows of dY); one tcgen05.mma.cta_group::2 issued by the even
// CTA reads both CTAs' A halves and B halves.  A 512-token tile uses two
// accumulators of 256 columns (the whole TMEM), tokens 0..255 and 256..511: each
// stage's A tile then feeds twice the MMA work, which halves the dequant, the A
// stores and their fences per flop.
//
// The MMA issue is effectively synchronous with the issuing thread, so the MMA
// thread does one barrier wait and one commit per stage of 64 n (four MMAs of
// 256 x BN x 16 per accumulator): it waits on a_full of the stage's slot s % kS,
// which the even CTA's dequant warps arrive on only after they have seen the stage's
// dY tile land, and commits to free[s % kS], which releases the dY slot and the A
// slot of the stage in both CTAs.
//   producer (warp 0)    one TMA instruction per stage: this CTA's dY half,
//                        counted on the even CTA's y_full
//   producer (warp 3)    packed codes, 64 kCS n rows x 128 k (kCS stages) per TMA
//                        instruction
//   dequant group s % 4  (4 warps, thread = one 64-block: a row n and a 64-k half)
//                        expands the stage's weights ahead of its slot
//                        expands the block through the register level tables
//                        (codes4_to_bf16x2) times the bf16 block scale, stores it
//                        swizzled into A slot s % kS, then arrives on a_full
//   MMA (warp 1, even)   four tcgen05.mma (K = 16) per accumulator, A and B from
//                        shared memory
// Commits are multicast to both CTAs (free, acc_full); each CTA then reads back
// its own 128 x BN accumulator and writes dX, or, when the contraction over n is
// split across blockIdx.z (few output tiles: small M), adds it into an fp32
// accumulator that a finalize kernel rounds to bf16.
//
// kQ8 selects the Q8_0 route (GGUF page, sections 1.1 and 2.2): one int8 code per
// weight and an fp16 scale per 32 weights; a code chunk row then holds 128 bytes
// (128-byte swizzle) and the dequant threads expand int8 x fp16 scale in registers.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "scale_src.cuh"

namespace qlora {
namespace bwdp {

constexpr int BM = 128;                       // k columns of W0 per CTA (256 per pair)
constexpr int SC = 2;                         // code ring chunks (kCS stages each)
// kS stage slots (dY ring = A ring) and kS dequant groups of four warps: stage s goes to
// slot and group s % kS, so that a group never reaches a slot's barriers a phase early.
// A code chunk holds kCS stages (64 n rows each).
__host__ __device__ constexpr int threads_for(int kS) { return 128 + 128 * kS; }
__host__ __device__ constexpr int chunk_rows(int kCS) { return 64 * kCS; }
constexpr int kAStageBytes = 64 * BM * 2;     // 64 n x 128 k bf16
constexpr int kLutWords = 256 * 32;

struct Params {
    ScaleSrc sc;             // first-level scales of the weight's storage format (4-bit codes)
    const uint16_t *d8;      // Q8_0: fp16 scale of each 32 weights, [N, K/32]
    const uint16_t *Alora;   // [r, K] bf16 or nullptr
    uint16_t *dX;            // [M, K] bf16 (one split)
    float *dXacc;            // [M, K] fp32 accumulator, zeroed by the host (several splits), or nullptr
    int M, N, K, r, BN;      // BN: tokens per pair tile, a multiple of 32 up to 256, or 512
    int nb_per_split;        // 64-n stages per split along blockIdx.z (a multiple of 4)
    int raster_mode, raster_group;   // tile order of the pairs (raster_tile)
    float level[16];
};

// code rows of 64 (4-bit) or 128 (8-bit) bytes
__host__ __device__ constexpr int smem_bytes(int BN, bool q8, int kS, int kCS) {
    return 1024 + kS * (BN / 2) * 128 + kS * kAStageBytes + SC * chunk_rows(kCS) * (q8 ? 128 : 64) + 512;
}
__host__ __device__ constexpr uint32_t tmem_cols(int BN) {
    return BN <= 32 ? 32u : BN <= 64 ? 64u : BN <= 128 ? 128u : BN <= 256 ? 256u : 512u;
}

template <bool kQ8, int kS, int kCS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_for(kS), 1)
    fused_bwd_pair_kernel(const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmC,
                          const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmD,
                          const Params p) {
    constexpr int kGroups = kS;
    // Group g reads code chunk s / kCS of each stage s = g (mod kS) and waits on its slot's
    // c_full by parity.  A parity wait is only sound when the waiter saw the slot's
    // previous phase complete, so every group must read every chunk: kCS >= kS.  (With
    // two-stage chunks and three groups a group skips a chunk, and its next wait on that
    // slot could pass while the skipped chunk was still in flight.)
    static_assert(kCS >= kS, "every dequant group must read every code chunk");
    constexpr int kCB = chunk_rows(kCS) * (kQ8 ? 128 : 64);   // one code chunk in shared memory
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int half_bn = p.BN / 2;
    const int ysb = half_bn * 128;                // this CTA's dY half for one stage
    const int nacc = p.BN > 256 ? 2 : 1;          // accumulators of bna tokens each
    const int bna = p.BN > 256 ? 256 : p.BN;
    const int yab = (bna / 2) * 128;              // this CTA's share of one accumulator's dY, per stage
    uint8_t *sY = smem;
    uint8_t *sA = sY + kS * ysb;
    uint8_t *sC = sA + kS * kAStageBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sC + SC * kCB);
    uint64_t *y_full = bars, *free_b = bars + kS;
    uint64_t *c_full = bars + 2 * kS, *c_empty = c_full + SC;
    uint64_t *a_full = c_empty + SC;
    uint64_t *acc_full = a_full + kS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *s_level = reinterpret_cast<float *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();      // 0: even CTA (issues the MMAs), 1: its peer
    // this pair's tile: 256 k columns x BN tokens, in the L2-friendly order of raster_tile
    int wt, tt;
    raster_tile(blockIdx.y * (gridDim.x / 2) + (blockIdx.x >> 1), gridDim.x / 2, gridDim.y, p.raster_mode,
                p.raster_group, wt, tt);
    const int k0 = (2 * wt + int(rank)) * BM;
    const int m0 = tt * p.BN;
    const int my_m0 = m0 + int(rank) * (bna / 2);   // this CTA's tokens: my_m0 + 256 j + [0, bna / 2)
    const int KB = p.K / 64;
    const int NB_all = (p.N + 63) / 64;
    const int nb_begin = blockIdx.z * p.nb_per_split;          // first 64-n stage of this split
    const int NB = min(NB_all, nb_begin + p.nb_per_split) - nb_begin;   // main stages (64 n each)
    // adapter stages (64 j each), on the last split only
    const int LS = (p.r > 0 && nb_begin + NB == NB_all) ? (p.r + 63) / 64 : 0;
    const int total = NB + LS;
    const int nchunk = (NB + kCS - 1) / kCS;
    const uint32_t ncols = tmem_cols(p.BN);

    if (threadIdx.x < 16) {
        float v = 0.f;  // constant-index reads keep the parameter block out of local memory
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (threadIdx.x == i) v = p.level[i];
        s_level[threadIdx.x] = v;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kS; ++i) {
            mbar_init(&y_full[i], 1);
            mbar_init(&free_b[i], 1);
            mbar_init(&a_full[i], 8);             // 4 warps x 2 CTAs
        }
        // a chunk is read by the groups of its kCS stages (four warps each)
        for (int i = 0; i < SC; ++i) { mbar_init(&c_full[i], 1); mbar_init(&c_empty[i], 4 * kCS); }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc_pair(tmem_slot, ncols);
        tmem_relinquish_pair();
    }
    __syncthreads();
    tc_fence_before();
    // both CTAs' barriers are initialised before either signals the other's
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_acc = *tmem_slot;

    if (warp == 0) {
        // ---------------- dY producer
        if (lane == 0) {
            tma_prefetch_desc(&tmY);
            if (LS) tma_prefetch_desc(&tmG);
            int issued = 0;
            for (int s = 0; s < total; ++s) {
                const int sx = s % kS;
                if (!mbar_wait_cluster(&free_b[sx], ((s / kS) & 1) ^ 1, abort_flag)) break;
                const uint32_t bar0 = mapa_shared(smem_u32(&y_full[sx]), 0);
                if (rank == 0) mbar_arrive_expect_tx(&y_full[sx], 2 * ysb);
                for (int j = 0; j < nacc; ++j) {
                    if (s < NB)
                        tma_load_2d_pair(sY + sx * ysb + j * yab, &tmY, bar0, (nb_begin + s) * 64, my_m0 + 256 * j);
                    else
                        tma_load_2d_pair(sY + sx * ysb + j * yab, &tmG, bar0, (s - NB) * 64, my_m0 + 256 * j);
                }
                issued = s + 1;
            }
            // the even CTA sees both CTAs' copies complete on its barriers
            if (rank == 0)
                for (int s = max(0, issued - kS); s < issued; ++s) mbar_drain(&y_full[s % kS], (s / kS) & 1);
            // producer tail: the release commits of the last stages land on this CTA's barriers
            // before it exits, so none can reach the shared memory of a CTA launched after it
            for (int s = max(0, issued - kS); s < issued; ++s) mbar_drain_cluster(&free_b[s % kS], (s / kS) & 1);
        }
    } else if (warp == 3) {
        // ---------------- packed-code producer (local to each CTA)
        if (lane == 0) {
            tma_prefetch_desc(&tmC);
            int issued = 0;
            for (int c = 0; c < nchunk; ++c) {
                const int sc = c % SC;
                if (!mbar_wait(&c_empty[sc], ((c / SC) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&c_full[sc], kCB);
                // rows n = 64 (nb_begin + kCS c) .., bytes k0/2 .. k0/2 + 63 (4-bit) or k0 .. k0 + 127 (8-bit)
                tma_load_2d(sC + sc * kCB, &tmC, &c_full[sc], kQ8 ? k0 : k0 / 2, nb_begin * 64 + c * chunk_rows(kCS));
                issued = c + 1;
            }
            for (int c = max(0, issued - SC); c < issued; ++c) mbar_drain(&c_full[c % SC], (c / SC) & 1);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (even CTA only)
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = make_idesc_bf16(2 * BM, bna, 1, 0);
            for (int s = 0; s < total; ++s) {
                const int g = s % kS;
                if (!mbar_wait_cluster(&a_full[g], (s / kS) & 1, abort_flag)) break;
                tc_fence_after();
                const int nk = (s < NB) ? 4 : min(4, (p.r - (s - NB) * 64 + 15) / 16);
                const uint32_t ybase = smem_u32(sY + g * ysb);
                const uint32_t abase = smem_u32(sA + g * kAStageBytes);
                for (int kk = 0; kk < nk; ++kk) {
                    const uint64_t adesc = make_sdesc_sw128(abase + kk * 2048, 8192, 1024);
                    for (int j = 0; j < nacc; ++j) {
                        const uint64_t bdesc = make_sdesc_sw128(ybase + j * yab + kk * 32, 16, 1024);
                        mma_ss_pair(tmem_acc + 256 * j, adesc, bdesc, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc_commit_pair(&free_b[g]);
            }
            tc_commit_pair(acc_full);
            mbar_drain(acc_full, 0);
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
        const LevelBytes lvb = level_bytes(*reinterpret_cast<const float (*)[16]>(s_level));
        const uint32_t sAu = smem_u32(sA);
        // 64-byte code rows, 64-byte swizzle: 16-byte chunk c of row q sits at chunk c ^ ((q >> 1) & 3);
        // stage rows start at multiples of 64, so the phase depends on nl only
        const uint32_t c_swz = (nl >> 1) & 3;
        const uint32_t a_off = h * 8192 + nl * 128;
        bool ok = true;

        // the raw scale words of this thread's 64-weight run in stage s (zero past the end);
        // they are converted only when the stage is expanded, three group iterations later
        auto load_scale = [&](int s, uint32_t &qv, float &dv) {
            const int n = (nb_begin + s) * 64 + nl;
            qv = 0u;
            dv = 0.f;
            if (!kQ8 && kvalid && s < NB && n < p.N) scale_load(p.sc, int64_t(n) * KB + kblk, qv, dv);
        };
        // Q8_0: the two fp16 scales of this thread's 64 weights of stage s (as one word)
        auto load_d8 = [&](int s) -> uint32_t {
            const int n = (nb_begin + s) * 64 + nl;
            if (!kQ8 || !kvalid || s >= NB || n >= p.N) return 0u;
            return __ldg(reinterpret_cast<const uint32_t *>(p.d8 + int64_t(n) * (p.K / 32)) + kblk);
        };
        uint32_t ua = load_d8(grp), ub = load_d8(grp + kGroups), uc = load_d8(grp + 2 * kGroups);
        // block scales of this group's next three stages
        uint32_t qa, qb, qc;
        float da, db, dc;
        load_scale(grp, qa, da);
        load_scale(grp + kGroups, qb, db);
        load_scale(grp + 2 * kGroups, qc, dc);

        for (int s = grp; s < total && ok; s += kGroups) {
            const int g = s % kS;                   // stage slot
            uint32_t out[32];
            if (kQ8 && s < NB) {
                const int ci = s / kCS, sc = ci % SC;
                if (!mbar_wait(&c_full[sc], (ci / SC) & 1, abort_flag)) { ok = false; break; }
                const uint32_t dd = ua;
                ua = ub; ub = uc;
                uc = load_d8(s + 3 * kGroups);
                // 128-byte code rows, 128-byte swizzle: 16-byte chunk j of row q sits at chunk j ^ (q & 7)
                const uint32_t cbase = smem_u32(sC) + sc * kCB + ((s % kCS) * 64 + nl) * 128;
                uint4 cv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) cv[i] = lds128(cbase + (((4u * h + uint32_t(i)) ^ uint32_t(nl & 7)) << 4));
                const float d_lo = __half2float(__ushort_as_half(static_cast<unsigned short>(dd & 0xFFFFu)));
                const float d_hi = __half2float(__ushort_as_half(static_cast<unsigned short>(dd >> 16)));
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float d = v < 2 ? d_lo : d_hi;           // 32 weights per scale
                    q8_word_to_bf16x2(cv[v].x, d, out[8 * v + 0], out[8 * v + 1]);
                    q8_word_to_bf16x2(cv[v].y, d, out[8 * v + 2], out[8 * v + 3]);
                    q8_word_to_bf16x2(cv[v].z, d, out[8 * v + 4], out[8 * v + 5]);
                    q8_word_to_bf16x2(cv[v].w, d, out[8 * v + 6], out[8 * v + 7]);
                }
                // released only once every code of the chunk this thread read has been used: a
                // release right after the loads let the next copy overwrite codes still being read
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[sc]);
            } else if (s < NB) {
                const int ci = s / kCS, sc = ci % SC;
                if (!mbar_wait(&c_full[sc], (ci / SC) & 1, abort_flag)) { ok = false; break; }
                const float sv = scale_of(p.sc, qa, da);
                qa = qb; da = db; qb = qc; db = dc;
                load_scale(s + 3 * kGroups, qc, dc);
                __nv_bfloat162 s2b = __float2bfloat162_rn(sv);
                const uint32_t s2 = *reinterpret_cast<uint32_t *>(&s2b);
                const uint32_t cbase = smem_u32(sC) + sc * kCB + ((s % kCS) * 64 + nl) * 64;
                const uint4 c0 = lds128(cbase + (((2u * h + 0u) ^ c_swz) << 4));
                const uint4 c1 = lds128(cbase + (((2u * h + 1u) ^ c_swz) << 4));
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                // levels from the register byte tables (no shared-memory traffic)
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8) {
                    codes4_to_bf16x2(words[w8], lvb, out[w8 * 4 + 0], out[w8 * 4 + 1]);
                    codes4_to_bf16x2(words[w8] >> 16, lvb, out[w8 * 4 + 2], out[w8 * 4 + 3]);
#pragma unroll
                    for (int by = 0; by < 4; ++by) out[w8 * 4 + by] = bf16x2_mul(out[w8 * 4 + by], s2);
                }
                // released only once every code of the chunk this thread read has been used: a
                // release right after the loads let the next copy overwrite codes still being read
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[sc]);
            } else {
                // adapter chunk: row j of A [r, K], 64 k starting at k0 + 64h (zero past r / K)
                const int j = (s - NB) * 64 + nl;
                const int kk0 = k0 + h * 64;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (j < p.r && kk0 < p.K)
                        w = __ldg(reinterpret_cast<const uint4 *>(p.Alora + int64_t(j) * p.K + kk0 + v * 8));
                    out[v * 4 + 0] = w.x; out[v * 4 + 1] = w.y; out[v * 4 + 2] = w.z; out[v * 4 + 3] = w.w;
                }
            }
            // A slot g is free once the MMAs of stage s - kS have completed
            if (!mbar_wait_cluster(&free_b[g], ((s / kS) & 1) ^ 1, abort_flag)) { ok = false; break; }
            const uint32_t abase = sAu + g * kAStageBytes + a_off;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t chunk = uint32_t(i) ^ uint32_t(nl & 7);
                sts128(abase + (chunk << 4), make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]));
            }
            fence_proxy_async_smem();
            // the even CTA's warps arrive only once the stage's dY tile (both halves) has landed,
            // so a completed a_full also means a completed y_full for the MMA thread
            if (rank == 0 && !mbar_wait_cluster(&y_full[g], (s / kS) & 1, abort_flag)) { ok = false; break; }
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&a_full[g]), 0));
        }

        // ---------------- epilogue: this CTA's 128 k rows x BN tokens
        const bool have = ok && mbar_wait_cluster(acc_full, 0, abort_flag);
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int k = k0 + row;
        const uint32_t lane_addr = uint32_t(quad * 32) << 16;
        const int nchunks = p.BN / 16;
        if (have) {
            tc_fence_after();
            if (p.dXacc) {
                for (int ch = grp; ch < nchunks; ch += kGroups) {
                    uint32_t v[16];
                    tmem_ld16(tmem_acc + lane_addr + ch * 16, v);
                    tmem_wait_ld16(v);
                    if (k < p.K) {
                        const int mb = m0 + ch * 16;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (mb + i < p.M) atomicAdd(p.dXacc + int64_t(mb + i) * p.K + k, __uint_as_float(v[i]));
                    }
                }
            } else {
                // bf16 tile [token][128 k] in the ring memory, idle once the last MMAs completed
                const uint32_t stage = smem_u32(smem);
                for (int ch = grp; ch < nchunks; ch += kGroups) {
                    uint32_t v[16];
                    tmem_ld16(tmem_acc + lane_addr + ch * 16, v);
                    tmem_wait_ld16(v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat16 hv = __float2bfloat16_rn(__uint_as_float(v[i]));
                        sts16(stage + uint32_t(((ch * 16 + i) * BM + row) * 2), *reinterpret_cast<uint16_t *>(&hv));
                    }
                }
            }
        }
        if (!p.dXacc) {
            // every dequant warp passes here once, with or without a tile; one thread then
            // stores the tile with TMA (the map clips tokens past M and columns past K)
            fence_proxy_async_smem();
            named_bar_sync(1, 128 * kS);
            if (dw == 0 && lane == 0 && have && *abort_flag == 0) {
                for (int h = 0; h * 256 < p.BN; ++h)
                    tma_store_2d(&tmD, smem + h * 256 * BM * 2, k0, m0 + 256 * h);
                bulk_commit_group();
                bulk_wait_all();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA leaves (or frees TMEM) while the pair may still touch its memory
    cluster_sync();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_acc, ncols);
    }
}

}  // namespace bwdp
}  // namespace qlora
