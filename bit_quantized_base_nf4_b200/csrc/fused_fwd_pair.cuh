// fused_fwd_pair.cuh -- forward GEMM with NF4 dequant, on CTA pairs (tcgen05 cta_group::2).
//
//   D[n, m] = sum_k W'[n, k] X[m, k] (+ adapter chunk),  n in 256 rows (128 per CTA), m in BN tokens
//
// Two CTAs on two SMs form one 256-row x BN-token tile.  Each CTA dequantizes
// its own 128 W rows into its own TMEM (the MMA's A operand) and loads only its
// half of the token tile (BN/2 rows of X) into its own shared memory; one
// tcgen05.mma.cta_group::2 issued by the even CTA reads both halves.
//
// The MMA issue is effectively synchronous with the issuing thread, so every
// barrier operation of that thread is lost tensor time.  The pipeline is built
// to keep them rare: a stage is 128 K (eight MMAs), the MMA thread waits on one
// barrier per stage (a_full, which the even CTA's dequant warps only arrive on
// after they have seen the stage's X tile land) and commits once per stage to
// free[s % 4], which releases both the X slot and the TMEM A slot of the stage.
//   producer (warp 0)    one 3-D TMA instruction per stage: two 64-K chunks of
//                        this CTA's X half, counted on the even CTA's x_full
//   producer (warp 3)    packed codes, 256 K (two stages) per TMA instruction
//   dequant group q % 4  (4 warps, thread = one W row) expands the stage's 128
//                        weights of its row through a shared-memory table
//                        byte -> (level[lo], level[hi]) as bf16x2 times the bf16
//                        block scale, into TMEM slot q % 4 (64 columns), then
//                        arrives on the even CTA's a_full
//   MMA (warp 1, even)   eight tcgen05.mma (K = 16), A from TMEM, B from smem
// Commits are multicast to both CTAs (free, acc_full).  Each CTA
// finally reads back its own 128 x BN accumulator.
//
// kQ8 selects the Q8_0 route (GGUF page, sections 1.1 and 2.2): one int8 code per
// weight and an fp16 scale per 32 weights; a code chunk then holds one stage (128 K)
// and the dequant warps expand int8 x fp16 scale to bf16 in registers (no table).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "scale_src.cuh"

namespace qlora {
namespace fwdp {

constexpr int BM = 128;            // W rows per CTA (256 per pair)
constexpr int kStageK = 128;       // K per pipeline stage (two 64-K chunks, eight MMAs)
constexpr int SX = 4;              // X ring slots (one stage each) = dequant groups
constexpr int SC = 4;              // code ring chunks (256 K = two stages each)
constexpr int kGroups = 4;         // dequant groups = TMEM A slots (64 columns each)
constexpr int kDqWarps = 4 * kGroups;
constexpr int kThreads = 128 + 32 * kDqWarps;
constexpr int kCodeChunkBytes = BM * 128;     // 128 rows x 128 bytes (256 weights)
constexpr int kLutWords = 256 * 32;           // byte -> bf16x2, replicated per lane

struct Params {
    ScaleSrc sc;             // first-level scales of the weight's storage format (4-bit codes)
    const uint16_t *d8;      // Q8_0: fp16 scale of each 32 weights, [N, K/32]
    const uint16_t *Blora;   // [N, r] bf16 or nullptr
    uint16_t *Y;             // [M, N] bf16
    int M, N, K, r, BN;      // BN: tokens per pair tile, a multiple of 32
    int raster_mode, raster_group;   // tile order of the pairs (raster_tile)
    float level[16];
};

__host__ __device__ constexpr int smem_bytes(int BN, bool = false) {
    return 1024 /*align slack*/ + SX * 2 * (BN / 2) * 128 + SC * kCodeChunkBytes + 512 /*barriers*/;
}
// A slots at columns [0, 256), accumulator at [256, 256 + BN)
__host__ __device__ constexpr uint32_t tmem_cols(int) { return 512u; }

template <bool kQ8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    fused_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                          const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmY,
                          const Params p) {
    constexpr int kStagesPerChunk = kQ8 ? 1 : 2;   // a 128-byte code row holds 256 (4-bit) or 128 (8-bit) K
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int half_bn = p.BN / 2;
    const int xsb = half_bn * 128;               // this CTA's half X tile for one 64-K chunk
    const int slotb = 2 * xsb;                   // one X ring slot (one stage)
    uint8_t *sX = smem;
    uint8_t *sC = sX + SX * slotb;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sC + SC * kCodeChunkBytes);
    // stage slot g = q % 4: X slot g and TMEM A slot g share one release barrier free[g]
    uint64_t *x_full = bars, *free_b = bars + SX;
    uint64_t *c_full = bars + 2 * SX, *c_empty = c_full + SC;
    uint64_t *a_full = c_empty + SC;
    uint64_t *acc_full = a_full + kGroups;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *s_level = reinterpret_cast<float *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();      // 0: even CTA (issues the MMAs), 1: its peer
    // this pair's tile: 256 W rows x BN tokens, in the L2-friendly order of raster_tile
    int wt, tt;
    raster_tile(blockIdx.y * (gridDim.x / 2) + (blockIdx.x >> 1), gridDim.x / 2, gridDim.y, p.raster_mode,
                p.raster_group, wt, tt);
    const int n0 = (2 * wt + int(rank)) * BM;
    const int m0 = tt * p.BN;
    const int my_m0 = m0 + int(rank) * half_bn;
    const int KB = p.K / 64;                      // 64-K chunks of the base
    const int QM = (KB + 1) / 2;                  // main stages
    const int Q = QM + (p.r > 0 ? 1 : 0);         // + one adapter stage (r <= 128)
    const int nchunk = (KB + 2 * kStagesPerChunk - 1) / (2 * kStagesPerChunk);   // code chunks

    if (threadIdx.x < 16) {
        float v = 0.f;  // constant-index reads keep the parameter block out of local memory
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (threadIdx.x == i) v = p.level[i];
        s_level[threadIdx.x] = v;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < SX; ++i) { mbar_init(&x_full[i], 1); mbar_init(&free_b[i], 1); }
        // a chunk is read by the groups of its stages (four warps each)
        for (int i = 0; i < SC; ++i) { mbar_init(&c_full[i], 1); mbar_init(&c_empty[i], 4 * kStagesPerChunk); }
        for (int i = 0; i < kGroups; ++i) mbar_init(&a_full[i], 8);
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc_pair(tmem_slot, tmem_cols(p.BN));
        tmem_relinquish_pair();
    }
    __syncthreads();
    tc_fence_before();
    // both CTAs' barriers are initialised before either signals the other's
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_a = tmem;          // A slots: columns g*64 .. g*64+63
    const uint32_t tmem_acc = tmem + 256;  // accumulator: columns 256 .. 256+BN-1

    if (warp == 0) {
        // ---------------- X producer
        if (lane == 0) {
            tma_prefetch_desc(&tmX);
            if (p.r > 0) tma_prefetch_desc(&tmU);
            int issued = 0;
            for (int q = 0; q < Q; ++q) {
                const int sx = q % SX;
                if (!mbar_wait_cluster(&free_b[sx], ((q / SX) & 1) ^ 1, abort_flag)) break;
                const uint32_t bar0 = mapa_shared(smem_u32(&x_full[sx]), 0);
                uint8_t *slot = sX + sx * slotb;
                if (q < QM) {
                    if (rank == 0) mbar_arrive_expect_tx(&x_full[sx], 2 * slotb);
                    tma_load_3d_pair(slot, &tmX, bar0, 0, my_m0, 2 * q);
                } else {
                    const int nv = (p.r + 63) / 64;
                    if (rank == 0) mbar_arrive_expect_tx(&x_full[sx], 2 * nv * xsb);
                    for (int d = 0; d < nv; ++d) tma_load_2d_pair(slot + d * xsb, &tmU, bar0, d * 64, my_m0);
                }
                issued = q + 1;
            }
            // the even CTA sees both CTAs' copies complete on its barriers
            if (rank == 0)
                for (int q = max(0, issued - SX); q < issued; ++q) mbar_drain(&x_full[q % SX], (q / SX) & 1);
            // producer tail: the release commits of the last stages land on this CTA's barriers
            // before it exits, so none can reach the shared memory of a CTA launched after it
            for (int q = max(0, issued - SX); q < issued; ++q) mbar_drain_cluster(&free_b[q % SX], (q / SX) & 1);
        }
    } else if (warp == 3) {
        // ---------------- packed-code producer (local to each CTA)
        if (lane == 0) {
            tma_prefetch_desc(&tmC);
            int issued = 0;
            for (int c = 0; c < nchunk; ++c) {
                const int sc = c % SC;
                if (!mbar_wait(&c_empty[sc], ((c / SC) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&c_full[sc], kCodeChunkBytes);
                tma_load_2d(sC + sc * kCodeChunkBytes, &tmC, &c_full[sc], c * 128, n0);
                issued = c + 1;
            }
            for (int c = max(0, issued - SC); c < issued; ++c) mbar_drain(&c_full[c % SC], (c / SC) & 1);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (even CTA only)
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = make_idesc_bf16(2 * BM, p.BN, 0, 0);
            for (int q = 0; q < Q; ++q) {
                const int sx = q % SX, g = q % kGroups;
                // the peer CTA's half of the A operand was written by its threads: acquire at cluster scope
                if (!mbar_wait_cluster(&a_full[g], (q / kGroups) & 1, abort_flag)) break;
                tc_fence_after();
                // MMAs of this stage: 8 for a full main stage, 4 for the last odd chunk,
                // ceil(r/16) for the adapter stage
                const int nk = q < QM ? (2 * q + 1 < KB ? 8 : 4) : (p.r + 15) / 16;
                const uint32_t xbase = smem_u32(sX + sx * slotb);
                for (int kk = 0; kk < nk; ++kk) {
                    const uint64_t bdesc = make_sdesc_sw128(xbase + (kk >> 2) * xsb + (kk & 3) * 32, 16, 1024);
                    mma_ts_pair(tmem_acc, tmem_a + g * 64 + kk * 8, bdesc, idesc, (q > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit_pair(&free_b[sx]);
            }
            tc_commit_pair(acc_full);
            mbar_drain(acc_full, 0);
        }
    } else if (warp >= 4) {
        // ---------------- dequant into this CTA's TMEM, then epilogue
        const int dw = warp - 4;
        const int grp = dw >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int n = n0 + row;
        const bool valid = n < p.N;
        const LevelBytes lvb = level_bytes(*reinterpret_cast<const float (*)[16]>(s_level));
        const uint32_t lane_addr = uint32_t(quad * 32) << 16;
        // 128-byte code rows, 128-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ (r & 7)
        const uint32_t code_row = smem_u32(sC) + row * 128;
        const uint32_t cswz = row & 7;
        bool ok = true;
        const int64_t row_block0 = int64_t(n) * KB;
        // the raw scale words of a 64-weight run (zero past the row end)
        auto load_scale = [&](int kb, uint32_t &av, float &dv) {
            av = 0u;
            dv = 0.f;
            if (!kQ8 && valid && kb < KB) scale_load(p.sc, row_block0 + kb, av, dv);
        };
        // Q8_0: the four fp16 scales of a 128-K stage (two words)
        auto load_d8 = [&](int q, uint32_t &w0, uint32_t &w1) {
            w0 = 0u;
            w1 = 0u;
            if (kQ8 && valid && q < QM) {
                const uint32_t *drow = reinterpret_cast<const uint32_t *>(p.d8 + int64_t(n) * (p.K / 32));
                w0 = __ldg(drow + 2 * q);
                if (2 * q + 1 < KB) w1 = __ldg(drow + 2 * q + 1);
            }
        };
        // scales of this group's next stage, loaded one group iteration (four stages) ahead
        uint32_t q0, q1, e0, e1;
        float d0, d1;
        load_scale(2 * grp, q0, d0);
        load_scale(2 * grp + 1, q1, d1);
        load_d8(grp, e0, e1);

        for (int q = grp; q < Q && ok; q += kGroups) {
            const int g = grp;
            const uint32_t slot = tmem_a + lane_addr + g * 64;
            // a main stage has two 64-K halves except an odd last one; the adapter stage
            // has a second half only for r > 64
            const bool two = q < QM ? 2 * q + 1 < KB : p.r > 64;
            // TMEM slot g is free once the MMAs of stage q - 4 have completed.  The first
            // half of the stage is expanded before this wait, the second while the first
            // is stored, so the wait is followed by stores rather than by the whole expansion.
            auto wait_slot = [&]() -> bool {
                if (!mbar_wait_cluster(&free_b[g], ((q / kGroups) & 1) ^ 1, abort_flag)) return false;
                tc_fence_after();
                return true;
            };
            uint32_t out[32];
            if (kQ8 && q < QM) {
                // Q8_0: this stage's 128 code bytes of the row and its four fp16 scales
                const int sc = q % SC;
                if (!mbar_wait(&c_full[sc], (q / SC) & 1, abort_flag)) { ok = false; break; }
                const uint32_t cbase = code_row + sc * kCodeChunkBytes;
                uint4 cv[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) cv[i] = lds128(cbase + ((uint32_t(i) ^ cswz) << 4));
                const uint32_t dpair[2] = {e0, e1};
                load_d8(q + kGroups, e0, e1);
                auto expand = [&](int sub) {
                    const float d_lo = __half2float(__ushort_as_half(static_cast<unsigned short>(dpair[sub] & 0xFFFFu)));
                    const float d_hi = __half2float(__ushort_as_half(static_cast<unsigned short>(dpair[sub] >> 16)));
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 c = cv[4 * sub + v];
                        const float d = v < 2 ? d_lo : d_hi;       // 32 weights per scale
                        q8_word_to_bf16x2(c.x, d, out[8 * v + 0], out[8 * v + 1]);
                        q8_word_to_bf16x2(c.y, d, out[8 * v + 2], out[8 * v + 3]);
                        q8_word_to_bf16x2(c.z, d, out[8 * v + 4], out[8 * v + 5]);
                        q8_word_to_bf16x2(c.w, d, out[8 * v + 6], out[8 * v + 7]);
                    }
                };
                expand(0);
                if (!wait_slot()) { ok = false; break; }
                tmem_st32_checked(slot, out);
                if (two) {
                    expand(1);
                    tmem_st32_checked(slot + 32, out);
                }
                // released only once every code of the chunk this thread read has been used: a
                // release right after the loads let the next copy overwrite codes still being read
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[sc]);
            } else if (q < QM) {
                const int ci = q >> 1, sc = ci % SC;
                if (!mbar_wait(&c_full[sc], (ci / SC) & 1, abort_flag)) { ok = false; break; }
                const uint32_t cbase = code_row + sc * kCodeChunkBytes;
                const uint32_t jq = 4u * uint32_t(q & 1);          // first 16-byte chunk of this stage
                const uint4 c0 = lds128(cbase + (((jq + 0u) ^ cswz) << 4));
                const uint4 c1 = lds128(cbase + (((jq + 1u) ^ cswz) << 4));
                const uint4 c2 = lds128(cbase + (((jq + 2u) ^ cswz) << 4));
                const uint4 c3 = lds128(cbase + (((jq + 3u) ^ cswz) << 4));
                const float sv0 = scale_of(p.sc, q0, d0);
                const float sv1 = scale_of(p.sc, q1, d1);
                load_scale(2 * (q + kGroups), q0, d0);
                load_scale(2 * (q + kGroups) + 1, q1, d1);
                auto expand = [&](int sub) {
                    __nv_bfloat162 s2b = __float2bfloat162_rn(sub ? sv1 : sv0);
                    const uint32_t s2 = *reinterpret_cast<uint32_t *>(&s2b);
                    const uint4 ca = sub ? c2 : c0, cb = sub ? c3 : c1;
                    const uint32_t words[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                    // levels from the register byte tables (no shared-memory traffic)
#pragma unroll
                    for (int w8 = 0; w8 < 8; ++w8) {
                        codes4_to_bf16x2(words[w8], lvb, out[w8 * 4 + 0], out[w8 * 4 + 1]);
                        codes4_to_bf16x2(words[w8] >> 16, lvb, out[w8 * 4 + 2], out[w8 * 4 + 3]);
#pragma unroll
                        for (int by = 0; by < 4; ++by) out[w8 * 4 + by] = bf16x2_mul(out[w8 * 4 + by], s2);
                    }
                };
                expand(0);
                if (!wait_slot()) { ok = false; break; }
                tmem_st32_checked(slot, out);
                if (two) {
                    expand(1);
                    tmem_st32_checked(slot + 32, out);
                }
                // released only once every code of the chunk this thread read has been used: a
                // release right after the loads let the next copy overwrite codes still being read
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[sc]);
            } else {
                // adapter stage: A operand = B_lora row n, elements 0 .. 127 (zero past r)
                auto fill = [&](int sub) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        uint4 w = make_uint4(0, 0, 0, 0);
                        const int e = sub * 64 + v * 8;
                        if (valid && e < p.r)
                            w = __ldg(reinterpret_cast<const uint4 *>(p.Blora + int64_t(n) * p.r + e));
                        out[v * 4 + 0] = w.x; out[v * 4 + 1] = w.y; out[v * 4 + 2] = w.z; out[v * 4 + 3] = w.w;
                    }
                };
                fill(0);
                if (!wait_slot()) { ok = false; break; }
                tmem_st32_checked(slot, out);
                if (two) {
                    fill(1);
                    tmem_st32_checked(slot + 32, out);
                }
            }
            tc_fence_before();
            // the even CTA's warps arrive only once the stage's X tile (both halves) has landed,
            // so a completed a_full also means a completed x_full for the MMA thread
            if (rank == 0 && !mbar_wait_cluster(&x_full[g], (q / kGroups) & 1, abort_flag)) { ok = false; break; }
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&a_full[g]), 0));
        }

        // ---------------- epilogue: this CTA's 128 rows x BN tokens, staged as a bf16
        // [token][128 n] tile in the X ring (idle once the last MMAs completed), then one
        // TMA store (the map clips tokens past M and rows past N)
        const bool have = ok && mbar_wait_cluster(acc_full, 0, abort_flag);
        if (have) {
            tc_fence_after();
            const uint32_t stage = smem_u32(sX);
            const int nchunks = p.BN / 16;
            for (int ch = grp; ch < nchunks; ch += kGroups) {
                uint32_t v[16];
                tmem_ld16(tmem_acc + lane_addr + ch * 16, v);
                tmem_wait_ld16(v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[i]));
                    sts16(stage + uint32_t(((ch * 16 + i) * BM + row) * 2), *reinterpret_cast<uint16_t *>(&h));
                }
            }
        }
        // every dequant warp passes here once, with or without a tile
        fence_proxy_async_smem();
        named_bar_sync(1, 32 * kDqWarps);
        if (dw == 0 && lane == 0 && have && *abort_flag == 0) {
            tma_store_2d(&tmY, sX, n0, m0);
            bulk_commit_group();
            bulk_wait_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA leaves (or frees TMEM) while the pair may still touch its memory
    cluster_sync();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, tmem_cols(p.BN));
    }
}

}  // namespace fwdp
}  // namespace qlora
