// decode_mma.cuh -- small-M forward (M <= 16 tokens): the weight-streaming path.
//
//   Y[m, n] = sum_k X[m, k] W'[n, k] + scaling * sum_j U[m, j] B[n, j],   U = X A^T
//
// With at most 16 tokens the forward is bound by streaming the packed weight
// (0.516 B per weight) from HBM.  tcgen05 cannot keep up at such a narrow N (its
// per-instruction cost is paid for 128 x 16 x 16 of work), so the contraction runs
// on warp MMAs, mma.sync m16n8k16 bf16 -> fp32, with the tokens as the m16 operand
// (rows past M are zero) and eight dequantized W rows as the n8 operand, built in
// registers from codes through a byte -> bf16x2 table.
//
// Work split.  A unit is 32 W rows over all of K, so no partial sum ever leaves its
// CTA.  One persistent CTA per SM takes a contiguous run of units.
//
// Data movement (two producer warps, eight consumer warps):
//   - codes: a ring of 8 KB stages, each two TMA boxes of [32 rows x 128 B] (512 k)
//     with the 128-byte swizzle, 8 stages deep: about 64 KB in flight per SM;
//   - activations X (and, during a CTA's first unit, the adapter rows A): a second
//     ring of [8 chunks x 8|16 rows x 128 B] swizzled boxes, 2-4 stages deep, fed by
//     the second producer warp (these come from L2);
//   - block scales of a unit: one bulk copy of its 32 x K/64 bytes (contiguous in the
//     packed layout) plus the unit's second-level steps, double-buffered per unit.
//
// Fragment mapping.  Consumer warp w takes block pair w % 4 of each stage (blocks
// 2(w%4), 2(w%4)+1) and n8 groups 2(w/4), 2(w/4)+1 of the unit.  Lane (g, t) owns 32
// consecutive weights: half t % 2 of block 2(w%4) + t/2, i.e. one 16-byte unit of
// the swizzled code row, which it reads with one conflict-free 128-bit load.  MMA
// column g is W row sigma(g) = 4 (g % 2) + g / 2 of the n8 group, chosen so that
// the two rows read by each quarter-warp fall in different swizzle halves.  In
// k-step j the lane supplies weights 4j .. 4j+3 of its 32 as B and the activations
// at the same k positions as A; the MMA sums over its k slots in any order, so this
// pairing only has to agree between A and B.
//
// The adapter product U = X A^T uses the same loop with the rows of A as extra n8
// operands; every CTA computes it during its first unit and keeps it in shared
// memory for the adapter term of all its units.
//
// Overlap with the preceding kernel (programmatic dependent launch): before waiting
// on the preceding grid a CTA builds its table, initialises its barriers and
// prefetches the code bytes of its first units into L2 (which is coherent);
// every load into shared memory and every activation access follows
// griddepcontrol.wait.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {
namespace dec {

constexpr int kRows = 32;                       // W rows per unit
constexpr int kStageK = 512;                    // k per pipeline stage
constexpr int kStageBlocks = kStageK / 64;
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 64;       // + two producer warps
constexpr int kMaxRank = 16;                    // adapter ranks fused on this path
constexpr int kMaxKB = 512;                     // 64-k blocks per row (n_in <= 32768)
constexpr int kCodeStage = kRows * kStageK / 2; // 8 KB
constexpr int kLutBytes = 256 * 32 * 4;         // one bf16x2 per byte value per lane
constexpr int kMaxCodeStages = 8;
constexpr int kMaxXaStages = 4;
constexpr int kPartFloats = 4 * kRows * 16;     // [block pair][row][token]
constexpr int kSmemLimit = 232448;

struct Params {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *scales2;
    const uint16_t *Blora;   // [N, r] or nullptr
    uint16_t *Y;             // [M, N]
    uint16_t *U_save;        // [M, r] or nullptr
    int M, N, K, r;
    int units;               // ceil(N / 32)
    int dc, dx;              // ring depths (codes, activations)
    int mbox, rbox;          // rows of the X and A boxes (8 or 16; rbox 0 without adapter)
    // byte offsets from the 1024-aligned shared-memory base
    int off_code, off_xa, xa_stage, off_sc, sc_stage, sc_q, off_part, off_upart, off_ufin, off_bars;
    float scaling;
    float level[16];
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// global -> shared bulk copy (16-byte aligned addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// 4-byte asynchronous copy reading only `src_bytes` (0-4) bytes; the rest is zero
__device__ __forceinline__ void cp_async4(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
// arrive on `bar` once this thread's earlier cp.async copies have landed (counted in
// the barrier's expected arrivals)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }
__device__ __forceinline__ uint8_t lds_u8(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
    return static_cast<uint8_t>(v);
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

template <int NT>   // token tiles of 8: 1 for M <= 8, 2 for M <= 16
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmA, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.off_bars);
    uint64_t *code_full = bars, *code_empty = bars + kMaxCodeStages;
    uint64_t *xa_full = bars + 2 * kMaxCodeStages, *xa_empty = xa_full + kMaxXaStages;
    uint64_t *sc_full = xa_empty + kMaxXaStages, *sc_empty = sc_full + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = p.K / 64;
    const int nst = (KB + kStageBlocks - 1) / kStageBlocks;          // stages per unit
    const int u0 = static_cast<int>(int64_t(p.units) * blockIdx.x / gridDim.x);
    const int u1 = static_cast<int>(int64_t(p.units) * (blockIdx.x + 1) / gridDim.x);
    const int nu = u1 - u0;
    const int nA = p.rbox / 8;                                        // adapter n8 groups

    // 1. let the next kernel in the stream start launching
    pdl_launch_dependents();

    // 2. byte -> bf16x2 (level[lo], level[hi]) table, one copy per lane
    for (int e = threadIdx.x; e < 256; e += kThreads) {
        float lo = 0.f, hi = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {   // constant-index reads keep the parameter block out of local memory
            if ((e & 15) == i) lo = p.level[i];
            if ((e >> 4) == i) hi = p.level[i];
        }
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        const uint32_t w = *reinterpret_cast<uint32_t *>(&v);
        const uint32_t base = smem_u32(smem) + e * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) sts128(base + c * 16, make_uint4(w, w, w, w));
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxCodeStages; ++i) { mbar_init(&code_full[i], 1); mbar_init(&code_empty[i], kConsumerWarps); }
        for (int i = 0; i < kMaxXaStages; ++i) { mbar_init(&xa_full[i], 1); mbar_init(&xa_empty[i], kConsumerWarps); }
        for (int i = 0; i < 2; ++i) { mbar_init(&sc_full[i], 33); mbar_init(&sc_empty[i], kConsumerWarps); }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kConsumerWarps && lane == 0 && nu > 0) {
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmX);
        if (nA > 0) tma_prefetch_desc(&tmA);
        // the code rows of the first two units are contiguous: warm L2 with them
        const int64_t row_bytes = p.K / 2;
        const int64_t r0 = int64_t(u0) * kRows;
        const int64_t r1 = min(int64_t(p.N), int64_t(min(u1, u0 + 2)) * kRows);
        const uint8_t *src = p.codes + r0 * row_bytes;
        for (int64_t off = 0, n = (r1 - r0) * row_bytes; off < n; off += 16384)
            prefetch_l2_bulk(src + off, static_cast<uint32_t>((n - off < 16384 ? n - off : int64_t(16384))));
    }
    __syncthreads();

    // 3. everything below may read what the preceding grid wrote
    pdl_wait();
    if (nu <= 0) return;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------- code and scale producer
        const int T = nu * nst;
        int issued = 0, sc_issued = 0;
        for (int i = 0; i < T; ++i) {
            const int ui = i / nst, j = i - ui * nst;
            const int u = u0 + ui;
            if (j == 0) {   // this unit's block scales and second-level steps
                const int sb = ui & 1;
                if (ui >= 2 && !mbar_wait(&sc_empty[sb], ((ui >> 1) - 1) & 1, abort_flag)) break;
                uint8_t *sq = smem + p.off_sc + sb * p.sc_stage;
                float *s2 = reinterpret_cast<float *>(sq + p.sc_q);
                const int rows = min(kRows, p.N - u * kRows);
                const uint32_t bytes = static_cast<uint32_t>(rows * KB);
                const uint32_t bulk = bytes & ~15u;
                const int64_t fb0 = int64_t(u) * kRows * KB;   // first flat block of the unit
                const int64_t g0 = fb0 >> 8, g1 = (fb0 + bytes - 1) >> 8;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sc_full[sb], bulk);
                    if (bulk) bulk_g2s(sq, p.scales + fb0, bulk, &sc_full[sb]);
                }
                if (lane < 4) {
                    const uint32_t off = bulk + 4u * lane;
                    if (off < bytes) cp_async4(sq + off, p.scales + fb0 + off, min(4u, bytes - off));
                }
                for (int k = lane; k <= int(g1 - g0); k += 32) cp_async4(s2 + k, p.scales2 + g0 + k, 4u);
                cp_async_arrive_noinc(&sc_full[sb]);
                sc_issued = ui + 1;
            }
            const int slot = i % p.dc;
            if (i >= p.dc && !mbar_wait(&code_empty[slot], ((i / p.dc) - 1) & 1, abort_flag)) break;
            if (lane == 0) {
                uint8_t *dst = smem + p.off_code + slot * kCodeStage;
                mbar_arrive_expect_tx(&code_full[slot], kCodeStage);
                tma_load_2d(dst, &tmC, &code_full[slot], j * (kStageK / 2), u * kRows);
                tma_load_2d(dst + kCodeStage / 2, &tmC, &code_full[slot], j * (kStageK / 2) + 128, u * kRows);
            }
            issued = i + 1;
        }
        // nothing this warp issued may land after the CTA has exited
        if (lane == 0)
            for (int i = max(0, issued - p.dc); i < issued; ++i) mbar_drain(&code_full[i % p.dc], (i / p.dc) & 1);
        for (int ui = max(0, sc_issued - 2); ui < sc_issued; ++ui) mbar_drain(&sc_full[ui & 1], (ui >> 1) & 1);
        return;
    }
    if (warp == kConsumerWarps + 1) {
        // ------------------------------------------- activation (and adapter) producer
        if (lane == 0) {
            const int T = nu * nst;
            int issued = 0;
            for (int i = 0; i < T; ++i) {
                const int ui = i / nst, j = i - ui * nst;
                const int slot = i % p.dx;
                if (i >= p.dx && !mbar_wait(&xa_empty[slot], ((i / p.dx) - 1) & 1, abort_flag)) break;
                const bool with_a = ui == 0 && nA > 0;
                uint8_t *dst = smem + p.off_xa + slot * p.xa_stage;
                mbar_arrive_expect_tx(&xa_full[slot], (p.mbox + (with_a ? p.rbox : 0)) * 1024);
                tma_load_3d(dst, &tmX, &xa_full[slot], 0, 0, j * kStageBlocks);
                if (with_a) tma_load_3d(dst + p.mbox * 1024, &tmA, &xa_full[slot], 0, 0, j * kStageBlocks);
                issued = i + 1;
            }
            for (int i = max(0, issued - p.dx); i < issued; ++i) mbar_drain(&xa_full[i % p.dx], (i / p.dx) & 1);
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int pr = warp & 3, gs = warp >> 2;
    const int g = lane >> 2, t = lane & 3;
    const int sg = ((g & 1) << 2) | (g >> 1);          // W row (in its n8 group) of MMA column g
    const int ctid = threadIdx.x;                      // 0 .. kConsumers-1
    const uint32_t lut = smem_u32(smem) + lane * 4;
    const uint32_t code_base = smem_u32(smem + p.off_code);
    const uint32_t xa_base = smem_u32(smem + p.off_xa);
    float *part_all = reinterpret_cast<float *>(smem + p.off_part);
    float *upart = reinterpret_cast<float *>(smem + p.off_upart);
    float *ufin = reinterpret_cast<float *>(smem + p.off_ufin);
    const bool tok0 = g < p.M, tok1 = NT > 1 && g + 8 < p.M;
    const int chunk = 2 * pr + (t >> 1);               // 64-k chunk of the stage this lane reads
    // byte offsets inside a stage: X row g (and g+8) of `chunk`, A row 8 gs + g, code row
    const uint32_t x_off0 = uint32_t((chunk * p.mbox + g) * 128);
    const uint32_t x_off1 = uint32_t((chunk * p.mbox + g + 8) * 128);
    const uint32_t a_off = uint32_t(p.mbox * 1024 + (chunk * p.rbox + 8 * gs + g) * 128);
    const uint32_t c_off = uint32_t((pr >> 1) * (kCodeStage / 2) + (((4 * (pr & 1) + t) ^ sg) << 4));
    const bool do_u = gs < nA;
    const int brow = ctid & 31;                         // epilogue row

    int i = 0;   // stage counter
    for (int ui = 0; ui < nu; ++ui) {
        const int u = u0 + ui;
        const int n0 = u * kRows;
        const int sb = ui & 1;
        const bool first = ui == 0;
        // adapter row of B for the epilogue, loaded while the unit streams
        uint4 bv0 = make_uint4(0, 0, 0, 0), bv1 = make_uint4(0, 0, 0, 0);
        if (p.r > 0 && n0 + brow < p.N) {
            const uint16_t *bp = p.Blora + int64_t(n0 + brow) * p.r;
            bv0 = *reinterpret_cast<const uint4 *>(bp);
            if (p.r > 8) bv1 = *reinterpret_cast<const uint4 *>(bp + 8);
        }
        mbar_wait(&sc_full[sb], (ui >> 1) & 1, abort_flag);
        const uint32_t sq = smem_u32(smem + p.off_sc + sb * p.sc_stage);
        const uint32_t s2 = sq + p.sc_q;
        // flat block index of the unit's first block, modulo one second-level group: the
        // unit's steps were copied starting from the group holding that block
        const int fb_lo = static_cast<int>((int64_t(n0) * KB) & 255);
        // per group: this lane's W row in the code box and in the unit's scale rows
        uint32_t row_off[2];
        int row_q[2];
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
            const int row = 8 * (2 * gs + gg) + sg;
            row_off[gg] = uint32_t(row * 128);
            row_q[gg] = row * KB;
        }

        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float accU[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < nst; ++j, ++i) {
            const int slot = i % p.dc, xslot = i % p.dx;
            mbar_wait(&code_full[slot], (i / p.dc) & 1, abort_flag);
            mbar_wait(&xa_full[xslot], (i / p.dx) & 1, abort_flag);
            const int kb = j * kStageBlocks + chunk;
            const bool kv = kb < KB;
            const uint32_t xs = xa_base + uint32_t(xslot * p.xa_stage);
            uint4 xw[4], xh[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t sw = uint32_t(((4 * (t & 1) + q) ^ g) << 4);
                xw[q] = tok0 ? lds128(xs + x_off0 + sw) : make_uint4(0, 0, 0, 0);
                xh[q] = tok1 ? lds128(xs + x_off1 + sw) : make_uint4(0, 0, 0, 0);
            }
            const uint32_t cs = code_base + uint32_t(slot * kCodeStage) + c_off;
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                uint32_t sc = 0;
                if (kv) {
                    const uint32_t q = lds_u8(sq + uint32_t(row_q[gg] + kb));
                    const float d = lds_f32(s2 + uint32_t(((fb_lo + row_q[gg] + kb) >> 8) << 2));
                    __nv_bfloat162 s2b = __float2bfloat162_rn(__fmul_rn(static_cast<float>(q), d));
                    sc = *reinterpret_cast<uint32_t *>(&s2b);
                }
                const uint4 cw = lds128(cs + row_off[gg]);
                const uint32_t cwv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const uint32_t word = cwv[jj >> 1];
                    const uint32_t sh = 16 * (jj & 1);
                    const uint32_t e0 = (word >> sh) & 0xFFu, e1 = (word >> (sh + 8)) & 0xFFu;
                    const uint32_t b0 = bf16x2_mul(lds32(lut + (e0 << 7)), sc);
                    const uint32_t b1 = bf16x2_mul(lds32(lut + (e1 << 7)), sc);
                    const uint4 &xa = xw[jj >> 1];
                    const uint4 &xb = xh[jj >> 1];
                    const uint32_t a0 = (jj & 1) ? xa.z : xa.x, a2 = (jj & 1) ? xa.w : xa.y;
                    const uint32_t a1 = (jj & 1) ? xb.z : xb.x, a3 = (jj & 1) ? xb.w : xb.y;
                    mma_bf16_16816(acc[gg], a0, NT > 1 ? a1 : 0u, a2, NT > 1 ? a3 : 0u, b0, b1);
                }
            }
            if (first && do_u) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t sw = uint32_t(((4 * (t & 1) + q) ^ g) << 4);
                    const uint4 aw = lds128(xs + a_off + sw);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 &xa = xw[q];
                        const uint4 &xb = xh[q];
                        const uint32_t a0 = h ? xa.z : xa.x, a2 = h ? xa.w : xa.y;
                        const uint32_t a1 = h ? xb.z : xb.x, a3 = h ? xb.w : xb.y;
                        mma_bf16_16816(accU, a0, NT > 1 ? a1 : 0u, a2, NT > 1 ? a3 : 0u, h ? aw.z : aw.x,
                                       h ? aw.w : aw.y);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&code_empty[slot]);
                mbar_arrive(&xa_empty[xslot]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sc_empty[sb]);

        // partial sums of this block pair -> part[pr][row][token]
        float *part = part_all + sb * kPartFloats;
        float *pb = part + pr * kRows * 16;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
            const int grp = 2 * gs + gg;
            const int c0 = 2 * t, c1 = 2 * t + 1;
            const int R0 = 8 * grp + (((c0 & 1) << 2) | (c0 >> 1));
            const int R1 = 8 * grp + (((c1 & 1) << 2) | (c1 >> 1));
            pb[R0 * 16 + g] = acc[gg][0];
            pb[R1 * 16 + g] = acc[gg][1];
            pb[R0 * 16 + g + 8] = acc[gg][2];
            pb[R1 * 16 + g + 8] = acc[gg][3];
        }
        if (first && do_u) {
            float *ub = upart + pr * 256;
            const int j0 = 8 * gs + 2 * t;
            ub[g * 16 + j0] = accU[0];
            ub[g * 16 + j0 + 1] = accU[1];
            ub[(g + 8) * 16 + j0] = accU[2];
            ub[(g + 8) * 16 + j0 + 1] = accU[3];
        }
        consumer_sync();
        if (first && p.r > 0) {
            for (int e = ctid; e < 256; e += kConsumers)
                ufin[e] = upart[e] + upart[256 + e] + upart[512 + e] + upart[768 + e];
            consumer_sync();
            if (p.U_save && blockIdx.x == 0) {
                for (int e = ctid; e < p.M * p.r; e += kConsumers) {
                    const int m = e / p.r, jr = e - m * p.r;
                    __nv_bfloat16 h = __float2bfloat16_rn(ufin[m * 16 + jr]);
                    p.U_save[e] = *reinterpret_cast<uint16_t *>(&h);
                }
            }
        }
        // outputs: thread -> row (ctid % 32), tokens ctid / 32, + 8
        const int n = n0 + brow;
        if (n < p.N) {
            const uint32_t bw[8] = {bv0.x, bv0.y, bv0.z, bv0.w, bv1.x, bv1.y, bv1.z, bv1.w};
            for (int m = ctid >> 5; m < p.M; m += kConsumerWarps) {
                const float base = part[brow * 16 + m] + part[kRows * 16 + brow * 16 + m] +
                                   part[2 * kRows * 16 + brow * 16 + m] + part[3 * kRows * 16 + brow * 16 + m];
                float l = 0.f;
                if (p.r > 0) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        if (e < p.r) {
                            const float b = __uint_as_float((e & 1) ? (bw[e >> 1] & 0xFFFF0000u) : (bw[e >> 1] << 16));
                            l = fmaf(ufin[m * 16 + e], b, l);
                        }
                    }
                }
                __nv_bfloat16 h = __float2bfloat16_rn(fmaf(p.scaling, l, base));
                p.Y[int64_t(m) * p.N + n] = *reinterpret_cast<uint16_t *>(&h);
            }
        }
    }
}

}  // namespace dec
}  // namespace qlora
