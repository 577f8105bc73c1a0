// decode_mma.cuh -- small-M forward (M <= 16 tokens): the weight-streaming path.
//
//   Y[m, n] = sum_k X[m, k] W'[n, k] + scaling * sum_j U[m, j] B[n, j],   U = X A^T
//
// With at most 16 tokens the forward is bound by streaming the packed weight
// (0.516 B per weight) from HBM.  tcgen05 cannot keep up at such a narrow N (its
// per-instruction cost is paid for 128 x 16 x 16 of work), so the contraction runs
// on warp MMAs, mma.sync m16n8k16 bf16 -> fp32, with sixteen W rows as the m16
// operand and the tokens as the n8 operand (one or two 8-token tiles; columns past M
// are zero).  The W operand is W' = bf16(level * bf16(s'_b)), the same values the
// tensor-core kernels use, built in registers from the codes through a byte -> bf16x2
// table and one bf16x2 multiply per two weights.
//
// Work split.  A unit is 32 W rows over all of K, so no partial sum ever leaves its
// CTA.  One persistent CTA per SM takes a contiguous run of units.
//
// Data movement (two producer warps, eight consumer warps).  A stage is 1024 k:
//   - codes: a ring of 16 KB stages, [4 chunks x 32 rows x 128 B] with the 128-byte
//     swizzle, one 3-D TMA box per stage (four 2-D boxes when K is not a multiple of
//     256), 3-6 stages deep.  TMA instructions are few and large because each costs
//     a fixed few hundred nanoseconds of the SM's copy engine;
//   - activations X (and, during a CTA's first unit, the adapter rows A): a second
//     ring of [16 chunks x M rows x 128 B] (and [16 x r x 128 B]) swizzled boxes, fed
//     by the second producer warp (these come from L2);
//   - block scales of a unit: one bulk copy of its 32 x K/64 bytes (contiguous in the
//     packed layout) plus the unit's second-level steps, double-buffered per unit.
//
// Fragment mapping.  Consumer warp w takes rows 16 (w % 2) .. +15 of the unit and the
// four blocks of 256-k chunk w / 2 of each stage.  In a block, lane (g, t) owns rows g
// and g + 8 of its tile and the 16 weights k = 16t .. 16t + 15 of each: 8 code bytes
// per row, one 64-bit load from the swizzled code row.  k-step q takes bytes 2q and
// 2q + 1 (k = 16t + 4q + {0,1} in slots 2t, 2t+1 and k = 16t + 4q + {2,3} in slots
// 2t+8, 2t+9); the lane's activations of token g (and g + 8) at the same 16 k are two
// 128-bit loads.  The MMA sums over its k slots in any order, so this pairing only has
// to agree between the two operands.  A table lookup is one byte permute and one
// 32-bit shared load per two weights.  A stage's four blocks are straight-line code
// (no per-block branch) into four (two for 16 tokens) accumulator sets, so their MMA
// chains overlap.
//
// The adapter product U = X A^T uses the same loop with the rows of A (bf16, r <= 16)
// as a second m16 operand; the warps of the first row tile compute it during the
// CTA's first unit, and the CTA keeps it in shared memory for the adapter term of all
// its units.
//
// Overlap with the preceding kernel (programmatic dependent launch): before waiting
// on the preceding grid a CTA only builds its table and initialises its barriers;
// every load follows griddepcontrol.wait.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {
namespace dec {

constexpr int kRows = 32;                       // W rows per unit
constexpr int kStageK = 1024;                   // k per pipeline stage
constexpr int kStageBlocks = kStageK / 64;      // 16 blocks = 8 block pairs
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 64;       // + two producer warps
constexpr int kMaxRank = 16;                    // adapter ranks fused on this path
constexpr int kMaxKB = 512;                     // 64-k blocks per row (n_in <= 32768)
constexpr int kCodeStage = kRows * kStageK / 2; // 16 KB
constexpr int kLutBytes = 256 * 32 * 4;         // one bf16x2 per byte value per lane
constexpr int kMaxCodeStages = 6;
constexpr int kMaxXaStages = 4;
constexpr int kPartFloats = 4 * kRows * 16;     // [chunk][row][token]
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
    int c3d;                 // codes map is 3-D (one box per stage)
    // byte offsets from the 1024-aligned shared-memory base
    int off_code, off_xa, xa_stage, off_sc, sc_stage, sc_q, off_part, off_upart, off_ufin, off_bars;
    float scaling;
    float level[16];
};

// d += A B
__device__ __forceinline__ void mma_acc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// This lane's table entry for byte c of w: (level[lo], level[hi]) as bf16x2.  The
// table is written before the CTA's first __syncthreads and only read afterwards, and
// w comes from a barrier-guarded load, so the load is free to move with its address.
__device__ __forceinline__ uint32_t lut_at(uint32_t lut_lane, uint32_t w, int c) {
    const uint32_t e = __byte_perm(w, 0u, 0x4440u | static_cast<uint32_t>(c));
    uint32_t v;
    asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(lut_lane + (e << 7)));
    return v;
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
    const int nA = p.r / 8;                                           // adapter n8 groups

    // 1. let the next kernel in the stream start launching
    pdl_launch_dependents();

    // 2. byte -> bf16x2 (level[lo], level[hi]) table, one copy per lane.  Lane i holds
    // level[i % 16] (constant-index reads keep the parameter block out of local
    // memory); a thread writes 16-byte piece f % 8 of entry f / 8, so a warp's stores
    // cover 512 contiguous bytes and no two lanes meet in a bank
    {
        float lvl = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((lane & 15) == i) lvl = p.level[i];
        const uint32_t base = smem_u32(smem);
        for (int f0 = 0; f0 < 256 * 8; f0 += kThreads) {
            const int f = f0 + static_cast<int>(threadIdx.x);
            const int e = min(f, 256 * 8 - 1) >> 3;
            const float lo = __shfl_sync(0xffffffffu, lvl, e & 15);
            const float hi = __shfl_sync(0xffffffffu, lvl, e >> 4);
            __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
            const uint32_t w = *reinterpret_cast<uint32_t *>(&v);
            if (f < 256 * 8) sts128(base + f * 16, make_uint4(w, w, w, w));
        }
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxCodeStages; ++i) { mbar_init(&code_full[i], 1); mbar_init(&code_empty[i], kConsumerWarps); }
        for (int i = 0; i < kMaxXaStages; ++i) { mbar_init(&xa_full[i], 1); mbar_init(&xa_empty[i], kConsumerWarps); }
        for (int i = 0; i < 2; ++i) { mbar_init(&sc_full[i], 33); mbar_init(&sc_empty[i], kConsumerWarps); }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kConsumerWarps && lane == 0) {
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmX);
        if (nA > 0) tma_prefetch_desc(&tmA);
    }
    __syncthreads();

    // 3. everything below may read what the preceding grid wrote
    pdl_wait();
    if (nu <= 0) return;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------- code and scale producer
        int slot = 0, round = 0, issued = 0, sc_issued = 0;
        bool ok = true;
        for (int ui = 0; ui < nu && ok; ++ui) {
            const int u = u0 + ui;
            // this unit's block scales and second-level steps
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
            // this unit's code stages
            for (int j = 0; j < nst; ++j) {
                if (round > 0 && !mbar_wait(&code_empty[slot], (round & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *dst = smem + p.off_code + slot * kCodeStage;
                    mbar_arrive_expect_tx(&code_full[slot], kCodeStage);
                    if (p.c3d) {
                        tma_load_3d(dst, &tmC, &code_full[slot], 0, u * kRows, j * (kStageK / 256));
                    } else {
#pragma unroll
                        for (int q = 0; q < kStageK / 256; ++q)
                            tma_load_2d(dst + q * (kRows * 128), &tmC, &code_full[slot], j * (kStageK / 2) + q * 128,
                                        u * kRows);
                    }
                }
                ++issued;
                if (++slot == p.dc) { slot = 0; ++round; }
            }
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
            int slot = 0, round = 0, issued = 0;
            bool ok = true;
            for (int ui = 0; ui < nu && ok; ++ui) {
                for (int j = 0; j < nst; ++j) {
                    if (round > 0 && !mbar_wait(&xa_empty[slot], (round & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const bool with_a = ui == 0 && nA > 0;
                    uint8_t *dst = smem + p.off_xa + slot * p.xa_stage;
                    mbar_arrive_expect_tx(&xa_full[slot], (p.M + (with_a ? p.r : 0)) * (kStageBlocks * 128));
                    tma_load_3d(dst, &tmX, &xa_full[slot], 0, 0, j * kStageBlocks);
                    if (with_a)
                        tma_load_3d(dst + p.M * (kStageBlocks * 128), &tmA, &xa_full[slot], 0, 0, j * kStageBlocks);
                    ++issued;
                    if (++slot == p.dx) { slot = 0; ++round; }
                }
            }
            for (int i = max(0, issued - p.dx); i < issued; ++i) mbar_drain(&xa_full[i % p.dx], (i / p.dx) & 1);
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    // A wait that times out sets the CTA's abort flag and the device error word (which
    // the host reports); the consumers then run on without waiting, so that all eight
    // consumer warps still reach every named barrier and the CTA exits.
    const int rt = warp & 1, bq = warp >> 1;            // row tile (16 rows), 256-k chunk of each stage
    const int g = lane >> 2, t = lane & 3;
    const int ctid = threadIdx.x;                      // 0 .. kConsumers-1
    const uint32_t lut_lane = smem_u32(smem) + lane * 4;
    const uint32_t code_base = smem_u32(smem + p.off_code);
    const uint32_t xa_base = smem_u32(smem + p.off_xa);
    float *part = reinterpret_cast<float *>(smem + p.off_part);
    float *upart = reinterpret_cast<float *>(smem + p.off_upart);
    float *ufin = reinterpret_cast<float *>(smem + p.off_ufin);
    const bool tok0 = g < p.M, tok1 = NT > 1 && g + 8 < p.M;
    const bool do_u = rt == 0 && p.r > 0;               // these warps also form U = X A^T
    const bool arow1 = g + 8 < p.r;                     // A row g + 8 exists (r = 16)
    const int brow = ctid & 31;                         // epilogue row
    const int R0 = 16 * rt + g;                         // unit rows of this lane: R0 and R0 + 8
    // this lane's 8 code bytes of block c of its chunk in row R0: 16-byte unit 2c + t/2
    // of the row's 128 bytes (stored at unit (2c + t/2) ^ (R0 % 8), R0 % 8 = g), half t%2
    const uint32_t c_lane =
        code_base + uint32_t(bq * (kRows * 128) + R0 * 128 + ((((t >> 1) ^ g) << 4) | ((t & 1) << 3)));
    // X and A lines of the stage's 64-k chunks: line * 128 + (unit ^ (line % 8)) * 16
    auto line_addr = [](uint32_t base, int line, int unit) {
        return base + uint32_t(line) * 128u + (uint32_t(unit ^ (line & 7)) << 4);
    };

    int cslot = 0, cph = 0, xslot = 0, xph = 0;
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
        if (lane == 0) mbar_wait(&sc_full[sb], (ui >> 1) & 1, abort_flag);
        __syncwarp();
        const uint32_t sq = smem_u32(smem + p.off_sc + sb * p.sc_stage);
        const uint32_t s2 = sq + p.sc_q;
        // flat block index of the unit's first block, modulo one second-level group: the
        // unit's steps were copied starting from the group holding that block
        const int fb_lo = static_cast<int>((int64_t(n0) * KB) & 255);
        const int row_q0 = R0 * KB, row_q1 = (R0 + 8) * KB;

        // the block's scale s'_b = q_b * d_g of a row, rounded to bf16 and paired; a block
        // past the end of K gets 0 (its codes and activations are the copies' zero fill)
        auto scale_pair = [&](int row_q, int kb) {
            const float sv = static_cast<float>(lds_u8(sq + uint32_t(row_q + kb))) *
                             lds_f32(s2 + uint32_t(((fb_lo + row_q + kb) >> 8) << 2));
            __nv_bfloat162 v = __float2bfloat162_rn(kb < KB ? sv : 0.f);
            return *reinterpret_cast<uint32_t *>(&v);
        };
        // kAcc accumulator sets, one per block modulo kAcc, keep independent MMA chains
        constexpr int kAcc = NT == 1 ? 4 : 2;
        float acc[kAcc][NT][4], accU[NT][4];
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                accU[a][b] = 0.f;
#pragma unroll
                for (int h = 0; h < kAcc; ++h) acc[h][a][b] = 0.f;
            }
        // one stage of this warp: the four blocks of its chunk, straight-line code
        auto stage = [&](auto with_u, uint32_t cs, uint32_t xs, int j) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int kc = 4 * bq + c;                   // 64-k chunk of the stage
                const int kb = j * kStageBlocks + kc;        // block of the row
                // rows R0, R0 + 8: 16 weights each, k = 16t .. 16t + 15 of the block
                const uint32_t ca = cs ^ uint32_t(c << 5);
                const uint2 w0 = lds64(ca);
                const uint2 w1 = lds64(ca + 8 * 128);
                // tokens g and g + 8 at the same 16 k
                uint4 xa0 = make_uint4(0, 0, 0, 0), xb0 = xa0, xa1 = xa0, xb1 = xa0;
                if (tok0) {
                    xa0 = lds128(line_addr(xs, kc * p.M + g, 2 * t));
                    xb0 = lds128(line_addr(xs, kc * p.M + g, 2 * t + 1));
                }
                if (tok1) {
                    xa1 = lds128(line_addr(xs, kc * p.M + g + 8, 2 * t));
                    xb1 = lds128(line_addr(xs, kc * p.M + g + 8, 2 * t + 1));
                }
                const uint32_t s0 = scale_pair(row_q0, kb), s1 = scale_pair(row_q1, kb);
                // k-step q takes bytes 2q, 2q+1 of each row's 8: k = 16t + 4q + {0,1} in
                // slots 2t, 2t+1 and 16t + 4q + {2,3} in slots 2t+8, 2t+9; the activations
                // supply the same k in the same slots.  W' = bf16(level * bf16(s'_b)).
                const uint32_t xw0[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xb0.x, xb0.y, xb0.z, xb0.w};
                const uint32_t xw1[8] = {xa1.x, xa1.y, xa1.z, xa1.w, xb1.x, xb1.y, xb1.z, xb1.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t r0w = (q < 2) ? w0.x : w0.y, r1w = (q < 2) ? w1.x : w1.y;
                    const int by = 2 * (q & 1);
                    const uint32_t a0 = bf16x2_mul(lut_at(lut_lane, r0w, by), s0);
                    const uint32_t a2 = bf16x2_mul(lut_at(lut_lane, r0w, by + 1), s0);
                    const uint32_t a1 = bf16x2_mul(lut_at(lut_lane, r1w, by), s1);
                    const uint32_t a3 = bf16x2_mul(lut_at(lut_lane, r1w, by + 1), s1);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint32_t *xw = nt ? xw1 : xw0;
                        mma_acc(acc[c % kAcc][nt], a0, a1, a2, a3, xw[2 * q], xw[2 * q + 1]);
                    }
                }
                if constexpr (decltype(with_u)::value) {
                    // A rows g and g + 8 at the same 16 k, straight from the stage (bf16)
                    const int al = kc * p.r + g;
                    const uint32_t ab = xs + uint32_t(p.M * (kStageBlocks * 128));
                    const uint4 aa0 = lds128(line_addr(ab, al, 2 * t)), ab0 = lds128(line_addr(ab, al, 2 * t + 1));
                    uint4 aa1 = make_uint4(0, 0, 0, 0), ab1 = aa1;
                    if (arow1) {
                        aa1 = lds128(line_addr(ab, al + 8, 2 * t));
                        ab1 = lds128(line_addr(ab, al + 8, 2 * t + 1));
                    }
                    const uint32_t aw0[8] = {aa0.x, aa0.y, aa0.z, aa0.w, ab0.x, ab0.y, ab0.z, ab0.w};
                    const uint32_t aw1[8] = {aa1.x, aa1.y, aa1.z, aa1.w, ab1.x, ab1.y, ab1.z, ab1.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint32_t *xw = nt ? xw1 : xw0;
                            mma_acc(accU[nt], aw0[2 * q], aw1[2 * q], aw0[2 * q + 1], aw1[2 * q + 1], xw[2 * q],
                                    xw[2 * q + 1]);
                        }
                }
            }
        };
        const bool u_here = first && do_u;
        for (int j = 0; j < nst; ++j) {
            if (lane == 0) {   // one lane polls; the warp barrier orders the others after it
                mbar_wait(&code_full[cslot], cph, abort_flag);
                mbar_wait(&xa_full[xslot], xph, abort_flag);
            }
            __syncwarp();
            const uint32_t cs = c_lane + uint32_t(cslot * kCodeStage);
            const uint32_t xs = xa_base + uint32_t(xslot * p.xa_stage);
            if (u_here) stage(std::true_type{}, cs, xs, j);
            else stage(std::false_type{}, cs, xs, j);
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&code_empty[cslot]);
                mbar_arrive(&xa_empty[xslot]);
            }
            if (++cslot == p.dc) { cslot = 0; cph ^= 1; }
            if (++xslot == p.dx) { xslot = 0; xph ^= 1; }
        }
#pragma unroll
        for (int h = 1; h < kAcc; ++h)
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[0][a][b] += acc[h][a][b];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sc_empty[sb]);

        // partial sums of chunk bq -> part[bq][row][token]; D[row][token] of the MMA has
        // rows g, g + 8 and tokens 2t, 2t + 1 of each 8-token tile in this lane
        float *pb = part + bq * kRows * 16;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int m0 = 8 * nt + 2 * t;
            pb[R0 * 16 + m0] = acc[0][nt][0];
            pb[R0 * 16 + m0 + 1] = acc[0][nt][1];
            pb[(R0 + 8) * 16 + m0] = acc[0][nt][2];
            pb[(R0 + 8) * 16 + m0 + 1] = acc[0][nt][3];
        }
        if (first && do_u) {
            float *ub = upart + bq * 256;   // [adapter row][token]
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int m0 = 8 * nt + 2 * t;
                ub[g * 16 + m0] = accU[nt][0];
                ub[g * 16 + m0 + 1] = accU[nt][1];
                ub[(g + 8) * 16 + m0] = accU[nt][2];
                ub[(g + 8) * 16 + m0 + 1] = accU[nt][3];
            }
        }
        consumer_sync();
        if (first && p.r > 0) {
            // ufin[token][adapter row]
            for (int e = ctid; e < 256; e += kConsumers) {
                const int m = e >> 4, jr = e & 15;
                const int src = jr * 16 + m;
                ufin[e] = upart[src] + upart[256 + src] + upart[512 + src] + upart[768 + src];
            }
            consumer_sync();
            if (p.U_save && blockIdx.x == 0) {
                for (int e = ctid; e < p.M * p.r; e += kConsumers) {
                    const int m = e / p.r, jr = e - m * p.r;
                    __nv_bfloat16 hv = __float2bfloat16_rn(ufin[m * 16 + jr]);
                    p.U_save[e] = *reinterpret_cast<uint16_t *>(&hv);
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
                __nv_bfloat16 hv = __float2bfloat16_rn(fmaf(p.scaling, l, base));
                p.Y[int64_t(m) * p.N + n] = *reinterpret_cast<uint16_t *>(&hv);
            }
        }
        if (ui + 1 < nu) consumer_sync();   // the next unit rewrites the partial sums
    }
}

}  // namespace dec
}  // namespace qlora
