// decode_mma.cuh -- small-M forward (M <= 16 tokens): the weight-streaming path.
//
//   Y[m, n] = sum_k X[m, k] W'[n, k] + scaling * sum_j U[m, j] B[n, j],   U = X A^T
//
// With at most 16 tokens the forward is bound by streaming the packed weight
// (0.516 B per weight) from HBM.  tcgen05 cannot keep up at such a narrow N (its
// per-instruction cost is paid for 128 x 16 x 16 of work), so the contraction runs
// on warp MMAs, mma.sync m16n8k16 bf16 -> fp32, with the tokens as the m16 operand
// (rows past M are zero) and eight dequantized W rows as the n8 operand, which a
// thread builds in registers straight from the codes it loaded.
//
// Operand pairing.  A thread (g = lane / 4, t = lane % 4) loads bytes [8t, 8t+8)
// of each 32-byte (64-weight) block of W row n0 + 8*grp + g.  In k-step j (four per
// block) its two B registers are the bf16x2 expansions of bytes 2j and 2j+1, i.e.
// weights k = 16t + 4j .. 16t + 4j + 3 of the block; its A registers are the same
// four k of tokens g and g+8.  The MMA sums over k in its own order, so this pairing
// of fragment slots with k positions only has to agree between A and B.
//
// Work split.  A CTA (4 warps) owns 64 W rows and a contiguous range of 64-k blocks;
// the S CTAs of a cluster cover all of K for the same rows (S = 1, 2, 4 or 8).
// Each warp takes a contiguous quarter of the CTA's blocks and accumulates all 64 rows.  Partial sums
// are added across warps in shared memory and across the cluster through
// distributed shared memory by the cluster's first CTA, which also adds the
// adapter term and writes Y.  U is computed by the same loop: the rows of A are a
// second set of n8 operands (bf16, no dequant), summed like the base rows.
//
// Overlap with the preceding kernel (programmatic dependent launch): the weights
// are frozen, so before waiting on the preceding grid a CTA only prefetches its
// code and scale bytes into L2 (which is coherent) and builds its lookup table;
// every real load follows griddepcontrol.wait.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {
namespace dec {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kRows = 64;                  // W rows per CTA
constexpr int kGroups = kRows / 8;         // n8 operands per k-step
constexpr int kMaxRank = 16;               // adapter ranks fused on this path
constexpr int kMaxBlocks = 64;             // 64-k blocks per CTA (scale table size)
constexpr int kLutWords = 256 * 32;

struct Params {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *scales2;
    const uint16_t *X;       // [M, K]
    const uint16_t *Alora;   // [r, K] or nullptr
    const uint16_t *Blora;   // [N, r] or nullptr
    uint16_t *Y;             // [M, N]
    uint16_t *U_save;        // [M, r] or nullptr
    int M, N, K, r;
    int S;                   // CTAs per cluster along K
    int blocks_per_cta;      // 64-k blocks per CTA (<= kMaxBlocks)
    float scaling;
    float level[16];
};

// LUT 32 KB (reused for the per-warp partials after the main loop), scale table,
// then this CTA's partial sums (read by the cluster's first CTA)
constexpr int kScaleBytes = 0;
constexpr int kPartFloats = 16 * kRows + 16 * kMaxRank;
__host__ __device__ constexpr int smem_bytes() { return 128 + kLutWords * 4 + kScaleBytes + kPartFloats * 4; }

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
    return v;
}
__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
// 8 bytes of a code row; a miss fetches the whole 256-byte aligned span into L2, which
// holds the warp's next blocks of the same row
__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L2::256B.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

template <int NT>   // token tiles of 8: 1 for M <= 8, 2 for M <= 16
__global__ void __launch_bounds__(kThreads) decode_kernel(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint32_t *sLut = reinterpret_cast<uint32_t *>(smem);
    float *red = reinterpret_cast<float *>(smem);                       // after the main loop
    float *redU = red + kWarps * 16 * kRows;
    float *part = reinterpret_cast<float *>(smem + kLutWords * 4 + kScaleBytes);   // [16][kRows]
    float *partU = part + 16 * kRows;                                             // [16][kMaxRank]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t rank = p.S > 1 ? cluster_ctarank() : 0u;
    const int n0 = (blockIdx.x / p.S) * kRows;
    const int KB = p.K / 64;
    const int kb0 = int(rank) * p.blocks_per_cta;
    const int kb1 = min(KB, kb0 + p.blocks_per_cta);
    const int nbc = max(0, kb1 - kb0);
    const int64_t row_bytes = p.K / 2;

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
        const uint32_t base = smem_u32(sLut + e * 32);
#pragma unroll
        for (int c = 0; c < 8; ++c) sts128(base + c * 16, make_uint4(w, w, w, w));
    }

    // 3. everything below may read what the preceding grid wrote
    pdl_wait();
    __syncthreads();   // the table is complete

    // 5. main loop: this warp's blocks, all 64 rows (+ the adapter rows)
    const uint32_t lut = smem_u32(sLut) + lane * 4;
    const int nU = (p.Alora && p.r > 0) ? (p.r + 7) / 8 : 0;
    float acc[kGroups][4];
    float accU[kMaxRank / 8][4];
#pragma unroll
    for (int i = 0; i < kGroups; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxRank / 8; ++i) accU[i][0] = accU[i][1] = accU[i][2] = accU[i][3] = 0.f;

    const bool tok0 = g < p.M, tok1 = NT > 1 && g + 8 < p.M;
    const uint16_t *xrow0 = p.X + int64_t(g) * p.K + 16 * t;
    const uint16_t *xrow1 = p.X + int64_t(g + 8) * p.K + 16 * t;
    const uint8_t *crow[kGroups];
    bool rvalid[kGroups];
#pragma unroll
    for (int grp = 0; grp < kGroups; ++grp) {
        const int n = n0 + 8 * grp + g;
        rvalid[grp] = n < p.N;
        crow[grp] = p.codes + int64_t(rvalid[grp] ? n : 0) * row_bytes + 8 * t;
    }

    const uint8_t *srow[kGroups];
#pragma unroll
    for (int grp = 0; grp < kGroups; ++grp) {
        const int n = rvalid[grp] ? n0 + 8 * grp + g : 0;
        srow[grp] = p.scales + int64_t(n) * KB;
    }
    const int64_t s2base = int64_t(n0 + g) * KB;   // block index of row n0 + g, block 0
    const uint16_t *arow0 = p.Alora ? p.Alora + int64_t(g) * p.K + 16 * t : nullptr;

    // everything a block needs is loaded one block ahead: codes, block scales (q and the
    // group step d), activations of tokens g and g+8, and the adapter rows
    uint2 cnext[kGroups];
    uint32_t qn[kGroups];
    float dn[kGroups];
    uint4 xn[4];
    uint4 an[kMaxRank / 8][2];
    // warp w takes a contiguous run of the CTA's blocks
    const int per_warp = (nbc + kWarps - 1) / kWarps;
    const int wk0 = kb0 + warp * per_warp, wk1 = min(kb1, wk0 + per_warp);
    int kb = wk0;
    auto load_block = [&](int k) {
        const bool in = k < wk1;
#pragma unroll
        for (int grp = 0; grp < kGroups; ++grp) {
            const bool v = in && rvalid[grp];
            cnext[grp] = v ? ldg_nc_v2(crow[grp] + int64_t(k) * 32) : make_uint2(0, 0);
            qn[grp] = v ? uint32_t(__ldg(srow[grp] + k)) : 0u;
            dn[grp] = v ? __ldg(p.scales2 + ((s2base + int64_t(8 * grp) * KB + k) >> 8)) : 0.f;
        }
        // tokens g and g+8, k = 64 k + 16 t .. + 15
        xn[0] = xn[1] = xn[2] = xn[3] = make_uint4(0, 0, 0, 0);
        if (in && tok0) {
            xn[0] = ldg_nc_v4(xrow0 + int64_t(k) * 64);
            xn[1] = ldg_nc_v4(xrow0 + int64_t(k) * 64 + 8);
        }
        if (in && tok1) {
            xn[2] = ldg_nc_v4(xrow1 + int64_t(k) * 64);
            xn[3] = ldg_nc_v4(xrow1 + int64_t(k) * 64 + 8);
        }
#pragma unroll
        for (int u = 0; u < kMaxRank / 8; ++u) {
            an[u][0] = an[u][1] = make_uint4(0, 0, 0, 0);
            if (in && u < nU && 8 * u + g < p.r) {
                const uint16_t *ar = arow0 + int64_t(8 * u) * p.K + int64_t(k) * 64;
                an[u][0] = ldg_nc_v4(ar);
                an[u][1] = ldg_nc_v4(ar + 8);
            }
        }
    };
    load_block(kb);

    for (; kb < wk1; ++kb) {
        uint2 ccur[kGroups];
        uint32_t s2c[kGroups];
#pragma unroll
        for (int grp = 0; grp < kGroups; ++grp) {
            ccur[grp] = cnext[grp];
            __nv_bfloat162 s2b = __float2bfloat162_rn(__fmul_rn(static_cast<float>(qn[grp]), dn[grp]));
            s2c[grp] = *reinterpret_cast<uint32_t *>(&s2b);
        }
        const uint32_t xg[8] = {xn[0].x, xn[0].y, xn[0].z, xn[0].w, xn[1].x, xn[1].y, xn[1].z, xn[1].w};
        const uint32_t xh[8] = {xn[2].x, xn[2].y, xn[2].z, xn[2].w, xn[3].x, xn[3].y, xn[3].z, xn[3].w};
        uint32_t aw[kMaxRank / 8][8];
#pragma unroll
        for (int u = 0; u < kMaxRank / 8; ++u) {
            aw[u][0] = an[u][0].x; aw[u][1] = an[u][0].y; aw[u][2] = an[u][0].z; aw[u][3] = an[u][0].w;
            aw[u][4] = an[u][1].x; aw[u][5] = an[u][1].y; aw[u][6] = an[u][1].z; aw[u][7] = an[u][1].w;
        }
        load_block(kb + 1);

#pragma unroll
        for (int grp = 0; grp < kGroups; ++grp) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t word = j < 2 ? ccur[grp].x : ccur[grp].y;
                const uint32_t sh = 16 * (j & 1);
                const uint32_t e0 = (word >> sh) & 0xFFu, e1 = (word >> (sh + 8)) & 0xFFu;
                const uint32_t b0 = bf16x2_mul(lds32(lut + (e0 << 7)), s2c[grp]);
                const uint32_t b1 = bf16x2_mul(lds32(lut + (e1 << 7)), s2c[grp]);
                mma_bf16_16816(acc[grp], xg[2 * j], NT > 1 ? xh[2 * j] : 0u, xg[2 * j + 1],
                               NT > 1 ? xh[2 * j + 1] : 0u, b0, b1);
            }
        }
#pragma unroll
        for (int u = 0; u < kMaxRank / 8; ++u) {
            if (u < nU) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_bf16_16816(accU[u], xg[2 * j], NT > 1 ? xh[2 * j] : 0u, xg[2 * j + 1],
                                   NT > 1 ? xh[2 * j + 1] : 0u, aw[u][2 * j], aw[u][2 * j + 1]);
            }
        }
    }

    // 6. partial sums: warps -> shared memory -> this CTA's part
    __syncthreads();   // every warp is done with the table the partials overwrite
#pragma unroll
    for (int grp = 0; grp < kGroups; ++grp) {
        float *r0 = red + (warp * 16 + g) * kRows + 8 * grp + 2 * t;
        r0[0] = acc[grp][0];
        r0[1] = acc[grp][1];
        float *r1 = red + (warp * 16 + g + 8) * kRows + 8 * grp + 2 * t;
        r1[0] = acc[grp][2];
        r1[1] = acc[grp][3];
    }
#pragma unroll
    for (int u = 0; u < kMaxRank / 8; ++u) {
        float *r0 = redU + (warp * 16 + g) * kMaxRank + 8 * u + 2 * t;
        r0[0] = accU[u][0];
        r0[1] = accU[u][1];
        float *r1 = redU + (warp * 16 + g + 8) * kMaxRank + 8 * u + 2 * t;
        r1[0] = accU[u][2];
        r1[1] = accU[u][3];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 16 * kRows; i += kThreads) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w * 16 * kRows + i];
        part[i] = v;
    }
    for (int i = threadIdx.x; i < 16 * kMaxRank; i += kThreads) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += redU[w * 16 * kMaxRank + i];
        partU[i] = v;
    }

    // 7. the cluster's first CTA adds the other CTAs' partials and writes the outputs
    if (p.S > 1) cluster_sync(); else __syncthreads();
    if (rank == 0) {
        if (p.S > 1) {
            for (int i = threadIdx.x; i < 16 * kRows; i += kThreads) {
                const uint32_t a = smem_u32(part + i);
                float v[8];
#pragma unroll
                for (int rr = 1; rr < 8; ++rr) v[rr] = rr < p.S ? ld_dsmem_f32(mapa_shared(a, rr)) : 0.f;
                float sum = part[i];
#pragma unroll
                for (int rr = 1; rr < 8; ++rr) sum += v[rr];
                part[i] = sum;
            }
            for (int i = threadIdx.x; i < 16 * kMaxRank; i += kThreads) {
                const uint32_t a = smem_u32(partU + i);
                float v[8];
#pragma unroll
                for (int rr = 1; rr < 8; ++rr) v[rr] = rr < p.S ? ld_dsmem_f32(mapa_shared(a, rr)) : 0.f;
                float sum = partU[i];
#pragma unroll
                for (int rr = 1; rr < 8; ++rr) sum += v[rr];
                partU[i] = sum;
            }
        }
        __syncthreads();
        // thread -> (row, tokens): the adapter row of B is read once, 8 ranks per 16-byte load
        for (int i = threadIdx.x; i < kRows * ((p.M + 3) / 4); i += kThreads) {
            const int row = i % kRows, m0 = (i / kRows) * 4;
            const int n = n0 + row;
            if (n >= p.N) continue;
            float l[4] = {0.f, 0.f, 0.f, 0.f};
            if (nU > 0) {
                for (int j0 = 0; j0 < p.r; j0 += 8) {
                    const uint4 bv = ldg_nc_v4(p.Blora + int64_t(n) * p.r + j0);
                    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float b = __uint_as_float((e & 1) ? (bw[e >> 1] & 0xFFFF0000u) : (bw[e >> 1] << 16));
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) l[mm] = fmaf(partU[(m0 + mm) * kMaxRank + j0 + e], b, l[mm]);
                    }
                }
            }
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                const int m = m0 + mm;
                if (m < p.M) {
                    const float y = fmaf(p.scaling, l[mm], part[m * kRows + row]);
                    __nv_bfloat16 h = __float2bfloat16_rn(y);
                    p.Y[int64_t(m) * p.N + n] = *reinterpret_cast<uint16_t *>(&h);
                }
            }
        }
        if (p.U_save && nU > 0 && blockIdx.x == 0) {
            for (int i = threadIdx.x; i < p.M * p.r; i += kThreads) {
                const int m = i / p.r, j = i - m * p.r;
                __nv_bfloat16 h = __float2bfloat16_rn(partU[m * kMaxRank + j]);
                p.U_save[i] = *reinterpret_cast<uint16_t *>(&h);
            }
        }
    }
    // the first CTA has read the others' partials before any of them exits
    if (p.S > 1) cluster_sync();
}

}  // namespace dec
}  // namespace qlora
