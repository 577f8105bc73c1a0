// quant_kernels.cuh -- 4-bit block encode with (or without) double quantization of the
// scales, the standalone full-tensor dequant and the LoRA merge.  All are bit-exact.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "scale_src.cuh"

namespace qlora {

struct CodebookArg {
    float level[16];
    float thresh[16];
};

// Encode.  One CTA per 256 first-level blocks (one double-quant group): 8 warps; a
// warp step covers 128 consecutive weights, four per lane from one 128-bit load, so a
// block of 64 spans 16 lanes and a block of 128 the whole warp.  The block absmax is a
// shuffle reduction over the block's lanes; each lane then encodes its four weights
// into two code bytes (element 2j low nibble, 2j+1 high nibble).  Then the group max
// gives d_g and each thread quantizes one block scale (double quant), or stores the
// fp32 absmax itself (no double quant).  With kAfterDq the codes are taken in a second
// pass against the dequantized scale s'_b = fp32(q_b d_g) instead of a_b.
constexpr int kEncThreads = 256;

__device__ __forceinline__ uint32_t code_of(float n, const float *thr) {
    // #{k : n >= thr[k]} by binary search over the 15 sorted thresholds (thr[15] = inf)
    uint32_t c = 0;
    c += (n >= thr[c + 7]) ? 8u : 0u;
    c += (n >= thr[c + 3]) ? 4u : 0u;
    c += (n >= thr[c + 1]) ? 2u : 0u;
    c += (n >= thr[c]) ? 1u : 0u;
    return c;
}

__device__ __forceinline__ uint16_t encode4(float4 v, float scale, const float *thr) {
    float n0 = 0.f, n1 = 0.f, n2 = 0.f, n3 = 0.f;
    if (scale > 0.f) {
        n0 = __fdiv_rn(v.x, scale);
        n1 = __fdiv_rn(v.y, scale);
        n2 = __fdiv_rn(v.z, scale);
        n3 = __fdiv_rn(v.w, scale);
    }
    const uint32_t c = code_of(n0, thr) | (code_of(n1, thr) << 4) | (code_of(n2, thr) << 8) | (code_of(n3, thr) << 12);
    return static_cast<uint16_t>(c);
}

template <int kBlock, bool kDq, bool kAfterDq>
__global__ void __launch_bounds__(kEncThreads) nf4_encode_kernel(const float *__restrict__ W,
                                                                 uint8_t *__restrict__ codes,
                                                                 uint8_t *__restrict__ scales,
                                                                 float *__restrict__ scales2, int64_t nblocks,
                                                                 const CodebookArg cb) {
    static_assert(kBlock == 64 || kBlock == 128, "blocks of 64 or 128 weights");
    static_assert(kDq || !kAfterDq, "codes against the dequantized scale need double quantization");
    constexpr int kLanesPerBlock = kBlock / 4;
    constexpr int kBlocksPerStep = 128 / kBlock;
    constexpr int U = 4;                           // warp steps in flight
    __shared__ float s_thr[16];
    __shared__ float s_absmax[256];
    __shared__ float s_scale[kAfterDq ? 256 : 1];
    __shared__ float s_wmax[8];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < 16) s_thr[tid] = cb.thresh[tid];
    const int64_t g = blockIdx.x;
    const int64_t b0 = g * 256;
    const int nb = static_cast<int>(nblocks - b0 < 256 ? nblocks - b0 : 256);
    const int nsteps = (nb * kBlock + 127) / 128;
    const float *Wg = W + b0 * kBlock;
    uint16_t *Cg = reinterpret_cast<uint16_t *>(codes + b0 * (kBlock / 2));
    const int sub = lane / kLanesPerBlock;         // which block of the step this lane's weights are in
    __syncthreads();

    for (int t0 = warp; t0 < nsteps; t0 += 8 * U) {
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = t0 + 8 * u;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < nsteps && t * kBlocksPerStep + sub < nb)
                v[u] = __ldcs(reinterpret_cast<const float4 *>(Wg + int64_t(t) * 128) + lane);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = t0 + 8 * u;
            if (t >= nsteps) break;  // warp-uniform
            const int blk = t * kBlocksPerStep + sub;
            float a = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
#pragma unroll
            for (int o = kLanesPerBlock / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            if (blk < nb) {
                if (!kAfterDq) Cg[t * 32 + lane] = encode4(v[u], a, s_thr);
                if (lane % kLanesPerBlock == 0) s_absmax[blk] = a;
            }
        }
    }
    __syncthreads();

    if (kDq) {
        // second level: d_g = fp32(max a_b / 255); q_b = clamp(rint(fp32(a_b / d_g)), 0, 255)
        const float a = (tid < nb) ? s_absmax[tid] : 0.f;
        float m = a;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_wmax[warp] = m;
        __syncthreads();
        float c2 = s_wmax[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) c2 = fmaxf(c2, s_wmax[i]);
        const float d = __fdiv_rn(c2, 255.f);
        if (tid < nb) {
            uint32_t q = 0;
            if (d > 0.f) {
                const float r = rintf(__fdiv_rn(a, d));
                q = static_cast<uint32_t>(fminf(fmaxf(r, 0.f), 255.f));
            }
            scales[b0 + tid] = static_cast<uint8_t>(q);
            if (kAfterDq) s_scale[tid] = __fmul_rn(static_cast<float>(q), d);
        }
        if (tid == 0) scales2[g] = d;
    } else {
        if (tid < nb) reinterpret_cast<float *>(scales)[b0 + tid] = s_absmax[tid];
    }

    if (kAfterDq) {
        __syncthreads();
        // codes against s'_b: the group's weights again (mostly from L2)
        for (int t0 = warp; t0 < nsteps; t0 += 8 * U) {
            float4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int t = t0 + 8 * u;
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (t < nsteps && t * kBlocksPerStep + sub < nb)
                    v[u] = __ldcs(reinterpret_cast<const float4 *>(Wg + int64_t(t) * 128) + lane);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int t = t0 + 8 * u;
                if (t >= nsteps) break;
                const int blk = t * kBlocksPerStep + sub;
                if (blk < nb) Cg[t * 32 + lane] = encode4(v[u], s_scale[blk], s_thr);
            }
        }
    }
}

// Full dequant: a thread handles 16 weights (8 code bytes, one 64-weight run has four
// threads).  kBf16 selects the output type: fp32 w' = fp32(c[code] * s_b), or
// bf16 = RNE(w').
template <bool kBf16>
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint8_t *__restrict__ codes, const ScaleSrc sc,
                                                          void *__restrict__ out, int64_t n16, const CodebookArg cb) {
    __shared__ float s_lv[16];
    if (threadIdx.x < 16) s_lv[threadIdx.x] = cb.level[threadIdx.x];
    __syncthreads();
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n16; i += int64_t(gridDim.x) * blockDim.x) {
        const uint2 cw = __ldcs(reinterpret_cast<const uint2 *>(codes) + i);
        const float s = block_scale(sc, i >> 2);
        float w[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            w[j] = __fmul_rn(s_lv[(cw.x >> (4 * j)) & 15u], s);
            w[8 + j] = __fmul_rn(s_lv[(cw.y >> (4 * j)) & 15u], s);
        }
        if (kBf16) {
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                __nv_bfloat162 p = __floats2bfloat162_rn(w[2 * j], w[2 * j + 1]);
                o[j] = *reinterpret_cast<uint32_t *>(&p);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(out) + 2 * i;
            __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
            __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
        } else {
            float4 *dst = reinterpret_cast<float4 *>(out) + 4 * i;
#pragma unroll
            for (int j = 0; j < 4; ++j) __stcs(dst + j, make_float4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]));
        }
    }
}

// Q8_0 encode ("Training LoRA directly on GGUF quantized weights" page, section 1.1:
// 32 weights share one fp16 scale).  A lane takes four weights (one 128-bit load), so a
// block spans 8 lanes and a warp step covers 128 weights.  d = fp16(a / 127), taken
// from the float32 quotient (fp32 keeps 24 >= 2 * 11 + 2 bits, so rounding twice gives
// the fp16 of the exact quotient); q = clamp(rint(fp32(w / d)), -127, 127); d = 0 gives
// q = 0.
__global__ void __launch_bounds__(256) q8_0_encode_kernel(const float *__restrict__ W, int8_t *__restrict__ q,
                                                          uint16_t *__restrict__ d, int64_t numel) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nsteps = (numel + 127) / 128;
    for (int64_t t = int64_t(blockIdx.x) * 8 + warp; t < nsteps; t += int64_t(gridDim.x) * 8) {
        const int64_t e0 = t * 128 + lane * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e0 < numel) v = __ldcs(reinterpret_cast<const float4 *>(W + e0));
        float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const __half dh = __float2half_rn(__fdiv_rn(a, 127.f));
        const float df = __half2float(dh);
        auto code = [&](float x) -> uint32_t {
            if (!(df > 0.f)) return 0u;
            const float r = fminf(fmaxf(rintf(__fdiv_rn(x, df)), -127.f), 127.f);
            return static_cast<uint32_t>(static_cast<int32_t>(r)) & 0xFFu;
        };
        if (e0 < numel) {
            reinterpret_cast<uint32_t *>(q)[e0 >> 2] = code(v.x) | (code(v.y) << 8) | (code(v.z) << 16) | (code(v.w) << 24);
            if ((lane & 7) == 0) d[e0 >> 5] = __half_as_ushort(dh);
        }
    }
}

// Q8_0 dequant: a thread handles 16 weights (one 128-bit load of codes, one fp16
// scale): w' = q * d, exact in float32, or bf16 = RNE(w').
template <bool kBf16>
__global__ void __launch_bounds__(256) q8_0_dequant_kernel(const int8_t *__restrict__ q,
                                                           const uint16_t *__restrict__ d, void *__restrict__ out,
                                                           int64_t n16) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n16; i += int64_t(gridDim.x) * blockDim.x) {
        const uint4 c = __ldcs(reinterpret_cast<const uint4 *>(q) + i);
        const float s = __half2float(__ushort_as_half(__ldg(d + (i >> 1))));
        const uint32_t words[4] = {c.x, c.y, c.z, c.w};
        if (kBf16) {
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) q8_word_to_bf16x2(words[j], s, o[2 * j], o[2 * j + 1]);
            uint4 *dst = reinterpret_cast<uint4 *>(out) + 2 * i;
            __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
            __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
        } else {
            float4 *dst = reinterpret_cast<float4 *>(out) + 4 * i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int32_t w = static_cast<int32_t>(words[j]);
                const float f0 = __fmul_rn(static_cast<float>(static_cast<int8_t>(w & 0xFF)), s);
                const float f1 = __fmul_rn(static_cast<float>(static_cast<int8_t>((w >> 8) & 0xFF)), s);
                const float f2 = __fmul_rn(static_cast<float>(static_cast<int8_t>((w >> 16) & 0xFF)), s);
                const float f3 = __fmul_rn(static_cast<float>(static_cast<int8_t>((w >> 24) & 0xFF)), s);
                __stcs(dst + j, make_float4(f0, f1, f2, f3));
            }
        }
    }
}

// LoRA merge, the step before requantization.
//   m = bf16(RN32(bf16(w') + s * sum_j B[n, j] A[j, k])):
// the dequantized base in bf16, the adapter product and the add in fp64 with j
// ascending, then float32 and bf16 rounding; m is stored as float32, the input of the
// encode kernel.  A bf16 x bf16 product is exact in fp64 (16 significant bits, and the
// exponent range of fp64 holds every such product), so the fused multiply-add
// RN(acc + b a) used here equals the separate product and sum.
// A thread takes kMergeCols consecutive weights of kMergeRows rows: each A value it
// loads and widens serves every row, and B of the CTA's rows sits in shared memory as
// fp64.  Rows run over blockIdx.y (in groups of kMergeRows), weights over x.
constexpr int kMergeRows = 4, kMergeCols = 4, kMergeThreads = 256, kMergeMaxR = 128;
__device__ __forceinline__ float merge_one(float level, float s, double sd, double acc) {
    const float wb = __bfloat162float(__float2bfloat16_rn(__fmul_rn(level, s)));
    const double t = __dadd_rn(static_cast<double>(wb), __dmul_rn(sd, acc));
    return __bfloat162float(__float2bfloat16_rn(__double2float_rn(t)));
}
__global__ void __launch_bounds__(kMergeThreads) nf4_lora_merge_kernel(const uint8_t *__restrict__ codes,
                                                                       const ScaleSrc sc,
                                                                       const uint16_t *__restrict__ A,
                                                                       const uint16_t *__restrict__ B, int r,
                                                                       float scaling, int64_t N, int64_t K,
                                                                       float *__restrict__ out,
                                                                       const CodebookArg cb) {
    __shared__ float s_lv[16];
    __shared__ double s_b[kMergeRows][kMergeMaxR];
    float lv = 0.f;
#pragma unroll
    for (int l = 0; l < 16; ++l)   // constant indices keep the parameter block out of local memory
        if ((threadIdx.x & 15) == l) lv = cb.level[l];
    if (threadIdx.x < 16) s_lv[threadIdx.x] = lv;
    const double sd = static_cast<double>(scaling);
    const int64_t KC = K / kMergeCols;            // column groups of a row
    for (int64_t n0 = int64_t(blockIdx.y) * kMergeRows; n0 < N; n0 += int64_t(gridDim.y) * kMergeRows) {
        __syncthreads();   // the previous row group is done with s_b
        for (int t = threadIdx.x; t < kMergeRows * r; t += blockDim.x) {
            const int rr = t / r, j = t - rr * r;
            const int64_t n = n0 + rr;
            s_b[rr][j] = n < N ? static_cast<double>(__uint_as_float(uint32_t(__ldg(B + n * r + j)) << 16)) : 0.0;
        }
        __syncthreads();
        for (int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; c < KC; c += int64_t(gridDim.x) * blockDim.x) {
            const int64_t k0 = kMergeCols * c;
            double acc[kMergeRows][kMergeCols];
#pragma unroll
            for (int rr = 0; rr < kMergeRows; ++rr)
#pragma unroll
                for (int e = 0; e < kMergeCols; ++e) acc[rr][e] = 0.0;
            for (int j = 0; j < r; ++j) {
                const uint2 av = __ldg(reinterpret_cast<const uint2 *>(A + int64_t(j) * K + k0));
                const double a0 = static_cast<double>(__uint_as_float(av.x << 16));
                const double a1 = static_cast<double>(__uint_as_float(av.x & 0xFFFF0000u));
                const double a2 = static_cast<double>(__uint_as_float(av.y << 16));
                const double a3 = static_cast<double>(__uint_as_float(av.y & 0xFFFF0000u));
#pragma unroll
                for (int rr = 0; rr < kMergeRows; ++rr) {
                    const double b = s_b[rr][j];
                    acc[rr][0] = __fma_rn(b, a0, acc[rr][0]);
                    acc[rr][1] = __fma_rn(b, a1, acc[rr][1]);
                    acc[rr][2] = __fma_rn(b, a2, acc[rr][2]);
                    acc[rr][3] = __fma_rn(b, a3, acc[rr][3]);
                }
            }
#pragma unroll
            for (int rr = 0; rr < kMergeRows; ++rr) {
                const int64_t n = n0 + rr;
                if (n >= N) break;
                const int64_t w0 = n * K + k0;                          // first weight of the group
                const uint32_t cw = __ldg(reinterpret_cast<const uint16_t *>(codes) + w0 / 4);   // 4 codes
                const float s = block_scale(sc, w0 >> 6);
                float m[kMergeCols];
#pragma unroll
                for (int e = 0; e < kMergeCols; ++e) m[e] = merge_one(s_lv[(cw >> (4 * e)) & 15u], s, sd, acc[rr][e]);
                reinterpret_cast<float4 *>(out)[w0 / 4] = make_float4(m[0], m[1], m[2], m[3]);
            }
        }
    }
}

}  // namespace qlora
