// quant_kernels.cuh -- NF4 block encode with double quantization of the scales,
// and the standalone full-tensor dequant.  Both are HBM-bound and bit-exact.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {

struct CodebookArg {
    float level[16];
    float thresh[16];
};

// One CTA per group of 256 blocks (16384 weights); 8 warps, each warp walks 32
// blocks, 4 at a time.  Per block: absmax by warp shuffles, each lane encodes two
// neighbouring weights into one byte (element 2j low nibble, 2j+1 high nibble).
// Then the group max gives d_g and each thread quantizes one block scale.
constexpr int kEncThreads = 256;

__global__ void __launch_bounds__(kEncThreads) nf4_encode_dq_kernel(const float *__restrict__ W,
                                                                    uint8_t *__restrict__ codes,
                                                                    uint8_t *__restrict__ scales,
                                                                    float *__restrict__ scales2,
                                                                    int64_t nblocks, const CodebookArg cb) {
    __shared__ float s_thr[16];
    __shared__ float s_absmax[256];
    __shared__ float s_wmax[8];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < 16) s_thr[tid] = cb.thresh[tid];
    const int64_t g = blockIdx.x;
    const int64_t b0 = g * 256;
    const int nb = static_cast<int>(nblocks - b0 < 256 ? nblocks - b0 : 256);
    __syncthreads();

    // encode: warp w handles blocks w*32 .. w*32+31 of the group
    for (int it = 0; it < 32; it += 4) {
        float2 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int lb = warp * 32 + it + u;
            v[u] = make_float2(0.f, 0.f);
            if (lb < nb) v[u] = __ldcs(reinterpret_cast<const float2 *>(W + (b0 + lb) * 64) + lane);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int lb = warp * 32 + it + u;
            if (lb >= nb) break;  // warp-uniform
            float a = fmaxf(fabsf(v[u].x), fabsf(v[u].y));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            float n0 = 0.f, n1 = 0.f;
            if (a > 0.f) {
                n0 = __fdiv_rn(v[u].x, a);
                n1 = __fdiv_rn(v[u].y, a);
            }
            // code = #{k : n >= thresh[k]} by binary search over the 15 sorted thresholds
            int c0 = 0, c1 = 0;
            c0 += (n0 >= s_thr[c0 + 7]) ? 8 : 0;
            c1 += (n1 >= s_thr[c1 + 7]) ? 8 : 0;
            c0 += (n0 >= s_thr[c0 + 3]) ? 4 : 0;
            c1 += (n1 >= s_thr[c1 + 3]) ? 4 : 0;
            c0 += (n0 >= s_thr[c0 + 1]) ? 2 : 0;
            c1 += (n1 >= s_thr[c1 + 1]) ? 2 : 0;
            c0 += (n0 >= s_thr[c0]) ? 1 : 0;
            c1 += (n1 >= s_thr[c1]) ? 1 : 0;
            codes[(b0 + lb) * 32 + lane] = static_cast<uint8_t>(c0 | (c1 << 4));
            if (lane == 0) s_absmax[lb] = a;
        }
    }
    __syncthreads();

    // second level: d_g = fp32(max a_b / 255); q_b = clamp(rint(fp32(a_b / d_g)), 0, 255)
    float a = (tid < nb) ? s_absmax[tid] : 0.f;
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
        uint8_t q = 0;
        if (d > 0.f) {
            const float r = rintf(__fdiv_rn(a, d));
            q = static_cast<uint8_t>(fminf(fmaxf(r, 0.f), 255.f));
        }
        scales[b0 + tid] = q;
    }
    if (tid == 0) scales2[g] = d;
}

// Full dequant: thread handles 8 weights (4 code bytes).  out_bf16 selects the
// output type: fp32 w' = fp32(c[code] * fp32(q * d)), or bf16 = RNE(w').
template <bool kBf16>
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint8_t *__restrict__ codes,
                                                          const uint8_t *__restrict__ scales,
                                                          const float *__restrict__ scales2,
                                                          void *__restrict__ out, int64_t n8, const CodebookArg cb) {
    __shared__ float s_lv[16];
    if (threadIdx.x < 16) s_lv[threadIdx.x] = cb.level[threadIdx.x];
    __syncthreads();
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
        const uint32_t cw = __ldg(reinterpret_cast<const uint32_t *>(codes) + i);
        const int64_t blk = i >> 3;  // 8 weights per thread, 64 per block
        const float s = __fmul_rn(static_cast<float>(__ldg(scales + blk)), __ldg(scales2 + (blk >> 8)));
        float w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = __fmul_rn(s_lv[(cw >> (4 * j)) & 15u], s);
        if (kBf16) {
            uint4 o;
            __nv_bfloat162 p0 = __floats2bfloat162_rn(w[0], w[1]);
            __nv_bfloat162 p1 = __floats2bfloat162_rn(w[2], w[3]);
            __nv_bfloat162 p2 = __floats2bfloat162_rn(w[4], w[5]);
            __nv_bfloat162 p3 = __floats2bfloat162_rn(w[6], w[7]);
            o.x = *reinterpret_cast<uint32_t *>(&p0);
            o.y = *reinterpret_cast<uint32_t *>(&p1);
            o.z = *reinterpret_cast<uint32_t *>(&p2);
            o.w = *reinterpret_cast<uint32_t *>(&p3);
            __stcs(reinterpret_cast<uint4 *>(out) + i, o);
        } else {
            float4 *o = reinterpret_cast<float4 *>(out) + 2 * i;
            __stcs(o, make_float4(w[0], w[1], w[2], w[3]));
            __stcs(o + 1, make_float4(w[4], w[5], w[6], w[7]));
        }
    }
}

// LoRA merge, the step before requantization.  Rows run over blockIdx.y, the row's
// code words over x; a thread handles 8 weights (one code word).
//   m = bf16(RN32(bf16(w') + s * sum_j B[n, j] A[j, k])):
// the dequantized base in bf16, the adapter product and the add in fp64 with j
// ascending and no fused multiply-add (bf16 x bf16 products are exact in fp64), then
// float32 and bf16 rounding.  m is stored as float32, the input of the encode kernel.
__device__ __forceinline__ float merge_one(float level, float s, double sd, double acc) {
    const float wb = __bfloat162float(__float2bfloat16_rn(__fmul_rn(level, s)));
    const double t = __dadd_rn(static_cast<double>(wb), __dmul_rn(sd, acc));
    return __bfloat162float(__float2bfloat16_rn(__double2float_rn(t)));
}
__global__ void __launch_bounds__(256) nf4_lora_merge_kernel(const uint8_t *__restrict__ codes,
                                                             const uint8_t *__restrict__ scales,
                                                             const float *__restrict__ scales2,
                                                             const uint16_t *__restrict__ A,
                                                             const uint16_t *__restrict__ B, int r, float scaling,
                                                             int64_t N, int64_t K, float *__restrict__ out,
                                                             const CodebookArg cb) {
    __shared__ float s_lv[16];
    float lv = 0.f;
#pragma unroll
    for (int l = 0; l < 16; ++l)   // constant indices keep the parameter block out of local memory
        if ((threadIdx.x & 15) == l) lv = cb.level[l];
    if (threadIdx.x < 16) s_lv[threadIdx.x] = lv;
    __syncthreads();
    const double sd = static_cast<double>(scaling);
    const int64_t K8 = K / 8;
    for (int64_t n = blockIdx.y; n < N; n += gridDim.y) {
        for (int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; c < K8; c += int64_t(gridDim.x) * blockDim.x) {
            const int64_t i = n * K8 + c;   // code word index; 8 weights per word, 64 per block
            const int64_t k0 = 8 * c;
            const uint32_t cw = __ldg(reinterpret_cast<const uint32_t *>(codes) + i);
            const int64_t blk = i >> 3;
            const float s = __fmul_rn(static_cast<float>(__ldg(scales + blk)), __ldg(scales2 + (blk >> 8)));
            double acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0;
            for (int j = 0; j < r; ++j) {
                const double b = static_cast<double>(__uint_as_float(uint32_t(__ldg(B + n * r + j)) << 16));
                const uint4 av = __ldg(reinterpret_cast<const uint4 *>(A + int64_t(j) * K + k0));
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t word = (e >> 1) == 0 ? av.x : (e >> 1) == 1 ? av.y : (e >> 1) == 2 ? av.z : av.w;
                    const float a = __uint_as_float((e & 1) ? (word & 0xFFFF0000u) : (word << 16));
                    acc[e] = __dadd_rn(acc[e], __dmul_rn(b, static_cast<double>(a)));
                }
            }
            float m[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = merge_one(s_lv[(cw >> (4 * e)) & 15u], s, sd, acc[e]);
            float4 *o = reinterpret_cast<float4 *>(out) + 2 * i;
            o[0] = make_float4(m[0], m[1], m[2], m[3]);
            o[1] = make_float4(m[4], m[5], m[6], m[7]);
        }
    }
}

}  // namespace qlora
