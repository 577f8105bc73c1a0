// lora_kernels.cuh -- the rank-r side products of the adapter (CUDA cores, fp32
// accumulation) and small helpers.
//
//   proj:  C[m, j] = sum_t P[m, t] Q(j, t)      U = X A^T (Q = A [r, K]) and
//                                               G = dY B  (Q = B [N, r], read transposed)
//          writes save[m, j] = bf16(C) and scaled[m, j] = bf16(scaling * C)
//   grad:  C[i, j] (+)= scaling * sum_m P[m, i] Q[m, j]
//                                               dA^T (P = X, Q = G), dB (P = dY, Q = U)
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace qlora {

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&h);
}

constexpr int kProjTM = 16;   // tokens per CTA
constexpr int kProjTT = 32;   // contraction chunk
constexpr int kMaxR = 128;

// 256 threads: thread -> token tid/16, ranks (tid%16) + 16*i.
__global__ void __launch_bounds__(256) lora_proj_kernel(const uint16_t *__restrict__ P, int64_t M, int64_t T,
                                                        const uint16_t *__restrict__ Q, int64_t q_ld_j,
                                                        int64_t q_ld_t, int r, float scaling,
                                                        uint16_t *__restrict__ save, uint16_t *__restrict__ scaled) {
    __shared__ float Ps[kProjTM][kProjTT + 1];
    __shared__ float Qs[kProjTT][kMaxR];
    const int tid = threadIdx.x;
    const int ml = tid >> 4, jl = tid & 15;
    const int64_t m0 = int64_t(blockIdx.x) * kProjTM;
    const int nj = (r + 15) / 16;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int64_t t0 = 0; t0 < T; t0 += kProjTT) {
        for (int i = tid; i < kProjTM * kProjTT; i += 256) {
            const int mm = i / kProjTT, tt = i % kProjTT;
            const int64_t m = m0 + mm, t = t0 + tt;
            Ps[mm][tt] = (m < M && t < T) ? bf16_to_f32(P[m * T + t]) : 0.f;
        }
        for (int i = tid; i < kProjTT * r; i += 256) {
            int tt, j;
            if (q_ld_t == 1) { j = i / kProjTT; tt = i % kProjTT; } else { tt = i / r; j = i % r; }
            const int64_t t = t0 + tt;
            Qs[tt][j] = (t < T) ? bf16_to_f32(Q[j * q_ld_j + t * q_ld_t]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < kProjTT; ++tt) {
            const float pv = Ps[ml][tt];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i < nj && jl + 16 * i < r) acc[i] = fmaf(pv, Qs[tt][jl + 16 * i], acc[i]);
        }
        __syncthreads();
    }
    const int64_t m = m0 + ml;
    if (m < M) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = jl + 16 * i;
            if (i < nj && j < r) {
                if (save) save[m * r + j] = f32_to_bf16(acc[i]);
                if (scaled) scaled[m * r + j] = f32_to_bf16(scaling * acc[i]);
            }
        }
    }
}

constexpr int kGradTI = 64;   // output rows i per CTA
constexpr int kGradTM = 32;   // tokens per chunk
constexpr int kGradMPerCta = 512;

// 256 threads: thread -> row tid%64, ranks tid/64 + 4*jj.  blockIdx.y splits the tokens;
// partial sums are added atomically (the output is zeroed first unless accumulating).
__global__ void __launch_bounds__(256) lora_grad_kernel(const uint16_t *__restrict__ P, int64_t M, int64_t I,
                                                        const uint16_t *__restrict__ Q, int r, float scaling,
                                                        float *__restrict__ C, int64_t c_ld_i, int64_t c_ld_j) {
    __shared__ float Ps[kGradTM][kGradTI];
    __shared__ float Qs[kGradTM][kMaxR];
    const int tid = threadIdx.x;
    const int il = tid & 63, jg = tid >> 6;
    const int64_t i0 = int64_t(blockIdx.x) * kGradTI;
    const int64_t mbeg = int64_t(blockIdx.y) * kGradMPerCta;
    const int64_t mend = (mbeg + kGradMPerCta < M) ? mbeg + kGradMPerCta : M;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    const int njj = r / 4;
    for (int64_t mc = mbeg; mc < mend; mc += kGradTM) {
        for (int k = tid; k < kGradTM * kGradTI; k += 256) {
            const int mm = k / kGradTI, ii = k % kGradTI;
            const int64_t m = mc + mm, i = i0 + ii;
            Ps[mm][ii] = (m < mend && i < I) ? bf16_to_f32(P[m * I + i]) : 0.f;
        }
        for (int k = tid; k < kGradTM * r; k += 256) {
            const int mm = k / r, j = k % r;
            const int64_t m = mc + mm;
            Qs[mm][j] = (m < mend) ? bf16_to_f32(Q[m * r + j]) : 0.f;
        }
        __syncthreads();
        for (int mm = 0; mm < kGradTM; ++mm) {
            const float pv = Ps[mm][il];
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
                if (jj < njj) acc[jj] = fmaf(pv, Qs[mm][jg + 4 * jj], acc[jj]);
        }
        __syncthreads();
    }
    const int64_t i = i0 + il;
    if (i < I) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
            if (jj < njj) atomicAdd(C + i * c_ld_i + int64_t(jg + 4 * jj) * c_ld_j, scaling * acc[jj]);
    }
}

__global__ void f32_to_bf16_kernel(const float *__restrict__ in, uint16_t *__restrict__ out, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        out[i] = f32_to_bf16(in[i]);
}

}  // namespace qlora
