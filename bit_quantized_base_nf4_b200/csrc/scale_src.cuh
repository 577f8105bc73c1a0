// scale_src.cuh -- where the first-level scale of a run of 64 weights comes from, for
// every storage format of the packed weight: blocks of 64 or 128 weights, and the block
// absmaxes either double-quantized (u8 q_b times an fp32 step d_g per 256 blocks) or
// kept as fp32 ("QLoRA double quantization and block-wise quantization memory" page,
// sections 3.1 and 3.2: block size 64 or 128, the double-quantization switch).
#pragma once

#include <cstdint>

namespace qlora {

struct ScaleSrc {
    const uint8_t *scales;   // u8 q_b per block (double quant) or fp32 a_b per block (none)
    const float *scales2;    // fp32 d_g per 256 blocks (double quant only)
    int blk_shift;           // log2(block size / 64): 0 for blocks of 64, 1 for blocks of 128
    int dq;                  // 1: s_b = fp32(q_b * d_g); 0: s_b = a_b
};

// The two factors of the scale of the 64-weight run b64 (row-major flattening):
// s_b = fp32(sa * sb).  Without double quantization sb = 1, so the product is a_b itself.
__device__ __forceinline__ void scale_parts(const ScaleSrc &s, int64_t b64, float &sa, float &sb) {
    const int64_t b = b64 >> s.blk_shift;
    if (s.dq) {
        sa = static_cast<float>(__ldg(s.scales + b));
        sb = __ldg(s.scales2 + (b >> 8));
    } else {
        sa = __ldg(reinterpret_cast<const float *>(s.scales) + b);
        sb = 1.f;
    }
}

// The same two factors as raw loaded words: the u8 q_b (or the bits of the fp32 a_b) and
// d_g (1 without double quantization).  Nothing here uses the loaded values, so a load
// issued well ahead of its use does not wait for memory until scale_of runs.
__device__ __forceinline__ void scale_load(const ScaleSrc &s, int64_t b64, uint32_t &a, float &d) {
    const int64_t b = b64 >> s.blk_shift;
    if (s.dq) {
        a = __ldg(s.scales + b);
        d = __ldg(s.scales2 + (b >> 8));
    } else {
        a = __ldg(reinterpret_cast<const uint32_t *>(s.scales) + b);
        d = 1.f;
    }
}
// s_b from the raw words of scale_load: fp32(q_b * d_g), or a_b itself
__device__ __forceinline__ float scale_of(const ScaleSrc &s, uint32_t a, float d) {
    return s.dq ? __fmul_rn(static_cast<float>(a), d) : __uint_as_float(a);
}

__device__ __forceinline__ float block_scale(const ScaleSrc &s, int64_t b64) {
    float sa, sb;
    scale_parts(s, b64, sa, sb);
    return __fmul_rn(sa, sb);
}

}  // namespace qlora
