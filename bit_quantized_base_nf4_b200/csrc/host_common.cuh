// host_common.cuh -- host-side pieces of the library: the NF4 codebook, argument
// validation, error reporting and TMA tensor-map construction.
#pragma once

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "qlora_nf4.h"

namespace qlora {

// ------------------------------------------------------------------ errors
static thread_local char t_last_error[512] = "";

static qlora_status fail(qlora_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
    return st;
}

static qlora_status cuda_check(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return QLORA_OK;
    return fail(QLORA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define QL_TRY(expr)                           \
    do {                                       \
        qlora_status _st = (expr);             \
        if (_st != QLORA_OK) return _st;       \
    } while (0)

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ NF4 codebook
// Inverse normal CDF by Wichura's algorithm AS241 (PPND16, Applied Statistics
// 37(3), 1988): rational approximations in three regions, relative accuracy
// about 1e-16.
static double norm_ppf_as241(double p) {
    const double q = p - 0.5;
    if (std::fabs(q) <= 0.425) {
        const double r = 0.180625 - q * q;
        const double num =
            (((((((2509.0809287301226727 * r + 33430.575583588128105) * r + 67265.770927008700853) * r +
                 45921.953931549871457) * r + 13731.693765509461125) * r + 1971.5909503065514427) * r +
              133.14166789178437745) * r + 3.387132872796366608);
        const double den =
            (((((((5226.495278852545925 * r + 28729.085735721942674) * r + 39307.89580009271061) * r +
                 21213.794301586595867) * r + 5394.1960214247511077) * r + 687.1870074920579083) * r +
              42.313330701600911252) * r + 1.0);
        return q * num / den;
    }
    double r = q < 0 ? p : 1.0 - p;
    r = std::sqrt(-std::log(r));
    double num, den;
    if (r <= 5.0) {
        r -= 1.6;
        num = (((((((7.7454501427834140764e-4 * r + 0.0227238449892691845833) * r + 0.24178072517745061177) * r +
                   1.27045825245236838258) * r + 3.64784832476320460504) * r + 5.7694972214606914055) * r +
                4.6303378461565452959) * r + 1.42343711074968357734);
        den = (((((((1.05075007164441684324e-9 * r + 5.475938084995344946e-4) * r + 0.0151986665636164571966) * r +
                   0.14810397642748007459) * r + 0.68976733498510000455) * r + 1.6763848301838038494) * r +
                2.05319162663775882187) * r + 1.0);
    } else {
        r -= 5.0;
        num = (((((((2.01033439929228813265e-7 * r + 2.71155556874348757815e-5) * r + 0.0012426609473880784386) * r +
                   0.026532189526576123093) * r + 0.29656057182850489123) * r + 1.7848265399172913358) * r +
                5.4637849111641143699) * r + 6.6579046435011037772);
        den = (((((((2.04426310338993978564e-15 * r + 1.4215117583164458887e-7) * r + 1.8463183175100546818e-5) * r +
                   7.868691311456132591e-4) * r + 0.0148753612908506148525) * r + 0.13692988092273580531) * r +
                0.59983220655588793769) * r + 1.0);
    }
    const double x = num / den;
    return q < 0 ? -x : x;
}

struct Codebook {
    float level[16];     // ascending levels, float32
    float thresh[16];    // thresh[k] = smallest float32 above the exact midpoint of levels k, k+1; [15] = +inf
};

// Levels rounded to float32 and the encode thresholds: a value n takes code
// #{k : n >= thresh[k]}, the nearest level with exact ties to the lower index (two
// equal levels, the FP4 table's -0 and +0, split by sign: the threshold between
// them is the smallest positive float32).
static void fill_codebook(Codebook &cb, const double (&v)[16]) {
    for (int i = 0; i < 16; ++i) cb.level[i] = static_cast<float>(v[i]);
    for (int k = 0; k < 15; ++k) {
        // midpoint of two floats: exact in double
        const double mid = (static_cast<double>(cb.level[k]) + static_cast<double>(cb.level[k + 1])) * 0.5;
        float t = static_cast<float>(mid);
        if (static_cast<double>(t) <= mid) t = std::nextafter(t, INFINITY);
        cb.thresh[k] = t;
    }
    cb.thresh[15] = INFINITY;
}

// NF4 levels: normal quantiles at equal probability steps inside the offset
// delta, normalised by Phi^-1(delta), 7 negative + exact 0 + 8 positive.
static const Codebook &codebook() {
    static Codebook cb;
    static std::once_flag once;
    std::call_once(once, [] {
        const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
        const double top = norm_ppf_as241(delta);
        double v[16];
        for (int j = 1; j <= 7; ++j) v[7 - j] = -norm_ppf_as241(0.5 + j * (delta - 0.5) / 7.0) / top;
        v[7] = 0.0;
        for (int j = 1; j <= 8; ++j) v[7 + j] = norm_ppf_as241(0.5 + j * (delta - 0.5) / 8.0) / top;
        v[0] = -1.0;
        v[15] = 1.0;
        fill_codebook(cb, v);
    });
    return cb;
}

// FP4 levels: the E2M1 4-bit float magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 divided by
// 6 (largest 1), both signs, ascending; index 7 is -0 and index 8 is +0.
static const Codebook &fp4_codebook() {
    static Codebook cb;
    static std::once_flag once;
    std::call_once(once, [] {
        const double mags[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
        double v[16];
        for (int i = 0; i < 8; ++i) {
            v[7 - i] = -mags[i] / 6.0;
            v[8 + i] = mags[i] / 6.0;
        }
        fill_codebook(cb, v);
    });
    return cb;
}

// The table of a weight's 4-bit quant type (checked by check_weight).
static const Codebook &codebook_for(int32_t quant_type) {
    return quant_type == QLORA_QT_FP4 ? fp4_codebook() : codebook();
}

// ------------------------------------------------------------------ TMA descriptors
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D tiled map over a row-major [rows, cols] tensor; box = [box_rows, box_cols].
static qlora_status make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                                 uint64_t rows, uint64_t cols, uint64_t row_stride_elems, uint32_t box_rows,
                                 uint32_t box_cols, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return fail(QLORA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_stride_elems * static_cast<uint64_t>(elem_bytes)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QLORA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rows=%llu cols=%llu box=%ux%u", int(r),
                    (unsigned long long)rows, (unsigned long long)cols, box_rows, box_cols);
    return QLORA_OK;
}

// 3-D map viewing a row-major [rows, cols] bf16 tensor as [cols/64 chunks][rows][64]:
// one box = `depth` consecutive 64-column chunks of `box_rows` rows, each chunk a
// 128-byte-swizzled [box_rows x 128 B] tile, stored chunk after chunk.
static qlora_status make_tmap_chunks(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                                     uint32_t box_rows, uint32_t depth) {
    auto fn = encode_fn();
    if (!fn) return fail(QLORA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    cuuint64_t dims[3] = {64, rows, (cols + 63) / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, depth};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QLORA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d) rows=%llu cols=%llu box=%ux64x%u", int(r),
                    (unsigned long long)rows, (unsigned long long)cols, box_rows, depth);
    return QLORA_OK;
}

// 3-D map viewing packed codes, u8 [rows, K/2], as [K/256 chunks][rows][128 B]: one box
// = `depth` consecutive 128-byte chunks of `box_rows` rows, each a 128-byte-swizzled
// [box_rows x 128 B] tile, stored chunk after chunk.  K must be a multiple of 256.
static qlora_status make_tmap_code_chunks(CUtensorMap *map, const void *codes, uint64_t rows, uint64_t K,
                                          uint32_t box_rows, uint32_t depth) {
    auto fn = encode_fn();
    if (!fn) return fail(QLORA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    cuuint64_t dims[3] = {128, rows, K / 256};
    cuuint64_t strides[2] = {K / 2, 128};
    cuuint32_t box[3] = {128, box_rows, depth};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(codes), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QLORA_ERR_CUDA, "cuTensorMapEncodeTiled (codes, 3-D) failed (%d) rows=%llu K=%llu", int(r),
                    (unsigned long long)rows, (unsigned long long)K);
    return QLORA_OK;
}

// ------------------------------------------------------------------ device checks
static qlora_status require_sm100() {
    int dev = 0;
    QL_TRY(cuda_check(cudaGetDevice(&dev), "cudaGetDevice"));
    int major = 0, minor = 0;
    QL_TRY(cuda_check(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "cc major"));
    QL_TRY(cuda_check(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "cc minor"));
    if (major != 10 || minor != 0)
        return fail(QLORA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev,
                    major, minor);
    return QLORA_OK;
}

static int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

// The storage format flags of a weight (QLORA_FMT_*).
static bool fmt_valid(int32_t f) {
    return (f & ~(QLORA_FMT_BLOCK128 | QLORA_FMT_NO_DQ | QLORA_FMT_CODES_AFTER_DQ)) == 0 &&
           !((f & QLORA_FMT_NO_DQ) && (f & QLORA_FMT_CODES_AFTER_DQ));
}
static int fmt_block(int32_t f) { return (f & QLORA_FMT_BLOCK128) ? 128 : 64; }
static bool fmt_dq(int32_t f) { return (f & QLORA_FMT_NO_DQ) == 0; }

static qlora_status check_weight(const qlora_nf4_weight *w) {
    if (!w) return fail(QLORA_ERR_ARG, "weight descriptor is NULL");
    if (!fmt_valid(w->format))
        return fail(QLORA_ERR_ARG, "format (%d) is not a valid combination of QLORA_FMT_* flags", w->format);
    const int blk = fmt_block(w->format);
    const bool dq = fmt_dq(w->format);
    if (w->n_out <= 0 || w->n_in <= 0) return fail(QLORA_ERR_SHAPE, "n_out and n_in must be positive");
    if (w->n_in % blk) return fail(QLORA_ERR_SHAPE, "n_in (%lld) must be a multiple of the block (%d)", (long long)w->n_in, blk);
    if (w->n_out > (int64_t(1) << 31) || w->n_in > (int64_t(1) << 31))
        return fail(QLORA_ERR_SHAPE, "n_out and n_in must be below 2^31");
    if (!w->codes || !w->scales || (dq && !w->scales2)) return fail(QLORA_ERR_ARG, "weight buffers must be non-NULL");
    if (!aligned16(w->codes) || !aligned16(w->scales) || (dq && !aligned16(w->scales2)))
        return fail(QLORA_ERR_ALIGN, "weight buffers must be 16-byte aligned");
    if (w->quant_type != QLORA_QT_NF4 && w->quant_type != QLORA_QT_FP4)
        return fail(QLORA_ERR_ARG, "quant_type (%d) must be QLORA_QT_NF4 (0) or QLORA_QT_FP4 (1)", w->quant_type);
    return QLORA_OK;
}

}  // namespace qlora
