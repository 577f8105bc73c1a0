// qlora_nf4.cu -- C ABI of the library: validation, launch planning and kernel launches.
// Every kernel lives in a header of this directory; this file is the only translation unit.

#include <algorithm>
#include <cstdint>

#include "host_common.cuh"
#include "ptx.cuh"
#include "quant_kernels.cuh"
#include "lora_kernels.cuh"
#include "fused_fwd.cuh"
#include "fused_bwd.cuh"

using namespace qlora;

namespace {

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

CodebookArg codebook_arg() {
    CodebookArg a;
    const Codebook &cb = codebook();
    for (int i = 0; i < 16; ++i) {
        a.level[i] = cb.level[i];
        a.thresh[i] = cb.thresh[i];
    }
    return a;
}

// Token-tile width: the MMA N dimension (multiple of 16, at most 256), chosen
// to split M into equal tiles with little padding.
int token_tile(int64_t M) {
    const int64_t tiles = ceil_div(M, 256);
    const int64_t bn = ceil_div(ceil_div(M, tiles), 16) * 16;
    return static_cast<int>(std::max<int64_t>(16, std::min<int64_t>(256, bn)));
}

struct GemmPlan {
    int BN;
    int64_t tiles_rows, tiles_tok;
    int splits;
    int stages_per_split;
};

// rows = output rows of the MMA M dimension (N for forward, K for dX),
// stages = 64-wide contraction stages.  Split the contraction across CTAs only
// when the output tiles leave most SMs idle (small-M decode shapes).
GemmPlan plan_gemm(int64_t M, int64_t rows, int64_t stages) {
    GemmPlan g;
    g.BN = token_tile(M);
    g.tiles_rows = ceil_div(rows, 128);
    g.tiles_tok = ceil_div(M, g.BN);
    const int64_t tiles = g.tiles_rows * g.tiles_tok;
    const int sms = sm_count();
    int splits = 1;
    if (tiles * 2 <= sms) {
        const int64_t want = ceil_div(2 * sms, tiles);
        const int64_t maxs = std::max<int64_t>(1, stages / 4);
        splits = static_cast<int>(std::min(want, maxs));
    }
    g.stages_per_split = static_cast<int>(ceil_div(stages, splits));
    g.splits = static_cast<int>(ceil_div(stages, g.stages_per_split));
    return g;
}

size_t fwd_ws_bytes(int64_t M, int64_t N, int64_t K, int r) {
    const GemmPlan g = plan_gemm(M, N, K / 64);
    size_t b = round256(size_t(M) * size_t(std::max(r, 0)) * 2);
    if (g.splits > 1) b += round256(size_t(M) * size_t(N) * 4);
    return b;
}
size_t bwd_ws_bytes(int64_t M, int64_t N, int64_t K, int r) {
    const GemmPlan g = plan_gemm(M, K, ceil_div(N, 64));
    size_t b = round256(size_t(M) * size_t(std::max(r, 0)) * 2);
    if (g.splits > 1) b += round256(size_t(M) * size_t(K) * 4);
    return b;
}

qlora_status check_rank(int r, float scaling, const void *A, const void *B) {
    if (r == 0) return QLORA_OK;
    if (r < 8 || r > 128 || r % 8) return fail(QLORA_ERR_SHAPE, "r (%d) must be 0 or a multiple of 8 in [8, 128]", r);
    if (!A || !B) return fail(QLORA_ERR_ARG, "A and B must be non-NULL when r > 0");
    if (!aligned16(A) || !aligned16(B)) return fail(QLORA_ERR_ALIGN, "A and B must be 16-byte aligned");
    if (!std::isfinite(scaling)) return fail(QLORA_ERR_ARG, "scaling must be finite");
    return QLORA_OK;
}

qlora_status check_ws(void *ws, size_t ws_bytes, size_t need) {
    if (need == 0) return QLORA_OK;
    if (!ws) return fail(QLORA_ERR_WORKSPACE, "workspace is NULL but %zu bytes are needed", need);
    if (!aligned16(ws)) return fail(QLORA_ERR_ALIGN, "workspace must be 16-byte aligned");
    if (ws_bytes < need) return fail(QLORA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    return QLORA_OK;
}

template <typename K>
qlora_status set_smem(K kernel, int bytes) {
    return cuda_check(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
                      "cudaFuncSetAttribute(max dynamic smem)");
}

qlora_status launch_check(const char *what) { return cuda_check(cudaGetLastError(), what); }

}  // namespace

extern "C" {

size_t qlora_packed_bytes(int64_t numel) {
    if (numel <= 0 || numel % 64) return 0;
    const int64_t nb = numel / 64;
    return size_t(numel / 2) + size_t(nb) + 4 * size_t(ceil_div(nb, 256));
}

qlora_status qlora_nf4_codebook(float out[16]) {
    if (!out) return fail(QLORA_ERR_ARG, "out is NULL");
    const Codebook &cb = codebook();
    for (int i = 0; i < 16; ++i) out[i] = cb.level[i];
    return QLORA_OK;
}

const char *qlora_last_error(void) { return t_last_error; }

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return std::max<size_t>(256, std::max(fwd_ws_bytes(M, N, K, r), bwd_ws_bytes(M, N, K, r)));
}

qlora_status qlora_sync_status(void *stream) {
    QL_TRY(cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize"));
    int v = 0;
    QL_TRY(cuda_check(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)), "read device error word"));
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
        return fail(QLORA_ERR_TIMEOUT, "a kernel pipeline wait timed out (device error %d)", v);
    }
    return QLORA_OK;
}

qlora_status qlora_quantize_nf4_dq(const float *W, const qlora_nf4_weight *w, void *stream) {
    QL_TRY(check_weight(w));
    if (!W) return fail(QLORA_ERR_ARG, "W is NULL");
    if (!aligned16(W)) return fail(QLORA_ERR_ALIGN, "W must be 16-byte aligned");
    QL_TRY(require_sm100());
    const int64_t numel = w->n_out * w->n_in;
    const int64_t nblocks = numel / 64;
    const int64_t ngroups = ceil_div(nblocks, 256);
    if (ngroups > INT32_MAX) return fail(QLORA_ERR_SHAPE, "weight too large");
    nf4_encode_dq_kernel<<<static_cast<unsigned>(ngroups), kEncThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        W, w->codes, w->scales, w->scales2, nblocks, codebook_arg());
    return launch_check("nf4_encode_dq_kernel launch");
}

qlora_status qlora_dequant(const qlora_nf4_weight *w, void *out, int out_is_bf16, void *stream) {
    QL_TRY(check_weight(w));
    if (!out) return fail(QLORA_ERR_ARG, "out is NULL");
    if (!aligned16(out)) return fail(QLORA_ERR_ALIGN, "out must be 16-byte aligned");
    if (out_is_bf16 != 0 && out_is_bf16 != 1) return fail(QLORA_ERR_ARG, "out_is_bf16 must be 0 or 1");
    QL_TRY(require_sm100());
    const int64_t n8 = w->n_out * w->n_in / 8;
    const int64_t grid = std::min<int64_t>(ceil_div(n8, 256), int64_t(sm_count()) * 16);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (out_is_bf16)
        nf4_dequant_kernel<true><<<static_cast<unsigned>(grid), 256, 0, st>>>(w->codes, w->scales, w->scales2, out,
                                                                               n8, codebook_arg());
    else
        nf4_dequant_kernel<false><<<static_cast<unsigned>(grid), 256, 0, st>>>(w->codes, w->scales, w->scales2, out,
                                                                                n8, codebook_arg());
    return launch_check("nf4_dequant_kernel launch");
}

qlora_status qlora_lora_linear_fwd(const qlora_nf4_weight *w, const qlora_bf16 *X, int64_t M, const qlora_bf16 *A,
                                   const qlora_bf16 *B, int r, float scaling, qlora_bf16 *Y, qlora_bf16 *U_save,
                                   void *ws, size_t ws_bytes, void *stream) {
    QL_TRY(check_weight(w));
    if (!X || !Y) return fail(QLORA_ERR_ARG, "X and Y must be non-NULL");
    if (!aligned16(X) || !aligned16(Y)) return fail(QLORA_ERR_ALIGN, "X and Y must be 16-byte aligned");
    if (U_save && !aligned16(U_save)) return fail(QLORA_ERR_ALIGN, "U_save must be 16-byte aligned");
    if (M <= 0 || M > INT32_MAX) return fail(QLORA_ERR_SHAPE, "M (%lld) must be in [1, 2^31)", (long long)M);
    QL_TRY(check_rank(r, scaling, A, B));
    const int64_t N = w->n_out, K = w->n_in;
    const size_t need = fwd_ws_bytes(M, N, K, r);
    QL_TRY(check_ws(ws, ws_bytes, need));
    QL_TRY(require_sm100());
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const GemmPlan g = plan_gemm(M, N, K / 64);
    uint16_t *us = static_cast<uint16_t *>(ws);
    float *yacc = g.splits > 1 ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + round256(size_t(M) * r * 2))
                               : nullptr;
    if (r > 0) {
        lora_proj_kernel<<<static_cast<unsigned>(ceil_div(M, kProjTM)), 256, 0, st>>>(X, M, K, A, K, 1, r, scaling,
                                                                                       U_save, us);
        QL_TRY(launch_check("lora_proj_kernel (X A^T) launch"));
    }
    if (yacc) QL_TRY(cuda_check(cudaMemsetAsync(yacc, 0, size_t(M) * N * 4, st), "zero split accumulator"));

    CUtensorMap tmX, tmC, tmU;
    QL_TRY(make_tmap_2d(&tmX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, K, g.BN, 64,
                        CU_TENSOR_MAP_SWIZZLE_128B));
    QL_TRY(make_tmap_2d(&tmC, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, 128, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B));
    if (r > 0)
        QL_TRY(make_tmap_2d(&tmU, us, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, r, r, g.BN, 64,
                            CU_TENSOR_MAP_SWIZZLE_128B));
    else
        tmU = tmX;

    fwd::Params p;
    p.scales = w->scales;
    p.scales2 = w->scales2;
    p.Blora = B;
    p.Y = Y;
    p.Yacc = yacc;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.r = r;
    p.BN = g.BN;
    p.kb_per_split = g.stages_per_split;
    const Codebook &cb = codebook();
    for (int i = 0; i < 16; ++i) p.level[i] = cb.level[i];

    const int smem = fwd::smem_bytes(g.BN);
    QL_TRY(set_smem(fwd::fused_fwd_kernel, fwd::smem_bytes(256)));
    dim3 grid(static_cast<unsigned>(g.tiles_rows), static_cast<unsigned>(g.tiles_tok), static_cast<unsigned>(g.splits));
    fwd::fused_fwd_kernel<<<grid, fwd::kThreads, smem, st>>>(tmX, tmC, tmU, p);
    QL_TRY(launch_check("fused_fwd_kernel launch"));
    if (yacc) {
        const int64_t n = M * N;
        f32_to_bf16_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 4096)), 256, 0, st>>>(yacc, Y, n);
        QL_TRY(launch_check("split finalize launch"));
    }
    return QLORA_OK;
}

qlora_status qlora_lora_linear_bwd_dx(const qlora_nf4_weight *w, const qlora_bf16 *dY, int64_t M, const qlora_bf16 *A,
                                      const qlora_bf16 *B, int r, float scaling, qlora_bf16 *dX, qlora_bf16 *G_save,
                                      void *ws, size_t ws_bytes, void *stream) {
    QL_TRY(check_weight(w));
    if (!dY || !dX) return fail(QLORA_ERR_ARG, "dY and dX must be non-NULL");
    if (!aligned16(dY) || !aligned16(dX)) return fail(QLORA_ERR_ALIGN, "dY and dX must be 16-byte aligned");
    if (G_save && !aligned16(G_save)) return fail(QLORA_ERR_ALIGN, "G_save must be 16-byte aligned");
    if (M <= 0 || M > INT32_MAX) return fail(QLORA_ERR_SHAPE, "M (%lld) must be in [1, 2^31)", (long long)M);
    QL_TRY(check_rank(r, scaling, A, B));
    const int64_t N = w->n_out, K = w->n_in;
    if (N % 8) return fail(QLORA_ERR_SHAPE, "n_out (%lld) must be a multiple of 8 for the dX pass", (long long)N);
    const size_t need = bwd_ws_bytes(M, N, K, r);
    QL_TRY(check_ws(ws, ws_bytes, need));
    QL_TRY(require_sm100());
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const GemmPlan g = plan_gemm(M, K, ceil_div(N, 64));
    uint16_t *gs = static_cast<uint16_t *>(ws);
    float *dxacc = g.splits > 1 ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + round256(size_t(M) * r * 2))
                                : nullptr;
    if (r > 0) {
        lora_proj_kernel<<<static_cast<unsigned>(ceil_div(M, kProjTM)), 256, 0, st>>>(dY, M, N, B, 1, r, r, scaling,
                                                                                       G_save, gs);
        QL_TRY(launch_check("lora_proj_kernel (dY B) launch"));
    }
    if (dxacc) QL_TRY(cuda_check(cudaMemsetAsync(dxacc, 0, size_t(M) * K * 4, st), "zero split accumulator"));

    CUtensorMap tmY, tmC, tmG;
    QL_TRY(make_tmap_2d(&tmY, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, N, g.BN, 64,
                        CU_TENSOR_MAP_SWIZZLE_128B));
    QL_TRY(make_tmap_2d(&tmC, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, 64, 64,
                        CU_TENSOR_MAP_SWIZZLE_64B));
    if (r > 0)
        QL_TRY(make_tmap_2d(&tmG, gs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, r, r, g.BN, 64,
                            CU_TENSOR_MAP_SWIZZLE_128B));
    else
        tmG = tmY;

    bwd::Params p;
    p.scales = w->scales;
    p.scales2 = w->scales2;
    p.Alora = A;
    p.dX = dX;
    p.dXacc = dxacc;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.r = r;
    p.BN = g.BN;
    p.nb_per_split = g.stages_per_split;
    const Codebook &cb = codebook();
    for (int i = 0; i < 16; ++i) p.level[i] = cb.level[i];

    const int smem = bwd::smem_bytes(g.BN);
    QL_TRY(set_smem(bwd::fused_bwd_dx_kernel, bwd::smem_bytes(256)));
    dim3 grid(static_cast<unsigned>(g.tiles_rows), static_cast<unsigned>(g.tiles_tok), static_cast<unsigned>(g.splits));
    bwd::fused_bwd_dx_kernel<<<grid, bwd::kThreads, smem, st>>>(tmY, tmC, tmG, p);
    QL_TRY(launch_check("fused_bwd_dx_kernel launch"));
    if (dxacc) {
        const int64_t n = M * K;
        f32_to_bf16_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 4096)), 256, 0, st>>>(dxacc, dX,
                                                                                                            n);
        QL_TRY(launch_check("split finalize launch"));
    }
    return QLORA_OK;
}

qlora_status qlora_lora_grad_AB(const qlora_bf16 *X, const qlora_bf16 *dY, const qlora_bf16 *U, const qlora_bf16 *G,
                                int64_t M, int64_t N, int64_t K, int r, float scaling, float *dA, float *dB,
                                int accumulate, void *stream) {
    if (!X || !dY || !U || !G || !dA || !dB) return fail(QLORA_ERR_ARG, "all tensors must be non-NULL");
    if (!aligned16(X) || !aligned16(dY) || !aligned16(U) || !aligned16(G) || !aligned16(dA) || !aligned16(dB))
        return fail(QLORA_ERR_ALIGN, "all tensors must be 16-byte aligned");
    if (M <= 0 || N <= 0 || K <= 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
        return fail(QLORA_ERR_SHAPE, "M, N and K must be in [1, 2^31)");
    if (r < 8 || r > 128 || r % 8) return fail(QLORA_ERR_SHAPE, "r (%d) must be a multiple of 8 in [8, 128]", r);
    if (accumulate != 0 && accumulate != 1) return fail(QLORA_ERR_ARG, "accumulate must be 0 or 1");
    if (!std::isfinite(scaling)) return fail(QLORA_ERR_ARG, "scaling must be finite");
    QL_TRY(require_sm100());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!accumulate) {
        QL_TRY(cuda_check(cudaMemsetAsync(dA, 0, size_t(r) * K * 4, st), "zero dA"));
        QL_TRY(cuda_check(cudaMemsetAsync(dB, 0, size_t(N) * r * 4, st), "zero dB"));
    }
    const unsigned ms = static_cast<unsigned>(ceil_div(M, kGradMPerCta));
    lora_grad_kernel<<<dim3(static_cast<unsigned>(ceil_div(K, kGradTI)), ms), 256, 0, st>>>(X, M, K, G, r, scaling, dA,
                                                                                           1, K);
    QL_TRY(launch_check("lora_grad_kernel (dA) launch"));
    lora_grad_kernel<<<dim3(static_cast<unsigned>(ceil_div(N, kGradTI)), ms), 256, 0, st>>>(dY, M, N, U, r, scaling, dB,
                                                                                           r, 1);
    QL_TRY(launch_check("lora_grad_kernel (dB) launch"));
    return QLORA_OK;
}

}  // extern "C"
