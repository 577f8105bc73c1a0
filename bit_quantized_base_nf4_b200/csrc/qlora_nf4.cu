// qlora_nf4.cu -- C ABI of the library: validation, launch planning and kernel launches.
// Every kernel lives in a header of this directory; this file is the only translation unit.

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include "host_common.cuh"
#include "ptx.cuh"
#include "quant_kernels.cuh"
#include "skinny_mma.cuh"
#include "fused_fwd.cuh"
#include "fused_fwd_pair.cuh"
#include "fused_bwd_pair.cuh"
#include "decode_mma.cuh"

using namespace qlora;

// Scratch of qlora_lora_linear_fwd_static_ws: part of this module's global
// memory on every device where the module is loaded; zero-filled at load, and
// each call clears the parts it accumulates into.
static __device__ __align__(256) uint8_t g_static_scratch[QLORA_STATIC_SCRATCH_BYTES];

// Self-test of the bounded-wait path: one thread waits on a barrier that nothing
// arrives on, with the same wait every pipeline uses; it gives up after the
// current limit, raises the device error word and returns.
__global__ void wait_probe_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag);
}

namespace {

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

static_assert(sizeof(qlora_nf4_weight) == 48 && offsetof(qlora_nf4_weight, quant_type) == 40 &&
                  offsetof(qlora_nf4_weight, format) == 44,
              "the weight descriptor layout is part of the ABI");

// Where the kernels find a weight's first-level scales (see scale_src.cuh).
ScaleSrc scale_src(const qlora_nf4_weight *w) {
    ScaleSrc sc;
    sc.scales = w->scales;
    sc.scales2 = w->scales2;
    sc.blk_shift = fmt_block(w->format) == 128 ? 1 : 0;
    sc.dq = fmt_dq(w->format) ? 1 : 0;
    return sc;
}

CodebookArg codebook_arg(int32_t quant_type) {
    CodebookArg a;
    const Codebook &cb = codebook_for(quant_type);
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
    // whole four-stage code chunks per split
    g.stages_per_split = static_cast<int>(ceil_div(ceil_div(stages, splits), 4) * 4);
    g.splits = static_cast<int>(ceil_div(stages, g.stages_per_split));
    return g;
}

// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the current
// device; the attribute is set once per (kernel, device, size increase), so calls
// after the first make no CUDA call here.
struct SmemSetting {
    const void *kernel;
    int dev, bytes;
};
template <typename K>
qlora_status set_smem(K kernel, int bytes) {
    static std::mutex mu;
    static SmemSetting done[256];
    static int ndone = 0;
    const void *key = reinterpret_cast<const void *>(kernel);
    int dev = 0;
    QL_TRY(cuda_check(cudaGetDevice(&dev), "cudaGetDevice"));
    std::lock_guard<std::mutex> lock(mu);
    int slot = -1;
    for (int i = 0; i < ndone; ++i)
        if (done[i].kernel == key && done[i].dev == dev) slot = i;
    if (slot >= 0 && done[slot].bytes >= bytes) return QLORA_OK;
    QL_TRY(cuda_check(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
                      "cudaFuncSetAttribute(max dynamic smem)"));
    if (slot < 0 && ndone < 256) slot = ndone++;
    if (slot >= 0) done[slot] = SmemSetting{key, dev, bytes};
    return QLORA_OK;
}

qlora_status launch_check(const char *what) { return cuda_check(cudaGetLastError(), what); }

// Workspace layout of the forward / dX calls:
//   [0, a)      bf16 [M, r]   scaling * (X A^T) or scaling * (dY B): the adapter chunk operand
//   [a, a+b)    fp32 [M, r]   accumulator of that rank-r product
//   [a+b, ...)  fp32 [M, N] or [M, K]  split-K accumulator (small-M shapes only)
struct WsLayout {
    size_t rank_bf16, rank_acc, split_acc, total;
};
WsLayout ws_layout(int64_t M, int64_t rows, int r, bool split) {
    WsLayout w;
    w.rank_bf16 = round256(size_t(M) * size_t(std::max(r, 0)) * 2);
    w.rank_acc = round256(size_t(M) * size_t(std::max(r, 0)) * 4);
    w.split_acc = split ? round256(size_t(M) * size_t(rows) * 4) : 0;
    w.total = w.rank_bf16 + w.rank_acc + w.split_acc;
    return w;
}
// Forward kernel choice: CTA pairs (cta_group::2, 256 W rows per tile) from 64
// tokens up; the single-CTA kernel with split-K below that (decode shapes).
bool use_pair_fwd(int64_t M) { return M >= 64; }
int pair_token_tile(int64_t M) {
    const int64_t tiles = ceil_div(M, 256);
    const int64_t bn = ceil_div(ceil_div(M, tiles), 32) * 32;
    return static_cast<int>(std::max<int64_t>(32, std::min<int64_t>(256, bn)));
}
// Shared-memory plan of the small-M kernel (decode_mma.cuh): table, code ring,
// activation ring, two scale buffers, partial sums, barriers.  The rings are as deep
// as the 227 KB allow; a shape whose shallowest rings do not fit is not planned.
struct DecodePlan {
    dec::Params p;
    int smem;
    bool fits;
};
DecodePlan plan_decode(int64_t M, int64_t K, int r) {
    DecodePlan d{};
    dec::Params &p = d.p;
    const int KB = static_cast<int>(K / 64);
    const int sc_q = (dec::kRows * KB + 16 + 15) & ~15;
    const int s2_floats = ((dec::kRows * KB) / 256 + 2 + 3) & ~3;
    p.sc_q = sc_q;
    p.sc_stage = (sc_q + 4 * s2_floats + 127) & ~127;
    p.xa_stage = static_cast<int>((M + r) * dec::kStageBlocks * 128);
    p.c3d = (K % 256 == 0) ? 1 : 0;
    auto total = [&](int dc, int dx) {
        p.dc = dc;
        p.dx = dx;
        p.off_code = dec::kLutBytes;
        p.off_xa = p.off_code + dc * dec::kCodeStage;
        p.off_sc = p.off_xa + dx * p.xa_stage;
        p.off_part = p.off_sc + 2 * p.sc_stage;
        p.off_upart = p.off_part + dec::kPartFloats * 4;
        p.off_ufin = p.off_upart + 4 * 256 * 4;
        p.off_bars = p.off_ufin + 256 * 4;
        const int bars = (2 * dec::kMaxCodeStages + 2 * dec::kMaxXaStages + 4) * 8 + 16;
        return 1024 + p.off_bars + bars;   // + alignment slack of the dynamic base
    };
    int dc = dec::kMaxCodeStages, dx = dec::kMaxXaStages;
    while (total(dc, dx) > dec::kSmemLimit && (dx > 2 || dc > 3)) {
        if (dx > 2) --dx;
        else --dc;
    }
    d.smem = total(dc, dx);
    d.fits = d.smem <= dec::kSmemLimit;
    return d;
}
// Small-M forward: the weight-streaming warp-MMA kernel, which needs no workspace,
// for up to 16 tokens, adapter ranks up to 16 and n_in up to 32768 (when its rings fit).
// (Default storage format only: other formats take the tensor-core path.)
bool use_decode(int64_t M, int64_t K, int r, int32_t format) {
    return format == 0 && M <= 16 && r <= dec::kMaxRank && K / 64 <= dec::kMaxKB && plan_decode(M, K, r).fits;
}
// format < 0: the largest need over every storage format
size_t fwd_ws_bytes(int64_t M, int64_t N, int64_t K, int r, int32_t format) {
    if (format >= 0 && use_decode(M, K, r, format)) return 0;
    const bool split = !use_pair_fwd(M) && plan_gemm(M, N, K / 64).splits > 1;
    return ws_layout(M, N, r, split).total;
}
// dX plan: CTA pairs (256 k columns x BN tokens per pair) at every M.  When the pair
// tiles would fill less than half of the SM pairs (small M), the contraction over n
// is split along blockIdx.z into whole four-stage code chunks, and the splits add
// into an fp32 accumulator.
struct DxPlan {
    int BN;
    int64_t pairs, tiles_tok;
    int splits, nb_per_split;
};
// Tiles of the dX kernel.  wide: 512-token tiles (two accumulators) are allowed.  They are taken
// when the estimated time of the whole grid is lower: per pair tile about 0.73 us per
// 64-n stage at 256 tokens and 0.97 us at 512 (measured on the 70B shapes), plus about
// 10 us of set-up and epilogue, times the number of waves of the pair tiles over the SM pairs.
DxPlan plan_dx(int64_t M, int64_t N, int64_t K, bool wide) {
    DxPlan d;
    d.BN = pair_token_tile(M);
    d.pairs = ceil_div(K, 2 * bwdp::BM);
    d.tiles_tok = ceil_div(M, d.BN);
    const int64_t nb = ceil_div(N, 64);
    const int64_t tiles = d.pairs * d.tiles_tok;
    const int64_t pair_slots = std::max(1, sm_count() / 2);
    int64_t splits = 1;
    if (tiles * 2 <= pair_slots) splits = std::min(ceil_div(pair_slots, tiles), std::max<int64_t>(1, nb / 4));
    d.nb_per_split = static_cast<int>(ceil_div(ceil_div(nb, splits), 4) * 4);
    d.splits = static_cast<int>(ceil_div(nb, d.nb_per_split));
    if (wide && d.splits == 1 && M > 256) {
        const int64_t t512 = ceil_div(M, 512);
        const double w256 = double(ceil_div(tiles, pair_slots)), w512 = double(ceil_div(d.pairs * t512, pair_slots));
        if (w512 * (double(nb) * 0.97 + 10.0) < w256 * (double(nb) * 0.73 + 10.0)) {
            d.BN = 512;
            d.tiles_tok = t512;
        }
    }
    return d;
}
size_t bwd_ws_bytes(int64_t M, int64_t N, int64_t K, int r) {
    return ws_layout(M, K, r, plan_dx(M, N, K, false).splits > 1).total;
}

// Launches the rank-r tensor-core product out[i*ld_i + j*ld_j] += scaling *
// sum_t P(i, t) Q(j, t) (see skinny_mma.cuh) over bf16 operands:
//   P: p_mn = 0 -> [I, T] row-major (t contiguous); p_mn = 1 -> [T, I] row-major
//   Q: q_mn = 0 -> [r, T] row-major;                q_mn = 1 -> [T, r] row-major
// The output must already hold zeros or the values to accumulate into.
qlora_status launch_skinny(const void *P, int p_mn, const void *Q, int q_mn, int64_t T, int64_t I, int r,
                           float scaling, float *out, int64_t ld_i, int64_t ld_j, cudaStream_t st) {
    using namespace skinny;
    Params p;
    p.T = static_cast<int>(T);
    p.I = static_cast<int>(I);
    p.r = r;
    p.p_mn = p_mn;
    p.q_mn = q_mn;
    CUtensorMap tmP, tmQ;
    // P: one 3-D box per stage when the t (K-major) or i (MN-major) extent is whole 64-element chunks
    const int64_t p_rows = p_mn ? T : I, p_cols = p_mn ? I : T;
    p.p_3d = p_cols % 64 == 0;
    if (p.p_3d)
        QL_TRY(make_tmap_chunks(&tmP, P, p_rows, p_cols, BT, 2));
    else
        QL_TRY(make_tmap_2d(&tmP, P, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p_rows, p_cols, p_cols, BT, 64,
                            CU_TENSOR_MAP_SWIZZLE_128B));
    if (!q_mn) {
        // [r, T]: Nq rows per 64-t chunk, rows past r zero-filled
        p.Nq = static_cast<int>(ceil_div(r, 16) * 16);
        p.q_3d = T % 64 == 0;
        p.q_atoms = 0;
        p.q_span = 128;
        p.q_bytes = 2 * p.Nq * 128;
        if (p.q_3d)
            QL_TRY(make_tmap_chunks(&tmQ, Q, r, T, p.Nq, 2));
        else
            QL_TRY(make_tmap_2d(&tmQ, Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, T, T, p.Nq, 64,
                                CU_TENSOR_MAP_SWIZZLE_128B));
    } else {
        // [T, r]: j contiguous; the narrowest swizzle atom that covers r (16, 32 or 64 elements)
        p.Nq = r <= 16 ? 16 : (r <= 32 ? 32 : (r <= 64 ? 64 : 128));
        p.q_span = p.Nq >= 64 ? 128 : p.Nq * 2;
        p.q_atoms = p.Nq >= 64 ? p.Nq / 64 : 1;
        p.q_3d = 0;
        p.q_bytes = p.q_atoms * BT * p.q_span;
        const CUtensorMapSwizzle swz = p.q_span == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : p.q_span == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                        : CU_TENSOR_MAP_SWIZZLE_32B;
        QL_TRY(make_tmap_2d(&tmQ, Q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, r, r, BT, p.q_span / 2, swz));
    }
    p.stages = std::min(kMaxStages, kRingBudget / stage_bytes(p.q_bytes));
    p.units = ceil_div(I, BI) * ceil_div(T, BT);
    p.scaling = scaling;
    p.out = out;
    p.ld_i = ld_i;
    p.ld_j = ld_j;
    const int smem = smem_bytes(p.stages, p.q_bytes);
    QL_TRY(set_smem(skinny_mma_kernel, smem));
    // stream-K: two CTAs per SM, each a contiguous run of (tile, stage) units
    const int64_t grid = std::min<int64_t>(p.units, 2 * sm_count());
    skinny_mma_kernel<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(tmP, tmQ, p);
    return launch_check("skinny_mma_kernel launch");
}

qlora_status launch_finalize(const float *acc, int64_t n, float scaling, uint16_t *save, uint16_t *scaled,
                             cudaStream_t st) {
    skinny::finalize_rank_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 2048)), 256, 0, st>>>(
        acc, n, scaling, save, scaled);
    return launch_check("finalize_rank_kernel launch");
}

qlora_status check_rank(int r, float scaling, const void *A, const void *B) {
    if (r == 0) return QLORA_OK;
    if (r < 8 || r > 128 || r % 8) return fail(QLORA_ERR_SHAPE, "r (%d) must be 0 or a multiple of 8 in [8, 128]", r);
    if (!A || !B) return fail(QLORA_ERR_ARG, "A and B must be non-NULL when r > 0");
    if (!aligned16(A) || !aligned16(B)) return fail(QLORA_ERR_ALIGN, "A and B must be 16-byte aligned");
    if (!std::isfinite(scaling)) return fail(QLORA_ERR_ARG, "scaling must be finite");
    return QLORA_OK;
}

// Device address of g_static_scratch on the current device, looked up by the
// first call on that device and cached (one lookup per device, under a lock).
qlora_status static_scratch(void **out) {
    constexpr int kMaxDevices = 64;
    static void *ptrs[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    QL_TRY(cuda_check(cudaGetDevice(&dev), "cudaGetDevice"));
    if (dev < 0 || dev >= kMaxDevices)
        return fail(QLORA_ERR_UNSUPPORTED, "device %d: the static scratch serves devices 0..%d", dev, kMaxDevices - 1);
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        QL_TRY(cuda_check(cudaGetSymbolAddress(&p, g_static_scratch), "cudaGetSymbolAddress(static scratch)"));
        if (!p) return fail(QLORA_ERR_CUDA, "cudaGetSymbolAddress returned NULL for the static scratch");
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return QLORA_OK;
}

// The packed base weight as the CTA-pair GEMM kernels see it: 4-bit codes with the
// scales of their storage format and the levels of their quant type, or Q8_0 int8
// codes with an fp16 scale per 32 weights.
struct BaseW {
    const uint8_t *codes;     // [N, K/2] (4-bit) or [N, K] (int8) bytes
    bool q8;
    ScaleSrc sc;              // 4-bit only
    const uint16_t *d8;       // Q8_0 only
    const float *level;       // 4-bit only: the 16 levels
};

// Tile order of a pair kernel (raster_tile in ptx.cuh): nw weight tiles of w_bytes each
// and nt token tiles of t_bytes each.  A band of tiles that fits the L2 budget is read
// from DRAM once; the other operand streams once per band.  Mode 0 keeps a band of
// weight tiles (DRAM bytes: all weight + all tokens x bands), mode 1 a band of token
// tiles (all tokens + all weight x bands); the smaller total wins.
struct Raster {
    int mode, group;
};
Raster pair_raster(int64_t nw, int64_t nt, double w_bytes, double t_bytes) {
    const double budget = 64e6;   // half of the 126 MB L2: the rest holds the stream and the output
    const int64_t g0 = std::max<int64_t>(1, std::min<int64_t>(nw, static_cast<int64_t>(budget / w_bytes)));
    const int64_t g1 = std::max<int64_t>(1, std::min<int64_t>(nt, static_cast<int64_t>(budget / t_bytes)));
    const double wt = double(nw) * w_bytes, tt = double(nt) * t_bytes;
    const double c0 = wt + tt * double(ceil_div(nw, g0));
    const double c1 = tt + wt * double(ceil_div(nt, g1));
    return c0 <= c1 ? Raster{0, static_cast<int>(g0)} : Raster{1, static_cast<int>(g1)};
}

// Forward base GEMM plus the adapter stage on CTA pairs: Y = X W'^T + us B^T, with
// us = bf16(scaling * U) [M, r] already in the workspace (r > 0).
qlora_status launch_fwd_pair(const BaseW &bw, const qlora_bf16 *X, int64_t M, int64_t N, int64_t K,
                             const qlora_bf16 *B, int r, const uint16_t *us, qlora_bf16 *Y, cudaStream_t st) {
    const int BN = pair_token_tile(M);
    CUtensorMap tmX, tmC, tmU;
    QL_TRY(make_tmap_chunks(&tmX, X, M, K, BN / 2, 2));
    const uint64_t row_bytes = bw.q8 ? uint64_t(K) : uint64_t(K / 2);
    QL_TRY(make_tmap_2d(&tmC, bw.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, row_bytes, row_bytes, 128, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B));
    if (r > 0)
        QL_TRY(make_tmap_2d(&tmU, us, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, r, r, BN / 2, 64,
                            CU_TENSOR_MAP_SWIZZLE_128B));
    else
        tmU = tmX;
    // the Y tile store of each CTA: [BN tokens, 128 rows of W] boxes, unswizzled
    CUtensorMap tmY;
    QL_TRY(make_tmap_2d(&tmY, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, N, BN, fwdp::BM,
                        CU_TENSOR_MAP_SWIZZLE_NONE));
    fwdp::Params p;
    p.sc = bw.sc;
    p.d8 = bw.d8;
    p.Blora = B;
    p.Y = Y;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.r = r;
    p.BN = BN;
    const int64_t nw = ceil_div(N, 256), nt = ceil_div(M, BN);
    // launch order (weight tile fastest): measured as fast as any banded order here, where
    // the re-read weight tiles come at well under the DRAM bandwidth
    p.raster_mode = 0;
    p.raster_group = static_cast<int>(nw);
    for (int i = 0; i < 16; ++i) p.level[i] = bw.q8 ? 0.f : bw.level[i];
    dim3 grid(static_cast<unsigned>(2 * nw), static_cast<unsigned>(nt), 1);
    if (bw.q8) {
        QL_TRY(set_smem(fwdp::fused_fwd_pair_kernel<true>, fwdp::smem_bytes(256, true)));
        fwdp::fused_fwd_pair_kernel<true><<<grid, fwdp::kThreads, fwdp::smem_bytes(BN, true), st>>>(tmX, tmC, tmU, tmY, p);
    } else {
        QL_TRY(set_smem(fwdp::fused_fwd_pair_kernel<false>, fwdp::smem_bytes(256)));
        fwdp::fused_fwd_pair_kernel<false><<<grid, fwdp::kThreads, fwdp::smem_bytes(BN), st>>>(tmX, tmC, tmU, tmY, p);
    }
    return launch_check("fused_fwd_pair_kernel launch");
}

// dX kernel forms (stage slots = dequant groups kS, stages per code chunk kCS): 4-bit
// codes take kS = kCS = 4 at every tile (165 KB of shared memory at 256 tokens, 226 KB at
// 512); 8-bit codes take kS = kCS = 4 up to 256 tokens (198 KB) and kS = kCS = 3 at 512
// (194 KB: four-stage 8-bit chunks do not fit beside the 512-token rings).
template <bool kQ8, int kS, int kCS>
qlora_status launch_dx_variant(dim3 grid, int BN, int most, const CUtensorMap &tmY, const CUtensorMap &tmC,
                               const CUtensorMap &tmG, const CUtensorMap &tmD, const bwdp::Params &p,
                               cudaStream_t st) {
    // most: the largest tile this form runs, which sets its shared-memory limit
    QL_TRY(set_smem(bwdp::fused_bwd_pair_kernel<kQ8, kS, kCS>, bwdp::smem_bytes(most, kQ8, kS, kCS)));
    bwdp::fused_bwd_pair_kernel<kQ8, kS, kCS>
        <<<grid, bwdp::threads_for(kS), bwdp::smem_bytes(BN, kQ8, kS, kCS), st>>>(tmY, tmC, tmG, tmD, p);
    return QLORA_OK;
}

// dX = dY W' + gs A on CTA pairs (gs = bf16(scaling * G) [M, r] in the workspace when
// r > 0), split over n into dxacc (zeroed by the caller) when the plan says so.
qlora_status launch_dx_pair(const BaseW &bw, const DxPlan &g, const qlora_bf16 *dY, int64_t M, int64_t N, int64_t K,
                            const qlora_bf16 *A, int r, const uint16_t *gs, qlora_bf16 *dX, float *dxacc,
                            cudaStream_t st) {
    const int BN = g.BN;
    const int box = std::min(BN, 256) / 2;        // dY rows per TMA box: one CTA's share of an accumulator
    CUtensorMap tmY, tmC, tmG;
    QL_TRY(make_tmap_2d(&tmY, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, N, box, 64,
                        CU_TENSOR_MAP_SWIZZLE_128B));
    const int crow = bwdp::chunk_rows(bw.q8 && BN > 256 ? 3 : 4);   // code rows per TMA box
    if (bw.q8)
        QL_TRY(make_tmap_2d(&tmC, bw.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, K, crow, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B));
    else
        QL_TRY(make_tmap_2d(&tmC, bw.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, crow, 64,
                            CU_TENSOR_MAP_SWIZZLE_64B));
    if (r > 0)
        QL_TRY(make_tmap_2d(&tmG, gs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, r, r, box, 64,
                            CU_TENSOR_MAP_SWIZZLE_128B));
    else
        tmG = tmY;
    // the dX tile store: [tokens, 128 k] boxes, unswizzled (with splits the epilogue adds into dxacc instead)
    CUtensorMap tmD;
    if (!dxacc)
        QL_TRY(make_tmap_2d(&tmD, dX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, K, std::min(BN, 256),
                            bwdp::BM, CU_TENSOR_MAP_SWIZZLE_NONE));
    else
        tmD = tmY;
    bwdp::Params p;
    p.sc = bw.sc;
    p.d8 = bw.d8;
    p.Alora = A;
    p.dX = dX;
    p.dXacc = dxacc;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.r = r;
    p.BN = BN;
    p.nb_per_split = g.nb_per_split;
    // a weight tile: 256 columns of codes over the split's n rows; a token tile: BN rows of dY
    const double n_split = double(std::min<int64_t>(N, int64_t(g.nb_per_split) * 64));
    const Raster ras = pair_raster(g.pairs, g.tiles_tok, 256.0 * n_split * (bw.q8 ? 1.0 : 0.5),
                                   double(BN) * n_split * 2.0);
    p.raster_mode = ras.mode;
    p.raster_group = ras.group;
    for (int i = 0; i < 16; ++i) p.level[i] = bw.q8 ? 0.f : bw.level[i];
    dim3 grid(static_cast<unsigned>(2 * g.pairs), static_cast<unsigned>(g.tiles_tok), static_cast<unsigned>(g.splits));
    if (bw.q8 && BN > 256)
        QL_TRY((launch_dx_variant<true, 3, 3>(grid, BN, 512, tmY, tmC, tmG, tmD, p, st)));
    else if (bw.q8)
        QL_TRY((launch_dx_variant<true, 4, 4>(grid, BN, 256, tmY, tmC, tmG, tmD, p, st)));
    else
        QL_TRY((launch_dx_variant<false, 4, 4>(grid, BN, 512, tmY, tmC, tmG, tmD, p, st)));
    QL_TRY(launch_check("fused_bwd_pair_kernel launch"));
    if (dxacc) QL_TRY(launch_finalize(dxacc, M * K, 1.0f, dX, nullptr, st));
    return QLORA_OK;
}

// The rank-r side product of the forward (U = X A^T: us = bf16(scaling U), U_save = bf16(U))
// or of dX (G = dY B), into the workspace.
qlora_status rank_side_product(bool fwd, const qlora_bf16 *act, int64_t M, int64_t width, const qlora_bf16 *factor,
                               int r, float scaling, uint16_t *scaled, float *acc, qlora_bf16 *save, cudaStream_t st) {
    QL_TRY(cuda_check(cudaMemsetAsync(acc, 0, size_t(M) * r * 4, st), "zero rank accumulator"));
    if (fwd) QL_TRY(launch_skinny(act, 0, factor, 0, width, M, r, 1.0f, acc, r, 1, st));
    else QL_TRY(launch_skinny(act, 0, factor, 1, width, M, r, 1.0f, acc, r, 1, st));
    return launch_finalize(acc, M * r, scaling, save, scaled, st);
}

BaseW base_of(const qlora_nf4_weight *w, const Codebook &cb) {
    BaseW b;
    b.codes = w->codes;
    b.q8 = false;
    b.sc = scale_src(w);
    b.d8 = nullptr;
    b.level = cb.level;
    return b;
}

qlora_status check_ws(void *ws, size_t ws_bytes, size_t need) {
    if (need == 0) return QLORA_OK;
    if (!ws) return fail(QLORA_ERR_WORKSPACE, "workspace is NULL but %zu bytes are needed", need);
    if (!aligned16(ws)) return fail(QLORA_ERR_ALIGN, "workspace must be 16-byte aligned");
    if (ws_bytes < need) return fail(QLORA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    return QLORA_OK;
}


}  // namespace

extern "C" {

size_t qlora_packed_bytes(int64_t numel) { return qlora_packed_bytes_fmt(numel, 0); }

size_t qlora_packed_bytes_fmt(int64_t numel, int32_t format) {
    if (!fmt_valid(format)) return 0;
    const int64_t blk = fmt_block(format);
    if (numel <= 0 || numel % blk) return 0;
    const int64_t nb = numel / blk;
    if (!fmt_dq(format)) return size_t(numel / 2) + 4 * size_t(nb);
    return size_t(numel / 2) + size_t(nb) + 4 * size_t(ceil_div(nb, 256));
}

qlora_status qlora_nf4_codebook(float out[16]) {
    if (!out) return fail(QLORA_ERR_ARG, "out is NULL");
    const Codebook &cb = codebook();
    for (int i = 0; i < 16; ++i) out[i] = cb.level[i];
    return QLORA_OK;
}

qlora_status qlora_codebook(int quant_type, float *out) {
    if (!out) return fail(QLORA_ERR_ARG, "out is NULL");
    if (quant_type != QLORA_QT_NF4 && quant_type != QLORA_QT_FP4)
        return fail(QLORA_ERR_ARG, "quant_type (%d) must be QLORA_QT_NF4 (0) or QLORA_QT_FP4 (1)", quant_type);
    const Codebook &cb = codebook_for(quant_type);
    for (int i = 0; i < 16; ++i) out[i] = cb.level[i];
    return QLORA_OK;
}

const char *qlora_last_error(void) { return t_last_error; }

qlora_status qlora_set_wait_limit_ns(uint64_t ns) {
    if (ns < 1000000ull || ns > 60000000000ull)
        return fail(QLORA_ERR_ARG, "wait limit %llu ns outside [1e6, 6e10]", (unsigned long long)ns);
    QL_TRY(require_sm100());
    const unsigned long long v = ns;
    return cuda_check(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)), "set the wait limit");
}

qlora_status qlora_probe_wait_timeout(void *stream) {
    QL_TRY(require_sm100());
    wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
    return launch_check("wait_probe_kernel launch");
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return std::max<size_t>(256, std::max(fwd_ws_bytes(M, N, K, r, -1), bwd_ws_bytes(M, N, K, r)));
}

qlora_status qlora_sync_status(void *stream) {
    QL_TRY(cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize"));
    int v = 0;
    QL_TRY(cuda_check(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)), "read device error word"));
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
        if (v == kDeviceErrTmemStore)
            return fail(QLORA_ERR_CUDA, "a tensor-memory store did not read back as written (device error %d)", v);
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
    const int blk = fmt_block(w->format);
    const int64_t nblocks = numel / blk;
    const int64_t ngroups = ceil_div(nblocks, 256);
    if (ngroups > INT32_MAX) return fail(QLORA_ERR_SHAPE, "weight too large");
    const dim3 grid(static_cast<unsigned>(ngroups));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const CodebookArg cb = codebook_arg(w->quant_type);
    const bool dq = fmt_dq(w->format), after = (w->format & QLORA_FMT_CODES_AFTER_DQ) != 0;
#define QL_ENC(B, D, A) nf4_encode_kernel<B, D, A><<<grid, kEncThreads, 0, st>>>(W, w->codes, w->scales, w->scales2, nblocks, cb)
    if (blk == 64) {
        if (!dq) QL_ENC(64, false, false);
        else if (after) QL_ENC(64, true, true);
        else QL_ENC(64, true, false);
    } else {
        if (!dq) QL_ENC(128, false, false);
        else if (after) QL_ENC(128, true, true);
        else QL_ENC(128, true, false);
    }
#undef QL_ENC
    return launch_check("nf4_encode_kernel launch");
}

qlora_status qlora_dequant(const qlora_nf4_weight *w, void *out, int out_is_bf16, void *stream) {
    QL_TRY(check_weight(w));
    if (!out) return fail(QLORA_ERR_ARG, "out is NULL");
    if (!aligned16(out)) return fail(QLORA_ERR_ALIGN, "out must be 16-byte aligned");
    if (out_is_bf16 != 0 && out_is_bf16 != 1) return fail(QLORA_ERR_ARG, "out_is_bf16 must be 0 or 1");
    QL_TRY(require_sm100());
    const int64_t n16 = w->n_out * w->n_in / 16;
    const int64_t grid = std::min<int64_t>(ceil_div(n16, 256), int64_t(sm_count()) * 8);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (out_is_bf16)
        nf4_dequant_kernel<true><<<static_cast<unsigned>(grid), 256, 0, st>>>(w->codes, scale_src(w), out, n16,
                                                                               codebook_arg(w->quant_type));
    else
        nf4_dequant_kernel<false><<<static_cast<unsigned>(grid), 256, 0, st>>>(w->codes, scale_src(w), out, n16,
                                                                                codebook_arg(w->quant_type));
    return launch_check("nf4_dequant_kernel launch");
}

qlora_status qlora_lora_merge_requant(const qlora_nf4_weight *w_in, const qlora_bf16 *A, const qlora_bf16 *B, int r,
                                      float scaling, float *W_scratch, const qlora_nf4_weight *w_out, void *stream) {
    QL_TRY(check_weight(w_in));
    QL_TRY(check_weight(w_out));
    if (w_out->n_out != w_in->n_out || w_out->n_in != w_in->n_in)
        return fail(QLORA_ERR_SHAPE, "w_out must have the shape of w_in");
    QL_TRY(check_rank(r, scaling, A, B));
    if (!W_scratch) return fail(QLORA_ERR_ARG, "W_scratch is NULL");
    if (!aligned16(W_scratch)) return fail(QLORA_ERR_ALIGN, "W_scratch must be 16-byte aligned");
    QL_TRY(require_sm100());
    // x: a row's groups of kMergeCols weights; y: groups of kMergeRows rows, about 8 CTAs per SM in all
    const int64_t gx = std::min<int64_t>(ceil_div(w_in->n_in / kMergeCols, kMergeThreads), 32);
    const int64_t gy = std::min<int64_t>(ceil_div(w_in->n_out, kMergeRows),
                                         std::max<int64_t>(1, int64_t(sm_count()) * 8 / gx));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    nf4_lora_merge_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kMergeThreads, 0, st>>>(
        w_in->codes, scale_src(w_in), r > 0 ? reinterpret_cast<const uint16_t *>(A) : nullptr,
        r > 0 ? reinterpret_cast<const uint16_t *>(B) : nullptr, r, r > 0 ? scaling : 0.f, w_in->n_out, w_in->n_in,
        W_scratch, codebook_arg(w_in->quant_type));
    QL_TRY(launch_check("nf4_lora_merge_kernel launch"));
    return qlora_quantize_nf4_dq(W_scratch, w_out, stream);
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
    const size_t need = fwd_ws_bytes(M, N, K, r, w->format);
    QL_TRY(check_ws(ws, ws_bytes, need));
    QL_TRY(require_sm100());
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (use_decode(M, K, r, w->format)) {
        DecodePlan d = plan_decode(M, K, r);
        dec::Params &p = d.p;
        p.codes = w->codes;
        p.scales = w->scales;
        p.scales2 = w->scales2;
        p.Blora = r > 0 ? B : nullptr;
        p.Y = Y;
        p.U_save = r > 0 ? U_save : nullptr;
        p.M = static_cast<int>(M);
        p.N = static_cast<int>(N);
        p.K = static_cast<int>(K);
        p.r = r;
        p.units = static_cast<int>(ceil_div(N, dec::kRows));
        p.scaling = scaling;
        const Codebook &cbd = codebook_for(w->quant_type);
        for (int i = 0; i < 16; ++i) p.level[i] = cbd.level[i];
        // codes as u8 [N, K/2] in [32 rows x 128 B] boxes (3-D: four 256-k chunks per box);
        // X and A as [K/64][rows][64] bf16 chunks, sixteen chunks per box
        CUtensorMap tmC, tmX, tmA;
        if (p.c3d) QL_TRY(make_tmap_code_chunks(&tmC, w->codes, N, K, dec::kRows, dec::kStageK / 256));
        else QL_TRY(make_tmap_2d(&tmC, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, K / 2, dec::kRows, 128,
                                 CU_TENSOR_MAP_SWIZZLE_128B));
        QL_TRY(make_tmap_chunks(&tmX, X, M, K, static_cast<uint32_t>(M), dec::kStageBlocks));
        if (r > 0) QL_TRY(make_tmap_chunks(&tmA, A, r, K, static_cast<uint32_t>(r), dec::kStageBlocks));
        else tmA = tmX;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(p.units, sm_count())));
        cfg.blockDim = dim3(dec::kThreads);
        cfg.dynamicSmemBytes = d.smem;
        cfg.stream = st;
        // programmatic dependent launch: the kernel builds its table and initialises its
        // barriers before waiting for the preceding grid
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        if (M <= 8) {
            QL_TRY(set_smem(dec::decode_kernel<1>, d.smem));
            QL_TRY(cuda_check(cudaLaunchKernelEx(&cfg, dec::decode_kernel<1>, tmC, tmX, tmA, p), "decode_kernel launch"));
        } else {
            QL_TRY(set_smem(dec::decode_kernel<2>, d.smem));
            QL_TRY(cuda_check(cudaLaunchKernelEx(&cfg, dec::decode_kernel<2>, tmC, tmX, tmA, p), "decode_kernel launch"));
        }
        return QLORA_OK;
    }

    const bool pair = use_pair_fwd(M);
    const GemmPlan g = plan_gemm(M, N, K / 64);
    const bool split = !pair && g.splits > 1;
    const WsLayout L = ws_layout(M, N, r, split);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    uint16_t *us = reinterpret_cast<uint16_t *>(wsb);
    float *uacc = reinterpret_cast<float *>(wsb + L.rank_bf16);
    float *yacc = split ? reinterpret_cast<float *>(wsb + L.rank_bf16 + L.rank_acc) : nullptr;
    // U = X A^T on tensor cores, then bf16 copies: U (saved) and scaling * U (adapter chunk)
    if (r > 0) QL_TRY(rank_side_product(true, X, M, K, A, r, scaling, us, uacc, U_save, st));
    const Codebook &cb = codebook_for(w->quant_type);

    if (pair) return launch_fwd_pair(base_of(w, cb), X, M, N, K, B, r, us, Y, st);

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
    p.sc = scale_src(w);
    p.Blora = B;
    p.Y = Y;
    p.Yacc = yacc;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.r = r;
    p.BN = g.BN;
    p.kb_per_split = g.stages_per_split;
    for (int i = 0; i < 16; ++i) p.level[i] = cb.level[i];

    const int smem = fwd::smem_bytes(g.BN);
    QL_TRY(set_smem(fwd::fused_fwd_kernel, fwd::smem_bytes(256)));
    dim3 grid(static_cast<unsigned>(g.tiles_rows), static_cast<unsigned>(g.tiles_tok), static_cast<unsigned>(g.splits));
    fwd::fused_fwd_kernel<<<grid, fwd::kThreads, smem, st>>>(tmX, tmC, tmU, p);
    QL_TRY(launch_check("fused_fwd_kernel launch"));
    if (yacc) QL_TRY(launch_finalize(yacc, M * N, 1.0f, Y, nullptr, st));
    return QLORA_OK;
}

qlora_status qlora_lora_linear_fwd_static_ws(const qlora_nf4_weight *w, const qlora_bf16 *X, int64_t M,
                                             const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                             qlora_bf16 *Y, qlora_bf16 *U_save, void *stream) {
    // the size check needs only host arithmetic: reject before any CUDA call
    QL_TRY(check_weight(w));
    if (M <= 0 || M > INT32_MAX) return fail(QLORA_ERR_SHAPE, "M (%lld) must be in [1, 2^31)", (long long)M);
    QL_TRY(check_rank(r, scaling, A, B));
    const size_t need = fwd_ws_bytes(M, w->n_out, w->n_in, r, w->format);
    if (need > QLORA_STATIC_SCRATCH_BYTES)
        return fail(QLORA_ERR_WORKSPACE,
                    "M=%lld N=%lld K=%lld r=%d needs %zu bytes of scratch; the static scratch holds %zu "
                    "(use qlora_lora_linear_fwd with a caller workspace)",
                    (long long)M, (long long)w->n_out, (long long)w->n_in, r, need,
                    size_t(QLORA_STATIC_SCRATCH_BYTES));
    QL_TRY(require_sm100());
    void *scratch = nullptr;
    QL_TRY(static_scratch(&scratch));
    return qlora_lora_linear_fwd(w, X, M, A, B, r, scaling, Y, U_save, scratch, QLORA_STATIC_SCRATCH_BYTES, stream);
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

    // CTA pairs at every M; split-K over n when the output tiles are few
    const DxPlan g = plan_dx(M, N, K, true);
    const bool split = g.splits > 1;
    const WsLayout L = ws_layout(M, K, r, split);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    uint16_t *gs = reinterpret_cast<uint16_t *>(wsb);
    float *gacc = reinterpret_cast<float *>(wsb + L.rank_bf16);
    float *dxacc = split ? reinterpret_cast<float *>(wsb + L.rank_bf16 + L.rank_acc) : nullptr;
    // G = dY B on tensor cores (B read MN-major), then bf16 copies G and scaling * G
    if (r > 0) QL_TRY(rank_side_product(false, dY, M, N, B, r, scaling, gs, gacc, G_save, st));
    if (dxacc) QL_TRY(cuda_check(cudaMemsetAsync(dxacc, 0, size_t(M) * K * 4, st), "zero split accumulator"));
    return launch_dx_pair(base_of(w, codebook_for(w->quant_type)), g, dY, M, N, K, A, r, gs, dX, dxacc, st);
}

// ------------------------------------------------------------------ Q8_0 route

static qlora_status check_q8(const qlora_q8_0_weight *w) {
    if (!w) return fail(QLORA_ERR_ARG, "weight descriptor is NULL");
    if (w->n_out <= 0 || w->n_in <= 0) return fail(QLORA_ERR_SHAPE, "n_out and n_in must be positive");
    if (w->n_in % 64) return fail(QLORA_ERR_SHAPE, "n_in (%lld) must be a multiple of 64", (long long)w->n_in);
    if (w->n_out > (int64_t(1) << 31) || w->n_in > (int64_t(1) << 31))
        return fail(QLORA_ERR_SHAPE, "n_out and n_in must be below 2^31");
    if (!w->q || !w->d) return fail(QLORA_ERR_ARG, "weight buffers must be non-NULL");
    if (!aligned16(w->q) || !aligned16(w->d)) return fail(QLORA_ERR_ALIGN, "weight buffers must be 16-byte aligned");
    return QLORA_OK;
}

static BaseW base_of_q8(const qlora_q8_0_weight *w) {
    BaseW b;
    b.codes = reinterpret_cast<const uint8_t *>(w->q);
    b.q8 = true;
    b.sc = ScaleSrc{nullptr, nullptr, 0, 1};
    b.d8 = w->d;
    b.level = nullptr;
    return b;
}

size_t qlora_q8_0_packed_bytes(int64_t numel) {
    if (numel <= 0 || numel % 32) return 0;
    return size_t(numel) + 2 * size_t(numel / 32);
}

qlora_status qlora_quantize_q8_0(const float *W, const qlora_q8_0_weight *w, void *stream) {
    QL_TRY(check_q8(w));
    if (!W) return fail(QLORA_ERR_ARG, "W is NULL");
    if (!aligned16(W)) return fail(QLORA_ERR_ALIGN, "W must be 16-byte aligned");
    QL_TRY(require_sm100());
    const int64_t numel = w->n_out * w->n_in;
    const int64_t grid = std::min<int64_t>(ceil_div(ceil_div(numel, 128), 8), int64_t(sm_count()) * 16);
    q8_0_encode_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(W, w->q, w->d,
                                                                                                 numel);
    return launch_check("q8_0_encode_kernel launch");
}

qlora_status qlora_dequant_q8_0(const qlora_q8_0_weight *w, void *out, int out_is_bf16, void *stream) {
    QL_TRY(check_q8(w));
    if (!out) return fail(QLORA_ERR_ARG, "out is NULL");
    if (!aligned16(out)) return fail(QLORA_ERR_ALIGN, "out must be 16-byte aligned");
    if (out_is_bf16 != 0 && out_is_bf16 != 1) return fail(QLORA_ERR_ARG, "out_is_bf16 must be 0 or 1");
    QL_TRY(require_sm100());
    const int64_t n16 = w->n_out * w->n_in / 16;
    const int64_t grid = std::min<int64_t>(ceil_div(n16, 256), int64_t(sm_count()) * 8);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (out_is_bf16) q8_0_dequant_kernel<true><<<static_cast<unsigned>(grid), 256, 0, st>>>(w->q, w->d, out, n16);
    else q8_0_dequant_kernel<false><<<static_cast<unsigned>(grid), 256, 0, st>>>(w->q, w->d, out, n16);
    return launch_check("q8_0_dequant_kernel launch");
}

qlora_status qlora_q8_0_lora_linear_fwd(const qlora_q8_0_weight *w, const qlora_bf16 *X, int64_t M,
                                        const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                        qlora_bf16 *Y, qlora_bf16 *U_save, void *ws, size_t ws_bytes, void *stream) {
    QL_TRY(check_q8(w));
    if (!X || !Y) return fail(QLORA_ERR_ARG, "X and Y must be non-NULL");
    if (!aligned16(X) || !aligned16(Y)) return fail(QLORA_ERR_ALIGN, "X and Y must be 16-byte aligned");
    if (U_save && !aligned16(U_save)) return fail(QLORA_ERR_ALIGN, "U_save must be 16-byte aligned");
    if (M <= 0 || M > INT32_MAX) return fail(QLORA_ERR_SHAPE, "M (%lld) must be in [1, 2^31)", (long long)M);
    QL_TRY(check_rank(r, scaling, A, B));
    const int64_t N = w->n_out, K = w->n_in;
    const WsLayout L = ws_layout(M, N, r, false);
    QL_TRY(check_ws(ws, ws_bytes, L.total));
    QL_TRY(require_sm100());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    uint16_t *us = reinterpret_cast<uint16_t *>(wsb);
    if (r > 0)
        QL_TRY(rank_side_product(true, X, M, K, A, r, scaling, us, reinterpret_cast<float *>(wsb + L.rank_bf16),
                                 U_save, st));
    // every M on CTA pairs (a small M pads the token tile)
    return launch_fwd_pair(base_of_q8(w), X, M, N, K, B, r, us, Y, st);
}

qlora_status qlora_q8_0_lora_linear_bwd_dx(const qlora_q8_0_weight *w, const qlora_bf16 *dY, int64_t M,
                                           const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                           qlora_bf16 *dX, qlora_bf16 *G_save, void *ws, size_t ws_bytes,
                                           void *stream) {
    QL_TRY(check_q8(w));
    if (!dY || !dX) return fail(QLORA_ERR_ARG, "dY and dX must be non-NULL");
    if (!aligned16(dY) || !aligned16(dX)) return fail(QLORA_ERR_ALIGN, "dY and dX must be 16-byte aligned");
    if (G_save && !aligned16(G_save)) return fail(QLORA_ERR_ALIGN, "G_save must be 16-byte aligned");
    if (M <= 0 || M > INT32_MAX) return fail(QLORA_ERR_SHAPE, "M (%lld) must be in [1, 2^31)", (long long)M);
    QL_TRY(check_rank(r, scaling, A, B));
    const int64_t N = w->n_out, K = w->n_in;
    if (N % 8) return fail(QLORA_ERR_SHAPE, "n_out (%lld) must be a multiple of 8 for the dX pass", (long long)N);
    const DxPlan g = plan_dx(M, N, K, true);
    const bool split = g.splits > 1;
    const WsLayout L = ws_layout(M, K, r, split);
    QL_TRY(check_ws(ws, ws_bytes, L.total));
    QL_TRY(require_sm100());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    uint16_t *gs = reinterpret_cast<uint16_t *>(wsb);
    float *dxacc = split ? reinterpret_cast<float *>(wsb + L.rank_bf16 + L.rank_acc) : nullptr;
    if (r > 0)
        QL_TRY(rank_side_product(false, dY, M, N, B, r, scaling, gs, reinterpret_cast<float *>(wsb + L.rank_bf16),
                                 G_save, st));
    if (dxacc) QL_TRY(cuda_check(cudaMemsetAsync(dxacc, 0, size_t(M) * K * 4, st), "zero split accumulator"));
    return launch_dx_pair(base_of_q8(w), g, dY, M, N, K, A, r, gs, dX, dxacc, st);
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
    if (K % 64 || N % 8) return fail(QLORA_ERR_SHAPE, "K must be a multiple of 64 and N a multiple of 8");
    if (accumulate != 0 && accumulate != 1) return fail(QLORA_ERR_ARG, "accumulate must be 0 or 1");
    if (!std::isfinite(scaling)) return fail(QLORA_ERR_ARG, "scaling must be finite");
    QL_TRY(require_sm100());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!accumulate) {
        QL_TRY(cuda_check(cudaMemsetAsync(dA, 0, size_t(r) * K * 4, st), "zero dA"));
        QL_TRY(cuda_check(cudaMemsetAsync(dB, 0, size_t(N) * r * 4, st), "zero dB"));
    }
    // dA^T [K, r] = s X^T G  and  dB [N, r] = s dY^T U, contraction over the M tokens
    QL_TRY(launch_skinny(X, 1, G, 1, M, K, r, scaling, dA, 1, K, st));
    QL_TRY(launch_skinny(dY, 1, U, 1, M, N, r, scaling, dB, r, 1, st));
    return QLORA_OK;
}

}  // extern "C"
