// tm_gemm.cu -- instantiations and launchers of the tcgen05 kernels (grouped GEMM, fused sub-layer).
#include <string.h>
#include "tm_fused128.cuh"
#include "tm_internal.h"

namespace tml {

template <int W, int AM>
static cudaError_t launch_fused_one(const CUtensorMap& a, const CUtensorMap& g, const CUtensorMap& u,
                                    const CUtensorMap& d, const FusedParams& p, int grid, cudaStream_t st) {
    using C = FusedCfg<W, AM>;
    auto kern = fused_swiglu_kernel<W, AM>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    ProfileScope ps_("fused_swiglu", st);
    kern<<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(a, g, u, d, p);
    return cudaGetLastError();
}

template <int W, int AM, bool F8>
static cudaError_t launch_fused128_one(const CUtensorMap& a, const CUtensorMap& g, const CUtensorMap& u,
                                       const CUtensorMap& d, const CUtensorMap& r, const CUtensorMap& e,
                                       const CUtensorMap& o, const FusedParams& p, int grid, cudaStream_t st) {
    using C = Fused128Cfg<W, AM, F8>;
    auto kern = fused128_swiglu_kernel<W, AM, F8>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    ProfileScope ps_(F8 ? "fused_swiglu_fp8" : "fused_swiglu", st);
    kern<<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(a, g, u, d, r, e, o, a, g, u, d, o, p);
    return cudaGetLastError();
}

// A whole dense block in one launch.  Cooperative, so that all CTAs are resident together: a
// reverting tile waits for mixing tiles that other CTAs run.
template <int W, bool F8>
static cudaError_t launch_fused128_block_one(const FusedMaps& mix, const FusedMaps& rev, const CUtensorMap& r,
                                             const CUtensorMap& e, const FusedParams& p, int grid, cudaStream_t st) {
    using C = Fused128Cfg<W, A_BLOCK, F8>;
    auto kern = fused128_swiglu_kernel<W, A_BLOCK, F8>;
    static bool configured = false;
    if (!configured) {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (err != cudaSuccess) return err;
        configured = true;
    }
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(C::NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ProfileScope ps_(F8 ? "fused_swiglu_fp8" : "fused_swiglu", st);
    return cudaLaunchKernelEx(&cfg, kern, mix.a, mix.g, mix.u, mix.d, r, e, mix.o, rev.a, rev.g, rev.u, rev.d, rev.o, p);
}

cudaError_t launch_fused128_block(int W, bool f8, const FusedMaps& mix, const FusedMaps& rev, const CUtensorMap& r,
                                  const CUtensorMap& e, const FusedParams& p, int grid, cudaStream_t st) {
    if (W == 256) return f8 ? launch_fused128_block_one<256, true>(mix, rev, r, e, p, grid, st)
                            : launch_fused128_block_one<256, false>(mix, rev, r, e, p, grid, st);
    if (W == 128) return f8 ? launch_fused128_block_one<128, true>(mix, rev, r, e, p, grid, st)
                            : launch_fused128_block_one<128, false>(mix, rev, r, e, p, grid, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_fused128(int W, int a_mode, bool f8, const CUtensorMap& a, const CUtensorMap& g,
                            const CUtensorMap& u, const CUtensorMap& d, const CUtensorMap& r, const CUtensorMap& e,
                            const CUtensorMap& o, const FusedParams& p, int grid, cudaStream_t st) {
#define TM_F128(WW, AMM)                                                                                      \
    if (W == WW && a_mode == AMM)                                                                             \
        return f8 ? launch_fused128_one<WW, AMM, true>(a, g, u, d, r, e, o, p, grid, st)                      \
                  : launch_fused128_one<WW, AMM, false>(a, g, u, d, r, e, o, p, grid, st);
    TM_F128(256, A_TMA_MIX) TM_F128(256, A_TMA_3D) TM_F128(128, A_TMA_MIX) TM_F128(128, A_TMA_3D)
#undef TM_F128
    return cudaErrorInvalidValue;
}

bool fused_supported(int W, int a_mode) {
    return (W == 128 || W == 256) && (a_mode == A_TMA_MIX || a_mode == A_TMA_3D);
}

cudaError_t launch_fused(int W, int a_mode, const CUtensorMap& a, const CUtensorMap& g, const CUtensorMap& u,
                         const CUtensorMap& d, const FusedParams& p, int grid, cudaStream_t st) {
    if (W == 256 && a_mode == A_TMA_MIX) return launch_fused_one<256, A_TMA_MIX>(a, g, u, d, p, grid, st);
    if (W == 256 && a_mode == A_TMA_3D) return launch_fused_one<256, A_TMA_3D>(a, g, u, d, p, grid, st);
    if (W == 128 && a_mode == A_TMA_MIX) return launch_fused_one<128, A_TMA_MIX>(a, g, u, d, p, grid, st);
    if (W == 128 && a_mode == A_TMA_3D) return launch_fused_one<128, A_TMA_3D>(a, g, u, d, p, grid, st);
    return cudaErrorInvalidValue;
}

template <int BN, int AM, int EPI, bool PAIR, bool F8 = false>
static cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& s0,
                              const CUtensorMap& s1, const CUtensorMap& s2, const CUtensorMap& o, const GemmParams& p,
                              int grid, cudaStream_t st) {
    using C = GemmCfg<BN, AM, EPI, PAIR, F8>;
    auto kern = grouped_gemm_kernel<BN, AM, EPI, PAIR, F8>;
    static bool configured = false;   // attribute set once per instantiation (per process)
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    ProfileScope ps_(EPI == EPI_ROUTE                           ? "router"
                     : F8 ? "gemm_swiglu_fp8"
                     : (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_NORM) ? "gemm_swiglu"
                     : EPI == EPI_RESID                         ? "gemm_resid"
                     : (EPI == EPI_SLOT || EPI == EPI_SLOT_PERM) ? "gemm_slot"
                                                                 : "gemm_combine",
                     st);
    if (!PAIR) {
        kern<<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(a, b0, b1, s0, s1, s2, o, p);
        return cudaGetLastError();
    }
    // pair mode: clusters of two CTAs (grid even)
    if (grid % 2) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(C::NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, b0, b1, s0, s1, s2, o, p);
}

// Supported (BN, A mode, epilogue, pair mode) combinations.
//   GEMM1 (SwiGLU): A from x (3-D rows map, 4-D mixed map, or gather) or bucketed rows, BN 256 or 128
//   GEMM2:          A = hidden rows (2-D map), BN 256, 192 or 128
//   pair mode (CTA pairs, M = 256): the MoE GEMMs and the combine
#define TM_GEMM_TABLE(X)                                  \
    X(256, A_TMA_3D, EPI_SWIGLU, 0) X(128, A_TMA_3D, EPI_SWIGLU, 0) \
    X(256, A_TMA_MIX, EPI_SWIGLU, 0) X(128, A_TMA_MIX, EPI_SWIGLU, 0) \
    X(256, A_TMA_3D, EPI_SWIGLU_NORM, 0) X(128, A_TMA_3D, EPI_SWIGLU_NORM, 0) \
    X(256, A_TMA_MIX, EPI_SWIGLU_NORM, 0) X(128, A_TMA_MIX, EPI_SWIGLU_NORM, 0) \
    X(256, A_GATHER, EPI_SWIGLU, 0) X(128, A_GATHER, EPI_SWIGLU, 0) \
    X(256, A_TMA_2D, EPI_SWIGLU, 0) X(128, A_TMA_2D, EPI_SWIGLU, 0) \
    X(256, A_TMA_2D, EPI_RESID, 0) X(192, A_TMA_2D, EPI_RESID, 0) X(128, A_TMA_2D, EPI_RESID, 0) \
    X(256, A_TMA_2D, EPI_SLOT, 0) X(192, A_TMA_2D, EPI_SLOT, 0) X(128, A_TMA_2D, EPI_SLOT, 0) \
    X(256, A_TMA_2D, EPI_COMBINE, 0) X(192, A_TMA_2D, EPI_COMBINE, 0) X(128, A_TMA_2D, EPI_COMBINE, 0) \
    X(256, A_TMA_2D, EPI_SLOT_PERM, 0) X(192, A_TMA_2D, EPI_SLOT_PERM, 0) X(128, A_TMA_2D, EPI_SLOT_PERM, 0) \
    X(256, A_TMA_2D, EPI_SUM, 0) X(192, A_TMA_2D, EPI_SUM, 0) X(128, A_TMA_2D, EPI_SUM, 0) \
    X(64, A_TMA_3D, EPI_ROUTE, 0) X(64, A_TMA_MIX, EPI_ROUTE, 0) \
    X(256, A_TMA_2D, EPI_SUM, 1) X(192, A_TMA_2D, EPI_SUM, 1) X(128, A_TMA_2D, EPI_SUM, 1) \
    X(256, A_TMA_3D, EPI_SWIGLU, 1) X(128, A_TMA_3D, EPI_SWIGLU, 1) \
    X(256, A_TMA_MIX, EPI_SWIGLU, 1) X(128, A_TMA_MIX, EPI_SWIGLU, 1)

cudaError_t launch_grouped_gemm_src(int bn, int a_mode, int epi, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                    const CUtensorMap& tmB1, const CUtensorMap& tmS0, const CUtensorMap& tmS1,
                                    const CUtensorMap& tmS2, const GemmParams& p, int grid, cudaStream_t st,
                                    const CUtensorMap* tmO, bool pair) {
    // the SwiGLU, combine, plain-row and expert-row epilogues store through the output map
    if ((epi == EPI_SWIGLU || epi == EPI_SWIGLU_NORM || epi == EPI_SUM || epi == EPI_SLOT || epi == EPI_SLOT_PERM) &&
        !tmO)
        return cudaErrorInvalidValue;
    CUtensorMap none;
    memset(&none, 0, sizeof(none));
    const CUtensorMap& o = tmO ? *tmO : none;
#define X(BN, AM, EP, PR)                                               \
    if (bn == BN && a_mode == AM && epi == EP && pair == (PR != 0))     \
        return launch_one<BN, AM, EP, PR != 0>(tmA, tmB0, tmB1, tmS0, tmS1, tmS2, o, p, grid, st);
    TM_GEMM_TABLE(X)
#undef X
    return cudaErrorInvalidValue;
}

// GEMM1 + SwiGLU on E4M3 operands (kind::f8f6f4): A through a 2-D map (bucket-order rows) or a
// 3-D map ([B, banks, W] rows) of codes with 128-code boxes, B the E4M3 gate / up maps.
cudaError_t launch_grouped_gemm_f8(int bn, int a_mode, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                   const CUtensorMap& tmB1, const GemmParams& p, int grid, cudaStream_t st,
                                   const CUtensorMap* tmO) {
    if (!tmO || !p.w8_sgate || !p.w8_sup) return cudaErrorInvalidValue;
    CUtensorMap none;
    memset(&none, 0, sizeof(none));
    if (bn == 256 && a_mode == A_TMA_2D)
        return launch_one<256, A_TMA_2D, EPI_SWIGLU, false, true>(tmA, tmB0, tmB1, none, none, none, *tmO, p, grid, st);
    if (bn == 128 && a_mode == A_TMA_2D)
        return launch_one<128, A_TMA_2D, EPI_SWIGLU, false, true>(tmA, tmB0, tmB1, none, none, none, *tmO, p, grid, st);
    if (bn == 256 && a_mode == A_TMA_3D)
        return launch_one<256, A_TMA_3D, EPI_SWIGLU, false, true>(tmA, tmB0, tmB1, none, none, none, *tmO, p, grid, st);
    if (bn == 128 && a_mode == A_TMA_3D)
        return launch_one<128, A_TMA_3D, EPI_SWIGLU, false, true>(tmA, tmB0, tmB1, none, none, none, *tmO, p, grid, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_grouped_gemm(int bn, int a_mode, int epi, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                const CUtensorMap& tmB1, const GemmParams& p, int grid, cudaStream_t st,
                                const CUtensorMap* tmO, bool pair) {
    CUtensorMap none;
    memset(&none, 0, sizeof(none));
    return launch_grouped_gemm_src(bn, a_mode, epi, tmA, tmB0, tmB1, none, none, none, p, grid, st, tmO, pair);
}

}  // namespace tml
