// tm_gemm.cu -- instantiations and launcher of the tcgen05 grouped GEMM.
#include "tm_internal.h"

namespace tml {

template <int BN, int AM, int EPI>
static cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const GemmParams& p,
                              int grid, cudaStream_t st) {
    using C = GemmCfg<BN, AM>;
    auto kern = grouped_gemm_kernel<BN, AM, EPI>;
    static bool configured = false;   // attribute set once per instantiation (per process)
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    ProfileScope ps_(EPI == EPI_SWIGLU ? "gemm_swiglu" : EPI == EPI_RESID ? "gemm_resid" : EPI == EPI_SLOT ? "gemm_slot" : "gemm_combine", st);
    kern<<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(a, b0, b1, p);
    return cudaGetLastError();
}

// Supported (BN, A mode, epilogue) combinations.
//   GEMM1 (SwiGLU): A from x (3-D rows map, 4-D mixed map, or gather), BN 256 or 128
//   GEMM2:          A = hidden rows (2-D map), BN 256, 192 or 128
#define TM_GEMM_TABLE(X)                                  \
    X(256, A_TMA_3D, EPI_SWIGLU) X(128, A_TMA_3D, EPI_SWIGLU) \
    X(256, A_TMA_MIX, EPI_SWIGLU) X(128, A_TMA_MIX, EPI_SWIGLU) \
    X(256, A_GATHER, EPI_SWIGLU) X(128, A_GATHER, EPI_SWIGLU) \
    X(256, A_TMA_2D, EPI_RESID) X(192, A_TMA_2D, EPI_RESID) X(128, A_TMA_2D, EPI_RESID) \
    X(256, A_TMA_2D, EPI_SLOT) X(192, A_TMA_2D, EPI_SLOT) X(128, A_TMA_2D, EPI_SLOT) \
    X(256, A_TMA_2D, EPI_COMBINE) X(192, A_TMA_2D, EPI_COMBINE) X(128, A_TMA_2D, EPI_COMBINE)

bool grouped_gemm_supported(int bn, int a_mode, int epi) {
#define X(BN, AM, EP) if (bn == BN && a_mode == AM && epi == EP) return true;
    TM_GEMM_TABLE(X)
#undef X
    return false;
}

int grouped_gemm_smem(int bn, int a_mode) {
    if (a_mode == A_GATHER) return bn == 256 ? GemmCfg<256, A_GATHER>::SMEM_BYTES : GemmCfg<128, A_GATHER>::SMEM_BYTES;
    switch (bn) {
        case 256: return GemmCfg<256, A_TMA_2D>::SMEM_BYTES;
        case 192: return GemmCfg<192, A_TMA_2D>::SMEM_BYTES;
        default: return GemmCfg<128, A_TMA_2D>::SMEM_BYTES;
    }
}

cudaError_t launch_grouped_gemm(int bn, int a_mode, int epi, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                const CUtensorMap& tmB1, const GemmParams& p, int grid, cudaStream_t st) {
#define X(BN, AM, EP) \
    if (bn == BN && a_mode == AM && epi == EP) return launch_one<BN, AM, EP>(tmA, tmB0, tmB1, p, grid, st);
    TM_GEMM_TABLE(X)
#undef X
    return cudaErrorInvalidValue;
}

}  // namespace tml
