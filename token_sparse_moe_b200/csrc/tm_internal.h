// tm_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "tm_gemm.cuh"
#include "tm_fused128.cuh"

namespace tml {

constexpr int kRouterChunk = 128;

// Counts the launch and, while profiling is on, brackets it with a CUDA event pair.
class ProfileScope {
   public:
    ProfileScope(const char* name, cudaStream_t st);
    ~ProfileScope();

   private:
    cudaStream_t st_;
    int ev_;
    const char* name_;
};
void note_cuda_error(const char* where, cudaError_t e);   // samples per router block: one bucketing chunk

// ---- tcgen05 grouped GEMM (bf16) ------------------------------------------------
// a_mode: AMode; epi: Epi; bn: tile width.  maps are passed by value into the kernel.
// with the EPI_SUM source maps: s0 residual, s1 inter-residual (row geometry of the output),
// s2 the sample-order expert rows [B, banks, k, W]
// tmO: the output map, required by EPI_SWIGLU (the hidden rows, 64-column x 32-row boxes) and
// EPI_SUM (y in its row geometry: 3-D rows or the 4-D Revert map, 32-row boxes)
// pair: CTA pairs (clusters of two, M = 256 per tile, grid even, weight maps with BN/2-row boxes;
// groups of equal rows, sched 0)
cudaError_t launch_grouped_gemm_src(int bn, int a_mode, int epi, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                    const CUtensorMap& tmB1, const CUtensorMap& tmS0, const CUtensorMap& tmS1,
                                    const CUtensorMap& tmS2, const GemmParams& p, int grid, cudaStream_t st,
                                    const CUtensorMap* tmO = nullptr, bool pair = false);
cudaError_t launch_grouped_gemm(int bn, int a_mode, int epi, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                const CUtensorMap& tmB1, const GemmParams& p, int grid, cudaStream_t st,
                                const CUtensorMap* tmO = nullptr, bool pair = false);

// GEMM1 + SwiGLU on E4M3 operands: A codes through a 2-D (bucket-order rows) or 3-D ([B, banks, W])
// map with 128-code boxes and 128-byte swizzle, tmB0 / tmB1 the E4M3 gate / up maps (BN/2-row boxes);
// p.w8_sgate / p.w8_sup the matrices' scales per group; the row factor by position (p.pos_scale) or
// by row (p.inv_rms)
cudaError_t launch_grouped_gemm_f8(int bn, int a_mode, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                   const CUtensorMap& tmB1, const GemmParams& p, int grid, cudaStream_t st,
                                   const CUtensorMap* tmO);

// ---- fused dense sub-layer (row width 128 / 256) --------------------------------
bool fused_supported(int W, int a_mode);
cudaError_t launch_fused(int W, int a_mode, const CUtensorMap& a, const CUtensorMap& g, const CUtensorMap& u,
                         const CUtensorMap& d, const FusedParams& p, int grid, cudaStream_t st);
// 128-wide hidden chunks (F % 128 == 0); gate/up maps with 128-row boxes; r / e: residual and
// inter-residual maps in the geometry of a (read when p.res_mode == RES_STREAM / p.has_extra);
// o: the output in the geometry of a with 32-row boxes
// f8: the FP8 serving path (E4M3 gate / up maps, scales in p.s_gate / p.s_up)
cudaError_t launch_fused128(int W, int a_mode, bool f8, const CUtensorMap& a, const CUtensorMap& g,
                            const CUtensorMap& u, const CUtensorMap& d, const CUtensorMap& r, const CUtensorMap& e,
                            const CUtensorMap& o, const FusedParams& p, int grid, cudaStream_t st);
// The maps of one sub-layer of a fused block: A (input rows), gate, up, down, output.
struct FusedMaps {
    CUtensorMap a, g, u, d, o;
};
// A whole dense block (both sub-layers of row width W) in one cooperative launch: mix in the Mix
// geometry (output through the Revert map into X_revert), rev in the row geometry over X_revert;
// r / e: the reverting sub-layer's residual (X) and inter-residual; p.dep: [ceil(B/128)] zeroed
// counters; grid <= the number of SMs.
cudaError_t launch_fused128_block(int W, bool f8, const FusedMaps& mix, const FusedMaps& rev, const CUtensorMap& r,
                                  const CUtensorMap& e, const FusedParams& p, int grid, cudaStream_t st);

// ---- CUDA-core kernels ------------------------------------------------------------
// dtype: 0 fp32, 1 bf16.
cudaError_t launch_rms(int dtype, const void* x, RowMap m, int B, float eps, float* inv_rms, cudaStream_t st);
cudaError_t launch_router(int dtype, const void* x, RowMap m, int B, float eps, const void* gain, const float* w_router,
                          int E, int k, float alpha, int32_t* idx, float* gate, float* inv_rms, float* logit_gap,
                          int32_t* counts, cudaStream_t st);
// tile_info (optional): one {group, first row position, rows, tile within the group} per 128-row tile
cudaError_t launch_offsets(const int32_t* counts_in, int32_t* chunk_prefix, int banks, int nchunks, int E,
                           int32_t* bucket_offsets, int32_t* tile_start, cudaStream_t st, int4* tile_info = nullptr);
// perm, inv_pos, gate_pos (optional, by bucket position): the combine-order row (bank * k + j) * B + b,
// the row's 1/rms (from inv_rms [B * banks]) and the choice's gate (from gate [B * banks * k])
// limit: entries of bucket_rows (positions at or past it are reported as a bounds error and not
// written); < 0: B * banks * k
cudaError_t launch_scatter(const int32_t* idx, const int32_t* chunk_prefix, const int32_t* bucket_offsets, int B,
                           int banks, int E, int k, int32_t* bucket_rows, int32_t* slot_of, cudaStream_t st,
                           int32_t* perm = nullptr, const float* inv_rms = nullptr, const float* gate = nullptr,
                           float* inv_pos = nullptr, float* gate_pos = nullptr, int limit = -1);
// bounded-wait self-test (one CTA): res [4] device memory or NULL
cudaError_t launch_wait_selftest(unsigned long long* res, cudaStream_t st);
// tensor-core router weights: [banks][64][W] bf16, rows e / E+e / 2E+e = hi / mid / lo of w * gain
cudaError_t launch_router_split(int dtype, const float* w_router, const void* gain, int banks, int E, int W,
                                void* out, cudaStream_t st);
// MoEPermute data copy: each source row to the k bucketed row positions of its choices (slot_of
// [B * banks * k], k <= 8), out [routed, W] (see scatter_rows_kernel)
cudaError_t launch_scatter_rows(int dtype, const void* x, RowMap m, int B, int k, const int32_t* slot_of, size_t routed,
                                void* out, cudaStream_t st);
// FP8 E4M3 (bf16 inputs): the codes of `groups` weight matrices of n elements (rows of `cols`)
// with one scale per matrix (gain optional, folded first), and the per-row activation codes
// [B * banks, W] with rowscale = 2^e / rms(x), 2^e the row's power-of-two E4M3 scale
cudaError_t launch_quant_matrices(const void* w, const void* gain, int groups, size_t n, int cols, uint8_t* q,
                                  float* scale, cudaStream_t st);
// slot_of (optional, [B * banks, k]): the codes and row factors also to the rows' k bucket positions
// (qpos [routed, W], scale_pos [routed]); q / rowscale may then be NULL
cudaError_t launch_quant_act_rows(const void* x, RowMap m, int B, float eps, uint8_t* q, float* rowscale,
                                  cudaStream_t st, const int32_t* slot_of = nullptr, int k = 0, size_t routed = 0,
                                  uint8_t* qpos = nullptr, float* scale_pos = nullptr);
// Token Parallel: exchange buffer [P][B][Tp][Dp] <-> local [B][Tp][P][Dp] (cols_shard) or [B][P][Tp][Dp]
cudaError_t launch_tp_layout(const void* src, void* dst, int P, int B, int Tp, int Dp, int esz, bool cols_shard,
                             bool to_exchange, cudaStream_t st);
cudaError_t launch_permute(int dtype, const void* src, void* dst, int B, int T, int D, int H, bool to_mixed,
                           cudaStream_t st);
cudaError_t launch_fold_gain(int dtype, const void* w, const void* gain, void* out, size_t rows, int width,
                             cudaStream_t st);
// scoring head: logits [B] fp32 = mean over tokens of X [B,T,D] projected on w [D]
cudaError_t launch_head(int dtype, const void* X, const void* w, int B, int T, int D, float* logits, cudaStream_t st);
cudaError_t launch_tokenize(int dtype, const void* groups, const void* w_group, const void* w_global, int dg, int B,
                            int T, int D, void* X, cudaStream_t st);

// ---- dense sub-layer backward (bf16; tm_backward.cu) ------------------------------
// row pass: inv_rms [banks][B], xh = x * inv_rms and a copy of dy, both bank-major [banks][B][W]
cudaError_t launch_bwd_rows(const void* x, const void* dy, RowMap m, int B, float eps, void* xh, void* dyb,
                            float* inv_rms, cudaStream_t st);
// out[g][c][r] = in[g][r][c] (r < R, c < C), zero for R <= r < Rp; element strides per group / row;
// C, Rp, strides multiples of 8 elements, bases 16-byte aligned (else cudaErrorInvalidValue)
cudaError_t launch_transpose(const void* in, size_t in_gs, int in_ld, int R, int C, void* out, size_t out_gs,
                             int out_ld, int Rp, int groups, cudaStream_t st);
// SwiGLU derivative over [rows, F]: dGU [rows, 2F] = (dg | du), Hd [rows, F] = silu(g) * u
cudaError_t launch_swiglu_bwd(const void* Gp, const void* Up, const void* dH, size_t rows, int F, void* dGU, void* Hd,
                              cudaStream_t st);
// RMSNorm derivative: dx = inv_rms (dn - xh mean(dn xh)) + add0 + add1 + add2 through the row map
cudaError_t launch_rms_bwd(const void* x, const void* dN, const float* inv_rms, const void* add0, const void* add1,
                           const void* add2, RowMap m, int B, void* dx, cudaStream_t st);

// fp32 CUDA-core grouped GEMM with the same tile space and epilogues as the tcgen05 one.
// A is x (gathered through amap) when epi == EPI_SWIGLU, else hidden rows [positions, K].
struct SimtGemmArgs {
    GemmParams p;            // pointer fields reinterpret bf16 as float
    const float* a;          // x or hidden
    const float* w0;         // gate / down
    const float* w1;         // up (SwiGLU)
};
cudaError_t launch_simt_gemm(int epi, const SimtGemmArgs& a, int max_tiles, cudaStream_t st);

}  // namespace tml
