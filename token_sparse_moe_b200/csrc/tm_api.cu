// tm_api.cu -- host side of the C ABI declared in include/tm.h: validation, workspace
// carving, TMA tensor maps and the launch sequence of every call.  Nothing here
// allocates device memory or synchronises (except tm_get_device_error).
#include <math.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include "tm.h"
#include "tm_internal.h"

namespace tml {
namespace {

// ------------------------------------------------------------------ small utilities
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// aligned to one element of the shape's dtype (the element-wise kernels' only requirement)
inline bool al_elem(const void* p, int dtype) {
    return (reinterpret_cast<uintptr_t>(p) & (dtype == TM_BF16 ? 1u : 3u)) == 0;
}
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Carve {
    uint8_t* base;
    size_t off = 0;
    template <class T>
    T* take(size_t n) {
        off = align256(off);
        T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
        off += n * sizeof(T);
        return p;
    }
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 tensor map; dims/box innermost first, strides in bytes for dims 1..r-1.  The box's
// inner extent always equals the swizzle span (128 B with SWIZZLE_128B, 32 B with SWIZZLE_32B).
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// [rows, cols] row-major bf16 matrix, box = 64 columns x box_rows rows
bool map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    uint64_t dims[2] = {cols, rows};
    uint64_t strides[1] = {cols * 2};
    uint32_t box[2] = {64, box_rows};
    return make_map(m, base, 2, dims, strides, box);
}

// E4M3 codes (1-byte elements): dims / box innermost first in elements, strides in bytes;
// 128-byte swizzle with a 128-element inner box.
bool make_map_u8(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                 const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 148;
    }
    return cache[dev];
}

tm_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TM_OK;
    note_cuda_error("launch", e);
    return TM_ERR_CUDA;
}

// ------------------------------------------------------------------ geometry and validation
struct Geo {
    int B, banks, W, dtype;
    size_t esz;
    float eps;
    RowMap map;
};

tm_status check_shape(const tm_shape* s) {
    if (!s) return TM_ERR_INVALID_ARG;
    if (s->B <= 0 || s->T <= 0 || s->D <= 0 || s->H <= 0 || s->D % s->H != 0) return TM_ERR_INVALID_ARG;
    if (s->dtype != TM_F32 && s->dtype != TM_BF16) return TM_ERR_INVALID_ARG;
    if (!(s->eps >= 0.f) || !isfinite(s->eps)) return TM_ERR_INVALID_ARG;
    // a sample's T * D elements are indexed with 32-bit integers inside the kernels
    if ((long long)s->T * s->D > INT32_MAX) return TM_ERR_UNSUPPORTED;
    return TM_OK;
}

// Geometry of a sub-layer with `banks` banks of width `width` seen through `layout`.
tm_status make_geo(const tm_shape* s, int layout, int banks, int width, Geo* g) {
    tm_status st = check_shape(s);
    if (st != TM_OK) return st;
    const int dh = s->D / s->H;
    if (layout == TM_LAYOUT_MIXED) {
        if (banks != s->H || width != s->T * dh) return TM_ERR_INVALID_ARG;
    } else if (layout == TM_LAYOUT_ROWS) {
        if (banks <= 0 || width <= 0) return TM_ERR_INVALID_ARG;
    } else {
        return TM_ERR_INVALID_ARG;
    }
    // row counts (B * banks, times k <= 8 for the routed rows) are 32-bit tensor-map coordinates
    if ((long long)s->B * banks > (1LL << 28)) return TM_ERR_UNSUPPORTED;
    const int V = s->dtype == TM_BF16 ? 8 : 4;   // elements per 16-byte vector
    if (width % V != 0) return TM_ERR_UNSUPPORTED;
    if (layout == TM_LAYOUT_MIXED && dh % V != 0) return TM_ERR_UNSUPPORTED;
    g->B = s->B;
    g->banks = banks;
    g->W = width;
    g->dtype = s->dtype;
    g->esz = s->dtype == TM_BF16 ? 2 : 4;
    g->eps = s->eps;
    g->map = RowMap{layout == TM_LAYOUT_MIXED ? 1 : 0, banks, width, s->T, s->D, dh};
    return TM_OK;
}

// K and N granularity of the GEMMs: 64 for the tcgen05 path (64-wide K slabs), 32 for fp32.
int gran(const Geo& g) { return g.dtype == TM_BF16 ? 64 : 32; }

tm_status check_dense(const Geo& g, const tm_swiglu_w* w) {
    if (!w || w->banks != g.banks || w->width != g.W || w->hidden <= 0) return TM_ERR_INVALID_ARG;
    if (!w->w_gate || !w->w_up || !w->w_down) return TM_ERR_INVALID_ARG;
    if (!al16(w->w_gate) || !al16(w->w_up) || !al16(w->w_down)) return TM_ERR_INVALID_ARG;
    if (w->hidden % gran(g) || g.W % gran(g)) return TM_ERR_UNSUPPORTED;
    return TM_OK;
}

tm_status check_moe(const Geo& g, const tm_moe_w* w) {
    if (!w || w->banks != g.banks || w->width != g.W) return TM_ERR_INVALID_ARG;
    if (w->E < 1 || w->k < 1 || w->k > w->E || w->hidden_e <= 0 || w->hidden_s < 0) return TM_ERR_INVALID_ARG;
    if (!isfinite(w->alpha)) return TM_ERR_INVALID_ARG;
    if (w->E > 32 || w->k > 8) return TM_ERR_UNSUPPORTED;
    if ((size_t)w->banks * w->E > 4096) return TM_ERR_UNSUPPORTED;
    // router weights (expert count rounded up to a power of two, rows padded by 4) and each
    // warp's two staging buffers of rows, all in shared memory
    {
        const size_t ep = w->E <= 4 ? 4 : w->E <= 8 ? 8 : w->E <= 16 ? 16 : 32;
        const size_t group = 32 / ep > 4 ? 32 / ep : 4;
        if (ep * (w->width + 4) * 4 + 16 * group * (size_t)w->width * g.esz > 220 * 1024) return TM_ERR_UNSUPPORTED;
    }
    if (!w->w_router || !w->we_gate || !w->we_up || !w->we_down) return TM_ERR_INVALID_ARG;
    if (!al16(w->w_router) || !al16(w->we_gate) || !al16(w->we_up) || !al16(w->we_down)) return TM_ERR_INVALID_ARG;
    if (w->hidden_s > 0) {
        if (!w->ws_gate || !w->ws_up || !w->ws_down) return TM_ERR_INVALID_ARG;
        if (!al16(w->ws_gate) || !al16(w->ws_up) || !al16(w->ws_down)) return TM_ERR_INVALID_ARG;
        if (w->hidden_s % gran(g)) return TM_ERR_UNSUPPORTED;
    }
    if (w->hidden_e % gran(g) || g.W % gran(g)) return TM_ERR_UNSUPPORTED;
    return TM_OK;
}

// ------------------------------------------------------------------ GEMM helpers
int pick_bn_swiglu(int F) { return F % 128 == 0 ? 256 : 128; }
int pick_bn_out(int W) { return W % 256 == 0 ? 256 : (W % 192 == 0 ? 192 : 128); }

// The A operand of GEMM1 read straight from x: a 3-D map over [B, banks, W] rows, or the 4-D Mix
// map (j16, q, t, b) over the token tensor, q = the 16-column piece of a token (head h owns
// q = h*dh/16 .. h*dh/16 + dh/16 - 1), when the head width is a multiple of 16.
int gemm1_amode(const Geo& g) {
    if (g.map.layout == 0) return A_TMA_3D;
    return (g.map.dh % 16 == 0) ? A_TMA_MIX : A_GATHER;
}
// bytes of the split router weights when the tensor-core router applies (bf16 rows read through a
// 3-D or mixed tensor map, E <= kRouteMaxE), else 0
size_t route_split_bytes(const Geo& g, const tm_moe_w* w) {
    const int am = gemm1_amode(g);
    if (g.dtype != TM_BF16 || (am != A_TMA_3D && am != A_TMA_MIX) || w->E > kRouteMaxE) return 0;
    return (size_t)g.banks * 64 * g.W * 2;
}

bool gemm1_amap(const Geo& g, const void* x, int amode, CUtensorMap* m, uint32_t box_rows = 128) {
    if (amode == A_TMA_3D) {
        uint64_t dims[3] = {(uint64_t)g.W, (uint64_t)g.banks, (uint64_t)g.B};
        uint64_t strides[2] = {(uint64_t)g.W * 2, (uint64_t)g.banks * g.W * 2};
        uint32_t box[3] = {64, 1, box_rows};
        return make_map(m, x, 3, dims, strides, box);
    }
    if (amode == A_TMA_MIX) {
        const RowMap& r = g.map;
        uint64_t dims[4] = {16, (uint64_t)r.D / 16, (uint64_t)r.T, (uint64_t)g.B};
        uint64_t strides[3] = {32, (uint64_t)r.D * 2, (uint64_t)r.T * r.D * 2};
        uint32_t box[4] = {16, 1, 1, box_rows};
        return make_map(m, x, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_32B);
    }
    memset(m, 0, sizeof(*m));
    return true;
}

GemmParams base_params(const Geo& g) {
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.banks = g.banks;
    p.rows = g.B;
    p.groups = g.banks;
    p.E = 1;
    p.amap = g.map;
    p.omap = g.map;
    p.pos_limit = g.B * g.banks;
    return p;
}

// Banks per chunk of the sched-0 tile order (a power of two): as many as keep one row block's working
// set of the chunk -- each bank's weight tiles (w_bytes) and the rows it streams for one row block
// (row_bytes) -- within 24 MB of the 126 MB L2.  A bank's weights are then read from DRAM about once
// per chunk instead of once per row block: with all 48 banks of the large MoE stack in one cycle
// (113 MB of shared-expert gate / up weights) the shared GEMM1 read 12 GB for 1.3 GB of data.
int bank_chunk(double w_bytes, double row_bytes) {
    const double per = w_bytes + row_bytes;
    int c = 1;
    while (c < (1 << 20) && 2.0 * c * per <= 24.0 * (1 << 20)) c *= 2;
    return c;
}

int dense_grid(const GemmParams& p) {
    const long tiles = (long)p.groups * ((p.rows + 127) / 128) * p.n_tiles;
    return (int)(tiles < num_sms() ? tiles : num_sms());
}

bool env_is(const char* name, char v);

// CTA pairs (M = 256 per tile, each SM streaming half of the weight rows) for the combine of bf16
// rows and the MoE shared expert's GEMM1: the combine (the shared expert's down projection beside
// its k + 1 source slabs) measured 7-10% faster so on the MoE stacks, the shared GEMM1 of the large
// stack up to 20%; the routed GEMM2, whose epilogue bounds it, was slower (a pair waits for the
// slower of its two epilogues).  TM_PAIR=0 in the environment keeps one CTA per tile: the tests use
// it to show that both forms give the same bits.
bool use_pair(const Geo& g, int amode) {
    return g.dtype == TM_BF16 && amode != A_GATHER && !env_is("TM_PAIR", '0');
}
// grid of a pair-mode launch: two CTAs per cluster, at most one cluster per two SMs
int pair_grid(long pair_tiles) {
    const long c = pair_tiles < num_sms() / 2 ? pair_tiles : num_sms() / 2;
    return (int)(2 * (c > 0 ? c : 1));
}
// grid of a launch over dense groups (sched 0) in either form
int sched0_grid(const GemmParams& p, bool pair) {
    if (!pair) return dense_grid(p);
    return pair_grid((long)p.groups * ((p.rows + 255) / 256) * p.n_tiles);
}

// SwiGLU GEMM1 over x (dense groups = banks, rows = B): hidden [banks*B, F].  inv_rms NULL (bf16 rows
// read through a 3-D or Mix map): the kernel takes the row statistics itself (EPI_SWIGLU_NORM).
tm_status gemm1_dense(const Geo& g, const void* x, const void* wg, const void* wu, int F, const float* inv_rms,
                      void* hidden, cudaStream_t st) {
    GemmParams p = base_params(g);
    p.sched = 0;
    p.K = g.W;
    p.N = 2 * F;
    p.inv_rms = inv_rms;
    p.out = (__nv_bfloat16*)hidden;
    p.out_ld = F;
    p.out_elems = (size_t)g.banks * g.B * F;
    p.a_ptr = (const __nv_bfloat16*)x;
    if (g.dtype == TM_F32) {
        p.n_tiles = F / 32;
        SimtGemmArgs a{p, (const float*)x, (const float*)wg, (const float*)wu};
        return cuda_status(launch_simt_gemm(EPI_SWIGLU, a, p.groups * ((p.rows + 127) / 128) * p.n_tiles, st));
    }
    const int bn = pick_bn_swiglu(F);
    p.n_tiles = p.N / bn;
    p.bank_chunk = bank_chunk(2.0 * 2 * F * g.W, 128.0 * 2 * (g.W + F));
    const int am = gemm1_amode(g);
    const int epi = inv_rms ? EPI_SWIGLU : EPI_SWIGLU_NORM;
    if (!inv_rms && am != A_TMA_3D && am != A_TMA_MIX) return TM_ERR_UNSUPPORTED;
    p.r_eps = g.eps;
    CUtensorMap ma, mg, mu, mo;
    if (!gemm1_amap(g, x, am, &ma)) return TM_ERR_CUDA;
    if (!map_2d(&mg, wg, (uint64_t)g.banks * F, g.W, bn / 2) || !map_2d(&mu, wu, (uint64_t)g.banks * F, g.W, bn / 2) ||
        !map_2d(&mo, hidden, (uint64_t)g.banks * g.B, F, 32))
        return TM_ERR_CUDA;
    // CTA pairs when the row factors come in (the MoE shared expert): up to 20% faster on the large
    // stack.  With the row statistics in the kernel the pair form has to relay each stage's arrival
    // to the peer's statistics warps, which measured 1.85x slower: the dense path keeps one CTA.
    const bool pair = use_pair(g, am) && epi == EPI_SWIGLU;
    return cuda_status(launch_grouped_gemm(bn, am, epi, ma, mg, mu, p, sched0_grid(p, pair), st, &mo, pair));
}

// GEMM2 over dense hidden rows [banks*B, F] with the residual / combine epilogue into y (omap).
tm_status gemm2_dense(const Geo& g, const void* hidden, const void* wd, int F, int epi, const void* resid,
                      const void* extra, void* y, const float* gate, const int* slot_of, const void* slots, int k,
                      cudaStream_t st) {
    GemmParams p = base_params(g);
    p.sched = 0;
    p.K = F;
    p.N = g.W;
    p.out = (__nv_bfloat16*)y;
    p.out_elems = (size_t)g.B * g.banks * g.W;
    p.resid = (const __nv_bfloat16*)resid;
    p.extra = (const __nv_bfloat16*)extra;
    p.gate = gate;
    p.slot_of = slot_of;
    p.slots = (const __nv_bfloat16*)slots;
    p.k = k;
    if (epi == EPI_COMBINE) p.pos_limit = g.B * g.banks * k;   // slot rows
    if (g.dtype == TM_F32) {
        p.n_tiles = g.W / 32;
        SimtGemmArgs a{p, (const float*)hidden, (const float*)wd, nullptr};
        return cuda_status(launch_simt_gemm(epi, a, p.groups * ((p.rows + 127) / 128) * p.n_tiles, st));
    }
    const int bn = pick_bn_out(g.W);
    p.n_tiles = g.W / bn;
    p.bank_chunk = bank_chunk(2.0 * F * g.W, 128.0 * 2 * (F + (3 + k) * g.W));
    CUtensorMap ma, mb;
    if (!map_2d(&ma, hidden, (uint64_t)g.banks * g.B, F, 128) || !map_2d(&mb, wd, (uint64_t)g.banks * g.W, F, bn))
        return TM_ERR_CUDA;
    return cuda_status(launch_grouped_gemm(bn, A_TMA_2D, epi, ma, mb, mb, p, dense_grid(p), st));
}

// ------------------------------------------------------------------ fused dense sub-layer
// One launch for row widths 128 / 256: statistics, GEMM1, SwiGLU, GEMM2, residual.  Hidden widths
// that are multiples of 128 take the 128-wide-chunk kernel (tm_fused128.cuh), the others (F % 128
// == 64) the 64-wide-chunk kernel (tm_fused.cuh).
tm_status fused_dense(const Geo& g, const void* x, const void* wg, const void* wu, const void* wd, int F,
                      const void* resid, const void* extra, void* y, cudaStream_t st) {
    const int am = gemm1_amode(g);
    const bool wide = F % 128 == 0 && (uintptr_t)y % 32 == 0;
    const uint32_t gu_box = wide ? 128 : 64;
    CUtensorMap ma, mg, mu, md;
    if (!gemm1_amap(g, x, am, &ma)) return TM_ERR_CUDA;
    if (!map_2d(&mg, wg, (uint64_t)g.banks * F, g.W, gu_box) || !map_2d(&mu, wu, (uint64_t)g.banks * F, g.W, gu_box) ||
        !map_2d(&md, wd, (uint64_t)g.banks * g.W, F, g.W))
        return TM_ERR_CUDA;
    FusedParams p;
    memset(&p, 0, sizeof(p));
    p.banks = g.banks;
    p.rows = g.B;
    p.F = F;
    p.amap = g.map;
    p.eps = g.eps;
    p.out = (__nv_bfloat16*)y;
    p.resid = (const __nv_bfloat16*)resid;
    p.extra = (const __nv_bfloat16*)extra;
    p.omap = g.map;
    p.out_elems = (size_t)g.B * g.banks * g.W;
    const long tiles = (long)g.banks * ((g.B + 127) / 128);
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    if (wide) {
        // residual: the A tile itself when it is the sub-layer input (same tensor, same row map),
        // else streamed with the A geometry; the inter-residual likewise
        CUtensorMap mr, me;
        memset(&mr, 0, sizeof(mr));
        memset(&me, 0, sizeof(me));
        p.res_mode = resid == nullptr ? RES_NONE : resid == x ? RES_FROM_A : RES_STREAM;
        p.has_extra = extra != nullptr;
        if (p.res_mode == RES_STREAM && !gemm1_amap(g, resid, am, &mr)) return TM_ERR_CUDA;
        if (p.has_extra && !gemm1_amap(g, extra, am, &me)) return TM_ERR_CUDA;
        // output: the same row geometry, 32-row boxes (one per epilogue warp)
        CUtensorMap mo;
        if (!gemm1_amap(g, y, am, &mo, 32)) return TM_ERR_CUDA;
        return cuda_status(launch_fused128(g.W, am, false, ma, mg, mu, md, mr, me, mo, p, grid, st));
    }
    return cuda_status(launch_fused(g.W, am, ma, mg, mu, md, p, grid, st));
}

// ------------------------------------------------------------------ dense sub-layer
struct DenseWs {
    float* inv_rms;
    void* hidden;
    void* wg;
    void* wu;
};
DenseWs carve_dense(Carve& c, const Geo& g, int F, bool gain) {
    DenseWs w;
    w.inv_rms = c.take<float>((size_t)g.B * g.banks);
    w.hidden = c.take<uint8_t>((size_t)g.banks * g.B * F * g.esz);
    w.wg = gain ? c.take<uint8_t>((size_t)g.banks * F * g.W * g.esz) : nullptr;
    w.wu = gain ? c.take<uint8_t>((size_t)g.banks * F * g.W * g.esz) : nullptr;
    return w;
}

tm_status combine_sum(const Geo& g, const void* hidden_s, const void* wd, int Fs, const void* resid, const void* extra,
                      void* y, const void* slots, int k, cudaStream_t st);

tm_status run_dense(const Geo& g, const void* x, const void* resid, const void* extra, const void* gain,
                    const tm_swiglu_w* w, void* y, void* ws, size_t wsb, cudaStream_t st) {
    Carve c{(uint8_t*)ws};
    DenseWs d = carve_dense(c, g, w->hidden, gain != nullptr);
    if (!ws || wsb < c.off || !al16(ws)) return TM_ERR_WORKSPACE;
    const void* wg = w->w_gate;
    const void* wu = w->w_up;
    tm_status s;
    if (gain) {
        const size_t rows = (size_t)g.banks * w->hidden;
        if ((s = cuda_status(launch_fold_gain(g.dtype, wg, gain, d.wg, rows, g.W, st))) != TM_OK) return s;
        if ((s = cuda_status(launch_fold_gain(g.dtype, wu, gain, d.wu, rows, g.W, st))) != TM_OK) return s;
        wg = d.wg;
        wu = d.wu;
    }
    if (g.dtype == TM_BF16 && fused_supported(g.W, gemm1_amode(g)) && w->hidden % 64 == 0)
        return fused_dense(g, x, wg, wu, w->w_down, w->hidden, resid, extra, y, st);
    // bf16 rows read through a tensor map: GEMM1 takes the row statistics itself; otherwise they come
    // from rms_kernel first
    const int am = gemm1_amode(g);
    const bool stats_in_gemm = g.dtype == TM_BF16 && (am == A_TMA_3D || am == A_TMA_MIX);
    if (!stats_in_gemm && (s = cuda_status(launch_rms(g.dtype, x, g.map, g.B, g.eps, d.inv_rms, st))) != TM_OK) return s;
    if ((s = gemm1_dense(g, x, wg, wu, w->hidden, stats_in_gemm ? nullptr : d.inv_rms, d.hidden, st)) != TM_OK) return s;
    // bf16 with a tensor-map row geometry: GEMM2 with the residual and inter-residual entering the
    // accumulator through identity MMAs and bulk tensor stores out (the combine kernel, no expert rows)
    if (g.dtype == TM_BF16 && (am == A_TMA_3D || am == A_TMA_MIX))
        return combine_sum(g, d.hidden, w->w_down, w->hidden, resid, extra, y, nullptr, 0, st);
    return gemm2_dense(g, d.hidden, w->w_down, w->hidden, EPI_RESID, resid, extra, y, nullptr, nullptr, nullptr, 0, st);
}

// ------------------------------------------------------------------ MoE sub-layer
struct MoeWs {
    float* inv_rms;
    int32_t *idx, *slot_of, *bucket_rows, *offsets, *tile_start, *counts, *perm;
    int4* tile_info;
    float *gate, *inv_pos, *gate_pos;
    void *hidden_r, *slots, *hidden_s;
    void *weg, *weu, *wsg, *wsu;
    void* wsplit;
};
MoeWs carve_moe(Carve& c, const Geo& g, const tm_moe_w* w, bool gain) {
    MoeWs m;
    const size_t rows = (size_t)g.B * g.banks;
    const size_t routed = rows * w->k;
    const int nchunks = (g.B + kRouterChunk - 1) / kRouterChunk;
    const size_t G = (size_t)g.banks * w->E;
    m.inv_rms = c.take<float>(rows);
    m.idx = c.take<int32_t>(routed);
    m.gate = c.take<float>(routed);
    m.slot_of = c.take<int32_t>(routed);
    m.bucket_rows = c.take<int32_t>(routed);
    m.perm = c.take<int32_t>(routed);
    m.inv_pos = c.take<float>(routed);
    m.gate_pos = c.take<float>(routed);
    m.offsets = c.take<int32_t>(G + 1);
    m.tile_start = c.take<int32_t>(G + 1);
    m.tile_info = c.take<int4>(routed / 128 + G);   // at most this many 128-row tiles
    m.counts = c.take<int32_t>((size_t)g.banks * nchunks * w->E);
    m.hidden_r = c.take<uint8_t>(routed * w->hidden_e * g.esz);
    m.slots = c.take<uint8_t>(routed * g.W * g.esz);
    m.hidden_s = w->hidden_s > 0 ? c.take<uint8_t>(rows * w->hidden_s * g.esz) : nullptr;
    const size_t split = route_split_bytes(g, w);
    m.wsplit = split ? c.take<uint8_t>(split) : nullptr;
    m.weg = gain ? c.take<uint8_t>(G * w->hidden_e * g.W * g.esz) : nullptr;
    m.weu = gain ? c.take<uint8_t>(G * w->hidden_e * g.W * g.esz) : nullptr;
    m.wsg = gain && w->hidden_s ? c.take<uint8_t>((size_t)g.banks * w->hidden_s * g.W * g.esz) : nullptr;
    m.wsu = gain && w->hidden_s ? c.take<uint8_t>((size_t)g.banks * w->hidden_s * g.W * g.esz) : nullptr;
    return m;
}

struct RouteOut {
    int32_t *idx, *offsets, *tile_start, *bucket_rows, *slot_of, *counts;
    float *gate, *inv_rms;
    int32_t* perm = nullptr;   // optional: sample-order row of each bucket position
    void* wsplit = nullptr;    // optional: [banks][64][W] bf16 split router weights (tensor-core router)
    int4* tile_info = nullptr; // optional: per 128-row tile descriptors of the buckets
    float* inv_pos = nullptr;  // optional: 1/rms of each bucket position's row
    float* gate_pos = nullptr; // optional: gate of each bucket position's choice
    float* gap = nullptr;      // optional: logit gap z_(k) - z_(k+1) of each row [B * banks]
};


tm_status run_route(const Geo& g, const void* x, const void* gain, const tm_moe_w* w, const RouteOut& r,
                    cudaStream_t st) {
    tm_status s;
    const int nchunks = (g.B + kRouterChunk - 1) / kRouterChunk;
    if (r.wsplit && route_split_bytes(g, w) > 0) {
        // router on the tensor core: split weights, then one grouped-GEMM launch (N = 64) whose
        // epilogue writes top-k, gates, 1/rms and the per-chunk expert counts (zeroed first)
        const int am = gemm1_amode(g);
        if ((s = cuda_status(cudaMemsetAsync(r.counts, 0, (size_t)g.banks * nchunks * w->E * sizeof(int32_t), st))) !=
            TM_OK)
            return s;
        if ((s = cuda_status(launch_router_split(g.dtype, w->w_router, gain, g.banks, w->E, g.W, r.wsplit, st))) != TM_OK)
            return s;
        GemmParams p = base_params(g);
        p.sched = 0;
        p.K = g.W;
        p.N = 64;
        p.n_tiles = 1;
        p.E = w->E;
        p.k = w->k;
        p.r_idx = r.idx;
        p.r_gate = r.gate;
        p.r_inv_rms = r.inv_rms;
        p.r_gap = r.gap;
        p.r_counts = r.counts;
        p.r_nchunks = nchunks;
        p.r_alpha = w->alpha;
        p.r_eps = g.eps;
        CUtensorMap ma, mb;
        if (!gemm1_amap(g, x, am, &ma) || !map_2d(&mb, r.wsplit, (uint64_t)g.banks * 64, g.W, 64)) return TM_ERR_CUDA;
        if ((s = cuda_status(launch_grouped_gemm(64, am, EPI_ROUTE, ma, mb, mb, p, dense_grid(p), st))) != TM_OK) return s;
    } else if ((s = cuda_status(launch_router(g.dtype, x, g.map, g.B, g.eps, gain, w->w_router, w->E, w->k, w->alpha,
                                              r.idx, r.gate, r.inv_rms, r.gap, r.counts, st))) != TM_OK) {
        return s;
    }
    if ((s = cuda_status(launch_offsets(r.counts, r.counts, g.banks, nchunks, w->E, r.offsets, r.tile_start, st,
                                        r.tile_info))) != TM_OK)
        return s;
    return cuda_status(launch_scatter(r.idx, r.counts, r.offsets, g.B, g.banks, w->E, w->k, r.bucket_rows, r.slot_of, st,
                                      r.perm, r.inv_rms, r.gate, r.inv_pos, r.gate_pos));
}

// MoE combine on the tensor core: Y = residual (+ inter-residual) + sum_j (gate-scaled expert row j
// of the sample) + Shared(n), one grouped-GEMM launch: the sources enter the accumulator through
// identity MMAs (tensor maps in the output's row geometry and over the bank-major expert rows
// [banks][k][B][W]), then the shared expert's GEMM2 accumulates onto them.
tm_status combine_sum(const Geo& g, const void* hidden_s, const void* wd, int Fs, const void* resid, const void* extra,
                      void* y, const void* slots, int k, cudaStream_t st) {
    GemmParams p = base_params(g);
    p.sched = 0;
    p.K = Fs;
    p.N = g.W;
    p.out = (__nv_bfloat16*)y;
    p.out_elems = (size_t)g.B * g.banks * g.W;
    p.k = k;
    p.src_resid = resid != nullptr;
    p.src_extra = extra != nullptr;
    const int am = gemm1_amode(g);                  // the residual's geometry is that of x's rows
    p.src_mix = am == A_TMA_MIX;
    if (am != A_TMA_MIX && am != A_TMA_3D) return TM_ERR_UNSUPPORTED;
    const int bn = pick_bn_out(g.W);
    p.n_tiles = g.W / bn;
    const bool pair = use_pair(g, A_TMA_2D);
    p.bank_chunk = bank_chunk(2.0 * Fs * g.W, (pair ? 256.0 : 128.0) * 2 * (Fs + (3 + k) * g.W));
    CUtensorMap ma, mb, m0, m1, m2, mo;
    memset(&m0, 0, sizeof(m0));
    memset(&m1, 0, sizeof(m1));
    if (!map_2d(&ma, hidden_s, (uint64_t)g.banks * g.B, Fs, 128) ||
        !map_2d(&mb, wd, (uint64_t)g.banks * g.W, Fs, pair ? bn / 2 : bn) || !gemm1_amap(g, y, am, &mo, 32))
        return TM_ERR_CUDA;
    if (resid && !gemm1_amap(g, resid, am, &m0)) return TM_ERR_CUDA;
    if (extra && !gemm1_amap(g, extra, am, &m1)) return TM_ERR_CUDA;
    memset(&m2, 0, sizeof(m2));
    if (k > 0) {
        // the gate-scaled expert rows, bank-major [banks * k][B][W]: 128 consecutive samples per box
        uint64_t dims[3] = {(uint64_t)g.W, (uint64_t)g.B, (uint64_t)g.banks * k};
        uint64_t strides[2] = {(uint64_t)g.W * 2, (uint64_t)g.B * g.W * 2};
        uint32_t box[3] = {64, 128, 1};
        if (!make_map(&m2, slots, 3, dims, strides, box)) return TM_ERR_CUDA;
    }
    return cuda_status(
        launch_grouped_gemm_src(bn, A_TMA_2D, EPI_SUM, ma, mb, mb, m0, m1, m2, p, sched0_grid(p, pair), st, &mo, pair));
}

// The routed GEMM2: expert rows scaled by their gates, written to their combine positions by scatter
// stores of one-row boxes; p carries the bucket schedule.
tm_status routed_gemm2(const Geo& g, GemmParams p, const void* hidden_r, const void* wd, int Fe, size_t routed, long max_mt,
                       void* slots, cudaStream_t st) {
    p.K = Fe;
    p.N = g.W;
    p.out = (__nv_bfloat16*)slots;
    p.out_ld = g.W;
    p.out_elems = routed * g.W;
    const int bn = pick_bn_out(g.W);
    p.n_tiles = g.W / bn;
    CUtensorMap ma, mb, mo;
    if (!map_2d(&ma, hidden_r, routed, Fe, 128) || !map_2d(&mb, wd, (uint64_t)p.groups * g.W, Fe, bn) ||
        !map_2d(&mo, slots, routed, g.W, 1))
        return TM_ERR_CUDA;
    const long grid = max_mt * p.n_tiles < num_sms() ? max_mt * p.n_tiles : num_sms();
    return cuda_status(launch_grouped_gemm(bn, A_TMA_2D, EPI_SLOT_PERM, ma, mb, mb, p, (int)grid, st, &mo));
}

tm_status run_moe(const Geo& g, const void* x, const void* resid, const void* extra, const void* gain,
                  const tm_moe_w* w, void* y, void* ws, size_t wsb, cudaStream_t st) {
    Carve c{(uint8_t*)ws};
    MoeWs m = carve_moe(c, g, w, gain != nullptr);
    if (!ws || wsb < c.off || !al16(ws)) return TM_ERR_WORKSPACE;
    if (w->hidden_s == 0) return TM_ERR_UNSUPPORTED;
    const void *weg = w->we_gate, *weu = w->we_up, *wsg = w->ws_gate, *wsu = w->ws_up;
    tm_status s;
    const size_t G = (size_t)g.banks * w->E;
    if (gain) {
        if ((s = cuda_status(launch_fold_gain(g.dtype, weg, gain, m.weg, G * w->hidden_e, g.W, st))) != TM_OK) return s;
        if ((s = cuda_status(launch_fold_gain(g.dtype, weu, gain, m.weu, G * w->hidden_e, g.W, st))) != TM_OK) return s;
        if ((s = cuda_status(launch_fold_gain(g.dtype, wsg, gain, m.wsg, (size_t)g.banks * w->hidden_s, g.W, st))) != TM_OK)
            return s;
        if ((s = cuda_status(launch_fold_gain(g.dtype, wsu, gain, m.wsu, (size_t)g.banks * w->hidden_s, g.W, st))) != TM_OK)
            return s;
        weg = m.weg; weu = m.weu; wsg = m.wsg; wsu = m.wsu;
    }
    RouteOut r{m.idx, m.offsets, m.tile_start, m.bucket_rows, m.slot_of, m.counts, m.gate, m.inv_rms};
    const bool bf16_path = g.dtype == TM_BF16;
    if (bf16_path) {
        r.perm = m.perm;
        r.inv_pos = m.inv_pos;
        r.gate_pos = m.gate_pos;
    }
    r.wsplit = m.wsplit;
    r.tile_info = m.tile_info;
    if ((s = run_route(g, x, gain, w, r, st)) != TM_OK) return s;

    const size_t routed = (size_t)g.B * g.banks * w->k;
    const int Fe = w->hidden_e;
    // routed experts, GEMM1 + SwiGLU over the buckets (rows gathered through the row map)
    GemmParams p = base_params(g);
    p.sched = 1;
    p.groups = (int)G;
    p.E = w->E;
    p.row_start = m.offsets;
    p.tile_start = m.tile_start;
    p.tile_info = m.tile_info;
    p.bucket_rows = m.bucket_rows;
    p.pos_scale = bf16_path ? m.inv_pos : nullptr;
    p.pos_limit = (int)routed;
    p.K = g.W;
    p.N = 2 * Fe;
    p.inv_rms = m.inv_rms;
    p.out = (__nv_bfloat16*)m.hidden_r;
    p.out_ld = Fe;
    p.out_elems = routed * Fe;
    p.a_ptr = (const __nv_bfloat16*)x;
    const long max_mt = (long)(routed / 128) + (long)G;   // 128-row tiles of the buckets, at most
    if (g.dtype == TM_F32) {
        p.n_tiles = Fe / 32;
        SimtGemmArgs a{p, (const float*)x, (const float*)weg, (const float*)weu};
        if ((s = cuda_status(launch_simt_gemm(EPI_SWIGLU, a, (int)(max_mt * p.n_tiles), st))) != TM_OK) return s;
    } else {
        // MoEPermute: copy the routed rows into bucket order (the slot buffer, [routed, W], is free
        // until the routed GEMM2 writes it), then GEMM1 reads A as contiguous rows through a 2-D
        // tensor map.  (Gathering the rows inside GEMM1 instead measured slower than this copy plus one
        // 16 KB box per K slab: by tile::gather4 TMA loads of one-row boxes 2.2x, by the gatherer
        // warps' cp.async 3-6x; every N tile gathers its A rows again.)
        const int bn = pick_bn_swiglu(Fe);
        p.n_tiles = p.N / bn;
        CUtensorMap ma, mg, mu, mo;
        if (!map_2d(&mg, weg, G * Fe, g.W, bn / 2) || !map_2d(&mu, weu, G * Fe, g.W, bn / 2) ||
            !map_2d(&mo, m.hidden_r, routed, Fe, 32))
            return TM_ERR_CUDA;
        if ((s = cuda_status(launch_scatter_rows(g.dtype, x, g.map, g.B, w->k, m.slot_of, routed, m.slots, st))) != TM_OK)
            return s;
        if (!map_2d(&ma, m.slots, routed, g.W, 128)) return TM_ERR_CUDA;
        const long grid = max_mt * p.n_tiles < num_sms() ? max_mt * p.n_tiles : num_sms();
        if ((s = cuda_status(launch_grouped_gemm(bn, A_TMA_2D, EPI_SWIGLU, ma, mg, mu, p, (int)grid, st, &mo))) != TM_OK)
            return s;
    }
    // shared expert GEMM1 (dense rows)
    if ((s = gemm1_dense(g, x, wsg, wsu, w->hidden_s, m.inv_rms, m.hidden_s, st)) != TM_OK) return s;
    // routed experts GEMM2 -> slot rows
    p.K = Fe;
    p.N = g.W;
    p.out = (__nv_bfloat16*)m.slots;
    p.out_ld = g.W;
    p.out_elems = routed * g.W;
    if (g.dtype == TM_F32) {
        p.n_tiles = g.W / 32;
        SimtGemmArgs a{p, (const float*)m.hidden_r, (const float*)w->we_down, nullptr};
        if ((s = cuda_status(launch_simt_gemm(EPI_SLOT, a, (int)(max_mt * p.n_tiles), st))) != TM_OK) return s;
    } else {
        // rows written in combine order ((bank * k + j) * B + b) and scaled by their gate, so that
        // the combine reads each tile's expert rows as one contiguous tensor-map box per choice; they
        // leave through scatter stores of one-row boxes into the slot rows
        p.perm = m.perm;
        p.gate = m.gate;
        p.pos_scale = m.gate_pos;
        if ((s = routed_gemm2(g, p, m.hidden_r, w->we_down, Fe, routed, max_mt, m.slots, st)) != TM_OK) return s;
        return combine_sum(g, m.hidden_s, w->ws_down, w->hidden_s, resid, extra, y, m.slots, w->k, st);
    }
    // shared expert GEMM2 + deterministic combine + residual(s), stored through the row map
    return gemm2_dense(g, m.hidden_s, w->ws_down, w->hidden_s, EPI_COMBINE, resid, extra, y, m.gate, m.slot_of,
                       m.slots, w->k, st);
}

// ------------------------------------------------------------------ FP8 E4M3 dense sub-layer
bool env_is(const char* name, char v);

tm_status check_dense8(const Geo& g, const tm_swiglu_w8* w) {
    if (!w || w->banks != g.banks || w->width != g.W || w->hidden <= 0) return TM_ERR_INVALID_ARG;
    if (!w->q_gate || !w->q_up || !w->s_gate || !w->s_up || !w->w_down) return TM_ERR_INVALID_ARG;
    if (!al16(w->q_gate) || !al16(w->q_up) || !al16(w->s_gate) || !al16(w->s_up) || !al16(w->w_down))
        return TM_ERR_INVALID_ARG;
    if (g.dtype != TM_BF16 || (g.W != 128 && g.W != 256) || w->hidden % 128) return TM_ERR_UNSUPPORTED;
    const int am = gemm1_amode(g);
    if (am != A_TMA_MIX && am != A_TMA_3D) return TM_ERR_UNSUPPORTED;
    return TM_OK;
}

// E4M3 gate / up maps of a bank set: [banks * F rows, W] codes, 128 x 128 boxes
bool maps_e4m3(const Geo& g, const tm_swiglu_w8* w, CUtensorMap* mg, CUtensorMap* mu) {
    uint64_t dims[2] = {(uint64_t)g.W, (uint64_t)g.banks * w->hidden};
    uint64_t strides[1] = {(uint64_t)g.W};
    uint32_t box[2] = {128, 128};
    return make_map_u8(mg, w->q_gate, 2, dims, strides, box) && make_map_u8(mu, w->q_up, 2, dims, strides, box);
}

// One launch of the fused kernel in its FP8 mode: the kernel quantizes each A tile itself (row
// statistics and E4M3 codes from the resident bf16 tile), so no workspace is needed.
tm_status run_dense8(const Geo& g, const void* x, const void* resid, const void* extra, const tm_swiglu_w8* w, void* y,
                     cudaStream_t st) {
    if ((uintptr_t)y % 32) return TM_ERR_INVALID_ARG;
    const int am = gemm1_amode(g), F = w->hidden;
    CUtensorMap ma, mg, mu, md, mr, me, mo;
    memset(&mr, 0, sizeof(mr));
    memset(&me, 0, sizeof(me));
    if (!gemm1_amap(g, x, am, &ma) || !maps_e4m3(g, w, &mg, &mu) || !map_2d(&md, w->w_down, (uint64_t)g.banks * g.W, F, g.W) ||
        !gemm1_amap(g, y, am, &mo, 32))
        return TM_ERR_CUDA;
    FusedParams p;
    memset(&p, 0, sizeof(p));
    // residual: the A tile itself when it is the sub-layer input, else streamed; the inter-residual likewise
    p.res_mode = resid == nullptr ? RES_NONE : resid == x ? RES_FROM_A : RES_STREAM;
    p.has_extra = extra != nullptr;
    if (p.res_mode == RES_STREAM && !gemm1_amap(g, resid, am, &mr)) return TM_ERR_CUDA;
    if (extra && !gemm1_amap(g, extra, am, &me)) return TM_ERR_CUDA;
    p.banks = g.banks;
    p.rows = g.B;
    p.F = F;
    p.amap = g.map;
    p.omap = g.map;
    p.eps = g.eps;
    p.out = (__nv_bfloat16*)y;
    p.out_elems = (size_t)g.B * g.banks * g.W;
    p.s_gate = w->s_gate;
    p.s_up = w->s_up;
    const long tiles = (long)g.banks * ((g.B + 127) / 128);
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    return cuda_status(launch_fused128(g.W, am, true, ma, mg, mu, md, mr, me, mo, p, grid, st));
}

// Both sub-layers of an FP8 block in one launch (block mode, as fused_block): same row width
// (T == H), head width a multiple of 16.  counters: ceil(B/128) uint32 of workspace.
bool block8_fusable(const Geo& gm, const Geo& gr, const void* Y, const void* Xr) {
    if (gm.W != gr.W || gm.banks != gr.banks || gemm1_amode(gm) != A_TMA_MIX) return false;
    if ((uintptr_t)Y % 32 || (uintptr_t)Xr % 32 || env_is("TM_FUSED_BLOCK", '0')) return false;
    return true;
}

tm_status fused_block8(const tm_block_fp8* b, const Geo& gm, const Geo& gr, const void* X, void* Y, void* Xr,
                       unsigned* dep, cudaStream_t st) {
    const int W = gm.W, mt = (gm.B + 127) / 128;
    tm_status s;
    if ((s = cuda_status(cudaMemsetAsync(dep, 0, (size_t)mt * sizeof(unsigned), st))) != TM_OK) return s;
    FusedMaps mm, mr;
    CUtensorMap mres, mext;
    memset(&mext, 0, sizeof(mext));
    if (!gemm1_amap(gm, X, A_TMA_MIX, &mm.a) || !gemm1_amap(gm, Xr, A_TMA_MIX, &mm.o, 32) ||
        !maps_e4m3(gm, &b->mix, &mm.g, &mm.u) || !map_2d(&mm.d, b->mix.w_down, (uint64_t)gm.banks * W, b->mix.hidden, W))
        return TM_ERR_CUDA;
    if (!gemm1_amap(gr, Xr, A_TMA_3D, &mr.a) || !gemm1_amap(gr, Y, A_TMA_3D, &mr.o, 32) ||
        !maps_e4m3(gr, &b->rev, &mr.g, &mr.u) || !map_2d(&mr.d, b->rev.w_down, (uint64_t)gr.banks * W, b->rev.hidden, W) ||
        !gemm1_amap(gr, X, A_TMA_3D, &mres))
        return TM_ERR_CUDA;
    FusedParams p;
    memset(&p, 0, sizeof(p));
    p.banks = gm.banks;
    p.rows = gm.B;
    p.F = b->mix.hidden;
    p.F2 = b->rev.hidden;
    p.amap = gm.map;
    p.omap = gm.map;
    p.eps = gm.eps;
    p.out = (__nv_bfloat16*)Y;
    p.out_elems = (size_t)gm.B * gm.banks * W;
    p.res_mode = RES_FROM_A;
    p.res_mode2 = RES_STREAM;
    p.dep = dep;
    p.s_gate = b->mix.s_gate;
    p.s_up = b->mix.s_up;
    p.s_gate2 = b->rev.s_gate;
    p.s_up2 = b->rev.s_up;
    const long tiles = 2L * gm.banks * mt;
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    return cuda_status(launch_fused128_block(W, true, mm, mr, mres, mext, p, grid, st));
}

// block geometry of the FP8 path
tm_status check_block8(const tm_shape* s, const tm_block_fp8* b, Geo* gm, Geo* gr) {
    if (!b) return TM_ERR_INVALID_ARG;
    tm_status st = make_geo(s, TM_LAYOUT_MIXED, b->mix.banks, b->mix.width, gm);
    if (st == TM_OK) st = check_dense8(*gm, &b->mix);
    if (st == TM_OK) st = make_geo(s, TM_LAYOUT_ROWS, b->rev.banks, b->rev.width, gr);
    if (st == TM_OK) st = check_dense8(*gr, &b->rev);
    if (st == TM_OK && (gr->banks != s->T || gr->W != s->D)) st = TM_ERR_INVALID_ARG;
    return st;
}

// workspace of an FP8 block: X_revert and the row-block counters of block mode
size_t block8_ws(const Geo& gm, const Geo&, const tm_shape* s) {
    return align256((size_t)s->B * s->T * s->D * 2) + align256((size_t)(gm.B + 127) / 128 * sizeof(unsigned));
}

// ------------------------------------------------------------------ FP8 E4M3 MoE sub-layer
// The routing view of an FP8 MoE bank (router, counts, k, alpha) with its code matrices standing in
// for the bf16 gate / up weights, so that the bf16 path's checks and workspace carve apply.
tm_moe_w moe_view(const tm_moe_w8* w) {
    tm_moe_w v;
    v.banks = w->banks;
    v.width = w->width;
    v.E = w->E;
    v.k = w->k;
    v.hidden_e = w->hidden_e;
    v.hidden_s = w->hidden_s;
    v.alpha = w->alpha;
    v.w_router = w->w_router;
    v.we_gate = w->qe_gate;
    v.we_up = w->qe_up;
    v.we_down = w->we_down;
    v.ws_gate = w->qs_gate;
    v.ws_up = w->qs_up;
    v.ws_down = w->ws_down;
    return v;
}

tm_status check_moe8(const Geo& g, const tm_moe_w8* w) {
    if (!w) return TM_ERR_INVALID_ARG;
    const tm_moe_w v = moe_view(w);
    tm_status s = check_moe(g, &v);
    if (s != TM_OK) return s;
    if (!w->se_gate || !w->se_up || !al16(w->se_gate) || !al16(w->se_up)) return TM_ERR_INVALID_ARG;
    if (w->hidden_s > 0 && (!w->ss_gate || !w->ss_up || !al16(w->ss_gate) || !al16(w->ss_up))) return TM_ERR_INVALID_ARG;
    if (g.dtype != TM_BF16 || w->hidden_s == 0) return TM_ERR_UNSUPPORTED;
    // E4M3 K slabs of 128 codes; the quantizer holds a row in one warp's registers
    if (g.W % 128 || g.W > 1024 || w->hidden_e % 128 || w->hidden_s % 128) return TM_ERR_UNSUPPORTED;
    if (g.map.layout == 1 && g.map.dh % 8) return TM_ERR_UNSUPPORTED;
    const int am = gemm1_amode(g);
    if (am != A_TMA_MIX && am != A_TMA_3D) return TM_ERR_UNSUPPORTED;   // the combine's residual maps
    return TM_OK;
}

// The bf16 MoE workspace (routing tables, hidden rows, slot rows) plus the rows' E4M3 factors.  The
// codes live in the slot buffer, which is free until the routed GEMM2 writes it: the bucket-order
// codes [routed, W] first, then the row-order codes [B * banks, W] (routed * W * 2 bytes hold both).
struct Moe8Ws {
    MoeWs m;
    float* rowscale;
    uint8_t *qpos, *q;
};
Moe8Ws carve_moe8(Carve& c, const Geo& g, const tm_moe_w8* w) {
    Moe8Ws r;
    const tm_moe_w v = moe_view(w);
    r.m = carve_moe(c, g, &v, false);
    r.rowscale = c.take<float>((size_t)g.B * g.banks);
    const size_t routed = (size_t)g.B * g.banks * w->k;
    r.qpos = (uint8_t*)r.m.slots;
    r.q = r.qpos + routed * g.W;
    return r;
}

// E4M3 GEMM1 + SwiGLU over `groups` groups of code rows (tmA), weights q_gate / q_up [groups * F, W]
tm_status gemm1_f8(GemmParams p, int a_mode, const CUtensorMap& ma, const uint8_t* qg, const uint8_t* qu, int F,
                   const float* sg, const float* su, void* hidden, size_t rows_out, int grid, cudaStream_t st) {
    const int bn = pick_bn_swiglu(F);
    p.N = 2 * F;
    p.n_tiles = p.N / bn;
    p.out = (__nv_bfloat16*)hidden;
    p.out_ld = F;
    p.out_elems = rows_out * F;
    p.w8_sgate = sg;
    p.w8_sup = su;
    uint64_t dims[2] = {(uint64_t)p.K, (uint64_t)p.groups * F};
    uint64_t strides[1] = {(uint64_t)p.K};
    uint32_t box[2] = {128, (uint32_t)bn / 2};
    CUtensorMap mg, mu, mo;
    if (!make_map_u8(&mg, qg, 2, dims, strides, box) || !make_map_u8(&mu, qu, 2, dims, strides, box) ||
        !map_2d(&mo, hidden, rows_out, F, 32))
        return TM_ERR_CUDA;
    if (grid <= 0) grid = dense_grid(p);
    return cuda_status(launch_grouped_gemm_f8(bn, a_mode, ma, mg, mu, p, grid, st, &mo));
}

// The MoE sub-layer with E4M3 GEMM1s: route (bf16 path's router) -> quantize every row once, writing
// its codes in row order and at its k bucket positions -> routed GEMM1 over the buckets, shared GEMM1
// over the rows (both kind::f8f6f4) -> the bf16 routed GEMM2 into combine order -> combine + shared
// GEMM2 + residuals.
tm_status run_moe8(const Geo& g, const void* x, const void* resid, const void* extra, const void* gain,
                   const tm_moe_w8* w, void* y, void* ws, size_t wsb, cudaStream_t st) {
    Carve c{(uint8_t*)ws};
    Moe8Ws q = carve_moe8(c, g, w);
    MoeWs& m = q.m;
    if (!ws || wsb < c.off || !al16(ws)) return TM_ERR_WORKSPACE;
    const tm_moe_w v = moe_view(w);
    tm_status s;
    RouteOut r{m.idx, m.offsets, m.tile_start, m.bucket_rows, m.slot_of, m.counts, m.gate, m.inv_rms};
    r.perm = m.perm;
    r.inv_pos = nullptr;        // the row factors by position come from the quantizer
    r.gate_pos = m.gate_pos;
    r.wsplit = m.wsplit;
    r.tile_info = m.tile_info;
    if ((s = run_route(g, x, gain, &v, r, st)) != TM_OK) return s;

    const size_t rows = (size_t)g.B * g.banks, routed = rows * w->k;
    if ((s = cuda_status(launch_quant_act_rows(x, g.map, g.B, g.eps, q.q, q.rowscale, st, m.slot_of, w->k, routed,
                                               q.qpos, m.inv_pos))) != TM_OK)
        return s;
    const size_t G = (size_t)g.banks * w->E;
    const int Fe = w->hidden_e;
    const long max_mt = (long)(routed / 128) + (long)G;
    // routed experts: bucket-order codes through a 2-D map, row factor by bucket position
    GemmParams p = base_params(g);
    p.sched = 1;
    p.groups = (int)G;
    p.E = w->E;
    p.row_start = m.offsets;
    p.tile_start = m.tile_start;
    p.tile_info = m.tile_info;
    p.bucket_rows = m.bucket_rows;
    p.pos_scale = m.inv_pos;
    p.pos_limit = (int)routed;
    p.K = g.W;
    {
        uint64_t dims[2] = {(uint64_t)g.W, (uint64_t)routed};
        uint64_t strides[1] = {(uint64_t)g.W};
        uint32_t box[2] = {128, 128};
        CUtensorMap ma;
        if (!make_map_u8(&ma, q.qpos, 2, dims, strides, box)) return TM_ERR_CUDA;
        const int nt = 2 * Fe / pick_bn_swiglu(Fe);
        const long grid = max_mt * nt < num_sms() ? max_mt * nt : num_sms();
        if ((s = gemm1_f8(p, A_TMA_2D, ma, w->qe_gate, w->qe_up, Fe, w->se_gate, w->se_up, m.hidden_r, routed, (int)grid,
                          st)) != TM_OK)
            return s;
    }
    // shared expert: row-order codes [B, banks, W] through a 3-D map, row factor by row
    {
        GemmParams ps = base_params(g);
        ps.sched = 0;
        ps.K = g.W;
        ps.inv_rms = q.rowscale;
        ps.bank_chunk = bank_chunk(2.0 * w->hidden_s * g.W, 128.0 * (g.W + 2.0 * w->hidden_s));
        uint64_t dims[3] = {(uint64_t)g.W, (uint64_t)g.banks, (uint64_t)g.B};
        uint64_t strides[2] = {(uint64_t)g.W, (uint64_t)g.banks * g.W};
        uint32_t box[3] = {128, 1, 128};
        CUtensorMap ma;
        if (!make_map_u8(&ma, q.q, 3, dims, strides, box)) return TM_ERR_CUDA;
        if ((s = gemm1_f8(ps, A_TMA_3D, ma, w->qs_gate, w->qs_up, w->hidden_s, w->ss_gate, w->ss_up, m.hidden_s, rows, 0,
                          st)) != TM_OK)
            return s;
    }
    // routed GEMM2 (bf16) into combine order, gate-scaled, then the combine with the shared GEMM2
    p.pos_scale = m.gate_pos;
    p.perm = m.perm;
    p.gate = m.gate;
    if ((s = routed_gemm2(g, p, m.hidden_r, w->we_down, Fe, routed, max_mt, m.slots, st)) != TM_OK) return s;
    return combine_sum(g, m.hidden_s, w->ws_down, w->hidden_s, resid, extra, y, m.slots, w->k, st);
}

tm_status check_sublayer8(const tm_shape* shape, int layout, const tm_sublayer8* sub, Geo* g) {
    if (!sub) return TM_ERR_INVALID_ARG;
    const int banks = sub->is_moe ? sub->moe.banks : sub->dense.banks;
    const int width = sub->is_moe ? sub->moe.width : sub->dense.width;
    tm_status s = make_geo(shape, layout, banks, width, g);
    if (s != TM_OK) return s;
    if (sub->norm_gain && !al16(sub->norm_gain)) return TM_ERR_INVALID_ARG;
    if (!sub->is_moe && sub->norm_gain) return TM_ERR_INVALID_ARG;   // folded into the codes
    return sub->is_moe ? check_moe8(*g, &sub->moe) : check_dense8(*g, &sub->dense);
}

// ------------------------------------------------------------------ sub-layer dispatch
int sub_banks(const tm_sublayer* s) { return s->is_moe ? s->moe.banks : s->dense.banks; }
int sub_width(const tm_sublayer* s) { return s->is_moe ? s->moe.width : s->dense.width; }

tm_status check_sublayer(const tm_shape* shape, int layout, const tm_sublayer* sub, Geo* g) {
    if (!sub) return TM_ERR_INVALID_ARG;
    tm_status s = make_geo(shape, layout, sub_banks(sub), sub_width(sub), g);
    if (s != TM_OK) return s;
    if (sub->norm_gain && !al16(sub->norm_gain)) return TM_ERR_INVALID_ARG;
    if (sub->is_moe) {
        s = check_moe(*g, &sub->moe);
        if (s == TM_OK && sub->moe.hidden_s == 0) s = TM_ERR_UNSUPPORTED;
        // the bf16 combine reads the residual through a tensor map: mixed rows need 16-column head
        // pieces (refused here, before the routing and the GEMMs are launched)
        if (s == TM_OK && g->dtype == TM_BF16 && gemm1_amode(*g) == A_GATHER) s = TM_ERR_UNSUPPORTED;
        return s;
    }
    return check_dense(*g, &sub->dense);
}

size_t sublayer_ws(const Geo& g, const tm_sublayer* sub) {
    Carve c{nullptr};
    if (sub->is_moe) carve_moe(c, g, &sub->moe, sub->norm_gain != nullptr);
    else carve_dense(c, g, sub->dense.hidden, sub->norm_gain != nullptr);
    return align256(c.off);
}

tm_status run_sublayer(const Geo& g, const void* x, const void* resid, const void* extra, const tm_sublayer* sub,
                       void* y, void* ws, size_t wsb, cudaStream_t st) {
    if (sub->is_moe) return run_moe(g, x, resid, extra, sub->norm_gain, &sub->moe, y, ws, wsb, st);
    return run_dense(g, x, resid, extra, sub->norm_gain, &sub->dense, y, ws, wsb, st);
}

// block geometry: mixing sub-layer (MIXED, banks H) and reverting sub-layer (ROWS, banks T, width D)
tm_status check_block(const tm_shape* s, const tm_block* b, Geo* gm, Geo* gr) {
    if (!b) return TM_ERR_INVALID_ARG;
    tm_status st = check_sublayer(s, TM_LAYOUT_MIXED, &b->mix, gm);
    if (st != TM_OK) return st;
    st = check_sublayer(s, TM_LAYOUT_ROWS, &b->rev, gr);
    if (st != TM_OK) return st;
    if (gr->banks != s->T || gr->W != s->D) return TM_ERR_INVALID_ARG;
    return TM_OK;
}

// ------------------------------------------------------------------ fused dense block
// Both sub-layers of a block in one launch (launch_fused128_block): dense bf16 sub-layers of the
// same row width 128 or 256 (T == H), head width a multiple of 16, hidden widths multiples of 128.
// TM_FUSED_BLOCK=0 in the environment keeps one launch per sub-layer: the tests use it to show
// that the one-launch block gives the same bits as the per-sub-layer launches.
bool env_is(const char* name, char v) {
    const char* e = getenv(name);
    return e && e[0] == v;
}

bool block_fusable(const tm_shape* s, const tm_block* b, const Geo& gm, const Geo& gr, const void* Y, const void* Xr) {
    if (s->dtype != TM_BF16 || b->mix.is_moe || b->rev.is_moe) return false;
    if (gm.W != gr.W || (gm.W != 128 && gm.W != 256) || gm.banks != gr.banks) return false;
    if (gemm1_amode(gm) != A_TMA_MIX) return false;
    if (b->mix.dense.hidden % 128 || b->rev.dense.hidden % 128) return false;
    if ((uintptr_t)Y % 32 || (uintptr_t)Xr % 32) return false;
    if (env_is("TM_FUSED_BLOCK", '0')) return false;
    return true;
}

struct BlockWs {
    unsigned* dep;
    void *wg1, *wu1, *wg2, *wu2;
};
BlockWs carve_block(Carve& c, const Geo& gm, const Geo& gr, const tm_block* b) {
    BlockWs w;
    w.dep = c.take<unsigned>((size_t)(gm.B + 127) / 128);
    const size_t n1 = (size_t)gm.banks * b->mix.dense.hidden * gm.W * gm.esz;
    const size_t n2 = (size_t)gr.banks * b->rev.dense.hidden * gr.W * gr.esz;
    w.wg1 = b->mix.norm_gain ? c.take<uint8_t>(n1) : nullptr;
    w.wu1 = b->mix.norm_gain ? c.take<uint8_t>(n1) : nullptr;
    w.wg2 = b->rev.norm_gain ? c.take<uint8_t>(n2) : nullptr;
    w.wu2 = b->rev.norm_gain ? c.take<uint8_t>(n2) : nullptr;
    return w;
}

size_t block_ws(const Geo& gm, const Geo& gr, const tm_block* b) {
    if (b->mix.is_moe || b->rev.is_moe) return 0;
    Carve c{nullptr};
    carve_block(c, gm, gr, b);
    return align256(c.off);
}

// The gate and up weights of a dense sub-layer with its norm gain folded in (into ws), or as given.
tm_status dense_gate_up(const Geo& g, const tm_sublayer* sub, void* wg_ws, void* wu_ws, const void** wg, const void** wu,
                        cudaStream_t st) {
    *wg = sub->dense.w_gate;
    *wu = sub->dense.w_up;
    if (!sub->norm_gain) return TM_OK;
    const size_t rows = (size_t)g.banks * sub->dense.hidden;
    tm_status s;
    if ((s = cuda_status(launch_fold_gain(g.dtype, *wg, sub->norm_gain, wg_ws, rows, g.W, st))) != TM_OK) return s;
    if ((s = cuda_status(launch_fold_gain(g.dtype, *wu, sub->norm_gain, wu_ws, rows, g.W, st))) != TM_OK) return s;
    *wg = wg_ws;
    *wu = wu_ws;
    return TM_OK;
}

tm_status fused_block(const tm_block* b, const Geo& gm, const Geo& gr, const void* X, const void* extra, void* Y,
                      void* Xr, void* ws, size_t wsb, cudaStream_t st) {
    Carve c{(uint8_t*)ws};
    BlockWs w = carve_block(c, gm, gr, b);
    if (!ws || wsb < c.off || !al16(ws)) return TM_ERR_WORKSPACE;
    const int W = gm.W, F1 = b->mix.dense.hidden, F2 = b->rev.dense.hidden;
    const void *wg1, *wu1, *wg2, *wu2;
    tm_status s;
    if ((s = dense_gate_up(gm, &b->mix, w.wg1, w.wu1, &wg1, &wu1, st)) != TM_OK) return s;
    if ((s = dense_gate_up(gr, &b->rev, w.wg2, w.wu2, &wg2, &wu2, st)) != TM_OK) return s;
    const int mt = (gm.B + 127) / 128;
    if ((s = cuda_status(cudaMemsetAsync(w.dep, 0, (size_t)mt * sizeof(unsigned), st))) != TM_OK) return s;
    FusedMaps mm, mr;
    CUtensorMap mres, mext;
    memset(&mext, 0, sizeof(mext));
    // mixing: A through the Mix map over X, output through the Revert map into X_revert
    if (!gemm1_amap(gm, X, A_TMA_MIX, &mm.a) || !gemm1_amap(gm, Xr, A_TMA_MIX, &mm.o, 32) ||
        !map_2d(&mm.g, wg1, (uint64_t)gm.banks * F1, W, 128) || !map_2d(&mm.u, wu1, (uint64_t)gm.banks * F1, W, 128) ||
        !map_2d(&mm.d, b->mix.dense.w_down, (uint64_t)gm.banks * W, F1, W))
        return TM_ERR_CUDA;
    // reverting: A = rows of X_revert, residual X (and the inter-residual) streamed, output Y
    if (!gemm1_amap(gr, Xr, A_TMA_3D, &mr.a) || !gemm1_amap(gr, Y, A_TMA_3D, &mr.o, 32) ||
        !map_2d(&mr.g, wg2, (uint64_t)gr.banks * F2, W, 128) || !map_2d(&mr.u, wu2, (uint64_t)gr.banks * F2, W, 128) ||
        !map_2d(&mr.d, b->rev.dense.w_down, (uint64_t)gr.banks * W, F2, W) || !gemm1_amap(gr, X, A_TMA_3D, &mres) ||
        (extra && !gemm1_amap(gr, extra, A_TMA_3D, &mext)))
        return TM_ERR_CUDA;
    FusedParams p;
    memset(&p, 0, sizeof(p));
    p.banks = gm.banks;
    p.rows = gm.B;
    p.F = F1;
    p.F2 = F2;
    p.amap = gm.map;
    p.omap = gm.map;
    p.eps = gm.eps;
    p.out = (__nv_bfloat16*)Y;
    p.out_elems = (size_t)gm.B * gm.banks * W;
    p.res_mode = RES_FROM_A;
    p.has_extra = 0;
    p.res_mode2 = RES_STREAM;
    p.has_extra2 = extra != nullptr;
    p.dep = w.dep;
    const long tiles = 2L * gm.banks * mt;
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    return cuda_status(launch_fused128_block(W, false, mm, mr, mres, mext, p, grid, st));
}

size_t stack_ws(const tm_shape* s, const tm_block* blocks, int L, int gap, bool* ok) {
    size_t sub = 0;
    for (int l = 0; l < L; ++l) {
        Geo gm, gr;
        if (check_block(s, &blocks[l], &gm, &gr) != TM_OK) { *ok = false; return 0; }
        const size_t a = sublayer_ws(gm, &blocks[l].mix), b = sublayer_ws(gr, &blocks[l].rev);
        const size_t f = block_ws(gm, gr, &blocks[l]);
        sub = a > sub ? a : sub;
        sub = b > sub ? b : sub;
        sub = f > sub ? f : sub;
    }
    *ok = true;
    const size_t tok = align256((size_t)s->B * s->T * s->D * (s->dtype == TM_BF16 ? 2 : 4));
    const int ring = L > 1 ? (gap > 0 ? gap + 1 : 2) : 0;
    return tok * (1 + ring) + sub;
}

tm_status run_block(const tm_shape* s, const tm_block* b, const void* X, const void* extra, void* Y, void* Xr,
                    void* sub_ws, size_t sub_wsb, cudaStream_t st) {
    Geo gm, gr;
    tm_status r = check_block(s, b, &gm, &gr);
    if (r != TM_OK) return r;
    if (block_fusable(s, b, gm, gr, Y, Xr)) return fused_block(b, gm, gr, X, extra, Y, Xr, sub_ws, sub_wsb, st);
    // H_next = FFN_mix(Norm(Mix(X))) + Mix(X), written through Revert straight into X_rev
    if ((r = run_sublayer(gm, X, X, nullptr, &b->mix, Xr, sub_ws, sub_wsb, st)) != TM_OK) return r;
    // Y = FFN_rev(Norm(X_rev)) + X (+ inter-residual)
    return run_sublayer(gr, Xr, X, extra, &b->rev, Y, sub_ws, sub_wsb, st);
}

// ------------------------------------------------------------------ dense sub-layer backward
// Gradients of the FFN term y = SwiGLU_bank(RMSNorm(x)) of a dense bf16 sub-layer (gain 1) for an
// upstream gradient dy.  Every contraction runs on the tcgen05 grouped GEMM with its plain bf16
// store epilogue (both operands K-major, fp32 accumulation in TMEM):
//   G = xh Wg^T, U = xh Wu^T                   recomputed, A = xh [banks][B][W]
//   dH = dy Wd                                 B operand Wd^T [banks][F][W]
//   dWd = dy^T H                               A = dy^T [banks][W][Bp], B operand H^T [banks][F][Bp]
//   dWg = dG^T xh, dWu = dU^T xh               A = dG^T, dU^T [banks][F][Bp], B operand xh^T [banks][W][Bp]
//   dN = dG Wg + dU Wu = (dG | dU) (Wg ; Wu)   B operand (Wg ; Wu)^T [banks][W][2F]
// with Bp = B rounded up to the 64-wide K slab (the transposes write zeros into the padding).  The
// CUDA-core kernels of tm_backward.cu do the row pass, the transposes, the SwiGLU derivative and
// the RMSNorm derivative.
struct DenseBwdWs {
    float* inv_rms;
    uint16_t *xh, *dyb, *G, *U, *dH, *dGU, *Hd, *dN, *WdT, *WguT, *dyT, *HT, *dgT, *duT, *xhT;
};
DenseBwdWs carve_dense_bwd(Carve& c, const Geo& g, int F) {
    const size_t nb = g.banks, B = g.B, W = g.W, Bp = (B + 63) / 64 * 64;
    DenseBwdWs w;
    w.inv_rms = c.take<float>(nb * B);
    w.xh = c.take<uint16_t>(nb * B * W);
    w.dyb = c.take<uint16_t>(nb * B * W);
    w.G = c.take<uint16_t>(nb * B * F);
    w.U = c.take<uint16_t>(nb * B * F);
    w.dH = c.take<uint16_t>(nb * B * F);
    w.dGU = c.take<uint16_t>(nb * B * 2 * F);
    w.Hd = c.take<uint16_t>(nb * B * F);
    w.dN = c.take<uint16_t>(nb * B * W);
    w.WdT = c.take<uint16_t>(nb * F * W);
    w.WguT = c.take<uint16_t>(nb * W * 2 * F);
    w.dyT = c.take<uint16_t>(nb * W * Bp);
    w.HT = c.take<uint16_t>(nb * F * Bp);
    w.dgT = c.take<uint16_t>(nb * F * Bp);
    w.duT = c.take<uint16_t>(nb * F * Bp);
    w.xhT = c.take<uint16_t>(nb * W * Bp);
    return w;
}
size_t dense_bwd_ws(const Geo& g, int F) {
    Carve c{nullptr};
    carve_dense_bwd(c, g, F);
    return align256(c.off);
}

// bf16 only, gain 1 (NULL), row and hidden widths multiples of 128 (64-wide K slabs, N tiles of
// 128 / 192 / 256 columns)
tm_status check_dense_bwd(const Geo& g, const tm_swiglu_w* w, const void* gain) {
    tm_status s = check_dense(g, w);
    if (s != TM_OK) return s;
    if (g.dtype != TM_BF16 || gain) return TM_ERR_UNSUPPORTED;
    if (g.W % 128 || w->hidden % 128) return TM_ERR_UNSUPPORTED;
    return TM_OK;
}

// out[g*rows + r][n] = sum_k A[g*rows + r][k] * Bm[g*N + n][k] for every group g (bf16 out, fp32
// accumulation): the grouped GEMM with its plain store epilogue.  K % 64 == 0, N % 128 == 0.
tm_status gemm_plain(const void* A, int groups, int rows, int K, const void* Bm, int N, void* out, cudaStream_t st) {
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.sched = 0;
    p.groups = groups;
    p.rows = rows;
    p.banks = groups;
    p.E = 1;
    p.K = K;
    p.N = N;
    const int bn = pick_bn_out(N);
    p.n_tiles = N / bn;
    p.out = (__nv_bfloat16*)out;
    p.out_ld = N;
    p.out_elems = (size_t)groups * rows * N;
    p.pos_limit = groups * rows;
    CUtensorMap ma, mb, mo;
    if (!map_2d(&ma, A, (uint64_t)groups * rows, K, 128) || !map_2d(&mb, Bm, (uint64_t)groups * N, K, bn) ||
        !map_2d(&mo, out, (uint64_t)groups * rows, N, 32))
        return TM_ERR_CUDA;
    return cuda_status(launch_grouped_gemm(bn, A_TMA_2D, EPI_SLOT, ma, mb, mb, p, dense_grid(p), st, &mo));
}

// dx = d(FFN term)/dx applied to dy, plus add0, add1 and add2 (NULL: none; all in dx's row layout);
// the weight gradients dwg, dwu [banks, F, W] and dwd [banks, W, F].
tm_status run_dense_bwd(const Geo& g, const void* x, const void* dy, const void* add0, const void* add1,
                        const void* add2, const tm_swiglu_w* w, void* dx, void* dwg, void* dwu, void* dwd, void* ws,
                        size_t wsb, cudaStream_t st) {
    const int B = g.B, W = g.W, F = w->hidden, nb = g.banks;
    const int Bp = (B + 63) / 64 * 64;
    Carve c{(uint8_t*)ws};
    DenseBwdWs d = carve_dense_bwd(c, g, F);
    if (!ws || wsb < c.off || !al16(ws)) return TM_ERR_WORKSPACE;
    const size_t BW = (size_t)B * W, BF = (size_t)B * F, FW = (size_t)F * W;
    tm_status s;
#define TM_TRY(expr)                         \
    do {                                     \
        if ((s = (expr)) != TM_OK) return s; \
    } while (0)
    TM_TRY(cuda_status(launch_bwd_rows(x, dy, g.map, B, g.eps, d.xh, d.dyb, d.inv_rms, st)));
    // the recomputed projections and the gradient at the down projection's input
    TM_TRY(gemm_plain(d.xh, nb, B, W, w->w_gate, F, d.G, st));
    TM_TRY(gemm_plain(d.xh, nb, B, W, w->w_up, F, d.U, st));
    TM_TRY(cuda_status(launch_transpose(w->w_down, FW, F, W, F, d.WdT, FW, W, W, nb, st)));
    TM_TRY(gemm_plain(d.dyb, nb, B, W, d.WdT, F, d.dH, st));
    TM_TRY(cuda_status(launch_swiglu_bwd(d.G, d.U, d.dH, (size_t)nb * B, F, d.dGU, d.Hd, st)));
    // weight gradients: contractions over the samples
    TM_TRY(cuda_status(launch_transpose(d.dyb, BW, W, B, W, d.dyT, (size_t)W * Bp, Bp, Bp, nb, st)));
    TM_TRY(cuda_status(launch_transpose(d.Hd, BF, F, B, F, d.HT, (size_t)F * Bp, Bp, Bp, nb, st)));
    TM_TRY(gemm_plain(d.dyT, nb, W, Bp, d.HT, F, dwd, st));
    TM_TRY(cuda_status(launch_transpose(d.dGU, 2 * BF, 2 * F, B, F, d.dgT, (size_t)F * Bp, Bp, Bp, nb, st)));
    TM_TRY(cuda_status(launch_transpose(d.dGU + F, 2 * BF, 2 * F, B, F, d.duT, (size_t)F * Bp, Bp, Bp, nb, st)));
    TM_TRY(cuda_status(launch_transpose(d.xh, BW, W, B, W, d.xhT, (size_t)W * Bp, Bp, Bp, nb, st)));
    TM_TRY(gemm_plain(d.dgT, nb, F, Bp, d.xhT, W, dwg, st));
    TM_TRY(gemm_plain(d.duT, nb, F, Bp, d.xhT, W, dwu, st));
    // the gradient at the normalised row, then through the RMSNorm
    TM_TRY(cuda_status(launch_transpose(w->w_gate, FW, W, F, W, d.WguT, (size_t)W * 2 * F, 2 * F, F, nb, st)));
    TM_TRY(cuda_status(launch_transpose(w->w_up, FW, W, F, W, d.WguT + F, (size_t)W * 2 * F, 2 * F, F, nb, st)));
    TM_TRY(gemm_plain(d.dGU, nb, B, 2 * F, d.WguT, W, d.dN, st));
    TM_TRY(cuda_status(launch_rms_bwd(x, d.dN, d.inv_rms, add0, add1, add2, g.map, B, dx, st)));
#undef TM_TRY
    return TM_OK;
}

bool grads_ok(const tm_swiglu_grads* gr) {
    return gr && gr->dw_gate && gr->dw_up && gr->dw_down && al16(gr->dw_gate) && al16(gr->dw_up) && al16(gr->dw_down);
}

// Block backward: both sub-layers dense bf16 with gain 1.  Workspace: X_rev, dX_rev, then one
// region shared by the mixing sub-layer's forward (X_rev recomputed) and the two backward passes.
tm_status check_block_bwd(const tm_shape* s, const tm_block* b, Geo* gm, Geo* gr) {
    tm_status st = check_block(s, b, gm, gr);
    if (st != TM_OK) return st;
    if (b->mix.is_moe || b->rev.is_moe) return TM_ERR_UNSUPPORTED;
    if ((st = check_dense_bwd(*gm, &b->mix.dense, b->mix.norm_gain)) != TM_OK) return st;
    return check_dense_bwd(*gr, &b->rev.dense, b->rev.norm_gain);
}
size_t block_bwd_sub_ws(const Geo& gm, const Geo& gr, const tm_block* b) {
    size_t n = sublayer_ws(gm, &b->mix);
    const size_t m = dense_bwd_ws(gm, b->mix.dense.hidden), r = dense_bwd_ws(gr, b->rev.dense.hidden);
    n = m > n ? m : n;
    return r > n ? r : n;
}

// One block's backward: X_rev recomputed into Xr, dX_rev into dXr (both [B,T,D] scratch), then
// dX = dY + Revert(dH) + extra (extra: NULL or a further gradient of X, e.g. an inter-residual's).
tm_status run_block_bwd(const Geo& gm, const Geo& gr, const tm_block* b, const void* X, const void* dY,
                        const void* extra, void* dX, const tm_block_grads* grads, void* Xr, void* dXr, void* ws,
                        size_t wsb, cudaStream_t st) {
    tm_status s;
    // X_rev = Revert(FFN_mix(Norm(Mix(X))) + Mix(X)), as the forward stored it
    if ((s = run_sublayer(gm, X, X, nullptr, &b->mix, Xr, ws, wsb, st)) != TM_OK) return s;
    // reverting sub-layer: dX_rev = d FFN_rev(Norm(X_rev)) / d X_rev applied to dY
    if ((s = run_dense_bwd(gr, Xr, dY, nullptr, nullptr, nullptr, &b->rev.dense, dXr, grads->rev.dw_gate,
                           grads->rev.dw_up, grads->rev.dw_down, ws, wsb, st)) != TM_OK)
        return s;
    // mixing sub-layer on mixed rows: dH_next = Mix(dX_rev); dX = dY + Revert(d FFN_mix applied to
    // dH_next + dH_next) (+ extra), written through the same row map
    return run_dense_bwd(gm, X, dXr, dXr, dY, extra, &b->mix.dense, dX, grads->mix.dw_gate, grads->mix.dw_up,
                         grads->mix.dw_down, ws, wsb, st);
}

}  // namespace
}  // namespace tml

using namespace tml;

extern "C" {

const char* tm_status_string(tm_status s) {
    switch (s) {
        case TM_OK: return "ok";
        case TM_ERR_INVALID_ARG: return "invalid argument";
        case TM_ERR_UNSUPPORTED: return "unsupported configuration";
        case TM_ERR_WORKSPACE: return "workspace missing or too small";
        case TM_ERR_CUDA: return "CUDA error";
        case TM_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case TM_ERR_DEVICE_BOUNDS: return "device bounds check failed";
    }
    return "unknown status";
}

int tm_version(void) { return 100; }

size_t tm_sublayer_workspace_bytes(const tm_shape* shape, tm_layout layout, const tm_sublayer* sub) {
    Geo g;
    if (check_sublayer(shape, layout, sub, &g) != TM_OK) return 0;
    return sublayer_ws(g, sub);
}

size_t tm_route_workspace_bytes(const tm_shape* shape, tm_layout layout, const tm_moe_w* w) {
    Geo g;
    if (!w || make_geo(shape, layout, w->banks, w->width, &g) != TM_OK || check_moe(g, w) != TM_OK) return 0;
    const int nchunks = (g.B + kRouterChunk - 1) / kRouterChunk;
    return align256((size_t)g.banks * nchunks * w->E * sizeof(int32_t)) + align256(((size_t)g.banks * w->E + 1) * 4) +
           align256(route_split_bytes(g, w));
}

size_t tm_workspace_bytes(const tm_shape* shape, const tm_block* blocks, int L, int gap) {
    if (!blocks || L < 1 || gap < 0) return 0;
    bool ok = false;
    const size_t n = stack_ws(shape, blocks, L, gap, &ok);
    return ok ? n : 0;
}

tm_status tm_tokenize_stub(const void* groups, const void* w_group, const void* w_global, int dg,
                           const tm_shape* shape, void* X_out, void* stream) {
    tm_status s = check_shape(shape);
    if (s != TM_OK) return s;
    if (!groups || !w_global || !X_out || dg <= 0 || shape->T < 2) return TM_ERR_INVALID_ARG;
    if (!w_group) return TM_ERR_INVALID_ARG;
    if (!al_elem(groups, shape->dtype) || !al_elem(w_group, shape->dtype) || !al_elem(w_global, shape->dtype) ||
        !al_elem(X_out, shape->dtype))
        return TM_ERR_INVALID_ARG;
    return cuda_status(launch_tokenize(shape->dtype, groups, w_group, w_global, dg, shape->B, shape->T, shape->D, X_out,
                                       (cudaStream_t)stream));
}

tm_status tm_head_forward(const void* X, const tm_shape* shape, const void* w_head, float* logits, void* stream) {
    tm_status s = check_shape(shape);
    if (s != TM_OK) return s;
    if (!X || !w_head || !logits || !al16(X) || !al16(w_head) || (reinterpret_cast<uintptr_t>(logits) & 3))
        return TM_ERR_INVALID_ARG;
    return cuda_status(launch_head(shape->dtype, X, w_head, shape->B, shape->T, shape->D, logits, (cudaStream_t)stream));
}

size_t tm_model_workspace_bytes(const tm_shape* shape, const tm_block* blocks, int L, int gap) {
    const size_t st = tm_workspace_bytes(shape, blocks, L, gap);
    if (st == 0) return 0;
    const size_t tok = align256((size_t)shape->B * shape->T * shape->D * (shape->dtype == TM_BF16 ? 2 : 4));
    return 2 * tok + st;
}

tm_status tm_model_forward(const void* groups, const void* w_group, const void* w_global, int dg, const tm_block* blocks,
                           int L, int gap, const void* w_head, const tm_shape* shape, float* logits, void* workspace,
                           size_t workspace_bytes, void* stream) {
    const size_t need = tm_model_workspace_bytes(shape, blocks, L, gap);
    if (need == 0) return TM_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need || !al16(workspace)) return TM_ERR_WORKSPACE;
    const size_t tok = align256((size_t)shape->B * shape->T * shape->D * (shape->dtype == TM_BF16 ? 2 : 4));
    uint8_t* X = (uint8_t*)workspace;
    uint8_t* Y = X + tok;
    tm_status s;
    if ((s = tm_tokenize_stub(groups, w_group, w_global, dg, shape, X, stream)) != TM_OK) return s;
    if ((s = tm_stack_forward(X, blocks, L, gap, shape, Y, Y + tok, workspace_bytes - 2 * tok, stream)) != TM_OK)
        return s;
    return tm_head_forward(Y, shape, w_head, logits, stream);
}

tm_status tm_mix(const void* X, void* Hm, const tm_shape* shape, void* stream) {
    tm_status s = check_shape(shape);
    if (s != TM_OK) return s;
    if (!X || !Hm || X == Hm || !al_elem(X, shape->dtype) || !al_elem(Hm, shape->dtype)) return TM_ERR_INVALID_ARG;
    return cuda_status(launch_permute(shape->dtype, X, Hm, shape->B, shape->T, shape->D, shape->H, true,
                                      (cudaStream_t)stream));
}

tm_status tm_tp_exchange_layout(const void* src, void* dst, int P, int B, int Tp, int Dp, tm_dtype dtype,
                                int local_layout, int to_exchange, void* stream) {
    if (!src || !dst || src == dst || P < 1 || B < 1 || Tp < 1 || Dp < 1) return TM_ERR_INVALID_ARG;
    if ((dtype != TM_F32 && dtype != TM_BF16) || (local_layout != TM_TP_TOKEN_SHARD && local_layout != TM_TP_HEAD_SHARD))
        return TM_ERR_INVALID_ARG;
    const int esz = dtype == TM_BF16 ? 2 : 4;
    if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & (uintptr_t)(esz - 1)) != 0)
        return TM_ERR_INVALID_ARG;
    if (((size_t)Dp * esz) % 16 == 0 && (!al16(src) || !al16(dst))) return TM_ERR_INVALID_ARG;
    return cuda_status(launch_tp_layout(src, dst, P, B, Tp, Dp, esz, local_layout == TM_TP_TOKEN_SHARD, to_exchange != 0,
                                        (cudaStream_t)stream));
}

tm_status tm_revert(const void* Hm, void* X, const tm_shape* shape, void* stream) {
    tm_status s = check_shape(shape);
    if (s != TM_OK) return s;
    if (!X || !Hm || X == Hm || !al_elem(X, shape->dtype) || !al_elem(Hm, shape->dtype)) return TM_ERR_INVALID_ARG;
    return cuda_status(launch_permute(shape->dtype, Hm, X, shape->B, shape->T, shape->D, shape->H, false,
                                      (cudaStream_t)stream));
}

tm_status tm_route_topk(const void* x, tm_layout layout, const tm_shape* shape, const void* norm_gain,
                        const tm_moe_w* w, int32_t* topk_idx, float* topk_gate, float* logit_gap_opt, float* inv_rms,
                        int32_t* bucket_offsets, int32_t* bucket_rows, int32_t* slot_of, void* workspace,
                        size_t workspace_bytes, void* stream) {
    Geo g;
    if (!w) return TM_ERR_INVALID_ARG;
    tm_status s = make_geo(shape, layout, w->banks, w->width, &g);
    if (s != TM_OK) return s;
    if ((s = check_moe(g, w)) != TM_OK) return s;
    if (!x || !al16(x) || !topk_idx || !topk_gate || !bucket_offsets || !bucket_rows || !slot_of)
        return TM_ERR_INVALID_ARG;
    if (norm_gain && !al16(norm_gain)) return TM_ERR_INVALID_ARG;
    if ((logit_gap_opt && (reinterpret_cast<uintptr_t>(logit_gap_opt) & 3)) ||
        (inv_rms && (reinterpret_cast<uintptr_t>(inv_rms) & 3)))
        return TM_ERR_INVALID_ARG;
    const size_t need = tm_route_workspace_bytes(shape, layout, w);
    if (!workspace || workspace_bytes < need || !al16(workspace)) return TM_ERR_WORKSPACE;
    Carve c{(uint8_t*)workspace};
    const int nchunks = (g.B + kRouterChunk - 1) / kRouterChunk;
    int32_t* counts = c.take<int32_t>((size_t)g.banks * nchunks * w->E);
    int32_t* tiles = c.take<int32_t>((size_t)g.banks * w->E + 1);
    RouteOut r{topk_idx, bucket_offsets, tiles, bucket_rows, slot_of, counts, topk_gate, inv_rms};
    r.gap = logit_gap_opt;
    const size_t split = route_split_bytes(g, w);
    r.wsplit = split ? c.take<uint8_t>(split) : nullptr;
    return run_route(g, x, norm_gain, w, r, (cudaStream_t)stream);
}

tm_status tm_pertoken_swiglu(const void* x, const void* residual, tm_layout layout, const tm_shape* shape,
                             const void* norm_gain, const tm_swiglu_w* w, void* y, void* workspace,
                             size_t workspace_bytes, void* stream) {
    tm_sublayer sub;
    memset(&sub, 0, sizeof(sub));
    if (!w) return TM_ERR_INVALID_ARG;
    sub.norm_gain = norm_gain;
    sub.is_moe = 0;
    sub.dense = *w;
    Geo g;
    tm_status s = check_sublayer(shape, layout, &sub, &g);
    if (s != TM_OK) return s;
    if (!x || !y || !al16(x) || !al16(y) || x == y || (residual && !al16(residual))) return TM_ERR_INVALID_ARG;
    return run_sublayer(g, x, residual, nullptr, &sub, y, workspace, workspace_bytes, (cudaStream_t)stream);
}

tm_status tm_sparse_pertoken_moe(const void* x, const void* residual, tm_layout layout, const tm_shape* shape,
                                 const void* norm_gain, const tm_moe_w* w, void* y, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    tm_sublayer sub;
    memset(&sub, 0, sizeof(sub));
    if (!w) return TM_ERR_INVALID_ARG;
    sub.norm_gain = norm_gain;
    sub.is_moe = 1;
    sub.moe = *w;
    Geo g;
    tm_status s = check_sublayer(shape, layout, &sub, &g);
    if (s != TM_OK) return s;
    if (!x || !y || !al16(x) || !al16(y) || x == y || (residual && !al16(residual))) return TM_ERR_INVALID_ARG;
    return run_sublayer(g, x, residual, nullptr, &sub, y, workspace, workspace_bytes, (cudaStream_t)stream);
}

tm_status tm_sublayer_forward(const void* x, const void* residual, const void* extra, tm_layout layout,
                              const tm_shape* shape, const tm_sublayer* sub, void* y, void* workspace,
                              size_t workspace_bytes, void* stream) {
    Geo g;
    tm_status s = check_sublayer(shape, layout, sub, &g);
    if (s != TM_OK) return s;
    if (!x || !y || !al16(x) || !al16(y) || x == y || (residual && !al16(residual))) return TM_ERR_INVALID_ARG;
    if (extra && (!al16(extra) || extra == y)) return TM_ERR_INVALID_ARG;
    return run_sublayer(g, x, residual, extra, sub, y, workspace, workspace_bytes, (cudaStream_t)stream);
}

tm_status tm_block_forward(const void* X, const tm_block* block, const tm_shape* shape, void* Y, void* X_revert_opt,
                           void* workspace, size_t workspace_bytes, void* stream) {
    bool ok = false;
    const size_t need = block ? stack_ws(shape, block, 1, 0, &ok) : 0;
    if (!ok) {
        Geo a, b;
        tm_status s = check_block(shape, block, &a, &b);
        return s == TM_OK ? TM_ERR_INVALID_ARG : s;
    }
    if (!X || !Y || X == Y || !al16(X) || !al16(Y) || (X_revert_opt && !al16(X_revert_opt))) return TM_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need || !al16(workspace)) return TM_ERR_WORKSPACE;
    Carve c{(uint8_t*)workspace};
    const size_t tok = (size_t)shape->B * shape->T * shape->D * (shape->dtype == TM_BF16 ? 2 : 4);
    void* xr = c.take<uint8_t>(tok);
    if (X_revert_opt) xr = X_revert_opt;
    c.off = align256(c.off);
    return run_block(shape, block, X, nullptr, Y, xr, (uint8_t*)workspace + c.off, workspace_bytes - c.off,
                     (cudaStream_t)stream);
}

tm_status tm_stack_step(const void* X, const void* X_skip, const tm_block* block, const tm_shape* shape, void* Y,
                        void* X_revert_opt, void* workspace, size_t workspace_bytes, void* stream) {
    bool ok = false;
    const size_t need = block ? stack_ws(shape, block, 1, 0, &ok) : 0;
    if (!ok) {
        Geo a, b;
        tm_status s = check_block(shape, block, &a, &b);
        return s == TM_OK ? TM_ERR_INVALID_ARG : s;
    }
    if (!X || !Y || X == Y || !al16(X) || !al16(Y) || (X_revert_opt && !al16(X_revert_opt))) return TM_ERR_INVALID_ARG;
    if (X_skip && (!al16(X_skip) || X_skip == Y || X_skip == X_revert_opt)) return TM_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need || !al16(workspace)) return TM_ERR_WORKSPACE;
    Carve c{(uint8_t*)workspace};
    const size_t tok = (size_t)shape->B * shape->T * shape->D * (shape->dtype == TM_BF16 ? 2 : 4);
    void* xr = c.take<uint8_t>(tok);
    if (X_revert_opt) xr = X_revert_opt;
    c.off = align256(c.off);
    return run_block(shape, block, X, X_skip, Y, xr, (uint8_t*)workspace + c.off, workspace_bytes - c.off,
                     (cudaStream_t)stream);
}

tm_status tm_stack_forward(const void* X, const tm_block* blocks, int L, int gap, const tm_shape* shape, void* Y,
                           void* workspace, size_t workspace_bytes, void* stream) {
    if (!blocks || L < 1 || gap < 0) return TM_ERR_INVALID_ARG;
    bool ok = false;
    const size_t need = stack_ws(shape, blocks, L, gap, &ok);
    if (!ok) {
        for (int l = 0; l < L; ++l) {
            Geo a, b;
            tm_status s = check_block(shape, &blocks[l], &a, &b);
            if (s != TM_OK) return s;
        }
        return TM_ERR_INVALID_ARG;
    }
    if (!X || !Y || X == Y || !al16(X) || !al16(Y)) return TM_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need || !al16(workspace)) return TM_ERR_WORKSPACE;
    const size_t tok = (size_t)shape->B * shape->T * shape->D * (shape->dtype == TM_BF16 ? 2 : 4);
    Carve c{(uint8_t*)workspace};
    void* xr = c.take<uint8_t>(tok);
    const int R = L > 1 ? (gap > 0 ? gap + 1 : 2) : 0;
    void* ring[64];
    if (R > 64) return TM_ERR_UNSUPPORTED;
    for (int i = 0; i < R; ++i) ring[i] = c.take<uint8_t>(tok);
    c.off = align256(c.off);
    void* sub_ws = (uint8_t*)workspace + c.off;
    const size_t sub_wsb = workspace_bytes - c.off;
    cudaStream_t st = (cudaStream_t)stream;
    // X_l for l >= 1 lives in ring[l % R] (the last one in Y); X_0 is the caller's X
    auto xl = [&](int l) -> const void* { return l == 0 ? X : (l == L ? Y : ring[l % R]); };
    for (int l = 1; l <= L; ++l) {
        const void* in = xl(l - 1);
        void* out = l == L ? Y : ring[l % R];
        const void* extra = (gap > 0 && l % gap == 0 && l < L) ? xl(l - gap) : nullptr;
        tm_status s = run_block(shape, &blocks[l - 1], in, extra, out, xr, sub_ws, sub_wsb, st);
        if (s != TM_OK) return s;
    }
    return TM_OK;
}

tm_status tm_quantize_fp8_weights(const void* w, const void* gain, int groups, size_t rows, int cols, uint8_t* q,
                                  float* scale, void* stream) {
    if (!w || !q || !scale || groups <= 0 || rows == 0 || cols <= 0 || (rows * cols) % 2) return TM_ERR_INVALID_ARG;
    if (!al16(w) || !al16(q) || (gain && !al16(gain)) || (reinterpret_cast<uintptr_t>(scale) & 3)) return TM_ERR_INVALID_ARG;
    return cuda_status(launch_quant_matrices(w, gain, groups, rows * (size_t)cols, cols, q, scale, (cudaStream_t)stream));
}

tm_status tm_quantize_fp8_act(const void* x, tm_layout layout, const tm_shape* shape, int banks, int width, uint8_t* q,
                              float* rowscale, void* stream) {
    Geo g;
    tm_status s = make_geo(shape, layout, banks, width, &g);
    if (s != TM_OK) return s;
    if (!x || !q || !rowscale || !al16(x) || !al16(q) || (reinterpret_cast<uintptr_t>(rowscale) & 3))
        return TM_ERR_INVALID_ARG;
    if (g.dtype != TM_BF16 || g.W > 1024 || (g.map.layout == 1 && g.map.dh % 8)) return TM_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_act_rows(x, g.map, g.B, g.eps, q, rowscale, (cudaStream_t)stream));
}

size_t tm_sublayer_fp8_workspace_bytes(const tm_shape* shape, tm_layout layout, const tm_sublayer8* sub) {
    Geo g;
    if (check_sublayer8(shape, layout, sub, &g) != TM_OK) return 0;
    if (!sub->is_moe) return 256;
    Carve c{nullptr};
    carve_moe8(c, g, &sub->moe);
    return align256(c.off);
}

tm_status tm_sublayer_forward_fp8(const void* x, const void* residual, const void* extra, tm_layout layout,
                                  const tm_shape* shape, const tm_sublayer8* sub, void* y, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    Geo g;
    tm_status s = check_sublayer8(shape, layout, sub, &g);
    if (s != TM_OK) return s;
    if (!x || !y || !al16(x) || !al16(y) || x == y || (residual && (!al16(residual) || residual == y)))
        return TM_ERR_INVALID_ARG;
    if (extra && (!al16(extra) || extra == y)) return TM_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    if (sub->is_moe) return run_moe8(g, x, residual, extra, sub->norm_gain, &sub->moe, y, workspace, workspace_bytes, st);
    return run_dense8(g, x, residual, extra, &sub->dense, y, st);
}

tm_status tm_sparse_pertoken_moe_fp8(const void* x, const void* residual, tm_layout layout, const tm_shape* shape,
                                     const void* norm_gain, const tm_moe_w8* w, void* y, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    if (!w) return TM_ERR_INVALID_ARG;
    tm_sublayer8 sub;
    memset(&sub, 0, sizeof(sub));
    sub.norm_gain = norm_gain;
    sub.is_moe = 1;
    sub.moe = *w;
    return tm_sublayer_forward_fp8(x, residual, nullptr, layout, shape, &sub, y, workspace, workspace_bytes, stream);
}

size_t tm_pertoken_swiglu_fp8_workspace_bytes(const tm_shape* shape, tm_layout layout, const tm_swiglu_w8* w) {
    Geo g;
    if (!w || make_geo(shape, layout, w->banks, w->width, &g) != TM_OK || check_dense8(g, w) != TM_OK) return 0;
    return 256;   // nothing is needed; a minimal size keeps the workspace convention of the ABI
}

tm_status tm_pertoken_swiglu_fp8(const void* x, const void* residual, tm_layout layout, const tm_shape* shape,
                                 const tm_swiglu_w8* w, void* y, void* workspace, size_t workspace_bytes, void* stream) {
    Geo g;
    if (!w) return TM_ERR_INVALID_ARG;
    tm_status s = make_geo(shape, layout, w->banks, w->width, &g);
    if (s != TM_OK) return s;
    if ((s = check_dense8(g, w)) != TM_OK) return s;
    if (!x || !y || x == y || !al16(x) || !al16(y) || (residual && !al16(residual))) return TM_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < 256 || !al16(workspace)) return TM_ERR_WORKSPACE;
    return run_dense8(g, x, residual, nullptr, w, y, (cudaStream_t)stream);
}

size_t tm_block_fp8_workspace_bytes(const tm_shape* shape, const tm_block_fp8* block) {
    Geo gm, gr;
    if (check_block8(shape, block, &gm, &gr) != TM_OK) return 0;
    return block8_ws(gm, gr, shape);
}

tm_status tm_block_forward_fp8(const void* X, const tm_block_fp8* block, const tm_shape* shape, void* Y,
                               void* X_revert_opt, void* workspace, size_t workspace_bytes, void* stream) {
    Geo gm, gr;
    tm_status s = check_block8(shape, block, &gm, &gr);
    if (s != TM_OK) return s;
    if (!X || !Y || X == Y || !al16(X) || !al16(Y) || (X_revert_opt && !al16(X_revert_opt))) return TM_ERR_INVALID_ARG;
    const size_t need = block8_ws(gm, gr, shape);
    if (!workspace || workspace_bytes < need || !al16(workspace)) return TM_ERR_WORKSPACE;
    Carve c{(uint8_t*)workspace};
    void* xr = c.take<uint8_t>((size_t)shape->B * shape->T * shape->D * 2);
    unsigned* dep = c.take<unsigned>((size_t)(gm.B + 127) / 128);
    if (X_revert_opt) xr = X_revert_opt;
    cudaStream_t st = (cudaStream_t)stream;
    if (block8_fusable(gm, gr, Y, xr)) return fused_block8(block, gm, gr, X, Y, xr, dep, st);
    // H_next = FFN_mix(Norm(Mix(X))) + Mix(X) through Revert into X_rev; Y = FFN_rev(Norm(X_rev)) + X
    if ((s = run_dense8(gm, X, X, nullptr, &block->mix, xr, st)) != TM_OK) return s;
    return run_dense8(gr, xr, X, nullptr, &block->rev, Y, st);
}

size_t tm_pertoken_swiglu_backward_workspace_bytes(const tm_shape* shape, tm_layout layout, const tm_swiglu_w* w) {
    Geo g;
    if (!w || make_geo(shape, layout, w->banks, w->width, &g) != TM_OK || check_dense_bwd(g, w, nullptr) != TM_OK)
        return 0;
    return dense_bwd_ws(g, w->hidden);
}

tm_status tm_pertoken_swiglu_backward(const void* x, const void* dy, const void* dx_add, tm_layout layout,
                                      const tm_shape* shape, const void* norm_gain, const tm_swiglu_w* w, void* dx,
                                      const tm_swiglu_grads* grads, void* workspace, size_t workspace_bytes,
                                      void* stream) {
    if (!w) return TM_ERR_INVALID_ARG;
    Geo g;
    tm_status s = make_geo(shape, layout, w->banks, w->width, &g);
    if (s != TM_OK) return s;
    if (norm_gain && !al16(norm_gain)) return TM_ERR_INVALID_ARG;
    if ((s = check_dense_bwd(g, w, norm_gain)) != TM_OK) return s;
    if (!x || !dy || !dx || !al16(x) || !al16(dy) || !al16(dx) || (dx_add && !al16(dx_add)) || dx == x || dx == dy ||
        !grads_ok(grads))
        return TM_ERR_INVALID_ARG;
    return run_dense_bwd(g, x, dy, dx_add, nullptr, nullptr, w, dx, grads->dw_gate, grads->dw_up, grads->dw_down, workspace,
                         workspace_bytes, (cudaStream_t)stream);
}

size_t tm_block_backward_workspace_bytes(const tm_shape* shape, const tm_block* block) {
    Geo gm, gr;
    if (!block || check_block_bwd(shape, block, &gm, &gr) != TM_OK) return 0;
    const size_t tok = align256((size_t)shape->B * shape->T * shape->D * 2);
    return 2 * tok + block_bwd_sub_ws(gm, gr, block);
}

tm_status tm_block_backward(const void* X, const void* dY, const tm_block* block, const tm_shape* shape, void* dX,
                            const tm_block_grads* grads, void* workspace, size_t workspace_bytes, void* stream) {
    Geo gm, gr;
    if (!block) return TM_ERR_INVALID_ARG;
    tm_status s = check_block_bwd(shape, block, &gm, &gr);
    if (s != TM_OK) return s;
    if (!X || !dY || !dX || !al16(X) || !al16(dY) || !al16(dX) || dX == X || dX == dY || !grads ||
        !grads_ok(&grads->mix) || !grads_ok(&grads->rev))
        return TM_ERR_INVALID_ARG;
    const size_t tok = align256((size_t)shape->B * shape->T * shape->D * 2);
    const size_t sub = block_bwd_sub_ws(gm, gr, block);
    if (!workspace || workspace_bytes < 2 * tok + sub || !al16(workspace)) return TM_ERR_WORKSPACE;
    uint8_t* base = (uint8_t*)workspace;
    return run_block_bwd(gm, gr, block, X, dY, nullptr, dX, grads, base, base + tok, base + 2 * tok, sub,
                         (cudaStream_t)stream);
}

size_t tm_stack_backward_workspace_bytes(const tm_shape* shape, const tm_block* blocks, int L, int gap) {
    if (!blocks || L < 1 || gap < 0) return 0;
    size_t sub = 0;
    for (int l = 0; l < L; ++l) {
        Geo gm, gr;
        if (check_block_bwd(shape, &blocks[l], &gm, &gr) != TM_OK) return 0;
        // the block backward's region, and the one a block forward (run_block) needs
        const size_t n[4] = {block_bwd_sub_ws(gm, gr, &blocks[l]), sublayer_ws(gm, &blocks[l].mix),
                             sublayer_ws(gr, &blocks[l].rev), block_ws(gm, gr, &blocks[l])};
        for (size_t v : n) sub = v > sub ? v : sub;
    }
    const size_t tok = align256((size_t)shape->B * shape->T * shape->D * 2);
    return tok * (2 + 2 * (size_t)(L - 1)) + sub;
}

tm_status tm_stack_backward(const void* X, const void* dY, const tm_block* blocks, int L, int gap,
                            const tm_shape* shape, void* dX, const tm_block_grads* grads, void* workspace,
                            size_t workspace_bytes, void* stream) {
    if (!blocks || L < 1 || gap < 0 || !grads) return TM_ERR_INVALID_ARG;
    Geo gm[64], gr[64];
    if (L > 64) return TM_ERR_UNSUPPORTED;
    for (int l = 0; l < L; ++l) {
        tm_status s = check_block_bwd(shape, &blocks[l], &gm[l], &gr[l]);
        if (s != TM_OK) return s;
        if (!grads_ok(&grads[l].mix) || !grads_ok(&grads[l].rev)) return TM_ERR_INVALID_ARG;
    }
    if (!X || !dY || !dX || !al16(X) || !al16(dY) || !al16(dX) || dX == X || dX == dY) return TM_ERR_INVALID_ARG;
    const size_t need = tm_stack_backward_workspace_bytes(shape, blocks, L, gap);
    if (need == 0) return TM_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < need || !al16(workspace)) return TM_ERR_WORKSPACE;
    const size_t tok = align256((size_t)shape->B * shape->T * shape->D * 2);
    uint8_t* base = (uint8_t*)workspace;
    void* Xr = base;
    void* dXr = base + tok;
    // xs[l] = X_l (l = 1 .. L-1), gs[l] = the gradient of X_l (l = 1 .. L-1)
    uint8_t* xs = base + 2 * tok;
    uint8_t* gs = xs + (size_t)(L - 1) * tok;
    void* ws = gs + (size_t)(L - 1) * tok;
    const size_t wsb = workspace_bytes - (size_t)((uint8_t*)ws - base);
    auto xl = [&](int l) -> const void* { return l == 0 ? X : (const void*)(xs + (size_t)(l - 1) * tok); };
    auto gl = [&](int l) -> void* { return l == 0 ? dX : (l == L ? const_cast<void*>(dY) : (void*)(gs + (size_t)(l - 1) * tok)); };
    cudaStream_t st = (cudaStream_t)stream;
    tm_status s;
    // the forward again, keeping every block input: X_l = Block_l(X_{l-1}) (+ X_{l-gap}), as
    // tm_stack_forward computes it
    for (int l = 1; l < L; ++l) {
        const void* extra = (gap > 0 && l % gap == 0 && l < L) ? xl(l - gap) : nullptr;
        if ((s = run_block(shape, &blocks[l - 1], xl(l - 1), extra, (void*)xl(l), Xr, ws, wsb, st)) != TM_OK) return s;
    }
    // backward, last block first: the gradient of X_{l-1} is block l's input gradient plus, when
    // X_{l-1+gap} = Block(...) + X_{l-1} (an inter-residual), the gradient of X_{l-1+gap}
    for (int l = L; l >= 1; --l) {
        const int j = l - 1 + gap;
        const void* extra = (gap > 0 && j % gap == 0 && j < L) ? gl(j) : nullptr;
        if ((s = run_block_bwd(gm[l - 1], gr[l - 1], &blocks[l - 1], xl(l - 1), gl(l), extra, gl(l - 1), &grads[l - 1],
                               Xr, dXr, ws, wsb, st)) != TM_OK)
            return s;
    }
    return TM_OK;
}

static unsigned g_last_site = 0;   // site of the last device error tm_get_device_error returned

unsigned tm_last_device_error_site(void) { return g_last_site; }

tm_status tm_get_device_error(void* stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) { note_cuda_error("tm_get_device_error: stream synchronize", e); return TM_ERR_CUDA; }
    unsigned int h[2] = {0, 0};
    e = cudaMemcpyFromSymbol(h, g_error, sizeof(h));
    if (e != cudaSuccess) { note_cuda_error("tm_get_device_error: read error word", e); return TM_ERR_CUDA; }
    g_last_site = h[0] ? h[1] : 0u;
    if (h[0] == 0) return TM_OK;
    char where[64];
    snprintf(where, sizeof(where), "device error %u at site 0x%x", h[0], h[1]);
    note_cuda_error(where, cudaErrorUnknown);
    const unsigned int z[2] = {0, 0};
    e = cudaMemcpyToSymbol(g_error, z, sizeof(z));
    if (e != cudaSuccess) { note_cuda_error("tm_get_device_error: clear error word", e); return TM_ERR_CUDA; }
    return h[0] == ERR_TIMEOUT ? TM_ERR_DEVICE_TIMEOUT : TM_ERR_DEVICE_BOUNDS;
}

tm_status tm_set_wait_limit_ns(uint64_t ns) {
    if (ns < 1000ull || ns > 60000000000ull) return TM_ERR_INVALID_ARG;
    const unsigned long long v = ns;
    cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
    if (e != cudaSuccess) { note_cuda_error("tm_set_wait_limit_ns", e); return TM_ERR_CUDA; }
    return TM_OK;
}

tm_status tm_selftest_wait(uint64_t* result_opt, void* stream) {
    if (result_opt && (reinterpret_cast<uintptr_t>(result_opt) & 7)) return TM_ERR_INVALID_ARG;
    return cuda_status(launch_wait_selftest(reinterpret_cast<unsigned long long*>(result_opt), (cudaStream_t)stream));
}

tm_status tm_selftest_bucket_scatter(const int32_t* topk_idx, const int32_t* chunk_prefix, const int32_t* bucket_offsets,
                                     int B, int banks, int E, int k, int32_t* bucket_rows, int capacity,
                                     int32_t* slot_of, void* stream) {
    if (!topk_idx || !chunk_prefix || !bucket_offsets || !bucket_rows || !slot_of) return TM_ERR_INVALID_ARG;
    if (B <= 0 || banks <= 0 || E < 1 || k < 1 || k > E || capacity < 0) return TM_ERR_INVALID_ARG;
    if (E > 64 || k > 8) return TM_ERR_UNSUPPORTED;
    return cuda_status(launch_scatter(topk_idx, chunk_prefix, bucket_offsets, B, banks, E, k, bucket_rows, slot_of,
                                      (cudaStream_t)stream, nullptr, nullptr, nullptr, nullptr, nullptr, capacity));
}

}  // extern "C"
