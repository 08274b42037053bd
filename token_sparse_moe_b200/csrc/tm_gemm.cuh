// tm_gemm.cuh -- the grouped bf16 GEMM on tcgen05 tensor cores that carries every
// per-token FFN of the TokenMixer-Large forward.
//
// One persistent kernel shape serves four jobs, chosen at compile time:
//   EPI_SWIGLU : hidden = silu(s * A Wg^T) * (s * A Wu^T)   (GEMM1 of a SwiGLU bank,
//                s = per-row 1/rms, i.e. the pre-RMSNorm folded into the epilogue)
//   EPI_RESID  : y = A Wd^T + residual (+ inter-residual), stored through the row map
//                (for mixed rows this store IS the Revert permutation)
//   EPI_SLOT   : plain rows out = A B^T (bf16), staged and bulk-stored (the backward's contractions)
//   EPI_COMBINE: y = A Ws^T + sum_j gate_j * slot_j + residual (+ inter-residual):
//                shared expert GEMM2 plus the MoE combine, in fixed order
// A operand sources: a plain 2-D TMA map (hidden rows), a 3-D TMA map over
// [B, banks, W] rows, a 4-D TMA map that reads mixed rows straight out of the token
// tensor (Mix folded into the tensor map: each 16-column piece of a mixed row is a
// 32-byte run of one token, fetched as a 128-row box with 32-byte swizzle), or a
// cp.async row gather (routed rows).
//
// Output: GEMM1 hidden rows and the combine's rows go out through bulk tensor stores (tmO: the
// hidden rows with 32 x 64 boxes, or the row / Revert geometry of y), one 4 KB box per epilogue
// warp staged in shared memory; the routed GEMM2's sample-order rows are scattered, so they are
// staged the same way and written by the warp four whole 128-byte row pieces per instruction.
//
// Tile: 128 rows x BN columns, K in 64-wide slabs with 128-byte swizzle.  Warp roles:
// warp 0 TMA producer, warp 1 MMA issuer (one thread) and TMEM owner, warps 2-5
// epilogue (TMEM lane quarter = warp % 4), warps 6-9 row gatherers (gather mode).
// TMEM holds two accumulators so the epilogue of tile i overlaps the MMAs of i+1.
//
// Pair mode (PAIR, groups of equal rows): a cluster of two CTAs on two SMs works on 256 rows of one
// group; each CTA loads its own 128 A rows and half of the BN weight rows (GEMM1: the leader the
// gate rows, the peer the up rows; otherwise the two halves of the N tile), and the leader issues one
// tcgen05.mma.cta_group::2 (M = 256) per K step, so each SM streams half the weight bytes of a
// 128-row tile.  Both CTAs' loads complete on the leader's stage barriers; the leader's commits
// arrive on the barriers of both CTAs; each CTA's epilogue reads its own accumulator rows and
// arrives on the leader's accumulator-free barrier.  No load and no commit uses multicast.
#pragma once
#include "tm_device.cuh"

namespace tml {

enum AMode : int { A_TMA_2D = 0, A_TMA_3D = 1, A_TMA_MIX = 2, A_GATHER = 3 };
// EPI_SLOT_PERM: routed GEMM2 rows written in combine order (row perm[pos] = (bank * k + j) * B + b)
// and scaled by their gate.
// EPI_SUM: the combine with its sources (residual, inter-residual, the k gate-scaled expert rows of
// each sample) added on the tensor core before the shared expert's GEMM2; plain output epilogue.
// EPI_ROUTE: the router on the tensor core; B holds each fp32 router row split exactly into three
// bf16 rows (hi, mid, lo), the accumulator's columns e, E+e, 2E+e add up to the fp32 logit; four
// extra warps take each row's sum of squares from the A stages as they pass; the epilogue does
// the scale, softmax, top-k, gates and the per-chunk expert counts.
// EPI_SWIGLU_NORM: EPI_SWIGLU with the pre-RMSNorm's row statistics taken in the kernel: four extra
// warps sum each row's squares from the A stages as they pass (as for EPI_ROUTE), the epilogue
// scales by 1/sqrt(sum / K + eps) (dense groups of rows read through a 3-D or Mix map).
enum Epi : int { EPI_SWIGLU = 0, EPI_RESID = 1, EPI_SLOT = 2, EPI_COMBINE = 3, EPI_SLOT_PERM = 4, EPI_SUM = 5,
                 EPI_ROUTE = 6, EPI_SWIGLU_NORM = 7 };
constexpr int kRouteMaxE = 21;   // 3 * E <= 64 accumulator columns

// Where element c of the row (sample b, bank) of a sub-layer lives in a tensor.
//   layout 0 (rows):  [B, banks, W]
//   layout 1 (mixed): token tensor [B, T, D]; c = t*dh + j  ->  [b, t, bank*dh + j]
struct RowMap {
    int layout, banks, W, T, D, dh;
};
__host__ __device__ __forceinline__ size_t row_elem(const RowMap& m, int b, int bank, int c) {
    if (m.layout == 0) return ((size_t)b * m.banks + bank) * m.W + c;
    const int t = c / m.dh;
    const int j = c - t * m.dh;
    return ((size_t)b * m.T + t) * m.D + (size_t)bank * m.dh + j;
}

struct GemmParams {
    // tile space
    int sched;                 // 0: groups of `rows` rows (dense banks); 1: bucketed (routed experts)
    int bank_chunk;            // sched 0: banks per chunk of the tile order (0: all); see decode_tile
    int groups;                // number of groups (sched 1: banks * E)
    int rows;                  // sched 0: rows per group (= B)
    int banks;                 // sub-layer banks
    int E;                     // sched 1: experts per bank (bank = g / E)
    const int* row_start;      // sched 1: [groups+1] first row position of each group
    const int* tile_start;     // sched 1: [groups+1] prefix of 128-row tiles per group
    const int4* tile_info;     // sched 1: per 128-row tile {group, first row position, rows, tile in group}
    const int* bucket_rows;    // sched 1: sample index of each row position
    const float* pos_scale;    // sched 1 (optional): per row position, 1/rms (EPI_SWIGLU) or gate (EPI_SLOT_PERM)
    int pos_limit;             // row positions in hidden / slot buffers (bounds check)
    size_t out_elems;          // elements of `out` (and of resid / extra for the row-map epilogues)
    int K, N, n_tiles;         // reduction length, output columns per group, N / BN
    // gathered A
    const __nv_bfloat16* a_ptr;
    RowMap amap;
    // epilogue
    const float* inv_rms;      // [B * banks]
    __nv_bfloat16* out;        // hidden / slot rows [row positions, out_ld] or y (omap)
    int out_ld;
    const __nv_bfloat16* resid;
    const __nv_bfloat16* extra;
    RowMap omap;
    const float* gate;         // combine: [B, banks, k]
    const int* slot_of;        // combine: [B, banks, k]
    const __nv_bfloat16* slots;// combine: [row positions, W]
    int k;
    const int* perm;           // EPI_SLOT_PERM: combine-order row (bank * k + j) * B + b of each position
    int src_resid, src_extra;  // EPI_SUM: residual / inter-residual present (maps tmS0 / tmS1)
    int src_mix;               // EPI_SUM: residual maps use the 4-D mixed geometry (16-column boxes)
    // EPI_ROUTE outputs ([B, banks, k] rows of top-k, [B, banks] 1/rms, [banks][chunks][E] counts)
    int32_t* r_idx;
    float* r_gate;
    float* r_inv_rms;
    float* r_gap;              // optional [B, banks]: logit gap z_(k) - z_(k+1) (+inf when k == E)
    int32_t* r_counts;
    int r_nchunks;
    float r_alpha, r_eps;
    // F8 (E4M3 GEMM1): the gate / up weight matrices' scales, one per group
    const float* w8_sgate;
    const float* w8_sup;
};

template <int BN, int AMODE, int EPI = EPI_SWIGLU, bool PAIR = false, bool F8 = false>
struct GemmCfg {
    static constexpr int BM = 128, BK = 64;
    // K elements per 128-byte slab row: 64 bf16, or 128 E4M3 codes (F8: GEMM1 on kind::f8f6f4)
    static constexpr int KSLAB = F8 ? 128 : 64;
    static_assert(!F8 || (EPI == EPI_SWIGLU && !PAIR && (AMODE == A_TMA_2D || AMODE == A_TMA_3D)),
                  "the E4M3 mode covers GEMM1 with plain row maps");
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * BK * 2;   // this CTA's weight rows of a stage
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // the scattered-row epilogue is latency-bound per warp: two warps per TMEM lane quarter, each
    // taking half of the tile's columns
    static constexpr int EPI_WARPS = (EPI == EPI_SLOT_PERM && BN % 128 == 0) ? 8 : 4;
    static constexpr int STG_BYTES_ = (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_NORM || EPI == EPI_SLOT_PERM ||
                                       EPI == EPI_SUM || EPI == EPI_SLOT)
                                          ? EPI_WARPS * 4096 : 0;
    // the row-statistics warps (6-9) of the router and of GEMM1 with the norm in the kernel
    static constexpr bool STATS = EPI == EPI_ROUTE || EPI == EPI_SWIGLU_NORM;
    static_assert(!(PAIR && STATS), "the statistics warps wait on this CTA's own stage barriers, which the "
                                    "pair-mode loads (completing on the leader's) never complete");
    // pair mode: as many stages as the shared memory holds, at most 8
    static constexpr int PAIR_STAGES_ = (232448 - 2304 - STG_BYTES_) / STAGE_BYTES;
    static constexpr int STAGES = PAIR ? (PAIR_STAGES_ > 8 ? 8 : PAIR_STAGES_)
                                       : (BN >= 256 ? 4 : (BN >= 192 ? (EPI_WARPS == 8 ? 4 : 5) : 6));
    static_assert(!PAIR || (AMODE != A_GATHER && EPI != EPI_ROUTE && EPI != EPI_RESID && EPI != EPI_COMBINE),
                  "pair mode covers tensor-map A operands and the staged epilogues");
    static constexpr int NWARPS = (AMODE == A_GATHER || STATS) ? 10 : 2 + EPI_WARPS;
    static_assert(EPI != EPI_SWIGLU_NORM || AMODE == A_TMA_3D || AMODE == A_TMA_MIX,
                  "in-kernel row statistics read rows through a 3-D or Mix map");
    static constexpr int NTHREADS = NWARPS * 32;
    static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
    // output staging: one 32-row x 64-column bf16 box (4 KB) per epilogue warp
    static constexpr bool STAGED =
        EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_NORM || EPI == EPI_SLOT_PERM || EPI == EPI_SUM || EPI == EPI_SLOT;
    static constexpr int OFF_STG = STAGES * STAGE_BYTES;
    static constexpr int STG_BYTES = STAGED ? EPI_WARPS * 4096 : 0;
    static constexpr int OFF_ID = OFF_STG + STG_BYTES;             // 16 x 16 identity (EPI_SUM), 1 KB
    static constexpr int SMEM_BYTES = OFF_ID + 1024 + 1024 + 256;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct TileInfo {
    int g, m, n, row0, nrows;
};

__device__ __forceinline__ int total_tiles(const GemmParams& p) {
    if (p.sched == 0) return p.groups * ((p.rows + 127) / 128) * p.n_tiles;
    return __ldg(&p.tile_start[p.groups]) * p.n_tiles;
}

// Pair mode (groups of equal rows, sched 0): tiles of 256 rows, two CTAs' 128-row halves.
__device__ __forceinline__ int total_tiles_pair(const GemmParams& p) {
    return p.groups * ((p.rows + 255) / 256) * p.n_tiles;
}

// This CTA's 128-row half (rank 0: the first) of 256-row tile t, in decode_tile's order (bank chunks,
// row block major inside a chunk); a half past the group's end has nrows = 0 (its rows are loaded,
// multiplied and never stored).
__device__ __forceinline__ TileInfo decode_tile_pair(const GemmParams& p, int t, int rank) {
    TileInfo ti;
    const int gm = t / p.n_tiles;
    ti.n = t - gm * p.n_tiles;
    const int mt2 = (p.rows + 255) / 256;
    const int cb = (p.bank_chunk > 0 && p.bank_chunk < p.groups) ? p.bank_chunk : p.groups;
    const int c = gm / (cb * mt2);
    const int rr = gm - c * cb * mt2;
    const int g0 = c * cb, nb = min(cb, p.groups - g0);
    const int m2 = rr / nb;
    ti.g = g0 + (rr - m2 * nb);
    ti.m = 2 * m2 + rank;
    ti.row0 = ti.g * p.rows + ti.m * 128;
    ti.nrows = max(0, min(128, p.rows - ti.m * 128));
    return ti;
}

__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, int t) {
    TileInfo ti;
    const int gm = t / p.n_tiles;
    ti.n = t - gm * p.n_tiles;
    if (p.sched == 0) {
        // chunks of banks whose weights fit in the L2 together, in turn; inside a chunk row block
        // major with the banks innermost: the CTAs running side by side read the same samples'
        // token rows (whole sectors when a bank's segment of a row is short, as with the Mix map)
        // while the chunk's weights stay in the L2 from one row block to the next
        const int mt = (p.rows + 127) / 128;
        const int cb = (p.bank_chunk > 0 && p.bank_chunk < p.groups) ? p.bank_chunk : p.groups;
        const int c = gm / (cb * mt);
        const int rr = gm - c * cb * mt;
        const int g0 = c * cb, nb = min(cb, p.groups - g0);
        ti.m = rr / nb;
        ti.g = g0 + (rr - ti.m * nb);
        ti.row0 = ti.g * p.rows + ti.m * 128;
        ti.nrows = min(128, p.rows - ti.m * 128);
    } else if (p.tile_info) {
        const int4 d = __ldg(&p.tile_info[gm]);
        ti.g = d.x;
        ti.row0 = d.y;
        ti.nrows = d.z;
        ti.m = d.w;
    } else {
        int lo = 0, hi = p.groups;   // invariant: tile_start[lo] <= gm < tile_start[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(&p.tile_start[mid]) <= gm) lo = mid; else hi = mid;
        }
        ti.g = lo;
        ti.m = gm - __ldg(&p.tile_start[lo]);
        ti.row0 = __ldg(&p.row_start[lo]) + ti.m * 128;
        ti.nrows = min(128, __ldg(&p.row_start[lo + 1]) - ti.row0);
    }
    return ti;
}

// The same wait with cluster-scope acquire: for barriers that the other CTA of a pair (its loads,
// commits or arrivals) completes.
__device__ __forceinline__ bool wait_or_abort_cl(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                 unsigned where) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns(), lim = wait_limit_ns();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > lim) {
            record_error(ERR_TIMEOUT, where);
            *abort_flag = 1;
            return false;
        }
    }
}

// Bounded wait that also gives up as soon as another role of the CTA has given up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns(), lim = wait_limit_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > lim) {
            record_error(ERR_TIMEOUT, where);
            *abort_flag = 1;
            return false;
        }
    }
}

template <int BN, int AMODE, int EPI, bool PAIR, bool F8>
__global__ void __launch_bounds__(GemmCfg<BN, AMODE, EPI, PAIR, F8>::NTHREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmS0,
                        const __grid_constant__ CUtensorMap tmS1, const __grid_constant__ CUtensorMap tmS2,
                        const __grid_constant__ CUtensorMap tmO, const GemmParams p) {
    using C = GemmCfg<BN, AMODE, EPI, PAIR, F8>;
    constexpr int STAGES = C::STAGES;
    constexpr int KSLAB = C::KSLAB;
    // pair mode: the two CTAs of a cluster share the tile sequence (cluster index cid), each taking
    // its 128-row half; both return here together, so both reach the closing cluster barrier
    const int rank = PAIR ? (int)cluster_ctarank() : 0;
    const bool leader = rank == 0;
    const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int ncid = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int ntile = PAIR ? total_tiles_pair(p) : total_tiles(p);
    if (cid >= ntile) return;
    auto dec = [&](int t) -> TileInfo { return PAIR ? decode_tile_pair(p, t, rank) : decode_tile(p, t); };
    // EPI_SUM source stages per tile: residual, inter-residual, then expert choice j = 0..k-1, each
    // as BN / 64 slabs of 128 rows x 64 columns (one ring stage each, A part only)
    const int n_src = EPI == EPI_SUM ? (p.src_resid + p.src_extra + p.k) : 0;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sI = smem + C::OFF_ID;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_ID + 1024);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* st_full = drain + 1;         // [2] statistics warps: row sums of squares of a tile written
    uint64_t* st_empty = st_full + 2;      // [2] ... and read by the epilogue
    float* ssbuf = reinterpret_cast<float*>(sI);   // statistics: [2][128] (the identity slot is unused)
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(st_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int KB = p.K / KSLAB;
    // pair mode: the leader's copy (L) and the peer's copy (P) of a barrier of this CTA's layout
    auto L = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 0); };
    auto P = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 1); };
    // waits on barriers that the other CTA of a pair completes take cluster-scope acquire
    auto wait = [&](uint64_t* b, uint32_t par, unsigned where) -> bool {
        return PAIR ? wait_or_abort_cl(b, par, abort_flag, where) : wait_or_abort(b, par, abort_flag, where);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], AMODE == A_GATHER ? 1 + 128 : 1);
            mbar_init(&empty[s], C::STATS ? 1 + 4 : 1);   // + the four statistics warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], C::EPI_WARPS * (PAIR ? 2 : 1));   // pair: both CTAs' epilogue warps
        }
        mbar_init(drain, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&st_full[b], 4);
            mbar_init(&st_empty[b], 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (EPI == EPI_SUM && warp == 0) {
        // identity B operand: 16 rows n x 16 columns k, 32-byte rows, 32-byte swizzle (the 16-byte
        // half of row n that holds column k sits at half (k / 8) ^ ((n / 4) % 2)).  Pair mode: the N
        // rows are split between the CTAs, so this CTA holds identity rows n = 8 rank + i as its
        // local rows i = 0..7.
        const int i = lane & 15, hf = lane >> 4;
        const int n = PAIR ? 8 * rank + (i & 7) : i;
        const uint32_t one = (PAIR && i >= 8) ? 0u : ((n >> 3) == hf ? ((n & 1) ? 0x3F800000u : 0x00003F80u) : 0u);
        const int wi = (n & 7) >> 1;
        *reinterpret_cast<uint4*>(sI + i * 32 + ((hf ^ ((i >> 2) & 1)) << 4)) =
            make_uint4(wi == 0 ? one : 0u, wi == 1 ? one : 0u, wi == 2 ? one : 0u, wi == 3 ? one : 0u);
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(tmem_base_smem, C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_base_smem, C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if (PAIR) cluster_sync_all();            // both CTAs' barriers exist before any remote use
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            if (AMODE != A_GATHER) tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB0);
            if (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_NORM) tma_prefetch_desc(&tmB1);
            int s = 0;
            uint32_t ph = 0;
            // a stage's loads count their bytes on this CTA's full barrier, or in pair mode on the
            // leader's, which expects both CTAs' bytes
            const uint32_t bytes_src = (PAIR ? 2 : 1) * C::A_BYTES;
            const uint32_t bytes_k = (PAIR ? 2 : 1) * ((AMODE == A_GATHER ? 0 : C::A_BYTES) + C::B_BYTES);
            auto begin_stage = [&](uint32_t bytes) {
                if (!PAIR) mbar_arrive_expect_tx(&full[s], bytes);
                else if (leader) mbar_arrive_expect_tx(&full[s], bytes);
            };
            auto ld2 = [&](void* dst, const CUtensorMap* m, int c0, int c1) {
                if (PAIR) tma_load_2d_pair(dst, m, L(&full[s]), c0, c1);
                else tma_load_2d(dst, m, &full[s], c0, c1);
            };
            auto ld3 = [&](void* dst, const CUtensorMap* m, int c0, int c1, int c2) {
                if (PAIR) tma_load_3d_pair(dst, m, L(&full[s]), c0, c1, c2);
                else tma_load_3d(dst, m, &full[s], c0, c1, c2);
            };
            auto ld4 = [&](void* dst, const CUtensorMap* m, int c0, int c1, int c2, int c3) {
                if (PAIR) tma_load_4d_pair(dst, m, L(&full[s]), c0, c1, c2, c3);
                else tma_load_4d(dst, m, &full[s], c0, c1, c2, c3);
            };
            TileInfo tn = dec(cid);
            for (int t = cid; t < ntile; t += ncid) {
                const TileInfo ti = tn;
                if (t + ncid < ntile) tn = dec(t + ncid);   // in flight meanwhile
                if (EPI == EPI_SUM) {
                    // source slabs: rows of this tile's samples, output columns n*BN .. +BN
#pragma unroll 1
                    for (int src = 0; src < n_src; ++src) {
                        const int kind = src < p.src_resid ? 0 : (src < p.src_resid + p.src_extra ? 1 : 2);
                        const int j = src - p.src_resid - p.src_extra;
#pragma unroll 1
                        for (int sl = 0; sl < BN / 64; ++sl) {
                            if (!wait(&empty[s], ph ^ 1, 0x103)) goto producer_done;
                            uint8_t* sa = smem + s * C::STAGE_BYTES;
                            begin_stage(bytes_src);
                            const int col = ti.n * BN + sl * 64;
                            if (kind == 2) {
                                // choice j's expert rows of the tile's 128 samples: rows m*128.. of
                                // region (bank, j) of the bank-major expert rows
                                ld3(sa, &tmS2, col, ti.m * 128, ti.g * p.k + j);
                            } else if (p.src_mix) {
                                const int per = p.omap.dh >> 4;
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int c16 = (col >> 4) + i, tk = c16 / per, jj = c16 - tk * per;
                                    ld4(sa + i * 4096, kind == 0 ? &tmS0 : &tmS1, 0, ti.g * per + jj, tk, ti.m * 128);
                                }
                            } else {
                                ld3(sa, kind == 0 ? &tmS0 : &tmS1, col, ti.g, ti.m * 128);
                            }
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                    }
                }
                for (int kb = 0; kb < KB; ++kb) {
                    if (!wait(&empty[s], ph ^ 1, 0x100)) goto producer_done;
                    uint8_t* sa = smem + s * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    begin_stage(bytes_k);
                    if (AMODE == A_TMA_2D) {
                        ld2(sa, &tmA, kb * KSLAB, ti.row0);
                    } else if (AMODE == A_TMA_3D) {
                        ld3(sa, &tmA, kb * KSLAB, ti.g, ti.m * 128);
                    } else if (AMODE == A_TMA_MIX) {
                        // mixed-row columns c16*16 .. +15 = token t, head piece jj of head ti.g
                        const int per = p.amap.dh >> 4;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int c16 = kb * 4 + i;
                            const int t = c16 / per, jj = c16 - t * per;
                            ld4(sa + i * 4096, &tmA, 0, ti.g * per + jj, t, ti.m * 128);
                        }
                    }
                    if (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_NORM) {
                        const int F = p.N >> 1;
                        const int r0 = ti.g * F + ti.n * (BN / 2);
                        if (PAIR) {
                            // the leader holds the BN/2 gate rows (N rows 0 .. BN/2-1), the peer the up rows
                            ld2(sb, leader ? &tmB0 : &tmB1, kb * KSLAB, r0);
                        } else {
                            ld2(sb, &tmB0, kb * KSLAB, r0);
                            ld2(sb + (BN / 2) * 128, &tmB1, kb * KSLAB, r0);
                        }
                    } else {
                        // pair mode: this CTA's half of the N tile's weight rows
                        ld2(sb, &tmB0, kb * 64, ti.g * p.N + ti.n * BN + (PAIR ? rank * (BN / 2) : 0));
                    }
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
            }
        }
    producer_done:;
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (pair mode: leader)
        if (lane == 0 && leader) {
            constexpr uint32_t idesc = F8 ? umma_idesc_e4m3(128, BN) : umma_idesc_bf16(PAIR ? 256 : 128, BN);
            // an MMA of this CTA (M = 128) or of the pair (M = 256); commits arrive on this CTA's
            // barrier, or on the same barrier of both CTAs
            auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
                if (PAIR) umma_bf16_pair(d, a, b, id, acc);
                else if (F8) umma_e4m3(d, a, b, id, acc);    // K = 32 codes per instruction
                else umma_bf16(d, a, b, id, acc);
            };
            auto commit = [&](uint64_t* b) {
                if (PAIR) {
                    umma_commit_pair(L(b));
                    umma_commit_pair(P(b));
                } else {
                    umma_commit(b);
                }
            };
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            for (int t = cid; t < ntile; t += ncid, ++lt) {
                const int buf = lt & 1;
                const uint32_t aph = (lt >> 1) & 1;
                if (!wait(&acc_empty[buf], aph ^ 1, 0x200)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * BN;
                bool ok = true;
                if (EPI == EPI_SUM) {
                    // Y = residual + inter-residual + sum_j gate_j expert_j: one N = 16 identity MMA per
                    // 16 columns and source (bf16 times one summed in fp32 is exact)
                    constexpr uint32_t idescI = umma_idesc_bf16(PAIR ? 256 : 128, 16);
                    const uint64_t idB = umma_sdesc_sw32(smem_u32(sI));
#pragma unroll 1
                    for (int src = 0; src < n_src && ok; ++src) {
                        const bool mixed = src < p.src_resid + p.src_extra && p.src_mix;
#pragma unroll 1
                        for (int sl = 0; sl < BN / 64; ++sl) {
                            if (!wait(&full[s], ph, 0x203)) { ok = false; break; }
                            tc_fence_after();
                            const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t a_k = mixed ? umma_sdesc_sw32(sa + kk * 4096) : umma_sdesc_sw128(sa) + 2 * kk;
                                mma(d + sl * 64 + kk * 16, a_k, idB, idescI, src > 0 ? 1u : 0u);
                            }
                            commit(&empty[s]);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                    }
                    if (!ok) break;
                }
                for (int kb = 0; kb < KB; ++kb) {
                    if (!wait(&full[s], ph, 0x201)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t sb = sa + C::A_BYTES;
                    const uint64_t ad = umma_sdesc_sw128(sa);
                    const uint64_t bd = umma_sdesc_sw128(sb);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // A: one 32-byte-swizzled 4 KB sub-slab per K step (mixed rows) or the
                        // 128-byte-swizzled 64-wide slab advanced by 32 bytes per K step
                        const uint64_t a_k = AMODE == A_TMA_MIX ? umma_sdesc_sw32(sa + kk * 4096) : ad + 2 * kk;
                        mma(d, a_k, bd + 2 * kk, idesc, (EPI == EPI_SUM && n_src > 0) || (kb | kk) != 0);
                    }
                    commit(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                commit(&acc_full[buf]);
            }
            // every MMA this thread issued must be complete before TMEM is released
            if (PAIR) umma_commit_pair(L(drain));
            else umma_commit(drain);
            wait_or_abort(drain, 0, abort_flag, 0x202);
        }
    } else if (warp >= 2 && warp < 2 + C::EPI_WARPS) {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int r = q * 32 + lane;
        // with 8 epilogue warps, warps 2-5 take columns [0, BN/2) and warps 6-9 [BN/2, BN)
        const int c_lo = C::EPI_WARPS == 8 ? ((warp - 2) >> 2) * (BN / 2) : 0;
        const int c_hi = C::EPI_WARPS == 8 ? c_lo + BN / 2 : BN;
        uint8_t* stg = smem + C::OFF_STG + (warp - 2) * 4096;         // this warp's 32 x 64 staging box
        // this thread's row (lane) of a 64-column bf16 chunk into the box, 128-byte swizzled rows,
        // once the warp's previous bulk store has read it
        auto stage_row = [&](const uint32_t(&pk)[32]) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8)
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((c8 ^ (lane & 7)) << 4)) =
                    make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        };
        // the staged box to global rows: row rr (lane rr's my_off: element offset of its chunk
        // start, < 0 skips the row) gets columns col .. col + 63; four rows per store instruction
        auto copy_rows = [&](long long my_off, int col) {
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int rr = it * 4 + (lane >> 3), cc = lane & 7;
                const long long off = __shfl_sync(0xffffffffu, my_off, rr);
                const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((cc ^ (rr & 7)) << 4));
                if (off >= 0) *reinterpret_cast<uint4*>(p.out + off + col + cc * 8) = v;
            }
            __syncwarp();
        };
        // This thread's row of a tile: sample b, sample-order slot e (EPI_SLOT_PERM), scale s (1/rms
        // for EPI_SWIGLU, the gate for EPI_SLOT_PERM).  The loads are issued a tile ahead (and the
        // tile descriptor two tiles ahead) and only waited for when the tile is processed.
        struct RowMeta {
            int b, e;
            float s;
        };
        const bool by_pos = p.sched == 1 && p.pos_scale != nullptr;
        auto row_meta = [&](const TileInfo& ti) -> RowMeta {
            RowMeta m{0, 0, 0.f};
            const int pos = ti.row0 + r;
            if (r >= ti.nrows || pos < 0 || pos >= p.pos_limit) return m;
            const bool need_b = p.sched == 1 && !(EPI == EPI_SLOT_PERM || (EPI == EPI_SWIGLU && by_pos));
            m.b = p.sched == 0 ? ti.m * 128 + r : (need_b ? __ldg(&p.bucket_rows[pos]) : 0);
            if (EPI == EPI_SWIGLU) {
                const int bank = p.sched == 0 ? ti.g : ti.g / p.E;
                m.s = by_pos ? __ldg(&p.pos_scale[pos]) : __ldg(&p.inv_rms[(size_t)m.b * p.banks + bank]);
            } else if (EPI == EPI_SLOT_PERM) {
                m.e = __ldg(&p.perm[pos]);
                m.s = by_pos ? __ldg(&p.pos_scale[pos]) : 0.f;
            }
            return m;
        };
        TileInfo ti_n1 = dec(cid), ti_n2 = ti_n1;
        RowMeta rm_n1 = row_meta(ti_n1);
        if (cid + ncid < ntile) ti_n2 = dec(cid + ncid);
        int lt = 0;
        for (int t = cid; t < ntile; t += ncid, ++lt) {
            const TileInfo ti = ti_n1;
            const RowMeta rm = rm_n1;
            if (t + ncid < ntile) {
                ti_n1 = ti_n2;
                rm_n1 = row_meta(ti_n1);
                if (t + 2 * ncid < ntile) ti_n2 = dec(t + 2 * ncid);
            }
            const int buf = lt & 1;
            const uint32_t aph = (lt >> 1) & 1;
            if (!wait(&acc_full[buf], aph, 0x300)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + buf * BN;
            bool valid = r < ti.nrows;
            const int pos = ti.row0 + r;                      // row position (hidden / slot index)
            const int b = rm.b;
            const int bank = p.sched == 0 ? ti.g : ti.g / p.E;
            if (valid && (b < 0 || b >= p.rows || pos < 0 || pos >= p.pos_limit)) {
                record_error(ERR_BOUNDS, 0x310);
                valid = false;
            }
            if (valid && EPI != EPI_RESID && EPI != EPI_COMBINE && EPI != EPI_SUM && EPI != EPI_ROUTE &&
                (size_t)(pos + 1) * p.out_ld > p.out_elems) {
                record_error(ERR_BOUNDS, 0x312);
                valid = false;
            }
            if (EPI == EPI_ROUTE) {
                // row statistics of this tile from the statistics warps
                if (!wait_or_abort(&st_full[buf], aph, abort_flag, 0x330)) break;
                const float ssq = ssbuf[buf * 128 + r];
                __syncwarp();
                if (lane == 0) mbar_arrive(&st_empty[buf]);
                const int E = p.E;
                const float irs = 1.0f / sqrtf(ssq / (float)p.K + p.r_eps);
                // the three parts of logit e sit in columns e, E + e and 2E + e: one load from each
                // base (columns past the accumulator's 3E are read and ignored)
                float vh[32], vm[32], vl[32];
                tmem_ld32(taddr, vh);
                tmem_ld32(taddr + E, vm);
                tmem_ld32(taddr + 2 * E, vl);
                // logit e = (hi + mid) + lo, scaled by 1/rms; softmax; top-k with ties to the lower index.
                // The loops are unrolled for register-resident arrays and leave at E (uniform across the
                // warp), so only E experts' instructions issue.
                float z[kRouteMaxE];
                float zmax = -INFINITY;
#pragma unroll
                for (int e = 0; e < kRouteMaxE; ++e) {
                    if (e >= E) break;
                    z[e] = ((vh[e] + vm[e]) + vl[e]) * irs;
                    zmax = fmaxf(zmax, z[e]);
                }
                float pe[kRouteMaxE];
                float sum = 0.f;
#pragma unroll
                for (int e = 0; e < kRouteMaxE; ++e) {
                    if (e >= E) break;
                    pe[e] = expf(z[e] - zmax);
                    sum += pe[e];
                }
                const size_t rowi = (size_t)b * p.banks + bank;
                uint32_t chosen = 0;
                float zk = INFINITY;   // logit of the k-th choice
#pragma unroll 1
                for (int j = 0; j < p.k; ++j) {
                    int be = -1;
                    float bz = -INFINITY, bp = 0.f;
#pragma unroll
                    for (int e = 0; e < kRouteMaxE; ++e) {
                        if (e >= E) break;
                        if (!((chosen >> e) & 1u) && (be < 0 || z[e] > bz)) { bz = z[e]; be = e; bp = pe[e]; }
                    }
                    chosen |= 1u << be;
                    zk = bz;
                    if (valid) {
                        p.r_idx[rowi * p.k + j] = be;
                        p.r_gate[rowi * p.k + j] = p.r_alpha * (bp / sum);
                    }
                }
                if (valid && p.r_inv_rms) p.r_inv_rms[rowi] = irs;
                if (valid && p.r_gap) {
                    // distance of the k-th choice to the best expert left out (none left: +inf)
                    float zn = -INFINITY;
#pragma unroll
                    for (int e = 0; e < kRouteMaxE; ++e) {
                        if (e >= E) break;
                        if (!((chosen >> e) & 1u)) zn = fmaxf(zn, z[e]);
                    }
                    p.r_gap[rowi] = zk - zn;
                }
                // per 128-row chunk: rows of this bank that chose expert e
                for (int e = 0; e < E; ++e) {
                    const unsigned bal = __ballot_sync(0xffffffffu, valid && ((chosen >> e) & 1u));
                    if (lane == 0 && bal)
                        atomicAdd(&p.r_counts[((size_t)bank * p.r_nchunks + ti.m) * E + e], __popc(bal));
                }
            } else if (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_NORM) {
                float sc = valid ? rm.s : 0.f;
                // F8: the row factor (E4M3 row scale / rms) times each projection's matrix scale
                const float sg8 = F8 ? __ldg(&p.w8_sgate[ti.g]) : 1.f, su8 = F8 ? __ldg(&p.w8_sup[ti.g]) : 1.f;
                if (EPI == EPI_SWIGLU_NORM) {
                    // 1/rms of this row from the statistics warps' sum of squares over the K columns
                    if (!wait_or_abort(&st_full[buf], aph, abort_flag, 0x331)) break;
                    const float ssq = ssbuf[buf * 128 + r];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&st_empty[buf]);
                    sc = valid ? 1.0f / sqrtf(ssq / (float)p.K + p.r_eps) : 0.f;
                }
                // a bulk tensor store per 32 x 64 box when all 32 rows of this warp belong to the
                // tile's group; else the valid rows through coalesced stores
                const bool box = __all_sync(0xffffffffu, valid);
                const long long my_off = valid ? (long long)pos * p.out_ld + ti.n * (BN / 2) : -1ll;
#pragma unroll 1
                for (int c = 0; c < BN / 2; c += 64) {
                    uint32_t pk[32];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float gv[32], uv[32];
                        tmem_ld32(taddr + c + 32 * h, gv);
                        tmem_ld32(taddr + BN / 2 + c + 32 * h, uv);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float h0, h1;
                            if (F8) {
                                const float sg = sc * sg8, su = sc * su8;
                                h0 = silu_tanh(sg * gv[2 * i]) * (su * uv[2 * i]);
                                h1 = silu_tanh(sg * gv[2 * i + 1]) * (su * uv[2 * i + 1]);
                            } else {
                                h0 = silu_tanh(sc * gv[2 * i]) * (sc * uv[2 * i]);
                                h1 = silu_tanh(sc * gv[2 * i + 1]) * (sc * uv[2 * i + 1]);
                            }
                            pk[16 * h + i] = pack_bf16x2(h0, h1);
                        }
                    }
                    stage_row(pk);
                    if (box) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmO, stg, ti.n * (BN / 2) + c, ti.row0 + q * 32);
                            bulk_commit_group();
                        }
                    } else {
                        copy_rows(my_off, c);
                    }
                }
            } else if (EPI == EPI_SLOT_PERM) {
                // the row of choice j of sample b (bank of the group), scaled by its gate: rows are
                // scattered, so each 64-column chunk is staged, then written by eight tile::scatter4 bulk
                // stores of four rows each (lanes 0-7: rows 4l .. 4l+3 of the warp's 32) when all 32 rows
                // are valid, else four whole rows per store instruction of the warp
                const int e = valid ? rm.e : 0;
                if (valid && (e < 0 || e >= p.pos_limit)) {
                    record_error(ERR_BOUNDS, 0x314);
                    valid = false;
                }
                const float gsc = valid ? (by_pos ? rm.s : __ldg(&p.gate[e])) : 0.f;
                const long long my_off = valid ? (long long)e * p.out_ld + ti.n * BN : -1ll;
                const bool whole = __all_sync(0xffffffffu, valid);
                int e4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) e4[i] = __shfl_sync(0xffffffffu, e, (4 * lane + i) & 31);
#pragma unroll 1
                for (int c = c_lo; c < c_hi; c += 64) {
                    uint32_t pk[32];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float v[32];
                        tmem_ld32(taddr + c + 32 * h, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[16 * h + i] = pack_bf16x2(gsc * v[2 * i], gsc * v[2 * i + 1]);
                    }
                    if (lane < 8) bulk_wait_read_all();   // this lane's previous scatter stores have read the box
                    __syncwarp();
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8)
                        *reinterpret_cast<uint4*>(stg + lane * 128 + ((c8 ^ (lane & 7)) << 4)) =
                            make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
                    if (whole) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane < 8) {
                            tma_scatter4(&tmO, stg + lane * 512, ti.n * BN + c, e4[0], e4[1], e4[2], e4[3]);
                            bulk_commit_group();
                        }
                    } else {
                        copy_rows(my_off, c);
                    }
                }
            } else if (EPI == EPI_SUM) {
                // Y already holds every term: bf16 through the output's row or Revert geometry, one
                // bulk tensor store per 32 x 64 box (rows past B are clipped by the map)
                const int b0 = ti.m * 128 + q * 32;
                const bool mixed = p.omap.layout == 1;
#pragma unroll 1
                for (int c = 0; c < BN; c += 64) {
                    uint32_t pk[32];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float v[32];
                        tmem_ld32(taddr + c + 32 * h, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[16 * h + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                    }
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        uint8_t* dst = mixed ? stg + (c8 >> 1) * 1024 + lane * 32 + (((c8 & 1) ^ ((lane >> 2) & 1)) << 4)
                                             : stg + lane * 128 + ((c8 ^ (lane & 7)) << 4);
                        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && b0 < p.rows) {
                        const int col = ti.n * BN + c;
                        if (mixed) {
                            const int per = p.omap.dh >> 4;
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4) {
                                const int ci = (col >> 4) + k4, tok = ci / per, jj = ci - tok * per;
                                tma_store_4d(&tmO, stg + k4 * 1024, 0, bank * per + jj, tok, b0);
                            }
                        } else {
                            tma_store_3d(&tmO, stg, col, bank, b0);
                        }
                        bulk_commit_group();
                    }
                }
            } else if (EPI == EPI_SLOT) {
                // plain rows out[pos, n*BN + c]: a bulk tensor store per 32 x 64 box when all 32 rows of
                // this warp belong to the tile's group (tmO: the output rows, 32-row boxes); else the
                // valid rows through coalesced stores from the same staged box
                const bool box = __all_sync(0xffffffffu, valid);
                const long long my_off = valid ? (long long)pos * p.out_ld + ti.n * BN : -1ll;
#pragma unroll 1
                for (int c = 0; c < BN; c += 64) {
                    uint32_t pk[32];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float v[32];
                        tmem_ld32(taddr + c + 32 * h, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) pk[16 * h + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                    }
                    stage_row(pk);
                    if (box) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmO, stg, ti.n * BN + c, ti.row0 + q * 32);
                            bulk_commit_group();
                        }
                    } else {
                        copy_rows(my_off, c);
                    }
                }
            } else {   // EPI_RESID / EPI_COMBINE
                int spos[8];
                float sg[8];
                if (EPI == EPI_COMBINE) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        spos[j] = 0;
                        sg[j] = 0.f;
                        if (j < p.k && valid) {
                            const size_t e = ((size_t)b * p.banks + bank) * p.k + j;
                            spos[j] = __ldg(&p.slot_of[e]);
                            sg[j] = __ldg(&p.gate[e]);
                            if (spos[j] < 0 || spos[j] >= p.pos_limit) {
                                record_error(ERR_BOUNDS, 0x311);
                                spos[j] = 0;
                                sg[j] = 0.f;
                            }
                        }
                    }
                }
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    float v[32];
                    tmem_ld32(taddr + c, v);
                    if (!valid) continue;
                    const int col0 = ti.n * BN + c;
                    // all global reads of this 32-column slice are issued before any arithmetic:
                    // residual and inter-residual first, then the slot rows two experts at a time
                    size_t off[4];
                    uint4 rv[4], ev[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        off[i] = row_elem(p.omap, b, bank, col0 + 8 * i);
                        const bool in = off[i] + 8 <= p.out_elems;
                        rv[i] = (p.resid && in) ? __ldg(reinterpret_cast<const uint4*>(p.resid + off[i])) : make_uint4(0, 0, 0, 0);
                        ev[i] = (p.extra && in) ? __ldg(reinterpret_cast<const uint4*>(p.extra + off[i])) : make_uint4(0, 0, 0, 0);
                    }
                    if (EPI == EPI_COMBINE) {
#pragma unroll
                        for (int j = 0; j < 8; j += 2) {
                            if (j >= p.k) break;
                            const bool two = j + 1 < p.k;
                            const uint4* s0 = reinterpret_cast<const uint4*>(p.slots + (size_t)spos[j] * p.omap.W + col0);
                            const uint4* s1 = reinterpret_cast<const uint4*>(p.slots + (size_t)spos[two ? j + 1 : j] * p.omap.W + col0);
                            uint4 a0[4], a1[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                a0[i] = __ldg(s0 + i);
                                a1[i] = two ? __ldg(s1 + i) : make_uint4(0, 0, 0, 0);
                            }
                            const float g0 = sg[j], g1 = two ? sg[j + 1] : 0.f;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint32_t w0[4] = {a0[i].x, a0[i].y, a0[i].z, a0[i].w};
                                const uint32_t w1[4] = {a1[i].x, a1[i].y, a1[i].z, a1[i].w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    v[8 * i + 2 * e] += g0 * bf16_lo(w0[e]) + g1 * bf16_lo(w1[e]);
                                    v[8 * i + 2 * e + 1] += g0 * bf16_hi(w0[e]) + g1 * bf16_hi(w1[e]);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (off[i] + 8 > p.out_elems) {
                            record_error(ERR_BOUNDS, 0x313);
                            continue;
                        }
                        const uint32_t rw[4] = {rv[i].x, rv[i].y, rv[i].z, rv[i].w};
                        const uint32_t ew[4] = {ev[i].x, ev[i].y, ev[i].z, ev[i].w};
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            o[2 * e] = v[8 * i + 2 * e] + bf16_lo(rw[e]) + bf16_lo(ew[e]);
                            o[2 * e + 1] = v[8 * i + 2 * e + 1] + bf16_hi(rw[e]) + bf16_hi(ew[e]);
                        }
                        *reinterpret_cast<uint4*>(p.out + off[i]) =
                            make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                       pack_bf16x2(o[6], o[7]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR) mbar_arrive_cluster(L(&acc_empty[buf]));     // the leader issues the next MMAs
                else mbar_arrive(&acc_empty[buf]);
            }
        }
        if (C::STAGED && lane < 8) bulk_wait_all();                   // stores complete before exit
        __syncwarp();
    } else if (C::STATS) {
        // ---------------------------------------------------------------- row statistics (warps 6-9)
        // Each lane sums the squares of its row of every A stage (a second consumer of the stage:
        // the empty barrier also waits for these four warps), then hands the tile's sums over.
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int s = 0, lt = 0;
        uint32_t ph = 0;
        for (int t = cid; t < ntile; t += ncid, ++lt) {
            const int buf = lt & 1;
            float ss = 0.f;
            bool ok = true;
            for (int kb = 0; kb < KB; ++kb) {
                if (!wait_or_abort(&full[s], ph, abort_flag, 0x420)) { ok = false; break; }
                const uint8_t* sa = smem + s * C::STAGE_BYTES;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    // logical 16-byte piece v of the row (column order, wherever the row sits in the
                    // tile): 32-byte swizzle stores half h at h ^ ((r / 4) % 2), 128-byte swizzle
                    // stores piece v at v ^ (r % 8)
                    const uint4 w4 = AMODE == A_TMA_MIX
                                         ? *reinterpret_cast<const uint4*>(sa + (v >> 1) * 4096 + r * 32 +
                                                                           (((v & 1) ^ ((r >> 2) & 1)) << 4))
                                         : *reinterpret_cast<const uint4*>(sa + r * 128 + (((v ^ r) & 7) << 4));
                    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a = bf16_lo(wv[e]), c = bf16_hi(wv[e]);
                        ss = fmaf(a, a, fmaf(c, c, ss));
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
            if (!ok) break;
            if (!wait_or_abort(&st_empty[buf], ((lt >> 1) & 1) ^ 1, abort_flag, 0x421)) break;
            ssbuf[buf * 128 + r] = ss;
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_full[buf]);
        }
    } else if (AMODE == A_GATHER) {
        // ---------------------------------------------------------------- row gatherers (warps 6-9)
        // Thread gt copies 16-byte chunk (gt % 8) of rows (gt / 8) + 16 * i, i = 0..7, into the
        // 128-byte-swizzled K-major A slab; copies land asynchronously and are published to the
        // MMA one stage late (commit group, wait, proxy fence, arrive).
        const int gt = threadIdx.x - 6 * 32;
        const int chunk = gt & 7;
        const int rsub = gt >> 3;
        int s = 0, pend_s = -1;
        uint32_t ph = 0;
        for (int t = cid; t < ntile; t += ncid) {
            const TileInfo ti = dec(t);
            int rb[8];
            int bank = p.sched == 0 ? ti.g : ti.g / p.E;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int rr = rsub + 16 * i;
                rb[i] = -1;
                if (rr < ti.nrows) rb[i] = p.sched == 0 ? ti.m * 128 + rr : __ldg(&p.bucket_rows[ti.row0 + rr]);
                if (rb[i] >= p.rows) {
                    record_error(ERR_BOUNDS, 0x410);
                    rb[i] = -1;
                }
            }
            for (int kb = 0; kb < KB; ++kb) {
                if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x400)) goto gather_done;
                const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
                const int col = kb * 64 + chunk * 8;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = rsub + 16 * i;
                    const uint32_t dst = sa + rr * 128 + ((chunk ^ (rr & 7)) << 4);
                    const __nv_bfloat16* src = rb[i] >= 0 ? p.a_ptr + row_elem(p.amap, rb[i], bank, col) : p.a_ptr;
                    cp_async_16(dst, src, rb[i] >= 0 ? 16u : 0u);
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
                if (pend_s >= 0) {
                    asm volatile("cp.async.wait_group 1;" ::: "memory");
                    fence_proxy_async_smem();
                    mbar_arrive(&full[pend_s]);
                }
                pend_s = s;
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
        }
    gather_done:
        cp_async_wait_all();
        if (pend_s >= 0) {
            fence_proxy_async_smem();
            mbar_arrive(&full[pend_s]);
        }
    }

    tc_fence_before();
    // pair mode: neither CTA releases its tensor memory or exits while the other may still arrive
    // on its barriers or be the target of the pair's MMAs
    if (PAIR) cluster_sync_all();
    else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace tml
