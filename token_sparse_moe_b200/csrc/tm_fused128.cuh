// tm_fused128.cuh -- the fused dense sub-layer (row width W = 128 or 256, hidden F % 128 == 0)
// with 128-wide hidden chunks:  y = SwiGLU_bank(RMSNorm(x)) + residual (+ inter-residual).
//
// Per 128-row tile the A tile stays resident in shared memory.  For each 128-wide hidden chunk c:
//   GEMM1(c): TMEM g1 = A . [Wg; Wu][chunk c]^T   (N = 256: 128 gate + 128 up)
//   epilogue: h = silu(s*g) * (s*u)  -> bf16 chunk in shared memory (s = 1/rms of the row)
//   GEMM2(c): TMEM Y += h . Wd[:, chunk c]^T       (N = W, K = 128)
// issued in the order G1(0), G1(1), G2(0), G1(2), G2(1), ...: the epilogue copies g1 out of TMEM
// and releases it at once, so G1(c+1) queues behind G2(c-1) while the SwiGLU of chunk c runs.
// TMEM: Y in columns [0, W), the GEMM1 buffer in [256, 512).
//
// The residual is added by the tensor core: GEMM2(0) initialises the accumulator Y, and after
// GEMM2(1) the residual tile times a 16 x 16 identity is accumulated into it (one N = 16 MMA per 16
// columns; bf16 times one summed in fp32 is exact).  When the residual is the sub-layer input
// itself (the mixing sub-layer) the resident A tile is that operand; otherwise the residual tile,
// and the inter-residual of a gap layer, stream through the weight ring with the same tensor-map
// geometry as A, prefetched like any weight stage.  The output epilogue is then only
// TMEM -> bf16 -> shared memory -> bulk tensor store.  A is loaded and released slab by slab
// (64 columns), so the next tile's A streams in while the last GEMM1 of this one still runs.
//
// The epilogue warps are software-pipelined across tiles: after the last hidden chunk of tile t
// they compute the row statistics of tile t+1 (its A tile is already loaded), run the SwiGLU of
// chunk 0 of t+1 (which releases the GEMM1 buffer for GEMM1(1) of t+1), and only then read Y of
// tile t out, so the tensor pipe has GEMM1 work for t+1 while Y of t drains.
//
// Warp roles: warp 0 TMA producer (and builds the identity tile), warp 1 MMA issuer and TMEM
// owner, warps 2-9 epilogue (TMEM lane quarter = warp % 4; warps 2-5 / 6-9 take the two column
// halves).
//
// Block mode (AMODE = A_BLOCK, when both sub-layers of a block are dense with the same row width,
// i.e. T == H): one launch runs the whole block.  The tiles of the mixing sub-layer (A through the
// Mix map, residual = A, output stored through the Revert map into X_revert) come first, then
// those of the reverting sub-layer (A = rows of X_revert, residual X streamed), both ordered by
// 128-sample row block.  A reverting tile of row block m reads X_revert rows that every mixing
// tile of block m writes, so its A load waits for a per-block counter: each epilogue warp of a
// mixing tile adds one with release semantics once its bulk stores are complete in global
// memory.  No SM idles between the two sub-layers: the partial last wave of the mixing tiles is
// filled with reverting tiles whose row blocks finished long before.  The launch is cooperative
// (all CTAs resident), and a mixing tile's count never waits on a reverting tile (see the
// epilogue), so every wait ends.
#pragma once
#include "tm_fused.cuh"

namespace tml {

enum FusedResid : int { RES_NONE = 0, RES_FROM_A = 1, RES_STREAM = 2 };
constexpr int A_BLOCK = 4;   // fused128 kernel: a whole dense block (mixing tiles, then reverting tiles)
// FP8 serving path (F8 = true, any A mode): the bf16 A tile arrives as in the bf16 kernel; the
// epilogue warps' statistics pass also takes each row's max|x| and writes the row's E4M3 codes
// (its power-of-two scale, exact scaling) into an E4M3 copy of the tile, which GEMM1 reads with
// kind::f8f6f4 MMAs against E4M3 gate / up weights; the SwiGLU takes back the row factor
// 2^e / rms and the bank's gate / up weight scales.  GEMM2, the residual and the output are
// those of the bf16 kernel.
template <int W, int AMODE, bool F8 = false>
struct Fused128Cfg {
    static_assert(W == 128 || W == 256, "fused sub-layer supports row widths 128 and 256");
    static constexpr int A_BYTES = 128 * W * 2;                   // the bf16 A tile, W / 64 slabs
    static constexpr int A_SLABS = W / 64;
    static constexpr int A8_BYTES = F8 ? 128 * W : 0;             // FP8: its E4M3 copy, W / 128 slabs of 128 columns
    static constexpr int HID_BYTES = 128 * 128 * 2;               // one 128-wide hidden chunk, 2 K-slabs
    static constexpr int SB = 32768;                              // ring stage
    static constexpr int G1_STAGES = F8 ? W / 128 : W / 64;       // 256 rows x 64 K (bf16) or 128 K (E4M3) per stage
    static constexpr int G2_STAGES = W == 256 ? 2 : 1;            // W rows x 128 K per chunk
    static constexpr int R_STAGES = W / 128;                      // residual tile: 128 rows x 128 columns per stage
    static constexpr int STAGES = F8 ? (W == 256 ? 3 : 4) : (W == 256 ? 4 : 5);
    static constexpr int NTHREADS = 10 * 32;
    static constexpr int OFF_A8 = A_BYTES;
    static constexpr int OFF_HID = A_BYTES + A8_BYTES;
    static constexpr int OFF_RING = OFF_HID + HID_BYTES;
    static constexpr int OFF_ID = OFF_RING + STAGES * SB;         // 16 x 16 identity, 32-byte swizzled K-major
    static constexpr int OFF_XCH = OFF_ID + 512;                  // row statistics exchange, 2 x 128 floats
    static constexpr int OFF_BAR = OFF_XCH + 1024;
    static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
    static constexpr int G1COL = 256;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};


// One work item of a CTA: tile t (bank g, row tile m), hidden chunks [c0, c1); sec: a tile of the
// second (reverting) sub-layer in block mode; mx: A, the residual stream and the output use the
// Mix geometry.
struct F128Item {
    int t, g, m, c0, c1;
    bool sec, mx;
};

// The kernel body; the tensor maps are the kernel's __grid_constant__ parameters, passed by
// reference so that the bulk tensor instructions see their parameter-space addresses.
template <int W, int AMODE, bool F8>
__device__ __forceinline__ void fused128_body(const CUtensorMap& tmA, const CUtensorMap& tmG, const CUtensorMap& tmU,
                                              const CUtensorMap& tmD, const CUtensorMap& tmR, const CUtensorMap& tmE,
                                              const CUtensorMap& tmO, const CUtensorMap& tmA2, const CUtensorMap& tmG2,
                                              const CUtensorMap& tmU2, const CUtensorMap& tmD2, const CUtensorMap& tmO2,
                                              const FusedParams& p) {
    // Maps: A, G, U, D, O of the (first) sub-layer; R / E the streamed residual and inter-residual
    // (in block mode those of the reverting sub-layer); A2, G2, U2, D2, O2 the reverting
    // sub-layer's in block mode (unused otherwise).
    using C = Fused128Cfg<W, AMODE, F8>;
    constexpr bool BLK = AMODE == A_BLOCK;
    constexpr bool MIXG = AMODE == A_TMA_MIX;                       // Mix geometry outside block mode
    constexpr int STAGES = C::STAGES;
    const int mt = (p.rows + 127) / 128;
    const int ntile1 = p.banks * mt;                 // tiles of one sub-layer
    const int ntile = BLK ? 2 * ntile1 : ntile1;
    if ((int)blockIdx.x >= ntile) return;
    const int NC = p.F / 128;
    // GEMM2(c) is issued in step c + LAG, after GEMM1(c + LAG).  LAG = 1: the SwiGLU of chunk c
    // overlaps GEMM1(c+1) and its hidden write waits only for GEMM2(c-1).  (A lag of 2 measured
    // 16% slower on the dense block workload: each hidden write then waits behind a whole GEMM1.)
    constexpr int LAG = 1;
    // Work items of this CTA: tile t = blockIdx.x + k * gridDim.x, all hidden chunks of the tile.
    // Block mode: tiles [0, ntile1) mixing, [ntile1, 2 ntile1) reverting, each numbered
    // m * banks + g.
    const int full_waves = ntile / (int)gridDim.x;
    const int n_rem = ntile - full_waves * (int)gridDim.x;
    auto item = [&](int k, F128Item& it) -> bool {
        const int b = blockIdx.x;
        it.c0 = 0;
        if (BLK) {
            it.t = b + k * (int)gridDim.x;
            if (it.t >= ntile) return false;
            it.sec = it.t >= ntile1;
            it.mx = !it.sec;
            const int tt = it.sec ? it.t - ntile1 : it.t;
            it.m = tt / p.banks;
            it.g = tt - it.m * p.banks;
            it.c1 = (it.sec ? p.F2 : p.F) / 128;
            return true;
        }
        it.sec = false;
        it.mx = MIXG;
        it.c1 = NC;
        if (k < full_waves) {
            it.t = b + k * (int)gridDim.x;
        } else if (k > full_waves) {
            return false;
        } else {
            if (b >= n_rem) return false;
            it.t = full_waves * (int)gridDim.x + b;
        }
        it.g = it.t / mt;
        it.m = it.t - it.g * mt;
        return true;
    };
    // per-item choices (compile-time constants outside block mode)
    auto amix = [&](const F128Item& it) { return BLK ? it.mx : MIXG; };
    auto rmode = [&](const F128Item& it) { return BLK && it.sec ? p.res_mode2 : p.res_mode; };
    auto n_res = [&](const F128Item& it) { return rmode(it) == RES_STREAM ? C::R_STAGES : 0; };
    auto n_ext = [&](const F128Item& it) { return (BLK && it.sec ? p.has_extra2 : p.has_extra) ? C::R_STAGES : 0; };
    // per item with nc chunks: steps 0 .. nc + LAG - 1; the residual / inter-residual identity pass
    // (only in the item that starts at chunk 0) runs in step s_r, after GEMM2(min(1, nc-1)): Y is
    // initialised by the item's first GEMM2, and the streamed tiles come through the ring like
    // any weight stage
    auto id_step = [&](int nc) { return (nc < 2 ? 0 : 1) + LAG; };

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sA8 = smem + C::OFF_A8;
    uint8_t* sH = smem + C::OFF_HID;
    uint8_t* sR = smem + C::OFF_RING;
    uint8_t* sI = smem + C::OFF_ID;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bar;                  // [STAGES]
    uint64_t* empty = full + STAGES;       // [STAGES]
    uint64_t* a_full = empty + STAGES;
    uint64_t* a_empty = a_full + 1;        // [A_SLABS]: one per 64-column slab of A
    uint64_t* g1_full = a_empty + C::A_SLABS;
    uint64_t* g1_empty = g1_full + 1;
    uint64_t* hid_full = g1_empty + 1;
    uint64_t* hid_empty = hid_full + 1;
    uint64_t* y_full = hid_empty + 1;
    uint64_t* y_empty = y_full + 1;
    uint64_t* drain = y_empty + 1;
    uint64_t* stats_bar = drain + 1;       // both halves' partial row sums written
    uint64_t* stats_done = stats_bar + 1;  // both halves' partial row sums read
    uint64_t* a8_full = stats_done + 1;    // FP8: the tile's E4M3 codes written (8 epilogue warps)
    uint64_t* a8_empty = a8_full + 1;      // FP8: the item's GEMM1s are done with them
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(a8_empty + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(a_full, 1);
        // per slab of A: the MMA (last read issued) + the epilogue warps that read it (the 4 of the
        // half on the bf16 path; all 8 on the FP8 path, whose statistics read whole rows)
        for (int q = 0; q < C::A_SLABS; ++q) mbar_init(&a_empty[q], F8 ? 1 + 8 : 1 + 4);
        mbar_init(a8_full, 8);
        mbar_init(a8_empty, 1);
        mbar_init(g1_full, 1);
        mbar_init(g1_empty, 8);
        mbar_init(hid_full, 8);
        mbar_init(hid_empty, 1);
        mbar_init(y_full, 1);
        mbar_init(y_empty, 8);
        mbar_init(drain, 1);
        mbar_init(stats_bar, 8);
        mbar_init(stats_done, 8);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        // identity B operand: 16 rows n x 16 columns k, 32-byte rows, 32-byte swizzle (the 16-byte
        // half of row n that holds column k sits at half (k / 8) ^ ((n / 4) % 2))
        const int n = lane & 15, hf = lane >> 4;
        const uint32_t one = (n >> 3) == hf ? ((n & 1) ? 0x3F800000u : 0x00003F80u) : 0u;
        const int wi = (n & 7) >> 1;
        *reinterpret_cast<uint4*>(sI + n * 32 + ((hf ^ ((n >> 2) & 1)) << 4)) =
            make_uint4(wi == 0 ? one : 0u, wi == 1 ? one : 0u, wi == 2 ? one : 0u, wi == 3 ? one : 0u);
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmG);
            tma_prefetch_desc(&tmU);
            tma_prefetch_desc(&tmD);
            if (BLK) {
                tma_prefetch_desc(&tmA2);
                tma_prefetch_desc(&tmG2);
                tma_prefetch_desc(&tmU2);
                tma_prefetch_desc(&tmD2);
            }
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            bool ok = true;
            // 128 rows x (16 * n16) columns from column 16 * col16 of a row tensor, in the A geometry
            auto load_rows = [&](const CUtensorMap* map, bool mx, uint8_t* dst, uint64_t* b, int g, int m0, int col16,
                                 int n16) {
                if (mx) {
                    const int per = p.amap.dh >> 4;
#pragma unroll 1
                    for (int i = 0; i < n16; ++i) {
                        const int ci = col16 + i, tok = ci / per, jj = ci - tok * per;
                        tma_load_4d(dst + i * 4096, map, b, 0, g * per + jj, tok, m0);
                    }
                } else {
#pragma unroll 1
                    for (int i = 0; i < n16 / 4; ++i) tma_load_3d(dst + i * 16384, map, b, col16 * 16 + i * 64, g, m0);
                }
            };
            // block mode: every mixing tile of row block m has stored its X_revert rows (8 epilogue
            // warps per tile count once each)
            auto wait_block = [&](int m) -> bool {
                const unsigned* ctr = p.dep + m;
                const unsigned target = 8u * (unsigned)p.banks;
                if (ld_acquire(ctr) < target) {
                    const uint64_t t0 = globaltimer_ns(), lim = wait_limit_ns();
                    while (ld_acquire(ctr) < target) {
                        if (*abort_flag) return false;
                        if (globaltimer_ns() - t0 > lim) {
                            record_error(ERR_TIMEOUT, 0x3108);
                            *abort_flag = 1;
                            return false;
                        }
                        __nanosleep(64);
                    }
                }
                fence_proxy_async_global();   // the bulk tensor loads below come after the acquire
                return true;
            };
            F128Item it;
            for (; ok && item(lt, it); ++lt) {
                const int g = it.g, m = it.m, c0 = it.c0;
                const int nc = it.c1 - it.c0, n_steps = nc + LAG, s_r = c0 == 0 ? id_step(nc) : -1;
                const bool mx = amix(it);
                const int F = BLK && it.sec ? p.F2 : p.F;
                const int res_stages = n_res(it), ext_stages = n_ext(it);
                const CUtensorMap* mA = BLK && it.sec ? &tmA2 : &tmA;
                const CUtensorMap* mG = BLK && it.sec ? &tmG2 : &tmG;
                const CUtensorMap* mU = BLK && it.sec ? &tmU2 : &tmU;
                const CUtensorMap* mD = BLK && it.sec ? &tmD2 : &tmD;
                if (BLK && it.sec && !wait_block(m)) break;
                // A slab by slab, each as soon as the previous tile has released it
#pragma unroll 1
                for (int qa = 0; qa < C::A_SLABS && ok; ++qa) {
                    if (!wait_or_abort(&a_empty[qa], (lt & 1) ^ 1, abort_flag, 0x3100)) { ok = false; break; }
                    if (qa == 0) mbar_arrive_expect_tx(a_full, C::A_BYTES);
                    load_rows(mA, mx, sA + qa * 16384, a_full, g, m * 128, qa * 4, 4);
                }
                if (!ok) break;
                // ring order per step: G1(step) (step < NC), G2(step - LAG) (step >= LAG), and at step
                // s_r the residual and inter-residual tiles
#pragma unroll 1
                for (int step = 0; step < n_steps && ok; ++step) {
                    if (step < nc) {
                        const int c = c0 + step;
#pragma unroll 1
                        for (int q = 0; q < C::G1_STAGES; ++q) {             // K slab q: 128 gate + 128 up rows
                            if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x3101)) { ok = false; break; }
                            uint8_t* st = sR + s * C::SB;
                            mbar_arrive_expect_tx(&full[s], C::SB);
                            const int kq = F8 ? q * 128 : q * 64;
                            tma_load_2d(st, mG, &full[s], kq, g * F + c * 128);
                            tma_load_2d(st + 16384, mU, &full[s], kq, g * F + c * 128);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                    }
                    if (step >= LAG && ok) {
                        const int c = c0 + step - LAG;
#pragma unroll 1
                        for (int q = 0; q < C::G2_STAGES; ++q) {
                            if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x3102)) { ok = false; break; }
                            uint8_t* st = sR + s * C::SB;
                            mbar_arrive_expect_tx(&full[s], C::SB);
                            if (W == 256) {
                                tma_load_2d(st, mD, &full[s], c * 128 + q * 64, g * W);          // 256 rows x 64 K
                            } else {
                                tma_load_2d(st, mD, &full[s], c * 128, g * W);                   // 128 rows x 64 K
                                tma_load_2d(st + 16384, mD, &full[s], c * 128 + 64, g * W);      // next 64 K
                            }
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                    }
                    if (step == s_r && ok) {
#pragma unroll 1
                        for (int i = 0; i < res_stages + ext_stages; ++i) {    // 128 columns per stage
                            if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x3103)) { ok = false; break; }
                            uint8_t* st = sR + s * C::SB;
                            mbar_arrive_expect_tx(&full[s], C::SB);
                            const int q = i < res_stages ? i : i - res_stages;
                            load_rows(i < res_stages ? &tmR : &tmE, mx, st, &full[s], g, m * 128, q * 8, 8);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                    }

                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // Barrier checks are batched: the GEMM1 buffer barrier and all stages of a GEMM1 (or the
        // hidden barrier and the stages of a GEMM2) are tested together without blocking, so their
        // latencies overlap; only a stage that is not ready yet is waited for on its own.
        if (lane == 0) {
            constexpr uint32_t idesc1 = F8 ? umma_idesc_e4m3(128, 256) : umma_idesc_bf16(128, 256);
            constexpr uint32_t idesc2 = umma_idesc_bf16(128, W);
            constexpr uint32_t idescI = umma_idesc_bf16(128, 16);
            const uint32_t aS = smem_u32(sA), hS = smem_u32(sH), rS = smem_u32(sR);
            uint64_t adesc[W / 16];
            auto set_adesc = [&](bool mx) {
#pragma unroll
                for (int k16 = 0; k16 < W / 16; ++k16)
                    adesc[k16] = mx ? umma_sdesc_sw32(aS + k16 * 4096)
                                    : umma_sdesc_sw128(aS + (k16 >> 2) * 16384) + 2 * (k16 & 3);
            };
            set_adesc(AMODE == A_TMA_MIX);
            const uint64_t hdesc0 = umma_sdesc_sw128(hS), hdesc1 = umma_sdesc_sw128(hS + 16384);
            // FP8: the E4M3 copy of A, 128-column slabs with 128-byte swizzle, 32 columns per MMA
            uint64_t a8desc[F8 ? W / 32 : 1];
#pragma unroll
            for (int k = 0; k < (F8 ? W / 32 : 1); ++k)
                a8desc[k] = umma_sdesc_sw128(smem_u32(sA8) + (k >> 2) * 16384) + 2 * (k & 3);
            const uint64_t rdesc0 = umma_sdesc_sw128(rS);
            const uint64_t rdesc32 = umma_sdesc_sw32(rS);
            const uint64_t idB = umma_sdesc_sw32(smem_u32(sI));
            constexpr uint64_t kStageDesc = C::SB >> 4;               // descriptor start-address step per stage
            uint32_t ubase = 0;                                        // chunks of the items before this one
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            bool ok = true;
            F128Item it;
            for (; ok && item(lt, it); ++lt) {
                const int nc = it.c1 - it.c0, n_steps = nc + LAG, s_r = it.c0 == 0 ? id_step(nc) : -1;
                const bool mx = amix(it);
                const int rm = rmode(it), res_stages = n_res(it), ext_stages = n_ext(it);
                if (BLK) set_adesc(mx);
                // A is released slab by slab after the item's last GEMM1, or after the identity pass
                // when that reads A and comes later.  FP8: GEMM1 reads the E4M3 copy, so the bf16 tile
                // is released after the identity pass when that reads it, else at once.
                const bool a_after_id = rm == RES_FROM_A && (F8 || s_r >= nc - 1);
                if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x3200)) break;
                if (F8) {
                    if (!a_after_id) {
#pragma unroll
                        for (int q = 0; q < C::A_SLABS; ++q) umma_commit(&a_empty[q]);
                    }
                    if (!wait_or_abort(a8_full, lt & 1, abort_flag, 0x3208)) break;   // the item's E4M3 codes
                }
                tc_fence_after();
#pragma unroll 1
                for (int step = 0; step < n_steps && ok; ++step) {
                    if (step < nc) {                                   // ---- GEMM1(c0 + step)
                        const uint32_t use = ubase + step;
                        bool rdy[C::G1_STAGES];
                        const bool e_rdy = mbar_test(g1_empty, (use & 1) ^ 1);
                        {
                            int ss = s;
                            uint32_t pp = ph;
#pragma unroll
                            for (int q = 0; q < C::G1_STAGES; ++q) {
                                rdy[q] = mbar_test(&full[ss], pp);
                                if (++ss == STAGES) { ss = 0; pp ^= 1; }
                            }
                        }
                        if (!e_rdy && !wait_or_abort(g1_empty, (use & 1) ^ 1, abort_flag, 0x3201)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int q = 0; q < C::G1_STAGES; ++q) {
                            if (!rdy[q]) {
                                if (!wait_or_abort(&full[s], ph, abort_flag, 0x3202)) { ok = false; break; }
                                tc_fence_after();
                            }
                            const uint64_t bd = rdesc0 + (uint64_t)s * kStageDesc;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                if (F8) umma_e4m3(tmem + C::G1COL, a8desc[q * 4 + kk], bd + 2 * kk, idesc1, (q | kk) != 0);
                                else umma_bf16(tmem + C::G1COL, adesc[q * 4 + kk], bd + 2 * kk, idesc1, (q | kk) != 0);
                            umma_commit(&empty[s]);
                            if (!F8 && step == nc - 1 && !a_after_id) umma_commit(&a_empty[q]);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                        umma_commit(g1_full);
                        if (F8 && step == nc - 1) umma_commit(a8_empty);   // the E4M3 copy is free
                    }
                    if (step >= LAG) {                                 // ---- GEMM2(c0 + step - LAG)
                        const int c = step - LAG;                      // relative to c0
                        const uint32_t use = ubase + c;
                        if (c == 0) {                                  // GEMM2(0) initialises Y: wait until it is free
                            if (!wait_or_abort(y_empty, (lt & 1) ^ 1, abort_flag, 0x3204)) { ok = false; break; }
                            tc_fence_after();
                        }
                        bool rdy[C::G2_STAGES];
                        const bool h_rdy = mbar_test(hid_full, use & 1);
                        {
                            int ss = s;
                            uint32_t pp = ph;
#pragma unroll
                            for (int q = 0; q < C::G2_STAGES; ++q) {
                                rdy[q] = mbar_test(&full[ss], pp);
                                if (++ss == STAGES) { ss = 0; pp ^= 1; }
                            }
                        }
                        if (!h_rdy && !wait_or_abort(hid_full, use & 1, abort_flag, 0x3203)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int q = 0; q < C::G2_STAGES; ++q) {
                            if (!rdy[q]) {
                                if (!wait_or_abort(&full[s], ph, abort_flag, 0x3205)) { ok = false; break; }
                                tc_fence_after();
                            }
                            const uint64_t bd = rdesc0 + (uint64_t)s * kStageDesc;
#pragma unroll
                            for (int kq = 0; kq < (W == 256 ? 1 : 2); ++kq) {   // 64-wide K slabs in this stage
                                const uint64_t hd = ((q + kq) ? hdesc1 : hdesc0);
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_bf16(tmem, hd + 2 * kk, bd + kq * (16384 >> 4) + 2 * kk, idesc2,
                                              (c | q | kq | kk) != 0 ? 1u : 0u);
                            }
                            umma_commit(&empty[s]);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                        umma_commit(hid_empty);
                    }
                    if (step == s_r) {                                 // ---- Y += residual (+ inter-residual)
                        if (rm == RES_FROM_A) {
#pragma unroll
                            for (int k16 = 0; k16 < W / 16; ++k16) umma_bf16(tmem + 16 * k16, adesc[k16], idB, idescI, 1);
                            if (a_after_id) {
#pragma unroll
                                for (int q = 0; q < C::A_SLABS; ++q) umma_commit(&a_empty[q]);
                            }
                        }
#pragma unroll 1
                        for (int i = 0; i < res_stages + ext_stages; ++i) {
                            if (!wait_or_abort(&full[s], ph, abort_flag, 0x3207)) { ok = false; break; }
                            tc_fence_after();
                            const int q = i < res_stages ? i : i - res_stages;
                            const uint32_t st = rS + s * C::SB;
#pragma unroll
                            for (int k16 = 0; k16 < 8; ++k16) {
                                const uint64_t rd = mx
                                                        ? rdesc32 + (uint64_t)s * kStageDesc + k16 * (4096 >> 4)
                                                        : umma_sdesc_sw128(st + (k16 >> 2) * 16384) + 2 * (k16 & 3);
                                umma_bf16(tmem + 16 * (q * 8 + k16), rd, idB, idescI, 1);
                            }
                            umma_commit(&empty[s]);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                    }
                    if (step == n_steps - 1) umma_commit(y_full);
                }
                ubase += nc;
            }
            umma_commit(drain);
            wait_or_abort(drain, 0, abort_flag, 0x3206);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-9)
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        const uint32_t trow = tmem + (uint32_t(q * 32) << 16);
        float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);      // [half][row] partial sums of squares
        uint8_t* stg = sH + half * 16384 + q * 4096;                  // this warp's 32 rows of the hidden buffer
        int n_stats = 0;
        // Block mode: the row block of the last mixing tile whose bulk stores this warp issued and has
        // not counted yet (-1: none).  Its count is added at this warp's next output, by which time
        // the stores are long complete, or at once when the next item is a reverting tile or there
        // is none (so a mixing tile's count never waits on a reverting tile).
        int pend_m = -1;
        auto flush_block = [&]() {
            if (BLK && pend_m >= 0) {
                if (lane == 0) {
                    bulk_wait_all();                                   // this warp's stores are in global memory
                    fence_proxy_async_global();
                    red_release_add(p.dep + pend_m, 1u);
                }
                __syncwarp();
                pend_m = -1;
            }
        };
        // 1/rms of this thread's row of the tile in the A buffer (0 for rows past the end).  Each half
        // sums the squares of its half of the row; the two partials meet in shared memory and are
        // added in the same order by both threads of the row.
        auto row_scale = [&](int m_tile, bool mx, float& out) -> bool {
            float ss = 0.f;
            if (mx) {
#pragma unroll 4
                for (int i = 0; i < W / 32; ++i) {
                    const uint4* rp = reinterpret_cast<const uint4*>(sA + (half * (W / 32) + i) * 4096 + r * 32);
#pragma unroll
                    for (int v = 0; v < 2; ++v) {
                        // logical half v (the 32-byte swizzle stores it at v ^ ((r / 4) % 2)): every row
                        // sums in column order wherever it sits in the tile
                        const uint4 w4 = rp[v ^ ((r >> 2) & 1)];
                        const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo = bf16_lo(wv[e]), hi = bf16_hi(wv[e]);
                            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int i = 0; i < W / 128; ++i) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const uint4 w4 = *reinterpret_cast<const uint4*>(sA + (half * (W / 128) + i) * 16384 + r * 128 +
                                                                         (((v ^ r) & 7) << 4));
                        const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo = bf16_lo(wv[e]), hi = bf16_hi(wv[e]);
                            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                        }
                    }
                }
            }
            // the other half has read the previous round's partial before this one overwrites it
            if (n_stats > 0 && !wait_or_abort(stats_done, (n_stats - 1) & 1, abort_flag, 0x3305)) return false;
            xch[half * 128 + r] = ss;
            __syncwarp();
            if (lane == 0) mbar_arrive(stats_bar);
            if (!wait_or_abort(stats_bar, n_stats & 1, abort_flag, 0x3306)) return false;
            const float tot = xch[r] + xch[128 + r];
            __syncwarp();
            if (lane == 0) mbar_arrive(stats_done);
            ++n_stats;
            out = r < p.rows - m_tile * 128 ? 1.0f / sqrtf(tot / (float)W + p.eps) : 0.f;
            return true;
        };
        // FP8: 8 bf16 of row r at column col (a multiple of 8) of the A tile, in either geometry
        auto a_chunk = [&](bool mx, int col) -> uint4 {
            if (mx)   // 16-column boxes of 128 rows x 32 bytes, 32-byte swizzle
                return *reinterpret_cast<const uint4*>(sA + (col >> 4) * 4096 + r * 32 +
                                                       ((((col >> 3) & 1) ^ ((r >> 2) & 1)) << 4));
            return *reinterpret_cast<const uint4*>(sA + (col >> 6) * 16384 + r * 128 +   // 64-column slabs, 128-byte swizzle
                                                   ((((col >> 3) & 7) ^ (r & 7)) << 4));
        };
        // FP8: the row's statistics over the whole row (both threads of a row sum in the same order,
        // so they agree without an exchange), then this thread's half of the row as E4M3 codes in
        // the tile's E4M3 copy (128-column slabs, 128-byte swizzle) with the row's power-of-two
        // scale 2^e (the smallest with max|x| * 2^-e <= 448); out = 2^e / rms(x)
        int n_q = 0;
        auto row_scale8 = [&](int m_tile, bool mx, float& out) -> bool {
            float ss = 0.f, amax = 0.f;
#pragma unroll 4
            for (int col = 0; col < W; col += 8) {
                const uint4 w4 = a_chunk(mx, col);
                const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = bf16_lo(wv[e]), hi = bf16_hi(wv[e]);
                    ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                    amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
                }
            }
            const int ex = pow2_exponent(amax);
            const float inv = pow2f(-ex);
            // the previous item's GEMM1s are done with the E4M3 copy
            if (n_q > 0 && !wait_or_abort(a8_empty, (n_q - 1) & 1, abort_flag, 0x3307)) return false;
#pragma unroll 2
            for (int col = half * (W / 2); col < (half + 1) * (W / 2); col += 16) {
                const uint4 lo4 = a_chunk(mx, col), hi4 = a_chunk(mx, col + 8);
                const uint32_t av[8] = {lo4.x, lo4.y, lo4.z, lo4.w, hi4.x, hi4.y, hi4.z, hi4.w};
                uint32_t q4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    q4[e] = uint32_t(e4m3x2(bf16_lo(av[2 * e]) * inv, bf16_hi(av[2 * e]) * inv)) |
                            (uint32_t(e4m3x2(bf16_lo(av[2 * e + 1]) * inv, bf16_hi(av[2 * e + 1]) * inv)) << 16);
                const int k = (col & 127) >> 4;
                *reinterpret_cast<uint4*>(sA8 + (col >> 7) * 16384 + r * 128 + ((k ^ (r & 7)) << 4)) =
                    make_uint4(q4[0], q4[1], q4[2], q4[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(a8_full);
            ++n_q;
            out = r < p.rows - m_tile * 128 ? pow2f(ex) * (1.0f / sqrtf(ss / (float)W + p.eps)) : 0.f;
            return true;
        };
        // Y of tile (g, m) (residual already accumulated) -> bf16 -> this warp's rows of the idle hidden
        // buffer in the output box layout -> bulk tensor store, 64 columns per round; releases Y
        auto output_tile = [&](int g, int m, int ylt, bool mx, bool sec) -> bool {
            if (!wait_or_abort(y_full, ylt & 1, abort_flag, 0x3303)) return false;
            tc_fence_after();
            flush_block();                                            // the previous mixing tile's stores are done
            const CUtensorMap* mo = BLK && sec ? &tmO2 : &tmO;
            const int b0 = m * 128 + q * 32;                          // first row of this warp's box
#pragma unroll
            for (int j = 0; j < W / 128; ++j) {
                const int col0 = half * (W / 2) + j * 64;
                uint32_t v0[32], v1[32];
                tmem_ld32_async(trow + col0, v0);
                tmem_ld32_async(trow + col0 + 32, v1);
                tmem_wait_ld_tie(v0);
                tmem_wait_ld_tie(v1);
                if (j == W / 128 - 1) {                                // Y fully read: release it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(y_empty);
                }
                if (j > 0) {                                           // the previous round's store has read the rows
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                }
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {                       // 8 columns per 16-byte piece
                    const uint32_t* vv = c8 < 4 ? v0 : v1;
                    const int o = (c8 & 3) * 8;
                    const uint4 w4 = make_uint4(pack_bf16x2(__uint_as_float(vv[o + 0]), __uint_as_float(vv[o + 1])),
                                                pack_bf16x2(__uint_as_float(vv[o + 2]), __uint_as_float(vv[o + 3])),
                                                pack_bf16x2(__uint_as_float(vv[o + 4]), __uint_as_float(vv[o + 5])),
                                                pack_bf16x2(__uint_as_float(vv[o + 6]), __uint_as_float(vv[o + 7])));
                    uint8_t* dst = mx ? stg + (c8 >> 1) * 1024 + lane * 32 + (((c8 & 1) ^ ((lane >> 2) & 1)) << 4)
                                      : stg + lane * 128 + ((c8 ^ (lane & 7)) << 4);
                    *reinterpret_cast<uint4*>(dst) = w4;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && b0 < p.rows) {
                    if (mx) {
                        const int per = p.omap.dh >> 4;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int ci = (col0 >> 4) + k, tok = ci / per, jj = ci - tok * per;
                            tma_store_4d(mo, stg + k * 1024, 0, g * per + jj, tok, b0);
                        }
                    } else {
                        tma_store_3d(mo, stg, col0, g, b0);
                    }
                    bulk_commit_group();
                }
                __syncwarp();
            }
            if (BLK && !sec) pend_m = m;                              // counted once the stores complete
            return true;
        };
        int lt = 0;
        float sc = 0.f;
        // the statistics of a tile read the A slabs of this thread's half (FP8: of its whole row);
        // release them afterwards
        auto release_a = [&]() {
            __syncwarp();
            if (lane == 0) {
                if (F8) {
#pragma unroll
                    for (int qa = 0; qa < C::A_SLABS; ++qa) mbar_arrive(&a_empty[qa]);
                } else {
#pragma unroll
                    for (int qa = 0; qa < C::A_SLABS / 2; ++qa) mbar_arrive(&a_empty[half * (C::A_SLABS / 2) + qa]);
                }
            }
        };
        auto tile_scale = [&](const F128Item& t_it, float& out) -> bool {
            return F8 ? row_scale8(t_it.m, amix(t_it), out) : row_scale(t_it.m, amix(t_it), out);
        };

        F128Item it;
        bool have = item(0, it);
        bool ok = have && wait_or_abort(a_full, 0, abort_flag, 0x3300) && tile_scale(it, sc);
        if (ok) release_a();
        F128Item prev = it;
        bool prev_pending = false;                                     // prev's output is still to be written
        auto output_prev = [&](int ylt) -> bool { return output_tile(prev.g, prev.m, ylt, amix(prev), prev.sec); };
        uint32_t ubase = 0;                                            // chunks of the items before this one
        for (; ok && have; ++lt) {
            const int c0 = it.c0, c1 = it.c1;
            const float sgw = F8 ? __ldg(&(BLK && it.sec ? p.s_gate2 : p.s_gate)[it.g]) : 1.f;
            const float suw = F8 ? __ldg(&(BLK && it.sec ? p.s_up2 : p.s_up)[it.g]) : 1.f;
            // ---- SwiGLU chunks: this thread owns hidden columns [half*64, half*64 + 64) of its row
#pragma unroll 1
            for (int c = c0; c < c1; ++c) {
                const uint32_t use = ubase + (c - c0);
                if (!wait_or_abort(g1_full, use & 1, abort_flag, 0x3301)) { ok = false; break; }
                tc_fence_after();
                // all four loads in flight, one wait, then the GEMM1 buffer is released before the math
                uint32_t g0[32], u0[32], g1[32], u1[32];
                const uint32_t tg = trow + C::G1COL + half * 64;
                tmem_ld32_async(tg, g0);
                tmem_ld32_async(tg + 128, u0);
                tmem_ld32_async(tg + 32, g1);
                tmem_ld32_async(tg + 160, u1);
                tmem_wait_ld_tie(g0);
                tmem_wait_ld_tie(u0);
                tmem_wait_ld_tie(g1);
                tmem_wait_ld_tie(u1);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(g1_empty);
                uint32_t pk[32];
                // silu(sg * g) * (su * u): sg = su = 1/rms of the row; on the FP8 path the row factor
                // times the bank's gate / up weight scale
                const float hsc = 0.5f * (F8 ? sc * sgw : sc), scu = F8 ? sc * suw : sc;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 h0 = swiglu2(hsc, scu, make_float2(__uint_as_float(g0[2 * i]), __uint_as_float(g0[2 * i + 1])),
                                              make_float2(__uint_as_float(u0[2 * i]), __uint_as_float(u0[2 * i + 1])));
                    const float2 h1 = swiglu2(hsc, scu, make_float2(__uint_as_float(g1[2 * i]), __uint_as_float(g1[2 * i + 1])),
                                              make_float2(__uint_as_float(u1[2 * i]), __uint_as_float(u1[2 * i + 1])));
                    pk[i] = pack_bf16x2(h0.x, h0.y);
                    pk[16 + i] = pack_bf16x2(h1.x, h1.y);
                }
                if (c == c0 && prev_pending) {
                    // the previous item's output, now that this item's second GEMM1 can run (the
                    // buffer is released above); the hidden rows are its staging, so this chunk's
                    // hidden write waits until the bulk stores have read them
                    if (!output_prev(lt - 1)) { ok = false; break; }
                    prev_pending = false;
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                }
                if (!wait_or_abort(hid_empty, (use & 1) ^ 1, abort_flag, 0x3302)) { ok = false; break; }
                // hidden chunk: 2 K-slabs of 64 columns (128-byte swizzled rows); this half is slab `half`
                uint8_t* hrow = sH + half * 16384 + r * 128;
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    *reinterpret_cast<uint4*>(hrow + ((v ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(hid_full);
            }
            if (!ok) break;
            ubase += c1 - c0;
            prev = it;
            prev_pending = true;
            have = item(lt + 1, it);
            // Block mode, last mixing tile of this CTA: its output and count go out now, before this
            // warp waits for anything of the next item (a reverting tile's A load may wait for it).
            if (BLK && !prev.sec && (!have || it.sec)) {
                if (!output_prev(lt)) { ok = false; break; }
                prev_pending = false;
                flush_block();
            }
            // ---- statistics of the next item (its A tile is loaded once this item's last read of A is issued)
            if (have) {
                if (!wait_or_abort(a_full, (lt + 1) & 1, abort_flag, 0x3304) || !tile_scale(it, sc)) {
                    ok = false;
                    break;
                }
                release_a();
            }
        }
        if (ok && prev_pending) ok = output_prev(lt - 1);
        flush_block();
        if (lane == 0) bulk_wait_all();                                // stores complete before exit
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int W, int AMODE, bool F8 = false>
__global__ void __launch_bounds__(Fused128Cfg<W, AMODE, F8>::NTHREADS, 1)
    fused128_swiglu_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmG,
                           const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmD,
                           const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmE,
                           const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmA2,
                           const __grid_constant__ CUtensorMap tmG2, const __grid_constant__ CUtensorMap tmU2,
                           const __grid_constant__ CUtensorMap tmD2, const __grid_constant__ CUtensorMap tmO2,
                           const FusedParams p) {
    fused128_body<W, AMODE, F8>(tmA, tmG, tmU, tmD, tmR, tmE, tmO, tmA2, tmG2, tmU2, tmD2, tmO2, p);
}

}  // namespace tml
