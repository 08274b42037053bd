// tm_fused.cuh -- one kernel for a whole dense per-token SwiGLU sub-layer with row width
// W = 128 or 256:  y = SwiGLU_bank(RMSNorm(x)) + residual (+ inter-residual).
//
// Per 128-row tile of one bank the A tile (x rows, read through the Mix tensor map for the
// mixing sub-layer) stays resident in shared memory for the whole tile.  The hidden width F
// is walked in 64-wide chunks:
//   GEMM1(c): TMEM g1[c % 2] = A . [Wg; Wu][chunk c]^T       (N = 128: 64 gate + 64 up)
//   epilogue: h = silu(s*g) * (s*u), s = 1/rms of the row    -> bf16 chunk in shared memory
//   GEMM2(c): TMEM Y += h . Wd[:, chunk c]^T                 (N = W)
// and after the last chunk the epilogue adds the residual and stores Y through the row map
// (for mixed rows that store is the Revert).  The row statistics come from the resident A
// tile, so the sub-layer is one launch with no intermediate tensor in HBM.  The MMA issue
// order G1(0), G1(1), G2(0), G1(2), G2(1), ... lets the SwiGLU of chunk c overlap G1(c+1).
//
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, warps 2-9 epilogue
// (TMEM lane quarter = warp % 4, warps 2-5 and 6-9 split the columns in two halves).
#pragma once
#include "tm_gemm.cuh"

namespace tml {

struct FusedParams {
    int banks, rows, F;        // groups (banks), rows per group (B), hidden width
    RowMap amap;               // x rows
    float eps;
    __nv_bfloat16* out;        // y (omap)
    const __nv_bfloat16* resid;
    const __nv_bfloat16* extra;
    RowMap omap;
    size_t out_elems;
    int res_mode;              // 128-wide-chunk kernel: residual none / from the A tile / streamed (FusedResid)
    int has_extra;             // 128-wide-chunk kernel: inter-residual streamed
    // Whole dense block in one launch (128-wide-chunk kernel, block mode): the fields above describe
    // the mixing sub-layer, these the reverting one (same banks and row width).
    int F2;                    // reverting hidden width
    int res_mode2, has_extra2; // reverting residual (streamed) and inter-residual
    unsigned* dep;             // [row tiles] finished-mixing-tile counters, zero at launch
    // FP8 GEMM1 (128-wide-chunk kernel, F8): per bank the gate / up weight matrix scales of the
    // (first) sub-layer, and of the reverting one in block mode
    const float* s_gate;
    const float* s_up;
    const float* s_gate2;
    const float* s_up2;
};

// Output epilogue of a fused tile for one thread: row b of bank g, columns [c_begin, c_begin + W/2).
// The residual segment is loaded into registers before the accumulator is ready (all loads in
// flight at once: a thread's row is spread over W/16 separate 16-byte pieces in memory), then
// each 32-column TMEM slice is added to it and stored through the row map.
template <int W>
struct YEpilogue {
    uint4 rv[W / 16];
    __device__ __forceinline__ void prefetch(const FusedParams& p, int b, int g, int c_begin, bool valid) {
#pragma unroll
        for (int i = 0; i < W / 16; ++i) {
            rv[i] = make_uint4(0, 0, 0, 0);
            if (valid && p.resid) {
                const size_t off = row_elem(p.omap, b, g, c_begin + 8 * i);
                if (off + 8 <= p.out_elems) rv[i] = __ldg(reinterpret_cast<const uint4*>(p.resid + off));
            }
        }
    }
    __device__ __forceinline__ void store(const FusedParams& p, uint32_t tmem_row, int b, int g, int c_begin, bool valid) {
#pragma unroll
        for (int j = 0; j < W / 64; ++j) {
            float v[32];
            tmem_ld32(tmem_row + c_begin + 32 * j, v);
            if (!valid) continue;
            uint4 ev[4];
            size_t off[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                off[i] = row_elem(p.omap, b, g, c_begin + 32 * j + 8 * i);
                ev[i] = make_uint4(0, 0, 0, 0);
                if (p.extra && off[i] + 8 <= p.out_elems) ev[i] = __ldg(reinterpret_cast<const uint4*>(p.extra + off[i]));
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (off[i] + 8 > p.out_elems) {
                    record_error(ERR_BOUNDS, 0x1310);
                    continue;
                }
                const uint4 r4 = rv[4 * j + i];
                const uint32_t rw[4] = {r4.x, r4.y, r4.z, r4.w};
                const uint32_t ew[4] = {ev[i].x, ev[i].y, ev[i].z, ev[i].w};
                float o[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    o[2 * e] = v[8 * i + 2 * e] + bf16_lo(rw[e]) + bf16_lo(ew[e]);
                    o[2 * e + 1] = v[8 * i + 2 * e + 1] + bf16_hi(rw[e]) + bf16_hi(ew[e]);
                }
                *reinterpret_cast<uint4*>(p.out + off[i]) = make_uint4(
                    pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
            }
        }
    }
};

template <int W, int AMODE>
struct FusedCfg {
    static_assert(W == 128 || W == 256, "fused sub-layer supports row widths 128 and 256");
    static constexpr int A_BYTES = 128 * W * 2;
    static constexpr int HID_BYTES = 128 * 64 * 2;              // one 64-wide hidden chunk
    static constexpr int SB = W * 128;                          // ring stage: W rows x 64 K, or 128 rows x W/2 K
    static constexpr int STAGES = W == 256 ? 4 : 8;
    static constexpr int NTHREADS = 10 * 32;
    static constexpr int OFF_HID = A_BYTES;
    static constexpr int OFF_RING = A_BYTES + 2 * HID_BYTES;
    static constexpr int OFF_BAR = OFF_RING + STAGES * SB;
    static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
    static constexpr int G1COL = W;                             // TMEM: Y at [0, W), g1 buffers after
};

template <int W, int AMODE>
__global__ void __launch_bounds__(FusedCfg<W, AMODE>::NTHREADS, 1)
    fused_swiglu_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmG,
                        const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmD,
                        const FusedParams p) {
    using C = FusedCfg<W, AMODE>;
    constexpr int STAGES = C::STAGES;
    const int mt = (p.rows + 127) / 128;
    const int ntile = p.banks * mt;
    if ((int)blockIdx.x >= ntile) return;
    const int NC = p.F / 64;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sH = smem + C::OFF_HID;
    uint8_t* sR = smem + C::OFF_RING;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bar;                  // [STAGES]
    uint64_t* empty = full + STAGES;       // [STAGES]
    uint64_t* a_full = empty + STAGES;
    uint64_t* a_empty = a_full + 1;
    uint64_t* g1_full = a_empty + 1;       // [2]
    uint64_t* g1_empty = g1_full + 2;      // [2]
    uint64_t* hid_full = g1_empty + 2;     // [2]
    uint64_t* hid_empty = hid_full + 2;    // [2]
    uint64_t* y_full = hid_empty + 2;
    uint64_t* y_empty = y_full + 1;
    uint64_t* drain = y_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(a_full, 1);
        mbar_init(a_empty, 1 + 8);             // MMA (last GEMM1 done) + each epilogue warp (statistics read)
        for (int b = 0; b < 2; ++b) {
            mbar_init(&g1_full[b], 1);
            mbar_init(&g1_empty[b], 8);
            mbar_init(&hid_full[b], 8);
            mbar_init(&hid_empty[b], 1);
        }
        mbar_init(y_full, 1);
        mbar_init(y_empty, 8);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
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
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            for (int t = blockIdx.x; t < ntile; t += gridDim.x, ++lt) {
                const int g = t / mt, m = t - g * mt;
                if (!wait_or_abort(a_empty, (lt & 1) ^ 1, abort_flag, 0x1100)) break;
                mbar_arrive_expect_tx(a_full, C::A_BYTES);
                if (AMODE == A_TMA_MIX) {
                    const int per = p.amap.dh >> 4;
#pragma unroll 1
                    for (int i = 0; i < W / 16; ++i) {
                        const int tok = i / per, jj = i - tok * per;
                        tma_load_4d(sA + i * 4096, &tmA, a_full, 0, g * per + jj, tok, m * 128);
                    }
                } else {
#pragma unroll 1
                    for (int i = 0; i < W / 64; ++i) tma_load_3d(sA + i * 16384, &tmA, a_full, i * 64, g, m * 128);
                }
                // weight stream in MMA order: G1(0), then per chunk c: G1(c+1), G2(c)
                auto load_g1 = [&](int c) -> bool {
#pragma unroll 1
                    for (int q = 0; q < 2; ++q) {
                        if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x1101)) return false;
                        uint8_t* st = sR + s * C::SB;
                        mbar_arrive_expect_tx(&full[s], C::SB);
#pragma unroll
                        for (int j = 0; j < W / 128; ++j) {
                            const int kc = q * (W / 2) + j * 64;
                            tma_load_2d(st + j * 16384, &tmG, &full[s], kc, g * p.F + c * 64);
                            tma_load_2d(st + j * 16384 + 8192, &tmU, &full[s], kc, g * p.F + c * 64);
                        }
                        if (++s == STAGES) { s = 0; ph ^= 1; }
                    }
                    return true;
                };
                auto load_g2 = [&](int c) -> bool {
                    if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x1102)) return false;
                    uint8_t* st = sR + s * C::SB;
                    mbar_arrive_expect_tx(&full[s], C::SB);
                    tma_load_2d(st, &tmD, &full[s], c * 64, g * W);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                    return true;
                };
                bool ok = load_g1(0);
                for (int c = 0; c < NC && ok; ++c) {
                    if (c + 1 < NC) ok = load_g1(c + 1);
                    if (ok) ok = load_g2(c);
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // Buffer b (= chunk & 1) is used cnt_b = (NC + 1 - b) / 2 times per tile, so the use index of
        // chunk c in the tile lt is lt * cnt_b + c / 2; barrier parities follow from it (no arrays).
        if (lane == 0) {
            constexpr uint32_t idesc1 = umma_idesc_bf16(128, 128);
            constexpr uint32_t idesc2 = umma_idesc_bf16(128, W);
            const uint32_t cnt0 = (NC + 1) >> 1, cnt1 = NC >> 1;
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            bool ok = true;
            const uint32_t aS = smem_u32(sA);
            for (int t = blockIdx.x; t < ntile && ok; t += gridDim.x, ++lt) {
                if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x1200)) break;
                tc_fence_after();
                // chunk order: G1(0), then for c: G1(c+1), G2(c)
#pragma unroll 1
                for (int step = -1; step < NC && ok; ++step) {
                    // ---- GEMM1 of chunk c1 = step + 1
                    const int c1 = step + 1;
                    if (c1 < NC) {
                        const int b = c1 & 1;
                        const uint32_t use = lt * (b ? cnt1 : cnt0) + (c1 >> 1);
                        if (!wait_or_abort(&g1_empty[b], (use & 1) ^ 1, abort_flag, 0x1201)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t d = tmem + C::G1COL + b * 128;
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            if (!wait_or_abort(&full[s], ph, abort_flag, 0x1202)) { ok = false; break; }
                            tc_fence_after();
                            const uint32_t st = smem_u32(sR + s * C::SB);
#pragma unroll
                            for (int kk = 0; kk < W / 32; ++kk) {
                                const int k16 = q * (W / 32) + kk;
                                const uint64_t ad = AMODE == A_TMA_MIX ? umma_sdesc_sw32(aS + k16 * 4096)
                                                                       : umma_sdesc_sw128(aS + (k16 >> 2) * 16384) + 2 * (k16 & 3);
                                const uint64_t bd = umma_sdesc_sw128(st + (kk >> 2) * 16384) + 2 * (kk & 3);
                                umma_bf16(d, ad, bd, idesc1, (q | kk) != 0);
                            }
                            umma_commit(&empty[s]);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                        umma_commit(&g1_full[b]);
                        if (c1 == NC - 1) umma_commit(a_empty);       // last read of the A tile issued
                    }
                    // ---- GEMM2 of chunk c2 = step
                    const int c2 = step;
                    if (c2 >= 0) {
                        const int b = c2 & 1;
                        const uint32_t use = lt * (b ? cnt1 : cnt0) + (c2 >> 1);
                        if (!wait_or_abort(&hid_full[b], use & 1, abort_flag, 0x1203)) { ok = false; break; }
                        if (c2 == 0 && !wait_or_abort(y_empty, (lt & 1) ^ 1, abort_flag, 0x1204)) { ok = false; break; }
                        if (!wait_or_abort(&full[s], ph, abort_flag, 0x1205)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t st = smem_u32(sR + s * C::SB);
                        const uint64_t hd = umma_sdesc_sw128(smem_u32(sH + b * C::HID_BYTES));
                        const uint64_t bd = umma_sdesc_sw128(st);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) umma_bf16(tmem, hd + 2 * kk, bd + 2 * kk, idesc2, (c2 | kk) != 0);
                        umma_commit(&empty[s]);
                        umma_commit(&hid_empty[b]);
                        if (++s == STAGES) { s = 0; ph ^= 1; }
                        if (c2 == NC - 1) umma_commit(y_full);
                    }
                }
            }
            umma_commit(drain);
            wait_or_abort(drain, 0, abort_flag, 0x1206);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-9)
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        const uint32_t cnt0 = (NC + 1) >> 1, cnt1 = NC >> 1;
        int lt = 0;
        for (int t = blockIdx.x; t < ntile; t += gridDim.x, ++lt) {
            const int g = t / mt, m = t - g * mt;
            const int nrows = min(128, p.rows - m * 128);
            const bool valid = r < nrows;
            const int b = m * 128 + r;
            if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x1300)) break;
            // ---- row statistics from the resident A tile (each epilogue warp reads its rows in full)
            float ss = 0.f;
            if (AMODE == A_TMA_MIX) {
#pragma unroll 1
                for (int i = 0; i < W / 16; ++i) {
                    const uint4* rp = reinterpret_cast<const uint4*>(sA + i * 4096 + r * 32);
#pragma unroll
                    for (int v = 0; v < 2; ++v) {
                        // logical half v (stored at v ^ ((r / 4) % 2) by the 32-byte swizzle): both
                        // halves and every row position sum in column order
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
                for (int i = 0; i < W / 64; ++i) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const uint4 w4 = *reinterpret_cast<const uint4*>(sA + i * 16384 + r * 128 + (((v ^ r) & 7) << 4));
                        const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo = bf16_lo(wv[e]), hi = bf16_hi(wv[e]);
                            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                        }
                    }
                }
            }
            const float sc = valid ? 1.0f / sqrtf(ss / (float)W + p.eps) : 0.f;
            __syncwarp();
            if (lane == 0) mbar_arrive(a_empty);
            // ---- SwiGLU chunks
            bool ok = true;
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                const int bb = c & 1;
                const uint32_t use = lt * (bb ? cnt1 : cnt0) + (c >> 1);
                if (!wait_or_abort(&g1_full[bb], use & 1, abort_flag, 0x1301)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + C::G1COL + bb * 128 + half * 32;
                float gv[32], uv[32];
                tmem_ld32(ta, gv);
                tmem_ld32(ta + 64, uv);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&g1_empty[bb]);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(silu_tanh(sc * gv[2 * i]) * (sc * uv[2 * i]),
                                        silu_tanh(sc * gv[2 * i + 1]) * (sc * uv[2 * i + 1]));
                if (!wait_or_abort(&hid_empty[bb], (use & 1) ^ 1, abort_flag, 0x1302)) { ok = false; break; }
                uint8_t* hrow = sH + bb * C::HID_BYTES + r * 128;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int chunk = half * 4 + v;
                    *reinterpret_cast<uint4*>(hrow + ((chunk ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&hid_full[bb]);
            }
            if (!ok) break;
            // ---- output tile: Y + residual (+ inter-residual), stored through the row map
            YEpilogue<W> ye;
            ye.prefetch(p, b, g, half * (W / 2), valid);
            if (!wait_or_abort(y_full, lt & 1, abort_flag, 0x1303)) break;
            tc_fence_after();
            ye.store(p, tmem + (uint32_t(q * 32) << 16), b, g, half * (W / 2), valid);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(y_empty);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tml
