// tm_fused128.cuh -- the fused dense sub-layer (row width W = 128 or 256, hidden F % 128 == 0)
// with 128-wide hidden chunks:  y = SwiGLU_bank(RMSNorm(x)) + residual (+ inter-residual).
//
// Per 128-row tile the A tile stays resident in shared memory.  For each 128-wide hidden chunk c:
//   GEMM1(c): TMEM g1 = A . [Wg; Wu][chunk c]^T   (N = 256: 128 gate + 128 up)
//   epilogue: h = silu(s*g) * (s*u)  -> bf16 chunk in shared memory (s = 1/rms of the row)
//   GEMM2(c): TMEM Y += h . Wd[:, chunk c]^T       (N = W, K = 128)
// issued in the order G1(0), G1(1), G2(0), G1(2), G2(1), ...: the epilogue copies g1 out of TMEM
// while the tensor pipe runs G2(c-1) (so GEMM1 needs only one TMEM buffer) and computes the
// SwiGLU while it runs G1(c+1).  TMEM: Y in columns [0, W), the GEMM1 buffer in [256, 512).
//
// The output epilogue is coalesced: residual slices are read 8 rows per warp instruction (4 lanes
// per 64-byte row piece), prefetched before the accumulator is ready, transposed to one row per
// thread through the warp's own rows of the (then idle) hidden buffer, added to the accumulator
// in fp32 with a single rounding, and written back the same way.
//
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, warps 2-9 epilogue
// (TMEM lane quarter = warp % 4; warps 2-5 / 6-9 take the two column halves).
#pragma once
#include "tm_fused.cuh"

namespace tml {

template <int W, int AMODE>
struct Fused128Cfg {
    static_assert(W == 128 || W == 256, "fused sub-layer supports row widths 128 and 256");
    static constexpr int A_BYTES = 128 * W * 2;
    static constexpr int HID_BYTES = 128 * 128 * 2;               // one 128-wide hidden chunk, 2 K-slabs
    static constexpr int SB = 32768;                              // ring stage
    static constexpr int G1_STAGES = W / 64;                      // 256 rows x 64 K per stage
    static constexpr int G2_STAGES = W == 256 ? 2 : 1;            // W rows x 128 K per chunk
    static constexpr int STAGES = W == 256 ? 4 : 5;
    static constexpr int NTHREADS = 10 * 32;
    static constexpr int OFF_HID = A_BYTES;
    static constexpr int OFF_RING = A_BYTES + HID_BYTES;
    static constexpr int OFF_BAR = OFF_RING + STAGES * SB;
    static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
    static constexpr int G1COL = 256;
    static_assert(2 * 32 * 64 <= 4096, "output staging (residual + inter-residual) fits in a warp's hidden rows");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int W, int AMODE>
__global__ void __launch_bounds__(Fused128Cfg<W, AMODE>::NTHREADS, 1)
    fused128_swiglu_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmG,
                           const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmD,
                           const FusedParams p) {
    using C = Fused128Cfg<W, AMODE>;
    constexpr int STAGES = C::STAGES;
    const int mt = (p.rows + 127) / 128;
    const int ntile = p.banks * mt;
    if ((int)blockIdx.x >= ntile) return;
    const int NC = p.F / 128;

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
    uint64_t* g1_full = a_empty + 1;
    uint64_t* g1_empty = g1_full + 1;
    uint64_t* hid_full = g1_empty + 1;
    uint64_t* hid_empty = hid_full + 1;
    uint64_t* y_full = hid_empty + 1;
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
        mbar_init(g1_full, 1);
        mbar_init(g1_empty, 8);
        mbar_init(hid_full, 8);
        mbar_init(hid_empty, 1);
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
            bool ok = true;
            for (int t = blockIdx.x; t < ntile && ok; t += gridDim.x, ++lt) {
                const int g = t / mt, m = t - g * mt;
                if (!wait_or_abort(a_empty, (lt & 1) ^ 1, abort_flag, 0x3100)) break;
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
                // weights in MMA order: G1(0); then for c >= 1: G1(c), G2(c-1); finally G2(NC-1)
#pragma unroll 1
                for (int step = 0; step <= NC && ok; ++step) {
                    if (step < NC) {
                        const int c = step;
#pragma unroll 1
                        for (int q = 0; q < C::G1_STAGES; ++q) {             // K slab q: 128 gate + 128 up rows
                            if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x3101)) { ok = false; break; }
                            uint8_t* st = sR + s * C::SB;
                            mbar_arrive_expect_tx(&full[s], C::SB);
                            tma_load_2d(st, &tmG, &full[s], q * 64, g * p.F + c * 128);
                            tma_load_2d(st + 16384, &tmU, &full[s], q * 64, g * p.F + c * 128);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                    }
                    if (step >= 1 && ok) {
                        const int c = step - 1;
#pragma unroll 1
                        for (int q = 0; q < C::G2_STAGES; ++q) {
                            if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x3102)) { ok = false; break; }
                            uint8_t* st = sR + s * C::SB;
                            mbar_arrive_expect_tx(&full[s], C::SB);
                            if (W == 256) {
                                tma_load_2d(st, &tmD, &full[s], c * 128 + q * 64, g * W);          // 256 rows x 64 K
                            } else {
                                tma_load_2d(st, &tmD, &full[s], c * 128, g * W);                   // 128 rows x 64 K
                                tma_load_2d(st + 16384, &tmD, &full[s], c * 128 + 64, g * W);      // next 64 K
                            }
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc1 = umma_idesc_bf16(128, 256);
            constexpr uint32_t idesc2 = umma_idesc_bf16(128, W);
            const uint32_t aS = smem_u32(sA), hS = smem_u32(sH), rS = smem_u32(sR);
            uint64_t adesc[W / 16];
#pragma unroll
            for (int k16 = 0; k16 < W / 16; ++k16)
                adesc[k16] = AMODE == A_TMA_MIX ? umma_sdesc_sw32(aS + k16 * 4096)
                                                : umma_sdesc_sw128(aS + (k16 >> 2) * 16384) + 2 * (k16 & 3);
            const uint64_t hdesc0 = umma_sdesc_sw128(hS), hdesc1 = umma_sdesc_sw128(hS + 16384);
            const uint64_t rdesc0 = umma_sdesc_sw128(rS);
            constexpr uint64_t kStageDesc = C::SB >> 4;               // descriptor start-address step per stage
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntile && ok; t += gridDim.x, ++lt) {
                if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x3200)) break;
                tc_fence_after();
#pragma unroll 1
                for (int step = 0; step <= NC && ok; ++step) {
                    if (step < NC) {                                   // ---- GEMM1(step)
                        const uint32_t use = lt * NC + step;
                        if (!wait_or_abort(g1_empty, (use & 1) ^ 1, abort_flag, 0x3201)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int q = 0; q < C::G1_STAGES; ++q) {
                            if (!wait_or_abort(&full[s], ph, abort_flag, 0x3202)) { ok = false; break; }
                            tc_fence_after();
                            const uint64_t bd = rdesc0 + (uint64_t)s * kStageDesc;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_bf16(tmem + C::G1COL, adesc[q * 4 + kk], bd + 2 * kk, idesc1, (q | kk) != 0);
                            umma_commit(&empty[s]);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                        umma_commit(g1_full);
                        if (step == NC - 1) umma_commit(a_empty);
                    }
                    if (step >= 1) {                                   // ---- GEMM2(step - 1)
                        const int c = step - 1;
                        const uint32_t use = lt * NC + c;
                        if (!wait_or_abort(hid_full, use & 1, abort_flag, 0x3203)) { ok = false; break; }
                        if (c == 0 && !wait_or_abort(y_empty, (lt & 1) ^ 1, abort_flag, 0x3204)) { ok = false; break; }
#pragma unroll
                        for (int q = 0; q < C::G2_STAGES; ++q) {
                            if (!wait_or_abort(&full[s], ph, abort_flag, 0x3205)) { ok = false; break; }
                            tc_fence_after();
                            const uint64_t bd = rdesc0 + (uint64_t)s * kStageDesc;
#pragma unroll
                            for (int kq = 0; kq < (W == 256 ? 1 : 2); ++kq) {   // 64-wide K slabs in this stage
                                const uint64_t hd = ((q + kq) ? hdesc1 : hdesc0);
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_bf16(tmem, hd + 2 * kk, bd + kq * (16384 >> 4) + 2 * kk, idesc2,
                                              (c | q | kq | kk) != 0);
                            }
                            umma_commit(&empty[s]);
                            if (++s == STAGES) { s = 0; ph ^= 1; }
                        }
                        if (!ok) break;
                        umma_commit(hid_empty);
                        if (c == NC - 1) umma_commit(y_full);
                    }
                }
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
        // output staging: inside this warp's own 32 rows of the hidden buffer (4 KB per half and
        // lane quarter), which no other warp writes and the MMA no longer reads after y_full
        uint8_t* stg = sH + half * 16384 + q * 4096;
        int lt = 0;
        for (int t = blockIdx.x; t < ntile; t += gridDim.x, ++lt) {
            const int g = t / mt, m = t - g * mt;
            const int nrows = min(128, p.rows - m * 128);
            const bool valid = r < nrows;
            if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x3300)) break;
            // ---- row statistics from the resident A tile (each warp reads its rows in full)
            float ss = 0.f;
            if (AMODE == A_TMA_MIX) {
#pragma unroll 4
                for (int i = 0; i < W / 16; ++i) {
                    const uint4* rp = reinterpret_cast<const uint4*>(sA + i * 4096 + r * 32);
#pragma unroll
                    for (int v = 0; v < 2; ++v) {
                        const uint4 w4 = rp[v ^ half];
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
            // ---- SwiGLU chunks: this thread owns hidden columns [half*64, half*64 + 64) of its row
            bool ok = true;
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                const uint32_t use = lt * NC + c;
                if (!wait_or_abort(g1_full, use & 1, abort_flag, 0x3301)) { ok = false; break; }
                tc_fence_after();
                uint32_t pk[32];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float gv[32], uv[32];
                    tmem_ld32(trow + C::G1COL + half * 64 + hh * 32, gv);
                    tmem_ld32(trow + C::G1COL + 128 + half * 64 + hh * 32, uv);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[hh * 16 + i] = pack_bf16x2(silu_tanh(sc * gv[2 * i]) * (sc * uv[2 * i]),
                                                      silu_tanh(sc * gv[2 * i + 1]) * (sc * uv[2 * i + 1]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(g1_empty);
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
            // ---- output tile, coalesced: lane l moves 16 bytes of row (i*8 + l/4) of a 32-column slice.
            // Staging rows are 64 bytes with the 16-byte piece index XORed by (row / 2) % 4, so both the
            // 8-rows-per-instruction phase and the row-per-thread phase are free of bank conflicts.
            const int c_begin = half * (W / 2);
            const int b_warp = m * 128 + q * 32;                      // first row of this warp
            const int lr = lane >> 2, lp = lane & 3;
            uint8_t* stg_e = stg + 32 * 64;                            // inter-residual slice
            uint4 rv[W / 16];                                          // W/64 slices x 4 row groups
#pragma unroll
            for (int j = 0; j < W / 64; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = i * 8 + lr;
                    rv[j * 4 + i] = make_uint4(0, 0, 0, 0);
                    if (p.resid && q * 32 + rr < nrows) {
                        const size_t off = row_elem(p.omap, b_warp + rr, g, c_begin + j * 32 + lp * 8);
                        if (off + 8 <= p.out_elems) rv[j * 4 + i] = __ldg(reinterpret_cast<const uint4*>(p.resid + off));
                    }
                }
            if (!wait_or_abort(y_full, lt & 1, abort_flag, 0x3303)) break;
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < W / 64; ++j) {
                float v[32];
                tmem_ld32(trow + c_begin + j * 32, v);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = i * 8 + lr;
                    const int so = rr * 64 + ((lp ^ ((rr >> 1) & 3)) << 4);
                    *reinterpret_cast<uint4*>(stg + so) = rv[j * 4 + i];
                    if (p.extra) {
                        uint4 e4 = make_uint4(0, 0, 0, 0);
                        if (q * 32 + rr < nrows) {
                            const size_t off = row_elem(p.omap, b_warp + rr, g, c_begin + j * 32 + lp * 8);
                            if (off + 8 <= p.out_elems) e4 = __ldg(reinterpret_cast<const uint4*>(p.extra + off));
                        }
                        *reinterpret_cast<uint4*>(stg_e + so) = e4;
                    }
                }
                __syncwarp();
                // one row per thread: Y + residual (+ inter-residual) in fp32, one rounding, back in place
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    const int so = lane * 64 + ((pp ^ ((lane >> 1) & 3)) << 4);
                    const uint4 x4 = *reinterpret_cast<const uint4*>(stg + so);
                    const uint4 e4 = p.extra ? *reinterpret_cast<const uint4*>(stg_e + so) : make_uint4(0, 0, 0, 0);
                    const uint32_t a[4] = {x4.x, x4.y, x4.z, x4.w}, e[4] = {e4.x, e4.y, e4.z, e4.w};
                    uint32_t o[4];
#pragma unroll
                    for (int z = 0; z < 4; ++z)
                        o[z] = pack_bf16x2(v[pp * 8 + 2 * z] + bf16_lo(a[z]) + bf16_lo(e[z]),
                                           v[pp * 8 + 2 * z + 1] + bf16_hi(a[z]) + bf16_hi(e[z]));
                    *reinterpret_cast<uint4*>(stg + so) = make_uint4(o[0], o[1], o[2], o[3]);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = i * 8 + lr;
                    if (q * 32 + rr >= nrows) continue;
                    const size_t off = row_elem(p.omap, b_warp + rr, g, c_begin + j * 32 + lp * 8);
                    if (off + 8 > p.out_elems) {
                        record_error(ERR_BOUNDS, 0x3310);
                        continue;
                    }
                    *reinterpret_cast<uint4*>(p.out + off) =
                        *reinterpret_cast<const uint4*>(stg + rr * 64 + ((lp ^ ((rr >> 1) & 3)) << 4));
                }
                __syncwarp();
            }
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
