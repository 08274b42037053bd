// tm_fused2.cuh -- the fused dense sub-layer (row width W = 128 or 256) on CTA pairs with
// 2-SM tensor-core MMAs:  y = SwiGLU_bank(RMSNorm(x)) + residual (+ inter-residual).
//
// Same dataflow as tm_fused.cuh, but a cluster of two CTAs on two SMs works on 256 rows of one
// bank (each CTA owns 128 rows: its A tile, its hidden chunks, its TMEM accumulators) and every
// weight tile is split between them: in GEMM1 the leader CTA holds the 64 gate rows of a chunk
// and the peer the 64 up rows; in GEMM2 each holds half of the W output rows of Wd.  One
// tcgen05.mma.cta_group::2 issued by the leader then computes M=256 rows.  Each SM streams half
// the weight bytes per chunk, so the same shared-memory ring hides twice the latency.
//
// Synchronisation: the leader's MMA thread waits on barriers in the leader CTA; the peer's TMA
// loads count their bytes on the leader's stage barriers (cta_group::2 completion), its
// epilogue warps arrive on the leader's barriers through mapa addresses, and the MMA commits
// signal the barriers of both CTAs.  No load or commit uses multicast.
#pragma once
#include "tm_fused.cuh"

namespace tml {

template <int W, int AMODE>
struct Fused2Cfg {
    static_assert(W == 128 || W == 256, "fused sub-layer supports row widths 128 and 256");
    static constexpr int A_BYTES = 128 * W * 2;
    static constexpr int HID_BYTES = 128 * 64 * 2;
    static constexpr int SB = W * 64;                           // per CTA: 64 rows x W/2 K, or W/2 rows x 64 K
    static constexpr int STAGES = W == 256 ? 8 : 16;
    static constexpr int NTHREADS = 10 * 32;
    static constexpr int OFF_HID = A_BYTES;
    static constexpr int OFF_RING = A_BYTES + 2 * HID_BYTES;
    static constexpr int OFF_BAR = OFF_RING + STAGES * SB;
    static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
    static constexpr int G1COL = W;
};

__device__ __forceinline__ bool wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort_flag, unsigned where) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(ERR_TIMEOUT, where);
            *abort_flag = 1;
            return false;
        }
    }
}

template <int W, int AMODE>
__global__ void __launch_bounds__(Fused2Cfg<W, AMODE>::NTHREADS, 1)
    fused2_swiglu_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmG,
                         const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmD,
                         const FusedParams p) {
    using C = Fused2Cfg<W, AMODE>;
    constexpr int STAGES = C::STAGES;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int mt = (p.rows + 127) / 128;
    const int mt2 = (mt + 1) / 2;
    const int npt = p.banks * mt2;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    if (pair >= npt) return;                 // both CTAs of a cluster share `pair`
    const int NC = p.F / 64;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sH = smem + C::OFF_HID;
    uint8_t* sR = smem + C::OFF_RING;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bar;                  // [STAGES]  leader: both CTAs' stage bytes
    uint64_t* empty = full + STAGES;       // [STAGES]  each CTA: MMA done with the stage
    uint64_t* a_full = empty + STAGES;     // each CTA: own A tile landed
    uint64_t* a_ready = a_full + 1;        // leader: peer's A tile landed (relayed)
    uint64_t* a_empty = a_ready + 1;       // each CTA: MMA + own epilogue done with A
    uint64_t* g1_full = a_empty + 1;       // [2] each CTA
    uint64_t* g1_empty = g1_full + 2;      // [2] leader: 8 warps x 2 CTAs
    uint64_t* hid_full = g1_empty + 2;     // [2] leader: 8 warps x 2 CTAs
    uint64_t* hid_empty = hid_full + 2;    // [2] each CTA
    uint64_t* y_full = hid_empty + 2;      // each CTA
    uint64_t* y_empty = y_full + 1;        // leader: 8 warps x 2 CTAs
    uint64_t* drain = y_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto L = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 0); };   // leader's copy
    auto P = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 1); };   // peer's copy

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(a_full, 1);
        mbar_init(a_ready, 1);
        mbar_init(a_empty, 1 + 8);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&g1_full[b], 1);
            mbar_init(&g1_empty[b], 16);
            mbar_init(&hid_full[b], 16);
            mbar_init(&hid_empty[b], 1);
        }
        mbar_init(y_full, 1);
        mbar_init(y_empty, 16);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();                      // both CTAs' barriers exist before any remote use
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(leader ? &tmG : &tmU);
            tma_prefetch_desc(&tmD);
            const CUtensorMap* tmGU = leader ? &tmG : &tmU;     // leader: gate rows, peer: up rows
            int s = 0;
            uint32_t ph = 0;
            int lt = 0;
            for (int pt = pair; pt < npt; pt += npairs, ++lt) {
                const int g = pt / mt2, m = 2 * (pt - g * mt2) + (int)rank;
                if (!wait_or_abort(a_empty, (lt & 1) ^ 1, abort_flag, 0x2100)) break;
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
                auto stage_begin = [&]() -> uint8_t* {
                    if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, 0x2101)) return nullptr;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::SB);
                    return sR + s * C::SB;
                };
                auto stage_end = [&]() { if (++s == STAGES) { s = 0; ph ^= 1; } };
                auto load_g1 = [&](int c) -> bool {
#pragma unroll 1
                    for (int q = 0; q < 2; ++q) {
                        uint8_t* st = stage_begin();
                        if (!st) return false;
                        const uint32_t fb = L(&full[s]);
#pragma unroll
                        for (int j = 0; j < W / 128; ++j)
                            tma_load_2d_pair(st + j * 8192, tmGU, fb, q * (W / 2) + j * 64, g * p.F + c * 64);
                        stage_end();
                    }
                    return true;
                };
                auto load_g2 = [&](int c) -> bool {
                    uint8_t* st = stage_begin();
                    if (!st) return false;
                    tma_load_2d_pair(st, &tmD, L(&full[s]), c * 64, g * W + (int)rank * (W / 2));
                    stage_end();
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
        if (!leader) {
            // ---------------------------------------------------------------- peer: relay "A landed"
            if (lane == 0) {
                int lt = 0;
                for (int pt = pair; pt < npt; pt += npairs, ++lt) {
                    if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x2200)) break;
                    mbar_arrive_cluster(L(a_ready));
                }
            }
        } else if (lane == 0) {
            // ---------------------------------------------------------------- leader: MMA issuer
            constexpr uint32_t idesc1 = umma_idesc_bf16(256, 128);
            constexpr uint32_t idesc2 = umma_idesc_bf16(256, W);
            int s = 0;
            uint32_t ph = 0;
            uint32_t u1[2] = {0, 0}, u2[2] = {0, 0};
            int lt = 0;
            bool ok = true;
            auto commit_both = [&](uint64_t* b) {
                umma_commit_pair(L(b));
                umma_commit_pair(P(b));
            };
            for (int pt = pair; pt < npt && ok; pt += npairs, ++lt) {
                if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x2300)) break;
                if (!wait_cl(a_ready, lt & 1, abort_flag, 0x2301)) break;
                tc_fence_after();
                const uint32_t aS = smem_u32(sA);
                auto gemm1 = [&](int c) -> bool {
                    const int b = c & 1;
                    if (!wait_cl(&g1_empty[b], (u1[b] & 1) ^ 1, abort_flag, 0x2302)) return false;
                    tc_fence_after();
                    const uint32_t d = tmem + C::G1COL + b * 128;
                    for (int q = 0; q < 2; ++q) {
                        if (!wait_cl(&full[s], ph, abort_flag, 0x2303)) return false;
                        tc_fence_after();
                        const uint32_t st = smem_u32(sR + s * C::SB);
#pragma unroll
                        for (int kk = 0; kk < W / 32; ++kk) {
                            const int k16 = q * (W / 32) + kk;
                            const uint64_t ad = AMODE == A_TMA_MIX ? umma_sdesc_sw32(aS + k16 * 4096)
                                                                   : umma_sdesc_sw128(aS + (k16 >> 2) * 16384) + 2 * (k16 & 3);
                            const uint64_t bd = umma_sdesc_sw128(st + (kk >> 2) * 8192) + 2 * (kk & 3);
                            umma_bf16_pair(d, ad, bd, idesc1, (q | kk) != 0);
                        }
                        commit_both(&empty[s]);
                        if (++s == STAGES) { s = 0; ph ^= 1; }
                    }
                    commit_both(&g1_full[b]);
                    ++u1[b];
                    return true;
                };
                auto gemm2 = [&](int c) -> bool {
                    const int b = c & 1;
                    if (!wait_cl(&hid_full[b], u2[b] & 1, abort_flag, 0x2304)) return false;
                    if (c == 0 && !wait_cl(y_empty, (lt & 1) ^ 1, abort_flag, 0x2305)) return false;
                    if (!wait_cl(&full[s], ph, abort_flag, 0x2306)) return false;
                    tc_fence_after();
                    const uint32_t st = smem_u32(sR + s * C::SB);
                    const uint64_t hd = umma_sdesc_sw128(smem_u32(sH + b * C::HID_BYTES));
                    const uint64_t bd = umma_sdesc_sw128(st);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) umma_bf16_pair(tmem, hd + 2 * kk, bd + 2 * kk, idesc2, (c | kk) != 0);
                    commit_both(&empty[s]);
                    commit_both(&hid_empty[b]);
                    ++u2[b];
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                    return true;
                };
                ok = gemm1(0);
                if (ok && NC == 1) commit_both(a_empty);
                for (int c = 0; c < NC && ok; ++c) {
                    if (c + 1 < NC) {
                        ok = gemm1(c + 1);
                        if (ok && c + 1 == NC - 1) commit_both(a_empty);
                    }
                    if (ok) ok = gemm2(c);
                }
                if (ok) commit_both(y_full);
            }
            umma_commit_pair(L(drain));
            wait_or_abort(drain, 0, abort_flag, 0x2307);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-9, both CTAs)
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        uint32_t u1[2] = {0, 0}, u2[2] = {0, 0};
        int lt = 0;
        for (int pt = pair; pt < npt; pt += npairs, ++lt) {
            const int g = pt / mt2, m = 2 * (pt - g * mt2) + (int)rank;
            const int nrows = min(128, p.rows - m * 128);       // <= 0 for the peer's tile past the end
            const bool valid = r < nrows;
            const int b = m * 128 + r;
            if (!wait_or_abort(a_full, lt & 1, abort_flag, 0x2400)) break;
            float ss = 0.f;
            if (AMODE == A_TMA_MIX) {
#pragma unroll 1
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
            bool ok = true;
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                const int bb = c & 1;
                if (!wait_cl(&g1_full[bb], u1[bb] & 1, abort_flag, 0x2401)) { ok = false; break; }
                ++u1[bb];
                tc_fence_after();
                const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + C::G1COL + bb * 128 + half * 32;
                float gv[32], uv[32];
                tmem_ld32(ta, gv);
                tmem_ld32(ta + 64, uv);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(L(&g1_empty[bb]));
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(silu_tanh(sc * gv[2 * i]) * (sc * uv[2 * i]),
                                        silu_tanh(sc * gv[2 * i + 1]) * (sc * uv[2 * i + 1]));
                if (!wait_cl(&hid_empty[bb], (u2[bb] & 1) ^ 1, abort_flag, 0x2402)) { ok = false; break; }
                ++u2[bb];
                uint8_t* hrow = sH + bb * C::HID_BYTES + r * 128;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int chunk = half * 4 + v;
                    *reinterpret_cast<uint4*>(hrow + ((chunk ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(L(&hid_full[bb]));
            }
            if (!ok) break;
            YEpilogue<W> ye;
            ye.prefetch(p, b, g, half * (W / 2), valid);
            if (!wait_cl(y_full, lt & 1, abort_flag, 0x2403)) break;
            tc_fence_after();
            ye.store(p, tmem + (uint32_t(q * 32) << 16), b, g, half * (W / 2), valid);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(L(y_empty));
        }
    }

    // no CTA of the pair may release TMEM or exit while the other still uses its barriers/TMEM
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

}  // namespace tml
