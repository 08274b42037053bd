// tm_kernels.cu -- CUDA-core kernels of the TokenMixer-Large forward:
//   * per-row RMSNorm statistics (1/rms) for dense sub-layers,
//   * the MoE router (fp32 logits, softmax, top-k, alpha-scaled gates) with the
//     per-chunk expert histogram, the offsets scan and the stable scatter that
//     together give the expert-first row buckets ("MoEPermute" in the
//     TokenMixer-Large digest, section 2.5.1),
//   * Mix / Revert as plain permutations (API utilities; the GEMM path never calls them),
//   * the gain fold, the tokenizer stub, and the fp32 grouped GEMM used for fp32 tensors.
#include "tm_internal.h"

namespace tml {


// ------------------------------------------------------------------ vector loads
template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ static void load(const float* p, float* o) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
    __device__ static void load_shared(const float* p, float* o) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const __nv_bfloat16* p, float* o) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) { o[2 * i] = bf16_lo(w[i]); o[2 * i + 1] = bf16_hi(w[i]); }
    }
    __device__ static void load_shared(const __nv_bfloat16* p, float* o) {
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) { o[2 * i] = bf16_lo(w[i]); o[2 * i + 1] = bf16_hi(w[i]); }
    }
};
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f(float v, float* d) { *d = v; }
__device__ __forceinline__ void from_f(float v, __nv_bfloat16* d) { *d = __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------------ RMS statistics
// inv_rms[b * banks + bank] = 1 / sqrt(mean(row^2) + eps), one warp per row.
template <typename T>
__global__ void rms_kernel(const T* __restrict__ x, RowMap m, int B, float eps, float* __restrict__ inv_rms) {
    constexpr int V = Vec<T>::N;
    const int lane = threadIdx.x & 31;
    const int nrows = B * m.banks;
    const int wstride = gridDim.x * (blockDim.x >> 5);
    for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < nrows; row += wstride) {
        const int b = row / m.banks, bank = row - b * m.banks;
        float ss = 0.f;
        for (int c = lane * V; c < m.W; c += 32 * V) {
            float v[V];
            Vec<T>::load(x + row_elem(m, b, bank, c), v);
#pragma unroll
            for (int i = 0; i < V; ++i) ss = fmaf(v[i], v[i], ss);
        }
        ss = warp_sum(ss);
        if (lane == 0) inv_rms[row] = 1.0f / sqrtf(ss / (float)m.W + eps);
    }
}

// ------------------------------------------------------------------ router
// Block (bank = blockIdx.y, chunk = blockIdx.x) routes samples [chunk*128, chunk*128 + 128) of one
// bank; warp w owns 16 of them.  Lane l works on the pair (row l / EP, expert l % EP) with EP the
// expert count rounded up to a power of two: it walks the whole row in shared memory (x reads are
// broadcasts among the row's lanes; router-weight rows are padded by 4 floats, so the float4 reads
// of the EP lanes hit distinct banks) and accumulates its logit and the row's sum of squares.
// Softmax and top-k then reduce over the EP lanes of a row only.  Each warp stages its own rows
// with cp.async, double-buffered, so no block-wide barrier is needed after the weights load.
template <typename T, int EP>
__global__ void __launch_bounds__(256) router_kernel(const T* __restrict__ x, RowMap m, int B, float eps,
                                                     const T* __restrict__ gain, const float* __restrict__ w_router,
                                                     int E, int k, float alpha, int32_t* __restrict__ idx,
                                                     float* __restrict__ gate, float* __restrict__ inv_rms,
                                                     float* __restrict__ logit_gap, int32_t* __restrict__ counts) {
    constexpr int V = Vec<T>::N;
    constexpr int ROWS = 32 / EP;                 // rows per warp pass
    constexpr int GROUP = ROWS > 4 ? ROWS : 4;    // rows per staging buffer
    constexpr int WARP_ROWS = kRouterChunk / 8;   // 16
    static_assert(WARP_ROWS % GROUP == 0, "router row groups");
    extern __shared__ __align__(16) float wr[];   // [EP][W + 4], then per warp 2 x [GROUP][W] rows
    __shared__ int cnt[32];
    const int bank = blockIdx.y, chunk = blockIdx.x, W = m.W, WP = W + 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < EP * WP; i += blockDim.x) {
        const int e = i / WP, c = i - e * WP;
        float v = 0.f;
        if (e < E && c < W) v = w_router[((size_t)bank * E + e) * W + c] * (gain ? to_f(gain[c]) : 1.0f);
        wr[i] = v;
    }
    if (threadIdx.x < 32) cnt[threadIdx.x] = 0;
    __syncthreads();

    T* xb = reinterpret_cast<T*>(wr + EP * WP) + (size_t)warp * 2 * GROUP * W;
    const size_t row_stride = m.layout == 0 ? (size_t)m.banks * W : (size_t)m.T * m.D;   // sample b -> b+1
    const int b_first = chunk * kRouterChunk + warp * WARP_ROWS;
    auto stage = [&](int grp, int buf) {
        T* dst = xb + (size_t)buf * GROUP * W;
        for (int c = lane * V; c < W; c += 32 * V) {
            const size_t base = row_elem(m, 0, bank, c);
#pragma unroll
            for (int r = 0; r < GROUP; ++r) {
                const int b = b_first + grp * GROUP + r;
                const uint32_t d = smem_u32(dst + (size_t)r * W + c);
                if (b < B) cp_async_16(d, x + base + (size_t)b * row_stride, 16u);
                else cp_async_16(d, x, 0u);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    constexpr int NG = WARP_ROWS / GROUP;
    stage(0, 0);
    const int rl = lane / EP, e = lane % EP;
#pragma unroll 1
    for (int gi = 0; gi < NG; ++gi) {
        if (gi + 1 < NG) {
            stage(gi + 1, (gi + 1) & 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();
        const T* xr0 = xb + (size_t)(gi & 1) * GROUP * W;
#pragma unroll 1
        for (int pass = 0; pass < GROUP / ROWS; ++pass) {
            const int r = pass * ROWS + rl;
            const int b = b_first + gi * GROUP + r;
            const T* xr = xr0 + (size_t)r * W;
            const float* wrow = wr + e * WP;
            float dot = 0.f, ss = 0.f;
            for (int c = 0; c < W; c += V) {
                float xv[V];
                Vec<T>::load_shared(xr + c, xv);
#pragma unroll
                for (int q = 0; q < V; q += 4) {
                    const float4 w4 = *reinterpret_cast<const float4*>(wrow + c + q);
                    dot = fmaf(w4.x, xv[q], dot);
                    dot = fmaf(w4.y, xv[q + 1], dot);
                    dot = fmaf(w4.z, xv[q + 2], dot);
                    dot = fmaf(w4.w, xv[q + 3], dot);
                }
#pragma unroll
                for (int q = 0; q < V; ++q) ss = fmaf(xv[q], xv[q], ss);
            }
            const float irs = 1.0f / sqrtf(ss / (float)W + eps);
            float z = e < E ? dot * irs : -INFINITY;
            float zmax = z;
#pragma unroll
            for (int o = 1; o < EP; o <<= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
            const float pe = e < E ? expf(z - zmax) : 0.f;
            float sum = pe;
#pragma unroll
            for (int o = 1; o < EP; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const float p = pe / sum;
            const size_t rowi = (size_t)b * m.banks + bank;
            float zc = z;                       // candidate logit; -inf once taken
            float zk = INFINITY;                // logit of the k-th choice
            for (int j = 0; j < k; ++j) {
                float bz = zc;
                int be = zc == -INFINITY ? 1 << 30 : e;   // ties and exhausted lanes: lower index wins
#pragma unroll
                for (int o = 1; o < EP; o <<= 1) {
                    const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                    if (oz > bz || (oz == bz && oe < be)) { bz = oz; be = oe; }
                }
                const float pb = __shfl_sync(0xffffffffu, p, (lane & ~(EP - 1)) + (be < EP ? be : 0));
                if (e == be) zc = -INFINITY;
                zk = bz;
                if (e == 0 && b < B && be < E) {
                    idx[rowi * k + j] = be;
                    gate[rowi * k + j] = alpha * pb;
                    atomicAdd(&cnt[be], 1);
                }
            }
            if (e == 0 && b < B && inv_rms) inv_rms[rowi] = irs;
            if (logit_gap) {
                // the best logit left after the k choices (lanes taken or past E hold -inf)
                float zn = zc;
#pragma unroll
                for (int o = 1; o < EP; o <<= 1) zn = fmaxf(zn, __shfl_xor_sync(0xffffffffu, zn, o));
                if (e == 0 && b < B) logit_gap[rowi] = zk - zn;
            }
        }
        __syncwarp();                          // buffer (gi & 1) is refilled two groups later
    }
    __syncthreads();
    if (threadIdx.x < E) counts[((size_t)bank * gridDim.x + chunk) * E + threadIdx.x] = cnt[threadIdx.x];
}

// counts [banks][nchunks][E] -> (in place) exclusive prefix over chunks, plus the group
// offsets and the 128-row tile prefix over groups g = bank*E + e, and (optional) one descriptor
// per 128-row tile {group, first row position, rows, tile within the group}.  One block.
__global__ void __launch_bounds__(1024) offsets_kernel(int32_t* counts, int banks, int nchunks, int E,
                                                       int32_t* bucket_offsets, int32_t* tile_start, int4* tile_info) {
    __shared__ int tot[4096];
    const int G = banks * E;
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int bank = g / E, e = g - bank * E;
        int run = 0;
        // sixteen chunks' counts loaded before any of them is rewritten, so the loads overlap
        for (int c0 = 0; c0 < nchunks; c0 += 16) {
            int v[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
                v[c] = c0 + c < nchunks ? counts[((size_t)bank * nchunks + c0 + c) * E + e] : 0;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                if (c0 + c < nchunks) counts[((size_t)bank * nchunks + c0 + c) * E + e] = run;
                run += v[c];
            }
        }
        tot[g] = run;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int per = (G + 31) / 32;
        const int lo = min(G, lane * per), hi = min(G, lo + per);
        int s1 = 0, s2 = 0;
        for (int g = lo; g < hi; ++g) { s1 += tot[g]; s2 += (tot[g] + 127) / 128; }
        int e1 = s1, e2 = s2;   // inclusive scan across lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, e1, o), b2 = __shfl_up_sync(0xffffffffu, e2, o);
            if (lane >= o) { e1 += a; e2 += b2; }
        }
        int r1 = e1 - s1, r2 = e2 - s2;
        for (int g = lo; g < hi; ++g) {
            bucket_offsets[g] = r1;
            tile_start[g] = r2;
            r1 += tot[g];
            r2 += (tot[g] + 127) / 128;
        }
        if (lane == 31) { bucket_offsets[G] = e1; tile_start[G] = e2; }
    }
    if (!tile_info) return;
    __syncthreads();                         // offsets and tile prefix written by warp 0
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int n = tot[g], r0 = bucket_offsets[g], t0 = tile_start[g];
        for (int m = 0; m * 128 < n; ++m) tile_info[t0 + m] = make_int4(g, r0 + m * 128, min(128, n - m * 128), m);
    }
}

// Stable scatter: position of (b, bank, j) = group offset + earlier chunks + earlier rows of
// this chunk routed to the same expert (warp ballots keep ascending b).
__global__ void __launch_bounds__(kRouterChunk) scatter_kernel(const int32_t* __restrict__ idx,
                                                               const int32_t* __restrict__ chunk_prefix,
                                                               const int32_t* __restrict__ bucket_offsets, int B,
                                                               int banks, int E, int k, int limit,
                                                               int32_t* __restrict__ bucket_rows,
                                                               int32_t* __restrict__ slot_of, int32_t* __restrict__ perm,
                                                               const float* __restrict__ inv_rms,
                                                               const float* __restrict__ gate, float* __restrict__ inv_pos,
                                                               float* __restrict__ gate_pos) {
    __shared__ int wcount[kRouterChunk / 32][64];
    __shared__ int base[64];   // per expert: the bucket's offset plus the earlier chunks' rows
    const int bank = blockIdx.y, chunk = blockIdx.x, nchunks = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = chunk * kRouterChunk + threadIdx.x;
    const bool valid = b < B;
    const size_t rowi = (size_t)b * banks + bank;
    // every global load the block needs is issued here, before any of it is used
    if (threadIdx.x < E)
        base[threadIdx.x] = bucket_offsets[bank * E + threadIdx.x] +
                            chunk_prefix[((size_t)bank * nchunks + chunk) * E + threadIdx.x];
    int my[8], rank[8];
    float gv[8];
    float irs = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) { my[j] = -1; rank[j] = 0; gv[j] = 0.f; }
    if (valid) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (j < k) {
                my[j] = idx[rowi * k + j];
                if (gate_pos) gv[j] = gate[rowi * k + j];
            }
        }
        if (inv_pos) irs = inv_rms[rowi];
    }
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int e = 0; e < E; ++e) {
        bool has = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) has |= (my[j] == e);
        const unsigned bal = __ballot_sync(0xffffffffu, has);
        if (lane == 0) wcount[warp][e] = __popc(bal);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (my[j] == e) rank[j] = __popc(bal & lt_mask);
    }
    __syncthreads();
    if (!valid) return;
    // positions must fall inside the caller's bucket_rows (limit entries): a table that does not
    // match the choices is reported, never written out of range
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (j >= k) break;
        const int e = my[j];
        if (e < 0 || e >= E) {
            record_error(ERR_BOUNDS, 0x500);
            continue;
        }
        int pos = base[e] + rank[j];
        for (int w = 0; w < warp; ++w) pos += wcount[w][e];
        if (pos < 0 || pos >= limit) {
            record_error(ERR_BOUNDS, 0x501);
            continue;
        }
        slot_of[rowi * k + j] = pos;
        bucket_rows[pos] = b;
        // (optional) the combine-order row of this choice: bank-major, (bank * k + j) * B + b, so a
        // tile of 128 samples of one bank reads each choice's expert rows as one contiguous box
        if (perm) perm[pos] = (int32_t)(((size_t)bank * k + j) * B + b);
        // (optional) the row's 1/rms and the choice's gate by bucket position, so that the routed
        // GEMMs read them as contiguous per-row values
        if (inv_pos) inv_pos[pos] = irs;
        if (gate_pos) gate_pos[pos] = gv[j];
    }
}

// ------------------------------------------------------------------ Mix / Revert utilities
template <typename T>
__global__ void permute_kernel(const T* __restrict__ src, T* __restrict__ dst, int B, int T_, int D, int H,
                               bool to_mixed) {
    const size_t total = (size_t)B * T_ * D;
    const int dh = D / H;
    for (size_t o = blockIdx.x * (size_t)blockDim.x + threadIdx.x; o < total; o += (size_t)gridDim.x * blockDim.x) {
        const size_t b = o / ((size_t)T_ * D);
        const int rem = (int)(o - b * (size_t)T_ * D);
        const int t = rem / D, d = rem - t * D;
        const int h = d / dh, j = d - h * dh;
        const size_t mo = (b * H + h) * (size_t)T_ * dh + (size_t)t * dh + j;   // Hm[b, h, t*dh + j]
        if (to_mixed) dst[mo] = src[o]; else dst[o] = src[mo];
    }
}

template <typename T>
__global__ void fold_gain_kernel(const T* __restrict__ w, const T* __restrict__ gain, T* __restrict__ out, size_t n,
                                 int width) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        from_f(to_f(w[i]) * to_f(gain[i % width]), &out[i]);
}

template <typename T>
__global__ void tokenize_kernel(const T* __restrict__ groups, const T* __restrict__ w_group,
                                const T* __restrict__ w_global, int dg, int B, int T_, int D, T* __restrict__ X) {
    const int G = T_ - 1;
    const size_t total = (size_t)B * T_ * D;
    for (size_t o = blockIdx.x * (size_t)blockDim.x + threadIdx.x; o < total; o += (size_t)gridDim.x * blockDim.x) {
        const size_t b = o / ((size_t)T_ * D);
        const int rem = (int)(o - b * (size_t)T_ * D);
        const int t = rem / D, d = rem - t * D;
        float acc = 0.f;
        const T* gb = groups + b * (size_t)G * dg;
        if (t == 0) {
            const T* wrow = w_global + (size_t)d * G * dg;
            for (int i = 0; i < G * dg; ++i) acc = fmaf(to_f(wrow[i]), to_f(gb[i]), acc);
        } else {
            const T* wrow = w_group + ((size_t)(t - 1) * D + d) * dg;
            const T* g = gb + (size_t)(t - 1) * dg;
            for (int c = 0; c < dg; ++c) acc = fmaf(to_f(wrow[c]), to_f(g[c]), acc);
        }
        from_f(acc, &X[o]);
    }
}

// ------------------------------------------------------------------ fp32 grouped GEMM (CUDA cores)
// Same tile space (128-row tiles, groups, buckets) and epilogues as the tcgen05 kernel, 32 output
// columns per block; used for fp32 tensors, where bf16 tensor cores would lose precision.
template <int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtGemmArgs a) {
    const GemmParams& p = a.p;
    const int t = blockIdx.x;
    if (t >= total_tiles(p)) return;
    const TileInfo ti = decode_tile(p, t);
    constexpr bool SW = EPI == EPI_SWIGLU;
    __shared__ float As[32][129];
    __shared__ float Bs[SW ? 2 : 1][32][33];
    __shared__ int rowb[128];
    const int tid = threadIdx.x;
    const int bank = p.sched == 0 ? ti.g : ti.g / p.E;
    if (tid < 128) {
        int b = -1;
        if (tid < ti.nrows) b = p.sched == 0 ? ti.m * 128 + tid : p.bucket_rows[ti.row0 + tid];
        if (b >= p.rows || ti.row0 + tid >= p.pos_limit) {
            if (tid < ti.nrows) record_error(ERR_BOUNDS, 0x600);
            b = -1;
        }
        rowb[tid] = b;
    }
    __syncthreads();
    const int tx = tid & 7, ty = tid >> 3;   // 4 columns x 4 rows per thread
    const int Nrows = SW ? (p.N >> 1) : p.N; // weight rows per group
    const int col0 = ti.n * 32;
    float acc0[4][4] = {}, acc1[4][4] = {};
    for (int k0 = 0; k0 < p.K; k0 += 32) {
        {
            const int kk = tid & 31;
            const int kq = k0 + kk;
            for (int i = 0; i < 16; ++i) {
                const int r = (tid >> 5) + 8 * i;
                float v = 0.f;
                const int b = rowb[r];
                if (b >= 0 && kq < p.K)
                    v = SW ? a.a[row_elem(p.amap, b, bank, kq)] : a.a[(size_t)(ti.row0 + r) * p.K + kq];
                As[kk][r] = v;
            }
            for (int i = 0; i < 4; ++i) {
                const int c = (tid >> 5) + 8 * i;
                const size_t wrow = (size_t)ti.g * Nrows + col0 + c;
                const bool ok = kq < p.K && col0 + c < Nrows;
                Bs[0][kk][c] = ok ? a.w0[wrow * p.K + kq] : 0.f;
                if (SW) Bs[SW ? 1 : 0][kk][c] = ok ? a.w1[wrow * p.K + kq] : 0.f;
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            float av[4], bv[4], uv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { av[i] = As[kk][ty * 4 + i]; bv[i] = Bs[0][kk][tx * 4 + i]; }
            if (SW) {
#pragma unroll
                for (int i = 0; i < 4; ++i) uv[i] = Bs[SW ? 1 : 0][kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc0[i][j] = fmaf(av[i], bv[j], acc0[i][j]);
                    if (SW) acc1[i][j] = fmaf(av[i], uv[j], acc1[i][j]);
                }
        }
        __syncthreads();
    }
    float* out = reinterpret_cast<float*>(p.out);
    const float* resid = reinterpret_cast<const float*>(p.resid);
    const float* extra = reinterpret_cast<const float*>(p.extra);
    const float* slots = reinterpret_cast<const float*>(p.slots);
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        const int b = rowb[r];
        if (b < 0) continue;
        const int pos = ti.row0 + r;
        for (int j = 0; j < 4; ++j) {
            const int col = col0 + tx * 4 + j;
            if (col >= Nrows) continue;
            if (SW) {
                const float s = p.inv_rms[(size_t)b * p.banks + bank];
                const float g = s * acc0[i][j], u = s * acc1[i][j];
                out[(size_t)pos * p.out_ld + col] = g / (1.0f + expf(-g)) * u;
            } else if (EPI == EPI_SLOT) {
                out[(size_t)pos * p.out_ld + col] = acc0[i][j];
            } else {
                float v = acc0[i][j];
                if (EPI == EPI_COMBINE) {
                    const size_t e0 = ((size_t)b * p.banks + bank) * p.k;
                    for (int q = 0; q < p.k; ++q) {
                        const int sp = p.slot_of[e0 + q];
                        if (sp < 0 || sp >= p.pos_limit) { record_error(ERR_BOUNDS, 0x601); continue; }
                        v += p.gate[e0 + q] * slots[(size_t)sp * p.omap.W + col];
                    }
                }
                const size_t off = row_elem(p.omap, b, bank, col);
                if (resid) v += resid[off];
                if (extra) v += extra[off];
                out[off] = v;
            }
        }
    }
}

// MoEPermute, data part: each source row (sample b, bank), read once through the row map, is
// copied to the k bucketed row positions of its choices (slot_of[(b * banks + bank) * k + j]), so
// that the routed GEMM1 reads its A operand as plain contiguous rows.  Rows are visited in sample
// order with the bank innermost: neighbouring warps read neighbouring head segments of the same
// token rows (for the mixing sub-layer, 16 columns of every token of a sample per bank), so the
// token rows' sectors are used whole.  One warp per source row; 16-byte pieces when a head
// segment holds whole pieces, element copies otherwise.
template <typename T>
__global__ void __launch_bounds__(256) scatter_rows_kernel(const T* __restrict__ x, RowMap m, int B, int k,
                                                           const int32_t* __restrict__ slot_of, int routed,
                                                           T* __restrict__ out) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int W = m.W, banks = m.banks;
    constexpr int V = 16 / sizeof(T);
    const bool vec = (m.layout == 0 || m.dh % V == 0) && W % V == 0;
    const int rows = B * banks;
    for (int row = warp; row < rows; row += nwarps) {
        const int b = row / banks, bank = row - b * banks;
        int pos[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            pos[j] = j < k ? __ldg(&slot_of[(size_t)row * k + j]) : -1;
            if (j < k && (pos[j] < 0 || pos[j] >= routed)) {
                if (lane == 0) record_error(ERR_BOUNDS, 0x520);
                pos[j] = -1;
            }
        }
        if (vec) {
            // up to four 16-byte pieces per lane loaded before any store, so a row's reads are all
            // in flight together
            for (int c0 = lane * V; c0 < W; c0 += 4 * 32 * V) {
                uint4 v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = c0 + i * 32 * V;
                    if (c < W) v[i] = __ldg(reinterpret_cast<const uint4*>(x + row_elem(m, b, bank, c)));
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (pos[j] < 0) continue;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = c0 + i * 32 * V;
                        if (c < W) *reinterpret_cast<uint4*>(out + (size_t)pos[j] * W + c) = v[i];
                    }
                }
            }
        } else {
            for (int c = lane; c < W; c += 32) {
                const T v = x[row_elem(m, b, bank, c)];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (pos[j] >= 0) out[(size_t)pos[j] * W + c] = v;
            }
        }
    }
}

// The same copy for bf16 rows of width <= 256 * NP whose head segments hold whole 16-byte pieces:
// each warp takes two source rows at a time and issues all their loads (bucket positions, row
// pieces) before any store, with NP and the bucket positions held (KMAX >= k) as template
// constants so that the registers hold only what the rows need.
template <int NP, int KMAX>
__global__ void __launch_bounds__(256) scatter_rows_vec_kernel(const __nv_bfloat16* __restrict__ x, RowMap m, int B,
                                                               int k, const int32_t* __restrict__ slot_of, int routed,
                                                               __nv_bfloat16* __restrict__ out) {
    constexpr int R = 2;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int W = m.W, banks = m.banks, rows = B * banks;
    for (int row0 = warp * R; row0 < rows; row0 += nwarps * R) {
        int pos[R][KMAX];
        uint4 v[R][NP];
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
            const int row = row0 + rr;
            const bool ok = row < rows;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) pos[rr][j] = (ok && j < k) ? __ldg(&slot_of[(size_t)row * k + j]) : -1;
            const int b = ok ? row / banks : 0, bank = ok ? row - b * banks : 0;
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                const int c = lane * 8 + 256 * i;
                if (ok && c < W) v[rr][i] = __ldg(reinterpret_cast<const uint4*>(x + row_elem(m, b, bank, c)));
            }
        }
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < k && row0 + rr < rows && (pos[rr][j] < 0 || pos[rr][j] >= routed)) {
                    if (lane == 0) record_error(ERR_BOUNDS, 0x521);
                    pos[rr][j] = -1;
                }
                if (pos[rr][j] < 0) continue;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const int c = lane * 8 + 256 * i;
                    if (c < W) *reinterpret_cast<uint4*>(out + (size_t)pos[rr][j] * W + c) = v[rr][i];
                }
            }
        }
    }
}

// Router weights for the tensor-core router: each fp32 weight (times the RMSNorm gain) split
// exactly into three bf16 parts, hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi - mid) (each
// difference is exact in fp32; hi + mid + lo matches v to about 2^-24 relative), stored as rows
// e, E + e, 2E + e of a [banks][64][W] bf16 matrix (rows 3E .. 63 zero).
template <typename T>
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ w, const T* __restrict__ gain,
                                                           int banks, int E, int W, __nv_bfloat16* __restrict__ out) {
    const size_t n = (size_t)banks * 64 * W;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % W);
        const int row = (int)((i / W) % 64);
        const int bank = (int)(i / ((size_t)64 * W));
        __nv_bfloat16 o = __float2bfloat16_rn(0.f);
        if (row < 3 * E) {
            const int part = row / E, e = row - part * E;
            const float v = w[((size_t)bank * E + e) * W + c] * (gain ? to_f(gain[c]) : 1.0f);
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const float r1 = v - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(mid);
            o = part == 0 ? hi : (part == 1 ? mid : __float2bfloat16_rn(r2));
        }
        out[i] = o;
    }
}

// ------------------------------------------------------------------ launchers
static int grid_for(size_t n, int threads) {
    size_t g = (n + threads - 1) / threads;
    return (int)(g > 65535 * 8 ? 65535 * 8 : (g < 1 ? 1 : g));
}

cudaError_t launch_rms(int dtype, const void* x, RowMap m, int B, float eps, float* inv_rms, cudaStream_t st) {
    ProfileScope ps_("rms", st);
    const size_t rows = (size_t)B * m.banks;
    const int grid = grid_for(rows * 32, 256);
    if (dtype == 1)
        rms_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, m, B, eps, inv_rms);
    else
        rms_kernel<float><<<grid, 256, 0, st>>>((const float*)x, m, B, eps, inv_rms);
    return cudaGetLastError();
}

template <typename T, int EP>
static cudaError_t router_launch(const void* x, RowMap m, int B, float eps, const void* gain, const float* w_router,
                                 int E, int k, float alpha, int32_t* idx, float* gate, float* inv_rms,
                                 float* logit_gap, int32_t* counts, cudaStream_t st) {
    constexpr int GROUP = 32 / EP > 4 ? 32 / EP : 4;
    const size_t smem = (size_t)EP * (m.W + 4) * sizeof(float) + (size_t)8 * 2 * GROUP * m.W * sizeof(T);
    auto kern = router_kernel<T, EP>;
    static size_t configured = 0;   // largest dynamic size enabled so far for this instantiation
    if (smem > configured) {
        // dynamic + static shared memory may exceed the 48 KB default: always raise the limit
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = smem;
    }
    dim3 grid((B + kRouterChunk - 1) / kRouterChunk, m.banks);
    kern<<<grid, 256, smem, st>>>((const T*)x, m, B, eps, (const T*)gain, w_router, E, k, alpha, idx, gate, inv_rms,
                                  logit_gap, counts);
    return cudaGetLastError();
}

cudaError_t launch_router(int dtype, const void* x, RowMap m, int B, float eps, const void* gain,
                          const float* w_router, int E, int k, float alpha, int32_t* idx, float* gate, float* inv_rms,
                          float* logit_gap, int32_t* counts, cudaStream_t st) {
    ProfileScope ps_("router", st);
#define TM_ROUTER(T)                                                                                                  \
    if (E <= 4) return router_launch<T, 4>(x, m, B, eps, gain, w_router, E, k, alpha, idx, gate, inv_rms, logit_gap, counts, st);  \
    if (E <= 8) return router_launch<T, 8>(x, m, B, eps, gain, w_router, E, k, alpha, idx, gate, inv_rms, logit_gap, counts, st);  \
    if (E <= 16) return router_launch<T, 16>(x, m, B, eps, gain, w_router, E, k, alpha, idx, gate, inv_rms, logit_gap, counts, st); \
    return router_launch<T, 32>(x, m, B, eps, gain, w_router, E, k, alpha, idx, gate, inv_rms, logit_gap, counts, st);
    if (dtype == 1) { TM_ROUTER(__nv_bfloat16) }
    TM_ROUTER(float)
#undef TM_ROUTER
}

cudaError_t launch_offsets(const int32_t* counts_in, int32_t* chunk_prefix, int banks, int nchunks, int E,
                           int32_t* bucket_offsets, int32_t* tile_start, cudaStream_t st, int4* tile_info) {
    ProfileScope ps_("route_offsets", st);
    if (counts_in != chunk_prefix) return cudaErrorInvalidValue;   // the scan runs in place
    offsets_kernel<<<1, 1024, 0, st>>>(chunk_prefix, banks, nchunks, E, bucket_offsets, tile_start, tile_info);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const int32_t* idx, const int32_t* chunk_prefix, const int32_t* bucket_offsets, int B,
                           int banks, int E, int k, int32_t* bucket_rows, int32_t* slot_of, cudaStream_t st, int32_t* perm,
                           const float* inv_rms, const float* gate, float* inv_pos, float* gate_pos, int limit) {
    if ((inv_pos && !inv_rms) || (gate_pos && !gate)) return cudaErrorInvalidValue;
    if (E > 64 || k > 8) return cudaErrorInvalidValue;
    ProfileScope ps_("route_scatter", st);
    dim3 grid((B + kRouterChunk - 1) / kRouterChunk, banks);
    scatter_kernel<<<grid, kRouterChunk, 0, st>>>(idx, chunk_prefix, bucket_offsets, B, banks, E, k,
                                                  limit < 0 ? B * banks * k : limit, bucket_rows, slot_of, perm,
                                                  inv_rms, gate, inv_pos, gate_pos);
    return cudaGetLastError();
}

// Self-test of the bounded waits: no arrival ever comes, so each wait must give up, record where
// and return (it never traps and never spins on).  Thread 0: first a plain bounded wait on barrier
// 0 (site 0x7001), which runs out after the configured limit; then, with the CTA's abort flag set,
// the role wait of the grouped GEMM on barrier 1, which must return at once without a record of its
// own.  res[0], res[2]: nanoseconds each wait took; res[1], res[3]: 1 where the wait reported failure.
__global__ void wait_selftest_kernel(unsigned long long* res) {
    __shared__ uint64_t bars[2];
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_barrier_init();
    uint64_t t0 = globaltimer_ns();
    const bool ok0 = mbar_wait(&bars[0], 0, 0x7001);
    uint64_t t1 = globaltimer_ns();
    if (!ok0) abort_flag = 1;
    const bool ok1 = wait_or_abort(&bars[1], 0, reinterpret_cast<volatile int*>(&abort_flag), 0x7002);
    uint64_t t2 = globaltimer_ns();
    if (res) {
        res[0] = t1 - t0;
        res[1] = ok0 ? 0ull : 1ull;
        res[2] = t2 - t1;
        res[3] = ok1 ? 0ull : 1ull;
    }
}

cudaError_t launch_wait_selftest(unsigned long long* res, cudaStream_t st) {
    ProfileScope ps_("wait_selftest", st);
    wait_selftest_kernel<<<1, 32, 0, st>>>(res);
    return cudaGetLastError();
}

cudaError_t launch_router_split(int dtype, const float* w_router, const void* gain, int banks, int E, int W,
                                void* out, cudaStream_t st) {
    ProfileScope ps_("router_split", st);
    const int grid = grid_for((size_t)banks * 64 * W, 256);
    if (dtype == 1)
        router_split_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(w_router, (const __nv_bfloat16*)gain, banks, E, W,
                                                                 (__nv_bfloat16*)out);
    else
        router_split_kernel<float><<<grid, 256, 0, st>>>(w_router, (const float*)gain, banks, E, W, (__nv_bfloat16*)out);
    return cudaGetLastError();
}

cudaError_t launch_scatter_rows(int dtype, const void* x, RowMap m, int B, int k, const int32_t* slot_of, size_t routed,
                                void* out, cudaStream_t st) {
    ProfileScope ps_("moe_permute", st);
    const int np = (m.W + 255) / 256, kmax = k <= 2 ? 2 : k <= 4 ? 4 : 8;
    if (dtype == 1 && (m.layout == 0 || m.dh % 8 == 0) && m.W % 8 == 0 && np <= 4 && k >= 1 && k <= 8) {
        const int gv = grid_for(((size_t)B * m.banks + 1) / 2 * 32, 256);
#define SLAUNCH(NP, KM)                                                                                               \
        if (np == NP && kmax == KM) {                                                                                 \
            scatter_rows_vec_kernel<NP, KM><<<gv, 256, 0, st>>>((const __nv_bfloat16*)x, m, B, k, slot_of, (int)routed, \
                                                               (__nv_bfloat16*)out);                                  \
            return cudaGetLastError();                                                                                \
        }
#define SLAUNCH_NP(NP) SLAUNCH(NP, 2) SLAUNCH(NP, 4) SLAUNCH(NP, 8)
        SLAUNCH_NP(1) SLAUNCH_NP(2) SLAUNCH_NP(3) SLAUNCH_NP(4)
#undef SLAUNCH_NP
#undef SLAUNCH
    }
    const int grid = grid_for((size_t)B * m.banks * 32, 256);
    if (dtype == 1)
        scatter_rows_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, m, B, k, slot_of, (int)routed,
                                                                 (__nv_bfloat16*)out);
    else
        scatter_rows_kernel<float><<<grid, 256, 0, st>>>((const float*)x, m, B, k, slot_of, (int)routed, (float*)out);
    return cudaGetLastError();
}

// Token Parallel exchange layouts: the all-to-all buffer E [P][B][Tp][Dp] (chunk q for / from rank
// q) against a rank's local tensor, either its token shard of the full width, L [B][Tp][P][Dp]
// (columns q * Dp .. of token t), or its head-column shard of every token, L [B][P][Tp][Dp] (token
// q * Tp + t).  One 16-byte piece per thread when Dp * esz is a multiple of 16, else one element.
template <typename V>
__global__ void tp_layout_kernel(const V* __restrict__ src, V* __restrict__ dst, int P, int B, int Tp, int dv,
                                 int cols_shard, int to_exchange) {
    const size_t n = (size_t)P * B * Tp * dv;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        // i indexes the exchange layout: (q, b, t, j)
        const int j = (int)(i % dv);
        size_t r = i / dv;
        const int t = (int)(r % Tp);
        r /= Tp;
        const int b = (int)(r % B);
        const int q = (int)(r / B);
        const size_t l = cols_shard ? (((size_t)b * Tp + t) * P + q) * dv + j : (((size_t)b * P + q) * Tp + t) * dv + j;
        if (to_exchange) dst[i] = src[l];
        else dst[l] = src[i];
    }
}

cudaError_t launch_tp_layout(const void* src, void* dst, int P, int B, int Tp, int Dp, int esz, bool cols_shard,
                             bool to_exchange, cudaStream_t st) {
    ProfileScope ps_("tp_layout", st);
    const size_t row = (size_t)Dp * esz;
    if (row % 16 == 0) {
        const int dv = (int)(row / 16);
        tp_layout_kernel<uint4><<<grid_for((size_t)P * B * Tp * dv, 256), 256, 0, st>>>(
            (const uint4*)src, (uint4*)dst, P, B, Tp, dv, cols_shard, to_exchange);
    } else if (esz == 2) {
        tp_layout_kernel<uint16_t><<<grid_for((size_t)P * B * Tp * Dp, 256), 256, 0, st>>>(
            (const uint16_t*)src, (uint16_t*)dst, P, B, Tp, Dp, cols_shard, to_exchange);
    } else if (esz == 4) {
        tp_layout_kernel<uint32_t><<<grid_for((size_t)P * B * Tp * Dp, 256), 256, 0, st>>>(
            (const uint32_t*)src, (uint32_t*)dst, P, B, Tp, Dp, cols_shard, to_exchange);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_permute(int dtype, const void* src, void* dst, int B, int T, int D, int H, bool to_mixed,
                           cudaStream_t st) {
    ProfileScope ps_(to_mixed ? "mix" : "revert", st);
    const size_t n = (size_t)B * T * D;
    const int grid = grid_for(n, 256);
    if (dtype == 1)
        permute_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)src, (__nv_bfloat16*)dst, B, T, D, H,
                                                            to_mixed);
    else
        permute_kernel<float><<<grid, 256, 0, st>>>((const float*)src, (float*)dst, B, T, D, H, to_mixed);
    return cudaGetLastError();
}

cudaError_t launch_fold_gain(int dtype, const void* w, const void* gain, void* out, size_t rows, int width,
                             cudaStream_t st) {
    ProfileScope ps_("fold_gain", st);
    const size_t n = rows * width;
    const int grid = grid_for(n, 256);
    if (dtype == 1)
        fold_gain_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)w, (const __nv_bfloat16*)gain,
                                                              (__nv_bfloat16*)out, n, width);
    else
        fold_gain_kernel<float><<<grid, 256, 0, st>>>((const float*)w, (const float*)gain, (float*)out, n, width);
    return cudaGetLastError();
}

// Scoring head ([readme] block diagram: mean-pool over tokens, projection head to one logit, no
// bias): logit[b] = (1/T) sum_t sum_d X[b,t,d] w[d], fp32 accumulation.  One warp per sample,
// each lane a strided slice of the sample's T*D elements, then a shuffle sum.
template <typename T>
__global__ void __launch_bounds__(256) head_kernel(const T* __restrict__ X, const T* __restrict__ w, int B, int T_,
                                                   int D, float* __restrict__ logits) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const size_t n = (size_t)T_ * D;
    for (int b = warp; b < B; b += nwarps) {
        const T* xb = X + (size_t)b * n;
        float acc = 0.f;
        for (size_t i = lane; i < n; i += 32) acc = fmaf(to_f(xb[i]), to_f(w[i % D]), acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) logits[b] = acc / (float)T_;
    }
}

cudaError_t launch_head(int dtype, const void* X, const void* w, int B, int T, int D, float* logits, cudaStream_t st) {
    ProfileScope ps_("head", st);
    const int grid = grid_for((size_t)B * 32, 256);
    if (dtype == 1)
        head_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)X, (const __nv_bfloat16*)w, B, T, D, logits);
    else
        head_kernel<float><<<grid, 256, 0, st>>>((const float*)X, (const float*)w, B, T, D, logits);
    return cudaGetLastError();
}

cudaError_t launch_tokenize(int dtype, const void* groups, const void* w_group, const void* w_global, int dg, int B,
                            int T, int D, void* X, cudaStream_t st) {
    ProfileScope ps_("tokenize", st);
    const size_t n = (size_t)B * T * D;
    const int grid = grid_for(n, 256);
    if (dtype == 1)
        tokenize_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)groups, (const __nv_bfloat16*)w_group,
                                                             (const __nv_bfloat16*)w_global, dg, B, T, D,
                                                             (__nv_bfloat16*)X);
    else
        tokenize_kernel<float><<<grid, 256, 0, st>>>((const float*)groups, (const float*)w_group,
                                                     (const float*)w_global, dg, B, T, D, (float*)X);
    return cudaGetLastError();
}

cudaError_t launch_simt_gemm(int epi, const SimtGemmArgs& a, int max_tiles, cudaStream_t st) {
    if (max_tiles <= 0) return cudaSuccess;
    ProfileScope ps_(epi == EPI_SWIGLU ? "simt_swiglu" : epi == EPI_RESID ? "simt_resid" : epi == EPI_SLOT ? "simt_slot" : "simt_combine", st);
    switch (epi) {
        case EPI_SWIGLU: simt_gemm_kernel<EPI_SWIGLU><<<max_tiles, 256, 0, st>>>(a); break;
        case EPI_RESID: simt_gemm_kernel<EPI_RESID><<<max_tiles, 256, 0, st>>>(a); break;
        case EPI_SLOT: simt_gemm_kernel<EPI_SLOT><<<max_tiles, 256, 0, st>>>(a); break;
        default: simt_gemm_kernel<EPI_COMBINE><<<max_tiles, 256, 0, st>>>(a); break;
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------ FP8 E4M3 serving path


// E4M3 quantization of bf16 weight matrices, one scale per matrix ([digest] 2.5.2 FP8
// quantization; the gate / up projections of each bank): `groups` matrices of n elements each,
// the norm gain (optional, one per column of `cols`) multiplied in and rounded to bf16 first, as
// the bf16 path folds it.  scale = 2^e (above), code = E4M3(w * 2^-e).  Three passes: the matrix
// maxima (float bit patterns of non-negative values order like the values, so an integer atomic
// max is exact), the codes, and the scales written over the maxima.
__device__ __forceinline__ float folded_weight(const __nv_bfloat16* w, const __nv_bfloat16* gain, size_t i, int cols) {
    float v = __bfloat162float(w[i]);
    if (gain) v = __bfloat162float(__float2bfloat16_rn(v * __bfloat162float(gain[i % cols])));
    return v;
}

__global__ void __launch_bounds__(256) quant_matrix_amax_kernel(const __nv_bfloat16* __restrict__ w,
                                                                const __nv_bfloat16* __restrict__ gain, size_t n,
                                                                int cols, unsigned* __restrict__ amax_bits) {
    const int g = blockIdx.y;
    const __nv_bfloat16* wg = w + (size_t)g * n;
    float m = 0.f;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(folded_weight(wg, gain, i, cols)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(&amax_bits[g], __float_as_uint(m));
}
__global__ void __launch_bounds__(256) quant_matrix_codes_kernel(const __nv_bfloat16* __restrict__ w,
                                                                 const __nv_bfloat16* __restrict__ gain, size_t n,
                                                                 int cols, const unsigned* __restrict__ amax_bits,
                                                                 uint8_t* __restrict__ q) {
    const int g = blockIdx.y;
    const float inv = pow2f(-pow2_exponent(__uint_as_float(amax_bits[g])));
    const __nv_bfloat16* wg = w + (size_t)g * n;
    uint8_t* qg = q + (size_t)g * n;
    for (size_t i = 2 * (blockIdx.x * (size_t)blockDim.x + threadIdx.x); i < n; i += 2 * (size_t)gridDim.x * blockDim.x)
        *reinterpret_cast<uint16_t*>(qg + i) =
            e4m3x2(folded_weight(wg, gain, i, cols) * inv, folded_weight(wg, gain, i + 1, cols) * inv);
}
__global__ void quant_matrix_scales_kernel(unsigned* __restrict__ scale_bits, int groups) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g < groups) scale_bits[g] = __float_as_uint(pow2f(pow2_exponent(__uint_as_float(scale_bits[g]))));
}

// Per-row E4M3 quantization of the activation rows of a sub-layer, read through the row map
// (the Mix permutation for the mixing sub-layer), written as plain rows [B * banks, W] (row
// b * banks + bank).  One warp per row: sum of squares and max|x| by shuffles; codes =
// E4M3(x * 2^-e) with the row's power-of-two scale 2^e; rowscale = 2^e / rms(x), the factor the
// FP8 GEMM1 output takes back per row.
// With slot_of (the bucketing of tm_route_topk, [B * banks, k]) the row's codes and row factor also
// go to its k bucket positions (qpos [routed, W], scale_pos [routed]): the MoEPermute copy of the
// FP8 path, one byte per element.
// Each warp takes QROWS rows at a time and issues all their loads (bucket positions and row pieces)
// before any reduction or store, so that a warp keeps QROWS rows of reads in flight.  NP: 8-element
// pieces per lane (W <= 256 * NP); KMAX: bucket positions per row held (k <= KMAX; 0: no scatter),
// both compile-time so that the registers hold only what the row needs.
constexpr int QROWS = 2;
template <int NP, int KMAX>
__global__ void __launch_bounds__(256) quant_act_rows_kernel(const __nv_bfloat16* __restrict__ x, RowMap m, int B,
                                                             float eps, uint8_t* __restrict__ q,
                                                             float* __restrict__ rowscale,
                                                             const int32_t* __restrict__ slot_of, int k, int routed,
                                                             uint8_t* __restrict__ qpos, float* __restrict__ scale_pos) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int W = m.W, banks = m.banks, nrows = B * banks;
    for (int row0 = warp * QROWS; row0 < nrows; row0 += nwarps * QROWS) {
        // the rows' bucket positions (FP8 MoE path) and the rows themselves, all loads issued before
        // they are used
        int pos[QROWS][KMAX > 0 ? KMAX : 1];
        uint4 v[QROWS][NP];
#pragma unroll
        for (int rr = 0; rr < QROWS; ++rr) {
            const int row = row0 + rr;
            const bool ok = row < nrows;
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                pos[rr][j] = (ok && j < k) ? __ldg(&slot_of[(size_t)row * k + j]) : -1;
            const int b = ok ? row / banks : 0, bank = ok ? row - b * banks : 0;
#pragma unroll
            for (int kk = 0; kk < NP; ++kk) {
                const int c = lane * 8 + 256 * kk;
                v[rr][kk] = (ok && c < W) ? __ldg(reinterpret_cast<const uint4*>(x + row_elem(m, b, bank, c)))
                                          : make_uint4(0, 0, 0, 0);
            }
        }
        // sum of squares in fp32 on element pairs (paired FMA: the even and odd elements accumulate
        // apart and are added at the end); max|x| on the packed bf16 magnitudes as 16-bit integers
        // (non-negative floats order as their bit patterns), widened once per row
        float ss[QROWS], amax[QROWS];
#pragma unroll
        for (int rr = 0; rr < QROWS; ++rr) {
            float2 s2 = make_float2(0.f, 0.f);
            uint32_t m2 = 0;
#pragma unroll
            for (int kk = 0; kk < NP; ++kk) {
                const uint32_t wv[4] = {v[rr][kk].x, v[rr][kk].y, v[rr][kk].z, v[rr][kk].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 p2 = make_float2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
                    s2 = __ffma2_rn(p2, p2, s2);
                    m2 = __vmaxu2(m2, wv[e] & 0x7FFF7FFFu);
                }
            }
            ss[rr] = s2.x + s2.y;
            amax[rr] = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int rr = 0; rr < QROWS; ++rr) {
                ss[rr] += __shfl_xor_sync(0xffffffffu, ss[rr], o);
                amax[rr] = fmaxf(amax[rr], __shfl_xor_sync(0xffffffffu, amax[rr], o));
            }
        }
#pragma unroll
        for (int rr = 0; rr < QROWS; ++rr) {
            const int row = row0 + rr;
            if (row >= nrows) break;
            const int ex = pow2_exponent(amax[rr]);
            const float s = pow2f(ex), inv = pow2f(-ex);
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < k && (pos[rr][j] < 0 || pos[rr][j] >= routed)) {
                    if (lane == 0) record_error(ERR_BOUNDS, 0x530);
                    pos[rr][j] = -1;
                }
            }
#pragma unroll
            for (int kk = 0; kk < NP; ++kk) {
                const int c = lane * 8 + 256 * kk;
                if (c >= W) break;
                const uint32_t wv[4] = {v[rr][kk].x, v[rr][kk].y, v[rr][kk].z, v[rr][kk].w};
                uint16_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 t = __fmul2_rn(make_float2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u)),
                                                make_float2(inv, inv));
                    o4[e] = e4m3x2(t.x, t.y);
                }
                const uint2 w2 = make_uint2(o4[0] | (uint32_t(o4[1]) << 16), o4[2] | (uint32_t(o4[3]) << 16));
                if (q) *reinterpret_cast<uint2*>(q + (size_t)row * W + c) = w2;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (pos[rr][j] >= 0) *reinterpret_cast<uint2*>(qpos + (size_t)pos[rr][j] * W + c) = w2;
            }
            const float rs = s * (1.0f / sqrtf(ss[rr] / (float)W + eps));
            if (lane == 0) {
                if (rowscale) rowscale[row] = rs;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (pos[rr][j] >= 0 && scale_pos) scale_pos[pos[rr][j]] = rs;
            }
        }
    }
}

cudaError_t launch_quant_matrices(const void* w, const void* gain, int groups, size_t n, int cols, uint8_t* q,
                                  float* scale, cudaStream_t st) {
    ProfileScope ps_("fp8_quant_weights", st);
    if (n % 2 || n % cols) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(scale, 0, (size_t)groups * sizeof(float), st);
    if (e != cudaSuccess) return e;
    size_t bx = (n + 2047) / 2048;
    dim3 grid((unsigned)(bx < 1024 ? bx : 1024), groups);
    quant_matrix_amax_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)w, (const __nv_bfloat16*)gain, n, cols,
                                                   (unsigned*)scale);
    quant_matrix_codes_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)w, (const __nv_bfloat16*)gain, n, cols,
                                                    (const unsigned*)scale, q);
    quant_matrix_scales_kernel<<<(groups + 255) / 256, 256, 0, st>>>((unsigned*)scale, groups);
    return cudaGetLastError();
}

cudaError_t launch_quant_act_rows(const void* x, RowMap m, int B, float eps, uint8_t* q, float* rowscale,
                                  cudaStream_t st, const int32_t* slot_of, int k, size_t routed, uint8_t* qpos,
                                  float* scale_pos) {
    ProfileScope ps_(slot_of ? "fp8_quant_permute" : "fp8_quant_rows", st);
    if (m.W % 8 || m.W > 1024 || (m.layout == 1 && m.dh % 8)) return cudaErrorInvalidValue;
    if (slot_of && (k < 1 || k > 8 || !qpos)) return cudaErrorInvalidValue;
    const int grid = grid_for(((size_t)B * m.banks + QROWS - 1) / QROWS * 32, 256);
    const int np = (m.W + 255) / 256, kmax = !slot_of ? 0 : k <= 2 ? 2 : k <= 4 ? 4 : 8;
#define QLAUNCH(NP, KM)                                                                                              \
    if (np == NP && kmax == KM) {                                                                                    \
        quant_act_rows_kernel<NP, KM><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, m, B, eps, q, rowscale, slot_of, \
                                                            k, (int)routed, qpos, scale_pos);                         \
        return cudaGetLastError();                                                                                   \
    }
#define QLAUNCH_NP(NP) QLAUNCH(NP, 0) QLAUNCH(NP, 2) QLAUNCH(NP, 4) QLAUNCH(NP, 8)
    QLAUNCH_NP(1) QLAUNCH_NP(2) QLAUNCH_NP(3) QLAUNCH_NP(4)
#undef QLAUNCH_NP
#undef QLAUNCH
    return cudaErrorInvalidValue;
}

}  // namespace tml
