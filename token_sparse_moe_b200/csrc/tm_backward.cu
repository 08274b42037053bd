// tm_backward.cu -- CUDA-core kernels of the dense sub-layer backward.  The seven contractions
// of the backward (the recomputed gate / up projections, the down projection's input gradient,
// the input gradient of the gate / up projections and the three weight gradients) run on the
// tensor-core grouped GEMM; these kernels do the memory-bound steps between them:
//   * the row pass: 1/rms of every input row, the normalised row xh = x / rms and the row of
//     the upstream gradient, both copied bank-major ([banks][B][W]) for the GEMMs;
//   * a tiled transpose, which turns bank-major [rows, cols] operands into the K-major
//     [cols, rows] operands of the weight-gradient GEMMs (contraction over the B samples);
//   * the SwiGLU derivative, elementwise over the hidden rows;
//   * the RMSNorm derivative (no centring), one warp per row, plus the residual addends.
// Derivatives (the dense sub-layer y = Wd (silu(Wg n) * (Wu n)), n = x / rms(x)):
//   dWd = dy^T h,  dh = dy Wd,  dg = dh u s (1 + g (1 - s)),  du = dh g s,  s = sigmoid(g),
//   dWg = dg^T n,  dWu = du^T n,  dn = dg Wg + du Wu,  dx = r (dn - xh mean(dn xh)).
// Part of the single translation unit (after tm_kernels.cu, whose vector loads and warp
// reduction it uses).

namespace tml {

// One warp per (b, bank) row, rows read through the sub-layer's row map (x and dy share it:
// a sub-layer's output rows sit where its input rows do).
__global__ void __launch_bounds__(256) bwd_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                       const __nv_bfloat16* __restrict__ dy, RowMap m, int B,
                                                       float eps, __nv_bfloat16* __restrict__ xh,
                                                       __nv_bfloat16* __restrict__ dyb, float* __restrict__ inv_rms) {
    const int lane = threadIdx.x & 31;
    const int nrows = B * m.banks;
    const int wstride = gridDim.x * (blockDim.x >> 5);
    for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < nrows; row += wstride) {
        const int b = row / m.banks, bank = row - b * m.banks;
        float ss = 0.f;
        for (int c = lane * 8; c < m.W; c += 256) {
            float v[8];
            Vec<__nv_bfloat16>::load(x + row_elem(m, b, bank, c), v);
#pragma unroll
            for (int i = 0; i < 8; ++i) ss = fmaf(v[i], v[i], ss);
        }
        ss = warp_sum(ss);
        const float r = 1.0f / sqrtf(ss / (float)m.W + eps);
        const size_t o = ((size_t)bank * B + b) * m.W;
        for (int c = lane * 8; c < m.W; c += 256) {
            const size_t e = row_elem(m, b, bank, c);
            float v[8];
            Vec<__nv_bfloat16>::load(x + e, v);
            *reinterpret_cast<uint4*>(xh + o + c) =
                make_uint4(pack_bf16x2(v[0] * r, v[1] * r), pack_bf16x2(v[2] * r, v[3] * r),
                           pack_bf16x2(v[4] * r, v[5] * r), pack_bf16x2(v[6] * r, v[7] * r));
            *reinterpret_cast<uint4*>(dyb + o + c) = __ldg(reinterpret_cast<const uint4*>(dy + e));
        }
        if (lane == 0) inv_rms[(size_t)bank * B + b] = r;
    }
}

// out[g][c][r] = in[g][r][c] for r < R and 0 for R <= r < Rp (c < C): 64 x 64 tiles staged in
// shared memory, read with 16-byte loads along c and written with 16-byte stores along r (eight
// threads cover 128 contiguous bytes on both sides).  Grid (Rp / 64, C / 64, groups), 256 threads.
// In shared memory element (r, c) of the tile sits in row r at 8-element piece (c / 8) ^ (r / 8 % 8),
// so the column reads of a warp (eight row pieces, four columns) fall in distinct banks.  C, Rp,
// the leading dimensions and group strides are multiples of 8 elements and both bases 16-byte
// aligned (checked by the launcher), so every 8-element piece is whole and aligned.
__global__ void __launch_bounds__(256) transpose_kernel(const __nv_bfloat16* __restrict__ in, size_t in_gs, int in_ld,
                                                        int R, int C, __nv_bfloat16* __restrict__ out, size_t out_gs,
                                                        int out_ld, int Rp) {
    __shared__ __align__(16) uint16_t tile[64 * 64];
    const int g = blockIdx.z;
    const int r0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
    const __nv_bfloat16* src = in + (size_t)g * in_gs;
#pragma unroll
    for (int i = threadIdx.x; i < 512; i += 256) {
        const int rr = i >> 3, q = i & 7;
        const int r = r0 + rr, c = c0 + q * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < R && c < C) v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * in_ld + c));
        *reinterpret_cast<uint4*>(&tile[rr * 64 + ((q ^ ((rr >> 3) & 7)) << 3)]) = v;
    }
    __syncthreads();
    __nv_bfloat16* dst = out + (size_t)g * out_gs;
#pragma unroll
    for (int i = threadIdx.x; i < 512; i += 256) {
        const int cc = i >> 3, q = i & 7;
        const int c = c0 + cc, r = r0 + q * 8;
        if (c >= C || r >= Rp) continue;
        const int col = (((cc >> 3) ^ q) << 3) + (cc & 7);   // rows q*8 .. q*8+7 share the piece swizzle q
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = (uint32_t)tile[(q * 8 + 2 * k) * 64 + col] | ((uint32_t)tile[(q * 8 + 2 * k + 1) * 64 + col] << 16);
        *reinterpret_cast<uint4*>(dst + (size_t)c * out_ld + r) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Per 8 elements of the hidden rows ([rows, F], rows = banks * B): g, u (the recomputed gate and
// up projections) and dh give dg, du (the two halves of a [rows, 2F] row) and h = silu(g) * u.
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const __nv_bfloat16* __restrict__ Gp,
                                                         const __nv_bfloat16* __restrict__ Up,
                                                         const __nv_bfloat16* __restrict__ dH, size_t rows, int F,
                                                         __nv_bfloat16* __restrict__ dGU, __nv_bfloat16* __restrict__ Hd) {
    const size_t n8 = rows * (size_t)F / 8;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i * 8;
        const size_t row = e / F;
        const int col = (int)(e - row * F);
        float g[8], u[8], d[8];
        Vec<__nv_bfloat16>::load(Gp + e, g);
        Vec<__nv_bfloat16>::load(Up + e, u);
        Vec<__nv_bfloat16>::load(dH + e, d);
        float dg[8], du[8], h[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float s = 1.0f / (1.0f + __expf(-g[k]));
            const float sg = g[k] * s;                       // silu(g)
            h[k] = sg * u[k];
            du[k] = d[k] * sg;
            dg[k] = d[k] * u[k] * (s + sg * (1.0f - s));     // s (1 + g (1 - s))
        }
        __nv_bfloat16* o = dGU + row * 2 * (size_t)F + col;
        *reinterpret_cast<uint4*>(o) = make_uint4(pack_bf16x2(dg[0], dg[1]), pack_bf16x2(dg[2], dg[3]),
                                                  pack_bf16x2(dg[4], dg[5]), pack_bf16x2(dg[6], dg[7]));
        *reinterpret_cast<uint4*>(o + F) = make_uint4(pack_bf16x2(du[0], du[1]), pack_bf16x2(du[2], du[3]),
                                                      pack_bf16x2(du[4], du[5]), pack_bf16x2(du[6], du[7]));
        *reinterpret_cast<uint4*>(Hd + e) = make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]),
                                                       pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
    }
}

// One warp per (b, bank) row: dx = r (dn - xh mean(dn xh)) + add0 + add1 + add2, with xh = x r (x
// re-read through the row map, r from the row pass), dn bank-major [banks][B][W]; dx and the
// optional addends go through the row map.
__global__ void __launch_bounds__(256) rms_bwd_kernel(const __nv_bfloat16* __restrict__ x,
                                                      const __nv_bfloat16* __restrict__ dN,
                                                      const float* __restrict__ inv_rms,
                                                      const __nv_bfloat16* __restrict__ add0,
                                                      const __nv_bfloat16* __restrict__ add1,
                                                      const __nv_bfloat16* __restrict__ add2, RowMap m, int B,
                                                      __nv_bfloat16* __restrict__ dx) {
    const int lane = threadIdx.x & 31;
    const int nrows = B * m.banks;
    const int wstride = gridDim.x * (blockDim.x >> 5);
    for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < nrows; row += wstride) {
        const int b = row / m.banks, bank = row - b * m.banks;
        const float r = __ldg(&inv_rms[(size_t)bank * B + b]);
        const __nv_bfloat16* dn = dN + ((size_t)bank * B + b) * m.W;
        float dot = 0.f;
        for (int c = lane * 8; c < m.W; c += 256) {
            float v[8], d[8];
            Vec<__nv_bfloat16>::load(x + row_elem(m, b, bank, c), v);
            Vec<__nv_bfloat16>::load(dn + c, d);
#pragma unroll
            for (int i = 0; i < 8; ++i) dot = fmaf(d[i], v[i] * r, dot);
        }
        const float mean = warp_sum(dot) / (float)m.W;
        for (int c = lane * 8; c < m.W; c += 256) {
            const size_t e = row_elem(m, b, bank, c);
            float v[8], d[8], a0[8], a1[8], a2[8];
            Vec<__nv_bfloat16>::load(x + e, v);
            Vec<__nv_bfloat16>::load(dn + c, d);
#pragma unroll
            for (int i = 0; i < 8; ++i) a0[i] = a1[i] = a2[i] = 0.f;
            if (add0) Vec<__nv_bfloat16>::load(add0 + e, a0);
            if (add1) Vec<__nv_bfloat16>::load(add1 + e, a1);
            if (add2) Vec<__nv_bfloat16>::load(add2 + e, a2);
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = r * (d[i] - v[i] * r * mean) + a0[i] + a1[i] + a2[i];
            *reinterpret_cast<uint4*>(dx + e) = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                                           pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
        }
    }
}

static int rows_grid(long nrows) {
    const long blocks = (nrows + 7) / 8;               // 8 warps (rows) per block
    return (int)(blocks < 148L * 16 ? blocks : 148L * 16);
}

cudaError_t launch_bwd_rows(const void* x, const void* dy, RowMap m, int B, float eps, void* xh, void* dyb,
                            float* inv_rms, cudaStream_t st) {
    ProfileScope ps_("bwd_rows", st);
    bwd_rows_kernel<<<rows_grid((long)B * m.banks), 256, 0, st>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)dy, m, B, eps, (__nv_bfloat16*)xh, (__nv_bfloat16*)dyb, inv_rms);
    return cudaGetLastError();
}

cudaError_t launch_transpose(const void* in, size_t in_gs, int in_ld, int R, int C, void* out, size_t out_gs,
                             int out_ld, int Rp, int groups, cudaStream_t st) {
    if (groups <= 0 || R <= 0 || C <= 0 || Rp < R) return cudaErrorInvalidValue;
    if ((C + 63) / 64 > 65535 || groups > 65535) return cudaErrorInvalidValue;
    if (C % 8 || Rp % 8 || in_ld % 8 || out_ld % 8 || in_gs % 8 || out_gs % 8 || in_ld < C || out_ld < Rp ||
        ((uintptr_t)in & 15) || ((uintptr_t)out & 15))
        return cudaErrorInvalidValue;
    ProfileScope ps_("transpose", st);
    dim3 grid((Rp + 63) / 64, (C + 63) / 64, groups);
    transpose_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)in, in_gs, in_ld, R, C, (__nv_bfloat16*)out, out_gs,
                                           out_ld, Rp);
    return cudaGetLastError();
}

cudaError_t launch_swiglu_bwd(const void* Gp, const void* Up, const void* dH, size_t rows, int F, void* dGU, void* Hd,
                              cudaStream_t st) {
    ProfileScope ps_("swiglu_bwd", st);
    const size_t n8 = rows * (size_t)F / 8;
    const size_t want = (n8 + 255) / 256;
    const int grid = (int)(want < 148u * 16 ? want : 148u * 16);
    swiglu_bwd_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>((const __nv_bfloat16*)Gp, (const __nv_bfloat16*)Up,
                                                          (const __nv_bfloat16*)dH, rows, F, (__nv_bfloat16*)dGU,
                                                          (__nv_bfloat16*)Hd);
    return cudaGetLastError();
}

cudaError_t launch_rms_bwd(const void* x, const void* dN, const float* inv_rms, const void* add0, const void* add1,
                           const void* add2, RowMap m, int B, void* dx, cudaStream_t st) {
    ProfileScope ps_("rms_bwd", st);
    rms_bwd_kernel<<<rows_grid((long)B * m.banks), 256, 0, st>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)dN, inv_rms, (const __nv_bfloat16*)add0,
        (const __nv_bfloat16*)add1, (const __nv_bfloat16*)add2, m, B, (__nv_bfloat16*)dx);
    return cudaGetLastError();
}

}  // namespace tml
