// incoherence.cuh -- incoherence processing of Q and K before NVFP4.
//
// "Search Your Block Floating Point Scales!" (gist.science summary),
// "ScaleSearchAttention", 비일관성 처리 (IP) 및 크기 감소: Q and K are rotated by
// a Hadamard transform with random signs (as in QuIP#) and balanced by a
// linear pair Q' = Q~ R^-T, K' = K~ R, which keeps every score
// Q' K'^T = Q~ K~^T and shrinks the outliers the block scales must cover.
//
// Reading (the pages give the transform only in prose): H is the orthonormal
// Sylvester matrix, S a diagonal of signs (an input), Q~ = Q H S,
// K~ = (K - mu) H S with mu the smoothing mean of K, and R the diagonal that
// minimises |Q~ R^-1|^2 + |K~ R|^2: r_c = (sum_t q~_tc^2 / sum_t k~_tc^2)^(1/4)
// (1 when either sum is 0).  Arithmetic: the rotation in FP32 as the fast
// Walsh-Hadamard butterfly (stages of span 1, 2, ..., D/2, (a, b) ->
// (a + b, a - b)), then y_j = fl(t_j hn) s_j with hn = fl32(1/sqrt(D)); the
// sums of squares in FP64, rows ascending inside each 128-row tile, then the
// tiles ascending; r and the reciprocal 1/r in FP64 (the pair is Q~ R^-1,
// K~ R); Q' = fl32(y (1/r)), K' = fl32(y r).  Q' and K'
// are then quantised like Q rows (own tensor scale, 16-channel blocks, no
// further smoothing).
//
// One CTA of 128 threads per (128-row tile, b*h, tensor): thread t owns row t
// of the tile and rotates it in registers (no shared-memory transpose); each
// pass re-reads the bf16 rows instead of keeping FP32 copies in HBM:
//   ip_sums_kernel   per channel, the tile's FP64 sum of squares (the rows go
//                    through shared memory so that a thread per channel adds
//                    them in row order);
//   ip_r_kernel      per (b*h, channel): tile partials ascending -> r;
//   ip_amax_kernel   tensor amax of Q' and of K';
//   ip_quant_kernel  Q' and K' encoded into the Q/K code and scale layouts.
#pragma once

#include "quant.cuh"

namespace sa {

struct IpParams {
    const uint16_t* x[2];  // bf16 [B*H, N, D]: Q, K
    const float* k_mean;   // [B*H, D] or nullptr (K not smoothed)
    const int8_t* signs;   // [D], +-1
    float hn;              // fl32(1 / sqrt(D))
    int N, T;
    double* part[2];       // [B*H, T, D] per-tile sums of squares
    double* r;             // [B*H, 2, D]: r, then 1/r
    float* r_out;          // [B*H, D] or nullptr
    unsigned* amax;        // [2] FP32 bit patterns of amax(Q'), amax(K')
};

// Row `row` of tensor `which` (0: Q, 1: K minus its mean) rotated: y = FWHT(x)
// * hn * s, FP32, into registers.
template <int D>
SA_DEV void ip_rotate_row(const IpParams& p, int which, size_t bh, int row, const float* sgn, float (&y)[D])
{
    const uint4* src = reinterpret_cast<const uint4*>(p.x[which] + (bh * p.N + row) * D);
    const float* mu = (which == 1 && p.k_mean) ? p.k_mean + bh * D : nullptr;
#pragma unroll
    for (int c = 0; c < D / 8; c++) {
        const uint4 w = __ldg(src + c);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            y[8 * c + 2 * i] = __uint_as_float(ww[i] << 16);
            y[8 * c + 2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
        }
    }
    if (mu) {
#pragma unroll
        for (int j = 0; j < D; j++) y[j] = __fsub_rn(y[j], __ldg(mu + j));
    }
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
#pragma unroll
        for (int j = 0; j < D; j++) {
            if (j & h) continue;  // j is the lower index of the pair (j, j + h)
            const float a = y[j], b = y[j + h];
            y[j] = __fadd_rn(a, b);
            y[j + h] = __fsub_rn(a, b);
        }
    }
#pragma unroll
    for (int j = 0; j < D; j++) y[j] = __fmul_rn(__fmul_rn(y[j], p.hn), sgn[j]);
}

template <int D>
SA_DEV void ip_load_signs(const IpParams& p, float* sgn)
{
    for (int j = threadIdx.x; j < D; j += blockDim.x) sgn[j] = p.signs[j] < 0 ? -1.0f : 1.0f;
}

// grid (T, B*H, 2), 128 threads, dynamic shared memory 128 (D + 1) floats.
template <int D>
__global__ void __launch_bounds__(128) ip_sums_kernel(const IpParams p)
{
    extern __shared__ float ys[];  // [128][D + 1]
    __shared__ float sgn[D];
    const int tile = blockIdx.x, which = blockIdx.z, t = threadIdx.x;
    const size_t bh = blockIdx.y;
    const int rows = min(128, p.N - tile * 128);
    ip_load_signs<D>(p, sgn);
    __syncthreads();
    if (t < rows) {
        float y[D];
        ip_rotate_row<D>(p, which, bh, tile * 128 + t, sgn, y);
#pragma unroll
        for (int j = 0; j < D; j++) ys[t * (D + 1) + j] = y[j];
    }
    __syncthreads();
    if (t < D) {
        double a = 0.0;
        for (int r = 0; r < rows; r++) {
            const double v = ys[r * (D + 1) + t];
            a = __dadd_rn(a, __dmul_rn(v, v));
        }
        p.part[which][(bh * p.T + tile) * D + t] = a;
    }
}

// grid B*H, D threads.
__global__ void ip_r_kernel(const IpParams p, int D)
{
    const size_t bh = blockIdx.x;
    const int c = threadIdx.x;
    double a = 0.0, b = 0.0;
    for (int tile = 0; tile < p.T; tile++) {
        a = __dadd_rn(a, p.part[0][(bh * p.T + tile) * D + c]);
        b = __dadd_rn(b, p.part[1][(bh * p.T + tile) * D + c]);
    }
    const double r = (a > 0.0 && b > 0.0) ? __dsqrt_rn(__dsqrt_rn(__ddiv_rn(a, b))) : 1.0;
    p.r[bh * 2 * D + c] = r;
    p.r[bh * 2 * D + D + c] = __ddiv_rn(1.0, r);
    if (p.r_out) p.r_out[bh * D + c] = __double2float_rn(r);
}

// The balancing factors of tensor `which`: 1/r for Q' (which = 0), r for K'.
SA_DEV const double* ip_factors(const IpParams& p, int which, size_t bh, int D)
{
    return p.r + bh * 2 * D + (which ? 0 : D);
}

// Q' = fl32(y (1/r)), K' = fl32(y r) for one element.
SA_DEV float ip_balance1(float y, const double* f, int j)
{
    return __double2float_rn(__dmul_rn((double)y, __ldg(f + j)));
}

// grid (T, B*H, 2), 128 threads.
template <int D>
__global__ void __launch_bounds__(128) ip_amax_kernel(const IpParams p)
{
    __shared__ float sgn[D];
    const int tile = blockIdx.x, which = blockIdx.z, t = threadIdx.x;
    const size_t bh = blockIdx.y;
    const int rows = min(128, p.N - tile * 128);
    ip_load_signs<D>(p, sgn);
    __syncthreads();
    float m = 0.0f;
    bool bad = false;
    if (t < rows) {
        float y[D];
        ip_rotate_row<D>(p, which, bh, tile * 128 + t, sgn, y);
        const double* f = ip_factors(p, which, bh, D);
#pragma unroll
        for (int j = 0; j < D; j++) {
            const float v = ip_balance1(y[j], f, j);
            bad |= !isfinite(v);
            m = fmaxf(m, fabsf(v));
        }
    }
    if (bad) sa_raise(SA_ERR_NONFINITE);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & 31) == 0 && m > 0.0f) atomicMax(&p.amax[which], __float_as_uint(m));
}

struct IpOut {
    uint8_t* codes[2];   // [B*H, N, D/2]
    uint8_t* scales[2];  // Q/K scale atoms
    float* g[2];         // {g, 1/g}
    int8_t* ss_off[2];   // [B*H, N, D/16] or nullptr
    int f_lo, f_hi;
};

// grid (T, B*H, 2), 128 threads: thread t encodes the D/16 blocks of row t.
template <int D, bool SEARCH>
__global__ void __launch_bounds__(128) ip_quant_kernel(const IpParams p, const IpOut o)
{
    constexpr int NB = D / 16;
    __shared__ float sgn[D];
    __shared__ float rcp[128];
    __shared__ uint32_t atoms[2 * 128];
    const int tile = blockIdx.x, which = blockIdx.z, t = threadIdx.x;
    const size_t bh = blockIdx.y;
    const int rows = min(128, p.N - tile * 128);
    ip_load_signs<D>(p, sgn);
    fill_rcp_table(rcp);
    for (int i = t; i < 256; i += blockDim.x) atoms[i] = 0u;
    float g, inv_g;
    tensor_scale(__uint_as_float(p.amax[which]), g, inv_g);
    if (tile == 0 && bh == 0 && t == 0) {
        o.g[which][0] = g;
        o.g[which][1] = inv_g;
    }
    __syncthreads();
    if (t < rows) {
        float y[D];
        ip_rotate_row<D>(p, which, bh, tile * 128 + t, sgn, y);
        const double* f = ip_factors(p, which, bh, D);
        const size_t row = bh * p.N + (size_t)tile * 128 + t;
        uint2* codes = reinterpret_cast<uint2*>(o.codes[which]) + row * NB;
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < NB; j++) {
            float xt[16];
#pragma unroll
            for (int i = 0; i < 16; i++) xt[i] = __fmul_rn(ip_balance1(y[16 * j + i], f, 16 * j + i), inv_g);
            uint32_t c0, c1, sc;
            int off;
            quant16<SEARCH>(xt, o.f_lo, o.f_hi, c0, c1, sc, off, rcp);
            codes[j] = make_uint2(c0, c1);
            if (o.ss_off[which]) o.ss_off[which][row * NB + j] = (int8_t)off;
            word |= sc << (8 * (j & 3));
            if ((j & 3) == 3) {
                atoms[(j >> 2) * 128 + (t & 31) * 4 + (t >> 5)] = word;
                word = 0;
            }
        }
    }
    __syncthreads();
    store_rows_atoms<D>(atoms, bh, tile, p.T, o.scales[which]);
}

// Workspace: amax words, the K statistics of the smoothing mean, the tile
// sums of squares and r.
struct IpWs {
    unsigned* amax;  // [0] Q', [1] K', [2] K - mu (written by the mean pass, unused)
    QuantWs kst;     // K statistics (psum, pmax, pmin, kmean)
    double* part[2];
    double* r;
    size_t bytes;
};

static IpWs ip_ws_layout(void* base, int B, int H, int N, int D)
{
    IpWs w{};
    char* p = (char*)base;
    const size_t BH = (size_t)B * H, T = (size_t)sa_cdiv(N, kTile);
    w.amax = (unsigned*)p;
    size_t off = 256;
    w.kst = quant_ws_layout(p ? p + off : nullptr, B, H, N, D, SA_ROLE_K);
    off += w.kst.bytes;
    for (int i = 0; i < 2; i++) {
        w.part[i] = (double*)(p + off);
        off += sa_align256(BH * T * D * sizeof(double));
    }
    w.r = (double*)(p + off);
    off += sa_align256(BH * 2 * D * sizeof(double));
    w.bytes = off;
    return w;
}

}  // namespace sa
