// quant.cuh -- NVFP4 pre-pass: K smoothing statistics, per-tensor amax and
// block quantisation (max-scaling or ScaleSearch).
//
// "Search Your Block Floating Point Scales!" (gist.science summary),
// "방법론 / ScaleSearch": max-scaling s = round(max|x|/6); ScaleSearch tries
// E4M3 scale bytes c0+f and keeps the lowest block squared error.
// "SageAttention" (hotpaper.ai), "기술적 접근법": K minus its per-channel
// mean over tokens.
//
// Kernels (all HBM-streaming, 16-byte loads where the layout allows):
//   amax_bf16_kernel   max |x| over a tensor on the bf16 bit patterns
//                      (|x| order == unsigned order of (bits & 0x7FFF)).
//   kstats_kernel      per (b,h,128-token tile, channel): FP64 sum in token
//                      order, max, min.
//   kfinal_kernel      per (b,h,channel): tile partials in tile order -> mean;
//                      amax of K - mean from max/min (rounding is monotone).
//   quant_rows_kernel  Q/K: one thread per 16-channel block.
//   quant_v_kernel     V: one thread per 16-token block of four channels.
#pragma once

#include "common.cuh"

namespace sa {

constexpr int kTile = 128;

// ---------------------------------------------------------------------------
// Block quantisation (device)
// ---------------------------------------------------------------------------

// Codes of 16 g-normalised values for scale byte c: r = 1/s (IEEE),
// y = x~ * r (IEEE), E2M1 round-to-nearest-even.  c == 0 -> all zero.
SA_DEV void encode16(const float (&xt)[16], uint32_t c, uint32_t& w0, uint32_t& w1)
{
    if (c == 0) {
        w0 = w1 = 0;
        return;
    }
    float r = __frcp_rn(e4m3_to_f32(c));
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; i++) y[i] = __fmul_rn(xt[i], r);
    w0 = pack8_e2m1(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
    w1 = pack8_e2m1(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
}

// Squared error of a coded block: e_i = x~_i - v_i*s (v_i*s exact), two
// interleaved fmaf accumulators, summed at the end.
SA_DEV float err16(const float (&xt)[16], uint32_t c, uint32_t w0, uint32_t w1)
{
    float s = e4m3_to_f32(c);
    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) {
        uint32_t nib = ((i < 8 ? w0 : w1) >> (4 * (i & 7))) & 15u;
        float e = __fsub_rn(xt[i], __fmul_rn(e2m1_to_f32(nib), s));
        if (i & 1)
            a1 = __fmaf_rn(e, e, a1);
        else
            a0 = __fmaf_rn(e, e, a0);
    }
    return __fadd_rn(a0, a1);
}

// One block: max-scaling base byte c0 = E4M3(amax/6); with SEARCH, offsets
// f in [f_lo, f_hi) \ {0} are tried in ascending order and replace the best
// only when strictly better (f = 0 wins ties, then the lowest f).
template <bool SEARCH>
SA_DEV void quant16(const float (&xt)[16], int f_lo, int f_hi, uint32_t& w0, uint32_t& w1, uint32_t& sc, int& off)
{
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) amax = fmaxf(amax, fabsf(xt[i]));
    uint32_t c0 = f32_to_e4m3(__fdiv_rn(amax, 6.0f));
    encode16(xt, c0, w0, w1);
    sc = c0;
    off = 0;
    if (SEARCH && c0 != 0) {
        float best = err16(xt, c0, w0, w1);
        for (int f = f_lo; f < f_hi; ++f) {
            int c = (int)c0 + f;
            if (f == 0 || c < 0 || c > 0x7E) continue;
            uint32_t t0, t1;
            encode16(xt, (uint32_t)c, t0, t1);
            float e = err16(xt, (uint32_t)c, t0, t1);
            if (e < best) {
                best = e;
                sc = (uint32_t)c;
                off = f;
                w0 = t0;
                w1 = t1;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Statistics kernels
// ---------------------------------------------------------------------------

// max |x| over n16 groups of 8 bf16; raises SA_ERR_NONFINITE on inf/NaN.
// Four independent 16-byte loads per thread and iteration.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint4* __restrict__ x, size_t n16,
                                                        unsigned* __restrict__ amax_word)
{
    uint32_t m = 0;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; u++) v[u] = __ldcs(x + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; u++) {
            m = __vmaxu2(m, v[u].x & 0x7FFF7FFFu);
            m = __vmaxu2(m, v[u].y & 0x7FFF7FFFu);
            m = __vmaxu2(m, v[u].z & 0x7FFF7FFFu);
            m = __vmaxu2(m, v[u].w & 0x7FFF7FFFu);
        }
    }
    for (; i < n16; i += stride) {
        uint4 v = __ldcs(x + i);
        m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    }
    uint32_t mm = max(m & 0xFFFFu, m >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mm = max(mm, __shfl_xor_sync(0xffffffffu, mm, o));
    __shared__ uint32_t red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mm;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) b = max(b, red[w]);
        if (b >= 0x7F80u) sa_raise(SA_ERR_NONFINITE);
        atomicMax(amax_word, __float_as_uint(bf16_bits_to_f32(b)));
    }
}

// K statistics per (b,h, 128-token tile): each thread owns a channel pair and
// walks the tile's tokens in ascending order (FP64 sum, FP32 max/min).
template <int D>
__global__ void __launch_bounds__(256) kstats_kernel(const uint32_t* __restrict__ x, int N, int T,
                                                     double* __restrict__ psum, float* __restrict__ pmax,
                                                     float* __restrict__ pmin)
{
    constexpr int P = D / 2;       // channel pairs per row
    constexpr int TPB = 256 / P;   // tiles per block
    int cp = threadIdx.x % P;
    int tile = blockIdx.x * TPB + threadIdx.x / P;
    size_t bh = blockIdx.y;
    if (tile >= T) return;
    int r0 = tile * kTile;
    int rows = min(kTile, N - r0);
    const uint32_t* p = x + (bh * N + r0) * P + cp;
    double s0 = 0.0, s1 = 0.0;
    float mx0 = -INFINITY, mx1 = -INFINITY, mn0 = INFINITY, mn1 = INFINITY;
    bool bad = false;
    for (int r0b = 0; r0b < rows; r0b += 16) {
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < 16; u++) w[u] = r0b + u < rows ? __ldcs(p + (size_t)(r0b + u) * P) : 0u;
        const int nr = min(16, rows - r0b);
#pragma unroll
        for (int u = 0; u < 16; u++) {
            if (u >= nr) break;
            float a = bf16_bits_to_f32(w[u] & 0xFFFFu), b = bf16_bits_to_f32(w[u] >> 16);
            bad |= !isfinite(a) || !isfinite(b);
            s0 = __dadd_rn(s0, (double)a);  // tokens in ascending order
            s1 = __dadd_rn(s1, (double)b);
            mx0 = fmaxf(mx0, a);
            mx1 = fmaxf(mx1, b);
            mn0 = fminf(mn0, a);
            mn1 = fminf(mn1, b);
        }
    }
    if (bad) sa_raise(SA_ERR_NONFINITE);
    size_t o = (bh * T + tile) * D + 2 * cp;
    psum[o] = s0;
    psum[o + 1] = s1;
    pmax[o] = mx0;
    pmax[o + 1] = mx1;
    pmin[o] = mn0;
    pmin[o + 1] = mn1;
}

// Per (b,h,channel): sum the tile partials in tile order, mean = FP32(sum/N);
// amax contribution max(fl(max - mean), fl(mean - min)).
__global__ void __launch_bounds__(128) kfinal_kernel(const double* __restrict__ psum,
                                                     const float* __restrict__ pmax,
                                                     const float* __restrict__ pmin, int N, int T, int D,
                                                     float* __restrict__ kmean, unsigned* __restrict__ amax_word)
{
    size_t bh = blockIdx.x;
    int c = threadIdx.x;
    float a = 0.0f;
    if (c < D) {
        double total = 0.0;
        float mx = -INFINITY, mn = INFINITY;
        for (int t0 = 0; t0 < T; t0 += 8) {
            double ps[8];
            float px[8], pn[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const size_t o = (bh * T + min(t0 + u, T - 1)) * D + c;
                ps[u] = psum[o];
                px[u] = pmax[o];
                pn[u] = pmin[o];
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                if (t0 + u >= T) break;
                total = __dadd_rn(total, ps[u]);  // tiles in ascending order
                mx = fmaxf(mx, px[u]);
                mn = fminf(mn, pn[u]);
            }
        }
        float mu = __double2float_rn(__ddiv_rn(total, (double)N));
        kmean[bh * D + c] = mu;
        a = fmaxf(__fsub_rn(mx, mu), __fsub_rn(mu, mn));
        a = fmaxf(a, 0.0f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_word, __float_as_uint(a));
}

// ---------------------------------------------------------------------------
// Quantisation kernels
// ---------------------------------------------------------------------------

// Q/K: thread per 16-channel block.  nblk = B*H*N*(D/16).
template <int D, bool SMOOTH, bool SEARCH>
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint4* __restrict__ x, size_t nblk, int N, int RT,
                                                         const float* __restrict__ kmean,
                                                         const unsigned* __restrict__ amax_word, int f_lo,
                                                         int f_hi, uint2* __restrict__ codes,
                                                         uint8_t* __restrict__ scales,
                                                         int8_t* __restrict__ ss_off, float* __restrict__ g_out)
{
    constexpr int NB = D / 16, CK = D / 64;
    float g, inv_g;
    tensor_scale(__uint_as_float(*amax_word), g, inv_g);
    size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t b0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b0 == 0) {
        g_out[0] = g;
        g_out[1] = inv_g;
    }
    for (size_t b = b0; b < nblk; b += stride) {
        size_t row = b / NB;
        int j = (int)(b % NB);
        size_t bh = row / N;
        int n = (int)(row % N);
        uint4 u0 = __ldcs(x + 2 * b), u1 = __ldcs(x + 2 * b + 1);
        uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        float xt[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            float v = bf16_bits_to_f32((w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
            if (SMOOTH) v = __fsub_rn(v, __ldg(kmean + bh * D + j * 16 + i));
            xt[i] = __fmul_rn(v, inv_g);
        }
        uint32_t c0, c1, sc;
        int off;
        quant16<SEARCH>(xt, f_lo, f_hi, c0, c1, sc, off);
        codes[b] = make_uint2(c0, c1);
        size_t atom = (bh * RT + (size_t)(n >> 7)) * CK + (size_t)(j >> 2);
        scales[atom * 512 + sf_atom_offset((uint32_t)(n & 127), (uint32_t)(j & 3))] = (uint8_t)sc;
        if (ss_off) ss_off[b] = (int8_t)off;
    }
}

// V: thread per (4 channels, 16-token block); codes land in 128-token tiles
// [B,H,ceil(N/128),D,64] (each tile's V^T block is one contiguous D x 64-byte
// region, the operand of one P V MMA).
// nblk4 = B*H*(N/16)*(D/4), channel group fastest so a warp reads 256
// contiguous bytes of each token row.
template <bool SEARCH>
__global__ void __launch_bounds__(256) quant_v_kernel(const uint16_t* __restrict__ x, size_t nblk4, int N, int D,
                                                      const unsigned* __restrict__ amax_word, int f_lo, int f_hi,
                                                      uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                      int8_t* __restrict__ ss_off, float* __restrict__ g_out)
{
    float g, inv_g;
    tensor_scale(__uint_as_float(*amax_word), g, inv_g);
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t b0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b0 == 0) {
        g_out[0] = g;
        g_out[1] = inv_g;
    }
    const int NBT = N / 16, D4 = D / 4;
    const int RT = (D + 127) / 128, CK = (N + 63) / 64, NT = (N + 127) / 128;
    for (size_t b = b0; b < nblk4; b += stride) {
        const int c0 = (int)(b % D4) * 4;
        const size_t rest = b / D4;
        const int nb = (int)(rest % NBT);
        const size_t bh = rest / NBT;
        const uint16_t* p = x + (bh * N + (size_t)nb * 16) * D + c0;
        uint2 w[16];
#pragma unroll
        for (int i = 0; i < 16; i++) w[i] = __ldcs(reinterpret_cast<const uint2*>(p + (size_t)i * D));
#pragma unroll
        for (int cc = 0; cc < 4; cc++) {
            float xt[16];
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const uint32_t word = cc < 2 ? w[i].x : w[i].y;
                xt[i] = __fmul_rn(bf16_bits_to_f32((word >> (16 * (cc & 1))) & 0xFFFFu), inv_g);
            }
            uint32_t q0, q1, sc;
            int off;
            quant16<SEARCH>(xt, f_lo, f_hi, q0, q1, sc, off);
            const int c = c0 + cc;
            const size_t crow = bh * D + c;
            *reinterpret_cast<uint2*>(codes + ((bh * NT + (size_t)(nb >> 3)) * D + c) * 64 + (size_t)(nb & 7) * 8) =
                make_uint2(q0, q1);
            const size_t atom = (bh * RT + (size_t)(c >> 7)) * CK + (size_t)(nb >> 2);
            scales[atom * 512 + sf_atom_offset((uint32_t)(c & 127), (uint32_t)(nb & 3))] = (uint8_t)sc;
            if (ss_off) ss_off[crow * NBT + nb] = (int8_t)off;
        }
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct QuantWs {
    unsigned* amax;
    double* psum;
    float* pmax;
    float* pmin;
    float* kmean;
    size_t bytes;
};

static QuantWs quant_ws_layout(void* base, int B, int H, int N, int D, sa_role role)
{
    QuantWs w{};
    char* p = (char*)base;
    size_t off = 0;
    w.amax = (unsigned*)(p + off);
    off += 256;
    if (role == SA_ROLE_K) {
        size_t BH = (size_t)B * H, T = (size_t)sa_cdiv(N, kTile);
        w.psum = (double*)(p + off);
        off += sa_align256(BH * T * D * sizeof(double));
        w.pmax = (float*)(p + off);
        off += sa_align256(BH * T * D * sizeof(float));
        w.pmin = (float*)(p + off);
        off += sa_align256(BH * T * D * sizeof(float));
        w.kmean = (float*)(p + off);
        off += sa_align256(BH * D * sizeof(float));
    }
    w.bytes = off;
    return w;
}

static int grid_for(size_t work, int threads)
{
    size_t g = (work + threads - 1) / threads;
    size_t cap = 148 * 16;
    return (int)(g < cap ? (g > 0 ? g : 1) : cap);
}

}  // namespace sa
