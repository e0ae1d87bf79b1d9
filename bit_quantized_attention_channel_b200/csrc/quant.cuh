// quant.cuh -- NVFP4 pre-pass: K smoothing statistics, per-tensor amax and
// block quantisation (max-scaling or ScaleSearch).
//
// "Search Your Block Floating Point Scales!" (gist.science summary),
// "방법론 / ScaleSearch": max-scaling s = round(max|x|/6); ScaleSearch tries
// E4M3 scale bytes c0+f and keeps the lowest block squared error.
// "SageAttention" (hotpaper.ai), "기술적 접근법": K minus its per-channel
// mean over tokens.
//
// Kernels (all HBM-streaming; tiles move by 16-byte loads or bulk copies):
//   Per tensor (sa_quant_nvfp4):
//   amax_bf16_kernel      max |x| over a tensor on the bf16 bit patterns
//                         (|x| order == unsigned order of (bits & 0x7FFF)).
//   kstats_kernel         per (b,h,128-token tile, channel): FP64 sum in
//                         token order, max, min.
//   kfinal_kernel         per (b,h,channel): tile partials in tile order ->
//                         mean; amax of K - mean from max/min (rounding is
//                         monotone).
//   quant_rows_kernel     Q/K: one CTA per 128-row tile, one bulk copy.
//   quant_v_kernel        V: one CTA per 128-token tile, one bulk copy.
//   Q, K and V together (sa_quant_nvfp4_qkv), the same bytes:
//   prepass_stats_kernel  K tiles (statistics, ticketed final reduction),
//                         then the Q and V amax.
//   prepass_quant_kernel  persistent; V, Q, K tiles double-buffered in
//                         shared memory.
#pragma once

#include "common.cuh"
#include "tc.cuh"

namespace sa {

constexpr int kTile = 128;

// ---------------------------------------------------------------------------
// Block quantisation (device)
// ---------------------------------------------------------------------------

// x / 6 rounded to nearest even.  Method: P. Markstein's FMA correction of a
// reciprocal-product quotient ("Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): q0 = RN(x y) with
// y = RN(1/6), the remainder r = x - 6 q0 exact in one FMA, then
// q = RN(q0 + r y).  For x >= 2^-120 this equals the IEEE quotient (checked
// exhaustively over every float in that range against the hardware's
// correctly rounded division); smaller x divide directly.
SA_DEV float div6_rn(float x)
{
    if (x < 7.52316384526264e-37f) return __fdiv_rn(x, 6.0f);  // 2^-120
    const float r6 = 0.16666667163372040f;                    // RN(1/6)
    const float q0 = __fmul_rn(x, r6);
    return __fmaf_rn(__fmaf_rn(-q0, 6.0f, x), r6, q0);
}

// Exact reciprocals of the 127 nonzero E4M3 scale values (IEEE RN), one
// table per CTA in shared memory.
SA_DEV void fill_rcp_table(float* rcp)
{
    for (int c = threadIdx.x; c < 128; c += blockDim.x) rcp[c] = c ? __frcp_rn(e4m3_to_f32((uint32_t)c)) : 0.0f;
}

// Two products a_i * b in one instruction (IEEE RN per lane).
SA_DEV void mul2_rn(float a0, float a1, float b, float& r0, float& r1)
{
    asm("{\n\t.reg .b64 a, bb, d;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 bb, {%4, %4};\n\t"
        "mul.rn.f32x2 d, a, bb;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b));
}

// Codes of 16 g-normalised values for scale byte c: r = 1/s (IEEE),
// y = x~ * r (IEEE), E2M1 round-to-nearest-even.  c == 0 -> all zero.
SA_DEV void encode16(const float (&xt)[16], uint32_t c, uint32_t& w0, uint32_t& w1, const float* rcp)
{
    if (c == 0) {
        w0 = w1 = 0;
        return;
    }
    const float r = rcp[c];
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; i += 2) mul2_rn(xt[i], xt[i + 1], r, y[i], y[i + 1]);
    w0 = pack8_e2m1(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
    w1 = pack8_e2m1(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
}

// The eight E2M1 codes of a word (byte k = elements 2k, 2k+1, low nibble
// first) as exact floats: one hardware conversion per byte to an f16 pair,
// then f16 -> f32 (every E2M1 value is exact in both).
SA_DEV void e2m1x8_to_f32(uint32_t w, float (&v)[8])
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 h0, h1, h2, h3;\n\t.reg .b16 l0, u0, l1, u1, l2, u2, l3, u3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %8;\n\t"
        "cvt.rn.f16x2.e2m1x2 h0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 h2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
        "mov.b32 {l0, u0}, h0;\n\t"
        "mov.b32 {l1, u1}, h1;\n\t"
        "mov.b32 {l2, u2}, h2;\n\t"
        "mov.b32 {l3, u3}, h3;\n\t"
        "cvt.f32.f16 %0, l0;\n\t"
        "cvt.f32.f16 %1, u0;\n\t"
        "cvt.f32.f16 %2, l1;\n\t"
        "cvt.f32.f16 %3, u1;\n\t"
        "cvt.f32.f16 %4, l2;\n\t"
        "cvt.f32.f16 %5, u2;\n\t"
        "cvt.f32.f16 %6, l3;\n\t"
        "cvt.f32.f16 %7, u3;\n\t}"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "r"(w));
}

// d_i = a_i * b_i + c_i for a pair (IEEE RN per lane, one instruction).
SA_DEV void fma2_rn(float a0, float a1, float b0, float b1, float c0, float c1, float& d0, float& d1)
{
    asm("{\n\t.reg .b64 a, b, c, d;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 b, {%4, %5};\n\t"
        "mov.b64 c, {%6, %7};\n\t"
        "fma.rn.f32x2 d, a, b, c;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// Squared error of a coded block: e_i = x~_i - v_i*s (v_i*s is exact, so one
// rounded fma(-v_i, s, x~_i) gives it), two interleaved accumulators
// a_(i mod 2) = fma(e_i, e_i, a_(i mod 2)) over i ascending, summed at the
// end.  Elements 2k and 2k+1 share one paired instruction, lane 0 even.
SA_DEV float err16(const float (&xt)[16], uint32_t c, uint32_t w0, uint32_t w1)
{
    const float s = e4m3_to_f32(c);
    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
    for (int h = 0; h < 2; h++) {
        float v[8];
        e2m1x8_to_f32(h ? w1 : w0, v);
#pragma unroll
        for (int k = 0; k < 4; k++) {
            float e0, e1;
            fma2_rn(-v[2 * k], -v[2 * k + 1], s, s, xt[8 * h + 2 * k], xt[8 * h + 2 * k + 1], e0, e1);
            fma2_rn(e0, e1, e0, e1, a0, a1, a0, a1);
        }
    }
    return __fadd_rn(a0, a1);
}

// One block: max-scaling base byte c0 = E4M3(amax/6); with SEARCH, offsets
// f in [f_lo, f_hi) \ {0} are tried in ascending order and replace the best
// only when strictly better (f = 0 wins ties, then the lowest f).
template <bool SEARCH>
SA_DEV void quant16(const float (&xt)[16], int f_lo, int f_hi, uint32_t& w0, uint32_t& w1, uint32_t& sc, int& off,
                    const float* rcp)
{
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; i++) a[i] = fmaxf(fabsf(xt[2 * i]), fabsf(xt[2 * i + 1]));
    const float amax = fmaxf(fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])), fmaxf(fmaxf(a[4], a[5]), fmaxf(a[6], a[7])));
    uint32_t c0 = f32_to_e4m3(div6_rn(amax));
    encode16(xt, c0, w0, w1, rcp);
    sc = c0;
    off = 0;
    if (SEARCH && c0 != 0) {
        float best = err16(xt, c0, w0, w1);
#pragma unroll 1
        for (int f = f_lo; f < f_hi; ++f) {
            int c = (int)c0 + f;
            if (f == 0 || c < 0 || c > 0x7E) continue;
            uint32_t t0, t1;
            encode16(xt, (uint32_t)c, t0, t1, rcp);
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

// K statistics of one (b,h, 128-token tile, channel pair): tokens in ascending
// order (FP64 sum, FP32 max/min).  Returns false on a non-finite value.
template <int D>
SA_DEV bool kstats_pair(const uint32_t* __restrict__ x, int N, int T, size_t bh, int tile, int cp,
                        double* __restrict__ psum, float* __restrict__ pmax, float* __restrict__ pmin)
{
    constexpr int P = D / 2;  // channel pairs per row
    const int r0 = tile * kTile;
    const int rows = min(kTile, N - r0);
    const uint32_t* p = x + (bh * N + r0) * P + cp;
    double s0 = 0.0, s1 = 0.0;
    float mx0 = -INFINITY, mx1 = -INFINITY, mn0 = INFINITY, mn1 = INFINITY;
    bool bad = false;
    for (int r0b = 0; r0b < rows; r0b += 32) {
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 32; u++) w[u] = r0b + u < rows ? __ldg(p + (size_t)(r0b + u) * P) : 0u;
        const int nr = min(32, rows - r0b);
#pragma unroll
        for (int u = 0; u < 32; u++) {
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
    const size_t o = (bh * T + tile) * D + 2 * cp;
    psum[o] = s0;
    psum[o + 1] = s1;
    pmax[o] = mx0;
    pmax[o + 1] = mx1;
    pmin[o] = mn0;
    pmin[o + 1] = mn1;
    return !bad;
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
    const int cp = threadIdx.x % P;
    const int tile = blockIdx.x * TPB + threadIdx.x / P;
    if (tile >= T) return;
    if (!kstats_pair<D>(x, N, T, blockIdx.y, tile, cp, psum, pmax, pmin)) sa_raise(SA_ERR_NONFINITE);
}

// Per (b,h,channel): sum the tile partials in tile order, mean = FP32(sum/N);
// returns the amax contribution max(fl(max - mean), fl(mean - min)), >= 0.
// Partials are read through L2 (they may come from other CTAs of this grid).
SA_DEV float kfinal_channel(const double* __restrict__ psum, const float* __restrict__ pmax,
                            const float* __restrict__ pmin, int N, int T, int D, size_t bh, int c,
                            float* __restrict__ kmean)
{
    double total = 0.0;
    float mx = -INFINITY, mn = INFINITY;
    for (int t0 = 0; t0 < T; t0 += 8) {
        double ps[8];
        float px[8], pn[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const size_t o = (bh * T + min(t0 + u, T - 1)) * D + c;
            ps[u] = __ldcg(psum + o);
            px[u] = __ldcg(pmax + o);
            pn[u] = __ldcg(pmin + o);
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            if (t0 + u >= T) break;
            total = __dadd_rn(total, ps[u]);  // tiles in ascending order
            mx = fmaxf(mx, px[u]);
            mn = fminf(mn, pn[u]);
        }
    }
    const float mu = __double2float_rn(__ddiv_rn(total, (double)N));
    kmean[bh * D + c] = mu;
    return fmaxf(fmaxf(__fsub_rn(mx, mu), __fsub_rn(mu, mn)), 0.0f);
}

__global__ void __launch_bounds__(128) kfinal_kernel(const double* __restrict__ psum,
                                                     const float* __restrict__ pmax,
                                                     const float* __restrict__ pmin, int N, int T, int D,
                                                     float* __restrict__ kmean, unsigned* __restrict__ amax_word)
{
    const size_t bh = blockIdx.x;
    const int c = threadIdx.x;
    float a = c < D ? kfinal_channel(psum, pmax, pmin, N, T, D, bh, c, kmean) : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_word, __float_as_uint(a));
}

// ---------------------------------------------------------------------------
// Quantisation kernels
// ---------------------------------------------------------------------------

// ---------------------------------------------------------------------------
// Tile quantisers: one (b,h, 128-row tile) of Q/K or (b,h, 128-token tile) of
// V, already in shared memory as row-major bf16 (rows x D, the bytes of one
// bulk copy: a tile is contiguous in the [B,H,N,D] input).  Each CTA has 2 D
// threads.  Codes go out coalesced; the four scale bytes of a 64-element
// chunk form one word of the tile's scale atoms in shared memory, which the
// caller writes out (padding zero) after a barrier.  Per block the arithmetic
// is quant16.
// ---------------------------------------------------------------------------

// Bytes of tile `tile` of a [*, N, D] bf16 tensor slice bh, and its address.
SA_DEV uint32_t tile_bytes(int N, int D, int tile) { return (uint32_t)(min(kTile, N - tile * kTile) * D * 2); }
SA_DEV const void* tile_src(const void* x, size_t bh, int N, int D, int tile)
{
    return (const uint8_t*)x + ((bh * N + (size_t)tile * kTile) * D) * 2;
}

// Q/K: thread t encodes blocks b = t + 2 D k (k = 0..3), row b / (D/16),
// block j = b % (D/16).  The eight threads of a shared-memory phase read
// eight consecutive blocks (32 bytes each); thread t reads the half
// ((t >> 2) & 1) first, so each phase touches eight different bank groups.
template <int D, bool SMOOTH, bool SEARCH>
SA_DEV void quant_rows_smem(const uint4* xs, size_t bh, int tile, int N, const float* __restrict__ kmean, float inv_g,
                            int f_lo, int f_hi, uint2* __restrict__ codes, int8_t* __restrict__ ss_off,
                            uint32_t* atoms /* shared, D/64 * 128 words */, const float* rcp)
{
    constexpr int NB = D / 16, RP = D / 8, NTH = 2 * D;
    const int t = threadIdx.x;
    const int rows = min(kTile, N - tile * kTile);
    const int sw = (t >> 2) & 1;
    float km[16];  // NTH is a multiple of NB: the block column j is t % NB on every pass
    if (SMOOTH) {
#pragma unroll
        for (int i = 0; i < 16; i++) km[i] = __ldg(kmean + bh * D + (t % NB) * 16 + i);
    }
#pragma unroll 1
    for (int k = 0; k < 4; k++) {
        const int b = t + k * NTH, r = b / NB, j = b % NB;
        uint32_t sc = 0;
        if (r < rows) {
            const uint4 pa = xs[r * RP + 2 * j + sw], pb = xs[r * RP + 2 * j + 1 - sw];
            const uint4 lo = sw ? pb : pa, hi = sw ? pa : pb;
            const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            float xt[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                float v0 = __uint_as_float(w[i >> 1] << 16), v1 = __uint_as_float(w[i >> 1] & 0xFFFF0000u);
                if (SMOOTH) {
                    v0 = __fsub_rn(v0, km[i]);
                    v1 = __fsub_rn(v1, km[i + 1]);
                }
                mul2_rn(v0, v1, inv_g, xt[i], xt[i + 1]);
            }
            uint32_t c0, c1;
            int off;
            quant16<SEARCH>(xt, f_lo, f_hi, c0, c1, sc, off, rcp);
            const size_t row = bh * N + (size_t)tile * kTile + r;
            codes[row * NB + j] = make_uint2(c0, c1);
            if (ss_off) ss_off[row * NB + j] = (int8_t)off;
        }
        // the four lanes t & ~3 .. t | 3 hold blocks 4 m .. 4 m + 3 of row r
        uint32_t word = sc << (8 * (j & 3));
        word |= __shfl_xor_sync(0xffffffffu, word, 1);
        word |= __shfl_xor_sync(0xffffffffu, word, 2);
        if ((j & 3) == 0) atoms[(j >> 2) * 128 + (r & 31) * 4 + (r >> 5)] = word;
    }
}

// Q/K scale atoms (bh, tile, chunk): 512 bytes = 32 x uint4 each.
template <int D>
SA_DEV void store_rows_atoms(const uint32_t* atoms, size_t bh, int tile, int T, uint8_t* __restrict__ scales)
{
    constexpr int CK = D / 64;
    for (int i = threadIdx.x; i < CK * 32; i += blockDim.x) {
        const int ck = i / 32, q = i % 32;
        const uint32_t* a = atoms + ck * 128 + q * 4;
        reinterpret_cast<uint4*>(scales + (((size_t)bh * T + tile) * CK + ck) * 512)[q] = make_uint4(a[0], a[1], a[2], a[3]);
    }
}

// V: thread t -> channel t % D, token half t / D (blocks 4 half .. 4 half + 3
// of the tile, 16 tokens each).  Atom words of padded rows are written zero.
template <int D, bool SEARCH>
SA_DEV void quant_v_smem(const uint16_t* xs, size_t bh, int tile, int N, float inv_g, int f_lo, int f_hi,
                         uint8_t* __restrict__ codes, int8_t* __restrict__ ss_off,
                         uint32_t* atoms /* shared, 2 * 128 words */, const float* rcp)
{
    const int t = threadIdx.x;
    const int NT = (N + 127) / 128, NBT = N / 16;
    const int rows = min(kTile, N - tile * kTile);
    const int c = t % D, half = t / D;
    uint32_t word = 0, offw = 0;
    uint2 cw[4] = {make_uint2(0, 0), make_uint2(0, 0), make_uint2(0, 0), make_uint2(0, 0)};
#pragma unroll
    for (int jb = 0; jb < 4; jb++) {
        const int tok0 = half * 64 + jb * 16;
        if (tok0 >= rows) break;
        float xt[16];
#pragma unroll
        for (int i = 0; i < 16; i += 2)
            mul2_rn(bf16_bits_to_f32(xs[(tok0 + i) * D + c]), bf16_bits_to_f32(xs[(tok0 + i + 1) * D + c]), inv_g,
                    xt[i], xt[i + 1]);
        uint32_t q0, q1, sc;
        int off;
        quant16<SEARCH>(xt, f_lo, f_hi, q0, q1, sc, off, rcp);
        cw[jb] = make_uint2(q0, q1);
        word |= sc << (8 * jb);
        offw |= ((uint32_t)(uint8_t)(int8_t)off) << (8 * jb);
    }
    const int nblk_here = min(4, max(0, (rows - half * 64) / 16));
    if (nblk_here > 0) {
        uint8_t* dst = codes + (((size_t)bh * NT + tile) * D + c) * 64 + half * 32;
        if (nblk_here == 4) {
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
        } else {
            for (int jb = 0; jb < nblk_here; jb++) reinterpret_cast<uint2*>(dst)[jb] = cw[jb];
        }
        if (ss_off) {
            int8_t* so = ss_off + ((size_t)bh * D + c) * NBT + tile * 8 + half * 4;
            for (int jb = 0; jb < nblk_here; jb++) so[jb] = (int8_t)(offw >> (8 * jb));
        }
    }
    // channel rows D..127 of the atom stay zero (written by the caller once)
    atoms[half * 128 + (c & 31) * 4 + ((c & 127) >> 5)] = word;
}

// V scale atoms (bh, channel tile 0, chunks 2 tile, 2 tile + 1), only chunks
// inside N.
SA_DEV void store_v_atoms(const uint32_t* atoms, size_t bh, int tile, int N, uint8_t* __restrict__ scales)
{
    const int CK = (N + 63) / 64;
    for (int i = threadIdx.x; i < 64; i += blockDim.x) {
        const int h2 = i / 32, q = i % 32;
        const int ck = 2 * tile + h2;
        if (ck >= CK) continue;
        const uint32_t* a = atoms + h2 * 128 + q * 4;
        reinterpret_cast<uint4*>(scales + ((size_t)bh * CK + ck) * 512)[q] = make_uint4(a[0], a[1], a[2], a[3]);
    }
}

// One CTA = one tile: a single bulk copy into shared memory, then the tile
// quantiser.  Returns false (status raised) when the copy never lands.
SA_DEV bool load_tile_once(void* xs, const void* src, uint32_t bytes, uint64_t* bar)
{
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_expect_tx(bar, bytes);
        bulk_load(xs, src, bytes, bar);
    }
    if (__syncthreads_or(!mbar_wait(bar, 0))) {
        if (threadIdx.x == 0) sa_raise(SA_ERR_TIMEOUT);
        return false;
    }
    return true;
}

// Q/K: grid (ceil(N/128), B*H), 2 D threads.
template <int D, bool SMOOTH, bool SEARCH>
__global__ void __launch_bounds__(2 * D) quant_rows_kernel(const uint4* __restrict__ x, int N,
                                                           const float* __restrict__ kmean,
                                                           const unsigned* __restrict__ amax_word, int f_lo, int f_hi,
                                                           uint2* __restrict__ codes, uint8_t* __restrict__ scales,
                                                           int8_t* __restrict__ ss_off, float* __restrict__ g_out)
{
    __shared__ __align__(128) uint4 xs[kTile * D / 8];
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t atoms[2 * 128];
    __shared__ float rcp[128];
    fill_rcp_table(rcp);
    float g, inv_g;
    tensor_scale(__uint_as_float(*amax_word), g, inv_g);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        g_out[0] = g;
        g_out[1] = inv_g;
    }
    const int tile = blockIdx.x;
    if (!load_tile_once(xs, tile_src(x, blockIdx.y, N, D, tile), tile_bytes(N, D, tile), &bar)) return;
    quant_rows_smem<D, SMOOTH, SEARCH>(xs, blockIdx.y, tile, N, kmean, inv_g, f_lo, f_hi, codes, ss_off, atoms, rcp);
    __syncthreads();
    store_rows_atoms<D>(atoms, blockIdx.y, tile, (N + kTile - 1) / kTile, scales);
}

// V: grid (ceil(N/128), B*H), 2 D threads.
template <int D, bool SEARCH>
__global__ void __launch_bounds__(2 * D) quant_v_kernel(const uint16_t* __restrict__ x, int N,
                                                        const unsigned* __restrict__ amax_word, int f_lo, int f_hi,
                                                        uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                        int8_t* __restrict__ ss_off, float* __restrict__ g_out)
{
    __shared__ __align__(128) uint16_t xs[kTile * D];
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t atoms[2 * 128];
    __shared__ float rcp[128];
    fill_rcp_table(rcp);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) atoms[i] = 0u;
    float g, inv_g;
    tensor_scale(__uint_as_float(*amax_word), g, inv_g);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        g_out[0] = g;
        g_out[1] = inv_g;
    }
    const int tile = blockIdx.x;
    if (!load_tile_once(xs, tile_src(x, blockIdx.y, N, D, tile), tile_bytes(N, D, tile), &bar)) return;
    quant_v_smem<D, SEARCH>(xs, blockIdx.y, tile, N, inv_g, f_lo, f_hi, codes, ss_off, atoms, rcp);
    __syncthreads();
    store_v_atoms(atoms, blockIdx.y, tile, N, scales);
}

// ---------------------------------------------------------------------------
// Fused pre-pass of Q, K and V (one statistics launch, one quantisation launch)
// ---------------------------------------------------------------------------

// max over the uint4 groups base + tid + 256 u (u < kAmaxPer) of the bf16
// magnitude bits (|x| order == unsigned order of bits & 0x7FFF): a block
// reads one contiguous 32 KB chunk, so the blocks in flight cover one
// contiguous range and spread over all HBM channels.  All loads are issued
// before the first use.  Normal (L2-keeping) loads: the quantisation pass
// reads the same bytes next.
constexpr int kAmaxPer = 8;
SA_DEV uint32_t amax_bits_batch(const uint4* __restrict__ x, size_t n16, size_t base, int tid)
{
    uint4 v[kAmaxPer];
#pragma unroll
    for (int u = 0; u < kAmaxPer; u++) {
        const size_t i = base + tid + 256 * u;
        v[u] = i < n16 ? __ldg(x + i) : make_uint4(0, 0, 0, 0);
    }
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < kAmaxPer; u++) {
        m = __vmaxu2(m, v[u].x & 0x7FFF7FFFu);
        m = __vmaxu2(m, v[u].y & 0x7FFF7FFFu);
        m = __vmaxu2(m, v[u].z & 0x7FFF7FFFu);
        m = __vmaxu2(m, v[u].w & 0x7FFF7FFFu);
    }
    return max(m & 0xFFFFu, m >> 16);
}

struct PrepassParams {
    const uint4* q;  // bf16 [B,H,N,D]
    const uint4* k;
    const uint4* v;
    int BH, N, T;
    int smooth_k;
    unsigned* amax;    // [3]: Q, K, V (FP32 bits)
    unsigned* ticket;  // [BH]: K-statistics blocks finished per (b,h)
    double* psum;
    float* pmax;
    float* pmin;
    float* kmean;
    int nA;   // amax blocks per tensor (nA * 256 * kAmaxPer >= B H N D / 8)
    int nKS;  // K-statistics blocks (smoothing on): B H T, one tile each
    // quantisation
    uint2* qc;
    uint8_t* qs;
    float* qg;
    uint2* kc;
    uint8_t* ks;
    float* kg;
    uint8_t* vc;
    uint8_t* vs;
    float* vg;
    int f_lo, f_hi;
};

// Channel c of one K tile in shared memory (rows x D bf16, rows % 16 == 0):
// FP64 sum over the tokens in ascending order, FP32 max and min.  A
// non-finite input makes the FP64 sum non-finite (the sum of at most 2^20
// finite bf16 values cannot overflow FP64), which the caller checks.
template <int D>
SA_DEV void kstats_channel_smem(const uint16_t* xs, int rows, int c, double& s, float& mx, float& mn)
{
    s = 0.0;
    mx = -INFINITY;
    mn = INFINITY;
    for (int r0 = 0; r0 < rows; r0 += 16) {
        float x[16];
#pragma unroll
        for (int u = 0; u < 16; u++) x[u] = bf16_bits_to_f32(xs[(r0 + u) * D + c]);
#pragma unroll
        for (int u = 0; u < 16; u++) {
            s = __dadd_rn(s, (double)x[u]);  // tokens in ascending order
            mx = fmaxf(mx, x[u]);
            mn = fminf(mn, x[u]);
        }
    }
}

// With smoothing, blocks [0, B H T) take the K statistics of one (b,h, tile)
// each: one bulk copy of the tile into shared memory, then one FP64 chain per
// channel.  The last block of each (b,h) to finish (a ticket) reduces the
// tile partials: threads [0, D) sum them in tile order (mean), threads
// [D, 2 D) take their max and min (order-free), and the K amax is
// max(fl(max - mean), fl(mean - min)) over the channels.  The K blocks come
// first; the amax blocks that follow (nA for Q, then nA for V; without
// smoothing a third nA for K) stream around them.
template <int D>
__global__ void __launch_bounds__(256) prepass_stats_kernel(const PrepassParams p)
{
    extern __shared__ __align__(128) uint16_t ks_tile[];  // kTile x D bf16 (K blocks only)
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t red[8];
    __shared__ int last;
    __shared__ float fred[8];
    __shared__ float mu_s[128], mx_s[128], mn_s[128];
    const int bid = blockIdx.x, tid = threadIdx.x;
    const size_t n16 = (size_t)p.BH * p.N * D / 8;
    const bool kstat = p.smooth_k && bid < p.nKS;
    if (!kstat) {
        const int a = p.smooth_k ? bid - p.nKS : bid;
        const int which = a < p.nA ? 0 : (a < 2 * p.nA ? 2 : 1);
        const uint4* x = which == 0 ? p.q : (which == 2 ? p.v : p.k);
        const int lb = a - (which == 0 ? 0 : (which == 2 ? p.nA : 2 * p.nA));
        // nA * 256 * kAmaxPer >= n16: one batch per block covers the tensor
        uint32_t mm = amax_bits_batch(x, n16, (size_t)lb * 256 * kAmaxPer, tid);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mm = max(mm, __shfl_xor_sync(0xffffffffu, mm, o));
        if ((tid & 31) == 0) red[tid >> 5] = mm;
        __syncthreads();
        if (tid == 0) {
            uint32_t b = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); w++) b = max(b, red[w]);
            if (b >= 0x7F80u) sa_raise(SA_ERR_NONFINITE);
            atomicMax(&p.amax[which], __float_as_uint(bf16_bits_to_f32(b)));
        }
        return;
    }
    const int bh = bid / p.T, tile = bid - bh * p.T;
    const int rows = min(kTile, p.N - tile * kTile);
    if (!load_tile_once(ks_tile, tile_src(p.k, bh, p.N, D, tile), tile_bytes(p.N, D, tile), &bar)) return;
    if (tid < D) {
        double sum;
        float mx, mn;
        kstats_channel_smem<D>(ks_tile, rows, tid, sum, mx, mn);
        if (!isfinite(sum)) sa_raise(SA_ERR_NONFINITE);
        const size_t o = ((size_t)bh * p.T + tile) * D + tid;
        p.psum[o] = sum;
        p.pmax[o] = mx;
        p.pmin[o] = mn;
    }
    __threadfence();  // partials visible device-wide before the ticket
    __syncthreads();
    if (tid == 0) last = atomicAdd(&p.ticket[bh], 1u) == (unsigned)(p.T - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int T = p.T;
    if (tid < D) {
        double total = 0.0;
        for (int t0 = 0; t0 < T; t0 += 16) {
            double ps[16];
#pragma unroll
            for (int u = 0; u < 16; u++) ps[u] = __ldcg(p.psum + ((size_t)bh * T + min(t0 + u, T - 1)) * D + tid);
#pragma unroll
            for (int u = 0; u < 16; u++)
                if (t0 + u < T) total = __dadd_rn(total, ps[u]);  // tiles in ascending order
        }
        const float mu = __double2float_rn(__ddiv_rn(total, (double)p.N));
        p.kmean[(size_t)bh * D + tid] = mu;
        mu_s[tid] = mu;
    } else if (tid < 2 * D) {
        const int c = tid - D;
        float mx = -INFINITY, mn = INFINITY;
        for (int t0 = 0; t0 < T; t0 += 16) {
            float px[16], pn[16];
#pragma unroll
            for (int u = 0; u < 16; u++) {
                const size_t o = ((size_t)bh * T + min(t0 + u, T - 1)) * D + c;
                px[u] = __ldcg(p.pmax + o);
                pn[u] = __ldcg(p.pmin + o);
            }
#pragma unroll
            for (int u = 0; u < 16; u++) {
                mx = fmaxf(mx, px[u]);  // clamped repeats of tile T - 1 change nothing
                mn = fminf(mn, pn[u]);
            }
        }
        mx_s[c] = mx;
        mn_s[c] = mn;
    }
    __syncthreads();
    float a = 0.0f;
    if (tid < D) a = fmaxf(fmaxf(__fsub_rn(mx_s[tid], mu_s[tid]), __fsub_rn(mu_s[tid], mn_s[tid])), 0.0f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((tid & 31) == 0) fred[tid >> 5] = a;
    __syncthreads();
    if (tid == 0) {
        float b = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) b = fmaxf(b, fred[w]);
        atomicMax(&p.amax[1], __float_as_uint(b));
    }
}

// Persistent quantisation of Q, K and V: gridDim.x CTAs of 2 D threads walk
// the 3 B H T tiles with stride gridDim.x, in the order V, Q, K (the
// statistics pass streams K first, so V and Q are the likelier L2 hits).
// Each CTA double-buffers its tiles in shared memory: the bulk copy of the
// next tile is in flight while the current one is encoded.
template <int D>
struct PqSmem {
    uint4 x[2][kTile * D / 8];
    uint64_t full[2];
    uint32_t atoms[2 * 128];
    float rcp[128];
};

template <int D, bool SEARCH, bool SMOOTH>
__global__ void __launch_bounds__(2 * D) prepass_quant_kernel(const PrepassParams p)
{
    extern __shared__ __align__(128) uint8_t pq_raw[];
    PqSmem<D>& s = *reinterpret_cast<PqSmem<D>*>(pq_raw);
    const int nt = p.BH * p.T, total = 3 * nt;
    // tile j -> tensor (0 Q, 1 K, 2 V), bh, tile
    auto decode = [&](int j, int& which, int& bh, int& tile) {
        const int w = j / nt, lb = j - w * nt;
        which = w == 0 ? 2 : w - 1;
        bh = lb / p.T;
        tile = lb - bh * p.T;
    };
    auto issue = [&](int j, int b) {
        int which, bh, tile;
        decode(j, which, bh, tile);
        const void* x = which == 0 ? (const void*)p.q : (which == 1 ? (const void*)p.k : (const void*)p.v);
        const uint32_t bytes = tile_bytes(p.N, D, tile);
        mbar_expect_tx(&s.full[b], bytes);
        bulk_load(s.x[b], tile_src(x, bh, p.N, D, tile), bytes, &s.full[b]);
    };
    fill_rcp_table(s.rcp);
    if (threadIdx.x == 0) {
        mbar_init(&s.full[0], 1);
        mbar_init(&s.full[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    int j = blockIdx.x;
    if (threadIdx.x == 0 && j < total) issue(j, 0);
    float g[3], inv_g[3];
#pragma unroll
    for (int w = 0; w < 3; w++) tensor_scale(__uint_as_float(p.amax[w]), g[w], inv_g[w]);
    if (blockIdx.x == 0 && threadIdx.x < 3) {
        float* go = threadIdx.x == 0 ? p.qg : (threadIdx.x == 1 ? p.kg : p.vg);
        go[0] = g[threadIdx.x];
        go[1] = inv_g[threadIdx.x];
    }
    for (int it = 0; j < total; it++, j += gridDim.x) {
        const int b = it & 1;
        const bool next = j + (int)gridDim.x < total;
        // buffer b ^ 1 was released by the barrier that ended the previous tile
        if (threadIdx.x == 0 && next) issue(j + gridDim.x, b ^ 1);
        if (__syncthreads_or(!mbar_wait(&s.full[b], (it >> 1) & 1))) {
            if (threadIdx.x == 0) {
                sa_raise(SA_ERR_TIMEOUT);
                if (next) mbar_wait(&s.full[b ^ 1], ((it + 1) >> 1) & 1);  // bounded: the copy in flight
            }
            return;
        }
        int which, bh, tile;
        decode(j, which, bh, tile);
        if (which == 2) {
            for (int i = D + threadIdx.x; i < 128; i += blockDim.x) {  // channel rows D..127 of the atoms
                s.atoms[(i & 31) * 4 + (i >> 5)] = 0u;
                s.atoms[128 + (i & 31) * 4 + (i >> 5)] = 0u;
            }
            quant_v_smem<D, SEARCH>(reinterpret_cast<const uint16_t*>(s.x[b]), bh, tile, p.N, inv_g[2], p.f_lo,
                                    p.f_hi, p.vc, nullptr, s.atoms, s.rcp);
            __syncthreads();
            store_v_atoms(s.atoms, bh, tile, p.N, p.vs);
        } else if (which == 0) {
            quant_rows_smem<D, false, SEARCH>(s.x[b], bh, tile, p.N, nullptr, inv_g[0], p.f_lo, p.f_hi, p.qc, nullptr,
                                              s.atoms, s.rcp);
            __syncthreads();
            store_rows_atoms<D>(s.atoms, bh, tile, p.T, p.qs);
        } else {
            quant_rows_smem<D, SMOOTH, SEARCH>(s.x[b], bh, tile, p.N, p.kmean, inv_g[1], p.f_lo, p.f_hi, p.kc,
                                               nullptr, s.atoms, s.rcp);
            __syncthreads();
            store_rows_atoms<D>(s.atoms, bh, tile, p.T, p.ks);
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
