// select.cuh -- ThriftAttention-style block selector.
//
// "ThriftAttention: 5%의 연산량으로 90%의 품질 유지" (molayo1419.me): a small
// share (about 5 %) of query-key blocks is computed in high precision.  The
// page leaves the selector open; the one used here mean-pools 128-row tiles of
// raw Q and K (bf16 means), scores tile pairs with an FP32 fmaf chain, and keeps
// the top ceil(n_valid * frac / 10000) valid pairs per (b, h), ties broken by
// the lower linear index t*T+u.
//
// Kernels:
//   pool_kernel    thread per channel: FP32 sum over the tile rows in order
//                  (optionally of fl(k - mu_c)), / row count, rounded to bf16
//                  (kept as float).
//   score_kernel   one thread per (t, u): fmaf chain over channels ascending.
//   topk_kernel    one CTA per (b, h): 4-pass 8-bit radix select of the k-th
//                  largest score key, then an index-ordered scan that admits
//                  the needed number of keys equal to the threshold.
//   topk_row_kernel  the same rule per query tile (one warp per row).
#pragma once

#include "common.cuh"

namespace sa {

// Block (32 u) x (8 t); scores for all (t, u) (invalid ones are ignored later).
__global__ void __launch_bounds__(256) score_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
                                                    int D, int T, float* __restrict__ scores)
{
    __shared__ float sq[8][129];
    __shared__ float sk[32][129];
    size_t bh = blockIdx.z;
    int u0 = blockIdx.x * 32, t0 = blockIdx.y * 8;
    for (int i = threadIdx.x; i < 8 * D; i += 256) {
        int r = i / D, c = i % D;
        sq[r][c] = (t0 + r < T) ? qbar[(bh * T + t0 + r) * D + c] : 0.0f;
    }
    for (int i = threadIdx.x; i < 32 * D; i += 256) {
        int r = i / D, c = i % D;
        sk[r][c] = (u0 + r < T) ? kbar[(bh * T + u0 + r) * D + c] : 0.0f;
    }
    __syncthreads();
    int ui = threadIdx.x & 31, ti = threadIdx.x >> 5;
    int t = t0 + ti, u = u0 + ui;
    float acc = 0.0f;
    for (int c = 0; c < D; c++) acc = __fmaf_rn(sq[ti][c], sk[ui][c], acc);
    if (t < T && u < T) scores[(bh * T + t) * T + u] = acc;
}

// Order-preserving key of a finite score (larger score -> larger key);
// -0 is first turned into +0 so equal scores compare equal.
SA_DEV uint32_t score_key(float s)
{
    uint32_t u = __float_as_uint(__fadd_rn(s, 0.0f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTopkThreads = 1024;

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int T, int causal,
                                                            int frac_bp, uint8_t* __restrict__ mask,
                                                            int32_t* __restrict__ nsel)
{
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_prefix, s_need;
    __shared__ uint32_t scan[kTopkThreads];
    size_t bh = blockIdx.x;
    const float* sc = scores + bh * (size_t)T * T;
    uint8_t* mk = mask + bh * (size_t)T * T;
    const int total = T * T;
    long long nvalid = causal ? (long long)T * (T + 1) / 2 : (long long)T * T;
    uint32_t ksel = (uint32_t)((nvalid * frac_bp + 9999) / 10000);
    if (threadIdx.x == 0) {
        s_prefix = 0;
        s_need = ksel;
        if (nsel) nsel[bh] = (int32_t)ksel;
    }
    // radix select over the key bits, most significant byte first: find the
    // key value of the ksel-th largest valid element.
    uint32_t prefix_mask = 0;
    for (int pass = 0; pass < 4; pass++) {
        int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        uint32_t prefix = s_prefix;
        if (s_need > 0) {
            for (int i = threadIdx.x; i < total; i += blockDim.x) {
                int t = i / T, u = i % T;
                if (causal && u > t) continue;
                uint32_t key = score_key(sc[i]);
                if ((key & prefix_mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t need = s_need, acc = 0;
            int d = 255;
            if (need > 0) {
                for (; d >= 0; d--) {
                    if (acc + hist[d] >= need) break;
                    acc += hist[d];
                }
                s_need = need - acc;
                s_prefix = prefix | ((uint32_t)d << shift);
            }
        }
        prefix_mask |= 255u << shift;
        __syncthreads();
    }
    uint32_t thr = s_prefix;       // key of the ksel-th largest
    uint32_t need_eq = s_need;     // how many keys equal to thr to admit
    bool any = ksel > 0;
    // index-ordered admission of ties: each thread owns a contiguous range
    int per = (total + blockDim.x - 1) / blockDim.x;
    int lo = threadIdx.x * per, hi = min(total, lo + per);
    uint32_t cnt = 0;
    if (any)
        for (int i = lo; i < hi; i++) {
            int t = i / T, u = i % T;
            if (causal && u > t) continue;
            cnt += score_key(sc[i]) == thr;
        }
    scan[threadIdx.x] = cnt;
    __syncthreads();
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
        uint32_t v = threadIdx.x >= (unsigned)o ? scan[threadIdx.x - o] : 0u;
        __syncthreads();
        scan[threadIdx.x] += v;
        __syncthreads();
    }
    uint32_t before = scan[threadIdx.x] - cnt;
    for (int i = lo; i < hi; i++) {
        int t = i / T, u = i % T;
        uint8_t m = 0;
        if (any && !(causal && u > t)) {
            uint32_t key = score_key(sc[i]);
            if (key > thr) {
                m = 1;
            } else if (key == thr) {
                m = before < need_eq;
                before++;
            }
        }
        mk[i] = m;
    }
}

static size_t select_ws_bytes(int B, int H, int N, int D)
{
    size_t BH = (size_t)B * H, T = (size_t)sa_cdiv(N, 128);
    return 2 * sa_align256(BH * T * D * sizeof(float)) + sa_align256(BH * T * T * sizeof(float));
}


// ---------------------------------------------------------------------------
// Selector variants ("ThriftAttention" leaves the selector open; these are two
// further readings of it):
//   - per_row: query tile t keeps ceil(n_valid_t * frac / 10000) of its valid
//     key tiles, highest score first, the lower key tile on a tie;
//   - k_mean: key tiles are pooled from fl(k - mu_c), the smoothed keys.
// ---------------------------------------------------------------------------


// pool_kernel with an optional channel mean subtracted from the K rows
// (FP32 per element, before the FP32 row-ordered sum), as the oracle pools.
__global__ void __launch_bounds__(128) pool_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                      const float* __restrict__ k_mean, int N, int D, int T,
                                                      float* __restrict__ qbar, float* __restrict__ kbar)
{
    int t = blockIdx.x;
    size_t bh = blockIdx.y;
    const bool is_k = blockIdx.z != 0;
    const uint16_t* src = is_k ? k : q;
    float* dst = is_k ? kbar : qbar;
    int c = threadIdx.x;
    if (c >= D) return;
    const float mu = (is_k && k_mean) ? k_mean[bh * D + c] : 0.0f;
    const bool sub = is_k && k_mean;
    int r0 = t * 128, r1 = min(N, r0 + 128);
    const uint16_t* p = src + (bh * N) * D + c;
    float acc = 0.0f;
#pragma unroll 8
    for (int r = r0; r < r1; r++) {
        float v = bf16_bits_to_f32(__ldcs(p + (size_t)r * D));
        if (sub) v = __fsub_rn(v, mu);
        acc = __fadd_rn(acc, v);
    }
    float mean = __fdiv_rn(acc, (float)(r1 - r0));
    dst[(bh * T + t) * D + c] = __bfloat162float(__float2bfloat16_rn(mean));
}

constexpr int kRowWarps = 8;  // rows (query tiles) per CTA, one warp each

// Per-row top-k: one warp per (b,h, query tile t).  A 4-pass 8-bit radix
// select over the order-preserving score keys finds the key of the k_t-th
// largest valid score; keys above it are admitted, and keys equal to it in
// ascending key-tile order until k_t.  nsel[bh] (zeroed by the caller)
// receives the sum of the rows' budgets.
__global__ void __launch_bounds__(32 * kRowWarps) topk_row_kernel(const float* __restrict__ scores, int BH, int T,
                                                                  int causal, int frac_bp,
                                                                  uint8_t* __restrict__ mask,
                                                                  int32_t* __restrict__ nsel)
{
    __shared__ uint32_t hist_all[kRowWarps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * kRowWarps + warp;
    if (row >= (long)BH * T) return;  // whole warps only
    const size_t bh = (size_t)(row / T);
    const int t = (int)(row % T);
    const float* sc = scores + (bh * T + t) * (size_t)T;
    uint8_t* mk = mask + (bh * T + t) * (size_t)T;
    const int nv = causal ? t + 1 : T;
    const uint32_t k = (uint32_t)(((long long)nv * frac_bp + 9999) / 10000);
    uint32_t* hist = hist_all[warp];
    uint32_t prefix = 0, pmask = 0, need = k;
    for (int pass = 0; pass < 4; pass++) {
        const int shift = 24 - 8 * pass;
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        if (need > 0)
            for (int u = lane; u < nv; u += 32) {
                const uint32_t key = score_key(sc[u]);
                if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
        __syncwarp();
        uint32_t d_sel = 0, acc_sel = 0;
        if (lane == 0 && need > 0) {
            uint32_t acc = 0;
            int d = 255;
            for (; d > 0; d--) {
                if (acc + hist[d] >= need) break;
                acc += hist[d];
            }
            d_sel = (uint32_t)d;
            acc_sel = acc;
        }
        d_sel = __shfl_sync(0xffffffffu, d_sel, 0);
        acc_sel = __shfl_sync(0xffffffffu, acc_sel, 0);
        if (need > 0) {
            need -= acc_sel;
            prefix |= d_sel << shift;
        }
        pmask |= 255u << shift;
        __syncwarp();  // the histogram is rewritten by the next pass
    }
    const uint32_t thr = prefix, need_eq = need;
    uint32_t eq_before = 0;
    for (int u0 = 0; u0 < T; u0 += 32) {
        const int u = u0 + lane;
        const bool valid = k > 0 && u < nv;
        const uint32_t key = valid ? score_key(sc[u]) : 0u;
        const bool gt = valid && key > thr, eq = valid && key == thr;
        const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
        const uint32_t rank = eq_before + __popc(eqm & ((1u << lane) - 1u));
        if (u < T) mk[u] = (uint8_t)(gt || (eq && rank < need_eq));
        eq_before += __popc(eqm);
    }
    if (lane == 0 && nsel) atomicAdd(&nsel[bh], (int)k);
}

}  // namespace sa
