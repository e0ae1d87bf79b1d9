// decode.cuh -- one query token per sequence over an NVFP4 KV cache.
//
// "Search Your Block Floating Point Scales!" (gist.science summary),
// "ScaleSearchAttention": the KV cache is kept in 4-bit NVFP4 and attention
// runs on FP4 tensor cores.  Grouped-query heads: query head h reads kv head
// h / G, G = Hq / Hkv.
//
// One CTA per (b, kv head, split of 4096 keys).  The G query heads of the
// group form the N side of a swapped MMA so the 128 keys of a tile fill the
// M = 128 side:
//   S^T[128 keys, 8] = K_tile (A, TMA, scale atoms) x q^T (B, G rows + zero rows)
//   per head (column): running max over keys (shuffles + shared memory),
//   P~ = exp2(S c - m), per 16 keys (16 lanes) scale E4M3(max p/6), E2M1 codes
//   -> P^T (B operand: 8 rows x 128 keys, 64-byte swizzle) + scale atom
//   O^T[D, 8] += V^T_tile (A) x P^T; the row sums l add up the dequantised
//   P (code x scale) of each head on the CUDA cores (warp shuffles, then the
//   four warps in a fixed order), rescaled with the same running max as O.
// q is quantised in the kernel with the tensor-wide g from a preceding amax
// pass (same block rule as the pre-pass: 16 channels, max-scaling).
// Each split writes (m, l, O) unnormalised; decode_combine_kernel merges the
// splits exactly: O = sum_s 2^(m_s-M) O_s / sum_s 2^(m_s-M) l_s.
//
// Attention-sink-aware mixed-precision cache (same page, "ScaleSearchAttention":
// the first and last blocks of the cache stay at full precision): with SINK,
// the first sink_first and the last sink_last 128-key tiles of the cache come
// from a compact bf16 copy of just those tiles and take the mixed-block
// arithmetic inside the same online softmax: scores of raw bf16 q against raw
// bf16 k minus its channel mean, P~ rounded to bf16, raw bf16 V.  These tiles
// are a few per cache and their MMA shape (128 keys x G heads) is mostly
// padding, so they run on the CUDA cores with FP32 accumulation, reading K and
// V straight from global memory; the kernel keeps the plain decode's shared
// memory (and occupancy).  Their P·V adds into the TMEM accumulator in its
// NVFP4 units: O += (2688 P_b) (V / g_V), l += 2688 P_b.
#pragma once

#include <cstddef>

#include "attn.cuh"
#include "quant.cuh"

namespace sa {

// E2M1 code (low nibble) of one float: one conversion, round to nearest
// even, saturating, sign kept.
SA_DEV uint32_t e2m1_code1(float y)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0;\n\t.reg .b16 h;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %1, %2;\n\t"
        "mov.b16 h, {b0, b0};\n\t"
        "cvt.u32.u16 %0, h;\n\t}"
        : "=r"(out)
        : "f"(0.0f), "f"(y));
    return out & 15u;
}

constexpr int kSplit = 4096;
constexpr int kDecN = 8;  // MMA N (query heads of a group, zero-padded)

template <int D>
struct DecSmem {
    alignas(1024) uint8_t k[128 * D / 2];    // K tile (A), D/2-byte swizzle
    alignas(1024) uint8_t v[128 * 64];       // V^T tile (A): 128 rows (rows >= D stay zero), 64-byte swizzle
    alignas(1024) uint8_t q[kDecN * D / 2];  // q^T (B): 8 rows, D/2-byte swizzle
    alignas(1024) uint8_t p[kDecN * 64];     // P^T (B): 8 rows x 128 keys, 64-byte swizzle
    uint8_t ksf[D / 64 * 512];
    uint8_t vsf[2 * 512];
    alignas(16) uint8_t qsf[D / 64 * 512];
    uint8_t psf[2 * 512];
    alignas(16) uint16_t pb16[kDecN * 128];  // bf16 P of a full-precision tile, [head][key]
    float rcp[128];    // reciprocals of the E4M3 scale values
    float lg2sc[128];  // log2 of each nonzero E4M3 scale value
    float lred[4][kDecN];  // per-warp partial sums of the dequantised P
    float lrun[kDecN];     // running l per column (query head)
    float red[4][kDecN];
    float mnew[kDecN];
    float alpha[kDecN];
    uint64_t k_bar;  // K tile + K scale atoms landed
    uint64_t v_bar;  // V tile + V scale atoms landed
    uint64_t mma_bar;
    uint32_t tmem_slot;
};

// A full-precision tile stages 128 D bytes across the K stage and the start of
// the V stage, which must be adjacent.
static_assert(offsetof(DecSmem<128>, v) == 128 * 128 / 2 && offsetof(DecSmem<64>, v) == 128 * 64 / 2,
              "K and V stages are adjacent");
// ... and keeps the group's raw q (G <= 8 rows of D bf16) and the K channel means
// (D floats) in the bytes of the NVFP4 tile's P and K / V scale atoms, adjacent too.
template <int D>
constexpr bool dec_scratch_fits()
{
    return offsetof(DecSmem<D>, ksf) == offsetof(DecSmem<D>, p) + sizeof(DecSmem<D>::p) &&
           offsetof(DecSmem<D>, vsf) == offsetof(DecSmem<D>, ksf) + sizeof(DecSmem<D>::ksf) &&
           sizeof(DecSmem<D>::p) + sizeof(DecSmem<D>::ksf) + sizeof(DecSmem<D>::vsf) >= kDecN * D * 2 + D * 4;
}
static_assert(dec_scratch_fits<128>() && dec_scratch_fits<64>(), "raw q and K means fit the NVFP4 tile's scratch");

// TMEM columns (64 allocated)
constexpr uint32_t DM_S = 0, DM_O = 8, DM_SFK = 24, DM_SFQ = 32, DM_SFV = 40, DM_SFP = 48;

struct DecParams {
    const uint16_t* q;  // bf16 [B, Hq, D]
    const unsigned* q_amax;
    const uint8_t* k_sf;
    const uint8_t* v_sf;
    const float* k_g;
    const float* v_g;
    float* part;  // [B*Hq, nsplit, D + 2]: O (D), l, m
    int L, Hq, Hkv, G, nsplit, RTk, CKv;
    float sm_scale;
    // full-precision tiles (SINK): bf16 [B, Hkv, NS, D], NS = 128 (sink_first + sink_last),
    // the first tiles then the last ones; k_mean [B, Hkv, D] (nullptr: K not smoothed)
    const uint16_t* k_sink;
    const uint16_t* v_sink;
    const float* k_mean;
    int sink_first, sink_last, NS;
};

// Full-precision tiles go through shared memory in halves of 64 keys (128 D
// bytes: the K stage and the first bytes of the V stage, which that tile does
// not use; rows D.. of the V stage, zero for D = 64, stay untouched), by
// 16-byte cp.async copies.  K rows are stored with their 16-byte chunks
// swizzled by the row (chunk c at c ^ (row mod D/8)) so that the score loop
// below reads without bank conflicts; V rows are stored plain.
template <int D>
SA_DEV void dec_stage_half(uint8_t* stage, const uint16_t* src, bool swz)
{
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    const int tid = threadIdx.x;
#pragma unroll
    for (int j = 0; j < 64 * CPR / 128; j++) {
        const int idx = tid + 128 * j, row = idx / CPR, c = idx % CPR;
        const int pc = swz ? (c ^ (row & (CPR - 1))) : c;
        cp_async16(smem_u32(stage + row * (2 * D) + pc * 16), src + (size_t)row * D + c * 8);
    }
    cp_async_commit();
}

// Scores of one staged half: threads 2k and 2k + 1 take key k's two halves of
// the channels, sv = q.(k - mu) per head (h < G; padding heads 0), summed
// over the pair so both hold the key's score.
template <int D>
SA_DEV void dec_sink_half_scores(const uint8_t* stage, const DecParams& p, const uint16_t* qs, const float* mu,
                                 float (&sv)[kDecN])
{
    constexpr int CPR = D / 8, PC = CPR / 2;
    const int tid = threadIdx.x, kk = tid >> 1, part = tid & 1;
#pragma unroll
    for (int h = 0; h < kDecN; h++) sv[h] = 0.0f;
#pragma unroll 1
    for (int i = 0; i < PC; i++) {
        const int c = part * PC + i;
        const uint4 kr = *reinterpret_cast<const uint4*>(stage + kk * (2 * D) + ((c ^ (kk & (CPR - 1))) * 16));
        const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            kf[2 * e] = __uint_as_float(kw[e] << 16);
            kf[2 * e + 1] = __uint_as_float(kw[e] & 0xFFFF0000u);
        }
        if (mu) {
            const float4 m0 = *reinterpret_cast<const float4*>(mu + 8 * c);
            const float4 m1 = *reinterpret_cast<const float4*>(mu + 8 * c + 4);
            kf[0] -= m0.x, kf[1] -= m0.y, kf[2] -= m0.z, kf[3] -= m0.w;
            kf[4] -= m1.x, kf[5] -= m1.y, kf[6] -= m1.z, kf[7] -= m1.w;
        }
#pragma unroll
        for (int h = 0; h < kDecN; h++) {
            if (h >= p.G) break;
            const uint4 qr = *reinterpret_cast<const uint4*>(qs + h * D + 8 * c);
            const uint32_t qw[4] = {qr.x, qr.y, qr.z, qr.w};
            float a = sv[h];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                a = fmaf(__uint_as_float(qw[e] << 16), kf[2 * e], a);
                a = fmaf(__uint_as_float(qw[e] & 0xFFFF0000u), kf[2 * e + 1], a);
            }
            sv[h] = a;
        }
    }
#pragma unroll
    for (int h = 0; h < kDecN; h++) sv[h] += __shfl_xor_sync(0xffffffffu, sv[h], 1);
}

// P.V of one staged V half for channel d = tid (d < D): acc[h] += sum over its
// 64 keys of P_b[h][key0 + key] V[key][d]; P_b from its bf16 bits.
template <int D>
SA_DEV void dec_sink_half_pv(const uint8_t* stage, const uint16_t* pb, int key0, const DecParams& p,
                             float (&acc)[kDecN])
{
    const int tid = threadIdx.x;
    if (tid >= D) return;
    const uint16_t* vcol = reinterpret_cast<const uint16_t*>(stage) + tid;
#pragma unroll 1
    for (int k0 = 0; k0 < 64; k0 += 8) {
        float vv[8];
#pragma unroll
        for (int i = 0; i < 8; i++) vv[i] = __uint_as_float((uint32_t)vcol[(k0 + i) * D] << 16);
#pragma unroll
        for (int h = 0; h < kDecN; h++) {
            if (h >= p.G) break;
            const uint4 pw = *reinterpret_cast<const uint4*>(pb + h * 128 + key0 + k0);  // broadcast
            const uint32_t w[4] = {pw.x, pw.y, pw.z, pw.w};
            float a = acc[h];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                a = fmaf(__uint_as_float(w[e] << 16), vv[2 * e], a);
                a = fmaf(__uint_as_float(w[e] & 0xFFFF0000u), vv[2 * e + 1], a);
            }
            acc[h] = a;
        }
    }
}

// Running max per column (query head) after one tile: max over the 128 keys
// of sv * c (columns past the group's G heads are padding and keep m = 0,
// alpha = 1).  Returns the new max m2 and the rescale factor alpha per column.
template <int D>
SA_DEV void dec_running_max(DecSmem<D>& s, const DecParams& p, const float (&sv)[kDecN], float c,
                            float (&m2)[kDecN], float (&alpha)[kDecN])
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int h = 0; h < kDecN; h++) {
        if (h >= p.G) break;
        float mx = sv[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) s.red[warp][h] = mx;
    }
    __syncthreads();
    if (tid < p.G) {
        const float tmax = fmaxf(fmaxf(s.red[0][tid], s.red[1][tid]), fmaxf(s.red[2][tid], s.red[3][tid]));
        const float mo = s.mnew[tid];  // the running max (-inf before the first tile)
        const float mn = fmaxf(mo, tmax * c);
        s.mnew[tid] = mn;
        s.alpha[tid] = ex2f(mo - mn);
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kDecN; h++) {
        m2[h] = s.mnew[h];
        alpha[h] = s.alpha[h];
    }
}

// l = alpha l + the tile's per-warp sums of P (warps in a fixed order).
template <int D>
SA_DEV void dec_l_update(DecSmem<D>& s, const DecParams& p, int u)
{
    const int tid = threadIdx.x;
    if (tid < p.G) {
        const float t = (s.lred[0][tid] + s.lred[1][tid]) + (s.lred[2][tid] + s.lred[3][tid]);
        s.lrun[tid] = (u > 0 ? s.lrun[tid] * s.alpha[tid] : 0.0f) + t;
    }
}

// One full-precision cache tile (rows srow.. of the compact bf16 copy): the
// scores of both key halves, the running max, P_b = bf16(2^(t c - m)) into
// shared memory (bf16 bits, exact), P.V on the CUDA cores in FP32, then
// O^T = alpha O^T + kappa acc in TMEM (kappa = 2688 / g_V, the accumulator's
// NVFP4 units) and l += 2688 P_b.  The first V half is copied while the max
// and P are formed.
template <int D>
SA_DEV bool dec_sink_tile(DecSmem<D>& s, const DecParams& p, int b, int hk, int srow, int u, float c,
                          uint32_t tbase, uint32_t lane_off)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t kv = (size_t)b * p.Hkv + hk;
    const uint16_t* ks = p.k_sink + (kv * p.NS + srow) * D;
    const uint16_t* vs = p.v_sink + (kv * p.NS + srow) * D;
    const uint16_t* qg = p.q + ((size_t)b * p.Hq + (size_t)hk * p.G) * D;
    const float* mug = p.k_mean ? p.k_mean + kv * D : nullptr;
    uint8_t* stage = s.k;
    // the group's raw q rows and the K means, copied with the first K half
    uint16_t* qs = reinterpret_cast<uint16_t*>(s.p);
    float* mu = mug ? reinterpret_cast<float*>(s.p + kDecN * D * 2) : nullptr;
    if (tid < p.G * D / 8) cp_async16(smem_u32(qs + 8 * tid), qg + 8 * tid);
    if (mug && tid < D / 4) cp_async16(smem_u32(mu + 4 * tid), mug + 4 * tid);
    {  // scores, running max and P (alpha is re-read from shared memory below)
    float sa[kDecN], sb[kDecN];
    dec_stage_half<D>(stage, ks, true);
    cp_async_wait_all();
    __syncthreads();
    dec_sink_half_scores<D>(stage, p, qs, mu, sa);
    __syncthreads();
    dec_stage_half<D>(stage, ks + 64 * D, true);
    cp_async_wait_all();
    __syncthreads();
    dec_sink_half_scores<D>(stage, p, qs, mu, sb);
    __syncthreads();
    dec_stage_half<D>(stage, vs, false);  // lands while the max and P are formed
    float mx[kDecN], m2[kDecN], alpha[kDecN];
#pragma unroll
    for (int h = 0; h < kDecN; h++) mx[h] = fmaxf(sa[h], sb[h]);
    dec_running_max(s, p, mx, c, m2, alpha);
    const int kk = tid >> 1;
    const bool lead = (tid & 1) == 0;  // the even thread of a key pair writes its P
#pragma unroll
    for (int h = 0; h < kDecN; h++) {
        if (h >= p.G) break;
        const __nv_bfloat16 pa = __float2bfloat16_rn(ex2f(fmaf(sa[h], c, -m2[h])));
        const __nv_bfloat16 pb = __float2bfloat16_rn(ex2f(fmaf(sb[h], c, -m2[h])));
        if (lead) {
            s.pb16[h * 128 + kk] = __bfloat16_as_ushort(pa);
            s.pb16[h * 128 + 64 + kk] = __bfloat16_as_ushort(pb);
        }
        // each P_b times 2688 is exact (8 significant bits times 21 * 2^7)
        float pv = lead ? __bfloat162float(pa) * 2688.0f + __bfloat162float(pb) * 2688.0f : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pv += __shfl_xor_sync(0xffffffffu, pv, o);
        if (lane == 0) s.lred[warp][h] = pv;
    }
    }
    cp_async_wait_all();
    __syncthreads();
    float acc[kDecN];
#pragma unroll
    for (int h = 0; h < kDecN; h++) acc[h] = 0.0f;
    dec_sink_half_pv<D>(stage, s.pb16, 0, p, acc);
    __syncthreads();
    dec_stage_half<D>(stage, vs + 64 * D, false);
    cp_async_wait_all();
    __syncthreads();
    dec_sink_half_pv<D>(stage, s.pb16, 64, p, acc);
    const float kappa = 2688.0f / p.v_g[0];
    uint32_t r[kDecN];
    if (u > 0)
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
            "tcgen05.wait::ld.sync.aligned;"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
            : "r"(tbase + lane_off + DM_O)
            : "memory");
#pragma unroll
    for (int h = 0; h < kDecN; h++) {
        const float o = u > 0 ? __uint_as_float(r[h]) * s.alpha[h] : 0.0f;
        r[h] = __float_as_uint(fmaf(acc[h], kappa, o));
    }
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(tbase + lane_off + DM_O),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
    fence_proxy_async();  // the staged and scratch bytes go back to the tensor copies
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    dec_l_update(s, p, u);
    return true;
}

template <int D, bool SINK>
SA_DEV bool decode_body(DecSmem<D>& s, const CUtensorMap* tm_k, const CUtensorMap* tm_v, const DecParams& p,
                        int b, int hk, int split, uint32_t tbase)
{
    constexpr int KB = D / 64;
    constexpr uint32_t KSW = D == 128 ? 4u : 6u;
    constexpr uint32_t KSBO = 8 * D / 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int bhk = b * p.Hkv + hk;

    const int key0 = split * kSplit;
    const int nkeys = min(kSplit, p.L - key0);
    const int ntiles = nkeys / 128;
    const float c_sink = p.sm_scale * kLog2e;  // full-precision tiles: t = q.(k - mu) sm_scale log2(e)
    // Row of tile u in the compact full-precision copy, or -1 for an NVFP4 tile.
    auto sink_row = [&](int u) -> int {
        if constexpr (SINK) {
            const int kt = key0 / 128 + u;
            if (kt < p.sink_first) return kt * 128;
            if (kt >= p.RTk - p.sink_last) return (p.sink_first + kt - (p.RTk - p.sink_last)) * 128;
        }
        return -1;
    };
    // The K stage (with its scale atoms) and the V stage are loaded separately:
    // the next tile's K as soon as this tile's Q K^T has read the K stage, its
    // V as soon as this tile's P V has read the V stage, so each copy overlaps
    // the rest of the tile (no extra shared memory).
    auto load_k = [&](int kt) {
        mbar_expect_tx(&s.k_bar, 128 * D / 2 + KB * 512);
        tma_load_3d(s.k, tm_k, &s.k_bar, 0, kt * 128, bhk);
        bulk_load(s.ksf, p.k_sf + ((size_t)bhk * p.RTk + kt) * KB * 512, KB * 512, &s.k_bar);
    };
    auto load_v = [&](int kt) {
        mbar_expect_tx(&s.v_bar, D * 64 + 2 * 512);
        tma_load_3d(s.v, tm_v, &s.v_bar, 0, kt * D, bhk);
        bulk_load(s.vsf, p.v_sf + ((size_t)bhk * p.CKv + 2 * kt) * 512, 2 * 512, &s.v_bar);
    };
    bool kin = false, vin = false;  // this tile's K / V copies already issued (prefetched)
    // the first tile's copies go out before q is quantised (they do not depend on it)
    if (sink_row(0) < 0) {
        if (tid == 0) {
            load_k(key0 / 128);
            load_v(key0 / 128);
        }
        kin = vin = true;
    }

    // full-precision tiles of this split: start their K and V on the way to L2
    // now, ahead of their turn in the key loop
    if constexpr (SINK) {
        if (tid < 2) {
            const int t0 = split * (kSplit / 128), t1 = min(t0 + kSplit / 128, p.RTk);
            for (int kt = t0; kt < t1; kt++) {
                int sr = -1;
                if (kt < p.sink_first)
                    sr = kt * 128;
                else if (kt >= p.RTk - p.sink_last)
                    sr = (p.sink_first + kt - (p.RTk - p.sink_last)) * 128;
                if (sr < 0) continue;
                const uint16_t* base = (tid ? p.v_sink : p.k_sink) + ((size_t)(b * p.Hkv + hk) * p.NS + sr) * D;
                bulk_prefetch_l2(base, 128 * D * 2);
            }
        }
    }
    // ---- quantise the group's query rows (q^T operand + its scale atom)
    {
        float g, inv_g;
        tensor_scale(__uint_as_float(*p.q_amax), g, inv_g);
        fill_rcp_table(s.rcp);
        for (int e = tid; e < kDecN * D / 2; e += blockDim.x) s.q[e] = 0;
        for (int e = tid; e < KB * 512; e += blockDim.x) s.qsf[e] = 0;
        __syncthreads();
        const int nblk = p.G * (D / 16);
        if (tid < nblk) {
            const int hi = tid / (D / 16), j = tid % (D / 16);
            const uint16_t* src = p.q + ((size_t)b * p.Hq + hk * p.G + hi) * D + j * 16;
            float xt[16];
#pragma unroll
            for (int i = 0; i < 16; i++) xt[i] = __fmul_rn(bf16_bits_to_f32(src[i]), inv_g);
            uint32_t c0, c1, sc;
            int off;
            quant16<false>(xt, 0, 1, c0, c1, sc, off, s.rcp);
            // row hi, bytes 8j..8j+7 of a (D/2)-byte row, swizzled in 16-byte chunks
            const int byte = 8 * j;
            const int chunk = byte >> 4;
            const int sw = D == 128 ? (chunk ^ ((hi & 7) >> 1)) : (chunk ^ ((hi & 7) >> 2));
            *reinterpret_cast<uint2*>(s.q + hi * (D / 2) + sw * 16 + (byte & 15)) = make_uint2(c0, c1);
            s.qsf[(j >> 2) * 512 + sf_atom_offset((uint32_t)hi, (uint32_t)(j & 3))] = (uint8_t)sc;
        }
    }
    float gq, inv_gq;
    tensor_scale(__uint_as_float(*p.q_amax), gq, inv_gq);
    const float cexp = gq * p.k_g[0] * p.sm_scale * kLog2e;
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    uint32_t kph = 0, vph = 0, mma_phase = 0;
    if (tid == 0) {
        tc_fence_after();
        for (int kb = 0; kb < KB; kb++) tc_cp_sf(tbase + DM_SFQ + 4 * kb, smem_u32(s.qsf + 512 * kb));
    }

    if (tid < kDecN) {  // read after the first tile's barriers; padding columns stay at alpha 1
        s.mnew[tid] = tid < p.G ? -INFINITY : 0.0f;
        s.alpha[tid] = 1.0f;
    }
    // before giving up, let the copies in flight land (bounded) so none writes
    // shared memory after the CTA has left
    auto drain = [&]() {
        if (tid == 0) {
            if (kin) mbar_wait(&s.k_bar, kph);
            if (vin) mbar_wait(&s.v_bar, vph);
        }
        return false;
    };
    for (int u = 0; u < ntiles; u++) {
        const int ktile = key0 / 128 + u;
        const int srow = sink_row(u);
        if (srow >= 0) {  // full-precision tile (no copy in flight: none is prefetched for it)
            if (!dec_sink_tile<D>(s, p, b, hk, srow, u, c_sink, tbase, lane_off)) return false;
            continue;
        }
        // prefetch the next tile when it is NVFP4 (not in the kernel with full-precision
        // tiles, whose register budget it would overrun)
        const bool next = !SINK && u + 1 < ntiles;
        if (tid == 0) {
            if (!kin) load_k(ktile);
            if (!vin) load_v(ktile);
        }
        kin = vin = true;
        if (__syncthreads_or(!mbar_wait(&s.k_bar, kph))) return drain();
        kph ^= 1;
        kin = false;
        if (tid == 0) {
            tc_fence_after();
            for (int kb = 0; kb < KB; kb++) tc_cp_sf(tbase + DM_SFK + 4 * kb, smem_u32(s.ksf + 512 * kb));
            for (int kb = 0; kb < KB; kb++)
                mma_fp4(tbase + DM_S, make_sdesc(smem_u32(s.k) + 32 * kb, KSBO, 16, KSW),
                        make_sdesc(smem_u32(s.q) + 32 * kb, KSBO, 16, KSW), idesc_fp4(128, kDecN),
                        tbase + DM_SFK + 4 * kb, tbase + DM_SFQ + 4 * kb, kb > 0);
            tc_commit(&s.mma_bar);
        }
        if (__syncthreads_or(!mbar_wait(&s.mma_bar, mma_phase))) return drain();
        mma_phase ^= 1;
        tc_fence_after();
        if (next) {  // the K stage is free: the next tile's K lands during this one
            if (tid == 0) load_k(ktile + 1);
            kin = true;
        }

        // ---- scores of this thread's key for the 8 columns
        float sv[kDecN];
        {
            uint32_t r[kDecN];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
                "tcgen05.wait::ld.sync.aligned;"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                : "r"(tbase + lane_off + DM_S)
                : "memory");
#pragma unroll
            for (int h = 0; h < kDecN; h++) sv[h] = __uint_as_float(r[h]);
        }
        float alpha[kDecN];
        float m2[kDecN];
        dec_running_max(s, p, sv, cexp, m2, alpha);
        // P^T codes and scales: block of 16 keys = 16 lanes
#pragma unroll
        for (int h = 0; h < kDecN; h++) {
            if (h >= p.G) break;  // padding columns keep P = 0 (their O columns are not read)
            const float x = fmaf(sv[h], cexp, kLog2_2688 - m2[h]);
            float bm = x;
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            const uint32_t sc = f32_to_e4m3(ex2f(bm) * (1.0f / 6.0f));
            const float y = sc ? ex2f(x - s.lg2sc[sc]) : 0.0f;
            const uint32_t code = e2m1_code1(y);
            // this key's dequantised P (in units of 1/2688), summed over the tile's keys
            float pv = e2m1_to_f32(code) * e4m3_to_f32(sc);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) pv += __shfl_xor_sync(0xffffffffu, pv, o);
            if (lane == 0) s.lred[warp][h] = pv;
            const uint32_t hi_code = __shfl_down_sync(0xffffffffu, code, 1);
            if ((lane & 1) == 0) {
                const int byte = tid >> 1;        // key pair index within the 128 keys
                const int chunk = byte >> 4;
                const int sw = chunk ^ ((h & 7) >> 1);
                s.p[h * 64 + sw * 16 + (byte & 15)] = (uint8_t)(code | (hi_code << 4));
            }
            if ((lane & 15) == 0) {
                const int blk = tid >> 4;  // 0..7 over the 128 keys
                s.psf[(blk >> 2) * 512 + sf_atom_offset((uint32_t)h, (uint32_t)(blk & 3))] = (uint8_t)sc;
            }
        }
        // rescale O^T and L columns whose head max moved
        bool any = false;
#pragma unroll
        for (int h = 0; h < kDecN; h++) any |= alpha[h] != 1.0f;
        if (u > 0 && any) {
            uint32_t r[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
                "%14, %15}, [%16];\n\t"
                "tcgen05.wait::ld.sync.aligned;"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                  "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                  "=r"(r[15])
                : "r"(tbase + lane_off + DM_O)
                : "memory");
#pragma unroll
            for (int i = 0; i < 16; i++) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha[i & 7]);
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                "%13, %14, %15, %16};\n\t"
                "tcgen05.wait::st.sync.aligned;" ::"r"(tbase + lane_off + DM_O),
                "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
                "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
                : "memory");
        }
        fence_proxy_async();
        tc_fence_before();
        if (__syncthreads_or(!mbar_wait(&s.v_bar, vph))) return drain();  // this tile's V has landed
        vph ^= 1;
        vin = false;
        dec_l_update(s, p, u);
        if (tid == 0) {
            tc_fence_after();
            for (int kb = 0; kb < 2; kb++) tc_cp_sf(tbase + DM_SFV + 4 * kb, smem_u32(s.vsf + 512 * kb));
            for (int kb = 0; kb < 2; kb++) tc_cp_sf(tbase + DM_SFP + 4 * kb, smem_u32(s.psf + 512 * kb));
            for (int kb = 0; kb < 2; kb++) {
                const uint64_t pd = make_sdesc(smem_u32(s.p) + 32 * kb, 512, 16, 4);
                const uint32_t acc = (u > 0 || kb > 0) ? 1u : 0u;
                mma_fp4(tbase + DM_O, make_sdesc(smem_u32(s.v) + 32 * kb, 512, 16, 4), pd, idesc_fp4(128, kDecN),
                        tbase + DM_SFV + 4 * kb, tbase + DM_SFP + 4 * kb, acc);
            }
            tc_commit(&s.mma_bar);
        }
        if (__syncthreads_or(!mbar_wait(&s.mma_bar, mma_phase))) return drain();
        mma_phase ^= 1;
        tc_fence_after();
        if (next) {  // the V stage is free: the next tile's V lands during its Q K^T
            if (tid == 0) load_v(ktile + 1);
            vin = true;
        }
    }

    // ---- write this split's unnormalised O (lane = channel), l and m
    uint32_t o[kDecN];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]), "=r"(o[7])
        : "r"(tbase + lane_off + DM_O)
        : "memory");
#pragma unroll
    for (int h = 0; h < kDecN; h++) {  // constant indices keep o in registers
        if (h >= p.G) break;
        float* dst = p.part + (((size_t)b * p.Hq + hk * p.G + h) * p.nsplit + split) * (D + 2);
        if (tid < D) dst[tid] = __uint_as_float(o[h]);
        if (tid == 0) {
            dst[D] = s.lrun[h];
            dst[D + 1] = s.mnew[h];
        }
    }
    return true;
}

template <int D, bool SINK>
__global__ void __launch_bounds__(128, 8) decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                     const __grid_constant__ CUtensorMap tm_v, const DecParams p)
{
    extern __shared__ uint8_t smem_raw[];
    DecSmem<D>& s = *reinterpret_cast<DecSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                   ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    if (warp == 0) {
        tmem_alloc(&s.tmem_slot, 64);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&s.k_bar, 1);
        mbar_init(&s.v_bar, 1);
        mbar_init(&s.mma_bar, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (tid < 128) {  // (e - 7) + log2(1 + m/8) for normal bytes, -7 + log2(m/4) for subnormal ones
        const uint32_t e = (uint32_t)tid >> 3, m = (uint32_t)tid & 7u;
        const float sig = e ? log2f(1.0f + m * 0.125f) : log2f(m * 0.25f);
        s.lg2sc[tid] = (e ? (float)((int)e - 7) : -7.0f) + sig;
    }
    for (int i = tid; i < kDecN * 64 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(s.p)[i] = 0u;
    for (int i = tid; i < 2 * 512 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(s.psf)[i] = 0u;
    for (int i = D * 64 / 4 + tid; i < 128 * 64 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(s.v)[i] = 0u;
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s.tmem_slot;
    if (!decode_body<D, SINK>(s, &tm_k, &tm_v, p, b, hk, split, tbase) && tid == 0) sa_raise(SA_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 64);
}

// Merge the splits of one (b, query head): thread per channel.
__global__ void decode_combine_kernel(const float* __restrict__ part, int nsplit, int D, const float* __restrict__ v_g,
                                      float* __restrict__ out)
{
    const size_t bq = blockIdx.x;
    const int d = threadIdx.x;
    const float* pp = part + bq * nsplit * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < nsplit; s++) M = fmaxf(M, pp[s * (D + 2) + D + 1]);
    float num = 0.0f, den = 0.0f;
    for (int s = 0; s < nsplit; s++) {
        const float w = ex2f(pp[s * (D + 2) + D + 1] - M);
        den = fmaf(w, pp[s * (D + 2) + D], den);
        if (d < D) num = fmaf(w, pp[s * (D + 2) + d], num);
    }
    if (d < D) out[bq * D + d] = num / den * v_g[0];
}

}  // namespace sa
