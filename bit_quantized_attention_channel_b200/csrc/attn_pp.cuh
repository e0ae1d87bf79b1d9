// attn_pp.cuh -- NVFP4 attention forward, two query tiles per work item,
// persistent CTAs.
//
// Same mathematics and schedule as attn.cuh ("Search Your Block Floating
// Point Scales!", "ScaleSearchAttention / native NVFP4 execution": Q K^T and
// P V as block-scaled FP4 tensor-core MMAs with FP32 accumulation; online
// softmax over key tiles of 128; P requantised per 16 keys with scale 1/2688).
//
// A work item is (b, h, pair): tile A (query rows 256p..256p+127) and tile B
// (the next 128).  Each K/V tile is loaded once for both.  The grid holds one
// CTA per SM; CTA c takes items c, 2G-1-c, 2G+c, ... of the list ordered
// heaviest causal pair first (a zigzag that evens the per-CTA work).
//   warp 0        TMA producer: Q tiles (double-buffered across items) and
//                 a K/V ring whose stages run on across items.
//   warp 1        MMA issuer (one lane).
//   warps 4..7    softmax of tile A: one thread per query row (TMEM lane).
//   warps 8..11   softmax of tile B.
// The two softmax warpgroups never wait on each other: on each SMSP one warp
// of A and one of B run independently, so the special-function work of one
// overlaps the loads, reductions and TMEM traffic of the other.  Across items
// the next item's loads and first Q K^T proceed while the softmax warps write
// the previous item's output.
//
// TMEM: one S buffer (128 columns) shared by the two tiles and handed back and
// forth: Q_A K_u^T -> A loads S -> Q_B K_u^T -> B loads S -> Q_A K_{u+1}^T ...
// plus [O_x | l_x] for each tile and the scale factors (472 of 512 columns).
// The row sum l accumulates the same dequantised P as O: the V operand of
// P V carries 16 extra rows of E2M1 1.0 (scale 1.0) after row 127, so column
// 128 of [O_x | l_x] is l (for D = 64, rows 64..127 of the operand are zero).
// The softmax warps write P's block scales straight into TMEM.  Every barrier
// phase is counted over the CTA's whole item sequence.
#pragma once

#include "attn.cuh"

namespace sa {

constexpr int kPpStages = 4;
constexpr int kPpThreads = 384;

template <int D>
struct PpSmem {
    alignas(1024) uint8_t q[2][2][128 * D / 2];  // [item % 2][tile]
    alignas(1024) uint8_t k[kPpStages][128 * D / 2];
    alignas(1024) uint8_t v[kPpStages][128 * 64 + 16 * 64];  // V^T (D rows), zero rows to 128, 16 rows of 1.0
    alignas(1024) uint8_t p[2][128 * 64];
    alignas(16) uint8_t qsf[2][2][D / 64 * 512];
    uint8_t ksf[kPpStages][D / 64 * 512];
    uint8_t vsf[kPpStages][2 * 512];
    float lg2sc[128];  // log2 of each nonzero E4M3 scale value: exponent + log2 of the significand
    uint64_t q_full[2];   // [item % 2]: Q tiles and scale atoms landed
    uint64_t q_empty[2];  // [item % 2]: every Q K^T of the item completed
    uint64_t kv_full[kPpStages];
    uint64_t kv_empty[kPpStages];
    uint64_t s_full[2];  // [tile]: S holds this tile's scores
    uint64_t s_free[2];  // [tile]: this tile's warps have read S
    uint64_t p_full[2];
    uint64_t o_done[2];
    uint32_t tmem_slot;
    int abort;
};

// TMEM columns
// TMEM columns: [O_x | l_x] is PP_OW wide at PP_O + PP_OW x (l in column 128);
// SFV: 64-key block kb at + 8 kb (V rows in + 0..3, the 1.0 rows' scale at + 4);
// SFP: tile x at + 8 x, block kb at + 4 kb.
constexpr uint32_t PP_S = 0, PP_O = 128, PP_OW = 144, PP_SFQ = 416, PP_SFK = 432, PP_SFV = 440, PP_SFP = 456;

SA_DEV bool pp_wait(uint64_t* bar, uint32_t parity, volatile int* abort)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > SA_WAIT_CYCLES) {
            *abort = 1;
            sa_raise(SA_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

SA_DEV float pp_max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Maximum of 16 values, three-input max tree (depth 3).
SA_DEV float pp_max16(const float* v)
{
    const float a = pp_max3(v[0], v[1], v[2]), b = pp_max3(v[3], v[4], v[5]), c = pp_max3(v[6], v[7], v[8]);
    const float d = pp_max3(v[9], v[10], v[11]), e = pp_max3(v[12], v[13], v[14]);
    return fmaxf(pp_max3(a, b, c), pp_max3(d, e, v[15]));
}

template <int N>
SA_DEV void pp_setmaxnreg_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
SA_DEV void pp_setmaxnreg_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Work item of the zigzag schedule: round j of this CTA, or -1 past the end.
struct PpItem {
    int bh, pair, nuA, nuB, nu;
    bool hasB;
};

SA_DEV int pp_item_index(int j, int nitems)
{
    const int G = gridDim.x;
    const int c = (j & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x;
    const int i = j * G + c;
    return i < nitems ? i : -1;
}

SA_DEV PpItem pp_item(const AttnParams& p, int i)
{
    const int nbh = p.B * p.H, npairs = (p.T + 1) / 2;
    const int r = i / nbh;
    PpItem it;
    it.bh = i - r * nbh;
    it.pair = p.causal ? npairs - 1 - r : r;  // heaviest causal pairs first
    const int Tk = (p.N + 127) / 128;
    const int tA = 2 * it.pair, tB = tA + 1;
    it.hasB = tB < p.T;
    it.nuA = p.causal ? min(tA + 1, Tk) : Tk;
    it.nuB = it.hasB ? (p.causal ? min(tB + 1, Tk) : Tk) : 0;
    it.nu = max(it.nuA, it.nuB);
    return it;
}

template <int D>
__global__ void __launch_bounds__(kPpThreads, 1) attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                    const __grid_constant__ CUtensorMap tm_k,
                                                                    const __grid_constant__ CUtensorMap tm_v,
                                                                    const AttnParams p)
{
    constexpr int KB = D / 64;
    constexpr uint32_t QSW = D == 128 ? 4u : 6u;
    constexpr uint32_t QSBO = 8 * D / 2;
    extern __shared__ uint8_t smem_raw[];
    PpSmem<D>& s = *reinterpret_cast<PpSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nitems = p.B * p.H * ((p.T + 1) / 2);
    const int nrounds = (nitems + (int)gridDim.x - 1) / (int)gridDim.x;
    volatile int* abort = &s.abort;

    if (warp == 0) {
        tmem_alloc(&s.tmem_slot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        s.abort = 0;
        for (int i = 0; i < 2; i++) {
            mbar_init(&s.q_full[i], 1);
            mbar_init(&s.q_empty[i], 1);
        }
        for (int i = 0; i < kPpStages; i++) {
            mbar_init(&s.kv_full[i], 1);
            mbar_init(&s.kv_empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&s.s_full[i], 1);
            mbar_init(&s.s_free[i], 4);
            mbar_init(&s.p_full[i], 4);
            mbar_init(&s.o_done[i], 1);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (tid < 128) {
        // (e - 7) + log2(1 + m/8) for normal bytes, -7 + log2(m/4) for subnormal ones
        const uint32_t e = (uint32_t)tid >> 3, m = (uint32_t)tid & 7u;
        const float sig = e ? log2f(1.0f + m * 0.125f) : log2f(m * 0.25f);
        s.lg2sc[tid] = (e ? (float)((int)e - 7) : -7.0f) + sig;
    }
    // rows D..127 of every V stage are zero, rows 128..143 are E2M1 1.0
    for (int i = tid; i < kPpStages * (144 - D) * 16; i += blockDim.x) {
        const int st = i / ((144 - D) * 16), w = i % ((144 - D) * 16);
        reinterpret_cast<uint32_t*>(s.v[st] + D * 64)[w] = w >= (128 - D) * 16 ? 0x22222222u : 0u;
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s.tmem_slot;
    if (warp < 4) {
        // scale 1.0 for the 1.0 rows of the V operand (B-operand rows 128..143 of
        // each 64-key block read column base + 4), every lane quadrant
        const uint32_t one4 = 0x38383838u;
        for (int kb = 0; kb < 2; kb++)
            for (int c = 4; c < 8; c++)
                tmem_st1(tbase + ((uint32_t)(warp * 32) << 16) + PP_SFV + 8 * kb + c, __uint_as_float(one4));
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp < 4) pp_setmaxnreg_dec<40>();
    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int g = 0;   // K/V tiles loaded so far (ring position)
            int it = 0;  // items of this CTA so far
            for (int j = 0; ok && j < nrounds; j++) {
                const int i = pp_item_index(j, nitems);
                if (i < 0) continue;
                const PpItem I = pp_item(p, i);
                const int qs = it & 1;
                // Q buffers of this parity are free once the item two back issued its last Q K^T
                if (it >= 2 && !pp_wait(&s.q_empty[qs], ((it >> 1) - 1) & 1, abort)) break;
                const int nq = I.hasB ? 2 : 1;
                mbar_expect_tx(&s.q_full[qs], nq * (128 * D / 2 + KB * 512));
                for (int x = 0; x < nq; x++) {
                    const int tt = 2 * I.pair + x;
                    tma_load_3d(s.q[qs][x], &tm_q, &s.q_full[qs], 0, tt * 128, I.bh);
                    bulk_load(s.qsf[qs][x], p.q_sf + ((size_t)I.bh * p.T + tt) * KB * 512, KB * 512, &s.q_full[qs]);
                }
                for (int u = 0; u < I.nu; u++, g++) {
                    const int st = g % kPpStages;
                    if (g >= kPpStages && !pp_wait(&s.kv_empty[st], ((g / kPpStages) & 1) ^ 1, abort)) {
                        ok = false;
                        break;
                    }
                    const int nk = min(128, p.N - u * 128);
                    const int kblocks = nk > 64 ? 2 : 1;
                    mbar_expect_tx(&s.kv_full[st], 128 * D / 2 + KB * 512 + D * 64 + kblocks * 512);
                    tma_load_3d(s.k[st], &tm_k, &s.kv_full[st], 0, u * 128, I.bh);
                    bulk_load(s.ksf[st], p.k_sf + ((size_t)I.bh * p.T + u) * KB * 512, KB * 512, &s.kv_full[st]);
                    tma_load_3d(s.v[st], &tm_v, &s.kv_full[st], 0, u * D, I.bh);
                    bulk_load(s.vsf[st], p.v_sf + ((size_t)I.bh * p.CKv + 2 * u) * 512, kblocks * 512,
                              &s.kv_full[st]);
                }
                it++;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            int g0 = 0;  // ring position of the current item's key tile 0
            int kv_waited = -1, sfk_tile = -1, last_x = -1, last_idx = -1;
            int nS[2] = {0, 0}, nP[2] = {0, 0};  // Q_x K^T and P_x V issued so far
            int it = 0;
            for (int j = 0; ok && j < nrounds; j++) {
                const int i = pp_item_index(j, nitems);
                if (i < 0) continue;
                const PpItem I = pp_item(p, i);
                const int qs = it & 1;
                if (!pp_wait(&s.q_full[qs], (it >> 1) & 1, abort)) break;
                tc_fence_after();
                for (int x = 0; x < (I.hasB ? 2 : 1); x++)
                    for (int kb = 0; kb < KB; kb++)
                        tc_cp_sf(tbase + PP_SFQ + 8 * x + 4 * kb, smem_u32(s.qsf[qs][x] + 512 * kb));
                // Q_x K_u^T into the shared S buffer once its previous reader is done
                auto qk = [&](int x, int u) -> bool {
                    const int gt = g0 + u, st = gt % kPpStages;
                    if (gt > kv_waited) {
                        if (!pp_wait(&s.kv_full[st], (gt / kPpStages) & 1, abort)) return false;
                        kv_waited = gt;
                    }
                    if (last_x >= 0 && !pp_wait(&s.s_free[last_x], last_idx & 1, abort)) return false;
                    tc_fence_after();
                    if (sfk_tile != gt) {
                        for (int kb = 0; kb < KB; kb++)
                            tc_cp_sf(tbase + PP_SFK + 4 * kb, smem_u32(s.ksf[st] + 512 * kb));
                        sfk_tile = gt;
                    }
                    for (int kb = 0; kb < KB; kb++)
                        mma_fp4(tbase + PP_S, make_sdesc(smem_u32(s.q[qs][x]) + 32 * kb, QSBO, 16, QSW),
                                make_sdesc(smem_u32(s.k[st]) + 32 * kb, QSBO, 16, QSW), idesc_fp4(128, 128),
                                tbase + PP_SFQ + 8 * x + 4 * kb, tbase + PP_SFK + 4 * kb, kb > 0);
                    tc_commit(&s.s_full[x]);
                    last_x = x;
                    last_idx = nS[x]++;
                    return true;
                };
                // [O_x | l_x] (+)= P_x [V_u | 0 | 1]
                auto pv = [&](int x, int u) -> bool {
                    if (!pp_wait(&s.p_full[x], nP[x] & 1, abort)) return false;
                    tc_fence_after();
                    const int nk = min(128, p.N - u * 128);
                    const int kblocks = nk > 64 ? 2 : 1;
                    const int st = (g0 + u) % kPpStages;
                    for (int kb = 0; kb < kblocks; kb++) {
                        const uint64_t pd = make_sdesc(smem_u32(s.p[x]) + 32 * kb, 512, 16, 4);
                        const uint32_t acc = (u > 0 || kb > 0) ? 1u : 0u;
                        mma_fp4(tbase + PP_O + PP_OW * x, pd, make_sdesc(smem_u32(s.v[st]) + 32 * kb, 512, 16, 4),
                                idesc_fp4(128, PP_OW), tbase + PP_SFP + 8 * x + 4 * kb, tbase + PP_SFV + 8 * kb,
                                acc);
                    }
                    tc_commit(&s.o_done[x]);
                    nP[x]++;
                    return true;
                };
                // Issue order, steady state: P_A V_u, Q_B K_{u+1}^T, P_B V_u, Q_A K_{u+2}^T.
                // Scores are consumed in the order A0 B0 A1 B1 ...
                ok = qk(0, 0);
                if (ok && I.hasB) ok = qk(1, 0);
                if (ok && I.nuA > 1) ok = qk(0, 1);
                for (int u = 0; ok && u < I.nu; u++) {
                    const int st = (g0 + u) % kPpStages;
                    // V scale atoms of key tile u (P V of the tile before was issued earlier)
                    const int nk = min(128, p.N - u * 128);
                    const int kblocks = nk > 64 ? 2 : 1;
                    for (int kb = 0; kb < kblocks; kb++)
                        tc_cp_sf(tbase + PP_SFV + 8 * kb, smem_u32(s.vsf[st] + 512 * kb));
                    if (u < I.nuA && !(ok = pv(0, u))) break;
                    if (u + 1 < I.nuB && !(ok = qk(1, u + 1))) break;
                    if (u < I.nuB && !(ok = pv(1, u))) break;
                    tc_commit(&s.kv_empty[st]);
                    if (u + 2 < I.nuA && !(ok = qk(0, u + 2))) break;
                }
                // every Q K^T of this item has been issued: release its Q buffers
                if (ok) tc_commit(&s.q_empty[qs]);
                g0 += I.nu;
                it++;
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax
        pp_setmaxnreg_inc<232>();
        const int x = (warp - 4) >> 2;  // 0: tile A, 1: tile B
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float c2 = p.q_g[0] * p.k_g[0] * p.sm_scale * kLog2e;
        bool ok = true;
        int k = 0;  // key-tile steps of this tile role so far (all items)
        for (int j = 0; ok && j < nrounds; j++) {
            const int i = pp_item_index(j, nitems);
            if (i < 0) continue;
            const PpItem I = pp_item(p, i);
            const int nux = x == 0 ? I.nuA : I.nuB;
            if (nux == 0) continue;
            const int tq = 2 * I.pair + x;
            const int row = tq * 128 + r;
            float m2 = -INFINITY;
            for (int u = 0; u < nux; u++, k++) {
                if (!pp_wait(&s.s_full[x], k & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float sv[128];
#pragma unroll
                for (int c = 0; c < 4; c++)
                    tmem_ld32(tbase + lane_off + PP_S + 32 * c, *reinterpret_cast<float(*)[32]>(&sv[32 * c]));
                tmem_wait_ld();
                reg_fence(sv);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.s_free[x]);

                const int kbase = u * 128;
                if ((p.causal && u == tq) || (kbase + 128 > p.N)) {
#pragma unroll
                    for (int i2 = 0; i2 < 128; i2++) {
                        const int key = kbase + i2;
                        if (key >= p.N || (p.causal && key > row)) sv[i2] = -INFINITY;
                    }
                }
                float bmax[8];
#pragma unroll
                for (int blk = 0; blk < 8; blk++) bmax[blk] = pp_max16(&sv[16 * blk]);
                const float tmax = fmaxf(pp_max3(bmax[0], bmax[1], bmax[2]),
                                         fmaxf(pp_max3(bmax[3], bmax[4], bmax[5]), fmaxf(bmax[6], bmax[7])));
                const float m2_new = fmaxf(m2, tmax * c2);
                const float msub = m2_new == -INFINITY ? 0.0f : m2_new;
                const float alpha = ex2f(m2 - msub);
                m2 = m2_new;
                // block scales first (eight independent chains): E4M3 of (block max of
                // P * 2688) / 6, and log2 of the scale value from the exponent and a
                // table of significands
                const float lm = kLog2_2688 - msub;
                float bias[8];
                uint32_t scw0 = 0, scw1 = 0;
#pragma unroll
                for (int bp = 0; bp < 8; bp += 2) {
                    const uint32_t sc2 = f32x2_to_e4m3x2(ex2f(fmaf(bmax[bp], c2, lm)) * (1.0f / 6.0f),
                                                         ex2f(fmaf(bmax[bp + 1], c2, lm)) * (1.0f / 6.0f));
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const int blk = bp + h;
                        const uint32_t sc = (sc2 >> (8 * h)) & 0xFFu;
                        bias[blk] = sc ? lm - s.lg2sc[sc] : -INFINITY;
                        if (blk < 4)
                            scw0 |= sc << (8 * blk);
                        else
                            scw1 |= sc << (8 * (blk - 4));
                    }
                }
                // y = P * 2688 / scale, rounded to E2M1
                uint32_t codes[16];
#pragma unroll
                for (int blk = 0; blk < 8; blk++) {
                    float y[16];
#pragma unroll
                    for (int i2 = 0; i2 < 16; i2++) y[i2] = ex2f(fmaf(sv[16 * blk + i2], c2, bias[blk]));
                    codes[2 * blk] = pack8_e2m1(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
                    codes[2 * blk + 1] = pack8_e2m1(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
                }
                // P buffer and O are free once this role's previous P V finished
                // (for u = 0 that is the previous item's last one)
                if (k > 0 && !pp_wait(&s.o_done[x], (k - 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint8_t* prow = s.p[x] + (r >> 3) * 512 + (r & 7) * 64;
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    const int cs = c ^ ((r & 7) >> 1);
                    *reinterpret_cast<uint4*>(prow + cs * 16) =
                        make_uint4(codes[4 * c], codes[4 * c + 1], codes[4 * c + 2], codes[4 * c + 3]);
                }
                // P's block scales into TMEM: row r reads (lane r, column base + r / 32)
                tmem_st1(tbase + lane_off + PP_SFP + 8 * x + quad, __uint_as_float(scw0));
                tmem_st1(tbase + lane_off + PP_SFP + 8 * x + 4 + quad, __uint_as_float(scw1));
                if (u > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                    // rescale this row of O (64 columns per round trip) and l
                    const uint32_t oa = tbase + lane_off + PP_O + PP_OW * x;
#pragma unroll
                    for (int h = 0; h < D / 64; h++) {
                        float o0[32], o1[32];
                        tmem_ld32(oa + 64 * h, o0);
                        tmem_ld32(oa + 64 * h + 32, o1);
                        tmem_wait_ld();
                        reg_fence(o0);
                        reg_fence(o1);
#pragma unroll
                        for (int i2 = 0; i2 < 32; i2++) {
                            o0[i2] *= alpha;
                            o1[i2] *= alpha;
                        }
                        tmem_st32(oa + 64 * h, o0);
                        tmem_st32(oa + 64 * h + 32, o1);
                    }
                    const float lv = tmem_ld1_sync(oa + 128);
                    tmem_st1(oa + 128, lv * alpha);
                }
                tmem_wait_st();
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.p_full[x]);
            }
            // ---- epilogue of this item: out = O / l * g_V (O is reused by the next item
            // only after this role's next p_full arrival, which follows these loads)
            if (!ok || !pp_wait(&s.o_done[x], (k - 1) & 1, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float l = tmem_ld1_sync(tbase + lane_off + PP_O + PP_OW * x + 128);
            const float scale = p.v_g[0] / l;
            {
                // Stage 32 rows x 16 floats of O per round in this warp's 2 KB of the
                // tile's P buffer (idle until the next item's first P), 16-byte units
                // XOR-swizzled by row / 2, then write 64-byte row segments: each store
                // instruction covers 8 rows.
                float4* stage = reinterpret_cast<float4*>(s.p[x] + quad * 2048);
                const int row0 = tq * 128 + quad * 32;
                float* obase = p.out + ((size_t)I.bh * p.N + row0) * D;
#pragma unroll 1
                for (int c = 0; c < D / 16; c++) {
                    uint32_t o[16];
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                        "%12, %13, %14, %15}, [%16];\n\t"
                        "tcgen05.wait::ld.sync.aligned;"
                        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]),
                          "=r"(o[7]), "=r"(o[8]), "=r"(o[9]), "=r"(o[10]), "=r"(o[11]), "=r"(o[12]), "=r"(o[13]),
                          "=r"(o[14]), "=r"(o[15])
                        : "r"(tbase + lane_off + PP_O + PP_OW * x + 16 * c)
                        : "memory");
#pragma unroll
                    for (int j2 = 0; j2 < 4; j2++)
                        stage[lane * 4 + (j2 ^ ((lane >> 1) & 3))] =
                            make_float4(__uint_as_float(o[4 * j2]) * scale, __uint_as_float(o[4 * j2 + 1]) * scale,
                                        __uint_as_float(o[4 * j2 + 2]) * scale, __uint_as_float(o[4 * j2 + 3]) * scale);
                    __syncwarp();
#pragma unroll
                    for (int i2 = 0; i2 < 4; i2++) {
                        const int rr = 8 * i2 + (lane >> 2), jj = lane & 3;
                        if (row0 + rr < p.N)
                            *reinterpret_cast<float4*>(obase + (size_t)rr * D + 16 * c + 4 * jj) =
                                stage[rr * 4 + (jj ^ ((rr >> 1) & 3))];
                    }
                    __syncwarp();
                }
            }
            if (p.lse && row < p.N) p.lse[(size_t)I.bh * p.N + row] = m2 * kLn2 + logf(l * (1.0f / 2688.0f));
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace sa
