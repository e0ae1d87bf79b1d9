// attn_ws.cuh -- warp-specialised NVFP4 attention forward (all blocks FP4).
//
// Same mathematics and schedule as attn.cuh ("Search Your Block Floating
// Point Scales!", "ScaleSearchAttention / 네이티브 NVFP4 실행": Q K^T and P V
// as block-scaled FP4 tensor-core MMAs with FP32 accumulation; online softmax
// over key tiles of 128; P requantised per 16 keys with scale 1/2688), laid
// out as a pipeline so the tensor core, TMA and softmax overlap:
//
//   warp 0       TMA producer: Q once, then K/V codes + scale atoms through an
//                NS-stage ring.
//   warp 1       MMA issuer (one lane): scale atoms -> TMEM (tcgen05.cp),
//                S[j%2] = Q K_j^T, then O += P_{j-1} V_{j-1}, l += P_{j-1} 1.
//   warp 2       owns the TMEM allocation.
//   warps 4..11  softmax: warp 4+q and warp 8+q share TMEM lane quadrant q
//                (32 query rows); the first takes key columns 0..63 of each
//                tile, the second 64..127.  The two halves exchange their row
//                maxima through shared memory (named barrier per quadrant
//                pair), then each writes its half of the P codes, one P scale
//                atom, and rescales its half of the O columns.
//
// TMEM (512 columns): S0 S1 | O | l | scale atoms.  S is double buffered so
// Q K^T of tile j+1 runs while the softmax of tile j does.
#pragma once

#include "attn.cuh"

namespace sa {

constexpr int kWsStages = 4;
constexpr int kWsThreads = 384;

template <int D>
struct WsSmem {
    alignas(1024) uint8_t q[128 * D / 2];
    alignas(1024) uint8_t k[kWsStages][128 * D / 2];
    alignas(1024) uint8_t v[kWsStages][D * 64];
    alignas(1024) uint8_t p[128 * 64];
    alignas(1024) uint8_t ones[16 * 64];
    alignas(16) uint8_t qsf[D / 64 * 512];
    uint8_t ksf[kWsStages][D / 64 * 512];
    uint8_t vsf[kWsStages][2 * 512];
    uint8_t psf[2 * 512];
    uint8_t onesf[512];
    float xmax[2][2][128];  // [tile parity][half][row] partial row maxima
    uint64_t q_full;
    uint64_t kv_full[kWsStages];
    uint64_t kv_empty[kWsStages];
    uint64_t s_full[2];
    uint64_t s_free[2];
    uint64_t p_full;
    uint64_t o_done;
    uint64_t xbar[2][4];  // [tile parity][quadrant]: both halves wrote their maxima
    uint32_t tmem_slot;
    int abort;
};

// TMEM columns
constexpr uint32_t WS_S = 0, WS_O = 256, WS_L = 384, WS_SFQ = 400, WS_SFK = 408, WS_SFV = 424, WS_SFP = 440,
                   WS_SF1 = 448;

// Bounded wait that also gives up as soon as another role has given up.
SA_DEV bool ws_wait(uint64_t* bar, uint32_t parity, volatile int* abort)
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

template <int D>
__global__ void __launch_bounds__(kWsThreads, 1) attn_fwd_ws_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                    const __grid_constant__ CUtensorMap tm_k,
                                                                    const __grid_constant__ CUtensorMap tm_v,
                                                                    const AttnParams p)
{
    constexpr int KB = D / 64;
    constexpr uint32_t QSW = D == 128 ? 4u : 6u;
    constexpr uint32_t QSBO = 8 * D / 2;
    extern __shared__ uint8_t smem_raw[];
    WsSmem<D>& s = *reinterpret_cast<WsSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
    const int bh = blockIdx.z * p.H + blockIdx.y;
    const int Tk = (p.N + 127) / 128;
    const int nt = p.causal ? min(t + 1, Tk) : Tk;
    volatile int* abort = &s.abort;

    if (warp == 2) {
        tmem_alloc(&s.tmem_slot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        s.abort = 0;
        mbar_init(&s.q_full, 1);
        for (int i = 0; i < kWsStages; i++) {
            mbar_init(&s.kv_full[i], 1);
            mbar_init(&s.kv_empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&s.s_full[i], 1);
            mbar_init(&s.s_free[i], 8);
        }
        mbar_init(&s.p_full, 8);
        mbar_init(&s.o_done, 1);
        for (int i = 0; i < 8; i++) mbar_init(&s.xbar[i >> 2][i & 3], 64);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    for (int i = tid; i < 16 * 64 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(s.ones)[i] = 0x22222222u;
    for (int i = tid; i < 512 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(s.onesf)[i] = 0x38383838u;
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s.tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            mbar_expect_tx(&s.q_full, 128 * D / 2 + KB * 512);
            tma_load_3d(s.q, &tm_q, &s.q_full, 0, t * 128, bh);
            bulk_load(s.qsf, p.q_sf + ((size_t)bh * p.T + t) * KB * 512, KB * 512, &s.q_full);
            for (int j = 0; j < nt; j++) {
                const int st = j % kWsStages;
                if (j >= kWsStages && !ws_wait(&s.kv_empty[st], ((j / kWsStages) & 1) ^ 1, abort)) break;
                const int nk = min(128, p.N - j * 128);
                const int kblocks = nk > 64 ? 2 : 1;
                mbar_expect_tx(&s.kv_full[st], 128 * D / 2 + KB * 512 + D * 64 + kblocks * 512);
                tma_load_3d(s.k[st], &tm_k, &s.kv_full[st], 0, j * 128, bh);
                bulk_load(s.ksf[st], p.k_sf + ((size_t)bh * p.T + j) * KB * 512, KB * 512, &s.kv_full[st]);
                tma_load_3d(s.v[st], &tm_v, &s.kv_full[st], j * 64, 0, bh);
                bulk_load(s.vsf[st], p.v_sf + ((size_t)bh * p.CKv + 2 * j) * 512, kblocks * 512, &s.kv_full[st]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = ws_wait(&s.q_full, 0, abort);
            if (ok) {
                tc_fence_after();
                for (int kb = 0; kb < KB; kb++) tc_cp_sf(tbase + WS_SFQ + 4 * kb, smem_u32(s.qsf + 512 * kb));
                tc_cp_sf(tbase + WS_SF1, smem_u32(s.onesf));
            }
            auto issue_pv = [&](int i) -> bool {
                if (!ws_wait(&s.p_full, i & 1, abort)) return false;
                tc_fence_after();
                const int st = i % kWsStages, b = i & 1;
                const int nk = min(128, p.N - i * 128);
                const int kblocks = nk > 64 ? 2 : 1;
                for (int kb = 0; kb < kblocks; kb++) tc_cp_sf(tbase + WS_SFP + 4 * kb, smem_u32(s.psf + 512 * kb));
                for (int kb = 0; kb < kblocks; kb++) {
                    const uint64_t pd = make_sdesc(smem_u32(s.p) + 32 * kb, 512, 16, 4);
                    const uint32_t acc = (i > 0 || kb > 0) ? 1u : 0u;
                    mma_fp4(tbase + WS_O, pd, make_sdesc(smem_u32(s.v[st]) + 32 * kb, 512, 16, 4),
                            idesc_fp4(128, D), tbase + WS_SFP + 4 * kb, tbase + WS_SFV + 8 * b + 4 * kb, acc);
                    mma_fp4(tbase + WS_L, pd, make_sdesc(smem_u32(s.ones) + 32 * kb, 512, 16, 4),
                            idesc_fp4(128, 16), tbase + WS_SFP + 4 * kb, tbase + WS_SF1, acc);
                }
                tc_commit(&s.o_done);
                tc_commit(&s.kv_empty[st]);
                return true;
            };
            for (int j = 0; ok && j < nt; j++) {
                const int st = j % kWsStages, b = j & 1;
                if (!ws_wait(&s.kv_full[st], (j / kWsStages) & 1, abort)) break;
                if (j >= 2 && !ws_wait(&s.s_free[b], ((j - 2) >> 1) & 1, abort)) break;
                tc_fence_after();
                const int nk = min(128, p.N - j * 128);
                const int kblocks = nk > 64 ? 2 : 1;
                for (int kb = 0; kb < KB; kb++)
                    tc_cp_sf(tbase + WS_SFK + 8 * b + 4 * kb, smem_u32(s.ksf[st] + 512 * kb));
                for (int kb = 0; kb < kblocks; kb++)
                    tc_cp_sf(tbase + WS_SFV + 8 * b + 4 * kb, smem_u32(s.vsf[st] + 512 * kb));
                for (int kb = 0; kb < KB; kb++)
                    mma_fp4(tbase + WS_S + 128 * b, make_sdesc(smem_u32(s.q) + 32 * kb, QSBO, 16, QSW),
                            make_sdesc(smem_u32(s.k[st]) + 32 * kb, QSBO, 16, QSW), idesc_fp4(128, 128),
                            tbase + WS_SFQ + 4 * kb, tbase + WS_SFK + 8 * b + 4 * kb, kb > 0);
                tc_commit(&s.s_full[b]);
                if (j >= 1 && !issue_pv(j - 1)) break;
            }
            if (ok && !*abort) issue_pv(nt - 1);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax
        const int quad = warp & 3, half = (warp - 4) >> 2;
        const int r = quad * 32 + lane;  // TMEM lane = row in the tile
        const int row = t * 128 + r;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float c2 = p.q_g[0] * p.k_g[0] * p.sm_scale * kLog2e;
        float m2 = -INFINITY;
        bool ok = true;
        for (int j = 0; j < nt; j++) {
            const int b = j & 1;
            if (!ws_wait(&s.s_full[b], (j >> 1) & 1, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[64];
            tmem_ld32(tbase + lane_off + WS_S + 128 * b + 64 * half, *reinterpret_cast<float(*)[32]>(&sv[0]));
            tmem_ld32(tbase + lane_off + WS_S + 128 * b + 64 * half + 32, *reinterpret_cast<float(*)[32]>(&sv[32]));
            tmem_wait_ld();
            reg_fence(sv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.s_free[b]);

            const int kbase = j * 128 + 64 * half;
            const bool need_mask = (p.causal && j == t) || (j * 128 + 128 > p.N);
            if (need_mask) {
#pragma unroll
                for (int i = 0; i < 64; i++) {
                    const int key = kbase + i;
                    if (key >= p.N || (p.causal && key > row)) sv[i] = -INFINITY;
                }
            }
            float bmax[4];
#pragma unroll
            for (int blk = 0; blk < 4; blk++) {
                float mx = sv[16 * blk];
#pragma unroll
                for (int i = 1; i < 16; i++) mx = fmaxf(mx, sv[16 * blk + i]);
                bmax[blk] = mx;
            }
            const float hmax = fmaxf(fmaxf(bmax[0], bmax[1]), fmaxf(bmax[2], bmax[3]));
            s.xmax[b][half][r] = hmax;
            mbar_arrive(&s.xbar[b][quad]);
            if (!ws_wait(&s.xbar[b][quad], (j >> 1) & 1, abort)) {
                ok = false;
                break;
            }
            const float tmax = fmaxf(hmax, s.xmax[b][half ^ 1][r]);
            const float m2_new = fmaxf(m2, tmax * c2);
            const float msub = m2_new == -INFINITY ? 0.0f : m2_new;
            const float alpha = ex2f(m2 - msub);
            m2 = m2_new;
            uint32_t codes[8];
            uint32_t scw = 0;
#pragma unroll
            for (int blk = 0; blk < 4; blk++) {
                const float pmax = ex2f(fmaf(bmax[blk], c2, kLog2_2688 - msub));
                const uint32_t sc = f32_to_e4m3(pmax * (1.0f / 6.0f));
                const float bias = sc ? (kLog2_2688 - msub - lg2f(e4m3_to_f32(sc))) : -INFINITY;
                float y[16];
#pragma unroll
                for (int i = 0; i < 16; i++) y[i] = ex2f(fmaf(sv[16 * blk + i], c2, bias));
                codes[2 * blk] = pack8_e2m1(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
                codes[2 * blk + 1] = pack8_e2m1(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
                scw |= sc << (8 * blk);
            }
            // P buffer and O are free once P V of the previous tile finished
            if (j > 0 && !ws_wait(&s.o_done, (j - 1) & 1, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint8_t* prow = s.p + (r >> 3) * 512 + (r & 7) * 64;
#pragma unroll
            for (int c = 0; c < 2; c++) {
                const int cs = (2 * half + c) ^ ((r & 7) >> 1);
                *reinterpret_cast<uint4*>(prow + cs * 16) =
                    make_uint4(codes[4 * c], codes[4 * c + 1], codes[4 * c + 2], codes[4 * c + 3]);
            }
            *reinterpret_cast<uint32_t*>(s.psf + 512 * half + (r & 31) * 16 + (r >> 5) * 4) = scw;
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                tmem_scale_cols(tbase + lane_off + WS_O + half * (D / 2), D / 2, alpha);
                if (half == 0) {
                    const float l = tmem_ld1_sync(tbase + lane_off + WS_L);
                    tmem_st1(tbase + lane_off + WS_L, l * alpha);
                    tmem_wait_st();
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.p_full);
        }
        // ---- epilogue: out = O / l * g_V for this half of the row
        if (ok && ws_wait(&s.o_done, (nt - 1) & 1, abort)) {
            tc_fence_after();
            const float l = tmem_ld1_sync(tbase + lane_off + WS_L);
            const float scale = p.v_g[0] / l;
            float* orow = p.out + ((size_t)bh * p.N + row) * D + half * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 64; c++) {
                float o[32];
                tmem_ld32(tbase + lane_off + WS_O + half * (D / 2) + 32 * c, o);
                tmem_wait_ld();
                reg_fence(o);
                if (row < p.N) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(orow + 32 * c + i) =
                            make_float4(o[i] * scale, o[i + 1] * scale, o[i + 2] * scale, o[i + 3] * scale);
                }
            }
            if (half == 0 && p.lse && row < p.N)
                p.lse[(size_t)bh * p.N + row] = m2 * kLn2 + logf(l * (1.0f / 2688.0f));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) tmem_dealloc(tbase, 512);
}

}  // namespace sa
