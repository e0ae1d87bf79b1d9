// attn.cuh -- parameters and constants shared by the NVFP4 attention kernels.
//
// "Search Your Block Floating Point Scales!" (gist.science summary),
// "ScaleSearchAttention / 네이티브 NVFP4 실행": Q K^T and P V run natively in
// NVFP4 on tensor cores with FP32 accumulation.  SageAttention3 article
// (dasgeld.co): FP4 tensor-core attention on Blackwell.  "ThriftAttention:
// 5%의 연산량으로 90%의 품질 유지": a few query-key blocks in high precision
// inside one joint softmax.
//
// Score arithmetic common to the kernels (log2 units throughout):
//   NVFP4 block:  t = S c2, c2 = g_Q g_K sm_scale log2(e), S the block-scaled
//                 MMA result of the codes;
//   bf16 block:   t = (q.k - c_i) sm_scale log2(e), q.k from the raw bf16
//                 inputs, c_i = q_i . mean(K) (so both kinds of block carry
//                 the same per-row offset as the smoothed keys);
//   running max m, P~ = 2^(t - m); NVFP4 P: per 16 keys, scale
//   E4M3(max(2688 P~) / 6) and E2M1 codes of 2688 P~ / scale, computed as
//   2^(t + log2(2688) - m - log2(scale)).
#pragma once

#include "tc.cuh"

namespace sa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2_2688 = 11.392317422778761f;

struct AttnParams {
    const uint8_t* q_sf;
    const uint8_t* k_sf;
    const uint8_t* v_sf;
    const float* q_g;
    const float* k_g;
    const float* v_g;
    float* out;
    float* lse;
    int N, H, B;
    int T;    // 128-row tiles of Q/K (= scale row tiles per (b,h))
    int CKv;  // 64-key chunks of the V scale atoms per (b,h)
    int causal;
    float sm_scale;
    const uint8_t* mask;  // mixed: [B,H,T,T] high-precision block flags
    const uint16_t* q_bf16;
    const float* k_mean;  // mixed: channel means of K (nullptr: not smoothed)
    long long wait_cycles;  // limit of every pipeline wait (SM clock cycles)
};

SA_DEV float tmem_ld1_sync(uint32_t taddr)
{
    uint32_t r;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r)
        : "r"(taddr)
        : "memory");
    return __uint_as_float(r);
}

}  // namespace sa
