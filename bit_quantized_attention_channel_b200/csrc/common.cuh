// common.cuh -- shared device helpers of libsa: status word, NVFP4 number
// formats, launch checks.  Everything here is exact integer or IEEE
// round-to-nearest-even arithmetic; nothing depends on compiler contraction.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sa.h"

#define SA_DEV __device__ __forceinline__

// Library status word (one per device); kernels record the first device-side
// problem here, sa_device_status() reads it.
__device__ int g_sa_status;

SA_DEV void sa_raise(int code) { atomicCAS(&g_sa_status, 0, code); }

// Upper bound for any wait inside a kernel: about 2 s at the B200 clock.
#define SA_WAIT_CYCLES (4000000000LL)

// ---------------------------------------------------------------------------
// NVFP4 number formats
// ---------------------------------------------------------------------------

// E4M3 scale byte (0..0x7E) -> exact float: 4 exponent bits (bias 7),
// 3 mantissa bits, exponent field 0 subnormal (m * 2^-9).
SA_DEV float e4m3_to_f32(uint32_t c)
{
    uint32_t e = (c >> 3) & 15u, m = c & 7u;
    if (e == 0) return (float)m * 0.001953125f;
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Non-negative finite float -> E4M3 byte, round to nearest even, saturating
// to 448 (hardware conversion; the high byte of the pair is unused).
SA_DEV uint32_t f32_to_e4m3(float x)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return r & 0xFFu;
}

// Two non-negative finite floats -> two E4M3 bytes (a in the low byte), each
// rounded and saturated as f32_to_e4m3 does, in one conversion.
SA_DEV uint32_t f32x2_to_e4m3x2(float a, float b)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

// Eight floats -> eight E2M1 nibbles (round to nearest even, saturating to
// +-6, sign kept), element 0 in the lowest nibble.
SA_DEV uint32_t pack8_e2m1(float y0, float y1, float y2, float y3, float y4, float y5, float y6, float y7)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "f"(y4), "f"(y5), "f"(y6), "f"(y7));
    return out;
}

// E2M1 nibble -> exact float: sign, 2 exponent bits (bias 1), 1 mantissa
// bit; exponent field 0 is 0 or 0.5.
SA_DEV float e2m1_to_f32(uint32_t n)
{
    uint32_t e = (n >> 1) & 3u, m = n & 1u;
    uint32_t bits = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
    return __uint_as_float(bits | ((n & 8u) << 28));
}

SA_DEV float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// Tensor-core scale-factor atom: byte offset of (row r within a 128-row
// tile, block j within a 4-block chunk) inside its 512-byte atom.
SA_DEV uint32_t sf_atom_offset(uint32_t r, uint32_t j) { return (r & 31u) * 16u + (r >> 5) * 4u + j; }

// Per-tensor scale pair from the amax: g = A/2688, 1/g = 2688/A (IEEE
// division), an all-zero tensor uses 1.
SA_DEV void tensor_scale(float amax, float& g, float& inv_g)
{
    if (amax == 0.0f) {
        g = 1.0f;
        inv_g = 1.0f;
    } else {
        g = __fdiv_rn(amax, 2688.0f);
        inv_g = __fdiv_rn(2688.0f, amax);
    }
}

// ---------------------------------------------------------------------------
// Host helpers
// ---------------------------------------------------------------------------
#define SA_CHECK_LAUNCH()                                   \
    do {                                                    \
        if (cudaPeekAtLastError() != cudaSuccess) {         \
            cudaGetLastError();                             \
            return SA_ERR_CUDA;                             \
        }                                                   \
    } while (0)

static inline size_t sa_align256(size_t x) { return (x + 255) & ~(size_t)255; }
static inline int sa_cdiv(int a, int b) { return (a + b - 1) / b; }
