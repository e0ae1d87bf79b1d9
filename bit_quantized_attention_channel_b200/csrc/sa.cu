// sa.cu -- the C ABI of libsa (declared in include/sa.h): argument checks,
// TMA tensor maps, workspace carving and kernel launches.  One translation
// unit so the device status word is a single object.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>

#include "attn_pp.cuh"
#include "decode.cuh"
#include "incoherence.cuh"
#include "quant.cuh"
#include "select.cuh"

using namespace sa;

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// The driver's tensor-map encoder, resolved once (thread-safe static
// initialisation); null when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    }();
    return fn;
}

// Streaming multiprocessors of the current device (cached per device; host
// threads may race on the first query, which stores the same value).
int sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// One value per device (kernel attributes and occupancy are per device:
// cudaFuncSetAttribute and the occupancy query act on the current one).
// Host threads may race on a device's first use; they store the same value.
struct PerDevice {
    std::atomic<int> v[64];
};

int current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev >= 0 && dev < 64 ? dev : -1;
}

// Run `set` (returning a positive value, or <= 0 on failure) once per device
// and return the cached value; 0 on failure.
template <typename F>
int once_per_device(PerDevice& pd, F&& set)
{
    const int dev = current_device();
    if (dev < 0) return 0;
    int v = pd.v[dev].load(std::memory_order_acquire);
    if (v > 0) return v;
    v = set();
    if (v <= 0) return 0;
    pd.v[dev].store(v, std::memory_order_release);
    return v;
}

// Opt a kernel into `smem` bytes of dynamic shared memory on the current
// device (once per device); false on failure.
template <typename K>
bool allow_smem(PerDevice& pd, K kernel, int smem)
{
    return once_per_device(pd, [&] {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess ? 1 : 0;
    }) > 0;
}

// Limit of every pipeline wait of the attention kernel, in SM clock cycles
// (0: the library default, about 2 s at the B200 clock).
std::atomic<long long> g_wait_cycles{0};

// The attention kernel moves registers between its warps with setmaxnreg;
// an increase waits until the CTA's launch allocation (threads x registers
// per thread, fixed by the compiler) has room, so a split larger than that
// allocation would never proceed.  Refuse to launch such a build.
template <typename K>
bool pp_regs_fit(K kernel)
{
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return false;
    return (long)fa.numRegs * kPpThreads >= 128L * PP_REG_CTL + 512L * PP_REG_SM;
}

// 3-D byte tensor {d0 (contiguous), d1, d2}; box {b0, b1, 1}.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                 uint32_t b1, CUtensorMapSwizzle swz)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0, d0 * d1};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D bf16 tensor {d0 (contiguous, elements), d1, d2}; box {64, 128, 1} with
// the 128-byte swizzle (one 128-byte row of 64 elements per box row).
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int rt_ck(int R, int C, int* RT, int* CK)
{
    *RT = sa_cdiv(R, 128);
    *CK = sa_cdiv(C, 64);
    return 0;
}

}  // namespace

extern "C" {

const char* sa_status_string(sa_status s)
{
    switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    case SA_ERR_NONFINITE: return "SA_ERR_NONFINITE";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
    case SA_ERR_DEVICE_ASSERT: return "SA_ERR_DEVICE_ASSERT";
    }
    return "SA_ERR_UNKNOWN";
}

void sa_set_wait_cycles(long long cycles) { g_wait_cycles.store(cycles > 0 ? cycles : 0, std::memory_order_relaxed); }

sa_status sa_device_status(cudaStream_t stream, int reset)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_sa_status, sizeof(int)) != cudaSuccess) return SA_ERR_CUDA;
    if (reset) {
        int z = 0;
        if (cudaMemcpyToSymbol(g_sa_status, &z, sizeof(int)) != cudaSuccess) return SA_ERR_CUDA;
    }
    return (sa_status)v;
}

size_t sa_codes_bytes(int B, int H, int N, int D, sa_role role)
{
    if (B < 0 || H < 0 || N < 0 || D < 0) return 0;
    if (role == SA_ROLE_V) return (size_t)B * H * sa_cdiv(N, 128) * D * 64;  // whole 128-token tiles
    return (size_t)B * H * N * D / 2;
}

size_t sa_scales_bytes(int B, int H, int N, int D, sa_role role)
{
    if (B < 0 || H < 0 || N < 0 || D < 0) return 0;
    int RT, CK;
    if (role == SA_ROLE_V)
        rt_ck(D, N, &RT, &CK);
    else
        rt_ck(N, D, &RT, &CK);
    return (size_t)B * H * RT * CK * 512;
}

size_t sa_quant_workspace_size(int B, int H, int N, int D, sa_role role)
{
    if (B < 0 || H < 0 || N < 0 || D < 0) return 0;
    return quant_ws_layout(nullptr, B, H, N, D, role).bytes;
}

sa_status sa_quant_nvfp4(const void* x_dev, int B, int H, int N, int D, sa_role role, int smooth,
                         sa_scale_mode mode, int f_lo, int f_hi, uint8_t* codes_dev, uint8_t* scales_dev,
                         float* g_dev, float* k_mean_dev, int8_t* ss_off_dev, void* ws_dev, size_t ws_bytes,
                         cudaStream_t stream)
{
    if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
    if (role != SA_ROLE_Q && role != SA_ROLE_K && role != SA_ROLE_V) return SA_ERR_INVALID_ARG;
    if (mode != SA_SCALE_MAX && mode != SA_SCALE_SEARCH) return SA_ERR_INVALID_ARG;
    if (mode == SA_SCALE_SEARCH && !(f_lo >= -16 && f_lo <= 0 && f_hi > 0 && f_hi <= 16)) return SA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
    if (N % 16) return SA_ERR_INVALID_ARG;
    if ((size_t)B * H * N == 0) return SA_OK;
    if (!x_dev || !codes_dev || !scales_dev || !g_dev || !ws_dev) return SA_ERR_INVALID_ARG;
    if (!aligned16(x_dev) || ((uintptr_t)codes_dev & 7u) || ((uintptr_t)ws_dev & 255u)) return SA_ERR_INVALID_ARG;
    if (role != SA_ROLE_K) smooth = 0;
    QuantWs w = quant_ws_layout(ws_dev, B, H, N, D, role);
    if (ws_bytes < w.bytes) return SA_ERR_WORKSPACE;
    const size_t BH = (size_t)B * H;
    const int T = sa_cdiv(N, kTile);

    if (cudaMemsetAsync(w.amax, 0, 4, stream) != cudaSuccess) return SA_ERR_CUDA;

    float* kmean = k_mean_dev ? k_mean_dev : w.kmean;
    if (smooth) {
        dim3 g1(sa_cdiv(T, 256 / (D / 2)), (unsigned)BH);
        if (D == 128)
            kstats_kernel<128><<<g1, 256, 0, stream>>>((const uint32_t*)x_dev, N, T, w.psum, w.pmax, w.pmin);
        else
            kstats_kernel<64><<<g1, 256, 0, stream>>>((const uint32_t*)x_dev, N, T, w.psum, w.pmax, w.pmin);
        SA_CHECK_LAUNCH();
        kfinal_kernel<<<(unsigned)BH, 128, 0, stream>>>(w.psum, w.pmax, w.pmin, N, T, D, kmean, w.amax);
        SA_CHECK_LAUNCH();
    } else {
        size_t n16 = BH * N * D / 8;
        amax_bf16_kernel<<<grid_for(n16, 256 * 4), 256, 0, stream>>>((const uint4*)x_dev, n16, w.amax);
        SA_CHECK_LAUNCH();
    }

    const bool ss = mode == SA_SCALE_SEARCH;
    const dim3 grid((unsigned)T, (unsigned)BH);
    if (role == SA_ROLE_V) {
        const uint16_t* x = (const uint16_t*)x_dev;
#define SA_QV(DD, SS) quant_v_kernel<DD, SS><<<grid, 2 * DD, 0, stream>>>(x, N, w.amax, f_lo, f_hi, codes_dev, \
                                                                           scales_dev, ss_off_dev, g_dev)
        if (D == 128) {
            if (ss) SA_QV(128, true); else SA_QV(128, false);
        } else {
            if (ss) SA_QV(64, true); else SA_QV(64, false);
        }
#undef SA_QV
    } else {
        const uint4* x = (const uint4*)x_dev;
        uint2* c = (uint2*)codes_dev;
#define SA_QR(DD, SM, SS)                                                                                    \
    quant_rows_kernel<DD, SM, SS><<<grid, 2 * DD, 0, stream>>>(x, N, kmean, w.amax, f_lo, f_hi, c, scales_dev, \
                                                              ss_off_dev, g_dev)
        if (D == 128) {
            if (smooth) {
                if (ss) SA_QR(128, true, true); else SA_QR(128, true, false);
            } else {
                if (ss) SA_QR(128, false, true); else SA_QR(128, false, false);
            }
        } else {
            if (smooth) {
                if (ss) SA_QR(64, true, true); else SA_QR(64, true, false);
            } else {
                if (ss) SA_QR(64, false, true); else SA_QR(64, false, false);
            }
        }
#undef SA_QR
    }
    SA_CHECK_LAUNCH();
    return SA_OK;
}

size_t sa_quant_ip_workspace_size(int B, int H, int N, int D)
{
    if (B < 0 || H < 0 || N < 0 || D < 0) return 0;
    return ip_ws_layout(nullptr, B, H, N, D).bytes;
}

sa_status sa_quant_nvfp4_ip(const void* q_dev, const void* k_dev, int B, int H, int N, int D,
                            const int8_t* signs_dev, int smooth, sa_scale_mode mode, int f_lo, int f_hi,
                            uint8_t* q_codes_dev, uint8_t* q_scales_dev, float* q_g_dev, uint8_t* k_codes_dev,
                            uint8_t* k_scales_dev, float* k_g_dev, float* k_mean_dev, float* r_dev,
                            int8_t* q_ss_off_dev, int8_t* k_ss_off_dev, void* ws_dev, size_t ws_bytes,
                            cudaStream_t stream)
{
    if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
    if (mode != SA_SCALE_MAX && mode != SA_SCALE_SEARCH) return SA_ERR_INVALID_ARG;
    if (mode == SA_SCALE_SEARCH && !(f_lo >= -16 && f_lo <= 0 && f_hi > 0 && f_hi <= 16)) return SA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
    if (N % 16) return SA_ERR_INVALID_ARG;
    if ((size_t)B * H * N == 0) return SA_OK;
    if ((size_t)B * H > 65535) return SA_ERR_UNSUPPORTED;
    if (!q_dev || !k_dev || !signs_dev || !q_codes_dev || !q_scales_dev || !q_g_dev || !k_codes_dev ||
        !k_scales_dev || !k_g_dev || !ws_dev)
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q_dev) || !aligned16(k_dev) || ((uintptr_t)q_codes_dev & 7u) || ((uintptr_t)k_codes_dev & 7u) ||
        ((uintptr_t)ws_dev & 255u) || ((uintptr_t)k_mean_dev & 15u))
        return SA_ERR_INVALID_ARG;
    IpWs w = ip_ws_layout(ws_dev, B, H, N, D);
    if (ws_bytes < w.bytes) return SA_ERR_WORKSPACE;
    const size_t BH = (size_t)B * H;
    const int T = sa_cdiv(N, kTile);
    if (cudaMemsetAsync(w.amax, 0, 16, stream) != cudaSuccess) return SA_ERR_CUDA;
    float* kmean = k_mean_dev ? k_mean_dev : w.kst.kmean;
    if (smooth) {
        dim3 g1(sa_cdiv(T, 256 / (D / 2)), (unsigned)BH);
        if (D == 128)
            kstats_kernel<128><<<g1, 256, 0, stream>>>((const uint32_t*)k_dev, N, T, w.kst.psum, w.kst.pmax,
                                                        w.kst.pmin);
        else
            kstats_kernel<64><<<g1, 256, 0, stream>>>((const uint32_t*)k_dev, N, T, w.kst.psum, w.kst.pmax,
                                                       w.kst.pmin);
        SA_CHECK_LAUNCH();
        kfinal_kernel<<<(unsigned)BH, 128, 0, stream>>>(w.kst.psum, w.kst.pmax, w.kst.pmin, N, T, D, kmean,
                                                         w.amax + 2);
        SA_CHECK_LAUNCH();
    }
    IpParams p{};
    p.x[0] = (const uint16_t*)q_dev;
    p.x[1] = (const uint16_t*)k_dev;
    p.k_mean = smooth ? kmean : nullptr;
    p.signs = signs_dev;
    p.hn = (float)(1.0 / std::sqrt((double)D));
    p.N = N;
    p.T = T;
    p.part[0] = w.part[0];
    p.part[1] = w.part[1];
    p.r = w.r;
    p.r_out = r_dev;
    p.amax = w.amax;
    IpOut o{};
    o.codes[0] = q_codes_dev;
    o.codes[1] = k_codes_dev;
    o.scales[0] = q_scales_dev;
    o.scales[1] = k_scales_dev;
    o.g[0] = q_g_dev;
    o.g[1] = k_g_dev;
    o.ss_off[0] = q_ss_off_dev;
    o.ss_off[1] = k_ss_off_dev;
    o.f_lo = f_lo;
    o.f_hi = f_hi;
    const dim3 grid3((unsigned)T, (unsigned)BH, 2);
    const bool ss = mode == SA_SCALE_SEARCH;
#define SA_IP(DD)                                                                                          \
    do {                                                                                                   \
        const int smem = 128 * (DD + 1) * (int)sizeof(float);                                              \
        static PerDevice attr;                                                                             \
        if (!allow_smem(attr, ip_sums_kernel<DD>, smem)) return SA_ERR_CUDA;                               \
        ip_sums_kernel<DD><<<grid3, 128, smem, stream>>>(p);                                               \
        SA_CHECK_LAUNCH();                                                                                 \
        ip_r_kernel<<<(unsigned)BH, DD, 0, stream>>>(p, DD);                                               \
        SA_CHECK_LAUNCH();                                                                                 \
        ip_amax_kernel<DD><<<grid3, 128, 0, stream>>>(p);                                                  \
        SA_CHECK_LAUNCH();                                                                                 \
        if (ss) ip_quant_kernel<DD, true><<<grid3, 128, 0, stream>>>(p, o);                                \
        else ip_quant_kernel<DD, false><<<grid3, 128, 0, stream>>>(p, o);                                  \
    } while (0)
    if (D == 128) SA_IP(128);
    else SA_IP(64);
#undef SA_IP
    SA_CHECK_LAUNCH();
    return SA_OK;
}

// Workspace of the fused pre-pass: amax words and K tickets (cleared per call),
// then the K tile partials and channel means.
struct QkvWs {
    unsigned* amax;    // [3]
    unsigned* ticket;  // [B*H]
    size_t zero_bytes;
    double* psum;
    float* pmax;
    float* pmin;
    float* kmean;
    size_t bytes;
};

static QkvWs qkv_ws_layout(void* base, int B, int H, int N, int D)
{
    QkvWs w{};
    char* p = (char*)base;
    const size_t BH = (size_t)B * H, T = (size_t)sa_cdiv(N, kTile);
    w.amax = (unsigned*)p;
    w.ticket = (unsigned*)(p + 16);
    w.zero_bytes = sa_align256(16 + BH * sizeof(unsigned));
    size_t off = w.zero_bytes;
    w.psum = (double*)(p + off);
    off += sa_align256(BH * T * D * sizeof(double));
    w.pmax = (float*)(p + off);
    off += sa_align256(BH * T * D * sizeof(float));
    w.pmin = (float*)(p + off);
    off += sa_align256(BH * T * D * sizeof(float));
    w.kmean = (float*)(p + off);
    off += sa_align256(BH * D * sizeof(float));
    w.bytes = off;
    return w;
}

size_t sa_quant_qkv_workspace_size(int B, int H, int N, int D)
{
    if (B < 0 || H < 0 || N < 0 || D < 0) return 0;
    return qkv_ws_layout(nullptr, B, H, N, D).bytes;
}

sa_status sa_quant_nvfp4_qkv(const void* q_dev, const void* k_dev, const void* v_dev, int B, int H, int N, int D,
                             int smooth_k, sa_scale_mode mode, int f_lo, int f_hi, uint8_t* q_codes_dev,
                             uint8_t* q_scales_dev, float* q_g_dev, uint8_t* k_codes_dev, uint8_t* k_scales_dev,
                             float* k_g_dev, float* k_mean_dev, uint8_t* v_codes_dev, uint8_t* v_scales_dev,
                             float* v_g_dev, void* ws_dev, size_t ws_bytes, cudaStream_t stream)
{
    if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
    if (mode != SA_SCALE_MAX && mode != SA_SCALE_SEARCH) return SA_ERR_INVALID_ARG;
    if (mode == SA_SCALE_SEARCH && !(f_lo >= -16 && f_lo <= 0 && f_hi > 0 && f_hi <= 16)) return SA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
    if (N % 16) return SA_ERR_INVALID_ARG;
    if ((size_t)B * H * N == 0) return SA_OK;
    if (!q_dev || !k_dev || !v_dev || !q_codes_dev || !q_scales_dev || !q_g_dev || !k_codes_dev || !k_scales_dev ||
        !k_g_dev || !v_codes_dev || !v_scales_dev || !v_g_dev || !ws_dev)
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(v_dev) || ((uintptr_t)q_codes_dev & 7u) ||
        ((uintptr_t)k_codes_dev & 7u) || ((uintptr_t)v_codes_dev & 7u) || ((uintptr_t)ws_dev & 255u))
        return SA_ERR_INVALID_ARG;
    QkvWs w = qkv_ws_layout(ws_dev, B, H, N, D);
    if (ws_bytes < w.bytes) return SA_ERR_WORKSPACE;
    const int BH = B * H, T = sa_cdiv(N, kTile);

    if (cudaMemsetAsync(w.amax, 0, w.zero_bytes, stream) != cudaSuccess) return SA_ERR_CUDA;

    PrepassParams p{};
    p.q = (const uint4*)q_dev;
    p.k = (const uint4*)k_dev;
    p.v = (const uint4*)v_dev;
    p.BH = BH;
    p.N = N;
    p.T = T;
    p.smooth_k = smooth_k ? 1 : 0;
    p.amax = w.amax;
    p.ticket = w.ticket;
    p.psum = w.psum;
    p.pmax = w.pmax;
    p.pmin = w.pmin;
    p.kmean = k_mean_dev ? k_mean_dev : w.kmean;
    const size_t n16 = (size_t)BH * N * D / 8;
    // one batch of kAmaxPer 16-byte loads per amax thread
    p.nA = (int)std::max<size_t>((n16 + 256 * kAmaxPer - 1) / (256 * kAmaxPer), 1);
    p.nKS = BH * T;
    p.qc = (uint2*)q_codes_dev;
    p.qs = q_scales_dev;
    p.qg = q_g_dev;
    p.kc = (uint2*)k_codes_dev;
    p.ks = k_scales_dev;
    p.kg = k_g_dev;
    p.vc = v_codes_dev;
    p.vs = v_scales_dev;
    p.vg = v_g_dev;
    p.f_lo = f_lo;
    p.f_hi = f_hi;

    const unsigned gs = (unsigned)(2 * p.nA + (p.smooth_k ? p.nKS : p.nA));
    const size_t ks_smem = (size_t)kTile * D * 2;  // one K tile (smoothing blocks)
    if (D == 128)
        prepass_stats_kernel<128><<<gs, 256, ks_smem, stream>>>(p);
    else
        prepass_stats_kernel<64><<<gs, 256, ks_smem, stream>>>(p);
    SA_CHECK_LAUNCH();
    const bool ss = mode == SA_SCALE_SEARCH, sm = p.smooth_k != 0;
    // persistent: as many CTAs as fit on the GPU, each double-buffering tiles
#define SA_PQ(DD, SS, SM)                                                                                      \
    do {                                                                                                       \
        const int smem = (int)sizeof(PqSmem<DD>);                                                              \
        /* set on a device's first call, outside any stream capture */                                      \
        static PerDevice per_sm_cache;                                                                         \
        const int per_sm = once_per_device(per_sm_cache, [&] {                                                 \
            int n = 0;                                                                                         \
            if (cudaFuncSetAttribute(prepass_quant_kernel<DD, SS, SM>,                                         \
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||      \
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prepass_quant_kernel<DD, SS, SM>, 2 * DD,    \
                                                              smem) != cudaSuccess)                            \
                return 0;                                                                                      \
            return n;                                                                                          \
        });                                                                                                    \
        if (per_sm < 1) return SA_ERR_CUDA;                                                                    \
        const unsigned gq = (unsigned)std::min<long>(3L * BH * T, (long)per_sm * sm_count());                  \
        prepass_quant_kernel<DD, SS, SM><<<gq, 2 * DD, smem, stream>>>(p);                                     \
    } while (0)
    if (D == 128) {
        if (ss) { if (sm) SA_PQ(128, true, true); else SA_PQ(128, true, false); }
        else { if (sm) SA_PQ(128, false, true); else SA_PQ(128, false, false); }
    } else {
        if (ss) { if (sm) SA_PQ(64, true, true); else SA_PQ(64, true, false); }
        else { if (sm) SA_PQ(64, false, true); else SA_PQ(64, false, false); }
    }
#undef SA_PQ
    SA_CHECK_LAUNCH();
    return SA_OK;
}

size_t sa_select_workspace_size(int B, int H, int N, int D)
{
    if (B < 0 || H < 0 || N < 0 || D < 0) return 0;
    return select_ws_bytes(B, H, N, D);
}

sa_status sa_thrift_select_ex(const void* q_dev, const void* k_dev, const float* k_mean_dev, int B, int H, int N,
                              int D, int causal, int frac_bp, int per_row, uint8_t* mask_dev, int32_t* nsel_dev,
                              void* ws_dev, size_t ws_bytes, cudaStream_t stream)
{
    if (B < 0 || H < 0 || N < 0 || frac_bp < 0 || frac_bp > 10000) return SA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
    if ((size_t)B * H * N == 0) return SA_OK;
    if (!q_dev || !k_dev || !mask_dev || !ws_dev) return SA_ERR_INVALID_ARG;
    if ((uintptr_t)ws_dev & 255u) return SA_ERR_INVALID_ARG;
    if (ws_bytes < select_ws_bytes(B, H, N, D)) return SA_ERR_WORKSPACE;
    const int T = sa_cdiv(N, 128);
    const size_t BH = (size_t)B * H;
    float* qbar = (float*)ws_dev;
    float* kbar = (float*)((char*)ws_dev + sa_align256(BH * T * D * sizeof(float)));
    float* scores = (float*)((char*)ws_dev + 2 * sa_align256(BH * T * D * sizeof(float)));
    pool_kernel<<<dim3(T, (unsigned)BH, 2), 128, 0, stream>>>((const uint16_t*)q_dev, (const uint16_t*)k_dev,
                                                             k_mean_dev, N, D, T, qbar, kbar);
    SA_CHECK_LAUNCH();
    score_kernel<<<dim3(sa_cdiv(T, 32), sa_cdiv(T, 8), (unsigned)BH), 256, 0, stream>>>(qbar, kbar, D, T, scores);
    SA_CHECK_LAUNCH();
    if (per_row) {
        if (nsel_dev && cudaMemsetAsync(nsel_dev, 0, BH * sizeof(int32_t), stream) != cudaSuccess) return SA_ERR_CUDA;
        const size_t rows = BH * (size_t)T;
        topk_row_kernel<<<(unsigned)((rows + kRowWarps - 1) / kRowWarps), 32 * kRowWarps, 0, stream>>>(
            scores, (int)BH, T, causal, frac_bp, mask_dev, nsel_dev);
    } else {
        topk_kernel<<<(unsigned)BH, kTopkThreads, 0, stream>>>(scores, T, causal, frac_bp, mask_dev, nsel_dev);
    }
    SA_CHECK_LAUNCH();
    return SA_OK;
}

sa_status sa_thrift_select(const void* q_dev, const void* k_dev, int B, int H, int N, int D, int causal,
                           int frac_bp, uint8_t* mask_dev, int32_t* nsel_dev, void* ws_dev, size_t ws_bytes,
                           cudaStream_t stream)
{
    return sa_thrift_select_ex(q_dev, k_dev, nullptr, B, H, N, D, causal, frac_bp, 0, mask_dev, nsel_dev, ws_dev,
                               ws_bytes, stream);
}

sa_status sa_attn_fwd_ex(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev, const float* q_g_dev,
                         const uint8_t* k_codes_dev, const uint8_t* k_scales_dev, const float* k_g_dev,
                         const uint8_t* v_codes_dev, const uint8_t* v_scales_dev, const float* v_g_dev, int B, int H,
                         int N, int D, int causal, float sm_scale, int p_mode, const uint8_t* mask_dev,
                         const void* q_bf16_dev, const void* k_bf16_dev, const void* v_bf16_dev,
                         const float* k_mean_dev, float* out_dev, float* lse_dev, cudaStream_t stream)
{
    if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
    if (p_mode != SA_SCALE_MAX && p_mode != SA_SCALE_SEARCH) return SA_ERR_INVALID_ARG;
    if (p_mode == SA_SCALE_SEARCH && mask_dev) return SA_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
    if (N % 32) return SA_ERR_INVALID_ARG;
    if ((size_t)B * H * N == 0) return SA_OK;
    if (!q_codes_dev || !q_scales_dev || !q_g_dev || !k_codes_dev || !k_scales_dev || !k_g_dev || !v_codes_dev ||
        !v_scales_dev || !v_g_dev || !out_dev)
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q_codes_dev) || !aligned16(k_codes_dev) || !aligned16(v_codes_dev) || !aligned16(q_scales_dev) ||
        !aligned16(k_scales_dev) || !aligned16(v_scales_dev) || !aligned16(out_dev))
        return SA_ERR_INVALID_ARG;
    const bool mixed = mask_dev != nullptr;
    if (mixed && (!q_bf16_dev || !k_bf16_dev || !v_bf16_dev || !aligned16(q_bf16_dev) || !aligned16(k_bf16_dev) ||
                  !aligned16(v_bf16_dev)))
        return SA_ERR_INVALID_ARG;
    if (!(sm_scale > 0.0f)) sm_scale = 1.0f / sqrtf((float)D);
    const uint64_t BH = (uint64_t)B * H;
    const CUtensorMapSwizzle qsw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    CUtensorMap tq, tk, tv, tqb, tkb, tvb;
    if (!make_map_u8(&tq, q_codes_dev, D / 2, N, BH, D / 2, 128, qsw) ||
        !make_map_u8(&tk, k_codes_dev, D / 2, N, BH, D / 2, 128, qsw) ||
        !make_map_u8(&tv, v_codes_dev, 64, (uint64_t)D * sa_cdiv(N, 128), BH, 64, D, CU_TENSOR_MAP_SWIZZLE_64B))
        return SA_ERR_CUDA;
    if (mixed) {
        if (!make_map_bf16(&tqb, q_bf16_dev, D, N, BH) || !make_map_bf16(&tkb, k_bf16_dev, D, N, BH) ||
            !make_map_bf16(&tvb, v_bf16_dev, D, N, BH))
            return SA_ERR_CUDA;
    } else {
        tqb = tq;
        tkb = tk;
        tvb = tv;
    }
    AttnParams p{};
    p.q_sf = q_scales_dev;
    p.k_sf = k_scales_dev;
    p.v_sf = v_scales_dev;
    p.q_g = q_g_dev;
    p.k_g = k_g_dev;
    p.v_g = v_g_dev;
    p.out = out_dev;
    p.lse = lse_dev;
    p.N = N;
    p.H = H;
    p.B = B;
    p.T = sa_cdiv(N, 128);
    p.CKv = sa_cdiv(N, 64);
    p.causal = causal ? 1 : 0;
    p.sm_scale = sm_scale;
    p.mask = mask_dev;
    p.q_bf16 = (const uint16_t*)q_bf16_dev;
    p.k_mean = k_mean_dev;
    const long long wc = g_wait_cycles.load(std::memory_order_relaxed);
    p.wait_cycles = wc > 0 ? wc : SA_WAIT_CYCLES;
    const long nitems = (long)B * H * ((p.T + 1) / 2);
    const int nsm = sm_count();
    if (nsm <= 0) return SA_ERR_CUDA;
    const unsigned grid = (unsigned)(nitems < nsm ? nitems : nsm);  // persistent: one CTA per SM
#define SA_ATTN_LAUNCH(DD, MX, PS)                                                                          \
    do {                                                                                                    \
        const int smem = (int)sizeof(PpSmem<DD, MX>) + 1024;                                                \
        static PerDevice attr; /* set on a device's first call, outside any stream capture */              \
        if (!allow_smem(attr, attn_fwd_pp_kernel<DD, MX, PS>, smem)) return SA_ERR_CUDA;                    \
        static PerDevice regs_ok; /* the kernel's register split must fit its launch allocation */         \
        if (once_per_device(regs_ok, [] { return pp_regs_fit(attn_fwd_pp_kernel<DD, MX, PS>) ? 1 : 0; }) <= 0) \
            return SA_ERR_UNSUPPORTED;                                                                      \
        attn_fwd_pp_kernel<DD, MX, PS><<<grid, kPpThreads, smem, stream>>>(tq, tk, tv, tqb, tkb, tvb, p);   \
    } while (0)
    const bool ps = p_mode == SA_SCALE_SEARCH;
    if (D == 128) {
        if (mixed) SA_ATTN_LAUNCH(128, true, false);
        else if (ps) SA_ATTN_LAUNCH(128, false, true);
        else SA_ATTN_LAUNCH(128, false, false);
    } else {
        if (mixed) SA_ATTN_LAUNCH(64, true, false);
        else if (ps) SA_ATTN_LAUNCH(64, false, true);
        else SA_ATTN_LAUNCH(64, false, false);
    }
#undef SA_ATTN_LAUNCH
    SA_CHECK_LAUNCH();
    return SA_OK;
}

sa_status sa_attn_fwd(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev, const float* q_g_dev,
                      const uint8_t* k_codes_dev, const uint8_t* k_scales_dev, const float* k_g_dev,
                      const uint8_t* v_codes_dev, const uint8_t* v_scales_dev, const float* v_g_dev, int B, int H,
                      int N, int D, int causal, float sm_scale, const uint8_t* mask_dev, const void* q_bf16_dev,
                      const void* k_bf16_dev, const void* v_bf16_dev, const float* k_mean_dev, float* out_dev,
                      float* lse_dev, cudaStream_t stream)
{
    return sa_attn_fwd_ex(q_codes_dev, q_scales_dev, q_g_dev, k_codes_dev, k_scales_dev, k_g_dev, v_codes_dev,
                          v_scales_dev, v_g_dev, B, H, N, D, causal, sm_scale, SA_SCALE_MAX, mask_dev, q_bf16_dev,
                          k_bf16_dev, v_bf16_dev, k_mean_dev, out_dev, lse_dev, stream);
}

size_t sa_decode_workspace_size(int B, int Hq, int Hkv, int L, int D)
{
    if (B < 0 || Hq < 0 || Hkv <= 0 || L < 0 || D < 0) return 0;
    const int nsplit = sa_cdiv(L, kSplit);
    return 256 + sa_align256((size_t)B * Hq * nsplit * (D + 2) * sizeof(float));
}

sa_status sa_attn_decode_kvfp4_sink(const void* q_dev, const uint8_t* k_codes_dev, const uint8_t* k_scales_dev,
                                    const float* k_g_dev, const uint8_t* v_codes_dev, const uint8_t* v_scales_dev,
                                    const float* v_g_dev, int B, int Hq, int Hkv, int L, int D, float sm_scale,
                                    int sink_first, int sink_last, const void* k_sink_dev, const void* v_sink_dev,
                                    const float* k_mean_dev, float* out_dev, void* ws_dev, size_t ws_bytes,
                                    cudaStream_t stream)
{
    if (B < 0 || Hq < 0 || Hkv <= 0 || L < 0) return SA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SA_ERR_UNSUPPORTED;
    if (Hq % Hkv || Hq / Hkv > kDecN || L % 128) return SA_ERR_INVALID_ARG;
    if (sink_first < 0 || sink_last < 0 || (long)(sink_first + (long)sink_last) * 128 > L) return SA_ERR_INVALID_ARG;
    const bool sink = sink_first > 0 || sink_last > 0;
    if ((size_t)B * Hq == 0) return SA_OK;
    if (L == 0) return SA_ERR_INVALID_ARG;
    if (!q_dev || !k_codes_dev || !k_scales_dev || !k_g_dev || !v_codes_dev || !v_scales_dev || !v_g_dev ||
        !out_dev || !ws_dev)
        return SA_ERR_INVALID_ARG;
    if (sink && (!k_sink_dev || !v_sink_dev || !aligned16(k_sink_dev) || !aligned16(v_sink_dev) ||
                 ((uintptr_t)k_mean_dev & 15u)))
        return SA_ERR_INVALID_ARG;
    if (!aligned16(q_dev) || !aligned16(k_codes_dev) || !aligned16(v_codes_dev) || !aligned16(k_scales_dev) ||
        !aligned16(v_scales_dev) || ((uintptr_t)ws_dev & 255u))
        return SA_ERR_INVALID_ARG;
    if (ws_bytes < sa_decode_workspace_size(B, Hq, Hkv, L, D)) return SA_ERR_WORKSPACE;
    if (!(sm_scale > 0.0f)) sm_scale = 1.0f / sqrtf((float)D);
    const uint64_t BHk = (uint64_t)B * Hkv;
    const int nsplit = sa_cdiv(L, kSplit);
    unsigned* amax = (unsigned*)ws_dev;
    float* part = (float*)((char*)ws_dev + 256);
    if (cudaMemsetAsync(amax, 0, 4, stream) != cudaSuccess) return SA_ERR_CUDA;
    size_t n16 = (size_t)B * Hq * D / 8;
    amax_bf16_kernel<<<grid_for(n16, 256), 256, 0, stream>>>((const uint4*)q_dev, n16, amax);
    SA_CHECK_LAUNCH();
    const CUtensorMapSwizzle ksw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    CUtensorMap tk, tv;
    if (!make_map_u8(&tk, k_codes_dev, D / 2, L, BHk, D / 2, 128, ksw) ||
        !make_map_u8(&tv, v_codes_dev, 64, (uint64_t)D * sa_cdiv(L, 128), BHk, 64, D, CU_TENSOR_MAP_SWIZZLE_64B))
        return SA_ERR_CUDA;
    DecParams p{};
    p.q = (const uint16_t*)q_dev;
    p.q_amax = amax;
    p.k_sf = k_scales_dev;
    p.v_sf = v_scales_dev;
    p.k_g = k_g_dev;
    p.v_g = v_g_dev;
    p.part = part;
    p.L = L;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.nsplit = nsplit;
    p.RTk = sa_cdiv(L, 128);
    p.CKv = sa_cdiv(L, 64);
    p.sm_scale = sm_scale;
    if (sink) {
        p.k_sink = (const uint16_t*)k_sink_dev;
        p.v_sink = (const uint16_t*)v_sink_dev;
        p.k_mean = k_mean_dev;
        p.sink_first = sink_first;
        p.sink_last = sink_last;
        p.NS = 128 * (sink_first + sink_last);
    }
    dim3 grid(nsplit, Hkv, B);
    if (D == 128) {
        const int smem = (int)sizeof(DecSmem<128>) + 1024;
        if (sink) {
            static PerDevice attr;
            if (!allow_smem(attr, decode_kernel<128, true>, smem)) return SA_ERR_CUDA;
            decode_kernel<128, true><<<grid, 128, smem, stream>>>(tk, tv, p);
        } else {
            static PerDevice attr;
            if (!allow_smem(attr, decode_kernel<128, false>, smem)) return SA_ERR_CUDA;
            decode_kernel<128, false><<<grid, 128, smem, stream>>>(tk, tv, p);
        }
    } else {
        const int smem = (int)sizeof(DecSmem<64>) + 1024;
        if (sink) {
            static PerDevice attr;
            if (!allow_smem(attr, decode_kernel<64, true>, smem)) return SA_ERR_CUDA;
            decode_kernel<64, true><<<grid, 128, smem, stream>>>(tk, tv, p);
        } else {
            static PerDevice attr;
            if (!allow_smem(attr, decode_kernel<64, false>, smem)) return SA_ERR_CUDA;
            decode_kernel<64, false><<<grid, 128, smem, stream>>>(tk, tv, p);
        }
    }
    SA_CHECK_LAUNCH();
    decode_combine_kernel<<<(unsigned)(B * Hq), 128, 0, stream>>>(part, nsplit, D, v_g_dev, out_dev);
    SA_CHECK_LAUNCH();
    return SA_OK;
}

sa_status sa_attn_decode_kvfp4(const void* q_dev, const uint8_t* k_codes_dev, const uint8_t* k_scales_dev,
                               const float* k_g_dev, const uint8_t* v_codes_dev, const uint8_t* v_scales_dev,
                               const float* v_g_dev, int B, int Hq, int Hkv, int L, int D, float sm_scale,
                               float* out_dev, void* ws_dev, size_t ws_bytes, cudaStream_t stream)
{
    return sa_attn_decode_kvfp4_sink(q_dev, k_codes_dev, k_scales_dev, k_g_dev, v_codes_dev, v_scales_dev, v_g_dev, B,
                                     Hq, Hkv, L, D, sm_scale, 0, 0, nullptr, nullptr, nullptr, out_dev, ws_dev,
                                     ws_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// sa_quant_nvfp4_noalloc: the pre-pass with library-owned scratch.
// The scratch is a file-scope device array in this module (every GPU that
// loads the module keeps it until the process exits).  Host code cannot pass
// the array's name to a kernel (on the host it names a stand-in object, not
// device memory), so each device's address is looked up once with
// cudaGetSymbolAddress while that device is current.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
// per device: the scratch address and the context it was resolved in (a
// device reset creates a new context, where the module and its array may sit
// elsewhere, so the address is looked up again)
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
CUcontext g_noalloc_ctx[kNoAllocMaxDevices] = {};

// The current driver context, through the runtime's driver entry point (no
// link-time dependency on the driver library); null if unavailable.
CUcontext current_context()
{
    using Fn = CUresult (*)(CUcontext*);
    static const Fn fn = [] {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<Fn>(ptr);
        return (Fn) nullptr;
    }();
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}
}  // namespace

extern "C" sa_status sa_quant_nvfp4_noalloc(const void* x_dev, int B, int H, int N, int D, sa_role role, int smooth,
                                            sa_scale_mode mode, int f_lo, int f_hi, uint8_t* codes_dev,
                                            uint8_t* scales_dev, float* g_dev, float* k_mean_dev,
                                            int8_t* ss_off_dev, cudaStream_t stream)
{
    if (B < 0 || H < 0 || N < 0 || D < 0) return SA_ERR_INVALID_ARG;
    if (role != SA_ROLE_Q && role != SA_ROLE_K && role != SA_ROLE_V) return SA_ERR_INVALID_ARG;
    // size check first: nothing is launched or dereferenced for a call that
    // does not fit the scratch
    if (sa_quant_workspace_size(B, H, N, D, role) > kNoAllocScratchBytes) return SA_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return SA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        const CUcontext ctx = current_context();
        if (!g_noalloc_ptr[dev] || !ctx || ctx != g_noalloc_ctx[dev]) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
                cudaGetLastError();
                return SA_ERR_CUDA;
            }
            g_noalloc_ptr[dev] = ptr;
            g_noalloc_ctx[dev] = ctx;
        }
        scratch = g_noalloc_ptr[dev];
    }
    // the allocating entry point clears the parts of the workspace that must
    // start at zero (the amax word) on `stream` before its kernels use them
    return sa_quant_nvfp4(x_dev, B, H, N, D, role, smooth, mode, f_lo, f_hi, codes_dev, scales_dev, g_dev,
                          k_mean_dev, ss_off_dev, scratch, kNoAllocScratchBytes, stream);
}
