/*
 * sa.h -- C ABI of the B200-native NVFP4 attention library (libsa.so).
 *
 * Method (web pages this follows, cited by title and section):
 *  - "Search Your Block Floating Point Scales!" (gist.science summary):
 *    NVFP4 microscaling with an E4M3 block scale ("특수 하드웨어: NVFP4",
 *    "문제 제기"); max-scaling s = round(max|x|/6) and ScaleSearch over
 *    integer offsets of the E4M3 scale byte ("방법론 / ScaleSearch");
 *    ScaleSearchAttention runs Q K^T and P V natively in NVFP4 with FP32
 *    accumulation and keeps a 4-bit KV cache ("ScaleSearchAttention").
 *  - "SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
 *    Acceleration" (hotpaper.ai), "기술적 접근법": per-channel smoothing of K.
 *  - SageAttention3 article (dasgeld.co): microscaling FP4 attention on
 *    Blackwell FP4 tensor cores.
 *  - "ThriftAttention: 5%의 연산량으로 90%의 품질 유지" (molayo1419.me):
 *    about 5 % of query-key blocks in high precision, one joint softmax.
 *
 * Conventions (all entry points):
 *  - The caller owns every buffer; the library never allocates device memory.
 *    Pointers named *_dev are device pointers; everything else is host data
 *    passed by value.
 *  - Every call is asynchronous on `stream` and does not synchronise, except
 *    sa_device_status().  Argument errors are reported before any launch;
 *    launch failures return SA_ERR_CUDA.  Device-side conditions (non-finite
 *    input, a pipeline wait that gave up) are recorded in a library status
 *    word that sa_device_status() reads.
 *  - Host threads may call the entry points concurrently (each call with its
 *    own buffers, workspace and stream); the library's only process-wide
 *    state is per-kernel attribute and per-device caches, set race-free on
 *    first use.  sa_quant_nvfp4_noalloc is the exception: its calls share one
 *    scratch per device and must not overlap.
 *  - bf16 tensors are dense row-major [B, H, N, D].
 *  - Sizes: D in {64, 128}; N >= 1 with N % 16 == 0 (16 = NVFP4 block).
 *    B = 0 or H = 0 is a valid empty call that launches nothing.
 *
 * NVFP4 storage (per tensor):
 *  - g: device float[2] = {g, 1/g}, g = amax / 2688 (2688 = 6 * 448: the
 *    tensor amax maps onto the largest E2M1 element times the largest E4M3
 *    scale); an all-zero tensor has g = 1.
 *  - codes: E2M1 nibbles, two per byte, even element in the low nibble.
 *    Q and K: [B, H, N, D/2] (blocks of 16 consecutive channels of a token).
 *    V:       blocks of 16 consecutive tokens of a channel (the key axis is
 *    the reduction axis of P V, the only axis a block-scaled MMA can scale
 *    along), stored in 128-token tiles [B, H, ceil(N/128), D, 64]: byte
 *    ((b*H + h)*ceil(N/128) + n/128)*D*64 + d*64 + (n%128)/2 holds tokens n, n+1
 *    (n even) of channel d, so each tile's V^T block is one contiguous
 *    D x 64-byte region.  Bytes past token N in the last tile are unspecified.
 *    Size: sa_codes_bytes().
 *  - scales: E4M3 bytes, one per block, in the tensor-core "atom" layout.
 *    View each (b, h) slice as a matrix with R rows and C block-running
 *    columns (Q, K: R = N, C = D; V: R = D, C = N).  Rows are grouped into
 *    tiles of 128 (RT = ceil(R/128)) and columns into chunks of 64 elements
 *    (CK = ceil(C/64), four blocks).  Each (row tile, chunk) is a 512-byte
 *    atom at index ((b*H + h)*RT + rt)*CK + ck; inside it, the scale of row r
 *    (0..127 within the tile) and block j (0..3 within the chunk) is byte
 *    (r % 32)*16 + (r / 32)*4 + j.  Padding bytes are 0.  Total size:
 *    sa_scales_bytes().  (A 32x128-bit tcgen05.cp moves one atom into tensor
 *    memory unchanged.)
 */
#ifndef SA_H
#define SA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,   /* null pointer, bad size or mode */
    SA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. D not 64/128) */
    SA_ERR_WORKSPACE = 3,     /* workspace smaller than the *_workspace_size() */
    SA_ERR_NONFINITE = 4,     /* device: input held inf or NaN */
    SA_ERR_CUDA = 5,          /* a CUDA call or launch failed */
    SA_ERR_TIMEOUT = 6,       /* device: a pipeline wait gave up (bounded) */
    SA_ERR_DEVICE_ASSERT = 7  /* device: an internal consistency check failed */
} sa_status;

typedef enum { SA_ROLE_Q = 0, SA_ROLE_K = 1, SA_ROLE_V = 2 } sa_role;
typedef enum { SA_SCALE_MAX = 0, SA_SCALE_SEARCH = 1 } sa_scale_mode;

/* Human-readable name of a status code (static string). */
const char* sa_status_string(sa_status s);

/* Synchronises `stream`, then returns the device status word recorded by
 * earlier calls (SA_OK if none) and clears it when `reset` != 0. */
sa_status sa_device_status(cudaStream_t stream, int reset);

/* Limit, in SM clock cycles, of every pipeline wait inside sa_attn_fwd's
 * kernel, for the calls made after it (process-wide); cycles <= 0 restores
 * the default (about 2 s at the B200 clock).  A wait that reaches the limit
 * records SA_ERR_TIMEOUT, every warp of the CTA unwinds, copies and
 * tensor-core work already issued are waited for, and the kernel returns;
 * the output of that call is then undefined, and later calls run normally.
 * A short limit (hundreds of cycles, below one copy's latency) makes a call
 * give up on purpose, which is how the timeout path is tested. */
void sa_set_wait_cycles(long long cycles);

/* Byte sizes of the NVFP4 code and scale buffers of one tensor. */
size_t sa_codes_bytes(int B, int H, int N, int D, sa_role role);
size_t sa_scales_bytes(int B, int H, int N, int D, sa_role role);

/* ------------------------------------------------------------------------
 * sa_quant_nvfp4 -- smoothing + NVFP4 quantisation pre-pass.
 * "Search Your Block Floating Point Scales!", "방법론 / ScaleSearch"
 * ("메커니즘", "검색 전략"); "SageAttention", "기술적 접근법" (smoothing).
 *
 *  x_dev       bf16 [B,H,N,D] input.
 *  role        Q, K or V (V is written token-blocked and transposed).
 *  smooth      K only: subtract the per-(b,h,channel) mean over tokens
 *              (FP64 sum: tokens ascending inside 128-token tiles, then the
 *              tile partials ascending; rounded to FP32) before quantising.
 *  mode        SA_SCALE_MAX: block scale E4M3(max|x~|/6), x~ = x'/g.
 *              SA_SCALE_SEARCH: try scale bytes c0+f for f in [f_lo, f_hi)
 *              (f = 0 always included and preferred on ties, then the lowest
 *              f); keep the lowest block squared error in the x~ domain
 *              (FP32, two interleaved fmaf accumulators).  Requires
 *              -16 <= f_lo <= 0 < f_hi <= 16.
 *  codes_dev   sa_codes_bytes() bytes, written.
 *  scales_dev  sa_scales_bytes() bytes, written (padding zeroed).
 *  g_dev       float[2] {g, 1/g}, written.
 *  k_mean_dev  float [B,H,D] channel means (written when smooth), may be NULL.
 *  ss_off_dev  int8, one per block in the logical row-major block layout
 *              ([B,H,N,D/16] for Q/K, [B,H,D,N/16] for V): the chosen f
 *              (0 in max mode).  May be NULL.
 *  ws_dev      scratch of sa_quant_workspace_size() bytes (256-byte aligned).
 * Rounding: every scale and code decision is IEEE FP32 round-to-nearest-
 * even exactly as stated, so results are bit-exact across runs and devices.
 * ------------------------------------------------------------------------ */
size_t sa_quant_workspace_size(int B, int H, int N, int D, sa_role role);
sa_status sa_quant_nvfp4(const void* x_dev, int B, int H, int N, int D, sa_role role, int smooth,
                         sa_scale_mode mode, int f_lo, int f_hi, uint8_t* codes_dev, uint8_t* scales_dev,
                         float* g_dev, float* k_mean_dev, int8_t* ss_off_dev, void* ws_dev, size_t ws_bytes,
                         cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_quant_nvfp4_qkv -- the pre-pass of a whole attention call: Q, K and V of
 * one shape in two kernel launches (one for the statistics of all three
 * tensors, one for their quantisation) instead of up to three each.
 * Same operation, arguments and bit-identical outputs as calling
 * sa_quant_nvfp4 for role Q (smooth 0), K (smooth = smooth_k) and V with the
 * same mode and offsets; no ScaleSearch offset outputs.
 *  q_dev, k_dev, v_dev   bf16 [B,H,N,D] inputs, 16-byte aligned.
 *  *_codes, *_scales, *_g   outputs as sa_quant_nvfp4 for each role (codes
 *              8-byte aligned).
 *  k_mean_dev  float [B,H,D] channel means of K (written when smooth_k), may
 *              be NULL.
 *  ws_dev      scratch of sa_quant_qkv_workspace_size() bytes (256-byte
 *              aligned); the call resets the part it needs with one
 *              cudaMemsetAsync on the stream.
 * The quantisation kernel is persistent over 128-row tiles.  The first call
 * in a process also sets its shared-memory attribute and reads its occupancy
 * (host-side, no stream work); make that first call outside any stream
 * capture (later calls may be captured into a CUDA graph).
 * Errors: as sa_quant_nvfp4 (argument errors before any launch; non-finite
 * input in any of the three tensors -> SA_ERR_NONFINITE in the status word).
 * ------------------------------------------------------------------------ */
size_t sa_quant_qkv_workspace_size(int B, int H, int N, int D);
sa_status sa_quant_nvfp4_qkv(const void* q_dev, const void* k_dev, const void* v_dev, int B, int H, int N, int D,
                             int smooth_k, sa_scale_mode mode, int f_lo, int f_hi, uint8_t* q_codes_dev,
                             uint8_t* q_scales_dev, float* q_g_dev, uint8_t* k_codes_dev, uint8_t* k_scales_dev,
                             float* k_g_dev, float* k_mean_dev, uint8_t* v_codes_dev, uint8_t* v_scales_dev,
                             float* v_g_dev, void* ws_dev, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_quant_nvfp4_noalloc -- sa_quant_nvfp4 without a caller workspace.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory: hosts whose device memory is all owned
 * by a fixed pool or an external allocator, plug-ins that are handed buffers
 * but no allocator, and latency-critical loops where the device-wide
 * synchronisation of cudaMalloc/cudaFree is not allowed.
 * Such a caller passes only its inputs and outputs (same meaning, layout and
 * results as sa_quant_nvfp4); the scratch is an 8 MiB array inside libsa,
 * held on every GPU that loads the library until the process exits.
 *  - Limit: sa_quant_workspace_size(B,H,N,D,role) must be <= 8 MiB, else
 *    SA_ERR_WORKSPACE is returned before anything is launched.  Q and V need
 *    256 bytes.  K needs 256 + a(8*B*H*T*D) + 2*a(4*B*H*T*D) + a(4*B*H*D)
 *    bytes, T = ceil(N/128) and a() rounding up to a multiple of 256 (about
 *    16*B*H*T*D bytes: at D = 128, B*H*T up to about 4080, the exact figure
 *    depending on B*H; sa_quant_workspace_size gives it for any shape).
 *  - The first call on a device (and the first after a reset of that device)
 *    looks up the scratch address for the device's current context
 *    (cudaGetSymbolAddress, with the device current); make that call before
 *    any stream capture.
 *  - Calls share the scratch and it keeps the last call's contents; the call
 *    clears what must start at zero.  Calls that overlap on the GPU (for
 *    example on two streams at once) race: serialise them.
 *  - Allocates nothing: no cudaMalloc/cudaFree and no allocating library.
 * ------------------------------------------------------------------------ */
sa_status sa_quant_nvfp4_noalloc(const void* x_dev, int B, int H, int N, int D, sa_role role, int smooth,
                                 sa_scale_mode mode, int f_lo, int f_hi, uint8_t* codes_dev, uint8_t* scales_dev,
                                 float* g_dev, float* k_mean_dev, int8_t* ss_off_dev, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_thrift_select -- pick the high-precision (query tile, key tile) blocks.
 * "ThriftAttention: 5%의 연산량으로 90%의 품질 유지" (the share of blocks and
 * the joint softmax; the page does not define the selector, so a mean-pooled
 * score is used): for each 128-row tile t, qbar_t[c] = bf16(FP32 sum of the
 * rows in ascending order / row count), kbar_u likewise from raw K; score =
 * FP32 fmaf chain over c ascending of qbar_t[c]*kbar_u[c].  Valid blocks: all,
 * or u <= t when causal.  Per (b,h) the top ceil(n_valid*frac_bp/10000)
 * blocks by (score descending, t*T+u ascending) are selected.
 *
 *  q_dev, k_dev   bf16 [B,H,N,D].
 *  frac_bp        budget in basis points (500 = 5 %), 0..10000.
 *  mask_dev       uint8 [B,H,T,T], T = ceil(N/128): 1 = high precision.
 *  nsel_dev       int32 [B,H] selected counts, may be NULL.
 *  ws_dev         sa_select_workspace_size() bytes.
 * ------------------------------------------------------------------------ */
size_t sa_select_workspace_size(int B, int H, int N, int D);
sa_status sa_thrift_select(const void* q_dev, const void* k_dev, int B, int H, int N, int D, int causal,
                           int frac_bp, uint8_t* mask_dev, int32_t* nsel_dev, void* ws_dev, size_t ws_bytes,
                           cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_thrift_select_ex -- sa_thrift_select with two further readings of the
 * selector that "ThriftAttention" leaves open (the page fixes only the share
 * of high-precision blocks and the joint softmax):
 *  k_mean_dev   NULL: pool raw K (as sa_thrift_select).  Else float [B,H,D]
 *               channel means (the K pre-pass output): each key row is pooled
 *               as fl(k - mu_c), the smoothed keys the NVFP4 path quantises.
 *  per_row      0: one budget per (b,h) over all valid blocks (as
 *               sa_thrift_select).  1: one budget per query tile t,
 *               ceil(n_valid_t*frac_bp/10000) of its valid key tiles (u <= t
 *               when causal), by (score descending, u ascending); nsel_dev
 *               (if not NULL) receives the per-(b,h) total.
 * Other arguments, workspace and errors as sa_thrift_select.
 * ------------------------------------------------------------------------ */
sa_status sa_thrift_select_ex(const void* q_dev, const void* k_dev, const float* k_mean_dev, int B, int H, int N,
                              int D, int causal, int frac_bp, int per_row, uint8_t* mask_dev, int32_t* nsel_dev,
                              void* ws_dev, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_quant_nvfp4_ip -- incoherence processing of Q and K, then their NVFP4
 * pre-pass ("Search Your Block Floating Point Scales!", "ScaleSearchAttention",
 * 비일관성 처리 (IP) 및 크기 감소: a Hadamard rotation with random signs, as in
 * QuIP#, and a linear pair Q' = Q R^-T, K' = K R that keeps every score).
 * Reading: Q~ = Q H S, K~ = (K - mu) H S (H the orthonormal Sylvester
 * Hadamard matrix, S = diag(signs), mu the K channel mean when smooth), R
 * diagonal with r_c = (sum_t q~_tc^2 / sum_t k~_tc^2)^(1/4) (1 when a sum is
 * 0), Q' = Q~ R^-1, K' = K~ R; Q'K'^T = Q (K - mu)^T.  Arithmetic: the
 * rotation in FP32 as the fast Walsh-Hadamard butterfly, then times
 * fl32(1/sqrt(D)) and the sign; the sums of squares in FP64 (rows ascending
 * inside 128-row tiles, then tiles ascending); r and 1/r in FP64;
 * Q' = fl32(y (1/r)), K' = fl32(y r).  Q' and K' are each quantised like a Q tensor (own tensor
 * scale g = amax/2688, 16-channel blocks, max-scaling or ScaleSearch, no
 * further smoothing) into the Q/K layouts of sa_quant_nvfp4; the attention
 * consumes them unchanged (sa_attn_fwd with V quantised as usual).
 *
 *  q_dev, k_dev    bf16 [B,H,N,D], 16-byte aligned; D = 64 or 128;
 *                  N % 16 == 0; B*H <= 65535.
 *  signs_dev       int8 [D] of +1 / -1 (device memory; a negative entry is -1).
 *  smooth          1: subtract the K channel mean before the rotation.
 *  mode, f_lo,
 *  f_hi            block rule, as sa_quant_nvfp4.
 *  q_* / k_*       codes, scale atoms and {g, 1/g} of Q' and of K', sized and
 *                  laid out as sa_quant_nvfp4's role-Q outputs.
 *  k_mean_dev      FP32 [B,H,D] receives mu when smooth (may be NULL).
 *  r_dev           FP32 [B,H,D] receives fl32(r) (may be NULL).
 *  q_ss_off_dev,
 *  k_ss_off_dev    int8 [B,H,N,D/16] ScaleSearch offsets, or NULL.
 *  ws_dev          sa_quant_ip_workspace_size() bytes, 256-byte aligned.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED (D, B*H), SA_ERR_WORKSPACE;
 * inf/NaN in the rotated values sets SA_ERR_NONFINITE in the device status.
 * Caller-owned buffers, none retained.
 * ------------------------------------------------------------------------ */
size_t sa_quant_ip_workspace_size(int B, int H, int N, int D);
sa_status sa_quant_nvfp4_ip(const void* q_dev, const void* k_dev, int B, int H, int N, int D,
                            const int8_t* signs_dev, int smooth, sa_scale_mode mode, int f_lo, int f_hi,
                            uint8_t* q_codes_dev, uint8_t* q_scales_dev, float* q_g_dev, uint8_t* k_codes_dev,
                            uint8_t* k_scales_dev, float* k_g_dev, float* k_mean_dev, float* r_dev,
                            int8_t* q_ss_off_dev, int8_t* k_ss_off_dev, void* ws_dev, size_t ws_bytes,
                            cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_attn_fwd -- NVFP4 attention forward (prefill).
 * "Search Your Block Floating Point Scales!", "ScaleSearchAttention /
 * 네이티브 NVFP4 실행": Q K^T and P V as block-scaled FP4 tensor-core MMAs
 * with FP32 accumulation.  Schedule: query rows independent; key tiles of 128
 * in ascending order with an online softmax (m updated every tile); causal
 * masks j > i and skips tiles past the diagonal; P~ = exp(S - m) is
 * requantised per 16 keys to NVFP4 with the fixed second-level scale 1/2688
 * and max-scaling before P V; the denominator l sums the dequantised P;
 * out = O / l.  Optional high-precision blocks ("ThriftAttention"): where
 * mask[b,h,t,u] = 1 the block's scores are q.(k - k_mean) from the raw bf16
 * inputs, P is rounded to bf16 and multiplied by raw bf16 V, inside the same
 * online softmax.
 *
 *  q/k/v codes, scales, g: outputs of sa_quant_nvfp4 for roles Q, K, V.
 *  sm_scale      score scale; <= 0 means 1/sqrt(D).
 *  mask_dev      NULL (all NVFP4) or uint8 [B,H,T,T] from sa_thrift_select;
 *                then q_bf16_dev, k_bf16_dev, v_bf16_dev (raw inputs) and
 *                k_mean_dev (from the K pre-pass; NULL if K was not smoothed)
 *                are required.
 *  out_dev       FP32 [B,H,N,D].
 *  lse_dev       FP32 [B,H,N] natural-log log-sum-exp of the scaled scores
 *                (m + ln l), may be NULL.
 * ------------------------------------------------------------------------ */
sa_status sa_attn_fwd(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev, const float* q_g_dev,
                      const uint8_t* k_codes_dev, const uint8_t* k_scales_dev, const float* k_g_dev,
                      const uint8_t* v_codes_dev, const uint8_t* v_scales_dev, const float* v_g_dev, int B, int H,
                      int N, int D, int causal, float sm_scale, const uint8_t* mask_dev, const void* q_bf16_dev,
                      const void* k_bf16_dev, const void* v_bf16_dev, const float* k_mean_dev, float* out_dev,
                      float* lse_dev, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_attn_fwd_ex -- sa_attn_fwd with the block rule of the requantised P
 * chosen: p_mode SA_SCALE_MAX is sa_attn_fwd; SA_SCALE_SEARCH applies
 * ScaleSearch to P ("Search Your Block Floating Point Scales!", "ScaleSearch":
 * the same candidates as for Q, K and V, i.e. per 16 keys the scale codes
 * c0 + f, f in [-2, 6), c0 = E4M3(max p~ / 6), on p~ = P~ * 2688, keeping the
 * least squared error of p~, ties to the lower candidate in the order
 * f = 0, -2, -1, 1, ..., 5).  The search costs about eight block encodings
 * per 16 keys on the softmax's critical path.  SA_SCALE_SEARCH with a
 * high-precision block mask returns SA_ERR_UNSUPPORTED; another p_mode
 * returns SA_ERR_INVALID_ARG.  Other arguments and errors as sa_attn_fwd.
 * ------------------------------------------------------------------------ */
sa_status sa_attn_fwd_ex(const uint8_t* q_codes_dev, const uint8_t* q_scales_dev, const float* q_g_dev,
                         const uint8_t* k_codes_dev, const uint8_t* k_scales_dev, const float* k_g_dev,
                         const uint8_t* v_codes_dev, const uint8_t* v_scales_dev, const float* v_g_dev, int B, int H,
                         int N, int D, int causal, float sm_scale, int p_mode, const uint8_t* mask_dev,
                         const void* q_bf16_dev, const void* k_bf16_dev, const void* v_bf16_dev,
                         const float* k_mean_dev, float* out_dev, float* lse_dev, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_attn_decode_kvfp4 -- one query token per sequence over an NVFP4 KV
 * cache ("ScaleSearchAttention": the KV cache kept in 4 bits), grouped-query
 * heads (query head h reads kv head h / (Hq/Hkv)).  q is quantised like a Q
 * tensor (its own g over [B,Hq,D], blocks along D, max-scaling).  Keys are
 * processed in splits of 4096 (each split its own online softmax over key
 * tiles of 128, P requantised as in sa_attn_fwd), then merged exactly:
 * O = sum_s e^(m_s-M) O_s / sum_s e^(m_s-M) l_s.
 *
 *  q_dev           bf16 [B,Hq,D].
 *  k/v codes etc.  sa_quant_nvfp4 outputs for the caches viewed as
 *                  [B,Hkv,L,D] (roles K and V).
 *  out_dev         FP32 [B,Hq,D].
 *  ws_dev          sa_decode_workspace_size() bytes.
 * Requires L % 128 == 0.
 * ------------------------------------------------------------------------ */
size_t sa_decode_workspace_size(int B, int Hq, int Hkv, int L, int D);
sa_status sa_attn_decode_kvfp4(const void* q_dev, const uint8_t* k_codes_dev, const uint8_t* k_scales_dev,
                               const float* k_g_dev, const uint8_t* v_codes_dev, const uint8_t* v_scales_dev,
                               const float* v_g_dev, int B, int Hq, int Hkv, int L, int D, float sm_scale,
                               float* out_dev, void* ws_dev, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * sa_attn_decode_kvfp4_sink -- sa_attn_decode_kvfp4 over an attention-sink-
 * aware mixed-precision cache ("Search Your Block Floating Point Scales!",
 * "ScaleSearchAttention": the first and last blocks of the cache are kept at
 * full precision, the middle ones in NVFP4).  Reading: a block is a 128-key
 * cache tile and "full precision" is the raw bf16 cache.  The first
 * sink_first and the last sink_last tiles of each (b, kv head) take the
 * mixed-block arithmetic of sa_attn_fwd's high-precision blocks inside the
 * same split-wise online softmax: score = q . (k - mean(K)) * sm_scale with
 * the raw bf16 q and k (the mean only when K was smoothed), P rounded to
 * bf16, raw bf16 V.  The NVFP4 codes of those tiles are not read.
 *
 *  sink_first,
 *  sink_last       tiles kept at full precision at each end of the cache;
 *                  (0, 0) is sa_attn_decode_kvfp4.  128 (sink_first +
 *                  sink_last) <= L, otherwise SA_ERR_INVALID_ARG.
 *  k_sink_dev,
 *  v_sink_dev      bf16 [B, Hkv, 128 (sink_first + sink_last), D], 16-byte
 *                  aligned: per (b, kv head) the first sink_first tiles of the
 *                  cache, then its last sink_last tiles, keys ascending.
 *  k_mean_dev      FP32 [B, Hkv, D], the channel means that smoothed the K
 *                  cache (sa_quant_nvfp4's k_mean output), or NULL when K was
 *                  quantised without smoothing.
 * The other arguments, the workspace and the errors are those of
 * sa_attn_decode_kvfp4.  Caller-owned buffers, none retained.
 * ------------------------------------------------------------------------ */
sa_status sa_attn_decode_kvfp4_sink(const void* q_dev, const uint8_t* k_codes_dev, const uint8_t* k_scales_dev,
                                    const float* k_g_dev, const uint8_t* v_codes_dev, const uint8_t* v_scales_dev,
                                    const float* v_g_dev, int B, int Hq, int Hkv, int L, int D, float sm_scale,
                                    int sink_first, int sink_last, const void* k_sink_dev, const void* v_sink_dev,
                                    const float* k_mean_dev, float* out_dev, void* ws_dev, size_t ws_bytes,
                                    cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SA_H */
