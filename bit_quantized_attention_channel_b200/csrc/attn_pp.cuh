// attn_pp.cuh -- NVFP4 attention forward (prefill): persistent CTAs, two
// query tiles per work item, two softmax threads per query row, optional
// bf16 blocks inside the same online softmax.
//
// "Search Your Block Floating Point Scales!", "ScaleSearchAttention / native
// NVFP4 execution": Q K^T and P V as block-scaled FP4 tensor-core MMAs with
// FP32 accumulation; online softmax over key tiles of 128; P requantised per
// 16 keys with the fixed second-level scale 1/2688.  "ThriftAttention": where
// the block mask is set, the block's Q K^T and P V run on the raw bf16 inputs
// (kind::f16 MMAs) inside the same softmax.
//
// A work item is (b, h, pair): tile A (query rows 256p..256p+127) and tile B
// (the next 128).  Each K/V tile is loaded once for both.  The grid holds one
// CTA per SM; CTA c takes items c, 2G-1-c, 2G+c, ... of the list ordered
// heaviest causal pair first.
//   warp 0        producer (one lane): Q tiles, a ring of NVFP4 K/V stages
//                 and, with bf16 blocks, the raw K, V and Q tiles they need.
//   warp 1        Q K^T issuer (one lane).
//   warp 2        P V issuer (one lane): the two MMA streams wait on different
//                 events, so a new S is issued the moment its buffer is free
//                 rather than behind a P V (and each issuer shares its SM
//                 sub-partition's issue slots with four softmax warps).
//   warp 3        idle (it keeps five warps on every SM sub-partition, whose
//                 register files set the launch allocation).
//   warps 4..11   softmax of tile A, warps 12..19 of tile B: warp w reads the
//                 TMEM lane quadrant w % 4 (query rows 32(w%4)..+31) and the
//                 key half h = ((w - 4) / 4) % 2 (columns 64h..64h+63).  The
//                 two halves of a row meet once per key tile, through shared
//                 memory and an mbarrier of the quadrant's two warps (a
//                 bounded wait), to agree on the row max; each half then
//                 computes its four 16-key block scales
//                 (one 32-bit scale word of P), its 64 codes and the rescale
//                 of its half of [O | l].
// Every SM sub-partition (warps w with equal w % 4) runs two softmax warps of
// each tile, so the special-function
// work of one overlaps the TMEM traffic, reductions and waits of the others.
//
// TMEM (512 columns): one S buffer (128) handed between the tiles
// (Q_A K_u^T -> A reads -> Q_B K_u^T -> B reads -> Q_A K_{u+1}^T ...), the
// accumulators [O_x | l_x] (144 each; the V operand carries 16 rows of E2M1
// 1.0 after row 127, so column 128 sums the dequantised P exactly) and the
// scale factors.  bf16 blocks accumulate into the same O_x: their P, rounded
// to bf16, is scaled by 2688 / g_V (the ratio between the NVFP4 accumulator's
// units and raw-V units) and rounded to bf16 again; their row sums stay in
// registers.
// Every barrier phase is counted over the CTA's whole item sequence.
#pragma once

#include "attn.cuh"
#include "quant.cuh"

namespace sa {

constexpr int kPpThreads = 640;  // 20 warps
constexpr int kPpStagesF = 4;  // NVFP4 K/V ring of the all-NVFP4 kernel
constexpr int kPpStagesM = 3;  // ... of the kernel with bf16 blocks

template <int D, bool MIXED>
struct PpSmem {
    static constexpr int S = MIXED ? kPpStagesM : kPpStagesF;
    static constexpr int QB = MIXED ? 1 : 2;            // Q buffers (items in flight)
    static constexpr int RB = MIXED ? D / 64 : 1;        // 64-channel regions of a raw bf16 tile
    static constexpr int RBYTES = MIXED ? 16384 : 1024;  // 128 rows x 128 bytes, 128-byte swizzle
    alignas(1024) uint8_t q[QB][2][128 * D / 2];
    alignas(1024) uint8_t k[S][128 * D / 2];
    alignas(1024) uint8_t v[S][128 * 64 + 16 * 64];  // V^T (D rows), zero rows to 128, 16 rows of 1.0
    alignas(1024) uint8_t p[2][128 * 64];            // NVFP4 P of each tile; epilogue staging
    alignas(1024) uint8_t qb[RB][RBYTES];            // raw bf16 Q of one query tile
    alignas(1024) uint8_t kb[RB][RBYTES];            // raw bf16 K tile (K-major)
    alignas(1024) uint8_t vb[RB][RBYTES];            // raw bf16 V tile (rows = keys, MN-major operand)
    alignas(1024) uint8_t pb[2][RBYTES];             // bf16 P of one query tile: 2 x 64 keys
    alignas(16) uint8_t qsf[QB][2][D / 64 * 512];
    uint8_t ksf[S][D / 64 * 512];
    uint8_t vsf[S][2 * 512];
    // Key tiles holding a bf16 block, in schedule order: {item count, key tile,
    // flags (bit x: query tile x), b*H + h | pair << 16}.  The producer pushes
    // an entry just before it loads that tile into the ring, so every role
    // that has waited for the tile finds it; at most S such tiles are in
    // flight, far below the 16 slots.
    int4 bfq[16];
    int bfq_n;                // entries pushed
    float lg2sc[128];         // log2 of each nonzero E4M3 scale value
    float rcp[128];           // 1 / each E4M3 scale value (ScaleSearch on P)
    float xch[2][2][2][128];  // half-row exchange: [use parity][tile][half][row]
    uint64_t q_full[QB];      // Q tiles and scale atoms landed
    uint64_t q_empty[QB];     // every Q K^T of the item completed
    uint64_t kv_full[S];
    uint64_t kv_empty[S];
    uint64_t s_full[2];  // [tile]: S holds this tile's scores
    uint64_t s_free[2];  // [tile]: this tile's 8 warps have read S
    uint64_t p_full[2];  // [tile]: this tile's 8 warps wrote P and rescaled O
    uint64_t o_done[2];  // [tile]: the tile's P V completed
    uint64_t xbar[2][4]; // [tile][quadrant]: both halves of the rows posted their value
    uint64_t drain;      // both issuers' tensor-core work has completed (kernel exit)
    // bf16 blocks: raw K / V tiles (one per key tile that has a bf16 block),
    // raw Q tiles (reloaded when the next bf16 block is another query tile's:
    // qb_empty completes once per reload) and the bf16 P buffer, shared by the
    // two tiles one block at a time (pb_grant[x] completes once per bf16 block
    // of tile x, when the block before it has finished its P V).  Each phase
    // of every barrier is awaited in order by its waiters, as parity waits need.
    uint64_t kb_full, kb_empty, vb_full, vb_empty, qb_full, qb_empty, pb_grant[2];
    uint32_t tmem_slot;
    int abort;
};

// TMEM columns: [O_x | l_x] is PP_OW wide at PP_O + PP_OW x (l in column 128);
// SFQ: tile x at + 8 x; SFV: 64-key block kb at + 8 kb (V rows in + 0..3, the
// 1.0 rows' scale at + 4); SFP: tile x at + 8 x, block kb at + 4 kb.
constexpr int PP_REG_CTL = 64, PP_REG_SM = 104;  // 128 x 64 + 512 x 104 = 640 x 96
static_assert(128 * PP_REG_CTL + 512 * PP_REG_SM <= kPpThreads * 96, "register split exceeds the launch allocation");
constexpr uint32_t PP_S = 0, PP_O = 128, PP_OW = 144, PP_SFQ = 416, PP_SFK = 432, PP_SFV = 440, PP_SFP = 456;

// Bounded wait for the phase of `bar` with the given parity.  Gives up (false)
// when another role has aborted, or after `lim` cycles, when it records
// SA_ERR_TIMEOUT and raises the CTA's abort flag so every role unwinds.
SA_DEV bool pp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, long long lim)
{
    if (mbar_test(bar, parity)) return true;
    const uint32_t hint = (uint32_t)min(max(lim / 4, 32LL), 1000000LL);  // ns, below the limit in cycles
    const long long t0 = clock64();
    while (!mbar_try_wait_hint(bar, parity, hint)) {
        if (*abort) return false;
        if (clock64() - t0 > lim) {
            *abort = 1;
            sa_raise(SA_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Wait (bounded by the library default) for a phase the caller knows will
// complete: the copies and tensor-core work a role issued, drained before the
// CTA releases its shared memory and tensor memory.
SA_DEV void pp_drain(uint64_t* bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > SA_WAIT_CYCLES) {
            sa_raise(SA_ERR_TIMEOUT);
            return;
        }
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

// Work item of the zigzag schedule.
struct PpItem {
    int bh, pair, nuA, nuB, nu;
    bool hasB;
};

// Item index of round j of this CTA, or -1 past the end.
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

// bf16 flags of key tiles [base, base + 32) of an item's two query tiles, read
// from the mask once per 32 tiles instead of per tile.
struct PpFlags {
    int base;
    uint32_t a, b;
};

// 16 mask bytes -> 16 bits (bit i set when byte i is nonzero).
SA_DEV uint32_t pp_bytes_to_bits(uint4 w)
{
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
    uint32_t bits = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t nz = __vcmpne4(v[i], 0u) & 0x01010101u;  // one bit per nonzero byte, at bit 8j
        bits |= ((nz * 0x01020408u) >> 24) << (4 * i);         // gather bits 0, 8, 16, 24 to 0..3
    }
    return bits;
}

template <bool MIXED>
SA_DEV void pp_flags_fill(PpFlags& f, const AttnParams& p, const PpItem& I, int base)
{
    f.base = base;
    f.a = f.b = 0;
    if (!MIXED) return;
    const uint8_t* ra = p.mask + ((size_t)I.bh * p.T + 2 * I.pair) * p.T + base;
    const uint8_t* rb = ra + p.T;
    if ((p.T & 15) == 0 && base + 32 <= p.T) {
        f.a = pp_bytes_to_bits(__ldg(reinterpret_cast<const uint4*>(ra))) |
              (pp_bytes_to_bits(__ldg(reinterpret_cast<const uint4*>(ra + 16))) << 16);
        if (I.hasB)
            f.b = pp_bytes_to_bits(__ldg(reinterpret_cast<const uint4*>(rb))) |
                  (pp_bytes_to_bits(__ldg(reinterpret_cast<const uint4*>(rb + 16))) << 16);
    } else {
        for (int i = 0; i < 32 && base + i < p.T; i++) {
            f.a |= (uint32_t)(__ldg(ra + i) != 0) << i;
            if (I.hasB) f.b |= (uint32_t)(__ldg(rb + i) != 0) << i;
        }
    }
    // only key tiles the query tile visits count
    const int na = I.nuA - base, nb = I.nuB - base;
    f.a &= na >= 32 ? ~0u : (na <= 0 ? 0u : (1u << na) - 1u);
    f.b &= nb >= 32 ? ~0u : (nb <= 0 ? 0u : (1u << nb) - 1u);
}

// bf16 flags of key tile u for query tiles A (bit 0) and B (bit 1).
template <bool MIXED>
SA_DEV uint32_t pp_flags(PpFlags& f, const AttnParams& p, const PpItem& I, int u)
{
    if (!MIXED) return 0;
    if (u < f.base || u >= f.base + 32) pp_flags_fill<MIXED>(f, p, I, u & ~31);
    const int i = u - f.base;
    return ((f.a >> i) & 1u) | (((f.b >> i) & 1u) << 1);
}

// bf16 flags of key tile u of the item counted `it` (bit x: query tile x),
// read from the queue the producer fills; `qi` is the caller's read position
// (entries are in schedule order, so it only moves forward).
template <bool MIXED, typename Q>
SA_DEV uint32_t pp_bf16_flags(const Q& s, int& qi, int it, int u)
{
    if (!MIXED) return 0;
    const int n = *reinterpret_cast<const volatile int*>(&s.bfq_n);
    const long long key = ((long long)it << 32) | (unsigned)u;
    while (qi < n) {
        const int4 e = s.bfq[qi & 15];
        const long long ek = ((long long)e.x << 32) | (unsigned)e.y;
        if (ek > key) return 0;
        qi++;
        if (ek == key) return (uint32_t)e.z;
    }
    return 0;
}

// Position of the producer's walk over this CTA's items and their key tiles.
struct PpCursor {
    int j;   // round
    int it;  // items passed
    int i;   // item index, -1 past the end
    int u;   // key tile
    int x;   // query tile (event walks)
    PpItem I;
};

SA_DEV void pp_cursor_seek_item(PpCursor& c, const AttnParams& p, int nitems, int nrounds)
{
    c.i = -1;
    for (; c.j < nrounds; c.j++) {
        c.i = pp_item_index(c.j, nitems);
        if (c.i >= 0) {
            c.I = pp_item(p, c.i);
            return;
        }
    }
    c.i = -1;
}

SA_DEV void pp_cursor_next_item(PpCursor& c, const AttnParams& p, int nitems, int nrounds)
{
    c.j++;
    c.it++;
    c.u = 0;
    c.x = 0;
    pp_cursor_seek_item(c, p, nitems, nrounds);
}

// The P of a bf16 block for one half row, eight keys at a time from S (which
// the block still holds): t = (S - c_i) sm_scale log2(e) (masked keys none),
// P^ = bf16(2^(t - m)) as the method rounds it, then P' = bf16(P^ kappa) in
// the NVFP4 accumulator's units (kappa = 2688 / g_V), written to the bf16 P
// row (128-byte swizzle).  Returns the sum of P'.  Kept out of line: bf16
// blocks are few and the softmax loop stays compact.
__device__ __noinline__ float pp_bf16_p_row(uint8_t* prow, uint32_t s_col, int swz, int kbase, bool edge, int N,
                                            bool causal, int row, float crow, float cb, float msub, float kappa)
{
    float ls = 0.0f;
#pragma unroll 1
    for (int cc = 0; cc < 8; cc++) {
        float sc[8];
        tmem_ld8_sync(s_col + 8 * cc, sc);
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            float t2[2];
#pragma unroll
            for (int j2 = 0; j2 < 2; j2++) {
                const int key = kbase + 8 * cc + 2 * e + j2;
                const bool valid = !edge || (key < N && (!causal || key <= row));
                t2[j2] = valid ? ex2f(__fsub_rn(sc[2 * e + j2], crow) * cb - msub) : 0.0f;
            }
            const __nv_bfloat162 ph = __floats2bfloat162_rn(t2[0], t2[1]);
            const __nv_bfloat162 pr = __floats2bfloat162_rn(__low2float(ph) * kappa, __high2float(ph) * kappa);
            ls += __low2float(pr);
            ls += __high2float(pr);
            w4[e] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        *reinterpret_cast<uint4*>(prow + ((cc ^ swz) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    return ls;
}

// The softmax side of one bf16 block, inline (a call site in the softmax loop
// slowed the NVFP4 tiles more than the code it moved out saved; the P row
// below it stays a call): wait until O is free (o_done, when this tile had a
// P V before) and the shared bf16 P buffer is granted, write this
// half row's P, release S, then bring this half's columns of [O | l] to the new
// max (o_half: its first O column; l_col: the l column when this half keeps l,
// else 0): on the tile's first key tile l starts at 0, later O and l are
// rescaled by alpha when any row's max moved; finally hand P to the P V
// issuer.  Returns the half row's sum of P (units of 2688 / g_V), or -1 when a
// wait gave up.
SA_DEV float pp_bf16_tile(uint64_t* o_done, uint32_t od_parity, uint64_t* pb_grant, uint32_t pg_parity,
                          uint64_t* s_free, uint64_t* p_full, volatile int* abort, long long lim, uint8_t* prow,
                          uint32_t s_col, int swz, int kbase, bool edge, int N, bool causal, int row, float crow,
                          float cb, float msub, float kappa, bool first, float alpha, uint32_t o_half, int hd,
                          uint32_t l_col)
{
    if ((o_done && !pp_wait(o_done, od_parity, abort, lim)) || !pp_wait(pb_grant, pg_parity, abort, lim))
        return -1.0f;
    tc_fence_after();
    const float ls = pp_bf16_p_row(prow, s_col, swz, kbase, edge, N, causal, row, crow, cb, msub, kappa);
    tc_fence_before();
    __syncwarp();
    const bool lead = (threadIdx.x & 31) == 0;
    if (lead) mbar_arrive(s_free);  // S is read
    if (first) {
        if (l_col) tmem_st1(l_col, 0.0f);  // l starts at 0 (no NVFP4 P V yet)
    } else if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
        for (int c = 0; c < hd; c += 32) {
            float o[32];
            tmem_ld32(o_half + c, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int i2 = 0; i2 < 32; i2++) o[i2] *= alpha;
            tmem_st32(o_half + c, o);
        }
        if (l_col) {
            const float lv = tmem_ld1_sync(l_col);
            tmem_st1(l_col, lv * alpha);
        }
    }
    tmem_wait_st();
    fence_proxy_async();
    tc_fence_before();
    __syncwarp();
    if (lead) mbar_arrive(p_full);
    return ls;
}

// c_i = q_i . mean(K) for one query row (bf16 q, FP32 means), an FP32 fma
// chain over the channels in order.  Once per item; kept out of line.
__device__ __noinline__ float pp_row_offset(const uint16_t* qrow, const float* mu, int d)
{
    float c = 0.0f;
#pragma unroll 1
    for (int c8 = 0; c8 < d / 8; c8++) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(qrow) + c8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            c = __fmaf_rn(bf16_bits_to_f32(ww[e] & 0xFFFFu), __ldg(mu + 8 * c8 + 2 * e), c);
            c = __fmaf_rn(bf16_bits_to_f32(ww[e] >> 16), __ldg(mu + 8 * c8 + 2 * e + 1), c);
        }
    }
    return c;
}

template <int D, bool MIXED, bool PSEARCH>
__global__ void __launch_bounds__(kPpThreads, 1) attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                    const __grid_constant__ CUtensorMap tm_k,
                                                                    const __grid_constant__ CUtensorMap tm_v,
                                                                    const __grid_constant__ CUtensorMap tm_qb,
                                                                    const __grid_constant__ CUtensorMap tm_kb,
                                                                    const __grid_constant__ CUtensorMap tm_vb,
                                                                    const AttnParams p)
{
    using Sm = PpSmem<D, MIXED>;
    constexpr int S = Sm::S, QB = Sm::QB;
    constexpr int KB = D / 64;
    constexpr int HD = D / 2;  // O columns of one softmax half
    constexpr uint32_t QSW = D == 128 ? 4u : 6u;
    constexpr uint32_t QSBO = 8 * D / 2;
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nitems = p.B * p.H * ((p.T + 1) / 2);
    const int nrounds = (nitems + (int)gridDim.x - 1) / (int)gridDim.x;
    volatile int* abort = &s.abort;
    const long long lim = p.wait_cycles;

    if (warp == 0) {
        tmem_alloc(&s.tmem_slot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        s.abort = 0;
        s.bfq_n = 0;
        for (int i = 0; i < 16; i++) s.bfq[i] = make_int4(-1, -1, 0, 0);
        for (int i = 0; i < QB; i++) {
            mbar_init(&s.q_full[i], 1);
            mbar_init(&s.q_empty[i], 1);
        }
        for (int i = 0; i < S; i++) {
            mbar_init(&s.kv_full[i], 1);
            mbar_init(&s.kv_empty[i], 2);  // released by both issuers
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&s.s_full[i], 1);
            mbar_init(&s.s_free[i], 8);
            mbar_init(&s.p_full[i], 8);
            mbar_init(&s.o_done[i], 1);
            for (int q = 0; q < 4; q++) mbar_init(&s.xbar[i][q], 2);
        }
        if (MIXED) {
            mbar_init(&s.kb_full, 1);
            mbar_init(&s.kb_empty, 1);
            mbar_init(&s.vb_full, 1);
            mbar_init(&s.vb_empty, 1);
            mbar_init(&s.qb_full, 1);
            mbar_init(&s.qb_empty, 1);
            mbar_init(&s.pb_grant[0], 1);
            mbar_init(&s.pb_grant[1], 1);
        }
        mbar_init(&s.drain, 2);  // both issuers
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (MIXED) {
            tma_prefetch_desc(&tm_qb);
            tma_prefetch_desc(&tm_kb);
            tma_prefetch_desc(&tm_vb);
        }
    }
    if (PSEARCH) fill_rcp_table(s.rcp);
    if (tid < 128) {
        // (e - 7) + log2(1 + m/8) for normal bytes, -7 + log2(m/4) for subnormal ones
        const uint32_t e = (uint32_t)tid >> 3, m = (uint32_t)tid & 7u;
        const float sig = e ? log2f(1.0f + m * 0.125f) : log2f(m * 0.25f);
        s.lg2sc[tid] = (e ? (float)((int)e - 7) : -7.0f) + sig;
    }
    // rows D..127 of every V stage are zero, rows 128..143 are E2M1 1.0
    for (int i = tid; i < S * (144 - D) * 16; i += blockDim.x) {
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

    // register split: 128 x PP_REG_CTL + 512 x PP_REG_SM <= 640 x 96, the launch
    // allocation (five warps per SM sub-partition cap it at 96 per thread)
    if (warp < 4) pp_setmaxnreg_dec<PP_REG_CTL>();
    if (warp == 0) {
        // ------------------------------------------------ producer
        // Independent streams, each in its own order, polled in turn so that
        // none blocks another: (Q) NVFP4 Q tiles of each item, (R) the NVFP4
        // K/V ring; with bf16 blocks (K) raw K tiles, (V) raw V tiles and
        // (B) raw Q tiles.
        if (lane == 0) {
            PpCursor cf{}, cr{};  // streams Q and R
            pp_cursor_seek_item(cf, p, nitems, nrounds);
            cr = cf;
            int rg = 0;  // K/V tiles loaded so far (ring position)
            int nqf[QB] = {};  // Q loads per Q buffer
            // bf16 streams read the queue the ring fills: raw K and raw V tiles in
            // queue order, raw Q tiles per bf16 block (query tile x of an entry)
            int kq = 0, vq = 0, qq = 0, qx = 0;        // queue positions of the three streams
            int nk = 0, nv = 0, nrl = 0, qhold = -1;  // raw K, V tiles and raw Q reloads issued
            PpFlags fr{-64, 0, 0};                    // the ring's view of the mask
            int fr_it = -1;
            long long t_last = clock64();
            while (cf.i >= 0 || cr.i >= 0 || (MIXED && (kq < s.bfq_n || vq < s.bfq_n || qq < s.bfq_n))) {
                bool prog = false;
                if (cf.i >= 0) {
                    const PpItem& I = cf.I;
                    const int qs = cf.it % QB;
                    // Q buffers are free once the item QB back issued its last Q K^T
                    if (cf.it < QB || mbar_test(&s.q_empty[qs], ((cf.it / QB) - 1) & 1)) {
                        const int nq = I.hasB ? 2 : 1;
                        mbar_expect_tx(&s.q_full[qs], nq * (128 * D / 2 + KB * 512));
                        for (int x = 0; x < nq; x++) {
                            const int tt = 2 * I.pair + x;
                            tma_load_3d(s.q[qs][x], &tm_q, &s.q_full[qs], 0, tt * 128, I.bh);
                            bulk_load(s.qsf[qs][x], p.q_sf + ((size_t)I.bh * p.T + tt) * KB * 512, KB * 512,
                                      &s.q_full[qs]);
                        }
                        nqf[qs]++;
                        pp_cursor_next_item(cf, p, nitems, nrounds);
                        prog = true;
                    }
                }
                if (cr.i >= 0) {
                    const PpItem& I = cr.I;
                    const int st = rg % S, u = cr.u;
                    if (rg < S || mbar_test(&s.kv_empty[st], ((rg / S) & 1) ^ 1)) {
                        if (MIXED) {
                            // publish the tile's bf16 flags before its data can be waited for
                            if (fr_it != cr.it) {
                                fr = PpFlags{-64, 0, 0};
                                fr_it = cr.it;
                            }
                            const uint32_t f = pp_flags<MIXED>(fr, p, I, u);
                            if (f) {
                                const int n = s.bfq_n;
                                s.bfq[n & 15] = make_int4(cr.it, u, (int)f, I.bh | (I.pair << 16));
                                *reinterpret_cast<volatile int*>(&s.bfq_n) = n + 1;
                            }
                        }
                        const int nk2 = min(128, p.N - u * 128);
                        const int kblocks = nk2 > 64 ? 2 : 1;
                        mbar_expect_tx(&s.kv_full[st], 128 * D / 2 + KB * 512 + D * 64 + kblocks * 512);
                        tma_load_3d(s.k[st], &tm_k, &s.kv_full[st], 0, u * 128, I.bh);
                        bulk_load(s.ksf[st], p.k_sf + ((size_t)I.bh * p.T + u) * KB * 512, KB * 512,
                                  &s.kv_full[st]);
                        tma_load_3d(s.v[st], &tm_v, &s.kv_full[st], 0, u * D, I.bh);
                        bulk_load(s.vsf[st], p.v_sf + ((size_t)I.bh * p.CKv + 2 * u) * 512, kblocks * 512,
                                  &s.kv_full[st]);
                        rg++;
                        prog = true;
                        if (++cr.u == I.nu) pp_cursor_next_item(cr, p, nitems, nrounds);
                    }
                }
                if (MIXED) {
                    const int n = s.bfq_n;
                    // raw K of the next queued tile: the previous one's Q K^T have completed
                    if (kq < n && (nk == 0 || mbar_test(&s.kb_empty, (nk - 1) & 1))) {
                        const int4 e = s.bfq[kq & 15];
                        mbar_expect_tx(&s.kb_full, 128 * D * 2);
                        for (int r = 0; r < D / 64; r++)
                            tma_load_3d(s.kb[r], &tm_kb, &s.kb_full, 64 * r, e.y * 128, e.w & 0xFFFF);
                        nk++;
                        kq++;
                        prog = true;
                    }
                    // raw V of the next queued tile: the previous one's P V have completed
                    if (vq < n && (nv == 0 || mbar_test(&s.vb_empty, (nv - 1) & 1))) {
                        const int4 e = s.bfq[vq & 15];
                        mbar_expect_tx(&s.vb_full, 128 * D * 2);
                        for (int r = 0; r < D / 64; r++)
                            tma_load_3d(s.vb[r], &tm_vb, &s.vb_full, 64 * r, e.y * 128, e.w & 0xFFFF);
                        nv++;
                        vq++;
                        prog = true;
                    }
                    // raw Q for the next bf16 block: reload when it is another query
                    // tile's, once the issuer has released the buffer (one qb_empty
                    // phase per reload)
                    if (qq < n) {
                        const int4 e = s.bfq[qq & 15];
                        if (!((e.z >> qx) & 1)) {
                            if (++qx == 2) {
                                qx = 0;
                                qq++;
                            }
                            prog = true;
                        } else {
                            const int want = e.x * 2 + qx;
                            bool go = want == qhold;
                            if (!go && (nrl == 0 || mbar_test(&s.qb_empty, (nrl - 1) & 1))) {
                                mbar_expect_tx(&s.qb_full, 128 * D * 2);
                                for (int r = 0; r < D / 64; r++)
                                    tma_load_3d(s.qb[r], &tm_qb, &s.qb_full, 64 * r, (2 * (e.w >> 16) + qx) * 128,
                                                e.w & 0xFFFF);
                                qhold = want;
                                nrl++;
                                go = true;
                            }
                            if (go) {
                                if (++qx == 2) {
                                    qx = 0;
                                    qq++;
                                }
                                prog = true;
                            }
                        }
                    }
                }
                if (prog) {
                    t_last = clock64();
                } else {
                    if (*abort) break;
                    if (clock64() - t_last > lim) {
                        *abort = 1;
                        sa_raise(SA_ERR_TIMEOUT);
                        break;
                    }
                    // nothing to do yet: back off instead of taking issue slots from
                    // the softmax warps of this SM sub-partition (the ring holds
                    // several key tiles of slack)
                    __nanosleep(128);
                }
            }
            // every copy issued has landed before the CTA releases its shared memory
            // (after an abort too): wait for each barrier's last issued phase
            for (int b = 0; b < QB; b++)
                if (nqf[b] > 0) pp_drain(&s.q_full[b], (nqf[b] - 1) & 1);
            for (int st = 0; st < S; st++) {
                const int c = (rg - st + S - 1) / S;  // loads into stage st
                if (c > 0) pp_drain(&s.kv_full[st], (c - 1) & 1);
            }
            if (MIXED) {
                if (nk > 0) pp_drain(&s.kb_full, (nk - 1) & 1);
                if (nv > 0) pp_drain(&s.vb_full, (nv - 1) & 1);
                if (nrl > 0) pp_drain(&s.qb_full, (nrl - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ Q K^T issuer (one lane)
        // Key tiles in order; per tile Q_A K_u^T then Q_B K_u^T into the shared S
        // buffer, each once the previous S has been read.  Descriptors are bases
        // plus byte offsets / 16 (the address field of a shared-memory descriptor).
        if (lane == 0) {
            const uint64_t dq0 = make_sdesc(smem_u32(&s.q[0][0][0]), QSBO, 16, QSW);
            const uint64_t dk0 = make_sdesc(smem_u32(&s.k[0][0]), QSBO, 16, QSW);
            const uint32_t idq = idesc_fp4(128, 128);
            bool ok = true;
            int g0 = 0;  // ring position of the current item's key tile 0
            int last_x = -1, last_idx = -1;
            int nS[2] = {0, 0};
            int it = 0;
            int bk = 0, bq = 0, qhold = -1;  // bf16: raw K tiles and raw Q loads used so far
            int bq_pos = 0;                  // read position in the bf16 tile queue
            for (int j = 0; ok && j < nrounds; j++) {
                const int i = pp_item_index(j, nitems);
                if (i < 0) continue;
                const PpItem I = pp_item(p, i);
                const int qs = it % QB;
                if (!pp_wait(&s.q_full[qs], (it / QB) & 1, abort, lim)) break;
                tc_fence_after();
                for (int x = 0; x < (I.hasB ? 2 : 1); x++)
                    for (int kb = 0; kb < KB; kb++)
                        tc_cp_sf(tbase + PP_SFQ + 8 * x + 4 * kb, smem_u32(s.qsf[qs][x] + 512 * kb));
                for (int u = 0; ok && u < I.nu; u++) {
                    const int gt = g0 + u, st = gt % S;
                    if (!(ok = pp_wait(&s.kv_full[st], (gt / S) & 1, abort, lim))) break;
                    const uint32_t f = pp_bf16_flags<MIXED>(s, bq_pos, it, u);
                    // K scale atoms of this tile, queued behind the previous tile's Q K^T
                    // (the tensor pipe runs them in issue order) while S is still busy
                    tc_fence_after();
                    for (int kb = 0; kb < KB; kb++)
                        tc_cp_sf(tbase + PP_SFK + 4 * kb, smem_u32(s.ksf[st] + 512 * kb));
                    for (int x = 0; x < 2; x++) {
                        if (u >= (x ? I.nuB : I.nuA)) continue;
                        if (last_x >= 0 && !(ok = pp_wait(&s.s_free[last_x], last_idx & 1, abort, lim))) break;
                        tc_fence_after();
                        if (MIXED && ((f >> x) & 1)) {
                            // bf16 block: S = q.k on the raw tiles (K = 16 per MMA)
                            if ((x == 0 || !(f & 1)) && !(ok = pp_wait(&s.kb_full, bk & 1, abort, lim))) break;
                            const int want = it * 2 + x;
                            if (want != qhold) {
                                // hand the raw Q buffer back (once the Q K^T issued so far
                                // complete) and wait for this query tile's
                                if (qhold >= 0) tc_commit(&s.qb_empty);
                                if (!(ok = pp_wait(&s.qb_full, bq & 1, abort, lim))) break;
                                bq++;
                                qhold = want;
                            }
                            tc_fence_after();
                            const uint64_t dqb = make_sdesc(smem_u32(&s.qb[0][0]), 1024, 16, 2);
                            const uint64_t dkb = make_sdesc(smem_u32(&s.kb[0][0]), 1024, 16, 2);
#pragma unroll
                            for (int ks = 0; ks < D / 16; ks++) {
                                const uint64_t o = (uint64_t)(((ks >> 2) * 16384 + 32 * (ks & 3)) >> 4);
                                mma_bf16(tbase + PP_S, dqb + o, dkb + o, idesc_bf16(128, 128, 0), ks > 0);
                            }
                            if (x == 1 || !(f & 2)) {  // last bf16 Q K^T of this key tile
                                tc_commit(&s.kb_empty);
                                bk++;
                            }
                        } else {
                            const uint64_t dq = dq0 + (uint64_t)(((qs * 2 + x) * (128 * D / 2)) >> 4);
                            const uint64_t dk = dk0 + (uint64_t)((st * (128 * D / 2)) >> 4);
#pragma unroll
                            for (int kb = 0; kb < KB; kb++)
                                mma_fp4(tbase + PP_S, dq + 2 * kb, dk + 2 * kb, idq, tbase + PP_SFQ + 8 * x + 4 * kb,
                                        tbase + PP_SFK + 4 * kb, kb > 0);
                        }
                        tc_commit(&s.s_full[x]);
                        last_x = x;
                        last_idx = nS[x]++;
                    }
                    if (!ok) break;
                    tc_commit(&s.kv_empty[st]);  // this tile's Q K^T are issued (one of two releases)
                }
                // every Q K^T of this item has been issued: release its Q buffers
                if (ok) tc_commit(&s.q_empty[qs]);
                g0 += I.nu;
                it++;
            }
            // every MMA and scale copy issued has completed before TMEM is released
            tc_commit(&s.drain);
            pp_drain(&s.drain, 0);
        }
    } else if (warp == 2) {
        // ------------------------------------------------ P V issuer (one lane)
        // Key tiles in order; per tile [O_A | l_A] (+)= P_A [V_u | 0 | 1] then the
        // same for B (or O_x += P_x V_u for a bf16 block), each once its P is in.
        if (lane == 0) {
            const uint64_t dp0 = make_sdesc(smem_u32(&s.p[0][0]), 512, 16, 4);
            const uint64_t dv0 = make_sdesc(smem_u32(&s.v[0][0]), 512, 16, 4);
            const uint32_t idv = idesc_fp4(128, PP_OW);
            bool ok = true;
            int g0 = 0;
            int nP[2] = {0, 0};
            int bv = 0;  // bf16: raw V tiles used so far
            bool first_bf = true;  // no bf16 block handed the bf16 P buffer yet
            int bq_pos = 0;        // read position in the bf16 tile queue
            int it = 0;
            for (int j = 0; ok && j < nrounds; j++) {
                const int i = pp_item_index(j, nitems);
                if (i < 0) continue;
                const PpItem I = pp_item(p, i);
                for (int u = 0; ok && u < I.nu; u++) {
                    const int gt = g0 + u, st = gt % S;
                    if (!(ok = pp_wait(&s.kv_full[st], (gt / S) & 1, abort, lim))) break;
                    const uint32_t f = pp_bf16_flags<MIXED>(s, bq_pos, it, u);
                    tc_fence_after();
                    // V scale atoms of key tile u (the P V of the tile before was issued earlier)
                    const int nk = min(128, p.N - u * 128);
                    const int kblocks = nk > 64 ? 2 : 1;
                    for (int kb = 0; kb < kblocks; kb++)
                        tc_cp_sf(tbase + PP_SFV + 8 * kb, smem_u32(s.vsf[st] + 512 * kb));
                    for (int x = 0; x < 2; x++) {
                        if (u >= (x ? I.nuB : I.nuA)) continue;
                        if (MIXED && ((f >> x) & 1)) {
                            // this bf16 block may write the shared bf16 P buffer once the
                            // P V issued so far (the previous bf16 block's among them)
                            // have completed
                            if (first_bf)
                                mbar_arrive(&s.pb_grant[x]);
                            else
                                tc_commit(&s.pb_grant[x]);
                            first_bf = false;
                        }
                        if (!(ok = pp_wait(&s.p_full[x], nP[x] & 1, abort, lim))) break;
                        tc_fence_after();
                        if (MIXED && ((f >> x) & 1)) {
                            if ((x == 0 || !(f & 1)) && !(ok = pp_wait(&s.vb_full, bv & 1, abort, lim))) break;
                            tc_fence_after();
                            const uint64_t dpb = make_sdesc(smem_u32(&s.pb[0][0]), 1024, 16, 2);
                            const uint64_t dvb = make_sdesc(smem_u32(&s.vb[0][0]), 1024, 16384, 2);
#pragma unroll
                            for (int ks = 0; ks < 8; ks++)
                                mma_bf16(tbase + PP_O + PP_OW * x,
                                         dpb + (uint64_t)(((ks >> 2) * 16384 + 32 * (ks & 3)) >> 4),
                                         dvb + (uint64_t)((2048 * ks) >> 4), idesc_bf16(128, D, 1),
                                         (u > 0 || ks > 0) ? 1u : 0u);
                            if (x == 1 || !(f & 2)) {  // last bf16 P V of this key tile
                                tc_commit(&s.vb_empty);
                                bv++;
                            }
                        } else {
                            const uint64_t dp = dp0 + (uint64_t)((x * (128 * 64)) >> 4);
                            const uint64_t dv = dv0 + (uint64_t)((st * (128 * 64 + 16 * 64)) >> 4);
                            for (int kb = 0; kb < kblocks; kb++)
                                mma_fp4(tbase + PP_O + PP_OW * x, dp + 2 * kb, dv + 2 * kb, idv,
                                        tbase + PP_SFP + 8 * x + 4 * kb, tbase + PP_SFV + 8 * kb,
                                        (u > 0 || kb > 0) ? 1u : 0u);
                        }
                        tc_commit(&s.o_done[x]);
                        nP[x]++;
                    }
                    if (!ok) break;
                    tc_commit(&s.kv_empty[st]);  // this tile's P V are issued (the second release)
                }
                g0 += I.nu;
                it++;
            }
            tc_commit(&s.drain);
            pp_drain(&s.drain, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax
        pp_setmaxnreg_inc<PP_REG_SM>();
        const int sw = warp - 4;
        const int x = sw >> 3;        // 0: tile A, 1: tile B
        const int h = (sw >> 2) & 1;  // key half: columns 64h..64h+63 of S
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t o_col = tbase + lane_off + PP_O + PP_OW * x;
        const float c2 = p.q_g[0] * p.k_g[0] * p.sm_scale * kLog2e;
        const float cb = p.sm_scale * kLog2e;              // bf16 scores -> log2 units
        const float kappa = MIXED ? 2688.0f * p.v_g[1] : 0.0f;  // 2688 / g_V: raw-V units -> accumulator units
        bool ok = true;
        int k = 0;   // key-tile steps of this tile so far (all items)
        int nb = 0;  // this tile's bf16 blocks so far
        int bq_pos = 0, it = -1;  // read position in the bf16 tile queue; items so far
        int xp = 0;  // half-row exchanges so far
        // post this half's value of row r and return the other half's (bounded
        // wait: both halves count the same exchanges, two slots alternate)
        auto exchange = [&](float v, float& other) -> bool {
            s.xch[xp & 1][x][h][r] = v;
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.xbar[x][quad]);
            // the partner half is normally a few instructions away: poll briefly
            // before a suspending wait
            for (int n = 0; n < 32 && !mbar_test(&s.xbar[x][quad], xp & 1); n++) {
            }
            if (!pp_wait(&s.xbar[x][quad], xp & 1, abort, lim)) return false;
            other = s.xch[xp & 1][x][h ^ 1][r];
            xp++;
            return true;
        };
        for (int j = 0; ok && j < nrounds; j++) {
            const int i = pp_item_index(j, nitems);
            if (i < 0) continue;
            const PpItem I = pp_item(p, i);
            it++;
            const int nux = x == 0 ? I.nuA : I.nuB;
            const int tq = 2 * I.pair + x;
            const int row = tq * 128 + r;
            float crow = 0.0f;  // c_i = q_i . mean(K) for this row's bf16 scores
            if (MIXED && nux > 0 && p.k_mean)
                crow = pp_row_offset(p.q_bf16 + ((size_t)I.bh * p.N + min(row, p.N - 1)) * D,
                                     p.k_mean + (size_t)I.bh * D, D);
            float m2 = -INFINITY;
            float lb = 0.0f;  // this half's share of the bf16 row sum (units of 2688 / g_V)
            for (int u = 0; u < nux; u++, k++) {
                if (!pp_wait(&s.s_full[x], k & 1, abort, lim)) {
                    ok = false;
                    break;
                }
                const bool bfx = MIXED && ((pp_bf16_flags<MIXED>(s, bq_pos, it, u) >> x) & 1u);
                tc_fence_after();
                float sv[64];
                tmem_ld32(tbase + lane_off + PP_S + 64 * h, *reinterpret_cast<float(*)[32]>(&sv[0]));
                tmem_ld32(tbase + lane_off + PP_S + 64 * h + 32, *reinterpret_cast<float(*)[32]>(&sv[32]));
                tmem_wait_ld();
                reg_fence(sv);
                if (!(MIXED && bfx)) {  // a bf16 block re-reads S below and releases it then
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.s_free[x]);
                }

                const int kbase = u * 128 + 64 * h;
                const bool edge = (p.causal && u == tq) || (u * 128 + 128 > p.N);  // keys to mask
                if (edge) {
                    // the masked keys (key >= N, or key > row when causal) are a suffix
                    // of this half: keep the first nv
                    const int nv = min(p.N, p.causal ? row + 1 : p.N) - kbase;
#pragma unroll
                    for (int i2 = 0; i2 < 64; i2++) sv[i2] = i2 < nv ? sv[i2] : -INFINITY;
                }
                float bmax[4];
#pragma unroll
                for (int blk = 0; blk < 4; blk++) bmax[blk] = pp_max16(&sv[16 * blk]);
                // this half's max: raw S units for NVFP4; for a bf16 block the log2-unit
                // score (S - c_i) sm_scale log2(e), a monotone map of S, so the max maps
                float hm = fmaxf(fmaxf(bmax[0], bmax[1]), fmaxf(bmax[2], bmax[3]));
                if (MIXED && bfx && hm != -INFINITY) hm = __fsub_rn(hm, crow) * cb;
                // the two halves agree on the row max
                float om;
                if (!exchange(hm, om)) {
                    ok = false;
                    break;
                }
                const float tmax = fmaxf(hm, om);
                const float m2_new = fmaxf(m2, (MIXED && bfx) ? tmax : tmax * c2);
                const float msub = m2_new == -INFINITY ? 0.0f : m2_new;
                const float alpha = ex2f(m2 - msub);
                m2 = m2_new;

                if (MIXED && bfx) {
                    // bf16 block: wait for the buffers first, then write P eight keys
                    // at a time (no array of packed P held across the waits).  O is free
                    // once this tile's previous P V finished; the shared bf16 P buffer
                    // once the bf16 block before this one (either tile) finished its P V.
                    const float ls = pp_bf16_tile(k > 0 ? &s.o_done[x] : nullptr, (k - 1) & 1, &s.pb_grant[x], nb & 1,
                                                  &s.s_free[x], &s.p_full[x], abort, lim,
                                                  s.pb[h] + (r >> 3) * 1024 + (r & 7) * 128,
                                                  tbase + lane_off + PP_S + 64 * h, r & 7, kbase, edge, p.N,
                                                  p.causal != 0, row, crow, cb, msub, kappa, u == 0, alpha,
                                                  o_col + HD * h, HD, h == 1 ? o_col + 128 : 0u);
                    if (ls < 0.0f) {
                        ok = false;
                        break;
                    }
                    nb++;
                    lb = lb * alpha + ls;
                    continue;  // the bf16 tile is complete (P handed over)
                } else {
                    const float lm = kLog2_2688 - msub;
                    uint32_t scw = 0;
                    uint32_t codes[8];
                    if constexpr (PSEARCH) {
                        // ScaleSearch on P ("Search Your Block Floating Point Scales!",
                        // "ScaleSearch" applied to the requantised P): per 16 keys the block
                        // rule of the pre-pass on p~ = P * 2688, scale codes c0 + f for f in
                        // [-2, 6), the least squared error kept
#pragma unroll
                        for (int blk = 0; blk < 4; blk++) {
                            float xt[16];
#pragma unroll
                            for (int i2 = 0; i2 < 16; i2++) xt[i2] = ex2f(fmaf(sv[16 * blk + i2], c2, lm));
                            uint32_t sc;
                            int off;
                            quant16<true>(xt, -2, 6, codes[2 * blk], codes[2 * blk + 1], sc, off, s.rcp);
                            scw |= sc << (8 * blk);
                        }
                    } else {
                        // block scales first: E4M3 of (block max of P * 2688) / 6, and log2 of
                        // the scale value from a table
                        float bias[4];
#pragma unroll
                        for (int bp = 0; bp < 4; bp += 2) {
                            const uint32_t sc2 = f32x2_to_e4m3x2(ex2f(fmaf(bmax[bp], c2, lm)) * (1.0f / 6.0f),
                                                                 ex2f(fmaf(bmax[bp + 1], c2, lm)) * (1.0f / 6.0f));
#pragma unroll
                            for (int hh = 0; hh < 2; hh++) {
                                const int blk = bp + hh;
                                const uint32_t sc = (sc2 >> (8 * hh)) & 0xFFu;
                                bias[blk] = sc ? lm - s.lg2sc[sc] : -INFINITY;
                                scw |= sc << (8 * blk);
                            }
                        }
                        // y = P * 2688 / scale, rounded to E2M1
#pragma unroll
                        for (int c8 = 0; c8 < 8; c8++) {
                            const float* sp = &sv[8 * c8];
                            const float bs = bias[c8 >> 1];
                            codes[c8] = pack8_e2m1(ex2f(fmaf(sp[0], c2, bs)), ex2f(fmaf(sp[1], c2, bs)),
                                                   ex2f(fmaf(sp[2], c2, bs)), ex2f(fmaf(sp[3], c2, bs)),
                                                   ex2f(fmaf(sp[4], c2, bs)), ex2f(fmaf(sp[5], c2, bs)),
                                                   ex2f(fmaf(sp[6], c2, bs)), ex2f(fmaf(sp[7], c2, bs)));
                        }
                    }
                    if (MIXED) lb *= alpha;
                    // P buffer and O are free once this tile's previous P V finished
                    // (for u = 0 that is the previous item's last one)
                    if (k > 0 && !pp_wait(&s.o_done[x], (k - 1) & 1, abort, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* prow = s.p[x] + (r >> 3) * 512 + (r & 7) * 64;
#pragma unroll
                    for (int c = 0; c < 2; c++) {
                        const int cs = (2 * h + c) ^ ((r & 7) >> 1);
                        *reinterpret_cast<uint4*>(prow + cs * 16) =
                            make_uint4(codes[4 * c], codes[4 * c + 1], codes[4 * c + 2], codes[4 * c + 3]);
                    }
                    // this half's scale word of P: row r reads (lane r, column base + r / 32)
                    tmem_st1(tbase + lane_off + PP_SFP + 8 * x + 4 * h + quad, __uint_as_float(scw));
                }
                if (u > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                    // rescale this half's columns of O (and l, kept by the second half)
#pragma unroll
                    for (int c = 0; c < HD; c += 32) {
                        float o[32];
                        tmem_ld32(o_col + HD * h + c, o);
                        tmem_wait_ld();
                        reg_fence(o);
#pragma unroll
                        for (int i2 = 0; i2 < 32; i2++) o[i2] *= alpha;
                        tmem_st32(o_col + HD * h + c, o);
                    }
                    if (h == 1) {
                        const float lv = tmem_ld1_sync(o_col + 128);
                        tmem_st1(o_col + 128, lv * alpha);
                    }
                }
                tmem_wait_st();
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.p_full[x]);
            }
            if (!ok) break;
            if (nux == 0) continue;
            // ---- epilogue of this item: out = O / l * g_V (O is reused by the next item
            // only after this tile's next p_full arrival, which follows these loads)
            if (!pp_wait(&s.o_done[x], (k - 1) & 1, abort, lim)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float den = tmem_ld1_sync(o_col + 128);
            if (MIXED) {
                float lo;
                if (!exchange(lb, lo)) {
                    ok = false;
                    break;
                }
                den = fmaf(p.v_g[0], lb + lo, den);
            }
            const float scale = p.v_g[0] / den;
            {
                // Stage 32 rows x 8 floats per round in this warp's 1 KB of the tile's P
                // buffer (bytes of its own quadrant's rows, which only its partner half
                // writes, after the next item's first row exchange), 16-byte units
                // swizzled by row / 4, then
                // write 32-byte row segments: each store instruction covers 16 rows.
                float4* stage = reinterpret_cast<float4*>(s.p[x] + quad * 2048 + h * 1024);
                const int row0 = tq * 128 + quad * 32;
                float* obase = p.out + ((size_t)I.bh * p.N + row0) * D + HD * h;
#pragma unroll 1
                for (int c = 0; c < HD / 8; c++) {
                    uint32_t o[8];
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
                        "tcgen05.wait::ld.sync.aligned;"
                        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]),
                          "=r"(o[7])
                        : "r"(o_col + HD * h + 8 * c)
                        : "memory");
#pragma unroll
                    for (int j2 = 0; j2 < 2; j2++)
                        stage[2 * lane + (j2 ^ ((lane >> 2) & 1))] =
                            make_float4(__uint_as_float(o[4 * j2]) * scale, __uint_as_float(o[4 * j2 + 1]) * scale,
                                        __uint_as_float(o[4 * j2 + 2]) * scale, __uint_as_float(o[4 * j2 + 3]) * scale);
                    __syncwarp();
#pragma unroll
                    for (int i2 = 0; i2 < 2; i2++) {
                        const int rr = 16 * i2 + (lane >> 1), uu = lane & 1;
                        if (row0 + rr < p.N)
                            *reinterpret_cast<float4*>(obase + (size_t)rr * D + 8 * c + 4 * uu) =
                                stage[2 * rr + (uu ^ ((rr >> 2) & 1))];
                    }
                    __syncwarp();
                }
            }
            if (p.lse && h == 0 && row < p.N)
                p.lse[(size_t)I.bh * p.N + row] = m2 * kLn2 + logf(den * (1.0f / 2688.0f));
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace sa
