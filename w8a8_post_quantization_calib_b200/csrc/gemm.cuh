// gemm.cuh -- tcgen05 tensor-core GEMM for sm_100a with fused epilogues.
//
//   acc[i, j] = sum_k A[i, k] * B[j, k]      (A, B K-major in global memory)
//
// kind::i8 (s8 x s8 -> s32) for the W8A8 linear, kind::f8f6f4 (E4M3 x E4M3 ->
// f32) for its FP8 variant, kind::f16 (f16 x f16 -> f32) for the unquantised
// reference product of the alpha search.
//
// Two kernels, each with 192 threads per CTA:
//   warp 0      TMA producer: the stage's A and B tiles (128-byte swizzle,
//               one or two 128-byte K blocks per load) into a ring of stages
//   warp 1      MMA issuer: tcgen05.mma per 32-byte K step into a TMEM
//               accumulator; tcgen05.commit frees the stage / hands a
//               finished accumulator to the epilogue
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31), dequant / SiLU*mul / requant, stores
// TMEM holds two accumulators (2 x BN columns) so that the epilogue of one
// tile overlaps the mainloop of the next.
//
// k_gemm2 (M > 128, and the swapped form for 64 < M <= 128): clusters of two
// CTAs on two SMs, one persistent cluster per SM pair walking tiles in
// raster groups; the leader issues tcgen05.mma.cta_group::2 (M = 256), each
// CTA loads its 128 rows of A and BN/2 rows of B.  Normal orientation: A =
// activations xq [M, K], B = weights wq [N, K]; a TMEM lane is a token row, a
// column an output channel; TMA stores of the outputs.  Swapped (EPI_DEQUANT_T):
// A = weights, B = the token tile, output stored transposed.
//
// k_gemm_swap (M <= 128): A = weights, B = activations (BN = 16..128 tokens),
// so the 128-row MMA is filled with weight rows and the kernel streams the
// weight matrix; a TMEM lane is an output channel, a column a token.  One
// weight tile per CTA, or, when that would leave most SMs idle, a cluster of
// 2 or 4 CTAs sharing each tile's K range and combining their partial sums
// through distributed shared memory.  With the cluster split off, the
// (tile, K block) iterations may be spread evenly over the SMs (stream-K),
// the partial sums of shared tiles going through a workspace.
//
// Every mbarrier wait is bounded (ptx::wait_bounded): on expiry the kernel
// records an error code, stops issuing, waits (bounded) for its own TMA loads
// and MMAs in flight, frees its TMEM and returns.
#pragma once

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace sq {
namespace gemm {

enum Kind : int { KIND_I8 = 0, KIND_F16 = 1, KIND_F8 = 2 };   // F8: E4M3 x E4M3 -> fp32
// EPI_DEQUANT_T: the CTA-pair kernel with the weights as its A operand and
// the tokens as B (small M), writing the dequantised output transposed.
enum Epi : int { EPI_DEQUANT = 0, EPI_S32 = 1, EPI_GATEUP = 2, EPI_F16 = 3, EPI_DEQUANT_T = 4 };

constexpr int BM = 128;            // MMA M: rows of the A operand per tile
constexpr int BKB = 128;           // bytes of K per stage (one swizzle row)
constexpr int NUM_THREADS = 192;
constexpr int GROUP_R = 16;        // raster group along A-row tiles (L2 reuse of B)
constexpr int SMEM_BUDGET = 200 * 1024;
constexpr int STG_BYTES = 4096;    // one epilogue staging buffer: 32 rows x up to 128 bytes

// error codes recorded on a barrier timeout: 0x100 | role << 4 | where
constexpr unsigned ERR_PRODUCER = 0x110, ERR_MMA = 0x120, ERR_EPI = 0x130, ERR_DRAIN = 0x140;

__host__ __device__ constexpr int pow2_at_least(int v, int lo)
{
    int r = lo;
    while (r < v) r <<= 1;
    return r;
}

// KBO: 128-byte K blocks per stage (one TMA load of each operand per stage)
template <int BN, int KBO = 1>
struct TileCfg {
    static constexpr int A_KB = BM * BKB;          // one K block of A: a 128 x 128-byte swizzle tile
    static constexpr int B_KB = BN * BKB;
    static constexpr int A_BYTES = A_KB * KBO;
    static constexpr int B_BYTES = B_KB * KBO;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
    static constexpr int TMEM_COLS = pow2_at_least(2 * BN, 32);
    static constexpr int CW = BN < 32 ? BN : 32;   // TMEM columns per epilogue load
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 512;
    static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert((2 * STAGES + 7) * 8 + 16 <= 512, "barrier area");
};

struct Params {
    int M, N, K;               // logical problem: out[M, N] from x[M, K], w[N, K]
    int rows_a, rows_b;        // rows of the A / B operand tensors
    int num_kb;                // K blocks of 128 bytes
    int tiles_r, tiles_c;      // tiles along A rows (BM) and B rows (BN)
    int num_units;             // CTA-pair path: tiles_r * tiles_c
    int sk_iters, sk_ctas;     // swap path: tiles * num_kb iterations shared by sk_ctas CTAs
    int sk_slot;               // swap path: int32 per partial-sum slot (BM * BN)
    int ring;                  // swap path: shared-memory stages in use (<= STAGES)
    const float *a_scale;      // [1] or [M] (fp16 values when scales_f16)
    int per_token;
    const float *w_scale;      // [N] (fp16 values when scales_f16)
    int scales_f16;            // a_scale / w_scale hold fp16 values (widened exactly on load)
    const void *bias;          // [N] of out_dt or null
    void *out;                 // [M, N] (gate/up: h [M, N/2] or null)
    int out_dt;
    int32_t *ws_acc;           // swap path: partial-sum slots [sk_ctas][BN][BM] (one per CTA, slot blockIdx.x)
    int *ws_cnt;               // swap path: arrival counters [tiles]
    const float *s2;           // gate/up: smoothing of h [N/2]
    const float *a2;           // gate/up: static scale of h [1]
    int8_t *hq;                // gate/up: codes of h [M, N/2] or null
    float *hmax;               // gate/up: running column max of |h| [N/2] or null
    unsigned long long timeout_ns;
    int inject;                // failure-detection test: 1 = CTA 0 withholds its first stage
};

// The dequant scales, stored as fp32 or as fp16 (widened exactly).
__device__ __forceinline__ float load_scale(const float *p, int f16, int64_t i)
{
    return f16 ? __half2float(reinterpret_cast<const __half *>(p)[i]) : p[i];
}

__device__ __forceinline__ float a_scale_of(const Params &p, int64_t m)
{
    return load_scale(p.a_scale, p.scales_f16, p.per_token ? m : 0);
}

// Tile u of the CTA-pair grid in raster-group order (GROUP_R A-row tiles per
// group, so that consecutive tiles share B tiles in L2).
__device__ __forceinline__ void decode_unit(const Params &p, int u, int &tr, int &tc)
{
    const int tile = u;
    const int group = tile / (GROUP_R * p.tiles_c);
    const int first = group * GROUP_R;
    const int gsz = min(GROUP_R, p.tiles_r - first);
    const int r = tile - group * GROUP_R * p.tiles_c;
    tr = first + r % gsz;
    tc = r / gsz;
}

__device__ __forceinline__ void tmem_load_chunk(uint32_t taddr, uint32_t (&r)[32], int cw)
{
    if (cw == 32) {
        ptx::tmem_ld32(taddr, r);
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
              "=r"(r[14]), "=r"(r[15])
            : "r"(taddr)
            : "memory");
    }
}

__device__ __forceinline__ void store_out(void *out, int out_dt, int64_t idx, float v)
{
    if (out_dt == DT_F32) static_cast<float *>(out)[idx] = v;
    else if (out_dt == DT_F16) static_cast<__half *>(out)[idx] = __float2half_rn(v);
    else static_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16_rn(v);
}

// 8 fp32 values -> 16 bytes of out_dt at out + idx (idx a multiple of 8 / 4)
__device__ __forceinline__ void store_out8(void *out, int out_dt, int64_t idx, const float *v)
{
    if (out_dt == DT_F32) {
        float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + idx);
        o[0] = make_float4(v[0], v[1], v[2], v[3]);
        o[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else if (out_dt == DT_F16) {
        uint4 w;
        __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
        __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
        w.x = *reinterpret_cast<uint32_t *>(&h0); w.y = *reinterpret_cast<uint32_t *>(&h1);
        w.z = *reinterpret_cast<uint32_t *>(&h2); w.w = *reinterpret_cast<uint32_t *>(&h3);
        *reinterpret_cast<uint4 *>(static_cast<__half *>(out) + idx) = w;
    } else {
        uint4 w;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]), h3 = __floats2bfloat162_rn(v[6], v[7]);
        w.x = *reinterpret_cast<uint32_t *>(&h0); w.y = *reinterpret_cast<uint32_t *>(&h1);
        w.z = *reinterpret_cast<uint32_t *>(&h2); w.w = *reinterpret_cast<uint32_t *>(&h3);
        *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + idx) = w;
    }
}

__device__ __forceinline__ float load_bias(const void *bias, int out_dt, int64_t n)
{
    return bias == nullptr ? 0.0f : load_elem_dt(bias, out_dt, n);
}

// Dequant: fmaf((float)acc, fl(a*w), bias) (plain product without bias).
__device__ __forceinline__ float dequant(int32_t acc, float c, const void *bias, float b)
{
    const float af = __int2float_rn(acc);
    return bias != nullptr ? __fmaf_rn(af, c, b) : __fmul_rn(af, c);
}

// The same epilogue on an fp32 accumulator (the FP8 GEMM).
__device__ __forceinline__ float dequant(float acc, float c, const void *bias, float b)
{
    return bias != nullptr ? __fmaf_rn(acc, c, b) : __fmul_rn(acc, c);
}

// An accumulator element from its 32-bit pattern (TMEM, shared or global
// memory): int32 for kind::i8, fp32 for kind::f8f6f4.
template <int KIND> struct AccOf {
    using T = int32_t;
    __device__ __forceinline__ static T from(uint32_t b) { return static_cast<int32_t>(b); }
};
template <> struct AccOf<KIND_F8> {
    using T = float;
    __device__ __forceinline__ static T from(uint32_t b) { return __uint_as_float(b); }
};

// ---------------------------------------------------------------------------
// Gate/up epilogue of one 128-row accumulator (TMEM lane = token row m): the
// columns come as 32 gate channels, then the same 32 channels' up rows,
// repeated.  ws_tile holds the tile's BN w_scale values and s2inv_tile the
// BN/2 channels' fl(1/s2), staged in shared memory while the tile's MMAs ran.
// SiLU uses the fast exponential and division (h is rounded to bf16
// afterwards: a few fp32 ulp are far below its precision).  h leaves through
// the same swizzled staging + TMA store as epilogue_tma (a warp's 32 rows x
// 32 channels of bf16 per box, rows >= M clipped by the tensor map); the
// requantised codes go straight to global memory (one 32-byte sector per
// row and chunk).
// ---------------------------------------------------------------------------
template <int BN, int NBUF>
__device__ __forceinline__ void epilogue_gateup(const Params &p, const CUtensorMap *omap_h, uint32_t tbase, int tr,
                                                int tc, int q, int lane, const float *ws_tile,
                                                const float *s2inv_tile, uint32_t stg, int &nstore)
{
    const int m = tr * BM + q * 32 + lane;
    const int mrow0 = tr * BM + q * 32;
    const bool mok = m < p.M;
    const float am = mok ? a_scale_of(p, m) : 0.0f;
    const int Nh = p.N >> 1;
    const float inv_a2 = p.hq != nullptr ? recip_or_zero(p.a2[0]) : 0.0f;
#pragma unroll 1
    for (int c = 0; c < BN / 64; ++c) {
        uint32_t rg[32], ru[32];
        ptx::tmem_ld32(tbase + c * 64, rg);
        ptx::tmem_ld32(tbase + c * 64 + 32, ru);
        ptx::tmem_ld_wait();
        const int row0 = tc * BN + c * 64;             // first gate row of this pair of chunks
        if (row0 >= p.N) continue;
        const int ch0 = row0 >> 1;
        float h[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float g = __fmul_rn(__int2float_rn(static_cast<int32_t>(rg[i])), __fmul_rn(am, ws_tile[c * 64 + i]));
            const float u = __fmul_rn(__int2float_rn(static_cast<int32_t>(ru[i])), __fmul_rn(am, ws_tile[c * 64 + 32 + i]));
            const float sg = __fdividef(g, __fadd_rn(1.0f, __expf(-g)));
            h[i] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sg, u)));   // h as bf16
        }
        if (p.out != nullptr) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(h[2 * i], h[2 * i + 1]);   // exact: h is bf16 already
                w[i] = *reinterpret_cast<uint32_t *>(&b2);
            }
            if constexpr (NBUF == 2) {
                if (lane == 0 && nstore >= 2) ptx::bulk_wait_read_1();
            } else {
                if (lane == 0 && nstore >= 1) ptx::bulk_wait_read_0();
            }
            __syncwarp();
            const uint32_t buf = stg + static_cast<uint32_t>(NBUF == 2 ? (nstore & 1) : 0) * STG_BYTES;
#pragma unroll
            for (int k = 0; k < 4; ++k) {          // 64-byte rows, 64-byte swizzle: chunk ^= (row >> 1) & 3
                const uint32_t a = buf + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[4 * k]), "r"(w[4 * k + 1]),
                             "r"(w[4 * k + 2]), "r"(w[4 * k + 3])
                             : "memory");
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::tma_store_2d(omap_h, buf, ch0, mrow0);
                ptx::bulk_commit();
            }
            ++nstore;
        }
        if (p.hmax != nullptr) {
            // calibration statistic of h (the down projection's input): the
            // column max of |h| over this warp's 32 rows, one warp max per
            // channel (|h| >= 0 orders like its bit pattern), then one
            // atomicMax per channel; h itself is not written
            uint32_t mine = 0u;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t mx = __reduce_max_sync(0xffffffffu, mok ? __float_as_uint(fabsf(h[i])) : 0u);
                if (lane == i) mine = mx;
            }
            if (ch0 + lane < Nh) atomicMax(reinterpret_cast<unsigned int *>(p.hmax) + ch0 + lane, mine);
        }
        if (p.hq != nullptr && mok) {
            // s2 == null: 1/s2 was folded into the up rows of the weight (the
            // cross-layer fold), so h is already smoothed
            const bool folded = p.s2 == nullptr;
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                int qv[4];
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    qv[t] = folded ? quant8(__fmul_rn(h[i + t], inv_a2))
                                   : quant8(__fmul_rn(__fmul_rn(h[i + t], s2inv_tile[c * 32 + i + t]), inv_a2));
                w[i / 4] = pack4(qv[0], qv[1], qv[2], qv[3]);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(p.hq + static_cast<int64_t>(m) * Nh + ch0);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
}

// ---------------------------------------------------------------------------
// Small-M kernel: swap orientation (A = weights wq [N, K], B = activations
// xq [M, K]; TMEM lane = output channel n, column = token), one persistent CTA
// per SM on a stream-K schedule.
//
// The T = tiles * num_kb (tile, 128-byte K block) iterations are laid end to
// end in tile order and CTA c of G takes iterations [floor(cT/G),
// floor((c+1)T/G)), so every SM streams the same share of the weight bytes
// whatever the tile count.  A CTA walks its share from the end to the start,
// one segment per tile it touches.  A tile inside one CTA's share is finished
// by that CTA.  A tile shared by CTAs c0 < ... < c1 is finished by its owner
// c1, for which the tile's start is the start of its share, i.e. its last
// segment; c0 reaches its part of the tile first and the middle CTAs (whose
// whole share lies inside the tile) at their end.  Each non-owner stores its
// int32 partial sums into its own slot of the workspace (a CTA is a non-owner
// of at most one tile: the one its share ends in) and bumps the tile's
// arrival counter with release semantics; the owner's epilogue warps, idle
// while their own last segment streams, wait for the counter to reach
// c1 - c0, add the slots into registers, and once their accumulator is ready
// add it, apply the epilogue and reset the counter to zero.  A CTA waits only
// for CTAs of lower index, which the hardware starts no later than itself, and
// every wait is bounded.  The integer sums are exact, so the result does not
// depend on G.  G = tiles gives the plain one-tile-per-CTA schedule, which
// needs no workspace.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int sk_begin(const Params &p, int c)
{
    return static_cast<int>(static_cast<int64_t>(c) * p.sk_iters / p.sk_ctas);
}

// The CTA whose share holds iteration i: the largest c with sk_begin(c) <= i.
__device__ __forceinline__ int sk_owner(const Params &p, int i)
{
    return static_cast<int>((static_cast<int64_t>(i + 1) * p.sk_ctas - 1) / p.sk_iters);
}

// One segment of a share walked backwards: iterations [lo, hi] of one tile.
struct Seg {
    int tile, kb_lo, kb_hi;
};

__device__ __forceinline__ Seg sk_segment(const Params &p, int it, int it_begin)
{
    Seg s;
    s.tile = it / p.num_kb;
    s.kb_hi = it - s.tile * p.num_kb;
    s.kb_lo = max(0, s.kb_hi - (it - it_begin));
    return s;
}

// acc[i] += slot_cc[(t0 + i) * BM + r] over the contributors' slots cc in
// [c0, c1) for tokens t0 + i < mval; the loads of up to 64 / CW slots are in
// flight together.
template <int CW, int KIND>
__device__ __forceinline__ void add_slots(const Params &p, typename AccOf<KIND>::T (&acc)[CW], int c0, int c1, int t0,
                                          int mval, int r)
{
    constexpr int U = (64 / CW) > 1 ? 64 / CW : 1;
    constexpr int64_t SLOT_STRIDE = BM;                // 32-bit words per token row of a slot
#pragma unroll 1
    for (int cc = c0; cc < c1; cc += U) {
        uint32_t v[U][CW];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t *sl = reinterpret_cast<const uint32_t *>(p.ws_acc) + static_cast<int64_t>(cc + u) * p.sk_slot;
#pragma unroll
            for (int i = 0; i < CW; ++i)
                v[u][i] = (cc + u < c1 && t0 + i < mval) ? __ldcg(sl + (t0 + i) * SLOT_STRIDE + r) : 0u;
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] += AccOf<KIND>::from(v[u][i]);
    }
}

// Epilogue of one segment.  q: TMEM lane quarter of this warp; row r = 32q +
// lane of the weight tile is output channel n = tr*BM + r.  wsn / bn:
// w_scale[n] and bias[n] (loaded before the accumulator is ready); s_am: the
// token scales in shared memory.  tfull_wait() waits for the accumulator and
// returns false on a timeout.
template <int BN, int EPI, int KIND, typename TfullWait>
__device__ __forceinline__ bool epilogue_sk(const Params &p, uint32_t tbase, int tr, int tc, int tile, int q,
                                            int lane, int *flag, volatile int *abort_flag, float wsn, float bn,
                                            const float *s_am, TfullWait tfull_wait)
{
    using AT = typename AccOf<KIND>::T;
    constexpr int CW = TileCfg<BN>::CW;
    constexpr int64_t SLOT = static_cast<int64_t>(BM) * BN;
    const int r = q * 32 + lane;
    const int n = tr * BM + r;
    const bool nok = n < p.N;
    const int m0 = tc * BN;
    const int mval = min(BN, p.M - m0);                 // valid tokens of this tile
    auto emit = [&](int m, AT acc) {
        const int64_t o = static_cast<int64_t>(m) * p.N + n;
        if constexpr (EPI == EPI_S32) {
            static_cast<int32_t *>(p.out)[o] = static_cast<int32_t>(acc);
        } else {
            store_out(p.out, p.out_dt, o, dequant(acc, __fmul_rn(s_am[m - m0], wsn), p.bias, bn));
        }
    };

    const int t0 = tile * p.num_kb;
    const int c0 = sk_owner(p, t0), c1 = sk_owner(p, t0 + p.num_kb - 1);
    const int me = static_cast<int>(blockIdx.x);
    const bool shared = c0 != c1, owner = me == c1;

    // the owner waits for the other contributors and pre-adds their slots
    // for the first chunk while its own last segment is still streaming
    AT pre[CW];
#pragma unroll
    for (int i = 0; i < CW; ++i) pre[i] = 0;
    if (shared && owner) {
        if (q == 2 && lane == 0) {
            const bool ok = ptx::wait_count_bounded(p.ws_cnt + tile, c1 - c0, p.timeout_ns, abort_flag, ERR_EPI + 2);
            if (ok) p.ws_cnt[tile] = 0;                 // every contributor has counted in: reset for the next call
            *flag = ok ? 1 : 0;
        }
        ptx::named_bar_sync(1, 128);
        if (*flag == 0) return tfull_wait();
        ptx::fence_acq_rel_gpu();
        add_slots<CW, KIND>(p, pre, c0, c1, 0, mval, r);
    }
    if (!tfull_wait()) return false;
    ptx::tc_fence_after();

    if (!shared || owner) {
#pragma unroll 1
        for (int c = 0; c < BN / CW; ++c) {
            uint32_t v[32];
            tmem_load_chunk(tbase + c * CW, v, CW);
            ptx::tmem_ld_wait();
            AT acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = AccOf<KIND>::from(v[i]);
            if (shared) {
                if (c == 0) {
#pragma unroll
                    for (int i = 0; i < CW; ++i) acc[i] += pre[i];
                } else {
                    add_slots<CW, KIND>(p, acc, c0, c1, c * CW, mval, r);
                }
            }
            if (!nok) continue;
#pragma unroll
            for (int i = 0; i < CW; ++i)
                if (c * CW + i < mval) emit(m0 + c * CW + i, acc[i]);
        }
        return true;
    }

    // non-owner: publish the partial sums (slot layout [token][BM]) and count in
    int32_t *mine = p.ws_acc + static_cast<int64_t>(me) * SLOT;
#pragma unroll 1
    for (int c = 0; c < BN / CW; ++c) {
        uint32_t v[32];
        tmem_load_chunk(tbase + c * CW, v, CW);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < CW; ++i)
            if (c * CW + i < mval) __stcg(mine + (c * CW + i) * BM + r, static_cast<int32_t>(v[i]));
    }
    ptx::fence_acq_rel_gpu();
    ptx::named_bar_sync(1, 128);
    if (q == 2 && lane == 0) ptx::red_add_release_gpu(p.ws_cnt + tile, 1);
    return true;
}

// KBO = 1: 2D maps over wq [N, K] and xq [M, K] (any K, ragged last block
// zero-filled); KBO > 1: 3D maps viewing them as [K/128][rows][128 bytes]
// (K a multiple of 128), so that one TMA load brings KBO K blocks (one
// 128-row swizzle tile each) -- a single CTA streams far more bytes per
// second with fewer, larger loads.  An iteration is then a group of KBO
// blocks; blocks past K are zero-filled.
// Epilogue of the cluster split (CS > 1): the CS CTAs of a cluster share one
// weight tile's K range equally (the stream-K partition with sk_ctas = tiles
// x CS never crosses a tile).  Once its own MMAs are done, the leader (rank
// 0) no longer needs its pipeline stages: it releases them to the others,
// which store their int32 partial sums there through distributed shared
// memory ([rank-1][BN/4][BM][4] int32) and arrive on its barrier; the leader adds
// them to its own accumulator and applies the epilogue.  Every wait is
// bounded.
template <int BN, int EPI, int CS, int KIND, typename TfullWait>
__device__ __forceinline__ bool epilogue_cs(const Params &p, uint32_t tbase, int tr, int tc, int q, int lane,
                                            uint32_t rank, float wsn, float bn, const float *s_am,
                                            TfullWait tfull_wait, uint32_t go_bar, uint32_t part_bar,
                                            uint32_t sbase, volatile int *abort_flag)
{
    using AT = typename AccOf<KIND>::T;
    constexpr int CW = TileCfg<BN>::CW;
    const int r = q * 32 + lane;
    const int n = tr * BM + r;
    const bool nok = n < p.N;
    const int m0 = tc * BN;
    const int mval = min(BN, p.M - m0);
    // partial sums of CTA j + 1 in the leader's stages: [j][BN / 4][BM][4]
    // int32 (four token columns of one row per 16 bytes), so that a warp's
    // 16-byte stores and loads cover 512 contiguous bytes
    auto part_off = [](int j, int g, int row) -> uint32_t {
        return static_cast<uint32_t>(((j * (BN / 4) + g) * BM + row) * 16);
    };
    if (!tfull_wait()) return false;
    ptx::tc_fence_after();
    if (rank == 0) {
        // this CTA's stages are no longer read: the others may write them
        if (q == 2 && lane >= 1 && lane < CS) ptx::mbar_arrive_cluster(ptx::map_to_rank(go_bar, lane));
        int ok = 1;
        if (lane == 0) ok = ptx::wait_bounded_cluster(part_bar, 0u, p.timeout_ns, abort_flag, ERR_EPI + 3) ? 1 : 0;
        if (__shfl_sync(0xffffffffu, ok, 0) == 0) return false;
#pragma unroll 1
        for (int c = 0; c < BN / CW; ++c) {
            uint32_t v[32];
            tmem_load_chunk(tbase + c * CW, v, CW);
            ptx::tmem_ld_wait();
            AT acc[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) acc[i] = AccOf<KIND>::from(v[i]);
#pragma unroll
            for (int j = 1; j < CS; ++j) {
#pragma unroll
                for (int g = 0; g < CW / 4; ++g) {
                    if (c * CW + 4 * g < mval) {
                        uint32_t t0, t1, t2, t3;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(t0), "=r"(t1), "=r"(t2), "=r"(t3)
                                     : "r"(sbase + part_off(j - 1, c * CW / 4 + g, r))
                                     : "memory");
                        acc[4 * g] += AccOf<KIND>::from(t0);
                        acc[4 * g + 1] += AccOf<KIND>::from(t1);
                        acc[4 * g + 2] += AccOf<KIND>::from(t2);
                        acc[4 * g + 3] += AccOf<KIND>::from(t3);
                    }
                }
            }
            if (!nok) continue;
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                if (c * CW + i < mval) {
                    const int m = m0 + c * CW + i;
                    const int64_t o = static_cast<int64_t>(m) * p.N + n;
                    if constexpr (EPI == EPI_S32) {
                        static_cast<int32_t *>(p.out)[o] = static_cast<int32_t>(acc[i]);
                    } else {
                        store_out(p.out, p.out_dt, o, dequant(acc[i], __fmul_rn(s_am[m - m0], wsn), p.bias, bn));
                    }
                }
            }
        }
        return true;
    }
    // rank > 0: wait until the leader's stages are free, then send the partial sums
    int ok = 1;
    if (lane == 0) ok = ptx::wait_bounded_cluster(go_bar, 0u, p.timeout_ns, abort_flag, ERR_EPI + 4) ? 1 : 0;
    if (__shfl_sync(0xffffffffu, ok, 0) == 0) return false;
    const uint32_t remote = ptx::map_to_rank(sbase, 0);
#pragma unroll 1
    for (int c = 0; c < BN / CW; ++c) {
        uint32_t v[32];
        tmem_load_chunk(tbase + c * CW, v, CW);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < CW / 4; ++g)
            if (c * CW + 4 * g < mval)
                ptx::st_dsmem_v4(remote + part_off(static_cast<int>(rank) - 1, c * CW / 4 + g, r), v[4 * g],
                                 v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
    }
    ptx::fence_acq_rel_cluster();
    ptx::named_bar_sync(1, 128);
    if (q == 2 && lane == 0) ptx::mbar_arrive_cluster(ptx::map_to_rank(part_bar, 0));
    return true;
}

template <int BN, int EPI, int KBO, int CS, int KIND = KIND_I8>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_swap(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x, const Params p)
{
    using C = TileCfg<BN, KBO>;
    static_assert(CS >= 1 && CS <= 4, "cluster split of 1..4 CTAs");
    static_assert((CS - 1) * BN * BM * 4 <= C::STAGES * C::STAGE_BYTES, "partial sums must fit the leader's stages");
    static_assert(KIND == KIND_I8 || (KIND == KIND_F8 && EPI == EPI_DEQUANT), "the FP8 swap kernel dequantises");
    constexpr int S = C::STAGES;
    constexpr uint32_t IDESC = KIND == KIND_F8 ? ptx::idesc_e4m3(BN) : ptx::idesc_i8(BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * C::STAGE_BYTES);
    const uint32_t bar0 = ptx::smem_addr(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
    const uint32_t done_bar = bar0 + 8u * (2 * S + 4);
    const uint32_t go_bar = bar0 + 8u * (2 * S + 5);      // cluster split: leader's stages free
    const uint32_t part_bar = bar0 + 8u * (2 * S + 6);    // cluster split: partial sums arrived
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 7);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *flag = reinterpret_cast<int *>(tmem_slot + 2);
    __shared__ float s_am[BN];
    const uint32_t sbase = ptx::smem_addr(smem);
    const int ring = (p.ring >= 2 && p.ring <= S) ? p.ring : S;   // stages in use

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(full_bar(s), 1);
            ptx::mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(tfull_bar(b), 1);
            ptx::mbar_init(tempty_bar(b), 4);
        }
        ptx::mbar_init(done_bar, 1);
        if constexpr (CS > 1) {
            ptx::mbar_init(go_bar, 1);
            ptx::mbar_init(part_bar, CS - 1);
        }
        *abort_flag = 0;
        *flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&map_w);
        ptx::tma_prefetch_desc(&map_x);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (CS > 1) ptx::cluster_sync();   // every CTA's barriers exist before any remote arrive
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t tmo = p.timeout_ns;
    const int it_begin = sk_begin(p, blockIdx.x), it_end = sk_begin(p, blockIdx.x + 1);
    pdl_wait();                        // operands and scales come from the previous kernels

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            for (int it = it_end - 1; it >= it_begin && !*abort_flag; --it) {
                const int tile = it / p.num_kb, kb = it - tile * p.num_kb;
                const int tr = tile / p.tiles_c, tc = tile - tr * p.tiles_c;
                if (!ptx::wait_bounded(empty_bar(stage), phase ^ 1u, tmo, abort_flag, ERR_PRODUCER)) break;
                const bool withhold = p.inject == 1 && blockIdx.x == 0 && issued == 0;
                if (!withhold) {
                    ptx::mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
                    const uint32_t sa = sbase + stage * C::STAGE_BYTES;
                    if constexpr (KBO == 1) {
                        ptx::tma_load_2d(sa, &map_w, full_bar(stage), kb * BKB, tr * BM);
                        ptx::tma_load_2d(sa + C::A_BYTES, &map_x, full_bar(stage), kb * BKB, tc * BN);
                    } else {
                        ptx::tma_load_3d(sa, &map_w, full_bar(stage), 0, tr * BM, kb * KBO);
                        ptx::tma_load_3d(sa + C::A_BYTES, &map_x, full_bar(stage), 0, tc * BN, kb * KBO);
                    }
                }
                ++issued;
                if (++stage == ring) { stage = 0; phase ^= 1u; }
            }
            // drain: every issued load lands before the CTA exits
            const int n_wait = issued < ring ? issued : ring;
            for (int i = 0; i < n_wait; ++i) {
                int s = stage - 1 - i;
                uint32_t ph = phase;
                if (s < 0) { s += ring; ph ^= 1u; }
                volatile int no_abort = 0;
                ptx::wait_bounded(full_bar(s), ph, tmo, &no_abort, ERR_DRAIN);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, local = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int it = it_end - 1; it >= it_begin && ok; ++local) {
                const Seg sg = sk_segment(p, it, it_begin);
                const int b = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1) & 1u;
                if (!ptx::wait_bounded(tempty_bar(b), use ^ 1u, tmo, abort_flag, ERR_MMA)) break;
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(b * BN);
                for (int kb = sg.kb_hi; kb >= sg.kb_lo; --kb) {
                    if (!ptx::wait_bounded(full_bar(stage), phase, tmo, abort_flag, ERR_MMA + 1)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sa = sbase + stage * C::STAGE_BYTES;
#pragma unroll
                    for (int j = 0; j < KBO; ++j) {
                        const uint64_t ad = ptx::sdesc_kmajor_sw128(sa + j * C::A_KB);
                        const uint64_t bd = ptx::sdesc_kmajor_sw128(sa + C::A_BYTES + j * C::B_KB);
#pragma unroll
                        for (int k = 0; k < BKB / 32; ++k) {
                            const uint32_t acc = (kb < sg.kb_hi || j > 0 || k > 0) ? 1u : 0u;
                            if constexpr (KIND == KIND_F8) ptx::mma_f8(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                            else ptx::mma_i8(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                        }
                    }
                    ptx::tc_commit(empty_bar(stage));
                    if (++stage == ring) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::tc_commit(tfull_bar(b));
                it -= sg.kb_hi - sg.kb_lo + 1;
            }
            // drain: all issued MMAs complete before TMEM is released
            ptx::tc_commit(done_bar);
            volatile int no_abort = 0;
            ptx::wait_bounded(done_bar, 0u, tmo, &no_abort, ERR_DRAIN + 1);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3;
        if constexpr (EPI == EPI_DEQUANT) {
            // the token scales of the (single) token tile, staged once
            const int t = threadIdx.x - 64;
            for (int m = t; m < BN; m += 128) {
                const int mg = min(m, p.M - 1);
                s_am[m] = a_scale_of(p, mg);
            }
            ptx::named_bar_sync(1, 128);
        }
        int local = 0;
        for (int it = it_end - 1; it >= it_begin; ++local) {
            const Seg sg = sk_segment(p, it, it_begin);
            const int tr = sg.tile / p.tiles_c, tc = sg.tile - tr * p.tiles_c;
            const int b = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1) & 1u;
            float wsn = 0.0f, bn = 0.0f;
            if constexpr (EPI == EPI_DEQUANT) {
                const int n = tr * BM + q * 32 + lane;
                if (n < p.N) {
                    wsn = load_scale(p.w_scale, p.scales_f16, n);
                    bn = load_bias(p.bias, p.out_dt, n);
                }
            }
            auto tfull_wait = [&]() {
                int ok = 1;
                if (lane == 0) ok = ptx::wait_bounded(tfull_bar(b), use, tmo, abort_flag, ERR_EPI) ? 1 : 0;
                return __shfl_sync(0xffffffffu, ok, 0) != 0;
            };
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BN);
            if constexpr (CS > 1) {
                if (!epilogue_cs<BN, EPI, CS, KIND>(p, tbase, tr, tc, q, lane, ptx::cluster_ctarank(), wsn, bn,
                                                    s_am, tfull_wait, go_bar, part_bar, sbase, abort_flag))
                    break;
            } else if (!epilogue_sk<BN, EPI, KIND>(p, tbase, tr, tc, sg.tile, q, lane, flag, abort_flag, wsn, bn,
                                                   s_am, tfull_wait)) {
                break;
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(tempty_bar(b));
            it -= sg.kb_hi - sg.kb_lo + 1;
        }
    }

    // warps 0 and 1 ran their role on lane 0 alone: reconverge them first, so
    // that the CTA barrier waits for every role to finish before TMEM is
    // released
    __syncwarp();
    __syncthreads();
    pdl_trigger();                     // every output of this CTA is written
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}
// ---------------------------------------------------------------------------
// Epilogue of one 128-row accumulator with coalesced output: each warp packs
// its 32 rows x 32 columns into a shared-memory staging buffer in the
// tensor map's swizzled layout (64-byte rows for 16-bit outputs, 128-byte rows
// for 32-bit ones) and one lane issues an asynchronous TMA store of the
// 32 x 32 box; rows >= M and columns >= N of a box are not written.  Two
// buffers per warp: a buffer is reused only after the store issued from it
// two boxes earlier has finished reading shared memory.
// ---------------------------------------------------------------------------
template <int BN, int KIND, int EPI, int NBUF>
__device__ __forceinline__ void epilogue_tma(const Params &p, const CUtensorMap *omap, uint32_t tbase, int tr,
                                             int tc, int q, int lane, uint32_t stg, int &nstore,
                                             const float *ws_tile, const float *bias_tile, float am)
{
    const int mrow0 = tr * BM + q * 32;
    const bool wide = (EPI == EPI_S32) || (EPI == EPI_DEQUANT && p.out_dt == DT_F32);   // 4-byte outputs

#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(tbase + c * 32, r);
        ptx::tmem_ld_wait();
        const int n0 = tc * BN + c * 32;
        if (n0 >= p.N) continue;
        const int nval = min(32, p.N - n0);
        uint32_t w[32];                       // packed output words of this row's 32 columns
        if constexpr (EPI == EPI_S32) {
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = r[i];
        } else {
            float v[32];
            if constexpr (EPI == EPI_F16) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 w4 = *reinterpret_cast<const float4 *>(ws_tile + c * 32 + i);     // broadcast
                    const float4 b4 = *reinterpret_cast<const float4 *>(bias_tile + c * 32 + i);
                    const float ws[4] = {w4.x, w4.y, w4.z, w4.w};
                    const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        if constexpr (KIND == KIND_F8)
                            v[i + t] = dequant(__uint_as_float(r[i + t]), __fmul_rn(am, ws[t]), p.bias, bb[t]);
                        else
                            v[i + t] = dequant(static_cast<int32_t>(r[i + t]), __fmul_rn(am, ws[t]), p.bias, bb[t]);
                    }
                }
            }
            const int odt = (EPI == EPI_F16) ? DT_F16 : p.out_dt;
            if (odt == DT_F32) {
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
            } else if (odt == DT_F16) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
                    w[i] = *reinterpret_cast<uint32_t *>(&h);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                    w[i] = *reinterpret_cast<uint32_t *>(&h);
                }
            }
        }
        // a staging buffer is rewritten only once the store issued from it has
        // finished reading shared memory
        if constexpr (NBUF == 2) {
            if (lane == 0 && nstore >= 2) ptx::bulk_wait_read_1();
        } else {
            if (lane == 0 && nstore >= 1) ptx::bulk_wait_read_0();
        }
        __syncwarp();
        const uint32_t buf = stg + static_cast<uint32_t>(NBUF == 2 ? (nstore & 1) : 0) * STG_BYTES;
        if (wide) {                           // 128-byte rows, 128-byte swizzle: chunk ^= row & 7
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t a = buf + lane * 128 + ((k ^ (lane & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[4 * k]), "r"(w[4 * k + 1]),
                             "r"(w[4 * k + 2]), "r"(w[4 * k + 3])
                             : "memory");
            }
        } else {                              // 64-byte rows, 64-byte swizzle: chunk ^= (row >> 1) & 3
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t a = buf + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[4 * k]), "r"(w[4 * k + 1]),
                             "r"(w[4 * k + 2]), "r"(w[4 * k + 3])
                             : "memory");
            }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            ptx::tma_store_2d(omap, buf, n0, mrow0);
            ptx::bulk_commit();
        }
        ++nstore;
    }
}

// ---------------------------------------------------------------------------
// Epilogue of the swapped CTA-pair tile (EPI_DEQUANT_T): TMEM lane = weight
// row n (output channel), column = token m.  Each thread holds w_scale[n] and
// bias[n]; the tile's token scales are staged in a_tile.  out[m, n] =
// dequant(acc, fl(a_m * w_n), bias_n), stored directly: for each token the
// warp's 32 lanes write 32 consecutive channels.
// ---------------------------------------------------------------------------
template <int BN, int KIND>
__device__ __forceinline__ void epilogue_t(const Params &p, uint32_t tbase, int trow, int tc, int q, int lane,
                                           const float *a_tile)
{
    using AT = typename AccOf<KIND>::T;
    const int n = trow * BM + q * 32 + lane;
    const bool nok = n < p.N;
    const float wsn = nok ? load_scale(p.w_scale, p.scales_f16, n) : 0.0f;
    const float bn = nok ? load_bias(p.bias, p.out_dt, n) : 0.0f;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
        const int m0 = tc * BN + c * 32;
        if (m0 >= p.M) break;
        uint32_t r[32];
        ptx::tmem_ld32(tbase + c * 32, r);
        ptx::tmem_ld_wait();
        if (!nok) continue;
        const int mval = min(32, p.M - m0);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i < mval) {
                const int64_t o = static_cast<int64_t>(m0 + i) * p.N + n;
                store_out(p.out, p.out_dt, o,
                          dequant(AccOf<KIND>::from(r[i]), __fmul_rn(a_tile[c * 32 + i], wsn), p.bias, bn));
            }
        }
    }
}

// ===========================================================================
// CTA-pair variant (cta_group::2): a cluster of two CTAs on two SMs computes a
// 256 x BN tile.  Each CTA loads its own 128 rows of A and BN/2 rows of B
// (32 KB per stage at BN = 256, so 6 stages fit), the leader CTA (rank 0)
// issues tcgen05.mma.cta_group::2 (M = 256) that reads both CTAs' shared
// memory and writes a 128 x BN int32 accumulator into each CTA's TMEM.  Half
// the operand bytes per MAC of the single-CTA tile.
//
// Barriers: full[s] lives in the leader (its producer posts the transaction
// bytes of both halves; both CTAs' TMA loads complete on it); empty[s] and
// tfull[b] live in both CTAs and receive multicast tcgen05.commit arrivals
// from the leader's MMA thread; tempty[b] lives in the leader and collects
// one arrival per epilogue warp of both CTAs (8).
// ===========================================================================
template <int BN, int KBO = 1>
struct PairCfg {
    static constexpr int A_KB = BM * BKB;                 // this CTA's 128 rows of A, one K block
    static constexpr int B_KB = (BN / 2) * BKB;           // this CTA's BN/2 rows of B, one K block
    static constexpr int A_BYTES = A_KB * KBO;
    static constexpr int B_BYTES = B_KB * KBO;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // epilogue staging: 2 buffers per epilogue warp, 1 for the 256-wide
    // two-block tile, which needs the room for a third stage
    static constexpr int STG_BUFS = (KBO > 1 && BN == 256) ? 1 : 2;
    static constexpr int STG_TOTAL = 4 * STG_BUFS * STG_BYTES;
    static constexpr int COLS_BYTES = 2 * 2 * 256 * 4;    // per accumulator buffer: w_scale + bias, 256 each
    static constexpr int FIXED_BYTES = 1024 + STG_TOTAL + COLS_BYTES + 256;
    static constexpr int STAGES_RAW = (227 * 1024 - FIXED_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 10 ? 10 : STAGES_RAW;
    static constexpr int TMEM_COLS = pow2_at_least(2 * BN, 32);
    static constexpr int SMEM_BYTES = FIXED_BYTES + STAGES * STAGE_BYTES;
    static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair MMA N");
    static_assert(TMEM_COLS <= 512, "two accumulators must fit TMEM");
};

// KBO > 1 (kind::i8, K a multiple of 128): 3D operand maps, KBO K blocks per
// TMA load (see k_gemm_swap); num_kb then counts groups of KBO blocks.
template <int BN, int KIND, int EPI, int KBO = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    k_gemm2(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
            const __grid_constant__ CUtensorMap map_o, const Params p)
{
    using C = PairCfg<BN, KBO>;
    constexpr int S = C::STAGES;
    constexpr int BKE = (KIND == KIND_F16) ? BKB / 2 : BKB;          // K elements per 128-byte block
    constexpr uint32_t IDESC = (KIND == KIND_I8)    ? ptx::idesc_i8_m256(BN)
                               : (KIND == KIND_F8) ? ptx::idesc_e4m3_m256(BN)
                                                   : ptx::idesc_f16_m256(BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * C::STAGE_BYTES + C::STG_TOTAL + C::COLS_BYTES);
    const uint32_t bar0 = ptx::smem_addr(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
    const uint32_t done_bar = bar0 + 8u * (2 * S + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *ok_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);     // [2]
    const uint32_t sbase = ptx::smem_addr(smem);
    const uint32_t stg_base = sbase + S * C::STAGE_BYTES;      // 1024-aligned staging buffers
    float *cols = reinterpret_cast<float *>(smem + S * C::STAGE_BYTES + C::STG_TOTAL);   // [2][w_scale 256 | bias 256]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = (rank == 0);
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(full_bar(s), 1);
            ptx::mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(tfull_bar(b), 1);
            ptx::mbar_init(tempty_bar(b), 8);
        }
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&map_a);
        ptx::tma_prefetch_desc(&map_b);
        if constexpr (EPI != EPI_GATEUP && EPI != EPI_DEQUANT_T) ptx::tma_prefetch_desc(&map_o);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_addr(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();               // both CTAs' barriers exist before any remote use
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t tmo = p.timeout_ns;
    pdl_wait();                        // operands and scales come from the previous kernels

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            for (int u = cluster; u < p.num_units && !*abort_flag; u += nclusters) {
                int tr, tc;
                decode_unit(p, u, tr, tc);
                bool ok = true;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!ptx::wait_bounded(empty_bar(stage), phase ^ 1u, tmo, abort_flag, ERR_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const bool withhold = p.inject == 1 && blockIdx.x == 0 && issued == 0;
                    if (!withhold) {
                        if (leader) ptx::mbar_arrive_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
                        const uint32_t fb = ptx::map_to_rank(full_bar(stage), 0);
                        const uint32_t sa = sbase + stage * C::STAGE_BYTES;
                        const int ya = tr * (2 * BM) + static_cast<int>(rank) * BM;
                        const int yb = tc * BN + static_cast<int>(rank) * (BN / 2);
                        if constexpr (KBO == 1) {
                            ptx::tma_load_2d_pair(sa, &map_a, fb, kb * BKE, ya);
                            ptx::tma_load_2d_pair(sa + C::A_BYTES, &map_b, fb, kb * BKE, yb);
                        } else {
                            ptx::tma_load_3d_pair(sa, &map_a, fb, 0, ya, kb * KBO);
                            ptx::tma_load_3d_pair(sa + C::A_BYTES, &map_b, fb, 0, yb, kb * KBO);
                        }
                    }
                    ++issued;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
            // drain: the leader's full barriers count both CTAs' bytes
            if (leader) {
                const int n_wait = issued < S ? issued : S;
                for (int i = 0; i < n_wait; ++i) {
                    int s = stage - 1 - i;
                    uint32_t ph = phase;
                    if (s < 0) { s += S; ph ^= 1u; }
                    volatile int no_abort = 0;
                    ptx::wait_bounded(full_bar(s), ph, tmo, &no_abort, ERR_DRAIN);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (lane == 0 && leader) {
            int stage = 0, local = 0;
            uint32_t phase = 0;
            for (int u = cluster; u < p.num_units; u += nclusters, ++local) {
                const int b = local & 1;
                const uint32_t use = static_cast<uint32_t>(local >> 1) & 1u;
                if (!ptx::wait_bounded(tempty_bar(b), use ^ 1u, tmo, abort_flag, ERR_MMA)) break;
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(b * BN);
                bool ok = true;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!ptx::wait_bounded(full_bar(stage), phase, tmo, abort_flag, ERR_MMA + 1)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sa = sbase + stage * C::STAGE_BYTES;
#pragma unroll
                    for (int j = 0; j < KBO; ++j) {
                        const uint64_t ad = ptx::sdesc_kmajor_sw128(sa + j * C::A_KB);
                        const uint64_t bd = ptx::sdesc_kmajor_sw128(sa + C::A_BYTES + j * C::B_KB);
#pragma unroll
                        for (int k = 0; k < BKB / 32; ++k) {
                            const uint32_t acc = (kb > 0 || j > 0 || k > 0) ? 1u : 0u;
                            if constexpr (KIND == KIND_I8)
                                ptx::mma_i8_pair(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                            else if constexpr (KIND == KIND_F8)
                                ptx::mma_f8_pair(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                            else
                                ptx::mma_f16_pair(d, ad + 2 * k, bd + 2 * k, IDESC, acc);
                        }
                    }
                    ptx::tc_commit_pair_mc(empty_bar(stage), 0x3);
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::tc_commit_pair_mc(tfull_bar(b), 0x3);
            }
            ptx::tc_commit_pair(done_bar);
            volatile int no_abort = 0;
            ptx::wait_bounded(done_bar, 0u, tmo, &no_abort, ERR_DRAIN + 1);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int q = warp & 3;
        const uint32_t stg = stg_base + static_cast<uint32_t>((warp - 2) * C::STG_BUFS * STG_BYTES);
        int nstore = 0;
        int local = 0;
        for (int u = cluster; u < p.num_units; u += nclusters, ++local) {
            int tr, tc;
            decode_unit(p, u, tr, tc);
            const int b = local & 1;
            const uint32_t use = static_cast<uint32_t>(local >> 1) & 1u;
            // while the MMAs of this tile run: stage its per-column scales / bias
            // and fetch this thread's row scale
            float *ws_tile = cols + b * 512;
            float *bias_tile = ws_tile + 256;
            float am = 0.0f;
            if constexpr (EPI == EPI_DEQUANT) {
                const int et = threadIdx.x - 64;             // 0..127
                for (int t = et; t < BN; t += 128) {
                    const int n = tc * BN + t;
                    ws_tile[t] = n < p.N ? load_scale(p.w_scale, p.scales_f16, n) : 0.0f;
                    bias_tile[t] = (n < p.N && p.bias != nullptr) ? load_bias(p.bias, p.out_dt, n) : 0.0f;
                }
                const int m = (2 * tr + static_cast<int>(rank)) * BM + q * 32 + lane;
                if (m < p.M) am = a_scale_of(p, m);
            } else if constexpr (EPI == EPI_DEQUANT_T) {
                // the tile's token scales (its columns)
                const int et = threadIdx.x - 64;
                for (int t = et; t < BN; t += 128) {
                    const int m = tc * BN + t;
                    ws_tile[t] = a_scale_of(p, m < p.M ? m : p.M - 1);
                }
            } else if constexpr (EPI == EPI_GATEUP) {
                // w_scale of the tile's gate/up rows, fl(1/s2) of its channels
                const int et = threadIdx.x - 64;
                for (int t = et; t < BN; t += 128) {
                    const int n = tc * BN + t;
                    ws_tile[t] = n < p.N ? load_scale(p.w_scale, p.scales_f16, n) : 0.0f;
                }
                if (p.hq != nullptr && p.s2 != nullptr) {
                    for (int t = et; t < BN / 2; t += 128) {
                        const int ch = (tc * BN) / 2 + t;
                        bias_tile[t] = ch < (p.N >> 1) ? recip_or_zero(p.s2[ch]) : 0.0f;
                    }
                }
            }
            // one thread waits for the accumulator; the 128 epilogue threads
            // then take the same decision (no warp is left at a barrier alone)
            if (threadIdx.x == 64) ok_flag[b] = ptx::wait_bounded(tfull_bar(b), use, tmo, abort_flag, ERR_EPI) ? 1 : 0;
            ptx::named_bar_sync(1, 128);
            if (!ok_flag[b]) break;
            ptx::tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BN);
            // this CTA's accumulator rows are the tile's rows rank*128 .. rank*128+127
            if constexpr (EPI == EPI_GATEUP)
                epilogue_gateup<BN, C::STG_BUFS>(p, &map_o, tbase, 2 * tr + static_cast<int>(rank), tc, q, lane,
                                                 ws_tile, bias_tile, stg, nstore);
            else if constexpr (EPI == EPI_DEQUANT_T)
                epilogue_t<BN, KIND>(p, tbase, 2 * tr + static_cast<int>(rank), tc, q, lane, ws_tile);
            else
                epilogue_tma<BN, KIND, EPI, C::STG_BUFS>(p, &map_o, tbase, 2 * tr + static_cast<int>(rank), tc, q, lane, stg,
                                            nstore, ws_tile, bias_tile, am);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(ptx::map_to_rank(tempty_bar(b), 0));
        }
        if (lane == 0) ptx::bulk_wait_all();     // output stores complete before the CTA exits
        __syncwarp();
    }

    ptx::tc_fence_before();
    ptx::cluster_sync();               // no CTA leaves while its peer may still signal it
    pdl_trigger();                     // every output of this CTA is written (TMA stores waited for)
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace sq
