// quant.cuh -- smoothing factors, the offline weight transform + per-row INT8
// quantisation, the runtime smooth + quantise of activations (static or
// per-token), RMSNorm with 1/s folded into its gain, and the squared-error
// reduction of the alpha search.
//
// Row kernels (HBM-bound): a block of ROW_T threads owns whole rows.  A row
// is read once into registers as 16-byte vectors (vector i*ROW_T + tid), the
// per-row statistic (absmax or sum of squares) is reduced across the block,
// and the codes are written from the same registers, so every element moves
// through HBM exactly once (16-bit in, 8-bit out).  The per-column constant
// of the step (s_j, fl(1/s_j) or fl(gamma_j * fl(1/s_j))) is computed once
// per block into shared memory.  Blocks loop over rows (grid <= rows).
#pragma once

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace sq {

// ---------------------------------------------------------------------------
// s_j = max(a_j,1e-5)^alpha / max(w_j,1e-5)^(1-alpha) in fp64, rounded once
// (kwkr.cn blog 2.2; aiunderstanding.org technical insight; "010. SmoothQuant
// Integration" context step 1; the 1e-5 clamp follows tbr8.org's example).
// Optionally a_static = fl(max_j fl(act_max_j * recip(s_j)) / qmax), the closed
// form of "010. SmoothQuant Integration" key design point 1 (qmax = 127 for
// INT8 codes, 448 for E4M3).  x -> fl(x/qmax) is monotone, so max_b
// fl(m_b/qmax) = fl(max_b m_b / qmax): blocks combine with atomicMax on the
// (non-negative) float bits; *a_static is zeroed first.
// A single-block launch (small K) writes the scale directly.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float smoothing_factor(float act_max, float w_max, double al)
{
    const double a = fmax(static_cast<double>(act_max), 1e-5);
    const double w = fmax(static_cast<double>(w_max), 1e-5);
    // a^alpha / w^(1-alpha) = 2^(alpha log2 a - (1-alpha) log2 w): fp64 log2/exp2
    // carry ~1e-15 relative error, far below the one fp32 rounding that follows
    return static_cast<float>(exp2(al * log2(a) - (1.0 - al) * log2(w)));
}

// K <= 8 * 1024: one 8-CTA thread-block cluster, one channel per thread (the
// fp64 log2/exp2 chains spread over 8 SMs).  Each CTA reduces its
// fl(act_max_j * recip(s_j)) maximum into its shared memory; CTA 0 reads the 8
// partial maxima through distributed shared memory and writes the static
// scale, so no pre-zeroing and no atomics are needed.
__global__ void __cluster_dims__(8, 1, 1) __launch_bounds__(1024)
    k_smooth_scales_cluster(const float *__restrict__ act_max, const float *__restrict__ w_max, int K, float alpha,
                            float *__restrict__ s, float *__restrict__ a_static, float qmax)
{
    __shared__ float red[32];
    __shared__ float cta_max;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    float m = 0.0f;
    pdl_wait();
    if (j < K) {
        const float am = act_max[j];
        const float sj = smoothing_factor(am, w_max[j], static_cast<double>(alpha));
        s[j] = sj;
        m = __fmul_rn(am, recip_or_zero(sj));
    }
    m = block_max(m, red);
    if (threadIdx.x == 0) cta_max = m;
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
    if (blockIdx.x == 0 && threadIdx.x < 32 && a_static != nullptr) {
        float v = 0.0f;
        if (threadIdx.x < 8) {
            uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(&cta_max)), remote;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(threadIdx.x));
            asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
        }
        v = warp_max(v);
        if (threadIdx.x == 0) *a_static = __fdiv_rn(v, qmax);
    }
    // no CTA leaves while CTA 0 may still read its shared memory
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
    __syncthreads();
    pdl_trigger();
}

__global__ void __launch_bounds__(1024)
    k_smooth_scales(const float *__restrict__ act_max, const float *__restrict__ w_max, int64_t K,
                    float alpha, float *__restrict__ s, float *__restrict__ a_static, float qmax)
{
    __shared__ float red[32];
    const double al = static_cast<double>(alpha);
    float m = 0.0f;
    pdl_wait();
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < K;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float sj = smoothing_factor(act_max[j], w_max[j], al);
        s[j] = sj;
        m = fmaxf(m, __fmul_rn(act_max[j], recip_or_zero(sj)));
    }
    if (a_static != nullptr) {
        m = block_max(m, red);
        if (threadIdx.x == 0) {
            if (gridDim.x == 1) *a_static = __fdiv_rn(m, qmax);      // one block: no pre-zeroing needed
            else atomicMax(reinterpret_cast<int *>(a_static), __float_as_int(__fdiv_rn(m, qmax)));
        }
    }
    __syncthreads();
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// Row kernels
// ---------------------------------------------------------------------------
enum RowMode : int {
    ROW_WEIGHT = 0,      // W' = fl(w*s_j); per-row scale; codes
    ROW_ACT_STATIC = 1,  // x' = fl(x*fl(1/s_j)); codes with the given scale
    ROW_ACT_TOKEN = 2,   // x' as above; per-row scale written; codes
    ROW_RMSNORM = 3,     // y = fl(fl(x*r)*fl(gamma_j*fl(1/s_j))); codes with the given scale
    ROW_RMS_STAT = 4     // running column max of |fl(fl(x*r)*gamma_j)| into scale_out[K] (no codes)
};
// Added to ROW_WEIGHT / ROW_ACT_STATIC / ROW_ACT_TOKEN: E4M3 codes and
// absmax / 448 scales instead of INT8 codes and absmax / 127.
constexpr int ROW_FP8 = 8;
// Added to ROW_WEIGHT: the cross-layer fold.  Row n of the weight is first
// multiplied by fl(1/s_next) of the channel it feeds in the next layer
// (fold_s[n]; for the gate/up interleave only the up rows, fold_s indexed by
// channel), W'[n,j] = fl(fl(W[n,j] * recip(s_next_n)) * s_j).
constexpr int ROW_FOLD = 16;
constexpr int ROW_MODE_MASK = 7;

constexpr int ROW_T = 256;
constexpr int RMS_CL = 8;          // cluster of the norm-output statistic (see k_rows)

struct RowArgs {
    const uint8_t *src0;     // input rows (row r at src0 + r*row_bytes)
    const uint8_t *src1;     // gate/up: up rows (src0 = gate rows), else null
    int64_t rows;            // rows to produce
    int64_t K;               // elements per row
    int64_t row_bytes;       // K * element size
    const float *s;          // [K]
    const float *gamma;      // [K] (RMSNorm)
    float eps;
    const float *a_in;       // static scale [1] (act static, RMSNorm)
    float *scale_out;        // per-row scales [rows] (weight, per-token)
    float *rstd_out;         // RMSNorm r_m [rows] or null
    int8_t *out;             // codes [rows, K]
    unsigned long long timeout_ns;   // bound of the row-ring waits
    const float *fold_s;     // ROW_FOLD: the next layer's smoothing factors of the folded rows
};

// fl(1/s_next) of output row `row` under ROW_FOLD (1 for the gate rows of the
// gate/up interleave, which feed no smoothed layer directly: fl(x * 1) = x)
__device__ __forceinline__ float row_fold_factor(const RowArgs &p, int64_t row)
{
    if (p.src1 != nullptr) {
        const int64_t w = row & 63;
        return w < 32 ? 1.0f : recip_or_zero(p.fold_s[((row >> 6) << 5) + (w & 31)]);
    }
    return recip_or_zero(p.fold_s[row]);
}

// Rows in flight per block in the shared-memory row ring of k_rows, and the
// error code a timed-out ring wait records.
constexpr int RING_ROWS = 3;
constexpr unsigned ERR_ROW_RING = 0x150;

// Codes of EPV values (already multiplied by the scale reciprocal) -> global.
// INRANGE: the values come from a per-row scale and cannot saturate.
template <int EPV, bool INRANGE = false, bool F8 = false>
__device__ __forceinline__ void store_codes(int8_t *dst_row, int64_t v, const float *f)
{
    if constexpr (F8) {
        if constexpr (EPV == 8) {
            uint2 o;
            o.x = e4m3x4_bits(f[0], f[1], f[2], f[3]);
            o.y = e4m3x4_bits(f[4], f[5], f[6], f[7]);
            *reinterpret_cast<uint2 *>(dst_row + v * 8) = o;
        } else {
            *reinterpret_cast<uint32_t *>(dst_row + v * 4) = e4m3x4_bits(f[0], f[1], f[2], f[3]);
        }
    } else {
        uint32_t b[EPV];
#pragma unroll
        for (int e = 0; e < EPV; e += 2) quant8_bits2<INRANGE>(f[e], f[e + 1], b[e], b[e + 1]);
        if constexpr (EPV == 8) {
            uint2 o;
            o.x = pack4_bits(b[0], b[1], b[2], b[3]);
            o.y = pack4_bits(b[4], b[5], b[6], b[7]);
            *reinterpret_cast<uint2 *>(dst_row + v * 8) = o;
        } else {
            *reinterpret_cast<uint32_t *>(dst_row + v * 4) = pack4_bits(b[0], b[1], b[2], b[3]);
        }
    }
}

// y[e] = fl(x[e] * c[e]) for EPV (even) values, two per packed multiply
template <int EPV>
__device__ __forceinline__ void mul_rn_v(float (&y)[EPV], const float (&x)[EPV], const float (&c)[EPV])
{
#pragma unroll
    for (int e = 0; e < EPV; e += 2) {
        const float2 t = __fmul2_rn(make_float2(x[e], x[e + 1]), make_float2(c[e], c[e + 1]));
        y[e] = t.x;
        y[e + 1] = t.y;
    }
}

// y[e] = fl(x[e] * k) for one multiplier k
template <int EPV>
__device__ __forceinline__ void mul_rn_s(float (&y)[EPV], const float (&x)[EPV], float k)
{
#pragma unroll
    for (int e = 0; e < EPV; e += 2) {
        const float2 t = __fmul2_rn(make_float2(x[e], x[e + 1]), make_float2(k, k));
        y[e] = t.x;
        y[e + 1] = t.y;
    }
}

template <int MODE>
__device__ __forceinline__ float column_constant(const RowArgs &p, int64_t j)
{
    if constexpr (MODE == ROW_WEIGHT) return p.s[j];
    else if constexpr (MODE == ROW_RMSNORM) return __fmul_rn(p.gamma[j], recip_or_zero(p.s[j]));
    else if constexpr (MODE == ROW_RMS_STAT) return p.gamma[j];
    else return recip_or_zero(p.s[j]);
}

// The same constants for the four columns 4q..4q+3 from 16-byte loads
// (caller checks that s and gamma are 16-byte aligned).
template <int MODE>
__device__ __forceinline__ float4 column_constant4(const RowArgs &p, int64_t q)
{
    if constexpr (MODE == ROW_WEIGHT) return __ldg(reinterpret_cast<const float4 *>(p.s) + q);
    else if constexpr (MODE == ROW_RMS_STAT) return __ldg(reinterpret_cast<const float4 *>(p.gamma) + q);
    else {
        const float4 s = __ldg(reinterpret_cast<const float4 *>(p.s) + q);
        float4 c = make_float4(recip_or_zero(s.x), recip_or_zero(s.y), recip_or_zero(s.z), recip_or_zero(s.w));
        if constexpr (MODE == ROW_RMSNORM) {
            const float4 g = __ldg(reinterpret_cast<const float4 *>(p.gamma) + q);
            c = make_float4(__fmul_rn(g.x, c.x), __fmul_rn(g.y, c.y), __fmul_rn(g.z, c.z), __fmul_rn(g.w, c.w));
        }
        return c;
    }
}

__device__ __forceinline__ bool constants_aligned16(const RowArgs &p)
{
    return ((reinterpret_cast<uintptr_t>(p.s) | reinterpret_cast<uintptr_t>(p.gamma)) & 15u) == 0;
}

// Thread `tid` owns the 16-byte vectors v = i*NT + tid (i < VPT) of every
// row it touches, so its per-column constants are row-invariant.  REG: they
// (and the pass-1 values) live in registers; otherwise they are read from
// shared memory laid out as EPV/4 planes of float4 (plane h holds elements
// 4h..4h+3 of every vector), which makes the per-thread float4 reads
// conflict-free.  The kernels are issue-bound rather than DRAM-bound at
// these sizes, so vectors past the row end are computed on zeros and only
// their stores are predicated (no divergent branches), and NT = 128 threads
// per row for rows of up to 4096 16-bit elements halves the per-row cost of
// the block reductions.
//
// RING (rows held in registers, modes with a per-row block reduction): the
// rows come through a ring of RING_ROWS row buffers in shared memory filled
// by bulk copies (one per row, issued by thread 0 on an mbarrier), so that
// RING_ROWS rows per block are in flight from HBM whatever the registers
// allow.  A buffer is refilled once every thread has moved its row into
// registers, which the row's block reduction barrier guarantees.  The waits
// are bounded: on expiry the kernel records the error and finishes on
// whatever data it has (no thread leaves early, so no barrier is left short).
template <int DT, int VPT, int MODEF, int NT, bool RING = false>
__global__ void __launch_bounds__(NT) k_rows(RowArgs p)
{
    constexpr int MODE = MODEF & ROW_MODE_MASK;
    constexpr bool F8 = (MODEF & ROW_FP8) != 0;
    constexpr bool FOLD = (MODEF & ROW_FOLD) != 0;
    constexpr int EPV = VecT<DT>::EPV;
    // per-column constants (and the pass-1 values) in registers; 1024-thread
    // rows (long rows) keep them in shared memory to stay within 64 registers,
    // and so does RMSNorm + quant, whose register row and constants would
    // leave room for only 2 blocks per SM (80 registers and 3 blocks with the
    // constants in shared memory: 0.60 -> 0.66 of HBM on 8192-element bf16
    // rows, 0.67 -> 0.72 on 4096-element fp16 rows)
    constexpr bool REG = (VPT * EPV <= 32) && NT <= ROW_T && MODE != ROW_RMSNORM;
    static_assert(!RING || (REG && MODE != ROW_ACT_STATIC), "the row ring needs register rows and a row barrier");
    extern __shared__ __align__(128) float4 colv4[];
    __shared__ float red[32];
    __shared__ double red64[32];
    __shared__ __align__(8) uint64_t ring_full[RING ? RING_ROWS : 1];
    __shared__ int ring_abort;

    const int tid = threadIdx.x;
    const int64_t nvec = p.K / EPV;
    const int64_t plane = nvec;            // float4 entries per plane
    // ring buffers after the statistic's column maxima (the other modes keep
    // no per-column table in shared memory when the row is in registers)
    uint8_t *ring = reinterpret_cast<uint8_t *>(colv4) +
                    (MODE == ROW_RMS_STAT ? ((static_cast<size_t>(p.K) * 4 + 127) & ~size_t(127)) : 0);
    const uint32_t row_bytes32 = static_cast<uint32_t>(p.row_bytes);
    if constexpr (RING) {
        if (tid == 0) {
            for (int s = 0; s < RING_ROWS; ++s) ptx::mbar_init(ptx::smem_addr(&ring_full[s]), 1);
            ring_abort = 0;
            ptx::fence_barrier_init();
        }
        __syncthreads();
    }
    pdl_wait();

    auto row_src = [&](int64_t row) -> const uint8_t * {
        if (p.src1 != nullptr) {          // gate/up interleave: blocks of 64 output rows
            const int64_t b = row >> 6, w = row & 63;
            return (w < 32 ? p.src0 : p.src1) + ((b << 5) + (w & 31)) * p.row_bytes;
        }
        return p.src0 + row * p.row_bytes;
    };
    auto load_row = [&](int64_t row, uint4 (&dst)[VPT]) {
        const uint4 *src = reinterpret_cast<const uint4 *>(row_src(row));
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int64_t v = static_cast<int64_t>(i) * NT + tid;
            dst[i] = (v < nvec) ? __ldcs(src + v) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // local row i of this block -> ring buffer i % RING_ROWS
    auto ring_issue = [&](int64_t i) {
        const int64_t row = blockIdx.x + i * gridDim.x;
        if (row < p.rows) {
            const int sl = static_cast<int>(i % RING_ROWS);
            const uint32_t bar = ptx::smem_addr(&ring_full[sl]);
            ptx::mbar_arrive_expect_tx(bar, row_bytes32);
            ptx::bulk_load(ptx::smem_addr(ring) + static_cast<uint32_t>(sl) * row_bytes32, row_src(row), row_bytes32,
                           bar);
        }
    };
    auto ring_take = [&](int64_t i, uint4 (&dst)[VPT]) {
        const int sl = static_cast<int>(i % RING_ROWS);
        const uint32_t par = static_cast<uint32_t>((i / RING_ROWS) & 1);
        ptx::wait_bounded(ptx::smem_addr(&ring_full[sl]), par, p.timeout_ns, &ring_abort, ERR_ROW_RING);
        const uint4 *src = reinterpret_cast<const uint4 *>(ring + static_cast<size_t>(sl) * p.row_bytes);
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int64_t v = static_cast<int64_t>(k) * NT + tid;
            dst[k] = (v < nvec) ? src[v] : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // Without the ring, rows of up to 8 vectors per thread keep the next
    // row's loads in flight while a row is processed; the first row is
    // requested before the per-column constants, so that the two loads
    // overlap.
    constexpr bool PF = !RING && VPT <= 8;
    uint4 nxt[PF ? VPT : 1];
    if constexpr (PF) {
        if (blockIdx.x < p.rows) load_row(blockIdx.x, nxt);
    }
    if constexpr (RING) {
        if (tid == 0)
            for (int i = 0; i < RING_ROWS; ++i) ring_issue(i);
    }

    const bool c16 = constants_aligned16(p);
    float creg[REG ? VPT : 1][REG ? EPV : 1];
    if constexpr (REG) {
        if (c16) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int64_t v = static_cast<int64_t>(i) * NT + tid;
#pragma unroll
                for (int h = 0; h < EPV / 4; ++h) {
                    const float4 t = (v < nvec) ? column_constant4<MODE>(p, v * (EPV / 4) + h)
                                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    creg[i][4 * h] = t.x; creg[i][4 * h + 1] = t.y; creg[i][4 * h + 2] = t.z; creg[i][4 * h + 3] = t.w;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int64_t v = static_cast<int64_t>(i) * NT + tid;
#pragma unroll
                for (int e = 0; e < EPV; ++e) creg[i][e] = (v < nvec) ? column_constant<MODE>(p, v * EPV + e) : 0.0f;
            }
        }
    } else if (c16) {
        // 16-byte loads, 8 per thread in flight: float4 q holds columns 4q..4q+3,
        // i.e. plane q % (EPV/4) of vector q / (EPV/4)
        const int64_t nq = p.K / 4;
        for (int64_t q0 = tid; q0 < nq; q0 += 8 * NT) {
            float4 c[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t q = q0 + static_cast<int64_t>(u) * NT;
                if (q < nq) c[u] = column_constant4<MODE>(p, q);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t q = q0 + static_cast<int64_t>(u) * NT;
                if (q < nq) colv4[(q % (EPV / 4)) * plane + q / (EPV / 4)] = c[u];
            }
        }
        __syncthreads();
    } else {
        // 8 columns per step: the loads of a step are independent and overlap
        float *cv = reinterpret_cast<float *>(colv4);
        for (int64_t j0 = tid; j0 < p.K; j0 += 8 * NT) {
            float c[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t j = j0 + static_cast<int64_t>(u) * NT;
                c[u] = (j < p.K) ? column_constant<MODE>(p, j) : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t j = j0 + static_cast<int64_t>(u) * NT;
                if (j < p.K) {
                    const int64_t v = j / EPV;
                    const int e = static_cast<int>(j % EPV);
                    cv[((e >> 2) * plane + v) * 4 + (e & 3)] = c[u];
                }
            }
        }
        __syncthreads();
    }
    // constants of vector slot i (vectors past the row end read a valid
    // entry; their results are never stored)
    auto colc = [&](int i, int64_t v, float (&c)[EPV]) {
        if constexpr (REG) {
#pragma unroll
            for (int e = 0; e < EPV; ++e) c[e] = creg[i][e];
        } else {
            const int64_t vc = v < nvec ? v : nvec - 1;
#pragma unroll
            for (int h = 0; h < EPV / 4; ++h) {
                const float4 t = colv4[h * plane + vc];
                c[4 * h] = t.x; c[4 * h + 1] = t.y; c[4 * h + 2] = t.z; c[4 * h + 3] = t.w;
            }
        }
    };
    float inv_a_static = 0.0f;
    if constexpr (MODE == ROW_ACT_STATIC || MODE == ROW_RMSNORM) inv_a_static = recip_or_zero(p.a_in[0]);
    const bool k_pow2 = (p.K & (p.K - 1)) == 0;
    const double k_recip = 1.0 / static_cast<double>(p.K);
    float cmax[MODE == ROW_RMS_STAT ? VPT : 1][MODE == ROW_RMS_STAT ? EPV : 1];
    if constexpr (MODE == ROW_RMS_STAT) {
        static_assert(REG, "the norm-output statistic keeps its column maxima in registers");
#pragma unroll
        for (int i = 0; i < VPT; ++i)
#pragma unroll
            for (int e = 0; e < EPV; ++e) cmax[i][e] = 0.0f;
    }

    int64_t li = 0;                        // local row index (ring position)
    for (int64_t row = blockIdx.x; row < p.rows; row += gridDim.x, ++li) {
        uint4 raw[VPT];
        if constexpr (RING) {
            ring_take(li, raw);
        } else if constexpr (PF) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) raw[i] = nxt[i];
            if (row + gridDim.x < p.rows) load_row(row + gridDim.x, nxt);
        } else {
            load_row(row, raw);
        }
        // after the row's block barrier every thread holds its part of the
        // row in registers: refill the buffer with the row RING_ROWS ahead
        auto ring_refill = [&]() {
            if constexpr (RING) {
                if (tid == 0) {
                    ptx::fence_proxy_async_smem();
                    ring_issue(li + RING_ROWS);
                }
            }
        };
        int8_t *dst = p.out + row * p.K;

        if constexpr (MODE == ROW_ACT_STATIC) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int64_t v = static_cast<int64_t>(i) * NT + tid;
                float f[EPV], c[EPV];
                widen<DT>(raw[i], f);
                colc(i, v, c);
                mul_rn_v(f, f, c);
                mul_rn_s(f, f, inv_a_static);
                if (v < nvec) store_codes<EPV, false, F8>(dst, v, f);
            }
            continue;
        }

        if constexpr (MODE == ROW_RMSNORM || MODE == ROW_RMS_STAT) {
            // pass 1: sum of squares in fp64 (exact squares); REG keeps the
            // widened row for pass 2
            // (four independent partial sums: the row's latency rather than
            // the issue rate bounds this kernel, and a single chain of
            // dependent fp64 adds per thread was a large part of it)
            float fk[REG ? VPT : 1][REG ? EPV : 1];
            double ss4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float f[EPV];
                widen<DT>(raw[i], f);
#pragma unroll
                for (int e = 0; e < EPV; ++e) {
                    ss4[e & 3] += static_cast<double>(f[e]) * static_cast<double>(f[e]);
                    if constexpr (REG) fk[i][e] = f[e];
                }
            }
            const double tot = block_sum_f64_nw<NT / 32>((ss4[0] + ss4[1]) + (ss4[2] + ss4[3]), red64);
            ring_refill();
            // a power-of-two K divides exactly by its reciprocal (the same result as the division)
            const double mean64 = k_pow2 ? tot * k_recip : tot / static_cast<double>(p.K);
            const float mean = __double2float_rn(mean64);
            const float r_m = __frcp_rn(__fsqrt_rn(__fadd_rn(mean, p.eps)));
            if (tid == 0 && p.rstd_out != nullptr) p.rstd_out[row] = r_m;
            // pass 2: y = fl(fl(x * r_m) * c_j), then (RMSNorm) v = fl(y * recip(a)).
            // With the row in registers the values v overwrite it until the
            // thread's largest magnitude is known: below 127.5 (and not NaN)
            // no code saturates and the clamp is skipped.  Otherwise the check
            // is made per vector.
            float vmax = 0.0f;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int64_t v = static_cast<int64_t>(i) * NT + tid;
                float f[EPV], c[EPV];
                if constexpr (REG) {
#pragma unroll
                    for (int e = 0; e < EPV; ++e) f[e] = fk[i][e];
                } else {
                    widen<DT>(raw[i], f);
                }
                colc(i, v, c);
                mul_rn_s(f, f, r_m);
                mul_rn_v(f, f, c);
                if constexpr (MODE == ROW_RMS_STAT) {
#pragma unroll
                    for (int e = 0; e < EPV; ++e) cmax[i][e] = fmaxf(cmax[i][e], fabsf(f[e]));
                } else {
                    mul_rn_s(f, f, inv_a_static);
                    float m = 0.0f;
#pragma unroll
                    for (int e = 0; e < EPV; e += 2) m = max3_abs_nan(m, f[e], f[e + 1]);
                    if constexpr (REG) {
#pragma unroll
                        for (int e = 0; e < EPV; ++e) fk[i][e] = f[e];
                        vmax = max3_abs_nan(vmax, m, 0.0f);
                    } else if (v < nvec) {
                        if (m < 127.5f) store_codes<EPV, true>(dst, v, f);
                        else store_codes<EPV, false>(dst, v, f);
                    }
                }
            }
            if constexpr (MODE == ROW_RMSNORM && REG) {
                if (vmax < 127.5f) {
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int64_t v = static_cast<int64_t>(i) * NT + tid;
                        if (v < nvec) store_codes<EPV, true>(dst, v, fk[i]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int64_t v = static_cast<int64_t>(i) * NT + tid;
                        if (v < nvec) store_codes<EPV, false>(dst, v, fk[i]);
                    }
                }
            }
            continue;
        }

        // ROW_WEIGHT / ROW_ACT_TOKEN: pass 1 y = fl(x * c_j) and the row absmax,
        // pass 2 codes of fl(y * recip(scale)).  REG keeps y in registers.
        float ykeep[REG ? VPT : 1][REG ? EPV : 1];
        float mx = 0.0f;
        const float rf = FOLD ? row_fold_factor(p, row) : 1.0f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int64_t v = static_cast<int64_t>(i) * NT + tid;
            float f[EPV], c[EPV];
            widen<DT>(raw[i], f);
            colc(i, v, c);
            if constexpr (FOLD) mul_rn_s(f, f, rf);
            mul_rn_v(f, f, c);
#pragma unroll
            for (int e = 0; e < EPV; e += 2) {
                mx = max3_abs(mx, f[e], f[e + 1]);
                if constexpr (REG) {
                    ykeep[i][e] = f[e];
                    ykeep[i][e + 1] = f[e + 1];
                }
            }
        }
        const float sc = scale_from_absmax_q<F8>(block_max(mx, red));
        ring_refill();
        const float inv = recip_or_zero(sc);
        if (tid == 0) p.scale_out[row] = sc;
        // with a normal (or zero) scale the row's codes cannot saturate
        const bool inrange = (sc == 0.0f) || (sc >= 1.17549435e-38f);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int64_t v = static_cast<int64_t>(i) * NT + tid;
            float f[EPV];
            if constexpr (REG) {
                mul_rn_s(f, ykeep[i], inv);
            } else {
                float c[EPV];
                widen<DT>(raw[i], f);
                colc(i, v, c);
                if constexpr (FOLD) mul_rn_s(f, f, rf);
                mul_rn_v(f, f, c);
                mul_rn_s(f, f, inv);
            }
            if (v < nvec) {
                if (F8) store_codes<EPV, false, F8>(dst, v, f);
                else if (inrange) store_codes<EPV, true>(dst, v, f);
                else store_codes<EPV, false>(dst, v, f);
            }
        }
    }
    if constexpr (RING) {
        // after a timed-out wait, no block leaves while a bulk copy may still
        // be writing its shared memory
        if (tid == 0 && ring_abort) {
            volatile int no_abort = 0;
            for (int64_t i = li > RING_ROWS ? li - RING_ROWS : 0; i < li; ++i)
                ptx::wait_bounded(ptx::smem_addr(&ring_full[i % RING_ROWS]), static_cast<uint32_t>((i / RING_ROWS) & 1),
                                  p.timeout_ns, &no_abort, ERR_ROW_RING);
        }
    }
    if constexpr (MODE == ROW_RMS_STAT) {
        // Launched in clusters (few rows per block, where the atomics would
        // dominate), the blocks of a cluster first combine their column maxima
        // through distributed shared memory: CTA r takes every n-th slice of
        // the columns and issues the atomics for it, n times fewer atomics on
        // the same addresses than one per column per block.
        float *cm = reinterpret_cast<float *>(colv4);    // [K] (dynamic shared memory)
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int64_t v = static_cast<int64_t>(i) * NT + tid;
            if (v < nvec) {
#pragma unroll
                for (int e = 0; e < EPV; ++e) cm[v * EPV + e] = cmax[i][e];
            }
        }
        ptx::cluster_sync();                            // every block's maxima written
        const uint32_t rank = ptx::cluster_ctarank();
        const int ncl = static_cast<int>(ptx::cluster_nctarank());   // 1 when launched without a cluster
        const uint32_t local = ptx::smem_addr(cm);
        for (int64_t j = static_cast<int64_t>(rank) * NT + tid; j < p.K; j += static_cast<int64_t>(ncl) * NT) {
            float m = 0.0f;
#pragma unroll 1
            for (int c = 0; c < ncl; ++c) {
                float o;
                asm volatile("ld.shared::cluster.f32 %0, [%1];"
                             : "=f"(o)
                             : "r"(ptx::map_to_rank(local + static_cast<uint32_t>(j) * 4u, static_cast<uint32_t>(c)))
                             : "memory");
                m = fmaxf(m, o);
            }
            atomicMax(reinterpret_cast<int *>(p.scale_out + j), __float_as_int(m));
        }
        ptx::cluster_sync();                            // no block leaves while its maxima are read
    }
    __syncthreads();
    pdl_trigger();
}

// Static (per-tensor) activation quantisation is elementwise: code(x) =
// q(fl(fl(x * recip(s_j)) * recip(a))).  It streams like the calibration
// kernel: a block is a strip of 32 16-byte column vectors x 8 row lanes, each
// thread keeps its vector's 1/s_j in registers and walks a slab of rows,
// four rows at a time with the next four rows' loads in flight, writing 8
// codes (16-bit inputs) or 4 (fp32) per vector: a warp reads 512 and writes
// 256 contiguous bytes.
constexpr int QS_TX = 32, QS_TY = 8, QS_UNROLL = 4;

// ONE: every slab is at most one batch (QS_UNROLL x QS_TY rows), so no
// second batch buffer is kept (fewer registers, more blocks resident: small
// tensors are latency-bound).
template <int DT, bool STREAM, bool ONE, bool F8 = false>
__global__ void __launch_bounds__(QS_TX *QS_TY)
    k_quant_static(const uint8_t *__restrict__ x, int64_t rows, int64_t nvec, const float *__restrict__ s,
                   const float *__restrict__ a_in, int64_t row_slab, int8_t *__restrict__ out)
{
    constexpr int EPV = VecT<DT>::EPV;
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int64_t v = static_cast<int64_t>(blockIdx.x) * QS_TX + tx;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * row_slab;
    const int64_t r1 = min(rows, r0 + row_slab);
    const int64_t K = nvec * EPV;
    pdl_wait();
    if (v < nvec) {
        const uint8_t *col = x + v * 16;
        auto load = [&](int64_t r) {
            const uint4 *p = reinterpret_cast<const uint4 *>(col + r * nvec * 16);
            if constexpr (STREAM) return __ldcs(p);
            else return __ldg(p);
        };
        // first rows in flight before the constants
        uint4 t[QS_UNROLL];
        int64_t r = r0 + ty;
#pragma unroll
        for (int u = 0; u < QS_UNROLL; ++u)
            if (r + u * QS_TY < r1) t[u] = load(r + u * QS_TY);
        float c[EPV];
        if ((reinterpret_cast<uintptr_t>(s) & 15u) == 0) {
#pragma unroll
            for (int h = 0; h < EPV / 4; ++h) {
                const float4 w = __ldg(reinterpret_cast<const float4 *>(s) + v * (EPV / 4) + h);
                c[4 * h] = recip_or_zero(w.x); c[4 * h + 1] = recip_or_zero(w.y);
                c[4 * h + 2] = recip_or_zero(w.z); c[4 * h + 3] = recip_or_zero(w.w);
            }
        } else {
#pragma unroll
            for (int e = 0; e < EPV; ++e) c[e] = recip_or_zero(s[v * EPV + e]);
        }
        const float inv_a = recip_or_zero(a_in[0]);
        auto emit = [&](int64_t row, const uint4 &raw) {
            float f[EPV];
            widen<DT>(raw, f);
            mul_rn_v(f, f, c);
            mul_rn_s(f, f, inv_a);
            int8_t *dst = out + row * K;
            if constexpr (F8) {
                if constexpr (EPV == 8) {
                    __stcs(reinterpret_cast<uint2 *>(dst + v * 8), make_uint2(e4m3x4_bits(f[0], f[1], f[2], f[3]),
                                                                              e4m3x4_bits(f[4], f[5], f[6], f[7])));
                } else {
                    __stcs(reinterpret_cast<uint32_t *>(dst + v * 4), e4m3x4_bits(f[0], f[1], f[2], f[3]));
                }
            } else {
                // always clamped: skipping the clamp behind a per-vector range
                // check split the four unrolled rows into separate branches
                // and measured 8 % slower (0.86 -> 0.79 of HBM)
                uint32_t b[EPV];
#pragma unroll
                for (int e = 0; e < EPV; e += 2) quant8_bits2<false>(f[e], f[e + 1], b[e], b[e + 1]);
                if constexpr (EPV == 8)
                    __stcs(reinterpret_cast<uint2 *>(dst + v * 8),
                           make_uint2(pack4_bits(b[0], b[1], b[2], b[3]), pack4_bits(b[4], b[5], b[6], b[7])));
                else
                    __stcs(reinterpret_cast<uint32_t *>(dst + v * 4), pack4_bits(b[0], b[1], b[2], b[3]));
            }
        };
        if constexpr (ONE) {
#pragma unroll
            for (int u = 0; u < QS_UNROLL; ++u)
                if (r + u * QS_TY < r1) emit(r + u * QS_TY, t[u]);
        } else {
            // the next batch of rows is requested before this one is converted
            for (;;) {
                const int64_t rn = r + QS_UNROLL * QS_TY;
                uint4 n[QS_UNROLL];
#pragma unroll
                for (int u = 0; u < QS_UNROLL; ++u)
                    if (rn + u * QS_TY < r1) n[u] = load(rn + u * QS_TY);
#pragma unroll
                for (int u = 0; u < QS_UNROLL; ++u)
                    if (r + u * QS_TY < r1) emit(r + u * QS_TY, t[u]);
                if (rn >= r1) break;
#pragma unroll
                for (int u = 0; u < QS_UNROLL; ++u) t[u] = n[u];
                r = rn;
            }
        }
    }
    __syncthreads();
    pdl_trigger();
}

// Few rows (decode-size activations): a cluster of CS CTAs shares each row,
// CTA r of the cluster taking the 16-byte vectors [r*vpc, (r+1)*vpc) with
// vpc = nvec / CS <= ROW_T, one vector per thread.  The row-wide reduction
// (absmax, or the fp64 sum of squares of RMSNorm) combines the CTAs'
// partials through distributed shared memory, in rank order, so that every
// CTA of the cluster obtains the same value; the arithmetic per element is
// that of k_rows.  grid = (CS, rows), cluster = (CS, 1, 1).
__device__ __forceinline__ double ld_dsmem_f64(uint32_t addr)
{
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(addr) : "memory");
    return v;
}

template <int DT, int MODEF>
__global__ void __launch_bounds__(ROW_T) k_rows_split(RowArgs p)
{
    constexpr int MODE = MODEF & ROW_MODE_MASK;
    constexpr bool F8 = (MODEF & ROW_FP8) != 0;
    constexpr bool FOLD = (MODEF & ROW_FOLD) != 0;
    constexpr int EPV = VecT<DT>::EPV;
    __shared__ float red[32];
    __shared__ double red64[32];
    __shared__ double part;            // this CTA's partial of the row reduction
    __shared__ double total;           // the combined value
    const int tid = threadIdx.x;
    const int cs = static_cast<int>(gridDim.x);
    const uint32_t rank = ptx::cluster_ctarank();
    const int64_t row = blockIdx.y;
    const int64_t nvec = p.K / EPV;
    const int64_t vpc = nvec / cs;
    const int64_t v = static_cast<int64_t>(rank) * vpc + tid;
    const bool act = tid < vpc;
    pdl_wait();

    const uint8_t *src;
    if (p.src1 != nullptr) {
        const int64_t b = row >> 6, w = row & 63;
        src = (w < 32 ? p.src0 : p.src1) + ((b << 5) + (w & 31)) * p.row_bytes;
    } else {
        src = p.src0 + row * p.row_bytes;
    }
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (act) raw = __ldcs(reinterpret_cast<const uint4 *>(src) + v);
    float c[EPV];
    if (act) {
        if (constants_aligned16(p)) {
#pragma unroll
            for (int h = 0; h < EPV / 4; ++h) {
                const float4 t = column_constant4<MODE>(p, v * (EPV / 4) + h);
                c[4 * h] = t.x; c[4 * h + 1] = t.y; c[4 * h + 2] = t.z; c[4 * h + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < EPV; ++e) c[e] = column_constant<MODE>(p, v * EPV + e);
        }
    } else {
#pragma unroll
        for (int e = 0; e < EPV; ++e) c[e] = 0.0f;
    }
    float f[EPV];
    widen<DT>(raw, f);
    int8_t *dst = p.out + row * p.K;

    // row-wide value through the cluster: partials in rank order
    auto cluster_combine = [&](double mine, bool is_max) -> double {
        if (tid == 0) part = mine;
        ptx::cluster_sync();                           // every partial written
        if (tid == 0) {
            const uint32_t local = ptx::smem_addr(&part);
            double acc = 0.0;
            for (int r = 0; r < cs; ++r) {
                const double o = ld_dsmem_f64(ptx::map_to_rank(local, static_cast<uint32_t>(r)));
                acc = is_max ? fmax(acc, o) : acc + o;
            }
            total = acc;
        }
        ptx::cluster_sync();                           // every partial read: peers may exit
        return total;
    };

    if constexpr (MODE == ROW_ACT_STATIC) {
        if (act) {
            const float inv_a = recip_or_zero(p.a_in[0]);
#pragma unroll
            for (int e = 0; e < EPV; ++e) f[e] = __fmul_rn(__fmul_rn(f[e], c[e]), inv_a);
            store_codes<EPV, false, F8>(dst, v, f);
        }
    } else if constexpr (MODE == ROW_RMSNORM || MODE == ROW_RMS_STAT) {
        double ss = 0.0;
        if (act) {
#pragma unroll
            for (int e = 0; e < EPV; ++e) ss += static_cast<double>(f[e]) * static_cast<double>(f[e]);
        }
        const double tot = cluster_combine(block_sum_f64(ss, red64), false);
        const float mean = __double2float_rn(tot / static_cast<double>(p.K));
        const float r_m = __frcp_rn(__fsqrt_rn(__fadd_rn(mean, p.eps)));
        if (rank == 0 && tid == 0 && p.rstd_out != nullptr) p.rstd_out[row] = r_m;
        if (act) {
            if constexpr (MODE == ROW_RMS_STAT) {
#pragma unroll
                for (int e = 0; e < EPV; ++e)
                    atomicMax(reinterpret_cast<int *>(p.scale_out + v * EPV + e),
                              __float_as_int(fabsf(__fmul_rn(__fmul_rn(f[e], r_m), c[e]))));
            } else {
                const float inv_a = recip_or_zero(p.a_in[0]);
#pragma unroll
                for (int e = 0; e < EPV; ++e) f[e] = __fmul_rn(__fmul_rn(__fmul_rn(f[e], r_m), c[e]), inv_a);
                store_codes<EPV>(dst, v, f);
            }
        }
    } else {
        // ROW_WEIGHT / ROW_ACT_TOKEN: y = fl(x * c_j), row absmax, codes of fl(y * recip(scale))
        float mx = 0.0f;
        const float rf = FOLD ? row_fold_factor(p, row) : 1.0f;
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
            f[e] = __fmul_rn(FOLD ? __fmul_rn(f[e], rf) : f[e], c[e]);
            mx = fmaxf(mx, fabsf(f[e]));
        }
        const float rmax = static_cast<float>(cluster_combine(static_cast<double>(block_max(mx, red)), true));
        const float sc = scale_from_absmax_q<F8>(rmax);
        const float inv = recip_or_zero(sc);
        if (rank == 0 && tid == 0) p.scale_out[row] = sc;
        if (act) {
#pragma unroll
            for (int e = 0; e < EPV; ++e) f[e] = __fmul_rn(f[e], inv);
            if (F8) store_codes<EPV, false, F8>(dst, v, f);
            else if ((sc == 0.0f) || (sc >= 1.17549435e-38f)) store_codes<EPV, true>(dst, v, f);
            else store_codes<EPV, false>(dst, v, f);
        }
    }
    __syncthreads();
    pdl_trigger();
}

// Unaligned / very wide rows: one block per row, elementwise, two passes
// over global memory (correct for any K; not tuned).
template <int MODEF>
__global__ void __launch_bounds__(ROW_T) k_rows_scalar(RowArgs p, int dt)
{
    constexpr int MODE = MODEF & ROW_MODE_MASK;
    constexpr bool F8 = (MODEF & ROW_FP8) != 0;
    constexpr bool FOLD = (MODEF & ROW_FOLD) != 0;
    __shared__ float red[32];
    __shared__ double red64[32];
    const int tid = threadIdx.x;
    pdl_wait();
    float inv_a_static = 0.0f;
    if constexpr (MODE == ROW_ACT_STATIC || MODE == ROW_RMSNORM) inv_a_static = recip_or_zero(p.a_in[0]);
    for (int64_t row = blockIdx.x; row < p.rows; row += gridDim.x) {
        const uint8_t *src;
        if (p.src1 != nullptr) {
            const int64_t b = row >> 6, w = row & 63;
            src = (w < 32 ? p.src0 : p.src1) + ((b << 5) + (w & 31)) * p.row_bytes;
        } else {
            src = p.src0 + row * p.row_bytes;
        }
        auto colc = [&](int64_t j) -> float {
            if constexpr (MODE == ROW_WEIGHT) return p.s[j];
            else if constexpr (MODE == ROW_RMSNORM) return __fmul_rn(p.gamma[j], recip_or_zero(p.s[j]));
            else if constexpr (MODE == ROW_RMS_STAT) return p.gamma[j];
            else return recip_or_zero(p.s[j]);
        };
        float stat = 0.0f;
        double ss = 0.0;
        const float rf = FOLD ? row_fold_factor(p, row) : 1.0f;
        if constexpr (MODE != ROW_ACT_STATIC) {
            for (int64_t j = tid; j < p.K; j += ROW_T) {
                const float x = FOLD ? __fmul_rn(load_elem_dt(src, dt, j), rf) : load_elem_dt(src, dt, j);
                if constexpr (MODE == ROW_RMSNORM || MODE == ROW_RMS_STAT)
                    ss += static_cast<double>(x) * static_cast<double>(x);
                else stat = fmaxf(stat, fabsf(__fmul_rn(x, colc(j))));
            }
        }
        float mul_a, r_m = 0.0f;
        if constexpr (MODE == ROW_ACT_STATIC) {
            mul_a = inv_a_static;
        } else if constexpr (MODE == ROW_RMSNORM || MODE == ROW_RMS_STAT) {
            const double tot = block_sum_f64(ss, red64);
            const float mean = __double2float_rn(tot / static_cast<double>(p.K));
            r_m = __frcp_rn(__fsqrt_rn(__fadd_rn(mean, p.eps)));
            mul_a = inv_a_static;
            if (tid == 0 && p.rstd_out != nullptr) p.rstd_out[row] = r_m;
        } else {
            const float sc = scale_from_absmax_q<F8>(block_max(stat, red));
            mul_a = recip_or_zero(sc);
            if (tid == 0) p.scale_out[row] = sc;
        }
        for (int64_t j = tid; j < p.K; j += ROW_T) {
            const float x = FOLD ? __fmul_rn(load_elem_dt(src, dt, j), rf) : load_elem_dt(src, dt, j);
            float y;
            if constexpr (MODE == ROW_RMSNORM || MODE == ROW_RMS_STAT) y = __fmul_rn(__fmul_rn(x, r_m), colc(j));
            else y = __fmul_rn(x, colc(j));
            if constexpr (MODE == ROW_RMS_STAT)
                atomicMax(reinterpret_cast<int *>(p.scale_out + j), __float_as_int(fabsf(y)));
            else if constexpr (F8)
                p.out[row * p.K + j] = static_cast<int8_t>(e4m3x2_bits(__fmul_rn(y, mul_a), 0.0f) & 0xffu);
            else
                p.out[row * p.K + j] = static_cast<int8_t>(quant8(__fmul_rn(y, mul_a)));
        }
        __syncthreads();
    }
    __syncthreads();
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// fp16 storage of scales ("010. SmoothQuant Integration", consequences:
// storage): fp32 -> fp16 round to nearest even, and the exact widening back.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_f32_to_f16(const float *__restrict__ in, int64_t n, __half *__restrict__ out)
{
    pdl_wait();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[i] = __float2half_rn(in[i]);
    __syncthreads();
    pdl_trigger();
}

__global__ void __launch_bounds__(256) k_f16_to_f32(const __half *__restrict__ in, int64_t n, float *__restrict__ out)
{
    pdl_wait();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[i] = __half2float(in[i]);
    __syncthreads();
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// Sum of squared differences of two fp16 tensors, fp64 accumulation.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    k_sse_f16(const __half *__restrict__ y, const __half *__restrict__ r, int64_t n, double *__restrict__ sse)
{
    __shared__ double red[8];
    double acc = 0.0;
    const int64_t nv = n / 8;
    pdl_wait();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nv; v += stride) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(y) + v);
        const uint4 b = __ldg(reinterpret_cast<const uint4 *>(r) + v);
        const __half *ha = reinterpret_cast<const __half *>(&a);
        const __half *hb = reinterpret_cast<const __half *>(&b);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double d = static_cast<double>(__half2float(ha[e])) - static_cast<double>(__half2float(hb[e]));
            acc += d * d;
        }
    }
    for (int64_t i = nv * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        const double d = static_cast<double>(__half2float(y[i])) - static_cast<double>(__half2float(r[i]));
        acc += d * d;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int i = 0; i < (blockDim.x >> 5); ++i) t += red[i];
        atomicAdd(sse, t);
    }
    __syncthreads();
    pdl_trigger();
}

}  // namespace sq
