// robust.cuh -- robust calibration statistics (kwkr.cn blog 3.1: in place of
// the per-channel max, a high quantile such as 99.9 % of |X_j| over the
// calibration tokens, or the mean of several samples' maxima, so that one
// abnormal token does not set the channel's smoothing factor).
//
// Mean of per-batch maxima: per calibration batch, the ordinary column absmax
// (k_colabsmax) into a zeroed fp32 scratch vector, then k_batchmax_accumulate
// adds it to an fp64 running sum (one add per batch, in call order) and
// re-zeroes the scratch; k_mean_of_max divides by the batch count in fp64 and
// rounds once to fp32.
//
// Quantile by nearest rank: the k-th smallest |x_tj| of each column, k =
// ceil(p * T) (host, fp64).  |x| of a 16-bit or fp32 value is its bit pattern
// with the sign cleared, and non-negative floats order like those integers,
// so the k-th smallest value is found by a radix select on the magnitude
// bits, most significant digit first: 15 bits (fp16 / bf16) in digits of 8
// and 7 bits, 31 bits (fp32) in 8 + 8 + 8 + 7.  Each digit is one streaming
// pass over the tensor (k_quantile_hist: a per-column histogram of the digit
// among the elements whose higher bits equal the column's prefix so far) and
// one small pass over the histograms (k_quantile_select: the bin holding
// rank k, which extends the prefix and lowers k by the count below it).  The
// result is one of the data values, exactly.
#pragma once

#include "common.cuh"

namespace sq {

// ------------------------------------------------------------- mean of maxima
__global__ void __launch_bounds__(256)
    k_batchmax_accumulate(float *__restrict__ batch_max, double *__restrict__ sum_max, int64_t cols)
{
    pdl_wait();
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < cols;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        sum_max[j] += static_cast<double>(batch_max[j]);
        batch_max[j] = 0.0f;
    }
    __syncthreads();
    pdl_trigger();
}

__global__ void __launch_bounds__(256)
    k_mean_of_max(const double *__restrict__ sum_max, int64_t cols, double n_batches, float *__restrict__ out)
{
    pdl_wait();
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < cols;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[j] = __double2float_rn(__ddiv_rn(sum_max[j], n_batches));
    __syncthreads();
    pdl_trigger();
}

// ------------------------------------------------------------- quantile
constexpr int QH_COLS = 128;       // columns per block strip
constexpr int QH_THREADS = 512;
constexpr int QH_BINS = 256;       // bins of one digit (at most 8 bits)
constexpr int QH_STRIDE = 257;     // shared histogram row stride: column c's bin b sits in bank (c + b) % 32
constexpr int QH_UNROLL = 4;
constexpr int QH_SMEM = QH_COLS * QH_STRIDE * 4;

template <int DT> struct MagBits {
    static constexpr int NB = DT == DT_F32 ? 31 : 15;     // magnitude bits
};

// the magnitude bit patterns of the EPV elements of a 16-byte vector
template <int DT>
__device__ __forceinline__ void mag_bits(const uint4 &v, uint32_t (&b)[VecT<DT>::EPV])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if constexpr (DT == DT_F32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) b[i] = w[i] & 0x7fffffffu;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            b[2 * i] = w[i] & 0x7fffu;
            b[2 * i + 1] = (w[i] >> 16) & 0x7fffu;
        }
    }
}

// One digit pass: hist[col][digit] += #{t : bits(x_t,col) >> (shift + width) == prefix[col]},
// digit = (bits >> shift) & (2^width - 1).  prefix == nullptr: the first digit
// (every element counts).  A block takes a strip of QH_COLS columns and a slab
// of rows; its histogram lives in shared memory and is added to the global one
// (nonzero bins only) at the end.  Rows are 16-byte aligned (ld_bytes % 16 == 0).
template <int DT>
__global__ void __launch_bounds__(QH_THREADS)
    k_quantile_hist(const uint8_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld_bytes, int64_t row_slab,
                    int shift, int width, const uint32_t *__restrict__ prefix, uint32_t *__restrict__ hist)
{
    constexpr int EPV = VecT<DT>::EPV;
    constexpr int VPS = QH_COLS / EPV;                 // vectors per strip
    constexpr int LANES = QH_THREADS / VPS;            // row lanes
    extern __shared__ uint32_t sh[];                   // [QH_COLS][QH_STRIDE]
    const int tid = threadIdx.x;
    const int tx = tid % VPS, ty = tid / VPS;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * QH_COLS;
    const int64_t col = c0 + static_cast<int64_t>(tx) * EPV;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * row_slab;
    const int64_t r1 = min(rows, r0 + row_slab);
    const int hi = shift + width;
    const uint32_t mask = (1u << width) - 1u;

    for (int i = tid; i < QH_COLS * QH_STRIDE; i += QH_THREADS) sh[i] = 0u;
    pdl_wait();
    uint32_t pre[EPV];
#pragma unroll
    for (int e = 0; e < EPV; ++e) pre[e] = (prefix != nullptr && col + e < cols) ? prefix[col + e] : 0u;
    __syncthreads();

    if (col < cols) {                                   // cols is a multiple of EPV (aligned rows)
        const uint8_t *p = x + col * (DT == DT_F32 ? 4 : 2);
        uint32_t *hrow = sh + tx * EPV * QH_STRIDE;
        auto count = [&](const uint4 &v) {
            uint32_t b[EPV];
            mag_bits<DT>(v, b);
#pragma unroll
            for (int e = 0; e < EPV; ++e)
                if ((b[e] >> hi) == pre[e]) atomicAdd(hrow + e * QH_STRIDE + ((b[e] >> shift) & mask), 1u);
        };
        int64_t r = r0 + ty;
        for (; r + (QH_UNROLL - 1) * LANES < r1; r += QH_UNROLL * LANES) {
            uint4 t[QH_UNROLL];
#pragma unroll
            for (int u = 0; u < QH_UNROLL; ++u)
                t[u] = __ldcs(reinterpret_cast<const uint4 *>(p + (r + u * LANES) * ld_bytes));
#pragma unroll
            for (int u = 0; u < QH_UNROLL; ++u) count(t[u]);
        }
        for (; r < r1; r += LANES) count(__ldcs(reinterpret_cast<const uint4 *>(p + r * ld_bytes)));
    }
    __syncthreads();
    const int nb = 1 << width;
    for (int i = tid; i < QH_COLS * nb; i += QH_THREADS) {
        const int c = i / nb, b = i - c * nb;
        const uint32_t n = sh[c * QH_STRIDE + b];
        if (n != 0u && c0 + c < cols) atomicAdd(hist + (c0 + c) * QH_BINS + b, n);
    }
    __syncthreads();
    pdl_trigger();
}

// One warp per column: find the bin of the column's histogram that holds
// rank krem (1-based, ascending), extend the prefix by it, lower krem by the
// count of the bins below, and zero the histogram row for the next digit.
// first: prefix 0 and krem = k for every column.  last: write the value
// whose magnitude bits are the completed prefix.
template <int DT>
__device__ __forceinline__ void quantile_select_column(uint32_t *__restrict__ hist, int64_t cols, int width,
                                                       uint32_t k, int first, int last, uint32_t *__restrict__ prefix,
                                                       uint32_t *__restrict__ krem, float *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int64_t j = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (j >= cols) return;
    uint32_t *h = hist + j * QH_BINS;
    const int nb = 1 << width;                        // 128 or 256 bins: 4 or 8 per lane
    const int per = nb / 32;
    uint32_t cnt[8];
    uint32_t tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        cnt[i] = i < per ? h[lane * per + i] : 0u;
        tot += cnt[i];
    }
    // inclusive prefix sum of the lanes' totals
    uint32_t inc = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    const uint32_t kr = first ? k : krem[j];
    const uint32_t below_lane = inc - tot;
    // the lane whose range holds rank kr: below_lane < kr <= inc
    const unsigned hit = __ballot_sync(0xffffffffu, below_lane < kr && kr <= inc);
    const int src = hit ? __ffs(hit) - 1 : 31;
    uint32_t bin = 0, below = 0;
    if (lane == src) {
        // the first bin b of this lane with below_lane + cnt[0..b] >= kr
        uint32_t c = below_lane;
        int b = per - 1;
        bool found = false;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (!found && i < per) {
                if (c + cnt[i] >= kr) {
                    b = i;
                    found = true;
                } else {
                    c += cnt[i];
                }
            }
        }
        bin = static_cast<uint32_t>(lane * per + b);
        below = c;
    }
    bin = __shfl_sync(0xffffffffu, bin, src);
    below = __shfl_sync(0xffffffffu, below, src);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i < per) h[lane * per + i] = 0u;
    if (lane == 0) {
        const uint32_t pf = ((first ? 0u : prefix[j]) << width) | bin;
        if (last) {
            if constexpr (DT == DT_F32) out[j] = __uint_as_float(pf);
            else if constexpr (DT == DT_F16) out[j] = __half2float(__ushort_as_half(static_cast<unsigned short>(pf)));
            else out[j] = __uint_as_float(pf << 16);
        } else {
            prefix[j] = pf;
            krem[j] = kr - below;
        }
    }
}

template <int DT>
__global__ void __launch_bounds__(256)
    k_quantile_select(uint32_t *__restrict__ hist, int64_t cols, int width, uint32_t k, int first, int last,
                      uint32_t *__restrict__ prefix, uint32_t *__restrict__ krem, float *__restrict__ out)
{
    pdl_wait();
    quantile_select_column<DT>(hist, cols, width, k, first, last, prefix, krem, out);
    __syncthreads();
    pdl_trigger();
}

}  // namespace sq
