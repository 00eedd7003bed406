// calib.cuh -- per-column absolute maximum of a row-major [rows, cols] tensor,
// accumulated into a running fp32 maximum (the SmoothQuant calibration
// statistic max|X_j| of kwkr.cn blog 3.1; "010. SmoothQuant Integration" key
// design point 1: the running per-channel max-abs is the only state kept).
//
// HBM-bound: one streaming read of the tensor.  Each warp reads 512
// contiguous bytes of a row per step (16 B per lane), a block covers a strip
// of 32 vectors x 8 row lanes and walks a slab of rows with four independent
// 16-byte loads in flight per thread.  Partial maxima are combined in
// registers (packed half2/bfloat162 max for 16-bit data, exact), then across
// the block's row lanes in shared memory, then across blocks with atomicMax
// on the float bit pattern (non-negative floats order like their bits).
#pragma once

#include "common.cuh"

namespace sq {

constexpr int CALIB_TX = 32;      // vectors per block strip
constexpr int CALIB_TY = 8;       // row lanes per block
constexpr int CALIB_UNROLL = 4;   // rows in flight per thread

template <bool STREAM>
__device__ __forceinline__ uint4 load16(const uint8_t *p)
{
    if constexpr (STREAM) return __ldcs(reinterpret_cast<const uint4 *>(p));
    else return __ldg(reinterpret_cast<const uint4 *>(p));
}

template <int DT>
struct AbsMaxAcc {
    static constexpr int EPV = VecT<DT>::EPV;
    uint32_t m[4];   // packed running maxima of |x| (16-bit: 2 per word; fp32: 1 per word)

    __device__ __forceinline__ void init() { m[0] = m[1] = m[2] = m[3] = 0u; }

    __device__ __forceinline__ void add(const uint4 &v)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (DT == DT_F32) {
                m[i] = max(m[i], w[i] & 0x7fffffffu);   // |x| bits; order of non-negative floats
            } else if constexpr (DT == DT_F16) {
                __half2 a = __habs2(*reinterpret_cast<const __half2 *>(&w[i]));
                __half2 b = __hmax2(*reinterpret_cast<__half2 *>(&m[i]), a);
                m[i] = *reinterpret_cast<uint32_t *>(&b);
            } else {
                __nv_bfloat162 a = __habs2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
                __nv_bfloat162 b = __hmax2(*reinterpret_cast<__nv_bfloat162 *>(&m[i]), a);
                m[i] = *reinterpret_cast<uint32_t *>(&b);
            }
        }
    }

    __device__ __forceinline__ void to_float(float (&f)[EPV]) const
    {
        if constexpr (DT == DT_F32) {
#pragma unroll
            for (int i = 0; i < 4; ++i) f[i] = __uint_as_float(m[i]);
        } else {
            uint4 v = make_uint4(m[0], m[1], m[2], m[3]);
            widen<DT>(v, f);
        }
    }
};

// STREAM: evict-first loads for tensors much larger than L2 (calibration
// batches); otherwise normal loads, so that a tensor read again right after
// (the weight: statistic, then transform) can still be found in L2.
template <int DT, bool STREAM>
__global__ void __launch_bounds__(CALIB_TX *CALIB_TY)
    k_colabsmax(const uint8_t *__restrict__ x, int64_t rows, int64_t nvec, int64_t ld_bytes,
                int64_t row_slab, float *__restrict__ absmax)
{
    constexpr int EPV = VecT<DT>::EPV;
    __shared__ float red[CALIB_TY][CALIB_TX * EPV];

    const int tx = threadIdx.x, ty = threadIdx.y;
    const int64_t v = static_cast<int64_t>(blockIdx.x) * CALIB_TX + tx;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * row_slab;
    const int64_t r1 = min(rows, r0 + row_slab);

    AbsMaxAcc<DT> acc;
    acc.init();
    pdl_wait();
    if (v < nvec) {
        const uint8_t *col = x + v * 16;
        int64_t r = r0 + ty;
        for (; r + (CALIB_UNROLL - 1) * CALIB_TY < r1; r += CALIB_UNROLL * CALIB_TY) {
            uint4 t[CALIB_UNROLL];
#pragma unroll
            for (int u = 0; u < CALIB_UNROLL; ++u)
                t[u] = load16<STREAM>(col + (r + u * CALIB_TY) * ld_bytes);
#pragma unroll
            for (int u = 0; u < CALIB_UNROLL; ++u) acc.add(t[u]);
        }
        for (; r < r1; r += CALIB_TY) acc.add(load16<STREAM>(col + r * ld_bytes));
    }
    float f[EPV];
    acc.to_float(f);
#pragma unroll
    for (int e = 0; e < EPV; ++e) red[ty][tx * EPV + e] = f[e];
    __syncthreads();

    // combine the row lanes; one atomic per column per block
    for (int c = ty * CALIB_TX + tx; c < CALIB_TX * EPV; c += CALIB_TX * CALIB_TY) {
        const int64_t col = static_cast<int64_t>(blockIdx.x) * CALIB_TX * EPV + c;
        if (col < nvec * EPV) {
            float m = red[0][c];
#pragma unroll
            for (int i = 1; i < CALIB_TY; ++i) m = fmaxf(m, red[i][c]);
            atomicMax(reinterpret_cast<int *>(absmax + col), __float_as_int(m));
        }
    }
    __syncthreads();
    pdl_trigger();
}

// Fallback for tensors whose rows are not 16-byte aligned: one thread per
// column, a slab of rows per block row.
__global__ void k_colabsmax_scalar(const void *__restrict__ x, int dt, int64_t rows, int64_t cols,
                                   int64_t ld, int64_t row_slab, float *__restrict__ absmax)
{
    pdl_wait();
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j < cols) {
        const int64_t r0 = static_cast<int64_t>(blockIdx.y) * row_slab;
        const int64_t r1 = min(rows, r0 + row_slab);
        float m = 0.0f;
        for (int64_t r = r0; r < r1; ++r) m = fmaxf(m, fabsf(load_elem_dt(x, dt, r * ld + j)));
        atomicMax(reinterpret_cast<int *>(absmax + j), __float_as_int(m));
    }
    __syncthreads();
    pdl_trigger();
}

}  // namespace sq
