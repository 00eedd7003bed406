// common.cuh -- shared device helpers of libsq (dtype widening, the canonical
// fp32 quantisation steps, block reductions, the device error word).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace sq {

enum DType : int { DT_F32 = 0, DT_F16 = 1, DT_BF16 = 2 };

__host__ __device__ constexpr int dtype_size(int dt) { return dt == DT_F32 ? 4 : 2; }

// First barrier-timeout code recorded by any kernel of this library on this
// device (0 = none).  Read and cleared by sq_sync_status.
__device__ unsigned int g_error_word;

// Programmatic dependent launch.  On created streams every kernel of this
// library is launched with programmatic stream serialisation and executes
// pdl_wait() before it reads any global input.  Each kernel triggers its
// dependents (pdl_trigger) only at its very end: every thread of a CTA, after
// a block-wide barrier that follows the CTA's last global write, so that the
// next kernel's launch and prologue overlap this kernel's teardown.  Measured
// on B200, global writes a kernel made AFTER its trigger were not visible to
// the dependent past its griddepcontrol.wait (a chain of small dependent
// kernels that triggered at their start read stale histograms and prefixes);
// with the trigger after the last write the chain was exact.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Canonical fp32 steps (round-to-nearest intrinsics so that nvcc never fuses
// a product into a multiply-add).  Symmetric INT8 quantisation, zero point 0:
// kwkr.cn blog 1.2 (x_q = round(x / s)) and 3.3; "010. SmoothQuant
// Integration" key design point 6 (symmetric only).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float recip_or_zero(float v) { return v > 0.0f ? __frcp_rn(v) : 0.0f; }

__device__ __forceinline__ float scale_from_absmax(float m) { return __fdiv_rn(m, 127.0f); }

// round half to even, saturate to [-127, 127]
__device__ __forceinline__ int quant8(float v)
{
    int r = __float2int_rn(v);
    return min(max(r, -127), 127);
}

// The same code as quant8, computed on the FMA/ALU pipes: clamp in fp32, then
// add 1.5 * 2^23 so that the fp32 add itself rounds half to even to an
// integer; the low byte of the sum's bit pattern is the two's-complement
// code.  Clamping first gives the same result as rounding first (both ends of
// [-127, 127] are integers), for every non-NaN v.
__device__ __forceinline__ uint32_t quant8_bits(float v)
{
    const float c = fminf(fmaxf(v, -127.0f), 127.0f);
    return __float_as_uint(__fadd_rn(c, 12582912.0f));
}

// quant8_bits for values already known to lie in [-127.5, 127.5): the
// per-row (weight) and per-token codes, whose row maximum maps to
// fl(m * fl(1 / fl(m / 127))) <= 127 * (1 + 3 * 2^-24) < 127.5, so the clamp
// of quant8_bits cannot bind there.
__device__ __forceinline__ uint32_t quant8_bits_inrange(float v) { return __float_as_uint(__fadd_rn(v, 12582912.0f)); }

// quant8_bits (INRANGE: quant8_bits_inrange) of a pair of values with one
// packed fp32 add (sm_100's f32x2 arithmetic rounds each lane like the
// scalar instruction).
template <bool INRANGE>
__device__ __forceinline__ void quant8_bits2(float a, float b, uint32_t &qa, uint32_t &qb)
{
    const float2 c = INRANGE ? make_float2(a, b)
                             : make_float2(fminf(fmaxf(a, -127.0f), 127.0f), fminf(fmaxf(b, -127.0f), 127.0f));
    const float2 t = __fadd2_rn(c, make_float2(12582912.0f, 12582912.0f));
    qa = __float_as_uint(t.x);
    qb = __float_as_uint(t.y);
}

// max(m, |a|, |b|) in one instruction (sm_100's three-input max).  max3_abs
// skips a NaN input like fmaxf; max3_abs_nan returns NaN when any input is
// NaN, so that a range check on its result fails for NaN.
__device__ __forceinline__ float max3_abs(float m, float a, float b)
{
    float r;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m), "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float max3_abs_nan(float m, float a, float b)
{
    float r;
    asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m), "f"(a), "f"(b));
    return r;
}

// low bytes of four quant8_bits results -> one packed word (byte 0 = a)
__device__ __forceinline__ uint32_t pack4_bits(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d)
{
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

// ---------------------------------------------------------------------------
// FP8 (E4M3) codes for the FP8 variant of the layer (aiunderstanding.org,
// "SmoothQuant 和激活量化": the smoothing carries over to FP8 tensor cores).
// E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, largest finite
// value 448.  The conversion rounds to nearest even and saturates magnitudes
// beyond the largest finite value to +-448 (satfinite); the scale of a row or
// tensor maps its absmax to 448.
// ---------------------------------------------------------------------------
constexpr float E4M3_MAX = 448.0f;

// codes of (lo, hi) as two bytes: lo in bits 0..7, hi in bits 8..15
__device__ __forceinline__ uint32_t e4m3x2_bits(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// four codes packed into one word (byte 0 = a)
__device__ __forceinline__ uint32_t e4m3x4_bits(float a, float b, float c, float d)
{
    return e4m3x2_bits(a, b) | (e4m3x2_bits(c, d) << 16);
}

// the absmax scale of the code format: fl(m / 127) for INT8, fl(m / 448) for E4M3
template <bool F8>
__device__ __forceinline__ float scale_from_absmax_q(float m)
{
    return F8 ? __fdiv_rn(m, E4M3_MAX) : __fdiv_rn(m, 127.0f);
}

// ---------------------------------------------------------------------------
// 16-byte vectors: EPV elements of dtype DT, widened exactly to fp32.
// ---------------------------------------------------------------------------
template <int DT> struct VecT { static constexpr int EPV = 16 / dtype_size(DT); };

template <int DT>
__device__ __forceinline__ void widen(const uint4 &v, float (&f)[VecT<DT>::EPV])
{
    if constexpr (DT == DT_F32) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    } else {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (DT == DT_F16) {
                __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
                float2 t = __half22float2(h);
                f[2 * i] = t.x; f[2 * i + 1] = t.y;
            } else {
                f[2 * i] = __uint_as_float(w[i] << 16);
                f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
        }
    }
}

template <int DT> __device__ __forceinline__ float load_elem(const void *p, int64_t i)
{
    if constexpr (DT == DT_F32) return static_cast<const float *>(p)[i];
    else if constexpr (DT == DT_F16) return __half2float(static_cast<const __half *>(p)[i]);
    else return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ float load_elem_dt(const void *p, int dt, int64_t i)
{
    if (dt == DT_F32) return load_elem<DT_F32>(p, i);
    if (dt == DT_F16) return load_elem<DT_F16>(p, i);
    return load_elem<DT_BF16>(p, i);
}

// ---------------------------------------------------------------------------
// Block reductions (blockDim.x a multiple of 32, <= 1024).  `red` holds 32 floats.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float block_max(float v, float *red)
{
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();                       // protect `red` from the previous use
    if (l == 0) red[w] = v;
    __syncthreads();
    float r = (l < nw) ? red[l] : 0.0f;
    return warp_max(r);
}

__device__ __forceinline__ double block_sum_f64(double v, double *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = (l < nw) ? red[l] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    return r;
}

// block_sum_f64 for a compile-time warp count NW (a power of two): the
// second level reduces only the NW warp sums, giving the same sum as
// block_sum_f64 (whose lanes past NW add zeros).
template <int NW>
__device__ __forceinline__ double block_sum_f64_nw(double v, double *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = red[l & (NW - 1)];
#pragma unroll
    for (int o = NW / 2; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    return r;
}

}  // namespace sq
