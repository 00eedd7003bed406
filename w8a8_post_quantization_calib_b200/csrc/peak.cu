// peak.cu -- measurement library (libsq_peak.so): the dense INT8 and FP8
// tensor-core rate of one B200, the denominator of the GEMMs' roofline.
//
// The kernel is the W8A8 GEMM's mainloop without its operand traffic: a
// cluster of two CTAs (one per SM) issues tcgen05.mma.cta_group::2 of shape
// M = 256, N = 256, K = 32 bytes (kind::i8, s8 x s8 -> s32, or kind::f8f6f4,
// E4M3 x E4M3 -> f32) back to back on operands that stay in shared memory,
// accumulating into one TMEM accumulator.  One launch runs `iters` groups of
// four MMAs (one 128-byte K block) on every cluster; the host times launches
// with CUDA events, so the rate is 2 * 256 * 256 * 128 * iters * clusters /
// time.  Nothing is read from or written to global memory besides the error
// word of the bounded wait.
//
// The second measurement is the read rate of one launch that streams a
// buffer once: the ceiling of a decode-size GEMM, which reads its weights
// once per launch.  Each block of 512 threads streams a contiguous share with
// 16-byte evict-first loads, four in flight per thread; the loaded words are
// folded into a value that is written only if it equals an impossible
// constant, so the loads cannot be dropped.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace {

constexpr int SR_THREADS = 512;

__global__ void __launch_bounds__(SR_THREADS) k_stream_read(const uint4 *__restrict__ buf, long long n16,
                                                            unsigned int *sink)
{
    const long long per = (n16 + gridDim.x - 1) / gridDim.x;
    const long long a = static_cast<long long>(blockIdx.x) * per;
    const long long b = a + per < n16 ? a + per : n16;
    uint32_t acc = 0;
    long long i = a + threadIdx.x;
    for (; i + 3 * SR_THREADS < b; i += 4 * SR_THREADS) {
        const uint4 t0 = __ldcs(buf + i), t1 = __ldcs(buf + i + SR_THREADS);
        const uint4 t2 = __ldcs(buf + i + 2 * SR_THREADS), t3 = __ldcs(buf + i + 3 * SR_THREADS);
        acc ^= (t0.x ^ t0.y ^ t0.z ^ t0.w) + (t1.x ^ t1.y ^ t1.z ^ t1.w) + (t2.x ^ t2.y ^ t2.z ^ t2.w) +
               (t3.x ^ t3.y ^ t3.z ^ t3.w);
    }
    for (; i < b; i += SR_THREADS) {
        const uint4 t = __ldcs(buf + i);
        acc ^= t.x ^ t.y ^ t.z ^ t.w;
    }
    if (acc == 0x9e3779b9u && sink != nullptr) *sink = acc;
}

constexpr int PK_THREADS = 128;
constexpr int PK_TILE = 128 * 128;           // one 128-row x 128-byte operand tile per CTA
constexpr int PK_SMEM = 1024 + 2 * PK_TILE + 64;

template <int KIND>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PK_THREADS, 1) k_mma_peak(int iters, unsigned long long timeout_ns)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *done = reinterpret_cast<uint64_t *>(smem + 2 * PK_TILE);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5;
    const uint32_t rank = sq::ptx::cluster_ctarank();

    // operands: a fixed pseudo-random byte pattern (finite E4M3 values for kind::f8f6f4)
    for (int i = threadIdx.x; i < 2 * PK_TILE / 4; i += PK_THREADS) {
        uint32_t v = (static_cast<uint32_t>(i) * 2654435761u) ^ (rank * 0x9e3779b9u);
        if (KIND == 2) v &= 0x3e3e3e3eu;       // exponent below the NaN pattern
        reinterpret_cast<uint32_t *>(smem)[i] = v;
    }
    if (threadIdx.x == 0) {
        sq::ptx::mbar_init(sq::ptx::smem_addr(done), 1);
        *abort_flag = 0;
        sq::ptx::fence_barrier_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // operand bytes visible to the tensor core
    if (warp == 0) {
        sq::ptx::tmem_alloc_pair(sq::ptx::smem_addr(tmem_slot), 256);
        sq::ptx::tmem_relinquish_pair();
    }
    sq::ptx::tc_fence_before();
    sq::ptx::cluster_sync();
    sq::ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (rank == 0 && threadIdx.x == 0) {
        const uint32_t sa = sq::ptx::smem_addr(smem);
        const uint64_t ad = sq::ptx::sdesc_kmajor_sw128(sa);
        const uint64_t bd = sq::ptx::sdesc_kmajor_sw128(sa + PK_TILE);
        constexpr uint32_t IDESC = KIND == 2 ? sq::ptx::idesc_e4m3_m256(256) : sq::ptx::idesc_i8_m256(256);
#pragma unroll 1
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if constexpr (KIND == 2) sq::ptx::mma_f8_pair(tmem, ad + 2 * k, bd + 2 * k, IDESC, (it | k) ? 1u : 0u);
                else sq::ptx::mma_i8_pair(tmem, ad + 2 * k, bd + 2 * k, IDESC, (it | k) ? 1u : 0u);
            }
        }
        sq::ptx::tc_commit_pair_mc(sq::ptx::smem_addr(done), 0x3);
    }
    if (threadIdx.x == 0) sq::ptx::wait_bounded(sq::ptx::smem_addr(done), 0u, timeout_ns, abort_flag, 0x160);
    __syncthreads();
    sq::ptx::tc_fence_before();
    sq::ptx::cluster_sync();
    if (warp == 0) {
        sq::ptx::tc_fence_after();
        sq::ptx::tmem_dealloc_pair(tmem, 256);
    }
}

}  // namespace

extern "C" {

// Largest number of co-resident two-CTA clusters of the peak kernel (one per
// SM pair), or -1 on a CUDA error.
int sqpeak_clusters(int kind)
{
    const void *k = kind == 2 ? reinterpret_cast<const void *>(k_mma_peak<2>) : reinterpret_cast<const void *>(k_mma_peak<0>);
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PK_SMEM) != cudaSuccess) return -1;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2));
    cfg.blockDim = dim3(PK_THREADS);
    cfg.dynamicSmemBytes = PK_SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess) return -1;
    return n;
}

// One launch of `clusters` clusters x `iters` K blocks on `stream`.  kind: 0 =
// INT8 (kind::i8), 2 = FP8 E4M3 (kind::f8f6f4).  Returns 0 or a cudaError_t.
// MACs per launch: 256 * 256 * 128 * iters * clusters.
int sqpeak_launch(int kind, int clusters, int iters, void *stream)
{
    // at most 2^20 K blocks per launch: 0.3 s at the nominal 4.5 POPS, so a
    // launch ends far inside the kernel's bounded wait (10 s) at any rate
    // above ~130 TOPS
    if (clusters <= 0 || iters <= 0 || iters > (1 << 20)) return static_cast<int>(cudaErrorInvalidValue);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(PK_THREADS);
    cfg.dynamicSmemBytes = PK_SMEM;
    cfg.stream = static_cast<cudaStream_t>(stream);
    const unsigned long long tmo = 10000000000ull;
    cudaError_t e = kind == 2 ? cudaLaunchKernelEx(&cfg, k_mma_peak<2>, iters, tmo)
                              : cudaLaunchKernelEx(&cfg, k_mma_peak<0>, iters, tmo);
    if (e == cudaSuccess) e = cudaGetLastError();
    return static_cast<int>(e);
}

// One launch of the streaming read over `bytes` bytes at `buf` (16-byte
// aligned, bytes a multiple of 16) with `blocks` blocks of 512 threads on
// `stream`; `sink` is a device word the kernel may write (never in practice).
// Returns 0 or a cudaError_t.
int sqpeak_stream_read(const void *buf, size_t bytes, int blocks, unsigned int *sink, void *stream)
{
    if (buf == nullptr || blocks <= 0 || (bytes % 16) != 0 || (reinterpret_cast<uintptr_t>(buf) % 16) != 0)
        return static_cast<int>(cudaErrorInvalidValue);
    k_stream_read<<<blocks, SR_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(buf), static_cast<long long>(bytes / 16), sink);
    return static_cast<int>(cudaGetLastError());
}

// First barrier-timeout code recorded by the peak kernel (0 = none), cleared.
int sqpeak_error_word(void)
{
    unsigned int w = 0, z = 0;
    if (cudaMemcpyFromSymbol(&w, sq::g_error_word, sizeof(w)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(sq::g_error_word, &z, sizeof(z));
    return static_cast<int>(w);
}

}  // extern "C"
