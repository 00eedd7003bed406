// libsq.cu -- the C ABI of the SmoothQuant W8A8 linear layer for B200
// (sm_100a).  One translation unit: the kernels live in the included .cuh
// files; this file validates arguments, sizes grids for the device, encodes
// TMA tensor maps and launches.  Declarations and the full contract of every
// entry point are in include/sq.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <utility>

#include "sq.h"
#include "common.cuh"
#include "ptx_sm100.cuh"
#include "calib.cuh"
#include "robust.cuh"
#include "quant.cuh"
#include "gemm.cuh"

using namespace sq;

namespace {

thread_local int t_last_cuda_error = 0;
unsigned long long g_timeout_ns = 2000000000ull;   // bounded barrier waits: 2 s
int g_inject = 0;                                  // failure-detection test knob

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
std::mutex g_mu;

inline cudaStream_t as_stream(sq_stream s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool valid_dt(int dt) { return dt == SQ_F32 || dt == SQ_F16 || dt == SQ_BF16; }

inline sq_status cuda_fail(cudaError_t e)
{
    t_last_cuda_error = static_cast<int>(e);
    return SQ_ERR_CUDA;
}

inline sq_status check_launch()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SQ_OK : cuda_fail(e);
}

int sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (g_sm_count[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_sm_count[dev] = n > 0 ? n : 148;
    }
    return g_sm_count[dev];
}

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Programmatic dependent launch is used only on explicitly created streams;
// on the legacy and per-thread default streams launches go without the
// attribute (plain stream order), which is where the chains that first showed
// the early-trigger hazard (see pdl_wait in common.cuh) ran.
inline bool pdl_stream(cudaStream_t st)
{
    return st != nullptr && st != cudaStreamLegacy && st != cudaStreamPerThread;
}

// Launch with programmatic stream serialisation (see pdl_wait in common.cuh):
// the kernel may begin while the previous kernel of the stream drains.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_stream(st) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// launch_pdl with a runtime cluster shape (cluster_x CTAs along x) and
// dynamic shared memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster_smem(void (*kern)(KArgs...), dim3 grid, dim3 block, unsigned cluster_x, size_t smem,
                                    cudaStream_t st, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_stream(st) ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// launch_pdl with a runtime cluster shape (cluster_x CTAs along x).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, unsigned cluster_x, cudaStream_t st,
                               Args &&...args)
{
    return launch_pdl_cluster_smem(kern, grid, block, cluster_x, 0, st, std::forward<Args>(args)...);
}

// Per (device, kernel): dynamic shared memory already granted, and the
// occupancy figures the launch sizes its grid with.  Queried once.
struct KernelInfo {
    int smem_set = 0;
    int per_sm = 0;           // resident blocks per SM with per_sm_smem bytes of dynamic shared memory
    int per_sm_smem = -1;
    int clusters = 0;
};
std::unordered_map<uint64_t, KernelInfo> g_kinfo;

KernelInfo &kinfo(const void *kern)
{
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t key = (static_cast<uint64_t>(dev) << 56) ^ reinterpret_cast<uint64_t>(kern);
    return g_kinfo[key];
}

// Grants `smem` bytes of dynamic shared memory to `kern` (once per size increase).
cudaError_t ensure_smem(const void *kern, int smem)
{
    std::lock_guard<std::mutex> lk(g_mu);
    KernelInfo &ki = kinfo(kern);
    if (ki.smem_set >= smem) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) ki.smem_set = smem;
    return e;
}

// ------------------------------------------------------------------ TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2D row-major [rows, inner] tensor of 1- or 2-byte elements; box of
// box_rows x 128 bytes with the 128-byte swizzle; out-of-range reads are zero.
bool make_map(CUtensorMap *m, const void *base, bool f16, int64_t inner, int64_t rows, uint32_t box_rows)
{
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const int elt = f16 ? 2 : 1;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner * elt)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elt), box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                          const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3D view of a row-major [rows, K] int8 tensor (K a multiple of 128) as
// [K/128][rows][128 bytes]: box = box_rows x 128 bytes x kbo blocks, each
// block landing as its own 128-byte-swizzled tile.
bool make_map3(CUtensorMap *m, const void *base, int64_t K, int64_t rows, uint32_t box_rows, uint32_t kbo)
{
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 128)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), 128};
    cuuint32_t box[3] = {128, box_rows, kbo};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM launch
// Small-M (swap) launch: map_w over the weights [N, K] in 128-row boxes, map_x
// over the activations [M, K] in BN-row boxes; one CTA per stream-K share.
template <int BN, int EPI, int KBO, int CS, int KIND = gemm::KIND_I8>
sq_status launch_swap(gemm::Params p, const void *w, const void *x, cudaStream_t st)
{
    using C = gemm::TileCfg<BN, KBO>;
    CUtensorMap mw, mx;
    if constexpr (KBO == 1) {
        if (!make_map(&mw, w, false, p.K, p.N, gemm::BM)) return SQ_ERR_CUDA;
        if (!make_map(&mx, x, false, p.K, p.M, BN)) return SQ_ERR_CUDA;
    } else {
        if (!make_map3(&mw, w, p.K, p.N, gemm::BM, KBO)) return SQ_ERR_CUDA;
        if (!make_map3(&mx, x, p.K, p.M, BN, KBO)) return SQ_ERR_CUDA;
    }
    auto kern = gemm::k_gemm_swap<BN, EPI, KBO, CS, KIND>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    p.timeout_ns = g_timeout_ns;
    p.inject = g_inject & 1;
    if constexpr (CS > 1)
        e = launch_pdl_cluster_smem(kern, dim3(p.sk_ctas), dim3(gemm::NUM_THREADS), CS, C::SMEM_BYTES, st, mw, mx, p);
    else
        e = launch_pdl(kern, dim3(p.sk_ctas), dim3(gemm::NUM_THREADS), C::SMEM_BYTES, st, mw, mx, p);
    return e == cudaSuccess ? check_launch() : cuda_fail(e);
}

template <int EPI, int KBO, int CS, int KIND>
sq_status launch_swap_bn(gemm::Params &p, int bn, const void *wq, const void *xq, cudaStream_t st)
{
    switch (bn) {
    case 16: return launch_swap<16, EPI, KBO, CS, KIND>(p, wq, xq, st);
    case 32: return launch_swap<32, EPI, KBO, CS, KIND>(p, wq, xq, st);
    case 64: return launch_swap<64, EPI, KBO, CS, KIND>(p, wq, xq, st);
    default: return launch_swap<128, EPI, KBO, CS, KIND>(p, wq, xq, st);
    }
}

// CTA-pair launch: grid = 2 x (co-resident clusters, at most one per unit).
// Output map for the epilogue's TMA stores: [M, N] row-major, 32 x 32 boxes,
// swizzle matching the staging layout (64-byte rows for 2-byte elements,
// 128-byte rows for 4-byte ones).
bool make_out_map(CUtensorMap *m, void *base, int out_dt, bool s32, int64_t M, int64_t N)
{
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    CUtensorMapDataType t;
    int elt;
    if (s32) { t = CU_TENSOR_MAP_DATA_TYPE_INT32; elt = 4; }
    else if (out_dt == SQ_F32) { t = CU_TENSOR_MAP_DATA_TYPE_FLOAT32; elt = 4; }
    else if (out_dt == SQ_F16) { t = CU_TENSOR_MAP_DATA_TYPE_FLOAT16; elt = 2; }
    else { t = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; elt = 2; }
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N * elt)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, t, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          elt == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN, int KIND, int EPI, int KBO>
sq_status launch_gemm2(gemm::Params p, const void *a, const void *b, cudaStream_t st)
{
    using C = gemm::PairCfg<BN, KBO>;
    const bool f16 = (KIND == gemm::KIND_F16);
    CUtensorMap ma, mb, mo;
    if constexpr (KBO == 1) {
        if (!make_map(&ma, a, f16, p.K, p.rows_a, gemm::BM)) return SQ_ERR_CUDA;
        if (!make_map(&mb, b, f16, p.K, p.rows_b, BN / 2)) return SQ_ERR_CUDA;
    } else {
        static_assert(KIND != gemm::KIND_F16, "3D operand maps are of 1-byte elements");
        if (!make_map3(&ma, a, p.K, p.rows_a, gemm::BM, KBO)) return SQ_ERR_CUDA;
        if (!make_map3(&mb, b, p.K, p.rows_b, BN / 2, KBO)) return SQ_ERR_CUDA;
    }
    if constexpr (EPI == gemm::EPI_DEQUANT_T) {
        std::memset(&mo, 0, sizeof(mo));            // direct stores (see epilogue_t)
    } else if constexpr (EPI == gemm::EPI_GATEUP) {
        // h [M, N/2] bf16, written with TMA stores when requested
        std::memset(&mo, 0, sizeof(mo));
        if (p.out != nullptr && !make_out_map(&mo, p.out, SQ_BF16, false, p.M, p.N / 2)) return SQ_ERR_CUDA;
    } else {
        const int odt = (EPI == gemm::EPI_F16) ? SQ_F16 : p.out_dt;
        if (!make_out_map(&mo, p.out, odt, EPI == gemm::EPI_S32, p.M, p.N)) return SQ_ERR_CUDA;
    }
    auto kern = gemm::k_gemm2<BN, KIND, EPI, KBO>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    int max_clusters = 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        max_clusters = kinfo(reinterpret_cast<const void *>(kern)).clusters;
    }
    if (max_clusters == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
        cfg.blockDim = dim3(gemm::NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void *>(kern), &cfg) != cudaSuccess || n <= 0)
            n = sm_count() / 2;
        cudaGetLastError();
        max_clusters = n;
        std::lock_guard<std::mutex> lk(g_mu);
        kinfo(reinterpret_cast<const void *>(kern)).clusters = n;
    }
    p.timeout_ns = g_timeout_ns;
    p.inject = g_inject & 1;
    const int clusters = static_cast<int>(std::min<int64_t>(p.num_units, max_clusters));
    e = launch_pdl(kern, dim3(2 * clusters), dim3(gemm::NUM_THREADS), C::SMEM_BYTES, st, ma, mb, mo, p);
    return e == cudaSuccess ? check_launch() : cuda_fail(e);
}

void fill_tiles_pair(gemm::Params &p, int bn, int kb_bytes_per_elem)
{
    p.rows_a = p.M;
    p.rows_b = p.N;
    p.num_kb = static_cast<int>(cdiv(static_cast<int64_t>(p.K) * kb_bytes_per_elem, 128));
    p.tiles_r = static_cast<int>(cdiv(p.M, 2 * gemm::BM));
    p.tiles_c = static_cast<int>(cdiv(p.N, bn));
    p.num_units = p.tiles_r * p.tiles_c;
}

// Pair-tile width with the fewest waves x tile width (ties to the wider tile).
int pick_pair_bn(int64_t M, int64_t N)
{
    const int64_t clusters = std::max(1, sm_count() / 2);
    const int cands[4] = {256, 224, 192, 128};
    // measured time per output column of a full wave relative to the 256-wide
    // tile (narrower tiles move more operand bytes per MAC), all with two K
    // blocks per load, on the Llama-7B QKV and MLP shapes; the 128-wide
    // figure predates the two-block loads
    const double eff[4] = {1.0, 0.92, 0.85, 0.77};
    int best = 256;
    double best_cost = -1.0;
    for (int i = 0; i < 4; ++i) {
        const int bn = cands[i];
        const int64_t tiles = cdiv(M, 2 * gemm::BM) * cdiv(N, bn);
        const double cost = static_cast<double>(cdiv(tiles, clusters) * bn) / eff[i];
        if (best_cost < 0 || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

template <int KIND, int EPI>
sq_status dispatch_pair(gemm::Params &p, const void *a, const void *b, cudaStream_t st, int force_bn = 0)
{
    const int bn = force_bn ? force_bn : pick_pair_bn(p.M, p.N);
    fill_tiles_pair(p, bn, KIND == gemm::KIND_F16 ? 2 : 1);
    if constexpr (KIND != gemm::KIND_F16) {
        // two K blocks per TMA load: 3 stages of 56 KB (192-wide) hold the
        // same 6 blocks as 6 single-block stages with half the loads; the
        // 256-wide tile fits 3 stages of 64 KB with one epilogue staging
        // buffer per warp
        if (bn >= 192 && (p.K % 128) == 0) {
            p.num_kb = static_cast<int>(cdiv(p.num_kb, 2));
            if (bn == 256) return launch_gemm2<256, KIND, EPI, 2>(p, a, b, st);
            if (bn == 224) return launch_gemm2<224, KIND, EPI, 2>(p, a, b, st);
            return launch_gemm2<192, KIND, EPI, 2>(p, a, b, st);
        }
    }
    switch (bn) {
    case 256: return launch_gemm2<256, KIND, EPI, 1>(p, a, b, st);
    case 224: return launch_gemm2<224, KIND, EPI, 1>(p, a, b, st);
    case 192: return launch_gemm2<192, KIND, EPI, 1>(p, a, b, st);
    default: return launch_gemm2<128, KIND, EPI, 1>(p, a, b, st);
    }
}

// Small M (64 < M <= 128) with many weight rows: the CTA-pair kernel with the
// weights as its A operand (256 rows per pair, 128 per CTA) and the tokens as
// B (BN = 128, half per CTA).  The pair's MMA reads the token tile from both
// CTAs, so each CTA loads only half of it: with one weight tile per CTA, a
// CTA of the weight-streaming kernel loads its 128 weight rows and the whole
// token tile (the MLP-7B up projection at M = 128: 512 KB + 512 KB per CTA),
// a pair CTA its 128 weight rows and half the tokens (768 KB).  Measured on
// that projection: 22.7 -> 22.05 us at M = 128, 21.4 -> 20.9 at M = 100; at
// M = 33 and 64 (BN = 64) it was no faster (14.9 -> 15.1, 16.7 -> 16.75 us),
// so it serves only M > 64.  Its gain is small because a launch that streams
// the 45 MB of weights once is itself bounded near 10 us.
template <int KIND>
sq_status dispatch_pair_t(gemm::Params &p, const void *xq, const void *wq, cudaStream_t st)
{
    constexpr int bn = 128;
    p.rows_a = p.N;
    p.rows_b = p.M;
    p.num_kb = static_cast<int>(cdiv(p.K, 128));
    p.tiles_r = static_cast<int>(cdiv(p.N, 2 * gemm::BM));
    p.tiles_c = static_cast<int>(cdiv(p.M, bn));
    p.num_units = p.tiles_r * p.tiles_c;
    if ((p.K % 128) == 0) {
        p.num_kb = static_cast<int>(cdiv(p.num_kb, 2));
        return launch_gemm2<bn, KIND, gemm::EPI_DEQUANT_T, 2>(p, wq, xq, st);
    }
    return launch_gemm2<bn, KIND, gemm::EPI_DEQUANT_T, 1>(p, wq, xq, st);
}

void fill_tiles(gemm::Params &p, int bn, int64_t rows_a, int64_t rows_b)
{
    p.rows_a = static_cast<int>(rows_a);
    p.rows_b = static_cast<int>(rows_b);
    p.num_kb = static_cast<int>(cdiv(p.K, 128 / 1));
    p.tiles_r = static_cast<int>(cdiv(rows_a, gemm::BM));
    p.tiles_c = static_cast<int>(cdiv(rows_b, bn));
    p.num_units = p.tiles_r * p.tiles_c;
}

constexpr int64_t kSwapMaxM = 128;

int swap_bn(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

int64_t swap_tiles(int64_t M, int64_t N) { return cdiv(N, gemm::BM) * cdiv(M, swap_bn(M)); }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Stream-K CTA count of the small-M path.  Decode-size GEMMs are a stream of
// the weight matrix, and one SM takes in only about 55 GB/s (measured with
// TMA loads of two 16 KB blocks), so the weight bytes must be spread over
// the SMs to reach the HBM rate: the 32 tiles of an 11008 -> 4096 projection
// on 32 SMs cap near 2 TB/s.  The (tile, K block) iterations are then shared
// evenly by min(SMs, iterations) CTAs.  Combining a shared tile costs a
// partial-sum round trip (publish, arrival count, slot loads) of about 3 us
// at the end of the owner's share, growing with the token tile, so sharing is
// used only when one tile per CTA would leave more than half of the SMs idle
// and the token tile is at most 32 (measured on the MLP-7B shapes: the
// 32-tile projection gains from sharing at M = 1, 16 and loses at M = 64,
// 128; the 86-tile one streams faster unshared at every M).  Otherwise, and
// when the slots do not fit `slot_cap` bytes with at least min(tiles, SMs)
// CTAs, the plain one-tile-per-CTA schedule runs: G = tiles.
int64_t swap_grid(int64_t M, int64_t N, int64_t K, size_t slot_cap)
{
    const int64_t tiles = swap_tiles(M, N);
    const int64_t iters = tiles * ((K % 128) == 0 ? cdiv(K / 128, 2) : cdiv(K, 128));
    const int64_t sms = sm_count();
    if (tiles % sms == 0 || 2 * tiles > sms || swap_bn(M) > 32) return tiles;
    int64_t g = std::min(sms, iters);
    const size_t slot = static_cast<size_t>(gemm::BM) * swap_bn(M) * 4;
    g = std::min<int64_t>(g, static_cast<int64_t>(slot_cap / slot));
    if (g < std::min(tiles, sms)) return tiles;
    return g;
}

// Workspace of a stream-K launch with G CTAs: G partial-sum slots of
// BM x BN int32 (one per CTA), then one int32 arrival counter per tile.
size_t swap_slot_bytes(int64_t M, int64_t G)
{
    return align_up(static_cast<size_t>(G) * gemm::BM * swap_bn(M) * 4, 256);
}

int swap_cluster_split(int64_t M, int64_t N, int64_t K);

size_t ws_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M > kSwapMaxM || swap_cluster_split(M, N, K) > 1) return 0;
    const int64_t g = swap_grid(M, N, K, SIZE_MAX);
    if (g == swap_tiles(M, N)) return 0;
    return swap_slot_bytes(M, g) + align_up(static_cast<size_t>(swap_tiles(M, N)) * 4, 256);
}

// CTAs per cluster of the cluster split (1 = none): when one tile per CTA
// would leave more than half of the SMs idle, CS = 2 or 4 CTAs of a cluster
// share each tile's K range and combine their partial sums through
// distributed shared memory (needs at least CS iterations per tile).
// Measured on the MLP-7B 32-tile projection against the stream-K schedule
// (whose combine goes through global memory): 14.1 -> 12.2 us at M = 1,
// 15.1 -> 13.4 at M = 16, 25.3 -> 19.2 at M = 64, 34.3 -> 28.0 at M = 128.
// sq_debug_inject(2) turns it off (tests of the other schedules).
int swap_cluster_split(int64_t M, int64_t N, int64_t K)
{
    if (g_inject & 2) return 1;
    const int64_t tiles = swap_tiles(M, N);
    const int64_t iters = (K % 128) == 0 ? cdiv(K / 128, 2) : cdiv(K, 128);
    const int64_t sms = sm_count();
    if (2 * tiles > sms) return 1;
    const int64_t c = std::min<int64_t>(sms / tiles, iters);
    return c >= 4 ? 4 : c >= 2 ? 2 : 1;
}

// The swapped CTA-pair kernel (dispatch_pair_t) serves 64 < M <= 128 where the
// weight-streaming kernel would run one 128-row weight tile per CTA (no
// cluster split) and the pair tiles fill at least half of the clusters.
// Measured on the MLP-7B up projection (86 tiles): see dispatch_pair_t.  The
// cluster split off (sq_debug_inject(2)) keeps the weight-streaming schedules.
bool use_pair_t(int64_t M, int64_t N, int64_t K)
{
    if (M <= 64 || M > kSwapMaxM || (g_inject & 2)) return false;
    if (swap_cluster_split(M, N, K) > 1) return false;
    return 2 * cdiv(N, 2 * gemm::BM) >= sm_count() / 2;
}

// p.ws_acc / p.ws_cnt must hold a workspace for `grid` CTAs unless grid is
// the tile count (then they are ignored).  cs > 1: cluster split, grid =
// tiles x cs, no workspace.
template <int EPI, int KIND = gemm::KIND_I8>
sq_status dispatch_swap(gemm::Params &p, const void *xq, const void *wq, cudaStream_t st, int64_t grid,
                        int cs = 1)
{
    const int bn = swap_bn(p.M);
    fill_tiles(p, bn, p.N, p.M);
    const bool kb2 = (p.K % 128) == 0;             // two K blocks per load (3D maps)
    if (kb2) p.num_kb = static_cast<int>(cdiv(p.num_kb, 2));   // iterations: groups of 2 blocks
    const int64_t tiles = static_cast<int64_t>(p.tiles_r) * p.tiles_c;
    const int64_t iters = tiles * p.num_kb;
    if (iters >= (int64_t(1) << 31)) return SQ_ERR_UNSUPPORTED;
    if (cs > 1) grid = tiles * cs;
    p.sk_iters = static_cast<int>(iters);
    p.sk_ctas = static_cast<int>(grid);
    p.sk_slot = gemm::BM * bn;
    p.ring = 0;                         // every stage of the ring
    if (grid == tiles || cs > 1) {
        p.ws_acc = nullptr;
        p.ws_cnt = nullptr;
    }
    if (kb2) {
        if (cs == 4) return launch_swap_bn<EPI, 2, 4, KIND>(p, bn, wq, xq, st);
        if (cs == 2) return launch_swap_bn<EPI, 2, 2, KIND>(p, bn, wq, xq, st);
        return launch_swap_bn<EPI, 2, 1, KIND>(p, bn, wq, xq, st);
    }
    if (cs == 4) return launch_swap_bn<EPI, 1, 4, KIND>(p, bn, wq, xq, st);
    if (cs == 2) return launch_swap_bn<EPI, 1, 2, KIND>(p, bn, wq, xq, st);
    return launch_swap_bn<EPI, 1, 1, KIND>(p, bn, wq, xq, st);
}

// ------------------------------------------------------------------ row kernels
// One row-kernel launch: opt-in shared memory, a grid of (blocks per SM, from
// the occupancy calculator, cached per kernel and size) x SMs, and for the
// norm-output statistic with few rows per block a cluster launch, so that the
// blocks combine their column maxima before the atomics.
template <int MODE>
cudaError_t launch_row_kernel(void (*kern)(RowArgs), int nt, size_t smem, const RowArgs &a, cudaStream_t st)
{
    cudaError_t e = cudaSuccess;
    if (smem > 0) {       // with the kernel's static shared memory it may pass the 48 KB default
        e = ensure_smem(reinterpret_cast<const void *>(kern), static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    {   // occupancy per kernel and shared-memory size, queried once
        std::lock_guard<std::mutex> lk(g_mu);
        const KernelInfo &ki = kinfo(reinterpret_cast<const void *>(kern));
        if (ki.per_sm_smem == static_cast<int>(smem)) per_sm = ki.per_sm;
    }
    if (per_sm == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, nt, smem);
        if (e != cudaSuccess) return e;
        std::lock_guard<std::mutex> lk(g_mu);
        KernelInfo &ki = kinfo(reinterpret_cast<const void *>(kern));
        ki.per_sm = per_sm;
        ki.per_sm_smem = static_cast<int>(smem);
    }
    const int sms = sm_count();
    int64_t grid = std::min<int64_t>(a.rows, static_cast<int64_t>(sms) * std::max(1, per_sm));
    if (MODE == ROW_RMS_STAT && a.rows <= 8 * grid) {
        grid = cdiv(grid, RMS_CL) * RMS_CL;       // whole clusters (blocks past the rows idle)
        return launch_pdl_cluster_smem(kern, dim3(static_cast<unsigned>(grid)), dim3(nt), RMS_CL, smem, st, a);
    }
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(nt), smem, st, a);
}

template <int DT, int MODEF>
sq_status launch_rows_dt(RowArgs a, cudaStream_t st)
{
    constexpr int MODE = MODEF & ROW_MODE_MASK;     // MODEF may carry ROW_FP8
    constexpr int EPV = VecT<DT>::EPV;
    const bool vec = aligned16(a.src0) && (a.src1 == nullptr || aligned16(a.src1)) &&
                     (a.out == nullptr || aligned16(a.out)) && (a.K % EPV) == 0 &&
                     (MODE != ROW_RMS_STAT || cdiv(a.K / EPV, ROW_T) * EPV <= 32);
    const int64_t nvec = a.K / EPV;
    // 128 threads per row for rows of up to 512 vectors, else 256
    const int nt = nvec <= 4 * 128 ? 128 : ROW_T;
    const int64_t vpt = cdiv(nvec, nt);
    // per-column constants in registers when VPT * EPV <= 32, else in shared
    // memory; the norm-output statistic stages its column maxima there
    const bool reg_rows = vpt * EPV <= 32 && MODE != ROW_RMSNORM;      // as k_rows' REG
    size_t smem = (reg_rows && MODE != ROW_RMS_STAT) ? 0 : static_cast<size_t>(a.K) * 4;
    const int sms = sm_count();
    // Rows held in registers arrive through the shared-memory row ring where
    // that measured faster (256 MiB inputs, 256-thread rows of 8192 16-bit
    // elements: per-token 0.82 -> 0.88 of HBM, weight transform 0.86 -> 0.95;
    // norm-output statistic 0.41 -> 0.56, and 0.56 -> 0.58 at 4096).  It was
    // slower for the 128-thread rows of the weight transform and for RMSNorm
    // + quant at both lengths, and for the statistic of a 2048-token batch.
    constexpr bool kRingMode = MODE == ROW_WEIGHT || MODE == ROW_ACT_TOKEN || MODE == ROW_RMS_STAT;
    const bool ring = kRingMode && reg_rows &&
                      (MODE == ROW_RMS_STAT ? a.rows >= 64 * static_cast<int64_t>(sms) : nt == ROW_T);
    if (ring) smem = ((smem + 127) & ~size_t(127)) + static_cast<size_t>(RING_ROWS) * a.row_bytes;
    a.timeout_ns = g_timeout_ns;
    // Fewer rows than SMs: the row kernel would run one latency-bound row per
    // block on a few SMs; a cluster of CTAs per row (one vector per thread)
    // spreads each row instead.  The cluster size is the smallest power of
    // two up to 8 that divides the row's vectors into at most ROW_T each.
    if (vec && a.rows < sms && a.src1 == nullptr) {
        int cs = 0;
        for (int c = 2; c <= 8; c *= 2)
            if (nvec % c == 0 && nvec / c <= ROW_T) { cs = c; break; }
        if (cs > 0) {
            const cudaError_t e = launch_pdl_cluster(k_rows_split<DT, MODEF>,
                                                     dim3(static_cast<unsigned>(cs), static_cast<unsigned>(a.rows)),
                                                     dim3(ROW_T), static_cast<unsigned>(cs), st, a);
            if (e != cudaSuccess) return cuda_fail(e);
            return check_launch();
        }
    }
    // Long rows (more than 8 vectors per thread of a 256-thread block, up to
    // 4 of a 1024-thread one): 1024 threads per row, constants in shared
    // memory, the next row's loads in flight -- 32 warps per SM where the
    // 256-thread block with 16 vectors per thread ran 8 (the 28672-element
    // rows of a 70B down projection: one block per SM either way, the
    // constants taking 114 KB).
    if constexpr (MODE == ROW_WEIGHT || MODE == ROW_ACT_TOKEN) {
        const int64_t smem_long = static_cast<size_t>(a.K) * 4;
        if (vec && nvec > 8 * ROW_T && cdiv(nvec, 1024) <= 4 && smem_long <= 200 * 1024) {
            auto kern = k_rows<DT, 4, MODEF, 1024>;
            cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), static_cast<int>(smem_long));
            if (e != cudaSuccess) return cuda_fail(e);
            const int64_t grid = std::min<int64_t>(a.rows, static_cast<int64_t>(sms));
            e = launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(1024), static_cast<size_t>(smem_long), st, a);
            if (e != cudaSuccess) return cuda_fail(e);
            return check_launch();
        }
    }
    if (vec && vpt <= 16 && smem <= 160 * 1024) {
        void (*kern)(RowArgs) = nullptr;
        if constexpr (kRingMode) {
            if (ring) {
                if (nt == 128) {
                    if constexpr (MODE == ROW_RMS_STAT) {
                        if (vpt <= 1) kern = k_rows<DT, 1, MODEF, 128, true>;
                        else if (vpt <= 2) kern = k_rows<DT, 2, MODEF, 128, true>;
                        else kern = k_rows<DT, 4, MODEF, 128, true>;
                    }
                } else if (vpt <= 1) {
                    kern = k_rows<DT, 1, MODEF, ROW_T, true>;
                } else if (vpt <= 2) {
                    kern = k_rows<DT, 2, MODEF, ROW_T, true>;
                } else if (vpt <= 4) {
                    kern = k_rows<DT, 4, MODEF, ROW_T, true>;
                } else {
                    kern = k_rows<DT, (DT == DT_F32 ? 8 : 4), MODEF, ROW_T, true>;
                }
            }
        }
        if (kern != nullptr) {
        } else if (nt == 128) {
            if (vpt <= 1) kern = k_rows<DT, 1, MODEF, 128>;
            else if (vpt <= 2) kern = k_rows<DT, 2, MODEF, 128>;
            else kern = k_rows<DT, 4, MODEF, 128>;
        } else if (vpt <= 1) {
            kern = k_rows<DT, 1, MODEF, ROW_T>;
        } else if (vpt <= 2) {
            kern = k_rows<DT, 2, MODEF, ROW_T>;
        } else if constexpr (MODE == ROW_RMS_STAT) {
            kern = k_rows<DT, (DT == DT_F32 ? 8 : 4), MODEF, ROW_T>;
        } else if (vpt <= 4) {
            kern = k_rows<DT, 4, MODEF, ROW_T>;
        } else if (vpt <= 8) {
            kern = k_rows<DT, 8, MODEF, ROW_T>;
        } else {
            kern = k_rows<DT, 16, MODEF, ROW_T>;
        }
        const cudaError_t e = launch_row_kernel<MODE>(kern, nt, smem, a, st);
        if (e != cudaSuccess) return cuda_fail(e);
    } else {
        const int64_t grid = std::min<int64_t>(a.rows, static_cast<int64_t>(sms) * 8);
        const cudaError_t e = launch_pdl(k_rows_scalar<MODEF>, dim3(static_cast<unsigned>(grid)), dim3(ROW_T), 0, st,
                                         a, static_cast<int>(DT));
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return check_launch();
}

template <int MODE>
sq_status launch_rows(RowArgs a, int dt, cudaStream_t st)
{
    if (a.rows == 0) return SQ_OK;
    if (dt == SQ_F32) return launch_rows_dt<DT_F32, MODE>(a, st);
    if (dt == SQ_F16) return launch_rows_dt<DT_F16, MODE>(a, st);
    return launch_rows_dt<DT_BF16, MODE>(a, st);
}

}  // namespace

// ---------------------------------------------------------------------------
// Fixed device scratch for sq_linear_w8a8_noalloc.  Some callers cannot call
// cudaMalloc at all: a plugin inside a host engine that owns every device
// buffer and hands the plugin only its inputs and outputs, or a serving loop
// that must never pay cudaMalloc's implicit device-wide synchronisation.  For
// them the small-M stream-K schedule (used when the cluster split is off)
// keeps its int32 partial sums and per-tile arrival counters in this
// file-scope array instead of a caller workspace.
// Every GPU that loads the library holds it (8 MiB + 64 KiB) until exit.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocAccBytes = size_t(8) << 20;            // int32 partial sums
constexpr size_t kNoAllocCntBytes = size_t(64) << 10;           // int32 tile counters
// sq_debug_inject(4): the partial-sum capacity the size check assumes, so
// that tests reach the rejection (the whole array is always allocated)
constexpr size_t kNoAllocTestCapBytes = size_t(64) << 10;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocAccBytes + kNoAllocCntBytes];

namespace {

void *g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch for the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
sq_status noalloc_scratch(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return SQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SQ_OK;
}

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

const char *sq_status_string(sq_status st)
{
    switch (st) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED";
    case SQ_ERR_MISALIGNED: return "SQ_ERR_MISALIGNED";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT";
    case SQ_ERR_WORKSPACE: return "SQ_ERR_WORKSPACE";
    }
    return "SQ_ERR_UNKNOWN";
}

int sq_last_cuda_error(void) { return t_last_cuda_error; }

void sq_set_wait_timeout_ns(unsigned long long ns) { g_timeout_ns = ns > 0 ? ns : 2000000000ull; }

void sq_debug_inject(int what) { g_inject = what & 7; }

sq_status sq_sync_status(sq_stream stream)
{
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int word = 0;
    e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word != 0) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
        return SQ_ERR_TIMEOUT;
    }
    return SQ_OK;
}

sq_status sq_calib_absmax(const void *x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld, float *absmax,
                          sq_stream stream)
{
    if (x == nullptr || absmax == nullptr || !valid_dt(dt)) return SQ_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || ld < cols || rows > (int64_t(1) << 40)) return SQ_ERR_INVALID_ARG;
    if (rows == 0) return SQ_OK;
    const cudaStream_t st = as_stream(stream);
    const int elt = dtype_size(dt);
    const int sms = sm_count();
    const bool vec = aligned16(x) && (cols * elt) % 16 == 0 && (ld * elt) % 16 == 0;
    if (vec) {
        const int64_t nvec = cols * elt / 16;
        const int64_t gx = cdiv(nvec, CALIB_TX);
        const int64_t target = static_cast<int64_t>(sms) * 8;
        int64_t gy = std::max<int64_t>(1, std::min<int64_t>(cdiv(rows, CALIB_TY * CALIB_UNROLL), cdiv(target, gx)));
        gy = std::min<int64_t>(gy, 65535);
        const int64_t slab = cdiv(rows, gy);
        gy = cdiv(rows, slab);
        dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), block(CALIB_TX, CALIB_TY);
        const uint8_t *xb = static_cast<const uint8_t *>(x);
        const int64_t ldb = ld * elt;
        const bool stream_hint = rows * ldb > (int64_t(100) << 20);     // much larger than L2 share
        cudaError_t e;
        if (stream_hint) {
            if (dt == SQ_F32) e = launch_pdl(k_colabsmax<DT_F32, true>, grid, block, 0, st, xb, rows, nvec, ldb, slab, absmax);
            else if (dt == SQ_F16) e = launch_pdl(k_colabsmax<DT_F16, true>, grid, block, 0, st, xb, rows, nvec, ldb, slab, absmax);
            else e = launch_pdl(k_colabsmax<DT_BF16, true>, grid, block, 0, st, xb, rows, nvec, ldb, slab, absmax);
        } else {
            if (dt == SQ_F32) e = launch_pdl(k_colabsmax<DT_F32, false>, grid, block, 0, st, xb, rows, nvec, ldb, slab, absmax);
            else if (dt == SQ_F16) e = launch_pdl(k_colabsmax<DT_F16, false>, grid, block, 0, st, xb, rows, nvec, ldb, slab, absmax);
            else e = launch_pdl(k_colabsmax<DT_BF16, false>, grid, block, 0, st, xb, rows, nvec, ldb, slab, absmax);
        }
        if (e != cudaSuccess) return cuda_fail(e);
    } else {
        const int64_t gx = cdiv(cols, 256);
        int64_t gy = std::max<int64_t>(1, std::min<int64_t>(cdiv(rows, 64), cdiv(static_cast<int64_t>(sms) * 8, gx)));
        gy = std::min<int64_t>(gy, 65535);
        const int64_t slab = cdiv(rows, gy);
        gy = cdiv(rows, slab);
        const cudaError_t e = launch_pdl(k_colabsmax_scalar, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                         dim3(256), 0, st, x, static_cast<int>(dt), rows, cols, ld, slab, absmax);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return check_launch();
}

static sq_status smooth_scales_q(const float *act_max, const float *w_max, int64_t K, float alpha, float *s,
                                 float *a_static, float qmax, sq_stream stream)
{
    if (act_max == nullptr || w_max == nullptr || s == nullptr || K <= 0) return SQ_ERR_INVALID_ARG;
    if (!(alpha >= 0.0f && alpha <= 1.0f)) return SQ_ERR_INVALID_ARG;
    const cudaStream_t st = as_stream(stream);
    if (K <= 8 * 1024) {    // one cluster of 8 CTAs writes the static scale itself (no pre-zeroing)
        const int threads = static_cast<int>(std::min<int64_t>(1024, ((cdiv(K, 8) + 31) / 32) * 32));
        const cudaError_t e = launch_pdl(k_smooth_scales_cluster, dim3(8), dim3(threads), 0, st, act_max, w_max,
                                         static_cast<int>(K), alpha, s, a_static, qmax);
        return e == cudaSuccess ? check_launch() : cuda_fail(e);
    }
    if (a_static != nullptr) {
        const cudaError_t e = cudaMemsetAsync(a_static, 0, sizeof(float), st);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    // one channel per thread: the fp64 log2/exp2 chain is latency-bound
    const int64_t grid = std::max<int64_t>(2, cdiv(K, 128));
    const cudaError_t e = launch_pdl(k_smooth_scales, dim3(static_cast<unsigned>(grid)), dim3(128), 0, st, act_max,
                                     w_max, K, alpha, s, a_static, qmax);
    if (e != cudaSuccess) return cuda_fail(e);
    return check_launch();
}

sq_status sq_calib_batchmax_accumulate(const void *x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                                       float *batch_max, double *sum_max, sq_stream stream)
{
    if (x == nullptr || batch_max == nullptr || sum_max == nullptr || !valid_dt(dt)) return SQ_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || ld < cols) return SQ_ERR_INVALID_ARG;
    sq_status r = sq_calib_absmax(x, dt, rows, cols, ld, batch_max, stream);
    if (r != SQ_OK) return r;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(cdiv(cols, 256), sm_count()));
    const cudaError_t e = launch_pdl(k_batchmax_accumulate, dim3(static_cast<unsigned>(grid)), dim3(256), 0,
                                     as_stream(stream), batch_max, sum_max, cols);
    return e == cudaSuccess ? check_launch() : cuda_fail(e);
}

sq_status sq_calib_mean_of_max(const double *sum_max, int64_t cols, int64_t n_batches, float *out, sq_stream stream)
{
    if (sum_max == nullptr || out == nullptr || cols <= 0 || n_batches <= 0) return SQ_ERR_INVALID_ARG;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(cdiv(cols, 256), sm_count()));
    const cudaError_t e = launch_pdl(k_mean_of_max, dim3(static_cast<unsigned>(grid)), dim3(256), 0,
                                     as_stream(stream), sum_max, cols, static_cast<double>(n_batches), out);
    return e == cudaSuccess ? check_launch() : cuda_fail(e);
}

static size_t quantile_ws_layout(int64_t cols, size_t off[3])
{
    size_t o = 0;
    off[0] = o; o = align_up(o + static_cast<size_t>(cols) * QH_BINS * 4, 256);    // histograms
    off[1] = o; o = align_up(o + static_cast<size_t>(cols) * 4, 256);              // prefixes
    off[2] = o; o = align_up(o + static_cast<size_t>(cols) * 4, 256);              // remaining ranks
    return o;
}

size_t sq_calib_quantile_workspace_size(int64_t cols)
{
    if (cols <= 0) return 0;
    size_t off[3];
    return quantile_ws_layout(cols, off);
}

extern "C++" {
template <int DT>
static sq_status quantile_dt(const void *x, int64_t rows, int64_t cols, int64_t ld, uint32_t k, float *out,
                             uint8_t *ws, const size_t off[3], cudaStream_t st)
{
    constexpr int EPV = VecT<DT>::EPV;
    uint32_t *hist = reinterpret_cast<uint32_t *>(ws + off[0]);
    uint32_t *prefix = reinterpret_cast<uint32_t *>(ws + off[1]);
    uint32_t *krem = reinterpret_cast<uint32_t *>(ws + off[2]);
    cudaError_t e = cudaMemsetAsync(hist, 0, static_cast<size_t>(cols) * QH_BINS * 4, st);
    if (e != cudaSuccess) return cuda_fail(e);
    auto hk = k_quantile_hist<DT>;
    e = ensure_smem(reinterpret_cast<const void *>(hk), QH_SMEM);
    if (e != cudaSuccess) return cuda_fail(e);
    constexpr int LANES = QH_THREADS / (QH_COLS / EPV);
    const int64_t gx = cdiv(cols, QH_COLS);
    int64_t gy = std::max<int64_t>(1, std::min<int64_t>(cdiv(rows, LANES * QH_UNROLL), cdiv(2 * sm_count(), gx)));
    gy = std::min<int64_t>(gy, 65535);
    const int64_t slab = cdiv(rows, gy);
    gy = cdiv(rows, slab);
    const int64_t ldb = ld * dtype_size(DT);
    // digits of the magnitude bits, most significant first: (shift, width)
    const int nd = DT == DT_F32 ? 4 : 2;
    const int shifts[4] = {DT == DT_F32 ? 23 : 7, DT == DT_F32 ? 15 : 0, 7, 0};
    const int widths[4] = {8, DT == DT_F32 ? 8 : 7, 8, 7};
    const unsigned sel_grid = static_cast<unsigned>(cdiv(cols * 32, 256));
    for (int i = 0; i < nd; ++i) {
        e = launch_pdl(hk, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), dim3(QH_THREADS),
                       static_cast<size_t>(QH_SMEM), st, static_cast<const uint8_t *>(x), rows, cols, ldb, slab,
                       shifts[i], widths[i], i == 0 ? static_cast<const uint32_t *>(nullptr) : prefix, hist);
        if (e != cudaSuccess) return cuda_fail(e);
        e = launch_pdl(k_quantile_select<DT>, dim3(sel_grid), dim3(256), 0, st, hist, cols, widths[i], k,
                       i == 0 ? 1 : 0, i == nd - 1 ? 1 : 0, prefix, krem, out);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return check_launch();
}
}  // extern "C++"

sq_status sq_calib_quantile(const void *x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld, double p, float *out,
                            void *workspace, size_t workspace_bytes, sq_stream stream)
{
    if (x == nullptr || out == nullptr || !valid_dt(dt)) return SQ_ERR_INVALID_ARG;
    if (rows <= 0 || rows >= (int64_t(1) << 32) || cols <= 0 || ld < cols) return SQ_ERR_INVALID_ARG;
    if (!(p > 0.0 && p <= 1.0)) return SQ_ERR_INVALID_ARG;
    size_t off[3];
    const size_t need = quantile_ws_layout(cols, off);
    if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return SQ_ERR_WORKSPACE;
    const int elt = dtype_size(dt);
    if (!aligned16(x) || (cols * elt) % 16 != 0 || (ld * elt) % 16 != 0) return SQ_ERR_MISALIGNED;
    // nearest rank: k = ceil(p * T) in fp64, within [1, T]
    const double kd = std::ceil(p * static_cast<double>(rows));
    const uint32_t k = static_cast<uint32_t>(std::min<double>(static_cast<double>(rows), std::max(1.0, kd)));
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const cudaStream_t st = as_stream(stream);
    if (dt == SQ_F32) return quantile_dt<DT_F32>(x, rows, cols, ld, k, out, ws, off, st);
    if (dt == SQ_F16) return quantile_dt<DT_F16>(x, rows, cols, ld, k, out, ws, off, st);
    return quantile_dt<DT_BF16>(x, rows, cols, ld, k, out, ws, off, st);
}

sq_status sq_smooth_scales(const float *act_max, const float *w_max, int64_t K, float alpha, float *s,
                           float *a_static, sq_stream stream)
{
    return smooth_scales_q(act_max, w_max, K, alpha, s, a_static, 127.0f, stream);
}

sq_status sq_smooth_scales_fp8(const float *act_max, const float *w_max, int64_t K, float alpha, float *s,
                               float *a_static, sq_stream stream)
{
    return smooth_scales_q(act_max, w_max, K, alpha, s, a_static, E4M3_MAX, stream);
}

extern "C++" {
template <int FMT>
static sq_status quant_weight_impl(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s, int8_t *wq,
                                   float *w_scale, sq_stream stream)
{
    if (w == nullptr || s == nullptr || wq == nullptr || w_scale == nullptr || !valid_dt(dt)) return SQ_ERR_INVALID_ARG;
    if (N < 0 || K <= 0) return SQ_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(wq)) return SQ_ERR_MISALIGNED;
    RowArgs a{};
    a.src0 = static_cast<const uint8_t *>(w);
    a.rows = N;
    a.K = K;
    a.row_bytes = K * dtype_size(dt);
    a.s = s;
    a.scale_out = w_scale;
    a.out = wq;
    return launch_rows<ROW_WEIGHT | FMT>(a, dt, as_stream(stream));
}
}  // extern "C++"

sq_status sq_quant_weight(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s, int8_t *wq,
                          float *w_scale, sq_stream stream)
{
    return quant_weight_impl<0>(w, dt, N, K, s, wq, w_scale, stream);
}

sq_status sq_quant_weight_fp8(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s, uint8_t *wq8,
                              float *w_scale, sq_stream stream)
{
    return quant_weight_impl<ROW_FP8>(w, dt, N, K, s, reinterpret_cast<int8_t *>(wq8), w_scale, stream);
}

sq_status sq_quant_weight_fold(const void *w, sq_dtype dt, int64_t N, int64_t K, const float *s, const float *s_next,
                               int8_t *wq, float *w_scale, sq_stream stream)
{
    if (w == nullptr || s == nullptr || s_next == nullptr || wq == nullptr || w_scale == nullptr || !valid_dt(dt))
        return SQ_ERR_INVALID_ARG;
    if (N < 0 || K <= 0) return SQ_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(wq)) return SQ_ERR_MISALIGNED;
    RowArgs a{};
    a.src0 = static_cast<const uint8_t *>(w);
    a.rows = N;
    a.K = K;
    a.row_bytes = K * dtype_size(dt);
    a.s = s;
    a.fold_s = s_next;
    a.scale_out = w_scale;
    a.out = wq;
    return launch_rows<ROW_WEIGHT | ROW_FOLD>(a, dt, as_stream(stream));
}

static sq_status quant_weight_gateup_impl(const void *w_gate, const void *w_up, sq_dtype dt, int64_t N_h, int64_t K,
                                          const float *s, const float *s_next, int8_t *wq_gu, float *w_scale_gu,
                                          sq_stream stream);

sq_status sq_quant_weight_gateup(const void *w_gate, const void *w_up, sq_dtype dt, int64_t N_h, int64_t K,
                                 const float *s, int8_t *wq_gu, float *w_scale_gu, sq_stream stream)
{
    return quant_weight_gateup_impl(w_gate, w_up, dt, N_h, K, s, nullptr, wq_gu, w_scale_gu, stream);
}

sq_status sq_quant_weight_gateup_fold(const void *w_gate, const void *w_up, sq_dtype dt, int64_t N_h, int64_t K,
                                      const float *s, const float *s_next, int8_t *wq_gu, float *w_scale_gu,
                                      sq_stream stream)
{
    if (s_next == nullptr) return SQ_ERR_INVALID_ARG;
    return quant_weight_gateup_impl(w_gate, w_up, dt, N_h, K, s, s_next, wq_gu, w_scale_gu, stream);
}

static sq_status quant_weight_gateup_impl(const void *w_gate, const void *w_up, sq_dtype dt, int64_t N_h, int64_t K,
                                          const float *s, const float *s_next, int8_t *wq_gu, float *w_scale_gu,
                                          sq_stream stream)
{
    if (w_gate == nullptr || w_up == nullptr || s == nullptr || wq_gu == nullptr || w_scale_gu == nullptr ||
        !valid_dt(dt))
        return SQ_ERR_INVALID_ARG;
    if (N_h <= 0 || K <= 0 || (N_h % 32) != 0) return SQ_ERR_INVALID_ARG;
    if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(wq_gu)) return SQ_ERR_MISALIGNED;
    RowArgs a{};
    a.src0 = static_cast<const uint8_t *>(w_gate);
    a.src1 = static_cast<const uint8_t *>(w_up);
    a.rows = 2 * N_h;
    a.K = K;
    a.row_bytes = K * dtype_size(dt);
    a.s = s;
    a.fold_s = s_next;
    a.scale_out = w_scale_gu;
    a.out = wq_gu;
    if (s_next != nullptr) return launch_rows<ROW_WEIGHT | ROW_FOLD>(a, dt, as_stream(stream));
    return launch_rows<ROW_WEIGHT>(a, dt, as_stream(stream));
}

extern "C++" {
template <int FMT>
static sq_status smooth_quant_act_impl(const void *x, sq_dtype dt, int64_t M, int64_t K, const float *s,
                                       sq_act_mode mode, float *a_scale, int8_t *xq, sq_stream stream)
{
    constexpr bool F8 = FMT != 0;
    if (x == nullptr || s == nullptr || a_scale == nullptr || xq == nullptr || !valid_dt(dt)) return SQ_ERR_INVALID_ARG;
    if (M < 0 || K <= 0 || (mode != SQ_ACT_STATIC && mode != SQ_ACT_PER_TOKEN)) return SQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(xq)) return SQ_ERR_MISALIGNED;
    RowArgs a{};
    a.src0 = static_cast<const uint8_t *>(x);
    a.rows = M;
    a.K = K;
    a.row_bytes = K * dtype_size(dt);
    a.s = s;
    a.out = xq;
    if (mode == SQ_ACT_STATIC) {
        a.a_in = a_scale;
        const int elt = dtype_size(dt);
        if (M > 0 && (K * elt) % 16 == 0) {
            // elementwise: column strips x row slabs, like the calibration statistic
            const int64_t nvec = K * elt / 16;
            const int64_t gx = cdiv(nvec, QS_TX);
            const int64_t target = static_cast<int64_t>(sm_count()) * 8;
            int64_t gy = std::max<int64_t>(1, std::min<int64_t>(cdiv(M, QS_TY * QS_UNROLL), cdiv(target, gx)));
            gy = std::min<int64_t>(gy, 65535);
            const int64_t slab = cdiv(M, gy);
            gy = cdiv(M, slab);
            const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), block(QS_TX, QS_TY);
            const uint8_t *xb = static_cast<const uint8_t *>(x);
            const bool big = M * K * elt > (int64_t(100) << 20);
            const bool one = slab <= QS_UNROLL * QS_TY;
            const cudaStream_t st = as_stream(stream);
            auto go = [&](auto kern) { return launch_pdl(kern, grid, block, 0, st, xb, M, nvec, s, a_scale, slab, xq); };
            cudaError_t e;
            if (dt == SQ_F32)
                e = big ? go(k_quant_static<DT_F32, true, false, F8>)
                        : one ? go(k_quant_static<DT_F32, false, true, F8>)
                              : go(k_quant_static<DT_F32, false, false, F8>);
            else if (dt == SQ_F16)
                e = big ? go(k_quant_static<DT_F16, true, false, F8>)
                        : one ? go(k_quant_static<DT_F16, false, true, F8>)
                              : go(k_quant_static<DT_F16, false, false, F8>);
            else
                e = big ? go(k_quant_static<DT_BF16, true, false, F8>)
                        : one ? go(k_quant_static<DT_BF16, false, true, F8>)
                              : go(k_quant_static<DT_BF16, false, false, F8>);
            if (e != cudaSuccess) return cuda_fail(e);
            return check_launch();
        }
        return launch_rows<ROW_ACT_STATIC | FMT>(a, dt, as_stream(stream));
    }
    a.scale_out = a_scale;
    return launch_rows<ROW_ACT_TOKEN | FMT>(a, dt, as_stream(stream));
}
}  // extern "C++"

sq_status sq_smooth_quant_act(const void *x, sq_dtype dt, int64_t M, int64_t K, const float *s, sq_act_mode mode,
                              float *a_scale, int8_t *xq, sq_stream stream)
{
    return smooth_quant_act_impl<0>(x, dt, M, K, s, mode, a_scale, xq, stream);
}

sq_status sq_smooth_quant_act_fp8(const void *x, sq_dtype dt, int64_t M, int64_t K, const float *s,
                                  sq_act_mode mode, float *a_scale, uint8_t *xq8, sq_stream stream)
{
    return smooth_quant_act_impl<ROW_FP8>(x, dt, M, K, s, mode, a_scale, reinterpret_cast<int8_t *>(xq8), stream);
}


sq_status sq_rmsnorm_quant(const void *x, sq_dtype dt, int64_t M, int64_t d, const float *gamma, const float *s,
                           float eps, const float *a_scale, int8_t *xq, float *rstd, sq_stream stream)
{
    if (x == nullptr || gamma == nullptr || s == nullptr || a_scale == nullptr || xq == nullptr || !valid_dt(dt))
        return SQ_ERR_INVALID_ARG;
    if (M < 0 || d <= 0 || !(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(xq)) return SQ_ERR_MISALIGNED;
    RowArgs a{};
    a.src0 = static_cast<const uint8_t *>(x);
    a.rows = M;
    a.K = d;
    a.row_bytes = d * dtype_size(dt);
    a.s = s;
    a.gamma = gamma;
    a.eps = eps;
    a.a_in = a_scale;
    a.rstd_out = rstd;
    a.out = xq;
    return launch_rows<ROW_RMSNORM>(a, dt, as_stream(stream));
}

sq_status sq_rmsnorm_absmax(const void *x, sq_dtype dt, int64_t M, int64_t d, const float *gamma, float eps,
                            float *absmax, sq_stream stream)
{
    if (x == nullptr || gamma == nullptr || absmax == nullptr || !valid_dt(dt)) return SQ_ERR_INVALID_ARG;
    if (M < 0 || d <= 0 || !(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
    if (!aligned16(x)) return SQ_ERR_MISALIGNED;
    RowArgs a{};
    a.src0 = static_cast<const uint8_t *>(x);
    a.rows = M;
    a.K = d;
    a.row_bytes = d * dtype_size(dt);
    a.gamma = gamma;
    a.eps = eps;
    a.scale_out = absmax;
    return launch_rows<ROW_RMS_STAT>(a, dt, as_stream(stream));
}

size_t sq_linear_workspace_size(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return ws_bytes(M, N, K);
}

static sq_status check_gemm_shape(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K)
{
    if (xq == nullptr || wq == nullptr) return SQ_ERR_INVALID_ARG;
    if (M < 1 || N < 16 || K < 16 || (N % 16) != 0 || (K % 16) != 0) return SQ_ERR_INVALID_ARG;
    if (K >= 133144 || M > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return SQ_ERR_UNSUPPORTED;
    if (!aligned16(xq) || !aligned16(wq)) return SQ_ERR_MISALIGNED;
    return SQ_OK;
}

static sq_status linear_w8a8_impl(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                                  const float *a_scale, sq_act_mode mode, const float *w_scale, int scales_f16,
                                  const void *bias, sq_dtype out_dt, void *y, void *workspace,
                                  size_t workspace_bytes, sq_stream stream)
{
    const cudaStream_t st = as_stream(stream);
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.a_scale = a_scale;
    p.per_token = (mode == SQ_ACT_PER_TOKEN) ? 1 : 0;
    p.w_scale = w_scale;
    p.scales_f16 = scales_f16;
    p.bias = bias;
    p.out = y;
    p.out_dt = out_dt;
    if (use_pair_t(M, N, K)) return dispatch_pair_t<gemm::KIND_I8>(p, xq, wq, st);
    if (M <= kSwapMaxM) {
        const int64_t tiles = swap_tiles(M, N);
        if (const int cs = swap_cluster_split(M, N, K); cs > 1)
            return dispatch_swap<gemm::EPI_DEQUANT>(p, xq, wq, st, tiles, cs);
        const int64_t g = swap_grid(M, N, K, SIZE_MAX);
        const size_t need = ws_bytes(M, N, K);
        if (g != tiles && workspace != nullptr && workspace_bytes >= need && aligned16(workspace)) {
            p.ws_acc = static_cast<int32_t *>(workspace);
            p.ws_cnt = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + swap_slot_bytes(M, g));
            return dispatch_swap<gemm::EPI_DEQUANT>(p, xq, wq, st, g);
        }
        return dispatch_swap<gemm::EPI_DEQUANT>(p, xq, wq, st, tiles);
    }
    return dispatch_pair<gemm::KIND_I8, gemm::EPI_DEQUANT>(p, xq, wq, st);
}

sq_status sq_linear_w8a8(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K, const float *a_scale,
                         sq_act_mode mode, const float *w_scale, const void *bias, sq_dtype out_dt, void *y,
                         void *workspace, size_t workspace_bytes, sq_stream stream)
{
    sq_status r = check_gemm_shape(xq, wq, M, N, K);
    if (r != SQ_OK) return r;
    if (a_scale == nullptr || w_scale == nullptr || y == nullptr || !valid_dt(out_dt)) return SQ_ERR_INVALID_ARG;
    if (mode != SQ_ACT_STATIC && mode != SQ_ACT_PER_TOKEN) return SQ_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(w_scale)) return SQ_ERR_MISALIGNED;
    return linear_w8a8_impl(xq, wq, M, N, K, a_scale, mode, w_scale, 0, bias, out_dt, y, workspace, workspace_bytes,
                            stream);
}

sq_status sq_linear_fp8(const uint8_t *xq8, const uint8_t *wq8, int64_t M, int64_t N, int64_t K,
                        const float *a_scale, sq_act_mode mode, const float *w_scale, const void *bias,
                        sq_dtype out_dt, void *y, sq_stream stream)
{
    sq_status r = check_gemm_shape(reinterpret_cast<const int8_t *>(xq8), reinterpret_cast<const int8_t *>(wq8), M,
                                   N, K);
    if (r != SQ_OK) return r;
    if (a_scale == nullptr || w_scale == nullptr || y == nullptr || !valid_dt(out_dt)) return SQ_ERR_INVALID_ARG;
    if (mode != SQ_ACT_STATIC && mode != SQ_ACT_PER_TOKEN) return SQ_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(w_scale)) return SQ_ERR_MISALIGNED;
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.a_scale = a_scale;
    p.per_token = (mode == SQ_ACT_PER_TOKEN) ? 1 : 0;
    p.w_scale = w_scale;
    p.bias = bias;
    p.out = y;
    p.out_dt = out_dt;
    const cudaStream_t st = as_stream(stream);
    if (use_pair_t(M, N, K)) return dispatch_pair_t<gemm::KIND_F8>(p, xq8, wq8, st);
    if (M <= kSwapMaxM) {
        // weight streaming (the weights fill the 128-row MMA): the cluster
        // split when one tile per CTA would leave most SMs idle, else one
        // tile per CTA (the stream-K schedule needs a workspace: not used here)
        const int cs = swap_cluster_split(M, N, K);
        return dispatch_swap<gemm::EPI_DEQUANT, gemm::KIND_F8>(p, xq8, wq8, st, swap_tiles(M, N), cs);
    }
    return dispatch_pair<gemm::KIND_F8, gemm::EPI_DEQUANT>(p, xq8, wq8, st);
}

sq_status sq_scales_to_f16(const float *in, int64_t n, uint16_t *out, sq_stream stream)
{
    if (in == nullptr || out == nullptr || n < 0) return SQ_ERR_INVALID_ARG;
    if (n == 0) return SQ_OK;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(cdiv(n, 256), 4 * sm_count()));
    const cudaError_t e = launch_pdl(k_f32_to_f16, dim3(static_cast<unsigned>(grid)), dim3(256), 0, as_stream(stream),
                                     in, n, reinterpret_cast<__half *>(out));
    return e == cudaSuccess ? check_launch() : cuda_fail(e);
}

sq_status sq_scales_from_f16(const uint16_t *in, int64_t n, float *out, sq_stream stream)
{
    if (in == nullptr || out == nullptr || n < 0) return SQ_ERR_INVALID_ARG;
    if (n == 0) return SQ_OK;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(cdiv(n, 256), 4 * sm_count()));
    const cudaError_t e = launch_pdl(k_f16_to_f32, dim3(static_cast<unsigned>(grid)), dim3(256), 0, as_stream(stream),
                                     reinterpret_cast<const __half *>(in), n, out);
    return e == cudaSuccess ? check_launch() : cuda_fail(e);
}

sq_status sq_linear_w8a8_f16scales(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                                   const uint16_t *a_scale_f16, sq_act_mode mode, const uint16_t *w_scale_f16,
                                   const void *bias, sq_dtype out_dt, void *y, void *workspace,
                                   size_t workspace_bytes, sq_stream stream)
{
    sq_status r = check_gemm_shape(xq, wq, M, N, K);
    if (r != SQ_OK) return r;
    if (a_scale_f16 == nullptr || w_scale_f16 == nullptr || y == nullptr || !valid_dt(out_dt))
        return SQ_ERR_INVALID_ARG;
    if (mode != SQ_ACT_STATIC && mode != SQ_ACT_PER_TOKEN) return SQ_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(w_scale_f16)) return SQ_ERR_MISALIGNED;
    return linear_w8a8_impl(xq, wq, M, N, K, reinterpret_cast<const float *>(a_scale_f16), mode,
                            reinterpret_cast<const float *>(w_scale_f16), 1, bias, out_dt, y, workspace,
                            workspace_bytes, stream);
}

size_t sq_linear_w8a8_noalloc_max_elems(void) { return kNoAllocAccBytes / 4; }

sq_status sq_linear_w8a8_noalloc(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                                 const float *a_scale, sq_act_mode mode, const float *w_scale, const void *bias,
                                 sq_dtype out_dt, void *y, sq_stream stream)
{
    sq_status r = check_gemm_shape(xq, wq, M, N, K);
    if (r != SQ_OK) return r;
    if (a_scale == nullptr || w_scale == nullptr || y == nullptr || !valid_dt(out_dt)) return SQ_ERR_INVALID_ARG;
    if (mode != SQ_ACT_STATIC && mode != SQ_ACT_PER_TOKEN) return SQ_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(w_scale)) return SQ_ERR_MISALIGNED;
    if (M > kSwapMaxM)      // the large-M path needs no scratch: same launch as sq_linear_w8a8
        return sq_linear_w8a8(xq, wq, M, N, K, a_scale, mode, w_scale, bias, out_dt, y, nullptr, 0, stream);
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.a_scale = a_scale;
    p.per_token = (mode == SQ_ACT_PER_TOKEN) ? 1 : 0;
    p.w_scale = w_scale;
    p.bias = bias;
    p.out = y;
    p.out_dt = out_dt;
    const cudaStream_t st = as_stream(stream);
    if (use_pair_t(M, N, K)) return dispatch_pair_t<gemm::KIND_I8>(p, xq, wq, st);   // no scratch
    const int64_t tiles = swap_tiles(M, N);
    if (const int cs = swap_cluster_split(M, N, K); cs > 1)   // partial sums stay on chip: no scratch
        return dispatch_swap<gemm::EPI_DEQUANT>(p, xq, wq, st, tiles, cs);
    // the stream-K schedule of sq_linear_w8a8 (same CTAs, same partial sums):
    // it is the only schedule that needs scratch, and only when tiles are shared
    const int64_t g = swap_grid(M, N, K, SIZE_MAX);
    if (g == tiles) return dispatch_swap<gemm::EPI_DEQUANT>(p, xq, wq, st, tiles);
    const size_t acc_cap = (g_inject & 4) ? kNoAllocTestCapBytes : kNoAllocAccBytes;
    const size_t cnt_bytes = static_cast<size_t>(tiles) * 4;
    if (swap_slot_bytes(M, g) > acc_cap || cnt_bytes > kNoAllocCntBytes) return SQ_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((r = noalloc_scratch(&scratch)) != SQ_OK) return r;
    int *cnt = reinterpret_cast<int *>(static_cast<unsigned char *>(scratch) + kNoAllocAccBytes);
    // the array keeps whatever the previous call left (a call that timed out
    // leaves its counters raised): the per-tile arrival counters must start at
    // zero; a partial-sum slot is always written before it is read
    cudaError_t e = cudaMemsetAsync(cnt, 0, cnt_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e);
    p.ws_acc = static_cast<int32_t *>(scratch);
    p.ws_cnt = cnt;
    return dispatch_swap<gemm::EPI_DEQUANT>(p, xq, wq, st, g);
}

sq_status sq_gemm_s32(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K, int32_t *acc,
                      sq_stream stream)
{
    sq_status r = check_gemm_shape(xq, wq, M, N, K);
    if (r != SQ_OK) return r;
    if (acc == nullptr) return SQ_ERR_INVALID_ARG;
    if (!aligned16(acc)) return SQ_ERR_MISALIGNED;
    const cudaStream_t st = as_stream(stream);
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.out = acc;
    if (M <= kSwapMaxM) return dispatch_swap<gemm::EPI_S32>(p, xq, wq, st, swap_tiles(M, N), swap_cluster_split(M, N, K));
    return dispatch_pair<gemm::KIND_I8, gemm::EPI_S32>(p, xq, wq, st);
}

sq_status sq_linear_w8a8_gateup_silu(const int8_t *xq, const int8_t *wq_gu, int64_t M, int64_t N_h, int64_t K,
                                     const float *a_scale, sq_act_mode mode, const float *w_scale_gu, void *h,
                                     const float *s2, const float *a2, int8_t *hq, sq_stream stream)
{
    sq_status r = check_gemm_shape(xq, wq_gu, M, 2 * N_h, K);
    if (r != SQ_OK) return r;
    if (a_scale == nullptr || w_scale_gu == nullptr || (h == nullptr && hq == nullptr)) return SQ_ERR_INVALID_ARG;
    if ((N_h % 128) != 0) return SQ_ERR_INVALID_ARG;
    if (hq != nullptr && a2 == nullptr) return SQ_ERR_INVALID_ARG;     // s2 == null: folded into W_up
    if (mode != SQ_ACT_STATIC && mode != SQ_ACT_PER_TOKEN) return SQ_ERR_INVALID_ARG;
    if ((h != nullptr && !aligned16(h)) || (hq != nullptr && !aligned16(hq))) return SQ_ERR_MISALIGNED;
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(2 * N_h);
    p.K = static_cast<int>(K);
    p.a_scale = a_scale;
    p.per_token = (mode == SQ_ACT_PER_TOKEN) ? 1 : 0;
    p.w_scale = w_scale_gu;
    p.out = h;
    p.out_dt = SQ_BF16;
    p.s2 = s2;
    p.a2 = a2;
    p.hq = hq;
    return dispatch_pair<gemm::KIND_I8, gemm::EPI_GATEUP>(p, xq, wq_gu, as_stream(stream), 256);
}

sq_status sq_linear_w8a8_gateup_silu_absmax(const int8_t *xq, const int8_t *wq_gu, int64_t M, int64_t N_h,
                                            int64_t K, const float *a_scale, sq_act_mode mode,
                                            const float *w_scale_gu, float *h_absmax, sq_stream stream)
{
    sq_status r = check_gemm_shape(xq, wq_gu, M, 2 * N_h, K);
    if (r != SQ_OK) return r;
    if (a_scale == nullptr || w_scale_gu == nullptr || h_absmax == nullptr) return SQ_ERR_INVALID_ARG;
    if ((N_h % 128) != 0) return SQ_ERR_INVALID_ARG;
    if (mode != SQ_ACT_STATIC && mode != SQ_ACT_PER_TOKEN) return SQ_ERR_INVALID_ARG;
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(2 * N_h);
    p.K = static_cast<int>(K);
    p.a_scale = a_scale;
    p.per_token = (mode == SQ_ACT_PER_TOKEN) ? 1 : 0;
    p.w_scale = w_scale_gu;
    p.out = nullptr;
    p.out_dt = SQ_BF16;
    p.hmax = h_absmax;
    return dispatch_pair<gemm::KIND_I8, gemm::EPI_GATEUP>(p, xq, wq_gu, as_stream(stream), 256);
}

sq_status sq_gemm_f16_ref(const void *x, const void *w, int64_t M, int64_t N, int64_t K, void *y, sq_stream stream)
{
    if (x == nullptr || w == nullptr || y == nullptr) return SQ_ERR_INVALID_ARG;
    if (M < 1 || N < 16 || K < 8 || (N % 16) != 0 || (K % 8) != 0) return SQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return SQ_ERR_MISALIGNED;
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.out = y;
    p.out_dt = SQ_F16;
    return dispatch_pair<gemm::KIND_F16, gemm::EPI_F16>(p, x, w, as_stream(stream), 256);
}

sq_status sq_sse_f16(const void *y, const void *y_ref, int64_t n, double *sse, sq_stream stream)
{
    if (y == nullptr || y_ref == nullptr || sse == nullptr || n < 0) return SQ_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(y_ref)) return SQ_ERR_MISALIGNED;
    if (n == 0) return SQ_OK;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(cdiv(n, 8 * 256), static_cast<int64_t>(sm_count()) * 4));
    const cudaError_t e = launch_pdl(k_sse_f16, dim3(static_cast<unsigned>(grid)), dim3(256), 0, as_stream(stream),
                                     static_cast<const __half *>(y), static_cast<const __half *>(y_ref), n, sse);
    if (e != cudaSuccess) return cuda_fail(e);
    return check_launch();
}

static size_t alpha_ws_layout(int64_t Mh, int64_t N, int64_t K, int n_alpha, size_t off[8])
{
    size_t o = 0;
    off[0] = o; o = align_up(o + static_cast<size_t>(K) * 4, 256);          // s
    off[1] = o; o = align_up(o + 4, 256);                                   // a
    off[2] = o; o = align_up(o + static_cast<size_t>(N * K), 256);          // wq
    off[3] = o; o = align_up(o + static_cast<size_t>(N) * 4, 256);          // w_scale
    off[4] = o; o = align_up(o + static_cast<size_t>(Mh * K), 256);         // xq
    off[5] = o; o = align_up(o + static_cast<size_t>(Mh * N) * 2, 256);     // y
    off[6] = o; o = align_up(o + static_cast<size_t>(Mh * N) * 2, 256);     // y_ref
    off[7] = o; o = align_up(o + static_cast<size_t>(n_alpha) * 8, 256);    // sse
    const size_t lin = ws_bytes(Mh, N, K);
    return o + lin;
}

size_t sq_alpha_search_workspace_size(int64_t M_held, int64_t N, int64_t K, int n_alpha)
{
    if (M_held <= 0 || N <= 0 || K <= 0 || n_alpha <= 0) return 0;
    size_t off[8];
    return alpha_ws_layout(M_held, N, K, n_alpha, off);
}

sq_status sq_alpha_search(const void *x_held, const void *w, int64_t M_held, int64_t N, int64_t K,
                          const float *act_max, const float *w_max, const float *alphas, int n_alpha,
                          void *workspace, size_t workspace_bytes, float *best_alpha, double *mse,
                          sq_stream stream)
{
    if (x_held == nullptr || w == nullptr || act_max == nullptr || w_max == nullptr || alphas == nullptr ||
        best_alpha == nullptr || workspace == nullptr)
        return SQ_ERR_INVALID_ARG;
    if (n_alpha < 1 || n_alpha > 16) return SQ_ERR_INVALID_ARG;
    for (int i = 0; i < n_alpha; ++i)
        if (!(alphas[i] >= 0.0f && alphas[i] <= 1.0f) || (i > 0 && !(alphas[i] > alphas[i - 1])))
            return SQ_ERR_INVALID_ARG;
    size_t off[8];
    const size_t need = alpha_ws_layout(M_held, N, K, n_alpha, off);
    if (workspace_bytes < need || !aligned16(workspace)) return SQ_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *s = reinterpret_cast<float *>(ws + off[0]);
    float *a = reinterpret_cast<float *>(ws + off[1]);
    int8_t *wq = reinterpret_cast<int8_t *>(ws + off[2]);
    float *w_scale = reinterpret_cast<float *>(ws + off[3]);
    int8_t *xq = reinterpret_cast<int8_t *>(ws + off[4]);
    void *y = ws + off[5];
    void *y_ref = ws + off[6];
    double *sse = reinterpret_cast<double *>(ws + off[7]);
    void *lin_ws = ws + (need - ws_bytes(M_held, N, K));
    const size_t lin_bytes = ws_bytes(M_held, N, K);
    const cudaStream_t st = as_stream(stream);

    sq_status r = sq_gemm_f16_ref(x_held, w, M_held, N, K, y_ref, stream);
    if (r != SQ_OK) return r;
    cudaError_t e = cudaMemsetAsync(sse, 0, static_cast<size_t>(n_alpha) * 8, st);
    if (e != cudaSuccess) return cuda_fail(e);
    if (lin_bytes > 0) {
        e = cudaMemsetAsync(lin_ws, 0, lin_bytes, st);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    for (int i = 0; i < n_alpha; ++i) {
        if ((r = sq_smooth_scales(act_max, w_max, K, alphas[i], s, a, stream)) != SQ_OK) return r;
        if ((r = sq_quant_weight(w, SQ_F16, N, K, s, wq, w_scale, stream)) != SQ_OK) return r;
        if ((r = sq_smooth_quant_act(x_held, SQ_F16, M_held, K, s, SQ_ACT_STATIC, a, xq, stream)) != SQ_OK) return r;
        if ((r = sq_linear_w8a8(xq, wq, M_held, N, K, a, SQ_ACT_STATIC, w_scale, nullptr, SQ_F16, y, lin_ws,
                                lin_bytes, stream)) != SQ_OK)
            return r;
        if ((r = sq_sse_f16(y, y_ref, M_held * N, sse + i, stream)) != SQ_OK) return r;
    }
    double host_sse[16];
    e = cudaMemcpyAsync(host_sse, sse, static_cast<size_t>(n_alpha) * 8, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e);
    r = sq_sync_status(stream);
    if (r != SQ_OK) return r;
    const double n = static_cast<double>(M_held) * static_cast<double>(N);
    int best = 0;
    for (int i = 0; i < n_alpha; ++i) {
        const double m = host_sse[i] / n;
        if (mse != nullptr) mse[i] = m;
        if (i > 0 && m < (host_sse[best] / n) * (1.0 - 1e-6)) best = i;
    }
    *best_alpha = alphas[best];
    return SQ_OK;
}

}  // extern "C"
