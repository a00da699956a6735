// C-ABI entry points of libpgf8: argument checks, kernel choice, tensor-map
// encoding and launches.  The operations are specified in include/pgf8.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cmath>
#include <cstring>
#include <mutex>

#include "pgf8.h"
#include "gemm.cuh"
#include "kvcache.cuh"
#include "attention.cuh"
#include "attention_context.cuh"
#include "gemm_persistent.cuh"
#include "gemm_streamk.cuh"
#include "gemm_2sm.cuh"
#include "gemm_group.cuh"
#include "gemm_pair_group.cuh"
#include "gemm_persistent_swap.cuh"
#include "quantize.cuh"

// Pipeline depths and stream-K occupancy (compile-time tuning constants).
#ifndef PGF8_SKINNY16_STAGES
#define PGF8_SKINNY16_STAGES 6
#endif
// Skinny split-K grids are kept within this many CTAs per SM, times 4.
#ifndef PGF8_SKINNY_CTAS_PER_SM_X4
#define PGF8_SKINNY_CTAS_PER_SM_X4 7
#endif
// In-GEMM quantisation of dynamic activations is used up to this many tokens
// and this many K-splits (beyond: the quantisation kernel, then the GEMM).
#ifndef PGF8_FUSED_MAX_M
#define PGF8_FUSED_MAX_M 32
#endif
#ifndef PGF8_FUSED_MAX_SPLITS
#define PGF8_FUSED_MAX_SPLITS 8
#endif
#ifndef PGF8_STREAMK16_STAGES
#define PGF8_STREAMK16_STAGES 6
#endif
// Layers of a grouped call with at most this many tokens run in the grouped
// weight-streaming kernel; larger ones take the per-layer kernels.
#ifndef PGF8_GROUP_MAX_M
#define PGF8_GROUP_MAX_M 256
#endif
#ifndef PGF8_STREAMK_CTAS_PER_SM
#define PGF8_STREAMK_CTAS_PER_SM 1
#endif

namespace pgf8 {

static thread_local int tl_last_cuda_error = 0;

static pgf8_status cuda_fail(cudaError_t e)
{
    tl_last_cuda_error = static_cast<int>(e);
    return PGF8_ERR_CUDA;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
static size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------------ per-device set-up
// Kernel attributes (dynamic shared-memory limit, carveout), occupancy
// answers and SM counts belong to one device: a process that drives several
// GPUs sets and queries them once for each device, on the first launch with
// that device current.  Ordinals past kSetupDevices are set up on every call.
constexpr int kSetupDevices = 64;

struct PerDeviceSetup {
    std::mutex mu;
    bool done[kSetupDevices] = {};
    cudaError_t err[kSetupDevices] = {};
    int value[kSetupDevices] = {};
};

// Runs `fn` (returning cudaError_t, writing an int) once per device and
// returns its cached status; `*value` receives the cached int.
template <class Fn> static cudaError_t setup_once_per_device(PerDeviceSetup &st, Fn fn, int *value = nullptr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kSetupDevices) {
        int v = 0;
        e = fn(dev, &v);
        if (value)
            *value = v;
        return e;
    }
    std::lock_guard<std::mutex> lock(st.mu);
    if (!st.done[dev]) {
        st.err[dev] = fn(dev, &st.value[dev]);
        st.done[dev] = true;
    }
    if (value)
        *value = st.value[dev];
    return st.err[dev];
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major [rows, cols] tensor; box = box_cols x box_rows; element
// size from dtype.  Out-of-range elements of a box read as zero.
static bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t rows,
                     uint64_t cols, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw,
                     uint64_t row_stride_elems = 0)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {(row_stride_elems ? row_stride_elems : cols) * static_cast<uint64_t>(elem_bytes)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM launch
struct GemmLaunch {
    int kind;          // OpKind
    const void *x;     // E4M3 codes or FP16 activations [M, K]
    const void *w;     // E4M3 codes or hi plane [N, K]
    const void *w2;    // lo plane (kNested16)
    const float *sa, *sw;
    void *y;
    int M, N, K;
    int pdl;           // launch with programmatic stream serialization
    int prefetch_w;    // weights may be read before the dependency resolves
    pgf8_linear_opts opts;
    cudaStream_t stream;
    void *ws;          // stream-K region of the workspace (flags, then partial slots), or null
    size_t ws_bytes;
    // in-kernel quantisation (XQ kernels): raw activations and side outputs
    const void *xraw = nullptr;
    int64_t ldx = 0;
    int out_f32 = 0;   // pair kernel: f32 outputs
    uint8_t *q_out = nullptr;
    float *sa_out = nullptr;
};

// Tensor maps of the two operands for a kernel configuration C (tile rows
// C::kRowsX / C::kRowsW, 128 bytes of K per box).
template <class C> static bool make_operand_maps(const GemmLaunch &L, CUtensorMap &tmX, CUtensorMap &tmW,
                                                 CUtensorMap &tmW2)
{
    const bool nest16 = (C::KIND == kNested16);
    std::memset(&tmW2, 0, sizeof(tmW2));
    bool ok;
    if constexpr (C::XQ != 0) {
        // the kernel loads the activations itself; only the weight map is used
        std::memset(&tmX, 0, sizeof(tmX));
        ok = make_map(&tmW, L.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.N, L.K, 128, C::kRowsW,
                      CU_TENSOR_MAP_SWIZZLE_128B);
        tmW2 = tmW;
    } else if (nest16) {
        ok = make_map(&tmX, L.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, L.M, L.K, 64, C::kRowsX,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&tmW, L.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.N, L.K, 64, C::kRowsW,
                      CU_TENSOR_MAP_SWIZZLE_NONE) &&
             make_map(&tmW2, L.w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.N, L.K, 64, C::kRowsW,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        ok = make_map(&tmX, L.x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.M, L.K, 128, C::kRowsX,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
             make_map(&tmW, L.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.N, L.K, 128, C::kRowsW,
                      CU_TENSOR_MAP_SWIZZLE_128B);
        tmW2 = tmW;
    }
    return ok;
}

static GemmParams make_params(const GemmLaunch &L, int splits)
{
    const bool nest16 = (L.kind == kNested16);
    GemmParams p;
    p.M = L.M;
    p.N = L.N;
    p.K = L.K;
    p.kblocks = static_cast<int>((static_cast<int64_t>(L.K) * (nest16 ? 2 : 1) + 127) / 128);
    p.splits = splits;
    p.prefetch_w = L.prefetch_w;
    p.sa = L.sa;
    p.sw = L.sw;
    p.y = L.y;
    p.out_f32 = L.out_f32;
    p.x = L.xraw;
    p.ldx = L.ldx;
    p.q_out = L.q_out;
    p.sa_out = L.sa_out;
    return p;
}

static void fill_attrs(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attrs, int cluster_z, int pdl,
                       int cluster_x = 1)
{
    int na = 0;
    if (cluster_z > 1 || cluster_x > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = static_cast<unsigned>(cluster_z);
        ++na;
    }
    if (pdl) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
}

template <class C> static pgf8_status launch_cfg(const GemmLaunch &L, int splits)
{
    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        // the largest shared-memory carveout: the default sizes the SM's
        // L1 / shared split for one CTA, which leaves the skinny kernels
        // (about 110 KB each) at one CTA per SM
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemm_kernel<C>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared);
        return e;
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    CUtensorMap tmX, tmW, tmW2;
    if (!make_operand_maps<C>(L, tmX, tmW, tmW2))
        return PGF8_ERR_UNSUPPORTED;
    const GemmParams p = make_params(L, splits);

    const int rows_a = C::SWAP ? L.N : L.M;   // A side: 128-row tiles
    const int rows_b = C::SWAP ? L.M : L.N;   // B side: BN-row tiles
    dim3 grid((rows_a + 127) / 128, (rows_b + C::BN - 1) / C::BN, splits);

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = L.stream;
    cudaLaunchAttribute attrs[2];
    fill_attrs(cfg, attrs, C::SPLIT ? splits : 1, L.pdl);
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_kernel<C>, tmX, tmW, tmW2, p);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

static int num_sms();

// Persistent tiled kernel: one CTA per SM (at most one per tile).
template <class C> static pgf8_status launch_persistent(const GemmLaunch &L)
{
    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        return cudaFuncSetAttribute(gemm_persistent_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    CUtensorMap tmX, tmW, tmW2;
    if (!make_operand_maps<C>(L, tmX, tmW, tmW2))
        return PGF8_ERR_UNSUPPORTED;
    const GemmParams p = make_params(L, 1);
    const int64_t tiles = static_cast<int64_t>((L.M + 127) / 128) * ((L.N + C::BN - 1) / C::BN);
    const int sms = num_sms();
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(tiles < sms ? tiles : sms), 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = L.stream;
    cudaLaunchAttribute attrs[2];
    fill_attrs(cfg, attrs, 1, L.pdl);
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_persistent_kernel<C>, tmX, tmW, tmW2, p);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

// NestedFP FP16 mode, swapped orientation: one CTA per SM (at most one per
// tile of 128 weight rows x BN tokens).
template <class C> static pgf8_status launch_persistent_swap(const GemmLaunch &L)
{
    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        return cudaFuncSetAttribute(gemm_persistent_swap_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    CUtensorMap tmX, tmW, tmW2;
    if (!make_operand_maps<C>(L, tmX, tmW, tmW2))
        return PGF8_ERR_UNSUPPORTED;
    const GemmParams p = make_params(L, 1);
    const int64_t tiles = static_cast<int64_t>((L.M + C::BN - 1) / C::BN) * ((L.N + 127) / 128);
    const int sms = num_sms();
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(tiles < sms ? tiles : sms), 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = L.stream;
    cudaLaunchAttribute attrs[2];
    fill_attrs(cfg, attrs, 1, L.pdl);
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_persistent_swap_kernel<C>, tmX, tmW, tmW2, p);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

// Pair kernel: clusters of 2 CTAs, one 256 x 256 tile per pair at a time.
template <class C> static pgf8_status launch_pair(const GemmLaunch &L)
{
    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        return cudaFuncSetAttribute(gemm_pair_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    CUtensorMap tmX, tmW, tmW2;
    if (!make_operand_maps<C>(L, tmX, tmW, tmW2))
        return PGF8_ERR_UNSUPPORTED;
    const GemmParams p = make_params(L, 1);
    const int64_t tiles = static_cast<int64_t>((L.M + 255) / 256) * ((L.N + C::BN - 1) / C::BN);
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = L.stream;
    cudaLaunchAttribute attrs[2];
    // A persistent grid must not hold more pairs than can run at once (a
    // pair needs two SMs of one GPC): ask the occupancy calculator.
    static PerDeviceSetup fit_setup;
    int pairs_fit = 1;
    const cudaError_t fit_err = setup_once_per_device(fit_setup, [&cfg](int, int *v) {
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3(2 * num_sms(), 1, 1);
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = 2;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        q.attrs = qa;
        q.numAttrs = 1;
        int n = 0;
        const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<C>, &q);
        *v = n > 0 ? n : 1;
        return e;
    }, &pairs_fit);
    if (fit_err != cudaSuccess)
        return cuda_fail(fit_err);
    // Stream-K region (on request, when the workspace holds the partial
    // slots and the tiles do not fill whole rounds): one full round plus the
    // ragged tail, split in equal k-block ranges over every pair.
    PairSK sk;
    std::memset(&sk, 0, sizeof(sk));
    int64_t pairs = tiles < pairs_fit ? tiles : pairs_fit;
    const int64_t sk_pairs = pairs_fit < kPairSKMaxCtas / 2 ? pairs_fit : kPairSKMaxCtas / 2;
    if ((L.opts.flags & PGF8_FLAG_STREAM_K_TAIL) && L.ws != nullptr && L.ws_bytes >= pair_sk_workspace_bytes(C::BN) &&
        tiles % sk_pairs != 0 && L.opts.split_k == 0) {
        const int64_t rounds = tiles / sk_pairs;
        sk.t0 = static_cast<int>((rounds > 1 ? rounds - 1 : 0) * sk_pairs);
        sk.units = (tiles - sk.t0) * p.kblocks;
        sk.flags = static_cast<unsigned *>(L.ws);
        sk.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(L.ws) + kPairSKFlagBytes);
        pairs = sk_pairs < sk.units ? sk_pairs : sk.units;
    }
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    fill_attrs(cfg, attrs, 1, L.pdl, 2);
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel<C>, tmX, tmW, tmW2, p, sk);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

template <int KIND> static pgf8_status launch_pair_bn(const GemmLaunch &L, int bn)
{
    if constexpr (KIND == kNested16) {
        // FP16 mode: 256-wide tiles only (6 stages of 16 KB activations +
        // 16 KB rebuilt weights per CTA)
        if (bn != 256)
            return PGF8_ERR_UNSUPPORTED;
        return launch_pair<PairCfg<256, 6, KIND>>(L);
    } else {
        if (bn == 128)
            return launch_pair<PairCfg<128, 8, KIND>>(L);
        if (bn == 192)
            return launch_pair<PairCfg<192, 7, KIND>>(L);
        return launch_pair<PairCfg<256, 6, KIND>>(L);
    }
}

// Several layers' 256 x 256 tiles in one persistent launch on SM pairs.
static pgf8_status launch_pair_group(const PairGroupParams &gp, cudaStream_t cs)
{
    using C = PairCfg<256, 6, kE4M3>;
    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        return cudaFuncSetAttribute(gemm_pair_group_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = cs;
    // no more pairs than can run at once (a pair needs two SMs of one GPC)
    static PerDeviceSetup fit_setup;
    int pairs_fit = 1;
    const cudaError_t fit_err = setup_once_per_device(fit_setup, [&cfg](int, int *v) {
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3(2 * num_sms(), 1, 1);
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = 2;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        q.attrs = qa;
        q.numAttrs = 1;
        int n = 0;
        const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm_pair_group_kernel<C>, &q);
        *v = n > 0 ? n : 1;
        return e;
    }, &pairs_fit);
    if (fit_err != cudaSuccess)
        return cuda_fail(fit_err);
    const int pairs = gp.total < pairs_fit ? gp.total : pairs_fit;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    cudaLaunchAttribute attrs[2];
    fill_attrs(cfg, attrs, 1, 1, 2);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_pair_group_kernel<C>, gp);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

// Stream-K skinny kernel: one CTA per SM, equal shares of the weight stream.
template <class C> static pgf8_status launch_streamk(const GemmLaunch &L)
{
    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        return cudaFuncSetAttribute(gemm_streamk_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    CUtensorMap tmX, tmW, tmW2;
    if (!make_operand_maps<C>(L, tmX, tmW, tmW2))
        return PGF8_ERR_UNSUPPORTED;
    const GemmParams p = make_params(L, 1);
    StreamKParams q;
    q.units = static_cast<int64_t>((L.N + 127) / 128) * p.kblocks;
    q.flags = static_cast<unsigned *>(L.ws);
    q.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(L.ws) + kStreamKFlagBytes);
    int slots = num_sms() * PGF8_STREAMK_CTAS_PER_SM;
    if (slots > kStreamKMaxCtas)
        slots = kStreamKMaxCtas;
    const int64_t grid = q.units < slots ? q.units : slots;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = L.stream;
    cudaLaunchAttribute attrs[2];
    fill_attrs(cfg, attrs, 1, L.pdl);
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_streamk_kernel<C>, tmX, tmW, tmW2, p, q);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

template <int KIND, bool SWAP, int BN, int STAGES, int XQ = 0>
static pgf8_status launch_split_or_not(const GemmLaunch &L, int splits)
{
    if (splits > 1)
        return launch_cfg<GemmCfg<SWAP, BN, STAGES, KIND, true, XQ>>(L, splits);
    return launch_cfg<GemmCfg<SWAP, BN, STAGES, KIND, false, XQ>>(L, 1);
}

static int num_sms()
{
    static PerDeviceSetup setup;
    int sms = 0;
    setup_once_per_device(setup, [](int dev, int *v) {
        int n = 0;
        const cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        *v = (e == cudaSuccess && n > 0) ? n : 148;
        return cudaSuccess;
    }, &sms);
    return sms > 0 ? sms : 148;
}

// The largest power-of-two split that keeps a skinny grid within ~1.75 CTAs
// per SM (measured on B200 over the 7B and 70B decode shapes: 64 weight
// tiles -> 4, 80-96 -> 2, >= 172 -> 1); beyond that the extra CTAs wait for
// a second wave.
static int skinny_auto_splits(int tiles, int sms)
{
    int splits = 1;
    while (splits < 8 && tiles * splits * 2 * 4 <= sms * PGF8_SKINNY_CTAS_PER_SM_X4)
        splits *= 2;
    return splits;
}

template <int KIND, int BN, int STAGES, int XQ> static pgf8_status launch_xq_cfg(const GemmLaunch &L, int splits)
{
    // two CTAs per SM: 228 KB per SM, 1 KB reserved per CTA, 128 bytes static
    static_assert(GemmCfg<true, BN, STAGES, KIND, true, XQ>::kSmemBytes + 128 + 1024 <= 228 * 1024 / 2,
                  "fused-quantisation configuration exceeds half an SM's shared memory");
    if (splits > 1)
        return launch_cfg<GemmCfg<true, BN, STAGES, KIND, true, XQ>>(L, splits);
    return launch_cfg<GemmCfg<true, BN, STAGES, KIND, false, XQ>>(L, 1);
}

// Split and tile of the skinny GEMM that quantises its activations itself,
// and whether it applies: each CTA holds its whole activation slice (M rows
// x its K-slice) in the registers of 128 threads, at most 4 chunks of 16
// f32 or 8 of 16 f16 per thread.  L.opts.path is AUTO or SKINNY, tile_n 0 /
// 16 / 32 (>= M), split_k 0..8 (checked by the caller).
static bool xq_plan(const GemmLaunch &L, int xq, int &bn, int &splits)
{
    const int kblocks = (L.K + 127) / 128;
    bn = L.opts.tile_n != 0 ? L.opts.tile_n : (L.M <= 16 ? 16 : 32);
    splits = L.opts.split_k != 0 ? L.opts.split_k : skinny_auto_splits((L.N + 127) / 128, num_sms());
    if (splits > kblocks)
        splits = kblocks;
    const int slice_kb = (kblocks + splits - 1) / splits;
    const int64_t chunks = static_cast<int64_t>(L.M) * slice_kb * 8;
    return chunks <= 128 * (xq == 1 ? 4 : 8) && L.M <= PGF8_FUSED_MAX_M && splits <= PGF8_FUSED_MAX_SPLITS;
}

// Whether a dynamic call with these (checked) arguments quantises inside the
// GEMM, and with which tile width and split.
static bool fused_quant_plan(int64_t M, int64_t N, int64_t K, pgf8_dtype xdt, const pgf8_linear_opts &o, int &bn,
                             int &splits)
{
    const bool eligible = (o.flags & PGF8_FLAG_FUSED_QUANT) && M <= 32 &&
                          (o.path == PGF8_PATH_AUTO || o.path == PGF8_PATH_SKINNY) &&
                          (o.tile_n == 0 || ((o.tile_n == 16 || o.tile_n == 32) && o.tile_n >= M)) &&
                          o.split_k >= 0 && o.split_k <= 8;
    if (!eligible)
        return false;
    GemmLaunch P;
    P.M = static_cast<int>(M);
    P.N = static_cast<int>(N);
    P.K = static_cast<int>(K);
    P.opts = o;
    return xq_plan(P, xdt == PGF8_F32 ? 1 : 2, bn, splits);
}

template <int KIND, int XQ> static pgf8_status launch_gemm_xq(const GemmLaunch &L, int bn, int splits)
{
    // the skinny kernel's stage counts (both fit two CTAs per SM)
    if (bn == 16)
        return launch_xq_cfg<KIND, 16, 6, XQ>(L, splits);
    return launch_xq_cfg<KIND, 32, 5, XQ>(L, splits);
}

template <int KIND> static pgf8_status launch_gemm(const GemmLaunch &L)
{
    // argument checks first: nothing below may touch the device before they pass
    const int elem = (KIND == kNested16) ? 2 : 1;
    const int kblocks = static_cast<int>((static_cast<int64_t>(L.K) * elem + 127) / 128);
    int path = L.opts.path;
    int bn = L.opts.tile_n;
    int splits = L.opts.split_k;
    const int sk_bn = L.M <= 16 ? 16 : 32;
    const bool sk_ws = L.M <= 32 && L.ws != nullptr && L.ws_bytes >= streamk_workspace_bytes(sk_bn);
    // AUTO never picks stream-K: on B200 the cluster split-K kernel streams
    // the decode shapes faster (its partial tiles stay in distributed shared
    // memory instead of a global fix-up); stream-K is selected explicitly.
    if (path == PGF8_PATH_AUTO)
        path = (L.M <= 128) ? PGF8_PATH_SKINNY : PGF8_PATH_TILED;
    if (path == PGF8_PATH_STREAMK) {
        if (L.M > 32)
            return PGF8_ERR_UNSUPPORTED;
        if (!sk_ws)
            return PGF8_ERR_INVALID_ARG;
        if (sk_bn == 16)
            return launch_streamk<StreamKCfg<16, PGF8_STREAMK16_STAGES, KIND>>(L);
        return launch_streamk<StreamKCfg<32, 5, KIND>>(L);
    }
    if (path == PGF8_PATH_TILED_PAIR) {
        if (bn != 0 && bn != 128 && bn != 192 && bn != 256)
            return PGF8_ERR_INVALID_ARG;
        return launch_pair_bn<KIND>(L, bn == 0 ? 256 : bn);
    }
    if (path != PGF8_PATH_SKINNY && path != PGF8_PATH_TILED)
        return PGF8_ERR_INVALID_ARG;
    if (splits < 0 || splits > 8)
        return PGF8_ERR_INVALID_ARG;
    if (path == PGF8_PATH_SKINNY) {
        if (L.M > 128)
            return PGF8_ERR_UNSUPPORTED;
        if (bn == 0)
            bn = L.M <= 16 ? 16 : L.M <= 32 ? 32 : L.M <= 64 ? 64 : 128;
        if (bn < L.M || (bn != 16 && bn != 32 && bn != 64 && bn != 128))
            return PGF8_ERR_INVALID_ARG;
    } else if (bn != 0 && bn != 128 && bn != 256) {
        return PGF8_ERR_INVALID_ARG;
    }

    const int sms = (splits == 0 || bn == 0) ? num_sms() : 148;
    if (path == PGF8_PATH_SKINNY) {
        const int tiles = (L.N + 127) / 128;
        if (splits == 0)
            splits = skinny_auto_splits(tiles, sms);
        if (splits > kblocks)
            splits = kblocks;
        switch (bn) {
        case 16: return launch_split_or_not<KIND, true, 16, PGF8_SKINNY16_STAGES>(L, splits);
        case 32: return launch_split_or_not<KIND, true, 32, 8>(L, splits);
        case 64: return launch_split_or_not<KIND, true, 64, 8>(L, splits);
        default: return launch_split_or_not<KIND, true, 128, 6>(L, splits);
        }
    }
    // FP8 operands with at least about half a round of 256 x 256 tiles (74
    // SM pairs): the pair kernel.  Measured on B200 over every tiled 7B /
    // 70B shape (M = 256 .. 4096): with 40 or more tiles it is the fastest or
    // within 3 %; with 32 tiles the one-CTA persistent kernel below is
    // faster (more SMs busy on 128-row tiles).
    // NestedFP FP16 mode, automatic choice, M > 256 with at least 96 tiles
    // of 128 weight rows x 256 tokens: the one-CTA kernel with the rebuilt
    // weights as the 128-row operand (less shared-memory traffic per
    // k-step).  Measured on B200 over the 7B / 70B shapes at M = 512 ..
    // 4096: 20-28 % faster from M = 1024 on (7B QKV at M = 1024: 891 against
    // 735 TFLOP/s), slower only with 64 tiles (7B down at M = 512: 103
    // against 81 us).  (The SM-pair form measured 1.6-1.8x slower at every
    // shape; it stays selectable through PGF8_PATH_TILED_PAIR, the
    // tokens-as-A kernel through path / tile_n.)
    if constexpr (KIND == kNested16) {
        const int64_t swap_tiles = static_cast<int64_t>((L.M + 255) / 256) * ((L.N + 127) / 128);
        if (L.opts.path == PGF8_PATH_AUTO && bn == 0 && splits == 0 && L.M > 256 && swap_tiles >= 96)
            return launch_persistent_swap<PersistSwapCfg<256, 4>>(L);
    } else {
        const int64_t tiles_pair = static_cast<int64_t>((L.M + 255) / 256) * ((L.N + 255) / 256);
        // (the 192 / 128 widths fill the last round better but measured slower
        // per tile than 256 on nearly every 7B / 70B shape; they stay
        // selectable through tile_n)
        if (L.opts.path == PGF8_PATH_AUTO && bn == 0 && splits == 0 && tiles_pair >= 40)
            return launch_pair_bn<KIND>(L, 256);
    }
    const int mt = (L.M + 127) / 128;
    // fraction of the CTA slots the last wave of a persistent launch keeps busy
    auto wave_eff = [&](int b) {
        const int64_t t = static_cast<int64_t>(mt) * ((L.N + b - 1) / b);
        const int64_t waves = (t + sms - 1) / sms;
        return static_cast<double>(t) / static_cast<double>(waves * sms);
    };
    // Tile choice (measured on B200 over the 7B prefill shapes): 128 x 256
    // tiles in the persistent kernel whenever they give at least half a wave;
    // with fewer tiles, a two-way cluster split of K for long K, else the
    // narrower 128 x 128 tile.
    const int64_t tiles256 = static_cast<int64_t>(mt) * ((L.N + 255) / 256);
    const bool few = tiles256 * 2 < sms;
    if (bn == 0)
        bn = (few && kblocks < 64) ? 128 : (wave_eff(128) > wave_eff(256) + 0.15 ? 128 : 256);
    if (splits == 0)
        splits = (few && bn == 256) ? 2 : 1;
    if (splits > kblocks)
        splits = kblocks;
    if (splits == 1) {
        if (bn == 256)
            return launch_persistent<PersistCfg<256, 4, KIND>>(L);
        return launch_persistent<PersistCfg<128, 6, KIND>>(L);
    }
    if (bn == 256)
        return launch_split_or_not<KIND, false, 256, 4>(L, splits);
    return launch_split_or_not<KIND, false, 128, 6>(L, splits);
}

static pgf8_status check_dims(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 16 || K < 16 || M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30))
        return PGF8_ERR_INVALID_ARG;
    if (K % 16 != 0 || N % 16 != 0)
        return PGF8_ERR_ALIGNMENT;
    return PGF8_OK;
}

static pgf8_linear_opts opts_or_default(const pgf8_linear_opts *o)
{
    pgf8_linear_opts d;
    std::memset(&d, 0, sizeof(d));
    if (o)
        d = *o;
    return d;
}

static pgf8_status quantize_launch(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                   uint8_t *q, float *scales, int mode, cudaStream_t st, int pdl,
                                   int trigger_early)
{
    const int qflags = trigger_early ? kQuantTriggerEarly : 0;
    if (rows == 0)
        return PGF8_OK;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    // rows held in registers by the smallest CTA footprint that fits them
    // (1, 2 or 4 chunks of 16 per thread of 256); longer rows take the
    // two-pass kernel (measured faster at 28672 than a 512-thread CTA
    // holding the row)
    const int64_t nchunk = cols / 16;
    cudaError_t e;
    auto launch = [&](auto kern, unsigned threads, auto xp) {
        cfg.blockDim = dim3(threads);
        return cudaLaunchKernelEx(&cfg, kern, xp, rows, cols, ldx, q, scales, mode, qflags);
    };
    const float *xf = static_cast<const float *>(x);
    const __half *xh = static_cast<const __half *>(x);
    if (xdt == PGF8_F32) {
        if (nchunk <= 256)
            e = launch(quantize_rows_held_kernel<float, 1, 256>, 256, xf);
        else if (nchunk <= 512)
            e = launch(quantize_rows_held_kernel<float, 2, 256>, 256, xf);
        else if (nchunk <= 1024)
            e = launch(quantize_rows_held_kernel<float, 4, 256>, 256, xf);
        else
            e = launch(quantize_rows_kernel<float>, kQuantThreads, xf);
    } else {
        if (nchunk <= 256)
            e = launch(quantize_rows_held_kernel<__half, 1, 256>, 256, xh);
        else if (nchunk <= 512)
            e = launch(quantize_rows_held_kernel<__half, 2, 256>, 256, xh);
        else if (nchunk <= 1024)
            e = launch(quantize_rows_held_kernel<__half, 4, 256>, 256, xh);
        else
            e = launch(quantize_rows_kernel<__half>, kQuantThreads, xh);
    }
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

static pgf8_status check_quantize_args(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                       const uint8_t *q, const float *scales, int mode)
{
    if (rows < 0 || cols < 16 || ldx < cols || rows > (1ll << 31) - 1)
        return PGF8_ERR_INVALID_ARG;
    if (rows == 0)
        return PGF8_OK;   // nothing to read or write; pointers may be null
    if (!x || !q || !scales)
        return PGF8_ERR_INVALID_ARG;
    if (xdt != PGF8_F32 && xdt != PGF8_F16)
        return PGF8_ERR_UNSUPPORTED;
    if (mode != PGF8_SCALE_DYNAMIC && mode != PGF8_SCALE_STATIC)
        return PGF8_ERR_INVALID_ARG;
    const int eb = xdt == PGF8_F32 ? 4 : 2;
    if (cols % 16 != 0 || (ldx * eb) % 16 != 0 || !aligned16(x) || !aligned16(q) || !aligned4(scales))
        return PGF8_ERR_ALIGNMENT;
    return PGF8_OK;
}

// Checks of the per-tensor scaling calls: x and (when given) q as for the
// per-row quantisation; scales may be null.
static pgf8_status check_tensor_args(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                     const uint8_t *q, bool need_q, const float *scales)
{
    if (rows < 0 || cols < 16 || ldx < cols || rows > (1ll << 31) - 1)
        return PGF8_ERR_INVALID_ARG;
    if (rows == 0)
        return PGF8_OK;
    if (!x || (need_q && !q))
        return PGF8_ERR_INVALID_ARG;
    if (xdt != PGF8_F32 && xdt != PGF8_F16)
        return PGF8_ERR_UNSUPPORTED;
    const int eb = xdt == PGF8_F32 ? 4 : 2;
    if (cols % 16 != 0 || (ldx * eb) % 16 != 0 || !aligned16(x) || (q && !aligned16(q)) ||
        (scales && !aligned4(scales)))
        return PGF8_ERR_ALIGNMENT;
    return PGF8_OK;
}

// Launches a kernel, optionally with programmatic stream serialization
// (the kernel waits on the grid dependency before its first read).
template <typename... Args>
static pgf8_status launch_grid(void (*kernel)(Args...), dim3 grid, dim3 block, cudaStream_t st, int pdl,
                               Args... args)
{
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    return e == cudaSuccess ? PGF8_OK : cuda_fail(e);
}

// A 256-thread quantisation-family kernel on a 1-D grid.
template <typename... Args>
static pgf8_status launch_quant(void (*kernel)(Args...), unsigned grid, cudaStream_t st, int pdl, Args... args)
{
    return launch_grid(kernel, dim3(grid), dim3(kQuantThreads), st, pdl, args...);
}

// ------------------------------------------------------------------ decode attention plan
// Query heads per CTA: the largest of 8, 4, 2, 1 that divides the group
// size Hq / Hkv (the heads of one CTA share every K / V load).
static int attn_heads_per_cta(int64_t G)
{
    for (int gt = 8; gt > 1; gt >>= 1)
        if (G % gt == 0)
            return gt;
    return 1;
}

constexpr int64_t kAttnCtasPerSm = 4;     // CTAs per SM the automatic split aims for
constexpr int64_t kAttnMinChunk = 256;    // positions per split at least (automatic split)

struct AttnPlan {
    int64_t nsplit, chunk;
    int gt, groups;
};

// Splits the context [0, max_ctx) into nsplit chunks of `chunk` positions.
// Automatic (splits == 0): enough chunks for ~kAttnCtasPerSm CTAs per SM,
// no chunk under kAttnMinChunk positions, chunks a multiple of 64 (whole
// 16-position steps for each of the 4 warps).  Forced: at most `splits`
// chunks, a multiple of 16 positions.
static AttnPlan attn_plan(int64_t seqs, int64_t Hq, int64_t Hkv, int64_t max_ctx, int64_t splits)
{
    AttnPlan p;
    p.gt = attn_heads_per_cta(Hq / Hkv);
    p.groups = static_cast<int>(Hq / Hkv / p.gt);
    if (max_ctx <= kAttnStep) {
        p.nsplit = 1;
        p.chunk = kAttnStep;
        return p;
    }
    int64_t ns;
    if (splits > 0) {
        const int64_t steps = (max_ctx + kAttnStep - 1) / kAttnStep;
        ns = splits < steps ? splits : steps;
    } else {
        const int64_t ctas = seqs * Hkv * p.groups;
        const int64_t target = static_cast<int64_t>(num_sms()) * kAttnCtasPerSm;
        const int64_t cap = max_ctx / kAttnMinChunk;   // every chunk >= kAttnMinChunk positions
        ns = (target + ctas - 1) / ctas;
        if (ns > cap)
            ns = cap;
        if (ns < 1)
            ns = 1;
    }
    const int64_t gran = splits > 0 ? kAttnStep : kAttnStep * kAttnWarps;
    const int64_t per = (max_ctx + ns - 1) / ns;
    p.chunk = (per + gran - 1) / gran * gran;
    p.nsplit = (max_ctx + p.chunk - 1) / p.chunk;
    return p;
}

static size_t attn_workspace_bytes(int64_t seqs, int64_t Hq, int64_t D, const AttnPlan &p)
{
    return p.nsplit > 1 ? static_cast<size_t>(seqs * Hq * p.nsplit * (D + 2)) * sizeof(float) : 0;
}

static bool attn_shape_ok(int64_t seqs, int64_t Hq, int64_t Hkv, int64_t D, int64_t max_ctx)
{
    return seqs >= 0 && seqs <= 65535 && Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0 && Hq <= 65535 &&
           (D == 64 || D == 128 || D == 256) && max_ctx >= 0 && max_ctx <= (1ll << 30);
}

template <int D, int GT>
static pgf8_status launch_attn_gt(const AttnDecodeArgs &a, int64_t seqs, cudaStream_t st, int pdl)
{
    const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(a.Hkv * a.groups),
                    static_cast<unsigned>(seqs));
    return launch_grid(attn_decode_paged_kernel<D, GT>, grid, dim3(kAttnThreads), st, pdl, a);
}

template <int D>
static pgf8_status launch_attn(const AttnDecodeArgs &a, int gt, bool mma, int64_t seqs, cudaStream_t st, int pdl)
{
    pgf8_status r;
    if (mma) {
        // up to 8 query heads of one KV head per CTA: the MMA's N dimension
        AttnDecodeArgs am = a;
        am.groups = static_cast<int>((a.Hq / a.Hkv + 7) / 8);
        const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(a.Hkv * am.groups),
                        static_cast<unsigned>(seqs));
        r = launch_grid(attn_decode_mma_kernel<D>, grid, dim3(kAttnThreads), st, pdl, am);
    } else {
        switch (gt) {
        case 8: r = launch_attn_gt<D, 8>(a, seqs, st, pdl); break;
        case 4: r = launch_attn_gt<D, 4>(a, seqs, st, pdl); break;
        case 2: r = launch_attn_gt<D, 2>(a, seqs, st, pdl); break;
        default: r = launch_attn_gt<D, 1>(a, seqs, st, pdl); break;
        }
    }
    if (r != PGF8_OK || a.nsplit == 1)
        return r;
    // the merge overlaps the chunk kernel's tail and waits for its results
    return launch_grid(attn_decode_combine_kernel<D>, dim3(static_cast<unsigned>(seqs * a.Hq)), dim3(D), st, 1,
                       static_cast<const float *>(a.part), a.nsplit, a.Hq, a.Hkv, a.sv, a.out, a.ldo, a.odt);
}

} // namespace pgf8

using namespace pgf8;

extern "C" {

pgf8_status pgf8_fp8_amax_accumulate(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                     float *amax, void *stream)
{
    pgf8_status st = check_tensor_args(x, xdt, rows, cols, ldx, nullptr, false, nullptr);
    if (st != PGF8_OK)
        return st;
    if (!amax)
        return PGF8_ERR_INVALID_ARG;
    if (!aligned4(amax))
        return PGF8_ERR_ALIGNMENT;
    if (rows == 0)
        return PGF8_OK;
    const int64_t chunks = rows * (cols / 16);
    const int64_t want = (chunks + kQuantThreads - 1) / kQuantThreads;
    const unsigned grid = static_cast<unsigned>(want < num_sms() * 4 ? want : num_sms() * 4);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    unsigned *bits = reinterpret_cast<unsigned *>(amax);
    if (xdt == PGF8_F32)
        return launch_quant(amax_accumulate_kernel<float>, grid, cs, 0, static_cast<const float *>(x), rows, cols,
                            ldx, bits);
    return launch_quant(amax_accumulate_kernel<__half>, grid, cs, 0, static_cast<const __half *>(x), rows, cols, ldx,
                        bits);
}

pgf8_status pgf8_fp8_quantize_tensor(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                     const float *amax, uint8_t *q, float *scales, int32_t flags, void *stream)
{
    pgf8_status st = check_tensor_args(x, xdt, rows, cols, ldx, q, true, scales);
    if (st != PGF8_OK)
        return st;
    if (rows == 0)
        return PGF8_OK;
    if (!amax)
        return PGF8_ERR_INVALID_ARG;
    if (!aligned4(amax))
        return PGF8_ERR_ALIGNMENT;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>(rows);
    const int pdl = (flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    if (xdt == PGF8_F32)
        return launch_quant(quantize_tensor_kernel<float>, grid, cs, pdl, static_cast<const float *>(x), cols, ldx,
                            amax, q, scales);
    return launch_quant(quantize_tensor_kernel<__half>, grid, cs, pdl, static_cast<const __half *>(x), cols, ldx,
                        amax, q, scales);
}

pgf8_status pgf8_delayed_state_init(pgf8_delayed_state *state, float *history, int32_t history_len,
                                    float initial_scale, void *stream)
{
    if (!state || !history || history_len < 1 || history_len > (1 << 24) || !(initial_scale > 0.0f) ||
        !std::isfinite(initial_scale))
        return PGF8_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(state) & 15u) != 0 || !aligned4(history))
        return PGF8_ERR_ALIGNMENT;
    const unsigned grid = static_cast<unsigned>((history_len + kQuantThreads - 1) / kQuantThreads);
    return launch_quant(delayed_init_kernel, grid < 1024u ? grid : 1024u, static_cast<cudaStream_t>(stream), 0,
                        history, static_cast<int>(history_len), reinterpret_cast<DelayedState *>(state),
                        initial_scale);
}

pgf8_status pgf8_fp8_quantize_delayed(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                      uint8_t *q, float *scales, float *history, int32_t history_len,
                                      pgf8_delayed_state *state, int64_t step, int32_t flags, void *stream)
{
    pgf8_status st = check_tensor_args(x, xdt, rows, cols, ldx, q, true, scales);
    if (st != PGF8_OK)
        return st;
    if (!state || !history || history_len < 1 || history_len > (1 << 24) || step < 0)
        return PGF8_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(state) & 15u) != 0 || !aligned4(history))
        return PGF8_ERR_ALIGNMENT;
    if (rows == 0)
        return PGF8_ERR_INVALID_ARG;   // a step needs its amax: at least one row
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>(rows);
    DelayedState *ds = reinterpret_cast<DelayedState *>(state);
    const int pdl = (flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    if (xdt == PGF8_F32)
        return launch_quant(quantize_delayed_kernel<float>, grid, cs, pdl, static_cast<const float *>(x), cols, ldx,
                            q, scales, history, static_cast<int>(history_len), ds, step);
    return launch_quant(quantize_delayed_kernel<__half>, grid, cs, pdl, static_cast<const __half *>(x), cols, ldx, q,
                        scales, history, static_cast<int>(history_len), ds, step);
}

pgf8_status pgf8_fp8_norm_quantize(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                   const float *gamma, const float *beta, float eps, uint8_t *q, float *scales,
                                   int32_t flags, void *stream)
{
    pgf8_status st = check_quantize_args(x, xdt, rows, cols, ldx, q, scales, PGF8_SCALE_DYNAMIC);
    if (st != PGF8_OK)
        return st;
    if (rows == 0)
        return PGF8_OK;
    if (!gamma || !(eps >= 0.0f) || !std::isfinite(eps))
        return PGF8_ERR_INVALID_ARG;
    if (!aligned4(gamma) || (beta && !aligned4(beta)))
        return PGF8_ERR_ALIGNMENT;
    if (cols > static_cast<int64_t>(kRegChunks) * kQuantThreads * 16)
        return PGF8_ERR_UNSUPPORTED;   // the row is held in registers
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int pdl = (flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    const unsigned grid = static_cast<unsigned>(rows);
    if (xdt == PGF8_F32)
        return launch_quant(norm_quantize_kernel<float>, grid, cs, pdl, static_cast<const float *>(x), cols, ldx,
                            gamma, beta, eps, q, scales);
    return launch_quant(norm_quantize_kernel<__half>, grid, cs, pdl, static_cast<const __half *>(x), cols, ldx,
                        gamma, beta, eps, q, scales);
}

pgf8_status pgf8_fp8_silu_mul_quantize(const void *gu, pgf8_dtype gdt, int64_t rows, int64_t inter, int64_t ldg,
                                       uint8_t *q, float *scales, int32_t flags, void *stream)
{
    if (rows < 0 || inter < 16 || ldg < 2 * inter || rows > (1ll << 31) - 1)
        return PGF8_ERR_INVALID_ARG;
    if (rows == 0)
        return PGF8_OK;
    if (!gu || !q || !scales)
        return PGF8_ERR_INVALID_ARG;
    if (gdt != PGF8_BF16 && gdt != PGF8_F32)
        return PGF8_ERR_UNSUPPORTED;
    const int eb = gdt == PGF8_F32 ? 4 : 2;
    if (inter % 16 != 0 || (ldg * eb) % 16 != 0 || !aligned16(gu) || !aligned16(q) || !aligned4(scales))
        return PGF8_ERR_ALIGNMENT;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int pdl = (flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    const unsigned grid = static_cast<unsigned>(rows);
    if (gdt == PGF8_F32)
        return launch_quant(silu_mul_quantize_kernel<float>, grid, cs, pdl, static_cast<const float *>(gu), inter,
                            ldg, q, scales);
    return launch_quant(silu_mul_quantize_kernel<__nv_bfloat16>, grid, cs, pdl,
                        static_cast<const __nv_bfloat16 *>(gu), inter, ldg, q, scales);
}

pgf8_status pgf8_fp8_kv_write_paged(const void *kv, pgf8_dtype dt, int64_t tokens, int64_t heads, int64_t head_dim,
                                    int64_t ldkv, const float *scales, int64_t first_pos, int64_t block_size,
                                    const int32_t *block_table, int64_t table_len, int64_t num_blocks,
                                    uint8_t *cache, int32_t *bad_blocks, int32_t flags, void *stream)
{
    if (tokens < 0 || heads < 1 || head_dim < 16 || block_size < 1 || first_pos < 0 || num_blocks < 1 ||
        table_len < 1 || ldkv < heads * head_dim || tokens > (1ll << 40))
        return PGF8_ERR_INVALID_ARG;
    if (tokens == 0)
        return PGF8_OK;
    if (!kv || !scales || !block_table || !cache)
        return PGF8_ERR_INVALID_ARG;
    if ((first_pos + tokens - 1) / block_size >= table_len)
        return PGF8_ERR_INVALID_ARG;   // positions beyond the block table
    if (dt != PGF8_F32 && dt != PGF8_F16 && dt != PGF8_BF16)
        return PGF8_ERR_UNSUPPORTED;
    const int eb = dt == PGF8_F32 ? 4 : 2;
    if (head_dim % 16 != 0 || (ldkv * eb) % 16 != 0 || !aligned16(kv) || !aligned16(cache) || !aligned4(scales) ||
        !aligned4(block_table) || (bad_blocks && !aligned4(bad_blocks)))
        return PGF8_ERR_ALIGNMENT;
    const int64_t items = tokens * heads * (head_dim / 16);
    const int64_t want = (items + kQuantThreads - 1) / kQuantThreads;
    const unsigned grid = static_cast<unsigned>(want < num_sms() * 8 ? want : num_sms() * 8);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int pdl = (flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    if (dt == PGF8_F32)
        return launch_quant(kv_write_paged_kernel<float>, grid, cs, pdl, static_cast<const float *>(kv), tokens,
                            heads, head_dim, ldkv, scales, first_pos, block_size, block_table, num_blocks, cache,
                            bad_blocks);
    if (dt == PGF8_F16)
        return launch_quant(kv_write_paged_kernel<__half>, grid, cs, pdl, static_cast<const __half *>(kv), tokens,
                            heads, head_dim, ldkv, scales, first_pos, block_size, block_table, num_blocks, cache,
                            bad_blocks);
    return launch_quant(kv_write_paged_kernel<__nv_bfloat16>, grid, cs, pdl, static_cast<const __nv_bfloat16 *>(kv),
                        tokens, heads, head_dim, ldkv, scales, first_pos, block_size, block_table, num_blocks, cache,
                        bad_blocks);
}

pgf8_status pgf8_fp8_attention_decode_plan(int64_t seqs, int64_t q_heads, int64_t kv_heads, int64_t head_dim,
                                           int64_t max_context, int64_t splits, int64_t *nsplit, int64_t *chunk)
{
    if (!attn_shape_ok(seqs, q_heads, kv_heads, head_dim, max_context) || splits < 0)
        return PGF8_ERR_INVALID_ARG;
    const AttnPlan p = attn_plan(seqs, q_heads, kv_heads, max_context, splits);
    if (nsplit)
        *nsplit = p.nsplit;
    if (chunk)
        *chunk = p.chunk;
    return PGF8_OK;
}

size_t pgf8_fp8_attention_decode_workspace_size(int64_t seqs, int64_t q_heads, int64_t kv_heads, int64_t head_dim,
                                                int64_t max_context, int64_t splits)
{
    if (!attn_shape_ok(seqs, q_heads, kv_heads, head_dim, max_context) || splits < 0)
        return 0;
    return attn_workspace_bytes(seqs, q_heads, head_dim, attn_plan(seqs, q_heads, kv_heads, max_context, splits));
}

pgf8_status pgf8_fp8_attention_decode_paged(const void *q, pgf8_dtype q_dt, int64_t seqs, int64_t q_heads,
                                            int64_t ldq, const pgf8_paged_kv_cache *cache,
                                            const int32_t *block_tables, int64_t table_stride,
                                            const int32_t *context_lens, int64_t max_context, void *out,
                                            pgf8_dtype out_dt, int64_t ldo, int64_t splits, void *workspace,
                                            size_t workspace_bytes, int32_t *errors, int32_t flags, void *stream)
{
    if (!cache)
        return PGF8_ERR_INVALID_ARG;
    const int64_t Hkv = cache->kv_heads, D = cache->head_dim, B = cache->block_size;
    if (!attn_shape_ok(seqs, q_heads, Hkv, D, max_context) || splits < 0 || cache->num_blocks < 1 || B < 16 ||
        B % 16 != 0 || ldq < q_heads * D || ldo < q_heads * D || table_stride < 1 ||
        max_context > table_stride * B || seqs * q_heads > 0x7fffffffll)
        return PGF8_ERR_INVALID_ARG;
    if (seqs == 0)
        return PGF8_OK;
    if (!q || !out || !cache->k_cache || !cache->v_cache || !cache->k_scales || !cache->v_scales || !block_tables ||
        !context_lens)
        return PGF8_ERR_INVALID_ARG;
    const bool qok = q_dt == PGF8_F32 || q_dt == PGF8_F16 || q_dt == PGF8_BF16;
    const bool ook = out_dt == PGF8_F32 || out_dt == PGF8_F16 || out_dt == PGF8_BF16;
    if (!qok || !ook)
        return PGF8_ERR_UNSUPPORTED;
    const uintptr_t qa = q_dt == PGF8_F32 ? 3u : 1u, oa = out_dt == PGF8_F32 ? 3u : 1u;
    if (!aligned16(cache->k_cache) || !aligned16(cache->v_cache) || !aligned4(cache->k_scales) ||
        !aligned4(cache->v_scales) || !aligned4(block_tables) || !aligned4(context_lens) ||
        (errors && !aligned4(errors)) || (reinterpret_cast<uintptr_t>(q) & qa) ||
        (reinterpret_cast<uintptr_t>(out) & oa))
        return PGF8_ERR_ALIGNMENT;
    const AttnPlan p = attn_plan(seqs, q_heads, Hkv, max_context, splits);
    const size_t need = attn_workspace_bytes(seqs, q_heads, D, p);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return PGF8_ERR_INVALID_ARG;
    if (need > 0 && !aligned4(workspace))
        return PGF8_ERR_ALIGNMENT;

    AttnDecodeArgs a;
    a.q = q;
    a.ldq = ldq;
    a.qdt = static_cast<int>(q_dt);
    a.kc = cache->k_cache;
    a.vc = cache->v_cache;
    a.sk = cache->k_scales;
    a.sv = cache->v_scales;
    a.tables = block_tables;
    a.table_stride = table_stride;
    a.ctx_lens = context_lens;
    a.num_blocks = cache->num_blocks;
    a.Hkv = Hkv;
    a.Hq = q_heads;
    a.B = B;
    a.max_ctx = max_context;
    a.chunk = p.chunk;
    a.nsplit = static_cast<int>(p.nsplit);
    a.groups = p.groups;
    a.qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));   // log2(e) / sqrt(D)
    a.out = out;
    a.ldo = ldo;
    a.odt = static_cast<int>(out_dt);
    a.part = static_cast<float *>(workspace);
    a.errors = errors;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int pdl = (flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    const bool mma = (flags & PGF8_FLAG_ATTN_MMA) != 0;
    if (D == 64)
        return launch_attn<64>(a, p.gt, mma, seqs, cs, pdl);
    if (D == 128)
        return launch_attn<128>(a, p.gt, mma, seqs, cs, pdl);
    return launch_attn<256>(a, p.gt, mma, seqs, cs, pdl);
}

pgf8_status pgf8_fp8_attention_context_paged(const uint8_t *q_codes, const float *q_scales,
                                             const int32_t *q_start, int64_t seqs, int64_t total_q,
                                             int64_t max_q_len, int64_t q_heads, const pgf8_paged_kv_cache *cache,
                                             const int32_t *block_tables, int64_t table_stride,
                                             const int32_t *context_lens, int64_t max_context, void *out,
                                             pgf8_dtype out_dt, int64_t ldo, int32_t *errors, void *stream)
{
    if (!cache)
        return PGF8_ERR_INVALID_ARG;
    const int64_t Hkv = cache->kv_heads, D = cache->head_dim, B = cache->block_size;
    if (seqs < 0 || seqs > 65535 || total_q < 0 || total_q >= (1ll << 31) || max_q_len < 0 ||
        max_q_len >= (1ll << 31) || (max_q_len + 127) / 128 * q_heads >= (1ll << 31) || Hkv < 1 ||
        q_heads < Hkv || q_heads % Hkv != 0 || q_heads > 65535 || B < 16 || B % 16 != 0 || cache->num_blocks < 1 ||
        max_context < 0 || table_stride < 1 || max_context > table_stride * B || max_context >= (1ll << 31) ||
        ldo < q_heads * 128 || cache->num_blocks * Hkv * B >= (1ll << 31) - 1)
        return PGF8_ERR_INVALID_ARG;
    if (D != 128)
        return PGF8_ERR_UNSUPPORTED;
    if (seqs == 0 || total_q == 0 || max_q_len == 0)
        return PGF8_OK;
    if (!q_codes || !q_scales || !q_start || !out || !cache->k_cache || !cache->v_cache || !cache->k_scales ||
        !cache->v_scales || !block_tables || !context_lens)
        return PGF8_ERR_INVALID_ARG;
    if (out_dt != PGF8_F32 && out_dt != PGF8_F16 && out_dt != PGF8_BF16)
        return PGF8_ERR_UNSUPPORTED;
    const uintptr_t oa = out_dt == PGF8_F32 ? 3u : 1u;
    if (!aligned16(q_codes) || !aligned16(cache->k_cache) || !aligned16(cache->v_cache) || !aligned4(q_scales) ||
        !aligned4(q_start) || !aligned4(cache->k_scales) || !aligned4(cache->v_scales) || !aligned4(block_tables) ||
        !aligned4(context_lens) || (errors && !aligned4(errors)) || (reinterpret_cast<uintptr_t>(out) & oa))
        return PGF8_ERR_ALIGNMENT;

    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        return cudaFuncSetAttribute(attn_context_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCtxSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    const uint64_t cache_rows = static_cast<uint64_t>(cache->num_blocks * Hkv * B);
    CUtensorMap tmQ, tmK, tmV;
    if (!make_map(&tmQ, q_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(total_q),
                  static_cast<uint64_t>(q_heads * 128), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmK, cache->k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache_rows, 128, 128, 16,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tmV, cache->v_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache_rows, 128, 128, 16,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return PGF8_ERR_UNSUPPORTED;

    AttnCtxParams a;
    a.q_scales = q_scales;
    a.q_start = q_start;
    a.ctx_lens = context_lens;
    a.tables = block_tables;
    a.table_stride = table_stride;
    a.sk = cache->k_scales;
    a.sv = cache->v_scales;
    a.Hq = static_cast<int>(q_heads);
    a.Hkv = static_cast<int>(Hkv);
    a.B = static_cast<int>(B);
    a.num_blocks = cache->num_blocks;
    a.cache_rows = static_cast<int>(cache_rows);
    a.max_ctx = static_cast<int>(max_context);
    a.total_q = static_cast<int>(total_q);
    a.out = out;
    a.ldo = ldo;
    a.odt = static_cast<int>(out_dt);
    a.vec_out = aligned16(out) && (ldo * (out_dt == PGF8_F32 ? 4 : 2)) % 16 == 0;
    a.errors = errors;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>((max_q_len + 127) / 128 * q_heads), 1, static_cast<unsigned>(seqs));
    cfg.blockDim = dim3(kCtxThreads);
    cfg.dynamicSmemBytes = kCtxSmemBytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_context_kernel, tmQ, tmK, tmV, a);
    return e == cudaSuccess ? PGF8_OK : cuda_fail(e);
}

pgf8_status pgf8_fp8_quantize_rows(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                   uint8_t *q, float *scales, pgf8_scale_mode mode, void *stream)
{
    pgf8_status st = check_quantize_args(x, xdt, rows, cols, ldx, q, scales, mode);
    if (st != PGF8_OK)
        return st;
    // a plain launch that signals no early trigger: a following kernel that
    // may overlap its predecessor (e.g. a GEMM reading these codes as weights)
    // cannot start before this one has finished
    return quantize_launch(x, xdt, rows, cols, ldx, q, scales, static_cast<int>(mode),
                           static_cast<cudaStream_t>(stream), 0, 0);
}

pgf8_status pgf8_fp8_row_amax(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx, float *amax,
                              void *stream)
{
    pgf8_status st = check_tensor_args(x, xdt, rows, cols, ldx, nullptr, false, amax);
    if (st != PGF8_OK)
        return st;
    if (rows > 0 && !amax)
        return PGF8_ERR_INVALID_ARG;
    return quantize_launch(x, xdt, rows, cols, ldx, nullptr, amax, kQuantAmaxOnly, static_cast<cudaStream_t>(stream),
                           0, 0);
}

pgf8_status pgf8_fp8_quantize_rows_amax(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                        uint8_t *q, float *amax_scales, void *stream)
{
    pgf8_status st = check_quantize_args(x, xdt, rows, cols, ldx, q, amax_scales, PGF8_SCALE_DYNAMIC);
    if (st != PGF8_OK)
        return st;
    return quantize_launch(x, xdt, rows, cols, ldx, q, amax_scales, kQuantFromAmax,
                           static_cast<cudaStream_t>(stream), 0, 0);
}

static size_t streamk_bytes_for(int64_t M) { return M >= 1 && M <= 32 ? streamk_workspace_bytes(M <= 16 ? 16 : 32) : 0; }

// Workspace of an FP8 linear call: the stream-K region of the kernel the
// call takes (flag words at offset 0 in every layout): skinny stream-K slots
// for M <= 32, the pair kernel's partial slots for M > 128.
static_assert(kPairSKFlagBytes == kStreamKFlagBytes && kGroupFlagBytes == kStreamKFlagBytes,
              "flag words at the start of every workspace layout");
static_assert(streamk_workspace_bytes(16) == group_workspace_bytes(16) &&
                  streamk_workspace_bytes(32) == group_workspace_bytes(32),
              "an M <= 32 workspace holds the grouped kernel's slots");

static size_t linear_ws_bytes(int64_t M)
{
    if (M >= 1 && M <= 32)
        return streamk_bytes_for(M);
    if (M > 128)
        return pair_sk_workspace_bytes(256);
    return 0;
}

// The grouped kernel's flags and partial slots for one layer of M tokens
// (the NestedFP layers with M <= PGF8_GROUP_MAX_M run it): equal to the
// skinny stream-K region for M <= 32.
static size_t group_one_ws_bytes(int64_t M)
{
    if (M < 1 || M > PGF8_GROUP_MAX_M)
        return 0;
    return group_workspace_bytes(M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256);
}

size_t pgf8_fp8_linear_workspace_size(int64_t M, int64_t, int64_t) { return linear_ws_bytes(M); }

pgf8_status pgf8_fp8_linear_ex(const uint8_t *aq, const float *sa, int64_t M, int64_t K, const uint8_t *wq,
                               const float *sw, int64_t N, void *y, void *workspace, size_t workspace_bytes,
                               const pgf8_linear_opts *opts, void *stream)
{
    pgf8_status st = check_dims(M, N, K);
    if (st != PGF8_OK)
        return st;
    if (!aq || !sa || !wq || !sw || !y)
        return PGF8_ERR_INVALID_ARG;
    if (!aligned16(aq) || !aligned16(wq) || !aligned16(y) || !aligned4(sa) || !aligned4(sw) ||
        !aligned16(workspace))
        return PGF8_ERR_ALIGNMENT;
    GemmLaunch L;
    L.ws = workspace;
    L.ws_bytes = workspace ? workspace_bytes : 0;
    L.kind = kE4M3;
    L.x = aq;
    L.w = wq;
    L.w2 = nullptr;
    L.sa = sa;
    L.sw = sw;
    L.y = y;
    L.M = static_cast<int>(M);
    L.N = static_cast<int>(N);
    L.K = static_cast<int>(K);
    L.pdl = 1;
    L.opts = opts_or_default(opts);
    L.prefetch_w = (L.opts.flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    L.stream = static_cast<cudaStream_t>(stream);
    return launch_gemm<kE4M3>(L);
}

pgf8_status pgf8_fp8_linear(const uint8_t *aq, const float *sa, int64_t M, int64_t K, const uint8_t *wq,
                            const float *sw, int64_t N, void *y, void *workspace, size_t workspace_bytes,
                            void *stream)
{
    return pgf8_fp8_linear_ex(aq, sa, M, K, wq, sw, N, y, workspace, workspace_bytes, nullptr, stream);
}

// Dynamic workspace layout: stream-K flag words (always, so they are never
// overwritten by codes when one workspace serves layers of different shapes)
// | partial slots (M <= 256: the grouped kernel's for one layer, equal to the
// skinny stream-K slots for M <= 32; M > 128: the pair kernel's) | codes
// [M, K] | scales [M].
size_t pgf8_fp8_linear_dynamic_codes_offset(int64_t M, int64_t K)
{
    if (M < 0 || K < 0)
        return 0;
    const size_t b = linear_ws_bytes(M);
    return b > kStreamKFlagBytes ? b : kStreamKFlagBytes;
}

// NestedFP FP8 mode through the grouped kernel (M <= PGF8_GROUP_MAX_M): the
// grouped kernel's flags and partial slots at offset 0, then the codes and
// the scales (a larger region than a dynamic FP8 call's, so that the latter
// keeps its size).
static size_t nested8_codes_offset(int64_t M)
{
    size_t b = linear_ws_bytes(M);
    b = group_one_ws_bytes(M) > b ? group_one_ws_bytes(M) : b;
    return b > kStreamKFlagBytes ? b : kStreamKFlagBytes;
}

static size_t nested8_scales_offset(int64_t M, int64_t K)
{
    return nested8_codes_offset(M) + round_up(static_cast<size_t>(M) * static_cast<size_t>(K), 256);
}

size_t pgf8_fp8_linear_dynamic_scales_offset(int64_t M, int64_t K)
{
    if (M < 0 || K < 0)
        return 0;
    return pgf8_fp8_linear_dynamic_codes_offset(M, K) + round_up(static_cast<size_t>(M) * static_cast<size_t>(K), 256);
}

size_t pgf8_fp8_linear_dynamic_workspace_size(int64_t M, int64_t, int64_t K)
{
    if (M < 0 || K < 0)
        return 0;
    return pgf8_fp8_linear_dynamic_scales_offset(M, K) + round_up(static_cast<size_t>(M) * 4, 256);
}

// Argument checks of a dynamic linear call (nothing is enqueued).
static pgf8_status check_linear_dynamic(const void *x, pgf8_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                       const void *w, const float *sw, int64_t N, void *y, void *workspace,
                                       size_t workspace_bytes, int kind)
{
    pgf8_status st = check_dims(M, N, K);
    if (st != PGF8_OK)
        return st;
    if (!workspace || !w || !y || (kind == kE4M3 && !sw))
        return PGF8_ERR_INVALID_ARG;
    if (workspace_bytes < pgf8_fp8_linear_dynamic_workspace_size(M, N, K))
        return PGF8_ERR_INVALID_ARG;
    if (!aligned16(workspace) || !aligned16(w) || !aligned16(y) || (sw && !aligned4(sw)))
        return PGF8_ERR_ALIGNMENT;
    uint8_t *aq = static_cast<uint8_t *>(workspace) + pgf8_fp8_linear_dynamic_codes_offset(M, K);
    float *sa = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                          pgf8_fp8_linear_dynamic_scales_offset(M, K));
    return check_quantize_args(x, xdt, M, K, ldx, aq, sa, PGF8_SCALE_DYNAMIC);
}

static pgf8_status linear_dynamic_impl(const void *x, pgf8_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                       const void *w, const void *w2, const float *sw, int64_t N, void *y,
                                       void *workspace, size_t workspace_bytes, const pgf8_linear_opts *opts,
                                       void *stream, int kind)
{
    pgf8_status st = check_linear_dynamic(x, xdt, M, K, ldx, w, sw, N, y, workspace, workspace_bytes, kind);
    if (st != PGF8_OK)
        return st;
    uint8_t *aq = static_cast<uint8_t *>(workspace) + pgf8_fp8_linear_dynamic_codes_offset(M, K);
    float *sa = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                          pgf8_fp8_linear_dynamic_scales_offset(M, K));
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const pgf8_linear_opts o = opts_or_default(opts);
    const int overlap = (o.flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    int xq_bn = 0, xq_splits = 0;
    if (fused_quant_plan(M, N, K, xdt, o, xq_bn, xq_splits)) {
        // one kernel: the GEMM quantises the activations of its K-slice itself
        // and writes the codes and scales to the workspace as a side output
        GemmLaunch L;
        L.ws = nullptr;
        L.ws_bytes = 0;
        L.kind = kind;
        L.x = nullptr;
        L.w = w;
        L.w2 = nullptr;
        L.sa = sa;
        L.sw = sw;
        L.y = y;
        L.M = static_cast<int>(M);
        L.N = static_cast<int>(N);
        L.K = static_cast<int>(K);
        L.pdl = overlap;
        L.prefetch_w = 1;   // weights never wait for the previous kernel (see PGF8_FLAG_OVERLAP_PREVIOUS)
        L.opts = o;
        L.stream = cs;
        L.xraw = x;
        L.ldx = ldx;
        L.q_out = aq;
        L.sa_out = sa;
        if (kind == kNested8)   // NestedFP activations are f16
            return launch_gemm_xq<kNested8, 2>(L, xq_bn, xq_splits);
        return xdt == PGF8_F32 ? launch_gemm_xq<kE4M3, 1>(L, xq_bn, xq_splits)
                               : launch_gemm_xq<kE4M3, 2>(L, xq_bn, xq_splits);
    }
    // the quantisation signals its dependent (this call's GEMM) at once: the
    // GEMM loads its first weight tiles while the activations are quantised
    st = quantize_launch(x, xdt, M, K, ldx, aq, sa, 0, cs, overlap, 1);
    if (st != PGF8_OK)
        return st;
    GemmLaunch L;
    L.ws = workspace;   // the stream-K region is at offset 0
    L.ws_bytes = pgf8_fp8_linear_dynamic_codes_offset(M, K);
    L.kind = kind;
    L.x = aq;
    L.w = w;
    L.w2 = w2;
    L.sa = sa;
    L.sw = sw;
    L.y = y;
    L.M = static_cast<int>(M);
    L.N = static_cast<int>(N);
    L.K = static_cast<int>(K);
    L.pdl = 1;
    L.prefetch_w = 1;   // the quantisation kernel writes only aq / sa
    L.opts = o;
    L.stream = cs;
    if (kind == kNested8)
        return launch_gemm<kNested8>(L);
    return launch_gemm<kE4M3>(L);
}

pgf8_status pgf8_fp8_linear_dynamic(const void *x, pgf8_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                    const uint8_t *wq, const float *sw, int64_t N, void *y, void *workspace,
                                    size_t workspace_bytes, const pgf8_linear_opts *opts, void *stream)
{
    return linear_dynamic_impl(x, xdt, M, K, ldx, wq, nullptr, sw, N, y, workspace, workspace_bytes, opts, stream,
                               kE4M3);
}

pgf8_status pgf8_fp8_linear_dynamic_plan(int64_t M, int64_t N, int64_t K, pgf8_dtype xdt,
                                         const pgf8_linear_opts *opts, int32_t *fused, int32_t *split_k)
{
    if (!fused || !split_k)
        return PGF8_ERR_INVALID_ARG;
    pgf8_status st = check_dims(M, N, K);
    if (st != PGF8_OK)
        return st;
    if (xdt != PGF8_F32 && xdt != PGF8_F16)
        return PGF8_ERR_UNSUPPORTED;
    const pgf8_linear_opts o = opts_or_default(opts);
    *fused = 0;
    *split_k = 0;
    int bn = 0, splits = 0;
    if (fused_quant_plan(M, N, K, xdt, o, bn, splits)) {
        *fused = 1;
        *split_k = splits;
        return PGF8_OK;
    }
    const bool skinny = (o.path == PGF8_PATH_AUTO && M <= 128) || o.path == PGF8_PATH_SKINNY;
    if (skinny && M <= 128) {
        const int kblocks = static_cast<int>((K + 127) / 128);
        int sp = o.split_k != 0 ? o.split_k : skinny_auto_splits(static_cast<int>((N + 127) / 128), num_sms());
        *split_k = sp > kblocks ? kblocks : sp;
    }
    return PGF8_OK;
}

pgf8_status pgf8_fp8_linear_dynamic_many(const pgf8_fp8_layer *layers, int64_t count, const pgf8_linear_opts *opts,
                                         void *stream)
{
    if (count < 0 || (count > 0 && !layers))
        return PGF8_ERR_INVALID_ARG;
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_fp8_layer &l = layers[i];
        pgf8_status st = check_linear_dynamic(l.x, static_cast<pgf8_dtype>(l.xdt), l.M, l.K, l.ldx, l.wq, l.sw, l.N,
                                              l.y, l.workspace, l.workspace_bytes, kE4M3);
        if (st != PGF8_OK)
            return st;
    }
    pgf8_linear_opts o = opts_or_default(opts);
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_fp8_layer &l = layers[i];
        if (i > 0)
            o.flags |= PGF8_FLAG_OVERLAP_PREVIOUS;
        pgf8_status st = linear_dynamic_impl(l.x, static_cast<pgf8_dtype>(l.xdt), l.M, l.K, l.ldx, l.wq, nullptr,
                                             l.sw, l.N, l.y, l.workspace, l.workspace_bytes, &o, stream, kE4M3);
        if (st != PGF8_OK)
            return st;
    }
    return PGF8_OK;
}

} // extern "C"

namespace pgf8 {

static int group_bn(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

static bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return na > 0 && nb > 0 && a0 < b0 + nb && b0 < a0 + na;
}

// Bytes of a layer's activations [M, K] at row stride ldx.
static size_t x_span(const pgf8_fp8_layer &l)
{
    const size_t eb = l.xdt == PGF8_F32 ? 4 : 2;
    return (static_cast<size_t>(l.M - 1) * static_cast<size_t>(l.ldx) + static_cast<size_t>(l.K)) * eb;
}

template <class C> static pgf8_status launch_group_cfg(const GroupParams &p, int grid, cudaStream_t st)
{
    static PerDeviceSetup setup;
    const cudaError_t attr_err = setup_once_per_device(setup, [](int, int *) {
        return cudaFuncSetAttribute(gemm_group_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err);
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_group_kernel<C>, p);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

// The grouped kernel for the layers described in gp (units already set),
// token tile bnmax, one CTA per SM at most.
template <int KIND = kE4M3> static pgf8_status launch_group(const GroupParams &gp, int bnmax, cudaStream_t cs)
{
    int grid = num_sms();
    if (grid > kGroupMaxCtas)
        grid = kGroupMaxCtas;
    if (static_cast<int64_t>(grid) > gp.units)
        grid = static_cast<int>(gp.units);
    switch (bnmax) {
    case 16:
        return launch_group_cfg<GroupCfg<16, 12, KIND>>(gp, grid, cs);
    case 32:
        return launch_group_cfg<GroupCfg<32, 11, KIND>>(gp, grid, cs);
    case 64:
        return launch_group_cfg<GroupCfg<64, 9, KIND>>(gp, grid, cs);
    case 128:
        return launch_group_cfg<GroupCfg<128, 6, KIND>>(gp, grid, cs);
    default:
        return launch_group_cfg<GroupCfg<256, 4, KIND>>(gp, grid, cs);
    }
}

// One NestedFP layer of a grouped launch: its operands and, in FP8 mode,
// where its codes and scales go.
struct NestedItem {
    const void *x;
    int64_t M, K, N;
    const uint8_t *hi, *lo;
    void *y;
    uint8_t *aq;
    float *sa;
};

// Up to kGroupMaxLayers NestedFP layers with M <= PGF8_GROUP_MAX_M through
// one grouped launch (every SM streams an equal share of all their weight
// planes).  FP8 mode: the f16 activations are quantised per token first
// (one launch), the hi plane is read as E5M2; FP16 mode: the f16
// activations are read as they are and the weights rebuilt from both
// planes.  group_ws holds the flags and partial slots.
static pgf8_status nested_group_chunk(const NestedItem *it, int n, pgf8_nested_mode mode, void *group_ws,
                                      int overlap, cudaStream_t cs)
{
    GroupParams gp;
    std::memset(&gp, 0, sizeof(gp));
    int64_t units = 0;
    int bnmax = 16;
    const bool fp8 = (mode == PGF8_NESTED_FP8);
    for (int i = 0; i < n; ++i) {
        const NestedItem &l = it[i];
        const int bn = group_bn(l.M);
        bnmax = bn > bnmax ? bn : bnmax;
        GroupLayer &g = gp.L[i];
        g.unit0 = units;
        g.M = static_cast<int>(l.M);
        g.N = static_cast<int>(l.N);
        g.K = static_cast<int>(l.K);
        g.bn = bn;
        g.y = l.y;
        bool ok;
        if (fp8) {
            g.kblocks = static_cast<int>((l.K + 127) / 128);
            g.sa = l.sa;
            ok = make_map(&gp.tmW[i], l.hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.N),
                          static_cast<uint64_t>(l.K), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
                 make_map(&gp.tmX[i], l.aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.M),
                          static_cast<uint64_t>(l.K), 128, static_cast<uint32_t>(bn), CU_TENSOR_MAP_SWIZZLE_128B);
        } else {
            g.kblocks = static_cast<int>((l.K * 2 + 127) / 128);
            ok = make_map(&gp.tmW[i], l.hi, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.N),
                          static_cast<uint64_t>(l.K), 64, 128, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                 make_map(&gp.tmW2[i], l.lo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.N),
                          static_cast<uint64_t>(l.K), 64, 128, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                 make_map(&gp.tmX[i], l.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, static_cast<uint64_t>(l.M),
                          static_cast<uint64_t>(l.K), 64, static_cast<uint32_t>(bn), CU_TENSOR_MAP_SWIZZLE_128B);
        }
        if (!ok)
            return PGF8_ERR_UNSUPPORTED;
        units += static_cast<int64_t>((l.N + 127) / 128) * g.kblocks;
    }
    gp.nlayers = n;
    gp.units = units;
    gp.flags = static_cast<unsigned *>(group_ws);
    gp.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(group_ws) + kGroupFlagBytes);
    if (!fp8) {
        gp.prefetch_w = overlap;   // the weight planes may come from the kernel before (the split)
        return launch_group<kNested16>(gp, bnmax, cs);
    }
    gp.prefetch_w = 1;   // the quantisation before writes only codes and scales
    if (n == 1) {
        // one layer: the row kernels, which signal the grouped GEMM at once
        // (it loads its first weight tiles while the activations are quantised)
        const pgf8_status st = quantize_launch(it[0].x, PGF8_F16, it[0].M, it[0].K, it[0].K, it[0].aq, it[0].sa, 0,
                                               cs, overlap, 1);
        if (st != PGF8_OK)
            return st;
        return launch_group<kNested8>(gp, bnmax, cs);
    }
    QuantGroupParams qp;
    std::memset(&qp, 0, sizeof(qp));
    int64_t rows = 0;
    for (int i = 0; i < n; ++i) {
        QuantGroupLayer &q = qp.L[i];
        q.x = it[i].x;
        q.ldx = it[i].K;
        q.cols = it[i].K;
        q.row0 = rows;
        q.rows = it[i].M;
        q.q = it[i].aq;
        q.scales = it[i].sa;
        q.xdt = 1;
        rows += it[i].M;
    }
    qp.nlayers = n;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    if (overlap) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    const cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_group_kernel, qp);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return launch_group<kNested8>(gp, bnmax, cs);
}

// A NestedFP layer with M <= PGF8_GROUP_MAX_M through the grouped kernel
// alone: the workspace holds the flags and partial slots at offset 0 and, in
// FP8 mode, the codes and scales after them.
static pgf8_status nested_group_one(const void *x, int64_t M, int64_t K, const uint8_t *hi, const uint8_t *lo,
                                    int64_t N, pgf8_nested_mode mode, void *y, void *workspace, int overlap,
                                    cudaStream_t cs)
{
    NestedItem it;
    it.x = x;
    it.M = M;
    it.K = K;
    it.N = N;
    it.hi = hi;
    it.lo = lo;
    it.y = y;
    it.aq = static_cast<uint8_t *>(workspace) + nested8_codes_offset(M);
    it.sa = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + nested8_scales_offset(M, K));
    return nested_group_chunk(&it, 1, mode, workspace, overlap, cs);
}

// One grouped launch pair for up to kGroupMaxLayers small-M layers: the
// per-token quantisation of all of them, then the grouped GEMM, which
// streams its first ring of weights while the quantisation runs.
// Layers with more 256 x 256 tiles than this (four rounds of the 74 SM
// pairs) run one launch each: measured on B200 over the llama70b step, one
// launch over every M > 128 layer ran 8 % slower than one launch per layer
// (8.24 against 7.62 ms), while on the 7B prefill layers (a few rounds
// each) the shared launch was 9 % faster.
constexpr int64_t kPairGroupMaxTiles = 296;

// Up to kPairGroupMaxLayers pre-quantised FP8 GEMMs: one persistent launch
// on SM pairs over all the 256 x 256 tiles of the layers with at most
// kPairGroupMaxTiles tiles, then one tiled launch for each larger layer (all
// with programmatic stream serialization: nothing is read before the
// previous kernel has completed).
static pgf8_status tiled_group_launch(const pgf8_fp8_gemm_layer *ls, int n, cudaStream_t cs)
{
    PairGroupParams gp;   // about 10 KB: passed by value as the kernel's parameter block
    std::memset(&gp, 0, sizeof(gp));
    int64_t tiles = 0;
    int ng = 0;
    auto ntiles = [](const pgf8_fp8_gemm_layer &l) { return ((l.M + 255) / 256) * ((l.N + 255) / 256); };
    // The shared list takes the layers in order of K (stable): the pairs
    // walk it round-robin, and tiles of one length keep them in step, so the
    // tiles in flight at any time stay neighbours (their operands shared in
    // L2); a pair that met a longer tile would otherwise fall behind its
    // neighbours for the rest of the list.
    int order[kPairGroupMaxLayers];
    for (int i = 0; i < n; ++i)
        order[i] = i;
    for (int i = 1; i < n; ++i)
        for (int j = i; j > 0 && ls[order[j - 1]].K > ls[order[j]].K; --j) {
            const int t = order[j];
            order[j] = order[j - 1];
            order[j - 1] = t;
        }
    for (int oi = 0; oi < n; ++oi) {
        const pgf8_fp8_gemm_layer &l = ls[order[oi]];
        if (ntiles(l) > kPairGroupMaxTiles)
            continue;
        const int gi = ng++;
        PairGroupLayer &g = gp.L[gi];
        g.M = static_cast<int>(l.M);
        g.N = static_cast<int>(l.N);
        g.kblocks = static_cast<int>((l.K + 127) / 128);
        g.m_tiles = static_cast<int>((l.M + 255) / 256);
        g.tile0 = static_cast<int>(tiles);
        g.sa = l.sa;
        g.sw = l.sw;
        g.y = l.y;
        tiles += ntiles(l);
        if (!make_map(&gp.tmX[gi], l.aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.M),
                      static_cast<uint64_t>(l.K), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&gp.tmW[gi], l.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.N),
                      static_cast<uint64_t>(l.K), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
            return PGF8_ERR_UNSUPPORTED;
    }
    if (ng > 0) {
        gp.nlayers = ng;
        gp.total = static_cast<int>(tiles);
        const pgf8_status st = launch_pair_group(gp, cs);
        if (st != PGF8_OK)
            return st;
    }
    for (int i = 0; i < n; ++i) {
        const pgf8_fp8_gemm_layer &l = ls[i];
        if (ntiles(l) <= kPairGroupMaxTiles)
            continue;
        GemmLaunch L;
        L.ws = nullptr;
        L.ws_bytes = 0;
        L.kind = kE4M3;
        L.x = l.aq;
        L.w = l.wq;
        L.w2 = nullptr;
        L.sa = l.sa;
        L.sw = l.sw;
        L.y = l.y;
        L.M = static_cast<int>(l.M);
        L.N = static_cast<int>(l.N);
        L.K = static_cast<int>(l.K);
        L.pdl = 1;
        L.prefetch_w = 1;   // nothing before writes the weights
        L.opts = opts_or_default(nullptr);
        L.stream = cs;
        const pgf8_status st = launch_gemm<kE4M3>(L);
        if (st != PGF8_OK)
            return st;
    }
    return PGF8_OK;
}

// Up to kPairGroupMaxLayers tiled layers (M > 128): the per-token
// quantisation of all of them (one launch), then their GEMMs as
// tiled_group_launch runs them.
static pgf8_status pair_group_chunk(const pgf8_fp8_layer *const *ls, int n, int first_pdl, cudaStream_t cs)
{
    QuantGroupParams qp;
    std::memset(&qp, 0, sizeof(qp));
    pgf8_fp8_gemm_layer gl[kPairGroupMaxLayers];
    int64_t rows = 0;
    for (int i = 0; i < n; ++i) {
        const pgf8_fp8_layer &l = *ls[i];
        uint8_t *aq = static_cast<uint8_t *>(l.workspace) + pgf8_fp8_linear_dynamic_codes_offset(l.M, l.K);
        float *sa = reinterpret_cast<float *>(static_cast<uint8_t *>(l.workspace) +
                                              pgf8_fp8_linear_dynamic_scales_offset(l.M, l.K));
        QuantGroupLayer &q = qp.L[i];
        q.x = l.x;
        q.ldx = l.ldx;
        q.cols = l.K;
        q.row0 = rows;
        q.rows = l.M;
        q.q = aq;
        q.scales = sa;
        q.xdt = l.xdt == PGF8_F32 ? 0 : 1;
        rows += l.M;
        gl[i].aq = aq;
        gl[i].sa = sa;
        gl[i].wq = l.wq;
        gl[i].sw = l.sw;
        gl[i].y = l.y;
        gl[i].M = l.M;
        gl[i].K = l.K;
        gl[i].N = l.N;
    }
    if (rows > (1ll << 31) - 1)
        return PGF8_ERR_UNSUPPORTED;
    qp.nlayers = n;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    if (first_pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    const cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_group_kernel, qp);
    if (e != cudaSuccess)
        return cuda_fail(e);
    return tiled_group_launch(gl, n, cs);
}

static pgf8_status group_chunk(const pgf8_fp8_layer *const *ls, int n, void *group_ws, int first_pdl,
                               cudaStream_t cs)
{
    QuantGroupParams qp;
    std::memset(&qp, 0, sizeof(qp));
    GroupParams gp;   // about 10 KB: passed by value as the kernel's parameter block
    std::memset(&gp, 0, sizeof(gp));
    int64_t rows = 0, units = 0;
    int bnmax = 16;
    for (int i = 0; i < n; ++i) {
        const pgf8_fp8_layer &l = *ls[i];
        uint8_t *aq = static_cast<uint8_t *>(l.workspace) + pgf8_fp8_linear_dynamic_codes_offset(l.M, l.K);
        float *sa = reinterpret_cast<float *>(static_cast<uint8_t *>(l.workspace) +
                                              pgf8_fp8_linear_dynamic_scales_offset(l.M, l.K));
        QuantGroupLayer &q = qp.L[i];
        q.x = l.x;
        q.ldx = l.ldx;
        q.cols = l.K;
        q.row0 = rows;
        q.rows = l.M;
        q.q = aq;
        q.scales = sa;
        q.xdt = l.xdt == PGF8_F32 ? 0 : 1;
        rows += l.M;

        const int bn = group_bn(l.M);
        bnmax = bn > bnmax ? bn : bnmax;
        GroupLayer &g = gp.L[i];
        g.unit0 = units;
        g.M = static_cast<int>(l.M);
        g.N = static_cast<int>(l.N);
        g.K = static_cast<int>(l.K);
        g.kblocks = static_cast<int>((l.K + 127) / 128);
        g.bn = bn;
        g.sa = sa;
        g.sw = l.sw;
        g.y = l.y;
        units += static_cast<int64_t>((l.N + 127) / 128) * g.kblocks;
        if (!make_map(&gp.tmW[i], l.wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.N),
                      static_cast<uint64_t>(l.K), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&gp.tmX[i], aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(l.M),
                      static_cast<uint64_t>(l.K), 128, static_cast<uint32_t>(bn), CU_TENSOR_MAP_SWIZZLE_128B))
            return PGF8_ERR_UNSUPPORTED;
    }
    qp.nlayers = n;
    gp.nlayers = n;
    gp.prefetch_w = 1;   // the quantisation kernel writes only codes and scales
    gp.units = units;
    gp.flags = static_cast<unsigned *>(group_ws);
    gp.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(group_ws) + kGroupFlagBytes);

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    if (first_pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_group_kernel, qp);
    if (e != cudaSuccess)
        return cuda_fail(e);

    return launch_group(gp, bnmax, cs);
}

} // namespace pgf8

extern "C" {

size_t pgf8_fp8_linear_group_workspace_size(int64_t max_m)
{
    if (max_m < 1)
        return kGroupFlagBytes;
    return group_workspace_bytes(group_bn(max_m < PGF8_GROUP_MAX_M ? max_m : PGF8_GROUP_MAX_M));
}

pgf8_status pgf8_fp8_linear_dynamic_group(const pgf8_fp8_layer *layers, int64_t count, void *group_workspace,
                                          size_t group_workspace_bytes, const pgf8_linear_opts *opts, void *stream)
{
    if (count < 0 || (count > 0 && !layers))
        return PGF8_ERR_INVALID_ARG;
    int64_t max_small = 0;
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_fp8_layer &l = layers[i];
        pgf8_status st = check_linear_dynamic(l.x, static_cast<pgf8_dtype>(l.xdt), l.M, l.K, l.ldx, l.wq, l.sw, l.N,
                                              l.y, l.workspace, l.workspace_bytes, kE4M3);
        if (st != PGF8_OK)
            return st;
        if (l.M <= PGF8_GROUP_MAX_M && l.M > max_small)
            max_small = l.M;
    }
    // independent layers only: no layer writes (y, workspace) what another
    // layer reads or writes
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_fp8_layer &a = layers[i];
        const size_t ya = static_cast<size_t>(a.M) * static_cast<size_t>(a.N) * 2;
        for (int64_t j = 0; j < count; ++j) {
            const pgf8_fp8_layer &b = layers[j];
            if (ranges_overlap(a.y, ya, b.x, x_span(b)) ||
                ranges_overlap(a.workspace, a.workspace_bytes, b.x, x_span(b)))
                return PGF8_ERR_INVALID_ARG;
            if (i != j && (ranges_overlap(a.y, ya, b.y, static_cast<size_t>(b.M) * static_cast<size_t>(b.N) * 2) ||
                           ranges_overlap(a.workspace, a.workspace_bytes, b.workspace, b.workspace_bytes) ||
                           ranges_overlap(a.y, ya, b.workspace, b.workspace_bytes)))
                return PGF8_ERR_INVALID_ARG;
        }
    }
    if (max_small > 0) {
        if (!group_workspace || group_workspace_bytes < pgf8_fp8_linear_group_workspace_size(max_small))
            return PGF8_ERR_INVALID_ARG;
        if (!aligned16(group_workspace))
            return PGF8_ERR_ALIGNMENT;
    }
    pgf8_linear_opts o = opts_or_default(opts);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    int pdl = (o.flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    // small layers: grouped, kGroupMaxLayers per launch pair, in call order:
    // one launch for the layers with M <= 128 (its ring sized for the widest
    // of their token tiles: measured faster on B200 than one launch per
    // 16 / 32 / 64 / 128 class, which pays a launch's start and end per
    // class), one for 128 < M <= 256 (256-token tiles, a 4-deep ring:
    // measured 11 % faster than the per-layer kernels at 70B M = 256)
    // With the automatic kernel choice every layer with M > 128 joins one
    // tiled launch on SM pairs (per kPairGroupMaxLayers layers), after one
    // quantisation launch for all of them: measured on B200 faster than the
    // grouped kernel's 256-token tiles for 128 < M <= 256 and than one pair
    // of launches per larger layer (whose last round of tiles leaves SMs idle).
    const bool auto_choice = o.path == PGF8_PATH_AUTO && o.tile_n == 0 && o.split_k == 0;
    const pgf8_fp8_layer *chunk[kGroupMaxLayers];
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1 && auto_choice)
            break;
        const int64_t lo = pass == 0 ? 0 : 128, hi = pass == 0 ? 128 : PGF8_GROUP_MAX_M;
        int n = 0;
        for (int64_t i = 0; i <= count; ++i) {
            if (i < count && layers[i].M > lo && layers[i].M <= hi)
                chunk[n++] = &layers[i];
            if (n == kGroupMaxLayers || (i == count && n > 0)) {
                pgf8_status st = group_chunk(chunk, n, group_workspace, pdl, cs);
                if (st != PGF8_OK)
                    return st;
                n = 0;
                pdl = 1;
            }
        }
    }
    if (auto_choice) {
        static_assert(kPairGroupMaxLayers <= kGroupMaxLayers && kPairGroupMaxLayers <= kQuantGroupMaxLayers,
                      "chunk sizes");
        int n = 0;
        for (int64_t i = 0; i <= count; ++i) {
            if (i < count && layers[i].M > 128)
                chunk[n++] = &layers[i];
            if (n == kPairGroupMaxLayers || (i == count && n > 0)) {
                pgf8_status st = pair_group_chunk(chunk, n, pdl, cs);
                if (st != PGF8_OK)
                    return st;
                n = 0;
                pdl = 1;
            }
        }
        return PGF8_OK;
    }
    // explicit kernel options: the layers with M > PGF8_GROUP_MAX_M one
    // dynamic call each, overlapping the previous one
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_fp8_layer &l = layers[i];
        if (l.M <= PGF8_GROUP_MAX_M)
            continue;
        if (pdl)
            o.flags |= PGF8_FLAG_OVERLAP_PREVIOUS;
        pgf8_status st = linear_dynamic_impl(l.x, static_cast<pgf8_dtype>(l.xdt), l.M, l.K, l.ldx, l.wq, nullptr,
                                             l.sw, l.N, l.y, l.workspace, l.workspace_bytes, &o, stream, kE4M3);
        if (st != PGF8_OK)
            return st;
        pdl = 1;
    }
    return PGF8_OK;
}

pgf8_status pgf8_fp8_linear_group(const pgf8_fp8_gemm_layer *layers, int64_t count, const pgf8_linear_opts *opts,
                                  void *stream)
{
    if (count < 0 || (count > 0 && !layers))
        return PGF8_ERR_INVALID_ARG;
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_fp8_gemm_layer &l = layers[i];
        pgf8_status st = check_dims(l.M, l.N, l.K);
        if (st != PGF8_OK)
            return st;
        if (!l.aq || !l.sa || !l.wq || !l.sw || !l.y)
            return PGF8_ERR_INVALID_ARG;
        if (!aligned16(l.aq) || !aligned16(l.wq) || !aligned16(l.y) || !aligned4(l.sa) || !aligned4(l.sw))
            return PGF8_ERR_ALIGNMENT;
        if (l.M > (1ll << 30) || l.N > (1ll << 30))
            return PGF8_ERR_UNSUPPORTED;
    }
    // no layer's output overlaps any layer's operands or another layer's output
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_fp8_gemm_layer &a = layers[i];
        const size_t ya = static_cast<size_t>(a.M) * static_cast<size_t>(a.N) * 2;
        for (int64_t j = 0; j < count; ++j) {
            const pgf8_fp8_gemm_layer &b = layers[j];
            if (ranges_overlap(a.y, ya, b.aq, static_cast<size_t>(b.M) * static_cast<size_t>(b.K)) ||
                ranges_overlap(a.y, ya, b.sa, static_cast<size_t>(b.M) * 4) ||
                ranges_overlap(a.y, ya, b.wq, static_cast<size_t>(b.N) * static_cast<size_t>(b.K)) ||
                ranges_overlap(a.y, ya, b.sw, static_cast<size_t>(b.N) * 4))
                return PGF8_ERR_INVALID_ARG;
            if (i != j && ranges_overlap(a.y, ya, b.y, static_cast<size_t>(b.M) * static_cast<size_t>(b.N) * 2))
                return PGF8_ERR_INVALID_ARG;
        }
    }
    const pgf8_linear_opts o = opts_or_default(opts);
    if (o.path != PGF8_PATH_AUTO || o.split_k != 0 || o.tile_n != 0)
        return PGF8_ERR_UNSUPPORTED;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    for (int64_t c0 = 0; c0 < count; c0 += kPairGroupMaxLayers) {
        const int n = static_cast<int>(count - c0 < kPairGroupMaxLayers ? count - c0 : kPairGroupMaxLayers);
        const pgf8_status st = tiled_group_launch(layers + c0, n, cs);
        if (st != PGF8_OK)
            return st;
    }
    return PGF8_OK;
}

size_t pgf8_fp8_linear_partial_workspace_size(int64_t M, int64_t, int64_t)
{
    if (M < 1)
        return 0;
    return M <= PGF8_GROUP_MAX_M ? group_workspace_bytes(group_bn(M)) : pair_sk_workspace_bytes(256);
}

pgf8_status pgf8_fp8_linear_partial(const uint8_t *aq, const float *sa, int64_t M, int64_t K, const uint8_t *wq,
                                    const float *sw, int64_t N, float *y_f32, void *workspace, size_t workspace_bytes,
                                    void *stream)
{
    pgf8_status st = check_dims(M, N, K);
    if (st != PGF8_OK)
        return st;
    if (!aq || !sa || !wq || !sw || !y_f32 || !workspace)
        return PGF8_ERR_INVALID_ARG;
    if (workspace_bytes < pgf8_fp8_linear_partial_workspace_size(M, N, K))
        return PGF8_ERR_INVALID_ARG;
    if (!aligned16(aq) || !aligned16(wq) || !aligned16(y_f32) || !aligned4(sa) || !aligned4(sw) ||
        !aligned16(workspace))
        return PGF8_ERR_ALIGNMENT;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (M <= PGF8_GROUP_MAX_M) {
        GroupParams gp;
        std::memset(&gp, 0, sizeof(gp));
        const int bn = group_bn(M);
        GroupLayer &g = gp.L[0];
        g.unit0 = 0;
        g.M = static_cast<int>(M);
        g.N = static_cast<int>(N);
        g.K = static_cast<int>(K);
        g.kblocks = static_cast<int>((K + 127) / 128);
        g.bn = bn;
        g.sa = sa;
        g.sw = sw;
        g.y = y_f32;
        g.out_f32 = 1;
        if (!make_map(&gp.tmW[0], wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(N),
                      static_cast<uint64_t>(K), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&gp.tmX[0], aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(M),
                      static_cast<uint64_t>(K), 128, static_cast<uint32_t>(bn), CU_TENSOR_MAP_SWIZZLE_128B))
            return PGF8_ERR_UNSUPPORTED;
        gp.nlayers = 1;
        gp.prefetch_w = 0;
        gp.units = static_cast<int64_t>((N + 127) / 128) * g.kblocks;
        gp.flags = static_cast<unsigned *>(workspace);
        gp.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kGroupFlagBytes);
        return launch_group(gp, bn, cs);
    }
    GemmLaunch L;
    L.ws = workspace;
    L.ws_bytes = workspace_bytes;
    L.kind = kE4M3;
    L.x = aq;
    L.w = wq;
    L.w2 = nullptr;
    L.sa = sa;
    L.sw = sw;
    L.y = y_f32;
    L.M = static_cast<int>(M);
    L.N = static_cast<int>(N);
    L.K = static_cast<int>(K);
    L.pdl = 1;
    L.prefetch_w = 0;
    L.opts = opts_or_default(nullptr);
    L.stream = cs;
    L.out_f32 = 1;
    return launch_pair_bn<kE4M3>(L, 256);
}

pgf8_status pgf8_round_bf16(const float *x, int64_t n, void *y_bf16, void *stream)
{
    if (n < 0 || (n > 0 && (!x || !y_bf16)))
        return PGF8_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y_bf16) || n % 8 != 0)
        return PGF8_ERR_ALIGNMENT;
    if (n == 0)
        return PGF8_OK;
    const int64_t n8 = n / 8;
    const int64_t want = (n8 + 255) / 256;
    const unsigned grid = static_cast<unsigned>(want < 148 * 16 ? want : 148 * 16);
    round_bf16_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<const float4 *>(x), n8,
                                                                          static_cast<uint4 *>(y_bf16));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

pgf8_status pgf8_nestedfp_split(const void *w, int64_t N, int64_t K, uint8_t *hi, uint8_t *lo, void *stream)
{
    if (!w || !hi || !lo || N < 0 || K < 0)
        return PGF8_ERR_INVALID_ARG;
    const int64_t count = N * K;
    if (count % 8 != 0 || !aligned16(w) || !aligned16(hi) || !aligned16(lo))
        return PGF8_ERR_ALIGNMENT;
    if (count == 0)
        return PGF8_OK;
    const int64_t n8 = count / 8;
    const int64_t blocks_needed = (n8 + 255) / 256;
    const unsigned grid = static_cast<unsigned>(blocks_needed < 148 * 16 ? blocks_needed : 148 * 16);
    nestedfp_split_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(w), n8, reinterpret_cast<uint2 *>(hi), reinterpret_cast<uint2 *>(lo));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

size_t pgf8_nestedfp_linear_workspace_size(int64_t M, int64_t N, int64_t K, pgf8_nested_mode mode)
{
    if (mode == PGF8_NESTED_FP8) {
        if (M < 0 || K < 0)
            return 0;
        const size_t dyn = pgf8_fp8_linear_dynamic_workspace_size(M, N, K);
        const size_t grp = nested8_scales_offset(M, K) + round_up(static_cast<size_t>(M) * 4, 256);
        return M >= 1 && M <= PGF8_GROUP_MAX_M && grp > dyn ? grp : dyn;
    }
    return group_one_ws_bytes(M);
}

pgf8_status pgf8_nestedfp_linear_ex(const void *x, int64_t M, int64_t K, const uint8_t *hi, const uint8_t *lo,
                                    int64_t N, pgf8_nested_mode mode, void *y, void *workspace,
                                    size_t workspace_bytes, const pgf8_linear_opts *opts, void *stream)
{
    const pgf8_linear_opts o = opts_or_default(opts);
    // automatic choice, 16 < M <= 256: the grouped weight-streaming kernel
    // with this one layer (measured on B200 faster than the split-K skinny
    // kernel from M = 128 on every 7B / 70B shape; at M <= 16 the skinny
    // kernel's shorter start and end win for a layer called alone)
    const bool grouped = M > 16 && M <= PGF8_GROUP_MAX_M && o.path == PGF8_PATH_AUTO && o.split_k == 0 &&
                         o.tile_n == 0 && !(o.flags & PGF8_FLAG_FUSED_QUANT);
    const int overlap = (o.flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    if (mode == PGF8_NESTED_FP8) {
        if (!grouped)
            return linear_dynamic_impl(x, PGF8_F16, M, K, K, hi, nullptr, nullptr, N, y, workspace, workspace_bytes,
                                       opts, stream, kNested8);
        pgf8_status st = check_linear_dynamic(x, PGF8_F16, M, K, K, hi, nullptr, N, y, workspace, workspace_bytes,
                                              kNested8);
        if (st != PGF8_OK)
            return st;
        if (workspace_bytes < pgf8_nestedfp_linear_workspace_size(M, N, K, mode))
            return PGF8_ERR_INVALID_ARG;
        return nested_group_one(x, M, K, hi, nullptr, N, mode, y, workspace, overlap,
                                static_cast<cudaStream_t>(stream));
    }
    if (mode != PGF8_NESTED_FP16)
        return PGF8_ERR_INVALID_ARG;
    pgf8_status st = check_dims(M, N, K);
    if (st != PGF8_OK)
        return st;
    if (!x || !hi || !lo || !y)
        return PGF8_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(hi) || !aligned16(lo) || !aligned16(y) || !aligned16(workspace))
        return PGF8_ERR_ALIGNMENT;
    if (grouped) {
        if (!workspace || workspace_bytes < pgf8_nestedfp_linear_workspace_size(M, N, K, mode))
            return PGF8_ERR_INVALID_ARG;
        return nested_group_one(x, M, K, hi, lo, N, mode, y, workspace, overlap, static_cast<cudaStream_t>(stream));
    }
    GemmLaunch L;
    L.ws = workspace;
    L.ws_bytes = workspace ? workspace_bytes : 0;
    L.kind = kNested16;
    L.x = x;
    L.w = hi;
    L.w2 = lo;
    L.sa = nullptr;
    L.sw = nullptr;
    L.y = y;
    L.M = static_cast<int>(M);
    L.N = static_cast<int>(N);
    L.K = static_cast<int>(K);
    L.pdl = 1;
    L.opts = opts_or_default(opts);
    L.prefetch_w = (L.opts.flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    L.stream = static_cast<cudaStream_t>(stream);
    return launch_gemm<kNested16>(L);
}

pgf8_status pgf8_nestedfp_linear(const void *x, int64_t M, int64_t K, const uint8_t *hi, const uint8_t *lo,
                                 int64_t N, pgf8_nested_mode mode, void *y, void *workspace, size_t workspace_bytes,
                                 void *stream)
{
    return pgf8_nestedfp_linear_ex(x, M, K, hi, lo, N, mode, y, workspace, workspace_bytes, nullptr, stream);
}

pgf8_status pgf8_nestedfp_linear_group(const pgf8_nested_layer *layers, int64_t count, pgf8_nested_mode mode,
                                       void *group_workspace, size_t group_workspace_bytes,
                                       const pgf8_linear_opts *opts, void *stream)
{
    if (count < 0 || (count > 0 && !layers))
        return PGF8_ERR_INVALID_ARG;
    if (mode != PGF8_NESTED_FP16 && mode != PGF8_NESTED_FP8)
        return PGF8_ERR_INVALID_ARG;
    const bool fp8 = (mode == PGF8_NESTED_FP8);
    int64_t max_small = 0;
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_nested_layer &l = layers[i];
        pgf8_status st;
        if (fp8) {
            st = check_linear_dynamic(l.x_f16, PGF8_F16, l.M, l.K, l.K, l.hi, nullptr, l.N, l.y_f16, l.workspace,
                                      l.workspace_bytes, kNested8);
            if (st == PGF8_OK && l.workspace_bytes < pgf8_nestedfp_linear_workspace_size(l.M, l.N, l.K, mode))
                st = PGF8_ERR_INVALID_ARG;
        } else {
            st = check_dims(l.M, l.N, l.K);
            if (st == PGF8_OK && (!l.x_f16 || !l.hi || !l.lo || !l.y_f16))
                st = PGF8_ERR_INVALID_ARG;
            if (st == PGF8_OK && (!aligned16(l.x_f16) || !aligned16(l.hi) || !aligned16(l.lo) || !aligned16(l.y_f16)))
                st = PGF8_ERR_ALIGNMENT;
        }
        if (st != PGF8_OK)
            return st;
        if (l.M <= PGF8_GROUP_MAX_M && l.M > max_small)
            max_small = l.M;
    }
    // independent layers only: no layer writes (y, workspace) what another
    // layer reads or writes
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_nested_layer &a = layers[i];
        const size_t ya = static_cast<size_t>(a.M) * static_cast<size_t>(a.N) * 2;
        const size_t wa = fp8 ? a.workspace_bytes : 0;
        for (int64_t j = 0; j < count; ++j) {
            const pgf8_nested_layer &b = layers[j];
            const size_t xb = static_cast<size_t>(b.M) * static_cast<size_t>(b.K) * 2;
            if (ranges_overlap(a.y_f16, ya, b.x_f16, xb) || (wa && ranges_overlap(a.workspace, wa, b.x_f16, xb)))
                return PGF8_ERR_INVALID_ARG;
            const size_t wb = fp8 ? b.workspace_bytes : 0;
            if (i != j && (ranges_overlap(a.y_f16, ya, b.y_f16, static_cast<size_t>(b.M) * static_cast<size_t>(b.N) * 2) ||
                           (wa && wb && ranges_overlap(a.workspace, wa, b.workspace, wb)) ||
                           (wb && ranges_overlap(a.y_f16, ya, b.workspace, wb))))
                return PGF8_ERR_INVALID_ARG;
        }
    }
    if (max_small > 0) {
        if (!group_workspace || group_workspace_bytes < pgf8_fp8_linear_group_workspace_size(max_small))
            return PGF8_ERR_INVALID_ARG;
        if (!aligned16(group_workspace))
            return PGF8_ERR_ALIGNMENT;
    }
    pgf8_linear_opts o = opts_or_default(opts);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    int pdl = (o.flags & PGF8_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
    // small layers: grouped as in pgf8_fp8_linear_dynamic_group, codes and
    // scales (FP8 mode) at the dynamic layout's offsets of each workspace
    NestedItem chunk[kGroupMaxLayers];
    for (int pass = 0; pass < 2; ++pass) {
        const int64_t lo = pass == 0 ? 0 : 128, hi = pass == 0 ? 128 : PGF8_GROUP_MAX_M;
        int n = 0;
        for (int64_t i = 0; i <= count; ++i) {
            if (i < count && layers[i].M > lo && layers[i].M <= hi) {
                const pgf8_nested_layer &l = layers[i];
                NestedItem &it = chunk[n++];
                it.x = l.x_f16;
                it.M = l.M;
                it.K = l.K;
                it.N = l.N;
                it.hi = l.hi;
                it.lo = l.lo;
                it.y = l.y_f16;
                it.aq = fp8 ? static_cast<uint8_t *>(l.workspace) + pgf8_fp8_linear_dynamic_codes_offset(l.M, l.K)
                            : nullptr;
                it.sa = fp8 ? reinterpret_cast<float *>(static_cast<uint8_t *>(l.workspace) +
                                                        pgf8_fp8_linear_dynamic_scales_offset(l.M, l.K))
                            : nullptr;
            }
            if (n == kGroupMaxLayers || (i == count && n > 0)) {
                const pgf8_status st = nested_group_chunk(chunk, n, mode, group_workspace, pdl, cs);
                if (st != PGF8_OK)
                    return st;
                n = 0;
                pdl = 1;
            }
        }
    }
    // large layers: one call each (the tiled kernels), overlapping the previous one
    for (int64_t i = 0; i < count; ++i) {
        const pgf8_nested_layer &l = layers[i];
        if (l.M <= PGF8_GROUP_MAX_M)
            continue;
        pgf8_linear_opts ol = o;
        ol.path = PGF8_PATH_AUTO;
        ol.split_k = 0;
        ol.tile_n = 0;
        ol.flags = pdl ? PGF8_FLAG_OVERLAP_PREVIOUS : 0;
        const pgf8_status st = pgf8_nestedfp_linear_ex(l.x_f16, l.M, l.K, l.hi, fp8 ? nullptr : l.lo, l.N, mode,
                                                       l.y_f16, l.workspace, l.workspace_bytes, &ol, stream);
        if (st != PGF8_OK)
            return st;
        pdl = 1;
    }
    return PGF8_OK;
}

pgf8_status pgf8_last_cuda_error(int *cuda_err)
{
    if (!cuda_err)
        return PGF8_ERR_INVALID_ARG;
    *cuda_err = tl_last_cuda_error;
    return PGF8_OK;
}

pgf8_status pgf8_selftest_bounded_wait(int64_t limit_ns, void *stream)
{
    if (limit_ns < 1000 || limit_ns > 2000000000ll)
        return PGF8_ERR_INVALID_ARG;
    selftest_bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(limit_ns));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

pgf8_status pgf8_selftest_row_division(const float *divisors, int32_t count, unsigned long long *mismatches,
                                       void *stream)
{
    if (!divisors || !mismatches || count < 1 || count > 64)
        return PGF8_ERR_INVALID_ARG;
    if (!aligned4(divisors) || (reinterpret_cast<uintptr_t>(mismatches) & 7u) != 0)
        return PGF8_ERR_ALIGNMENT;
    dim3 grid(static_cast<unsigned>(num_sms() * 8), static_cast<unsigned>(count));
    selftest_row_division_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(divisors, count, mismatches);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e);
    return PGF8_OK;
}

pgf8_status pgf8_device_status(void *stream)
{
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e);
    unsigned int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
        if (e != cudaSuccess)
            return cuda_fail(e);
        return PGF8_ERR_TIMEOUT;
    }
    return PGF8_OK;
}

const char *pgf8_status_str(pgf8_status s)
{
    switch (s) {
    case PGF8_OK: return "ok";
    case PGF8_ERR_INVALID_ARG: return "invalid argument";
    case PGF8_ERR_ALIGNMENT: return "alignment or divisibility requirement violated";
    case PGF8_ERR_UNSUPPORTED: return "unsupported configuration";
    case PGF8_ERR_CUDA: return "CUDA error";
    case PGF8_ERR_TIMEOUT: return "device-side bounded wait expired";
    case PGF8_ERR_TOO_LARGE: return "problem exceeds the fixed scratch array of the allocation-free entry point";
    }
    return "unknown status";
}

int pgf8_version(void) { return 200; }   // 0.2.0: per-tensor scaling, norm / gate fusion, FP8 KV cache and attention

} // extern "C"

// ------------------------------------------------------------------ allocation-free entry point
// The scratch of pgf8_fp8_linear_dynamic_noalloc: a fixed array in device
// memory (zero-filled at module load like any static storage).  In host code
// its name is only a host-side stand-in, so its device address is looked up
// once per device with cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) uint8_t g_noalloc_scratch[PGF8_NOALLOC_SCRATCH_BYTES];

namespace pgf8 {
constexpr int kMaxDevices = 64;
static std::mutex g_noalloc_mutex;
static void *g_noalloc_addr[kMaxDevices];

// Device address of the scratch array on the current device (set-up on the
// first call per device, with that device current).
static pgf8_status noalloc_scratch(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices)
        return PGF8_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return cuda_fail(e);
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return PGF8_OK;
}
} // namespace pgf8

extern "C" {

pgf8_status pgf8_fp8_linear_dynamic_noalloc(const void *x, pgf8_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                            const uint8_t *wq, const float *sw, int64_t N, void *y, void *stream)
{
    pgf8_status st = check_dims(M, N, K);
    if (st != PGF8_OK)
        return st;
    const size_t need = pgf8_fp8_linear_dynamic_workspace_size(M, N, K);
    if (need > PGF8_NOALLOC_SCRATCH_BYTES)
        return PGF8_ERR_TOO_LARGE;
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != PGF8_OK)
        return st;
    return pgf8_fp8_linear_dynamic(x, xdt, M, K, ldx, wq, sw, N, y, scratch, need, nullptr, stream);
}

} // extern "C"
