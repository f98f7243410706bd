// fa2_api.cu -- the C ABI of libfa2.so (declared in include/fa2.h): argument
// validation, tensor-map construction and kernel launches for the
// FlashAttention-2 forward and backward passes on sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>

#include <mutex>
#include <utility>
#include <vector>
#include <type_traits>

#include "../../include/fa2.h"
#include "fa2_bwd.cuh"
#include "fa2_bwd_fused.cuh"
#include "fa2_bwd32.cuh"
#include "fa2_fwd.cuh"
#include "fa2_fwd2.cuh"

namespace fa2 {
namespace {

// Per-device status word written by the kernels' pipeline watchdog.
__device__ uint32_t g_device_status;

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
// Whether flags = 0 selects the one-pass backward where it applies (else only
// FA2_BWD_ONE_PASS does).
constexpr bool kOnePassDefault = false;
constexpr int kMaxDevices = 64;
constexpr int kSmCount = 148;   // streaming multiprocessors of a B200
constexpr int kMaxN = 1 << 24;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mutex;
EncodeTiledFn g_encode = nullptr;
uint32_t* g_status_ptr[kMaxDevices] = {};
int g_device_cc[kMaxDevices] = {};  // 0 = not queried yet

fa2_status init_device(int* dev_out, uint32_t** status_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_device_cc[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return FA2_ERR_CUDA;
        g_device_cc[dev] = major * 10 + minor;
    }
    if (g_device_cc[dev] != 100) return FA2_ERR_UNSUPPORTED_DEVICE;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return FA2_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return FA2_ERR_CUDA;
        g_status_ptr[dev] = static_cast<uint32_t*>(p);
    }
    *dev_out = dev;
    *status_out = g_status_ptr[dev];
    return FA2_OK;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream is still finishing (every kernel of
// this library starts with griddepcontrol.launch_dependents and then waits,
// with griddepcontrol.wait, for the previous kernel before touching global
// memory), which hides the launch latency between the kernels of a pass.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

bool head_dim_supported(int d) { return d == 16 || d == 32 || d == 64 || d == 80 || d == 128; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

fa2_status check_common(int B, int H, int N, int d, int causal, float scale, fa2_dtype dtype) {
    if (dtype != FA2_BF16 && dtype != FA2_FP32 && dtype != FA2_FP16) return FA2_ERR_UNSUPPORTED_DTYPE;
    if (B < 1 || H < 1 || N < 1 || N > kMaxN) return FA2_ERR_BAD_SHAPE;
    if (static_cast<long long>(B) * H > (1ll << 31) - 1) return FA2_ERR_BAD_SHAPE;
    const long long tiles = (N + kTileRows - 1) / kTileRows;
    if (tiles * B * H > (1ll << 31) - 1) return FA2_ERR_BAD_SHAPE;
    if (!head_dim_supported(d)) return FA2_ERR_UNSUPPORTED_HEAD_DIM;
    if (causal != 0 && causal != 1) return FA2_ERR_BAD_ARGUMENT;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA2_ERR_BAD_ARGUMENT;
    return FA2_OK;
}

// Tensor maps are encoded on the host for every call; the last few are kept,
// keyed by everything that enters the encoding, so a caller that passes the
// same buffers again (a training loop) skips the driver call.
struct MapKey {
    const void* ptr;
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    int dtype, swizzle;
    bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};
constexpr int kMapCache = 64;
std::mutex g_map_mutex;
MapKey g_map_keys[kMapCache];
CUtensorMap g_map_vals[kMapCache];
int g_map_used = 0, g_map_next = 0;

fa2_status encode_cached(CUtensorMap* m, CUtensorMapDataType type, const void* ptr, const cuuint64_t* dims,
                         const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
    MapKey key;
    std::memset(&key, 0, sizeof(key));
    key.ptr = ptr;
    for (int i = 0; i < 3; ++i) { key.dims[i] = dims[i]; key.box[i] = box[i]; }
    for (int i = 0; i < 2; ++i) key.strides[i] = strides[i];
    key.dtype = static_cast<int>(type);
    key.swizzle = static_cast<int>(sw);
    {
        std::lock_guard<std::mutex> lock(g_map_mutex);
        for (int i = 0; i < g_map_used; ++i)
            if (g_map_keys[i] == key) { *m = g_map_vals[i]; return FA2_OK; }
    }
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, type, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return FA2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_map_mutex);
    g_map_keys[g_map_next] = key;
    g_map_vals[g_map_next] = *m;
    g_map_next = (g_map_next + 1) % kMapCache;
    if (g_map_used < kMapCache) ++g_map_used;
    return FA2_OK;
}

// 3-D view [BH][N][d] of a contiguous [B,H,N,d] tensor, loaded/stored in boxes
// of box_cols x 128 rows x 1 head.
fa2_status make_map(CUtensorMap* m, const void* ptr, fa2_dtype dtype, int d, int N, int BH,
                    int box_cols, int row_bytes, bool mn_major_f32, int box_rows = kTileRows) {
    const int es = dtype == FA2_FP32 ? 4 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * es,
                             static_cast<cuuint64_t>(d) * es * static_cast<cuuint64_t>(N)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    CUtensorMapSwizzle sw = mn_major_f32       ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                            : row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                            : row_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_32B;
    return encode_cached(m,
                         dtype == FA2_BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                         : dtype == FA2_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                         ptr, dims, strides, box, sw);
}

// [BH][n_pad][d] fp32 accumulator, reduce-added in boxes of box_cols columns x
// 128 rows x 1 head whose rows use the swizzle of their width (128 or 64 bytes).
fa2_status make_map_f32_reduce(CUtensorMap* m, void* ptr, int d, int n_pad, int BH, int box_cols) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n_pad),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                             static_cast<cuuint64_t>(d) * 4 * static_cast<cuuint64_t>(n_pad)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(kTileRows), 1};
    const CUtensorMapSwizzle sw = box_cols * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ptr, dims, strides, box, sw);
}

template <int ES, int D>
fa2_status make_maps_kmajor(CUtensorMap* m, const void* ptr, fa2_dtype dtype, int N, int BH) {
    using G = TileGeom<ES, D>;
    return make_map(m, ptr, dtype, D, N, BH, G::kBoxK, G::kRowBK, false);
}

template <int ES, int D>
fa2_status make_maps_mnmajor(CUtensorMap* m, const void* ptr, fa2_dtype dtype, int N, int BH,
                             int box_rows = kTileRows) {
    using G = TileGeom<ES, D>;
    return make_map(m, ptr, dtype, D, N, BH, G::kBoxMN, G::kRowBMN, G::kF32, box_rows);
}

// The dynamic shared memory limit of a kernel is raised once per device.
std::mutex g_attr_mutex;
std::vector<std::pair<const void*, int>> g_attr_done;

template <class Kernel>
fa2_status set_smem(Kernel k, int bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA2_ERR_CUDA;
    const void* fn = reinterpret_cast<const void*>(k);
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    for (const auto& e : g_attr_done)
        if (e.first == fn && e.second == dev) return FA2_OK;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return FA2_ERR_CUDA;
    g_attr_done.emplace_back(fn, dev);
    return FA2_OK;
}

// The two-query-tile forward serves 16-bit inputs, and fp32 (TF32) inputs up to
// d = 64 (its warp 3 rounds their tiles).  fp32 at d = 80 and 128 uses the
// one-tile kernel (two query tiles of fp32 leave too little shared memory).
template <int ES, int D>
constexpr bool use_two_tile_forward() {
    return (ES == 2 || D <= 64) && Fwd2Cfg<ES, D>::kFits;
}

template <int ES, int D, bool F16 = false>
fa2_status launch_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int H, int H_kv, int N, int Nk, int causal, float scale, fa2_dtype dtype,
                          cudaStream_t stream, uint32_t* status, const uint8_t* block_mask = nullptr) {
    using Cfg = FwdCfg<ES, D>;
    const int BH = B * H;
    const int BH_kv = B * H_kv;
    CUtensorMap mq, mk, mv, mo;
    fa2_status st;
    if ((st = make_maps_kmajor<ES, D>(&mq, q, dtype, N, BH)) != FA2_OK) return st;
    if ((st = make_maps_kmajor<ES, D>(&mk, k, dtype, Nk, BH_kv)) != FA2_OK) return st;
    // V in the one-tile kernel arrives in parts of kVPartRows keys.
    constexpr int v_rows = use_two_tile_forward<ES, D>() ? kTileRows : Cfg::kVPartRows;
    if ((st = make_maps_mnmajor<ES, D>(&mv, v, dtype, Nk, BH_kv, v_rows)) != FA2_OK) return st;
    if ((st = make_maps_kmajor<ES, D>(&mo, o, dtype, N, BH)) != FA2_OK) return st;
    FwdParams p;
    p.lse = lse;
    p.status = status;
    p.N = N;
    p.Nk = Nk;
    p.BH = BH;
    p.H = H;
    p.H_kv = H_kv;
    p.group = H / H_kv;
    p.n_tiles = (N + kTileRows - 1) / kTileRows;
    p.n_tiles_k = (Nk + kTileRows - 1) / kTileRows;
    p.causal = causal;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = kDefaultTimeoutNs;
    p.block_mask = block_mask;
    p.q32 = ES == 4 ? static_cast<const float*>(q) : nullptr;
    // Two query tiles per CTA (the softmax of one overlaps the MMAs of the
    // other), unless the pairs would leave SMs idle: then one tile per CTA.
    const long long pair_items = static_cast<long long>((p.n_tiles + 1) / 2) * BH;
    p.one_tile = pair_items < kSmCount ? 1 : 0;
    const int n_items = p.one_tile ? p.n_tiles : (p.n_tiles + 1) / 2;
    p.head_group = heads_per_group(BH, n_items);
    if constexpr (use_two_tile_forward<ES, D>()) {
        using Cfg2 = Fwd2Cfg<ES, D, F16>;
        auto kern = block_mask ? fa2_fwd2_kernel<ES, D, F16, true> : fa2_fwd2_kernel<ES, D, F16, false>;
        if ((st = set_smem(kern, Cfg2::kSmemBytes)) != FA2_OK) return st;
        launch_pdl(kern, dim3(static_cast<unsigned>(n_items) * static_cast<unsigned>(BH)), dim3(Cfg2::kThreads), Cfg2::kSmemBytes, stream, mq, mk, mv, mo, p);
    } else {
        auto kern = block_mask ? fa2_fwd_kernel<ES, D, true> : fa2_fwd_kernel<ES, D, false>;
        if ((st = set_smem(kern, Cfg::kSmemBytes)) != FA2_OK) return st;
        const unsigned grid = static_cast<unsigned>(p.n_tiles) * static_cast<unsigned>(BH);
        launch_pdl(kern, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, mq, mk, mv, mo, p);
    }
    return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_CUDA;
}

template <int ES, bool F16 = false>
fa2_status dispatch_forward(int d, const void* q, const void* k, const void* v, void* o,
                            float* lse, int B, int H, int H_kv, int N, int Nk, int causal, float scale,
                            fa2_dtype dtype, cudaStream_t stream, uint32_t* status,
                            const uint8_t* block_mask = nullptr) {
    switch (d) {
        case 16: return launch_forward<ES, 16, F16>(q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, stream, status, block_mask);
        case 32: return launch_forward<ES, 32, F16>(q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, stream, status, block_mask);
        case 64: return launch_forward<ES, 64, F16>(q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, stream, status, block_mask);
        case 80: return launch_forward<ES, 80, F16>(q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, stream, status, block_mask);
        case 128: return launch_forward<ES, 128, F16>(q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, stream, status, block_mask);
        default: return FA2_ERR_UNSUPPORTED_HEAD_DIM;
    }
}

template <int ES, int D, bool F16 = false>
fa2_status launch_backward_t(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int B, int H, int H_kv, int N, int Nk, int causal, float scale, fa2_dtype dtype,
                             uint8_t* ws_base, const BwdWorkspace& ws, cudaStream_t stream,
                             uint32_t* status, unsigned long long timeout_ns,
                             void* const* events, const uint8_t* block_mask, unsigned flags) {
    using T = typename std::conditional<ES == 2, uint16_t, float>::type;
    using Cfg = BwdCfg<ES, D, F16>;
    // One pass (key tiles outer, dQ by fp32 reduce-add) where it applies and the
    // caller did not ask for the bitwise-reproducible two-pass form.
    const bool want_one = (flags & FA2_BWD_ONE_PASS) || (kOnePassDefault && !(flags & FA2_BWD_DETERMINISTIC));
    const bool one_pass = want_one && ws.dqacc_off != 0 &&
                          one_pass_applies((Nk + kTileRows - 1) / kTileRows, ES, ws.kv_splits, block_mask != nullptr);
    float* dq_acc = one_pass ? reinterpret_cast<float*>(ws_base + ws.dqacc_off) : nullptr;
    auto mark = [&](int i) -> bool {
        if (!events || !events[i]) return true;
        return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream) == cudaSuccess;
    };
    const int BH = B * H;
    float* l2 = reinterpret_cast<float*>(ws_base + ws.l2_off);
    float* dvec = reinterpret_cast<float*>(ws_base + ws.d_off);
    fa2_status st;
    // 1. D and log2-scaled L.
    const long long rows = static_cast<long long>(BH) * ws.n_pad;
    if (!mark(0)) return FA2_ERR_CUDA;
    constexpr int kPreRows = BwdPreCfg<D>::kRowsPerBlock;
    launch_pdl(fa2_bwd_pre_kernel<D, F16>, dim3(static_cast<unsigned>((rows + kPreRows - 1) / kPreRows)), dim3(256), 0, stream, 
        static_cast<const T*>(o), static_cast<const T*>(dout), lse, l2, dvec, N, ws.n_pad, rows, dq_acc);
    if (cudaGetLastError() != cudaSuccess || !mark(1)) return FA2_ERR_CUDA;
    CUtensorMap mq, mk, mv, mdo, mdk, mdv, mdq;
    if ((st = make_maps_kmajor<ES, D>(&mq, q, dtype, N, BH)) != FA2_OK) return st;
    const int BH_kv = B * H_kv;
    if ((st = make_maps_kmajor<ES, D>(&mk, k, dtype, Nk, BH_kv)) != FA2_OK) return st;
    if ((st = make_maps_kmajor<ES, D>(&mv, v, dtype, Nk, BH_kv)) != FA2_OK) return st;
    if ((st = make_maps_kmajor<ES, D>(&mdo, dout, dtype, N, BH)) != FA2_OK) return st;
    if ((st = make_maps_kmajor<ES, D>(&mdk, dk, dtype, Nk, BH_kv)) != FA2_OK) return st;
    if ((st = make_maps_kmajor<ES, D>(&mdv, dv, dtype, Nk, BH_kv)) != FA2_OK) return st;
    if ((st = make_maps_kmajor<ES, D>(&mdq, dq, dtype, N, BH)) != FA2_OK) return st;
    BwdParams p;
    p.k32 = p.q32 = p.do32 = nullptr;
    p.l2 = l2;
    p.dvec = dvec;
    p.status = status;
    p.N = N;
    p.Nk = Nk;
    p.BH = BH;
    p.H = H;
    p.H_kv = H_kv;
    p.group = H / H_kv;
    p.BH_kv = B * H_kv;
    p.n_tiles = (N + kTileRows - 1) / kTileRows;
    p.n_tiles_k = (Nk + kTileRows - 1) / kTileRows;
    p.n_pad = ws.n_pad;
    p.causal = causal;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.scale = scale;
    p.timeout_ns = timeout_ns;
    p.block_mask = block_mask;
    p.kv_splits = ws.kv_splits;
    p.part = ws.kv_splits > 1 ? reinterpret_cast<float*>(ws_base + ws.part_off) : nullptr;
    p.item0 = 0;
    // Work items in groups of heads (grouped_item), set per launch below.
    const int hg_q = heads_per_group(BH, p.n_tiles);                        // query-tile pass
    const int hg_kv = heads_per_group(p.BH_kv * p.kv_splits, p.n_tiles_k);  // key-tile passes
    if (one_pass) {
        // 2. dQ and D of the query tiles whose rows see a single key tile (causal:
        // query tile 0 of every head, the pass's last BH work items).
        if (causal) {
            auto kern = fa2_bwd_dq_kernel<ES, D, F16, false>;
            if ((st = set_smem(kern, Cfg::kDqSmemBytes)) != FA2_OK) return st;
            p.item0 = (p.n_tiles - 1) * BH;   // the last BH items of the plain order
            p.head_group = BH;
            launch_pdl(kern, dim3(static_cast<unsigned>(BH)), dim3(Cfg::kThreadsDq), Cfg::kDqSmemBytes, stream, mq, mk, mv, mdo, mdq, p);
            p.item0 = 0;
            if (cudaGetLastError() != cudaSuccess) return FA2_ERR_CUDA;
        }
        if (!mark(2)) return FA2_ERR_CUDA;
        // 3. dK, dV and the other query tiles' dQ in one key-tile-outer pass, then
        // dQ = scale * dQ_acc rounded once.
        using FC = BwdFusedCfg<ES, D, F16>;
        auto kern = fa2_bwd_fused_kernel<ES, D, F16>;
        p.head_group = hg_kv;
        if ((st = set_smem(kern, FC::kSmemBytes)) != FA2_OK) return st;
        const unsigned grid_f = static_cast<unsigned>(p.n_tiles_k) * static_cast<unsigned>(p.BH_kv);
        CUtensorMap macc;
        if ((st = make_map_f32_reduce(&macc, dq_acc, D, ws.n_pad, BH, FC::kCW)) != FA2_OK) return st;
        launch_pdl(kern, dim3(grid_f), dim3(FC::kThreads), FC::kSmemBytes, stream, mq, mk, mv, mdo, mdk, mdv, macc, p);
        if (cudaGetLastError() != cudaSuccess || !mark(3)) return FA2_ERR_CUDA;
        const long long groups8 = static_cast<long long>(BH) * N * D / 8;
        launch_pdl(fa2_bwd_dq_finalize_kernel<F16>, dim3(static_cast<unsigned>((groups8 + 255) / 256)), dim3(256), 0, stream, 
            dq_acc, static_cast<uint16_t*>(dq), N, ws.n_pad, D, groups8, causal ? kTileRows : 0, scale);
        if (cudaGetLastError() != cudaSuccess) return FA2_ERR_CUDA;
        return FA2_OK;
    }
    // dK/dV pass: kv_splits CTAs per (key tile, key/value head); dQ pass: one per
    // (query tile, query head).
    const unsigned grid_kv = static_cast<unsigned>(p.n_tiles_k) * static_cast<unsigned>(p.BH_kv) *
                             static_cast<unsigned>(p.kv_splits);
    const unsigned grid = static_cast<unsigned>(p.n_tiles) * static_cast<unsigned>(BH);
    // 2. dQ: query-tile-outer pass.  It runs first because a query tile that sees
    // a single key tile rewrites its rows' D (formed there from P and dP), which
    // the dK/dV pass then reads.
    {
        auto kern = block_mask ? fa2_bwd_dq_kernel<ES, D, F16, true> : fa2_bwd_dq_kernel<ES, D, F16, false>;
        if ((st = set_smem(kern, Cfg::kDqSmemBytes)) != FA2_OK) return st;
        p.head_group = hg_q;
        launch_pdl(kern, dim3(grid), dim3(Cfg::kThreadsDq), Cfg::kDqSmemBytes, stream, mq, mk, mv, mdo, mdq, p);
        if (cudaGetLastError() != cudaSuccess || !mark(2)) return FA2_ERR_CUDA;
    }
    // 3. dK, dV: key/value-tile-outer pass (+ the sum of a split group's partials).
    {
        auto kern = block_mask ? fa2_bwd_dkdv_kernel<ES, D, F16, true> : fa2_bwd_dkdv_kernel<ES, D, F16, false>;
        if ((st = set_smem(kern, Cfg::kSmemBytes)) != FA2_OK) return st;
        p.head_group = hg_kv;
        launch_pdl(kern, dim3(grid_kv), dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, mq, mk, mv, mdo, mdk, mdv, p);
        if (cudaGetLastError() != cudaSuccess) return FA2_ERR_CUDA;
        if (p.kv_splits > 1) {
            const size_t groups4 = 2 * static_cast<size_t>(p.BH_kv) * Nk * D / 4;
            launch_pdl(fa2_bwd_kv_reduce_kernel<F16>, dim3(static_cast<unsigned>((groups4 + 255) / 256)), dim3(256), 0, stream, 
                p.part, static_cast<uint16_t*>(dk), static_cast<uint16_t*>(dv), p.kv_splits, p.BH_kv, Nk,
                p.n_tiles_k * kTileRows, D, scale);
            if (cudaGetLastError() != cudaSuccess) return FA2_ERR_CUDA;
        }
        if (!mark(3)) return FA2_ERR_CUDA;
    }
    return FA2_OK;
}

// fp32 inputs: TF32 kernels whose streamed operands arrive in sub-tiles of
// W rows and, where a contraction runs over rows, in a second (MN-major) copy.
template <int D>
fa2_status launch_backward32_t(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv,
                               int B, int H, int H_kv, int N, int Nk, int causal, float scale, uint8_t* ws_base,
                               const BwdWorkspace& ws, cudaStream_t stream, uint32_t* status,
                               unsigned long long timeout_ns, void* const* events,
                               const uint8_t* block_mask) {
    using Cfg = Bwd32Cfg<D>;
    using G = typename Cfg::G;
    constexpr fa2_dtype dt = FA2_FP32;
    auto mark = [&](int i) -> bool {
        if (!events || !events[i]) return true;
        return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream) == cudaSuccess;
    };
    const int BH = B * H;
    float* l2 = reinterpret_cast<float*>(ws_base + ws.l2_off);
    float* dvec = reinterpret_cast<float*>(ws_base + ws.d_off);
    fa2_status st;
    const long long rows = static_cast<long long>(BH) * ws.n_pad;
    if (!mark(0)) return FA2_ERR_CUDA;
    // TF32-rounded copies of the operands; every tensor map below reads those.
    float* qr = reinterpret_cast<float*>(ws_base + ws.q_off);
    float* kr = reinterpret_cast<float*>(ws_base + ws.k_off);
    float* vr = reinterpret_cast<float*>(ws_base + ws.v_off);
    float* dor = reinterpret_cast<float*>(ws_base + ws.do_off);
    launch_pdl(fa2_bwd32_pre_kernel<D>, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, stream, 
        static_cast<const float*>(q), static_cast<const float*>(o), static_cast<const float*>(dout),
        lse, qr, dor, l2, dvec, N, ws.n_pad, rows);
    const size_t kv4 = static_cast<size_t>(B) * H_kv * Nk * D / 4;  // D is a multiple of 4
    const unsigned round_grid = static_cast<unsigned>((kv4 + 255) / 256 < 4096 ? (kv4 + 255) / 256 : 4096);
    launch_pdl(fa2_round_tf32_kernel, dim3(round_grid), dim3(256), 0, stream, static_cast<const float4*>(k), reinterpret_cast<float4*>(kr), kv4);
    launch_pdl(fa2_round_tf32_kernel, dim3(round_grid), dim3(256), 0, stream, static_cast<const float4*>(v), reinterpret_cast<float4*>(vr), kv4);
    if (cudaGetLastError() != cudaSuccess || !mark(1)) return FA2_ERR_CUDA;
    q = qr;
    k = kr;
    v = vr;
    dout = dor;
    // q, dout, dq have B*H heads; k, v, dk, dv B*H_kv.
    const int BH_kv = B * H_kv;
    // Query-side tensors (q, dout, dq): B*H heads of N rows; key-side (k, v, dk, dv): B*H_kv of Nk.
    auto kmap = [&](CUtensorMap* m, const void* ptr, int box_rows, int heads, int rows) {
        return make_map(m, ptr, dt, D, rows, heads, G::kBoxK, G::kRowBK, false, box_rows);
    };
    auto mnmap = [&](CUtensorMap* m, const void* ptr, int box_rows, int heads, int rows) {
        return make_map(m, ptr, dt, D, rows, heads, G::kBoxMN, G::kRowBMN, true, box_rows);
    };
    BwdParams p;
    p.l2 = l2;
    p.dvec = dvec;
    p.status = status;
    p.N = N;
    p.Nk = Nk;
    p.BH = BH;
    p.H = H;
    p.H_kv = H_kv;
    p.group = H / H_kv;
    p.BH_kv = BH_kv;
    p.n_tiles = (N + kTileRows - 1) / kTileRows;
    p.n_tiles_k = (Nk + kTileRows - 1) / kTileRows;
    p.n_pad = ws.n_pad;
    p.causal = causal;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.scale = scale;
    p.timeout_ns = timeout_ns;
    p.block_mask = block_mask;
    p.kv_splits = 1;                                     // fp32: one CTA per group
    p.k32 = kr;
    p.q32 = qr;
    p.do32 = dor;
    p.part = nullptr;
    p.item0 = 0;
    p.head_group = 1;
    // dK/dV pass: one CTA per (key tile, key/value head); dQ pass: per (query tile, query head).
    const unsigned grid_kv = static_cast<unsigned>(p.n_tiles_k) * static_cast<unsigned>(p.BH_kv);
    const unsigned grid = static_cast<unsigned>(p.n_tiles) * static_cast<unsigned>(BH);
    // dQ pass first, then dK/dV (the order of the 16-bit path).
    {
        constexpr int W = Cfg::kWq;
        CUtensorMap mq, mdo, mkk, mkmn, mvk, mdq;
        if ((st = kmap(&mq, q, kTileRows, BH, N)) != FA2_OK || (st = kmap(&mdo, dout, kTileRows, BH, N)) != FA2_OK ||
            (st = kmap(&mkk, k, W, BH_kv, Nk)) != FA2_OK || (st = mnmap(&mkmn, k, W, BH_kv, Nk)) != FA2_OK ||
            (st = kmap(&mvk, v, W, BH_kv, Nk)) != FA2_OK || (st = kmap(&mdq, dq, kTileRows, BH, N)) != FA2_OK)
            return st;
        auto kern = block_mask ? fa2_bwd32_dq_kernel<D, true> : fa2_bwd32_dq_kernel<D, false>;
        if ((st = set_smem(kern, Cfg::kSmemQ)) != FA2_OK) return st;
        launch_pdl(kern, dim3(grid), dim3(Cfg::kThreadsQ), Cfg::kSmemQ, stream, mq, mdo, mkk, mkmn, mvk, mdq, p);
        if (cudaGetLastError() != cudaSuccess || !mark(2)) return FA2_ERR_CUDA;
    }
    {
        constexpr int W = Cfg::kWkv;
        CUtensorMap mqk, mqmn, mk, mv, mdok, mdomn, mdk, mdv;
        if ((st = kmap(&mqk, q, W, BH, N)) != FA2_OK || (st = mnmap(&mqmn, q, W, BH, N)) != FA2_OK ||
            (st = kmap(&mk, k, kTileRows, BH_kv, Nk)) != FA2_OK || (st = kmap(&mv, v, kTileRows, BH_kv, Nk)) != FA2_OK ||
            (st = kmap(&mdok, dout, W, BH, N)) != FA2_OK || (st = mnmap(&mdomn, dout, W, BH, N)) != FA2_OK ||
            (st = kmap(&mdk, dk, kTileRows, BH_kv, Nk)) != FA2_OK || (st = kmap(&mdv, dv, kTileRows, BH_kv, Nk)) != FA2_OK)
            return st;
        auto kern = block_mask ? fa2_bwd32_dkdv_kernel<D, true> : fa2_bwd32_dkdv_kernel<D, false>;
        if ((st = set_smem(kern, Cfg::kSmemKV)) != FA2_OK) return st;
        launch_pdl(kern, dim3(grid_kv), dim3(Cfg::kThreadsKV), Cfg::kSmemKV, stream, mqk, mqmn, mk, mv, mdok, mdomn, mdk, mdv, p);
        if (cudaGetLastError() != cudaSuccess || !mark(3)) return FA2_ERR_CUDA;
    }
    return FA2_OK;
}

fa2_status launch_backward(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                           int H, int H_kv, int N, int Nk, int d, int causal, float scale, fa2_dtype dtype,
                           uint8_t* ws_base, const BwdWorkspace& ws, cudaStream_t stream,
                           uint32_t* status, unsigned long long timeout_ns, void* const* events,
                           const uint8_t* block_mask, unsigned flags) {
#define FA2_BWD_CASE(DD)                                                                      \
    case DD:                                                                                  \
        if (dtype == FA2_FP32)                                                                \
            return launch_backward32_t<DD>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, Nk, causal, \
                                           scale, ws_base, ws, stream, status, timeout_ns, events, \
                                           block_mask);                                  \
        if (dtype == FA2_FP16)                                                                \
            return launch_backward_t<2, DD, true>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, Nk, \
                                                  causal, scale, dtype, ws_base, ws, stream,    \
                                                  status, timeout_ns, events, block_mask,       \
                                                  flags);                                       \
        return launch_backward_t<2, DD>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, Nk, causal, \
                                        scale, dtype, ws_base, ws, stream, status, timeout_ns, events, \
                                        block_mask, flags);
    switch (d) {
        FA2_BWD_CASE(16)
        FA2_BWD_CASE(32)
        FA2_BWD_CASE(64)
        FA2_BWD_CASE(80)
        FA2_BWD_CASE(128)
        default: return FA2_ERR_UNSUPPORTED_HEAD_DIM;
    }
#undef FA2_BWD_CASE
}

}  // namespace
}  // namespace fa2

using namespace fa2;

namespace fa2 {
namespace {

fa2_status check_heads(int H, int H_kv) {
    return (H_kv >= 1 && H_kv <= H && H % H_kv == 0) ? FA2_OK : FA2_ERR_BAD_SHAPE;
}

// Key/value length: the same bounds as the query length.
fa2_status check_keys(int B, int H_kv, int Nk) {
    if (Nk < 1 || Nk > kMaxN) return FA2_ERR_BAD_SHAPE;
    const long long tiles = (Nk + kTileRows - 1) / kTileRows;
    if (tiles * B * H_kv > (1ll << 31) - 1) return FA2_ERR_BAD_SHAPE;
    return FA2_OK;
}

fa2_status forward_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                        fa2_dtype dtype, fa2_stream_t stream, const uint8_t* block_mask = nullptr) {
    fa2_status st = check_common(B, H, N, d, causal, scale, dtype);
    if (st != FA2_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA2_OK) return st;
    if ((st = check_keys(B, H_kv, Nk)) != FA2_OK) return st;
    if (!q || !k || !v || !o || !lse) return FA2_ERR_NULL_PTR;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(lse, 4))
        return FA2_ERR_MISALIGNED;
    int dev;
    uint32_t* status;
    if ((st = init_device(&dev, &status)) != FA2_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == FA2_BF16)
        return dispatch_forward<2>(d, q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, s, status,
                                   block_mask);
    if (dtype == FA2_FP16)
        return dispatch_forward<2, true>(d, q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, s,
                                         status, block_mask);
    return dispatch_forward<4>(d, q, k, v, o, lse, B, H, H_kv, N, Nk, causal, scale, dtype, s, status,
                               block_mask);
}

fa2_status backward_impl(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                         int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                         fa2_dtype dtype, void* workspace, size_t workspace_bytes,
                         fa2_stream_t stream, void* const* events, const uint8_t* block_mask = nullptr,
                         unsigned flags = 0) {
    fa2_status st = check_common(B, H, N, d, causal, scale, dtype);
    if (st != FA2_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA2_OK) return st;
    if ((st = check_keys(B, H_kv, Nk)) != FA2_OK) return st;
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
        return FA2_ERR_NULL_PTR;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4) || !aligned(workspace, 256))
        return FA2_ERR_MISALIGNED;
    // The two-pass form needs no dQ accumulator, so it accepts the smaller workspace.
    const bool two_pass_only = (flags & FA2_BWD_DETERMINISTIC) ||
                               (!kOnePassDefault && !(flags & FA2_BWD_ONE_PASS)) || block_mask;
    const BwdWorkspace ws = bwd_workspace_layout(B * H, N, B * H_kv, Nk, d, dtype == FA2_FP32 ? 4 : 2,
                                                 !two_pass_only);
    if (workspace_bytes < ws.total) return FA2_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    uint32_t* status;
    if ((st = init_device(&dev, &status)) != FA2_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return launch_backward(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, Nk, d, causal, scale,
                           dtype, static_cast<uint8_t*>(workspace), ws, s, status,
                           kDefaultTimeoutNs, events, block_mask, flags);
}

}  // namespace
}  // namespace fa2

extern "C" {

fa2_status fa2_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int N, int d, int causal, float scale, fa2_dtype dtype,
                       fa2_stream_t stream) {
    return forward_impl(q, k, v, o, lse, B, H, H, N, N, d, causal, scale, dtype, stream);
}

fa2_status fa2_forward_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                          fa2_dtype dtype, fa2_stream_t stream) {
    return forward_impl(q, k, v, o, lse, B, H, H_kv, N, Nk, d, causal, scale, dtype, stream);
}

size_t fa2_backward_workspace_bytes(int B, int H, int N, int d, fa2_dtype dtype) {
    if (check_common(B, H, N, d, 0, 1.f, dtype) != FA2_OK) return 0;
    return bwd_workspace_layout(B * H, N, B * H, N, d, dtype == FA2_FP32 ? 4 : 2).total;
}

size_t fa2_backward_workspace_bytes_ex(int B, int H, int H_kv, int N, int Nk, int d,
                                       fa2_dtype dtype) {
    if (check_common(B, H, N, d, 0, 1.f, dtype) != FA2_OK || check_heads(H, H_kv) != FA2_OK ||
        check_keys(B, H_kv, Nk) != FA2_OK)
        return 0;
    return bwd_workspace_layout(B * H, N, B * H_kv, Nk, d, dtype == FA2_FP32 ? 4 : 2).total;
}

fa2_status fa2_backward_timed(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dout, void* dq, void* dk, void* dv,
                              int B, int H, int N, int d, int causal, float scale,
                              fa2_dtype dtype, void* workspace, size_t workspace_bytes,
                              fa2_stream_t stream, void* const* events) {
    return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, N, d, causal, scale, dtype,
                         workspace, workspace_bytes, stream, events);
}

fa2_status fa2_backward(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                        int H, int N, int d, int causal, float scale, fa2_dtype dtype,
                        void* workspace, size_t workspace_bytes, fa2_stream_t stream) {
    return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, N, d, causal, scale, dtype,
                         workspace, workspace_bytes, stream, nullptr);
}

fa2_status fa2_backward_ex(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                           int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                           fa2_dtype dtype, void* workspace, size_t workspace_bytes,
                           fa2_stream_t stream) {
    return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, Nk, d, causal, scale,
                         dtype, workspace, workspace_bytes, stream, nullptr);
}

fa2_status fa2_forward_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                                    int B, int H, int H_kv, int N, int Nk, int d, int causal,
                                    float scale, fa2_dtype dtype, const uint8_t* block_mask,
                                    fa2_stream_t stream) {
    if (!block_mask) return FA2_ERR_NULL_PTR;
    return forward_impl(q, k, v, o, lse, B, H, H_kv, N, Nk, d, causal, scale, dtype, stream,
                        block_mask);
}

fa2_status fa2_backward_block_sparse(const void* q, const void* k, const void* v, const void* o,
                                     const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                     int B, int H, int H_kv, int N, int Nk, int d, int causal,
                                     float scale, fa2_dtype dtype, const uint8_t* block_mask,
                                     void* workspace, size_t workspace_bytes, fa2_stream_t stream) {
    if (!block_mask) return FA2_ERR_NULL_PTR;
    return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, Nk, d, causal, scale,
                         dtype, workspace, workspace_bytes, stream, nullptr, block_mask);
}

fa2_status fa2_backward_opts(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int B, int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                             fa2_dtype dtype, const uint8_t* block_mask, unsigned flags,
                             void* workspace, size_t workspace_bytes, fa2_stream_t stream) {
    if ((flags & ~(FA2_BWD_DETERMINISTIC | FA2_BWD_ONE_PASS)) ||
        ((flags & FA2_BWD_DETERMINISTIC) && (flags & FA2_BWD_ONE_PASS)))
        return FA2_ERR_BAD_ARGUMENT;
    return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, Nk, d, causal, scale,
                         dtype, workspace, workspace_bytes, stream, nullptr, block_mask, flags);
}

fa2_status fa2_last_device_status(void) {
    int dev;
    uint32_t* status;
    fa2_status st = init_device(&dev, &status);
    if (st != FA2_OK) return st;
    uint32_t v = 0;
    if (cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FA2_ERR_CUDA;
    return static_cast<fa2_status>(v);
}

fa2_status fa2_clear_device_status(void) {
    int dev;
    uint32_t* status;
    fa2_status st = init_device(&dev, &status);
    if (st != FA2_OK) return st;
    const uint32_t zero = 0;
    if (cudaMemcpy(status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return FA2_ERR_CUDA;
    return FA2_OK;
}

const char* fa2_status_string(fa2_status status) {
    switch (status) {
        case FA2_OK: return "FA2_OK";
        case FA2_ERR_NULL_PTR: return "FA2_ERR_NULL_PTR: a required pointer is NULL";
        case FA2_ERR_BAD_SHAPE: return "FA2_ERR_BAD_SHAPE: B, H or N out of range";
        case FA2_ERR_UNSUPPORTED_HEAD_DIM: return "FA2_ERR_UNSUPPORTED_HEAD_DIM: d must be 16, 32, 64, 80 or 128";
        case FA2_ERR_UNSUPPORTED_DTYPE: return "FA2_ERR_UNSUPPORTED_DTYPE: dtype must be FA2_BF16, FA2_FP32 or FA2_FP16";
        case FA2_ERR_MISALIGNED: return "FA2_ERR_MISALIGNED: tensors need 16-byte, lse 4-byte, workspace 256-byte alignment";
        case FA2_ERR_WORKSPACE_TOO_SMALL: return "FA2_ERR_WORKSPACE_TOO_SMALL: see fa2_backward_workspace_bytes";
        case FA2_ERR_CUDA: return "FA2_ERR_CUDA: a CUDA call or kernel launch failed";
        case FA2_ERR_DEVICE_TIMEOUT: return "FA2_ERR_DEVICE_TIMEOUT: a kernel pipeline wait expired";
        case FA2_ERR_UNSUPPORTED_DEVICE: return "FA2_ERR_UNSUPPORTED_DEVICE: needs an sm_100 (B200) device";
        case FA2_ERR_BAD_ARGUMENT: return "FA2_ERR_BAD_ARGUMENT: causal must be 0/1, scale finite and > 0, a watchdog limit in [1e3, 1e10] ns";
        case FA2_ERR_SCRATCH_TOO_SMALL: return "FA2_ERR_SCRATCH_TOO_SMALL: the problem needs more than the 64 MiB built-in scratch of fa2_backward_noalloc; use fa2_backward with a workspace";
    }
    return "unknown fa2_status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fa2_backward_noalloc: the backward pass with its scratch in a fixed device
// array, for callers that cannot allocate device memory (see fa2.h).

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, not a device address: the address is looked up per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
unsigned char* g_noalloc_ptr[fa2::kMaxDevices] = {};

// Device address of the scratch array on the current device `dev`, looked up
// once per device (with that device current) and cached.
fa2_status noalloc_scratch(int dev, unsigned char** out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return FA2_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return FA2_OK;
}

}  // namespace

extern "C" fa2_status fa2_backward_noalloc(const void* q, const void* k, const void* v,
                                           const void* o, const float* lse, const void* dout,
                                           void* dq, void* dk, void* dv, int B, int H, int N,
                                           int d, int causal, float scale, fa2_dtype dtype,
                                           fa2_stream_t stream) {
    fa2_status st = check_common(B, H, N, d, causal, scale, dtype);
    if (st != FA2_OK) return st;
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA2_ERR_NULL_PTR;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4))
        return FA2_ERR_MISALIGNED;
    // The two-pass (deterministic) form: its scratch holds no dQ accumulator.
    const BwdWorkspace ws = bwd_workspace_layout(B * H, N, B * H, N, d, dtype == FA2_FP32 ? 4 : 2, false);
    if (ws.total > kNoAllocScratchBytes) return FA2_ERR_SCRATCH_TOO_SMALL;
    int dev;
    uint32_t* status;
    if ((st = init_device(&dev, &status)) != FA2_OK) return st;
    unsigned char* scratch = nullptr;
    if ((st = noalloc_scratch(dev, &scratch)) != FA2_OK) return st;
    return launch_backward(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, N, d, causal, scale, dtype,
                           scratch, ws, reinterpret_cast<cudaStream_t>(stream), status,
                           kDefaultTimeoutNs, nullptr, nullptr, FA2_BWD_DETERMINISTIC);
}

// ---------------------------------------------------------------------------
// fa2_watchdog_selftest: proves on the running device that a pipeline wait
// which is never satisfied ends after its limit and is reported through the
// status word (see fa2.h), without faulting or hanging the GPU.

namespace fa2 {

constexpr unsigned long long kSelftestMinNs = 1000ull;            // 1 us
constexpr unsigned long long kSelftestMaxNs = 10000000000ull;     // 10 s

// One warp.  Thread 0 sets up an mbarrier that expects one arrival, which no
// thread ever makes, and waits for its first phase with the same bounded wait
// the attention kernels use; on expiry it records the timeout exactly as they
// do.  Nothing else is touched.
__global__ void __launch_bounds__(32, 1)
fa2_watchdog_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ volatile uint32_t abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        const bool done = ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns);
        if (!done && abort_flag) atomicCAS(status, 0u, kDevStatusTimeout);
    }
}

}  // namespace fa2

extern "C" fa2_status fa2_watchdog_selftest(unsigned long long limit_ns, fa2_stream_t stream) {
    if (limit_ns < kSelftestMinNs || limit_ns > kSelftestMaxNs) return FA2_ERR_BAD_ARGUMENT;
    int dev;
    uint32_t* status;
    fa2_status st = init_device(&dev, &status);
    if (st != FA2_OK) return st;
    fa2_watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status,
                                                                                      limit_ns);
    return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_CUDA;
}
