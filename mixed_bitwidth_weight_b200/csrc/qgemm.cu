// C-ABI entry points of the qgemm library (see include/qgemm.h).
//
// This file is the library's only translation unit: it includes the kernels,
// validates every argument on the host before anything is launched, sizes the
// launches for the current device and maps CUDA failures to qgemm_status.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>
#include <cmath>

#include "common.cuh"
#include "gemv.cuh"
#include "gemv_int.cuh"
#include "gemm.cuh"
#include "quantize.cuh"
#include "kv_cache.cuh"

namespace {

using namespace qg;

constexpr int kVersion = 100;  // 0.1.0

struct DeviceInfo {
    int sms = 0;
    bool gemv_attr[2] = {false, false};
    bool int_attr[3] = {false, false, false};
    bool gemm_attr[2] = {false, false};
    bool quant_attr = false;
};

DeviceInfo g_devs[64];
std::mutex g_dev_mu;

int current_device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QGEMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_devs[dev];
    if (d.sms == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return QGEMM_ERR_CUDA;
        d.sms = sms;
    }
    *out = &d;
    return QGEMM_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int K, int N) {
    if (K <= 0 || K % kBlockRows != 0 || K > kMaxK) return QGEMM_ERR_SHAPE;
    if (N <= 0 || N % 8 != 0 || N > (1 << 24)) return QGEMM_ERR_SHAPE;
    return QGEMM_OK;
}

int check_rows(int K, int64_t qw_rows) {
    const int64_t nb = K / kBlockRows;
    if (qw_rows < 2 * nb || qw_rows > 8 * nb) return QGEMM_ERR_SHAPE;
    return QGEMM_OK;
}

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QGEMM_OK : QGEMM_ERR_CUDA;
}

// ------------------------------------------------------------------ GEMV
int gemv_mt(int M) { return M <= 8 ? 1 : 2; }
int gemv_tiles(int N) { return (N + kGemvTileCols - 1) / kGemvTileCols; }
int gemv_groups(int K) { return (K / kBlockRows + kGemvGroupBlocks - 1) / kGemvGroupBlocks; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Every kernel family keeps its tickets (per-tile counters that read zero when
// a call starts and are zero again when it completes) in one leading region of
// the workspace that no family writes data into, sized for the family with the
// most tiles.  Calls of different families (a tuned choice, the autotuner's
// candidates) can then share one workspace.
int64_t gemm_tiles_of(int M, int N);
size_t ticket_region(int M, int N) {
    return align_up((size_t)std::max<int64_t>(gemv_tiles(N), gemm_tiles_of(M, N)) * 4, 256);
}

size_t gemv_fixed_smem(int nb) {
    size_t o = align_up((size_t)(nb + 1) * 4, 16) + 2 * kGemvSlots * 8 + 2 * kGemvAStages * 8 + 2 * 2 * 8 + 8 + 128;
    return align_up(o, 128);
}

// Largest grid the GEMV may use (bounds the workspace).
int64_t gemv_max_grid(int K, int N, int sms) {
    const int64_t U = (int64_t)gemv_tiles(N) * gemv_groups(K);
    return std::min<int64_t>(U, (int64_t)4 * sms);
}

// Workspace: [tickets][partial slots][activation records][row shifts].
struct GemvWs {
    size_t tickets, slots, xdec, xshift, total;
};

GemvWs gemv_ws_layout(int M, int K, int N, int sms) {
    const int mp = gemv_mt(M) * 8;
    const int nb = K / kBlockRows;
    GemvWs w;
    w.tickets = 0;
    w.slots = ticket_region(M, N);
    w.xdec = w.slots + align_up((size_t)gemv_max_grid(K, N, sms) * 2 * mp * kGemvTileCols * 4, 256);
    w.xshift = w.xdec + align_up((size_t)(nb + 8) * 64 * mp, 256);
    w.total = w.xshift + 256;
    return w;
}

struct GemvPlan {
    int grid = 0, ring = 0, span_cap = 0;
    size_t smem = 0;
};

// One CTA per SM (each holds all 512 TMEM columns).  Every CTA's cost share
// must hold a whole unit (<= 32 word rows + 1 scale row) so that no CTA's
// range is empty: the reduction relies on it.
int plan_gemv(int M, int K, int N, int64_t qw_rows, int sms, GemvPlan* plan) {
    const int nb = K / kBlockRows;
    const int64_t U = (int64_t)gemv_tiles(N) * gemv_groups(K);
    const int64_t C = (int64_t)gemv_tiles(N) * (qw_rows + gemv_groups(K));
    const int64_t gcap = std::max<int64_t>(1, C / (8 * kGemvGroupBlocks + 2));
    const int64_t G = std::min<int64_t>(std::min<int64_t>(U, gcap), sms);
    const size_t fixed = gemv_fixed_smem(nb);
    const size_t budget = (size_t)227 * 1024;
    if (fixed + (size_t)kGemvMinRing * kGemvRowBytes > budget) return QGEMM_ERR_UNSUPPORTED;
    const int ring = (int)std::min<size_t>(kGemvMaxRing, (budget - fixed) / kGemvRowBytes);
    plan->grid = (int)G;
    plan->ring = ring;
    plan->span_cap = 0;
    plan->smem = fixed + (size_t)ring * kGemvRowBytes;
    return QGEMM_OK;
}

int run_gemv(const void* x, int x_dtype, const int32_t* perm, const uint32_t* qw, int64_t qw_rows,
             const uint16_t* scales, const uint8_t* bits, const int32_t* offs, int M, int K, int N,
             uint16_t* y, void* ws, size_t ws_bytes, cudaStream_t stream, DeviceInfo* dev) {
    GemvPlan plan;
    int st = plan_gemv(M, K, N, qw_rows, dev->sms, &plan);
    if (st != QGEMM_OK) return st;
    const GemvWs L = gemv_ws_layout(M, K, N, dev->sms);
    if (ws_bytes < L.total || ws == nullptr) return QGEMM_ERR_WORKSPACE;
    const int mt = gemv_mt(M);
    if (!dev->gemv_attr[mt - 1]) {
        cudaError_t e = (mt == 1)
            ? cudaFuncSetAttribute(gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024)
            : cudaFuncSetAttribute(gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return QGEMM_ERR_CUDA;
        dev->gemv_attr[mt - 1] = true;
    }
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    const int nb = K / kBlockRows;

    XprepParams xp;
    xp.x = x;
    xp.perm = perm;
    xp.bits = bits;
    xp.offs = offs;
    xp.xdec = reinterpret_cast<__half*>(w8 + L.xdec);
    xp.xshift = reinterpret_cast<int*>(w8 + L.xshift);
    xp.M = M;
    xp.K = K;
    xp.nb = nb;
    xp.mp = mt * 8;
    xp.x_bf16 = (x_dtype == QGEMM_BF16);
    xprep_kernel<<<(nb + 7) / 8, 256, 0, stream>>>(xp);
    if ((st = launch_status()) != QGEMM_OK) return st;

    GemvParams p;
    p.xdec = xp.xdec;
    p.xshift = xp.xshift;
    p.qw = qw;
    p.qw_rows = qw_rows;
    p.scales = reinterpret_cast<const __half*>(scales);
    p.bits = bits;
    p.offs = offs;
    p.y = reinterpret_cast<__half*>(y);
    p.tickets = reinterpret_cast<int*>(w8 + L.tickets);
    p.slots = reinterpret_cast<float*>(w8 + L.slots);
    p.M = M;
    p.K = K;
    p.N = N;
    p.nb = nb;
    p.ng = gemv_groups(K);
    p.tiles = gemv_tiles(N);
    p.ring_rows = plan.ring;

    // launched as a programmatic dependent of xprep: starts streaming weights
    // while xprep runs and waits for it (griddepcontrol.wait) before reading x
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(kGemvThreads);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = (mt == 1) ? cudaLaunchKernelEx(&cfg, gemv_kernel<1>, p)
                                    : cudaLaunchKernelEx(&cfg, gemv_kernel<2>, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return QGEMM_ERR_CUDA;
    }
    return launch_status();
}

// ----------------------------------------------------------- integer GEMV
constexpr int kPathGemvInt = 0, kPathGemvTc = 1, kPathGemm = 2;
// M served by the integer GEMV (measured: above four tokens the tensor-core
// GEMV is faster)
constexpr int kIntPathMaxM = 4;
// M served by the allocation-free decode entry point
constexpr int kNoAllocMaxM = 4;

int int_mp(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : 4; }
int int_ctas_per_sm(int mp) { return mp <= 2 ? 2 : 1; }

size_t int_fixed_smem(int nb, int mp) {
    const size_t o = align_up((size_t)(nb + 1) * 4, 16) + 2 * kGemvSlots * 8 + 64 +
                     (size_t)3 * kGemvTileCols * mp * 4;
    return align_up(o, 1024);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library does not link the driver library itself).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// Tensor maps depend only on pointers and shapes, so each set is encoded once
// and kept: an eager call loop then spends no host time re-encoding them.
// The key holds the device and every value the encoding reads; the table is
// emptied when it reaches kMapCacheEntries sets.
struct MapKey {
    int64_t v[6];
    bool operator==(const MapKey& o) const { return std::memcmp(v, o.v, sizeof v) == 0; }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        uint64_t h = 0x9E3779B97F4A7C15ull;
        for (int64_t x : k.v) h = (h ^ (uint64_t)x) * 0x100000001B3ull;
        return (size_t)(h ^ (h >> 29));
    }
};
constexpr size_t kMapCacheEntries = 4096;

template <typename Maps, typename Encode>
int cached_maps(const MapKey& key, Maps* out, Encode encode) {
    static std::unordered_map<MapKey, Maps, MapKeyHash> table;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = table.find(key);
        if (it != table.end()) {
            *out = it->second;
            return QGEMM_OK;
        }
    }
    const int st = encode(out);
    if (st != QGEMM_OK) return st;
    std::lock_guard<std::mutex> lk(mu);
    if (table.size() >= kMapCacheEntries) table.clear();
    table.emplace(key, *out);
    return QGEMM_OK;
}

// Maps over qw [qw_rows][N] uint32 with boxes of 256 columns x 2^i rows.
int make_int_maps(const uint32_t* qw, int64_t qw_rows, int N, IntMaps* maps) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return QGEMM_ERR_CUDA;
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)qw_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)N * 4};
    const cuuint32_t estr[2] = {1, 1};
    for (int i = 0; i < kIntBoxMaps; ++i) {
        const cuuint32_t box[2] = {(cuuint32_t)kGemvTileCols, (cuuint32_t)(1u << i)};
        const CUresult r = fn(&maps->box[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(qw), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return QGEMM_ERR_CUDA;
    }
    return QGEMM_OK;
}

// Workspace: [tickets][partial slots][activation records].
struct IntWs {
    size_t tickets, slots, rec, total;
};

// min_tickets: a larger leading ticket region (the allocation-free entry
// point keeps one fixed region for every shape it serves).
IntWs int_ws_layout(int M, int K, int N, int sms, size_t min_tickets = 0) {
    const int mp = int_mp(M);
    const int nb = K / kBlockRows;
    IntWs w;
    w.tickets = 0;
    w.slots = std::max(ticket_region(M, N), min_tickets);
    w.rec = w.slots + align_up((size_t)gemv_max_grid(K, N, sms) * 2 * mp * kGemvTileCols * 4, 256);
    w.total = w.rec + align_up((size_t)(nb + 8) * int_rec_bytes(mp), 256);
    return w;
}

// Two CTAs per SM for M <= 2 (one for M <= 4, whose activations need more
// registers); grid capped as for the tensor-core GEMV so that every CTA's
// range holds at least one unit.
// cps_req: CTAs per SM (1 or 2), 0 for the default of this M.
int plan_int(int M, int K, int N, int64_t qw_rows, int sms, GemvPlan* plan, int* cps_out, int cps_req = 0) {
    const int nb = K / kBlockRows;
    const int mp = int_mp(M);
    const int cps = (cps_req == 1 || cps_req == 2) ? cps_req : int_ctas_per_sm(mp);
    // units of two 128-row groups: cost = word rows + 1, at most 8 * 8 + 1
    const int64_t nu = (nb + kIntUnitBlocks - 1) / kIntUnitBlocks;
    const int64_t U = (int64_t)gemv_tiles(N) * nu;
    const int64_t C = (int64_t)gemv_tiles(N) * (qw_rows + nu);
    const int64_t gcap = std::max<int64_t>(1, C / (8 * kIntUnitBlocks + 2));
    const int64_t G = std::min<int64_t>(std::min<int64_t>(U, gcap), (int64_t)cps * sms);
    const size_t fixed = int_fixed_smem(nb, mp);
    const size_t budget = (size_t)(cps == 2 ? 113 : 227) * 1024;
    if (fixed + (size_t)kGemvMinRing * kIntRowBytes > budget) return QGEMM_ERR_UNSUPPORTED;
    const int ring = (int)std::min<size_t>(kGemvMaxRing, (budget - fixed) / kIntRowBytes);
    plan->grid = (int)G;
    plan->ring = ring;
    plan->span_cap = 0;
    plan->smem = fixed + (size_t)ring * kIntRowBytes;
    if (cps_out) *cps_out = cps;
    return QGEMM_OK;
}

template <int MP>
cudaError_t launch_int(const GemvPlan& plan, const IntParams& p, const IntMaps& maps, cudaStream_t stream,
                       bool* attr_done) {
    if (!*attr_done) {
        cudaError_t e = cudaFuncSetAttribute(gemv_int_kernel<MP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             227 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemv_int_kernel<MP>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        *attr_done = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(kIntThreads);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_int_kernel<MP>, p, maps);
}

int launch_xprep_int(const void* x, int x_dtype, const int32_t* perm, const uint8_t* bits, int M, int K,
                     uint8_t* rec, cudaStream_t stream) {
    IntPrepParams xp;
    xp.x = x;
    xp.perm = perm;
    xp.bits = bits;
    xp.rec = rec;
    xp.M = M;
    xp.K = K;
    xp.nb = K / kBlockRows;
    xp.mp = int_mp(M);
    xp.x_bf16 = (x_dtype == QGEMM_BF16);
    // programmatic dependent of the previous grid (it waits for it on the
    // device), so its launch overlaps that grid's tail
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((xp.nb + 7) / 8);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, xprep_int_kernel, xp) != cudaSuccess) {
        cudaGetLastError();
        return QGEMM_ERR_CUDA;
    }
    return QGEMM_OK;
}

int run_gemv_int(const void* x, int x_dtype, const int32_t* perm, const uint32_t* qw, int64_t qw_rows,
                 const uint16_t* scales, const uint8_t* bits, const int32_t* offs, int M, int K, int N,
                 uint16_t* y, void* ws, size_t ws_bytes, cudaStream_t stream, DeviceInfo* dev, int cps_req = 0,
                 size_t min_tickets = 0) {
    GemvPlan plan;
    int st = plan_int(M, K, N, qw_rows, dev->sms, &plan, nullptr, cps_req);
    if (st != QGEMM_OK) return st;
    const IntWs L = int_ws_layout(M, K, N, dev->sms, min_tickets);
    if (ws_bytes < L.total || ws == nullptr) return QGEMM_ERR_WORKSPACE;
    int devid = 0;
    if (cudaGetDevice(&devid) != cudaSuccess) return QGEMM_ERR_CUDA;
    IntMaps maps;
    const MapKey key{{devid, 0, (int64_t)(uintptr_t)qw, qw_rows, N, 0}};
    st = cached_maps(key, &maps, [&](IntMaps* m) { return make_int_maps(qw, qw_rows, N, m); });
    if (st != QGEMM_OK) return st;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    const int nb = K / kBlockRows;
    const int mp = int_mp(M);

    if ((st = launch_xprep_int(x, x_dtype, perm, bits, M, K, w8 + L.rec, stream)) != QGEMM_OK) return st;

    IntParams p;
    p.rec = w8 + L.rec;
    p.qw = qw;
    p.qw_rows = qw_rows;
    p.scales = reinterpret_cast<const __half*>(scales);
    p.bits = bits;
    p.offs = offs;
    p.y = reinterpret_cast<__half*>(y);
    p.tickets = reinterpret_cast<int*>(w8 + L.tickets);
    p.slots = reinterpret_cast<float*>(w8 + L.slots);
    p.M = M;
    p.K = K;
    p.N = N;
    p.nb = nb;
    p.ng = gemv_groups(K);
    p.tiles = gemv_tiles(N);
    p.ring_rows = plan.ring;
    // programmatic dependent of xprep_int, as for the tensor-core GEMV
    const cudaError_t e = (mp == 1)   ? launch_int<1>(plan, p, maps, stream, &dev->int_attr[0])
                          : (mp == 2) ? launch_int<2>(plan, p, maps, stream, &dev->int_attr[1])
                                      : launch_int<4>(plan, p, maps, stream, &dev->int_attr[2]);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return QGEMM_ERR_CUDA;
    }
    return launch_status();
}

// ------------------------------------------------------------------ GEMM
int gemm_mtiles(int M) { return (M + kGemmBM - 1) / kGemmBM; }
int gemm_ntiles(int N) { return (N + kGemmBN - 1) / kGemmBN; }
int64_t gemm_tiles_of(int M, int N) { return (int64_t)gemm_mtiles(M) * gemm_ntiles(N); }
size_t gemm_smem(int nb) { return (size_t)kGemmFixedSmem + 512 + (size_t)(nb + 1) * 4; }

// Grid shape: whole waves of tiles (one tile per CTA), then the remaining
// tiles with their k range split so that they fill one more wave (each split
// at least eight 64-row steps, at most kGemmMaxSplit splits).  Few tiles
// (small M) means all are split.
struct GemmGrid {
    int64_t tiles, full, rest;
    int ksplit;
    int64_t grid() const { return full + rest * ksplit; }
};

GemmGrid gemm_grid(int M, int K, int N, int sms, int max_split = kGemmMaxSplit) {
    GemmGrid g;
    g.tiles = (int64_t)gemm_mtiles(M) * gemm_ntiles(N);
    g.full = g.tiles / sms * sms;
    g.rest = g.tiles - g.full;
    const int nk = (K + kGemmBK - 1) / kGemmBK;
    max_split = std::max(1, std::min(max_split, kGemmMaxSplit));
    g.ksplit = g.rest ? (int)std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(sms / g.rest, nk / 8),
                                                                    max_split))
                      : 1;
    if (g.ksplit == 1) {  // nothing to split: every tile whole
        g.full = g.tiles;
        g.rest = 0;
    }
    return g;
}

// Workspace: [tickets (the shared leading region)][x_p fp16 M x K][row shifts int32 M][fp32 partial tiles].
struct GemmWs {
    size_t xp;
    size_t xshift, tickets, partial, total;
};

GemmWs gemm_ws_layout(int M, int K, int N, int sms, int max_split = kGemmMaxSplit) {
    const GemmGrid gg = gemm_grid(M, K, N, sms, max_split);
    GemmWs w;
    w.tickets = 0;
    w.xp = ticket_region(M, N);
    w.xshift = w.xp + align_up((size_t)M * K * 2, 256);
    w.partial = w.xshift + align_up((size_t)M * 4, 256);
    w.total = w.partial + (size_t)gg.rest * gg.ksplit * kGemmBM * kGemmBN * 4;
    return w;
}

int make_gemm_maps(const void* xp, int x_dtype, int M, int K, const uint32_t* qw, int64_t qw_rows, int N,
                   GemmMaps* maps) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return QGEMM_ERR_CUDA;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kGemmBK, (cuuint32_t)kGemmBM};
        const cuuint32_t estr[2] = {1, 1};
        (void)x_dtype;  // x_p is fp16 for both input types
        const CUresult r = fn(&maps->a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(xp), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return QGEMM_ERR_CUDA;
        const cuuint32_t box64[2] = {(cuuint32_t)kGemmBK, 64u};
        const CUresult r64 = fn(&maps->a64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(xp), dims, strides,
                                box64, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r64 != CUDA_SUCCESS) return QGEMM_ERR_CUDA;
    }
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)qw_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)N * 4};
    const cuuint32_t estr[2] = {1, 1};
    for (int i = 0; i < kGemmBoxMaps; ++i) {
        const cuuint32_t box[2] = {(cuuint32_t)kGemmBN, (cuuint32_t)(1u << i)};
        const CUresult r = fn(&maps->w[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(qw), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return QGEMM_ERR_CUDA;
    }
    return QGEMM_OK;
}

int run_gemm(const void* x, int x_dtype, const int32_t* perm, const uint32_t* qw, int64_t qw_rows,
             const uint16_t* scales, const uint8_t* bits, const int32_t* offs, int M, int K, int N, uint16_t* y,
             void* ws, size_t ws_bytes, cudaStream_t stream, DeviceInfo* dev, int max_split = kGemmMaxSplit) {
    const GemmWs L = gemm_ws_layout(M, K, N, dev->sms, max_split);
    if (ws == nullptr || ws_bytes < L.total) return QGEMM_ERR_WORKSPACE;
    const int nb = K / kBlockRows;
    const size_t smem = gemm_smem(nb);
    if (smem > (size_t)227 * 1024) return QGEMM_ERR_UNSUPPORTED;
    const bool bf16 = (x_dtype == QGEMM_BF16);
    if (!dev->gemm_attr[0]) {
        if (cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess)
            return QGEMM_ERR_CUDA;
        dev->gemm_attr[0] = true;
    }
    int* xshift = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.xshift);
    int devid = 0;
    if (cudaGetDevice(&devid) != cudaSuccess) return QGEMM_ERR_CUDA;
    GemmMaps maps;
    const MapKey key{{devid, 1 + (int64_t)M * 2 + (x_dtype == QGEMM_BF16), (int64_t)(uintptr_t)qw, qw_rows,
                      ((int64_t)K << 32) | (uint32_t)N, (int64_t)(uintptr_t)ws}};
    int st = cached_maps(key, &maps,
                         [&](GemmMaps* m) {
                             return make_gemm_maps(static_cast<uint8_t*>(ws) + L.xp, x_dtype, M, K, qw, qw_rows, N,
                                                   m);
                         });
    if (st != QGEMM_OK) return st;

    XpermParams xq;
    xq.x = static_cast<const uint16_t*>(x);
    xq.perm = perm;
    xq.bits = bits;
    xq.xp = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + L.xp);
    xq.xshift = xshift;
    xq.M = M;
    xq.K = K;
    xq.x_bf16 = bf16;
    {
        // rows in groups of kXpermRows; split k so that there are about 4
        // CTAs per SM, each with at least 2048 k
        const int64_t rg = (M + kXpermRows - 1) / kXpermRows;
        const int64_t kspl = std::max<int64_t>(1, std::min<int64_t>(K / 2048, (4 * dev->sms + rg - 1) / rg));
        xperm_kernel<<<dim3((unsigned)rg, (unsigned)kspl), 256, 0, stream>>>(xq);
    }
    if ((st = launch_status()) != QGEMM_OK) return st;

    GemmParams p;
    p.xshift = xshift;
    p.scales = reinterpret_cast<const __half*>(scales);
    p.bits = bits;
    p.offs = offs;
    p.qw_rows = qw_rows;
    p.y = reinterpret_cast<__half*>(y);
    p.M = M;
    p.K = K;
    p.N = N;
    p.nb = nb;
    const GemmGrid gg = gemm_grid(M, K, N, dev->sms, max_split);
    p.mtiles = gemm_mtiles(M);
    p.ntiles = gemm_ntiles(N);
    p.full_tiles = (int)gg.full;
    p.ksplit = gg.ksplit;
    p.tickets = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.tickets);
    p.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.partial);
    p.x_bf16 = bf16;
    const unsigned grid = (unsigned)gg.grid();
    gemm_kernel<false><<<grid, kGemmThreads, smem, stream>>>(p, maps);
    return launch_status();
}

// ------------------------------------------------ allocation-free decode
// Scratch of qgemm_decode_noalloc, built into the library so that the call
// allocates nothing.  Zero-initialised at module load; every call re-zeroes
// the tickets it needs at zero.  In host code `g_noalloc_scratch` names a
// host-side stand-in, not device memory: kernels get the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QGEMM_NOALLOC_SCRATCH_BYTES];

// Its first kNoAllocTickets bytes hold the tickets of every shape served (the
// largest N accepted has 65536 tiles): no call writes data there, and every
// completed call leaves its tickets at zero, so the region is zero at every
// call without a memset (it is zero when the module loads).
constexpr size_t kNoAllocTickets = (size_t)256 << 10;

void* g_noalloc_ptr[64];
std::mutex g_noalloc_mu;

// Device address of the buffer on the current device, looked up once per device.
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QGEMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return QGEMM_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return QGEMM_OK;
}

// ------------------------------------------------------------- quantiser
// Workspace: [group bases float G x N][qmax float N][column errors double
// 96 x N][candidate errors double 96][chosen index int32].
struct QuantWs {
    size_t base, qmax, colerr, err, best, total;
};

QuantWs quant_ws_layout(int K, int N) {
    const size_t G = (size_t)(K + kGroupRows - 1) / kGroupRows;
    QuantWs w;
    w.base = 0;
    w.qmax = align_up(G * N * 4, 256);
    w.colerr = w.qmax + align_up((size_t)N * 4, 256);
    w.err = w.colerr + align_up((size_t)kQuantCands * N * 8, 256);
    w.best = w.err + align_up((size_t)kQuantCands * 8, 256);
    w.total = w.best + 256;
    return w;
}

size_t quant_scan_smem(int K) {
    return (size_t)kQuantCands * kQuantCols * 8 + (size_t)128 * kQuantCols * 2 + (size_t)K / kBlockRows;
}

// ------------------------------------------------------------ variants
// A kernel variant: the family and its one tunable knob.
//   kPathGemvInt: CTAs per SM (1 or 2);
//   kPathGemvTc:  none (0);
//   kPathGemm:    the largest k split of a tile (1 .. kGemmMaxSplit).
struct Variant {
    int path, knob;
};

// The library's built-in choice (crossovers measured on B200): the integer
// GEMV for M <= 4; the tensor-core GEMV for 5..16 rows, except from 12 rows
// on when the GEMM splits k across the SMs (few output tiles), where it
// measured faster; the GEMM above 16 rows.
Variant default_variant(int M, int K, int N, int sms) {
    if (M <= kIntPathMaxM) return {kPathGemvInt, int_ctas_per_sm(int_mp(M))};
    if (M > 16) return {kPathGemm, kGemmMaxSplit};
    if (M >= 12 && K > 0 && N > 0 && gemm_grid(M, K, N, sms).ksplit > 1) return {kPathGemm, kGemmMaxSplit};
    return {kPathGemvTc, 0};
}

// Every variant that can serve M rows, in a fixed order.
std::vector<Variant> candidate_variants(int M) {
    std::vector<Variant> v;
    if (M <= kIntPathMaxM) {
        v.push_back({kPathGemvInt, 1});
        v.push_back({kPathGemvInt, 2});
    }
    if (M <= 16) v.push_back({kPathGemvTc, 0});
    for (int s = 1; s <= kGemmMaxSplit; s *= 2) v.push_back({kPathGemm, s});
    return v;
}

bool variant_valid(int M, const Variant& v) {
    for (const Variant& c : candidate_variants(M))
        if (c.path == v.path && c.knob == v.knob) return true;
    return false;
}

size_t variant_ws_bytes(const Variant& v, int M, int K, int N, int sms) {
    if (v.path == kPathGemvInt) return int_ws_layout(M, K, N, sms).total;
    if (v.path == kPathGemvTc) return gemv_ws_layout(M, K, N, sms).total;
    return gemm_ws_layout(M, K, N, sms, v.knob).total;
}

// Choices made by qgemm_autotune (or recorded by the caller), per device and
// shape.  Looked up by every dispatch; a shape without an entry takes the
// built-in choice.
struct TuneKey {
    int dev, M, K, N;
    bool operator==(const TuneKey& o) const { return dev == o.dev && M == o.M && K == o.K && N == o.N; }
};
struct TuneKeyHash {
    size_t operator()(const TuneKey& k) const {
        return ((size_t)k.dev * 0x9E3779B1u) ^ ((size_t)k.M * 0x85EBCA6Bu) ^ ((size_t)k.K * 0xC2B2AE35u) ^
               ((size_t)k.N * 0x27D4EB2Fu);
    }
};
std::unordered_map<TuneKey, Variant, TuneKeyHash> g_tuned;
std::mutex g_tune_mu;
int g_autotune_mode = 0;  // 1: qgemm() tunes a shape on its first eager call

int current_dev_or_zero() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) {
        cudaGetLastError();
        d = 0;
    }
    return d;
}

bool tuned_variant(int M, int K, int N, Variant* out) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    auto it = g_tuned.find(TuneKey{current_dev_or_zero(), M, K, N});
    if (it == g_tuned.end()) return false;
    *out = it->second;
    return true;
}

int device_sms() {
    DeviceInfo* dev = nullptr;
    return (current_device_info(&dev) == QGEMM_OK) ? dev->sms : 148;
}

Variant choose_variant(int M, int K, int N) {
    Variant v;
    if (tuned_variant(M, K, N, &v)) return v;
    return default_variant(M, K, N, device_sms());
}

// Interquartile mean used to rank variants: the mean of the sorted values
// from the 5/16 to the 11/16 quantile (at least one value).
double iqm_of(std::vector<float> v) {
    if (v.empty()) return 0.0;
    std::sort(v.begin(), v.end());
    const size_t n = v.size();
    const size_t a = std::min(n - 1, (size_t)((double)n * 5.0 / 16.0));
    const size_t b = std::max(a + 1, (size_t)std::ceil((double)n * 11.0 / 16.0));
    double s = 0.0;
    for (size_t i = a; i < b; ++i) s += v[i];
    return s / (double)(b - a);
}

int run_variant(const Variant& v, const void* x, int x_dtype, const int32_t* perm, const uint32_t* qw,
                int64_t qw_rows, const uint16_t* scales, const uint8_t* bits, const int32_t* offs, int M, int K,
                int N, uint16_t* y, void* ws, size_t ws_bytes, cudaStream_t s, DeviceInfo* dev) {
    if (v.path == kPathGemvInt)
        return run_gemv_int(x, x_dtype, perm, qw, qw_rows, scales, bits, offs, M, K, N, y, ws, ws_bytes, s, dev,
                            v.knob);
    if (v.path == kPathGemvTc)
        return run_gemv(x, x_dtype, perm, qw, qw_rows, scales, bits, offs, M, K, N, y, ws, ws_bytes, s, dev);
    if (v.path == kPathGemm)
        return run_gemm(x, x_dtype, perm, qw, qw_rows, scales, bits, offs, M, K, N, y, ws, ws_bytes, s, dev,
                        v.knob);
    return QGEMM_ERR_UNSUPPORTED;
}

// Times every candidate variant on the caller's operands (warmup untimed
// calls, then iters calls with an event between consecutive calls), ranks
// them by the IQM of the per-call times and records the fastest for this
// device and shape.  Variants whose workspace exceeds ws_bytes are skipped.
// Rows of out: {path, knob, IQM in ns (or -1 when skipped / failed)}.
int autotune_shape(const void* x, int x_dtype, const int32_t* perm, const uint32_t* qw, int64_t qw_rows,
                   const uint16_t* scales, const uint8_t* bits, const int32_t* offs, int M, int K, int N,
                   uint16_t* y, void* ws, size_t ws_bytes, int warmup, int iters, cudaStream_t s, DeviceInfo* dev,
                   int64_t* out, int max_out) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return QGEMM_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return QGEMM_ERR_UNSUPPORTED;  // timing needs a live stream
    const std::vector<Variant> cands = candidate_variants(M);
    std::vector<cudaEvent_t> ev((size_t)iters + 1);
    for (auto& e : ev)
        if (cudaEventCreate(&e) != cudaSuccess) return QGEMM_ERR_CUDA;
    double best = 1e300;
    int bi = -1, rows = 0;
    int st = QGEMM_OK;
    for (size_t c = 0; c < cands.size(); ++c) {
        const Variant& v = cands[c];
        double t = -1.0;
        if (variant_ws_bytes(v, M, K, N, dev->sms) <= ws_bytes) {
            int vs = QGEMM_OK;
            for (int i = 0; i < warmup && vs == QGEMM_OK; ++i)
                vs = run_variant(v, x, x_dtype, perm, qw, qw_rows, scales, bits, offs, M, K, N, y, ws, ws_bytes, s,
                                 dev);
            for (int i = 0; i < iters && vs == QGEMM_OK; ++i) {
                if (cudaEventRecord(ev[i], s) != cudaSuccess) vs = QGEMM_ERR_CUDA;
                if (vs == QGEMM_OK)
                    vs = run_variant(v, x, x_dtype, perm, qw, qw_rows, scales, bits, offs, M, K, N, y, ws, ws_bytes,
                                     s, dev);
            }
            if (vs == QGEMM_OK && cudaEventRecord(ev[iters], s) != cudaSuccess) vs = QGEMM_ERR_CUDA;
            if (vs == QGEMM_OK && cudaEventSynchronize(ev[iters]) != cudaSuccess) vs = QGEMM_ERR_CUDA;
            if (vs == QGEMM_OK) {
                std::vector<float> ms((size_t)iters);
                for (int i = 0; i < iters && vs == QGEMM_OK; ++i)
                    if (cudaEventElapsedTime(&ms[i], ev[i], ev[i + 1]) != cudaSuccess) vs = QGEMM_ERR_CUDA;
                if (vs == QGEMM_OK) t = iqm_of(ms) * 1e6;  // ns
            }
            if (vs == QGEMM_ERR_CUDA) {
                st = vs;
                break;
            }
            if (t >= 0.0 && t < best) {
                best = t;
                bi = (int)c;
            }
        }
        if (out && rows < max_out) {
            out[3 * rows + 0] = v.path;
            out[3 * rows + 1] = v.knob;
            out[3 * rows + 2] = (int64_t)std::llround(t);
            ++rows;
        }
    }
    for (auto& e : ev) cudaEventDestroy(e);
    if (st != QGEMM_OK) return st;
    if (bi < 0) return QGEMM_ERR_WORKSPACE;  // no variant fits the workspace
    {
        std::lock_guard<std::mutex> lk(g_tune_mu);
        g_tuned[TuneKey{current_dev_or_zero(), M, K, N}] = cands[(size_t)bi];
    }
    return rows;
}

// The KV quantiser instantiated for the code width.
template <int E>
void launch_kv_quant(dim3 grid, dim3 block, cudaStream_t s, const __half* v, int64_t nvec, int bits,
                     uint32_t* codes, __half* sc) {
    switch (bits) {
        case 2: kv_quant_kernel<E, 2><<<grid, block, 0, s>>>(v, nvec, codes, sc); break;
        case 3: kv_quant_kernel<E, 3><<<grid, block, 0, s>>>(v, nvec, codes, sc); break;
        case 4: kv_quant_kernel<E, 4><<<grid, block, 0, s>>>(v, nvec, codes, sc); break;
        case 5: kv_quant_kernel<E, 5><<<grid, block, 0, s>>>(v, nvec, codes, sc); break;
        case 6: kv_quant_kernel<E, 6><<<grid, block, 0, s>>>(v, nvec, codes, sc); break;
        default: kv_quant_kernel<E, 8><<<grid, block, 0, s>>>(v, nvec, codes, sc); break;
    }
}

}  // namespace

// =========================================================== C ABI
extern "C" {

int qgemm_version(void) { return kVersion; }

const char* qgemm_status_string(int status) {
    switch (status) {
        case QGEMM_OK: return "ok";
        case QGEMM_ERR_NULL: return "null pointer";
        case QGEMM_ERR_SHAPE: return "unsupported shape";
        case QGEMM_ERR_BITS: return "invalid bit schedule";
        case QGEMM_ERR_ALIGN: return "pointer not 16-byte aligned";
        case QGEMM_ERR_WORKSPACE: return "workspace missing or too small";
        case QGEMM_ERR_DTYPE: return "invalid activation dtype";
        case QGEMM_ERR_CUDA: return "CUDA error";
        case QGEMM_ERR_UNSUPPORTED: return "unsupported request";
        default: return "unknown status";
    }
}

int64_t qgemm_packed_word_rows(const uint8_t* h_bits, int K) {
    if (!h_bits) return QGEMM_ERR_NULL;
    if (K <= 0 || K % kBlockRows != 0 || K > kMaxK) return QGEMM_ERR_SHAPE;
    int64_t s = 0;
    for (int j = 0; j < K / kBlockRows; ++j) {
        const int b = h_bits[j];
        if (!(b == 2 || b == 3 || b == 4 || b == 5 || b == 6 || b == 8)) return QGEMM_ERR_BITS;
        s += b;
    }
    return s;
}

int qgemm_offsets(const uint8_t* h_bits, int K, int32_t* h_offs) {
    if (!h_offs) return QGEMM_ERR_NULL;
    const int64_t rows = qgemm_packed_word_rows(h_bits, K);
    if (rows < 0) return (int)rows;
    int32_t s = 0;
    for (int j = 0; j < K / kBlockRows; ++j) {
        h_offs[j] = s;
        s += h_bits[j];
    }
    h_offs[K / kBlockRows] = s;
    return QGEMM_OK;
}

int qgemm_validate_schedule(const uint8_t* h_bits, const int32_t* h_offs, int K, int64_t qw_rows) {
    if (!h_bits || !h_offs) return QGEMM_ERR_NULL;
    const int64_t rows = qgemm_packed_word_rows(h_bits, K);
    if (rows < 0) return (int)rows;
    if (rows != qw_rows) return QGEMM_ERR_BITS;
    int64_t s = 0;
    for (int j = 0; j <= K / kBlockRows; ++j) {
        if (h_offs[j] != s) return QGEMM_ERR_BITS;
        if (j < K / kBlockRows) s += h_bits[j];
    }
    return QGEMM_OK;
}

size_t qgemm_packed_bytes(int64_t qw_rows, int N) {
    return qw_rows > 0 && N > 0 ? (size_t)qw_rows * (size_t)N * 4 : 0;
}

size_t qgemm_scale_bytes(int K, int N) {
    return K > 0 && N > 0 ? (size_t)((K + kGroupRows - 1) / kGroupRows) * (size_t)N * 2 : 0;
}

int qgemm_path_for(int M, int K, int N) {
    if (M <= 0) return kPathGemvInt;
    return choose_variant(M, K, N).path;
}

size_t qgemm_workspace_bytes(int M, int K, int N) {
    if (M <= 0 || check_shape(K, N) != QGEMM_OK) return 0;
    const int sms = device_sms();
    // enough for every variant of this M, so that a tuned choice always fits
    size_t w = 0;
    for (const Variant& v : candidate_variants(M)) w = std::max(w, variant_ws_bytes(v, M, K, N, sms));
    return w;
}

int qgemm_plan_info(int M, int K, int N, int64_t qw_rows, int64_t* out) {
    if (!out) return QGEMM_ERR_NULL;
    int st = check_shape(K, N);
    if (st != QGEMM_OK) return st;
    if (M <= 0) return QGEMM_ERR_SHAPE;
    if ((st = check_rows(K, qw_rows)) != QGEMM_OK) return st;
    DeviceInfo* dev = nullptr;
    const int sms = (current_device_info(&dev) == QGEMM_OK) ? dev->sms : 148;
    for (int i = 0; i < 6; ++i) out[i] = 0;
    const Variant var = choose_variant(M, K, N);
    out[0] = var.path;
    out[5] = sms;
    if (out[0] == kPathGemvInt) {
        GemvPlan plan;
        int cps = 1;
        if ((st = plan_int(M, K, N, qw_rows, sms, &plan, &cps, var.knob)) != QGEMM_OK) return st;
        out[1] = plan.grid;
        out[2] = plan.ring;
        out[3] = cps;
        out[4] = (int64_t)plan.smem;
        return QGEMM_OK;
    }
    if (out[0] == kPathGemvTc) {
        GemvPlan plan;
        if ((st = plan_gemv(M, K, N, qw_rows, sms, &plan)) != QGEMM_OK) return st;
        out[1] = plan.grid;
        out[2] = plan.ring;
        out[3] = 1;
        out[4] = (int64_t)plan.smem;
        return QGEMM_OK;
    }
    if (out[0] == kPathGemm) {
        const GemmGrid gg = gemm_grid(M, K, N, sms, var.knob);
        out[1] = gg.grid();
        out[2] = gg.ksplit;
        out[3] = 1;
        out[4] = (int64_t)gemm_smem(K / kBlockRows);
        return QGEMM_OK;
    }
    return QGEMM_ERR_UNSUPPORTED;
}

int qgemm_device_error(int* h_code, int clear) {
    if (!h_code) return QGEMM_ERR_NULL;
    if (cudaMemcpyFromSymbol(h_code, qg::g_dev_error, sizeof(int)) != cudaSuccess) return QGEMM_ERR_CUDA;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(qg::g_dev_error, &zero, sizeof(int)) != cudaSuccess) return QGEMM_ERR_CUDA;
    }
    return QGEMM_OK;
}

int qgemm_pack(const uint8_t* d_codes, const uint8_t* d_bits, const int32_t* d_offs, int K, int N,
               int64_t qw_rows, uint32_t* d_qw, void* stream) {
    if (!d_codes || !d_bits || !d_offs || !d_qw) return QGEMM_ERR_NULL;
    int st = check_shape(K, N);
    if (st != QGEMM_OK) return st;
    if ((st = check_rows(K, qw_rows)) != QGEMM_OK) return st;
    if (!aligned16(d_codes) || !aligned16(d_qw)) return QGEMM_ERR_ALIGN;
    const dim3 grid((N / 4 + 127) / 128, K / kBlockRows);
    pack_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(d_codes, d_bits, d_offs, K, N,
                                                                      qw_rows, d_qw);
    return launch_status();
}

int qgemm_dequant(const uint32_t* d_qw, int64_t qw_rows, const uint16_t* d_scales,
                  const uint8_t* d_bits, const int32_t* d_offs, int K, int N, uint16_t* d_w,
                  void* stream) {
    if (!d_qw || !d_scales || !d_bits || !d_offs || !d_w) return QGEMM_ERR_NULL;
    int st = check_shape(K, N);
    if (st != QGEMM_OK) return st;
    if ((st = check_rows(K, qw_rows)) != QGEMM_OK) return st;
    if (!aligned16(d_qw) || !aligned16(d_scales) || !aligned16(d_w)) return QGEMM_ERR_ALIGN;
    const dim3 grid((N / 4 + 127) / 128, K / kBlockRows);
    dequant_kernel<<<grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(
        d_qw, qw_rows, reinterpret_cast<const __half*>(d_scales), d_bits, d_offs, K, N,
        reinterpret_cast<__half*>(d_w));
    return launch_status();
}

int qgemm(const void* d_x, int x_dtype, const int32_t* d_perm, const uint32_t* d_qw,
          int64_t qw_rows, const uint16_t* d_scales, const uint8_t* d_bits,
          const int32_t* d_offs, int M, int K, int N, uint16_t* d_y, void* d_ws,
          size_t ws_bytes, void* stream) {
    if (!d_x || !d_perm || !d_qw || !d_scales || !d_bits || !d_offs || !d_y) return QGEMM_ERR_NULL;
    if (x_dtype != QGEMM_F16 && x_dtype != QGEMM_BF16) return QGEMM_ERR_DTYPE;
    int st = check_shape(K, N);
    if (st != QGEMM_OK) return st;
    if (M <= 0 || M > (1 << 20)) return QGEMM_ERR_SHAPE;
    if ((st = check_rows(K, qw_rows)) != QGEMM_OK) return st;
    if (!aligned16(d_x) || !aligned16(d_perm) || !aligned16(d_qw) || !aligned16(d_scales) ||
        !aligned16(d_y) || (d_ws && !aligned16(d_ws)))
        return QGEMM_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    if ((st = current_device_info(&dev)) != QGEMM_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Variant v;
    if (!tuned_variant(M, K, N, &v)) {
        v = default_variant(M, K, N, dev->sms);
        if (g_autotune_mode) {
            // first eager call of this shape: time the variants on these
            // operands (never inside a stream capture, which keeps the
            // built-in choice), then run the chosen one below
            cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
            if (cudaStreamIsCapturing(s, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusNone) {
                st = autotune_shape(d_x, x_dtype, d_perm, d_qw, qw_rows, d_scales, d_bits, d_offs, M, K, N, d_y,
                                    d_ws, ws_bytes, 20, 200, s, dev, nullptr, 0);
                if (st < 0 && st != QGEMM_ERR_WORKSPACE) return st;
                tuned_variant(M, K, N, &v);
            } else {
                cudaGetLastError();
            }
        }
    }
    return run_variant(v, d_x, x_dtype, d_perm, d_qw, qw_rows, d_scales, d_bits, d_offs, M, K, N, d_y, d_ws,
                       ws_bytes, s, dev);
}

int qgemm_autotune(const void* d_x, int x_dtype, const int32_t* d_perm, const uint32_t* d_qw, int64_t qw_rows,
                   const uint16_t* d_scales, const uint8_t* d_bits, const int32_t* d_offs, int M, int K, int N,
                   uint16_t* d_y, void* d_ws, size_t ws_bytes, int warmup, int iters, void* stream,
                   int64_t* h_results, int max_results) {
    if (!d_x || !d_perm || !d_qw || !d_scales || !d_bits || !d_offs || !d_y) return QGEMM_ERR_NULL;
    if (x_dtype != QGEMM_F16 && x_dtype != QGEMM_BF16) return QGEMM_ERR_DTYPE;
    int st = check_shape(K, N);
    if (st != QGEMM_OK) return st;
    if (M <= 0 || M > (1 << 20)) return QGEMM_ERR_SHAPE;
    if (warmup < 0 || iters < 1 || iters > 100000 || max_results < 0) return QGEMM_ERR_SHAPE;
    if ((st = check_rows(K, qw_rows)) != QGEMM_OK) return st;
    if (!aligned16(d_x) || !aligned16(d_perm) || !aligned16(d_qw) || !aligned16(d_scales) ||
        !aligned16(d_y) || (d_ws && !aligned16(d_ws)))
        return QGEMM_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    if ((st = current_device_info(&dev)) != QGEMM_OK) return st;
    return autotune_shape(d_x, x_dtype, d_perm, d_qw, qw_rows, d_scales, d_bits, d_offs, M, K, N, d_y, d_ws,
                          ws_bytes, warmup, iters, static_cast<cudaStream_t>(stream), dev, h_results, max_results);
}

int qgemm_set_autotune(int mode) {
    if (mode != 0 && mode != 1) return QGEMM_ERR_SHAPE;
    std::lock_guard<std::mutex> lk(g_tune_mu);
    g_autotune_mode = mode;
    return QGEMM_OK;
}

int qgemm_tune_lookup(int M, int K, int N, int* h_path, int* h_knob) {
    if (!h_path || !h_knob) return QGEMM_ERR_NULL;
    Variant v;
    if (!tuned_variant(M, K, N, &v)) return 0;
    *h_path = v.path;
    *h_knob = v.knob;
    return 1;
}

int qgemm_tune_record(int M, int K, int N, int path, int knob) {
    if (M <= 0 || check_shape(K, N) != QGEMM_OK) return QGEMM_ERR_SHAPE;
    if (!variant_valid(M, Variant{path, knob})) return QGEMM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_tune_mu);
    g_tuned[TuneKey{current_dev_or_zero(), M, K, N}] = Variant{path, knob};
    return QGEMM_OK;
}

int qgemm_tune_clear(void) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    g_tuned.clear();
    return QGEMM_OK;
}

double qgemm_iqm(const float* h_values, int n) {
    if (!h_values || n <= 0) return -1.0;
    return iqm_of(std::vector<float>(h_values, h_values + n));
}

size_t qgemm_quantize_workspace_bytes(int K, int N) {
    if (check_shape(K, N) != QGEMM_OK) return 0;
    return quant_ws_layout(K, N).total;
}

int qgemm_quantize(const uint16_t* d_w, const uint8_t* d_bits, int K, int N, uint8_t* d_codes, uint16_t* d_scales,
                   double* d_err, int32_t* d_best, void* d_ws, size_t ws_bytes, void* stream) {
    if (!d_w || !d_bits || !d_codes || !d_scales || !d_ws) return QGEMM_ERR_NULL;
    int st = check_shape(K, N);
    if (st != QGEMM_OK) return st;
    if (!aligned16(d_w) || !aligned16(d_codes) || !aligned16(d_scales) || !aligned16(d_ws) ||
        (d_err && ((uintptr_t)d_err & 7)) || (d_best && ((uintptr_t)d_best & 3)))
        return QGEMM_ERR_ALIGN;
    const QuantWs L = quant_ws_layout(K, N);
    if (ws_bytes < L.total) return QGEMM_ERR_WORKSPACE;
    DeviceInfo* dev = nullptr;
    if ((st = current_device_info(&dev)) != QGEMM_OK) return st;
    const size_t smem = quant_scan_smem(K);
    if (!dev->quant_attr) {  // a per-device setting
        if (cudaFuncSetAttribute(quant_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess)
            return QGEMM_ERR_CUDA;
        dev->quant_attr = true;
    }
    if (smem > (size_t)227 * 1024) return QGEMM_ERR_UNSUPPORTED;
    uint8_t* w8 = static_cast<uint8_t*>(d_ws);
    QuantParams p;
    p.w = reinterpret_cast<const __half*>(d_w);
    p.bits = d_bits;
    p.base = reinterpret_cast<float*>(w8 + L.base);
    p.qmax = reinterpret_cast<float*>(w8 + L.qmax);
    p.colerr = reinterpret_cast<double*>(w8 + L.colerr);
    p.err = d_err ? d_err : reinterpret_cast<double*>(w8 + L.err);
    p.best = d_best ? d_best : reinterpret_cast<int32_t*>(w8 + L.best);
    p.codes = d_codes;
    p.scales = reinterpret_cast<__half*>(d_scales);
    p.K = K;
    p.N = N;
    p.G = (K + kGroupRows - 1) / kGroupRows;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    quant_scan_kernel<<<(unsigned)((N + kQuantCols - 1) / kQuantCols), kQuantCols, smem, s>>>(p);
    if ((st = launch_status()) != QGEMM_OK) return st;
    quant_pick_kernel<<<1, kQuantCands, 0, s>>>(p);
    if ((st = launch_status()) != QGEMM_OK) return st;
    quant_emit_kernel<<<(unsigned)((N + 127) / 128), 128, 0, s>>>(p);
    return launch_status();
}

int qgemm_kv_quantize(const uint16_t* d_v, int64_t nvec, int D, int bits, uint32_t* d_codes, uint16_t* d_scales,
                      void* stream) {
    if (!d_v || !d_codes || !d_scales) return QGEMM_ERR_NULL;
    if (nvec < 0 || nvec > ((int64_t)1 << 36) || (D != 32 && D != 64 && D != 128 && D != 256))
        return QGEMM_ERR_SHAPE;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 5 || bits == 6 || bits == 8)) return QGEMM_ERR_BITS;
    if (((uintptr_t)d_v & 7) || ((uintptr_t)d_codes & 3) || ((uintptr_t)d_scales & 1)) return QGEMM_ERR_ALIGN;
    if (nvec == 0) return QGEMM_OK;
    const dim3 grid((unsigned)((nvec + kKvWarps - 1) / kKvWarps)), block(32 * kKvWarps);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const __half* v = reinterpret_cast<const __half*>(d_v);
    __half* sc = reinterpret_cast<__half*>(d_scales);
    switch (D / 32) {
        case 1: launch_kv_quant<1>(grid, block, s, v, nvec, bits, d_codes, sc); break;
        case 2: launch_kv_quant<2>(grid, block, s, v, nvec, bits, d_codes, sc); break;
        case 4: launch_kv_quant<4>(grid, block, s, v, nvec, bits, d_codes, sc); break;
        default: launch_kv_quant<8>(grid, block, s, v, nvec, bits, d_codes, sc); break;
    }
    return launch_status();
}

int qgemm_kv_dequantize(const uint32_t* d_codes, const uint16_t* d_scales, int64_t nvec, int D, int bits,
                        uint16_t* d_v, void* stream) {
    if (!d_v || !d_codes || !d_scales) return QGEMM_ERR_NULL;
    if (nvec < 0 || nvec > ((int64_t)1 << 36) || (D != 32 && D != 64 && D != 128 && D != 256))
        return QGEMM_ERR_SHAPE;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 5 || bits == 6 || bits == 8)) return QGEMM_ERR_BITS;
    if (((uintptr_t)d_v & 7) || ((uintptr_t)d_codes & 3) || ((uintptr_t)d_scales & 1)) return QGEMM_ERR_ALIGN;
    if (nvec == 0) return QGEMM_OK;
    const dim3 grid((unsigned)((nvec + kKvWarps - 1) / kKvWarps)), block(32 * kKvWarps);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    __half* v = reinterpret_cast<__half*>(d_v);
    const __half* sc = reinterpret_cast<const __half*>(d_scales);
    switch (D / 32) {
        case 1: kv_dequant_kernel<1><<<grid, block, 0, s>>>(d_codes, sc, nvec, bits, v); break;
        case 2: kv_dequant_kernel<2><<<grid, block, 0, s>>>(d_codes, sc, nvec, bits, v); break;
        case 4: kv_dequant_kernel<4><<<grid, block, 0, s>>>(d_codes, sc, nvec, bits, v); break;
        default: kv_dequant_kernel<8><<<grid, block, 0, s>>>(d_codes, sc, nvec, bits, v); break;
    }
    return launch_status();
}

size_t qgemm_noalloc_scratch_bytes(int M, int K, int N) {
    if (M < 1 || M > kNoAllocMaxM || check_shape(K, N) != QGEMM_OK) return 0;
    return int_ws_layout(M, K, N, device_sms(), kNoAllocTickets).total;
}

int qgemm_decode_noalloc(const void* d_x, int x_dtype, const int32_t* d_perm, const uint32_t* d_qw,
                         int64_t qw_rows, const uint16_t* d_scales, const uint8_t* d_bits,
                         const int32_t* d_offs, int M, int K, int N, uint16_t* d_y, void* stream) {
    if (!d_x || !d_perm || !d_qw || !d_scales || !d_bits || !d_offs || !d_y) return QGEMM_ERR_NULL;
    if (x_dtype != QGEMM_F16 && x_dtype != QGEMM_BF16) return QGEMM_ERR_DTYPE;
    int st = check_shape(K, N);
    if (st != QGEMM_OK) return st;
    if (M < 1 || M > kNoAllocMaxM) return QGEMM_ERR_SHAPE;
    if ((st = check_rows(K, qw_rows)) != QGEMM_OK) return st;
    if (!aligned16(d_x) || !aligned16(d_perm) || !aligned16(d_qw) || !aligned16(d_scales) || !aligned16(d_y))
        return QGEMM_ERR_ALIGN;
    DeviceInfo* dev = nullptr;
    if ((st = current_device_info(&dev)) != QGEMM_OK) return st;
    const IntWs L = int_ws_layout(M, K, N, dev->sms, kNoAllocTickets);
    if (L.slots > kNoAllocTickets || L.total > QGEMM_NOALLOC_SCRATCH_BYTES) return QGEMM_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != QGEMM_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the CTA count qgemm() would use: a tuned integer-GEMV variant, else the built-in one
    Variant v;
    const int cps = (tuned_variant(M, K, N, &v) && v.path == kPathGemvInt) ? v.knob : 0;
    return run_gemv_int(d_x, x_dtype, d_perm, d_qw, qw_rows, d_scales, d_bits, d_offs, M, K, N, d_y, scratch,
                        QGEMM_NOALLOC_SCRATCH_BYTES, s, dev, cps, kNoAllocTickets);
}

int qgemm_noalloc_reset(void* stream) {
    void* scratch = nullptr;
    const int st = noalloc_scratch(&scratch);
    if (st != QGEMM_OK) return st;
    if (cudaMemsetAsync(scratch, 0, kNoAllocTickets, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return QGEMM_ERR_CUDA;
    }
    return QGEMM_OK;
}

}  // extern "C"
