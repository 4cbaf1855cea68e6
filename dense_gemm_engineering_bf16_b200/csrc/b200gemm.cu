// Host side of the C ABI declared in include/b200gemm.h: argument checks
// (the correctness contract of "GPU 执行模型", section "正确性契约"),
// shape-bucket configuration choice (section "编译与 autotune": choices are
// cached per device and shape class, with no compilation or tuning on the
// call path), TMA tensor-map encoding ("Modern GPU Programming For MLSys -
// 书籍总结", section 2.5), and the cluster launch of the persistent kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "b200gemm.h"
#include "gemm_bf16_sm100.cuh"
#include "gemm_bf16_skinny_sm100.cuh"
#include "gemm_bf16_small_sm100.cuh"
#include "gemm_mxfp8_sm100.cuh"

namespace {

using b200::DeviceStatus;

// ---------------------------------------------------------------- configs --

using Cfg1x256F32 = b200::GemmBf16Cfg<1, 256, 4, 0>;
using Cfg1x256B16 = b200::GemmBf16Cfg<1, 256, 4, 1>;
using Cfg1x128F32 = b200::GemmBf16Cfg<1, 128, 6, 0>;
using Cfg1x128B16 = b200::GemmBf16Cfg<1, 128, 6, 1>;
using Cfg2x256F32 = b200::GemmBf16Cfg<2, 256, 6, 0>;
using Cfg2x256B16 = b200::GemmBf16Cfg<2, 256, 6, 1>;
using Cfg2x256F32C = b200::GemmBf16Cfg<2, 256, 6, 0, true>;
using Cfg2x256B16C = b200::GemmBf16Cfg<2, 256, 6, 1, true>;
using Cfg1x256F32C = b200::GemmBf16Cfg<1, 256, 4, 0, true>;
using Cfg1x256B16C = b200::GemmBf16Cfg<1, 256, 4, 1, true>;
// two MMA consumers sharing B: 512 x 256 pair tiles, single-buffered TMEM
using Cfg2x512F32C = b200::GemmBf16Cfg<2, 256, 4, 0, true, 2>;
using Cfg2x512B16C = b200::GemmBf16Cfg<2, 256, 4, 1, true, 2>;
// stream-K over the (tile, K block) iterations: pair tiles 256 x 256, static grid
using Cfg2x256F32S = b200::GemmBf16Cfg<2, 256, 6, 0, false, 1, true>;
using Cfg2x256B16S = b200::GemmBf16Cfg<2, 256, 6, 1, false, 1, true>;
// pair tiles 256 x 224 (fp32 C: 7 chunks of 32 columns), static grid
using Cfg2x224F32 = b200::GemmBf16Cfg<2, 224, 6, 0>;
// the 256 x 256 CLC pair kernel storing every chunk to further copies of C
// (gemm_bf16_allgather)
using Cfg2x256F32CP = b200::GemmBf16Cfg<2, 256, 6, 0, true, 1, false, true>;
using Cfg2x256B16CP = b200::GemmBf16Cfg<2, 256, 6, 1, true, 1, false, true>;
// cluster split-K: 2-8 CTAs per tile, each over a share of K, partials summed
// through distributed shared memory
using Cfg1x128F32K = b200::GemmBf16Cfg<1, 128, 6, 0, false, 1, false, false, true>;
using Cfg1x128B16K = b200::GemmBf16Cfg<1, 128, 6, 1, false, 1, false, false, true>;
using Cfg1x256F32K = b200::GemmBf16Cfg<1, 256, 4, 0, false, 1, false, false, true>;
using Cfg1x256B16K = b200::GemmBf16Cfg<1, 256, 4, 1, false, 1, false, false, true>;
using CfgMxf8 = b200::GemmMxf8Cfg<1, 4>;
using CfgMxf8Pair = b200::GemmMxf8Cfg<2, 6>;
using CfgSk64F32 = b200::GemmSkinnyCfg<64, 8, 0>;
using CfgSk64B16 = b200::GemmSkinnyCfg<64, 8, 1>;
// the skinny tile with its K split over a cluster (partials in DSMEM)
using CfgSk64F32C = b200::GemmSkinnyCfg<64, 8, 0, 1, true>;
using CfgSk64B16C = b200::GemmSkinnyCfg<64, 8, 1, 1, true>;
using CfgSk128F32 = b200::GemmSkinnyCfg<128, 6, 0>;
using CfgSk128B16 = b200::GemmSkinnyCfg<128, 6, 1>;
using CfgSk256F32 = b200::GemmSkinnyCfg<256, 4, 0>;
using CfgSk256B16 = b200::GemmSkinnyCfg<256, 4, 1>;

constexpr int kMaxDevices = 64;
// internal configuration slot of the CLC pair kernel with further copies of C
constexpr gemm_config_t kCfgAllgather = static_cast<gemm_config_t>(GEMM_CFG_COUNT_);

struct DeviceState {
    bool ready = false;
    bool supported = false;
    int sm_count = 0;
    // watchdog status blocks: `status` from cudaMalloc (first allocating call
    // on the device), `noalloc_status` the device address of the library's
    // static scratch array (first gemm_bf16_noalloc call on the device)
    DeviceStatus *status = nullptr;
    DeviceStatus *noalloc_status = nullptr;
    // per (config, out type): smem attribute set, co-resident clusters
    bool attr_done[GEMM_CFG_COUNT_ + 1][2] = {};     // + the all-gather kernel (kCfgAllgather)
    int max_clusters[GEMM_CFG_COUNT_ + 1][2] = {};
    // split-K configurations: co-resident CTAs with clusters of 2, 4 and 8
    int splitk_ctas[GEMM_CFG_COUNT_ + 1][2][3] = {};
    // block-scaled path: kernel attributes (1-CTA, pair), repacked-scale workspace
    bool mx_attr_done[2] = {};
    int mx_max_clusters[2] = {};
    uint8_t *mx_ws = nullptr;
    size_t mx_ws_bytes = 0;
    // skinny path: kernel attributes (per template), split-tile workspace;
    // the cluster-split templates (fp32, bf16 C): co-resident CTAs with
    // clusters of 2 and 4
    bool sk_attr_done[6] = {};
    bool skc_attr_done[2] = {};
    int skc_ctas[2][2] = {};
    uint8_t *sk_ws = nullptr;
    size_t sk_ws_bytes = 0;
    uint32_t sk_epoch = 0;
    // Workspaces replaced by larger ones.  They are kept, not freed: a CUDA
    // graph captured earlier still holds their addresses.
    std::vector<void *> retired;
};

std::mutex g_mutex;
DeviceState g_devices[kMaxDevices];
std::atomic<int> g_forced{GEMM_CFG_AUTO};
thread_local int g_last_cuda_error = 0;
int32_t g_last_where = -1;
int32_t g_last_block = -1;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

gemm_status_t cuda_fail(cudaError_t e) {
    g_last_cuda_error = static_cast<int>(e);
    return GEMM_ERR_LAUNCH;
}

uint64_t watchdog_ns(int64_t K) {
    static const uint64_t base = [] {
        const char *s = std::getenv("B200GEMM_WATCHDOG_MS");
        const long long ms = s ? std::atoll(s) : 2000;
        return static_cast<uint64_t>(ms > 0 ? ms : 2000) * 1000000ull;
    }();
    // One tile's main loop grows with K; allow ~100 ns per K element on top.
    return base + static_cast<uint64_t>(K) * 100ull;
}

// Tile rows per raster group: tiles are walked column by column inside
// groups of this many tile rows, so the CTAs running at the same time share A
// row-panels and B column-panels in L2.  B200GEMM_GROUP_M overrides it.
int raster_group_m() {
    static const int g = [] {
        const char *s = std::getenv("B200GEMM_GROUP_M");
        const int v = s ? std::atoi(s) : 8;
        return v > 0 ? v : 8;
    }();
    return g;
}

// Split factor of the split-K configurations: B200GEMM_KSPLIT = 2, 4 or 8
// forces it (tests: every factor, including shares with no K block); unset,
// choose_ksplit picks it by shape.  Read once.
int forced_ksplit() {
    static const int v = [] {
        const char *s = std::getenv("B200GEMM_KSPLIT");
        const int k = s ? std::atoi(s) : 0;
        return (k == 2 || k == 4 || k == 8) ? k : 0;
    }();
    return v;
}

// K order of the dense kernels' tiles: serpentine (odd waves of tiles walk K
// backwards, reusing the K slices the previous wave left in L2) unless
// B200GEMM_SERPENTINE=0.
bool serpentine_k() {
    static const bool on = [] {
        const char *s = std::getenv("B200GEMM_SERPENTINE");
        return !(s && s[0] == '0');
    }();
    return on;
}

// Test-only: B200GEMM_INJECT_TIMEOUT holds one character per launch of the
// dense bf16 kernels, in launch order; a '1' makes that launch drop one
// pipeline arrival in CTA 0 so the device watchdog fires.  The variable is
// read once, at the first launch; unset or empty, launches only test one
// static flag.
uint32_t inject_flags() {
    static const std::string mask = [] {
        const char *s = std::getenv("B200GEMM_INJECT_TIMEOUT");
        return std::string(s ? s : "");
    }();
    if (mask.empty()) return 0u;
    static std::atomic<size_t> launches{0};
    const size_t i = launches.fetch_add(1, std::memory_order_relaxed);
    return (i < mask.size() && mask[i] == '1') ? b200::kInjectDropFirstStage : 0u;
}

// True while `stream` is being captured into a CUDA graph (or when that
// cannot be told, so that no one-time set-up runs inside a capture).
bool capturing(cudaStream_t stream) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        (void)cudaGetLastError();
        return true;
    }
    return cs != cudaStreamCaptureStatusNone;
}

// Device of the current thread, checked to be compute capability 10.0, with
// the tensor-map encoder looked up.  Allocates nothing.  The one-time
// set-up may not run inside a stream capture: GEMM_ERR_CAPTURE then.
gemm_status_t current_device(int &dev, DeviceState *&st, cudaStream_t stream) {
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        g_last_cuda_error = static_cast<int>(e);
        return GEMM_ERR_UNSUPPORTED_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    st = &g_devices[dev];
    if (!st->ready) {
        if (capturing(stream)) return GEMM_ERR_CAPTURE;
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            return GEMM_ERR_UNSUPPORTED_DEVICE;
        }
        st->supported = (major == 10 && minor == 0);
        if (!st->supported) {
            st->ready = true;
            return GEMM_ERR_UNSUPPORTED_DEVICE;
        }
        if ((e = cudaDeviceGetAttribute(&st->sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e);
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cuda_fail(e);
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        st->ready = true;
    }
    return st->supported ? GEMM_OK : GEMM_ERR_UNSUPPORTED_DEVICE;
}

// current_device, plus the device's status block from cudaMalloc (first
// call on the device; a blocking cudaMemset zeroes it).
gemm_status_t current_device_alloc(int &dev, DeviceState *&st, cudaStream_t stream) {
    gemm_status_t s = current_device(dev, st, stream);
    if (s != GEMM_OK) return s;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!st->status) {
        if (capturing(stream)) return GEMM_ERR_CAPTURE;
        cudaError_t e;
        DeviceStatus *p = nullptr;
        if ((e = cudaMalloc(&p, sizeof(DeviceStatus))) != cudaSuccess) return cuda_fail(e);
        if ((e = cudaMemset(p, 0, sizeof(DeviceStatus))) != cudaSuccess) return cuda_fail(e);
        st->status = p;
    }
    return GEMM_OK;
}

// [begin, end) byte ranges of a row-major rows x cols matrix with leading dim ld.
bool overlaps(const void *p, int64_t rows, int64_t cols, int64_t ld, int64_t esize,
              const void *q, int64_t qrows, int64_t qcols, int64_t qld, int64_t qesize) {
    if (rows <= 0 || cols <= 0 || qrows <= 0 || qcols <= 0 || !p || !q) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p);
    const uintptr_t a1 = a0 + static_cast<uintptr_t>(((rows - 1) * ld + cols) * esize);
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(q);
    const uintptr_t b1 = b0 + static_cast<uintptr_t>(((qrows - 1) * qld + qcols) * qesize);
    return a0 < b1 && b0 < a1;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = 0x7FFFFFFF;

// Checks shared by every entry point.  elem sizes in bytes; a_mn / b_mn:
// A stored K x M, B stored K x N (else M x K and N x K).
gemm_status_t check_args(const void *A, const void *B, const void *C, int64_t M, int64_t N, int64_t K,
                         int64_t lda, int64_t ldb, int64_t ldc, int64_t ea, int64_t eb, int64_t ec,
                         bool a_mn = false, bool b_mn = false) {
    if (M < 0 || N < 0 || K < 0) return GEMM_ERR_INVALID_VALUE;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return GEMM_ERR_TOO_LARGE;
    if (M == 0 || N == 0) return GEMM_OK;
    if (!C) return GEMM_ERR_INVALID_VALUE;
    if (ldc < N) return GEMM_ERR_INVALID_VALUE;
    if (K > 0) {
        const int64_t a_rows = a_mn ? K : M, a_cols = a_mn ? M : K;
        const int64_t b_rows = b_mn ? K : N, b_cols = b_mn ? N : K;
        if (!A || !B) return GEMM_ERR_INVALID_VALUE;
        if (lda < a_cols || ldb < b_cols) return GEMM_ERR_INVALID_VALUE;
        if (!aligned16(A) || !aligned16(B)) return GEMM_ERR_MISALIGNED;
        if ((lda * ea) % 16 || (ldb * eb) % 16) return GEMM_ERR_MISALIGNED;
        if (lda * ea >= (int64_t(1) << 40) || ldb * eb >= (int64_t(1) << 40)) return GEMM_ERR_TOO_LARGE;
        if (overlaps(C, M, N, ldc, ec, A, a_rows, a_cols, lda, ea) ||
            overlaps(C, M, N, ldc, ec, B, b_rows, b_cols, ldb, eb))
            return GEMM_ERR_ALIAS;
    }
    if (!aligned16(C) || (ldc * ec) % 16) return GEMM_ERR_MISALIGNED;
    if (ldc * ec >= (int64_t(1) << 40)) return GEMM_ERR_TOO_LARGE;
    return GEMM_OK;
}

// ------------------------------------------------------------ tensor maps --

gemm_status_t encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *ptr, int64_t inner,
                        int64_t outer, int64_t ld_bytes, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_bytes)};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dtype, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = static_cast<int>(r);
        return GEMM_ERR_LAUNCH;
    }
    return GEMM_OK;
}

// --------------------------------------------------------------- launches --

// Predicted time (us) of one launch of a dense configuration on a B200 (148
// SMs): a fixed cost plus, per wave of tiles, the work one SM does in it
// (tile rows x columns x K, a pair tile's split over its two SMs), at the
// configuration's own rate.  The constants are least-squares fits to event
// timings of every configuration over about 60 shapes from 64 x 4096 x 4096
// to 4096^3 (fp32 C, L2 flushed before each call): the autotuning search
// over tile shape and persistent strategy ("GPU 执行模型", section "编译与
// autotune"), run once offline so that no call pays for it.  They rank the
// candidates; they are not a performance claim.
struct CostModel {
    int tile_m, tile_n, slots;   // tile, co-resident tiles (one per SM or per pair)
    double fixed_us, us_per_gunit;
};
double predicted_us(const CostModel &c, int64_t M, int64_t N, int64_t K) {
    const int64_t tiles = ((M + c.tile_m - 1) / c.tile_m) * ((N + c.tile_n - 1) / c.tile_n);
    const int64_t waves = (tiles + c.slots - 1) / c.slots;
    const double per_sm = static_cast<double>(c.tile_m) * c.tile_n / (c.slots == 74 ? 2.0 : 1.0);
    return c.fixed_us + c.us_per_gunit * 1e-9 * static_cast<double>(waves) * per_sm * static_cast<double>(K);
}

gemm_config_t select_config(int64_t M, int64_t N, int64_t K) {
    const int forced = g_forced.load(std::memory_order_relaxed);
    if (forced != GEMM_CFG_AUTO && forced != GEMM_CFG_MXFP8_1CTA_128x256 && forced != GEMM_CFG_MXFP8_2CTA_256x256)
        return static_cast<gemm_config_t>(forced);
    // A tiny product: the latency path (no tensor memory, no pipeline to
    // fill).  Measured against the tcgen05 choice, L2 flushed: 128^3 6.7 vs
    // 12.1 us, 512^3 10.2 vs 13.3, 128 x 128 x 2048 14.4 vs 20.6,
    // 16 x 4096 x 2048 16.0 vs 20.1; it ties at 768^3, 1024 x 1024 x 256 and
    // 1024 x 1024 x 128, and loses at 1024^3, 128 x 256 x 4096 and on wide C
    // with a tiny K (2048 x 2048 x 32: 18.6 vs 12.5), where its 32 x 32 tiles
    // are too many.
    if (M * N * K <= (int64_t(1) << 27) && K <= 2048 && M * N <= (int64_t(1) << 20)) return GEMM_CFG_SMALL;
    // A few rows and a long K: swap A and B, so 128 rows of B fill the MMA,
    // and split K (over a cluster per tile of B, else stream-K over every
    // SM).  Past 32 rows the split-K tile kernels win.
    if (M <= 32 && K >= 4096) return GEMM_CFG_SKINNY;
    // Tiles for at most half the SMs and a long K: split each tile's K over
    // a cluster (2-8 CTAs), the partials summed on chip.
    const int64_t tiles128 = ((M + 127) / 128) * ((N + 127) / 128);
    const int64_t tiles256 = ((M + 127) / 128) * ((N + 255) / 256);
    if (K >= 2048 && tiles128 <= 74) return GEMM_CFG_1CTA_128x128_SPLITK;
    if (K >= 2048 && tiles256 <= 74) return GEMM_CFG_1CTA_128x256_SPLITK;
    // Every 128 x 128 tile on an SM of its own: the most SMs streaming.
    if (tiles128 <= 148) return GEMM_CFG_1CTA_128x128;
    struct Candidate {
        gemm_config_t cfg;
        CostModel cost;
    };
    static constexpr Candidate kCandidates[] = {
        {GEMM_CFG_1CTA_128x256, {128, 256, 148, 9.51, 192.3}},
        {GEMM_CFG_2CTA_256x256, {256, 256, 74, 11.90, 178.6}},
        {GEMM_CFG_2CTA_256x256_CLC, {256, 256, 74, 12.78, 169.5}},
        {GEMM_CFG_2CTA_512x256_CLC, {512, 256, 74, 16.90, 151.95}},
        {GEMM_CFG_1CTA_128x256_CLC, {128, 256, 148, 9.19, 198.7}},
    };
    gemm_config_t best = GEMM_CFG_1CTA_128x128;
    double best_us = 0.0;
    for (const Candidate &c : kCandidates) {
        const CostModel &m = c.cost;
        const int64_t waves = (((M + m.tile_m - 1) / m.tile_m) * ((N + m.tile_n - 1) / m.tile_n) + m.slots - 1) / m.slots;
        // One-CTA 256-wide tiles load 50 % more operand bytes per FLOP than
        // a pair's: past two waves L2 cannot feed them.  The 512 x 256 tile
        // holds one tile in TMEM, so its drain is not hidden behind the
        // next tile's MMAs: it pays off only over a long K.
        if ((c.cfg == GEMM_CFG_1CTA_128x256 || c.cfg == GEMM_CFG_1CTA_128x256_CLC) && waves > 2) continue;
        if ((c.cfg == GEMM_CFG_2CTA_512x256_CLC || c.cfg == GEMM_CFG_1CTA_128x256_CLC) && K < 8192) continue;
        // a later candidate must win by more than the model's noise
        const double us = predicted_us(m, M, N, K);
        if (best_us == 0.0 || us < best_us * 0.98) {
            best = c.cfg;
            best_us = us;
        }
    }
    // Over a short K, the static pair schedule beats Cluster Launch Control:
    // a tile is too short for the scheduler round trip to hide.
    if (best == GEMM_CFG_2CTA_256x256_CLC && K <= 2048) best = GEMM_CFG_2CTA_256x256;
    return best;
}

gemm_status_t sk_workspace(DeviceState *st, size_t bytes, uint8_t *&ws, cudaStream_t stream);

// First launch of a configuration on a device: its shared-memory attribute
// and how many of its clusters fit on the SMs at once (for split-K, with
// clusters of 2, 4 and 8 CTAs).  Refused inside a stream capture.
template <class Cfg>
gemm_status_t setup_attrs(DeviceState *st, gemm_config_t cfg_id, cudaStream_t stream) {
    auto kernel = b200::gemm_bf16_sm100_kernel<Cfg>;
    const int oi = Cfg::OUT;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (st->attr_done[cfg_id][oi]) return GEMM_OK;
    if (capturing(stream)) return GEMM_ERR_CAPTURE;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES)) !=
        cudaSuccess)
        return cuda_fail(e);
    // the narrow-tail twin (same shared memory, same co-resident count) is
    // set up with it, so that a later launch that splits its tail needs no
    // first-call work (it may be inside a stream capture)
    if constexpr (Cfg::TAIL_OK) {
        if ((e = cudaFuncSetAttribute(b200::gemm_bf16_sm100_kernel<typename Cfg::Tail>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::Tail::SMEM_BYTES)) !=
            cudaSuccess)
            return cuda_fail(e);
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Cfg::CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t lc = {};
    lc.blockDim = dim3(Cfg::THREADS, 1, 1);
    lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
    lc.stream = stream;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int clusters = st->sm_count / Cfg::CG;
    if (Cfg::CG > 1 && !Cfg::CLC) {
        lc.gridDim = dim3(Cfg::CG * clusters, 1, 1);
        int n = 0;
        if ((e = cudaOccupancyMaxActiveClusters(&n, kernel, &lc)) != cudaSuccess) return cuda_fail(e);
        if (n > 0) clusters = n;
    }
    if constexpr (Cfg::SPLITK) {
        for (int li = 0; li < 3; ++li) {
            const int S = 2 << li;
            attr[0].val.clusterDim.x = S;
            lc.gridDim = dim3(S * (st->sm_count / S), 1, 1);
            int n = 0;
            if ((e = cudaOccupancyMaxActiveClusters(&n, kernel, &lc)) != cudaSuccess) return cuda_fail(e);
            st->splitk_ctas[cfg_id][oi][li] = n * S;
        }
    }
    st->max_clusters[cfg_id][oi] = clusters;
    st->attr_done[cfg_id][oi] = true;
    return GEMM_OK;
}

// Cluster size of a split-K launch: the largest S of 8, 4, 2 whose clusters
// all fit on the SMs at once (one tile per cluster), that leaves every member
// at least two 64-wide K blocks, and whose column slices (BN / S) are whole
// store chunks.  1: no split pays (the caller runs the unsplit kernel).
template <class Cfg>
int choose_ksplit(const DeviceState *st, gemm_config_t cfg_id, int64_t M, int64_t N, int64_t K) {
    const int64_t tiles = ((M + Cfg::BM - 1) / Cfg::BM) * ((N + Cfg::BN - 1) / Cfg::BN);
    const int64_t num_kb = (K + Cfg::BK - 1) / Cfg::BK;
    for (int li = 2; li >= 0; --li) {
        const int S = 2 << li;
        if ((Cfg::BN / S) % Cfg::EPI_COLS != 0) continue;
        if (num_kb < 2 * S) continue;
        if (tiles * S > st->splitk_ctas[cfg_id][Cfg::OUT][li]) continue;
        // the other members' partials of a slice fit in the operand ring
        if (static_cast<int64_t>(S - 1) * 128 * (Cfg::BN / S) * 4 > static_cast<int64_t>(Cfg::STAGES) * Cfg::STAGE_BYTES)
            continue;
        return S;
    }
    return 1;
}

// `status`: the watchdog status block the kernel records a timeout in;
// `peers`: the further copies of C of a PEERS configuration (else unused);
// `ksplit`: the cluster size of a split-K configuration (else unused).
template <class Cfg>
gemm_status_t launch_bf16(DeviceState *st, DeviceStatus *status, gemm_config_t cfg_id, const void *A,
                          const void *B, void *C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                          int64_t ldc, cudaStream_t stream, const b200::Epilogue &epi = b200::plain_epilogue(),
                          uint32_t layout = 0, const b200::PeerC *peers = nullptr, int ksplit = 1);

// A split-K configuration: the cluster size by shape (or forced); where no
// split pays, the same tile without one (`plain_id`, config CfgPlain).
template <class CfgK, class CfgPlain>
gemm_status_t launch_splitk(DeviceState *st, DeviceStatus *status, gemm_config_t cfg_id, gemm_config_t plain_id,
                            const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K, int64_t lda,
                            int64_t ldb, int64_t ldc, cudaStream_t stream, const b200::Epilogue &epi,
                            uint32_t layout) {
    gemm_status_t s;
    if ((s = setup_attrs<CfgK>(st, cfg_id, stream)) != GEMM_OK) return s;
    int S = forced_ksplit();
    if (S == 0 || (CfgK::BN / S) % CfgK::EPI_COLS) S = choose_ksplit<CfgK>(st, cfg_id, M, N, K);
    if (S < 2)
        return launch_bf16<CfgPlain>(st, status, plain_id, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout,
                                     nullptr, 1);
    return launch_bf16<CfgK>(st, status, cfg_id, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout, nullptr, S);
}

template <class Cfg>
gemm_status_t launch_bf16(DeviceState *st, DeviceStatus *status, gemm_config_t cfg_id, const void *A,
                          const void *B, void *C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                          int64_t ldc, cudaStream_t stream, const b200::Epilogue &epi, uint32_t layout,
                          const b200::PeerC *peers, int ksplit) {
    auto kernel = b200::gemm_bf16_sm100_kernel<Cfg>;
    const int oi = Cfg::OUT;
    typename Cfg::PeerArg peer_arg{};
    if constexpr (Cfg::PEERS) {
        if (!peers) return GEMM_ERR_INVALID_VALUE;
        peer_arg = *peers;
    } else {
        (void)peers;
    }
    // MN-major tiles arrive as 64-wide boxes: whole boxes per CTA only
    if (((layout & b200::kLayoutBMajorN) && Cfg::B_ROWS % 64) || ((layout & b200::kLayoutAMajorM) && Cfg::BM_CTA % 64))
        return GEMM_ERR_INVALID_VALUE;
    // split-K: 2, 4 or 8 CTAs per cluster, one cluster per tile; the column
    // slices are whole store chunks, and the others' partials of a slice fit
    // in the operand ring they are received in
    if (Cfg::SPLITK && (ksplit < 2 || ksplit > 8 || (ksplit & (ksplit - 1)) || (Cfg::BN / ksplit) % Cfg::EPI_COLS ||
                        static_cast<int64_t>(ksplit - 1) * 128 * (Cfg::BN / ksplit) * 4 >
                            static_cast<int64_t>(Cfg::STAGES) * Cfg::STAGE_BYTES))
        return GEMM_ERR_INVALID_VALUE;
    cudaError_t e;
    gemm_status_t s;
    if constexpr (!Cfg::TAIL) {   // (a narrow-tail twin is set up with its whole-tile kernel)
        if ((s = setup_attrs<Cfg>(st, cfg_id, stream)) != GEMM_OK) return s;
    }
    const int64_t tiles = ((M + Cfg::BM - 1) / Cfg::BM) * ((N + Cfg::BN - 1) / Cfg::BN);
    const int64_t resident = st->max_clusters[cfg_id][oi];
    const bool b_kmajor = !(layout & b200::kLayoutBMajorN);
    // Narrow tail: a last wave of R tiles that would leave at least half of
    // the co-resident clusters idle (0 < 2 R <= resident) runs as 2 R
    // half-width units on the tile's twin kernel, so that every cluster has
    // work at the end (measured: 102.0 -> 100.8 us at 4096^3 on 256 x 256
    // pair tiles, 107.1 -> 103.4 on 128 x 256 one-CTA tiles; the halves
    // reread A, so the tail shrinks by less than half a tile).
    const int64_t rem = resident > 0 ? tiles % resident : 0;
    const bool split_tail = b_kmajor && rem > 0 && 2 * rem <= resident;
    if constexpr (Cfg::TAIL_OK && !Cfg::TAIL) {
        if (split_tail)
            return launch_bf16<typename Cfg::Tail>(st, status, cfg_id, A, B, C, M, N, K, lda, ldb, ldc, stream, epi,
                                                   layout, peers, ksplit);
    }
    const int cluster_ctas = Cfg::SPLITK ? ksplit : Cfg::CG;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster_ctas);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t lc = {};
    lc.blockDim = dim3(Cfg::THREADS, 1, 1);
    lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
    lc.stream = stream;
    lc.attrs = attr;
    lc.numAttrs = 1;
    const CUtensorMapDataType cdt = Cfg::OUT == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int64_t ec = Cfg::OUT == 0 ? 4 : 2;
    alignas(64) CUtensorMap tmA, tmB, tmC, tmBt;
    // K-major operands: boxes of 64 (K) x rows; MN-major (stored K x M / K x N):
    // boxes of 64 (MN) x 64 (K)
    if (layout & b200::kLayoutAMajorM)
        s = encode_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, M, K, lda * 2, 64, Cfg::BK);
    else
        s = encode_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, M, lda * 2, Cfg::BK, Cfg::BM_CTA);
    if (s != GEMM_OK) return s;
    if (layout & b200::kLayoutBMajorN)
        s = encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, K, ldb * 2, 64, Cfg::BK);
    else
        s = encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, K, N, ldb * 2, Cfg::BK, Cfg::B_ROWS);
    if (s != GEMM_OK) return s;
    // B for the half-width units of a narrow tail (K-major B only)
    if (Cfg::TAIL) {
        if ((s = encode_2d(&tmBt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, K, N, ldb * 2, Cfg::BK, Cfg::B_ROWS / 2)) !=
            GEMM_OK)
            return s;
    } else {
        tmBt = tmB;
    }
    // The store map covers the columns that end on a 16-byte granule; the
    // kernel writes the rest of each row ([n_tma, N)) with plain stores.  If
    // no whole granule exists the map is a placeholder the kernel never uses.
    const int64_t n_tma = (N * ec / 16) * 16 / ec;
    if ((s = encode_2d(&tmC, cdt, C, n_tma > 0 ? n_tma : 16 / ec, M, ldc * ec, Cfg::EPI_COLS, 32)) != GEMM_OK)
        return s;

    // Static schedule: as many clusters as fit at once, each striding over
    // the tiles.  CLC: one cluster per tile; running clusters claim the rest.
    // Split-K: one cluster of `ksplit` CTAs per tile.  Stream-K: every
    // co-resident cluster, each with an equal share of the (tile, K block)
    // iterations.
    // (the twin runs units [0, tiles - R) as whole tiles, then 2 R halves)
    int64_t tail_first = tiles, units = tiles;
    if (Cfg::TAIL && split_tail) {
        tail_first = tiles - rem;
        units = tiles + rem;
    }
    int64_t clusters = (Cfg::CLC || Cfg::SPLITK) ? units : (units > resident ? resident : units);
    if constexpr (Cfg::SK) {
        // Every cluster's range must hold at least one iteration (the
        // fix-up counts a split tile's contributors as the consecutive range
        // owners), and a range of fewer than 4 K blocks barely fills the
        // pipeline: at most one cluster per 4 iterations.
        const int64_t iters = tiles * ((K + Cfg::BK - 1) / Cfg::BK);
        const int64_t want = (iters + 3) / 4;
        clusters = want < resident ? want : resident;
    }
    lc.gridDim = dim3(static_cast<unsigned>(clusters * cluster_ctas), 1, 1);
    // tiles that run at the same time: one wave (for CLC, as many clusters
    // as fit on the SMs at once); stream-K keeps K ascending
    const int wave_tiles = (serpentine_k() && !Cfg::SK && !Cfg::SPLITK) ? static_cast<int>(resident) : 0;
    // Stream-K workspace: two [128][BN] fp32 partial slots per CTA (the
    // first and the last tile of its range may be split), then one 64-bit
    // arrival counter per (tile, CTA of the cluster).
    float *sk_partials = nullptr;
    unsigned long long *sk_counters = nullptr;
    uint32_t epoch = 0;
    if constexpr (Cfg::SK) {
        const int64_t partial_bytes = clusters * Cfg::CG * 2 * 128 * Cfg::BN * 4;
        uint8_t *ws = nullptr;
        if ((s = sk_workspace(st, static_cast<size_t>(partial_bytes + tiles * Cfg::CG * 8), ws, stream)) != GEMM_OK)
            return s;
        sk_partials = reinterpret_cast<float *>(ws);
        sk_counters = reinterpret_cast<unsigned long long *>(ws + partial_bytes);
        std::lock_guard<std::mutex> lock(g_mutex);
        epoch = ++st->sk_epoch;
        if (epoch == 0) epoch = ++st->sk_epoch;
    }
    e = cudaLaunchKernelEx(&lc, kernel, tmA, tmB, tmC, tmBt, static_cast<int>(M), static_cast<int>(N),
                           static_cast<int>(K), C, ldc, static_cast<int>(n_tma), raster_group_m(), wave_tiles,
                           static_cast<int>(tail_first), units > tiles ? 2 : 1, status, watchdog_ns(K), inject_flags(),
                           epi, layout, sk_partials, sk_counters, epoch, peer_arg);
    if (e != cudaSuccess) return cuda_fail(e);
    return GEMM_OK;
}

// ------------------------------------------------------------ skinny path --

// Workspace of the skinny path: per persistent CTA `slots` partial tiles of
// 128 x MP fp32, then one 64-bit arrival counter per 128-row tile of B.
struct SkinnyLayout {
    int64_t grid, slots, tiles, partial_bytes, counter_bytes;
};

template <class Cfg>
SkinnyLayout skinny_layout(int64_t N, int64_t K, int sm_count) {
    SkinnyLayout l;
    const int64_t kb = (K + Cfg::SK - 1) / Cfg::SK;    // iterations (stages of SK) per tile
    l.tiles = (N + Cfg::TILE_N - 1) / Cfg::TILE_N;
    const int64_t total = l.tiles * kb;
    // at least 8 64-wide K blocks per CTA: a CTA with fewer barely fills its
    // pipeline, and a tile cut into many slivers costs a long fix-up
    constexpr int64_t kMinIters = 8 / Cfg::KBS > 0 ? 8 / Cfg::KBS : 1;
    const int64_t want = (total + kMinIters - 1) / kMinIters;
    l.grid = want < sm_count ? want : sm_count;
    const int64_t per = (total + l.grid - 1) / l.grid;
    l.slots = (per + kb - 1) / kb + 1;
    l.partial_bytes = l.grid * l.slots * Cfg::TILE_N * Cfg::MP * 4;
    l.counter_bytes = l.tiles * 8;
    return l;
}

// Grows the skinny workspace on demand (counters start at zero).  Growing
// is refused inside a stream capture; the old buffer is retired, not freed.
gemm_status_t sk_workspace(DeviceState *st, size_t bytes, uint8_t *&ws, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (st->sk_ws_bytes < bytes) {
        if (capturing(stream)) return GEMM_ERR_CAPTURE;
        cudaError_t e;
        if (st->sk_ws) {
            st->retired.push_back(st->sk_ws);
            st->sk_ws = nullptr;
            st->sk_ws_bytes = 0;
        }
        const size_t want = bytes < (size_t(4) << 20) ? (size_t(4) << 20) : bytes;
        if ((e = cudaMalloc(&st->sk_ws, want)) != cudaSuccess) return cuda_fail(e);
        if ((e = cudaMemset(st->sk_ws, 0, want)) != cudaSuccess) return cuda_fail(e);
        st->sk_ws_bytes = want;
    }
    ws = st->sk_ws;
    return GEMM_OK;
}

template <class Cfg>
gemm_status_t launch_skinny(DeviceState *st, int attr_slot, const void *A, const void *B, void *C, int64_t M,
                            int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc, cudaStream_t stream,
                            const b200::Epilogue &epi, uint32_t layout) {
    auto kernel = b200::gemm_bf16_skinny_sm100_kernel<Cfg>;
    cudaError_t e;
    uint32_t epoch;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!st->sk_attr_done[attr_slot]) {
            if (capturing(stream)) return GEMM_ERR_CAPTURE;
            if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          Cfg::SMEM_BYTES)) != cudaSuccess)
                return cuda_fail(e);
            st->sk_attr_done[attr_slot] = true;
        }
        epoch = ++st->sk_epoch;
        if (epoch == 0) epoch = ++st->sk_epoch;
    }
    const SkinnyLayout l = skinny_layout<Cfg>(N, K, st->sm_count);
    uint8_t *ws = nullptr;
    gemm_status_t s;
    if ((s = sk_workspace(st, static_cast<size_t>(l.partial_bytes + l.counter_bytes), ws, stream)) != GEMM_OK)
        return s;
    const int64_t mpad = (M + 15) / 16 * 16;
    alignas(64) CUtensorMap tmB, tmA;
    if (layout & b200::kLayoutBMajorN)
        s = encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, K, ldb * 2, 64, Cfg::BK);
    else
        s = encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, K, N, ldb * 2, Cfg::BK, Cfg::TILE_N / 2);
    if (s != GEMM_OK) return s;
    if ((s = encode_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, M, lda * 2, Cfg::BK,
                       static_cast<uint32_t>(mpad))) != GEMM_OK)
        return s;
    float *partials = reinterpret_cast<float *>(ws);
    unsigned long long *counters = reinterpret_cast<unsigned long long *>(ws + l.partial_bytes);
    kernel<<<static_cast<unsigned>(l.grid), Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(
        tmB, tmA, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>(mpad), C, ldc,
        partials, counters, static_cast<int>(l.slots), epoch, st->status, watchdog_ns(K), epi, layout);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
    return GEMM_OK;
}

// The skinny tile with K split over a cluster of S CTAs per 128-row tile of
// B (no workspace: the partials meet in shared memory).  S: 4 or 2, the
// largest whose clusters all fit at once, leave every member two 64-wide K
// blocks, keep at least 96 SMs streaming, and give no member more than 2048
// of K (a longer share streams better on all 148 SMs with stream-K:
// 16 x 8192 x 8192 ran 35.4 us that way against 36.9 split in clusters of
// two); 1 = none qualifies (the caller runs the stream-K kernel).
template <class Cfg>
gemm_status_t launch_skinny_cluster(DeviceState *st, DeviceStatus *status, int slot, const void *A, const void *B,
                                    void *C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                                    cudaStream_t stream, const b200::Epilogue &epi, uint32_t layout, bool &launched) {
    launched = false;
    auto kernel = b200::gemm_bf16_skinny_sm100_kernel<Cfg>;
    cudaError_t e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t lc = {};
    lc.blockDim = dim3(Cfg::THREADS, 1, 1);
    lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
    lc.stream = stream;
    lc.attrs = attr;
    lc.numAttrs = 1;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!st->skc_attr_done[slot]) {
            if (capturing(stream)) return GEMM_ERR_CAPTURE;
            if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES)) !=
                cudaSuccess)
                return cuda_fail(e);
            for (int li = 0; li < 2; ++li) {
                const int S = 2 << li;
                attr[0].val.clusterDim.x = S;
                lc.gridDim = dim3(S * (st->sm_count / S), 1, 1);
                int n = 0;
                if ((e = cudaOccupancyMaxActiveClusters(&n, kernel, &lc)) != cudaSuccess) return cuda_fail(e);
                st->skc_ctas[slot][li] = n * S;
            }
            st->skc_attr_done[slot] = true;
        }
    }
    const int64_t tiles = (N + Cfg::TILE_N - 1) / Cfg::TILE_N;
    const int64_t kb = (K + Cfg::BK - 1) / Cfg::BK;
    int S = 1;
    for (int li = 1; li >= 0; --li) {
        const int cand = 2 << li;
        if (tiles * cand <= st->skc_ctas[slot][li] && kb >= 2 * cand && tiles * cand >= 96 && K <= 2048 * cand) {
            S = cand;
            break;
        }
    }
    if (S < 2) return GEMM_OK;                    // not launched: the caller runs stream-K
    const int64_t mpad = (M + 15) / 16 * 16;
    alignas(64) CUtensorMap tmB, tmA;
    gemm_status_t s;
    if (layout & b200::kLayoutBMajorN)
        s = encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, K, ldb * 2, 64, Cfg::BK);
    else
        s = encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, K, N, ldb * 2, Cfg::BK, Cfg::TILE_N / 2);
    if (s != GEMM_OK) return s;
    if ((s = encode_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, M, lda * 2, Cfg::BK,
                       static_cast<uint32_t>(mpad))) != GEMM_OK)
        return s;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    lc.gridDim = dim3(static_cast<unsigned>(tiles * S), 1, 1);
    float *no_partials = nullptr;
    unsigned long long *no_counters = nullptr;
    e = cudaLaunchKernelEx(&lc, kernel, tmB, tmA, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
                           static_cast<int>(mpad), C, ldc, no_partials, no_counters, 0, 0u, status, watchdog_ns(K),
                           epi, layout);
    if (e != cudaSuccess) return cuda_fail(e);
    launched = true;
    return GEMM_OK;
}

gemm_status_t launch_skinny_any(DeviceState *st, bool f32, const void *A, const void *B, void *C, int64_t M,
                                int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc, cudaStream_t stream,
                                const b200::Epilogue &epi = b200::plain_epilogue(), uint32_t layout = 0) {
    // the skinny kernel reads A K-major only (A stored M x K)
    if (M > 256 || (layout & b200::kLayoutAMajorM)) return GEMM_ERR_INVALID_VALUE;
    if (M <= 64) {
        // enough 128-row tiles of B to keep most SMs streaming with K split
        // over a cluster: the partials stay on chip; otherwise stream-K
        bool launched = false;
        gemm_status_t s = f32 ? launch_skinny_cluster<CfgSk64F32C>(st, st->status, 0, A, B, C, M, N, K, lda, ldb,
                                                                   ldc, stream, epi, layout, launched)
                              : launch_skinny_cluster<CfgSk64B16C>(st, st->status, 1, A, B, C, M, N, K, lda, ldb,
                                                                   ldc, stream, epi, layout, launched);
        if (s != GEMM_OK || launched) return s;
        return f32 ? launch_skinny<CfgSk64F32>(st, 0, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                   : launch_skinny<CfgSk64B16>(st, 1, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
    }
    if (M <= 128)
        return f32 ? launch_skinny<CfgSk128F32>(st, 2, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                   : launch_skinny<CfgSk128B16>(st, 3, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
    return f32 ? launch_skinny<CfgSk256F32>(st, 4, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
               : launch_skinny<CfgSk256B16>(st, 5, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
}

// C = act(beta * C + bias) for K == 0 (the empty product, then the epilogue).
template <typename T>
gemm_status_t launch_epilogue_only(void *C, int64_t M, int64_t N, int64_t ldc, const b200::Epilogue &epi,
                                   int sm_count, cudaStream_t stream) {
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;
    const int64_t blocks = M < cap ? M : cap;
    b200::epilogue_only_kernel<T><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<T *>(C), M, N,
                                                                                      ldc, epi);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GEMM_OK : cuda_fail(e);
}

template <typename T>
gemm_status_t launch_zero(void *C, int64_t M, int64_t N, int64_t ldc, int sm_count, cudaStream_t stream) {
    const int64_t total = M * N;
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;
    if (blocks > cap) blocks = cap;
    b200::zero_fill_kernel<T><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(static_cast<T *>(C), M, N, ldc);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GEMM_OK : cuda_fail(e);
}

// The dense bf16 kernels, by configuration.
// `status`: the watchdog status block (the skinny kernel, which only the
// allocating entry points run, always uses the device's cudaMalloc'd one).
// The latency path: one ordinary launch, a 32 x 32 tile of C per CTA.
gemm_status_t launch_small(bool f32, const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                           int64_t lda, int64_t ldb, int64_t ldc, cudaStream_t stream, const b200::Epilogue &epi,
                           uint32_t layout) {
    const dim3 grid(static_cast<unsigned>((N + 31) / 32), static_cast<unsigned>((M + 31) / 32), 1);
    const uint16_t *a = static_cast<const uint16_t *>(A);
    const uint16_t *b = static_cast<const uint16_t *>(B);
    const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
    if (layout == 0) {   // K-major A and B: staged in shared memory
        if (f32) b200::gemm_bf16_small_kmajor_kernel<0><<<grid, 128, 0, stream>>>(a, b, C, m, n, k, lda, ldb, ldc, epi);
        else b200::gemm_bf16_small_kmajor_kernel<1><<<grid, 128, 0, stream>>>(a, b, C, m, n, k, lda, ldb, ldc, epi);
    } else {
        if (f32) b200::gemm_bf16_small_kernel<0><<<grid, 128, 0, stream>>>(a, b, C, m, n, k, lda, ldb, ldc, layout, epi);
        else b200::gemm_bf16_small_kernel<1><<<grid, 128, 0, stream>>>(a, b, C, m, n, k, lda, ldb, ldc, layout, epi);
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GEMM_OK : cuda_fail(e);
}

gemm_status_t launch_dense(DeviceState *st, DeviceStatus *status, gemm_config_t cfg, bool f32, const void *A,
                           const void *B, void *C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                           int64_t ldc, cudaStream_t stream, const b200::Epilogue &epi, uint32_t layout) {
    // the latency path's grid holds at most 65535 row blocks of 32
    if (cfg == GEMM_CFG_SMALL) {
        if ((M + 31) / 32 <= 65535)
            return launch_small(f32, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        cfg = GEMM_CFG_1CTA_128x128;
    }
    switch (cfg) {
        case GEMM_CFG_1CTA_128x256:
            return f32 ? launch_bf16<Cfg1x256F32>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_bf16<Cfg1x256B16>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_1CTA_128x128:
            return f32 ? launch_bf16<Cfg1x128F32>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_bf16<Cfg1x128B16>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_2CTA_256x256:
            return f32 ? launch_bf16<Cfg2x256F32>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_bf16<Cfg2x256B16>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_SKINNY:
            return launch_skinny_any(st, f32, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_2CTA_256x256_CLC:
            return f32 ? launch_bf16<Cfg2x256F32C>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_bf16<Cfg2x256B16C>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_2CTA_512x256_CLC:
            return f32 ? launch_bf16<Cfg2x512F32C>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_bf16<Cfg2x512B16C>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_2CTA_256x256_SK:
            return f32 ? launch_bf16<Cfg2x256F32S>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_bf16<Cfg2x256B16S>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_2CTA_256x224:
            // 224 columns are 3.5 chunks of 64 bf16, and each CTA's 112 rows
            // of a B stored K x N are not whole 64-wide MN-major boxes: those
            // take 256 x 256
            if (f32 && !(layout & b200::kLayoutBMajorN))
                return launch_bf16<Cfg2x224F32>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
            return launch_dense(st, status, GEMM_CFG_2CTA_256x256, f32, A, B, C, M, N, K, lda, ldb, ldc, stream, epi,
                                layout);
        case GEMM_CFG_1CTA_128x256_CLC:
            return f32 ? launch_bf16<Cfg1x256F32C>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_bf16<Cfg1x256B16C>(st, status, cfg, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_1CTA_128x128_SPLITK:
            return f32 ? launch_splitk<Cfg1x128F32K, Cfg1x128F32>(st, status, cfg, GEMM_CFG_1CTA_128x128, A, B, C, M,
                                                                   N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_splitk<Cfg1x128B16K, Cfg1x128B16>(st, status, cfg, GEMM_CFG_1CTA_128x128, A, B, C, M,
                                                                   N, K, lda, ldb, ldc, stream, epi, layout);
        case GEMM_CFG_1CTA_128x256_SPLITK:
            return f32 ? launch_splitk<Cfg1x256F32K, Cfg1x256F32>(st, status, cfg, GEMM_CFG_1CTA_128x256, A, B, C, M,
                                                                   N, K, lda, ldb, ldc, stream, epi, layout)
                       : launch_splitk<Cfg1x256B16K, Cfg1x256B16>(st, status, cfg, GEMM_CFG_1CTA_128x256, A, B, C, M,
                                                                   N, K, lda, ldb, ldc, stream, epi, layout);
        default:
            return GEMM_ERR_INVALID_VALUE;
    }
}

// ------------------------------------------------ allocation-free variant --
//
// gemm_bf16_noalloc runs the same kernels as gemm_bf16, but the kernels'
// scratch (the watchdog status block) lives in the file-scope array below
// instead of memory obtained from cudaMalloc.  The array is part of the
// library image: every GPU that loads the library holds its
// kNoAllocScratchBytes until the process exits.  All calls share it.  Kernel
// attributes and co-resident cluster counts are per kernel and device, so
// this entry point shares them with the others (g_devices).

constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Scratch one call needs: the status block, for every shape.
constexpr size_t noalloc_scratch_bytes() { return sizeof(DeviceStatus); }

// Per-device set-up, once, with the device current: the device checks of
// current_device, then the device address of the scratch array from
// cudaGetSymbolAddress (in host code the array's name is only a host-side
// stand-in, never a device address), zeroed once.  From then on the status
// block there is sticky: a recorded timeout stays until
// gemm_check_device_status() reads and clears it.
gemm_status_t noalloc_device(int &dev, DeviceState *&st, cudaStream_t stream) {
    gemm_status_t s = current_device(dev, st, stream);
    if (s != GEMM_OK) return s;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!st->noalloc_status) {
        if (capturing(stream)) return GEMM_ERR_CAPTURE;
        cudaError_t e;
        void *scratch = nullptr;
        if ((e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch)) != cudaSuccess || !scratch)
            return cuda_fail(e);
        if ((e = cudaMemset(scratch, 0, kNoAllocScratchBytes)) != cudaSuccess) return cuda_fail(e);
        st->noalloc_status = static_cast<DeviceStatus *>(scratch);
    }
    return GEMM_OK;
}

// ------------------------------------------------------ block-scaled path --

// Block-scaled configuration: CTA pairs (256 x 256) once there is a full wave
// of pair tiles, single CTAs (128 x 256) below that.
gemm_config_t select_mx_config(int64_t M, int64_t N) {
    const int forced = g_forced.load(std::memory_order_relaxed);
    if (forced == GEMM_CFG_MXFP8_1CTA_128x256 || forced == GEMM_CFG_MXFP8_2CTA_256x256)
        return static_cast<gemm_config_t>(forced);
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + 255) / 256);
    return pair_tiles >= 74 ? GEMM_CFG_MXFP8_2CTA_256x256 : GEMM_CFG_MXFP8_1CTA_128x256;
}

// Repacked-scale layout: 512-byte chunks, row block major ([rb][kb]).  A has
// a_blocks row blocks (padded to whole tiles), B has b_blocks (whole 256-row
// tiles); B's chunks follow A's.
struct MxLayout {
    int64_t kb, a_blocks, b_blocks;
    size_t bytes() const { return static_cast<size_t>((a_blocks + b_blocks) * kb * 512); }
};

MxLayout mx_layout(int64_t M, int64_t N, int64_t K, int cg) {
    MxLayout l;
    l.kb = (K + 127) / 128;
    l.a_blocks = cg == 2 ? 2 * ((M + 255) / 256) : (M + 127) / 128;
    l.b_blocks = 2 * ((N + 255) / 256);
    return l;
}

// Grows the device's workspace on demand.  Growing is refused inside a
// stream capture; the old buffer is retired, not freed (work queued on it,
// or a graph captured with its address, may still use it).
gemm_status_t mx_workspace(DeviceState *st, size_t bytes, uint8_t *&ws, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (st->mx_ws_bytes < bytes) {
        if (capturing(stream)) return GEMM_ERR_CAPTURE;
        cudaError_t e;
        if (st->mx_ws) {
            st->retired.push_back(st->mx_ws);
            st->mx_ws = nullptr;
            st->mx_ws_bytes = 0;
        }
        const size_t want = bytes < (size_t(1) << 20) ? (size_t(1) << 20) : bytes;
        if ((e = cudaMalloc(&st->mx_ws, want)) != cudaSuccess) return cuda_fail(e);
        st->mx_ws_bytes = want;
    }
    ws = st->mx_ws;
    return GEMM_OK;
}

template <class Cfg>
gemm_status_t launch_mxf8(DeviceState *st, int attr_slot, const void *A, const uint8_t *sfa, const void *B,
                          const uint8_t *sfb, void *C, int64_t M, int64_t N, int64_t K, int64_t lda,
                          int64_t ldb, int64_t ldc, cudaStream_t stream) {
    auto kernel = b200::gemm_mxf8_sm100_kernel<Cfg>;
    cudaError_t e;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Cfg::CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t lc = {};
    lc.blockDim = dim3(Cfg::THREADS, 1, 1);
    lc.dynamicSmemBytes = Cfg::SMEM_BYTES;
    lc.stream = stream;
    lc.attrs = attr;
    lc.numAttrs = 1;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!st->mx_attr_done[attr_slot]) {
            if (capturing(stream)) return GEMM_ERR_CAPTURE;
            if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          Cfg::SMEM_BYTES)) != cudaSuccess)
                return cuda_fail(e);
            int clusters = st->sm_count / Cfg::CG;
            if (Cfg::CG > 1) {
                lc.gridDim = dim3(Cfg::CG * clusters, 1, 1);
                int n = 0;
                if ((e = cudaOccupancyMaxActiveClusters(&n, kernel, &lc)) != cudaSuccess) return cuda_fail(e);
                if (n > 0) clusters = n;
            }
            st->mx_max_clusters[attr_slot] = clusters;
            st->mx_attr_done[attr_slot] = true;
        }
    }
    const MxLayout l = mx_layout(M, N, K, Cfg::CG);
    uint8_t *ws = nullptr;
    gemm_status_t s;
    if ((s = mx_workspace(st, l.bytes(), ws, stream)) != GEMM_OK) return s;

    // 1. scales -> TMEM-ready 512-byte chunks
    const int64_t blocks = (l.a_blocks + l.b_blocks) * ((l.kb + b200::kRepackKb - 1) / b200::kRepackKb);
    b200::mxf8_repack_scales_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        sfa, M, l.a_blocks, sfb, N, l.b_blocks, K / 32, l.kb, reinterpret_cast<uint32_t *>(ws));
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);

    // 2. the block-scaled GEMM; the scale chunks are read through a map that
    // sees the workspace as rows of 128 x 32-bit words (one chunk per row)
    alignas(64) CUtensorMap tmA, tmB, tmSF;
    if ((s = encode_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, lda, Cfg::BK, Cfg::BM_CTA)) != GEMM_OK) return s;
    if ((s = encode_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, ldb, Cfg::BK, Cfg::B_ROWS)) != GEMM_OK) return s;
    if ((s = encode_2d(&tmSF, CU_TENSOR_MAP_DATA_TYPE_UINT32, ws, 128, (l.a_blocks + l.b_blocks) * l.kb, 512, 128, 1,
                       CU_TENSOR_MAP_SWIZZLE_NONE)) != GEMM_OK)
        return s;
    const int64_t tiles = ((M + Cfg::BM - 1) / Cfg::BM) * ((N + Cfg::BN - 1) / Cfg::BN);
    const int64_t clusters = tiles < st->mx_max_clusters[attr_slot] ? tiles : st->mx_max_clusters[attr_slot];
    lc.gridDim = dim3(static_cast<unsigned>(clusters * Cfg::CG), 1, 1);
    // programmatic dependent launch: the GEMM's CTAs may start (barriers,
    // TMEM, tensor-map prefetch) while the repack finishes; its producer
    // waits on the repack's grid before the first load
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.numAttrs = 2;
    e = cudaLaunchKernelEx(&lc, kernel, tmA, tmB, tmSF, static_cast<int64_t>(l.a_blocks * l.kb),
                           static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), C, ldc, raster_group_m(),
                           st->status, watchdog_ns(K));
    if (e != cudaSuccess) return cuda_fail(e);
    return GEMM_OK;
}

}  // namespace

extern "C" {

gemm_status_t gemm_bf16_fused(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                              int64_t lda, int64_t ldb, int64_t ldc, gemm_out_t c_type, gemm_layout_t a_layout,
                              gemm_layout_t b_layout, float alpha, float beta, const float *bias, gemm_act_t act,
                              cudaStream_t stream) {
    if (c_type != GEMM_OUT_F32 && c_type != GEMM_OUT_BF16) return GEMM_ERR_INVALID_VALUE;
    if (act != GEMM_ACT_NONE && act != GEMM_ACT_RELU && act != GEMM_ACT_GELU && act != GEMM_ACT_GELU_TANH)
        return GEMM_ERR_INVALID_VALUE;
    if ((a_layout != GEMM_LAYOUT_KMAJOR && a_layout != GEMM_LAYOUT_MNMAJOR) ||
        (b_layout != GEMM_LAYOUT_KMAJOR && b_layout != GEMM_LAYOUT_MNMAJOR))
        return GEMM_ERR_INVALID_VALUE;
    const bool a_mn = a_layout == GEMM_LAYOUT_MNMAJOR, b_mn = b_layout == GEMM_LAYOUT_MNMAJOR;
    const int64_t ec = c_type == GEMM_OUT_F32 ? 4 : 2;
    gemm_status_t s = check_args(A, B, C, M, N, K, lda, ldb, ldc, 2, 2, ec, a_mn, b_mn);
    if (s != GEMM_OK || M == 0 || N == 0) return s;
    if (bias) {
        if (!aligned16(bias)) return GEMM_ERR_MISALIGNED;
        if (overlaps(C, M, N, ldc, ec, bias, 1, N, N, 4)) return GEMM_ERR_ALIAS;
    }
    const b200::Epilogue epi{alpha, beta, bias, static_cast<uint32_t>(act)};
    int dev;
    DeviceState *st;
    if ((s = current_device_alloc(dev, st, stream)) != GEMM_OK) return s;
    const bool f32 = c_type == GEMM_OUT_F32;
    if (K == 0) {
        // the empty sum: C = act(beta * C + bias); plain zeros (C not read)
        // when there is neither a beta term, a bias nor an activation
        if (beta == 0.0f && !bias && act == GEMM_ACT_NONE)
            return f32 ? launch_zero<uint32_t>(C, M, N, ldc, st->sm_count, stream)
                       : launch_zero<uint16_t>(C, M, N, ldc, st->sm_count, stream);
        return f32 ? launch_epilogue_only<float>(C, M, N, ldc, epi, st->sm_count, stream)
                   : launch_epilogue_only<__nv_bfloat16>(C, M, N, ldc, epi, st->sm_count, stream);
    }
    const uint32_t layout = (a_mn ? b200::kLayoutAMajorM : 0u) | (b_mn ? b200::kLayoutBMajorN : 0u);
    gemm_config_t cfg = select_config(M, N, K);
    // the skinny kernel reads A K-major only: an A stored K x M takes the
    // split-K tile kernel, which also spreads a long K over idle SMs
    if (cfg == GEMM_CFG_SKINNY && a_mn) cfg = GEMM_CFG_1CTA_128x128_SPLITK;
    // The two-consumer tile holds one tile in TMEM, so its epilogue stalls
    // the MMA; with epilogue work beyond the plain store (beta, bias, an
    // activation) the double-buffered 256 x 256 tile hides it instead.
    if (cfg == GEMM_CFG_2CTA_512x256_CLC && !epi.identity() && g_forced.load() == GEMM_CFG_AUTO)
        cfg = GEMM_CFG_2CTA_256x256_CLC;
    return launch_dense(st, st->status, cfg, f32, A, B, C, M, N, K, lda, ldb, ldc, stream, epi, layout);
}

gemm_status_t gemm_bf16_ex(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                           int64_t lda, int64_t ldb, int64_t ldc, gemm_out_t c_type, gemm_layout_t a_layout,
                           gemm_layout_t b_layout, float alpha, float beta, cudaStream_t stream) {
    return gemm_bf16_fused(A, B, C, M, N, K, lda, ldb, ldc, c_type, a_layout, b_layout, alpha, beta, nullptr,
                           GEMM_ACT_NONE, stream);
}

gemm_status_t gemm_bf16(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                        int64_t lda, int64_t ldb, int64_t ldc, gemm_out_t c_type, cudaStream_t stream) {
    return gemm_bf16_ex(A, B, C, M, N, K, lda, ldb, ldc, c_type, GEMM_LAYOUT_KMAJOR, GEMM_LAYOUT_KMAJOR, 1.0f, 0.0f,
                        stream);
}

gemm_status_t gemm_bf16_allgather(const void *A, const void *B, void *const *C_dst, int n_dst, int64_t M,
                                  int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int64_t row0,
                                  gemm_out_t c_type, cudaStream_t stream) {
    if (c_type != GEMM_OUT_F32 && c_type != GEMM_OUT_BF16) return GEMM_ERR_INVALID_VALUE;
    if (!C_dst || n_dst < 1 || n_dst > 1 + b200::kMaxPeerC || row0 < 0) return GEMM_ERR_INVALID_VALUE;
    const int64_t ec = c_type == GEMM_OUT_F32 ? 4 : 2;
    if (row0 > kMaxDim - M) return GEMM_ERR_TOO_LARGE;
    // each destination's slab: rows [row0, row0 + M) of a C with leading dimension ldc
    void *slab[1 + b200::kMaxPeerC];
    gemm_status_t s = GEMM_OK;
    for (int d = 0; d < n_dst; ++d) {
        if (!C_dst[d]) return GEMM_ERR_INVALID_VALUE;
        if (!aligned16(C_dst[d])) return GEMM_ERR_MISALIGNED;
        slab[d] = static_cast<uint8_t *>(C_dst[d]) + row0 * ldc * ec;
        if ((s = check_args(A, B, slab[d], M, N, K, lda, ldb, ldc, 2, 2, ec)) != GEMM_OK) return s;
        for (int e = 0; e < d; ++e)   // two destinations may not share bytes of the slab
            if (overlaps(slab[d], M, N, ldc, ec, slab[e], M, N, ldc, ec)) return GEMM_ERR_ALIAS;
    }
    if (M == 0 || N == 0) return GEMM_OK;
    int dev;
    DeviceState *st;
    if ((s = current_device_alloc(dev, st, stream)) != GEMM_OK) return s;
    const bool f32 = c_type == GEMM_OUT_F32;
    if (K == 0) {
        for (int d = 0; d < n_dst && s == GEMM_OK; ++d)
            s = f32 ? launch_zero<uint32_t>(slab[d], M, N, ldc, st->sm_count, stream)
                    : launch_zero<uint16_t>(slab[d], M, N, ldc, st->sm_count, stream);
        return s;
    }
    // The copies beyond the first: a tensor map of the slab in each (the same
    // box as the kernel's own C map) and the slab's base for the row ends.
    b200::PeerC peers{};
    peers.count = n_dst - 1;
    const int64_t n_tma = (N * ec / 16) * 16 / ec;
    const CUtensorMapDataType cdt = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint32_t box_cols = f32 ? Cfg2x256F32CP::EPI_COLS : Cfg2x256B16CP::EPI_COLS;
    for (int d = 1; d < n_dst; ++d) {
        if ((s = encode_2d(&peers.map[d - 1], cdt, slab[d], n_tma > 0 ? n_tma : 16 / ec, M, ldc * ec, box_cols, 32)) !=
            GEMM_OK)
            return s;
        peers.base[d - 1] = slab[d];
    }
    return f32 ? launch_bf16<Cfg2x256F32CP>(st, st->status, kCfgAllgather, A, B, slab[0], M, N, K, lda, ldb, ldc,
                                             stream, b200::plain_epilogue(), 0u, &peers)
               : launch_bf16<Cfg2x256B16CP>(st, st->status, kCfgAllgather, A, B, slab[0], M, N, K, lda, ldb, ldc,
                                             stream, b200::plain_epilogue(), 0u, &peers);
}

gemm_status_t gemm_mxfp8(const void *A, const uint8_t *sfa, const void *B, const uint8_t *sfb, void *C,
                         int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                         cudaStream_t stream) {
    gemm_status_t s = check_args(A, B, C, M, N, K, lda, ldb, ldc, 1, 1, 2);
    if (s != GEMM_OK || M == 0 || N == 0) return s;
    if (K % 32) return GEMM_ERR_INVALID_VALUE;
    if (K > 0) {
        if (!sfa || !sfb) return GEMM_ERR_INVALID_VALUE;
        if (overlaps(C, M, N, ldc, 2, sfa, 1, M * (K / 32), M * (K / 32), 1) ||
            overlaps(C, M, N, ldc, 2, sfb, 1, N * (K / 32), N * (K / 32), 1))
            return GEMM_ERR_ALIAS;
    }
    int dev;
    DeviceState *st;
    if ((s = current_device_alloc(dev, st, stream)) != GEMM_OK) return s;
    if (K == 0) return launch_zero<uint16_t>(C, M, N, ldc, st->sm_count, stream);
    if (select_mx_config(M, N) == GEMM_CFG_MXFP8_2CTA_256x256)
        return launch_mxf8<CfgMxf8Pair>(st, 1, A, sfa, B, sfb, C, M, N, K, lda, ldb, ldc, stream);
    return launch_mxf8<CfgMxf8>(st, 0, A, sfa, B, sfb, C, M, N, K, lda, ldb, ldc, stream);
}

gemm_status_t gemm_check_device_status(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e);
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GEMM_ERR_UNSUPPORTED_DEVICE;
    DeviceStatus *blocks[2];
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        blocks[0] = g_devices[dev].status;           // allocating entry points
        blocks[1] = g_devices[dev].noalloc_status;   // gemm_bf16_noalloc (static scratch)
    }
    // Both blocks are read and cleared; the first recorded event is reported.
    gemm_status_t result = GEMM_OK;
    for (DeviceStatus *status : blocks) {
        if (!status) continue;   // that entry point never ran on this device
        DeviceStatus h;
        if ((e = cudaMemcpy(&h, status, sizeof(h), cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e);
        if (h.code == 0) continue;
        if ((e = cudaMemset(status, 0, sizeof(DeviceStatus))) != cudaSuccess) return cuda_fail(e);
        if (result == GEMM_OK) {
            g_last_where = h.where;
            g_last_block = h.block;
            result = static_cast<gemm_status_t>(h.code);
        }
    }
    return result;
}

void gemm_last_timeout_detail(int32_t *where, int32_t *block) {
    if (where) *where = g_last_where;
    if (block) *block = g_last_block;
}

const char *gemm_status_string(gemm_status_t s) {
    switch (s) {
        case GEMM_OK: return "GEMM_OK: success";
        case GEMM_ERR_INVALID_VALUE: return "GEMM_ERR_INVALID_VALUE: negative size, leading dimension too small, null pointer or bad enum";
        case GEMM_ERR_MISALIGNED: return "GEMM_ERR_MISALIGNED: pointer or leading dimension not a multiple of 16 bytes";
        case GEMM_ERR_ALIAS: return "GEMM_ERR_ALIAS: C overlaps an input";
        case GEMM_ERR_UNSUPPORTED_DEVICE: return "GEMM_ERR_UNSUPPORTED_DEVICE: no CUDA device, or not compute capability 10.0 (B200)";
        case GEMM_ERR_LAUNCH: return "GEMM_ERR_LAUNCH: a CUDA runtime or driver call failed";
        case GEMM_ERR_TIMEOUT: return "GEMM_ERR_TIMEOUT: a bounded wait inside a kernel expired (device watchdog)";
        case GEMM_ERR_TOO_LARGE: return "GEMM_ERR_TOO_LARGE: a dimension or stride exceeds the TMA limits";
        case GEMM_ERR_CAPTURE: return "GEMM_ERR_CAPTURE: one-time set-up (device state, kernel attributes or workspace growth) cannot run inside a stream capture; make one call with the same shapes outside the capture first";
        default: return "unknown gemm_status_t";
    }
}

int gemm_last_cuda_error(void) { return g_last_cuda_error; }

gemm_status_t gemm_force_config(gemm_config_t config) {
    if (static_cast<int>(config) < 0 || static_cast<int>(config) >= GEMM_CFG_COUNT_) return GEMM_ERR_INVALID_VALUE;
    g_forced.store(static_cast<int>(config), std::memory_order_relaxed);
    return GEMM_OK;
}

gemm_config_t gemm_select_config(int64_t M, int64_t N, int64_t K) { return select_config(M, N, K); }

int gemm_launches_per_call(int64_t M, int64_t N, int64_t K, int block_scaled) {
    if (M <= 0 || N <= 0) return 0;
    return (block_scaled && K > 0) ? 2 : 1;
}

gemm_status_t gemm_bf16_noalloc(const void *A, const void *B, void *C, int64_t M, int64_t N, int64_t K,
                                int64_t lda, int64_t ldb, int64_t ldc, gemm_out_t c_type,
                                cudaStream_t stream) {
    if (c_type != GEMM_OUT_F32 && c_type != GEMM_OUT_BF16) return GEMM_ERR_INVALID_VALUE;
    const int64_t ec = c_type == GEMM_OUT_F32 ? 4 : 2;
    gemm_status_t s = check_args(A, B, C, M, N, K, lda, ldb, ldc, 2, 2, ec);
    if (s != GEMM_OK || M == 0 || N == 0) return s;
    if (noalloc_scratch_bytes() > kNoAllocScratchBytes) return GEMM_ERR_TOO_LARGE;
    int dev;
    DeviceState *st;
    if ((s = noalloc_device(dev, st, stream)) != GEMM_OK) return s;
    if (K == 0) {
        return c_type == GEMM_OUT_F32 ? launch_zero<uint32_t>(C, M, N, ldc, st->sm_count, stream)
                                      : launch_zero<uint16_t>(C, M, N, ldc, st->sm_count, stream);
    }
    // The stream-K kernels need a workspace; without one, small-M shapes run
    // on the skinny tile split over a cluster where that applies, else on
    // the split-K tile kernel (both sum their partials in shared memory),
    // and stream-K shapes on the CLC pair kernel.
    gemm_config_t cfg = select_config(M, N, K);
    if (cfg == GEMM_CFG_SKINNY) {
        bool launched = false;
        const bool f32 = c_type == GEMM_OUT_F32;
        s = f32 ? launch_skinny_cluster<CfgSk64F32C>(st, st->noalloc_status, 0, A, B, C, M, N, K, lda, ldb, ldc,
                                                     stream, b200::plain_epilogue(), 0u, launched)
                : launch_skinny_cluster<CfgSk64B16C>(st, st->noalloc_status, 1, A, B, C, M, N, K, lda, ldb, ldc,
                                                     stream, b200::plain_epilogue(), 0u, launched);
        if (s != GEMM_OK || launched) return s;
        cfg = GEMM_CFG_1CTA_128x128_SPLITK;
    }
    if (cfg == GEMM_CFG_2CTA_256x256_SK) cfg = GEMM_CFG_2CTA_256x256_CLC;   // stream-K needs a workspace too
    return launch_dense(st, st->noalloc_status, cfg, c_type == GEMM_OUT_F32, A, B, C, M, N, K, lda, ldb, ldc,
                        stream, b200::plain_epilogue(), 0u);
}

}  // extern "C"
