// pa_api.cu -- the extern "C" entry points of libpa_b200.so (declared and
// documented in include/pa.h): host-side validation, workspace layout,
// grid choice and kernel dispatch.  Every step of the computation runs in
// the kernels of pa_append.cuh, pa_prefix.cuh and pa_decode.cuh; there is no
// host or CPU fallback.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "pa_append.cuh"
#include "pa_decode.cuh"
#include "pa_device.cuh"
#include "pa_prefill.cuh"
#include "pa_prefill_tc.cuh"
#include "pa_prefix.cuh"

namespace {

constexpr int kBlockSize = 16;  // tokens per physical block the decode kernels are built for
constexpr int kMinPagesPerCta = 2;  // pages of a head group: fewest worth a CTA
constexpr int kMaxDevices = 64;
constexpr int kMaxCtas = 1024;  // the two-level split merge handles up to 16 x 64 pieces
constexpr float kLog2e = 1.4426950408889634f;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// The math policies: tensor-core (default) or fp32 CUDA-core for bf16
// caches; tensor-core for fp8 (E4M3) caches.
enum class MathKind { kMma, kSimt, kFp8 };

#ifndef PA_MAX_RING
#define PA_MAX_RING 64
#endif
// Deepest ring of stages whose CTA fits in shared memory, a multiple of
// the most stages a page can take (with 32 KB stages: 7 at head_dim 64,
// 6 at 128).
template <int D, int EB = 2>
constexpr int ring_fit() {
    using C1 = pa::DecodeCfg<D, kBlockSize, 1, EB>;
    int r = PA_MAX_RING;
    while (r > 1 && C1::kBaseBytes + (r - 1) * (C1::kStage + 16) > 232448) --r;
    r -= r % C1::kMaxSpl;
    return r;
}

// Fixed cost of finishing a segment, expressed as K+V bytes that could be
// streamed meanwhile, in pages of `heads` kv heads (rounded down);
// PA_SEG_WEIGHT_BYTES overrides it.
int32_t seg_weight_pages(int head_dim, int heads, int eb) {
    static const long long bytes = [] {
        const char* e = std::getenv("PA_SEG_WEIGHT_BYTES");
        return e ? std::atoll(e) : 65536LL;  // measured: 64 KB beats 32 KB on short contexts, equal on long
    }();
    const long long page = 2LL * kBlockSize * head_dim * eb * heads;
    return int32_t(bytes / page);
}

// kv heads per ring stage: as many whole K+V tiles (eb bytes per value) as a stage holds.
int heads_per_stage_max(int D, int eb) { return PA_STAGE_K_BYTES / (kBlockSize * D * eb); }

// kv heads per head group: the largest divisor of Hkv that is at most 8
// (one consumer warp per head) and splits into 1, 2, 4 or 8 equal stages.
int heads_per_group(int Hkv, int D, int eb) {
    const int hs = heads_per_stage_max(D, eb);
    for (int h = pa::kDecodeWarps; h > 1; --h) {
        if (Hkv % h) continue;
        for (int spl = 1; spl <= pa::kDecodeWarps; spl *= 2)
            if (h % spl == 0 && h / spl <= hs) return h;
    }
    return 1;
}

MathKind math_kind() {
    static const MathKind k = [] {
        const char* e = std::getenv("PA_DECODE_MATH");
        return (e && std::strcmp(e, "simt") == 0) ? MathKind::kSimt : MathKind::kMma;
    }();
    return k;
}

bool supported(int D, int G, MathKind mk) {
    if (D != 64 && D != 128) return false;
    if (G != 1 && G != 2 && G != 4 && G != 8) return false;
    return mk != MathKind::kSimt || G * D <= 256;
}

std::mutex g_mu;
int g_sms[kMaxDevices];

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int sm_count() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return -1;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

// Workspace layout: [counters: B*Hkv int32][part_o: grid*2*HG*G*D f32]
// [part_ml: grid*2*HG*G float2][group counters: grid*2*HG int32]
// [grid barrier of the fused append + decode: 2 uint32]
struct WsLayout {
    size_t counters, part_o, part_ml, slot_sync, grid_bar, total;
};

WsLayout ws_layout(const pa_dims& d, int grid) {
    // partial slots hold the query heads of one head group, at most min(Hkv, 8) kv heads (any cache format)
    const size_t hg_max = size_t(d.num_kv_heads < pa::kDecodeWarps ? d.num_kv_heads : pa::kDecodeWarps);
    const size_t hG = hg_max * (d.num_q_heads / d.num_kv_heads);
    WsLayout w;
    w.counters = 0;
    w.part_o = align_up(size_t(d.num_seqs) * d.num_kv_heads * 4, 256);
    w.part_ml = align_up(w.part_o + size_t(grid) * 2 * hG * d.head_dim * 4, 256);
    w.slot_sync = align_up(w.part_ml + size_t(grid) * 2 * hG * 8, 256);
    w.grid_bar = align_up(w.slot_sync + size_t(grid) * 2 * hg_max * 4, 256);
    w.total = w.grid_bar + 256;
    return w;
}

bool dims_ok(const pa_dims* d) {
    return d && d->num_seqs >= 0 && d->num_q_heads > 0 && d->num_kv_heads > 0 && d->head_dim > 0 &&
           d->block_size > 0 && d->num_blocks >= 0 && d->max_blocks_per_seq >= 0 &&
           d->num_q_heads % d->num_kv_heads == 0;
}

template <typename Kernel>
bool set_smem_once(Kernel kern, int bytes, unsigned* done_mask_per_device) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!done_mask_per_device[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return false;
        done_mask_per_device[dev] = 1;
    }
    return true;
}

#ifndef PA_L2_PROMOTION
#define PA_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif

// cuTensorMapEncodeTiled from the driver, found through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// A cache [NB][Hkv][bs][D] bf16 seen as a 4-D tensor {64 columns, bs rows,
// D/64 panels, NB*Hkv tiles} (strides D*2 B, 128 B, bs*D*2 B).  One box is
// `heads` consecutive (block, kv head) tiles whole: {64, bs, D/64, heads},
// landing in shared memory as [tile][panel][row][128 B] with the 128-byte
// swizzle.
bool make_cache_map(CUtensorMap* map, const void* base, int64_t tiles, int D, int bs, int heads) {
    auto fn = encode_tiled();
    if (!fn) return false;
    cuuint64_t dims[4] = {64, cuuint64_t(bs), cuuint64_t(D / 64), cuuint64_t(tiles)};
    cuuint64_t strides[3] = {cuuint64_t(D) * 2, 128, cuuint64_t(bs) * D * 2};
    cuuint32_t box[4] = {64, cuuint32_t(bs), cuuint32_t(D / 64), cuuint32_t(heads)};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, PA_L2_PROMOTION,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same 4-D view with a box of one 64-wide panel of one (block, kv head)
// tile: {64, 16, 1, 1} at {0, 0, panel, tile}, so a block of pages lands as
// [panel][tokens][128 bytes] (the tcgen05 operand layout).
bool make_panel_map(CUtensorMap* map, const void* base, int64_t tiles, int D, int bs) {
    auto fn = encode_tiled();
    if (!fn) return false;
    cuuint64_t dims[4] = {64, cuuint64_t(bs), cuuint64_t(D / 64), cuuint64_t(tiles)};
    cuuint64_t strides[3] = {cuuint64_t(D) * 2, 128, cuuint64_t(bs) * D * 2};
    cuuint32_t box[4] = {64, cuuint32_t(bs), 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, PA_L2_PROMOTION,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An fp8 cache seen as a 4-D uint8 tensor {128 bytes, D/8 lines, 1, NB*Hkv
// tiles} (rank 4 like the bf16 maps, so that the decode's 4-D tiled load
// {0, 0, 0, tile} serves both): one (block, kv head) tile is 16*D bytes =
// D/8 lines of 128 bytes (K: 16 tokens of D codes; V: D rows of 16 tokens).
// One box is `heads` consecutive tiles whole.  K takes the 128-byte swizzle
// (a line holds one token at head_dim 128, two at 64); V^T rows are 16
// bytes and need none.
bool make_fp8_map(CUtensorMap* map, const void* base, int64_t tiles, int D, int heads, bool swizzle) {
    auto fn = encode_tiled();
    if (!fn) return false;
    cuuint64_t dims[4] = {128, cuuint64_t(D / 8), 1, cuuint64_t(tiles)};
    cuuint64_t strides[3] = {128, cuuint64_t(16) * D, cuuint64_t(16) * D};
    cuuint32_t box[4] = {128, cuuint32_t(D / 8), 1, cuuint32_t(heads)};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              PA_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// pdl: launched as a programmatic dependent of the kernel before it in the
// stream (prefix_kernel), so that its set-up overlaps that kernel's end.
template <MathKind MK, int D, int G, bool DUMP, bool APPEND>
pa_status launch_decode(const pa::DecodeParams& p, int grid, cudaStream_t stream, bool pdl) {
    constexpr int EB = MK == MathKind::kFp8 ? 1 : 2;
    constexpr int R = ring_fit<D, EB>();
    using Cfg = pa::DecodeCfg<D, kBlockSize, R, EB>;
    auto kern = [] {
        if constexpr (MK == MathKind::kMma)
            return pa::decode_kernel<D, G, kBlockSize, R, DUMP, APPEND, pa::MmaMath>;
        else if constexpr (MK == MathKind::kFp8)
            return pa::decode_kernel<D, G, kBlockSize, R, DUMP, APPEND, pa::Fp8MmaMath>;
        else
            return pa::decode_kernel<D, G, kBlockSize, R, DUMP, APPEND, pa::SimtMath>;
    }();
    static unsigned attr_done[kMaxDevices];
    if (!set_smem_once(kern, Cfg::kSmemBytes, attr_done)) return PA_ERR_CUDA;
    // the rest of shared memory is needed only to stage prefix partials
    const int smem = p.num_groups > 0 ? Cfg::kSmemBytes : Cfg::kBaseBytes;
    if (APPEND && !p.app_local) {
        // the CTAs meet at a grid barrier: a cooperative launch guarantees they are all resident
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(Cfg::kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return PA_ERR_CUDA;
    } else if (pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(Cfg::kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return PA_ERR_CUDA;
    } else {
        kern<<<grid, Cfg::kThreads, smem, stream>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// The SIMT policy is built only for G*D <= 256 (its per-lane state grows with G*D).
template <MathKind MK, int D, int G, bool DUMP, bool APPEND>
pa_status launch_built(const pa::DecodeParams& p, int grid, cudaStream_t s, bool pdl) {
    if constexpr (MK == MathKind::kFp8 && DUMP)
        return PA_ERR_UNSUPPORTED;  // fp8: no partials test hook
    else if constexpr (MK != MathKind::kSimt || G * D <= 256)
        return launch_decode<MK, D, G, DUMP, APPEND>(p, grid, s, pdl);
    else
        return PA_ERR_UNSUPPORTED;
}

template <MathKind MK, bool DUMP, bool APPEND>
pa_status dispatch_d_g(int D, int G, const pa::DecodeParams& p, int grid, cudaStream_t s, bool pdl) {
    if (D == 64) {
        switch (G) {
            case 1: return launch_built<MK, 64, 1, DUMP, APPEND>(p, grid, s, pdl);
            case 2: return launch_built<MK, 64, 2, DUMP, APPEND>(p, grid, s, pdl);
            case 4: return launch_built<MK, 64, 4, DUMP, APPEND>(p, grid, s, pdl);
            case 8: return launch_built<MK, 64, 8, DUMP, APPEND>(p, grid, s, pdl);
        }
    } else if (D == 128) {
        switch (G) {
            case 1: return launch_built<MK, 128, 1, DUMP, APPEND>(p, grid, s, pdl);
            case 2: return launch_built<MK, 128, 2, DUMP, APPEND>(p, grid, s, pdl);
            case 4: return launch_built<MK, 128, 4, DUMP, APPEND>(p, grid, s, pdl);
            case 8: return launch_built<MK, 128, 8, DUMP, APPEND>(p, grid, s, pdl);
        }
    }
    return PA_ERR_UNSUPPORTED;
}

template <bool DUMP, bool APPEND = false>
pa_status dispatch_decode(int D, int G, const pa::DecodeParams& p, int grid, cudaStream_t s, bool pdl = false) {
    return math_kind() == MathKind::kMma ? dispatch_d_g<MathKind::kMma, DUMP, APPEND>(D, G, p, grid, s, pdl)
                                         : dispatch_d_g<MathKind::kSimt, DUMP, APPEND>(D, G, p, grid, s, pdl);
}

// tcgen05 prefill configurations: BN keys per block, KS blocks in the ring,
// CPS CTAs per SM.
template <int D, int BN> constexpr int tc_stages() {
    return BN == 128 ? (D == 64 ? 4 : 3) : (D == 64 ? 5 : 2);
}

template <int D, int BN>
struct TcShape {
    static constexpr int KS = tc_stages<D, BN>(), CPS = BN == 128 ? 1 : 2;
    // S buffers: as many as TMEM holds next to O for CPS CTAs per SM
    static constexpr int NS = (3 * BN + D) * CPS <= 512 ? 3 : 2;
    using Cfg = pa::TcPrefillCfg<D, BN, KS, NS>;
    static_assert(CPS * (Cfg::kSmemBytes + 1024) <= 233472, "CTAs per SM by shared memory");
    static_assert(CPS * Cfg::kTmemCols <= 512, "CTAs per SM by TMEM columns");
};

template <int D, int G, int BN>
pa_status launch_prefill_tc(const pa::PrefillParams& p, dim3 grid, cudaStream_t stream) {
    using S = TcShape<D, BN>;
    auto kern = pa::prefill_tc_kernel<D, G, BN, S::KS, S::CPS, S::NS>;
    static unsigned attr_done[kMaxDevices];
    if (!set_smem_once(kern, S::Cfg::kSmemBytes, attr_done)) return PA_ERR_CUDA;
    kern<<<grid, S::Cfg::kThreads, S::Cfg::kSmemBytes, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D, int G, int BN>
pa_status launch_prefix_tc(const pa::PrefixParams& p, dim3 grid, cudaStream_t stream) {
    using S = TcShape<D, BN>;
    auto kern = pa::prefix_tc_kernel<D, G, BN, S::KS, S::CPS, S::NS>;
    static unsigned attr_done[kMaxDevices];
    if (!set_smem_once(kern, S::Cfg::kSmemBytes, attr_done)) return PA_ERR_CUDA;
    kern<<<grid, S::Cfg::kThreads, S::Cfg::kSmemBytes, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// PA_PREFILL_BN=64|128 picks the block size (keys per softmax step).
int prefill_bn() {
    static const int v = [] {
        const char* e = std::getenv("PA_PREFILL_BN");
        return (e && std::atoi(e) == 128) ? 128 : 64;
    }();
    return v;
}

template <int D, int G>
pa_status launch_prefill_tc(const pa::PrefillParams& p, dim3 grid, cudaStream_t s) {
    return prefill_bn() == 128 ? launch_prefill_tc<D, G, 128>(p, grid, s) : launch_prefill_tc<D, G, 64>(p, grid, s);
}

template <int D, int G>
pa_status launch_prefix_tc(const pa::PrefixParams& p, dim3 grid, cudaStream_t s) {
    return prefill_bn() == 128 ? launch_prefix_tc<D, G, 128>(p, grid, s) : launch_prefix_tc<D, G, 64>(p, grid, s);
}

// PA_PREFILL_MMA=sync selects the warp-level mma.sync kernels (prefill and
// shared-prefix pass; kept for comparison).
bool prefill_use_mma_sync() {
    static const bool v = [] {
        const char* e = std::getenv("PA_PREFILL_MMA");
        return e && std::strcmp(e, "sync") == 0;
    }();
    return v;
}

// ---- shared-prefix pass ----------------------------------------------------
constexpr int kPrefixNW = 8;      // consumer warps: 128 query rows per CTA
constexpr int kPrefixStages = 8;  // ring of K+V pages
constexpr int kMaxPrefixSplits = 16;
// Time model of the shared-prefix pass (head_dim 128, 64-key blocks, B200),
// and a decode CTA's page stream meanwhile; they only weight the decode's split.
constexpr int32_t kPrefixPassNs = 7000;
constexpr int32_t kPrefixPassNsPerPage = 200;
constexpr int64_t kDecodeCtaBytesPerMs = 36000000;

int prefix_tiles(const pa_dims& d, int max_group_size) {
    const int64_t rows = int64_t(max_group_size) * (d.num_q_heads / d.num_kv_heads);
    return int((rows + 16 * kPrefixNW - 1) / (16 * kPrefixNW));
}

// Key ranges per (group, row tile, kv head): enough CTAs for half a wave, so
// that the decode starts at once on the SMs the pass leaves free (its split
// gives those CTAs more of the line); PA_PREFIX_SPLITS=n overrides, 1..16.
// Measured on the 256-member prefix batch: 47.9 us per step against 49.7 at a
// whole wave of equal shares.
int prefix_splits(const pa_dims& d, int num_groups, int max_group_size, int sms) {
    static const int forced = [] {
        const char* e = std::getenv("PA_PREFIX_SPLITS");
        return e ? std::atoi(e) : 0;
    }();
    if (forced >= 1 && forced <= kMaxPrefixSplits) return forced;
    const int64_t base = int64_t(num_groups) * prefix_tiles(d, max_group_size) * d.num_kv_heads;
    int64_t s = base > 0 ? sms / (2 * base) : 1;
    if (s < 1) s = 1;
    if (s > kMaxPrefixSplits) s = kMaxPrefixSplits;
    return int(s);
}

// The prefix partials follow the decode workspace: [o: splits*B*Hq*D f32][ml: splits*B*Hq float2]
struct PrefixWs {
    size_t o, ml, total;
};

PrefixWs prefix_ws(const pa_dims& d, size_t base, int splits) {
    const size_t rows = size_t(splits) * d.num_seqs * d.num_q_heads;
    PrefixWs w;
    w.o = align_up(base, 256);
    w.ml = align_up(w.o + rows * d.head_dim * 4, 256);
    w.total = w.ml + rows * 8;
    return w;
}

template <int D, int G>
pa_status launch_prefix(const pa::PrefixParams& p, dim3 grid, cudaStream_t stream) {
    using Cfg = pa::PrefixCfg<D, kPrefixNW, kPrefixStages>;
    auto kern = pa::prefix_kernel<D, G, kPrefixNW, kPrefixStages>;
    static unsigned attr_done[kMaxDevices];
    if (!set_smem_once(kern, Cfg::kSmemBytes, attr_done)) return PA_ERR_CUDA;
    kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status dispatch_prefix_tc(int D, int G, const pa::PrefixParams& p, dim3 grid, cudaStream_t s) {
    if (D == 64) {
        switch (G) {
            case 1: return launch_prefix_tc<64, 1>(p, grid, s);
            case 2: return launch_prefix_tc<64, 2>(p, grid, s);
            case 4: return launch_prefix_tc<64, 4>(p, grid, s);
            case 8: return launch_prefix_tc<64, 8>(p, grid, s);
        }
    } else if (D == 128) {
        switch (G) {
            case 1: return launch_prefix_tc<128, 1>(p, grid, s);
            case 2: return launch_prefix_tc<128, 2>(p, grid, s);
            case 4: return launch_prefix_tc<128, 4>(p, grid, s);
            case 8: return launch_prefix_tc<128, 8>(p, grid, s);
        }
    }
    return PA_ERR_UNSUPPORTED;
}

pa_status dispatch_prefix(int D, int G, const pa::PrefixParams& p, dim3 grid, cudaStream_t s) {
    if (!prefill_use_mma_sync()) return dispatch_prefix_tc(D, G, p, grid, s);
    if (D == 64) {
        switch (G) {
            case 1: return launch_prefix<64, 1>(p, grid, s);
            case 2: return launch_prefix<64, 2>(p, grid, s);
            case 4: return launch_prefix<64, 4>(p, grid, s);
            case 8: return launch_prefix<64, 8>(p, grid, s);
        }
    } else if (D == 128) {
        switch (G) {
            case 1: return launch_prefix<128, 1>(p, grid, s);
            case 2: return launch_prefix<128, 2>(p, grid, s);
            case 4: return launch_prefix<128, 4>(p, grid, s);
            case 8: return launch_prefix<128, 8>(p, grid, s);
        }
    }
    return PA_ERR_UNSUPPORTED;
}

// ---- multi-query (chunked prefill) attention -----------------------------------
template <int D, int G>
pa_status launch_prefill(const pa::PrefillParams& p, dim3 grid, cudaStream_t stream) {
    using Cfg = pa::PrefixCfg<D, kPrefixNW, kPrefixStages>;
    auto kern = pa::prefill_kernel<D, G, kPrefixNW, kPrefixStages>;
    static unsigned attr_done[kMaxDevices];
    if (!set_smem_once(kern, Cfg::kSmemBytes, attr_done)) return PA_ERR_CUDA;
    kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status dispatch_prefill_tc(int D, int G, const pa::PrefillParams& p, dim3 grid, cudaStream_t s) {
    if (D == 64) {
        switch (G) {
            case 1: return launch_prefill_tc<64, 1>(p, grid, s);
            case 2: return launch_prefill_tc<64, 2>(p, grid, s);
            case 4: return launch_prefill_tc<64, 4>(p, grid, s);
            case 8: return launch_prefill_tc<64, 8>(p, grid, s);
        }
    } else if (D == 128) {
        switch (G) {
            case 1: return launch_prefill_tc<128, 1>(p, grid, s);
            case 2: return launch_prefill_tc<128, 2>(p, grid, s);
            case 4: return launch_prefill_tc<128, 4>(p, grid, s);
            case 8: return launch_prefill_tc<128, 8>(p, grid, s);
        }
    }
    return PA_ERR_UNSUPPORTED;
}

pa_status dispatch_prefill(int D, int G, const pa::PrefillParams& p, dim3 grid, cudaStream_t s) {
    if (D == 64) {
        switch (G) {
            case 1: return launch_prefill<64, 1>(p, grid, s);
            case 2: return launch_prefill<64, 2>(p, grid, s);
            case 4: return launch_prefill<64, 4>(p, grid, s);
            case 8: return launch_prefill<64, 8>(p, grid, s);
        }
    } else if (D == 128) {
        switch (G) {
            case 1: return launch_prefill<128, 1>(p, grid, s);
            case 2: return launch_prefill<128, 2>(p, grid, s);
            case 4: return launch_prefill<128, 4>(p, grid, s);
            case 8: return launch_prefill<128, 8>(p, grid, s);
        }
    }
    return PA_ERR_UNSUPPORTED;
}

// Shared validation of pa_decode and pa_decode_partials; fills p.
pa_status prepare_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                         const int32_t* context_lens, float scale, void* out, const pa_dims* dims, int grid,
                         void* workspace, size_t workspace_bytes, pa::DecodeParams& p, int eb = 2) {
    if (!dims) return PA_ERR_NULL;
    if (!dims_ok(dims)) return PA_ERR_SHAPE;
    const pa_dims& d = *dims;
    const int G = d.num_q_heads / d.num_kv_heads;
    if (d.block_size != kBlockSize || !supported(d.head_dim, G, eb == 1 ? MathKind::kFp8 : math_kind()))
        return PA_ERR_UNSUPPORTED;
    if (d.num_seqs == 0) return PA_OK;
    // at least one block, so that a bad block id can be redirected to block 0
    if (d.num_blocks == 0) return PA_ERR_SHAPE;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out || !workspace) return PA_ERR_NULL;
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(workspace) || !aligned4(block_tables) || !aligned4(context_lens))
        return PA_ERR_ALIGN;
    if (grid <= 0) return PA_ERR_CUDA;
    if (grid > kMaxCtas) return PA_ERR_SHAPE;
    const WsLayout w = ws_layout(d, grid);
    if (workspace_bytes < w.total) return PA_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p = pa::DecodeParams{};
    const int64_t rows = int64_t(d.num_blocks) * d.num_kv_heads * d.block_size;
    if (rows >= (int64_t(1) << 31)) return PA_ERR_SHAPE;  // TMA coordinates are int32
    const int HG = heads_per_group(d.num_kv_heads, d.head_dim, eb);
    int SPL = 1;
    while (HG / SPL > heads_per_stage_max(d.head_dim, eb) || HG % SPL) SPL *= 2;
    const int HS = HG / SPL;
    const int64_t tiles = int64_t(d.num_blocks) * d.num_kv_heads;
    const bool maps_ok =
        eb == 2 ? make_cache_map(&p.tmap_k, k_cache, tiles, d.head_dim, d.block_size, HS) &&
                      make_cache_map(&p.tmap_v, v_cache, tiles, d.head_dim, d.block_size, HS)
                : make_fp8_map(&p.tmap_k, k_cache, tiles, d.head_dim, HS, true) &&
                      make_fp8_map(&p.tmap_v, v_cache, tiles, d.head_dim, HS, false);
    if (!maps_ok) return PA_ERR_CUDA;
    p.q = static_cast<const uint8_t*>(q);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.qscale = scale * kLog2e;
    p.B = d.num_seqs;
    p.Hq = d.num_q_heads;
    p.Hkv = d.num_kv_heads;
    p.NB = d.num_blocks;
    p.M = d.max_blocks_per_seq;
    p.HG = HG;
    p.NG = d.num_kv_heads / HG;
    p.HS = HS;
    p.SPL = SPL;
    p.SPL_LOG = SPL == 1 ? 0 : SPL == 2 ? 1 : SPL == 4 ? 2 : 3;
    p.min_pages = kMinPagesPerCta;
    p.seg_weight = seg_weight_pages(d.head_dim, HG, eb);
    p.counters = reinterpret_cast<int32_t*>(ws + w.counters);
    p.part_o = reinterpret_cast<float*>(ws + w.part_o);
    p.part_ml = reinterpret_cast<float2*>(ws + w.part_ml);
    p.slot_sync = reinterpret_cast<int32_t*>(ws + w.slot_sync);
    p.grid_bar = reinterpret_cast<unsigned int*>(ws + w.grid_bar);
    return PA_OK;
}

}  // namespace

// ---- scratch for the allocation-free decode (pa_decode_static_ws) ----------
// A fixed device array, present on every GPU that loads the library.  Host
// code may only use the name as a symbol handle: its device address comes
// from cudaGetSymbolAddress, looked up once per device with that device
// current (a kernel given the host-side name would read the wrong memory).
static __device__ __align__(256) unsigned char g_pa_static_scratch[PA_STATIC_SCRATCH_BYTES];

namespace {
void* g_static_scratch_addr[kMaxDevices];  // per device, guarded by g_mu

pa_status static_scratch_address(void** addr) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_static_scratch_addr[dev]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_pa_static_scratch) != cudaSuccess || !a) return PA_ERR_CUDA;
        g_static_scratch_addr[dev] = a;
    }
    *addr = g_static_scratch_addr[dev];
    return PA_OK;
}
}  // namespace

extern "C" {

const char* pa_status_string(int32_t status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_NULL: return "PA_ERR_NULL: a required pointer is NULL";
        case PA_ERR_SHAPE: return "PA_ERR_SHAPE: invalid or inconsistent sizes";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: head_dim/block_size/GQA group not built";
        case PA_ERR_ALIGN: return "PA_ERR_ALIGN: tensor pointer not 16-byte aligned";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace missing or too small";
        case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime call failed";
        case PA_ERR_SCRATCH_LIMIT:
            return "PA_ERR_SCRATCH_LIMIT: problem needs more scratch than PA_STATIC_SCRATCH_BYTES";
        default: return "unknown pa_status";
    }
}

pa_status pa_cache_append(const void* k_new, const void* v_new, const int32_t* slot_mapping, int32_t num_tokens,
                          void* k_cache, void* v_cache, const pa_dims* dims, void* stream) {
    if (!dims) return PA_ERR_NULL;
    const pa_dims& d = *dims;
    if (num_tokens < 0 || d.num_kv_heads <= 0 || d.head_dim <= 0 || d.block_size <= 0 || d.num_blocks < 0)
        return PA_ERR_SHAPE;
    if (d.head_dim % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache) return PA_ERR_NULL;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(slot_mapping))
        return PA_ERR_ALIGN;
    pa::AppendParams p;
    p.k_new = static_cast<const uint4*>(k_new);
    p.v_new = static_cast<const uint4*>(v_new);
    p.slot_mapping = slot_mapping;
    p.k_cache = static_cast<uint4*>(k_cache);
    p.v_cache = static_cast<uint4*>(v_cache);
    p.chunks_per_row = d.head_dim / 8;
    p.num_chunks = int64_t(num_tokens) * d.num_kv_heads * p.chunks_per_row;
    p.kv_heads = d.num_kv_heads;
    p.block_size = d.block_size;
    p.num_blocks = d.num_blocks;
    const int64_t blocks = (p.num_chunks + pa::kAppendThreads - 1) / pa::kAppendThreads;
    if (blocks > 0x7fffffff) return PA_ERR_SHAPE;
    pa::append_kernel<<<unsigned(blocks), pa::kAppendThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int32_t pa_decode_default_ctas(void) { return sm_count(); }

size_t pa_decode_workspace_bytes(const pa_dims* dims, int32_t num_ctas) {
    if (!dims_ok(dims)) return 0;
    const int grid = num_ctas > 0 ? num_ctas : sm_count();
    if (grid <= 0) return 0;
    return ws_layout(*dims, grid).total;
}

pa_status pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                    const int32_t* context_lens, float scale, void* out, const pa_dims* dims, void* workspace,
                    size_t workspace_bytes, void* stream) {
    pa::DecodeParams p;
    const int grid = sm_count();
    const pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, dims,
                                        grid, workspace, workspace_bytes, p);
    if (st != PA_OK || dims->num_seqs == 0) return st;
    return dispatch_decode<false>(dims->head_dim, dims->num_q_heads / dims->num_kv_heads, p, grid,
                                  static_cast<cudaStream_t>(stream));
}

pa_status pa_decode_partials(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             const int32_t* context_lens, float scale, void* out, const pa_dims* dims,
                             int32_t num_ctas, void* workspace, size_t workspace_bytes, int32_t capacity,
                             int32_t* seg_meta, float* seg_o, float* seg_m, float* seg_l, int32_t* seg_count,
                             void* stream) {
    if (num_ctas <= 0 || capacity < 0) return PA_ERR_SHAPE;
    pa::DecodeParams p;
    const pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, dims,
                                        num_ctas, workspace, workspace_bytes, p);
    if (st != PA_OK || dims->num_seqs == 0) return st;
    if (!seg_count || (capacity > 0 && (!seg_meta || !seg_o || !seg_m || !seg_l))) return PA_ERR_NULL;
    p.min_pages = 1;
    p.dump_capacity = capacity;
    p.seg_meta = seg_meta;
    p.seg_o = seg_o;
    p.seg_m = seg_m;
    p.seg_l = seg_l;
    p.seg_count = seg_count;
    return dispatch_decode<true>(dims->head_dim, dims->num_q_heads / dims->num_kv_heads, p, num_ctas,
                                 static_cast<cudaStream_t>(stream));
}

pa_status pa_append_decode(const void* k_new, const void* v_new, const int32_t* slot_mapping, int32_t num_tokens,
                           const void* q, void* k_cache, void* v_cache, const int32_t* block_tables,
                           const int32_t* context_lens, float scale, void* out, const pa_dims* dims, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (!dims) return PA_ERR_NULL;
    if (num_tokens < 0) return PA_ERR_SHAPE;
    pa::DecodeParams p;
    const int grid = sm_count();
    const pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, dims, grid,
                                        workspace, workspace_bytes, p);
    if (st != PA_OK) return st;
    if (num_tokens > 0) {
        if (!k_new || !v_new || !slot_mapping) return PA_ERR_NULL;
        if (!aligned16(k_new) || !aligned16(v_new) || !aligned4(slot_mapping)) return PA_ERR_ALIGN;
    }
    if (dims->num_seqs == 0) {  // nothing to attend over: the append alone
        return pa_cache_append(k_new, v_new, slot_mapping, num_tokens, k_cache, v_cache, dims, stream);
    }
    p.k_new = static_cast<const uint4*>(k_new);
    p.v_new = static_cast<const uint4*>(v_new);
    p.slot_mapping = slot_mapping;
    p.app_chunks = int64_t(num_tokens) * dims->num_kv_heads * (dims->head_dim / 8);
    p.app_tokens = num_tokens;
    p.app_local = num_tokens <= pa::kLocalMaxTokens;
    p.k_cache_w = static_cast<uint4*>(k_cache);
    p.v_cache_w = static_cast<uint4*>(v_cache);
    return dispatch_decode<false, true>(dims->head_dim, dims->num_q_heads / dims->num_kv_heads, p, grid,
                                        static_cast<cudaStream_t>(stream));
}

size_t pa_decode_shared_prefix_workspace_bytes(const pa_dims* dims, int32_t num_groups, int32_t max_group_size) {
    if (!dims_ok(dims) || num_groups < 0 || (num_groups > 0 && max_group_size <= 0)) return 0;
    const int grid = sm_count();
    if (grid <= 0) return 0;
    const size_t base = ws_layout(*dims, grid).total;
    if (num_groups == 0) return base;
    const int mgs = max_group_size < dims->num_seqs ? max_group_size : dims->num_seqs;
    return prefix_ws(*dims, base, prefix_splits(*dims, num_groups, mgs, grid)).total;
}

pa_status pa_decode_shared_prefix(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                                  int32_t num_tokens, const void* q, void* k_cache, void* v_cache,
                                  const int32_t* block_tables, const int32_t* context_lens, float scale,
                                  const int32_t* group_offsets, const int32_t* group_prefix_pages, int32_t num_groups,
                                  int32_t max_group_size, void* out, const pa_dims* dims, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    if (!dims) return PA_ERR_NULL;
    if (num_tokens < 0 || num_groups < 0 || (num_groups > 0 && max_group_size <= 0)) return PA_ERR_SHAPE;
    pa::DecodeParams p;
    const int grid = sm_count();
    const pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, dims, grid,
                                        workspace, workspace_bytes, p);
    if (st != PA_OK) return st;
    if (num_tokens > 0) {
        if (!k_new || !v_new || !slot_mapping) return PA_ERR_NULL;
        if (!aligned16(k_new) || !aligned16(v_new) || !aligned4(slot_mapping)) return PA_ERR_ALIGN;
    }
    const pa_dims& d = *dims;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d.num_seqs == 0)
        return num_tokens > 0 ? pa_cache_append(k_new, v_new, slot_mapping, num_tokens, k_cache, v_cache, dims, stream)
                              : PA_OK;
    const int G = d.num_q_heads / d.num_kv_heads;
    if (num_groups > 0) {
        if (!group_offsets || !group_prefix_pages) return PA_ERR_NULL;
        if (!aligned4(group_offsets) || !aligned4(group_prefix_pages)) return PA_ERR_ALIGN;
        const int mgs = max_group_size < d.num_seqs ? max_group_size : d.num_seqs;
        const int splits = prefix_splits(d, num_groups, mgs, grid);
        const PrefixWs w = prefix_ws(d, ws_layout(d, grid).total, splits);
        if (workspace_bytes < w.total) return PA_ERR_WORKSPACE;
        const int tiles = prefix_tiles(d, mgs);
        if (int64_t(num_groups) * tiles > 0x7fffffffLL || d.num_kv_heads > 65535) return PA_ERR_SHAPE;
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        pa::PrefixParams pp;
        const int64_t cache_tiles = int64_t(d.num_blocks) * d.num_kv_heads;
        const bool maps_ok =
            prefill_use_mma_sync()
                ? make_cache_map(&pp.tmap_k, k_cache, cache_tiles, d.head_dim, d.block_size, 1) &&
                      make_cache_map(&pp.tmap_v, v_cache, cache_tiles, d.head_dim, d.block_size, 1)
                : make_panel_map(&pp.tmap_k, k_cache, cache_tiles, d.head_dim, d.block_size) &&
                      make_panel_map(&pp.tmap_v, v_cache, cache_tiles, d.head_dim, d.block_size);
        if (!maps_ok)
            return PA_ERR_CUDA;
        pp.q = p.q;
        pp.block_tables = block_tables;
        pp.context_lens = context_lens;
        pp.group_offsets = group_offsets;
        pp.group_prefix_pages = group_prefix_pages;
        pp.num_groups = num_groups;
        pp.max_group_size = mgs;
        pp.tiles_per_group = tiles;
        pp.B = d.num_seqs;
        pp.Hq = d.num_q_heads;
        pp.Hkv = d.num_kv_heads;
        pp.NB = d.num_blocks;
        pp.M = d.max_blocks_per_seq;
        pp.qscale = p.qscale;
        pp.prefix_o = reinterpret_cast<float*>(ws + w.o);
        pp.prefix_ml = reinterpret_cast<float2*>(ws + w.ml);
        // Up to kLocalMaxTokens new rows are appended by the decode itself
        // (each CTA writes the rows of the blocks it reads), so the decode
        // streams its pages while the prefix pass runs and waits for the pass
        // only before reading its partials; more rows ride on the prefix
        // launch and the decode waits for the pass before reading anything.
        const bool local = num_tokens <= pa::kLocalMaxTokens;
        pp.k_new = static_cast<const uint4*>(k_new);
        pp.v_new = static_cast<const uint4*>(v_new);
        pp.slot_mapping = slot_mapping;
        pp.app_chunks = local ? 0 : int64_t(num_tokens) * d.num_kv_heads * (d.head_dim / 8);
        pp.k_cache_w = static_cast<uint4*>(k_cache);
        pp.v_cache_w = static_cast<uint4*>(v_cache);
        const pa_status ps = dispatch_prefix(d.head_dim, G, pp, dim3(unsigned(num_groups * tiles),
                                                                     unsigned(d.num_kv_heads), unsigned(splits)), s);
        if (ps != PA_OK) return ps;
        p.group_offsets = group_offsets;
        p.group_prefix_pages = group_prefix_pages;
        p.num_groups = num_groups;
        p.max_group_size = mgs;
        p.prefix_splits = splits;
        // CTAs that find an SM the prefix pass leaves free start at once and
        // take more of the line (the prefix pass, one CTA per SM, as measured:
        // ~7 us of set-up and end plus ~0.2 us per prefix page of its key range;
        // a CTA streams ~36 GB/s of pages meanwhile)
        const int64_t prefix_ctas = int64_t(num_groups) * tiles * d.num_kv_heads * splits;
        if (prefix_ctas < grid) {
            p.early_ctas = int32_t(grid - prefix_ctas);
            p.early_ns = kPrefixPassNs;
            p.early_ns_per_page = kPrefixPassNsPerPage;
            const int64_t unit_bytes = 2LL * kBlockSize * d.head_dim * 2 * p.HG;
            p.early_units_per_ms = int32_t(kDecodeCtaBytesPerMs / unit_bytes);
        }
        p.prefix_o = pp.prefix_o;
        p.prefix_ml = pp.prefix_ml;
        p.defer_dep = local ? 1 : 0;
        if (!local || num_tokens == 0) return dispatch_decode<false>(d.head_dim, G, p, grid, s, /*pdl=*/true);
        p.k_new = static_cast<const uint4*>(k_new);
        p.v_new = static_cast<const uint4*>(v_new);
        p.slot_mapping = slot_mapping;
        p.app_chunks = int64_t(num_tokens) * d.num_kv_heads * (d.head_dim / 8);
        p.app_tokens = num_tokens;
        p.app_local = 1;
        p.k_cache_w = static_cast<uint4*>(k_cache);
        p.v_cache_w = static_cast<uint4*>(v_cache);
        return dispatch_decode<false, true>(d.head_dim, G, p, grid, s, /*pdl=*/true);
    }
    if (num_tokens == 0) return dispatch_decode<false>(d.head_dim, G, p, grid, s);
    p.k_new = static_cast<const uint4*>(k_new);
    p.v_new = static_cast<const uint4*>(v_new);
    p.slot_mapping = slot_mapping;
    p.app_chunks = int64_t(num_tokens) * d.num_kv_heads * (d.head_dim / 8);
    p.app_tokens = num_tokens;
    p.app_local = num_tokens <= pa::kLocalMaxTokens;
    p.k_cache_w = static_cast<uint4*>(k_cache);
    p.v_cache_w = static_cast<uint4*>(v_cache);
    return dispatch_decode<false, true>(d.head_dim, G, p, grid, s);
}

pa_status pa_decode_static_ws(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                              const int32_t* context_lens, float scale, void* out, const pa_dims* dims,
                              void* stream) {
    if (!dims) return PA_ERR_NULL;
    if (!dims_ok(dims)) return PA_ERR_SHAPE;
    const int grid = sm_count();
    if (grid <= 0) return PA_ERR_CUDA;
    if (ws_layout(*dims, grid).total > size_t(PA_STATIC_SCRATCH_BYTES)) return PA_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    pa_status st = static_scratch_address(&scratch);
    if (st != PA_OK) return st;
    pa::DecodeParams p;
    st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, dims, grid, scratch,
                        PA_STATIC_SCRATCH_BYTES, p);
    if (st != PA_OK || dims->num_seqs == 0) return st;
    // the array keeps the last call's contents (another problem's partials may
    // sit where this one's counters go): the merge counters must start at zero
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const WsLayout w = ws_layout(*dims, grid);
    if (cudaMemsetAsync(p.counters, 0, size_t(dims->num_seqs) * dims->num_kv_heads * sizeof(int32_t), s) !=
            cudaSuccess ||
        cudaMemsetAsync(p.slot_sync, 0, w.grid_bar - w.slot_sync, s) != cudaSuccess)
        return PA_ERR_CUDA;
    return dispatch_decode<false>(dims->head_dim, dims->num_q_heads / dims->num_kv_heads, p, grid, s);
}

pa_status pa_cache_append_fp8(const void* k_new, const void* v_new, const int32_t* slot_mapping, int32_t num_tokens,
                              void* k_cache, void* v_cache, const float* k_scale, const float* v_scale,
                              const pa_dims* dims, void* stream) {
    if (!dims) return PA_ERR_NULL;
    const pa_dims& d = *dims;
    if (num_tokens < 0 || d.num_kv_heads <= 0 || d.head_dim <= 0 || d.block_size <= 0 || d.num_blocks < 0)
        return PA_ERR_SHAPE;
    if (d.block_size != kBlockSize || d.head_dim % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale) return PA_ERR_NULL;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(slot_mapping) || !aligned4(k_scale) || !aligned4(v_scale))
        return PA_ERR_ALIGN;
    pa::AppendFp8Params p;
    p.k_new = static_cast<const uint4*>(k_new);
    p.v_new = static_cast<const uint4*>(v_new);
    p.slot_mapping = slot_mapping;
    p.k_cache = static_cast<uint8_t*>(k_cache);
    p.v_cache = static_cast<uint8_t*>(v_cache);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.chunks_per_row = d.head_dim / 8;
    p.num_chunks = int64_t(num_tokens) * d.num_kv_heads * p.chunks_per_row;
    p.kv_heads = d.num_kv_heads;
    p.num_blocks = d.num_blocks;
    const int64_t blocks = (p.num_chunks + pa::kAppendThreads - 1) / pa::kAppendThreads;
    if (blocks > 0x7fffffff) return PA_ERR_SHAPE;
    pa::append_fp8_kernel<<<unsigned(blocks), pa::kAppendThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode_fp8(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                        const float* v_scale, const int32_t* block_tables, const int32_t* context_lens, float scale,
                        void* out, const pa_dims* dims, void* workspace, size_t workspace_bytes, void* stream) {
    pa::DecodeParams p;
    const int grid = sm_count();
    const pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, dims, grid,
                                        workspace, workspace_bytes, p, /*eb=*/1);
    if (st != PA_OK || dims->num_seqs == 0) return st;
    if (!k_scale || !v_scale) return PA_ERR_NULL;
    if (!aligned4(k_scale) || !aligned4(v_scale)) return PA_ERR_ALIGN;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    return dispatch_d_g<MathKind::kFp8, false, false>(dims->head_dim, dims->num_q_heads / dims->num_kv_heads, p,
                                                      grid, static_cast<cudaStream_t>(stream), false);
}

pa_status pa_append_decode_fp8(const void* k_new, const void* v_new, const int32_t* slot_mapping, int32_t num_tokens,
                               const void* q, void* k_cache, void* v_cache, const float* k_scale, const float* v_scale,
                               const int32_t* block_tables, const int32_t* context_lens, float scale, void* out,
                               const pa_dims* dims, void* workspace, size_t workspace_bytes, void* stream) {
    if (!dims) return PA_ERR_NULL;
    if (num_tokens < 0) return PA_ERR_SHAPE;
    pa::DecodeParams p;
    const int grid = sm_count();
    const pa_status st = prepare_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, dims, grid,
                                        workspace, workspace_bytes, p, /*eb=*/1);
    if (st != PA_OK) return st;
    if (!k_scale || !v_scale) return PA_ERR_NULL;
    if (!aligned4(k_scale) || !aligned4(v_scale)) return PA_ERR_ALIGN;
    if (num_tokens > 0) {
        if (!k_new || !v_new || !slot_mapping) return PA_ERR_NULL;
        if (!aligned16(k_new) || !aligned16(v_new) || !aligned4(slot_mapping)) return PA_ERR_ALIGN;
    }
    if (dims->num_seqs == 0)  // nothing to attend over: the append alone
        return pa_cache_append_fp8(k_new, v_new, slot_mapping, num_tokens, k_cache, v_cache, k_scale, v_scale, dims,
                                   stream);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.k_new = static_cast<const uint4*>(k_new);
    p.v_new = static_cast<const uint4*>(v_new);
    p.slot_mapping = slot_mapping;
    p.app_chunks = int64_t(num_tokens) * dims->num_kv_heads * (dims->head_dim / 8);
    p.app_tokens = num_tokens;
    p.app_local = num_tokens <= pa::kLocalMaxTokens;
    p.k_cache_w = static_cast<uint4*>(k_cache);
    p.v_cache_w = static_cast<uint4*>(v_cache);
    return dispatch_d_g<MathKind::kFp8, false, true>(dims->head_dim, dims->num_q_heads / dims->num_kv_heads, p, grid,
                                                     static_cast<cudaStream_t>(stream), false);
}

pa_status pa_prefill(const void* q, const int32_t* cu_q_lens, int32_t max_q_len, const void* k_cache,
                     const void* v_cache, const int32_t* block_tables, const int32_t* context_lens, float scale,
                     void* out, const pa_dims* dims, void* stream) {
    if (!dims) return PA_ERR_NULL;
    if (!dims_ok(dims) || max_q_len < 0) return PA_ERR_SHAPE;
    const pa_dims& d = *dims;
    const int G = d.num_q_heads / d.num_kv_heads;
    if (d.block_size != kBlockSize || !supported(d.head_dim, G, MathKind::kMma)) return PA_ERR_UNSUPPORTED;
    if (d.num_seqs == 0 || max_q_len == 0) return PA_OK;
    if (d.num_blocks == 0) return PA_ERR_SHAPE;
    if (!q || !cu_q_lens || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_NULL;
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned4(cu_q_lens) ||
        !aligned4(block_tables) || !aligned4(context_lens))
        return PA_ERR_ALIGN;
    const int64_t rows = int64_t(d.num_blocks) * d.num_kv_heads * d.block_size;
    if (rows >= (int64_t(1) << 31)) return PA_ERR_SHAPE;
    const int64_t tiles = (int64_t(max_q_len) * G + 16 * kPrefixNW - 1) / (16 * kPrefixNW);
    if (int64_t(d.num_seqs) * tiles > 0x7fffffffLL || d.num_kv_heads > 65535) return PA_ERR_SHAPE;
    pa::PrefillParams p;
    const int64_t cache_tiles = int64_t(d.num_blocks) * d.num_kv_heads;
    const bool sync_mma = prefill_use_mma_sync();
    const bool maps_ok =
        sync_mma ? make_cache_map(&p.tmap_k, k_cache, cache_tiles, d.head_dim, d.block_size, 1) &&
                       make_cache_map(&p.tmap_v, v_cache, cache_tiles, d.head_dim, d.block_size, 1)
                 : make_panel_map(&p.tmap_k, k_cache, cache_tiles, d.head_dim, d.block_size) &&
                       make_panel_map(&p.tmap_v, v_cache, cache_tiles, d.head_dim, d.block_size);
    if (!maps_ok) return PA_ERR_CUDA;
    p.q = static_cast<const uint8_t*>(q);
    p.cu_q_lens = cu_q_lens;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.B = d.num_seqs;
    p.Hq = d.num_q_heads;
    p.Hkv = d.num_kv_heads;
    p.NB = d.num_blocks;
    p.M = d.max_blocks_per_seq;
    p.tiles_per_seq = int32_t(tiles);
    p.qscale = scale * kLog2e;
    const dim3 grid(unsigned(d.num_seqs * tiles), unsigned(d.num_kv_heads));
    return sync_mma ? dispatch_prefill(d.head_dim, G, p, grid, static_cast<cudaStream_t>(stream))
                    : dispatch_prefill_tc(d.head_dim, G, p, grid, static_cast<cudaStream_t>(stream));
}

pa_status pa_test_wait_timeout(int64_t limit_ns, void* stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000LL) return PA_ERR_SHAPE;
    pa::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(limit_ns));
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_device_errors(int32_t* errors_out, int32_t clear) {
    if (!errors_out) return PA_ERR_NULL;
    if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, pa::g_device_errors, sizeof v) != cudaSuccess) return PA_ERR_CUDA;
    *errors_out = int32_t(v);
    if (clear) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(pa::g_device_errors, &zero, sizeof zero) != cudaSuccess) return PA_ERR_CUDA;
    }
    return PA_OK;
}

}  // extern "C"
