// videomla.cu -- the C ABI (include/videomla.h): argument validation, TMA
// tensor-map encoding, kernel-instance dispatch and launch.  This is the only
// translation unit of libvideomla.so; the kernels live in the included headers.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/videomla.h"
#include "attention.cuh"
#include "attention_pp.cuh"
#include "cache_write.cuh"
#include "dense_attention.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<int> g_tiling{VIDEOMLA_TILING_AUTO};

// ----------------------------------------------------------------------------
// driver entry point for cuTensorMapEncodeTiled (resolved through the runtime,
// so the library does not link libcuda directly)
// ----------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

CUtensorMapSwizzle swizzle_of(int bytes) {
    switch (bytes) {
        case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
        case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
        case 128: return CU_TENSOR_MAP_SWIZZLE_128B;
        default: return CU_TENSOR_MAP_SWIZZLE_NONE;
    }
}

// bf16 tensor map of rank ``rank``: dims/box innermost first, strides in bytes
// of dims 1..rank-1.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box, int swizzle_bytes,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) s[i] = strides[i];
    }
    return fn(m, dtype, rank, const_cast<void*>(base), d, s, bx, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(swizzle_bytes), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t n) { return (n + 255) / 256 * 256; }

// sm_100 check, cached per device.
int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return VIDEOMLA_ENODEVICE;
    static std::atomic<int> ok_mask[64];
    if (dev >= 0 && dev < 64 && ok_mask[dev].load() == 1) return VIDEOMLA_OK;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return VIDEOMLA_ENODEVICE;
    if (major != 10) return VIDEOMLA_ENODEVICE;
    if (dev >= 0 && dev < 64) ok_mask[dev].store(1);
    return VIDEOMLA_OK;
}

template <class K>
int launch_status(K kernel, int smem) {
    (void)kernel;
    (void)smem;
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? VIDEOMLA_OK : VIDEOMLA_ECUDA;
}

// Launch with programmatic stream serialisation: the kernel may start while the
// previous kernel of the stream drains, and it calls griddep_wait before it
// touches anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_programmatic(void (*kern)(KArgs...), dim3 grid, int threads, int smem, cudaStream_t st,
                                Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

bool basic_dims_ok(const videomla_dims* d) {
    if (!d) return false;
    if (d->d_model <= 0 || d->n_heads <= 0 || d->d_c <= 0 || d->d_rope <= 0 || d->d_nope <= 0 || d->d_v <= 0)
        return false;
    if (d->grid_h <= 0 || d->grid_w <= 0) return false;
    if (d->d_rope % 2) return false;
    if (d->pairs_t < 0 || d->pairs_h < 0 || d->pairs_w < 0) return false;
    if (2 * (d->pairs_t + d->pairs_h + d->pairs_w) != d->d_rope) return false;
    if (!(d->rope_base > 1.0f) || !(d->rms_eps >= 0.0f)) return false;
    if ((long long)d->grid_h * d->grid_w > (1 << 24)) return false;
    return true;
}

// ----------------------------------------------------------------------------
// cache_write
// ----------------------------------------------------------------------------
// SM count of the current device (148 on B200).
int sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms <= 0)
        return 148;
    return sms;
}

// K split of the cache write: CTAs per cluster (1-4) dividing the K chunks.
// Clusters are placed inside one GPC, so the number that fit at once
// (cudaOccupancyMaxActiveClusters) decides the waves; pick the split with the
// least work per SM = waves * chunks / ksplit (cached per device and shape).
template <class K>
int pick_ksplit(K kern, int threads, int smem, int chunks, int clusters, int max_split) {
    int dev = 0;
    cudaGetDevice(&dev);
    static std::mutex mu;
    static int cache[64][5] = {};  // max active clusters per (device, ksplit)
    int best = 1;
    long long best_cost = -1;
    for (int k = max_split; k >= 1; --k) {
        if (chunks % k != 0) continue;
        int active = 0;
        {
            std::lock_guard<std::mutex> lock(mu);
            if (dev >= 0 && dev < 64 && cache[dev][k] > 0) active = cache[dev][k];
        }
        if (active == 0) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(clusters, k, 1);
            cfg.blockDim = dim3(threads);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 1;
            attr[0].val.clusterDim.y = k;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess || active <= 0) {
                cudaGetLastError();
                continue;
            }
            std::lock_guard<std::mutex> lock(mu);
            if (dev >= 0 && dev < 64) cache[dev][k] = active;
        }
        const long long waves = (clusters + active - 1) / active;
        const long long cost = waves * (chunks / k) + 2 * k;  // + a small cost per extra cluster member
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = k;
        }
    }
    return best;
}

template <int DC, int DR>
int run_cache_write_cluster(const videomla_dims* d, const void* x, int B, int n_tok, const void* W_dkv, const void* W_kr,
                    const float* gamma, void* cache, int slots, int first_slot, unsigned flags, cudaStream_t st) {
    using C = vmla::ClusterWriteCfg<DC, DR>;
    const int T_f = d->grid_h * d->grid_w;
    CUtensorMap tx, tw, tr;
    {
        const uint64_t dims[3] = {uint64_t(d->d_model), uint64_t(n_tok), uint64_t(B)};
        const uint64_t str[2] = {uint64_t(d->d_model) * 2, uint64_t(n_tok) * d->d_model * 2};
        const uint32_t box[3] = {64, 128, 1};
        if (!make_map(&tx, x, 3, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    {
        const uint64_t dims[2] = {uint64_t(d->d_model), uint64_t(DC)};
        const uint64_t str[1] = {uint64_t(d->d_model) * 2};
        const uint32_t box[2] = {64, uint32_t(C::WBOX)};
        if (!make_map(&tw, W_dkv, 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    {
        const uint64_t dims[2] = {uint64_t(d->d_model), uint64_t(DR)};
        const uint64_t str[1] = {uint64_t(d->d_model) * 2};
        const uint32_t box[2] = {64, uint32_t(DR)};
        if (!make_map(&tr, W_kr, 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    auto kern = vmla::cache_write_cluster_kernel<DC, DR>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return VIDEOMLA_ECUDA;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess)
        return VIDEOMLA_ECUDA;
    const int tiles = (n_tok + C::BM - 1) / C::BM;
    const int ksplit = pick_ksplit(kern, C::THREADS, C::SMEM, d->d_model / C::BKK, tiles * B, C::KS_MAX);
    vmla::CacheWriteParams p;
    std::memset(&p, 0, sizeof(p));
    p.n_tok = n_tok;
    p.d_model = d->d_model;
    p.ksplit = ksplit;
    p.T_f = T_f;
    p.slots = slots;
    p.first_slot = first_slot;
    p.normalize = (flags & VIDEOMLA_CACHE_RAW_LATENT) ? 0 : 1;
    p.eps = d->rms_eps;
    p.gamma = gamma;
    p.cache = static_cast<__nv_bfloat16*>(cache);
    p.timeout_ns = g_timeout_ns.load();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles, ksplit, B);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = ksplit;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tx, tw, tr, p) != cudaSuccess) return VIDEOMLA_ECUDA;
    return launch_status(kern, C::SMEM);
}

// Many tiles: the persistent stream kernel, one CTA per SM walking the tiles.
template <int DC, int DR>
int run_cache_write_stream(const videomla_dims* d, const void* x, int B, int n_tok, const void* W_dkv,
                           const void* W_kr, const float* gamma, void* cache, int slots, int first_slot,
                           unsigned flags, cudaStream_t st) {
    using C = vmla::StreamWriteCfg<DC, DR>;
    const int T_f = d->grid_h * d->grid_w;
    CUtensorMap tx, tw, tr;
    {
        const uint64_t dims[3] = {uint64_t(d->d_model), uint64_t(n_tok), uint64_t(B)};
        const uint64_t str[2] = {uint64_t(d->d_model) * 2, uint64_t(n_tok) * d->d_model * 2};
        const uint32_t box[3] = {64, 128, 1};
        if (!make_map(&tx, x, 3, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    {
        const uint64_t dims[2] = {uint64_t(d->d_model), uint64_t(DC)};
        const uint64_t str[1] = {uint64_t(d->d_model) * 2};
        const uint32_t box[2] = {64, uint32_t(C::WBOX)};
        if (!make_map(&tw, W_dkv, 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    {
        const uint64_t dims[2] = {uint64_t(d->d_model), uint64_t(DR)};
        const uint64_t str[1] = {uint64_t(d->d_model) * 2};
        const uint32_t box[2] = {64, uint32_t(DR)};
        if (!make_map(&tr, W_kr, 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    auto kern = vmla::cache_write_stream_kernel<DC, DR>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return VIDEOMLA_ECUDA;
    vmla::CacheWriteParams p;
    std::memset(&p, 0, sizeof(p));
    p.n_tok = n_tok;
    p.d_model = d->d_model;
    p.tiles = (n_tok + C::BM - 1) / C::BM;
    p.units = p.tiles * B;
    p.k_chunks = d->d_model / C::BKK;
    p.T_f = T_f;
    p.slots = slots;
    p.first_slot = first_slot;
    p.normalize = (flags & VIDEOMLA_CACHE_RAW_LATENT) ? 0 : 1;
    p.eps = d->rms_eps;
    p.gamma = gamma;
    p.cache = static_cast<__nv_bfloat16*>(cache);
    p.timeout_ns = g_timeout_ns.load();
    const int sms = sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.units < sms ? p.units : sms, 1, 1);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the previous kernel
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tx, tw, tr, p) != cudaSuccess) {
        cudaGetLastError();
        return VIDEOMLA_ECUDA;
    }
    return launch_status(kern, 0);
}

// A chunk of few tiles (fewer than half the SMs) spreads each tile's K range over
// a cluster; more tiles stream through the persistent kernel, one tile per SM
// at a time.
template <int DC, int DR>
int run_cache_write(const videomla_dims* d, const void* x, int B, int n_tok, const void* W_dkv, const void* W_kr,
                    const float* gamma, void* cache, int slots, int first_slot, unsigned flags, cudaStream_t st) {
    const long long units = (long long)B * ((n_tok + 127) / 128);
    if (2 * units <= sm_count())
        return run_cache_write_cluster<DC, DR>(d, x, B, n_tok, W_dkv, W_kr, gamma, cache, slots, first_slot, flags, st);
    return run_cache_write_stream<DC, DR>(d, x, B, n_tok, W_dkv, W_kr, gamma, cache, slots, first_slot, flags, st);
}

// ----------------------------------------------------------------------------
// attention
// ----------------------------------------------------------------------------
// Valid physical rows of the window: one run, or two when the ring wraps.
void window_runs(const videomla_window* win, int T_f, int seg_start[3], int seg_len[3]) {
    seg_start[1] = seg_len[1] = 0;
    if (win->n_valid == win->slots) {
        seg_start[0] = 0;
        seg_len[0] = win->slots * T_f;
        return;
    }
    const int last = win->oldest_slot + win->n_valid;
    seg_start[0] = win->oldest_slot * T_f;
    seg_len[0] = (last <= win->slots ? win->n_valid : win->slots - win->oldest_slot) * T_f;
    if (last > win->slots) {
        seg_start[1] = 0;
        seg_len[1] = (last - win->slots) * T_f;
    }
}

// Split-KV of the attention: how many CTAs share the key tiles of one (query
// tile, head, batch) unit.  One CTA per SM; cost in key-tile times: the waves
// times the tiles per CTA (+2 for writing a partial), plus the merge of the
// other partials by the last CTA (1.5 per split).  At most 4 splits.
int attention_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

double split_cost(int units, int n_kt, int s, int sms) {
    const int tps = (n_kt + s - 1) / s;
    const long long waves = ((long long)units * s + sms - 1) / sms;
    return double(waves) * (tps + (s > 1 ? 2 : 0)) + 1.5 * (s - 1);
}

int preferred_split(int units, int n_kt, int batch) {
    const int sms = attention_sms();
    int best = 1;
    double best_cost = 0;
    for (int s = 1; s <= 4 && s <= n_kt && (long long)batch * s <= 65535; ++s) {
        const int tps = (n_kt + s - 1) / s;
        const int se = (n_kt + tps - 1) / tps;
        if (se != s) continue;
        const double cost = split_cost(units, n_kt, s, sms);
        if (s == 1 || cost < best_cost) {
            best = s;
            best_cost = cost;
        }
    }
    return best;
}

// Head-packed query tiles (one CTA per 128 consecutive rows of the head-major
// (head, query) order, no split-KV) against per-head tiles with their best
// split: the same wave-count cost, plus ~3 key-tile times for the second
// head's prologue and epilogue in a tile that holds two heads.  Only for the
// instances with Q in tensor memory and at least 128 queries (a tile then
// spans at most two heads).
bool use_packed_tiles(bool q_in_smem, int Nq, int H, int B, int n_kt, int units, int split) {
    const int mode = g_tiling.load();
    if (q_in_smem || Nq < 128 || mode == VIDEOMLA_TILING_PER_HEAD) return false;
    if (mode == VIDEOMLA_TILING_HEAD_PACKED) return true;
    const int sms = attention_sms();
    const long long packed_units = ((long long)H * Nq + 127) / 128 * B;
    const double packed = double((packed_units + sms - 1) / sms) * n_kt + (Nq % 128 != 0 ? 3.0 : 0.0);
    return packed < split_cost(units, n_kt, split, sms);
}

size_t split_part_bytes(int units, int split, int d_c) {  // partial O + (max, sum) per row + counters
    if (split <= 1) return 0;
    return size_t(units) * split * (128 * size_t(d_c) * 4 + 128 * 2 * 4) + align256(size_t(units) * 4);
}

template <int DC, int DR, int DN, int DV>
int run_attention(const videomla_dims* d, const void* q_nope, const void* q_rope, const void* W_uk, const void* W_uv,
                  const void* cache, const videomla_window* win, const void* sink, int n_sink, int B, int Nq,
                  void* out, float* lse, void* workspace, size_t workspace_bytes, cudaStream_t st) {
    using C = vmla::AttnCfg<DC, DR, DN, DV>;
    const int T_f = d->grid_h * d->grid_w;
    const int H = d->n_heads;
    const int rows = win->slots * T_f;
    vmla::AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.Nq = Nq;
    p.H = H;
    p.T_f = T_f;
    p.grid_w = d->grid_w;
    p.slots = win->slots;
    p.oldest = win->oldest_slot;
    window_runs(win, T_f, p.seg_start, p.seg_len);
    p.seg_start[2] = 0;
    p.seg_len[2] = n_sink * T_f;
    p.n_sink = n_sink;
    p.ws_rows = (win->slots + n_sink) * T_f;
    p.n_kt = 0;
    for (int r = 0; r < 3; ++r) p.n_kt += (p.seg_len[r] + C::BK - 1) / C::BK;
    {
        // split-KV, as far as the workspace holds the partials
        const int units = (Nq + C::BM - 1) / C::BM * H * B;
        const size_t rope_bytes = align256(size_t(B) * p.ws_rows * DR * 2);
        int sp = preferred_split(units, p.n_kt, B);
        while (sp > 1 && rope_bytes + split_part_bytes(units, sp, DC) > workspace_bytes) --sp;
        p.packed = use_packed_tiles(C::QS, Nq, H, B, p.n_kt, units, sp) ? 1 : 0;
        if (p.packed) sp = 1;
        p.tiles_per_split = (p.n_kt + sp - 1) / sp;
        p.n_split = (p.n_kt + p.tiles_per_split - 1) / p.tiles_per_split;
        p.n_units = units;
        uint8_t* wsb = static_cast<uint8_t*>(workspace);
        p.part_o = reinterpret_cast<float*>(wsb + rope_bytes);
        p.part_ml = p.part_o + size_t(units) * p.n_split * 128 * DC;
        p.counters = reinterpret_cast<int*>(p.part_ml + size_t(units) * p.n_split * 128 * 2);
    }
    // Narrow latents without split-KV or head-packed tiles run the two-group kernel,
    // whose key tiles are shorter: recount them and size the key maps' boxes for it.
    bool two_group = false;
    int bk = C::BK;
    if constexpr (vmla::pingpong_fits(DC)) {
        two_group = p.n_split == 1 && !p.packed;
        if (two_group) {
            bk = vmla::AttnPPCfg<DC, DR, DN, DV>::BK;
            p.n_kt = 0;
            for (int r = 0; r < 3; ++r) p.n_kt += (p.seg_len[r] + bk - 1) / bk;
            p.tiles_per_split = p.n_kt;
        }
    }
    p.q_first = (n_sink + win->n_valid) * T_f - Nq;
    p.n_t = d->pairs_t;
    p.n_h = d->pairs_h;
    // rope frequencies: an axis owning D_a dims of a full (d_nope + d_rope)-dim
    // head (h, w: floor(n/3) pairs each, t: the rest) uses base^(-2k / D_a)
    {
        const int n_full = (d->d_nope + d->d_rope) / 2;
        const int full_hw = n_full / 3;
        const int full_t = n_full - 2 * full_hw;
        const int cnt[3] = {d->pairs_t, d->pairs_h, d->pairs_w};
        const int D[3] = {2 * full_t, 2 * full_hw, 2 * full_hw};
        int pr = 0;
        for (int a = 0; a < 3; ++a)
            for (int k = 0; k < cnt[a]; ++k)
                p.omega[pr++] = float(std::pow(double(d->rope_base), -2.0 * k / double(D[a])));
    }
    p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(d->d_nope + d->d_rope)));
    p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.timeout_ns = g_timeout_ns.load();

    vmla::AttnMaps maps;
    const auto* cache_b = static_cast<const __nv_bfloat16*>(cache);
    const auto* krot = static_cast<const __half*>(workspace);
    const auto* sink_b = static_cast<const __nv_bfloat16*>(sink);
    for (int r = 0; r < 3; ++r) {
        const int run = p.seg_len[r] > 0 ? r : 0;  // an empty run reuses the first (never read)
        const bool is_sink = run == 2;
        const __nv_bfloat16* base = is_sink ? sink_b : cache_b + size_t(p.seg_start[run]) * C::W;
        const uint64_t batch_rows = is_sink ? uint64_t(n_sink) * T_f : uint64_t(rows);
        const uint64_t dc[3] = {uint64_t(C::W), uint64_t(p.seg_len[run]), uint64_t(B)};
        const uint64_t sc[2] = {uint64_t(C::W) * 2, batch_rows * C::W * 2};
        const uint32_t bc[3] = {64, uint32_t(bk), 1};
        if (!make_map(&maps.cc[r], base, 3, dc, sc, bc, 128)) return VIDEOMLA_ECUDA;
        const size_t ws_row0 = is_sink ? size_t(rows) : size_t(p.seg_start[run]);
        const uint64_t dr[3] = {uint64_t(DR), uint64_t(p.seg_len[run]), uint64_t(B)};
        const uint64_t sr[2] = {uint64_t(DR) * 2, uint64_t(p.ws_rows) * DR * 2};
        const uint32_t br[3] = {uint32_t(DR), uint32_t(bk), 1};
        if (!make_map(&maps.kr[r], krot + ws_row0 * DR, 3, dr, sr, br, DR * 2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
            return VIDEOMLA_ECUDA;
    }
    {
        const uint64_t dims[4] = {uint64_t(DN), uint64_t(H), uint64_t(Nq), uint64_t(B)};
        const uint64_t str[3] = {uint64_t(DN) * 2, uint64_t(H) * DN * 2, uint64_t(Nq) * H * DN * 2};
        const uint32_t box[4] = {16, 1, uint32_t(C::BM), 1};
        if (!make_map(&maps.qn, q_nope, 4, dims, str, box, 32)) return VIDEOMLA_ECUDA;
    }
    {
        const uint64_t dims[2] = {uint64_t(DC), uint64_t(H) * DN};
        const uint64_t str[1] = {uint64_t(DC) * 2};
        const uint32_t box[2] = {64, uint32_t(DN)};
        if (!make_map(&maps.wuk, W_uk, 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    {
        const uint64_t dims[2] = {uint64_t(DC), uint64_t(H) * DV};
        const uint64_t str[1] = {uint64_t(DC) * 2};
        const uint32_t box[2] = {64, uint32_t(DV)};
        if (!make_map(&maps.wuv, W_uv, 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    // 1) form the window: rotated rope keys into the workspace
    {
        const long long work = (long long)B * (p.seg_len[0] + p.seg_len[1] + p.seg_len[2]) * (DR / 8);
        const int blocks = int((work + 255) / 256);
        if (launch_programmatic(vmla::rope_window_kernel<DC, DR>, dim3(blocks), 256, 0, st, cache_b, sink_b,
                                static_cast<__half*>(workspace), p, B) != cudaSuccess) {
            cudaGetLastError();
            return VIDEOMLA_ECUDA;
        }
    }
    // 2) latent attention
    if constexpr (vmla::pingpong_fits(DC)) {
        if (two_group) {
            using PC = vmla::AttnPPCfg<DC, DR, DN, DV>;
            auto kern = vmla::attention_pp_kernel<PC>;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PC::SMEM) != cudaSuccess)
                return VIDEOMLA_ECUDA;
            // launched right behind the pre-pass, which lets it start only once all
            // kernels before the pass have finished
            if (launch_programmatic(kern, dim3((Nq + PC::BM - 1) / PC::BM, H, B), PC::THREADS, PC::SMEM, st, maps,
                                    p) != cudaSuccess) {
                cudaGetLastError();
                return VIDEOMLA_ECUDA;
            }
            return launch_status(kern, PC::SMEM);
        }
    }
    auto kern = p.n_split > 1 ? vmla::attention_kernel<C, true> : vmla::attention_kernel<C, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return VIDEOMLA_ECUDA;
    const dim3 grid = p.packed ? dim3(unsigned(((long long)H * Nq + C::BM - 1) / C::BM), 1, B)
                               : dim3((Nq + C::BM - 1) / C::BM, H, B * p.n_split);
    if (launch_programmatic(kern, grid, C::THREADS, C::SMEM, st, maps, p) != cudaSuccess) {
        cudaGetLastError();
        return VIDEOMLA_ECUDA;
    }
    return launch_status(kern, C::SMEM);
}


// ----------------------------------------------------------------------------
// dense multi-head attention baseline
// ----------------------------------------------------------------------------
template <int DN, int DR>
int run_dense_attention(const videomla_dims* d, const void* q_nope, const void* q_rope, const void* K, const void* V,
                        int B, int Nq, int Nk, void* out, cudaStream_t st) {
    using C = vmla::DenseCfg<DN, DR>;
    const int H = d->n_heads;
    vmla::DenseMaps maps;
    {
        const uint64_t dims[4] = {uint64_t(C::DH), uint64_t(H), uint64_t(Nk), uint64_t(B)};
        const uint64_t str[3] = {uint64_t(C::DH) * 2, uint64_t(H) * C::DH * 2, uint64_t(Nk) * H * C::DH * 2};
        const uint32_t box[4] = {64, 1, uint32_t(C::BK), 1};
        if (!make_map(&maps.k, K, 4, dims, str, box, 128)) return VIDEOMLA_ECUDA;
        if (!make_map(&maps.v, V, 4, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    vmla::DenseParams p;
    std::memset(&p, 0, sizeof(p));
    p.Nq = Nq;
    p.Nk = Nk;
    p.H = H;
    p.T_f = d->grid_h * d->grid_w;
    p.grid_w = d->grid_w;
    p.q_first = Nk - Nq;
    p.n_t = d->pairs_t;
    p.n_h = d->pairs_h;
    {
        // the latent kernel's rope frequencies (an axis owning D_a dims of the head
        // uses base^(-2k / D_a))
        const int n_full = (d->d_nope + d->d_rope) / 2;
        const int full_hw = n_full / 3;
        const int full_t = n_full - 2 * full_hw;
        const int cnt[3] = {d->pairs_t, d->pairs_h, d->pairs_w};
        const int D[3] = {2 * full_t, 2 * full_hw, 2 * full_hw};
        int pr = 0;
        for (int a = 0; a < 3; ++a)
            for (int k = 0; k < cnt[a]; ++k)
                p.omega[pr++] = float(std::pow(double(d->rope_base), -2.0 * k / double(D[a])));
    }
    p.scale_log2 = float(1.4426950408889634 / std::sqrt(double(C::DH)));
    p.q_nope = static_cast<const __nv_bfloat16*>(q_nope);
    p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.timeout_ns = g_timeout_ns.load();
    auto kern = vmla::dense_attention_kernel<C>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return VIDEOMLA_ECUDA;
    dim3 grid((Nq + C::BM - 1) / C::BM, H, B);
    kern<<<grid, C::THREADS, C::SMEM, st>>>(maps, p);
    return launch_status(kern, C::SMEM);
}

// ----------------------------------------------------------------------------
// projections: C_g [M, N_g] = A [M, K] . B_g [N_g, K]^T, one or two column groups
// ----------------------------------------------------------------------------
// Largest number of 2-CTA clusters of a kernel that can be resident at once (cached per device).
int max_pair_clusters(const void* kern, int threads, int smem) {
    int dev = 0;
    cudaGetDevice(&dev);
    static std::mutex mu;
    static int cache[64][2] = {};
    const int slot = smem > 140000 ? 1 : 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 0 && dev < 64 && cache[dev][slot] > 0) return cache[dev][slot];
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = sm_count() / 2;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64) cache[dev][slot] = n;
    return n;
}

// Optional epilogue work of a GEMM launch (see GemmParams).
struct GemmEpilogue {
    float* row_ss = nullptr;
    const float* col_scale = nullptr;
    const float* row_ss_in = nullptr;
    int ss_parts = 0;  // partial sums per row in row_ss_in
    int rms_dim = 1;
    float rms_eps = 0.f;
};

template <int BN, bool F32OUT>
int run_gemm_pair(const void* A, int M, int K, int groups, const void* B0, int N0, void* C0, int ldc0, const void* B1,
                  int N1, void* C1, int ldc1, cudaStream_t st, const GemmEpilogue& epi) {
    using C = vmla::GemmPairCfg<BN, F32OUT>;
    CUtensorMap ta, tb[2];
    {
        const uint64_t dims[2] = {uint64_t(K), uint64_t(M)};
        const uint64_t str[1] = {uint64_t(K) * 2};
        const uint32_t box[2] = {64, uint32_t(C::BM)};
        if (!make_map(&ta, A, 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    const void* Bs[2] = {B0, groups > 1 ? B1 : B0};
    const int Ns[2] = {N0, groups > 1 ? N1 : N0};
    for (int g = 0; g < 2; ++g) {
        const uint64_t dims[2] = {uint64_t(K), uint64_t(Ns[g])};
        const uint64_t str[1] = {uint64_t(K) * 2};
        const uint32_t box[2] = {64, uint32_t(C::BNH)};
        if (!make_map(&tb[g], Bs[g], 2, dims, str, box, 128)) return VIDEOMLA_ECUDA;
    }
    auto kern = vmla::gemm_pair_kernel<C>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return VIDEOMLA_ECUDA;
    vmla::GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.K = K;
    p.n_groups = groups;
    p.N[0] = N0;
    p.N[1] = groups > 1 ? N1 : 0;
    p.n_tiles[0] = (N0 + BN - 1) / BN;
    p.n_tiles[1] = groups > 1 ? (N1 + BN - 1) / BN : 0;
    p.m_tiles = (M + 255) / 256;
    p.tiles = p.m_tiles * (p.n_tiles[0] + p.n_tiles[1]);
    p.C[0] = C0;
    p.C[1] = C1;
    p.ldc[0] = ldc0;
    p.ldc[1] = ldc1;
    p.timeout_ns = g_timeout_ns.load();
    p.row_ss = epi.row_ss;
    p.col_scale = epi.col_scale;
    p.row_ss_in = epi.row_ss_in;
    p.ss_parts = epi.ss_parts;
    p.rms_dim = epi.rms_dim;
    p.rms_eps = epi.rms_eps;
    const int pairs_max = max_pair_clusters(reinterpret_cast<const void*>(kern), C::THREADS, C::SMEM);
    const int pairs = p.tiles < pairs_max ? p.tiles : pairs_max;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // set-up overlaps the previous kernel
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb[0], tb[1], p) != cudaSuccess) {
        cudaGetLastError();
        return VIDEOMLA_ECUDA;
    }
    return launch_status(kern, C::SMEM);
}

// Column tile width of the pair tiles: the one that puts the fewest columns on
// the busiest pair of the persistent grid (ties go to 256, fewer tiles).  The
// query path counts its per-tile row sums of squares with this same choice.
int gemm_pair_bn(int M, int N0, int N1, int groups) {
    const long long m_tiles = (M + 255) / 256;
    const int pairs = sm_count() / 2;
    long long cost[2];
    const int bns[2] = {256, 128};
    for (int i = 0; i < 2; ++i) {
        const int bn = bns[i];
        const long long t = m_tiles * ((N0 + bn - 1) / bn + (groups > 1 ? (N1 + bn - 1) / bn : 0));
        cost[i] = (t + pairs - 1) / pairs * bn;
    }
    return cost[1] < cost[0] ? 128 : 256;
}

// bf16 or fp32 C; one or two column groups sharing A; CTA-pair kernel.
int gemm2(const void* A, int M, int K, int groups, const void* B0, int N0, void* C0, int ldc0, const void* B1, int N1,
          void* C1, int ldc1, bool f32out, cudaStream_t st, const GemmEpilogue& epi = GemmEpilogue()) {
    if (gemm_pair_bn(M, N0, N1, groups) == 256)
        return f32out ? run_gemm_pair<256, true>(A, M, K, groups, B0, N0, C0, ldc0, B1, N1, C1, ldc1, st, epi)
                      : run_gemm_pair<256, false>(A, M, K, groups, B0, N0, C0, ldc0, B1, N1, C1, ldc1, st, epi);
    return f32out ? run_gemm_pair<128, true>(A, M, K, groups, B0, N0, C0, ldc0, B1, N1, C1, ldc1, st, epi)
                  : run_gemm_pair<128, false>(A, M, K, groups, B0, N0, C0, ldc0, B1, N1, C1, ldc1, st, epi);
}

int gemm(const void* A, const void* B, int M, int N, int K, void* Cmat, int ldc, bool f32out, cudaStream_t st,
         const GemmEpilogue& epi = GemmEpilogue()) {
    return gemm2(A, M, K, 1, B, N, Cmat, ldc, nullptr, 0, nullptr, 0, f32out, st, epi);
}

}  // namespace

extern "C" {

int videomla_cache_write(const videomla_dims* dims, const void* x, int batch, int n_tok, const void* W_dkv,
                         const void* W_kr, const float* gamma, void* cache, int slots, int first_slot, unsigned flags,
                         void* stream) {
    if (!basic_dims_ok(dims) || !x || !W_dkv || !W_kr || !cache) return VIDEOMLA_EINVAL;
    if (batch <= 0 || batch > 65535 || n_tok <= 0 || slots <= 0 || first_slot < 0 || first_slot >= slots)
        return VIDEOMLA_EINVAL;
    if (flags & ~VIDEOMLA_CACHE_RAW_LATENT) return VIDEOMLA_EINVAL;
    const long long T_f = (long long)dims->grid_h * dims->grid_w;
    if (n_tok % T_f != 0 || n_tok / T_f > slots) return VIDEOMLA_EINVAL;
    if ((long long)slots * T_f > (1ll << 30)) return VIDEOMLA_EINVAL;
    if (!aligned16(x) || !aligned16(W_dkv) || !aligned16(W_kr) || !aligned16(cache) ||
        (reinterpret_cast<uintptr_t>(gamma) & 7u))
        return VIDEOMLA_EINVAL;
    if (dims->d_model % 64 != 0) return VIDEOMLA_EUNSUPPORTED;
    if (int rc = check_device()) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int dc = dims->d_c, dr = dims->d_rope;
#define VMLA_CW(DC_, DR_) \
    if (dc == DC_ && dr == DR_) return run_cache_write<DC_, DR_>(dims, x, batch, n_tok, W_dkv, W_kr, gamma, cache, slots, first_slot, flags, st);
    VMLA_CW(192, 32)
    VMLA_CW(192, 16)
    VMLA_CW(192, 64)
    VMLA_CW(96, 32)
    VMLA_CW(384, 32)
#undef VMLA_CW
    return VIDEOMLA_EUNSUPPORTED;
}

size_t videomla_attention_sink_workspace_size(const videomla_dims* dims, const videomla_window* window, int n_sink,
                                              int batch) {
    if (!dims || !window || batch <= 0 || window->slots <= 0 || n_sink < 0 || dims->grid_h <= 0 ||
        dims->grid_w <= 0 || dims->d_rope <= 0)
        return 0;
    return size_t(batch) * (window->slots + n_sink) * size_t(dims->grid_h) * dims->grid_w * dims->d_rope * 2;
}

size_t videomla_attention_workspace_size(const videomla_dims* dims, const videomla_window* window, int batch) {
    return videomla_attention_sink_workspace_size(dims, window, 0, batch);
}

size_t videomla_attention_workspace_size_split(const videomla_dims* dims, const videomla_window* window, int n_sink,
                                               int batch, int n_query) {
    const size_t rope = videomla_attention_sink_workspace_size(dims, window, n_sink, batch);
    if (rope == 0 || n_query <= 0 || dims->n_heads <= 0) return 0;
    const int T_f = dims->grid_h * dims->grid_w;
    const int bk = (dims->d_c + 128 + 64 + (dims->d_c + dims->d_rope) / 2 > 512) ? 64 : 128;  // key tile
    // key tiles per run, as run_attention counts them
    videomla_window w = *window;
    if (w.slots <= 0 || w.n_valid < 1 || w.n_valid > w.slots || w.oldest_slot < 0 || w.oldest_slot >= w.slots)
        return 0;
    int seg_start[3], seg_len[3];
    window_runs(&w, T_f, seg_start, seg_len);
    seg_len[2] = n_sink * T_f;
    int n_kt = 0;
    for (int r = 0; r < 3; ++r) n_kt += (seg_len[r] + bk - 1) / bk;
    const int units = (n_query + 127) / 128 * dims->n_heads * batch;
    return align256(rope) + split_part_bytes(units, preferred_split(units, n_kt, batch), dims->d_c);
}

int videomla_attention_sink(const videomla_dims* dims, const void* q_nope, const void* q_rope, const void* W_uk,
                            const void* W_uv, const void* cache, const videomla_window* window, const void* sink_cache,
                            int n_sink, int batch, int n_query, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
    if (!basic_dims_ok(dims) || !q_nope || !q_rope || !W_uk || !W_uv || !cache || !window || !out || !workspace)
        return VIDEOMLA_EINVAL;
    const videomla_window w = *window;
    if (w.slots <= 0 || w.oldest_slot < 0 || w.oldest_slot >= w.slots || w.n_valid < 1 || w.n_valid > w.slots)
        return VIDEOMLA_EINVAL;
    if (n_sink < 0 || n_sink > VIDEOMLA_MAX_SINK_FRAMES || (n_sink > 0 && (!sink_cache || !aligned16(sink_cache))))
        return VIDEOMLA_EINVAL;
    const long long T_f = (long long)dims->grid_h * dims->grid_w;
    if (batch <= 0 || batch > 65535 || n_query <= 0 || n_query > (n_sink + w.n_valid) * T_f) return VIDEOMLA_EINVAL;
    if ((long long)(w.slots + n_sink) * T_f > (1ll << 30) || dims->n_heads > 65535) return VIDEOMLA_EINVAL;
    if (workspace_bytes < videomla_attention_sink_workspace_size(dims, window, n_sink, batch)) return VIDEOMLA_EINVAL;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(cache) ||
        !aligned16(out) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return VIDEOMLA_EINVAL;
    if (int rc = check_device()) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int dc = dims->d_c, dr = dims->d_rope, dn = dims->d_nope, dv = dims->d_v;
#define VMLA_AT(DC_, DR_, DN_, DV_)                        \
    if (dc == DC_ && dr == DR_ && dn == DN_ && dv == DV_) \
        return run_attention<DC_, DR_, DN_, DV_>(dims, q_nope, q_rope, W_uk, W_uv, cache, &w, sink_cache, n_sink, \
                                                 batch, n_query, out, lse, workspace, workspace_bytes, st);
    VMLA_AT(192, 32, 96, 128)
    VMLA_AT(192, 16, 112, 128)
    VMLA_AT(192, 64, 64, 128)
    VMLA_AT(96, 32, 96, 128)
    VMLA_AT(384, 32, 96, 128)
#undef VMLA_AT
    return VIDEOMLA_EUNSUPPORTED;
}

int videomla_attention(const videomla_dims* dims, const void* q_nope, const void* q_rope, const void* W_uk,
                       const void* W_uv, const void* cache, const videomla_window* window, int batch, int n_query,
                       void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    return videomla_attention_sink(dims, q_nope, q_rope, W_uk, W_uv, cache, window, nullptr, 0, batch, n_query, out,
                                   lse, workspace, workspace_bytes, stream);
}

int videomla_dense_attention(const videomla_dims* dims, const void* q_nope, const void* q_rope, const void* k,
                             const void* v, int batch, int n_query, int n_keys, void* out, void* stream) {
    if (!basic_dims_ok(dims) || !q_nope || !q_rope || !k || !v || !out) return VIDEOMLA_EINVAL;
    if (dims->d_nope + dims->d_rope != 128 || dims->d_v != 128) return VIDEOMLA_EUNSUPPORTED;
    const long long T_f = (long long)dims->grid_h * dims->grid_w;
    if (batch <= 0 || batch > 65535 || dims->n_heads > 65535 || n_keys <= 0 || n_keys % T_f != 0 || n_query <= 0 ||
        n_query > n_keys || (long long)n_keys * dims->n_heads > (1ll << 30))
        return VIDEOMLA_EINVAL;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return VIDEOMLA_EINVAL;
    if (int rc = check_device()) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int dn = dims->d_nope, dr = dims->d_rope;
#define VMLA_DA(DN_, DR_) \
    if (dn == DN_ && dr == DR_) return run_dense_attention<DN_, DR_>(dims, q_nope, q_rope, k, v, batch, n_query, n_keys, out, st);
    VMLA_DA(96, 32)
    VMLA_DA(112, 16)
    VMLA_DA(64, 64)
#undef VMLA_DA
    return VIDEOMLA_EUNSUPPORTED;
}

size_t videomla_query_projection_workspace_size(const videomla_dims* dims, int d_q, int batch, int n_tok) {
    if (!dims || d_q <= 0 || batch <= 0 || n_tok <= 0) return 0;
    const size_t m = size_t(batch) * n_tok;
    // per-row partial sums of squares (one per column tile of the first GEMM, at most
    // d_q / 128 of them), then g (.) c^Q in bf16
    return align256(m * 4 * size_t((d_q + 127) / 128)) + m * d_q * 2;
}

int videomla_query_projection(const videomla_dims* dims, int d_q, const void* x, int batch, int n_tok,
                              const void* W_dq, const float* gamma_q, const void* W_uq, const void* W_qr,
                              void* q_nope, void* q_rope, void* workspace, size_t workspace_bytes, void* stream) {
    if (!basic_dims_ok(dims) || !x || !W_dq || !W_uq || !W_qr || !q_nope || !q_rope || !workspace)
        return VIDEOMLA_EINVAL;
    if (d_q <= 0 || d_q % 64 != 0 || dims->d_model % 64 != 0 || batch <= 0 || n_tok <= 0) return VIDEOMLA_EINVAL;
    const long long M = (long long)batch * n_tok;
    const long long nq = (long long)dims->n_heads * dims->d_nope, nr = (long long)dims->n_heads * dims->d_rope;
    if (M > (1ll << 30) || nq % 8 != 0 || nr % 8 != 0 || nq > (1 << 30) || nr > (1 << 30)) return VIDEOMLA_EINVAL;
    if (workspace_bytes < videomla_query_projection_workspace_size(dims, d_q, batch, n_tok)) return VIDEOMLA_EINVAL;
    if (!aligned16(x) || !aligned16(W_dq) || !aligned16(W_uq) || !aligned16(W_qr) || !aligned16(q_nope) ||
        !aligned16(q_rope) || !aligned16(workspace) || !aligned16(gamma_q))
        return VIDEOMLA_EINVAL;
    if (int rc = check_device()) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // RMSNorm(c^Q) = g (.) c^Q / rms(c^Q) is linear in g (.) c^Q up to the per-row factor, so it
    // is split over the two GEMMs: the first writes g (.) c^Q (bf16) and, per column tile,
    // each row's sum of squares of c^Q (fp32, before g and rounding); the second, both
    // up-projections in one launch (two column groups), sums a row's parts and scales its
    // output row by 1 / rms.
    const int bn = gemm_pair_bn(int(M), d_q, 0, 1);
    const int parts = (d_q + bn - 1) / bn;
    float* ss = static_cast<float*>(workspace);
    auto* cqg = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) +
                                                 align256(size_t(M) * 4 * size_t((d_q + 127) / 128)));
    GemmEpilogue first;
    first.row_ss = ss;
    first.col_scale = gamma_q;
    if (int rc = gemm(x, W_dq, int(M), d_q, dims->d_model, cqg, d_q, false, st, first)) return rc;
    GemmEpilogue second;
    second.row_ss_in = ss;
    second.ss_parts = parts;
    second.rms_dim = d_q;
    second.rms_eps = dims->rms_eps;
    return gemm2(cqg, int(M), d_q, 2, W_uq, int(nq), q_nope, int(nq), W_qr, int(nr), q_rope, int(nr), false, st,
                 second);
}

int videomla_output_projection(const videomla_dims* dims, const void* o, int batch, int n_query, const void* W_O,
                               void* y, void* stream) {
    if (!basic_dims_ok(dims) || !o || !W_O || !y || batch <= 0 || n_query <= 0) return VIDEOMLA_EINVAL;
    const long long M = (long long)batch * n_query;
    const long long K = (long long)dims->n_heads * dims->d_v;
    if (M > (1ll << 30) || K % 64 != 0 || K > (1 << 30) || dims->d_model % 8 != 0) return VIDEOMLA_EINVAL;
    if (!aligned16(o) || !aligned16(W_O) || !aligned16(y)) return VIDEOMLA_EINVAL;
    if (int rc = check_device()) return rc;
    return gemm(o, W_O, int(M), dims->d_model, int(K), y, dims->d_model, false, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ----------------------------------------------------------------------------
// videomla_attention_static_workspace: the attention workspace lives in this
// fixed device array instead of caller memory.  In host code the name below is
// only a host-side stand-in; its device address comes from cudaGetSymbolAddress.
// ----------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_static_workspace[VIDEOMLA_STATIC_WORKSPACE_BYTES];

namespace {

// Device address of g_static_workspace in the current context, or nullptr.  It
// is looked up on every call (a cheap host query): a cached address could be
// stale after cudaDeviceReset or under another context on the same device.
void* static_workspace_address() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess) {
        cudaGetLastError();  // leave no sticky error for a later launch check
        return nullptr;
    }
    return p;
}

}  // namespace

extern "C" {

int videomla_attention_static_workspace(const videomla_dims* dims, const void* q_nope, const void* q_rope,
                                        const void* W_uk, const void* W_uv, const void* cache,
                                        const videomla_window* window, int batch, int n_query, void* out, float* lse,
                                        void* stream) {
    if (!dims || !window || batch <= 0) return VIDEOMLA_EINVAL;
    const size_t need = videomla_attention_workspace_size(dims, window, batch);
    if (need == 0 || need > VIDEOMLA_STATIC_WORKSPACE_BYTES) return VIDEOMLA_EINVAL;
    if (int rc = check_device()) return rc;
    void* ws = static_workspace_address();
    if (ws == nullptr) return VIDEOMLA_ECUDA;
    return videomla_attention(dims, q_nope, q_rope, W_uk, W_uv, cache, window, batch, n_query, out, lse, ws,
                              VIDEOMLA_STATIC_WORKSPACE_BYTES, stream);
}

const char* videomla_strerror(int code) {
    switch (code) {
        case VIDEOMLA_OK: return "ok";
        case VIDEOMLA_EINVAL: return "invalid argument";
        case VIDEOMLA_EUNSUPPORTED: return "unsupported geometry (no compiled kernel instance)";
        case VIDEOMLA_ECUDA: return "CUDA error";
        case VIDEOMLA_ETIMEOUT: return "a bounded device-side wait timed out";
        case VIDEOMLA_ENODEVICE: return "no sm_100 device is current";
        default: return "unknown error";
    }
}

int videomla_device_status(int reset) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, vmla::g_status, sizeof(int)) != cudaSuccess) return VIDEOMLA_ECUDA;
    if (reset) {
        const int z = 0;
        if (cudaMemcpyToSymbol(vmla::g_status, &z, sizeof(int)) != cudaSuccess) return VIDEOMLA_ECUDA;
    }
    return v == 0 ? VIDEOMLA_OK : VIDEOMLA_ETIMEOUT;
}

uint64_t videomla_set_wait_timeout_ns(uint64_t ns) {
    return g_timeout_ns.exchange(ns == 0 ? kDefaultTimeoutNs : ns);
}

int videomla_set_attention_tiling(int mode) {
    if (mode != VIDEOMLA_TILING_AUTO && mode != VIDEOMLA_TILING_PER_HEAD && mode != VIDEOMLA_TILING_HEAD_PACKED)
        return VIDEOMLA_EINVAL;
    return g_tiling.exchange(mode);
}

int videomla_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
    if (timeout_ns == 0 || timeout_ns > 10000000000ull) return VIDEOMLA_EINVAL;
    if (int rc = check_device()) return rc;
    vmla::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return cudaGetLastError() == cudaSuccess ? VIDEOMLA_OK : VIDEOMLA_ECUDA;
}

int videomla_version(void) { return 200; }

}  // extern "C"
