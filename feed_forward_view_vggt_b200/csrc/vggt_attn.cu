// vggt_attn.cu -- C ABI of the sm_100a attention hot path (see
// include/vggt_attn.h): argument validation, TMA tensor-map encoding
// (driver entry point fetched through the runtime, so the library does not
// link libcuda), launch configuration, and the device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "vggt_attn.h"

#include "attn_kernel.cuh"
#include "qkv_kernel.cuh"
#include "sga_kernels.cuh"

#define VGGT_API extern "C" __attribute__((visibility("default")))

namespace {

using vggt::AttnParams;

struct Dims {
    int64_t N, ns, h, w, H, L, S;
};

vggt_status check_shape(const vggt_shape &s, Dims &d)
{
    if (s.n_frames < 1 || s.n_special < 0 || s.patch_h < 0 || s.patch_w < 0 || s.n_heads < 1 || s.head_dim < 1)
        return VGGT_ERR_INVALID_ARG;
    d.N = s.n_frames;
    d.ns = s.n_special;
    d.h = s.patch_h;
    d.w = s.patch_w;
    d.H = s.n_heads;
    d.L = d.ns + d.h * d.w;
    if (d.L < 1)
        return VGGT_ERR_INVALID_ARG;
    d.S = d.N * d.L;
    if (s.head_dim != vggt::kHeadDim)
        return VGGT_ERR_UNSUPPORTED;
    if (s.n_heads > 64)
        return VGGT_ERR_UNSUPPORTED;
    // Token indices, TMA coordinates (+256 rows of overhang) and the
    // multiplicities are 32-bit.
    if (d.L > (1 << 24) || d.S > INT32_MAX - 1024)
        return VGGT_ERR_UNSUPPORTED;
    return VGGT_OK;
}

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int64_t axis_windows(int64_t n, int64_t s)
{
    return (n + s - 1) / s;
}

bool sga_counts(const Dims &d, int32_t s_h, int32_t s_w, int64_t &kept, int64_t &dropped)
{
    if (s_h < 1 || s_w < 1)
        return false;
    const int64_t kp = axis_windows(d.h, s_h) * axis_windows(d.w, s_w);
    kept = d.N * (d.ns + kp);
    dropped = d.N * (d.h * d.w - kp);
    return true;
}

size_t align256(size_t x)
{
    return (x + 255) & ~static_cast<size_t>(255);
}

struct SgaLayout {
    size_t kbar, vbar, partial, kc, vc, total;
};

SgaLayout sga_layout(const Dims &d, int64_t n_kept)
{
    const size_t hd = static_cast<size_t>(d.H) * vggt::kHeadDim;
    SgaLayout l;
    l.kbar = 0;
    l.vbar = hd * 4;
    l.partial = align256(2 * hd * 4);
    l.kc = align256(l.partial + static_cast<size_t>(vggt::kMeanfillBlocks) * 2 * hd * 4);
    l.vc = align256(l.kc + static_cast<size_t>(n_kept) * hd * 2);
    l.total = align256(l.vc + static_cast<size_t>(n_kept) * hd * 2);
    return l;
}

// ---------------------------------------------------------------- TMA maps

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// [rows, H, 64] bf16 viewed as a 3-D tensor (64, H, rows); box 64 x 1 x
// box_rows with the 128-byte swizzle the UMMA descriptors expect.
bool make_rows_map(CUtensorMap *map, const void *base, int64_t rows, int64_t H, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(vggt::kHeadDim), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(vggt::kHeadDim) * 2,
                                   static_cast<cuuint64_t>(H) * vggt::kHeadDim * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(vggt::kHeadDim), 1u, box_rows};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major bf16 matrix [rows][cols] tiled as [box_rows][64], 128-byte swizzle.
bool make_2d_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(vggt::kGemmBK), box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Store map of a row-major bf16 output block [rows][cols]: 32 x 32 boxes,
// 64-byte swizzle (the projection epilogue's staged chunks).
bool make_store_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {32u, 32u};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------ device symbols

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique ID of the calling thread's current context (never reused by the
// driver, so a context destroyed by cudaDeviceReset and created again gets
// a new one); 0 when it cannot be told.
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<CtxGetCurrentFn>(p);
    }();
    static CtxGetIdFn get_id = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<CtxGetIdFn>(p);
    }();
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device addresses of the library's file-scope device arrays, looked up
// once per device and context (host code cannot use a __device__ symbol as
// a device pointer; cudaDeviceReset gives the arrays a new context, whose
// new ID triggers a fresh lookup).
struct SymbolCache {
    std::mutex mu;
    void *ptr[64];
    unsigned long long ctx[64];
};

template <typename T>
vggt_status device_symbol(const T &symbol, SymbolCache &cache, void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (dev < 0 || dev >= 64)
        return VGGT_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(cache.mu);
    const unsigned long long ctx = current_context_id();
    if (!cache.ptr[dev] || ctx == 0 || ctx != cache.ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || !p)
            return VGGT_ERR_CUDA;
        cache.ptr[dev] = p;
        cache.ctx[dev] = current_context_id();  // the lookup has made the context current
    }
    *out = cache.ptr[dev];
    return VGGT_OK;
}

SymbolCache g_pace_cache;
std::atomic<unsigned int> g_pace_next{0};

// A zeroed pacing counter for one global-attention or SGA launch on
// `stream` (see the item pacing in the kernel), or nullptr if none can be
// had -- pacing is an optimisation, the launch runs without it.
unsigned int *pace_counter(cudaStream_t stream)
{
    void *base = nullptr;
    if (device_symbol(vggt::g_vggt_pace, g_pace_cache, &base) != VGGT_OK)
        return nullptr;
    unsigned int *slot = static_cast<unsigned int *>(base) + (g_pace_next.fetch_add(1) % vggt::kPaceSlots);
    if (cudaMemsetAsync(slot, 0, sizeof(unsigned int), stream) != cudaSuccess)
        return nullptr;
    return slot;
}

// ---------------------------------------------------------------- launches

std::mutex g_attr_mu;
bool g_attr_done[64];

vggt_status prepare_device(int &num_sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (dev < 0 || dev >= 64)
        return VGGT_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!g_attr_done[dev]) {
        if (cudaFuncSetAttribute(vggt::attn_fwd_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(vggt::kAttnSmemBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(vggt::attn_fwd_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(vggt::kAttnSmemBytes)) != cudaSuccess)
            return VGGT_ERR_CUDA;
        g_attr_done[dev] = true;
    }
    return VGGT_OK;
}

// The general instantiation when some item's two tiles lie in different
// units (an odd tile count per unit and more than one unit) or in register
// mode; the lean one otherwise.
void launch_kernel(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, int grid,
                   cudaStream_t stream)
{
    const bool general = p.mode == vggt::kModeRegister || ((p.qtiles & 1) && p.n_tiles > p.qtiles);
    if (general)
        vggt::attn_fwd_kernel<true><<<grid, vggt::kAttnThreads, vggt::kAttnSmemBytes, stream>>>(tq, tk, tv, p);
    else
        vggt::attn_fwd_kernel<false><<<grid, vggt::kAttnThreads, vggt::kAttnSmemBytes, stream>>>(tq, tk, tv, p);
}

vggt_status launch_attention(AttnParams &p, const void *q, const void *kmap_base, const void *vmap_base,
                             int64_t key_rows, const Dims &d, cudaStream_t stream)
{
    int num_sms = 0;
    vggt_status st = prepare_device(num_sms);
    if (st != VGGT_OK)
        return st;
    CUtensorMap tq, tk, tv;
    if (!make_rows_map(&tq, q, d.S, d.H, vggt::kBlockM) || !make_rows_map(&tk, kmap_base, key_rows, d.H, vggt::kBlockN) ||
        !make_rows_map(&tv, vmap_base, key_rows, d.H, vggt::kBlockN))
        return VGGT_ERR_CUDA;
    p.n_kt = (p.n_keys + vggt::kBlockN - 1) / vggt::kBlockN;
    const int grid = p.n_items < num_sms ? p.n_items : num_sms;
    if (grid < 1)
        return VGGT_OK;
    // Pacing for the launches whose items each stream a whole head's K/V,
    // once that K/V (n_keys x 2 x 128 B) is too large to sit in the L2
    // beside the streaming Q and O: above 48 MB (N = 100: 35 MB, none).
    const bool large_kv = static_cast<int64_t>(p.n_keys) * 2 * vggt::kHeadDim * 2 > (int64_t{48} << 20);
    p.pace = ((p.mode == vggt::kModeGlobal || p.mode == vggt::kModeSga) && large_kv) ? pace_counter(stream) : nullptr;
    launch_kernel(p, tq, tk, tv, grid, stream);
    return cudaGetLastError() == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

// Pointer checks of a call whose q, o (and lse) hold n_rows query rows and
// whose k, v hold all d.S tokens.
vggt_status check_rows(const void *q, const void *k, const void *v, const void *o, const float *lse,
                       const Dims &d, int64_t n_rows)
{
    if (!q || !k || !v || !o)
        return VGGT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return VGGT_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
        return VGGT_ERR_INVALID_ARG;
    const size_t rows = static_cast<size_t>(n_rows) * d.H * vggt::kHeadDim * 2;
    const size_t keys = static_cast<size_t>(d.S) * d.H * vggt::kHeadDim * 2;
    if (overlaps(o, rows, q, rows) || overlaps(o, rows, k, keys) || overlaps(o, rows, v, keys))
        return VGGT_ERR_INVALID_ARG;
    if (lse) {
        const size_t lb = static_cast<size_t>(n_rows) * d.H * 4;
        if (overlaps(lse, lb, o, rows) || overlaps(lse, lb, q, rows) || overlaps(lse, lb, k, keys) ||
            overlaps(lse, lb, v, keys))
            return VGGT_ERR_INVALID_ARG;
    }
    return VGGT_OK;
}

vggt_status check_qkvo(const void *q, const void *k, const void *v, const void *o, const float *lse,
                       const Dims &d)
{
    return check_rows(q, k, v, o, lse, d, d.S);
}

bool scale_ok(float scale)
{
    return std::isfinite(scale) && scale > 0.f;
}

// Query tiles of `units` units of `rows` rows each; false if the tile
// index would not fit in 32 bits.
bool set_tiles(AttnParams &p, int64_t rows, int64_t units)
{
    const int64_t qtiles = (rows + vggt::kBlockM - 1) / vggt::kBlockM;
    const int64_t tiles = qtiles * units;
    if (tiles + 2 > INT32_MAX)
        return false;
    p.qtiles = static_cast<int>(qtiles);
    p.n_tiles = static_cast<int>(tiles);
    p.n_items = static_cast<int>((tiles + 1) / 2);
    return true;
}

AttnParams base_params(int mode, const Dims &d, void *o, float *lse, float scale)
{
    AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.mode = mode;
    p.S = static_cast<int>(d.S);
    p.L = static_cast<int>(d.L);
    p.H = static_cast<int>(d.H);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.wait_limit_ns = vggt::kWaitLimitNs;
    p.stall_first_scores = 0;
    return p;
}

vggt_status attn_dense(int mode, const void *q, const void *k, const void *v, void *o, float *lse,
                       vggt_shape shape, float scale, void *stream, uint64_t wait_limit_ns = vggt::kWaitLimitNs,
                       int stall_first_scores = 0)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    if (!scale_ok(scale))
        return VGGT_ERR_INVALID_ARG;
    if ((st = check_qkvo(q, k, v, o, lse, d)) != VGGT_OK)
        return st;
    AttnParams p = base_params(mode, d, o, lse, scale);
    p.wait_limit_ns = wait_limit_ns;
    p.stall_first_scores = stall_first_scores;
    if (mode == vggt::kModeFrame) {
        p.n_keys = p.L;
        if (!set_tiles(p, p.L, d.N * d.H))
            return VGGT_ERR_UNSUPPORTED;
    } else {
        p.n_keys = p.S;
        if (!set_tiles(p, p.S, d.H))
            return VGGT_ERR_UNSUPPORTED;
    }
    return launch_attention(p, q, k, v, d.S, d, static_cast<cudaStream_t>(stream));
}

} // namespace

// ======================================================================= ABI

VGGT_API const char *vggt_status_string(vggt_status status)
{
    switch (status) {
    case VGGT_OK: return "VGGT_OK";
    case VGGT_ERR_INVALID_ARG: return "VGGT_ERR_INVALID_ARG";
    case VGGT_ERR_UNSUPPORTED: return "VGGT_ERR_UNSUPPORTED";
    case VGGT_ERR_WORKSPACE: return "VGGT_ERR_WORKSPACE";
    case VGGT_ERR_CUDA: return "VGGT_ERR_CUDA";
    case VGGT_ERR_TIMEOUT: return "VGGT_ERR_TIMEOUT";
    case VGGT_ERR_BOUNDS: return "VGGT_ERR_BOUNDS";
    }
    return "VGGT_ERR_UNKNOWN";
}

VGGT_API int32_t vggt_abi_version(void)
{
    return VGGT_ABI_VERSION;
}

VGGT_API int64_t vggt_num_tokens(vggt_shape shape)
{
    Dims d;
    const vggt_status st = check_shape(shape, d);
    return (st == VGGT_OK || st == VGGT_ERR_UNSUPPORTED) && d.L >= 1 && shape.n_frames >= 1 ? d.S : -1;
}

VGGT_API int64_t vggt_sga_num_kept(vggt_shape shape, int32_t s_h, int32_t s_w)
{
    Dims d;
    int64_t kept, dropped;
    if (check_shape(shape, d) != VGGT_OK || !sga_counts(d, s_h, s_w, kept, dropped))
        return -1;
    return kept;
}

VGGT_API int64_t vggt_sga_num_dropped(vggt_shape shape, int32_t s_h, int32_t s_w)
{
    Dims d;
    int64_t kept, dropped;
    if (check_shape(shape, d) != VGGT_OK || !sga_counts(d, s_h, s_w, kept, dropped))
        return -1;
    return dropped;
}

VGGT_API size_t vggt_sga_workspace_bytes(vggt_shape shape, int32_t s_h, int32_t s_w)
{
    Dims d;
    int64_t kept, dropped;
    if (check_shape(shape, d) != VGGT_OK || !sga_counts(d, s_h, s_w, kept, dropped))
        return 0;
    return sga_layout(d, kept).total;
}

VGGT_API vggt_status vggt_sga_build_index(vggt_shape shape, int32_t s_h, int32_t s_w, int32_t *kept_idx,
                                          int32_t *mult, void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    int64_t kept, dropped;
    if (!sga_counts(d, s_h, s_w, kept, dropped))
        return VGGT_ERR_INVALID_ARG;
    if (!kept_idx || !mult || (reinterpret_cast<uintptr_t>(kept_idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(mult) & 3u))
        return VGGT_ERR_INVALID_ARG;
    if (overlaps(kept_idx, static_cast<size_t>(kept) * 4, mult, static_cast<size_t>(d.S) * 4))
        return VGGT_ERR_INVALID_ARG;
    const int64_t total = d.S > kept ? d.S : kept;
    const int threads = 256;
    const int64_t blocks64 = (total + threads - 1) / threads;
    const int blocks = static_cast<int>(blocks64 < 65535 * 16 ? blocks64 : 65535 * 16);
    vggt::sga_index_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<int>(d.S), static_cast<int>(d.L), static_cast<int>(d.ns), static_cast<int>(d.h),
        static_cast<int>(d.w), s_h, s_w, static_cast<int>(kept), static_cast<int>(dropped), kept_idx, mult);
    return cudaGetLastError() == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

VGGT_API vggt_status vggt_attn_frame(const void *q, const void *k, const void *v, void *o, float *lse,
                                     vggt_shape shape, float scale, void *stream)
{
    return attn_dense(vggt::kModeFrame, q, k, v, o, lse, shape, scale, stream);
}

VGGT_API vggt_status vggt_attn_global(const void *q, const void *k, const void *v, void *o, float *lse,
                                      vggt_shape shape, float scale, void *stream)
{
    return attn_dense(vggt::kModeGlobal, q, k, v, o, lse, shape, scale, stream);
}

namespace {

// SGA for query rows [row0, row0 + n_rows) of the sequence: q, o (and lse)
// hold those rows, k and v all S tokens (the mean-fill and the kept keys
// cover the whole sequence; the diagonal term reads k, v at row0 + i).
// The gather + mean-fill pass over all rows of k and v ([d.S, H, 64]): the
// kept rows into kc / vc, per-block fp32 sums over the dropped tokens into
// partial ([blocks][2][H * 64]); blocks is set to the launch's block count.
vggt_status launch_gather_meanfill(const Dims &d, const void *k, const void *v, int32_t s_h, int32_t s_w,
                                   int64_t kept, float *partial, void *kc, void *vc, cudaStream_t s, int &blocks)
{
    int dev = 0, num_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return VGGT_ERR_CUDA;
    // A thread owns one 16-byte column vector of K or V: a row of both is
    // 2 * vpr threads, at most 2 * 8 * 64 = 1024; 4 blocks per SM.
    const int vpr = static_cast<int>(d.H) * vggt::kHeadDim / 8;
    const bool wide = 2 * vpr > 256;
    const int per_sm = wide ? 1 : 4;
    blocks = per_sm * num_sms < vggt::kMeanfillBlocks ? per_sm * num_sms : vggt::kMeanfillBlocks;
    const int threads = wide ? 2 * vpr : 2 * vpr * (256 / (2 * vpr));
    // reduction area + (frames up to kSlotTableMax tokens) the slot table
    const size_t red_bytes = static_cast<size_t>(threads) * 8 * sizeof(float) +
                             (d.L <= vggt::kSlotTableMax ? static_cast<size_t>(d.L) * sizeof(int) : 0);
    if (wide)
        vggt::sga_gather_meanfill_kernel<1024><<<blocks, threads, red_bytes, s>>>(
            static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<int>(d.S),
            static_cast<int>(d.L), static_cast<int>(d.ns), static_cast<int>(d.h), static_cast<int>(d.w), s_h, s_w,
            static_cast<int>(kept), vpr, partial, static_cast<uint4 *>(kc), static_cast<uint4 *>(vc));
    else
        vggt::sga_gather_meanfill_kernel<256><<<blocks, threads, red_bytes, s>>>(
            static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<int>(d.S),
            static_cast<int>(d.L), static_cast<int>(d.ns), static_cast<int>(d.h), static_cast<int>(d.w), s_h, s_w,
            static_cast<int>(kept), vpr, partial, static_cast<uint4 *>(kc), static_cast<uint4 *>(vc));
    return cudaGetLastError() == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

vggt_status sga_rows(const void *q, int64_t row0, int64_t n_rows, const void *k, const void *v, void *o, float *lse,
                     vggt_shape shape, int32_t s_h, int32_t s_w, const int32_t *kept_idx, const int32_t *mult,
                     void *workspace, size_t workspace_bytes, float scale, void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    int64_t kept, dropped;
    if (!sga_counts(d, s_h, s_w, kept, dropped) || !scale_ok(scale))
        return VGGT_ERR_INVALID_ARG;
    if (row0 < 0 || n_rows < 1 || row0 + n_rows > d.S)
        return VGGT_ERR_INVALID_ARG;
    if ((st = check_rows(q, k, v, o, lse, d, n_rows)) != VGGT_OK)
        return st;
    if (!kept_idx || !mult || (reinterpret_cast<uintptr_t>(kept_idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(mult) & 3u))
        return VGGT_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return VGGT_ERR_INVALID_ARG;
    const SgaLayout lay = sga_layout(d, kept);
    if (workspace_bytes < lay.total)
        return VGGT_ERR_WORKSPACE;
    const size_t qkv_bytes = static_cast<size_t>(d.S) * d.H * vggt::kHeadDim * 2;
    const size_t row_bytes = static_cast<size_t>(n_rows) * d.H * vggt::kHeadDim * 2;
    if (overlaps(workspace, lay.total, q, row_bytes) || overlaps(workspace, lay.total, k, qkv_bytes) ||
        overlaps(workspace, lay.total, v, qkv_bytes) || overlaps(workspace, lay.total, o, row_bytes) ||
        (lse && overlaps(workspace, lay.total, lse, static_cast<size_t>(n_rows) * d.H * 4)))
        return VGGT_ERR_INVALID_ARG;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *kbar = reinterpret_cast<float *>(ws + lay.kbar);
    float *vbar = reinterpret_cast<float *>(ws + lay.vbar);
    float *partial = reinterpret_cast<float *>(ws + lay.partial);
    void *kc = ws + lay.kc;
    void *vc = ws + lay.vc;

    // Gather of the kept rows + fp32 partial sums: one pass over every row of
    // K and V.
    int blocks = 0;
    if ((st = launch_gather_meanfill(d, k, v, s_h, s_w, kept, partial, kc, vc, s, blocks)) != VGGT_OK)
        return st;
    if (dropped > 0) {
        const int hd = static_cast<int>(d.H) * vggt::kHeadDim;
        vggt::sga_finalize_kernel<<<(2 * hd + vggt::kFinalizeCols - 1) / vggt::kFinalizeCols, 256, 0, s>>>(
            partial, hd, static_cast<int>(dropped), blocks, kbar, vbar);
        if (cudaGetLastError() != cudaSuccess)
            return VGGT_ERR_CUDA;
    }

    Dims dq = d;  // the query rows of this call
    dq.S = n_rows;
    AttnParams p = base_params(vggt::kModeSga, dq, o, lse, scale);
    p.n_keys = static_cast<int>(kept);
    if (!set_tiles(p, n_rows, d.H))
        return VGGT_ERR_UNSUPPORTED;
    p.row0 = static_cast<int>(row0);
    p.own_row0 = static_cast<int>(row0);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.mult = mult;
    p.kbar = kbar;
    p.vbar = vbar;
    p.n_dropped = static_cast<int>(dropped);
    return launch_attention(p, q, kc, vc, kept, dq, s);
}

} // namespace

VGGT_API vggt_status vggt_attn_sga(const void *q, const void *k, const void *v, void *o, float *lse,
                                   vggt_shape shape, int32_t s_h, int32_t s_w, const int32_t *kept_idx,
                                   const int32_t *mult, void *workspace, size_t workspace_bytes, float scale,
                                   void *stream)
{
    const int64_t S = vggt_num_tokens(shape);
    if (S < 1)
        return VGGT_ERR_INVALID_ARG;
    return sga_rows(q, 0, S, k, v, o, lse, shape, s_h, s_w, kept_idx, mult, workspace, workspace_bytes, scale,
                    stream);
}

VGGT_API vggt_status vggt_attn_sga_rows(const void *q_rows, int32_t row0, int32_t n_rows, const void *k,
                                        const void *v, void *o_rows, float *lse_rows, vggt_shape shape, int32_t s_h,
                                        int32_t s_w, const int32_t *kept_idx, const int32_t *mult, void *workspace,
                                        size_t workspace_bytes, float scale, void *stream)
{
    return sga_rows(q_rows, row0, n_rows, k, v, o_rows, lse_rows, shape, s_h, s_w, kept_idx, mult, workspace,
                    workspace_bytes, scale, stream);
}

VGGT_API size_t vggt_sga_partial_workspace_bytes(vggt_shape local_shape)
{
    Dims d;
    if (check_shape(local_shape, d) != VGGT_OK)
        return 0;
    return align256(static_cast<size_t>(vggt::kMeanfillBlocks) * 2 * d.H * vggt::kHeadDim * 4);
}

VGGT_API vggt_status vggt_sga_gather_partial(const void *k, const void *v, vggt_shape local_shape, int32_t s_h,
                                             int32_t s_w, void *kept_k, void *kept_v, float *dropped_sums,
                                             void *workspace, size_t workspace_bytes, void *stream)
{
    Dims d;
    vggt_status st = check_shape(local_shape, d);
    if (st != VGGT_OK)
        return st;
    int64_t kept, dropped;
    if (!sga_counts(d, s_h, s_w, kept, dropped))
        return VGGT_ERR_INVALID_ARG;
    if (!k || !v || !kept_k || !kept_v || !dropped_sums || !workspace || !aligned16(k) || !aligned16(v) ||
        !aligned16(kept_k) || !aligned16(kept_v) || !aligned16(dropped_sums) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return VGGT_ERR_INVALID_ARG;
    const size_t need = vggt_sga_partial_workspace_bytes(local_shape);
    if (workspace_bytes < need)
        return VGGT_ERR_WORKSPACE;
    const size_t hd = static_cast<size_t>(d.H) * vggt::kHeadDim;
    const size_t all = static_cast<size_t>(d.S) * hd * 2, kb = static_cast<size_t>(kept) * hd * 2, sb = 2 * hd * 4;
    const void *outs[4] = {kept_k, kept_v, dropped_sums, workspace};
    const size_t sizes[4] = {kb, kb, sb, need};
    for (int i = 0; i < 4; ++i) {
        if (overlaps(outs[i], sizes[i], k, all) || overlaps(outs[i], sizes[i], v, all))
            return VGGT_ERR_INVALID_ARG;
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(outs[i], sizes[i], outs[j], sizes[j]))
                return VGGT_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *partial = static_cast<float *>(workspace);
    int blocks = 0;
    if ((st = launch_gather_meanfill(d, k, v, s_h, s_w, kept, partial, kept_k, kept_v, s, blocks)) != VGGT_OK)
        return st;
    if (dropped == 0)
        return cudaMemsetAsync(dropped_sums, 0, sb, s) == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
    // the fixed-order reduction of the per-block sums, divided by 1: plain sums
    const int h2 = static_cast<int>(hd);
    vggt::sga_finalize_kernel<<<(2 * h2 + vggt::kFinalizeCols - 1) / vggt::kFinalizeCols, 256, 0, s>>>(
        partial, h2, 1, blocks, dropped_sums, dropped_sums + hd);
    return cudaGetLastError() == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

VGGT_API vggt_status vggt_attn_sga_gathered(const void *q_rows, int32_t row0, int32_t n_rows, const void *k_rows,
                                            const void *v_rows, const void *kept_k, const void *kept_v,
                                            const float *dropped_sums, const int32_t *mult, float *means,
                                            void *o_rows, float *lse_rows, vggt_shape shape, int32_t s_h,
                                            int32_t s_w, float scale, void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    int64_t kept, dropped;
    if (!sga_counts(d, s_h, s_w, kept, dropped) || !scale_ok(scale))
        return VGGT_ERR_INVALID_ARG;
    if (row0 < 0 || n_rows < 1 || static_cast<int64_t>(row0) + n_rows > d.S)
        return VGGT_ERR_INVALID_ARG;
    // q / o / own k, v: the n_rows rows; the kept rows stand in for "all keys"
    Dims dr = d;
    dr.S = n_rows;
    if ((st = check_rows(q_rows, k_rows, v_rows, o_rows, lse_rows, dr, n_rows)) != VGGT_OK)
        return st;
    if (!kept_k || !kept_v || !dropped_sums || !mult || !means || !aligned16(kept_k) || !aligned16(kept_v) ||
        !aligned16(dropped_sums) || !aligned16(means) || (reinterpret_cast<uintptr_t>(mult) & 3u))
        return VGGT_ERR_INVALID_ARG;
    const size_t hd = static_cast<size_t>(d.H) * vggt::kHeadDim;
    const size_t rows = static_cast<size_t>(n_rows) * hd * 2, kb = static_cast<size_t>(kept) * hd * 2;
    const size_t mb = 2 * hd * 4;
    if (overlaps(o_rows, rows, kept_k, kb) || overlaps(o_rows, rows, kept_v, kb) ||
        overlaps(means, mb, kept_k, kb) || overlaps(means, mb, kept_v, kb) || overlaps(means, mb, o_rows, rows) ||
        overlaps(means, mb, q_rows, rows) || overlaps(means, mb, k_rows, rows) || overlaps(means, mb, v_rows, rows) ||
        overlaps(means, mb, mult, static_cast<size_t>(d.S) * 4) ||
        (lse_rows && (overlaps(lse_rows, static_cast<size_t>(n_rows) * d.H * 4, kept_k, kb) ||
                      overlaps(lse_rows, static_cast<size_t>(n_rows) * d.H * 4, kept_v, kb) ||
                      overlaps(lse_rows, static_cast<size_t>(n_rows) * d.H * 4, means, mb))))
        return VGGT_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dropped > 0) {
        // k-bar, v-bar = the summed dropped rows / |D| (one "block" of sums)
        const int h2 = static_cast<int>(hd);
        vggt::sga_finalize_kernel<<<(2 * h2 + vggt::kFinalizeCols - 1) / vggt::kFinalizeCols, 256, 0, s>>>(
            dropped_sums, h2, static_cast<int>(dropped), 1, means, means + hd);
        if (cudaGetLastError() != cudaSuccess)
            return VGGT_ERR_CUDA;
    }
    AttnParams p = base_params(vggt::kModeSga, dr, o_rows, lse_rows, scale);
    p.n_keys = static_cast<int>(kept);
    if (!set_tiles(p, n_rows, d.H))
        return VGGT_ERR_UNSUPPORTED;
    p.row0 = static_cast<int>(row0);
    p.own_row0 = 0;  // k_rows / v_rows start at query row 0
    p.q = static_cast<const __nv_bfloat16 *>(q_rows);
    p.k = static_cast<const __nv_bfloat16 *>(k_rows);
    p.v = static_cast<const __nv_bfloat16 *>(v_rows);
    p.mult = mult;
    p.kbar = means;
    p.vbar = means + hd;
    p.n_dropped = static_cast<int>(dropped);
    return launch_attention(p, q_rows, kept_k, kept_v, kept, dr, s);
}

VGGT_API vggt_status vggt_attn_global_rows(const void *q_rows, int32_t n_rows, const void *k, const void *v,
                                           void *o_rows, float *lse_rows, vggt_shape shape, float scale,
                                           void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    if (!scale_ok(scale) || n_rows < 1 || n_rows > d.S)
        return VGGT_ERR_INVALID_ARG;
    if ((st = check_rows(q_rows, k, v, o_rows, lse_rows, d, n_rows)) != VGGT_OK)
        return st;
    Dims dq = d;
    dq.S = n_rows;
    AttnParams p = base_params(vggt::kModeGlobal, dq, o_rows, lse_rows, scale);
    p.n_keys = static_cast<int>(d.S);
    if (!set_tiles(p, n_rows, d.H))
        return VGGT_ERR_UNSUPPORTED;
    return launch_attention(p, q_rows, k, v, d.S, dq, static_cast<cudaStream_t>(stream));
}


VGGT_API vggt_status vggt_test_attn_global_stall(const void *q, const void *k, const void *v, void *o,
                                                 vggt_shape shape, float scale, uint64_t wait_limit_ns,
                                                 void *stream)
{
    if (wait_limit_ns < 1000000ull || wait_limit_ns > vggt::kWaitLimitNs)
        return VGGT_ERR_INVALID_ARG;
    return attn_dense(vggt::kModeGlobal, q, k, v, o, nullptr, shape, scale, stream, wait_limit_ns, 1);
}

// ------------------------------------------------------ register attention

namespace {

// The special tokens of [N, L, H, 64] bf16 seen as a 4-D tensor (64, H,
// n_special, N): dimension 2 steps one token (H*128 B), dimension 3 one
// frame (L*H*128 B).  Box 64 x 1 x n_special x frames = n_special * frames
// rows of 128 B, 128-byte swizzle.
bool make_special_map(CUtensorMap *map, const void *base, const Dims &d, uint32_t slots, uint32_t frames)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t row = static_cast<cuuint64_t>(d.H) * vggt::kHeadDim * 2;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(vggt::kHeadDim), static_cast<cuuint64_t>(d.H),
                                static_cast<cuuint64_t>(d.ns), static_cast<cuuint64_t>(d.N)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(vggt::kHeadDim) * 2, row,
                                   row * static_cast<cuuint64_t>(d.L)};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(vggt::kHeadDim), 1u, slots, frames};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace

VGGT_API vggt_status vggt_attn_register(const void *q, const void *k, const void *v, void *o, float *lse,
                                        vggt_shape shape, float scale, void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    if (d.ns < 1 || !scale_ok(scale))
        return VGGT_ERR_INVALID_ARG;
    if (d.ns > vggt::kBlockM)
        return VGGT_ERR_UNSUPPORTED;
    if ((st = check_qkvo(q, k, v, o, lse, d)) != VGGT_OK)
        return st;

    // A tile = the special tokens of `frames` whole frames, n_special *
    // frames <= 128 rows; tiles are numbered 128 rows apart.
    const int slots = static_cast<int>(d.ns);
    const int frames = vggt::kBlockM / slots;
    const int64_t tiles = (d.N + frames - 1) / frames;
    const int64_t padded = tiles * vggt::kBlockM;
    int num_sms = 0;
    if ((st = prepare_device(num_sms)) != VGGT_OK)
        return st;
    CUtensorMap tq, tk, tv;
    if (!make_special_map(&tq, q, d, slots, frames) || !make_special_map(&tk, k, d, slots, frames) ||
        !make_special_map(&tv, v, d, slots, frames))
        return VGGT_ERR_CUDA;
    AttnParams p = base_params(vggt::kModeRegister, d, o, lse, scale);
    p.S = static_cast<int>(padded);
    p.n_keys = static_cast<int>(padded);  // one key tile per frame tile; the valid columns per tile in the kernel
    if (!set_tiles(p, padded, d.H))
        return VGGT_ERR_UNSUPPORTED;
    p.tile_frames = frames;
    p.n_special = static_cast<int>(d.ns);
    p.n_frames = static_cast<int>(d.N);
    p.tile_rows = slots * frames;
    p.n_kt = (p.n_keys + vggt::kBlockN - 1) / vggt::kBlockN;
    const int grid = p.n_items < num_sms ? p.n_items : num_sms;
    launch_kernel(p, tq, tk, tv, grid, static_cast<cudaStream_t>(stream));
    return cudaGetLastError() == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

namespace {

struct SchedulePlan {
    int n_strides;
    int32_t stride[VGGT_MAX_SGA_STRIDES][2];
    int64_t kept[VGGT_MAX_SGA_STRIDES];
    size_t kept_off[VGGT_MAX_SGA_STRIDES], mult_off[VGGT_MAX_SGA_STRIDES];
    size_t sga_off, sga_bytes, total;
};

// Checks the descriptors and lays out the workspace; VGGT_OK or the reason.
vggt_status plan_schedule(const Dims &d, const vggt_layer *layers, int32_t n_layers, SchedulePlan &pl)
{
    std::memset(&pl, 0, sizeof pl);
    if (n_layers < 0 || n_layers > VGGT_MAX_LAYERS || (n_layers > 0 && !layers))
        return VGGT_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_layers; ++i) {
        const vggt_layer &ly = layers[i];
        if (ly.kind == VGGT_LAYER_REGISTER) {
            if (d.ns < 1)
                return VGGT_ERR_INVALID_ARG;
            if (d.ns > vggt::kBlockM)
                return VGGT_ERR_UNSUPPORTED;
        } else if (ly.kind == VGGT_LAYER_SGA) {
            int64_t kept, dropped;
            if (!sga_counts(d, ly.s_h, ly.s_w, kept, dropped))
                return VGGT_ERR_INVALID_ARG;
            int found = -1;
            for (int t = 0; t < pl.n_strides; ++t)
                if (pl.stride[t][0] == ly.s_h && pl.stride[t][1] == ly.s_w)
                    found = t;
            if (found < 0) {
                if (pl.n_strides == VGGT_MAX_SGA_STRIDES)
                    return VGGT_ERR_INVALID_ARG;
                pl.stride[pl.n_strides][0] = ly.s_h;
                pl.stride[pl.n_strides][1] = ly.s_w;
                pl.kept[pl.n_strides] = kept;
                const size_t sb = sga_layout(d, kept).total;
                pl.sga_bytes = sb > pl.sga_bytes ? sb : pl.sga_bytes;
                ++pl.n_strides;
            }
        } else if (ly.kind != VGGT_LAYER_FRAME && ly.kind != VGGT_LAYER_GLOBAL) {
            return VGGT_ERR_INVALID_ARG;
        }
    }
    size_t off = 0;
    for (int t = 0; t < pl.n_strides; ++t) {
        pl.kept_off[t] = off;
        off = align256(off + static_cast<size_t>(pl.kept[t]) * 4);
        pl.mult_off[t] = off;
        off = align256(off + static_cast<size_t>(d.S) * 4);
    }
    pl.sga_off = off;
    pl.total = align256(off + pl.sga_bytes);
    return VGGT_OK;
}

int stride_slot(const SchedulePlan &pl, const vggt_layer &ly)
{
    for (int t = 0; t < pl.n_strides; ++t)
        if (pl.stride[t][0] == ly.s_h && pl.stride[t][1] == ly.s_w)
            return t;
    return -1;
}

} // namespace

VGGT_API int64_t vggt_schedule_workspace_bytes(vggt_shape shape, const vggt_layer *layers, int32_t n_layers)
{
    Dims d;
    SchedulePlan pl;
    if (check_shape(shape, d) != VGGT_OK || plan_schedule(d, layers, n_layers, pl) != VGGT_OK)
        return -1;
    return static_cast<int64_t>(pl.total);
}

VGGT_API vggt_status vggt_attn_schedule(const void *const *q, const void *const *k, const void *const *v,
                                        void *const *o, vggt_shape shape, const vggt_layer *layers,
                                        int32_t n_layers, float scale, void *workspace, size_t workspace_bytes,
                                        void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    SchedulePlan pl;
    if ((st = plan_schedule(d, layers, n_layers, pl)) != VGGT_OK)
        return st;
    if (!scale_ok(scale))
        return VGGT_ERR_INVALID_ARG;
    if (n_layers == 0)
        return VGGT_OK;
    if (!q || !k || !v || !o)
        return VGGT_ERR_INVALID_ARG;
    if (pl.total > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return VGGT_ERR_INVALID_ARG;
    if (workspace_bytes < pl.total)
        return VGGT_ERR_WORKSPACE;
    const size_t qkv_bytes = static_cast<size_t>(d.S) * d.H * vggt::kHeadDim * 2;
    for (int32_t i = 0; i < n_layers; ++i) {
        if ((st = check_qkvo(q[i], k[i], v[i], o[i], nullptr, d)) != VGGT_OK)
            return st;
        if (pl.total > 0 && (overlaps(workspace, pl.total, q[i], qkv_bytes) || overlaps(workspace, pl.total, k[i], qkv_bytes) ||
            overlaps(workspace, pl.total, v[i], qkv_bytes) || overlaps(workspace, pl.total, o[i], qkv_bytes)))
            return VGGT_ERR_INVALID_ARG;
    }

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    for (int t = 0; t < pl.n_strides; ++t)
        if ((st = vggt_sga_build_index(shape, pl.stride[t][0], pl.stride[t][1],
                                       reinterpret_cast<int32_t *>(ws + pl.kept_off[t]),
                                       reinterpret_cast<int32_t *>(ws + pl.mult_off[t]), stream)) != VGGT_OK)
            return st;
    for (int32_t i = 0; i < n_layers; ++i) {
        const vggt_layer &ly = layers[i];
        switch (ly.kind) {
        case VGGT_LAYER_FRAME:
            st = vggt_attn_frame(q[i], k[i], v[i], o[i], nullptr, shape, scale, stream);
            break;
        case VGGT_LAYER_GLOBAL:
            st = vggt_attn_global(q[i], k[i], v[i], o[i], nullptr, shape, scale, stream);
            break;
        case VGGT_LAYER_SGA: {
            const int t = stride_slot(pl, ly);
            st = vggt_attn_sga(q[i], k[i], v[i], o[i], nullptr, shape, ly.s_h, ly.s_w,
                               reinterpret_cast<const int32_t *>(ws + pl.kept_off[t]),
                               reinterpret_cast<const int32_t *>(ws + pl.mult_off[t]), ws + pl.sga_off,
                               pl.sga_bytes, scale, stream);
            break;
        }
        default:
            st = vggt_attn_register(q[i], k[i], v[i], o[i], nullptr, shape, scale, stream);
            break;
        }
        if (st != VGGT_OK)
            return st;
    }
    return VGGT_OK;
}

namespace {

std::mutex g_qkv_mu;
bool g_qkv_done[3][64];
int g_qkv_pairs[64];  // co-resident CTA pairs of the pair form per device; -1: none

template <int BN, bool kPair>
bool qkv_set_smem(int slot, int dev)
{
    bool &done = g_qkv_done[slot][dev];
    if (!done) {
        if (cudaFuncSetAttribute(vggt::qkv_rope_kernel<BN, kPair>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(vggt::qkv_smem_bytes<BN, kPair>())) != cudaSuccess)
            return false;
        done = true;
    }
    return true;
}

template <int BN>
vggt_status launch_qkv(const CUtensorMap &tx, const CUtensorMap &tw, const vggt::QkvOutMaps &to,
                       vggt::QkvParams &p, int num_sms, int dev, cudaStream_t s)
{
    {
        std::lock_guard<std::mutex> lock(g_qkv_mu);
        if (!qkv_set_smem<BN, false>(BN == 256 ? 1 : 0, dev))
            return VGGT_ERR_CUDA;
    }
    p.n_tiles_n = p.n_out / BN;
    p.n_tiles = (p.S + vggt::kGemmBM - 1) / vggt::kGemmBM * p.n_tiles_n;
    const int grid = p.n_tiles < num_sms ? p.n_tiles : num_sms;
    vggt::qkv_rope_kernel<BN, false><<<grid, vggt::kGemmThreads, vggt::qkv_smem_bytes<BN, false>(), s>>>(tx, tw, to,
                                                                                                          p);
    return cudaGetLastError() == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

// Launch configuration of the pair form: clusters of two CTAs.
cudaLaunchConfig_t pair_config(int grid, cudaStream_t s, cudaLaunchAttribute *attr)
{
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(vggt::kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = vggt::qkv_smem_bytes<256, true>();
    cfg.stream = s;
    attr->id = cudaLaunchAttributeClusterDimension;
    attr->val.clusterDim.x = 2;
    attr->val.clusterDim.y = 1;
    attr->val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// How many CTA pairs of the pair form the device runs at once (0: it
// cannot launch them, so the single-CTA form is used); asked once per
// device.
int qkv_pair_slots(int dev, cudaStream_t s)
{
    std::lock_guard<std::mutex> lock(g_qkv_mu);
    int &slots = g_qkv_pairs[dev];
    if (slots == 0) {
        slots = -1;
        if (qkv_set_smem<256, true>(2, dev)) {
            cudaLaunchAttribute attr;
            cudaLaunchConfig_t cfg = pair_config(2, s, &attr);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, vggt::qkv_rope_kernel<256, true>, &cfg) == cudaSuccess && n > 0)
                slots = n;
        }
        (void)cudaGetLastError();
    }
    return slots > 0 ? slots : 0;
}

// The pair form (256 x 256 tiles); the X map has 128-row boxes (one CTA's
// rows), the W map 128-row boxes (half a tile's columns).
vggt_status launch_qkv_pair(const CUtensorMap &tx, const CUtensorMap &tw, const vggt::QkvOutMaps &to,
                            vggt::QkvParams &p, int slots, cudaStream_t s)
{
    constexpr int kTileM = vggt::QkvCfg<256, true>::kTileM;
    p.n_tiles_n = p.n_out / 256;
    p.n_tiles = (p.S + kTileM - 1) / kTileM * p.n_tiles_n;
    const int pairs = p.n_tiles < slots ? p.n_tiles : slots;
    cudaLaunchAttribute attr;
    cudaLaunchConfig_t cfg = pair_config(2 * pairs, s, &attr);
    if (cudaLaunchKernelEx(&cfg, vggt::qkv_rope_kernel<256, true>, tx, tw, to, p) != cudaSuccess)
        return VGGT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? VGGT_OK : VGGT_ERR_CUDA;
}

// Shared tail of the QKV and output projections: C a multiple of 256 takes
// the pair form when the device can co-schedule CTA pairs, else the
// single-CTA form with 256- or 128-column tiles.
vggt_status launch_projection(const void *x, const void *w, void *const *outs, int64_t n_out, vggt::QkvParams &p,
                              int num_sms, int dev, cudaStream_t s)
{
    const int64_t C = p.C;
    vggt::QkvOutMaps to;
    std::memset(&to, 0, sizeof to);
    for (int64_t i = 0; i * C < n_out; ++i)
        if (!make_store_map(&to.m[i], outs[i], p.S, C))
            return VGGT_ERR_CUDA;
    CUtensorMap tx, tw;
    if (C % 256 == 0) {
        const int slots = qkv_pair_slots(dev, s);
        if (slots > 0) {
            if (!make_2d_map(&tx, x, p.S, C, vggt::kGemmBM) ||
                !make_2d_map(&tw, w, n_out, C, static_cast<uint32_t>(vggt::QkvCfg<256, true>::kRowsB)))
                return VGGT_ERR_CUDA;
            return launch_qkv_pair(tx, tw, to, p, slots, s);
        }
    }
    const int bn = (C % 256 == 0) ? 256 : 128;
    if (!make_2d_map(&tx, x, p.S, C, vggt::kGemmBM) || !make_2d_map(&tw, w, n_out, C, static_cast<uint32_t>(bn)))
        return VGGT_ERR_CUDA;
    return bn == 256 ? launch_qkv<256>(tx, tw, to, p, num_sms, dev, s)
                     : launch_qkv<128>(tx, tw, to, p, num_sms, dev, s);
}

} // namespace

VGGT_API vggt_status vggt_qkv_rope(const void *x, const void *w, const float *bias, void *q, void *k, void *v,
                                   vggt_shape shape, float rope_base, void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    if (d.H % 2 != 0 || d.h > vggt::kRopeMaxPos || d.w > vggt::kRopeMaxPos)
        return VGGT_ERR_UNSUPPORTED;
    if (!std::isfinite(rope_base) || !(rope_base > 0.f))
        return VGGT_ERR_INVALID_ARG;
    if (!x || !w || !q || !k || !v || !aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) ||
        !aligned16(v) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return VGGT_ERR_INVALID_ARG;
    const int64_t C = d.H * vggt::kHeadDim;
    const size_t xb = static_cast<size_t>(d.S) * C * 2, wb = static_cast<size_t>(3 * C) * C * 2, bb = 3 * C * 4;
    const void *outs[3] = {q, k, v};
    for (int i = 0; i < 3; ++i) {
        if (overlaps(outs[i], xb, x, xb) || overlaps(outs[i], xb, w, wb) || (bias && overlaps(outs[i], xb, bias, bb)))
            return VGGT_ERR_INVALID_ARG;
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(outs[i], xb, outs[j], xb))
                return VGGT_ERR_INVALID_ARG;
    }
    int dev = 0, num_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (dev < 0 || dev >= 64)
        return VGGT_ERR_UNSUPPORTED;
    vggt::QkvParams p;
    std::memset(&p, 0, sizeof p);
    p.S = static_cast<int>(d.S);
    p.C = static_cast<int>(C);
    p.n_out = static_cast<int>(3 * C);
    p.rope_cols = static_cast<int>(2 * C);
    p.k_chunks = static_cast<int>(C / vggt::kGemmBK);
    p.L = static_cast<int>(d.L);
    p.n_special = static_cast<int>(d.ns);
    p.pw = d.w > 0 ? static_cast<int>(d.w) : 1;
    p.log2_base = std::log2(rope_base);
    p.bias = bias;
    p.wait_limit_ns = vggt::kWaitLimitNs;
    void *const blocks[3] = {q, k, v};
    return launch_projection(x, w, blocks, 3 * C, p, num_sms, dev, static_cast<cudaStream_t>(stream));
}

VGGT_API vggt_status vggt_out_proj(const void *o, const void *w, const float *bias, void *y, vggt_shape shape,
                                   void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    if (d.H % 2 != 0)
        return VGGT_ERR_UNSUPPORTED;
    if (!o || !w || !y || !aligned16(o) || !aligned16(w) || !aligned16(y) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return VGGT_ERR_INVALID_ARG;
    const int64_t C = d.H * vggt::kHeadDim;
    const size_t ob = static_cast<size_t>(d.S) * C * 2, wb = static_cast<size_t>(C) * C * 2;
    if (overlaps(y, ob, o, ob) || overlaps(y, ob, w, wb) || (bias && overlaps(y, ob, bias, C * 4)))
        return VGGT_ERR_INVALID_ARG;
    int dev = 0, num_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (dev < 0 || dev >= 64)
        return VGGT_ERR_UNSUPPORTED;
    vggt::QkvParams p;
    std::memset(&p, 0, sizeof p);
    p.S = static_cast<int>(d.S);
    p.C = static_cast<int>(C);
    p.n_out = static_cast<int>(C);
    p.rope_cols = 0;
    p.k_chunks = static_cast<int>(C / vggt::kGemmBK);
    p.L = static_cast<int>(d.L);
    p.n_special = static_cast<int>(d.ns);
    p.pw = d.w > 0 ? static_cast<int>(d.w) : 1;
    p.log2_base = 0.f;
    p.bias = bias;
    p.wait_limit_ns = vggt::kWaitLimitNs;
    void *const blocks[1] = {y};
    return launch_projection(o, w, blocks, C, p, num_sms, dev, static_cast<cudaStream_t>(stream));
}

VGGT_API vggt_status vggt_check(void *stream, uint32_t *detail)
{
    if (detail)
        *detail = 0;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return VGGT_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, vggt::g_vggt_error, sizeof word) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (word == 0)
        return VGGT_OK;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(vggt::g_vggt_error, &zero, sizeof zero) != cudaSuccess)
        return VGGT_ERR_CUDA;
    if (detail)
        *detail = word;
    return (word & vggt::kErrTimeout) ? VGGT_ERR_TIMEOUT : VGGT_ERR_BOUNDS;
}

VGGT_API int32_t vggt_debug_checks(void)
{
#ifdef VGGT_DEBUG
    return 1;
#else
    return 0;
#endif
}

// ------------------------------------------------ allocation-free SGA entry

namespace {

// Scratch for vggt_attn_sga_noalloc: replaces the caller's workspace.
static __device__ __align__(256) unsigned char g_sga_static_scratch[VGGT_SGA_STATIC_SCRATCH_BYTES];

SymbolCache g_static_cache;

// Device address of the scratch array on the current device, looked up once
// per device and context (see device_symbol).
vggt_status static_scratch(void **out)
{
    return device_symbol(g_sga_static_scratch, g_static_cache, out);
}

} // namespace

VGGT_API vggt_status vggt_attn_sga_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                           vggt_shape shape, int32_t s_h, int32_t s_w, const int32_t *kept_idx,
                                           const int32_t *mult, float scale, void *stream)
{
    Dims d;
    vggt_status st = check_shape(shape, d);
    if (st != VGGT_OK)
        return st;
    int64_t kept, dropped;
    if (!sga_counts(d, s_h, s_w, kept, dropped))
        return VGGT_ERR_INVALID_ARG;
    if (sga_layout(d, kept).total > VGGT_SGA_STATIC_SCRATCH_BYTES)
        return VGGT_ERR_WORKSPACE;
    // The argument checks of vggt_attn_sga, before the scratch lookup touches
    // the device: a bad pointer is VGGT_ERR_INVALID_ARG on any machine.
    if (!scale_ok(scale))
        return VGGT_ERR_INVALID_ARG;
    if ((st = check_qkvo(q, k, v, o, lse, d)) != VGGT_OK)
        return st;
    if (!kept_idx || !mult || (reinterpret_cast<uintptr_t>(kept_idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(mult) & 3u))
        return VGGT_ERR_INVALID_ARG;
    void *scratch = nullptr;
    if ((st = static_scratch(&scratch)) != VGGT_OK)
        return st;
    return vggt_attn_sga(q, k, v, o, lse, shape, s_h, s_w, kept_idx, mult, scratch,
                         VGGT_SGA_STATIC_SCRATCH_BYTES, scale, stream);
}
