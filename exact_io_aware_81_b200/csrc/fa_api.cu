// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument validation,
// TMA tensor-map encoding, kernel launches on the caller's stream, and the device error
// word.  The library owns no device memory on the compute path; the caller passes every
// buffer, including the decode workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_common.cuh"
#include "fa_decode_sm100.cuh"
#include "fa_prefill_sm100.cuh"

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;

thread_local char g_msg[512] = "";
unsigned long long g_wait_limit_ns = kDefaultWaitLimitNs;

int fail(int status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return status;
}

int ok()
{
    g_msg[0] = '\0';
    return FA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------ device facts, cached

struct DeviceInfo {
    bool valid = false;
    bool sm100 = false;
    int num_sms = 0;
    bool prefill_attr_set[2][2][2][2][2] = {};
    bool decode_attr_set[2][4][2][2] = {};
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device(int *dev, DeviceInfo **info)
{
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (*dev < 0 || *dev >= kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device index %d", *dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[*dev];
    if (!d.valid) {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev);
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev);
        if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        d.sm100 = (major == 10 && minor == 0);
        d.num_sms = sms;
        d.valid = true;
    }
    *info = &d;
    if (!d.sm100) return fail(FA_ERR_UNSUPPORTED, "libfa.so is built for sm_100a (B200) only");
    return FA_OK;
}

// -------------------------------------------------------------- TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Encoded maps are cached on the host, keyed by every argument of the encode call (data
// type, rank, base address, sizes, strides, box): a map is a pure function of these, so a
// hit returns exactly what re-encoding would.  Repeated calls on the same buffers (a
// serving loop, a benchmark) then skip the driver's encode, about a microsecond per map.
struct MapKey {
    int dtype, rank;
    const void *base;
    cuuint64_t dims[4], strides[3];
    cuuint32_t box[4];
};
constexpr int kMapCacheSize = 64;
struct MapCache {
    MapKey key[kMapCacheSize];
    CUtensorMap map[kMapCacheSize];
    bool used[kMapCacheSize] = {};
    int next = 0;
};
MapCache g_maps;
std::mutex g_maps_mu;

int encode_map_cached(CUtensorMap *m, CUtensorMapDataType dtype, int rank, const void *base,
                      const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box)
{
    MapKey k;
    memset(&k, 0, sizeof k);  // padding too: keys are compared bytewise
    k.dtype = (int)dtype;
    k.rank = rank;
    k.base = base;
    for (int i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        if (i + 1 < rank) k.strides[i] = strides[i];
    }
    {
        std::lock_guard<std::mutex> lk(g_maps_mu);
        for (int i = 0; i < kMapCacheSize; ++i)
            if (g_maps.used[i] && memcmp(&g_maps.key[i], &k, sizeof k) == 0) {
                *m = g_maps.map[i];
                return FA_OK;
            }
    }
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, dtype, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    std::lock_guard<std::mutex> lk(g_maps_mu);
    const int slot = g_maps.next;
    g_maps.next = (slot + 1) % kMapCacheSize;
    g_maps.key[slot] = k;
    g_maps.map[slot] = *m;
    g_maps.used[slot] = true;
    return FA_OK;
}

// A (D, rows, planes) bf16 tensor with boxes of `box_rows` rows x 64 columns, 128-byte
// swizzle.
int encode_rows_map(CUtensorMap *m, const void *base, int D, long long rows, long long planes,
                    unsigned box_rows = 128, bool fp8 = false)
{
    // one box row is 128 bytes: 64 bf16 or 128 FP8 (byte) elements
    const cuuint64_t eb = fp8 ? 1 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)planes};
    const cuuint64_t strides[2] = {(cuuint64_t)D * eb, (cuuint64_t)rows * D * eb};
    const cuuint32_t box[3] = {(cuuint32_t)(128 / eb), box_rows, 1};
    return encode_map_cached(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base,
                             dims, strides, box);
}

// A prefill operand as a 4-D (d, rows, heads, batch) tensor with boxes of `box_rows` rows x
// 128 bytes of one head (64 bf16 or 128 E4M3 columns), 128-byte swizzle.  The memory layout
// is (batch, heads, rows, d), or (batch, rows, heads, d) when `bshd`: only the strides differ.
int encode_heads_map(CUtensorMap *m, const void *base, int D, int rows, int heads, int batch, bool bshd,
                     unsigned box_rows = 128, bool fp8 = false)
{
    const cuuint64_t eb = fp8 ? 1 : 2;
    const cuuint64_t row = (cuuint64_t)D * eb, plane = (cuuint64_t)rows * heads * row;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)batch};
    const cuuint64_t strides[3] = {bshd ? heads * row : row, bshd ? row : rows * row, plane};
    const cuuint32_t box[4] = {(cuuint32_t)(128 / eb), box_rows, 1, 1};
    return encode_map_cached(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base,
                             dims, strides, box);
}

// ------------------------------------------------------------------- prefill

int validate_fwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                 int o_dtype)
{
    if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID, "null pointer argument");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0)
        return fail(FA_ERR_INVALID, "sizes must be positive (B=%d Hq=%d Hkv=%d Nq=%d Nk=%d d=%d)",
                    B, Hq, Hkv, Nq, Nk, d);
    if (Hq % Hkv != 0) return fail(FA_ERR_INVALID, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (causal && Nq > Nk) return fail(FA_ERR_INVALID, "causal attention needs Nq <= Nk (%d > %d)", Nq, Nk);
    if (!(scale > 0.f) || !std::isfinite(scale)) return fail(FA_ERR_INVALID, "scale must be finite and > 0");
    if (o_dtype != FA_BF16 && o_dtype != FA_F32) return fail(FA_ERR_INVALID, "unknown output dtype %d", o_dtype);
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(FA_ERR_UNSUPPORTED, "q, k, v and o must be 16-byte aligned");
    if ((long long)B * Hq > 0x7fffffffLL || (long long)B * Hkv * Nk > 0x7fffffffLL * 64LL)
        return fail(FA_ERR_UNSUPPORTED, "problem too large");
    return FA_OK;
}

template <int D, bool F32, bool SPLIT, bool WINDOW, bool FP8 = false>
int launch_prefill(const fa::PrefillParams &p, DeviceInfo *info, cudaStream_t st)
{
    using C = fa::prefill::Cfg<D, FP8>;
    static_assert(C::kSmemBytes <= 227 * 1024, "prefill shared memory");
    auto kern = fa::fa_prefill_kernel<D, F32, SPLIT, WINDOW, FP8>;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        bool &set = info->prefill_attr_set[D == 128][F32][SPLIT][WINDOW][FP8];
        if (!set) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 C::kSmemBytes);
            if (e != cudaSuccess)
                return fail(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            set = true;
        }
    }
    const int grid = p.n_slots < info->num_sms ? p.n_slots : info->num_sms;
    kern<<<grid, fa::prefill::kThreads, C::kSmemBytes, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
    return FA_OK;
}

// Kernel variant for one head dim, output type and input type: P handed over in halves for
// head-pair tiling, and the sliding-window variant only when a window is set.
template <int D, bool F32, bool FP8 = false>
int launch_prefill_variant(const fa::PrefillParams &p, DeviceInfo *info, cudaStream_t st)
{
    const bool win = p.window > 0;
    if (p.head_pair)
        return win ? launch_prefill<D, F32, true, true, FP8>(p, info, st)
                   : launch_prefill<D, F32, true, false, FP8>(p, info, st);
    return win ? launch_prefill<D, F32, false, true, FP8>(p, info, st)
               : launch_prefill<D, F32, false, false, FP8>(p, info, st);
}

// FP8 inputs: E4M3 Q, K, V with per-head scales (q_scale, k_scale, v_scale non-null).
struct Fp8Scales {
    const float *q, *k, *v;
};

int fwd_impl(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int causal, int window, int o_dtype,
             bool bshd, void *stream, int selftest_timeout, const Fp8Scales *fp8 = nullptr,
             bool debug_bounds_selftest = false)
{
    int rc = validate_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, o_dtype);
    if (rc != FA_OK) return rc;
    if (window < 0) return fail(FA_ERR_INVALID, "window must be >= 0 (got %d)", window);
    if (window > 0 && !causal) return fail(FA_ERR_INVALID, "a sliding window needs causal attention");
    if (fp8 && (!fp8->q || !fp8->k || !fp8->v)) return fail(FA_ERR_INVALID, "null scale pointer");
    if (fp8 && d != 128) return fail(FA_ERR_UNSUPPORTED, "FP8 prefill needs d = 128 (got %d)", d);
    int dev;
    DeviceInfo *info;
    if ((rc = current_device(&dev, &info)) != FA_OK) return rc;

    fa::PrefillParams p;
    memset(&p, 0, sizeof p);
    const bool f8 = fp8 != nullptr;
    if ((rc = encode_heads_map(&p.tm_q, q, d, Nq, Hq, B, bshd, 128, f8)) != FA_OK) return rc;
    if ((rc = encode_heads_map(&p.tm_k, k, d, Nk, Hkv, B, bshd, 128, f8)) != FA_OK) return rc;
    if ((rc = encode_heads_map(&p.tm_v, v, d, Nk, Hkv, B, bshd, 128, f8)) != FA_OK) return rc;
    // bf16 O leaves through TMA stores of one warp's 32 rows
    if (o_dtype == FA_BF16 && (rc = encode_heads_map(&p.tm_o, o, d, Nq, Hq, B, bshd, 32)) != FA_OK) return rc;
    if (f8) {
        p.q_scale = fp8->q;
        p.k_scale = fp8->k;
        p.v_scale = fp8->v;
    }
    p.o = o;
    p.o_sb = (long long)Hq * Nq * d;
    p.o_sh = bshd ? d : (long long)Nq * d;
    p.o_sn = bshd ? (long long)Hq * d : d;
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.R = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.window = window < Nk ? window : 0;  // a window of Nk or more keys is plain causal
    p.head_pair = (p.R % 2 == 0) ? 1 : 0;
    const int tiles = (Nq + 127) / 128;
    long long head_slots;
    if (p.head_pair) {
        p.T = tiles;
        head_slots = (long long)B * Hkv * (p.R / 2);
    } else {
        p.T = (tiles + 1) / 2;
        head_slots = (long long)B * Hq;
    }
    p.P = p.causal ? (p.T + 1) / 2 : p.T;
    const long long slots = head_slots * p.P;
    if (slots > 0x3fffffffLL) return fail(FA_ERR_UNSUPPORTED, "problem too large");
    p.n_slots = (int)slots;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.wait_limit_ns = g_wait_limit_ns;
    p.selftest_no_s_signal = selftest_timeout;
    // the debug build's bounds self-test moves every LSE index past the end of its buffer
    p.debug_lse_offset = debug_bounds_selftest ? (long long)B * Hq * Nq : 0;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool f32 = o_dtype == FA_F32;
    if (f8)
        rc = f32 ? launch_prefill_variant<128, true, true>(p, info, st)
                 : launch_prefill_variant<128, false, true>(p, info, st);
    else if (d == 128)
        rc = f32 ? launch_prefill_variant<128, true>(p, info, st) : launch_prefill_variant<128, false>(p, info, st);
    else
        rc = f32 ? launch_prefill_variant<64, true>(p, info, st) : launch_prefill_variant<64, false>(p, info, st);
    if (rc != FA_OK) return rc;
    return ok();
}

// -------------------------------------------------------------------- decode

long long decode_splits(int Nmax) { return (Nmax + fa::decode::kChunk - 1) / fa::decode::kChunk; }

// Rows per TMA box of the decode kernels: the 64-row stages of the bf16 kernel and the
// 64-key blocks of the FP8 one.
int decode_block_keys(int, bool fp8) { return fp8 ? fa::decode::kSK : fa::decode::kSub; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t decode_ws_bytes(int B, int Hq, int Nmax, int d)
{
    if (B <= 0 || Hq <= 0 || Nmax <= 0 || d <= 0) return 0;
    const size_t S = (size_t)decode_splits(Nmax);
    return align256((size_t)B * Hq * S * d * sizeof(float)) + align256((size_t)B * Hq * S * sizeof(float));
}

// Persistent split kernel, 3 CTAs per SM (at most one per candidate work item): the bf16
// kernel, or the FP8 one (head dim 128).
template <int D, int RG, bool PAGED, bool FP8>
int launch_split(fa::DecodeParams p, DeviceInfo *info, cudaStream_t st)
{
    static_assert(!FP8 || D == 128, "FP8 caches: head dim 128");
    constexpr int smem = FP8 ? fa::decode::WorkerCfg<RG>::kSmemBytes : fa::decode::SplitCfg<D, RG>::kSmemBytes;
    static_assert(smem * fa::decode::kCtasPerSm <= 227 * 1024, "decode CTAs per SM do not fit");
    void (*kern)(fa::DecodeParams);
    if constexpr (FP8) kern = fa::fa_decode_fp8_kernel<RG, PAGED>;
    else kern = fa::fa_decode_split_kernel<D, RG, PAGED>;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        bool &set = info->decode_attr_set[D == 128][RG == 8 ? 3 : RG == 4 ? 2 : RG == 2 ? 1 : 0][PAGED][FP8];
        if (!set) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess)
                return fail(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            set = true;
        }
    }
    p.n_hg = p.Hq / RG;
    p.n_items = p.S_max * p.B * p.n_hg;
    const int max_ctas = fa::decode::kCtasPerSm * info->num_sms;
    const int grid = p.n_items < max_ctas ? p.n_items : max_ctas;
    kern<<<grid, fa::decode::kThreads, smem, st>>>(p);
    return FA_OK;
}

template <int D, bool PAGED = false, bool FP8 = false>
int launch_split_rg(const fa::DecodeParams &p, int rg, DeviceInfo *info, cudaStream_t st)
{
    switch (rg) {
    case 8: return launch_split<D, 8, PAGED, FP8>(p, info, st);
    case 4: return launch_split<D, 4, PAGED, FP8>(p, info, st);
    case 2: return launch_split<D, 2, PAGED, FP8>(p, info, st);
    default: return launch_split<D, 1, PAGED, FP8>(p, info, st);
    }
}

// The merge kernel is launched as a programmatic dependent of the split kernel, so its
// launch overlaps the split kernel's tail; griddepcontrol.wait inside it orders the reads.
template <int D>
cudaError_t launch_merge(const fa::DecodeParams &p, cudaStream_t st)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.B * p.Hq));
    cfg.blockDim = dim3(32 * fa::kMergeWarps);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fa::fa_decode_merge_kernel<D>, p);
}

}  // namespace

namespace {

// The caches of a decode call beyond the contiguous bf16 layout of fa_decode.
struct CacheDesc {
    const void *k, *v;                // contiguous caches (B, Hkv, Nmax, d) or page pools
    bool fp8;                         // E4M3 bytes with per-head scales
    const float *k_scale, *v_scale;   // (Hkv) each, FP8 only
    bool paged;
    const int *block_table;           // (B, max_pages), paged only
    int num_pages, page_size, max_pages;
};

// Validation and launch shared by every decode entry point.  Nmax is the contiguous cache
// length (ignored when paged: page_size * max_pages).
int decode_general(const void *q, const CacheDesc &c, const int *seqlens, void *o, float *lse,
                   int B, int Hq, int Hkv, int Nmax, int d, float scale, void *workspace,
                   size_t workspace_bytes, void *stream, int o_dtype = FA_BF16, int selftest = 0)
{
    if (o_dtype != FA_BF16 && o_dtype != FA_F32) return fail(FA_ERR_INVALID, "unknown output dtype %d", o_dtype);
    if (!q || !c.k || !c.v || !seqlens || !o) return fail(FA_ERR_INVALID, "null pointer argument");
    if (c.fp8 && (!c.k_scale || !c.v_scale)) return fail(FA_ERR_INVALID, "null scale pointer");
    if (c.paged && !c.block_table) return fail(FA_ERR_INVALID, "null block table");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0)
        return fail(FA_ERR_INVALID, "sizes must be positive (B=%d Hq=%d Hkv=%d d=%d)", B, Hq, Hkv, d);
    if (c.paged) {
        if (c.num_pages <= 0 || c.page_size <= 0 || c.max_pages <= 0)
            return fail(FA_ERR_INVALID, "page sizes must be positive (num_pages=%d page_size=%d max_pages=%d)",
                        c.num_pages, c.page_size, c.max_pages);
    } else if (Nmax <= 0) {
        return fail(FA_ERR_INVALID, "Nmax must be positive (%d)", Nmax);
    }
    if (Hq % Hkv != 0) return fail(FA_ERR_INVALID, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (!(scale > 0.f) || !std::isfinite(scale)) return fail(FA_ERR_INVALID, "scale must be finite and > 0");
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    if (c.fp8 && d != 128) return fail(FA_ERR_UNSUPPORTED, "FP8 caches need d = 128 (got %d)", d);
    if (c.paged && c.page_size % 16 != 0)
        return fail(FA_ERR_UNSUPPORTED, "page_size %d is not a multiple of 16", c.page_size);
    if (!aligned16(q) || !aligned16(c.k) || !aligned16(c.v) || !aligned16(o))
        return fail(FA_ERR_UNSUPPORTED, "q, the caches and o must be 16-byte aligned");
    const long long nmax = c.paged ? (long long)c.page_size * c.max_pages : Nmax;
    const long long planes = c.paged ? (long long)c.num_pages * Hkv : (long long)B * Hkv;
    if (B > 65535 || nmax > 0x7fffffffLL || planes > 0x7fffffffLL)
        return fail(FA_ERR_UNSUPPORTED, "problem too large");
    Nmax = (int)nmax;
    const size_t need = decode_ws_bytes(B, Hq, Nmax, d);
    if (!workspace || workspace_bytes < need)
        return fail(FA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned16(workspace)) return fail(FA_ERR_WORKSPACE, "workspace must be 16-byte aligned");
    int dev, rc;
    DeviceInfo *info;
    if ((rc = current_device(&dev, &info)) != FA_OK) return rc;

    const int R = Hq / Hkv;
    const int rg = (R % 8 == 0) ? 8 : (R % 4 == 0) ? 4 : (R % 2 == 0) ? 2 : 1;
    if (Hq / rg > 65535) return fail(FA_ERR_UNSUPPORTED, "too many head groups");

    fa::DecodeParams p;
    memset(&p, 0, sizeof p);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    if (c.paged) {
        // rows per copy: the largest power of two that divides page_size, at most one block
        p.box_rows = c.page_size & -c.page_size;
        if (p.box_rows > decode_block_keys(d, c.fp8)) p.box_rows = decode_block_keys(d, c.fp8);
        p.block_table = c.block_table;
        p.page_size = c.page_size;
        p.max_pages = c.max_pages;
        p.num_pages = c.num_pages;
    } else {
        p.box_rows = decode_block_keys(d, c.fp8);
    }
    const long long map_rows = c.paged ? c.page_size : Nmax;
    if ((rc = encode_rows_map(&p.tm_k, c.k, d, map_rows, planes, p.box_rows, c.fp8)) != FA_OK) return rc;
    if ((rc = encode_rows_map(&p.tm_v, c.v, d, map_rows, planes, p.box_rows, c.fp8)) != FA_OK) return rc;
    p.k_scale = c.k_scale;
    p.v_scale = c.v_scale;
    p.seqlens = seqlens;
    p.S_max = (int)decode_splits(Nmax);
    p.part_o = static_cast<float *>(workspace);
    p.part_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                           align256((size_t)B * Hq * p.S_max * d * sizeof(float)));
    if (o_dtype == FA_F32) p.o_f32 = static_cast<float *>(o);
    else p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nmax = Nmax;
    p.R = R;
    p.scale_log2 = scale * 1.4426950408889634f;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    p.wait_limit_ns = g_wait_limit_ns;
    p.selftest_no_full = selftest;
    if (c.fp8)
        rc = c.paged ? launch_split_rg<128, true, true>(p, rg, info, st) : launch_split_rg<128, false, true>(p, rg, info, st);
    else if (c.paged)
        rc = (d == 128) ? launch_split_rg<128, true>(p, rg, info, st) : launch_split_rg<64, true>(p, rg, info, st);
    else
        rc = (d == 128) ? launch_split_rg<128, false>(p, rg, info, st) : launch_split_rg<64, false>(p, rg, info, st);
    if (rc != FA_OK) return rc;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "decode split launch: %s", cudaGetErrorString(e));
    e = (d == 128) ? launch_merge<128>(p, st) : launch_merge<64>(p, st);
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "decode merge launch: %s", cudaGetErrorString(e));
    return ok();
}

}  // namespace

extern "C" {

int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int d, float scale, int causal, void *stream)
{
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, FA_BF16, false, stream, 0);
}

int fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
              int Hkv, int Nq, int Nk, int d, float scale, int causal, int o_dtype, void *stream)
{
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, o_dtype, false, stream, 0);
}

int fa_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                  int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window, int o_dtype,
                  void *stream)
{
    if (window <= 0) return fail(FA_ERR_INVALID, "window must be >= 1 (got %d)", window);
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, 1, window, o_dtype, false, stream, 0);
}

int fa_fwd_bshd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int d, float scale, int causal, int window, int o_dtype,
                void *stream)
{
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, o_dtype, true, stream, 0);
}

int fa_fwd_fp8(const void *q, const void *k, const void *v, const float *q_scale, const float *k_scale,
               const float *v_scale, void *o, float *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
               float scale, int causal, int window, int o_dtype, void *stream)
{
    if (window > 0 && !causal) return fail(FA_ERR_INVALID, "a sliding window needs causal attention");
    const Fp8Scales sc{q_scale, k_scale, v_scale};
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, o_dtype, false, stream, 0, &sc);
}

int fa_fwd_selftest_timeout(const void *q, const void *k, const void *v, void *o, float *lse,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                            int causal, void *stream)
{
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, FA_BF16, false, stream, 1);
}

size_t fa_decode_workspace_size(int B, int Hq, int Nmax, int d) { return decode_ws_bytes(B, Hq, Nmax, d); }

int fa_decode(const void *q, const void *kcache, const void *vcache, const int *seqlens, void *o,
              float *lse, int B, int Hq, int Hkv, int Nmax, int d, float scale, void *workspace,
              size_t workspace_bytes, void *stream)
{
    const CacheDesc c{kcache, vcache, false, nullptr, nullptr, false, nullptr, 0, 0, 0};
    return decode_general(q, c, seqlens, o, lse, B, Hq, Hkv, Nmax, d, scale, workspace, workspace_bytes, stream);
}


int fa_decode_paged(const void *q, const void *kpages, const void *vpages, const int *block_table,
                    const int *seqlens, void *o, float *lse, int B, int Hq, int Hkv, int num_pages,
                    int page_size, int max_pages, int d, float scale, void *workspace,
                    size_t workspace_bytes, void *stream)
{
    const CacheDesc c{kpages, vpages, false, nullptr, nullptr, true, block_table, num_pages, page_size, max_pages};
    return decode_general(q, c, seqlens, o, lse, B, Hq, Hkv, 0, d, scale, workspace, workspace_bytes, stream);
}

int fa_decode_ex(const void *q, const void *kcache, const void *vcache, const int *seqlens, void *o,
                 float *lse, int B, int Hq, int Hkv, int Nmax, int d, float scale, int o_dtype,
                 void *workspace, size_t workspace_bytes, void *stream)
{
    const CacheDesc c{kcache, vcache, false, nullptr, nullptr, false, nullptr, 0, 0, 0};
    return decode_general(q, c, seqlens, o, lse, B, Hq, Hkv, Nmax, d, scale, workspace, workspace_bytes,
                          stream, o_dtype);
}

int fa_decode_selftest_timeout(const void *q, const void *kcache, const void *vcache, const float *k_scale,
                               const float *v_scale, const int *seqlens, void *o, float *lse, int B, int Hq,
                               int Hkv, int Nmax, int d, float scale, void *workspace, size_t workspace_bytes,
                               void *stream)
{
    if ((k_scale == nullptr) != (v_scale == nullptr))
        return fail(FA_ERR_INVALID, "give both FP8 scale pointers or neither");
    const bool fp8 = k_scale != nullptr;
    const CacheDesc c{kcache, vcache, fp8, k_scale, v_scale, false, nullptr, 0, 0, 0};
    return decode_general(q, c, seqlens, o, lse, B, Hq, Hkv, Nmax, d, scale, workspace, workspace_bytes,
                          stream, FA_BF16, 1);
}

int fa_merge_lse(const float *o_parts, const float *lse_parts, int P, int rows, int d, void *o,
                 float *lse, int o_dtype, void *stream)
{
    if (!o_parts || !lse_parts || !o) return fail(FA_ERR_INVALID, "null pointer argument");
    if (P <= 0 || rows <= 0 || d <= 0) return fail(FA_ERR_INVALID, "sizes must be positive (P=%d rows=%d d=%d)", P, rows, d);
    if (o_dtype != FA_BF16 && o_dtype != FA_F32) return fail(FA_ERR_INVALID, "unknown output dtype %d", o_dtype);
    if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    if ((long long)P * rows * d > 0x7fffffffffffLL) return fail(FA_ERR_UNSUPPORTED, "problem too large");
    int dev, rc;
    DeviceInfo *info;
    if ((rc = current_device(&dev, &info)) != FA_OK) return rc;
    fa::MergeLseParams m;
    m.o_parts = o_parts;
    m.lse_parts = lse_parts;
    m.o = o_dtype == FA_BF16 ? static_cast<__nv_bfloat16 *>(o) : nullptr;
    m.o_f32 = o_dtype == FA_F32 ? static_cast<float *>(o) : nullptr;
    m.lse = lse;
    m.P = P;
    m.rows = rows;
    const unsigned grid = (unsigned)((rows + fa::kMergeLseWarps - 1) / fa::kMergeLseWarps);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 128) fa::fa_merge_lse_kernel<128><<<grid, 32 * fa::kMergeLseWarps, 0, st>>>(m);
    else fa::fa_merge_lse_kernel<64><<<grid, 32 * fa::kMergeLseWarps, 0, st>>>(m);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
    return ok();
}

int fa_decode_fp8(const void *q, const void *kcache, const void *vcache, const float *k_scale,
                  const float *v_scale, const int *seqlens, void *o, float *lse, int B, int Hq,
                  int Hkv, int Nmax, int d, float scale, void *workspace, size_t workspace_bytes,
                  void *stream)
{
    const CacheDesc c{kcache, vcache, true, k_scale, v_scale, false, nullptr, 0, 0, 0};
    return decode_general(q, c, seqlens, o, lse, B, Hq, Hkv, Nmax, d, scale, workspace, workspace_bytes, stream);
}

int fa_decode_paged_fp8(const void *q, const void *kpages, const void *vpages, const float *k_scale,
                        const float *v_scale, const int *block_table, const int *seqlens, void *o,
                        float *lse, int B, int Hq, int Hkv, int num_pages, int page_size,
                        int max_pages, int d, float scale, void *workspace, size_t workspace_bytes,
                        void *stream)
{
    const CacheDesc c{kpages, vpages, true, k_scale, v_scale, true, block_table, num_pages, page_size, max_pages};
    return decode_general(q, c, seqlens, o, lse, B, Hq, Hkv, 0, d, scale, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------ allocation-free decode
//
// For callers that cannot allocate device memory (see fa_decode_noalloc in fa.h): the
// split-KV partials live in this fixed array instead of a caller workspace.  In host code
// `g_noalloc_scratch` only names a host-side stand-in; its device address is looked up
// with cudaGetSymbolAddress, with the device current, and that address is what the kernels
// get.  The lookup is done on a device's first call and again whenever the device's
// context has changed since (a cudaDeviceReset unloads the module and the array with it).
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

struct NoallocScratch {
    void *ptr = nullptr;
    unsigned long long ctx_id = 0;
};
NoallocScratch g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, in its current context.
int noalloc_scratch(int dev, void **out)
{
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoallocScratch &c = g_noalloc[dev];
    if (!c.ptr || ctx == 0 || ctx != c.ctx_id) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(FA_ERR_CUDA, "cudaGetSymbolAddress of the decode scratch: %s",
                        cudaGetErrorString(e));
        c.ptr = p;
        c.ctx_id = ctx;
    }
    *out = c.ptr;
    return FA_OK;
}

}  // namespace

int fa_decode_noalloc(const void *q, const void *kcache, const void *vcache, const int *seqlens,
                      void *o, float *lse, int B, int Hq, int Hkv, int Nmax, int d, float scale,
                      void *stream)
{
    // the partials must fit the fixed scratch; every other check is fa_decode's
    if (B > 0 && Hq > 0 && Nmax > 0 && d > 0) {
        const size_t need = decode_ws_bytes(B, Hq, Nmax, d);
        if (need > (size_t)FA_NOALLOC_SCRATCH_BYTES)
            return fail(FA_ERR_WORKSPACE,
                        "this decode needs %zu bytes of scratch; fa_decode_noalloc has %u bytes "
                        "(use fa_decode with a workspace for larger problems)",
                        need, (unsigned)FA_NOALLOC_SCRATCH_BYTES);
    }
    if (!q || !kcache || !vcache || !seqlens || !o) return fail(FA_ERR_INVALID, "null pointer argument");
    int dev, rc;
    DeviceInfo *info;
    if ((rc = current_device(&dev, &info)) != FA_OK) return rc;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(dev, &scratch)) != FA_OK) return rc;
    const CacheDesc c{kcache, vcache, false, nullptr, nullptr, false, nullptr, 0, 0, 0};
    return decode_general(q, c, seqlens, o, lse, B, Hq, Hkv, Nmax, d, scale, scratch,
                          (size_t)FA_NOALLOC_SCRATCH_BYTES, stream);
}

int fa_get_error(void *stream)
{
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
    unsigned int word = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&word, fa::g_error_word, sizeof word);
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
    if (word) {
        e = cudaMemcpyToSymbol(fa::g_error_word, &zero, sizeof zero);
        if (e != cudaSuccess) return fail(FA_ERR_CUDA, "clearing the error word: %s", cudaGetErrorString(e));
    }
    if (word & fa::kErrTimeout) return fail(FA_ERR_TIMEOUT, "a kernel pipeline wait exceeded its time limit");
    if (word & fa::kErrSeqlenRange) return fail(FA_ERR_DEVICE_ARG, "seqlens held a value outside [0, Nmax]");
    if (word & fa::kErrPageRange)
        return fail(FA_ERR_DEVICE_ARG, "the block table held a page outside [0, num_pages)");
    if (word & fa::kErrDebugBounds)
        return fail(FA_ERR_DEBUG_CHECK, "a kernel's global-memory index failed its bounds check (access skipped)");
    return ok();
}

void fa_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns = ns ? ns : kDefaultWaitLimitNs; }

const char *fa_status_str(int status)
{
    switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID: return "FA_ERR_INVALID";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_DEVICE_ARG: return "FA_ERR_DEVICE_ARG";
    case FA_ERR_DEBUG_CHECK: return "FA_ERR_DEBUG_CHECK";
    default: return "FA_ERR_UNKNOWN";
    }
}

const char *fa_last_error_message(void) { return g_msg; }

int fa_version(void) { return kVersion; }

int fa_build_flags(void) { return fa::kDebugChecks ? 1 : 0; }

int fa_debug_selftest_bounds(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                             int Hkv, int Nq, int Nk, int d, float scale, int causal, void *stream)
{
    if (!fa::kDebugChecks)
        return fail(FA_ERR_UNSUPPORTED, "bounds checks are compiled only into the debug build (libfa_debug.so)");
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, FA_BF16, false, stream, 0, nullptr,
                    true);
}

}  // extern "C"
