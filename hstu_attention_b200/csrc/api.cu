// api.cu -- the extern "C" entry points declared in include/hstu.h: argument validation,
// workspace accounting, TMA descriptor encoding and kernel dispatch.
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <map>
#include <mutex>
#include <stdint.h>
#include <utility>

#include "common.cuh"
#include "kernels.cuh"

namespace hstu {

__global__ void bucket_table_kernel(int32_t n, double ln_nmax, int32_t nb, const __grid_constant__ BucketBounds bb,
                                    int32_t* out)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n)
        return;
    if (bb.count > 0) {
        // the largest k with v[k] <= i: the same table the tensor-core kernels use
        int lo = 0, hi = bb.count - 1;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (bb.v[mid] <= i)
                lo = mid;
            else
                hi = mid;
        }
        out[i] = lo;
    } else {
        out[i] = bucket_of(i, ln_nmax, nb);
    }
}

// bucket(d) evaluated on the host in double precision (the library's definition).
static int host_bucket(int64_t d, double ln_nmax, int nb)
{
    if (nb <= 1 || d <= 0 || !(ln_nmax > 0.0))
        return 0;
    const double x = (double)(nb - 1) * log((double)d) / ln_nmax;
    const int64_t b = 1 + (int64_t)floor(x);
    return (int)(b > nb - 1 ? nb - 1 : b);
}

// Boundaries of the log-spaced buckets for (n_max, nb), cached per pair (a few hundred bytes).
static BucketBounds host_bounds(int32_t n_max, int32_t nb)
{
    static std::mutex mu;
    static std::map<std::pair<int32_t, int32_t>, BucketBounds> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(n_max, nb);
    auto it = cache.find(key);
    if (it != cache.end())
        return it->second;
    BucketBounds bb{};
    if (nb > kMaxParamNB) {
        bb.count = 0;
    } else {
        const double ln_nmax = log((double)n_max);
        bb.count = nb + 1;
        bb.v[0] = 0;
        for (int k = 1; k < nb; ++k) {
            int64_t c;
            if (nb <= 1 || !(ln_nmax > 0.0)) {
                c = 0x7fffffff;
            } else if (k == 1) {
                c = 1;
            } else {
                c = (int64_t)ceil(exp((double)(k - 1) * ln_nmax / (double)(nb - 1)));
                if (c < 1)
                    c = 1;
                while (c > 1 && host_bucket(c - 1, ln_nmax, nb) >= k)
                    --c;
                while (host_bucket(c, ln_nmax, nb) < k && c < 0x7fffffff)
                    ++c;
            }
            bb.v[k] = (int32_t)(c > 0x7fffffff ? 0x7fffffff : c);
        }
        bb.v[nb] = 0x7fffffff;
    }
    if (cache.size() > 64)
        cache.clear();
    cache[key] = bb;
    return bb;
}

// ------------------------------------------------------------------ helpers

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_params(const hstu_attn_params* p, bool paged)
{
    if (!p)
        return HSTU_ERR_INVALID_ARG;
    if (p->num_heads < 1 || p->num_buckets < 1 || p->num_buckets > 4096 || p->n_max < 1)
        return HSTU_ERR_INVALID_ARG;
    if (!(p->ln_eps >= 0.0f) || !isfinite(p->ln_eps))
        return HSTU_ERR_INVALID_ARG;
    if (p->flags & ~(uint32_t)(HSTU_FLAG_OVERLAP_PREVIOUS | HSTU_FLAG_LN_PER_HEAD))
        return HSTU_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(p->ln_weight) & 3u) || (reinterpret_cast<uintptr_t>(p->ln_bias) & 3u))
        return HSTU_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(p->ts_pages) & 3u)
        return HSTU_ERR_INVALID_ARG;
    if (p->rab_time &&
        (p->num_time_buckets < 1 || p->num_time_buckets > 64 || !p->timestamps ||
         (reinterpret_cast<uintptr_t>(p->rab_time) & 3u) || (reinterpret_cast<uintptr_t>(p->timestamps) & 3u)))
        return HSTU_ERR_INVALID_ARG;
    if (p->dtype != HSTU_DTYPE_BF16 && p->dtype != HSTU_DTYPE_FP32)
        return HSTU_ERR_UNSUPPORTED;
    if (p->head_dim != 32 && p->head_dim != 64 && p->head_dim != 128)
        return HSTU_ERR_UNSUPPORTED;
    if ((int64_t)p->num_heads * p->head_dim > 2048)
        return HSTU_ERR_UNSUPPORTED;
    if (paged) {
        const int P = p->page_size;
        if (P != 8 && P != 16 && P != 32 && P != 64 && P != 128)
            return HSTU_ERR_UNSUPPORTED;
        if (p->num_pages < 1 || p->max_pages_per_user < 1)
            return HSTU_ERR_INVALID_ARG;
        if ((int64_t)p->num_pages * p->num_heads * P >= (int64_t)1 << 31)
            return HSTU_ERR_UNSUPPORTED;     // TMA row coordinates are 32-bit
        if ((int64_t)p->max_pages_per_user * P >= (int64_t)1 << 30)
            return HSTU_ERR_UNSUPPORTED;
    }
    return HSTU_OK;
}

static int esize_of(const hstu_attn_params* p) { return p->dtype == HSTU_DTYPE_FP32 ? 4 : 2; }

static LnVariant ln_variant(const hstu_attn_params* p)
{
    LnVariant v;
    v.per_head = (p->flags & HSTU_FLAG_LN_PER_HEAD) != 0;
    v.D = p->head_dim;
    v.gamma = p->ln_weight;
    v.beta = p->ln_bias;
    return v;
}

// The tensor-core kernel handles bf16, head_dim 128 and up to 1024 buckets (staged in shared memory).
static bool use_tc(const hstu_attn_params* p)
{
    return p->dtype == HSTU_DTYPE_BF16 && p->head_dim == 128 && p->num_buckets <= 1024;
}

// SM count of the current device (cached per device; 148 if the query fails).
static int num_sms()
{
    static std::atomic<int> cached[64];
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 148;
    if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0)
        return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    if (dev >= 0 && dev < 64)
        cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

static size_t partial_bytes(const hstu_attn_params* p, int splits, int64_t tokens)
{
    return (size_t)splits * (size_t)tokens * (size_t)p->num_heads * (size_t)p->head_dim * sizeof(float);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// [rows][H][D] bf16 token rows; box = 64 channels x 1 head x 128 rows, 128B swizzle.
static bool encode_rows(CUtensorMap* m, const void* base, int64_t rows, int32_t H, int32_t D)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [num_pages*H*P][D] bf16 page rows; box = 64 channels x P rows, 128B swizzle.
static bool encode_pages(CUtensorMap* m, const void* base, int64_t rows, int32_t D, int32_t P)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)P};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int finish(cudaStream_t)
{
    return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

static constexpr uint64_t kTimeoutNs = 2000000000ull;   // 2 s per in-kernel wait

// Test-only fault injection (hstu_test_inject): an injected kind and the role-wait limit the
// tensor-core kernels then use; the waits for a CTA's own copies and products keep 2 s.
static std::atomic<uint32_t> g_inject_kind{0};
static std::atomic<uint64_t> g_inject_limit_ns{0};

static void set_waits(TcArgs& a)
{
    const uint32_t kind = g_inject_kind.load(std::memory_order_relaxed);
    a.inject = kind;
    a.timeout_ns = kind ? g_inject_limit_ns.load(std::memory_order_relaxed) : kTimeoutNs;
    a.drain_ns = kTimeoutNs;
}

// Scratch of hstu_attn_paged_fwd_noalloc: a fixed array in the library's own device image, so
// that callers which cannot hand over a workspace still get a paged forward.  Layout is the
// workspace layout (status block, split counts, fp32 partial planes).  Every call on a device
// shares it.
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;   // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;

// The array's address is looked up once per (device, CUDA context): after a device reset, or
// under another context, the library's module is loaded again and the address changes.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}

struct NoAllocEntry {
    CUcontext ctx;
    void* ptr;
};
static std::mutex g_noalloc_mu;
static NoAllocEntry g_noalloc[kNoAllocMaxDevices];

// Device address of g_noalloc_scratch for the current device and context.
static int noalloc_scratch(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return HSTU_ERR_CUDA;
    CtxGetCurrentFn fn = ctx_get_current();
    CUcontext ctx = nullptr;
    if (fn)
        fn(&ctx);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (dev >= 0 && dev < kNoAllocMaxDevices && ctx && g_noalloc[dev].ptr && g_noalloc[dev].ctx == ctx) {
        *out = g_noalloc[dev].ptr;
        return HSTU_OK;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
        return HSTU_ERR_CUDA;
    if (fn)
        fn(&ctx);                                  // the lookup may have created the context
    if (dev >= 0 && dev < kNoAllocMaxDevices && ctx)
        g_noalloc[dev] = NoAllocEntry{ctx, p};
    *out = p;
    return HSTU_OK;
}

}  // namespace hstu

using namespace hstu;

extern "C" {

const char* hstu_version(void) { return "hstu_b200 0.1 (sm_100a)"; }

const char* hstu_error_string(int code)
{
    switch (code) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID_ARG: return "invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case HSTU_ERR_WORKSPACE: return "workspace too small or misaligned";
    case HSTU_ERR_CUDA: return "CUDA error";
    case HSTU_ERR_SCRATCH_LIMIT:
        return "request needs more than the 8 MiB built-in scratch of hstu_attn_paged_fwd_noalloc";
    case HSTU_ERR_CACHE_FULL:
        return "the batch does not fit in the GPU tier of the KV cache even with every other user evicted";
    case HSTU_ERR_OUTPUT_CAPACITY: return "an output array of a cache call is too small";
    default: return "unknown error";
    }
}

size_t hstu_workspace_size(const hstu_attn_params* params, int32_t max_batch, int64_t max_tokens, int32_t max_new)
{
    if (check_params(params, false) != HSTU_OK || max_batch < 0 || max_tokens < 0 || max_new < 0)
        return 0;
    // the tensor-core paged path spreads a user's keys over up to kMaxSplits CTAs, each with
    // its own fp32 partial plane; every other path writes one plane
    const int planes = use_tc(params) ? kMaxSplits : 1;
    size_t bytes = kStatusBytes + counts_bytes(max_tokens) + partial_bytes(params, planes, max_tokens);
    return (bytes + 255) & ~(size_t)255;
}

int hstu_workspace_init(void* workspace, size_t workspace_bytes, void* stream)
{
    if (!workspace || workspace_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (cudaMemsetAsync(workspace, 0, kStatusBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return HSTU_ERR_CUDA;
    return HSTU_OK;
}

int hstu_read_status(void* workspace, void* stream, uint32_t* flags_out, int clear)
{
    if (!workspace || !flags_out)
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
        return HSTU_ERR_CUDA;
    *flags_out = v;
    if (clear && cudaMemset(workspace, 0, sizeof v) != cudaSuccess)
        return HSTU_ERR_CUDA;
    return HSTU_OK;
}

int hstu_bucket_table(const hstu_attn_params* params, int32_t n, int32_t* table_out, void* stream)
{
    if (check_params(params, false) != HSTU_OK || n < 0 || (n > 0 && !table_out))
        return HSTU_ERR_INVALID_ARG;
    if (n == 0)
        return HSTU_OK;
    const double ln_nmax = log((double)params->n_max);
    const BucketBounds bb = host_bounds(params->n_max, params->num_buckets);
    bucket_table_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        n, ln_nmax, params->num_buckets, bb, table_out);
    return finish(static_cast<cudaStream_t>(stream));
}

int hstu_kv_append(const hstu_attn_params* params, void* k_pages, void* v_pages, const int32_t* page_table,
                   const void* k_new, const void* v_new, const int32_t* cached_lens, const int32_t* new_lens,
                   const int32_t* num_targets, int32_t B, int64_t total_new, int32_t max_new, void* workspace,
                   size_t workspace_bytes, void* stream)
{
    int rc = check_params(params, true);
    if (rc != HSTU_OK)
        return rc;
    if (B < 0 || max_new < 0 || total_new < 0)
        return HSTU_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (B == 0 || max_new == 0 || total_new == 0)
        return HSTU_OK;
    if (!k_pages || !v_pages || !page_table || !k_new || !v_new || !cached_lens || !new_lens)
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(k_pages) || !aligned16(v_pages) || !aligned16(k_new) || !aligned16(v_new))
        return HSTU_ERR_INVALID_ARG;
    launch_kv_append(k_pages, v_pages, page_table, k_new, v_new, cached_lens, new_lens, num_targets, B, total_new,
                     params->num_heads, params->head_dim, esize_of(params), params->page_size, params->num_pages,
                     params->max_pages_per_user, max_new, workspace,
                     params->ts_pages && params->timestamps ? params->ts_pages : nullptr, params->timestamps,
                     static_cast<cudaStream_t>(stream));
    return finish(static_cast<cudaStream_t>(stream));
}

// `bytes` bytes from p are addressable by the current device: device memory of this device,
// managed memory, or pinned host memory mapped into the device's address space.  Both ends are
// checked and must belong to one mapping; *dev_out receives the device address of p.
static bool device_addressable(const void* p, size_t bytes, const void** dev_out)
{
    int dev = -1;
    if (!p || bytes == 0 || cudaGetDevice(&dev) != cudaSuccess)
        return false;
    const char* ends[2] = {static_cast<const char*>(p), static_cast<const char*>(p) + (bytes - 1)};
    const char* base = nullptr;
    for (int e = 0; e < 2; ++e) {
        cudaPointerAttributes a{};
        if (cudaPointerGetAttributes(&a, ends[e]) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        if (a.type == cudaMemoryTypeDevice) {
            if (a.device != dev)
                return false;
        } else if (a.type != cudaMemoryTypeHost && a.type != cudaMemoryTypeManaged) {
            return false;
        }
        const char* dp = static_cast<const char*>(a.devicePointer);
        if (!dp)
            return false;
        if (e == 0)
            base = dp;
        else if (dp != base + (bytes - 1))
            return false;
    }
    *dev_out = base;
    return true;
}

int hstu_kv_page_copy(const hstu_attn_params* params, const void* src_k, const void* src_v, int32_t src_pages,
                      void* dst_k, void* dst_v, int32_t dst_pages, const int32_t* pairs, int32_t n_pairs,
                      void* workspace, size_t workspace_bytes, void* stream)
{
    int rc = check_params(params, true);
    if (rc != HSTU_OK)
        return rc;
    if (n_pairs < 0 || src_pages < 0 || dst_pages < 0)
        return HSTU_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (n_pairs == 0)
        return HSTU_OK;
    if (!src_k || !src_v || !dst_k || !dst_v || !pairs || src_pages == 0 || dst_pages == 0)
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v))
        return HSTU_ERR_INVALID_ARG;
    const int64_t page_bytes =
        (int64_t)params->num_heads * params->page_size * params->head_dim * esize_of(params);
    const void *sk, *sv, *dk, *dv, *pr;
    if (!device_addressable(src_k, (size_t)(page_bytes * src_pages), &sk) ||
        !device_addressable(src_v, (size_t)(page_bytes * src_pages), &sv) ||
        !device_addressable(dst_k, (size_t)(page_bytes * dst_pages), &dk) ||
        !device_addressable(dst_v, (size_t)(page_bytes * dst_pages), &dv) ||
        !device_addressable(pairs, (size_t)n_pairs * 8, &pr))
        return HSTU_ERR_INVALID_ARG;
    launch_kv_page_copy(sk, sv, const_cast<void*>(dk), const_cast<void*>(dv), static_cast<const int32_t*>(pr),
                        n_pairs, src_pages, dst_pages, page_bytes, workspace, static_cast<cudaStream_t>(stream));
    return finish(static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ projections and the layer

// [rows][K] bf16 operand of the projection GEMM: box = 64 columns x 128 rows, 128B swizzle.
static bool encode_operand(CUtensorMap* m, const void* base, int64_t rows, int32_t K)
{
    return encode_pages(m, base, rows, K, 128);
}

static int linear(const void* x, const void* w, __nv_bfloat16* out, int64_t M, int32_t N, int32_t K, int32_t silu,
                  int32_t split, int64_t block_stride, void* ws, cudaStream_t s, bool pdl = false)
{
    CUtensorMap ta, tb;
    if (!encode_operand(&ta, x, M, K) || !encode_operand(&tb, w, N, K))
        return HSTU_ERR_CUDA;
    GemmArgs g{};
    g.M = (int32_t)M;
    g.N = N;
    g.K = K;
    g.split = split;
    g.block_stride = block_stride;
    g.ldo = split;
    g.out = out;
    g.silu = silu;
    g.ws = ws;
    g.timeout_ns = kTimeoutNs;
    g.drain_ns = kTimeoutNs;
    g.pdl = pdl ? 1 : 0;
    launch_gemm_bf16(ta, tb, g, s);
    return HSTU_OK;
}

int hstu_linear_fwd(const void* x, const void* w, void* y, int64_t M, int32_t N, int32_t K, int32_t activation,
                    void* workspace, size_t workspace_bytes, void* stream)
{
    if (M < 0 || M >= ((int64_t)1 << 31) || N <= 0 || K <= 0 || N % 128 || K % 64 || (activation != 0 && activation != 1))
        return HSTU_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (M == 0)
        return HSTU_OK;
    if (!x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y))
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int rc = linear(x, w, static_cast<__nv_bfloat16*>(y), M, N, K, activation, N, 0, workspace, s);
    return rc != HSTU_OK ? rc : finish(s);
}

static bool layer_shape_ok(const hstu_attn_params* p, int32_t d_model)
{
    return use_tc(p) && d_model > 0 && d_model % 128 == 0 && ((int64_t)p->num_heads * p->head_dim) % 128 == 0;
}

size_t hstu_workspace_size_layer(const hstu_attn_params* params, int32_t d_model, int32_t max_batch,
                                 int64_t max_tokens, int32_t max_new)
{
    if (check_params(params, false) != HSTU_OK || !layer_shape_ok(params, d_model) || max_tokens < 0)
        return 0;
    const size_t attn = hstu_workspace_size(params, max_batch, max_tokens, max_new);
    if (attn == 0)
        return 0;
    const size_t HD = (size_t)params->num_heads * params->head_dim;
    const size_t act = (5 * (size_t)max_tokens * HD * 2 + 255) & ~(size_t)255;   // q, k, v, u, gated
    return attn + act;
}

int hstu_layer_paged_fwd(const hstu_attn_params* params, int32_t d_model, const void* x_new, const void* w_qkvu,
                         const void* w_out, void* k_pages, void* v_pages, const int32_t* page_table,
                         const int32_t* cached_lens, const int32_t* new_lens, const int32_t* num_targets,
                         const float* rab, void* y, int32_t B, int64_t total_new, int32_t max_new, void* workspace,
                         size_t workspace_bytes, void* stream)
{
    int rc = check_params(params, true);
    if (rc != HSTU_OK)
        return rc;
    if (params->rab_time)
        return HSTU_ERR_UNSUPPORTED;   // the time bias exists in the jagged forward only
    if (!layer_shape_ok(params, d_model))
        return HSTU_ERR_UNSUPPORTED;
    if (B < 0 || total_new < 0 || max_new < 0 || total_new >= ((int64_t)1 << 31))
        return HSTU_ERR_INVALID_ARG;
    const size_t need = hstu_workspace_size_layer(params, d_model, B, total_new, max_new);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (B == 0 || total_new == 0)
        return HSTU_OK;
    if (!x_new || !w_qkvu || !w_out || !y || !aligned16(x_new) || !aligned16(w_qkvu) || !aligned16(w_out) ||
        !aligned16(y))
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t HD = (int64_t)params->num_heads * params->head_dim;
    const size_t attn = hstu_workspace_size(params, B, total_new, max_new);
    __nv_bfloat16* act = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(workspace) + attn);
    __nv_bfloat16* q = act;
    __nv_bfloat16* k = q + total_new * HD;
    __nv_bfloat16* v = k + total_new * HD;
    __nv_bfloat16* u = v + total_new * HD;
    __nv_bfloat16* gated = u + total_new * HD;
    // q, k, v, u = SiLU(x W_qkvu^T), one H*D-column block each
    const bool overlap = (params->flags & HSTU_FLAG_OVERLAP_PREVIOUS) != 0;
    rc = linear(x_new, w_qkvu, q, total_new, (int32_t)(4 * HD), d_model, 1, (int32_t)HD, total_new * HD, workspace, s,
                overlap);
    if (rc != HSTU_OK)
        return rc;
    // the new history tokens' K and V into the user's pages; the attention reads the new keys
    // from k and v directly, so it does not depend on the append
    rc = hstu_kv_append(params, k_pages, v_pages, page_table, k, v, cached_lens, new_lens, num_targets, B, total_new,
                        max_new, workspace, attn, stream);
    if (rc != HSTU_OK)
        return rc;
    // the attention's set-up may overlap the append: before its dependency wait it reads only
    // the length arrays, the page table and rab, which the append does not write
    hstu_attn_params pa = *params;
    pa.flags |= HSTU_FLAG_OVERLAP_PREVIOUS;
    rc = hstu_attn_paged_fwd(&pa, q, k, v, u, k_pages, v_pages, page_table, cached_lens, new_lens, num_targets, rab,
                             gated, B, total_new, max_new, workspace, attn, stream);
    if (rc != HSTU_OK)
        return rc;
    // y = gated W_out^T
    // the output projection's set-up overlaps the LayerNorm kernel (it waits before reading gated)
    rc = linear(gated, w_out, static_cast<__nv_bfloat16*>(y), total_new, d_model, (int32_t)HD, 0, d_model, 0,
                workspace, s, true);
    return rc != HSTU_OK ? rc : finish(s);
}

int hstu_test_inject(uint32_t kind, uint64_t wait_limit_ns)
{
    if (kind & ~(uint32_t)HSTU_INJECT_STALL_V)
        return HSTU_ERR_INVALID_ARG;
    if (kind && (wait_limit_ns < 1000000ull || wait_limit_ns > kTimeoutNs))
        return HSTU_ERR_INVALID_ARG;
    g_inject_limit_ns.store(wait_limit_ns, std::memory_order_relaxed);
    g_inject_kind.store(kind == HSTU_INJECT_STALL_V ? kInjectStallV : 0u, std::memory_order_relaxed);
    return HSTU_OK;
}

int hstu_ts_page_copy(const int32_t* src, int32_t src_pages, int32_t* dst, int32_t dst_pages, int32_t page_size,
                      const int32_t* pairs, int32_t n_pairs, void* workspace, size_t workspace_bytes, void* stream)
{
    if (n_pairs < 0 || src_pages < 0 || dst_pages < 0 || page_size < 4 || page_size % 4)
        return HSTU_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (n_pairs == 0)
        return HSTU_OK;
    if (!src || !dst || !pairs || src_pages == 0 || dst_pages == 0 || !aligned16(src) || !aligned16(dst))
        return HSTU_ERR_INVALID_ARG;
    const int64_t page_bytes = (int64_t)page_size * 4;
    const void *sp, *dp, *pr;
    if (!device_addressable(src, (size_t)(page_bytes * src_pages), &sp) ||
        !device_addressable(dst, (size_t)(page_bytes * dst_pages), &dp) ||
        !device_addressable(pairs, (size_t)n_pairs * 8, &pr))
        return HSTU_ERR_INVALID_ARG;
    launch_kv_page_copy(sp, nullptr, const_cast<void*>(dp), nullptr, static_cast<const int32_t*>(pr), n_pairs,
                        src_pages, dst_pages, page_bytes, workspace, static_cast<cudaStream_t>(stream));
    return finish(static_cast<cudaStream_t>(stream));
}

int hstu_host_copy(void* dst, const void* src, size_t bytes, void* stream)
{
    if (bytes == 0)
        return HSTU_OK;
    if (!dst || !src || !aligned16(dst) || !aligned16(src))
        return HSTU_ERR_INVALID_ARG;
    const void *d, *s;
    if (!device_addressable(dst, bytes, &d) || !device_addressable(src, bytes, &s))
        return HSTU_ERR_INVALID_ARG;
    const char* dc = static_cast<const char*>(d);
    const char* sc = static_cast<const char*>(s);
    if (dc < sc + bytes && sc < dc + bytes)
        return HSTU_ERR_INVALID_ARG;    // overlapping ranges
    launch_flat_copy(const_cast<void*>(d), s, (int64_t)bytes, static_cast<cudaStream_t>(stream));
    return finish(static_cast<cudaStream_t>(stream));
}

// The attention part of the jagged forward: O / n_max of every query row into the fp32 plane
// `part` ([tokens][H][D]); device-detected errors go to the workspace status word.
static int jagged_attention(const hstu_attn_params* params, const void* q, const void* k, const void* v,
                            const int32_t* seq_offsets, const int32_t* num_targets, const float* rab, int32_t B,
                            int64_t total_tokens, int32_t max_seqlen, void* workspace, float* part, cudaStream_t s)
{
    const double ln_nmax = log((double)params->n_max);
    const bool fp32 = params->dtype == HSTU_DTYPE_FP32;
    if (use_tc(params)) {
        TcMaps m;
        if (!encode_rows(&m.q, q, total_tokens, params->num_heads, 128) ||
            !encode_rows(&m.k, k, total_tokens, params->num_heads, 128) ||
            !encode_rows(&m.v, v, total_tokens, params->num_heads, 128))
            return HSTU_ERR_CUDA;
        m.kp = m.k;
        m.vp = m.v;
        TcArgs a{};
        a.seq_offsets = seq_offsets;
        a.num_targets = num_targets;
        a.rab = rab;
        a.ws = workspace;
        a.part = part;
        a.counts = nullptr;
        a.total_tokens = total_tokens;
        a.max_len = max_seqlen;
        a.H = params->num_heads;
        a.NB = params->num_buckets;
        a.n_max = params->n_max;
        a.P = 1;
        a.num_pages = 0;
        a.max_pages = 0;
        a.B = B;
        a.max_splits = 1;
        a.target_ctas = num_sms();
        a.qblocks = (max_seqlen + 127) / 128;
        a.ln_nmax = ln_nmax;
        a.inv_n = (float)(1.0 / (double)params->n_max);
        a.overlap_previous = (params->flags & HSTU_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
        a.rab_time = params->rab_time;
        a.ts = params->timestamps;
        a.NBT = params->num_time_buckets;
        set_waits(a);
        launch_attn_tc(m, a, host_bounds(params->n_max, params->num_buckets), B, s);
    } else {
        SimtArgs a{};
        a.q = q;
        a.k = k;
        a.v = v;
        a.seq_offsets = seq_offsets;
        a.num_targets = num_targets;
        a.rab = rab;
        a.ws = workspace;
        a.part = part;
        a.total_tokens = total_tokens;
        a.max_len = max_seqlen;
        a.H = params->num_heads;
        a.D = params->head_dim;
        a.NB = params->num_buckets;
        a.n_max = params->n_max;
        a.P = 1;
        a.ln_nmax = ln_nmax;
        launch_attn_simt(a, false, fp32, B, s);
    }
    return HSTU_OK;
}

int hstu_attn_jagged_fwd(const hstu_attn_params* params, const void* q, const void* k, const void* v, const void* u,
                         const int32_t* seq_offsets, const int32_t* num_targets, const float* rab, void* out,
                         int32_t B, int64_t total_tokens, int32_t max_seqlen, void* workspace,
                         size_t workspace_bytes, void* stream)
{
    int rc = check_params(params, false);
    if (rc != HSTU_OK)
        return rc;
    if (params->rab_time && !use_tc(params))
        return HSTU_ERR_UNSUPPORTED;   // the time bias exists on the tensor-core path only
    if (B < 0 || total_tokens < 0 || max_seqlen < 0 || total_tokens >= ((int64_t)1 << 31))
        return HSTU_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (B == 0 || total_tokens == 0 || max_seqlen == 0)
        return HSTU_OK;
    if (!q || !k || !v || !u || !out || !seq_offsets || !rab)
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(u) || !aligned16(out))
        return HSTU_ERR_INVALID_ARG;
    if (workspace_bytes < kStatusBytes + counts_bytes(total_tokens) + partial_bytes(params, 1, total_tokens))
        return HSTU_ERR_WORKSPACE;
    float* part = partials(workspace, total_tokens);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool fp32 = params->dtype == HSTU_DTYPE_FP32;
    rc = jagged_attention(params, q, k, v, seq_offsets, num_targets, rab, B, total_tokens, max_seqlen, workspace, part,
                          s);
    if (rc != HSTU_OK)
        return rc;
    launch_ln_gate(part, 1, nullptr, total_tokens, params->num_heads * params->head_dim, u, out, fp32, params->ln_eps,
                   ln_variant(params), s);
    return finish(s);
}

static size_t bwd_bf16_bytes(const hstu_attn_params* p, int64_t tokens)
{
    return ((size_t)tokens * p->num_heads * p->head_dim * 2 + 255) & ~(size_t)255;
}

size_t hstu_workspace_size_bwd(const hstu_attn_params* params, int64_t max_tokens)
{
    if (check_params(params, false) != HSTU_OK || max_tokens < 0)
        return 0;
    // o and its gradient (fp32), then the gradient in bf16 for the tensor-core kernels
    const size_t bytes = kStatusBytes + 2 * partial_bytes(params, 1, max_tokens) + bwd_bf16_bytes(params, max_tokens);
    return (bytes + 255) & ~(size_t)255;
}

int hstu_attn_jagged_bwd(const hstu_attn_params* params, const void* q, const void* k, const void* v, const void* u,
                         const int32_t* seq_offsets, const int32_t* num_targets, const float* rab, const void* dout,
                         float* dq, float* dk, float* dv, float* du, float* drab, int32_t B, int64_t total_tokens,
                         int32_t max_seqlen, void* workspace, size_t workspace_bytes, void* stream)
{
    int rc = check_params(params, false);
    if (rc != HSTU_OK)
        return rc;
    if ((params->flags & HSTU_FLAG_LN_PER_HEAD) || params->ln_weight || params->ln_bias || params->rab_time)
        return HSTU_ERR_UNSUPPORTED;   // the backward pass implements the base epilogue and bias only
    if (B < 0 || total_tokens < 0 || max_seqlen < 0 || total_tokens >= ((int64_t)1 << 31))
        return HSTU_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (!drab)
        return HSTU_ERR_INVALID_ARG;
    const bool empty = B == 0 || total_tokens == 0 || max_seqlen == 0;
    if (!empty) {
        // every host-detectable error is reported before anything is enqueued
        if (!q || !k || !v || !u || !dout || !dq || !dk || !dv || !du || !seq_offsets || !rab)
            return HSTU_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(u) || !aligned16(dout) || !aligned16(dq) ||
            !aligned16(dk) || !aligned16(dv) || !aligned16(du))
            return HSTU_ERR_INVALID_ARG;
        if (workspace_bytes < kStatusBytes + 2 * partial_bytes(params, 1, total_tokens) +
                                  bwd_bf16_bytes(params, total_tokens))
            return HSTU_ERR_WORKSPACE;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // drab accumulates over pairs: it starts from zero (also for an empty batch)
    if (cudaMemsetAsync(drab, 0, sizeof(float) * (size_t)params->num_heads * params->num_buckets, s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    if (empty)
        return finish(s);
    float* o = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
    const int64_t HD = (int64_t)params->num_heads * params->head_dim;
    rc = jagged_attention(params, q, k, v, seq_offsets, num_targets, rab, B, total_tokens, max_seqlen, workspace, o, s);
    if (rc != HSTU_OK)
        return rc;
    BwdArgs a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.seq_offsets = seq_offsets;
    a.num_targets = num_targets;
    a.rab = rab;
    a.dO = o + total_tokens * HD;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.drab = drab;
    a.total_tokens = total_tokens;
    a.B = B;
    a.H = params->num_heads;
    a.D = params->head_dim;
    a.NB = params->num_buckets;
    a.n_max = params->n_max;
    a.max_seqlen = max_seqlen;
    a.ln_nmax = log((double)params->n_max);
    a.inv_n = (float)(1.0 / (double)params->n_max);
    if (!use_tc(params)) {
        launch_jagged_bwd(a, o, u, dout, du, params->ln_eps, params->dtype == HSTU_DTYPE_FP32, s);
        return finish(s);
    }
    // tensor-core path: the LayerNorm-gate backward also leaves do in bf16, then dq/drab and dk/dv
    __nv_bfloat16* dO16 = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<char*>(o) + 2 * partial_bytes(params, 1,
                                                                                                        total_tokens));
    BwdTcMaps m;
    if (!encode_rows(&m.q, q, total_tokens, params->num_heads, 128) ||
        !encode_rows(&m.k, k, total_tokens, params->num_heads, 128) ||
        !encode_rows(&m.v, v, total_tokens, params->num_heads, 128) ||
        !encode_rows(&m.dO, dO16, total_tokens, params->num_heads, 128))
        return HSTU_ERR_CUDA;
    BwdArgs a16 = a;
    a16.dO = nullptr;                    // the tensor-core kernels read the bf16 copy only
    launch_ln_gate_bwd(a16, o, u, dout, du, dO16, params->ln_eps, false, s);
    BwdTcArgs t{};
    t.seq_offsets = seq_offsets;
    t.num_targets = num_targets;
    t.rab = rab;
    t.ws = workspace;
    t.dq = dq;
    t.dk = dk;
    t.dv = dv;
    t.drab = drab;
    t.total_tokens = total_tokens;
    t.max_len = max_seqlen;
    t.H = params->num_heads;
    t.NB = params->num_buckets;
    t.n_max = params->n_max;
    t.B = B;
    t.qblocks = (max_seqlen + 127) / 128;
    t.ln_nmax = a.ln_nmax;
    t.inv_n = a.inv_n;
    t.timeout_ns = kTimeoutNs;
    t.drain_ns = kTimeoutNs;
    if (t.qblocks > 65535 || (int64_t)t.H * B >= ((int64_t)1 << 31))
        return HSTU_ERR_UNSUPPORTED;
    launch_bwd_tc(m, t, host_bounds(params->n_max, params->num_buckets), s);
    return finish(s);
}

int hstu_attn_paged_fwd(const hstu_attn_params* params, const void* q_new, const void* k_new, const void* v_new,
                        const void* u_new, const void* k_pages, const void* v_pages, const int32_t* page_table,
                        const int32_t* cached_lens, const int32_t* new_lens, const int32_t* num_targets,
                        const float* rab, void* out, int32_t B, int64_t total_new, int32_t max_new, void* workspace,
                        size_t workspace_bytes, void* stream)
{
    int rc = check_params(params, true);
    if (rc != HSTU_OK)
        return rc;
    if (params->rab_time && (!use_tc(params) || !params->ts_pages))
        return HSTU_ERR_UNSUPPORTED;   // the time bias: tensor-core path, cached timestamps in ts_pages
    if (B < 0 || total_new < 0 || max_new < 0 || total_new >= ((int64_t)1 << 31))
        return HSTU_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return HSTU_ERR_WORKSPACE;
    if (B == 0 || total_new == 0 || max_new == 0)
        return HSTU_OK;
    if (!q_new || !k_new || !v_new || !u_new || !k_pages || !v_pages || !page_table || !cached_lens || !new_lens ||
        !rab || !out)
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q_new) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(u_new) || !aligned16(k_pages) ||
        !aligned16(v_pages) || !aligned16(out))
        return HSTU_ERR_INVALID_ARG;
    if (use_tc(params) && B > paged_max_users())
        return HSTU_ERR_UNSUPPORTED;
    const size_t one = partial_bytes(params, 1, total_new);
    const size_t fixed = kStatusBytes + counts_bytes(total_new);
    if (workspace_bytes < fixed + one)
        return HSTU_ERR_WORKSPACE;
    float* part = partials(workspace, total_new);
    int32_t* counts = split_counts(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const double ln_nmax = log((double)params->n_max);
    const bool fp32 = params->dtype == HSTU_DTYPE_FP32;
    int splits = 1;
    if (use_tc(params)) {
        // as many partial planes as the workspace holds, up to kMaxSplits
        splits = (int)((workspace_bytes - fixed) / one);
        if (splits > kMaxSplits)
            splits = kMaxSplits;
        TcMaps m;
        const int64_t page_rows = (int64_t)params->num_pages * params->num_heads * params->page_size;
        if (!encode_rows(&m.q, q_new, total_new, params->num_heads, 128) ||
            !encode_rows(&m.k, k_new, total_new, params->num_heads, 128) ||
            !encode_rows(&m.v, v_new, total_new, params->num_heads, 128) ||
            !encode_pages(&m.kp, k_pages, page_rows, 128, params->page_size) ||
            !encode_pages(&m.vp, v_pages, page_rows, 128, params->page_size))
            return HSTU_ERR_CUDA;
        TcArgs a{};
        a.cached_lens = cached_lens;
        a.new_lens = new_lens;
        a.num_targets = num_targets;
        a.page_table = page_table;
        a.rab = rab;
        a.ws = workspace;
        a.part = part;
        a.counts = counts;
        a.total_tokens = total_new;
        a.max_len = max_new;
        a.H = params->num_heads;
        a.NB = params->num_buckets;
        a.n_max = params->n_max;
        a.P = params->page_size;
        a.num_pages = params->num_pages;
        a.max_pages = params->max_pages_per_user;
        a.B = B;
        a.max_splits = splits;
        a.target_ctas = num_sms();
        a.qblocks = (max_new + 127) / 128;
        a.ln_nmax = ln_nmax;
        a.inv_n = (float)(1.0 / (double)params->n_max);
        a.overlap_previous = (params->flags & HSTU_FLAG_OVERLAP_PREVIOUS) ? 1 : 0;
        a.rab_time = params->rab_time;
        a.ts = params->timestamps;
        a.ts_pages = params->ts_pages;
        a.NBT = params->num_time_buckets;
        set_waits(a);
        launch_attn_paged(m, a, host_bounds(params->n_max, params->num_buckets), num_sms(), s);
    } else {
        SimtArgs a{};
        a.q = q_new;
        a.k = k_new;
        a.v = v_new;
        a.k_pages = k_pages;
        a.v_pages = v_pages;
        a.page_table = page_table;
        a.cached_lens = cached_lens;
        a.new_lens = new_lens;
        a.num_targets = num_targets;
        a.rab = rab;
        a.ws = workspace;
        a.part = part;
        a.total_tokens = total_new;
        a.max_len = max_new;
        a.H = params->num_heads;
        a.D = params->head_dim;
        a.NB = params->num_buckets;
        a.n_max = params->n_max;
        a.P = params->page_size;
        a.num_pages = params->num_pages;
        a.max_pages = params->max_pages_per_user;
        a.ln_nmax = ln_nmax;
        launch_attn_simt(a, true, fp32, B, s);
    }
    launch_ln_gate(part, splits, use_tc(params) ? counts : nullptr, total_new, params->num_heads * params->head_dim,
                   u_new, out, fp32, params->ln_eps, ln_variant(params), s);
    return finish(s);
}


int hstu_attn_paged_fwd_noalloc(const hstu_attn_params* params, const void* q_new, const void* k_new,
                                const void* v_new, const void* u_new, const void* k_pages, const void* v_pages,
                                const int32_t* page_table, const int32_t* cached_lens, const int32_t* new_lens,
                                const int32_t* num_targets, const float* rab, void* out, int32_t B,
                                int64_t total_new, int32_t max_new, uint32_t* flags_out, void* stream)
{
    int rc = check_params(params, true);
    if (rc != HSTU_OK)
        return rc;
    if (params->rab_time && (!use_tc(params) || !params->ts_pages))
        return HSTU_ERR_UNSUPPORTED;   // the time bias: tensor-core path, cached timestamps in ts_pages
    if (B < 0 || total_new < 0 || max_new < 0 || total_new >= ((int64_t)1 << 31))
        return HSTU_ERR_INVALID_ARG;
    if (flags_out && (reinterpret_cast<uintptr_t>(flags_out) & 3u))
        return HSTU_ERR_INVALID_ARG;
    // the status block, the split counts and at least one partial plane must fit; more room
    // only buys more key splits
    const size_t need = kStatusBytes + counts_bytes(total_new) + partial_bytes(params, 1, total_new);
    if (need > kNoAllocScratchBytes)
        return HSTU_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != HSTU_OK)
        return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the status word is the only part that must start at zero: cleared for every call
    if (cudaMemsetAsync(scratch, 0, kStatusBytes, s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    rc = hstu_attn_paged_fwd(params, q_new, k_new, v_new, u_new, k_pages, v_pages, page_table, cached_lens,
                             new_lens, num_targets, rab, out, B, total_new, max_new, scratch, kNoAllocScratchBytes,
                             stream);
    if (rc != HSTU_OK)
        return rc;
    if (flags_out &&
        cudaMemcpyAsync(flags_out, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    return HSTU_OK;
}

}  // extern "C"
