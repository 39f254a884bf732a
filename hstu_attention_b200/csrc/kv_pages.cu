// kv_pages.cu -- whole-page copies between KV pools: the onboard (pinned host pool -> GPU pool),
// offload (GPU pool -> pinned host pool) and compaction (within the GPU pool) moves of the
// two-tier KV cache (NVIDIA blog "Deploying an HSTU Generative Recommender with NVIDIA
// Dynamo-Triton", section "Why serving large sequential recommenders is hard": a host tier
// beside the paged GPU table, with onboard and offload operations).
//
// A page is H * P * D elements, the same contiguous block in both pools, so a copy is a
// gather/scatter of fixed-size blocks by page id.  Grid (chunks of a page, pairs, {K, V}); a
// thread moves kUnroll 16-byte vectors and issues all its loads before its stores, so each
// block keeps 16 KB of reads in flight.  That covers HBM latency for the in-pool copy and the
// much longer latency of reads from pinned host memory over the host link (the SMs address the
// host pool directly; no staging buffer and no per-page copy call).
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads)
kv_page_copy_kernel(const uint4* __restrict__ src_k, const uint4* __restrict__ src_v, uint4* __restrict__ dst_k,
                    uint4* __restrict__ dst_v, const int32_t* __restrict__ pairs, int32_t n_pairs, int32_t src_pages,
                    int32_t dst_pages, int64_t page_vecs, void* ws)
{
    const uint4* src = blockIdx.z ? src_v : src_k;
    uint4* dst = blockIdx.z ? dst_v : dst_k;
    const int64_t first = (int64_t)blockIdx.x * (kCopyThreads * kCopyUnroll) + threadIdx.x;
    for (int64_t i = blockIdx.y; i < n_pairs; i += gridDim.y) {
        const int32_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= src_pages || d < 0 || d >= dst_pages) {
            if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0)
                set_flag(ws, HSTU_DEV_BAD_PAGE);
            continue;
        }
        const uint4* sp = src + (int64_t)s * page_vecs;
        uint4* dp = dst + (int64_t)d * page_vecs;
        uint4 r[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t x = first + u * kCopyThreads;
            if (x < page_vecs)
                r[u] = sp[x];
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t x = first + u * kCopyThreads;
            if (x < page_vecs)
                dp[x] = r[u];
        }
    }
}

void launch_kv_page_copy(const void* src_k, const void* src_v, void* dst_k, void* dst_v, const int32_t* pairs,
                         int32_t n_pairs, int32_t src_pages, int32_t dst_pages, int64_t page_bytes, void* ws,
                         cudaStream_t stream)
{
    if (n_pairs <= 0)
        return;
    const int64_t page_vecs = page_bytes / 16;
    const int64_t per_block = (int64_t)kCopyThreads * kCopyUnroll;
    // z = the pools copied: K and V, or one pool when src_v is null (the timestamp pages)
    dim3 grid((unsigned)((page_vecs + per_block - 1) / per_block), (unsigned)(n_pairs < 65535 ? n_pairs : 65535),
              src_v ? 2 : 1);
    kv_page_copy_kernel<<<grid, kCopyThreads, 0, stream>>>(
        static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v), static_cast<uint4*>(dst_k),
        static_cast<uint4*>(dst_v), pairs, n_pairs, src_pages, dst_pages, page_vecs, ws);
}

}  // namespace hstu

namespace hstu {

// A flat copy of `nvec` 16-byte vectors plus a `tail` of fewer than 16 bytes, between any two
// buffers the device addresses (device memory, or pinned host memory read or written over the
// host link).  Blocks stride over the buffer; a thread keeps kFlatUnroll vectors in flight, so a
// block has 16 KB of reads outstanding -- enough for the host link's latency with a few dozen
// blocks.  128-thread blocks with few registers fit beside a resident attention CTA on its SM.
constexpr int kFlatThreads = 128;
constexpr int kFlatUnroll = 8;

__global__ void __launch_bounds__(kFlatThreads)
flat_copy_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src, int64_t nvec,
                 unsigned char* __restrict__ dtail, const unsigned char* __restrict__ stail, int tail)
{
    const int64_t per_block = (int64_t)kFlatThreads * kFlatUnroll;
    for (int64_t base = (int64_t)blockIdx.x * per_block + threadIdx.x; base < nvec;
         base += (int64_t)gridDim.x * per_block) {
        uint4 r[kFlatUnroll];
#pragma unroll
        for (int u = 0; u < kFlatUnroll; ++u) {
            const int64_t x = base + u * kFlatThreads;
            if (x < nvec)
                r[u] = src[x];
        }
#pragma unroll
        for (int u = 0; u < kFlatUnroll; ++u) {
            const int64_t x = base + u * kFlatThreads;
            if (x < nvec)
                dst[x] = r[u];
        }
    }
    if (blockIdx.x == 0 && threadIdx.x < tail)
        dtail[threadIdx.x] = stail[threadIdx.x];
}

void launch_flat_copy(void* dst, const void* src, int64_t bytes, cudaStream_t stream)
{
    if (bytes <= 0)
        return;
    const int64_t nvec = bytes / 16;
    const int tail = (int)(bytes - nvec * 16);
    const int64_t per_block = (int64_t)kFlatThreads * kFlatUnroll;
    int64_t blocks = (nvec + per_block - 1) / per_block;
    if (blocks > 256)
        blocks = 256;
    if (blocks < 1)
        blocks = 1;
    flat_copy_kernel<<<(unsigned)blocks, kFlatThreads, 0, stream>>>(
        static_cast<uint4*>(dst), static_cast<const uint4*>(src), nvec, static_cast<unsigned char*>(dst) + nvec * 16,
        static_cast<const unsigned char*>(src) + nvec * 16, tail);
}

}  // namespace hstu
