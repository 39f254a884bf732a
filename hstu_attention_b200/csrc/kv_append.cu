// kv_append.cu -- scatter new K/V rows into the paged KV table (bit-exact 16-byte copies).
//
// The KV cache "append" of the HSTU serving path (NVIDIA blog "Deploying an HSTU Generative
// Recommender with NVIDIA Dynamo-Triton", section "Why serving large sequential recommenders
// is hard": the GPU cache is a paged KV table supporting lookup, allocate, append, evict).
//
// Grid: (ceil(max_new / kTokPerBlock), B).  Block b.y = user; each block copies up to
// kTokPerBlock of that user's appended tokens.  A token's K (or V) row for all heads is H*D
// contiguous elements in k_new; in the pages each head's row is D contiguous elements at
// [page][h][slot].  Threads move 16-byte chunks, so loads are fully coalesced and every
// store writes whole 16-byte vectors.
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {

constexpr int kAppendThreads = 256;
constexpr int kTokPerBlock = 16;

__global__ void __launch_bounds__(kAppendThreads)
kv_append_kernel(uint4* __restrict__ k_pages, uint4* __restrict__ v_pages, const int32_t* __restrict__ page_table,
                 const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                 const int32_t* __restrict__ cached_lens, const int32_t* __restrict__ new_lens,
                 const int32_t* __restrict__ num_targets, int64_t total_new, int32_t H,
                 int32_t row_chunks /* D*esize/16 */, int32_t P, int32_t num_pages, int32_t max_pages,
                 int32_t max_new, void* ws, int32_t* __restrict__ ts_pages, const int32_t* __restrict__ ts_new)
{
    __shared__ int64_t s_off;
    __shared__ int32_t s_ok;
    __shared__ int32_t s_pages[kTokPerBlock];
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * kTokPerBlock;
    const int32_t C = cached_lens[b], N = new_lens[b];
    const int32_t T = num_targets ? num_targets[b] : 0;
    const int32_t n_app = N - T;
    if (threadIdx.x < 32) {
        int64_t off = warp_prefix_offset(new_lens, b);
        if (threadIdx.x == 0) {
            s_off = off;
            const bool ok = C >= 0 && N >= 0 && T >= 0 && n_app >= 0 && N <= max_new && off + N <= total_new;
            s_ok = ok;
            if (!ok && blockIdx.x == 0)
                set_flag(ws, HSTU_DEV_BAD_LENGTH);
        }
    }
    __syncthreads();
    if (threadIdx.x < kTokPerBlock) {
        int32_t page = -1;
        const int t = t0 + threadIdx.x;
        if (s_ok && t < n_app) {
            int64_t pos = (int64_t)C + t;
            int64_t lp = pos / P;
            if (lp >= max_pages) {
                set_flag(ws, HSTU_DEV_BAD_LENGTH);
            } else {
                int32_t pg = page_table[(int64_t)b * max_pages + lp];
                if (pg < 0 || pg >= num_pages)
                    set_flag(ws, HSTU_DEV_BAD_PAGE);
                else
                    page = pg;
            }
        }
        s_pages[threadIdx.x] = page;
        if (ts_pages && page >= 0) {
            // the token's timestamp goes beside its K and V (slot for slot)
            const int64_t pos = (int64_t)C + t;
            ts_pages[(int64_t)page * P + pos % P] = ts_new[s_off + t];
        }
    }
    __syncthreads();
    const int64_t off = s_off;
    const int32_t tok_chunks = H * row_chunks;            // 16-byte chunks per token
    const int32_t total = kTokPerBlock * tok_chunks;
    for (int x = threadIdx.x; x < total; x += kAppendThreads) {
        const int tl = x / tok_chunks;
        const int page = s_pages[tl];
        if (page < 0)
            continue;
        const int within = x - tl * tok_chunks;
        const int h = within / row_chunks;
        const int ch = within - h * row_chunks;
        const int64_t pos = (int64_t)C + t0 + tl;
        const int64_t slot = pos % P;
        const int64_t src = (off + t0 + tl) * tok_chunks + within;
        const int64_t dst = (((int64_t)page * H + h) * P + slot) * row_chunks + ch;
        k_pages[dst] = k_new[src];
        v_pages[dst] = v_new[src];
    }
}

void launch_kv_append(void* k_pages, void* v_pages, const int32_t* page_table, const void* k_new,
                      const void* v_new, const int32_t* cached_lens, const int32_t* new_lens,
                      const int32_t* num_targets, int32_t B, int64_t total_new, int32_t H, int32_t D,
                      int32_t esize,
                      int32_t P, int32_t num_pages, int32_t max_pages, int32_t max_new, void* ws,
                      int32_t* ts_pages, const int32_t* ts_new, cudaStream_t stream)
{
    if (B <= 0 || max_new <= 0)
        return;
    dim3 grid((max_new + kTokPerBlock - 1) / kTokPerBlock, B);
    kv_append_kernel<<<grid, kAppendThreads, 0, stream>>>(
        static_cast<uint4*>(k_pages), static_cast<uint4*>(v_pages), page_table, static_cast<const uint4*>(k_new),
        static_cast<const uint4*>(v_new), cached_lens, new_lens, num_targets, total_new, H, D * esize / 16, P,
        num_pages, max_pages, max_new, ws, ts_pages, ts_new);
}

}  // namespace hstu
