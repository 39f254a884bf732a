// kernels.cuh -- launch interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hstu {

struct SimtArgs {
    const void *q, *k, *v;                 // jagged rows, or q_new / k_new / v_new
    const void *k_pages, *v_pages;         // paged only
    const int32_t* page_table;
    const int32_t* seq_offsets;            // jagged
    const int32_t *cached_lens, *new_lens; // paged
    const int32_t* num_targets;
    const float* rab;
    void* ws;                              // status word
    float* part;                           // fp32 partial outputs [tokens][H][D] (one plane)
    int64_t total_tokens;                  // jagged: all tokens; paged: all new tokens
    int32_t max_len;                       // jagged: max_seqlen; paged: max_new
    int32_t H, D, NB, n_max, P, num_pages, max_pages;
    double ln_nmax;
};

struct TcArgs {
    const int32_t* seq_offsets;
    const int32_t* cached_lens;
    const int32_t* new_lens;
    const int32_t* num_targets;
    const int32_t* page_table;
    const float* rab;
    void* ws;               // status word
    float* part;            // fp32 partial outputs [max_splits][tokens][H][D]
    int32_t* counts;        // paged: per-token number of partial planes written (split count)
    int64_t total_tokens;   // rows of q/k/v/u (jagged) or of the new-token arrays (paged)
    int32_t max_len;        // jagged: max_seqlen; paged: max_new
    int32_t H, NB, n_max, P, num_pages, max_pages, qblocks;
    int32_t B;              // users
    int32_t max_splits;     // paged: partial planes available
    int32_t target_ctas;    // paged: CTAs the balanced split aims for (one per SM)
    double ln_nmax;
    float inv_n;
    uint64_t timeout_ns;    // limit of a role's wait for another role (then the CTA aborts)
    uint64_t drain_ns;      // limit of the waits for a CTA's own copies and products in flight
    int32_t overlap_previous;   // paged: launched as a programmatic dependent of the previous kernel
    uint32_t inject;        // test-only fault injection (kInjectStallV), 0 in normal calls
    const float* rab_time;  // jagged tensor-core path: [H][NBT] second (time) bias, or null
    const int32_t* ts;      // [tokens] timestamps (with rab_time): all tokens (jagged) or new tokens (paged)
    const int32_t* ts_pages;    // paged: [num_pages][P] timestamps of the cached tokens
    int32_t NBT;            // time buckets
};

// inject bit: the V producer issues no load, so the first wait on a V tile runs out (tests of
// the time-out path; every other role then aborts through its bounded waits)
constexpr uint32_t kInjectStallV = 1u << 0;

// The paged tensor-core kernel (attn_paged.cu) takes the same argument block; seq_offsets and
// target_ctas are unused there.
using PagedArgs = TcArgs;

struct TcMaps {
    CUtensorMap q, k, v, kp, vp;
};

// Bucket boundaries computed on the host: v[k] = smallest distance d with bucket(d) >= k for
// k < count - 1, v[count - 1] = INT_MAX.  count == 0 means "not passed" (too many buckets for
// the parameter block); the kernels then evaluate them on the device.
constexpr int kMaxParamNB = 512;
struct BucketBounds {
    int32_t count;
    int32_t v[kMaxParamNB + 1];
};

void launch_kv_page_copy(const void* src_k, const void* src_v, void* dst_k, void* dst_v, const int32_t* pairs,
                         int32_t n_pairs, int32_t src_pages, int32_t dst_pages, int64_t page_bytes, void* ws,
                         cudaStream_t stream);

void launch_flat_copy(void* dst, const void* src, int64_t bytes, cudaStream_t stream);

// C = act(A B^T) on tensor cores (gemm.cu): A [M, K] and B [N, K] bf16 (TMA maps with 64 x 128
// boxes), N a multiple of 128, K a multiple of 64.  Output column n goes to
// out[(n / split) * block_stride + m * ldo + n % split].
struct GemmArgs {
    int32_t M, N, K;
    int32_t split;              // columns per output block (a multiple of 128)
    int64_t block_stride;       // elements between output blocks
    int64_t ldo;                // elements between output rows
    __nv_bfloat16* out;
    int32_t silu;               // apply SiLU before rounding
    void* ws;                   // status word (time-outs), may be null
    uint64_t timeout_ns, drain_ns;
    int32_t pdl;                // launch as a programmatic dependent of the previous kernel
};
void launch_gemm_bf16(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmArgs& g, cudaStream_t stream);

void launch_kv_append(void* k_pages, void* v_pages, const int32_t* page_table, const void* k_new,
                      const void* v_new, const int32_t* cached_lens, const int32_t* new_lens,
                      const int32_t* num_targets, int32_t B, int64_t total_new, int32_t H, int32_t D,
                      int32_t esize,
                      int32_t P, int32_t num_pages, int32_t max_pages, int32_t max_new, void* ws,
                      int32_t* ts_pages, const int32_t* ts_new, cudaStream_t stream);
// counts == nullptr: every token has S partial planes; otherwise token t has counts[t].
// LayerNorm-gate variants (the base kernels run when none is set)
struct LnVariant {
    bool per_head = false;        // statistics per head (D values) instead of per token (H*D)
    int32_t D = 0;
    const float* gamma = nullptr; // [H*D] or null (1)
    const float* beta = nullptr;  // [H*D] or null (0)
    bool any() const { return per_head || gamma || beta; }
};
void launch_ln_gate(const float* part, int32_t S, const int32_t* counts, int64_t ntok, int32_t HD, const void* u,
                    void* out, bool fp32, float eps, const LnVariant& var, cudaStream_t stream);
// Backward pass of the jagged attention (attn_bwd.cu).
struct BwdArgs {
    const void *q, *k, *v;                 // [tokens][H][D], params dtype
    const int32_t* seq_offsets;
    const int32_t* num_targets;
    const float* rab;                      // [H][NB]
    float* dO;                             // [tokens][H][D] fp32: gradient of o (workspace)
    float *dq, *dk, *dv;                   // [tokens][H][D] fp32, written
    float* drab;                           // [H][NB] fp32, accumulated (zeroed by the caller)
    int64_t total_tokens;
    int32_t B, H, D, NB, n_max;
    int32_t max_seqlen;                    // users longer than this are rejected (as in the forward)
    double ln_nmax;
    float inv_n;
};

void launch_jagged_bwd(const BwdArgs& a, const float* o, const void* u, const void* dout, float* du, float eps,
                       bool fp32, cudaStream_t stream);
// Only the LayerNorm-gate backward (du; do in fp32 when a.dO is not null, in bf16 when dO16 is not null).
void launch_ln_gate_bwd(const BwdArgs& a, const float* o, const void* u, const void* dout, float* du,
                        __nv_bfloat16* dO16, float eps, bool fp32, cudaStream_t stream);

// Backward on tensor cores (attn_bwd_tc.cu; bf16, D = 128): maps over q, k, v and the bf16
// gradient of o, all [tokens][H][D] rows with {64, 1, 128} boxes.
struct BwdTcMaps {
    CUtensorMap q, k, v, dO;
};
struct BwdTcArgs {
    const int32_t* seq_offsets;
    const int32_t* num_targets;
    const float* rab;
    void* ws;
    float *dq, *dk, *dv, *drab;
    int64_t total_tokens;
    int32_t max_len;        // max_seqlen
    int32_t H, NB, n_max, B, qblocks;
    double ln_nmax;
    float inv_n;
    uint64_t timeout_ns, drain_ns;
};
void launch_bwd_tc(const BwdTcMaps& m, const BwdTcArgs& a, const BucketBounds& bb, cudaStream_t stream);

void launch_attn_simt(const SimtArgs& a, bool paged, bool fp32, int32_t B, cudaStream_t stream);
// Jagged prefill on tensor cores (bf16, D = 128).
void launch_attn_tc(const TcMaps& m, const TcArgs& a, const BucketBounds& bb, int32_t B, cudaStream_t stream);
// Paged cache hit on tensor cores (bf16, D = 128); at most paged_max_users() users per call.
void launch_attn_paged(const TcMaps& m, const PagedArgs& a, const BucketBounds& bb, int num_sms,
                       cudaStream_t stream);
int paged_max_users();

}  // namespace hstu
