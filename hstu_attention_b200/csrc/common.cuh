// common.cuh -- shared device helpers of the HSTU B200 library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu.h"

namespace hstu {

// ------------------------------------------------------------------ workspace layout
// [0, 256)                 : uint32 status word (HSTU_DEV_* bits), rest reserved
// [256, 256 + C)           : int32 per-token split counts (paged), C = tokens * 4 rounded to 256
// [256 + C, ...)           : fp32 partial outputs o[split][token][H][D] of the attention kernels
constexpr size_t kStatusBytes = 256;
constexpr int kMaxSplits = 8;

__host__ __device__ __forceinline__ size_t counts_bytes(int64_t tokens)
{
    return ((size_t)tokens * 4 + 255) & ~(size_t)255;
}

__device__ __forceinline__ void set_flag(void* ws, uint32_t bits)
{
    atomicOr(reinterpret_cast<unsigned int*>(ws), bits);
}

__host__ __device__ __forceinline__ int32_t* split_counts(void* ws)
{
    return reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws) + kStatusBytes);
}

__host__ __device__ __forceinline__ float* partials(void* ws, int64_t tokens)
{
    return reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kStatusBytes + counts_bytes(tokens));
}

// ------------------------------------------------------------------ relative-position bucket
// bucket(0) = 0; bucket(d) = min(NB-1, 1 + floor((NB-1) * ln d / ln n_max)) for d >= 1,
// evaluated in double precision.  inv_den = 1 / ln(n_max) is not used: the quotient is
// taken as written so the floor sees the same rounding as the plain formula.
__device__ __forceinline__ int bucket_of(int64_t d, double ln_nmax, int nb)
{
    if (nb <= 1 || d <= 0 || !(ln_nmax > 0.0))
        return 0;
    double x = (double)(nb - 1) * log((double)d) / ln_nmax;
    int64_t b = 1 + (int64_t)floor(x);
    return (int)(b > nb - 1 ? nb - 1 : b);
}

// ------------------------------------------------------------------ element types
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ float to_float(float x) { return x; }
    static __device__ __forceinline__ float from_float(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
};

// Sum of new_lens[0..b) computed by one warp (every lane returns the total).  Negative
// lengths count as 0 here; the caller flags them.
__device__ __forceinline__ int64_t warp_prefix_offset(const int32_t* lens, int b)
{
    const int lane = threadIdx.x & 31;
    int64_t s = 0;
    for (int i = lane; i < b; i += 32) {
        int32_t x = lens[i];
        s += x > 0 ? x : 0;
    }
    for (int o = 16; o > 0; o >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Per-user geometry shared by the attention kernels.  For the jagged layout the queries
// are all L tokens; for the paged layout they are the N new tokens placed after C cached ones.
// The helpers only read the length arrays: a rejected user's status bits are returned in
// `flags`, and the kernel raises them once it may write the workspace.
struct UserGeom {
    int64_t tok0;      // first query token row in the q/u/out arrays
    int64_t key_row0;  // first row of this user's non-cached keys in k/v (or k_new/v_new)
    int32_t C;         // cached keys read from pages (0 for jagged)
    int32_t N;         // query tokens (jagged: L); rows that cannot be located count as 0
    int32_t L;         // total keys = C + N
    int32_t hist;      // L - num_targets
    uint32_t flags;    // HSTU_DEV_* bits of a rejected user (0 when ok)
    bool ok;
};

// Jagged geometry with validation.
__device__ __forceinline__ UserGeom jagged_geom(const int32_t* seq_offsets, const int32_t* num_targets,
                                                int b, int64_t total_tokens, int32_t max_seqlen, int32_t n_max)
{
    UserGeom g;
    int64_t s0 = seq_offsets[b], s1 = seq_offsets[b + 1];
    int32_t T = num_targets ? num_targets[b] : 0;
    int64_t L = s1 - s0;
    g.ok = true;
    g.flags = 0;
    if (s0 < 0 || s1 > total_tokens || L < 0 || T < 0 || T > L || L > max_seqlen) {
        g.flags = HSTU_DEV_BAD_LENGTH;
        g.ok = false;
    } else if (L > n_max) {
        g.flags = HSTU_DEV_BAD_NMAX;
        g.ok = false;
    }
    g.tok0 = s0;
    g.key_row0 = s0;
    g.C = 0;
    g.N = (s0 < 0 || s1 > total_tokens || L < 0) ? 0 : (int32_t)L;
    g.L = g.N;
    g.hist = g.N - (T > 0 && T <= g.N ? T : 0);
    return g;
}

// Paged geometry; must be called by a full warp (prefix sum of new_lens).
__device__ __forceinline__ UserGeom paged_geom(const int32_t* cached_lens, const int32_t* new_lens,
                                               const int32_t* num_targets, int b, int64_t total_new,
                                               int32_t max_new, int32_t max_cached, int32_t n_max)
{
    UserGeom g;
    int64_t off = warp_prefix_offset(new_lens, b);
    int32_t C = cached_lens[b], N = new_lens[b];
    int32_t T = num_targets ? num_targets[b] : 0;
    g.ok = true;
    g.flags = 0;
    if (C < 0 || N < 0 || T < 0 || T > N || N > max_new || C > max_cached || off + N > total_new) {
        g.flags = HSTU_DEV_BAD_LENGTH;
        g.ok = false;
    } else if ((int64_t)C + N > n_max) {
        g.flags = HSTU_DEV_BAD_NMAX;
        g.ok = false;
    }
    g.tok0 = off;
    g.key_row0 = off;
    g.C = C > 0 ? C : 0;
    g.N = N > 0 ? N : 0;
    g.L = g.C + g.N;
    g.hist = g.L - (T > 0 ? T : 0);
    if (off + g.N > total_new)
        g.N = 0;
    return g;
}

}  // namespace hstu
