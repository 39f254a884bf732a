// attn_bwd.cu -- backward pass of jagged HSTU attention on CUDA cores (fp32 arithmetic).
//
// Given the upstream gradient dout of out = LayerNorm(o) * u (o recomputed by the forward
// attention kernels into the workspace), the chain rule through the gate, the LayerNorm over
// each token's H*D vector and the SiLU-weighted aggregation gives (per user, head, allowed pair
// (i, j); allowed, bucket() and the 1/n_max scale as in the forward):
//     du  = xhat * dout,   dy = dout * u,   do = rstd * (dy - mean(dy) - xhat * mean(dy * xhat))
//     s   = q_i . k_j + rab[h][bucket(i - j)],   sig = sigmoid(s),   w = s * sig / n_max
//     ds  = (do_i . v_j) * sig * (1 + s * (1 - sig)) / n_max
//     dq_i += ds k_j,   dk_j += ds q_i,   dv_j += w do_i,   drab[h][bucket(i - j)] += ds
// SiLU replaces softmax in HSTU (aitrends.kr summary, section "HSTU의 순차 모델링";
// news.bpdata.com, section "HSTU"), so there is no row statistic to recompute: every pair's
// weight is a function of that pair alone.
//
// Kernels (one warp per (token, head), lanes own D/32 channels each):
//   ln_gate_bwd_kernel  du and do from o, u, dout (one warp per token)
//   attn_bwd_dq_kernel  dq_i and drab: walks the keys query i may see
//   attn_bwd_dkv_kernel dk_j, dv_j: walks the queries that may see key j
// A first, plain path: dot products are warp reductions per pair, drab is accumulated with
// atomics.
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {

constexpr int kBwdThreads = 128;                       // four warps per block

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// User of token t (largest b with seq_offsets[b] <= t); -1 when the offsets do not cover it.
__device__ __forceinline__ int user_of(const int32_t* off, int32_t B, int64_t t)
{
    int lo = 0, hi = B;                                // off[lo] <= t < off[hi] when covered
    if (t < off[0] || t >= off[B])
        return -1;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= t)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
ln_gate_bwd_kernel(const float* __restrict__ o, const T* __restrict__ u, const T* __restrict__ dout,
                   float* __restrict__ du, float* __restrict__ dO, __nv_bfloat16* __restrict__ dO16, int64_t ntok,
                   int32_t HD, float eps)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (kBwdThreads / 32) + (threadIdx.x >> 5);
    if (t >= ntok)
        return;
    const float* x = o + t * HD;
    float sum = 0.f;
    for (int e = lane; e < HD; e += 32)
        sum += x[e];
    const float mean = warp_sum(sum) / (float)HD;
    float sq = 0.f;
    for (int e = lane; e < HD; e += 32)
        sq += (x[e] - mean) * (x[e] - mean);
    const float rstd = 1.0f / sqrtf(warp_sum(sq) / (float)HD + eps);
    float mdy = 0.f, mdyx = 0.f;
    for (int e = lane; e < HD; e += 32) {
        const float xhat = (x[e] - mean) * rstd;
        const float g = Elem<T>::to_float(dout[t * HD + e]);
        du[t * HD + e] = xhat * g;
        const float dy = g * Elem<T>::to_float(u[t * HD + e]);
        mdy += dy;
        mdyx += dy * xhat;
    }
    mdy = warp_sum(mdy) / (float)HD;
    mdyx = warp_sum(mdyx) / (float)HD;
    for (int e = lane; e < HD; e += 32) {
        const float xhat = (x[e] - mean) * rstd;
        const float dy = Elem<T>::to_float(dout[t * HD + e]) * Elem<T>::to_float(u[t * HD + e]);
        const float g = rstd * (dy - mdy - xhat * mdyx);
        if (dO)
            dO[t * HD + e] = g;
        if (dO16)
            dO16[t * HD + e] = __float2bfloat16_rn(g);
    }
}

// s and d(weight)/ds for one pair: returns ds, writes w.
__device__ __forceinline__ float pair_grad(float s, float dw, float inv_n, float& w)
{
    const float sig = 1.0f / (1.0f + expf(-s));
    w = s * sig * inv_n;
    return dw * sig * (1.0f + s * (1.0f - sig)) * inv_n;
}

template <typename T, int kC>
__global__ void __launch_bounds__(kBwdThreads)
attn_bwd_dq_kernel(BwdArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * (kBwdThreads / 32) + (threadIdx.x >> 5);
    const int H = a.H, D = kC * 32;
    if (wid >= a.total_tokens * H)
        return;
    const int64_t t = wid / H;
    const int h = (int)(wid % H);
    const int64_t HD = (int64_t)H * D;
    float acc[kC];
#pragma unroll
    for (int c = 0; c < kC; ++c)
        acc[c] = 0.f;
    const int b = user_of(a.seq_offsets, a.B, t);
    if (b >= 0) {
        const int64_t s0 = a.seq_offsets[b], L = a.seq_offsets[b + 1] - s0;
        const int32_t nt = a.num_targets ? a.num_targets[b] : 0;
        // the forward's rule (jagged_geom): a rejected user has o = 0 and contributes nothing
        const bool ok = s0 >= 0 && L > 0 && s0 + L <= a.total_tokens && nt >= 0 && nt <= L && L <= a.n_max &&
                        L <= a.max_seqlen;
        const int64_t hist = L - nt, i = t - s0;
        const T* q = static_cast<const T*>(a.q);
        const T* k = static_cast<const T*>(a.k);
        const T* v = static_cast<const T*>(a.v);
        float qi[kC], doi[kC];
#pragma unroll
        for (int c = 0; c < kC; ++c) {
            qi[c] = Elem<T>::to_float(q[t * HD + (int64_t)h * D + lane + 32 * c]);
            doi[c] = a.dO[t * HD + (int64_t)h * D + lane + 32 * c];
        }
        // keys visible to query i: history up to i (history query) or all history plus itself
        const int64_t jn = !ok ? 0 : (i < hist ? i + 1 : hist + 1);
        for (int64_t n = 0; n < jn; ++n) {
            const int64_t j = (i >= hist && n == hist) ? i : n;
            const int64_t kr = (s0 + j) * HD + (int64_t)h * D;
            float s = 0.f, dw = 0.f, kj[kC];
#pragma unroll
            for (int c = 0; c < kC; ++c) {
                kj[c] = Elem<T>::to_float(k[kr + lane + 32 * c]);
                s += qi[c] * kj[c];
                dw += doi[c] * Elem<T>::to_float(v[kr + lane + 32 * c]);
            }
            const int bk = bucket_of(i - j, a.ln_nmax, a.NB);
            s = warp_sum(s) + a.rab[(int64_t)h * a.NB + bk];
            dw = warp_sum(dw);
            float w;
            const float ds = pair_grad(s, dw, a.inv_n, w);
#pragma unroll
            for (int c = 0; c < kC; ++c)
                acc[c] += ds * kj[c];
            if (lane == 0)
                atomicAdd(&a.drab[(int64_t)h * a.NB + bk], ds);
        }
    }
#pragma unroll
    for (int c = 0; c < kC; ++c)
        a.dq[t * HD + (int64_t)h * D + lane + 32 * c] = acc[c];
}

template <typename T, int kC>
__global__ void __launch_bounds__(kBwdThreads)
attn_bwd_dkv_kernel(BwdArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * (kBwdThreads / 32) + (threadIdx.x >> 5);
    const int H = a.H, D = kC * 32;
    if (wid >= a.total_tokens * H)
        return;
    const int64_t t = wid / H;
    const int h = (int)(wid % H);
    const int64_t HD = (int64_t)H * D;
    float dk[kC], dv[kC];
#pragma unroll
    for (int c = 0; c < kC; ++c)
        dk[c] = dv[c] = 0.f;
    const int b = user_of(a.seq_offsets, a.B, t);
    if (b >= 0) {
        const int64_t s0 = a.seq_offsets[b], L = a.seq_offsets[b + 1] - s0;
        const int32_t nt = a.num_targets ? a.num_targets[b] : 0;
        // the forward's rule (jagged_geom): a rejected user has o = 0 and contributes nothing
        const bool ok = s0 >= 0 && L > 0 && s0 + L <= a.total_tokens && nt >= 0 && nt <= L && L <= a.n_max &&
                        L <= a.max_seqlen;
        const int64_t hist = L - nt, j = t - s0;
        const T* q = static_cast<const T*>(a.q);
        const T* k = static_cast<const T*>(a.k);
        const T* v = static_cast<const T*>(a.v);
        float kj[kC], vj[kC];
#pragma unroll
        for (int c = 0; c < kC; ++c) {
            kj[c] = Elem<T>::to_float(k[t * HD + (int64_t)h * D + lane + 32 * c]);
            vj[c] = Elem<T>::to_float(v[t * HD + (int64_t)h * D + lane + 32 * c]);
        }
        // queries that see key j: every query from j on (history key), or only j (candidate)
        const int64_t i_end = !ok ? j : (j < hist ? L : j + 1);
        for (int64_t i = j; i < i_end; ++i) {
            const int64_t qr = (s0 + i) * HD + (int64_t)h * D;
            float s = 0.f, dw = 0.f, qv[kC], dov[kC];
#pragma unroll
            for (int c = 0; c < kC; ++c) {
                qv[c] = Elem<T>::to_float(q[qr + lane + 32 * c]);
                dov[c] = a.dO[qr + lane + 32 * c];
                s += qv[c] * kj[c];
                dw += dov[c] * vj[c];
            }
            s = warp_sum(s) + a.rab[(int64_t)h * a.NB + bucket_of(i - j, a.ln_nmax, a.NB)];
            dw = warp_sum(dw);
            float w;
            const float ds = pair_grad(s, dw, a.inv_n, w);
#pragma unroll
            for (int c = 0; c < kC; ++c) {
                dk[c] += ds * qv[c];
                dv[c] += w * dov[c];
            }
        }
    }
#pragma unroll
    for (int c = 0; c < kC; ++c) {
        a.dk[t * HD + (int64_t)h * D + lane + 32 * c] = dk[c];
        a.dv[t * HD + (int64_t)h * D + lane + 32 * c] = dv[c];
    }
}

template <typename T, int kC>
static void launch_pair_kernels(const BwdArgs& a, cudaStream_t s)
{
    const int64_t warps = a.total_tokens * a.H;
    const unsigned grid = (unsigned)((warps + kBwdThreads / 32 - 1) / (kBwdThreads / 32));
    attn_bwd_dq_kernel<T, kC><<<grid, kBwdThreads, 0, s>>>(a);
    attn_bwd_dkv_kernel<T, kC><<<grid, kBwdThreads, 0, s>>>(a);
}

template <typename T>
static void launch_typed(const BwdArgs& a, const float* o, const void* u, const void* dout, float* du, float eps,
                         cudaStream_t s)
{
    const int32_t HD = a.H * a.D;
    const unsigned lgrid = (unsigned)((a.total_tokens + kBwdThreads / 32 - 1) / (kBwdThreads / 32));
    ln_gate_bwd_kernel<T><<<lgrid, kBwdThreads, 0, s>>>(o, static_cast<const T*>(u), static_cast<const T*>(dout),
                                                        du, a.dO, nullptr, a.total_tokens, HD, eps);
    switch (a.D) {
    case 32: launch_pair_kernels<T, 1>(a, s); break;
    case 64: launch_pair_kernels<T, 2>(a, s); break;
    default: launch_pair_kernels<T, 4>(a, s); break;
    }
}

void launch_ln_gate_bwd(const BwdArgs& a, const float* o, const void* u, const void* dout, float* du,
                        __nv_bfloat16* dO16, float eps, bool fp32, cudaStream_t stream)
{
    if (a.total_tokens <= 0)
        return;
    const int32_t HD = a.H * a.D;
    const unsigned lgrid = (unsigned)((a.total_tokens + kBwdThreads / 32 - 1) / (kBwdThreads / 32));
    if (fp32)
        ln_gate_bwd_kernel<float><<<lgrid, kBwdThreads, 0, stream>>>(
            o, static_cast<const float*>(u), static_cast<const float*>(dout), du, a.dO, dO16, a.total_tokens, HD, eps);
    else
        ln_gate_bwd_kernel<__nv_bfloat16><<<lgrid, kBwdThreads, 0, stream>>>(
            o, static_cast<const __nv_bfloat16*>(u), static_cast<const __nv_bfloat16*>(dout), du, a.dO, dO16,
            a.total_tokens, HD, eps);
}

void launch_jagged_bwd(const BwdArgs& a, const float* o, const void* u, const void* dout, float* du, float eps,
                       bool fp32, cudaStream_t stream)
{
    if (a.total_tokens <= 0)
        return;
    if (fp32)
        launch_typed<float>(a, o, u, dout, du, eps, stream);
    else
        launch_typed<__nv_bfloat16>(a, o, u, dout, du, eps, stream);
}

}  // namespace hstu
