// attn_simt.cu -- CUDA-core HSTU attention (fp32 inputs, and any supported head_dim).
//
// Computes, per user b, head h and query row i, the pre-normalisation output
//   o[i,h,:] = sum_j allowed(i,j) * SiLU(q_i . k_j + rab[h][bucket(i-j)]) / n_max * v[j,h,:]
// (SiLU weighting instead of softmax plus a relative attention bias: aitrends.kr summary,
// section "HSTU의 순차 모델링"; news.bpdata.com, section "HSTU") into the workspace as fp32.
// The LayerNorm(o) * u gate runs afterwards in combine.cu.
//
// This is the exact-arithmetic path: fp32 products and sums, SiLU through expf.  The bf16
// head_dim-128 workloads use the tcgen05 kernel in attn_tc.cu instead.
//
// Layout: one CTA = (32 query rows, head h, user b); 4 threads per query row, each owning
// D/4 contiguous channels.  Keys are staged in shared memory 32 at a time, widened to fp32;
// keys come from the jagged k/v rows, or (paged) from pages for positions < cached_len and
// from k_new/v_new after that.
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {

constexpr int kSimtRows = 32;
constexpr int kSimtKeys = 32;
constexpr int kSimtThreads = 128;
constexpr int kSimtMaxD = 128;

template <typename T, bool kPaged>
__global__ void __launch_bounds__(kSimtThreads) attn_simt_kernel(SimtArgs a)
{
    __shared__ float sK[kSimtKeys][kSimtMaxD];
    __shared__ float sV[kSimtKeys][kSimtMaxD];
    __shared__ float sWin[2 * kSimtKeys];
    __shared__ UserGeom sG;

    const int b = blockIdx.z, h = blockIdx.y, qb = blockIdx.x;
    const int H = a.H, D = a.D;
    const int64_t HD = (int64_t)H * D;
    if (threadIdx.x < 32) {
        UserGeom g = kPaged ? paged_geom(a.cached_lens, a.new_lens, a.num_targets, b, a.total_tokens, a.max_len,
                                         a.max_pages * a.P, a.n_max)
                            : jagged_geom(a.seq_offsets, a.num_targets, b, a.total_tokens, a.max_len, a.n_max);
        if (threadIdx.x == 0)
            sG = g;
    }
    __syncthreads();
    const UserGeom g = sG;
    if (!g.ok) {
        // a rejected user: the q-block-0 CTA of each head zeroes that head's slice of every row
        // of the user, including rows past the grid (a user longer than the host's bound)
        if (qb == 0) {
            if (h == 0 && threadIdx.x == 0)
                set_flag(a.ws, g.flags);
            for (int64_t x = threadIdx.x; x < (int64_t)g.N * D; x += kSimtThreads)
                a.part[(g.tok0 + x / D) * HD + (int64_t)h * D + x % D] = 0.f;
        }
        return;
    }
    const int r = threadIdx.x >> 2;            // query row within the block
    const int part = threadIdx.x & 3;          // channel quarter
    const int dq = D >> 2;                     // channels per thread
    const int c0 = part * dq;
    const int tq = qb * kSimtRows + r;         // query index among this user's queries
    if (qb * kSimtRows >= g.N)
        return;                                // past this user's queries (uniform)
    const bool row_ok = tq < g.N;
    const int i = g.C + tq;                    // absolute position
    float* out = a.part;

    float acc[kSimtMaxD / 4];
#pragma unroll
    for (int c = 0; c < kSimtMaxD / 4; ++c)
        acc[c] = 0.f;
    float qv[kSimtMaxD / 4];
    const T* qp = static_cast<const T*>(a.q) + (g.tok0 + (row_ok ? tq : 0)) * HD + (int64_t)h * D + c0;
#pragma unroll
    for (int c = 0; c < kSimtMaxD / 4; ++c)
        qv[c] = (c < dq && row_ok && g.ok) ? Elem<T>::to_float(qp[c]) : 0.f;

    if (g.ok) {
        const int i0 = g.C + qb * kSimtRows;
        const int last_q = min(g.N, (qb + 1) * kSimtRows) - 1;
        const int kend = min(g.L, g.C + last_q + 1);             // keys beyond the last query are never seen
        const float inv_n = 1.0f / (float)a.n_max;
        const int lim = row_ok ? min(i + 1, g.hist) : -1;        // allowed: j < lim, or j == i
        const int diag = row_ok ? i : -1;
        for (int j0 = 0; j0 < kend; j0 += kSimtKeys) {
            __syncthreads();
            // stage keys j0 .. j0+31 (widened to fp32), invalid rows as zeros
            for (int x = threadIdx.x; x < kSimtKeys * D; x += kSimtThreads) {
                const int kk = x / D, c = x - kk * D;
                const int j = j0 + kk;
                float kx = 0.f, vx = 0.f;
                if (j < kend) {
                    if (kPaged && j < g.C) {
                        const int32_t page = a.page_table[(int64_t)b * a.max_pages + j / a.P];
                        if (page >= 0 && page < a.num_pages) {
                            const int64_t idx = (((int64_t)page * H + h) * a.P + j % a.P) * D + c;
                            kx = Elem<T>::load(static_cast<const T*>(a.k_pages) + idx);
                            vx = Elem<T>::load(static_cast<const T*>(a.v_pages) + idx);
                        } else if (c == 0) {
                            set_flag(a.ws, HSTU_DEV_BAD_PAGE);
                        }
                    } else {
                        const int64_t idx = (g.key_row0 + (j - g.C)) * HD + (int64_t)h * D + c;
                        kx = Elem<T>::load(static_cast<const T*>(a.k) + idx);
                        vx = Elem<T>::load(static_cast<const T*>(a.v) + idx);
                    }
                }
                sK[kk][c] = kx;
                sV[kk][c] = vx;
            }
            // bias window: entry e holds rab[h][bucket(i0 - j0 - 31 + e)] (0 for negative distance)
            if (threadIdx.x < 2 * kSimtKeys - 1) {
                const int64_t dist = (int64_t)i0 - j0 - (kSimtKeys - 1) + threadIdx.x;
                sWin[threadIdx.x] = dist >= 0 ? a.rab[(int64_t)h * a.NB + bucket_of(dist, a.ln_nmax, a.NB)] : 0.f;
            }
            __syncthreads();
            const int nk = min(kSimtKeys, kend - j0);
            for (int kk = 0; kk < nk; ++kk) {
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < kSimtMaxD / 4; ++c)
                    if (c < dq)
                        s = fmaf(qv[c], sK[kk][c0 + c], s);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                const int j = j0 + kk;
                const bool allowed = (j < lim) || (j == diag);
                if (!allowed)
                    continue;
                s += sWin[r - kk + (kSimtKeys - 1)];
                const float w = s / (1.0f + expf(-s)) * inv_n;
#pragma unroll
                for (int c = 0; c < kSimtMaxD / 4; ++c)
                    if (c < dq)
                        acc[c] = fmaf(w, sV[kk][c0 + c], acc[c]);
            }
        }
    }
    if (row_ok) {
        float* op = out + (g.tok0 + tq) * HD + (int64_t)h * D + c0;
#pragma unroll
        for (int c = 0; c < kSimtMaxD / 4; ++c)
            if (c < dq)
                op[c] = acc[c];
    }
}

void launch_attn_simt(const SimtArgs& a, bool paged, bool fp32, int32_t B, cudaStream_t stream)
{
    const int qblocks = (a.max_len + kSimtRows - 1) / kSimtRows;
    if (B <= 0 || qblocks <= 0)
        return;
    dim3 grid(qblocks, a.H, B);
    if (fp32) {
        if (paged)
            attn_simt_kernel<float, true><<<grid, kSimtThreads, 0, stream>>>(a);
        else
            attn_simt_kernel<float, false><<<grid, kSimtThreads, 0, stream>>>(a);
    } else {
        if (paged)
            attn_simt_kernel<__nv_bfloat16, true><<<grid, kSimtThreads, 0, stream>>>(a);
        else
            attn_simt_kernel<__nv_bfloat16, false><<<grid, kSimtThreads, 0, stream>>>(a);
    }
}

}  // namespace hstu
