// combine.cu -- the fused epilogue out = LayerNorm(o) * u over each token's H*D vector.
//
// Elementwise gating before the output projection (aitrends.kr summary, section
// "HSTU의 순차 모델링"; news.bpdata.com, section "HSTU"); the library normalises the whole
// H*D vector of a token (biased variance, eps inside the square root, no affine), or, as
// variants, each head's D values and/or with an affine gamma, beta before the gate.
//
// The attention kernels leave fp32 partial outputs o[split][token][H][D] in the workspace
// (several splits when a user's keys were divided across CTAs; HSTU has no softmax
// normaliser, so partials simply add).  One warp per token: each lane owns kVec float4
// chunks of the H*D vector; the loads of every split are issued before any of them is used
// (the kernel is bound by memory latency, not arithmetic), the splits are summed in fixed
// order, the mean and then the variance come from registers, and (o - mean) * rstd * u is
// written with vector stores.
#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {

constexpr int kCombineThreads = 128;   // small blocks fit beside a resident attention CTA

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    using type = float4;
    static __device__ __forceinline__ float4 to_f4(const float4& v) { return v; }
    static __device__ __forceinline__ float4 from_f4(const float4& v) { return v; }
};
template <> struct Vec4<__nv_bfloat16> {
    using type = uint2;   // four bf16
    static __device__ __forceinline__ float4 to_f4(const uint2& v)
    {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
        return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
    }
    static __device__ __forceinline__ uint2 from_f4(const float4& f)
    {
        __nv_bfloat162 a = __floats2bfloat162_rn(f.x, f.y);
        __nv_bfloat162 b = __floats2bfloat162_rn(f.z, f.w);
        uint2 r;
        r.x = *reinterpret_cast<uint32_t*>(&a);
        r.y = *reinterpret_cast<uint32_t*>(&b);
        return r;
    }
};

// kVec = float4 chunks per lane (H*D = 128 * kVec); kMaxS = splits held in flight at once.
template <typename T, int kVec>
__global__ void __launch_bounds__(kCombineThreads)
ln_gate_kernel(const float* __restrict__ part, int32_t S_all, const int32_t* __restrict__ counts, int64_t ntok,
               int32_t HD, const T* __restrict__ u, T* __restrict__ out, float eps)
{
    using V = typename Vec4<T>::type;
    // the next attention call (a programmatic dependent of this grid) may start its set-up now;
    // it waits for this grid's completion before it touches anything this grid reads or writes
    sm100::pdl_launch_dependents();
    sm100::pdl_wait_primary();          // launched early behind the attention grid
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (kCombineThreads / 32) + (threadIdx.x >> 5);
    if (t >= ntok)
        return;
    const int32_t S = counts ? max(1, min(counts[t], S_all)) : S_all;
    const int64_t plane = ntok * (int64_t)HD;              // floats per split
    const float4* p = reinterpret_cast<const float4*>(part + t * HD);
    const V* uv = reinterpret_cast<const V*>(u + t * HD);
    V ur[kVec];
#pragma unroll
    for (int m = 0; m < kVec; ++m)
        ur[m] = uv[lane + 32 * m];                          // u early: its latency overlaps the sums
    float4 x[kVec];
#pragma unroll
    for (int m = 0; m < kVec; ++m)
        x[m] = p[lane + 32 * m];
    int s = 1;
    for (; s + 3 < S; s += 4) {                             // four splits in flight
        float4 y[4][kVec];
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int m = 0; m < kVec; ++m)
                y[k][m] = p[(s + k) * (plane / 4) + lane + 32 * m];
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int m = 0; m < kVec; ++m) {
                x[m].x += y[k][m].x;
                x[m].y += y[k][m].y;
                x[m].z += y[k][m].z;
                x[m].w += y[k][m].w;
            }
    }
    for (; s < S; ++s) {
#pragma unroll
        for (int m = 0; m < kVec; ++m) {
            const float4 y = p[s * (plane / 4) + lane + 32 * m];
            x[m].x += y.x;
            x[m].y += y.y;
            x[m].z += y.z;
            x[m].w += y.w;
        }
    }
    float sum = 0.f;
#pragma unroll
    for (int m = 0; m < kVec; ++m)
        sum += (x[m].x + x[m].y) + (x[m].z + x[m].w);
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum / (float)HD;
    float sq = 0.f;
#pragma unroll
    for (int m = 0; m < kVec; ++m) {
        const float a = x[m].x - mean, b = x[m].y - mean, c = x[m].z - mean, d = x[m].w - mean;
        sq += (a * a + b * b) + (c * c + d * d);
    }
    for (int o = 16; o > 0; o >>= 1)
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rstd = 1.0f / sqrtf(sq / (float)HD + eps);
    V* ov = reinterpret_cast<V*>(out + t * HD);
#pragma unroll
    for (int m = 0; m < kVec; ++m) {
        const float4 g = Vec4<T>::to_f4(ur[m]);
        ov[lane + 32 * m] = Vec4<T>::from_f4(make_float4((x[m].x - mean) * rstd * g.x, (x[m].y - mean) * rstd * g.y,
                                                         (x[m].z - mean) * rstd * g.z, (x[m].w - mean) * rstd * g.w));
    }
}

// Fallback for H*D not a multiple of 128: one warp per token, scalar accesses.
template <typename T>
__global__ void __launch_bounds__(kCombineThreads)
ln_gate_kernel_scalar(const float* __restrict__ part, int32_t S_all, const int32_t* __restrict__ counts,
                      int64_t ntok, int32_t HD, const T* __restrict__ u, T* __restrict__ out, float eps)
{
    sm100::pdl_launch_dependents();
    sm100::pdl_wait_primary();
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (kCombineThreads / 32) + (threadIdx.x >> 5);
    if (t >= ntok)
        return;
    const int32_t S = counts ? max(1, min(counts[t], S_all)) : S_all;
    float x[64];
    float sum = 0.f;
#pragma unroll
    for (int m = 0; m < 64; ++m) {
        const int e = lane + 32 * m;
        float acc = 0.f;
        if (e < HD)
            for (int s = 0; s < S; ++s)
                acc += part[((int64_t)s * ntok + t) * HD + e];
        x[m] = acc;
        sum += acc;
    }
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum / (float)HD;
    float sq = 0.f;
#pragma unroll
    for (int m = 0; m < 64; ++m) {
        const int e = lane + 32 * m;
        const float dlt = e < HD ? x[m] - mean : 0.f;
        sq += dlt * dlt;
    }
    for (int o = 16; o > 0; o >>= 1)
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rstd = 1.0f / sqrtf(sq / (float)HD + eps);
#pragma unroll
    for (int m = 0; m < 64; ++m) {
        const int e = lane + 32 * m;
        if (e < HD) {
            const int64_t idx = t * HD + e;
            out[idx] = Elem<T>::from_float((x[m] - mean) * rstd * Elem<T>::to_float(u[idx]));
        }
    }
}

// The variants (per-head statistics and/or an affine gamma, beta before the gate): one warp per
// token as above; the token's summed o is staged in shared memory (H*D <= 2048 floats per warp),
// then each normalisation group -- the whole vector, or one head's D values -- gets its own
// two-pass mean and variance.  out = ((o - mean) * rstd * gamma + beta) * u.
template <typename T>
__global__ void __launch_bounds__(kCombineThreads)
ln_gate_variant_kernel(const float* __restrict__ part, int32_t S_all, const int32_t* __restrict__ counts,
                       int64_t ntok, int32_t HD, int32_t group, const float* __restrict__ gamma,
                       const float* __restrict__ beta, const T* __restrict__ u, T* __restrict__ out, float eps)
{
    extern __shared__ float xs_all[];
    sm100::pdl_launch_dependents();
    sm100::pdl_wait_primary();
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (kCombineThreads / 32) + (threadIdx.x >> 5);
    if (t >= ntok)
        return;
    float* xs = xs_all + (threadIdx.x >> 5) * HD;
    const int32_t S = counts ? max(1, min(counts[t], S_all)) : S_all;
    for (int e = lane; e < HD; e += 32) {
        float acc = 0.f;
        for (int s = 0; s < S; ++s)
            acc += part[((int64_t)s * ntok + t) * HD + e];
        xs[e] = acc;
    }
    __syncwarp();
    for (int g0 = 0; g0 < HD; g0 += group) {
        float sum = 0.f;
        for (int e = g0 + lane; e < g0 + group; e += 32)
            sum += xs[e];
        for (int o = 16; o > 0; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float mean = sum / (float)group;
        float sq = 0.f;
        for (int e = g0 + lane; e < g0 + group; e += 32) {
            const float d = xs[e] - mean;
            sq += d * d;
        }
        for (int o = 16; o > 0; o >>= 1)
            sq += __shfl_xor_sync(0xffffffffu, sq, o);
        const float rstd = 1.0f / sqrtf(sq / (float)group + eps);
        for (int e = g0 + lane; e < g0 + group; e += 32) {
            const int64_t idx = t * HD + e;
            const float g = gamma ? gamma[e] : 1.0f;
            const float b = beta ? beta[e] : 0.0f;
            out[idx] = Elem<T>::from_float(((xs[e] - mean) * rstd * g + b) * Elem<T>::to_float(u[idx]));
        }
    }
}

// Launch with programmatic stream serialization: the grid may be scheduled while the
// previous kernel on the stream is still running; the kernel waits (griddepcontrol.wait)
// before it touches that kernel's results.
template <typename... KArgs, typename... Args>
static void launch_pdl_smem(void (*kern)(KArgs...), unsigned grid, size_t smem, cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename... KArgs, typename... Args>
static void launch_pdl(void (*kern)(KArgs...), unsigned grid, cudaStream_t stream, Args... args)
{
    launch_pdl_smem(kern, grid, 0, stream, args...);
}

template <typename T>
static void launch_typed(const float* part, int32_t S, const int32_t* counts, int64_t ntok, int32_t HD, const void* u,
                         void* out, float eps, const LnVariant& var, cudaStream_t stream)
{
    const int per_warp = kCombineThreads / 32;
    const unsigned grid = (unsigned)((ntok + per_warp - 1) / per_warp);
    const T* uu = static_cast<const T*>(u);
    T* oo = static_cast<T*>(out);
    if (var.any()) {
        const int32_t group = var.per_head ? var.D : HD;
        launch_pdl_smem(ln_gate_variant_kernel<T>, grid, (size_t)per_warp * HD * sizeof(float), stream, part, S,
                        counts, ntok, HD, group, var.gamma, var.beta, uu, oo, eps);
        return;
    }
    if (HD % 128 == 0) {
        switch (HD / 128) {
        case 1: launch_pdl(ln_gate_kernel<T, 1>, grid, stream, part, S, counts, ntok, HD, uu, oo, eps); return;
        case 2: launch_pdl(ln_gate_kernel<T, 2>, grid, stream, part, S, counts, ntok, HD, uu, oo, eps); return;
        case 4: launch_pdl(ln_gate_kernel<T, 4>, grid, stream, part, S, counts, ntok, HD, uu, oo, eps); return;
        case 8: launch_pdl(ln_gate_kernel<T, 8>, grid, stream, part, S, counts, ntok, HD, uu, oo, eps); return;
        case 16: launch_pdl(ln_gate_kernel<T, 16>, grid, stream, part, S, counts, ntok, HD, uu, oo, eps); return;
        default: break;
        }
    }
    launch_pdl(ln_gate_kernel_scalar<T>, grid, stream, part, S, counts, ntok, HD, uu, oo, eps);
}

void launch_ln_gate(const float* part, int32_t S, const int32_t* counts, int64_t ntok, int32_t HD, const void* u,
                    void* out, bool fp32, float eps, const LnVariant& var, cudaStream_t stream)
{
    if (ntok <= 0)
        return;
    if (fp32)
        launch_typed<float>(part, S, counts, ntok, HD, u, out, eps, var, stream);
    else
        launch_typed<__nv_bfloat16>(part, S, counts, ntok, HD, u, out, eps, var, stream);
}

}  // namespace hstu
