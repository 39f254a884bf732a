// combine.cu -- the fused epilogue out = LayerNorm(o) * u over each token's H*D vector.
//
// Elementwise gating before the output projection (aitrends.kr summary, section
// "HSTU의 순차 모델링"; news.bpdata.com, section "HSTU"); the library normalises the whole
// H*D vector of a token (biased variance, eps inside the square root, no affine).
//
// The attention kernels leave fp32 partial outputs o[split][token][H][D] in the workspace
// (several splits when a user's keys were divided across CTAs; HSTU has no softmax
// normaliser, so partials simply add).  One warp per token sums the splits in fixed order,
// takes the mean and then the variance from registers, and writes (o - mean) * rstd * u.
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {

constexpr int kCombineThreads = 256;

template <typename T, int kPerLane>
__global__ void __launch_bounds__(kCombineThreads)
ln_gate_kernel(const float* __restrict__ part, int32_t S, int64_t ntok, int32_t HD, const T* __restrict__ u,
               T* __restrict__ out, float eps)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (kCombineThreads / 32) + (threadIdx.x >> 5);
    if (t >= ntok)
        return;
    float x[kPerLane];
    float sum = 0.f;
#pragma unroll
    for (int m = 0; m < kPerLane; ++m) {
        const int e = lane + 32 * m;
        float acc = 0.f;
        if (e < HD) {
            for (int s = 0; s < S; ++s)
                acc += part[((int64_t)s * ntok + t) * HD + e];
        }
        x[m] = acc;
        sum += acc;
    }
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum / (float)HD;
    float sq = 0.f;
#pragma unroll
    for (int m = 0; m < kPerLane; ++m) {
        const int e = lane + 32 * m;
        const float dlt = e < HD ? x[m] - mean : 0.f;
        sq += dlt * dlt;
    }
    for (int o = 16; o > 0; o >>= 1)
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rstd = 1.0f / sqrtf(sq / (float)HD + eps);
#pragma unroll
    for (int m = 0; m < kPerLane; ++m) {
        const int e = lane + 32 * m;
        if (e < HD) {
            const int64_t idx = t * HD + e;
            out[idx] = Elem<T>::from_float((x[m] - mean) * rstd * Elem<T>::to_float(u[idx]));
        }
    }
}

template <typename T>
static void launch_typed(const float* part, int32_t S, int64_t ntok, int32_t HD, const void* u, void* out, float eps,
                         cudaStream_t stream)
{
    const int per_warp = kCombineThreads / 32;
    const unsigned grid = (unsigned)((ntok + per_warp - 1) / per_warp);
    const T* uu = static_cast<const T*>(u);
    T* oo = static_cast<T*>(out);
    const int per_lane = (HD + 31) / 32;
    if (per_lane <= 2)
        ln_gate_kernel<T, 2><<<grid, kCombineThreads, 0, stream>>>(part, S, ntok, HD, uu, oo, eps);
    else if (per_lane <= 4)
        ln_gate_kernel<T, 4><<<grid, kCombineThreads, 0, stream>>>(part, S, ntok, HD, uu, oo, eps);
    else if (per_lane <= 8)
        ln_gate_kernel<T, 8><<<grid, kCombineThreads, 0, stream>>>(part, S, ntok, HD, uu, oo, eps);
    else if (per_lane <= 16)
        ln_gate_kernel<T, 16><<<grid, kCombineThreads, 0, stream>>>(part, S, ntok, HD, uu, oo, eps);
    else if (per_lane <= 32)
        ln_gate_kernel<T, 32><<<grid, kCombineThreads, 0, stream>>>(part, S, ntok, HD, uu, oo, eps);
    else
        ln_gate_kernel<T, 64><<<grid, kCombineThreads, 0, stream>>>(part, S, ntok, HD, uu, oo, eps);
}

void launch_ln_gate(const float* part, int32_t S, int64_t ntok, int32_t HD, const void* u, void* out, bool fp32,
                    float eps, cudaStream_t stream)
{
    if (ntok <= 0)
        return;
    if (fp32)
        launch_typed<float>(part, S, ntok, HD, u, out, eps, stream);
    else
        launch_typed<__nv_bfloat16>(part, S, ntok, HD, u, out, eps, stream);
}

}  // namespace hstu
