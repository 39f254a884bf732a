// gemm.cu -- the HSTU layer's projections on Blackwell tensor cores: C = act(A B^T), bf16 in,
// fp32 accumulate in tensor memory, bf16 out.
//
// The layer around the attention (aitrends.kr summary, section "HSTU의 순차 모델링";
// news.bpdata.com, section "HSTU"): a SiLU projection of the input produces q, k, v and u, and
// the gated attention output goes through an output projection.  Both are A [M, K] times
// B [N, K]^T with B a weight matrix stored one output feature per row.
//
// One CTA per 128 x 128 output tile; 256 threads:
//   warp 0 lane 0   TMA producer: per 64-wide K step one A box and one B box (128 rows x 128
//                   bytes, 128-byte swizzle) into a 4-stage ring
//   warp 1          allocates 128 TMEM columns; lane 0 issues four M=128 N=128 K=16 MMAs per
//                   K step and frees the stage when they complete
//   warps 4-7       epilogue: warp w reads TMEM lanes 32(w%4).. (= output rows), 32 columns at
//                   a time, applies SiLU = x/2 (1 + tanh(x/2)) when asked, rounds to bf16 and
//                   writes 64 contiguous bytes per row and batch
// Output columns are split into blocks of `split` columns (a multiple of 128), block b going to
// out + b * block_stride: the projection's q, k, v and u land in four separate [M, H*D] arrays.
// Rows of A past M read as zeros (TMA bounds) and are not stored.  Every wait is bounded.
#include <atomic>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {
using namespace sm100;

namespace gm {

constexpr int kThreads = 256;
constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kStages = 4;
constexpr uint32_t kTileA = kBM * kBK * 2;             // 16 KB
constexpr uint32_t kTileB = kBN * kBK * 2;             // 16 KB
constexpr uint32_t kStageBytes = kTileA + kTileB;
constexpr uint32_t kOffBar = kStages * kStageBytes;
constexpr int kNumBars = 2 * kStages + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;       // room to align the base to 1024 bytes
constexpr uint32_t kTmemCols = 128;

static_assert(kOffBar % 8 == 0, "mbarrier alignment");

__global__ void __launch_bounds__(kThreads)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, const GemmArgs g)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_u32 & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw_u32 + pad;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int32_t m0 = (int32_t)blockIdx.x * kBM;
    const int32_t n0 = (int32_t)blockIdx.y * kBN;
    const int nk = g.K / kBK;

    if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < kStages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            mbar_init(acc_full, 1);
            *abort_flag = 0;
            fence_mbar_init();
        }
        __syncwarp();
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t tmo = g.timeout_ns, drain = g.drain_ns;
    // launched as a programmatic dependent of the previous kernel (g.pdl): the set-up above ran
    // early; A and the outputs are touched only after that kernel has finished (a no-op otherwise)
    pdl_launch_dependents();
    pdl_wait_primary();

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        int issued = 0;
        for (int kt = 0; kt < nk; ++kt) {
            const int st = kt % kStages;
            if (kt >= kStages && !mbar_wait(&empty[st], ((kt / kStages) & 1) ^ 1, abort_flag, tmo))
                break;
            const uint32_t sa = sbase + st * kStageBytes;
            mbar_arrive_expect_tx(&full[st], kStageBytes);
            tma_load_2d(&tm_a, sa, &full[st], kt * kBK, m0);
            tma_load_2d(&tm_b, sa + kTileA, &full[st], kt * kBK, n0);
            issued = kt + 1;
        }
        volatile int never = 0;
        for (int kt = (issued > kStages ? issued - kStages : 0); kt < issued; ++kt)
            mbar_wait(&full[kt % kStages], (kt / kStages) & 1, &never, drain);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
        for (int kt = 0; kt < nk; ++kt) {
            const int st = kt % kStages;
            if (!mbar_wait(&full[st], (kt / kStages) & 1, abort_flag, tmo))
                break;
            tc_fence_after();
            const uint32_t sa = sbase + st * kStageBytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                // K-major operands, 128-byte rows: a K step of 16 elements is 32 bytes into the row
                const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(sa + kTileA + kk * 32, 16, 1024);
                umma_bf16_ss(tmem, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&empty[st]);
        }
        umma_commit(acc_full);
        volatile int never = 0;
        mbar_wait(acc_full, 0, &never, drain);
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const bool ok = mbar_wait_warp(acc_full, 0, abort_flag, tmo);
        if (ok && !*abort_flag) {
            tc_fence_after();
            const int r = ((warp & 3) << 5) + lane;
            const int32_t m = m0 + r;
            const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;
            const int32_t blk = n0 / g.split;
            const int32_t col0 = n0 - blk * g.split;
            __nv_bfloat16* orow = g.out + (int64_t)blk * g.block_stride + (int64_t)m * g.ldo + col0;
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + lane_base + c0, v);
                tmem_wait_ld();
                uint32_t packed[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float x0 = __uint_as_float(v[2 * e]), x1 = __uint_as_float(v[2 * e + 1]);
                    if (g.silu) {
                        const float h0 = 0.5f * x0, h1 = 0.5f * x1;
                        x0 = h0 + h0 * tanh_approx(h0);
                        x1 = h1 + h1 * tanh_approx(h1);
                    }
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                    packed[e] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                if (m < g.M) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag && g.ws)
        set_flag(g.ws, HSTU_DEV_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace gm

void launch_gemm_bf16(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmArgs& g, cudaStream_t stream)
{
    if (g.M <= 0 || g.N <= 0)
        return;
    static std::atomic<uint32_t> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaFuncSetAttribute(gm::gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gm::kSmemBytes);
        if (dev >= 0 && dev < 64)
            attr_set[dev].store(1, std::memory_order_relaxed);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((g.M + gm::kBM - 1) / gm::kBM), (unsigned)(g.N / gm::kBN), 1);
    cfg.blockDim = dim3(gm::kThreads, 1, 1);
    cfg.dynamicSmemBytes = gm::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g.pdl ? 1 : 0;
    cudaLaunchKernelEx(&cfg, gm::gemm_bf16_kernel, tm_a, tm_b, g);
}

}  // namespace hstu
