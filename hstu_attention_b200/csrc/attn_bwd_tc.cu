// attn_bwd_tc.cu -- backward pass of jagged HSTU attention on Blackwell tensor cores (bf16
// operands, fp32 accumulation, D = 128).
//
// The gradients (chain rule through the forward definition; per user b, head h and allowed pair
// (query i, key j), s = q_i . k_j + rab[h][bucket(i - j)], sig = sigmoid(s)):
//     P_ij  = s sig / n_max                        (the forward weight)
//     dP_ij = do_i . v_j
//     dS_ij = dP_ij sig (1 + s (1 - sig)) / n_max
//     dq_i = sum_j dS_ij k_j,   dk_j = sum_i dS_ij q_i,   dv_j = sum_i P_ij do_i,
//     drab[h][bucket(i - j)] += dS_ij
// SiLU weighting instead of softmax (aitrends.kr summary, section "HSTU의 순차 모델링";
// news.bpdata.com, section "HSTU") means every pair's weight depends on that pair alone: no row
// statistics, so both kernels below recompute S tile by tile and need nothing else.
//
// bwd_dq_kernel   one CTA per (user, head, 128-query block), grid and order as the forward:
//                 per key tile  S = Q K^T (tcgen05, A = Q copied into TMEM once) and dP = dO V^T
//                 (tcgen05, SS), pointwise dS -> bf16 in TMEM, dQ += dS K (tcgen05, A = dS from
//                 TMEM, B = the K tile read MN-major); the next tile's S and dP are issued as soon
//                 as the pointwise warps hold this tile's in registers.  drab: dS summed along the
//                 tile's 255 diagonals (a shuffle reduction per 32 x 32 block into per-warp arrays,
//                 two buffers), folded by warp 3 into per-CTA bucket sums (runs of equal buckets
//                 summed across lanes first), one global atomic per bucket at the end.
// bwd_dkv_kernel  one CTA per (user, head, 128-key block), the blocks with most queries first:
//                 per query tile the transposed products S^T = K Q^T and dP^T = V dO^T, pointwise
//                 P^T and dS^T -> bf16 in TMEM (written over the S^T / dP^T columns already read),
//                 dV += P^T dO and dK += dS^T Q (A from TMEM, B = the dO / Q tile read MN-major);
//                 products and pointwise stage alternate per tile (TMEM is full).
// Every wait is bounded (HSTU_DEV_TIMEOUT).
//
// CTA roles (384 threads): warp 0 lane 0 TMA producer; warp 1 allocates all 512 TMEM columns and
// lane 0 issues the MMAs; warp 2 builds each tile's bias window (255 values rab[h][bucket(i-j)],
// eight per lane with interleaved binary searches; for the dQ kernel also the bucket index per
// diagonal) into a two-slot ring; warp 3 (dQ kernel) folds the diagonal sums; warps 4-11
// pointwise and epilogue (warpgroup g owns tile columns [64g, 64g + 64), warp w%4 owns TMEM lanes
// [32(w%4), +32)), with no barrier among them inside the tile loop.
#include <atomic>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {
using namespace sm100;

namespace bt {

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kThreads = 384;
constexpr int kMaxNB = 1024;
constexpr uint32_t kHalf = 128 * 128;           // 128 rows x 128 bytes
constexpr uint32_t kTileBytes = 2 * kHalf;      // a 128 x 128 bf16 operand
// shared memory: two fixed operands (Q, dO or K, V), a 2-stage ring of operand pairs, the
// window area (a two-slot ring of bias windows and bucket indices), diagonal sums (buffer 0;
// buffer 1 of the dQ kernel reuses the Q tile's space), bucket sums, bounds, rab
constexpr uint32_t kOffFix0 = 0;
constexpr uint32_t kOffFix1 = kTileBytes;
constexpr uint32_t kOffRing = 2 * kTileBytes;                // 2 stages x 2 operands
constexpr uint32_t kStageBytes = 2 * kTileBytes;
constexpr uint32_t kWinPad = 4;
constexpr uint32_t kWinStride = 264;
constexpr uint32_t kOffWin = kOffRing + 2 * kStageBytes;
constexpr uint32_t kOffWinK = kOffWin + 4 * kWinStride * 4;  // bucket index per window position
constexpr uint32_t kOffDiag = kOffWinK + 256 * 4;           // [8 pointwise warps][256] diagonal sums
constexpr uint32_t kOffBsum = kOffDiag + 8 * 256 * 4;
constexpr uint32_t kOffBounds = kOffBsum + kMaxNB * 4;
constexpr uint32_t kOffRab = kOffBounds + (kMaxNB + 4) * 4;
constexpr uint32_t kOffBar = kOffRab + kMaxNB * 4;
// fix, ring full/empty, sp_full, pd_full, pd_empty, acc, sp_empty; the dQ kernel adds qt_full,
// win_full/empty [2] and diag_full/empty [2]
constexpr int kNumBars = 1 + 2 + 2 + 1 + 1 + 1 + 1 + 1 + 1 + 2 + 2 + 2 + 2;
// dQ kernel: bias windows in a two-slot ring (one copy each, then the bucket index per position)
constexpr uint32_t kWinSlotFloats = 264;                    // pad + 256 + 4
constexpr uint32_t kWinSlotBytes = kWinSlotFloats * 4 + 256 * 4;
static_assert(2 * kWinSlotBytes <= kOffDiag - kOffWin, "window ring fits the window area");
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
constexpr uint32_t kTmemCols = 512;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");

__device__ int bucket_bound_bt(int k, double ln_nmax, int nb)
{
    if (nb <= 1 || !(ln_nmax > 0.0))
        return 0x7fffffff;
    if (k == 1)
        return 1;
    double root = exp((double)(k - 1) * ln_nmax / (double)(nb - 1));
    int64_t c = (int64_t)ceil(root);
    if (c < 1)
        c = 1;
    for (int it = 0; it < 8 && c > 1 && bucket_of(c - 1, ln_nmax, nb) >= k; ++it)
        --c;
    for (int it = 0; it < 8 && bucket_of(c, ln_nmax, nb) < k; ++it)
        ++c;
    return c > 0x7ffffffe ? 0x7ffffffe : (int)c;
}

// per-element gradient pieces from s (bias included) and dP; returns dS and writes P
__device__ __forceinline__ float pair_terms(float s, float dp, float inv_n, float& p)
{
    const float sig = 0.5f + 0.5f * tanh_approx(0.5f * s);
    p = s * sig * inv_n;
    return dp * sig * (1.0f + s * (1.0f - sig)) * inv_n;
}

struct Smem {
    uint8_t* base;
    uint32_t sbase;
    uint64_t *fix_full, *ring_full, *ring_empty, *sp_full, *sp_empty, *pd_full, *pd_empty, *acc_full;
    uint64_t *qt_full, *win_full, *win_empty, *diag_full, *diag_empty;    // dQ kernel
    uint32_t* tmem_slot;
    volatile int* abort_flag;
    float* diag;
    float* bsum;
    int32_t* bounds;
    float* rab;
};

__device__ __forceinline__ Smem carve(uint8_t* smem_raw)
{
    Smem m;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    m.base = smem_raw + pad;
    m.sbase = raw + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(m.base + kOffBar);
    m.fix_full = bars;
    m.ring_full = bars + 1;
    m.ring_empty = bars + 3;
    m.sp_full = bars + 5;
    m.pd_full = bars + 6;
    m.pd_empty = bars + 7;
    m.acc_full = bars + 8;
    m.sp_empty = bars + 9;
    m.qt_full = bars + 10;
    m.win_full = bars + 11;
    m.win_empty = bars + 13;
    m.diag_full = bars + 15;
    m.diag_empty = bars + 17;
    m.tmem_slot = reinterpret_cast<uint32_t*>(m.base + kOffMisc);
    m.abort_flag = reinterpret_cast<volatile int*>(m.base + kOffMisc + 4);
    m.diag = reinterpret_cast<float*>(m.base + kOffDiag);
    m.bsum = reinterpret_cast<float*>(m.base + kOffBsum);
    m.bounds = reinterpret_cast<int32_t*>(m.base + kOffBounds);
    m.rab = reinterpret_cast<float*>(m.base + kOffRab);
    return m;
}

// barrier init (thread 0) and TMEM allocation (warp 1), then a CTA barrier
// roles: 1 = the dQ kernel (window ring read by the pointwise warps and the fold warp, diagonal
// buffers, Q in TMEM), 2 = the dK/dV kernel (window ring read by the pointwise warps)
__device__ __forceinline__ uint32_t setup(const Smem& m, int warp, int roles)
{
    if (threadIdx.x == 0) {
        if (roles == 1)
            mbar_init(m.qt_full, 128);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m.win_full[s], 32);
            mbar_init(&m.win_empty[s], roles == 1 ? 256 + 32 : 256);
            if (roles == 1) {
                mbar_init(&m.diag_full[s], 256);
                mbar_init(&m.diag_empty[s], 32);
            }
        }
        mbar_init(m.fix_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m.ring_full[s], 1);
            mbar_init(&m.ring_empty[s], 1);
        }
        mbar_init(m.sp_full, 1);
        mbar_init(m.sp_empty, 256);
        mbar_init(m.pd_full, 256);
        mbar_init(m.pd_empty, 1);
        mbar_init(m.acc_full, 1);
        *m.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(m.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *m.tmem_slot;
}

__device__ __forceinline__ void teardown(const Smem& m, int warp, uint32_t tmem, void* ws)
{
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *m.abort_flag)
        set_flag(ws, HSTU_DEV_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// rab[h] and the bucket bounds into shared memory (the 256 pointwise threads), zeroed sums
__device__ __forceinline__ void stage_bias(const Smem& m, const BwdTcArgs& a, const BucketBounds& bb, int h, int pt)
{
    for (int k = pt; k < a.NB; k += 256) {
        m.rab[k] = a.rab[(int64_t)h * a.NB + k];
        m.bsum[k] = 0.f;
    }
    for (int k = pt; k <= a.NB; k += 256)
        m.bounds[k] = bb.count > 0 ? bb.v[k]
                                   : (k == 0 ? 0 : (k == a.NB ? 0x7fffffff : bucket_bound_bt(k, a.ln_nmax, a.NB)));
    for (int x = pt; x < 8 * 256; x += 256)
        m.diag[x] = 0.f;
}

// ============================================================================ dQ and drab
__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ BucketBounds bb, const BwdTcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x % a.H;
    const int b = blockIdx.x / a.H;
    const int qblk = a.qblocks - 1 - (int)blockIdx.y;
    const UserGeom g = jagged_geom(a.seq_offsets, a.num_targets, b, a.total_tokens, a.max_len, a.n_max);
    const int64_t HD = (int64_t)a.H * kD;
    const int32_t qrow0 = qblk * kTile;
    if (!g.ok) {
        // a rejected user: zero gradients (the q-block-0 CTA of each head clears its dq slice)
        if (qblk == 0) {
            if (h == 0 && threadIdx.x == 0)
                set_flag(a.ws, g.flags);
            for (int64_t x = threadIdx.x; x < (int64_t)g.N * (kD / 4); x += kThreads) {
                const int64_t r = x / (kD / 4);
                const int c4 = (int)(x % (kD / 4));
                reinterpret_cast<float4*>(a.dq + (g.tok0 + r) * HD + (int64_t)h * kD)[c4] =
                    make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        return;
    }
    if (qrow0 >= g.N)
        return;
    const int32_t last_q = min(g.N, qrow0 + kTile) - 1;
    const int n = last_q / kTile + 1;                 // key tiles 0 .. n - 1 (keys up to last_q)

    const Smem m = carve(smem_raw);
    const uint32_t tmem = setup(m, warp, 1);
    const uint64_t tmo = a.timeout_ns, drain = a.drain_ns;
    // TMEM: S [0,128) | dP [128,256) | dQ [256,384) | dS bf16 [384,448) | Q bf16 [448,512)
    constexpr uint32_t cS = 0, cDP = 128, cDQ = 256, cDS = 384, cQ = 448;
    // diagonal sums of tile t go to buffer t & 1: buffer 0 in its own area, buffer 1 in the Q
    // tile's space once Q has been copied into TMEM
    float* const diag_buf[2] = {m.diag, reinterpret_cast<float*>(m.base + kOffFix0)};

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        mbar_arrive_expect_tx(m.fix_full, 2 * kTileBytes);
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(&tm_q, m.sbase + kOffFix0 + hf * kHalf, m.fix_full, hf * 64, h, (int32_t)(g.tok0 + qrow0));
            tma_load_3d(&tm_do, m.sbase + kOffFix1 + hf * kHalf, m.fix_full, hf * 64, h, (int32_t)(g.tok0 + qrow0));
        }
        int issued = 0;
        for (int t = 0; t < n; ++t) {
            const int st = t & 1;
            if (t >= 2 && !mbar_wait(&m.ring_empty[st], ((t >> 1) & 1) ^ 1, m.abort_flag, tmo))
                break;
            const uint32_t dst = m.sbase + kOffRing + st * kStageBytes;
            mbar_arrive_expect_tx(&m.ring_full[st], kStageBytes);
            const int32_t row = (int32_t)(g.tok0 + t * kTile);
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_3d(&tm_k, dst + hf * kHalf, &m.ring_full[st], hf * 64, h, row);
                tma_load_3d(&tm_v, dst + kTileBytes + hf * kHalf, &m.ring_full[st], hf * 64, h, row);
            }
            issued = t + 1;
        }
        volatile int never = 0;
        mbar_wait(m.fix_full, 0, &never, drain);
        for (int t = (issued > 2 ? issued - 2 : 0); t < issued; ++t)
            mbar_wait(&m.ring_full[t & 1], (t >> 1) & 1, &never, drain);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_kmaj = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idesc_ts = idesc_bf16_f32(128, 128, 0, 1);
        bool ok = mbar_wait(m.fix_full, 0, m.abort_flag, tmo) && mbar_wait(m.qt_full, 0, m.abort_flag, tmo);
        // S(t) = Q K_t^T (A = Q from TMEM) and dP(t) = dO V_t^T (both operands in shared memory)
        auto issue_sdp = [&](int t) -> bool {
            const int st = t & 1;
            const uint32_t kb = m.sbase + kOffRing + st * kStageBytes;
            const uint32_t vb = kb + kTileBytes;
            if (!mbar_wait(&m.ring_full[st], (t >> 1) & 1, m.abort_flag, tmo))
                return false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kHalf + (kk & 3) * 32;
                umma_bf16_ts(tmem + cS, tmem + cQ + kk * 8, smem_desc_sw128(kb + ko, 16, 1024), idesc_kmaj,
                             kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kHalf + (kk & 3) * 32;
                umma_bf16_ss(tmem + cDP, smem_desc_sw128(m.sbase + kOffFix1 + ko, 16, 1024),
                             smem_desc_sw128(vb + ko, 16, 1024), idesc_kmaj, kk > 0 ? 1u : 0u);
            }
            umma_commit(m.sp_full);
            return true;
        };
        if (ok && n > 0)
            ok = issue_sdp(0);
        for (int t = 0; ok && t < n; ++t) {
            const int st = t & 1;
            const uint32_t kb = m.sbase + kOffRing + st * kStageBytes;
            // the pointwise warps have S(t) and dP(t) in registers: the next tile's products may
            // overwrite those columns while they compute dS(t)
            if (t + 1 < n) {
                if (!mbar_wait(m.sp_empty, t & 1, m.abort_flag, tmo) || !issue_sdp(t + 1)) {
                    ok = false;
                    break;
                }
            }
            // dQ += dS(t) K_t: A = dS (keys = K dimension, in TMEM), B = the K tile read MN-major;
            // it runs while the pointwise warps work on tile t + 1
            if (!mbar_wait(m.pd_full, t & 1, m.abort_flag, tmo)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma_bf16_ts(tmem + cDQ, tmem + cDS + kk * 8, smem_desc_sw128(kb + kk * 2048, kHalf, 1024), idesc_ts,
                             (t > 0 || kk > 0) ? 1u : 0u);
            umma_commit(m.pd_empty);
            umma_commit(&m.ring_empty[st]);
        }
        umma_commit(m.acc_full);
        volatile int never = 0;
        mbar_wait(m.acc_full, 0, &never, drain);
    } else if (warp == 2) {
        // ------------------------------------------------------------ bias windows
        // window t (slot t & 1): position y = 127 - r + c of query row r and key column c has
        // distance d = i - j = (qrow0 - j0 + 127) - y; value rab[bucket(d)] (0 for d < 0 or
        // y > 254) and the bucket index (-1 there) for the fold.  Eight positions per lane, their
        // binary searches interleaved.
        named_barrier_sync(2, 320);                        // bounds and rab staged
        const int nb = a.NB;
        int top = 1;
        while (top * 2 <= nb)
            top *= 2;
        for (int t = 0; t < n; ++t) {
            const int sl = t & 1;
            if (t >= 2 && !mbar_wait_warp(&m.win_empty[sl], ((t >> 1) & 1) ^ 1, m.abort_flag, tmo))
                break;
            float* win = reinterpret_cast<float*>(m.base + kOffWin + sl * kWinSlotBytes);
            int32_t* wk = reinterpret_cast<int32_t*>(m.base + kOffWin + sl * kWinSlotBytes + kWinSlotFloats * 4);
            const int32_t dist0 = qrow0 - t * kTile + (kTile - 1);
            int k[8];
            int32_t d[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                d[e] = dist0 - (lane + 32 * e);
                k[e] = 0;
            }
            for (int step = top; step > 0; step >>= 1) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    k[e] += (m.bounds[min(k[e] + step, nb)] <= d[e]) ? step : 0;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int y = lane + 32 * e;
                const bool live = (y <= 2 * kTile - 2) && d[e] >= 0;
                win[kWinPad + y] = live ? m.rab[k[e]] : 0.f;
                wk[y] = live ? k[e] : -1;
            }
            mbar_arrive(&m.win_full[sl]);
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ drab fold
        // tile t's diagonal sums (buffer t & 1, one array per pointwise warp) into the bucket
        // sums, then the buffer is cleared for tile t + 2; one global atomic per bucket at the end
        named_barrier_sync(2, 320);                        // bucket sums zeroed
        bool ok = true;
        for (int t = 0; ok && t < n; ++t) {
            const int sl = t & 1;
            ok = mbar_wait_warp(&m.diag_full[sl], (t >> 1) & 1, m.abort_flag, tmo);
            if (!ok)
                break;
            float* db = diag_buf[sl];
            const int32_t* wk =
                reinterpret_cast<const int32_t*>(m.base + kOffWin + sl * kWinSlotBytes + kWinSlotFloats * 4);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int y = lane + 32 * e;
                const bool live = y <= 2 * kTile - 2;
                float v = 0.f;
                if (live) {
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        v += db[w * 256 + y];
                        db[w * 256 + y] = 0.f;
                    }
                }
                const int kb = live ? wk[y] : -1;
                // buckets do not increase along y, so equal buckets are runs of lanes: a suffix
                // sum within each run leaves the run's total in its first lane, which alone
                // adds it to the bucket (one shared atomic per run instead of one per lane)
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float vo = __shfl_down_sync(0xffffffffu, v, o);
                    const int ko = __shfl_down_sync(0xffffffffu, kb, o);
                    if (lane + o < 32 && ko == kb)
                        v += vo;
                }
                const int kprev = __shfl_up_sync(0xffffffffu, kb, 1);
                if (kb >= 0 && (lane == 0 || kprev != kb) && v != 0.f)
                    atomicAdd(&m.bsum[kb], v);
            }
            __syncwarp();
            mbar_arrive(&m.diag_empty[sl]);
            mbar_arrive(&m.win_empty[sl]);
        }
        __syncwarp();
        if (ok)
            for (int k = lane; k < a.NB; k += 32)
                if (m.bsum[k] != 0.f)
                    atomicAdd(&a.drab[(int64_t)h * a.NB + k], m.bsum[k]);
    } else if (warp >= 4) {
        // ------------------------------------------------------------ pointwise + epilogue
        const int pt = threadIdx.x - 128;
        stage_bias(m, a, bb, h, pt);
        named_barrier_sync(2, 320);
        const int wg = (warp - 4) >> 2;
        const int r = ((warp & 3) << 5) + lane;            // query row (= TMEM lane)
        const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;
        const int32_t i = qrow0 + r;                       // query position
        const bool row_valid = i < g.N;
        const int32_t lim = row_valid ? min(i + 1, g.hist) : -1;   // keys j < lim are visible, and j == i
        const int32_t diag_key = row_valid ? i : -1;
        const float inv_n = a.inv_n;
        bool ok = true;
        if (wg == 0) {
            // Q into TMEM for the Q K^T products: row r of the tile (128-byte swizzle: the 16-byte
            // chunk c of a row sits at chunk c ^ (r & 7)) goes to lane r, channels (2c, 2c+1) to
            // column c; then the tile's space is cleared for diagonal buffer 1
            ok = __all_sync(0xffffffffu, mbar_wait(m.fix_full, 0, m.abort_flag, tmo));
            if (ok) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint8_t* qrow = m.base + kOffFix0 + hf * kHalf + r * 128;
                    uint32_t qv[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 x = *reinterpret_cast<const uint4*>(qrow + ((c ^ (r & 7)) << 4));
                        qv[4 * c] = x.x;
                        qv[4 * c + 1] = x.y;
                        qv[4 * c + 2] = x.z;
                        qv[4 * c + 3] = x.w;
                    }
                    tmem_st_32x32b_x32(tmem + lane_base + cQ + hf * 32, qv);
                }
                tmem_wait_st();
            }
            named_barrier_sync(5, 128);                    // every row of Q has been read
            for (int x = pt; x < 8 * 256; x += 128)
                diag_buf[1][x] = 0.f;
            tc_fence_before();
            mbar_arrive(m.qt_full);
        }
        // diagonal buffer 1 is cleared and Q is in TMEM
        ok = ok && mbar_wait_warp(m.qt_full, 0, m.abort_flag, tmo);
        for (int t = 0; t < n; ++t) {
            const int32_t j0 = t * kTile;
            const int sl = t & 1;
            ok = ok && mbar_wait_warp(&m.win_full[sl], (t >> 1) & 1, m.abort_flag, tmo) &&
                 mbar_wait_warp(m.sp_full, t & 1, m.abort_flag, tmo);
            if (ok && t >= 2)
                ok = mbar_wait_warp(&m.diag_empty[sl], ((t >> 1) & 1) ^ 1, m.abort_flag, tmo);
            if (ok) {
                tc_fence_after();
                const float* win = reinterpret_cast<const float*>(m.base + kOffWin + sl * kWinSlotBytes);
                float* wdiag = diag_buf[sl] + (warp - 4) * 256;
                const int y0 = (kTile - 1) - r + 64 * wg;
#pragma unroll 1
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    uint32_t sv[32], dv[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + cS + 64 * wg + c0, sv);
                    tmem_ld_32x32b_x32(tmem + lane_base + cDP + 64 * wg + c0, dv);
                    tmem_wait_ld();
                    if (c0 == 32) {
                        // S(t) and dP(t) are in registers: the next tile's products may start
                        tc_fence_before();
                        mbar_arrive(m.sp_empty);
                    } else if (t >= 1) {
                        // dS(t - 1) must have been read by its dQ product before dS(t) is written
                        ok = mbar_wait_warp(m.pd_empty, (t - 1) & 1, m.abort_flag, tmo);
                        tc_fence_after();
                    }
                    uint32_t packed[16];
                    float dsv[32];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int c = 64 * wg + c0 + e + q;
                            const int32_t j = j0 + c;
                            const int y = y0 + c0 + e + q;
                            const float s = __uint_as_float(sv[e + q]) + win[kWinPad + y];
                            float p;
                            const float ds = pair_terms(s, __uint_as_float(dv[e + q]), inv_n, p);
                            const bool allowed = (j < lim) | (j == diag_key);
                            dsv[e + q] = allowed ? ds : 0.f;
                        }
                        const __nv_bfloat162 bb2 = __floats2bfloat162_rn(dsv[e], dsv[e + 1]);
                        packed[e >> 1] = *reinterpret_cast<const uint32_t*>(&bb2);
                    }
                    // diagonal sums of this warp's 32 x 32 block: element (lane, k) lies on diagonal
                    // Y0 - lane + k.  At step k lane l takes element k of lane (l + k) % 32, which lies
                    // on diagonal Y0 - l (no wrap) or Y0 - l + 32 (wrap), so every lane ends with two
                    // diagonal sums; the lanes' targets are all distinct, in this batch and the next
                    {
                        const int Y0 = (kTile - 1) - ((warp & 3) << 5) + 64 * wg + c0;
                        float lo = 0.f, hi = 0.f;
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const float v = __shfl_sync(0xffffffffu, dsv[k], (lane + k) & 31);
                            const bool wrap = lane + k >= 32;
                            lo += wrap ? 0.f : v;
                            hi += wrap ? v : 0.f;
                        }
                        wdiag[Y0 - lane] += lo;
                        wdiag[Y0 - lane + 32] += hi;
                    }
                    __syncwarp();
                    tmem_st_32x32b_x16(tmem + lane_base + cDS + 32 * wg + (c0 >> 1), packed);
                }
            }
            __syncwarp();
            tmem_wait_st();
            if (ok) {
                tc_fence_before();
                mbar_arrive(m.pd_full);
                mbar_arrive(&m.diag_full[sl]);             // this tile's diagonal sums are complete
                mbar_arrive(&m.win_empty[sl]);             // and its window has been read
            }
        }
        // ------------------------------------------------------------ epilogue
        // tcgen05.ld is a warp-wide instruction: every lane loads, only the rows of queries store
        ok = ok && mbar_wait_warp(m.acc_full, 0, m.abort_flag, tmo);
        if (ok) {
            tc_fence_after();
            float* dst = a.dq + (g.tok0 + i) * HD + (int64_t)h * kD + 64 * wg;
#pragma unroll 1
            for (int c0 = 0; c0 < 64; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + lane_base + cDQ + 64 * wg + c0, v);
                tmem_wait_ld();
                if (row_valid) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        reinterpret_cast<float4*>(dst + c0)[q] =
                            make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                        __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                }
                __syncwarp();
            }
        }
    }
    teardown(m, warp, tmem, a.ws);
}

// ============================================================================ dK and dV
__global__ void __launch_bounds__(kThreads, 1)
bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ BucketBounds bb, const BwdTcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x % a.H;
    const int b = blockIdx.x / a.H;
    const int kblk = (int)blockIdx.y;                 // most queries first
    const UserGeom g = jagged_geom(a.seq_offsets, a.num_targets, b, a.total_tokens, a.max_len, a.n_max);
    const int64_t HD = (int64_t)a.H * kD;
    const int32_t j0 = kblk * kTile;
    if (!g.ok) {
        if (kblk == 0)
            for (int64_t x = threadIdx.x; x < (int64_t)g.N * (kD / 4); x += kThreads) {
                const int64_t r = x / (kD / 4);
                const int c4 = (int)(x % (kD / 4));
                const int64_t o = (g.tok0 + r) * HD + (int64_t)h * kD;
                reinterpret_cast<float4*>(a.dk + o)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
                reinterpret_cast<float4*>(a.dv + o)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        return;
    }
    if (j0 >= g.N)
        return;
    const int nq_tiles = (g.N + kTile - 1) / kTile;
    const int t0 = kblk;                              // query tiles t0 .. nq_tiles - 1 see these keys
    const int n = nq_tiles - t0;

    const Smem m = carve(smem_raw);
    const uint32_t tmem = setup(m, warp, 2);
    const uint64_t tmo = a.timeout_ns, drain = a.drain_ns;
    // TMEM: S^T [0,128) (P^T bf16 written over it) | dP^T [128,256) (dS^T over it) | dV | dK
    constexpr uint32_t cS = 0, cDP = 128, cDV = 256, cDK = 384;

    if (warp == 0 && lane == 0) {
        mbar_arrive_expect_tx(m.fix_full, 2 * kTileBytes);
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(&tm_k, m.sbase + kOffFix0 + hf * kHalf, m.fix_full, hf * 64, h, (int32_t)(g.tok0 + j0));
            tma_load_3d(&tm_v, m.sbase + kOffFix1 + hf * kHalf, m.fix_full, hf * 64, h, (int32_t)(g.tok0 + j0));
        }
        int issued = 0;
        for (int t = 0; t < n; ++t) {
            const int st = t & 1;
            if (t >= 2 && !mbar_wait(&m.ring_empty[st], ((t >> 1) & 1) ^ 1, m.abort_flag, tmo))
                break;
            const uint32_t dst = m.sbase + kOffRing + st * kStageBytes;
            mbar_arrive_expect_tx(&m.ring_full[st], kStageBytes);
            const int32_t row = (int32_t)(g.tok0 + (t0 + t) * kTile);
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_3d(&tm_q, dst + hf * kHalf, &m.ring_full[st], hf * 64, h, row);
                tma_load_3d(&tm_do, dst + kTileBytes + hf * kHalf, &m.ring_full[st], hf * 64, h, row);
            }
            issued = t + 1;
        }
        volatile int never = 0;
        mbar_wait(m.fix_full, 0, &never, drain);
        for (int t = (issued > 2 ? issued - 2 : 0); t < issued; ++t)
            mbar_wait(&m.ring_full[t & 1], (t >> 1) & 1, &never, drain);
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t idesc_ss = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idesc_ts = idesc_bf16_f32(128, 128, 0, 1);
        bool ok = mbar_wait(m.fix_full, 0, m.abort_flag, tmo);
        for (int t = 0; ok && t < n; ++t) {
            const int st = t & 1;
            const uint32_t qb = m.sbase + kOffRing + st * kStageBytes;
            const uint32_t ob = qb + kTileBytes;
            if (!mbar_wait(&m.ring_full[st], (t >> 1) & 1, m.abort_flag, tmo)) {
                ok = false;
                break;
            }
            // the previous tile's dV / dK products read P^T and dS^T from these columns
            if (t >= 1 && !mbar_wait(m.pd_empty, (t - 1) & 1, m.abort_flag, tmo)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kHalf + (kk & 3) * 32;
                umma_bf16_ss(tmem + cS, smem_desc_sw128(m.sbase + kOffFix0 + ko, 16, 1024),
                             smem_desc_sw128(qb + ko, 16, 1024), idesc_ss, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * kHalf + (kk & 3) * 32;
                umma_bf16_ss(tmem + cDP, smem_desc_sw128(m.sbase + kOffFix1 + ko, 16, 1024),
                             smem_desc_sw128(ob + ko, 16, 1024), idesc_ss, kk > 0 ? 1u : 0u);
            }
            umma_commit(m.sp_full);
            if (!mbar_wait(m.pd_full, t & 1, m.abort_flag, tmo)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // dV += P^T dO and dK += dS^T Q: K dimension = the tile's queries; warpgroup g wrote
            // queries [64g, 64g + 64) at columns [64g, 64g + 32) of its region
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
                umma_bf16_ts(tmem + cDV, tmem + cS + acol, smem_desc_sw128(ob + kk * 2048, kHalf, 1024), idesc_ts,
                             (t > 0 || kk > 0) ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
                umma_bf16_ts(tmem + cDK, tmem + cDP + acol, smem_desc_sw128(qb + kk * 2048, kHalf, 1024), idesc_ts,
                             (t > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(m.pd_empty);
            umma_commit(&m.ring_empty[st]);
        }
        umma_commit(m.acc_full);
        volatile int never = 0;
        mbar_wait(m.acc_full, 0, &never, drain);
    } else if (warp == 2) {
        // ------------------------------------------------------------ bias windows
        // window t (slot t & 1): position y = 127 - r + c of key row r and query column c has
        // distance d = i - j = (i0 - j0 - 127) + y; value rab[bucket(d)] (0 for d < 0 or
        // y > 254).  Eight positions per lane, their binary searches interleaved.
        named_barrier_sync(2, 288);                        // bounds and rab staged
        const int nb = a.NB;
        int top = 1;
        while (top * 2 <= nb)
            top *= 2;
        for (int t = 0; t < n; ++t) {
            const int sl = t & 1;
            if (t >= 2 && !mbar_wait_warp(&m.win_empty[sl], ((t >> 1) & 1) ^ 1, m.abort_flag, tmo))
                break;
            float* win = reinterpret_cast<float*>(m.base + kOffWin + sl * kWinSlotBytes);
            const int32_t dist0 = (t0 + t) * kTile - j0 - (kTile - 1);
            int k[8];
            int32_t d[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                d[e] = dist0 + (lane + 32 * e);
                k[e] = 0;
            }
            for (int step = top; step > 0; step >>= 1) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    k[e] += (m.bounds[min(k[e] + step, nb)] <= d[e]) ? step : 0;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int y = lane + 32 * e;
                win[kWinPad + y] = ((y <= 2 * kTile - 2) && d[e] >= 0) ? m.rab[k[e]] : 0.f;
            }
            mbar_arrive(&m.win_full[sl]);
        }
    } else if (warp >= 4) {
        const int pt = threadIdx.x - 128;
        stage_bias(m, a, bb, h, pt);
        named_barrier_sync(2, 288);
        const int wg = (warp - 4) >> 2;
        const int r = ((warp & 3) << 5) + lane;            // key row (= TMEM lane)
        const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;
        const int32_t j = j0 + r;                          // key position
        const bool key_valid = j < g.N;
        // query i sees key j when (j < hist and i >= j) or i == j
        const int32_t lo = (key_valid && j < g.hist) ? j : 0x7fffffff;
        const int32_t self = key_valid ? j : -1;
        const float inv_n = a.inv_n;
        bool ok = true;
        for (int t = 0; t < n; ++t) {
            const int32_t i0 = (t0 + t) * kTile;
            const int sl = t & 1;
            ok = ok && mbar_wait_warp(&m.win_full[sl], (t >> 1) & 1, m.abort_flag, tmo) &&
                 mbar_wait_warp(m.sp_full, t & 1, m.abort_flag, tmo);
            if (ok) {
                tc_fence_after();
                const float* win = reinterpret_cast<const float*>(m.base + kOffWin + sl * kWinSlotBytes);
                const int y0 = (kTile - 1) - r + 64 * wg;
#pragma unroll 1
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    uint32_t sv[32], dv[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + cS + 64 * wg + c0, sv);
                    tmem_ld_32x32b_x32(tmem + lane_base + cDP + 64 * wg + c0, dv);
                    tmem_wait_ld();
                    uint32_t pk[16], dk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float p2[2], ds2[2];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int c = 64 * wg + c0 + e + q;
                            const int32_t i = i0 + c;
                            const int y = y0 + c0 + e + q;
                            const float s = __uint_as_float(sv[e + q]) + win[kWinPad + y];
                            float p;
                            const float ds = pair_terms(s, __uint_as_float(dv[e + q]), inv_n, p);
                            const bool allowed = (i < g.N) & ((i >= lo) | (i == self));
                            p2[q] = allowed ? p : 0.f;
                            ds2[q] = allowed ? ds : 0.f;
                        }
                        const __nv_bfloat162 pp = __floats2bfloat162_rn(p2[0], p2[1]);
                        const __nv_bfloat162 dd = __floats2bfloat162_rn(ds2[0], ds2[1]);
                        pk[e >> 1] = *reinterpret_cast<const uint32_t*>(&pp);
                        dk[e >> 1] = *reinterpret_cast<const uint32_t*>(&dd);
                    }
                    // over columns this thread has already read (its own lane, its own half)
                    __syncwarp();
                    tmem_st_32x32b_x16(tmem + lane_base + cS + 64 * wg + (c0 >> 1), pk);
                    tmem_st_32x32b_x16(tmem + lane_base + cDP + 64 * wg + (c0 >> 1), dk);
                }
            }
            __syncwarp();
            tmem_wait_st();
            if (ok) {
                tc_fence_before();
                mbar_arrive(m.pd_full);
                mbar_arrive(&m.win_empty[sl]);             // this tile's window has been read
            }
        }
        // warp-wide TMEM loads, per-lane stores (only the rows of keys of the user)
        ok = ok && mbar_wait_warp(m.acc_full, 0, m.abort_flag, tmo);
        if (ok) {
            tc_fence_after();
            const int64_t o = (g.tok0 + j) * HD + (int64_t)h * kD + 64 * wg;
#pragma unroll 1
            for (int w = 0; w < 2; ++w) {
                float* dst = (w ? a.dk : a.dv) + o;
                const uint32_t col = (w ? cDK : cDV) + 64 * wg;
#pragma unroll 1
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + col + c0, v);
                    tmem_wait_ld();
                    if (key_valid) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            reinterpret_cast<float4*>(dst + c0)[q] =
                                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                    }
                    __syncwarp();
                }
            }
        }
    }
    teardown(m, warp, tmem, a.ws);
}

}  // namespace bt

void launch_bwd_tc(const BwdTcMaps& m, const BwdTcArgs& a, const BucketBounds& bb, cudaStream_t stream)
{
    if (a.B <= 0 || a.qblocks <= 0)
        return;
    static std::atomic<uint32_t> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaFuncSetAttribute(bt::bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bt::kSmemBytes);
        cudaFuncSetAttribute(bt::bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bt::kSmemBytes);
        if (dev >= 0 && dev < 64)
            attr_set[dev].store(1, std::memory_order_relaxed);
    }
    const dim3 grid((unsigned)((int64_t)a.H * a.B), (unsigned)a.qblocks, 1);
    bt::bwd_dq_kernel<<<grid, bt::kThreads, bt::kSmemBytes, stream>>>(m.q, m.k, m.v, m.dO, bb, a);
    bt::bwd_dkv_kernel<<<grid, bt::kThreads, bt::kSmemBytes, stream>>>(m.q, m.k, m.v, m.dO, bb, a);
}

}  // namespace hstu
