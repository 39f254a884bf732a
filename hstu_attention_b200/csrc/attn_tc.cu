// attn_tc.cu -- jagged-prefill HSTU attention on Blackwell tensor cores (bf16 in, fp32
// accumulate, D = 128).  (The paged cache hit has its own kernel, attn_paged.cu.)
//
// What it computes (per user b, head h): for a block of 128 query rows and the key tiles the
// block may see,
//     S = Q K^T                               tcgen05.mma (A = Q in TMEM, B = K in smem), S in TMEM
//     P = allowed ? SiLU(S + rab[h][bucket(i-j)]) : 0      registers -> bf16 P in TMEM
//     O += P V                                tcgen05.mma (A = P in TMEM, B = V in smem)
//     O / n_max -> workspace (fp32)
// SiLU weighting replaces softmax, so there is no running max or row sum and key tiles can be
// split across CTAs and summed afterwards (aitrends.kr summary, section "HSTU의 순차 모델링";
// news.bpdata.com, section "HSTU").  combine.cu applies LayerNorm(O) * U to the fp32 outputs.
//
// CTA roles (384 threads):
//   warp 0      TMA producer of Q and of the K tiles (2-stage ring; a K stage frees as soon as
//               Q K^T has read it).
//   warp 3      TMA producer of the V tiles (3-stage ring, freed after P V).
//   warp 1      allocates all 512 TMEM columns; lane 0 issues every MMA:
//               S_t = Q K_t^T, then O += P_{t-1} V_{t-1}.  One S buffer: the pointwise warps
//               move S_t into registers first, so S_{t+1} is computed while they work on S_t.
//               Both products take A from TMEM (Q, P) and only B from shared memory, which
//               leaves shared-memory bandwidth to the pointwise warps while a product runs (a
//               product with both operands in shared memory takes all of it).
//   warp 2      bias windows: for every tile the 255 distinct values rab[h][bucket(i-j)]/2 the
//               tile needs (eight per lane, their binary searches interleaved), in four copies
//               shifted by one float so each reader gets 16-byte vectors, into a ring of four
//               windows (mbarriers full / empty), up to four tiles ahead of the pointwise warps;
//               with the second bias also the tile's key timestamps.
//   warps 4-11  Two warpgroups; warpgroup g owns key columns [64g, 64g+64) of every tile,
//               warp w%4 owns TMEM lanes (= query rows) [32(w%4), +32).  They load S from
//               TMEM, form x/2 = S/2 + rab/2 with packed fp32x2 FMAs, mask, compute
//               SiLU(x) = x/2 * (1 + tanh(x/2)), and store it as bf16 P into TMEM (P buffer
//               t%2), where the P V MMA reads it.  The 1/n_max scale is applied to O once,
//               when it leaves TMEM.  At the start warpgroup 0 copies the Q tile from shared
//               memory into TMEM (row r -> lane r, two bf16 per column).
//   epilogue    O / n_max leaves TMEM row per thread into a padded fp32 tile in the (then
//               idle) K and V rings; each pointwise warp then stores whole 512-byte rows.
// Grid: (head, user) x query block, heaviest query blocks first.  With
// HSTU_FLAG_OVERLAP_PREVIOUS the grid is a programmatic dependent of the previous kernel: the
// set-up runs early, and every access to inputs or the workspace -- the status word included --
// waits for that kernel (griddepcontrol.wait).
// TMEM columns: S [0,128) | O [128,256) | P0 [256,320) | P1 [320,384) | Q [384,448)
// Shared memory (1024-byte aligned, 128B swizzle for every MMA operand):
//   Q 32 KB | K 2 x 32 KB | V 3 x 32 KB | 4 bias windows | bucket bounds | rab | key timestamps
//   | mbarriers
// Every wait is bounded (HSTU_DEV_TIMEOUT) so a logic error cannot hang the GPU.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "kernels.cuh"

namespace hstu {
using namespace sm100;

constexpr int kTcD = 128;
constexpr int kTile = 128;                    // query rows per CTA and keys per tile
constexpr int kKStages = 2;
constexpr int kVStages = 3;
constexpr int kTcThreads = 384;
constexpr int kMaxNB = 1024;                  // buckets staged in shared memory
constexpr uint32_t kHalf = 128 * 128;         // 128 rows x 128 bytes = 16 KB (one swizzle column)
constexpr uint32_t kTileBytes = 2 * kHalf;    // one 128 x 128 bf16 operand
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTileBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;
constexpr uint32_t kWinPad = 4;               // floats before each shifted copy (stores at y - s >= -3)
constexpr uint32_t kWinStride = 264;          // floats per copy: pad + 256 + 4 (spreads banks)
constexpr uint32_t kWinBuf = 4 * kWinStride * 4;
constexpr int kWinRing = 4;                   // bias windows (and key timestamps) in flight
constexpr uint32_t kOffWin = kOffV + kVStages * kTileBytes;
constexpr uint32_t kOffBounds = kOffWin + kWinRing * kWinBuf;
constexpr uint32_t kOffRab = kOffBounds + (kMaxNB + 4) * 4;
constexpr int kMaxNBT = 64;                   // time buckets (second bias)
constexpr uint32_t kOffRabT = kOffRab + kMaxNB * 4;
constexpr uint32_t kOffTs = kOffRabT + kMaxNBT * 4;           // key timestamps of a tile, one per window
constexpr uint32_t kOffBar = kOffTs + kWinRing * kTile * 4;
constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 1 + 1 + 2 + 2 + 1 + 1 + 2 * kWinRing;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;     // slack to align the base to 1024
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 128, kColP0 = 256, kColP1 = 320, kColQ = 384;

constexpr uint32_t kOStride = kTcD + 4;       // floats per row of the staged O tile (epilogue)
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffK + kTile * kOStride * 4 <= kOffWin, "epilogue staging fits the K and V rings");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");

struct TileGeo {
    int32_t j0;       // position of key row 0 of the tile
    int32_t kvend;    // keys at positions >= kvend are not valid data for this tile
};

__device__ __forceinline__ TileGeo tile_geo(int32_t t, int32_t L)
{
    TileGeo g;
    g.j0 = t * kTile;
    g.kvend = L;
    return g;
}

// bucket(d) for kN distances at once: the largest k with bounds[k] <= d, where bounds[k] is
// the smallest distance in bucket k (bounds[0] = 0, bounds[nb] = INT_MAX, d < 0 -> 0).  A
// branchless binary search on shared memory, the searches interleaved so their load latencies
// overlap.  Only integer and load instructions: the special-function pipe stays free for tanh.
template <int kN>
__device__ __forceinline__ void bucket_search(const int32_t* bounds, int nb, int top, const int32_t (&d)[kN],
                                              int (&k)[kN])
{
#pragma unroll
    for (int e = 0; e < kN; ++e)
        k[e] = 0;
    // Written without short-circuit logic: a data-dependent && / || here compiles to branches
    // that diverge across lanes and serialise the warp.
    for (int step = top; step > 0; step >>= 1) {
#pragma unroll
        for (int e = 0; e < kN; ++e)
            k[e] += (bounds[min(k[e] + step, nb)] <= d[e]) ? step : 0;
    }
}

// SiLU weights of 32 consecutive key columns of one query row: x/2 = S/2 + bias (bias holds
// rab/2), w = x/2 * (1 + tanh(x/2)), masked to 0 where the key is not visible, packed to
// bf16x2 rounding to nearest even (one conversion per pair: 1 % faster on the prefill batch than
// rounding with integer operations, so the conversion does not compete with tanh here).
// kMasked selects the per-column visibility test at compile time, so the full-tile loop has
// no branch and the compiler can interleave the independent tanh chains.
// Time bucket of a timestamp difference: 0 for d <= 0, else min(nbt - 1, bit length of d).
__device__ __forceinline__ int time_bucket(int32_t d, int nbt)
{
    return d <= 0 ? 0 : min(nbt - 1, 32 - __clz(d));
}

template <bool kMasked, bool kTime = false>
__device__ __forceinline__ void silu_cols32(const uint32_t* sv, const float4* wv, uint32_t* packed, int jc,
                                            int32_t lim, int32_t diag, int32_t ts_row = 0,
                                            const int32_t* tsk = nullptr, const float* rabt = nullptr, int nbt = 1)
{
    const uint64_t half2 = f2pack(0.5f, 0.5f);
#pragma unroll
    for (int q4 = 0; q4 < 8; ++q4) {
        float4 bias = wv[q4];
        if (kTime) {
            // second bias: rab_time[h][bucket(ts_i - ts_j)] / 2 (the pipeline works on halves)
            const int4 tj = reinterpret_cast<const int4*>(tsk)[q4];
            bias.x += rabt[time_bucket(ts_row - tj.x, nbt)];
            bias.y += rabt[time_bucket(ts_row - tj.y, nbt)];
            bias.z += rabt[time_bucket(ts_row - tj.z, nbt)];
            bias.w += rabt[time_bucket(ts_row - tj.w, nbt)];
        }
        const uint64_t xa = f2fma(f2pack(__uint_as_float(sv[4 * q4]), __uint_as_float(sv[4 * q4 + 1])), half2,
                                  f2pack(bias.x, bias.y));
        const uint64_t xb = f2fma(f2pack(__uint_as_float(sv[4 * q4 + 2]), __uint_as_float(sv[4 * q4 + 3])), half2,
                                  f2pack(bias.z, bias.w));
        float a0, a1, a2, a3;
        f2unpack(xa, a0, a1);
        f2unpack(xb, a2, a3);
        const uint64_t wa = f2fma(xa, f2pack(tanh_approx(a0), tanh_approx(a1)), xa);
        const uint64_t wb = f2fma(xb, f2pack(tanh_approx(a2), tanh_approx(a3)), xb);
        float w0, w1, w2, w3;
        f2unpack(wa, w0, w1);
        f2unpack(wb, w2, w3);
        if (kMasked) {
            const int j = jc + 4 * q4;           // bitwise | : no lane-divergent branches
            w0 = ((j < lim) | (j == diag)) ? w0 : 0.f;
            w1 = ((j + 1 < lim) | (j + 1 == diag)) ? w1 : 0.f;
            w2 = ((j + 2 < lim) | (j + 2 == diag)) ? w2 : 0.f;
            w3 = ((j + 3 < lim) | (j + 3 == diag)) ? w3 : 0.f;
        }
        const __nv_bfloat162 b01 = __floats2bfloat162_rn(w0, w1);
        const __nv_bfloat162 b23 = __floats2bfloat162_rn(w2, w3);
        packed[2 * q4] = *reinterpret_cast<const uint32_t*>(&b01);
        packed[2 * q4 + 1] = *reinterpret_cast<const uint32_t*>(&b23);
    }
}

// Smallest d >= 0 with bucket(d) >= k (bucket_of() of common.cuh, double precision), k >= 1.
// Used when the host did not pass the bounds (more buckets than the parameter block holds).
__device__ int bucket_bound(int k, double ln_nmax, int nb)
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

template <bool kTime>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ BucketBounds bb, const TcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ UserGeom sG;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // grid: x = (head, user), y = query block, heaviest blocks first
    const int h = blockIdx.x % a.H;
    const int b = blockIdx.x / a.H;
    const int qblk = a.qblocks - 1 - (int)blockIdx.y;
    if (warp == 0) {
        UserGeom g = jagged_geom(a.seq_offsets, a.num_targets, b, a.total_tokens, a.max_len, a.n_max);
        if (lane == 0)
            sG = g;
    }
    __syncthreads();
    const UserGeom g = sG;
    const int32_t qrow0 = qblk * kTile;
    const int64_t HD = (int64_t)a.H * kTcD;
    float* part = a.part;
    if (!g.ok) {
        // a rejected user: the q-block-0 CTA of each head writes zeros into that head's slice of
        // every row of the user (also rows past the grid when the user is longer than max_seqlen)
        pdl_wait_primary();
        if (qblk == 0) {
            if (h == 0 && threadIdx.x == 0)
                set_flag(a.ws, g.flags);
            for (int64_t x = threadIdx.x; x < (int64_t)g.N * (kTcD / 4); x += kTcThreads) {
                const int64_t r = x / (kTcD / 4);
                const int c4 = (int)(x % (kTcD / 4));
                reinterpret_cast<float4*>(part + (g.tok0 + r) * HD + (int64_t)h * kTcD)[c4] =
                    make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        pdl_launch_dependents();
        return;
    }
    if (qrow0 >= g.N)
        return;                                               // no queries here (uniform)

    const int32_t i0 = qrow0;                                 // position of row 0
    const int32_t last_q = min(g.N, qrow0 + kTile) - 1;
    const int32_t kend = min(g.L, last_q + 1);                // later keys are never visible
    const int n = (kend + kTile - 1) / kTile;                 // key tiles (>= 1)

    // ---------------------------------------------------------------- shared memory carve-up
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_u32 & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw_u32 + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars;
    uint64_t* k_full = q_full + 1;              // [kKStages]
    uint64_t* k_empty = k_full + kKStages;      // [kKStages]
    uint64_t* v_full = k_empty + kKStages;      // [kVStages]
    uint64_t* v_empty = v_full + kVStages;      // [kVStages]
    uint64_t* s_full = v_empty + kVStages;
    uint64_t* s_empty = s_full + 1;
    uint64_t* p_full = s_empty + 1;             // [2]
    uint64_t* p_empty = p_full + 2;             // [2]
    uint64_t* o_full = p_empty + 2;
    uint64_t* qt_full = o_full + 1;             // Q copied into TMEM
    uint64_t* win_full = qt_full + 1;           // [kWinRing] bias window t % kWinRing built
    uint64_t* win_empty = win_full + kWinRing;  // [kWinRing] ... and read by every pointwise thread
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    float* win = reinterpret_cast<float*>(smem + kOffWin);
    int32_t* s_bounds = reinterpret_cast<int32_t*>(smem + kOffBounds);
    float* s_rab = reinterpret_cast<float*>(smem + kOffRab);
    float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);
    int32_t* s_ts = reinterpret_cast<int32_t*>(smem + kOffTs);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_empty, 256);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&p_full[s], 256);
            mbar_init(&p_empty[s], 1);
        }
        mbar_init(o_full, 1);
        mbar_init(qt_full, 128);
        for (int s = 0; s < kWinRing; ++s) {
            mbar_init(&win_full[s], 32);
            mbar_init(&win_empty[s], 256);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t tmo = a.timeout_ns;
    const uint64_t drain = a.drain_ns;
    // everything above only read the length arrays and the page table; inputs and the workspace
    // are touched only after the previous kernel on the stream has finished (a no-op unless
    // this grid was launched as a programmatic dependent)
    pdl_wait_primary();

    if ((warp == 0 || warp == 3) && lane == 0) {
        // ============================================================ TMA producers
        // warp 0 loads Q and the K tiles, warp 3 the V tiles
        const bool is_v = warp == 3;
        uint64_t* full = is_v ? v_full : k_full;
        uint64_t* empty = is_v ? v_empty : k_empty;
        const int stages = is_v ? kVStages : kKStages;
        const uint32_t ring = sbase + (is_v ? kOffV : kOffK);
        const CUtensorMap* tm_rows = is_v ? &tm_v : &tm_k;
        tma_prefetch_desc(tm_rows);
        if (!is_v) {
            tma_prefetch_desc(&tm_q);
            mbar_arrive_expect_tx(q_full, kTileBytes);
            for (int hf = 0; hf < 2; ++hf)
                tma_load_3d(&tm_q, sbase + kOffQ + hf * kHalf, q_full, hf * 64, h, (int32_t)(g.tok0 + qrow0));
        }
        int issued = 0;
        const int n_issue = (is_v && (a.inject & kInjectStallV)) ? 0 : n;
        for (int t = 0; t < n_issue; ++t) {
            const TileGeo tg = tile_geo(t, g.L);
            const int st = t % stages;
            // tile t goes into stage t % stages once the MMA that read tile t - stages is done
            if (t >= stages && !mbar_wait(&empty[st], ((t / stages) & 1) ^ 1, abort_flag, tmo))
                break;
            const uint32_t dst = ring + st * kTileBytes;
            const int32_t row = (int32_t)(g.key_row0 + tg.j0);
            mbar_arrive_expect_tx(&full[st], kTileBytes);
            for (int hf = 0; hf < 2; ++hf)
                tma_load_3d(tm_rows, dst + hf * kHalf, &full[st], hf * 64, h, row);
            issued = t + 1;
        }
        // drain: loads still in flight must land before the CTA may exit (a local flag, so
        // the drain itself never raises the CTA-wide abort)
        volatile int never = 0;
        if (!is_v)
            mbar_wait(q_full, 0, &never, drain);
        for (int t = (issued > stages ? issued - stages : 0); t < issued; ++t)
            mbar_wait(&full[t % stages], (t / stages) & 1, &never, drain);
    } else if (warp == 1 && lane == 0) {
        // ============================================================ MMA issuer
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
        bool ok = mbar_wait(qt_full, 0, abort_flag, tmo);
        auto issue_pv = [&](int u) -> bool {
            const int vst = u % kVStages;
            const int pb = u & 1;
            if (!mbar_wait(&p_full[pb], (u >> 1) & 1, abort_flag, tmo))
                return false;
            if (!mbar_wait(&v_full[vst], (u / kVStages) & 1, abort_flag, tmo))
                return false;
            tc_fence_after();
            const uint32_t vbase = sbase + kOffV + vst * kTileBytes;
            const uint32_t pcol = tmem + (pb ? kColP1 : kColP0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t bd = smem_desc_sw128(vbase + kk * 2048, kHalf, 1024);
                umma_bf16_ts(tmem + kColO, pcol + kk * 8, bd, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&p_empty[pb]);
            umma_commit(&v_empty[vst]);
            return true;
        };
        for (int t = 0; ok && t < n; ++t) {
            const int kst = t % kKStages;
            if (!mbar_wait(&k_full[kst], (t / kKStages) & 1, abort_flag, tmo)) {
                ok = false;
                break;
            }
            // the S buffer is free once the pointwise warps hold S(t-1) in registers
            if (t >= 1 && !mbar_wait(s_empty, (t - 1) & 1, abort_flag, tmo)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t kbase = sbase + kOffK + kst * kTileBytes;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                // 16 head-dim channels per step: A = Q from TMEM (8 columns of bf16 pairs),
                // B = K tile (keys x D, 128-byte rows) from shared memory
                const uint64_t bd = smem_desc_sw128(kbase + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
                umma_bf16_ts(tmem + kColS, tmem + kColQ + kk * 8, bd, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(s_full);
            umma_commit(&k_empty[kst]);
            if (t >= 1 && !issue_pv(t - 1)) {
                ok = false;
                break;
            }
        }
        if (ok)
            ok = issue_pv(n - 1);
        // o_full fires once every MMA issued so far has completed (also on the abort path,
        // so tensor memory is idle before it is released)
        umma_commit(o_full);
        volatile int never = 0;
        mbar_wait(o_full, 0, &never, drain);
    } else if (warp == 2) {
        // ============================================================ bias windows
        // rab[h]/2 and the bucket bounds (from the host, or evaluated here for many buckets)
        for (int k = lane; k < a.NB; k += 32)
            s_rab[k] = 0.5f * a.rab[(int64_t)h * a.NB + k];
        for (int k = lane; k <= a.NB; k += 32)
            s_bounds[k] = bb.count > 0 ? bb.v[k]
                                       : (k == 0 ? 0 : (k == a.NB ? 0x7fffffff : bucket_bound(k, a.ln_nmax, a.NB)));
        __syncwarp();
        const int nb = a.NB;
        int top = 1;
        while (top * 2 <= nb)
            top *= 2;
        // window t holds the 255 values rab[h][bucket(d)]/2 the tile needs: window index y <->
        // distance d = (i0 - j0 + 127) - y, so query row r and key column c meet at y =
        // 127 - r + c.  Copy s holds the window shifted by s floats after a 4-float pad, so
        // every reader gets 16-byte aligned vectors.  Eight values per lane, searched together
        // so their load latencies overlap; the ring lets this warp run up to four tiles ahead.
        for (int t = 0; t < n; ++t) {
            const int wb = t % kWinRing;
            if (t >= kWinRing && !mbar_wait_warp(&win_empty[wb], ((t / kWinRing) & 1) ^ 1, abort_flag, tmo))
                break;
            const TileGeo tg = tile_geo(t, g.L);
            float* wbuf = win + wb * (kWinBuf / 4);
            const int32_t dist0 = i0 - tg.j0 + (kTile - 1);
            int32_t d[8];
            int k[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                d[e] = dist0 - (lane + 32 * e);
            bucket_search<8>(s_bounds, nb, top, d, k);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int y = lane + 32 * e;
                const float val = ((y <= 2 * kTile - 2) & (d[e] >= 0)) ? s_rab[k[e]] : 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    wbuf[c * kWinStride + kWinPad + (y - c)] = val;
            }
            if (kTime) {
                // the tile's key timestamps (0 past the user's keys)
#pragma unroll
                for (int e = 0; e < kTile / 32; ++e) {
                    const int32_t j = tg.j0 + lane + 32 * e;
                    s_ts[wb * kTile + lane + 32 * e] = j < g.L ? a.ts[g.key_row0 + j] : 0;
                }
            }
            mbar_arrive(&win_full[wb]);
        }
    } else if (warp >= 4) {
        // ============================================================ pointwise + epilogue
        const int pt = threadIdx.x - 128;                 // 0..255
        if (kTime) {
            for (int k = pt; k < a.NBT; k += 256)
                s_rabt[k] = 0.5f * a.rab_time[(int64_t)h * a.NBT + k];
            named_barrier_sync(2, 256);
        }
        const int wg = (warp - 4) >> 2;                   // key-column half
        const int r = ((warp & 3) << 5) + lane;           // query row in the block (= TMEM lane)
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool row_valid = qrow0 + r < g.N;
        const int32_t i_abs = i0 + r;
        const int32_t lim_row = row_valid ? min(i_abs + 1, g.hist) : -1;
        const int32_t ts_row = (kTime && row_valid) ? a.ts[g.tok0 + i_abs] : 0;
        // window: this thread's 64 bias values start at index y0 = 127 - r + 64 wg; copy s holds
        // the window shifted by s floats, so (y0 - s) is a multiple of 4
        const int y0 = (kTile - 1) - r + 64 * wg;
        const int wsel = y0 & 3;
        const int woff = wsel * kWinStride + kWinPad + (y0 - wsel);
        bool ok = true;
        if (wg == 0) {
            // Q into TMEM for the Q K^T products: row r of the tile (128-byte swizzle: the
            // 16-byte chunk c of a row sits at chunk c ^ (r & 7)) goes to lane r, head-dim
            // channels (2c, 2c+1) to column c, the lower channel in the low half
            ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, tmo));
            if (ok) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint8_t* qrow = smem + kOffQ + hf * kHalf + r * 128;
                    uint32_t qv[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 x = *reinterpret_cast<const uint4*>(qrow + ((c ^ (r & 7)) << 4));
                        qv[4 * c] = x.x;
                        qv[4 * c + 1] = x.y;
                        qv[4 * c + 2] = x.z;
                        qv[4 * c + 3] = x.w;
                    }
                    tmem_st_32x32b_x32(tmem + lane_base + kColQ + hf * 32, qv);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(qt_full);
            }
        }
        for (int t = 0; ok && t < n; ++t) {
            const int vst = t % kVStages;
            const int sb = t & 1;
            const int wb = t % kWinRing;
            const TileGeo tg = tile_geo(t, g.L);
            ok = mbar_wait_warp(&win_full[wb], (t / kWinRing) & 1, abort_flag, tmo) &&
                 mbar_wait_warp(s_full, t & 1, abort_flag, tmo);
            if (!ok)
                break;
            tc_fence_after();
            const float4* wv = reinterpret_cast<const float4*>(win + wb * (kWinBuf / 4) + woff);
            const bool full = (qrow0 + kTile - 1 < g.N) && (tg.j0 + kTile - 1 < tg.kvend) &&
                              (tg.j0 + kTile - 1 <= i0) && (tg.j0 + kTile - 1 < g.hist);
            const int32_t lim = min(lim_row, tg.kvend);
            const int32_t diag = row_valid ? i_abs : -1;
            const int jc0 = tg.j0 + wg * 64;                  // key position of column 0 of this half
            const uint32_t scol = tmem + lane_base + kColS + wg * 64;
            uint32_t sv[32], sv2[32];
            uint32_t packed[32];
            // both halves of this thread's 64 columns into registers, then the S buffer is
            // released: S(t+1) is computed while this tile's SiLU runs
            tmem_ld_32x32b_x32(scol, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld_32x32b_x32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv2[0]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(s_empty);
            const int32_t* tsk = s_ts + wb * kTile + wg * 64;
            if (full)
                silu_cols32<false, kTime>(sv, wv, packed, jc0, lim, diag, ts_row, tsk, s_rabt, a.NBT);
            else
                silu_cols32<true, kTime>(sv, wv, packed, jc0, lim, diag, ts_row, tsk, s_rabt, a.NBT);
            if (full)
                silu_cols32<false, kTime>(sv2, wv + 8, packed + 16, jc0 + 32, lim, diag, ts_row, tsk + 32, s_rabt, a.NBT);
            else
                silu_cols32<true, kTime>(sv2, wv + 8, packed + 16, jc0 + 32, lim, diag, ts_row, tsk + 32, s_rabt, a.NBT);
            mbar_arrive(&win_empty[wb]);                       // done with this window
            // P buffer sb is free once P V of tile t - 2 completed
            if (t >= 2) {
                ok = ok && mbar_wait_warp(&p_empty[sb], ((t >> 1) & 1) ^ 1, abort_flag, tmo);
                if (!ok)
                    continue;
            }
            tmem_st_32x32b_x32(tmem + lane_base + (sb ? kColP1 : kColP0) + wg * 32,
                               *reinterpret_cast<const uint32_t(*)[32]>(&packed[0]));
            const int vz = tg.kvend - tg.j0;                   // valid key rows in this tile
            if (vz < kTile) {
                // rows past the valid keys may hold anything (page tails, other users): zero
                // them so that 0 * NaN cannot reach O
                ok = ok && mbar_wait_warp(&v_full[vst], (t / kVStages) & 1, abort_flag, tmo);
                if (ok) {
                    uint8_t* vt = smem + kOffV + vst * kTileBytes;
                    const int first = vz > 0 ? vz : 0;
                    const int nchunks = (kTile - first) * 16;
                    for (int x = pt; x < nchunks; x += 256) {
                        const int row = first + (x >> 4), hf = (x >> 3) & 1, ch = x & 7;
                        *reinterpret_cast<uint4*>(vt + hf * kHalf + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
            }
            __syncwarp();                                      // .sync.aligned below
            tmem_wait_st();
            if (ok) {
                tc_fence_before();
                mbar_arrive(&p_full[sb]);
            }
        }
        // ------------------------------------------------------------ epilogue: O / n_max -> workspace
        // the LayerNorm kernel queued behind this grid may start launching now; it waits for
        // this grid's completion (and memory flush) before it reads the partial outputs
        pdl_launch_dependents();
        ok = ok && mbar_wait_warp(o_full, 0, abort_flag, tmo);
        // every MMA has completed, so the K and V rings are free: O (scaled by 1/n_max) goes
        // row by row into a padded fp32 tile there, then each warp writes whole rows (512
        // contiguous bytes per instruction) instead of one 16-byte piece per row
        float* ostage = reinterpret_cast<float*>(smem + kOffK);
        if (ok) {
            tc_fence_after();
            uint32_t ov[64];
            const uint32_t ocol = tmem + lane_base + kColO + wg * 64;
            tmem_ld_32x32b_x32(ocol, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
            tmem_ld_32x32b_x32(ocol + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
            tmem_wait_ld();
            const float inv_n = a.inv_n;
            float4* srow = reinterpret_cast<float4*>(ostage + r * kOStride + wg * 64);
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4)
                srow[c4] = make_float4(__uint_as_float(ov[4 * c4]) * inv_n, __uint_as_float(ov[4 * c4 + 1]) * inv_n,
                                       __uint_as_float(ov[4 * c4 + 2]) * inv_n,
                                       __uint_as_float(ov[4 * c4 + 3]) * inv_n);
        }
        named_barrier_sync(3, 256);                           // the eight pointwise warps
        if (ok) {
            const int pw = pt >> 5;                           // 0..7
            const int nrows = min(kTile, g.N - qrow0);
            for (int row = pw; row < nrows; row += 8) {
                const float4 v = reinterpret_cast<const float4*>(ostage + row * kOStride)[lane];
                reinterpret_cast<float4*>(part + (g.tok0 + qrow0 + row) * HD + (int64_t)h * kTcD)[lane] = v;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag)
        set_flag(a.ws, HSTU_DEV_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

void launch_attn_tc(const TcMaps& m, const TcArgs& a, const BucketBounds& bb, int32_t B, cudaStream_t stream)
{
    if (B <= 0 || a.qblocks <= 0)
        return;
    // the shared-memory opt-in is a per-device setting of the kernel
    static std::atomic<uint32_t> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (dev >= 0 && dev < 64)
            attr_set[dev].store(1, std::memory_order_relaxed);
    }
    // (head, user) x query block
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)a.H * B), (unsigned)a.qblocks, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.overlap_previous ? 1 : 0;          // programmatic dependent launch on request
    if (a.rab_time)
        cudaLaunchKernelEx(&cfg, attn_tc_kernel<true>, m.q, m.k, m.v, bb, a);
    else
        cudaLaunchKernelEx(&cfg, attn_tc_kernel<false>, m.q, m.k, m.v, bb, a);
}

}  // namespace hstu
