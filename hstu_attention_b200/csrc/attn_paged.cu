// attn_paged.cu -- the paged cache hit of HSTU attention on Blackwell tensor cores (bf16 in,
// fp32 accumulate, D = 128).
//
// What it computes (per user b, head h, for the user's new tokens as queries): keys are the
// user's cached history, read through its page table, followed by its new tokens (NVIDIA blog
// "Deploying an HSTU Generative Recommender with NVIDIA Dynamo-Triton", section "Why serving
// large sequential recommenders is hard": the KV cache holds the history and only new tokens
// are computed).  Per key tile of up to 128 keys, for a group of up to 128 queries:
//     S = Q K^T                     tcgen05.mma, A = Q (smem), B = K tile (smem), S in TMEM
//     P = allowed ? SiLU(S + rab[h][bucket(i-j)]) : 0       registers -> bf16 P in TMEM
//     O += P V                      tcgen05.mma, A = P (TMEM), B = V tile (smem)
// SiLU weighting replaces softmax (aitrends.kr summary, section "HSTU의 순차 모델링"), so key
// ranges can be split across CTAs and their partial outputs simply added; combine.cu applies
// LayerNorm(O) * U afterwards.
//
// Work plan: a query group is up to 128 new tokens of one user; its key range (cached keys,
// then the new keys up to its last query) is cut into units of max(32, P) keys, and the units
// of each (group, head) into at most kMaxSplits contiguous pieces, sized so that all pieces fit
// the grid (one CTA per SM for small batches, whole waves for big ones).  Every CTA computes the
// same plan from the length arrays and takes piece blockIdx.x.
//
// Pipeline.  P stays in tensor memory, so a K stage is free as soon as Q K^T has read it and a V
// stage once P V has; the K ring runs three tiles ahead of the products, the V ring two.  The
// pointwise stage is split into two warpgroups that take alternate tiles (warpgroup t%2 owns tile
// t and all of its 128 key columns), so one group's TMEM and barrier latencies overlap the other
// group's arithmetic, and the MMA thread issues Q K^T two tiles ahead of P V: S buffer t%2 frees
// once its warpgroup has read S(t) into registers, well before P(t) is complete.  The pages of the
// first tiles are requested into L2 before the dependency wait, later ones a few tiles ahead.
//
// CTA roles (384 threads):
//   warp 0 lane 0   TMA producer: Q, then the K tiles (3-stage ring); cached tiles are
//                   gathered page by page (one box of P rows per page and channel half)
//   warp 3 lane 0   TMA producer of the V tiles (2-stage ring)
//   warp 1          allocates TMEM; lane 0 issues S(t+2) = Q K_{t+2}^T into S buffer t%2,
//                   then O += P_t V_t
//   warp 2          page-id staging in the prologue only
//   warps 4-11      pointwise, warpgroup t%2 on tile t: it first writes the tile's 255 bias
//                   values rab[h][bucket(d)]/2 (four copies shifted by one float, so every thread
//                   reads 16-byte vectors), then warp w reads TMEM lanes (= queries) 32(w%4).. and
//                   the tile's 128 key columns in four batches; x/2 = S/2 + rab/2,
//                   mask, SiLU = x/2 (1 + tanh(x/2)), bf16 P into TMEM buffer t%2; warps whose
//                   32 lanes hold no query of the group skip the arithmetic.  Epilogue:
//                   O / n_max -> padded fp32 tile in the rings -> 512-byte rows of the plane.
// TMEM columns: S0 [0,128) | S1 [128,256) | O [256,384) | P0 [384,448) | P1 [448,512).
// Shared memory: Q 32 KB | K 3 x 32 KB | V 2 x 32 KB | bias windows | bucket bounds | rab | page
// ids | mbarriers.  Every mbarrier wait is bounded (HSTU_DEV_TIMEOUT).
#include <atomic>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace hstu {
using namespace sm100;

namespace pg {

constexpr int kD = 128;
constexpr int kKeys = 128;                    // keys per tile (N of Q K^T, K of P V)
constexpr int kMaxQ = 128;                    // queries per CTA (M of both products)
constexpr int kThreads = 384;
constexpr int kKStages = 3;                   // K ring
constexpr int kVStages = 2;                   // V ring
constexpr int kMaxNB = 1024;
constexpr int kMaxPageIds = 1024;
constexpr uint32_t kHalf = 128 * 128;         // 128 rows x 128 bytes: one swizzle column
constexpr uint32_t kTileBytes = 2 * kHalf;    // 128 x 128 bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;
constexpr uint32_t kWinPad = 4;
constexpr uint32_t kWinStride = 264;
constexpr uint32_t kWinBuf = 4 * kWinStride * 4;
constexpr uint32_t kOffWin = kOffV + kVStages * kTileBytes;
constexpr uint32_t kRingBytes = (kKStages + kVStages) * kTileBytes;
constexpr uint32_t kOffBounds = kOffWin + 4 * kWinBuf;    // two windows per warpgroup
constexpr uint32_t kOffRab = kOffBounds + (kMaxNB + 4) * 4;
constexpr uint32_t kOffPages = kOffRab + kMaxNB * 4;
constexpr int kMaxNBT = 64;                   // time buckets (second bias)
constexpr uint32_t kOffRabT = kOffPages + kMaxPageIds * 4;
constexpr uint32_t kOffTs = kOffRabT + kMaxNBT * 4;           // key timestamps: a buffer per window
constexpr uint32_t kOffBar = kOffTs + 4 * kKeys * 4;
constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 2 + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
// the plan's per-user arrays (5 x int32) live in the K and V rings before the first load is issued
constexpr int kPlanMaxUsers = (int)(kRingBytes / 20);
constexpr int kPrefetchTiles = 6;             // key tiles requested into L2 ahead of their loads
constexpr uint32_t kOStride = kD + 4;         // floats per row of the staged O tile (epilogue)
static_assert(kMaxQ * kOStride * 4 <= kRingBytes, "epilogue staging fits the K and V rings");
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");

// The piece a CTA works on and its user's geometry (shared memory).
struct Piece {
    int32_t found;
    int32_t b, g, h, s, ns;       // user, query group, head, split index, splits of the group
    int32_t u0, u1;               // unit range of the piece within the group's units
    int32_t C, N, hist;           // cached keys, new tokens, history length of the user
    int32_t off;                  // first new-token row of the user
    int32_t valid;
    uint32_t flags;               // status bits to raise once the dependency wait is over
};

struct Tile {
    int32_t j0;        // absolute position of key row 0
    int32_t nvalid;    // key rows of this tile that hold keys of the user
    bool cached;
};

// Units of entry e = (user, query group): cached units plus the new-key units up to the group's
// last query; an invalid user keeps one unit on group 0 (one piece per head writes its zero rows
// and reports it).
__device__ __forceinline__ int entry_units(const int32_t* sCu, const int32_t* sN, int e, int qblocks, int us_log2)
{
    const int b = e / qblocks, g = e - b * qblocks;
    const int32_t cu = sCu[b], N = sN[b];
    if (cu < 0)
        return g == 0 ? 1 : 0;
    if (g * kMaxQ >= N)
        return 0;
    const int32_t kn = min(N, (g + 1) * kMaxQ);
    return cu + ((kn + (1 << us_log2) - 1) >> us_log2);
}

// min(ceil(u / c), max_splits) by comparisons.
__device__ __forceinline__ int splits_of(int u, int c, int max_splits)
{
    int s = 0;
#pragma unroll
    for (int k = 0; k < kMaxSplits; ++k)
        s += ((k < max_splits) & (u > k * c)) ? 1 : 0;
    return s;
}

// Whole warp 0.  Reads the length arrays once, stages per-user facts in shared memory, picks the
// units per piece and finds piece blockIdx.x.
__device__ void make_plan(const PagedArgs& a, int32_t* sCu, int32_t* sN, int32_t* sOff, int32_t* sC, int32_t* sT,
                          Piece* out)
{
    const int lane = threadIdx.x & 31;
    const int us_log2 = a.P > 32 ? (a.P == 64 ? 6 : 7) : 5;
    const int32_t max_cached = a.max_pages * a.P;
    int64_t run = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
        const int b = b0 + lane;
        int32_t C = 0, N = 0, T = 0;
        if (b < a.B) {
            C = a.cached_lens[b];
            N = a.new_lens[b];
            T = a.num_targets ? a.num_targets[b] : 0;
        }
        const int32_t npos = (b < a.B && N > 0) ? N : 0;
        int32_t incl = npos;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += y;
        }
        const int64_t off = run + (incl - npos);
        if (b < a.B) {
            // cached units, or -1 (bad lengths) / -2 (longer than n_max) for a rejected user
            const bool len_ok = C >= 0 && N >= 0 && T >= 0 && T <= N && N <= a.max_len && C <= max_cached &&
                                off + N <= a.total_tokens;
            const bool ok = len_ok && (int64_t)C + N <= a.n_max;
            sCu[b] = ok ? (C + (1 << us_log2) - 1) >> us_log2 : (len_ok ? -2 : -1);
            sN[b] = npos;
            sOff[b] = (int32_t)off;
            sC[b] = C;
            sT[b] = T;
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    const int E = a.B * a.qblocks;
    int64_t w = 0;
    for (int e = lane; e < E; e += 32)
        w += entry_units(sCu, sN, e, a.qblocks, us_log2);
    for (int o = 16; o > 0; o >>= 1)
        w += __shfl_xor_sync(0xffffffffu, w, o);
    w *= a.H;
    const int64_t grid = gridDim.x;
    int c = (int)((w + grid - 1) / grid);
    if (c < 1)
        c = 1;
    for (int it = 0; it < 256; ++it) {
        int64_t pieces = 0;
        for (int e = lane; e < E; e += 32)
            pieces += splits_of(entry_units(sCu, sN, e, a.qblocks, us_log2), c, a.max_splits);
        for (int o = 16; o > 0; o >>= 1)
            pieces += __shfl_xor_sync(0xffffffffu, pieces, o);
        if (pieces * a.H <= grid)
            break;
        c += c < 64 ? 1 : c / 16;                 // the smallest piece size that fits the grid
    }
    // find piece blockIdx.x: pieces are numbered entry by entry, (head, split) inside an entry
    const int want = (int)blockIdx.x;
    int base = 0;
    int found_e = -1, local = 0, ns = 1, units = 0;
    for (int e0 = 0; e0 < E && found_e < 0; e0 += 32) {
        const int e = e0 + lane;
        const int u = e < E ? entry_units(sCu, sN, e, a.qblocks, us_log2) : 0;
        const int n = splits_of(u, c, a.max_splits);
        const int cnt = a.H * n;
        int incl = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += y;
        }
        const int excl = incl - cnt;
        const bool mine = cnt > 0 && want >= base + excl && want < base + incl;
        const unsigned who = __ballot_sync(0xffffffffu, mine);
        if (who) {
            const int src = __ffs(who) - 1;
            found_e = __shfl_sync(0xffffffffu, e, src);
            local = __shfl_sync(0xffffffffu, want - base - excl, src);
            ns = __shfl_sync(0xffffffffu, n, src);
            units = __shfl_sync(0xffffffffu, u, src);
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        Piece p{};
        p.found = found_e >= 0;
        if (p.found) {
            const int b = found_e / a.qblocks;
            p.b = b;
            p.g = found_e - b * a.qblocks;
            p.ns = ns;
            p.h = local / ns;
            p.s = local - p.h * ns;
            p.u0 = (int32_t)(((int64_t)units * p.s) / ns);
            p.u1 = (int32_t)(((int64_t)units * (p.s + 1)) / ns);
            const int32_t C = sC[b], T = sT[b];
            p.valid = sCu[b] >= 0;
            p.off = sOff[b];
            p.C = C > 0 ? C : 0;
            p.N = sN[b];
            if ((int64_t)sOff[b] + p.N > a.total_tokens)
                p.N = 0;                          // rows that cannot be located are never written
            p.hist = p.C + p.N - (T > 0 ? T : 0);
            p.flags = 0;
            if (!p.valid && p.g == 0 && p.h == 0 && p.s == 0)
                p.flags = sCu[b] == -2 ? HSTU_DEV_BAD_NMAX : HSTU_DEV_BAD_LENGTH;
        }
        *out = p;
    }
}

// Tile t of the piece: the cached part first (tiles start at the piece's first unit), then the
// new keys (tiles restart at the first new key of the piece).
struct PieceTiles {
    int32_t cbeg, cend;     // cached key range [cbeg, cend)
    int32_t nbeg, nend;     // new-key range, relative to C
    int32_t nct, n;         // cached tiles, all tiles
};

__device__ __forceinline__ PieceTiles piece_tiles(const Piece& p, int us_log2)
{
    PieceTiles r;
    const int32_t cu = (p.C + (1 << us_log2) - 1) >> us_log2;
    const int32_t qrow0 = p.g * kMaxQ;
    const int32_t kn = min(p.N, qrow0 + kMaxQ);
    r.cbeg = p.u0 << us_log2;
    r.cend = min(min(p.u1, cu) << us_log2, p.C);
    r.nct = r.cend > r.cbeg ? (r.cend - r.cbeg + kKeys - 1) / kKeys : 0;
    r.nbeg = (max(p.u0, cu) - cu) << us_log2;
    r.nend = min((p.u1 - cu) << us_log2, kn);
    const int32_t nnt = r.nend > r.nbeg ? (r.nend - r.nbeg + kKeys - 1) / kKeys : 0;
    r.n = r.nct + nnt;
    return r;
}

__device__ __forceinline__ Tile tile_of(const PieceTiles& pt, int t, int32_t C)
{
    Tile g;
    if (t < pt.nct) {
        g.j0 = pt.cbeg + t * kKeys;
        g.nvalid = min(kKeys, pt.cend - g.j0);
        g.cached = true;
    } else {
        const int32_t r0 = pt.nbeg + (t - pt.nct) * kKeys;
        g.j0 = C + r0;
        g.nvalid = min(kKeys, pt.nend - r0);
        g.cached = false;
    }
    return g;
}

// bucket(d) for kN distances: the largest k with bounds[k] <= d (bounds[0] = 0,
// bounds[nb] = INT_MAX).  Branchless binary search, the kN searches interleaved.
template <int kN>
__device__ __forceinline__ void bucket_search(const int32_t* bounds, int nb, int top, const int32_t (&d)[kN],
                                              int (&k)[kN])
{
#pragma unroll
    for (int e = 0; e < kN; ++e)
        k[e] = 0;
    for (int step = top; step > 0; step >>= 1) {
#pragma unroll
        for (int e = 0; e < kN; ++e)
            k[e] += (bounds[min(k[e] + step, nb)] <= d[e]) ? step : 0;
    }
}

// Smallest d >= 0 with bucket(d) >= k, k >= 1 (used when the host did not pass the bounds).
__device__ int bucket_bound_dev(int k, double ln_nmax, int nb)
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

// SiLU weights of 32 consecutive key columns of one query row: x/2 = S/2 + bias (bias holds
// rab/2), w = x/2 (1 + tanh(x/2)), masked to 0 where the key is not visible (j < lim or
// j == diag), packed to bf16 pairs with integer rounding (see bf16x2_round_int).
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
        packed[2 * q4] = bf16x2_round_int(w0, w1);
        packed[2 * q4 + 1] = bf16x2_round_int(w2, w3);
    }
}

// Request tile t of the piece (K or V, both channel halves) into L2.  A prefetch returns no
// data to the SM and L2 is the device's point of coherence, so it may run before the
// dependency wait: later loads still see whatever the previous kernel wrote.
__device__ __forceinline__ void prefetch_tile(const CUtensorMap* tm_pages, const CUtensorMap* tm_rows,
                                              const PieceTiles& pt, int t, const Piece& p, const int32_t* s_pages,
                                              int32_t lp_begin, int P, int H)
{
    const Tile tg = tile_of(pt, t, p.C);
    if (tg.cached) {
        const int lp0 = tg.j0 / P;
        const int npg = (tg.nvalid + P - 1) / P;
        for (int k = 0; k < npg; ++k) {
            const int rel = lp0 + k - lp_begin;
            const int32_t pg = rel < kMaxPageIds ? s_pages[rel] : -1;
            if (pg >= 0)
                for (int hf = 0; hf < 2; ++hf)
                    tma_prefetch_l2_2d(tm_pages, hf * 64, (pg * H + p.h) * P);
        }
    } else {
        for (int hf = 0; hf < 2; ++hf)
            tma_prefetch_l2_3d(tm_rows, hf * 64, p.h, (int32_t)(p.off + (tg.j0 - p.C)));
    }
}

template <bool kTime>
__global__ void __maxnreg__(128)
attn_paged_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                  const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ BucketBounds bb,
                  const PagedArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ Piece sP;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_u32 & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw_u32 + pad;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars;
    uint64_t* k_full = q_full + 1;              // [kKStages]
    uint64_t* k_empty = k_full + kKStages;      // [kKStages]: released after Q K^T of the tile
    uint64_t* v_full = k_empty + kKStages;      // [kVStages]
    uint64_t* v_empty = v_full + kVStages;      // [kVStages]: released after P V of the tile
    uint64_t* s_full = v_empty + kVStages;      // [2]
    uint64_t* s_empty = s_full + 2;             // [2]: warpgroup has S in registers
    uint64_t* p_full = s_empty + 2;             // [2]: P of tile t in TMEM buffer t%2
    uint64_t* p_empty = p_full + 2;             // [2]: P V of the buffer's last tile completed
    uint64_t* o_full = p_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    float* win = reinterpret_cast<float*>(smem + kOffWin);
    int32_t* s_bounds = reinterpret_cast<int32_t*>(smem + kOffBounds);
    float* s_rab = reinterpret_cast<float*>(smem + kOffRab);
    int32_t* s_pages = reinterpret_cast<int32_t*>(smem + kOffPages);
    float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);
    int32_t* s_ts = reinterpret_cast<int32_t*>(smem + kOffTs);

    // ---------------------------------------------------------------- plan and set-up
    // only the length arrays and the page table are read before the dependency wait
    if (warp == 0) {
        int32_t* sCu = reinterpret_cast<int32_t*>(smem + kOffK);
        make_plan(a, sCu, sCu + kPlanMaxUsers, sCu + 2 * kPlanMaxUsers, sCu + 3 * kPlanMaxUsers,
                  sCu + 4 * kPlanMaxUsers, &sP);
    } else if (warp == 1) {
        if (lane == 0) {
            mbar_init(q_full, 1);
            for (int s = 0; s < kKStages; ++s) {
                mbar_init(&k_full[s], 1);
                mbar_init(&k_empty[s], 1);
            }
            for (int s = 0; s < kVStages; ++s) {
                mbar_init(&v_full[s], 1);
                mbar_init(&v_empty[s], 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(&s_full[s], 1);
                mbar_init(&s_empty[s], 128);
                mbar_init(&p_full[s], 128);
                mbar_init(&p_empty[s], 1);
            }
            mbar_init(o_full, 1);
            *abort_flag = 0;
            *reinterpret_cast<unsigned int*>(smem + kOffMisc + 8) = 0u;   // a staged page id was bad
            fence_mbar_init();
        }
        __syncwarp();
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const Piece p = sP;
    // the LayerNorm kernel queued behind this grid may be scheduled now; it waits for this
    // grid's completion before it reads anything this grid writes
    pdl_launch_dependents();
    const uint32_t tmem = *tmem_slot;
    const int us_log2 = a.P > 32 ? (a.P == 64 ? 6 : 7) : 5;
    const int64_t HD = (int64_t)a.H * kD;

    if (!p.found || !p.valid) {
        pdl_wait_primary();
        if (p.found) {
            if (threadIdx.x == 0 && p.flags)
                set_flag(a.ws, p.flags);
            // a rejected user: this head's slice of every row is zero in plane 0, one plane
            float* part = a.part;
            for (int64_t x = threadIdx.x; x < (int64_t)p.N * (kD / 4); x += kThreads) {
                const int64_t r = x / (kD / 4);
                const int c4 = (int)(x % (kD / 4));
                reinterpret_cast<float4*>(part + (p.off + r) * HD + (int64_t)p.h * kD)[c4] =
                    make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (p.h == 0)
                for (int r = threadIdx.x; r < p.N; r += kThreads)
                    a.counts[p.off + r] = 1;
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, kTmemCols);
        }
        return;
    }

    const PieceTiles pt = piece_tiles(p, us_log2);
    const int n = pt.n;
    const int32_t qrow0 = p.g * kMaxQ;
    const int32_t nq = min(kMaxQ, p.N - qrow0);           // queries of this group (>= 1)
    const int32_t i0 = p.C + qrow0;                        // absolute position of query row 0
    const int P = a.P;
    const int32_t lp_begin = pt.cbeg / P;
    const int32_t lp_end = pt.cend > pt.cbeg ? (pt.cend + P - 1) / P : lp_begin;

    if (warp == 2 || warp == 3) {
        // the piece's page ids, validated (-1 = skip the load; reported after the wait)
        bool bad = false;
        const int ht = threadIdx.x - 64;
        for (int k = ht; k < lp_end - lp_begin && k < kMaxPageIds; k += 64) {
            int32_t pg = a.page_table[(int64_t)p.b * a.max_pages + lp_begin + k];
            if (pg < 0 || pg >= a.num_pages) {
                pg = -1;
                bad = true;
            }
            s_pages[k] = pg;
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0)
            atomicOr(reinterpret_cast<unsigned int*>(smem + kOffMisc + 8), 1u);
    }
    __syncthreads();
    const bool bad_page_staged = *reinterpret_cast<volatile unsigned int*>(smem + kOffMisc + 8) != 0;
    const uint64_t tmo = a.timeout_ns;
    const uint64_t drain = a.drain_ns;
    if ((warp == 0 || warp == 3) && lane == 0) {
        // start streaming the first tiles from HBM while the previous kernel finishes
        const bool is_v = warp == 3;
        for (int t = 0; t < n && t < kPrefetchTiles; ++t)
            prefetch_tile(is_v ? &tm_vp : &tm_kp, is_v ? &tm_v : &tm_k, pt, t, p, s_pages, lp_begin, P, a.H);
        if (!is_v)
            for (int hf = 0; hf < 2; ++hf)
                tma_prefetch_l2_3d(&tm_q, hf * 64, p.h, (int32_t)(p.off + qrow0));
    }
    // inputs and the workspace are touched only after the previous kernel on the stream finished
    pdl_wait_primary();
    if (threadIdx.x == 0 && bad_page_staged)
        set_flag(a.ws, HSTU_DEV_BAD_PAGE);
    if (p.h == 0 && p.s == 0)
        for (int r = threadIdx.x; r < nq; r += kThreads)
            a.counts[p.off + qrow0 + r] = p.ns;

    if ((warp == 0 || warp == 3) && lane == 0) {
        // ============================================================ TMA producers
        const bool is_v = warp == 3;
        uint64_t* full = is_v ? v_full : k_full;
        uint64_t* empty = is_v ? v_empty : k_empty;
        const int stages = is_v ? kVStages : kKStages;
        const uint32_t ring = sbase + (is_v ? kOffV : kOffK);
        const CUtensorMap* tm_rows = is_v ? &tm_v : &tm_k;
        const CUtensorMap* tm_pages = is_v ? &tm_vp : &tm_kp;
        if (!is_v) {
            mbar_arrive_expect_tx(q_full, kTileBytes);
            for (int hf = 0; hf < 2; ++hf)
                tma_load_3d(&tm_q, sbase + kOffQ + hf * kHalf, q_full, hf * 64, p.h, (int32_t)(p.off + qrow0));
        }
        int issued = 0;
        const int n_issue = (is_v && (a.inject & kInjectStallV)) ? 0 : n;
        for (int t = 0; t < n_issue; ++t) {
            const Tile tg = tile_of(pt, t, p.C);
            const int st = t % stages;
            if (t + kPrefetchTiles < n)
                prefetch_tile(tm_pages, tm_rows, pt, t + kPrefetchTiles, p, s_pages, lp_begin, P, a.H);
            if (t >= stages && !mbar_wait(&empty[st], ((t / stages) & 1) ^ 1, abort_flag, tmo))
                break;
            const uint32_t dst = ring + st * kTileBytes;
            if (tg.cached) {
                const int lp0 = tg.j0 / P;
                const int npg = (tg.nvalid + P - 1) / P;
                int32_t pages[kKeys / 8];
                uint32_t bytes = 0;
                for (int k = 0; k < npg; ++k) {
                    const int rel = lp0 + k - lp_begin;
                    int32_t pg;
                    if (rel < kMaxPageIds) {
                        pg = s_pages[rel];
                    } else {
                        pg = a.page_table[(int64_t)p.b * a.max_pages + lp0 + k];
                        if (pg < 0 || pg >= a.num_pages) {
                            set_flag(a.ws, HSTU_DEV_BAD_PAGE);
                            pg = -1;
                        }
                    }
                    if (pg >= 0)
                        bytes += (uint32_t)P * 128u * 2u;
                    pages[k] = pg;
                }
                mbar_arrive_expect_tx(&full[st], bytes);
                for (int k = 0; k < npg; ++k)
                    if (pages[k] >= 0)
                        for (int hf = 0; hf < 2; ++hf)
                            tma_load_2d(tm_pages, dst + hf * kHalf + k * P * 128, &full[st], hf * 64,
                                        (pages[k] * a.H + p.h) * P);
            } else {
                const int32_t row = (int32_t)(p.off + (tg.j0 - p.C));
                mbar_arrive_expect_tx(&full[st], kTileBytes);
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_3d(tm_rows, dst + hf * kHalf, &full[st], hf * 64, p.h, row);
            }
            issued = t + 1;
        }
        // loads still in flight must land before the CTA exits (a local flag: the drain never
        // raises the CTA-wide abort)
        volatile int never = 0;
        if (!is_v)
            mbar_wait(q_full, 0, &never, drain);
        for (int t = (issued > stages ? issued - stages : 0); t < issued; ++t)
            mbar_wait(&full[t % stages], (t / stages) & 1, &never, drain);
    } else if (warp == 1 && lane == 0) {
        // ============================================================ MMA issuer
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
        const uint32_t qbase = sbase + kOffQ;
        bool ok = mbar_wait(q_full, 0, abort_flag, tmo);
        auto issue_qk = [&](int t) -> bool {
            const int kst = t % kKStages;
            const int sb = t & 1;
            if (!mbar_wait(&k_full[kst], (t / kKStages) & 1, abort_flag, tmo))
                return false;
            if (t >= 2 && !mbar_wait(&s_empty[sb], ((t >> 1) & 1) ^ 1, abort_flag, tmo))
                return false;
            tc_fence_after();
            const uint32_t kbase = sbase + kOffK + kst * kTileBytes;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                // 16 head-dim channels per step: A = Q (queries x D), B = K tile (keys x D)
                const uint64_t ad = smem_desc_sw128(qbase + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(kbase + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
                umma_bf16_ss(tmem + (sb ? kColS1 : kColS0), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[sb]);
            umma_commit(&k_empty[kst]);
            return true;
        };
        auto issue_pv = [&](int u) -> bool {
            const int vst = u % kVStages, pb = u & 1;
            if (!mbar_wait(&p_full[pb], (u >> 1) & 1, abort_flag, tmo))
                return false;
            if (!mbar_wait(&v_full[vst], (u / kVStages) & 1, abort_flag, tmo))
                return false;
            tc_fence_after();
            const uint32_t vbase = sbase + kOffV + vst * kTileBytes;
            const uint32_t pcol = tmem + (pb ? kColP1 : kColP0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                // 16 keys per step: A = P (TMEM, two keys per column), B = V tile (D contiguous)
                const uint64_t bd = smem_desc_sw128(vbase + kk * 2048, kHalf, 1024);
                umma_bf16_ts(tmem + kColO, pcol + kk * 8, bd, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&p_empty[pb]);
            umma_commit(&v_empty[vst]);
            return true;
        };
        // Q K^T runs two tiles ahead of P V: S buffer t%2 frees as soon as warpgroup t%2 holds
        // S(t) in registers, long before its P(t) is complete
        for (int t = 0; ok && t < 2 && t < n; ++t)
            ok = issue_qk(t);
        for (int t = 0; ok && t < n; ++t) {
            if (t + 2 < n && !issue_qk(t + 2)) {
                ok = false;
                break;
            }
            if (!issue_pv(t)) {
                ok = false;
                break;
            }
        }
        // o_full fires once every MMA issued so far has completed (also on the abort path,
        // so tensor memory is idle before it is released)
        umma_commit(o_full);
        volatile int never = 0;
        mbar_wait(o_full, 0, &never, drain);
    } else if (warp >= 4) {
        // ============================================================ pointwise + epilogue
        // rab[h]/2 and the bucket bounds (from the host, or evaluated here for many buckets)
        const int pt_id = threadIdx.x - 128;
        for (int k = pt_id; k < a.NB; k += 256)
            s_rab[k] = 0.5f * a.rab[(int64_t)p.h * a.NB + k];
        if (kTime)
            for (int k = pt_id; k < a.NBT; k += 256)
                s_rabt[k] = 0.5f * a.rab_time[(int64_t)p.h * a.NBT + k];
        for (int k = pt_id; k <= a.NB; k += 256)
            s_bounds[k] = bb.count > 0 ? bb.v[k]
                                       : (k == 0 ? 0 : (k == a.NB ? 0x7fffffff : bucket_bound_dev(k, a.ln_nmax, a.NB)));
        named_barrier_sync(2, 256);
        const int nb = a.NB;
        int top = 1;
        while (top * 2 <= nb)
            top *= 2;
        const int wg = (warp - 4) >> 2;                   // this warpgroup owns tiles wg, wg + 2, ...
        const int wt = threadIdx.x - 128 - 128 * wg;      // 0..127 within the warpgroup
        const int q0 = (warp & 3) << 5;                   // first query row (= TMEM lane) of this warp
        const int r = q0 + lane;
        const uint32_t lane_base = (uint32_t)q0 << 16;
        const bool warp_active = q0 < nq;                 // some row of this warp is a query
        const bool row_valid = r < nq;
        const int32_t i_abs = i0 + r;
        const int32_t lim_row = row_valid ? min(i_abs + 1, p.hist) : -1;
        const int32_t ts_row = (kTime && row_valid) ? a.ts[p.off + qrow0 + r] : 0;   // a new token's timestamp
        const int y0 = (kKeys - 1) - r;                   // window index of (row r, key column 0)
        const int wsel = y0 & 3;
        const int woff = wsel * kWinStride + kWinPad + (y0 - wsel);
        bool ok = true;
        for (int t = wg; t < n; t += 2) {
            const int sb = t & 1;                         // == wg
            const Tile tg = tile_of(pt, t, p.C);
            // the tile's bias window, built by the warpgroup itself (two of the 255 values per
            // thread): window index y <-> distance d = (i0 - j0 + 127) - y, so query row r and key
            // column c meet at y = 127 - r + c.  Copy s holds the window shifted by s floats after a
            // 4-float pad, so every reader gets 16-byte aligned vectors.  Two buffers per warpgroup:
            // the barrier below also orders this write after every read of the buffer two tiles ago.
            float* wbuf = win + (2 * wg + ((t >> 1) & 1)) * (kWinBuf / 4);
            int32_t* tsbuf = s_ts + (2 * wg + ((t >> 1) & 1)) * kKeys;
            if (kTime) {
                // the tile's key timestamps: cached keys from the timestamp pages (same page ids as
                // K and V), new keys from the new tokens' timestamps; past the valid keys 0
                const int32_t j = tg.j0 + wt;
                int32_t tsv = 0;
                if (wt < tg.nvalid) {
                    if (tg.cached) {
                        const int32_t lp = j / P;
                        const int32_t rel = lp - lp_begin;
                        int32_t pg = rel < kMaxPageIds ? s_pages[rel] : a.page_table[(int64_t)p.b * a.max_pages + lp];
                        if (pg >= 0 && pg < a.num_pages)
                            tsv = a.ts_pages[(int64_t)pg * P + (j - lp * P)];
                    } else {
                        tsv = a.ts[p.off + (j - p.C)];
                    }
                }
                tsbuf[wt] = tsv;
            }
            {
                const int32_t dist0 = i0 - tg.j0 + (kKeys - 1);
                int32_t d[2];
                int k[2];
                d[0] = dist0 - wt;
                d[1] = dist0 - (wt + 128);
                bucket_search<2>(s_bounds, nb, top, d, k);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int y = wt + 128 * e;
                    const float val = ((y <= 2 * kKeys - 2) & (d[e] >= 0)) ? s_rab[k[e]] : 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        wbuf[c * kWinStride + kWinPad + (y - c)] = val;
                }
            }
            // every warp of the warpgroup takes this barrier once per tile, also after a timed-out
            // wait (the rest of the iteration is then skipped, never left early)
            named_barrier_sync(4 + wg, 128);
            ok = ok && mbar_wait_warp(&s_full[sb], (t >> 1) & 1, abort_flag, tmo);
            if (!ok)
                continue;
            tc_fence_after();
            const int32_t kvend = tg.j0 + tg.nvalid;
            const bool full = tg.cached && tg.nvalid == kKeys;
            const int32_t lim = min(lim_row, kvend);
            const int32_t diag = (row_valid && !tg.cached) ? i_abs : -1;
            const uint32_t scol = tmem + lane_base + (sb ? kColS1 : kColS0);
            const uint32_t pcol = tmem + lane_base + (sb ? kColP1 : kColP0);
            const float4* wv = reinterpret_cast<const float4*>(wbuf + woff);
            // P buffer sb is free once P V of tile t - 2 completed
            if (t >= 2) {
                ok = ok && mbar_wait_warp(&p_empty[sb], ((t >> 1) & 1) ^ 1, abort_flag, tmo);
                if (!ok)
                    continue;
            }
            if (warp_active) {
#pragma unroll 1
                for (int c0 = 0; c0 < kKeys; c0 += 32) {
                    uint32_t sv[32];
                    tmem_ld_32x32b_x32(scol + c0, sv);
                    tmem_wait_ld();
                    if (c0 == kKeys - 32) {
                        tc_fence_before();
                        mbar_arrive(&s_empty[sb]);
                    }
                    uint32_t packed[16];
                    if (full)
                        silu_cols32<false, kTime>(sv, wv + (c0 >> 2), packed, tg.j0 + c0, lim, diag, ts_row,
                                                  tsbuf + c0, s_rabt, a.NBT);
                    else
                        silu_cols32<true, kTime>(sv, wv + (c0 >> 2), packed, tg.j0 + c0, lim, diag, ts_row,
                                                 tsbuf + c0, s_rabt, a.NBT);
                    tmem_st_32x32b_x16(pcol + (c0 >> 1), packed);
                }
            } else {
                mbar_arrive(&s_empty[sb]);               // no query rows here: nothing to compute
            }
            if (tg.nvalid < kKeys) {
                // V rows past the user's keys may hold anything (page tails, stale tiles):
                // zero them so that 0 * NaN cannot reach O
                const int vst = t % kVStages;
                ok = ok && mbar_wait_warp(&v_full[vst], (t / kVStages) & 1, abort_flag, tmo);
                if (ok) {
                    uint8_t* vt = smem + kOffV + vst * kTileBytes;
                    const int first = tg.nvalid > 0 ? tg.nvalid : 0;
                    const int nchunks = (kKeys - first) * 16;
                    for (int x = wt; x < nchunks; x += 128) {
                        const int row = first + (x >> 4), hf = (x >> 3) & 1, ch = x & 7;
                        *reinterpret_cast<uint4*>(vt + hf * kHalf + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
            }
            __syncwarp();
            tmem_wait_st();
            if (ok) {
                tc_fence_before();
                mbar_arrive(&p_full[sb]);
            }
        }
        // ------------------------------------------------------------ epilogue: O / n_max -> plane
        // every product has completed, so the K and V rings are free: O (scaled by 1/n_max) goes
        // row by row into a padded fp32 tile there (warpgroup g: head-dim columns 64g..64g+63),
        // then each warp stores whole 512-byte rows of the partial plane
        ok = ok && mbar_wait_warp(o_full, 0, abort_flag, tmo);
        float* ostage = reinterpret_cast<float*>(smem + kOffK);
        if (ok && warp_active) {
            tc_fence_after();
            const float inv_n = a.inv_n;
            const uint32_t ocol = tmem + lane_base + kColO + wg * 64;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
                uint32_t ov[32];
                tmem_ld_32x32b_x32(ocol + c0, ov);
                tmem_wait_ld();
                float4* srow = reinterpret_cast<float4*>(ostage + r * kOStride + wg * 64 + c0);
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4)
                    srow[c4] = make_float4(__uint_as_float(ov[4 * c4]) * inv_n, __uint_as_float(ov[4 * c4 + 1]) * inv_n,
                                           __uint_as_float(ov[4 * c4 + 2]) * inv_n,
                                           __uint_as_float(ov[4 * c4 + 3]) * inv_n);
            }
        }
        named_barrier_sync(3, 256);
        if (ok) {
            float* part = a.part + (int64_t)p.s * a.total_tokens * HD + (int64_t)p.h * kD;
            const int64_t row0 = p.off + qrow0;
            for (int c = (threadIdx.x - 128) >> 5; c < nq; c += 8) {
                const float4 v = reinterpret_cast<const float4*>(ostage + c * kOStride)[lane];
                reinterpret_cast<float4*>(part + (row0 + c) * HD)[lane] = v;
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

}  // namespace pg

int paged_max_users() { return pg::kPlanMaxUsers; }

void launch_attn_paged(const TcMaps& m, const PagedArgs& a, const BucketBounds& bb, int num_sms,
                       cudaStream_t stream)
{
    if (a.B <= 0 || a.qblocks <= 0)
        return;
    static std::atomic<uint32_t> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaFuncSetAttribute(pg::attn_paged_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pg::kSmemBytes);
        cudaFuncSetAttribute(pg::attn_paged_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, pg::kSmemBytes);
        if (dev >= 0 && dev < 64)
            attr_set[dev].store(1, std::memory_order_relaxed);
    }
    // whole waves of one CTA per SM, at least two pieces' worth per (group, head) of the largest
    // batch the bounds allow: the plan sizes its pieces to fill exactly this grid
    const int64_t groups = (int64_t)a.B * a.qblocks * a.H;
    const int64_t sms = num_sms > 0 ? num_sms : 148;
    int64_t waves = (2 * groups + sms - 1) / sms;
    if (waves < 1)
        waves = 1;
    if (groups <= sms)
        waves = 1;
    const int64_t grid = waves * sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(pg::kThreads, 1, 1);
    cfg.dynamicSmemBytes = pg::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.overlap_previous ? 1 : 0;
    if (a.rab_time)
        cudaLaunchKernelEx(&cfg, pg::attn_paged_kernel<true>, m.q, m.k, m.v, m.kp, m.vp, bb, a);
    else
        cudaLaunchKernelEx(&cfg, pg::attn_paged_kernel<false>, m.q, m.k, m.v, m.kp, m.vp, bb, a);
}

}  // namespace hstu
