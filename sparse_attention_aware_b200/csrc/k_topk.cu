// Anchor-layer exact top-k per query head.
//
// Method: "Kascade稀疏注意力…", sections "核心机制：Anchor + Reuse" (exact
// top-k key indices on the anchor layer) and "头部感知（head-aware）是精度关键"
// (every head selects on its own; heads of one GQA group share only the K
// stream).
//
// k_topk_score: streams the whole K context once.  One CTA = (token chunk,
// kv head g, sequence b), 256 threads.  K rows arrive in shared memory through
// a ring of untiled bulk copies (page-row granular), and a group of G = D/8
// lanes reads one token row from there (16 B per lane) and computes the raw
// dot product with every query head of the GQA group, so K is read once for
// all of them.  Scores (fp32, unscaled) go to the workspace.
//
// k_topk_select: one CTA of 1024 threads per (sequence, query head).  An
// exact radix select on the order-preserving uint32 image of the fp32 score:
// three digit passes (11, 11, 10 bits) narrow the k-th largest key to a
// single value T and the number r of elements equal to T that are still to be
// taken; the output is every element above T and the first r elements equal
// to T (ties to the lower position), in ascending position order.  Only the
// first two passes read the whole row (see the kernel comment).
#include "sa_internal.h"
#include "tc_ptx.cuh"

namespace sa {
namespace {

constexpr int kScoreChunk = 4096;   // tokens per scoring CTA
constexpr int kSelThreads = 1024;

// Sum G partials held by each of G lanes so that lane l ends with the total of
// partial index l: at every butterfly step a lane keeps the lower half of its
// positions and sends the upper half to its partner (G - 1 shuffles in all).
// The caller stores partial p at position p ^ l (bits of l below G), which is
// what makes "keep the lower half" right for every lane without selects: at
// the step over lane bit o the lower half holds exactly the partials whose
// bit o equals l's, and the partner's upper half holds the same partials.
template <int G>
__device__ __forceinline__ float transpose_reduce(float (&v)[G])
{
#pragma unroll
    for (int cnt = G / 2; cnt >= 1; cnt >>= 1) {
#pragma unroll
        for (int i = 0; i < cnt; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i + cnt], cnt);
    }
    return v[0];
}

// Tile geometry of the scoring kernel.  One group of G = D/8 lanes owns U =
// G/HPG consecutive token rows per step (STEP rows per CTA step); a ring stage
// holds TT >= 64 tokens (R steps) of one kv head's K rows.
template <int D, int HPG>
struct ScoreGeom {
    static constexpr int G = D / 8, GPW = 32 / G, NG = 8 * GPW, U = G / HPG;
    static constexpr int STEP = NG * U;
    static constexpr int TT = STEP >= 64 ? STEP : 64;
    static constexpr int R = TT / STEP;
    static constexpr int STAGE = TT * D * 2;
    static constexpr int NS0 = (64 * 1024) / STAGE;   // 3 CTAs per SM at D=128
    static constexpr int NS = NS0 < 2 ? 2 : (NS0 > 8 ? 8 : NS0);
    static constexpr int MAXJ = (TT + 31) / 32;   // page spans per lane of the producer warp
    static constexpr int SMEM = NS * STAGE + 2 * NS * 8 + NS * 8 * 4 + 16;
    static constexpr int THREADS = 8 * 32 + 32;    // 8 consumer warps + 1 producer warp
};

constexpr uint64_t kScoreWaitNs = 1000ull * 1000 * 1000;   // 1 s

// The K rows of a CTA's token chunk stream through an NS-stage shared-memory
// ring filled by untiled bulk copies (one per page span of a tile: whole page
// rows when P <= TT, else a TT-token piece of one).  Warp 8 is the producer:
// it refills a stage once all 8 consumer warps have released it (per-stage
// "empty" mbarriers, so consumer warps drift freely within the ring) and keeps
// the page-table entries of the next tile in registers.  Rows whose page
// entry is out of range are recorded as a device fault and score -inf, so they
// are never selected.
template <int D, int HPG, bool QF32>
__global__ void __launch_bounds__(ScoreGeom<D, HPG>::THREADS) k_topk_score(const TopkArgs a)
{
    pdl_wait();
    pdl_trigger();
    using Gm = ScoreGeom<D, HPG>;
    constexpr int G = Gm::G, GPW = Gm::GPW, U = Gm::U, TT = Gm::TT, NS = Gm::NS, MAXJ = Gm::MAXJ;
    constexpr int HL = HPG == 1 ? 0 : HPG == 2 ? 1 : HPG == 4 ? 2 : 3;   // log2(HPG)
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + NS * Gm::STAGE);
    uint64_t *empty = full + NS;
    uint32_t *badm = reinterpret_cast<uint32_t *>(empty + NS);   // [NS][8] bad-span bits
    volatile int *abort_flag = reinterpret_cast<volatile int *>(badm + NS * 8);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int Lcap = a.c.max_pages << a.c.Plog2;
    int L = __ldg(a.c.sl + b);
    if (L < 0 || L > Lcap) {
        if (threadIdx.x == 0 && chunk == 0 && g == 0) fault(a.st, CHK_SEQ_LEN, L);
        L = L < 0 ? 0 : Lcap;
    }
    const int t0 = chunk * kScoreChunk;
    const int t1 = min(t0 + kScoreChunk, L);
    if (t0 >= t1) return;
    const int ntiles = (t1 - t0 + TT - 1) / TT;
    // page spans: SPAN = min(P, TT) tokens, nsp = TT / SPAN per tile
    constexpr int TL = TT == 64 ? 6 : TT == 128 ? 7 : 8;   // log2(TT)
    static_assert((1 << TL) == TT, "tile size");
    const int slog2 = min(a.c.Plog2, TL);
    const int SPAN = 1 << slog2;
    const int nsp = TT >> slog2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            tc::mbar_init(full + s, 1);
            tc::mbar_init(empty + s, 8);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    const uint64_t deadline = tc::globaltimer() + kScoreWaitNs;

    if (warp == 8) {
        // ---------------------------------------------------------------- producer
        const int32_t *ptb = a.c.pt + (size_t)b * a.c.max_pages;
        const int Pm = (1 << a.c.Plog2) - 1;
        int pg[MAXJ];
        auto fetch = [&](int tile) {
#pragma unroll
            for (int j = 0; j < MAXJ; ++j) {
                const int sp = lane + 32 * j;
                const int ts = t0 + tile * TT + (sp << slog2);
                pg[j] = (tile < ntiles && sp < nsp && ts < t1) ? __ldg(ptb + (ts >> a.c.Plog2)) : -1;
            }
        };
        fetch(0);
        int issued = 0;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % NS;
            if (i >= NS) {
                const bool ok = __all_sync(
                    0xffffffffu, tc::mbar_wait(empty + s, (uint32_t)((i / NS) - 1) & 1u, deadline, abort_flag));
                if (!ok) break;
            }
            uint8_t *dst = sm + s * Gm::STAGE;
            uint32_t bytes = 0;
            bool go[MAXJ];
#pragma unroll
            for (int j = 0; j < MAXJ; ++j) {
                const int sp = lane + 32 * j;
                const int ts = t0 + i * TT + (sp << slog2);
                const bool need = sp < nsp && ts < t1;
                const bool bad = need && (pg[j] < 0 || pg[j] >= a.c.num_pages);
                if (bad) fault(a.st, CHK_PAGE, pg[j]);
                go[j] = need && !bad;
                if (go[j]) bytes += (uint32_t)SPAN * D * 2;
                const unsigned bw = __ballot_sync(0xffffffffu, bad);
                if (lane == 0) badm[s * 8 + j] = bw;
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, o);
            if (lane == 0) tc::mbar_arrive_expect_tx(full + s, bytes);
            __syncwarp();
#pragma unroll
            for (int j = 0; j < MAXJ; ++j) {
                if (!go[j]) continue;
                const int sp = lane + 32 * j;
                const int ts = t0 + i * TT + (sp << slog2);
                const uint16_t *src =
                    a.c.k + ((((size_t)pg[j] * a.c.Hkv + g) << a.c.Plog2) + (ts & Pm)) * D;
                tc::bulk_load(dst + ((size_t)sp << slog2) * D * 2, src, (uint32_t)SPAN * D * 2, full + s);
            }
            issued = i + 1;
            fetch(i + 1);
        }
        if (issued < ntiles) {
            // the consumers stopped releasing stages: record it and wait
            // (bounded) for the copies still in flight before the CTA's shared
            // memory is released
            *abort_flag = 1;
            if (lane == 0) {
                record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, issued);
                const uint64_t dl = tc::globaltimer() + kScoreWaitNs;
                volatile int zero = 0;
                for (int j = max(0, issued - NS); j < issued; ++j)
                    tc::mbar_wait(full + j % NS, (uint32_t)(j / NS) & 1u, dl, &zero);
            }
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int gl = lane & (G - 1), sub = lane / G;
    // partial p = (row u, head j) = u * HPG + j lives at position p ^ gl, so the
    // lane reads its rows in the order u ^ (gl >> HL) and holds its query heads
    // in the order j ^ (gl & (HPG - 1))
    const int ux = gl >> HL, jx = gl & (HPG - 1);
    float qv[HPG][8];
#pragma unroll
    for (int jj = 0; jj < HPG; ++jj) {
        const size_t row = (size_t)b * a.Hq + g * HPG + (jj ^ jx);
        if (QF32) {
            const float4 *qp = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.q) +
                                                                row * D + gl * 8);
            float4 x0 = __ldg(qp), x1 = __ldg(qp + 1);
            qv[jj][0] = x0.x; qv[jj][1] = x0.y; qv[jj][2] = x0.z; qv[jj][3] = x0.w;
            qv[jj][4] = x1.x; qv[jj][5] = x1.y; qv[jj][6] = x1.z; qv[jj][7] = x1.w;
        } else {
            uint4 w = ldg_nc_v4(reinterpret_cast<const uint16_t *>(a.q) + row * D + gl * 8);
            qv[jj][0] = bf_lo(w.x); qv[jj][1] = bf_hi(w.x); qv[jj][2] = bf_lo(w.y); qv[jj][3] = bf_hi(w.y);
            qv[jj][4] = bf_lo(w.z); qv[jj][5] = bf_hi(w.z); qv[jj][6] = bf_lo(w.w); qv[jj][7] = bf_hi(w.w);
        }
    }
    // after the reduction lane gl holds partial gl: row gl >> HL, head gl & (HPG-1)
    float *sout = a.scores + ((size_t)b * a.Hq + g * HPG + (gl & (HPG - 1))) * a.Lcap;
    const int my_u = gl >> HL;

    for (int i = 0; i < ntiles; ++i) {
        const int s = i % NS;
        const bool ok = __all_sync(0xffffffffu,
                                   tc::mbar_wait(full + s, (uint32_t)(i / NS) & 1u, deadline, abort_flag));
        if (!ok) {
            // a copy never completed: record it and stop this warp
            *abort_flag = 1;
            if (lane == 0) record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, i);
            break;
        }
        const uint8_t *stage = sm + s * Gm::STAGE + gl * 16;
        const int tb = t0 + i * TT;
#pragma unroll
        for (int st = 0; st < Gm::R; ++st) {
            const int r0 = st * Gm::STEP + (warp * GPW + sub) * U;   // first row of this group
            float part[G];
#pragma unroll
            for (int uu = 0; uu < U; ++uu) {
                const uint4 kr = *reinterpret_cast<const uint4 *>(stage + (size_t)(r0 + (uu ^ ux)) * D * 2);
                const float kf[8] = {bf_lo(kr.x), bf_hi(kr.x), bf_lo(kr.y), bf_hi(kr.y),
                                     bf_lo(kr.z), bf_hi(kr.z), bf_lo(kr.w), bf_hi(kr.w)};
#pragma unroll
                for (int jj = 0; jj < HPG; ++jj) {
                    float p = qv[jj][0] * kf[0];
#pragma unroll
                    for (int e = 1; e < 8; ++e) p = fmaf(qv[jj][e], kf[e], p);
                    part[uu * HPG + jj] = p;
                }
            }
            const float sc = transpose_reduce<G>(part);
            const int r = r0 + my_u;
            const int sp = r >> slog2;
            const bool bad = (badm[s * 8 + (sp >> 5)] >> (sp & 31)) & 1u;
            if (tb + r < t1) sout[tb + r] = bad ? -INFINITY : sc;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(empty + s);
    }
}

// block-wide exclusive scan of small non-negative ints; returns the total
__device__ __forceinline__ int block_excl_scan(int v, int *warp_tot, int &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (blockDim.x >> 5) ? warp_tot[lane] : 0;
        int z = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += y;
        }
        warp_tot[lane] = z - w;          // exclusive prefix of warp totals
        if (lane == 31) warp_tot[32] = z;
    }
    __syncthreads();
    const int r = warp_tot[warp] + x - v;
    total = warp_tot[32];
    __syncthreads();
    return r;
}

// One radix digit pass over the elements whose key matches (prefix, pmask):
// histogram of the digit at `shift` (nbits wide), then the digit D holding the
// need-th largest element; `need` drops by the count above D.
// Digit selection after a histogram pass: the digit D holding the need-th
// largest element among those matching (prefix, pmask); `need` drops by the
// count above D and D is appended to the prefix.
__device__ void pick_digit(int shift, int nbits, uint32_t &prefix, uint32_t &pmask, unsigned &need,
                           unsigned *hist, int *warp_tot, unsigned &s_digit, unsigned &s_above)
{
    const int tid = threadIdx.x;
    const int nb = 1 << nbits;
    // thread i owns bins in descending order [nb - (i+1)*per, nb - i*per)
    const int per = nb / kSelThreads;
    int mine = 0;
    for (int j = 0; j < per; ++j) mine += hist[nb - 1 - tid * per - j];
    int total;
    const int before = block_excl_scan(mine, warp_tot, total);   // count in higher bins
    if ((unsigned)before < need && need <= (unsigned)(before + mine)) {
        int run = before;
        for (int j = 0; j < per; ++j) {
            const int bin = nb - 1 - tid * per - j;
            const int c = hist[bin];
            if ((unsigned)(run + c) >= need) {
                s_digit = (unsigned)bin;
                s_above = (unsigned)run;
                break;
            }
            run += c;
        }
    }
    __syncthreads();
    need -= s_above;
    prefix |= s_digit << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    __syncthreads();
}

// BATCH keys per thread are loaded before any is counted, so that many loads
// are in flight.
template <int BATCH, typename KeyAt>
__device__ void digit_pass(KeyAt key_at, int n, int shift, int nbits, uint32_t &prefix, uint32_t &pmask,
                           unsigned &need, unsigned *hist, int *warp_tot, unsigned &s_digit, unsigned &s_above)
{
    const int tid = threadIdx.x;
    const int nb = 1 << nbits;
    for (int i = tid; i < nb; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int t0 = 0; t0 < n; t0 += kSelThreads * BATCH) {
        uint32_t kk[BATCH];
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int t = t0 + u * kSelThreads + tid;
            kk[u] = t < n ? key_at(t) : 0u;
        }
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int t = t0 + u * kSelThreads + tid;
            const bool act = t < n && (kk[u] & pmask) == prefix;
            if (act) atomicAdd(&hist[(kk[u] >> shift) & (nb - 1)], 1u);
        }
    }
    __syncthreads();
    pick_digit(shift, nbits, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
}

constexpr int kCandCap = 4096;

// Exact top-k of one (sequence, query head) score row.  Pass 1 histograms the
// top 11 bits of the order-preserving key over the whole row; pass 2 reads the
// row once more, writing a position bitmap of the elements whose top digit is
// above the threshold digit (warp ballots, no atomics) and collecting the
// threshold-digit elements as candidates in shared memory.  The remaining 21
// bits are resolved on the candidates only, and the output is emitted in
// position order from the bitmaps.  If the candidates overflow their buffer,
// the remaining digit passes and the emission read the full row instead.
// Dynamic shared memory: 2 bitmaps of Lcap bits + 2 x kCandCap words.
__global__ void __launch_bounds__(kSelThreads, 2) k_topk_select(const TopkArgs a)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t dsm[];
    __shared__ unsigned hist[2048];
    __shared__ int warp_tot[33];
    __shared__ unsigned s_digit, s_above, s_ncand;

    const int row = blockIdx.x;
    const int b = row / a.Hq;
    const int tid = threadIdx.x, lane = tid & 31;
    const int Lcap = a.c.max_pages << a.c.Plog2;
    int L = __ldg(a.c.sl + b);
    if (L < 0 || L > Lcap) L = L < 0 ? 0 : Lcap;   // recorded by the scoring kernel
    const int k = a.k;
    int32_t *idx = a.idx + (size_t)row * k;
    const float *sc = a.scores + (size_t)row * a.Lcap;

    if (L <= k) {
        for (int i = tid; i < k; i += kSelThreads) idx[i] = i < L ? i : -1;
        if (tid == 0) a.cnt[row] = L;
        return;
    }
    const int nw = (L + 31) >> 5;
    uint32_t *above = dsm;                 // [nw] elements certainly selected
    uint32_t *eqmap = dsm + ((Lcap + 31) >> 5);   // [nw] elements equal to the threshold
    uint32_t *ckey = eqmap + ((Lcap + 31) >> 5);
    uint32_t *cpos = ckey + kCandCap;
    auto full_key = [&](int t) { return f2key(__ldcg(sc + t)); };

    // pass 1: histogram of the top 11 key bits over the whole row, 16-byte
    // loads (the row buffer holds a multiple of 16 entries, so the last vector
    // is readable; entries at or past L are not counted)
    const float4 *row4 = reinterpret_cast<const float4 *>(sc);
    const int nv = (L + 3) >> 2;
    for (int i = tid; i < 2048; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int v0 = 0; v0 < nv; v0 += kSelThreads * 4) {
        float4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int v = v0 + u * kSelThreads + tid;
            x[u] = v < nv ? __ldcg(row4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int t = (v0 + u * kSelThreads + tid) * 4;
            if (t + 3 < L) {
                atomicAdd(&hist[f2key(x[u].x) >> 21], 1u);
                atomicAdd(&hist[f2key(x[u].y) >> 21], 1u);
                atomicAdd(&hist[f2key(x[u].z) >> 21], 1u);
                atomicAdd(&hist[f2key(x[u].w) >> 21], 1u);
            } else if (t < L) {
                atomicAdd(&hist[f2key(x[u].x) >> 21], 1u);
                if (t + 1 < L) atomicAdd(&hist[f2key(x[u].y) >> 21], 1u);
                if (t + 2 < L) atomicAdd(&hist[f2key(x[u].z) >> 21], 1u);
            }
        }
    }
    __syncthreads();
    uint32_t prefix = 0, pmask = 0;
    unsigned need = (unsigned)k;
    pick_digit(21, 11, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
    const uint32_t D1 = prefix >> 21;

    // pass 2: bitmap of top digit > D1, candidates with top digit == D1.  A
    // lane holds 8 consecutive entries (two adjacent 16-byte loads), so 4
    // lanes make one 32-bit bitmap word: each lane's byte is shifted into
    // place and OR-ed across the 4 lanes with two xor shuffles.
    if (tid == 0) s_ncand = 0;
    __syncthreads();
    const int no = (L + 7) >> 3;   // octets of entries (the row buffer is a multiple of 16 long)
    for (int o = tid; o - tid < no; o += kSelThreads) {
        const float4 x0 = o < no ? __ldcg(row4 + 2 * o) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 x1 = o < no ? __ldcg(row4 + 2 * o + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        const int t = o * 8;
        const uint32_t kk[8] = {f2key(x0.x), f2key(x0.y), f2key(x0.z), f2key(x0.w),
                                f2key(x1.x), f2key(x1.y), f2key(x1.z), f2key(x1.w)};
        uint32_t hb = 0, eb = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool in = t + j < L;
            const uint32_t dg = kk[j] >> 21;
            hb |= (uint32_t)(in && dg > D1) << j;
            eb |= (uint32_t)(in && dg == D1) << j;
        }
        uint32_t hw = hb << (8 * (lane & 3));
        hw |= __shfl_xor_sync(0xffffffffu, hw, 1);
        hw |= __shfl_xor_sync(0xffffffffu, hw, 2);
        if ((lane & 3) == 0 && (o >> 2) < nw) {
            above[o >> 2] = hw;
            eqmap[o >> 2] = 0u;
        }
        if (eb) {
            unsigned slot = atomicAdd(&s_ncand, (unsigned)__popc(eb));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (eb >> j & 1) {
                    if (slot < kCandCap) {
                        ckey[slot] = kk[j];
                        cpos[slot] = (uint32_t)(t + j);
                    }
                    ++slot;
                }
            }
        }
    }
    __syncthreads();
    const unsigned ncand = s_ncand;
    int written = 0;
    if (ncand <= kCandCap) {
        auto cand_key = [&](int i) { return ckey[i]; };
        digit_pass<2>(cand_key, (int)ncand, 10, 11, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
        digit_pass<2>(cand_key, (int)ncand, 0, 10, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
        const uint32_t T = prefix;   // the k-th largest key; take `need` elements equal to T
        for (int i = tid; i < (int)ncand; i += kSelThreads) {
            const uint32_t key = ckey[i], t = cpos[i];
            if (key > T) atomicOr(&above[t >> 5], 1u << (t & 31));
            else if (key == T) atomicOr(&eqmap[t >> 5], 1u << (t & 31));
        }
        __syncthreads();
        // keep the first `need` equal elements (position order), then emit
        const int per = (nw + kSelThreads - 1) / kSelThreads;
        const int w0 = tid * per, w1 = min(w0 + per, nw);
        int eqc = 0;
        for (int w = w0; w < w1; ++w) eqc += __popc(eqmap[w]);
        int eq_tot;
        int eq_before = block_excl_scan(eqc, warp_tot, eq_tot);
        int selc = 0;
        for (int w = w0; w < w1; ++w) {
            uint32_t e = eqmap[w];
            while (e) {
                const int bit = __ffs(e) - 1;
                e &= e - 1;
                if ((unsigned)eq_before < need) above[w] |= 1u << bit;
                ++eq_before;
            }
            selc += __popc(above[w]);
        }
        int sel_tot;
        int pos = block_excl_scan(selc, warp_tot, sel_tot);
        for (int w = w0; w < w1; ++w) {
            uint32_t m = above[w];
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1;
                if (pos < k) idx[pos] = w * 32 + bit;
                ++pos;
            }
        }
        written = sel_tot;
    } else {
        // candidate overflow (many equal or clustered scores): full-row passes
        digit_pass<8>(full_key, L, 10, 11, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
        digit_pass<8>(full_key, L, 0, 10, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
        const uint32_t T = prefix;
        int eq_seen = 0;
#pragma unroll 1
        for (int t0 = 0; t0 < L; t0 += kSelThreads) {
            const int t = t0 + tid;
            const uint32_t key = t < L ? full_key(t) : 0u;
            const int is_eq = (t < L && key == T) ? 1 : 0;
            int eq_tot;
            const int eq_rank = block_excl_scan(is_eq, warp_tot, eq_tot);
            const int sel = (t < L && (key > T || (is_eq && (unsigned)(eq_seen + eq_rank) < need))) ? 1 : 0;
            int sel_tot;
            const int pos = block_excl_scan(sel, warp_tot, sel_tot);
            if (sel) idx[written + pos] = t;
            written += sel_tot;
            eq_seen += eq_tot;
        }
    }
    if (tid == 0) a.cnt[row] = written;
}

size_t select_smem_bytes(int Lcap) { return (size_t)2 * ((Lcap + 31) / 32) * 4 + (size_t)2 * kCandCap * 4; }

template <int D, int HPG, bool QF32>
cudaError_t launch_score(const TopkArgs &a, cudaStream_t s)
{
    const int Lcap = a.c.max_pages << a.c.Plog2;
    dim3 grid((Lcap + kScoreChunk - 1) / kScoreChunk, a.c.Hkv, a.c.B);
    constexpr int smem = ScoreGeom<D, HPG>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(k_topk_score<D, HPG, QF32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (cudaError_t e_ = launch_pdl(k_topk_score<D, HPG, QF32>, dim3(grid), dim3(ScoreGeom<D, HPG>::THREADS), smem, s, a)) return e_;
    return cudaGetLastError();
}

template <int D, bool QF32>
cudaError_t launch_score_hpg(const TopkArgs &a, int hpg, cudaStream_t s)
{
    switch (hpg) {
    case 1: return launch_score<D, 1, QF32>(a, s);
    case 2: return launch_score<D, 2, QF32>(a, s);
    case 4: return launch_score<D, 4, QF32>(a, s);
    case 8: return launch_score<D, 8, QF32>(a, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t s)
{
    if (a.c.B * a.Hq == 0) return cudaSuccess;
    const int hpg = a.Hq / a.c.Hkv;
    cudaError_t e;
    if (a.c.D == 64)
        e = a.q_f32 ? launch_score_hpg<64, true>(a, hpg, s) : launch_score_hpg<64, false>(a, hpg, s);
    else
        e = a.q_f32 ? launch_score_hpg<128, true>(a, hpg, s) : launch_score_hpg<128, false>(a, hpg, s);
    if (e != cudaSuccess) return e;
    const int Lcap = a.c.max_pages << a.c.Plog2;
    const size_t smem = select_smem_bytes(Lcap);
    e = cudaFuncSetAttribute(k_topk_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (cudaError_t e_ = launch_pdl(k_topk_select, dim3(a.c.B * a.Hq), dim3(kSelThreads), smem, s, a)) return e_;
    return cudaGetLastError();
}

}  // namespace sa
