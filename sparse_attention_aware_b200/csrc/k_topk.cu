// Anchor-layer exact top-k per query head.
//
// Method: "Kascade稀疏注意力…", sections "核心机制：Anchor + Reuse" (exact
// top-k key indices on the anchor layer) and "头部感知（head-aware）是精度关键"
// (every head selects on its own; heads of one GQA group share only the K
// stream).
//
// k_topk_score: streams the whole K context once.  One CTA = (token chunk,
// kv head g, sequence b), 256 threads; a group of G = D/8 lanes owns one token
// row (16 B per lane, coalesced 256 B rows at D=128) and computes the raw dot
// product with every query head of the GQA group, so K is read once for all
// of them.  Scores (fp32, unscaled) go to the workspace.
//
// k_topk_select: one CTA of 1024 threads per (sequence, query head).  An
// exact radix select on the order-preserving uint32 image of the fp32 score:
// three digit passes (11, 11, 10 bits) narrow the k-th largest key to a
// single value T and the number r of elements equal to T that are still to be
// taken; the output is every element above T and the first r elements equal
// to T (ties to the lower position), in ascending position order.  Only the
// first two passes read the whole row (see the kernel comment).
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kScoreChunk = 4096;   // tokens per scoring CTA
constexpr int kSelThreads = 1024;

// Sum N = G values held by each of G lanes across the G lanes so that lane l
// ends with the full sum of value index (l % G): at every butterfly step a lane
// keeps the half of its values its lane bit selects and adds the partner's
// copy of that half (G - 1 shuffles in total instead of N * log2(G)).
template <int G>
__device__ __forceinline__ float transpose_reduce(float (&v)[G], int lane)
{
#pragma unroll
    for (int o = G / 2, cnt = G / 2; o >= 1; o >>= 1, cnt >>= 1) {
        const bool upper = lane & o;
#pragma unroll
        for (int i = 0; i < cnt; ++i) {
            const float send = upper ? v[i] : v[i + cnt];
            const float keep = upper ? v[i + cnt] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

// One group of G = D/8 lanes owns U = G/HPG consecutive token rows per step;
// the G partial sums (U rows x HPG heads) are reduced with transpose_reduce,
// after which lane gl holds row gl / HPG, head gl % HPG.
template <int D, int HPG, bool QF32>
__global__ void __launch_bounds__(256) k_topk_score(const TopkArgs a)
{
    constexpr int G = D / 8, GPW = 32 / G, NG = 8 * GPW;
    constexpr int U = G / HPG;
    static_assert(U >= 1 && U * HPG == G, "rows per step");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gl = lane & (G - 1), sub = lane / G;
    const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int Lcap = a.c.max_pages << a.c.Plog2;
    int L = __ldg(a.c.sl + b);
    if (L < 0 || L > Lcap) {
        fault(a.st, CHK_SEQ_LEN, L);
        L = L < 0 ? 0 : Lcap;
    }
    const int t0 = chunk * kScoreChunk;
    const int t1 = min(t0 + kScoreChunk, L);
    if (t0 >= t1) return;

    float qv[HPG][8];
#pragma unroll
    for (int j = 0; j < HPG; ++j) {
        const size_t row = (size_t)b * a.Hq + g * HPG + j;
        if (QF32) {
            const float4 *qp = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.q) +
                                                                row * D + gl * 8);
            float4 x0 = __ldg(qp), x1 = __ldg(qp + 1);
            qv[j][0] = x0.x; qv[j][1] = x0.y; qv[j][2] = x0.z; qv[j][3] = x0.w;
            qv[j][4] = x1.x; qv[j][5] = x1.y; qv[j][6] = x1.z; qv[j][7] = x1.w;
        } else {
            uint4 w = ldg_nc_v4(reinterpret_cast<const uint16_t *>(a.q) + row * D + gl * 8);
            qv[j][0] = bf_lo(w.x); qv[j][1] = bf_hi(w.x); qv[j][2] = bf_lo(w.y); qv[j][3] = bf_hi(w.y);
            qv[j][4] = bf_lo(w.z); qv[j][5] = bf_hi(w.z); qv[j][6] = bf_lo(w.w); qv[j][7] = bf_hi(w.w);
        }
    }
    const int32_t *ptb = a.c.pt + (size_t)b * a.c.max_pages;
    const int Pm = (1 << a.c.Plog2) - 1;
    float *srow = a.scores + ((size_t)b * a.Hq + g * HPG) * a.Lcap;
    const int my_u = gl / HPG, my_j = gl % HPG;

    for (int base0 = t0 + warp * GPW * U; base0 < t1; base0 += NG * U) {
        const int base = base0 + sub * U;
        uint4 kr[U];
        bool ok[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = base + u;
            ok[u] = t < t1;
            int page = 0;
            if (ok[u]) {
                page = __ldg(ptb + (t >> a.c.Plog2));
                if (page < 0 || page >= a.c.num_pages) {
                    fault(a.st, CHK_PAGE, page);
                    ok[u] = false;
                }
            }
            const size_t off = ((((size_t)page * a.c.Hkv + g) << a.c.Plog2) + (t & Pm)) * D + gl * 8;
            kr[u] = ok[u] ? ldg_nc_v4(a.c.k + off) : make_uint4(0, 0, 0, 0);
        }
        float part[G];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float kf[8] = {bf_lo(kr[u].x), bf_hi(kr[u].x), bf_lo(kr[u].y), bf_hi(kr[u].y),
                                 bf_lo(kr[u].z), bf_hi(kr[u].z), bf_lo(kr[u].w), bf_hi(kr[u].w)};
#pragma unroll
            for (int j = 0; j < HPG; ++j) {
                float p = qv[j][0] * kf[0];
#pragma unroll
                for (int e = 1; e < 8; ++e) p = fmaf(qv[j][e], kf[e], p);
                part[u * HPG + j] = p;
            }
        }
        const float sc = transpose_reduce<G>(part, gl);
        const int t = base + my_u;
        bool okm = false;
#pragma unroll
        for (int u = 0; u < U; ++u) okm = (u == my_u) ? ok[u] : okm;
        // an unreadable row (bad page) scores -inf so it is never selected
        if (t < t1) srow[(size_t)my_j * a.Lcap + t] = okm ? sc : -INFINITY;
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
template <typename KeyAt>
__device__ void digit_pass(KeyAt key_at, int n, int shift, int nbits, uint32_t &prefix, uint32_t &pmask,
                           unsigned &need, unsigned *hist, int *warp_tot, unsigned &s_digit, unsigned &s_above)
{
    const int tid = threadIdx.x;
    const int nb = 1 << nbits;
    for (int i = tid; i < nb; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int t = tid; t < n; t += kSelThreads) {
        const uint32_t key = key_at(t);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
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
__global__ void __launch_bounds__(kSelThreads) k_topk_select(const TopkArgs a)
{
    extern __shared__ uint32_t dsm[];
    __shared__ unsigned hist[2048];
    __shared__ int warp_tot[33];
    __shared__ unsigned s_digit, s_above, s_ncand;

    const int row = blockIdx.x;
    const int b = row / a.Hq;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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

    uint32_t prefix = 0, pmask = 0;
    unsigned need = (unsigned)k;
    digit_pass(full_key, L, 21, 11, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
    const uint32_t D1 = prefix >> 21;

    // pass 2: bitmap of top digit > D1, candidates with top digit == D1
    if (tid == 0) s_ncand = 0;
    __syncthreads();
    for (int w0 = warp * 32; w0 < nw * 32; w0 += kSelThreads) {
        const int t = w0 + lane;
        const uint32_t key = t < L ? full_key(t) : 0u;
        const uint32_t dg = key >> 21;
        const unsigned hi = __ballot_sync(0xffffffffu, t < L && dg > D1);
        const unsigned eq = __ballot_sync(0xffffffffu, t < L && dg == D1);
        if (lane == 0) {
            above[w0 >> 5] = hi;
            eqmap[w0 >> 5] = 0u;
        }
        if (eq) {
            unsigned base = 0;
            if (lane == 0) base = atomicAdd(&s_ncand, (unsigned)__popc(eq));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (eq >> lane & 1) {
                const unsigned slot = base + __popc(eq & ((1u << lane) - 1u));
                if (slot < kCandCap) {
                    ckey[slot] = key;
                    cpos[slot] = (uint32_t)t;
                }
            }
        }
    }
    __syncthreads();
    const unsigned ncand = s_ncand;
    int written = 0;
    if (ncand <= kCandCap) {
        auto cand_key = [&](int i) { return ckey[i]; };
        digit_pass(cand_key, (int)ncand, 10, 11, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
        digit_pass(cand_key, (int)ncand, 0, 10, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
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
        digit_pass(full_key, L, 10, 11, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
        digit_pass(full_key, L, 0, 10, prefix, pmask, need, hist, warp_tot, s_digit, s_above);
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
    k_topk_score<D, HPG, QF32><<<grid, 256, 0, s>>>(a);
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
    k_topk_select<<<a.c.B * a.Hq, kSelThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace sa
