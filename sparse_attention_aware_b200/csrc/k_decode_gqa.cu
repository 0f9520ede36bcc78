// Split-KV decode over a block-list selection for a whole GQA group, on
// mma.sync tensor cores.
//
// Method: the block-aligned span masks of the DA modes and of LoZA streaming
// ("语言模型能自己决定该看哪里吗？", DA state machine section;
// "稀疏注意力机制创新…", section "二、ZigZag架构") select one set of page
// segments per sequence, shared by every head.  So the query heads of a GQA
// group read the same K/V rows, and with 8 heads per kv head the work is
// ~8 flop per byte of K/V -- at the limit of fp32 SIMT issue, so the two
// contractions go to the tensor cores.  Partials per split are merged by the
// common combine kernel ("稀疏注意力机制创新…", section "四、从外卖到AI":
// SplitKV-and-Combine).
//
// One CTA = (split s, kv head g, sequence b), kPW warps.  The split owns a
// contiguous range of the sequence's list entries (balanced by entry count;
// an entry is at most one page); a sequence uses only as many of the S splits
// as give each at least ~128 tokens.  The warps take the split's entries
// round-robin and run independently until the final merge: a warp holds up
// to 32 of its entries in registers (one per lane: validated, page-mapped)
// and walks them as pieces of at most 16 consecutive rows of one page.  A
// piece's 16 K rows and 16 V rows are fetched by 32 bulk copies (one row per
// lane; rows past the entry's end repeat its last row, so every piece is
// 16 finite rows and its probability is 0 there) into the warp's kNST-stage
// ring, rows padded to D*2 + 16 bytes so that 8-row ldmatrix reads hit 32
// distinct banks; each stage completes on its own mbarrier.  Every wait is
// bounded (globaltimer deadline, shared abort flag): on expiry the warp
// records SA_ERR_TIMEOUT, waits (bounded) for its copies still in flight and
// leaves its loop.
//
// The contractions take the 16 tokens of a piece as the M rows and the
// group's heads as the N columns of m16n8k16 (no padding rows for 8 heads):
// S^T = K Q^T (fp32 accumulate; an fp32 query is split into bf16 high and low
// parts, two MMAs), online softmax per head (column) in the base-2 domain,
// P^T as bf16 moved into the B-operand layout with movmatrix, then
// O^T += V^T P^T with V^T read by transposing ldmatrix.
#include "sa_internal.h"
#include "tc_ptx.cuh"

namespace sa {
namespace {

constexpr int kPW = 4;                   // warps per CTA
constexpr int kGThreads = kPW * 32;
constexpr int kPR = 16;                  // rows per piece (the MMA's M)
constexpr int kNST = 2;                  // ring stages per warp
constexpr int kSplitTokens = 128;        // a split of a sequence's list covers at least ~this many tokens
constexpr uint64_t kGqaWaitNs = 1000ull * 1000 * 1000;   // 1 s

template <int D>
struct GqaSmem {
    static constexpr int ROW = D * 2 + 16;                      // padded row, bytes
    static constexpr int STAGE = 2 * kPR * ROW;                 // K rows, then V rows
    static constexpr int RING = kPW * kNST * STAGE;
    static constexpr int MERGE = kPW * (16 * D + 32) * 4;       // per-warp O, m, l (up to 16 heads)
    static constexpr int BODY = RING > MERGE ? RING : MERGE;
    static constexpr int BYTES = BODY + kPW * kNST * 8 + 16;    // + mbarriers, abort flag
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// transpose of an 8x8 b16 matrix held in the mma fragment layout
__device__ __forceinline__ uint32_t movm_t(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi)
{
    return (uint32_t)f2bf(lo) | ((uint32_t)f2bf(hi) << 16);
}

__device__ __forceinline__ float bf_round(float x) { return __uint_as_float((uint32_t)f2bf(x) << 16); }

// Query words for head row `row_off` (zero for padding heads), element pair
// (col, col + 1): bf16 high part, and for an fp32 query also the bf16 low part
// (x - bf16(x)), so that hi + lo carries the query to ~16 bits.
template <bool QF32>
__device__ __forceinline__ void q_pair(const void *q, size_t row_off, bool valid, int col, uint32_t &hi, uint32_t &lo)
{
    hi = 0u;
    lo = 0u;
    if (!valid) return;
    if (QF32) {
        const float2 x = *reinterpret_cast<const float2 *>(reinterpret_cast<const float *>(q) + row_off + col);
        const float h0 = bf_round(x.x), h1 = bf_round(x.y);
        hi = pack_bf2(h0, h1);
        lo = pack_bf2(x.x - h0, x.y - h1);
    } else {
        hi = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint16_t *>(q) + row_off + col);
    }
}

// NH = 8-head column blocks (1: up to 8 heads per kv head, 2: up to 16)
template <int D, int NH, bool QF32>
__global__ void __launch_bounds__(kGThreads) k_decode_gqa_blocks(const DecodeArgs a)
{
    pdl_wait();
    pdl_trigger();
    using SM = GqaSmem<D>;
    constexpr int KK = D / 16;   // k-steps of S^T = K Q^T
    constexpr int MT = D / 16;   // m-tiles of O^T
    constexpr int NQ = QF32 ? 2 : 1;
    extern __shared__ __align__(128) uint8_t sm[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SM::BODY);   // [kPW][kNST]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + kPW * kNST);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;   // mma group id / thread in group
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int HPG = a.Hq / a.c.Hkv;
    DevStatus *st = a.st;

    const int Lcap = a.c.max_pages << a.c.Plog2;
    int L = __ldg(a.c.sl + b);
    if (L < 0 || L > Lcap) {
        if (tid == 0 && s == 0 && g == 0) fault(st, CHK_SEQ_LEN, L);
        L = L < 0 ? 0 : Lcap;
    }
    int ne = __ldg(a.ecnt + b);
    if (ne < 0 || ne > a.max_blocks) {
        if (tid == 0 && s == 0 && g == 0) fault(st, CHK_BLOCK_ENTRY, ne);
        ne = ne < 0 ? 0 : a.max_blocks;
    }
    // The sequence uses Sb <= S splits of at least kSplitTokens / P entries
    // each (an entry is at most one page), so a short list is not spread over
    // many CTAs that each pay the fixed cost of a split; the splits past Sb
    // leave an empty partial (l = 0), which the combine skips.
    const int per = max(1, kSplitTokens >> a.c.Plog2);
    const int Sb = min(a.S, max(1, (ne + per - 1) / per));
    if (s >= Sb) {
        for (int j = tid; j < min(HPG, 16); j += kGThreads) {
            const size_t row = (size_t)b * a.Hq + g * HPG + j;
            a.part_ml[(row * a.S + s) * 2 + 0] = -INFINITY;
            a.part_ml[(row * a.S + s) * 2 + 1] = 0.f;
        }
        return;
    }
    const int e0 = (int)((long long)ne * s / Sb), e1 = (int)((long long)ne * (s + 1) / Sb);
    const int4 *ent = reinterpret_cast<const int4 *>(a.ent) + (size_t)b * a.max_blocks;
    const int32_t *ptb = a.c.pt + (size_t)b * a.c.max_pages;
    const int P = 1 << a.c.Plog2;

    if (tid == 0) {
        for (int i = 0; i < kPW * kNST; ++i) tc::mbar_init(bars + i, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    // this lane's entry of the warp's first window, loaded before the query so
    // that the two loads overlap
    int4 en_first = make_int4(0, 0, 0, 0);
    if (e0 + warp + kPW * lane < e1) en_first = ent[e0 + warp + kPW * lane];

    // query B fragments: column n of block nh is head nh*8 + gq (zero past HPG);
    // k pairs (2tq, 2tq+1) and (2tq+8, 2tq+9) of k-step kk
    uint32_t qb[NQ][NH][KK][2];
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) {
        const int h = nh * 8 + gq;
        const size_t r0 = ((size_t)b * a.Hq + g * HPG + h) * D;
        const bool v = h < HPG;
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            uint32_t lo0, lo1;
            q_pair<QF32>(a.q, r0, v, kk * 16 + 2 * tq, qb[0][nh][kk][0], lo0);
            q_pair<QF32>(a.q, r0, v, kk * 16 + 2 * tq + 8, qb[0][nh][kk][1], lo1);
            if (QF32) {
                qb[NQ - 1][nh][kk][0] = lo0;
                qb[NQ - 1][nh][kk][1] = lo1;
            }
        }
    }
    __syncthreads();   // mbarriers initialised

    // O^T fragments: o[mt][nh][i] = O[head nh*8 + 2tq + (i & 1)][d = mt*16 + gq + 8*(i >> 1)]
    float o[MT][NH][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nh = 0; nh < NH; ++nh) o[mt][nh][0] = o[mt][nh][1] = o[mt][nh][2] = o[mt][nh][3] = 0.f;
    float mh[NH][2], lh[NH][2];   // heads nh*8 + 2tq + j (l: this thread's tokens only)
#pragma unroll
    for (int nh = 0; nh < NH; ++nh) mh[nh][0] = mh[nh][1] = -INFINITY, lh[nh][0] = lh[nh][1] = 0.f;

    uint64_t *wbar = bars + warp * kNST;
    const uint32_t wring = sbase + warp * kNST * SM::STAGE;
    uint8_t *wring_g = sm + warp * kNST * SM::STAGE;
    const uint64_t deadline = tc::globaltimer() + kGqaWaitNs;
    int gpc = 0;          // pieces this warp has consumed (stage = gpc % kNST, parity = (gpc / kNST) & 1)
    bool alive = true;

    // this warp's entries: e0 + warp + kPW * j
    for (int wb = e0 + warp; wb < e1 && alive; wb += 32 * kPW) {
        // one entry per lane: validate and map (len 0 = skipped)
        const int e = wb + kPW * lane;
        int pg = 0, lo = 0, len = 0;
        if (e < e1) {
            const int4 en = wb == e0 + warp ? en_first : ent[e];
            const int x = en.x, l0 = en.y, hi = en.z;
            bool ok = l0 >= 0 && l0 < hi && hi <= P && x >= 0 && x < a.c.max_pages;
            if (!ok) fault(st, CHK_BLOCK_ENTRY, e);
            if (ok && (x << a.c.Plog2) + hi > L) {
                fault(st, CHK_INDEX, (x << a.c.Plog2) + hi - 1);
                ok = false;
            }
            if (ok) {
                pg = __ldg(ptb + x);
                if (pg < 0 || pg >= a.c.num_pages) {
                    fault(st, CHK_PAGE, pg);
                    ok = false;
                }
            }
            if (ok) {
                lo = l0;
                len = hi - l0;
            }
        }
        // pieces per entry, inclusive prefix over the lanes
        const int npc = (len + kPR - 1) / kPR;
        int incl = npc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const int np = __shfl_sync(0xffffffffu, incl, 31);

        // piece n: lane of its entry, then its first row and row count
        auto locate = [&](int n, size_t &row0, int &cnt) {
            const unsigned m = __ballot_sync(0xffffffffu, incl > n);
            const int src = __ffs(m) - 1;
            const int e_pg = __shfl_sync(0xffffffffu, pg, src);
            const int e_lo = __shfl_sync(0xffffffffu, lo, src);
            const int e_len = __shfl_sync(0xffffffffu, len, src);
            const int e_ex = __shfl_sync(0xffffffffu, incl - npc, src);
            const int j = n - e_ex;
            cnt = min(kPR, e_len - j * kPR);
            row0 = (((size_t)e_pg * a.c.Hkv + g) << a.c.Plog2) + e_lo + j * kPR;
        };
        auto issue = [&](int n, int stage) {
            size_t row0;
            int cnt;
            locate(n, row0, cnt);
            if (lane == 0) tc::mbar_arrive_expect_tx(wbar + stage, (uint32_t)(2 * kPR * D * 2));
            __syncwarp();
            const int r = lane & (kPR - 1);
            const size_t row = row0 + min(r, cnt - 1);
            const uint16_t *src = (lane < kPR ? a.c.k : a.c.v) + row * D;
            tc::bulk_load(wring_g + stage * SM::STAGE + (lane >> 4) * kPR * SM::ROW + r * SM::ROW, src,
                          (uint32_t)(D * 2), wbar + stage);
        };

        const int pre = min(np, kNST);
        for (int n = 0; n < pre; ++n) issue(n, (gpc + n) % kNST);
        int n = 0;
        for (; n < np; ++n, ++gpc) {
            const int stage = gpc % kNST;
            const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(wbar + stage, (uint32_t)(gpc / kNST) & 1u,
                                                                  deadline, abort_flag));
            if (!ok) {
                *abort_flag = 1;
                if (lane == 0) record(st, SA_ERR_TIMEOUT, CHK_WAIT, n);
                alive = false;
                break;
            }
            size_t row0_unused;
            int cnt;
            locate(n, row0_unused, cnt);
            const uint32_t kt = wring + stage * SM::STAGE, vt = kt + kPR * SM::ROW;

            // ---- S^T = K Q^T: 16 tokens x (NH*8) heads
            float sc[NH][4];
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) sc[nh][0] = sc[nh][1] = sc[nh][2] = sc[nh][3] = 0.f;
            {
                const int mi = lane >> 3;
                const uint32_t rowa = kt + ((mi & 1) * 8 + (lane & 7)) * SM::ROW + (mi >> 1) * 16;
#pragma unroll
                for (int kk = 0; kk < KK; ++kk) {
                    uint32_t ka[4];
                    ldsm_x4(rowa + kk * 32, ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
                        for (int qi = 0; qi < NQ; ++qi) mma16816(sc[nh], ka, qb[qi][nh][kk][0], qb[qi][nh][kk][1]);
                }
            }
            // ---- online softmax per head column; rows gq (elements 0, 1) and gq + 8 (2, 3)
            const bool ok0 = gq < cnt, ok1 = gq + 8 < cnt;
            uint32_t pb[NH][2];
#pragma unroll
            for (int nh = 0; nh < NH; ++nh) {
                const float s0 = ok0 ? sc[nh][0] * a.qscale : -INFINITY;
                const float s1 = ok0 ? sc[nh][1] * a.qscale : -INFINITY;
                const float s2 = ok1 ? sc[nh][2] * a.qscale : -INFINITY;
                const float s3 = ok1 ? sc[nh][3] * a.qscale : -INFINITY;
                float x0 = fmaxf(s0, s2), x1 = fmaxf(s1, s3);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
                    x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
                }
                const float n0 = fmaxf(mh[nh][0], x0), n1 = fmaxf(mh[nh][1], x1);
                const float b0 = n0 == -INFINITY ? 0.f : n0, b1 = n1 == -INFINITY ? 0.f : n1;
                const float al0 = ex2(mh[nh][0] - b0), al1 = ex2(mh[nh][1] - b1);   // 0 while a head is empty
                mh[nh][0] = n0;
                mh[nh][1] = n1;
                const float p0 = ex2(s0 - b0), p1 = ex2(s1 - b1), p2 = ex2(s2 - b0), p3 = ex2(s3 - b1);
                lh[nh][0] = lh[nh][0] * al0 + (p0 + p2);
                lh[nh][1] = lh[nh][1] * al1 + (p1 + p3);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    o[mt][nh][0] *= al0;
                    o[mt][nh][1] *= al1;
                    o[mt][nh][2] *= al0;
                    o[mt][nh][3] *= al1;
                }
                // P^T rows 0-7 / 8-15 (tokens) x 8 heads -> B fragments (k = tokens)
                pb[nh][0] = movm_t(pack_bf2(p0, p1));
                pb[nh][1] = movm_t(pack_bf2(p2, p3));
            }
            // ---- O^T += V^T P^T
            {
                const int mi = lane >> 3;
                const uint32_t rowa = vt + ((mi >> 1) * 8 + (lane & 7)) * SM::ROW + (mi & 1) * 16;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t va[4];
                    ldsm_x4_t(rowa + mt * 32, va[0], va[1], va[2], va[3]);
#pragma unroll
                    for (int nh = 0; nh < NH; ++nh) mma16816(o[mt][nh], va, pb[nh][0], pb[nh][1]);
                }
            }
            __syncwarp();   // every lane is done with this stage before it is refilled
            if (n + kNST < np) issue(n + kNST, stage);
        }
        if (!alive) {
            // copies still in flight land before the CTA's shared memory is released
            const uint64_t dl = tc::globaltimer() + kGqaWaitNs;
            volatile int zero = 0;
            for (int m = n; m < min(np, n + kNST); ++m, ++gpc)
                tc::mbar_wait(wbar + gpc % kNST, (uint32_t)(gpc / kNST) & 1u, dl, &zero);
        }
    }

    // ---- merge the warps' states through shared memory
#pragma unroll
    for (int nh = 0; nh < NH; ++nh)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) lh[nh][j] += __shfl_xor_sync(0xffffffffu, lh[nh][j], off);
    __syncthreads();
    float *mo = reinterpret_cast<float *>(sm);                 // [warp][16][D]
    float *mm = mo + kPW * 16 * D;                              // [warp][16]
    float *ml = mm + kPW * 16;                                  // [warp][16]
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nh = 0; nh < NH; ++nh)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int h = nh * 8 + 2 * tq + (i & 1), d = mt * 16 + gq + 8 * (i >> 1);
                mo[(warp * 16 + h) * D + d] = o[mt][nh][i];
            }
    if (gq == 0) {
#pragma unroll
        for (int nh = 0; nh < NH; ++nh)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                mm[warp * 16 + nh * 8 + 2 * tq + j] = mh[nh][j];
                ml[warp * 16 + nh * 8 + 2 * tq + j] = lh[nh][j];
            }
    }
    __syncthreads();
    const int nrow = min(HPG, NH * 8);
    for (int i = tid; i < nrow * D; i += kGThreads) {
        const int j = i / D, c = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kPW; ++w) M = fmaxf(M, mm[w * 16 + j]);
        float O = 0.f, Ls = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kPW; ++w) {
                const float mw = mm[w * 16 + j];
                if (mw == -INFINITY) continue;
                const float wgt = ex2(mw - M);
                O = fmaf(wgt, mo[(w * 16 + j) * D + c], O);
                Ls = fmaf(wgt, ml[w * 16 + j], Ls);
            }
        }
        const size_t row = (size_t)b * a.Hq + g * HPG + j;
        a.part_o[(row * a.S + s) * D + c] = O;
        if (c == 0) {
            a.part_ml[(row * a.S + s) * 2 + 0] = M;
            a.part_ml[(row * a.S + s) * 2 + 1] = Ls;
        }
    }
}

template <int D, int NH, bool QF32>
cudaError_t launch_gqa(const DecodeArgs &a, cudaStream_t s)
{
    constexpr int smem = GqaSmem<D>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(k_decode_gqa_blocks<D, NH, QF32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.S, a.c.Hkv, a.c.B);
    if (cudaError_t e_ = launch_pdl(k_decode_gqa_blocks<D, NH, QF32>, dim3(grid), dim3(kGThreads), smem, s, a))
        return e_;
    return cudaGetLastError();
}

template <int D, bool QF32>
cudaError_t launch_gqa_nh(const DecodeArgs &a, cudaStream_t s)
{
    return a.Hq / a.c.Hkv <= 8 ? launch_gqa<D, 1, QF32>(a, s) : launch_gqa<D, 2, QF32>(a, s);
}

}  // namespace

bool decode_gqa_supported(const DecodeArgs &a) { return a.blocks && a.Hq / a.c.Hkv <= 16; }

cudaError_t launch_decode_gqa_split(const DecodeArgs &a, cudaStream_t s)
{
    if (a.c.D == 64) return a.q_f32 ? launch_gqa_nh<64, true>(a, s) : launch_gqa_nh<64, false>(a, s);
    return a.q_f32 ? launch_gqa_nh<128, true>(a, s) : launch_gqa_nh<128, false>(a, s);
}

}  // namespace sa
