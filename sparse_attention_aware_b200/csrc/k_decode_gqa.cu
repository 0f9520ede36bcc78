// Split-KV decode over a block-list selection for a whole GQA group, on
// mma.sync tensor cores.
//
// Method: the block-aligned span masks of the DA modes and of LoZA streaming
// ("语言模型能自己决定该看哪里吗？", DA state machine section;
// "稀疏注意力机制创新…", section "二、ZigZag架构") select one set of page
// segments per sequence, shared by every head.  So the query heads of a GQA
// group read the same K/V rows, and with 8 heads per kv head the work is
// ~8 flop per byte of K/V -- at the limit of fp32 SIMT issue, so the two
// contractions (Q K^T and P V) go to the tensor cores with the group's heads
// as the M rows of an m16n8k16 MMA.  Partials per split are merged by the
// common combine kernel ("稀疏注意力机制创新…", section "四、从外卖到AI":
// SplitKV-and-Combine).
//
// One CTA = (split s, kv head g, sequence b), 4 warps.  The split owns a
// contiguous range of the sequence's list entries (balanced by entry count;
// an entry is at most one page); a sequence uses only as many of the S splits
// as give each at least ~128 tokens.  Entries are staged in shared memory in
// windows of up to kWin, validated, mapped to physical pages once, and
// prefix-summed into positions; each entry's K and V rows are prefetched into
// L2 right away (one bulk prefetch each), so the latency of the scattered page
// reads is paid about once per CTA, not once per tile.  64-token tiles of K and V rows are gathered
// with 16-byte cp.async into a double-buffered, XOR-swizzled tile (rows of
// D*2 bytes; 16-byte chunk c of row r lives at chunk c ^ (r & 7), so the
// 8-row ldmatrix reads are free of bank conflicts).  Warp w owns tokens
// [16w, 16w + 16) of a tile: S = Q K^T (fp32 accumulate; an fp32 query is
// split into bf16 high and low parts, two MMAs), online softmax per head in
// the base-2 domain, P as bf16, O += P V.  The warps' states are merged
// through shared memory at the end and written as one split partial.
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kGT = 64;                  // tokens per tile
constexpr int kGWarps = 4;               // a warp owns 16 tokens of a tile
constexpr int kGThreads = kGWarps * 32;
constexpr int kWin = 512;                // list entries staged per window
constexpr int kSplitTokens = 128;        // a split of a sequence's list covers at least ~this many tokens

template <int D>
struct GqaSmem {
    static constexpr int TILE = kGT * D * 2;                   // one K or V tile, bytes
    static constexpr int KV = 2 * 2 * TILE;                    // K and V, double buffered
    static constexpr int MERGE = kGWarps * (16 * D + 32) * 4;  // per-warp O, m, l
    static constexpr int BODY = KV > MERGE ? KV : MERGE;
    static constexpr int ENT = kWin * 16 + (kWin + 1) * 4 + kGT * 2 * 4 + 16;   // went, pre, rowok, total
    static constexpr int BYTES = BODY + ENT;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool pred)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(pred ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

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

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// start moving `bytes` (a multiple of 16, 16-byte aligned) into L2
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi)
{
    return (uint32_t)f2bf(lo) | ((uint32_t)f2bf(hi) << 16);
}

__device__ __forceinline__ float bf_round(float x) { return __uint_as_float((uint32_t)f2bf(x) << 16); }

// Query fragment words for row m (zero for padding rows), element pair
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

template <int D, bool QF32>
__global__ void __launch_bounds__(kGThreads) k_decode_gqa_blocks(const DecodeArgs a)
{
    pdl_wait();
    pdl_trigger();
    using SM = GqaSmem<D>;
    constexpr int KK = D / 16;   // k-steps of Q K^T
    constexpr int NB = D / 8;    // n-blocks of the output
    constexpr int CH = D / 8;    // 16-byte chunks per row
    extern __shared__ __align__(128) uint8_t sm[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
    int4 *went = reinterpret_cast<int4 *>(sm + SM::BODY);             // [kWin] {lo, len, page, -}
    int *pre = reinterpret_cast<int *>(sm + SM::BODY + kWin * 16);    // [kWin + 1] first position
    int *rowok = pre + kWin + 1;                                       // [2][kGT]
    int *s_tot = rowok + 2 * kGT;

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

    // query fragments: rows m = gq and gq + 8 are heads g*HPG + m when m < HPG
    uint32_t qa[KK][4], ql[QF32 ? KK : 1][4];
    {
        const size_t r0 = ((size_t)b * a.Hq + g * HPG + gq) * D;
        const size_t r1 = r0 + (size_t)8 * D;
        const bool v0 = gq < HPG, v1 = gq + 8 < HPG;
#pragma unroll
        for (int kk = 0; kk < KK; ++kk) {
            const int c = kk * 16 + 2 * tq;
            uint32_t lo[4];
            q_pair<QF32>(a.q, r0, v0, c, qa[kk][0], lo[0]);
            q_pair<QF32>(a.q, r1, v1, c, qa[kk][1], lo[1]);
            q_pair<QF32>(a.q, r0, v0, c + 8, qa[kk][2], lo[2]);
            q_pair<QF32>(a.q, r1, v1, c + 8, qa[kk][3], lo[3]);
            if (QF32) {
#pragma unroll
                for (int i = 0; i < 4; ++i) ql[QF32 ? kk : 0][i] = lo[i];
            }
        }
    }

    float o[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows gq, gq + 8 (l: this thread's part)

    for (int wb = e0; wb < e1; wb += kWin) {
        const int nE = min(kWin, e1 - wb);
        __syncthreads();   // previous window's tiles are done with went / pre
        // stage, validate and map the window's entries; lengths into pre[]
        for (int i = tid; i < nE; i += kGThreads) {
            const int4 en = ent[wb + i];
            const int x = en.x, lo = en.y, hi = en.z;
            bool ok = lo >= 0 && lo < hi && hi <= P && x >= 0 && x < a.c.max_pages;
            if (!ok) fault(st, CHK_BLOCK_ENTRY, wb + i);
            if (ok && (x << a.c.Plog2) + hi > L) {
                fault(st, CHK_INDEX, (x << a.c.Plog2) + hi - 1);
                ok = false;
            }
            int page = 0;
            if (ok) {
                page = __ldg(ptb + x);
                if (page < 0 || page >= a.c.num_pages) {
                    fault(st, CHK_PAGE, page);
                    ok = false;
                }
            }
            went[i] = make_int4(lo, ok ? hi - lo : 0, page, 0);
            if (ok) {
                // the tiles read this entry's rows one after another: start all
                // of them towards L2 now, so that only the first tile waits on DRAM
                const size_t off = ((((size_t)page * a.c.Hkv + g) << a.c.Plog2) + lo) * D;
                prefetch_l2(a.c.k + off, (uint32_t)(hi - lo) * D * 2);
                prefetch_l2(a.c.v + off, (uint32_t)(hi - lo) * D * 2);
            }
        }
        __syncthreads();
        if (warp == 0) {
            // exclusive prefix of the lengths (serial over 32-entry runs per lane)
            const int per = (nE + 31) / 32;
            const int i0 = min(lane * per, nE), i1 = min(i0 + per, nE);
            int run = 0;
            for (int i = i0; i < i1; ++i) run += went[i].y;
            int incl = run;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            int base = incl - run;
            for (int i = i0; i < i1; ++i) {
                pre[i] = base;
                base += went[i].y;
            }
            if (lane == 31) *s_tot = incl;
        }
        __syncthreads();
        const int nw = *s_tot;
        const int ntile = (nw + kGT - 1) / kGT;

        // gather: thread -> (row r, half of the row's chunks), K and V
        auto issue = [&](int tile, int buf) {
            const int r = tid >> 1;
            const int p = tile * kGT + r;
            const bool ok = p < nw;
            size_t src = 0;
            if (ok) {
                int lo = 0, hi = nE - 1;   // last entry with pre[e] <= p
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (pre[mid] <= p) lo = mid; else hi = mid - 1;
                }
                const int4 en = went[lo];
                const int tok = en.x + (p - pre[lo]);
                src = ((((size_t)en.z * a.c.Hkv + g) << a.c.Plog2) + tok) * D;
            }
            if ((tid & 1) == 0) rowok[buf * kGT + r] = ok ? 1 : 0;
            const uint32_t kd = sbase + buf * SM::TILE + r * D * 2;
            const uint32_t vd = sbase + 2 * SM::TILE + buf * SM::TILE + r * D * 2;
#pragma unroll
            for (int j = 0; j < CH / 2; ++j) {
                const int c = (tid & 1) * (CH / 2) + j;
                const uint32_t sw = (uint32_t)((c ^ (r & 7)) * 16);
                cp_async16(kd + sw, a.c.k + src + c * 8, ok);
                cp_async16(vd + sw, a.c.v + src + c * 8, ok);
            }
        };

        if (ntile > 0) issue(0, 0);
        cp_async_commit();
        for (int t = 0; t < ntile; ++t) {
            const int buf = t & 1;
            if (t + 1 < ntile) issue(t + 1, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
            __syncthreads();

            // ---- S = Q K^T for this warp's 16 tokens (two n-blocks of 8)
            float sc[2][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sc[0][i] = sc[1][i] = 0.f;
            const uint32_t kt = sbase + buf * SM::TILE;
            {
                const int mi = lane >> 3, ri = lane & 7;
                const int tok = warp * 16 + ri + (mi >> 1) * 8;
                const uint32_t rowa = kt + tok * D * 2;
#pragma unroll
                for (int kk = 0; kk < KK; ++kk) {
                    const int c = kk * 2 + (mi & 1);
                    uint32_t b00, b01, b10, b11;
                    ldsm_x4(rowa + ((c ^ (tok & 7)) * 16), b00, b01, b10, b11);
                    mma16816(sc[0], qa[kk], b00, b01);
                    mma16816(sc[1], qa[kk], b10, b11);
                    if (QF32) {
                        mma16816(sc[0], ql[QF32 ? kk : 0], b00, b01);
                        mma16816(sc[1], ql[QF32 ? kk : 0], b10, b11);
                    }
                }
            }
            // scale into the base-2 domain, mask rows that are not selected
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const int tk = warp * 16 + nb * 8 + 2 * tq;
                const bool ok0 = rowok[buf * kGT + tk] != 0, ok1 = rowok[buf * kGT + tk + 1] != 0;
                sc[nb][0] = ok0 ? sc[nb][0] * a.qscale : -INFINITY;
                sc[nb][1] = ok1 ? sc[nb][1] * a.qscale : -INFINITY;
                sc[nb][2] = ok0 ? sc[nb][2] * a.qscale : -INFINITY;
                sc[nb][3] = ok1 ? sc[nb][3] * a.qscale : -INFINITY;
            }
            // ---- online softmax, rows gq (elements 0, 1) and gq + 8 (2, 3)
            float x0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
            float x1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
            x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
            x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
            x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
            x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
            const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
            const float b0 = n0 == -INFINITY ? 0.f : n0, b1 = n1 == -INFINITY ? 0.f : n1;
            const float al0 = ex2(m0 - b0), al1 = ex2(m1 - b1);   // 0 while a row is still empty
            m0 = n0;
            m1 = n1;
            float p[2][4];
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                p[nb][0] = ex2(sc[nb][0] - b0);
                p[nb][1] = ex2(sc[nb][1] - b0);
                p[nb][2] = ex2(sc[nb][2] - b1);
                p[nb][3] = ex2(sc[nb][3] - b1);
            }
            l0 = l0 * al0 + (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
            l1 = l1 * al1 + (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                o[nb][0] *= al0;
                o[nb][1] *= al0;
                o[nb][2] *= al1;
                o[nb][3] *= al1;
            }
            // ---- O += P V: P (16 heads x 16 tokens) is the A operand
            const uint32_t pa[4] = {pack_bf2(p[0][0], p[0][1]), pack_bf2(p[0][2], p[0][3]),
                                    pack_bf2(p[1][0], p[1][1]), pack_bf2(p[1][2], p[1][3])};
            const uint32_t vt = sbase + 2 * SM::TILE + buf * SM::TILE;
            {
                const int mi = lane >> 3, ri = lane & 7;
                const int tok = warp * 16 + ri + (mi & 1) * 8;
                const uint32_t rowa = vt + tok * D * 2;
#pragma unroll
                for (int dn = 0; dn < D / 16; ++dn) {
                    const int c = dn * 2 + (mi >> 1);
                    uint32_t r0, r1, r2, r3;
                    ldsm_x4_t(rowa + ((c ^ (tok & 7)) * 16), r0, r1, r2, r3);
                    mma16816(o[2 * dn], pa, r0, r1);
                    mma16816(o[2 * dn + 1], pa, r2, r3);
                }
            }
            __syncthreads();   // this buffer is refilled by the issue two tiles on
        }
        cp_async_wait<0>();
    }

    // ---- merge the 4 warps' states through shared memory
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    __syncthreads();
    float *mo = reinterpret_cast<float *>(sm);                 // [warp][16][D]
    float *mm = mo + kGWarps * 16 * D;                          // [warp][16]
    float *ml = mm + kGWarps * 16;                              // [warp][16]
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int c = nb * 8 + 2 * tq;
        mo[(warp * 16 + gq) * D + c] = o[nb][0];
        mo[(warp * 16 + gq) * D + c + 1] = o[nb][1];
        mo[(warp * 16 + gq + 8) * D + c] = o[nb][2];
        mo[(warp * 16 + gq + 8) * D + c + 1] = o[nb][3];
    }
    if (tq == 0) {
        mm[warp * 16 + gq] = m0;
        mm[warp * 16 + gq + 8] = m1;
        ml[warp * 16 + gq] = l0;
        ml[warp * 16 + gq + 8] = l1;
    }
    __syncthreads();
    const int nrow = min(HPG, 16);
    for (int i = tid; i < nrow * D; i += kGThreads) {
        const int j = i / D, c = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kGWarps; ++w) M = fmaxf(M, mm[w * 16 + j]);
        float O = 0.f, Ls = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kGWarps; ++w) {
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

template <int D, bool QF32>
cudaError_t launch_gqa(const DecodeArgs &a, cudaStream_t s)
{
    constexpr int smem = GqaSmem<D>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(k_decode_gqa_blocks<D, QF32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.S, a.c.Hkv, a.c.B);
    if (cudaError_t e_ = launch_pdl(k_decode_gqa_blocks<D, QF32>, dim3(grid), dim3(kGThreads), smem, s, a)) return e_;
    return cudaGetLastError();
}

}  // namespace

bool decode_gqa_supported(const DecodeArgs &a) { return a.blocks && a.Hq / a.c.Hkv <= 16; }

cudaError_t launch_decode_gqa_split(const DecodeArgs &a, cudaStream_t s)
{
    if (a.c.D == 64) return a.q_f32 ? launch_gqa<64, true>(a, s) : launch_gqa<64, false>(a, s);
    return a.q_f32 ? launch_gqa<128, true>(a, s) : launch_gqa<128, false>(a, s);
}

}  // namespace sa
