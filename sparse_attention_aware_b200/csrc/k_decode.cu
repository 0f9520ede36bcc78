// Split-KV sparse decode attention and its combine pass.
//
// Method: attention of one query token over a selected token set -- the
// anchor's top-k positions, reused unchanged by the following layers
// ("Kascade稀疏注意力…", section "核心机制：Anchor + Reuse"), or the page
// segments of a block-aligned span mask ("语言模型能自己决定该看哪里吗？",
// DA state machine section).  The selected set is cut into S contiguous
// parts; each CTA reduces one part to (max, sum, unnormalised output) and a
// combine kernel merges the parts ("稀疏注意力机制创新…", section
// "四、从外卖到AI": SplitKV-and-Combine).
//
// k_decode_split: one CTA = (split s, query head h, sequence b), 256 threads.
// Lanes are grouped by G = D/8: a group owns one token row at a time and each
// lane holds 8 of its D elements (one 16-byte load of K and one of V).
// Every group walks U consecutive list positions per step, so each lane has
// 2U independent 16-byte loads in flight (for token lists the positions of a
// window are first resolved to row offsets in shared memory, so those loads
// wait on nothing else); the row is reduced over the group
// with xor shuffles and folded into a per-group online softmax (base-2
// exponentials on log2(e)-prescaled scores).  The groups' partial states are
// merged through shared memory at the end.  The kernel is bound by the HBM
// gather of the selected rows (512 B of K+V per token at D=128).
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kStage = 1024;   // token-list positions resolved per window

template <int D>
struct DecodeCfg {
    static constexpr int G = D / 8;      // lanes per token row
    static constexpr int GPW = 32 / G;   // groups per warp
    static constexpr int NG = 8 * GPW;   // groups per CTA
};

// Position -> token for the block-list selection: binary search of the entry
// whose prefix "tokens before" covers pos.
__device__ __forceinline__ int locate_entry(const int4 *ent, int ne, int pos)
{
    int lo = 0, hi = ne - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(&ent[mid].w) <= pos) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int D, bool QF32, bool BLOCKS, int U>
__global__ void __launch_bounds__(256) k_decode_split(const DecodeArgs a)
{
    pdl_wait();
    pdl_trigger();
    using C = DecodeCfg<D>;
    constexpr int G = C::G, GPW = C::GPW, NG = C::NG;
    __shared__ float s_m[NG], s_l[NG];
    __shared__ float s_acc[NG * D];
    __shared__ long long s_off[BLOCKS ? 1 : kStage];   // token lists: element offsets of a window's rows

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gl = lane & (G - 1);
    const int sub = lane / G;
    const int grp = warp * GPW + sub;
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int group = a.Hq / a.c.Hkv;
    const int g = h / group;
    const int row = b * a.Hq + h;
    DevStatus *st = a.st;

    const int Lcap = a.c.max_pages << a.c.Plog2;
    int L = __ldg(a.c.sl + b);
    if (L < 0 || L > Lcap) {
        fault(st, CHK_SEQ_LEN, L);
        L = L < 0 ? 0 : Lcap;
    }

    // list length
    int n = 0, ne = 0;
    const int4 *ent = nullptr;
    if (!BLOCKS) {
        n = __ldg(a.cnt + row);
        if (n < 0 || n > a.kcap) {
            fault(st, CHK_COUNT, n);
            n = n < 0 ? 0 : a.kcap;
        }
    } else {
        ne = __ldg(a.ecnt + b);
        if (ne < 0 || ne > a.max_blocks) {
            fault(st, CHK_BLOCK_ENTRY, ne);
            ne = ne < 0 ? 0 : a.max_blocks;
        }
        ent = reinterpret_cast<const int4 *>(a.ent) + (size_t)b * a.max_blocks;
        if (ne > 0) {
            int4 last = ent[ne - 1];
            n = last.w + (last.z - last.y);
            if (n < 0 || last.w < 0 || last.z < last.y) {
                fault(st, CHK_BLOCK_ENTRY, n);
                n = 0;
            }
        }
    }
    const int chunk = (n + a.S - 1) / a.S;
    const int lo = min(s * chunk, n), hi = min(lo + chunk, n);

    // query slice, prescaled into the base-2 domain
    float qv[8];
    if (QF32) {
        const float4 *qp = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.q) +
                                                            (size_t)row * D + gl * 8);
        float4 x0 = __ldg(qp), x1 = __ldg(qp + 1);
        qv[0] = x0.x; qv[1] = x0.y; qv[2] = x0.z; qv[3] = x0.w;
        qv[4] = x1.x; qv[5] = x1.y; qv[6] = x1.z; qv[7] = x1.w;
    } else {
        uint4 w = ldg_nc_v4(reinterpret_cast<const uint16_t *>(a.q) + (size_t)row * D + gl * 8);
        qv[0] = bf_lo(w.x); qv[1] = bf_hi(w.x); qv[2] = bf_lo(w.y); qv[3] = bf_hi(w.y);
        qv[4] = bf_lo(w.z); qv[5] = bf_hi(w.z); qv[6] = bf_lo(w.w); qv[7] = bf_hi(w.w);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] *= a.qscale;

    float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    const uint16_t *kbase = a.c.k, *vbase = a.c.v;
    const int32_t *ptb = a.c.pt + (size_t)b * a.c.max_pages;
    const int Pm = (1 << a.c.Plog2) - 1;

    // the U rows of one step -> online softmax state of the group
    auto consume = [&](const uint4 (&kr)[U], const uint4 (&vr)[U], const bool (&ok)[U]) {
        float sc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float p = qv[0] * bf_lo(kr[u].x);
            p = fmaf(qv[1], bf_hi(kr[u].x), p);
            p = fmaf(qv[2], bf_lo(kr[u].y), p);
            p = fmaf(qv[3], bf_hi(kr[u].y), p);
            p = fmaf(qv[4], bf_lo(kr[u].z), p);
            p = fmaf(qv[5], bf_hi(kr[u].z), p);
            p = fmaf(qv[6], bf_lo(kr[u].w), p);
            p = fmaf(qv[7], bf_hi(kr[u].w), p);
#pragma unroll
            for (int o = G / 2; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            sc[u] = ok[u] ? p : -INFINITY;
        }
        float mx = sc[0];
#pragma unroll
        for (int u = 1; u < U; ++u) mx = fmaxf(mx, sc[u]);
        const float mn = fmaxf(m, mx);
        if (mn != -INFINITY) {
            const float alpha = ex2(m - mn);
            l *= alpha;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float pw = ex2(sc[u] - mn);
                l += pw;
                acc[0] = fmaf(pw, bf_lo(vr[u].x), acc[0]);
                acc[1] = fmaf(pw, bf_hi(vr[u].x), acc[1]);
                acc[2] = fmaf(pw, bf_lo(vr[u].y), acc[2]);
                acc[3] = fmaf(pw, bf_hi(vr[u].y), acc[3]);
                acc[4] = fmaf(pw, bf_lo(vr[u].z), acc[4]);
                acc[5] = fmaf(pw, bf_hi(vr[u].z), acc[5]);
                acc[6] = fmaf(pw, bf_lo(vr[u].w), acc[6]);
                acc[7] = fmaf(pw, bf_hi(vr[u].w), acc[7]);
            }
            m = mn;
        }
    };

    if (!BLOCKS) {
        // Token lists: the part's positions are resolved (index -> page ->
        // element offset of the row, -1 if invalid) into shared memory a
        // window at a time, so the main loop's loads depend on nothing but
        // a shared-memory read.
        for (int w0 = lo; w0 < hi; w0 += kStage) {
            const int wn = min(kStage, hi - w0);
            __syncthreads();   // the previous window has been consumed
            for (int i = threadIdx.x; i < wn; i += blockDim.x) {
                const int t = __ldg(a.idx + (size_t)row * a.kcap + w0 + i);
                long long off = -1;
                if (t < 0 || t >= L) {
                    fault(st, CHK_INDEX, t);
                } else {
                    const int page = __ldg(ptb + (t >> a.c.Plog2));
                    if (page < 0 || page >= a.c.num_pages)
                        fault(st, CHK_PAGE, page);
                    else
                        off = (long long)(((((size_t)page * a.c.Hkv + g) << a.c.Plog2) + (t & Pm)) * D);
                }
                s_off[i] = off;
            }
            __syncthreads();
            // warp-uniform loop: every lane of a warp runs the same iterations
            for (int base0 = warp * GPW * U; base0 < wn; base0 += NG * U) {
                const int base = base0 + sub * U;
                uint4 kr[U], vr[U];
                bool ok[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int pos = base + u;
                    const long long off = pos < wn ? s_off[pos] : -1;
                    ok[u] = off >= 0;
                    if (ok[u]) {
                        kr[u] = ldg_nc_v4(kbase + off + gl * 8);
                        vr[u] = ldg_nc_v4(vbase + off + gl * 8);
                    } else {
                        kr[u] = make_uint4(0, 0, 0, 0);
                        vr[u] = make_uint4(0, 0, 0, 0);
                    }
                }
                consume(kr, vr, ok);
            }
        }
    } else {
        // block lists: positions map to tokens through the entries
        for (int base0 = lo + warp * GPW * U; base0 < hi; base0 += NG * U) {
            const int base = base0 + sub * U;
            uint4 kr[U], vr[U];
            bool ok[U];
            int e_idx = 0, e_off = 0;
            int4 e_cur = make_int4(0, 0, 0, 0);
            if (base < hi) {
                e_idx = locate_entry(ent, ne, base);
                e_cur = ent[e_idx];
                e_off = base - e_cur.w;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int pos = base + u;
                ok[u] = pos < hi;
                int t = 0;
                if (ok[u]) {
                    while (e_off >= e_cur.z - e_cur.y && e_idx + 1 < ne) {
                        e_off -= e_cur.z - e_cur.y;
                        e_cur = ent[++e_idx];
                    }
                    t = (e_cur.x << a.c.Plog2) + e_cur.y + e_off;
                    ++e_off;
                    if (t < 0 || t >= L) {
                        fault(st, CHK_INDEX, t);
                        ok[u] = false;
                    }
                }
                int page = 0;
                if (ok[u]) {
                    page = __ldg(ptb + (t >> a.c.Plog2));
                    if (page < 0 || page >= a.c.num_pages) {
                        fault(st, CHK_PAGE, page);
                        ok[u] = false;
                    }
                }
                const size_t off = ((((size_t)page * a.c.Hkv + g) << a.c.Plog2) + (t & Pm)) * D + gl * 8;
                if (ok[u]) {
                    kr[u] = ldg_nc_v4(kbase + off);
                    vr[u] = ldg_nc_v4(vbase + off);
                } else {
                    kr[u] = make_uint4(0, 0, 0, 0);
                    vr[u] = make_uint4(0, 0, 0, 0);
                }
            }
            consume(kr, vr, ok);
        }
    }

    // merge the groups' states
#pragma unroll
    for (int e = 0; e < 8; ++e) s_acc[grp * D + gl * 8 + e] = acc[e];
    if (gl == 0) {
        s_m[grp] = m;
        s_l[grp] = l;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        float M = -INFINITY;
#pragma unroll 4
        for (int i = 0; i < NG; ++i) M = fmaxf(M, s_m[i]);
        float o = 0.f, Ls = 0.f;
        if (M != -INFINITY) {
            for (int i = 0; i < NG; ++i) {
                const float mi = s_m[i];
                if (mi == -INFINITY) continue;
                const float w = ex2(mi - M);
                o = fmaf(w, s_acc[i * D + c], o);
                Ls = fmaf(w, s_l[i], Ls);
            }
        }
        a.part_o[((size_t)row * a.S + s) * D + c] = o;
        if (c == 0) {
            a.part_ml[((size_t)row * a.S + s) * 2 + 0] = M;
            a.part_ml[((size_t)row * a.S + s) * 2 + 1] = Ls;
        }
    }
}

// Combine: m = max m_s over non-empty parts; l = sum l_s 2^(m_s-m);
// out = sum 2^(m_s-m) O_s / l; lse = (m + log2 l) ln 2.
template <int D>
__global__ void __launch_bounds__(D) k_decode_combine(const float *__restrict__ part_o,
                                                       const float *__restrict__ part_ml, int S,
                                                       uint16_t *__restrict__ out,
                                                       float *__restrict__ lse)
{
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x, c = threadIdx.x;
    const float *ml = part_ml + (size_t)row * S * 2;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s)
        if (ml[2 * s + 1] > 0.f) M = fmaxf(M, ml[2 * s]);
    float o = 0.f, Ls = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < S; ++s) {
            const float ls = ml[2 * s + 1];
            if (!(ls > 0.f)) continue;
            const float w = ex2(ml[2 * s] - M);
            Ls = fmaf(w, ls, Ls);
            o = fmaf(w, part_o[((size_t)row * S + s) * D + c], o);
        }
        o = o / Ls;
    }
    out[(size_t)row * D + c] = f2bf(o);
    if (lse && c == 0) lse[row] = (M != -INFINITY) ? (M + lg2(Ls)) * kLn2 : -INFINITY;
}

template <int D, bool QF32, bool BLOCKS>
cudaError_t launch_split(const DecodeArgs &a, cudaStream_t s)
{
    dim3 grid(a.S, a.Hq, a.c.B);
    if (cudaError_t e_ = launch_pdl(k_decode_split<D, QF32, BLOCKS, 4>, dim3(grid), dim3(256), 0, s, a)) return e_;
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const DecodeArgs &a, cudaStream_t s)
{
    cudaError_t e;
    if (decode_gqa_supported(a))
        e = launch_decode_gqa_split(a, s);
    else if (a.blocks)
        e = a.q_f32 ? launch_split<D, true, true>(a, s) : launch_split<D, false, true>(a, s);
    else
        e = a.q_f32 ? launch_split<D, true, false>(a, s) : launch_split<D, false, false>(a, s);
    if (e != cudaSuccess) return e;
    if (cudaError_t e_ = launch_pdl(k_decode_combine<D>, dim3(a.c.B * a.Hq), dim3(D), 0, s, a.part_o, a.part_ml, a.S, a.out, a.lse)) return e_;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s)
{
    if (a.c.B * a.Hq == 0) return cudaSuccess;
    return a.c.D == 64 ? launch_d<64>(a, s) : launch_d<128>(a, s);
}

}  // namespace sa
