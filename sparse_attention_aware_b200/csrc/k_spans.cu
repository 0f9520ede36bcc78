// Span masks -> page-segment block lists.
//
// Method: "语言模型能自己决定该看哪里吗？" (DA state machine: a chunk-level
// mask of allowed KV positions; kept ranges rounded OUT to the KV-block edges
// because paged kernels read whole blocks), "百万上下文，模型终于会挑重点了"
// (section "三种模式": global / focus / local), and "稀疏注意力机制创新…"
// (section "二、ZigZag架构": a fixed 1024-token streaming window, token-exact).
//
// One CTA per sequence.  Thread 0 rounds, clips, sorts and merges the spans
// (span counts are small); the CTA then writes one entry per touched page,
// {logical page, lo, hi, tokens before}, in ascending token order.  Every
// token of the union appears exactly once.
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kMaxSpans = 1024;

__global__ void __launch_bounds__(256) k_span_blocks(const SpanArgs a)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int2 rng[kMaxSpans];        // merged [start, end)
    __shared__ int ent_base[kMaxSpans + 1];
    __shared__ int tok_base[kMaxSpans + 1];
    __shared__ int s_nr;

    const int b = blockIdx.x;
    const int P = 1 << a.c.Plog2;
    const int Lcap = a.c.max_pages << a.c.Plog2;
    int L = __ldg(a.c.sl + b);
    if (L < 0 || L > Lcap) {
        if (threadIdx.x == 0) fault(a.st, CHK_SEQ_LEN, L);
        L = L < 0 ? 0 : Lcap;
    }

    if (threadIdx.x == 0) {
        int ns = a.span_counts[b];
        if (ns < 0 || ns > a.max_spans) {
            fault(a.st, CHK_SPAN, ns);
            ns = ns < 0 ? 0 : a.max_spans;
        }
        int nr = 0;
        for (int i = 0; i < ns; ++i) {
            long long s0 = a.spans[((size_t)b * a.max_spans + i) * 2 + 0];
            long long s1 = a.spans[((size_t)b * a.max_spans + i) * 2 + 1];
            if (a.span_round[(size_t)b * a.max_spans + i]) {
                // round out: [floor(s0/P)P, ceil(s1/P)P)
                s0 = (s0 >= 0 ? s0 / P : -((-s0 + P - 1) / P)) * P;
                s1 = (s1 >= 0 ? (s1 + P - 1) / P : -((-s1) / P)) * P;
            }
            if (s0 < 0) s0 = 0;
            if (s1 > L) s1 = L;
            if (s0 >= s1) continue;
            // insertion by start
            int j = nr++;
            while (j > 0 && rng[j - 1].x > (int)s0) {
                rng[j] = rng[j - 1];
                --j;
            }
            rng[j] = make_int2((int)s0, (int)s1);
        }
        // merge overlapping / touching ranges
        int m = 0;
        for (int i = 0; i < nr; ++i) {
            if (m > 0 && rng[i].x <= rng[m - 1].y) {
                rng[m - 1].y = max(rng[m - 1].y, rng[i].y);
            } else {
                rng[m++] = rng[i];
            }
        }
        int e = 0, t = 0;
        for (int i = 0; i < m; ++i) {
            ent_base[i] = e;
            tok_base[i] = t;
            e += (rng[i].y - 1) / P - rng[i].x / P + 1;
            t += rng[i].y - rng[i].x;
        }
        ent_base[m] = e;
        tok_base[m] = t;
        s_nr = m;
        if (e > a.max_blocks) record(a.st, SA_ERR_CAPACITY, CHK_CAPACITY_BLOCKS, e);
        a.ecnt[b] = min(e, a.max_blocks);
    }
    __syncthreads();
    const int m = s_nr;
    int4 *out = reinterpret_cast<int4 *>(a.ent) + (size_t)b * a.max_blocks;
    for (int i = 0; i < m; ++i) {
        const int s0 = rng[i].x, s1 = rng[i].y;
        const int p0 = s0 / P, p1 = (s1 - 1) / P;
        for (int p = p0 + threadIdx.x; p <= p1; p += blockDim.x) {
            const int e = ent_base[i] + (p - p0);
            if (e >= a.max_blocks) break;
            const int a0 = max(s0, p * P), a1 = min(s1, (p + 1) * P);
            out[e] = make_int4(p, a0 - p * P, a1 - p * P, tok_base[i] + (a0 - s0));
        }
    }
}

}  // namespace

cudaError_t launch_spans(const SpanArgs &a, cudaStream_t s)
{
    if (a.c.B == 0) return cudaSuccess;
    if (a.max_spans > kMaxSpans) return cudaErrorInvalidValue;
    if (cudaError_t e_ = launch_pdl(k_span_blocks, dim3(a.c.B), dim3(256), 0, s, a)) return e_;
    return cudaGetLastError();
}

}  // namespace sa
