// Causal block-sparse prefill attention on tcgen05 tensor cores.
//
// Method: the block-sparse attention path that the RBS selection feeds
// ("RBS-Attention: Radius-Bounded Sparse Prefill…", section "关键技术点",
// item 2): for query block i of head h, attend only to the key blocks of CSR
// row (h, i), causal inside the diagonal block, exact softmax over them.
//
// B200 design.  tcgen05 MMAs run at full rate with M = 128 rows, while a
// query block has 64.  One CTA therefore serves a work item of two 64-row
// halves that share their K/V tiles: two rows (query head, query block) of
// one GQA group, from a window of nearby query blocks (the pairing is chosen
// by k_prefill_schedule_window, greedily by the key blocks the two rows do not
// share), or, for odd group sizes, two adjacent query blocks of one head.  The CTA walks the union of the two rows;
// a key block listed by one half only is masked (p = 0) for the other half.
//   warp 0      K producer: the Q halves (3-D map over [T][Hq][128]), then
//               per key block of the merged list the K page tile (2-D map over
//               the paged cache; page table resolved per block), 128-byte
//               swizzle, 3-stage ring released as soon as S = QK^T of that
//               block has completed.  It merges the two CSR rows and posts
//               (block, half mask) per stage, with an end sentinel.
//   warp 6      V producer: the V page tiles of the same merged list into their
//               own 2-stage ring, released when PV of that block completes.
//   warp 1      MMA issuer (one thread) and TMEM owner: S = Q K^T (M=128, N=64,
//               K=128) into one of two TMEM S buffers; O += P V (M=128, N=128,
//               K=64) with P read from TMEM, where the softmax wrote it over
//               the first 32 columns of S's buffer; order S_0, S_1, PV_0, S_2,
//               PV_1, S_3, ...  It forwards each block's (index, half mask) to
//               the softmax through a shared ring published by a release-arrive
//               on the S-ready barrier.
//   warps 2-5   softmax: one query row per thread (TMEM lane); half-selection
//               and causal masks (only the diagonal block needs per-element
//               masking); base-2 online softmax with the scale folded into the
//               exponent's FMA and lazy rescaling (O and l rescaled only when
//               the running max grows by more than 2^8); P written to TMEM as
//               bf16 pairs; it waits for PV only before a rescale of O and at
//               the end; final O / l -> bf16 and LSE.
// Every wait is bounded (globaltimer deadline, shared abort flag): on expiry
// the kernel records SA_ERR_TIMEOUT, drains its own outstanding copies and
// MMAs with bounded waits, frees its TMEM and returns.
#include <cudaTypedefs.h>

#include "sa_internal.h"
#include "tc_ptx.cuh"

namespace sa {

namespace {
constexpr int kMaxPairGroup = 16;   // GQA groups up to 16 heads are head-paired
}

int prefill_items(int Hq, int Hkv, int nQB)
{
    const int G = Hq / Hkv;
    if (G % 2 == 0 && G <= kMaxPairGroup) return (Hq / 2) * nQB;
    return Hq * ((nQB + 1) / 2);
}

namespace {

using namespace tc;

constexpr int kThreads = 224;
constexpr int kTmemCols = 256;                 // S0/P0 [0,64) S1/P1 [64,128) O [128,256)
constexpr uint32_t kQBytes = 128 * 128 * 2;     // 32 KB
constexpr uint32_t kKVBytes = 64 * 128 * 2;     // 16 KB per K (or V) block
constexpr uint64_t kWaitNs = 400ull * 1000 * 1000;   // 0.4 s

constexpr uint32_t IDESC_S = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, 0, 1);

template <int NSK, int NSV>
struct Smem {
    static constexpr uint32_t Q = 0;
    static constexpr uint32_t K = Q + kQBytes;
    static constexpr uint32_t V = K + NSK * kKVBytes;
    static constexpr uint32_t BAR = V + NSV * kKVBytes;
    // q_full, kfull[NSK], k_empty[NSK], vfull[NSV], v_empty[NSV], s_full[2], p_full[2], pv_done
    static constexpr int NBAR = 1 + 2 * NSK + 2 * NSV + 5;
    static constexpr uint32_t SLOT = BAR + NBAR * 8;       // int2 slot[NSK]: K producer -> MMA
    static constexpr uint32_t SINFO = SLOT + NSK * 8;      // int2 sinfo[4]: MMA -> softmax
    static constexpr uint32_t MISC = SINFO + 4 * 8;
    static constexpr uint32_t TOTAL = MISC + 16;
};

// Valid extent of CSR row `row` (entries <= lim): its first column pointer
// and length, clamped to the cols capacity; malformed rows are recorded and
// read as empty.
__device__ __forceinline__ int csr_row(const PrefillArgs &a, int row, int lim, const int32_t *&ptr)
{
    const int b = __ldg(a.row_ptr + row), e = __ldg(a.row_ptr + row + 1);
    int n = e - b;
    ptr = a.cols + (b > 0 ? b : 0);
    if (b < 0 || n < 0 || n > lim + 1) {
        fault(a.st, CHK_CSR, row);
        return 0;
    }
    if ((long long)b + n > a.nnz_cap) {
        fault(a.st, CHK_CSR, row);
        n = (long long)b >= a.nnz_cap ? 0 : (int)(a.nnz_cap - b);
    }
    return n;
}

// Ascending merge of the two rows of a work item -> (key block, half mask).
// Entries out of [0, lim] or not strictly ascending are recorded and skipped.
struct Merge {
    const int32_t *c[2];
    int n[2], i[2], lim[2], last[2];
    DevStatus *st;

    __device__ int head(int h)
    {
        while (i[h] < n[h]) {
            const int v = __ldg(c[h] + i[h]);
            if (v > last[h] && v <= lim[h]) return v;
            fault(st, CHK_CSR, v);
            ++i[h];
        }
        return INT_MAX;
    }

    __device__ bool next(int &j, int &m)
    {
        const int v0 = head(0), v1 = head(1);
        if (v0 == INT_MAX && v1 == INT_MAX) return false;
        j = min(v0, v1);
        m = (v0 == j ? 1 : 0) | (v1 == j ? 2 : 0);
        if (v0 == j) { last[0] = v0; ++i[0]; }
        if (v1 == j) { last[1] = v1; ++i[1]; }
        return true;
    }
};

template <int NSK, int NSV>
__global__ void __launch_bounds__(kThreads, 2)
    k_prefill_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    using L = Smem<NSK, NSV>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {   // uniform for the whole CTA
        if (threadIdx.x == 0) record(a.st, SA_ERR_CUDA, CHK_WAIT, (int)(sbase & 1023u));
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR);
    uint64_t *q_full = bars;
    uint64_t *kfull = bars + 1;
    uint64_t *k_empty = kfull + NSK;
    uint64_t *vfull = k_empty + NSK;
    uint64_t *v_empty = vfull + NSV;
    uint64_t *s_full = v_empty + NSV;
    uint64_t *p_full = s_full + 2;     // per S buffer: the softmax may run one block ahead
    uint64_t *pv_done = p_full + 2;
    volatile int *slots = reinterpret_cast<volatile int *>(smem + L::SLOT);   // (j, mask) per K stage
    volatile int *sinfo = reinterpret_cast<volatile int *>(smem + L::SINFO); // (j, mask) per S, ring of 4
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nQB = (a.T + 63) >> 6;
    const int4 item = a.items[blockIdx.x];
    const bool has_b = item.z >= 0;
    const int hq[2] = {item.x, has_b ? item.z : item.x};
    const int iq[2] = {item.y, has_b ? item.w : item.y};
    const int g = hq[0] / (a.Hq / a.c.Hkv);

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NSK; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(k_empty + s, 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(vfull + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full + b, 2);
            mbar_init(p_full + b, 128);
        }
        mbar_init(pv_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = globaltimer() + kWaitNs * 4;

    auto init_merge = [&](Merge &mg) {
        mg.st = a.st;
        mg.n[0] = csr_row(a, hq[0] * nQB + iq[0], iq[0], mg.c[0]);
        mg.n[1] = has_b ? csr_row(a, hq[1] * nQB + iq[1], iq[1], mg.c[1]) : 0;
        if (!has_b) mg.c[1] = mg.c[0];
        mg.i[0] = mg.i[1] = 0;
        mg.lim[0] = iq[0];
        mg.lim[1] = iq[1];
        mg.last[0] = mg.last[1] = -1;
    };
    auto page_row = [&](int j) {
        int page = __ldg(a.c.pt + j);
        if (page < 0 || page >= a.c.num_pages) {
            fault(a.st, CHK_PAGE, page);
            page = 0;
        }
        return (page * a.c.Hkv + g) * 64;
    };

    if (warp == 0 || warp == 6) {
        // ------------------------------------------------------ K / V producers
        if (lane == 0) {
            const bool is_k = warp == 0;
            const int NS = is_k ? NSK : NSV;
            uint64_t *full = is_k ? kfull : vfull;
            uint64_t *empty = is_k ? k_empty : v_empty;
            const CUtensorMap *map = is_k ? &tmK : &tmV;
            uint8_t *ring = smem + (is_k ? L::K : L::V);
            prefetch_tmap(map);
            if (is_k) {
                prefetch_tmap(&tmQ);
                mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(smem + L::Q + c * (kQBytes / 2) + hf * (kQBytes / 4), &tmQ, q_full, 64 * c,
                                    hq[hf], 64 * iq[hf]);
            }
            Merge mg;
            init_merge(mg);
            int n = 0, j, m;
            bool ok = true;
            for (;;) {
                const int s = n % NS;
                if (n >= NS) ok = mbar_wait(empty + s, ((n / NS) - 1) & 1, deadline, abort_flag);
                if (!ok) break;
                if (!mg.next(j, m)) {
                    if (is_k) {
                        slots[2 * s] = -1;             // end of the list
                        slots[2 * s + 1] = 0;
                        mbar_arrive(kfull + s);
                    }
                    break;
                }
                const int row = page_row(j);
                if (is_k) {
                    slots[2 * s] = j;
                    slots[2 * s + 1] = m;
                }
                uint8_t *dst = ring + s * kKVBytes;
                mbar_arrive_expect_tx(full + s, kKVBytes);
                tma_load_2d(dst, map, full + s, 0, row);
                tma_load_2d(dst + kKVBytes / 2, map, full + s, 64, row);
                ++n;
            }
            if (!ok) {
                *abort_flag = 1;
                record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, is_k ? 0 : 3);
                // never leave with copies in flight
                const uint64_t dl2 = globaltimer() + kWaitNs;
                volatile int never = 0;
                for (int p = max(0, n - NS); p < n; ++p) mbar_wait(full + p % NS, (p / NS) & 1, dl2, &never);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        // order: S_0, S_1, then PV_n, S_{n+2}, PV_{n+1}, S_{n+3}, ...  P_n lives
        // in TMEM over S_n's columns, so S_{n+2} (same buffer) follows PV_n.
        if (lane == 0) {
            const uint32_t qa = sbase + L::Q;
            int ns = 0, total = -1;
            auto issue_s = [&]() -> bool {
                const int s = ns % NSK;
                if (!mbar_wait(kfull + s, (ns / NSK) & 1, deadline, abort_flag)) return false;
                const int j = slots[2 * s], m = slots[2 * s + 1];
                sinfo[2 * (ns & 3)] = j;
                sinfo[2 * (ns & 3) + 1] = m;
                if (j < 0) {
                    total = ns;
                    mbar_arrive(s_full + (ns & 1));
                    mbar_arrive(s_full + (ns & 1));
                    return true;
                }
                fence_after_sync();
                const uint32_t ka = sbase + L::K + s * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = smem_desc_sw128(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(ka + (kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32, 16, 1024);
                    mma_f16(tmem + (ns & 1) * 64, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full + (ns & 1));
                mma_commit(k_empty + s);
                mbar_arrive(s_full + (ns & 1));   // publishes sinfo (release)
                ++ns;
                return true;
            };
            bool ok = mbar_wait(q_full, 0, deadline, abort_flag);
            if (ok) ok = issue_s();
            if (ok && total < 0) ok = issue_s();
            for (int n = 0; ok; ++n) {
                if (total >= 0 && n >= total) break;
                const int sp = n % NSV;
                ok = mbar_wait(vfull + sp, (n / NSV) & 1, deadline, abort_flag) &&
                     mbar_wait(p_full + (n & 1), (n >> 1) & 1, deadline, abort_flag);
                if (!ok) break;
                fence_after_sync();
                const uint32_t va = sbase + L::V + sp * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bd = smem_desc_sw128(va + kk * 2048, 8192, 1024);
                    mma_f16_ts(tmem + 128, tmem + (n & 1) * 64 + kk * 8, bd, IDESC_PV, (n > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(pv_done);
                mma_commit(v_empty + sp);
                if (total < 0) ok = issue_s();
            }
            if (!ok) {
                *abort_flag = 1;
                record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, 1);
            }
        }
    } else if (warp >= 2 && warp <= 5) {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const int hf = r >> 6;                       // warp-uniform half
        const int rr = r & 63;
        const int qpos = 64 * iq[hf] + rr;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        const float C = a.scale * kLog2e;            // > 0 (checked on the host)
        float m_used = -INFINITY, l = 0.f;
        int n = 0;
        bool ok = true;
        for (;;) {
            ok = __all_sync(0xffffffffu, mbar_wait(s_full + (n & 1), (n >> 1) & 1, deadline, abort_flag));
            if (!ok) break;
            const int2 sl = make_int2(sinfo[2 * (n & 3)], sinfo[2 * (n & 3) + 1]);
            if (sl.x < 0) break;
            fence_after_sync();
            const bool sel = (sl.y >> hf) & 1;       // warp-uniform
            uint32_t pk[32];
            float alpha = 1.f;
            bool rescale = false;
            if (sel) {
                uint32_t sr[64];
                tmem_ld32(lane_base + (n & 1) * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld32(lane_base + (n & 1) * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_wait_ld();
                float v[64];
                if (sl.x == iq[hf]) {                // diagonal block: causal inside
#pragma unroll
                    for (int c = 0; c < 64; ++c) v[c] = c <= rr ? __uint_as_float(sr[c]) : -INFINITY;
                } else {
#pragma unroll
                    for (int c = 0; c < 64; ++c) v[c] = __uint_as_float(sr[c]);
                }
                // row max with 8 independent chains
                float m8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) m8[k] = v[k];
#pragma unroll
                for (int c = 8; c < 64; ++c) m8[c & 7] = fmaxf(m8[c & 7], v[c]);
                const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                const float m_new = fmaxf(m_used, mx * C);
                if (m_new > -INFINITY) {
                    if (m_used == -INFINITY) {
                        m_used = m_new;
                    } else if (m_new > m_used + 8.f) {
                        alpha = ex2(m_used - m_new);
                        l *= alpha;
                        m_used = m_new;
                        rescale = true;
                    }
                }
                const float nb = (m_used == -INFINITY) ? 0.f : -m_used;
                const float2 C2 = make_float2(C, C), nb2 = make_float2(nb, nb);
                float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                make_float2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float2 x = ffma2(make_float2(v[c], v[c + 1]), C2, nb2);
                    const float2 p = make_float2(ex2(x.x), ex2(x.y));
                    ps[(c >> 1) & 3] = fadd2(ps[(c >> 1) & 3], p);
                    pk[c >> 1] = pack_bf16x2(p.x, p.y);
                }
                const float2 s01 = fadd2(ps[0], ps[1]), s23 = fadd2(ps[2], ps[3]);
                const float2 s4 = fadd2(s01, s23);
                l += s4.x + s4.y;
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = 0u;
            }
            if (__any_sync(0xffffffffu, rescale)) {
                // O must be stable: PV_{n-1} complete
                if (n > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (n - 1) & 1, deadline, abort_flag));
                    if (!ok) break;
                    fence_after_sync();
                }
#pragma unroll 1
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + 128 + 32 * c4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(lane_base + 128 + 32 * c4, o);
                }
                tmem_wait_st();
            }
            // P_n (bf16 pairs) over the first 32 columns of S_n's buffer
            tmem_st32(lane_base + (n & 1) * 64, pk);
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(p_full + (n & 1));
            ++n;
        }
        if (ok && n > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (n - 1) & 1, deadline, abort_flag));
            fence_after_sync();
        }
        if (!ok) {
            *abort_flag = 1;
            record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, 2);
        }
        // epilogue: O / l -> bf16, LSE (the second half of a one-row item is
        // never stored)
        const bool store = qpos < a.T && ok && (hf == 0 || has_b);
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint16_t *orow = a.out + ((size_t)qpos * a.Hq + hq[hf]) * 128;
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t o[32];
            if (n > 0 && ok) {
                tmem_ld32(lane_base + 128 + 32 * c4, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = 0u;
            }
            if (store) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv, __uint_as_float(o[e + 1]) * inv);
                    w.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                    w.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                    w.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
                    *reinterpret_cast<uint4 *>(orow + 32 * c4 + e) = w;
                }
            }
        }
        if (store && a.lse) a.lse[(size_t)qpos * a.Hq + hq[hf]] = l > 0.f ? (m_used + lg2(l)) * kLn2 : -INFINITY;
        fence_before_sync();
    }

    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        if (*abort_flag) {
            // bounded drain of outstanding MMAs before TMEM is freed: a fresh
            // commit on pv_done arrives once every earlier tcgen05 op of the
            // issuing thread has completed
            if (lane == 0) {
                volatile int never = 0;
                const uint64_t dl = globaltimer() + kWaitNs;
                mma_commit(pv_done);
                mbar_wait(pv_done, 0, dl, &never);
                mbar_wait(pv_done, 1, dl, &never);
            }
            __syncwarp();
        }
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Work items.  Even GQA group sizes (<= 16): the rows (query head, query
// block) of one kv head are paired within windows of Wq = 64 / G consecutive
// query blocks, so a window holds G * Wq <= 64 rows of the group.  A pair's
// waste is |A xor B|, the key blocks listed by one row only, which the CTA
// executes for both halves; rows are paired greedily, smallest waste first,
// ties to the lowest pair index (as rounds of mutually-best pairs), then
// improved by 2-opt exchanges.  Wastes come from per-row bitmaps in shared
// memory (popcounts of xor), over chunks of kSchedBits key blocks.  One CTA
// per (kv head, window); items are ordered kv-head-major, latest windows
// first.
// ---------------------------------------------------------------------------
constexpr int kSchedRows = 64;
constexpr int kSchedWords = 64;                 // bitmap words per row per chunk
constexpr int kSchedBits = 32 * kSchedWords;    // key blocks per chunk
constexpr int kSchedPairs = kSchedRows * (kSchedRows - 1) / 2;
constexpr int kSchedSwaps = (kSchedRows / 2) * (kSchedRows / 2 - 1) / 2;   // pairs of pairs

__device__ __forceinline__ int pair_index(int ka, int kb, int nc)
{
    return ka * nc - ka * (ka + 1) / 2 + (kb - ka - 1);
}

__global__ void __launch_bounds__(256) k_prefill_schedule_window(const PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    __shared__ uint32_t bits[kSchedRows][kSchedWords + 1];   // +1: conflict-free column reads
    __shared__ int cost[kSchedPairs];
    __shared__ int red_c[2][8], red_p[2][8];   // double-buffered by iteration
    __shared__ int pr_a[kSchedRows / 2], pr_b[kSchedRows / 2];
    __shared__ int s_best[kSchedRows], s_taken;
    __shared__ unsigned long long s_used;
    __shared__ uint8_t sw_x[kSchedSwaps], sw_y[kSchedSwaps];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nQB = (a.T + 63) >> 6;
    const int G = a.Hq / a.c.Hkv;
    const int Wq = kSchedRows / G;
    const int nW = (nQB + Wq - 1) / Wq;
    const int g = blockIdx.x / nW, I = blockIdx.x % nW;
    if (g >= a.c.Hkv) return;
    const int i0 = I * Wq, i1 = min(i0 + Wq, nQB);
    const int nc = G * (i1 - i0);                // even: G is even
    const int np = nc * (nc - 1) / 2;
    // row k of the window: head g*G + k % G, query block i0 + k / G
    for (int p = tid; p < np; p += 256) cost[p] = 0;
    for (int kb0 = 0; kb0 < i1; kb0 += kSchedBits) {
        __syncthreads();
        for (int w = tid; w < nc * kSchedWords; w += 256) bits[w / kSchedWords][w % kSchedWords] = 0u;
        __syncthreads();
        // the warp's rows k = warp + 8 j: lane j resolves row j's CSR extent,
        // so the eight row-pointer loads are in flight together
        int rb = 0, rn = 0;
        if (lane < 8 && warp + 8 * lane < nc) {
            const int k = warp + 8 * lane, i = i0 + k / G;
            const int32_t *c;
            rn = csr_row(a, (g * G + k % G) * nQB + i, i, c);
            rb = (int)(c - a.cols);
        }
        for (int j = 0; j < 8 && warp + 8 * j < nc; ++j) {
            const int k = warp + 8 * j, i = i0 + k / G;
            const int n = __shfl_sync(0xffffffffu, rn, j);
            const int32_t *c = a.cols + __shfl_sync(0xffffffffu, rb, j);
            for (int e0 = 0; e0 < n; e0 += 128) {
                int v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + 32 * u + lane;
                    v[u] = e < n ? __ldg(c + e) : 0;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int rel = v[u] - kb0;   // out-of-range entries are the kernel's to record
                    if (e0 + 32 * u + lane < n && rel >= 0 && rel < kSchedBits && rel + kb0 <= i)
                        atomicOr(&bits[k][rel >> 5], 1u << (rel & 31));
                }
            }
        }
        __syncthreads();
        const int words = min(kSchedWords, (i1 - kb0 + 31) >> 5);
        for (int ka = warp; ka < nc; ka += 8) {
            for (int kb = ka + 1 + lane; kb < nc; kb += 32) {
                int x = 0;
                for (int w = 0; w < words; ++w) x += __popc(bits[ka][w] ^ bits[kb][w]);
                cost[pair_index(ka, kb, nc)] += x;
            }
        }
    }
    // Greedy pairing (repeatedly take the free pair of smallest (waste, row,
    // row) key), computed as rounds of locally dominant pairs: every free row
    // finds its best free partner, and two rows that pick each other are
    // paired.  Under a strict order on the pairs this takes exactly the pairs
    // of the sequential greedy, and every round takes at least one (the
    // smallest free pair).  Keys: waste clamped to 20 bits, then the two
    // 6-bit row ids.
    __syncthreads();
    if (tid == 0) {
        s_used = 0ull;
        s_taken = 0;
    }
    __syncthreads();
    const int base = g * nQB * (G / 2) + (nQB - i1) * (G / 2);
    for (int round = 0; round < kSchedRows; ++round) {
        const unsigned long long u = s_used;
        if (s_taken >= nc / 2) break;   // uniform: read after a barrier
        // each warp's rows ka = warp + 8 j, all eight reduced together so that
        // their shuffle chains overlap; lanes scan the partners kb = lane, lane + 32
        uint32_t bk[kSchedRows / 8];
#pragma unroll
        for (int j = 0; j < kSchedRows / 8; ++j) {
            const int ka = warp + 8 * j;
            bk[j] = 0xFFFFFFFFu;
            if (ka < nc && !(u >> ka & 1ull)) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int kb = lane + 32 * hh;
                    if (kb < nc && kb != ka && !(u >> kb & 1ull)) {
                        const int lo = min(ka, kb), hi = max(ka, kb);
                        const uint32_t key =
                            ((uint32_t)min(cost[pair_index(lo, hi, nc)], (1 << 20) - 1) << 12) | (lo << 6) | hi;
                        bk[j] = min(bk[j], key);
                    }
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int j = 0; j < kSchedRows / 8; ++j) bk[j] = min(bk[j], __shfl_xor_sync(0xffffffffu, bk[j], o));
        uint32_t mine = bk[0];
#pragma unroll
        for (int j = 1; j < kSchedRows / 8; ++j)
            if (lane == j) mine = bk[j];
        if (lane < kSchedRows / 8 && warp + 8 * lane < nc) {
            const int ka = warp + 8 * lane, lo = (mine >> 6) & 63, hi = mine & 63;
            s_best[ka] = mine == 0xFFFFFFFFu ? -1 : (lo == ka ? hi : lo);
        }
        __syncthreads();
        if (warp == 0) {
            // the mutually-best pairs (x < y) in increasing x, two rows per lane
            bool f[2];
            int yy[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int x = lane + 32 * hh;
                const int y = x < nc ? s_best[x] : -1;
                f[hh] = x < nc && y > x && !(u >> x & 1ull) && s_best[y] == x;
                yy[hh] = y;
            }
            const unsigned b0 = __ballot_sync(0xffffffffu, f[0]), b1 = __ballot_sync(0xffffffffu, f[1]);
            const unsigned lt = (1u << lane) - 1u;
            const int t = s_taken;
            unsigned long long mine = 0ull;
            if (f[0]) {
                const int p = t + __popc(b0 & lt);
                pr_a[p] = lane;
                pr_b[p] = yy[0];
                mine |= (1ull << lane) | (1ull << yy[0]);
            }
            if (f[1]) {
                const int p = t + __popc(b0) + __popc(b1 & lt);
                pr_a[p] = lane + 32;
                pr_b[p] = yy[1];
                mine |= (1ull << (lane + 32)) | (1ull << yy[1]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mine |= __shfl_xor_sync(0xffffffffu, mine, o);
            if (lane == 0) {
                s_used = u | mine;
                s_taken = t + __popc(b0) + __popc(b1);
            }
        }
        __syncthreads();
    }
    if (tid == 0 && s_taken < nc / 2) {
        // not reached (every round takes the smallest free pair); kept so that
        // every row is in an item whatever happens above
        int t = s_taken, prev = -1;
        for (int x = 0; x < nc; ++x) {
            if (s_used >> x & 1ull) continue;
            if (prev < 0) {
                prev = x;
            } else {
                pr_a[t] = prev;
                pr_b[t] = x;
                ++t;
                prev = -1;
            }
        }
        s_taken = t;
    }
    __syncthreads();
    // 2-opt: repeatedly apply the exchange of partners between two pairs that
    // lowers the total waste most (ties to the lowest pair of pairs), until
    // none does
    const int npr = nc / 2, nsw = npr * (npr - 1) / 2;
    auto cst = [&](int x, int y) { return cost[x < y ? pair_index(x, y, nc) : pair_index(y, x, nc)]; };
    // exchange q <-> pairs (x, y), x < y, in the order (0,1), (0,2), ..., (1,2), ...
    for (int q = tid; q < nsw; q += 256) {
        int x = 0, rem = q;
        while (rem >= npr - 1 - x) {
            rem -= npr - 1 - x;
            ++x;
        }
        sw_x[q] = (uint8_t)x;
        sw_y[q] = (uint8_t)(x + 1 + rem);
    }
    __syncthreads();
    for (int it = 0; it < 4 * kSchedRows; ++it) {
        int bg = 0, bq = INT_MAX;   // best gain (> 0), its exchange index and kind (bit 0)
        for (int q = tid; q < nsw; q += 256) {
            const int x = sw_x[q], y = sw_y[q];
            const int ax = pr_a[x], bx = pr_b[x], ay = pr_a[y], by = pr_b[y];
            const int cur = cst(ax, bx) + cst(ay, by);
            const int o1 = cst(ax, ay) + cst(bx, by), o2 = cst(ax, by) + cst(bx, ay);
            const int gain = cur - min(o1, o2);
            const int code = 2 * q + (o1 <= o2 ? 0 : 1);
            if (gain > bg || (gain == bg && gain > 0 && code < bq)) {
                bg = gain;
                bq = code;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const int og = __shfl_xor_sync(0xffffffffu, bg, o), oq = __shfl_xor_sync(0xffffffffu, bq, o);
            if (og > bg || (og == bg && oq < bq)) {
                bg = og;
                bq = oq;
            }
        }
        const int rb = it & 1;           // this iteration's buffer: the next one writes the other
        if (lane == 0) {
            red_c[rb][warp] = bg;
            red_p[rb][warp] = bq;
        }
        __syncthreads();
        bg = red_c[rb][0];
        bq = red_p[rb][0];
        for (int w = 1; w < 8; ++w)
            if (red_c[rb][w] > bg || (red_c[rb][w] == bg && red_p[rb][w] < bq)) {
                bg = red_c[rb][w];
                bq = red_p[rb][w];
            }
        if (bg <= 0) break;              // uniform: every thread reduced the same values
        if (tid == 0) {
            const int x = sw_x[bq >> 1], y = sw_y[bq >> 1];
            const int bx = pr_b[x];
            if ((bq & 1) == 0) {         // (ax, ay), (bx, by)
                pr_b[x] = pr_a[y];
                pr_a[y] = bx;
            } else {                     // (ax, by), (bx, ay)
                pr_b[x] = pr_b[y];
                pr_b[y] = bx;
            }
        }
        __syncthreads();
    }
    for (int t = tid; t < npr; t += 256) {
        const int ka = pr_a[t], kb = pr_b[t];
        a.items[base + t] = make_int4(g * G + ka % G, i0 + ka / G, g * G + kb % G, i0 + kb / G);
    }
}

// Odd group sizes: adjacent query blocks (2I, 2I+1) of one head; head-major,
// latest blocks first.
__global__ void k_prefill_schedule_adjacent(const PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const int nQB = (a.T + 63) >> 6, nSB = (nQB + 1) >> 1;
    const int x = blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= a.Hq * nSB) return;
    const int h = x / nSB, I = nSB - 1 - x % nSB;   // head-major (kv heads' K/V stay in L2)
    a.items[x] = make_int4(h, 2 * I, 2 * I + 1 < nQB ? h : -1, 2 * I + 1);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

constexpr int kKStages = 3, kVStages = 2;

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t s)
{
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv;
    {
        cuuint64_t dims[3] = {128, (cuuint64_t)a.Hq, (cuuint64_t)a.T};
        cuuint64_t strides[2] = {256, (cuuint64_t)a.Hq * 256};
        cuuint32_t box[3] = {64, 1, 64};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void *)a.q, dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const cuuint64_t rows = (cuuint64_t)a.c.num_pages * a.c.Hkv * 64;
    for (int w = 0; w < 2; ++w) {
        cuuint64_t dims[2] = {128, rows};
        cuuint64_t strides[1] = {256};
        cuuint32_t box[2] = {64, 64};
        cuuint32_t es[2] = {1, 1};
        if (enc(w == 0 ? &mk : &mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void *)(w == 0 ? a.c.k : a.c.v), dims,
                strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int nQB = (a.T + 63) / 64;
    const int G = a.Hq / a.c.Hkv;
    if (a.n_items <= 0) return cudaSuccess;
    if (G % 2 == 0 && G <= kMaxPairGroup) {
        const int nW = (nQB + kSchedRows / G - 1) / (kSchedRows / G);
        if (cudaError_t e_ = launch_pdl(k_prefill_schedule_window, dim3(a.c.Hkv * nW), dim3(256), 0, s, a))
            return e_;
    } else {
        if (cudaError_t e_ = launch_pdl(k_prefill_schedule_adjacent, dim3((a.n_items + 255) / 256), dim3(256), 0, s, a))
            return e_;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    using L = Smem<kKStages, kVStages>;
    const size_t smem = L::TOTAL;
    e = cudaFuncSetAttribute(k_prefill_tc<kKStages, kVStages>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (cudaError_t e_ = launch_pdl(k_prefill_tc<kKStages, kVStages>, dim3((unsigned)a.n_items), dim3(kThreads), smem, s, mq, mk, mv, a)) return e_;
    return cudaGetLastError();
}

}  // namespace sa
