// Causal block-sparse prefill attention on tcgen05 tensor cores.
//
// Method: the block-sparse attention path that the RBS selection feeds
// ("RBS-Attention: Radius-Bounded Sparse Prefill…", section "关键技术点",
// item 2): for query block i of head h, attend only to the key blocks of CSR
// row (h, i), causal inside the diagonal block, exact softmax over them.
//
// B200 design (one CTA = 128 query rows = query blocks 2I and 2I+1 of one
// head, over the union of their two CSR rows; 192 threads, 2 CTAs per SM):
//   warp 0      TMA producer: Q tile once (3-D map over [T][Hq][128]), then per
//               selected key block the K and V page tiles (2-D maps over the
//               paged cache; page table resolved per block), 128-byte swizzle,
//               into an NS-stage ring guarded by mbarriers.
//   warp 1      MMA issuer (one thread) and TMEM owner: S = Q K^T (M=128, N=64,
//               K=128) into one of two TMEM S buffers, then O += P V (M=128,
//               N=128, K=64) into the TMEM O accumulator, in the order
//               S_0, S_1, PV_0, S_2, PV_1, ... so the next scores are computed
//               while the softmax of the current block runs.
//   warps 2-5   softmax: one query row per thread (TMEM lane), row-half
//               selection mask and causal mask, online softmax in the base-2
//               domain with lazy rescaling (O and l are rescaled only when
//               the running max grows by more than 2^8), P written to shared
//               memory as bf16 in the swizzled K-major layout the next MMA
//               reads; final O / l -> bf16 and LSE.
// The two rows of a super-block share each K/V tile; a block listed by only
// one row is masked (p = 0) for the other row's queries.
// Every wait is bounded (globaltimer deadline, shared abort flag): on expiry
// the kernel records SA_ERR_TIMEOUT, drains its own outstanding copies and
// MMAs with bounded waits, frees its TMEM and returns.
#include <cudaTypedefs.h>

#include "sa_internal.h"
#include "tc_ptx.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int kThreads = 192;
constexpr int kTmemCols = 256;                 // S0 [0,64) S1 [64,128) O [128,256)
constexpr uint32_t kQBytes = 128 * 128 * 2;     // 32 KB
constexpr uint32_t kKVBytes = 64 * 128 * 2;     // 16 KB per K (or V) block
constexpr uint32_t kPBytes = 128 * 64 * 2;      // 16 KB
constexpr uint64_t kWaitNs = 400ull * 1000 * 1000;   // 0.4 s per wait

constexpr uint32_t IDESC_S = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, 0, 1);

template <int NS>
struct Smem {
    static constexpr uint32_t Q = 0;
    static constexpr uint32_t K = Q + kQBytes;
    static constexpr uint32_t V = K + NS * kKVBytes;
    static constexpr uint32_t P = V + NS * kKVBytes;
    static constexpr uint32_t BAR = P + kPBytes;
    // barriers: q_full, kfull[NS], vfull[NS], kv_empty[NS], s_full[2], s_empty[2], p_full, pv_done
    static constexpr int NBAR = 1 + 3 * NS + 6;
    static constexpr uint32_t MISC = BAR + NBAR * 8;
    static constexpr uint32_t TOTAL = MISC + 16;
};

// Ascending merge of the two CSR rows of a super-block; yields (key block,
// row-half mask).  Entries out of [0, i] or not strictly ascending are
// recorded as a fault and skipped (identically by every role).
struct Merge {
    const int32_t *c0, *c1;
    int n0, n1, i0, i1, lim0, lim1, last0, last1;
    DevStatus *st;

    __device__ void init(const PrefillArgs &a, int r0, int lim_0, bool has1)
    {
        st = a.st;
        // rows are read only inside [0, nnz_cap): a truncated (overflowed) CSR
        // loses its tail entries, it never reads past the cols buffer
        const int b0 = __ldg(a.row_ptr + r0), e0 = __ldg(a.row_ptr + r0 + 1);
        c0 = a.cols + (b0 > 0 ? b0 : 0);
        n0 = e0 - b0;
        if (b0 < 0 || n0 < 0 || n0 > lim_0 + 1) {
            fault(st, CHK_CSR, r0);
            n0 = 0;
        } else if ((long long)b0 + n0 > a.nnz_cap) {
            fault(st, CHK_CSR, r0);
            n0 = (long long)b0 >= a.nnz_cap ? 0 : (int)(a.nnz_cap - b0);
        }
        n1 = 0;
        c1 = c0;
        if (has1) {
            const int b1 = __ldg(a.row_ptr + r0 + 1), e1 = __ldg(a.row_ptr + r0 + 2);
            c1 = a.cols + (b1 > 0 ? b1 : 0);
            n1 = e1 - b1;
            if (b1 < 0 || n1 < 0 || n1 > lim_0 + 2) {
                fault(st, CHK_CSR, r0 + 1);
                n1 = 0;
            } else if ((long long)b1 + n1 > a.nnz_cap) {
                fault(st, CHK_CSR, r0 + 1);
                n1 = (long long)b1 >= a.nnz_cap ? 0 : (int)(a.nnz_cap - b1);
            }
        }
        i0 = i1 = 0;
        lim0 = lim_0;
        lim1 = lim_0 + 1;
        last0 = last1 = -1;
    }

    __device__ bool next(int &j, int &m)
    {
        int v0 = INT_MAX, v1 = INT_MAX;
        while (i0 < n0) {
            v0 = __ldg(c0 + i0);
            if (v0 > last0 && v0 <= lim0) break;
            fault(st, CHK_CSR, v0);
            v0 = INT_MAX;
            ++i0;
        }
        while (i1 < n1) {
            v1 = __ldg(c1 + i1);
            if (v1 > last1 && v1 <= lim1) break;
            fault(st, CHK_CSR, v1);
            v1 = INT_MAX;
            ++i1;
        }
        if (i0 >= n0) v0 = INT_MAX;
        if (i1 >= n1) v1 = INT_MAX;
        if (v0 == INT_MAX && v1 == INT_MAX) return false;
        j = min(v0, v1);
        m = (v0 == j ? 1 : 0) | (v1 == j ? 2 : 0);
        if (v0 == j) { last0 = v0; ++i0; }
        if (v1 == j) { last1 = v1; ++i1; }
        return true;
    }
};

template <int NS>
__global__ void __launch_bounds__(kThreads, 2)
    k_prefill_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const PrefillArgs a)
{
    using L = Smem<NS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {   // uniform for the whole CTA
        if (threadIdx.x == 0) record(a.st, SA_ERR_CUDA, CHK_WAIT, (int)(sbase & 1023u));
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR);
    uint64_t *q_full = bars;
    uint64_t *kfull = bars + 1;
    uint64_t *vfull = kfull + NS;
    uint64_t *kv_empty = vfull + NS;
    uint64_t *s_full = kv_empty + NS;
    uint64_t *s_empty = s_full + 2;
    uint64_t *p_full = s_empty + 2;
    uint64_t *pv_done = p_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nQB = (a.T + 63) >> 6, nSB = (nQB + 1) >> 1;
    const int I = nSB - 1 - (int)(blockIdx.x / a.Hq);   // heavy (late) rows first
    const int h = (int)(blockIdx.x % a.Hq);
    const int g = h / (a.Hq / a.c.Hkv);
    const int r0 = h * nQB + 2 * I;
    const bool has1 = 2 * I + 1 < nQB;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(vfull + s, 1);
            mbar_init(kv_empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full + b, 1);
            mbar_init(s_empty + b, 128);
        }
        mbar_init(p_full, 128);
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

    Merge mg;
    mg.init(a, r0, 2 * I, has1);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_arrive_expect_tx(q_full, kQBytes);
            tma_load_3d(smem + L::Q, &tmQ, q_full, 0, h, 128 * I);
            tma_load_3d(smem + L::Q + kQBytes / 2, &tmQ, q_full, 64, h, 128 * I);
            int n = 0, j, m;
            bool ok = true;
            while (ok && mg.next(j, m)) {
                const int s = n % NS;
                if (n >= NS) ok = mbar_wait(kv_empty + s, ((n / NS) - 1) & 1, deadline, abort_flag);
                if (!ok) break;
                int page = __ldg(a.c.pt + j);
                if (page < 0 || page >= a.c.num_pages) {
                    fault(a.st, CHK_PAGE, page);
                    page = 0;
                }
                const int row = (page * a.c.Hkv + g) * 64;
                uint8_t *kd = smem + L::K + s * kKVBytes;
                uint8_t *vd = smem + L::V + s * kKVBytes;
                mbar_arrive_expect_tx(kfull + s, kKVBytes);
                tma_load_2d(kd, &tmK, kfull + s, 0, row);
                tma_load_2d(kd + kKVBytes / 2, &tmK, kfull + s, 64, row);
                mbar_arrive_expect_tx(vfull + s, kKVBytes);
                tma_load_2d(vd, &tmV, vfull + s, 0, row);
                tma_load_2d(vd + kKVBytes / 2, &tmV, vfull + s, 64, row);
                ++n;
            }
            if (!ok) {
                *abort_flag = 1;
                record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, 0);
            }
            // never leave with copies in flight: the last NS loads are consumed
            // by the MMA thread in the normal case; on abort wait for them here
            if (*abort_flag) {
                const uint64_t dl2 = globaltimer() + kWaitNs;
                volatile int never = 0;
                for (int p = max(0, n - NS); p < n; ++p) {
                    mbar_wait(kfull + p % NS, (p / NS) & 1, dl2, &never);
                    mbar_wait(vfull + p % NS, (p / NS) & 1, dl2, &never);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            const uint32_t qa = sbase + L::Q;
            int n = 0, j, m;
            bool ok = mbar_wait(q_full, 0, deadline, abort_flag);
            auto issue_pv = [&](int p) -> bool {
                const int sp = p % NS;
                if (!mbar_wait(vfull + sp, (p / NS) & 1, deadline, abort_flag)) return false;
                if (!mbar_wait(p_full, p & 1, deadline, abort_flag)) return false;
                fence_after_sync();
                const uint32_t pa = sbase + L::P;
                const uint32_t va = sbase + L::V + sp * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = smem_desc_sw128(pa + kk * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(va + kk * 2048, 8192, 1024);
                    mma_f16(tmem + 128, ad, bd, IDESC_PV, (p > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(pv_done);
                mma_commit(kv_empty + sp);
                return true;
            };
            while (ok && mg.next(j, m)) {
                const int s = n % NS;
                ok = mbar_wait(kfull + s, (n / NS) & 1, deadline, abort_flag);
                if (ok && n >= 2) ok = mbar_wait(s_empty + (n & 1), ((n - 2) >> 1) & 1, deadline, abort_flag);
                if (!ok) break;
                fence_after_sync();
                const uint32_t ka = sbase + L::K + s * kKVBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = smem_desc_sw128(qa + (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(ka + (kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32, 16, 1024);
                    mma_f16(tmem + (n & 1) * 64, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full + (n & 1));
                if (n >= 1) ok = issue_pv(n - 1);
                ++n;
            }
            if (ok && n >= 1) ok = issue_pv(n - 1);
            if (!ok) {
                *abort_flag = 1;
                record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, 1);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const int qpos = 128 * I + r;
        const int half = r >> 6;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        const float C = a.scale * kLog2e;
        float m_used = -INFINITY, l = 0.f;
        int n = 0, j, msk;
        bool ok = true;
        uint8_t *prow = smem + L::P + r * 128;
        while (ok && mg.next(j, msk)) {
            ok = __all_sync(0xffffffffu, mbar_wait(s_full + (n & 1), (n >> 1) & 1, deadline, abort_flag));
            if (!ok) break;
            fence_after_sync();
            uint32_t sr[64];
            tmem_ld32(lane_base + (n & 1) * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(lane_base + (n & 1) * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
            fence_before_sync();
            mbar_arrive(s_empty + (n & 1));

            const bool sel = (msk >> half) & 1;
            const int kb = 64 * j;
            const int lim = qpos - kb;   // key offsets c <= lim are causal-valid
            float v[64];
            float rowmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const bool valid = sel && (c <= lim);
                const float x = valid ? __uint_as_float(sr[c]) * C : -INFINITY;
                v[c] = x;
                rowmax = fmaxf(rowmax, x);
            }
            const float m_new = fmaxf(m_used, rowmax);
            bool rescale = false;
            float alpha = 1.f;
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
            const float base = (m_used == -INFINITY) ? 0.f : m_used;
            uint32_t pk[32];
            float psum = 0.f;
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
                const float p0 = ex2(v[c] - base);
                const float p1 = ex2(v[c + 1] - base);
                psum += p0 + p1;
                pk[c >> 1] = pack_bf16x2(p0, p1);
            }
            l += psum;
            if (n > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (n - 1) & 1, deadline, abort_flag));
                if (!ok) break;
                fence_after_sync();
            }
            if (__any_sync(0xffffffffu, rescale)) {
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
            // P row: 8 chunks of 16 B, 128-byte swizzle (chunk c at c ^ (r & 7))
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 w = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                *reinterpret_cast<uint4 *>(prow + ((c ^ (r & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();
            fence_before_sync();
            mbar_arrive(p_full);
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
        // epilogue: O / l -> bf16, LSE
        const bool store = qpos < a.T && ok;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint16_t *orow = a.out + ((size_t)qpos * a.Hq + h) * 128;
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
        if (store && a.lse) a.lse[(size_t)qpos * a.Hq + h] = l > 0.f ? (m_used + lg2(l)) * kLn2 : -INFINITY;
        fence_before_sync();
    }

    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        if (*abort_flag) {
            // bounded drain of outstanding MMAs before TMEM is freed: a fresh
            // commit on the (otherwise idle) pv_done barrier arrives once every
            // earlier tcgen05 op of the issuing thread has completed
            if (lane == 0) {
                volatile int never = 0;
                const uint64_t dl = globaltimer() + kWaitNs;
                mma_commit(pv_done);
                // either phase may be the drain's; wait for both parities in turn
                mbar_wait(pv_done, 0, dl, &never);
                mbar_wait(pv_done, 1, dl, &never);
            }
            __syncwarp();
        }
        tmem_dealloc(tmem, kTmemCols);
    }
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

constexpr int kStages = 2;

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t s)
{
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv;
    {
        cuuint64_t dims[3] = {128, (cuuint64_t)a.Hq, (cuuint64_t)a.T};
        cuuint64_t strides[2] = {256, (cuuint64_t)a.Hq * 256};
        cuuint32_t box[3] = {64, 1, 128};
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
    using L = Smem<kStages>;
    const size_t smem = L::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(k_prefill_tc<kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int nQB = (a.T + 63) / 64, nSB = (nQB + 1) / 2;
    const long long grid = (long long)nSB * a.Hq;
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    k_prefill_tc<kStages><<<(unsigned)grid, kThreads, smem, s>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

}  // namespace sa
