// RBS two-branch block selection for causal block-sparse prefill.
//
// Method: "RBS-Attention: Radius-Bounded Sparse Prefill…" (blog summary),
// section "关键技术点": (1) a centroid base branch scoring a block by its
// average relevance and a rescue branch using the block's maximum key radius,
// which catches blocks whose mean is diluted by irrelevant tokens; (2) each
// branch is thresholded on its own and the masks are OR'd, feeding an
// unchanged block-sparse attention path.
//
// Kernels (one launch sequence per call):
//   k_block_stats  per (key block j, kv head g): c_j = mean of the block's keys,
//                  r_j = max ||k - c_j||, from one read of the block (staged in
//                  shared memory); c_j is written as a split-bf16 tile image
//                  for the tensor cores.
//   k_pool_q       per (query block i, q head h): qbar_i = mean of the block's
//                  queries (tile image, as c_j), ||qbar_i||.
//   k_pair_tc      (k_pair_tc.cu) per (128-block row tile, q head) on tcgen05:
//                  the pooled dot products qbar_i . c_j, both branch scores,
//                  thresholds, OR with the forced diagonal and first block ->
//                  mask bits and per-row counts.  In quantile mode the scores
//                  are stored instead and
//   k_qhist/k_qpick  find each head's lower quantile (exact radix select on
//                  the order-preserving key, grid-wide histograms) and
//   k_mask_scores  thresholds the stored scores.
//   k_csr_scan / k_csr_fill  turn counts and bits into CSR (ascending cols).
#include <cuda_bf16.h>

#include "sa_internal.h"

namespace sa {

size_t rbs_workspace_layout(int Hq, int Hkv, int D, int nB, bool quantile, size_t *offs)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t words = rbs_mask_words(nB);
    const size_t nP = (size_t)nB * (nB + 1) / 2;
    size_t o = 0;
    const size_t img = (size_t)rbs_img_tiles(nB) * kRbsImgBytes;   // per matrix (D = 128)
    offs[0] = o; o += up((size_t)Hkv * img);              // centroid tile images
    offs[1] = o; o += up((size_t)Hkv * rbs_img_tiles(nB) * kRbsImgRows * 4);   // radii, rows padded to whole tiles
    offs[2] = o; o += up((size_t)Hq * img);               // pooled-query tile images
    offs[3] = o; o += up((size_t)Hq * nB * 4);            // pooled query norms
    offs[4] = o; o += up((size_t)2 * Hq * 4);             // thresholds
    offs[5] = o; o += up((size_t)Hq * nB * words * 4);    // mask bits
    offs[6] = o; o += up((size_t)Hq * nB * 4 + 16 + ((size_t)Hq * nB / 1024 + 2) * 8);   // row counts + chunk sums
    offs[7] = o; if (quantile) o += up((size_t)2 * Hq * nP * 4);   // pair scores
    // radix-select scratch: per (branch, head) a 2048-bin histogram for each of
    // the 3 digit passes + state {prefix, mask, need}
    offs[8] = o; if (quantile) o += up((size_t)2 * Hq * (3 * 2048 + 4) * 4);
    return o;
}

namespace {

constexpr int BS = 64;   // block size (tokens); query and key blocks alike

// x -> (hi, lo) = (bf16(x), bf16(x - hi)) at element (row, k) of a tile image
__device__ __forceinline__ void store_split(uint8_t *img, int row, int k, float x)
{
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
    *reinterpret_cast<__nv_bfloat16 *>(img + rbs_img_offset(row, k, 0)) = hi;
    *reinterpret_cast<__nv_bfloat16 *>(img + rbs_img_offset(row, k, 1)) = lo;
}

// ---------------------------------------------------------------------------
// Block statistics (one CTA per key block and kv head; the block's rows stay
// in registers: column sums, then squared distances from the centroid) and
// query pooling (one
// CTA per query block and q head), two launches over nB rounded up to whole
// 128-row tile images, whose padding rows are zeroed.  The pooling CTA of
// (i, h) also clears row i's mask count of head h, and the first statistics
// CTA copies explicit thresholds into place.  (One launch with both kinds of
// CTA was measured 10% slower.)
// ---------------------------------------------------------------------------
struct StatsSmem {
    float csum[8][128];        // per-warp column sums
    float cen[128];
    float wmax[8];
};
struct PoolSmem {
    float part[16][128];
    float red[4];
};

__device__ void block_stats_cta(const RbsArgs &a, StatsSmem &sm, int j, int g)
{
    constexpr int D = 128;
    const int rad_rows = rbs_img_tiles(a.nB) * kRbsImgRows;
    uint8_t *img = a.cen + ((size_t)g * rbs_img_tiles(a.nB) + (j >> 7)) * kRbsImgBytes;
    if (j >= a.nB) {   // padding row of the last tile image
        if (threadIdx.x < D) {
            *reinterpret_cast<uint16_t *>(img + rbs_img_offset(j & 127, threadIdx.x, 0)) = 0;
            *reinterpret_cast<uint16_t *>(img + rbs_img_offset(j & 127, threadIdx.x, 1)) = 0;
        }
        if (threadIdx.x == 0) a.rad[(size_t)g * rad_rows + j] = 0.f;
        return;
    }
    const int n = min(BS, a.T - j * BS);
    const int P = 1 << a.c.Plog2;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c8 = tid & 15;                 // this thread's 8 columns: 8*c8 ..
    // rows (tid >> 4) + 16u, u = 0..3, held in registers (16-byte loads, all
    // in flight at once); the block starts on a page edge (P divides 64)
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int r = (tid >> 4) + 16 * u;
        v[u] = make_uint4(0, 0, 0, 0);
        if (r < n) {
            int page = __ldg(a.c.pt + ((j * BS + r) >> a.c.Plog2));
            if (page < 0 || page >= a.c.num_pages) {
                fault(a.st, CHK_PAGE, page);
            } else {
                const size_t off = ((((size_t)page * a.c.Hkv + g) << a.c.Plog2) + ((j * BS + r) & (P - 1))) * D + c8 * 8;
                v[u] = ldg_nc_v4(a.c.k + off);
            }
        }
    }
    // column sums: the thread's rows, then the other row group of the warp
    // (lane ^ 16 holds the same columns), then the eight warps via shared memory
    float cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            cs[2 * q] += bf_lo(w[q]);
            cs[2 * q + 1] += bf_hi(w[q]);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 16);
    if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.csum[warp][8 * c8 + e] = cs[e];
    }
    __syncthreads();
    if (tid < D) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += sm.csum[w][tid];
        const float c = t / (float)n;
        sm.cen[tid] = c;
        store_split(img, j & 127, tid, c);
    }
    __syncthreads();
    // max radius: squared distance of each row from the centroid, summed over
    // the 16 lanes that hold the row, max over rows; sqrt is monotone, so the
    // root of the largest square is the largest radius
    float cc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cc[e] = sm.cen[8 * c8 + e];
    float mx = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        float d = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x0 = bf_lo(w[q]) - cc[2 * q], x1 = bf_hi(w[q]) - cc[2 * q + 1];
            d = fmaf(x0, x0, d);
            d = fmaf(x1, x1, d);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if ((tid >> 4) + 16 * u < n) mx = fmaxf(mx, d);
    }
    mx = warp_max(mx);
    if (lane == 0) sm.wmax[warp] = mx;
    __syncthreads();
    if (tid == 0) {
        float m = 0.f;
        for (int w = 0; w < 8; ++w) m = fmaxf(m, sm.wmax[w]);
        a.rad[(size_t)g * rad_rows + j] = sqrtf(m);
    }
}

__device__ void pool_q_cta(const RbsArgs &a, PoolSmem &sm, int i, int h)
{
    constexpr int D = 128;
    uint8_t *img = a.qbar + ((size_t)h * rbs_img_tiles(a.nB) + (i >> 7)) * kRbsImgBytes;
    if (i >= a.nB) {   // padding row of the last tile image
        if (threadIdx.x < D) {
            *reinterpret_cast<uint16_t *>(img + rbs_img_offset(i & 127, threadIdx.x, 0)) = 0;
            *reinterpret_cast<uint16_t *>(img + rbs_img_offset(i & 127, threadIdx.x, 1)) = 0;
        }
        return;
    }
    if (threadIdx.x == 0) a.rowcnt[(size_t)h * a.nB + i] = 0;
    const int n = min(BS, a.T - i * BS);
    const int lane16 = threadIdx.x & 15, rs = threadIdx.x >> 4;   // 16 row slots
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = rs; r < n; r += 16) {
        const size_t t = (size_t)i * BS + r;
        uint4 w = ldg_nc_v4(a.q + (t * a.Hq + h) * D + lane16 * 8);
        acc[0] += bf_lo(w.x); acc[1] += bf_hi(w.x); acc[2] += bf_lo(w.y); acc[3] += bf_hi(w.y);
        acc[4] += bf_lo(w.z); acc[5] += bf_hi(w.z); acc[6] += bf_lo(w.w); acc[7] += bf_hi(w.w);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) sm.part[rs][lane16 * 8 + e] = acc[e];
    __syncthreads();
    float sq = 0.f;
    if (threadIdx.x < D) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) s += sm.part[r][threadIdx.x];
        const float qb = s / (float)n;
        store_split(img, i & 127, threadIdx.x, qb);
        sq = qb * qb;
    }
    sq = warp_sum(sq);
    if ((threadIdx.x & 31) == 0 && threadIdx.x < D) sm.red[threadIdx.x >> 5] = sq;
    __syncthreads();
    if (threadIdx.x == 0) a.qnorm[(size_t)h * a.nB + i] = sqrtf((sm.red[0] + sm.red[1]) + (sm.red[2] + sm.red[3]));
}

__global__ void __launch_bounds__(256) k_block_stats(const RbsArgs a)
{
    pdl_wait();
    pdl_trigger();
    __shared__ __align__(16) uint8_t raw[sizeof(StatsSmem)];
    if (blockIdx.x == 0 && blockIdx.y == 0 && a.tau_c) {   // explicit thresholds
        for (int h = threadIdx.x; h < a.Hq; h += blockDim.x) {
            a.tau[h] = a.tau_c[h];
            a.tau[a.Hq + h] = a.tau_r[h];
        }
    }
    block_stats_cta(a, *reinterpret_cast<StatsSmem *>(raw), blockIdx.x, blockIdx.y);
}

__global__ void __launch_bounds__(256) k_pool_q(const RbsArgs a)
{
    pdl_wait();
    pdl_trigger();
    __shared__ __align__(16) uint8_t raw[sizeof(PoolSmem)];
    pool_q_cta(a, *reinterpret_cast<PoolSmem *>(raw), blockIdx.x, blockIdx.y);
}

// ---------------------------------------------------------------------------
// block-wide exclusive scan helper (1024 threads max)
__device__ __forceinline__ long long block_excl_scan_ll(long long v, long long *wt, long long &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wt[warp] = x;
    __syncthreads();
    if (warp == 0) {
        long long w = lane < (int)(blockDim.x >> 5) ? wt[lane] : 0;
        long long z = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            long long y = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += y;
        }
        wt[lane] = z - w;
        if (lane == 31) wt[32] = z;
    }
    __syncthreads();
    const long long r = wt[warp] + x - v;
    total = wt[32];
    __syncthreads();
    return r;
}

// Lower quantile of each (branch, head)'s causal pair scores, the element at
// ascending rank floor(p*(n-1)): an exact radix select on the order-preserving
// key in three digit passes (11, 11, 10 bits).  Each pass is a grid-wide
// histogram (k_qhist: many CTAs per score array, shared-memory histograms
// flushed to global memory) followed by a one-CTA digit pick (k_qpick) that
// narrows (prefix, mask, need).  Scratch per array: 3 x 2048 bins + state.
constexpr int kQChunk = 1 << 17;   // scores per histogram CTA

__device__ __forceinline__ uint32_t *qhist_of(const RbsArgs &a, int arr, int pass)
{
    return a.qhist + (size_t)arr * (3 * 2048 + 4) + pass * 2048;
}
__device__ __forceinline__ uint32_t *qstate_of(const RbsArgs &a, int arr)
{
    return a.qhist + (size_t)arr * (3 * 2048 + 4) + 3 * 2048;
}

__global__ void __launch_bounds__(512) k_qhist(const RbsArgs a, int pass)
{
    pdl_wait();
    pdl_trigger();
    __shared__ unsigned hist[2048];
    const int arr = blockIdx.y;          // branch * Hq + h
    const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
    const size_t t0 = (size_t)blockIdx.x * kQChunk;
    if (t0 >= nP) return;
    const size_t t1 = min(t0 + (size_t)kQChunk, nP);
    const int shift = pass == 0 ? 21 : pass == 1 ? 10 : 0;
    const int nb = pass == 2 ? 1024 : 2048;
    uint32_t prefix = 0, pmask = 0;
    if (pass > 0) {
        const uint32_t *st = qstate_of(a, arr);
        prefix = st[0];
        pmask = st[1];
    }
    for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const float *x = a.pair_sc + (size_t)arr * nP;
    auto count = [&](float v) {
        const uint32_t key = f2key(v);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
    };
    // 16-byte loads over the aligned middle of [t0, t1); an array need not
    // start on a 16-byte boundary, so up to 3 scores at each end are read singly
    const size_t head = min((size_t)((16u - ((uintptr_t)(x + t0) & 15u)) & 15u) / 4, t1 - t0);
    const size_t ta = t0 + head, nv = (t1 - ta) / 4, tb = ta + 4 * nv;
    if (threadIdx.x < head) count(__ldcs(x + t0 + threadIdx.x));
    const float4 *x4 = reinterpret_cast<const float4 *>(x + ta);
    for (size_t v = threadIdx.x; v < nv; v += blockDim.x) {
        const float4 f = __ldcs(x4 + v);
        count(f.x);
        count(f.y);
        count(f.z);
        count(f.w);
    }
    if (threadIdx.x < t1 - tb) count(__ldcs(x + tb + threadIdx.x));
    __syncthreads();
    uint32_t *gh = qhist_of(a, arr, pass);
    for (int i = threadIdx.x; i < nb; i += blockDim.x)
        if (hist[i]) atomicAdd(&gh[i], hist[i]);
}

__global__ void __launch_bounds__(1024) k_qpick(const RbsArgs a, int pass)
{
    pdl_wait();
    pdl_trigger();
    __shared__ long long wt[33];
    __shared__ unsigned s_digit;
    __shared__ long long s_below;
    const int arr = blockIdx.x;
    const int branch = arr / a.Hq, h = arr % a.Hq;
    const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
    uint32_t *st = qstate_of(a, arr);
    uint32_t prefix = 0, pmask = 0;
    long long need;
    if (pass == 0) {
        const float p = branch == 0 ? a.p_c : a.p_r;
        need = (long long)floor((double)p * (double)(nP - 1)) + 1;   // 1-based ascending rank
    } else {
        prefix = st[0];
        pmask = st[1];
        need = (long long)st[2] | ((long long)st[3] << 32);
    }
    const int shift = pass == 0 ? 21 : pass == 1 ? 10 : 0;
    const int nb = pass == 2 ? 1024 : 2048;
    const uint32_t *hist = qhist_of(a, arr, pass);
    const int per = nb / blockDim.x;
    long long mine = 0;
    for (int q = 0; q < per; ++q) mine += hist[threadIdx.x * per + q];
    long long total;
    const long long before = block_excl_scan_ll(mine, wt, total);   // count in lower digits
    if (before < need && need <= before + mine) {
        long long run = before;
        for (int q = 0; q < per; ++q) {
            const int bin = threadIdx.x * per + q;
            if (run + hist[bin] >= need) {
                s_digit = (unsigned)bin;
                s_below = run;
                break;
            }
            run += hist[bin];
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        need -= s_below;
        prefix |= s_digit << shift;
        pmask |= (uint32_t)(nb - 1) << shift;
        st[0] = prefix;
        st[1] = pmask;
        st[2] = (uint32_t)(need & 0xffffffffu);
        st[3] = (uint32_t)(need >> 32);
        if (pass == 2) {
            const uint32_t u = (prefix & 0x80000000u) ? (prefix & 0x7fffffffu) : ~prefix;
            a.tau[branch * a.Hq + h] = __uint_as_float(u);
        }
    }
}

// quantile mode: threshold the stored pair scores; one warp per row (h, i),
// four 32-column words in flight per iteration
__global__ void __launch_bounds__(256) k_mask_scores(const RbsArgs a)
{
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.Hq * a.nB) return;
    const int h = row / a.nB, i = row % a.nB;
    const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
    const float *sc = a.pair_sc + (size_t)h * nP + (size_t)i * (i + 1) / 2;
    const float *sr = a.pair_sc + ((size_t)a.Hq + h) * nP + (size_t)i * (i + 1) / 2;
    const float tc = a.tau[h], tr = a.tau[a.Hq + h];
    const int words = rbs_mask_words(a.nB);
    const int nw = i / 32 + 1;
    int cnt = 0;
    for (int w0 = 0; w0 < nw; w0 += 8) {   // 16 loads per lane in flight
        float vc[8], vr[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = (w0 + u) * 32 + lane;
            vc[u] = j <= i ? __ldcs(sc + j) : 0.f;
            vr[u] = j <= i ? __ldcs(sr + j) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = (w0 + u) * 32 + lane;
            const bool keep = j <= i && (vc[u] > tc || vr[u] > tr || (a.force_diag && j == i) ||
                                         (a.force_first && j == 0));
            const uint32_t w = __ballot_sync(0xffffffffu, keep);
            if (lane == 0 && w0 + u < nw) a.bits[(size_t)row * words + w0 + u] = w;
            cnt += __popc(w);
        }
    }
    if (lane == 0) a.rowcnt[row] = cnt;
}

// CSR row pointers: exclusive prefix sum of the row counts in three short
// launches (per-chunk sums, one scan of the chunk sums, per-chunk write-out).
constexpr int kScanChunk = 1024;   // rows per CTA (one per thread)

__global__ void __launch_bounds__(kScanChunk) k_csr_sum(const RbsArgs a, long long *chunk_sum)
{
    pdl_wait();
    pdl_trigger();
    __shared__ long long wt[33];
    const int R = a.Hq * a.nB;
    const int r = blockIdx.x * kScanChunk + threadIdx.x;
    long long total;
    block_excl_scan_ll(r < R ? a.rowcnt[r] : 0, wt, total);
    if (threadIdx.x == 0) chunk_sum[blockIdx.x] = total;
}

__global__ void __launch_bounds__(1024) k_csr_chunks(const RbsArgs a, long long *chunk_sum, int nchunks)
{
    pdl_wait();
    pdl_trigger();
    __shared__ long long wt[33];
    long long run = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 1024) {
        const int c = c0 + threadIdx.x;
        const long long v = c < nchunks ? chunk_sum[c] : 0;
        long long total;
        const long long ex = block_excl_scan_ll(v, wt, total);
        if (c < nchunks) chunk_sum[c] = run + ex;
        run += total;
    }
    if (threadIdx.x == 0) {
        const int R = a.Hq * a.nB;
        a.row_ptr[R] = (int32_t)min(run, (long long)INT32_MAX);
        if (run > a.nnz_cap) record(a.st, SA_ERR_CAPACITY, CHK_CAPACITY_CSR, (int)min(run, (long long)INT32_MAX));
    }
}

__global__ void __launch_bounds__(kScanChunk) k_csr_scan(const RbsArgs a, const long long *chunk_off)
{
    pdl_wait();
    pdl_trigger();
    __shared__ long long wt[33];
    const int R = a.Hq * a.nB;
    const int r = blockIdx.x * kScanChunk + threadIdx.x;
    long long total;
    const long long ex = block_excl_scan_ll(r < R ? a.rowcnt[r] : 0, wt, total);
    if (r < R) a.row_ptr[r] = (int32_t)min(chunk_off[blockIdx.x] + ex, (long long)INT32_MAX);
}

__global__ void __launch_bounds__(256) k_csr_fill(const RbsArgs a)
{
    pdl_wait();
    pdl_trigger();
    if (blockIdx.x == 0 && a.tau_out)
        for (int x = threadIdx.x; x < 2 * a.Hq; x += blockDim.x) a.tau_out[x] = a.tau[x];
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.Hq * a.nB) return;
    const int i = row % a.nB;
    const int words = rbs_mask_words(a.nB);
    const int nw = i / 32 + 1;
    long long base = a.row_ptr[row];
    for (int w0 = 0; w0 < nw; w0 += 32) {
        const int w = w0 + lane;
        const uint32_t bits = w < nw ? a.bits[(size_t)row * words + w] : 0u;
        const int c = __popc(bits);
        int pre = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, pre, o);
            if (lane >= o) pre += y;
        }
        const int tot = __shfl_sync(0xffffffffu, pre, 31);
        long long pos = base + pre - c;
        uint32_t b = bits;
        while (b) {
            const int bit = __ffs(b) - 1;
            b &= b - 1;
            if (pos < a.nnz_cap) a.cols[pos] = w * 32 + bit;
            ++pos;
        }
        base += tot;
    }
}

}  // namespace

cudaError_t launch_rbs(const RbsArgs &a, cudaStream_t s)
{
    if (a.c.D != 128) return cudaErrorNotSupported;
    const bool quant = a.tau_c == nullptr;
    cudaError_t e;
    // per-kv-head block statistics on sequence 0's keys
    const int img_rows = rbs_img_tiles(a.nB) * kRbsImgRows;   // padding rows are zeroed
    if (cudaError_t e_ = launch_pdl(k_block_stats, dim3(img_rows, a.c.Hkv), dim3(256), 0, s, a)) return e_;
    if (cudaError_t e_ = launch_pdl(k_pool_q, dim3(img_rows, a.Hq), dim3(256), 0, s, a)) return e_;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (quant) {
        if ((e = launch_pair_tc(a, true, s)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(a.qhist, 0, (size_t)2 * a.Hq * (3 * 2048 + 4) * 4, s)) != cudaSuccess) return e;
        const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
        const dim3 hgrid((unsigned)((nP + kQChunk - 1) / kQChunk), 2 * a.Hq);
        for (int pass = 0; pass < 3; ++pass) {
            if (cudaError_t e_ = launch_pdl(k_qhist, dim3(hgrid), dim3(512), 0, s, a, pass)) return e_;
            if (cudaError_t e_ = launch_pdl(k_qpick, dim3(2 * a.Hq), dim3(1024), 0, s, a, pass)) return e_;
        }
        if (cudaError_t e_ = launch_pdl(k_mask_scores, dim3((a.Hq * a.nB + 7) / 8), dim3(256), 0, s, a)) return e_;
    } else {
        if ((e = launch_pair_tc(a, false, s)) != cudaSuccess) return e;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        const int R = a.Hq * a.nB;
        const int nch = (R + kScanChunk - 1) / kScanChunk;
        long long *chunk = reinterpret_cast<long long *>(a.rowcnt + R + 1 + ((R + 1) & 1));   // 8-byte aligned
        if (cudaError_t e_ = launch_pdl(k_csr_sum, dim3(nch), dim3(kScanChunk), 0, s, a, chunk)) return e_;
        if (cudaError_t e_ = launch_pdl(k_csr_chunks, dim3(1), dim3(1024), 0, s, a, chunk, nch)) return e_;
        if (cudaError_t e_ = launch_pdl(k_csr_scan, dim3(nch), dim3(kScanChunk), 0, s, a, chunk)) return e_;
    }
    if (cudaError_t e_ = launch_pdl(k_csr_fill, dim3((a.Hq * a.nB + 7) / 8), dim3(256), 0, s, a)) return e_;
    return cudaGetLastError();
}

}  // namespace sa
