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
//                  shared memory).
//   k_pool_q       per (query block i, q head h): qbar_i = mean of the block's
//                  queries, ||qbar_i||.
//   k_pair_tile    per (64x64 tile of causal block pairs, q head): the pooled
//                  dot products qbar_i . c_j (fp32 SIMT tile product), both
//                  branch scores, thresholds, OR with the forced diagonal and
//                  first block -> mask bits and per-row counts.  In quantile
//                  mode the scores are stored instead and
//   k_quantile     finds each head's lower quantile (exact radix select on the
//                  order-preserving key) and
//   k_mask_scores  thresholds the stored scores.
//   k_csr_scan / k_csr_fill  turn counts and bits into CSR (ascending cols).
#include "sa_internal.h"

namespace sa {

size_t rbs_workspace_layout(int Hq, int Hkv, int D, int nB, bool quantile, size_t *offs)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t nTB = (nB + 63) / 64;
    const size_t words = 2 * nTB;
    const size_t nP = (size_t)nB * (nB + 1) / 2;
    size_t o = 0;
    offs[0] = o; o += up((size_t)Hkv * nB * D * 4);       // centroids
    offs[1] = o; o += up((size_t)Hkv * nB * 4);           // radii
    offs[2] = o; o += up((size_t)Hq * nB * D * 4);        // pooled queries
    offs[3] = o; o += up((size_t)Hq * nB * 4);            // pooled query norms
    offs[4] = o; o += up((size_t)2 * Hq * 4);             // thresholds
    offs[5] = o; o += up((size_t)Hq * nB * words * 4);    // mask bits
    offs[6] = o; o += up((size_t)Hq * nB * 4 + 4);        // row counts
    offs[7] = o; if (quantile) o += up((size_t)2 * Hq * nP * 4);   // pair scores
    offs[8] = o; if (quantile) o += up((size_t)2 * Hq * 4);        // unused scratch
    return o;
}

namespace {

constexpr int BS = 64;   // block size (tokens); query and key blocks alike

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_block_stats(const RbsArgs a)
{
    constexpr int D = 128;
    __shared__ __align__(16) uint16_t tile[BS * D];
    __shared__ float cen[D];
    __shared__ float wmax[8];
    const int j = blockIdx.x, g = blockIdx.y;
    const int n = min(BS, a.T - j * BS);
    const int P = 1 << a.c.Plog2;
    // stage the block's rows (16-byte chunks; 16 per row)
    for (int ch = threadIdx.x; ch < n * (D / 8); ch += blockDim.x) {
        const int r = ch >> 4, c8 = ch & 15;
        const int t = j * BS + r;
        int page = __ldg(a.c.pt + (t >> a.c.Plog2));
        uint4 v = make_uint4(0, 0, 0, 0);
        if (page < 0 || page >= a.c.num_pages) {
            fault(a.st, CHK_PAGE, page);
        } else {
            const size_t off = ((((size_t)page * a.c.Hkv + g) << a.c.Plog2) + (t & (P - 1))) * D + c8 * 8;
            v = ldg_nc_v4(a.c.k + off);
        }
        *reinterpret_cast<uint4 *>(&tile[r * D + c8 * 8]) = v;
    }
    __syncthreads();
    if (threadIdx.x < D) {
        float s = 0.f;
        for (int r = 0; r < n; ++r) s += __uint_as_float((uint32_t)tile[r * D + threadIdx.x] << 16);
        const float c = s / (float)n;
        cen[threadIdx.x] = c;
        a.cen[((size_t)g * a.nB + j) * D + threadIdx.x] = c;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float mx = 0.f;
    for (int r = warp; r < n; r += 8) {
        float e = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int col = lane * 4 + q;
            const float dlt = __uint_as_float((uint32_t)tile[r * D + col] << 16) - cen[col];
            e = fmaf(dlt, dlt, e);
        }
        e = warp_sum(e);
        mx = fmaxf(mx, sqrtf(e));
    }
    if (lane == 0) wmax[warp] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int w = 0; w < 8; ++w) m = fmaxf(m, wmax[w]);
        a.rad[(size_t)g * a.nB + j] = m;
    }
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pool_q(const RbsArgs a)
{
    constexpr int D = 128;
    __shared__ float part[16][D];
    __shared__ float red[4];
    const int i = blockIdx.x, h = blockIdx.y;
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
    for (int e = 0; e < 8; ++e) part[rs][lane16 * 8 + e] = acc[e];
    __syncthreads();
    float sq = 0.f;
    if (threadIdx.x < D) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) s += part[r][threadIdx.x];
        const float qb = s / (float)n;
        a.qbar[((size_t)h * a.nB + i) * D + threadIdx.x] = qb;
        sq = qb * qb;
    }
    sq = warp_sum(sq);
    if ((threadIdx.x & 31) == 0 && threadIdx.x < D) red[threadIdx.x >> 5] = sq;
    __syncthreads();
    if (threadIdx.x == 0) a.qnorm[(size_t)h * a.nB + i] = sqrtf((red[0] + red[1]) + (red[2] + red[3]));
}

// ---------------------------------------------------------------------------
// lower-triangular tile index -> (I, J), J <= I
__device__ __forceinline__ void tri_index(int x, int &I, int &J)
{
    int r = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
    while ((r + 1) * (r + 2) / 2 <= x) ++r;
    while (r * (r + 1) / 2 > x) --r;
    I = r;
    J = x - r * (r + 1) / 2;
}

template <bool QUANT>
__global__ void __launch_bounds__(256) k_pair_tile(const RbsArgs a)
{
    constexpr int D = 128;
    extern __shared__ __align__(16) float smem[];
    float *sQ = smem;             // [D][64] transposed pooled queries
    float *sC = smem + D * 64;    // [D][64] transposed centroids
    int I, J;
    tri_index(blockIdx.x, I, J);
    const int h = blockIdx.y;
    const int g = h / (a.Hq / a.c.Hkv);
    const int tid = threadIdx.x;
    // load the two 64 x 128 fp32 tiles, transposed
    for (int x = tid; x < 64 * (D / 4); x += 256) {
        const int r = x & 63, kq = x >> 6;     // row, float4 column index
        const int i = I * 64 + r, j = J * 64 + r;
        float4 qv = make_float4(0, 0, 0, 0), cv = make_float4(0, 0, 0, 0);
        if (i < a.nB) qv = *reinterpret_cast<const float4 *>(a.qbar + ((size_t)h * a.nB + i) * D + kq * 4);
        if (j < a.nB) cv = *reinterpret_cast<const float4 *>(a.cen + ((size_t)g * a.nB + j) * D + kq * 4);
        sQ[(kq * 4 + 0) * 64 + r] = qv.x; sQ[(kq * 4 + 1) * 64 + r] = qv.y;
        sQ[(kq * 4 + 2) * 64 + r] = qv.z; sQ[(kq * 4 + 3) * 64 + r] = qv.w;
        sC[(kq * 4 + 0) * 64 + r] = cv.x; sC[(kq * 4 + 1) * 64 + r] = cv.y;
        sC[(kq * 4 + 2) * 64 + r] = cv.z; sC[(kq * 4 + 3) * 64 + r] = cv.w;
    }
    __syncthreads();
    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; ++k) {
        const float4 qa = *reinterpret_cast<const float4 *>(&sQ[k * 64 + ty * 4]);
        const float4 cb = *reinterpret_cast<const float4 *>(&sC[k * 64 + tx * 4]);
        const float qr[4] = {qa.x, qa.y, qa.z, qa.w};
        const float cr[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(qr[r], cr[c], acc[r][c]);
    }
    const float tc = QUANT ? 0.f : __ldg(a.tau_c + h);
    const float tr = QUANT ? 0.f : __ldg(a.tau_r + h);
    const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int i = I * 64 + ty * 4 + r;
        const float qn = i < a.nB ? a.qnorm[(size_t)h * a.nB + i] : 0.f;
        uint32_t nib = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int j = J * 64 + tx * 4 + c;
            if (i >= a.nB || j > i) continue;
            const float qc = acc[r][c];
            const float sc = a.scale * qc;
            const float sr = a.scale * fmaf(qn, a.rad[(size_t)g * a.nB + j], qc);
            if (QUANT) {
                const size_t p = (size_t)i * (i + 1) / 2 + j;
                a.pair_sc[(size_t)h * nP + p] = sc;
                a.pair_sc[((size_t)a.Hq + h) * nP + p] = sr;
            } else {
                const bool keep = sc > tc || sr > tr || (a.force_diag && j == i) || (a.force_first && j == 0);
                nib |= (uint32_t)keep << c;
            }
        }
        if (!QUANT) {
            uint32_t w = nib << ((tx & 7) * 4);
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) w |= __shfl_xor_sync(0xffffffffu, w, o);
            if ((tx & 7) == 0 && i < a.nB) {
                const int words = 2 * ((a.nB + 63) / 64);
                a.bits[((size_t)h * a.nB + i) * words + J * 2 + (tx >> 3)] = w;
                if (w) atomicAdd(&a.rowcnt[h * a.nB + i], __popc(w));
            }
        }
    }
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

// Lower quantile: the element at ascending rank floor(p*(n-1)) among head h's
// causal pair scores of one branch (exact, three radix digit passes).
__global__ void __launch_bounds__(1024) k_quantile(const RbsArgs a)
{
    __shared__ unsigned hist[2048];
    __shared__ long long wt[33];
    __shared__ unsigned s_digit;
    __shared__ long long s_below;
    const int branch = blockIdx.x / a.Hq, h = blockIdx.x % a.Hq;
    const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
    const float *x = a.pair_sc + ((size_t)branch * a.Hq + h) * nP;
    const float p = branch == 0 ? a.p_c : a.p_r;
    long long need = (long long)floor((double)p * (double)(nP - 1)) + 1;   // 1-based ascending rank
    uint32_t prefix = 0, pmask = 0;
    const int shifts[3] = {21, 10, 0}, nbits[3] = {11, 11, 10};
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = shifts[pass], nb = 1 << nbits[pass];
        for (int t = threadIdx.x; t < nb; t += blockDim.x) hist[t] = 0;
        __syncthreads();
        for (size_t t = threadIdx.x; t < nP; t += blockDim.x) {
            const uint32_t key = f2key(x[t]);
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
        }
        __syncthreads();
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
        need -= s_below;
        prefix |= s_digit << shift;
        pmask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const uint32_t u = (prefix & 0x80000000u) ? (prefix & 0x7fffffffu) : ~prefix;
        a.tau[branch * a.Hq + h] = __uint_as_float(u);
    }
}

// quantile mode: threshold the stored pair scores; one warp per row (h, i)
__global__ void __launch_bounds__(256) k_mask_scores(const RbsArgs a)
{
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.Hq * a.nB) return;
    const int h = row / a.nB, i = row % a.nB;
    const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
    const float *sc = a.pair_sc + (size_t)h * nP + (size_t)i * (i + 1) / 2;
    const float *sr = a.pair_sc + ((size_t)a.Hq + h) * nP + (size_t)i * (i + 1) / 2;
    const float tc = a.tau[h], tr = a.tau[a.Hq + h];
    const int words = 2 * ((a.nB + 63) / 64);
    int cnt = 0;
    for (int w0 = 0; w0 <= i / 32; ++w0) {
        const int j = w0 * 32 + lane;
        bool keep = false;
        if (j <= i) keep = sc[j] > tc || sr[j] > tr || (a.force_diag && j == i) || (a.force_first && j == 0);
        const uint32_t w = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) a.bits[(size_t)row * words + w0] = w;
        cnt += __popc(w);
    }
    if (lane == 0) a.rowcnt[row] = cnt;
}

__global__ void __launch_bounds__(1024) k_csr_scan(const RbsArgs a)
{
    __shared__ long long wt[33];
    const int R = a.Hq * a.nB;
    const int per = (R + blockDim.x - 1) / blockDim.x;
    const int r0 = threadIdx.x * per, r1 = min(r0 + per, R);
    long long s = 0;
    for (int r = r0; r < r1; ++r) s += a.rowcnt[r];
    long long total;
    long long run = block_excl_scan_ll(s, wt, total);
    for (int r = r0; r < r1; ++r) {
        a.row_ptr[r] = (int32_t)min(run, (long long)INT32_MAX);
        run += a.rowcnt[r];
    }
    if (threadIdx.x == 0) {
        a.row_ptr[R] = (int32_t)min(total, (long long)INT32_MAX);
        if (total > a.nnz_cap) record(a.st, SA_ERR_CAPACITY, CHK_CAPACITY_CSR, (int)min(total, (long long)INT32_MAX));
    }
}

__global__ void __launch_bounds__(256) k_csr_fill(const RbsArgs a)
{
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= a.Hq * a.nB) return;
    const int i = row % a.nB;
    const int words = 2 * ((a.nB + 63) / 64);
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

__global__ void k_copy_tau(const RbsArgs a)
{
    const int h = threadIdx.x + blockIdx.x * blockDim.x;
    if (h >= a.Hq) return;
    a.tau[h] = a.tau_c[h];
    a.tau[a.Hq + h] = a.tau_r[h];
}

__global__ void k_tau_out(const RbsArgs a)
{
    const int x = threadIdx.x + blockIdx.x * blockDim.x;
    if (x < 2 * a.Hq) a.tau_out[x] = a.tau[x];
}

}  // namespace

cudaError_t launch_rbs(const RbsArgs &a, cudaStream_t s)
{
    if (a.c.D != 128) return cudaErrorNotSupported;
    const bool quant = a.tau_c == nullptr;
    cudaError_t e;
    // per-kv-head block statistics on sequence 0's keys
    k_block_stats<<<dim3(a.nB, a.c.Hkv), 256, 0, s>>>(a);
    k_pool_q<<<dim3(a.nB, a.Hq), 256, 0, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int nTB = (a.nB + 63) / 64;
    const int tiles = nTB * (nTB + 1) / 2;
    const size_t smem = 2 * 128 * 64 * sizeof(float);
    if (quant) {
        cudaFuncSetAttribute(k_pair_tile<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_pair_tile<true><<<dim3(tiles, a.Hq), 256, smem, s>>>(a);
        k_quantile<<<2 * a.Hq, 1024, 0, s>>>(a);
        k_mask_scores<<<(a.Hq * a.nB + 7) / 8, 256, 0, s>>>(a);
    } else {
        cudaFuncSetAttribute(k_pair_tile<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_copy_tau<<<(a.Hq + 127) / 128, 128, 0, s>>>(a);
        if ((e = cudaMemsetAsync(a.rowcnt, 0, (size_t)a.Hq * a.nB * sizeof(int32_t), s)) != cudaSuccess) return e;
        k_pair_tile<false><<<dim3(tiles, a.Hq), 256, smem, s>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_csr_scan<<<1, 1024, 0, s>>>(a);
    k_csr_fill<<<(a.Hq * a.nB + 7) / 8, 256, 0, s>>>(a);
    if (a.tau_out) k_tau_out<<<(2 * a.Hq + 127) / 128, 128, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace sa
