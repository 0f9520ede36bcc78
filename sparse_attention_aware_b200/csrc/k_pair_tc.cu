// RBS pair scores on tcgen05 tensor cores.
//
// Method: "RBS-Attention: Radius-Bounded Sparse Prefill…" (blog summary),
// section "关键技术点", items 1-2: for every causal pair of query block i and
// key block j <= i of head h, the centroid score S_c = scale * qbar_i . c_j
// and the rescue score S_r = scale * (qbar_i . c_j + ||qbar_i|| r_j); each
// branch is compared with its own threshold and the two masks are OR'd with
// the forced diagonal and first block.
//
// The pooled products qbar . c of one head are a dense contraction (nB x nB x
// d, causal half), so they run on the tensor cores.  The operands are fp32
// means of bf16 rows; k_pool_q and k_block_stats store each value x as two
// bf16 parts, hi = bf16(x) and lo = bf16(x - hi) (x - hi is exact), already
// in the swizzled shared-memory layout of the MMA (tile images), and a
// product is taken as lo.hi + hi.lo + hi.hi with fp32 accumulation in tensor
// memory.  Every bf16 x bf16 product is exact in fp32; the dropped lo.lo term
// and the rounding of lo leave a relative error of at most 3 * 2^-18 per
// product, so |S - S_exact| <= 3 * 2^-18 * scale * sum_k |qbar_k c_k| plus the
// fp32 accumulation error -- about 1e-4 for pooled statistics of unit-scale
// keys at d = 128, inside the 1e-3 score gaps that the thresholds of this
// selector are placed in for parity.
//
// One CTA per (row tile I of 128 query blocks, head h), rows issued longest
// first so that the grid balances over the SMs; the CTA walks the column
// tiles J = 0..I.
//   warp 8     producer and MMA issuer (one thread): bulk copies of the
//              row's query tile image (once) and of each column's centroid
//              image and radii into a 2-stage ring; per column 24 MMAs
//              (M = N = 128, K = 16: lo.hi, hi.lo, hi.hi per K step) into
//              one of two TMEM accumulators, committed to that accumulator's
//              mbarrier; a stage is refilled as soon as the MMAs that read
//              it complete.
//   warps 0-7  epilogue: warp w reads TMEM lanes 32 (w % 4).. (its query
//              blocks) and columns 64 (w / 4).. of the accumulator and forms
//              the thresholded branch scores and their OR as one 32-bit mask
//              word per 32 columns (causal and forced bits applied per word
//              in the first and diagonal column tiles), or in quantile mode
//              stores the two scores; it then frees the accumulator for the
//              MMAs two columns on.  Per-row kept counts are summed over the
//              row and added once.
// Waits are bounded (globaltimer deadline, shared abort flag); on expiry the
// kernel records SA_ERR_TIMEOUT, every role leaves its loop, the producer
// waits (bounded) for its outstanding copies and MMAs, TMEM is freed and the
// CTA returns.
#include "sa_internal.h"
#include "tc_ptx.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int kD = 128;                       // head dim (pooled vectors)
constexpr int kT = kRbsImgRows;               // tile edge (blocks)
constexpr int kEpiThreads = 256;              // warps 0-7
constexpr int kThr = kEpiThreads + 32;        // + producer warp
constexpr uint32_t kOp = kRbsImgBytes / 2;    // one part (hi or lo) of a tile image: 32 KB
constexpr uint32_t kPiece = 16384;            // bulk-copy piece

constexpr int kRadStages = 4;                 // radii ring (see the producer's refill rule)
constexpr int kStgStride = 17;                // quantile-mode staging row stride (floats)

constexpr uint32_t OFF_A = 0;                           // query tile image (hi, lo)
constexpr uint32_t OFF_B = OFF_A + kRbsImgBytes;        // 2 stages of centroid tile images
constexpr uint32_t OFF_RAD = OFF_B + 2 * kRbsImgBytes;  // radii ring [kRadStages][kT]
constexpr uint32_t OFF_STG = OFF_RAD + kRadStages * kT * 4;   // per epilogue warp: 32 x 16 scores
constexpr uint32_t OFF_BAR = OFF_STG + 8 * 32 * kStgStride * 4;   // a_full, b_full[2], mma_done[2], acc_free[2], drain
constexpr int kNumBars = 8;
constexpr uint32_t OFF_MISC = OFF_BAR + kNumBars * 8;   // TMEM base, abort flag
constexpr uint32_t kSmem = OFF_MISC + 8 + 1024;         // + slack for the 1024-byte alignment
constexpr uint32_t kTmemCols = 2 * kT;                  // two 128-column fp32 accumulators
constexpr uint32_t IDESC = idesc_bf16(128, 128, 0, 0);
constexpr uint64_t kWaitNs = 200ull * 1000 * 1000;      // 0.2 s

__device__ __forceinline__ uint64_t op_desc(uint32_t base, int kk)
{
    return smem_desc_sw128(base + (uint32_t)(kk >> 2) * (kOp / 2) + (uint32_t)(kk & 3) * 32, 16, 1024);
}

// one column tile: its centroid image and its 128 radii, on one barrier
__device__ __forceinline__ void load_column(uint8_t *dst, const uint8_t *src, float *rad_dst, const float *rad_src,
                                           uint64_t *bar)
{
    mbar_arrive_expect_tx(bar, kRbsImgBytes + kT * 4);
#pragma unroll
    for (int q = 0; q < (int)(kRbsImgBytes / kPiece); ++q) bulk_load(dst + q * kPiece, src + q * kPiece, kPiece, bar);
    bulk_load(rad_dst, rad_src, kT * 4, bar);
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
    return *reinterpret_cast<float2 *>(&d);
}

template <bool QUANT>
__global__ void __launch_bounds__(kThr, 1) k_pair_tc(const RbsArgs a, int nTB)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint8_t dsm[];
    uint8_t *smem = dsm + ((1024u - (smem_u32(dsm) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = nTB - 1 - (int)(blockIdx.x / (unsigned)a.Hq);   // longest rows first
    const int h = (int)(blockIdx.x % (unsigned)a.Hq);
    const int g = h / (a.Hq / a.c.Hkv);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *a_full = bars, *b_full = bars + 1, *mma_done = bars + 3, *acc_free = bars + 5, *drain = bars + 7;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    float *srad = reinterpret_cast<float *>(smem + OFF_RAD);
    const int rad_rows = nTB * kT;

    if (tid == 0) {
        mbar_init(a_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(b_full + s, 1);
            mbar_init(mma_done + s, 1);
            mbar_init(acc_free + s, kEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) tmem_alloc(tmem_slot, kTmemCols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint64_t deadline = globaltimer() + kWaitNs * 4;

    if (warp == 8) {
        // ---------------- producer + MMA issuer ----------------
        if (lane == 0) {
            const uint8_t *qimg = a.qbar + ((size_t)h * nTB + I) * kRbsImgBytes;
            const uint8_t *cimg = a.cen + (size_t)g * nTB * kRbsImgBytes;
            const float *radg = a.rad + (size_t)g * rad_rows;
            int loads[2] = {0, 0}, waited[2] = {0, 0};   // column copies issued / consumed per stage
            bool a_pending = true;
            mbar_arrive_expect_tx(a_full, kRbsImgBytes);
            for (int q = 0; q < (int)(kRbsImgBytes / kPiece); ++q)
                bulk_load(smem + OFF_A + q * kPiece, qimg + q * kPiece, kPiece, a_full);
            // Column J goes to image stage J % 2 and radii stage J % 4.  It is
            // loaded after the MMAs of column J - 2 complete (the last reader
            // of its image stage); those MMAs were issued after the epilogue
            // of column J - 4 released its accumulator, so the radii stage of
            // column J - 4 is free as well.
            auto load_col = [&](int J) {
                load_column(smem + OFF_B + (J & 1) * kRbsImgBytes, cimg + (size_t)J * kRbsImgBytes,
                            srad + (J % kRadStages) * kT, radg + (size_t)J * kT, b_full + (J & 1));
                ++loads[J & 1];
            };
            for (int J = 0; J <= I && J < 2; ++J) load_col(J);
            const uint32_t a_base = smem_u32(smem + OFF_A);
            bool ok = true;
            for (int J = 0; J <= I && ok; ++J) {
                const int s = J & 1;
                const uint32_t b_base = smem_u32(smem + OFF_B + s * kRbsImgBytes);
                if (a_pending) {
                    ok = mbar_wait(a_full, 0, deadline, abort_flag);
                    a_pending = !ok;
                }
                ok = ok && mbar_wait(b_full + s, (uint32_t)(J >> 1) & 1u, deadline, abort_flag);
                if (ok) ++waited[s];
                // the epilogue of column J - 2 is done with accumulator s
                if (ok && J >= 2) ok = mbar_wait(acc_free + s, (uint32_t)((J - 2) >> 1) & 1u, deadline, abort_flag);
                if (!ok) break;
                fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(s * kT);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t ah = op_desc(a_base, kk), al = op_desc(a_base + kOp, kk);
                    const uint64_t bh = op_desc(b_base, kk), bl = op_desc(b_base + kOp, kk);
                    mma_f16(d, al, bh, IDESC, kk > 0 ? 1u : 0u);
                    mma_f16(d, ah, bl, IDESC, 1u);
                    mma_f16(d, ah, bh, IDESC, 1u);
                }
                mma_commit(mma_done + s);
                // refill the other stage with column J + 1 once the MMAs of
                // column J - 1 (its last reader) have completed
                if (J >= 1 && J + 1 <= I) {
                    const int o = s ^ 1;
                    ok = mbar_wait(mma_done + o, (uint32_t)((J - 1) >> 1) & 1u, deadline, abort_flag);
                    if (!ok) break;
                    load_col(J + 1);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, 5);
                // bounded drain of this CTA's copies in flight
                volatile int never = 0;
                const uint64_t dl = globaltimer() + kWaitNs;
                if (a_pending) mbar_wait(a_full, 0, dl, &never);
                for (int s = 0; s < 2; ++s)
                    for (int n = waited[s]; n < loads[s]; ++n) mbar_wait(b_full + s, (uint32_t)n & 1u, dl, &never);
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue ----------------
        const int quarter = warp & 3, colh = warp >> 2;
        const int row0 = I * kT + 32 * quarter;
        const int i = row0 + lane;   // this thread's query block
        const bool row_ok = i < a.nB;
        const float qn = row_ok ? a.qnorm[(size_t)h * a.nB + i] : 0.f;
        const float tcs = QUANT ? 0.f : __ldg(a.tau_c + h) / a.scale;
        const float trs = QUANT ? 0.f : __ldg(a.tau_r + h) / a.scale;
        const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
        const int words = rbs_mask_words(a.nB);
        const float2 sc2 = make_float2(a.scale, a.scale), qn2 = make_float2(qn, qn);
        float *stg = reinterpret_cast<float *>(smem + OFF_STG) + warp * 32 * kStgStride;
        int kept = 0;
        for (int J = 0; J <= I; ++J) {
            const int s = J & 1;
            const bool w = mbar_wait(mma_done + s, (uint32_t)(J >> 1) & 1u, deadline, abort_flag);
            if (!__all_sync(0xffffffffu, w)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    record(a.st, SA_ERR_TIMEOUT, CHK_WAIT, 4);
                }
                break;
            }
            fence_after_sync();
            uint32_t v[2][32];
            const uint32_t ta = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(s * kT + 64 * colh);
            tmem_ld32(ta, v[0]);
            tmem_ld32(ta + 32, v[1]);
            tmem_wait_ld();
            const float *rs = srad + (J % kRadStages) * kT + 64 * colh;
            const int j0 = J * kT + 64 * colh;
            if constexpr (!QUANT) {
                // S_c > tau_c  <=>  qc > tau_c / scale, and S_r > tau_r  <=>
                // qc + qn r > tau_r / scale (scale > 0): one FMA, two
                // compares and one predicated OR per pair
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    uint32_t word = 0;
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        const float4 r4 = *reinterpret_cast<const float4 *>(rs + 32 * t + c);
                        const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float qc = __uint_as_float(v[t][c + e]);
                            if (qc > tcs || fmaf(qn, rr[e], qc) > trs) word |= 1u << (c + e);
                        }
                    }
                    const int jt = j0 + 32 * t;   // column of bit 0
                    if (J == I) {
                        // diagonal tile: causal bits only, diagonal forced
                        const int dd = i - jt;     // bit of j == i
                        word &= dd >= 31 ? 0xffffffffu : (dd < 0 ? 0u : (2u << dd) - 1u);
                        if (a.force_diag && dd >= 0 && dd < 32) word |= 1u << dd;
                    }
                    if (a.force_first && jt == 0) word |= 1u;
                    if (row_ok) {
                        a.bits[((size_t)h * a.nB + i) * words + J * 4 + 2 * colh + t] = word;
                        kept += __popc(word);
                    }
                }
            } else {
                // both scores of every causal pair, 16 columns at a time, staged
                // through shared memory so that each store instruction writes
                // two rows x 16 consecutive pairs
#pragma unroll
                for (int c16 = 0; c16 < 64; c16 += 16) {
                    const int t = c16 >> 5, cb = c16 & 31;
                    float sc[16], sr[16];
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        const float2 q2 = make_float2(__uint_as_float(v[t][cb + e]), __uint_as_float(v[t][cb + e + 1]));
                        const float2 x = fmul2(sc2, q2);
                        const float2 y = fmul2(sc2, ffma2(qn2, make_float2(rs[c16 + e], rs[c16 + e + 1]), q2));
                        sc[e] = x.x; sc[e + 1] = x.y; sr[e] = y.x; sr[e + 1] = y.y;
                    }
#pragma unroll
                    for (int br = 0; br < 2; ++br) {
                        __syncwarp();
#pragma unroll
                        for (int e = 0; e < 16; ++e) stg[lane * kStgStride + e] = br ? sr[e] : sc[e];
                        __syncwarp();
                        float *dst = a.pair_sc + ((size_t)br * a.Hq + h) * nP;
                        const int col = lane & 15, j = j0 + c16 + col;
#pragma unroll 4
                        for (int r2 = 0; r2 < 32; r2 += 2) {
                            const int rr = r2 + (lane >> 4), ir = row0 + rr;
                            if (ir < a.nB && j <= ir) dst[(size_t)ir * (ir + 1) / 2 + j] = stg[rr * kStgStride + col];
                        }
                    }
                }
            }
            // this column's accumulator and radii stage are no longer read
            fence_before_sync();
            mbar_arrive(acc_free + s);
        }
        if (!QUANT && row_ok && kept) atomicAdd(&a.rowcnt[h * a.nB + i], kept);
    }

    __syncthreads();
    if (warp == 8) {
        fence_after_sync();
        if (*abort_flag) {
            // bounded drain: a fresh commit arrives once every MMA this CTA
            // issued has completed
            if (lane == 0) {
                volatile int never = 0;
                mma_commit(drain);
                mbar_wait(drain, 0, globaltimer() + kWaitNs, &never);
            }
            __syncwarp();
        }
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_pair_tc(const RbsArgs &a, bool quant, cudaStream_t s)
{
    if (a.c.D != kD || a.Hq <= 0 || a.nB <= 0) return cudaErrorInvalidValue;
    const int nTB = rbs_img_tiles(a.nB);
    void (*kern)(const RbsArgs, int) = quant ? k_pair_tc<true> : k_pair_tc<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    if (cudaError_t e_ = launch_pdl(kern, dim3((unsigned)(nTB * a.Hq)), dim3(kThr), kSmem, s, a, nTB)) return e_;
    return cudaGetLastError();
}

}  // namespace sa
