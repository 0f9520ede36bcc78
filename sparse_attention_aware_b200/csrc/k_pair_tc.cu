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
//              image into a 2-stage ring; per column 24 MMAs (M = N = 128,
//              K = 16: lo.hi, hi.lo, hi.hi per K step) into one of two TMEM
//              accumulators, committed to that accumulator's mbarrier; a
//              stage is refilled as soon as the MMAs that read it complete.
//   warps 0-7  epilogue: warp w reads TMEM lanes 32 (w % 4).. (its query
//              blocks) and columns 64 (w / 4).. of the accumulator, frees it
//              for the MMAs two columns on, then forms both branch scores,
//              the thresholds and the OR (causal and forced blocks only in
//              the first and diagonal column tiles) -> one 32-bit mask word
//              per 32 columns, or in quantile mode stores the two scores.
//              Per-row kept counts are summed over the row and added once.
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

constexpr uint32_t OFF_A = 0;                           // query tile image (hi, lo)
constexpr uint32_t OFF_B = OFF_A + kRbsImgBytes;        // 2 stages of centroid tile images
constexpr uint32_t OFF_BAR = OFF_B + 2 * kRbsImgBytes;  // a_full, b_full[2], mma_done[2], acc_free[2], drain
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

__device__ __forceinline__ void load_image(uint8_t *dst, const uint8_t *src, uint64_t *bar)
{
    mbar_arrive_expect_tx(bar, kRbsImgBytes);
#pragma unroll
    for (int q = 0; q < (int)(kRbsImgBytes / kPiece); ++q) bulk_load(dst + q * kPiece, src + q * kPiece, kPiece, bar);
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
            int loads[2] = {0, 0}, waited[2] = {0, 0};   // centroid copies issued / consumed per stage
            bool a_pending = true;
            load_image(smem + OFF_A, qimg, a_full);
            for (int J = 0; J <= I && J < 2; ++J) {
                load_image(smem + OFF_B + J * kRbsImgBytes, cimg + (size_t)J * kRbsImgBytes, b_full + J);
                ++loads[J];
            }
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
                // the epilogue of column J - 2 has read accumulator s
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
                    load_image(smem + OFF_B + o * kRbsImgBytes, cimg + (size_t)(J + 1) * kRbsImgBytes, b_full + o);
                    ++loads[o];
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
        const int i = I * kT + 32 * quarter + lane;   // this thread's query block
        const bool row_ok = i < a.nB;
        const float qn = row_ok ? a.qnorm[(size_t)h * a.nB + i] : 0.f;
        const float tc = QUANT ? 0.f : __ldg(a.tau_c + h);
        const float tr = QUANT ? 0.f : __ldg(a.tau_r + h);
        const size_t nP = (size_t)a.nB * (a.nB + 1) / 2;
        const int words = rbs_mask_words(a.nB);
        const float *radg = a.rad + (size_t)g * a.nB;
        // 16-byte radius loads only where the kv head's row starts aligned
        const bool rad16 = (reinterpret_cast<uintptr_t>(radg) & 15) == 0;
        const float2 sc2 = make_float2(a.scale, a.scale), qn2 = make_float2(qn, qn);
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
            fence_before_sync();
            mbar_arrive(acc_free + s);
            const int j0 = J * kT + 64 * colh;
            // interior column tiles hold neither the diagonal nor block 0, and
            // every pair in them is causal
            const bool edge = J == 0 || J == I;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                uint32_t word = 0;
#pragma unroll
                for (int c8 = 0; c8 < 32; c8 += 8) {
                    const int jb = j0 + 32 * t + c8;
                    float rr[8];
                    if (rad16 && jb + 8 <= a.nB) {
                        const float4 r0 = __ldg(reinterpret_cast<const float4 *>(radg + jb));
                        const float4 r1 = __ldg(reinterpret_cast<const float4 *>(radg + jb + 4));
                        rr[0] = r0.x; rr[1] = r0.y; rr[2] = r0.z; rr[3] = r0.w;
                        rr[4] = r1.x; rr[5] = r1.y; rr[6] = r1.z; rr[7] = r1.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) rr[e] = jb + e < a.nB ? __ldg(radg + jb + e) : 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const int c = c8 + e;
                        const float2 qc = make_float2(__uint_as_float(v[t][c]), __uint_as_float(v[t][c + 1]));
                        const float2 sc = fmul2(sc2, qc);
                        const float2 sr = fmul2(sc2, ffma2(qn2, make_float2(rr[e], rr[e + 1]), qc));
                        if (QUANT) {
                            const int j = jb + e;
                            if (row_ok && j <= i) {
                                const size_t p = (size_t)i * (i + 1) / 2 + j;
                                a.pair_sc[(size_t)h * nP + p] = sc.x;
                                a.pair_sc[((size_t)a.Hq + h) * nP + p] = sr.x;
                                if (j + 1 <= i) {
                                    a.pair_sc[(size_t)h * nP + p + 1] = sc.y;
                                    a.pair_sc[((size_t)a.Hq + h) * nP + p + 1] = sr.y;
                                }
                            }
                        } else {
                            bool k0 = sc.x > tc || sr.x > tr;
                            bool k1 = sc.y > tc || sr.y > tr;
                            if (edge) {
                                const int j = jb + e;
                                k0 = j <= i && (k0 || (a.force_diag && j == i) || (a.force_first && j == 0));
                                k1 = j + 1 <= i && (k1 || (a.force_diag && j + 1 == i));
                            }
                            word |= ((uint32_t)k0 << c) | ((uint32_t)k1 << (c + 1));
                        }
                    }
                }
                if (!QUANT && row_ok) {
                    a.bits[((size_t)h * a.nB + i) * words + J * 4 + 2 * colh + t] = word;
                    kept += __popc(word);
                }
            }
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
