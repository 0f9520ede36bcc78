// Internal launch interface between the C-ABI layer (sa_api.cu) and the
// kernel translation units.  Not installed; not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sa.h"
#include "sa_common.cuh"

namespace sa {

struct CacheArgs {
    const uint16_t *k;
    const uint16_t *v;
    const int32_t *pt;
    const int32_t *sl;
    int B, Hkv, D, P, Plog2, max_pages, num_pages;
};

// ---- decode -----------------------------------------------------------------
struct DecodeArgs {
    CacheArgs c;
    const void *q;
    bool q_f32;
    int Hq;
    float qscale;  // scale * log2(e)
    bool blocks;   // SA_SEL_BLOCKS
    const int32_t *idx;
    const int32_t *cnt;
    int kcap;
    const int32_t *ent;   // [B][max_blocks][4]
    const int32_t *ecnt;  // [B]
    int max_blocks;
    int S;
    float *part_o;   // [B*Hq][S][D]
    float *part_ml;  // [B*Hq][S][2]
    uint16_t *out;   // bf16 [B*Hq][D]
    float *lse;      // [B*Hq] or null
    DevStatus *st;
};
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
// bytes of workspace sa_sparse_decode_attn needs (status header + partials)
size_t decode_workspace_bytes(const sa_kv_cache *kv, int Hq, int S);

// ---- host-tier page fetch ---------------------------------------------------
struct FetchArgs {
    const void *host_k, *host_v;   // pinned host memory, device-readable
    void *dev_k, *dev_v;
    const int32_t *pairs;          // [n][2] {host page, device slot}
    int n;
    long long host_pages, dev_pages;
    size_t page_bytes;
    DevStatus *st;
};
cudaError_t launch_fetch(const FetchArgs &a, cudaStream_t s);
// block-list selections with at most 16 query heads per kv head: one CTA per
// (split, kv head, sequence) on mma.sync (k_decode_gqa.cu)
bool decode_gqa_supported(const DecodeArgs &a);
cudaError_t launch_decode_gqa_split(const DecodeArgs &a, cudaStream_t s);

// ---- top-k ------------------------------------------------------------------
struct TopkArgs {
    CacheArgs c;
    const void *q;
    bool q_f32;
    int Hq;
    int k;
    float *scores;  // [B*Hq][Lcap]
    int Lcap;
    int32_t *idx;
    int32_t *cnt;
    DevStatus *st;
};
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t s);
// diagnostic bounded wait (k_diag.cu)
cudaError_t launch_wait_diag(DevStatus *st, unsigned long long timeout_ns, cudaStream_t s);

// ---- spans ------------------------------------------------------------------
struct SpanArgs {
    CacheArgs c;
    const int32_t *spans;
    const int32_t *span_counts;
    const uint8_t *span_round;
    int max_spans;
    int32_t *ent;
    int32_t *ecnt;
    int max_blocks;
    DevStatus *st;
};
cudaError_t launch_spans(const SpanArgs &a, cudaStream_t s);

// ---- RBS selection ------------------------------------------------------------
struct RbsArgs {
    CacheArgs c;
    const uint16_t *q;  // bf16 [T][Hq][D]
    int Hq, T, bs, nB;
    float scale;
    const float *tau_c, *tau_r;  // explicit (device) or null
    float p_c, p_r;
    int force_diag, force_first;
    // workspace pieces
    uint8_t *cen;    // centroids, tile images [Hkv][nTB][64 KB] (rbs_img_offset)
    float *rad;      // [Hkv][nTB * 128] (rows past nB are 0)
    uint8_t *qbar;   // pooled queries, tile images [Hq][nTB][64 KB]
    float *qnorm;    // [Hq][nB]
    float *tau;      // [2][Hq] thresholds in use
    uint32_t *bits;  // [Hq][nB][rbs_mask_words(nB)] mask bits
    int32_t *rowcnt; // [Hq*nB]
    float *pair_sc;  // quantile mode: [Hq][nP] S_c, [Hq][nP] S_r
    uint32_t *qhist; // quantile mode scratch
    // outputs
    int32_t *row_ptr;
    int32_t *cols;
    int64_t nnz_cap;
    float *tau_out;
    DevStatus *st;
};
// mask bit words per (head, query block) row: 4 per 128-wide column tile
__host__ __device__ inline int rbs_mask_words(int nB) { return 4 * ((nB + 127) / 128); }
// Pooled vectors (d = 128) as tensor-core tile images: each fp32 value x is
// kept as two bf16 parts, hi = bf16(x) and lo = bf16(x - hi); 128 blocks form
// a 64 KB tile [part][K half][row][128 bytes] in the 128-byte-swizzled K-major
// layout (16-byte chunk c of a row's K half stored at chunk c ^ (row % 8)).
// Tile t of matrix m (a head or kv head) starts at (m * nTB + t) * 64 KB.
constexpr int kRbsImgRows = 128;
constexpr uint32_t kRbsImgBytes = 65536;
__host__ __device__ inline int rbs_img_tiles(int nB) { return (nB + kRbsImgRows - 1) / kRbsImgRows; }
__host__ __device__ inline uint32_t rbs_img_offset(int row, int k, int part)
{
    return (uint32_t)(part * 2 + (k >> 6)) * 16384u + (uint32_t)row * 128u +
           ((uint32_t)(((k & 63) >> 3) ^ (row & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}
size_t rbs_workspace_layout(int Hq, int Hkv, int D, int nB, bool quantile, size_t *offs);
cudaError_t launch_rbs(const RbsArgs &a, cudaStream_t s);
// pair scores + thresholds + OR + forced blocks on tcgen05 (mask words and
// row counts; in quantile mode the two scores of every causal pair)
cudaError_t launch_pair_tc(const RbsArgs &a, bool quant, cudaStream_t s);

// ---- prefill ------------------------------------------------------------------
struct PrefillArgs {
    CacheArgs c;
    const uint16_t *q;  // bf16 [T][Hq][128]
    int Hq, T;
    float scale;
    const int32_t *row_ptr;
    const int32_t *cols;
    int64_t nnz_cap;
    uint16_t *out;
    float *lse;
    int4 *items;    // workspace: per CTA {head A, q-block A, head B (-1: none), q-block B}
    int n_items;
    DevStatus *st;
};
// number of prefill work items (two 64-row halves each) for a problem
int prefill_items(int Hq, int Hkv, int nQB);
cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t s);

}  // namespace sa
