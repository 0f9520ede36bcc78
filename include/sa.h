/*
 * sa.h -- C ABI of libsa: head-aware sparse attention over a paged bf16 KV
 * cache, built for NVIDIA B200 (sm_100a).
 *
 * The library implements the two parts of the method:
 *   - selection: exact per-head top-k on an anchor layer (Kascade), the
 *     two-branch centroid / radius-rescue block score (RBS-Attention), and
 *     block-aligned span masks (Declarative Attention focus/local/global,
 *     LoZA streaming window);
 *   - sparse attention: split-KV decode with a combine pass, and causal
 *     block-sparse prefill on tcgen05 tensor cores.
 *
 * Sources (page titles; sections named per entry point below):
 *  [Kascade] "Kascade稀疏注意力：让长上下文大模型更快落地物流供应链"
 *  [DA-1]    "语言模型能自己决定该看哪里吗？"
 *  [RBS]     "RBS-Attention: Radius-Bounded Sparse Prefill for Long-Context
 *             Large Language Models" (blog summary)
 *  [DA-2]    "百万上下文，模型终于会挑重点了"
 *  [LoZA]    "稀疏注意力机制创新：美团新技术如何提升大模型的效率与成本控制？"
 *
 * Conventions (all entry points):
 *  - Memory: every buffer argument is DEVICE memory owned by the caller,
 *    unless the comment says "host".  The library allocates nothing, keeps
 *    no pointer after a call returns and has no global state.
 *  - Asynchrony: work is enqueued on `stream`; nothing synchronises except
 *    sa_read_device_status().  A call returning SA_OK has only been
 *    enqueued.
 *  - Alignment: cache, query, output and workspace pointers must be 16-byte
 *    aligned; workspaces 256-byte aligned.
 *  - Errors: argument checks run on the host before any launch and return
 *    SA_ERR_INVALID_ARGUMENT / SA_ERR_UNSUPPORTED / SA_ERR_WORKSPACE with no
 *    work enqueued.  A failed launch returns SA_ERR_CUDA.  Bad DEVICE data
 *    (a page-table entry or index out of range, a sequence length above the
 *    cache capacity, an output capacity overflow) cannot be seen on the host:
 *    the kernel skips the bad access, records the first such error in the
 *    workspace status word, and sa_read_device_status() reports it.
 *  - Determinism: results are bitwise reproducible run to run (fixed split
 *    and reduction orders, no floating-point atomics).
 *  - Device: the current CUDA device; all pointers must live on it.
 *  - Launch: every kernel is launched with programmatic dependent launch
 *    allowed ([LoZA] "四、从外卖到AI" names PDL) and waits for the previous
 *    kernel in the stream to complete before it touches memory; it lets the
 *    next kernel be scheduled early.  A caller's kernel launched after it
 *    with the programmatic attribute must itself wait (griddepcontrol.wait /
 *    cudaGridDependencySynchronize) before reading these outputs; kernels
 *    launched without the attribute are ordered as usual.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(SA_BUILD) && defined(__GNUC__)
#define SA_API __attribute__((visibility("default")))
#else
#define SA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st *sa_stream_t;

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, misaligned pointer  */
    SA_ERR_UNSUPPORTED = 2,      /* head_dim, page size or head ratio not built  */
    SA_ERR_WORKSPACE = 3,        /* workspace missing or smaller than required   */
    SA_ERR_CUDA = 4,             /* a CUDA launch or runtime call failed         */
    SA_ERR_DEVICE_FAULT = 5,     /* recorded by a kernel: bad device-side data   */
    SA_ERR_TIMEOUT = 6,          /* recorded by a kernel: a bounded wait expired */
    SA_ERR_CAPACITY = 7          /* recorded by a kernel: an output buffer overflowed */
} sa_status;

typedef enum { SA_DTYPE_F32 = 0, SA_DTYPE_BF16 = 1 } sa_dtype;

/*
 * Paged KV cache ([DA-1], DA state machine section: vLLM keeps the KV cache in
 * fixed-size blocks and attention kernels read whole blocks).
 *   k, v        bf16 [num_pages][num_kv_heads][page_size][head_dim]; one
 *               (page, kv head) tile is contiguous.
 *   page_table  int32 [batch][max_pages_per_seq]: logical page -> physical page.
 *   seq_lens    int32 [batch]: tokens of each sequence (<= max_pages_per_seq *
 *               page_size; larger values are clamped and recorded as a fault).
 * Slots of a page past seq_len must hold finite values (the prefill tensor-core
 * product multiplies them by an exact zero weight).
 * Supported: head_dim in {64, 128} (prefill: 128), page_size in {16, 64}
 * (prefill: 64), num_q_heads % num_kv_heads == 0.
 */
typedef struct {
    const void *k;
    const void *v;
    const int32_t *page_table;
    const int32_t *seq_lens;
    int32_t batch;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t page_size;
    int32_t max_pages_per_seq;
    int32_t num_pages;
} sa_kv_cache;

/* ------------------------------------------------------------------------ */
/* Selection results consumed by the attention entry points                 */
/* ------------------------------------------------------------------------ */
typedef enum { SA_SEL_TOKENS = 1, SA_SEL_BLOCKS = 2 } sa_selection_kind;

/*
 * SA_SEL_TOKENS: per (sequence, query head) token positions, ascending
 *   idx   int32 [batch][num_q_heads][k_cap], entries [0, count) valid
 *   count int32 [batch][num_q_heads]
 * SA_SEL_BLOCKS: per sequence, shared by every head, a list of page segments
 *   blocks int32 [batch][max_blocks][4] = {logical page, lo, hi, tokens before}
 *          -- tokens page*P + lo .. page*P + hi - 1; "tokens before" is the
 *          number of selected tokens in earlier entries (a prefix sum);
 *   block_counts int32 [batch].
 */
typedef struct {
    sa_selection_kind kind;
    const int32_t *idx;
    const int32_t *count;
    int32_t k_cap;
    const int32_t *blocks;
    const int32_t *block_counts;
    int32_t max_blocks;
} sa_selection;

/* ------------------------------------------------------------------------ */
/* 1. sa_select_topk -- anchor-layer exact top-k per query head             */
/* ------------------------------------------------------------------------ */
/*
 * [Kascade] sections "核心机制：Anchor + Reuse" (exact top-k key indices on an
 * anchor layer, reused by the following layers) and "头部感知（head-aware）是
 * 精度关键" (selection per head).
 *
 * For every sequence b and query head h (kv head g = h / (Hq/Hkv)):
 *   r_t = q_h . k_{g,t}  for t < seq_lens[b]   (fp32 accumulate, unscaled)
 * and the min(k, L_b) largest r_t are kept, ties to the lower position.
 *   q          [batch][num_q_heads][head_dim], fp32 or bf16 (q_dtype)
 *   idx_out    int32 [batch][num_q_heads][k], ascending positions, -1 padded
 *   count_out  int32 [batch][num_q_heads] = min(k, L_b)
 *   ws         workspace of sa_workspace_bytes(SA_OP_SELECT_TOPK, ...) bytes
 * Errors: SA_ERR_INVALID_ARGUMENT (k < 1, k > 65536, null pointers),
 * SA_ERR_UNSUPPORTED (also: max_pages_per_seq * page_size > 2^19 tokens),
 * SA_ERR_WORKSPACE.
 */
SA_API sa_status sa_select_topk(const sa_kv_cache *kv, const void *q, sa_dtype q_dtype,
                         int32_t num_q_heads, int32_t k, int32_t *idx_out, int32_t *count_out,
                         void *ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* 2. sa_select_blocks -- block-level selection                             */
/* ------------------------------------------------------------------------ */
typedef enum { SA_SEL_RBS = 1, SA_SEL_SPANS = 2 } sa_select_mode;

/*
 * SA_SEL_RBS ([RBS] section "关键技术点": 1. centroid base branch and radius
 * rescue branch; 2. independent thresholds, masks OR'd, block-sparse
 * FlashAttention path unchanged).  Causal prefill of sequence 0 of `kv`,
 * blocks of block_size tokens (query blocks and key blocks alike):
 *   c_j = mean of block j's keys, r_j = max ||k - c_j||  (per kv head)
 *   qbar_i = mean of block i's queries                    (per q head)
 *   S_c = scale * qbar_i . c_j,  S_r = scale * (qbar_i . c_j + ||qbar_i|| r_j)
 *   M(i,j) = [S_c > tau_c] | [S_r > tau_r] | [j == i]*force_diag | [j == 0]*force_first,
 *   for j <= i.  Thresholds: explicit per head (tau_c, tau_r: device fp32
 *   [num_q_heads]) or, when tau_c == NULL, the lower quantile p of the head's
 *   causal pair scores: sorted_asc[floor(p*(n-1))] (p_c, p_r).
 *   scale must be finite and > 0 (SA_ERR_INVALID_ARGUMENT otherwise).
 *   Precision: the products qbar_i . c_j run on tensor cores with each fp32
 *   operand split into bf16 hi + lo parts (lo.hi + hi.lo + hi.hi, fp32
 *   accumulation): |error| <= 3 * 2^-18 * scale * sum_k |qbar_ik c_jk| plus
 *   fp32 rounding.  Explicit thresholds are applied as qbar.c > tau_c / scale
 *   and qbar.c + ||qbar|| r > tau_r / scale (the same test up to fp32
 *   rounding of the quotients).
 *   q          bf16 [num_tokens][num_q_heads][head_dim]
 *   Output: CSR over rows (h, i), row = h * nQB + i, nQB = ceil(T / block_size):
 *     row_ptr int32 [num_q_heads*nQB + 1], cols int32 [nnz_capacity] ascending.
 *     An overflow of nnz_capacity is recorded as SA_ERR_CAPACITY; row_ptr
 *     still holds the true counts.
 *     tau_out (nullable) fp32 [2][num_q_heads]: the thresholds applied.
 *
 * SA_SEL_SPANS ([DA-1] DA state machine: chunk-level mask, kept ranges
 * rounded OUT to KV-block edges; [DA-2] "三种模式"; [LoZA] "二、ZigZag架构":
 * fixed streaming window).  Per sequence b, spans int32 [batch][max_spans][2]
 * = [start, end) token ranges (span_counts[b] of them); span_round uint8
 * [batch][max_spans] = 1 to round the span out to page edges.  Spans are
 * clipped to [0, L_b) and merged so every token counts once.
 *   Output: blocks int32 [batch][max_blocks][4] (see sa_selection), block_counts
 *   int32 [batch].  An overflow of max_blocks is recorded as SA_ERR_CAPACITY.
 */
typedef struct {
    sa_select_mode mode;
    /* RBS */
    const void *q;
    int32_t num_q_heads;
    int32_t num_tokens;
    int32_t block_size;       /* 64 */
    float scale;
    const float *tau_c;       /* device [Hq] or NULL (quantile mode) */
    const float *tau_r;       /* device [Hq] or NULL (quantile mode) */
    float p_c, p_r;
    int32_t force_diag, force_first;
    /* SPANS */
    const int32_t *spans;
    const int32_t *span_counts;
    const uint8_t *span_round;
    int32_t max_spans;
} sa_block_select_args;

typedef struct {
    /* RBS */
    int32_t *row_ptr;
    int32_t *cols;
    int64_t nnz_capacity;
    float *tau_out;
    /* SPANS */
    int32_t *blocks;
    int32_t *block_counts;
    int32_t max_blocks;
} sa_block_list;

SA_API sa_status sa_select_blocks(const sa_kv_cache *kv, const sa_block_select_args *args,
                           sa_block_list *out, void *ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* 3. sa_sparse_decode_attn -- split-KV sparse decode + combine             */
/* ------------------------------------------------------------------------ */
/*
 * [Kascade] "核心机制" (attention only over the k selected positions, on the
 * anchor and on reuse layers alike); [DA-1] (block-aligned masks read whole
 * KV blocks); [LoZA] "四、从外卖到AI" (SplitKV-and-Combine).
 * One query token per sequence.  For query head h of sequence b over the
 * selected token set S (tokens or blocks, see sa_selection):
 *   s_t = scale * q.k_t;  out = sum softmax(s)_t v_t;  lse = log sum exp s_t.
 * The set is cut into num_splits contiguous parts (split-KV); every part
 * yields (max, sum, partial output) and a combine pass merges them.  An
 * empty set gives out = 0 and lse = -inf.
 * Block lists (one list per sequence, shared by every head) with at most 16
 * query heads per kv head are computed per GQA group on tensor cores: the
 * parts are runs of list entries balanced by entry count, a sequence using
 * only as many of the num_splits parts as give each at least ~128 tokens
 * (max(1, 128 / page_size) entries; the rest stay empty), S = q.k is
 * accumulated in fp32 (an fp32 query as bf16 high + low parts), and the
 * softmax weights enter the P.V product as bf16.
 *   q        [batch][num_q_heads][head_dim], fp32 or bf16
 *   out      bf16 [batch][num_q_heads][head_dim]
 *   lse_out  fp32 [batch][num_q_heads] natural log, nullable
 *   num_splits in [1, 64]
 */
SA_API sa_status sa_sparse_decode_attn(const sa_kv_cache *kv, const void *q, sa_dtype q_dtype,
                                int32_t num_q_heads, const sa_selection *sel, float scale,
                                int32_t num_splits, void *out, float *lse_out, void *ws,
                                size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* 3b. sa_sparse_decode_attn_noalloc -- decode without a caller workspace   */
/* ------------------------------------------------------------------------ */
/*
 * The pages have no counterpart to this entry point.  It is for callers that
 * are not able to allocate device memory: for example a plugin that its host
 * engine hands only input and output buffers (the engine owns every device
 * allocation), or a latency-critical serving loop that must never call into
 * an allocator.  Such callers cannot provide the workspace that
 * sa_sparse_decode_attn needs for its split-KV partial states.
 *
 * It computes exactly what sa_sparse_decode_attn computes (same kernels, same
 * arguments except the workspace, bitwise the same results) and allocates
 * nothing: its scratch is a device array of SA_NOALLOC_DECODE_SCRATCH_BYTES
 * (8 MiB) built into libsa, which every GPU that loads the library holds
 * until the process exits.
 *   Limit: 256 + round_up_256(batch*num_q_heads*num_splits*head_dim*4)
 *          + round_up_256(batch*num_q_heads*num_splits*8) must not exceed
 *          8 MiB; larger calls return SA_ERR_UNSUPPORTED with nothing enqueued.
 *   Set-up: the first call on each device looks up the array's device address
 *          (with that device current); make that first call before any stream
 *          capture begins.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *          call's contents.  Calls whose GPU work overlaps in time (different
 *          streams, or threads without ordering) race on it and corrupt each
 *          other's results; order them.  Nothing in it needs to start zeroed:
 *          each call rewrites every partial state it reads.
 *   Errors: the same host-side checks as sa_sparse_decode_attn.  Bad device
 *          data is still skipped by the kernels, but its record stays inside
 *          the library's array and is not reported; use sa_sparse_decode_attn
 *          with a workspace when those checks must be read.
 */
#define SA_NOALLOC_DECODE_SCRATCH_BYTES (8u * 1024u * 1024u)

SA_API sa_status sa_sparse_decode_attn_noalloc(const sa_kv_cache *kv, const void *q, sa_dtype q_dtype,
                                               int32_t num_q_heads, const sa_selection *sel,
                                               float scale, int32_t num_splits, void *out,
                                               float *lse_out, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* 4. sa_sparse_prefill_attn -- causal block-sparse prefill (tcgen05)       */
/* ------------------------------------------------------------------------ */
/*
 * [RBS] "关键技术点" 2 (selection feeds an unchanged block-sparse attention
 * path).  Sequence 0 of `kv` holds the keys/values of the num_tokens prompt
 * tokens (page_size must equal the 64-token block).  For query token t of head
 * h in query block i = t / 64, attend to tokens t' <= t whose key block
 * t'/64 is listed in CSR row h*nQB + i (csr->row_ptr / csr->cols /
 * csr->nnz_capacity as produced by sa_select_blocks(SA_SEL_RBS); column
 * entries at or past nnz_capacity, out of [0, i] or not strictly ascending are
 * recorded as a device fault and skipped).
 *   q        bf16 [num_tokens][num_q_heads][128]
 *   out      bf16 [num_tokens][num_q_heads][128]
 *   lse_out  fp32 [num_tokens][num_q_heads] natural log, nullable
 *   causal   must be 1; scale must be finite and > 0.
 * Work is scheduled in pairs of 64-row query blocks that share their K/V
 * tiles: two (head, query block) rows of one GQA group from a window of
 * 64/G nearby query blocks, matched greedily by the key blocks the two rows
 * do not share and refined by pair exchanges (adjacent query blocks of one
 * head when the group size is odd or above 16); the pairing list lives in
 * the workspace.  Results do not depend on the pairing.
 */
SA_API sa_status sa_sparse_prefill_attn(const sa_kv_cache *kv, const void *q, int32_t num_q_heads,
                                 int32_t num_tokens, const sa_block_list *csr, float scale,
                                 int32_t causal, void *out, float *lse_out, void *ws, size_t ws_bytes,
                                 sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* 5. sa_fetch_pages -- bring KV pages from a host tier into device slots   */
/* ------------------------------------------------------------------------ */
/*
 * [DA-1] (a step only hides context, it deletes none, so the KV pages no
 * step is reading can sit in an outer memory tier and be fetched back,
 * overlapped with decoding, when a declaration names them again); [DA-2]
 * "对百万上下文产品意味着什么" (the KV cache as tiered storage: recent content
 * in HBM, focus regions loaded on demand, far history in CPU memory).
 * For pair i = {src, dst} (int32 [n][2] in device memory), page src of the
 * host tier goes to page slot dst of the device pools, K and V alike:
 *   host_k, host_v  page-major arrays of page_bytes-sized pages in pinned host
 *                   memory the device reads at the same address (cudaHostAlloc
 *                   / cudaMallocHost / a pinned torch tensor, with unified
 *                   addressing); host_pages pages each
 *   dev_k, dev_v    the cache pools (kv->k, kv->v layout), dev_pages slots
 *   page_bytes      num_kv_heads*page_size*head_dim*2, a multiple of 16
 * One kernel gathers every pair with 16-byte loads over the host link (no
 * per-page copy calls).  A pair whose src is outside [0, host_pages) or whose
 * dst is outside [0, dev_pages) is skipped and recorded as
 * SA_ERR_DEVICE_FAULT in ws.  Two pairs must not name the same dst.
 *   ws  any workspace of at least 256 bytes (only its status word is used).
 */
SA_API sa_status sa_fetch_pages(const void *host_k, const void *host_v, void *dev_k, void *dev_v,
                                const int32_t *pairs, int32_t n, int64_t host_pages, int64_t dev_pages,
                                size_t page_bytes, void *ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------------ */
/* 5b. sa_tier_plan -- host-side slot planning for a tiered KV cache        */
/* ------------------------------------------------------------------------ */
/*
 * [DA-1], [DA-2] as for sa_fetch_pages: before a step, the host pages it reads
 * are mapped onto the fixed pool of device page slots.  Host code only (no GPU
 * work, no stream); the caller's state arrays are updated in place:
 *   slot_of   int32 [host_pages]  slot holding each host page, -1 if none
 *   page_in   int32 [slots]       host page in each slot, -1 if the slot is free
 *   last_use  int64 [slots]       tick of each slot's last use
 * wanted (int32 [n_wanted], pages in [0, host_pages), duplicates allowed) are
 * the pages of this step; keep (int32 [n_keep]) the pages of the step still in
 * flight, which are never evicted.  Each distinct wanted page, in order of
 * first occurrence: a resident page is a hit (its slot's last_use becomes
 * tick); a missing page takes the next free slot in ascending order, then the
 * least recently used slot (ties to the lower slot) whose page is neither
 * wanted nor kept, evicting that page.
 * Outputs (capacity `slots` entries each):
 *   pairs    int32 [n][2] {host page, slot} of the missing pages, in order
 *   evicted  int32 [m] host pages removed from their slots, in claim order
 *   counts   int32 [4] {n, m, hits, distinct wanted pages}
 *   scratch  int32 [scratch_ints], scratch_ints >= sa_tier_plan_scratch_ints(
 *            host_pages, slots); zero-filled before the first call and then
 *            kept with the state arrays (it holds the page marks between
 *            calls); the library allocates nothing and keeps no state.
 * Errors: SA_ERR_INVALID_ARGUMENT (a null pointer, slots or host_pages < 1, a
 * wanted or kept page out of range); SA_ERR_WORKSPACE (scratch too small);
 * SA_ERR_CAPACITY (more distinct wanted pages than slots, or too few slots that
 * may be evicted).  On an error the state arrays are left unchanged.  Calls on
 * distinct state and scratch arrays may run concurrently.
 */
SA_API sa_status sa_tier_plan(int32_t *slot_of, int64_t host_pages, int32_t *page_in, int64_t *last_use,
                              int32_t slots, int64_t tick, const int32_t *wanted, int32_t n_wanted,
                              const int32_t *keep, int32_t n_keep, int32_t *pairs, int32_t *evicted,
                              int32_t *counts, int32_t *scratch, int64_t scratch_ints);

/* int32 words of scratch sa_tier_plan needs: 1 + host_pages + 4 * slots (0 if
 * either argument is < 1). */
SA_API int64_t sa_tier_plan_scratch_ints(int64_t host_pages, int32_t slots);

/* ------------------------------------------------------------------------ */
/* Workspace sizing, status                                                 */
/* ------------------------------------------------------------------------ */
typedef enum {
    SA_OP_SELECT_TOPK = 1,
    SA_OP_SELECT_BLOCKS = 2,
    SA_OP_DECODE = 3,
    SA_OP_PREFILL = 4
} sa_op;

/* Host-side description of a call, for sizing.  Fields an op does not use
 * are ignored: SELECT_TOPK {num_q_heads, k}; SELECT_BLOCKS {block_args};
 * DECODE {num_q_heads, num_splits}; PREFILL {num_q_heads, num_tokens}. */
typedef struct {
    int32_t num_q_heads;
    int32_t k;
    int32_t num_splits;
    int32_t num_tokens;
    const sa_block_select_args *block_args;
} sa_ws_query;

/* Bytes of device workspace the op needs (a multiple of 256, at least 256
 * for the status word); 0 when the description is invalid.  Host only. */
SA_API size_t sa_workspace_bytes(sa_op op, const sa_kv_cache *kv, const sa_ws_query *query);

/* Zero the status word at the head of a workspace (asynchronous).  Call once
 * after allocating a workspace that was not zero-filled. */
SA_API sa_status sa_workspace_init(void *ws, size_t ws_bytes, sa_stream_t stream);

/* Diagnostic of the bounded waits: enqueues one CTA whose thread waits, with
 * the bounded-wait helper every kernel uses, on an mbarrier that nothing ever
 * arrives on.  After timeout_ns (0 < timeout_ns <= 1e10) the wait gives up,
 * SA_ERR_TIMEOUT (check id 11, value -1) is recorded in ws as a kernel would
 * record it, and the kernel returns; the context stays usable.
 *   ws  any workspace of at least 256 bytes (only its status word is used).
 * Errors: SA_ERR_INVALID_ARGUMENT (timeout out of range), SA_ERR_WORKSPACE. */
SA_API sa_status sa_check_bounded_wait(int64_t timeout_ns, void *ws, size_t ws_bytes, sa_stream_t stream);

/* Synchronises `stream`, then returns and clears the first error a kernel
 * recorded in `ws` (SA_OK if none).  detail (host, nullable) receives
 * {status, check id, offending value}. */
SA_API sa_status sa_read_device_status(void *ws, sa_stream_t stream, int32_t *detail);

SA_API const char *sa_status_string(sa_status status);

/* Library version (major*10000 + minor*100 + patch). */
SA_API int32_t sa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SA_H_ */
