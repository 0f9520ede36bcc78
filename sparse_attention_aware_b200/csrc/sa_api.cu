// C-ABI entry points of libsa: host-side argument validation, workspace
// layout and kernel launches.  Every check here runs before any launch, so a
// rejected call enqueues nothing.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "sa.h"
#include "sa_internal.h"

using namespace sa;

namespace sa {
// status header + split-KV partial outputs + (m, l) pairs, each rounded up to
// 256 bytes (the layout sa_sparse_decode_attn carves out of its workspace)
size_t decode_workspace_bytes(const sa_kv_cache *kv, int Hq, int S)
{
    const size_t rows = (size_t)kv->batch * Hq;
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return sizeof(DevStatus) + up(rows * S * kv->head_dim * sizeof(float)) + up(rows * S * 2 * sizeof(float));
}
}  // namespace sa

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeader = sizeof(DevStatus);

inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

inline int ilog2(int x)
{
    int r = 0;
    while ((1 << r) < x) ++r;
    return (1 << r) == x ? r : -1;
}

// Validate the cache descriptor (host-visible fields and pointers).
sa_status check_cache(const sa_kv_cache *kv, CacheArgs *c)
{
    if (!kv) return SA_ERR_INVALID_ARGUMENT;
    if (kv->batch < 0 || kv->num_kv_heads <= 0 || kv->head_dim <= 0 || kv->page_size <= 0 ||
        kv->max_pages_per_seq < 0 || kv->num_pages < 0)
        return SA_ERR_INVALID_ARGUMENT;
    if (kv->head_dim != 64 && kv->head_dim != 128) return SA_ERR_UNSUPPORTED;
    if (kv->page_size != 16 && kv->page_size != 64) return SA_ERR_UNSUPPORTED;
    if ((long long)kv->max_pages_per_seq * kv->page_size > (1LL << 30)) return SA_ERR_UNSUPPORTED;
    if (kv->batch > 0) {
        if (!kv->k || !kv->v || !kv->page_table || !kv->seq_lens) return SA_ERR_INVALID_ARGUMENT;
        if (!aligned(kv->k, 16) || !aligned(kv->v, 16) || !aligned(kv->page_table, 4) ||
            !aligned(kv->seq_lens, 4))
            return SA_ERR_INVALID_ARGUMENT;
    }
    if (c) {
        c->k = static_cast<const uint16_t *>(kv->k);
        c->v = static_cast<const uint16_t *>(kv->v);
        c->pt = kv->page_table;
        c->sl = kv->seq_lens;
        c->B = kv->batch;
        c->Hkv = kv->num_kv_heads;
        c->D = kv->head_dim;
        c->P = kv->page_size;
        c->Plog2 = ilog2(kv->page_size);
        c->max_pages = kv->max_pages_per_seq;
        c->num_pages = kv->num_pages;
    }
    return SA_OK;
}

sa_status check_ws(void *ws, size_t ws_bytes, size_t need)
{
    if (need == 0) return SA_ERR_INVALID_ARGUMENT;
    if (!ws || ws_bytes < need) return SA_ERR_WORKSPACE;
    if (!aligned(ws, kAlign)) return SA_ERR_WORKSPACE;
    return SA_OK;
}

sa_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return SA_OK;
    cudaGetLastError();  // clear the sticky-free launch error
    return SA_ERR_CUDA;
}

// ---------------- workspace sizes ----------------
size_t ws_topk(const sa_kv_cache *kv, int Hq)
{
    const size_t Lcap = (size_t)kv->max_pages_per_seq * kv->page_size;
    return kHeader + up((size_t)kv->batch * Hq * Lcap * sizeof(float));
}

size_t ws_decode(const sa_kv_cache *kv, int Hq, int S) { return sa::decode_workspace_bytes(kv, Hq, S); }

size_t ws_blocks(const sa_kv_cache *kv, const sa_block_select_args *a)
{
    if (!a) return 0;
    if (a->mode == SA_SEL_SPANS) return kHeader;
    if (a->mode != SA_SEL_RBS) return 0;
    if (a->num_q_heads <= 0 || a->num_tokens <= 0 || a->block_size <= 0) return 0;
    const int nB = (a->num_tokens + a->block_size - 1) / a->block_size;
    size_t offs[16];
    return kHeader + rbs_workspace_layout(a->num_q_heads, kv->num_kv_heads, kv->head_dim, nB,
                                          a->tau_c == nullptr, offs);
}

size_t ws_prefill(const sa_kv_cache *kv, int Hq, int T)
{
    const int nQB = (T + 63) / 64;
    return kHeader + up((size_t)prefill_items(Hq, kv->num_kv_heads, nQB) * sizeof(int4) + 16);
}

}  // namespace

extern "C" {

int32_t sa_version(void) { return 100; }

const char *sa_status_string(sa_status s)
{
    switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARGUMENT: return "SA_ERR_INVALID_ARGUMENT: invalid argument";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED: configuration not supported";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case SA_ERR_CUDA: return "SA_ERR_CUDA: CUDA launch or runtime call failed";
    case SA_ERR_DEVICE_FAULT: return "SA_ERR_DEVICE_FAULT: kernel found invalid device data";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT: bounded device wait expired";
    case SA_ERR_CAPACITY: return "SA_ERR_CAPACITY: output capacity exceeded";
    default: return "unknown sa_status";
    }
}

size_t sa_workspace_bytes(sa_op op, const sa_kv_cache *kv, const sa_ws_query *q)
{
    if (check_cache(kv, nullptr) != SA_OK || !q) return 0;
    switch (op) {
    case SA_OP_SELECT_TOPK:
        if (q->num_q_heads <= 0 || q->k <= 0) return 0;
        return ws_topk(kv, q->num_q_heads);
    case SA_OP_SELECT_BLOCKS:
        return ws_blocks(kv, q->block_args);
    case SA_OP_DECODE:
        if (q->num_q_heads <= 0 || q->num_splits <= 0 || q->num_splits > 64) return 0;
        return ws_decode(kv, q->num_q_heads, q->num_splits);
    case SA_OP_PREFILL:
        if (q->num_q_heads <= 0 || q->num_tokens < 0) return 0;
        if (q->num_q_heads % kv->num_kv_heads) return 0;
        return ws_prefill(kv, q->num_q_heads, q->num_tokens);
    default:
        return 0;
    }
}

sa_status sa_fetch_pages(const void *host_k, const void *host_v, void *dev_k, void *dev_v, const int32_t *pairs,
                         int32_t n, int64_t host_pages, int64_t dev_pages, size_t page_bytes, void *ws,
                         size_t ws_bytes, sa_stream_t stream)
{
    if (n < 0 || host_pages < 0 || dev_pages < 0 || page_bytes == 0 || page_bytes % 16) return SA_ERR_INVALID_ARGUMENT;
    if (n > 0 && (!host_k || !host_v || !dev_k || !dev_v || !pairs)) return SA_ERR_INVALID_ARGUMENT;
    if (!aligned(host_k, 16) || !aligned(host_v, 16) || !aligned(dev_k, 16) || !aligned(dev_v, 16) ||
        !aligned(pairs, 8))
        return SA_ERR_INVALID_ARGUMENT;
    sa_status st = check_ws(ws, ws_bytes, kHeader);
    if (st != SA_OK) return st;
    FetchArgs a{};
    a.host_k = host_k;
    a.host_v = host_v;
    a.dev_k = dev_k;
    a.dev_v = dev_v;
    a.pairs = pairs;
    a.n = n;
    a.host_pages = host_pages;
    a.dev_pages = dev_pages;
    a.page_bytes = page_bytes;
    a.st = static_cast<DevStatus *>(ws);
    return cuda_status(launch_fetch(a, (cudaStream_t)stream));
}

sa_status sa_workspace_init(void *ws, size_t ws_bytes, sa_stream_t stream)
{
    if (!ws || ws_bytes < kHeader || !aligned(ws, kAlign)) return SA_ERR_WORKSPACE;
    return cuda_status(cudaMemsetAsync(ws, 0, kHeader, (cudaStream_t)stream));
}

sa_status sa_check_bounded_wait(int64_t timeout_ns, void *ws, size_t ws_bytes, sa_stream_t stream)
{
    if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return SA_ERR_INVALID_ARGUMENT;
    sa_status st = check_ws(ws, ws_bytes, kHeader);
    if (st != SA_OK) return st;
    return cuda_status(sa::launch_wait_diag(static_cast<DevStatus *>(ws), (unsigned long long)timeout_ns,
                                            (cudaStream_t)stream));
}

sa_status sa_read_device_status(void *ws, sa_stream_t stream, int32_t *detail)
{
    if (!ws || !aligned(ws, kAlign)) return SA_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    DevStatus h;
    if (cudaMemcpyAsync(&h, ws, 16, cudaMemcpyDeviceToHost, s) != cudaSuccess) return cuda_status(cudaErrorUnknown);
    if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_status(cudaErrorUnknown);
    if (h.code != 0) {
        if (cudaMemsetAsync(ws, 0, 16, s) != cudaSuccess) return cuda_status(cudaErrorUnknown);
        if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_status(cudaErrorUnknown);
    }
    if (detail) {
        detail[0] = (int32_t)h.code;
        detail[1] = (int32_t)h.detail;
        detail[2] = h.value;
    }
    return (sa_status)h.code;
}

// ---------------------------------------------------------------------------
sa_status sa_select_topk(const sa_kv_cache *kv, const void *q, sa_dtype q_dtype, int32_t num_q_heads,
                         int32_t k, int32_t *idx_out, int32_t *count_out, void *ws, size_t ws_bytes,
                         sa_stream_t stream)
{
    TopkArgs a{};
    sa_status st = check_cache(kv, &a.c);
    if (st != SA_OK) return st;
    if (num_q_heads <= 0 || k <= 0 || k > 65536) return SA_ERR_INVALID_ARGUMENT;
    if (q_dtype != SA_DTYPE_F32 && q_dtype != SA_DTYPE_BF16) return SA_ERR_INVALID_ARGUMENT;
    if (num_q_heads % kv->num_kv_heads) return SA_ERR_UNSUPPORTED;
    const int hpg = num_q_heads / kv->num_kv_heads;
    if (hpg != 1 && hpg != 2 && hpg != 4 && hpg != 8) return SA_ERR_UNSUPPORTED;
    if (kv->batch > 0 && (!q || !idx_out || !count_out)) return SA_ERR_INVALID_ARGUMENT;
    if (!aligned(q, 16) || !aligned(idx_out, 4) || !aligned(count_out, 4)) return SA_ERR_INVALID_ARGUMENT;
    // the selection keeps two bitmaps of the context in shared memory
    if ((long long)kv->max_pages_per_seq * kv->page_size > (1LL << 19)) return SA_ERR_UNSUPPORTED;
    st = check_ws(ws, ws_bytes, ws_topk(kv, num_q_heads));
    if (st != SA_OK) return st;
    a.q = q;
    a.q_f32 = q_dtype == SA_DTYPE_F32;
    a.Hq = num_q_heads;
    a.k = k;
    a.Lcap = kv->max_pages_per_seq * kv->page_size;
    a.scores = reinterpret_cast<float *>(static_cast<char *>(ws) + kHeader);
    a.idx = idx_out;
    a.cnt = count_out;
    a.st = static_cast<DevStatus *>(ws);
    return cuda_status(launch_topk(a, (cudaStream_t)stream));
}

sa_status sa_sparse_decode_attn(const sa_kv_cache *kv, const void *q, sa_dtype q_dtype,
                                int32_t num_q_heads, const sa_selection *sel, float scale,
                                int32_t num_splits, void *out, float *lse_out, void *ws,
                                size_t ws_bytes, sa_stream_t stream)
{
    DecodeArgs a{};
    sa_status st = check_cache(kv, &a.c);
    if (st != SA_OK) return st;
    if (num_q_heads <= 0 || !sel || num_splits < 1 || num_splits > 64) return SA_ERR_INVALID_ARGUMENT;
    if (q_dtype != SA_DTYPE_F32 && q_dtype != SA_DTYPE_BF16) return SA_ERR_INVALID_ARGUMENT;
    if (num_q_heads % kv->num_kv_heads) return SA_ERR_UNSUPPORTED;
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY) return SA_ERR_INVALID_ARGUMENT;
    if (kv->batch > 0 && (!q || !out)) return SA_ERR_INVALID_ARGUMENT;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(lse_out, 4)) return SA_ERR_INVALID_ARGUMENT;
    if (sel->kind == SA_SEL_TOKENS) {
        if (sel->k_cap < 0 || (kv->batch > 0 && sel->k_cap > 0 && (!sel->idx || !sel->count)))
            return SA_ERR_INVALID_ARGUMENT;
        if (kv->batch > 0 && !sel->count) return SA_ERR_INVALID_ARGUMENT;
    } else if (sel->kind == SA_SEL_BLOCKS) {
        if (sel->max_blocks < 0 || (kv->batch > 0 && (!sel->block_counts || (sel->max_blocks > 0 && !sel->blocks))))
            return SA_ERR_INVALID_ARGUMENT;
        if (!aligned(sel->blocks, 16)) return SA_ERR_INVALID_ARGUMENT;
    } else {
        return SA_ERR_INVALID_ARGUMENT;
    }
    st = check_ws(ws, ws_bytes, ws_decode(kv, num_q_heads, num_splits));
    if (st != SA_OK) return st;
    char *w = static_cast<char *>(ws);
    const size_t rows = (size_t)kv->batch * num_q_heads;
    a.q = q;
    a.q_f32 = q_dtype == SA_DTYPE_F32;
    a.Hq = num_q_heads;
    a.qscale = scale * kLog2e;
    a.blocks = sel->kind == SA_SEL_BLOCKS;
    a.idx = sel->idx;
    a.cnt = sel->count;
    a.kcap = sel->k_cap;
    a.ent = sel->blocks;
    a.ecnt = sel->block_counts;
    a.max_blocks = sel->max_blocks;
    a.S = num_splits;
    a.part_o = reinterpret_cast<float *>(w + kHeader);
    a.part_ml = reinterpret_cast<float *>(w + kHeader + up(rows * num_splits * kv->head_dim * sizeof(float)));
    a.out = static_cast<uint16_t *>(out);
    a.lse = lse_out;
    a.st = static_cast<DevStatus *>(ws);
    return cuda_status(launch_decode(a, (cudaStream_t)stream));
}

sa_status sa_select_blocks(const sa_kv_cache *kv, const sa_block_select_args *args, sa_block_list *out,
                           void *ws, size_t ws_bytes, sa_stream_t stream)
{
    CacheArgs c{};
    sa_status st = check_cache(kv, &c);
    if (st != SA_OK) return st;
    if (!args || !out) return SA_ERR_INVALID_ARGUMENT;
    if (args->mode == SA_SEL_SPANS) {
        if (args->max_spans < 0 || args->max_spans > 1024 || out->max_blocks < 0) return SA_ERR_INVALID_ARGUMENT;
        if (kv->batch > 0 && (!args->span_counts || !out->block_counts)) return SA_ERR_INVALID_ARGUMENT;
        if (kv->batch > 0 && args->max_spans > 0 && (!args->spans || !args->span_round))
            return SA_ERR_INVALID_ARGUMENT;
        if (kv->batch > 0 && out->max_blocks > 0 && !out->blocks) return SA_ERR_INVALID_ARGUMENT;
        if (!aligned(out->blocks, 16)) return SA_ERR_INVALID_ARGUMENT;
        st = check_ws(ws, ws_bytes, ws_blocks(kv, args));
        if (st != SA_OK) return st;
        SpanArgs a{};
        a.c = c;
        a.spans = args->spans;
        a.span_counts = args->span_counts;
        a.span_round = args->span_round;
        a.max_spans = args->max_spans;
        a.ent = out->blocks;
        a.ecnt = out->block_counts;
        a.max_blocks = out->max_blocks;
        a.st = static_cast<DevStatus *>(ws);
        return cuda_status(launch_spans(a, (cudaStream_t)stream));
    }
    if (args->mode != SA_SEL_RBS) return SA_ERR_INVALID_ARGUMENT;
    // RBS
    const int Hq = args->num_q_heads, T = args->num_tokens, bs = args->block_size;
    if (Hq <= 0 || T <= 0 || bs <= 0) return SA_ERR_INVALID_ARGUMENT;
    if (bs != 64) return SA_ERR_UNSUPPORTED;
    if (Hq % kv->num_kv_heads) return SA_ERR_UNSUPPORTED;
    if (kv->batch < 1) return SA_ERR_INVALID_ARGUMENT;
    if ((long long)T > (long long)kv->max_pages_per_seq * kv->page_size) return SA_ERR_INVALID_ARGUMENT;
    if (!args->q || !aligned(args->q, 16)) return SA_ERR_INVALID_ARGUMENT;
    if ((args->tau_c == nullptr) != (args->tau_r == nullptr)) return SA_ERR_INVALID_ARGUMENT;
    if (!args->tau_c && !(args->p_c >= 0.f && args->p_c <= 1.f && args->p_r >= 0.f && args->p_r <= 1.f))
        return SA_ERR_INVALID_ARGUMENT;
    if (!(args->scale > 0.f) || args->scale == INFINITY) return SA_ERR_INVALID_ARGUMENT;
    if (!out->row_ptr || !out->cols || out->nnz_capacity < 0) return SA_ERR_INVALID_ARGUMENT;
    const int nB = (T + bs - 1) / bs;
    if (nB > 65536) return SA_ERR_UNSUPPORTED;
    st = check_ws(ws, ws_bytes, ws_blocks(kv, args));
    if (st != SA_OK) return st;
    size_t offs[16];
    const bool quant = args->tau_c == nullptr;
    rbs_workspace_layout(Hq, kv->num_kv_heads, kv->head_dim, nB, quant, offs);
    char *w = static_cast<char *>(ws) + kHeader;
    RbsArgs a{};
    a.c = c;
    a.q = static_cast<const uint16_t *>(args->q);
    a.Hq = Hq;
    a.T = T;
    a.bs = bs;
    a.nB = nB;
    a.scale = args->scale;
    a.tau_c = args->tau_c;
    a.tau_r = args->tau_r;
    a.p_c = args->p_c;
    a.p_r = args->p_r;
    a.force_diag = args->force_diag;
    a.force_first = args->force_first;
    a.cen = reinterpret_cast<uint8_t *>(w + offs[0]);
    a.rad = reinterpret_cast<float *>(w + offs[1]);
    a.qbar = reinterpret_cast<uint8_t *>(w + offs[2]);
    a.qnorm = reinterpret_cast<float *>(w + offs[3]);
    a.tau = reinterpret_cast<float *>(w + offs[4]);
    a.bits = reinterpret_cast<uint32_t *>(w + offs[5]);
    a.rowcnt = reinterpret_cast<int32_t *>(w + offs[6]);
    a.pair_sc = quant ? reinterpret_cast<float *>(w + offs[7]) : nullptr;
    a.qhist = quant ? reinterpret_cast<uint32_t *>(w + offs[8]) : nullptr;
    a.row_ptr = out->row_ptr;
    a.cols = out->cols;
    a.nnz_cap = out->nnz_capacity;
    a.tau_out = out->tau_out;
    a.st = static_cast<DevStatus *>(ws);
    cudaError_t e = launch_rbs(a, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return SA_ERR_UNSUPPORTED;
    return cuda_status(e);
}

sa_status sa_sparse_prefill_attn(const sa_kv_cache *kv, const void *q, int32_t num_q_heads,
                                 int32_t num_tokens, const sa_block_list *csr, float scale,
                                 int32_t causal, void *out, float *lse_out, void *ws, size_t ws_bytes,
                                 sa_stream_t stream)
{
    PrefillArgs a{};
    sa_status st = check_cache(kv, &a.c);
    if (st != SA_OK) return st;
    if (num_q_heads <= 0 || num_tokens < 0) return SA_ERR_INVALID_ARGUMENT;
    if (causal != 1) return SA_ERR_UNSUPPORTED;
    if (kv->head_dim != 128 || kv->page_size != 64) return SA_ERR_UNSUPPORTED;
    if (num_q_heads % kv->num_kv_heads) return SA_ERR_UNSUPPORTED;
    if (kv->batch < 1) return SA_ERR_INVALID_ARGUMENT;
    if ((long long)num_tokens > (long long)kv->max_pages_per_seq * kv->page_size) return SA_ERR_INVALID_ARGUMENT;
    if (!(scale == scale)) return SA_ERR_INVALID_ARGUMENT;
    if (num_tokens > 0 && (!q || !csr || !csr->row_ptr || !csr->cols || !out)) return SA_ERR_INVALID_ARGUMENT;
    if (csr && csr->nnz_capacity < 0) return SA_ERR_INVALID_ARGUMENT;
    if ((long long)kv->num_pages * kv->num_kv_heads * 64 >= (1LL << 31)) return SA_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(lse_out, 4)) return SA_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.f) || scale == INFINITY) return SA_ERR_INVALID_ARGUMENT;
    st = check_ws(ws, ws_bytes, ws_prefill(kv, num_q_heads, num_tokens));
    if (st != SA_OK) return st;
    a.q = static_cast<const uint16_t *>(q);
    a.Hq = num_q_heads;
    a.T = num_tokens;
    a.scale = scale;
    if (num_tokens == 0) return SA_OK;
    a.row_ptr = csr->row_ptr;
    a.cols = csr->cols;
    a.nnz_cap = csr->nnz_capacity;
    a.out = static_cast<uint16_t *>(out);
    a.lse = lse_out;
    a.items = reinterpret_cast<int4 *>(static_cast<char *>(ws) + kHeader);
    a.n_items = prefill_items(num_q_heads, kv->num_kv_heads, (num_tokens + 63) / 64);
    a.st = static_cast<DevStatus *>(ws);
    if (num_tokens == 0) return SA_OK;
    cudaError_t e = launch_prefill(a, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return SA_ERR_UNSUPPORTED;
    return cuda_status(e);
}

}  // extern "C"
