// sa_sparse_decode_attn_noalloc: split-KV sparse decode for callers that
// cannot allocate device memory.
//
// Its scratch (the split-KV partial states and a status header) lives in a
// file-scope device array of fixed size, compiled into the library.  Host code
// never passes the array's name to a kernel (in host code it only stands in
// for the symbol); the device address is looked up once per device with
// cudaGetSymbolAddress and handed to the same decode kernels the workspace
// entry point launches.
#include <cuda_runtime.h>
#include <mutex>

#include "sa.h"
#include "sa_internal.h"

using namespace sa;

namespace {

constexpr size_t kNoAllocBytes = SA_NOALLOC_DECODE_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

// Every GPU that loads libsa holds this array until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (set up on the
// first call per device).
sa_status scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return SA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SA_OK;
}

}  // namespace

extern "C" sa_status sa_sparse_decode_attn_noalloc(const sa_kv_cache *kv, const void *q, sa_dtype q_dtype,
                                                   int32_t num_q_heads, const sa_selection *sel, float scale,
                                                   int32_t num_splits, void *out, float *lse_out,
                                                   sa_stream_t stream)
{
    // argument checks: identical rules to sa_sparse_decode_attn, run first
    if (!kv || !sel) return SA_ERR_INVALID_ARGUMENT;
    if (kv->batch < 0 || kv->num_kv_heads <= 0 || kv->head_dim <= 0 || kv->page_size <= 0 ||
        kv->max_pages_per_seq < 0 || kv->num_pages < 0)
        return SA_ERR_INVALID_ARGUMENT;
    if (kv->head_dim != 64 && kv->head_dim != 128) return SA_ERR_UNSUPPORTED;
    if (kv->page_size != 16 && kv->page_size != 64) return SA_ERR_UNSUPPORTED;
    if (num_q_heads <= 0 || num_splits < 1 || num_splits > 64) return SA_ERR_INVALID_ARGUMENT;
    if (num_q_heads % kv->num_kv_heads) return SA_ERR_UNSUPPORTED;
    // the same layout the workspace entry point carves out of its workspace
    if (decode_workspace_bytes(kv, num_q_heads, num_splits) > kNoAllocBytes)
        return SA_ERR_UNSUPPORTED;   // beyond the built-in scratch
    void *base = nullptr;
    sa_status st = scratch_address(&base);
    if (st != SA_OK) return st;
    // the workspace entry point does the remaining checks and the launches,
    // with the static scratch standing in for the caller's workspace
    return sa_sparse_decode_attn(kv, q, q_dtype, num_q_heads, sel, scale, num_splits, out, lse_out, base,
                                 kNoAllocBytes, stream);
}
