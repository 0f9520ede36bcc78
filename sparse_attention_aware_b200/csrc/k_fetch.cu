// Page fetch from a host memory tier into device KV page slots.
//
// Method: the KV pages a DA step does not read stay valid, so they can live
// in an outer tier and return when a declaration names them again, loaded
// alongside decoding ("语言模型能自己决定该看哪里吗？", on moving ignored KV
// to outer memory; "百万上下文，模型终于会挑重点了", "对百万上下文产品意味着
// 什么": tiered KV storage).
//
// k_fetch_pages: grid (pairs, 2 [K, V], chunks of 64 KB); each thread issues
// its 16-byte loads from pinned host memory (device-readable at the host
// address under unified addressing) before any store, so a CTA keeps up to
// 64 KB of host-link reads in flight.  Bad pairs are skipped and recorded.
#include "sa_internal.h"

namespace sa {
namespace {

constexpr int kFetchThreads = 256;
constexpr int kFetchPer = 16;                                   // 16-byte words per thread per chunk
constexpr size_t kFetchChunk = (size_t)kFetchThreads * kFetchPer * 16;   // 64 KB

__global__ void __launch_bounds__(kFetchThreads) k_fetch_pages(const FetchArgs a)
{
    pdl_wait();
    pdl_trigger();
    const int i = blockIdx.x;
    const int2 pr = reinterpret_cast<const int2 *>(a.pairs)[i];
    if (pr.x < 0 || pr.x >= a.host_pages || pr.y < 0 || pr.y >= a.dev_pages) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
            fault(a.st, CHK_PAGE, pr.x < 0 || pr.x >= a.host_pages ? pr.x : pr.y);
        return;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(
        static_cast<const char *>(blockIdx.y == 0 ? a.host_k : a.host_v) + (size_t)pr.x * a.page_bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<char *>(blockIdx.y == 0 ? a.dev_k : a.dev_v) +
                                           (size_t)pr.y * a.page_bytes);
    const size_t words = a.page_bytes / 16;
    const size_t w0 = (size_t)blockIdx.z * (kFetchChunk / 16);
    uint4 v[kFetchPer];
#pragma unroll
    for (int u = 0; u < kFetchPer; ++u) {
        const size_t w = w0 + (size_t)u * kFetchThreads + threadIdx.x;
        if (w < words) v[u] = src[w];
    }
#pragma unroll
    for (int u = 0; u < kFetchPer; ++u) {
        const size_t w = w0 + (size_t)u * kFetchThreads + threadIdx.x;
        if (w < words) dst[w] = v[u];
    }
}

}  // namespace

cudaError_t launch_fetch(const FetchArgs &a, cudaStream_t s)
{
    if (a.n == 0) return cudaSuccess;
    const unsigned chunks = (unsigned)((a.page_bytes + kFetchChunk - 1) / kFetchChunk);
    if (cudaError_t e = launch_pdl(k_fetch_pages, dim3((unsigned)a.n, 2, chunks), dim3(kFetchThreads), 0, s, a))
        return e;
    return cudaGetLastError();
}

}  // namespace sa
