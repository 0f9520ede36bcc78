// Shared device helpers for libsa (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sa.h"

namespace sa {

// ---------------------------------------------------------------------------
// workspace header: status word recorded by kernels, read by
// sa_read_device_status().  The first 256 bytes of every workspace.
// ---------------------------------------------------------------------------
struct DevStatus {
    unsigned code;    // sa_status of the first recorded error (0 = none)
    unsigned detail;  // check id (enum Check)
    int value;        // offending value
    unsigned pad[61];
};
static_assert(sizeof(DevStatus) == 256, "status header is 256 bytes");

enum Check : unsigned {
    CHK_NONE = 0,
    CHK_SEQ_LEN = 1,        // seq_lens[b] outside [0, max_pages*P]
    CHK_PAGE = 2,           // page_table entry outside [0, num_pages)
    CHK_INDEX = 3,          // token index outside [0, L_b)
    CHK_COUNT = 4,          // count[b,h] outside [0, k_cap]
    CHK_BLOCK_ENTRY = 5,    // block-list entry malformed
    CHK_CSR = 6,            // CSR row_ptr / col malformed
    CHK_CAPACITY_CSR = 7,   // cols capacity exceeded
    CHK_CAPACITY_BLOCKS = 8,// block-list capacity exceeded
    CHK_SPAN = 9,           // span count outside [0, max_spans]
    CHK_TOPK_SCRATCH = 10,  // top-k candidate buffer overflow
    CHK_WAIT = 11           // bounded wait expired
};

__device__ __forceinline__ void record(DevStatus *st, sa_status code, unsigned chk, int value)
{
    if (atomicCAS(&st->code, 0u, (unsigned)code) == 0u) {
        st->detail = chk;
        st->value = value;
    }
}

__device__ __forceinline__ void fault(DevStatus *st, unsigned chk, int value)
{
    record(st, SA_ERR_DEVICE_FAULT, chk, value);
}

// ---------------------------------------------------------------------------
// numerics
// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation allowed (launch_pdl) and starts with
// pdl_wait(), which returns once the previous kernel in the stream has
// completed and its writes are visible (at once if it was launched without
// the attribute), and pdl_trigger(), which lets the next kernel's CTAs be
// scheduled while this one is still running.  So a dependent kernel's launch
// latency overlaps its predecessor's tail, and no kernel touches global
// memory before its predecessor is done.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// hardware base-2 exponential / logarithm (PTX ex2.approx / lg2.approx)
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// fp32 -> bf16 round to nearest even (finite inputs)
__device__ __forceinline__ uint16_t f2bf(float f)
{
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)((u >> 16) | ((u & 0xffff) ? 0x40 : 0));
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// ---------------------------------------------------------------------------
// memory
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg_nc_v4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ int ldg_i32(const int32_t *p) { return __ldg(p); }

// order-preserving map fp32 -> uint32 (larger float -> larger key)
__device__ __forceinline__ uint32_t f2key(float f)
{
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

}  // namespace sa
