// Shared device helpers of the ragged pipeline kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ragged.h"

namespace ragged {

// Per-device status word; bits are RAGGED_DEV_* from ragged.h.  Kernels only
// OR bits in; ragged_get_device_status reads and clears it.
__device__ unsigned int g_dev_status;

__device__ __forceinline__ void raise_status(unsigned int bits) { atomicOr(&g_dev_status, bits); }

// Reads cu[b], cu[b+1] and checks them against the host bound.  Returns false
// (and flags the status word) when the sequence must be skipped.
__device__ __forceinline__ bool read_sequence(const int32_t* __restrict__ cu, int b, int max_seqlen,
                                              int& start, int& len) {
    start = __ldg(cu + b);
    const int end = __ldg(cu + b + 1);
    len = end - start;
    if (start < 0 || len < 0 || len > max_seqlen) {
        raise_status(RAGGED_DEV_BAD_SEQLENS);
        return false;
    }
    return true;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy; src_bytes = 0 zero-fills the
// destination without reading the source.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ int warp_sum(int x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace ragged
