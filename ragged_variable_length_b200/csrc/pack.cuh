// Pack, scatter-back and CLS-extraction kernels.
//
// Pack ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// radpulse article, section "Integrated pack pipeline": cu_seqlens first,
// then a coalesced copy of the survivors into one contiguous flat buffer) is a
// single launch with no inter-CTA communication:
//   grid = (splits, B); CTA (s, b) handles a contiguous slice of image b's
//   survivors.  Every CTA
//     1. counts the kept tokens of images 0..b-1 itself (16-byte mask loads,
//        byte-wise compare-and-popcount), which gives cu[b] without a
//        separate scan launch or a device-wide wait;
//     2. ranks image b's survivors with one warp ballot/popcount scan per 256
//        mask bytes, building the list of kept token indices in shared memory;
//     3. copies its slice of rows as 16-byte vectors, all threads striding
//        over (row, vector) pairs so that every row length keeps all lanes busy.
//   The dense rows are read with streaming (evict-first) loads; the packed
//   rows are stored normally so that the attention launch that follows finds
//   them in L2.
#pragma once

#include "common.cuh"

namespace ragged {

constexpr int kPackThreads = 256;
constexpr int kPackUnroll = 4;

__device__ __forceinline__ int nonzero_bytes(uint32_t w) { return __popc(__vcmpne4(w, 0u)) >> 3; }

// Nonzero bytes in p[0, n) plus every thread's `extra`, summed over the CTA
// of NT threads (result in every thread).  s_red holds NT / 32 ints.
template <int NT>
__device__ __forceinline__ int cta_count_nonzero(const uint8_t* __restrict__ p, int64_t n,
                                                 int extra, int* s_red) {
    const int tid = threadIdx.x;
    int cnt = extra;
    int64_t head = (16 - (reinterpret_cast<uintptr_t>(p) & 15)) & 15;
    if (head > n) head = n;
    for (int64_t i = tid; i < head; i += NT) cnt += p[i] != 0;
    const uint4* v = reinterpret_cast<const uint4*>(p + head);
    const int64_t nv = (n - head) >> 4;
    for (int64_t i = tid; i < nv; i += NT) {
        const uint4 x = __ldg(v + i);
        cnt += nonzero_bytes(x.x) + nonzero_bytes(x.y) + nonzero_bytes(x.z) + nonzero_bytes(x.w);
    }
    for (int64_t i = head + nv * 16 + tid; i < n; i += NT) cnt += p[i] != 0;
    cnt = warp_sum(cnt);
    if ((tid & 31) == 0) s_red[tid >> 5] = cnt;
    __syncthreads();
    int total = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) total += s_red[w];
    __syncthreads();
    return total;
}

// Ranks the survivors of one image with a CTA of NT threads: s_kept[r] =
// token index of the r-th survivor (CLS at r = 0).  Returns the survivor
// count L_b (in every thread).
template <int NT>
__device__ __forceinline__ int cta_rank_survivors(const uint8_t* __restrict__ kb, int L_full,
                                                  int* s_kept, int* s_red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int running = 0;
    for (int j0 = 0; j0 < L_full; j0 += NT) {
        const int j = j0 + tid;
        const bool kept = j < L_full && (j == 0 || kb[j] != 0);
        const unsigned bal = __ballot_sync(0xffffffffu, kept);
        if (lane == 0) s_red[warp] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) {
            const int x = s_red[w];
            before += (w < warp) ? x : 0;
            total += x;
        }
        if (kept) s_kept[running + before + __popc(bal & ((1u << lane) - 1u))] = j;
        running += total;
        __syncthreads();
    }
    return running;
}

// Copies rows r in [r0, r1) between the flat row flat_row0 + r and the listed
// row list_row0 + s_kept[r].
// GATHER: the source row is listed (dense) and the destination is flat
// (packed); otherwise the other way round.
template <bool GATHER>
__device__ __forceinline__ void cta_copy_rows(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                              const int* s_kept, int r0, int r1, int64_t list_row0,
                                              int64_t flat_row0, uint32_t nvec) {
    const uint32_t total = static_cast<uint32_t>(r1 - r0) * nvec;
    for (uint32_t i0 = threadIdx.x; i0 < total; i0 += kPackThreads * kPackUnroll) {
        uint4 buf[kPackUnroll];
        int64_t dst_off[kPackUnroll];
#pragma unroll
        for (int u = 0; u < kPackUnroll; ++u) {
            const uint32_t i = i0 + u * kPackThreads;
            if (i < total) {
                const uint32_t r = i / nvec;
                const uint32_t v = i - r * nvec;
                const int64_t listed = (list_row0 + s_kept[r0 + r]) * nvec + v;
                const int64_t flat = (flat_row0 + r0 + r) * nvec + v;
                const int64_t src_off = GATHER ? listed : flat;
                dst_off[u] = GATHER ? flat : listed;
                buf[u] = __ldcs(src + src_off);
            }
        }
#pragma unroll
        for (int u = 0; u < kPackUnroll; ++u) {
            const uint32_t i = i0 + u * kPackThreads;
            if (i < total) dst[dst_off[u]] = buf[u];
        }
    }
}

__global__ void __launch_bounds__(kPackThreads)
    pack_kernel(const uint4* __restrict__ dense, int L_full, uint32_t nvec,
                const uint8_t* __restrict__ keep, uint4* __restrict__ packed,
                int32_t* __restrict__ cu, int32_t* __restrict__ src_idx) {
    extern __shared__ int s_kept[];
    __shared__ int s_red[kPackThreads / 32];
    const int b = blockIdx.y;
    const int split = blockIdx.x, splits = gridDim.x;

    // cu[b]: survivors of the images before this one.  CLS is kept even when
    // its mask byte is zero, so each such image adds one.
    const int64_t prev = static_cast<int64_t>(b) * L_full;
    int forced = 0;
    for (int i = threadIdx.x; i < b; i += kPackThreads)
        forced += keep[static_cast<int64_t>(i) * L_full] == 0;
    const int base = cta_count_nonzero<kPackThreads>(keep, prev, forced, s_red);

    const int L_b = cta_rank_survivors<kPackThreads>(keep + prev, L_full, s_kept, s_red);
    if (split == 0 && threadIdx.x == 0) {
        cu[b + 1] = base + L_b;
        if (b == 0) cu[0] = 0;
    }
    const int r0 = static_cast<int>(static_cast<int64_t>(L_b) * split / splits);
    const int r1 = static_cast<int>(static_cast<int64_t>(L_b) * (split + 1) / splits);
    if (src_idx != nullptr)
        for (int r = r0 + threadIdx.x; r < r1; r += kPackThreads)
            src_idx[base + r] = static_cast<int32_t>(prev + s_kept[r]);
    cta_copy_rows<true>(dense, packed, s_kept, r0, r1, prev, base, nvec);
}

// Scatter back: dense_out[b, kept j] <- packed[cu[b] + rank(j)].
__global__ void __launch_bounds__(kPackThreads)
    unpack_kernel(const uint4* __restrict__ packed, const int32_t* __restrict__ cu, int L_full,
                  uint32_t nvec, const uint8_t* __restrict__ keep, uint4* __restrict__ dense_out) {
    extern __shared__ int s_kept[];
    __shared__ int s_red[kPackThreads / 32];
    const int b = blockIdx.y;
    const int split = blockIdx.x, splits = gridDim.x;
    const int64_t prev = static_cast<int64_t>(b) * L_full;
    const int L_b = cta_rank_survivors<kPackThreads>(keep + prev, L_full, s_kept, s_red);
    const int base = __ldg(cu + b);
    if (base < 0 || __ldg(cu + b + 1) - base != L_b) {
        if (threadIdx.x == 0) raise_status(RAGGED_DEV_BAD_SEQLENS);
        return;
    }
    const int r0 = static_cast<int>(static_cast<int64_t>(L_b) * split / splits);
    const int r1 = static_cast<int>(static_cast<int64_t>(L_b) * (split + 1) / splits);
    cta_copy_rows<false>(packed, dense_out, s_kept, r0, r1, prev, base, nvec);
}

// cls_out[b] <- packed[cu[b]]; one thread per 16-byte vector.
__global__ void __launch_bounds__(256)
    unpack_cls_kernel(const uint4* __restrict__ packed, const int32_t* __restrict__ cu, int B,
                      uint32_t nvec, uint4* __restrict__ cls_out) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<int64_t>(B) * nvec) return;
    const int b = static_cast<int>(i / nvec);
    const uint32_t v = static_cast<uint32_t>(i - static_cast<int64_t>(b) * nvec);
    const int row = __ldg(cu + b);
    if (row < 0 || __ldg(cu + b + 1) <= row) {
        if (v == 0) raise_status(RAGGED_DEV_BAD_SEQLENS);
        return;
    }
    cls_out[i] = packed[static_cast<int64_t>(row) * nvec + v];
}

}  // namespace ragged
