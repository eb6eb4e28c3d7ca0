// Device-side keep-mask producers ("Dispatch-Aware Ragged Attention for Pruned
// Vision Transformers", radpulse article, section "Integrated pack pipeline":
// the pipeline is independent of the pruning method; Threshold-l2 is among the
// methods it names).  The pages give neither rule in detail; the readings:
//   Threshold-l2  token j of image b is kept when the Euclidean norm of its
//                 feature vector is at least tau;
//   top-k         image b keeps CLS and the k_b - 1 other tokens with the
//                 highest scores, ties going to the lower index and NaN
//                 ranking below every number; k_b is clamped to [1, L_full].
// CLS (index 0) is always kept.
//
// mask_l2_kernel writes a keep mask for ragged_pack.  pack_topk_kernel is the
// top-k selection fused into pack: since image b keeps exactly k_b tokens,
// cu[b] is the sum of the earlier k_b, and each CTA ranks its image's scores
// itself, so selection, cu_seqlens and the survivor copy are one launch.
#pragma once

#include "pack.cuh"

namespace ragged {

template <typename T>
__device__ __forceinline__ double widen(const void* p, int64_t i);
template <>
__device__ __forceinline__ double widen<__half>(const void* p, int64_t i) {
    return static_cast<double>(__half2float(static_cast<const __half*>(p)[i]));
}
template <>
__device__ __forceinline__ double widen<__nv_bfloat16>(const void* p, int64_t i) {
    return static_cast<double>(__bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]));
}
template <>
__device__ __forceinline__ double widen<float>(const void* p, int64_t i) {
    return static_cast<double>(static_cast<const float*>(p)[i]);
}

constexpr int kMaskThreads = 256;   // 8 tokens per CTA, one warp each

// keep[t] for the tokens t = 0 .. tokens - 1 (t = b * L_full + j) of x, token t
// being the C elements from element t * tok_stride.  The sum of squares is
// formed in fp64 in a fixed order, so that the keep decision at the threshold
// is reproducible: lane l adds the squares of elements l, l + 32, l + 64, ...
// in turn (every square of an f16, bf16 or f32 element is exact in fp64), then
// the 32 partial sums are combined pairwise with xor-shuffles 16, 8, 4, 2, 1.
// Explicit round-to-nearest intrinsics keep the compiler from contracting the
// multiply-add.
template <typename T>
__global__ void __launch_bounds__(kMaskThreads)
    mask_l2_kernel(const void* __restrict__ x, int64_t tokens, int L_full, int C, int64_t tok_stride, double tau,
                   uint8_t* __restrict__ keep) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (kMaskThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= tokens) return;   // warp-uniform
    const int64_t base = t * tok_stride;
    double ss = 0.0;
    for (int c = lane; c < C; c += 32) {
        const double v = widen<T>(x, base + c);
        ss = __dadd_rn(ss, __dmul_rn(v, v));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
    if (lane == 0) keep[t] = (t % L_full == 0 || __dsqrt_rn(ss) >= tau) ? 1 : 0;
}

// Does score a (token ia) rank before score b (token ib)?
__device__ __forceinline__ bool ranks_before(float a, int ia, float b, int ib) {
    const bool na = isnan(a), nb = isnan(b);
    if (na != nb) return nb;   // every number ranks before NaN
    if (!na && a != b) return a > b;
    return ia < ib;
}

__device__ __forceinline__ int clamp_count(int k, int L_full) { return k < 1 ? 1 : (k > L_full ? L_full : k); }

// grid = (splits, B).  Dynamic shared memory: L_full scores, then L_full ints
// of survivor list.  Each CTA ranks image b's non-CLS tokens against each other
// (O(L_full^2 / threads) comparisons; fine for ViT token counts), builds the
// survivor list in token order with the ballot scan of pack, and copies its
// slice of rows.  Split 0 also writes cu[b + 1] and, when asked, the keep row.
__global__ void __launch_bounds__(kPackThreads)
    pack_topk_kernel(const uint4* __restrict__ dense, int L_full, uint32_t nvec, const float* __restrict__ scores,
                     const int32_t* __restrict__ keep_count, uint4* __restrict__ packed, int32_t* __restrict__ cu,
                     int32_t* __restrict__ src_idx, uint8_t* __restrict__ keep_out) {
    extern __shared__ int smem_i[];
    float* s_score = reinterpret_cast<float*>(smem_i);
    int* s_kept = smem_i + L_full;
    __shared__ int s_red[kPackThreads / 32];
    const int b = blockIdx.y;
    const int split = blockIdx.x, splits = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // cu[b]: the clamped counts of the images before this one.
    int part = 0;
    for (int i = tid; i < b; i += kPackThreads) part += clamp_count(__ldg(keep_count + i), L_full);
    part = warp_sum(part);
    if (lane == 0) s_red[warp] = part;
    __syncthreads();
    int base = 0;
#pragma unroll
    for (int w = 0; w < kPackThreads / 32; ++w) base += s_red[w];
    const int k = clamp_count(__ldg(keep_count + b), L_full);
    const int64_t row0 = static_cast<int64_t>(b) * L_full;
    for (int j = tid; j < L_full; j += kPackThreads) s_score[j] = __ldg(scores + row0 + j);
    __syncthreads();

    // Token j (> 0) is kept when fewer than k - 1 other non-CLS tokens rank
    // before it; the survivors are listed in token order (CLS first).
    int running = 0;
    for (int j0 = 0; j0 < L_full; j0 += kPackThreads) {
        const int j = j0 + tid;
        bool kept = false;
        if (j == 0) {
            kept = true;
        } else if (j < L_full) {
            const float sj = s_score[j];
            int before = 0;
            for (int i = 1; i < L_full && before < k - 1; ++i) before += ranks_before(s_score[i], i, sj, j);
            kept = before < k - 1;
        }
        if (keep_out != nullptr && split == 0 && j < L_full) keep_out[row0 + j] = kept ? 1 : 0;
        const unsigned bal = __ballot_sync(0xffffffffu, kept);
        __syncthreads();   // s_red of the count above / the previous round is free
        if (lane == 0) s_red[warp] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kPackThreads / 32; ++w) {
            const int xw = s_red[w];
            before += (w < warp) ? xw : 0;
            total += xw;
        }
        if (kept) s_kept[running + before + __popc(bal & ((1u << lane) - 1u))] = j;
        running += total;
    }
    __syncthreads();
    // running == k: exactly the clamped count is selected.
    if (split == 0 && tid == 0) {
        cu[b + 1] = base + running;
        if (b == 0) cu[0] = 0;
    }
    const int r0 = static_cast<int>(static_cast<int64_t>(running) * split / splits);
    const int r1 = static_cast<int>(static_cast<int64_t>(running) * (split + 1) / splits);
    if (src_idx != nullptr)
        for (int r = r0 + tid; r < r1; r += kPackThreads) src_idx[base + r] = static_cast<int32_t>(row0 + s_kept[r]);
    cta_copy_rows<true>(dense, packed, s_kept, r0, r1, row0, base, nvec);
}

}  // namespace ragged
