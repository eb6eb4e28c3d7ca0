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
// cu[b] is the sum of the earlier k_b, and each CTA sorts its image's scores
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
constexpr int kMaskMaxImages = 65535;   // images per launch (grid y)

// keep[b * L_full + j] for the tokens j of the images b = blockIdx.y (one warp
// per token, blockIdx.x covering 8 tokens of the image); token (b, j) is the C
// elements from element (b * L_full + j) * tok_stride.  The sum of squares is
// formed in fp64 in a fixed order, so that the keep decision at the threshold
// is reproducible: lane l adds the squares of elements l, l + 32, l + 64, ...
// in turn (every square of an f16, bf16 or f32 element is exact in fp64), then
// the 32 partial sums are combined pairwise with xor-shuffles 16, 8, 4, 2, 1.
// Explicit round-to-nearest intrinsics keep the compiler from contracting the
// multiply-add.
template <typename T>
__global__ void __launch_bounds__(kMaskThreads)
    mask_l2_kernel(const void* __restrict__ x, int L_full, int C, int64_t tok_stride, double tau,
                   uint8_t* __restrict__ keep) {
    const int j = blockIdx.x * (kMaskThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (j >= L_full) return;   // warp-uniform
    const int64_t t = static_cast<int64_t>(blockIdx.y) * L_full + j;
    const int64_t base = t * tok_stride;
    double ss = 0.0;
    for (int c = lane; c < C; c += 32) {
        const double v = widen<T>(x, base + c);
        ss = __dadd_rn(ss, __dmul_rn(v, v));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
    if (lane == 0) keep[t] = (j == 0 || __dsqrt_rn(ss) >= tau) ? 1 : 0;
}

// The top-k order as one unsigned key per token, larger key = ranks earlier:
// the high word maps the score's bits so that unsigned order is float order
// (-0 folded onto +0, so the two zeros tie) and sends NaN, of any payload, to 0
// below -inf; the low word is ~j, so equal scores go to the lower index.  Keys
// of distinct tokens differ, and every token j < 2^31 has a key above 0.
// Integer operations only, so no flush-to-zero setting can merge scores.
__device__ __forceinline__ uint64_t topk_key(float score, int j) {
    uint32_t bits = __float_as_uint(score);
    const uint32_t mag = bits & 0x7fffffffu;
    uint32_t hi;
    if (mag > 0x7f800000u) {
        hi = 0u;                                    // NaN
    } else {
        if (mag == 0u) bits = 0u;                   // -0 -> +0
        hi = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
    }
    return (static_cast<uint64_t>(hi) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(j));
}

__device__ __forceinline__ int clamp_count(int k, int L_full) { return k < 1 ? 1 : (k > L_full ? L_full : k); }

__host__ __device__ constexpr int topk_pow2(int n) {
    int p = 2;
    while (p < n) p <<= 1;
    return p;
}

// grid = (splits, B).  Dynamic shared memory: P = topk_pow2(L_full) 8-byte
// keys, then L_full ints of survivor list.  Each CTA sorts image b's keys in
// descending order (bitonic network over P slots; CLS and the padding slots
// hold key 0, which every other token's key exceeds), so the (k_b - 1)-th
// largest key is the cut: a non-CLS token is kept when its key is at least
// that.  The survivor list is then built in token order with the ballot scan
// of pack, and the CTA copies its slice of rows.  Split 0 also writes
// cu[b + 1] and, when asked, the keep row.
__global__ void __launch_bounds__(kPackThreads)
    pack_topk_kernel(const uint4* __restrict__ dense, int L_full, uint32_t nvec, const float* __restrict__ scores,
                     const int32_t* __restrict__ keep_count, uint4* __restrict__ packed, int32_t* __restrict__ cu,
                     int32_t* __restrict__ src_idx, uint8_t* __restrict__ keep_out) {
    extern __shared__ uint64_t smem_k[];
    const int P = topk_pow2(L_full);
    uint64_t* s_key = smem_k;
    int* s_kept = reinterpret_cast<int*>(smem_k + P);
    __shared__ int s_red[kPackThreads / 32];
    const int b = blockIdx.y;
    const int split = blockIdx.x, splits = gridDim.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // cu[b]: the clamped counts of the images before this one.
    int part = 0;
    for (int i = tid; i < b; i += kPackThreads) part += clamp_count(__ldg(keep_count + i), L_full);
    part = warp_sum(part);
    if (lane == 0) s_red[warp] = part;
    const int k = clamp_count(__ldg(keep_count + b), L_full);
    const int64_t row0 = static_cast<int64_t>(b) * L_full;

    // Bitonic sort, descending: in the merge of blocks of `size`, pairs
    // (lo, lo + stride) are ordered descending where lo & size is 0, else
    // ascending; the last merge (size = P) is descending throughout.
    if (P <= kPackThreads) {
        // One key per thread (slot tid).  A slot's partner is tid ^ stride, in
        // the same block of `size` <= P, so slots below P only ever meet
        // slots below P; the slots from P up hold keys nobody reads.  Strides
        // below 32 pair lanes of one warp (a shuffle, no barrier); the others
        // exchange through shared memory.
        uint64_t key = (tid > 0 && tid < L_full) ? topk_key(__ldg(scores + row0 + tid), tid) : 0ull;
        for (int size = 2; size <= P; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                uint64_t other;
                if (stride >= 32) {
                    if (tid < P) s_key[tid] = key;
                    __syncthreads();
                    other = tid < P ? s_key[tid ^ stride] : key;
                    __syncthreads();
                } else {
                    other = __shfl_xor_sync(0xffffffffu, key, stride);
                }
                const bool desc = (tid & size) == 0, lower = (tid & stride) == 0;
                key = (lower == desc) ? (key > other ? key : other) : (key < other ? key : other);
            }
        }
        if (tid < P) s_key[tid] = key;
        __syncthreads();
    } else {
        for (int j = tid; j < P; j += kPackThreads)
            s_key[j] = (j > 0 && j < L_full) ? topk_key(__ldg(scores + row0 + j), j) : 0ull;
        __syncthreads();
        for (int size = 2; size <= P; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int t = tid; t < P / 2; t += kPackThreads) {
                    const int lo = 2 * t - (t & (stride - 1));
                    const int hi = lo + stride;
                    const uint64_t a = s_key[lo], c = s_key[hi];
                    const bool desc = (lo & size) == 0;
                    if ((a < c) == desc) {
                        s_key[lo] = c;
                        s_key[hi] = a;
                    }
                }
                __syncthreads();
            }
        }
    }
    int base = 0;
#pragma unroll
    for (int w = 0; w < kPackThreads / 32; ++w) base += s_red[w];
    // k >= 2: the (k - 1)-th largest non-CLS key; k == 1: nothing beside CLS.
    const uint64_t cut = k >= 2 ? s_key[k - 2] : ~0ull;

    // Survivors in token order (CLS first).
    int running = 0;
    for (int j0 = 0; j0 < L_full; j0 += kPackThreads) {
        const int j = j0 + tid;
        bool kept = false;
        if (j == 0)
            kept = true;
        else if (j < L_full)
            kept = topk_key(__ldg(scores + row0 + j), j) >= cut;
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
