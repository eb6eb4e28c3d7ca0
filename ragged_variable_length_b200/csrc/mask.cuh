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

#include <type_traits>

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

// ---- exact Threshold-l2 decision ------------------------------------------
//
// The keep bit is the exact comparison sum(x_c^2) >= tau^2 (tau > 0), so that
// no summation order or rounding decides it.  A token's sum is first formed in
// fp64 in whatever order the warp finds fast; every square of an f16, bf16 or
// f32 value is exact in fp64 and only the additions round, so for n <= 2^24 +
// 32 terms the sum is within a relative 2^-29 of the exact one.  Outside a
// relative band of 2^-26 around tau^2 that settles the bit.  Inside it (ties
// and near-ties only), one lane recomputes the sum exactly: every such value
// is an integer multiple of 2^-149, so the sum of squares is an integer number
// of units of 2^-298, below 2^578 units, held in 24 32-bit limbs, and tau^2 is
// compared with it in the same units.
constexpr int kL2Unit = 298;
constexpr int kL2Limbs = 24;

// |v| = m * 2^e with m odd; v a finite, nonzero, normal double.
__device__ __forceinline__ void l2_odd_parts(double v, uint64_t& m, int& e) {
    const uint64_t bits = static_cast<uint64_t>(__double_as_longlong(v)) & 0x7fffffffffffffffull;
    m = (bits & 0xfffffffffffffull) | (1ull << 52);
    e = static_cast<int>(bits >> 52) - 1075;
    const int tz = __ffsll(static_cast<long long>(m)) - 1;
    m >>= tz;
    e += tz;
}

// acc += v * 2^shift, 0 <= shift, the result within kL2Limbs limbs.
__device__ __noinline__ void l2_big_add(uint32_t* acc, unsigned __int128 v, int shift) {
    const int w = shift >> 5, off = shift & 31;
    uint32_t part[5];
    const unsigned __int128 lo = v << off;                          // bits 0..127 of v * 2^off
    const uint32_t top = off ? static_cast<uint32_t>(v >> (128 - off)) : 0u;   // bits 128..159
#pragma unroll
    for (int i = 0; i < 4; ++i) part[i] = static_cast<uint32_t>(lo >> (32 * i));
    part[4] = top;
    uint64_t carry = 0;
    for (int i = w; i < kL2Limbs; ++i) {
        const uint64_t sum = static_cast<uint64_t>(acc[i]) + (i - w < 5 ? part[i - w] : 0u) + carry;
        acc[i] = static_cast<uint32_t>(sum);
        carry = sum >> 32;
    }
}

// Exact: does sum over c of x[base + c]^2 reach tau^2?  (0 < tau < 2^141, the
// elements finite.)
template <typename T>
__device__ __noinline__ bool l2_exact_reaches(const void* x, int64_t base, int C, double tau) {
    uint32_t S[kL2Limbs], Tq[kL2Limbs];
    for (int i = 0; i < kL2Limbs; ++i) S[i] = Tq[i] = 0u;
    for (int c = 0; c < C; ++c) {
        const double v = widen<T>(x, base + c);
        if (v == 0.0) continue;
        uint64_t m;
        int e;
        l2_odd_parts(v, m, e);   // m < 2^24, e >= -149 for every f32 value
        l2_big_add(S, static_cast<unsigned __int128>(m * m), 2 * e + kL2Unit);
    }
    uint64_t M;
    int E;
    l2_odd_parts(tau, M, E);
    const unsigned __int128 M2 = static_cast<unsigned __int128>(M) * M;   // < 2^106
    const int shift = 2 * E + kL2Unit;
    if (shift >= 0) {
        int bits = 0;
        for (unsigned __int128 r = M2; r != 0; r >>= 1) ++bits;
        if (bits + shift > 32 * kL2Limbs) return false;
        l2_big_add(Tq, M2, shift);
    } else {
        const int c = -shift;   // S is whole units: S >= M2 / 2^c  <=>  S >= ceil(M2 / 2^c)
        const unsigned __int128 q =
            c >= 128 ? static_cast<unsigned __int128>(1)
                     : (M2 >> c) + ((M2 & ((static_cast<unsigned __int128>(1) << c) - 1)) != 0);
        l2_big_add(Tq, q, 0);
    }
    for (int i = kL2Limbs - 1; i >= 0; --i)
        if (S[i] != Tq[i]) return S[i] > Tq[i];
    return true;
}

// keep[b * L_full + j] for the tokens j of the images b = blockIdx.y (one warp
// per token, blockIdx.x covering 8 tokens of the image); token (b, j) is the C
// elements from element (b * L_full + j) * tok_stride.  Kept: CLS; a token
// whose norm is infinite; otherwise, without a NaN element, sum x^2 >= tau^2
// exactly (every token when tau <= 0).
template <typename T>
__global__ void __launch_bounds__(kMaskThreads)
    mask_l2_kernel(const void* __restrict__ x, int L_full, int C, int64_t tok_stride, double tau,
                   uint8_t* __restrict__ keep) {
    const int j = blockIdx.x * (kMaskThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (j >= L_full) return;   // warp-uniform
    const int64_t t = static_cast<int64_t>(blockIdx.y) * L_full + j;
    const int64_t base = t * tok_stride;
    double s0 = 0.0, s1 = 0.0;
    int c = lane;
    for (; c + 32 < C; c += 64) {
        const double v0 = widen<T>(x, base + c), v1 = widen<T>(x, base + c + 32);
        s0 = __dadd_rn(s0, __dmul_rn(v0, v0));
        s1 = __dadd_rn(s1, __dmul_rn(v1, v1));
    }
    if (c < C) {
        const double v0 = widen<T>(x, base + c);
        s0 = __dadd_rn(s0, __dmul_rn(v0, v0));
    }
    double ss = __dadd_rn(s0, s1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
    // ss is the same in every lane: the decision below is warp-uniform.
    bool kept;
    if (j == 0) kept = true;
    else if (isnan(ss)) kept = false;                    // a NaN element
    else if (isinf(ss) || !(tau > 0.0)) kept = true;    // an infinite element (squares of finite values stay below 2^280)
    else if (tau > 0x1p+140) kept = false;               // tau^2 > 2^280 > any finite sum
    else if (tau < 0x1p-400) kept = ss > 0.0;            // tau^2 below the smallest nonzero square, 2^-298
    else {
        const double t2 = __dmul_rn(tau, tau);
        if (ss > __dmul_rn(t2, 1.0 + 0x1p-26)) kept = true;
        else if (ss < __dmul_rn(t2, 1.0 - 0x1p-26)) kept = false;
        else kept = lane == 0 ? l2_exact_reaches<T>(x, base, C, tau) : false;
    }
    if (lane == 0) keep[t] = kept ? 1 : 0;
}

// ---- vector path for f16 / bf16 rows -----------------------------------------
//
// Used when the rows are 16-byte aligned (x and tok_stride * 2), C is a
// multiple of 8 and at most kMaskVecMaxC.  One half-warp per token, each lane
// reading whole 16-byte vectors (8 elements).  A square of an f16 or bf16
// value is exact in fp32 unless it leaves fp32's normal range (only bf16 can),
// and each lane adds its squares into two fp32 accumulators with an
// error-free two-sum, keeping the rounding errors in a second pair: with n
// terms per accumulator the pair (s, c) is within a relative n^2 2^-48 of its
// exact sum (n = C / 32 <= 256 here: 2^-32).  The 32 pairs of a token are then added in
// fp64 (a relative 2^-48 more).  That sum is trusted where it is finite and
// at least 2^-100 (squares below fp32's normal range then add at most a
// relative 2^-37; f16 squares never leave it, so an f16 sum of 0 is exact
// too); elsewhere (NaN, an infinite element, a bf16 overflow or underflow)
// the token falls back to the fp64 sum of mask_l2_kernel.  The decision is
// the same as there, on a sum within a relative 2^-29 of the exact one.
constexpr int kMaskVecMaxC = 8192;   // at most 256 terms per accumulator

__device__ __forceinline__ void two_sum_acc(float& s, float& c, float y) {
    const float t = __fadd_rn(s, y);
    const float bp = __fsub_rn(t, s);
    const float e = __fadd_rn(__fsub_rn(s, __fsub_rn(t, bp)), __fsub_rn(y, bp));
    s = t;
    c = __fadd_rn(c, e);
}

template <typename T>
__device__ __forceinline__ float2 widen2(uint32_t w);
template <>
__device__ __forceinline__ float2 widen2<__half>(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
template <>
__device__ __forceinline__ float2 widen2<__nv_bfloat16>(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <typename T>
__global__ void __launch_bounds__(kMaskThreads)
    mask_l2_vec_kernel(const void* __restrict__ x, int L_full, int C, int64_t tok_stride, double tau,
                       uint8_t* __restrict__ keep) {
    const int j = blockIdx.x * (kMaskThreads / 16) + (threadIdx.x >> 4);
    const int hl = threadIdx.x & 15;                    // lane within the half-warp
    const unsigned hmask = 0xffffu << (threadIdx.x & 16);
    if (j >= L_full) return;   // uniform over the half-warp
    const int64_t t = static_cast<int64_t>(blockIdx.y) * L_full + j;
    const int64_t base = t * tok_stride;
    const uint4* row = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + base);
    const int nvec = C >> 3;
    float s0 = 0.f, c0 = 0.f, s1 = 0.f, c1 = 0.f;
    // One vector per lane and step.  Requesting four vectors before any
    // arithmetic, or two or four tokens per half-warp, measured slower.
    for (int v = hl; v < nvec; v += 16) {
        const uint4 q = __ldg(row + v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = widen2<T>(w[i]);
            two_sum_acc(s0, c0, __fmul_rn(f.x, f.x));
            two_sum_acc(s1, c1, __fmul_rn(f.y, f.y));
        }
    }
    double ss = __dadd_rn(__dadd_rn(static_cast<double>(s0), static_cast<double>(c0)),
                          __dadd_rn(static_cast<double>(s1), static_cast<double>(c1)));
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(hmask, ss, off));
    const bool trusted = isfinite(ss) && (ss >= 0x1p-100 || (ss == 0.0 && std::is_same<T, __half>::value));
    if (!trusted) {   // uniform over the half-warp: the fp64 sum of mask_l2_kernel
        double acc = 0.0;
        for (int c = hl; c < C; c += 16) {
            const double v = widen<T>(x, base + c);
            acc = __dadd_rn(acc, __dmul_rn(v, v));
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) acc = __dadd_rn(acc, __shfl_xor_sync(hmask, acc, off));
        ss = acc;
    }
    bool kept;
    if (j == 0) kept = true;
    else if (isnan(ss)) kept = false;
    else if (isinf(ss) || !(tau > 0.0)) kept = true;
    else if (tau > 0x1p+140) kept = false;
    else if (tau < 0x1p-400) kept = ss > 0.0;
    else {
        const double t2 = __dmul_rn(tau, tau);
        if (ss > __dmul_rn(t2, 1.0 + 0x1p-26)) kept = true;
        else if (ss < __dmul_rn(t2, 1.0 - 0x1p-26)) kept = false;
        else kept = hl == 0 ? l2_exact_reaches<T>(x, base, C, tau) : false;
    }
    if (hl == 0) keep[t] = kept ? 1 : 0;
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
