// Ragged bidirectional attention, f16 / bf16 inputs, warp-level tensor-core
// MMA (mma.sync m16n8k16, fp32 accumulate), head_dim 64.
//
// Operation ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// abstract; radpulse section "Bypassing the binding": bidirectional, no causal
// mask, no KV cache): for every sequence b of the packed buffer and head h,
// O = softmax(scale Q K^T) V over the L_b rows cu[b] .. cu[b+1]-1 only.
//
// Schedule: one CTA per (64-query tile, head, sequence); grid (ceil(max_seqlen
// / 64), H, B) where max_seqlen is the host's bound, so no host sync is needed
// to size the launch.  A CTA reads cu[b], cu[b+1] and returns at once when its
// tile starts past L_b.  Four warps own 16 query rows each.  K/V tiles of 64
// keys are double-buffered through shared memory with cp.async (rows past L_b
// are zero-filled), the softmax is the streaming (online) form in fp32 with
// quad shuffles for row max / sum, and the output is staged through shared
// memory so that every global store is a full 128-byte row.  No softmax
// log-sum-exp is written and nothing is allocated.
//
// Precision: S = Q K^T is exact products summed in fp32.  P = exp2(S * scale *
// log2 e - m) is fp32.  For f16, P is rounded to f16 for the PV product.  For
// bf16, P is split as P_hi = bf16(P), P_lo = bf16(P - P_hi) and both halves are
// multiplied with V (two MMAs), so the PV error is ~2^-17 relative instead of
// bf16's 2^-9; this keeps the result within the rounding of the bf16 output.
#pragma once

#include "mma_common.cuh"

namespace ragged {
namespace mma_attn {

constexpr int kHeadDim = 64;
constexpr int kBlockM = 64;   // query rows per CTA
constexpr int kBlockN = 64;   // keys per shared-memory tile
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kTileBytes = kBlockM * kHeadDim * 2;   // 8 KB per 64 x 64 16-bit tile
constexpr int kSmemBytes = kTileBytes * 5;            // Q, K[2], V[2]

// Loads rows [row0, row0 + 64) of one head of one sequence into a swizzled
// shared tile.  `g` points at element (row 0, head h, dim 0).
__device__ __forceinline__ void load_tile(uint32_t s_tile, const uint16_t* __restrict__ g,
                                          int64_t tok_stride, int row0, int len) {
#pragma unroll
    for (int i = threadIdx.x; i < kBlockM * 8; i += kThreads) {
        const int r = i >> 3, c = i & 7;
        const int row = row0 + r;
        const bool ok = row < len;
        const uint16_t* src = g + static_cast<int64_t>(ok ? row : 0) * tok_stride + c * 8;
        cp_async_16(s_tile + swz(r, c), src, ok ? 16 : 0);
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
    attn_fwd_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                    const uint16_t* __restrict__ v, int64_t tok_stride, int64_t head_stride,
                    const int32_t* __restrict__ cu, int max_seqlen, int H, float scale_log2,
                    uint16_t* __restrict__ out, int64_t out_tok_stride,
                    uint16_t* __restrict__ cls_out) {
    extern __shared__ __align__(128) uint8_t smem[];
    // The query tile is the slowest grid index: a launch is sized by the host
    // bound max_seqlen, and with short sequences most CTAs of the later query
    // tiles exit at once, so the ones with work are all dispatched first.
    const int qt = blockIdx.z, h = blockIdx.x, b = blockIdx.y;
    int start, len;
    if (!read_sequence(cu, b, max_seqlen, start, len)) return;
    const int q0 = qt * kBlockM;
    if (q0 >= len) return;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Shared layout: Q | K0 | K1 | V0 | V1, one 8 KB tile each.
    const uint32_t s_q = smem_addr(smem);
    auto s_k = [&](int i) { return s_q + (1 + i) * kTileBytes; };
    auto s_v = [&](int i) { return s_q + (3 + i) * kTileBytes; };

    const int64_t seq_off = static_cast<int64_t>(start) * tok_stride + static_cast<int64_t>(h) * head_stride;
    const uint16_t* gq = q + seq_off;
    const uint16_t* gk = k + seq_off;
    const uint16_t* gv = v + seq_off;

    const int n_tiles = (len + kBlockN - 1) / kBlockN;
    load_tile(s_q, gq, tok_stride, q0, len);
    load_tile(s_k(0), gk, tok_stride, 0, len);
    load_tile(s_v(0), gv, tok_stride, 0, len);
    cp_async_commit();

    const bool warp_active = q0 + warp * 16 < len;
    const int g = lane >> 2, tig = lane & 3;

    uint32_t qf[4][4];
    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[j][e] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;   // running max of rows g and g+8 (log2 units)
    float l0 = 0.f, l1 = 0.f;               // this thread's share of the running sums

    for (int t = 0; t < n_tiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < n_tiles) {
            load_tile(s_k(buf ^ 1), gk, tok_stride, (t + 1) * kBlockN, len);
            load_tile(s_v(buf ^ 1), gv, tok_stride, (t + 1) * kBlockN, len);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();

        if (warp_active) {
            if (t == 0) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    ldmatrix_x4(qf[ks], s_q + swz(warp * 16 + (lane & 15), ks * 2 + (lane >> 4)));
            }
            // S = Q K^T for 16 rows x 64 keys.
            float s[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[j][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                for (int jp = 0; jp < 4; ++jp) {
                    uint32_t kb[4];
                    const int key = jp * 16 + (lane & 7) + ((lane >> 4) << 3);
                    const int chunk = ks * 2 + ((lane >> 3) & 1);
                    ldmatrix_x4(kb, s_k(buf) + swz(key, chunk));
                    Mma<T>::run(s[2 * jp], qf[ks], kb[0], kb[1]);
                    Mma<T>::run(s[2 * jp + 1], qf[ks], kb[2], kb[3]);
                }
            }
            // Keys past the end of the sequence take no weight.
            const int kv0 = t * kBlockN;
            if (kv0 + kBlockN > len) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int key = kv0 + j * 8 + tig * 2;
                    if (key >= len) { s[j][0] = -INFINITY; s[j][2] = -INFINITY; }
                    if (key + 1 >= len) { s[j][1] = -INFINITY; s[j][3] = -INFINITY; }
                }
            }
            // Online softmax in base 2: logits are s * scale * log2(e).
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
                mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0 * scale_log2);
            const float mn1 = fmaxf(m1, mx1 * scale_log2);
            const float alpha0 = fast_exp2(m0 - mn0);
            const float alpha1 = fast_exp2(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                s[j][0] = fast_exp2(fmaf(s[j][0], scale_log2, -mn0));
                s[j][1] = fast_exp2(fmaf(s[j][1], scale_log2, -mn0));
                s[j][2] = fast_exp2(fmaf(s[j][2], scale_log2, -mn1));
                s[j][3] = fast_exp2(fmaf(s[j][3], scale_log2, -mn1));
                rs0 += s[j][0] + s[j][1];
                rs1 += s[j][2] + s[j][3];
            }
            l0 = l0 * alpha0 + rs0;
            l1 = l1 * alpha1 + rs1;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                o[j][0] *= alpha0; o[j][1] *= alpha0;
                o[j][2] *= alpha1; o[j][3] *= alpha1;
            }
            // O += P V.
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t pa[4];
                pa[0] = Mma<T>::pack(s[2 * ks][0], s[2 * ks][1]);
                pa[1] = Mma<T>::pack(s[2 * ks][2], s[2 * ks][3]);
                pa[2] = Mma<T>::pack(s[2 * ks + 1][0], s[2 * ks + 1][1]);
                pa[3] = Mma<T>::pack(s[2 * ks + 1][2], s[2 * ks + 1][3]);
                uint32_t pr[4];
                if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                    pr[0] = Mma<T>::pack_residual(s[2 * ks][0], s[2 * ks][1], pa[0]);
                    pr[1] = Mma<T>::pack_residual(s[2 * ks][2], s[2 * ks][3], pa[1]);
                    pr[2] = Mma<T>::pack_residual(s[2 * ks + 1][0], s[2 * ks + 1][1], pa[2]);
                    pr[3] = Mma<T>::pack_residual(s[2 * ks + 1][2], s[2 * ks + 1][3], pa[3]);
                }
#pragma unroll
                for (int dp = 0; dp < 4; ++dp) {
                    uint32_t vb[4];
                    const int key = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int chunk = dp * 2 + (lane >> 4);
                    ldmatrix_x4_trans(vb, s_v(buf) + swz(key, chunk));
                    Mma<T>::run(o[2 * dp], pa, vb[0], vb[1]);
                    Mma<T>::run(o[2 * dp + 1], pa, vb[2], vb[3]);
                    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                        Mma<T>::run(o[2 * dp], pr, vb[0], vb[1]);
                        Mma<T>::run(o[2 * dp + 1], pr, vb[2], vb[3]);
                    }
                }
            }
        }
        __syncthreads();
    }

    if (!warp_active) return;
    // Normalise and stage this warp's 16 rows in its own rows of the Q tile
    // (its Q fragments are already in registers).
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    uint8_t* s_o = smem;
    const int r_lo = warp * 16 + g, r_hi = r_lo + 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        *reinterpret_cast<uint32_t*>(s_o + swz(r_lo, j) + tig * 4) = Mma<T>::pack(o[j][0] * inv0, o[j][1] * inv0);
        *reinterpret_cast<uint32_t*>(s_o + swz(r_hi, j) + tig * 4) = Mma<T>::pack(o[j][2] * inv1, o[j][3] * inv1);
    }
    __syncwarp();
#pragma unroll
    for (int i = lane; i < 16 * 8; i += 32) {
        const int r = i >> 3, c = i & 7;
        const int row = q0 + warp * 16 + r;
        if (row < len) {
            const uint4 val = *reinterpret_cast<const uint4*>(s_o + swz(warp * 16 + r, c));
            *reinterpret_cast<uint4*>(out + static_cast<int64_t>(start + row) * out_tok_stride +
                                      h * kHeadDim + c * 8) = val;
            if (row == 0 && cls_out != nullptr)
                *reinterpret_cast<uint4*>(cls_out + (static_cast<int64_t>(b) * H + h) * kHeadDim + c * 8) = val;
        }
    }
}

}  // namespace mma_attn
}  // namespace ragged
