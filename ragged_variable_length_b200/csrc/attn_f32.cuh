// Ragged bidirectional attention, fp32 check path: plain FFMA arithmetic (no
// tensor cores, so no TF32 rounding), head_dim 64.
//
// Same operation as the tensor-core kernel (per sequence b and head h,
// O = softmax(scale Q K^T) V over the rows cu[b] .. cu[b+1]-1).  One CTA per
// (32-query tile, head, sequence); 8 warps, each warp owns 4 query rows and
// walks the keys in shared-memory tiles of 64 with the streaming softmax.  A
// lane computes the logit of one key per 32-key chunk; the output row is held
// as two dims per lane.  exp is CUDA's expf.
#pragma once

#include "common.cuh"

namespace ragged {
namespace f32_attn {

constexpr int kHeadDim = 64;
constexpr int kBlockM = 32;
constexpr int kBlockN = 64;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerWarp = kBlockM / kWarps;
constexpr int kPad = kHeadDim + 1;   // odd row pitch: lane j reading row j is conflict-free
constexpr int kSmemBytes = (2 * kBlockN * kPad + kBlockM * kHeadDim) * 4;

__global__ void __launch_bounds__(kThreads)
    attn_fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                        const float* __restrict__ v, int64_t tok_stride, int64_t head_stride,
                        const int32_t* __restrict__ cu, int max_seqlen, int H, float scale,
                        float* __restrict__ out, int64_t out_tok_stride, float* __restrict__ cls_out) {
    extern __shared__ float smem_f[];
    float* s_k = smem_f;                         // [64][65]
    float* s_v = s_k + kBlockN * kPad;           // [64][65]
    float* s_q = s_v + kBlockN * kPad;           // [32][64]
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    int start, len;
    if (!read_sequence(cu, b, max_seqlen, start, len)) return;
    const int q0 = qt * kBlockM;
    if (q0 >= len) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t seq_off = static_cast<int64_t>(start) * tok_stride + static_cast<int64_t>(h) * head_stride;

    for (int i = tid; i < kBlockM * kHeadDim; i += kThreads) {
        const int r = i / kHeadDim, c = i % kHeadDim;
        s_q[i] = (q0 + r < len) ? q[seq_off + static_cast<int64_t>(q0 + r) * tok_stride + c] : 0.f;
    }
    float m[kRowsPerWarp], l[kRowsPerWarp], acc0[kRowsPerWarp], acc1[kRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) { m[i] = -INFINITY; l[i] = 0.f; acc0[i] = 0.f; acc1[i] = 0.f; }

    for (int kv0 = 0; kv0 < len; kv0 += kBlockN) {
        __syncthreads();
        for (int i = tid; i < kBlockN * kHeadDim; i += kThreads) {
            const int r = i / kHeadDim, c = i % kHeadDim;
            const bool ok = kv0 + r < len;
            const int64_t off = seq_off + static_cast<int64_t>(kv0 + r) * tok_stride + c;
            s_k[r * kPad + c] = ok ? k[off] : 0.f;
            s_v[r * kPad + c] = ok ? v[off] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int r = warp * kRowsPerWarp + i;
            const float* qr = s_q + r * kHeadDim;
            for (int c0 = 0; c0 < kBlockN; c0 += 32) {
                const int key = kv0 + c0 + lane;
                float sc = 0.f;
#pragma unroll 16
                for (int c = 0; c < kHeadDim; ++c) sc = fmaf(qr[c], s_k[(c0 + lane) * kPad + c], sc);
                sc = (key < len) ? sc * scale : -INFINITY;
                float cmax = sc;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
                const float mn = fmaxf(m[i], cmax);
                if (mn == -INFINITY) continue;    // whole chunk past the end
                const float alpha = expf(m[i] - mn);
                const float p = expf(sc - mn);
                float psum = p;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
                l[i] = l[i] * alpha + psum;
                float a0 = acc0[i] * alpha, a1 = acc1[i] * alpha;
#pragma unroll 8
                for (int j = 0; j < 32; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, p, j);
                    a0 = fmaf(pj, s_v[(c0 + j) * kPad + lane], a0);
                    a1 = fmaf(pj, s_v[(c0 + j) * kPad + lane + 32], a1);
                }
                acc0[i] = a0;
                acc1[i] = a1;
                m[i] = mn;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int row = q0 + warp * kRowsPerWarp + i;
        if (row >= len) continue;
        const float o0 = acc0[i] / l[i], o1 = acc1[i] / l[i];
        float* dst = out + static_cast<int64_t>(start + row) * out_tok_stride + h * kHeadDim;
        dst[lane] = o0;
        dst[lane + 32] = o1;
        if (row == 0 && cls_out != nullptr) {
            float* c = cls_out + (static_cast<int64_t>(b) * H + h) * kHeadDim;
            c[lane] = o0;
            c[lane + 32] = o1;
        }
    }
}

}  // namespace f32_attn
}  // namespace ragged
