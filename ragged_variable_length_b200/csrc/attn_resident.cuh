// Ragged bidirectional attention with the whole sequence resident in shared
// memory (sequences up to 640 keys), f16 / bf16, mma.sync m16n8k16, and the
// single-launch pack -> attend -> CLS pipeline built on it.
//
// Operation ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// abstract; radpulse section "Bypassing the binding"): per sequence b and head
// h, O = softmax(scale Q K^T) V over the sequence's own L_b rows, no causal
// mask, no KV cache, no padding.
//
// ViT sequences are short (197 tokens at 224x224, 577 at 384x384), so one
// CTA can hold all of a head's K and V: each CTA (64-query tile, head,
// sequence) issues every load of its Q tile and of all K/V tiles at once
// (cp.async, one commit group per 64-key tile) and consumes the tiles as they
// land.  A streaming kernel pays one DRAM round trip per K/V tile; this one
// pays one for the whole sequence.
//
// Work split inside a CTA (template KSPLIT): the 4 warps cover RB = 4 / KSPLIT
// blocks of 16 query rows, and the KSPLIT warps of one row block share its
// keys, each taking every KSPLIT-th 64-key tile; their partial softmax states
// (max, sum, unnormalised output) are merged through shared memory at the
// end.  KSPLIT = 1 (64-row tiles) suits long, throughput-bound launches;
// KSPLIT = 4 (16-row tiles, four warps per row block) cuts the serial chain of
// each warp to a quarter for the short, latency-bound launches of serving.
//
// Row sources:
//   PackedRows  rows cu[b] .. cu[b+1]-1 of packed q/k/v views (ragged_attn_fwd)
//   DenseRows   the survivors of image b read straight from the dense fused
//               q/k/v buffer: the CTA ranks the keep mask itself (warp ballot
//               scan) and counts the survivors of the images before b for
//               cu[b], so pack, attention and CLS extraction are one launch
//               and the packed q/k/v never has to be written (it is, when the
//               caller asks for it).  radpulse, "Integrated pack pipeline":
//               cu_seqlens, survivor copy, attention, CLS extraction.
#pragma once

#include "mma_common.cuh"
#include "pack.cuh"

namespace ragged {
namespace resident {

using mma_attn::Mma;
using mma_attn::fast_exp2;
using mma_attn::ldmatrix_x4;
using mma_attn::ldmatrix_x4_trans;
using mma_attn::swz;

constexpr int kHeadDim = 64;
constexpr int kBlockM = 64;
constexpr int kBlockN = 64;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kTileBytes = kBlockM * kHeadDim * 2;
constexpr int kMaxKeyTiles = 10;
constexpr int kMaxKeys = kMaxKeyTiles * kBlockN;   // 640

// Dynamic shared memory: Q tile, key_tiles K tiles, key_tiles V tiles, then
// the survivor list (list_entries ints, DenseRows only).
__host__ __device__ constexpr int smem_bytes(int key_tiles, int list_entries) {
    return kTileBytes * (1 + 2 * key_tiles) + ((list_entries * 4 + 15) / 16) * 16;
}

// cp.async.wait_group needs an immediate; pending is at most kMaxKeyTiles - 1.
__device__ __forceinline__ void cp_async_wait_pending(int pending) {
    switch (pending) {
        case 0: cp_async_wait<0>(); break;
        case 1: cp_async_wait<1>(); break;
        case 2: cp_async_wait<2>(); break;
        case 3: cp_async_wait<3>(); break;
        case 4: cp_async_wait<4>(); break;
        case 5: cp_async_wait<5>(); break;
        case 6: cp_async_wait<6>(); break;
        case 7: cp_async_wait<7>(); break;
        case 8: cp_async_wait<8>(); break;
        default: cp_async_wait<9>(); break;
    }
}

struct PackedRows {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    int64_t tok_stride, head_stride;   // elements
    const int32_t* cu;
    int max_seqlen;
    // per CTA
    int start, len;
    int64_t head_off;

    __device__ __forceinline__ bool begin(int b, int h, int* /*s_list*/, int* /*s_red*/) {
        if (!read_sequence(cu, b, max_seqlen, start, len)) return false;
        head_off = static_cast<int64_t>(h) * head_stride;
        return true;
    }
    // which: 0 = q, 1 = k, 2 = v; r < len
    __device__ __forceinline__ const uint16_t* row(int which, int r) const {
        const uint16_t* base = which == 0 ? q : (which == 1 ? k : v);
        return base + static_cast<int64_t>(start + r) * tok_stride + head_off;
    }
};

struct DenseRows {
    const uint16_t* dense;      // [B, L_full, 3, H, 64]
    const uint8_t* keep;        // [B, L_full]
    int32_t* cu_out;            // [B + 1]
    int L_full, H;
    // per CTA
    int start, len;
    int64_t row0;               // flat dense row of token 0 of image b
    int h;
    const int* s_list;

    __device__ __forceinline__ bool begin(int b, int h_, int* s_list_, int* s_red) {
        h = h_;
        s_list = s_list_;
        row0 = static_cast<int64_t>(b) * L_full;
        const uint8_t* kb = keep + row0;
        // This image's mask bytes are read before anything depends on them, so
        // their latency overlaps the count over the earlier images.
        uint8_t mine[kMaxKeys / kThreads];
#pragma unroll
        for (int i = 0; i < kMaxKeys / kThreads; ++i) {
            const int j = threadIdx.x + i * kThreads;
            mine[i] = j < L_full ? kb[j] : 0;
        }
        // Pull this head's q/k/v rows of the surviving tokens towards L2 while
        // the mask is ranked; the CTAs of one (image, head) share the
        // prefetches.  Each prefetch waits only for its own token's keep byte,
        // so dropped tokens' rows are never read.
        const int share = gridDim.x;
        const int64_t row_elems = 3LL * H * kHeadDim;
        for (int j = blockIdx.x + share * (threadIdx.x / 3); j < L_full; j += share * (kThreads / 3)) {
            if (threadIdx.x >= (kThreads / 3) * 3) break;
            const uint16_t* p = dense + (row0 + j) * row_elems + ((threadIdx.x % 3) * H + h) * kHeadDim;
            if (j == 0 || kb[j] != 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
        }
        int forced = 0;
        for (int i = threadIdx.x; i < b; i += kThreads) forced += keep[static_cast<int64_t>(i) * L_full] == 0;
        start = cta_count_nonzero<kThreads>(keep, row0, forced, s_red);
        len = rank_from_registers(mine, L_full, s_list_, s_red);
        if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) {
            cu_out[b + 1] = start + len;
            if (b == 0) cu_out[0] = 0;
        }
        return true;
    }

    // Warp-ballot ranking of the survivors (CLS always kept) from mask bytes
    // already held in registers: byte i of thread t is token t + i * kThreads.
    __device__ __forceinline__ static int rank_from_registers(const uint8_t (&mine)[kMaxKeys / kThreads],
                                                              int L_full, int* s_kept, int* s_red) {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        int running = 0;
#pragma unroll
        for (int i = 0; i < kMaxKeys / kThreads; ++i) {
            const int j0 = i * kThreads;
            if (j0 >= L_full) break;
            const int j = j0 + threadIdx.x;
            const bool kept = j < L_full && (j == 0 || mine[i] != 0);
            const unsigned bal = __ballot_sync(0xffffffffu, kept);
            if (lane == 0) s_red[warp] = __popc(bal);
            __syncthreads();
            int before = 0, total = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
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
    __device__ __forceinline__ const uint16_t* row(int which, int r) const {
        return dense + (row0 + s_list[r]) * (3LL * H * kHeadDim) + (which * H + h) * kHeadDim;
    }
};

// Issues the loads of rows [row0, row0 + ROWS) of `which` into a swizzled
// tile; rows at or past len are zero-filled.
template <int ROWS, class Src>
__device__ __forceinline__ void load_tile(uint32_t s_tile, const Src& src, int which, int row0, int len) {
#pragma unroll
    for (int i = threadIdx.x; i < ROWS * 8; i += kThreads) {
        const int r = i >> 3, c = i & 7;
        const int row = row0 + r;
        const bool ok = row < len;
        const uint16_t* g = src.row(which, ok ? row : 0) + c * 8;
        cp_async_16(s_tile + swz(r, c), g, ok ? 16 : 0);
    }
}

// Copies rows [row0, min(row0 + ROWS, len)) of a shared tile to the packed
// fused buffer (part 0/1/2 = q/k/v of head h).
template <int ROWS>
__device__ __forceinline__ void store_packed_tile(const uint8_t* s_tile, uint16_t* packed, int64_t row_elems,
                                                  int start, int row0, int len, int part, int H, int h) {
    for (int i = threadIdx.x; i < ROWS * 8; i += kThreads) {
        const int r = i >> 3, c = i & 7;
        if (row0 + r >= len) continue;
        const uint4 val = *reinterpret_cast<const uint4*>(s_tile + swz(r, c));
        *reinterpret_cast<uint4*>(packed + static_cast<int64_t>(start + row0 + r) * row_elems +
                                  (part * H + h) * kHeadDim + c * 8) = val;
    }
}

// Copies ROWS rows of a 64-row shared tile starting at tile row r0 (rows
// row0 .. row0 + ROWS - 1 of the sequence, those below len) to the packed
// fused buffer.
template <int ROWS>
__device__ __forceinline__ void store_packed_rows(const uint8_t* s_tile, int r0, uint16_t* packed, int64_t row_elems,
                                                  int start, int row0, int len, int part, int H, int h) {
    for (int i = threadIdx.x; i < ROWS * 8; i += kThreads) {
        const int r = i >> 3, c = i & 7;
        if (row0 + r >= len) continue;
        const uint4 val = *reinterpret_cast<const uint4*>(s_tile + swz(r0 + r, c));
        *reinterpret_cast<uint4*>(packed + static_cast<int64_t>(start + row0 + r) * row_elems +
                                  (part * H + h) * kHeadDim + c * 8) = val;
    }
}

template <typename T, class Src, int KSPLIT>
__global__ void __launch_bounds__(kThreads)
    attn_resident_kernel(Src src, int key_tiles, float scale_log2, int H, uint16_t* __restrict__ out,
                         int64_t out_tok_stride, uint16_t* __restrict__ cls_out,
                         uint16_t* __restrict__ packed_out) {
    static_assert(KSPLIT == 1 || KSPLIT == 2 || KSPLIT == 4, "KSPLIT must divide the 4 warps");
    constexpr int RB = kWarps / KSPLIT;          // 16-row blocks per CTA
    constexpr int kRows = 16 * RB;               // query rows per CTA
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_red[kWarps];
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    int* s_list = reinterpret_cast<int*>(smem + kTileBytes * (1 + 2 * key_tiles));
    if (!src.begin(b, h, s_list, s_red)) return;
    const int len = src.len, start = src.start;
    const int q0 = qt * kRows;
    if (q0 >= len) return;
    const int nt = (len + kBlockN - 1) / kBlockN;   // <= key_tiles (host bound)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rb = warp % RB, kg = warp / RB;      // row block, key group
    const uint32_t s_q = smem_addr(smem);
    auto s_k = [&](int t) { return s_q + (1 + t) * kTileBytes; };
    auto s_v = [&](int t) { return s_q + (1 + key_tiles + t) * kTileBytes; };

    // Every load of the CTA is in flight before any compute: group 0 = Q and
    // key tile 0, group t = key tile t.
    load_tile<kRows>(s_q, src, 0, q0, len);
    for (int t = 0; t < nt; ++t) {
        load_tile<kBlockN>(s_k(t), src, 1, t * kBlockN, len);
        load_tile<kBlockN>(s_v(t), src, 2, t * kBlockN, len);
        cp_async_commit();
    }

    const bool rows_active = q0 + rb * 16 < len;
    const int g = lane >> 2, tig = lane & 3;
    uint32_t qf[4][4];
    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[j][e] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool have_q = false;

    // Rounds of KSPLIT tiles: round r needs load groups 0 .. (r+1)*KSPLIT - 1.
    const int rounds = (nt + KSPLIT - 1) / KSPLIT;
    for (int r = 0; r < rounds; ++r) {
        const int last = min(nt - 1, (r + 1) * KSPLIT - 1);
        cp_async_wait_pending(nt - 1 - last);
        __syncthreads();
        const int t = r * KSPLIT + kg;
        if (!rows_active || t >= nt) continue;
        if (!have_q) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                ldmatrix_x4(qf[ks], s_q + swz(rb * 16 + (lane & 15), ks * 2 + (lane >> 4)));
            have_q = true;
        }
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
                ldmatrix_x4(kb, s_k(t) + swz(key, chunk));
                Mma<T>::run(s[2 * jp], qf[ks], kb[0], kb[1]);
                Mma<T>::run(s[2 * jp + 1], qf[ks], kb[2], kb[3]);
            }
        }
        const int kv0 = t * kBlockN;
        if (kv0 + kBlockN > len) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int key = kv0 + j * 8 + tig * 2;
                if (key >= len) { s[j][0] = -INFINITY; s[j][2] = -INFINITY; }
                if (key + 1 >= len) { s[j][1] = -INFINITY; s[j][3] = -INFINITY; }
            }
        }
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
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t pa[4], pr[4];
            pa[0] = Mma<T>::pack(s[2 * ks][0], s[2 * ks][1]);
            pa[1] = Mma<T>::pack(s[2 * ks][2], s[2 * ks][3]);
            pa[2] = Mma<T>::pack(s[2 * ks + 1][0], s[2 * ks + 1][1]);
            pa[3] = Mma<T>::pack(s[2 * ks + 1][2], s[2 * ks + 1][3]);
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
                ldmatrix_x4_trans(vb, s_v(t) + swz(key, chunk));
                Mma<T>::run(o[2 * dp], pa, vb[0], vb[1]);
                Mma<T>::run(o[2 * dp + 1], pa, vb[2], vb[3]);
                if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                    Mma<T>::run(o[2 * dp], pr, vb[0], vb[1]);
                    Mma<T>::run(o[2 * dp + 1], pr, vb[2], vb[3]);
                }
            }
        }
    }

    // Optional packed q/k/v for the caller (fused pipeline): every CTA writes
    // the q, k and v rows of head h for its own query rows [q0, q0 + kRows),
    // so the CTAs of a (sequence, head) cover each packed row exactly once.
    if (packed_out != nullptr) {
        const int64_t row_elems = 3LL * H * kHeadDim;
        store_packed_tile<kRows>(smem, packed_out, row_elems, start, q0, len, 0, H, h);
        const int t = q0 / kBlockN, r0 = q0 % kBlockN;
        store_packed_rows<kRows>(smem + (1 + t) * kTileBytes, r0, packed_out, row_elems, start, q0, len, 1, H, h);
        store_packed_rows<kRows>(smem + (1 + key_tiles + t) * kTileBytes, r0, packed_out, row_elems, start, q0, len,
                                 2, H, h);
    }

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    if constexpr (KSPLIT > 1) {
        // Merge the KSPLIT partial states of each row block.  The K/V tiles are
        // dead now; their space holds per-warp partials in fragment order:
        // float4 per (warp, n-tile, lane) for O, float4 per (warp, lane) for
        // (m0, m1, l0, l1).
        __syncthreads();
        float4* s_po = reinterpret_cast<float4*>(smem + kTileBytes);
        float4* s_pm = s_po + kWarps * 8 * 32;
        if (kg != 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j) s_po[(warp * 8 + j) * 32 + lane] = make_float4(o[j][0], o[j][1], o[j][2], o[j][3]);
            s_pm[warp * 32 + lane] = make_float4(m0, m1, l0, l1);
        }
        __syncthreads();
        if (kg != 0) return;
#pragma unroll
        for (int p = 1; p < KSPLIT; ++p) {
            const int w2 = p * RB + rb;
            const float4 ml = s_pm[w2 * 32 + lane];
            const float M0 = fmaxf(m0, ml.x), M1 = fmaxf(m1, ml.y);
            // exp2(-inf - M) = 0 handles partials without any key
            const float a0 = fast_exp2(m0 - M0), b0 = fast_exp2(ml.x - M0);
            const float a1 = fast_exp2(m1 - M1), b1 = fast_exp2(ml.y - M1);
            l0 = l0 * a0 + ml.z * b0;
            l1 = l1 * a1 + ml.w * b1;
            m0 = M0;
            m1 = M1;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 po = s_po[(w2 * 8 + j) * 32 + lane];
                o[j][0] = o[j][0] * a0 + po.x * b0;
                o[j][1] = o[j][1] * a0 + po.y * b0;
                o[j][2] = o[j][2] * a1 + po.z * b1;
                o[j][3] = o[j][3] * a1 + po.w * b1;
            }
        }
    } else if (packed_out != nullptr) {
        __syncthreads();   // the Q tile is reused below to stage the output
    }

    if (!rows_active) return;
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    uint8_t* s_o = smem;
    const int r_lo = rb * 16 + g, r_hi = r_lo + 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        *reinterpret_cast<uint32_t*>(s_o + swz(r_lo, j) + tig * 4) = Mma<T>::pack(o[j][0] * inv0, o[j][1] * inv0);
        *reinterpret_cast<uint32_t*>(s_o + swz(r_hi, j) + tig * 4) = Mma<T>::pack(o[j][2] * inv1, o[j][3] * inv1);
    }
    __syncwarp();
#pragma unroll
    for (int i = lane; i < 16 * 8; i += 32) {
        const int r = i >> 3, c = i & 7;
        const int row = q0 + rb * 16 + r;
        if (row < len) {
            const uint4 val = *reinterpret_cast<const uint4*>(s_o + swz(rb * 16 + r, c));
            *reinterpret_cast<uint4*>(out + static_cast<int64_t>(start + row) * out_tok_stride + h * kHeadDim + c * 8) = val;
            if (row == 0 && cls_out != nullptr)
                *reinterpret_cast<uint4*>(cls_out + (static_cast<int64_t>(b) * H + h) * kHeadDim + c * 8) = val;
        }
    }
}

}  // namespace resident
}  // namespace ragged
