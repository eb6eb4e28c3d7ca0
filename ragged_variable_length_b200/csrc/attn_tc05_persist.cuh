// Persistent, warp-specialised ragged attention on the 5th-generation tensor
// cores (tcgen05.mma with TMEM accumulators, TMA loads), f16 / bf16,
// head_dim 64.
//
// Operation ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// abstract; radpulse section "Bypassing the binding"): per sequence b and head
// h, O = softmax(scale Q K^T) V over the sequence's own rows, no causal mask,
// no padding.
//
// Work items are (sequence, 128-query tile, head) triples, numbered densely.
// Each CTA copies cu_seqlens into shared memory once, forms the exclusive
// prefix of H * ceil(L_b / 128) over the sequences, and takes items
// blockIdx.x, blockIdx.x + gridDim.x, ...; two CTAs share an SM.  TMEM
// (256 columns: S of two tiles, each overwritten in place by its P, and two
// O buffers for alternate items) and the mbarriers are set up once per CTA,
// so the per-launch fixed costs of a CTA (cu_seqlens read, TMEM allocation,
// first loads) are paid once, and the loads of the next item run under the
// softmax of the current one.
//
// Warp roles; they hand off through mbarriers only:
//   warp 5     loads.  Full tiles by TMA from 3-D tensor maps over
//              [rows, head, 64] with the 128-byte swizzle, which is the
//              canonical SWIZZLE_128B operand layout of tcgen05; partial tiles
//              (the last rows of a sequence) by cp.async with zero fill, each
//              lane's arrival triggered by the completion of its copies
//              (cp.async.mbarrier.arrive.noinc).  Q is double-buffered, K/V
//              flow through a 4-stage ring; the stage of an item's last tile
//              is handed back by the softmax warps once the epilogue has used
//              it to stage O for row-contiguous stores.
//   warp 4     one thread issues every tcgen05.mma.  Q K^T runs two tiles
//              ahead of P V: P V(g) as soon as P(g) is in TMEM, then S of tile
//              g + 2 into TMEM buffer g & 1 (in order behind P V(g), which
//              read P(g) from it).  Across items the walks simply continue.
//   warps 0-3  softmax, one thread per query row (TMEM lane = row), single
//              pass with a reference maximum that is raised (and the running
//              sum and O rescaled) only when a tile exceeds it by more than
//              2^8; P (bf16: hi and lo parts) replaces S in its TMEM buffer.
//              The pairwise fp32 work uses the packed f32x2 instructions of
//              sm_100.  An item's epilogue (O / l and the CLS row) runs after
//              the first tile of the next item, from the item's own O buffer,
//              so the softmax warps never wait at an item boundary for the
//              last product.
// The tile counter g runs across items, so every buffer parity carries over
// from one item to the next.
//
// Every mbarrier wait is bounded; a wait that gives up sets RAGGED_DEV_TIMEOUT
// in the status word, every role leaves its loop, the MMA thread waits for its
// own MMAs and the load warp for its own copies, and TMEM is freed.
#pragma once

#include <cuda.h>

#include "attn_tc05.cuh"

namespace ragged {
namespace tc05 {

constexpr int kPersistThreads = 192;
constexpr int kPersistStages = 4;
// TMEM per CTA (256 columns): S of two tiles at [0, 64) and [64, 128), each
// overwritten in place by its P (16-bit pairs; bf16 as hi + lo halves), and
// two O buffers at [128, 192) and [192, 256), one per alternate item.
constexpr uint32_t kOBufCol = 128;
constexpr int kPersistMaxB = 1024;   // cu_seqlens and item offsets live in shared memory
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr uint32_t kFullMask = 0xffffffffu;

// Dynamic shared memory: alignment slack, two Q buffers, the K/V ring, then
// cu_seqlens and the item offsets (B + 1 ints each).
__host__ __device__ constexpr int persist_smem_bytes(int B) {
    return 1024 + 2 * kQBytes + kPersistStages * 2 * kKVTileBytes + 2 * (B + 1) * 4;
}

struct PersistArgs {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    int64_t tok_stride, head_stride;   // elements
    const int32_t* cu;
    int B, H, max_seqlen;
    float scale_log2;
    uint16_t* out;
    int64_t out_tok_stride;
    uint16_t* cls_out;
};

// ---- mbarrier, TMA and packed-fp32 wrappers --------------------------------

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}
// One box of a 3-D tensor map (coordinates innermost first) into shared
// memory, completing `bytes` of the transaction count of mbar.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(mbar)
        : "memory");
}
// Arrives on mbar once every cp.async this thread has issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t mbar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(mbar) : "memory");
}
// Waits for every cp.async this thread has issued (commits them first).
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// 32 consecutive fp32 columns of this thread's TMEM lane, one load and its wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 consecutive 32-bit TMEM columns of this thread's lane <- v (no wait).
__device__ __forceinline__ void tmem_st16_u(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
        :
        : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Rows [row0, row0 + ROWS) of one head of a sequence (base = its row 0) into a
// swizzled tile by the 32 lanes of a warp; rows at or past len are zero-filled
// without being read.
template <int ROWS>
__device__ __forceinline__ void warp_load_rows(uint32_t s_tile, const uint16_t* base, int64_t tok_stride, int row0,
                                               int len, int lane) {
#pragma unroll 4
    for (int i = lane; i < ROWS * 8; i += 32) {
        const int r = i >> 3, c = i & 7;
        const int row = row0 + r;
        const bool ok = row < len;
        cp_async_16(s_tile + swz(r, c), base + static_cast<int64_t>(ok ? row : 0) * tok_stride + c * 8, ok ? 16 : 0);
    }
}

struct Item {
    int h, q0, start, len, nt, b;
};

// Item j -> (sequence, query tile, head); s_ip holds the exclusive item
// prefix over sequences (s_ip[B] = number of items > j).
__device__ __forceinline__ Item decode_item(int j, const int* s_cu, const int* s_ip, int B, int H) {
    int lo = 0, hi = B;   // s_ip[lo] <= j < s_ip[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_ip[mid] <= j) lo = mid;
        else hi = mid;
    }
    Item it;
    it.b = lo;
    const int r = j - s_ip[lo];
    const int qt = r / H;
    it.h = r - qt * H;
    it.q0 = qt * kRows;
    it.start = s_cu[lo];
    it.len = s_cu[lo + 1] - it.start;
    it.nt = (it.len + kTileN - 1) / kTileN;
    return it;
}

// Cursor over the tiles of a CTA's items: item j (the k-th of this CTA),
// key tile t of it.
struct Walk {
    int j, k, t, total;
    bool valid;
    Item it;
    const int* s_cu;
    const int* s_ip;
    int B, H;
    __device__ __forceinline__ Walk(int j0, int total_, const int* cu, const int* ip, int B_, int H_)
        : j(j0), k(0), t(0), total(total_), valid(j0 < total_), s_cu(cu), s_ip(ip), B(B_), H(H_) {
        if (valid) it = decode_item(j, s_cu, s_ip, B, H);
    }
    __device__ __forceinline__ void next() {
        if (++t < it.nt) return;
        t = 0;
        ++k;
        j += gridDim.x;
        valid = j < total;
        if (valid) it = decode_item(j, s_cu, s_ip, B, H);
    }
};

template <typename T>
__global__ void __launch_bounds__(kPersistThreads, 2)
    attn_tc05_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const PersistArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // kv_full[S], kv_empty[S], q_full[2], q_empty[2], s_full[2], p_full[0..1], pv_done[2], o_empty[0], drain,
    // o_empty[1], (unused), p_full[2..3], o_staged, o_stored
    __shared__ __align__(8) uint64_t s_bar[2 * kPersistStages + 18];
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int S = kPersistStages;
    constexpr int kParts = Cvt<T>::kParts;

    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sQ = (raw + 1023u) & ~1023u;   // Q buffer i at sQ + i * 16 KB
    const uint32_t sRing = sQ + 2 * kQBytes;      // stage s: K at sRing + s * 16 KB, V 8 KB further
    int* s_cu = reinterpret_cast<int*>(smem_raw + (sRing - raw) + S * 2 * kKVTileBytes);
    int* s_ip = s_cu + (a.B + 1);

    const uint32_t bar0 = smem_addr(&s_bar[0]);
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (S + s); };
    auto q_full = [&](int i) { return bar0 + 8u * (2 * S + i); };
    auto q_empty = [&](int i) { return bar0 + 8u * (2 * S + 2 + i); };
    auto s_full = [&](int i) { return bar0 + 8u * (2 * S + 4 + i); };
    // P of tile g is signalled on p_full(g & 3): warps with no rows in the
    // current query tile skip the softmax and may arrive for tile g + 2 while
    // another warp is still working on tile g, so tiles two apart must not
    // share a barrier (three tiles apart is impossible: Q K^T of tile g + 3
    // waits until every warp has read S(g + 1)).
    auto p_full = [&](int i) { return bar0 + 8u * (i < 2 ? 2 * S + 6 + i : 2 * S + 14 + (i - 2)); };
    auto pv_done = [&](int i) { return bar0 + 8u * (2 * S + 8 + i); };
    // O buffer i has been read out by the epilogue of its item.
    auto o_empty = [&](int i) { return bar0 + 8u * (i == 0 ? 2 * S + 10 : 2 * S + 12); };
    const uint32_t drain = bar0 + 8u * (2 * S + 11);
    // The epilogue's O tile is staged in shared memory / has been stored
    // (128 arrivals each, one phase per item).
    const uint32_t o_staged = bar0 + 8u * (2 * S + 16);
    const uint32_t o_stored = bar0 + 8u * (2 * S + 17);
    volatile int* fail_flag = &s_fail;

    // ---- setup: cu_seqlens, barriers, TMEM, item offsets ----
    for (int i = tid; i <= a.B; i += kPersistThreads) s_cu[i] = __ldg(a.cu + i);
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(kv_full(s), 32);
            mbar_init(kv_empty(s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(q_full(i), 32);
            mbar_init(q_empty(i), 1);
            mbar_init(s_full(i), 1);
            mbar_init(p_full(i), kSoftmaxThreads);
            mbar_init(p_full(i + 2), kSoftmaxThreads);
            mbar_init(pv_done(i), 1);
            mbar_init(o_empty(i), kSoftmaxThreads);
        }
        mbar_init(o_staged, kSoftmaxThreads);
        mbar_init(o_stored, kSoftmaxThreads);
        mbar_init(drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_fail = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem)),
                     "r"(kStreamTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == kLoadWarp) {   // item offsets: warp-wide inclusive scans over 32 sequences at a time
        int carry = 0;
        if (lane == 0) s_ip[0] = 0;
        for (int c0 = 0; c0 < a.B; c0 += 32) {
            const int b = c0 + lane;
            int n = 0;
            if (b < a.B) {
                const int st = s_cu[b], len = s_cu[b + 1] - st;
                // The tensor maps cover rows [0, B * max_seqlen): a sequence
                // reaching past them (cu[0] != 0 can shift one there) would
                // read zero fill, so it is flagged and skipped like the rest.
                if (st < 0 || len < 0 || len > a.max_seqlen ||
                    static_cast<int64_t>(st) + len > static_cast<int64_t>(a.B) * a.max_seqlen)
                    raise_status(RAGGED_DEV_BAD_SEQLENS);
                else n = ((len + kRows - 1) / kRows) * a.H;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFullMask, n, o);
                if (lane >= o) n += y;
            }
            if (b < a.B) s_ip[b + 1] = carry + n;
            carry += __shfl_sync(kFullMask, n, 31);
        }
    }
    __syncthreads();
    const int total = s_ip[a.B];
    const uint32_t tmem = s_tmem;

    if (warp == kLoadWarp) {
        // ---------------- loads ----------------
        // Warp-uniform bounded wait (every lane acquires the barrier).
        auto warp_wait = [&](uint32_t mbar, uint32_t parity) {
            const bool ok = __all_sync(kFullMask, mbar_wait(mbar, parity));
            if (!ok && lane == 0) atomicExch(&s_fail, 1);
            return ok;
        };
        // A partial tile is published without blocking the warp: each lane's
        // arrival is triggered by the completion of its own copies
        // (cp.async.mbarrier.arrive.noinc).  The MMA thread orders the
        // copies' generic-proxy writes before the tensor core's reads with a
        // proxy fence after its wait.
        auto publish_copies = [&](uint32_t mbar) { cp_async_arrive_noinc(mbar); };
        uint32_t g = 0;
        int k = 0;
        bool ok = !test_hook(1);
        for (int j = blockIdx.x; ok && j < total; j += gridDim.x, ++k) {
            if (__any_sync(kFullMask, *fail_flag != 0)) break;
            const Item it = decode_item(j, s_cu, s_ip, a.B, a.H);
            const int64_t seq_off = static_cast<int64_t>(it.start) * a.tok_stride +
                                    static_cast<int64_t>(it.h) * a.head_stride;
            const int qb = k & 1;
            if (k >= 2 && !warp_wait(q_empty(qb), ((k >> 1) - 1) & 1)) break;
            const uint32_t sq = sQ + qb * kQBytes;
            if (it.q0 + kRows <= it.len) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(q_full(qb), kQBytes);
                    tma_load_3d(sq, &tm_q, 0, it.h, it.start + it.q0, q_full(qb));
                } else {
                    mbar_arrive(q_full(qb));
                }
            } else {
                warp_load_rows<kRows>(sq, a.q + seq_off, a.tok_stride, it.q0, it.len, lane);
                publish_copies(q_full(qb));
            }
            for (int t = 0; t < it.nt; ++t, ++g) {
                const int s = static_cast<int>(g % S);
                if (g >= static_cast<uint32_t>(S) && !warp_wait(kv_empty(s), ((g / S) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const uint32_t sk = sRing + s * 2 * kKVTileBytes;
                const int r0 = t * kTileN;
                if (r0 + kTileN <= it.len) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(kv_full(s), 2 * kKVTileBytes);
                        tma_load_3d(sk, &tm_k, 0, it.h, it.start + r0, kv_full(s));
                        tma_load_3d(sk + kKVTileBytes, &tm_v, 0, it.h, it.start + r0, kv_full(s));
                    } else {
                        mbar_arrive(kv_full(s));
                    }
                } else {
                    warp_load_rows<kTileN>(sk, a.k + seq_off, a.tok_stride, r0, it.len, lane);
                    warp_load_rows<kTileN>(sk + kKVTileBytes, a.v + seq_off, a.tok_stride, r0, it.len, lane);
                    publish_copies(kv_full(s));
                }
            }
        }
        cp_async_wait_all();
        if (*fail_flag) {
            // Let the TMA loads still in flight land before the CTA can exit:
            // the newest tile of each ring stage and the newest Q loads.
            for (uint32_t x = g > static_cast<uint32_t>(S) ? g - S : 0; x < g; ++x) mbar_wait(kv_full(x % S), (x / S) & 1);
            for (int x = k > 2 ? k - 2 : 0; x < k; ++x) mbar_wait(q_full(x & 1), (x >> 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issue (one thread) ----------------
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc(Cvt<T>::kFormat, 0, kTileN);
            const uint32_t idesc_pv = make_idesc(Cvt<T>::kFormat, 1, 64);
            // P V of tile x (the first of its item when `first`, item index kk).
            // The stage of an item's last tile is released by the epilogue,
            // which stages O there.
            // P V of tile x of item kk: P sits in S buffer x & 1, O in buffer
            // kk & 1.  An item's first product overwrites its O buffer, which
            // the epilogue of item kk - 2 must have read out.
            auto issue_pv = [&](uint32_t x, bool first, bool last, int kk) {
                if (!mbar_wait(p_full(x & 3), (x >> 2) & 1)) return false;
                if (first && kk >= 2 && !mbar_wait(o_empty(kk & 1), ((kk >> 1) - 1) & 1)) return false;
                fence_after_sync();
                const uint32_t p_addr = tmem + (x & 1) * static_cast<uint32_t>(kTileN);
                const uint32_t o_addr = tmem + kOBufCol + (kk & 1) * 64u;
                const uint32_t sv = sRing + (x % S) * 2 * kKVTileBytes + kKVTileBytes;
#pragma unroll
                for (int part = 0; part < kParts; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16_ts(o_addr, p_addr + part * 32 + ks * 8, make_sdesc(sv + ks * 2048),
                                   idesc_pv, (first && part == 0 && ks == 0) ? 0u : 1u);
                mma_commit(pv_done(x & 1));
                if (!last) mma_commit(kv_empty(x % S));
                return true;
            };
            // Two walks over this CTA's tiles: Q K^T runs two tiles ahead of
            // P V.  P V(g) is issued as soon as P(g) is in TMEM, then Q K^T of
            // tile g + 2 into S buffer g & 1: the tensor core executes one
            // thread's MMAs in order, so P V(g) has read P(g) out of that
            // buffer before the new scores land in it.  The scores of tile
            // g + 1 are already there, so the softmax never waits for them.
            Walk wq(blockIdx.x, total, s_cu, s_ip, a.B, a.H);
            Walk wp = wq;
            uint32_t gq = 0;
            auto issue_qk = [&]() {
                const int qb = wq.k & 1;
                if (wq.t == 0 && !mbar_wait(q_full(qb), (wq.k >> 1) & 1)) return false;
                const int s = static_cast<int>(gq % S);
                if (!mbar_wait(kv_full(s), (gq / S) & 1)) return false;
                // Tiles filled by cp.async were written through the generic
                // proxy; order them before the tensor core's reads.
                fence_async_smem();
                fence_after_sync();
                const uint32_t d = tmem + (gq & 1) * static_cast<uint32_t>(kTileN);
                const uint32_t sq = sQ + qb * kQBytes;
                const uint32_t sk = sRing + s * 2 * kKVTileBytes;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(d, make_sdesc(sq + ks * 32), make_sdesc(sk + ks * 32), idesc_qk, ks > 0);
                mma_commit(s_full(gq & 1));
                if (wq.t == wq.it.nt - 1) mma_commit(q_empty(qb));
                ++gq;
                wq.next();
                return true;
            };
            bool ok = true;
            for (int i = 0; ok && i < 2 && wq.valid; ++i) ok = issue_qk();
            for (uint32_t gp = 0; ok && wp.valid; ++gp) {
                if (!issue_pv(gp, wp.t == 0, wp.t == wp.it.nt - 1, wp.k)) ok = false;
                else if (wq.valid && !issue_qk()) ok = false;
                wp.next();
            }
            if (!ok) atomicExch(&s_fail, 1);
            // Every MMA this thread issued has completed before TMEM is freed.
            mma_commit(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ---------------- softmax and epilogue (one thread per query row) ----------------
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        // Every product up to tile x has finished.  The phases of each pv_done
        // barrier are waited for one by one, in order: a parity wait is only
        // exact while the barrier is at most one phase behind the target.
        int pv_seen = -1;
        auto confirm_pv = [&](int x) {
            while (pv_seen < x) {
                ++pv_seen;
                if (!mbar_wait(pv_done(pv_seen & 1), (pv_seen >> 1) & 1)) {
                    atomicExch(&s_fail, 1);
                    pv_seen = x;
                }
            }
        };
        // Epilogue of item kk (its last tile gl, running sum lsum): once the
        // item's last product is done, the K/V stage of tile gl is no longer
        // read by anything (its release to the load warp is left to this
        // epilogue), so O / l is staged there: each thread writes its row
        // (swizzled 16-byte chunks), O buffer kk & 1 is released, and the four
        // warps store the tile four 128-byte rows per instruction.
        auto epilogue = [&](const Item& it, int kk, int gl, float lsum) {
            confirm_pv(gl);
            fence_after_sync();
            fence_async_smem();
            const int last_stage = gl % S;
            uint8_t* stage = smem_raw + (sRing - raw) + last_stage * 2 * kKVTileBytes;
            if (it.q0 + warp * 32 < it.len) {
                const float inv = 1.f / lsum;
                const uint64_t inv2 = f2(inv, inv);
                const uint32_t o_addr = t_lane + kOBufCol + (kk & 1) * 64u;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float ov[32];
                    tmem_ld32(o_addr + hf * 32, ov);
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float o0, o1;
                        f2_split(f2_mul(f2(ov[2 * i], ov[2 * i + 1]), inv2), o0, o1);
                        w[i] = Cvt<T>::pack(o0, o1);
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(stage + swz(tid, hf * 4 + c)) =
                            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                }
            }
            fence_before_sync();
            mbar_arrive(o_empty(kk & 1));
            mbar_arrive(o_staged);
            if (!mbar_wait(o_staged, kk & 1)) {
                atomicExch(&s_fail, 1);
                return false;
            }
            const int rows = min(kRows, it.len - it.q0);
            const int c = lane & 7;
            uint16_t* cls = a.cls_out != nullptr && it.q0 == 0
                                ? a.cls_out + (static_cast<int64_t>(it.b) * a.H + it.h) * 64
                                : nullptr;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = i * 16 + warp * 4 + (lane >> 3);
                if (r < rows) {
                    const uint4 val = *reinterpret_cast<const uint4*>(stage + swz(r, c));
                    *reinterpret_cast<uint4*>(a.out + static_cast<int64_t>(it.start + it.q0 + r) * a.out_tok_stride +
                                              it.h * 64 + c * 8) = val;
                    if (r == 0 && cls != nullptr) *reinterpret_cast<uint4*>(cls + c * 8) = val;
                }
            }
            // The stage goes back to the load warp once every read of it is done.
            fence_async_smem();
            mbar_arrive(o_stored);
            if (tid == 0) {
                if (mbar_wait(o_stored, kk & 1)) mbar_arrive(kv_empty(last_stage));
                else atomicExch(&s_fail, 1);
            }
            return true;
        };
        const uint64_t sl2 = f2(a.scale_log2, a.scale_log2);
        // The epilogue of an item runs after the first tile of the next one,
        // by when its last product has long finished.
        bool pending = false;
        Item p_it{};
        int p_k = 0, p_gl = 0;
        float p_l = 0.f;
        int g = 0;
        int k = 0;
        bool ok = true;
        for (int j = blockIdx.x; ok && j < total; j += gridDim.x, ++k) {
            if (*fail_flag) break;
            const Item it = decode_item(j, s_cu, s_ip, a.B, a.H);
            const bool warp_rows = it.q0 + warp * 32 < it.len;
            const uint32_t o_buf = t_lane + kOBufCol + (k & 1) * 64u;
            float m_ref = -INFINITY;   // reference maximum (log2 units) of this row
            float l0 = 0.f, l1 = 0.f;  // running sum, even / odd keys
            for (int t = 0; t < it.nt; ++t, ++g) {
                if (!mbar_wait(s_full(g & 1), (g >> 1) & 1)) {
                    atomicExch(&s_fail, 1);
                    ok = false;
                    break;
                }
                fence_after_sync();
                const uint32_t s_buf = t_lane + static_cast<uint32_t>((g & 1) * kTileN);
                if (warp_rows) {
                    float sv[64];
                    tmem_ld64(s_buf, sv);
                    const int valid = min(kTileN, it.len - t * kTileN);
                    if (valid < kTileN) {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            if (i >= valid) sv[i] = -INFINITY;
                    }
                    float mq[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float m = fmax3(sv[16 * c], sv[16 * c + 1], sv[16 * c + 2]);
#pragma unroll
                        for (int i = 3; i < 15; i += 2) m = fmax3(m, sv[16 * c + i], sv[16 * c + i + 1]);
                        mq[c] = fmaxf(m, sv[16 * c + 15]);
                    }
                    const float mt = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]) * a.scale_log2;
                    // Raise the reference only when the tile's maximum exceeds it
                    // by more than the threshold (always on the first tile).
                    const bool grow = mt > m_ref + kRescaleThreshold;
                    float alpha = 1.f;
                    if (grow) {
                        alpha = mma_attn::fast_exp2(m_ref - mt);
                        l0 *= alpha;
                        l1 *= alpha;
                        m_ref = mt;
                    }
                    if (t > 0 && __any_sync(kFullMask, grow)) {
                        // O holds the finished products of this item's tiles so far;
                        // 16 columns at a time, since sv is still live here.
                        confirm_pv(g - 1);
                        fence_after_sync();
                        const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            float part[16];
                            tmem_ld16(o_buf + q * 16, part);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                f2_split(f2_mul(f2(part[2 * i], part[2 * i + 1]), a2), part[2 * i], part[2 * i + 1]);
                            tmem_st16(o_buf + q * 16, part);
                        }
                    }
                    // P(g) replaces S(g) in its TMEM buffer: the product that
                    // read the buffer's previous P was issued, and so executed,
                    // before the scores that have just been read.
                    const uint64_t nm = f2(-m_ref, -m_ref);
                    uint64_t lsum = f2(l0, l1);
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t p_hi[16], p_lo[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int c = hf * 16 + i;
                            float x0, x1;
                            f2_split(f2_fma(f2(sv[2 * c], sv[2 * c + 1]), sl2, nm), x0, x1);
                            const float e0 = mma_attn::fast_exp2(x0), e1 = mma_attn::fast_exp2(x1);   // -inf -> 0
                            const uint64_t e = f2(e0, e1);
                            lsum = f2_add(lsum, e);
                            const uint32_t w = Cvt<T>::pack(e0, e1);
                            p_hi[i] = w;
                            if constexpr (kParts == 2) {
                                // bf16 -> fp32 is a 16-bit shift; the residual is rounded again.
                                float r0, r1;
                                f2_split(f2_sub(e, f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u))),
                                         r0, r1);
                                p_lo[i] = Cvt<T>::pack(r0, r1);
                            }
                        }
                        tmem_st16_u(s_buf + hf * 16, p_hi);
                        if constexpr (kParts == 2) tmem_st16_u(s_buf + 32 + hf * 16, p_lo);
                    }
                    f2_split(lsum, l0, l1);
                    tmem_wait_st();
                }
                // Every warp, rows or not, takes each pv_done phase while it is
                // the barrier's next one (products up to g - 2 are long done).
                // This comes before the arrival for tile g: after it, P V(g)
                // may complete and move barrier g & 1 one phase past g - 2.
                if (g >= 2) confirm_pv(g - 2);
                fence_before_sync();
                mbar_arrive(p_full(g & 3));
                if (t == 0 && pending) {
                    if (!epilogue(p_it, p_k, p_gl, p_l)) {
                        ok = false;
                        break;
                    }
                    pending = false;
                }
            }
            if (!ok || *fail_flag) break;
            pending = true;
            p_it = it;
            p_k = k;
            p_gl = g - 1;
            p_l = l0 + l1;
        }
        if (ok && pending && !*fail_flag) epilogue(p_it, p_k, p_gl, p_l);
    }

    fence_before_sync();
    __syncthreads();
    if (*fail_flag && tid == 0) raise_status(RAGGED_DEV_TIMEOUT);
    if (warp == 0) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kStreamTmemCols)
                     : "memory");
    }
}

}  // namespace tc05
}  // namespace ragged
