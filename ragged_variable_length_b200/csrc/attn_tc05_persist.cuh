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
// prefix of H * ceil(L_b / 128) over the sequences, and decodes its own items
// (blockIdx.x, blockIdx.x + gridDim.x, ...) once into a list of packed words,
// so that each role reads its next item with one shared-memory load; two CTAs
// share an SM.  TMEM (256 columns: S of three tiles, each overwritten in
// place by its P, and O) and the mbarriers are set up once per CTA, so the
// per-launch fixed costs of a CTA (cu_seqlens read, TMEM allocation, first
// loads) are paid once, and the loads of the next item run under the softmax
// of the current one.
//
// Warp roles; they hand off through mbarriers only:
//   warp 5     loads.  Full tiles by TMA from 3-D tensor maps over
//              [rows, head, 64] with the 128-byte swizzle, which is the
//              canonical SWIZZLE_128B operand layout of tcgen05; partial tiles
//              (the last rows of a sequence) by cp.async with zero fill, each
//              lane's arrival triggered by the completion of its copies
//              (cp.async.mbarrier.arrive.noinc).  Q is double-buffered; K and
//              V flow through separate rings (3 and 5 stages), each stage
//              handed back by the completion of the product that read it.
//   warp 4     one thread issues every tcgen05.mma.  Q K^T runs three tiles
//              ahead of P V: P V(g) as soon as P(g) is in TMEM, then S of tile
//              g + 3 into TMEM buffer g % 3 (in order behind P V(g), which
//              read P(g) from it).  Across items the walks simply continue.
//   warps 0-3  softmax, one thread per query row (TMEM lane = row), single
//              pass with a reference maximum that is raised (and the running
//              sum and O rescaled) only when a tile exceeds it by more than
//              2^8; P (bf16: hi and lo parts) replaces S in its TMEM buffer.
//              The pairwise fp32 work uses the packed f32x2 instructions of
//              sm_100.  An item's epilogue (O / l and the CLS row) runs at the
//              first tile of the next item, before that tile's P is handed
//              over (its product overwrites O): each thread reads its row of
//              O from TMEM and stores it with 32-byte stores.
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
// TMEM per CTA (256 columns): S of three tiles at [0, 64), [64, 128) and
// [128, 192), each overwritten in place by its P (16-bit pairs; bf16 as hi +
// lo halves), and O at [192, 256).
constexpr int kSBufs = 3;
// K tiles are read once, by the Q K^T of their tile, and V tiles by its P V,
// kSBufs tiles later: K and V flow through separate rings.  K stage g % kSBufs
// is refilled once the Q K^T of tile g - kSBufs has finished, which the scores
// barrier of the same index reports (its next phase needs the new K tile, so
// a parity wait on it is exact); V stage g % 5 once the P V of tile g - 5 has.
constexpr int kKStages = kSBufs;
constexpr int kVStages = 5;
constexpr uint32_t kOCol = kSBufs * 64;
constexpr int kPersistMaxB = 1024;   // cu_seqlens and item offsets live in shared memory
// Each CTA decodes its own work items once, into shared memory (one packed
// word each: sequence, head, query tile), so that every role reads an item
// with a single shared-memory load instead of a binary search.
constexpr int kPersistMaxItems = 1024;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr uint32_t kFullMask = 0xffffffffu;

// Dynamic shared memory: alignment slack, two Q buffers, the K ring, the V
// ring, cu_seqlens and the item offsets (B + 1 ints each), then the CTA's
// item list (items_cap words).
__host__ __device__ constexpr int persist_smem_bytes(int B, int items_cap) {
    return 1024 + 2 * kQBytes + (kKStages + kVStages) * kKVTileBytes + 2 * (B + 1) * 4 + items_cap * 4;
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
    int items_cap;   // at least the number of items of any CTA
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

// An item packed into one word: sequence (11 bits), head (10), query tile (11).
__device__ __forceinline__ uint32_t pack_item(const Item& it) {
    return static_cast<uint32_t>(it.b) | (static_cast<uint32_t>(it.h) << 11) |
           (static_cast<uint32_t>(it.q0 / kRows) << 21);
}
__device__ __forceinline__ Item unpack_item(uint32_t w, const int* s_cu) {
    Item it;
    it.b = static_cast<int>(w & 2047u);
    it.h = static_cast<int>((w >> 11) & 1023u);
    it.q0 = static_cast<int>(w >> 21) * kRows;
    it.start = s_cu[it.b];
    it.len = s_cu[it.b + 1] - it.start;
    it.nt = (it.len + kTileN - 1) / kTileN;
    return it;
}

// Cursor over the tiles of a CTA's items: its k-th item, key tile t of it.
struct Walk {
    int k, t, n;
    bool valid;
    Item it;
    const uint32_t* items;
    const int* s_cu;
    __device__ __forceinline__ Walk(int n_, const uint32_t* items_, const int* cu)
        : k(0), t(0), n(n_), valid(n_ > 0), items(items_), s_cu(cu) {
        if (valid) it = unpack_item(items[0], s_cu);
    }
    __device__ __forceinline__ void next() {
        if (++t < it.nt) return;
        t = 0;
        ++k;
        valid = k < n;
        if (valid) it = unpack_item(items[k], s_cu);
    }
};

template <typename T>
__global__ void __launch_bounds__(kPersistThreads, 2)
    attn_tc05_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const PersistArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // kv_full[3], q_full[2], q_empty[2], s_full[kSBufs], p_full[4], pv_done[5], drain
    __shared__ __align__(8) uint64_t s_bar[17 + kSBufs];
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kParts = Cvt<T>::kParts;

    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sQ = (raw + 1023u) & ~1023u;     // Q buffer i at sQ + i * 16 KB
    const uint32_t sK = sQ + 2 * kQBytes;           // K stage s at sK + s * 8 KB
    const uint32_t sV = sK + kKStages * kKVTileBytes;   // V stage s at sV + s * 8 KB
    int* s_cu = reinterpret_cast<int*>(smem_raw + (sV - raw) + kVStages * kKVTileBytes);
    int* s_ip = s_cu + (a.B + 1);
    uint32_t* s_items = reinterpret_cast<uint32_t*>(s_ip + (a.B + 1));

    const uint32_t bar0 = smem_addr(&s_bar[0]);
    // K and V of tile g have landed (g % 3; a K stage is refilled only after the
    // Q K^T that read it, so a tile three ahead cannot reach the barrier first).
    auto kv_full = [&](int i) { return bar0 + 8u * i; };
    auto q_full = [&](int i) { return bar0 + 8u * (3 + i); };
    auto q_empty = [&](int i) { return bar0 + 8u * (5 + i); };
    // S of tile g is in TMEM buffer g % 3; the same completion frees K stage g % 3.
    auto s_full = [&](int i) { return bar0 + 8u * (7 + i); };
    // P of tile g is in TMEM (g & 3): warps with no rows in the current query
    // tile skip the softmax and can run up to three tiles ahead of a warp
    // that has rows (Q K^T of tile g waits for P of tile g - 3), so four tiles
    // in a row must not share a barrier.
    auto p_full = [&](int i) { return bar0 + 8u * (7 + kSBufs + i); };
    // P V of tile g has finished (g % 5); the same completion frees V stage g % 5.
    auto pv_done = [&](int i) { return bar0 + 8u * (11 + kSBufs + i); };
    const uint32_t drain = bar0 + 8u * (16 + kSBufs);
    volatile int* fail_flag = &s_fail;

    // ---- setup: cu_seqlens, barriers, TMEM, item offsets ----
    for (int i = tid; i <= a.B; i += kPersistThreads) s_cu[i] = __ldg(a.cu + i);
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(kv_full(i), 32);
        for (int i = 0; i < kSBufs; ++i) mbar_init(s_full(i), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(q_full(i), 32);
            mbar_init(q_empty(i), 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(p_full(i), kSoftmaxThreads);
        for (int i = 0; i < 5; ++i) mbar_init(pv_done(i), 1);
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
    // Item offsets: s_ip[b] = items of the sequences before b.  Every thread
    // takes a contiguous run of at most six sequences (B <= 1024), and the run
    // totals are scanned across the block (a warp scan, then the six warp
    // totals), so the scan takes a few shared-memory round trips whatever B
    // is; one warp walking 32 sequences at a time took ~3 us at B = 512.
    {
        constexpr int kWarps = kPersistThreads / 32;
        __shared__ int s_wsum[kWarps];
        const int per = (a.B + kPersistThreads - 1) / kPersistThreads;
        const int b0 = min(a.B, tid * per), b1 = min(a.B, b0 + per);
        int n[(kPersistMaxB + kPersistThreads - 1) / kPersistThreads];
        int run = 0;
#pragma unroll
        for (int i = 0; i < (kPersistMaxB + kPersistThreads - 1) / kPersistThreads; ++i) {
            const int b = b0 + i;
            n[i] = 0;
            if (b < b1) {
                const int st = s_cu[b], len = s_cu[b + 1] - st;
                // The tensor maps cover rows [0, B * max_seqlen): a sequence
                // reaching past them (cu[0] != 0 can shift one there) would
                // read zero fill, so it is flagged and skipped like the rest.
                if (st < 0 || len < 0 || len > a.max_seqlen ||
                    static_cast<int64_t>(st) + len > static_cast<int64_t>(a.B) * a.max_seqlen)
                    raise_status(RAGGED_DEV_BAD_SEQLENS);
                else
                    n[i] = ((len + kRows - 1) / kRows) * a.H;
                run += n[i];
            }
        }
        int incl = run;   // inclusive scan of the run totals within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFullMask, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int before = incl - run;
        for (int w = 0; w < warp; ++w) before += s_wsum[w];
        if (tid == 0) s_ip[0] = 0;
#pragma unroll
        for (int i = 0; i < (kPersistMaxB + kPersistThreads - 1) / kPersistThreads; ++i) {
            const int b = b0 + i;
            if (b < b1) {
                before += n[i];
                s_ip[b + 1] = before;
            }
        }
    }
    __syncthreads();
    // This CTA's items (blockIdx.x, blockIdx.x + gridDim.x, ...), decoded once.
    const int total = s_ip[a.B];
    int n_items = static_cast<int>(blockIdx.x) < total ? (total - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
    if (n_items > a.items_cap) {   // the host sizes items_cap from B, H and max_seqlen; never reached
        if (tid == 0) raise_status(RAGGED_DEV_BAD_SEQLENS);
        n_items = 0;
    }
    for (int k = tid; k < n_items; k += kPersistThreads)
        s_items[k] = pack_item(decode_item(static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), s_cu, s_ip,
                                           a.B, a.H));
    __syncthreads();
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
        for (; ok && k < n_items; ++k) {
            if (__any_sync(kFullMask, *fail_flag != 0)) break;
            const Item it = unpack_item(s_items[k], s_cu);
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
                // K stage g % 3 is free once the Q K^T of tile g - 3 has
                // finished, V stage g % 5 once the P V of tile g - 5 has.
                if (g >= static_cast<uint32_t>(kKStages) &&
                    !warp_wait(s_full(g % kSBufs), ((g - kKStages) / kSBufs) & 1)) {
                    ok = false;
                    break;
                }
                if (g >= static_cast<uint32_t>(kVStages) &&
                    !warp_wait(pv_done(g % kVStages), ((g - kVStages) / kVStages) & 1)) {
                    ok = false;
                    break;
                }
                const uint32_t sk = sK + (g % kKStages) * kKVTileBytes;
                const uint32_t sv = sV + (g % kVStages) * kKVTileBytes;
                const uint32_t full = kv_full(g % kKStages);
                const int r0 = t * kTileN;
                if (r0 + kTileN <= it.len) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(full, 2 * kKVTileBytes);
                        tma_load_3d(sk, &tm_k, 0, it.h, it.start + r0, full);
                        tma_load_3d(sv, &tm_v, 0, it.h, it.start + r0, full);
                    } else {
                        mbar_arrive(full);
                    }
                } else {
                    warp_load_rows<kTileN>(sk, a.k + seq_off, a.tok_stride, r0, it.len, lane);
                    warp_load_rows<kTileN>(sv, a.v + seq_off, a.tok_stride, r0, it.len, lane);
                    publish_copies(full);
                }
            }
        }
        cp_async_wait_all();
        if (*fail_flag) {
            // Let the TMA loads still in flight land before the CTA can exit:
            // the newest tile of each K/V barrier and the newest Q loads.
            for (uint32_t x = g > static_cast<uint32_t>(kKStages) ? g - kKStages : 0; x < g; ++x)
                mbar_wait(kv_full(x % kKStages), (x / kKStages) & 1);
            for (int x = k > 2 ? k - 2 : 0; x < k; ++x) mbar_wait(q_full(x & 1), (x >> 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issue (one thread) ----------------
        if (lane == 0) {
            const uint32_t idesc_qk = make_idesc(Cvt<T>::kFormat, 0, kTileN);
            const uint32_t idesc_pv = make_idesc(Cvt<T>::kFormat, 1, 64);
            // P V of tile x: P sits in S buffer x % 3; the item's first
            // product overwrites O, which the softmax warps have read out for
            // the item before (they do so before handing over this tile's P).
            auto issue_pv = [&](uint32_t x, bool first) {
                if (!mbar_wait(p_full(x & 3), (x >> 2) & 1)) return false;
                fence_after_sync();
                const uint32_t p_addr = tmem + (x % kSBufs) * static_cast<uint32_t>(kTileN);
                const uint32_t o_addr = tmem + kOCol;
                const uint32_t sv = sV + (x % kVStages) * kKVTileBytes;
#pragma unroll
                for (int part = 0; part < kParts; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16_ts(o_addr, p_addr + part * 32 + ks * 8, make_sdesc(sv + ks * 2048),
                                   idesc_pv, (first && part == 0 && ks == 0) ? 0u : 1u);
                mma_commit(pv_done(x % kVStages));
                return true;
            };
            // Two walks over this CTA's tiles: Q K^T runs three tiles ahead
            // of P V.  P V(g) is issued as soon as P(g) is in TMEM, then Q K^T
            // of tile g + 3 into S buffer g % 3: the tensor core executes one
            // thread's MMAs in order, so P V(g) has read P(g) out of that
            // buffer before the new scores land in it.  The scores of tiles
            // g + 1 and g + 2 are already there.
            Walk wq(n_items, s_items, s_cu);
            Walk wp = wq;
            uint32_t gq = 0;
            auto issue_qk = [&]() {
                const int qb = wq.k & 1;
                if (wq.t == 0 && !mbar_wait(q_full(qb), (wq.k >> 1) & 1)) return false;
                if (!mbar_wait(kv_full(gq % kKStages), (gq / kKStages) & 1)) return false;
                // Tiles filled by cp.async were written through the generic
                // proxy; order them before the tensor core's reads.
                fence_async_smem();
                fence_after_sync();
                const uint32_t d = tmem + (gq % kSBufs) * static_cast<uint32_t>(kTileN);
                const uint32_t sk = sK + (gq % kKStages) * kKVTileBytes;
                const uint32_t sq = sQ + qb * kQBytes;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(d, make_sdesc(sq + ks * 32), make_sdesc(sk + ks * 32), idesc_qk, ks > 0);
                mma_commit(s_full(gq % kSBufs));
                if (wq.t == wq.it.nt - 1) mma_commit(q_empty(qb));
                ++gq;
                wq.next();
                return true;
            };
            bool ok = true;
            for (int i = 0; ok && i < kSBufs && wq.valid; ++i) ok = issue_qk();
            for (uint32_t gp = 0; ok && wp.valid; ++gp) {
                if (!issue_pv(gp, wp.t == 0)) ok = false;
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
        const uint32_t o_lane = t_lane + kOCol;
        // Every product up to tile x has finished.  The phases of each pv_done
        // barrier are waited for one by one, in order: a parity wait is only
        // exact while the barrier is at most one phase behind the target.
        int pv_seen = -1;
        auto confirm_pv = [&](int x) {
            while (pv_seen < x) {
                ++pv_seen;
                if (!mbar_wait(pv_done(pv_seen % kVStages), (pv_seen / kVStages) & 1)) {
                    atomicExch(&s_fail, 1);
                    pv_seen = x;
                }
            }
        };
        // This thread's row of O / l, packed to 16-bit pairs, once every
        // product of the item ending at tile gl has finished.
        auto read_o = [&](int gl, float lsum, uint32_t (&w)[32]) {
            confirm_pv(gl);
            fence_after_sync();
            const float inv = 1.f / lsum;
            const uint64_t inv2 = f2(inv, inv);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float ov[32];
                tmem_ld32(o_lane + hf * 32, ov);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float o0, o1;
                    f2_split(f2_mul(f2(ov[2 * i], ov[2 * i + 1]), inv2), o0, o1);
                    w[hf * 16 + i] = Cvt<T>::pack(o0, o1);
                }
            }
        };
        // Row tid of the item to out (and to cls_out for row 0 of a
        // sequence), eight 16-byte stores.
        auto store_o = [&](const Item& it, const uint32_t (&w)[32]) {
            const int r = it.q0 + tid;
            if (r >= it.len) return;
            uint16_t* dst = a.out + static_cast<int64_t>(it.start + r) * a.out_tok_stride + it.h * 64;
            // 32-byte stores need 32-byte aligned rows (a row stride of a
            // multiple of 16 elements); 16-byte stores otherwise.  A warp's
            // store instruction then writes 32 whole sectors instead of 32
            // half sectors.
            if ((a.out_tok_stride & 15) == 0 && (reinterpret_cast<uintptr_t>(a.out) & 31) == 0) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + c * 16),
                                 "r"(w[8 * c]), "r"(w[8 * c + 1]), "r"(w[8 * c + 2]), "r"(w[8 * c + 3]),
                                 "r"(w[8 * c + 4]), "r"(w[8 * c + 5]), "r"(w[8 * c + 6]), "r"(w[8 * c + 7])
                                 : "memory");
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(dst + c * 8) =
                        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            }
            if (a.cls_out != nullptr && r == 0) {
                uint16_t* cls = a.cls_out + (static_cast<int64_t>(it.b) * a.H + it.h) * 64;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(cls + c * 8) =
                        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            }
        };
        const uint64_t sl2 = f2(a.scale_log2, a.scale_log2);
        // The epilogue of an item runs at the first tile of the next one,
        // before that tile's P is handed over (the next product overwrites O).
        bool pending = false;
        Item p_it{};
        int p_gl = 0;
        float p_l = 0.f;
        int g = 0;
        bool ok = true;
        for (int k = 0; ok && k < n_items; ++k) {
            const Item it = unpack_item(s_items[k], s_cu);
            const bool warp_rows = it.q0 + warp * 32 < it.len;
            float m_ref = -INFINITY;   // reference maximum (log2 units) of this row
            float l0 = 0.f, l1 = 0.f;  // running sum, even / odd keys
            for (int t = 0; t < it.nt; ++t, ++g) {
                if (!mbar_wait(s_full(g % kSBufs), (g / kSBufs) & 1)) {
                    atomicExch(&s_fail, 1);
                    ok = false;
                    break;
                }
                fence_after_sync();
                const uint32_t s_buf = t_lane + static_cast<uint32_t>((g % kSBufs) * kTileN);
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
                            tmem_ld16(o_lane + q * 16, part);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                f2_split(f2_mul(f2(part[2 * i], part[2 * i + 1]), a2), part[2 * i], part[2 * i + 1]);
                            tmem_st16(o_lane + q * 16, part);
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
                if (t == 0 && pending) {
                    // The previous item's O, read out and stored before this
                    // tile's P is handed over: its first product overwrites O.
                    if (p_it.q0 + warp * 32 < p_it.len) {
                        uint32_t ow[32];
                        read_o(p_gl, p_l, ow);
                        store_o(p_it, ow);
                    } else {
                        confirm_pv(p_gl);
                    }
                    pending = false;
                }
                // Every warp, rows or not, takes each pv_done phase while it is
                // the barrier's next one (products up to g - 2 are long done).
                // This comes before the arrival for tile g: after it, P V(g)
                // may complete and move barrier g % 5 one phase past g - 5.
                if (g >= 2) confirm_pv(g - 2);
                fence_before_sync();
                mbar_arrive(p_full(g & 3));
            }
            if (!ok || *fail_flag) break;
            pending = true;
            p_it = it;
            p_gl = g - 1;
            p_l = l0 + l1;
        }
        if (ok && pending && !*fail_flag && p_it.q0 + warp * 32 < p_it.len) {
            uint32_t ow[32];
            read_o(p_gl, p_l, ow);
            store_o(p_it, ow);
        }
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
