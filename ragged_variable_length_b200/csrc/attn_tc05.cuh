// Ragged bidirectional attention on the 5th-generation tensor cores
// (tcgen05.mma with TMEM accumulators), f16 / bf16, head_dim 64: the shared
// tcgen05 / TMEM / mbarrier helpers and the per-tile streaming kernel.
//
// Operation ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
// abstract; radpulse section "Bypassing the binding"): per sequence b and head
// h, O = softmax(scale Q K^T) V over the sequence's own rows.
//
// Shared-memory operand tiles use the 128-byte XOR swizzle of mma_attn::swz,
// which is the canonical SWIZZLE_128B layout of tcgen05 (K-major for Q, K and
// P; MN-major for V; 8-row groups 1024 bytes apart).  Every mbarrier wait is
// bounded; a wait that gives up sets RAGGED_DEV_TIMEOUT in the status word and
// the CTA skips to its teardown (TMEM is always freed).
#pragma once

#include "attn_resident.cuh"

namespace ragged {
namespace tc05 {

using mma_attn::swz;
using resident::PackedRows;

constexpr int kRows = 128;            // query rows per CTA (MMA M)
constexpr int kTileN = 64;            // keys per tile
constexpr int kQBytes = kRows * 128;               // 16 KB
constexpr int kKVTileBytes = kTileN * 128;         // 8 KB
constexpr uint32_t kSpinLimit = 1u << 22;

#ifdef RAGGED_TEST_HOOKS
// Test builds only (libragged_testhooks.so, never the product library): a
// test can shorten every bounded wait and tell a kernel's producer to issue
// nothing, so that the waits on it expire without any fault, and then check
// that the status word reports it, TMEM comes back and the next launch is
// exact.  g_test_hook: 1 = the persistent kernel's load warp issues no load;
// 2 = the per-tile kernel's MMA thread issues no product.
__device__ uint32_t g_test_spin_limit = kSpinLimit;
__device__ int g_test_hook = 0;
__device__ __forceinline__ uint32_t spin_limit() { return g_test_spin_limit; }
__device__ __forceinline__ bool test_hook(int which) { return g_test_hook == which; }
#else
__device__ __forceinline__ constexpr uint32_t spin_limit() { return kSpinLimit; }
__device__ __forceinline__ constexpr bool test_hook(int) { return false; }
#endif

// ---- instruction and shared-memory descriptors -------------------------------

// kind::f16 instruction descriptor: fp32 accumulate, A/B format (0 = f16,
// 1 = bf16), A K-major, B K-major (0) or MN-major (1), M = 128, N.
__device__ __forceinline__ uint32_t make_idesc(uint32_t ab_format, uint32_t b_mn_major, uint32_t n) {
    return (1u << 4)                  // D format: f32
           | (ab_format << 7)         // A format
           | (ab_format << 10)        // B format
           | (b_mn_major << 16)       // B major
           | ((n >> 3) << 17)         // N / 8
           | ((kRows >> 4) << 24);    // M / 16
}

// Shared-memory matrix descriptor for a 128-byte-swizzled tile whose 8-row
// groups are 1024 bytes apart (both the K-major and the MN-major forms used
// here); base must sit in a 1024-byte aligned atom.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t smem_byte_addr) {
    return static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFFu)     // start address
           | (static_cast<uint64_t>(1) << 16)                          // leading byte offset (unused)
           | (static_cast<uint64_t>(1024 >> 4) << 32)                  // stride byte offset
           | (static_cast<uint64_t>(1) << 46)                          // descriptor version
           | (static_cast<uint64_t>(2) << 61);                         // SWIZZLE_128B
}

// ---- tcgen05 / mbarrier wrappers -------------------------------------------

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

// Waits for the phase with the given parity to complete; false after the
// bounded number of polls.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
    const uint32_t limit = spin_limit();
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    // The load and its wait sit in one statement so no use of r can be
    // scheduled before the data has arrived.
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Stores 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
        "tcgen05.wait::st.sync.aligned;\n"
        :
        : "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15]))
        : "memory");
}

// exp2 for the rescale factor; exp2(-inf) = 0 (a row with no reference yet).
__device__ __forceinline__ float fast_exp2_guard(float x) { return mma_attn::fast_exp2(x); }

template <typename T>
struct Cvt;
template <>
struct Cvt<__half> {
    static constexpr uint32_t kFormat = 0;
    static constexpr int kParts = 1;
    __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};
template <>
struct Cvt<__nv_bfloat16> {
    static constexpr uint32_t kFormat = 1;
    static constexpr int kParts = 2;   // P = hi + lo
    __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

// ---------------------------------------------------------------------------
// Per-tile streaming kernel: one CTA per (128-query tile, head, sequence),
// two CTAs per SM.
//
// The K/V tiles of a sequence flow through a 5-stage shared-memory ring (loads
// run four tiles ahead), and the probabilities never touch shared memory:
// each softmax thread stores its row of P into TMEM (16-bit values packed two
// per column, row = lane) and the P V product reads its A operand from TMEM.  TMEM per CTA (256 columns):
//   [0, 64) and [64, 128)   S of tiles t (even / odd)
//   [128, 192)              P: two f16 slots of 32 columns, or the bf16 hi/lo pair
//   [192, 256)              O
// so two CTAs share each SM.  S = Q K^T of tile t + 1 is issued before the
// softmax of tile t.  The softmax is single-pass: each row keeps a reference
// maximum and rescales its running sum and O (in TMEM) only when a tile
// raises the row maximum by more than 2^8 in base 2; otherwise the
// probabilities exp2(s - reference) stay below 256 and the reference is kept.
// The final division by the running sum makes the result independent of the
// reference.  Warps whose 32 query rows all lie past the sequence end skip
// the softmax; fully-masked 16-key groups of the last tile are skipped too.
// ---------------------------------------------------------------------------

constexpr uint32_t kStreamTmemCols = 256;
constexpr uint32_t kStreamPCol = 128;
constexpr uint32_t kStreamOCol = 192;
constexpr int kStages = 5;
constexpr float kRescaleThreshold = 8.f;       // log2 units

__host__ __device__ constexpr int stream_smem_bytes(int /*p_parts*/) {
    return 1024 + kQBytes + kStages * 2 * kKVTileBytes;   // alignment slack, Q, K/V ring
}

// 32 consecutive 32-bit TMEM columns of this thread's lane <- v.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
        :
        : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
          "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
          "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 64 consecutive fp32 columns of this thread's TMEM lane, one load and one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}



// O (TMEM) += P (TMEM, A operand) x V (shared memory, B operand).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
        :
        : "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}

// Warp roles: warps 0-3 (128 threads, one per query row) load K/V tiles with
// cp.async and run the softmax; warp 4 issues every tcgen05.mma.  They hand
// off through mbarriers only, so no CTA-wide barrier sits in the tile loop:
//   kv_ready[stage]  (128 arrivals) the tile in that ring stage has landed and
//                    is visible to the tensor core;
//   s_ready[t & 1]   (commit)       S of tile t is in TMEM;
//   p_ready[t & 1]   (128 arrivals) P of tile t is in TMEM and S of tile t has
//                    been read, so that S buffer may be overwritten;
//   pv_done[t & 1]   (commit)       the P V product of tile t (and everything
//                    issued before it) has finished.
// The MMA warp issues Q K^T(t) as soon as tile t has landed, then P V(t - 1)
// once P(t - 1) is ready, so the S of the next tile is always computed while
// the softmax of the current one runs.
constexpr int kStreamThreads = 160;
constexpr int kSoftmaxThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kStreamThreads, 2)
    attn_tc05_stream_kernel(PackedRows src, float scale_log2, int H, uint16_t* __restrict__ out,
                            int64_t out_tok_stride, uint16_t* __restrict__ cls_out) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t s_kv_ready[kStages];
    __shared__ __align__(8) uint64_t s_s_ready[2];
    __shared__ __align__(8) uint64_t s_p_ready[2];
    __shared__ __align__(8) uint64_t s_pv_done[2];
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;

    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    if (!src.begin(b, h, nullptr, nullptr)) return;
    const int len = src.len, start = src.start;
    const int q0 = qt * kRows;
    if (q0 >= len) return;
    const int nt = (len + kTileN - 1) / kTileN;
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool mma_warp = warp == 4;
    constexpr int kParts = Cvt<T>::kParts;

    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sQ = (raw + 1023u) & ~1023u;
    const uint32_t sRing = sQ + kQBytes;                         // stage s: K at +s*16K, V at +8K
    auto stage_k = [&](int t) { return sRing + (t % kStages) * 2 * kKVTileBytes; };
    auto stage_v = [&](int t) { return stage_k(t) + kKVTileBytes; };
    auto load_kv = [&](int t) {
        resident::load_tile<kTileN>(stage_k(t), src, 1, t * kTileN, len);
        resident::load_tile<kTileN>(stage_v(t), src, 2, t * kTileN, len);
        cp_async_commit();
    };

    // Loads by the softmax threads: group 0 = Q + tile 0, then one group per
    // tile, up to four ahead.
    int issued = min(nt, kStages - 1);
    if (!mma_warp) {
        resident::load_tile<kRows>(sQ, src, 0, q0, len);
        for (int t = 0; t < issued; ++t) load_kv(t);
    }

    const uint32_t kv_ready0 = smem_addr(&s_kv_ready[0]);
    const uint32_t s_ready0 = smem_addr(&s_s_ready[0]);
    const uint32_t p_ready0 = smem_addr(&s_p_ready[0]);
    const uint32_t pv_done0 = smem_addr(&s_pv_done[0]);
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(kv_ready0 + 8 * i, kSoftmaxThreads);
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_ready0 + 8 * i, 1);
            mbar_init(p_ready0 + 8 * i, kSoftmaxThreads);
            mbar_init(pv_done0 + 8 * i, 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_fail = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem)),
                     "r"(kStreamTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = s_tmem;

    // Event waits; an event is awaited only while the next event on the same
    // barrier cannot have completed yet, so a parity wait never misses a phase.
    auto wait_event = [&](uint32_t mbar, uint32_t parity) {
        if (!mbar_wait(mbar, parity)) atomicExch(&s_fail, 1);
    };
    auto arrive = [&](uint32_t mbar) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
    };

    if (mma_warp) {
        // ---------------- MMA issuer (one thread) ----------------
        if ((tid & 31) == 0 && !test_hook(2)) {
            const uint32_t idesc_qk = make_idesc(Cvt<T>::kFormat, 0, kTileN);
            const uint32_t idesc_pv = make_idesc(Cvt<T>::kFormat, 1, 64);
            auto issue_pv = [&](int t) {   // P V of tile t, once P(t) is ready
                wait_event(p_ready0 + 8 * (t & 1), (t >> 1) & 1);
                fence_after_sync();
                const uint32_t p_addr = tmem + kStreamPCol + (kParts == 2 ? 0u : static_cast<uint32_t>((t & 1) * 32));
#pragma unroll
                for (int part = 0; part < kParts; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16_ts(tmem + kStreamOCol, p_addr + part * 32 + ks * 8,
                                   make_sdesc(stage_v(t) + ks * 2048), idesc_pv,
                                   (t > 0 || part > 0 || ks > 0) ? 1u : 0u);
                mma_commit(pv_done0 + 8 * (t & 1));
            };
            for (int t = 0; t < nt && !s_fail; ++t) {
                // Q K^T(t): the tile has landed, and S buffer t & 1 was released by
                // p_ready(t - 2), which issue_pv(t - 2) has already waited for.
                wait_event(kv_ready0 + 8 * (t % kStages), (t / kStages) & 1);
                fence_after_sync();
                const uint32_t d = tmem + static_cast<uint32_t>((t & 1) * kTileN);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16(d, make_sdesc(sQ + ks * 32), make_sdesc(stage_k(t) + ks * 32), idesc_qk, ks > 0);
                mma_commit(s_ready0 + 8 * (t & 1));
                if (t >= 1) issue_pv(t - 1);
            }
            if (!s_fail) issue_pv(nt - 1);
        }
    } else {
        // ---------------- loads + softmax (one thread per query row) ----------------
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const int row = q0 + tid;
        const bool warp_rows = q0 + warp * 32 < len;
        constexpr int kPLag = kParts == 2 ? 1 : 2;
        int pv_seen = -1;
        auto confirm_pv = [&](int x) {
            if (x > pv_seen) {
                wait_event(pv_done0 + 8 * (x & 1), (x >> 1) & 1);
                pv_seen = x;
            }
        };
        // Publish tile t (its copies, and every earlier group, have landed).
        auto publish = [&](int t) {
            resident::cp_async_wait_pending(issued - 1 - t);
            fence_async_smem();
            arrive(kv_ready0 + 8 * (t % kStages));
        };
        publish(0);

        float m_ref = -INFINITY;   // reference maximum (log2 units) of this row
        float l = 0.f;
        for (int t = 0; t < nt; ++t) {
            if (s_fail) break;
            // Refill the ring: the stage of tile x is free once P V(x) is done.
            if (issued < nt && issued - kStages <= t - kPLag) {
                if (t >= kPLag) confirm_pv(t - kPLag);
                load_kv(issued);
                ++issued;
            }
            // Let the MMA warp start Q K^T(t + 1) while this tile's softmax runs.
            if (t + 1 < nt) publish(t + 1);

            wait_event(s_ready0 + 8 * (t & 1), (t >> 1) & 1);
            fence_after_sync();
            const int valid = min(kTileN, len - t * kTileN);
            if (warp_rows) {
                float sv[64];
                tmem_ld64(t_lane + static_cast<uint32_t>((t & 1) * kTileN), sv);
                if (valid < kTileN) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (i >= valid) sv[i] = -INFINITY;
                }
                float mx = -INFINITY;
#pragma unroll
                for (int i = 0; i < 64; ++i) mx = fmaxf(mx, sv[i]);
                // Rescale only when the tile's maximum exceeds the reference by
                // more than the threshold (always for the first tile).
                const float mt = mx * scale_log2;
                const bool grow = mt > m_ref + kRescaleThreshold;
                float alpha = 1.f;
                if (grow) {
                    alpha = fast_exp2_guard(m_ref - mt);
                    l *= alpha;
                    m_ref = mt;
                }
                if (t > 0 && __any_sync(0xffffffffu, grow)) {
                    // O must hold the finished products of tiles 0 .. t - 1.
                    confirm_pv(t - 1);
                    fence_after_sync();
                    float ov[64];
                    tmem_ld64(t_lane + kStreamOCol, ov);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float part[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) part[i] = ov[g * 16 + i] * alpha;
                        tmem_st16(t_lane + kStreamOCol + g * 16, part);
                    }
                }
                uint32_t p_hi[32], p_lo[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float a = mma_attn::fast_exp2(fmaf(sv[2 * i], scale_log2, -m_ref));   // -inf -> 0
                    const float c = mma_attn::fast_exp2(fmaf(sv[2 * i + 1], scale_log2, -m_ref));
                    l += a + c;
                    const uint32_t w = Cvt<T>::pack(a, c);
                    p_hi[i] = w;
                    if constexpr (kParts == 2) {
                        __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162*>(&w);
                        const float2 f = __bfloat1622float2(hb);
                        p_lo[i] = Cvt<T>::pack(a - f.x, c - f.y);
                    }
                }
                // The P slot is free once the product that last read it is done.
                if (t >= kPLag) confirm_pv(t - kPLag);
                fence_after_sync();
                const uint32_t p_col = t_lane + kStreamPCol + (kParts == 2 ? 0u : static_cast<uint32_t>((t & 1) * 32));
                tmem_st32(p_col, p_hi);
                if constexpr (kParts == 2) tmem_st32(p_col + 32, p_lo);
                tmem_wait_st();
            }
            fence_before_sync();
            arrive(p_ready0 + 8 * (t & 1));
        }

        // Epilogue: wait for the last product, O / l.
        if (!s_fail) {
            confirm_pv(nt - 1);
            if (!s_fail && warp_rows) {
                fence_after_sync();
                const float inv = 1.f / l;
                float v[64];
                tmem_ld64(t_lane + kStreamOCol, v);
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = Cvt<T>::pack(v[2 * i] * inv, v[2 * i + 1] * inv);
                if (row < len) {
                    uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(start + row) * out_tok_stride +
                                                          h * 64);
#pragma unroll
                    for (int c = 0; c < 8; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    if (row == 0 && cls_out != nullptr) {
                        uint4* cd = reinterpret_cast<uint4*>(cls_out + (static_cast<int64_t>(b) * H + h) * 64);
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            cd[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    }
                }
            }
        }
        cp_async_wait<0>();
    }

    fence_before_sync();
    __syncthreads();
    if (s_fail && tid == 0) raise_status(RAGGED_DEV_TIMEOUT);
    if (warp == 0) {
        fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kStreamTmemCols)
                     : "memory");
    }
}

}  // namespace tc05
}  // namespace ragged
