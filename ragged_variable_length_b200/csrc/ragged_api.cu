// C ABI of the ragged pack -> attend -> unpack library (declared in ragged.h).
//
// The host side of every call is a handful of integer checks followed by one
// kernel launch: no allocation, no synchronisation, no per-call workspace
// (the paper's radpulse section "Bypassing the binding" locates the
// dispatch floor of FA2's varlen path in argument conversion, output and
// softmax_lse allocation and the launch itself).
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <type_traits>

#include "attn_f32.cuh"
#include "attn_mma.cuh"
#include "attn_resident.cuh"
#include "attn_tc05.cuh"
#include "attn_tc05_persist.cuh"
#include <atomic>
#include <cudaTypedefs.h>
#include <mutex>
#include <new>
#include "common.cuh"
#include "mask.cuh"
#include "pack.cuh"

namespace {

constexpr int32_t kAbiVersion = 1;
constexpr int kMaxDevices = 64;
// Shared memory of the pack / unpack survivor list at the largest L_full.
constexpr int kMaxListBytes = RAGGED_MAX_TOKENS * static_cast<int>(sizeof(int));

thread_local char g_last_error[256] = "";

ragged_status fail(ragged_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

ragged_status cuda_check(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return RAGGED_OK;
    return fail(RAGGED_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device flags and caches may be touched by several host threads at once;
// the values they hold are idempotent (a second thread repeats the same query
// or attribute call), so relaxed atomics are enough to make that well defined.
using DeviceFlags = std::atomic<bool>[kMaxDevices];

// Multiprocessor count of the current device, cached per device.
int sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Opt-in shared-memory sizes are set once per device and kernel.
template <typename Kernel>
ragged_status ensure_smem(Kernel kernel, int bytes, DeviceFlags& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return fail(RAGGED_ERR_CUDA, "cudaGetDevice failed");
    if (!done[dev].load(std::memory_order_relaxed)) {
        ragged_status s = cuda_check(
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
            "cudaFuncSetAttribute");
        if (s != RAGGED_OK) return s;
        done[dev].store(true, std::memory_order_relaxed);
    }
    return RAGGED_OK;
}

ragged_status check_rows(int64_t B, int64_t L_full, int64_t row_bytes) {
    if (B < 0) return fail(RAGGED_ERR_INVALID_ARG, "B = %lld is negative", (long long)B);
    if (B > 65535) return fail(RAGGED_ERR_UNSUPPORTED, "B = %lld exceeds 65535", (long long)B);
    if (L_full < 1 || L_full > RAGGED_MAX_TOKENS)
        return fail(RAGGED_ERR_INVALID_ARG, "L_full = %lld outside [1, %d]", (long long)L_full,
                    RAGGED_MAX_TOKENS);
    if (B * L_full >= (int64_t(1) << 31))
        return fail(RAGGED_ERR_UNSUPPORTED, "B * L_full = %lld does not fit int32 offsets",
                    (long long)(B * L_full));
    if (row_bytes <= 0 || row_bytes % 16 != 0)
        return fail(RAGGED_ERR_INVALID_ARG, "row_bytes = %lld must be a positive multiple of 16",
                    (long long)row_bytes);
    if (L_full * (row_bytes / 16) >= (int64_t(1) << 31))
        return fail(RAGGED_ERR_UNSUPPORTED, "rows of %lld bytes are too long", (long long)row_bytes);
    return RAGGED_OK;
}

// Row splits per image: enough CTAs to cover every SM a few times, but at
// least eight rows per CTA on average.
int pack_splits(int64_t B, int64_t L_full) {
    const int64_t target = 4LL * sm_count();
    int64_t s = (target + B - 1) / B;
    const int64_t cap = (L_full + 7) / 8;
    if (s > cap) s = cap;
    if (s < 1) s = 1;
    if (s > 65535) s = 65535;
    return static_cast<int>(s);
}

DeviceFlags g_pack_smem, g_unpack_smem, g_topk_smem;
// Largest L_full of the fused top-k pack: sort keys and survivor list in shared memory.
constexpr int kTopkMaxTokens = 8192;
// pack_topk_kernel's dynamic shared memory: the padded key array, then the
// survivor list.
constexpr int topk_smem_bytes(int L_full) {
    return ragged::topk_pow2(L_full) * static_cast<int>(sizeof(uint64_t)) + L_full * static_cast<int>(sizeof(int));
}
DeviceFlags g_mma_f16_smem, g_mma_bf16_smem, g_f32_smem;

// Largest dynamic shared memory of the resident kernels: 640 keys and a
// 640-entry survivor list.
constexpr int kResidentSmemMax = ragged::resident::smem_bytes(ragged::resident::kMaxKeyTiles,
                                                              ragged::resident::kMaxKeys);

// Warps per row block in the resident kernel: split the keys of a sequence
// across warps when the launch is too small to fill the GPU twice over with
// 64-row tiles (the latency-bound serving regime); keep 64-row tiles otherwise.
int resident_ksplit(int64_t B, int64_t H, int key_tiles) {
    if (key_tiles <= 1) return 1;
    const int64_t ctas64 = static_cast<int64_t>(key_tiles) * H * B;
    if (ctas64 >= 2LL * sm_count()) return 1;
    return key_tiles == 2 ? 2 : 4;
}

template <typename T, class Src, int KS>
ragged_status launch_resident_ks(const Src& src, int64_t B, int64_t H, int key_tiles, int list_entries,
                                 float scale, void* out, int64_t out_tok_stride, void* cls_out, void* packed_out,
                                 DeviceFlags& smem_done, cudaStream_t s) {
    using namespace ragged::resident;
    auto kernel = attn_resident_kernel<T, Src, KS>;
    ragged_status st = ensure_smem(kernel, kResidentSmemMax, smem_done);
    if (st != RAGGED_OK) return st;
    constexpr int rows = 16 * (kWarps / KS);
    const int64_t max_rows = static_cast<int64_t>(key_tiles) * kBlockN;
    const dim3 grid(static_cast<unsigned>((max_rows + rows - 1) / rows), static_cast<unsigned>(H),
                    static_cast<unsigned>(B));
    kernel<<<grid, kThreads, smem_bytes(key_tiles, list_entries), s>>>(
        src, key_tiles, scale * 1.4426950408889634f, static_cast<int>(H), static_cast<uint16_t*>(out),
        out_tok_stride, static_cast<uint16_t*>(cls_out), static_cast<uint16_t*>(packed_out));
    return cuda_check(cudaGetLastError(), "resident attention launch");
}

std::atomic<int> g_attn_kernel{RAGGED_ATTN_AUTO};
DeviceFlags g_tc05_smem[2];

template <typename T>
ragged_status launch_tc05(const ragged::resident::PackedRows& src, int64_t B, int64_t H, int64_t max_seqlen,
                          float scale, void* out, int64_t out_tok_stride, void* cls_out, int slot, cudaStream_t s) {
    using namespace ragged::tc05;
    auto kernel = attn_tc05_stream_kernel<T>;
    const int smem = stream_smem_bytes(std::is_same<T, __nv_bfloat16>::value ? 2 : 1);
    ragged_status st = ensure_smem(kernel, smem, g_tc05_smem[slot]);
    if (st != RAGGED_OK) return st;
    const dim3 grid(static_cast<unsigned>((max_seqlen + kRows - 1) / kRows), static_cast<unsigned>(H),
                    static_cast<unsigned>(B));
    kernel<<<grid, kStreamThreads, smem, s>>>(src, scale * 1.4426950408889634f, static_cast<int>(H),
                                        static_cast<uint16_t*>(out), out_tok_stride, static_cast<uint16_t*>(cls_out));
    return cuda_check(cudaGetLastError(), "tcgen05 attention launch");
}

// ---- TMA tensor maps for the persistent kernel ------------------------------

// cuTensorMapEncodeTiled from the driver, found once through the runtime (the
// library links no driver library of its own).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Encoded maps are cached by their parameters, so repeated calls on the same
// buffers encode nothing.
struct MapKey {
    const void* ptr;
    int64_t H, rows, head_stride, tok_stride;
    int box_rows;
    bool operator==(const MapKey& o) const {
        return ptr == o.ptr && H == o.H && rows == o.rows && head_stride == o.head_stride &&
               tok_stride == o.tok_stride && box_rows == o.box_rows;
    }
};
constexpr int kMapCache = 24;
struct MapCache {
    std::mutex mu;
    MapKey key[kMapCache];
    CUtensorMap map[kMapCache];
    int used = 0, next = 0;
};
MapCache g_maps;

// 3-D map over one operand of a [rows, H, 64] 16-bit view (token stride and
// head stride in elements): box = 64 elements x 1 head x box_rows rows with the
// 128-byte swizzle.  False when the driver rejects the layout.
bool tensor_map_3d(CUtensorMap* out, const void* ptr, int64_t H, int64_t rows, int64_t head_stride,
                   int64_t tok_stride, int box_rows) {
    const MapKey key{ptr, H, rows, head_stride, tok_stride, box_rows};
    std::lock_guard<std::mutex> lock(g_maps.mu);
    for (int i = 0; i < g_maps.used; ++i)
        if (g_maps.key[i] == key) {
            *out = g_maps.map[i];
            return true;
        }
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (encode == nullptr) return false;
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
    // A single head has no head stride of its own; any legal value will do.
    const int64_t hs = H == 1 ? 64 : head_stride;
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(hs * 2), static_cast<cuuint64_t>(tok_stride * 2)};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap m;
    if (encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    const int slot = g_maps.used < kMapCache ? g_maps.used++ : (g_maps.next++ % kMapCache);
    g_maps.key[slot] = key;
    g_maps.map[slot] = m;
    *out = m;
    return true;
}

DeviceFlags g_persist_smem[2];

// Launches the persistent tcgen05 kernel; *launched = false (and nothing is
// enqueued) when the launch shape is outside what it supports.
template <typename T>
ragged_status launch_tc05_persist(const ragged::resident::PackedRows& src, int64_t B, int64_t H,
                                  int64_t max_seqlen, float scale, void* out, int64_t out_tok_stride, void* cls_out,
                                  int slot, cudaStream_t s, bool* launched) {
    using namespace ragged::tc05;
    *launched = false;
    const int64_t q_tiles = (max_seqlen + kRows - 1) / kRows;
    // Items are packed into 32-bit words (sequence: 11 bits, head: 10, query
    // tile: 11), and each CTA keeps at most kPersistMaxItems of them.
    if (B > kPersistMaxB || H > 1023 || q_tiles > 2047) return RAGGED_OK;
    const int64_t items_bound = B * H * q_tiles;
    const int64_t ctas = std::min<int64_t>(items_bound, 2LL * sm_count());
    const int64_t items_cap = (items_bound + ctas - 1) / ctas;
    if (items_cap > kPersistMaxItems) return RAGGED_OK;
    // Full tiles never reach past the last row of their sequence, and every
    // sequence ends within B * max_seqlen rows.
    const int64_t rows = B * max_seqlen;
    CUtensorMap tq, tk, tv;
    if (!tensor_map_3d(&tq, src.q, H, rows, src.head_stride, src.tok_stride, kRows) ||
        !tensor_map_3d(&tk, src.k, H, rows, src.head_stride, src.tok_stride, kTileN) ||
        !tensor_map_3d(&tv, src.v, H, rows, src.head_stride, src.tok_stride, kTileN))
        return RAGGED_OK;
    auto kernel = attn_tc05_persist_kernel<T>;
    ragged_status st = ensure_smem(kernel, persist_smem_bytes(kPersistMaxB, kPersistMaxItems), g_persist_smem[slot]);
    if (st != RAGGED_OK) return st;
    PersistArgs args{src.q, src.k, src.v, src.tok_stride, src.head_stride, src.cu, static_cast<int>(B),
                     static_cast<int>(H), static_cast<int>(max_seqlen), scale * 1.4426950408889634f,
                     static_cast<uint16_t*>(out), out_tok_stride, static_cast<uint16_t*>(cls_out),
                     static_cast<int>(items_cap)};
    kernel<<<static_cast<unsigned>(ctas), kPersistThreads,
             persist_smem_bytes(static_cast<int>(B), static_cast<int>(items_cap)), s>>>(tq, tk, tv, args);
    *launched = true;
    return cuda_check(cudaGetLastError(), "persistent tcgen05 attention launch");
}

// slot: 0/1 packed f16/bf16, 2/3 dense f16/bf16 (one set of smem flags per kernel).
DeviceFlags g_res_smem_ks[4][3];

template <typename T, class Src>
ragged_status launch_resident(const Src& src, int64_t B, int64_t H, int key_tiles, int list_entries,
                              float scale, void* out, int64_t out_tok_stride, void* cls_out, void* packed_out,
                              int slot, cudaStream_t s) {
    switch (resident_ksplit(B, H, key_tiles)) {
        case 4:
            return launch_resident_ks<T, Src, 4>(src, B, H, key_tiles, list_entries, scale, out, out_tok_stride,
                                                 cls_out, packed_out, g_res_smem_ks[slot][2], s);
        case 2:
            return launch_resident_ks<T, Src, 2>(src, B, H, key_tiles, list_entries, scale, out, out_tok_stride,
                                                 cls_out, packed_out, g_res_smem_ks[slot][1], s);
        default:
            return launch_resident_ks<T, Src, 1>(src, B, H, key_tiles, list_entries, scale, out, out_tok_stride,
                                                 cls_out, packed_out, g_res_smem_ks[slot][0], s);
    }
}

// ---- fixed scratch of ragged_pipeline_noalloc ---------------------------------
//
// The packed q/k/v between the pack and the attention launch, for callers that
// cannot allocate device memory.  It is part of this library's device image:
// every GPU on which the library's kernels are loaded holds these bytes until
// the process exits, whether or not the entry point is ever called.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RAGGED_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch, looked up once per device.  In host
// code the array's name only stands in for the symbol; the address a kernel
// may use comes from cudaGetSymbolAddress with that device current.
std::atomic<void*> g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mu;

ragged_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return fail(RAGGED_ERR_CUDA, "cudaGetDevice failed");
    void* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        p = g_noalloc_addr[dev].load(std::memory_order_relaxed);
        if (p == nullptr) {
            ragged_status st = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch),
                                          "cudaGetSymbolAddress of the fixed scratch");
            if (st != RAGGED_OK) return st;
            if (p == nullptr) return fail(RAGGED_ERR_CUDA, "cudaGetSymbolAddress returned NULL");
            g_noalloc_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return RAGGED_OK;
}

}  // namespace

extern "C" {

int32_t ragged_abi_version(void) { return kAbiVersion; }

int32_t ragged_set_attn_kernel(int32_t kernel) {
    if (kernel < RAGGED_ATTN_AUTO || kernel > RAGGED_ATTN_PERSISTENT) return -1;
    return g_attn_kernel.exchange(kernel);
}

const char* ragged_last_error(void) { return g_last_error; }

const char* ragged_status_string(ragged_status s) {
    switch (s) {
        case RAGGED_OK: return "ok";
        case RAGGED_ERR_INVALID_ARG: return "invalid argument";
        case RAGGED_ERR_UNSUPPORTED: return "unsupported";
        case RAGGED_ERR_CUDA: return "CUDA runtime error";
        case RAGGED_ERR_DEVICE: return "device-side error";
    }
    return "unknown status";
}

ragged_status ragged_pack(const void* dense, int64_t B, int64_t L_full, int64_t row_bytes,
                          const uint8_t* keep, void* packed, int32_t* cu_seqlens,
                          int32_t* src_idx, void* stream) {
    ragged_status st = check_rows(B, L_full, row_bytes);
    if (st != RAGGED_OK) return st;
    if (cu_seqlens == nullptr) return fail(RAGGED_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(src_idx) & 3u))
        return fail(RAGGED_ERR_INVALID_ARG, "cu_seqlens / src_idx must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (B == 0) return cuda_check(cudaMemsetAsync(cu_seqlens, 0, sizeof(int32_t), s), "cudaMemsetAsync");
    if (dense == nullptr || keep == nullptr || packed == nullptr)
        return fail(RAGGED_ERR_INVALID_ARG, "dense, keep and packed must not be NULL");
    if (!aligned16(dense) || !aligned16(packed))
        return fail(RAGGED_ERR_INVALID_ARG, "dense and packed must be 16-byte aligned");
    const int smem = static_cast<int>(L_full * sizeof(int));
    st = ensure_smem(ragged::pack_kernel, kMaxListBytes, g_pack_smem);
    if (st != RAGGED_OK) return st;
    const dim3 grid(pack_splits(B, L_full), static_cast<unsigned>(B));
    ragged::pack_kernel<<<grid, ragged::kPackThreads, smem, s>>>(
        static_cast<const uint4*>(dense), static_cast<int>(L_full),
        static_cast<uint32_t>(row_bytes / 16), keep, static_cast<uint4*>(packed), cu_seqlens, src_idx);
    return cuda_check(cudaGetLastError(), "pack launch");
}

ragged_status ragged_mask_l2(const void* x, int64_t B, int64_t L_full, int64_t C, int64_t tok_stride,
                             ragged_dtype dtype, double tau, uint8_t* keep, void* stream) {
    if (B < 0) return fail(RAGGED_ERR_INVALID_ARG, "B = %lld is negative", (long long)B);
    if (L_full < 1 || L_full > RAGGED_MAX_TOKENS)
        return fail(RAGGED_ERR_INVALID_ARG, "L_full = %lld outside [1, %d]", (long long)L_full, RAGGED_MAX_TOKENS);
    if (B * L_full >= (int64_t(1) << 31))
        return fail(RAGGED_ERR_UNSUPPORTED, "B * L_full = %lld does not fit int32 offsets", (long long)(B * L_full));
    if (C < 1 || C > (int64_t(1) << 24))
        return fail(RAGGED_ERR_INVALID_ARG, "C = %lld outside [1, 2^24]", (long long)C);
    if (tok_stride < C) return fail(RAGGED_ERR_INVALID_ARG, "tok_stride must be >= C");
    if (dtype != RAGGED_F16 && dtype != RAGGED_BF16 && dtype != RAGGED_F32)
        return fail(RAGGED_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (tau != tau) return fail(RAGGED_ERR_INVALID_ARG, "tau is NaN");
    if (B == 0) return RAGGED_OK;
    if (x == nullptr || keep == nullptr) return fail(RAGGED_ERR_INVALID_ARG, "x and keep must not be NULL");
    const int64_t esz = dtype == RAGGED_F32 ? 4 : 2;
    if (reinterpret_cast<uintptr_t>(x) % esz) return fail(RAGGED_ERR_INVALID_ARG, "x is not element-aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int L = static_cast<int>(L_full), Ci = static_cast<int>(C);
    // 16-bit rows that start on 16-byte boundaries go through the vector path
    // (one half-warp per token, 16-byte loads, fp32 two-sum accumulation).
    const bool vec = esz == 2 && aligned16(x) && (tok_stride * 2) % 16 == 0 && C % 8 == 0 && C <= ragged::kMaskVecMaxC;
    const int per_cta = vec ? ragged::kMaskThreads / 16 : ragged::kMaskThreads / 32;
    const unsigned chunks = static_cast<unsigned>((L_full + per_cta - 1) / per_cta);
    for (int64_t b0 = 0; b0 < B; b0 += ragged::kMaskMaxImages) {
        const int64_t nb = B - b0 < ragged::kMaskMaxImages ? B - b0 : ragged::kMaskMaxImages;
        const dim3 grid(chunks, static_cast<unsigned>(nb));
        const void* xb = static_cast<const char*>(x) + b0 * L_full * tok_stride * esz;
        uint8_t* kb = keep + b0 * L_full;
        if (vec && dtype == RAGGED_F16)
            ragged::mask_l2_vec_kernel<__half><<<grid, ragged::kMaskThreads, 0, s>>>(xb, L, Ci, tok_stride, tau, kb);
        else if (vec)
            ragged::mask_l2_vec_kernel<__nv_bfloat16><<<grid, ragged::kMaskThreads, 0, s>>>(xb, L, Ci, tok_stride, tau,
                                                                                           kb);
        else if (dtype == RAGGED_F16)
            ragged::mask_l2_kernel<__half><<<grid, ragged::kMaskThreads, 0, s>>>(xb, L, Ci, tok_stride, tau, kb);
        else if (dtype == RAGGED_BF16)
            ragged::mask_l2_kernel<__nv_bfloat16><<<grid, ragged::kMaskThreads, 0, s>>>(xb, L, Ci, tok_stride, tau, kb);
        else
            ragged::mask_l2_kernel<float><<<grid, ragged::kMaskThreads, 0, s>>>(xb, L, Ci, tok_stride, tau, kb);
    }
    return cuda_check(cudaGetLastError(), "mask_l2 launch");
}

ragged_status ragged_pack_topk(const void* dense, int64_t B, int64_t L_full, int64_t row_bytes, const float* scores,
                               const int32_t* keep_count, void* packed, int32_t* cu_seqlens, int32_t* src_idx,
                               uint8_t* keep_out, void* stream) {
    ragged_status st = check_rows(B, L_full, row_bytes);
    if (st != RAGGED_OK) return st;
    if (L_full > kTopkMaxTokens)
        return fail(RAGGED_ERR_UNSUPPORTED, "L_full = %lld exceeds %d for the top-k selection", (long long)L_full,
                    kTopkMaxTokens);
    if (cu_seqlens == nullptr) return fail(RAGGED_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(src_idx) & 3u))
        return fail(RAGGED_ERR_INVALID_ARG, "cu_seqlens / src_idx must be 4-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (B == 0) return cuda_check(cudaMemsetAsync(cu_seqlens, 0, sizeof(int32_t), s), "cudaMemsetAsync");
    if (dense == nullptr || scores == nullptr || keep_count == nullptr || packed == nullptr)
        return fail(RAGGED_ERR_INVALID_ARG, "dense, scores, keep_count and packed must not be NULL");
    if (!aligned16(dense) || !aligned16(packed))
        return fail(RAGGED_ERR_INVALID_ARG, "dense and packed must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(scores) & 3u) || (reinterpret_cast<uintptr_t>(keep_count) & 3u))
        return fail(RAGGED_ERR_INVALID_ARG, "scores / keep_count must be 4-byte aligned");
    st = ensure_smem(ragged::pack_topk_kernel, topk_smem_bytes(kTopkMaxTokens), g_topk_smem);
    if (st != RAGGED_OK) return st;
    const int smem = topk_smem_bytes(static_cast<int>(L_full));
    const dim3 grid(pack_splits(B, L_full), static_cast<unsigned>(B));
    ragged::pack_topk_kernel<<<grid, ragged::kPackThreads, smem, s>>>(
        static_cast<const uint4*>(dense), static_cast<int>(L_full), static_cast<uint32_t>(row_bytes / 16), scores,
        keep_count, static_cast<uint4*>(packed), cu_seqlens, src_idx, keep_out);
    return cuda_check(cudaGetLastError(), "pack_topk launch");
}

ragged_status ragged_unpack(const void* packed, const int32_t* cu_seqlens, const uint8_t* keep,
                            int64_t B, int64_t L_full, int64_t row_bytes, void* dense_out,
                            void* stream) {
    ragged_status st = check_rows(B, L_full, row_bytes);
    if (st != RAGGED_OK) return st;
    if (B == 0) return RAGGED_OK;
    if (packed == nullptr || cu_seqlens == nullptr || keep == nullptr || dense_out == nullptr)
        return fail(RAGGED_ERR_INVALID_ARG, "packed, cu_seqlens, keep and dense_out must not be NULL");
    if (!aligned16(packed) || !aligned16(dense_out) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return fail(RAGGED_ERR_INVALID_ARG, "packed / dense_out must be 16-byte aligned, cu_seqlens 4-byte");
    const int smem = static_cast<int>(L_full * sizeof(int));
    st = ensure_smem(ragged::unpack_kernel, kMaxListBytes, g_unpack_smem);
    if (st != RAGGED_OK) return st;
    const dim3 grid(pack_splits(B, L_full), static_cast<unsigned>(B));
    ragged::unpack_kernel<<<grid, ragged::kPackThreads, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(packed), cu_seqlens, static_cast<int>(L_full),
        static_cast<uint32_t>(row_bytes / 16), keep, static_cast<uint4*>(dense_out));
    return cuda_check(cudaGetLastError(), "unpack launch");
}

ragged_status ragged_unpack_cls(const void* packed, const int32_t* cu_seqlens, int64_t B,
                                int64_t row_bytes, void* cls_out, void* stream) {
    if (B < 0) return fail(RAGGED_ERR_INVALID_ARG, "B = %lld is negative", (long long)B);
    if (row_bytes <= 0 || row_bytes % 16 != 0)
        return fail(RAGGED_ERR_INVALID_ARG, "row_bytes = %lld must be a positive multiple of 16",
                    (long long)row_bytes);
    if (B == 0) return RAGGED_OK;
    if (packed == nullptr || cu_seqlens == nullptr || cls_out == nullptr)
        return fail(RAGGED_ERR_INVALID_ARG, "packed, cu_seqlens and cls_out must not be NULL");
    if (!aligned16(packed) || !aligned16(cls_out) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return fail(RAGGED_ERR_INVALID_ARG, "packed / cls_out must be 16-byte aligned, cu_seqlens 4-byte");
    const int64_t n = B * (row_bytes / 16);
    if (B > (int64_t(1) << 31) || n >= (int64_t(1) << 40))
        return fail(RAGGED_ERR_UNSUPPORTED, "CLS extraction too large");
    const int64_t blocks = (n + 255) / 256;
    ragged::unpack_cls_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(packed), cu_seqlens, static_cast<int>(B),
        static_cast<uint32_t>(row_bytes / 16), static_cast<uint4*>(cls_out));
    return cuda_check(cudaGetLastError(), "unpack_cls launch");
}

ragged_status ragged_attn_fwd(const void* q, const void* k, const void* v, int64_t tok_stride,
                              int64_t head_stride, const int32_t* cu_seqlens, int64_t B,
                              int64_t max_seqlen, int64_t H, int64_t head_dim, float scale,
                              ragged_dtype dtype, void* out, int64_t out_tok_stride,
                              void* cls_out, void* stream) {
    if (B < 0) return fail(RAGGED_ERR_INVALID_ARG, "B = %lld is negative", (long long)B);
    if (B > 65535) return fail(RAGGED_ERR_UNSUPPORTED, "B = %lld exceeds 65535", (long long)B);
    if (dtype != RAGGED_F16 && dtype != RAGGED_BF16 && dtype != RAGGED_F32)
        return fail(RAGGED_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (head_dim != 64) return fail(RAGGED_ERR_UNSUPPORTED, "head_dim = %lld (only 64 is implemented)", (long long)head_dim);
    if (H < 1 || H > 65535) return fail(RAGGED_ERR_INVALID_ARG, "H = %lld outside [1, 65535]", (long long)H);
    if (max_seqlen < 1 || max_seqlen > RAGGED_MAX_TOKENS)
        return fail(RAGGED_ERR_INVALID_ARG, "max_seqlen = %lld outside [1, %d]", (long long)max_seqlen,
                    RAGGED_MAX_TOKENS);
    if (!(scale > 0.f) || scale > 3.0e38f)
        return fail(RAGGED_ERR_INVALID_ARG, "scale must be a positive finite number");
    if (B == 0) return RAGGED_OK;
    if (!q || !k || !v || !out || !cu_seqlens)
        return fail(RAGGED_ERR_INVALID_ARG, "q, k, v, out and cu_seqlens must not be NULL");
    const int64_t esz = dtype == RAGGED_F32 ? 4 : 2;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cls_out) ||
        (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return fail(RAGGED_ERR_INVALID_ARG, "q, k, v, out, cls_out must be 16-byte aligned");
    if (tok_stride <= 0 || head_stride < 0 || (tok_stride * esz) % 16 || (head_stride * esz) % 16)
        return fail(RAGGED_ERR_INVALID_ARG, "tok_stride / head_stride must be multiples of 16 bytes");
    if (out_tok_stride < H * head_dim || (out_tok_stride * esz) % 16)
        return fail(RAGGED_ERR_INVALID_ARG, "out_tok_stride must be >= H * head_dim and a multiple of 16 bytes");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ragged_status st;
    if (dtype == RAGGED_F32) {
        using namespace ragged::f32_attn;
        st = ensure_smem(attn_fwd_f32_kernel, kSmemBytes, g_f32_smem);
        if (st != RAGGED_OK) return st;
        const dim3 grid(static_cast<unsigned>((max_seqlen + kBlockM - 1) / kBlockM), static_cast<unsigned>(H),
                        static_cast<unsigned>(B));
        attn_fwd_f32_kernel<<<grid, kThreads, kSmemBytes, s>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            tok_stride, head_stride, cu_seqlens, static_cast<int>(max_seqlen), static_cast<int>(H), scale,
            static_cast<float*>(out), out_tok_stride, static_cast<float*>(cls_out));
        return cuda_check(cudaGetLastError(), "attention (f32) launch");
    }
    // Kernel choice.  AUTO: whole-sequence residency pays off in the
    // latency-bound regime (few CTAs: keys split across warps) and for
    // single-tile sequences; launches with at least eight (sequence, query
    // tile, head) items per SM go to the persistent tcgen05 kernel, whose
    // per-CTA set-up is paid once; the rest stream K/V tiles.
    const int res_tiles = static_cast<int>((max_seqlen + 63) / 64);
    const int64_t q_tiles = (max_seqlen + 127) / 128;
    int kernel_choice = g_attn_kernel.load(std::memory_order_relaxed);
    if (kernel_choice == RAGGED_ATTN_AUTO) {
        if (max_seqlen <= ragged::resident::kMaxKeys && (res_tiles == 1 || resident_ksplit(B, H, res_tiles) > 1))
            kernel_choice = RAGGED_ATTN_RESIDENT;
        else if (B <= ragged::tc05::kPersistMaxB && B * H * q_tiles >= 8LL * sm_count())
            kernel_choice = RAGGED_ATTN_PERSISTENT;
        else if (res_tiles > 4)
            kernel_choice = RAGGED_ATTN_TCGEN05;   // long sequences: many key tiles per query tile
        else
            kernel_choice = RAGGED_ATTN_STREAMING;
    }
    if (kernel_choice == RAGGED_ATTN_RESIDENT && max_seqlen > ragged::resident::kMaxKeys)
        return fail(RAGGED_ERR_UNSUPPORTED, "the resident attention kernel holds at most 640 keys");
    ragged::resident::PackedRows src{static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                     static_cast<const uint16_t*>(v), tok_stride, head_stride, cu_seqlens,
                                     static_cast<int>(max_seqlen), 0, 0, 0};
    if (kernel_choice == RAGGED_ATTN_PERSISTENT) {
        bool launched = false;
        st = dtype == RAGGED_F16
                 ? launch_tc05_persist<__half>(src, B, H, max_seqlen, scale, out, out_tok_stride, cls_out, 0, s,
                                               &launched)
                 : launch_tc05_persist<__nv_bfloat16>(src, B, H, max_seqlen, scale, out, out_tok_stride, cls_out, 1,
                                                      s, &launched);
        if (st != RAGGED_OK || launched) return st;
        kernel_choice = RAGGED_ATTN_TCGEN05;
    }
    if (kernel_choice == RAGGED_ATTN_TCGEN05) {
        if (dtype == RAGGED_F16)
            return launch_tc05<__half>(src, B, H, max_seqlen, scale, out, out_tok_stride, cls_out, 0, s);
        return launch_tc05<__nv_bfloat16>(src, B, H, max_seqlen, scale, out, out_tok_stride, cls_out, 1, s);
    }
    if (kernel_choice == RAGGED_ATTN_RESIDENT) {
        if (dtype == RAGGED_F16)
            return launch_resident<__half>(src, B, H, res_tiles, 0, scale, out, out_tok_stride, cls_out, nullptr, 0, s);
        return launch_resident<__nv_bfloat16>(src, B, H, res_tiles, 0, scale, out, out_tok_stride, cls_out, nullptr,
                                              1, s);
    }
    using namespace ragged::mma_attn;
    const dim3 grid(static_cast<unsigned>(H), static_cast<unsigned>(B),
                    static_cast<unsigned>((max_seqlen + kBlockM - 1) / kBlockM));
    const float scale_log2 = scale * 1.4426950408889634f;
    if (dtype == RAGGED_F16) {
        st = ensure_smem(attn_fwd_kernel<__half>, kSmemBytes, g_mma_f16_smem);
        if (st != RAGGED_OK) return st;
        attn_fwd_kernel<__half><<<grid, kThreads, kSmemBytes, s>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
            tok_stride, head_stride, cu_seqlens, static_cast<int>(max_seqlen), static_cast<int>(H),
            scale_log2, static_cast<uint16_t*>(out), out_tok_stride, static_cast<uint16_t*>(cls_out));
    } else {
        st = ensure_smem(attn_fwd_kernel<__nv_bfloat16>, kSmemBytes, g_mma_bf16_smem);
        if (st != RAGGED_OK) return st;
        attn_fwd_kernel<__nv_bfloat16><<<grid, kThreads, kSmemBytes, s>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
            tok_stride, head_stride, cu_seqlens, static_cast<int>(max_seqlen), static_cast<int>(H),
            scale_log2, static_cast<uint16_t*>(out), out_tok_stride, static_cast<uint16_t*>(cls_out));
    }
    return cuda_check(cudaGetLastError(), "attention launch");
}

ragged_status ragged_pipeline(const void* dense_qkv, const uint8_t* keep, int64_t B, int64_t L_full,
                              int64_t H, int64_t head_dim, float scale, ragged_dtype dtype,
                              void* packed_qkv, int32_t* cu_seqlens, void* out, void* cls_out,
                              uint32_t flags, void* stream) {
    if (head_dim != 64) return fail(RAGGED_ERR_UNSUPPORTED, "head_dim = %lld (only 64 is implemented)", (long long)head_dim);
    if (H < 1 || H > 65535) return fail(RAGGED_ERR_INVALID_ARG, "H = %lld outside [1, 65535]", (long long)H);
    if (dtype != RAGGED_F16 && dtype != RAGGED_BF16 && dtype != RAGGED_F32)
        return fail(RAGGED_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if ((flags & ~(RAGGED_PIPELINE_FUSED | RAGGED_PIPELINE_SPLIT | RAGGED_PIPELINE_SYNC)) != 0 ||
        (flags & (RAGGED_PIPELINE_FUSED | RAGGED_PIPELINE_SPLIT)) == (RAGGED_PIPELINE_FUSED | RAGGED_PIPELINE_SPLIT))
        return fail(RAGGED_ERR_INVALID_ARG, "flags = %u is not a valid pipeline mode", flags);
    if (flags & RAGGED_PIPELINE_SYNC) {
        ragged_status st = ragged_pipeline(dense_qkv, keep, B, L_full, H, head_dim, scale, dtype, packed_qkv,
                                           cu_seqlens, out, cls_out, flags & ~RAGGED_PIPELINE_SYNC, stream);
        if (st != RAGGED_OK) return st;
        return cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize");
    }
    const int64_t esz = dtype == RAGGED_F32 ? 4 : 2;
    const int64_t D = H * head_dim;
    ragged_status st = check_rows(B, L_full, 3 * D * esz);
    if (st != RAGGED_OK) return st;
    if (!(scale > 0.f) || scale > 3.0e38f)
        return fail(RAGGED_ERR_INVALID_ARG, "scale must be a positive finite number");
    // One fused launch when the whole sequence fits the resident kernel and
    // the per-CTA survivor counting stays small; pack + attention otherwise.
    const int64_t key_tiles = (L_full + 63) / 64;
    const bool fusable = dtype != RAGGED_F32 && L_full <= ragged::resident::kMaxKeys;
    // Every CTA of image b reads the b * L_full mask bytes before it.
    const int64_t rows_per_cta = 16 * (4 / resident_ksplit(B, H, static_cast<int>(key_tiles)));
    const int64_t ctas_per_image = (key_tiles * 64 + rows_per_cta - 1) / rows_per_cta * H;
    const int64_t count_bytes = ctas_per_image * L_full * (B * B / 2);
    bool fused = fusable && count_bytes <= (int64_t(32) << 20);
    if (flags & RAGGED_PIPELINE_FUSED) {
        if (!fusable) return fail(RAGGED_ERR_UNSUPPORTED, "the fused pipeline needs f16/bf16 and L_full <= %d",
                                  ragged::resident::kMaxKeys);
        fused = true;
    }
    if (flags & RAGGED_PIPELINE_SPLIT) fused = false;
    if (!fused) {
        if (packed_qkv == nullptr)
            return fail(RAGGED_ERR_INVALID_ARG, "packed_qkv is required when the pipeline runs as two launches");
        st = ragged_pack(dense_qkv, B, L_full, 3 * D * esz, keep, packed_qkv, cu_seqlens, nullptr, stream);
        if (st != RAGGED_OK || B == 0) return st;
        const char* base = static_cast<const char*>(packed_qkv);
        return ragged_attn_fwd(base, base + D * esz, base + 2 * D * esz, 3 * D, head_dim, cu_seqlens, B,
                               L_full, H, head_dim, scale, dtype, out, D, cls_out, stream);
    }
    if (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return fail(RAGGED_ERR_INVALID_ARG, "cu_seqlens must be a 4-byte aligned device pointer");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (B == 0) return cuda_check(cudaMemsetAsync(cu_seqlens, 0, sizeof(int32_t), s), "cudaMemsetAsync");
    if (dense_qkv == nullptr || keep == nullptr || out == nullptr)
        return fail(RAGGED_ERR_INVALID_ARG, "dense_qkv, keep and out must not be NULL");
    if (!aligned16(dense_qkv) || !aligned16(out) || !aligned16(cls_out) || !aligned16(packed_qkv))
        return fail(RAGGED_ERR_INVALID_ARG, "dense_qkv, packed_qkv, out and cls_out must be 16-byte aligned");
    ragged::resident::DenseRows src{static_cast<const uint16_t*>(dense_qkv), keep, cu_seqlens,
                                    static_cast<int>(L_full), static_cast<int>(H), 0, 0, 0, 0, nullptr};
    if (dtype == RAGGED_F16)
        return launch_resident<__half>(src, B, H, static_cast<int>(key_tiles), static_cast<int>(L_full), scale, out,
                                       D, cls_out, packed_qkv, 2, s);
    return launch_resident<__nv_bfloat16>(src, B, H, static_cast<int>(key_tiles), static_cast<int>(L_full), scale,
                                          out, D, cls_out, packed_qkv, 3, s);
}

ragged_status ragged_get_device_status(uint32_t* host_out, void* stream) {
    if (host_out == nullptr) return fail(RAGGED_ERR_INVALID_ARG, "host_out is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int value = 0, zero = 0;
    ragged_status st = cuda_check(
        cudaMemcpyFromSymbolAsync(&value, ragged::g_dev_status, sizeof value, 0, cudaMemcpyDeviceToHost, s),
        "reading the device status word");
    if (st != RAGGED_OK) return st;
    st = cuda_check(cudaMemcpyToSymbolAsync(ragged::g_dev_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s),
                    "clearing the device status word");
    if (st != RAGGED_OK) return st;
    st = cuda_check(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    if (st != RAGGED_OK) return st;
    *host_out = value;
    return RAGGED_OK;
}

ragged_status ragged_pipeline_noalloc(const void* dense_qkv, const uint8_t* keep, int64_t B, int64_t L_full,
                                      int64_t H, int64_t head_dim, float scale, ragged_dtype dtype,
                                      int32_t* cu_seqlens, void* out, void* cls_out, void* stream) {
    if (head_dim != 64) return fail(RAGGED_ERR_UNSUPPORTED, "head_dim = %lld (only 64 is implemented)", (long long)head_dim);
    if (H < 1 || H > 65535) return fail(RAGGED_ERR_INVALID_ARG, "H = %lld outside [1, 65535]", (long long)H);
    if (dtype != RAGGED_F16 && dtype != RAGGED_BF16 && dtype != RAGGED_F32)
        return fail(RAGGED_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    const int64_t row_bytes = 3 * H * head_dim * (dtype == RAGGED_F32 ? 4 : 2);
    ragged_status st = check_rows(B, L_full, row_bytes);
    if (st != RAGGED_OK) return st;
    // Every one of the B * L_full rows may survive, so that is what must fit.
    if (B * L_full > static_cast<int64_t>(RAGGED_NOALLOC_SCRATCH_BYTES) / row_bytes)
        return fail(RAGGED_ERR_UNSUPPORTED,
                    "B * L_full * row_bytes = %lld bytes of packed q/k/v exceed the fixed scratch of %lld bytes",
                    (long long)(B * L_full * row_bytes), (long long)RAGGED_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != RAGGED_OK) return st;
    return ragged_pipeline(dense_qkv, keep, B, L_full, H, head_dim, scale, dtype, scratch, cu_seqlens, out,
                           cls_out, RAGGED_PIPELINE_SPLIT, stream);
}


#ifdef RAGGED_TEST_HOOKS
// Test builds only; declared in ragged_test_hooks.h.
RAGGED_API ragged_status ragged_test_set_hooks(int32_t hook, uint32_t spin_limit) {
    if (hook < 0 || hook > 2 || spin_limit == 0) return fail(RAGGED_ERR_INVALID_ARG, "bad test hook settings");
    ragged_status st = cuda_check(cudaMemcpyToSymbol(ragged::tc05::g_test_hook, &hook, sizeof hook), "test hook");
    if (st != RAGGED_OK) return st;
    return cuda_check(cudaMemcpyToSymbol(ragged::tc05::g_test_spin_limit, &spin_limit, sizeof spin_limit),
                      "test spin limit");
}
#endif

// ---- library-owned CUDA graph of one pipeline call -------------------------

struct ragged_pipeline_graph {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    int device;
};

ragged_status ragged_pipeline_graph_create(const void* dense_qkv, const uint8_t* keep, int64_t B, int64_t L_full,
                                           int64_t H, int64_t head_dim, float scale, ragged_dtype dtype,
                                           void* packed_qkv, int32_t* cu_seqlens, void* out, void* cls_out,
                                           uint32_t flags, void* stream, ragged_pipeline_graph** graph_out) {
    if (graph_out == nullptr) return fail(RAGGED_ERR_INVALID_ARG, "graph_out is NULL");
    *graph_out = nullptr;
    if (flags & RAGGED_PIPELINE_SYNC) return fail(RAGGED_ERR_INVALID_ARG, "RAGGED_PIPELINE_SYNC cannot be recorded");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (s == nullptr) return fail(RAGGED_ERR_INVALID_ARG, "a graph is recorded on a created stream, not the default one");
    // One call outside the capture: argument checks, and the per-device
    // set-up (kernel attributes, tensor maps) that must not be recorded.
    ragged_status st = ragged_pipeline(dense_qkv, keep, B, L_full, H, head_dim, scale, dtype, packed_qkv, cu_seqlens,
                                       out, cls_out, flags, stream);
    if (st != RAGGED_OK) return st;
    int dev = 0;
    st = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
    if (st != RAGGED_OK) return st;
    st = cuda_check(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal), "cudaStreamBeginCapture");
    if (st != RAGGED_OK) return st;
    const ragged_status call = ragged_pipeline(dense_qkv, keep, B, L_full, H, head_dim, scale, dtype, packed_qkv,
                                               cu_seqlens, out, cls_out, flags, stream);
    cudaGraph_t graph = nullptr;
    st = cuda_check(cudaStreamEndCapture(s, &graph), "cudaStreamEndCapture");
    if (call != RAGGED_OK || st != RAGGED_OK) {
        if (graph != nullptr) cudaGraphDestroy(graph);
        return call != RAGGED_OK ? call : st;
    }
    cudaGraphExec_t exec = nullptr;
    st = cuda_check(cudaGraphInstantiate(&exec, graph, 0), "cudaGraphInstantiate");
    if (st != RAGGED_OK) {
        cudaGraphDestroy(graph);
        return st;
    }
    ragged_pipeline_graph* g = new (std::nothrow) ragged_pipeline_graph{graph, exec, dev};
    if (g == nullptr) {
        cudaGraphExecDestroy(exec);
        cudaGraphDestroy(graph);
        return fail(RAGGED_ERR_CUDA, "out of host memory");
    }
    *graph_out = g;
    return RAGGED_OK;
}

ragged_status ragged_pipeline_graph_launch(ragged_pipeline_graph* graph, void* stream, uint32_t flags) {
    if (graph == nullptr) return fail(RAGGED_ERR_INVALID_ARG, "graph is NULL");
    if ((flags & ~RAGGED_PIPELINE_SYNC) != 0) return fail(RAGGED_ERR_INVALID_ARG, "flags = %u", flags);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ragged_status st = cuda_check(cudaGraphLaunch(graph->exec, s), "cudaGraphLaunch");
    if (st != RAGGED_OK || !(flags & RAGGED_PIPELINE_SYNC)) return st;
    return cuda_check(cudaStreamSynchronize(s), "cudaStreamSynchronize");
}

ragged_status ragged_pipeline_graph_destroy(ragged_pipeline_graph* graph) {
    if (graph == nullptr) return RAGGED_OK;
    ragged_status st = cuda_check(cudaGraphExecDestroy(graph->exec), "cudaGraphExecDestroy");
    const ragged_status st2 = cuda_check(cudaGraphDestroy(graph->graph), "cudaGraphDestroy");
    delete graph;
    return st != RAGGED_OK ? st : st2;
}

}  // extern "C"
