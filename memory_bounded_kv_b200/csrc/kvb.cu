// libkvb: C ABI (include/kvb.h) over the sm_100a kernels. Host code here
// validates arguments, picks the kernel instantiation and launches it on the
// caller's stream; it allocates nothing.
#include <cmath>
#include <cstdint>
#include <map>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <numeric>
#include <tuple>
#include <utility>

#include "../../include/kvb.h"
#include "schedule.h"
#include "asm_lookup.cuh"
#include "asm_planes.cuh"
#include "asm_hier.cuh"
#include "asm_build.cuh"
#include "common.cuh"
#include "compact_blocks.cuh"
#include "decode_attn_tc.cuh"
#include "decode_attn_qb.cuh"
#include "decode_attn_qbt.cuh"
#include "evict_insert.cuh"
#include "merge_states.cuh"
#include "paged.cuh"

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline kvb_status launched() { return cudaGetLastError() == cudaSuccess ? KVB_OK : KVB_ECUDA; }

// Raises a kernel's dynamic shared-memory limit once per (kernel, device):
// later calls (e.g. inside a stream capture) make no runtime call here.
template <typename Kern>
kvb_status set_smem(Kern kern, size_t bytes) {
    if (bytes <= 48 * 1024) return KVB_OK;
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, size_t> granted;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVB_ECUDA;
    std::lock_guard<std::mutex> lock(mu);
    size_t& g = granted[{reinterpret_cast<const void*>(kern), dev}];
    if (g >= bytes) return KVB_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return KVB_ECUDA;
    g = bytes;
    return KVB_OK;
}

// ---- tensor maps (driver entry point, no link against libcuda) -------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 4-D view (d, slot, kv head, sequence) of a [B, Hkv, cap, d] bf16 cache, loaded in boxes of
// 64 dims x `rows` slots with the 128-byte swizzle.
bool make_kv_map(CUtensorMap* map, const void* base, int d, int cap, int Hkv, int Bk, long long kv_sh,
                 long long kv_sb, int rows) {
    EncodeTiledFn fn = encode_tiled();
    if (fn == nullptr) return false;
    const cuuint64_t row_bytes = (cuuint64_t)d * 2;
    const cuuint64_t sh = (Hkv == 1 && kv_sh == 0) ? row_bytes * cap : (cuuint64_t)kv_sh * 2;
    const cuuint64_t sb = (Bk == 1) ? sh * Hkv : (cuuint64_t)kv_sb * 2;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)cap, (cuuint64_t)Hkv, (cuuint64_t)Bk};
    cuuint64_t strides[3] = {row_bytes, sh, sb};
    cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The query rows of the query-batched tensor-core kernel: q [B][Hq][d] with strides q_sb, q_sh
// (elements), boxes of 64 dims x G heads x BQ rows b (128-byte swizzle; rows past B read zeros).
bool make_q_map(CUtensorMap* map, const void* q, int d, int Hq, int B, long long q_sh, long long q_sb, int G,
                int BQ) {
    EncodeTiledFn fn = encode_tiled();
    if (fn == nullptr || q_sh <= 0 || q_sb <= 0) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)Hq, (cuuint64_t)B, 1};
    cuuint64_t strides[3] = {(cuuint64_t)q_sh * 2, (cuuint64_t)q_sb * 2, (cuuint64_t)q_sb * 2 * (cuuint64_t)B};
    cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)BQ, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The queries of the prepared-memory lookup: q [N][H][d] bf16 (d = 128, rows contiguous), boxes of
// 64 dims x 1 head x 128 queries (128-byte swizzle; queries past N read zeros).
bool make_asm_q_map(CUtensorMap* map, const void* q, int N, int H) {
    EncodeTiledFn fn = encode_tiled();
    if (fn == nullptr) return false;
    const int d = kvb::kAsmD;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kvb::kUQ};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Resident CTAs the device holds for a kernel (SMs x blocks per SM), once per (kernel, smem, device).
template <typename Kern>
int resident_ctas(Kern kern, int threads, size_t smem) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, size_t, int>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_tuple(reinterpret_cast<const void*>(kern), smem, dev);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess) return 0;
    const int n = sms * (per_sm > 0 ? per_sm : 1);
    cache[key] = n;
    return n;
}

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream drains; its first instruction waits for that
// kernel's completion (griddepcontrol.wait), so only the launch latency overlaps.
template <typename... KArgs, typename... Args>
kvb_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? KVB_OK : KVB_ECUDA;
}

// The merge of the split states, after either attention kernel.
template <int D>
kvb_status launch_merge(const float* o_part, const float* lse_part, int R, int S, void* o, int o_bf16, float* lse,
                        cudaStream_t st) {
    // few rows with many splits: a CTA per row keeps more loads in flight per row
    if (S > 16 && R < 4 * 148)
        return launch_pdl(kvb::merge_splits_cta_kernel<D>, dim3(R), dim3(256), 0, st, o_part, lse_part, R, S, o,
                          o_bf16, lse);
    return launch_pdl(kvb::merge_splits_kernel<D>, dim3((R + 7) / 8), dim3(256), 0, st, o_part, lse_part, R, S, o,
                      o_bf16, lse);
}

template <int D, int G, bool BIAS, bool INS = false>
kvb_status launch_decode_tc(const kvb::DecodeTcParams& p, const kvb_attn_args* a, cudaStream_t st) {
    using SH = kvb::TcShape<D, G>;
    auto kern = kvb::decode_attn_tc_kernel<D, G, BIAS, false, INS>;
    const size_t smem = SH::SMEM;
    if (set_smem(kern, smem) != KVB_OK) return KVB_ECUDA;
    CUtensorMap mk, mv;
    const int Bk = p.kv_shared ? 1 : a->B;
    if (!make_kv_map(&mk, a->k, D, a->cap, a->Hkv, Bk, a->kv_stride_h, a->kv_stride_b, SH::T) ||
        !make_kv_map(&mv, a->v, D, a->cap, a->Hkv, Bk, a->kv_stride_h, a->kv_stride_b, SH::T))
        return KVB_EINVAL;
    const int slots = resident_ctas(kern, SH::NT, smem);
    if (slots <= 0) return KVB_ECUDA;
    const int grid = kvb::rr_grid(p.units, slots, p.S, p.split_len > 0);
    if (launch_pdl(kern, dim3(grid), dim3(SH::NT), smem, st, p, mk, mv) != KVB_OK) return KVB_ECUDA;
    if (p.S > 1)
        return launch_merge<D>(p.o_part, p.lse_part, a->B * a->Hq, p.S, p.o, p.o_bf16, p.lse, st);
    return KVB_OK;
}

template <int D, int G, bool BIAS>
kvb_status launch_decode_qb(const kvb::DecodeQbParams& p, const kvb_attn_args* a, cudaStream_t st) {
    using SH = kvb::QbShape<D, G>;
    auto kern = kvb::decode_attn_qb_kernel<D, G, BIAS>;
    const size_t smem = SH::SMEM;
    if (set_smem(kern, smem) != KVB_OK) return KVB_ECUDA;
    CUtensorMap mk, mv;
    if (!make_kv_map(&mk, a->k, D, a->cap, a->Hkv, 1, a->kv_stride_h, 0, SH::T) ||
        !make_kv_map(&mv, a->v, D, a->cap, a->Hkv, 1, a->kv_stride_h, 0, SH::T))
        return KVB_EINVAL;
    const int slots = resident_ctas(kern, SH::NT, smem);
    if (slots <= 0) return KVB_ECUDA;
    const int per_cta = (p.units + slots - 1) / slots;
    const int grid = (p.units + per_cta - 1) / per_cta;
    if (launch_pdl(kern, dim3(grid), dim3(SH::NT), smem, st, p, mk, mv) != KVB_OK) return KVB_ECUDA;
    if (p.S > 1)
        return launch_merge<D>(p.o_part, p.lse_part, a->B * a->Hq, p.S, p.o, p.o_bf16, p.lse, st);
    return KVB_OK;
}

// The tensor-core (tcgen05) shared-prefix kernel: 128 query rows per unit.
template <int G, bool BIAS>
kvb_status launch_decode_qbt(kvb::DecodeQbParams p, const kvb_attn_args* a, const CUtensorMap& mq,
                             cudaStream_t st) {
    using SH = kvb::QbtShape<G>;
    auto kern = kvb::decode_attn_qbt_kernel<G, BIAS>;
    const size_t smem = SH::SMEM;
    if (set_smem(kern, smem) != KVB_OK) return KVB_ECUDA;
    CUtensorMap mk, mv;
    if (!make_kv_map(&mk, a->k, SH::D, a->cap, a->Hkv, 1, a->kv_stride_h, 0, SH::T) ||
        !make_kv_map(&mv, a->v, SH::D, a->cap, a->Hkv, 1, a->kv_stride_h, 0, SH::T))
        return KVB_EINVAL;
    p.blocks = (a->B + SH::BQ - 1) / SH::BQ;
    const long long units = (long long)p.blocks * a->Hkv * a->num_splits;
    if (units > 0x7fffffffLL) return KVB_EINVAL;
    p.units = (int)units;
    const int slots = resident_ctas(kern, SH::NT, smem);
    if (slots <= 0) return KVB_ECUDA;
    const int per_cta = (p.units + slots - 1) / slots;
    const int grid = (p.units + per_cta - 1) / per_cta;
    if (launch_pdl(kern, dim3(grid), dim3(SH::NT), smem, st, p, mk, mv, mq) != KVB_OK) return KVB_ECUDA;
    if (p.S > 1)
        return launch_merge<128>(p.o_part, p.lse_part, a->B * a->Hq, p.S, p.o, p.o_bf16, p.lse, st);
    return KVB_OK;
}

template <int D>
kvb_status qb_dispatch(const kvb::DecodeQbParams& p, const kvb_attn_args* a, int G, bool bias, cudaStream_t st) {
    // enough query rows to fill the 128 rows of a tcgen05 tile (and queries a tensor map can
    // describe): the tensor-core kernel
    CUtensorMap mq;
    if (D == 128 && (G == 2 || G == 4 || G == 8) && (long long)a->B * G >= 64 &&
        make_q_map(&mq, a->q, D, a->Hq, a->B, a->q_stride_h, a->q_stride_b, G, 128 / G)) {
        switch (G) {
            case 2: return bias ? launch_decode_qbt<2, true>(p, a, mq, st) : launch_decode_qbt<2, false>(p, a, mq, st);
            case 4: return bias ? launch_decode_qbt<4, true>(p, a, mq, st) : launch_decode_qbt<4, false>(p, a, mq, st);
            default: return bias ? launch_decode_qbt<8, true>(p, a, mq, st) : launch_decode_qbt<8, false>(p, a, mq, st);
        }
    }
    switch (G) {
        case 1: return bias ? launch_decode_qb<D, 1, true>(p, a, st) : launch_decode_qb<D, 1, false>(p, a, st);
        case 2: return bias ? launch_decode_qb<D, 2, true>(p, a, st) : launch_decode_qb<D, 2, false>(p, a, st);
        case 4: return bias ? launch_decode_qb<D, 4, true>(p, a, st) : launch_decode_qb<D, 4, false>(p, a, st);
        case 8: return bias ? launch_decode_qb<D, 8, true>(p, a, st) : launch_decode_qb<D, 8, false>(p, a, st);
        default: return KVB_EINVAL;
    }
}

// Attention over a paged cache: the tensor maps cover the page pool ([pages * T rows, d]).
template <int D, int G, bool BIAS>
kvb_status launch_decode_paged(const kvb::DecodeTcParams& p, const kvb_paged_cache* c, int Hq, cudaStream_t st) {
    using SH = kvb::TcShape<D, G>;
    static_assert(SH::T == kvb::kPageSlots, "a tile is a page");
    auto kern = kvb::decode_attn_tc_kernel<D, G, BIAS, true>;
    const size_t smem = SH::SMEM;
    if (set_smem(kern, smem) != KVB_OK) return KVB_ECUDA;
    CUtensorMap mk, mv;
    const int rows = c->num_pages * kvb::kPageSlots;
    if (!make_kv_map(&mk, c->k_pages, D, rows, 1, 1, 0, 0, SH::T) ||
        !make_kv_map(&mv, c->v_pages, D, rows, 1, 1, 0, 0, SH::T))
        return KVB_EINVAL;
    const int slots = resident_ctas(kern, SH::NT, smem);
    if (slots <= 0) return KVB_ECUDA;
    const int grid = kvb::rr_grid(p.units, slots, p.S, p.split_len > 0);
    if (launch_pdl(kern, dim3(grid), dim3(SH::NT), smem, st, p, mk, mv) != KVB_OK) return KVB_ECUDA;
    if (p.S > 1) return launch_merge<D>(p.o_part, p.lse_part, c->B * Hq, p.S, p.o, p.o_bf16, p.lse, st);
    return KVB_OK;
}

template <int D>
kvb_status paged_dispatch(const kvb::DecodeTcParams& p, const kvb_paged_cache* c, int Hq, int G, bool bias,
                          cudaStream_t st) {
    switch (G) {
        case 1: return bias ? launch_decode_paged<D, 1, true>(p, c, Hq, st) : launch_decode_paged<D, 1, false>(p, c, Hq, st);
        case 2: return bias ? launch_decode_paged<D, 2, true>(p, c, Hq, st) : launch_decode_paged<D, 2, false>(p, c, Hq, st);
        case 4: return bias ? launch_decode_paged<D, 4, true>(p, c, Hq, st) : launch_decode_paged<D, 4, false>(p, c, Hq, st);
        case 8: return bias ? launch_decode_paged<D, 8, true>(p, c, Hq, st) : launch_decode_paged<D, 8, false>(p, c, Hq, st);
        default: return KVB_EINVAL;
    }
}

// Host checks shared by the paged entry points; fills the kernels' view of the cache.
kvb_status paged_view(const kvb_paged_cache* c, kvb::PagedCache* out) {
    if (c == nullptr) return KVB_EINVAL;
    if (c->B < 1 || c->Hkv < 1 || c->d < 8 || c->d > 1024 || (c->d % 8) || c->max_pages < 1 || c->num_pages < 1)
        return KVB_EINVAL;
    if ((long long)c->B * c->Hkv > 0x7fffffffLL || (long long)c->max_pages * kvb::kPageSlots > 0x7fffffffLL ||
        (long long)c->num_pages * kvb::kPageSlots > 0x7fffffffLL)
        return KVB_EINVAL;
    if (!c->k_pages || !c->v_pages || !c->pos_pages || !c->table || !c->len || !c->free_pages || !c->free_count)
        return KVB_EINVAL;
    if (!aligned16(c->k_pages) || !aligned16(c->v_pages) || !aligned16(c->pos_pages) ||
        (c->log_beta_pages && !aligned16(c->log_beta_pages)))
        return KVB_EINVAL;
    *out = kvb::PagedCache{c->k_pages, c->v_pages, c->log_beta_pages, c->pos_pages, c->table, c->len,
                           c->free_pages, c->free_count, c->Hkv, c->d, c->max_pages, c->num_pages};
    return KVB_OK;
}

template <int D, int G, bool INS>
kvb_status tc_bias(const kvb::DecodeTcParams& p, const kvb_attn_args* a, bool bias, cudaStream_t st) {
    return bias ? launch_decode_tc<D, G, true, INS>(p, a, st) : launch_decode_tc<D, G, false, INS>(p, a, st);
}

template <int D, bool INS = false>
kvb_status tc_g(const kvb::DecodeTcParams& p, const kvb_attn_args* a, int G, bool bias, cudaStream_t st) {
    switch (G) {
        case 1: return tc_bias<D, 1, INS>(p, a, bias, st);
        case 2: return tc_bias<D, 2, INS>(p, a, bias, st);
        case 4: return tc_bias<D, 4, INS>(p, a, bias, st);
        case 8: return tc_bias<D, 8, INS>(p, a, bias, st);
        default: return KVB_EINVAL;
    }
}

// ---- fixed scratch of kvb_decode_attn_noalloc ------------------------------
// The split states of the no-allocation entry point live here instead of in
// caller memory. Host code must not use the symbol itself
// as a device address: it is a host-side stand-in. The device address is
// looked up once per device with cudaGetSymbolAddress (that device current).
static __device__ __align__(256) unsigned char g_noalloc_scratch[KVB_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

kvb_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVB_ECUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return KVB_ECUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return KVB_OK;
}

inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Test hook of kvb_test_withhold_next_decode: the wait limit (ns) the next decode launch uses
// with its producers withholding their copies; 0 = off. Taken (and cleared) by one call.
std::atomic<unsigned long long> g_withhold_next{0};

}  // namespace

extern "C" {

int32_t kvb_abi_version(void) { return 7; }

kvb_status kvb_test_withhold_next_decode(uint64_t wait_limit_ns) {
    if (wait_limit_ns < 1000ull || wait_limit_ns > 1000000000ull) return KVB_EINVAL;
    g_withhold_next.store(wait_limit_ns);
    return KVB_OK;
}

const char* kvb_status_str(kvb_status s) {
    switch (s) {
        case KVB_OK: return "ok";
        case KVB_EINVAL: return "invalid argument";
        case KVB_ECUDA: return "CUDA error";
        case KVB_EDEVICE: return "inconsistent device data";
        default: return "unknown status";
    }
}

kvb_status kvb_get_error(kvb_stream stream, uint32_t* bits) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVB_ECUDA;
    unsigned w = 0;
    if (cudaMemcpyFromSymbol(&w, kvb::g_error_word, sizeof w) != cudaSuccess) return KVB_ECUDA;
    if (bits != nullptr) *bits = w;
    if (w == 0) return KVB_OK;
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(kvb::g_error_word, &zero, sizeof zero) != cudaSuccess) return KVB_ECUDA;
    return KVB_EDEVICE;
}

}  // extern "C"

namespace {

// The host checks of kvb_decode_attn (and kvb_decode_step), and the kernel parameters.
kvb_status attn_params(const kvb_attn_args* a, kvb::DecodeTcParams* out, int* G_out) {
    if (a == nullptr) return KVB_EINVAL;
    if (a->B < 1 || a->Hq < 1 || a->Hkv < 1 || a->cap < 1) return KVB_EINVAL;
    if (a->d != 64 && a->d != 128) return KVB_EINVAL;
    if (a->Hq % a->Hkv != 0) return KVB_EINVAL;
    const int G = a->Hq / a->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return KVB_EINVAL;
    if (a->num_splits < 1 || a->num_splits > 1024 || a->split_len < 0) return KVB_EINVAL;
    if (a->B > 65535 || a->Hkv > 65535) return KVB_EINVAL;
    if ((long long)a->B * a->Hq > 0x7fffffffLL) return KVB_EINVAL;   // rows of the merge and the outputs
    if (!std::isfinite(a->scale)) return KVB_EINVAL;
    if (!a->q || !a->k || !a->v || !a->len || !a->o) return KVB_EINVAL;
    if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v)) return KVB_EINVAL;
    if (!aligned16(a->o) || (a->o_part != nullptr && !aligned16(a->o_part))) return KVB_EINVAL;
    if (a->q_stride_b < 0 || a->q_stride_h < 0 || a->kv_stride_b < 0 || a->kv_stride_h < 0) return KVB_EINVAL;
    if ((a->q_stride_b % 8) || (a->q_stride_h % 8) || (a->kv_stride_b % 8) || (a->kv_stride_h % 8)) return KVB_EINVAL;
    const bool bias = a->log_beta != nullptr;
    if (bias && (!a->pos || !a->t)) return KVB_EINVAL;
    if (bias && (a->meta_stride_b < 0 || a->meta_stride_h < 0)) return KVB_EINVAL;
    if (a->evict_cand != nullptr &&
        (!a->pos || !a->t || a->meta_stride_b < 0 || a->meta_stride_h < 0 ||
         (reinterpret_cast<uintptr_t>(a->evict_cand) & 15u)))
        return KVB_EINVAL;
    if (a->o_dtype != KVB_OUT_F32 && a->o_dtype != KVB_OUT_BF16) return KVB_EINVAL;
    if (a->num_splits > 1 && (!a->o_part || !a->lse_part)) return KVB_EINVAL;
    if ((a->o_part == nullptr) != (a->lse_part == nullptr)) return KVB_EINVAL;

    if (a->Hkv > 1 && a->kv_stride_h == 0) return KVB_EINVAL;
    const long long units = (long long)a->B * a->Hkv * a->num_splits;
    if (units > 0x7fffffffLL) return KVB_EINVAL;

    kvb::DecodeTcParams& p = *out;
    p = kvb::DecodeTcParams{};
    p.q = a->q; p.q_sb = a->q_stride_b; p.q_sh = a->q_stride_h;
    p.lb = a->log_beta; p.pos = a->pos; p.m_sb = a->meta_stride_b; p.m_sh = a->meta_stride_h;
    p.len = a->len; p.t = a->t;
    p.Hq = a->Hq; p.Hkv = a->Hkv; p.cap = a->cap; p.S = a->num_splits; p.split_len = a->split_len;
    p.units = (int)units;
    p.kv_shared = (a->kv_stride_b == 0 && a->B > 1) ? 1 : 0;
    const double scale = (a->scale == 0.0f) ? 1.0 / std::sqrt((double)a->d) : (double)a->scale;
    p.scale = (float)scale;
    p.o_part = a->o_part; p.lse_part = a->lse_part;
    p.o = a->o; p.o_bf16 = (a->o_dtype == KVB_OUT_BF16); p.lse = a->lse;
    p.cand = static_cast<kvb::EvictCand*>(a->evict_cand);
    p.wait_ns = 1000000000ull;
    p.withhold = 0;
    *G_out = G;
    return KVB_OK;
}

}  // namespace

extern "C" {

kvb_status kvb_decode_attn(const kvb_attn_args* a, kvb_stream stream) {
    kvb::DecodeTcParams p;
    int G = 0;
    const kvb_status chk = attn_params(a, &p, &G);
    if (chk != KVB_OK) return chk;
    const bool bias = a->log_beta != nullptr;
    if (g_withhold_next.load(std::memory_order_relaxed) != 0) {
        const unsigned long long lim = g_withhold_next.exchange(0);
        if (lim != 0) {
            p.wait_ns = lim;
            p.withhold = 1;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // many rows over one shared cache (and shared log beta / pos): the query-batched kernel reads
    // every K/V tile once per block of rows. Needs split boundaries common to all rows (a fixed
    // split length, or one split) and no eviction candidates (they are per row).
    const bool meta_shared = (a->log_beta == nullptr && a->pos == nullptr) || a->meta_stride_b == 0;
    if (p.kv_shared && meta_shared && a->evict_cand == nullptr && (a->num_splits == 1 || a->split_len > 0)) {
        kvb::DecodeQbParams q;
        q.q = a->q; q.q_sb = a->q_stride_b; q.q_sh = a->q_stride_h;
        q.lb = a->log_beta; q.pos = a->pos; q.m_sh = a->meta_stride_h;
        q.len = a->len; q.t = a->t;
        q.B = a->B; q.Hq = a->Hq; q.Hkv = a->Hkv; q.cap = a->cap; q.S = a->num_splits; q.split_len = a->split_len;
        const int BQ = 16 / G;
        q.blocks = (a->B + BQ - 1) / BQ;
        const long long qunits = (long long)q.blocks * a->Hkv * a->num_splits;
        if (qunits > 0x7fffffffLL) return KVB_EINVAL;
        q.units = (int)qunits;
        q.scale = p.scale;
        q.o_part = a->o_part; q.lse_part = a->lse_part;
        q.o = a->o; q.o_bf16 = p.o_bf16; q.lse = a->lse;
        q.wait_ns = p.wait_ns; q.withhold = p.withhold;
        return a->d == 128 ? qb_dispatch<128>(q, a, G, bias, st) : qb_dispatch<64>(q, a, G, bias, st);
    }
    return a->d == 128 ? tc_g<128>(p, a, G, bias, st) : tc_g<64>(p, a, G, bias, st);
}

kvb_status kvb_decode_step(const kvb_attn_args* a, const uint16_t* k_new, const uint16_t* v_new,
                           const float* log_beta_new, int32_t M, const kvb_evict_cand* cand_in, int32_t* victim,
                           kvb_stream stream) {
    kvb::DecodeTcParams p;
    int G = 0;
    const kvb_status chk = attn_params(a, &p, &G);
    if (chk != KVB_OK) return chk;
    const bool bias = a->log_beta != nullptr;
    // one cache row per (b, g): no batch stride 0; the records in and out are different arrays
    if (a->kv_stride_b == 0 || a->meta_stride_b == 0 || !a->pos || !a->t || !a->evict_cand || !cand_in) return KVB_EINVAL;
    if (cand_in == a->evict_cand || (reinterpret_cast<uintptr_t>(cand_in) & 15u)) return KVB_EINVAL;
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return KVB_EINVAL;
    if (bias != (log_beta_new != nullptr)) return KVB_EINVAL;
    if (M < 1 || M > a->cap) return KVB_EINVAL;
    p.k_w = const_cast<uint16_t*>(a->k);
    p.v_w = const_cast<uint16_t*>(a->v);
    p.kv_sb = a->kv_stride_b;
    p.kv_sh = a->kv_stride_h;
    p.lb_w = const_cast<float*>(a->log_beta);
    p.pos_w = const_cast<int32_t*>(a->pos);
    p.k_new = k_new;
    p.v_new = v_new;
    p.lb_new = log_beta_new;
    p.cand_in = reinterpret_cast<const kvb::EvictCand*>(cand_in);
    p.victim = victim;
    p.M = M;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return a->d == 128 ? tc_g<128, true>(p, a, G, bias, st) : tc_g<64, true>(p, a, G, bias, st);
}

kvb_status kvb_decode_attn_noalloc(const kvb_attn_args* a, kvb_stream stream) {
    if (a == nullptr) return KVB_EINVAL;
    if (a->o_part != nullptr || a->lse_part != nullptr || a->counters != nullptr) return KVB_EINVAL;
    kvb_attn_args b = *a;
    if (a->num_splits > 1) {
        if (a->B < 1 || a->Hq < 1 || a->Hkv < 1 || (a->d != 64 && a->d != 128) || a->num_splits > 1024 ||
            a->B > 65535 || a->Hkv > 65535 || a->Hq > 65535)
            return KVB_EINVAL;
        const size_t rows = (size_t)a->B * a->Hq * a->num_splits;
        const size_t o_off = round256(rows * sizeof(float));
        const size_t need = o_off + rows * a->d * sizeof(float);
        if (need > (size_t)KVB_NOALLOC_SCRATCH_BYTES) return KVB_EINVAL;
        void* base = nullptr;
        const kvb_status st = noalloc_scratch(&base);
        if (st != KVB_OK) return st;
        // every call writes all the split states it reads back: nothing needs clearing
        unsigned char* s = static_cast<unsigned char*>(base);
        b.lse_part = reinterpret_cast<float*>(s);
        b.o_part = reinterpret_cast<float*>(s + o_off);
    }
    return kvb_decode_attn(&b, stream);
}

kvb_status kvb_merge_states(const float* o_in, const float* lse_in, int64_t o_stride_n, int64_t o_stride_r,
                            int64_t lse_stride_n, int64_t lse_stride_r, int32_t n, int32_t R, int32_t d,
                            float* o_out, float* lse_out, kvb_stream stream) {
    if (!o_in || !lse_in || !o_out) return KVB_EINVAL;
    if (n < 1 || R < 0 || d < 1 || d > 1024) return KVB_EINVAL;
    if (R == 0) return KVB_OK;
    kvb::MergeParams p{o_in, lse_in, o_stride_n, o_stride_r, lse_stride_n, lse_stride_r, n, R, d, o_out, lse_out};
    const bool vec4 = (d % 4 == 0) && aligned16(o_in) && aligned16(o_out) && (o_stride_n % 4 == 0) &&
                      (o_stride_r % 4 == 0);
    const dim3 grid((R + 7) / 8);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (vec4) {
        kvb::merge_states_kernel<true><<<grid, 256, 0, st>>>(p);
    } else {
        kvb::merge_states_kernel<false><<<grid, 256, 0, st>>>(p);
    }
    return launched();
}

kvb_status kvb_evict_insert(uint16_t* k, uint16_t* v, float* log_beta, int32_t* pos, int32_t* len,
                            const uint16_t* k_new, const uint16_t* v_new, const float* log_beta_new,
                            const int32_t* t, int32_t B, int32_t Hkv, int32_t d, int32_t cap, int32_t M,
                            int32_t* victim, const void* cand, int32_t cand_n, kvb_stream stream) {
    if (B < 1 || Hkv < 1 || d < 8 || d > 1024 || (d % 8) || cap < 1 || M < 1 || M > cap) return KVB_EINVAL;
    if ((long long)B * Hkv > 0x7fffffffLL) return KVB_EINVAL;
    if (!pos || !len || !t) return KVB_EINVAL;
    if ((k_new == nullptr) != (v_new == nullptr)) return KVB_EINVAL;
    if (k_new && (!k || !v || !aligned16(k) || !aligned16(v) || !aligned16(k_new) || !aligned16(v_new)))
        return KVB_EINVAL;
    if (log_beta && !log_beta_new) return KVB_EINVAL;
    if (cand != nullptr && (cand_n < 1 || cand_n > 1024 || (reinterpret_cast<uintptr_t>(cand) & 15u))) return KVB_EINVAL;
    const int vec4 = (cap % 4 == 0) && aligned16(pos) && (log_beta == nullptr || aligned16(log_beta)) ? 1 : 0;
    kvb::EvictParams p{k, v, log_beta, pos, len, k_new, v_new, log_beta_new, t, Hkv, d, cap, M, victim, vec4,
                       static_cast<const kvb::EvictCand*>(cand), cand_n};
    return launch_pdl(kvb::evict_insert_kernel<256>, dim3(B * Hkv), dim3(256), 0, static_cast<cudaStream_t>(stream),
                      p);
}

kvb_status kvb_compact_blocks(uint16_t* k, uint16_t* v, int32_t* pos, float* log_beta, int32_t* len,
                              const int32_t* rm_start, const int32_t* rm_len, int32_t B, int32_t Hkv,
                              int32_t d, int32_t cap, kvb_stream stream) {
    if (B < 1 || Hkv < 1 || d < 8 || d > 1024 || (d % 8) || cap < 1) return KVB_EINVAL;
    if ((long long)B * Hkv > 0x7fffffffLL) return KVB_EINVAL;
    if (!k || !v || !pos || !len || !rm_start || !rm_len) return KVB_EINVAL;
    if (!aligned16(k) || !aligned16(v)) return KVB_EINVAL;
    const int row_bytes = 2 * d * 2 + 8;
    int W = 32768 / row_bytes;
    W = W < 1 ? 1 : (W > 64 ? 64 : W);
    kvb::CompactParams p{k, v, pos, log_beta, len, rm_start, rm_len, Hkv, d, cap, W};
    const size_t smem = (size_t)W * row_bytes;
    kvb::compact_blocks_kernel<256><<<B * Hkv, 256, smem, static_cast<cudaStream_t>(stream)>>>(p);
    return launched();
}

kvb_status kvb_paged_reset(const kvb_paged_cache* c, kvb_stream stream) {
    kvb::PagedCache pc;
    if (paged_view(c, &pc) != KVB_OK) return KVB_EINVAL;
    const long long rows = (long long)c->B * c->Hkv;
    const long long n = std::max((long long)c->num_pages, rows * c->max_pages);
    kvb::paged_reset_kernel<<<(unsigned)std::min<long long>((n + 255) / 256, 65535), 256, 0,
                              static_cast<cudaStream_t>(stream)>>>(pc, c->B);
    return launched();
}

kvb_status kvb_paged_evict_insert(const kvb_paged_cache* c, const uint16_t* k_new, const uint16_t* v_new,
                                  const float* log_beta_new, const int32_t* t, int32_t M, int32_t* victim,
                                  const void* cand, int32_t cand_n, kvb_stream stream) {
    kvb::PagedCache pc;
    if (paged_view(c, &pc) != KVB_OK) return KVB_EINVAL;
    if (!t || M < 1 || (long long)M > (long long)c->max_pages * kvb::kPageSlots) return KVB_EINVAL;
    if ((k_new == nullptr) != (v_new == nullptr)) return KVB_EINVAL;
    if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return KVB_EINVAL;
    if (c->log_beta_pages && !log_beta_new) return KVB_EINVAL;
    if (cand != nullptr && (cand_n < 1 || cand_n > 1024 || (reinterpret_cast<uintptr_t>(cand) & 15u))) return KVB_EINVAL;
    kvb::PagedEvictParams p{pc, k_new, v_new, log_beta_new, t, M, victim, static_cast<const kvb::EvictCand*>(cand),
                            cand_n};
    return launch_pdl(kvb::paged_evict_insert_kernel<256>, dim3(c->B * c->Hkv), dim3(256), 0,
                      static_cast<cudaStream_t>(stream), p);
}

kvb_status kvb_paged_compact_blocks(const kvb_paged_cache* c, const int32_t* rm_start, const int32_t* rm_len,
                                    kvb_stream stream) {
    kvb::PagedCache pc;
    if (paged_view(c, &pc) != KVB_OK) return KVB_EINVAL;
    if (!rm_start || !rm_len) return KVB_EINVAL;
    const int row_bytes = 2 * c->d * 2 + 8;
    int W = 32768 / row_bytes;
    W = W < 1 ? 1 : (W > 64 ? 64 : W);
    kvb::PagedCompactParams p{pc, rm_start, rm_len, W};
    const size_t smem = (size_t)W * row_bytes;
    return launch_pdl(kvb::paged_compact_kernel<256>, dim3(c->B * c->Hkv), dim3(256), smem,
                      static_cast<cudaStream_t>(stream), p);
}

kvb_status kvb_paged_decode_attn(const kvb_paged_cache* c, const uint16_t* q, const int32_t* t, int32_t Hq,
                                 float scale, int32_t num_splits, int32_t split_len, float* o_part, float* lse_part,
                                 void* o, int32_t o_dtype, float* lse, void* evict_cand, kvb_stream stream) {
    kvb::PagedCache pc;
    if (paged_view(c, &pc) != KVB_OK) return KVB_EINVAL;
    if (c->d != 64 && c->d != 128) return KVB_EINVAL;
    if (Hq < 1 || Hq % c->Hkv != 0) return KVB_EINVAL;
    const int G = Hq / c->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return KVB_EINVAL;
    if (c->B > 65535 || c->Hkv > 65535 || (long long)c->B * Hq > 0x7fffffffLL) return KVB_EINVAL;
    if (num_splits < 1 || num_splits > 1024 || split_len < 0) return KVB_EINVAL;
    // every split starts on a page: one split, or a split length that is a multiple of a page
    if (num_splits > 1 && (split_len == 0 || split_len % kvb::kPageSlots != 0)) return KVB_EINVAL;
    if (!std::isfinite(scale) || !q || !o || !aligned16(q) || !aligned16(o)) return KVB_EINVAL;
    if (o_part != nullptr && !aligned16(o_part)) return KVB_EINVAL;
    const bool bias = c->log_beta_pages != nullptr;
    if ((bias || evict_cand) && !t) return KVB_EINVAL;
    if (evict_cand && (reinterpret_cast<uintptr_t>(evict_cand) & 15u)) return KVB_EINVAL;
    if (o_dtype != KVB_OUT_F32 && o_dtype != KVB_OUT_BF16) return KVB_EINVAL;
    if (num_splits > 1 && (!o_part || !lse_part)) return KVB_EINVAL;
    if ((o_part == nullptr) != (lse_part == nullptr)) return KVB_EINVAL;
    const long long units = (long long)c->B * c->Hkv * num_splits;
    if (units > 0x7fffffffLL) return KVB_EINVAL;
    kvb::DecodeTcParams p{};
    p.q = q; p.q_sb = (long long)Hq * c->d; p.q_sh = c->d;
    p.lb = c->log_beta_pages; p.pos = c->pos_pages; p.m_sb = 0; p.m_sh = 0;
    p.len = c->len; p.t = t;
    p.Hq = Hq; p.Hkv = c->Hkv; p.cap = c->max_pages * kvb::kPageSlots; p.S = num_splits; p.split_len = split_len;
    p.units = (int)units;
    p.kv_shared = 0;
    p.scale = (scale == 0.0f) ? (float)(1.0 / std::sqrt((double)c->d)) : scale;
    p.o_part = o_part; p.lse_part = lse_part;
    p.o = o; p.o_bf16 = (o_dtype == KVB_OUT_BF16); p.lse = lse;
    p.cand = static_cast<kvb::EvictCand*>(evict_cand);
    p.wait_ns = 1000000000ull;
    p.withhold = 0;
    p.table = c->table; p.max_pages = c->max_pages; p.num_pages = c->num_pages;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return c->d == 128 ? paged_dispatch<128>(p, c, Hq, G, bias, st) : paged_dispatch<64>(p, c, Hq, G, bias, st);
}

size_t kvb_asm_workspace_bytes(int32_t N, int32_t H, int32_t K) {
    if (N < 1 || H < 1 || K < 1) return 0;
    return (size_t)kvb::asm_ksplit(K) * N * H * sizeof(unsigned long long);
}

kvb_status kvb_asm_lookup_merge_grouped(const uint16_t* q, const float* qbar, const uint16_t* abar,
                                        const float* log_zbar, const float* o_self, const float* lse_self,
                                        int32_t N, int32_t H, int32_t H_tables, int32_t K, int32_t d, int32_t* idx,
                                        float* o, float* lse, void* workspace, size_t workspace_bytes,
                                        kvb_stream stream) {
    if (d != kvb::kAsmD || N < 1 || H < 1 || K < 1 || H > 65535) return KVB_EINVAL;
    if (H_tables < 1 || H % H_tables != 0) return KVB_EINVAL;
    if (!q || !qbar || !workspace) return KVB_EINVAL;
    if (o == nullptr) {   // assignment only
        if (idx == nullptr) return KVB_EINVAL;
    } else if (!abar || !log_zbar || !o_self || !lse_self || !aligned16(abar) || !aligned16(o_self) ||
               !aligned16(o)) {
        return KVB_EINVAL;
    }
    if (!aligned16(q) || !aligned16(qbar) || !aligned16(workspace)) return KVB_EINVAL;
    if (workspace_bytes < kvb_asm_workspace_bytes(N, H, K)) return KVB_EINVAL;
    const int qtiles = (N + kvb::kUMT * kvb::kUQ - 1) / (kvb::kUMT * kvb::kUQ);
    const long long items = (long long)H * qtiles * kvb::asm_ksplit(K);
    if (items > (1ll << 30)) return KVB_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (set_smem(kvb::asm_score_umma_kernel, kvb::kUSmem) != KVB_OK) return KVB_ECUDA;
    // persistent: one CTA per SM (the shared memory allows no second), items split evenly
    const int slots = resident_ctas(kvb::asm_score_umma_kernel, kvb::kUThreads, kvb::kUSmem);
    if (slots < 1) return KVB_ECUDA;
    const int per_cta = (int)((items + slots - 1) / slots);
    const int grid = (int)((items + per_cta - 1) / per_cta);
    kvb::AsmParams p{q, qbar, abar, log_zbar, o_self, lse_self, N, H, K, kvb::asm_ksplit(K), kvb::asm_kchunk(K),
                     qtiles, per_cta, idx, o, lse, static_cast<unsigned long long*>(workspace), H / H_tables};
    kvb::asm_score_umma_kernel<<<grid, kvb::kUThreads, kvb::kUSmem, st>>>(p);
    if (launched() != KVB_OK) return KVB_ECUDA;
    const long long rows = (long long)N * H;
    // programmatic launch: the merge's CTAs wait on the device for the lookup instead of being launched after it
    return launch_pdl(kvb::asm_merge_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, st, p);
}

size_t kvb_asm_planes_bytes(int32_t H_tables, int32_t K) {
    if (H_tables < 1 || K < 1) return 0;
    return (size_t)H_tables * kvb::asm_plane_tiles(K) * kvb::kPImg;
}

kvb_status kvb_asm_prepare(const float* qbar, int32_t H_tables, int32_t K, int32_t d, void* planes,
                           size_t planes_bytes, kvb_stream stream) {
    if (d != kvb::kAsmD || H_tables < 1 || K < 1 || !qbar || !planes) return KVB_EINVAL;
    if (!aligned16(qbar) || !aligned16(planes) || planes_bytes < kvb_asm_planes_bytes(H_tables, K)) return KVB_EINVAL;
    const long long rows = (long long)H_tables * (long long)kvb::asm_plane_tiles(K) * kvb::kPT;
    if ((rows + 7) / 8 > 0x7fffffffLL) return KVB_EINVAL;
    kvb::asm_prepare_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        qbar, H_tables, K, static_cast<unsigned char*>(planes));
    return launched();
}

kvb_status kvb_asm_lookup_merge_planes(const uint16_t* q, const void* planes, size_t planes_bytes,
                                       const uint16_t* abar, const float* log_zbar, const float* o_self,
                                       const float* lse_self, int32_t N, int32_t H, int32_t H_tables, int32_t K,
                                       int32_t d, int32_t* idx, float* o, float* lse, void* workspace,
                                       size_t workspace_bytes, kvb_stream stream) {
    if (d != kvb::kAsmD || N < 1 || H < 1 || K < 1 || H > 65535) return KVB_EINVAL;
    if (H_tables < 1 || H % H_tables != 0) return KVB_EINVAL;
    if (!q || !planes || !workspace) return KVB_EINVAL;
    if (planes_bytes < kvb_asm_planes_bytes(H_tables, K)) return KVB_EINVAL;
    if (o == nullptr) {   // assignment only
        if (idx == nullptr) return KVB_EINVAL;
    } else if (!abar || !log_zbar || !o_self || !lse_self || !aligned16(abar) || !aligned16(o_self) ||
               !aligned16(o)) {
        return KVB_EINVAL;
    }
    if (!aligned16(q) || !aligned16(planes) || !aligned16(workspace)) return KVB_EINVAL;
    if (workspace_bytes < kvb_asm_workspace_bytes(N, H, K)) return KVB_EINVAL;
    const int qtiles = (N + kvb::kUMT * kvb::kUQ - 1) / (kvb::kUMT * kvb::kUQ);
    if ((long long)H * qtiles > (1ll << 30)) return KVB_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (set_smem(kvb::asm_score_planes_kernel, kvb::kPSmem) != KVB_OK) return KVB_ECUDA;
    const int slots = resident_ctas(kvb::asm_score_planes_kernel, kvb::kPThreads, kvb::kPSmem);
    if (slots < 1) return KVB_ECUDA;
    // ranges of whole 128-centroid tiles, as many per (head, query block) as there are CTAs for it
    const int kchunk = kvb::asm_planes_kchunk(K, H * qtiles, slots);
    const int ksplit = (K + kchunk - 1) / kchunk;   // <= asm_ksplit(K): the workspace holds it
    const long long items = (long long)H * qtiles * ksplit;
    if (items > (1ll << 30)) return KVB_EINVAL;
    const int per_cta = (int)((items + slots - 1) / slots);
    const int grid = (int)((items + per_cta - 1) / per_cta);
    kvb::AsmPlanesParams pp;
    pp.a = kvb::AsmParams{q, nullptr, abar, log_zbar, o_self, lse_self, N, H, K, ksplit, kchunk, qtiles, per_cta, idx,
                          o, lse, static_cast<unsigned long long*>(workspace), H / H_tables};
    pp.planes = static_cast<const unsigned char*>(planes);
    pp.wait_ns = 1000000000ull;
    CUtensorMap mq;
    if (!make_asm_q_map(&mq, q, N, H)) return KVB_EINVAL;
    kvb::asm_score_planes_kernel<<<grid, kvb::kPThreads, kvb::kPSmem, st>>>(pp, mq);
    if (launched() != KVB_OK) return KVB_ECUDA;
    const long long rows = (long long)N * H;
    return launch_pdl(kvb::asm_merge_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, st, pp.a);
}

kvb_status kvb_asm_lookup_merge(const uint16_t* q, const float* qbar, const uint16_t* abar, const float* log_zbar,
                                const float* o_self, const float* lse_self, int32_t N, int32_t H, int32_t K,
                                int32_t d, int32_t* idx, float* o, float* lse, void* workspace,
                                size_t workspace_bytes, kvb_stream stream) {
    return kvb_asm_lookup_merge_grouped(q, qbar, abar, log_zbar, o_self, lse_self, N, H, H, K, d, idx, o, lse,
                                        workspace, workspace_bytes, stream);
}

size_t kvb_asm_hier_workspace_bytes(int32_t N, int32_t H, int32_t m) {
    if (N < 1 || H < 1 || m < 1) return 0;
    return (size_t)N * H * m * (sizeof(unsigned long long) + sizeof(int32_t));
}

kvb_status kvb_asm_hier_lookup_merge(const uint16_t* q, const float* qhat, const int32_t* offsets,
                                     const int32_t* members, const float* qbar, const uint16_t* abar,
                                     const float* log_zbar, const float* o_self, const float* lse_self,
                                     int32_t N, int32_t H, int32_t K, int32_t C, int32_t m, int32_t d,
                                     int32_t* idx, float* o, float* lse, void* workspace,
                                     size_t workspace_bytes, kvb_stream stream) {
    if (d != kvb::kHierD || N < 1 || H < 1 || K < 1 || C < 1 || C > kvb::kHierMaxC || m < 1 ||
        m > kvb::kHierMaxM)
        return KVB_EINVAL;
    if (!q || !qhat || !offsets || !members || !qbar || !abar || !log_zbar || !o_self || !lse_self || !o ||
        !workspace)
        return KVB_EINVAL;
    if (!aligned16(q) || !aligned16(qhat) || !aligned16(qbar) || !aligned16(abar) || !aligned16(o_self) ||
        !aligned16(o) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(offsets) & 3) ||
        (reinterpret_cast<uintptr_t>(members) & 3))
        return KVB_EINVAL;
    if (workspace_bytes < kvb_asm_hier_workspace_bytes(N, H, m)) return KVB_EINVAL;
    const long long nh = (long long)N * H;
    if (nh * m > (1ll << 31) - 1) return KVB_EINVAL;   // one CTA per (selected cluster, query, head)
    auto* keys = static_cast<unsigned long long*>(workspace);
    auto* sel = reinterpret_cast<int32_t*>(keys + nh * m);
    kvb::AsmHierParams hp{q, qhat, offsets, members, qbar, N, H, K, C, m, sel, keys};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // three launches chained by programmatic dependent launch: each waits (griddepcontrol.wait)
    // for its predecessor's results, only the launch latency overlaps
    const size_t smem = kvb::hier_select_smem(C);
    if (launch_pdl(kvb::asm_hier_select_kernel, dim3((unsigned)nh), dim3(256), smem, st, hp) != KVB_OK)
        return KVB_ECUDA;
    if (launch_pdl(kvb::asm_hier_score_kernel, dim3((unsigned)(nh * m)), dim3(256), 0, st, hp) != KVB_OK)
        return KVB_ECUDA;
    // reduction over the m selected clusters' keys + merge: the linear lookup's merge kernel
    kvb::AsmParams p{q, qbar, abar, log_zbar, o_self, lse_self, N, H, K, m, 0, 0, 0, idx, o, lse, keys, 1};
    return launch_pdl(kvb::asm_merge_kernel, dim3((unsigned)((nh + 7) / 8)), dim3(256), 0, st, p);
}

size_t kvb_asm_aggregate_workspace_bytes(int32_t H, int32_t K) {
    if (H < 1 || K < 1) return 0;
    const size_t hk = (size_t)H * K;
    return hk * (3 * sizeof(uint32_t)) + 2 * hk * kvb::kBuildD * sizeof(float);
}

kvb_status kvb_asm_aggregate_grouped(const uint16_t* q, const float* a, const float* lse, const int32_t* idx,
                                     int32_t M, int32_t H, int32_t H_tables, int32_t K, int32_t d, int32_t z_mean,
                                     float* qbar, uint16_t* abar, float* log_zbar, int32_t* count,
                                     void* workspace, size_t workspace_bytes, kvb_stream stream) {
    if (d != kvb::kBuildD || M < 1 || H < 1 || K < 1) return KVB_EINVAL;
    if (H_tables < 1 || H % H_tables != 0) return KVB_EINVAL;
    if (!q || !idx || !qbar || !workspace) return KVB_EINVAL;
    if ((a == nullptr) != (lse == nullptr)) return KVB_EINVAL;
    if (a != nullptr && (!abar || !log_zbar || !aligned16(a) || !aligned16(abar))) return KVB_EINVAL;
    if (!aligned16(q) || !aligned16(qbar) || !aligned16(workspace)) return KVB_EINVAL;
    if (workspace_bytes < kvb_asm_aggregate_workspace_bytes(H_tables, K)) return KVB_EINVAL;
    const long long rows = (long long)M * H, hk = (long long)H_tables * K;
    if (rows > (1ll << 34) || hk * kvb::kBuildD > (1ll << 34)) return KVB_EINVAL;
    // workspace: qsum [H, K, d], asum [H, K, d], wsum [H, K], cmax [H, K], cnt [H, K]
    auto* base = static_cast<unsigned char*>(workspace);
    float* qsum = reinterpret_cast<float*>(base);
    float* asum = qsum + hk * kvb::kBuildD;
    float* wsum = asum + hk * kvb::kBuildD;
    auto* cmax = reinterpret_cast<unsigned*>(wsum + hk);
    int* cnt = reinterpret_cast<int*>(cmax + hk);
    kvb::AsmBuildParams p{q, a, lse, idx, M, H, K, z_mean ? 1 : 0, qbar, abar, log_zbar, count,
                          cmax, cnt, wsum, qsum, asum, H / H_tables};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t words = kvb_asm_aggregate_workspace_bytes(H_tables, K) / sizeof(unsigned);
    kvb::asm_build_zero_kernel<<<(unsigned)std::min<size_t>((words + 255) / 256, 4096), 256, 0, st>>>(
        static_cast<unsigned*>(workspace), words);
    if (launched() != KVB_OK) return KVB_ECUDA;
    kvb::asm_build_pass1_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
    if (launched() != KVB_OK) return KVB_ECUDA;
    if (a != nullptr) {
        kvb::asm_build_pass2_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
        if (launched() != KVB_OK) return KVB_ECUDA;
    }
    kvb::asm_build_final_kernel<<<(unsigned)((hk + 7) / 8), 256, 0, st>>>(p);
    return launched();
}

kvb_status kvb_asm_aggregate(const uint16_t* q, const float* a, const float* lse, const int32_t* idx,
                             int32_t M, int32_t H, int32_t K, int32_t d, int32_t z_mean,
                             float* qbar, uint16_t* abar, float* log_zbar, int32_t* count,
                             void* workspace, size_t workspace_bytes, kvb_stream stream) {
    return kvb_asm_aggregate_grouped(q, a, lse, idx, M, H, H, K, d, z_mean, qbar, abar, log_zbar, count, workspace,
                                     workspace_bytes, stream);
}

kvb_status kvb_asm_entries_bf16(const float* qbar, int32_t H, int32_t K, int32_t d, uint16_t* q,
                                kvb_stream stream) {
    if (d != kvb::kBuildD || H < 1 || K < 1 || !qbar || !q || !aligned16(qbar) || !aligned16(q)) return KVB_EINVAL;
    const long long total = (long long)H * K * (kvb::kBuildD / 4);
    if ((total + 255) / 256 > 0x7fffffffll) return KVB_EINVAL;
    kvb::asm_entries_bf16_kernel<<<(unsigned)((total + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        qbar, H, K, q);
    return launched();
}

size_t kvb_asm_index_workspace_bytes(int32_t H, int32_t C) {
    if (H < 1 || C < 1) return 0;
    return (size_t)H * C * sizeof(int32_t);
}

kvb_status kvb_asm_index_csr(const int32_t* idx, int32_t K, int32_t H, int32_t C, int32_t* offsets,
                             int32_t* members, void* workspace, size_t workspace_bytes, kvb_stream stream) {
    if (K < 1 || H < 1 || C < 1 || C > 65536 || !idx || !offsets || !members || !workspace) return KVB_EINVAL;
    if (!aligned16(workspace) || workspace_bytes < kvb_asm_index_workspace_bytes(H, C)) return KVB_EINVAL;
    if ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(offsets) |
         reinterpret_cast<uintptr_t>(members)) & 3)
        return KVB_EINVAL;
    kvb::AsmCsrParams p{idx, K, H, C, offsets, members, static_cast<int32_t*>(workspace)};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)(((long long)H * C + 7) / 8);
    kvb::asm_csr_kernel<0><<<grid, 256, 0, st>>>(p);
    if (launched() != KVB_OK) return KVB_ECUDA;
    kvb::asm_csr_scan_kernel<<<(unsigned)H, 32, 0, st>>>(p);
    if (launched() != KVB_OK) return KVB_ECUDA;
    kvb::asm_csr_kernel<1><<<grid, 256, 0, st>>>(p);
    return launched();
}

}  // extern "C"
