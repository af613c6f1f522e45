// Split-K GQA decode attention with the retention bias of "Cache What Lasts"
// section 2.1 (logit = scale * q.k_i + (t - i) log beta_i) and the (o, lse)
// state of "Context Memorization" core method step 1. With several splits
// the kernel writes every split's state and merge_splits_kernel (below)
// combines them with that page's step-2 operator. (Merging in the last CTA
// of each (sequence, kv head) to finish was measured and rejected: a CTA
// that lags once is likely to be last again, so merges pile up on it.)
//
// Persistent, warp-specialised kernel:
//  - The work is a list of units (sequence b, kv head g, split j); CTA c
//    takes units c, c + grid, c + 2*grid, ...
//  - One producer warp streams each unit's K/V tiles (T slots) with TMA
//    tensor loads (128-byte swizzle) into a STAGES-deep shared-memory ring.
//    With every tile it also copies the tile's pos and log beta into the
//    stage (4-byte cp.async; the consumers form the bias (t - pos) * log beta
//    and mask the slots past the split's end) and, with a unit's first tile,
//    the unit's G query rows (bulk copy); one "full" mbarrier per stage counts
//    the bytes and the producer lanes' cp.async arrivals, one "empty" mbarrier
//    the consumers' release. The producer itself waits for no load: staging
//    the bias through its registers put a DRAM round trip on every tile's
//    path, which set the pace of short units.
//  - Four consumer warps each own 16 slots of a tile. Both products run on
//    the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate) with the
//    G query heads in the N dimension (8 columns, heads >= G zero), so that
//    the 16 slots fill the M rows:
//      S^T = K . Q^T     A = K via ldmatrix, B = q columns (registers)
//      O^T += V^T . P^T  A = V^T via ldmatrix.trans, B = P^T: the accumulator
//                        of S^T with each 8x8 block transposed in registers
//                        (movmatrix); P is split into a bf16 high part and a
//                        bf16 residual, two mma each, which keeps ~16 bits of
//                        P (a single bf16 P would cost ~1e-3 relative error
//                        in o).
//    Online softmax per warp and head (maxima in natural units, exp2 of
//    scaled differences), O rescaled only when a maximum moved.
//  - At the end of a unit each consumer warp posts its unscaled O, its
//    (m, l) per head and its lanes' eviction candidates to shared memory
//    (mbarrier epi_full) and goes on with the next unit; one epilogue warp
//    combines the four states, reduces the candidates, writes the split's
//    state and frees the buffer (epi_empty). The epilogue of one unit thus
//    overlaps the next unit's tiles.
//  - The fused decode step (INS): the producer also takes each row's victim
//    from the previous step's records and the consumer warp owning the
//    victim's slot swaps the new token into the staged tile and the cache.
// Every wait is bounded (wait_ns, 1 s by default); on a timeout the CTA
// records KVB_DERR_TIMEOUT, stops, drains the copies it issued (bounded) and
// writes the empty state for every unit it owns.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace kvb {

struct DecodeTcParams {
    const uint16_t* q;
    long long q_sb, q_sh;
    const float* lb;
    const int* pos;
    long long m_sb, m_sh;
    const int* len;
    const int* t;
    int Hq, Hkv, cap, S, split_len;
    int units;      // B * Hkv * S
    int kv_shared;  // kv_stride_b == 0: every row reads sequence 0's cache
    float scale;
    float* o_part;
    float* lse_part;
    void* o;
    int o_bf16;
    float* lse;
    EvictCand* cand;  // nullable: per-split eviction candidates for position t + 1
    unsigned long long wait_ns;  // limit of every mbarrier wait
    int withhold;     // test hook: the producer issues nothing, so the consumers' first wait runs out
    // paged cache (PAGED kernels): K, V, pos, log beta in pages of T slots from one pool;
    // logical slot s of (b, g) is row s % T of page table[(b * Hkv + g) * max_pages + s / T]
    const int* table;
    int max_pages, num_pages;
    // fused insertion (INS kernels, a decode step in one launch): in every full row (len == M) the
    // new token replaces the victim named by the previous attention's records cand_in (stamped
    // t); the unit holding the victim patches its staged tile and writes the new row to the cache
    uint16_t* k_w;
    uint16_t* v_w;
    long long kv_sb, kv_sh;   // element strides of the cache (slot stride D)
    float* lb_w;              // log beta and pos of the cache, writable (meta strides m_sb, m_sh)
    int* pos_w;
    const uint16_t* k_new;    // [B, Hkv, D] bf16
    const uint16_t* v_new;
    const float* lb_new;      // [B, Hkv]; nullptr with lb == nullptr
    const EvictCand* cand_in; // [B, Hkv, S]
    int* victim;              // nullable [B, Hkv]: the slot replaced, -1 if none
    int M;
};

template <int D, int G>
struct TcShape {
    static constexpr int NWC = 4;                 // consumer warps
    static constexpr int NT = (NWC + 2) * 32;     // + one producer warp, one epilogue warp
    static constexpr int T = 16 * NWC;            // slots per tile
    static constexpr int STAGES = 3;
    static constexpr int HALVES = D / 64;         // 128-byte swizzle rows hold 64 bf16
    static constexpr int HALF_BYTES = T * 128;
    static constexpr int TILE_BYTES = HALVES * HALF_BYTES;  // one of K or V
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int KSTEPS = D / 16;
    static constexpr int NTILES = D / 8;          // n-tiles of the PV product
    static constexpr int QBYTES = G * D * 2;
    // shared-memory layout (offsets from a 1024-aligned base)
    static constexpr int RING_OFF = 0;
    static constexpr int Q_OFF = RING_OFF + STAGES * STAGE_BYTES;       // [ST][G][D] bf16
    static constexpr int CPOS_OFF = Q_OFF + STAGES * QBYTES;            // [ST][T] int (pos: bias, candidates)
    static constexpr int CLB_OFF = CPOS_OFF + STAGES * T * 4;           // [ST][T] f32 (log beta)
    static constexpr int META_OFF = CLB_OFF + STAGES * T * 4;           // [ST][16] int
    static constexpr int BAR_OFF = META_OFF + STAGES * 64;              // full[ST], empty[ST], epi full/empty
    static constexpr int MISC_OFF = BAR_OFF + (2 * STAGES + 2) * 8;     // abort, issued, -, -, unit record [5]
    static constexpr int EPI_LD = D + 4;   // row stride (floats): the posting lanes' rows fall in distinct banks
    static constexpr int EPI_OFF = (MISC_OFF + 64 + 15) / 16 * 16;      // [NWC][G][EPI_LD] f32
    static constexpr int ML_OFF = EPI_OFF + NWC * G * EPI_LD * 4;       // [NWC][G][2] f32
    static constexpr int CAND_OFF = ML_OFF + NWC * G * 2 * 4;           // [NWC][16] keys, then [NWC][16] slots
    // fused insertion: per stage the new token's K and V rows and its log beta
    static constexpr int PATCH_BYTES = 4 * D + 16;
    static constexpr int PATCH_OFF = (CAND_OFF + NWC * 16 * 12 + 15) / 16 * 16;  // [ST][PATCH_BYTES]
    static constexpr int END_OFF = PATCH_OFF + STAGES * PATCH_BYTES;
    static constexpr size_t SMEM = 1024 + END_OFF;
    static_assert(D == 64 || D == 128, "d");
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "G");
    static_assert(STAGE_BYTES % 1024 == 0 && Q_OFF % 16 == 0 && PATCH_BYTES % 16 == 0, "alignment");
};
// two CTAs per SM at the Qwen3-8B-like shape (228 KB of shared memory per SM, 1 KB reserved per CTA)
static_assert(2 * (TcShape<128, 4>::SMEM + 1024) <= 228 * 1024, "two CTAs per SM");

// ---- PTX wrappers -------------------------------------------------------------

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A . B + C, m16n8k16, bf16 inputs, fp32 accumulators; A rows 8..15 are zero.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// D = A . B + C, m16n8k16, bf16 inputs, fp32 accumulators, all 16 rows of A.
__device__ __forceinline__ void mma_bf16_a(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// the transpose of an 8x8 b16 matrix held as the warp's standard fragment (lane l: row l / 4,
// columns 2 (l % 4) and 2 (l % 4) + 1)
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 4-byte asynchronous global -> shared copy (cp.async), and the arrival on an mbarrier that happens
// once every cp.async this thread issued has landed (it counts as one of the barrier's arrivals)
__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// A bounded wait that sleeps between its checks (for a warp whose waits are long and off the
// critical path: it leaves the issue slots to the warps that compute)
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, unsigned parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(256);
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz; 2^-inf = 0)
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- unit bookkeeping shared by producer and consumers --------------------------

struct UnitInfo {
    int b, g, split, s0, nk, ntiles, n;  // n: the (b, g) length after the validity checks
};

// The two loads a unit's geometry depends on; fetched one unit ahead by the producer.
struct UnitRaw {
    int len, t;
};

// Unit u is split u mod S of row u / S, rows (b, g) in order. (A split-major order, meant to mix
// the split indices of a CTA's round-robin units on ragged rows, measured slower on the memento
// workload: 106.4 against 98.8 us per step.)
__device__ __forceinline__ void unit_coords(const DecodeTcParams& p, int u, int& b, int& g, int& split) {
    const int per_b = p.Hkv * p.S;
    b = u / per_b;
    const int rem = u - b * per_b;
    g = rem / p.S;
    split = rem - g * p.S;
}

__device__ __forceinline__ UnitRaw unit_raw(const DecodeTcParams& p, long long ul) {
    UnitRaw r{0, 0};
    if (ul < p.units) {
        int b, g, split;
        unit_coords(p, (int)ul, b, g, split);
        r.len = p.len[b * p.Hkv + g];
        r.t = (p.t == nullptr) ? 0 : p.t[b];
    }
    return r;
}

template <int T>
__device__ __forceinline__ UnitInfo unit_info(const DecodeTcParams& p, int u, UnitRaw raw, bool record_errors) {
    UnitInfo r;
    unit_coords(p, u, r.b, r.g, r.split);
    int n = raw.len;
    const bool active = (p.t == nullptr) || (raw.t >= 0);
    const bool bad_len = n < 0 || n > p.cap;
    const bool bad_split = !bad_len && p.split_len > 0 && (long long)n > (long long)p.S * p.split_len;
    if (record_errors && (bad_len || bad_split) && r.split == 0) raise_error(bad_len ? KVB_DERR_LEN : KVB_DERR_SPLIT);
    if (bad_len || bad_split || !active) n = 0;
    const long long C = p.split_len > 0 ? (long long)p.split_len : (long long)((n + p.S - 1) / p.S);
    r.s0 = (int)min((long long)r.split * C, (long long)n);
    const int s1 = (int)min((long long)r.s0 + C, (long long)n);
    r.nk = s1 - r.s0;
    r.ntiles = (r.nk + T - 1) / T;
    r.n = n;
    return r;
}

// Fused insertion ("Cache What Lasts" section 2.1 at inference, as kvb_evict_insert): the slot of
// row (b, g) that the new token takes. The victim is the smallest (score, pos) key among the row's
// S records of the previous attention, which scored every slot for this position t.
// RowRecords holds a lane's share of one row's records (records lane and lane + 32), loaded a unit
// ahead of their use; rows of more than 64 splits read the rest when they are used.
struct RowRecords {
    EvictCand r[2];
};

__device__ __forceinline__ RowRecords load_row_records(const DecodeTcParams& p, int u, int lane) {
    RowRecords x;
    x.r[0] = x.r[1] = EvictCand{~0ull, -1, 0};
    if (u < p.units) {
        int b, g, split;
        unit_coords(p, u, b, g, split);
        const EvictCand* rec = p.cand_in + ((size_t)b * p.Hkv + g) * p.S;
        if (lane < p.S) x.r[0] = rec[lane];
        if (lane + 32 < p.S) x.r[1] = rec[lane + 32];
    }
    return x;
}

// Warp-collective (every lane of the producer warp). Returns -1 for an inactive row (t < 0:
// nothing is inserted), -2 for a row the fused step cannot update (not full: len != M) and -3
// when the records cannot name the victim (one scored for another position, or none naming a
// slot): then row_scan_victim finds it.
__device__ __forceinline__ int row_victim(const DecodeTcParams& p, const RowRecords& x, int b, int g, int tb, int n,
                                          int lane) {
    unsigned long long best = ~0ull;
    int best_slot = 0x7fffffff;
    bool stale = false;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        if (lane + 32 * k < p.S) {
            stale = stale || x.r[k].t != tb;
            if (x.r[k].slot >= 0) argmin_merge(best, best_slot, x.r[k].key, x.r[k].slot);
        }
    }
    const EvictCand* rec = p.cand_in + ((size_t)b * p.Hkv + g) * p.S;
    for (int j = lane + 64; j < p.S; j += 32) {
        const EvictCand c = rec[j];
        stale = stale || c.t != tb;
        if (c.slot >= 0) argmin_merge(best, best_slot, c.key, c.slot);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const unsigned long long k2 = __shfl_xor_sync(kFull, best, m);
        const int s2 = __shfl_xor_sync(kFull, best_slot, m);
        argmin_merge(best, best_slot, k2, s2);
    }
    stale = __any_sync(kFull, stale);
    if (tb < 0) return -1;
    if (n != p.M) return -2;
    if (stale || best == ~0ull || best_slot >= n) return -3;
    return best_slot;
}

// The victim of a full row from its slots, as kvb_evict_insert's scan: the smallest key
// (order key of the score (t - pos) log beta, one float32 product) << 32 | the order key of pos.
// Warp-collective; every unit of the row repeats it, which only happens when the records were not
// left for this position.
__device__ __noinline__ int row_scan_victim(const DecodeTcParams& p, int b, int g, int tb, int n, int lane) {
    const size_t base = (size_t)b * p.m_sb + (size_t)g * p.m_sh;
    const int* ps = p.pos + base;
    const float* lb = p.lb != nullptr ? p.lb + base : nullptr;
    unsigned long long best = ~0ull;
    int best_slot = 0x7fffffff;
    for (int s0 = lane; s0 < n; s0 += 32 * 4) {
        int pv[4];
        float lv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // four independent loads of each kind in flight
            const int s = s0 + 32 * k;
            pv[k] = s < n ? ps[s] : 0;
            lv[k] = (lb != nullptr && s < n) ? lb[s] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int s = s0 + 32 * k;
            if (s < n) {
                const float sc = lb != nullptr ? __fmul_rn(__int2float_rn(tb - pv[k]), lv[k]) : 0.f;
                const unsigned long long key =
                    ((unsigned long long)float_order_key(sc) << 32) | (unsigned)(pv[k] ^ 0x80000000);
                argmin_merge(best, best_slot, key, s);
            }
        }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const unsigned long long k2 = __shfl_xor_sync(kFull, best, m);
        const int s2 = __shfl_xor_sync(kFull, best_slot, m);
        argmin_merge(best, best_slot, k2, s2);
    }
    return best_slot;
}

template <int D, int G, bool BIAS, bool PAGED = false, bool INS = false>
__global__ void __launch_bounds__(TcShape<D, G>::NT, 2)
    decode_attn_tc_kernel(const __grid_constant__ DecodeTcParams p, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV) {
    using SH = TcShape<D, G>;
    constexpr int NWC = SH::NWC, T = SH::T, ST = SH::STAGES;
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
    uint16_t* s_q = reinterpret_cast<uint16_t*>(smem + SH::Q_OFF);
    int* s_meta = reinterpret_cast<int*>(smem + SH::META_OFF);
    int* s_pos = reinterpret_cast<int*>(smem + SH::CPOS_OFF);
    float* s_lb = reinterpret_cast<float*>(smem + SH::CLB_OFF);
    unsigned long long* s_ck = reinterpret_cast<unsigned long long*>(smem + SH::CAND_OFF);
    int* s_cs = reinterpret_cast<int*>(smem + SH::CAND_OFF + NWC * 16 * 8);
    uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + SH::BAR_OFF);
    uint64_t* s_empty = s_full + ST;
    uint64_t* epi_full = s_empty + ST;    // the four consumer warps posted a unit's partial states
    uint64_t* epi_empty = epi_full + 1;   // the epilogue warp has read them
    volatile int* s_abort = reinterpret_cast<int*>(smem + SH::MISC_OFF);
    int* s_issued = reinterpret_cast<int*>(smem + SH::MISC_OFF) + 1;
    volatile int* s_epi = reinterpret_cast<int*>(smem + SH::MISC_OFF) + 4;   // b, g, split, t, stop
    float* s_o = reinterpret_cast<float*>(smem + SH::EPI_OFF);
    float* s_ml = reinterpret_cast<float*>(smem + SH::ML_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // set-up that reads nothing the previous kernel in the stream writes runs before the wait
    // for it: the barriers, and the tensor maps (kernel parameters) into the TMA unit's cache
    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&s_full[s], 33);          // producer lane 0's expect_tx + 32 producer lanes
            mbar_init(&s_empty[s], NWC * 32);   // every consumer lane
        }
        mbar_init(epi_full, NWC);
        mbar_init(epi_empty, 1);
        *s_abort = 0;
        *s_issued = 0;
        fence_mbar_init();
    }
    if (warp == NWC && lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    griddep_wait();  // the previous kernel in the stream (e.g. the insertion) has finished writing
    griddep_launch_dependents();
    // the producer's first lengths and positions are in flight during the barrier below
    UnitRaw first_raw{0, 0};
    RowRecords next_rec;   // fused insertion: the records of the producer's next unit's row
    if (warp == NWC) {
        first_raw = unit_raw(p, (long long)blockIdx.x + (long long)lane * gridDim.x);
        if constexpr (INS) next_rec = load_row_records(p, blockIdx.x, lane);
    }
    __syncthreads();

    if (warp == NWC) {
        // ======================= producer warp =======================
        int it = 0;
        bool stop = false;
        // this CTA's units: blockIdx.x, blockIdx.x + gridDim.x, ... (round robin)
        const int u_lo = blockIdx.x, u_hi = p.units, u_step = gridDim.x;
        // lane l holds the length and position of this CTA's unit 32 * (k / 32) + l: one round trip
        // per 32 units, so that empty units (ragged lengths) cost no load latency each
        UnitRaw lane_raw{0, 0};
        for (int u = u_lo, k = 0; !stop; u += u_step, ++k) {
            const bool end = u >= u_hi;  // one end record after the last unit
            if (k == 0) {
                lane_raw = first_raw;
            } else if ((k & 31) == 0) {
                lane_raw = unit_raw(p, (long long)u + (long long)lane * u_step);
            }
            const UnitRaw raw{__shfl_sync(kFull, lane_raw.len, k & 31), __shfl_sync(kFull, lane_raw.t, k & 31)};
            UnitInfo ui{};
            if (!end) ui = unit_info<T>(p, u, raw, lane == 0);
            int victim = -1;   // fused insertion: the slot (of the row) the new token takes, -1: none
            if constexpr (INS) {
                const RowRecords cur = next_rec;
                next_rec = load_row_records(p, end ? p.units : u + u_step, lane);
                if (!end) {
                    victim = row_victim(p, cur, ui.b, ui.g, raw.t, raw.len, lane);
                    if (victim == -3) victim = row_scan_victim(p, ui.b, ui.g, raw.t, raw.len, lane);
                    if (ui.split == 0 && lane == 0) {
                        if (victim == -2) raise_error(KVB_DERR_STEP);
                        if (p.victim != nullptr) p.victim[ui.b * p.Hkv + ui.g] = max(victim, -1);
                    }
                    if (victim == -2) ui.ntiles = 0;   // a row the step cannot update: the empty state
                }
            }
            if (!end && ui.ntiles == 0) {
                // an empty split (ragged lengths, inactive rows): write its empty state here;
                // no record reaches the consumers
                const size_t row0 = (size_t)ui.b * p.Hq + ui.g * G;
                // lse = -inf marks the empty state; its o_part row is not written (no merge reads it)
                if (p.o_part != nullptr && lane < G) p.lse_part[(row0 + lane) * p.S + ui.split] = -INFINITY;
                if (p.S == 1) {
                    for (int idx = lane; idx < G * D; idx += 32) {
                        const size_t oi = row0 * D + idx;
                        if (p.o_bf16) {
                            reinterpret_cast<__nv_bfloat16*>(p.o)[oi] = __float2bfloat16_rn(0.f);
                        } else {
                            reinterpret_cast<float*>(p.o)[oi] = 0.f;
                        }
                    }
                    if (lane < G && p.lse != nullptr) p.lse[row0 + lane] = -INFINITY;
                }
                if (lane == 0 && p.cand != nullptr) {
                    EvictCand* c = p.cand + ((size_t)ui.b * p.Hkv + ui.g) * p.S + ui.split;
                    c->key = ~0ull;
                    c->slot = -1;
                    c->t = raw.t + 1;
                }
                continue;
            }
            const int records = end ? 1 : ui.ntiles;
            const int tb = raw.t;
            const size_t m_off = end ? 0 : (size_t)ui.b * p.m_sb + (size_t)ui.g * p.m_sh + (size_t)ui.s0;
            const bool want_cand = p.cand != nullptr;
            if (p.withhold) {   // test hook: no copy, no arrival; the consumers' wait runs out
                stop = true;
                break;
            }
            // paged: lane l holds the page of the unit's tile 32 * (i / 32) + l (units start on a page)
            int lane_page = 0;
            const size_t trow = PAGED && !end ? ((size_t)ui.b * p.Hkv + ui.g) * p.max_pages + ui.s0 / T : 0;
            for (int i = 0; i < records; ++i, ++it) {
                const int st = it % ST;
                int page = 0;
                if constexpr (PAGED) {
                    if (!end && (i & 31) == 0) {
                        int pg = 0;
                        if (i + lane < ui.ntiles) {
                            pg = p.table[trow + i + lane];
                            if (pg < 0 || pg >= p.num_pages) {   // not a page of the pool: read page 0
                                raise_error(KVB_DERR_RANGE);
                                pg = 0;
                            }
                        }
                        lane_page = pg;
                    }
                    page = __shfl_sync(kFull, lane_page, i & 31);
                }
                // the stage's record and copies (lane 0)
                const bool data = !end && ui.ntiles > 0;
                auto issue = [&]() {
                    if (lane == 0) {
                        int* m = s_meta + st * 16;
                        m[0] = end ? -1 : u;
                        m[1] = i;
                        m[2] = end ? 0 : ui.ntiles;
                        m[3] = data ? min(T, ui.nk - i * T) : 0;
                        m[4] = ui.b;
                        m[5] = ui.g;
                        m[6] = ui.split;
                        m[7] = ui.n;
                        m[8] = tb;
                        m[9] = ui.s0 + i * T;
                        // fused insertion: the victim's row in this tile (or -1), and the new row
                        const int vrow = (INS && data && victim >= m[9] && victim < m[9] + m[3]) ? victim - m[9] : -1;
                        m[10] = vrow;
                        unsigned tx = data ? (unsigned)SH::STAGE_BYTES : 0u;
                        const bool with_q = data && i == 0;
                        if (with_q) tx += SH::QBYTES;
                        if (vrow >= 0) tx += 4 * D;
                        mbar_arrive_expect_tx(&s_full[st], tx);
                        if (data) {
                            unsigned char* kt = smem + SH::RING_OFF + st * SH::STAGE_BYTES;
                            unsigned char* vt = kt + SH::TILE_BYTES;
                            // paged: the page's rows in the pool (one kv head, one "sequence" in the map)
                            const int row = PAGED ? page * T : ui.s0 + i * T;
                            const int gg = PAGED ? 0 : ui.g;
                            const int bb = (PAGED || p.kv_shared) ? 0 : ui.b;
#pragma unroll
                            for (int h = 0; h < SH::HALVES; ++h) {
                                tma_load_4d(kt + h * SH::HALF_BYTES, &tmK, 64 * h, row, gg, bb, &s_full[st]);
                                tma_load_4d(vt + h * SH::HALF_BYTES, &tmV, 64 * h, row, gg, bb, &s_full[st]);
                            }
                        }
                        if (vrow >= 0) {
                            unsigned char* pt = smem + SH::PATCH_OFF + st * SH::PATCH_BYTES;
                            const size_t nrow = ((size_t)ui.b * p.Hkv + ui.g) * D;
                            bulk_g2s(pt, p.k_new + nrow, (unsigned)(2 * D), &s_full[st]);
                            bulk_g2s(pt + 2 * D, p.v_new + nrow, (unsigned)(2 * D), &s_full[st]);
                            if (BIAS) cp_async4(pt + 4 * D, p.lb_new + (size_t)ui.b * p.Hkv + ui.g);
                        }
                        if (with_q) {
                            const uint16_t* qsrc = p.q + (size_t)ui.b * p.q_sb + (size_t)(ui.g * G) * p.q_sh;
                            uint16_t* qdst = s_q + st * G * D;
                            if (p.q_sh == D) {
                                bulk_g2s(qdst, qsrc, (unsigned)SH::QBYTES, &s_full[st]);
                            } else {
                                for (int hh = 0; hh < G; ++hh)
                                    bulk_g2s(qdst + hh * D, qsrc + (size_t)hh * p.q_sh, (unsigned)(D * 2), &s_full[st]);
                            }
                        }
                    }
                };
                if (it >= ST && !mbar_wait(&s_empty[st], (unsigned)((it / ST) - 1) & 1u, p.wait_ns)) {
                    if (lane == 0) {
                        raise_error(KVB_DERR_TIMEOUT);
                        *s_abort = 1;
                    }
                    stop = true;
                    break;
                }
                if (*s_abort) {
                    stop = true;
                    break;
                }
                issue();
                // this tile's pos (for the bias and the eviction candidates) and log beta go into the
                // stage by asynchronous 4-byte copies that the stage's full barrier counts: no load
                // round trip on this warp's path (the consumers form the bias); slots past the
                // split's end are not copied (the consumers mask them)
                if (BIAS || want_cand) {
                    const size_t mt = PAGED ? (size_t)page * T : m_off + (size_t)i * T;
#pragma unroll
                    for (int j = 0; j < T / 32; ++j) {
                        const int key = i * T + lane + 32 * j;
                        if (!end && key < ui.nk) {
                            cp_async4(s_pos + st * T + lane + 32 * j, p.pos + mt + lane + 32 * j);
                            if constexpr (BIAS) cp_async4(s_lb + st * T + lane + 32 * j, p.lb + mt + lane + 32 * j);
                        }
                    }
                }
                cp_async_mbar_arrive(&s_full[st]);   // one arrival per lane once its copies have landed
            }
            if (end) break;
        }
        if (lane == 0) *s_issued = it;
    } else if (warp < NWC) {
        // ======================= consumer warps =======================
        // Both products keep the G query heads in the N dimension (8 columns, heads >= G zero):
        //   S^T = K Q^T     A = this warp's 16 slots of K (ldmatrix), B = Q^T (registers)
        //   O^T += V^T P^T  A = V^T (ldmatrix.trans), B = P^T, the accumulator of S^T with each
        //                   8x8 block transposed in registers (movmatrix)
        // so a warp issues D/16 + 2 D/16 mma per tile, and the fragments a lane holds are slots
        // kw + r and kw + r + 8 of heads 2 cq and 2 cq + 1 (S), dims 16 m + r and 16 m + r + 8 of
        // the same heads (O).
        const int r = lane >> 2;          // fragment row; also the head whose Q column this lane loads
        const int cq = lane & 3;          // fragment column pair: heads 2 cq, 2 cq + 1
        const int kw = 16 * warp;         // this warp's first slot in a tile
        const uint32_t ring = smem_u32(smem + SH::RING_OFF);
        // ldmatrix row addresses (relative to a tile half): swizzle xor = row & 7 = lane & 7
        const int ka_row = kw + (lane & 7) + (((lane >> 3) & 1) << 3);   // K as A: slots 0-7, 8-15
        const int ka_hi = lane >> 4;                                     // then dims 8-15 of the step
        const int va_row = kw + (lane & 7) + ((lane >> 4) << 3);         // V^T as A (transposed copy)
        const int va_hi = (lane >> 3) & 1;
        const int sw = lane & 7;

        uint32_t qa[SH::KSTEPS][2];       // Q^T fragments (B operand of S^T)
        float acc[D / 16][4];             // O^T fragments
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2 cq, 2 cq + 1
        const bool want_cand = p.cand != nullptr;
        unsigned long long cand_key = ~0ull;  // this lane's best eviction key in the unit
        int cand_slot = 0x7fffffff;
        int it = 0;
        bool aborted = false;
        int units_posted = 0;   // units whose partial states went to the epilogue warp
        while (true) {
            const int st = it % ST;
            if (!mbar_wait(&s_full[st], (unsigned)(it / ST) & 1u, p.wait_ns)) {
                if (lane == 0) {
                    raise_error(KVB_DERR_TIMEOUT);
                    *s_abort = 1;
                }
                aborted = true;
                break;
            }
            const int* m = s_meta + st * 16;
            const int u = m[0], i = m[1], ntiles = m[2], rows = m[3];
            if (u < 0) break;
            const int ub = m[4], ug = m[5], usplit = m[6], ut = m[8];   // (read before the stage is released)
            if constexpr (INS) {
                const int vrow = m[10];
                if (vrow >= kw && vrow < kw + 16) {
                    // fused insertion, the victim among this warp's slots: the new token's K and V
                    // rows replace the staged ones (same 128-byte swizzle as the copy) and go to the
                    // cache; its pos is t and its log beta the new one. No other CTA reads this slot.
                    const unsigned char* pt = smem + SH::PATCH_OFF + st * SH::PATCH_BYTES;
                    unsigned char* tile = smem + SH::RING_OFF + st * SH::STAGE_BYTES;
                    const int slot = m[9] + vrow;
                    const size_t crow = (size_t)ub * p.kv_sb + (size_t)ug * p.kv_sh + (size_t)slot * D;
                    for (int c = lane; c < D / 4; c += 32) {   // 16-byte chunks: D/8 of K, then D/8 of V
                        const int kv = c / (D / 8), cc = c % (D / 8);
                        const uint4 x = *reinterpret_cast<const uint4*>(pt + kv * 2 * D + cc * 16);
                        *reinterpret_cast<uint4*>(tile + kv * SH::TILE_BYTES + (cc >> 3) * SH::HALF_BYTES + vrow * 128 +
                                                  (((cc & 7) ^ (vrow & 7)) << 4)) = x;
                        *reinterpret_cast<uint4*>((kv ? p.v_w : p.k_w) + crow + cc * 8) = x;
                    }
                    if (lane == 0) {
                        const size_t mrow = (size_t)ub * p.m_sb + (size_t)ug * p.m_sh + slot;
                        s_pos[st * T + vrow] = ut;
                        p.pos_w[mrow] = ut;
                        if constexpr (BIAS) {
                            const float lbn = *reinterpret_cast<const float*>(pt + 4 * D);
                            s_lb[st * T + vrow] = lbn;
                            p.lb_w[mrow] = lbn;
                        }
                    }
                    fence_proxy_async_smem();   // the stage's next copy (async proxy) follows these writes
                    __syncwarp();
                }
            }
            if (i == 0) {
                cand_key = ~0ull;
                cand_slot = 0x7fffffff;
            }
            if (want_cand && ntiles > 0 && lane < 16 && kw + lane < rows) {
                // eviction key of this slot for position t + 1 (one lane per slot)
                const int kk = kw + lane;
                const int ps = s_pos[st * T + kk];
                const float sc = BIAS ? __fmul_rn(__int2float_rn(m[8] + 1 - ps), s_lb[st * T + kk]) : 0.f;
                const unsigned long long k64 =
                    ((unsigned long long)float_order_key(sc) << 32) | (unsigned)(ps ^ 0x80000000);
                const int slot = m[9] + kk;
                if (k64 < cand_key || (k64 == cand_key && slot < cand_slot)) {
                    cand_key = k64;
                    cand_slot = slot;
                }
            }
            if (i == 0) {
                m_run[0] = m_run[1] = -INFINITY;
                l_run[0] = l_run[1] = 0.f;
#pragma unroll
                for (int j = 0; j < D / 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
                if (ntiles > 0) {
                    const uint16_t* qs = s_q + st * G * D;
#pragma unroll
                    for (int s = 0; s < SH::KSTEPS; ++s) {
                        uint32_t a0 = 0u, a2 = 0u;
                        if (r < G) {
                            a0 = *reinterpret_cast<const uint32_t*>(qs + r * D + 16 * s + 2 * cq);
                            a2 = *reinterpret_cast<const uint32_t*>(qs + r * D + 16 * s + 8 + 2 * cq);
                        }
                        qa[s][0] = a0;
                        qa[s][1] = a2;
                    }
                }
            }
            if (ntiles > 0) {
                const uint32_t kt = ring + st * SH::STAGE_BYTES;
                const uint32_t vt = kt + SH::TILE_BYTES;
                // ---- S^T = K Q^T for this warp's 16 slots
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s = 0; s < SH::KSTEPS; ++s) {
                    const int chunk = 2 * (s & 3) + ka_hi;
                    const uint32_t addr =
                        kt + (s >> 2) * SH::HALF_BYTES + ka_row * 128 + ((chunk ^ sw) << 4);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(addr, a0, a1, a2, a3);
                    mma_bf16_a(sc, a0, a1, a2, a3, qa[s][0], qa[s][1]);
                }
                if (rows < T && kw + 16 > rows) {
                    // tail: zero this warp's V rows past the split end (K rows there are masked)
                    for (int idx = lane; idx < 16 * SH::HALVES * 8; idx += 32) {
                        const int row = kw + idx / (SH::HALVES * 8);
                        const int c = idx % (SH::HALVES * 8);
                        if (row >= rows) {
                            unsigned char* vp = smem + SH::RING_OFF + st * SH::STAGE_BYTES + SH::TILE_BYTES +
                                                (c >> 3) * SH::HALF_BYTES + row * 128 + ((c & 7) << 4);
                            *reinterpret_cast<uint4*>(vp) = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                // ---- logits, online softmax (slots sa = kw + r and sb = sa + 8 of this lane, heads 2 cq and
                // 2 cq + 1): scale q.k + (t - pos) log beta (one float32 product), -inf past the split's end
                const int sa = kw + r, sb = sa + 8;
                float ba = 0.f, bb = 0.f;
                if constexpr (BIAS) {
                    ba = __fmul_rn(__int2float_rn(ut - s_pos[st * T + sa]), s_lb[st * T + sa]);
                    bb = __fmul_rn(__int2float_rn(ut - s_pos[st * T + sb]), s_lb[st * T + sb]);
                }
                float x[4];
                x[0] = (sa < rows) ? fmaf(sc[0], p.scale, ba) : -INFINITY;   // slot sa, head 2 cq
                x[1] = (sa < rows) ? fmaf(sc[1], p.scale, ba) : -INFINITY;   // slot sa, head 2 cq + 1
                x[2] = (sb < rows) ? fmaf(sc[2], p.scale, bb) : -INFINITY;   // slot sb, head 2 cq
                x[3] = (sb < rows) ? fmaf(sc[3], p.scale, bb) : -INFINITY;   // slot sb, head 2 cq + 1
                // each head's maximum over the warp's 16 slots: the lanes with the same cq hold them
                float t0 = fmaxf(x[0], x[2]), t1 = fmaxf(x[1], x[3]);
#pragma unroll
                for (int o2 = 4; o2 <= 16; o2 <<= 1) {
                    t0 = fmaxf(t0, __shfl_xor_sync(kFull, t0, o2));
                    t1 = fmaxf(t1, __shfl_xor_sync(kFull, t1, o2));
                }
                const float mn0 = fmaxf(m_run[0], t0), mn1 = fmaxf(m_run[1], t1);
                const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0, mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
                const float al0 = ex2_fast((m_run[0] - mu0) * kLog2e), al1 = ex2_fast((m_run[1] - mu1) * kLog2e);
                float pr[4];
                pr[0] = ex2_fast((x[0] - mu0) * kLog2e);
                pr[1] = ex2_fast((x[1] - mu1) * kLog2e);
                pr[2] = ex2_fast((x[2] - mu0) * kLog2e);
                pr[3] = ex2_fast((x[3] - mu1) * kLog2e);
                l_run[0] = fmaf(l_run[0], al0, pr[0] + pr[2]);   // this lane's slots; summed over lanes at the end
                l_run[1] = fmaf(l_run[1], al1, pr[1] + pr[3]);
                m_run[0] = mn0;
                m_run[1] = mn1;
                if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                    for (int j = 0; j < D / 16; ++j) {
                        acc[j][0] *= al0;
                        acc[j][1] *= al1;
                        acc[j][2] *= al0;
                        acc[j][3] *= al1;
                    }
                }
                // ---- P^T as the B operand: high bf16 part and bf16 residual; the accumulator of S^T holds
                // (slot, head) blocks, the B fragment wants (head, slot): one movmatrix per 8x8 block
                const uint32_t h0 = pack_bf16(pr[0], pr[1]);
                const uint32_t h1 = pack_bf16(pr[2], pr[3]);
                const uint32_t l0 = pack_bf16(pr[0] - __uint_as_float(h0 << 16),
                                              pr[1] - __uint_as_float(h0 & 0xffff0000u));
                const uint32_t l1 = pack_bf16(pr[2] - __uint_as_float(h1 << 16),
                                              pr[3] - __uint_as_float(h1 & 0xffff0000u));
                const uint32_t bh0 = movmatrix_t(h0), bh1 = movmatrix_t(h1);
                const uint32_t bl0 = movmatrix_t(l0), bl1 = movmatrix_t(l1);
                // ---- O^T += V^T P^T, D / 16 tiles of 16 dims
#pragma unroll
                for (int j = 0; j < D / 16; ++j) {
                    const int chunk = 2 * (j & 3) + va_hi;
                    const uint32_t addr =
                        vt + (j >> 2) * SH::HALF_BYTES + va_row * 128 + ((chunk ^ sw) << 4);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(addr, a0, a1, a2, a3);
                    mma_bf16_a(acc[j], a0, a1, a2, a3, bh0, bh1);
                    mma_bf16_a(acc[j], a0, a1, a2, a3, bl0, bl1);
                }
            }
            __syncwarp();
            mbar_arrive(&s_empty[st]);
            ++it;
            if (ntiles > 0 && i != ntiles - 1) continue;

            // ======== end of unit: post this warp's partial state to the epilogue warp ========
#pragma unroll
            for (int o2 = 4; o2 <= 16; o2 <<= 1) {
                l_run[0] += __shfl_xor_sync(kFull, l_run[0], o2);
                l_run[1] += __shfl_xor_sync(kFull, l_run[1], o2);
            }
            // the buffer holds the previous unit until the epilogue warp has read it
            if (units_posted > 0 &&
                !__all_sync(kFull, mbar_wait(epi_empty, (unsigned)(units_posted - 1) & 1u, p.wait_ns))) {
                if (lane == 0) {
                    raise_error(KVB_DERR_TIMEOUT);
                    *s_abort = 1;
                }
                aborted = true;
                break;
            }
#pragma unroll
            for (int jh = 0; jh < 2; ++jh) {
                const int h = 2 * cq + jh;
                if (h < G) {
                    float* dst = s_o + (warp * G + h) * SH::EPI_LD + r;
#pragma unroll
                    for (int j = 0; j < D / 16; ++j) {
                        dst[16 * j] = acc[j][jh];
                        dst[16 * j + 8] = acc[j][2 + jh];
                    }
                    if (r == 0) {
                        s_ml[(warp * G + h) * 2] = m_run[jh];
                        s_ml[(warp * G + h) * 2 + 1] = l_run[jh];
                    }
                }
            }
            if (lane < 16) {   // each slot lane's best candidate; the epilogue warp reduces the 64
                s_ck[warp * 16 + lane] = cand_key;
                s_cs[warp * 16 + lane] = cand_slot;
            }
            if (lane == 0) {
                if (warp == 0) {
                    s_epi[0] = ub;
                    s_epi[1] = ug;
                    s_epi[2] = usplit;
                    s_epi[3] = ut;
                    s_epi[4] = 0;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_full);
            ++units_posted;
        }
        if (!aborted) {
            // the end: once the epilogue warp has read the last unit, tell it to stop
            if (units_posted > 0 &&
                !__all_sync(kFull, mbar_wait(epi_empty, (unsigned)(units_posted - 1) & 1u, p.wait_ns))) {
                if (lane == 0) {
                    raise_error(KVB_DERR_TIMEOUT);
                    *s_abort = 1;
                }
            } else {
                if (warp == 0 && lane == 0) s_epi[4] = 1;
                __syncwarp();
                if (lane == 0) mbar_arrive(epi_full);
            }
        }
        (void)aborted;
    } else {
        // ======================= epilogue warp =======================
        // Combines a unit's four partial states while the consumers go on with the next unit: each
        // warp's share of a row is exp2(m_w - M) / L (M, L over the four warps); lane w G + r holds
        // the share of warp w for row r, and every output is the shares' sum of the four posted O.
        // Its waits back off (nanosleep) so that it takes no issue slots from the consumers.
        const bool want_cand = p.cand != nullptr;
        const int S = p.S;
        constexpr int NV = G * D / 4;   // float4 outputs of a unit
        for (int k = 0;; ++k) {
            if (!__all_sync(kFull, mbar_wait_backoff(epi_full, (unsigned)k & 1u, p.wait_ns))) {
                if (lane == 0) {
                    raise_error(KVB_DERR_TIMEOUT);
                    *s_abort = 1;
                }
                break;
            }
            if (s_epi[4] != 0) break;   // the consumers' stop
            const int ub = s_epi[0], ug = s_epi[1], usplit = s_epi[2], ut = s_epi[3];
            float fsh = 0.f;
            if (lane < NWC * G) {
                const int r = lane % G, w = lane / G;
                float mw[NWC], lw[NWC];
#pragma unroll
                for (int v = 0; v < NWC; ++v) {
                    const float2 x = *reinterpret_cast<const float2*>(s_ml + (v * G + r) * 2);
                    mw[v] = x.x;
                    lw[v] = x.y;
                }
                float M = -INFINITY;
#pragma unroll
                for (int v = 0; v < NWC; ++v) M = fmaxf(M, mw[v]);
                const float Mu = (M == -INFINITY) ? 0.f : M;
                float L = 0.f;
#pragma unroll
                for (int v = 0; v < NWC; ++v) L = fmaf(ex2_fast((mw[v] - Mu) * kLog2e), lw[v], L);
                float mine = mw[0];
#pragma unroll
                for (int v = 1; v < NWC; ++v) mine = (v == w) ? mw[v] : mine;
                fsh = (L > 0.f) ? ex2_fast((mine - Mu) * kLog2e) * __frcp_rn(L) : 0.f;
                if (w == 0) {
                    const float lse = (L > 0.f) ? M + log2f(L) * kLn2 : -INFINITY;
                    const size_t row = (size_t)ub * p.Hq + ug * G + r;
                    if (p.o_part != nullptr) p.lse_part[row * S + usplit] = lse;
                    if (S == 1 && p.lse != nullptr) p.lse[row] = lse;
                }
            }
#pragma unroll
            for (int v0 = 0; v0 < NV; v0 += 32) {   // every lane runs every round (the shuffles)
                const int idx = v0 + lane;
                const int hh = (4 * min(idx, NV - 1)) / D, e = (4 * min(idx, NV - 1)) % D;
                float4 out = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int w = 0; w < NWC; ++w) {
                    const float f = __shfl_sync(kFull, fsh, w * G + hh);
                    const float4 x = *reinterpret_cast<const float4*>(s_o + (w * G + hh) * SH::EPI_LD + e);
                    out.x = fmaf(f, x.x, out.x);
                    out.y = fmaf(f, x.y, out.y);
                    out.z = fmaf(f, x.z, out.z);
                    out.w = fmaf(f, x.w, out.w);
                }
                if (idx < NV) {
                    const size_t row = (size_t)ub * p.Hq + ug * G + hh;
                    if (p.o_part != nullptr) *reinterpret_cast<float4*>(p.o_part + (row * S + usplit) * D + e) = out;
                    if (S == 1) {
                        if (p.o_bf16) {
                            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.o) + row * D + e;
                            *reinterpret_cast<uint2*>(dst) =
                                make_uint2(pack_bf16(out.x, out.y), pack_bf16(out.z, out.w));
                        } else {
                            *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o) + row * D + e) = out;
                        }
                    }
                }
            }
            if (want_cand) {   // the best of the consumer lanes' 64 candidates (key, then slot)
                unsigned long long bk = s_ck[lane];
                int bs = s_cs[lane];
                if (s_ck[lane + 32] < bk || (s_ck[lane + 32] == bk && s_cs[lane + 32] < bs)) {
                    bk = s_ck[lane + 32];
                    bs = s_cs[lane + 32];
                }
#pragma unroll
                for (int o2 = 16; o2 >= 1; o2 >>= 1) {
                    const unsigned long long k2 = __shfl_xor_sync(kFull, bk, o2);
                    const int s2 = __shfl_xor_sync(kFull, bs, o2);
                    if (k2 < bk || (k2 == bk && s2 < bs)) {
                        bk = k2;
                        bs = s2;
                    }
                }
                if (lane == 0) {
                    EvictCand* c = p.cand + ((size_t)ub * p.Hkv + ug) * p.S + usplit;
                    c->key = bk;
                    c->slot = (bk == ~0ull) ? -1 : bs;
                    c->t = ut + 1;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_empty);
        }
    }

    // drain: copies issued into stages that no consumer waited for
    __syncthreads();
    if (!*s_abort) return;
    if (tid == 0) {
        const int issued = *s_issued;
        for (int k = max(0, issued - ST); k < issued; ++k) mbar_wait(&s_full[k % ST], (unsigned)(k / ST) & 1u, 100000000ull);
    }
    __syncthreads();
    // a CTA that gave up leaves every unit it owns in the empty state (and no eviction candidate)
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
        int b, g, split;
        unit_coords(p, u, b, g, split);
        const size_t row0 = (size_t)b * p.Hq + g * G;
        if (p.o_part != nullptr && tid < G) p.lse_part[(row0 + tid) * p.S + split] = -INFINITY;
        if (p.S == 1) {
            for (int idx = tid; idx < G * D; idx += SH::NT) {
                if (p.o_bf16) {
                    reinterpret_cast<__nv_bfloat16*>(p.o)[row0 * D + idx] = __float2bfloat16_rn(0.f);
                } else {
                    reinterpret_cast<float*>(p.o)[row0 * D + idx] = 0.f;
                }
            }
            if (tid < G && p.lse != nullptr) p.lse[row0 + tid] = -INFINITY;
        }
        if (tid == 0 && p.cand != nullptr) {
            EvictCand* c = p.cand + ((size_t)b * p.Hkv + g) * p.S + split;
            c->key = ~0ull;
            c->slot = -1;
            c->t = (p.t == nullptr) ? 0 : p.t[b] + 1;
        }
    }
}

// Merge of the num_splits states of each (b, query head) row, [ASM] step 2's
// operator with Z carried as lse. One warp per row, one pass over chunks of
// 32 splits: lane j loads split j's lse, the warp forms the running maximum
// and sum, and every lane accumulates its D/32 dims from eight independent
// L2 loads at a time (splits with zero weight are not read). Two dependent
// memory round trips for up to 32 splits.
template <int D>
__global__ void __launch_bounds__(256) merge_splits_kernel(const float* __restrict__ o_part,
                                                           const float* __restrict__ lse_part, int R, int S,
                                                           void* o, int o_bf16, float* lse) {
    griddep_wait();
    griddep_launch_dependents();
    constexpr int E = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + warp;
    if (r >= R) return;
    const float* lp = lse_part + (size_t)r * S;
    const float* op = o_part + (size_t)r * S * D + lane * E;
    float m_run = -INFINITY, s_run = 0.f;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    // the o rows of splits j + k, k < min(8, n), whose weight w (lane j + k of the chunk, or any
    // split when `spec`) is positive: empty splits are not read
    float v[8][E];
    auto load_batch = [&](int j, int n, float w, bool spec) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float* src = op + (size_t)(j + k) * D;
            const bool use = k < n && (spec || __shfl_sync(kFull, w, (j + k) & 31) > 0.f);
            if constexpr (E == 4) {
                const float4 x = use ? __ldcg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[k][0] = x.x; v[k][1] = x.y; v[k][2] = x.z; v[k][3] = x.w;
            } else {
                const float2 x = use ? __ldcg(reinterpret_cast<const float2*>(src)) : make_float2(0.f, 0.f);
                v[k][0] = x.x; v[k][1] = x.y;
            }
        }
    };
    for (int j0 = 0; j0 < S; j0 += 32) {
        const int cnt = min(32, S - j0);
        const float l = (lane < cnt) ? __ldcg(lp + j0 + lane) : -INFINITY;
        float cm = l;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, m));
        const float m_new = fmaxf(m_run, cm);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        const float a = exp2f((m_run - mu) * kLog2e);
        const float wl = exp2f((l - mu) * kLog2e);
        float ws = wl;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) ws += __shfl_xor_sync(kFull, ws, m);
        s_run = fmaf(s_run, a, ws);
        m_run = m_new;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= a;
        for (int k0 = 0; k0 < cnt; k0 += 8) {
            load_batch(j0 + k0, cnt - k0, wl, false);
            float w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = __shfl_sync(kFull, wl, (k0 + k) & 31);
            // an empty split (weight 0) contributes nothing; its o rows were never written, so they are
            // skipped rather than multiplied by 0
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k0 + k < cnt && w[k] > 0.f) {
#pragma unroll
                    for (int e = 0; e < E; ++e) acc[e] = fmaf(w[k], v[k][e], acc[e]);
                }
        }
    }
    const float inv = (s_run > 0.f) ? 1.f / s_run : 0.f;
    if (o_bf16) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(o) + (size_t)r * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) out[e] = __float2bfloat16_rn(acc[e] * inv);
    } else {
        float* out = reinterpret_cast<float*>(o) + (size_t)r * D + lane * E;
        if constexpr (E == 4) {
            *reinterpret_cast<float4*>(out) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        } else {
            *reinterpret_cast<float2*>(out) = make_float2(acc[0] * inv, acc[1] * inv);
        }
    }
    if (lane == 0 && lse != nullptr) lse[r] = (s_run > 0.f) ? m_run + log2f(s_run) * kLn2 : -INFINITY;
}

// Merge for many splits: one CTA per (b, query head) row; warp w folds a contiguous chunk of the
// splits exactly as merge_splits_kernel does, then warp 0 combines the eight partial states
// through shared memory. Every warp has at most ceil(S/8) splits in flight.
template <int D>
__global__ void __launch_bounds__(256) merge_splits_cta_kernel(const float* __restrict__ o_part,
                                                               const float* __restrict__ lse_part, int R, int S,
                                                               void* o, int o_bf16, float* lse) {
    griddep_wait();
    griddep_launch_dependents();
    constexpr int E = D / 32, NWM = 8;
    __shared__ float s_m[NWM], s_s[NWM];
    __shared__ __align__(16) float s_acc[NWM][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x;
    const int cs = (S + NWM - 1) / NWM;
    const int j_beg = min(S, warp * cs), j_end = min(S, j_beg + cs);
    const float* lp = lse_part + (size_t)r * S;
    const float* op = o_part + (size_t)r * S * D + lane * E;
    float m_run = -INFINITY, s_run = 0.f;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    // the o rows of splits j + k, k < min(8, n), whose weight w (lane j + k of the chunk, or any
    // split when `spec`) is positive: empty splits are not read
    float v[8][E];
    auto load_batch = [&](int j, int n, float w, bool spec) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float* src = op + (size_t)(j + k) * D;
            const bool use = k < n && (spec || __shfl_sync(kFull, w, (j + k) & 31) > 0.f);
            if constexpr (E == 4) {
                const float4 x = use ? __ldcg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[k][0] = x.x; v[k][1] = x.y; v[k][2] = x.z; v[k][3] = x.w;
            } else {
                const float2 x = use ? __ldcg(reinterpret_cast<const float2*>(src)) : make_float2(0.f, 0.f);
                v[k][0] = x.x; v[k][1] = x.y;
            }
        }
    };
    for (int j0 = j_beg; j0 < j_end; j0 += 32) {
        const int cnt = min(32, j_end - j0);
        load_batch(j0, cnt, 0.f, true);   // (rows here are few and their splits mostly full)
        const float l = (lane < cnt) ? __ldcg(lp + j0 + lane) : -INFINITY;
        float cm = l;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, m));
        const float m_new = fmaxf(m_run, cm);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        const float a = exp2f((m_run - mu) * kLog2e);
        const float wl = exp2f((l - mu) * kLog2e);
        float ws = wl;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) ws += __shfl_xor_sync(kFull, ws, m);
        s_run = fmaf(s_run, a, ws);
        m_run = m_new;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= a;
        for (int k0 = 0; k0 < cnt; k0 += 8) {
            if (k0 > 0) load_batch(j0 + k0, cnt - k0, wl, false);
            float w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = __shfl_sync(kFull, wl, (k0 + k) & 31);
            // an empty split (weight 0) contributes nothing; its o rows were never written, so they are
            // skipped rather than multiplied by 0
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k0 + k < cnt && w[k] > 0.f) {
#pragma unroll
                    for (int e = 0; e < E; ++e) acc[e] = fmaf(w[k], v[k][e], acc[e]);
                }
        }
    }
    if (lane == 0) {
        s_m[warp] = m_run;
        s_s[warp] = s_run;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) s_acc[warp][lane * E + e] = acc[e];
    __syncthreads();
    if (warp != 0) return;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWM; ++w) M = fmaxf(M, s_m[w]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float tot = 0.f;
    float out[E];
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = 0.f;
#pragma unroll
    for (int w = 0; w < NWM; ++w) {
        const float f = exp2f((s_m[w] - Mu) * kLog2e);
        tot = fmaf(f, s_s[w], tot);
#pragma unroll
        for (int e = 0; e < E; ++e) out[e] = fmaf(f, s_acc[w][lane * E + e], out[e]);
    }
    const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
    if (o_bf16) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(o) + (size_t)r * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) dst[e] = __float2bfloat16_rn(out[e] * inv);
    } else {
        float* dst = reinterpret_cast<float*>(o) + (size_t)r * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) dst[e] = out[e] * inv;
    }
    if (lane == 0 && lse != nullptr) lse[r] = (tot > 0.f) ? M + log2f(tot) * kLn2 : -INFINITY;
}

}  // namespace kvb
