// Query-batched decode attention over one shared cache on the 5th-generation
// tensor cores: the same computation as decode_attn_qb_kernel (many rows b
// over one cache with batch stride 0, each with its own length and position;
// "Cache What Lasts" section 2.1 logits, "Context Memorization" core method
// step 1 state, splits of a fixed length), with 128 query rows per unit:
// a unit is (block of 128 / G rows b, kv head g, split j), so every K/V tile
// is read once per 128 query rows and both products run as tcgen05.mma with
// the accumulators in tensor memory.
//
// Roles (352 threads, one CTA per SM):
//   warp 0     producer: the unit's 128 query rows by TMA (a 3-D box of 64
//              dims x G heads x 128 / G rows b, K-major with the 128-byte
//              swizzle, two buffers), K/V tiles by TMA into a 4-stage ring with
//              their pos / log beta (bias) and the tile's record;
//   warp 1     S issuer (one lane): S = Q K^T (M = 128, N = 64, K = 128) into
//              one of two S buffers, so the softmax of tile i overlaps S(i + 1);
//   warp 10    P V issuer (one lane): O += P V (M = 128, N = 128, K = 64) with
//              P read from tensor memory (A operand) and V from shared memory
//              as an MN-major B operand (two issuing threads: one thread
//              issuing both products spent most of a tile waiting to issue);
//   warps 2-9  softmax, two threads per query row (tensor-memory lane = row;
//              warps w and w + 4 share a lane quarter, each takes 32 of the
//              tile's 64 scores and 64 of O's 128 columns): read S, mask by the
//              row's length, add the row's bias, exchange the half-row maxima
//              (an mbarrier per lane quarter), keep the running maximum and
//              sum, write P as a bf16 high part and a bf16 residual (two
//              products each, ~16 bits of P) into tensor memory; at the end of
//              the unit exchange the half-row sums, read O and write the state.
// The running maximum is updated lazily: P is formed against a reference
// maximum and O is rescaled (read, scaled, written back in tensor memory)
// only when a row's maximum exceeds the reference by more than 2^8 in the
// exponent, so P <= 256; the result is the same softmax.
// Every wait is bounded (wait_ns); a CTA that gives up records
// KVB_DERR_TIMEOUT, lets its copies and MMAs finish (bounded) and writes the
// empty state for every unit it owns.
#pragma once

#include <cuda.h>

#include "asm_planes.cuh"
#include "decode_attn_qb.cuh"

namespace kvb {

template <int G>
struct QbtShape {
    static constexpr int D = 128;
    static constexpr int R = 128;             // query rows per unit = tensor-memory lanes
    static constexpr int BQ = R / G;          // rows b per unit
    static constexpr int T = 64;              // slots per tile
    static constexpr int ST = 4;              // K/V ring stages (3 left the copies of a stage freed by P V late)
    static constexpr int NT = 11 * 32;        // producer, S issuer, 8 softmax warps, P V issuer
    static constexpr int QHALF = R * 128;     // 128 rows x 64 dims of bf16
    static constexpr int QBUF = 2 * QHALF;
    static constexpr int KVHALF = T * 128;
    static constexpr int KVTILE = 2 * KVHALF;
    static constexpr int STAGE = 2 * KVTILE;  // K tile, V tile
    static constexpr int META = 16 + 2 * 64;  // tile record + (first tile) the rows' lengths, positions
    static constexpr int Q_OFF = 0;
    static constexpr int RING_OFF = Q_OFF + 2 * QBUF;
    static constexpr int POS_OFF = RING_OFF + ST * STAGE;
    static constexpr int LB_OFF = POS_OFF + ST * T * 4;
    static constexpr int META_OFF = LB_OFF + ST * T * 4;
    static constexpr int XCH_OFF = (META_OFF + ST * META * 4 + 15) / 16 * 16;   // half-row maxima [2][2][R], sums [2][R]
    static constexpr int BAR_OFF = XCH_OFF + 6 * R * 4;
    // kv full/empty [ST] each; q, s, p full/empty [2] each; pv_done [2]; o_free; fin [2]; the maxima
    // exchange [4 quarters][2]; the sums exchange [4]
    static constexpr int NBAR = 2 * ST + 6 * 2 + 2 + 1 + 2 + 8 + 4;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int END = MISC_OFF + 32;
    static constexpr size_t SMEM = 1024 + END;
    static constexpr int TM_O = 0, TM_S = 128, TM_P = 256, TM_COLS = 512;
    static_assert(G == 2 || G == 4 || G == 8, "G");
    static_assert(BQ <= 64, "rows per unit");
    static_assert(RING_OFF % 1024 == 0 && STAGE % 1024 == 0, "alignment");
    static_assert(MISC_OFF >= BAR_OFF + NBAR * 8 && BAR_OFF % 8 == 0, "barriers before the misc words");
};

// kind::f16 instruction descriptor with an MN-major B operand (bit 16)
__host__ __device__ constexpr uint32_t umma_idesc_bf16_bmn(int M, int N) { return umma_idesc_bf16(M, N) | (1u << 16); }

// 32 lanes x 16 consecutive columns from registers (lane i of the warp writes lane base + i)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A bounded wait whose outcome is the same for the whole warp (the warp then runs warp-collective
// tensor-memory instructions or leaves together).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, unsigned parity, unsigned long long ns) {
    return __all_sync(kFull, mbar_wait(bar, parity, ns));
}

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzle: 64-element MN groups
// `lbo` bytes apart, 8-row K groups `sbo` bytes apart.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

template <int G, bool BIAS>
__global__ void __launch_bounds__(QbtShape<G>::NT, 1)
    decode_attn_qbt_kernel(const __grid_constant__ DecodeQbParams p, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ) {
    using SH = QbtShape<G>;
    constexpr int D = SH::D, R = SH::R, BQ = SH::BQ, T = SH::T, ST = SH::ST;
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    int* s_pos = reinterpret_cast<int*>(smem + SH::POS_OFF);
    float* s_lb = reinterpret_cast<float*>(smem + SH::LB_OFF);
    int* s_meta = reinterpret_cast<int*>(smem + SH::META_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SH::BAR_OFF);
    uint64_t* kv_full = bars;
    uint64_t* kv_empty = bars + ST;
    uint64_t* q_full = bars + 2 * ST;
    uint64_t* q_empty = q_full + 2;
    uint64_t* s_full = q_empty + 2;
    uint64_t* s_empty = s_full + 2;
    uint64_t* p_full = s_empty + 2;
    uint64_t* p_empty = p_full + 2;
    // P V of tile i is committed to pv_done[i & 1]: a tile's softmax knows that P V(i - 2) is done
    // (it follows S(i)) and P V(i + 1) not issued, so a parity wait for P V(i - 1) or P V(i) on its
    // own barrier can never be two phases behind
    uint64_t* pv_done = p_empty + 2;
    uint64_t* o_free = pv_done + 2;
    uint64_t* fin = o_free + 1;   // [2] each MMA issuer's last commit: every operation it issued is done
    uint64_t* xm_bar = fin + 2;   // [quarter][tile parity]: both warps of a lane quarter posted their maxima
    uint64_t* xl_bar = xm_bar + 8;   // [quarter]: both posted their sums (once per unit)
    // (xl_bar + 4 == bars + NBAR: the last barrier)
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + SH::MISC_OFF);
    volatile int* s_abort = reinterpret_cast<int*>(smem + SH::MISC_OFF) + 1;
    int* s_issued = reinterpret_cast<int*>(smem + SH::MISC_OFF) + 2;   // tiles the producer issued
    int* s_qloads = reinterpret_cast<int*>(smem + SH::MISC_OFF) + 4;   // query blocks the producer loaded

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // set-up that reads nothing the previous kernel in the stream writes runs before the wait
    // for it: the barriers, and the tensor maps (kernel parameters) into the TMA unit's cache
    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&kv_full[s], 33);   // the copy's expect_tx + 32 producer lanes
            mbar_init(&kv_empty[s], 1);   // the MMA warp's commit after P V
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_full[b], 1);     // the producer's expect_tx; the copy's bytes
            mbar_init(&q_empty[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 8);    // the 8 softmax warps
            mbar_init(&p_full[b], 8);
            mbar_init(&p_empty[b], 1);
        }
        mbar_init(&pv_done[0], 1);
        mbar_init(&pv_done[1], 1);
        mbar_init(o_free, 8);
        mbar_init(&fin[0], 1);
        mbar_init(&fin[1], 1);
        for (int k = 0; k < 8; ++k) mbar_init(&xm_bar[k], 2);
        for (int k = 0; k < 4; ++k) mbar_init(&xl_bar[k], 2);
        *s_abort = 0;
        *s_issued = 0;
        *s_qloads = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmQ);
    }
    griddep_wait();
    griddep_launch_dependents();
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                     "r"(SH::TM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const int per_blk = p.Hkv * p.S;

    if (warp == 0) {
        // ======================= producer =======================
        int it = 0, ucount = 0;
        bool stop = false;
        for (int u = blockIdx.x; u < p.units + gridDim.x && !stop; u += gridDim.x) {
            const bool end = u >= p.units;
            int blk = 0, g = 0, split = 0, s0 = 0, nk = 0, ntiles = 0;
            int len_r[2] = {0, 0}, t_r[2] = {0, 0};   // rows lane, lane + 32 of the block
            if (!end) {
                blk = u / per_blk;
                g = (u - blk * per_blk) / p.S;
                split = u - blk * per_blk - g * p.S;
                int maxlen = 0;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int bq = lane + 32 * k, b = blk * BQ + bq;
                    if (bq < BQ && b < p.B) {
                        const int n = p.len[(size_t)b * p.Hkv + g];
                        const int tt = (p.t == nullptr) ? 0 : p.t[b];
                        const bool active = (p.t == nullptr) || tt >= 0;
                        const bool bad_len = n < 0 || n > p.cap;
                        const bool bad_split =
                            !bad_len && p.split_len > 0 && (long long)n > (long long)p.S * p.split_len;
                        if ((bad_len || bad_split) && split == 0) raise_error(bad_len ? KVB_DERR_LEN : KVB_DERR_SPLIT);
                        len_r[k] = (bad_len || bad_split || !active) ? 0 : n;
                        t_r[k] = tt;
                    }
                    maxlen = max(maxlen, len_r[k]);
                }
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) maxlen = max(maxlen, __shfl_xor_sync(kFull, maxlen, m));
                const long long C = p.split_len > 0 ? (long long)p.split_len : (long long)maxlen;
                s0 = (int)min((long long)split * C, (long long)maxlen);
                const int s1 = (int)min((long long)s0 + C, (long long)maxlen);
                nk = s1 - s0;
                ntiles = (nk + T - 1) / T;
                if (ntiles == 0) {
                    for (int r = 0; r < R; ++r) {
                        const int b = blk * BQ + r / G;
                        if (b >= p.B) continue;
                        const size_t row = (size_t)b * p.Hq + g * G + r % G;
                        if (lane == 0 && p.o_part != nullptr) p.lse_part[row * p.S + split] = -INFINITY;
                        if (p.S == 1) {
                            for (int e = lane; e < D; e += 32) {
                                if (p.o_bf16) {
                                    reinterpret_cast<__nv_bfloat16*>(p.o)[row * D + e] = __float2bfloat16_rn(0.f);
                                } else {
                                    reinterpret_cast<float*>(p.o)[row * D + e] = 0.f;
                                }
                            }
                            if (lane == 0 && p.lse != nullptr) p.lse[row] = -INFINITY;
                        }
                    }
                    continue;
                }
            }
            if (p.withhold) {   // test hook: no copy, no arrival; the other roles' waits run out
                stop = true;
                break;
            }
            int qb = 0;
            if (!end) {
                // the unit's queries into buffer qb (free once the MMAs of the unit two back are done):
                // rows b = blk * BQ .. (zeros past B), heads g * G .., both 64-dim halves
                qb = ucount & 1;
                if (ucount >= 2 && !warp_wait(&q_empty[qb], (unsigned)((ucount >> 1) - 1) & 1u, p.wait_ns)) {
                    if (lane == 0) {
                        raise_error(KVB_DERR_TIMEOUT);
                        *s_abort = 1;
                    }
                    break;
                }
                if (lane == 0) {
                    unsigned char* qbuf = smem + SH::Q_OFF + qb * SH::QBUF;
                    mbar_arrive_expect_tx(&q_full[qb], (unsigned)SH::QBUF);
                    tma_load_4d(qbuf, &tmQ, 0, g * G, blk * BQ, 0, &q_full[qb]);
                    tma_load_4d(qbuf + SH::QHALF, &tmQ, 64, g * G, blk * BQ, 0, &q_full[qb]);
                }
                ++ucount;
            }
            const int records = end ? 1 : ntiles;
            const size_t m_off = end ? 0 : (size_t)g * p.m_sh + (size_t)s0;
            for (int i = 0; i < records; ++i, ++it) {
                const int st = it % ST;
                int psv[2];
                float lbv[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int key = i * T + lane + 32 * j;
                    psv[j] = 0;
                    lbv[j] = 0.f;
                    if (BIAS && !end && key < nk) {
                        psv[j] = p.pos[m_off + key];
                        lbv[j] = p.lb[m_off + key];
                    }
                }
                if (it >= ST && !warp_wait(&kv_empty[st], (unsigned)((it / ST) - 1) & 1u, p.wait_ns)) {
                    if (lane == 0) {
                        raise_error(KVB_DERR_TIMEOUT);
                        *s_abort = 1;
                    }
                    stop = true;
                    break;
                }
                if (__any_sync(kFull, *s_abort != 0)) {
                    stop = true;
                    break;
                }
                int* m = s_meta + st * SH::META;
                if (lane == 0) {
                    m[0] = end ? -1 : u;
                    m[1] = i;
                    m[2] = end ? 0 : ntiles;
                    m[3] = end ? 0 : min(T, nk - i * T);
                    m[4] = blk;
                    m[5] = g;
                    m[6] = split;
                    m[7] = s0 + i * T;
                    m[8] = s0 + nk;
                    m[9] = qb;
                    mbar_arrive_expect_tx(&kv_full[st], end ? 0u : (unsigned)SH::STAGE);
                    if (!end) {
                        unsigned char* kt = smem + SH::RING_OFF + st * SH::STAGE;
                        unsigned char* vt = kt + SH::KVTILE;
                        const int row = s0 + i * T;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            tma_load_4d(kt + h * SH::KVHALF, &tmK, 64 * h, row, g, 0, &kv_full[st]);
                            tma_load_4d(vt + h * SH::KVHALF, &tmV, 64 * h, row, g, 0, &kv_full[st]);
                        }
                    }
                }
                if (!end && i == 0) {
#pragma unroll
                    for (int k = 0; k < 2; ++k)
                        if (lane + 32 * k < BQ) {
                            m[16 + lane + 32 * k] = len_r[k];
                            m[16 + 64 + lane + 32 * k] = t_r[k];
                        }
                }
                if (BIAS) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        s_pos[st * T + lane + 32 * j] = psv[j];
                        s_lb[st * T + lane + 32 * j] = lbv[j];
                    }
                }
                __syncwarp();
                mbar_arrive(&kv_full[st]);
            }
        }
        if (lane == 0) {
            *s_issued = it;
            *s_qloads = ucount;
        }
    } else if (warp == 1 || warp == SH::NT / 32 - 1) {
        // ============ MMA issuers: S = Q K^T (warp 1), O += P V (the last warp) ============
        // Two threads, so that neither product's issue waits behind the other's: tile i's P V
        // needs P(i), hence S(i), hence Q K^T(i) done, so the stage it frees (kv_empty, committed
        // after P V) is no longer read by either.
        if (lane == 0) {
            const bool qk = warp == 1;
            constexpr uint32_t idesc_s = umma_idesc_bf16(R, T);          // S: 128 x 64
            constexpr uint32_t idesc_o = umma_idesc_bf16_bmn(R, D);      // O: 128 x 128, V MN-major
            int units = 0;
            auto fail = [&]() {
                raise_error(KVB_DERR_TIMEOUT);
                *s_abort = 1;
            };
            for (int i = 0;; ++i) {
                const int st = i % ST;
                if (!mbar_wait(&kv_full[st], (unsigned)(i / ST) & 1u, p.wait_ns)) { fail(); break; }
                const int* m = s_meta + st * SH::META;
                const int u = m[0];
                if (u < 0) break;   // the end record
                const int ti = m[1], ntiles = m[2], qb = m[9];
                const int sb = i & 1;
                if (qk) {
                    // S(i) into buffer i % 2; a unit's first tile waits for its queries (the k-th unit
                    // uses query buffer k % 2 for the (k / 2)-th time)
                    if (ti == 0) {
                        if (!mbar_wait(&q_full[qb], (unsigned)(units >> 1) & 1u, p.wait_ns)) { fail(); break; }
                        ++units;
                    }
                    if (i >= 2 && !mbar_wait(&s_empty[sb], (unsigned)((i >> 1) - 1) & 1u, p.wait_ns)) { fail(); break; }
                    tc_fence_after();
                    const uint32_t qa = sbase + SH::Q_OFF + qb * SH::QBUF;
                    const uint32_t kt = sbase + SH::RING_OFF + st * SH::STAGE;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t aoff = (kk >> 2) * SH::QHALF + (kk & 3) * 32;
                        const uint32_t boff = (kk >> 2) * SH::KVHALF + (kk & 3) * 32;
                        umma_bf16(tmem + SH::TM_S + sb * 64, umma_desc_sw128(qa + aoff), umma_desc_sw128(kt + boff),
                                  idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[sb]);
                    if (ti == ntiles - 1) umma_commit(&q_empty[qb]);
                } else {
                    // O += P(i) V(i); a unit's first tile waits until the previous unit's O was read
                    const int pb = sb;
                    if (!mbar_wait(&p_full[pb], (unsigned)(i >> 1) & 1u, p.wait_ns)) { fail(); break; }
                    if (ti == 0) {
                        if (units > 0 && !mbar_wait(o_free, (unsigned)(units - 1) & 1u, p.wait_ns)) { fail(); break; }
                        ++units;
                    }
                    tc_fence_after();
                    const uint32_t vt = sbase + SH::RING_OFF + st * SH::STAGE + SH::KVTILE;
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int kk = 0; kk < T / 16; ++kk) {
                            const uint32_t a = tmem + SH::TM_P + pb * 64 + part * 32 + kk * 8;
                            const uint64_t bd = umma_desc_sw128_mn(vt + kk * 2048, SH::KVHALF, 1024);
                            umma_bf16_ts(tmem + SH::TM_O, a, bd, idesc_o, (ti == 0 && part == 0 && kk == 0) ? 0u : 1u);
                        }
                    umma_commit(&kv_empty[st]);
                    umma_commit(&p_empty[pb]);
                    umma_commit(&pv_done[pb]);
                }
            }
        }
    } else {
        // ======================= softmax warps (2 .. 9) =======================
        const int quarter = warp & 3;             // tensor-memory lanes 32 * quarter ..
        const int half = (warp - 2) >> 2;         // scores 32 half .. of a tile, O columns 64 half ..
        const int r = 32 * quarter + lane;        // this thread's query row
        const int sidx = (warp - 2) * 32 + lane;  // 0 .. 255
        const uint32_t tl = tmem + ((uint32_t)(32 * quarter) << 16);
        float* xm = reinterpret_cast<float*>(smem + SH::XCH_OFF);   // [tile parity][half][R]
        float* xl = xm + 4 * R;                                      // [half][R]
        const float C = p.scale * kLog2e;         // scores in log2 units: the maxima and P below are too
        float m_ref = -INFINITY, l_sum = 0.f;
        int lim = 0, trow = 0, units_done = 0;
        auto fail = [&]() {
            if (lane == 0) {
                raise_error(KVB_DERR_TIMEOUT);
                *s_abort = 1;
            }
        };
        for (int i = 0;; ++i) {
            const int st = i % ST;
            if (!warp_wait(&kv_full[st], (unsigned)(i / ST) & 1u, p.wait_ns)) { fail(); break; }
            const int* m = s_meta + st * SH::META;
            const int u = m[0];
            if (u < 0) break;
            const int ti = m[1], ntiles = m[2], rows = m[3], ublk = m[4], ug = m[5], usplit = m[6], base = m[7],
                      s1 = m[8];
            if (rows < T) {
                // V rows past the unit's last slot may hold any bytes: zero them (their P is 0, and
                // 0 times a NaN would not be); the tensor cores read them only in P V(i), after p_full
                unsigned char* vt = smem + SH::RING_OFF + st * SH::STAGE + SH::KVTILE;
                for (int idx = sidx; idx < (T - rows) * 16; idx += 256) {
                    const int row = rows + (idx >> 4), c = idx & 15;
                    *reinterpret_cast<uint4*>(vt + (c >> 3) * SH::KVHALF + row * 128 + (((c & 7) ^ (row & 7)) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
            }
            if (ti == 0) {
                lim = min(m[16 + r / G], s1);
                trow = m[16 + 64 + r / G];
                m_ref = -INFINITY;
                l_sum = 0.f;
            }
            const int sb = i & 1;
            if (!warp_wait(&s_full[sb], (unsigned)(i >> 1) & 1u, p.wait_ns)) { fail(); break; }
            tc_fence_after();
            float x[32];
            tmem_ld32(tl + SH::TM_S + sb * 64 + 32 * half, x);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[sb]);
            const int c0 = base + 32 * half;
            float mh = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float bj = 0.f;
                if constexpr (BIAS)
                    bj = __fmul_rn(__int2float_rn(trow - s_pos[st * T + 32 * half + j]), s_lb[st * T + 32 * half + j]) *
                         kLog2e;
                x[j] = (c0 + j < lim) ? fmaf(x[j], C, bj) : -INFINITY;
                mh = fmaxf(mh, x[j]);
            }
            // the row's maximum over both halves (slot i % 2: the partner reads slot i % 2 before it can
            // post tile i + 2's maximum there, since that needs this thread's post of tile i + 1)
            xm[(sb * 2 + half) * R + r] = mh;
            __syncwarp();
            if (lane == 0) mbar_arrive(&xm_bar[quarter * 2 + sb]);
            if (!warp_wait(&xm_bar[quarter * 2 + sb], (unsigned)(i >> 1) & 1u, p.wait_ns)) { fail(); break; }
            const float mt = fmaxf(mh, xm[(sb * 2 + 1 - half) * R + r]);
            // the reference moves when the row's maximum passes it by more than 2^8; the rows that
            // had one already rescale their half of O. Tensor-memory loads and stores are
            // warp-collective, so the whole warp takes the rescale when any of its rows needs it.
            const bool grow = mt > m_ref && (m_ref == -INFINITY || mt - m_ref > 8.f);
            const bool resc = grow && m_ref != -INFINITY;
            if (__any_sync(kFull, resc)) {
                // every earlier P V product of this unit first (P V(i - 1); i > 0 here)
                if (!warp_wait(&pv_done[(i - 1) & 1], (unsigned)((i - 1) >> 1) & 1u, p.wait_ns)) { fail(); break; }
                tc_fence_after();
                const float alpha = resc ? ex2_approx(m_ref - mt) : 1.f;
#pragma unroll
                for (int c = 0; c < 64; c += 32) {
                    float o[32];
                    tmem_ld32(tl + SH::TM_O + 64 * half + c, o);
                    tmem_ld_wait();
                    uint32_t w[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(o[e] * alpha);
                    tmem_st32(tl + SH::TM_O + 64 * half + c, w);
                }
                tmem_st_wait();
                l_sum *= alpha;
            }
            if (grow) m_ref = mt;
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            uint32_t hi[16], lo[16];
            float ssum = 0.f;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const float p0 = ex2_approx(x[j] - m_use), p1 = ex2_approx(x[j + 1] - m_use);
                ssum += p0 + p1;
                hi[j / 2] = pack_bf16(p0, p1);
                lo[j / 2] = pack_bf16(p0 - __uint_as_float(hi[j / 2] << 16), p1 - __uint_as_float(hi[j / 2] & 0xffff0000u));
            }
            l_sum += ssum;
            const int pb = i & 1;
            if (i >= 2 && !warp_wait(&p_empty[pb], (unsigned)((i >> 1) - 1) & 1u, p.wait_ns)) { fail(); break; }
            tc_fence_after();
            tmem_st16(tl + SH::TM_P + pb * 64 + 16 * half, hi);
            tmem_st16(tl + SH::TM_P + pb * 64 + 32 + 16 * half, lo);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[pb]);
            if (ti != ntiles - 1) continue;

            // ---- end of unit: the row's sum over both halves; this thread's half of O, divided by it
            if (!warp_wait(&pv_done[i & 1], (unsigned)(i >> 1) & 1u, p.wait_ns)) { fail(); break; }
            tc_fence_after();
            float o[64];
            tmem_ld32(tl + SH::TM_O + 64 * half, o);
            tmem_ld32(tl + SH::TM_O + 64 * half + 32, o + 32);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
            xl[half * R + r] = l_sum;
            __syncwarp();
            if (lane == 0) mbar_arrive(&xl_bar[quarter]);
            if (!warp_wait(&xl_bar[quarter], (unsigned)units_done & 1u, p.wait_ns)) { fail(); break; }
            const float lt = l_sum + xl[(1 - half) * R + r];
            // the partner has read this thread's sum before it can post the next unit's (that needs
            // this thread's maxima of the next unit's first tile)
            ++units_done;
            const int b = ublk * BQ + r / G;
            if (b < p.B) {
                const size_t row = (size_t)b * p.Hq + ug * G + r % G;
                const float inv = (lt > 0.f) ? 1.f / lt : 0.f;
                const float lse = (lt > 0.f) ? (m_ref + log2f(lt)) * kLn2 : -INFINITY;
                if (p.o_part != nullptr) {
                    float4* dst = reinterpret_cast<float4*>(p.o_part + (row * p.S + usplit) * D + 64 * half);
#pragma unroll
                    for (int e = 0; e < 64; e += 4)
                        dst[e / 4] = make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
                    if (half == 0) p.lse_part[row * p.S + usplit] = lse;
                }
                if (p.S == 1) {
                    if (p.o_bf16) {
                        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.o) + row * D + 64 * half;
#pragma unroll
                        for (int e = 0; e < 64; ++e) dst[e] = __float2bfloat16_rn(o[e] * inv);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o) + row * D + 64 * half);
#pragma unroll
                        for (int e = 0; e < 64; e += 4)
                            dst[e / 4] = make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv);
                    }
                    if (half == 0 && p.lse != nullptr) p.lse[row] = lse;
                }
            }
        }
    }

    // ---- teardown: copies and MMAs in flight finish (bounded) before the tensor memory goes
    tc_fence_before();
    __syncthreads();
    if ((warp == 1 || warp == SH::NT / 32 - 1) && lane == 0) {
        uint64_t* f = &fin[warp == 1 ? 0 : 1];
        umma_commit(f);   // arrives when every tensor-core operation this thread issued is done
        mbar_wait(f, 0u, p.wait_ns);
    }
    if (tid == 0 && *s_abort) {
        const int issued = *s_issued;
        for (int k = max(0, issued - ST); k < issued; ++k)
            mbar_wait(&kv_full[k % ST], (unsigned)(k / ST) & 1u, 100000000ull);
        // query copies: at most one in flight per buffer (the one before it was consumed)
        const int ql = *s_qloads;
        for (int k = max(0, ql - 2); k < ql; ++k) mbar_wait(&q_full[k & 1], (unsigned)(k >> 1) & 1u, 100000000ull);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(SH::TM_COLS) : "memory");
    }
    if (!*s_abort) return;
    // a CTA that gave up leaves every unit it owns in the empty state
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
        const int blk = u / per_blk;
        const int g = (u - blk * per_blk) / p.S;
        const int split = u - blk * per_blk - g * p.S;
        for (int r = warp; r < R; r += SH::NT / 32) {
            const int b = blk * BQ + r / G;
            if (b >= p.B) continue;
            const size_t row = (size_t)b * p.Hq + g * G + r % G;
            if (lane == 0 && p.o_part != nullptr) p.lse_part[row * p.S + split] = -INFINITY;
            if (p.S == 1) {
                for (int e = lane; e < D; e += 32) {
                    if (p.o_bf16) {
                        reinterpret_cast<__nv_bfloat16*>(p.o)[row * D + e] = __float2bfloat16_rn(0.f);
                    } else {
                        reinterpret_cast<float*>(p.o)[row * D + e] = 0.f;
                    }
                }
                if (lane == 0 && p.lse != nullptr) p.lse[row] = -INFINITY;
            }
        }
    }
}

}  // namespace kvb
