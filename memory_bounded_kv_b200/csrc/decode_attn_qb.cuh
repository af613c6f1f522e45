// Query-batched decode attention over one cache shared by many rows (batch
// stride 0): the queries of several consecutive positions of one sequence
// attending to a common prefix, each with its own length (causal) and, with
// the retention bias of "Cache What Lasts" section 2.1, its own position t.
// Same state and split semantics as decode_attn_tc_kernel ("Context
// Memorization" core method step 1; splits of a fixed length), but a unit is
// (block of BQ = 16 / G rows b, kv head g, split j): the BQ x G query rows of
// the block fill all 16 M rows of the m16n8k16 tensor-core tiles, and every
// K/V tile is read from memory once per block instead of once per row b.
//
// Structure as decode_attn_tc_kernel: one producer warp streams the split's
// K/V tiles by TMA into a STAGES-deep ring (with the tile's pos and log beta
// when the bias is on), four consumer warps each own 16 slots of a tile.
// Differences: every lane holds two query rows (r and r + 8) of the
// accumulator layout; the length mask and the bias are formed per row in the
// consumers; the unit's geometry is the longest row of the block.
// Every wait is bounded (wait_ns); a CTA that gives up records
// KVB_DERR_TIMEOUT, drains its copies and writes the empty state for every
// unit it owns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode_attn_tc.cuh"

namespace kvb {

struct DecodeQbParams {
    const uint16_t* q;
    long long q_sb, q_sh;
    const float* lb;      // [Hkv, cap] (one shared row per kv head), nullable
    const int* pos;
    long long m_sh;
    const int* len;       // [B, Hkv]
    const int* t;         // [B], nullable without bias
    int B, Hq, Hkv, cap, S, split_len;   // split_len > 0, or S == 1
    int blocks;           // ceil(B / BQ)
    int units;            // blocks * Hkv * S
    float scale;
    float* o_part;
    float* lse_part;
    void* o;
    int o_bf16;
    float* lse;
    unsigned long long wait_ns;
    int withhold;
};

template <int D, int G>
struct QbShape {
    static constexpr int BQ = 16 / G;             // rows b per unit
    static constexpr int R = 16;                  // query rows per unit (BQ x G)
    static constexpr int NWC = 4;
    static constexpr int NT = (NWC + 1) * 32;
    static constexpr int T = 16 * NWC;
    static constexpr int STAGES = 2;              // two CTAs per SM: 8 consumer warps hide the MMA latency
    static constexpr int HALVES = D / 64;
    static constexpr int HALF_BYTES = T * 128;
    static constexpr int TILE_BYTES = HALVES * HALF_BYTES;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int KSTEPS = D / 16;
    static constexpr int NTILES = D / 8;
    static constexpr int QBYTES = R * D * 2;
    static constexpr int META = 64;               // ints per stage: unit fields, BQ lengths, BQ positions
    static constexpr int RING_OFF = 0;
    static constexpr int Q_OFF = RING_OFF + STAGES * STAGE_BYTES;       // [ST][R][D] bf16
    static constexpr int POS_OFF = Q_OFF + STAGES * QBYTES;             // [ST][T] int
    static constexpr int LB_OFF = POS_OFF + STAGES * T * 4;             // [ST][T] f32
    static constexpr int META_OFF = LB_OFF + STAGES * T * 4;            // [ST][META] int
    static constexpr int BAR_OFF = META_OFF + STAGES * META * 4;        // full[ST], empty[ST]
    static constexpr int MISC_OFF = BAR_OFF + 2 * STAGES * 8;           // abort, issued
    static constexpr int EPI_OFF = (MISC_OFF + 16 + 15) / 16 * 16;      // [NWC][R][D] f32
    static constexpr int ML_OFF = EPI_OFF + NWC * R * D * 4;            // [NWC][R][2] f32
    static constexpr int END_OFF = ML_OFF + NWC * R * 2 * 4;
    static constexpr size_t SMEM = 1024 + END_OFF;
    static_assert(D == 64 || D == 128, "d");
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "G");
    static_assert(STAGE_BYTES % 1024 == 0 && Q_OFF % 16 == 0, "alignment");
    static_assert(16 + 2 * BQ <= META, "meta");
};

// D = A . B + C, m16n8k16, bf16 inputs, fp32 accumulators, all 16 A rows.
__device__ __forceinline__ void mma_bf16_16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Writes the empty state (o = 0, lse = -inf; only lse_part with several splits) of query row r
// (0 <= r < 16) of unit (blk, g, split); rows past B are skipped.
template <int D, int G>
__device__ __forceinline__ void qb_empty_row(const DecodeQbParams& p, int blk, int g, int split, int r, int lane0,
                                             int stride) {
    const int b = blk * (16 / G) + r / G;
    if (b >= p.B) return;
    const size_t row = (size_t)b * p.Hq + g * G + r % G;
    if (lane0 == 0 && p.o_part != nullptr) p.lse_part[row * p.S + split] = -INFINITY;
    if (p.S == 1) {
        for (int e = lane0; e < D; e += stride) {
            if (p.o_bf16) {
                reinterpret_cast<__nv_bfloat16*>(p.o)[row * D + e] = __float2bfloat16_rn(0.f);
            } else {
                reinterpret_cast<float*>(p.o)[row * D + e] = 0.f;
            }
        }
        if (lane0 == 0 && p.lse != nullptr) p.lse[row] = -INFINITY;
    }
}

template <int D, int G, bool BIAS>
__global__ void __launch_bounds__(QbShape<D, G>::NT, 2)
    decode_attn_qb_kernel(const __grid_constant__ DecodeQbParams p, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV) {
    using SH = QbShape<D, G>;
    constexpr int NWC = SH::NWC, T = SH::T, ST = SH::STAGES, BQ = SH::BQ, R = SH::R;
    extern __shared__ unsigned char smem_dyn[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
    uint16_t* s_q = reinterpret_cast<uint16_t*>(smem + SH::Q_OFF);
    int* s_pos = reinterpret_cast<int*>(smem + SH::POS_OFF);
    float* s_lb = reinterpret_cast<float*>(smem + SH::LB_OFF);
    int* s_meta = reinterpret_cast<int*>(smem + SH::META_OFF);
    uint64_t* s_full = reinterpret_cast<uint64_t*>(smem + SH::BAR_OFF);
    uint64_t* s_empty = s_full + ST;
    volatile int* s_abort = reinterpret_cast<int*>(smem + SH::MISC_OFF);
    int* s_issued = reinterpret_cast<int*>(smem + SH::MISC_OFF) + 1;
    float* s_o = reinterpret_cast<float*>(smem + SH::EPI_OFF);
    float* s_ml = reinterpret_cast<float*>(smem + SH::ML_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_wait();
    griddep_launch_dependents();
    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&s_full[s], 33);
            mbar_init(&s_empty[s], NWC * 32);
        }
        *s_abort = 0;
        *s_issued = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int per_blk = p.Hkv * p.S;

    if (warp == NWC) {
        // ======================= producer warp =======================
        int it = 0;
        bool stop = false;
        for (int u = blockIdx.x; u < p.units + gridDim.x && !stop; u += gridDim.x) {
            const bool end = u >= p.units;
            int blk = 0, g = 0, split = 0, s0 = 0, nk = 0, ntiles = 0, my_len = 0, my_t = 0;
            if (!end) {
                blk = u / per_blk;
                g = (u - blk * per_blk) / p.S;
                split = u - blk * per_blk - g * p.S;
                // lane r < BQ: row b = blk * BQ + r of the block
                const int b = blk * BQ + lane;
                if (lane < BQ && b < p.B) {
                    const int n = p.len[(size_t)b * p.Hkv + g];
                    my_t = (p.t == nullptr) ? 0 : p.t[b];
                    const bool active = (p.t == nullptr) || my_t >= 0;
                    const bool bad_len = n < 0 || n > p.cap;
                    const bool bad_split = !bad_len && p.split_len > 0 && (long long)n > (long long)p.S * p.split_len;
                    if ((bad_len || bad_split) && split == 0) raise_error(bad_len ? KVB_DERR_LEN : KVB_DERR_SPLIT);
                    my_len = (bad_len || bad_split || !active) ? 0 : n;
                }
                int maxlen = my_len;
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) maxlen = max(maxlen, __shfl_xor_sync(kFull, maxlen, m));
                const long long C = p.split_len > 0 ? (long long)p.split_len : (long long)maxlen;
                s0 = (int)min((long long)split * C, (long long)maxlen);
                const int s1 = (int)min((long long)s0 + C, (long long)maxlen);
                nk = s1 - s0;
                ntiles = (nk + T - 1) / T;
                if (ntiles == 0) {
                    // nothing of this split is visible to any row of the block: empty states
                    for (int r = 0; r < R; ++r) qb_empty_row<D, G>(p, blk, g, split, r, lane, 32);
                    continue;
                }
            }
            if (p.withhold) {   // test hook: no copy, no arrival; the consumers' wait runs out
                stop = true;
                break;
            }
            const int records = end ? 1 : ntiles;
            const size_t m_off = end ? 0 : (size_t)g * p.m_sh + (size_t)s0;
            for (int i = 0; i < records; ++i, ++it) {
                const int st = it % ST;
                int psv[T / 32];
                float lbv[T / 32];
#pragma unroll
                for (int j = 0; j < T / 32; ++j) {
                    const int key = i * T + lane + 32 * j;
                    psv[j] = 0;
                    lbv[j] = 0.f;
                    if (BIAS && !end && key < nk) {
                        psv[j] = p.pos[m_off + key];
                        lbv[j] = p.lb[m_off + key];
                    }
                }
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
                int* m = s_meta + st * SH::META;
                const bool with_q = !end && i == 0;
                if (lane == 0) {
                    m[0] = end ? -1 : u;
                    m[1] = i;
                    m[2] = end ? 0 : ntiles;
                    m[3] = end ? 0 : min(T, nk - i * T);   // valid slots of this tile
                    m[4] = blk;
                    m[5] = g;
                    m[6] = split;
                    m[7] = s0 + i * T;                       // first slot of the tile
                    m[8] = s0 + nk;                          // end of the unit's slot range
                    unsigned tx = end ? 0u : (unsigned)SH::STAGE_BYTES;
                    if (with_q) {
                        for (int bq = 0; bq < BQ; ++bq)
                            if (blk * BQ + bq < p.B) tx += G * D * 2;
                    }
                    mbar_arrive_expect_tx(&s_full[st], tx);
                    if (!end) {
                        unsigned char* kt = smem + SH::RING_OFF + st * SH::STAGE_BYTES;
                        unsigned char* vt = kt + SH::TILE_BYTES;
                        const int row = s0 + i * T;
#pragma unroll
                        for (int h = 0; h < SH::HALVES; ++h) {
                            tma_load_4d(kt + h * SH::HALF_BYTES, &tmK, 64 * h, row, g, 0, &s_full[st]);
                            tma_load_4d(vt + h * SH::HALF_BYTES, &tmV, 64 * h, row, g, 0, &s_full[st]);
                        }
                    }
                    if (with_q) {
                        uint16_t* qdst = s_q + st * R * D;
                        for (int bq = 0; bq < BQ; ++bq) {
                            const int b = blk * BQ + bq;
                            if (b >= p.B) continue;
                            const uint16_t* qsrc = p.q + (size_t)b * p.q_sb + (size_t)(g * G) * p.q_sh;
                            if (p.q_sh == D) {
                                bulk_g2s(qdst + bq * G * D, qsrc, (unsigned)(G * D * 2), &s_full[st]);
                            } else {
                                for (int hh = 0; hh < G; ++hh)
                                    bulk_g2s(qdst + (bq * G + hh) * D, qsrc + (size_t)hh * p.q_sh, (unsigned)(D * 2),
                                             &s_full[st]);
                            }
                        }
                    }
                }
                if (with_q) {
                    // per-row length and position for the consumers; rows past B get zero queries
                    if (lane < BQ) {
                        m[16 + lane] = my_len;
                        m[16 + BQ + lane] = my_t;
                    }
                    for (int bq = 0; bq < BQ; ++bq) {
                        if (blk * BQ + bq < p.B) continue;
                        uint32_t* z = reinterpret_cast<uint32_t*>(s_q + st * R * D + bq * G * D);
                        for (int e = lane; e < G * D / 2; e += 32) z[e] = 0u;
                    }
                }
                if (BIAS) {
#pragma unroll
                    for (int j = 0; j < T / 32; ++j) {
                        s_pos[st * T + lane + 32 * j] = psv[j];
                        s_lb[st * T + lane + 32 * j] = lbv[j];
                    }
                }
                __syncwarp();
                mbar_arrive(&s_full[st]);
            }
        }
        if (lane == 0) *s_issued = it;
    } else {
        // ======================= consumer warps =======================
        const int r0 = lane >> 2, r1 = r0 + 8;   // this lane's two query rows
        const int cq = lane & 3;
        const int kw = 16 * warp;
        const uint32_t ring = smem_u32(smem + SH::RING_OFF);
        const int kq_row = kw + (lane & 7) + ((lane >> 4) << 3);
        const int kq_hi = (lane >> 3) & 1;
        const int v_row = kw + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int v_hi = lane >> 4;
        const int sw = lane & 7;

        uint32_t qa[SH::KSTEPS][4];
        float acc[SH::NTILES][4];
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
        int lim[2] = {0, 0}, trow[2] = {0, 0};
        int it = 0;
        while (true) {
            const int st = it % ST;
            if (!mbar_wait(&s_full[st], (unsigned)(it / ST) & 1u, p.wait_ns)) {
                if (lane == 0) {
                    raise_error(KVB_DERR_TIMEOUT);
                    *s_abort = 1;
                }
                break;
            }
            const int* m = s_meta + st * SH::META;
            const int u = m[0], i = m[1], ntiles = m[2], rows = m[3];
            if (u < 0) break;
            const int ublk = m[4], ug = m[5], usplit = m[6], base = m[7], s1 = m[8];
            if (i == 0) {
                m_run[0] = m_run[1] = -INFINITY;
                l_run[0] = l_run[1] = 0.f;
#pragma unroll
                for (int j = 0; j < SH::NTILES; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
                const uint16_t* qs = s_q + st * R * D;
#pragma unroll
                for (int s = 0; s < SH::KSTEPS; ++s) {
                    qa[s][0] = *reinterpret_cast<const uint32_t*>(qs + r0 * D + 16 * s + 2 * cq);
                    qa[s][1] = *reinterpret_cast<const uint32_t*>(qs + r1 * D + 16 * s + 2 * cq);
                    qa[s][2] = *reinterpret_cast<const uint32_t*>(qs + r0 * D + 16 * s + 8 + 2 * cq);
                    qa[s][3] = *reinterpret_cast<const uint32_t*>(qs + r1 * D + 16 * s + 8 + 2 * cq);
                }
                lim[0] = min(m[16 + r0 / G], s1);
                lim[1] = min(m[16 + r1 / G], s1);
                trow[0] = m[16 + BQ + r0 / G];
                trow[1] = m[16 + BQ + r1 / G];
            }
            const uint32_t kt = ring + st * SH::STAGE_BYTES;
            const uint32_t vt = kt + SH::TILE_BYTES;
            // ---- S = Q K^T for this warp's 16 slots (two n-tiles of 8), all 16 query rows; even and
            // odd K steps accumulate separately (two independent chains), then add
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            float sd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int s = 0; s < SH::KSTEPS; ++s) {
                const int chunk = 2 * (s & 3) + kq_hi;
                const uint32_t addr = kt + (s >> 2) * SH::HALF_BYTES + kq_row * 128 + ((chunk ^ sw) << 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(addr, b0, b1, b2, b3);
                float (&c0)[4] = (s & 1) ? sd[0] : sc[0];
                float (&c1)[4] = (s & 1) ? sd[1] : sc[1];
                mma_bf16_16(c0, qa[s][0], qa[s][1], qa[s][2], qa[s][3], b0, b1);
                mma_bf16_16(c1, qa[s][0], qa[s][1], qa[s][2], qa[s][3], b2, b3);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sc[0][j] += sd[0][j];
                sc[1][j] += sd[1][j];
            }
            if (rows < T && kw + 16 > rows) {
                // tail: zero this warp's V rows past the unit's last slot (K there is masked)
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
            // ---- logits per row: slots kw+2cq, +1, kw+8+2cq, +1 of the tile
            const int sl[4] = {kw + 2 * cq, kw + 2 * cq + 1, kw + 8 + 2 * cq, kw + 8 + 2 * cq + 1};
            float bias[2][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if constexpr (BIAS) {
                    const int ps = s_pos[st * T + sl[j]];
                    const float l = s_lb[st * T + sl[j]];
                    bias[0][j] = __fmul_rn(__int2float_rn(trow[0] - ps), l);
                    bias[1][j] = __fmul_rn(__int2float_rn(trow[1] - ps), l);
                } else {
                    bias[0][j] = bias[1][j] = 0.f;
                }
            }
            float pr[2][4];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                float x[4];
                const float raw[4] = {sc[0][2 * rr], sc[0][2 * rr + 1], sc[1][2 * rr], sc[1][2 * rr + 1]};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    x[j] = (base + sl[j] < lim[rr]) ? fmaf(raw[j], p.scale, bias[rr][j]) : -INFINITY;
                float tmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
                tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 1));
                tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 2));
                const float m_new = fmaxf(m_run[rr], tmax);
                const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
                const float alpha = exp2f((m_run[rr] - m_use) * kLog2e);
#pragma unroll
                for (int j = 0; j < 4; ++j) pr[rr][j] = exp2f((x[j] - m_use) * kLog2e);
                l_run[rr] = fmaf(l_run[rr], alpha, (pr[rr][0] + pr[rr][1]) + (pr[rr][2] + pr[rr][3]));
                m_run[rr] = m_new;
                if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
                    for (int j = 0; j < SH::NTILES; ++j) {
                        acc[j][2 * rr] *= alpha;
                        acc[j][2 * rr + 1] *= alpha;
                    }
                }
            }
            // ---- P as the A operand (rows r0, r1; slots 2cq.., 8+2cq..): high bf16 part and residual
            const uint32_t ph0 = pack_bf16(pr[0][0], pr[0][1]);
            const uint32_t ph1 = pack_bf16(pr[1][0], pr[1][1]);
            const uint32_t ph2 = pack_bf16(pr[0][2], pr[0][3]);
            const uint32_t ph3 = pack_bf16(pr[1][2], pr[1][3]);
            const uint32_t pl0 = pack_bf16(pr[0][0] - __uint_as_float(ph0 << 16), pr[0][1] - __uint_as_float(ph0 & 0xffff0000u));
            const uint32_t pl1 = pack_bf16(pr[1][0] - __uint_as_float(ph1 << 16), pr[1][1] - __uint_as_float(ph1 & 0xffff0000u));
            const uint32_t pl2 = pack_bf16(pr[0][2] - __uint_as_float(ph2 << 16), pr[0][3] - __uint_as_float(ph2 & 0xffff0000u));
            const uint32_t pl3 = pack_bf16(pr[1][2] - __uint_as_float(ph3 << 16), pr[1][3] - __uint_as_float(ph3 & 0xffff0000u));
            // ---- O += P V
#pragma unroll
            for (int j = 0; j < SH::NTILES / 2; ++j) {
                const int chunk = 2 * (j & 3) + v_hi;
                const uint32_t addr = vt + (j >> 2) * SH::HALF_BYTES + v_row * 128 + ((chunk ^ sw) << 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(addr, b0, b1, b2, b3);
                mma_bf16_16(acc[2 * j], ph0, ph1, ph2, ph3, b0, b1);
                mma_bf16_16(acc[2 * j], pl0, pl1, pl2, pl3, b0, b1);
                mma_bf16_16(acc[2 * j + 1], ph0, ph1, ph2, ph3, b2, b3);
                mma_bf16_16(acc[2 * j + 1], pl0, pl1, pl2, pl3, b2, b3);
            }
            __syncwarp();
            mbar_arrive(&s_empty[st]);
            ++it;
            if (i != ntiles - 1) continue;

            // ======== end of unit: combine warps, write the split's state of every row ========
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                l_run[rr] += __shfl_xor_sync(kFull, l_run[rr], 1);
                l_run[rr] += __shfl_xor_sync(kFull, l_run[rr], 2);
            }
#pragma unroll
            for (int j = 0; j < SH::NTILES; ++j) {
                *reinterpret_cast<float2*>(s_o + (warp * R + r0) * D + 8 * j + 2 * cq) = make_float2(acc[j][0], acc[j][1]);
                *reinterpret_cast<float2*>(s_o + (warp * R + r1) * D + 8 * j + 2 * cq) = make_float2(acc[j][2], acc[j][3]);
            }
            if (cq == 0) {
                s_ml[(warp * R + r0) * 2] = m_run[0];
                s_ml[(warp * R + r0) * 2 + 1] = l_run[0];
                s_ml[(warp * R + r1) * 2] = m_run[1];
                s_ml[(warp * R + r1) * 2 + 1] = l_run[1];
            }
            named_bar(1, NWC * 32);
            const int S = p.S;
            for (int idx = tid; idx < R * D; idx += NWC * 32) {
                const int rr = idx / D, e = idx % D;
                const int b = ublk * BQ + rr / G;
                if (b >= p.B) continue;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NWC; ++w) M = fmaxf(M, s_ml[(w * R + rr) * 2]);
                const float Mu = (M == -INFINITY) ? 0.f : M;
                float L = 0.f, O = 0.f;
#pragma unroll
                for (int w = 0; w < NWC; ++w) {
                    const float f = exp2f((s_ml[(w * R + rr) * 2] - Mu) * kLog2e);
                    L = fmaf(f, s_ml[(w * R + rr) * 2 + 1], L);
                    O = fmaf(f, s_o[(w * R + rr) * D + e], O);
                }
                const float out = (L > 0.f) ? O / L : 0.f;
                const float lse = (L > 0.f) ? M + log2f(L) * kLn2 : -INFINITY;
                const size_t row = (size_t)b * p.Hq + ug * G + rr % G;
                if (p.o_part != nullptr) {
                    p.o_part[(row * S + usplit) * D + e] = out;
                    if (e == 0) p.lse_part[row * S + usplit] = lse;
                }
                if (S == 1) {
                    if (p.o_bf16) {
                        reinterpret_cast<__nv_bfloat16*>(p.o)[row * D + e] = __float2bfloat16_rn(out);
                    } else {
                        reinterpret_cast<float*>(p.o)[row * D + e] = out;
                    }
                    if (e == 0 && p.lse != nullptr) p.lse[row] = lse;
                }
            }
            named_bar(1, NWC * 32);
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
    // a CTA that gave up leaves every unit it owns in the empty state
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
        const int blk = u / per_blk;
        const int g = (u - blk * per_blk) / p.S;
        const int split = u - blk * per_blk - g * p.S;
        for (int r = warp; r < R; r += NWC + 1) qb_empty_row<D, G>(p, blk, g, split, r, lane, 32);
    }
}

}  // namespace kvb
