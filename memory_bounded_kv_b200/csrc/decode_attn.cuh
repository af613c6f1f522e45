// Split-K GQA decode attention with the retention bias of "Cache What Lasts"
// section 2.1 (logit = scale * q.k_i + (t - i) log beta_i) and the (o, lse)
// attention state of "Context Memorization" core method step 1. The splits'
// states are combined with that page's merge operator (step 2) by the last
// CTA of each (sequence, kv head) to finish: an atomic ticket, no waiting.
//
// One CTA = one (split, kv head g, sequence b). All G query heads of the
// group are served from one read of the K/V rows. Layout of the work:
//  - K and V tiles of T slots are contiguous byte ranges of the cache
//    ([cap, d] per (b, g)); one thread streams them into a STAGES-deep ring
//    of shared-memory buffers with cp.async.bulk, completion counted on one
//    mbarrier per stage.
//  - Each warp owns KPW = 32/G keys of a tile. QK: a group of LPK = d/8
//    lanes shares one key row, each lane holding 8 dims of q for all G
//    heads in registers; the LPK partial dots of KPG keys x G heads are
//    finished with a reduce-scatter over the group (log2(LPK) shuffle
//    steps), after which each lane holds one (key, head) logit.
//  - Online softmax per warp and head (maxima in natural units, exp2 of
//    scaled differences); p goes to shared
//    memory and is read back as a broadcast for PV, where each lane
//    accumulates 8 dims x G heads of the output over its group's keys.
//  - Epilogue: warps combine through shared memory into the split's state.
#pragma once

#include "common.cuh"

namespace kvb {

struct DecodeParams {
    const uint16_t* q;
    long long q_sb, q_sh;
    const uint16_t* k;
    const uint16_t* v;
    long long kv_sb, kv_sh;
    const float* lb;
    const int* pos;
    long long m_sb, m_sh;
    const int* len;
    const int* t;
    int Hq, Hkv, cap, S, split_len;
    float qscale;  // the logit scale (1/sqrt(d) unless given)
    float* o_part;
    float* lse_part;
    unsigned* counters;
    void* o;
    int o_bf16;
    float* lse;
};

template <int D, int G>
struct DecodeShape {
    static constexpr int LPK = D / 8;          // lanes that share one key row
    static constexpr int GPW = 32 / LPK;       // lane groups per warp
    static constexpr int KPG = LPK / G;        // keys per lane group per tile
    static constexpr int KPW = GPW * KPG;      // keys per warp per tile (= 32 / G)
    static constexpr int NW = (G >= 4) ? 8 : 2 * G;
    static constexpr int NT = NW * 32;
    static constexpr int T = NW * KPW;         // keys per tile
    static constexpr int STAGES = 3;
    static constexpr int TILE_ELEMS = T * D;
    static constexpr int STAGE_BYTES = 2 * TILE_ELEMS * 2;  // K and V tile, bf16
    static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
    static constexpr int EPI_BYTES = NW * G * (D + 2) * 4;  // epilogue reuses the ring
    // fixed area in front of the ring: mbarriers at 0, flag at 64, bias [2][T] at 128,
    // p [NW][32] after it (16-byte aligned: it is read back as float2/float4)
    static constexpr int BIAS_OFF = 128;
    static constexpr int P_OFF = BIAS_OFF + 2 * T * 4;
    static constexpr int FIXED_BYTES = ((P_OFF + NW * 32 * 4) + 127) / 128 * 128;
    static_assert(STAGES * 8 <= 64 && P_OFF % 16 == 0, "fixed-area layout");
    static_assert(LPK % G == 0, "G must divide d/8");
    static_assert(EPI_BYTES <= RING_BYTES, "epilogue must fit in the ring");
    // dynamic shared memory for S splits: the merge of S states needs G*(S+2) floats
    static size_t smem_bytes(int S) {
        const size_t merge = (size_t)G * (S + 2) * 4;
        return FIXED_BYTES + (merge > (size_t)RING_BYTES ? merge : (size_t)RING_BYTES);
    }
};

// Reduce-scatter of N partial sums across the N lanes of a group (xor masks
// N/2 .. 1): afterwards lane `sub` holds the full sum of value index `sub`.
template <int N>
__device__ __forceinline__ float reduce_scatter(float (&v)[N], int sub) {
#pragma unroll
    for (int m = N / 2; m >= 1; m /= 2) {
        const bool upper = (sub & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = upper ? v[i] : v[i + m];
            const float keep = upper ? v[i + m] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, m);
        }
    }
    return v[0];
}

template <int G>
__device__ __forceinline__ void load_p(const float* src, float (&pk)[G]) {
    if constexpr (G == 1) {
        pk[0] = src[0];
    } else if constexpr (G == 2) {
        const float2 a = *reinterpret_cast<const float2*>(src);
        pk[0] = a.x; pk[1] = a.y;
    } else {
#pragma unroll
        for (int i = 0; i < G; i += 4) {
            const float4 a = *reinterpret_cast<const float4*>(src + i);
            pk[i] = a.x; pk[i + 1] = a.y; pk[i + 2] = a.z; pk[i + 3] = a.w;
        }
    }
}

template <int D, int G, bool BIAS>
__global__ void __launch_bounds__(DecodeShape<D, G>::NT)
    decode_attn_kernel(const __grid_constant__ DecodeParams p) {
    using SH = DecodeShape<D, G>;
    constexpr int LPK = SH::LPK, KPG = SH::KPG, KPW = SH::KPW, NW = SH::NW, NT = SH::NT;
    constexpr int T = SH::T, ST = SH::STAGES;

    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint64_t* s_bar = reinterpret_cast<uint64_t*>(smem_raw);                 // [ST]
    int* s_flag = reinterpret_cast<int*>(smem_raw + 64);
    float* s_bias = reinterpret_cast<float*>(smem_raw + SH::BIAS_OFF);      // [2][T]
    float* s_p = reinterpret_cast<float*>(smem_raw + SH::P_OFF);            // [NW][32]
    unsigned char* smem = smem_raw + SH::FIXED_BYTES;                        // ring / epilogue / merge
    uint16_t* s_ring = reinterpret_cast<uint16_t*>(smem);

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gi = lane / LPK, sub = lane % LPK;
    const int bg = b * p.Hkv + g;
    const int S = p.S;

    // ---- this split's slot range ---------------------------------------
    int n = p.len[bg];
    const bool active = (p.t == nullptr) || (p.t[b] >= 0);
    const int tb = (p.t == nullptr) ? 0 : p.t[b];
    const bool bad_len = n < 0 || n > p.cap;
    const bool bad_split = !bad_len && p.split_len > 0 && (long long)n > (long long)S * p.split_len;
    if ((bad_len || bad_split) && split == 0 && tid == 0)
        raise_error(bad_len ? KVB_DERR_LEN : KVB_DERR_SPLIT);
    if (bad_len || bad_split || !active) n = 0;
    const long long C = p.split_len > 0 ? (long long)p.split_len : (long long)((n + S - 1) / S);
    const int s0 = (int)min((long long)split * C, (long long)n);
    const int s1 = (int)min((long long)s0 + C, (long long)n);
    const int nk = s1 - s0;
    const int ntiles = (nk + T - 1) / T;

    const size_t kv_off = (size_t)b * p.kv_sb + (size_t)g * p.kv_sh + (size_t)s0 * D;
    const uint16_t* gk = p.k + kv_off;
    const uint16_t* gv = p.v + kv_off;
    const size_t m_off = (size_t)b * p.m_sb + (size_t)g * p.m_sh + (size_t)s0;
    const float* glb = BIAS ? p.lb + m_off : nullptr;
    const int* gpos = BIAS ? p.pos + m_off : nullptr;

    auto bias_of = [&](int key) -> float {  // (t - pos) * log beta, -inf beyond the split
        if (key >= nk) return -INFINITY;
        if constexpr (BIAS) {
            return __fmul_rn(__int2float_rn(tb - gpos[key]), glb[key]);
        } else {
            return 0.f;
        }
    };

    auto issue = [&](int i) {
        const int st = i % ST;
        const int rows = min(T, nk - i * T);
        const unsigned bytes = (unsigned)rows * D * 2u;
        uint16_t* dk = s_ring + st * 2 * SH::TILE_ELEMS;
        mbar_arrive_expect_tx(&s_bar[st], 2u * bytes);
        bulk_g2s(dk, gk + (size_t)i * T * D, bytes, &s_bar[st]);
        bulk_g2s(dk + SH::TILE_ELEMS, gv + (size_t)i * T * D, bytes, &s_bar[st]);
    };

    if (tid == 0) {
#pragma unroll
        for (int st = 0; st < ST; ++st) mbar_init(&s_bar[st], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < min(ST, ntiles); ++i) issue(i);
    }

    // q for my 8 dims, all G heads, pre-multiplied by the logit scale
    float qf[G][8];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        const uint4 raw = *reinterpret_cast<const uint4*>(p.q + (size_t)b * p.q_sb +
                                                          (size_t)(g * G + hh) * p.q_sh + sub * 8);
        unpack8(raw, qf[hh]);
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[hh][e] *= p.qscale;
    }

    float acc[G][8];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
    float m_run = -INFINITY;  // running max of head (lane % G), same in all its lanes
    float l_run = 0.f;        // this lane's share of the partition sum of that head

    if (tid < T && ntiles > 0) s_bias[tid] = bias_of(tid);
    __syncthreads();

    float* s_pw = s_p + warp * 32;
    const int kbase = warp * KPW + gi * KPG;  // my group's first key in a tile
    bool timed_out = false;

#pragma unroll 1
    for (int i = 0; i < ntiles; ++i) {
        const int st = i % ST;
        const unsigned parity = (unsigned)(i / ST) & 1u;
        const int rows = min(T, nk - i * T);
        const bool has_next = i + 1 < ntiles;
        float next_bias = 0.f;
        if (tid < T && has_next) next_bias = bias_of((i + 1) * T + tid);

        const bool ok = mbar_wait(&s_bar[st], parity);
        uint16_t* sK = s_ring + st * 2 * SH::TILE_ELEMS;
        uint16_t* sV = sK + SH::TILE_ELEMS;
        if (rows < T) {  // tail tile: zero the rows the copy did not fill
            for (int idx = tid; idx < (T - rows) * D / 8; idx += NT) {
                reinterpret_cast<uint4*>(sK + rows * D)[idx] = make_uint4(0, 0, 0, 0);
                reinterpret_cast<uint4*>(sV + rows * D)[idx] = make_uint4(0, 0, 0, 0);
            }
            __syncthreads();
        }
        const float* sb = s_bias + (i & 1) * T;

        // ---- QK: partial dots of my 8 dims for KPG keys x G heads
        float part[LPK];
#pragma unroll
        for (int kk = 0; kk < KPG; ++kk) {
            const uint4 raw = *reinterpret_cast<const uint4*>(sK + (kbase + kk) * D + sub * 8);
            float kf[8];
            unpack8(raw, kf);
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                float a = qf[hh][0] * kf[0];
#pragma unroll
                for (int e = 1; e < 8; ++e) a = fmaf(qf[hh][e], kf[e], a);
                part[kk * G + hh] = a;
            }
        }
        float x = reduce_scatter<LPK>(part, sub) + sb[kbase + sub / G];

        // ---- online softmax, head = lane % G
        float tmax = x;
#pragma unroll
        for (int m = G; m < 32; m <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, m));
        const float m_new = fmaxf(m_run, tmax);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        // logits and maxima stay in natural units; only differences are scaled by log2(e)
        const float alpha = exp2f((m_run - m_use) * kLog2e);
        const float pv = exp2f((x - m_use) * kLog2e);
        l_run = fmaf(l_run, alpha, pv);
        m_run = m_new;
        if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                const float a = __shfl_sync(kFull, alpha, hh);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[hh][e] *= a;
            }
        }
        s_pw[lane] = pv;
        __syncwarp();

        // ---- PV: my 8 dims x G heads over my group's keys
#pragma unroll
        for (int kk = 0; kk < KPG; ++kk) {
            float pk[G];
            load_p<G>(s_pw + gi * LPK + kk * G, pk);
            const uint4 raw = *reinterpret_cast<const uint4*>(sV + (kbase + kk) * D + sub * 8);
            float vf[8];
            unpack8(raw, vf);
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[hh][e] = fmaf(pk[hh], vf[e], acc[hh][e]);
        }

        if (tid < T && has_next) s_bias[((i + 1) & 1) * T + tid] = next_bias;
        if (__syncthreads_or(!ok)) {
            // a copy did not arrive in time: record it, drain what is in flight, stop
            if (tid == 0) raise_error(KVB_DERR_TIMEOUT);
            for (int j = i + 1; j < min(i + ST, ntiles); ++j) mbar_wait(&s_bar[j % ST], (unsigned)(j / ST) & 1u);
            timed_out = true;
            break;
        }
        if (tid == 0 && i + ST < ntiles) issue(i + ST);
    }
    (void)timed_out;

    // ---- combine lanes: l over lanes of a head, acc over lane groups
#pragma unroll
    for (int m = G; m < 32; m <<= 1) l_run += __shfl_xor_sync(kFull, l_run, m);
#pragma unroll
    for (int m = LPK; m < 32; m <<= 1)
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[hh][e] += __shfl_xor_sync(kFull, acc[hh][e], m);

    // ---- combine warps through shared memory (the ring is free now)
    __syncthreads();
    float* s_o = reinterpret_cast<float*>(smem);  // [NW][G][D]
    float* s_ml = s_o + NW * G * D;               // [NW][G][2]
    if (gi == 0) {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            float4* dst = reinterpret_cast<float4*>(s_o + (warp * G + hh) * D + sub * 8);
            dst[0] = make_float4(acc[hh][0], acc[hh][1], acc[hh][2], acc[hh][3]);
            dst[1] = make_float4(acc[hh][4], acc[hh][5], acc[hh][6], acc[hh][7]);
        }
    }
    if (lane < G) {
        s_ml[(warp * G + lane) * 2] = m_run;
        s_ml[(warp * G + lane) * 2 + 1] = l_run;
    }
    __syncthreads();

    const bool final_direct = (S == 1);
    for (int idx = tid; idx < G * D; idx += NT) {
        const int hh = idx / D, e = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, s_ml[(w * G + hh) * 2]);
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float f = exp2f((s_ml[(w * G + hh) * 2] - Mu) * kLog2e);
            L = fmaf(f, s_ml[(w * G + hh) * 2 + 1], L);
            O = fmaf(f, s_o[(w * G + hh) * D + e], O);
        }
        const float out = (L > 0.f) ? O / L : 0.f;
        const float lse = (L > 0.f) ? M + log2f(L) * kLn2 : -INFINITY;
        const int h = g * G + hh;
        const size_t row = (size_t)b * p.Hq + h;
        if (p.o_part != nullptr) {
            p.o_part[(row * S + split) * D + e] = out;
            if (e == 0) p.lse_part[row * S + split] = lse;
        }
        if (final_direct) {
            if (p.o_bf16) {
                reinterpret_cast<__nv_bfloat16*>(p.o)[row * D + e] = __float2bfloat16_rn(out);
            } else {
                reinterpret_cast<float*>(p.o)[row * D + e] = out;
            }
            if (e == 0 && p.lse != nullptr) p.lse[row] = lse;
        }
    }
    if (final_direct) return;

    // ---- last split to finish merges all S states of this (b, g)
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(&p.counters[bg], 1u);
        *s_flag = (prev == (unsigned)(S - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (*s_flag == 0) return;
    __threadfence();

    // splits past the last non-empty one hold (0, -inf) and are skipped
    const int nz = (C > 0) ? (int)min((long long)S, ((long long)n + C - 1) / C) : 0;
    float* s_w = reinterpret_cast<float*>(smem);  // [G][S]: lse of each split, then its weight
    float* s_hl = s_w + G * S;                    // [G][2]: lse, 1/L
    if (warp < G) {
        const size_t row = (size_t)b * p.Hq + g * G + warp;
        float mx = -INFINITY;
        for (int j = lane; j < nz; j += 32) {
            const float lj = __ldcg(p.lse_part + row * S + j);
            s_w[warp * S + j] = lj;
            mx = fmaxf(mx, lj);
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
        const float mu = (mx == -INFINITY) ? 0.f : mx;
        float sum = 0.f;
        for (int j = lane; j < nz; j += 32) {
            const float w = exp2f((s_w[warp * S + j] - mu) * kLog2e);
            s_w[warp * S + j] = w;
            sum += w;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) sum += __shfl_xor_sync(kFull, sum, m);
        if (lane == 0) {
            s_hl[warp * 2] = (sum > 0.f) ? mx + log2f(sum) * kLn2 : -INFINITY;
            s_hl[warp * 2 + 1] = (sum > 0.f) ? 1.f / sum : 0.f;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += NT) {
        const int hh = idx / D, e = idx % D;
        const size_t row = (size_t)b * p.Hq + g * G + hh;
        float O = 0.f;
        for (int j = 0; j < nz; ++j) O = fmaf(s_w[hh * S + j], __ldcg(p.o_part + (row * S + j) * D + e), O);
        O *= s_hl[hh * 2 + 1];
        if (p.o_bf16) {
            reinterpret_cast<__nv_bfloat16*>(p.o)[row * D + e] = __float2bfloat16_rn(O);
        } else {
            reinterpret_cast<float*>(p.o)[row * D + e] = O;
        }
        if (e == 0 && p.lse != nullptr) p.lse[row] = s_hl[hh * 2];
    }
    if (tid == 0) p.counters[bg] = 0u;
}

}  // namespace kvb
