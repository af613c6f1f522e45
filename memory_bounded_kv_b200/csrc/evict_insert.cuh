// Budget enforcement of "Cache What Lasts" section 2.1 (inference): when the
// cache holds M tokens, the one with the lowest beta_i^(t-i) is evicted and
// the new token takes its slot. "Lowest beta^(t-i)" is computed as the
// lowest score (t - pos) * log beta, one float32 multiply rounded to nearest
// even, ties to the lower position (-0 == +0), which is bit-reproducible.
//
// One CTA per (sequence, kv head). Each thread scans a strided share of the
// slots keeping the best 64-bit key (order key of the score << 32 | order
// key of the position) with its slot; a warp-shuffle argmin and a shared-
// memory pass across warps give the victim; then the CTA writes the new row.
// When the preceding attention left per-split candidates (the same key for
// position t, computed while it read every slot), the victim is the best of
// those few records instead: the same argmin, since the splits partition
// the slots. The records carry the position they were scored for; a set in
// which any record was scored for another position is ignored (full scan).
#pragma once

#include "common.cuh"

namespace kvb {

struct EvictParams {
    uint16_t* k;
    uint16_t* v;
    float* lb;
    int* pos;
    int* len;
    const uint16_t* k_new;
    const uint16_t* v_new;
    const float* lb_new;
    const int* t;
    int Hkv, d, cap, M;
    int* victim;
    int vec4;  // pos/log_beta rows start 16-byte aligned (cap % 4 == 0, aligned bases)
    const EvictCand* cand;  // nullable: per-split candidates from the preceding attention
    int cand_n;
};

template <int NT>
__global__ void __launch_bounds__(NT) evict_insert_kernel(const __grid_constant__ EvictParams p) {
    __shared__ unsigned long long s_key[NT / 32];
    __shared__ int s_slot[NT / 32];
    __shared__ int s_cand;
    griddep_wait();  // the previous kernel in the stream (e.g. the last attention) has finished
    griddep_launch_dependents();
    const int bg = blockIdx.x, b = bg / p.Hkv, tid = threadIdx.x;
    // every load that does not depend on another is issued here, before any of them is used:
    // position, length, this thread's candidate record and its 16 bytes of the new row
    const int tb = p.t[b];
    const int n = p.len[bg];
    EvictCand my_cand{~0ull, -1, 0};
    if (p.cand != nullptr && tid < 32 && tid < p.cand_n) my_cand = p.cand[(size_t)bg * p.cand_n + tid];
    const int vecs = p.d / 8;
    uint4 row_part = make_uint4(0u, 0u, 0u, 0u);
    if (p.k_new != nullptr && tid < 2 * vecs)
        row_part = (tid < vecs) ? reinterpret_cast<const uint4*>(p.k_new + (size_t)bg * p.d)[tid]
                                : reinterpret_cast<const uint4*>(p.v_new + (size_t)bg * p.d)[tid - vecs];
    if (tb < 0) {
        if (tid == 0 && p.victim) p.victim[bg] = -1;
        return;
    }
    if (n < 0 || n > p.cap) {
        if (tid == 0) {
            raise_error(KVB_DERR_LEN);
            if (p.victim) p.victim[bg] = -1;
        }
        return;
    }
    int slot = -1;
    if (n >= p.M && p.cand != nullptr) {
        // the attention of the previous position already reduced every split's slots
        if (tid < 32) {
            unsigned long long best = ~0ull;
            int best_slot = 0x7fffffff;
            bool stale = tid < p.cand_n && my_cand.t != tb;
            if (my_cand.slot >= 0) argmin_merge(best, best_slot, my_cand.key, my_cand.slot);
            for (int j = tid + 32; j < p.cand_n; j += 32) {   // records past the first 32
                const EvictCand c = p.cand[(size_t)bg * p.cand_n + j];
                stale = stale || c.t != tb;
                if (c.slot >= 0) argmin_merge(best, best_slot, c.key, c.slot);
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
                const unsigned long long k2 = __shfl_xor_sync(kFull, best, m);
                const int s2 = __shfl_xor_sync(kFull, best_slot, m);
                argmin_merge(best, best_slot, k2, s2);
            }
            // records scored for another position rank the slots differently: scan instead
            stale = __any_sync(kFull, stale);
            if (tid == 0) s_cand = (!stale && best != ~0ull && best_slot < n) ? best_slot : -1;
        }
        __syncthreads();
        slot = s_cand;
    }
    if (n < p.M) {
        slot = n;
    } else if (slot < 0) {  // no usable candidates: scan every slot
        const size_t base = (size_t)bg * p.cap;
        const int* ps = p.pos + base;
        const float* lb = p.lb ? p.lb + base : nullptr;
        unsigned long long best = ~0ull;
        int best_slot = 0x7fffffff;
        auto consider = [&](int s, int ps_s, float l) {
            const float sc = lb ? __fmul_rn(__int2float_rn(tb - ps_s), l) : 0.f;
            const unsigned long long key =
                ((unsigned long long)float_order_key(sc) << 32) | (unsigned)(ps_s ^ 0x80000000);
            argmin_merge(best, best_slot, key, s);
        };
        int s_done = 0;
        if (p.vec4) {  // 16-byte loads: four slots per load, all issued before the compares
            const int n4 = n / 4;
            constexpr int U = 4;
            for (int base = 0; base < n4; base += U * NT) {
                int4 pv[U];
                float4 lv[U];
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int v = base + k * NT + tid;
                    if (v < n4) {
                        pv[k] = reinterpret_cast<const int4*>(ps)[v];
                        lv[k] = lb ? reinterpret_cast<const float4*>(lb)[v] : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
#pragma unroll
                for (int k = 0; k < U; ++k) {
                    const int v = base + k * NT + tid;
                    if (v < n4) {
                        consider(4 * v, pv[k].x, lv[k].x);
                        consider(4 * v + 1, pv[k].y, lv[k].y);
                        consider(4 * v + 2, pv[k].z, lv[k].z);
                        consider(4 * v + 3, pv[k].w, lv[k].w);
                    }
                }
            }
            s_done = n4 * 4;
        }
        for (int s = s_done + tid; s < n; s += NT) consider(s, ps[s], lb ? lb[s] : 0.f);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            const unsigned long long k2 = __shfl_xor_sync(kFull, best, m);
            const int s2 = __shfl_xor_sync(kFull, best_slot, m);
            argmin_merge(best, best_slot, k2, s2);
        }
        if ((tid & 31) == 0) {
            s_key[tid >> 5] = best;
            s_slot[tid >> 5] = best_slot;
        }
        __syncthreads();
        if (tid < 32) {
            best = (tid < NT / 32) ? s_key[tid] : ~0ull;
            best_slot = (tid < NT / 32) ? s_slot[tid] : 0x7fffffff;
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
                const unsigned long long k2 = __shfl_xor_sync(kFull, best, m);
                const int s2 = __shfl_xor_sync(kFull, best_slot, m);
                argmin_merge(best, best_slot, k2, s2);
            }
            if (tid == 0) s_slot[0] = best_slot;
        }
        __syncthreads();
        slot = s_slot[0];
    }
    const size_t row = (size_t)bg * p.cap + slot;
    if (p.k_new != nullptr) {
        if (tid < 2 * vecs) {
            if (tid < vecs) {
                reinterpret_cast<uint4*>(p.k + row * p.d)[tid] = row_part;
            } else {
                reinterpret_cast<uint4*>(p.v + row * p.d)[tid - vecs] = row_part;
            }
        }
        for (int i = tid + NT; i < 2 * vecs; i += NT) {   // rows wider than the block
            if (i < vecs) {
                reinterpret_cast<uint4*>(p.k + row * p.d)[i] =
                    reinterpret_cast<const uint4*>(p.k_new + (size_t)bg * p.d)[i];
            } else {
                reinterpret_cast<uint4*>(p.v + row * p.d)[i - vecs] =
                    reinterpret_cast<const uint4*>(p.v_new + (size_t)bg * p.d)[i - vecs];
            }
        }
    }
    if (tid == 0) {
        if (p.lb != nullptr) p.lb[row] = p.lb_new[bg];
        p.pos[row] = tb;
        if (n < p.M) p.len[bg] = n + 1;
        if (p.victim) p.victim[bg] = (n < p.M) ? -1 : slot;
    }
}

}  // namespace kvb
