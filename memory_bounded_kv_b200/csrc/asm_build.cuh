// Attention-state-memory offline build, "Context Memorization" core method
// step 2 (attention-aware aggregation): per table t and cluster k, over the
// calibration rows (i, h) of the table's heads (h / G == t) assigned to k,
//   qbar[t, k]     = mean of q[i, h]
//   (abar, Zbar)   = merge-fold of (a[i, h], Z[i, h]): Zbar = sum Z_i (the page's merge
//                    operator sums Z; z_mean divides by the member count),
//                    abar = sum Z_i a_i / Zbar, computed in the log domain:
//                    m = max ln Z_i, w_i = exp(ln Z_i - m), ln Zbar = m + ln sum w_i.
// Three passes over the rows (one warp per (i, h), lane l holding elements
// 4l..4l+3): counts, the running max of ln Z and the query sums; the weighted
// state sums; then one warp per (h, k) finalises. The sums are fp32 atomics
// (vector adds of 4), so their rounding order varies between runs.
#pragma once

#include "common.cuh"

namespace kvb {

constexpr int kBuildD = 128;

struct AsmBuildParams {
    const uint16_t* q;      // [M, H, d] bf16
    const float* a;         // [M, H, d] or null
    const float* lse;       // [M, H] or null
    const int32_t* idx;     // [M, H]: cluster, < 0 = none
    int M, H, K, z_mean;
    float* qbar;            // [H, K, d]
    uint16_t* abar;         // [H, K, d] bf16 (null when a is null)
    float* log_zbar;        // [H, K] (null when a is null)
    int32_t* count;         // [H, K] or null
    // workspace
    unsigned* cmax;         // [H, K] order key of the max ln Z (0: none)
    int* cnt;               // [H, K]
    float* wsum;            // [H, K]
    float* qsum;            // [H, K, d]
    float* asum;            // [H, K, d]
    int G;                  // query heads per table: row (i, h) goes to table h / G
};

__device__ __forceinline__ float float_from_order_key(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

__global__ void __launch_bounds__(256) asm_build_zero_kernel(unsigned* ws, size_t words) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < words; i += (size_t)gridDim.x * blockDim.x)
        ws[i] = 0u;
}

// pass 1: counts, max ln Z, query sums
__global__ void __launch_bounds__(256) asm_build_pass1_kernel(const __grid_constant__ AsmBuildParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * 8 + warp;   // i * H + h
    if (r >= (long long)p.M * p.H) return;
    const int h = (int)(r % p.H), k = p.idx[r];
    if (k < 0) return;
    if (k >= p.K) {
        if (lane == 0) raise_error(KVB_DERR_RANGE);
        return;
    }
    const size_t hk = (size_t)(h / p.G) * p.K + k;
    if (lane == 0) {
        atomicAdd(p.cnt + hk, 1);
        if (p.lse != nullptr) atomicMax(p.cmax + hk, float_order_key(p.lse[r]));
    }
    const uint2 w = *reinterpret_cast<const uint2*>(p.q + r * kBuildD + lane * 4);
    atomicAdd(reinterpret_cast<float4*>(p.qsum + hk * kBuildD + lane * 4),
              make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y)));
}

// pass 2: w_i = exp(ln Z_i - max), sum w_i and sum w_i a_i
__global__ void __launch_bounds__(256) asm_build_pass2_kernel(const __grid_constant__ AsmBuildParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * 8 + warp;
    if (r >= (long long)p.M * p.H) return;
    const int h = (int)(r % p.H), k = p.idx[r];
    if (k < 0 || k >= p.K) return;
    const size_t hk = (size_t)(h / p.G) * p.K + k;
    const float m = float_from_order_key(p.cmax[hk]);
    const float l = p.lse[r];
    if (l == -INFINITY || m == -INFINITY) return;   // Z_i = 0 contributes nothing
    const float wt = exp2f((l - m) * kLog2e);
    if (lane == 0) atomicAdd(p.wsum + hk, wt);
    const float4 x = *reinterpret_cast<const float4*>(p.a + r * kBuildD + lane * 4);
    atomicAdd(reinterpret_cast<float4*>(p.asum + hk * kBuildD + lane * 4),
              make_float4(wt * x.x, wt * x.y, wt * x.z, wt * x.w));
}

// finalise: one warp per (h, k)
__global__ void __launch_bounds__(256) asm_build_final_kernel(const __grid_constant__ AsmBuildParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long hk = (long long)blockIdx.x * 8 + warp;   // table * K + cluster
    if (hk >= (long long)(p.H / p.G) * p.K) return;
    const int n = p.cnt[hk];
    if (lane == 0 && p.count != nullptr) p.count[hk] = n;
    float4 qm = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n > 0) {
        const float4 s = *reinterpret_cast<const float4*>(p.qsum + hk * kBuildD + lane * 4);
        const float inv = 1.f / (float)n;
        qm = make_float4(s.x * inv, s.y * inv, s.z * inv, s.w * inv);
    }
    *reinterpret_cast<float4*>(p.qbar + hk * kBuildD + lane * 4) = qm;
    if (p.a == nullptr) return;
    const float ws = p.wsum[hk];
    uint2 ab = make_uint2(0u, 0u);
    float lz = -INFINITY;
    if (n > 0 && ws > 0.f) {
        const float4 s = *reinterpret_cast<const float4*>(p.asum + hk * kBuildD + lane * 4);
        const float inv = 1.f / ws;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(s.x * inv, s.y * inv);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(s.z * inv, s.w * inv);
        ab = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
        lz = float_from_order_key(p.cmax[hk]) + log2f(ws) * kLn2;
        if (p.z_mean) lz -= log2f((float)n) * kLn2;
    }
    *reinterpret_cast<uint2*>(p.abar + hk * kBuildD + lane * 4) = ab;
    if (lane == 0) p.log_zbar[hk] = lz;
}

// ---- two-level index of a memory -----------------------------------------------------------
// The entries are clustered like calibration queries (the lookup's cosine argmax + the mean
// update), so they are first laid out as bf16 queries: qbar [H, K, d] f32 -> q [K, H, d] bf16
// (round to nearest even); one thread per 4 elements.
__global__ void __launch_bounds__(256) asm_entries_bf16_kernel(const float* __restrict__ qbar, int H, int K,
                                                               uint16_t* __restrict__ q) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // (h, k, 4-element group)
    const long long total = (long long)H * K * (kBuildD / 4);
    if (i >= total) return;
    const int e4 = (int)(i % (kBuildD / 4));
    const long long hk = i / (kBuildD / 4);
    const int h = (int)(hk / K), k = (int)(hk % K);
    const float4 x = *reinterpret_cast<const float4*>(qbar + hk * kBuildD + e4 * 4);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(x.x, x.y), hi = __floats2bfloat162_rn(x.z, x.w);
    *reinterpret_cast<uint2*>(q + ((size_t)k * H + h) * kBuildD + e4 * 4) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}

// Cluster lists from an assignment idx [K, H] (entry k of head h in cluster idx[k, h]; values
// outside [0, C) are listed nowhere): counts, then offsets, then members in increasing entry
// order, deterministic (warp ballots in entry order, no atomics).
struct AsmCsrParams {
    const int32_t* idx;   // [K, H]
    int K, H, C;
    int32_t* offsets;     // [H, C + 1]
    int32_t* members;     // [H, K]
    int32_t* counts;      // [H, C] workspace
};

// one warp per (h, c): pass 0 counts the members, pass 1 writes them from offsets[h, c] on
template <int PASS>
__global__ void __launch_bounds__(256) asm_csr_kernel(const __grid_constant__ AsmCsrParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long hc = (long long)blockIdx.x * 8 + warp;
    if (hc >= (long long)p.H * p.C) return;
    const int h = (int)(hc / p.C), c = (int)(hc % p.C);
    int pos = (PASS == 0) ? 0 : p.offsets[(size_t)h * (p.C + 1) + c];
    for (int k0 = 0; k0 < p.K; k0 += 32) {
        const int k = k0 + lane;
        const bool in = k < p.K && p.idx[(size_t)k * p.H + h] == c;
        const unsigned mask = __ballot_sync(kFull, in);
        if (PASS == 1 && in) p.members[(size_t)h * p.K + pos + __popc(mask & ((1u << lane) - 1u))] = k;
        pos += __popc(mask);
    }
    if (PASS == 0 && lane == 0) p.counts[hc] = pos;
}

// one warp per head: offsets[h, 0] = 0, offsets[h, c + 1] = offsets[h, c] + counts[h, c]
__global__ void __launch_bounds__(32) asm_csr_scan_kernel(const __grid_constant__ AsmCsrParams p) {
    const int h = blockIdx.x, lane = threadIdx.x;
    const int32_t* cnt = p.counts + (size_t)h * p.C;
    int32_t* off = p.offsets + (size_t)h * (p.C + 1);
    if (lane == 0) off[0] = 0;
    int carry = 0;
    for (int c0 = 0; c0 < p.C; c0 += 32) {
        const int c = c0 + lane;
        int v = (c < p.C) ? cnt[c] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {   // inclusive warp scan
            const int u = __shfl_up_sync(kFull, v, o);
            if (lane >= o) v += u;
        }
        if (c < p.C) off[c + 1] = carry + v;
        carry += __shfl_sync(kFull, v, 31);
    }
}

}  // namespace kvb
