// Attention-state-memory offline build, "Context Memorization" core method
// step 2 (attention-aware aggregation): per head h and cluster k, over the
// calibration queries i assigned to k,
//   qbar[h, k]     = mean of q[i, h]
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
    const size_t hk = (size_t)h * p.K + k;
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
    const size_t hk = (size_t)h * p.K + k;
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
    const long long hk = (long long)blockIdx.x * 8 + warp;
    if (hk >= (long long)p.H * p.K) return;
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

}  // namespace kvb
