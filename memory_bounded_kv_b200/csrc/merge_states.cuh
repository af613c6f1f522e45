// n-way merge of attention states, the operator of "Context Memorization"
// core method step 2, merge((a_A, Z_A), (a_B, Z_B)) = ((Z_A a_A + Z_B a_B) /
// (Z_A + Z_B), Z_A + Z_B), with Z carried as lse = ln Z. One warp per row:
// the lanes first reduce max and sum of the n lse values, then each lane
// accumulates its share of the d output elements.
#pragma once

#include "common.cuh"

namespace kvb {

struct MergeParams {
    const float* o_in;
    const float* lse_in;
    long long o_sn, o_sr, l_sn, l_sr;
    int n, R, d;
    float* o_out;
    float* lse_out;
};

template <bool VEC4>
__global__ void __launch_bounds__(256) merge_states_kernel(const __grid_constant__ MergeParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + warp;
    if (r >= p.R) return;
    float mx = -INFINITY;
    for (int j = lane; j < p.n; j += 32) mx = fmaxf(mx, p.lse_in[j * p.l_sn + r * p.l_sr]);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    const float mu = (mx == -INFINITY) ? 0.f : mx;
    float sum = 0.f;
    for (int j = lane; j < p.n; j += 32) sum += exp2f((p.lse_in[j * p.l_sn + r * p.l_sr] - mu) * kLog2e);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) sum += __shfl_xor_sync(kFull, sum, m);
    // weight of state j: exp(lse_j - lse) = exp(lse_j - mu) / sum; maxima stay in natural units
    const float inv = (sum > 0.f) ? 1.f / sum : 0.f;
    if (lane == 0 && p.lse_out != nullptr) p.lse_out[r] = (sum > 0.f) ? mx + log2f(sum) * kLn2 : -INFINITY;
    float* out = p.o_out + (size_t)r * p.d;
    if constexpr (VEC4) {
        for (int e = lane * 4; e < p.d; e += 128) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < p.n; ++j) {
                const float w = exp2f((p.lse_in[j * p.l_sn + r * p.l_sr] - mu) * kLog2e);
                if (w == 0.f) continue;  // an empty state: its o is not read
                const float4 x = *reinterpret_cast<const float4*>(p.o_in + j * p.o_sn + r * p.o_sr + e);
                a.x = fmaf(w, x.x, a.x); a.y = fmaf(w, x.y, a.y);
                a.z = fmaf(w, x.z, a.z); a.w = fmaf(w, x.w, a.w);
            }
            *reinterpret_cast<float4*>(out + e) = make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
        }
    } else {
        for (int e = lane; e < p.d; e += 32) {
            float a = 0.f;
            for (int j = 0; j < p.n; ++j) {
                const float w = exp2f((p.lse_in[j * p.l_sn + r * p.l_sr] - mu) * kLog2e);
                if (w != 0.f) a = fmaf(w, p.o_in[j * p.o_sn + r * p.o_sr + e], a);
            }
            out[e] = a * inv;
        }
    }
}

}  // namespace kvb
