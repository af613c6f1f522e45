// Two-level attention-state-memory lookup, "Context Memorization" hierarchical
// lookup index: the query is scored against the C first-level centroids of its
// head, the m best clusters are kept, and the exact argmax runs over their
// members only; the merge is the linear lookup's (asm_merge_kernel).
//
// Nothing is reused across queries here (each (query, head) reads its own
// candidate rows), so these are gather kernels bound by memory traffic, not
// contractions: per (query, head), C + sum of the selected clusters' sizes rows
// of 512 bytes. The win over the linear lookup is at few queries per step.
//
//   asm_hier_select_kernel  one CTA per (n, h): C first-level scores, then m
//                           rounds of a warp argmax over packed (score, -c)
//                           keys -> sel [N, H, m]
//   asm_hier_score_kernel   one CTA per (selected cluster j, n, h): the
//                           members' scores, best (score, -k) key -> keys [m, N, H]
// Rows are read by whole warps (one coalesced 512-byte access per row, 8 rows
// in flight per warp): with one or a few query tokens per call the lookup is
// bound by the latency of these dependent reads, not by their bytes.
//
// Scores are q . x / |x| in fp32 (|q| is common to all candidates); -0 is folded
// into +0 so that equal scores compare equal as keys.
#pragma once

#include "common.cuh"

namespace kvb {

constexpr int kHierD = 128, kHierMaxC = 1024, kHierMaxM = 64;

struct AsmHierParams {
    const uint16_t* q;
    const float* qhat;
    const int32_t* offsets;
    const int32_t* members;
    const float* qbar;
    int N, H, K, C, m;
    int32_t* sel;               // [N][H][m]
    unsigned long long* keys;   // [m][N][H]
};

// bytes of shared memory of the select kernel: C scores, then C taken flags
__host__ __device__ inline size_t hier_select_smem(int C) { return (size_t)C * sizeof(float) + (size_t)C; }

// q[nh] (bf16, 128): lane l holds dims 4l..4l+3
__device__ __forceinline__ float4 hier_q4(const uint16_t* q, long long nh, int lane) {
    const uint2 w = *reinterpret_cast<const uint2*>(q + nh * kHierD + lane * 4);
    return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Scores q . x / |x| of up to 8 fp32 rows of 128 (0 for a zero row), the warp reading each
// row as one coalesced 512-byte access (lane l: elements 4l..4l+3), the 8 rows in flight at
// once. rows[r] == nullptr: no row (score unused). Every lane returns all 8 scores.
__device__ __forceinline__ void hier_score8(const float4 qv, const float* const (&rows)[8], float (&score)[8],
                                            int lane) {
    float dot[8], ss[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const float4 x = rows[r] ? __ldg(reinterpret_cast<const float4*>(rows[r]) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        dot[r] = fmaf(qv.x, x.x, fmaf(qv.y, x.y, fmaf(qv.z, x.z, qv.w * x.w)));
        ss[r] = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, x.w * x.w)));
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const float d = warp_sum(dot[r]), n = warp_sum(ss[r]);
        score[r] = (n > 0.f) ? d * (1.f / sqrtf(n)) : 0.f;
    }
}

__device__ __forceinline__ unsigned long long hier_key(float score, int id) {
    return ((unsigned long long)float_order_key(score + 0.f) << 32) | (0xffffffffu - (unsigned)id);
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const unsigned long long w = __shfl_xor_sync(kFull, v, o);
        v = v > w ? v : w;
    }
    return v;
}

// one CTA (8 warps) per (n, h): the C first-level scores, 64 rows at a time, then warp 0 takes
// the m best clusters in m rounds of a warp argmax over packed (score, -c) keys
__global__ void __launch_bounds__(256) asm_hier_select_kernel(const __grid_constant__ AsmHierParams p) {
    extern __shared__ __align__(16) float s_sc[];
    unsigned char* taken = reinterpret_cast<unsigned char*>(s_sc + p.C);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long nh = blockIdx.x;
    const int h = (int)(nh % p.H);
    griddep_wait();                 // inputs may come from the previous kernel in the stream
    griddep_launch_dependents();    // the member kernel may take its slots now; it waits for this grid
    const float4 qv = hier_q4(p.q, nh, lane);
    for (int c0 = warp * 8; c0 < p.C; c0 += 64) {
        const float* rows[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) rows[r] = (c0 + r < p.C) ? p.qhat + ((size_t)h * p.C + c0 + r) * kHierD : nullptr;
        float sc[8];
        hier_score8(qv, rows, sc, lane);
#pragma unroll
        for (int r = 0; r < 8; ++r)
            if (lane == r && c0 + r < p.C) {
                s_sc[c0 + r] = sc[r];
                taken[c0 + r] = 0;
            }
    }
    __syncthreads();
    if (warp != 0) return;
    const int mm = min(p.m, p.C);
    for (int j = 0; j < p.m; ++j) {
        int out = -1;
        if (j < mm) {
            unsigned long long best = 0ull;
            for (int c = lane; c < p.C; c += 32)
                if (!taken[c]) {
                    const unsigned long long k = hier_key(s_sc[c], c);
                    best = best > k ? best : k;
                }
            best = warp_max_u64(best);
            out = (int)(0xffffffffu - (unsigned)(best & 0xffffffffull));
            if (lane == 0) taken[out] = 1;
            __syncwarp();
        }
        if (lane == 0) p.sel[nh * p.m + j] = out;
    }
}

// one CTA (8 warps) per (selected cluster j, n, h): the cluster's members, 64 rows at a time,
// the best (score, -k) key of the CTA -> keys[j][n][h]
__global__ void __launch_bounds__(256) asm_hier_score_kernel(const __grid_constant__ AsmHierParams p) {
    __shared__ unsigned long long s_best[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long nhs = (long long)p.N * p.H;
    const long long w = blockIdx.x;   // j * N * H + nh
    const long long nh = w % nhs;
    const int j = (int)(w / nhs), h = (int)(nh % p.H);
    griddep_wait();                 // sel is written by the select kernel
    griddep_launch_dependents();
    const int c = p.sel[nh * p.m + j];
    unsigned long long best = 0ull;
    if (c >= 0 && c < p.C) {
        const float4 qv = hier_q4(p.q, nh, lane);
        const int32_t* off = p.offsets + (size_t)h * (p.C + 1);
        int i0 = off[c], i1 = off[c + 1];
        if (i0 < 0 || i1 > p.K || i0 > i1) {
            if (threadIdx.x == 0) raise_error(KVB_DERR_RANGE);
            i1 = i0;
        }
        const int32_t* mem = p.members + (size_t)h * p.K;
        for (int b = i0 + warp * 8; b < i1; b += 64) {
            int kk[8];
            const float* rows[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                kk[r] = (b + r < i1) ? mem[b + r] : -1;
                if (b + r < i1 && (kk[r] < 0 || kk[r] >= p.K)) {
                    if (lane == 0) raise_error(KVB_DERR_RANGE);
                    kk[r] = -1;
                }
                rows[r] = (kk[r] >= 0) ? p.qbar + ((size_t)h * p.K + kk[r]) * kHierD : nullptr;
            }
            float sc[8];
            hier_score8(qv, rows, sc, lane);
#pragma unroll
            for (int r = 0; r < 8; ++r)
                if (kk[r] >= 0) {
                    const unsigned long long key = hier_key(sc[r], kk[r]);
                    best = best > key ? best : key;
                }
        }
    }
    if (lane == 0) s_best[warp] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 1; i < 8; ++i) best = best > s_best[i] ? best : s_best[i];
        p.keys[w] = best;
    }
}

}  // namespace kvb
