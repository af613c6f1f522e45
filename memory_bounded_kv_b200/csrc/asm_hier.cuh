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
//   asm_hier_select_kernel  one CTA per (n, h): C first-level scores as packed
//                           (score, -c) keys; the m largest by rank (C <= 256,
//                           every thread ranks its clusters against all C) or
//                           by m rounds of a warp argmax -> sel [N, H, m]
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

// bytes of shared memory of the select kernel: C packed (score, -c) keys, then C taken flags
__host__ __device__ inline size_t hier_select_smem(int C) { return (size_t)C * 8 + (size_t)C; }

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
// once. rows[r] == nullptr: no row. The 16 partial sums (8 dots, 8 squared norms) are reduced
// by a butterfly that halves the values each step (16 shuffles in all): afterwards lanes 2r
// and 2r + 1 hold the score of row r; the return value is meaningful on those lanes.
__device__ __forceinline__ float hier_score8(const float4 qv, const float* const (&rows)[8], int lane) {
    float v[16];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const float4 x = rows[r] ? __ldg(reinterpret_cast<const float4*>(rows[r]) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[r] = fmaf(qv.x, x.x, fmaf(qv.y, x.y, fmaf(qv.z, x.z, qv.w * x.w)));
        v[8 + r] = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, x.w * x.w)));
    }
    // step with lane bit b: keep the half of the values selected by the bit, add the partner's
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 16;
        const float send = up ? v[i] : v[8 + i], keep = up ? v[8 + i] : v[i];
        v[i] = keep + __shfl_xor_sync(kFull, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 8;
        const float send = up ? v[i] : v[4 + i], keep = up ? v[4 + i] : v[i];
        v[i] = keep + __shfl_xor_sync(kFull, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 4;
        const float send = up ? v[i] : v[2 + i], keep = up ? v[2 + i] : v[i];
        v[i] = keep + __shfl_xor_sync(kFull, send, 4);
    }
    {
        const bool up = lane & 2;
        const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(kFull, send, 2);
    }
    v[0] += __shfl_xor_sync(kFull, v[0], 1);
    // lane l now holds value 8 (l >> 4 & 1) + 4 (l >> 3 & 1) + 2 (l >> 2 & 1) + (l >> 1 & 1):
    // lanes 2r, 2r + 1 the dot of row r, lanes 16 + 2r, 16 + 2r + 1 its squared norm
    const float ss = __shfl_xor_sync(kFull, v[0], 16);
    return (ss > 0.f) ? v[0] * (1.f / sqrtf(ss)) : 0.f;
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
    extern __shared__ __align__(16) unsigned long long s_key[];
    unsigned char* taken = reinterpret_cast<unsigned char*>(s_key + p.C);
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
        const float sc = hier_score8(qv, rows, lane);
        const int r = lane >> 1;
        if (lane < 16 && !(lane & 1) && c0 + r < p.C) {
            s_key[c0 + r] = hier_key(sc, c0 + r);
            taken[c0 + r] = 0;
        }
    }
    __syncthreads();
    const int mm = min(p.m, p.C);
    int32_t* sel = p.sel + nh * p.m;
    for (int j = mm + threadIdx.x; j < p.m; j += blockDim.x) sel[j] = -1;
    if (p.C <= 256) {
        // rank of each cluster = number of larger keys (keys are distinct: they carry c);
        // the clusters of rank < m are kept, best first
        for (int c = threadIdx.x; c < p.C; c += blockDim.x) {
            const unsigned long long kc = s_key[c];
            int rank = 0;
            for (int i = 0; i < p.C; ++i) rank += s_key[i] > kc;
            if (rank < mm) sel[rank] = c;
        }
        return;
    }
    if (warp != 0) return;
    for (int j = 0; j < mm; ++j) {   // many clusters: m rounds of a warp argmax
        unsigned long long best = 0ull;
        for (int c = lane; c < p.C; c += 32)
            if (!taken[c]) best = best > s_key[c] ? best : s_key[c];
        best = warp_max_u64(best);
        const int out = (int)(0xffffffffu - (unsigned)(best & 0xffffffffull));
        if (lane == 0) {
            taken[out] = 1;
            sel[j] = out;
        }
        __syncwarp();
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
            const float sc = hier_score8(qv, rows, lane);
            // lane 2r holds row r: select its entry id without indexing the array dynamically
            int kl = -1;
#pragma unroll
            for (int r = 0; r < 8; ++r) kl = (lane == 2 * r) ? kk[r] : kl;
            if (kl >= 0) {
                const unsigned long long key = hier_key(sc, kl);
                best = best > key ? best : key;
            }
        }
        best = warp_max_u64(best);
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
