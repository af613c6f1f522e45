// Attention-state-memory lookup and merge, "Context Memorization" core method
// steps 3-4: c* = argmax_k cos(q, qbar_k), then the retrieved state
// (abar_c*, Zbar_c*) is merged with the query's own attention state.
//
// Phase 1 (asm_score_kernel) is a dense fp32 contraction per head,
// [N queries x d] . [d x K centroids], fused with a running argmax: a CTA
// takes 64 queries x one range of centroids, stages the queries and a
// double-buffered pair of centroid tiles in shared memory (cp.async, the
// next tile lands while the current one is computed; rows padded by 4
// floats so the float4 reads of 8 threads touch 8 distinct bank quads) and
// each thread keeps a 4 x 4 block of dot products in registers. The compared value is q.qbar_k / |qbar_k|,
// which orders the centroids exactly as cos does for a fixed q. The best
// (value, -k) per query is packed into one 64-bit key and written per range.
// Phase 2 (asm_merge_kernel) reduces the ranges' keys, gathers abar_c* and
// merges it with the self state: one warp per (query, head).
//
// fp32 arithmetic throughout: tf32 tensor cores would reorder near-ties.
#pragma once

#include "common.cuh"

namespace kvb {

constexpr int kAsmD = 128, kAsmQT = 64, kAsmKT = 64, kAsmNT = 256, kAsmPad = 4;
constexpr int kAsmRow = kAsmD + kAsmPad;
// q tile, two centroid tiles (double buffer), two 1/|qbar| vectors
constexpr size_t kAsmSmem = (size_t)(kAsmQT + 2 * kAsmKT) * kAsmRow * 4 + 2 * kAsmKT * 4;

// 16-byte global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

struct AsmParams {
    const uint16_t* q;
    const float* qbar;
    const uint16_t* abar;
    const float* lz;
    const float* o_self;
    const float* lse_self;
    int N, H, K, ksplit, kchunk;
    int* idx;
    float* o;
    float* lse;
    unsigned long long* ws;  // [ksplit][N][H]
};

__host__ __device__ inline int asm_ksplit(int K) {
    int s = (K + 511) / 512;
    return s < 1 ? 1 : (s > 64 ? 64 : s);
}

__host__ __device__ inline int asm_kchunk(int K) {
    const int s = asm_ksplit(K);
    const int c = (K + s - 1) / s;
    return (c + kAsmKT - 1) / kAsmKT * kAsmKT;
}

__global__ void __launch_bounds__(kAsmNT) asm_score_kernel(const __grid_constant__ AsmParams p) {
    extern __shared__ __align__(16) float s_asm[];
    float* s_q = s_asm;                            // [QT][Row]
    float* s_cbuf = s_q + kAsmQT * kAsmRow;        // [2][KT][Row]
    float* s_invb = s_cbuf + 2 * kAsmKT * kAsmRow; // [2][KT]
    const int h = blockIdx.x, n0 = blockIdx.y * kAsmQT, ks = blockIdx.z;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int k_begin = ks * p.kchunk;
    const int k_end = min(p.K, k_begin + p.kchunk);
    const int ntile = (k_end > k_begin) ? (k_end - k_begin + kAsmKT - 1) / kAsmKT : 0;

    // centroid tile `it` -> buffer it & 1, 16 bytes per cp.async, rows past k_end zero-filled
    auto prefetch = [&](int it) {
        float* dst = s_cbuf + (it & 1) * kAsmKT * kAsmRow;
        const int kt = k_begin + it * kAsmKT;
        for (int i = tid; i < kAsmKT * (kAsmD / 4); i += kAsmNT) {
            const int r = i / (kAsmD / 4), c = i % (kAsmD / 4);
            const int k = kt + r;
            const bool in = k < k_end;
            const float* src = p.qbar + ((size_t)h * p.K + (in ? k : k_begin)) * kAsmD + c * 4;
            cp_async16(dst + r * kAsmRow + c * 4, src, in ? 16 : 0);
        }
        cp_async_commit();
    };
    if (ntile > 0) prefetch(0);

    for (int i = tid; i < kAsmQT * (kAsmD / 8); i += kAsmNT) {
        const int r = i / (kAsmD / 8), c = i % (kAsmD / 8);
        const int n = n0 + r;
        float f[8];
        if (n < p.N) {
            unpack8(*reinterpret_cast<const uint4*>(p.q + ((size_t)n * p.H + h) * kAsmD + c * 8), f);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = 0.f;
        }
        float4* dst = reinterpret_cast<float4*>(s_q + r * kAsmRow + c * 8);
        dst[0] = make_float4(f[0], f[1], f[2], f[3]);
        dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }

    unsigned long long best[4] = {0ull, 0ull, 0ull, 0ull};
    for (int it = 0; it < ntile; ++it) {
        const int kt = k_begin + it * kAsmKT;
        if (it + 1 < ntile) {
            prefetch(it + 1);      // lands while this tile is computed
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();           // tile `it` (and, first time, q) visible to all threads
        const float* s_c = s_cbuf + (it & 1) * kAsmKT * kAsmRow;
        float* s_inv = s_invb + (it & 1) * kAsmKT;
        {   // 1/|qbar_k| (0 for a zero vector: its cosine is defined as 0)
            const int r = tid >> 2, part = tid & 3;
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 x = *reinterpret_cast<const float4*>(s_c + r * kAsmRow + part * 32 + e);
                ss = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, ss))));
            }
            ss += __shfl_xor_sync(kFull, ss, 1);
            ss += __shfl_xor_sync(kFull, ss, 2);
            if (part == 0) s_inv[r] = (ss > 0.f) ? 1.f / sqrtf(ss) : 0.f;
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
        for (int e = 0; e < kAsmD; e += 4) {
            float4 a[4], c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(s_q + (ty * 4 + i) * kAsmRow + e);
#pragma unroll
            for (int j = 0; j < 4; ++j) c[j] = *reinterpret_cast<const float4*>(s_c + (tx + 16 * j) * kAsmRow + e);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][j] = fmaf(a[i].x, c[j].x, acc[i][j]);
                    acc[i][j] = fmaf(a[i].y, c[j].y, acc[i][j]);
                    acc[i][j] = fmaf(a[i].z, c[j].z, acc[i][j]);
                    acc[i][j] = fmaf(a[i].w, c[j].w, acc[i][j]);
                }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = tx + 16 * j;
            const int k = kt + r;
            if (k < k_end) {
                const float inv = s_inv[r];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const unsigned long long key =
                        ((unsigned long long)float_order_key(acc[i][j] * inv) << 32) | (0xffffffffu - (unsigned)k);
                    best[i] = best[i] > key ? best[i] : key;
                }
            }
        }
        __syncthreads();           // buffer it & 1 is refilled by the prefetch of tile it + 2
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int m = 8; m >= 1; m >>= 1) {
            const unsigned long long o = __shfl_xor_sync(kFull, best[i], m);
            best[i] = best[i] > o ? best[i] : o;
        }
        const int n = n0 + ty * 4 + i;
        if (tx == 0 && n < p.N) p.ws[((size_t)ks * p.N + n) * p.H + h] = best[i];
    }
}

__global__ void __launch_bounds__(256) asm_merge_kernel(const __grid_constant__ AsmParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long nh = (long long)blockIdx.x * 8 + warp;
    if (nh >= (long long)p.N * p.H) return;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    unsigned long long best = 0ull;
    for (int s = lane; s < p.ksplit; s += 32) {
        const unsigned long long x = p.ws[((size_t)s * p.N + n) * p.H + h];
        best = best > x ? best : x;
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const unsigned long long o = __shfl_xor_sync(kFull, best, m);
        best = best > o ? best : o;
    }
    const int k = (int)(0xffffffffu - (unsigned)(best & 0xffffffffull));
    if (lane == 0 && p.idx != nullptr) p.idx[nh] = k;
    const float ls = p.lse_self[nh];
    const float lm = p.lz[(size_t)h * p.K + k];
    const float mx = fmaxf(ls, lm);
    const float mu = (mx == -INFINITY) ? 0.f : mx;
    const float ws = exp2f((ls - mu) * kLog2e), wm = exp2f((lm - mu) * kLog2e);
    const float tot = ws + wm;
    const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
    if (lane == 0 && p.lse != nullptr) p.lse[nh] = (tot > 0.f) ? mx + log2f(tot) * kLn2 : -INFINITY;
    const float4 os = *reinterpret_cast<const float4*>(p.o_self + nh * kAsmD + lane * 4);
    const uint2 am = *reinterpret_cast<const uint2*>(p.abar + ((size_t)h * p.K + k) * kAsmD + lane * 4);
    float4 r;
    r.x = (ws * os.x + wm * bf16_lo(am.x)) * inv;
    r.y = (ws * os.y + wm * bf16_hi(am.x)) * inv;
    r.z = (ws * os.z + wm * bf16_lo(am.y)) * inv;
    r.w = (ws * os.w + wm * bf16_hi(am.y)) * inv;
    *reinterpret_cast<float4*>(p.o + nh * kAsmD + lane * 4) = r;
}

}  // namespace kvb
