// Attention-state-memory lookup and merge, "Context Memorization" core method
// steps 3-4: c* = argmax_k cos(q, qbar_k), then the retrieved state
// (abar_c*, Zbar_c*) is merged with the query's own attention state.
//
// Phase 1 (asm_score_tc_kernel) is a dense contraction per head,
// [N queries x d] . [d x K centroids], fused with a running argmax. The compared
// value is q.qbar_k / |qbar_k|, which orders the centroids exactly as cos does
// for a fixed q. The best (value, -k) per query is packed into one 64-bit key
// and written per range of centroids.
// Phase 2 (asm_merge_kernel) reduces the ranges' keys, gathers abar_c* and
// merges it with the self state: one warp per (query, head).
//
// The products are fp32-exact (bf16 q times an exact three-way bf16 split of
// the fp32 centroid) and accumulate in fp32; tf32 would round the centroids and
// reorder near-ties.
#pragma once

#include "common.cuh"

namespace kvb {

constexpr int kAsmD = 128, kAsmKT = 64;   // head dim; centroids per tile

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

// Phase 1: the contraction on the tensor cores, fp32-exact products. q is bf16, hence
// exact in bf16; each fp32 centroid element is split exactly into three bf16 parts
// (hi = rn(x), mid = rn(x - hi), lo = x - hi - mid), and q . qbar = q . hi + q . mid + q . lo
// with exact products and fp32 accumulation (mma.sync m16n8k16). A CTA owns 128 queries of one
// head (8 warps x 16 query rows, q held in registers as A fragments) and walks its range of
// centroids in tiles of 64: the fp32 tile arrives by cp.async, the CTA splits it into three
// padded bf16 tiles (row pitch 272 bytes: the 8 rows of an ldmatrix hit distinct bank groups) and takes the
// 1/|qbar| of each row, then each warp multiplies its rows by all 64 centroids.
constexpr int kAtQT = 128, kAtKT = kAsmKT, kAtNT = 256;
constexpr int kAtPitch = kAsmD + 8;   // bf16 elements per row of a part
constexpr int kAtSP = kAsmD + 16;     // floats per row of the fp32 stage
constexpr size_t kAtStage = (size_t)kAtKT * kAtSP * 4;                       // fp32 tile
constexpr size_t kAtPart = (size_t)kAtKT * kAtPitch * 2;                      // one bf16 part
constexpr size_t kAtSmem = kAtStage + 3 * kAtPart + kAtKT * 4;

__device__ __forceinline__ void mma_bf16_full(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_asm(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ unsigned short bf16_bits_rn(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__global__ void __launch_bounds__(kAtNT, 2) asm_score_tc_kernel(const __grid_constant__ AsmParams p) {
    extern __shared__ __align__(16) unsigned char s_at[];
    float* s_stage = reinterpret_cast<float*>(s_at);                                      // [KT][D] f32
    uint16_t* s_part = reinterpret_cast<uint16_t*>(s_at + kAtStage);                      // [3][KT][pitch]
    float* s_inv = reinterpret_cast<float*>(s_at + kAtStage + 3 * kAtPart);               // [KT]
    const int h = blockIdx.x, n0 = blockIdx.y * kAtQT, ks = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k_begin = ks * p.kchunk;
    const int k_end = min(p.K, k_begin + p.kchunk);
    const int ntile = (k_end > k_begin) ? (k_end - k_begin + kAtKT - 1) / kAtKT : 0;

    auto prefetch = [&](int it) {
        const int kt = k_begin + it * kAtKT;
        for (int i = tid; i < kAtKT * (kAsmD / 4); i += kAtNT) {
            const int r = i / (kAsmD / 4), c = i % (kAsmD / 4);
            const int k = kt + r;
            const bool in = k < k_end;
            const float* src = p.qbar + ((size_t)h * p.K + (in ? k : k_begin)) * kAsmD + c * 4;
            cp_async16(s_stage + r * kAtSP + c * 4, src, in ? 16 : 0);
        }
        cp_async_commit();
    };
    if (ntile > 0) prefetch(0);

    // A fragments of this warp's 16 query rows (rows past N are zero)
    const int qr = n0 + 16 * warp + (lane >> 2);
    uint32_t qa[kAsmD / 16][4];
#pragma unroll
    for (int s = 0; s < kAsmD / 16; ++s) {
        const int c0 = 16 * s + 2 * (lane & 3);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {   // rows qr, qr + 8
            const int n = qr + 8 * hf;
            uint32_t lo = 0u, hi = 0u;
            if (n < p.N) {
                const uint16_t* qp = p.q + ((size_t)n * p.H + h) * kAsmD;
                lo = *reinterpret_cast<const uint32_t*>(qp + c0);
                hi = *reinterpret_cast<const uint32_t*>(qp + c0 + 8);
            }
            qa[s][hf] = lo;       // a0 (row), a1 (row + 8)
            qa[s][2 + hf] = hi;   // a2 (row, col + 8), a3 (row + 8, col + 8)
        }
    }

    unsigned long long best[2] = {0ull, 0ull};   // rows qr and qr + 8
    const uint32_t part_base = smem_u32(s_part);
    for (int it = 0; it < ntile; ++it) {
        const int kt = k_begin + it * kAtKT;
        cp_async_wait<0>();
        __syncthreads();   // fp32 tile visible; the bf16 parts of the previous tile are no longer read
        {   // split into three bf16 parts; 1/|qbar| per row. Four threads per row, each taking
            // 4-float chunks 16 apart (stage pitch 144 floats: a quarter warp reads 32 distinct banks)
            const int r = tid >> 2, part = tid & 3;
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < kAsmD / 16; ++e) {
                const int col = part * 4 + 16 * e;
                const float4 x = *reinterpret_cast<const float4*>(s_stage + r * kAtSP + col);
                ss = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, ss))));
                const float xs[4] = {x.x, x.y, x.z, x.w};
                uint32_t hw[2] = {0u, 0u}, mw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const unsigned short hb = bf16_bits_rn(xs[c]);
                    const float r1 = xs[c] - __uint_as_float((unsigned)hb << 16);   // exact
                    const unsigned short mb = bf16_bits_rn(r1);
                    const float r2 = r1 - __uint_as_float((unsigned)mb << 16);      // exact
                    const unsigned short lb = bf16_bits_rn(r2);                     // exact: <= 8 bits left
                    hw[c >> 1] |= (uint32_t)hb << (16 * (c & 1));
                    mw[c >> 1] |= (uint32_t)mb << (16 * (c & 1));
                    lw[c >> 1] |= (uint32_t)lb << (16 * (c & 1));
                }
                const int off = r * kAtPitch + col;
                *reinterpret_cast<uint2*>(s_part + off) = make_uint2(hw[0], hw[1]);
                *reinterpret_cast<uint2*>(s_part + kAtKT * kAtPitch + off) = make_uint2(mw[0], mw[1]);
                *reinterpret_cast<uint2*>(s_part + 2 * kAtKT * kAtPitch + off) = make_uint2(lw[0], lw[1]);
            }
            ss += __shfl_xor_sync(kFull, ss, 1);
            ss += __shfl_xor_sync(kFull, ss, 2);
            if (part == 0) s_inv[r] = (ss > 0.f) ? 1.f / sqrtf(ss) : 0.f;
        }
        __syncthreads();                      // parts and norms ready; the stage buffer is free
        if (it + 1 < ntile) prefetch(it + 1); // lands while this tile is multiplied

        float acc[kAtKT / 8][4];
#pragma unroll
        for (int j = 0; j < kAtKT / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
        // ldmatrix row of this lane: centroid (8 x matrix) and 16-byte chunk
        const int lrow = (lane & 7) + ((lane >> 4) << 3);
        const int lchk = (lane >> 3) & 1;
        // k-step outermost: consecutive mma go to the 8 independent accumulators
#pragma unroll
        for (int pt = 0; pt < 3; ++pt) {
#pragma unroll
            for (int s = 0; s < kAsmD / 16; ++s) {
#pragma unroll
                for (int jp = 0; jp < kAtKT / 16; ++jp) {           // pairs of 8-centroid n-tiles
                    const uint32_t addr = part_base +
                        (uint32_t)(((pt * kAtKT + 16 * jp + lrow) * kAtPitch + 16 * s + 8 * lchk) * 2);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_asm(addr, b0, b1, b2, b3);
                    mma_bf16_full(acc[2 * jp], qa[s], b0, b1);
                    mma_bf16_full(acc[2 * jp + 1], qa[s], b2, b3);
                }
            }
        }
        // running argmax of q.qbar / |qbar| per query row (lowest k among equal values)
#pragma unroll
        for (int j = 0; j < kAtKT / 8; ++j) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int r = 8 * j + 2 * (lane & 3) + c;
                const int k = kt + r;
                if (k < k_end) {
                    const float inv = s_inv[r];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const unsigned long long key =
                            ((unsigned long long)float_order_key(acc[j][2 * hf + c] * inv) << 32) |
                            (0xffffffffu - (unsigned)k);
                        best[hf] = best[hf] > key ? best[hf] : key;
                    }
                }
            }
        }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int m = 1; m <= 2; m <<= 1) {
            const unsigned long long o = __shfl_xor_sync(kFull, best[hf], m);
            best[hf] = best[hf] > o ? best[hf] : o;
        }
        const int n = qr + 8 * hf;
        if ((lane & 3) == 0 && n < p.N) p.ws[((size_t)ks * p.N + n) * p.H + h] = best[hf];
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
