// Attention-state-memory lookup and merge, "Context Memorization" core method
// steps 3-4: c* = argmax_k cos(q, qbar_k), then the retrieved state
// (abar_c*, Zbar_c*) is merged with the query's own attention state.
//
// Phase 1 (asm_score_umma_kernel) is a dense contraction per head,
// [N queries x d] . [d x K centroids], on the 5th-generation tensor cores,
// fused with a running argmax. The compared value is q . (qbar_k / |qbar_k|),
// which orders the centroids as cos does for a fixed q. The best (value, -k)
// per query is packed into one 64-bit key and written per range of centroids.
// Phase 2 (asm_merge_kernel) reduces the ranges' keys, gathers abar_c* and
// merges it with the self state: one warp per (query, head).
//
// The products are fp32-exact: q is bf16, and each fp32 element x of a
// normalised centroid is split exactly into three bf16 parts (hi = rn(x),
// mid = rn(x - hi), lo = x - hi - mid, which fits in bf16), so that
// q . x = q . hi + q . mid + q . lo with exact products, accumulated in fp32.
// tf32 would round the centroids and reorder near-ties.
#pragma once

#include "common.cuh"

namespace kvb {

constexpr int kAsmD = 128, kAsmKT = 64;   // head dim; centroids per tile

struct AsmParams {
    const uint16_t* q;
    const float* qbar;
    const uint16_t* abar;
    const float* lz;
    const float* o_self;
    const float* lse_self;
    int N, H, K, ksplit, kchunk;
    int qtiles;     // ceil(N / 256): query blocks per head
    int per_cta;    // work items (head, query block, centroid range) per CTA
    int* idx;
    float* o;
    float* lse;
    unsigned long long* ws;  // [ksplit][N][H]
    int G;                   // query heads per table: head h reads table h / G
};

// Centroid ranges per head: ranges of 128 centroids (two tiles) or more, at most 64 of them,
// none empty.
__host__ __device__ inline int asm_kchunk(int K) {
    int s = (K + 127) / 128;
    s = s < 1 ? 1 : (s > 64 ? 64 : s);
    const int c = (K + s - 1) / s;
    return (c + kAsmKT - 1) / kAsmKT * kAsmKT;
}
__host__ __device__ inline int asm_ksplit(int K) {
    const int c = asm_kchunk(K);
    return K < 1 ? 1 : (K + c - 1) / c;
}

// ---- Phase 1 -------------------------------------------------------------------------------
// A work item is (head h, block of 256 queries, range of centroids); a CTA walks a contiguous
// run of items (head-major, so the queries change rarely) as one stream of centroid tiles.
// The queries are the A operand (two M = 128 tiles, bf16, reloaded only when the head or query
// block changes); a tile of 64 centroids is the B operand (N = 64). Both sit in shared memory
// in the K-major 128-byte-swizzled layout that the MMA descriptors name: rows of 128 bytes
// (64 bf16 of one 64-wide K half), 8-row groups of 1024 bytes, 16-byte chunk c of row r stored
// at chunk c ^ (r & 7). Accumulators live in tensor memory: tile g of M tile mt at columns
// ((g & 1) * 2 + mt) * 64, lane = query row. Each step g: warps 0-7 normalise and split the fp32
// tile g (held in registers) into the three bf16 parts of buffer g & 1 and arrive on named
// barrier 1 + (g & 1); warp 8 waits there, issues the 2 x 3 x 8 MMAs from one lane and commits
// them to an mbarrier; warps 0-7 meanwhile load tile g + 1 into registers and read back the
// accumulators of tile g - 1 (tcgen05.ld: warp w reads tensor-memory lanes 32 (w & 3) .. + 31
// of M tile w >> 2, one query row per thread over the 64 centroids). The two barriers
// alternate, so an arrival for tile g + 1 can never complete the barrier of tile g.
constexpr int kUQ = 128, kUMT = 2, kUKT = kAsmKT, kUNT = 256, kUCols = 256;
constexpr int kUThreads = kUNT + 32;   // 8 converting / read-back warps + the MMA warp
constexpr size_t kUA = 0;                                       // [mt][k half][128 rows][128 B]
constexpr size_t kUAHalf = (size_t)kUQ * 128;                   // 16 KB
constexpr size_t kUPartHalf = (size_t)kUKT * 128;               // 8 KB
constexpr size_t kUPart = 2 * kUPartHalf;                       // one bf16 part: two K halves
constexpr size_t kUBuf = 3 * kUPart;                            // hi, mid, lo
constexpr size_t kUB = kUA + kUMT * 2 * kUAHalf;                // [buf][part][k half][64 rows][128 B]
constexpr size_t kUBar = kUB + 2 * kUBuf;                       // 2 mbarriers
constexpr size_t kUSlot = kUBar + 16;                           // tensor-memory base address
constexpr size_t kUSmem = kUSlot + 16 + 1024;                   // + slack to align the base to 1024

__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)   // start address
         | (1ull << 16)                          // leading byte offset (unused for this layout)
         | (64ull << 32)                         // stride byte offset: 1024 B between 8-row groups
         | (1ull << 46)                          // descriptor version
         | (2ull << 61);                         // 128-byte swizzle
}

// kind::f16 instruction descriptor: f32 accumulator, bf16 A and B, both K-major, M x N
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// hi, mid, lo bf16 pairs of two fp32 values (x0 in the low half of each word)
__device__ __forceinline__ void split3_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
    __nv_bfloat162 t = __floats2bfloat162_rn(x0, x1);
    hi = *reinterpret_cast<uint32_t*>(&t);
    const float r0 = x0 - __uint_as_float(hi << 16), r1 = x1 - __uint_as_float(hi & 0xffff0000u);
    t = __floats2bfloat162_rn(r0, r1);
    mid = *reinterpret_cast<uint32_t*>(&t);
    const float s0 = r0 - __uint_as_float(mid << 16), s1 = r1 - __uint_as_float(mid & 0xffff0000u);
    t = __floats2bfloat162_rn(s0, s1);
    lo = *reinterpret_cast<uint32_t*>(&t);
}

// position of one centroid tile in a CTA's stream
struct AsmTile {
    int h, qt, ks;           // work item: head, query block, centroid range
    int kt, k_end;           // first centroid of the tile, end of the range
};

__device__ __forceinline__ void asm_tile_start(const AsmParams& p, AsmTile& c, int item) {
    c.h = item / (p.qtiles * p.ksplit);
    const int r = item % (p.qtiles * p.ksplit);
    c.qt = r / p.ksplit;
    c.ks = r % p.ksplit;
    c.kt = c.ks * p.kchunk;
    c.k_end = min(p.K, c.kt + p.kchunk);
}
// the next tile of the stream (every item has at least one tile; items are head-major)
__device__ __forceinline__ void asm_tile_next(const AsmParams& p, AsmTile& c) {
    c.kt += kUKT;
    if (c.kt < c.k_end) return;
    if (++c.ks == p.ksplit) {
        c.ks = 0;
        if (++c.qt == p.qtiles) {
            c.qt = 0;
            ++c.h;
        }
    }
    c.kt = c.ks * p.kchunk;
    c.k_end = min(p.K, c.kt + p.kchunk);
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id, int n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__global__ void __launch_bounds__(kUThreads, 1) asm_score_umma_kernel(const __grid_constant__ AsmParams p) {
    griddep_launch_dependents();   // the merge may be scheduled now; it waits for this grid before reading keys
    extern __shared__ unsigned char s_raw[];
    unsigned char* sm = s_raw + ((1024u - (smem_u32(s_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kUBar);
    uint32_t* slot = reinterpret_cast<uint32_t*>(sm + kUSlot);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int items = p.H * p.qtiles * p.ksplit;
    const int i0 = blockIdx.x * p.per_cta, i1 = min(items, i0 + p.per_cta);
    if (i0 >= i1) return;   // uniform over the CTA, before any allocation
    int G = 0;              // tiles in this CTA's stream
    for (int it = i0; it < i1; ++it) {
        const int kb = (it % p.ksplit) * p.kchunk;
        G += (min(p.K, kb + p.kchunk) - kb + kUKT - 1) / kUKT;
    }

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                     "r"(kUCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;

    if (warp == kUNT / 32) {
        // ---- MMA warp: tile g once its parts (and queries) are in shared memory
        AsmTile cm;
        asm_tile_start(p, cm, i0);
        constexpr uint32_t idesc = umma_idesc_bf16(kUQ, kUKT);
        const uint64_t a0 = umma_desc_sw128(sbase + (uint32_t)kUA);
        const uint64_t b0 = umma_desc_sw128(sbase + (uint32_t)kUB);
        for (int g = 0; g < G; ++g) {
            const int b = g & 1;
            named_bar_sync(1 + b, kUThreads);
            tc_fence_after();
            const int mts = min(kUMT, (p.N - cm.qt * (kUMT * kUQ) + kUQ - 1) / kUQ);
            if (lane == 0) {
                // the M tiles' products alternate (independent accumulators back to back)
#pragma unroll
                for (int pt = 0; pt < 3; ++pt)
#pragma unroll
                    for (int kk = 0; kk < kAsmD / 16; ++kk) {
                        // descriptors advance in 16-byte units of the start address
                        const uint32_t boff =
                            (uint32_t)(b * kUBuf + pt * kUPart + (kk >> 2) * kUPartHalf + (kk & 3) * 32);
#pragma unroll
                        for (int mt = 0; mt < kUMT; ++mt) {
                            if (mt >= mts) break;
                            const uint32_t d = tmem + (uint32_t)((b * kUMT + mt) * kUKT);
                            const uint32_t aoff = (uint32_t)(mt * 2 * kUAHalf + (kk >> 2) * kUAHalf + (kk & 3) * 32);
                            umma_bf16(d, a0 + (aoff >> 4), b0 + (boff >> 4), idesc, (pt | kk) != 0);
                        }
                    }
                umma_commit(&bar[b]);
            }
            __syncwarp();
            asm_tile_next(p, cm);
        }
    } else {
        // ---- warps 0-7: queries, centroid split, read-back and argmax
        // this thread's part of a centroid tile: row cr, four 8-float chunks (two per K half, the
        // pair order alternating with the row so that a quarter warp stores to 8 distinct chunks)
        const int cr = tid >> 2, ca = tid & 3;
        float4 x[4][2];
        auto load_tile = [&](const AsmTile& c) {
            const int k = c.kt + cr;
            const bool in = k < c.k_end;
            const float* src = p.qbar + ((size_t)(c.h / p.G) * p.K + (in ? k : 0)) * kAsmD;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = 8 * (i >> 1) + ca + 4 * ((i + cr) & 1);
                const float4* s4 = reinterpret_cast<const float4*>(src + 8 * j);
                x[i][0] = in ? __ldg(s4) : make_float4(0.f, 0.f, 0.f, 0.f);
                x[i][1] = in ? __ldg(s4 + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        AsmTile cc, ce;   // conversion cursor, read-back cursor
        asm_tile_start(p, cc, i0);
        asm_tile_start(p, ce, i0);
        load_tile(cc);

        const int emt = warp >> 2, elane = 32 * (warp & 3);   // read-back: M tile and lane quarter
        float bmax = -INFINITY;                               // running best of this thread's query row
        int bidx = -1;
        bool ok = true;
        int a_block = -1;                                     // query block in A

        auto readback = [&](int g) {
            const int b = g & 1;
            // warp-uniform outcome: the tensor-memory loads below are warp-collective
            if (!__all_sync(kFull, mbar_wait(&bar[b], (unsigned)(g >> 1) & 1u))) ok = false;
            tc_fence_after();
            const int n0 = ce.qt * (kUMT * kUQ);
            const int mts = min(kUMT, (p.N - n0 + kUQ - 1) / kUQ);
            if (ok && emt < mts) {
                float v[kUKT];
                const uint32_t ta = tmem + ((uint32_t)elane << 16) + (uint32_t)((b * kUMT + emt) * kUKT);
                tmem_ld32(ta, v);
                tmem_ld32(ta + 32, v + 32);
                tmem_ld_wait();
                if (ce.kt + kUKT > ce.k_end) {   // ragged last tile of a range
#pragma unroll
                    for (int c = 0; c < kUKT; ++c)
                        if (ce.kt + c >= ce.k_end) v[c] = -INFINITY;
                }
                float m[kUKT / 2];
#pragma unroll
                for (int c = 0; c < kUKT / 2; ++c) m[c] = fmaxf(v[c], v[c + kUKT / 2]);
#pragma unroll
                for (int w = kUKT / 4; w >= 1; w >>= 1)
#pragma unroll
                    for (int c = 0; c < w; ++c) m[c] = fmaxf(m[c], m[c + w]);
                if (m[0] > bmax) {   // strictly greater: an equal value in a later tile has a larger k
                    int first = kUKT - 1;
#pragma unroll
                    for (int c = kUKT - 1; c >= 0; --c) first = (v[c] == m[0]) ? c : first;
                    bmax = m[0];
                    bidx = ce.kt + first;
                }
            }
            tc_fence_before();
            if (ce.kt + kUKT >= ce.k_end) {   // end of the item: write this row's best, start afresh
                const int n = n0 + emt * kUQ + elane + lane;
                if (emt < mts && n < p.N) {
                    // +0.f folds -0 into +0, so that equal values compare equal as keys
                    const unsigned long long key =
                        (bidx < 0) ? 0ull
                                   : ((unsigned long long)float_order_key(bmax + 0.f) << 32) |
                                         (0xffffffffu - (unsigned)bidx);
                    p.ws[((size_t)ce.ks * p.N + n) * p.H + ce.h] = key;
                }
                bmax = -INFINITY;
                bidx = -1;
            }
            asm_tile_next(p, ce);
        };

        for (int g = 0; g < G; ++g) {
            const int b = g & 1;
            const int blk = cc.h * p.qtiles + cc.qt;
            if (blk != a_block) {
                // new queries: the MMAs still reading A (up to tile g - 1) finish first
                if (g > 0 && !mbar_wait(&bar[(g - 1) & 1], (unsigned)((g - 1) >> 1) & 1u)) ok = false;
                const int n0 = cc.qt * (kUMT * kUQ);
                for (int i = tid; i < kUMT * kUQ * 16; i += kUNT) {
                    const int row = i >> 4, j = i & 15;
                    const int n = n0 + row;
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (n < p.N)
                        v = *reinterpret_cast<const uint4*>(p.q + ((size_t)n * p.H + cc.h) * kAsmD + j * 8);
                    const int mt = row >> 7, r = row & 127, kh = j >> 3, c = j & 7;
                    *reinterpret_cast<uint4*>(sm + kUA + (mt * 2 + kh) * kUAHalf + r * 128 + ((c ^ (r & 7)) << 4)) =
                        v;
                }
                a_block = blk;
            }
            {   // normalise row cr and split it into the three parts of buffer b (whose previous
                // MMAs, tile g - 2, this thread saw complete in its read-back)
                float ss = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    ss = fmaf(x[i][0].x, x[i][0].x, fmaf(x[i][0].y, x[i][0].y, ss));
                    ss = fmaf(x[i][0].z, x[i][0].z, fmaf(x[i][0].w, x[i][0].w, ss));
                    ss = fmaf(x[i][1].x, x[i][1].x, fmaf(x[i][1].y, x[i][1].y, ss));
                    ss = fmaf(x[i][1].z, x[i][1].z, fmaf(x[i][1].w, x[i][1].w, ss));
                }
                ss += __shfl_xor_sync(kFull, ss, 1);
                ss += __shfl_xor_sync(kFull, ss, 2);
                const float inv = (ss > 0.f) ? 1.f / sqrtf(ss) : 0.f;   // a zero centroid has cos 0
                unsigned char* part = sm + kUB + b * kUBuf;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kh = i >> 1, c = ca + 4 * ((i + cr) & 1);
                    const float f[8] = {x[i][0].x * inv, x[i][0].y * inv, x[i][0].z * inv, x[i][0].w * inv,
                                        x[i][1].x * inv, x[i][1].y * inv, x[i][1].z * inv, x[i][1].w * inv};
                    uint32_t hw[4], mw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) split3_bf16x2(f[2 * e], f[2 * e + 1], hw[e], mw[e], lw[e]);
                    const size_t off = kh * kUPartHalf + cr * 128 + ((c ^ (cr & 7)) << 4);
                    *reinterpret_cast<uint4*>(part + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4*>(part + kUPart + off) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
                    *reinterpret_cast<uint4*>(part + 2 * kUPart + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
            fence_async_smem();   // A and the parts are read by the tensor cores (async proxy)
            tc_fence_before();    // tensor-memory reads of tile g - 2 precede the MMAs of tile g
            named_bar_arrive(1 + b, kUThreads);
            if (g + 1 < G) {      // tile g + 1 lands in registers while the MMAs run
                asm_tile_next(p, cc);
                load_tile(cc);
            }
            if (g > 0) readback(g - 1);
        }
        readback(G - 1);
        if (!ok) {
            raise_error(KVB_DERR_TIMEOUT);
            // give the last MMAs one more bounded wait before the tensor memory is released
            mbar_wait(&bar[(G - 1) & 1], (unsigned)((G - 1) >> 1) & 1u);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUCols) : "memory");
    }
}

__global__ void __launch_bounds__(256) asm_merge_kernel(const __grid_constant__ AsmParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long nh = (long long)blockIdx.x * 8 + warp;
    if (nh >= (long long)p.N * p.H) return;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    // the self state does not depend on the lookup: its loads go out before the keys'
    float4 os = make_float4(0.f, 0.f, 0.f, 0.f);
    float ls = 0.f;
    if (p.o != nullptr) {
        os = *reinterpret_cast<const float4*>(p.o_self + nh * kAsmD + lane * 4);
        ls = p.lse_self[nh];
    }
    griddep_wait();   // the keys come from the previous kernel (a no-op without programmatic launch)
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
    if (p.o == nullptr) {   // assignment only
        if (lane == 0) p.idx[nh] = (best == 0ull) ? -1 : (int)(0xffffffffu - (unsigned)(best & 0xffffffffull));
        return;
    }
    if (best == 0ull) {   // nothing retrieved (no candidate, or every score NaN): the self state
        if (lane == 0 && p.idx != nullptr) p.idx[nh] = -1;
        if (lane == 0 && p.lse != nullptr) p.lse[nh] = ls;
        *reinterpret_cast<float4*>(p.o + nh * kAsmD + lane * 4) = os;
        return;
    }
    const int k = (int)(0xffffffffu - (unsigned)(best & 0xffffffffull));
    if (lane == 0 && p.idx != nullptr) p.idx[nh] = k;
    const int t = h / p.G;   // the head's table
    const float lm = p.lz[(size_t)t * p.K + k];
    const float mx = fmaxf(ls, lm);
    const float mu = (mx == -INFINITY) ? 0.f : mx;
    const float ws = exp2f((ls - mu) * kLog2e), wm = exp2f((lm - mu) * kLog2e);
    const float tot = ws + wm;
    const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
    if (lane == 0 && p.lse != nullptr) p.lse[nh] = (tot > 0.f) ? mx + log2f(tot) * kLn2 : -INFINITY;
    const uint2 am = *reinterpret_cast<const uint2*>(p.abar + ((size_t)t * p.K + k) * kAsmD + lane * 4);
    float4 r;
    r.x = (ws * os.x + wm * bf16_lo(am.x)) * inv;
    r.y = (ws * os.y + wm * bf16_hi(am.x)) * inv;
    r.z = (ws * os.z + wm * bf16_lo(am.y)) * inv;
    r.w = (ws * os.w + wm * bf16_hi(am.y)) * inv;
    *reinterpret_cast<float4*>(p.o + nh * kAsmD + lane * 4) = r;
}

}  // namespace kvb
