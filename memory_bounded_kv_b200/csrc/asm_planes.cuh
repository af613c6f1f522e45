// Attention-state-memory lookup over a prepared memory ("Context Memorization"
// core method step 3: c* = argmax_k cos(q, qbar_k)). The memory is static once
// built, so the normalisation of every centroid and its exact split into three
// bf16 parts (hi = rn(x), mid = rn(x - hi), lo = x - hi - mid) are done once by
// asm_prepare_kernel, which writes each tile of 128 centroids as the exact
// shared-memory image the tensor-core MMA reads: [part][K half][128 rows][128 B],
// 16-byte chunk c of row r at chunk c ^ (r & 7) (the 128-byte swizzle).
//
// asm_score_planes_kernel streams those images with bulk copies, one part of a
// tile (32 KB) per stage of a 5-stage ring, and keeps the block's 256 queries in
// shared memory (one TMA box per M tile and K half, K-major, 128-byte swizzle):
// every tcgen05.mma is M = 128 queries, N = 128 centroids, K = 16, the shape the
// tensor cores run at full rate (N = 64 ran at ~70 %). A tile is two units, one
// per M tile; unit (g, m) accumulates in buffer 2 (g % 2) + m of four 128-column
// tensor-memory buffers, so tile g + 1's products never wait for tile g's
// read-back:
//   warp 9 (one lane)  the block's queries (-> a_full; a new block waits for
//                      a_empty), then the parts of each tile    -> b_full[s]
//   warp 8 (one lane)  per part 16 MMAs (8 K steps x 2 M tiles, the M tiles
//                      alternating), committed to b_empty[s]; each unit's
//                      buffer committed to acc_full[b] (the last part is issued
//                      one M tile after the other, so the first unit is ready a
//                      part's work earlier); a block's last tile -> a_empty
//   warps 0-7          warps 4 m .. 4 m + 3 read back unit m's 128 scores of
//                      their query row (tcgen05.ld), release the buffer
//                      (-> acc_empty[b]) and keep the running best.
// The per-range best keys go to the same workspace as asm_score_umma_kernel's,
// reduced and merged by asm_merge_kernel.
#pragma once

#include <cuda.h>

#include "asm_lookup.cuh"

namespace kvb {

constexpr int kPT = 128;                                        // centroids per tile (the MMA's N)
constexpr size_t kPHalf = (size_t)kPT * 128;                    // one K half of one part: 16 KB
constexpr size_t kPPart = 2 * kPHalf;                           // one part: 32 KB (a ring stage)
constexpr size_t kPImg = 3 * kPPart;                            // one tile image: 96 KB
constexpr int kPStages = 5;                                     // ring stages (one part each)
constexpr int kPAcc = 4;                                        // accumulator buffers: two per M tile
constexpr int kPThreads = kUNT + 64;                            // 8 read-back warps + MMA warp + copy warp
constexpr int kPCols = 512;                                     // kPAcc * kPT
constexpr size_t kPAHalf = (size_t)kUQ * 128;                   // queries: one M tile, one K half: 16 KB
constexpr size_t kPA = (size_t)kUMT * 2 * kPAHalf;              // queries [M tile][K half][128 rows][128 B]
constexpr size_t kPRing = kPA;                                  // the ring after the queries
constexpr size_t kPBar = kPRing + (size_t)kPStages * kPPart;    // after the ring
constexpr size_t kPSmem = kPBar + 256 + 1024;                   // barriers + slot, + alignment slack
static_assert(kPAcc * kPT == kPCols, "tensor memory budget");
static_assert(kPSmem <= 227 * 1024, "shared memory budget");

__host__ __device__ inline size_t asm_plane_tiles(int K) { return (size_t)(K + kPT - 1) / kPT; }

// Centroid ranges of the lookup over a prepared memory: whole tiles, as many ranges per (head,
// query block) as there are CTAs for it (so that a CTA's items seldom span two blocks), at most
// asm_ksplit(K) of them (the workspace holds that many).
__host__ inline int asm_planes_kchunk(int K, int blocks, int slots) {
    const int cpb = blocks >= slots ? 1 : slots / blocks;                  // CTAs per (head, query block)
    int c = (K + cpb - 1) / cpb;
    const int c_min = (K + asm_ksplit(K) - 1) / asm_ksplit(K);
    c = c < c_min ? c_min : c;
    return (c + kPT - 1) / kPT * kPT;
}

// ---- preparation: one warp per centroid row --------------------------------------------------
__global__ void __launch_bounds__(256) asm_prepare_kernel(const float* __restrict__ qbar, int H, int K,
                                                          unsigned char* __restrict__ planes) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t tiles = asm_plane_tiles(K);
    const long long row = (long long)blockIdx.x * 8 + warp;         // (table, tile row) over padded K
    if (row >= (long long)H * tiles * kPT) return;
    const int h = (int)(row / ((long long)tiles * kPT));
    const int kk = (int)(row % ((long long)tiles * kPT));           // centroid index (maybe >= K: zeros)
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (kk < K) x = reinterpret_cast<const float4*>(qbar + ((size_t)h * K + kk) * kAsmD)[lane];
    float ss = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, x.w * x.w)));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(kFull, ss, m);
    const float inv = (ss > 0.f) ? 1.f / sqrtf(ss) : 0.f;   // a zero centroid has cos 0
    uint32_t hw[2], mw[2], lw[2];
    split3_bf16x2(x.x * inv, x.y * inv, hw[0], mw[0], lw[0]);
    split3_bf16x2(x.z * inv, x.w * inv, hw[1], mw[1], lw[1]);
    // lane l holds elements 4l .. 4l + 3: K half l / 16, chunk (l % 16) / 2, bytes 8 (l % 2) .. + 7
    const int r = kk % kPT;
    const int kh = lane >> 4, c = (lane & 15) >> 1;
    unsigned char* img = planes + ((size_t)h * tiles + kk / kPT) * kPImg;
    const size_t off = kh * kPHalf + r * 128 + ((c ^ (r & 7)) << 4) + 8 * (lane & 1);
    *reinterpret_cast<uint2*>(img + off) = make_uint2(hw[0], hw[1]);
    *reinterpret_cast<uint2*>(img + kPPart + off) = make_uint2(mw[0], mw[1]);
    *reinterpret_cast<uint2*>(img + 2 * kPPart + off) = make_uint2(lw[0], lw[1]);
}

// ---- tensor-memory helpers of the lookup ------------------------------------------------------
// D (tensor memory) (+)= A (tensor memory) . B (shared memory descriptor)
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                             uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// 32 lanes x 32 consecutive columns from registers (lane i of the warp writes lane base + i)
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct AsmPlanesParams {
    AsmParams a;                   // queries, sizes, items, outputs (a.qbar unused)
    const unsigned char* planes;   // [H_tables][tiles][kPImg]
    unsigned long long wait_ns;
};

// 3-D box copy (x = dims, y = head, z = query) of the queries' tensor map into shared memory
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// The tile stream of a CTA: its run of items (head, query block, centroid range), each range
// walked in tiles of kPT centroids (items are head-major, so the queries change rarely).
struct PTile {
    int h, qt, ks, kt, k_end;
};
__device__ __forceinline__ void ptile_start(const AsmParams& p, PTile& c, int item) {
    c.h = item / (p.qtiles * p.ksplit);
    const int r = item % (p.qtiles * p.ksplit);
    c.qt = r / p.ksplit;
    c.ks = r % p.ksplit;
    c.kt = c.ks * p.kchunk;
    c.k_end = min(p.K, c.kt + p.kchunk);
}
__device__ __forceinline__ void ptile_next(const AsmParams& p, PTile& c) {
    c.kt += kPT;
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

__global__ void __launch_bounds__(kPThreads, 1) asm_score_planes_kernel(const __grid_constant__ AsmPlanesParams pp,
                                                                        const __grid_constant__ CUtensorMap tmQ) {
    griddep_launch_dependents();   // the merge may be scheduled now; it waits for this grid before reading keys
    if (threadIdx.x == 0) prefetch_tensormap(&tmQ);
    const AsmParams& p = pp.a;
    extern __shared__ unsigned char s_raw[];
    unsigned char* sm = s_raw + ((1024u - (smem_u32(s_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* b_full = reinterpret_cast<uint64_t*>(sm + kPBar);
    uint64_t* b_empty = b_full + kPStages;
    uint64_t* acc_full = b_empty + kPStages;
    uint64_t* acc_empty = acc_full + kPAcc;
    uint64_t* a_full = acc_empty + kPAcc;   // the block's queries landed
    uint64_t* a_empty = a_full + 1;         // every MMA that read them is done
    uint32_t* slot = reinterpret_cast<uint32_t*>(a_empty + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int items = p.H * p.qtiles * p.ksplit;
    const int i0 = blockIdx.x * p.per_cta, i1 = min(items, i0 + p.per_cta);
    if (i0 >= i1) return;   // uniform over the CTA, before any allocation
    int G = 0;              // tiles in this CTA's stream
    for (int it = i0; it < i1; ++it) {
        const int kb = (it % p.ksplit) * p.kchunk;
        G += (min(p.K, kb + p.kchunk) - kb + kPT - 1) / kPT;
    }
    const size_t tiles_per_table = asm_plane_tiles(p.K);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                     "r"(kPCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        for (int b = 0; b < kPAcc; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);   // the four warps of the unit's M tile
        }
        mbar_init(a_full, 1);
        mbar_init(a_empty, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    bool ok = true;

    if (warp == kUNT / 32 + 1) {
        // ---- copy warp: each block's queries, then the parts of each tile into the ring
        if (lane == 0) {
            PTile c;
            ptile_start(p, c, i0);
            int issued = 0, blocks = 0, a_block = -1;
            for (int g = 0; g < G && ok; ++g) {
                const int blk = c.h * p.qtiles + c.qt;
                if (blk != a_block) {
                    // the previous block's MMAs are done before its queries are replaced
                    if (blocks > 0 && !mbar_wait(a_empty, (unsigned)(blocks - 1) & 1u, pp.wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(a_full, (unsigned)kPA);
#pragma unroll
                    for (int mt = 0; mt < kUMT; ++mt)
#pragma unroll
                        for (int kh = 0; kh < 2; ++kh)   // rows past N read zeros
                            tma_load_3d(sm + (size_t)(mt * 2 + kh) * kPAHalf, &tmQ, 64 * kh, c.h,
                                        c.qt * (kUMT * kUQ) + mt * kUQ, a_full);
                    ++blocks;
                    a_block = blk;
                }
                const unsigned char* src = pp.planes + ((size_t)(c.h / p.G) * tiles_per_table + c.kt / kPT) * kPImg;
                for (int pt = 0; pt < 3; ++pt) {
                    const int j = 3 * g + pt, s = j % kPStages;
                    if (j >= kPStages && !mbar_wait(&b_empty[s], (unsigned)((j / kPStages) - 1) & 1u, pp.wait_ns)) {
                        ok = false;
                        break;
                    }
                    unsigned char* dst = sm + kPRing + (size_t)s * kPPart;
                    mbar_arrive_expect_tx(&b_full[s], (unsigned)kPPart);
                    bulk_g2s(dst, src + pt * kPPart, (unsigned)kPHalf, &b_full[s]);
                    bulk_g2s(dst + kPHalf, src + pt * kPPart + kPHalf, (unsigned)kPHalf, &b_full[s]);
                    issued = j + 1;
                }
                ptile_next(p, c);
            }
            // every copy lands before the CTA can exit (bounded): the last stage issued on each slot,
            // and the last block's queries
            for (int j = max(0, issued - kPStages); j < issued; ++j)
                mbar_wait(&b_full[j % kPStages], (unsigned)(j / kPStages) & 1u, 100000000ull);
            if (blocks > 0) mbar_wait(a_full, (unsigned)(blocks - 1) & 1u, 100000000ull);
        }
    } else if (warp == kUNT / 32) {
        // ---- MMA warp
        if (lane == 0) {
            PTile cm;
            ptile_start(p, cm, i0);
            constexpr uint32_t idesc = umma_idesc_bf16(kUQ, kPT);
            const uint64_t a0 = umma_desc_sw128(sbase);
            const uint64_t b0 = umma_desc_sw128(sbase + (uint32_t)kPRing);
            int a_block = -1, blocks = 0;
            for (int g = 0; g < G && ok; ++g) {
                // unit (g, m) takes buffer 2 (g % 2) + m, free once tile g - 2's unit m is read back
                uint32_t dacc[kUMT];
#pragma unroll
                for (int mt = 0; mt < kUMT; ++mt) {
                    const int b = 2 * (g & 1) + mt;
                    dacc[mt] = tmem + (uint32_t)(b * kPT);
                    if (g >= 2 && !mbar_wait(&acc_empty[b], (unsigned)((g >> 1) - 1) & 1u, pp.wait_ns)) ok = false;
                }
                if (!ok) break;
                const int blk = cm.h * p.qtiles + cm.qt;
                if (blk != a_block) {
                    if (!mbar_wait(a_full, (unsigned)blocks & 1u, pp.wait_ns)) { ok = false; break; }
                    ++blocks;
                    a_block = blk;
                }
                const int mts = min(kUMT, (p.N - cm.qt * (kUMT * kUQ) + kUQ - 1) / kUQ);
                for (int pt = 0; pt < 3 && ok; ++pt) {
                    const int j = 3 * g + pt, s = j % kPStages;
                    if (!mbar_wait(&b_full[s], (unsigned)(j / kPStages) & 1u, pp.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    if (pt < 2) {
#pragma unroll
                        for (int kk = 0; kk < kAsmD / 16; ++kk) {
                            const uint32_t boff = (uint32_t)(s * kPPart + (kk >> 2) * kPHalf + (kk & 3) * 32);
#pragma unroll
                            for (int mt = 0; mt < kUMT; ++mt) {   // the M tiles alternate (independent accumulators)
                                if (mt >= mts) break;
                                const uint32_t aoff = (uint32_t)((mt * 2 + (kk >> 2)) * kPAHalf + (kk & 3) * 32);
                                umma_bf16(dacc[mt], a0 + (aoff >> 4), b0 + (boff >> 4), idesc, (pt | kk) != 0);
                            }
                        }
                    } else {
                        // the last part one M tile after the other, each unit committed as soon as its
                        // products are issued: the first unit's read-back starts a part's work earlier
#pragma unroll
                        for (int mt = 0; mt < kUMT; ++mt) {
                            if (mt < mts) {
#pragma unroll
                                for (int kk = 0; kk < kAsmD / 16; ++kk) {
                                    const uint32_t boff = (uint32_t)(s * kPPart + (kk >> 2) * kPHalf + (kk & 3) * 32);
                                    const uint32_t aoff = (uint32_t)((mt * 2 + (kk >> 2)) * kPAHalf + (kk & 3) * 32);
                                    umma_bf16(dacc[mt], a0 + (aoff >> 4), b0 + (boff >> 4), idesc, 1u);
                                }
                            }
                            umma_commit(&acc_full[2 * (g & 1) + mt]);
                        }
                    }
                    umma_commit(&b_empty[s]);
                }
                if (!ok) break;
                PTile nx = cm;
                ptile_next(p, nx);
                // the block's last tile: its queries may be replaced once these products are done
                if (g == G - 1 || nx.h * p.qtiles + nx.qt != blk) umma_commit(a_empty);
                cm = nx;
            }
        }
    } else {
        // ---- warps 0-7: read-back and argmax (warps 4 m .. 4 m + 3 read M tile m's units)
        PTile ce;
        ptile_start(p, ce, i0);
        const int emt = warp >> 2, elane = 32 * (warp & 3);
        float bmax = -INFINITY;
        int bidx = -1;
        for (int g = 0; g < G; ++g) {
            const int n0 = ce.qt * (kUMT * kUQ);
            const int b = 2 * (g & 1) + emt;
            // warp-uniform outcome: the tensor-memory loads below are warp-collective
            if (!__all_sync(kFull, mbar_wait(&acc_full[b], (unsigned)(g >> 1) & 1u, pp.wait_ns))) ok = false;
            tc_fence_after();
            const int mts = min(kUMT, (p.N - n0 + kUQ - 1) / kUQ);
            const bool mine = ok && emt < mts;
            // the unit's 128 scores of this row: the best value and its first column
            float best = -INFINITY;
            int first = -1;
            if (mine) {
                // all four loads, one wait, release the buffer, then the arithmetic
                const uint32_t ta = tmem + ((uint32_t)elane << 16) + (uint32_t)(b * kPT);
                float v[kPT];
#pragma unroll
                for (int c = 0; c < kPT; c += 32) tmem_ld32(ta + c, v + c);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
                if (ce.kt + kPT > ce.k_end) {   // ragged last tile of a range
#pragma unroll
                    for (int c = 0; c < kPT; ++c)
                        if (ce.kt + c >= ce.k_end) v[c] = -INFINITY;
                }
                float m[kPT / 2];
#pragma unroll
                for (int c = 0; c < kPT / 2; ++c) m[c] = fmaxf(v[c], v[c + kPT / 2]);
#pragma unroll
                for (int w = kPT / 4; w >= 1; w >>= 1)
#pragma unroll
                    for (int c = 0; c < w; ++c) m[c] = fmaxf(m[c], m[c + w]);
                int f = kPT - 1;
#pragma unroll
                for (int c = kPT - 1; c >= 0; --c) f = (v[c] == m[0]) ? c : f;   // the first column of the max
                best = m[0];
                first = f;
            } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
            if (mine && best > bmax) {   // strictly greater: an equal value in a later tile has a larger k
                bmax = best;
                bidx = ce.kt + first;
            }
            if (ce.kt + kPT >= ce.k_end) {   // end of the item: write this row's best, start afresh
                const int n = n0 + emt * kUQ + elane + lane;
                if (emt < mts && n < p.N) {
                    const unsigned long long key =
                        (bidx < 0 || !ok) ? 0ull
                                          : ((unsigned long long)float_order_key(bmax + 0.f) << 32) |
                                                (0xffffffffu - (unsigned)bidx);
                    p.ws[((size_t)ce.ks * p.N + n) * p.H + ce.h] = key;
                }
                bmax = -INFINITY;
                bidx = -1;
            }
            ptile_next(p, ce);
        }
    }
    if (!ok) raise_error(KVB_DERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == kUNT / 32 && lane == 0 && G > 0) {
        // the last tile's MMAs complete before the tensor memory is released (bounded)
        mbar_wait(&acc_full[2 * ((G - 1) & 1) + 1], (unsigned)((G - 1) >> 1) & 1u, pp.wait_ns);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPCols) : "memory");
    }
}

}  // namespace kvb
