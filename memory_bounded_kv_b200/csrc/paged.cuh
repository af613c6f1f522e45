// Paged memory-bounded KV cache: the slots of every (sequence, kv head) live in
// pages of kPageSlots slots drawn from one pool, found through a block table.
// Logical slot s of (b, g) is row s % kPageSlots of page table[b, g, s / kPageSlots];
// the pages of a (b, g) hold its slots [0, len) contiguously, the last page
// partly. Free pages sit on a device-side stack (free_pages[0 .. *free_count)).
//
// Operations on the logical cache are those of the flat cache:
//  - paged_evict_insert_kernel: budget enforcement of "Cache What Lasts"
//    section 2.1 and insertion; an append at a page boundary pops a page;
//  - paged_compact_kernel: MEMENTO's in-place removal of a finished block's
//    slots (chunking/compression; dual information stream: the later entries
//    keep their bytes): the tail after the range moves down through the
//    table, and the pages the cache no longer reaches are pushed back.
// The attention reads pages through the table (decode_attn_tc_kernel<PAGED>).
#pragma once

#include "common.cuh"

namespace kvb {

constexpr int kPageSlots = 64;

struct PagedCache {
    uint16_t* k;       // [P, kPageSlots, d]
    uint16_t* v;
    float* lb;         // [P, kPageSlots] or null
    int* pos;          // [P, kPageSlots]
    int* table;        // [B, Hkv, max_pages]
    int* len;          // [B, Hkv]
    int* free_pages;   // [P]
    int* free_count;   // [1]
    int Hkv, d, max_pages, num_pages;
};

struct PagedEvictParams {
    PagedCache c;
    const uint16_t* k_new;
    const uint16_t* v_new;
    const float* lb_new;
    const int* t;
    int M;
    int* victim;
    const EvictCand* cand;
    int cand_n;
};

// The page holding logical page j of row bg, or -1 (recording KVB_DERR_RANGE) when the table
// names no page of the pool.
__device__ __forceinline__ int page_of(const PagedCache& c, size_t bg, int j) {
    const int pg = c.table[bg * c.max_pages + j];
    if (pg < 0 || pg >= c.num_pages) {
        raise_error(KVB_DERR_RANGE);
        return -1;
    }
    return pg;
}

template <int NT>
__global__ void __launch_bounds__(NT) paged_evict_insert_kernel(const __grid_constant__ PagedEvictParams p) {
    __shared__ unsigned long long s_key[NT / 32];
    __shared__ int s_slot[NT / 32];
    __shared__ int s_sel, s_page;
    griddep_wait();
    griddep_launch_dependents();
    const PagedCache& c = p.c;
    const int bg = blockIdx.x, b = bg / c.Hkv, tid = threadIdx.x;
    const int tb = p.t[b];
    const int n = c.len[bg];
    EvictCand my_cand{~0ull, -1, 0};
    if (p.cand != nullptr && tid < 32 && tid < p.cand_n) my_cand = p.cand[(size_t)bg * p.cand_n + tid];
    if (tb < 0) {
        if (tid == 0 && p.victim) p.victim[bg] = -1;
        return;
    }
    const int cap = c.max_pages * kPageSlots;
    if (n < 0 || n > cap) {
        if (tid == 0) {
            raise_error(KVB_DERR_LEN);
            if (p.victim) p.victim[bg] = -1;
        }
        return;
    }
    int slot = -1;
    if (n >= p.M && p.cand != nullptr) {
        if (tid < 32) {
            unsigned long long best = ~0ull;
            int best_slot = 0x7fffffff;
            bool stale = tid < p.cand_n && my_cand.t != tb;
            if (my_cand.slot >= 0) argmin_merge(best, best_slot, my_cand.key, my_cand.slot);
            for (int j = tid + 32; j < p.cand_n; j += 32) {
                const EvictCand cc = p.cand[(size_t)bg * p.cand_n + j];
                stale = stale || cc.t != tb;
                if (cc.slot >= 0) argmin_merge(best, best_slot, cc.key, cc.slot);
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
                const unsigned long long k2 = __shfl_xor_sync(kFull, best, m);
                const int s2 = __shfl_xor_sync(kFull, best_slot, m);
                argmin_merge(best, best_slot, k2, s2);
            }
            stale = __any_sync(kFull, stale);
            if (tid == 0) s_sel = (!stale && best != ~0ull && best_slot < n) ? best_slot : -1;
        }
        __syncthreads();
        slot = s_sel;
    }
    if (n < p.M) {
        slot = n;
    } else if (slot < 0) {
        // scan every slot, page by page: 16 threads per page, four slots each (16-byte loads)
        unsigned long long best = ~0ull;
        int best_slot = 0x7fffffff;
        const int pages = (n + kPageSlots - 1) / kPageSlots;
        for (int j = tid / 16; j < pages; j += NT / 16) {
            const int pg = page_of(c, bg, j);
            if (pg < 0) continue;
            const int q4 = tid % 16;
            const int s = j * kPageSlots + 4 * q4;
            const int4 pv = reinterpret_cast<const int4*>(c.pos + (size_t)pg * kPageSlots)[q4];
            const float4 lv = c.lb ? reinterpret_cast<const float4*>(c.lb + (size_t)pg * kPageSlots)[q4]
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            const int ps[4] = {pv.x, pv.y, pv.z, pv.w};
            const float ls[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (s + e >= n) continue;
                const float sc = c.lb ? __fmul_rn(__int2float_rn(tb - ps[e]), ls[e]) : 0.f;
                const unsigned long long key =
                    ((unsigned long long)float_order_key(sc) << 32) | (unsigned)(ps[e] ^ 0x80000000);
                argmin_merge(best, best_slot, key, s + e);
            }
        }
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
        if (slot >= n) {   // no readable page: nothing is evicted or written
            if (tid == 0 && p.victim) p.victim[bg] = -1;
            return;
        }
    }
    // the page of the written slot; an append at a page boundary takes a page off the free stack
    if (tid == 0) {
        int pg = -1;
        if (n < p.M && slot % kPageSlots == 0) {
            const int top = atomicSub(c.free_count, 1) - 1;
            if (top < 0 || top >= c.num_pages) {
                atomicAdd(c.free_count, 1);
                raise_error(KVB_DERR_PAGES);
            } else {
                pg = c.free_pages[top];
                if (pg < 0 || pg >= c.num_pages) {
                    raise_error(KVB_DERR_RANGE);
                    pg = -1;
                } else {
                    c.table[(size_t)bg * c.max_pages + slot / kPageSlots] = pg;
                }
            }
        } else {
            pg = page_of(c, bg, slot / kPageSlots);
        }
        s_page = pg;
    }
    __syncthreads();
    const int pg = s_page;
    if (pg < 0) {   // out of pages or a bad table entry: the token is not inserted
        if (tid == 0 && p.victim) p.victim[bg] = -1;
        return;
    }
    const size_t row = (size_t)pg * kPageSlots + slot % kPageSlots;
    const int vecs = c.d / 8;
    if (p.k_new != nullptr) {
        for (int i = tid; i < 2 * vecs; i += NT) {
            if (i < vecs) {
                reinterpret_cast<uint4*>(c.k + row * c.d)[i] = reinterpret_cast<const uint4*>(p.k_new + (size_t)bg * c.d)[i];
            } else {
                reinterpret_cast<uint4*>(c.v + row * c.d)[i - vecs] =
                    reinterpret_cast<const uint4*>(p.v_new + (size_t)bg * c.d)[i - vecs];
            }
        }
    }
    if (tid == 0) {
        if (c.lb != nullptr) c.lb[row] = p.lb_new[bg];
        c.pos[row] = tb;
        if (n < p.M) c.len[bg] = n + 1;
        if (p.victim) p.victim[bg] = (n < p.M) ? -1 : slot;
    }
}

struct PagedCompactParams {
    PagedCache c;
    const int* rm_start;
    const int* rm_len;
    int W;   // rows staged per chunk
};

// One CTA per (sequence, kv head): logical rows r0 + rl .. len - 1 move to r0 .. len - rl - 1 in
// chunks of W rows staged through shared memory (a chunk is read whole before it is written; its
// destination lies below every later chunk's source), then the pages past the new length go back
// on the free stack.
template <int NT>
__global__ void __launch_bounds__(NT) paged_compact_kernel(const __grid_constant__ PagedCompactParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const PagedCache& c = p.c;
    const int bg = blockIdx.x, b = bg / c.Hkv, tid = threadIdx.x;
    const int r0 = p.rm_start[b], rl = p.rm_len[b];
    if (rl == 0) return;
    const int n = c.len[bg];
    const int cap = c.max_pages * kPageSlots;
    if (r0 < 0 || rl < 0 || n < 0 || n > cap || (long long)r0 + rl > n) {
        if (tid == 0) raise_error(KVB_DERR_RANGE);
        return;
    }
    // every page the move touches must be a page of the pool
    __shared__ int s_bad;
    if (tid == 0) s_bad = 0;
    __syncthreads();
    for (int j = r0 / kPageSlots + tid; j < (n + kPageSlots - 1) / kPageSlots; j += NT) {
        const int pg = c.table[(size_t)bg * c.max_pages + j];
        if (pg < 0 || pg >= c.num_pages) s_bad = 1;
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) raise_error(KVB_DERR_RANGE);
        return;
    }
    const int tail = n - r0 - rl;
    const int vecs = c.d / 8;
    uint4* s_k = reinterpret_cast<uint4*>(smem);
    uint4* s_v = s_k + (size_t)p.W * vecs;
    int* s_pos = reinterpret_cast<int*>(s_v + (size_t)p.W * vecs);
    float* s_lb = reinterpret_cast<float*>(s_pos + p.W);
    const int* tab = c.table + (size_t)bg * c.max_pages;
    auto row_of = [&](int s) { return (size_t)tab[s / kPageSlots] * kPageSlots + (s % kPageSlots); };
    for (int c0 = 0; c0 < tail; c0 += p.W) {
        const int w = min(p.W, tail - c0);
        const int src = r0 + rl + c0, dst = r0 + c0;
        for (int i = tid; i < w * vecs; i += NT) {
            const size_t r = row_of(src + i / vecs);
            s_k[i] = reinterpret_cast<const uint4*>(c.k)[r * vecs + i % vecs];
            s_v[i] = reinterpret_cast<const uint4*>(c.v)[r * vecs + i % vecs];
        }
        for (int i = tid; i < w; i += NT) {
            const size_t r = row_of(src + i);
            s_pos[i] = c.pos[r];
            if (c.lb) s_lb[i] = c.lb[r];
        }
        __syncthreads();
        for (int i = tid; i < w * vecs; i += NT) {
            const size_t r = row_of(dst + i / vecs);
            reinterpret_cast<uint4*>(c.k)[r * vecs + i % vecs] = s_k[i];
            reinterpret_cast<uint4*>(c.v)[r * vecs + i % vecs] = s_v[i];
        }
        for (int i = tid; i < w; i += NT) {
            const size_t r = row_of(dst + i);
            c.pos[r] = s_pos[i];
            if (c.lb) c.lb[r] = s_lb[i];
        }
        __syncthreads();
    }
    if (tid == 0) {
        const int nn = n - rl;
        for (int j = (nn + kPageSlots - 1) / kPageSlots; j < (n + kPageSlots - 1) / kPageSlots; ++j) {
            const int top = atomicAdd(c.free_count, 1);
            if (top < 0 || top >= c.num_pages) {   // a stack already full: the free list is inconsistent
                atomicSub(c.free_count, 1);
                raise_error(KVB_DERR_RANGE);
                continue;
            }
            c.free_pages[top] = c.table[(size_t)bg * c.max_pages + j];
            c.table[(size_t)bg * c.max_pages + j] = -1;
        }
        c.len[bg] = nn;
    }
}

// The empty cache: every page on the free stack (in page order), no table entry, len 0.
__global__ void paged_reset_kernel(const __grid_constant__ PagedCache c, int B) {
    const long long rows = (long long)B * c.Hkv;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < rows * c.max_pages || i < c.num_pages ||
                                                                         i < rows;
         i += (long long)gridDim.x * blockDim.x) {
        if (i < c.num_pages) c.free_pages[i] = (int)i;
        if (i < rows * c.max_pages) c.table[i] = -1;
        if (i < rows) c.len[i] = 0;
        if (i == 0) *c.free_count = c.num_pages;
    }
}

}  // namespace kvb
