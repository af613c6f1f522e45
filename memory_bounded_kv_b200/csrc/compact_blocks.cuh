// In-place removal of a slot range, as MEMENTO does when a thinking block's
// memento is complete (sections on chunking/compression and the dual
// information stream): the block's KV entries disappear and the entries
// after it slide down unchanged, byte for byte.
//
// One CTA per (sequence, kv head). The tail after the removed range is moved
// in chunks of W rows staged through shared memory: chunk c is read whole
// before any of it is written, and its destination lies below every later
// chunk's source, so overlapping moves (a tail longer than the removed
// range) are safe without a second buffer.
#pragma once

#include "common.cuh"

namespace kvb {

struct CompactParams {
    uint16_t* k;
    uint16_t* v;
    int* pos;
    float* lb;
    int* len;
    const int* rm_start;
    const int* rm_len;
    int Hkv, d, cap, W;
};

template <int NT>
__global__ void __launch_bounds__(NT) compact_blocks_kernel(const __grid_constant__ CompactParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int bg = blockIdx.x, b = bg / p.Hkv, tid = threadIdx.x;
    const int r0 = p.rm_start[b], rl = p.rm_len[b];
    if (rl == 0) return;
    const int n = p.len[bg];
    if (r0 < 0 || rl < 0 || n < 0 || n > p.cap || (long long)r0 + rl > n) {
        if (tid == 0) raise_error(KVB_DERR_RANGE);
        return;
    }
    const int tail = n - r0 - rl;
    const int vecs = p.d / 8;  // 16-byte vectors per row
    uint4* s_k = reinterpret_cast<uint4*>(smem);
    uint4* s_v = s_k + (size_t)p.W * vecs;
    int* s_pos = reinterpret_cast<int*>(s_v + (size_t)p.W * vecs);
    float* s_lb = reinterpret_cast<float*>(s_pos + p.W);
    uint4* gk = reinterpret_cast<uint4*>(p.k + (size_t)bg * p.cap * p.d);
    uint4* gv = reinterpret_cast<uint4*>(p.v + (size_t)bg * p.cap * p.d);
    int* gpos = p.pos + (size_t)bg * p.cap;
    float* glb = p.lb ? p.lb + (size_t)bg * p.cap : nullptr;
    for (int c0 = 0; c0 < tail; c0 += p.W) {
        const int w = min(p.W, tail - c0);
        const int src = r0 + rl + c0, dst = r0 + c0;
        for (int i = tid; i < w * vecs; i += NT) {
            s_k[i] = gk[(size_t)src * vecs + i];
            s_v[i] = gv[(size_t)src * vecs + i];
        }
        for (int i = tid; i < w; i += NT) {
            s_pos[i] = gpos[src + i];
            if (glb) s_lb[i] = glb[src + i];
        }
        __syncthreads();
        for (int i = tid; i < w * vecs; i += NT) {
            gk[(size_t)dst * vecs + i] = s_k[i];
            gv[(size_t)dst * vecs + i] = s_v[i];
        }
        for (int i = tid; i < w; i += NT) {
            gpos[dst + i] = s_pos[i];
            if (glb) glb[dst + i] = s_lb[i];
        }
        __syncthreads();
    }
    if (tid == 0) p.len[bg] = n - rl;
}

}  // namespace kvb
