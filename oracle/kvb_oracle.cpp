// CPU oracle for the memory-bounded KV decode path.
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
// CPU-baseline leg may load this code; the library never does. It shares no
// code, header, table or helper with the CUDA path.
//
// Plain, slow, single-threaded, double-precision definitions of what the
// path computes, written from these sources:
//   [TRIM] "Cache What Lasts: Token Retention for Memory-Bounded KV Cache in
//          LLMs", section 2.1 (retention-gated attention: weight of key i at
//          step t proportional to exp(q.k_i + (t - i) log beta_i); inference:
//          when the cache exceeds the budget M, evict the token whose
//          beta_i^(t - i) is lowest).
//   [ASM]  "Context Memorization for Efficient Long Context Generation",
//          core method steps 1-4 (attention state a = attn(q, K, V),
//          Z = sum_k exp(q.k / sqrt(d_h)); merge((a_A, Z_A), (a_B, Z_B)) =
//          ((Z_A a_A + Z_B a_B) / (Z_A + Z_B), Z_A + Z_B); retrieval
//          c* = argmax_k cos(q, qbar_k); merge of the retrieved state with the
//          query's own attention) and the online-softmax identity of its
//          background section.
//   [MEM]  "MEMENTO: Teaching LLMs to Manage Their Own Context", sections on
//          chunking/compression and the dual information stream (a finished
//          thinking block's KV entries are physically removed in place; the
//          memento entries that follow it are kept bit for bit).
//
// Readings where the sources are silent (each is a line of the design notes):
//   - logits carry the 1/sqrt(d) scale of [ASM] plus the retention bias of
//     [TRIM]: l_i = scale * q.k_i + (t - pos_i) * log beta_i;
//   - an attention state is kept as (o, lse) with lse = ln Z (natural log);
//   - the empty state is (o = 0, lse = -inf) and is the merge identity;
//   - the eviction score is one float32 product (float)(t - pos) * log beta,
//     ties go to the lower position, -0 equals +0; "lowest beta^(t-i)" is
//     the lowest score because log is monotone;
//   - GQA: query head h reads kv head floor(h / (Hq / Hkv));
//   - cos(x, y) = 0 when either vector has zero norm;
//   - t[b] < 0 marks an inactive sequence (no insertion, empty attention).
//
// Status codes: 0 = ok, 1 = invalid argument, 3 = invalid data (a length,
// position or range that the preconditions exclude).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

double bf16_value(uint16_t bits) {
    uint32_t u = static_cast<uint32_t>(bits) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return static_cast<double>(f);
}

// Attention state of one query over slots [s0, s1) of one kv head: the
// softmax-weighted mean of the values (a) and ln of the partition sum (Z).
void attention_state(const uint16_t* q, const uint16_t* K, const uint16_t* V,
                     const float* log_beta, const int32_t* pos, int64_t t,
                     int64_t s0, int64_t s1, int d, double scale,
                     double* a, double* lse) {
    for (int e = 0; e < d; ++e) a[e] = 0.0;
    if (s1 <= s0) {
        *lse = kNegInf;
        return;
    }
    std::vector<double> logit(static_cast<size_t>(s1 - s0));
    double m = kNegInf;
    for (int64_t s = s0; s < s1; ++s) {
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += bf16_value(q[e]) * bf16_value(K[s * d + e]);
        double l = scale * dot;
        if (log_beta != nullptr) {
            l += static_cast<double>(t - pos[s]) * static_cast<double>(log_beta[s]);
        }
        logit[s - s0] = l;
        if (l > m) m = l;
    }
    double z = 0.0;
    for (int64_t s = s0; s < s1; ++s) {
        double w = std::exp(logit[s - s0] - m);
        z += w;
        for (int e = 0; e < d; ++e) a[e] += w * bf16_value(V[s * d + e]);
    }
    for (int e = 0; e < d; ++e) a[e] /= z;
    *lse = m + std::log(z);
}

// merge of two states, [ASM] step 2, with Z carried as ln Z.
void merge_two(double* a, double* lse, const double* b_a, double b_lse, int d) {
    if (b_lse == kNegInf) return;
    if (*lse == kNegInf) {
        for (int e = 0; e < d; ++e) a[e] = b_a[e];
        *lse = b_lse;
        return;
    }
    double m = *lse > b_lse ? *lse : b_lse;
    double za = std::exp(*lse - m);
    double zb = std::exp(b_lse - m);
    for (int e = 0; e < d; ++e) a[e] = (za * a[e] + zb * b_a[e]) / (za + zb);
    *lse = m + std::log(za + zb);
}

// The split covering slot range j of a sequence with n valid slots.
void split_range(int64_t n, int S, int split_len, int j, int64_t* s0, int64_t* s1) {
    int64_t c = split_len > 0 ? split_len : (n + S - 1) / S;
    int64_t lo = static_cast<int64_t>(j) * c;
    int64_t hi = lo + c;
    if (lo > n) lo = n;
    if (hi > n) hi = n;
    *s0 = lo;
    *s1 = hi;
}

float eviction_score(int64_t t, int32_t pos, const float* log_beta, int64_t s) {
    if (log_beta == nullptr) return 0.0f;
    volatile float dt = static_cast<float>(t - pos);
    volatile float prod = dt * log_beta[s];
    float r = prod;
    if (r == 0.0f) r = 0.0f;  // -0 counts as +0
    return r;
}

}  // namespace

extern "C" {

// Decode attention, [TRIM] 2.1 logits with the [ASM] scale, [ASM] (a, Z) state.
//   q [B, Hq, d] (element strides q_sb, q_sh; d contiguous), bf16 bits
//   k, v [B, Hkv, cap, d] (strides kv_sb, kv_sh; slot stride d), bf16 bits
//   log_beta, pos [B, Hkv, cap] (strides m_sb, m_sh); log_beta may be null
//   len [B, Hkv], t [B] (t may be null when log_beta is null)
//   o [B, Hq, d], lse [B, Hq]: the state over all len slots (no splitting)
//   o_part [B, Hq, S, d], lse_part [B, Hq, S] (nullable): the state of each
//     split j, which covers slots [j*C, min((j+1)*C, len)) with
//     C = split_len if split_len > 0 else ceil(len / S).
int oracle_decode_attn(const uint16_t* q, int64_t q_sb, int64_t q_sh,
                       const uint16_t* k, const uint16_t* v, int64_t kv_sb, int64_t kv_sh,
                       const float* log_beta, const int32_t* pos, int64_t m_sb, int64_t m_sh,
                       const int32_t* len, const int32_t* t,
                       int B, int Hq, int Hkv, int d, int cap, double scale,
                       int S, int split_len,
                       double* o, double* lse, double* o_part, double* lse_part) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || cap < 0 || S < 1 || split_len < 0) return 1;
    if (Hq % Hkv != 0) return 1;
    if (log_beta != nullptr && (pos == nullptr || t == nullptr)) return 1;
    if (scale == 0.0) scale = 1.0 / std::sqrt(static_cast<double>(d));
    const int G = Hq / Hkv;
    int status = 0;
    std::vector<double> tmp(static_cast<size_t>(d));
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            const int64_t n = len[b * Hkv + g];
            const bool active = (t == nullptr) || (t[b] >= 0);
            const int64_t tb = (t == nullptr) ? 0 : t[b];
            const uint16_t* qv = q + b * q_sb + h * q_sh;
            const uint16_t* K = k + b * kv_sb + g * kv_sh;
            const uint16_t* V = v + b * kv_sb + g * kv_sh;
            const float* lb = log_beta ? log_beta + b * m_sb + g * m_sh : nullptr;
            const int32_t* ps = pos ? pos + b * m_sb + g * m_sh : nullptr;
            double* ob = o + (static_cast<int64_t>(b) * Hq + h) * d;
            double* lb_out = lse + static_cast<int64_t>(b) * Hq + h;
            bool bad = n < 0 || n > cap || (split_len > 0 && n > static_cast<int64_t>(S) * split_len);
            if (bad) status = 3;
            const int64_t nn = (!active || bad) ? 0 : n;
            attention_state(qv, K, V, lb, ps, tb, 0, nn, d, scale, ob, lb_out);
            if (o_part != nullptr && lse_part != nullptr) {
                for (int j = 0; j < S; ++j) {
                    int64_t s0, s1;
                    split_range(nn, S, split_len, j, &s0, &s1);
                    double* op = o_part + ((static_cast<int64_t>(b) * Hq + h) * S + j) * d;
                    double* lp = lse_part + (static_cast<int64_t>(b) * Hq + h) * S + j;
                    attention_state(qv, K, V, lb, ps, tb, s0, s1, d, scale, op, lp);
                }
            }
        }
    }
    return status;
}

// n-way merge of attention states, a left fold of [ASM] step 2's operator.
//   state j of row r: o_in[j*o_sn + r*o_sr + e], lse_in[j*l_sn + r*l_sr]
//   -> o_out [R, d], lse_out [R]
int oracle_merge_states(const double* o_in, const double* lse_in,
                        int64_t o_sn, int64_t o_sr, int64_t l_sn, int64_t l_sr,
                        int n, int R, int d, double* o_out, double* lse_out) {
    if (n < 0 || R < 0 || d <= 0) return 1;
    for (int r = 0; r < R; ++r) {
        double* a = o_out + static_cast<int64_t>(r) * d;
        double* l = lse_out + r;
        for (int e = 0; e < d; ++e) a[e] = 0.0;
        *l = kNegInf;
        for (int j = 0; j < n; ++j) {
            merge_two(a, l, o_in + j * o_sn + r * o_sr, lse_in[j * l_sn + r * l_sr], d);
        }
    }
    return 0;
}

// Budget enforcement, [TRIM] 2.1 inference, for every (b, g) in order:
//   t[b] < 0: inactive, nothing changes, victim = -1;
//   len < M:  the token goes to slot len, len += 1, victim = -1;
//   else:     victim = argmin over slots s < len of (score_s, pos_s), the
//             token overwrites that slot.
// The token's row is k_new/v_new [B, Hkv, d] (both may be null: only
// log_beta and pos are written), log_beta_new [B, Hkv] (ignored when
// log_beta is null), position t[b]. Cache layout [B, Hkv, cap, d] and
// [B, Hkv, cap], contiguous.
int oracle_evict_insert(uint16_t* k, uint16_t* v, float* log_beta, int32_t* pos, int32_t* len,
                        const uint16_t* k_new, const uint16_t* v_new, const float* log_beta_new,
                        const int32_t* t, int B, int Hkv, int d, int cap, int M,
                        int32_t* victim) {
    if (B < 0 || Hkv <= 0 || d <= 0 || cap <= 0 || M < 1 || M > cap) return 1;
    if ((k_new == nullptr) != (v_new == nullptr)) return 1;
    if (log_beta != nullptr && log_beta_new == nullptr) return 1;
    int status = 0;
    for (int b = 0; b < B; ++b) {
        for (int g = 0; g < Hkv; ++g) {
            const int64_t bg = static_cast<int64_t>(b) * Hkv + g;
            victim[bg] = -1;
            if (t[b] < 0) continue;
            const int64_t n = len[bg];
            if (n < 0 || n > cap) {
                status = 3;
                continue;
            }
            int32_t* ps = pos + bg * cap;
            const float* lb = log_beta ? log_beta + bg * cap : nullptr;
            int64_t slot;
            if (n < M) {
                slot = n;
                len[bg] = static_cast<int32_t>(n + 1);
            } else {
                int64_t best = 0;
                float best_score = eviction_score(t[b], ps[0], lb, 0);
                for (int64_t s = 1; s < n; ++s) {
                    float sc = eviction_score(t[b], ps[s], lb, s);
                    if (sc < best_score || (sc == best_score && ps[s] < ps[best])) {
                        best = s;
                        best_score = sc;
                    }
                }
                slot = best;
                victim[bg] = static_cast<int32_t>(best);
            }
            if (k_new != nullptr) {
                for (int e = 0; e < d; ++e) {
                    k[(bg * cap + slot) * d + e] = k_new[bg * d + e];
                    v[(bg * cap + slot) * d + e] = v_new[bg * d + e];
                }
            }
            if (log_beta != nullptr) log_beta[bg * cap + slot] = log_beta_new[bg];
            ps[slot] = t[b];
        }
    }
    return status;
}

// In-place block removal, [MEM]: for every sequence b with rm_len[b] > 0 and
// every kv head g, slots [r0, r0 + rl) are removed, later slots move down by
// rl in order with their bytes unchanged, and len[b, g] -= rl. A range that
// does not lie inside [0, len) leaves that head untouched (status 3).
int oracle_compact_blocks(uint16_t* k, uint16_t* v, int32_t* pos, float* log_beta, int32_t* len,
                          const int32_t* rm_start, const int32_t* rm_len,
                          int B, int Hkv, int d, int cap) {
    if (B < 0 || Hkv <= 0 || d <= 0 || cap <= 0) return 1;
    int status = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t r0 = rm_start[b], rl = rm_len[b];
        if (rl == 0) continue;
        for (int g = 0; g < Hkv; ++g) {
            const int64_t bg = static_cast<int64_t>(b) * Hkv + g;
            const int64_t n = len[bg];
            if (r0 < 0 || rl < 0 || n > cap || r0 + rl > n) {
                status = 3;
                continue;
            }
            for (int64_t s = r0 + rl; s < n; ++s) {
                const int64_t dst = s - rl;
                for (int e = 0; e < d; ++e) {
                    k[(bg * cap + dst) * d + e] = k[(bg * cap + s) * d + e];
                    v[(bg * cap + dst) * d + e] = v[(bg * cap + s) * d + e];
                }
                pos[bg * cap + dst] = pos[bg * cap + s];
                if (log_beta != nullptr) log_beta[bg * cap + dst] = log_beta[bg * cap + s];
            }
            len[bg] = static_cast<int32_t>(n - rl);
        }
    }
    return status;
}

// cos(q[n, h], qbar[h, kk]) for kk in [0, K) -> out[K]   ([ASM] step 3)
int oracle_asm_cosines(const uint16_t* q, const float* qbar, int N, int H, int K, int d,
                       int n, int h, double* out) {
    if (n < 0 || n >= N || h < 0 || h >= H || K < 1 || d <= 0) return 1;
    const uint16_t* qv = q + (static_cast<int64_t>(n) * H + h) * d;
    double qq = 0.0;
    for (int e = 0; e < d; ++e) qq += bf16_value(qv[e]) * bf16_value(qv[e]);
    for (int kk = 0; kk < K; ++kk) {
        const float* c = qbar + (static_cast<int64_t>(h) * K + kk) * d;
        double dot = 0.0, cc = 0.0;
        for (int e = 0; e < d; ++e) {
            dot += bf16_value(qv[e]) * static_cast<double>(c[e]);
            cc += static_cast<double>(c[e]) * static_cast<double>(c[e]);
        }
        out[kk] = (qq > 0.0 && cc > 0.0) ? dot / (std::sqrt(qq) * std::sqrt(cc)) : 0.0;
    }
    return 0;
}

// Attention-state-memory lookup and merge, [ASM] steps 3-4, per (n, h):
//   c* = argmax_k cos(q, qbar_k) (first index among equal maxima);
//   (o, lse) = merge((o_self, lse_self), (abar[c*], log_zbar[c*])).
//   q [N, H, d] bf16; qbar [H, K, d] f32; abar [H, K, d] bf16; log_zbar [H, K];
//   o_self [N, H, d], lse_self [N, H] -> idx [N, H], o [N, H, d], lse [N, H].
int oracle_asm_lookup_merge(const uint16_t* q, const float* qbar, const uint16_t* abar,
                            const float* log_zbar, const float* o_self, const float* lse_self,
                            int N, int H, int K, int d,
                            int32_t* idx, double* o, double* lse) {
    if (N < 0 || H <= 0 || K < 1 || d <= 0) return 1;
    std::vector<double> cosv(static_cast<size_t>(K));
    std::vector<double> mem(static_cast<size_t>(d));
    for (int n = 0; n < N; ++n) {
        for (int h = 0; h < H; ++h) {
            oracle_asm_cosines(q, qbar, N, H, K, d, n, h, cosv.data());
            int best = 0;
            for (int kk = 1; kk < K; ++kk) {
                if (cosv[kk] > cosv[best]) best = kk;
            }
            const int64_t nh = static_cast<int64_t>(n) * H + h;
            idx[nh] = best;
            double* a = o + nh * d;
            for (int e = 0; e < d; ++e) a[e] = static_cast<double>(o_self[nh * d + e]);
            lse[nh] = static_cast<double>(lse_self[nh]);
            const int64_t hk = static_cast<int64_t>(h) * K + best;
            for (int e = 0; e < d; ++e) mem[e] = bf16_value(abar[hk * d + e]);
            merge_two(a, &lse[nh], mem.data(), static_cast<double>(log_zbar[hk]), d);
        }
    }
    return 0;
}

// Two-level attention-state-memory lookup and merge ([ASM] hierarchical lookup index), per (n, h):
//   s_c = cos(q, qhat_c) for the C first-level centroids of head h;
//   S = the m clusters with the largest s_c (the lower c among equal values), m = min(m, C);
//   c* = argmax of cos(q, qbar_k) over the members k of the clusters in S (the lowest k among
//        equal values); no member at all: c* = -1 and the state is the self state;
//   (o, lse) = merge((o_self, lse_self), (abar[c*], log_zbar[c*])).
// Cluster c of head h holds members[h * K + i] for offsets[h * (C + 1) + c] <= i < offsets[... + c + 1].
//   qhat [H, C, d] f32; offsets [H, C + 1]; members [H, K] in [0, K); the rest as oracle_asm_lookup_merge
//   -> sel [N, H, m] (the selected clusters, best first), idx [N, H], o [N, H, d], lse [N, H].
int oracle_asm_hier_lookup_merge(const uint16_t* q, const float* qhat, const int32_t* offsets,
                                 const int32_t* members, const float* qbar, const uint16_t* abar,
                                 const float* log_zbar, const float* o_self, const float* lse_self,
                                 int N, int H, int K, int C, int m, int d,
                                 int32_t* sel, int32_t* idx, double* o, double* lse) {
    if (N < 0 || H <= 0 || K < 1 || C < 1 || m < 1 || d <= 0) return 1;
    const int mm = m < C ? m : C;
    std::vector<double> coarse(static_cast<size_t>(C)), cosk(static_cast<size_t>(K));
    std::vector<char> taken(static_cast<size_t>(C));
    std::vector<double> mem(static_cast<size_t>(d));
    for (int n = 0; n < N; ++n) {
        for (int h = 0; h < H; ++h) {
            oracle_asm_cosines(q, qhat, N, H, C, d, n, h, coarse.data());
            oracle_asm_cosines(q, qbar, N, H, K, d, n, h, cosk.data());
            const int64_t nh = static_cast<int64_t>(n) * H + h;
            std::fill(taken.begin(), taken.end(), 0);
            int best = -1;
            for (int j = 0; j < mm; ++j) {
                int c_sel = -1;   // the largest cosine not taken yet, the lower c on ties
                for (int c = 0; c < C; ++c)
                    if (!taken[c] && (c_sel < 0 || coarse[c] > coarse[c_sel])) c_sel = c;
                taken[c_sel] = 1;
                sel[nh * m + j] = c_sel;
                const int32_t* off = offsets + static_cast<int64_t>(h) * (C + 1);
                if (off[c_sel] < 0 || off[c_sel + 1] > K) return 2;
                for (int32_t i = off[c_sel]; i < off[c_sel + 1]; ++i) {
                    const int32_t kk = members[static_cast<int64_t>(h) * K + i];
                    if (kk < 0 || kk >= K) return 2;
                    if (best < 0 || cosk[kk] > cosk[best] || (cosk[kk] == cosk[best] && kk < best)) best = kk;
                }
            }
            for (int j = mm; j < m; ++j) sel[nh * m + j] = -1;
            idx[nh] = best;
            double* a = o + nh * d;
            for (int e = 0; e < d; ++e) a[e] = static_cast<double>(o_self[nh * d + e]);
            lse[nh] = static_cast<double>(lse_self[nh]);
            if (best < 0) continue;
            const int64_t hk = static_cast<int64_t>(h) * K + best;
            for (int e = 0; e < d; ++e) mem[e] = bf16_value(abar[hk * d + e]);
            merge_two(a, &lse[nh], mem.data(), static_cast<double>(log_zbar[hk]), d);
        }
    }
    return 0;
}

// ---- parallel driver ------------------------------------------------------
// Runs `steps` decode steps -- budget enforcement + insertion
// (oracle_evict_insert), then attention (oracle_decode_attn, one split) -- for
// every (sequence b, kv head g) unit, spreading the units over `nthreads`
// threads (0 = every host core). Units are independent: each thread calls the
// single-threaded functions above, unchanged, on one unit's slice (B = 1,
// Hkv = 1, the unit's G query heads), so the results are the ones a serial
// call over the whole batch gives. Only the bench's CPU baseline and the
// tests use it, to spread long replays over the host's cores.
//   cache: k, v [B, Hkv, cap, d], log_beta (nullable), pos [B, Hkv, cap],
//          len [B, Hkv], contiguous, updated in place
//   per step s: q [steps, B, Hq, d] (null: no attention), k_new, v_new
//          [steps, B, Hkv, d] (both null: only log_beta and pos are written),
//          log_beta_new [steps, B, Hkv] (ignored when log_beta is null),
//          t [steps, B]
//   victim [steps, B, Hkv] (nullable); o [B, Hq, d], lse [B, Hq] (nullable):
//          the last step's attention state
// Returns the first nonzero status of any call (0 = ok).
int oracle_decode_steps_threads(uint16_t* k, uint16_t* v, float* log_beta, int32_t* pos, int32_t* len,
                                const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                const float* log_beta_new, const int32_t* t, int steps, int B, int Hq,
                                int Hkv, int d, int cap, int M, int nthreads, int32_t* victim, double* o,
                                double* lse) {
    if (steps < 0 || B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || cap <= 0) return 1;
    if (q != nullptr && (o == nullptr || lse == nullptr)) return 1;
    const int G = Hq / Hkv;
    const int64_t units = static_cast<int64_t>(B) * Hkv;
    int nt = nthreads > 0 ? nthreads : static_cast<int>(std::thread::hardware_concurrency());
    if (nt < 1) nt = 1;
    if (nt > units) nt = static_cast<int>(units > 0 ? units : 1);
    std::vector<int> status(static_cast<size_t>(nt), 0);
    auto work = [&](int w) {
        for (int64_t u = w; u < units; u += nt) {
            const int64_t b = u / Hkv, g = u % Hkv;
            uint16_t* ku = k + u * cap * d;
            uint16_t* vu = v + u * cap * d;
            float* lbu = log_beta ? log_beta + u * cap : nullptr;
            int32_t* pu = pos + u * cap;
            int32_t* lu = len + u;
            for (int s = 0; s < steps; ++s) {
                const int64_t sb = static_cast<int64_t>(s) * B + b;   // (step, sequence)
                const int64_t su = static_cast<int64_t>(s) * units + u;  // (step, unit)
                int32_t vic = -1;
                int st = oracle_evict_insert(ku, vu, lbu, pu, lu, k_new ? k_new + su * d : nullptr,
                                             v_new ? v_new + su * d : nullptr,
                                             log_beta_new ? log_beta_new + su : nullptr, t + sb, 1, 1, d, cap, M,
                                             &vic);
                if (victim != nullptr) victim[su] = vic;
                if (st != 0 && status[w] == 0) status[w] = st;
                if (q == nullptr) continue;
                const uint16_t* qu = q + (sb * Hq + g * G) * d;
                st = oracle_decode_attn(qu, static_cast<int64_t>(Hq) * d, d, ku, vu, static_cast<int64_t>(cap) * d,
                                        static_cast<int64_t>(cap) * d, lbu, pu, cap, cap, lu, t + sb, 1, G, 1, d, cap,
                                        0.0, 1, 0, o + (b * Hq + g * G) * d, lse + b * Hq + g * G, nullptr, nullptr);
                if (st != 0 && status[w] == 0) status[w] = st;
            }
        }
    };
    std::vector<std::thread> pool;
    for (int w = 1; w < nt; ++w) pool.emplace_back(work, w);
    work(0);
    for (auto& th : pool) th.join();
    for (int st : status)
        if (st != 0) return st;
    return 0;
}

}  // extern "C"
