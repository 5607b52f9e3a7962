// ra_oracle.cpp -- plain, slow fp64 CPU oracle for ring-chunked attention, the
// log-sum-exp merge and the Ulysses layout transforms.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
// baseline leg of the benchmark load this library.  It shares no code, header,
// table or helper with the CUDA library; the two see the same inputs only.
//
// Sources (cited by page title and section):
//   [SP-QA]    "Как работает sequence parallelism в контексте LLM?":
//              section 2 (contiguous chunking: rank i owns tokens
//              i*L/P .. (i+1)*L/P-1), section 3 (the ring: each step a rank
//              attends its queries to the K/V chunk it holds, passes that chunk
//              on and receives the previous rank's; P-1 exchanges), section 5
//              (per-chunk scores, row max, exp, sum, the online-softmax merge,
//              final division by the normaliser).
//   [ULYSSES]  "Метод контекстного параллелизма Ulysses": all-to-all from
//              [local_seqlen, global_heads, head_dim] to
//              [global_seqlen, local_heads, head_dim] and back; GQA KV heads
//              copied up to the CP-group size.
//
// Readings taken where the pages are silent or inconsistent (each is listed
// with its reason in the design notes of the repository):
//   * scores are multiplied by an explicit `scale` (the pseudocode has none);
//   * "lse" is the true natural-log log-sum-exp of the scaled scores, not the
//     row max the pseudocode stores under that name;
//   * the merge of two partials is the exact log-sum-exp combination
//       lse = log(e^lse_a + e^lse_b), o = e^(lse_a-lse) o_a + e^(lse_b-lse) o_b
//     (the pseudocode's update reuses the first step's weights and drops the
//     factor on the new term);
//   * at ring step s, rank i holds chunk (i - s) mod P (the stated intent of
//     section 3; the pseudocode re-sends its own chunk every step);
//   * causal masking, absent from the pages, is the global mask over the
//     concatenation of chunks in rank order, key position <= query position;
//   * GQA: query head h reads kv head h / (H_q / H_kv);
//   * the zigzag layout, only named in [ULYSSES] (introduction), is 2P segments of
//     Lc/2 tokens with rank i holding segment i then segment 2P-1-i; the causal mask
//     compares sequence positions, not rank-major indices;
//   * packed samples ([ACCEL-SP], position_ids instead of an attention mask): samples
//     are contiguous, position_ids count 0, 1, 2, ... within each, and a query sees
//     only the keys of its own sample (causal: those not after it);
//   * the backward pass is the derivative of the definition (the pages train with the
//     method but print no gradient formula); GQA gradients of a kv head sum over its
//     query heads;
//   * Ulysses rank r receives the contiguous head block [r*H/P, (r+1)*H/P),
//     the global sequence is source-rank-major, and KV replica j of H_out is
//     source head floor(j * H_in / H_out).
//
// Everything is fp64.  Inputs arrive as fp64 arrays holding the exact values
// of the bf16/fp32 inputs.  Threads (std::thread) split independent query rows;
// each row is computed by the same sequential loop whatever the thread count.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

const double NEG_INF = -std::numeric_limits<double>::infinity();

int pick_threads(int requested, long long work_items) {
    int n = requested > 0 ? requested : (int)std::thread::hardware_concurrency();
    if (n < 1) n = 1;
    if ((long long)n > work_items) n = (int)std::max<long long>(1, work_items);
    return n;
}

template <class F>
void parallel_for(long long n_items, int nthreads, F body) {
    int nt = pick_threads(nthreads, n_items);
    if (nt == 1) {
        for (long long i = 0; i < n_items; ++i) body(i);
        return;
    }
    std::vector<std::thread> pool;
    pool.reserve(nt);
    for (int w = 0; w < nt; ++w) {
        pool.emplace_back([=]() {
            for (long long i = w; i < n_items; i += nt) body(i);
        });
    }
    for (auto& th : pool) th.join();
}

// Attention of one query vector against keys [key_begin, key_end) of one
// (batch, kv head) sequence, by the plain definition ([SP-QA] section 5,
// read with the true log-sum-exp):
//   s_j = scale * <q, k_j>;  lse = log sum_j exp(s_j);  o = sum_j exp(s_j - lse) v_j
// `key_visible(j)` decides the mask.  With no visible key: o = 0, lse = -inf.
// k, v point at token 0 of the sequence, consecutive tokens `tok_stride` apart.
template <class Visible>
void attend_one(const double* qv, const double* k, const double* v, long long tok_stride,
                long long key_begin, long long key_end, int D, double scale, Visible key_visible,
                std::vector<double>& s, double* o, double* lse_out) {
    s.assign((size_t)std::max<long long>(0, key_end - key_begin), NEG_INF);
    double m = NEG_INF;
    for (long long j = key_begin; j < key_end; ++j) {
        if (!key_visible(j)) continue;
        const double* kj = k + j * tok_stride;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qv[d] * kj[d];
        double sj = scale * dot;
        s[(size_t)(j - key_begin)] = sj;
        if (sj > m) m = sj;
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (m == NEG_INF) {  // no visible key
        *lse_out = NEG_INF;
        return;
    }
    double sum = 0.0;
    for (long long j = key_begin; j < key_end; ++j) {
        double sj = s[(size_t)(j - key_begin)];
        if (sj == NEG_INF) continue;
        sum += std::exp(sj - m);
    }
    double lse = m + std::log(sum);
    for (long long j = key_begin; j < key_end; ++j) {
        double sj = s[(size_t)(j - key_begin)];
        if (sj == NEG_INF) continue;
        double w = std::exp(sj - lse);
        const double* vj = v + j * tok_stride;
        for (int d = 0; d < D; ++d) o[d] += w * vj[d];
    }
    *lse_out = lse;
}

// The exact merge of two partials over disjoint key sets ([SP-QA] section 5,
// merge step).  (o_a, lse_a) <- (o_a, lse_a) (+) (o_b, lse_b).
void merge_into(double* o_a, double* lse_a, const double* o_b, double lse_b, int D) {
    double la = *lse_a;
    if (lse_b == NEG_INF) {
        if (la == NEG_INF)
            for (int d = 0; d < D; ++d) o_a[d] = 0.0;
        return;
    }
    if (la == NEG_INF) {
        for (int d = 0; d < D; ++d) o_a[d] = o_b[d];
        *lse_a = lse_b;
        return;
    }
    double mx = std::max(la, lse_b);
    double lse = mx + std::log(std::exp(la - mx) + std::exp(lse_b - mx));
    double wa = std::exp(la - lse), wb = std::exp(lse_b - lse);
    for (int d = 0; d < D; ++d) o_a[d] = wa * o_a[d] + wb * o_b[d];
    *lse_a = lse;
}

}  // namespace

extern "C" {

// Plain (unchunked) attention, the definition every other form must equal.
//   q   [B][L][H_q][D]     k, v [B][L][H_kv][D]
//   out [B][L][H_q][D]     lse  [B][H_q][L]
int ora_attention(const double* q, const double* k, const double* v, int B, long long L, int H_q,
                  int H_kv, int D, double scale, int causal, double* out, double* lse,
                  int nthreads) {
    if (B < 1 || L < 1 || H_q < 1 || H_kv < 1 || D < 1 || H_q % H_kv != 0) return 1;
    const int group = H_q / H_kv;
    const long long n_rows = (long long)B * H_q * L;
    parallel_for(n_rows, nthreads, [&](long long row) {
        thread_local std::vector<double> s;
        const long long t = row % L;
        const int h = (int)((row / L) % H_q);
        const int b = (int)(row / L / H_q);
        const int g = h / group;
        const double* qv = q + (((long long)b * L + t) * H_q + h) * D;
        const double* kb = k + ((long long)b * L * H_kv + g) * D;
        const double* vb = v + ((long long)b * L * H_kv + g) * D;
        double* o = out + (((long long)b * L + t) * H_q + h) * D;
        auto visible = [&](long long j) { return !causal || j <= t; };
        attend_one(qv, kb, vb, (long long)H_kv * D, 0, L, D, scale, visible, s, o,
                   lse + ((long long)b * H_q + h) * L + t);
    });
    return 0;
}

// The same definition for a sample of query rows (b_i, t_i, h_i), for parity
// checks at sizes where computing every row is too slow.
//   q_rows [n][D] (the sampled query vectors)   k, v [B][L][H_kv][D]
//   out [n][D]   lse [n]
int ora_attention_rows(const double* q_rows, const int* rb, const long long* rt, const int* rh,
                       long long n, const double* k, const double* v, int B, long long L, int H_q,
                       int H_kv, int D, double scale, int causal, double* out, double* lse,
                       int nthreads) {
    if (B < 1 || L < 1 || H_q < 1 || H_kv < 1 || D < 1 || H_q % H_kv != 0) return 1;
    for (long long i = 0; i < n; ++i)
        if (rb[i] < 0 || rb[i] >= B || rt[i] < 0 || rt[i] >= L || rh[i] < 0 || rh[i] >= H_q)
            return 1;
    const int group = H_q / H_kv;
    parallel_for(n, nthreads, [&](long long i) {
        thread_local std::vector<double> s;
        const long long t = rt[i];
        const int g = rh[i] / group;
        const double* kb = k + ((long long)rb[i] * L * H_kv + g) * D;
        const double* vb = v + ((long long)rb[i] * L * H_kv + g) * D;
        auto visible = [&](long long j) { return !causal || j <= t; };
        attend_one(q_rows + i * D, kb, vb, (long long)H_kv * D, 0, L, D, scale, visible, s,
                   out + i * D, lse + i);
    });
    return 0;
}

// The ring form ([SP-QA] sections 2, 3, 5): queries of rank i attend, at step
// s = 0..P-1, to the chunk j = (i - step_offset[s]) mod P, and each partial is
// merged into the running result.  step_offset == NULL means the ring order
// step_offset[s] = s.  Any permutation of 0..P-1 gives another visiting order.
// `pos` gives the global sequence position of each of the P*Lc tokens in rank-major
// order (rank j's shard is tokens j*Lc .. j*Lc+Lc-1 of q and chunk j of k/v); the causal
// mask is pos[key] <= pos[query].  pos == NULL is the contiguous layout of [SP-QA]
// section 2 (pos[t] = t); any permutation of 0..P*Lc-1 is another assignment of
// sequence positions to shards (the zigzag layout is one, see ora_zigzag_positions).
// `lo` (NULL: none) gives, per batch row and rank-major token, the smallest key
// position its query may see: packed samples ([ACCEL-SP] section "Configuración del
// backend SP de ALST/Ulysses": several samples combined into one sequence, told apart by
// position_ids; see ora_packed_lower_bounds).
//   q  [B][P*Lc][H_q][D]    k, v [P][B][Lc][H_kv][D] (chunk j = rank j's K/V)
//   lo [B][P*Lc]
//   out [B][P*Lc][H_q][D]   lse [B][H_q][P*Lc]
int ora_ring_attention(const double* q, const double* k_chunks, const double* v_chunks, int P,
                       int B, long long Lc, int H_q, int H_kv, int D, double scale, int causal,
                       const int* step_offset, const long long* pos, const long long* lo,
                       double* out, double* lse, int nthreads) {
    if (P < 1 || B < 1 || Lc < 1 || H_q < 1 || H_kv < 1 || D < 1 || H_q % H_kv != 0) return 1;
    if (step_offset) {
        std::vector<int> seen(P, 0);
        for (int s = 0; s < P; ++s) {
            if (step_offset[s] < 0 || step_offset[s] >= P || seen[step_offset[s]]) return 1;
            seen[step_offset[s]] = 1;
        }
    }
    const long long L = (long long)P * Lc;
    if (pos) {
        std::vector<char> seen(L, 0);
        for (long long t = 0; t < L; ++t) {
            if (pos[t] < 0 || pos[t] >= L || seen[pos[t]]) return 1;
            seen[pos[t]] = 1;
        }
    }
    auto position = [&](long long t) { return pos ? pos[t] : t; };
    const int group = H_q / H_kv;
    const long long chunk_elems = (long long)B * Lc * H_kv * D;
    const long long n_rows = (long long)B * H_q * L;
    parallel_for(n_rows, nthreads, [&](long long row) {
        thread_local std::vector<double> s;
        thread_local std::vector<double> o_part;
        const long long t = row % L;
        const int h = (int)((row / L) % H_q);
        const int b = (int)(row / L / H_q);
        const int g = h / group;
        const int i = (int)(t / Lc);  // rank owning this query
        const double* qv = q + (((long long)b * L + t) * H_q + h) * D;
        double* o = out + (((long long)b * L + t) * H_q + h) * D;
        double* l = lse + ((long long)b * H_q + h) * L + t;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        *l = NEG_INF;
        o_part.assign(D, 0.0);
        for (int step = 0; step < P; ++step) {
            const int off = step_offset ? step_offset[step] : step;
            const int j = ((i - off) % P + P) % P;
            const double* kc = k_chunks + j * chunk_elems + ((long long)b * Lc * H_kv + g) * D;
            const double* vc = v_chunks + j * chunk_elems + ((long long)b * Lc * H_kv + g) * D;
            const long long key0 = (long long)j * Lc;  // rank-major index of the chunk's first key
            const long long qpos = position(t);
            const long long qlo = lo ? lo[(long long)b * L + t] : 0;
            auto visible = [&](long long c) {
                const long long kp = position(key0 + c);
                return (!causal || kp <= qpos) && kp >= qlo;
            };
            double lse_part;
            attend_one(qv, kc, vc, (long long)H_kv * D, 0, Lc, D, scale, visible, s,
                       o_part.data(), &lse_part);
            merge_into(o, l, o_part.data(), lse_part, D);
        }
    });
    return 0;
}

// The gradient of plain attention (the backward pass of the method: [SP-QA] trains the
// model, which needs d/dQ, d/dK, d/dV of O = softmax(scale Q K^T) V; the pages give no
// formula, so this is the derivative of the definition, written out):
//   P_ij  = exp(s_ij - lse_i),  s_ij = scale q_i . k_j  (visible j)
//   dP_ij = dO_i . v_j,          Delta_i = dO_i . O_i = sum_j P_ij dP_ij
//   dS_ij = P_ij (dP_ij - Delta_i)
//   dQ_i  = scale sum_j dS_ij k_j
//   dK_j  = scale sum_{i, h in j's group} dS_ij q_i,   dV_j = sum_{i, h} P_ij dO_i
// Three passes, each parallel over independent rows: the forward (lse_i, O_i, Delta_i),
// dQ per query row, dK and dV per (key row, kv head).
//   q, dout, dq [B][L][H_q][D]    k, v, dk, dv [B][L][H_kv][D]
int ora_attention_backward(const double* q, const double* k, const double* v,
                           const double* dout, int B, long long L, int H_q, int H_kv, int D,
                           double scale, int causal, double* dq, double* dk, double* dv,
                           int nthreads) {
    if (B < 1 || L < 1 || H_q < 1 || H_kv < 1 || D < 1 || H_q % H_kv != 0) return 1;
    const int group = H_q / H_kv;
    const long long n_rows = (long long)B * H_q * L;
    std::vector<double> lse(n_rows), delta(n_rows);
    auto qrow = [&](int b, long long t, int h) { return q + (((long long)b * L + t) * H_q + h) * D; };
    auto krow = [&](const double* x, int b, long long t, int g) {
        return x + (((long long)b * L + t) * H_kv + g) * D;
    };
    auto dot = [&](const double* a, const double* c) {
        double r = 0.0;
        for (int d = 0; d < D; ++d) r += a[d] * c[d];
        return r;
    };
    // pass 1: lse_i and Delta_i = dO_i . O_i
    parallel_for(n_rows, nthreads, [&](long long row) {
        thread_local std::vector<double> s, o;
        const long long t = row % L;
        const int h = (int)((row / L) % H_q), b = (int)(row / L / H_q), g = h / group;
        o.assign(D, 0.0);
        auto visible = [&](long long j) { return !causal || j <= t; };
        double l;
        attend_one(qrow(b, t, h), krow(k, b, 0, g), krow(v, b, 0, g), (long long)H_kv * D, 0, L,
                   D, scale, visible, s, o.data(), &l);
        lse[row] = l;
        delta[row] = dot(dout + (((long long)b * L + t) * H_q + h) * D, o.data());
    });
    auto P = [&](long long row, const double* qv, const double* kv) {
        return std::exp(scale * dot(qv, kv) - lse[row]);
    };
    // pass 2: dQ
    parallel_for(n_rows, nthreads, [&](long long row) {
        const long long t = row % L;
        const int h = (int)((row / L) % H_q), b = (int)(row / L / H_q), g = h / group;
        const double* qv = qrow(b, t, h);
        const double* dov = dout + (((long long)b * L + t) * H_q + h) * D;
        double* dqv = dq + (((long long)b * L + t) * H_q + h) * D;
        for (int d = 0; d < D; ++d) dqv[d] = 0.0;
        const long long jend = causal ? t + 1 : L;
        for (long long j = 0; j < jend; ++j) {
            const double p = P(row, qv, krow(k, b, j, g));
            const double ds = p * (dot(dov, krow(v, b, j, g)) - delta[row]);
            const double* kj = krow(k, b, j, g);
            for (int d = 0; d < D; ++d) dqv[d] += scale * ds * kj[d];
        }
    });
    // pass 3: dK, dV per (b, key j, kv head g)
    const long long n_keys = (long long)B * H_kv * L;
    parallel_for(n_keys, nthreads, [&](long long kr) {
        const long long j = kr % L;
        const int g = (int)((kr / L) % H_kv), b = (int)(kr / L / H_kv);
        double* dkv = const_cast<double*>(krow(dk, b, j, g));
        double* dvv = const_cast<double*>(krow(dv, b, j, g));
        for (int d = 0; d < D; ++d) dkv[d] = dvv[d] = 0.0;
        const double* kj = krow(k, b, j, g);
        const double* vj = krow(v, b, j, g);
        for (int h = g * group; h < (g + 1) * group; ++h)
            for (long long t = causal ? j : 0; t < L; ++t) {
                const long long row = ((long long)b * H_q + h) * L + t;
                const double* qv = qrow(b, t, h);
                const double* dov = dout + (((long long)b * L + t) * H_q + h) * D;
                const double p = P(row, qv, kj);
                const double ds = p * (dot(dov, vj) - delta[row]);
                for (int d = 0; d < D; ++d) {
                    dkv[d] += scale * ds * qv[d];
                    dvv[d] += p * dov[d];
                }
            }
    });
    return 0;
}

// One ring step's share of the gradients: the query rows of one chunk (Lq tokens) against the
// keys of one chunk (Lk tokens), with the softmax statistics of the WHOLE sequence given --
// out and lse are the forward's final output rows and log-sum-exps of these queries (the
// ring backward of "Как работает sequence parallelism в контексте LLM?", section 5, carried
// to the gradient: each step reuses the final LSE instead of recomputing a softmax).
//   P_ij = exp(scale q_i.k_j - lse_i),  Delta_i = dout_i . out_i,
//   dS_ij = P_ij (dout_i . v_j - Delta_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dout_i
// over the pairs (i, j) the step attends: every pair, or with causal (the chunk's own keys,
// Lq == Lk) only j <= i.  q, out, dout [B][Lq][H_q][D], lse [B][H_q][Lq], k, v
// [B][Lk][H_kv][D]; dq [B][Lq][H_q][D], dk, dv [B][Lk][H_kv][D] are written.  Summed over
// the chunks of the sequence, the shares are the gradients of ora_attention_backward.
int ora_attention_backward_pair(const double* q, const double* k, const double* v,
                                const double* out, const double* lse, const double* dout, int B,
                                long long Lq, long long Lk, int H_q, int H_kv, int D,
                                double scale, int causal, double* dq, double* dk, double* dv,
                                int nthreads) {
    if (B < 1 || Lq < 1 || Lk < 1 || H_q < 1 || H_kv < 1 || D < 1 || H_q % H_kv != 0) return 1;
    if (causal && Lq != Lk) return 1;
    const int group = H_q / H_kv;
    auto qoff = [&](int b, long long t, int h) { return (((long long)b * Lq + t) * H_q + h) * D; };
    auto koff = [&](int b, long long t, int g) { return (((long long)b * Lk + t) * H_kv + g) * D; };
    auto dot = [&](const double* a, const double* c) {
        double r = 0.0;
        for (int d = 0; d < D; ++d) r += a[d] * c[d];
        return r;
    };
    auto delta = [&](int b, long long t, int h) { return dot(dout + qoff(b, t, h), out + qoff(b, t, h)); };
    auto lse_of = [&](int b, long long t, int h) { return lse[((long long)b * H_q + h) * Lq + t]; };
    // dQ per query row
    const long long n_rows = (long long)B * Lq * H_q;
    parallel_for(n_rows, nthreads, [&](long long row) {
        const int h = (int)(row % H_q);
        const long long t = (row / H_q) % Lq;
        const int b = (int)(row / H_q / Lq), g = h / group;
        const double* qv = q + qoff(b, t, h);
        const double* dov = dout + qoff(b, t, h);
        const double dl = delta(b, t, h), l = lse_of(b, t, h);
        double* dqv = dq + qoff(b, t, h);
        for (int d = 0; d < D; ++d) dqv[d] = 0.0;
        const long long jend = causal ? t + 1 : Lk;
        for (long long j = 0; j < jend; ++j) {
            const double* kj = k + koff(b, j, g);
            const double p = std::exp(scale * dot(qv, kj) - l);
            const double ds = p * (dot(dov, v + koff(b, j, g)) - dl);
            for (int d = 0; d < D; ++d) dqv[d] += scale * ds * kj[d];
        }
    });
    // dK, dV per key row, summed over the query heads of its group
    const long long n_keys = (long long)B * Lk * H_kv;
    parallel_for(n_keys, nthreads, [&](long long kr) {
        const int g = (int)(kr % H_kv);
        const long long j = (kr / H_kv) % Lk;
        const int b = (int)(kr / H_kv / Lk);
        const double* kj = k + koff(b, j, g);
        const double* vj = v + koff(b, j, g);
        double* dkv = dk + koff(b, j, g);
        double* dvv = dv + koff(b, j, g);
        for (int d = 0; d < D; ++d) dkv[d] = dvv[d] = 0.0;
        for (int h = g * group; h < (g + 1) * group; ++h)
            for (long long t = causal ? j : 0; t < Lq; ++t) {
                const double* qv = q + qoff(b, t, h);
                const double* dov = dout + qoff(b, t, h);
                const double p = std::exp(scale * dot(qv, kj) - lse_of(b, t, h));
                const double ds = p * (dot(dov, vj) - delta(b, t, h));
                for (int d = 0; d < D; ++d) {
                    dkv[d] += scale * ds * qv[d];
                    dvv[d] += p * dov[d];
                }
            }
    });
    return 0;
}

// The same gradients for a sample of rows, at sizes where every row is too slow: dQ of
// the query rows (qb, qt, qh) and dK, dV of the key rows (kb, kt, kg).  Tokens are given
// in storage order; `pos` (NULL: pos[t] = t) gives the sequence position of each stored
// token and `lo` (NULL: none) the smallest key position each query of each batch row may
// see, as in ora_ring_attention, so one function serves the contiguous and zigzag shard
// layouts and packed samples.  Visibility of key j to query t (same batch row b):
//   (!causal || pos[j] <= pos[t]) && pos[j] >= lo[b][t].
// The formulas are those of ora_attention_backward.  A key row's dK, dV sum over every
// query row of its kv group that sees it, which needs lse and Delta of all those rows:
// pass 1 computes them for every row of each (b, h) with a sampled key row of its group,
// and for the sampled query rows.  A row that sees no key has P = 0 everywhere.
//   q, dout [B][L][H_q][D]   k, v [B][L][H_kv][D]   lo [B][L]   pos [L]
//   dq_rows [nq][D]   dk_rows, dv_rows [nk][D]
int ora_attention_backward_rows(const double* q, const double* k, const double* v,
                                const double* dout, int B, long long L, int H_q, int H_kv, int D,
                                double scale, int causal, const long long* pos,
                                const long long* lo, long long nq, const int* qb,
                                const long long* qt, const int* qh, long long nk, const int* kb,
                                const long long* kt, const int* kg, double* dq_rows,
                                double* dk_rows, double* dv_rows, int nthreads) {
    if (B < 1 || L < 1 || H_q < 1 || H_kv < 1 || D < 1 || H_q % H_kv != 0 || nq < 0 || nk < 0)
        return 1;
    for (long long i = 0; i < nq; ++i)
        if (qb[i] < 0 || qb[i] >= B || qt[i] < 0 || qt[i] >= L || qh[i] < 0 || qh[i] >= H_q)
            return 1;
    for (long long i = 0; i < nk; ++i)
        if (kb[i] < 0 || kb[i] >= B || kt[i] < 0 || kt[i] >= L || kg[i] < 0 || kg[i] >= H_kv)
            return 1;
    if (pos) {
        std::vector<char> seen(L, 0);
        for (long long t = 0; t < L; ++t) {
            if (pos[t] < 0 || pos[t] >= L || seen[pos[t]]) return 1;
            seen[pos[t]] = 1;
        }
    }
    const int group = H_q / H_kv;
    auto position = [&](long long t) { return pos ? pos[t] : t; };
    auto visible = [&](int b, long long t, long long j) {
        const long long kp = position(j);
        return (!causal || kp <= position(t)) && kp >= (lo ? lo[(long long)b * L + t] : 0);
    };
    auto qrow = [&](const double* x, int b, long long t, int h) {
        return x + (((long long)b * L + t) * H_q + h) * D;
    };
    auto krow = [&](const double* x, int b, long long t, int g) {
        return x + (((long long)b * L + t) * H_kv + g) * D;
    };
    auto dot = [&](const double* a, const double* c) {
        double r = 0.0;
        for (int d = 0; d < D; ++d) r += a[d] * c[d];
        return r;
    };
    // pass 1: which rows need lse and Delta, then compute them (lse_i and O_i by the
    // definition, Delta_i = dO_i . O_i)
    const long long n_rows = (long long)B * H_q * L;  // row index ((b * H_q + h) * L + t)
    std::vector<char> need(n_rows, 0);
    std::vector<char> whole_seq((size_t)B * H_q, 0);
    for (long long i = 0; i < nk; ++i)
        for (int h = kg[i] * group; h < (kg[i] + 1) * group; ++h)
            whole_seq[(size_t)kb[i] * H_q + h] = 1;
    for (long long r = 0; r < n_rows; ++r)
        if (whole_seq[(size_t)(r / L)]) need[r] = 1;
    for (long long i = 0; i < nq; ++i) need[((long long)qb[i] * H_q + qh[i]) * L + qt[i]] = 1;
    std::vector<long long> rows;
    for (long long r = 0; r < n_rows; ++r)
        if (need[r]) rows.push_back(r);
    std::vector<double> lse(n_rows, NEG_INF), delta(n_rows, 0.0);
    parallel_for((long long)rows.size(), nthreads, [&](long long ri) {
        thread_local std::vector<double> s, o;
        const long long row = rows[(size_t)ri];
        const long long t = row % L;
        const int h = (int)((row / L) % H_q), b = (int)(row / L / H_q), g = h / group;
        o.assign(D, 0.0);
        double l;
        attend_one(qrow(q, b, t, h), krow(k, b, 0, g), krow(v, b, 0, g), (long long)H_kv * D, 0,
                   L, D, scale, [&](long long j) { return visible(b, t, j); }, s, o.data(), &l);
        lse[row] = l;
        delta[row] = dot(qrow(dout, b, t, h), o.data());
    });
    // P_ij and dS_ij of one (query row, key) pair
    auto p_ds = [&](long long row, int b, long long t, int h, long long j, double* p,
                    double* ds) {
        const int g = h / group;
        *p = std::exp(scale * dot(qrow(q, b, t, h), krow(k, b, j, g)) - lse[row]);
        *ds = *p * (dot(qrow(dout, b, t, h), krow(v, b, j, g)) - delta[row]);
    };
    // pass 2: dQ of the sampled query rows
    parallel_for(nq, nthreads, [&](long long i) {
        const int b = qb[i], h = qh[i], g = h / group;
        const long long t = qt[i], row = ((long long)b * H_q + h) * L + t;
        double* dqv = dq_rows + i * D;
        for (int d = 0; d < D; ++d) dqv[d] = 0.0;
        for (long long j = 0; j < L; ++j) {
            if (!visible(b, t, j)) continue;
            double p, ds;
            p_ds(row, b, t, h, j, &p, &ds);
            const double* kj = krow(k, b, j, g);
            for (int d = 0; d < D; ++d) dqv[d] += scale * ds * kj[d];
        }
    });
    // pass 3: dK, dV of the sampled key rows, over every query head of the group and every
    // query row that sees the key
    parallel_for(nk, nthreads, [&](long long i) {
        const int b = kb[i], g = kg[i];
        const long long j = kt[i];
        double* dkv = dk_rows + i * D;
        double* dvv = dv_rows + i * D;
        for (int d = 0; d < D; ++d) dkv[d] = dvv[d] = 0.0;
        for (int h = g * group; h < (g + 1) * group; ++h)
            for (long long t = 0; t < L; ++t) {
                if (!visible(b, t, j)) continue;
                const long long row = ((long long)b * H_q + h) * L + t;
                double p, ds;
                p_ds(row, b, t, h, j, &p, &ds);
                const double* qv = qrow(q, b, t, h);
                const double* dov = qrow(dout, b, t, h);
                for (int d = 0; d < D; ++d) {
                    dkv[d] += scale * ds * qv[d];
                    dvv[d] += p * dov[d];
                }
            }
    });
    return 0;
}

// The zigzag layout (named beside the plain ring in [ULYSSES], introduction; the layout
// is a reading): the sequence of P*Lc tokens (Lc even) is cut into 2P segments of
// h = Lc/2 tokens and rank i holds segment i followed by segment 2P-1-i, so that under a
// causal mask every rank has the same work.  pos[i*Lc + t] is the sequence position of
// rank i's local token t.
int ora_zigzag_positions(int P, long long Lc, long long* pos) {
    if (P < 1 || Lc < 2 || Lc % 2 != 0) return 1;
    const long long h = Lc / 2;
    for (int i = 0; i < P; ++i)
        for (long long t = 0; t < Lc; ++t)
            pos[i * Lc + t] = t < h ? i * h + t : (2LL * P - 1 - i) * h + (t - h);
    return 0;
}

// Packed samples ([ACCEL-SP] section "Configuración del backend SP de ALST/Ulysses":
// sequence parallelism there is driven by position_ids, several samples combined into
// one sequence; the reading taken: samples are contiguous and a sample starts where
// position_ids is 0, position_ids counting 0, 1, 2, ... within it).  For every token t
// of every batch row, lo[t] = the position where t's sample starts = t - pid[t]; under
// the causal mask query t then sees exactly the keys lo[t] .. t of its own sample.
// Rejects ids that do not follow that rule (pid[t] = 0 or pid[t-1] + 1).
int ora_packed_lower_bounds(const int* pid, int B, long long L, long long* lo) {
    if (B < 1 || L < 1) return 1;
    for (int b = 0; b < B; ++b)
        for (long long t = 0; t < L; ++t) {
            const int v = pid[(long long)b * L + t];
            const bool ok = v == 0 || (t > 0 && v == pid[(long long)b * L + t - 1] + 1);
            if (!ok) return 1;
            lo[(long long)b * L + t] = t - v;
        }
    return 0;
}

// Elementwise merge, in place into a ([SP-QA] section 5, merge step).
//   o_a, o_b [B][L][H][D]   lse_a, lse_b [B][H][L]
int ora_lse_merge(double* o_a, double* lse_a, const double* o_b, const double* lse_b, int B,
                  int H, long long L, int D) {
    if (B < 1 || H < 1 || L < 1 || D < 1) return 1;
    for (int b = 0; b < B; ++b)
        for (long long t = 0; t < L; ++t)
            for (int h = 0; h < H; ++h) {
                const long long oi = (((long long)b * L + t) * H + h) * D;
                const long long li = ((long long)b * H + h) * L + t;
                merge_into(o_a + oi, lse_a + li, o_b + oi, lse_b[li], D);
            }
    return 0;
}

// Ulysses sequence-sharded -> head-sharded ([ULYSSES]: the all-to-all from
// [local_seqlen, global_heads, head_dim] to [global_seqlen, local_heads, head_dim]),
// with the head groups counted separately from the shards: G groups of Hl = H_out/G heads,
// each receiving every one of the P shards' tokens.  G = P is the Ulysses transform
// itself; G < P is the head split of the ring x Ulysses hybrid (USP), where only P/G ranks
// share a head group and the ring runs over the rest.  KV heads are copied up to H_out
// (GQA: replica j is source head floor(j * H_in / H_out)).
//   in  [P][B][Lc][H_in][D]  ->  out [G][B][P*Lc][Hl][D]
//   out[g][b][s*Lc+t][hh][:] = in[s][b][t][floor((g*Hl+hh)*H_in/H_out)][:]
int ora_seq2head(const void* in, void* out, int P, int G, int B, long long Lc, int H_in,
                 int H_out, int D, int esize) {
    if (P < 1 || G < 1 || B < 1 || Lc < 1 || H_in < 1 || H_out < 1 || D < 1 || esize < 1)
        return 1;
    if (H_out % G != 0 || H_out % H_in != 0) return 1;
    const int Hl = H_out / G;
    const unsigned char* src = (const unsigned char*)in;
    unsigned char* dst = (unsigned char*)out;
    for (int g = 0; g < G; ++g)
        for (int b = 0; b < B; ++b)
            for (int s = 0; s < P; ++s)
                for (long long t = 0; t < Lc; ++t)
                    for (int hh = 0; hh < Hl; ++hh) {
                        const int j = g * Hl + hh;                       // replicated head index
                        const int hs = (int)(((long long)j * H_in) / H_out);  // its source head
                        for (int d = 0; d < D; ++d) {
                            const long long di =
                                ((((long long)g * B + b) * (P * Lc) + (s * Lc + t)) * Hl + hh) * D + d;
                            const long long si =
                                ((((long long)s * B + b) * Lc + t) * H_in + hs) * D + d;
                            std::memcpy(dst + di * esize, src + si * esize, (size_t)esize);
                        }
                    }
    return 0;
}

// Ulysses head-sharded -> sequence-sharded ([ULYSSES]), the inverse transform, for G
// head groups and P shards.
//   in  [G][B][P*Lc][H/G][D]  ->  out [P][B][Lc][H][D]
//   out[s][b][t][g*Hl + hh][:] = in[g][b][s*Lc+t][hh][:],  Hl = H/G
int ora_head2seq(const void* in, void* out, int P, int G, int B, long long Lc, int H, int D,
                 int esize) {
    if (P < 1 || G < 1 || B < 1 || Lc < 1 || H < 1 || D < 1 || esize < 1 || H % G != 0) return 1;
    const int Hl = H / G;
    const unsigned char* src = (const unsigned char*)in;
    unsigned char* dst = (unsigned char*)out;
    for (int s = 0; s < P; ++s)
        for (int b = 0; b < B; ++b)
            for (long long t = 0; t < Lc; ++t)
                for (int g = 0; g < G; ++g)
                    for (int hh = 0; hh < Hl; ++hh)
                        for (int d = 0; d < D; ++d) {
                            const long long di =
                                ((((long long)s * B + b) * Lc + t) * H + (g * Hl + hh)) * D + d;
                            const long long si =
                                ((((long long)g * B + b) * (P * Lc) + (s * Lc + t)) * Hl + hh) * D + d;
                            std::memcpy(dst + di * esize, src + si * esize, (size_t)esize);
                        }
    return 0;
}

// The adjoint of the GQA copy in seq->head ("Метод контекстного параллелизма Ulysses": KV
// heads are copied so that every rank has one; H_in = H_out * rep replicas, replica j a copy
// of head j / rep): the gradient of a KV head is the sum of its replicas' gradients.
// in [rows][H_in][D], out [rows][H_out][D], out[r][g][d] = sum_{k < rep} in[r][g rep + k][d].
int ora_replica_sum(const double* in, double* out, long long rows, int H_in, int H_out, int D) {
    if (rows < 1 || H_in < 1 || H_out < 1 || D < 1 || H_in % H_out != 0) return 1;
    const int rep = H_in / H_out;
    for (long long r = 0; r < rows; ++r)
        for (int g = 0; g < H_out; ++g)
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int kk = 0; kk < rep; ++kk) acc += in[(r * H_in + g * rep + kk) * D + d];
                out[(r * H_out + g) * D + d] = acc;
            }
    return 0;
}

}  // extern "C"
