/*
 * oracle.c -- plain, slow, fp64 CPU reference of one Medusa speculative
 * decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the timed
 * CPU baseline of the benchmark use it.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Every function is the direct definition written out with loops, in double
 * precision, with no tiling, fusion or reordering beyond what the definition
 * states.  Inputs in bf16 / fp32 are widened to double exactly.
 *
 * Sources (public web pages on Medusa and speculative decoding):
 *   [SPEC]   "Speculative Decoding & Medusa Tree Attention: Accelerating LLM
 *            Inference by 3x Without Accuracy Loss"
 *   [GUIDE]  "Medusa Explained: Multi-Head Speculative Decoding Guide"
 *   [MTP]    "Multi-Token Prediction & Draft-Model-Free Speculative Decoding"
 *   [PHILOX] Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 *            1, 2, 3", SC'11, section 3 (Philox).
 * Readings where the pages are silent are stated beside each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1 };

/* exact widening of element i of a bf16 / fp32 buffer */
static double load(const void* p, int dtype, size_t i) {
    if (dtype == ORC_F32) return (double)((const float*)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Tree structure                                                            */
/* ------------------------------------------------------------------------ */

/*
 * Dense ancestor mask of a parent array: anc[i*T + j] = 1 iff j == i or j is
 * an ancestor of i, found by following parent pointers to a root (parent -1).
 * [MTP] "The 2D Tree Attention Mask": M[i,j] = 1 when node j is an ancestor
 * of node i or j = i; [GUIDE] "2. Single-Pass Tree Attention Verification":
 * the additive form (0 allowed, -inf blocked) of the same mask.  Forests are
 * accepted here (the parent-array example on [MTP] has two roots).
 * Returns 0, or -1 when a parent index is out of range or not smaller than
 * its child.
 */
int orc_tree_mask(const int32_t* parent, int T, uint8_t* anc) {
    for (int i = 0; i < T; ++i)
        if (parent[i] < -1 || parent[i] >= i) return -1;
    memset(anc, 0, (size_t)T * T);
    for (int i = 0; i < T; ++i)
        for (int cur = i; cur != -1; cur = parent[cur]) anc[(size_t)i * T + cur] = 1;
    return 0;
}

/*
 * Depth (root = 1) and sibling rank (number of siblings with a smaller
 * index) of every node of a single-rooted tree: node 0 is the root (parent
 * -1) and 0 <= parent[i] < i for i > 0.  Returns 0, or -1 when the array is
 * not such a tree.
 */
int orc_tree_shape(const int32_t* parent, int T, int32_t* depth, int32_t* rank) {
    if (T < 1 || parent[0] != -1) return -1;
    depth[0] = 1;
    rank[0] = 0;
    for (int i = 1; i < T; ++i) {
        if (parent[i] < 0 || parent[i] >= i) return -1;
        depth[i] = depth[parent[i]] + 1;
        int r = 0;
        for (int j = 1; j < i; ++j)
            if (parent[j] == parent[i]) ++r;
        rank[i] = r;
    }
    return 0;
}

/*
 * Cartesian-product candidate tree ([GUIDE] "1. Combinatorial Tree
 * Construction"; [MTP] "Tree-Structured Attention Verification": branching
 * (4,2,2) gives 16 trajectories).  Every candidate path picks one of the top
 * s_1 entries of head 1, one of the top s_2 of head 2, ...; the paths are
 * flattened into one node list, a node being a path prefix, numbered level by
 * level with prefixes in lexicographic order of their rank tuples.  Writes
 * the parent array and returns the node count, or -1 if it exceeds cap.
 */
int orc_product_tree(const int32_t* s, int K, int32_t* parent, int cap) {
    /* enumerate rank tuples level by level; a tuple's parent is its prefix */
    int level_start = 0, level_count = 1, n = 1;
    if (cap < 1) return -1;
    parent[0] = -1;
    for (int k = 0; k < K; ++k) {
        int next_start = n;
        for (int u = level_start; u < level_start + level_count; ++u)
            for (int r = 0; r < s[k]; ++r) {
                if (n >= cap) return -1;
                parent[n++] = u;
            }
        level_start = next_start;
        level_count = n - next_start;
    }
    return n;
}

/*
 * Round a double to the nearest bf16 value (8 significant bits, ties to
 * even), directly from the double so no intermediate rounding occurs.  Used
 * for the bf16 storage of the residual block's output (see orc_heads).
 */
double orc_round_bf16(double x) {
    if (x == 0.0 || x != x || isinf(x)) return x;
    int e;
    frexp(fabs(x), &e);              /* |x| = m 2^e, m in [0.5, 1) */
    int qe = e - 8;                  /* quantum of 8 significant bits */
    if (qe < -133) qe = -133;        /* bf16 subnormal spacing */
    double q = ldexp(1.0, qe);
    double r = nearbyint(x / q) * q; /* default rounding: to nearest, ties to even */
    if (fabs(r) > 3.3895313892515355e38) r = x > 0 ? INFINITY : -INFINITY;
    return r;
}

/* Threads an OpenMP build uses for its parallel loops (1 in the serial build). */
#ifdef _OPENMP
#include <omp.h>
int orc_threads(void) { return omp_get_max_threads(); }
#else
int orc_threads(void) { return 1; }
#endif

/* ------------------------------------------------------------------------ */
/* Medusa heads                                                              */
/* ------------------------------------------------------------------------ */

/*
 * [GUIDE] "The Architectural Blueprint": for head k,
 *     h^(k) = SiLU(W_res^(k) h) + h,     p^(k) = softmax(W_head^(k) h^(k)),
 * with SiLU(z) = z * sigma(z), sigma(z) = 1 / (1 + e^-z).  No bias (the
 * formula has none).  Reading on precision (the pages fix none): h^(k) is an
 * activation of the model's dtype, so for bf16 inputs it is stored rounded
 * to bf16 (from the exact fp64 value) before the vocabulary projection; the
 * top-s decision is then taken on the same operand precision as a bf16
 * kernel's.  round_hk = 0 keeps h^(k) at its exact fp64 value instead (the
 * formula read with no intermediate precision at all), so the distance
 * between the two readings can be measured.  Layouts: h [B,d]; W_res
 * [K,d,d] (output row, input column); W_head [K,V,d].  Outputs (each
 * nullable): hk [B,K,d], logits [B,K,V], probs [B,K,V].  Only sequence
 * b_only / head k_only is computed when those are >= 0 (others untouched).
 * The element loops are independent; an OpenMP build shares them among
 * threads with every element computed exactly as in the serial build.
 */
void orc_heads(const void* h, const void* W_res, const void* W_head, int dtype,
               int B, int d, int V, int K, int b_only, int k_only, int round_hk,
               double* hk_out, double* logits_out, double* probs_out) {
    double* hk = (double*)malloc(sizeof(double) * (size_t)d);
    double* logit = (double*)malloc(sizeof(double) * (size_t)V);
    for (int b = 0; b < B; ++b) {
        if (b_only >= 0 && b != b_only) continue;
        for (int k = 0; k < K; ++k) {
            if (k_only >= 0 && k != k_only) continue;
            /* residual block */
#pragma omp parallel for schedule(static)
            for (int o = 0; o < d; ++o) {
                double z = 0.0;
                for (int i = 0; i < d; ++i)
                    z += load(W_res, dtype, ((size_t)k * d + o) * d + i) * load(h, dtype, (size_t)b * d + i);
                double sig = 1.0 / (1.0 + exp(-z));
                hk[o] = z * sig + load(h, dtype, (size_t)b * d + o);
                if (dtype == ORC_BF16 && round_hk) hk[o] = orc_round_bf16(hk[o]);
            }
            /* projection to the vocabulary */
#pragma omp parallel for schedule(static)
            for (int v = 0; v < V; ++v) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i)
                    acc += load(W_head, dtype, ((size_t)k * V + v) * d + i) * hk[i];
                logit[v] = acc;
            }
            /* softmax */
            double m = -INFINITY;
            for (int v = 0; v < V; ++v)
                if (logit[v] > m) m = logit[v];
            double sum = 0.0;
            for (int v = 0; v < V; ++v) sum += exp(logit[v] - m);
            size_t base = ((size_t)b * K + k);
            if (hk_out)
                for (int o = 0; o < d; ++o) hk_out[base * d + o] = hk[o];
            if (logits_out)
                for (int v = 0; v < V; ++v) logits_out[base * V + v] = logit[v];
            if (probs_out)
                for (int v = 0; v < V; ++v) probs_out[base * V + v] = exp(logit[v] - m) / sum;
        }
    }
    free(hk);
    free(logit);
}

/*
 * Top-s of a vector ([GUIDE] "1. Combinatorial Tree Construction": each head
 * outputs its top-s_k highest-probability tokens).  Reading: the order is
 * value descending, lower index first among equal values (a stable sort of
 * -x); NaN entries are never chosen; missing entries are -1.  Softmax is
 * monotone, so ranking logits ranks probabilities.
 */
void orc_topk(const double* x, int n, int s, int32_t* idx) {
    for (int r = 0; r < s; ++r) {
        int best = -1;
        for (int i = 0; i < n; ++i) {
            if (x[i] != x[i]) continue; /* NaN */
            int taken = 0;
            for (int t = 0; t < r; ++t)
                if (idx[t] == i) taken = 1;
            if (taken) continue;
            if (best < 0 || x[i] > x[best]) best = i;
        }
        idx[r] = best;
    }
}

/*
 * Fill the candidate tree's tokens ([GUIDE] "1. Combinatorial Tree
 * Construction" and the head list of "The Architectural Blueprint": head 0,
 * the model's own LM head, gives w_{t+1}; Medusa head k gives w_{t+k+1}).
 * The root (depth 1) carries root_token[b] (w_{t+1}); a node at depth
 * dep >= 2 with sibling rank r carries entry r of Medusa head dep-1's top
 * list, i.e. topk_idx[b, dep-2, r]; node_q is that entry's probability (1 at
 * the root).  topk_idx / topk_p are [B, K, S].  Returns -1 when the tree is
 * deeper than K+1 or a rank is >= S.
 */
int orc_tree_fill(const int32_t* parent, int T, int B, int K, int S, const int32_t* root_token,
                  const int32_t* topk_idx, const double* topk_p, int32_t* node_tokens, double* node_q) {
    int32_t* depth = (int32_t*)malloc(sizeof(int32_t) * T);
    int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * T);
    int rc = orc_tree_shape(parent, T, depth, rank);
    for (int i = 0; rc == 0 && i < T; ++i)
        if (depth[i] > K + 1 || rank[i] >= S) rc = -1;
    for (int b = 0; rc == 0 && b < B; ++b)
        for (int i = 0; i < T; ++i) {
            if (i == 0) {
                node_tokens[(size_t)b * T] = root_token[b];
                node_q[(size_t)b * T] = 1.0;
            } else {
                size_t e = ((size_t)b * K + (depth[i] - 2)) * S + rank[i];
                node_tokens[(size_t)b * T + i] = topk_idx[e];
                node_q[(size_t)b * T + i] = topk_p[e];
            }
        }
    free(depth);
    free(rank);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Tree attention                                                            */
/* ------------------------------------------------------------------------ */

/*
 * [GUIDE] "2. Single-Pass Tree Attention Verification" and [MTP] "The 2D
 * Tree Attention Mask": every tree node attends to the whole prefix (the
 * historical context) and to the tree nodes j with M[i,j] = 1 (its ancestors
 * and itself); everything else is masked out.  For query row (b, i, h):
 *     s_j = scale * <q[b,i,h,:], k_j>,  O = sum_j softmax(s)_j v_j,
 *     lse = log sum_j exp(s_j)
 * where j runs over cache positions [0, prefix_len[b]) of kv-head g and over
 * the visible tree nodes, K/V of kv-head g, g = h / (Hq/Hkv) (grouped-query
 * reading; the pages are silent on GQA).  scale <= 0 means 1/sqrt(D).
 * Layouts: q [B,T,Hq,D]; k_tree, v_tree [B,T,Hkv,D]; k_cache, v_cache
 * [B,Hkv,S_max,D].  rows: nrows triples (b,i,h) to evaluate, or NULL for all
 * B*T*Hq rows in (b,i,h) order; out [nrows][D], lse [nrows] (nullable).
 * Returns -1 on a bad tree or row.
 */
int orc_tree_attention(const void* q, const void* k_tree, const void* v_tree, const void* k_cache,
                       const void* v_cache, const int32_t* prefix_len, int dtype, int B, int T, int Hq,
                       int Hkv, int D, int S_max, double scale, const int32_t* parent, int nrows,
                       const int32_t* rows, double* out, double* lse) {
    if (Hkv <= 0 || Hq % Hkv != 0) return -1;
    uint8_t* anc = (uint8_t*)malloc((size_t)T * T);
    if (orc_tree_mask(parent, T, anc) != 0) {
        free(anc);
        return -1;
    }
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
    int G = Hq / Hkv;
    int total = rows ? nrows : B * T * Hq;
    int maxkeys = S_max + T;
    int rc = 0;
    for (int r = 0; rows && r < total; ++r) {
        int b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
        if (b < 0 || b >= B || i < 0 || i >= T || h < 0 || h >= Hq) rc = -1;
    }
    for (int b = 0; b < B; ++b)
        if (prefix_len[b] < 0 || prefix_len[b] > S_max) rc = -1;
    if (rc != 0) {
        free(anc);
        return rc;
    }
    /* rows are independent: an OpenMP build shares them among threads, each
     * with its own score buffer and the same per-row arithmetic */
#pragma omp parallel
    {
    double* s = (double*)malloc(sizeof(double) * (size_t)maxkeys);
#pragma omp for schedule(dynamic, 8)
    for (int r = 0; r < total; ++r) {
        int b, i, h;
        if (rows) {
            b = rows[3 * r];
            i = rows[3 * r + 1];
            h = rows[3 * r + 2];
        } else {
            b = r / (T * Hq);
            i = (r / Hq) % T;
            h = r % Hq;
        }
        int g = h / G;
        int S = prefix_len[b];
        size_t qoff = (((size_t)b * T + i) * Hq + h) * D;
        /* scores over the visible keys: prefix, then visible tree nodes */
        int n = 0;
        for (int j = 0; j < S; ++j) {
            size_t koff = (((size_t)b * Hkv + g) * S_max + j) * D;
            double acc = 0.0;
            for (int e = 0; e < D; ++e) acc += load(q, dtype, qoff + e) * load(k_cache, dtype, koff + e);
            s[n++] = scale * acc;
        }
        for (int j = 0; j < T; ++j) {
            if (!anc[(size_t)i * T + j]) continue;
            size_t koff = (((size_t)b * T + j) * Hkv + g) * D;
            double acc = 0.0;
            for (int e = 0; e < D; ++e) acc += load(q, dtype, qoff + e) * load(k_tree, dtype, koff + e);
            s[n++] = scale * acc;
        }
        double m = -INFINITY;
        for (int t = 0; t < n; ++t)
            if (s[t] > m) m = s[t];
        double sum = 0.0;
        for (int t = 0; t < n; ++t) sum += exp(s[t] - m);
        double* o = out + (size_t)r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        n = 0;
        for (int j = 0; j < S; ++j) {
            double w = exp(s[n++] - m) / sum;
            size_t voff = (((size_t)b * Hkv + g) * S_max + j) * D;
            for (int e = 0; e < D; ++e) o[e] += w * load(v_cache, dtype, voff + e);
        }
        for (int j = 0; j < T; ++j) {
            if (!anc[(size_t)i * T + j]) continue;
            double w = exp(s[n++] - m) / sum;
            size_t voff = (((size_t)b * T + j) * Hkv + g) * D;
            for (int e = 0; e < D; ++e) o[e] += w * load(v_tree, dtype, voff + e);
        }
        if (lse) lse[r] = m + log(sum);
    }
    free(s);
    }
    free(anc);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Verification                                                              */
/* ------------------------------------------------------------------------ */

/* argmax of one row: largest value, lowest index among equal values; NaN
 * never wins; an all-NaN or all -inf row gives index 0. */
static int row_argmax(const void* x, int dtype, size_t base, int V) {
    double best = -INFINITY;
    int bi = 0;
    for (int v = 0; v < V; ++v) {
        double t = load(x, dtype, base + v);
        if (t > best) {
            best = t;
            bi = v;
        }
    }
    return bi;
}

/*
 * Greedy verification ([GUIDE] "2. Single-Pass Tree Attention Verification",
 * steps 2-4: the target's distribution at every node; the longest path whose
 * every token matches the target's greedy prediction; [MTP] "The 2D Tree
 * Attention Mask": commit the longest accepted path plus one bonus token
 * emitted by the target).  The target's prediction for the token after node
 * u is argmax(logits[b,u,:]).  The accepted set holds the root and every
 * node c whose parent is accepted and whose token equals the parent's
 * prediction.  The committed path ends at the deepest accepted node (lowest
 * index among equally deep ones); the bonus is that node's prediction.
 * Outputs: path [B, max_path] (node ids, root first, -1 padded), len [B],
 * bonus [B].  Returns -1 on a bad tree or a path longer than max_path.
 */
int orc_verify_greedy(const void* logits, int dtype, const int32_t* node_tokens, int B, int T, int V,
                      const int32_t* parent, int max_path, int32_t* path, int32_t* len, int32_t* bonus) {
    int32_t* depth = (int32_t*)malloc(sizeof(int32_t) * T);
    int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * T);
    int32_t* pred = (int32_t*)malloc(sizeof(int32_t) * T);
    uint8_t* acc = (uint8_t*)malloc((size_t)T);
    int rc = orc_tree_shape(parent, T, depth, rank);
    for (int b = 0; rc == 0 && b < B; ++b) {
#pragma omp parallel for schedule(static)
        for (int u = 0; u < T; ++u) pred[u] = row_argmax(logits, dtype, ((size_t)b * T + u) * V, V);
        acc[0] = 1;
        for (int c = 1; c < T; ++c)
            acc[c] = acc[parent[c]] && node_tokens[(size_t)b * T + c] == pred[parent[c]];
        int best = 0;
        for (int c = 1; c < T; ++c)
            if (acc[c] && depth[c] > depth[best]) best = c;
        int L = depth[best];
        if (L > max_path) {
            rc = -1;
            break;
        }
        for (int t = 0; t < max_path; ++t) path[(size_t)b * max_path + t] = -1;
        for (int cur = best, t = L - 1; cur != -1; cur = parent[cur], --t) path[(size_t)b * max_path + t] = cur;
        len[b] = L;
        bonus[b] = pred[best];
    }
    free(depth);
    free(rank);
    free(pred);
    free(acc);
    return rc;
}

/*
 * Philox4x32-10 [PHILOX]: ten rounds of the 4x32 S-box on a 128-bit counter
 * with a 64-bit key; each round multiplies counter words 0 and 2 by the two
 * round multipliers, takes high and low 32-bit halves, xors the high halves
 * with the other counter words and the round key, and permutes the words;
 * the key is bumped by the two Weyl constants between rounds.
 */
void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += W0;
            k1 += W1;
        }
        uint64_t p0 = (uint64_t)M0 * c0;
        uint64_t p1 = (uint64_t)M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0;
        c1 = n1;
        c2 = n2;
        c3 = n3;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* the Philox block of node `node` of sequence b at decode step `step`:
 * counter (b, node, step, 0), key (seed low word, seed high word) */
static void node_draw(uint64_t seed, uint32_t step, int b, int node, uint32_t out[4]) {
    uint32_t ctr[4] = {(uint32_t)b, (uint32_t)node, step, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    orc_philox4x32_10(ctr, key, out);
}

/*
 * Residual distribution of [SPEC] "2. The Mathematical Foundation of
 * Speculative Sampling": normalize(max(0, P_target - P_draft)), in the
 * quantised form the sampler uses (reading; the pages do not fix a
 * precision): W(y) = floor(max(0, P(y) - Q(y)) * 2^32), S = sum W,
 * out(y) = W(y) / S.  When S = 0 (P <= Q everywhere) out = P.  out may alias
 * P; W (length V) receives the integer weights.  Returns S.
 */
uint64_t orc_residual(const double* P, const float* Q, int V, double* out, uint64_t* W) {
    const double two32 = 4294967296.0;
    uint64_t S = 0;
    for (int y = 0; y < V; ++y) {
        double diff = P[y] - (double)Q[y];
        W[y] = diff > 0.0 ? (uint64_t)floor(diff * two32) : 0u;
        S += W[y];
    }
    for (int y = 0; y < V; ++y) out[y] = S > 0 ? (double)W[y] / (double)S : P[y];
    return S;
}

/*
 * Stochastic verification.  The chain rule of [SPEC] "2. The Mathematical
 * Foundation of Speculative Sampling": accept a drafted token x with
 * probability min(1, P_target(x) / P_draft(x)); on rejection draw the
 * replacement from normalize(max(0, P_target - P_draft)).  Extended to a tree
 * (reading; the pages give only the chain form): at the current node u with
 * current target distribution P (initially p[b,u,:]) and draft distribution
 * Q = q[b, q_row[u], :], the children of u are tried in index order:
 *   - child c with token x is accepted iff  u_c * Q(x) < P(x)  (u_c uniform
 *     in [0,1): min(1, P/Q) without a division); the walk moves to c with
 *     P = p[b,c,:];
 *   - on rejection, W(y) = floor(max(0, P(y) - Q(y)) * 2^32) for every y,
 *     S = sum W; if S > 0, P(y) = W(y) / S, else P is kept.
 * When u has no children left (a leaf, or all rejected), the bonus token is
 * drawn from P by inverse CDF on integer weights: W(y) = floor(P(y) * 2^32),
 * S = sum W, t = floor(U * S / 2^32) for a 32-bit uniform U, bonus = the
 * smallest y whose inclusive prefix sum of W exceeds t.
 * Uniforms: Philox4x32-10 block of (b, node, step); u_c = (word0 >> 8) * 2^-24
 * of child c's block, U = word1 of the block of the node where the walk ends.
 * p, q are fp32 [B,T,V] and [B,Qrows,V]; q_row NULL means q_row[u] = u.
 * Row b of the arrays is sequence b0 + b of the batch: its uniforms use the
 * counter of sequence b0 + b (so one sequence can be checked on its own).
 * Outputs as for orc_verify_greedy; status bit 1 is set when a bonus
 * distribution has zero total weight (bonus 0 then).
 */
void orc_softmax_temperature(const double* z, int V, double inv_tau, double* P);

/* where the walk's target rows come from: fp32 probabilities p, or logits
 * turned into probabilities by orc_softmax_temperature */
typedef struct {
    const float* p;      /* [B, T, V] f32, or NULL */
    const void* logits;  /* [B, T, V] of dtype `dtype` when p is NULL */
    int dtype;
    double inv_tau;
} row_source;

static void load_row(const row_source* src, size_t row, int V, double* P) {
    if (src->p) {
        for (int y = 0; y < V; ++y) P[y] = (double)src->p[row * V + y];
        return;
    }
    double* z = (double*)malloc(sizeof(double) * (size_t)V);
    for (int y = 0; y < V; ++y) z[y] = load(src->logits, src->dtype, row * V + y);
    orc_softmax_temperature(z, V, src->inv_tau, P);
    free(z);
}

static int stochastic_walk(const row_source* src, const float* q, int Qrows, const int32_t* q_row,
                           const int32_t* node_tokens, int B, int T, int V, const int32_t* parent,
                           uint64_t seed, uint32_t step, int max_path, int32_t* path, int32_t* len,
                           int32_t* bonus, int32_t* status, int b0) {
    int32_t* depth = (int32_t*)malloc(sizeof(int32_t) * T);
    int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * T);
    double* P = (double*)malloc(sizeof(double) * (size_t)V);
    uint64_t* W = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)V);
    const double two32 = 4294967296.0;
    int rc = orc_tree_shape(parent, T, depth, rank);
    if (status) *status = 0;
    for (int b = 0; rc == 0 && b < B; ++b) {
        int u = 0, L = 1;
        for (int t = 0; t < max_path; ++t) path[(size_t)b * max_path + t] = -1;
        path[(size_t)b * max_path] = 0;
        load_row(src, (size_t)b * T + u, V, P);
        for (;;) {
            int qr = q_row ? q_row[u] : u;
            if (qr < 0 || qr >= Qrows) {
                rc = -1;
                break;
            }
            const float* Q = q + ((size_t)b * Qrows + qr) * V;
            int moved = 0;
            for (int c = u + 1; c < T; ++c) {
                if (parent[c] != u) continue;
                int x = node_tokens[(size_t)b * T + c];
                if (x < 0 || x >= V) {
                    rc = -1;
                    break;
                }
                uint32_t r[4];
                node_draw(seed, step, b0 + b, c, r);
                double uc = (double)(r[0] >> 8) * (1.0 / 16777216.0);
                if (uc * (double)Q[x] < P[x]) {
                    u = c;
                    if (L >= max_path) {
                        rc = -1;
                        break;
                    }
                    path[(size_t)b * max_path + L] = c;
                    ++L;
                    load_row(src, (size_t)b * T + u, V, P);
                    moved = 1;
                    break;
                }
                orc_residual(P, Q, V, P, W);
            }
            if (rc != 0 || !moved) break;
        }
        if (rc != 0) break;
        /* bonus from the current P */
        uint64_t S = 0;
        for (int y = 0; y < V; ++y) {
            W[y] = P[y] > 0.0 ? (uint64_t)floor(P[y] * two32) : 0u;
            S += W[y];
        }
        uint32_t r[4];
        node_draw(seed, step, b0 + b, u, r);
        int tok = 0;
        if (S == 0) {
            if (status) *status |= 1;
        } else {
            unsigned __int128 prod = (unsigned __int128)r[1] * S;
            uint64_t t = (uint64_t)(prod >> 32);
            uint64_t run = 0;
            for (int y = 0; y < V; ++y) {
                run += W[y];
                if (run > t) {
                    tok = y;
                    break;
                }
            }
        }
        len[b] = L;
        bonus[b] = tok;
    }
    free(depth);
    free(rank);
    free(P);
    free(W);
    return rc;
}

int orc_verify_stochastic(const float* p, const float* q, int Qrows, const int32_t* q_row,
                          const int32_t* node_tokens, int B, int T, int V, const int32_t* parent,
                          uint64_t seed, uint32_t step, int max_path, int32_t* path, int32_t* len,
                          int32_t* bonus, int32_t* status, int b0) {
    row_source src = {p, NULL, 0, 1.0};
    return stochastic_walk(&src, q, Qrows, q_row, node_tokens, B, T, V, parent, seed, step, max_path, path, len,
                           bonus, status, b0);
}

/*
 * Target distribution from logits at temperature tau (reading: the pages
 * write P_target without saying how it is obtained from the target model's
 * logits; the plain softmax, tau = 1, is the pages' case, and tau > 0 is the
 * usual sampling temperature):
 *     m = max_y z(y),  e(y) = exp((z(y) - m) * (1/tau)),  Z = sum_y e(y)
 *     P(y) = e(y) * (1/Z)
 * in fp64, every product and difference rounded once, Z summed in index
 * order; inv_tau = 1/tau is passed in.  NaN logits are skipped by the max
 * and make P NaN (no mass), as does a row without a finite maximum.
 */
void orc_softmax_temperature(const double* z, int V, double inv_tau, double* P) {
    double m = -INFINITY;
    for (int y = 0; y < V; ++y) m = fmax(m, z[y]);
    double Z = 0.0;
    for (int y = 0; y < V; ++y) {
        P[y] = exp((z[y] - m) * inv_tau);
        Z += P[y];
    }
    const double r = 1.0 / Z;
    for (int y = 0; y < V; ++y) P[y] = P[y] * r;
}

/*
 * Stochastic verification reading the target's logits: the walk of
 * orc_verify_stochastic with each visited node's P computed from its logits
 * row by orc_softmax_temperature (logits dtype 0 = f32, 1 = bf16).
 */
int orc_verify_stochastic_logits(const void* logits, int dtype, double temperature, const float* q, int Qrows,
                                 const int32_t* q_row, const int32_t* node_tokens, int B, int T, int V,
                                 const int32_t* parent, uint64_t seed, uint32_t step, int max_path, int32_t* path,
                                 int32_t* len, int32_t* bonus, int32_t* status, int b0) {
    if (!(temperature > 0.0) || !isfinite(temperature)) return -1;
    row_source src = {NULL, logits, dtype, 1.0 / temperature};
    return stochastic_walk(&src, q, Qrows, q_row, node_tokens, B, T, V, parent, seed, step, max_path, path, len,
                           bonus, status, b0);
}

/* ------------------------------------------------------------------------ */
/* KV commit                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * The commit when the tree's K/V were appended to the cache right after each
 * prefix before attention ([MTP] "The 2D Tree Attention Mask": the longest
 * accepted path is kept; "Production Deployment Guidelines": the other
 * branches are culled): in every layer, the accepted path's rows move down to
 * just after the prefix,
 *     new cache_l[b, g, S + t, :] = old cache_l[b, g, S + path[b,t], :],  t < len[b]
 *     new_prefix_len[b] = S + len[b]          (S = prefix_len[b])
 * (old rows are copied out first, then written).  caches: n_layers blocks of
 * [B, Hkv, S_max, D], element size esize, copied bit for bit.  A sequence
 * whose path is not strictly increasing, holds a node id outside [0, T) or
 * has len outside [0, max_path] is left untouched (status bit 1), as is one
 * whose source rows reach S_max (status bit 2); its new_prefix_len is S.
 */
void orc_kv_compact(void* k_caches, void* v_caches, int n_layers, const int32_t* path, int max_path,
                    const int32_t* len, const int32_t* prefix_len, int32_t* new_prefix_len, int B, int Hkv, int D,
                    int S_max, int T, int esize, int32_t* status) {
    const size_t row = (size_t)D * esize;
    const size_t layer_bytes = (size_t)B * Hkv * S_max * row;
    unsigned char* tmp = (unsigned char*)malloc(row * (size_t)(max_path > 0 ? max_path : 1));
    if (status) *status = 0;
    for (int b = 0; b < B; ++b) {
        const int S = prefix_len[b], L = len[b];
        int ok = L >= 0 && L <= max_path && S >= 0;
        for (int t = 0; ok && t < L; ++t) {
            const int n = path[(size_t)b * max_path + t];
            const int prev = t > 0 ? path[(size_t)b * max_path + t - 1] : -1;
            if (n <= prev || n >= T) ok = 0;
        }
        if (!ok) {
            if (status) *status |= 1;
        } else if (L > 0 && (long)S + path[(size_t)b * max_path + L - 1] >= S_max) {
            ok = 0;
            if (status) *status |= 2;
        }
        new_prefix_len[b] = ok ? S + L : S;
        if (!ok) continue;
        for (int l = 0; l < n_layers; ++l)
            for (int kv = 0; kv < 2; ++kv) {
                unsigned char* c = (unsigned char*)(kv ? v_caches : k_caches) + (size_t)l * layer_bytes;
                for (int g = 0; g < Hkv; ++g) {
                    unsigned char* blk = c + ((size_t)b * Hkv + g) * S_max * row;
                    for (int t = 0; t < L; ++t)
                        memcpy(tmp + (size_t)t * row, blk + (size_t)(S + path[(size_t)b * max_path + t]) * row, row);
                    for (int t = 0; t < L; ++t) memcpy(blk + (size_t)(S + t) * row, tmp + (size_t)t * row, row);
                }
            }
    }
    free(tmp);
}

/*
 * [MTP] "The 2D Tree Attention Mask" (the engine commits the longest accepted
 * path) and "Production Deployment Guidelines" (unselected branches are
 * culled): the K/V rows of the accepted path's nodes are appended, in path
 * order, to each sequence's cache after its prefix; the others are dropped.
 *     cache[b, g, prefix_len[b] + t, :] = tree[b, path[b,t], g, :],  t < len[b]
 *     new_prefix_len[b] = prefix_len[b] + len[b]
 * Element size esize bytes (copied bit for bit).  A sequence whose commit
 * would pass S_max, or whose path holds a node id outside [0, T), is left
 * untouched and sets bit 1 of *status.
 */
void orc_kv_commit(void* k_cache, void* v_cache, const void* k_tree, const void* v_tree,
                   const int32_t* path, int max_path, const int32_t* len, const int32_t* prefix_len,
                   int32_t* new_prefix_len, int B, int Hkv, int D, int S_max, int T, int esize,
                   int32_t* status) {
    if (status) *status = 0;
    for (int b = 0; b < B; ++b) {
        int S = prefix_len[b], L = len[b];
        int ok = L >= 0 && L <= max_path && S >= 0 && S + L <= S_max;
        for (int t = 0; ok && t < L; ++t) {
            int n = path[(size_t)b * max_path + t];
            if (n < 0 || n >= T) ok = 0;
        }
        if (!ok) {
            if (status) *status |= 1;
            new_prefix_len[b] = S;
            continue;
        }
        for (int t = 0; t < L; ++t) {
            int n = path[(size_t)b * max_path + t];
            for (int g = 0; g < Hkv; ++g) {
                size_t dst = ((((size_t)b * Hkv + g) * S_max) + S + t) * D * esize;
                size_t src = ((((size_t)b * T + n) * Hkv) + g) * D * esize;
                memcpy((char*)k_cache + dst, (const char*)k_tree + src, (size_t)D * esize);
                memcpy((char*)v_cache + dst, (const char*)v_tree + src, (size_t)D * esize);
            }
        }
        new_prefix_len[b] = S + L;
    }
}

/* ------------------------------------------------------------------------ */
/* Paged KV cache                                                            */
/* ------------------------------------------------------------------------ */

/*
 * [MTP] "Production Deployment Guidelines": tree attention runs inside
 * PagedAttention, the cache held in non-contiguous physical blocks.  A page
 * pool pages [num_pages, Hkv, page_size, D] with a block table
 * table [B, max_pages]: position s of sequence b is slot s % page_size of page
 * table[b, s / page_size].  Paging is only where a position is stored, so the
 * attention of a paged cache is the attention of the contiguous cache this
 * gather builds:
 *     cache[b, g, s, :] = pages[table[b, s / page_size], g, s % page_size, :]
 * for s < n_pos[b]; other entries of cache are left as they are.  Returns -1
 * (nothing written for that sequence) when a needed table entry is outside
 * [0, num_pages) or s / page_size >= max_pages.
 */
int orc_gather_pages(const void* pages, const int32_t* table, int max_pages, int page_size, int num_pages,
                     const int32_t* n_pos, int B, int Hkv, int D, int S_max, int esize, void* cache) {
    int rc = 0;
    for (int b = 0; b < B; ++b) {
        int n = n_pos[b], ok = n >= 0 && n <= S_max;
        for (int s = 0; ok && s < n; ++s) {
            int blk = s / page_size;
            if (blk >= max_pages) ok = 0;
            else if (table[(size_t)b * max_pages + blk] < 0 || table[(size_t)b * max_pages + blk] >= num_pages) ok = 0;
        }
        if (!ok) {
            rc = -1;
            continue;
        }
        for (int g = 0; g < Hkv; ++g)
            for (int s = 0; s < n; ++s) {
                int page = table[(size_t)b * max_pages + s / page_size];
                size_t src = ((((size_t)page * Hkv + g) * page_size) + s % page_size) * D * esize;
                size_t dst = ((((size_t)b * Hkv + g) * S_max) + s) * D * esize;
                memcpy((char*)cache + dst, (const char*)pages + src, (size_t)D * esize);
            }
    }
    return rc;
}

/*
 * Commit into a paged cache: as orc_kv_commit, position prefix_len[b] + t of
 * sequence b being slot (prefix_len[b] + t) % page_size of page
 * table[b, (prefix_len[b] + t) / page_size].  A sequence whose new positions
 * need a block index >= max_pages, or a table entry outside [0, num_pages),
 * or whose path holds a node id outside [0, T), is left untouched and sets bit
 * 1 of *status.
 */
void orc_kv_commit_paged(void* k_pages, void* v_pages, const void* k_tree, const void* v_tree, const int32_t* table,
                         int max_pages, int page_size, int num_pages, const int32_t* path, int max_path,
                         const int32_t* len, const int32_t* prefix_len, int32_t* new_prefix_len, int B, int Hkv, int D,
                         int T, int esize, int32_t* status) {
    if (status) *status = 0;
    for (int b = 0; b < B; ++b) {
        int S = prefix_len[b], L = len[b];
        int ok = L >= 0 && L <= max_path && S >= 0;
        for (int t = 0; ok && t < L; ++t) {
            int n = path[(size_t)b * max_path + t];
            int blk = (S + t) / page_size;
            if (n < 0 || n >= T || blk >= max_pages) ok = 0;
            else if (table[(size_t)b * max_pages + blk] < 0 || table[(size_t)b * max_pages + blk] >= num_pages) ok = 0;
        }
        if (!ok) {
            if (status) *status |= 1;
            new_prefix_len[b] = S;
            continue;
        }
        for (int t = 0; t < L; ++t) {
            int n = path[(size_t)b * max_path + t];
            int page = table[(size_t)b * max_pages + (S + t) / page_size];
            for (int g = 0; g < Hkv; ++g) {
                size_t dst = ((((size_t)page * Hkv + g) * page_size) + (S + t) % page_size) * D * esize;
                size_t src = ((((size_t)b * T + n) * Hkv) + g) * D * esize;
                memcpy((char*)k_pages + dst, (const char*)k_tree + src, (size_t)D * esize);
                memcpy((char*)v_pages + dst, (const char*)v_tree + src, (size_t)D * esize);
            }
        }
        new_prefix_len[b] = S + L;
    }
}
