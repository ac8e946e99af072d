/*
 * spec_verify_oracle.c -- the CPU oracle for the speculative-decoding
 * verify-and-accept step.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the smoke
 * check and the CPU-baseline leg of the benchmark load this file's library.
 * It shares no code, header, table or constant generator with the CUDA
 * library: the Philox generator, the bf16 decoder, the softmax and the
 * argmax below are written out again, plainly, in double precision.
 *
 * What it computes (all in fp64; inputs are decoded exactly from fp32/bf16):
 *
 *  Stochastic verify.  "Accelerating Sonar through speculation" (Perplexity),
 *  section "Speculative decoding", stages "Acceptance" and "Target
 *  generation": the target is run over the drafted tokens, the longest
 *  acceptable prefix is found, and the target logits at the first mismatch
 *  (or after the last draft) are sampled for one more token, so n drafts can
 *  commit up to n+1 tokens.  Section "Draft-Target": acceptance compares the
 *  full draft and target probability distributions, and the logits set that
 *  the target always emits after the accepted prefix is sampled.  The pages
 *  do not write the comparison down; the oracle uses the speculative
 *  rejection-sampling rule (Leviathan et al. 2023; Chen et al. 2023):
 *      p_i = softmax(target[b,i,:] / T),  q_i = softmax(draft[b,i,:] / T)
 *      accept draft token x_i  <=>  u_i * q_i(x_i) < p_i(x_i)
 *                              (== u_i < min(1, p_i(x_i)/q_i(x_i)) for q>0)
 *      n = first rejected position, or k
 *      n < k : y ~ normalize(max(0, p_n - q_n))   (Gumbel-max)
 *      n = k : y ~ p_k                            (Gumbel-max)
 *
 *  Stochastic tree verify.  Same page, section "EAGLE": at every node of
 *  the draft tree the Top-K candidates are explored, and the longest
 *  acceptable path is kept with one more token from the target.  Reading
 *  (the page writes no rule down): Top-K siblings are fixed, not sampled, so
 *  the draft distribution behind each child is a point mass on its token,
 *  and the rejection rule above applied to the siblings one after another
 *  (multi-draft recursive rejection, as in SpecInfer and Sequoia) becomes:
 *      at node u, p = softmax(row u / T), R = 1, E = {};
 *      for each child c of u in node order, with token x_c:
 *          accept  <=>  x_c valid, x_c not in E, and u_c * R < p(x_c)
 *          else     E += {x_c},  R -= p(x_c)        (when x_c valid, new)
 *      an accepted child becomes u; otherwise y ~ p restricted to V \ E
 *      (Gumbel-max over l/T), which keeps the output distributed as p.
 *  Draws: u_c is the acceptance draw of position c - 1; the final draw uses
 *  position u with tag CORRECTION when u has children, BONUS when it is a
 *  leaf.  On a chain tree this is exactly stochastic verify with one-hot
 *  draft distributions.
 *
 *  Greedy verify.  Same page, section "Speculative decoding": the longest
 *  prefix that the target accepts, plus the target's own next token.  In
 *  greedy mode "accepts" means "equals the target argmax" (first maximum).
 *
 *  Threshold acceptance.  Same page, same section: each candidate prefix is
 *  scored by probability and the longest at or above the acceptance threshold
 *  is kept (the score is the prefix's probability under the target; see
 *  oracle_verify_threshold), plus the target's argmax as the extra token.
 *
 *  Multi-candidate (lookahead n-gram) verify.  "Lookahead decoding" news
 *  piece, section "Lookahead decoding breaks the order dependency" and
 *  steps 2-4: captured n-grams are validated against the target and the
 *  longest accepted one is appended; here every candidate branch g has its
 *  own target rows, the accepted length of branch g is its longest prefix
 *  equal to the row argmaxes, and the best branch is the longest one (lowest
 *  g on a tie).
 *
 *  Random draws.  Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
 *  Random Numbers: As Easy as 1, 2, 3", SC'11), written here from that
 *  definition.  key = (seed & 0xffffffff, seed >> 32); counter =
 *  (c0, position, sequence, tag).  The acceptance draw of position i uses
 *  c0 = 0, word 0.  A per-vocabulary draw for entry x uses c0 = x >> 2 and
 *  output word x & 3.  Uniforms: u = (w >> 8) * 2^-24 in [0,1) for
 *  acceptance; u' = ((w >> 9) + 0.5) * 2^-23 in (0,1) and
 *  g = -ln(-ln u') for Gumbel noise.  The pages fix none of this; it is the
 *  layout chosen so that the oracle and the GPU library draw the same
 *  numbers.
 *
 * Readings where the pages are silent (the same readings are made by the
 * GPU library):
 *   - the same temperature T divides both target and draft logits;
 *   - q(x_i) = 0 and p(x_i) > 0 accepts; p(x_i) = 0 rejects;
 *   - a draft token outside [0, V) has p = q = 0 and is rejected (flag bit 0);
 *   - if no x has p_n(x) - q_n(x) > 0 (possible only through rounding), the
 *     correction is drawn from p_n with the same CORRECTION stream (flag
 *     bit 1);
 *   - ties: lowest vocabulary index, lowest candidate index;
 *   - committed tokens: out[0..n-1] = drafts, out[n] = sampled token,
 *     out[n+1..k] = -1.
 *
 * Every row must contain at least one finite logit; +inf and NaN are not
 * valid logits.  -inf is allowed (probability zero).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1

#define TAG_ACCEPT 0u
#define TAG_CORRECTION 1u
#define TAG_BONUS 2u

/* ---------------------------------------------------------------- Philox */

static void philox_round(uint32_t c[4], const uint32_t key[2])
{
    /* One round: two 32x32->64 products, the high halves mixed with the
     * other two counter words and the key, the low halves passed on. */
    uint64_t prod0 = (uint64_t)0xD2511F53u * (uint64_t)c[0];
    uint64_t prod1 = (uint64_t)0xCD9E8D57u * (uint64_t)c[2];
    uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
    uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
    uint32_t next[4];
    next[0] = hi1 ^ c[1] ^ key[0];
    next[1] = lo1;
    next[2] = hi0 ^ c[3] ^ key[1];
    next[3] = lo0;
    memcpy(c, next, sizeof next);
}

void oracle_philox4x32_10(const uint32_t counter[4], const uint32_t key[2],
                          uint32_t out[4])
{
    uint32_t c[4], k[2];
    memcpy(c, counter, sizeof c);
    memcpy(k, key, sizeof k);
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { /* Weyl key schedule between rounds */
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        philox_round(c, k);
    }
    memcpy(out, c, sizeof c);
}

/* Batch form for tests: counters [n][4], one key from the 64-bit seed. */
void oracle_philox_batch(const uint32_t *counters, int64_t n, uint64_t seed,
                         uint32_t *out)
{
    uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    for (int64_t j = 0; j < n; ++j)
        oracle_philox4x32_10(counters + 4 * j, key, out + 4 * j);
}

static uint32_t draw_word(uint64_t seed, uint32_t c0, uint32_t pos,
                          uint32_t seq, uint32_t tag, int word)
{
    uint32_t ctr[4] = {c0, pos, seq, tag};
    uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[word];
}

static double accept_uniform(uint32_t w)
{
    return (double)(w >> 8) * 0x1p-24; /* [0, 1) */
}

static double gumbel_noise(uint32_t w)
{
    /* 23 random bits: ((w >> 9) + 0.5) * 2^-23 has at most 24 significant
     * bits, so it is exact in fp32 as well as fp64 */
    double u = ((double)(w >> 9) + 0.5) * 0x1p-23; /* (0, 1) */
    return -log(-log(u));
}

/* Gumbel noise of vocabulary entry x at (position, sequence, tag). */
static double vocab_gumbel(uint64_t seed, int64_t x, uint32_t pos,
                           uint32_t seq, uint32_t tag)
{
    return gumbel_noise(
        draw_word(seed, (uint32_t)(x >> 2), pos, seq, tag, (int)(x & 3)));
}

/* ---------------------------------------------------------------- logits */

static double logit_at(const void *base, int dtype, int64_t offset)
{
    if (dtype == OR_F32)
        return (double)((const float *)base)[offset];
    /* bf16: the upper 16 bits of an IEEE binary32 */
    uint32_t bits = (uint32_t)((const uint16_t *)base)[offset] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    const void *base;
    int dtype;
    int64_t offset; /* element offset of x = 0 */
} row_t;

static double row_at(row_t r, int64_t x) { return logit_at(r.base, r.dtype, r.offset + x); }

/* Temperature softmax statistics of a row: m = max_x l(x)/T and
 * s = sum_x exp(l(x)/T - m), so that p(x) = exp(l(x)/T - m) / s. */
static void softmax_stats(row_t r, int V, double T, double *m, double *s)
{
    double mx = -INFINITY;
    for (int64_t x = 0; x < V; ++x) {
        double z = row_at(r, x) / T;
        if (z > mx) mx = z;
    }
    double acc = 0.0;
    for (int64_t x = 0; x < V; ++x)
        acc += exp(row_at(r, x) / T - mx);
    *m = mx;
    *s = acc;
}

static double softmax_prob(row_t r, int64_t x, double T, double m, double s)
{
    return exp(row_at(r, x) / T - m) / s;
}

/* Scan of candidate scores in increasing x; keeps the first maximum and the
 * best score among the others (for the near-tie gap). */
typedef struct {
    double best, second;
    int64_t arg;
} scan_t;

static void scan_init(scan_t *s) { s->best = -INFINITY; s->second = -INFINITY; s->arg = -1; }

static void scan_push(scan_t *s, double score, int64_t x)
{
    if (s->arg < 0 || score > s->best) {
        if (s->arg >= 0) s->second = s->best;
        s->best = score;
        s->arg = x;
    } else if (score > s->second) {
        s->second = score;
    }
}

static double scan_gap(const scan_t *s)
{
    if (s->second == -INFINITY) return INFINITY;
    return s->best - s->second;
}

/* ------------------------------------------------------ stochastic verify */

/*
 * Sequences b in [b_begin, b_end) of a batch of B.  Layouts (element
 * strides, vocabulary contiguous):
 *   target[b][i][x] at b*t_sb + i*t_sp + x, i in [0, k]
 *   draft [b][i][x] at b*d_sb + i*d_sp + x, i in [0, k)
 *   tokens[b][i]    at b*k + i
 * Outputs ([B]-shaped, only rows b_begin..b_end-1 written):
 *   accepted_len[b], out_tokens[b][0..k], probs[b][i][0..1] = p_i(x_i),
 *   q_i(x_i); margins[b][i] = |u_i - p_i/q_i| (inf when q_i = 0 or the
 *   token is invalid); gaps[b] = best minus second-best score of the
 *   sampled row; flags[b] (bit 0: invalid draft token, bit 1: residual
 *   fallback).  probs, margins, gaps and flags may be NULL.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_verify_stochastic(const void *target, int t_dtype, int64_t t_sb, int64_t t_sp,
                             const void *draft, int d_dtype, int64_t d_sb, int64_t d_sp,
                             const int32_t *tokens, int B, int k, int V, double T,
                             uint64_t seed, uint32_t seq_offset, int b_begin, int b_end,
                             int32_t *accepted_len, int32_t *out_tokens, double *probs,
                             double *margins, double *gaps, int32_t *flags)
{
    if (!(T > 0.0) || V < 1 || k < 0 || B < 0 || b_begin < 0 || b_end > B)
        return -1;
    for (int b = b_begin; b < b_end; ++b) {
        uint32_t seq = (uint32_t)b + seq_offset;
        int32_t flag = 0;
        int n = k;
        /* every drafted position is scored, then the first rejection wins */
        for (int i = 0; i < k; ++i) {
            row_t rt = {target, t_dtype, (int64_t)b * t_sb + (int64_t)i * t_sp};
            row_t rd = {draft, d_dtype, (int64_t)b * d_sb + (int64_t)i * d_sp};
            int32_t x = tokens[(int64_t)b * k + i];
            double p = 0.0, q = 0.0;
            int valid = (x >= 0 && x < V);
            if (valid) {
                double mt, st, md, sd;
                softmax_stats(rt, V, T, &mt, &st);
                softmax_stats(rd, V, T, &md, &sd);
                p = softmax_prob(rt, x, T, mt, st);
                q = softmax_prob(rd, x, T, md, sd);
            } else {
                flag |= 1;
            }
            double u = accept_uniform(draw_word(seed, 0u, (uint32_t)i, seq, TAG_ACCEPT, 0));
            int accept = valid && (u * q < p);
            if (probs) {
                probs[((int64_t)b * k + i) * 2 + 0] = p;
                probs[((int64_t)b * k + i) * 2 + 1] = q;
            }
            if (margins)
                margins[(int64_t)b * k + i] = (valid && q > 0.0) ? fabs(u - p / q) : INFINITY;
            if (!accept && n == k)
                n = i;
        }

        scan_t sc;
        scan_init(&sc);
        int32_t y;
        if (n < k) {
            /* correction: Gumbel-max over ln(max(0, p_n - q_n)) */
            row_t rt = {target, t_dtype, (int64_t)b * t_sb + (int64_t)n * t_sp};
            row_t rd = {draft, d_dtype, (int64_t)b * d_sb + (int64_t)n * d_sp};
            double mt, st, md, sd;
            softmax_stats(rt, V, T, &mt, &st);
            softmax_stats(rd, V, T, &md, &sd);
            for (int64_t x = 0; x < V; ++x) {
                double r = softmax_prob(rt, x, T, mt, st) - softmax_prob(rd, x, T, md, sd);
                if (r > 0.0)
                    scan_push(&sc, log(r) + vocab_gumbel(seed, x, (uint32_t)n, seq, TAG_CORRECTION), x);
            }
            if (sc.arg < 0) {
                /* no positive residual mass: draw from p_n, same stream */
                flag |= 2;
                for (int64_t x = 0; x < V; ++x)
                    scan_push(&sc, row_at(rt, x) / T +
                                       vocab_gumbel(seed, x, (uint32_t)n, seq, TAG_CORRECTION), x);
            }
        } else {
            /* bonus: Gumbel-max over l_k / T, i.e. a draw from p_k */
            row_t rt = {target, t_dtype, (int64_t)b * t_sb + (int64_t)k * t_sp};
            for (int64_t x = 0; x < V; ++x)
                scan_push(&sc, row_at(rt, x) / T + vocab_gumbel(seed, x, (uint32_t)k, seq, TAG_BONUS), x);
        }
        y = (int32_t)sc.arg;

        accepted_len[b] = n;
        for (int i = 0; i <= k; ++i) {
            int32_t v = -1;
            if (i < n) v = tokens[(int64_t)b * k + i];
            else if (i == n) v = y;
            out_tokens[(int64_t)b * (k + 1) + i] = v;
        }
        if (gaps) gaps[b] = scan_gap(&sc);
        if (flags) flags[b] = flag;
    }
    return 0;
}

/* ------------------------------------------------- stochastic tree verify */

/*
 * Sequences b in [b_begin, b_end) of a batch of B trees of N nodes.
 * Layouts (element strides, vocabulary contiguous):
 *   logits[b][j][x] at b*sb + j*sn + x: the target's distribution after the
 *                   path root..j (node 0 is the root, the last committed
 *                   token)
 *   parent[b][j], tokens[b][j] at b*N + j (entries of node 0 unused); a node
 *                   j >= 1 with parent outside [0, j) is never entered
 * Outputs: accepted_len[b] = n; path[b][0..n] = accepted nodes from the
 * root, out_tokens[b][0..n] = their tokens then the drawn token (both -1
 * after); margins[b][j] = |u_j - p(x_j)/R| for every examined child j
 * (inf when it could not be accepted: invalid or repeated token; NaN when
 * not examined); gaps[b] = best minus second-best score of the final draw;
 * flags[b] (bit 0: invalid token, bit 1: no candidate left outside E, bit 5:
 * invalid parent).  margins, gaps and flags may be NULL.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_verify_tree_stochastic(const void *logits, int dtype, int64_t sb, int64_t sn,
                                  const int32_t *parent, const int32_t *tokens, int B, int N,
                                  int V, double T, uint64_t seed, uint32_t seq_offset,
                                  int b_begin, int b_end, int32_t *accepted_len, int32_t *path,
                                  int32_t *out_tokens, double *margins, double *gaps,
                                  int32_t *flags)
{
    if (!(T > 0.0) || V < 1 || N < 1 || N > 64 || B < 0 || b_begin < 0 || b_end > B)
        return -1;
    for (int b = b_begin; b < b_end; ++b) {
        const int32_t *par = parent + (int64_t)b * N;
        const int32_t *tok = tokens + (int64_t)b * N;
        uint32_t seq = (uint32_t)b + seq_offset;
        int32_t flag = 0;
        for (int j = 1; j < N; ++j)
            if (par[j] < 0 || par[j] >= j) flag |= 32;
        for (int j = 0; j < N; ++j) {
            if (margins) margins[(int64_t)b * N + j] = NAN;
            path[(int64_t)b * N + j] = -1;
            out_tokens[(int64_t)b * N + j] = -1;
        }

        int u = 0, n = 0;
        int32_t excl[64];
        int nexcl = 0, has_child = 0;
        path[(int64_t)b * N] = 0;
        for (;;) {
            row_t r = {logits, dtype, (int64_t)b * sb + (int64_t)u * sn};
            double m, s;
            softmax_stats(r, V, T, &m, &s);
            double R = 1.0;
            int next = -1;
            nexcl = 0;
            has_child = 0;
            for (int j = u + 1; j < N; ++j) {
                if (par[j] != u) continue;
                has_child = 1;
                int32_t x = tok[j];
                int valid = (x >= 0 && x < V);
                if (!valid) flag |= 1;
                int repeated = 0;
                for (int e = 0; e < nexcl; ++e)
                    if (excl[e] == x) repeated = 1;
                double uj = accept_uniform(draw_word(seed, 0u, (uint32_t)(j - 1), seq, TAG_ACCEPT, 0));
                double p = (valid && !repeated) ? softmax_prob(r, x, T, m, s) : 0.0;
                int open = valid && !repeated;
                if (margins)
                    margins[(int64_t)b * N + j] = (open && R > 0.0) ? fabs(uj - p / R) : INFINITY;
                if (open && uj * R < p) {
                    next = j;
                    break;
                }
                if (open) {
                    excl[nexcl++] = x;
                    R -= p;
                }
            }
            if (next < 0) break;
            u = next;
            out_tokens[(int64_t)b * N + n] = tok[u];
            ++n;
            path[(int64_t)b * N + n] = u;
        }

        /* the final draw: y ~ p_u outside E */
        row_t r = {logits, dtype, (int64_t)b * sb + (int64_t)u * sn};
        uint32_t tag = has_child ? TAG_CORRECTION : TAG_BONUS;
        scan_t sc;
        scan_init(&sc);
        for (int64_t x = 0; x < V; ++x) {
            double l = row_at(r, x);
            if (l == -INFINITY) continue;
            int in_e = 0;
            for (int e = 0; e < nexcl; ++e)
                if (excl[e] == x) in_e = 1;
            if (in_e) continue;
            scan_push(&sc, l / T + vocab_gumbel(seed, x, (uint32_t)u, seq, tag), x);
        }
        if (sc.arg < 0) {
            /* nothing left outside E (possible only through rounding) */
            flag |= 2;
            for (int64_t x = 0; x < V; ++x)
                scan_push(&sc, row_at(r, x) / T + vocab_gumbel(seed, x, (uint32_t)u, seq, tag), x);
        }
        out_tokens[(int64_t)b * N + n] = (int32_t)sc.arg;
        accepted_len[b] = n;
        if (gaps) gaps[b] = scan_gap(&sc);
        if (flags) flags[b] = flag;
    }
    return 0;
}

/* ---------------------------------------------------------- greedy verify */

/* First maximum of a row under '>' (so -0 == +0 and the lowest index wins). */
static int32_t row_argmax(row_t r, int V)
{
    double best = row_at(r, 0);
    int32_t arg = 0;
    for (int64_t x = 1; x < V; ++x) {
        double v = row_at(r, x);
        if (v > best) {
            best = v;
            arg = (int32_t)x;
        }
    }
    return arg;
}

/*
 * target[b][i][x] at b*t_sb + i*t_sp + x (i in [0, k]); tokens [B][k].
 * row_argmax_out (nullable) receives the argmax of every row, [B][k+1].
 */
int oracle_verify_greedy(const void *target, int t_dtype, int64_t t_sb, int64_t t_sp,
                         const int32_t *tokens, int B, int k, int V, int b_begin, int b_end,
                         int32_t *accepted_len, int32_t *out_tokens, int32_t *row_argmax_out)
{
    if (V < 1 || k < 0 || B < 0 || b_begin < 0 || b_end > B)
        return -1;
    for (int b = b_begin; b < b_end; ++b) {
        int n = k;
        int32_t a_n = -1;
        for (int i = 0; i <= k; ++i) {
            row_t rt = {target, t_dtype, (int64_t)b * t_sb + (int64_t)i * t_sp};
            int32_t a = row_argmax(rt, V);
            if (row_argmax_out) row_argmax_out[(int64_t)b * (k + 1) + i] = a;
            if (i < n && i < k && tokens[(int64_t)b * k + i] != a)
                n = i;
            if (i == n && a_n < 0)
                a_n = a;
        }
        accepted_len[b] = n;
        for (int i = 0; i <= k; ++i) {
            int32_t v = -1;
            if (i < n) v = tokens[(int64_t)b * k + i];
            else if (i == n) v = a_n;
            out_tokens[(int64_t)b * (k + 1) + i] = v;
        }
    }
    return 0;
}

/* ---------------------------------------------------- threshold acceptance */

/*
 * "Accelerating Sonar through speculation", section "Speculative decoding":
 * each candidate prefix is scored by its probability and the longest one at
 * or above an acceptance threshold is selected; the target gives one more
 * token.  Reading (the pages fix no scoring rule or threshold): the score of
 * the prefix of length j is its probability under the target,
 *     score(j) = prod_{i<j} p_i(x_i),   p_i = softmax(target[b,i,:] / T),
 * n = the largest j <= k with score(j) >= tau (score(0) = 1), and the extra
 * token is the target's argmax at row n (first maximum).  A draft token
 * outside [0, V) has p = 0.  log_scores[b*k + i] = ln score(i+1) for the
 * examined positions i <= n (i < k), -inf after a zero, for near-tie checks.
 */
int oracle_verify_threshold(const void *target, int t_dtype, int64_t t_sb, int64_t t_sp,
                            const int32_t *tokens, int B, int k, int V, double T, double tau,
                            int b_begin, int b_end, int32_t *accepted_len,
                            int32_t *out_tokens, double *log_scores)
{
    if (V < 1 || k < 0 || B < 0 || b_begin < 0 || b_end > B || !(T > 0.0) ||
        !(tau > 0.0) || !(tau <= 1.0))
        return -1;
    const double log_tau = log(tau);
    for (int b = b_begin; b < b_end; ++b) {
        int n = k;
        double acc = 0.0; /* ln score(i+1) */
        for (int i = 0; i < k; ++i) {
            row_t rt = {target, t_dtype, (int64_t)b * t_sb + (int64_t)i * t_sp};
            int32_t x = tokens[(int64_t)b * k + i];
            double lp = -INFINITY;
            if (x >= 0 && x < V) {
                double m, s;
                softmax_stats(rt, V, T, &m, &s);
                lp = log(softmax_prob(rt, x, T, m, s));
            }
            acc += lp;
            if (log_scores) log_scores[(int64_t)b * k + i] = acc;
            if (!(acc >= log_tau)) {
                n = i;
                break;
            }
        }
        if (log_scores)
            for (int i = n + 1; i < k; ++i) log_scores[(int64_t)b * k + i] = NAN;
        row_t rn = {target, t_dtype, (int64_t)b * t_sb + (int64_t)n * t_sp};
        int32_t a_n = row_argmax(rn, V);
        accepted_len[b] = n;
        for (int i = 0; i <= k; ++i) {
            int32_t v = -1;
            if (i < n) v = tokens[(int64_t)b * k + i];
            else if (i == n) v = a_n;
            out_tokens[(int64_t)b * (k + 1) + i] = v;
        }
    }
    return 0;
}

/* ------------------------------------------------- multi-candidate verify */

/*
 * target[b][g][i][x] at b*t_sb + g*t_sg + i*t_sp + x (i in [0, k]);
 * cand [B][G][k] contiguous.  best_g[b], accepted_len[b], out_tokens[b][0..k].
 * If every branch has length 0, branch 0 is chosen.
 */
int oracle_verify_multi(const void *target, int t_dtype, int64_t t_sb, int64_t t_sg,
                        int64_t t_sp, const int32_t *cand, int B, int G, int k, int V,
                        int b_begin, int b_end, int32_t *best_g, int32_t *accepted_len,
                        int32_t *out_tokens)
{
    if (V < 1 || k < 0 || B < 0 || G < 1 || b_begin < 0 || b_end > B)
        return -1;
    for (int b = b_begin; b < b_end; ++b) {
        int best = -1, best_n = -1;
        int32_t best_next = -1;
        for (int g = 0; g < G; ++g) {
            const int32_t *c = cand + ((int64_t)b * G + g) * k;
            int n = k;
            int32_t next = -1;
            for (int i = 0; i <= k; ++i) {
                row_t rt = {target, t_dtype,
                            (int64_t)b * t_sb + (int64_t)g * t_sg + (int64_t)i * t_sp};
                int32_t a = row_argmax(rt, V);
                if (i < k && c[i] != a) {
                    n = i;
                    next = a;
                    break;
                }
                if (i == k) next = a;
            }
            if (n > best_n) {
                best_n = n;
                best = g;
                best_next = next;
            }
        }
        const int32_t *c = cand + ((int64_t)b * G + best) * k;
        best_g[b] = best;
        accepted_len[b] = best_n;
        for (int i = 0; i <= k; ++i) {
            int32_t v = -1;
            if (i < best_n) v = c[i];
            else if (i == best_n) v = best_next;
            out_tokens[(int64_t)b * (k + 1) + i] = v;
        }
    }
    return 0;
}
