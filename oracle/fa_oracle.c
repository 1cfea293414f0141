/*
 * Oracle for the masked attention forward: plain, slow, fp64 CPU code.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the independent checker that the
 * CUDA path is compared against. Nothing in the product path includes, links
 * or calls it; it shares no header, helper or constant with the CUDA library.
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * load it.
 *
 * What it computes, and where each step comes from:
 *   - Visibility of key j to query i (the "Masked QK^T" geometry) for every
 *     sparseMode 0..8, decided element by element from the prose of the
 *     Ascend CANN page "sparseMode参数说明" (sections sparseMode=0 .. =8) and
 *     the attenMask rule on the same page (a True mask entry hides that QK^T
 *     position).
 *   - The attention itself as its plain definition: S = scale * Q K^T,
 *     softmax over the visible keys of each row, O = P V, and the per-row
 *     natural log-sum-exp. A row with no visible key gives O = 0, lse = -inf.
 *   - The occupancy of the visibility matrix by 128 x 128 blocks (which
 *     blocks hold no visible pair, which hold only visible pairs) and the
 *     range of key blocks each query block must visit: the sparseMode page
 *     has the operator compute only the part the mask and the band leave
 *     visible, and these are that statement summarised by block.
 *   - The same forward with keys and values read from paged caches (the
 *     "Norm" layout of the aclnnScatterPaKvCache page, scenario 2) through
 *     a per-sequence block table.
 *   - An optional ALiBi bias added to the scores of the visible pairs, as
 *     the Ascend ATB page "压缩mask" (alibi section) decomposes the alibi
 *     mask: a per-head coefficient (slopes) times an alibi bias, plus the
 *     triangular mask. Three biases, one per variant of that section:
 *     right-aligned, its square root, and left-aligned.
 *   - The tiled online-softmax recurrence (running max m_i, running sum l_i,
 *     normalised output) of the "FlashAttention tiling & online softmax"
 *     exercise page (section "Mục tiêu kiến thức"), used only to pin the
 *     recurrence against the unfused softmax.
 *
 * Readings of points the pages leave open (each one is listed with its
 * justification in the design notes):
 *   - Band bounds are inclusive: i - j <= pre and j - i <= next.
 *   - "Origin at the bottom-right" re-anchors row i at i + (Skv - Sq).
 *   - mode 5/6: rightDownCausal OR column j < prefix[b] (prefix block is
 *     anchored at the left edge for every row).
 *   - mode 7: the last sequence with Sq_b > 0 uses the mode-4 rule, all the
 *     others the mode-3 rule; mode 8: the first sequence with Sq_b > 0 uses
 *     the mode-4 rule, all the others the mode-2 rule.
 *   - Cumulative length arrays hold end offsets without a leading 0.
 *   - mode 0 without a mask computes everything (pre/next ignored); with a
 *     mask, the band AND the mask decide.
 *   - ALiBi (the page's formula and figures are lost): the right-aligned
 *     bias is the key's signed distance from the row's bottom-right-anchored
 *     diagonal, j - (i + Skv_b - Sq_b), 0 on the diagonal and negative to
 *     its left; the square-root variant takes the square root of that
 *     distance's size and keeps its sign; the left-aligned bias is the key
 *     position j itself (it differs from the right-aligned one by a
 *     constant per row, so only lse moves). The score is
 *     scale * q.k + slope_h * bias.
 *
 * Parity status: every function here is pinned by the CPU tests
 * (tests/test_oracle_pins.py) against library routines, closed forms and the
 * pages' worked examples. Parity is pinned for all functions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Layouts of Q/K/V/O (and the matching lse layout). */
enum { OR_BNSD = 0, OR_BSND = 1, OR_TND = 2 };
/* Shapes of the optional attenMask. */
enum { OR_MASK_NONE = 0, OR_MASK_SS = 1, OR_MASK_B1SS = 2, OR_MASK_BNSS = 3 };

typedef struct {
    int32_t layout;
    int32_t sparse_mode;
    int32_t mask_kind;
    int32_t pad_;
    int64_t B, N, Sq, Skv, D;     /* TND: Sq, Skv are the token totals */
    int64_t pre_tokens, next_tokens;
    double scale;
} oracle_desc;

/* Per-sequence extents: query/key token offsets and lengths. */
typedef struct {
    int64_t q_off, kv_off, sq, skv;
} seq_info;

static seq_info seq_of(const oracle_desc* d, const int64_t* cu_q,
                       const int64_t* cu_kv, int64_t b) {
    seq_info s;
    if (d->layout == OR_TND) {
        /* Cumulative ends without a leading 0: {3,5} means lengths 3 and 2. */
        s.q_off = b == 0 ? 0 : cu_q[b - 1];
        s.kv_off = b == 0 ? 0 : cu_kv[b - 1];
        s.sq = cu_q[b] - s.q_off;
        s.skv = cu_kv[b] - s.kv_off;
    } else {
        s.q_off = 0;
        s.kv_off = 0;
        s.sq = d->Sq;
        s.skv = d->Skv;
    }
    return s;
}

/* Band between pre and next, origin at the top-left corner (mode 0). */
static int band_top_left(int64_t i, int64_t j, int64_t pre, int64_t next) {
    return (i - j <= pre) && (j - i <= next);
}

/* Band between pre and next, origin at the bottom-right corner (mode 4):
 * the row is re-anchored so that the last query row meets the last key. */
static int band_bottom_right(int64_t i, int64_t j, int64_t sq, int64_t skv,
                             int64_t pre, int64_t next) {
    int64_t ir = i + (skv - sq);
    return (ir - j <= pre) && (j - ir <= next);
}

/* leftUpCausal: lower triangle split at the top-left vertex (mode 2). */
static int causal_left_up(int64_t i, int64_t j) { return j <= i; }

/* rightDownCausal: lower triangle split at the bottom-right vertex (mode 3). */
static int causal_right_down(int64_t i, int64_t j, int64_t sq, int64_t skv) {
    return j <= i + (skv - sq);
}

static int64_t mask_index(const oracle_desc* d, int64_t b, int64_t h,
                          int64_t i, int64_t j) {
    switch (d->mask_kind) {
    case OR_MASK_SS:
        return i * d->Skv + j;
    case OR_MASK_B1SS:
        return (b * d->Sq + i) * d->Skv + j;
    default: /* BNSS */
        return ((b * d->N + h) * d->Sq + i) * d->Skv + j;
    }
}

/* Index of the first / last sequence that has at least one query row. */
static int64_t first_nonempty(const oracle_desc* d, const int64_t* cu_q,
                              const int64_t* cu_kv) {
    for (int64_t b = 0; b < d->B; ++b)
        if (seq_of(d, cu_q, cu_kv, b).sq > 0) return b;
    return -1;
}
static int64_t last_nonempty(const oracle_desc* d, const int64_t* cu_q,
                             const int64_t* cu_kv) {
    for (int64_t b = d->B - 1; b >= 0; --b)
        if (seq_of(d, cu_q, cu_kv, b).sq > 0) return b;
    return -1;
}

/*
 * Does key j of sequence b contribute to query i of that sequence (head h)?
 * i and j are positions inside the sequence. One branch per sparseMode
 * section of the Ascend page.
 */
int oracle_visible(const oracle_desc* d, const int64_t* prefix,
                   const int64_t* cu_q, const int64_t* cu_kv,
                   const uint8_t* mask, int64_t b, int64_t h, int64_t i,
                   int64_t j) {
    seq_info s = seq_of(d, cu_q, cu_kv, b);
    if (i < 0 || i >= s.sq || j < 0 || j >= s.skv) return 0;
    switch (d->sparse_mode) {
    case 0:
        /* No mask: nothing is masked and pre/next are ignored.
         * With a mask: the part between pre and next is computed, and a
         * True mask entry hides its position. */
        if (mask == NULL || d->mask_kind == OR_MASK_NONE) return 1;
        if (!band_top_left(i, j, d->pre_tokens, d->next_tokens)) return 0;
        return mask[mask_index(d, b, h, i, j)] == 0;
    case 1:
        /* allMask: the full mask decides; pre/next are ignored. */
        return mask[mask_index(d, b, h, i, j)] == 0;
    case 2:
        return causal_left_up(i, j);
    case 3:
        return causal_right_down(i, j, s.sq, s.skv);
    case 4:
        return band_bottom_right(i, j, s.sq, s.skv, d->pre_tokens,
                                 d->next_tokens);
    case 5:
    case 6:
        /* rightDownCausal plus a block Sq long and prefix[b] wide on the
         * left. */
        return causal_right_down(i, j, s.sq, s.skv) || (j < prefix[b]);
    case 7:
        /* Split from a mode-3 job: the last non-empty sequence is the band. */
        if (b == last_nonempty(d, cu_q, cu_kv))
            return band_bottom_right(i, j, s.sq, s.skv, d->pre_tokens,
                                     d->next_tokens);
        return causal_right_down(i, j, s.sq, s.skv);
    case 8:
        /* Split from a mode-2 job: the first non-empty sequence is the band. */
        if (b == first_nonempty(d, cu_q, cu_kv))
            return band_bottom_right(i, j, s.sq, s.skv, d->pre_tokens,
                                     d->next_tokens);
        return causal_left_up(i, j);
    default:
        return 0;
    }
}

/* Element offset of token t (sequence-local position already resolved to a
 * global row) of head h, batch b, in the given layout. */
static int64_t row_offset(const oracle_desc* d, int64_t S, int64_t b,
                          int64_t h, int64_t t) {
    switch (d->layout) {
    case OR_BNSD:
        return ((b * d->N + h) * S + t) * d->D;
    case OR_BSND:
        return ((b * S + t) * d->N + h) * d->D;
    default: /* TND: t is the packed token index */
        return (t * d->N + h) * d->D;
    }
}

static int64_t lse_offset(const oracle_desc* d, int64_t b, int64_t h,
                          int64_t t) {
    if (d->layout == OR_TND) return h * d->Sq + t; /* [N, T_q] */
    return (b * d->N + h) * d->Sq + t;             /* [B, N, Sq] */
}

/* ALiBi variants (the three biases of the "压缩mask" page's alibi
 * section). */
enum { OR_ALIBI_NONE = 0, OR_ALIBI_RIGHT = 1, OR_ALIBI_SQRT = 2, OR_ALIBI_LEFT = 3 };

/* The alibi bias of query i and key j of a sequence with sq rows and skv
 * keys (positions inside the sequence). */
static double alibi_bias(int kind, int64_t i, int64_t j, int64_t sq, int64_t skv) {
    /* signed distance from the diagonal anchored at the bottom-right corner */
    const double dist = (double)(j - (i + (skv - sq)));
    switch (kind) {
    case OR_ALIBI_RIGHT:
        return dist;
    case OR_ALIBI_SQRT:
        return dist < 0 ? -sqrt(-dist) : sqrt(dist);
    case OR_ALIBI_LEFT:
        return (double)j;
    default:
        return 0.0;
    }
}

/*
 * One query row of the plain attention definition:
 *   s_j = scale * sum_d q_d k_jd (+ bias_row[j]) for the visible j,
 *   m = max s_j, l = sum exp(s_j - m), o = sum exp(s_j - m) v_j / l,
 *   lse = m + ln l.
 * vis_row holds the explicit visibility of the row's keys; bias_row (or
 * NULL) an additive term per key.
 */
static void attend_row(const oracle_desc* d, const double* q, const double* k,
                       const double* v, int64_t b, int64_t h, seq_info s,
                       int64_t i, const uint8_t* vis_row, const double* bias_row,
                       double* scores, double* o_row, double* lse_out) {
    const int64_t D = d->D;
    const double* qi = q + row_offset(d, d->Sq, b, h, s.q_off + i);
    double m = -INFINITY;
    for (int64_t j = 0; j < s.skv; ++j) {
        if (!vis_row[j]) continue;
        const double* kj = k + row_offset(d, d->Skv, b, h, s.kv_off + j);
        double acc = 0.0;
        for (int64_t x = 0; x < D; ++x) acc += qi[x] * kj[x];
        scores[j] = d->scale * acc + (bias_row ? bias_row[j] : 0.0);
        if (scores[j] > m) m = scores[j];
    }
    for (int64_t x = 0; x < D; ++x) o_row[x] = 0.0;
    if (m == -INFINITY) { /* no visible key */
        *lse_out = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int64_t j = 0; j < s.skv; ++j) {
        if (!vis_row[j]) continue;
        double p = exp(scores[j] - m);
        l += p;
        const double* vj = v + row_offset(d, d->Skv, b, h, s.kv_off + j);
        for (int64_t x = 0; x < D; ++x) o_row[x] += p * vj[x];
    }
    for (int64_t x = 0; x < D; ++x) o_row[x] /= l;
    *lse_out = m + log(l);
}

/*
 * Full forward with an optional ALiBi bias: O (same layout as Q) and lse for
 * every (b, h, row). For each (b, h) the explicit Sq_b x Skv_b boolean
 * visibility matrix is built first, then the plain softmax is applied row by
 * row, each visible score plus slopes[h] * alibi_bias(...) when alibi_kind
 * is not OR_ALIBI_NONE (slopes: [N]).
 */
int oracle_attn_alibi(const oracle_desc* d, const int64_t* prefix,
                      const int64_t* cu_q, const int64_t* cu_kv,
                      const uint8_t* mask, int32_t alibi_kind,
                      const double* slopes, const double* q, const double* k,
                      const double* v, double* o, double* lse) {
    const int64_t nb = d->B, nh = d->N;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t h = 0; h < nh; ++h) {
            seq_info s = seq_of(d, cu_q, cu_kv, b);
            if (s.sq <= 0) continue;
            int64_t skv_alloc = s.skv > 0 ? s.skv : 1;
            uint8_t* vis = (uint8_t*)malloc((size_t)(s.sq * skv_alloc));
            double* scores = (double*)malloc(sizeof(double) * skv_alloc);
            double* bias = (double*)malloc(sizeof(double) * skv_alloc);
            if (!vis || !scores || !bias) {
                free(vis);
                free(scores);
                free(bias);
#pragma omp atomic write
                err = 1;
                continue;
            }
            for (int64_t i = 0; i < s.sq; ++i)
                for (int64_t j = 0; j < s.skv; ++j)
                    vis[i * skv_alloc + j] = (uint8_t)oracle_visible(
                        d, prefix, cu_q, cu_kv, mask, b, h, i, j);
            for (int64_t i = 0; i < s.sq; ++i) {
                double* o_row = o + row_offset(d, d->Sq, b, h, s.q_off + i);
                if (alibi_kind != OR_ALIBI_NONE)
                    for (int64_t j = 0; j < s.skv; ++j)
                        bias[j] = slopes[h] * alibi_bias(alibi_kind, i, j, s.sq, s.skv);
                attend_row(d, q, k, v, b, h, s, i, vis + i * skv_alloc,
                           alibi_kind != OR_ALIBI_NONE ? bias : NULL, scores,
                           o_row, lse + lse_offset(d, b, h, s.q_off + i));
            }
            free(vis);
            free(scores);
            free(bias);
        }
    }
    return err;
}

/* The forward without a bias. */
int oracle_attn(const oracle_desc* d, const int64_t* prefix,
                const int64_t* cu_q, const int64_t* cu_kv,
                const uint8_t* mask, const double* q, const double* k,
                const double* v, double* o, double* lse) {
    return oracle_attn_alibi(d, prefix, cu_q, cu_kv, mask, OR_ALIBI_NONE, NULL,
                             q, k, v, o, lse);
}

/*
 * Selected rows only, for spot checks of large problems: rows[3*r + 0..2] =
 * (b, h, i) with i the position inside sequence b. o_rows is [nrows, D].
 * The bias, when alibi_kind is set, is oracle_attn_alibi's.
 */
int oracle_attn_rows_alibi(const oracle_desc* d, const int64_t* prefix,
                           const int64_t* cu_q, const int64_t* cu_kv,
                           const uint8_t* mask, int32_t alibi_kind,
                           const double* slopes, const double* q, const double* k,
                           const double* v, int64_t nrows, const int64_t* rows,
                           double* o_rows, double* lse_rows) {
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        seq_info s = seq_of(d, cu_q, cu_kv, b);
        int64_t skv_alloc = s.skv > 0 ? s.skv : 1;
        uint8_t* vis = (uint8_t*)malloc((size_t)skv_alloc);
        double* scores = (double*)malloc(sizeof(double) * skv_alloc);
        double* bias = (double*)malloc(sizeof(double) * skv_alloc);
        if (!vis || !scores || !bias) {
            free(vis);
            free(scores);
            free(bias);
#pragma omp atomic write
            err = 1;
            continue;
        }
        for (int64_t j = 0; j < s.skv; ++j) {
            vis[j] = (uint8_t)oracle_visible(d, prefix, cu_q, cu_kv, mask, b,
                                             h, i, j);
            if (alibi_kind != OR_ALIBI_NONE)
                bias[j] = slopes[h] * alibi_bias(alibi_kind, i, j, s.sq, s.skv);
        }
        attend_row(d, q, k, v, b, h, s, i, vis,
                   alibi_kind != OR_ALIBI_NONE ? bias : NULL, scores,
                   o_rows + r * d->D, lse_rows + r);
        free(vis);
        free(scores);
        free(bias);
    }
    return err;
}

int oracle_attn_rows(const oracle_desc* d, const int64_t* prefix,
                     const int64_t* cu_q, const int64_t* cu_kv,
                     const uint8_t* mask, const double* q, const double* k,
                     const double* v, int64_t nrows, const int64_t* rows,
                     double* o_rows, double* lse_rows) {
    return oracle_attn_rows_alibi(d, prefix, cu_q, cu_kv, mask, OR_ALIBI_NONE,
                                  NULL, q, k, v, nrows, rows, o_rows, lse_rows);
}

/*
 * Key or value row of logical key j of sequence b, head h, in a paged cache
 * laid out as [num_blocks, block_size, N, D], the "Norm" cache of the
 * aclnnScatterPaKvCache page (scenario 2). A token is written to slot
 * block * block_size + offset; sequence b's key j sits in block
 * block_table[b][j / block_size] at offset j % block_size.
 */
static const double* paged_row(const double* cache, const int32_t* block_table,
                               int64_t max_blocks, int64_t block_size,
                               int64_t N, int64_t D, int64_t b, int64_t h,
                               int64_t j) {
    const int64_t blk = block_table[b * max_blocks + j / block_size];
    const int64_t slot = blk * block_size + j % block_size;
    return cache + (slot * N + h) * D;
}

/*
 * Forward with the keys and values read from paged caches instead of packed
 * TND tensors. q, o: [T_q, N, D] (TND); lse: [N, T_q]; the visibility rule,
 * the lengths (cumulative cu_q / cu_kv) and the plain softmax are those of
 * oracle_attn; only where key j of sequence b is stored differs.
 */
int oracle_attn_paged(const oracle_desc* d, const int64_t* prefix,
                      const int64_t* cu_q, const int64_t* cu_kv,
                      const double* q, const double* k_cache,
                      const double* v_cache, const int32_t* block_table,
                      int64_t max_blocks, int64_t block_size, double* o,
                      double* lse) {
    int err = 0;
    const int64_t nb = d->B, nh = d->N, D = d->D;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t h = 0; h < nh; ++h) {
            seq_info s = seq_of(d, cu_q, cu_kv, b);
            int64_t skv_alloc = s.skv > 0 ? s.skv : 1;
            double* scores = (double*)malloc(sizeof(double) * skv_alloc);
            if (!scores) {
#pragma omp atomic write
                err = 1;
                continue;
            }
            for (int64_t i = 0; i < s.sq; ++i) {
                const double* qi = q + row_offset(d, d->Sq, b, h, s.q_off + i);
                double* oi = o + row_offset(d, d->Sq, b, h, s.q_off + i);
                double m = -INFINITY;
                for (int64_t j = 0; j < s.skv; ++j) {
                    scores[j] = -INFINITY;
                    if (!oracle_visible(d, prefix, cu_q, cu_kv, NULL, b, h, i, j))
                        continue;
                    const double* kj = paged_row(k_cache, block_table, max_blocks,
                                                 block_size, nh, D, b, h, j);
                    double acc = 0.0;
                    for (int64_t x = 0; x < D; ++x) acc += qi[x] * kj[x];
                    scores[j] = d->scale * acc;
                    if (scores[j] > m) m = scores[j];
                }
                for (int64_t x = 0; x < D; ++x) oi[x] = 0.0;
                double* li = lse + lse_offset(d, b, h, s.q_off + i);
                if (m == -INFINITY) {
                    *li = -INFINITY;
                    continue;
                }
                double l = 0.0;
                for (int64_t j = 0; j < s.skv; ++j) {
                    if (scores[j] == -INFINITY) continue;
                    const double p = exp(scores[j] - m);
                    l += p;
                    const double* vj = paged_row(v_cache, block_table, max_blocks,
                                                 block_size, nh, D, b, h, j);
                    for (int64_t x = 0; x < D; ++x) oi[x] += p * vj[x];
                }
                for (int64_t x = 0; x < D; ++x) oi[x] /= l;
                *li = m + log(l);
            }
            free(scores);
        }
    }
    return err;
}

/* Explicit visibility matrix of sequence b, head h: out is [Sq_b, Skv_b]. */
void oracle_mask(const oracle_desc* d, const int64_t* prefix,
                 const int64_t* cu_q, const int64_t* cu_kv,
                 const uint8_t* mask, int64_t b, int64_t h, uint8_t* out) {
    seq_info s = seq_of(d, cu_q, cu_kv, b);
    for (int64_t i = 0; i < s.sq; ++i)
        for (int64_t j = 0; j < s.skv; ++j)
            out[i * s.skv + j] = (uint8_t)oracle_visible(d, prefix, cu_q,
                                                         cu_kv, mask, b, h, i, j);
}

/*
 * Occupancy of the visibility matrix of sequence b, head h, summarised by
 * blocks of `tile` query rows x `tile` keys: out[qt * n_kt + kt] with
 * n_kt = ceil(Skv_b / tile) is
 *   0  when no pair of the block is visible,
 *   2  when every row of the block that exists (i < Sq_b) sees every one of
 *      the block's `tile` keys and all of them exist (j < Skv_b),
 *   1  otherwise.
 * This is what an attention over the matrix may skip (0) or compute without
 * looking at the mask (2); it follows from the visibility rule alone.
 */
void oracle_tile_classes(const oracle_desc* d, const int64_t* prefix,
                         const int64_t* cu_q, const int64_t* cu_kv,
                         const uint8_t* mask, int64_t b, int64_t h,
                         int64_t tile, uint8_t* out) {
    seq_info s = seq_of(d, cu_q, cu_kv, b);
    const int64_t n_qt = (s.sq + tile - 1) / tile;
    const int64_t n_kt = (s.skv + tile - 1) / tile;
    for (int64_t qt = 0; qt < n_qt; ++qt) {
        for (int64_t kt = 0; kt < n_kt; ++kt) {
            int any = 0, all = 1;
            for (int64_t i = qt * tile; i < (qt + 1) * tile && i < s.sq; ++i) {
                for (int64_t j = kt * tile; j < (kt + 1) * tile; ++j) {
                    const int v = j < s.skv &&
                                  oracle_visible(d, prefix, cu_q, cu_kv, mask,
                                                 b, h, i, j);
                    any |= v;
                    all &= v;
                }
            }
            out[qt * n_kt + kt] = (uint8_t)(any ? (all ? 2 : 1) : 0);
        }
    }
}

/*
 * The key-block range each query block of a class matrix (as written by
 * oracle_tile_classes, n_qt x n_kt) has to visit: out[4 qt + 0..3] =
 *   lo, hi         the first non-empty block and one past the last one;
 *   full_lo, full_hi  the longest run of consecutive class-2 blocks, the
 *                  earliest of equally long runs, or lo, lo when there is
 *                  no class-2 block.
 * A query block whose blocks are all empty gets 0, 0, 0, 0.
 */
void oracle_tile_ranges(const uint8_t* cls, int64_t n_qt, int64_t n_kt,
                        int32_t* out) {
    for (int64_t qt = 0; qt < n_qt; ++qt) {
        const uint8_t* c = cls + qt * n_kt;
        int64_t lo = -1, hi = 0, best_lo = 0, best_len = 0;
        for (int64_t kt = 0; kt < n_kt; ++kt) {
            if (c[kt] != 0) {
                if (lo < 0) lo = kt;
                hi = kt + 1;
            }
            if (c[kt] == 2 && (kt == 0 || c[kt - 1] != 2)) {
                int64_t e = kt;
                while (e < n_kt && c[e] == 2) ++e;
                if (e - kt > best_len) {
                    best_len = e - kt;
                    best_lo = kt;
                }
            }
        }
        int32_t* r = out + 4 * qt;
        if (lo < 0) {
            r[0] = r[1] = r[2] = r[3] = 0;
        } else {
            r[0] = (int32_t)lo;
            r[1] = (int32_t)hi;
            r[2] = (int32_t)(best_len > 0 ? best_lo : lo);
            r[3] = (int32_t)(best_len > 0 ? best_lo + best_len : lo);
        }
    }
}

/* Number of visible (b, h, i, j) pairs, by enumeration. */
int64_t oracle_visible_count(const oracle_desc* d, const int64_t* prefix,
                             const int64_t* cu_q, const int64_t* cu_kv,
                             const uint8_t* mask) {
    int64_t total = 0;
    const int64_t nb = d->B, nh = d->N;
#pragma omp parallel for collapse(2) reduction(+ : total) schedule(dynamic, 1)
    for (int64_t b = 0; b < nb; ++b) {
        for (int64_t h = 0; h < nh; ++h) {
            seq_info s = seq_of(d, cu_q, cu_kv, b);
            int64_t c = 0;
            for (int64_t i = 0; i < s.sq; ++i)
                for (int64_t j = 0; j < s.skv; ++j)
                    c += oracle_visible(d, prefix, cu_q, cu_kv, mask, b, h, i, j);
            total += c;
        }
    }
    return total;
}

/*
 * The exercise page's tiled CPU attention, in the page's normalised form.
 * q, k, v, out are [B, S, D]; keys are visited in blocks of `block` (the
 * last block may be shorter). vis (optional, [B, S, S], 1 = visible) masks
 * keys; a block with no visible key for a row leaves that row's state as it
 * was. For each block:
 *   m_new = max(m_old, m_blk)
 *   l_new = l_old e^(m_old - m_new) + sum_j e^(s_j - m_new)
 *   O_new = (O_old l_old e^(m_old - m_new) + sum_j e^(s_j - m_new) v_j) / l_new
 */
void oracle_flash_tiled(const double* q, const double* k, const double* v,
                        const uint8_t* vis, int64_t B, int64_t S, int64_t D,
                        int64_t block, double scale, double* out) {
    double* s_blk = (double*)malloc(sizeof(double) * (size_t)block);
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t i = 0; i < S; ++i) {
            const double* qi = q + (b * S + i) * D;
            double* oi = out + (b * S + i) * D;
            double m_old = -INFINITY, l_old = 0.0;
            for (int64_t x = 0; x < D; ++x) oi[x] = 0.0;
            for (int64_t j0 = 0; j0 < S; j0 += block) {
                int64_t j1 = j0 + block < S ? j0 + block : S;
                double m_blk = -INFINITY;
                for (int64_t j = j0; j < j1; ++j) {
                    if (vis && !vis[(b * S + i) * S + j]) {
                        s_blk[j - j0] = -INFINITY;
                        continue;
                    }
                    const double* kj = k + (b * S + j) * D;
                    double acc = 0.0;
                    for (int64_t x = 0; x < D; ++x) acc += qi[x] * kj[x];
                    s_blk[j - j0] = scale * acc;
                    if (s_blk[j - j0] > m_blk) m_blk = s_blk[j - j0];
                }
                if (m_blk == -INFINITY) continue; /* nothing visible here */
                double m_new = m_old > m_blk ? m_old : m_blk;
                double carry = (m_old == -INFINITY) ? 0.0 : exp(m_old - m_new);
                double l_new = l_old * carry;
                for (int64_t j = j0; j < j1; ++j)
                    if (s_blk[j - j0] != -INFINITY) l_new += exp(s_blk[j - j0] - m_new);
                for (int64_t x = 0; x < D; ++x) {
                    double acc = oi[x] * l_old * carry;
                    for (int64_t j = j0; j < j1; ++j)
                        if (s_blk[j - j0] != -INFINITY)
                            acc += exp(s_blk[j - j0] - m_new) * v[(b * S + j) * D + x];
                    oi[x] = acc / l_new;
                }
                m_old = m_new;
                l_old = l_new;
            }
        }
    }
    free(s_blk);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
