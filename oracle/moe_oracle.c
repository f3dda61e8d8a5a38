/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle of MoE token
 * dispatch / combine.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
 * CPU-baseline leg are the only users.  It shares no code, header, table or
 * helper with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes (the plainest reading of the pages; every reading that
 * goes beyond them is listed in the design notes):
 *
 *   layout    -- Triton-distributed issue #117, test snippet (split counts
 *                and their cumulative sum feed the all-to-all) and Purlin
 *                section 3.1 "Layouts" (scattered-V buffer: contiguous,
 *                variable-sized partitions indexed by destination).  Every
 *                routed pair (t, k) with expert e = topk_idx[t,k] and
 *                partition p = part_of[e] gets an expert row: its position in
 *                the list of all valid pairs sorted by the key (p, e, t, k).
 *                Per-partition dedup (Zyphra news item, "correlated expert
 *                placement": a token goes to a GPU once whatever the number
 *                of its experts there) makes the dispatch rows the distinct
 *                (t, p) pairs, ordered by (p, t).
 *   dispatch  -- issue #117, all_to_all_kernel arguments (data_src ->
 *                data_dst, optional scale_src -> scale_dst "WITH_SCALE"):
 *                dispatch row r receives a bit copy of token row
 *                x[disp_token[r]]; with FP8, each 128-column block is cast to
 *                e4m3 (round to nearest even, saturate to +-448) after
 *                division by scale = amax / 448.
 *   combine   -- Purlin section 3.3 "The Atom", SCORE: one owner per output
 *                element, accumulation in source order.  out[t, c] =
 *                bf16_rne(fma chain over k = 0..topk-1 of
 *                w[t,k] * y[exp_row[t,k], c]) in fp32 starting from +0.
 *   tiles     -- DeepSpeed PR #8180, "Key points": the per-tile -> group map
 *                of a grouped GEMM over the expert rows, from the offsets.
 *   ep_plan   -- the counts exchange of an expert-parallel all-to-all over W
 *                ranks (partition p = rank p): Triton-distributed issue #117,
 *                test snippet (split_send_buf -> split_recv_buf,
 *                send_split_cumsum), and Purlin section 3.1, the transposed-V
 *                layout: destination r receives partition r of every source
 *                and arranges it in source-rank order.  From the matrix of
 *                every rank's per-partition row counts it gives each rank's
 *                offsets: where its rows go in every destination, where its
 *                rows start in every source, where every source's rows land
 *                in its own receive buffer, and per (source, expert) blocks.
 *
 * Invalid input (expert id outside [0, G), placement entry outside
 * [0, E_part)) is never an error of the call: the offending pairs are left out
 * (exp_row = -1) and a status word records it (bit 1: bad expert id, bit 2:
 * bad placement entry).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BAD_EXPERT 1
#define ORACLE_BAD_PART 2

/* ------------------------------------------------------------------------ */
/* layout                                                                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t p, e, t, k;
} orc_pair_t;

static int orc_cmp_pair(const void *a, const void *b)
{
    const orc_pair_t *x = (const orc_pair_t *)a, *y = (const orc_pair_t *)b;
    if (x->p != y->p) return x->p < y->p ? -1 : 1;
    if (x->e != y->e) return x->e < y->e ? -1 : 1;
    if (x->t != y->t) return x->t < y->t ? -1 : 1;
    if (x->k != y->k) return x->k < y->k ? -1 : 1;
    return 0;
}

/* expert order of the expert-row space: by (partition, id); experts with an
 * invalid partition sort last (they own no rows) */
static int32_t orc_E_part_for_sort;
static const int32_t *orc_part_of_for_sort;

static int orc_expert_key_part(int32_t e)
{
    int32_t p = orc_part_of_for_sort[e];
    return (p >= 0 && p < orc_E_part_for_sort) ? p : orc_E_part_for_sort;
}

static int orc_cmp_expert(const void *a, const void *b)
{
    int32_t ea = *(const int32_t *)a, eb = *(const int32_t *)b;
    int pa = orc_expert_key_part(ea), pb = orc_expert_key_part(eb);
    if (pa != pb) return pa < pb ? -1 : 1;
    return ea < eb ? -1 : (ea > eb ? 1 : 0);
}

/*
 * Outputs (all caller-allocated):
 *   expert_count [G], expert_offset [G+1], part_count [E_part],
 *   part_offset [E_part+1], exp_row [M*topk], disp_token [M*topk],
 *   disp_row [M*E_part] (dedup only, else may be NULL),
 *   exp_to_disp [M*topk] (dedup only, else may be NULL), status [1].
 * Rows of disp_token / exp_to_disp beyond the totals are left untouched.
 * Returns 0, or -1 when a host allocation fails.
 */
int oracle_layout(int32_t M, int32_t G, int32_t topk, int32_t E_part,
                  int32_t dedup, const int32_t *topk_idx,
                  const int32_t *part_of, int32_t *expert_count,
                  int32_t *expert_offset, int32_t *part_count,
                  int32_t *part_offset, int32_t *exp_row, int32_t *disp_token,
                  int32_t *disp_row, int32_t *exp_to_disp, int32_t *status)
{
    int32_t st = 0;
    for (int32_t e = 0; e < G; ++e)
        if (part_of[e] < 0 || part_of[e] >= E_part) st |= ORACLE_BAD_PART;

    int64_t n_pairs = (int64_t)M * topk;
    orc_pair_t *pairs = (orc_pair_t *)malloc(sizeof(orc_pair_t) * (size_t)(n_pairs > 0 ? n_pairs : 1));
    int32_t *experts = (int32_t *)malloc(sizeof(int32_t) * (size_t)(G > 0 ? G : 1));
    if (!pairs || !experts) {
        free(pairs);
        free(experts);
        return -1;
    }

    /* 1. the list of valid routed pairs */
    int64_t n = 0;
    for (int32_t t = 0; t < M; ++t) {
        for (int32_t k = 0; k < topk; ++k) {
            int64_t i = (int64_t)t * topk + k;
            int32_t e = topk_idx[i];
            exp_row[i] = -1;
            if (e < 0 || e >= G) {
                st |= ORACLE_BAD_EXPERT;
                continue;
            }
            int32_t p = part_of[e];
            if (p < 0 || p >= E_part) continue;
            pairs[n].p = p;
            pairs[n].e = e;
            pairs[n].t = t;
            pairs[n].k = k;
            ++n;
        }
    }

    /* 2. expert-row space = sorted order of the key (p, e, t, k) */
    qsort(pairs, (size_t)n, sizeof(orc_pair_t), orc_cmp_pair);
    for (int64_t r = 0; r < n; ++r)
        exp_row[(int64_t)pairs[r].t * topk + pairs[r].k] = (int32_t)r;

    for (int32_t e = 0; e < G; ++e) expert_count[e] = 0;
    for (int64_t r = 0; r < n; ++r) expert_count[pairs[r].e] += 1;

    /* expert_offset[e]: rows of all experts ordered before e by (p, e) */
    for (int32_t e = 0; e < G; ++e) experts[e] = e;
    orc_E_part_for_sort = E_part;
    orc_part_of_for_sort = part_of;
    qsort(experts, (size_t)G, sizeof(int32_t), orc_cmp_expert);
    int64_t run = 0;
    for (int32_t j = 0; j < G; ++j) {
        int32_t e = experts[j];
        int32_t p = part_of[e];
        if (p >= 0 && p < E_part) {
            expert_offset[e] = (int32_t)run;
            run += expert_count[e];
        } else {
            expert_offset[e] = (int32_t)n;
        }
    }
    expert_offset[G] = (int32_t)n;

    /* 3. dispatch-row space */
    if (!dedup) {
        for (int32_t p = 0; p < E_part; ++p) part_count[p] = 0;
        for (int64_t r = 0; r < n; ++r) part_count[pairs[r].p] += 1;
        for (int64_t r = 0; r < n; ++r) disp_token[r] = pairs[r].t;
    } else {
        /* distinct (t, p) pairs, enumerated in (p, t) order */
        unsigned char *has = (unsigned char *)calloc((size_t)M * (size_t)E_part + 1, 1);
        if (!has) {
            free(pairs);
            free(experts);
            return -1;
        }
        for (int64_t r = 0; r < n; ++r)
            has[(int64_t)pairs[r].t * E_part + pairs[r].p] = 1;
        int64_t d = 0;
        for (int32_t p = 0; p < E_part; ++p) {
            part_count[p] = 0;
            for (int32_t t = 0; t < M; ++t) {
                int64_t j = (int64_t)t * E_part + p;
                if (has[j]) {
                    disp_row[j] = (int32_t)d;
                    disp_token[d] = t;
                    ++d;
                    part_count[p] += 1;
                } else {
                    disp_row[j] = -1;
                }
            }
        }
        for (int64_t r = 0; r < n; ++r)
            exp_to_disp[r] = disp_row[(int64_t)pairs[r].t * E_part + pairs[r].p];
        free(has);
    }
    int64_t acc = 0;
    for (int32_t p = 0; p < E_part; ++p) {
        part_offset[p] = (int32_t)acc;
        acc += part_count[p];
    }
    part_offset[E_part] = (int32_t)acc;

    *status = st;
    free(pairs);
    free(experts);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* number formats                                                           */
/* ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32 */
static float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even; NaN stays a quiet NaN */
static uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* nearest integer of q >= 0 (q < 2^23), ties to the even integer */
static int32_t orc_round_half_even(float q)
{
    float fl = floorf(q);
    float frac = q - fl; /* exact */
    int32_t n = (int32_t)fl;
    if (frac > 0.5f) n += 1;
    else if (frac == 0.5f) n += (n & 1);
    return n;
}

/*
 * binary32 -> OCP FP8 E4M3 ("e4m3fn"): 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite value
 * S.1111.110 = 448, smallest normal 2^-6, subnormals m * 2^-9.  Rounds to
 * nearest, ties to even; a finite value whose rounding would leave the
 * finite range is clamped to +-448 (saturating).  The sign bit is kept, so
 * negative values that round to zero give 0x80.
 */
static uint8_t orc_e4m3(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint8_t sign = (u >> 31) ? 0x80 : 0x00;
    float a = fabsf(f);
    if (a != a) return (uint8_t)(sign | 0x7F);
    if (a >= 512.0f) return (uint8_t)(sign | 0x7E);
    if (a < 0.015625f) { /* below 2^-6: quantum 2^-9 */
        int32_t n = orc_round_half_even(a * 512.0f); /* 0..8; 8 = 2^-6 */
        return (uint8_t)(sign | n);
    }
    int ex;
    (void)frexpf(a, &ex); /* a = m * 2^ex, m in [0.5, 1) */
    int32_t E = ex - 1;   /* floor(log2 a), in [-6, 8] */
    int32_t n = orc_round_half_even(ldexpf(a, 3 - E)); /* 8..16 */
    if (n == 16) {
        E += 1;
        n = 8;
    }
    int32_t code = ((E + 7) << 3) | (n - 8);
    if (E > 8 || code > 0x7E) code = 0x7E;
    return (uint8_t)(sign | code);
}

void oracle_bf16_round(int64_t n, const float *in, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(in[i]);
}

void oracle_e4m3_encode(int64_t n, const float *in, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3(in[i]);
}

/* ------------------------------------------------------------------------ */
/* dispatch                                                                 */
/* ------------------------------------------------------------------------ */

/* one 128-column block of a token row -> 128 e4m3 bytes and one fp32 scale */
static void orc_quantize_block(const uint16_t *xb, uint8_t *q, float *scale)
{
    float amax = 0.0f;
    for (int j = 0; j < 128; ++j) {
        float v = fabsf(orc_bf16_to_f32(xb[j]));
        if (v > amax) amax = v;
    }
    if (amax == 0.0f) { /* all-zero block: no quotient exists */
        *scale = 0.0f;
        memset(q, 0, 128);
        return;
    }
    float s = amax / 448.0f;
    *scale = s;
    for (int j = 0; j < 128; ++j) q[j] = orc_e4m3(orc_bf16_to_f32(xb[j]) / s);
}

/*
 * Dispatch rows rows[0..n_rows) (rows == NULL: rows 0..n_rows-1) into a
 * compact output: out row i holds dispatch row rows[i].
 *   fp8 == 0: recv is uint16 (bf16 bits) [n_rows, N]
 *   fp8 != 0: recv is uint8 [n_rows, N], recv_scale fp32 [n_rows, N/128]
 */
void oracle_dispatch(int32_t N, int32_t fp8, int64_t n_rows,
                     const int64_t *rows, const int32_t *disp_token,
                     const uint16_t *x, void *recv, float *recv_scale)
{
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = rows ? rows[i] : i;
        const uint16_t *src = x + (int64_t)disp_token[r] * N;
        if (!fp8) {
            memcpy((uint16_t *)recv + i * N, src, sizeof(uint16_t) * (size_t)N);
        } else {
            int32_t nb = N / 128;
            for (int32_t b = 0; b < nb; ++b)
                orc_quantize_block(src + b * 128, (uint8_t *)recv + i * N + b * 128,
                                   recv_scale + i * nb + b);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* combine                                                                  */
/* ------------------------------------------------------------------------ */

/*
 * out row i = combined token tokens[i] (tokens == NULL: token i).
 * y is bf16 bits [R, N] in expert-row space; w fp32 [M, topk].
 * Returns 0, or -1 when a host allocation fails.
 */
int oracle_combine(int32_t N, int32_t topk, int64_t n_tok,
                   const int64_t *tokens, const uint16_t *y, const float *w,
                   const int32_t *exp_row, uint16_t *out)
{
    float *acc = (float *)malloc(sizeof(float) * (size_t)(N > 0 ? N : 1));
    if (!acc) return -1;
    for (int64_t i = 0; i < n_tok; ++i) {
        int64_t t = tokens ? tokens[i] : i;
        for (int32_t c = 0; c < N; ++c) acc[c] = 0.0f;
        for (int32_t k = 0; k < topk; ++k) {
            int32_t r = exp_row[t * topk + k];
            if (r < 0) continue;
            float wk = w[t * topk + k];
            const uint16_t *yr = y + (int64_t)r * N;
            for (int32_t c = 0; c < N; ++c)
                acc[c] = fmaf(wk, orc_bf16_to_f32(yr[c]), acc[c]);
        }
        for (int32_t c = 0; c < N; ++c) out[i * N + c] = orc_f32_to_bf16(acc[c]);
    }
    free(acc);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* two-level combine (dedup return path)                                    */
/* ------------------------------------------------------------------------ */

/*
 * With per-partition dedup a token was sent once per partition; on the way
 * back each partition first reduces the outputs of the token's experts it
 * holds (Zyphra news item: one copy per GPU; Purlin section 3.3, SCORE:
 * ordered accumulation), then the token's owner sums the partitions.
 *
 * Partition side: for every dispatch row r = disp_row[t, p],
 *   z[r, c] = bf16( fma chain over k = 0..topk-1 with part_of[idx[t,k]] = p
 *                   of w[t,k] * y[exp_row[t,k], c], from +0 )
 * Token side:
 *   out[t, c] = bf16( sum over p = 0..E_part-1 with disp_row[t,p] >= 0 of
 *                     float(z[disp_row[t,p], c]), fp32 additions from +0 )
 * Pairs left out by the layout (exp_row = -1) contribute nothing.
 *
 * oracle_combine_partial writes z rows (uint16 bf16 bits) in dispatch-row
 * space for the tokens tokens[0..n_tok) (NULL: all M); z has R rows.
 * Returns 0, or -1 when a host allocation fails.
 */
int oracle_combine_partial(int32_t N, int32_t topk, int32_t E_part, int32_t G,
                           int64_t n_tok, const int64_t *tokens,
                           const int32_t *topk_idx, const int32_t *part_of,
                           const uint16_t *y, const float *w,
                           const int32_t *exp_row, const int32_t *disp_row,
                           uint16_t *z)
{
    float *acc = (float *)malloc(sizeof(float) * (size_t)(N > 0 ? N : 1));
    if (!acc) return -1;
    for (int64_t i = 0; i < n_tok; ++i) {
        int64_t t = tokens ? tokens[i] : i;
        for (int32_t p = 0; p < E_part; ++p) {
            int32_t r = disp_row[t * E_part + p];
            if (r < 0) continue;
            for (int32_t c = 0; c < N; ++c) acc[c] = 0.0f;
            for (int32_t k = 0; k < topk; ++k) {
                int32_t er = exp_row[t * topk + k];
                int32_t e = topk_idx[t * topk + k];
                if (er < 0 || e < 0 || e >= G || part_of[e] != p) continue;
                float wk = w[t * topk + k];
                const uint16_t *yr = y + (int64_t)er * N;
                for (int32_t c = 0; c < N; ++c)
                    acc[c] = fmaf(wk, orc_bf16_to_f32(yr[c]), acc[c]);
            }
            for (int32_t c = 0; c < N; ++c) z[(int64_t)r * N + c] = orc_f32_to_bf16(acc[c]);
        }
    }
    free(acc);
    return 0;
}

/* out row i = token tokens[i] (NULL: token i) summed over its partitions */
int oracle_combine_reduce(int32_t N, int32_t E_part, int64_t n_tok,
                          const int64_t *tokens, const uint16_t *z,
                          const int32_t *disp_row, uint16_t *out)
{
    float *acc = (float *)malloc(sizeof(float) * (size_t)(N > 0 ? N : 1));
    if (!acc) return -1;
    for (int64_t i = 0; i < n_tok; ++i) {
        int64_t t = tokens ? tokens[i] : i;
        for (int32_t c = 0; c < N; ++c) acc[c] = 0.0f;
        for (int32_t p = 0; p < E_part; ++p) {
            int32_t r = disp_row[t * E_part + p];
            if (r < 0) continue;
            const uint16_t *zr = z + (int64_t)r * N;
            for (int32_t c = 0; c < N; ++c) acc[c] = acc[c] + orc_bf16_to_f32(zr[c]);
        }
        for (int32_t c = 0; c < N; ++c) out[i * N + c] = orc_f32_to_bf16(acc[c]);
    }
    free(acc);
    return 0;
}

/*
 * Grouped-GEMM tile metadata (DeepSpeed PR #8180, "Key points": a grouped
 * GEMM over expert-contiguous rows maps each of its row tiles to a group,
 * computed from the offsets).  Tiles hold block_m rows and never straddle
 * two experts: expert e owns n_e = ceil(expert_count[e] / block_m) tiles.
 * Tiles are numbered in row order, so expert e's first tile is
 *     tile_first[e] = sum of n_f over the experts f whose rows start before
 *                     e's (expert_offset[f] < expert_offset[e]),
 * and tile_first[G] is the number of tiles.  Tile tile_first[e] + j covers
 * rows [expert_offset[e] + j * block_m, ... + tile_rows) with
 * tile_rows = min(block_m, expert_count[e] - j * block_m).
 * Returns the number of tiles; the tile arrays must hold that many.
 */
int64_t oracle_expert_tiles(int32_t G, int32_t block_m, const int32_t *expert_count,
                            const int32_t *expert_offset, int32_t *tile_first,
                            int32_t *tile_expert, int32_t *tile_row, int32_t *tile_rows)
{
    int64_t total = 0;
    for (int32_t e = 0; e < G; ++e) {
        int64_t first = 0;
        for (int32_t f = 0; f < G; ++f)
            if (expert_offset[f] < expert_offset[e])
                first += ((int64_t)expert_count[f] + block_m - 1) / block_m;
        tile_first[e] = (int32_t)first;
        total += ((int64_t)expert_count[e] + block_m - 1) / block_m;
    }
    tile_first[G] = (int32_t)total;
    for (int32_t e = 0; e < G; ++e) {
        int64_t n = ((int64_t)expert_count[e] + block_m - 1) / block_m;
        for (int64_t j = 0; j < n; ++j) {
            int64_t i = tile_first[e] + j;
            int64_t rest = expert_count[e] - j * block_m;
            tile_expert[i] = e;
            tile_row[i] = (int32_t)(expert_offset[e] + j * block_m);
            tile_rows[i] = (int32_t)(rest < block_m ? rest : block_m);
        }
    }
    return total;
}

/* ------------------------------------------------------------------------ */
/* expert-parallel exchange plan (counts exchange)                          */
/* ------------------------------------------------------------------------ */

#define ORACLE_BAD_COUNT 8

/* Stores v, or -1 and the status bit if v is negative or does not fit an int32. */
static int32_t orc_fit(int64_t v, int32_t *status)
{
    if (v < 0 || v > INT32_MAX) {
        *status |= ORACLE_BAD_COUNT;
        return -1;
    }
    return (int32_t)v;
}

/*
 * Plan of rank r of W for the exchange of dispatch rows.
 *   part_counts   [W][W]: row s = part_count of rank s's layout (rows that s
 *                 sends to each destination d)
 *   expert_counts [W][G] or NULL: row s = expert_count of rank s's layout
 *                 (without dedup, where dispatch rows are expert rows)
 *   part_of       [G]: rank of each expert (used with expert_counts)
 * Outputs, each a plain sum written out:
 *   send_offset[d]  = sum_{s<r} part_counts[s][d]   (r's rows start here in d's buffer)
 *   src_offset[s]   = sum_{d<r} part_counts[s][d]   (rows for r start here in s's buffer)
 *   recv_count[s]   = part_counts[s][r]
 *   recv_offset[s]  = sum_{s'<s} part_counts[s'][r], recv_offset[W] = sum over all s
 * and with expert_counts, for every expert e:
 *   recv_expert_count[e]    = sum_s expert_counts[s][e] if part_of[e] == r, else 0
 *   recv_block_offset[s][e] = recv_offset[s] + sum of expert_counts[s][f] over the
 *                             experts f < e with part_of[f] == r, if part_of[e] == r,
 *                             else -1
 *   (a source's rows for r are its expert rows of partition r, in expert-id order)
 * Negative counts, sums past INT32_MAX and, with expert_counts, a source whose
 * expert counts on r do not add up to part_counts[s][r] set bit 8 of *status.
 */
void oracle_ep_plan(int32_t W, int32_t r, int32_t G, const int32_t *part_counts,
                    const int32_t *expert_counts, const int32_t *part_of,
                    int32_t *send_offset, int32_t *src_offset, int32_t *recv_count,
                    int32_t *recv_offset, int32_t *recv_expert_count,
                    int32_t *recv_block_offset, int32_t *status)
{
    int32_t st = 0;
    for (int64_t i = 0; i < (int64_t)W * W; ++i)
        if (part_counts[i] < 0) st |= ORACLE_BAD_COUNT;
    for (int32_t d = 0; d < W; ++d) {
        int64_t sum = 0;
        for (int32_t s = 0; s < r; ++s) sum += part_counts[(int64_t)s * W + d];
        send_offset[d] = orc_fit(sum, &st);
    }
    for (int32_t s = 0; s < W; ++s) {
        int64_t sum = 0;
        for (int32_t d = 0; d < r; ++d) sum += part_counts[(int64_t)s * W + d];
        src_offset[s] = orc_fit(sum, &st);
        recv_count[s] = part_counts[(int64_t)s * W + r];
    }
    for (int32_t s = 0; s <= W; ++s) {
        int64_t sum = 0;
        for (int32_t q = 0; q < s; ++q) sum += part_counts[(int64_t)q * W + r];
        recv_offset[s] = orc_fit(sum, &st);
    }
    if (expert_counts) {
        for (int32_t e = 0; e < G; ++e) {
            int64_t sum = 0;
            if (part_of[e] == r)
                for (int32_t s = 0; s < W; ++s) sum += expert_counts[(int64_t)s * G + e];
            recv_expert_count[e] = orc_fit(sum, &st);
        }
        for (int32_t s = 0; s < W; ++s) {
            int64_t on_r = 0;
            for (int32_t e = 0; e < G; ++e) {
                const int64_t c = expert_counts[(int64_t)s * G + e];
                if (c < 0) st |= ORACLE_BAD_COUNT;
                if (part_of[e] != r) {
                    recv_block_offset[(int64_t)s * G + e] = -1;
                    continue;
                }
                int64_t before = 0;
                for (int32_t f = 0; f < e; ++f)
                    if (part_of[f] == r) before += expert_counts[(int64_t)s * G + f];
                recv_block_offset[(int64_t)s * G + e] =
                    orc_fit((int64_t)recv_offset[s] + before, &st);
                on_r += c;
            }
            if (on_r != part_counts[(int64_t)s * W + r]) st |= ORACLE_BAD_COUNT;
        }
    }
    *status = st;
}
