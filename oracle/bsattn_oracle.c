/*
 * bsattn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of block-sparse attention with the BLASST
 * softmax-threshold skip.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library; the product path never
 * does.  It shares no code, header or constant with the CUDA library.
 *
 * Sources followed (page titles as they appear on the web):
 *  - "BLASST: Dynamic Blocked Attention Sparsity via Softmax Thresholding",
 *    section 3.1.1 (the skip inequality: tile max minus running max below
 *    ln(lambda)) and Algorithm 1 (per query tile: scores, tile row max,
 *    running max updated before the test, skip, else exp / rowsum / PV).
 *  - "块稀疏Attention实战" (block-sparse attention for multimodal DiT),
 *    section 2.1 (0/1 block mask: a zero block takes no part in QK, softmax or
 *    PV), section 2.3 (mask stored as a sparse index; sparsity ratio) and
 *    section 5.2 (masked blocks contribute nothing to softmax statistics).
 *  - "Attention 的七十二变", section 1 (softmax(QK^T / sqrt(d)) V) and
 *    section 5.3-5.4 (GQA: query head h reads KV head floor(h / g)).
 *
 * Readings taken where the pages are silent or ambiguous:
 *  - Scores include the softmax scale; the threshold is compared in natural-log
 *    units of the scaled scores.
 *  - A tile is skipped only when every valid row of the query tile passes
 *    (the kernel design section's warp VOTE across the softmax warpgroup).
 *  - lambda = 0 means "never skip"; lambda must lie in [0, 1].
 *  - Rows whose running max is still -inf never pass ((-inf)-(-inf) is NaN,
 *    and NaN does not pass); a fully masked row (tile max -inf) with a finite
 *    running max passes.
 *  - The running max is updated with every visited tile, skipped or not
 *    (Algorithm 1 updates it before the test).
 *  - Visit order is ascending key-tile index (Algorithm 1's loop over j), or,
 *    on request, descending: the BLASST page's block-row reordering study
 *    (section on ablations, Figure 8) visits the tiles of a row in reverse so
 *    that the local window, which holds the largest scores, sets the running
 *    max first.
 *  - Decode: the query tile is the g query heads that share one KV head; the
 *    KV tiles are cut into num_splits contiguous chunks of ceil(T/num_splits)
 *    tiles and the running max starts again at -inf in each chunk.  On
 *    request (sink seeding) every chunk but the first starts instead from the
 *    row max of key tile 0, the tile that holds the attention sink; tile 0 is
 *    then scored by that chunk but neither visited nor executed by it.
 *  - Variable lengths (key padding, "块稀疏Attention实战" section 5.2: pad
 *    the batch to its longest sequence and mask the padding keys): sequence b
 *    has len_b valid tokens; keys at or past len_b take no part, key tiles
 *    wholly past it are not visited, and query rows at or past it are padding
 *    (no vote, O = 0, LSE = -inf).  A padded batch therefore equals every
 *    sequence computed alone at its own length; in decode the splits cut the
 *    sequence's own ceil(len_b / block) tiles.
 *  - The result is the exact softmax over the keys of the executed tiles,
 *    computed in two passes (max, then sum) -- algebraically what the online
 *    recurrence of Algorithm 1 reaches.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_CAPACITY (-4)

static double bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------
 * Mask -> per-query-block CSR.  Row i of mask head h lists, in ascending
 * order, every key block j with mask[h][i][j] != 0; with causal set, only
 * the key blocks whose first key is not after the query block's last query:
 * j * k_block <= (i + 1) * q_block - 1.
 * row_ptr has mask_heads * (nq + 1) entries and holds absolute offsets into
 * col_idx (head h's rows start where head h-1's end).
 */
int oracle_build_index(const uint8_t *mask, int mask_heads, int nq, int nk,
                       int q_block, int k_block, int causal,
                       int32_t *row_ptr, int32_t *col_idx, int64_t capacity,
                       int32_t *nnz)
{
    if (!mask || !row_ptr || !nnz || mask_heads < 1 || nq < 0 || nk < 0 ||
        q_block < 1 || k_block < 1)
        return ORACLE_ERR_ARG;
    int64_t pos = 0;
    int status = ORACLE_OK;
    for (int h = 0; h < mask_heads; ++h) {
        int64_t head_start = pos;
        for (int i = 0; i < nq; ++i) {
            row_ptr[(int64_t)h * (nq + 1) + i] = (int32_t)pos;
            for (int j = 0; j < nk; ++j) {
                int keep = mask[((int64_t)h * nq + i) * nk + j] != 0;
                if (causal && (int64_t)j * k_block > (int64_t)(i + 1) * q_block - 1)
                    keep = 0;
                if (keep) {
                    if (pos < capacity && col_idx)
                        col_idx[pos] = j;
                    else
                        status = ORACLE_ERR_CAPACITY;
                    pos++;
                }
            }
        }
        row_ptr[(int64_t)h * (nq + 1) + nq] = (int32_t)pos;
        nnz[h] = (int32_t)(pos - head_start);
    }
    return status;
}

/* ------------------------------------------------------------------------
 * One query tile: rows (query vectors) qrows[r] for r < nrows, each with its
 * query position qpos[r] (used only for the causal test), against the key
 * tiles tiles[0..ntiles) of one KV head.  Implements the visit + test of
 * Algorithm 1 and then the exact softmax over the executed tiles.
 *
 *   qrows:  nrows pointers to d bf16 values
 *   kbase, vbase: the KV head's keys / values, L rows of d bf16 values
 *   tiles:  key-tile indices in visit order; split_start[t] != 0 resets the
 *           running max before tile t (decode splits)
 *   out:    nrows x d doubles; lse: nrows doubles
 *   status: per visited tile, 1 = skipped, 2 = executed
 *   margin: per visited tile, max over rows of (tile max - running max)
 *           minus ln(lambda); +inf when the test cannot pass
 *   seed_tile: -1, or a key tile whose row max starts the running max at every
 *           split start whose first tile is another tile
 */
static void query_tile(const uint16_t *const *qrows, const int64_t *qpos, int nrows,
                       const uint16_t *kbase, const uint16_t *vbase, int64_t L,
                       int d, int block, double scale, int causal, double lambda,
                       const int32_t *tiles, const uint8_t *split_start, int ntiles,
                       int seed_tile,
                       double *out, double *lse, uint8_t *status, double *margin)
{
    const double ln_lambda = lambda > 0.0 ? log(lambda) : -INFINITY;
    double *mprev = malloc(sizeof(double) * nrows);
    double *tmax = malloc(sizeof(double) * (size_t)nrows * (ntiles > 0 ? ntiles : 1));
    uint8_t *exec = malloc(ntiles > 0 ? ntiles : 1);
    double *qv = malloc(sizeof(double) * (size_t)nrows * d);
    double *kv = malloc(sizeof(double) * (size_t)block * d);
    double *s = malloc(sizeof(double) * (size_t)nrows * block);

    for (int r = 0; r < nrows; ++r)
        for (int x = 0; x < d; ++x)
            qv[(size_t)r * d + x] = bf16_value(qrows[r][x]);

    /* Scores of one key tile: s[r][c] = scale * <q_r, k_c>, -inf where the
     * key is past the end or (causal) after the query. */
#define SCORE_TILE(jt)                                                              \
    do {                                                                            \
        int64_t k0 = (int64_t)(jt) * block;                                         \
        for (int c = 0; c < block; ++c) {                                           \
            int64_t key = k0 + c;                                                   \
            for (int x = 0; x < d; ++x)                                             \
                kv[(size_t)c * d + x] = key < L ? bf16_value(kbase[key * d + x]) : 0.0; \
        }                                                                           \
        for (int r = 0; r < nrows; ++r) {                                           \
            for (int c = 0; c < block; ++c) {                                       \
                int64_t key = k0 + c;                                               \
                double acc = 0.0;                                                   \
                for (int x = 0; x < d; ++x)                                         \
                    acc += qv[(size_t)r * d + x] * kv[(size_t)c * d + x];           \
                if (key >= L || (causal && key > qpos[r]))                          \
                    acc = -INFINITY;                                                \
                else                                                                \
                    acc *= scale;                                                   \
                s[(size_t)r * block + c] = acc;                                     \
            }                                                                       \
        }                                                                           \
    } while (0)

    /* Pass 1: visit in order, running max, skip test. */
    for (int r = 0; r < nrows; ++r)
        mprev[r] = -INFINITY;
    for (int t = 0; t < ntiles; ++t) {
        if (split_start && split_start[t]) {
            for (int r = 0; r < nrows; ++r)
                mprev[r] = -INFINITY;
            if (seed_tile >= 0 && tiles[t] != seed_tile) {
                SCORE_TILE(seed_tile);
                for (int r = 0; r < nrows; ++r)
                    for (int c = 0; c < block; ++c)
                        if (s[(size_t)r * block + c] > mprev[r])
                            mprev[r] = s[(size_t)r * block + c];
            }
        }
        SCORE_TILE(tiles[t]);
        double dmax = -INFINITY;
        for (int r = 0; r < nrows; ++r) {
            double mt = -INFINITY;
            for (int c = 0; c < block; ++c)
                if (s[(size_t)r * block + c] > mt)
                    mt = s[(size_t)r * block + c];
            tmax[(size_t)t * nrows + r] = mt;
            double dr = mt - mprev[r];
            if (isnan(dr))
                dr = INFINITY; /* (-inf) - (-inf): does not pass */
            if (dr > dmax)
                dmax = dr;
        }
        int skip = 0;
        double mg = INFINITY;
        if (lambda > 0.0) {
            mg = dmax - ln_lambda;
            skip = dmax < ln_lambda; /* every row below the threshold */
        }
        for (int r = 0; r < nrows; ++r) {
            double mt = tmax[(size_t)t * nrows + r];
            if (mt > mprev[r])
                mprev[r] = mt;
        }
        exec[t] = (uint8_t)!skip;
        if (status)
            status[t] = skip ? 1 : 2;
        if (margin)
            margin[t] = mg;
    }

    /* Pass 2: per-row maximum over the executed tiles. */
    for (int r = 0; r < nrows; ++r) {
        double mu = -INFINITY;
        for (int t = 0; t < ntiles; ++t)
            if (exec[t] && tmax[(size_t)t * nrows + r] > mu)
                mu = tmax[(size_t)t * nrows + r];
        mprev[r] = mu; /* reuse as the softmax shift */
    }

    /* Pass 3: exact softmax over the executed keys and the weighted sum. */
    double *z = calloc((size_t)nrows, sizeof(double));
    memset(out, 0, sizeof(double) * (size_t)nrows * d);
    for (int t = 0; t < ntiles; ++t) {
        if (!exec[t])
            continue;
        SCORE_TILE(tiles[t]);
        int64_t k0 = (int64_t)tiles[t] * block;
        for (int r = 0; r < nrows; ++r) {
            if (mprev[r] == -INFINITY)
                continue;
            for (int c = 0; c < block; ++c) {
                double sc = s[(size_t)r * block + c];
                if (sc == -INFINITY)
                    continue;
                double p = exp(sc - mprev[r]);
                z[r] += p;
                const uint16_t *vrow = vbase + (k0 + c) * d;
                for (int x = 0; x < d; ++x)
                    out[(size_t)r * d + x] += p * bf16_value(vrow[x]);
            }
        }
    }
    for (int r = 0; r < nrows; ++r) {
        if (z[r] > 0.0) {
            for (int x = 0; x < d; ++x)
                out[(size_t)r * d + x] /= z[r];
            lse[r] = mprev[r] + log(z[r]);
        } else {
            lse[r] = -INFINITY;
        }
    }
#undef SCORE_TILE
    free(z);
    free(mprev);
    free(tmax);
    free(exec);
    free(qv);
    free(kv);
    free(s);
}

/* ------------------------------------------------------------------------
 * Prefill.  q: [B][Hq][N][d], k, v: [B][Hkv][N][d] (bf16 bits).
 * mask: NULL (every key tile) or [mask_heads][nq][nk] with mask_heads 1 or Hq.
 * items: NULL (every (b, h, i)) or n_items triples (b, h, i) to compute.
 * o: [B][Hq][N][d], lse: [B][Hq][N] (doubles); tile_status / margin:
 * NULL or [B][Hq][nq][nk].  Only rows of the listed items are written.
 * reverse: 0 visits each row's key tiles in ascending order, 1 in descending.
 * seq_lens: NULL (every sequence has N tokens) or [B] valid lengths in [0, N].
 */
int oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   int B, int Hq, int Hkv, int N, int d, int block,
                   double scale, int causal, double lambda,
                   const uint8_t *mask, int mask_heads,
                   const int32_t *items, int n_items,
                   double *o, double *lse, uint8_t *tile_status, double *margin,
                   int reverse, const int32_t *seq_lens)
{
    if (!q || !k || !v || !o || !lse || B < 1 || Hq < 1 || Hkv < 1 ||
        Hq % Hkv != 0 || N < 1 || d < 1 || block < 1 ||
        !(lambda >= 0.0 && lambda <= 1.0))
        return ORACLE_ERR_ARG;
    if (mask && mask_heads != 1 && mask_heads != Hq)
        return ORACLE_ERR_ARG;
    if (seq_lens)
        for (int b = 0; b < B; ++b)
            if (seq_lens[b] < 0 || seq_lens[b] > N)
                return ORACLE_ERR_ARG;
    const int g = Hq / Hkv;
    const int nq = (N + block - 1) / block, nk = nq;
    const int64_t total = items ? n_items : (int64_t)B * Hq * nq;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t w = 0; w < total; ++w) {
        int b, h, i;
        if (items) {
            b = items[3 * w];
            h = items[3 * w + 1];
            i = items[3 * w + 2];
        } else {
            b = (int)(w / ((int64_t)Hq * nq));
            h = (int)((w / nq) % Hq);
            i = (int)(w % nq);
        }
        const int kvh = h / g;
        const int64_t r0 = (int64_t)i * block;
        const int nrows_all = (int)((r0 + block <= N) ? block : N - r0);
        const int64_t len = seq_lens ? seq_lens[b] : N;
        /* rows at or past the sequence's length are padding */
        const int nrows = r0 >= len ? 0 : (int)((r0 + nrows_all <= len) ? nrows_all : len - r0);
        for (int r = nrows; r < nrows_all; ++r) {
            double *orow_pad = o + (((int64_t)b * Hq + h) * N + r0 + r) * d;
            for (int x = 0; x < d; ++x)
                orow_pad[x] = 0.0;
            lse[((int64_t)b * Hq + h) * N + r0 + r] = -INFINITY;
        }
        const uint16_t *qrows[1024];
        int64_t qpos[1024];
        for (int r = 0; r < nrows; ++r) {
            qrows[r] = q + (((int64_t)b * Hq + h) * N + r0 + r) * d;
            qpos[r] = r0 + r;
        }
        int32_t *tiles = malloc(sizeof(int32_t) * (nk > 0 ? nk : 1));
        int nt = 0;
        const int mh = mask ? (mask_heads == 1 ? 0 : h) : 0;
        for (int j = 0; j < nk; ++j) {
            if (mask && !mask[((int64_t)mh * nq + i) * nk + j])
                continue;
            if (causal && (int64_t)j * block > (int64_t)(i + 1) * block - 1)
                continue;
            if ((int64_t)j * block >= len)   /* wholly padding keys */
                continue;
            tiles[nt++] = j;
        }
        if (reverse)
            for (int a = 0, z = nt - 1; a < z; ++a, --z) {
                int32_t x = tiles[a];
                tiles[a] = tiles[z];
                tiles[z] = x;
            }
        uint8_t *st = malloc(nt > 0 ? nt : 1);
        double *mg = malloc(sizeof(double) * (nt > 0 ? nt : 1));
        const uint16_t *kb = k + ((int64_t)b * Hkv + kvh) * N * d;
        const uint16_t *vb = v + ((int64_t)b * Hkv + kvh) * N * d;
        double *orow = o + (((int64_t)b * Hq + h) * N + r0) * d;
        double *lrow = lse + ((int64_t)b * Hq + h) * N + r0;
        if (nrows == 0)
            nt = 0;   /* a query tile of padding only visits nothing */
        query_tile(qrows, qpos, nrows, kb, vb, len, d, block, scale, causal, lambda,
                   tiles, NULL, nt, -1, orow, lrow, st, mg);
        int64_t sbase = (((int64_t)b * Hq + h) * nq + i) * nk;
        for (int t = 0; t < nt; ++t) {
            if (tile_status)
                tile_status[sbase + tiles[t]] = st[t];
            if (margin)
                margin[sbase + tiles[t]] = mg[t];
        }
        free(tiles);
        free(st);
        free(mg);
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Decode, over n_problems independent (sequence, KV head) problems.
 * q: [n][g][d] (the g query heads sharing the KV head), k, v: [n][L][d].
 * o: [n][g][d], lse: [n][g]; tile_status / margin: NULL or [n][T] with
 * T = ceil(L / block).  A single query at the last position sees all L keys.
 * sink_seed: 1 starts every split after the first from key tile 0's row max.
 * lens: NULL (every cache holds L tokens) or [n_problems] lengths in [0, L];
 *       problem p's splits cut its own ceil(lens[p] / block) tiles.
 */
int oracle_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  int n_problems, int g, int64_t L, int d, int block,
                  double scale, double lambda, int num_splits,
                  double *o, double *lse, uint8_t *tile_status, double *margin,
                  int sink_seed, const int64_t *lens)
{
    if (!q || !k || !v || !o || !lse || n_problems < 1 || g < 1 || g > 1024 ||
        L < 1 || d < 1 || block < 1 || num_splits < 1 ||
        !(lambda >= 0.0 && lambda <= 1.0))
        return ORACLE_ERR_ARG;
    const int T = (int)((L + block - 1) / block);
    if (lens)
        for (int p = 0; p < n_problems; ++p)
            if (lens[p] < 0 || lens[p] > L)
                return ORACLE_ERR_ARG;

#pragma omp parallel for schedule(dynamic, 1)
    for (int p = 0; p < n_problems; ++p) {
        const int64_t Lp = lens ? lens[p] : L;
        const int Tp = (int)((Lp + block - 1) / block);
        const int chunk = Tp > 0 ? (Tp + num_splits - 1) / num_splits : 1;
        const uint16_t *qrows[1024];
        int64_t qpos[1024];
        for (int r = 0; r < g; ++r) {
            qrows[r] = q + ((int64_t)p * g + r) * d;
            qpos[r] = Lp - 1;
        }
        int32_t *tiles = malloc(sizeof(int32_t) * (T > 0 ? T : 1));
        uint8_t *starts = malloc(T > 0 ? T : 1);
        for (int t = 0; t < Tp; ++t) {
            tiles[t] = t;
            starts[t] = (t % chunk) == 0;
        }
        uint8_t *st = calloc(T > 0 ? T : 1, 1);
        double *mg = malloc(sizeof(double) * (T > 0 ? T : 1));
        for (int t = 0; t < T; ++t)
            mg[t] = NAN;
        query_tile(qrows, qpos, g, k + (int64_t)p * L * d, v + (int64_t)p * L * d, Lp,
                   d, block, scale, 0, lambda, tiles, starts, Tp, sink_seed ? 0 : -1,
                   o + (int64_t)p * g * d, lse + (int64_t)p * g, st, mg);
        for (int t = 0; t < T; ++t) {
            if (tile_status)
                tile_status[(int64_t)p * T + t] = st[t];
            if (margin)
                margin[(int64_t)p * T + t] = mg[t];
        }
        free(tiles);
        free(starts);
        free(st);
        free(mg);
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Prefill backward, for sparsity-aware training ("BLASST: Dynamic Blocked
 * Attention Sparsity via Softmax Thresholding", section 3.3: fine-tuning runs
 * the forward with the skip, and the blocks it skipped receive no gradient
 * because they were never computed).  With the forward's executed tiles held
 * fixed (the skip decisions are piecewise constant in the inputs), O is the
 * exact softmax over the keys of those tiles, so the gradient is that of
 * softmax attention restricted to them.  Per query row r, over its executed,
 * unmasked keys c:
 *   S_rc = scale <q_r, k_c>,  P_rc = exp(S_rc - max_c S) / sum_c exp(...)
 *   dV_c += P_rc dO_r
 *   dP_rc = <dO_r, v_c>,  D_r = sum_c P_rc dP_rc
 *   dS_rc = P_rc (dP_rc - D_r)
 *   dQ_r = scale sum_c dS_rc k_c,  dK_c += scale dS_rc q_r
 * dK and dV of a KV head sum over the query heads that read it (GQA).
 *
 * q, dout: [B][Hq][N][d]; k, v: [B][Hkv][N][d] (doubles).
 * tile_status: [B][Hq][nq][nk] as the forward wrote it; only tiles marked 2
 *   (executed) take part.  Causal and key-padding masks apply inside them.
 * seq_lens: NULL or [B] valid lengths; padding query rows get dQ = 0.
 * dq: [B][Hq][N][d]; dk, dv: [B][Hkv][N][d]; all overwritten.
 */
int oracle_prefill_bwd(const double *q, const double *k, const double *v, const double *dout,
                       int B, int Hq, int Hkv, int N, int d, int block, double scale,
                       int causal, const uint8_t *tile_status, const int32_t *seq_lens,
                       double *dq, double *dk, double *dv)
{
    if (!q || !k || !v || !dout || !tile_status || !dq || !dk || !dv || B < 1 || Hq < 1 ||
        Hkv < 1 || Hq % Hkv != 0 || N < 1 || d < 1 || block < 1)
        return ORACLE_ERR_ARG;
    if (seq_lens)
        for (int b = 0; b < B; ++b)
            if (seq_lens[b] < 0 || seq_lens[b] > N)
                return ORACLE_ERR_ARG;
    const int g = Hq / Hkv;
    const int nq = (N + block - 1) / block, nk = nq;

    /* one (sequence, KV head) per task: its dK, dV and its group's dQ */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t w = 0; w < (int64_t)B * Hkv; ++w) {
        const int b = (int)(w / Hkv), kvh = (int)(w % Hkv);
        const int64_t len = seq_lens ? seq_lens[b] : N;
        const double *kb = k + w * N * d, *vb = v + w * N * d;
        double *dkb = dk + w * N * d, *dvb = dv + w * N * d;
        memset(dkb, 0, sizeof(double) * (size_t)N * d);
        memset(dvb, 0, sizeof(double) * (size_t)N * d);
        int64_t *keys = malloc(sizeof(int64_t) * (size_t)N);
        double *p = malloc(sizeof(double) * (size_t)N);
        double *dp = malloc(sizeof(double) * (size_t)N);
        for (int h = kvh * g; h < (kvh + 1) * g; ++h) {
            const int64_t bh = (int64_t)b * Hq + h;
            for (int64_t t = 0; t < N; ++t) {
                const double *qr = q + (bh * N + t) * d;
                const double *dor = dout + (bh * N + t) * d;
                double *dqr = dq + (bh * N + t) * d;
                for (int x = 0; x < d; ++x)
                    dqr[x] = 0.0;
                if (t >= len)
                    continue;                  /* padding query row */
                const int i = (int)(t / block);
                const uint8_t *st = tile_status + (bh * nq + i) * nk;
                /* the row's keys: in executed tiles, valid, not after it */
                int nkeys = 0;
                for (int j = 0; j < nk; ++j) {
                    if (st[j] != 2)
                        continue;
                    for (int64_t c = (int64_t)j * block; c < (int64_t)(j + 1) * block; ++c)
                        if (c < len && !(causal && c > t))
                            keys[nkeys++] = c;
                }
                if (nkeys == 0)
                    continue;
                /* P: the softmax of the row's scores over those keys */
                double mu = -INFINITY;
                for (int a = 0; a < nkeys; ++a) {
                    double acc = 0.0;
                    for (int x = 0; x < d; ++x)
                        acc += qr[x] * kb[keys[a] * d + x];
                    p[a] = scale * acc;
                    if (p[a] > mu)
                        mu = p[a];
                }
                double z = 0.0;
                for (int a = 0; a < nkeys; ++a) {
                    p[a] = exp(p[a] - mu);
                    z += p[a];
                }
                for (int a = 0; a < nkeys; ++a)
                    p[a] /= z;
                /* dP and D */
                double D = 0.0;
                for (int a = 0; a < nkeys; ++a) {
                    double acc = 0.0;
                    for (int x = 0; x < d; ++x)
                        acc += dor[x] * vb[keys[a] * d + x];
                    dp[a] = acc;
                    D += p[a] * acc;
                }
                /* dS, then the three gradients */
                for (int a = 0; a < nkeys; ++a) {
                    const double ds = p[a] * (dp[a] - D);
                    const int64_t c = keys[a];
                    for (int x = 0; x < d; ++x) {
                        dqr[x] += scale * ds * kb[c * d + x];
                        dkb[c * d + x] += scale * ds * qr[x];
                        dvb[c * d + x] += p[a] * dor[x];
                    }
                }
            }
        }
        free(keys);
        free(p);
        free(dp);
    }
    return ORACLE_OK;
}
