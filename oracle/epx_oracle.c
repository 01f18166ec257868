/*
 * CPU oracle for MoE token dispatch and combine -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, single-threaded C.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.  It
 * shares no code, header or table with the CUDA library.
 *
 * What it computes, and where the pages fix it:
 *
 *  - Routing layout.  A token travels once to every rank that owns at least
 *    one of its experts, carrying its top-k indices with it, and the layout
 *    ("handle") produced by dispatch is what combine consumes later
 *    (DeepEP issue #48 "How to apply Moe MLP to recv_x returned by dispatch
 *    when num_expert_per_rank > 1", question and answers).  Experts sit on
 *    ranks in contiguous blocks of num_experts / world_size
 *    (DeepEP issue #760, Reproduction: local_experts and topk_idx setup).
 *    A -1 index is a padding route and counts nowhere (same Reproduction:
 *    rows of -1 with zero weights; valid routes counted as topk_idx >= 0).
 *  - Dispatch then expand: a grouped-GEMM consumer needs one row per
 *    (token, expert) in expert-contiguous order, made from the row received
 *    once per rank (issue #48, answers on DeepGEMM and on the VRAM tradeoff).
 *  - Combine: each token's per-expert outputs are weighted by its gate
 *    weights and summed back into one row (issue #48, "reduction kernel
 *    before the combine all2all"; issue #760, Reproduction: fake expert
 *    output and the expected combined value 1 for the real row, 0 for
 *    padding rows).
 *  - Stand-in expert: expert e multiplies its rows by 1 + e/E in fp32.
 *
 * Readings taken where the pages are silent: row order inside an expert
 * segment and inside a rank segment is by token, then by k slot; each
 * duplicate occurrence of an expert in one row is its own route; weights are
 * used as given (no renormalisation); an index < -1 or >= E is counted as bad
 * and then treated as -1; a row with no valid route combines to +0.
 *
 * bf16 rounding is written from the IEEE-754 round-to-nearest-even
 * definition: one rounding from the exact (double) value.  Combine sums in
 * double in k order and rounds once.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ bf16 */

/* exact value of a bf16 bit pattern */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* bf16 (8 significant bits, exponent range of binary32) nearest to v, ties to
 * the even significand.  Overflow goes to +-inf, NaN stays NaN. */
uint16_t orc_bf16_from_double(double v)
{
    if (isnan(v))
        return 0x7FC0;
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    uint16_t sign = (uint16_t)(neg << 15);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80);

    /* quantum (ulp) of the bf16 grid at a's binade */
    int e;
    (void)frexp(a, &e);            /* a = m * 2^e, 0.5 <= m < 1 */
    int unbiased = e - 1;          /* a in [2^unbiased, 2^(unbiased+1)) */
    if (unbiased < -126)
        unbiased = -126;           /* subnormal range: fixed quantum 2^-133 */
    double quantum = ldexp(1.0, unbiased - 7);

    double q = a / quantum;        /* exact: power-of-two scaling */
    double fl = floor(q);
    double rem = q - fl;           /* exact */
    double n;
    if (rem > 0.5)
        n = fl + 1.0;
    else if (rem < 0.5)
        n = fl;
    else
        n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double r = n * quantum;        /* exact */

    if (r >= ldexp(1.0, 128))      /* beyond the largest finite bf16 */
        return (uint16_t)(sign | 0x7F80);
    float rf = (float)r;           /* exact: r is on the bf16 grid */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFF));
}

/* ---------------------------------------------------------------- layout */

static int64_t read_idx(const void *idx, int idx_bits, int64_t i)
{
    if (idx_bits == 64)
        return ((const int64_t *)idx)[i];
    return (int64_t)((const int32_t *)idx)[i];
}

/*
 * Routing layout from topk_idx[T, k].
 *   cnt_e[E]   routes per expert              off_e[E+1] exclusive scan
 *   cnt_r[R]   tokens per rank (deduplicated) off_r[R+1] exclusive scan
 *   pos[T*k]       row of route (t, j) in the expert-contiguous buffer, -1 if none
 *   recv_pos[T*R]  row of token t in rank r's receive segment, -1 if not sent
 *   totals[4]  N_route, N_recv, T_real (rows with >= 1 valid route), n_bad
 * Returns 0, or -1 on bad arguments (E % R != 0, sizes < 0).
 */
int orc_layout(const void *topk_idx, int idx_bits, int T, int k, int E, int R,
               int32_t *cnt_e, int32_t *off_e, int32_t *cnt_r, int32_t *off_r,
               int32_t *pos, int32_t *recv_pos, int64_t *totals)
{
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0)
        return -1;
    if (idx_bits != 32 && idx_bits != 64)
        return -1;
    const int epr = E / R;
    int64_t n_bad = 0, t_real = 0;
    char *seen = (char *)calloc((size_t)R, 1);
    int32_t *cur_e = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *cur_r = (int32_t *)malloc(sizeof(int32_t) * (size_t)R);
    if (!seen || !cur_e || !cur_r) {
        free(seen); free(cur_e); free(cur_r);
        return -2;
    }

    /* 1. counts */
    for (int e = 0; e < E; e++) cnt_e[e] = 0;
    for (int r = 0; r < R; r++) cnt_r[r] = 0;
    for (int t = 0; t < T; t++) {
        memset(seen, 0, (size_t)R);
        int any = 0;
        for (int j = 0; j < k; j++) {
            int64_t e = read_idx(topk_idx, idx_bits, (int64_t)t * k + j);
            if (e < -1 || e >= E) { n_bad++; continue; }
            if (e == -1) continue;
            any = 1;
            cnt_e[e]++;
            int r = (int)(e / epr);
            if (!seen[r]) { seen[r] = 1; cnt_r[r]++; }
        }
        t_real += any;
    }

    /* 2. exclusive scans */
    off_e[0] = 0;
    for (int e = 0; e < E; e++) off_e[e + 1] = off_e[e] + cnt_e[e];
    off_r[0] = 0;
    for (int r = 0; r < R; r++) off_r[r + 1] = off_r[r] + cnt_r[r];

    /* 3. positions: walk routes by token then k slot, with running cursors */
    for (int e = 0; e < E; e++) cur_e[e] = off_e[e];
    for (int r = 0; r < R; r++) cur_r[r] = off_r[r];
    for (int64_t i = 0; i < (int64_t)T * R; i++) recv_pos[i] = -1;
    for (int t = 0; t < T; t++) {
        memset(seen, 0, (size_t)R);
        for (int j = 0; j < k; j++) {
            int64_t e = read_idx(topk_idx, idx_bits, (int64_t)t * k + j);
            if (e < 0 || e >= E) { pos[(int64_t)t * k + j] = -1; continue; }
            pos[(int64_t)t * k + j] = cur_e[e]++;
            int r = (int)(e / epr);
            if (!seen[r]) {
                seen[r] = 1;
                recv_pos[(int64_t)t * R + r] = cur_r[r]++;
            }
        }
    }

    totals[0] = off_e[E];
    totals[1] = off_r[R];
    totals[2] = t_real;
    totals[3] = n_bad;
    free(seen); free(cur_e); free(cur_r);
    return 0;
}

/* ------------------------------------------------------- dispatch/expand */

/*
 * Dispatch: recv[recv_pos[t, r]] = x[t] for every rank r the token reaches.
 * Expand:   expanded[pos[t, j]] = recv[recv_pos[t, rank(e)]] for every valid
 *           route, i.e. the expert-contiguous copy is made from the row as
 *           received by the owning rank.
 * x, recv and expanded hold bf16 bit patterns, H per row.
 */
void orc_dispatch_expand(const uint16_t *x, int T, int H, int k, int E, int R,
                         const void *topk_idx, int idx_bits,
                         const int32_t *pos, const int32_t *recv_pos,
                         uint16_t *recv, uint16_t *expanded)
{
    const int epr = E / R;
    const size_t row = (size_t)H * sizeof(uint16_t);
    for (int t = 0; t < T; t++)
        for (int r = 0; r < R; r++) {
            int32_t d = recv_pos[(int64_t)t * R + r];
            if (d >= 0)
                memcpy(recv + (size_t)d * H, x + (size_t)t * H, row);
        }
    for (int t = 0; t < T; t++)
        for (int j = 0; j < k; j++) {
            int32_t p = pos[(int64_t)t * k + j];
            if (p < 0) continue;
            int64_t e = read_idx(topk_idx, idx_bits, (int64_t)t * k + j);
            int r = (int)(e / epr);
            int32_t d = recv_pos[(int64_t)t * R + r];
            memcpy(expanded + (size_t)p * H, recv + (size_t)d * H, row);
        }
}

/* ------------------------------------------------------ stand-in expert */

/* y[p] = bf16(float(expanded[p]) * (1 + e/E)) in fp32 for every row p of
 * expert e's segment [off_e[e], off_e[e+1]). */
void orc_standin(const uint16_t *expanded, int H, int E, const int32_t *off_e,
                 uint16_t *y)
{
    for (int e = 0; e < E; e++) {
        float scale = 1.0f + (float)e / (float)E;
        for (int32_t p = off_e[e]; p < off_e[e + 1]; p++)
            for (int h = 0; h < H; h++) {
                float xv = (float)orc_bf16_to_double(expanded[(size_t)p * H + h]);
                float yv = xv * scale;
                y[(size_t)p * H + h] = orc_bf16_from_double((double)yv);
            }
    }
}

/* --------------------------------------------------------------- combine */

/*
 * out[t, h] = bf16( sum over valid j, in k order, of w[t, j] * y[pos[t, j], h] ),
 * summed in double; a token with no valid route gives +0.
 * If out_exact is not NULL it also receives the unrounded double sums.
 */
void orc_combine(const uint16_t *y, const float *w, const int32_t *pos,
                 int T, int k, int H, uint16_t *out, double *out_exact)
{
    for (int t = 0; t < T; t++)
        for (int h = 0; h < H; h++) {
            double acc = 0.0;
            for (int j = 0; j < k; j++) {
                int32_t p = pos[(int64_t)t * k + j];
                if (p < 0) continue;
                acc += (double)w[(int64_t)t * k + j]
                       * orc_bf16_to_double(y[(size_t)p * H + h]);
            }
            out[(size_t)t * H + h] = orc_bf16_from_double(acc);
            if (out_exact)
                out_exact[(size_t)t * H + h] = acc;
        }
}

/* ------------------------------------------- two-stage combine (NEXT) */

/*
 * Local reduce before the combine all2all (DeepEP issue #48, answer on the
 * reduction kernel before the combine all2all): every rank sums, for each
 * token it received, its own experts' weighted outputs, giving one partial
 * row per (token, rank) in the receive layout:
 *   partial[recv_pos[t, r], h] = sum over valid j with rank(e_j) == r, in k
 *                                order, of w[t, j] * y[pos[t, j], h]
 * summed in double, then stored as fp32 (part_bits 32) or bf16 (16).
 * `partial` holds N_recv rows of H (float or uint16).
 */
void orc_combine_local(const uint16_t *y, const float *w, const void *topk_idx, int idx_bits,
                       const int32_t *pos, const int32_t *recv_pos, int T, int k, int E,
                       int R, int H, int part_bits, void *partial)
{
    const int epr = E / R;
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    for (int t = 0; t < T; t++)
        for (int r = 0; r < R; r++) {
            int32_t d = recv_pos[(int64_t)t * R + r];
            if (d < 0) continue;
            for (int h = 0; h < H; h++) acc[h] = 0.0;
            for (int j = 0; j < k; j++) {
                int32_t p = pos[(int64_t)t * k + j];
                if (p < 0) continue;
                int64_t e = read_idx(topk_idx, idx_bits, (int64_t)t * k + j);
                if ((int)(e / epr) != r) continue;
                double wj = (double)w[(int64_t)t * k + j];
                for (int h = 0; h < H; h++)
                    acc[h] += wj * orc_bf16_to_double(y[(size_t)p * H + h]);
            }
            for (int h = 0; h < H; h++) {
                if (part_bits == 32)
                    ((float *)partial)[(size_t)d * H + h] = (float)acc[h];
                else
                    ((uint16_t *)partial)[(size_t)d * H + h] = orc_bf16_from_double(acc[h]);
            }
        }
    free(acc);
}

/*
 * Combine epilogue (DeepEP issue #760: combine_reduce_epilogue reduces the
 * rows received back from every rank into the token's output): for every
 * token, the partial rows of the ranks it reached, in rank order, summed in
 * double, plus an optional residual row, rounded once to bf16.  A token that
 * reached no rank gives its residual row (or +0 without one).
 */
void orc_combine_epilogue(const void *partial, int part_bits, const int32_t *recv_pos,
                          const uint16_t *residual, int T, int R, int H, uint16_t *out)
{
    for (int t = 0; t < T; t++)
        for (int h = 0; h < H; h++) {
            double acc = residual ? orc_bf16_to_double(residual[(size_t)t * H + h]) : 0.0;
            for (int r = 0; r < R; r++) {
                int32_t d = recv_pos[(int64_t)t * R + r];
                if (d < 0) continue;
                acc += part_bits == 32
                           ? (double)((const float *)partial)[(size_t)d * H + h]
                           : orc_bf16_to_double(((const uint16_t *)partial)[(size_t)d * H + h]);
            }
            out[(size_t)t * H + h] = orc_bf16_from_double(acc);
        }
}

/* ------------------------------------------- dispatch without expand (NEXT) */

/*
 * Gather index for a consumer that reads the received rows directly instead
 * of an expanded copy (DeepEP issue #760, Reproduction: dispatch with
 * do_expand=False; issue #48, answer on the VRAM / performance tradeoff of
 * expanding): the expert-contiguous row of route (t, j) is served by the row
 * in which token t was received by the rank that owns expert e_j,
 *   src[pos[t, j]] = recv_pos[t, rank(e_j)]   for every valid route.
 * src has N_route entries.
 */
void orc_expand_index(const void *topk_idx, int idx_bits, const int32_t *pos,
                      const int32_t *recv_pos, int T, int k, int E, int R, int32_t *src)
{
    const int epr = E / R;
    for (int t = 0; t < T; t++)
        for (int j = 0; j < k; j++) {
            int32_t p = pos[(int64_t)t * k + j];
            if (p < 0) continue;
            int64_t e = read_idx(topk_idx, idx_bits, (int64_t)t * k + j);
            src[p] = recv_pos[(int64_t)t * R + (int)(e / epr)];
        }
}
