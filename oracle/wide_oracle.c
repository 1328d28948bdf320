/*
 * wide_oracle.c -- plain, slow, fp64 CPU reference for the masked WIDE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg load this library.  It shares no code,
 * header or table with the CUDA path.
 *
 * Source: "WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic
 * Width Pruning" (abstract; technical summary sections 1 and 2).
 *
 * Conventions (chosen here, because the pages fix no data layout):
 *   - a mask is bit-packed token-major, uint32 words[T][W] with W =
 *     ceil(G/32); group g of token t is bit (g % 32) of words[t][g / 32];
 *     a set bit means the token executes the group.
 *   - bf16 values are passed as their uint16 bit patterns and widened
 *     exactly to double; fp32 values are widened exactly to double.
 *   - every sum is accumulated in double, in index order, with no
 *     rounding to a narrower type.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL -1
#define ORC_EMASK -5

/* ---------------------------------------------------------------- helpers */

static double widen_bf16(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* element i of a tensor stored as bf16 (dtype 0) or fp32 (dtype 1) */
static double elem(const void *p, int64_t i, int dtype)
{
    if (dtype == 0)
        return widen_bf16(((const uint16_t *)p)[i]);
    return (double)((const float *)p)[i];
}

static int mask_bit(const uint32_t *mask, int64_t W, int64_t t, int64_t g)
{
    return (int)((mask[t * W + g / 32] >> (g % 32)) & 1u);
}

/* SiLU(a) = a * sigmoid(a) = a / (1 + e^-a). */
static double silu(double a)
{
    return a / (1.0 + exp(-a));
}

/* ------------------------------------------------------ mask validation */

/* Returns ORC_OK when no bit at or above G is set in any word. */
int oracle_check_mask(const uint32_t *mask, int64_t T, int64_t G)
{
    if (!mask || T < 0 || G <= 0)
        return ORC_EINVAL;
    int64_t W = (G + 31) / 32;
    int tail = (int)(G % 32);
    if (tail == 0)
        return ORC_OK;
    uint32_t bad = ~((1u << tail) - 1u);
    for (int64_t t = 0; t < T; t++)
        if (mask[t * W + W - 1] & bad)
            return ORC_EMASK;
    return ORC_OK;
}

/* --------------------------------------------------------- mask reordering
 *
 * Technical summary section 2.B (unified mask-reordering preprocessing): for
 * each routing group the binary mask is sorted along the token dimension M,
 * so that the group's active tokens form one contiguous prefix and a tile of
 * that order is dense up to a known active prefix.  The sort is read as a
 * stable partition: active tokens in ascending token order, then inactive
 * ones in ascending order, which makes the permutation unique.
 *
 * Outputs (all caller-owned):
 *   count[G]                  active tokens of each group
 *   perm[G][T]                the partition above, one row per group
 *   items[2 * n]              (group, tile index) pairs, group-major, one per
 *                             tile of tile_m rows that holds >= 1 active row
 *   *n_items                  number of pairs
 *   sig_perm[T]               tokens ordered by their mask row read as one
 *                             big-endian unsigned key (word W-1 most
 *                             significant, bit 31 of a word before bit 0),
 *                             ascending, ties by token index
 *   tile_union[nt][W]         OR of the mask rows of the tokens in each
 *                             tile_m-row tile of sig_perm, nt = ceil(T/tile_m)
 */

static const uint32_t *g_sort_mask;
static int64_t g_sort_W;

static int sig_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    for (int64_t w = g_sort_W - 1; w >= 0; w--) {
        uint32_t ka = g_sort_mask[(int64_t)a * g_sort_W + w];
        uint32_t kb = g_sort_mask[(int64_t)b * g_sort_W + w];
        if (ka != kb)
            return ka < kb ? -1 : 1;
    }
    return a < b ? -1 : (a > b ? 1 : 0);
}

int oracle_reorder(const uint32_t *mask, int64_t T, int64_t G, int64_t tile_m,
                   int32_t *count, int32_t *perm, int32_t *items, int64_t *n_items,
                   int32_t *sig_perm, uint32_t *tile_union)
{
    if (!mask || T < 0 || G <= 0 || tile_m <= 0)
        return ORC_EINVAL;
    int rc = oracle_check_mask(mask, T, G);
    if (rc != ORC_OK)
        return rc;
    int64_t W = (G + 31) / 32;

    /* per-group stable partition */
    int64_t n = 0;
    for (int64_t g = 0; g < G; g++) {
        int32_t *row = perm + g * T;
        int64_t k = 0;
        for (int64_t t = 0; t < T; t++)
            if (mask_bit(mask, W, t, g))
                row[k++] = (int32_t)t;
        count[g] = (int32_t)k;
        for (int64_t t = 0; t < T; t++)
            if (!mask_bit(mask, W, t, g))
                row[k++] = (int32_t)t;
        int64_t tiles = (count[g] + tile_m - 1) / tile_m;
        for (int64_t i = 0; i < tiles; i++) {
            items[2 * n] = (int32_t)g;
            items[2 * n + 1] = (int32_t)i;
            n++;
        }
    }
    *n_items = n;

    /* signature order: a library sort with an explicit total order */
    for (int64_t t = 0; t < T; t++)
        sig_perm[t] = (int32_t)t;
    g_sort_mask = mask;
    g_sort_W = W;
    qsort(sig_perm, (size_t)T, sizeof(int32_t), sig_cmp);

    int64_t nt = (T + tile_m - 1) / tile_m;
    for (int64_t s = 0; s < nt; s++) {
        for (int64_t w = 0; w < W; w++) {
            uint32_t u = 0;
            for (int64_t r = s * tile_m; r < T && r < (s + 1) * tile_m; r++)
                u |= mask[(int64_t)sig_perm[r] * W + w];
            tile_union[s * W + w] = u;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------ masked FFN, token loop
 *
 * Technical summary section 2.A: the FFN prunes contiguous channel groups of
 * the intermediate dimension D'; a token that skips group g does not compute
 * the g-th block of gate/up channels and does not use the matching columns
 * of the down projection.  Written here as the brute-force per-token loop
 * that visits only kept groups:
 *
 *   out[t][n] = sum over kept g, channels c of g:
 *                 silu(x[t].W_gate[c]) * (x[t].W_up[c]) * W_down[n][c]
 *
 * Shapes (nn.Linear layout): x[T][Hd], W_gate/W_up[I][Hd], W_down[Hd][I],
 * groups of gs consecutive channels, out[T][Hd] in double.
 * dtype: 0 = bf16 bit patterns, 1 = fp32.  Tokens run in parallel under
 * OpenMP when the library is built with it; each token's sums are serial.
 */
int oracle_ffn_token_loop(const void *x, const void *w_gate, const void *w_up,
                          const void *w_down, const uint32_t *mask,
                          int64_t T, int64_t Hd, int64_t I, int64_t gs, int dtype,
                          double *out)
{
    if (!x || !w_gate || !w_up || !w_down || !mask || !out || T < 0 || Hd <= 0 ||
        I <= 0 || gs <= 0 || I % gs != 0 || (dtype != 0 && dtype != 1))
        return ORC_EINVAL;
    int64_t G = I / gs, W = (G + 31) / 32;
    int rc = oracle_check_mask(mask, T, G);
    if (rc != ORC_OK)
        return rc;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; t++) {
        double *o = out + t * Hd;
        for (int64_t n = 0; n < Hd; n++)
            o[n] = 0.0;
        for (int64_t g = 0; g < G; g++) {
            if (!mask_bit(mask, W, t, g))
                continue;
            for (int64_t c = g * gs; c < (g + 1) * gs; c++) {
                double a = 0.0, b = 0.0;
                for (int64_t k = 0; k < Hd; k++) {
                    double xv = elem(x, t * Hd + k, dtype);
                    a += xv * elem(w_gate, c * Hd + k, dtype);
                    b += xv * elem(w_up, c * Hd + k, dtype);
                }
                double h = silu(a) * b;
                for (int64_t n = 0; n < Hd; n++)
                    o[n] += h * elem(w_down, n * I + c, dtype);
            }
        }
    }
    return ORC_OK;
}

/* Number of OpenMP threads the token loop would use (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
