/*
 * oracle.c -- plain, slow, CPU reference of the MoE SwiGLU FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header or table with the CUDA library.
 *
 * Arithmetic: every floating value is carried in fp64.  bf16 inputs are widened
 * exactly; nothing is rounded back to bf16.  Loops run in the order written, and
 * the file is compiled with -ffp-contract=off so that two loops that perform the
 * same operations in the same order give bit-identical fp64 results.
 *
 * What it computes (the layer, as the pages state it):
 *   - PTO MegaMoE article, section "MoE dispatch/combine 为什么慢": the chain is
 *     a local reorder of routed rows by expert, the expert FFN, and a top-k
 *     weighted accumulation back into token order.
 *   - same article, section "MegaMoE 融合算子七阶段": FrontReorder, Dispatch,
 *     GMM1, SwiGLU, GMM2, Combine, Unpermute.
 *   - Grouped GEMM article ("Grouped GEMM 为什么适合 MoE"), section "Grouped GEMM
 *     到底解决什么问题": C_i = A_i x B_i for independent problems i = 0..G-1.
 *   - same article, section "1. Tiling": each expert's rows cut into tiles of one
 *     uniform height.
 *   - COMET paper review, section 4.1.1 (shared tensor decomposition): layer 0
 *     is independent per token (M), layer 1 couples the top-k rows of a token
 *     through the reduction.
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes): SwiGLU is silu(gate) * up with silu(v) = v / (1 + exp(-v)); W1 [E,H,2F]
 * holds gate in columns [0,F) and up in [F,2F); the permutation is stable in the
 * flat index i = t*topk + k; gate weights are applied as given (no renormalising).
 *
 * Pins (tests that check this file against something other than itself):
 *   plan            python stable sort of (expert, i); invariants; worked tiling
 *                   example of the grouped GEMM article
 *   dispatch        unpermute(permute(x)) = x, bit-exact
 *   grouped GEMM    numpy float64 matmul per expert
 *   swiglu          closed form with math.exp on scalars
 *   layer           E=1,topk=1 equals a dense SwiGLU FFN (torch float64);
 *                   H=F=1 closed form; identical experts => out = FFN(x) * sum w;
 *                   linearity in w; per-token brute force equals the plan path
 *                   bit-exactly
 *   e4m3 codec      torch.float8_e4m3fn on every code and on rounding ties;
 *                   brute-force nearest grid value
 *   fp8 quantisers  torch fp32 division + torch e4m3 conversion; round trip
 *                   within half a grid step; the largest element maps to 448
 *   fp8 GEMM        numpy float64 matmul of the decoded operands
 *   fp8 layer       E=1,topk=1 equals torch's dense chain with the same
 *                   quantisation; within the e4m3 error bound of the exact layer
 *   mx fp8          the exponent rule vs a brute-force search; the quantisers vs
 *                   torch's e4m3 conversion of the exactly scaled values; the MX
 *                   GEMM vs numpy block by block; the MX layer within the E4M3
 *                   error bound of the exact layer
 *   gemm add        beta = 0 and alpha = 0 reduce to the layer and to the added
 *                   tensor exactly; (out - add) of the residual form equals the
 *                   layer; linear in alpha and beta
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_BAD_ID 3

static double bf16_widen(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

int oracle_abi_version(void) { return 1; }

/*
 * Routing plan: per-expert counts, offsets (exclusive prefix sum, E+1 entries),
 * and the stable permutation of the R = M*topk routed rows.
 *   perm[s] = i  -- slot s of the expert-ordered buffer holds flat row i = t*topk+k
 *   inv[i]  = s  -- inverse of perm
 *   w_sorted[s] = w[perm[s]]
 * Within one expert the slots follow ascending i (a counting sort).
 */
int oracle_plan(const int32_t *ids, const float *w, int64_t M, int32_t E, int32_t topk,
                int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                float *w_sorted)
{
    if (M < 0 || E < 1 || topk < 1 || topk > E)
        return ORACLE_ERR_ARG;
    int64_t R = M * (int64_t)topk;
    for (int64_t i = 0; i < R; i++)
        if (ids[i] < 0 || ids[i] >= E)
            return ORACLE_ERR_BAD_ID;

    for (int32_t e = 0; e < E; e++)
        counts[e] = 0;
    for (int64_t i = 0; i < R; i++)
        counts[ids[i]] += 1;

    offsets[0] = 0;
    for (int32_t e = 0; e < E; e++)
        offsets[e + 1] = offsets[e] + counts[e];

    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!cursor)
        return ORACLE_ERR_ARG;
    for (int32_t e = 0; e < E; e++)
        cursor[e] = offsets[e];
    for (int64_t i = 0; i < R; i++) {
        int32_t s = cursor[ids[i]]++;
        perm[s] = (int32_t)i;
        inv[i] = s;
    }
    free(cursor);
    if (w_sorted && w)
        for (int64_t s = 0; s < R; s++)
            w_sorted[s] = w[perm[s]];
    return ORACLE_OK;
}

/*
 * Tiling of the grouped problem: every expert's row segment [offsets[e],
 * offsets[e+1]) is cut into tiles of BM rows; the last tile of an expert may be
 * short, an expert with no rows has no tile.  Tiles are listed expert by expert,
 * top to bottom.  Returns the number of tiles, or -1 if max_tiles is too small.
 */
int64_t oracle_tile_table(const int32_t *offsets, int32_t E, int32_t BM,
                          int32_t *tile_expert, int32_t *tile_row0, int32_t *tile_row1,
                          int64_t max_tiles)
{
    int64_t n = 0;
    for (int32_t e = 0; e < E; e++) {
        for (int32_t r = offsets[e]; r < offsets[e + 1]; r += BM) {
            if (n >= max_tiles)
                return -1;
            tile_expert[n] = e;
            tile_row0[n] = r;
            tile_row1[n] = (r + BM < offsets[e + 1]) ? r + BM : offsets[e + 1];
            n++;
        }
    }
    return n;
}

/* Dispatch (permute): xp[s, :] = x[perm[s] / topk, :]; a copy of bf16 bits. */
void oracle_dispatch(const uint16_t *x, const int32_t *perm, int64_t M, int64_t H,
                     int32_t topk, uint16_t *xp)
{
    int64_t R = M * (int64_t)topk;
    for (int64_t s = 0; s < R; s++) {
        int64_t t = perm[s] / topk;
        memcpy(xp + s * H, x + t * H, sizeof(uint16_t) * (size_t)H);
    }
}

/* Unpermute of a copy: x_back[i, :] = xp[inv[i], :] for flat rows i. */
void oracle_unpermute_rows(const uint16_t *xp, const int32_t *inv, int64_t R, int64_t H,
                           uint16_t *x_back)
{
    for (int64_t i = 0; i < R; i++)
        memcpy(x_back + i * H, xp + (int64_t)inv[i] * H, sizeof(uint16_t) * (size_t)H);
}

/*
 * Grouped GEMM: for every expert e and every row s of its segment,
 *   C[s, n] = sum_{k=0}^{K-1} A[s, k] * B[e, k, n]      (k ascending)
 * A bf16 [R, K] row-major, B bf16 [E, K, N] row-major, C fp64 [R, N].
 */
void oracle_grouped_gemm(const uint16_t *A, const uint16_t *B, const int32_t *offsets,
                         int32_t E, int64_t K, int64_t N, double *C)
{
    for (int32_t e = 0; e < E; e++) {
        const uint16_t *Be = B + (int64_t)e * K * N;
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t s = offsets[e]; s < offsets[e + 1]; s++) {
            double *c = C + s * N;
            for (int64_t n = 0; n < N; n++)
                c[n] = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double a = bf16_widen(A[s * K + k]);
                const uint16_t *b = Be + k * N;
                for (int64_t n = 0; n < N; n++)
                    c[n] += a * bf16_widen(b[n]);
            }
        }
    }
}

/* SwiGLU on a gate|up row block: h[s, j] = silu(G[s, j]) * G[s, F + j]. */
void oracle_swiglu(const double *G, int64_t R, int64_t F, double *h)
{
    for (int64_t s = 0; s < R; s++)
        for (int64_t j = 0; j < F; j++)
            h[s * F + j] = silu(G[s * 2 * F + j]) * G[s * 2 * F + F + j];
}

/*
 * Combine of expert-ordered, unweighted rows:
 *   out[t, c] = sum_{k=0}^{topk-1} w[t, k] * yp[inv[t*topk + k], c]   (k ascending)
 */
void oracle_combine(const double *yp, const int32_t *inv, const float *w, int64_t M,
                    int64_t H, int32_t topk, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; t++) {
        double *o = out + t * H;
        for (int64_t c = 0; c < H; c++)
            o[c] = 0.0;
        for (int32_t k = 0; k < topk; k++) {
            int64_t i = t * topk + k;
            double wk = (double)w[i];
            const double *y = yp + (int64_t)inv[i] * H;
            for (int64_t c = 0; c < H; c++)
                o[c] += wk * y[c];
        }
    }
}

/*
 * One expert's FFN on one bf16 row v [H]:
 *   g = v . W1[e]            (2F values, sum over h ascending)
 *   a[j] = silu(g[j]) * g[F + j]
 *   y = a . W2[e]            (H values, sum over j ascending)
 * scratch must hold 2F + F doubles.
 */
static void expert_ffn_row(const uint16_t *v, const uint16_t *W1e, const uint16_t *W2e,
                           int64_t H, int64_t F, double *scratch, double *y)
{
    double *g = scratch;
    double *a = scratch + 2 * F;
    for (int64_t j = 0; j < 2 * F; j++)
        g[j] = 0.0;
    for (int64_t h = 0; h < H; h++) {
        double xv = bf16_widen(v[h]);
        const uint16_t *wrow = W1e + h * 2 * F;
        for (int64_t j = 0; j < 2 * F; j++)
            g[j] += xv * bf16_widen(wrow[j]);
    }
    for (int64_t j = 0; j < F; j++)
        a[j] = silu(g[j]) * g[F + j];
    for (int64_t c = 0; c < H; c++)
        y[c] = 0.0;
    for (int64_t j = 0; j < F; j++) {
        const uint16_t *wrow = W2e + j * H;
        for (int64_t c = 0; c < H; c++)
            y[c] += a[j] * bf16_widen(wrow[c]);
    }
}

/*
 * The whole layer through the plan, stage by stage:
 *   plan -> dispatch -> per expert (GEMM1, SwiGLU, GEMM2) on its row segment ->
 *   weighted combine back to token order (k ascending).
 * out fp64 [M, H].  Returns an ORACLE_* status.
 */
int oracle_moe_ffn(const uint16_t *x, const uint16_t *W1, const uint16_t *W2,
                   const int32_t *ids, const float *w, int64_t M, int64_t H, int64_t F,
                   int32_t E, int32_t topk, double *out)
{
    int64_t R = M * (int64_t)topk;
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R ? R : 1));
    int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R ? R : 1));
    uint16_t *xp = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(R ? R * H : 1));
    double *yp = (double *)malloc(sizeof(double) * (size_t)(R ? R * H : 1));
    int st = ORACLE_ERR_ARG;
    if (!counts || !offsets || !perm || !inv || !xp || !yp)
        goto done;
    st = oracle_plan(ids, w, M, E, topk, counts, offsets, perm, inv, NULL);
    if (st != ORACLE_OK)
        goto done;
    oracle_dispatch(x, perm, M, H, topk, xp);
    for (int32_t e = 0; e < E; e++) {
        const uint16_t *W1e = W1 + (int64_t)e * H * 2 * F;
        const uint16_t *W2e = W2 + (int64_t)e * F * H;
#pragma omp parallel
        {
            double *scratch = (double *)malloc(sizeof(double) * (size_t)(3 * F));
#pragma omp for schedule(dynamic, 4)
            for (int64_t s = offsets[e]; s < offsets[e + 1]; s++)
                expert_ffn_row(xp + s * H, W1e, W2e, H, F, scratch, yp + s * H);
            free(scratch);
        }
    }
    oracle_combine(yp, inv, w, M, H, topk, out);
done:
    free(counts);
    free(offsets);
    free(perm);
    free(inv);
    free(xp);
    free(yp);
    return st;
}

/*
 * Fused GemmAdd epilogue (grouped GEMM article, section "Fused GemmAdd"): the
 * accumulated result and an added tensor combined before the one output cast,
 *   y[i] = alpha * acc[i] + beta * add[i]
 * here applied to the layer output: acc fp64 [n] (e.g. oracle_moe_ffn's out),
 * add bf16 [n] (e.g. the residual stream x), y fp64 [n].  Nothing is rounded.
 */
void oracle_gemm_add(const double *acc, const uint16_t *add, double alpha, double beta, int64_t n,
                     double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++)
        y[i] = alpha * acc[i] + beta * bf16_widen(add[i]);
}

/*
 * Brute force, no plan: for each listed token t,
 *   out_rows[j, :] = sum_{k ascending} w[t, k] * FFN_{ids[t, k]}(x[t])
 * with the same per-row arithmetic as oracle_moe_ffn, so the two agree bit for
 * bit.  Used on small cases as a cross-check and on large cases to compute a
 * sample of output rows one by one.
 */
int oracle_bruteforce_tokens(const uint16_t *x, const uint16_t *W1, const uint16_t *W2,
                             const int32_t *ids, const float *w, int64_t H, int64_t F,
                             int32_t E, int32_t topk, const int64_t *tokens, int64_t n_tokens,
                             double *out_rows)
{
    for (int64_t j = 0; j < n_tokens; j++)
        for (int32_t k = 0; k < topk; k++) {
            int32_t e = ids[tokens[j] * topk + k];
            if (e < 0 || e >= E)
                return ORACLE_ERR_BAD_ID;
        }
#pragma omp parallel
    {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)(3 * F));
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(dynamic, 1)
        for (int64_t j = 0; j < n_tokens; j++) {
            int64_t t = tokens[j];
            double *o = out_rows + j * H;
            for (int64_t c = 0; c < H; c++)
                o[c] = 0.0;
            for (int32_t k = 0; k < topk; k++) {
                int32_t e = ids[t * topk + k];
                expert_ffn_row(x + t * H, W1 + (int64_t)e * H * 2 * F,
                               W2 + (int64_t)e * F * H, H, F, scratch, y);
                double wk = (double)w[t * topk + k];
                for (int64_t c = 0; c < H; c++)
                    o[c] += wk * y[c];
            }
        }
        free(scratch);
        free(y);
    }
    return ORACLE_OK;
}

/*
 * Router (the step before the layer; the grouped GEMM article's introduction:
 * the router hands each token to some experts).  Reading taken, since the pages
 * define no router: a token goes to the topk experts with the largest logits,
 * largest first, ties to the lower expert index; its gate weights are the
 * softmax over those topk logits:
 *   w[t, k] = exp(l[t, ids[t, k]]) / sum_j exp(l[t, ids[t, j]])
 * Selection compares the given fp32 values exactly; the softmax runs in fp64
 * (shifted by the largest chosen logit).  topk <= E; returns ORACLE_ERR_ARG
 * otherwise.
 */
int oracle_route(const float *logits, int64_t M, int32_t E, int32_t topk, int32_t *ids,
                 double *w)
{
    if (M < 0 || E < 1 || topk < 1 || topk > E)
        return ORACLE_ERR_ARG;
    for (int64_t t = 0; t < M; t++) {
        const float *l = logits + t * E;
        int32_t *out = ids + t * topk;
        for (int32_t k = 0; k < topk; k++) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; e++) {
                int taken = 0;
                for (int32_t j = 0; j < k; j++)
                    if (out[j] == e)
                        taken = 1;
                if (taken)
                    continue;
                if (best < 0 || l[e] > l[best])
                    best = e;
            }
            out[k] = best;
        }
        double mx = (double)l[out[0]];
        double sum = 0.0;
        for (int32_t k = 0; k < topk; k++)
            sum += exp((double)l[out[k]] - mx);
        for (int32_t k = 0; k < topk; k++)
            w[t * topk + k] = exp((double)l[out[k]] - mx) / sum;
    }
    return ORACLE_OK;
}

/* Number of OpenMP threads the oracle's parallel loops use. */
/* ------------------------------------------------------------------ FP8 (E4M3) */

/*
 * 8-bit floating point E4M3 (the OCP 8-bit format without infinities): bit 7
 * sign, bits 6..3 exponent with bias 7, bits 2..0 mantissa.  Exponent field 0 is
 * subnormal: value = m * 2^-9.  Otherwise value = (1 + m/8) * 2^(exp - 7).  The
 * pattern S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
 */
double oracle_e4m3_decode(uint8_t c)
{
    int sign = c >> 7, ex = (c >> 3) & 15, m = c & 7;
    double v;
    if (ex == 15 && m == 7)
        return NAN;
    if (ex == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, ex - 7);
    return sign ? -v : v;
}

/*
 * Nearest E4M3 value to v, ties to the even mantissa; magnitudes that round
 * beyond 448 saturate to 448 (the conversion the quantiser uses); NaN -> 0x7F.
 * Every step is exact in fp64: |v| is a float, the grid spacing a power of two.
 */
static uint8_t e4m3_encode_d(double v)
{
    if (isnan(v))
        return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    /* spacing of the grid around a: 2^(e-3) in binade [2^e, 2^(e+1)), e >= -6;
       the subnormal range [0, 2^-6) has spacing 2^-9 */
    int e = -6;
    if (a >= ldexp(1.0, -6)) {
        int ex;
        frexp(a, &ex); /* a = f * 2^ex with f in [0.5, 1) */
        e = ex - 1;
    }
    double step = ldexp(1.0, e - 3);
    double q = a / step; /* exact: division by a power of two */
    double fl = floor(q);
    double rem = q - fl;
    double n = fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))
        n = fl + 1.0;
    double r = n * step; /* rounded magnitude */
    if (r > 448.0)
        r = 448.0;
    if (r < ldexp(1.0, -6))
        return sign | (uint8_t)(r / ldexp(1.0, -9)); /* subnormal (or zero) */
    int ex;
    double f = frexp(r, &ex); /* r = f * 2^ex, f in [0.5, 1) */
    int be = ex - 1 + 7;     /* biased exponent */
    int m = (int)((f * 2.0 - 1.0) * 8.0);
    return sign | (uint8_t)(be << 3) | (uint8_t)m;
}

uint8_t oracle_e4m3_encode(float v) { return e4m3_encode_d((double)v); }

/*
 * Per-row scaled quantisation of a bf16 matrix A [R, K] (the SwiGLU output h):
 *   scale[r] = max_k |A[r, k]| / 448   (fp32 division; 1 for an all-zero row)
 *   q[r, k]  = e4m3(A[r, k] / scale[r]) (fp32 division, then the encoding above)
 * so that A[r, k] ~= scale[r] * decode(q[r, k]) and the largest element maps to
 * +-448.  This is the "quantise right after SwiGLU" step of the PTO MegaMoE
 * article (section "MegaMoE 融合算子七阶段"), with one scale per row (token).
 */
void oracle_quantize_rows_e4m3(const uint16_t *A, int64_t R, int64_t K, uint8_t *q, float *scale)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float v = fabsf((float)bf16_widen(A[r * K + k]));
            if (v > amax)
                amax = v;
        }
        float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        scale[r] = sc;
        for (int64_t k = 0; k < K; k++)
            q[r * K + k] = oracle_e4m3_encode((float)bf16_widen(A[r * K + k]) / sc);
    }
}

/*
 * Per-output-column scaled quantisation of bf16 weights B [E, K, N] (row-major, N
 * contiguous), written transposed so that K is contiguous:
 *   scale[e, n] = max_k |B[e, k, n]| / 448   (1 for an all-zero column)
 *   qT[e, n, k] = e4m3(B[e, k, n] / scale[e, n])
 */
void oracle_quantize_cols_e4m3(const uint16_t *B, int32_t E, int64_t K, int64_t N, uint8_t *qT,
                               float *scale)
{
    for (int32_t e = 0; e < E; e++) {
        const uint16_t *Be = B + (int64_t)e * K * N;
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; n++) {
            float amax = 0.0f;
            for (int64_t k = 0; k < K; k++) {
                float v = fabsf((float)bf16_widen(Be[k * N + n]));
                if (v > amax)
                    amax = v;
            }
            float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
            scale[(int64_t)e * N + n] = sc;
            uint8_t *qrow = qT + ((int64_t)e * N + n) * K;
            for (int64_t k = 0; k < K; k++)
                qrow[k] = oracle_e4m3_encode((float)bf16_widen(Be[k * N + n]) / sc);
        }
    }
}

/*
 * Grouped GEMM on quantised operands, dequantised exactly in fp64:
 *   C[s, n] = a_scale[s] * b_scale[e, n] * sum_k decode(Aq[s, k]) * decode(BqT[e, n, k])
 * for the rows s of expert e (Aq [R, K] row-major; BqT [E, N, K], K contiguous).
 */
void oracle_grouped_gemm_e4m3(const uint8_t *Aq, const float *a_scale, const uint8_t *BqT,
                              const float *b_scale, const int32_t *offsets, int32_t E,
                              int64_t K, int64_t N, double *C)
{
    double lut[256];
    for (int c = 0; c < 256; c++)
        lut[c] = oracle_e4m3_decode((uint8_t)c);
    for (int32_t e = 0; e < E; e++) {
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t s = offsets[e]; s < offsets[e + 1]; s++) {
            const uint8_t *a = Aq + s * K;
            for (int64_t n = 0; n < N; n++) {
                const uint8_t *b = BqT + ((int64_t)e * N + n) * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; k++)
                    acc += lut[a[k]] * lut[b[k]];
                C[s * N + n] = (double)a_scale[s] * (double)b_scale[(int64_t)e * N + n] * acc;
            }
        }
    }
}

/* ------------------------------------------------------- MX (block-scaled) FP8 */

/*
 * Microscaled E4M3: elements in blocks of 32 consecutive values along the
 * contraction dimension share one power-of-two scale 2^e, stored as the 8-bit
 * exponent code e + 127 (E8M0: code 0 is 2^-127, 254 is 2^127, 255 unused).
 * The reading taken here (the pages only say that SwiGLU quantises what it
 * consumes): e is the smallest integer with amax <= 448 * 2^e, amax the block's
 * largest magnitude, so no element of the block saturates; e = -127 for an
 * all-zero block, clamped to [-127, 127].  q = nearest E4M3 to v * 2^-e (the
 * scaling is exact, one rounding).
 */
int oracle_mx_exponent(double amax)
{
    if (!(amax > 0.0))
        return -127;
    int ex;
    frexp(amax, &ex); /* amax in [2^(ex-1), 2^ex) */
    /* 448 * 2^(ex-9) = 1.75 * 2^(ex-1) is the smallest candidate (448 * 2^(ex-10) < 2^(ex-1)) */
    int e = ex - 9;
    if (amax > ldexp(448.0, e))
        e += 1;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/*
 * Rows of A [R, K] (given values, e.g. the SwiGLU output h) quantised in blocks of
 * 32 along K: sf[r, b] = e + 127 of block b, q[r, k] = e4m3(A[r, k] * 2^-e).
 * K is a multiple of 32.
 */
void oracle_mx_quantize_rows(const double *A, int64_t R, int64_t K, uint8_t *q, uint8_t *sf)
{
    int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++) {
        for (int64_t b = 0; b < nb; b++) {
            const double *v = A + r * K + b * 32;
            double amax = 0.0;
            for (int k = 0; k < 32; k++)
                if (fabs(v[k]) > amax)
                    amax = fabs(v[k]);
            int e = oracle_mx_exponent(amax);
            sf[r * nb + b] = (uint8_t)(e + 127);
            for (int k = 0; k < 32; k++)
                q[r * K + b * 32 + k] = e4m3_encode_d(ldexp(v[k], -e));
        }
    }
}

/*
 * Weights B [E, K, N] (bf16, row-major, N contiguous) quantised per output column
 * in blocks of 32 along K, written transposed (K contiguous):
 *   sf[e, n, b] = e + 127 of the block B[e, 32b .. 32b+31, n]
 *   qT[e, n, k] = e4m3(B[e, k, n] * 2^-e)
 */
void oracle_mx_quantize_cols(const uint16_t *B, int32_t E, int64_t K, int64_t N, uint8_t *qT,
                             uint8_t *sf)
{
    int64_t nb = K / 32;
    for (int32_t e = 0; e < E; e++) {
        const uint16_t *Be = B + (int64_t)e * K * N;
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; n++) {
            for (int64_t b = 0; b < nb; b++) {
                double amax = 0.0;
                for (int k = 0; k < 32; k++) {
                    double v = fabs(bf16_widen(Be[(b * 32 + k) * N + n]));
                    if (v > amax)
                        amax = v;
                }
                int ex = oracle_mx_exponent(amax);
                sf[((int64_t)e * N + n) * nb + b] = (uint8_t)(ex + 127);
                for (int k = 0; k < 32; k++)
                    qT[((int64_t)e * N + n) * K + b * 32 + k] =
                        e4m3_encode_d(ldexp(bf16_widen(Be[(b * 32 + k) * N + n]), -ex));
            }
        }
    }
}

/*
 * Grouped GEMM on block-scaled operands, exact in fp64:
 *   C[s, n] = sum_b 2^(a_sf[s, b] - 127) * 2^(b_sf[e, n, b] - 127)
 *                   * sum_{k in block b} decode(Aq[s, k]) * decode(BqT[e, n, k])
 * for the rows s of expert e.  Aq [R, K], a_sf [R, K/32], BqT [E, N, K],
 * b_sf [E, N, K/32].
 */
void oracle_grouped_gemm_mx(const uint8_t *Aq, const uint8_t *a_sf, const uint8_t *BqT,
                            const uint8_t *b_sf, const int32_t *offsets, int32_t E, int64_t K,
                            int64_t N, double *C)
{
    double lut[256];
    for (int c = 0; c < 256; c++)
        lut[c] = oracle_e4m3_decode((uint8_t)c);
    int64_t nb = K / 32;
    for (int32_t e = 0; e < E; e++) {
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t s = offsets[e]; s < offsets[e + 1]; s++) {
            for (int64_t n = 0; n < N; n++) {
                const uint8_t *a = Aq + s * K;
                const uint8_t *bq = BqT + ((int64_t)e * N + n) * K;
                double acc = 0.0;
                for (int64_t b = 0; b < nb; b++) {
                    double part = 0.0;
                    for (int k = 0; k < 32; k++)
                        part += lut[a[b * 32 + k]] * lut[bq[b * 32 + k]];
                    acc += ldexp(part, (int)a_sf[s * nb + b] - 127 +
                                           (int)b_sf[((int64_t)e * N + n) * nb + b] - 127);
                }
                C[s * N + n] = acc;
            }
        }
    }
}

/* Round an fp64 value to the nearest bf16 (ties to even) and return its bits. */
static uint16_t bf16_round(double v)
{
    if (isnan(v))
        return 0x7FC0;
    /* bf16 keeps 8 significant bits; scale to an integer grid of that spacing */
    if (v == 0.0)
        return signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    int ex;
    frexp(a, &ex); /* a in [2^(ex-1), 2^ex) */
    int e = ex - 1;
    if (e < -126)
        e = -126; /* subnormal spacing 2^-133 */
    double step = ldexp(1.0, e - 7);
    double q = a / step;
    double fl = floor(q), rem = q - fl, n = fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0))
        n = fl + 1.0;
    float r = (float)(n * step); /* exact: n*step has at most 8 significant bits */
    if (v < 0)
        r = -r;
    uint32_t u;
    memcpy(&u, &r, sizeof u);
    return (uint16_t)(u >> 16);
}

/*
 * The layer with its down projection in FP8 (E4M3), stage by stage:
 *   plan -> dispatch -> GEMM1 + SwiGLU (fp64) -> h rounded to bf16 ->
 *   h quantised per row -> GEMM2 on the quantised h and the per-column quantised
 *   W2 (dequantised exactly) -> weighted combine (k ascending).
 * out fp64 [M, H].  Returns an ORACLE_* status.
 */
int oracle_moe_ffn_fp8(const uint16_t *x, const uint16_t *W1, const uint16_t *W2,
                       const int32_t *ids, const float *w, int64_t M, int64_t H, int64_t F,
                       int32_t E, int32_t topk, double *out)
{
    int64_t R = M * (int64_t)topk;
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R ? R : 1));
    int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R ? R : 1));
    uint16_t *xp = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(R ? R * H : 1));
    uint16_t *hb = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(R ? R * F : 1));
    uint8_t *hq = (uint8_t *)malloc((size_t)(R ? R * F : 1));
    float *hs = (float *)malloc(sizeof(float) * (size_t)(R ? R : 1));
    uint8_t *wq = (uint8_t *)malloc((size_t)(E * H * F));
    float *ws = (float *)malloc(sizeof(float) * (size_t)(E * H));
    double *yp = (double *)malloc(sizeof(double) * (size_t)(R ? R * H : 1));
    int st = ORACLE_ERR_ARG;
    if (!counts || !offsets || !perm || !inv || !xp || !hb || !hq || !hs || !wq || !ws || !yp)
        goto done;
    st = oracle_plan(ids, w, M, E, topk, counts, offsets, perm, inv, NULL);
    if (st != ORACLE_OK)
        goto done;
    oracle_dispatch(x, perm, M, H, topk, xp);
    for (int32_t e = 0; e < E; e++) {
        const uint16_t *W1e = W1 + (int64_t)e * H * 2 * F;
#pragma omp parallel
        {
            double *g = (double *)malloc(sizeof(double) * (size_t)(2 * F));
#pragma omp for schedule(dynamic, 4)
            for (int64_t s = offsets[e]; s < offsets[e + 1]; s++) {
                for (int64_t j = 0; j < 2 * F; j++)
                    g[j] = 0.0;
                for (int64_t h = 0; h < H; h++) {
                    double xv = bf16_widen(xp[s * H + h]);
                    const uint16_t *wrow = W1e + h * 2 * F;
                    for (int64_t j = 0; j < 2 * F; j++)
                        g[j] += xv * bf16_widen(wrow[j]);
                }
                for (int64_t j = 0; j < F; j++)
                    hb[s * F + j] = bf16_round(silu(g[j]) * g[F + j]);
            }
            free(g);
        }
    }
    oracle_quantize_rows_e4m3(hb, R, F, hq, hs);
    oracle_quantize_cols_e4m3(W2, E, F, H, wq, ws);
    oracle_grouped_gemm_e4m3(hq, hs, wq, ws, offsets, E, F, H, yp);
    oracle_combine(yp, inv, w, M, H, topk, out);
done:
    free(counts);
    free(offsets);
    free(perm);
    free(inv);
    free(xp);
    free(hb);
    free(hq);
    free(hs);
    free(wq);
    free(ws);
    free(yp);
    return st;
}

/*
 * The layer with a block-scaled (MX) E4M3 down projection, stage by stage:
 *   plan -> dispatch -> per expert GEMM1 and SwiGLU in fp64 -> h quantised in
 *   blocks of 32 columns (oracle_mx_quantize_rows on the fp64 values: the SwiGLU
 *   output feeds the quantiser directly, no bf16 rounding between) -> GEMM2 on the
 *   block-scaled operands (W2 quantised per output column in blocks of 32 rows of
 *   F) -> weighted combine.  out fp64 [M, H].
 */
int oracle_moe_ffn_mx(const uint16_t *x, const uint16_t *W1, const uint16_t *W2,
                      const int32_t *ids, const float *w, int64_t M, int64_t H, int64_t F,
                      int32_t E, int32_t topk, double *out)
{
    int64_t R = M * (int64_t)topk;
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R ? R : 1));
    int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R ? R : 1));
    uint16_t *xp = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(R ? R * H : 1));
    double *hd = (double *)malloc(sizeof(double) * (size_t)(R ? R * F : 1));
    uint8_t *hq = (uint8_t *)malloc((size_t)(R ? R * F : 1));
    uint8_t *hsf = (uint8_t *)malloc((size_t)(R ? R * (F / 32) : 1));
    uint8_t *wq = (uint8_t *)malloc((size_t)(E * H * F));
    uint8_t *wsf = (uint8_t *)malloc((size_t)(E * H * (F / 32)));
    double *yp = (double *)malloc(sizeof(double) * (size_t)(R ? R * H : 1));
    int st = ORACLE_ERR_ARG;
    if (F % 32 != 0 || !counts || !offsets || !perm || !inv || !xp || !hd || !hq || !hsf || !wq ||
        !wsf || !yp)
        goto done;
    st = oracle_plan(ids, w, M, E, topk, counts, offsets, perm, inv, NULL);
    if (st != ORACLE_OK)
        goto done;
    oracle_dispatch(x, perm, M, H, topk, xp);
    for (int32_t e = 0; e < E; e++) {
        const uint16_t *W1e = W1 + (int64_t)e * H * 2 * F;
#pragma omp parallel
        {
            double *g = (double *)malloc(sizeof(double) * (size_t)(2 * F));
#pragma omp for schedule(dynamic, 4)
            for (int64_t s = offsets[e]; s < offsets[e + 1]; s++) {
                for (int64_t j = 0; j < 2 * F; j++)
                    g[j] = 0.0;
                for (int64_t h = 0; h < H; h++) {
                    double xv = bf16_widen(xp[s * H + h]);
                    const uint16_t *wrow = W1e + h * 2 * F;
                    for (int64_t j = 0; j < 2 * F; j++)
                        g[j] += xv * bf16_widen(wrow[j]);
                }
                for (int64_t j = 0; j < F; j++)
                    hd[s * F + j] = silu(g[j]) * g[F + j];
            }
            free(g);
        }
    }
    oracle_mx_quantize_rows(hd, R, F, hq, hsf);
    oracle_mx_quantize_cols(W2, E, F, H, wq, wsf);
    oracle_grouped_gemm_mx(hq, hsf, wq, wsf, offsets, E, F, H, yp);
    oracle_combine(yp, inv, w, M, H, topk, out);
done:
    free(counts);
    free(offsets);
    free(perm);
    free(inv);
    free(xp);
    free(hd);
    free(hq);
    free(hsf);
    free(wq);
    free(wsf);
    free(yp);
    return st;
}

int oracle_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
