/*
 * sphkv_oracle.c -- plain fp64 CPU oracle for Spherical KV.
 *
 * TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU
 * baseline leg of the benchmark are the only callers of this library; the
 * product path never loads it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * What it follows.  "SPHERICAL KV: Angle-Domain Attention and Rate-Distortion
 * Retention for Efficient Long-Context Inference" (arXiv 2605.18856), Abstract
 * and AI Summary:
 *   - ADA keeps every key as a scalar radius plus compact angle codes (a point
 *     on the hypersphere) and gets the attention logits from those codes;
 *   - RDR chooses keep/drop and a precision tier for each unit under a fixed
 *     byte budget, as a rate-distortion problem, so that pages are
 *     tier-homogeneous.
 * The pages fix no formula, grid, bit width or layout.  The format written out
 * here is the one this project fixes: a recursive-polar (binary-tree)
 * parameterisation with d/2 leaf pair angles and d/2-1 upper angles, three
 * tiers (T1 8/8 bits + int8 V, T2 4/6 bits + int4 V, T3 3/4 bits + int4 V),
 * 16-token pages and a Lagrangian bisection for RDR.  Where the pages leave a
 * point open, the reading taken is stated next to the code that takes it.
 *
 * How.  Plain loops in fp64, compiled with -ffp-contract=off so no product is
 * ever fused into an add.  Attention is done the slow, obvious way: decode the
 * codes to a dense fp64 key, then dense softmax attention.  The bottom-up
 * logit tree is present only so the tests can check it against that.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_PAGE 16
#define ORC_D 128 /* head size of the packed page format */

/* ---------------------------------------------------------------- fp16 -- */

/* Round a double to IEEE binary16, round-half-to-even, one rounding step. */
uint16_t orc_f64_to_f16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(x)) return 0x7e00u;
    if (isinf(x)) return (uint16_t)(sign | 0x7c00u);
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1) */
    int E = e - 1;               /* a in [2^E, 2^(E+1)) */
    if (E < -14) E = -14;        /* subnormal range shares the 2^-24 quantum */
    double quantum = ldexp(1.0, E - 10);
    double n = rint(a / quantum); /* exact scaling by a power of two, then RNE */
    if (n >= 2048.0) { E += 1; n = n / 2.0; }
    if (E > 15) return (uint16_t)(sign | 0x7c00u);
    if (n < 1024.0) return (uint16_t)(sign | (uint16_t)n); /* subnormal */
    return (uint16_t)(sign | (uint16_t)(((E + 15) << 10) | ((int)n - 1024)));
}

double orc_f16_to_f64(uint16_t h)
{
    int s = (h >> 15) & 1, ex = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (ex == 0) v = ldexp((double)m, -24);
    else if (ex == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m + 1024), ex - 25);
    return s ? -v : v;
}

/* ------------------------------------------------------------- tiers -- */

/* Tier index 1..3 -> (b_leaf, b_up, v_bits).  0 is "drop". */
static const int ORC_BLEAF[4] = {0, 8, 4, 3};
static const int ORC_BUP[4] = {0, 8, 6, 4};
static const int ORC_VBITS[4] = {0, 8, 4, 4};

/* Bytes of the code blocks of one token (8 subtree blocks) and of one value
 * row, per tier. */
static int code_row_bytes(int t) { return t == 1 ? 128 : t == 2 ? 80 : 56; }
static int v_row_bytes(int t) { return ORC_D * ORC_VBITS[t] / 8; }

/* Field offsets inside a page: r[16] fp16, vscale[16] fp16, code planes,
 * value rows. */
static int off_codes(int t) { (void)t; return 2 * ORC_PAGE * 2; }
static int off_v(int t) { return off_codes(t) + ORC_PAGE * code_row_bytes(t); }

int orc_page_bytes(int t)
{
    if (t < 1 || t > 3) return 0;
    return off_v(t) + ORC_PAGE * v_row_bytes(t);
}

/* ------------------------------------------------------------ encode -- */

/* Leaf angle code.  phi = atan2(y, x) in (-pi, pi]; the grid is periodic with
 * 2^b points at c * 2pi / 2^b; rounding to nearest (ties to even); a zero pair
 * gets code 0. */
static int leaf_code(double x, double y, int b)
{
    long M = 1L << b;
    if (x == 0.0 && y == 0.0) return 0;
    double phi = atan2(y, x);
    double t = rint((phi * (double)M) / (2.0 * M_PI));
    long c = (long)t;
    c = ((c % M) + M) % M;
    return (int)c;
}

/* Upper angle code.  psi = atan2(|right|, |left|) in [0, pi/2]; the grid
 * includes both ends: c * (pi/2) / (2^b - 1), c = 0 .. 2^b - 1. */
static int upper_code(double ss_left, double ss_right, int b)
{
    long top = (1L << b) - 1;
    double nl = sqrt(ss_left), nr = sqrt(ss_right);
    double psi = (nl == 0.0 && nr == 0.0) ? 0.0 : atan2(nr, nl);
    double t = rint((psi * (double)top) / M_PI_2);
    if (t < 0.0) t = 0.0;
    if (t > (double)top) t = (double)top;
    return (int)t;
}

/* Encode one token of one head.  k, v: [d] fp64 (exact copies of the bf16 or
 * fp32 inputs).  leaf: [d/2] codes, up: [d/2-1] codes in level order (level 1
 * parents of leaves (2m, 2m+1) first, the root last).  Returns 0, or 1 when
 * the radius or the value scale overflows fp16. */
static int encode_one(int d, const double* k_in, const double* v, int b_leaf, int b_up,
                      int v_bits, uint8_t* leaf, uint8_t* up, uint16_t* r16, uint16_t* s16,
                      int8_t* vq, double* work)
{
    int L = d / 2;
    double* k = work;          /* [d] */
    double* ss = work + d;     /* [2L - 1]: leaves then upper nodes, level order */
    for (int i = 0; i < d; ++i) k[i] = k_in[i] + 0.0; /* -0 -> +0 */
    for (int j = 0; j < L; ++j) {
        double x = k[2 * j], y = k[2 * j + 1];
        ss[j] = x * x + y * y;
        leaf[j] = (uint8_t)leaf_code(x, y, b_leaf);
    }
    /* upper nodes: children of level-(l) node m are nodes 2m, 2m+1 of level l-1 */
    int child = 0, node = L, width = L / 2, u = 0;
    while (width >= 1) {
        for (int m = 0; m < width; ++m) {
            double sl = ss[child + 2 * m], sr = ss[child + 2 * m + 1];
            ss[node + m] = sl + sr;
            up[u++] = (uint8_t)upper_code(sl, sr, b_up);
        }
        child = node;
        node += width;
        width /= 2;
    }
    int bad = 0;
    double r = sqrt(ss[2 * L - 2]);
    *r16 = orc_f64_to_f16(r);
    if ((*r16 & 0x7c00u) == 0x7c00u) bad = 1;

    double Q = (v_bits == 8) ? 127.0 : 7.0;
    double a = 0.0;
    for (int c = 0; c < d; ++c) a = fmax(a, fabs(v[c]));
    *s16 = orc_f64_to_f16(a / Q);
    if ((*s16 & 0x7c00u) == 0x7c00u) bad = 1;
    double s = orc_f16_to_f64(*s16);
    for (int c = 0; c < d; ++c) {
        double t = (s == 0.0) ? 0.0 : rint(v[c] / s);
        if (t > Q) t = Q;
        if (t < -Q) t = -Q;
        vq[c] = (int8_t)t;
    }
    return bad;
}

/* Encode n tokens (rows of K and V, each [d]).  Returns the number of tokens
 * whose radius or value scale overflowed fp16. */
int64_t orc_encode_tokens(int64_t n, int d, const double* K, const double* V, int b_leaf,
                          int b_up, int v_bits, uint8_t* leaf, uint8_t* up, uint16_t* r16,
                          uint16_t* s16, int8_t* vq)
{
    int64_t bad = 0;
    int L = d / 2;
#pragma omp parallel reduction(+ : bad)
    {
        double* work = (double*)malloc(sizeof(double) * (size_t)(3 * d));
#pragma omp for schedule(static)
        for (int64_t i = 0; i < n; ++i)
            bad += encode_one(d, K + i * d, V + i * d, b_leaf, b_up, v_bits, leaf + i * L,
                              up + i * (L - 1), r16 + i, s16 + i, vq + i * d, work);
        free(work);
    }
    return bad;
}

/* ------------------------------------------------------------ decode -- */

static double leaf_angle(int c, int b) { return (2.0 * M_PI * (double)c) / (double)(1L << b); }
static double upper_angle(int c, int b) { return (M_PI_2 * (double)c) / (double)((1L << b) - 1); }

/* Unit direction from the codes, top-down: the root has weight 1, a left child
 * gets w*cos(psi), a right child w*sin(psi); leaf j gives
 * (w_j cos(phi_j), w_j sin(phi_j)). */
static void unit_vector(int d, const uint8_t* leaf, const uint8_t* up, int b_leaf, int b_up,
                        double* u, double* w)
{
    int L = d / 2;
    /* w holds node weights in level order (leaves 0..L-1, upper nodes after). */
    w[2 * L - 2] = 1.0;
    int node = 2 * L - 2, width = 1;
    /* walk levels from the root down; upper node index in up[] == node - L */
    while (width < L) {
        int child = node - 2 * width; /* first node of the level below */
        for (int m = 0; m < width; ++m) {
            double psi = upper_angle(up[node - L + m], b_up);
            double wn = w[node + m];
            w[child + 2 * m] = wn * cos(psi);
            w[child + 2 * m + 1] = wn * sin(psi);
        }
        node = child;
        width *= 2;
    }
    for (int j = 0; j < L; ++j) {
        double phi = leaf_angle(leaf[j], b_leaf);
        u[2 * j] = w[j] * cos(phi);
        u[2 * j + 1] = w[j] * sin(phi);
    }
}

/* k_hat = r_hat * u_hat for one token; w is [d] scratch. */
static void decode_key_one(int d, const uint8_t* leaf, const uint8_t* up, uint16_t r16,
                           int b_leaf, int b_up, double* khat, double* w)
{
    unit_vector(d, leaf, up, b_leaf, b_up, khat, w);
    double r = orc_f16_to_f64(r16);
    for (int c = 0; c < d; ++c) khat[c] = r * khat[c];
}

/* k_hat = r_hat * u_hat for n tokens. */
void orc_decode_keys(int64_t n, int d, const uint8_t* leaf, const uint8_t* up,
                     const uint16_t* r16, int b_leaf, int b_up, double* khat)
{
    int L = d / 2;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)(2 * L));
#pragma omp for schedule(static)
        for (int64_t i = 0; i < n; ++i)
            decode_key_one(d, leaf + i * L, up + i * (L - 1), r16[i], b_leaf, b_up,
                           khat + i * d, w);
        free(w);
    }
}

/* v_hat = code * scale for n tokens. */
void orc_decode_values(int64_t n, int d, const int8_t* vq, const uint16_t* s16, double* vhat)
{
    for (int64_t i = 0; i < n; ++i) {
        double s = orc_f16_to_f64(s16[i]);
        for (int c = 0; c < d; ++c) vhat[i * d + c] = (double)vq[i * d + c] * s;
    }
}

/* Bottom-up angle-domain logit: leaf S_j = q_2j cos(phi_j) + q_2j+1 sin(phi_j),
 * node S = cos(psi) S_left + sin(psi) S_right, logit = r_hat S_root / sqrt(d).
 * Used only by the tests, to check it against q . decode(codes) / sqrt(d). */
void orc_tree_logits(int64_t n, int d, const uint8_t* leaf, const uint8_t* up,
                     const uint16_t* r16, int b_leaf, int b_up, const double* q,
                     double* logits)
{
    int L = d / 2;
    double* S = (double*)malloc(sizeof(double) * (size_t)(2 * L));
    for (int64_t i = 0; i < n; ++i) {
        const uint8_t* lc = leaf + i * L;
        const uint8_t* uc = up + i * (L - 1);
        for (int j = 0; j < L; ++j) {
            double phi = leaf_angle(lc[j], b_leaf);
            S[j] = q[2 * j] * cos(phi) + q[2 * j + 1] * sin(phi);
        }
        int child = 0, node = L, width = L / 2;
        while (width >= 1) {
            for (int m = 0; m < width; ++m) {
                double psi = upper_angle(uc[node - L + m], b_up);
                S[node + m] = cos(psi) * S[child + 2 * m] + sin(psi) * S[child + 2 * m + 1];
            }
            child = node;
            node += width;
            width /= 2;
        }
        logits[i] = orc_f16_to_f64(r16[i]) * S[2 * L - 2] / sqrt((double)d);
    }
    free(S);
}

/* --------------------------------------------------------- attention -- */

/* Dense softmax attention of n_q query rows over n_keys (all kept) keys.
 * logit_t = q . k_t / sqrt(d); out = sum_t e^(l_t - M) v_t / sum_t e^(l_t - M);
 * lse = M + ln(sum_t e^(l_t - M)).  No keys: out = 0, lse = -inf. */
void orc_attention(int64_t n_keys, int d, const double* khat, const double* vhat, int n_q,
                   const double* q, double* out, double* lse)
{
    double* l = (double*)malloc(sizeof(double) * (size_t)(n_keys > 0 ? n_keys : 1));
    double sd = sqrt((double)d);
    for (int h = 0; h < n_q; ++h) {
        const double* qh = q + (int64_t)h * d;
        double* oh = out + (int64_t)h * d;
        for (int c = 0; c < d; ++c) oh[c] = 0.0;
        if (n_keys == 0) { lse[h] = -INFINITY; continue; }
        double M = -INFINITY;
        for (int64_t t = 0; t < n_keys; ++t) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qh[c] * khat[t * d + c];
            l[t] = dot / sd;
            if (l[t] > M) M = l[t];
        }
        double Z = 0.0;
        for (int64_t t = 0; t < n_keys; ++t) {
            double e = exp(l[t] - M);
            Z += e;
            for (int c = 0; c < d; ++c) oh[c] += e * vhat[t * d + c];
        }
        for (int c = 0; c < d; ++c) oh[c] /= Z;
        lse[h] = M + log(Z);
    }
    free(l);
}

/* Combine attention results over disjoint key sets of the same query rows
 * (split-KV: each part attended to its own keys; Spherical KV, Abstract:
 * long-context inference; the log-sum-exp combine is the one the decode path
 * uses to merge its own splits).  With M = max_r lse_r and w_r =
 * e^(lse_r - M):  out = sum_r w_r out_r / sum_r w_r,  lse = M + ln sum_r w_r,
 * which is attention over the union of the parts' keys.  A part with
 * lse = -inf (no keys) has w_r = 0; if every part is empty, out = 0 and
 * lse = -inf.  out_parts [n_parts][n_rows][d], lse_parts [n_parts][n_rows]. */
void orc_merge_partials(int n_parts, int64_t n_rows, int d, const double* out_parts, const double* lse_parts,
                        double* out, double* lse)
{
    for (int64_t i = 0; i < n_rows; ++i) {
        double M = -INFINITY;
        for (int r = 0; r < n_parts; ++r)
            if (lse_parts[(int64_t)r * n_rows + i] > M) M = lse_parts[(int64_t)r * n_rows + i];
        double* o = out + i * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (M == -INFINITY) { lse[i] = -INFINITY; continue; }
        double Z = 0.0;
        for (int r = 0; r < n_parts; ++r) {
            double l = lse_parts[(int64_t)r * n_rows + i];
            if (l == -INFINITY) continue;
            double w = exp(l - M);
            Z += w;
            const double* orow = out_parts + ((int64_t)r * n_rows + i) * d;
            for (int c = 0; c < d; ++c) o[c] += w * orow[c];
        }
        for (int c = 0; c < d; ++c) o[c] /= Z;
        lse[i] = M + log(Z);
    }
}

/* -------------------------------------------------------- page format -- */

/* The codes of one token regrouped into 8 subtree blocks, one per 8-leaf
 * subtree s:  L[s][j] = leaf 8s+j;  U[s][0..3] = level-1 nodes 4s..4s+3,
 * U[s][4..5] = level-2 nodes 2s, 2s+1, U[s][6] = level-3 node s, and
 * U[s][7] = top node s for s < 7, where the top nodes are level 4 (4 nodes),
 * level 5 (2 nodes) and the root; U[7][7] = 0.  Level-order index of level-1
 * node m is m, level 2 is 32 + m, level 3 is 48 + m, level 4 is 56 + m,
 * level 5 is 60 + m, the root 62. */
static void to_blocks(const uint8_t* leaf, const uint8_t* up, uint8_t L[8][8], uint8_t U[8][8])
{
    for (int s = 0; s < 8; ++s) {
        for (int j = 0; j < 8; ++j) L[s][j] = leaf[8 * s + j];
        for (int j = 0; j < 4; ++j) U[s][j] = up[4 * s + j];
        U[s][4] = up[32 + 2 * s];
        U[s][5] = up[32 + 2 * s + 1];
        U[s][6] = up[48 + s];
        U[s][7] = s < 7 ? up[56 + s] : 0;
    }
}

static void from_blocks(uint8_t L[8][8], uint8_t U[8][8], uint8_t* leaf, uint8_t* up)
{
    for (int s = 0; s < 8; ++s) {
        for (int j = 0; j < 8; ++j) leaf[8 * s + j] = L[s][j];
        for (int j = 0; j < 4; ++j) up[4 * s + j] = U[s][j];
        up[32 + 2 * s] = U[s][4];
        up[32 + 2 * s + 1] = U[s][5];
        up[48 + s] = U[s][6];
        if (s < 7) up[56 + s] = U[s][7];
    }
}

/* Value row position p = 16g + 2m + h (g, m = 0..7, h = 0..1) holds channel
 * 16m + g + 8h. */
static int v_channel_at(int p) { return 16 * ((p >> 1) & 7) + (p >> 4) + 8 * (p & 1); }

/* Byte of the value section that holds row position p (0..127) of token
 * `slot`.  int8 (T1): rows of 128 bytes, 16-byte chunk g = p/16 of row r
 * stored at chunk g ^ (r & 6).  int4 (T2, T3): tokens 2i and 2i+1 share a
 * 128-byte block of eight 16-byte chunks; chunk g ^ (2i & 6) holds 8 bytes of
 * token 2i then 8 bytes of token 2i+1 (positions 16g .. 16g+15, two per byte,
 * even position in the low nibble). */
static int v_byte_at(int t, int slot, int p)
{
    int g = p >> 4, j = p & 15;
    if (ORC_VBITS[t] == 8) return off_v(t) + slot * 128 + 16 * (g ^ (slot & 6)) + j;
    int i = slot >> 1;
    return off_v(t) + i * 128 + 16 * (g ^ ((2 * i) & 6)) + 8 * (slot & 1) + (j >> 1);
}

static void put_le(uint8_t* dst, int nbytes, uint64_t v)
{
    for (int i = 0; i < nbytes; ++i) dst[i] = (uint8_t)(v >> (8 * i));
}

static uint64_t get_le(const uint8_t* src, int nbytes)
{
    uint64_t v = 0;
    for (int i = 0; i < nbytes; ++i) v |= (uint64_t)src[i] << (8 * i);
    return v;
}

/* Store one token (d = 128) into slot `slot` of a page of tier t (1..3).
 * Code planes (each [16 tokens][8 blocks][width] bytes, in this order):
 *   T1: width 16: bytes 0..7 = L[s][0..7], bytes 8..15 = U[s][0..7];
 *   T2: width 8: u32 with nibble j = L[s][j], then the low 32 bits of the
 *       48-bit field with bits 6j..6j+5 = U[s][j];  width 2: u16 = the high
 *       16 bits of that field;
 *   T3: width 4: u32 with nibble j = U[s][j];  width 2: u16 = the low 16 bits
 *       of the 24-bit field with bits 3j..3j+2 = L[s][j];  width 1: u8 = its
 *       high 8 bits.
 * Multi-byte fields are little-endian.  Value row position p holds channel
 * v_channel_at(p), stored at v_byte_at (int4: two's complement nibbles). */
void orc_pack_token(int t, int slot, const uint8_t* leaf, const uint8_t* up, uint16_t r16,
                    uint16_t s16, const int8_t* vq, uint8_t* page)
{
    uint8_t L[8][8], U[8][8];
    to_blocks(leaf, up, L, U);
    put_le(page + 2 * slot, 2, r16);
    put_le(page + 2 * ORC_PAGE + 2 * slot, 2, s16);
    uint8_t* c = page + off_codes(t);
    for (int s = 0; s < 8; ++s) {
        int blk = slot * 8 + s;
        if (t == 1) {
            for (int j = 0; j < 8; ++j) {
                c[blk * 16 + j] = L[s][j];
                c[blk * 16 + 8 + j] = U[s][j];
            }
        } else if (t == 2) {
            uint64_t lf = 0, uf = 0;
            for (int j = 0; j < 8; ++j) {
                lf |= (uint64_t)L[s][j] << (4 * j);
                uf |= (uint64_t)U[s][j] << (6 * j);
            }
            put_le(c + blk * 8, 8, lf | (uf << 32));
            put_le(c + ORC_PAGE * 8 * 8 + blk * 2, 2, uf >> 32);
        } else {
            uint64_t uf = 0, lf = 0;
            for (int j = 0; j < 8; ++j) {
                uf |= (uint64_t)U[s][j] << (4 * j);
                lf |= (uint64_t)L[s][j] << (3 * j);
            }
            put_le(c + blk * 4, 4, uf);
            put_le(c + ORC_PAGE * 8 * 4 + blk * 2, 2, lf & 0xffff);
            put_le(c + ORC_PAGE * 8 * 6 + blk, 1, lf >> 16);
        }
    }
    for (int p = 0; p < ORC_D; ++p) {
        int code = vq[v_channel_at(p)];
        int off = v_byte_at(t, slot, p);
        if (ORC_VBITS[t] == 8) page[off] = (uint8_t)code;
        else if (p & 1) page[off] = (uint8_t)((page[off] & 0x0f) | ((code & 15) << 4));
        else page[off] = (uint8_t)((page[off] & 0xf0) | (code & 15));
    }
}

void orc_unpack_token(int t, int slot, const uint8_t* page, uint8_t* leaf, uint8_t* up,
                      uint16_t* r16, uint16_t* s16, int8_t* vq)
{
    uint8_t L[8][8], U[8][8];
    *r16 = (uint16_t)get_le(page + 2 * slot, 2);
    *s16 = (uint16_t)get_le(page + 2 * ORC_PAGE + 2 * slot, 2);
    const uint8_t* c = page + off_codes(t);
    for (int s = 0; s < 8; ++s) {
        int blk = slot * 8 + s;
        if (t == 1) {
            for (int j = 0; j < 8; ++j) {
                L[s][j] = c[blk * 16 + j];
                U[s][j] = c[blk * 16 + 8 + j];
            }
        } else if (t == 2) {
            uint64_t a = get_le(c + blk * 8, 8), b = get_le(c + ORC_PAGE * 8 * 8 + blk * 2, 2);
            uint64_t uf = (a >> 32) | (b << 32);
            for (int j = 0; j < 8; ++j) {
                L[s][j] = (uint8_t)((a >> (4 * j)) & 15);
                U[s][j] = (uint8_t)((uf >> (6 * j)) & 63);
            }
        } else {
            uint64_t a = get_le(c + blk * 4, 4), b = get_le(c + ORC_PAGE * 8 * 4 + blk * 2, 2),
                     e = get_le(c + ORC_PAGE * 8 * 6 + blk, 1);
            uint64_t lf = b | (e << 16);
            for (int j = 0; j < 8; ++j) {
                U[s][j] = (uint8_t)((a >> (4 * j)) & 15);
                L[s][j] = (uint8_t)((lf >> (3 * j)) & 7);
            }
        }
    }
    from_blocks(L, U, leaf, up);
    for (int p = 0; p < ORC_D; ++p) {
        int off = v_byte_at(t, slot, p);
        int raw;
        if (ORC_VBITS[t] == 8) raw = (int8_t)page[off];
        else {
            raw = (page[off] >> (4 * (p & 1))) & 15;
            if (raw >= 8) raw -= 16; /* two's complement */
        }
        vq[v_channel_at(p)] = (int8_t)raw;
    }
}

/* Bulk form of orc_pack_token: token i goes to page dst_page[i] of `pool`
 * (pages of tier t, orc_page_bytes(t) each), slot slot[i].  Codes are the
 * [n][64], [n][63], [n], [n], [n][128] arrays of orc_encode_tokens. */
void orc_pack_tokens(int64_t n, int t, const int64_t* dst_page, const int32_t* slot,
                     const uint8_t* leaf, const uint8_t* up, const uint16_t* r16,
                     const uint16_t* s16, const int8_t* vq, uint8_t* pool)
{
    int64_t pb = orc_page_bytes(t);
    for (int64_t i = 0; i < n; ++i)
        orc_pack_token(t, slot[i], leaf + i * (ORC_D / 2), up + i * (ORC_D / 2 - 1), r16[i], s16[i],
                       vq + i * ORC_D, pool + dst_page[i] * pb);
}

/* Page-table entry: bits 31..30 tier (0 drop, 1 T1, 2 T2, 3 T3), bits 29..0
 * the page's index in that tier's pool. */
void orc_build_page_table(int64_t n_entries, const uint8_t* tiers, const int32_t* perm1,
                          const int32_t* perm2, const int32_t* perm3, int32_t* table)
{
    const int32_t* perm[4] = {NULL, perm1, perm2, perm3};
    int64_t next[4] = {0, 0, 0, 0};
    for (int64_t i = 0; i < n_entries; ++i) {
        int t = tiers[i];
        if (t == 0) { table[i] = 0; continue; }
        int64_t k = next[t]++;
        int64_t phys = perm[t] ? perm[t][k] : k;
        table[i] = (int32_t)(((uint32_t)t << 30) | (uint32_t)phys);
    }
}

/* Decode attention over a paged cache, computed the slow way, for the units
 * (sequence b, kv head g) listed in sel_b/sel_g.  For each unit: unpack every
 * kept token (t < seq_len, page not dropped), decode it to a dense fp64 key and
 * value, then dense softmax attention for the G = H_q / H_kv query heads
 * h = g*G .. g*G+G-1 (query head h reads kv head h / G).
 * q: [B][H_q][128]; out: [n_sel][G][128]; lse: [n_sel][G].
 * page_table: [H_kv][total_pages]; page_offsets: [B+1] (pages of sequence b
 * are page_offsets[b] .. page_offsets[b+1]-1, for every kv head).
 * Returns 0, or 6 for an entry whose page index lies outside its pool. */
int orc_cache_attention(int B, int H_q, int H_kv, int64_t total_pages, const int32_t* page_offsets,
                        const int32_t* seq_lens, const int32_t* page_table, const uint8_t* pool1,
                        const uint8_t* pool2, const uint8_t* pool3, const int64_t* pool_pages,
                        const double* q, int n_sel, const int32_t* sel_b, const int32_t* sel_g,
                        double* out, double* lse)
{
    const uint8_t* pools[4] = {NULL, pool1, pool2, pool3};
    int G = H_q / H_kv;
    int status = 0;
    (void)B;
#pragma omp parallel for schedule(dynamic, 1)
    for (int s = 0; s < n_sel; ++s) {
        int b = sel_b[s], g = sel_g[s];
        int64_t len = seq_lens[b];
        int64_t first = page_offsets[b];
        double* K = (double*)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1) * ORC_D);
        double* V = (double*)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1) * ORC_D);
        uint8_t leaf[ORC_D / 2], up[ORC_D / 2 - 1];
        int8_t vq[ORC_D];
        double w[ORC_D];
        uint16_t r16, s16;
        int64_t n = 0;
        for (int64_t t = 0; t < len; ++t) {
            int32_t e = page_table[(int64_t)g * total_pages + first + t / ORC_PAGE];
            int tier = (int)(((uint32_t)e) >> 30);
            int64_t phys = (int64_t)(((uint32_t)e) & 0x3fffffffu);
            if (tier == 0) continue;
            if (phys >= pool_pages[tier - 1]) {
#pragma omp atomic write
                status = 6;
                continue;
            }
            const uint8_t* page = pools[tier] + phys * (int64_t)orc_page_bytes(tier);
            orc_unpack_token(tier, (int)(t % ORC_PAGE), page, leaf, up, &r16, &s16, vq);
            if (r16 & 0x8000u) continue; /* the token's drop flag (see orc_set_keep) */
            decode_key_one(ORC_D, leaf, up, r16, ORC_BLEAF[tier], ORC_BUP[tier], K + n * ORC_D, w);
            orc_decode_values(1, ORC_D, vq, &s16, V + n * ORC_D);
            ++n;
        }
        orc_attention(n, ORC_D, K, V, G, q + ((int64_t)b * H_q + (int64_t)g * G) * ORC_D,
                      out + (int64_t)s * G * ORC_D, lse + (int64_t)s * G);
        free(K);
        free(V);
    }
    return status;
}

/* Transcoding a stored token to a coarser tier, from its codes alone (the
 * dense key is gone once a page is written).  Reading (the pages give no
 * rule): each angle is moved to the nearest point of the coarser grid,
 * computed exactly on the code integers with ties to even, which is what
 * re-encoding the decoded angle would give without the rounding noise of
 * atan2; the radius (and its drop flag) is kept; the values are decoded
 * (code * scale, exact in fp64) and quantised again with the encoder's rule
 * for the new width. */

/* Round-half-even of num / den for num >= 0, den > 0. */
static int64_t div_rne(int64_t num, int64_t den)
{
    int64_t q = num / den, r = num % den;
    if (2 * r > den || (2 * r == den && (q & 1))) ++q;
    return q;
}

/* Leaf code on the periodic 2^b_from grid -> nearest point of the 2^b_to grid
 * (b_to <= b_from): c * 2^b_to / 2^b_from, ties to even, modulo 2^b_to. */
static int transcode_leaf(int c, int b_from, int b_to)
{
    return (int)(div_rne((int64_t)c << b_to, (int64_t)1 << b_from) % ((int64_t)1 << b_to));
}

/* Upper code on the end-inclusive grid with 2^b_from - 1 steps -> nearest
 * point of the 2^b_to - 1 step grid: c (2^b_to - 1) / (2^b_from - 1), ties to
 * even (the denominator is odd, so none occur). */
static int transcode_upper(int c, int b_from, int b_to)
{
    return (int)div_rne((int64_t)c * (((int64_t)1 << b_to) - 1), ((int64_t)1 << b_from) - 1);
}

/* One token from tier t_from to tier t_to (t_to no finer than t_from). */
void orc_transcode_token(int t_from, int t_to, const uint8_t* leaf, const uint8_t* up, uint16_t s16,
                         const int8_t* vq, uint8_t* leaf_out, uint8_t* up_out, uint16_t* s16_out, int8_t* vq_out)
{
    for (int j = 0; j < ORC_D / 2; ++j) leaf_out[j] = (uint8_t)transcode_leaf(leaf[j], ORC_BLEAF[t_from], ORC_BLEAF[t_to]);
    for (int j = 0; j < ORC_D / 2 - 1; ++j) up_out[j] = (uint8_t)transcode_upper(up[j], ORC_BUP[t_from], ORC_BUP[t_to]);
    double v[ORC_D];
    orc_decode_values(1, ORC_D, vq, &s16, v);
    double Q = (ORC_VBITS[t_to] == 8) ? 127.0 : 7.0;
    double a = 0.0;
    for (int c = 0; c < ORC_D; ++c) a = fmax(a, fabs(v[c]));
    *s16_out = orc_f64_to_f16(a / Q);
    double s = orc_f16_to_f64(*s16_out);
    for (int c = 0; c < ORC_D; ++c) {
        double t = (s == 0.0) ? 0.0 : rint(v[c] / s);
        if (t > Q) t = Q;
        if (t < -Q) t = -Q;
        vq_out[c] = (int8_t)t;
    }
}

/* Rewrite a cache into new pools after its tiers changed (RDR run again):
 * every present token of a page kept by the new table is transcoded from its
 * old page into its new page (a page whose tier did not change moves
 * unchanged: no re-quantisation); pages the new table
 * drops are not written.  The new pools must be zeroed by the caller.  A page
 * the new table makes finer than before, or keeps although it was dropped,
 * cannot be rebuilt from codes: status 6 (the page is skipped). */
int orc_migrate(int B, int H_kv, int64_t total_pages, const int32_t* page_offsets, const int32_t* seq_lens,
                const int32_t* old_table, const uint8_t* old1, const uint8_t* old2, const uint8_t* old3,
                const int64_t* old_pages, const int32_t* new_table, uint8_t* new1, uint8_t* new2, uint8_t* new3,
                const int64_t* new_pages)
{
    const uint8_t* olds[4] = {NULL, old1, old2, old3};
    uint8_t* news[4] = {NULL, new1, new2, new3};
    int status = 0;
    uint8_t leaf[ORC_D / 2], up[ORC_D / 2 - 1], leaf2[ORC_D / 2], up2[ORC_D / 2 - 1];
    int8_t vq[ORC_D], vq2[ORC_D];
    for (int g = 0; g < H_kv; ++g)
        for (int b = 0; b < B; ++b)
            for (int64_t t = 0; t < seq_lens[b]; ++t) {
                int64_t lp = (int64_t)g * total_pages + page_offsets[b] + t / ORC_PAGE;
                int32_t eo = old_table[lp], en = new_table[lp];
                int to = (int)(((uint32_t)eo) >> 30), tn = (int)(((uint32_t)en) >> 30);
                int64_t po = (int64_t)(((uint32_t)eo) & 0x3fffffffu), pn = (int64_t)(((uint32_t)en) & 0x3fffffffu);
                if (tn == 0) continue;
                if (to == 0 || tn < to || po >= old_pages[to - 1] || pn >= new_pages[tn - 1]) { status = 6; continue; }
                uint16_t r16, s16, s16b;
                int slot = (int)(t % ORC_PAGE);
                orc_unpack_token(to, slot, olds[to] + po * (int64_t)orc_page_bytes(to), leaf, up, &r16, &s16, vq);
                if (tn == to) /* same tier: the token moves unchanged */
                    orc_pack_token(tn, slot, leaf, up, r16, s16, vq, news[tn] + pn * (int64_t)orc_page_bytes(tn));
                else {
                    orc_transcode_token(to, tn, leaf, up, s16, vq, leaf2, up2, &s16b, vq2);
                    orc_pack_token(tn, slot, leaf2, up2, r16, s16b, vq2, news[tn] + pn * (int64_t)orc_page_bytes(tn));
                }
            }
    return status;
}

/* Per-token keep/drop inside kept pages.  Spherical KV, Abstract: RDR makes
 * keep/drop decisions per token and head.  Reading: a stored radius is
 * fp16(|k|) >= +0, so its sign bit is free; it is the token's drop flag (1 =
 * dropped), and attention skips a dropped token exactly as if it had been
 * deleted.  keep: [H_kv][total_pages * 16] bytes in the layout of RDR's
 * utility (slot s of logical page i at i * 16 + s); for every present token
 * (position < seq_len) of every page that is not dropped, the flag is set
 * when keep is 0 and cleared otherwise.  Pools are modified in place. */
int orc_set_keep(int B, int H_kv, int64_t total_pages, const int32_t* page_offsets, const int32_t* seq_lens,
                 const int32_t* page_table, uint8_t* pool1, uint8_t* pool2, uint8_t* pool3,
                 const int64_t* pool_pages, const uint8_t* keep)
{
    uint8_t* pools[4] = {NULL, pool1, pool2, pool3};
    int status = 0;
    for (int g = 0; g < H_kv; ++g)
        for (int b = 0; b < B; ++b)
            for (int64_t t = 0; t < seq_lens[b]; ++t) {
                int64_t lp = page_offsets[b] + t / ORC_PAGE;
                int32_t e = page_table[(int64_t)g * total_pages + lp];
                int tier = (int)(((uint32_t)e) >> 30);
                int64_t phys = (int64_t)(((uint32_t)e) & 0x3fffffffu);
                if (tier == 0) continue;
                if (phys >= pool_pages[tier - 1]) { status = 6; continue; }
                uint8_t* r = pools[tier] + phys * (int64_t)orc_page_bytes(tier) + 2 * (t % ORC_PAGE);
                uint16_t r16 = (uint16_t)get_le(r, 2);
                int k = keep[(int64_t)g * total_pages * ORC_PAGE + lp * ORC_PAGE + t % ORC_PAGE] != 0;
                r16 = k ? (uint16_t)(r16 & 0x7fffu) : (uint16_t)(r16 | 0x8000u);
                put_le(r, 2, r16);
            }
    return status;
}

/* ---------------------------------------------------------------- RDR -- */

/* Lagrangian tier choice for one unit: argmin over t of U*eps[t] + lambda*R[t],
 * ties to the lower index (higher precision).  Index 0..3 = T1, T2, T3, drop. */
static int rdr_choice(double U, const double* eps, const double* R, double lambda, int first)
{
    int best = first;
    double bc = U * eps[first] + lambda * R[first];
    for (int t = first + 1; t < 4; ++t) {
        double c = U * eps[t] + lambda * R[t];
        if (c < bc) { bc = c; best = t; }
    }
    return best;
}

/* Tier (1..3, 0 = drop) -> choice index (0..3 = T1, T2, T3, drop). */
static int tier_index(int tier) { return tier == 0 ? 3 : tier - 1; }

/* Rate-distortion retention.  Units are (kv head g, sequence b, page p) for
 * p < ceil(seq_len/16).  U = sum of the per-token utilities of the valid
 * tokens (t = 0..15 in order).  Rate R = page bytes of the tier (drop = 0);
 * distortion D = U * eps[tier].  The first n_sink and last n_recent pages of
 * each sequence are forced to T1 and count against the budget.  The other
 * units take argmin D + lambda R; lambda is found by doubling from 1 until the
 * bytes fit, then 100 bisection steps, keeping the feasible end.
 * utility: [H_kv][total_pages*16] (token slot of page i at i*16 + slot).
 * tiers: [H_kv][total_pages], written 1..3 or 0 (drop) for pages that hold
 * tokens; other entries are left untouched.
 * Returns 0, or 3 when the forced pages alone exceed the budget. */
static int rdr_run(int B, int H_kv, int64_t total_pages, const int32_t* page_offsets, const int32_t* seq_lens,
                   const float* utility, const double* eps, int64_t budget, int n_sink, int n_recent,
                   const uint8_t* cap, uint8_t* tiers, double* lambda_out, int64_t* bytes_out);

int orc_rdr_assign(int B, int H_kv, int64_t total_pages, const int32_t* page_offsets,
                   const int32_t* seq_lens, const float* utility, const double* eps,
                   int64_t budget, int n_sink, int n_recent, uint8_t* tiers,
                   double* lambda_out, int64_t* bytes_out)
{
    return rdr_run(B, H_kv, total_pages, page_offsets, seq_lens, utility, eps, budget, n_sink, n_recent, NULL,
                   tiers, lambda_out, bytes_out);
}

/* RDR run again on a cache whose pages already hold codes (the context has
 * grown; Spherical KV, AI Summary: retention allocates precision and storage
 * dynamically by estimated utility).  Reading: a page's codes can only be
 * made coarser without the dense key, so every unit's choices are limited to
 * its current tier and the coarser ones (drop included); forced units (first
 * n_sink, last n_recent pages) keep the finest tier they are allowed, i.e.
 * T1 if they are T1 and their current tier otherwise.  tiers holds the
 * current tiers on entry and the new ones on return (pages that hold tokens;
 * other entries untouched).  Otherwise exactly orc_rdr_assign. */
int orc_rdr_rerun(int B, int H_kv, int64_t total_pages, const int32_t* page_offsets, const int32_t* seq_lens,
                  const float* utility, const double* eps, int64_t budget, int n_sink, int n_recent,
                  uint8_t* tiers, double* lambda_out, int64_t* bytes_out)
{
    int64_t n = (int64_t)H_kv * total_pages;
    uint8_t* cap = (uint8_t*)malloc((size_t)(n > 0 ? n : 1));
    memcpy(cap, tiers, (size_t)n);
    int st = rdr_run(B, H_kv, total_pages, page_offsets, seq_lens, utility, eps, budget, n_sink, n_recent, cap,
                     tiers, lambda_out, bytes_out);
    free(cap);
    return st;
}

static int rdr_run(int B, int H_kv, int64_t total_pages, const int32_t* page_offsets, const int32_t* seq_lens,
                   const float* utility, const double* eps, int64_t budget, int n_sink, int n_recent,
                   const uint8_t* cap, uint8_t* tiers, double* lambda_out, int64_t* bytes_out)
{
    double R[4];
    for (int t = 0; t < 3; ++t) R[t] = (double)orc_page_bytes(t + 1);
    R[3] = 0.0;
    /* flatten units */
    int64_t n_units = 0;
    for (int b = 0; b < B; ++b) n_units += (seq_lens[b] + ORC_PAGE - 1) / ORC_PAGE;
    n_units *= H_kv;
    double* U = (double*)malloc(sizeof(double) * (size_t)(n_units > 0 ? n_units : 1));
    int64_t* idx = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_units > 0 ? n_units : 1));
    uint8_t* forced = (uint8_t*)malloc((size_t)(n_units > 0 ? n_units : 1));
    uint8_t* first = (uint8_t*)malloc((size_t)(n_units > 0 ? n_units : 1)); /* finest allowed choice */
    int64_t u = 0, forced_bytes = 0;
    for (int g = 0; g < H_kv; ++g)
        for (int b = 0; b < B; ++b) {
            int64_t len = seq_lens[b];
            int64_t np = (len + ORC_PAGE - 1) / ORC_PAGE;
            for (int64_t p = 0; p < np; ++p) {
                int64_t e = (int64_t)g * total_pages + page_offsets[b] + p;
                double s = 0.0;
                for (int k = 0; k < ORC_PAGE && p * ORC_PAGE + k < len; ++k)
                    s += (double)utility[e * ORC_PAGE + k];
                U[u] = s;
                idx[u] = e;
                first[u] = (uint8_t)(cap ? tier_index(cap[e]) : 0);
                forced[u] = (p < n_sink || p >= np - n_recent) ? 1 : 0;
                if (forced[u]) forced_bytes += (int64_t)R[first[u]];
                ++u;
            }
        }
    if (forced_bytes > budget) {
        free(U); free(idx); free(forced); free(first);
        return 3;
    }
#define RDR_BYTES(lam, out_bytes)                                               \
    do {                                                                        \
        int64_t acc_ = 0;                                                       \
        for (int64_t i_ = 0; i_ < n_units; ++i_)                                \
            acc_ += forced[i_] ? (int64_t)R[first[i_]]                          \
                               : (int64_t)R[rdr_choice(U[i_], eps, R, (lam), first[i_])]; \
        (out_bytes) = acc_;                                                     \
    } while (0)
    double lo = 0.0, hi = 1.0;
    int64_t bh;
    RDR_BYTES(hi, bh);
    for (int k = 0; k < 2000 && bh > budget; ++k) {
        hi = hi * 2.0;
        RDR_BYTES(hi, bh);
    }
    for (int it = 0; it < 100; ++it) {
        double mid = lo + (hi - lo) / 2.0;
        int64_t bm;
        RDR_BYTES(mid, bm);
        if (bm <= budget) hi = mid;
        else lo = mid;
    }
    RDR_BYTES(hi, bh);
#undef RDR_BYTES
    for (int64_t i = 0; i < n_units; ++i) {
        int t = forced[i] ? first[i] : rdr_choice(U[i], eps, R, hi, first[i]);
        tiers[idx[i]] = (uint8_t)(t == 3 ? 0 : t + 1);
    }
    *lambda_out = hi;
    *bytes_out = bh;
    free(U); free(idx); free(forced); free(first);
    return 0;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
