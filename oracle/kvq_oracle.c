/*
 * kvq_oracle.c -- plain, slow, single-threaded fp64 CPU oracle for decode
 * attention over a prunable 2-bit KV cache ("Dual-QK: Sharp Queries and Flat
 * Keys for Prunable 2-bit KV Caches").
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this file's library.  The
 * product path never calls it, and it shares no code, header, table or
 * constant with the CUDA library: the page layout below is written out here
 * on its own from the format's definition.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no contraction: every fused multiply-add below is an explicit fma()).
 *
 * What each function follows:
 *   orc_f16_rne / orc_bf16_rne  IEEE-754 binary16 / bfloat16, one rounding
 *                               to nearest, ties to even, from binary64.
 *   orc_transform               Dual-QK §3.1, Eq. (QA)(KB)^T = QK^T: rows are
 *                               multiplied by a fixed matrix; the sum over the
 *                               input channel runs c = 0..d-1 as a chain of
 *                               fma starting from 0.0.
 *   orc_quantize_group          Dual-QK §3.3 (asymmetric INT2 grid per token,
 *                               min/max range); group of channels, fp16 scale
 *                               and zero-point, codes = clamp(rint((x-z)/s)).
 *   orc_append_unit(_g)         Dual-QK §3.3 (channel 0 of K kept in BF16 and
 *                               excluded from the range; channel-major rows,
 *                               one 32-byte row per channel of a 128-token page);
 *                               groups of 32 channels, or of 128 -- the pages'
 *                               one INT2 grid per token and KV head.
 *   orc_quantize_group_clip     the same grid over [clip*min, clip*max]:
 *                               Dual-QK App. B.2 (values: per-token asymmetric
 *                               INT2 with a clipping ratio of 0.92; keys are
 *                               not clipped); orc_append_unit_c clips values.
 *   orc_num_selected, orc_select
 *                               Dual-QK §3.2, Eq. 4 (pooled query energy
 *                               e_j^2 = sum_h q'_{h,j}^2 over the GQA group);
 *                               channel 0 always kept; ties to the lower index.
 *   orc_select_scaled           §3.3 diagonal refinement and App. C.2: with
 *                               A = A0 D, selection uses the base queries
 *                               q A0 = (q A) D^{-1}, scores the final ones.
 *   orc_rope_unanchor, orc_decode_buckets
 *                               §3.4 and App. C.4 (bucket-relative RoPE):
 *                               keys are stored in the frame of their bucket's
 *                               anchor, z_n = k_n T_b B, the query of bucket b
 *                               is q T_b A, each bucket has its own channel
 *                               mask, one softmax over all buckets.  T_b
 *                               removes the anchor's rotary rotation (rotate-
 *                               half channel pairs).
 *   value rotation              §3.3 / App. B.2: values are multiplied by an
 *                               orthogonal rotation before quantization
 *                               (orc_transform) and the aggregated output by
 *                               its transpose (orc_transform with R^T).
 *   orc_dequant_unit            inverse of the quantizer: x = s*code + z.
 *   orc_decode_dense            Dual-QK §3.2 (retained channels, original
 *                               1/sqrt(d) normalisation) and §3.4 (one softmax
 *                               over all scores, then value aggregation).
 *   orc_attention               textbook softmax(q K^T / sqrt(d)) V.
 *   orc_protected_slot, orc_protect_store, orc_protect_dequant
 *                               Dual-QK §3.3 (the first 64 and the most
 *                               recent 256 tokens kept in BF16 for keys and
 *                               values, same query-channel mask) and §3.4
 *                               (all precision tiers share one softmax):
 *                               a sink slot per early position, a ring of
 *                               slots for the recent window, and the
 *                               dequantized cache with the protected
 *                               positions replaced by their BF16 values.
 *
 * Parity pins: every function here is checked by the CPU test suite against
 * closed forms, library routines or brute force (see tests/test_oracle_*.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_D 128           /* head dimension */
#define ORC_T 128           /* tokens per page */
#define ORC_G 32            /* channels per quantization group */
#define ORC_NG (ORC_D / ORC_G)

/* ------------------------------------------------------------------------ */
/* rounding of binary64 to binary16 / bfloat16                               */
/* ------------------------------------------------------------------------ */

/* Round |x| (finite, > 0) to a float format with `mbits` explicit mantissa
 * bits, exponent bias `bias` and `ebits` exponent bits.  Returns the encoded
 * magnitude bits.  Method: pick the spacing (ulp) of the target format at
 * x's binade (or the subnormal spacing), scale x to units of that spacing
 * (exact: a power of two), round with rint (nearest, ties to even), and
 * encode.  A carry to the next binade encodes naturally.                   */
static uint32_t round_magnitude(double ax, int mbits, int bias, int ebits)
{
    int emax = (1 << ebits) - 2 - bias;          /* largest normal exponent   */
    int emin = 1 - bias;                         /* smallest normal exponent  */
    int ex;
    frexp(ax, &ex);                              /* ax = f * 2^ex, f in [.5,1) */
    ex -= 1;                                     /* ax in [2^ex, 2^(ex+1))    */
    if (ex > emax)                               /* at or above 2^(emax+1)    */
        return (uint32_t)((1 << ebits) - 1) << mbits;   /* infinity          */
    int ulp_e = (ex >= emin) ? ex - mbits : emin - mbits;
    double r = rint(ldexp(ax, -ulp_e));          /* integer multiple of ulp   */
    if (ex < emin) {                             /* subnormal range           */
        /* r <= 2^mbits; r == 2^mbits is the smallest normal, encoded as-is  */
        return (uint32_t)r;
    }
    /* normal: r in [2^mbits, 2^(mbits+1)] */
    uint32_t m = (uint32_t)r;
    int e = ex;
    if (m == (1u << (mbits + 1))) {              /* carried into next binade */
        m >>= 1;
        e += 1;
        if (e > emax)
            return (uint32_t)((1 << ebits) - 1) << mbits;
    }
    return ((uint32_t)(e + bias) << mbits) | (m - (1u << mbits));
}

static uint16_t round_to_small_float(double x, int mbits, int bias, int ebits,
                                     uint16_t qnan)
{
    uint16_t sign = signbit(x) ? (uint16_t)(1u << (mbits + ebits)) : 0;
    if (isnan(x))
        return (uint16_t)(sign | qnan);
    if (isinf(x))
        return (uint16_t)(sign | (((1u << ebits) - 1) << mbits));
    if (x == 0.0)
        return sign;
    return (uint16_t)(sign | round_magnitude(fabs(x), mbits, bias, ebits));
}

uint16_t orc_f16_rne(double x)  { return round_to_small_float(x, 10, 15, 5, 0x7E00); }
uint16_t orc_bf16_rne(double x) { return round_to_small_float(x, 7, 127, 8, 0x7FC0); }

static double small_float_value(uint16_t h, int mbits, int bias, int ebits)
{
    int sign = (h >> (mbits + ebits)) & 1;
    int e = (h >> mbits) & ((1 << ebits) - 1);
    int m = h & ((1 << mbits) - 1);
    double v;
    if (e == (1 << ebits) - 1)
        v = m ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)m, 1 - bias - mbits);
    else
        v = ldexp((double)(m | (1 << mbits)), e - bias - mbits);
    return sign ? -v : v;
}

double orc_f16_to_f64(uint16_t h)  { return small_float_value(h, 10, 15, 5); }
double orc_bf16_to_f64(uint16_t h) { return small_float_value(h, 7, 127, 8); }

void orc_f16_rne_array(const double *x, long n, uint16_t *out)
{ for (long i = 0; i < n; i++) out[i] = orc_f16_rne(x[i]); }
void orc_bf16_rne_array(const double *x, long n, uint16_t *out)
{ for (long i = 0; i < n; i++) out[i] = orc_bf16_rne(x[i]); }

/* ------------------------------------------------------------------------ */
/* transform: Y[n][d] = X[n][d] . M[d][d]                                    */
/* ------------------------------------------------------------------------ */
void orc_transform(const double *X, const double *M, long n, int d, double *Y)
{
    for (long t = 0; t < n; t++)
        for (int j = 0; j < d; j++) {
            double acc = 0.0;
            for (int c = 0; c < d; c++)
                acc = fma(X[t * d + c], M[(long)c * d + j], acc);
            Y[t * d + j] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* quantizer for one (token, group)                                          */
/* ------------------------------------------------------------------------ */
/* levels = 2^bits - 1.  Writes the fp16 bit patterns of scale and zero and
 * one code per value.                                                       */
/* With a clipping ratio `clip` (0 < clip <= 1) the grid spans
 * [clip*min, clip*max] instead of [min, max]; values outside it take the end
 * codes.  clip = 1 is the plain min/max grid (the products are exact).       */
void orc_quantize_group_clip(const double *x, int len, int levels, double clip,
                             uint16_t *s16, uint16_t *z16, uint8_t *codes)
{
    double lo = x[0], hi = x[0];
    for (int i = 1; i < len; i++) {
        if (x[i] < lo) lo = x[i];
        if (x[i] > hi) hi = x[i];
    }
    lo = clip * lo;
    hi = clip * hi;
    uint16_t zb = orc_f16_rne(lo);
    uint16_t sb = orc_f16_rne((hi - lo) / (double)levels);
    double z = orc_f16_to_f64(zb), s = orc_f16_to_f64(sb);
    for (int i = 0; i < len; i++) {
        int c = 0;
        if (s != 0.0) {
            double r = rint((x[i] - z) / s);
            if (r < 0.0) r = 0.0;
            if (r > (double)levels) r = (double)levels;
            c = (int)r;
        }
        codes[i] = (uint8_t)c;
    }
    *s16 = sb;
    *z16 = zb;
}
void orc_quantize_group(const double *x, int len, int levels,
                        uint16_t *s16, uint16_t *z16, uint8_t *codes)
{
    orc_quantize_group_clip(x, len, levels, 1.0, s16, z16, codes);
}

/* ------------------------------------------------------------------------ */
/* page layout (one page = 128 tokens of one (batch, KV head))               */
/*                                                                           */
/*   rowbytes R = 128 * bits / 8; quantization groups of `group` channels    */
/*   (32: four groups; 128: the pages' one grid per token), ng = 128/group   */
/*   [0, 128R)            key codes, row r = channel r (row 0 unused, zero)  */
/*   [128R, 256R)         value codes, row r = channel r                     */
/*   [256R, 256R+256)     channel 0 of K' as bf16, one per token             */
/*   next 512*ng bytes    key metadata: 128*ng words {fp16 scale, fp16 zero}  */
/*   next 512*ng bytes    value metadata, same shape                         */
/*   metadata word of token t, group g: 128g + 4*sw(g, t/4) + t%4 with       */
/*   sw(g, c) = c XOR ((c/8) XOR 4*(g%2)) (chunks of 4 tokens XOR-permuted    */
/*   within blocks of 8 chunks).                                             */
/*   key group g covers channels max(1, g*group) .. (g+1)*group - 1 (channel */
/*   0 is kept in bf16); value group g covers g*group .. (g+1)*group - 1.    */
/*   codes: token t of the page sits in byte t*bits/8 of its row, at bit     */
/*   (t mod (8/bits))*bits (least significant first).                        */
/* ------------------------------------------------------------------------ */
long orc_page_bytes_g(int bits, int group)
{
    return 256L * (ORC_T * bits / 8) + 256 + 2L * 512 * (ORC_D / group);
}
long orc_page_bytes(int bits) { return orc_page_bytes_g(bits, ORC_G); }

static uint8_t *page_ptr(uint8_t *unit, int bits, int group, long page)
{ return unit + page * orc_page_bytes_g(bits, group); }

static void put_code(uint8_t *row, int bits, int t, int code)
{
    int per = 8 / bits;
    int sh = (t % per) * bits;
    uint8_t mask = (uint8_t)(((1 << bits) - 1) << sh);
    row[t / per] = (uint8_t)((row[t / per] & ~mask) | ((code << sh) & mask));
}

static int get_code(const uint8_t *row, int bits, int t)
{
    int per = 8 / bits;
    return (row[t / per] >> ((t % per) * bits)) & ((1 << bits) - 1);
}

static int meta_word_index(int g, int t)
{
    int chunk = t / 4;
    int perm = chunk ^ ((chunk / 8) ^ (4 * (g % 2)));
    return 128 * g + 4 * perm + t % 4;
}

static void put_u16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)(v & 0xFF); p[1] = (uint8_t)(v >> 8); }
static uint16_t get_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* Quantize n tokens (K' already transformed, V as given -- rotated or not;
 * both [n][128]) and write them at token positions pos0 .. pos0+n-1 of one
 * (batch, KV head) unit of pages with groups of `group` channels; the value
 * grids use the clipping ratio vclip, the key grids none.  Other tokens' bits
 * are left as they are.                                                     */
void orc_append_unit_c(uint8_t *unit, int bits, int group, double vclip, long pos0, long n,
                       const double *Kp, const double *V)
{
    const int R = ORC_T * bits / 8;
    const int levels = (1 << bits) - 1;
    const int ng = ORC_D / group;
    uint8_t codes[ORC_D];
    for (long i = 0; i < n; i++) {
        long pos = pos0 + i;
        uint8_t *pg = page_ptr(unit, bits, group, pos / ORC_T);
        int t = (int)(pos % ORC_T);
        const double *k = Kp + i * ORC_D;
        const double *v = V + i * ORC_D;
        uint8_t *kcodes = pg, *vcodes = pg + 128 * R;
        uint8_t *ch0 = pg + 256 * R, *kmeta = ch0 + 256, *vmeta = kmeta + 512 * ng;
        /* channel 0 of the key: bf16, not in any range */
        put_u16(ch0 + 2 * t, orc_bf16_rne(k[0]));
        for (int g = 0; g < ng; g++) {
            uint16_t s16, z16;
            /* keys: group 0 starts at channel 1 */
            int c0 = (g == 0) ? 1 : g * group;
            int len = (g + 1) * group - c0;
            orc_quantize_group(k + c0, len, levels, &s16, &z16, codes);
            for (int c = 0; c < len; c++)
                put_code(kcodes + (long)(c0 + c) * R, bits, t, codes[c]);
            put_u16(kmeta + 4 * meta_word_index(g, t), s16);
            put_u16(kmeta + 4 * meta_word_index(g, t) + 2, z16);
            /* values: group g covers channels g*group .. (g+1)*group-1 */
            orc_quantize_group_clip(v + g * group, group, levels, vclip, &s16, &z16, codes);
            for (int c = 0; c < group; c++)
                put_code(vcodes + (long)(g * group + c) * R, bits, t, codes[c]);
            put_u16(vmeta + 4 * meta_word_index(g, t), s16);
            put_u16(vmeta + 4 * meta_word_index(g, t) + 2, z16);
        }
    }
}
void orc_append_unit_g(uint8_t *unit, int bits, int group, long pos0, long n,
                       const double *Kp, const double *V)
{
    orc_append_unit_c(unit, bits, group, 1.0, pos0, n, Kp, V);
}
void orc_append_unit(uint8_t *unit, int bits, long pos0, long n, const double *Kp, const double *V)
{
    orc_append_unit_g(unit, bits, ORC_G, pos0, n, Kp, V);
}

/* Dequantize tokens 0 .. n-1 of one unit: Khat[n][128], Vhat[n][128].       */
void orc_dequant_unit_g(const uint8_t *unit, int bits, int group, long n, double *Khat, double *Vhat)
{
    const int R = ORC_T * bits / 8;
    const int ng = ORC_D / group;
    for (long pos = 0; pos < n; pos++) {
        const uint8_t *pg = page_ptr((uint8_t *)unit, bits, group, pos / ORC_T);
        int t = (int)(pos % ORC_T);
        const uint8_t *kcodes = pg, *vcodes = pg + 128 * R;
        const uint8_t *ch0 = pg + 256 * R, *kmeta = ch0 + 256, *vmeta = kmeta + 512 * ng;
        double *kh = Khat + pos * ORC_D, *vh = Vhat + pos * ORC_D;
        kh[0] = orc_bf16_to_f64(get_u16(ch0 + 2 * t));
        for (int c = 1; c < ORC_D; c++) {
            int g = c / group;
            double s = orc_f16_to_f64(get_u16(kmeta + 4 * meta_word_index(g, t)));
            double z = orc_f16_to_f64(get_u16(kmeta + 4 * meta_word_index(g, t) + 2));
            kh[c] = s * get_code(kcodes + (long)c * R, bits, t) + z;
        }
        for (int c = 0; c < ORC_D; c++) {
            int g = c / group;
            double s = orc_f16_to_f64(get_u16(vmeta + 4 * meta_word_index(g, t)));
            double z = orc_f16_to_f64(get_u16(vmeta + 4 * meta_word_index(g, t) + 2));
            vh[c] = s * get_code(vcodes + (long)c * R, bits, t) + z;
        }
    }
}
void orc_dequant_unit(const uint8_t *unit, int bits, long n, double *Khat, double *Vhat)
{
    orc_dequant_unit_g(unit, bits, ORC_G, n, Khat, Vhat);
}

/* ------------------------------------------------------------------------ */
/* channel selection                                                         */
/* ------------------------------------------------------------------------ */
/* k = ceil((1 - s) d), with a 1e-9 guard so exact products do not round up. */
int orc_num_selected(float sparsity, int d)
{
    return (int)ceil((1.0 - (double)sparsity) * d - 1e-9);
}

static const double *g_sel_e2;
static int cmp_energy_desc(const void *a, const void *b)
{
    int i = *(const int *)a, j = *(const int *)b;
    double ei = g_sel_e2[i], ej = g_sel_e2[j];
    if (ei > ej) return -1;
    if (ei < ej) return 1;
    return (i < j) ? -1 : (i > j);
}
static int cmp_int_asc(const void *a, const void *b)
{
    int i = *(const int *)a, j = *(const int *)b;
    return (i > j) - (i < j);
}

/* qp: [g][d] transformed queries of the heads sharing one KV head.
 * e2 (out, [d]): pooled energy, sum over h ascending as an fma chain.
 * idx (out, [k]): channel 0, then the k-1 channels of 1..d-1 with the
 * largest e2 (ties to the lower index), all sorted ascending.              */
/* With a diagonal refinement (delta != NULL: delta[j] > 0), qp holds the
 * final queries q A0 D and the energies are those of the base queries
 * q A0 = qp D^{-1}: u = qp[h][j] / delta[j] (one rounded division), e2[j] the
 * fma chain of u*u over h.  delta == NULL: u = qp[h][j].                    */
void orc_select_scaled(const double *qp, int g, int d, int k, const double *delta,
                       double *e2, int32_t *idx)
{
    int *order = (int *)malloc(sizeof(int) * d);
    for (int j = 0; j < d; j++) {
        double e = 0.0;
        for (int h = 0; h < g; h++) {
            double u = delta ? qp[h * d + j] / delta[j] : qp[h * d + j];
            e = fma(u, u, e);
        }
        e2[j] = e;
    }
    for (int j = 1; j < d; j++) order[j - 1] = j;
    g_sel_e2 = e2;
    qsort(order, d - 1, sizeof(int), cmp_energy_desc);
    int *sel = (int *)malloc(sizeof(int) * k);
    sel[0] = 0;
    for (int i = 1; i < k; i++) sel[i] = order[i - 1];
    qsort(sel, k, sizeof(int), cmp_int_asc);
    for (int i = 0; i < k; i++) idx[i] = sel[i];
    free(sel);
    free(order);
}
void orc_select(const double *qp, int g, int d, int k, double *e2, int32_t *idx)
{
    orc_select_scaled(qp, g, d, k, NULL, e2, idx);
}

/* ------------------------------------------------------------------------ */
/* attention                                                                 */
/* ------------------------------------------------------------------------ */
/* One softmax over all n tokens per query head, scores over the retained
 * channels idx[0..k-1] only, scaled by 1/sqrt(d) with the full d.
 * qp: [g][d], Khat, Vhat: [n][d], out: [g][d].                              */
void orc_decode_dense(const double *Khat, const double *Vhat, long n,
                      const double *qp, int g, int d,
                      const int32_t *idx, int k, double *out)
{
    double *sc = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
    double inv = 1.0 / sqrt((double)d);
    for (int h = 0; h < g; h++) {
        const double *q = qp + (long)h * d;
        double mx = -INFINITY;
        for (long t = 0; t < n; t++) {
            double s = 0.0;
            for (int i = 0; i < k; i++)
                s += q[idx[i]] * Khat[t * d + idx[i]];
            sc[t] = s * inv;
            if (sc[t] > mx) mx = sc[t];
        }
        double l = 0.0;
        double *o = out + (long)h * d;
        for (int c = 0; c < d; c++) o[c] = 0.0;
        for (long t = 0; t < n; t++) {
            double p = exp(sc[t] - mx);
            l += p;
            for (int c = 0; c < d; c++) o[c] += p * Vhat[t * d + c];
        }
        for (int c = 0; c < d; c++) o[c] = (n > 0) ? o[c] / l : 0.0;
    }
    free(sc);
}

/* softmax(q K^T / sqrt(d)) V for g query rows against n keys/values.        */
void orc_attention(const double *q, const double *K, const double *V, long n,
                   int g, int d, double *out)
{
    int32_t *all = (int32_t *)malloc(sizeof(int32_t) * d);
    for (int j = 0; j < d; j++) all[j] = j;
    orc_decode_dense(K, V, n, q, g, d, all, d, out);
    free(all);
}

/* ------------------------------------------------------------------------ */
/* bucket-relative RoPE                                                      */
/* ------------------------------------------------------------------------ */
/* Remove the anchor rotation of a bucket from rows of post-RoPE vectors:
 * channel i (< d/2) is paired with channel i + d/2 (the rotate-half layout)
 * and the pair is rotated by the angle -a*theta_i, given as cs[i] =
 * {cos(a theta_i), sin(a theta_i)}:
 *   y_i       = x_i cos + x_{i+d/2} sin
 *   y_{i+d/2} = x_{i+d/2} cos - x_i sin
 * each product rounded, then the sum or difference (no fused operations).   */
void orc_rope_unanchor(const double *X, long n, int d, const double *cs, double *Y)
{
    const int hd = d / 2;
    for (long t = 0; t < n; t++) {
        const double *x = X + t * d;
        double *y = Y + t * d;
        for (int i = 0; i < hd; i++) {
            double c = cs[2 * i], sn = cs[2 * i + 1];
            double a = x[i], b = x[i + hd];
            double p1 = a * c, p2 = b * sn, p3 = b * c, p4 = a * sn;
            y[i] = p1 + p2;
            y[i + hd] = p3 - p4;
        }
    }
}

/* Decode over buckets of w tokens: token t uses the queries and the channel
 * list of its bucket t / w (qp: [nb][g][d], idx: [nb][k]); one softmax over
 * all n tokens per query head, 1/sqrt(d) scaling.  out: [g][d].            */
void orc_decode_buckets(const double *Khat, const double *Vhat, long n, const double *qp, int g, int d,
                        const int32_t *idx, int k, long w, double *out)
{
    double *sc = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
    double inv = 1.0 / sqrt((double)d);
    for (int h = 0; h < g; h++) {
        double mx = -INFINITY;
        for (long t = 0; t < n; t++) {
            long b = t / w;
            const double *q = qp + (b * g + h) * (long)d;
            const int32_t *ix = idx + b * k;
            double s = 0.0;
            for (int i = 0; i < k; i++)
                s += q[ix[i]] * Khat[t * d + ix[i]];
            sc[t] = s * inv;
            if (sc[t] > mx) mx = sc[t];
        }
        double l = 0.0;
        double *o = out + (long)h * d;
        for (int c = 0; c < d; c++) o[c] = 0.0;
        for (long t = 0; t < n; t++) {
            double p = exp(sc[t] - mx);
            l += p;
            for (int c = 0; c < d; c++) o[c] += p * Vhat[t * d + c];
        }
        for (int c = 0; c < d; c++) o[c] = (n > 0) ? o[c] / l : 0.0;
    }
    free(sc);
}

/* ------------------------------------------------------------------------ */
/* protected BF16 tier                                                       */
/* ------------------------------------------------------------------------ */
/* Positions below n_sink keep slot pos; later positions use a ring of
 * n_recent slots after them.  -1: the position has no slot.                 */
long orc_protected_slot(long pos, int n_sink, int n_recent)
{
    if (pos < n_sink) return pos;
    if (n_recent <= 0) return -1;
    return n_sink + pos % n_recent;
}

/* Protected set of a sequence of length len: [0, sink_end) and
 * [recent_start, len).                                                      */
static void protected_bounds(long len, int n_sink, int n_recent, long *sink_end, long *recent_start)
{
    long se = len < n_sink ? len : n_sink;
    long rs = len - n_recent;
    if (rs < se) rs = se;
    *sink_end = se;
    *recent_start = rs;
}

int orc_is_protected(long pos, long len, int n_sink, int n_recent)
{
    long se, rs;
    protected_bounds(len, n_sink, n_recent, &se, &rs);
    return pos < se || (pos >= rs && pos < len);
}

/* Store tokens pos0 .. pos0+n-1 (K' transformed, V as given; [n][128]) of a
 * sequence whose length becomes len_after: a token gets its slot when it is
 * a sink token or one of the last n_recent tokens; each slot holds 128 BF16
 * key values then 128 BF16 value values.                                    */
void orc_protect_store(uint16_t *slots, int n_sink, int n_recent, long pos0, long n,
                       long len_after, const double *Kp, const double *V)
{
    for (long i = 0; i < n; i++) {
        long pos = pos0 + i;
        if (!(pos < n_sink || (n_recent > 0 && pos >= len_after - n_recent))) continue;
        long slot = orc_protected_slot(pos, n_sink, n_recent);
        uint16_t *dst = slots + slot * 2 * ORC_D;
        for (int c = 0; c < ORC_D; c++) dst[c] = orc_bf16_rne(Kp[i * ORC_D + c]);
        for (int c = 0; c < ORC_D; c++) dst[ORC_D + c] = orc_bf16_rne(V[i * ORC_D + c]);
    }
}

/* Replace the rows of protected positions of a dequantized cache (Khat,
 * Vhat: [len][128]) by their BF16 values from the slots.                    */
void orc_protect_dequant(const uint16_t *slots, int n_sink, int n_recent, long len,
                         double *Khat, double *Vhat)
{
    for (long pos = 0; pos < len; pos++) {
        if (!orc_is_protected(pos, len, n_sink, n_recent)) continue;
        const uint16_t *src = slots + orc_protected_slot(pos, n_sink, n_recent) * 2 * ORC_D;
        for (int c = 0; c < ORC_D; c++) {
            Khat[pos * ORC_D + c] = orc_bf16_to_f64(src[c]);
            Vhat[pos * ORC_D + c] = orc_bf16_to_f64(src[ORC_D + c]);
        }
    }
}
