/*
 * oracle.c -- plain, slow CPU oracle (fp64) for batch-1 MoE decode over MXFP4
 * experts and the online-FP8 LM head.  TEST INFRASTRUCTURE ONLY: see oracle.h
 * for the sources each function follows and the readings taken where the
 * pages are silent.  Nothing here is shared with the CUDA library.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (x86-64 SSE
 * arithmetic, so float operations round once to binary32, as IEEE 754 says).
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scalar format decoders: the closed forms of the format specifications.   */
/* ------------------------------------------------------------------------ */

double orc_bf16_to_double(uint16_t bits)
{
    /* bf16 is the upper half of an IEEE binary32. */
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double orc_e2m1_to_double(unsigned code)
{
    /* OCP MX v1.0 FP4 E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa
     * bit.  Normal (E > 0): 2^(E-1) * (1 + M/2).  Subnormal (E = 0): M/2.   */
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0u) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

double orc_e8m0_to_double(unsigned code)
{
    /* OCP MX v1.0 E8M0 scale: unsigned exponent, bias 127; 0xFF is NaN. */
    if (code == 255u)
        return NAN;
    return ldexp(1.0, (int)code - 127);
}

double orc_e4m3_to_double(unsigned code)
{
    /* OFP8 E4M3: bias 7; normal 2^(E-7) * (1 + M/8); subnormal 2^-6 * M/8;
     * S.1111.111 is NaN; there are no infinities.                          */
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    if (e == 15u && m == 7u)
        return NAN;
    double mag = (e == 0u) ? ldexp((double)m, -9) : ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* Decode tables for the inner loops, filled once from the closed forms above. */
static double g_e2m1[16];
static double g_e8m0[256];
static double g_e4m3[256];

__attribute__((constructor)) static void orc_fill_tables(void)
{
    for (unsigned c = 0; c < 16u; ++c)
        g_e2m1[c] = orc_e2m1_to_double(c);
    for (unsigned c = 0; c < 256u; ++c) {
        g_e8m0[c] = orc_e8m0_to_double(c);
        g_e4m3[c] = orc_e4m3_to_double(c);
    }
}

/* ------------------------------------------------------------------------ */
/* Scalar encoders.                                                          */
/* ------------------------------------------------------------------------ */

unsigned orc_e2m1_encode(double v)
{
    /* Nearest of the eight E2M1 magnitudes; on a tie the code whose mantissa
     * bit is 0 wins (round half to even).  Values past 6 land on 6, the
     * nearest magnitude, which is the saturating conversion.                */
    double a = fabs(v);
    unsigned best = 0u;
    double best_err = INFINITY;
    for (unsigned c = 0; c < 8u; ++c) {
        double err = fabs(a - orc_e2m1_to_double(c));
        if (err < best_err || (err == best_err && (c & 1u) == 0u)) {
            best = c;
            best_err = err;
        }
    }
    return best | (signbit(v) ? 8u : 0u);
}

unsigned orc_e4m3_encode_satfinite(double v)
{
    unsigned sign = signbit(v) ? 0x80u : 0u;
    double a = fabs(v);
    unsigned mag;
    if (a >= 448.0) {
        mag = 0x7Eu; /* satfinite: the largest finite magnitude, 448 */
    } else if (a < ldexp(1.0, -6)) {
        /* Subnormal range: multiples of 2^-9.  A result of 8 is 2^-6, whose
         * code 0x08 is the smallest normal, so the code is the count itself. */
        mag = (unsigned)nearbyint(ldexp(a, 9));
    } else {
        int e;
        double f = frexp(a, &e);             /* a = f * 2^e, f in [0.5, 1)   */
        double t = nearbyint(f * 16.0);      /* 1.mmm scaled by 8: [8, 16]   */
        int E = (e - 1) + 7;                 /* biased exponent              */
        if (t == 16.0) {                     /* rounded up to the next binade */
            t = 8.0;
            E += 1;
        }
        mag = ((unsigned)E << 3) | ((unsigned)t - 8u);
    }
    return sign | mag;
}

uint16_t orc_double_to_bf16(double v)
{
    /* One rounding from the exact double to 8 significant bits, ties to even.
     * Valid for values in the normal bf16 range (and zero).                 */
    if (v == 0.0)
        return signbit(v) ? 0x8000u : 0u;
    int e;
    double f = frexp(fabs(v), &e);           /* |v| = f * 2^e, f in [0.5, 1) */
    double t = nearbyint(ldexp(f, 8));       /* [128, 256]                    */
    float r = (float)ldexp(t, e - 8);        /* exact: 8 significant bits     */
    uint32_t u;
    memcpy(&u, &r, sizeof u);
    uint16_t b = (uint16_t)(u >> 16);
    return signbit(v) ? (uint16_t)(b | 0x8000u) : b;
}

/* ------------------------------------------------------------------------ */
/* Load-time quantisers.                                                     */
/* ------------------------------------------------------------------------ */

void orc_mxfp4_quantize(int64_t rows, int64_t K, const uint16_t* w_bf16,
                        uint8_t* data, uint8_t* scales)
{
    /* OCP MX v1.0 sec. 6.3: shared scale X = 2^(floor(log2(amax)) - emax_elem),
     * emax_elem = 2 for E2M1; each element is V/X converted to E2M1.       */
    const int64_t nb = K / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint16_t* blk = w_bf16 + r * K + b * 32;
            uint8_t* d = data + r * (K / 2) + b * 16;
            double amax = 0.0;
            int finite = 1;
            for (int i = 0; i < 32; ++i) {
                double v = orc_bf16_to_double(blk[i]);
                if (!isfinite(v))
                    finite = 0;
                else if (fabs(v) > amax)
                    amax = fabs(v);
            }
            if (!finite) {
                scales[r * nb + b] = 0xFFu; /* the block's scale is NaN */
                memset(d, 0, 16);
                continue;
            }
            int xexp;
            if (amax == 0.0) {
                xexp = -127;
            } else {
                int e;
                (void)frexp(amax, &e);       /* floor(log2(amax)) = e - 1 */
                xexp = (e - 1) - 2;
            }
            if (xexp < -127)
                xexp = -127;
            if (xexp > 127)
                xexp = 127;
            scales[r * nb + b] = (uint8_t)(xexp + 127);
            for (int i = 0; i < 32; i += 2) {
                unsigned lo = orc_e2m1_encode(ldexp(orc_bf16_to_double(blk[i]), -xexp));
                unsigned hi = orc_e2m1_encode(ldexp(orc_bf16_to_double(blk[i + 1]), -xexp));
                d[i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

double orc_mxfp4_element(int64_t K, const uint8_t* data, const uint8_t* scales,
                         int64_t r, int64_t j)
{
    uint8_t byte = data[r * (K / 2) + j / 2];
    unsigned code = (j & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 15u);
    return g_e2m1[code] * g_e8m0[scales[r * (K / 32) + j / 32]];
}

void orc_fp8_rowquant(int64_t V, int64_t H, const uint16_t* w_bf16, uint8_t* q, float* s)
{
    for (int64_t v = 0; v < V; ++v) {
        const uint16_t* row = w_bf16 + v * H;
        float amax = 0.0f;
        for (int64_t j = 0; j < H; ++j) {
            float a = fabsf((float)orc_bf16_to_double(row[j]));
            if (a > amax)
                amax = a;
        }
        float sv = (amax == 0.0f) ? 1.0f : amax / 448.0f; /* binary32 division */
        s[v] = sv;
        for (int64_t j = 0; j < H; ++j) {
            float t = (float)orc_bf16_to_double(row[j]) / sv; /* binary32 division */
            q[v * H + j] = (uint8_t)orc_e4m3_encode_satfinite((double)t);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Router, experts, LM head.                                                 */
/* ------------------------------------------------------------------------ */

void orc_topk(int64_t n, const double* v, int k, int32_t* ids, double* vals)
{
    unsigned char* taken = (unsigned char*)calloc((size_t)n, 1);
    for (int i = 0; i < k; ++i) {
        int64_t best = -1;
        for (int64_t j = 0; j < n; ++j) {
            if (taken[j])
                continue;
            if (best < 0 || v[j] > v[best]) /* strict: the lower index keeps a tie */
                best = j;
        }
        taken[best] = 1;
        ids[i] = (int32_t)best;
        vals[i] = v[best];
    }
    free(taken);
}

void orc_router(int M, int E, int H, int k, const uint16_t* x_bf16,
                const float* Wr, const float* bias,
                double* logits, int32_t* ids, double* w)
{
    double* sel = (double*)malloc(sizeof(double) * (size_t)k);
    for (int m = 0; m < M; ++m) {
        double* lg = logits + (int64_t)m * E;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < H; ++j)
                acc += orc_bf16_to_double(x_bf16[(int64_t)m * H + j]) * (double)Wr[(int64_t)e * H + j];
            if (bias)
                acc += (double)bias[e];
            lg[e] = acc;
        }
        orc_topk(E, lg, k, ids + (int64_t)m * k, sel);
        /* softmax over all E logits, renormalised over the k selected ones:
         * the full-softmax denominator cancels, leaving a softmax over sel. */
        double z = 0.0;
        for (int i = 0; i < k; ++i)
            z += exp(sel[i] - sel[0]);
        for (int i = 0; i < k; ++i)
            w[(int64_t)m * k + i] = exp(sel[i] - sel[0]) / z;
    }
    free(sel);
}

void orc_expert_mlp(int H, int I, const uint16_t* x_bf16,
                    const uint8_t* gate_d, const uint8_t* gate_s,
                    const uint8_t* up_d, const uint8_t* up_s,
                    const uint8_t* down_d, const uint8_t* down_s,
                    double* out, double* h_out)
{
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    for (int r = 0; r < I; ++r) {
        double g = 0.0, u = 0.0;
        for (int j = 0; j < H; ++j) {
            double xj = orc_bf16_to_double(x_bf16[j]);
            g += orc_mxfp4_element(H, gate_d, gate_s, r, j) * xj;
            u += orc_mxfp4_element(H, up_d, up_s, r, j) * xj;
        }
        h[r] = g / (1.0 + exp(-g)) * u; /* silu(g) * u, silu(g) = g * sigmoid(g) */
        if (h_out)
            h_out[r] = h[r];
    }
    for (int i = 0; i < H; ++i) {
        double acc = 0.0;
        for (int r = 0; r < I; ++r)
            acc += orc_mxfp4_element(I, down_d, down_s, i, r) * h[r];
        out[i] = acc;
    }
    free(h);
}

void orc_moe_layer(int M, int H, int I, int k, const uint16_t* x_bf16,
                   const int32_t* ids, const double* w,
                   const uint8_t* gate_d, const uint8_t* gate_s,
                   const uint8_t* up_d, const uint8_t* up_s,
                   const uint8_t* down_d, const uint8_t* down_s,
                   const uint8_t* sh_gate_d, const uint8_t* sh_gate_s,
                   const uint8_t* sh_up_d, const uint8_t* sh_up_s,
                   const uint8_t* sh_down_d, const uint8_t* sh_down_s,
                   double* y)
{
    const int64_t gu_d = (int64_t)I * H / 2, gu_s = (int64_t)I * H / 32; /* per expert */
    const int64_t dn_d = (int64_t)H * I / 2, dn_s = (int64_t)H * I / 32;
    double* out = (double*)malloc(sizeof(double) * (size_t)H);
    for (int m = 0; m < M; ++m) {
        const uint16_t* xm = x_bf16 + (int64_t)m * H;
        double* ym = y + (int64_t)m * H;
        for (int i = 0; i < H; ++i)
            ym[i] = 0.0;
        for (int i = 0; i < k; ++i) {
            int64_t e = ids[(int64_t)m * k + i];
            orc_expert_mlp(H, I, xm, gate_d + e * gu_d, gate_s + e * gu_s,
                           up_d + e * gu_d, up_s + e * gu_s,
                           down_d + e * dn_d, down_s + e * dn_s, out, NULL);
            for (int j = 0; j < H; ++j)
                ym[j] += w[(int64_t)m * k + i] * out[j];
        }
        /* the shared expert runs for every token, with weight 1 */
        orc_expert_mlp(H, I, xm, sh_gate_d, sh_gate_s, sh_up_d, sh_up_s,
                       sh_down_d, sh_down_s, out, NULL);
        for (int j = 0; j < H; ++j)
            ym[j] += out[j];
    }
    free(out);
}

void orc_lmhead_fp8(int64_t V, int64_t H, int M, const uint16_t* x_bf16,
                    const uint8_t* q, const float* s,
                    double* logits, double* abssum)
{
    double* xd = (double*)malloc(sizeof(double) * (size_t)H);
    for (int m = 0; m < M; ++m) {
        for (int64_t j = 0; j < H; ++j)
            xd[j] = orc_bf16_to_double(x_bf16[(int64_t)m * H + j]);
        for (int64_t v = 0; v < V; ++v) {
            const uint8_t* row = q + v * H;
            double acc = 0.0, aacc = 0.0;
            for (int64_t j = 0; j < H; ++j) {
                double t = g_e4m3[row[j]] * xd[j];
                acc += t;
                aacc += fabs(t);
            }
            logits[(int64_t)m * V + v] = (double)s[v] * acc;
            if (abssum)
                abssum[(int64_t)m * V + v] = fabs((double)s[v]) * aacc;
        }
    }
    free(xd);
}

void orc_lmhead_bf16(int64_t V, int64_t H, int M, const uint16_t* x_bf16,
                     const uint16_t* w_bf16, double* logits)
{
    double* xd = (double*)malloc(sizeof(double) * (size_t)H);
    for (int m = 0; m < M; ++m) {
        for (int64_t j = 0; j < H; ++j)
            xd[j] = orc_bf16_to_double(x_bf16[(int64_t)m * H + j]);
        for (int64_t v = 0; v < V; ++v) {
            double acc = 0.0;
            for (int64_t j = 0; j < H; ++j)
                acc += orc_bf16_to_double(w_bf16[v * H + j]) * xd[j];
            logits[(int64_t)m * V + v] = acc;
        }
    }
    free(xd);
}

void orc_rmsnorm_bf16(int H, const double* y, double eps, uint16_t* out)
{
    double ss = 0.0;
    for (int j = 0; j < H; ++j)
        ss += y[j] * y[j];
    double rms = sqrt(ss / (double)H + eps);
    for (int j = 0; j < H; ++j)
        out[j] = orc_double_to_bf16(y[j] / rms);
}

/* ---- sampled decode and speculative verify ---- */

int orc_sample_topk(int k, const double* vals, double temperature, double top_p, double u)
{
    double* p = (double*)malloc(sizeof(double) * (size_t)k);
    double total = 0.0;
    for (int i = 0; i < k; ++i) {
        p[i] = exp((vals[i] - vals[0]) / temperature);
        total += p[i];
    }
    /* nucleus: the smallest prefix whose mass reaches top_p of the total */
    int n = 0;
    double before = 0.0;
    while (n < k && before < top_p * total) {
        before += p[n];
        ++n;
    }
    double kept = 0.0;
    for (int i = 0; i < n; ++i)
        kept += p[i];
    const double r = u * kept;
    int pick = n - 1;
    double cum = 0.0;
    for (int i = 0; i < n; ++i) {
        cum += p[i];
        if (cum > r) {
            pick = i;
            break;
        }
    }
    free(p);
    return pick;
}

int orc_mtp_accept(int D, const int32_t* draft, const int32_t* verify, int32_t* emitted)
{
    int a = 0;
    while (a < D && draft[a] == verify[a]) {
        emitted[a] = draft[a];
        ++a;
    }
    emitted[a] = verify[a];
    return a + 1;
}
