/*
 * oracle.h -- plain, slow CPU oracle for batch-1 MoE decode (MXFP4 experts) and
 * the online-FP8 LM head.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library under moe_decode_gemv_b200/;
 * it has its own format decoders, written from the public format
 * specifications, and accumulates in fp64.
 *
 * Sources (the web pages describe the method; the formats come from public specs):
 *  - "NVIDIA shows 3 ways to speed up MoE inference on DGX Spark" (ncijnetwork.com),
 *    sections "Why is MoE decoding on DGX Spark memory-bound?" and
 *    "What are the 3 optimizations?": the two weight streams (MoE experts and
 *    the 157,184 x 2,560 LM head), load-time FP8 of the head only.
 *  - saipien.org analysis essay, section "Why one user waits on weights":
 *    8 of 512 routed experts plus one shared expert that always runs.
 *  - OCP Microscaling Formats (MX) Specification v1.0: E2M1 elements (sec. 5.3.3),
 *    E8M0 shared scale (sec. 5.4), block size 32, conversion rule (sec. 6.3).
 *  - OCP 8-bit Floating Point Specification (OFP8) rev 1.0: E4M3 (bias 7,
 *    max 448, no infinities, S.1111.111 is NaN).
 *
 * Readings taken where the pages are silent:
 *  - routing is softmax over the routed logits, top-k, renormalised over the
 *    selected k (equivalently a softmax over the k selected logits);
 *    ties go to the lower expert id;
 *  - routed experts are SwiGLU MLPs: h = silu(g) * u, g = Wg x, u = Wu x,
 *    out = Wd h; the shared expert has the same form and weight 1;
 *  - FP8 head: per-row scale s = amax/448 in fp32, q = E4M3_RNE_satfinite(w/s)
 *    with the division in fp32; logit = s * sum(q * x);
 *  - top-k lists are sorted by value, descending; ties go to the lower index.
 *
 * Parity pins: every function here is checked by the -m "not gpu" tests
 * against closed forms, library routines, brute force or page facts.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- scalar format decoders (closed forms from the specs) ---- */
double orc_bf16_to_double(uint16_t bits);
double orc_e2m1_to_double(unsigned code);   /* code in [0,15]; bit 3 = sign            */
double orc_e8m0_to_double(unsigned code);   /* 2^(code-127); code 255 = NaN            */
double orc_e4m3_to_double(unsigned code);   /* OFP8 E4M3; 0x7F / 0xFF = NaN            */

/* ---- scalar encoders ---- */
/* Nearest E2M1 code to v (ties to even mantissa), saturating at +-6; sign bit
 * copied from v (so -0.0 and tiny negatives give code 8).                       */
unsigned orc_e2m1_encode(double v);
/* E4M3 round-to-nearest-even, saturating to +-448 (satfinite).  v finite.      */
unsigned orc_e4m3_encode_satfinite(double v);
/* RNE of a finite double to bf16 bits (single rounding, no double rounding).    */
uint16_t orc_double_to_bf16(double v);

/* ---- load-time quantisers ---- */
/* MXFP4 (OCP MX): per row, per 32-element block along K:
 *   X = 2^(floor(log2(amax)) - 2), exponent clamped to [-127, 127];
 *   scale code = exponent + 127; element code = orc_e2m1_encode(v / X).
 * Blocks holding Inf or NaN get scale code 0xFF and element codes 0.
 * data [rows][K/2]: element 2j in the low nibble of byte j; scales [rows][K/32].
 * K must be a multiple of 32.                                                    */
void orc_mxfp4_quantize(int64_t rows, int64_t K, const uint16_t* w_bf16,
                        uint8_t* data, uint8_t* scales);
/* Dequantise one MXFP4 element (row r, column j) of a [rows][K] matrix.          */
double orc_mxfp4_element(int64_t K, const uint8_t* data, const uint8_t* scales,
                         int64_t r, int64_t j);

/* FP8 row quantiser: s_v = fp32(amax_v / 448) (s_v = 1 when amax_v = 0),
 * q[v][j] = E4M3_RNE_satfinite(fp32(w[v][j] / s_v)).                            */
void orc_fp8_rowquant(int64_t V, int64_t H, const uint16_t* w_bf16,
                      uint8_t* q, float* s);

/* ---- router ---- */
/* logits[m][e] = sum_j x[m][j] * Wr[e][j] (+ bias[e] when bias != NULL), fp64.
 * ids[m][0..k): the k largest logits, descending, ties -> lower expert id.
 * w[m][i] = exp(l_i - l_max) / sum_{selected} exp(l_j - l_max).               */
void orc_router(int M, int E, int H, int k, const uint16_t* x_bf16,
                const float* Wr, const float* bias,
                double* logits, int32_t* ids, double* w);

/* ---- expert MLP ---- */
/* One token through one SwiGLU expert held as MXFP4 matrices:
 *   gate, up : [I][H] (data I*H/2 bytes, scales I*H/32 bytes)
 *   down     : [H][I]
 * h[I] = silu(g) * u with g = deq(gate) x, u = deq(up) x;  out[H] = deq(down) h.
 * h may be NULL.                                                                */
void orc_expert_mlp(int H, int I, const uint16_t* x_bf16,
                    const uint8_t* gate_d, const uint8_t* gate_s,
                    const uint8_t* up_d, const uint8_t* up_s,
                    const uint8_t* down_d, const uint8_t* down_s,
                    double* out, double* h);

/* MoE layer given routing: for each token m,
 *   y[m] = sum_i w[m][i] * expert_{ids[m][i]}(x[m]) + shared(x[m]).
 * Expert banks are stacked [E][rows][K/2] / [E][rows][K/32]; only the experts
 * named in ids are read.  The shared expert is a single expert (E = 1).        */
void orc_moe_layer(int M, int H, int I, int k, const uint16_t* x_bf16,
                   const int32_t* ids, const double* w,
                   const uint8_t* gate_d, const uint8_t* gate_s,
                   const uint8_t* up_d, const uint8_t* up_s,
                   const uint8_t* down_d, const uint8_t* down_s,
                   const uint8_t* sh_gate_d, const uint8_t* sh_gate_s,
                   const uint8_t* sh_up_d, const uint8_t* sh_up_s,
                   const uint8_t* sh_down_d, const uint8_t* sh_down_s,
                   double* y);

/* ---- LM head ---- */
/* logits[m][v] = s_v * sum_j e4m3(q[v][j]) * x[m][j]  (fp64).
 * abssum[m][v] = |s_v| * sum_j |e4m3(q[v][j]) * x[m][j]| (may be NULL): the
 * scale of the rounding error any fp32 evaluation of the row can make.        */
void orc_lmhead_fp8(int64_t V, int64_t H, int M, const uint16_t* x_bf16,
                    const uint8_t* q, const float* s,
                    double* logits, double* abssum);
/* logits[m][v] = sum_j w[v][j] * x[m][j] with bf16 weights (the comparator). */
void orc_lmhead_bf16(int64_t V, int64_t H, int M, const uint16_t* x_bf16,
                     const uint16_t* w_bf16, double* logits);
/* The k largest of v[0..n), sorted descending, ties -> lower index.            */
void orc_topk(int64_t n, const double* v, int k, int32_t* ids, double* vals);

/* ---- sampled decode and speculative verify ---- */
/* One draw from a sorted top-k list (the sampled workload of the ncijnetwork
 * summary, "What are the 3 optimizations?": temperature 0.6, top-p 0.95,
 * top-k 29).  With vals[0] >= vals[1] >= ...:
 *   p_i = exp((vals[i] - vals[0]) / temperature), i < k        (softmax up to a factor)
 *   keep the smallest prefix n whose mass reaches top_p:
 *        i is kept while (p_0 + ... + p_{i-1}) < top_p * (p_0 + ... + p_{k-1})
 *   return the first i < n with p_0 + ... + p_i > u * (p_0 + ... + p_{n-1}), u in [0, 1).    */
int orc_sample_topk(int k, const double* vals, double temperature, double top_p, double u);
/* Greedy acceptance of D draft tokens against the D+1 argmaxes of the verify
 * step (the saipien.org essay, "Draft three tokens, verify four"): draft i is
 * accepted while it equals verify i and every earlier draft was accepted.
 * emitted = the accepted drafts, then verify[accepted] (the verify step's own
 * next token); returns accepted + 1 (1 .. D+1).                                */
int orc_mtp_accept(int D, const int32_t* draft, const int32_t* verify, int32_t* emitted);

/* ---- between-layer op of the layer stack ---- */
/* out[j] = bf16_RNE( y[j] / sqrt(mean(y^2) + eps) )  (gain 1).                 */
void orc_rmsnorm_bf16(int H, const double* y, double eps, uint16_t* out);

#ifdef __cplusplus
}
#endif
#endif
