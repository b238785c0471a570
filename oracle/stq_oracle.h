/*
 * stq_oracle.h -- plain, single-threaded CPU oracle for the quantized
 * Delta-rule recurrent-state decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or execute this code: only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py use it.  It shares no code,
 * header, table or constant generator with the CUDA library.
 *
 * What it computes, and where the pages say so:
 *   - the state S in R^{d_k x d_v} per (request, head); fp32, 128 x 128 in the
 *     serving setting ("STEPQuant" landing page, Fig. 5 / Figure B2 caption:
 *     128x128 states; freedom251 post, "Memory and speed gains": 144 MiB FP32
 *     per request = 2,304 heads x 128 x 128 x 4 B);
 *   - key rows split into groups of different bit widths, dequantized as
 *     z_ij * r_i * c_j with a key-row scale r and a value-column scale c
 *     ("DAMP" card page, STEPQuant abstract; freedom251 post, "STEPQuant:
 *     precision can be allocated selectively");
 *   - the DAMP-style format: selected key channels in FP16, the rest INT8
 *     with stochastic rounding (freedom251 post, "DAMP: accuracy depends on
 *     the task");
 *   - the delta rule S <- S(I - k k^T) + v k^T in the d_v x d_k convention
 *     (dev.to post, "The state is a running sum, not a buffer"), here in the
 *     d_k x d_v convention with a decay gate alpha and a write strength beta:
 *       S' = A S + beta k (v - (A S)^T k)^T,  A = alpha I (GDN) or diag(alpha) (KDA),
 *       o  = S'^T q;
 *   - around the step: the per-window variant that requantizes once per
 *     window (LeapQuant abstract, paper-cards page), the prefill of a prompt
 *     with one requantization at its end (repeated prefill: DASC card), and
 *     the calibration's lifetime row weights (STEPQuant landing page,
 *     Figure B1).
 *
 * Conventions: stored row s (group order), natural key channel perm[s].
 * Codes of INT rows are signed integers z in [-qmax, qmax], qmax = 2^(b-1)-1.
 * Every function returns 0 on success and a negative value on bad arguments.
 */
#ifndef STQ_ORACLE_H
#define STQ_ORACLE_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_KIND_INT = 0, ORC_KIND_FP16 = 1, ORC_KIND_FP32 = 2 };

#define ORC_MAX_GROUPS 8

/* Row-group description.  Groups are listed widest first; their row counts
 * sum to d_k.  FP32 rows are an oracle-only kind (an unquantized state, used
 * to check the retrieval invariant); the packed byte layout does not hold
 * them. */
typedef struct {
    int d_k, d_v;
    int n_groups;
    int group_rows[ORC_MAX_GROUPS];
    int group_kind[ORC_MAX_GROUPS];
    int group_bits[ORC_MAX_GROUPS];
    int col_scales;   /* 1: per-column scale c_j; 0: c_j == 1 */
    int stochastic;   /* 1: stochastic rounding on INT rows; 0: round to nearest even */
    int gate_vector;  /* 1: alpha is a vector over key channels (KDA); 0: scalar (GDN) */
} orc_format;

/* An unpacked page.  code[s*d_v + j] holds, for an INT row, the signed code;
 * for an FP16 row, the 16 raw bits; for an FP32 row, the 32 raw bits.
 * r[s] is the row scale (INT rows only; 0 elsewhere), c[j] the column scale
 * (1 when the format has none). */
typedef struct {
    int32_t *code;
    float *r;
    float *c;
} orc_page;

int orc_format_check(const orc_format *f);
int orc_row_qmax(const orc_format *f, int s);     /* qmax of stored row s, 0 for float rows */
int orc_row_kind(const orc_format *f, int s);
long orc_page_bytes(const orc_format *f);          /* packed bytes per page (d = 128 formats) */

/* ---- calibration: precision map (per head, shared by the batch) ---------- */
/* S: [B][H][d_k][d_v] natural order; row_weight: [H][d_k] or NULL;
 * perm_out: [H][d_k], perm_out[h*d_k + s] = natural key channel of stored row s. */
int orc_rank_rows(const orc_format *f, int B, int H, const float *S,
                  const float *row_weight, int32_t *perm_out);

/* ---- lifetime weights (STEPQuant's temporal allocation) -----------------
 * Per head h and key channel kappa, the expected persistence of what the
 * channel stores under geometric decay with the mean gate,
 * w = 1 / (1 - mean(alpha)) (capped at 2^24), as the row_weight of
 * orc_rank_rows: channels that keep their content longer rank higher
 * (STEPQuant landing page: errors in long-lived memory persist across many
 * steps; Figure B1: long gate half-lives hold most of the quantization
 * error).  alpha: [n_samples][B][H][d_k] (gate_vector) or [n_samples][B][H];
 * the mean is one double sum (samples in order, the requests of each in
 * order) divided by n_samples * B; row_weight: [H][d_k], rounded to float. */
int orc_lifetime_weights(const orc_format *f, int B, int H, int n_samples, const float *alpha,
                         float *row_weight);

/* ---- quantize / dequantize one page ------------------------------------- */
int orc_quantize_page(const orc_format *f, const float *S_nat, const int32_t *perm,
                      orc_page *out);
int orc_dequantize_page(const orc_format *f, const orc_page *p, const int32_t *perm,
                        float *S_nat);

/* ---- joint fit of row and column scales (STEPQuant) ---------------------
 * STEPQuant fits key-row and value-column scales jointly from the state's
 * distribution and each key row's impact on the output error (paper-cards
 * page, STEPQuant abstract; freedom251 post, "STEPQuant: precision can be
 * allocated selectively").  The pages give no objective; the one used: the
 * impact-weighted squared reconstruction error over the INT rows,
 *     E = sum_kappa w_kappa sum_j (S_kappa,j - z r c)^2,
 * w_kappa the row's readout impact (E[q_kappa^2] over calibration queries:
 * o = S^T q, so a row's error reaches o scaled by q_kappa), minimized by
 * alternating exact steps from the absmax scales, each of which cannot
 * raise E:  z <- the nearest codes for (r, c) (clamped);  r_s <- the least
 * squares row scale for z, c;  c_j <- the w-weighted least squares column
 * scale for z, r (col_scales formats).  After `iters` rounds the codes are
 * taken once more for the final scales.  Arithmetic in double with one
 * rounding of each scale to float per update; sums in order (j ascending for
 * rows, kappa ascending for columns); codes as S / (r c) by one double
 * division.  impact_nat: [d_k] natural order, or NULL for uniform weights.
 * err_out (optional, iters + 1 values): E before each round's scale updates
 * and for the final page.  iters = 0 is orc_quantize_page. */
int orc_quantize_page_fit(const orc_format *f, const float *S_nat, const int32_t *perm,
                          const float *impact_nat, int iters, orc_page *out, double *err_out);

/* ---- one decode step on one page: canonical fp32 evaluation -------------
 * The pages fix no fp32 summation order.  The canonical order is the decode
 * kernel's (a column sum deals the stored rows of every 16-row block into
 * four slices of four consecutive rows; the rows of one slice in one half of
 * the page form an fma chain in ascending stored row; per slice the two half
 * chains are added, the four slice sums as (R0 + R1) + (R2 + R3)), kept so
 * that the kernel can be checked bit for bit; orc_step_f32_plain below is the
 * order-free anchor.
 * page is updated in place.  alpha points to 1 value (GDN) or d_k values in
 * natural key order (KDA).  q, k, v: d_k, d_k, d_v values.  o_out: d_v.
 * Tp_out (optional, d_k*d_v, stored order): the updated state in
 * column-normalised units before requantization.
 * margin_out (optional, d_k*d_v, stored order): distance of each element's
 * pre-rounding value from the nearest rounding boundary, in units of the
 * row's rounding step (code units for INT rows, fp16 spacing for FP16 rows,
 * +inf for FP32 rows). */
int orc_step_f32(const orc_format *f, orc_page *page, const int32_t *perm,
                 const float *q, const float *k, const float *v,
                 const float *alpha, float beta, float *o_out,
                 uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                 float *Tp_out, double *margin_out);

/* ---- the same step, plain fp32 evaluation ------------------------------
 * As orc_step_f32 in every operation except the two column sums: each is one
 * fma chain from +0 over the key channels in natural order (kappa = 0, 1,
 * ...), the sum of the definition written left to right, with no blocking
 * or tree.  Any correct fp32 evaluation of the step lies within the fp32
 * rounding bound of this one; it anchors the GPU comparison, and the
 * canonical order above is a second, stricter check. */
int orc_step_f32_plain(const orc_format *f, orc_page *page, const int32_t *perm,
                       const float *q, const float *k, const float *v,
                       const float *alpha, float beta, float *o_out,
                       uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                       float *Tp_out, double *margin_out);

/* ---- the same step from the plain definition in fp64 -------------------
 * Dequantizes the page in double, then S' = A S + beta k (v - (A S)^T k)^T,
 * o = S'^T q.  Sp_out: d_k*d_v natural order (optional); o_out: d_v. */
int orc_step_f64(const orc_format *f, const orc_page *page, const int32_t *perm,
                 const float *q, const float *k, const float *v,
                 const float *alpha, float beta, double *o_out, double *Sp_out);

/* ---- per-window decode (LeapQuant's per-window quantization) ------------
 * Within a window of steps the packed page stays fixed; each step's output
 * comes from it together with a buffer of high-precision updates, and the
 * state is requantized once, at the window's last step (the LeapQuant
 * abstract on the paper-cards page: per-window quantization).  Buffer of one page (caller-owned, fp32):
 *   P[d_k]       cumulative decay per key channel (natural order); taken as
 *                1 at the window's first step (t = 0), whatever it holds;
 *   K[W][d_k]    entry tau's key, decayed to the current step (natural order);
 *   D[W][d_v]    entry tau's delta beta_tau e_tau (column-normalised units).
 * Step t (0-based position in the window) decays P and K[0..t-1] by alpha,
 * predicts u = S0^T (P k) + sum_{tau<t} (K[tau] . k) D[tau], sets
 * D[t] = beta (v / c - u), K[t] = k, and reads out
 * o = c (S0^T (P q) + sum_{tau<=t} (K[tau] . q) D[tau]), where S0 is the page
 * (column-normalised, undecayed).  With commit != 0 the state
 * T = P S0 + sum_tau K[tau] D[tau]^T is then requantized into the page
 * (as orc_step_f32 requantizes) and P is reset to 1.  The canonical fp32
 * order: the page's stored row s gets one factor a'_s = RN(P'_kappa r_s)
 * (FP16 rows: P'_kappa), as the decode step folds the decay into the row
 * scale; the S0 products are the column sums of orc_step_f32 with row
 * weights RN(k a') and RN(q a') on the exact codes z (FP16 rows: h); a
 * buffer dot product is 4-channel fma chains per lane (d_k / 4 lanes)
 * combined by an xor butterfly; the buffer terms are added by fmaf in entry
 * order; the committed element is an fma chain from RN(z a') over the
 * entries in order.  margin_out as orc_step_f32 (commit only). */
int orc_window_step_f32(const orc_format *f, orc_page *page, const int32_t *perm,
                        float *P, float *K, float *D, int t, int commit,
                        const float *q, const float *k, const float *v,
                        const float *alpha, float beta, float *o_out,
                        uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                        double *margin_out);
/* The same with the plain column sums of orc_step_f32_plain and every buffer
 * dot product one fma chain in channel order. */
int orc_window_step_f32_plain(const orc_format *f, orc_page *page, const int32_t *perm,
                              float *P, float *K, float *D, int t, int commit,
                              const float *q, const float *k, const float *v,
                              const float *alpha, float beta, float *o_out,
                              uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                              double *margin_out);

/* ---- prefill: a prompt of L tokens through one page --------------------
 * The page's state runs through L decode steps in fp32 without being
 * requantized between them, then is requantized once (the step before decode
 * that builds the state from a prompt; "repeated prefill" on the DASC card
 * page).  Token 0 dequantizes and decays the page exactly as orc_step_f32
 * (T = z (alpha r)); token l > 0 decays the fp32 state in place,
 * T = RN(alpha T); each token then takes orc_step_f32's prediction, update
 * and readout in its canonical order.  q, k: [L][d_k], v, o_out: [L][d_v],
 * alpha: [L][d_k] (gate_vector) or [L], beta: [L].  After the last token the
 * rows are requantized as orc_step_f32 requantizes (seed, step, b, h: the
 * stochastic-rounding counter).  Tp_out (optional): the final T before the
 * requantization, stored order, column-normalised.  With L = 1 this is
 * orc_step_f32. */
int orc_prefill_f32(const orc_format *f, orc_page *page, const int32_t *perm, int L,
                    const float *q, const float *k, const float *v,
                    const float *alpha, const float *beta, float *o_out,
                    uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                    float *Tp_out, double *margin_out);
/* The same with the plain column sums of orc_step_f32_plain. */
int orc_prefill_f32_plain(const orc_format *f, orc_page *page, const int32_t *perm, int L,
                          const float *q, const float *k, const float *v,
                          const float *alpha, const float *beta, float *o_out,
                          uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                          float *Tp_out, double *margin_out);

/* ---- prefill, chunkwise form: the chunk algebra in fp64 ----------------
 * The same L tokens as orc_prefill_f32, from the page's dequantized state,
 * in chunks of C tokens (the form a tensor-core prefill computes; repeated
 * prefill: DASC card page).  Within a chunk of n tokens from state S0, with
 * gam_i = prod of the gates of the chunk's tokens up to i (per key channel)
 * and rho_ij = gam_i / gam_j, evaluated as the product of the gates of tokens
 * j + 1 .. i (so defined where a gate is zero or gam vanishes):
 *   A_ij = beta_i sum_c k_ic k_jc rho_ijc                  (j < i)
 *   E    = (I + A)^-1 R,  R_i = beta_i (v_i - (gam_i k_i)^T S0)
 *          (forward substitution: E_i = R_i - sum_{j<i} A_ij E_j)
 *   o_i  = (gam_i q_i)^T S0 + sum_{j<=i} (sum_c q_ic k_jc rho_ijc) E_j
 *   S    = diag(gam_n) S0 + sum_j (rho_nj k_j) E_j^T;
 * E_i is the step's delta beta_i (v_i - S_{i-1}^T k_i) after the decay, so
 * the chunk reproduces the token recurrence exactly in exact arithmetic.
 * q, k: [L][d_k]; v: [L][d_v]; alpha: [L][d_k] or [L]; beta: [L];
 * o_out: [L][d_v] double; Sp_out (optional): the final state, natural order,
 * double.  No requantization. */
int orc_prefill_chunked_f64(const orc_format *f, const orc_page *page, const int32_t *perm, int L, int C,
                            const float *q, const float *k, const float *v,
                            const float *alpha, const float *beta, double *o_out, double *Sp_out);

/* ---- packed byte layout (d_k = d_v = 128, row groups multiples of 16) ---- */
int orc_pack_page(const orc_format *f, const orc_page *p, uint8_t *bytes);
int orc_unpack_page(const orc_format *f, const uint8_t *bytes, orc_page *p);

/* Packed-page step over a range of pages of a [B][H] batch (single thread).
 * pages: B*H*page_bytes; perm: [H][128]; q,k,v,o: [B][H][128];
 * alpha: [B][H] or [B][H][128]; beta: [B][H]. */
int orc_decode_step_pages(const orc_format *f, int B, int H, uint8_t *pages,
                          const int32_t *perm, const float *q, const float *k,
                          const float *v, const float *alpha, const float *beta,
                          float *o, uint64_t seed, uint32_t step,
                          long page_begin, long page_end);
/* The same with orc_step_f32_plain. */
int orc_decode_step_pages_plain(const orc_format *f, int B, int H, uint8_t *pages,
                                const int32_t *perm, const float *q, const float *k,
                                const float *v, const float *alpha, const float *beta,
                                float *o, uint64_t seed, uint32_t step,
                                long page_begin, long page_end);

/* ---- scalar building blocks, exported so tests can pin them ------------- */
uint16_t orc_f32_to_f16_rn(float x);
float orc_f16_to_f32(uint16_t h);
float orc_div_rz(float a, float b);
/* element-wise loops over the three functions above */
void orc_f32_to_f16_rn_n(const float *x, uint16_t *out, long n);
void orc_f16_to_f32_n(const uint16_t *x, float *out, long n);
void orc_div_rz_n(const float *a, const float *b, float *out, long n);
/* pcg4d (Jarzynski and Olano, JCGT 2020), the stochastic-rounding hash */
void orc_pcg4d(const uint32_t in[4], uint32_t out[4]);
/* stochastic-rounding offset u in [0, 1) (a multiple of 2^-16) for element
 * (s, j); the code is floor(x + u) */
float orc_sr_offset(uint64_t seed, uint32_t step, uint32_t b, uint32_t h,
                    int s, int j, int d_v);

#ifdef __cplusplus
}
#endif
#endif
