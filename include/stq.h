/*
 * stq.h -- C ABI of the quantized Delta-rule recurrent-state decode step
 * (Gated DeltaNet / Kimi Delta Attention) for NVIDIA B200 (sm_100a).
 *
 * The method.  Per (request b, head h) the recurrent state is
 * S in R^{128 x 128}, rows = key channels, columns = value channels
 * ("STEPQuant" landing page, Fig. 5 / Figure B2: 128x128 states).  Its key
 * rows are split into groups of different bit widths and every element is
 * stored as z_ij * r_i * c_j with a key-row scale r and a value-column scale
 * c (DAMP card page, STEPQuant abstract; freedom251 post, "STEPQuant:
 * precision can be allocated selectively"), or, in the DAMP-style format,
 * selected key rows in FP16 and the rest INT8 with stochastic rounding
 * (freedom251 post, "DAMP: accuracy depends on the task").  One decode step
 * applies the gated delta rule (dev.to post, "The state is a running sum, not
 * a buffer": S <- S(I - k k^T) + v k^T in the d_v x d_k convention; here the
 * d_k x d_v convention with a decay gate and a write strength):
 *     S' = A S + beta k (v - (A S)^T k)^T,  A = alpha I (GDN) or diag(alpha) (KDA)
 *     o  = S'^T q
 * and requantizes S' in place.
 *
 * Conventions for every entry point:
 *   - All tensors are caller-owned.  Pointers named d_* are device pointers,
 *     h_* host pointers.  The library allocates only the host descriptor
 *     (stq_state); it never allocates device memory and never synchronizes,
 *     except stq_device_status, which says so.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work is enqueued on it in call order.
 *   - fp32 tensors are row-major and contiguous: q, k, v, o are [B][H][128];
 *     a scalar (GDN) alpha is [B][H], a vector (KDA) alpha is [B][H][128] in
 *     natural key order; beta is [B][H].
 *   - Errors are returned as stq_status; arguments are checked on the host
 *     before anything is enqueued, so an error return means nothing was
 *     enqueued.  Launch failures map to STQ_ERR_CUDA.  A device-side wait that
 *     runs out (it has a bounded limit) sets the state's status word, read by
 *     stq_device_status.  Non-finite inputs give unspecified values but never
 *     fault or hang.
 */
#ifndef STQ_H
#define STQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    STQ_OK = 0,
    STQ_ERR_INVALID_ARG = 1,      /* null pointer, bad size, overlapping buffers */
    STQ_ERR_UNSUPPORTED = 2,      /* a format the kernels do not handle */
    STQ_ERR_BUFFER_TOO_SMALL = 3, /* caller buffer smaller than required */
    STQ_ERR_MISALIGNED = 4,       /* pointer not aligned as documented */
    STQ_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed */
    STQ_ERR_DEVICE_TIMEOUT = 6    /* a bounded device-side wait ran out */
} stq_status;

typedef enum { STQ_INT = 0, STQ_FP16 = 1 } stq_kind;

#define STQ_MAX_GROUPS 8

/* Row-group format of every page of a state.
 *   d_k = d_v = 128 (other sizes: STQ_ERR_UNSUPPORTED).
 *   Groups are listed in stored order, conventionally widest first; the rows
 *   of the widest group are the best-ranked key channels (calibration,
 *   stq_calibrate).  group_rows: multiples of 16 summing to 128.
 *   group_kind: STQ_INT (group_bits in 2..8, symmetric codes in
 *   [-(2^(b-1)-1), 2^(b-1)-1]) or STQ_FP16 (binary16 values, no row scale).
 *   col_scales: 1 = a per-column scale c_j is stored; 0 = c_j = 1.
 *   stochastic: 1 = INT rows are requantized with stochastic rounding (FP16
 *   rows always round to nearest); 0 = round to nearest even.
 *   gate_vector: 1 = alpha is a vector over key channels (KDA); 0 = scalar. */
typedef struct {
    int d_k, d_v;
    int n_groups;
    int group_rows[STQ_MAX_GROUPS];
    int group_kind[STQ_MAX_GROUPS];
    int group_bits[STQ_MAX_GROUPS];
    int col_scales;
    int stochastic;
    int gate_vector;
} stq_format;

typedef struct stq_state stq_state;   /* opaque host descriptor */

/* Bytes of one packed page (one request, one head) of format f; 0 if the
 * format is invalid or unsupported.  Layout: codes, then fp32 r for each INT
 * row (stored order), then fp32 c[128] if col_scales; a multiple of 16. */
size_t stq_page_bytes(const stq_format *f);

/* Bytes of device memory a state of B requests x H heads needs: a 256-byte
 * header (word 0 the status word, word 1 used by stq_prefill_chunked
 * between its two launches, the rest reserved), the precision map [H][128] (uint8, stored row ->
 * key channel) padded to 256 bytes, then B*H pages, page (b, h) at index
 * b*H + h.  0 on invalid arguments. */
size_t stq_state_bytes(const stq_format *f, int batch, int heads);

/* Bind a caller-owned device buffer (>= stq_state_bytes, 256-byte aligned)
 * to a new host descriptor.  Touches no device memory; the state holds
 * nothing valid until stq_calibrate (or a caller-written map) and
 * stq_quantize_state.  stq_quantize_state clears the status word; a caller
 * that writes the map and pages itself zeroes the 256-byte header first (or
 * calls stq_device_status with clear).  Errors: INVALID_ARG (nulls, batch/heads < 1),
 * UNSUPPORTED (format), MISALIGNED, BUFFER_TOO_SMALL. */
stq_status stq_state_alloc(const stq_format *f, int batch, int heads,
                           void *d_buf, size_t buf_bytes, stq_state **out);

/* Free the host descriptor only; the device buffer stays the caller's. */
void stq_state_free(stq_state *s);

/* Byte offsets inside the state buffer (any output may be NULL). */
stq_status stq_state_layout(const stq_state *s, size_t *page_bytes, size_t *perm_offset,
                            size_t *pages_offset, size_t *status_offset);

/* Workspace bytes stq_calibrate needs for this state (fp64 partial scores). */
size_t stq_calibrate_workspace_bytes(const stq_state *s);

/* Precision map (calibration; DAMP's ranking of key channels, freedom251
 * post, "DAMP: accuracy depends on the task"; STEPQuant's ranking of key
 * rows, landing page Fig. 2).  Per head h, key channel kappa scores
 *     sum_b sum_j S[b][h][kappa][j]^2  x  row_weight[h][kappa]
 * (the batch's row mean square up to a constant, times an optional retention
 * weight); channels are ranked by descending score (ties: lower channel
 * first), the best go to group 0, and inside a group rows are stored in
 * ascending channel.  d_S: [B][H][128][128] fp32, natural key order, 16-byte
 * aligned.  d_row_weight: [H][128] fp32 or NULL (weight 1).  d_workspace:
 * >= stq_calibrate_workspace_bytes, 8-byte aligned, contents on entry
 * ignored.  Writes the state's map. */
stq_status stq_calibrate(stq_state *s, const float *d_S, const float *d_row_weight,
                         void *d_workspace, size_t workspace_bytes, void *stream);

/* Upper bound of the scratch stq_calibrate_noalloc may use (1 MiB): it serves
 * states with stq_calibrate_workspace_bytes(s) <= this, e.g. up to 1,024
 * requests of 32 heads. */
#define STQ_CALIBRATE_NOALLOC_MAX_BYTES ((size_t)1 << 20)

/* stq_calibrate without a workspace argument and without allocating: for
 * callers that cannot call cudaMalloc or take device memory from anywhere at
 * that point -- a serving runtime whose device memory is a pool reserved up
 * front, code that must not add the synchronisation an allocation can bring
 * to its stream, or a host library handed only its inputs and outputs.  The
 * pages have no counterpart of this entry point; it computes exactly what
 * stq_calibrate computes.
 *   - Its scratch is a fixed 1 MiB array in the library's device image,
 *     present on every GPU that loads the library until the process exits.
 *     States needing more (stq_calibrate_workspace_bytes(s) >
 *     STQ_CALIBRATE_NOALLOC_MAX_BYTES) get STQ_ERR_BUFFER_TOO_SMALL.
 *   - A call looks up the array's device address (a CUDA runtime query,
 *     with the call's device current) unless its stream is being captured,
 *     so a context rebuilt after a device reset is seen; a call made during
 *     capture uses the address found by the device's last call outside it,
 *     so make the first call on a device before capturing the stream into
 *     a graph.
 *   - All calls share the array: calls that overlap on the GPU (other streams,
 *     other threads, other states) race on it and must be serialized by the
 *     caller.  Nothing in it needs clearing between calls.
 * Arguments and other errors as stq_calibrate. */
stq_status stq_calibrate_noalloc(stq_state *s, const float *d_S, const float *d_row_weight, void *stream);

/* Lifetime row weights for stq_calibrate (STEPQuant's temporal allocation,
 * landing page Figure B1: long gate half-lives hold most of the quantization
 * error).  Per head h and key channel kappa,
 *     w[h][kappa] = 1 / (1 - mean alpha)     (capped at 2^24),
 * the expected persistence of what the channel stores under geometric decay
 * with the mean gate; the mean runs over the samples and the state's
 * requests (a double sum, samples then requests ascending).  Pass w as
 * stq_calibrate's d_row_weight to rank long-lived channels into the widest
 * groups.  d_alpha: device, [n_samples][B][H] (GDN) or [n_samples][B][H][128]
 * (gate_vector, 16-byte aligned), gates in [0, 1]; d_row_weight: [H][128]
 * fp32, 16-byte aligned.  Neither may overlap the state or each other.
 * Errors: INVALID_ARG (nulls, n_samples < 1, overlap), MISALIGNED, CUDA. */
stq_status stq_lifetime_weights(const stq_state *s, const float *d_alpha, int n_samples, float *d_row_weight,
                                void *stream);

/* Quantize an fp32 state into every page using the state's precision map:
 * c_j = max_i |S_ij| (1 if 0; 1 without column scales); T = S * (1/c);
 * INT rows: r = max_j |T| / qmax, codes = round-to-nearest-even of
 * T * (qmax / max_j |T| rounded toward zero); FP16 rows: binary16(T).
 * Clears the status word.  d_S as in stq_calibrate. */
stq_status stq_quantize_state(stq_state *s, const float *d_S, void *stream);

/* Largest number of fitting rounds stq_quantize_state_fit accepts. */
#define STQ_FIT_MAX_ITERS 16

/* Quantize with jointly fitted row and column scales (STEPQuant's scale
 * fitting: key-row and value-column scales fitted to the state's
 * distribution and to each key row's impact on the output error; paper-cards
 * page, STEPQuant abstract; freedom251 post, "STEPQuant: precision can be
 * allocated selectively").  The pages give no objective; the one minimized
 * is the impact-weighted squared reconstruction error over the INT rows,
 *     E = sum_kappa w_kappa sum_j (S_kappa,j - z r c)^2,
 * from the absmax scales of stq_quantize_state by `iters` rounds of three
 * exact steps, none of which can raise E: the nearest codes for (r, c)
 * (z = RNE(S / (r c)) in double, clamped to +-qmax), the least-squares row
 * scale of each row for its codes, and the w-weighted least-squares column
 * scale of each column for the codes and the new r (column-scale formats);
 * then the codes once more for the final scales.  Double arithmetic, sums in
 * a fixed order, each scale rounded to float once per update.  FP16 rows are
 * stored as binary16(S / c) with the final c.  iters = 0 is
 * stq_quantize_state.  The decode step re-derives r from the row maximum at
 * its first requantization; c stays as fitted.
 *   d_S: as stq_quantize_state.  d_row_impact: device, [H][128] fp32 in
 *   natural key order (a row's readout impact, e.g. the mean of q_kappa^2
 *   over calibration queries: o = S^T q, so row kappa's error reaches o
 *   scaled by q_kappa), >= 0, 4-byte aligned, or NULL for equal weights;
 *   it must not overlap the state or d_S.
 * Errors: INVALID_ARG (null s or d_S, iters outside [0, STQ_FIT_MAX_ITERS],
 * overlap), MISALIGNED, CUDA.  Clears the status word. */
stq_status stq_quantize_state_fit(stq_state *s, const float *d_S, const float *d_row_impact, int iters,
                                  void *stream);

/* One decode step on every page, in place (see the header comment).
 * d_q, d_k, d_v, d_o: [B][H][128], 16-byte aligned.  d_alpha: [B][H]
 * (4-byte aligned) or [B][H][128] (16-byte aligned, gate_vector).  d_beta:
 * [B][H].  None may overlap the state buffer, and d_o may overlap no input.
 * seed and step feed the stochastic-rounding generator only (the pcg4d hash
 * of Jarzynski and Olano, JCGT 2020, of (tile, step, request ^ low seed word,
 * head ^ high seed word)).  q is used as given.
 * The kernel is launched as a programmatic dependent launch: it may become
 * resident while the previous kernel on `stream` finishes, and reads nothing
 * from global memory until that kernel has completed and its writes are
 * visible, so stream order holds as for a plain launch. */
stq_status stq_decode_step(stq_state *s, const float *d_q, const float *d_k, const float *d_v,
                           const float *d_alpha, const float *d_beta, float *d_o,
                           uint64_t seed, uint32_t step, void *stream);

/* The decode step on a subset of the state's requests, found through a slot
 * table: the shape a serving engine with a pool of state slots uses (packed
 * pages per request in an SGLang integration: freedom251 post, "Memory and
 * speed gains are implementation-specific").  Input row i (q, k, v, alpha, beta and o
 * row i, layouts as stq_decode_step with B = n_rows) belongs to the request in
 * state slot d_slots[i]; the pages (d_slots[i], h) are stepped in place and
 * no other page is touched.
 *   d_slots: device, [n_rows] int32, 4-byte aligned, caller-owned; slots must
 *   be distinct (two rows on one slot race on its pages: unspecified codes,
 *   never a fault).  1 <= n_rows <= the state's batch.
 *   Stochastic rounding counts by the slot (counter = (tile, step, slot,
 *   head)), so a request's rounding does not depend on its row.
 *   A slot outside [0, batch) is caught on the device before any access: its
 *   pages are not read or written, its o row is NaN, and stq_device_status
 *   reports STQ_ERR_INVALID_ARG.  Other errors as stq_decode_step. */
stq_status stq_decode_step_slots(stq_state *s, const int32_t *d_slots, int n_rows, const float *d_q,
                                 const float *d_k, const float *d_v, const float *d_alpha,
                                 const float *d_beta, float *d_o, uint64_t seed, uint32_t step,
                                 void *stream);

/* Byte offset (from the state buffer's start) and length of the pages of the
 * request in `slot` -- its H pages are contiguous -- so that a caller can copy
 * a request's state out (a checkpoint, a preemption) and back in with a
 * plain device copy.  Errors: INVALID_ARG (null state, slot out of range). */
stq_status stq_request_pages(const stq_state *s, int slot, size_t *offset, size_t *bytes);

/* ---- per-window decode ---------------------------------------------------
 * Per-window quantization (LeapQuant abstract, paper-cards page): within a
 * window of W steps (1 <= W <= STQ_WINDOW_MAX) the packed pages stay fixed;
 * each step's output comes from them together with a caller-owned fp32
 * buffer of the window's updates, and the window's committing step
 * requantizes every page once.
 * Buffer: device, stq_window_buffer_bytes(s, W) bytes, 256-byte aligned,
 * caller-owned, no initialisation needed; page (b, h) owns the
 * 512 (1 + 2W) bytes at (b H + h) 512 (1 + 2W):
 *   P[128]     cumulative decay of the window per key channel (natural order)
 *   K[W][128]  entry tau's key, decayed to the latest step (natural order)
 *   D[W][128]  entry tau's delta beta_tau (v_tau (1/c) - u_tau), divided by c
 * Step t (0-based position in the window) of every page, with S0 the page
 * (column-normalised, undecayed, stored row s = key channel perm[s]):
 *   P' = (t > 0 ? P : 1) alpha;   K[tau] <- K[tau] alpha   (tau < t)
 *   u = S0^T (P' k) + sum_{tau<t} (K[tau] . k) D[tau]
 *   D[t] = beta (v / c - u);   K[t] = k
 *   o = c (S0^T (P' q) + sum_{tau<=t} (K[tau] . q) D[tau])
 * i.e. the gated delta rule run exactly from the page for t + 1 steps.  In
 * fp32 the decay is folded into the row scale, one factor a' = RN(P' r) per
 * stored row (FP16 rows: P'), as stq_decode_step folds alpha into r: the
 * page's column sums take row weights RN(k a') and RN(q a') on the exact
 * codes in stq_decode_step's order; an entry's dot product is a 4-channel fma
 * chain per lane plus an xor butterfly over 32 lanes; the entries' terms are
 * added by fma in entry order; the commit rebuilds RN(z a') and adds
 * fma(K[tau], D[tau], .) for tau = 0 .. t.  A
 * step that does not commit writes P', K[0 .. t] and D[t] to the buffer and
 * leaves the pages unchanged.  A committing step (commit != 0; required at
 * t = W - 1, allowed at any t to end a window early) writes no buffer row;
 * it requantizes T = P' S0 + sum_{tau<=t} K[tau] D[tau]^T into every page as
 * stq_decode_step requantizes its updated state (same row scales, rounding
 * and stochastic-rounding counter, with `step`), and the next step is a new
 * window's t = 0, which reads nothing from the buffer.
 * Inputs, layouts and alignment as stq_decode_step; the buffer may overlap
 * neither the state nor an input or o.  Programmatic dependent launch as
 * stq_decode_step.  Errors: INVALID_ARG (null pointer, W outside
 * [1, STQ_WINDOW_MAX], t outside [0, W), t = W - 1 without commit, overlap),
 * MISALIGNED, BUFFER_TOO_SMALL (buf_bytes below stq_window_buffer_bytes),
 * CUDA; a bounded wait that ran out is reported by stq_device_status. */
#define STQ_WINDOW_MAX 16

/* Bytes of a window buffer for windows of W steps (0 on bad arguments). */
size_t stq_window_buffer_bytes(const stq_state *s, int window);

stq_status stq_window_step(stq_state *s, void *d_buf, size_t buf_bytes, int window, int t, int commit,
                           const float *d_q, const float *d_k, const float *d_v, const float *d_alpha,
                           const float *d_beta, float *d_o, uint64_t seed, uint32_t step, void *stream);

/* ---- prefill ------------------------------------------------------------
 * A prompt of L tokens through every page: the step before decode that
 * builds the state from a prompt ("repeated prefill", DASC card page).  Each
 * page's state runs through L decode steps in fp32 -- token 0 dequantizes and
 * decays the page exactly as stq_decode_step, token l > 0 decays the fp32
 * state in place (T = alpha T); every token then takes the decode step's
 * prediction, rank-1 update and readout -- and is requantized once, after
 * the last token, as stq_decode_step requantizes (row scales re-derived,
 * column scales kept; stochastic rounding with `step`).  With L = 1 this is
 * stq_decode_step.  To build a state from nothing, quantize a zero state
 * first (stq_quantize_state: codes 0, r = 0, c = 1).
 *   d_q, d_k, d_v, d_o: [L][B][H][128]; d_alpha: [L][B][H] or
 *   [L][B][H][128] (gate_vector); d_beta: [L][B][H]; alignment as
 *   stq_decode_step.  L >= 1 and L * B * H <= 2^31 - 16.
 *   d_S_out (optional, NULL = none): [B][H][128][128] fp32, 16-byte aligned,
 *   natural key order: the state after the last token before the
 *   requantization, S = T c; a caller can calibrate and quantize it afresh
 *   (stq_calibrate, stq_quantize_state) to fit new column scales.
 * No buffer may overlap the state, an input or another output.  Programmatic
 * dependent launch as stq_decode_step.  Errors: INVALID_ARG, MISALIGNED,
 * CUDA; a bounded wait that ran out is reported by stq_device_status, and
 * then pages that were not finished keep their codes. */
stq_status stq_prefill(stq_state *s, int L, const float *d_q, const float *d_k, const float *d_v,
                       const float *d_alpha, const float *d_beta, float *d_o, float *d_S_out, uint64_t seed,
                       uint32_t step, void *stream);

/* The same prefill in chunkwise form on the tensor cores.  The prompt runs
 * in chunks of 128 tokens;
 * per chunk, with gam_i the product of the chunk's gates up to token i, the
 * chunk's deltas E are the triangular solve (I + A) E = R,
 *     A_ij = beta_i (gam_i / gam_j) (k_i . k_j)  (j < i),
 *     R_i  = beta_i (v_i - gam_i S0^T k_i),
 * o_i = gam_i S0^T q_i + sum_{j<=i} (gam_i / gam_j) (q_i . k_j) E_j, and the
 * state becomes gam_n S0 + sum_j (gam_n / gam_j) k_j E_j^T, the token
 * recurrence of stq_prefill resolved a chunk at a time (repeated prefill,
 * DASC card page).  Any gates are accepted, zero included: a page with a
 * chunk whose cumulative gates leave [2^-100, 2^100] takes each
 * gam_i / gam_j as the product of the gates of tokens j + 1 .. i (in a
 * second launch; slower by about a sixth for that page).  The two launches
 * share the second 32-bit word of the state's header.
 * The products run as tf32 tensor-core MMAs with split
 * operands (fp32 = tf32 part + remainder, three products), the solve on the
 * CUDA cores; results agree with stq_prefill to fp32 rounding, not bit for
 * bit (the summation order differs), and the one requantization after the
 * last token is stq_prefill's.  Gate vectors (KDA): gam is per key channel
 * and folded into the operands (k gam, q gam, k / gam); a chunk with a gate
 * outside [0, 1] or a cumulative decay below 2^-100 runs token by token on
 * the CUDA cores instead.  Arguments, layouts and
 * errors as stq_prefill.  One CTA per page (the whole shared memory and tensor
 * memory of an SM); a bounded wait that ran out is reported by
 * stq_device_status. */
stq_status stq_prefill_chunked(stq_state *s, int L, const float *d_q, const float *d_k, const float *d_v,
                               const float *d_alpha, const float *d_beta, float *d_o, float *d_S_out,
                               uint64_t seed, uint32_t step, void *stream);

/* Device staging bytes stq_decode_step_host needs (q, k, v, alpha, beta, o). */
size_t stq_decode_io_bytes(const stq_state *s);

/* The same step with host-resident inputs and output: enqueues the
 * host-to-device copies of h_q, h_k, h_v, h_alpha, h_beta into d_io, the
 * step, and the device-to-host copy of o into h_o, all on `stream`.  Host
 * buffers should be pinned for the copies to be asynchronous.  d_io:
 * >= stq_decode_io_bytes, 256-byte aligned, caller-owned scratch.  The
 * caller synchronizes the stream before reading h_o. */
stq_status stq_decode_step_host(stq_state *s, const float *h_q, const float *h_k,
                                const float *h_v, const float *h_alpha, const float *h_beta,
                                float *h_o, void *d_io, size_t io_bytes,
                                uint64_t seed, uint32_t step, void *stream);

/* n_steps consecutive steps with host-resident inputs and outputs, the
 * copies overlapped with the steps: step i's inputs are read from h_x +
 * i * (one step's elements) (the layouts of stq_decode_step_host, steps
 * outermost), its o is written to h_o + i * B*H*128, and its stochastic-
 * rounding step index is step + i.  Two staging slots alternate: while step
 * i runs on `stream`, the inputs of step i + 1 are copied in and the o of
 * step i - 1 is copied out on two streams the call creates (and releases),
 * ordered by events, so every copy of every step still happens inside the
 * call.  The steps are the stq_decode_step kernel, so the results equal
 * n_steps calls of stq_decode_step_host.  d_io: >= 2 * stq_decode_io_bytes,
 * 256-byte aligned, caller-owned; host buffers pinned.  All work is ordered
 * before any later work on `stream`; the caller synchronizes it before
 * reading h_o.  Errors as stq_decode_step_host (BUFFER_TOO_SMALL below two
 * slots; INVALID_ARG for n_steps < 1); a CUDA error mid-way returns
 * STQ_ERR_CUDA with the steps so far enqueued. */
stq_status stq_decode_steps_host(stq_state *s, int n_steps, const float *h_q, const float *h_k,
                                 const float *h_v, const float *h_alpha, const float *h_beta,
                                 float *h_o, void *d_io, size_t io_bytes,
                                 uint64_t seed, uint32_t step, void *stream);

/* Dequantize every page to fp32 [B][H][128][128] in natural key order:
 * S_ij = (z_ij * r_i) * c_j (FP16 rows: h_ij * c_j).  d_S 16-byte aligned. */
stq_status stq_dequantize_state(const stq_state *s, float *d_S, void *stream);

/* Synchronizes `stream`, then reads the state's status word: STQ_OK, or
 * STQ_ERR_DEVICE_TIMEOUT if a bounded device wait ran out since the last
 * clear.  clear != 0 resets the word. */
stq_status stq_device_status(stq_state *s, void *stream, int clear);

/* Limit of every bounded device-side wait, in nanoseconds (default 1e9).
 * Test hook: stall_first_wait != 0 makes the next stq_decode_step's first
 * pipeline wait wait on a barrier nothing ever completes, so it runs out
 * after the limit, sets the status word and the kernel returns. */
stq_status stq_set_wait_limit(stq_state *s, uint64_t limit_ns, int stall_first_wait);

const char *stq_status_string(stq_status st);

/* Library version, 100 * major + minor. */
int stq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* STQ_H */
