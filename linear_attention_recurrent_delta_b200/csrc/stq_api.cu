// stq_api.cu -- the C ABI: argument validation, state layout, dispatch.
// Nothing here allocates device memory or synchronizes (except
// stq_device_status, which is documented to).
#include "stq_internal.h"
#include "stq_lifetime.h"

#include <cstring>
#include <mutex>
#include <new>

namespace stq {

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

stq_status build_dev_format(const stq_format *f, DevFormat *out) {
    if (!f) return STQ_ERR_INVALID_ARG;
    if (f->d_k != kD || f->d_v != kD) return STQ_ERR_UNSUPPORTED;
    if (f->n_groups < 1 || f->n_groups > STQ_MAX_GROUPS) return STQ_ERR_INVALID_ARG;
    if ((f->col_scales | f->stochastic | f->gate_vector) & ~1) return STQ_ERR_INVALID_ARG;
    int total = 0;
    for (int g = 0; g < f->n_groups; ++g) {
        const int rows = f->group_rows[g];
        if (rows <= 0) return STQ_ERR_INVALID_ARG;
        if (rows % 16) return STQ_ERR_UNSUPPORTED;
        if (f->group_kind[g] == STQ_INT) {
            if (f->group_bits[g] < 2 || f->group_bits[g] > 8) return STQ_ERR_UNSUPPORTED;
        } else if (f->group_kind[g] != STQ_FP16) {
            return STQ_ERR_INVALID_ARG;
        }
        total += rows;
    }
    if (total != kD) return STQ_ERR_INVALID_ARG;
    DevFormat F;
    std::memset(&F, 0, sizeof(F));
    int off = 0, rbase = 0, g = 0, g_end = f->group_rows[0];
    for (int blk = 0; blk < kBlocks; ++blk) {
        while (16 * blk >= g_end) { ++g; g_end += f->group_rows[g]; }
        const int kind = f->group_kind[g] == STQ_FP16 ? kKindFp16 : kKindInt;
        const int bits = kind == kKindFp16 ? 16 : f->group_bits[g];
        F.bits8 |= (uint64_t)bits << (8 * blk);
        F.rbase8 |= (uint64_t)rbase << (8 * blk);
        (blk < 4 ? F.off_lo : F.off_hi) |= (uint64_t)off << (16 * (blk & 3));
        off += 256 * bits;          // planes of a 16-row block: 256 bytes per bit
        if (kind == kKindInt) rbase += 16;
    }
    F.n_int_rows = rbase;
    F.r_off = off;
    F.c_off = off + 4 * rbase;
    F.page_bytes = F.c_off + (f->col_scales ? 4 * kD : 0);
    F.col_scales = f->col_scales;
    F.stochastic = f->stochastic;
    F.gate_vector = f->gate_vector;
    *out = F;
    return STQ_OK;
}

int persistent_grid(const void *kernel, int threads, size_t dyn_smem, long n_units) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, dyn_smem) != cudaSuccess)
        return -1;
    if (per_sm < 1) return -1;
    long g = (long)sms * per_sm;
    if (g > n_units) g = n_units;
    return (int)g;
}

}  // namespace stq

using namespace stq;

static bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + nb && y < x + na;
}

static bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

extern "C" {

int stq_version(void) { return 100; }

const char *stq_status_string(stq_status st) {
    switch (st) {
        case STQ_OK: return "ok";
        case STQ_ERR_INVALID_ARG: return "invalid argument";
        case STQ_ERR_UNSUPPORTED: return "unsupported format";
        case STQ_ERR_BUFFER_TOO_SMALL: return "buffer too small";
        case STQ_ERR_MISALIGNED: return "misaligned pointer";
        case STQ_ERR_CUDA: return "CUDA error";
        case STQ_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

size_t stq_page_bytes(const stq_format *f) {
    DevFormat F;
    if (build_dev_format(f, &F) != STQ_OK) return 0;
    return (size_t)F.page_bytes;
}

static size_t state_bytes_for(const DevFormat &F, int batch, int heads) {
    return kHeaderBytes + round_up((size_t)heads * kD, 256) + (size_t)batch * heads * F.page_bytes;
}

size_t stq_state_bytes(const stq_format *f, int batch, int heads) {
    DevFormat F;
    if (build_dev_format(f, &F) != STQ_OK || batch < 1 || heads < 1) return 0;
    if ((long long)batch * heads > 0x7FFFFFFFLL) return 0;
    return state_bytes_for(F, batch, heads);
}

stq_status stq_state_alloc(const stq_format *f, int batch, int heads, void *d_buf, size_t buf_bytes,
                           stq_state **out) {
    if (!out) return STQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (!f || !d_buf || batch < 1 || heads < 1) return STQ_ERR_INVALID_ARG;
    if ((long long)batch * heads > 0x7FFFFFFFLL) return STQ_ERR_INVALID_ARG;
    DevFormat F;
    stq_status st = build_dev_format(f, &F);
    if (st != STQ_OK) return st;
    if (!aligned(d_buf, 256)) return STQ_ERR_MISALIGNED;
    const size_t need = state_bytes_for(F, batch, heads);
    if (buf_bytes < need) return STQ_ERR_BUFFER_TOO_SMALL;
    stq_state *s = new (std::nothrow) stq_state;
    if (!s) return STQ_ERR_INVALID_ARG;
    s->fmt = *f;
    s->batch = batch;
    s->heads = heads;
    s->base = static_cast<uint8_t *>(d_buf);
    s->buf_bytes = buf_bytes;
    s->page_bytes = (size_t)F.page_bytes;
    s->status_offset = 0;
    s->perm_offset = kHeaderBytes;
    s->pages_offset = kHeaderBytes + round_up((size_t)heads * kD, 256);
    s->dev = F;
    s->wait_limit_ns = 1000000000ull;
    s->stall_first_wait = 0;
    *out = s;
    return STQ_OK;
}

void stq_state_free(stq_state *s) { delete s; }

stq_status stq_state_layout(const stq_state *s, size_t *page_bytes, size_t *perm_offset, size_t *pages_offset,
                            size_t *status_offset) {
    if (!s) return STQ_ERR_INVALID_ARG;
    if (page_bytes) *page_bytes = s->page_bytes;
    if (perm_offset) *perm_offset = s->perm_offset;
    if (pages_offset) *pages_offset = s->pages_offset;
    if (status_offset) *status_offset = s->status_offset;
    return STQ_OK;
}

size_t stq_calibrate_workspace_bytes(const stq_state *s) {
    if (!s) return 0;
    return calibrate_workspace_bytes(s->batch, s->heads);
}

static size_t state_span(const stq_state *s) {
    return state_bytes_for(s->dev, s->batch, s->heads);
}

}  // extern "C"

stq_status stq::check_calibrate_input(const stq_state *s, const float *d_S, const float *d_row_weight) {
    if (!s || !d_S) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_S, 16) || (d_row_weight && !aligned(d_row_weight, 4))) return STQ_ERR_MISALIGNED;
    const size_t nS = (size_t)s->batch * s->heads * kD * kD * sizeof(float);
    if (overlaps(d_S, nS, s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    return STQ_OK;
}

extern "C" {

stq_status stq_calibrate(stq_state *s, const float *d_S, const float *d_row_weight, void *d_workspace,
                         size_t workspace_bytes, void *stream) {
    if (!s || !d_S || !d_workspace) return STQ_ERR_INVALID_ARG;
    const stq_status in = stq::check_calibrate_input(s, d_S, d_row_weight);
    if (in != STQ_OK) return in;
    if (!aligned(d_workspace, 8)) return STQ_ERR_MISALIGNED;
    const size_t need = calibrate_workspace_bytes(s->batch, s->heads);
    if (workspace_bytes < need) return STQ_ERR_BUFFER_TOO_SMALL;
    const size_t nS = (size_t)s->batch * s->heads * kD * kD * sizeof(float);
    if (overlaps(d_workspace, need, s->base, state_span(s)) || overlaps(d_workspace, need, d_S, nS))
        return STQ_ERR_INVALID_ARG;
    cudaError_t err = launch_calibrate(s, d_S, d_row_weight, static_cast<double *>(d_workspace),
                                       static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

stq_status stq_lifetime_weights(const stq_state *s, const float *d_alpha, int n_samples, float *d_row_weight,
                                void *stream) {
    if (!s || !d_alpha || !d_row_weight || n_samples < 1) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_alpha, s->fmt.gate_vector ? 16 : 4) || !aligned(d_row_weight, 16)) return STQ_ERR_MISALIGNED;
    const size_t na = s->fmt.gate_vector ? kD : 1;
    const size_t n_alpha = (size_t)n_samples * s->batch * s->heads * na * sizeof(float);
    const size_t n_w = (size_t)s->heads * kD * sizeof(float);
    if (overlaps(d_alpha, n_alpha, s->base, state_span(s)) || overlaps(d_row_weight, n_w, s->base, state_span(s)) ||
        overlaps(d_row_weight, n_w, d_alpha, n_alpha))
        return STQ_ERR_INVALID_ARG;
    cudaError_t err = launch_lifetime(s, d_alpha, n_samples, d_row_weight, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

stq_status stq_quantize_state(stq_state *s, const float *d_S, void *stream) {
    if (!s || !d_S) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_S, 16)) return STQ_ERR_MISALIGNED;
    const size_t nS = (size_t)s->batch * s->heads * kD * kD * sizeof(float);
    if (overlaps(d_S, nS, s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(s->base + s->status_offset, 0, sizeof(uint32_t), cs) != cudaSuccess) return STQ_ERR_CUDA;
    cudaError_t err = launch_quantize(s, d_S, cs);
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

stq_status stq_quantize_state_fit(stq_state *s, const float *d_S, const float *d_row_impact, int iters,
                                  void *stream) {
    if (!s || !d_S || iters < 0 || iters > STQ_FIT_MAX_ITERS) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_S, 16) || (d_row_impact && !aligned(d_row_impact, 4))) return STQ_ERR_MISALIGNED;
    const size_t nS = (size_t)s->batch * s->heads * kD * kD * sizeof(float);
    const size_t nW = (size_t)s->heads * kD * sizeof(float);
    if (overlaps(d_S, nS, s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    if (d_row_impact && (overlaps(d_row_impact, nW, s->base, state_span(s)) || overlaps(d_row_impact, nW, d_S, nS)))
        return STQ_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(s->base + s->status_offset, 0, sizeof(uint32_t), cs) != cudaSuccess) return STQ_ERR_CUDA;
    cudaError_t err = launch_fit(s, d_S, d_row_impact, iters, cs);
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

// n_rows: request rows of the inputs and of o (the state's batch, or the
// length of a slot table)
static stq_status check_step_args(const stq_state *s, int n_rows, const float *q, const float *k,
                                  const float *v, const float *alpha, const float *beta, const float *o) {
    if (!s || !q || !k || !v || !alpha || !beta || !o) return STQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(beta, 4) ||
        !aligned(alpha, s->fmt.gate_vector ? 16 : 4))
        return STQ_ERR_MISALIGNED;
    const size_t n = (size_t)n_rows * s->heads;
    const size_t vec = n * kD * sizeof(float), sc = n * sizeof(float);
    const size_t na = s->fmt.gate_vector ? vec : sc;
    const size_t span = state_span(s);
    const void *in[5] = {q, k, v, alpha, beta};
    const size_t len[5] = {vec, vec, vec, na, sc};
    for (int i = 0; i < 5; ++i) {
        if (overlaps(in[i], len[i], s->base, span)) return STQ_ERR_INVALID_ARG;
        if (overlaps(in[i], len[i], o, vec)) return STQ_ERR_INVALID_ARG;
    }
    if (overlaps(o, vec, s->base, span)) return STQ_ERR_INVALID_ARG;
    return STQ_OK;
}

// The step behind both entry points.  early_launch: the launch may start while
// a preceding kernel on the stream finishes (the kernel waits for it before
// its first global read); the host entry point, whose step follows copies,
// launches plainly.
static stq_status decode_step(stq_state *s, const int32_t *d_slots, int n_rows, const float *d_q,
                              const float *d_k, const float *d_v, const float *d_alpha, const float *d_beta,
                              float *d_o, uint64_t seed, uint32_t step, void *stream, bool early_launch) {
    stq_status st = check_step_args(s, n_rows, d_q, d_k, d_v, d_alpha, d_beta, d_o);
    if (st != STQ_OK) return st;
    const int stall = s->stall_first_wait;
    s->stall_first_wait = 0;
    cudaError_t err = launch_decode(s, d_q, d_k, d_v, d_alpha, d_beta, d_o, seed, step, stall, early_launch,
                                    d_slots, n_rows, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

stq_status stq_decode_step(stq_state *s, const float *d_q, const float *d_k, const float *d_v,
                           const float *d_alpha, const float *d_beta, float *d_o, uint64_t seed, uint32_t step,
                           void *stream) {
    if (!s) return STQ_ERR_INVALID_ARG;
    return decode_step(s, nullptr, s->batch, d_q, d_k, d_v, d_alpha, d_beta, d_o, seed, step, stream, true);
}

stq_status stq_decode_step_slots(stq_state *s, const int32_t *d_slots, int n_rows, const float *d_q,
                                 const float *d_k, const float *d_v, const float *d_alpha, const float *d_beta,
                                 float *d_o, uint64_t seed, uint32_t step, void *stream) {
    if (!s || !d_slots) return STQ_ERR_INVALID_ARG;
    if (n_rows < 1 || n_rows > s->batch) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_slots, 4)) return STQ_ERR_MISALIGNED;
    if (overlaps(d_slots, (size_t)n_rows * sizeof(int32_t), s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    return decode_step(s, d_slots, n_rows, d_q, d_k, d_v, d_alpha, d_beta, d_o, seed, step, stream, true);
}

stq_status stq_request_pages(const stq_state *s, int slot, size_t *offset, size_t *bytes) {
    if (!s || slot < 0 || slot >= s->batch) return STQ_ERR_INVALID_ARG;
    if (offset) *offset = s->pages_offset + (size_t)slot * s->heads * s->page_bytes;
    if (bytes) *bytes = (size_t)s->heads * s->page_bytes;
    return STQ_OK;
}

size_t stq_window_buffer_bytes(const stq_state *s, int window) {
    if (!s || window < 1 || window > STQ_WINDOW_MAX) return 0;
    return (size_t)s->batch * s->heads * window_buffer_stride(window);
}

stq_status stq_window_step(stq_state *s, void *d_buf, size_t buf_bytes, int window, int t, int commit,
                           const float *d_q, const float *d_k, const float *d_v, const float *d_alpha,
                           const float *d_beta, float *d_o, uint64_t seed, uint32_t step, void *stream) {
    if (!s || !d_buf) return STQ_ERR_INVALID_ARG;
    if (window < 1 || window > STQ_WINDOW_MAX || t < 0 || t >= window || (t == window - 1 && !commit))
        return STQ_ERR_INVALID_ARG;
    stq_status st = check_step_args(s, s->batch, d_q, d_k, d_v, d_alpha, d_beta, d_o);
    if (st != STQ_OK) return st;
    if (!aligned(d_buf, 256)) return STQ_ERR_MISALIGNED;
    const size_t need = stq_window_buffer_bytes(s, window);
    if (buf_bytes < need) return STQ_ERR_BUFFER_TOO_SMALL;
    const size_t n = (size_t)s->batch * s->heads;
    const size_t vec = n * kD * sizeof(float), sc = n * sizeof(float);
    const void *io[6] = {d_q, d_k, d_v, d_alpha, d_beta, d_o};
    const size_t len[6] = {vec, vec, vec, s->fmt.gate_vector ? vec : sc, sc, vec};
    if (overlaps(d_buf, need, s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    for (int i = 0; i < 6; ++i)
        if (overlaps(d_buf, need, io[i], len[i])) return STQ_ERR_INVALID_ARG;
    const int stall = s->stall_first_wait;
    s->stall_first_wait = 0;
    cudaError_t err = launch_window(s, static_cast<uint8_t *>(d_buf), window, t, commit != 0, d_q, d_k, d_v,
                                    d_alpha, d_beta, d_o, seed, step, stall, true, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

stq_status stq_prefill(stq_state *s, int L, const float *d_q, const float *d_k, const float *d_v,
                       const float *d_alpha, const float *d_beta, float *d_o, float *d_S_out, uint64_t seed,
                       uint32_t step, void *stream) {
    if (!s || !d_q || !d_k || !d_v || !d_alpha || !d_beta || !d_o) return STQ_ERR_INVALID_ARG;
    const long long n = (long long)s->batch * s->heads;
    if (L < 1 || (long long)L * n > 0x7FFFFFF0LL) return STQ_ERR_INVALID_ARG;   // token indices (+ ring depth) fit an int
    if (!aligned(d_q, 16) || !aligned(d_k, 16) || !aligned(d_v, 16) || !aligned(d_o, 16) || !aligned(d_beta, 4) ||
        !aligned(d_alpha, s->fmt.gate_vector ? 16 : 4) || (d_S_out && !aligned(d_S_out, 16)))
        return STQ_ERR_MISALIGNED;
    const size_t vec = (size_t)L * n * kD * sizeof(float), sc = (size_t)L * n * sizeof(float);
    const size_t span = state_span(s);
    const void *in[5] = {d_q, d_k, d_v, d_alpha, d_beta};
    const size_t len[5] = {vec, vec, vec, s->fmt.gate_vector ? vec : sc, sc};
    const size_t nS = (size_t)n * kD * kD * sizeof(float);
    for (int i = 0; i < 5; ++i) {
        if (overlaps(in[i], len[i], s->base, span) || overlaps(in[i], len[i], d_o, vec)) return STQ_ERR_INVALID_ARG;
        if (d_S_out && overlaps(in[i], len[i], d_S_out, nS)) return STQ_ERR_INVALID_ARG;
    }
    if (overlaps(d_o, vec, s->base, span)) return STQ_ERR_INVALID_ARG;
    if (d_S_out && (overlaps(d_S_out, nS, s->base, span) || overlaps(d_S_out, nS, d_o, vec))) return STQ_ERR_INVALID_ARG;
    const int stall = s->stall_first_wait;
    s->stall_first_wait = 0;
    cudaError_t err = launch_prefill(s, L, d_q, d_k, d_v, d_alpha, d_beta, d_o, d_S_out, seed, step, stall, true,
                                     static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

stq_status stq_prefill_chunked(stq_state *s, int L, const float *d_q, const float *d_k, const float *d_v,
                               const float *d_alpha, const float *d_beta, float *d_o, float *d_S_out,
                               uint64_t seed, uint32_t step, void *stream) {
    if (!s || !d_q || !d_k || !d_v || !d_alpha || !d_beta || !d_o) return STQ_ERR_INVALID_ARG;
    const long long n = (long long)s->batch * s->heads;
    if (L < 1 || (long long)(L + 128) * n > 0x7FFFFFF0LL) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_q, 16) || !aligned(d_k, 16) || !aligned(d_v, 16) || !aligned(d_o, 16) || !aligned(d_beta, 4) ||
        !aligned(d_alpha, s->fmt.gate_vector ? 16 : 4) || (d_S_out && !aligned(d_S_out, 16)))
        return STQ_ERR_MISALIGNED;
    const size_t vec = (size_t)L * n * kD * sizeof(float), sc = (size_t)L * n * sizeof(float);
    const size_t span = state_span(s);
    const void *in[5] = {d_q, d_k, d_v, d_alpha, d_beta};
    const size_t len[5] = {vec, vec, vec, s->fmt.gate_vector ? vec : sc, sc};
    const size_t nS = (size_t)n * kD * kD * sizeof(float);
    for (int i = 0; i < 5; ++i) {
        if (overlaps(in[i], len[i], s->base, span) || overlaps(in[i], len[i], d_o, vec)) return STQ_ERR_INVALID_ARG;
        if (d_S_out && overlaps(in[i], len[i], d_S_out, nS)) return STQ_ERR_INVALID_ARG;
    }
    if (overlaps(d_o, vec, s->base, span)) return STQ_ERR_INVALID_ARG;
    if (d_S_out && (overlaps(d_S_out, nS, s->base, span) || overlaps(d_S_out, nS, d_o, vec))) return STQ_ERR_INVALID_ARG;
    const int stall = s->stall_first_wait;
    s->stall_first_wait = 0;
    cudaError_t err = launch_prefill_tc(s, L, d_q, d_k, d_v, d_alpha, d_beta, d_o, d_S_out, seed, step, stall,
                                        static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

struct IoLayout {
    size_t q, k, v, alpha, beta, o, total, vec, na, sc;
};

static IoLayout io_layout(const stq_state *s) {
    IoLayout L;
    const size_t n = (size_t)s->batch * s->heads;
    L.vec = n * kD * sizeof(float);
    L.sc = n * sizeof(float);
    L.na = s->fmt.gate_vector ? L.vec : L.sc;
    L.q = 0;
    L.k = round_up(L.q + L.vec, 256);
    L.v = round_up(L.k + L.vec, 256);
    L.alpha = round_up(L.v + L.vec, 256);
    L.beta = round_up(L.alpha + L.na, 256);
    L.o = round_up(L.beta + L.sc, 256);
    L.total = round_up(L.o + L.vec, 256);
    return L;
}

size_t stq_decode_io_bytes(const stq_state *s) { return s ? io_layout(s).total : 0; }

stq_status stq_decode_step_host(stq_state *s, const float *h_q, const float *h_k, const float *h_v,
                                const float *h_alpha, const float *h_beta, float *h_o, void *d_io,
                                size_t io_bytes, uint64_t seed, uint32_t step, void *stream) {
    if (!s || !h_q || !h_k || !h_v || !h_alpha || !h_beta || !h_o || !d_io) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_io, 256)) return STQ_ERR_MISALIGNED;
    const IoLayout L = io_layout(s);
    if (io_bytes < L.total) return STQ_ERR_BUFFER_TOO_SMALL;
    if (overlaps(d_io, L.total, s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    uint8_t *io = static_cast<uint8_t *>(d_io);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const struct { size_t off; const void *src; size_t n; } in[5] = {
        {L.q, h_q, L.vec}, {L.k, h_k, L.vec}, {L.v, h_v, L.vec}, {L.alpha, h_alpha, L.na}, {L.beta, h_beta, L.sc}};
    for (int i = 0; i < 5; ++i)
        if (cudaMemcpyAsync(io + in[i].off, in[i].src, in[i].n, cudaMemcpyHostToDevice, cs) != cudaSuccess)
            return STQ_ERR_CUDA;
    stq_status st = decode_step(s, nullptr, s->batch, reinterpret_cast<float *>(io + L.q),
                                reinterpret_cast<float *>(io + L.k),
                                reinterpret_cast<float *>(io + L.v), reinterpret_cast<float *>(io + L.alpha),
                                reinterpret_cast<float *>(io + L.beta), reinterpret_cast<float *>(io + L.o),
                                seed, step, stream, false);
    if (st != STQ_OK) return st;
    if (cudaMemcpyAsync(h_o, io + L.o, L.vec, cudaMemcpyDeviceToHost, cs) != cudaSuccess) return STQ_ERR_CUDA;
    return STQ_OK;
}

// Events and streams of one pipelined call, released on every return path.
namespace {
struct Pipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t in_ready[2] = {nullptr, nullptr}, step_done[2] = {nullptr, nullptr},
                out_done[2] = {nullptr, nullptr};
    bool ok = true;
    Pipe() {
        ok = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) == cudaSuccess;
        for (int i = 0; i < 2 && ok; ++i)
            ok = cudaEventCreateWithFlags(&in_ready[i], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&step_done[i], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&out_done[i], cudaEventDisableTiming) == cudaSuccess;
    }
    ~Pipe() {   // destroying them does not wait: the work in flight completes
        for (int i = 0; i < 2; ++i) {
            if (in_ready[i]) cudaEventDestroy(in_ready[i]);
            if (step_done[i]) cudaEventDestroy(step_done[i]);
            if (out_done[i]) cudaEventDestroy(out_done[i]);
        }
        if (h2d) cudaStreamDestroy(h2d);
        if (d2h) cudaStreamDestroy(d2h);
    }
};
}  // namespace

stq_status stq_decode_steps_host(stq_state *s, int n_steps, const float *h_q, const float *h_k, const float *h_v,
                                 const float *h_alpha, const float *h_beta, float *h_o, void *d_io, size_t io_bytes,
                                 uint64_t seed, uint32_t step, void *stream) {
    if (!s || !h_q || !h_k || !h_v || !h_alpha || !h_beta || !h_o || !d_io || n_steps < 1)
        return STQ_ERR_INVALID_ARG;
    if (!aligned(d_io, 256)) return STQ_ERR_MISALIGNED;
    const IoLayout L = io_layout(s);
    if (io_bytes < 2 * L.total) return STQ_ERR_BUFFER_TOO_SMALL;
    if (overlaps(d_io, 2 * L.total, s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    Pipe P;
    if (!P.ok) return STQ_ERR_CUDA;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t per_vec = L.vec / sizeof(float), per_na = L.na / sizeof(float), per_sc = L.sc / sizeof(float);
    for (int i = 0; i < n_steps; ++i) {
        const int slot = i & 1;
        uint8_t *io = static_cast<uint8_t *>(d_io) + slot * L.total;
        // inputs of step i into the slot, once step i - 2 (the slot's last
        // reader) is done
        if (i >= 2 && cudaStreamWaitEvent(P.h2d, P.step_done[slot], 0) != cudaSuccess) return STQ_ERR_CUDA;
        if (i == 0 && (cudaEventRecord(P.in_ready[1], cs) != cudaSuccess ||
                       cudaStreamWaitEvent(P.h2d, P.in_ready[1], 0) != cudaSuccess))
            return STQ_ERR_CUDA;   // the first copies follow the work already on `stream`
        const struct { size_t off; const void *src; size_t n; } in[5] = {
            {L.q, h_q + i * per_vec, L.vec}, {L.k, h_k + i * per_vec, L.vec}, {L.v, h_v + i * per_vec, L.vec},
            {L.alpha, h_alpha + i * per_na, L.na}, {L.beta, h_beta + i * per_sc, L.sc}};
        for (int j = 0; j < 5; ++j)
            if (cudaMemcpyAsync(io + in[j].off, in[j].src, in[j].n, cudaMemcpyHostToDevice, P.h2d) != cudaSuccess)
                return STQ_ERR_CUDA;
        if (cudaEventRecord(P.in_ready[slot], P.h2d) != cudaSuccess) return STQ_ERR_CUDA;
        // step i, once its inputs are in and the slot's o of step i - 2 is out
        if (cudaStreamWaitEvent(cs, P.in_ready[slot], 0) != cudaSuccess) return STQ_ERR_CUDA;
        if (i >= 2 && cudaStreamWaitEvent(cs, P.out_done[slot], 0) != cudaSuccess) return STQ_ERR_CUDA;
        stq_status st = decode_step(s, nullptr, s->batch, reinterpret_cast<float *>(io + L.q),
                                    reinterpret_cast<float *>(io + L.k), reinterpret_cast<float *>(io + L.v),
                                    reinterpret_cast<float *>(io + L.alpha), reinterpret_cast<float *>(io + L.beta),
                                    reinterpret_cast<float *>(io + L.o), seed, step + (uint32_t)i, stream, false);
        if (st != STQ_OK) return st;
        if (cudaEventRecord(P.step_done[slot], cs) != cudaSuccess) return STQ_ERR_CUDA;
        // o of step i out
        if (cudaStreamWaitEvent(P.d2h, P.step_done[slot], 0) != cudaSuccess) return STQ_ERR_CUDA;
        if (cudaMemcpyAsync(h_o + i * per_vec, io + L.o, L.vec, cudaMemcpyDeviceToHost, P.d2h) != cudaSuccess)
            return STQ_ERR_CUDA;
        if (cudaEventRecord(P.out_done[slot], P.d2h) != cudaSuccess) return STQ_ERR_CUDA;
    }
    // everything of the call precedes later work on `stream`
    for (int slot = 0; slot < 2 && slot < n_steps; ++slot)
        if (cudaStreamWaitEvent(cs, P.out_done[slot], 0) != cudaSuccess) return STQ_ERR_CUDA;
    return STQ_OK;
}

stq_status stq_dequantize_state(const stq_state *s, float *d_S, void *stream) {
    if (!s || !d_S) return STQ_ERR_INVALID_ARG;
    if (!aligned(d_S, 16)) return STQ_ERR_MISALIGNED;
    const size_t nS = (size_t)s->batch * s->heads * kD * kD * sizeof(float);
    if (overlaps(d_S, nS, s->base, state_span(s))) return STQ_ERR_INVALID_ARG;
    cudaError_t err = launch_dequantize(s, d_S, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}

stq_status stq_device_status(stq_state *s, void *stream, int clear) {
    if (!s) return STQ_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(cs) != cudaSuccess) return STQ_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, s->base + s->status_offset, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return STQ_ERR_CUDA;
    if (clear && cudaMemset(s->base + s->status_offset, 0, sizeof(uint32_t)) != cudaSuccess) return STQ_ERR_CUDA;
    if (word & kStatusTimeout) return STQ_ERR_DEVICE_TIMEOUT;
    return (word & kStatusBadSlot) ? STQ_ERR_INVALID_ARG : STQ_OK;
}

stq_status stq_set_wait_limit(stq_state *s, uint64_t limit_ns, int stall_first_wait) {
    if (!s) return STQ_ERR_INVALID_ARG;
    s->wait_limit_ns = limit_ns ? limit_ns : 1000000000ull;
    s->stall_first_wait = stall_first_wait ? 1 : 0;
    return STQ_OK;
}

}  // extern "C"
