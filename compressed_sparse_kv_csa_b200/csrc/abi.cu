// abi.cu -- the extern "C" entry points of libcsa: host-side argument checks, workspace
// carving and dispatch to the kernels.  No allocation, no synchronisation (except
// csa_device_error), no CPU fallback: every step of the path runs in this library's kernels.
#include <atomic>
#include <cmath>
#include <cstring>

#include "common.cuh"

namespace csa {
__device__ int g_dev_error = 0;

// Device address of g_dev_error for the current device, looked up once per device; callers on
// several host threads may race on the first lookup, and all of them store the same address.
int *dev_error_word()
{
    static std::atomic<int *> addr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int *a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) return nullptr;
        a = static_cast<int *>(p);
        addr[dev].store(a, std::memory_order_release);
    }
    return a;
}
// SM count of the current device (looked up once per device; 148 when no device answers).
int device_sms()
{
    static std::atomic<int> sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = sms[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
        sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}
cudaError_t launch_attn_prefill_generic(const PrefillArgs &a, cudaStream_t st);
cudaError_t launch_attn_prefill_tc(const PrefillArgs &a, cudaStream_t st, bool *handled, bool *keys_on_m);
cudaError_t launch_indexer_scores_tc(const IndexerArgs &a, cudaStream_t st, bool *handled);
size_t decode_indexer_workspace(int64_t Nq, int64_t max_nvis, int k);
size_t decode_indexer_need(int64_t Nq, int64_t max_nvis, int k);
bool decode_indexer_eligible(const IndexerArgs &a);
cudaError_t launch_indexer_decode(const IndexerArgs &a, void *ws, cudaStream_t st);
void decode_tc_plan(int64_t B, int64_t max_keys, int sms, int *chunk, int *n_chunks);
bool decode_attn_tc_eligible(const DecodeArgs &a);
cudaError_t launch_attn_decode_tc(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_decode_merge(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_decode_glue(const void *o, const void *P, const void *Rm, int64_t R, int c, int d,
                               void *q_next, const Fp4RowsDev *qI, int *err, cudaStream_t st);
} // namespace csa

using namespace csa;

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dtype_ok(int32_t d) { return d == CSA_F32 || d == CSA_BF16; }
inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }
inline int status_of(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }

bool kv_rows_ok(const csa_kv_rows *kv, int64_t n_min, int32_t c)
{
    if (!kv || !kv->fp8 || !kv->scale || kv->c != c || kv->n < n_min) return false;
    if (kv->rope_dims < 0 || kv->rope_dims > c || (kv->rope_dims % 16) || ((c - kv->rope_dims) % 16)) return false;
    if (kv->rope_dims > 0 && (!kv->rope || !aligned16(kv->rope))) return false;
    return aligned16(kv->fp8) && (reinterpret_cast<uintptr_t>(kv->scale) & 3u) == 0;
}

bool fp4_rows_ok(const csa_fp4_rows *f, int64_t n_min, int32_t d)
{
    if (!f || !f->codes || !f->scales || f->d != d || f->n < n_min || (d % 32)) return false;
    return aligned16(f->codes) && (reinterpret_cast<uintptr_t>(f->scales) & 3u) == 0;
}

KvRowsDev to_dev(const csa_kv_rows &k) { return KvRowsDev{k.fp8, k.rope, k.scale, k.n, k.c, k.rope_dims}; }
Fp4RowsDev to_dev(const csa_fp4_rows &f) { return Fp4RowsDev{f.codes, f.scales, f.n, f.d}; }

constexpr size_t kAlign = 256;
inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline int64_t score_ld(int64_t max_nvis) { return (max_nvis + 3) / 4 * 4; }

// The kernel path that served this host thread's last compute call (csa_last_path).
thread_local int32_t t_last_path = CSA_PATH_NONE;

// Limit of the bounded waits of the kernels that take one (csa_set_wait_limit_ns).
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
inline void note_path(int32_t p) { t_last_path = p; }

} // namespace

extern "C" {

int32_t csa_abi_version(void) { return 101; }

int32_t csa_last_path(void) { return t_last_path; }

uint64_t csa_set_wait_limit_ns(uint64_t ns)
{
    return g_wait_ns.exchange(ns ? ns : kDefaultWaitNs);
}

const char *csa_status_string(int32_t s)
{
    switch (s) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case CSA_ERR_CUDA: return "CUDA launch error";
    case CSA_ERR_WORKSPACE: return "workspace missing or too small";
    case CSA_ERR_SCRATCH_CAPACITY: return "request exceeds the static scratch capacity";
    default: return "unknown status";
    }
}

int csa_device_error(void *stream, int32_t *out)
{
    if (!out) return CSA_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(S(stream));
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int));
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int));
    *out = v;
    return status_of(e);
}

// ------------------------------------------------------------------------------------------

int csa_compress(const void *Ca, const void *Cb, const void *Za, const void *Zb, const float *B,
                 int64_t T, int32_t c, int32_t m, int32_t in_dtype, void *out, int32_t out_dtype,
                 const csa_kv_rows *out_kv, const csa_fp4_rows *out_fp4, void *stream)
{
    if (!Ca || !Cb || !Za || !Zb || !B || T < 0 || m < 1 || m > 64 || !dtype_ok(in_dtype))
        return CSA_ERR_INVALID_ARG;
    if (c <= 0 || c % 4 || c > 2048) return CSA_ERR_UNSUPPORTED;
    if (T / m == 0) return CSA_OK; // no complete block: nothing to write
    if (!out && !out_kv && !out_fp4) return CSA_ERR_INVALID_ARG;
    if (out && !dtype_ok(out_dtype)) return CSA_ERR_INVALID_ARG;
    if (!aligned16(B) || !aligned16(Ca) || !aligned16(Cb) || !aligned16(Za) || !aligned16(Zb))
        return CSA_ERR_INVALID_ARG;
    if (out && !aligned16(out)) return CSA_ERR_INVALID_ARG;
    const int64_t n = T / m;
    if (out_kv && !kv_rows_ok(out_kv, n, c)) return CSA_ERR_INVALID_ARG;
    if (out_fp4 && !fp4_rows_ok(out_fp4, n, c)) return CSA_ERR_INVALID_ARG;
    KvRowsDev kv;
    Fp4RowsDev f4;
    if (out_kv) kv = to_dev(*out_kv);
    if (out_fp4) f4 = to_dev(*out_fp4);
    return status_of(launch_compress(true, Ca, Cb, Za, Zb, B, T, c, m, in_dtype, out, out_dtype,
                                     out_kv ? &kv : nullptr, out_fp4 ? &f4 : nullptr, S(stream)));
}

int hca_compress(const void *C, const void *Z, const float *B, int64_t T, int32_t c, int32_t m,
                 int32_t in_dtype, void *out, int32_t out_dtype, const csa_kv_rows *out_kv,
                 void *stream)
{
    if (!C || !Z || !B || T < 0 || m < 1 || m > 1024 || !dtype_ok(in_dtype)) return CSA_ERR_INVALID_ARG;
    if (c <= 0 || c % 4 || c > 2048) return CSA_ERR_UNSUPPORTED;
    if (T / m == 0) return CSA_OK; // no complete block: nothing to write
    if (!out && !out_kv) return CSA_ERR_INVALID_ARG;
    if (out && !dtype_ok(out_dtype)) return CSA_ERR_INVALID_ARG;
    if (!aligned16(B) || !aligned16(C) || !aligned16(Z) || (out && !aligned16(out))) return CSA_ERR_INVALID_ARG;
    const int64_t n = T / m;
    if (out_kv && !kv_rows_ok(out_kv, n, c)) return CSA_ERR_INVALID_ARG;
    KvRowsDev kv;
    if (out_kv) kv = to_dev(*out_kv);
    return status_of(launch_compress(false, C, nullptr, Z, nullptr, B, T, c, m, in_dtype, out,
                                     out_dtype, out_kv ? &kv : nullptr, nullptr, S(stream)));
}

int csa_quantize_kv(const void *x, int32_t in_dtype, int64_t n, int32_t c, int32_t rope_dims,
                    const csa_kv_rows *out, void *stream)
{
    if (!x || n < 0 || !dtype_ok(in_dtype) || c <= 0 || c > 4096 || !aligned16(x)) return CSA_ERR_INVALID_ARG;
    if (!out || out->rope_dims != rope_dims || !kv_rows_ok(out, n, c)) return CSA_ERR_INVALID_ARG;
    return status_of(launch_quantize_kv(x, in_dtype, n, c, rope_dims, to_dev(*out), S(stream)));
}

int csa_quantize_fp4(const void *x, int32_t in_dtype, int64_t n, int32_t d,
                     const csa_fp4_rows *out, void *stream)
{
    if (!x || n < 0 || !dtype_ok(in_dtype) || d <= 0 || d % 32 || !aligned16(x)) return CSA_ERR_INVALID_ARG;
    if (!fp4_rows_ok(out, n, d)) return CSA_ERR_INVALID_ARG;
    return status_of(launch_quantize_fp4(x, in_dtype, n, d, to_dev(*out), S(stream)));
}

int csa_window_append(const void *x, int32_t in_dtype, int64_t B, int32_t c, const int64_t *pos, int32_t W,
                      const csa_kv_rows *win, void *stream)
{
    if (!x || !pos || B < 0 || !dtype_ok(in_dtype) || !aligned16(x) || W < 1 || W > 1024) return CSA_ERR_INVALID_ARG;
    if (c <= 0 || c % 4 || c > 4096) return CSA_ERR_UNSUPPORTED;
    if (!kv_rows_ok(win, B * (int64_t)W, c)) return CSA_ERR_INVALID_ARG;
    if (B == 0) return CSA_OK;
    return status_of(launch_window_append(x, in_dtype, B, c, pos, W, to_dev(*win), S(stream)));
}

int csa_compress_append(int32_t overlap, int64_t B, const int64_t *pos, int32_t c, int32_t m, int32_t in_dtype,
                        const void *Ca, const void *Cb, const void *Za, const void *Zb, void *tail_Ca,
                        void *tail_Cb, void *tail_Za, void *tail_Zb, const float *Bias, const csa_kv_rows *out_kv,
                        const csa_fp4_rows *out_fp4, const int32_t *pages, int32_t max_pages, int32_t page_rows,
                        const int64_t *comp_off, void *stream)
{
    if (!pos || B < 0 || !dtype_ok(in_dtype) || !Bias || !aligned16(Bias)) return CSA_ERR_INVALID_ARG;
    if (m < 1 || m > (overlap ? 64 : 1024)) return CSA_ERR_INVALID_ARG;
    if (c <= 0 || c % 4 || c > 2048) return CSA_ERR_UNSUPPORTED;
    const void *src[4] = {Ca, overlap ? Cb : Za, overlap ? Za : nullptr, overlap ? Zb : nullptr};
    void *tail[4] = {tail_Ca, overlap ? tail_Cb : tail_Za, overlap ? tail_Za : nullptr, overlap ? tail_Zb : nullptr};
    for (int a = 0; a < (overlap ? 4 : 2); ++a)
        if (!src[a] || !tail[a] || (reinterpret_cast<uintptr_t>(src[a]) & 7u) || (reinterpret_cast<uintptr_t>(tail[a]) & 7u))
            return CSA_ERR_INVALID_ARG;
    if (!out_kv == !out_fp4) return CSA_ERR_INVALID_ARG; // exactly one cache
    if (pages ? (max_pages < 1 || page_rows < 1) : !comp_off) return CSA_ERR_INVALID_ARG;
    if (out_kv && !kv_rows_ok(out_kv, 0, c)) return CSA_ERR_INVALID_ARG;
    if (out_fp4 && !fp4_rows_ok(out_fp4, 0, c)) return CSA_ERR_INVALID_ARG;
    if (B == 0) return CSA_OK;
    KvRowsDev kv;
    Fp4RowsDev f4;
    if (out_kv) kv = to_dev(*out_kv);
    if (out_fp4) f4 = to_dev(*out_fp4);
    const int64_t n_out = out_kv ? out_kv->n : out_fp4->n;
    return status_of(launch_compress_append(overlap != 0, B, pos, c, m, in_dtype, src, tail, Bias, out_kv ? &kv : nullptr,
                                            out_fp4 ? &f4 : nullptr, pages, max_pages, page_rows, comp_off, n_out,
                                            dev_error_word(), S(stream)));
}

int csa_prep_rows(const void *x, int32_t in_dtype, int64_t n, int32_t d, const float *g, float eps, int32_t rd,
                  const int64_t *pos, double base, int32_t hadamard, void *out, int32_t out_dtype,
                  const csa_kv_rows *out_kv, const csa_fp4_rows *out_fp4, void *stream)
{
    if (!x || n < 0 || !dtype_ok(in_dtype) || !aligned16(x)) return CSA_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 128 && d != 256 && d != 512) return CSA_ERR_UNSUPPORTED;
    if (rd < 0 || rd > d || (rd & 1) || (rd > 0 && (!pos || !(base > 1.0) || !std::isfinite(base)))) return CSA_ERR_INVALID_ARG;
    if (g && ((reinterpret_cast<uintptr_t>(g) & 3u) || !(eps >= 0.f) || !std::isfinite(eps))) return CSA_ERR_INVALID_ARG;
    if (!out && !out_kv && !out_fp4) return CSA_ERR_INVALID_ARG;
    if (out && (!dtype_ok(out_dtype) || !aligned16(out))) return CSA_ERR_INVALID_ARG;
    if (out_kv && !kv_rows_ok(out_kv, n, d)) return CSA_ERR_INVALID_ARG;
    if (out_fp4 && !fp4_rows_ok(out_fp4, n, d)) return CSA_ERR_INVALID_ARG;
    if (n == 0) return CSA_OK;
    KvRowsDev kv;
    Fp4RowsDev f4;
    if (out_kv) kv = to_dev(*out_kv);
    if (out_fp4) f4 = to_dev(*out_fp4);
    return status_of(launch_prep_rows(x, in_dtype, n, d, g, eps, rd, pos, base, hadamard ? 1 : 0, out, out_dtype,
                                      out_kv ? &kv : nullptr, out_fp4 ? &f4 : nullptr, S(stream)));
}

// ------------------------------------------------------------------------------------------

size_t indexer_topk_workspace_size(int64_t Nq, int64_t max_nvis, int32_t k)
{
    if (Nq < 0 || max_nvis < 0 || k < 0) return 0;
    const size_t dense = round_up((size_t)Nq * (size_t)score_ld(max_nvis) * sizeof(float)) + kAlign;
    const size_t decode = round_up(decode_indexer_workspace(Nq, max_nvis, k)) + kAlign;
    return dense > decode ? dense : decode;
}

} // extern "C"

namespace csa {

// Scratch bytes the path chosen for `a` needs on the current device (the FP4 decode path when it
// is eligible, else the dense score buffer), alignment slack included.
size_t indexer_path_need(const IndexerArgs &a)
{
    if (decode_indexer_eligible(a)) return round_up(decode_indexer_need(a.Nq, a.max_nvis, a.k)) + kAlign;
    return round_up((size_t)a.Nq * (size_t)score_ld(a.max_nvis) * sizeof(float)) + kAlign;
}

// indexer_topk and indexer_topk_static share the argument checks and the launch.  With
// scratch == nullptr the caller's workspace must hold indexer_topk_workspace_size(); otherwise
// `ws_bytes` is the static scratch's size, which must hold the chosen path's need, and
// scratch() supplies its device address (looked up only when there is work to launch).
int indexer_topk_impl(const void *q, const float *w, const void *keys, int32_t fmt, const int64_t *q_pos,
                      const int64_t *key_off, int64_t n_keys, int64_t Nq, int32_t H_I, int32_t d_I, int32_t m,
                      int32_t k, int64_t max_nvis, int32_t *idx_out, float *score_out, void *ws, size_t ws_bytes,
                      void *(*scratch)(cudaError_t *), void *stream, const int32_t *pages, int32_t max_pages,
                      int32_t page_rows)
{
    if (!q || !w || !keys || !idx_out || Nq < 0 || n_keys < 0 || m < 1 || max_nvis < 0)
        return CSA_ERR_INVALID_ARG;
    if (k < 1 || k > 2048 || H_I < 1 || H_I > 128 || d_I < 8 || d_I > 512 || d_I % 8) return CSA_ERR_UNSUPPORTED;
    if (fmt != CSA_F32 && fmt != CSA_BF16 && fmt != CSA_FP4) return CSA_ERR_INVALID_ARG;
    if (max_nvis > (int64_t)65535 * 128) return CSA_ERR_UNSUPPORTED;
    if (!aligned16(w)) return CSA_ERR_INVALID_ARG;
    IndexerArgs a;
    std::memset(&a, 0, sizeof(a));
    a.fmt = fmt;
    a.Nq = Nq;
    a.H = H_I;
    a.d = d_I;
    a.k = k;
    a.max_nvis = max_nvis;
    if (fmt == CSA_FP4) a.k4.n = static_cast<const csa_fp4_rows *>(keys)->n;
    if (!scratch) {
        if (Nq > 0 && (!ws || ws_bytes < indexer_topk_workspace_size(Nq, max_nvis, k))) return CSA_ERR_WORKSPACE;
    } else if (Nq > 0 && indexer_path_need(a) > ws_bytes) {
        return CSA_ERR_SCRATCH_CAPACITY;
    }
    if (fmt == CSA_FP4) {
        const csa_fp4_rows *q4 = (const csa_fp4_rows *)q, *k4 = (const csa_fp4_rows *)keys;
        if (d_I % 32 || !fp4_rows_ok(q4, Nq * H_I, d_I) || !fp4_rows_ok(k4, n_keys, d_I)) return CSA_ERR_INVALID_ARG;
        a.q4 = to_dev(*q4);
        a.k4 = to_dev(*k4);
    } else {
        if (!aligned16(q) || !aligned16(keys)) return CSA_ERR_INVALID_ARG;
        a.q = q;
        a.keys = keys;
    }
    if (Nq == 0) return CSA_OK;
    if (scratch) {
        cudaError_t e = cudaSuccess;
        ws = scratch(&e);
        if (!ws) return CSA_ERR_CUDA;
    }
    a.w = w;
    a.q_pos = q_pos;
    a.key_off = key_off;
    a.n_keys = n_keys;
    a.m = m;
    a.ld = score_ld(max_nvis);
    uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + kAlign - 1) / kAlign * kAlign;
    a.scores = reinterpret_cast<float *>(base);
    a.idx_out = idx_out;
    a.score_out = score_out;
    a.err = dev_error_word();
    a.pages = pages;
    a.max_pages = max_pages;
    a.page_rows = page_rows;
    if (pages && !decode_indexer_eligible(a)) return CSA_ERR_UNSUPPORTED; // paged keys: FP4 64 x 128 only
    if (decode_indexer_eligible(a)) { // FP4, 64 x 128: fused tensor-core scan + chunked top-k
        note_path(CSA_PATH_INDEXER_FP4_TC);
        return status_of(launch_indexer_decode(a, reinterpret_cast<void *>(base), S(stream)));
    }
    bool handled = false;
    cudaError_t e = launch_indexer_scores_tc(a, S(stream), &handled);
    if (!handled) e = launch_indexer_scores(a, S(stream));
    note_path(handled ? CSA_PATH_INDEXER_BF16_TC : CSA_PATH_INDEXER_GENERIC);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    return status_of(launch_topk(a, S(stream)));
}

} // namespace csa

extern "C" {

int csa_topk_merge(const float *scores, const int32_t *idx, const int64_t *bases, int64_t Nq, int32_t n_lists,
                   int32_t list_len, int32_t k, int32_t *idx_out, float *score_out, void *stream)
{
    if (!scores || !idx || !idx_out || Nq < 0 || n_lists < 1 || list_len < 1) return CSA_ERR_INVALID_ARG;
    if (k < 1 || k > 2048 || (int64_t)n_lists * list_len > 16384) return CSA_ERR_UNSUPPORTED;
    if (Nq == 0) return CSA_OK;
    return status_of(launch_topk_merge_lists(scores, idx, bases, Nq, n_lists, list_len, k, idx_out, score_out,
                                             S(stream)));
}

int indexer_topk_paged(const void *q, const float *w, const void *keys, const int64_t *q_pos, int64_t Nq,
                       int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis, const int32_t *pages,
                       int32_t max_pages, int32_t page_rows, int32_t *idx_out, float *score_out, void *ws,
                       size_t ws_bytes, void *stream)
{
    if (!pages || max_pages < 1 || page_rows < 1 || !keys) return CSA_ERR_INVALID_ARG;
    const int64_t n_keys = static_cast<const csa_fp4_rows *>(keys)->n;
    return indexer_topk_impl(q, w, keys, CSA_FP4, q_pos, nullptr, n_keys, Nq, H_I, d_I, m, k, max_nvis, idx_out,
                             score_out, ws, ws_bytes, nullptr, stream, pages, max_pages, page_rows);
}

int indexer_topk(const void *q, const float *w, const void *keys, int32_t fmt,
                 const int64_t *q_pos, const int64_t *key_off, int64_t n_keys, int64_t Nq,
                 int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis,
                 int32_t *idx_out, float *score_out, void *ws, size_t ws_bytes, void *stream)
{
    return indexer_topk_impl(q, w, keys, fmt, q_pos, key_off, n_keys, Nq, H_I, d_I, m, k, max_nvis, idx_out,
                             score_out, ws, ws_bytes, nullptr, stream);
}

// ------------------------------------------------------------------------------------------

int hybrid_attn_prefill(const void *q, const void *x_win, const void *kv_comp, int64_t n_comp,
                        const int32_t *idx, int32_t k, const float *sink, float scale, int64_t T,
                        int32_t H, int32_t c, int32_t m, int32_t W, int32_t dtype, void *o,
                        float *lse, void *stream)
{
    if (!q || !x_win || !sink || !o || T < 0 || n_comp < 0 || m < 1 || !dtype_ok(dtype)) return CSA_ERR_INVALID_ARG;
    if (n_comp > 0 && !kv_comp) return CSA_ERR_INVALID_ARG;
    if (idx && (k < 0 || k > 4096)) return CSA_ERR_INVALID_ARG;
    if (W < 1 || W > 1024 || H < 1 || H > 128) return CSA_ERR_UNSUPPORTED;
    if (c != 32 && c != 64 && c != 128 && c != 256 && c != 512) return CSA_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return CSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(x_win) || (kv_comp && !aligned16(kv_comp)) || !aligned16(o)) return CSA_ERR_INVALID_ARG;
    if (T == 0) return CSA_OK;
    PrefillArgs a{q, x_win, kv_comp, n_comp, idx, idx ? k : 0, sink, scale, T, H, c, m, W, dtype, o, lse,
                  dev_error_word()};
    bool handled = false, keys_on_m = false;
    cudaError_t e = launch_attn_prefill_tc(a, S(stream), &handled, &keys_on_m);
    if (handled) {
        note_path(keys_on_m ? CSA_PATH_PREFILL_KEYS_TC : CSA_PATH_PREFILL_TC);
        return status_of(e);
    }
    note_path(CSA_PATH_PREFILL_GENERIC);
    return status_of(launch_attn_prefill_generic(a, S(stream)));
}

size_t hybrid_attn_decode_workspace_size(int32_t B, int32_t H, int32_t c, int32_t k, int32_t W,
                                         int64_t max_nvis, int32_t use_idx)
{
    if (B <= 0 || H <= 0 || c <= 0) return 0;
    const int64_t max_keys = (int64_t)W + (use_idx ? k : max_nvis);
    if (max_keys > (int64_t)1 << 30) return 0;
    int nc, ch, nc_tc, ch_tc;
    decode_plan(B, H, c, (int)(max_keys > 0 ? max_keys : 1), &nc, &ch);
    decode_tc_plan(B, max_keys > 0 ? max_keys : 1, device_sms(), &ch_tc, &nc_tc); // tensor-core path
    if (nc_tc > nc) nc = nc_tc;
    return round_up((size_t)B * nc * H * (c + 2) * sizeof(float)) + kAlign;
}

} // extern "C"

static int hybrid_attn_decode_impl(const void *q, const csa_kv_rows *comp, const int64_t *comp_off,
                                   const int32_t *pages, int32_t max_pages, int32_t page_rows, const int64_t *pos,
                                   const csa_kv_rows *win, const int32_t *win_len, const int32_t *idx, int32_t k,
                                   const float *sink, float scale, int32_t B, int32_t H, int32_t c, int32_t m,
                                   int32_t W, int64_t max_nvis, void *o, float *lse, void *ws, size_t ws_bytes,
                                   void *stream)
{
    if (!q || !comp || !(comp_off || pages) || !pos || !win || !win_len || !sink || !o || B < 0 || m < 1 || max_nvis < 0)
        return CSA_ERR_INVALID_ARG;
    if (pages && (max_pages < 1 || page_rows < 1)) return CSA_ERR_INVALID_ARG;
    if (idx && (k < 1 || k > 4096)) return CSA_ERR_INVALID_ARG;
    if (W < 1 || W > 1024 || H < 1 || H > 128) return CSA_ERR_UNSUPPORTED;
    if (c != 32 && c != 64 && c != 128 && c != 256 && c != 512) return CSA_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return CSA_ERR_INVALID_ARG;
    if (!kv_rows_ok(comp, 0, c) || !kv_rows_ok(win, (int64_t)B * W, c)) return CSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o)) return CSA_ERR_INVALID_ARG;
    if (B == 0) return CSA_OK;
    const size_t need = hybrid_attn_decode_workspace_size(B, H, c, k, W, max_nvis, idx != nullptr);
    if (need == 0) return CSA_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < need) return CSA_ERR_WORKSPACE;
    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = (const uint16_t *)q;
    a.comp = to_dev(*comp);
    a.win = to_dev(*win);
    a.comp_off = comp_off;
    a.pages = pages;
    a.max_pages = max_pages;
    a.page_rows = page_rows;
    a.pos = pos;
    a.win_len = win_len;
    a.idx = idx;
    a.k = idx ? k : 0;
    a.sink = sink;
    a.scale = scale;
    a.B = B;
    a.H = H;
    a.c = c;
    a.m = m;
    a.W = W;
    a.max_nvis = max_nvis;
    a.o = (uint16_t *)o;
    a.lse = lse;
    a.err = dev_error_word();
    a.wait_ns = g_wait_ns.load();
    const int64_t max_keys = (int64_t)W + (idx ? k : max_nvis);
    uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + kAlign - 1) / kAlign * kAlign;
    a.part = reinterpret_cast<float *>(base);
    decode_tc_plan(B, max_keys, device_sms(), &a.chunk, &a.n_chunks);
    if (decode_attn_tc_eligible(a)) { // 64 heads x 512 channels: tcgen05 split-K + merge
        note_path(CSA_PATH_DECODE_TC);
        cudaError_t e = launch_attn_decode_tc(a, S(stream));
        if (e != cudaSuccess) return CSA_ERR_CUDA;
        return status_of(launch_decode_merge(a, S(stream)));
    }
    note_path(CSA_PATH_DECODE_GENERIC);
    decode_plan(B, H, c, (int)max_keys, &a.n_chunks, &a.chunk);
    return status_of(launch_attn_decode(a, S(stream)));
}

extern "C" {

int hybrid_attn_decode(const void *q, const csa_kv_rows *comp, const int64_t *comp_off,
                       const int64_t *pos, const csa_kv_rows *win, const int32_t *win_len,
                       const int32_t *idx, int32_t k, const float *sink, float scale, int32_t B,
                       int32_t H, int32_t c, int32_t m, int32_t W, int64_t max_nvis, void *o,
                       float *lse, void *ws, size_t ws_bytes, void *stream)
{
    if (!comp_off) return CSA_ERR_INVALID_ARG;
    return hybrid_attn_decode_impl(q, comp, comp_off, nullptr, 0, 0, pos, win, win_len, idx, k, sink, scale, B, H, c, m,
                                   W, max_nvis, o, lse, ws, ws_bytes, stream);
}

int hybrid_attn_decode_paged(const void *q, const csa_kv_rows *comp, const int32_t *pages, int32_t max_pages,
                             int32_t page_rows, const int64_t *pos, const csa_kv_rows *win, const int32_t *win_len,
                             const int32_t *idx, int32_t k, const float *sink, float scale, int32_t B, int32_t H,
                             int32_t c, int32_t m, int32_t W, int64_t max_nvis, void *o, float *lse, void *ws,
                             size_t ws_bytes, void *stream)
{
    if (!pages) return CSA_ERR_INVALID_ARG;
    return hybrid_attn_decode_impl(q, comp, nullptr, pages, max_pages, page_rows, pos, win, win_len, idx, k, sink, scale,
                                   B, H, c, m, W, max_nvis, o, lse, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------------------------------

int csa_decode_glue(const void *o, const void *P, const void *Rm, int64_t R, int32_t c, int32_t d,
                    void *q_next, const csa_fp4_rows *qI, void *stream)
{
    if (!o || !P || !q_next || R < 0 || R >= (1ll << 31)) return CSA_ERR_INVALID_ARG;
    if (c < 64 || c > 512 || c % 64) return CSA_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(P) || !aligned16(q_next)) return CSA_ERR_INVALID_ARG;
    if (qI) {
        if (!Rm || !aligned16(Rm) || d < 32 || d > 256 || d % 32 || !fp4_rows_ok(qI, R, d)) return CSA_ERR_INVALID_ARG;
    }
    if (R == 0) return CSA_OK;
    Fp4RowsDev q4{};
    if (qI) q4 = to_dev(*qI);
    const cudaError_t e = launch_decode_glue(o, P, Rm, R, c, d, q_next, qI ? &q4 : nullptr, dev_error_word(), S(stream));
    if (e == cudaErrorInvalidValue) return CSA_ERR_INVALID_ARG;
    return status_of(e);
}

} // extern "C"
