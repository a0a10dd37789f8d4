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
cudaError_t launch_attn_prefill_generic(const PrefillArgs &a, cudaStream_t st);
cudaError_t launch_attn_prefill_tc(const PrefillArgs &a, cudaStream_t st, bool *handled);
cudaError_t launch_indexer_scores_tc(const IndexerArgs &a, cudaStream_t st, bool *handled);
size_t decode_indexer_workspace(int64_t Nq, int64_t max_nvis, int k);
bool decode_indexer_eligible(const IndexerArgs &a);
cudaError_t launch_indexer_decode(const IndexerArgs &a, void *ws, cudaStream_t st);
int decode_tc_chunks(int64_t max_keys);
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

} // namespace

extern "C" {

int32_t csa_abi_version(void) { return 100; }

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

// ------------------------------------------------------------------------------------------

size_t indexer_topk_workspace_size(int64_t Nq, int64_t max_nvis, int32_t k)
{
    if (Nq < 0 || max_nvis < 0 || k < 0) return 0;
    const size_t dense = round_up((size_t)Nq * (size_t)score_ld(max_nvis) * sizeof(float)) + kAlign;
    const size_t decode = round_up(decode_indexer_workspace(Nq, max_nvis, k)) + kAlign;
    return dense > decode ? dense : decode;
}

int indexer_topk(const void *q, const float *w, const void *keys, int32_t fmt,
                 const int64_t *q_pos, const int64_t *key_off, int64_t n_keys, int64_t Nq,
                 int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis,
                 int32_t *idx_out, float *score_out, void *ws, size_t ws_bytes, void *stream)
{
    if (!q || !w || !keys || !idx_out || Nq < 0 || n_keys < 0 || m < 1 || max_nvis < 0)
        return CSA_ERR_INVALID_ARG;
    if (k < 1 || k > 2048 || H_I < 1 || H_I > 128 || d_I < 8 || d_I > 512 || d_I % 8) return CSA_ERR_UNSUPPORTED;
    if (fmt != CSA_F32 && fmt != CSA_BF16 && fmt != CSA_FP4) return CSA_ERR_INVALID_ARG;
    if (max_nvis > (int64_t)65535 * 128) return CSA_ERR_UNSUPPORTED;
    if (!aligned16(w)) return CSA_ERR_INVALID_ARG;
    const size_t need = indexer_topk_workspace_size(Nq, max_nvis, k);
    if (Nq > 0 && (!ws || ws_bytes < need)) return CSA_ERR_WORKSPACE;
    IndexerArgs a;
    std::memset(&a, 0, sizeof(a));
    a.fmt = fmt;
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
    a.w = w;
    a.q_pos = q_pos;
    a.key_off = key_off;
    a.n_keys = n_keys;
    a.Nq = Nq;
    a.H = H_I;
    a.d = d_I;
    a.m = m;
    a.k = k;
    a.max_nvis = max_nvis;
    a.ld = score_ld(max_nvis);
    uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + kAlign - 1) / kAlign * kAlign;
    a.scores = reinterpret_cast<float *>(base);
    a.idx_out = idx_out;
    a.score_out = score_out;
    if (Nq == 0) return CSA_OK;
    a.err = dev_error_word();
    if (decode_indexer_eligible(a)) // FP4, 64 x 128: fused tensor-core scan + chunked top-k
        return status_of(launch_indexer_decode(a, reinterpret_cast<void *>(base), S(stream)));
    bool handled = false;
    cudaError_t e = launch_indexer_scores_tc(a, S(stream), &handled);
    if (!handled) e = launch_indexer_scores(a, S(stream));
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    return status_of(launch_topk(a, S(stream)));
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
    bool handled = false;
    cudaError_t e = launch_attn_prefill_tc(a, S(stream), &handled);
    if (handled) return status_of(e);
    return status_of(launch_attn_prefill_generic(a, S(stream)));
}

size_t hybrid_attn_decode_workspace_size(int32_t B, int32_t H, int32_t c, int32_t k, int32_t W,
                                         int64_t max_nvis, int32_t use_idx)
{
    if (B <= 0 || H <= 0 || c <= 0) return 0;
    const int64_t max_keys = (int64_t)W + (use_idx ? k : max_nvis);
    if (max_keys > (int64_t)1 << 30) return 0;
    int nc, ch;
    decode_plan(B, H, c, (int)(max_keys > 0 ? max_keys : 1), &nc, &ch);
    const int nc_tc = decode_tc_chunks(max_keys > 0 ? max_keys : 1); // tensor-core path: 128-key chunks
    if (nc_tc > nc) nc = nc_tc;
    return round_up((size_t)B * nc * H * (c + 2) * sizeof(float)) + kAlign;
}

int hybrid_attn_decode(const void *q, const csa_kv_rows *comp, const int64_t *comp_off,
                       const int64_t *pos, const csa_kv_rows *win, const int32_t *win_len,
                       const int32_t *idx, int32_t k, const float *sink, float scale, int32_t B,
                       int32_t H, int32_t c, int32_t m, int32_t W, int64_t max_nvis, void *o,
                       float *lse, void *ws, size_t ws_bytes, void *stream)
{
    if (!q || !comp || !comp_off || !pos || !win || !win_len || !sink || !o || B < 0 || m < 1 || max_nvis < 0)
        return CSA_ERR_INVALID_ARG;
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
    const int64_t max_keys = (int64_t)W + (idx ? k : max_nvis);
    uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + kAlign - 1) / kAlign * kAlign;
    a.part = reinterpret_cast<float *>(base);
    // tensor-core path: items of tpc 128-key tiles, about four items per SM over the whole batch
    // (estimated from the longest key list); one tile per item when the batch is small
    {
        const int64_t tiles = decode_tc_chunks(max_keys);
        int64_t tpc = (int64_t)B * tiles / (4 * 148);
        tpc = tpc < 1 ? 1 : (tpc > 8 ? 8 : tpc);
        a.chunk = (int)(128 * tpc);
        a.n_chunks = (int)((tiles + tpc - 1) / tpc);
    }
    if (decode_attn_tc_eligible(a)) { // 64 heads x 512 channels: tcgen05 split-K + merge
        cudaError_t e = launch_attn_decode_tc(a, S(stream));
        if (e != cudaSuccess) return CSA_ERR_CUDA;
        return status_of(launch_decode_merge(a, S(stream)));
    }
    decode_plan(B, H, c, (int)max_keys, &a.n_chunks, &a.chunk);
    return status_of(launch_attn_decode(a, S(stream)));
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
