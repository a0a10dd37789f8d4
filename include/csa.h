/*
 * csa.h -- C ABI of libcsa: the hybrid compressed attention hot path of DeepSeek-V4 (CSA / HCA)
 * as hand-written CUDA for sm_100a (B200).
 *
 * Sources (page title and section):
 *   [notes]  "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper
 *            notes (jimmysue.github.io), Sec. 2.3 CSA (Eq. 11-12, Eq. 16, Compressor and Indexer
 *            listings) and Sec. 2.4 HCA (Eq. 22-23, Attention.forward listing).
 *   [qa]     itsolotime.com Q&A essay on DeepSeek-V4, Question 1 (sliding window, overlapped
 *            compression, attention sink) and Question 4 (FP4 E2M1, FP8 E4M3).
 *   [ledger] "Mind Observatory: Uncovering the technical ledger of DeepSeek-V4" (RoPE dims of the
 *            KV cache in BF16, the rest in FP8; indexer QK path in FP4).
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is DEVICE memory owned by the caller, unless stated otherwise.  The
 *     library allocates nothing; scratch comes from a caller-provided workspace whose size is
 *     returned by the matching *_workspace_size() call.
 *   - Arrays are row-major and densely packed.  T = tokens, c = KV channels, m = compression
 *     ratio, H = query heads, H_I / d_I = index heads / index head dim, W = window, k = top-k.
 *   - N_vis(t) = floor((t+1)/m) is the number of compressed entries visible to the query at
 *     0-based position t: an entry becomes visible once its last token is at or before t, so a
 *     query never sees the block it is still inside.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only enqueue work and
 *     return immediately; results are ready when the stream reaches them.
 *   - Return value: CSA_OK, or a negative status.  Argument checks run on the host before any
 *     work is enqueued, so an error return means nothing was launched.  CSA_ERR_CUDA means a
 *     launch failed (the CUDA error is left for cudaGetLastError()).  Kernels never trap: a
 *     bounded wait that runs out, or an index the kernel refuses to follow, sets a device error
 *     word that csa_device_error() reads back.
 *   - A call with nothing to compute (no complete block, no rows, no queries, no tokens, no
 *     sequences) runs its argument checks and returns CSA_OK without touching the device.
 *   - dtype codes: CSA_F32 (fp32) and CSA_BF16 (bf16, stored as uint16 bit patterns).
 *   - Numerics: inputs bf16 / fp32 / fp8 / fp4, all accumulation and softmax in fp32.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA_OK 0
#define CSA_ERR_INVALID_ARG (-1)   /* null pointer, bad size, unsupported combination */
#define CSA_ERR_UNSUPPORTED (-2)   /* valid request with no kernel instance (e.g. c % 32 != 0) */
#define CSA_ERR_CUDA (-3)          /* a kernel launch failed */
#define CSA_ERR_WORKSPACE (-5)     /* workspace missing or smaller than *_workspace_size() */

/* device error word bits (csa_device_error) */
#define CSA_DEVERR_TIMEOUT 1       /* a bounded wait ran out */
#define CSA_DEVERR_INDEX 2         /* an out-of-range index was skipped */

#define CSA_F32 0
#define CSA_BF16 1
#define CSA_FP4 2                  /* indexer only: q and keys given as csa_fp4_rows */

/*
 * Mixed-precision KV rows ([ledger]): the last `rope_dims` channels of each row (the RoPE dims;
 * the Indexer listing of [notes] rotates q[..., -rd:]) are kept as bf16, the first
 * c - rope_dims channels as FP8 E4M3 (OCP "fn" variant, max 448) with one fp32 scale per row:
 *   value[j] = e4m3(fp8[r, j]) * scale[r]        for j <  c - rope_dims
 *   value[j] = bf16(rope[r, j - (c-rope_dims)])  for j >= c - rope_dims
 * Planes: fp8 [n, c-rope_dims] bytes, rope [n, rope_dims] bf16 bits, scale [n] fp32.
 * The fp8 and rope plane bases must be 16-byte aligned, the scale plane 4-byte aligned, and
 * (c - rope_dims) and rope_dims multiples of 16 (so any row range of a plane is a valid plane).
 */
typedef struct csa_kv_rows {
    uint8_t *fp8;
    uint16_t *rope;
    float *scale;
    int64_t n;
    int32_t c;
    int32_t rope_dims;
} csa_kv_rows;

/*
 * FP4 rows ([qa] Question 4, [ledger]): E2M1 elements with one E8M0 scale per 32 consecutive
 * elements (OCP MX v1.0 layout): value[j] = e2m1(nibble j) * 2^(scales[r, j/32] - 127).
 * codes [n, d/2] bytes (element 2i in the low nibble of byte i), scales [n, d/32] bytes.
 * d must be a multiple of 32; codes 16-byte aligned, scales 4-byte aligned.
 */
typedef struct csa_fp4_rows {
    uint8_t *codes;
    uint8_t *scales;
    int64_t n;
    int32_t d;
} csa_fp4_rows;

/* ----------------------------------------------------------------------------------------- */

/*
 * csa_compress -- overlapped token-level compression of a CSA layer ([notes] Sec. 2.3,
 * Eq. 11-12 and the Compressor listing; [qa] Question 1 mechanism 2).
 *
 * Entry i (0 <= i < floor(T/m)) pools, per channel d, 2m candidates under ONE softmax:
 *   current block  p = i*m+j:     value Ca[p,d], logit Za[p,d] + B[j,d]
 *   previous block p = (i-1)*m+j: value Cb[p,d], logit Zb[p,d] + B[m+j,d]   (only for i >= 1)
 * so entry 0 pools only its own m tokens, and a trailing partial block is not emitted.
 *
 *   Ca, Cb, Za, Zb  [T, c] in `in_dtype` (CSA_F32 or CSA_BF16)
 *   B               [2m, c] fp32: rows 0..m-1 = B^a (current block), rows m..2m-1 = B^b
 *   T >= 0, 1 <= m <= 64, c a multiple of 4 and <= 2048
 * Outputs (any subset; at least one non-NULL unless floor(T/m) == 0, which writes nothing):
 *   out      [floor(T/m), c] in `out_dtype` (CSA_F32 or CSA_BF16)
 *   out_kv   mixed FP8/BF16 rows (quantise-on-write), out_kv->n >= floor(T/m), ->c == c
 *   out_fp4  FP4 rows (quantise-on-write, for index keys), ->n >= floor(T/m), ->d == c
 * Errors: CSA_ERR_INVALID_ARG for a null input, T < 0, m outside [1, 64], a dtype other than
 * CSA_F32 / CSA_BF16, no output while floor(T/m) > 0, an input or `out` not 16-byte aligned,
 * or an output row struct whose shape or alignment does not match; CSA_ERR_UNSUPPORTED for c
 * not a multiple of 4 in [4, 2048].
 */
int csa_compress(const void *Ca, const void *Cb, const void *Za, const void *Zb, const float *B,
                 int64_t T, int32_t c, int32_t m, int32_t in_dtype, void *out, int32_t out_dtype,
                 const csa_kv_rows *out_kv, const csa_fp4_rows *out_fp4, void *stream);

/*
 * hca_compress -- heavy compression of an HCA layer ([notes] Sec. 2.4, Eq. 22-23): entry i is
 * the per-channel softmax pooling of tokens i*m .. i*m+m-1 with logits Z[p,d] + B[p-i*m,d].
 * No overlap; a trailing partial block is not emitted.
 *   C, Z [T, c] in `in_dtype`;  B [m, c] fp32;  1 <= m <= 1024.
 * Outputs as for csa_compress (out, out_kv; at least one non-NULL).  Errors as for
 * csa_compress, with m outside [1, 1024].
 */
int hca_compress(const void *C, const void *Z, const float *B, int64_t T, int32_t c, int32_t m,
                 int32_t in_dtype, void *out, int32_t out_dtype, const csa_kv_rows *out_kv,
                 void *stream);

/*
 * csa_quantize_kv -- write rows x [n, c] (`in_dtype`) into the mixed FP8/BF16 layout of
 * csa_kv_rows ([ledger]).  Per row: s = amax(|x[0:c-rope]|) / 448 (fp32 division; s = 1 when
 * that is not positive), fp8 = e4m3(x / s) rounded to nearest even and saturated at 448,
 * rope = bf16(x[c-rope:c]) rounded to nearest even.
 * Errors: CSA_ERR_INVALID_ARG for a null x or out, n < 0, a dtype other than CSA_F32 /
 * CSA_BF16, c outside [1, 4096], x not 16-byte aligned, out->rope_dims != rope_dims, or an
 * `out` that does not hold n rows of c channels as described above.
 */
int csa_quantize_kv(const void *x, int32_t in_dtype, int64_t n, int32_t c, int32_t rope_dims,
                    const csa_kv_rows *out, void *stream);

/*
 * csa_quantize_fp4 -- write rows x [n, d] (`in_dtype`) as FP4 rows.  Per block of 32: the scale
 * exponent is the smallest e with amax <= 6 * 2^e (clamped to [-127, 127]; -127 for an all-zero
 * block), element = e2m1(x / 2^e) rounded to nearest even, every zero encoded as +0.
 * Errors: CSA_ERR_INVALID_ARG for a null x, n < 0, a dtype other than CSA_F32 / CSA_BF16, d not
 * a positive multiple of 32, x not 16-byte aligned, or an `out` that does not hold n rows of d.
 */
int csa_quantize_fp4(const void *x, int32_t in_dtype, int64_t n, int32_t d,
                     const csa_fp4_rows *out, void *stream);

/*
 * Decode append path ([qa] Question 5, KV-cache management: the sliding window and the tail
 * tokens of the block still being compressed form a fixed-size "state cache", and the compressed
 * entries live in block-managed pages whose size is the least common multiple of the ratios --
 * 128 tokens for m = 4 and m' = 128, i.e. 32 CSA entries or 1 HCA entry per page; [notes] Sec.
 * 2.3 Compressor listing: the decode branch emits an entry when a block completes).  One call of
 * each per layer and decode step, for a batch of B sequences whose new tokens sit at pos[b] (every
 * earlier token of the sequence must have been appended, in order; pos[b] < 0 skips b).
 *
 * csa_window_append: x [B, c] (in_dtype) are the new tokens' raw KV rows; row b is quantised (as
 * csa_quantize_kv does) into window row b * W + pos[b] % W of `win` (B * W rows): the ring of the
 * last min(pos + 1, W) tokens that hybrid_attn_decode reads with win_len[b] = min(pos[b] + 1, W).
 * Errors: CSA_ERR_INVALID_ARG for a null x or pos, B < 0, a bad dtype, x not 16-byte aligned, W
 * outside [1, 1024] or a `win` that does not hold B * W rows of c; CSA_ERR_UNSUPPORTED for c not a
 * multiple of 4 in [4, 4096].
 *
 * csa_compress_append: the new tokens' compressor rows -- overlap != 0 (CSA, as csa_compress):
 * Ca, Cb, Za, Zb [B, c]; overlap == 0 (HCA, as hca_compress): Ca = C, Za = Z, Cb = Zb = NULL --
 * go to slot pos[b] % L of sequence b's tail ring (tail_* [B, L, c] in in_dtype, L = 2m for CSA,
 * m for HCA; the caller allocates them once and keeps them across steps; HCA uses tail_Ca and
 * tail_Za only).  When pos[b] completes a block ((pos[b] + 1) % m == 0) the entry
 * e = (pos[b] + 1) / m - 1 is pooled from the ring exactly as the prefill compression pools it
 * (same arithmetic, same order: the entries are bit for bit those of csa_compress /
 * hca_compress) and written, quantised, into exactly one of out_kv (FP8/BF16 rows) or out_fp4
 * (FP4 rows, for index keys) at row
 *     pages[b * max_pages + e / page_rows] * page_rows + e % page_rows   (pages != NULL)
 *     comp_off[b] + e                                                       (pages == NULL)
 * A row outside the output, or a page index >= max_pages, is skipped and sets CSA_DEVERR_INDEX.
 * Bias is [2m, c] (CSA) or [m, c] (HCA) fp32, 16-byte aligned; row pointers 8-byte aligned.
 * Errors: CSA_ERR_INVALID_ARG for a null pos or Bias, B < 0, a bad dtype, m outside [1, 64] (CSA)
 * or [1, 1024] (HCA), a missing or misaligned row or tail pointer, not exactly one output, no
 * pages and no comp_off, or an output struct whose shape does not match c; CSA_ERR_UNSUPPORTED for
 * c not a multiple of 4 in [4, 2048].
 */
int csa_window_append(const void *x, int32_t in_dtype, int64_t B, int32_t c, const int64_t *pos, int32_t W,
                      const csa_kv_rows *win, void *stream);
int csa_compress_append(int32_t overlap, int64_t B, const int64_t *pos, int32_t c, int32_t m, int32_t in_dtype,
                        const void *Ca, const void *Cb, const void *Za, const void *Zb, void *tail_Ca,
                        void *tail_Cb, void *tail_Za, void *tail_Zb, const float *Bias, const csa_kv_rows *out_kv,
                        const csa_fp4_rows *out_fp4, const int32_t *pages, int32_t max_pages, int32_t page_rows,
                        const int64_t *comp_off, void *stream);

/*
 * csa_prep_rows -- the per-row transforms between a projection and the caches ([notes] Sec. 2.3:
 * the Compressor listing's RMSNorm of its entries; the Indexer listing's rotary embedding of
 * q[..., -rd:], rotate_activation (Hadamard) and FP4 quantisation, which the indexer's own
 * compressor (rotate=True) applies to its keys as well).  For each row r of x [n, d]:
 *   y = x[r]
 *   y = y / sqrt(mean(y^2) + eps) * g                 when g != NULL (g [d] fp32)
 *   y[d-rd+2i], y[d-rd+2i+1] rotated by the angle      when rd > 0: counter-clockwise by
 *       a = pos[r] * base^(-2i/rd)                     (pos [n] int64 positions)
 *   y = y H_d / sqrt(d)                                when hadamard != 0 (H_d Sylvester Hadamard:
 *                                                      H[j,i] = (-1)^popcount(i & j))
 * and y is written to any subset of out [n, d] (out_dtype), out_kv (FP8/BF16 rows quantised as
 * by csa_quantize_kv, out_kv->rope_dims giving the BF16 part) and out_fp4 (FP4 rows quantised as
 * by csa_quantize_fp4).  fp32 arithmetic, rotation angles in fp64.  Limits: d one of 32, 64,
 * 128, 256, 512; rd even, 0 <= rd <= d; base > 1 when rd > 0.
 * Errors: CSA_ERR_INVALID_ARG for a null x, n < 0, a bad dtype, x or out not 16-byte aligned, rd
 * odd or outside [0, d], rd > 0 without pos or with base <= 1, a g with a negative or non-finite
 * eps, no output, or an output row struct that does not hold n rows of d; CSA_ERR_UNSUPPORTED for
 * another d.
 */
int csa_prep_rows(const void *x, int32_t in_dtype, int64_t n, int32_t d, const float *g, float eps, int32_t rd,
                  const int64_t *pos, double base, int32_t hadamard, void *out, int32_t out_dtype,
                  const csa_kv_rows *out_kv, const csa_fp4_rows *out_fp4, void *stream);

/* ----------------------------------------------------------------------------------------- */

/*
 * indexer_topk -- lightning-indexer scores and per-query top-k ([notes] Sec. 2.3, Eq. 16 and
 * the Indexer listing):
 *   I[r, s] = sum_h w[r,h] * max(0, q[r,h,:] . K[key_off[r] + s, :])   for s < nv(r)
 *   nv(r)   = min(floor((q_pos[r]+1)/m), max_nvis, n_keys - key_off[r])
 * and idx_out[r, :] = the k_eff = min(k, nv(r)) entry indices s with the largest I[r, s],
 * ordered by score descending, equal scores by lower index; slots k_eff..k-1 hold -1.
 * One d_I-dim key per compressed entry is shared by all H_I index heads.
 *
 *   fmt = CSA_F32 / CSA_BF16: q [Nq, H_I, d_I] and keys [n_keys, d_I] dense in that dtype.
 *   fmt = CSA_FP4: q is a `const csa_fp4_rows*` with Nq*H_I rows of d_I (row r*H_I + h), keys
 *                  a `const csa_fp4_rows*` with n_keys rows of d_I.
 *   w        [Nq, H_I] fp32 head weights (any scaling already folded in by the caller)
 *   q_pos    [Nq] int64 absolute 0-based positions, or NULL for q_pos[r] = r (prefill)
 *   key_off  [Nq] int64 first key row of each query's sequence, or NULL for all 0
 *            (FP4 keys: sequences that start at a multiple of 4 rows, in a cache of a multiple of
 *            4 rows, take the faster tile path; any start is correct)
 *   max_nvis host-side upper bound of nv(r) (sizes the score buffer)
 *   idx_out  [Nq, k] int32;  score_out [Nq, k] fp32 scores of the selected entries (or NULL;
 *            -inf in padded slots)
 *   ws       workspace of at least indexer_topk_workspace_size(Nq, max_nvis, k) bytes, queried
 *            with the device current (the FP4 decode path's chunking follows its SM count)
 * Limits: 1 <= k <= 2048, 1 <= H_I <= 128, d_I a multiple of 32 (FP4) or 8 and <= 512.
 * Errors: CSA_ERR_INVALID_ARG for a null q, w, keys or idx_out, Nq < 0, n_keys < 0, m < 1,
 * max_nvis < 0, an unknown fmt, w (or dense q / keys) not 16-byte aligned, or FP4 rows that do
 * not hold Nq*H_I query rows / n_keys key rows of d_I (d_I a multiple of 32);
 * CSA_ERR_UNSUPPORTED for k, H_I or d_I outside the limits or max_nvis > 8,388,480;
 * CSA_ERR_WORKSPACE when Nq > 0 and ws is NULL or smaller than the size above.
 */
size_t indexer_topk_workspace_size(int64_t Nq, int64_t max_nvis, int32_t k);
int indexer_topk(const void *q, const float *w, const void *keys, int32_t fmt,
                 const int64_t *q_pos, const int64_t *key_off, int64_t n_keys, int64_t Nq,
                 int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis,
                 int32_t *idx_out, float *score_out, void *ws, size_t ws_bytes, void *stream);

/*
 * indexer_topk_paged -- indexer_topk (FP4 64 x 128 decode path) over paged index keys: entry s of
 * query r is key row pages[r * max_pages + s / page_rows] * page_rows + s % page_rows of `keys`
 * (a `const csa_fp4_rows*`), in place of key_off[r] + s; nv(r) = min(N_vis(q_pos[r]), max_nvis,
 * max_pages * page_rows).  page_rows must be a power of two in [8, 128] (whole pages per 128-key
 * tile).  A key whose page index or row is out of range gets score -inf and sets
 * CSA_DEVERR_INDEX.  Workspace and results as for indexer_topk; CSA_ERR_UNSUPPORTED for any
 * other shape or page size.
 */
int indexer_topk_paged(const void *q, const float *w, const void *keys, const int64_t *q_pos, int64_t Nq,
                       int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis, const int32_t *pages,
                       int32_t max_pages, int32_t page_rows, int32_t *idx_out, float *score_out, void *ws,
                       size_t ws_bytes, void *stream);

/*
 * csa_topk_merge -- the exact top-k of candidate lists: the last step of an indexer top-k whose
 * keys were scored in shards (one sequence's entries split over several GPUs, each GPU returning
 * its own k best with indexer_topk(score_out), gathered to every GPU).  The lists are stored
 * list-major: scores [n_lists, Nq, list_len] fp32 and idx [n_lists, Nq, list_len] int32, list
 * l's indices offset by bases[l] (int64, or NULL for 0); entries with idx < 0 are ignored.  Per
 * query r, idx_out [Nq, k] gets the k_eff = min(k, valid candidates) indices with the largest
 * scores, ordered by score descending, equal scores by lower index, then -1; score_out [Nq, k] (or
 * NULL) their scores, -inf in padded slots.  The indices of one query must be distinct.  Since
 * every list holds its shard's k best, the merge is the top-k of the whole sequence ([notes] Sec.
 * 2.3 Indexer listing; the pages do not shard the indexer: this is the split of one long sequence
 * across GPUs).  Errors: CSA_ERR_INVALID_ARG for a null array, Nq < 0, n_lists < 1 or
 * list_len < 1; CSA_ERR_UNSUPPORTED for k outside [1, 2048] or n_lists * list_len > 16384.
 */
int csa_topk_merge(const float *scores, const int32_t *idx, const int64_t *bases, int64_t Nq, int32_t n_lists,
                   int32_t list_len, int32_t k, int32_t *idx_out, float *score_out, void *stream);

/*
 * indexer_topk_static -- indexer_topk for callers that cannot allocate device memory (for
 * example runtimes that reserve the device memory for their own pools up front and give plugins
 * no allocator).  The pages have no counterpart: this is a library convenience.
 *
 * Same arguments, semantics, checks and results as indexer_topk, without the workspace: the
 * scratch is a file-scope device array of indexer_topk_static_capacity() = 16 MiB + 256 bytes,
 * which every GPU that loads this library holds until the process exits.  A request is refused
 * with CSA_ERR_SCRATCH_CAPACITY, before anything is launched, when the scratch of the path it
 * takes on this device does not fit: Nq * ceil4(max_nvis) * 4 bytes of scores (plus 256 of
 * alignment) on every path, plus, on the FP4 64 x 128 decode path, the per-chunk candidate
 * lists (at most Nq * 208,128 bytes; 12 sequences at 1M context fit, 16 do not).  No
 * cudaMalloc, cudaFree or allocating library routine is called.  An empty batch (Nq = 0) is
 * checked like any other and returns CSA_OK without touching the device.
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current); make that first call before any stream capture begins.
 *   - All calls on a device share the one array, which keeps the last call's contents.  Nothing
 *     in it needs to start at zero (each call writes every value it reads), but calls whose
 *     kernels overlap on the GPU (different streams without ordering) race on it: serialise them.
 */
#define CSA_ERR_SCRATCH_CAPACITY (-6) /* request exceeds the static scratch of *_static calls */
size_t indexer_topk_static_capacity(void); /* bytes */
int indexer_topk_static(const void *q, const float *w, const void *keys, int32_t fmt,
                        const int64_t *q_pos, const int64_t *key_off, int64_t n_keys, int64_t Nq,
                        int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis,
                        int32_t *idx_out, float *score_out, void *stream);

/* ----------------------------------------------------------------------------------------- */

/*
 * hybrid_attn_prefill -- shared-KV multi-query attention of T query tokens over the union of
 * an uncompressed sliding window and compressed entries, with a per-head sink ([notes]
 * Sec. 2.3 step 3 and Sec. 2.4 Attention.forward listing; [qa] Question 1 mechanisms 1, 3).
 * For query t and head h the keys are, concatenated with no de-duplication:
 *   window:     x_win[u] for u in [max(0, t-W+1), t]      (raw KV rows, the token itself included)
 *   compressed: kv_comp[s] for s in idx[t, :] with s >= 0  (CSA: the indexer's top-k), or for
 *               every s < min(N_vis(t), n_comp) when idx is NULL (HCA: all visible entries)
 * and, with z = scale * q[t,h,:] . key (the key vector is also the value vector),
 *   o[t,h,:] = sum e^z key / (e^{sink[h]} + sum e^z),  lse[t,h] = ln(e^{sink[h]} + sum e^z).
 *
 *   q [T, H, c], x_win [T, c], kv_comp [n_comp, c] in `dtype` (CSA_F32 / CSA_BF16)
 *   idx [T, k] int32 or NULL; negative entries (padding) are skipped; entries >= n_comp, and
 *            entries >= N_vis(t) (a block the query is still inside), are skipped and set
 *            CSA_DEVERR_INDEX
 *   sink [H] fp32 (-inf allowed: no sink);  o [T, H, c] in `dtype`;  lse [T, H] fp32 or NULL
 * Limits: c one of 32, 64, 128, 256, 512; 1 <= H <= 128; 1 <= W <= 1024; 0 <= k <= 4096.
 * Errors: CSA_ERR_INVALID_ARG for a null q, x_win, sink or o, T < 0, n_comp < 0, m < 1, a
 * dtype other than CSA_F32 / CSA_BF16, a NULL kv_comp with n_comp > 0, idx with k outside
 * [0, 4096], a non-finite scale, or q, x_win, kv_comp or o not 16-byte aligned;
 * CSA_ERR_UNSUPPORTED for c, H or W outside the limits.
 */
int hybrid_attn_prefill(const void *q, const void *x_win, const void *kv_comp, int64_t n_comp,
                        const int32_t *idx, int32_t k, const float *sink, float scale, int64_t T,
                        int32_t H, int32_t c, int32_t m, int32_t W, int32_t dtype, void *o,
                        float *lse, void *stream);

/*
 * hybrid_attn_decode -- the same attention for one new token of each of B sequences, reading
 * the mixed-precision caches ([ledger]).
 *   q        [B, H, c] bf16
 *   comp     compressed cache rows of all sequences; sequence b's entry s is row comp_off[b] + s
 *   comp_off [B] int64;  pos [B] int64 position t of the new token (N_vis = floor((t+1)/m))
 *   win      window cache rows, sequence b's rows are b*W .. b*W + win_len[b] - 1, in any order
 *   win_len  [B] int32 in [0, W]
 *   idx      [B, k] int32 compressed-entry indices (CSA, -1 = empty) or NULL (HCA: all
 *            s < min(N_vis, max_nvis)); entries s >= min(N_vis, max_nvis) (not yet visible), or
 *            whose row comp_off[b] + s lies outside comp, are skipped and set CSA_DEVERR_INDEX
 *   o        [B, H, c] bf16;  lse [B, H] fp32 or NULL
 *   ws       workspace of hybrid_attn_decode_workspace_size(...) bytes (split-K partials)
 * Limits: c one of 32, 64, 128, 256, 512; 1 <= H <= 128; 1 <= W <= 1024; 1 <= k <= 4096 with
 * idx; W + (k or max_nvis) <= 2^30.
 * Errors: CSA_ERR_INVALID_ARG for a null q, comp, comp_off, pos, win, win_len, sink or o,
 * B < 0, m < 1, max_nvis < 0, idx with k outside the limits, a non-finite scale, row structs
 * that do not match c (or, for win, hold fewer than B*W rows), or q / o not 16-byte aligned;
 * CSA_ERR_UNSUPPORTED for c, H, W or the key count outside the limits; CSA_ERR_WORKSPACE when
 * ws is NULL or smaller than the size above.
 */
/*
 * hybrid_attn_decode_paged -- hybrid_attn_decode over a paged compressed cache (the block-managed
 * cache of [qa] Question 5; pages of page_rows entries, e.g. 32 CSA entries or 1 HCA entry for
 * 128-token pages): entry s of sequence b is row pages[b * max_pages + s / page_rows] * page_rows
 * + s % page_rows of comp, in place of comp_off[b] + s.  A page index >= max_pages or a row
 * outside comp is skipped and sets CSA_DEVERR_INDEX.  Everything else, the workspace included,
 * is as for hybrid_attn_decode; CSA_ERR_INVALID_ARG also for a null pages, max_pages < 1 or
 * page_rows < 1.
 */
int hybrid_attn_decode_paged(const void *q, const csa_kv_rows *comp, const int32_t *pages, int32_t max_pages,
                             int32_t page_rows, const int64_t *pos, const csa_kv_rows *win, const int32_t *win_len,
                             const int32_t *idx, int32_t k, const float *sink, float scale, int32_t B, int32_t H,
                             int32_t c, int32_t m, int32_t W, int64_t max_nvis, void *o, float *lse, void *ws,
                             size_t ws_bytes, void *stream);

size_t hybrid_attn_decode_workspace_size(int32_t B, int32_t H, int32_t c, int32_t k, int32_t W,
                                         int64_t max_nvis, int32_t use_idx);
int hybrid_attn_decode(const void *q, const csa_kv_rows *comp, const int64_t *comp_off,
                       const int64_t *pos, const csa_kv_rows *win, const int32_t *win_len,
                       const int32_t *idx, int32_t k, const float *sink, float scale, int32_t B,
                       int32_t H, int32_t c, int32_t m, int32_t W, int64_t max_nvis, void *o,
                       float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * csa_decode_glue -- inter-layer projection for a stack of decode layers.  The pages describe a
 * single attention layer and give no counterpart: this is a fixed random projection that turns
 * one layer's attention output into the next layer's queries, so that several layers can run
 * back to back on a decode batch.  Per row r (one row per sequence and head):
 *     y = P o[r],   q_next[r] = bf16( y / rms(y) / sqrt(c) )
 *     z = Rm o[r],  qI rows r = FP4( z / rms(z) )      (index query of a following CSA layer)
 * with rms(v) = sqrt(mean(v^2)); an all-zero y or z gives an all-zero output row.  The FP4 rows
 * use the index-key format of csa_quantize_fp4 (same scale rule, round to nearest even).
 *   o       [R, c] bf16 (R = sequences x heads), 16-byte aligned
 *   P       [c, c] bf16, row i = output channel i (y_i = sum_j P[i,j] o_j), 16-byte aligned
 *   Rm      [d, c] bf16 or NULL when qI is NULL, 16-byte aligned
 *   q_next  [R, c] bf16 out, 16-byte aligned
 *   qI      FP4 rows out (->n >= R, ->d == d) or NULL (next layer has no indexer)
 * fp32 accumulation on the tensor cores.  Limits: c a multiple of 64 in [64, 512]; d a multiple
 * of 32 in [32, 256]; R < 2^31.  Caller-owned memory, nothing allocated; -1 on bad arguments.
 */
int csa_decode_glue(const void *o, const void *P, const void *Rm, int64_t R, int32_t c, int32_t d,
                    void *q_next, const csa_fp4_rows *qI, void *stream);

/* ----------------------------------------------------------------------------------------- */

/*
 * The kernel path that served the calling host thread's last indexer_topk(_static),
 * hybrid_attn_prefill or hybrid_attn_decode call that launched work (CSA_PATH_NONE before any).
 * Dispatch is by shape only: the tensor-core kernels take the 64-head x 512-channel attention
 * and the 64 x 128 indexer shapes, the CUDA-core kernels every other shape the limits allow.
 * A call whose shape belongs to a tensor-core kernel never moves to a CUDA-core one: if that
 * kernel cannot be set up (e.g. no tensor-map encoder), the call returns CSA_ERR_CUDA.
 */
#define CSA_PATH_NONE 0
#define CSA_PATH_INDEXER_FP4_TC 1   /* FP4 64 x 128: tcgen05 kind::mxf4 scan + threshold merge */
#define CSA_PATH_INDEXER_BF16_TC 2  /* bf16 64 x 128 prefill: tcgen05 scores + per-query top-k */
#define CSA_PATH_INDEXER_GENERIC 3  /* any other shape: CUDA-core scores + per-query top-k */
#define CSA_PATH_PREFILL_TC 4       /* bf16 64 x 512, W = 128, CSA (top-k lists): tcgen05, one token on M = 64 */
#define CSA_PATH_PREFILL_GENERIC 5
#define CSA_PATH_DECODE_TC 6        /* 64 x 512: tcgen05 split-K attention + merge */
#define CSA_PATH_DECODE_GENERIC 7
#define CSA_PATH_PREFILL_KEYS_TC 8   /* bf16 64 x 512, W = 128, HCA: tcgen05 with keys on M (M = 128 MMAs) */
int32_t csa_last_path(void);

/*
 * csa_set_wait_limit_ns -- how long the bounded waits of hybrid_attn_decode's tensor-core kernel
 * may wait before they give up (record CSA_DEVERR_TIMEOUT and wind the CTA down), in ns, for the
 * calls launched after it (process-wide); 0 restores the default of 2 s.  Returns the previous
 * limit.  A limit of 1 ns turns every such wait into one non-blocking test that gives up unless
 * its phase has already completed.  The pages have no counterpart: this exists so that a test can
 * make the waits run out on purpose and check that the kernel winds down cleanly (it copies
 * nothing asynchronously into shared memory, and its final drain of its own MMAs always allows
 * the full 2 s) and that the next call is correct.
 */
uint64_t csa_set_wait_limit_ns(uint64_t ns);

/* Synchronise `stream`, return the device error word (CSA_DEVERR_* bits) in *out and clear it. */
int csa_device_error(void *stream, int32_t *out);

/* Static description of a status code. */
const char *csa_status_string(int32_t status);

/* ABI version (major*100 + minor). */
int32_t csa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
