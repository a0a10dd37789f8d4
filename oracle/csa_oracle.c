/*
 * csa_oracle.c -- plain, slow fp64 CPU oracle for the hybrid compressed attention path
 * (CSA / HCA) of DeepSeek-V4.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
 * leg may load this library.  It shares no code, header, table or helper with the CUDA library
 * under compressed_sparse_kv_csa_b200/, and neither side includes or links the other.
 *
 * Sources (cited by page title and section):
 *   [notes]  "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence",
 *            paper notes (jimmysue.github.io): Sec. 2.3 CSA (Eq. 11-12, Eq. 16, Compressor and
 *            Indexer listings), Sec. 2.4 HCA (Eq. 22-23, Attention.forward listing).
 *   [qa]     itsolotime.com Q&A essay on DeepSeek-V4, Question 1 (mechanisms 1-3: sliding
 *            window, overlapped compression, attention sink), Question 4 (FP4 E2M1 / FP8 E4M3).
 *   [ledger] "Mind Observatory: Uncovering the technical ledger of DeepSeek-V4" (mixed-precision
 *            KV cache: RoPE dims BF16, the rest FP8; indexer QK path in FP4).
 *   [ocp8]   OCP 8-bit Floating Point Specification (OFP8), E4M3 encoding.
 *   [ocpmx]  OCP Microscaling Formats (MX) v1.0: FP4 E2M1 element, E8M0 shared scale, block 32.
 *
 * Conventions (all arrays row-major, caller-owned):
 *   T tokens, c channels, m compression ratio, H heads, d head dim, W window, k top-k.
 *   N_vis(t) = floor((t+1)/m): entries visible to the query at 0-based position t.
 *
 * Every floating-point result is fp64 except where a floating-point decision picks an integer
 * code (quantisers): those decisions are taken in fp32, the precision of the storage formats.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------------------ */
/* Token-level compression                                                                     */
/* ------------------------------------------------------------------------------------------ */

/*
 * Overlapped CSA compression, [notes] Sec. 2.3 Eq. 11-12 and the Compressor listing:
 * compressed entry i pools, per channel d, 2m candidates with one softmax over all of them:
 *   current block  p = i*m + j      value Ca[p,d], logit Za[p,d] + Ba[j,d]     (j < m)
 *   previous block p = (i-1)*m + j  value Cb[p,d], logit Zb[p,d] + Bb[j,d]     (j < m, i >= 1)
 * For i = 0 the previous block does not exist; its logits are -inf, so entry 0 pools only its
 * own m tokens.  B is [2m, c]: rows 0..m-1 are B^a, rows m..2m-1 are B^b.
 * out is [floor(T/m), c].
 */
void orc_csa_compress(const double *Ca, const double *Cb, const double *Za, const double *Zb,
                      const double *B, int64_t T, int c, int m, double *out)
{
    int64_t n = T / m;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        double *logit = (double *)malloc(sizeof(double) * 2 * (size_t)m);
        double *val = (double *)malloc(sizeof(double) * 2 * (size_t)m);
        for (int d = 0; d < c; d++) {
            int cnt = 0;
            for (int j = 0; j < m; j++) {
                int64_t p = i * m + j;
                val[cnt] = Ca[p * c + d];
                logit[cnt] = Za[p * c + d] + B[(int64_t)j * c + d];
                cnt++;
            }
            if (i > 0) {
                for (int j = 0; j < m; j++) {
                    int64_t p = (i - 1) * m + j;
                    val[cnt] = Cb[p * c + d];
                    logit[cnt] = Zb[p * c + d] + B[(int64_t)(m + j) * c + d];
                    cnt++;
                }
            }
            double mx = -INFINITY;
            for (int u = 0; u < cnt; u++) mx = logit[u] > mx ? logit[u] : mx;
            double den = 0.0, num = 0.0;
            for (int u = 0; u < cnt; u++) {
                double e = exp(logit[u] - mx);
                den += e;
                num += e * val[u];
            }
            out[i * c + d] = num / den;
        }
        free(logit);
        free(val);
    }
}

/*
 * HCA compression, [notes] Sec. 2.4 Eq. 22-23: no overlap; entry i is the per-channel softmax
 * pooling of tokens i*m .. i*m+m-1 with logits Z[p,d] + B[j,d].  A trailing partial block is not
 * emitted.  B is [m, c]; out is [floor(T/m), c].
 */
void orc_hca_compress(const double *C, const double *Z, const double *B, int64_t T, int c, int m,
                      double *out)
{
    int64_t n = T / m;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        for (int d = 0; d < c; d++) {
            double mx = -INFINITY;
            for (int j = 0; j < m; j++) {
                double z = Z[(i * m + j) * c + d] + B[(int64_t)j * c + d];
                mx = z > mx ? z : mx;
            }
            double den = 0.0, num = 0.0;
            for (int j = 0; j < m; j++) {
                int64_t p = i * m + j;
                double e = exp(Z[p * c + d] + B[(int64_t)j * c + d] - mx);
                den += e;
                num += e * C[p * c + d];
            }
            out[i * c + d] = num / den;
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Lightning indexer and top-k                                                                 */
/* ------------------------------------------------------------------------------------------ */

/*
 * Indexer score, [notes] Sec. 2.3 Eq. 16 and the Indexer listing:
 *   I[r, s] = sum_h w[r,h] * max(0, q[r,h,:] . K[kbase[r] + s, :])   for s < nvis[r].
 * One d-dim key per compressed entry, shared by all H index heads.  Entries s >= nvis[r] are
 * not visible and are left untouched.  S is [Nq, ldS].
 */
void orc_indexer_scores(const double *q, const double *w, const double *K, const int64_t *kbase,
                        const int64_t *nvis, int64_t Nq, int H, int d, int64_t ldS, double *S)
{
    /* every (row, entry) score is independent: parallelise over entries within each row */
    for (int64_t r = 0; r < Nq; r++) {
        const double *qr = q + r * (int64_t)H * d;
#pragma omp parallel for schedule(static)
        for (int64_t s = 0; s < nvis[r]; s++) {
            const double *ks = K + (kbase[r] + s) * (int64_t)d;
            double acc = 0.0;
            for (int h = 0; h < H; h++) {
                double dot = 0.0;
                for (int e = 0; e < d; e++) dot += qr[(int64_t)h * d + e] * ks[e];
                acc += w[r * H + h] * (dot > 0.0 ? dot : 0.0);
            }
            S[r * ldS + s] = acc;
        }
    }
}

typedef struct {
    double score;
    int64_t idx;
} orc_pair;

static int orc_pair_cmp(const void *a, const void *b)
{
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

/*
 * Top-k selection, [notes] Sec. 2.3 Indexer listing: k_eff = min(k, nvis[r]) indices of the
 * largest scores among s < nvis[r], ordered by score descending, equal scores by lower index.
 * Slots k_eff .. k-1 are -1.  idx is [Nq, k].
 */
void orc_topk(const double *S, int64_t ldS, const int64_t *nvis, int64_t Nq, int k, int32_t *idx)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < Nq; r++) {
        int64_t n = nvis[r];
        orc_pair *p = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
        for (int64_t s = 0; s < n; s++) {
            p[s].score = S[r * ldS + s];
            p[s].idx = s;
        }
        qsort(p, (size_t)n, sizeof(orc_pair), orc_pair_cmp);
        int64_t ke = n < k ? n : k;
        for (int64_t j = 0; j < k; j++) idx[r * k + j] = j < ke ? (int32_t)p[j].idx : -1;
        free(p);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Hybrid MQA attention with sink                                                              */
/* ------------------------------------------------------------------------------------------ */

/*
 * Attention of one query row set over explicit key lists, [notes] Sec. 2.3 (shared-KV MQA:
 * the key vector is also the value vector) and Sec. 2.4 Attention.forward listing (window keys
 * and compressed keys concatenated, no de-duplication), [qa] Question 1 mechanism 3 (one
 * learnable sink logit per head, added to the softmax denominator only):
 *   z_j    = scale * q[r,h,:] . P[key_j, :]
 *   o[r,h] = sum_j e^{z_j} P[key_j] / (e^{sink_h} + sum_j e^{z_j})
 *   lse    = ln(e^{sink_h} + sum_j e^{z_j})
 * Keys of row r are keys[off[r] .. off[r+1]-1], row indices into the pool P [*, c].
 * An empty key list gives o = 0 and lse = sink (which may be -inf).
 */
void orc_attn_rows(const double *q, int64_t Nq, int H, int c, const double *P, const int64_t *off,
                   const int64_t *keys, const double *sink, double scale, double *o, double *lse)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < Nq; r++) {
        int64_t nk = off[r + 1] - off[r];
        const int64_t *kl = keys + off[r];
        double *z = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
        for (int h = 0; h < H; h++) {
            const double *qh = q + (r * H + h) * (int64_t)c;
            double *oh = o + (r * H + h) * (int64_t)c;
            double mx = sink[h];
            for (int64_t j = 0; j < nk; j++) {
                const double *kv = P + kl[j] * (int64_t)c;
                double dot = 0.0;
                for (int e = 0; e < c; e++) dot += qh[e] * kv[e];
                z[j] = scale * dot;
                if (z[j] > mx) mx = z[j];
            }
            for (int e = 0; e < c; e++) oh[e] = 0.0;
            if (mx == -INFINITY) { /* no keys and a -inf sink */
                if (lse) lse[r * H + h] = -INFINITY;
                continue;
            }
            double den = exp(sink[h] - mx);
            for (int64_t j = 0; j < nk; j++) {
                double p = exp(z[j] - mx);
                den += p;
                const double *kv = P + kl[j] * (int64_t)c;
                for (int e = 0; e < c; e++) oh[e] += p * kv[e];
            }
            for (int e = 0; e < c; e++) oh[e] /= den;
            if (lse) lse[r * H + h] = mx + log(den);
        }
        free(z);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Storage formats (decisions in fp32)                                                         */
/* ------------------------------------------------------------------------------------------ */

/* Round half to even of a non-negative float holding a value < 2^23. */
static float orc_rne(float x) { return nearbyintf(x); }

/* bf16 bits of x, round to nearest even (finite inputs). */
uint16_t orc_bf16_bits(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16); /* inf / nan passthrough */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

double orc_bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/*
 * FP8 E4M3 (the "fn" variant of [ocp8]: exponent bias 7, no infinities, S.1111.111 is NaN,
 * largest finite 448, smallest normal 2^-6, subnormals j * 2^-9).  Round to nearest even,
 * saturating at 448.
 */
uint8_t orc_e4m3_encode(float v)
{
    uint8_t sign = (v < 0.0f) ? 0x80 : 0x00;
    float a = fabsf(v);
    if (a >= 448.0f) return (uint8_t)(sign | 0x7e);
    uint8_t code;
    if (a < ldexpf(1.0f, -6)) {
        /* subnormal grid j * 2^-9, j = 0..8 (j = 8 is the smallest normal, code 0x08) */
        float j = orc_rne(ldexpf(a, 9));
        code = (uint8_t)j;
    } else {
        int E;
        frexpf(a, &E);        /* a = f * 2^E, f in [0.5, 1) */
        int e = E - 1;        /* a in [2^e, 2^(e+1)), e in [-6, 8] */
        float q = orc_rne(ldexpf(a, 3 - e)); /* 8 .. 16 */
        if (q >= 16.0f) {
            e += 1;
            q = 8.0f;
        }
        code = (uint8_t)(((e + 7) << 3) | ((int)q - 8));
    }
    if ((code & 0x7f) == 0) return 0; /* +0 for every zero */
    return (uint8_t)(sign | code);
}

double orc_e4m3_decode(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 0xf, f = b & 7;
    if (e == 15 && f == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)f, -9) : ldexp(1.0 + f / 8.0, e - 7);
    return s ? -mag : mag;
}

/*
 * FP4 E2M1 element of [ocpmx]: values 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7) and their
 * negatives (sign bit 3).  Round to nearest even, saturating at 6; every zero encodes as +0.
 */
uint8_t orc_e2m1_encode(float v)
{
    float a = fabsf(v);
    int code;
    if (a >= 6.0f) code = 7;
    else if (a < 2.0f) code = (int)orc_rne(a * 2.0f);          /* 0, 0.5, 1, 1.5 grid; 2 -> 4 */
    else if (a < 4.0f) code = (int)orc_rne(a) + 2;              /* 2, 3, 4 -> codes 4, 5, 6 */
    else code = (int)orc_rne(a * 0.5f) + 4;                     /* 4, 6 -> codes 6, 7 */
    if (code == 0) return 0;
    return (uint8_t)(((v < 0.0f) ? 8 : 0) | code);
}

double orc_e2m1_decode(uint8_t b)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = mag[b & 7];
    return (b & 8) ? -v : v;
}

/*
 * Shared E8M0 scale exponent of one FP4 block ([ocpmx] with the scale chosen so that nothing
 * clips): the smallest integer e with amax <= 6 * 2^e, clamped to [-127, 127]; e = -127 when
 * amax = 0.  Decided exactly on the fp32 value of amax.
 */
int orc_fp4_scale_exp(float amax)
{
    if (!(amax > 0.0f)) return -127;
    int E;
    frexpf(amax, &E);
    int e0 = E - 1; /* amax in [2^e0, 2^(e0+1)) */
    int e = (amax <= ldexpf(1.5f, e0)) ? e0 - 2 : e0 - 1;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/*
 * FP4 rows ([ledger]; [qa] Question 4 names E2M1 with 1x32 blocks): x [n, d] fp32, d a multiple
 * of 32.  codes [n, d/2] (element 2j in the low nibble of byte j), scales [n, d/32] as E8M0
 * (biased by 127).
 */
void orc_quant_fp4(const float *x, int64_t n, int d, uint8_t *codes, uint8_t *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        for (int b = 0; b < d / 32; b++) {
            const float *xb = x + r * d + b * 32;
            float amax = 0.0f;
            for (int j = 0; j < 32; j++) amax = fmaxf(amax, fabsf(xb[j]));
            int e = orc_fp4_scale_exp(amax);
            scales[r * (d / 32) + b] = (uint8_t)(e + 127);
            for (int j = 0; j < 32; j += 2) {
                uint8_t lo = orc_e2m1_encode(ldexpf(xb[j], -e));
                uint8_t hi = orc_e2m1_encode(ldexpf(xb[j + 1], -e));
                codes[r * (d / 2) + (b * 32 + j) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* Dequantise FP4 rows to fp64: value = e2m1(code) * 2^(scale - 127). */
void orc_dequant_fp4(const uint8_t *codes, const uint8_t *scales, int64_t n, int d, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        for (int j = 0; j < d; j++) {
            uint8_t byte = codes[r * (d / 2) + j / 2];
            uint8_t nib = (j & 1) ? (byte >> 4) : (byte & 15);
            int e = (int)scales[r * (d / 32) + j / 32] - 127;
            out[r * d + j] = ldexp(orc_e2m1_decode(nib), e);
        }
    }
}

/*
 * Mixed-precision KV rows ([ledger]: RoPE dims kept in BF16, the rest in FP8): x [n, c] fp32.
 * The RoPE dims are the last `rope` channels (the Indexer listing rotates q[..., -rd:]).
 * The first c-rope channels use one fp32 scale per row: s = amax / 448 (s = 1 when that is not
 * positive) and code = e4m3(x / s), IEEE fp32 division.  The RoPE channels are bf16(x).
 * fp8 [n, c-rope], rope_bits [n, rope], scale [n].
 */
void orc_quant_kv(const float *x, int64_t n, int c, int rope, uint8_t *fp8, uint16_t *rope_bits,
                  float *scale)
{
    int cn = c - rope;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        const float *xr = x + r * c;
        float amax = 0.0f;
        for (int j = 0; j < cn; j++) amax = fmaxf(amax, fabsf(xr[j]));
        float s = amax / 448.0f;
        if (!(s > 0.0f)) s = 1.0f;
        scale[r] = s;
        for (int j = 0; j < cn; j++) {
            volatile float qv = xr[j] / s; /* keep the single fp32 division */
            fp8[r * cn + j] = orc_e4m3_encode(qv);
        }
        for (int j = 0; j < rope; j++) rope_bits[r * rope + j] = orc_bf16_bits(xr[cn + j]);
    }
}

/* Dequantise mixed KV rows to fp64: fp8 part e4m3(code) * s, RoPE part bf16 value. */
void orc_dequant_kv(const uint8_t *fp8, const uint16_t *rope_bits, const float *scale, int64_t n,
                    int c, int rope, double *out)
{
    int cn = c - rope;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        for (int j = 0; j < cn; j++) out[r * c + j] = orc_e4m3_decode(fp8[r * cn + j]) * (double)scale[r];
        for (int j = 0; j < rope; j++) out[r * c + cn + j] = orc_bf16_value(rope_bits[r * rope + j]);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Inter-layer glue of the stacked decode workload                                             */
/* ------------------------------------------------------------------------------------------ */

/*
 * The pages do not give this step: it stands in for the model's projections between the
 * attention layers of the stacked decode workload.  For each row r of o [R, c]:
 *   y = P o_r   (P [c, c], row-major as out x in),  q_next_r = y / rms(y) / sqrt(c)
 *   z = Rm o_r  (Rm [d, c]),                          zi_r     = z / rms(z)
 * with rms(v) = sqrt(mean(v^2)); a zero vector maps to zero.  q_next is the next layer's query
 * (before bf16 storage), zi the next CSA layer's index query (before FP4 quantisation).
 */
void orc_decode_glue(const double *o, const double *P, const double *Rm, int64_t R, int c, int d,
                     double *q_next, double *zi)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++) {
        const double *x = o + r * c;
        double ss = 0.0;
        for (int i = 0; i < c; i++) {
            double y = 0.0;
            for (int j = 0; j < c; j++) y += P[(int64_t)i * c + j] * x[j];
            q_next[r * c + i] = y;
            ss += y * y;
        }
        double f = ss > 0.0 ? 1.0 / sqrt(ss / c) / sqrt((double)c) : 0.0;
        for (int i = 0; i < c; i++) q_next[r * c + i] *= f;
        ss = 0.0;
        for (int i = 0; i < d; i++) {
            double z = 0.0;
            for (int j = 0; j < c; j++) z += Rm[(int64_t)i * c + j] * x[j];
            zi[r * d + i] = z;
            ss += z * z;
        }
        f = ss > 0.0 ? 1.0 / sqrt(ss / d) : 0.0;
        for (int i = 0; i < d; i++) zi[r * d + i] *= f;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Layer fidelity: RMSNorm of entries, rotary embedding of the last dims, Hadamard rotation      */
/* ------------------------------------------------------------------------------------------ */

/*
 * RMSNorm of rows, [notes] Sec. 2.3 Compressor listing (self.norm = RMSNorm(head_dim, norm_eps),
 * applied to the compressed entries) with the normalisation written out in the mHC listing
 * (rsqrt(mean(x^2) + eps)):  out[r, j] = x[r, j] / sqrt(mean_j x[r, j]^2 + eps) * g[j].
 */
void orc_rmsnorm(const double *x, const double *g, int64_t n, int d, double eps, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        double ss = 0.0;
        for (int j = 0; j < d; j++) ss += x[r * d + j] * x[r * d + j];
        const double f = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; j++) out[r * d + j] = x[r * d + j] * f * g[j];
    }
}

/*
 * Rotary embedding of the last rd channels of each row, [notes] Sec. 2.3 Indexer listing
 * (apply_rotary_emb(q[..., -rd:], freqs_cis)): inside that slice the channel pairs (2i, 2i+1)
 * rotate by the angle a = pos[r] * base^(-2i/rd):
 *   y[2i] = x[2i] cos a - x[2i+1] sin a,   y[2i+1] = x[2i] sin a + x[2i+1] cos a.
 * The first d - rd channels are copied.
 */
void orc_rope(const double *x, const int64_t *pos, int64_t n, int d, int rd, double base, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        const double *xr = x + r * d;
        double *yr = out + r * d;
        for (int j = 0; j < d - rd; j++) yr[j] = xr[j];
        for (int i = 0; i < rd / 2; i++) {
            const double a = (double)pos[r] * pow(base, -2.0 * i / rd);
            const double x0 = xr[d - rd + 2 * i], x1 = xr[d - rd + 2 * i + 1];
            yr[d - rd + 2 * i] = x0 * cos(a) - x1 * sin(a);
            yr[d - rd + 2 * i + 1] = x0 * sin(a) + x1 * cos(a);
        }
    }
}

/*
 * Hadamard rotation of rows of d = 2^p channels, [notes] Sec. 2.3 Indexer listing
 * (rotate_activation before the FP4 quantisation of the index queries and keys):
 *   out[r, i] = sum_j x[r, j] H[j, i] / sqrt(d),   H[j, i] = (-1)^popcount(i & j)
 * (the Sylvester matrix: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]), written as the plain sum.
 */
void orc_hadamard(const double *x, int64_t n, int d, double *out)
{
    const double s = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        for (int i = 0; i < d; i++) {
            double acc = 0.0;
            for (int j = 0; j < d; j++) acc += (__builtin_popcount((unsigned)(i & j)) & 1) ? -x[r * d + j] : x[r * d + j];
            out[r * d + i] = acc * s;
        }
    }
}
