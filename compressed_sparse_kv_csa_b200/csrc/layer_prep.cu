// layer_prep.cu -- the per-row transforms between the projections and the caches: RMSNorm of the
// compressed entries, rotary embedding of the last rd channels, Hadamard rotation, and the
// quantise-on-write into the cache formats.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3: the Compressor listing normalises its entries with an RMSNorm over the head dim; the
// Indexer listing rotates q[..., -rd:] (apply_rotary_emb), applies rotate_activation (a Hadamard
// transform that spreads outliers) and quantises to FP4; the indexer's own compressor does the
// same to its keys (rotate=True).  Cache formats: FP8 E4M3 + BF16 RoPE rows ("Mind Observatory:
// Uncovering the technical ledger of DeepSeek-V4"), FP4 E2M1 with E8M0 scales per 32 (OCP MX).
//
// One warp per row.  Lane l holds the elements l, l + 32, l + 64, ... (J = d / 32 of them in
// registers), so every 32-element block is one register across the warp: the RMS and the FP8 /
// FP4 scale maxima are warp reductions, the rotary pairs (2i, 2i + 1) are neighbouring lanes, and
// the Hadamard butterflies run over the lane bits with shuffles and over the register index in
// place.  HBM-bound: each row is read once and written once per requested output.
#include "common.cuh"

namespace csa {

namespace {

template <int J, typename Tin>
__global__ void __launch_bounds__(256) prep_rows_kernel(const Tin *x, int64_t n, int d, const float *g, float eps, int rd,
                                                        const int64_t *pos, double log_base, int hadamard, void *out,
                                                        int out_dtype, KvRowsDev kv, bool has_kv, Fp4RowsDev f4,
                                                        bool has_f4)
{
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= n) return;
    float v[J];
#pragma unroll
    for (int j = 0; j < J; ++j) v[j] = ld1<Tin>(x, row * d + 32 * j + lane);
    if (g) { // RMSNorm
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j) ss = fmaf(v[j], v[j], ss);
        ss = warp_sum(ss);
        const float f = 1.f / sqrtf(ss / (float)d + eps);
#pragma unroll
        for (int j = 0; j < J; ++j) v[j] = v[j] * f * __ldg(g + 32 * j + lane);
    }
    if (rd > 0) { // rotary embedding of the last rd channels; angles in fp64
        const int64_t p = pos[row];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int e = 32 * j + lane;
            const float partner = __shfl_xor_sync(0xffffffffu, v[j], 1);
            if (e >= d - rd) {
                const int i = (e - (d - rd)) >> 1;
                const double a = (double)p * exp(-(2.0 * i / rd) * log_base);
                double sn, cs;
                sincos(a, &sn, &cs);
                const float c = (float)cs, s = (float)sn;
                v[j] = (lane & 1) ? fmaf(partner, s, v[j] * c) : fmaf(v[j], c, -partner * s);
            }
        }
    }
    if (hadamard) { // y = x H_d / sqrt(d): butterflies over the lane bits, then over the register index
#pragma unroll
        for (int b = 1; b < 32; b <<= 1) {
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const float o = __shfl_xor_sync(0xffffffffu, v[j], b);
                v[j] = (lane & b) ? o - v[j] : v[j] + o;
            }
        }
#pragma unroll
        for (int s = 1; s < J; s <<= 1) {
#pragma unroll
            for (int j = 0; j < J; ++j) {
                if ((j & s) == 0) {
                    const float a = v[j], b = v[j + s];
                    v[j] = a + b;
                    v[j + s] = a - b;
                }
            }
        }
        const float f = 1.f / sqrtf((float)d);
#pragma unroll
        for (int j = 0; j < J; ++j) v[j] *= f;
    }
    if (out) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            if (out_dtype == CSA_F32) static_cast<float *>(out)[row * d + 32 * j + lane] = v[j];
            else static_cast<uint16_t *>(out)[row * d + 32 * j + lane] = f32_to_bf16_bits(v[j]);
        }
    }
    if (has_kv) { // FP8 E4M3 for the first d - rope channels with one row scale, BF16 for the rest
        const int cn = d - kv.rope_dims;
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j)
            if (32 * j + lane < cn) a = fmaxf(a, fabsf(v[j]));
        a = warp_max(a);
        float sc = __fdiv_rn(a, 448.f);
        if (!(sc > 0.f)) sc = 1.f;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int e = 32 * j + lane;
            if (e < cn) kv.fp8[row * cn + e] = e4m3_encode(__fdiv_rn(v[j], sc));
            else kv.rope[row * kv.rope_dims + (e - cn)] = f32_to_bf16_bits(v[j]);
        }
        if (lane == 0) kv.scale[row] = sc;
    }
    if (has_f4) { // FP4 E2M1, one E8M0 scale per 32-element block (= one register across the warp)
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const float a = warp_max(fabsf(v[j]));
            const int e = fp4_scale_exp(a);
            const float inv = exp2i(-e);
            const float hi = __shfl_down_sync(0xffffffffu, v[j], 1);
            if ((lane & 1) == 0) f4.codes[row * (d / 2) + 16 * j + (lane >> 1)] = e2m1x2_encode(v[j] * inv, hi * inv);
            if (lane == 0) f4.scales[row * (d / 32) + j] = uint8_t(e + 127);
        }
    }
}

template <int J>
cudaError_t launch_j(const void *x, int in_dtype, int64_t n, int d, const float *g, float eps, int rd,
                     const int64_t *pos, double base, int hadamard, void *out, int out_dtype, const KvRowsDev *kv,
                     const Fp4RowsDev *f4, cudaStream_t st)
{
    const unsigned grid = (unsigned)((n + 7) / 8);
    const KvRowsDev k = kv ? *kv : KvRowsDev{};
    const Fp4RowsDev f = f4 ? *f4 : Fp4RowsDev{};
    const double lb = log(base);
    if (in_dtype == CSA_F32)
        prep_rows_kernel<J, float><<<grid, 256, 0, st>>>((const float *)x, n, d, g, eps, rd, pos, lb, hadamard, out,
                                                         out_dtype, k, kv != nullptr, f, f4 != nullptr);
    else
        prep_rows_kernel<J, uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)x, n, d, g, eps, rd, pos, lb, hadamard,
                                                            out, out_dtype, k, kv != nullptr, f, f4 != nullptr);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_prep_rows(const void *x, int in_dtype, int64_t n, int d, const float *g, float eps, int rd,
                             const int64_t *pos, double base, int hadamard, void *out, int out_dtype,
                             const KvRowsDev *kv, const Fp4RowsDev *f4, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    switch (d / 32) {
    case 1: return launch_j<1>(x, in_dtype, n, d, g, eps, rd, pos, base, hadamard, out, out_dtype, kv, f4, st);
    case 2: return launch_j<2>(x, in_dtype, n, d, g, eps, rd, pos, base, hadamard, out, out_dtype, kv, f4, st);
    case 4: return launch_j<4>(x, in_dtype, n, d, g, eps, rd, pos, base, hadamard, out, out_dtype, kv, f4, st);
    case 8: return launch_j<8>(x, in_dtype, n, d, g, eps, rd, pos, base, hadamard, out, out_dtype, kv, f4, st);
    case 16: return launch_j<16>(x, in_dtype, n, d, g, eps, rd, pos, base, hadamard, out, out_dtype, kv, f4, st);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace csa
