// indexer.cu -- lightning-indexer scores, generic path (any H_I, d_I; fp32 / bf16 / FP4).
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 Eq. 16 and the Indexer listing: I[r,s] = sum_h w[r,h] * ReLU(q[r,h,:] . K[s,:]) with one
// key per compressed entry shared by all index heads; only entries s < N_vis(t) are scored.
// FP4 E2M1 operands with E8M0 block scales (Q&A essay on DeepSeek-V4, Question 4; "technical
// ledger" page: the indexer QK path runs in FP4).
//
// One CTA scores KT keys of one query row.  The query row (all heads) is dequantised into shared
// memory once; each thread owns one key, streams it in 8-element chunks and accumulates HG heads
// at a time in registers.  The scores go to a row of the workspace; top-k reads them back.
#include "common.cuh"

namespace csa {

namespace {

constexpr int KT = 128;     // keys per CTA (one per thread)
constexpr int HG = 8;       // heads accumulated per pass
constexpr int QS_MAX = 8192; // floats of the staged query (H_I * d_I)

__device__ __forceinline__ int64_t row_nvis(const IndexerArgs &a, int64_t r)
{
    const int64_t t = a.q_pos ? a.q_pos[r] : r;
    int64_t nv = (t + 1) / a.m;
    if (nv > a.max_nvis) nv = a.max_nvis;
    const int64_t base = a.key_off ? a.key_off[r] : 0;
    if (base < 0) return 0;
    if (nv > a.n_keys - base) nv = a.n_keys - base;
    return nv < 0 ? 0 : nv;
}

// 8 consecutive key elements [e, e+8) of key row `row` as fp32.
template <int FMT>
__device__ __forceinline__ void load_key8(const IndexerArgs &a, int64_t row, int e, float (&k)[8]);

template <>
__device__ __forceinline__ void load_key8<CSA_F32>(const IndexerArgs &a, int64_t row, int e, float (&k)[8])
{
    const float *p = (const float *)a.keys + row * a.d + e;
    float4 x = *reinterpret_cast<const float4 *>(p), y = *reinterpret_cast<const float4 *>(p + 4);
    k[0] = x.x; k[1] = x.y; k[2] = x.z; k[3] = x.w; k[4] = y.x; k[5] = y.y; k[6] = y.z; k[7] = y.w;
}

template <>
__device__ __forceinline__ void load_key8<CSA_BF16>(const IndexerArgs &a, int64_t row, int e, float (&k)[8])
{
    uint4 u = *reinterpret_cast<const uint4 *>((const uint16_t *)a.keys + row * a.d + e);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        k[2 * i] = __uint_as_float(w[i] << 16);
        k[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

template <>
__device__ __forceinline__ void load_key8<CSA_FP4>(const IndexerArgs &a, int64_t row, int e, float (&k)[8])
{
    const uint32_t u = *reinterpret_cast<const uint32_t *>(a.k4.codes + row * (a.d / 2) + e / 2);
    const float s = exp2i(int(a.k4.scales[row * (a.d / 32) + e / 32]) - 127);
#pragma unroll
    for (int i = 0; i < 8; ++i) k[i] = e2m1_decode((u >> (4 * i)) & 15u) * s;
}

template <int FMT>
__global__ void __launch_bounds__(KT) indexer_scores_kernel(IndexerArgs a)
{
    extern __shared__ float qs[]; // [hc][d] staged query heads, then w [H]
    const int64_t r = blockIdx.x;
    const int64_t nv = row_nvis(a, r);
    const int64_t s = (int64_t)blockIdx.y * KT + threadIdx.x;
    if ((int64_t)blockIdx.y * KT >= nv) return; // CTA-uniform
    const int H = a.H, d = a.d;
    const int64_t krow = (a.key_off ? a.key_off[r] : 0) + s;
    const bool act = s < nv;
    const int hc_max = QS_MAX / d < H ? QS_MAX / d : H;
    float *ws = qs + (size_t)hc_max * d;
    for (int h = threadIdx.x; h < H; h += KT) ws[h] = a.w[r * H + h];
    float score = 0.f;
    for (int h0 = 0; h0 < H; h0 += hc_max) {
        const int hc = (H - h0) < hc_max ? (H - h0) : hc_max;
        __syncthreads();
        for (int i = threadIdx.x; i < hc * d; i += KT) {
            const int h = h0 + i / d, e = i % d;
            float v;
            if (FMT == CSA_F32) v = ((const float *)a.q)[(r * H + h) * (int64_t)d + e];
            else if (FMT == CSA_BF16) v = bf16_to_f32(((const uint16_t *)a.q)[(r * H + h) * (int64_t)d + e]);
            else {
                const int64_t qr = r * H + h;
                const uint8_t byte = a.q4.codes[qr * (d / 2) + e / 2];
                v = e2m1_decode((e & 1) ? (byte >> 4) : (byte & 15)) *
                    exp2i(int(a.q4.scales[qr * (d / 32) + e / 32]) - 127);
            }
            qs[i] = v;
        }
        __syncthreads();
        if (!act) continue;
        for (int hg = 0; hg < hc; hg += HG) {
            float acc[HG];
#pragma unroll
            for (int u = 0; u < HG; ++u) acc[u] = 0.f;
            for (int e = 0; e < d; e += 8) {
                float k[8];
                load_key8<FMT>(a, krow, e, k);
#pragma unroll
                for (int u = 0; u < HG; ++u) {
                    if (hg + u < hc) {
                        const float *qh = qs + (size_t)(hg + u) * d + e;
                        float4 x = *reinterpret_cast<const float4 *>(qh);
                        float4 y = *reinterpret_cast<const float4 *>(qh + 4);
                        acc[u] = fmaf(x.x, k[0], acc[u]); acc[u] = fmaf(x.y, k[1], acc[u]);
                        acc[u] = fmaf(x.z, k[2], acc[u]); acc[u] = fmaf(x.w, k[3], acc[u]);
                        acc[u] = fmaf(y.x, k[4], acc[u]); acc[u] = fmaf(y.y, k[5], acc[u]);
                        acc[u] = fmaf(y.z, k[6], acc[u]); acc[u] = fmaf(y.w, k[7], acc[u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < HG; ++u)
                if (hg + u < hc) score = fmaf(ws[h0 + hg + u], fmaxf(acc[u], 0.f), score);
        }
    }
    if (act) a.scores[r * a.ld + s] = score;
}

} // namespace

cudaError_t launch_indexer_scores(const IndexerArgs &a, cudaStream_t st)
{
    if (a.Nq == 0 || a.max_nvis == 0) return cudaSuccess;
    const int hc_max = QS_MAX / a.d < a.H ? QS_MAX / a.d : a.H;
    const size_t smem = ((size_t)hc_max * a.d + a.H) * sizeof(float);
    dim3 grid((unsigned)a.Nq, (unsigned)((a.max_nvis + KT - 1) / KT));
    if (a.fmt == CSA_F32) {
        cudaFuncSetAttribute(indexer_scores_kernel<CSA_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        indexer_scores_kernel<CSA_F32><<<grid, KT, smem, st>>>(a);
    } else if (a.fmt == CSA_BF16) {
        cudaFuncSetAttribute(indexer_scores_kernel<CSA_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        indexer_scores_kernel<CSA_BF16><<<grid, KT, smem, st>>>(a);
    } else {
        cudaFuncSetAttribute(indexer_scores_kernel<CSA_FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        indexer_scores_kernel<CSA_FP4><<<grid, KT, smem, st>>>(a);
    }
    return cudaGetLastError();
}

} // namespace csa
