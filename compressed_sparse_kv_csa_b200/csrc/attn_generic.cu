// attn_generic.cu -- hybrid MQA attention with sink, generic CUDA-core path (any H, c % 32 == 0,
// fp32 or bf16), for prefill, plus the split-K decode path over the mixed FP8/BF16 caches.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 step 3 (shared-KV MQA: the key vector is also the value vector, all heads share it)
// and Sec. 2.4 Attention.forward listing (sliding-window keys and compressed keys concatenated,
// no de-duplication, one sparse attention over both); itsolotime.com Q&A essay on DeepSeek-V4,
// Question 1, mechanism 1 (window of the most recent 128 raw tokens) and mechanism 3 (one
// learnable sink logit per head in the softmax denominator only).
//
// Prefill: one CTA per query token; 8 warps each own one head per pass.  Keys are gathered in
// tiles of KT rows into shared memory (fp32); each lane owns c/32 channels of the query and of
// the running output and keeps the online softmax (max, sum) of its warp's head.
// Decode: the key list of each sequence is split into chunks; grid = (chunks, sequences); each
// CTA writes (max, sum, unnormalised output) per head to the workspace and a merge kernel folds
// the chunks and the sink.
#include "common.cuh"

namespace csa {

namespace {

constexpr int KT = 32;        // keys per shared-memory tile
constexpr int NWARP = 8;

template <int CPL> struct Online {
    float m, l, acc[CPL];
};

template <int CPL>
__device__ __forceinline__ void online_step(Online<CPL> &st, const float (&q)[CPL], const float *key,
                                            float scale, int lane)
{
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) dot = fmaf(q[i], key[lane + 32 * i], dot);
    dot = warp_sum(dot) * scale;
    const float nm = fmaxf(st.m, dot);
    const float corr = __expf(st.m - nm);
    const float p = __expf(dot - nm);
    st.l = st.l * corr + p;
#pragma unroll
    for (int i = 0; i < CPL; ++i) st.acc[i] = fmaf(p, key[lane + 32 * i], st.acc[i] * corr);
    st.m = nm;
}

// ----------------------------------------------------------------------------------------
// prefill
// ----------------------------------------------------------------------------------------

template <typename Tin, int CPL>
__global__ void __launch_bounds__(NWARP * 32) prefill_generic_kernel(PrefillArgs a)
{
    constexpr int C = CPL * 32;
    extern __shared__ float sm[];
    float *kt = sm;                  // [KT][C]
    int *kvalid = reinterpret_cast<int *>(sm + KT * C);
    const int64_t t = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = a.H;
    const Tin *q = (const Tin *)a.q, *X = (const Tin *)a.x_win, *KV = (const Tin *)a.kv_comp;
    const int64_t w0 = t - a.W + 1 > 0 ? t - a.W + 1 : 0;
    const int n_win = (int)(t - w0 + 1);
    int64_t n_cmp;
    if (a.idx) n_cmp = a.k;
    else {
        n_cmp = (t + 1) / a.m;
        if (n_cmp > a.n_comp) n_cmp = a.n_comp;
    }
    const int64_t n_keys = n_win + n_cmp;

    for (int h0 = 0; h0 < H; h0 += NWARP) {
        const int h = h0 + warp;
        const bool hact = h < H;
        float qv[CPL];
        Online<CPL> st;
        st.m = -INFINITY;
        st.l = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            st.acc[i] = 0.f;
            qv[i] = hact ? ld1<Tin>(q, (t * H + h) * (int64_t)C + lane + 32 * i) : 0.f;
        }
        for (int64_t j0 = 0; j0 < n_keys; j0 += KT) {
            __syncthreads();
            // gather KT key rows
            for (int e = threadIdx.x; e < KT * (C / 4); e += NWARP * 32) {
                const int jj = e / (C / 4), ch = (e % (C / 4)) * 4;
                const int64_t j = j0 + jj;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                int ok = 0;
                if (j < n_win) {
                    v = Ld4<Tin>::at(X, (w0 + j) * C + ch);
                    ok = 1;
                } else if (j < n_keys) {
                    int64_t s;
                    if (a.idx) {
                        s = a.idx[t * a.k + (j - n_win)];
                        if (s >= a.n_comp || s >= (t + 1) / a.m) { // missing, or not yet visible to t
                            if (ch == 0) flag_error(a.err, CSA_DEVERR_INDEX);
                            s = -1;
                        }
                    } else s = j - n_win;
                    if (s >= 0) {
                        v = Ld4<Tin>::at(KV, s * C + ch);
                        ok = 1;
                    }
                }
                *reinterpret_cast<float4 *>(kt + jj * C + ch) = v;
                if (ch == 0) kvalid[jj] = ok;
            }
            __syncthreads();
            if (hact) {
                const int nj = (int)((n_keys - j0) < KT ? (n_keys - j0) : KT);
                for (int jj = 0; jj < nj; ++jj)
                    if (kvalid[jj]) online_step<CPL>(st, qv, kt + jj * C, a.scale, lane);
            }
        }
        if (hact) {
            const float sk = a.sink[h];
            const float mf = fmaxf(st.m, sk);
            float o_scale = 0.f, lse = -INFINITY;
            if (mf > -INFINITY) {
                const float cm = __expf(st.m - mf);
                const float lf = st.l * cm + __expf(sk - mf);
                o_scale = cm / lf;
                lse = mf + __logf(lf);
            }
            Tin *o = (Tin *)a.o;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const float v = st.acc[i] * o_scale;
                const int64_t off = (t * H + h) * (int64_t)C + lane + 32 * i;
                if (sizeof(Tin) == 4) reinterpret_cast<float *>(o)[off] = v;
                else reinterpret_cast<uint16_t *>(o)[off] = f32_to_bf16_bits(v);
            }
            if (a.lse && lane == 0) a.lse[t * H + h] = lse;
        }
    }
}

template <typename Tin, int CPL>
cudaError_t prefill_generic_launch(const PrefillArgs &a, cudaStream_t st)
{
    const size_t smem = (size_t)KT * CPL * 32 * sizeof(float) + KT * sizeof(int);
    auto kern = prefill_generic_kernel<Tin, CPL>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<(unsigned)a.T, NWARP * 32, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t prefill_generic_dispatch(const PrefillArgs &a, cudaStream_t st)
{
    switch (a.c) {
    case 32: return prefill_generic_launch<Tin, 1>(a, st);
    case 64: return prefill_generic_launch<Tin, 2>(a, st);
    case 128: return prefill_generic_launch<Tin, 4>(a, st);
    case 256: return prefill_generic_launch<Tin, 8>(a, st);
    case 512: return prefill_generic_launch<Tin, 16>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

// ----------------------------------------------------------------------------------------
// decode (split-K over the key list, mixed FP8/BF16 rows)
// ----------------------------------------------------------------------------------------

__device__ __forceinline__ float4 kv_row4(const KvRowsDev &kv, int64_t row, int ch)
{
    const int cn = kv.c - kv.rope_dims;
    if (ch < cn) {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(kv.fp8 + row * cn + ch);
        const float s = kv.scale[row];
        return make_float4(e4m3_decode(u & 255) * s, e4m3_decode((u >> 8) & 255) * s,
                           e4m3_decode((u >> 16) & 255) * s, e4m3_decode(u >> 24) * s);
    }
    return Ld4<uint16_t>::at(kv.rope, row * kv.rope_dims + (ch - cn));
}

template <int CPL>
__global__ void __launch_bounds__(NWARP * 32) decode_partial_kernel(DecodeArgs a)
{
    constexpr int C = CPL * 32;
    extern __shared__ float sm[];
    float *kt = sm;
    int *kvalid = reinterpret_cast<int *>(sm + KT * C);
    const int b = blockIdx.y, chunk = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = a.H;
    const int n_win = a.win_len[b] < 0 ? 0 : (a.win_len[b] > a.W ? a.W : a.win_len[b]);
    int64_t n_cmp;
    if (a.idx) n_cmp = a.k;
    else {
        n_cmp = (a.pos[b] + 1) / a.m;
        if (n_cmp > a.max_nvis) n_cmp = a.max_nvis;
        if (n_cmp < 0) n_cmp = 0;
    }
    const int64_t n_keys = n_win + n_cmp;
    const int64_t c0 = (int64_t)chunk * a.chunk;
    const int64_t c1 = (c0 + a.chunk) < n_keys ? (c0 + a.chunk) : n_keys;
    const int64_t cbase = a.pages ? 0 : a.comp_off[b];
    int64_t n_vis = (a.pos[b] + 1) / a.m; // entries of this sequence the new token may see
    if (n_vis > a.max_nvis) n_vis = a.max_nvis;

    // gather key rows j0 .. j0+KT-1 of this sequence's list (dequantised to fp32) into the tile
    auto stage = [&](int64_t j0) {
        for (int e = threadIdx.x; e < KT * (C / 4); e += NWARP * 32) {
            const int jj = e / (C / 4), ch = (e % (C / 4)) * 4;
            const int64_t j = j0 + jj;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            int ok = 0;
            if (j < c1 && j < n_win) { // window row (rows b*W .. b*W+W-1 exist: checked on host)
                v = kv_row4(a.win, (int64_t)b * a.W + j, ch);
                ok = 1;
            } else if (j < c1) {        // compressed entry
                const int64_t s = a.idx ? (int64_t)a.idx[(int64_t)b * a.k + (j - n_win)] : (j - n_win);
                if (s >= 0) {
                    const int64_t row = paged_row(a.pages, a.max_pages, a.page_rows, b, s, cbase);
                    if (s < n_vis && row >= 0 && row < a.comp.n) {
                        v = kv_row4(a.comp, row, ch);
                        ok = 1;
                    } else if (ch == 0) {
                        flag_error(a.err, CSA_DEVERR_INDEX);
                    }
                }
            }
            *reinterpret_cast<float4 *>(kt + jj * C + ch) = v;
            if (ch == 0) kvalid[jj] = ok;
        }
    };
    // a chunk of at most one tile is staged once for all head passes
    const bool single = (c1 - c0) <= KT;
    if (single) {
        stage(c0);
        __syncthreads();
    }
    for (int h0 = 0; h0 < H; h0 += NWARP) {
        const int h = h0 + warp;
        const bool hact = h < H;
        float qv[CPL];
        Online<CPL> st;
        st.m = -INFINITY;
        st.l = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            st.acc[i] = 0.f;
            qv[i] = hact ? bf16_to_f32(a.q[((int64_t)b * H + h) * C + lane + 32 * i]) : 0.f;
        }
        for (int64_t j0 = c0; j0 < c1; j0 += KT) {
            if (!single) {
                __syncthreads();
                stage(j0);
                __syncthreads();
            }
            if (hact) {
                const int nj = (int)((c1 - j0) < KT ? (c1 - j0) : KT);
                for (int jj = 0; jj < nj; ++jj)
                    if (kvalid[jj]) online_step<CPL>(st, qv, kt + jj * C, a.scale, lane);
            }
        }
        if (hact) {
            float *p = a.part + (((int64_t)b * a.n_chunks + chunk) * H + h) * (C + 2);
            if (lane == 0) { p[0] = st.m; p[1] = st.l; }
#pragma unroll
            for (int i = 0; i < CPL; ++i) p[2 + lane + 32 * i] = st.acc[i];
        }
    }
}

// One CTA per (sequence, head): fold the chunks' (max, sum, unnormalised output) and the sink.
// The per-chunk weights e^{m_j - m} / denominator are computed once into shared memory.
constexpr int kMaxMergeChunks = 1024;

__global__ void __launch_bounds__(128) attn_merge_kernel(DecodeArgs a)
{
    __shared__ float fac[kMaxMergeChunks], lsum[kMaxMergeChunks];
    __shared__ float red[8];
    const int bh = blockIdx.x; // b * H + h
    const int b = bh / a.H, h = bh % a.H;
    const int C = a.c, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // only the chunks that hold keys of this sequence (the rest carry weight 0)
    int64_t n_keys;
    {
        const int nw = a.win_len[b] < 0 ? 0 : (a.win_len[b] > a.W ? a.W : a.win_len[b]);
        int64_t ncmp;
        if (a.idx) ncmp = a.k;
        else {
            ncmp = (a.pos[b] + 1) / a.m;
            if (ncmp > a.max_nvis) ncmp = a.max_nvis;
            if (ncmp < 0) ncmp = 0;
        }
        n_keys = nw + ncmp;
    }
    const int nc_all = a.n_chunks;
    const int nc = (int)min((int64_t)nc_all, (n_keys + a.chunk - 1) / a.chunk);
    const float *p0 = a.part + ((int64_t)b * nc_all * a.H + h) * (C + 2);
    const int64_t cstride = (int64_t)a.H * (C + 2);
    // 1. every chunk's (max, sum) in one pass; block max
    float mt = a.sink[h];
    for (int j = tid; j < nc; j += 128) {
        const float2 ml = *reinterpret_cast<const float2 *>(p0 + j * cstride);
        fac[j] = ml.x;
        lsum[j] = ml.y;
        mt = fmaxf(mt, ml.x);
    }
    mt = warp_max(mt);
    if (lane == 0) red[wid] = mt;
    __syncthreads();
    mt = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    // 2. the denominator: chunk sums rescaled to the common max, plus the sink
    float lt = 0.f;
    for (int j = tid; j < nc; j += 128) {
        const float mj = fac[j];
        lt += (mj > -INFINITY) ? lsum[j] * __expf(mj - mt) : 0.f;
    }
    lt = warp_sum(lt);
    __syncthreads();
    if (lane == 0) red[4 + wid] = lt;
    __syncthreads();
    lt = red[4] + red[5] + red[6] + red[7];
    if (mt > -INFINITY) lt += __expf(a.sink[h] - mt);
    const float inv = (mt > -INFINITY && lt > 0.f) ? 1.f / lt : 0.f;
    for (int j = tid; j < nc; j += 128) {
        const float mj = fac[j];
        fac[j] = (mj > -INFINITY) ? __expf(mj - mt) * inv : 0.f;
    }
    __syncthreads();
    // 3. the weighted sum of the chunk outputs, two channels per thread and step
    for (int ch = 2 * tid; ch < C; ch += 256) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int j = 0; j < nc; ++j) { // chunks without keys carry weight 0 and unwritten rows
            const float f = fac[j];
            if (f != 0.f) {
                const float2 v = *reinterpret_cast<const float2 *>(p0 + j * cstride + 2 + ch);
                acc.x = fmaf(v.x, f, acc.x);
                acc.y = fmaf(v.y, f, acc.y);
            }
        }
        *reinterpret_cast<uint32_t *>(a.o + (int64_t)bh * C + ch) =
            uint32_t(f32_to_bf16_bits(acc.x)) | (uint32_t(f32_to_bf16_bits(acc.y)) << 16);
    }
    if (a.lse && tid == 0) a.lse[bh] = (mt > -INFINITY) ? mt + __logf(lt) : -INFINITY;
}

template <int CPL>
cudaError_t decode_launch(const DecodeArgs &a, cudaStream_t st)
{
    const size_t smem = (size_t)KT * CPL * 32 * sizeof(float) + KT * sizeof(int);
    auto kern = decode_partial_kernel<CPL>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<dim3((unsigned)a.n_chunks, (unsigned)a.B), NWARP * 32, smem, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_merge_kernel<<<(unsigned)(a.B * a.H), 128, 0, st>>>(a);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_attn_prefill_generic(const PrefillArgs &a, cudaStream_t st)
{
    if (a.T == 0) return cudaSuccess;
    if (a.dtype == CSA_F32) return prefill_generic_dispatch<float>(a, st);
    return prefill_generic_dispatch<uint16_t>(a, st);
}

void decode_plan(int B, int H, int c, int max_keys, int *n_chunks, int *chunk)
{
    (void)H;
    (void)c;
    const int target = 2 * device_sms(); // two CTAs per SM over the batch
    int nc = (target + B - 1) / (B > 0 ? B : 1);
    const int max_nc = (max_keys + KT - 1) / KT;
    if (nc > max_nc) nc = max_nc;
    if (nc < 1) nc = 1;
    int ch = (max_keys + nc - 1) / nc;
    ch = ((ch + KT - 1) / KT) * KT;
    if (ch < KT) ch = KT;
    *n_chunks = (max_keys + ch - 1) / ch;
    if (*n_chunks < 1) *n_chunks = 1;
    *chunk = ch;
}

cudaError_t launch_decode_merge(const DecodeArgs &a, cudaStream_t st)
{
    if (a.n_chunks > kMaxMergeChunks) return cudaErrorInvalidValue;
    attn_merge_kernel<<<(unsigned)(a.B * a.H), 128, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_attn_decode(const DecodeArgs &a, cudaStream_t st)
{
    if (a.B == 0) return cudaSuccess;
    switch (a.c) {
    case 32: return decode_launch<1>(a, st);
    case 64: return decode_launch<2>(a, st);
    case 128: return decode_launch<4>(a, st);
    case 256: return decode_launch<8>(a, st);
    case 512: return decode_launch<16>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace csa
