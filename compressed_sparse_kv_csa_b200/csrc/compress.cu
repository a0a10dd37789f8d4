// compress.cu -- token-level KV compression (CSA overlapped m=4 and HCA m'=128) with optional
// quantise-on-write into the mixed FP8/BF16 KV layout or FP4 index-key rows.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 (Eq. 11-12, Compressor listing: per-channel softmax over the 2m candidates of the
// current and previous block, learned positional bias) and Sec. 2.4 (Eq. 22-23: HCA, m' tokens,
// no overlap).  Storage formats: "Mind Observatory: Uncovering the technical ledger of
// DeepSeek-V4" (RoPE dims BF16, the rest FP8; indexer keys FP4).
//
// HBM-bound.  Each thread owns 4 consecutive channels of one entry (one 8- or 16-byte load per
// array per token, coalesced across the channel dimension) and keeps an online softmax
// (max, denominator, numerator) per channel in registers.  HCA blocks are long (128 tokens), so
// the tokens of a block are split over TS threads whose partial softmax states are merged in
// shared memory.  Per entry the algorithmic bytes are (2 or 4 arrays) x m x c x sizeof(in).
#include "common.cuh"

namespace csa {

struct CompressParams {
    const void *Ca, *Cb, *Za, *Zb; // HCA: Ca = C, Za = Z, Cb = Zb = null
    const float *B;
    int64_t T, n_entries;
    int c, m;
    bool overlap;
    void *out;
    int out_dtype;
    KvRowsDev kv;
    bool has_kv;
    Fp4RowsDev fp4;
    bool has_fp4;
};

// Where the rows of an entry come from and where the entry goes.  Prefill: entry = the CTA slot,
// token p is row p of the inputs, the entry is row `entry` of the outputs.
struct PrefillRows {
    int64_t n_entries;
    __device__ bool entry(int64_t slot, int64_t &e) const
    {
        e = slot;
        return slot < n_entries;
    }
    __device__ int64_t in_row(int64_t, int64_t p) const { return p; }
    __device__ int64_t out_row(int64_t, int64_t e) const { return e; }
};

// Decode append: slot = sequence b, whose new token sits at position pos[b]; an entry is emitted
// only when that token completes a block ((pos + 1) % m == 0, entry (pos + 1) / m - 1).  Token p
// of sequence b is row b * L + p % L of the tail ring (the last L tokens' compressor rows); the
// entry lands in the sequence's page (pages[b * max_pages + e / page_rows] * page_rows +
// e % page_rows) or at comp_off[b] + e.  An entry whose page slot is missing or beyond the output
// rows is skipped and reported (CSA_DEVERR_INDEX).
struct AppendRows {
    const int64_t *pos;
    int64_t B;
    int m, L;
    const int32_t *pages;
    int max_pages, page_rows;
    const int64_t *comp_off;
    int64_t n_out;
    int *err;
    __device__ bool entry(int64_t b, int64_t &e) const
    {
        if (b >= B) return false;
        const int64_t t = pos[b];
        if (t < 0 || (t + 1) % m != 0) return false;
        e = (t + 1) / m - 1;
        return true;
    }
    __device__ int64_t in_row(int64_t b, int64_t p) const { return b * L + p % L; }
    __device__ int64_t out_row(int64_t b, int64_t e) const
    {
        int64_t r;
        if (pages) {
            const int64_t pg = e / page_rows;
            r = pg < max_pages ? (int64_t)pages[b * max_pages + pg] * page_rows + e % page_rows : -1;
        } else {
            r = comp_off[b] + e;
        }
        if (r < 0 || r >= n_out) {
            flag_error(err, CSA_DEVERR_INDEX);
            return -1;
        }
        return r;
    }
};

struct SoftState {
    float mx[4], den[4], num[4];
};

__device__ __forceinline__ void soft_add(SoftState &s, float4 v, float4 z)
{
    const float vv[4] = {v.x, v.y, v.z, v.w};
    const float zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        float nm = fmaxf(s.mx[u], zz[u]);
        float a = __expf(s.mx[u] - nm);   // rescale of the running sums (0 when empty)
        float e = __expf(zz[u] - nm);
        s.den[u] = s.den[u] * a + e;
        s.num[u] = s.num[u] * a + e * vv[u];
        s.mx[u] = nm;
    }
}

__device__ __forceinline__ void soft_merge(SoftState &s, const float *o)
{
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        float om = o[u], od = o[4 + u], on = o[8 + u];
        float nm = fmaxf(s.mx[u], om);
        if (nm == -INFINITY) continue;
        float a = __expf(s.mx[u] - nm), b = __expf(om - nm);
        s.den[u] = s.den[u] * a + od * b;
        s.num[u] = s.num[u] * a + on * b;
        s.mx[u] = nm;
    }
}

template <typename Tin, typename Rows>
__global__ void __launch_bounds__(512) compress_kernel(CompressParams p, int TS, Rows R)
{
    extern __shared__ float smem[];
    const int TPE = blockDim.x; // channel groups of 4
    const int x = threadIdx.x, y = threadIdx.y, z = threadIdx.z;
    const int64_t slot = (int64_t)blockIdx.x * blockDim.z + z;
    int64_t entry = 0;
    bool valid = R.entry(slot, entry);
    const int ch = 4 * x;
    const int c = p.c, m = p.m;

    SoftState s;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        s.mx[u] = -INFINITY;
        s.den[u] = 0.f;
        s.num[u] = 0.f;
    }
    if (valid) {
        const Tin *Ca = (const Tin *)p.Ca, *Za = (const Tin *)p.Za;
        const int j0 = (int)((int64_t)m * y / TS), j1 = (int)((int64_t)m * (y + 1) / TS);
        for (int j = j0; j < j1; ++j) { // current block
            const int64_t row = R.in_row(slot, entry * m + j);
            float4 v = Ld4<Tin>::at(Ca, row * c + ch);
            float4 zz = Ld4<Tin>::at(Za, row * c + ch);
            float4 b = *reinterpret_cast<const float4 *>(p.B + (int64_t)j * c + ch);
            zz.x += b.x; zz.y += b.y; zz.z += b.z; zz.w += b.w;
            soft_add(s, v, zz);
        }
        if (p.overlap && entry > 0) { // previous block (Cb / Zb, bias rows m..2m-1)
            const Tin *Cb = (const Tin *)p.Cb, *Zb = (const Tin *)p.Zb;
            for (int j = j0; j < j1; ++j) {
                const int64_t row = R.in_row(slot, (entry - 1) * m + j);
                float4 v = Ld4<Tin>::at(Cb, row * c + ch);
                float4 zz = Ld4<Tin>::at(Zb, row * c + ch);
                float4 b = *reinterpret_cast<const float4 *>(p.B + (int64_t)(m + j) * c + ch);
                zz.x += b.x; zz.y += b.y; zz.z += b.z; zz.w += b.w;
                soft_add(s, v, zz);
            }
        }
    }
    // output row of the entry (the policy may refuse it: nothing is written then)
    int64_t orow = 0;
    if (valid && y == 0 && x == 0) orow = R.out_row(slot, entry);
    // merge the token splits
    float *part = smem;                                       // [EPC][TS][TPE][12]
    int *amax_s = reinterpret_cast<int *>(smem + (size_t)blockDim.z * TS * TPE * 12); // [EPC]
    if (TS > 1) {
        float *mine = part + (((size_t)z * TS + y) * TPE + x) * 12;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            mine[u] = s.mx[u];
            mine[4 + u] = s.den[u];
            mine[8 + u] = s.num[u];
        }
    }
    int64_t *orow_s = reinterpret_cast<int64_t *>(amax_s + 2 * blockDim.z); // [EPC], 8-byte aligned
    if (x == 0 && y == 0) {
        amax_s[z] = 0;
        orow_s[z] = orow;
    }
    __syncthreads();
    orow = orow_s[z];
    if (orow < 0) valid = false;
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (y == 0) {
        for (int yy = 1; yy < TS; ++yy) soft_merge(s, part + (((size_t)z * TS + yy) * TPE + x) * 12);
        val = make_float4(s.num[0] / s.den[0], s.num[1] / s.den[1], s.num[2] / s.den[2],
                          s.num[3] / s.den[3]);
        if (valid && p.out) {
            if (p.out_dtype == CSA_F32) st4<float>((float *)p.out, orow * c + ch, val);
            else st4<uint16_t>((uint16_t *)p.out, orow * c + ch, val);
        }
        if (valid && p.has_kv && ch < c - p.kv.rope_dims) {
            float a = fmaxf(fmaxf(fabsf(val.x), fabsf(val.y)), fmaxf(fabsf(val.z), fabsf(val.w)));
            atomicMax(&amax_s[z], __float_as_int(a));
        }
    }
    __syncthreads();
    // y != 0 is warp-uniform (token splits only when a warp holds channels of one split), and
    // invalid entries stay in the warp so the FP4 shuffles below see every lane.
    if (y != 0) return;
    if (p.has_kv && valid) {
        const int cn = c - p.kv.rope_dims;
        if (ch < cn) {
            float amax = __int_as_float(amax_s[z]);
            float sc = __fdiv_rn(amax, 448.f);
            if (!(sc > 0.f)) sc = 1.f;
            uint32_t w = uint32_t(e4m3_encode(__fdiv_rn(val.x, sc))) |
                         (uint32_t(e4m3_encode(__fdiv_rn(val.y, sc))) << 8) |
                         (uint32_t(e4m3_encode(__fdiv_rn(val.z, sc))) << 16) |
                         (uint32_t(e4m3_encode(__fdiv_rn(val.w, sc))) << 24);
            *reinterpret_cast<uint32_t *>(p.kv.fp8 + orow * cn + ch) = w;
            if (x == 0) p.kv.scale[orow] = sc;
        } else {
            const int rd = p.kv.rope_dims;
            st4<uint16_t>(p.kv.rope, orow * rd + (ch - cn), val);
        }
    }
    if (p.has_fp4) {
        // block of 32 channels = 8 consecutive threads of one warp
        float a = fmaxf(fmaxf(fabsf(val.x), fabsf(val.y)), fmaxf(fabsf(val.z), fabsf(val.w)));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
        const int e = fp4_scale_exp(a);
        const float inv = exp2i(-e);
        uint16_t two = uint16_t(e2m1x2_encode(val.x * inv, val.y * inv)) |
                       (uint16_t(e2m1x2_encode(val.z * inv, val.w * inv)) << 8);
        if (valid) {
            *reinterpret_cast<uint16_t *>(p.fp4.codes + orow * (c / 2) + ch / 2) = two;
            if ((x & 7) == 0) p.fp4.scales[orow * (c / 32) + ch / 32] = uint8_t(e + 127);
        }
    }
}

// Block shape of the compression kernel: TPE = c / 4 threads per entry along the channels, TS
// token splits for long HCA blocks, EPC entries per CTA.  The append path uses the same shape for
// the same (overlap, c, m), so its entries are computed in the same order, bit for bit.
static void compress_shape(bool overlap, int c, int m, int64_t n_entries, int *TS_, int *EPC_)
{
    const int TPE = c / 4;
    int TS = 1;
    if (!overlap && TPE >= 32) { // long HCA blocks: split the tokens of a block over threads
        while (TS * 2 * TPE <= 512 && TS * 2 <= m && m / (TS * 2) >= 8) TS *= 2;
    }
    // whole warps only (the FP4 path shuffles with a full mask); extra entries are invalid lanes
    int EPC = (TPE * TS >= 32) ? 1 : 32 / (TPE * TS);
    while (EPC * 2 * TPE * TS <= 256 && EPC * 2 <= n_entries) EPC *= 2;
    *TS_ = TS;
    *EPC_ = EPC;
}

static size_t compress_smem(int EPC, int TS, int TPE)
{
    return (size_t)EPC * TS * TPE * 12 * sizeof(float) + (size_t)EPC * 2 * sizeof(int) + (size_t)EPC * sizeof(int64_t);
}

cudaError_t launch_compress(bool overlap, const void *Ca, const void *Cb, const void *Za,
                            const void *Zb, const float *B, int64_t T, int c, int m, int in_dtype,
                            void *out, int out_dtype, const KvRowsDev *kv, const Fp4RowsDev *fp4,
                            cudaStream_t st)
{
    CompressParams p;
    p.Ca = Ca; p.Cb = Cb; p.Za = Za; p.Zb = Zb; p.B = B;
    p.T = T; p.n_entries = T / m; p.c = c; p.m = m; p.overlap = overlap;
    p.out = out; p.out_dtype = out_dtype;
    p.has_kv = kv != nullptr;
    if (kv) p.kv = *kv;
    p.has_fp4 = fp4 != nullptr;
    if (fp4) p.fp4 = *fp4;
    if (p.n_entries == 0) return cudaSuccess;
    const int TPE = c / 4;
    int TS, EPC;
    compress_shape(overlap, c, m, p.n_entries, &TS, &EPC);
    dim3 block(TPE, TS, EPC);
    const int64_t grid = (p.n_entries + EPC - 1) / EPC;
    const size_t smem = compress_smem(EPC, TS, TPE);
    const PrefillRows R{p.n_entries};
    if (in_dtype == CSA_F32)
        compress_kernel<float, PrefillRows><<<(unsigned)grid, block, smem, st>>>(p, TS, R);
    else
        compress_kernel<uint16_t, PrefillRows><<<(unsigned)grid, block, smem, st>>>(p, TS, R);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// decode append: tail ring of the compressor inputs, block completion, window ring
// ------------------------------------------------------------------------------------------

// Copy the new token's compressor rows (narr arrays of [B, c]) into slot pos[b] % L of sequence b's
// tail ring ([B, L, c] per array).  8-byte moves (c a multiple of 4; bf16 rows are 8-byte aligned).
template <typename T>
__global__ void tail_one_kernel(const T *src, T *dst, const int64_t *pos, int c, int L)
{
    const int64_t b = blockIdx.x;
    const int64_t t = pos[b];
    if (t < 0) return;
    const T *s = src + b * c;
    T *d = dst + (b * L + t % L) * c;
    constexpr int V = 8 / sizeof(T);
    for (int i = threadIdx.x * V; i < c; i += blockDim.x * V)
        *reinterpret_cast<uint2 *>(d + i) = *reinterpret_cast<const uint2 *>(s + i);
}

cudaError_t launch_compress_append(bool overlap, int64_t B, const int64_t *pos, int c, int m, int in_dtype,
                                   const void *const new_rows[4], void *const tail[4], const float *Bias,
                                   const KvRowsDev *kv, const Fp4RowsDev *fp4, const int32_t *pages, int max_pages,
                                   int page_rows, const int64_t *comp_off, int64_t n_out, int *err, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    const int narr = overlap ? 4 : 2;
    const int L = overlap ? 2 * m : m;
    // 1. the new tokens into the tail rings, one launch per array
    for (int a = 0; a < narr; ++a) {
        if (in_dtype == CSA_F32)
            tail_one_kernel<float><<<(unsigned)B, 128, 0, st>>>((const float *)new_rows[a], (float *)tail[a], pos, c, L);
        else
            tail_one_kernel<uint16_t><<<(unsigned)B, 128, 0, st>>>((const uint16_t *)new_rows[a], (uint16_t *)tail[a], pos, c,
                                                                   L);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // 2. the entries completed by the new tokens, computed exactly as the prefill compression does
    CompressParams p;
    p.Ca = tail[0];
    p.Cb = overlap ? tail[1] : nullptr;
    p.Za = overlap ? tail[2] : tail[1];
    p.Zb = overlap ? tail[3] : nullptr;
    p.B = Bias;
    p.T = 0;
    p.n_entries = B;
    p.c = c;
    p.m = m;
    p.overlap = overlap;
    p.out = nullptr;
    p.out_dtype = 0;
    p.has_kv = kv != nullptr;
    if (kv) p.kv = *kv;
    p.has_fp4 = fp4 != nullptr;
    if (fp4) p.fp4 = *fp4;
    const int TPE = c / 4;
    int TS, EPC;
    compress_shape(overlap, c, m, B, &TS, &EPC);
    dim3 block(TPE, TS, EPC);
    const int64_t grid = (B + EPC - 1) / EPC;
    const size_t smem = compress_smem(EPC, TS, TPE);
    const AppendRows R{pos, B, m, L, pages, max_pages, page_rows, comp_off, n_out, err};
    if (in_dtype == CSA_F32)
        compress_kernel<float, AppendRows><<<(unsigned)grid, block, smem, st>>>(p, TS, R);
    else
        compress_kernel<uint16_t, AppendRows><<<(unsigned)grid, block, smem, st>>>(p, TS, R);
    return cudaGetLastError();
}

// The new tokens' raw KV rows into the window rings: row x[b] -> window row b * W + pos[b] % W,
// quantised exactly as csa_quantize_kv quantises a row.  One warp per row.
template <typename Tin>
__global__ void window_append_kernel(const Tin *x, int64_t B, int c, const int64_t *pos, int W, KvRowsDev out)
{
    const int64_t b = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (b >= B || pos[b] < 0) return;
    const int64_t row = b * W + pos[b] % W;
    const int rope = out.rope_dims, cn = c - rope;
    float a = 0.f;
    for (int j = lane * 4; j < cn; j += 128) {
        float4 v = Ld4<Tin>::at(x, b * c + j);
        a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    a = warp_max(a);
    float sc = __fdiv_rn(a, 448.f);
    if (!(sc > 0.f)) sc = 1.f;
    for (int j = lane * 4; j < cn; j += 128) {
        float4 v = Ld4<Tin>::at(x, b * c + j);
        uint32_t w = uint32_t(e4m3_encode(__fdiv_rn(v.x, sc))) | (uint32_t(e4m3_encode(__fdiv_rn(v.y, sc))) << 8) |
                     (uint32_t(e4m3_encode(__fdiv_rn(v.z, sc))) << 16) |
                     (uint32_t(e4m3_encode(__fdiv_rn(v.w, sc))) << 24);
        *reinterpret_cast<uint32_t *>(out.fp8 + row * cn + j) = w;
    }
    for (int j = lane * 4; j < rope; j += 128) st4<uint16_t>(out.rope, row * rope + j, Ld4<Tin>::at(x, b * c + cn + j));
    if (lane == 0) out.scale[row] = sc;
}

cudaError_t launch_window_append(const void *x, int in_dtype, int64_t B, int c, const int64_t *pos, int W,
                                 const KvRowsDev &out, cudaStream_t st)
{
    if (B == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((B + 7) / 8);
    if (in_dtype == CSA_F32) window_append_kernel<float><<<grid, 256, 0, st>>>((const float *)x, B, c, pos, W, out);
    else window_append_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)x, B, c, pos, W, out);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// standalone quantisers (window rows, index queries)
// ------------------------------------------------------------------------------------------

template <typename Tin>
__global__ void quantize_kv_kernel(const Tin *x, int64_t n, int c, int rope, KvRowsDev out)
{
    // one warp per row
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (row >= n) return;
    const int cn = c - rope;
    float a = 0.f;
    for (int j = lane * 4; j < cn; j += 128) {
        float4 v = Ld4<Tin>::at(x, row * c + j);
        a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    a = warp_max(a);
    float sc = __fdiv_rn(a, 448.f);
    if (!(sc > 0.f)) sc = 1.f;
    for (int j = lane * 4; j < cn; j += 128) {
        float4 v = Ld4<Tin>::at(x, row * c + j);
        uint32_t w = uint32_t(e4m3_encode(__fdiv_rn(v.x, sc))) |
                     (uint32_t(e4m3_encode(__fdiv_rn(v.y, sc))) << 8) |
                     (uint32_t(e4m3_encode(__fdiv_rn(v.z, sc))) << 16) |
                     (uint32_t(e4m3_encode(__fdiv_rn(v.w, sc))) << 24);
        *reinterpret_cast<uint32_t *>(out.fp8 + row * cn + j) = w;
    }
    for (int j = lane * 4; j < rope; j += 128) st4<uint16_t>(out.rope, row * rope + j, Ld4<Tin>::at(x, row * c + cn + j));
    if (lane == 0) out.scale[row] = sc;
}

template <typename Tin>
__global__ void quantize_fp4_kernel(const Tin *x, int64_t n, int d, Fp4RowsDev out)
{
    // 8 threads per 32-element block, 4 elements per thread
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; // group of 4 elements
    const int64_t total = n * (d / 4);
    const bool valid = g < total;
    const int64_t gg = valid ? g : total - 1;
    const int64_t row = gg / (d / 4);
    const int j = (int)(gg % (d / 4)) * 4;
    float4 v = Ld4<Tin>::at(x, row * d + j);
    float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
    if (!valid) return;
    const int e = fp4_scale_exp(a);
    const float inv = exp2i(-e);
    uint16_t two = uint16_t(e2m1x2_encode(v.x * inv, v.y * inv)) |
                   (uint16_t(e2m1x2_encode(v.z * inv, v.w * inv)) << 8);
    *reinterpret_cast<uint16_t *>(out.codes + row * (d / 2) + j / 2) = two;
    if ((j & 31) == 0) out.scales[row * (d / 32) + j / 32] = uint8_t(e + 127);
}

cudaError_t launch_quantize_kv(const void *x, int in_dtype, int64_t n, int c, int rope,
                               const KvRowsDev &out, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    const int rows_per_cta = 8;
    const unsigned grid = (unsigned)((n + rows_per_cta - 1) / rows_per_cta);
    if (in_dtype == CSA_F32) quantize_kv_kernel<float><<<grid, 256, 0, st>>>((const float *)x, n, c, rope, out);
    else quantize_kv_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)x, n, c, rope, out);
    return cudaGetLastError();
}

cudaError_t launch_quantize_fp4(const void *x, int in_dtype, int64_t n, int d,
                                const Fp4RowsDev &out, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    const int64_t groups = n * (d / 4);
    const unsigned grid = (unsigned)((groups + 255) / 256);
    if (in_dtype == CSA_F32) quantize_fp4_kernel<float><<<grid, 256, 0, st>>>((const float *)x, n, d, out);
    else quantize_fp4_kernel<uint16_t><<<grid, 256, 0, st>>>((const uint16_t *)x, n, d, out);
    return cudaGetLastError();
}

} // namespace csa
