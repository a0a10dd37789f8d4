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

template <typename Tin>
__global__ void __launch_bounds__(512) compress_kernel(CompressParams p, int TS)
{
    extern __shared__ float smem[];
    const int TPE = blockDim.x; // channel groups of 4
    const int x = threadIdx.x, y = threadIdx.y, z = threadIdx.z;
    const int64_t entry = (int64_t)blockIdx.x * blockDim.z + z;
    const bool valid = entry < p.n_entries;
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
            const int64_t row = entry * m + j;
            float4 v = Ld4<Tin>::at(Ca, row * c + ch);
            float4 zz = Ld4<Tin>::at(Za, row * c + ch);
            float4 b = *reinterpret_cast<const float4 *>(p.B + (int64_t)j * c + ch);
            zz.x += b.x; zz.y += b.y; zz.z += b.z; zz.w += b.w;
            soft_add(s, v, zz);
        }
        if (p.overlap && entry > 0) { // previous block (Cb / Zb, bias rows m..2m-1)
            const Tin *Cb = (const Tin *)p.Cb, *Zb = (const Tin *)p.Zb;
            for (int j = j0; j < j1; ++j) {
                const int64_t row = (entry - 1) * m + j;
                float4 v = Ld4<Tin>::at(Cb, row * c + ch);
                float4 zz = Ld4<Tin>::at(Zb, row * c + ch);
                float4 b = *reinterpret_cast<const float4 *>(p.B + (int64_t)(m + j) * c + ch);
                zz.x += b.x; zz.y += b.y; zz.z += b.z; zz.w += b.w;
                soft_add(s, v, zz);
            }
        }
    }
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
    if (x == 0 && y == 0) amax_s[z] = 0;
    __syncthreads();
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (y == 0) {
        for (int yy = 1; yy < TS; ++yy) soft_merge(s, part + (((size_t)z * TS + yy) * TPE + x) * 12);
        val = make_float4(s.num[0] / s.den[0], s.num[1] / s.den[1], s.num[2] / s.den[2],
                          s.num[3] / s.den[3]);
        if (valid && p.out) {
            if (p.out_dtype == CSA_F32) st4<float>((float *)p.out, entry * c + ch, val);
            else st4<uint16_t>((uint16_t *)p.out, entry * c + ch, val);
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
            *reinterpret_cast<uint32_t *>(p.kv.fp8 + entry * cn + ch) = w;
            if (x == 0) p.kv.scale[entry] = sc;
        } else {
            const int rd = p.kv.rope_dims;
            st4<uint16_t>(p.kv.rope, entry * rd + (ch - cn), val);
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
            *reinterpret_cast<uint16_t *>(p.fp4.codes + entry * (c / 2) + ch / 2) = two;
            if ((x & 7) == 0) p.fp4.scales[entry * (c / 32) + ch / 32] = uint8_t(e + 127);
        }
    }
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
    int TS = 1;
    if (!overlap && TPE >= 32) { // long HCA blocks: split the tokens of a block over threads
        while (TS * 2 * TPE <= 512 && TS * 2 <= m && m / (TS * 2) >= 8) TS *= 2;
    }
    // whole warps only (the FP4 path shuffles with a full mask); extra entries are invalid lanes
    int EPC = (TPE * TS >= 32) ? 1 : 32 / (TPE * TS);
    while (EPC * 2 * TPE * TS <= 256 && EPC * 2 <= p.n_entries) EPC *= 2;
    dim3 block(TPE, TS, EPC);
    const int64_t grid = (p.n_entries + EPC - 1) / EPC;
    size_t smem = (size_t)EPC * TS * TPE * 12 * sizeof(float) + EPC * sizeof(int);
    if (in_dtype == CSA_F32)
        compress_kernel<float><<<(unsigned)grid, block, smem, st>>>(p, TS);
    else
        compress_kernel<uint16_t><<<(unsigned)grid, block, smem, st>>>(p, TS);
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
