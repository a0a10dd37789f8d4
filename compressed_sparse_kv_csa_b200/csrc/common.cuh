// common.cuh -- device helpers shared by the libcsa kernels (sm_100a).
//
// Storage formats follow the OCP specifications: FP8 E4M3 ("fn": max 448, no infinities),
// FP4 E2M1 with E8M0 block scales (OCP MX v1.0), bf16 round-to-nearest-even.  Conversions use
// the CUDA conversion intrinsics (round to nearest even, saturating) and canonicalise -0 to +0.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

// Device error word (CSA_DEVERR_* bits), read and cleared by csa_device_error().  Kernels get
// its device address in their argument block (dev_error_word() on the host).
__device__ __forceinline__ void flag_error(int *err, int bit)
{
    if (err) atomicOr(err, bit);
}

// ------------------------------------------------------------------------------------------
// loads
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x)
{
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}

// Load 4 consecutive elements (fp32 or bf16 storage) starting at element `i` as fp32.
template <typename T> struct Ld4;
template <> struct Ld4<float> {
    static __device__ __forceinline__ float4 at(const float *p, int64_t i)
    {
        return *reinterpret_cast<const float4 *>(p + i);
    }
};
template <> struct Ld4<uint16_t> {
    static __device__ __forceinline__ float4 at(const uint16_t *p, int64_t i)
    {
        uint2 u = *reinterpret_cast<const uint2 *>(p + i);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
    }
};

template <typename T> __device__ __forceinline__ float ld1(const T *p, int64_t i);
template <> __device__ __forceinline__ float ld1<float>(const float *p, int64_t i) { return p[i]; }
template <> __device__ __forceinline__ float ld1<uint16_t>(const uint16_t *p, int64_t i) { return bf16_to_f32(p[i]); }

template <typename T> __device__ __forceinline__ void st4(T *p, int64_t i, float4 v);
template <> __device__ __forceinline__ void st4<float>(float *p, int64_t i, float4 v)
{
    *reinterpret_cast<float4 *>(p + i) = v;
}
template <> __device__ __forceinline__ void st4<uint16_t>(uint16_t *p, int64_t i, float4 v)
{
    uint2 u;
    u.x = uint32_t(f32_to_bf16_bits(v.x)) | (uint32_t(f32_to_bf16_bits(v.y)) << 16);
    u.y = uint32_t(f32_to_bf16_bits(v.z)) | (uint32_t(f32_to_bf16_bits(v.w)) << 16);
    *reinterpret_cast<uint2 *>(p + i) = u;
}

// ------------------------------------------------------------------------------------------
// FP8 E4M3 / FP4 E2M1 encoders and decoders
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ uint8_t e4m3_encode(float v)
{
    uint8_t b = (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
    return (b & 0x7f) ? b : (uint8_t)0;
}

__device__ __forceinline__ float e4m3_decode(uint8_t b)
{
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
    return __half2float(__half(h));
}

// Two E2M1 nibbles (lo = element 2i, hi = element 2i+1), round to nearest even, saturating.
__device__ __forceinline__ uint8_t e2m1x2_encode(float lo, float hi)
{
    uint8_t b = (uint8_t)__nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest);
    if ((b & 0x07) == 0) b &= 0xf0;
    if ((b & 0x70) == 0) b &= 0x0f;
    return b;
}

__device__ __forceinline__ float e2m1_decode(uint32_t nib)
{
    // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6
    const float mag = (nib & 4) ? ((nib & 2) ? ((nib & 1) ? 6.f : 4.f) : ((nib & 1) ? 3.f : 2.f))
                                : (float)(nib & 3) * 0.5f;
    return (nib & 8) ? -mag : mag;
}

// 2^e as an exact fp32 value, e in [-127, 127].
__device__ __forceinline__ float exp2i(int e)
{
    return (e >= -126) ? __uint_as_float(uint32_t(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Smallest e with amax <= 6 * 2^e, clamped to [-127, 127]; -127 for amax == 0.
__device__ __forceinline__ int fp4_scale_exp(float amax)
{
    if (!(amax > 0.f)) return -127;
    int bias = 0;
    if (amax < 1.17549435e-38f) { // subnormal: renormalise exactly
        amax *= 18446744073709551616.f; // 2^64
        bias = 64;
    }
    uint32_t u = __float_as_uint(amax);
    int e0 = int((u >> 23) & 0xff) - 127 - bias; // amax in [2^e0, 2^(e0+1))
    int e = ((u & 0x7fffff) <= 0x400000u) ? e0 - 2 : e0 - 1;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// Row of compressed entry s of sequence / query b in a paged cache (-1 when the page index is out
// of the table), else the contiguous row base + s.
__device__ __forceinline__ int64_t paged_row(const int32_t *pages, int max_pages, int page_rows, int64_t b, int64_t s,
                                             int64_t base)
{
    if (!pages) return base + s;
    const int64_t pg = s / page_rows;
    if (pg >= max_pages) return -1;
    return (int64_t)pages[b * max_pages + pg] * page_rows + s % page_rows;
}

// fp32 order-preserving key: larger float -> larger unsigned key.
__device__ __forceinline__ uint32_t float_key(float f)
{
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

} // namespace csa

// ------------------------------------------------------------------------------------------
// host-side launch helpers (implemented in the .cu files, called from abi.cu)
// ------------------------------------------------------------------------------------------
namespace csa {

int *dev_error_word(); // device address of the error word for the current device
int device_sms();      // SM count of the current device

struct KvRowsDev {
    uint8_t *fp8;
    uint16_t *rope;
    float *scale;
    int64_t n;
    int c, rope_dims;
};
struct Fp4RowsDev {
    uint8_t *codes;
    uint8_t *scales;
    int64_t n;
    int d;
};

cudaError_t launch_compress(bool overlap, const void *Ca, const void *Cb, const void *Za,
                            const void *Zb, const float *B, int64_t T, int c, int m, int in_dtype,
                            void *out, int out_dtype, const KvRowsDev *kv, const Fp4RowsDev *fp4,
                            cudaStream_t st);
cudaError_t launch_quantize_kv(const void *x, int in_dtype, int64_t n, int c, int rope,
                               const KvRowsDev &out, cudaStream_t st);
cudaError_t launch_quantize_fp4(const void *x, int in_dtype, int64_t n, int d,
                                const Fp4RowsDev &out, cudaStream_t st);
cudaError_t launch_compress_append(bool overlap, int64_t B, const int64_t *pos, int c, int m, int in_dtype,
                                   const void *const new_rows[4], void *const tail[4], const float *Bias,
                                   const KvRowsDev *kv, const Fp4RowsDev *fp4, const int32_t *pages, int max_pages,
                                   int page_rows, const int64_t *comp_off, int64_t n_out, int *err, cudaStream_t st);
cudaError_t launch_window_append(const void *x, int in_dtype, int64_t B, int c, const int64_t *pos, int W,
                                 const KvRowsDev &out, cudaStream_t st);
cudaError_t launch_prep_rows(const void *x, int in_dtype, int64_t n, int d, const float *g, float eps, int rd,
                             const int64_t *pos, double base, int hadamard, void *out, int out_dtype,
                             const KvRowsDev *kv, const Fp4RowsDev *f4, cudaStream_t st);

struct IndexerArgs {
    const void *q;        // dense [Nq,H,d] or null for fp4
    const float *w;
    const void *keys;     // dense [n_keys,d] or null for fp4
    Fp4RowsDev q4, k4;    // fp4 operands
    int fmt;
    const int64_t *q_pos, *key_off;
    int64_t n_keys, Nq;
    int H, d, m, k;
    int64_t max_nvis, ld;  // ld: row stride of the score buffer
    float *scores;         // [Nq, ld] workspace
    const int32_t *pages;  // paged keys: row of entry s of query r = pages[r*max_pages + s/page_rows]*page_rows + s%page_rows
    int max_pages, page_rows;
    int32_t *idx_out;
    float *score_out;
    void *topk_ws;
    int *err;
};
cudaError_t launch_indexer_scores(const IndexerArgs &a, cudaStream_t st);

// indexer_topk, indexer_topk_paged and indexer_topk_static: shared checks and launch (abi.cu).
// scratch == nullptr: the caller's workspace must hold indexer_topk_workspace_size(); otherwise
// ws_bytes is the static scratch's size and scratch() supplies its device address.
int indexer_topk_impl(const void *q, const float *w, const void *keys, int32_t fmt, const int64_t *q_pos,
                      const int64_t *key_off, int64_t n_keys, int64_t Nq, int32_t H_I, int32_t d_I, int32_t m,
                      int32_t k, int64_t max_nvis, int32_t *idx_out, float *score_out, void *ws, size_t ws_bytes,
                      void *(*scratch)(cudaError_t *), void *stream, const int32_t *pages = nullptr,
                      int32_t max_pages = 0, int32_t page_rows = 0);
cudaError_t launch_topk(const IndexerArgs &a, cudaStream_t st);
cudaError_t launch_topk_merge_lists(const float *scores, const int32_t *idx, const int64_t *bases, int64_t Nq,
                                    int n_lists, int list_len, int k, int32_t *idx_out, float *score_out,
                                    cudaStream_t st);

struct PrefillArgs {
    const void *q, *x_win, *kv_comp;
    int64_t n_comp;
    const int32_t *idx;
    int k;
    const float *sink;
    float scale;
    int64_t T;
    int H, c, m, W, dtype;
    void *o;
    float *lse;
    int *err;
};
cudaError_t launch_attn_prefill(const PrefillArgs &a, cudaStream_t st);

struct DecodeArgs {
    const uint16_t *q;
    KvRowsDev comp, win;
    const int64_t *comp_off, *pos;
    const int32_t *win_len, *idx;
    int k;
    const float *sink;
    float scale;
    int B, H, c, m, W;
    int64_t max_nvis;
    uint16_t *o;
    float *lse;
    float *part;          // split-K partials
    int n_chunks, chunk;  // chunks per sequence and keys per chunk
    const int32_t *pages; // paged cache: row of entry s of sequence b = pages[b*max_pages + s/page_rows]*page_rows + s%page_rows
    int max_pages, page_rows;
    uint64_t wait_ns;     // limit of the tensor-core kernel's bounded waits
    int *err;
};
void decode_plan(int B, int H, int c, int max_keys, int *n_chunks, int *chunk);
cudaError_t launch_attn_decode(const DecodeArgs &a, cudaStream_t st);

} // namespace csa
