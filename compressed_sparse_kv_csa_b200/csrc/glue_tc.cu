// glue_tc.cu -- inter-layer projection of a stacked decode (tcgen05 + TMEM).
//
// The pages describe one attention layer; a stack of layers needs the next layer's queries.
// This kernel takes the attention output o (one row of c channels per sequence and head) and
// forms, per row,
//     q_next = bf16( y / rms(y) / sqrt(c) ),   y = P o      (P: c x c, row i = output channel i)
//     q_I    = FP4 ( z / rms(z) ),             z = Rm o     (Rm: d x c)
// with rms(v) = sqrt(mean(v^2)) and an all-zero row mapped to zero.  The FP4 rows use the
// index-key format (E2M1 codes, one E8M0 scale per 32 elements), so q_I feeds the FP4 indexer
// directly.
//
// Tiling: 128 rows of o per CTA on the MMA M dimension (TMEM lanes), K = c in chunks of 64
// through a 2-stage TMA ring; pass 1 accumulates y for all c output channels (c <= 512 TMEM
// columns), its epilogue normalises and stores q_next, then pass 2 reuses the columns for z.
// Roles: warp 0 TMA producer (one lane), warp 1 TMEM allocation + MMA issue (one lane),
// warps 2-5 epilogue (one row per thread).  Every wait is bounded (%globaltimer) and a timeout
// sets CSA_DEVERR_TIMEOUT.
#include "common.cuh"
#include "tc_common.cuh"
#include "tma_host.cuh"

#include <string.h>

namespace csa {

namespace {

using namespace tc;

constexpr int kRows = 128, kStages = 2;
constexpr int kProdWarp = 0, kMmaWarp = 1, kEpiWarp0 = 2, kThreads = 6 * 32;

constexpr uint32_t A_BYTES = kRows * 128u;        // 128 rows x 64 bf16
constexpr uint32_t B_BYTES = 512u * 128u;         // up to 512 rows x 64 bf16
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_B = OFF_A + kStages * A_BYTES;
constexpr uint32_t OFF_BAR = OFF_B + kStages * B_BYTES;
constexpr uint32_t OFF_TMEM = OFF_BAR + 128;
constexpr uint32_t SMEM_USED = OFF_BAR + 256;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;
constexpr uint32_t TMEM_COLS = 512;

enum { B_FULL = 0, B_EMPTY = B_FULL + kStages, B_ACC1 = B_EMPTY + kStages, B_EPI1, B_ACC2, B_FINAL, NUM_BARS };

struct GlueArgs {
    int64_t R;
    int c, d;
    uint16_t *q_next;
    Fp4RowsDev qI;   // codes == nullptr: no index query
    int *err;
};

struct Maps {
    CUtensorMap o, P, Rm;
};

struct Sm {
    uint32_t base;
    __device__ uint32_t bar(int b) const { return base + OFF_BAR + 8u * (uint32_t)b; }
};

__device__ __forceinline__ int passes(const GlueArgs &a) { return a.qI.codes ? 2 : 1; }

__device__ bool producer_role(const GlueArgs &a, const Maps &M, Sm S, int32_t row0)
{
    const int kc = a.c / 64;
    uint32_t j = 0;
    for (int pass = 0; pass < passes(a); ++pass) {
        const CUtensorMap *bm = pass == 0 ? &M.P : &M.Rm;
        const int nb = ((pass == 0 ? a.c : a.d) + 63) / 64; // 64-row boxes of the B operand
        for (int kk = 0; kk < kc; ++kk, ++j) {
            const uint32_t st = j % kStages;
            if (j >= (uint32_t)kStages && !mbar_wait(S.bar(B_EMPTY + st), ((j / kStages) - 1) & 1)) return false;
            mbar_arrive_expect_tx(S.bar(B_FULL + st), A_BYTES + (uint32_t)nb * 8192u);
            tma_load_2d(S.base + OFF_A + st * A_BYTES, &M.o, 64 * kk, row0, S.bar(B_FULL + st));
            for (int b = 0; b < nb; ++b)
                tma_load_2d(S.base + OFF_B + st * B_BYTES + 8192u * b, bm, 64 * kk, 64 * b, S.bar(B_FULL + st));
        }
    }
    return true;
}

__device__ bool mma_role(const GlueArgs &a, Sm S, uint32_t tmem)
{
    const int kc = a.c / 64;
    uint32_t j = 0;
    for (int pass = 0; pass < passes(a); ++pass) {
        const int n_out = pass == 0 ? a.c : a.d;
        if (pass == 1) { // the epilogue must have read y out of the columns z overwrites
            if (!mbar_wait(S.bar(B_EPI1), 0)) return false;
        }
        for (int kk = 0; kk < kc; ++kk, ++j) {
            const uint32_t st = j % kStages;
            if (!mbar_wait(S.bar(B_FULL + st), (j / kStages) & 1)) return false;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc_sw128(S.base + OFF_A + st * A_BYTES + 32u * ks, 16, 1024);
                for (int n0 = 0; n0 < n_out; n0 += 256) {
                    const int n = n_out - n0 < 256 ? n_out - n0 : 256;
                    const uint64_t bd = sdesc_sw128(S.base + OFF_B + st * B_BYTES + 128u * n0 + 32u * ks, 16, 1024);
                    mma_bf16(tmem + (uint32_t)n0, ad, bd, idesc_bf16_f32(128, n, false, false), (kk | ks) != 0);
                }
            }
            mma_commit(S.bar(B_EMPTY + st));
        }
        mma_commit(S.bar(pass == 0 ? B_ACC1 : B_ACC2));
    }
    return true;
}

// Sum of squares of the first n columns of this thread's TMEM lane.
__device__ __forceinline__ float lane_sumsq(uint32_t taddr, int n)
{
    float ss = 0.f;
    for (int n0 = 0; n0 < n; n0 += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)n0, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ss);
    }
    return ss;
}

__device__ bool epilogue_role(const GlueArgs &a, Sm S, uint32_t tmem, int warp, int lane, int64_t row0)
{
    const int quad = warp & 3; // TMEM lane quadrant this warp may access
    const int64_t row = row0 + 32 * quad + lane;
    const bool live = row < a.R;
    const uint32_t taddr = tmem + ((uint32_t)(32 * quad) << 16);

    // pass 1: q_next = y / rms(y) / sqrt(c)
    if (!__all_sync(0xffffffffu, mbar_wait(S.bar(B_ACC1), 0))) return false;
    tc_fence_after();
    {
        const float ss = lane_sumsq(taddr, a.c);
        const float f = ss > 0.f ? 1.f / sqrtf(ss) : 0.f; // 1/sqrt(ss/c)/sqrt(c) = 1/sqrt(ss)
        for (int n0 = 0; n0 < a.c; n0 += 32) {
            uint32_t r[32];
            tmem_ld32(taddr + (uint32_t)n0, r);
            tmem_ld_wait();
            if (live) {
                uint32_t p[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    p[i] = uint32_t(f32_to_bf16_bits(__uint_as_float(r[2 * i]) * f)) |
                           (uint32_t(f32_to_bf16_bits(__uint_as_float(r[2 * i + 1]) * f)) << 16);
                uint4 *dst = reinterpret_cast<uint4 *>(a.q_next + row * a.c + n0);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
        }
    }
    tc_fence_before();
    mbar_arrive(S.bar(B_EPI1));
    if (!a.qI.codes) return true;

    // pass 2: q_I = FP4(z / rms(z))
    if (!__all_sync(0xffffffffu, mbar_wait(S.bar(B_ACC2), 0))) return false;
    tc_fence_after();
    const float ss = lane_sumsq(taddr, a.d);
    const float f = ss > 0.f ? 1.f / sqrtf(ss / (float)a.d) : 0.f;
    for (int n0 = 0; n0 < a.d; n0 += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)n0, r);
        tmem_ld_wait();
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float v = __uint_as_float(r[i]) * f;
            r[i] = __float_as_uint(v);
            amax = fmaxf(amax, fabsf(v));
        }
        const int e = fp4_scale_exp(amax);
        const float inv = exp2i(-e);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t x = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b)
                x |= uint32_t(e2m1x2_encode(__uint_as_float(r[8 * i + 2 * b]) * inv,
                                            __uint_as_float(r[8 * i + 2 * b + 1]) * inv))
                     << (8 * b);
            w[i] = x;
        }
        if (live) {
            *reinterpret_cast<uint4 *>(a.qI.codes + row * (a.d / 2) + n0 / 2) = make_uint4(w[0], w[1], w[2], w[3]);
            a.qI.scales[row * (a.d / 32) + n0 / 32] = uint8_t(e + 127);
        }
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) glue_tc_kernel(GlueArgs a, const __grid_constant__ Maps maps)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem_raw + (base - raw) + OFF_TMEM);
    Sm S{base};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t row0 = (int64_t)blockIdx.x * kRows;
    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) mbar_init(S.bar(b), b == B_EPI1 ? 4 * 32 : 1);
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(base + OFF_TMEM, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    if (warp >= kEpiWarp0) ok = epilogue_role(a, S, tmem, warp, lane, row0);
    else if (warp == kProdWarp) { if (lane == 0) ok = producer_role(a, maps, S, (int32_t)row0); }
    else if (lane == 0) ok = mma_role(a, S, tmem);
    if (!ok) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    if (warp == kMmaWarp && lane == 0) {
        mma_commit(S.bar(B_FINAL));
        if (!mbar_wait(S.bar(B_FINAL), 0)) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, TMEM_COLS);
}

} // namespace

// Shapes: c a multiple of 64 in [64, 512], d a multiple of 32 in [32, 256] (or no index query),
// R < 2^31.  Returns cudaErrorInvalidValue when a tensor map cannot be encoded.
cudaError_t launch_decode_glue(const void *o, const void *P, const void *Rm, int64_t R, int c, int d,
                               void *q_next, const Fp4RowsDev *qI, int *err, cudaStream_t st)
{
    if (R == 0) return cudaSuccess;
    Maps maps;
    memset(&maps, 0, sizeof(maps));
    if (!tma::encode_bf16_rows(&maps.o, o, (uint64_t)R, (uint64_t)c, kRows) ||
        !tma::encode_bf16_rows(&maps.P, P, (uint64_t)c, (uint64_t)c, 64))
        return cudaErrorInvalidValue;
    if (qI && !tma::encode_bf16_rows(&maps.Rm, Rm, (uint64_t)d, (uint64_t)c, 64)) return cudaErrorInvalidValue;
    GlueArgs a;
    a.R = R;
    a.c = c;
    a.d = qI ? d : 0;
    a.q_next = static_cast<uint16_t *>(q_next);
    a.qI = qI ? *qI : Fp4RowsDev{nullptr, nullptr, 0, 0};
    a.err = err;
    cudaError_t e = cudaFuncSetAttribute(glue_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const int64_t grid = (R + kRows - 1) / kRows;
    glue_tc_kernel<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(a, maps);
    return cudaGetLastError();
}

} // namespace csa
