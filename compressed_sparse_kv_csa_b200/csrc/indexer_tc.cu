// indexer_tc.cu -- lightning-indexer scores on the 5th-generation tensor cores (tcgen05 + TMEM)
// for the prefill shape: 64 index heads x 128 dims, bf16 queries and keys, positions 0..T-1.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 Eq. 16 and the Indexer listing: I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . K[s,:]), one
// key per compressed entry shared by the 64 index heads, only s < N_vis(t) = floor((t+1)/m).
//
// Tiling: keys on M (128 TMEM lanes), 4 query tokens x 64 heads on N (256 columns), K = 128.
// One tcgen05 M=128 x N=256 x K=128 product per (token group, key tile) lands in a
// double-buffered TMEM accumulator; 8 epilogue warps (two per TMEM lane quadrant, one per pair of
// tokens) read it with each lane owning one key, so the head reduction w . ReLU(.) is a per-lane
// loop with no cross-lane traffic, and the scores of consecutive keys are written coalesced.
// The 4-token query block (64 KB) stays in shared memory for the group; key tiles (32 KB) stream
// through a 4-stage TMA ring.  Roles: warps 0-7 epilogue, warp 8 TMA producer (one lane), warp 9
// TMEM allocation + MMA issue (one lane).  Every wait is bounded (%globaltimer) and a timeout sets
// CSA_DEVERR_TIMEOUT.
#include "common.cuh"
#include "tc_common.cuh"
#include "tma_host.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kHI = 64, kDI = 128, kG = 4, kMK = 128, kStages = 4;
constexpr int kEpiWarps = 8, kProdWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 10 * 32;

constexpr uint32_t OFF_Q = 0;                      // 2 sub-tiles [256 rows x 128 B]   64 KB
constexpr uint32_t OFF_K = 65536;                  // 4 stages x 2 sub-tiles [128 x 128 B]
constexpr uint32_t OFF_BAR = OFF_K + kStages * 32768;
constexpr uint32_t OFF_TMEM = OFF_BAR + 256;
constexpr uint32_t SMEM_USED = OFF_BAR + 512;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;

enum { B_QFULL = 0, B_QEMPTY = 1, B_KFULL = 2, B_KEMPTY = B_KFULL + kStages, B_AFULL = B_KEMPTY + kStages,
       B_AEMPTY = B_AFULL + 2, B_FINAL = B_AEMPTY + 2, NUM_BARS };

constexpr uint32_t IDESC = idesc_bf16_f32(128, 256, false, false);
constexpr uint32_t TMEM_COLS = 512;

struct Maps {
    CUtensorMap q, k;
};

struct Sm {
    uint32_t base;
    __device__ uint32_t bar(int b) const { return base + OFF_BAR + 8u * (uint32_t)b; }
};

__device__ __forceinline__ int64_t nv_of(const IndexerArgs &a, int64_t t)
{
    int64_t nv = (t + 1) / a.m;
    if (nv > a.max_nvis) nv = a.max_nvis;
    if (nv > a.n_keys) nv = a.n_keys;
    return nv;
}

// number of key tiles of the group starting at token t0 (0: nothing visible)
__device__ __forceinline__ int group_tiles(const IndexerArgs &a, int64_t t0)
{
    int64_t tl = t0 + kG - 1 < a.Nq - 1 ? t0 + kG - 1 : a.Nq - 1;
    const int64_t nv = nv_of(a, tl); // nv grows with t
    return (int)((nv + kMK - 1) / kMK);
}

__device__ __forceinline__ bool epi_wait(uint32_t bar, uint32_t parity)
{
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float4 ldw4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }

__device__ bool epilogue_role(const IndexerArgs &a, Sm S, uint32_t tmem, int warp, int lane)
{
    const int quad = warp & 3, half = warp >> 2; // TMEM lane quadrant, token pair
    const int64_t n_groups = (a.Nq + kG - 1) / kG;
    uint32_t kt = 0; // global tile counter (the same sequence as the other roles)
    for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x) {
        const int64_t t0 = g * kG;
        const int nt = group_tiles(a, t0);
        if (nt == 0) continue;
        const int64_t ta = t0 + 2 * half, tb = ta + 1;
        const int64_t nva = ta < a.Nq ? nv_of(a, ta) : 0, nvb = tb < a.Nq ? nv_of(a, tb) : 0;
        const float *wa = a.w + (ta < a.Nq ? ta : a.Nq - 1) * kHI; // weights: broadcast loads, L1-resident
        const float *wb = a.w + (tb < a.Nq ? tb : a.Nq - 1) * kHI;
        for (int i = 0; i < nt; ++i, ++kt) {
            const uint32_t buf = kt & 1;
            if (!epi_wait(S.bar(B_AFULL + buf), (kt >> 1) & 1)) return false;
            tc_fence_after();
            uint32_t r[4][32];
            const uint32_t taddr = tmem + buf * 256u + ((uint32_t)(32 * quad) << 16) + 128u * half;
            tmem_ld32(taddr + 0, r[0]);
            tmem_ld32(taddr + 32, r[1]);
            tmem_ld32(taddr + 64, r[2]);
            tmem_ld32(taddr + 96, r[3]);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(S.bar(B_AEMPTY + buf));
            float sa = 0.f, sb = 0.f;
#pragma unroll
            for (int h4 = 0; h4 < 16; ++h4) {
                const float4 w1 = ldw4(wa + 4 * h4), w2 = ldw4(wb + 4 * h4);
                const int c = (4 * h4) >> 5, e = (4 * h4) & 31;
                sa = fmaf(w1.x, fmaxf(__uint_as_float(r[c][e + 0]), 0.f), sa);
                sa = fmaf(w1.y, fmaxf(__uint_as_float(r[c][e + 1]), 0.f), sa);
                sa = fmaf(w1.z, fmaxf(__uint_as_float(r[c][e + 2]), 0.f), sa);
                sa = fmaf(w1.w, fmaxf(__uint_as_float(r[c][e + 3]), 0.f), sa);
                sb = fmaf(w2.x, fmaxf(__uint_as_float(r[2 + c][e + 0]), 0.f), sb);
                sb = fmaf(w2.y, fmaxf(__uint_as_float(r[2 + c][e + 1]), 0.f), sb);
                sb = fmaf(w2.z, fmaxf(__uint_as_float(r[2 + c][e + 2]), 0.f), sb);
                sb = fmaf(w2.w, fmaxf(__uint_as_float(r[2 + c][e + 3]), 0.f), sb);
            }
            const int64_t s = (int64_t)i * kMK + 32 * quad + lane;
            if (s < nva) a.scores[ta * a.ld + s] = sa;
            if (s < nvb) a.scores[tb * a.ld + s] = sb;
        }
    }
    return true;
}

__device__ bool producer_role(const IndexerArgs &a, const Maps &M, Sm S)
{
    const int64_t n_groups = (a.Nq + kG - 1) / kG;
    uint32_t kt = 0, gc = 0;
    for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x) {
        const int64_t t0 = g * kG;
        const int nt = group_tiles(a, t0);
        if (nt == 0) continue;
        if (gc > 0 && !mbar_wait(S.bar(B_QEMPTY), (gc - 1) & 1)) return false;
        mbar_arrive_expect_tx(S.bar(B_QFULL), 65536u);
        for (int sub = 0; sub < 2; ++sub)
            tma_load_2d(S.base + OFF_Q + 32768u * sub, &M.q, 64 * sub, (int32_t)(t0 * kHI), S.bar(B_QFULL));
        ++gc;
        for (int i = 0; i < nt; ++i, ++kt) {
            const uint32_t st = kt % kStages;
            if (kt >= (uint32_t)kStages && !mbar_wait(S.bar(B_KEMPTY + st), ((kt / kStages) - 1) & 1)) return false;
            mbar_arrive_expect_tx(S.bar(B_KFULL + st), 32768u);
            for (int sub = 0; sub < 2; ++sub)
                tma_load_2d(S.base + OFF_K + st * 32768u + 16384u * sub, &M.k, 64 * sub, i * kMK, S.bar(B_KFULL + st));
        }
    }
    return true;
}

__device__ bool mma_role(const IndexerArgs &a, Sm S, uint32_t tmem)
{
    const int64_t n_groups = (a.Nq + kG - 1) / kG;
    uint32_t kt = 0, gc = 0;
    for (int64_t g = blockIdx.x; g < n_groups; g += gridDim.x) {
        const int nt = group_tiles(a, g * kG);
        if (nt == 0) continue;
        if (!mbar_wait(S.bar(B_QFULL), gc & 1)) return false;
        ++gc;
        for (int i = 0; i < nt; ++i, ++kt) {
            const uint32_t st = kt % kStages, buf = kt & 1;
            if (!mbar_wait(S.bar(B_KFULL + st), (kt / kStages) & 1)) return false;
            if (kt >= 2 && !mbar_wait(S.bar(B_AEMPTY + buf), ((kt >> 1) - 1) & 1)) return false;
            tc_fence_after();
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = sdesc_sw128(S.base + OFF_K + st * 32768u + 16384u * sub + 32u * kk, 16, 1024);
                    const uint64_t bd = sdesc_sw128(S.base + OFF_Q + 32768u * sub + 32u * kk, 16, 1024);
                    mma_bf16(tmem + buf * 256u, ad, bd, IDESC, (sub | kk) != 0);
                }
            }
            mma_commit(S.bar(B_KEMPTY + st));
            mma_commit(S.bar(B_AFULL + buf));
        }
        mma_commit(S.bar(B_QEMPTY));
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) indexer_tc_kernel(IndexerArgs a, const __grid_constant__ Maps maps)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem_raw + (base - raw) + OFF_TMEM);
    Sm S{base};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            uint32_t cnt = 1;
            if (b >= B_AEMPTY && b < B_AEMPTY + 2) cnt = kEpiWarps * 32;
            mbar_init(S.bar(b), cnt);
        }
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(base + OFF_TMEM, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    if (warp < kEpiWarps) ok = epilogue_role(a, S, tmem, warp, lane);
    else if (warp == kProdWarp) { if (lane == 0) ok = producer_role(a, maps, S); }
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

cudaError_t launch_indexer_scores_tc(const IndexerArgs &a, cudaStream_t st, bool *handled)
{
    *handled = false;
    if (a.fmt != CSA_BF16 || a.H != kHI || a.d != kDI || a.q_pos || a.key_off || a.Nq <= 0 || a.n_keys <= 0)
        return cudaSuccess;
    if ((uint64_t)a.Nq * kHI >= (1ull << 31) || a.n_keys >= (1ll << 31)) return cudaSuccess;
    *handled = true; // the call is this kernel's: an encoding failure is an error, not a switch of kernels
    Maps maps;
    if (!tma::encode_bf16_rows(&maps.q, a.q, (uint64_t)a.Nq * kHI, kDI, 256) ||
        !tma::encode_bf16_rows(&maps.k, a.keys, (uint64_t)a.n_keys, kDI, kMK))
        return cudaErrorNotSupported;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(indexer_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const int64_t n_groups = (a.Nq + kG - 1) / kG;
    const int64_t grid = n_groups < sms ? n_groups : sms;
    indexer_tc_kernel<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(a, maps);
    return cudaGetLastError();
}

} // namespace csa
