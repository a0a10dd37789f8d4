// attn_prefill_tc.cu -- hybrid MQA prefill attention on the 5th-generation tensor cores
// (tcgen05 + TMEM) for the 64-head x 512-channel bf16 shape with a 128-token window.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 step 3 (shared-KV multi-query attention: all heads share one key vector, which is also
// the value vector) and Sec. 2.4 Attention.forward listing (the sliding-window keys and the
// selected / all visible compressed keys are concatenated, no de-duplication, one sparse
// attention over both); itsolotime.com Q&A essay on DeepSeek-V4, Question 1: window of the most
// recent 128 raw tokens (mechanism 1) and one learnable sink logit per head in the softmax
// denominator (mechanism 3).
//
// Design (one query token per CTA pass, persistent CTAs):
//   * S = Q K^T with Q [64 heads x 512] and a tile of 128 keys: tcgen05 M=64, N=128, K=512.
//     The M=64 accumulator sits in the upper 16 lanes of each TMEM sub-partition.
//   * O = P V with V = K (the same shared-memory tile, read MN-major): two M=64, N=256, K=128
//     MMAs accumulate O [64 x 512] fp32 in the lower 16 lanes of each sub-partition, all 512
//     columns.  So S and O use disjoint lane halves and the whole 64 x 512 fp32 output stays in
//     TMEM for the token's key loop.
//   * Softmax: warp w owns heads 16w..16w+15 (lanes 0-15 hold S rows, lanes 16-31 the matching O
//     rows).  Online softmax in the log2 domain with a lazy rescale: the running max moves (and O
//     is rescaled in TMEM) only when a tile raises it by more than 8.
//   * Keys per token: tile 0 = window rows t-127..t of x_win; then tiles of 128 compressed rows
//     (every visible entry for HCA, the top-k list for CSA).  Invalid slots are zero-filled and
//     masked.  Window and HCA tiles are contiguous rows (2-D TMA boxes); CSA tiles are gathered
//     through the top-k list with TMA gather4 (4 rows x 64 channels per instruction, one per
//     producer thread and half tile).  Both land 128-byte-swizzled in two halves of 256 channels,
//     each released as soon as its half of P V has consumed it.
//   * Roles: warps 0-3 softmax / rescale / epilogue, warps 4-7 producers, warp 8 TMEM allocation
//     and (one lane) MMA issue.  Every wait is an mbarrier wait bounded by %globaltimer; a wait
//     that runs out records CSA_DEVERR_TIMEOUT and the CTA winds down without trapping.
#include "common.cuh"
#include "tc_common.cuh"

#include "tma_host.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kH = 64, kC = 512, kKT = 128, kW = 128;
constexpr int kMmaWarp = 8;
constexpr int kThreads = (kMmaWarp + 1) * 32;

constexpr uint32_t OFF_Q = 0;          // 8 sub-tiles [64 rows x 128 B]           64 KB
constexpr uint32_t OFF_K = 65536;      // 8 sub-tiles [128 keys x 128 B]          128 KB
constexpr uint32_t OFF_P = 196608;     // 2 sub-tiles [64 rows x 128 B]           16 KB
constexpr uint32_t OFF_BAR = 212992;   // mbarriers
constexpr uint32_t OFF_TMEM = OFF_BAR + 128;
constexpr uint32_t SMEM_USED = OFF_BAR + 256;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024; // slack to align the base to 1024 bytes

enum { B_QFULL = 0, B_QEMPTY, B_KVFULL0, B_KVFULL1, B_KVEMPTY0, B_KVEMPTY1, B_SFULL, B_PFULL, B_PVDONE,
       B_FINAL, NUM_BARS };

constexpr uint32_t IDESC_S = idesc_bf16_f32(64, 128, false, false);
constexpr uint32_t IDESC_S64 = idesc_bf16_f32(64, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(64, 256, false, true);
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 16u << 16; // lane offset of O[:, 0:256] (the lower lane half)
constexpr uint32_t kColS = 256;         // TMEM column of the S tile (upper lane half)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.f;

__device__ __forceinline__ int64_t n_compressed(const PrefillArgs &a, int64_t t)
{
    if (a.idx) return a.k;
    int64_t n = (t + 1) / a.m;
    return n < a.n_comp ? n : a.n_comp;
}

__device__ __forceinline__ int n_tiles(int64_t n_cmp) { return 1 + (int)((n_cmp + kKT - 1) / kKT); }

// Key row of slot j of tile i for token t, or nullptr when the slot is empty.
__device__ __forceinline__ const uint16_t *key_row(const PrefillArgs &a, int64_t t, int i, int j, int64_t n_cmp,
                                                   int64_t nvt, bool report)
{
    if (i == 0) {
        const int64_t u = t - (kW - 1) + j;
        return u >= 0 ? (const uint16_t *)a.x_win + u * kC : nullptr;
    }
    const int64_t slot = (int64_t)(i - 1) * kKT + j;
    if (slot >= n_cmp) return nullptr;
    const int64_t s = a.idx ? (int64_t)a.idx[t * a.k + slot] : slot;
    if (s < 0) return nullptr;
    if (s >= a.n_comp || s >= nvt) { // missing, or not yet visible to t (nvt = N_vis(t))
        if (report) flag_error(a.err, CSA_DEVERR_INDEX);
        return nullptr;
    }
    return (const uint16_t *)a.kv_comp + s * kC;
}

__device__ __forceinline__ void sts16(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// 2^x with the hardware approximation (ex2.approx, flush-to-zero); 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Warp-uniform bounded wait: every lane waits, and the warp proceeds only if all lanes saw it.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity)
{
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// Tensor maps of q viewed as [T*64, 512], of x_win [T, 512] and of kv_comp [n_comp, 512], all
// bf16 with 64-channel boxes and 128-byte swizzle (rows: 64 for q, 128 for keys, 1 for the
// gather map of kv_comp).
struct TmaMaps {
    CUtensorMap q, x, kv, kvg;
};

// Compressed row of slot j of CSA tile i for token t, or -1 when the slot is empty or invalid.
__device__ __forceinline__ int32_t gather_row(const PrefillArgs &a, int64_t t, int i, int j, int64_t n_cmp,
                                              int64_t nvt, bool report)
{
    const int64_t slot = (int64_t)(i - 1) * kKT + j;
    if (slot >= n_cmp) return -1;
    const int32_t s = a.idx[t * a.k + slot];
    if (s >= a.n_comp || s >= nvt) { // missing, or not yet visible to t (nvt = N_vis(t))
        if (report) flag_error(a.err, CSA_DEVERR_INDEX);
        return -1;
    }
    return s;
}

struct Smem {
    uint32_t sQ, sK, sP, bars;
    __device__ uint32_t bar(int b) const { return bars + 8u * (uint32_t)b; }
};

// Softmax / rescale / epilogue (warps 0-3).  Returns false when a wait ran out.
// TMEM map (lane halves of each 32-lane sub-partition; M=64 rows r = 16*warp + (lane & 15)):
//   upper half (lanes 0-15):  O[:, 256:512] in columns 0-255, S in columns 256-383
//   lower half (lanes 16-31): O[:, 0:256]   in columns 0-255
// so one 32x32b TMEM access at columns 0-255 reaches both halves of a row's output, and the
// two lanes of a row split its 128 keys (lane l: keys 0-63, lane l+16: keys 64-127).
__device__ __forceinline__ bool softmax_role(const PrefillArgs &a, const Smem &S, uint32_t tmem, int warp, int lane)
{
    const float scale_log2 = a.scale * kLog2e;
    const bool upper = lane < 16;
    const int row = 16 * warp + (lane & 15); // head
    const int kbase = upper ? 0 : 64;        // this lane's half of the key tile
    const int obase = upper ? 256 : 0;       // this lane's half of the output channels
    const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);
    const float sink_l2 = a.sink[row] * kLog2e;
    uint32_t s_ph = 0, pv_ph = 0;
    for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
        const int64_t n_cmp = n_compressed(a, t);
        const int64_t nvt = (t + 1) / a.m; // N_vis(t), once per token
        const int nt = n_tiles(n_cmp);
        float m_run = -INFINITY, l_run = 0.f;
        for (int i = 0; i < nt; ++i) {
            if (!warp_wait(S.bar(B_SFULL), s_ph)) return false;
            s_ph ^= 1;
            tc_fence_after();
            float sv[64];
            {
                uint32_t r0[32], r1[32], r2[32], r3[32];
                tmem_ld32(tw + kColS + 0, r0);
                tmem_ld32(tw + kColS + 32, r1);
                tmem_ld32(tw + kColS + 64, r2);
                tmem_ld32(tw + kColS + 96, r3);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) { // keys 64-127 of the row move to the lower lane
                    const uint32_t x = __shfl_xor_sync(0xffffffffu, r2[e], 16);
                    const uint32_t y = __shfl_xor_sync(0xffffffffu, r3[e], 16);
                    sv[e] = __uint_as_float(upper ? r0[e] : x);
                    sv[32 + e] = __uint_as_float(upper ? r1[e] : y);
                }
            }
            uint32_t vm[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                vm[q] = __ballot_sync(0xffffffffu, key_row(a, t, i, lane + 32 * q, n_cmp, nvt, false) != nullptr);
            const uint32_t m0 = upper ? vm[0] : vm[2], m1 = upper ? vm[1] : vm[3];
            float mt = -INFINITY;
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                const uint32_t bit = (e < 32) ? (m0 >> e) & 1u : (m1 >> (e - 32)) & 1u;
                const float s = bit ? sv[e] * scale_log2 : -INFINITY;
                sv[e] = s;
                mt = fmaxf(mt, s);
            }
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
            const float m_new = fmaxf(m_run, mt);
            float resc = 1.f, m_use = m_run;
            if (m_new != -INFINITY && (m_run == -INFINITY || m_new > m_run + kRescaleThreshold)) {
                resc = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
                m_use = m_new;
            }
            float ls = 0.f;
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                const float p = (m_use == -INFINITY) ? 0.f : fast_exp2(sv[e] - m_use);
                sv[e] = p;
                ls += p;
            }
            ls += __shfl_xor_sync(0xffffffffu, ls, 16);
            l_run = l_run * resc + ls;
            m_run = m_use;
            if (i > 0) { // P V of the previous tile must be done: P buffer free, O settled
                if (!warp_wait(S.bar(B_PVDONE), pv_ph)) return false;
                pv_ph ^= 1;
                tc_fence_after();
            }
            if (__any_sync(0xffffffffu, i > 0 && resc != 1.f)) {
                for (int c = 0; c < 8; c += 2) {
                    uint32_t r[32], r2[32];
                    tmem_ld32(tw + 32u * c, r);
                    tmem_ld32(tw + 32u * (c + 1), r2);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        r[e] = __float_as_uint(__uint_as_float(r[e]) * resc);
                        r2[e] = __float_as_uint(__uint_as_float(r2[e]) * resc);
                    }
                    tmem_st32(tw + 32u * c, r);
                    tmem_st32(tw + 32u * (c + 1), r2);
                }
                tmem_st_wait();
            }
            { // P row half: keys kbase .. kbase+63 -> P sub-tile kbase/64
                const uint32_t psub = S.sP + (uint32_t)(kbase >> 6) * 8192u;
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    uint4 v;
                    v.x = pack_bf16(sv[8 * g + 0], sv[8 * g + 1]);
                    v.y = pack_bf16(sv[8 * g + 2], sv[8 * g + 3]);
                    v.z = pack_bf16(sv[8 * g + 4], sv[8 * g + 5]);
                    v.w = pack_bf16(sv[8 * g + 6], sv[8 * g + 7]);
                    sts16(psub + sw128_off(row, 8 * g), v);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(S.bar(B_PFULL));
        }
        // epilogue: wait for the token's last P V, normalise, write o and lse
        if (!warp_wait(S.bar(B_PVDONE), pv_ph)) return false;
        pv_ph ^= 1;
        tc_fence_after();
        const float den = l_run + fast_exp2(sink_l2 - m_run);
        const float inv = (den > 0.f && den < INFINITY) ? 1.f / den : 0.f;
        uint16_t *orow = (uint16_t *)a.o + ((t * kH) + row) * (int64_t)kC + obase;
        for (int c = 0; c < 8; c += 2) {
            uint32_t r[2][32];
            tmem_ld32(tw + 32u * c, r[0]);
            tmem_ld32(tw + 32u * (c + 1), r[1]);
            tmem_ld_wait();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t *x = r[hh] + 8 * g;
                    uint4 v;
                    v.x = pack_bf16(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv);
                    v.y = pack_bf16(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv);
                    v.z = pack_bf16(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv);
                    v.w = pack_bf16(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv);
                    *reinterpret_cast<uint4 *>(orow + 32 * (c + hh) + 8 * g) = v;
                }
            }
        }
        if (upper && a.lse) a.lse[t * kH + row] = (m_run == -INFINITY) ? a.sink[row] : (m_run + __log2f(den)) * kLn2;
        tc_fence_before();
    }
    return true;
}

// Producers (warps 4-7, 128 threads).  Q rows, window tiles and HCA tiles are contiguous rows:
// one thread issues 2-D TMA loads (64-channel x rows boxes, 128-byte swizzle, rows outside the
// tensor read as zeros) that complete the barrier's transaction count.  CSA tiles are gathered
// through the top-k list by all 128 threads (16-byte loads, swizzled shared stores, proxy fence).
__device__ __forceinline__ bool producer_role(const PrefillArgs &a, const TmaMaps &M, const Smem &S, int ptid)
{
    uint32_t qe_ph = 0, ke_ph[2] = {0, 0};
    bool first_q = true, first_h[2] = {true, true};
    for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
        const int64_t n_cmp = n_compressed(a, t);
        const int64_t nvt = (t + 1) / a.m; // N_vis(t), once per token
        const int nt = n_tiles(n_cmp);
        if (ptid == 0) { // Q [64 rows x 512] = 8 boxes of 64 x 64
            if (!first_q) {
                if (!mbar_wait(S.bar(B_QEMPTY), qe_ph)) return false;
                qe_ph ^= 1;
            }
            mbar_arrive_expect_tx(S.bar(B_QFULL), 65536u);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                tma_load_2d(S.sQ + (uint32_t)s * 8192u, &M.q, 64 * s, (int32_t)(t * kH), S.bar(B_QFULL));
        }
        first_q = false;
        for (int i = 0; i < nt; ++i) {
            const bool gather = (i > 0) && (a.idx != nullptr);
            for (int h = 0; h < 2; ++h) {
                if (!first_h[h]) {
                    if (!mbar_wait(S.bar(B_KVEMPTY0 + h), ke_ph[h])) return false;
                    ke_ph[h] ^= 1;
                }
                first_h[h] = false;
                const uint32_t dst = S.sK + (uint32_t)h * 65536u;
                if (!gather) {
                    if (ptid == 0) {
                        const CUtensorMap *m = (i == 0) ? &M.x : &M.kv;
                        const int32_t y = (i == 0) ? (int32_t)(t - (kW - 1)) : (int32_t)((i - 1) * kKT);
                        mbar_arrive_expect_tx(S.bar(B_KVFULL0 + h), 65536u);
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            tma_load_2d(dst + (uint32_t)s * 16384u, m, 256 * h + 64 * s, y, S.bar(B_KVFULL0 + h));
                    } else {
                        mbar_arrive(S.bar(B_KVFULL0 + h));
                    }
                    continue;
                }
                // gathered half h: 128 keys x 256 channels; thread = (4-key group g, 64-channel box q)
                // issues one gather4 of 512 bytes; empty slots read row 0 and are masked
                const int g = ptid >> 2, q = ptid & 3;
                int32_t rr[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int32_t s = gather_row(a, t, i, 4 * g + u, n_cmp, nvt, h == 0 && q == 0);
                    rr[u] = s < 0 ? 0 : s;
                }
                mbar_arrive_expect_tx(S.bar(B_KVFULL0 + h), 512u);
                tma_gather4(dst + (uint32_t)q * 16384u + (uint32_t)(4 * g) * 128u, &M.kvg, 256 * h + 64 * q, rr[0],
                            rr[1], rr[2], rr[3], S.bar(B_KVFULL0 + h));
            }
        }
    }
    return true;
}

// MMA issue (one thread of warp 8).
__device__ __forceinline__ bool mma_role(const PrefillArgs &a, const Smem &S, uint32_t tmem)
{
    uint32_t q_ph = 0, kf_ph[2] = {0, 0}, p_ph = 0;
    for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
        const int64_t n_cmp = n_compressed(a, t);
        const int nt = n_tiles(n_cmp);
        if (!mbar_wait(S.bar(B_QFULL), q_ph)) return false;
        q_ph ^= 1;
        for (int i = 0; i < nt; ++i) {
            // a compressed tile with at most 64 slots in use (its valid slots come first): half the
            // MMA work (N = 64 for S, 64 keys for P V); the softmax masks the other slots anyway
            const bool half = i > 0 && n_cmp - (int64_t)(i - 1) * kKT <= 64;
            for (int s = 0; s < 8; ++s) {
                if ((s & 3) == 0) { // each key half arrives separately
                    const int h = s >> 2;
                    if (!mbar_wait(S.bar(B_KVFULL0 + h), kf_ph[h])) return false;
                    kf_ph[h] ^= 1;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = sdesc_sw128(S.sQ + (uint32_t)s * 8192u + 32u * kk, 16, 1024);
                    const uint64_t bd = sdesc_sw128(S.sK + (uint32_t)s * 16384u + 32u * kk, 16, 1024);
                    mma_bf16(tmem + kColS, ad, bd, half ? IDESC_S64 : IDESC_S, (s | kk) != 0);
                }
            }
            mma_commit(S.bar(B_SFULL));
            if (i == nt - 1) mma_commit(S.bar(B_QEMPTY));
            if (!mbar_wait(S.bar(B_PFULL), p_ph)) return false;
            p_ph ^= 1;
            tc_fence_after();
            for (int h = 0; h < 2; ++h) {
                for (int kk = 0; kk < (half ? 4 : 8); ++kk) {
                    const uint64_t ad = sdesc_sw128(S.sP + (uint32_t)(kk >> 2) * 8192u + 32u * (kk & 3), 16, 1024);
                    const uint64_t bd = sdesc_sw128(S.sK + (uint32_t)h * 65536u + 2048u * kk, 16384, 1024);
                    mma_bf16(h ? tmem : tmem + TMEM_O, ad, bd, IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(S.bar(B_KVEMPTY0 + h));
            }
            mma_commit(S.bar(B_PVDONE));
        }
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) attn_prefill_tc_kernel(PrefillArgs a, const __grid_constant__ TmaMaps maps)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem_raw + (sbase - raw) + OFF_TMEM);
    Smem S{sbase + OFF_Q, sbase + OFF_K, sbase + OFF_P, sbase + OFF_BAR};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        const uint32_t counts[NUM_BARS] = {1, 1, 128, 128, 1, 1, 1, 128, 1, 1};
        for (int b = 0; b < NUM_BARS; ++b) mbar_init(S.bar(b), counts[b]);
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(sbase + OFF_TMEM, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    if (warp < 4) ok = softmax_role(a, S, tmem, warp, lane);
    else if (warp < kMmaWarp) ok = producer_role(a, maps, S, tid - 128);
    else if (lane == 0) ok = mma_role(a, S, tmem);
    if (!ok) flag_error(a.err, CSA_DEVERR_TIMEOUT);

    if (warp == kMmaWarp && lane == 0) {
        // every MMA issued by this thread completes before TMEM is released
        mma_commit(S.bar(B_FINAL));
        if (!mbar_wait(S.bar(B_FINAL), 0)) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, TMEM_COLS);
}

} // namespace

namespace {

bool encode_rows512(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows)
{
    return tma::encode_bf16_rows(m, base, rows, kC, box_rows);
}

} // namespace

cudaError_t launch_attn_prefill_keys(const PrefillArgs &a, cudaStream_t st, bool *handled);

cudaError_t launch_attn_prefill_tc(const PrefillArgs &a, cudaStream_t st, bool *handled, bool *keys_on_m)
{
    *handled = false;
    *keys_on_m = false;
    if (!a.idx) { // HCA: the kernel with keys on M (measured faster for every-visible-entry layers)
        cudaError_t e = launch_attn_prefill_keys(a, st, handled);
        if (*handled) {
            *keys_on_m = true;
            return e;
        }
    }
    if (a.dtype != CSA_BF16 || a.H != kH || a.c != kC || a.W != kW || a.T <= 0) return cudaSuccess;
    if (a.idx && a.k > 4096) return cudaSuccess;
    if ((uint64_t)a.T * kH >= (1ull << 31)) return cudaSuccess; // TMA row coordinates are int32
    // from here on the call is this kernel's: a tensor map that cannot be encoded is an error
    // (reported as a failed launch), never a silent switch to the CUDA-core kernel
    *handled = true;
    TmaMaps maps;
    if (!encode_rows512(&maps.q, a.q, (uint64_t)a.T * kH, 64) || !encode_rows512(&maps.x, a.x_win, (uint64_t)a.T, kKT))
        return cudaErrorNotSupported;
    const bool have_kv = a.kv_comp != nullptr && a.n_comp > 0;
    if (!encode_rows512(&maps.kv, have_kv ? a.kv_comp : a.x_win, have_kv ? (uint64_t)a.n_comp : (uint64_t)a.T, kKT) ||
        !encode_rows512(&maps.kvg, have_kv ? a.kv_comp : a.x_win, have_kv ? (uint64_t)a.n_comp : (uint64_t)a.T, 1))
        return cudaErrorNotSupported;
    const int sms = device_sms();
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const int64_t grid = a.T < sms ? a.T : sms;
    attn_prefill_tc_kernel<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(a, maps);
    return cudaGetLastError();
}

} // namespace csa
