// attn_prefill_keys.cu -- hybrid MQA prefill attention on the 5th-generation tensor cores
// (tcgen05 + TMEM) for the 64-head x 512-channel bf16 shape with a 128-token window, with the
// keys (and output channels) on the MMA's M dimension.  Used for HCA layers (every visible
// entry); CSA layers (top-k lists) use attn_prefill_tc.cu, which measured faster there.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 step 3 (shared-KV multi-query attention: all heads share one key vector, which is also
// the value vector) and Sec. 2.4 Attention.forward listing (the sliding-window keys and the
// selected / all visible compressed keys are concatenated, no de-duplication, one sparse
// attention over both); itsolotime.com Q&A essay on DeepSeek-V4, Question 1: window of the most
// recent 128 raw tokens (mechanism 1) and one learnable sink logit per head in the softmax
// denominator (mechanism 3).
//
// Design (one query token per CTA pass, persistent CTAs).  One token has only 64 query rows, and
// an M=64 MMA runs at half the tensor-core rate, so the products are taken transposed, with the
// 128 keys of a tile (and the 128 channels of an output quarter) on M:
//   * S^T = K Q^T: A = the key tile [128 keys x 512 ch] (K-major), B = Q [64 heads x 512 ch]
//     (K-major); M=128, N=64, K=512.  TMEM lane = key, column = head (64 columns at kColS).
//   * O^T += V^T P^T: A = the same key tile read MN-major (M = the 128 channels of quarter c),
//     B = P^T [64 heads x 128 keys] (K-major); M=128, N=64, K=128.  O^T of quarter c at columns
//     64c .. 64c+63, TMEM lane = channel 128c + lane; the whole 512 x 64 fp32 output stays in TMEM
//     for the token's key loop.
//   * Softmax over the keys = across TMEM lanes.  Eight warps: warps w and w+4 reach the lanes of
//     keys 32(w%4) .. 32(w%4)+31 and take heads 0-31 and 32-63 of them.  Per-head maxima go
//     through bf16 copies of the scores in the P^T buffer (four threads per head row, with a
//     margin for the copy's rounding); per-head sums in fp32 by a warp reduce-scatter, added
//     across the lane quarters at the end of the token.  Online softmax in the log2 domain with a
//     lazy rescale: a head's running max moves (and its O^T column is rescaled in TMEM) only when
//     a tile raises it by more than 8.
//   * The key tile arrives in four channel quarters; quarter c is released as soon as the O^T MMAs
//     of quarter c complete, so the next tile's loads overlap the rest of P V.
//   * Keys per token: tile 0 = window rows t-127..t of x_win; then tiles of 128 compressed rows
//     (every visible entry for HCA: 2-D TMA boxes; the top-k list for CSA: TMA gather4, 4 rows x 64
//     channels per instruction).  Invalid slots are masked; their rows are zeros (outside the
//     tensor) or a real row (gather of row 0), so P V stays finite.
//   * Roles: warps 0-7 softmax / rescale / epilogue, warps 8-11 producers, warp 12 TMEM allocation
//     and (one lane) MMA issue.  Every wait is an mbarrier wait bounded by %globaltimer; a wait
//     that runs out records CSA_DEVERR_TIMEOUT and the CTA winds down without trapping.
#include "common.cuh"
#include "tc_common.cuh"

#include "tma_host.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kH = 64, kC = 512, kKT = 128, kW = 128;
constexpr int kSoftWarps = 8, kProdWarp0 = 8, kMmaWarp = 12;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kSoftBar = 1; // named barrier of the softmax warps

constexpr uint32_t OFF_Q = 0;          // 8 sub-tiles [64 heads x 128 B]          64 KB
constexpr uint32_t OFF_K = 65536;      // 8 sub-tiles [128 keys x 128 B]          128 KB
constexpr uint32_t OFF_P = 196608;     // P^T: 2 sub-tiles [64 heads x 128 B]     16 KB
constexpr uint32_t OFF_RED = 212992;   // per head: running max, rescale factor, 1 / denominator; sums [4][64] (fp32)
constexpr uint32_t OFF_BAR = OFF_RED + 7 * 64 * 4;
constexpr uint32_t OFF_TMEM = OFF_BAR + 128;
constexpr uint32_t SMEM_USED = OFF_BAR + 256;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024; // slack to align the base to 1024 bytes
static_assert(SMEM_ALLOC <= 232448, "shared memory per block");

enum { B_QFULL = 0, B_QEMPTY, B_KFULL0, B_KEMPTY0 = B_KFULL0 + 4, B_SFULL = B_KEMPTY0 + 4, B_PFULL, B_PVDONE,
       B_FINAL, NUM_BARS };
static_assert(NUM_BARS * 8 <= 128, "barrier space");

constexpr uint32_t IDESC_ST = idesc_bf16_f32(128, 64, false, false); // S^T = K Q^T
constexpr uint32_t IDESC_OT = idesc_bf16_f32(128, 64, true, false);  // O^T += V^T P^T (A MN-major)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kColS = 256; // S^T; O^T quarter c at 64c
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

// Whether slot j of tile i holds a key of token t (nvt = N_vis(t)).
__device__ __forceinline__ bool key_ok(const PrefillArgs &a, int64_t t, int i, int j, int64_t n_cmp, int64_t nvt)
{
    if (i == 0) return t - (kW - 1) + j >= 0;
    const int64_t slot = (int64_t)(i - 1) * kKT + j;
    if (slot >= n_cmp) return false;
    if (!a.idx) return true;
    const int32_t s = a.idx[t * a.k + slot];
    return s >= 0 && s < a.n_comp && s < nvt;
}

// Compressed row of slot j of CSA tile i for token t, or -1 when the slot is empty or invalid
// (a missing or not yet visible entry is reported).
__device__ __forceinline__ int32_t gather_row(const PrefillArgs &a, int64_t t, int i, int j, int64_t n_cmp,
                                              int64_t nvt, bool report)
{
    const int64_t slot = (int64_t)(i - 1) * kKT + j;
    if (slot >= n_cmp) return -1;
    const int32_t s = a.idx[t * a.k + slot];
    if (s >= a.n_comp || s >= nvt) {
        if (report) flag_error(a.err, CSA_DEVERR_INDEX);
        return -1;
    }
    return s;
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

__device__ __forceinline__ void soft_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kSoftBar), "n"(kSoftThreads) : "memory"); }

__device__ __forceinline__ void sts16(uint32_t addr, uint16_t v)
{
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint16_t bf16_bits(float x)
{
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Tensor maps of q viewed as [T*64, 512], of x_win [T, 512] and of kv_comp [n_comp, 512], all
// bf16 with 64-channel boxes and 128-byte swizzle (rows: 64 for q, 128 for keys, 1 for the
// gather map of kv_comp).
struct TmaMaps {
    CUtensorMap q, x, kv, kvg;
};

struct Smem {
    uint32_t sQ, sK, sP, bars;
    float *red; // per head: m_use [64], resc [64], inv [64]
    __device__ uint32_t bar(int b) const { return bars + 8u * (uint32_t)b; }
    __device__ float *m_use() const { return red; }
    __device__ float *resc() const { return red + 64; }
    __device__ float *inv() const { return red + 128; }
    __device__ float *lsum(int q) const { return red + 192 + 64 * q; }
};

// Softmax / rescale / epilogue (warps 0-7).  Warps w and w + 4 reach TMEM lanes 32(w%4) ..
// 32(w%4)+31 (keys of the tile, channels of an O^T quarter); warp w takes heads 32(w/4) ..
// 32(w/4)+31 of those lanes.  Per-head maxima go through bf16 copies of the scores in the P^T
// buffer, four threads per head row (32 keys each); per-head sums in fp32 by a warp
// reduce-scatter (lane l ends with head 32(w/4) + l over the warp's 32 keys), kept per warp and
// added across the four lane quarters at the end of the token.  Returns false when a wait ran out.
__device__ __forceinline__ bool softmax_role(const PrefillArgs &a, const Smem &S, uint32_t tmem, int warp, int lane)
{
    const float scale_log2 = a.scale * kLog2e;
    const int quad = warp & 3, hf = warp >> 2;
    const uint32_t tw = tmem + ((uint32_t)(32 * quad) << 16);
    const int tid = 32 * warp + lane;
    const int key = 32 * quad + lane;                      // this thread's key of the tile
    const uint32_t pkey = S.sP + (uint32_t)(key >> 6) * 8192u;
    const uint32_t kcol = (uint32_t)(key & 63);
    const int hh = tid >> 2, kq = tid & 3;                  // head row and key quarter of the max pass
    const uint32_t prow = S.sP + (uint32_t)(kq >> 1) * 8192u + (uint32_t)hh * 128u;
    const int my_head = 32 * hf + lane;                     // head of this lane's partial sums
    uint32_t s_ph = 0, n_tiles_done = 0;
    for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
        const int64_t n_cmp = n_compressed(a, t);
        const int64_t nvt = (t + 1) / a.m;
        const int nt = n_tiles(n_cmp);
        float m_run = -INFINITY; // head hh (identical on its four threads)
        float l_w = 0.f;         // head my_head over this warp's keys
        for (int i = 0; i < nt; ++i, ++n_tiles_done) {
            const bool valid = key_ok(a, t, i, key, n_cmp, nvt);
            // S^T of tile i complete implies P V of tile i-1 complete (one thread commits both, in order)
            if (!warp_wait(S.bar(B_SFULL), s_ph)) return false;
            s_ph ^= 1;
            tc_fence_after();
            float s[32];
            {
                uint32_t r[32];
                tmem_ld32(tw + kColS + 32u * hf, r);
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < 32; ++h) s[h] = valid ? __uint_as_float(r[h]) * scale_log2 : -INFINITY;
            }
            soft_sync(); // every thread is done with the previous tile's P^T
#pragma unroll
            for (int h = 0; h < 32; ++h) sts16(pkey + sw128_off((uint32_t)(32 * hf + h), kcol), bf16_bits(s[h]));
            soft_sync();
            { // head hh: tile max over the bf16 copies, running max with the lazy rescale
                float mt = -INFINITY;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t ch = (uint32_t)((4 * (kq & 1) + g) ^ (hh & 7));
                    const uint4 v = lds128(prow + 16u * ch);
                    mt = fmaxf(mt, fmaxf(fmaxf(bf16_lo(v.x), bf16_hi(v.x)), fmaxf(bf16_lo(v.y), bf16_hi(v.y))));
                    mt = fmaxf(mt, fmaxf(fmaxf(bf16_lo(v.z), bf16_hi(v.z)), fmaxf(bf16_lo(v.w), bf16_hi(v.w))));
                }
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
                // a bf16 copy is within 2^-8 of the score: the margin keeps every 2^(s - m) <= 2^8
                mt = (mt == -INFINITY) ? mt : mt + fabsf(mt) * (1.f / 128.f);
                const float m_new = fmaxf(m_run, mt);
                float resc = 1.f, m_use = m_run;
                if (m_new != -INFINITY && (m_run == -INFINITY || m_new > m_run + kRescaleThreshold)) {
                    resc = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
                    m_use = m_new;
                }
                m_run = m_use;
                if (kq == 0) {
                    S.m_use()[hh] = m_use;
                    S.resc()[hh] = resc;
                }
            }
            soft_sync();
            // P^T = 2^(s - m_use[head]) (0 for a head with no key yet)
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const float4 m4 = *reinterpret_cast<const float4 *>(S.m_use() + 32 * hf + 4 * g);
                const float mh[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int h = 4 * g + u;
                    s[h] = (mh[u] == -INFINITY) ? 0.f : fast_exp2(s[h] - mh[u]);
                    sts16(pkey + sw128_off((uint32_t)(32 * hf + h), kcol), bf16_bits(s[h]));
                }
            }
            { // fp32 sums: warp reduce-scatter of the 32 heads, lane l ends with head 32 hf + l
                float a16[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const bool up = lane & 16;
                    const float keep = up ? s[16 + q] : s[q], send = up ? s[q] : s[16 + q];
                    a16[q] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int n = 8; n >= 1; n >>= 1) {
                    const bool up = lane & n;
#pragma unroll
                    for (int q = 0; q < n; ++q) {
                        const float keep = up ? a16[n + q] : a16[q], send = up ? a16[q] : a16[n + q];
                        a16[q] = keep + __shfl_xor_sync(0xffffffffu, send, n);
                    }
                }
                // after the rounds lane l holds head 16 b4 + 8 b3 + 4 b2 + 2 b1 + b0 = l of the half
                l_w = l_w * S.resc()[my_head] + a16[0];
            }
            if (i > 0) { // O^T columns of the heads whose max moved (P V of tile i-1 is complete)
                bool any = false;
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                    const float4 r4 = *reinterpret_cast<const float4 *>(S.resc() + 4 * g);
                    any |= (r4.x != 1.f) | (r4.y != 1.f) | (r4.z != 1.f) | (r4.w != 1.f);
                }
                if (any) { // the same answer on every thread
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tw + 64u * c + 32u * hf, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < 32; ++h)
                            r[h] = __float_as_uint(__uint_as_float(r[h]) * S.resc()[32 * hf + h]);
                        tmem_st32(tw + 64u * c + 32u * hf, r);
                    }
                    tmem_st_wait();
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(S.bar(B_PFULL));
        }
        // epilogue: the token's last P V, sums across the lane quarters, normalise, write o and lse
        if (!warp_wait(S.bar(B_PVDONE), (n_tiles_done - 1) & 1)) return false;
        tc_fence_after();
        S.lsum(quad)[my_head] = l_w;
        soft_sync();
        if (kq == 0) {
            const float l = S.lsum(0)[hh] + S.lsum(1)[hh] + S.lsum(2)[hh] + S.lsum(3)[hh];
            const float den = l + fast_exp2(a.sink[hh] * kLog2e - m_run);
            S.inv()[hh] = (den > 0.f && den < INFINITY) ? 1.f / den : 0.f;
            if (a.lse) a.lse[t * kH + hh] = (m_run == -INFINITY) ? a.sink[hh] : (m_run + __log2f(den)) * kLn2;
        }
        soft_sync();
        const bool odd = lane & 1;
        for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tw + 64u * c + 32u * hf, r);
            tmem_ld_wait();
            // lanes l, l^1 hold consecutive channels: even lanes store the channel pair of an even
            // head, odd lanes that of an odd head
            const int ch = 128 * c + 32 * quad + (lane & ~1);
            uint16_t *obase = (uint16_t *)a.o + (t * kH + 32 * hf) * (int64_t)kC + ch;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float2 iv = *reinterpret_cast<const float2 *>(S.inv() + 32 * hf + 2 * q);
                const float x0 = __uint_as_float(r[2 * q]) * iv.x, x1 = __uint_as_float(r[2 * q + 1]) * iv.y;
                const float send = odd ? x0 : x1;
                const float rr = __shfl_xor_sync(0xffffffffu, send, 1);
                const int h = 2 * q + (odd ? 1 : 0);
                *reinterpret_cast<uint32_t *>(obase + (int64_t)h * kC) = odd ? pack_bf16(rr, x1) : pack_bf16(x0, rr);
            }
        }
        tc_fence_before();
    }
    return true;
}

// Producers (warps 8-11, 128 threads).  Q rows, window tiles and HCA tiles are contiguous rows:
// one thread issues 2-D TMA loads (64-channel x rows boxes, 128-byte swizzle, rows outside the
// tensor read as zeros) that complete the quarter's transaction count.  CSA tiles are gathered
// through the top-k list: 64 threads per quarter, one gather4 (4 rows x 64 channels) each.
__device__ __forceinline__ bool producer_role(const PrefillArgs &a, const TmaMaps &M, const Smem &S, int ptid)
{
    uint32_t qe_ph = 0, ke_ph[4] = {0, 0, 0, 0};
    bool first_q = true, first_k = true;
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
            int32_t rr[4] = {0, 0, 0, 0};
            if (gather && ptid < 64) { // this thread's 4-key group (the same in every quarter)
                const int g = ptid >> 1;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int32_t s = gather_row(a, t, i, 4 * g + u, n_cmp, nvt, (ptid & 1) == 0);
                    rr[u] = s < 0 ? 0 : s;
                }
            }
            for (int c = 0; c < 4; ++c) {
                if (!first_k) {
                    if (!mbar_wait(S.bar(B_KEMPTY0 + c), ke_ph[c])) return false;
                    ke_ph[c] ^= 1;
                }
                const uint32_t dst = S.sK + (uint32_t)(2 * c) * 16384u; // sub-tiles 2c, 2c+1
                if (!gather) {
                    if (ptid == 0) {
                        const CUtensorMap *m = (i == 0) ? &M.x : &M.kv;
                        const int32_t y = (i == 0) ? (int32_t)(t - (kW - 1)) : (int32_t)((i - 1) * kKT);
                        mbar_arrive_expect_tx(S.bar(B_KFULL0 + c), 32768u);
                        tma_load_2d(dst, m, 128 * c, y, S.bar(B_KFULL0 + c));
                        tma_load_2d(dst + 16384u, m, 128 * c + 64, y, S.bar(B_KFULL0 + c));
                    } else {
                        mbar_arrive(S.bar(B_KFULL0 + c));
                    }
                } else if (ptid < 64) { // 32 groups of 4 keys x 2 boxes of 64 channels
                    const int g = ptid >> 1, q = ptid & 1;
                    mbar_arrive_expect_tx(S.bar(B_KFULL0 + c), 512u);
                    tma_gather4(dst + (uint32_t)q * 16384u + (uint32_t)(4 * g) * 128u, &M.kvg, 128 * c + 64 * q, rr[0],
                                rr[1], rr[2], rr[3], S.bar(B_KFULL0 + c));
                } else {
                    mbar_arrive(S.bar(B_KFULL0 + c));
                }
            }
            first_k = false;
        }
    }
    return true;
}

// MMA issue (one thread of warp 8).
__device__ __forceinline__ bool mma_role(const PrefillArgs &a, const Smem &S, uint32_t tmem)
{
    uint32_t q_ph = 0, kf_ph[4] = {0, 0, 0, 0}, p_ph = 0;
    for (int64_t t = blockIdx.x; t < a.T; t += gridDim.x) {
        const int64_t n_cmp = n_compressed(a, t);
        const int nt = n_tiles(n_cmp);
        if (!mbar_wait(S.bar(B_QFULL), q_ph)) return false;
        q_ph ^= 1;
        for (int i = 0; i < nt; ++i) {
            // S^T = K Q^T over the 8 channel sub-tiles, each quarter as it arrives
            for (int s = 0; s < 8; ++s) {
                if ((s & 1) == 0) {
                    const int c = s >> 1;
                    if (!mbar_wait(S.bar(B_KFULL0 + c), kf_ph[c])) return false;
                    kf_ph[c] ^= 1;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = sdesc_sw128(S.sK + (uint32_t)s * 16384u + 32u * kk, 16, 1024);
                    const uint64_t bd = sdesc_sw128(S.sQ + (uint32_t)s * 8192u + 32u * kk, 16, 1024);
                    mma_bf16(tmem + kColS, ad, bd, IDESC_ST, (s | kk) != 0);
                }
            }
            mma_commit(S.bar(B_SFULL));
            if (i == nt - 1) mma_commit(S.bar(B_QEMPTY));
            if (!mbar_wait(S.bar(B_PFULL), p_ph)) return false;
            p_ph ^= 1;
            tc_fence_after();
            // O^T (+)= V^T P^T per channel quarter; the quarter's key sub-tiles are free after it
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = sdesc_sw128(S.sK + (uint32_t)(2 * c) * 16384u + 2048u * kk, 16384, 1024);
                    const uint64_t bd = sdesc_sw128(S.sP + (uint32_t)(kk >> 2) * 8192u + 32u * (kk & 3), 16, 1024);
                    mma_bf16(tmem + 64u * (uint32_t)c, ad, bd, IDESC_OT, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(S.bar(B_KEMPTY0 + c));
            }
            mma_commit(S.bar(B_PVDONE));
        }
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) attn_prefill_keys_kernel(PrefillArgs a, const __grid_constant__ TmaMaps maps)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - raw);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sp + OFF_TMEM);
    Smem S{sbase + OFF_Q, sbase + OFF_K, sbase + OFF_P, sbase + OFF_BAR, reinterpret_cast<float *>(sp + OFF_RED)};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            uint32_t cnt = 1;
            if (b >= B_KFULL0 && b < B_KFULL0 + 4) cnt = 128; // every producer thread arrives
            if (b == B_PFULL) cnt = kSoftThreads;            // every softmax thread arrives
            mbar_init(S.bar(b), cnt);
        }
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(sbase + OFF_TMEM, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    if (warp < kSoftWarps) ok = softmax_role(a, S, tmem, warp, lane);
    else if (warp < kMmaWarp) ok = producer_role(a, maps, S, tid - 32 * kProdWarp0);
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

cudaError_t launch_attn_prefill_keys(const PrefillArgs &a, cudaStream_t st, bool *handled)
{
    *handled = false;
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
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const int64_t grid = a.T < sms ? a.T : sms;
    attn_prefill_keys_kernel<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(a, maps);
    return cudaGetLastError();
}

} // namespace csa
