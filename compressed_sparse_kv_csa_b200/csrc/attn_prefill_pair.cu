// attn_prefill_pair.cu -- HCA prefill attention on a 2-CTA cluster, two tokens per work item.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 step 3 (shared-KV MQA) and Sec. 2.4 Attention.forward listing (window keys and all
// visible compressed keys concatenated); itsolotime.com Q&A essay, Question 1 (window of the most
// recent 128 raw tokens; one sink logit per head in the softmax denominator).
//
// Why this shape: rows = 2 consecutive tokens x 64 heads = 128 (a full-width M=128 MMA), and
// the two tokens share almost all keys (window union of 129 rows, identical HCA entries but at
// block boundaries).  O for 128 rows x 512 fp32 channels would fill all of TMEM, so the two CTAs
// of a cluster split the output channels: CTA r keeps O[:, 256r : 256r+256] (256 TMEM columns)
// and holds only its channel half of Q (64 KB) and of every key tile.
//   * S = Q K^T is split the same way (K-dim = channels): CTA r computes the partial S_r over its
//     256 channels.  Rows are owned half by each CTA (CTA r finalises rows 64r..64r+63): a
//     "sender" warp pair forwards its partial of the peer's rows through distributed shared
//     memory; a "finaliser" pair adds the peer's partial to its own, runs the online softmax,
//     and writes its 64 rows of P (bf16) into BOTH CTAs' P buffers, with the rescale factor of
//     each row for the peer's half of O.
//   * O += P V (M=128, N=256, K=keys) runs in each CTA on its channel half.
//   * 64-key tiles: window tiles [t0-127, t0-64], [t0-63, t0], [t0+1 .. +15] (16 keys, only
//     the second token needs its key t0+1), then tiles of 64 HCA entries (the last one N rounded
//     up to 16).  Keys are masked per row by its own token.
//
// Shared memory per CTA (227 KB budget): Q half 64 KB, K ring 3 x 32 KB, P 2 x 16 KB, exchange
// 2 x 16 KB, alpha / inv 768 B, barriers.  TMEM: O at columns 0-255, four S buffers of 64
// columns at 256-511.
//
// Roles: warps 0-3 softmax (warp w = TMEM lanes 32w..32w+31 = rows; in CTA r warps 2r, 2r+1
// finalise, the other two send), warp 4 producer (TMA), warp 5 TMEM allocation and MMA issue.
// Every wait is bounded; a wait that runs out records CSA_DEVERR_TIMEOUT and the CTA winds
// down.  Both CTAs always reach the final cluster barrier, so neither leaves while the other may
// still write into its shared memory.
#include "common.cuh"
#include "tc_common.cuh"

#include "tma_host.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kH = 64, kC = 512, kW = 128, kKT = 64, kRows = 128, kHalf = 256;
constexpr int kSoftWarps = 4, kProdWarp = 4, kMmaWarp = 5;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kKSlots = 3, kSBufs = 4;

constexpr uint32_t SUB_Q = kRows * 128;              // [128 rows x 64 ch] bf16, 16 KB
constexpr uint32_t SUB_K = kKT * 128;                // [64 keys x 64 ch] bf16, 8 KB
constexpr uint32_t SLOT_K = 4 * SUB_K;               // 64 keys x 256 ch, 32 KB
constexpr uint32_t OFF_Q = 0;                        // 4 x 16 KB
constexpr uint32_t OFF_K = OFF_Q + 4 * SUB_Q;        // 3 x 32 KB
constexpr uint32_t OFF_P = OFF_K + kKSlots * SLOT_K; // 2 x [128 rows x 64 keys] bf16 (16 KB)
constexpr uint32_t OFF_X = OFF_P + 2 * SUB_Q;        // 2 x [16 key groups][64 rows][4] fp32 (16 KB)
constexpr uint32_t OFF_A = OFF_X + 2 * 16384;        // alpha [2][64] fp32, inv [64] fp32
constexpr uint32_t OFF_BAR = OFF_A + 768;
constexpr uint32_t OFF_TMEM = OFF_BAR + 256;
constexpr uint32_t SMEM_USED = OFF_TMEM + 16;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory per block");

enum {
    B_KFULL = 0, B_KEMPTY = B_KFULL + kKSlots, B_QFULL = B_KEMPTY + kKSlots, B_QEMPTY, B_SFULL,
    B_SFREE = B_SFULL + kSBufs, B_XFULL = B_SFREE + kSBufs, B_XFREE = B_XFULL + 2, B_AFULL = B_XFREE + 2,
    B_PFULL = B_AFULL + 2, B_PFREE = B_PFULL + 2, B_PVDONE = B_PFREE + 2, B_EFULL, B_FINAL, NUM_BARS
};
static_assert(NUM_BARS * 8 <= 256, "barrier space");

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kColS = 256; // S buffer b at column 256 + 64 b
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.f;

// ---------------------------------------------------------------------------------------------
// cluster helpers
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t n_clusters_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared::cta offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ void remote_arrive(uint32_t remote_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Bounded wait with cluster-scope acquire (for phases completed by the peer CTA).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint64_t limit_ns = 2000000000ull)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((it & 255u) == 0 && globaltimer() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

__device__ __forceinline__ bool warp_wait_cluster(uint32_t bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_wait_cluster(bar, parity));
}

// Arrive once on `bar` in every CTA of `cta_mask` when this thread's MMAs so far complete.
__device__ __forceinline__ void mma_commit_mc(uint32_t bar, uint16_t cta_mask)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
                 "h"(cta_mask)
                 : "memory");
}

// Orders this thread's earlier shared-memory accesses (local and remote) before a later release
// by another lane of the warp (after __syncwarp): each lane fences its own accesses.
__device__ __forceinline__ void fence_acq_rel_cluster()
{
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_cluster()
{
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

__device__ __forceinline__ void sts16(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void stc16(uint32_t addr, uint4 v)
{
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void stc4(uint32_t addr, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ float lds4(uint32_t addr)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float4 lds16f(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

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

// ---------------------------------------------------------------------------------------------
// the key tiles of a work item (tokens t0 = 2p, t1 = t0 + 1)
// ---------------------------------------------------------------------------------------------

struct Item {
    int64_t t0;
    bool has_t1;  // t0 + 1 < T
    int64_t nv0, nv1; // visible HCA entries of t0 and t1 (nv1 = nv0 without a second token)
    int n_win;    // 2 or 3 window tiles
    int n_tiles;
};

__device__ __forceinline__ int64_t nvis(const PrefillArgs &a, int64_t t)
{
    const int64_t n = (t + 1) / a.m;
    return n < a.n_comp ? n : a.n_comp;
}

__device__ __forceinline__ Item make_item(const PrefillArgs &a, int64_t p)
{
    Item it;
    it.t0 = 2 * p;
    it.has_t1 = it.t0 + 1 < a.T;
    it.nv0 = nvis(a, it.t0);
    it.nv1 = it.has_t1 ? nvis(a, it.t0 + 1) : it.nv0;
    it.n_win = it.has_t1 ? 3 : 2;
    it.n_tiles = it.n_win + (int)((it.nv1 + kKT - 1) / kKT);
    return it;
}

// Tile i of an item: first key (window row u0 or HCA entry s0), keys loaded (rows of the box
// that may be valid), and the MMA width N (a multiple of 16).
struct Tile {
    bool window;
    int64_t k0;
    int nk, n_mma;
};

__device__ __forceinline__ Tile tile_of(const Item &it, int i)
{
    Tile tl;
    if (i < it.n_win) {
        tl.window = true;
        tl.k0 = it.t0 - 127 + (int64_t)kKT * i; // i = 2: key t0 + 1 (the second token only)
        tl.nk = (i < 2) ? kKT : 1;
        tl.n_mma = (i < 2) ? kKT : 16;
    } else {
        tl.window = false;
        tl.k0 = (int64_t)kKT * (i - it.n_win);
        const int64_t left = it.nv1 - tl.k0;
        tl.nk = (int)(left < kKT ? left : kKT);
        tl.n_mma = (tl.nk + 15) & ~15;
    }
    return tl;
}

// Is key j of tile tl visible to token t?
__device__ __forceinline__ bool key_ok(const PrefillArgs &a, const Item &it, const Tile &tl, int j, int64_t t)
{
    if (j >= tl.nk) return false;
    const int64_t u = tl.k0 + j;
    if (tl.window) return u >= 0 && u >= t - (kW - 1) && u <= t;
    return u < (t == it.t0 ? it.nv0 : it.nv1);
}

struct Maps {
    CUtensorMap q, x, kv;
};

struct Smem {
    uint32_t base;
    __device__ uint32_t q(int s) const { return base + OFF_Q + (uint32_t)s * SUB_Q; }
    __device__ uint32_t k(int slot) const { return base + OFF_K + (uint32_t)slot * SLOT_K; }
    __device__ uint32_t p(int b) const { return base + OFF_P + (uint32_t)b * SUB_Q; }
    __device__ uint32_t x(int b) const { return base + OFF_X + (uint32_t)b * 16384u; }
    __device__ uint32_t alpha(int b) const { return base + OFF_A + (uint32_t)b * 256u; }
    __device__ uint32_t inv() const { return base + OFF_A + 512u; }
    __device__ uint32_t bar(int b) const { return base + OFF_BAR + 8u * (uint32_t)b; }
};

// ---------------------------------------------------------------------------------------------
// softmax warps
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ void rescale_rows(uint32_t tw, float f)
{
    for (int c = 0; c < 8; c += 2) {
        uint32_t r[32], r2[32];
        tmem_ld32(tw + 32u * c, r);
        tmem_ld32(tw + 32u * (c + 1), r2);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
            r2[e] = __float_as_uint(__uint_as_float(r2[e]) * f);
        }
        tmem_st32(tw + 32u * c, r);
        tmem_st32(tw + 32u * (c + 1), r2);
    }
    tmem_st_wait();
}

// Normalise this lane's O row (channel half `rank`) by `inv` and store it as bf16.
__device__ __forceinline__ void write_row(const PrefillArgs &a, uint32_t tw, int64_t t, int head, uint32_t rank, float inv)
{
    uint16_t *orow = (uint16_t *)a.o + ((t * kH) + head) * (int64_t)kC + kHalf * rank;
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
}

__device__ __forceinline__ bool softmax_role(const PrefillArgs &a, const Smem &S, uint32_t tmem, uint32_t rank, int warp,
                                             int lane)
{
    const uint32_t peer = rank ^ 1u;
    const bool own = (uint32_t)(warp >> 1) == rank; // finaliser of rows 64 rank .. 64 rank + 63
    const int row = 32 * warp + lane;               // 0..127 = (token half, head)
    const int rho = row & 63;                       // row within its owner's 64
    const int head = row & 63;
    const int tok = row >> 6;                       // 0: t0, 1: t1
    const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);
    const float scale_log2 = a.scale * kLog2e;
    const float sink_l2 = a.sink[head] * kLog2e;
    uint32_t kt = 0; // tiles processed by this CTA so far (all items)
    for (int64_t pi = cluster_id_x(); 2 * pi < a.T; pi += n_clusters_x()) {
        const Item it = make_item(a, pi);
        const int64_t t = it.t0 + tok;
        float m_run = -INFINITY, l_run = 0.f;
        for (int i = 0; i < it.n_tiles; ++i, ++kt) {
            const Tile tl = tile_of(it, i);
            const int sb = (int)(kt % kSBufs), xb = (int)(kt & 1);
            const uint32_t su = kt / kSBufs, xu = kt >> 1;
            if (!warp_wait(S.bar(B_SFULL + sb), su & 1)) return false;
            tc_fence_after();
            float sv[64];
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(tw + kColS + 64u * (uint32_t)sb, r0);
                tmem_ld32(tw + kColS + 64u * (uint32_t)sb + 32u, r1);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    sv[e] = __uint_as_float(r0[e]);
                    sv[32 + e] = __uint_as_float(r1[e]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S.bar(B_SFREE + sb));
            if (!own) {
                // forward the partial S of the peer's row rho into the peer's exchange buffer
                if (xu >= 1 && !warp_wait_cluster(S.bar(B_XFREE + xb), (xu - 1) & 1)) return false;
                const uint32_t dst = mapa(S.x(xb), peer);
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                    uint4 v;
                    v.x = __float_as_uint(sv[4 * g + 0]);
                    v.y = __float_as_uint(sv[4 * g + 1]);
                    v.z = __float_as_uint(sv[4 * g + 2]);
                    v.w = __float_as_uint(sv[4 * g + 3]);
                    stc16(dst + (uint32_t)(g * 64 + rho) * 16u, v);
                }
                fence_acq_rel_cluster();
                __syncwarp();
                if (lane == 0) remote_arrive(mapa(S.bar(B_XFULL + xb), peer));
                // the peer's P rows and rescale factors for these rows
                if (!warp_wait_cluster(S.bar(B_AFULL + xb), xu & 1)) return false;
                const float alpha = lds4(S.alpha(xb) + 4u * (uint32_t)rho);
                if (kt >= 1) {
                    if (!warp_wait(S.bar(B_PVDONE), (kt - 1) & 1)) return false;
                    tc_fence_after();
                }
                if (i > 0 && __any_sync(0xffffffffu, alpha != 1.f)) rescale_rows(tw, alpha);
            } else {
                if (!warp_wait_cluster(S.bar(B_XFULL + xb), xu & 1)) return false;
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                    const float4 v = lds16f(S.x(xb) + (uint32_t)(g * 64 + rho) * 16u);
                    sv[4 * g + 0] += v.x;
                    sv[4 * g + 1] += v.y;
                    sv[4 * g + 2] += v.z;
                    sv[4 * g + 3] += v.w;
                }
                fence_acq_rel_cluster();
                __syncwarp();
                if (lane == 0) remote_arrive(mapa(S.bar(B_XFREE + xb), peer));
                float mt = -INFINITY;
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const float s = key_ok(a, it, tl, e, t) ? sv[e] * scale_log2 : -INFINITY;
                    sv[e] = s;
                    mt = fmaxf(mt, s);
                }
                const float m_new = fmaxf(m_run, mt);
                float resc = 1.f, m_use = m_run;
                if (m_new != -INFINITY && (m_run == -INFINITY || m_new > m_run + kRescaleThreshold)) {
                    resc = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
                    m_use = m_new;
                }
                float ls = 0.f;
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const float pv = (m_use == -INFINITY) ? 0.f : fast_exp2(sv[e] - m_use);
                    sv[e] = pv;
                    ls += pv;
                }
                l_run = l_run * resc + ls;
                m_run = m_use;
                // P buffer xb is free once both CTAs' P V of tile kt - 2 is done
                if (xu >= 1 && !warp_wait_cluster(S.bar(B_PFREE + xb), (xu - 1) & 1)) return false;
                const uint32_t pl = S.p(xb), pr = mapa(S.p(xb), peer);
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    uint4 v;
                    v.x = pack_bf16(sv[8 * g + 0], sv[8 * g + 1]);
                    v.y = pack_bf16(sv[8 * g + 2], sv[8 * g + 3]);
                    v.z = pack_bf16(sv[8 * g + 4], sv[8 * g + 5]);
                    v.w = pack_bf16(sv[8 * g + 6], sv[8 * g + 7]);
                    const uint32_t off = sw128_off((uint32_t)row, (uint32_t)(8 * g));
                    sts16(pl + off, v);
                    stc16(pr + off, v);
                }
                stc4(mapa(S.alpha(xb) + 4u * (uint32_t)rho, peer), (i > 0) ? resc : 1.f);
                fence_proxy_async_cluster();
                fence_acq_rel_cluster();
                __syncwarp();
                if (lane == 0) remote_arrive(mapa(S.bar(B_AFULL + xb), peer));
                if (kt >= 1) {
                    if (!warp_wait(S.bar(B_PVDONE), (kt - 1) & 1)) return false;
                    tc_fence_after();
                }
                if (i > 0 && __any_sync(0xffffffffu, resc != 1.f)) rescale_rows(tw, resc);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S.bar(B_PFULL + xb));
        }
        // epilogue: the item's last P V, then normalise and store this CTA's channel half
        if (!warp_wait(S.bar(B_PVDONE), (kt - 1) & 1)) return false;
        tc_fence_after();
        const bool live = tok == 0 || it.has_t1;
        if (own) {
            const float den = l_run + fast_exp2(sink_l2 - m_run);
            const float inv = (den > 0.f && den < INFINITY) ? 1.f / den : 0.f;
            stc4(mapa(S.inv() + 4u * (uint32_t)rho, peer), inv);
            fence_acq_rel_cluster();
            __syncwarp();
            if (lane == 0) remote_arrive(mapa(S.bar(B_EFULL), peer));
            if (live) {
                write_row(a, tw, t, head, rank, inv);
                if (a.lse) a.lse[t * kH + head] = (m_run == -INFINITY) ? a.sink[head] : (m_run + __log2f(den)) * kLn2;
            }
        } else {
            const uint32_t item_no = (uint32_t)((pi - cluster_id_x()) / n_clusters_x());
            if (!warp_wait_cluster(S.bar(B_EFULL), item_no & 1)) return false;
            const float inv = lds4(S.inv() + 4u * (uint32_t)rho);
            if (live) write_row(a, tw, t, head, rank, inv);
        }
        tc_fence_before();
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// producer and MMA
// ---------------------------------------------------------------------------------------------

// Wait (full limit) for the TMA loads this producer has issued and nobody may consume any more:
// every FULL phase it armed completes when its bytes land, so once these waits return no copy
// into this CTA's shared memory is in flight.  kt = K tiles issued, nq = Q loads issued.
__device__ __forceinline__ void producer_drain(const Smem &S, uint32_t kt, uint32_t nq)
{
    for (uint32_t slot = 0; slot < (uint32_t)kKSlots; ++slot) {
        if (kt <= slot) continue;
        const uint32_t last = (kt - 1 - slot) / kKSlots * kKSlots + slot; // last tile issued into `slot`
        mbar_wait(S.bar(B_KFULL + (int)slot), (last / kKSlots) & 1);
    }
    if (nq > 0) mbar_wait(S.bar(B_QFULL), (nq - 1) & 1);
}

__device__ __forceinline__ bool producer_role(const PrefillArgs &a, const Maps &M, const Smem &S, uint32_t rank)
{
    uint32_t kt = 0, item_no = 0, nq = 0;
    bool ok = true;
    for (int64_t pi = cluster_id_x(); 2 * pi < a.T && ok; pi += n_clusters_x(), ++item_no) {
        const Item it = make_item(a, pi);
        if (item_no >= 1 && !mbar_wait(S.bar(B_QEMPTY), (item_no - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(S.bar(B_QFULL), 4 * SUB_Q);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            tma_load_2d(S.q(s), &M.q, kHalf * (int)rank + 64 * s, (int32_t)(it.t0 * kH), S.bar(B_QFULL));
        ++nq;
        for (int i = 0; i < it.n_tiles; ++i, ++kt) {
            const Tile tl = tile_of(it, i);
            const int slot = (int)(kt % kKSlots);
            const uint32_t use = kt / kKSlots;
            if (use >= 1 && !mbar_wait(S.bar(B_KEMPTY + slot), (use - 1) & 1)) { ok = false; break; }
            mbar_arrive_expect_tx(S.bar(B_KFULL + slot), SLOT_K);
            const CUtensorMap *m = tl.window ? &M.x : &M.kv;
#pragma unroll
            for (int s = 0; s < 4; ++s)
                tma_load_2d(S.k(slot) + (uint32_t)s * SUB_K, m, kHalf * (int)rank + 64 * s, (int32_t)tl.k0,
                            S.bar(B_KFULL + slot));
        }
    }
    producer_drain(S, kt, nq);
    return ok;
}

__device__ __forceinline__ void issue_s(const Smem &S, uint32_t tmem, uint32_t kt, int n_mma)
{
    const int slot = (int)(kt % kKSlots), sb = (int)(kt % kSBufs);
    const uint32_t idesc = idesc_bf16_f32(128, n_mma, false, false);
    for (int s = 0; s < 4; ++s) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(S.q(s) + 32u * kk, 16, 1024);
            const uint64_t bd = sdesc_sw128(S.k(slot) + (uint32_t)s * SUB_K + 32u * kk, 16, 1024);
            mma_bf16(tmem + kColS + 64u * (uint32_t)sb, ad, bd, idesc, (s | kk) != 0);
        }
    }
    mma_commit(S.bar(B_SFULL + sb));
}

__device__ __forceinline__ bool mma_role(const PrefillArgs &a, const Smem &S, uint32_t tmem)
{
    uint32_t kt = 0, item_no = 0;
    for (int64_t pi = cluster_id_x(); 2 * pi < a.T; pi += n_clusters_x(), ++item_no) {
        const Item it = make_item(a, pi);
        if (!mbar_wait(S.bar(B_QFULL), item_no & 1)) return false;
        const uint32_t kt0 = kt;
        // S runs one tile ahead of P V
        auto prep_s = [&](uint32_t k) -> bool {
            const int slot = (int)(k % kKSlots), sb = (int)(k % kSBufs);
            if (!mbar_wait(S.bar(B_KFULL + slot), (k / kKSlots) & 1)) return false;
            if (k / kSBufs >= 1 && !mbar_wait(S.bar(B_SFREE + sb), ((k / kSBufs) - 1) & 1)) return false;
            tc_fence_after();
            issue_s(S, tmem, k, tile_of(it, (int)(k - kt0)).n_mma);
            return true;
        };
        if (!prep_s(kt0)) return false;
        for (int i = 0; i < it.n_tiles; ++i, ++kt) {
            if (i + 1 < it.n_tiles) {
                if (!prep_s(kt + 1)) return false;
            } else {
                mma_commit(S.bar(B_QEMPTY)); // the item's last S has been issued: Q may be replaced
            }
            const int xb = (int)(kt & 1), slot = (int)(kt % kKSlots);
            if (!mbar_wait(S.bar(B_PFULL + xb), (kt >> 1) & 1)) return false;
            tc_fence_after();
            const int nk16 = tile_of(it, i).n_mma / 16;
            for (int kk = 0; kk < nk16; ++kk) {
                const uint64_t ad = sdesc_sw128(S.p(xb) + 32u * kk, 16, 1024);
                const uint64_t bd = sdesc_sw128(S.k(slot) + 2048u * kk, SUB_K, 1024);
                mma_bf16(tmem, ad, bd, IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(S.bar(B_KEMPTY + slot));
            mma_commit(S.bar(B_PVDONE));
            mma_commit_mc(S.bar(B_PFREE + xb), 0x3);
        }
    }
    return true;
}

// Launched in clusters of 2 CTAs (launch attribute; see launch_attn_prefill_pair).
__global__ void __launch_bounds__(kThreads, 1) attn_prefill_pair_kernel(PrefillArgs a, const __grid_constant__ Maps maps)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem_raw + (sbase - raw) + OFF_TMEM);
    const Smem S{sbase};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();

    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            uint32_t count = 1;
            if (b >= B_SFREE && b < B_SFREE + kSBufs) count = kSoftWarps;
            else if (b >= B_XFULL && b < B_PFULL) count = 2;      // XFULL, XFREE, AFULL: two peer warps
            else if (b >= B_PFULL && b < B_PFULL + 2) count = kSoftWarps;
            else if (b >= B_PFREE && b < B_PFREE + 2) count = 2;  // one commit from each CTA
            else if (b == B_EFULL) count = 2;
            mbar_init(S.bar(b), count);
        }
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(sbase + OFF_TMEM, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all(); // the peer's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    if (warp < kSoftWarps) ok = softmax_role(a, S, tmem, rank, warp, lane);
    else if (warp == kProdWarp) { if (lane == 0) ok = producer_role(a, maps, S, rank); }
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
    cluster_sync_all(); // neither CTA leaves while the other may still write into its shared memory
}

} // namespace

// HCA prefill (every visible entry, no top-k list) of the 64-head x 512-channel bf16 shape with a
// 128-token window; *handled = false leaves the call to the other paths.
cudaError_t launch_attn_prefill_pair(const PrefillArgs &a, cudaStream_t st, bool *handled)
{
    *handled = false;
    if (a.idx || a.dtype != CSA_BF16 || a.H != kH || a.c != kC || a.W != kW || a.T <= 0) return cudaSuccess;
    if ((uint64_t)a.T * kH >= (1ull << 31)) return cudaSuccess;
    Maps maps;
    if (!tma::encode_bf16_rows(&maps.q, a.q, (uint64_t)a.T * kH, kC, kRows) ||
        !tma::encode_bf16_rows(&maps.x, a.x_win, (uint64_t)a.T, kC, kKT))
        return cudaSuccess;
    const bool have_kv = a.kv_comp != nullptr && a.n_comp > 0;
    if (!tma::encode_bf16_rows(&maps.kv, have_kv ? a.kv_comp : a.x_win, have_kv ? (uint64_t)a.n_comp : (uint64_t)a.T,
                               kC, kKT))
        return cudaSuccess;
    *handled = true;
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_ALLOC;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2);
    int max_clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&max_clusters, attn_prefill_pair_kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (max_clusters < 1) return cudaErrorInvalidConfiguration;
    const int64_t items = (a.T + 1) / 2;
    const int64_t clusters = items < max_clusters ? items : max_clusters;
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    return cudaLaunchKernelEx(&cfg, attn_prefill_pair_kernel, a, maps);
}

} // namespace csa
