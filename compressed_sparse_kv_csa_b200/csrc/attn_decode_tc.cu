// attn_decode_tc.cu -- hybrid MQA decode attention on tcgen05 for 64 heads x 512 channels over the
// mixed FP8/BF16 caches: one new token per sequence, split-K over chunks of its key list.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 step 3 (shared-KV multi-query attention, the key vector is also the value vector) and
// Sec. 2.4 Attention.forward listing (window keys and selected / all visible compressed keys,
// concatenated); KV cache with BF16 RoPE dims and FP8 for the rest ("Mind Observatory: Uncovering
// the technical ledger of DeepSeek-V4"); the per-head sink is folded in by the merge kernel.
//
// Work items = (sequence, chunk of `chunk` keys); persistent CTAs walk the items.  Inside an
// item the 64-key tiles flow through a pipeline, so the next tile's rows are being gathered
// while the current one is in S, softmax and P V:
//   * warps 4-7 (gather): stage q [64 x 512] per item; per tile resolve the 64 key slots
//     (window row, top-k / visible compressed row, or empty), load each row's scale once, load
//     the rows with 16-byte loads (18 per thread in flight), dequantise the FP8 part (code x
//     row scale) to bf16 next to the BF16 RoPE part, and store them 128-byte-swizzled into one
//     of two key buffers (empty rows as zeros);
//   * warp 8 lane 0 (MMA): S = Q K^T (M=64, N=64, K=512) into one of two TMEM S tiles, one tile
//     ahead of O (+)= P V (two M=64 x N=256 x K=64 MMAs, V = the same key buffer read MN-major);
//   * warps 0-3 (softmax): as before (lanes l and l+16 split the tile's keys; lazy rescale of O
//     in TMEM when the max rises by more than 8), P into one of two buffers; at the end of the
//     item the (max, sum, unnormalised O) rows go to the workspace for the split-K merge.
// Every wait of the pipeline is bounded by a.wait_ns (2 s unless a caller lowers it); a wait that
// runs out records CSA_DEVERR_TIMEOUT and its role returns.  The wind-down is then safe because
// nothing asynchronous but the MMAs writes into this CTA: q and the key tiles are stored by the
// gather threads themselves (no TMA, no cp.async), and the MMA lane's final commit is waited for
// with the full 2 s limit before TMEM is released and the CTA exits.
#include "common.cuh"
#include "tc_common.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kH = 64, kC = 512, kKT = 64;
constexpr int kSoftWarps = 4, kGatherWarp0 = 4, kGatherWarps = 4, kMmaWarp = 8;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kGatherThreads = 32 * kGatherWarps;
constexpr int kGatherBar = 1; // named barrier of the gather warps

constexpr uint32_t SUB_Q = 64 * 128;              // [64 heads x 64 ch] bf16, 8 KB
constexpr uint32_t SUB_K = kKT * 128;             // [64 keys x 64 ch] bf16, 8 KB
constexpr uint32_t BUF_K = 8 * SUB_K;             // 64 keys x 512 ch, 64 KB
constexpr uint32_t OFF_Q = 0;                     // 8 x 8 KB
constexpr uint32_t OFF_K = OFF_Q + 8 * SUB_Q;     // 2 x 64 KB
constexpr uint32_t OFF_P = OFF_K + 2 * BUF_K;     // 2 x [64 x 128 B]
constexpr uint32_t OFF_VALID = OFF_P + 2 * 8192;  // 2 x 64 int32
constexpr uint32_t OFF_ROWS = OFF_VALID + 512;    // 64 int64 (gather warps only)
constexpr uint32_t OFF_SCALE = OFF_ROWS + 512;    // 64 fp32 (gather warps only)
constexpr int kSeqCache = 1024;
constexpr uint32_t OFF_SEQ = OFF_SCALE + 256;     // n_win [kSeqCache], n_keys [kSeqCache]
constexpr uint32_t OFF_BAR = OFF_SEQ + 8 * kSeqCache;
constexpr uint32_t OFF_TMEM = OFF_BAR + 128;
constexpr uint32_t SMEM_ALLOC = OFF_TMEM + 16 + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory per block");

enum { B_KFULL = 0, B_KEMPTY = 2, B_SFULL = 4, B_SFREE = 6, B_PFULL = 8, B_PVDONE = 10, B_QFULL, B_QEMPTY, B_FINAL,
       NUM_BARS };
static_assert(NUM_BARS * 8 <= 128, "barrier space");

constexpr uint32_t TMEM_O = 16u << 16; // O[:, 0:256] in the lower lane half; O[:, 256:512] upper
constexpr uint32_t kColS = 256;        // S tile b at columns 256 + 64 b (upper lane half)
constexpr uint32_t IDESC_S = idesc_bf16_f32(64, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(64, 256, false, true);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void sts4(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pk_bf16(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 8 FP8 E4M3 codes (one uint2) times the row scale -> 8 bf16 (one uint4)
__device__ __forceinline__ uint4 fp8x8_to_bf16(uint32_t w0, uint32_t w1, float s)
{
    const uint32_t w[2] = {w0, w1};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffff), __NV_E4M3);
        const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3);
        const float2 a = __half22float2(__half2(lo)), b = __half22float2(__half2(hi));
        o[2 * i] = pk_bf16(a.x * s, a.y * s);
        o[2 * i + 1] = pk_bf16(b.x * s, b.y * s);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit_ns));
}

__device__ __forceinline__ void gather_sync()
{
    asm volatile("bar.sync %0, %1;" ::"n"(kGatherBar), "n"(kGatherThreads) : "memory");
}

// The gather warps' collective verdict: true only if every gather thread passes `ok`.  The four
// warps then take the same branch, so none can be left behind at a later gather_sync().
__device__ __forceinline__ bool gather_all(bool ok)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.and.pred q, %2, %3, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)ok), "n"(kGatherBar), "n"(kGatherThreads)
                 : "memory");
    return r != 0;
}

struct Counts {
    int n_win;
    int64_t n_keys;
};

__device__ __forceinline__ Counts seq_counts(const DecodeArgs &a, int b)
{
    Counts r;
    r.n_win = a.win_len[b] < 0 ? 0 : (a.win_len[b] > a.W ? a.W : a.win_len[b]);
    int64_t nc;
    if (a.idx) nc = a.k;
    else {
        nc = (a.pos[b] + 1) / a.m;
        if (nc > a.max_nvis) nc = a.max_nvis;
        if (nc < 0) nc = 0;
    }
    r.n_keys = r.n_win + nc;
    return r;
}

// The item's tile range [t_beg, t_end) in 64-key tiles (empty when t_beg >= t_end).
struct ItemTiles {
    int b;
    int n_win;
    int64_t n_keys, t_beg, t_end;
};

// Entries of sequence b that its new token may see: min(N_vis(pos[b]), max_nvis).
__device__ __forceinline__ int64_t seq_nvis(const DecodeArgs &a, int b)
{
    int64_t nv = (a.pos[b] + 1) / a.m;
    return nv > a.max_nvis ? a.max_nvis : nv;
}

__device__ __forceinline__ ItemTiles item_tiles(const DecodeArgs &a, const int *s_nwin, const int *s_nkeys, int64_t item)
{
    ItemTiles it;
    it.b = (int)(item / a.n_chunks);
    const int chunk = (int)(item % a.n_chunks);
    if (it.b < kSeqCache) {
        it.n_win = s_nwin[it.b];
        it.n_keys = s_nkeys[it.b];
    } else {
        const Counts c = seq_counts(a, it.b);
        it.n_win = c.n_win;
        it.n_keys = c.n_keys;
    }
    const int tpc = a.chunk / kKT;
    const int64_t n_tiles = (it.n_keys + kKT - 1) / kKT;
    it.t_beg = (int64_t)chunk * tpc;
    it.t_end = it.t_beg + tpc < n_tiles ? it.t_beg + tpc : n_tiles;
    return it;
}

struct Smem {
    uint32_t base;
    uint8_t *p;
    __device__ uint32_t q(int s) const { return base + OFF_Q + (uint32_t)s * SUB_Q; }
    __device__ uint32_t k(int kb) const { return base + OFF_K + (uint32_t)kb * BUF_K; }
    __device__ uint32_t pb(int b) const { return base + OFF_P + (uint32_t)b * 8192u; }
    __device__ int *valid(int kb) const { return reinterpret_cast<int *>(p + OFF_VALID) + 64 * kb; }
    __device__ int64_t *rows() const { return reinterpret_cast<int64_t *>(p + OFF_ROWS); }
    __device__ float *scale() const { return reinterpret_cast<float *>(p + OFF_SCALE); }
    __device__ uint32_t bar(int b) const { return base + OFF_BAR + 8u * (uint32_t)b; }
};

// ---------------------------------------------------------------------------------------------
// gather warps
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ bool gather_role(const DecodeArgs &a, const Smem &S, const int *s_nwin, const int *s_nkeys,
                                            int gtid)
{
    const int warp = gtid >> 5, lane = gtid & 31;
    const int cn = kC - a.comp.rope_dims;         // FP8 channels (448), RoPE after them
    const int fp8_units = cn / 16;                // 16-byte FP8 loads per row (28)
    const int units = fp8_units + a.comp.rope_dims / 8; // + 16-byte RoPE loads (8): 36 per row
    const int64_t n_items = (int64_t)a.B * a.n_chunks;
    uint32_t kt = 0, nitem = 0;
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        const ItemTiles it = item_tiles(a, s_nwin, s_nkeys, item);
        if (it.t_beg >= it.t_end) continue;
        const int64_t n_vis = a.idx ? seq_nvis(a, it.b) : INT64_MAX;
        // ---- q of the item, once the previous item's last S has consumed the old one
        if (!gather_all(nitem == 0 || mbar_wait(S.bar(B_QEMPTY), (nitem - 1) & 1, a.wait_ns))) return false;
        for (int e0 = gtid; e0 < kH * (kC / 8); e0 += 16 * kGatherThreads) {
            uint4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int e = e0 + u * kGatherThreads;
                if (e < kH * (kC / 8))
                    v[u] = __ldg(reinterpret_cast<const uint4 *>(a.q + ((int64_t)it.b * kH + (e >> 6)) * kC + 8 * (e & 63)));
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int e = e0 + u * kGatherThreads;
                if (e < kH * (kC / 8)) {
                    const int h = e >> 6, cc = e & 63;
                    sts4(S.q(cc >> 3) + sw128_off(h, (cc & 7) * 8), v[u]);
                }
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.bar(B_QFULL));
        ++nitem;
        for (int64_t tile = it.t_beg; tile < it.t_end; ++tile, ++kt) {
            const int kb = (int)(kt & 1);
            const uint32_t use = kt >> 1;
            if (!gather_all(use == 0 || mbar_wait(S.bar(B_KEMPTY + kb), (use - 1) & 1, a.wait_ns))) return false;
            // ---- resolve the 64 key slots: window row, compressed row | 2^62, or -1 (empty)
            const int64_t j0 = tile * kKT;
            if (gtid < kKT) {
                const int64_t j = j0 + gtid;
                int64_t code = -1;
                float sc = 0.f;
                if (j < it.n_keys && j < it.n_win) {
                    code = (int64_t)it.b * a.W + j;
                    sc = __ldg(a.win.scale + code);
                } else if (j < it.n_keys) {
                    const int64_t s = a.idx ? (int64_t)a.idx[(int64_t)it.b * a.k + (j - it.n_win)] : (j - it.n_win);
                    if (s >= 0) { // a selected entry that is missing or not yet visible is skipped and reported
                        const int64_t r = paged_row(a.pages, a.max_pages, a.page_rows, it.b, s,
                                                    a.pages ? 0 : a.comp_off[it.b]);
                        if (s < n_vis && r >= 0 && r < a.comp.n) {
                            code = r | (1ll << 62);
                            sc = __ldg(a.comp.scale + r);
                        } else {
                            flag_error(a.err, CSA_DEVERR_INDEX);
                        }
                    }
                }
                S.rows()[gtid] = code;
                S.scale()[gtid] = sc;
                S.valid(kb)[gtid] = code >= 0 ? 1 : 0;
            }
            gather_sync();
            // ---- 64 rows x 36 sixteen-byte units, 18 per thread, all loads in flight together
            constexpr int kU = 18; // covers 64 rows x 36 units (RoPE dims <= 64)
            uint4 raw[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int e = gtid + u * kGatherThreads;
                raw[u] = make_uint4(0, 0, 0, 0);
                if (e < kKT * units) {
                    const int jj = e / units, q = e - jj * units;
                    const int64_t code = S.rows()[jj];
                    if (code >= 0) {
                        const bool comp = (code >> 62) != 0;
                        const int64_t rw = code & ((1ll << 62) - 1);
                        if (q < fp8_units) {
                            const uint8_t *fp8 = comp ? a.comp.fp8 : a.win.fp8;
                            raw[u] = __ldg(reinterpret_cast<const uint4 *>(fp8 + rw * cn + 16 * q));
                        } else {
                            const uint16_t *rope = comp ? a.comp.rope : a.win.rope;
                            raw[u] = __ldg(reinterpret_cast<const uint4 *>(rope + rw * a.comp.rope_dims + 8 * (q - fp8_units)));
                        }
                    }
                }
            }
            const uint32_t kbase = S.k(kb);
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int e = gtid + u * kGatherThreads;
                if (e < kKT * units) {
                    const int jj = e / units, q = e - jj * units;
                    if (q < fp8_units) { // channels 16q .. 16q+15: two 8-channel chunks
                        const float sc = S.scale()[jj];
                        const int ch = 16 * q;
                        const uint4 lo = fp8x8_to_bf16(raw[u].x, raw[u].y, sc);
                        const uint4 hi = fp8x8_to_bf16(raw[u].z, raw[u].w, sc);
                        sts4(kbase + (uint32_t)(ch >> 6) * SUB_K + sw128_off(jj, ch & 63), lo);
                        sts4(kbase + (uint32_t)((ch + 8) >> 6) * SUB_K + sw128_off(jj, (ch + 8) & 63), hi);
                    } else {
                        const int ch = cn + 8 * (q - fp8_units);
                        sts4(kbase + (uint32_t)(ch >> 6) * SUB_K + sw128_off(jj, ch & 63), raw[u]);
                    }
                }
            }
            fence_proxy_async_smem();
            gather_sync(); // rows / scale are rewritten by the next tile's resolve
            if (lane == 0) mbar_arrive(S.bar(B_KFULL + kb));
            (void)warp;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// MMA
// ---------------------------------------------------------------------------------------------

// S = Q K^T for tile k (key buffer k & 1) into TMEM S tile k & 1, once the keys are in and the
// softmax warps have read that S tile's previous use.
__device__ __forceinline__ bool issue_s(const Smem &S, uint32_t tmem, uint32_t k, uint64_t lim)
{
    const int kb = (int)(k & 1);
    if (!mbar_wait(S.bar(B_KFULL + kb), (k >> 1) & 1, lim)) return false;
    if ((k >> 1) >= 1 && !mbar_wait(S.bar(B_SFREE + kb), ((k >> 1) - 1) & 1, lim)) return false;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kColS + 64u * (uint32_t)kb, sdesc_sw128(S.q(s) + 32u * kk, 16, 1024),
                     sdesc_sw128(S.k(kb) + (uint32_t)s * SUB_K + 32u * kk, 16, 1024), IDESC_S, (s | kk) != 0);
    mma_commit(S.bar(B_SFULL + kb));
    return true;
}

__device__ __forceinline__ bool mma_role(const DecodeArgs &a, const Smem &S, uint32_t tmem, const int *s_nwin,
                                         const int *s_nkeys)
{
    const int64_t n_items = (int64_t)a.B * a.n_chunks;
    uint32_t kt = 0, nitem = 0;
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        const ItemTiles it = item_tiles(a, s_nwin, s_nkeys, item);
        if (it.t_beg >= it.t_end) continue;
        if (!mbar_wait(S.bar(B_QFULL), nitem & 1, a.wait_ns)) return false;
        ++nitem;
        const int n = (int)(it.t_end - it.t_beg);
        if (!issue_s(S, tmem, kt, a.wait_ns)) return false;
        for (int i = 0; i < n; ++i, ++kt) {
            if (i + 1 < n) {
                if (!issue_s(S, tmem, kt + 1, a.wait_ns)) return false;
            } else {
                mma_commit(S.bar(B_QEMPTY));
            }
            const int kb = (int)(kt & 1);
            if (!mbar_wait(S.bar(B_PFULL + kb), (kt >> 1) & 1, a.wait_ns)) return false;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(h ? tmem : tmem + TMEM_O, sdesc_sw128(S.pb(kb) + 32u * kk, 16, 1024),
                             sdesc_sw128(S.k(kb) + (uint32_t)h * 4u * SUB_K + 2048u * kk, SUB_K, 1024), IDESC_PV,
                             (i > 0 || kk > 0) ? 1u : 0u);
            mma_commit(S.bar(B_KEMPTY + kb));
            mma_commit(S.bar(B_PVDONE));
        }
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// softmax warps
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ bool softmax_role(const DecodeArgs &a, const Smem &S, uint32_t tmem, const int *s_nwin,
                                             const int *s_nkeys, int warp, int lane)
{
    const bool upper = lane < 16;
    const int row = 16 * warp + (lane & 15); // head
    const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);
    const float sl2 = a.scale * kLog2e;
    const int64_t n_items = (int64_t)a.B * a.n_chunks;
    uint32_t kt = 0;
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
        const ItemTiles it = item_tiles(a, s_nwin, s_nkeys, item);
        const int chunk = (int)(item % a.n_chunks);
        float *part = a.part + ((int64_t)it.b * a.n_chunks + chunk) * kH * (kC + 2);
        if (it.t_beg >= it.t_end) { // empty chunk: a neutral partial
            if (upper) {
                part[(int64_t)row * (kC + 2)] = -INFINITY;
                part[(int64_t)row * (kC + 2) + 1] = 0.f;
            }
            continue;
        }
        float m_run = -INFINITY, l_run = 0.f;
        const int n = (int)(it.t_end - it.t_beg);
        for (int i = 0; i < n; ++i, ++kt) {
            const int kb = (int)(kt & 1);
            const uint32_t use = kt >> 1;
            // the gather's valid flags of this tile, then S
            if (!warp_wait(S.bar(B_KFULL + kb), use & 1, a.wait_ns)) return false;
            if (!warp_wait(S.bar(B_SFULL + kb), use & 1, a.wait_ns)) return false;
            tc_fence_after();
            uint32_t r0[32], r1[32];
            tmem_ld32(tw + kColS + 64u * (uint32_t)kb, r0);
            tmem_ld32(tw + kColS + 64u * (uint32_t)kb + 32u, r1);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S.bar(B_SFREE + kb));
            const int *valid = S.valid(kb);
            const int koff = upper ? 0 : 32; // lane l: keys 0-31, lane l+16: keys 32-63
            float sv[32];
            float mt = -INFINITY;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const uint32_t x = __shfl_xor_sync(0xffffffffu, r1[e], 16);
                float s = __uint_as_float(upper ? r0[e] : x);
                s = valid[koff + e] ? s * sl2 : -INFINITY;
                sv[e] = s;
                mt = fmaxf(mt, s);
            }
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
            const float m_new = fmaxf(m_run, mt);
            float resc = 1.f, m_use = m_run;
            if (m_new != -INFINITY && (m_run == -INFINITY || m_new > m_run + 8.f)) {
                resc = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
                m_use = m_new;
            }
            float ls = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float pv = (m_use == -INFINITY) ? 0.f : ex2(sv[e] - m_use);
                sv[e] = pv;
                ls += pv;
            }
            ls += __shfl_xor_sync(0xffffffffu, ls, 16);
            l_run = l_run * resc + ls;
            m_run = m_use;
            // P V of the previous tile is complete: O settled, P buffer kb (tile kt - 2) free
            if (kt >= 1) {
                if (!warp_wait(S.bar(B_PVDONE), (kt - 1) & 1, a.wait_ns)) return false;
                tc_fence_after();
            }
            if (i > 0 && __any_sync(0xffffffffu, resc != 1.f)) {
                for (int c = 0; c < 8; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tw + 32u * c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * resc);
                    tmem_st32(tw + 32u * c, r);
                }
                tmem_st_wait();
            }
#pragma unroll
            for (int g = 0; g < 4; ++g)
                sts4(S.pb(kb) + sw128_off(row, koff + 8 * g),
                     make_uint4(pk_bf16(sv[8 * g], sv[8 * g + 1]), pk_bf16(sv[8 * g + 2], sv[8 * g + 3]),
                                pk_bf16(sv[8 * g + 4], sv[8 * g + 5]), pk_bf16(sv[8 * g + 6], sv[8 * g + 7])));
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S.bar(B_PFULL + kb));
        }
        // ---- the item's last P V, then (max, sum, unnormalised O) -> workspace
        if (!warp_wait(S.bar(B_PVDONE), (kt - 1) & 1, a.wait_ns)) return false;
        tc_fence_after();
        if (upper) {
            part[(int64_t)row * (kC + 2)] = (m_run == -INFINITY) ? -INFINITY : m_run * kLn2; // natural-log max
            part[(int64_t)row * (kC + 2) + 1] = l_run;
        }
        float *orow = part + (int64_t)row * (kC + 2) + 2 + (upper ? 256 : 0);
        for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            tmem_ld32(tw + 32u * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < 16; ++g)
                *reinterpret_cast<float2 *>(orow + 32 * c + 2 * g) =
                    make_float2(__uint_as_float(r[2 * g]), __uint_as_float(r[2 * g + 1]));
        }
        tc_fence_before();
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) decode_attn_tc_kernel(DecodeArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const Smem S{base, smem_raw + (base - raw)};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            uint32_t count = 1;
            if ((b >= B_SFREE && b < B_SFREE + 2) || (b >= B_PFULL && b < B_PFULL + 2)) count = kSoftWarps;
            else if ((b >= B_KFULL && b < B_KFULL + 2) || b == B_QFULL) count = kGatherWarps;
            mbar_init(S.bar(b), count);
        }
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(base + OFF_TMEM, 512);
    // window length and key count of every sequence, read once
    int *s_nwin = reinterpret_cast<int *>(S.p + OFF_SEQ), *s_nkeys = s_nwin + kSeqCache;
    for (int b = tid; b < a.B && b < kSeqCache; b += kThreads) {
        const Counts c = seq_counts(a, b);
        s_nwin[b] = c.n_win;
        s_nkeys[b] = (int)c.n_keys;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(S.p + OFF_TMEM);

    bool ok = true;
    if (warp < kSoftWarps) ok = softmax_role(a, S, tmem, s_nwin, s_nkeys, warp, lane);
    else if (warp < kMmaWarp) ok = gather_role(a, S, s_nwin, s_nkeys, tid - 32 * kGatherWarp0);
    else if (lane == 0) ok = mma_role(a, S, tmem, s_nwin, s_nkeys);
    if (!ok) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    if (warp == kMmaWarp && lane == 0) {
        mma_commit(S.bar(B_FINAL));
        if (!mbar_wait(S.bar(B_FINAL), 0)) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

} // namespace

// Work items of the tensor-core path: chunks of tpc 64-key tiles, about four items per SM over
// the batch (estimated from the longest key list), one tile per item when the batch is small.
void decode_tc_plan(int64_t B, int64_t max_keys, int sms, int *chunk, int *n_chunks)
{
    const int64_t tiles = (max_keys + kKT - 1) / kKT;
    int64_t tpc = B * tiles / (4 * (int64_t)sms);
    tpc = tpc < 1 ? 1 : (tpc > 16 ? 16 : tpc);
    *chunk = (int)(kKT * tpc);
    *n_chunks = (int)((tiles + tpc - 1) / tpc);
}

bool decode_attn_tc_eligible(const DecodeArgs &a)
{
    // the gather's 18 loads per thread cover 64 rows of (512 - R) / 16 + R / 8 units for R <= 64
    return a.H == kH && a.c == kC && a.comp.rope_dims == a.win.rope_dims && (kC - a.comp.rope_dims) % 16 == 0 &&
           a.comp.rope_dims % 8 == 0 && a.comp.rope_dims <= 64 && a.n_chunks <= 1024 && a.chunk % kKT == 0;
}

cudaError_t launch_attn_decode_tc(const DecodeArgs &a, cudaStream_t st)
{
    cudaError_t e = cudaFuncSetAttribute(decode_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t items = (int64_t)a.B * a.n_chunks;
    const int64_t grid = items < sms ? items : sms;
    decode_attn_tc_kernel<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(a);
    return cudaGetLastError();
}

} // namespace csa
