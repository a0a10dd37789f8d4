// attn_decode_tc.cu -- hybrid MQA decode attention on tcgen05 for 64 heads x 512 channels over the
// mixed FP8/BF16 caches: one new token per sequence, split-K over 128-key chunks of its key list.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 step 3 (shared-KV multi-query attention, the key vector is also the value vector) and
// Sec. 2.4 Attention.forward listing (window keys and selected / all visible compressed keys,
// concatenated); KV cache with BF16 RoPE dims and FP8 for the rest ("Mind Observatory: Uncovering
// the technical ledger of DeepSeek-V4"); the per-head sink is folded in by the merge kernel.
//
// Work items = (sequence, chunk of `chunk` keys = 1-8 tiles of 128 of its key list); persistent
// CTAs (one per SM) walk the items, so the many empty chunks of short sequences in a mixed batch
// cost no launch.  For each non-empty item a CTA stages q [64 x 512] (bf16) once, then for each
// 128-key tile of the item:
//   1. gathers its key rows -- window rows first, then the top-k (CSA) or visible (HCA)
//      compressed rows -- dequantising the FP8 part (code x row scale) to bf16 next to the BF16
//      RoPE part, in 128-byte-swizzled shared memory;
//   2. one thread issues S = Q K^T (tcgen05 M=64, N=128, K=512) into TMEM;
//   3. 4 warps take the online softmax of their 16 heads (lanes l and l+16 split the keys; the
//      running max moves, and O is rescaled in TMEM, only when a tile raises it by more than 8),
//      writing P (bf16) to shared memory;
//   4. O (+)= P V (two M=64 x N=256 x K=128 MMAs, V = the same tile read MN-major) in TMEM.
// The item's (max, sum, unnormalised O) rows go to the workspace for the split-K merge; O is staged
// through shared memory (the free K and P regions) so that the workspace writes are coalesced.
// Every wait of the tile chain is bounded by a.wait_ns (2 s unless a caller lowers it); a wait that
// runs out records CSA_DEVERR_TIMEOUT and every warp leaves the loop at the next CTA barrier.  The
// wind-down is safe because nothing asynchronous but the MMAs writes into this CTA: q and the key
// tiles are stored by the threads themselves, and the MMA lane's final commit is waited for with
// the full 2 s limit before TMEM is released and the CTA exits.
#include "common.cuh"
#include "tc_common.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kH = 64, kC = 512, kKT = 128;
constexpr int kThreads = 8 * 32 + 32; // 8 warps + 1 MMA / TMEM warp
constexpr int kMmaWarp = 8;
constexpr uint32_t OFF_Q = 0;        // 8 sub-tiles [64 x 128 B]   64 KB
constexpr uint32_t OFF_K = 65536;    // 8 sub-tiles [128 x 128 B]  128 KB
constexpr uint32_t OFF_P = 196608;   // 2 sub-tiles [64 x 128 B]   16 KB
constexpr int kStage = kC + 4;       // item end: O staged over the K and P regions, [64 x kStage] fp32
static_assert(OFF_K + 4u * kH * kStage <= OFF_P + 16384u, "O staging fits the K and P regions");
constexpr uint32_t OFF_VALID = 212992;          // 2 x 128 flags (this tile, the next)
constexpr uint32_t OFF_ROWS = OFF_VALID + 1024;  // 2 x 128 resolved key rows (int64)
constexpr int kSeqCache = 1024;                  // per-sequence key counts kept in shared memory
constexpr uint32_t OFF_SEQ = OFF_ROWS + 2048;    // n_win [kSeqCache], n_keys [kSeqCache] (int32)
constexpr uint32_t OFF_BAR = OFF_SEQ + 8 * kSeqCache;
constexpr uint32_t OFF_TMEM = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = OFF_TMEM + 64 + 1024;
constexpr uint32_t TMEM_O = 16u << 16;
constexpr uint32_t kColS = 256;
constexpr uint32_t IDESC_S = idesc_bf16_f32(64, 128, false, false);
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
__device__ __forceinline__ uint4 fp8x8_to_bf16(uint2 c, float s)
{
    const uint32_t w[2] = {c.x, c.y};
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

__global__ void __launch_bounds__(kThreads, 1) decode_attn_tc_kernel(DecodeArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (base - raw);
    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sP = base + OFF_P;
    const uint32_t bar_s = base + OFF_BAR, bar_o = base + OFF_BAR + 8, bar_f = base + OFF_BAR + 16;
    int *valid = reinterpret_cast<int *>(sp + OFF_VALID);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        mbar_init(bar_f, 1);
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(base + OFF_TMEM, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + OFF_TMEM);
    // window length and key count of every sequence, read once (the items loop checks them often)
    int *s_nwin = reinterpret_cast<int *>(sp + OFF_SEQ), *s_nkeys = s_nwin + kSeqCache;
    auto seq_counts = [&](int b, int &nw, int64_t &nk) {
        nw = a.win_len[b] < 0 ? 0 : (a.win_len[b] > a.W ? a.W : a.win_len[b]);
        int64_t nc;
        if (a.idx) nc = a.k;
        else {
            nc = (a.pos[b] + 1) / a.m;
            if (nc > a.max_nvis) nc = a.max_nvis;
            if (nc < 0) nc = 0;
        }
        nk = nw + nc;
    };
    for (int b = tid; b < a.B && b < kSeqCache; b += kThreads) {
        int nw;
        int64_t nk;
        seq_counts(b, nw, nk);
        s_nwin[b] = nw;
        s_nkeys[b] = (int)nk;
    }
    __syncthreads();
    const int64_t n_items = (int64_t)a.B * a.n_chunks;
    const int tpc = a.chunk / kKT; // 128-key tiles per item
    uint32_t ph = 0;               // parity of bar_s / bar_o for the next tile
    bool ok = true;
    int64_t *rows = reinterpret_cast<int64_t *>(sp + OFF_ROWS);
    const int cn = kC - a.comp.rope_dims; // FP8 channels (448), RoPE channels after them
    const bool upper = lane < 16;
    const int row = 16 * (warp & 3) + (lane & 15); // head of this softmax lane (warps 0-3)
    const float sl2 = a.scale * kLog2e;
    int b = 0, n_win = 0;
    int64_t n_keys = 0;
    // key j of sequence b: window row, or compressed row | 2^62, or -1 = empty; stored in slot sl
    auto resolve = [&](int64_t j, int64_t *rw, int *vd, int sl) -> int64_t {
        int64_t code = -1;
        if (j < n_keys && j < n_win) {
            code = (int64_t)b * a.W + j;
        } else if (j < n_keys) {
            const int64_t s = a.idx ? (int64_t)a.idx[(int64_t)b * a.k + (j - n_win)] : (j - n_win);
            if (s >= 0) { // a selected entry that is missing or not yet visible is skipped and reported
                int64_t nvb = (a.pos[b] + 1) / a.m;
                nvb = nvb > a.max_nvis ? a.max_nvis : nvb;
                const int64_t r = paged_row(a.pages, a.max_pages, a.page_rows, b, s, a.pages ? 0 : a.comp_off[b]);
                if (s < nvb && r >= 0 && r < a.comp.n) code = r | (1ll << 62);
                else flag_error(a.err, CSA_DEVERR_INDEX);
            }
        }
        rw[sl] = code;
        vd[sl] = code >= 0 ? 1 : 0;
        return code;
    };
    for (int64_t item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        b = (int)(item / a.n_chunks); // the sequence and key counts resolve() reads
        const int chunk = (int)(item % a.n_chunks);
        if (b < kSeqCache) {
            n_win = s_nwin[b];
            n_keys = s_nkeys[b];
        } else {
            seq_counts(b, n_win, n_keys);
        }
        const int64_t t_beg = (int64_t)chunk * tpc, n_tiles = (n_keys + kKT - 1) / kKT;
        const int64_t t_end = t_beg + tpc < n_tiles ? t_beg + tpc : n_tiles;
        float *part = a.part + ((int64_t)b * a.n_chunks + chunk) * kH * (kC + 2);
        if (t_beg >= t_end) { // empty chunk: a neutral partial (CTA-uniform)
            for (int h = tid; h < kH; h += kThreads) {
                part[(int64_t)h * (kC + 2)] = -INFINITY;
                part[(int64_t)h * (kC + 2) + 1] = 0.f;
            }
            continue;
        }
        // ---- stage q (all threads): 16 independent 16-byte loads per thread in flight
        for (int e0 = tid; e0 < kH * (kC / 8); e0 += 16 * kThreads) {
            uint4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int e = e0 + u * kThreads;
                if (e < kH * (kC / 8))
                    v[u] = __ldg(reinterpret_cast<const uint4 *>(a.q + ((int64_t)b * kH + (e >> 6)) * kC + 8 * (e & 63)));
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int e = e0 + u * kThreads;
                if (e < kH * (kC / 8)) {
                    const int h = e >> 6, cc = e & 63;
                    sts4(sQ + (uint32_t)(cc >> 3) * 8192u + sw128_off(h, (cc & 7) * 8), v[u]);
                }
            }
        }
        float m_run = -INFINITY, l_run = 0.f; // online softmax of this lane's row (log2 domain)
        for (int64_t tile = t_beg; tile < t_end && ok; ++tile) {
            const bool first = tile == t_beg;
            const int buf = (int)((tile - t_beg) & 1);
            int64_t *rw = rows + kKT * buf;
            int *vd = valid + kKT * buf;
            // ---- the item's first tile resolves its 128 key slots here; later tiles were resolved
            // (and their rows prefetched into L2) while the previous tile was computed
            if (first && tid < kKT) resolve(tile * kKT + tid, rw, vd, tid);
            __syncthreads();
            // ---- gather the key rows, FP8 part dequantised to bf16 (code x row scale), RoPE part as
            // is; 12 independent loads per thread in flight
            constexpr int kU = 12;
            for (int e0 = tid; e0 < kKT * (kC / 8); e0 += kU * kThreads) {
                uint4 raw[kU];
                float sc[kU];
                int kind[kU]; // 0 empty, 1 FP8, 2 RoPE
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int e = e0 + u * kThreads;
                    kind[u] = 0;
                    raw[u] = make_uint4(0, 0, 0, 0);
                    sc[u] = 0.f;
                    if (e < kKT * (kC / 8)) {
                        const int64_t code = rw[e >> 6];
                        if (code >= 0) {
                            const KvRowsDev &kv = (code >> 62) ? a.comp : a.win;
                            const int64_t rw = code & ((1ll << 62) - 1);
                            const int ch = 8 * (e & 63);
                            if (ch < cn) {
                                const uint2 c = __ldg(reinterpret_cast<const uint2 *>(kv.fp8 + rw * cn + ch));
                                raw[u].x = c.x;
                                raw[u].y = c.y;
                                sc[u] = __ldg(kv.scale + rw);
                                kind[u] = 1;
                            } else {
                                raw[u] = __ldg(reinterpret_cast<const uint4 *>(kv.rope + rw * kv.rope_dims + (ch - cn)));
                                kind[u] = 2;
                            }
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int e = e0 + u * kThreads;
                    if (e < kKT * (kC / 8)) {
                        const int jj = e >> 6, cc = e & 63;
                        const uint4 v = kind[u] == 1 ? fp8x8_to_bf16(make_uint2(raw[u].x, raw[u].y), sc[u]) : raw[u];
                        sts4(sK + (uint32_t)(cc >> 3) * 16384u + sw128_off(jj, (cc & 7) * 8), v);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            // warps 4-7 have nothing to do until the next gather: resolve the next tile of the item
            // into the other row buffer and start its rows on their way into L2
            if (warp >= 4 && warp < 8 && tile + 1 < t_end) {
                const int sl = tid - 128;
                const int64_t code = resolve((tile + 1) * kKT + sl, rows + kKT * (buf ^ 1), valid + kKT * (buf ^ 1), sl);
                if (code >= 0) {
                    const KvRowsDev &kv = (code >> 62) ? a.comp : a.win;
                    const int64_t rr = code & ((1ll << 62) - 1);
                    const uint8_t *f8 = kv.fp8 + rr * cn;
                    for (int o = 0; o < cn; o += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(f8 + o));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(kv.rope + rr * kv.rope_dims));
                }
            }

            if (warp == kMmaWarp && lane == 0) { // S = Q K^T
#pragma unroll
                for (int s = 0; s < 8; ++s)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tmem + kColS, sdesc_sw128(sQ + (uint32_t)s * 8192u + 32u * kk, 16, 1024),
                                 sdesc_sw128(sK + (uint32_t)s * 16384u + 32u * kk, 16, 1024), IDESC_S, (s | kk) != 0);
                mma_commit(bar_s);
            }
            if (warp < 4) { // softmax of the tile: lane l keys 0-63, lane l+16 keys 64-127 of head `row`
                const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);
                ok = __all_sync(0xffffffffu, mbar_wait(bar_s, ph, a.wait_ns));
                if (ok) {
                    tc_fence_after();
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    tmem_ld32(tw + kColS, r0);
                    tmem_ld32(tw + kColS + 32, r1);
                    tmem_ld32(tw + kColS + 64, r2);
                    tmem_ld32(tw + kColS + 96, r3);
                    tmem_ld_wait();
                    float sv[64];
                    const int kb = upper ? 0 : 64;
                    float mt = -INFINITY;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const uint32_t x = __shfl_xor_sync(0xffffffffu, r2[e], 16);
                        const uint32_t y = __shfl_xor_sync(0xffffffffu, r3[e], 16);
                        float s0 = __uint_as_float(upper ? r0[e] : x), s1 = __uint_as_float(upper ? r1[e] : y);
                        s0 = vd[kb + e] ? s0 * sl2 : -INFINITY;
                        s1 = vd[kb + 32 + e] ? s1 * sl2 : -INFINITY;
                        sv[e] = s0;
                        sv[32 + e] = s1;
                        mt = fmaxf(mt, fmaxf(s0, s1));
                    }
                    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                    // lazy rescale: the running max moves only when this tile raises it by more than 8
                    const float m_new = fmaxf(m_run, mt);
                    float resc = 1.f, m_use = m_run;
                    if (m_new != -INFINITY && (m_run == -INFINITY || m_new > m_run + 8.f)) {
                        resc = (m_run == -INFINITY) ? 0.f : ex2(m_run - m_new);
                        m_use = m_new;
                    }
                    float ls = 0.f;
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const float pv = (m_use == -INFINITY) ? 0.f : ex2(sv[e] - m_use);
                        sv[e] = pv;
                        ls += pv;
                    }
                    ls += __shfl_xor_sync(0xffffffffu, ls, 16);
                    l_run = l_run * resc + ls;
                    m_run = m_use;
                    // O of the earlier tiles (their P V is complete) moves to the new max
                    if (!first && __any_sync(0xffffffffu, resc != 1.f)) {
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
                    const uint32_t psub = sP + (uint32_t)(kb >> 6) * 8192u;
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        sts4(psub + sw128_off(row, 8 * g),
                             make_uint4(pk_bf16(sv[8 * g], sv[8 * g + 1]), pk_bf16(sv[8 * g + 2], sv[8 * g + 3]),
                                        pk_bf16(sv[8 * g + 4], sv[8 * g + 5]), pk_bf16(sv[8 * g + 6], sv[8 * g + 7])));
                }
                fence_proxy_async_smem();
                tc_fence_before();
            }
            ok = __syncthreads_and(ok);
            if (warp == kMmaWarp && lane == 0 && ok) { // O (+)= P V
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(h ? tmem : tmem + TMEM_O,
                                 sdesc_sw128(sP + (uint32_t)(kk >> 2) * 8192u + 32u * (kk & 3), 16, 1024),
                                 sdesc_sw128(sK + (uint32_t)h * 65536u + 2048u * kk, 16384, 1024), IDESC_PV,
                                 (!first || kk > 0) ? 1u : 0u);
                mma_commit(bar_o);
            }
            // the next tile's gather overwrites the keys (= values) and P: wait for P V everywhere
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_o, ph, a.wait_ns));
            tc_fence_after();
            ok = __syncthreads_and(ok);
            ph ^= 1;
        }
        if (warp < 4 && ok) { // (max, sum) -> workspace; unnormalised O -> shared memory (rows of kStage floats)
            const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);
            if (upper) {
                part[(int64_t)row * (kC + 2)] = (m_run == -INFINITY) ? -INFINITY : m_run * kLn2; // natural-log max
                part[(int64_t)row * (kC + 2) + 1] = l_run;
            }
            // lane l holds channels 256-511 of its head, lane l+16 channels 0-255; the row stride of
            // kStage floats puts the 8 rows of a quarter-warp's 16-byte stores in distinct banks
            const uint32_t srow = sK + 4u * (uint32_t)(row * kStage + (upper ? 256 : 0));
            for (int c = 0; c < 8; ++c) {
                uint32_t r[32];
                tmem_ld32(tw + 32u * c, r);
                tmem_ld_wait();
#pragma unroll
                for (int g = 0; g < 8; ++g)
                    sts4(srow + 128u * c + 16u * g, make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]));
            }
            tc_fence_before();
        }
        __syncthreads();
        if (ok) { // every thread: coalesced 8-byte stores (the accumulators start 8 bytes into a partial row)
            const float *stage = reinterpret_cast<const float *>(sp + OFF_K);
            for (int i = tid; i < kH * (kC / 2); i += kThreads) {
                const int h = i / (kC / 2), j = i % (kC / 2);
                *reinterpret_cast<float2 *>(part + (int64_t)h * (kC + 2) + 2 + 2 * j) =
                    *reinterpret_cast<const float2 *>(stage + h * kStage + 2 * j);
            }
        }
        // the item's TMEM and shared memory are free once every warp is past this point
        tc_fence_before();
        ok = __syncthreads_and(ok);
        tc_fence_after();
    } // items
    if (!ok && tid == 0) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    if (warp == kMmaWarp && lane == 0) {
        mma_commit(bar_f);
        if (!mbar_wait(bar_f, 0)) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

} // namespace

// Work items of the tensor-core path: chunks of tpc 128-key tiles, about four items per SM over
// the batch (estimated from the longest key list), one tile per item when the batch is small.
void decode_tc_plan(int64_t B, int64_t max_keys, int sms, int *chunk, int *n_chunks)
{
    const int64_t tiles = (max_keys + kKT - 1) / kKT;
    int64_t tpc = B * tiles / (4 * (int64_t)sms);
    tpc = tpc < 1 ? 1 : (tpc > 8 ? 8 : tpc);
    *chunk = (int)(kKT * tpc);
    *n_chunks = (int)((tiles + tpc - 1) / tpc);
}

bool decode_attn_tc_eligible(const DecodeArgs &a)
{
    return a.H == kH && a.c == kC && a.comp.rope_dims == a.win.rope_dims && (kC - a.comp.rope_dims) % 8 == 0 &&
           a.comp.rope_dims % 8 == 0 && a.n_chunks <= 1024;
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
