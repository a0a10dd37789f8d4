// indexer_decode.cu -- lightning-indexer scan + top-k for decode: few queries (one new token per
// sequence), very long key lists (262,144 FP4 keys per sequence at 1M context).
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 Eq. 16 and the Indexer listing (I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . K[s,:]) over
// s < N_vis(t), then the k best entries); the indexer's QK path runs in FP4 E2M1 with 32-element
// block scales (itsolotime.com Q&A essay on DeepSeek-V4, Question 4; "technical ledger" page).
//
// The FP4 rows are exactly the MX block-scaled format of the 5th-generation tensor cores (E2M1
// packed two per byte, one E8M0 scale per 32 elements), so the scan feeds them to tcgen05
// kind::mxf4 MMAs as they are stored: no conversion.
//
// Kernel 1 (grid = key chunks x queries, at most one CTA per SM): each CTA streams its chunk of
// up to 16,384 keys in 128-key tiles through an 8-stage ring:
//   * producer warp: one lane issues the TMA load of the tile's codes (128 rows x 64 bytes,
//     64-byte swizzle, the MMA's K-major layout); the 32 lanes copy the tile's scale words
//     (4 bytes per key) with cp.async into the 32-row x 16-byte block the scale-factor copy
//     reads (row l holds the words of keys l, l+32, l+64, l+96);
//   * MMA lane: copies the tile's scale words into TMEM (tcgen05.cp 32x128b.warpx4), then two
//     M=128 (keys) x N=64 (heads) x K=64 block-scaled MMAs into one of four TMEM accumulators;
//   * 8 epilogue warps in two groups taking alternate tiles (one key per lane, a warp per TMEM
//     lane quadrant): score = w . ReLU(row of 64 head dot products), then a
//     streaming filter: a key enters the chunk's candidate buffer only if it beats the current
//     k-th best; every 4 tiles, if the buffer is nearly full, an exact radix selection cuts it
//     back to k and raises the bar.  At the end the chunk's exact top-min(k, n) leave as 64-bit candidates
//     (score key << 32 | ~entry, so equal scores order the lower entry first).
// Kernel 2 (one CTA per query): the exact top-k of the union of its chunks' candidates (the
//   global top-k is contained in it), sorted by score descending then entry ascending.
// Every wait is bounded (%globaltimer); a timeout sets CSA_DEVERR_TIMEOUT and the CTA winds down.
#include "common.cuh"
#include "select.cuh"
#include "tc_common.cuh"
#include "tma_host.cuh"

#include <string.h>

namespace csa {

namespace {

using namespace tc;

constexpr int kHI = 64, kDI = 128, kKT = 128, kStages = 8;
constexpr int kChunk = 16384;                 // most keys per CTA
constexpr int kCap = 4096;                    // candidate buffer (> k + kCheck tiles for k <= 2048)
constexpr int kCheck = 4;                     // tiles between checks of the buffer's fill
constexpr int kProdWarp = 0, kEpiWarp0 = 1, kEpiWarps = 8, kMmaWarp = kEpiWarp0 + kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kEpiBar = 1;                    // named barrier of the 8 epilogue warps
constexpr uint32_t kTileCodes = kKT * kDI / 2; // 8192 B

constexpr uint32_t OFF_ST = 0;                              // 8 x 8 KB codes (64-byte swizzle)
constexpr uint32_t OFF_Q = OFF_ST + kStages * kTileCodes;    // query codes [64 x 64 B]
constexpr uint32_t OFF_SCL = OFF_Q + 4096;                   // 8 x 128 scale words, then the query's
constexpr uint32_t OFF_W = OFF_SCL + (kStages + 1) * 512;    // w [64] fp32
constexpr uint32_t OFF_BUF = OFF_W + 256;                    // 2 x kCap candidates
constexpr uint32_t OFF_SEL = OFF_BUF + 2 * kCap * 8;         // selection scratch (< 2 KB)
constexpr uint32_t OFF_MISC = OFF_SEL + 2048;                // counters
constexpr uint32_t OFF_BAR = OFF_MISC + 256;
constexpr uint32_t OFF_TMEM = OFF_BAR + 512;
constexpr uint32_t SMEM_USED = OFF_TMEM + 16;
constexpr uint32_t SMEM_ALLOC = ((SMEM_USED + 127) / 128) * 128 + 1024;

// TMEM columns: accumulators 64 per buffer at 0, 64, 128, 192; the scale words of stage s at
// 256 + 4s; the query's at kColSfb.  The 32x128b.warpx4 copy puts them in every lane quadrant:
// lane l of column c + j holds the word of row l + 32j.
constexpr int kDBufs = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kColSfa = 64 * kDBufs, kColSfb = kColSfa + 4 * kStages;

enum { B_FULL = 0, B_EMPTY = B_FULL + kStages, B_DFULL = B_EMPTY + kStages, B_DEMPTY = B_DFULL + kDBufs,
       B_QFULL = B_DEMPTY + kDBufs, B_FINAL, NUM_BARS };
static_assert(NUM_BARS * 8 <= 512, "barrier space");
static_assert(sizeof(SelectSmem<uint32_t>) <= 2048, "selection scratch");

enum { M_COUNT = 0, M_ABORT = 1, M_OUT = 2 };

struct Maps {
    CUtensorMap q, k;
};

__device__ __forceinline__ int64_t dec_nvis(const IndexerArgs &a, int64_t r)
{
    const int64_t t = a.q_pos ? a.q_pos[r] : r;
    int64_t nv = (t + 1) / a.m;
    if (nv > a.max_nvis) nv = a.max_nvis;
    const int64_t base = a.key_off ? a.key_off[r] : 0;
    if (base < 0) return 0;
    if (nv > a.n_keys - base) nv = a.n_keys - base;
    return nv < 0 ? 0 : nv;
}

__device__ __forceinline__ bool wwait(uint32_t bar, uint32_t parity)
{
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kEpiBar), "n"(kEpiThreads) : "memory"); }

// ------------------------------------------------------------------------------------------
// kernel 1: FP4 key scan (tcgen05 kind::mxf4) + streaming chunk top-k
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) decode_scan_kernel(IndexerArgs a, const __grid_constant__ Maps maps,
                                                                  int n_slots, int chunk, unsigned long long *cand,
                                                                  int *cand_count)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (base - raw);
    auto bar = [&](int b) { return base + OFF_BAR + 8u * (uint32_t)b; };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t r = blockIdx.y;
    const int slot = blockIdx.x;
    const int64_t nv = dec_nvis(a, r);
    const int64_t c0 = (int64_t)slot * chunk;
    const int n = (int)(nv - c0 < chunk ? (nv - c0 > 0 ? nv - c0 : 0) : chunk);
    unsigned long long *out = cand + ((int64_t)r * n_slots + slot) * a.k;
    int *out_count = cand_count + r * n_slots + slot;
    if (n == 0) { // nothing visible in this chunk (CTA-uniform)
        if (tid == 0) *out_count = 0;
        return;
    }
    const int64_t key0 = (a.key_off ? a.key_off[r] : 0) + c0; // first key row of the chunk
    const int ntiles = (n + kKT - 1) / kKT;
    int *misc = reinterpret_cast<int *>(sp + OFF_MISC);

    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            uint32_t cnt = 1;
            if (b >= B_FULL && b < B_FULL + kStages) cnt = 1 + 32; // expect_tx arrive + 32 cp.async arrivals
            if (b >= B_DEMPTY && b < B_DEMPTY + kDBufs) cnt = 4;
            mbar_init(bar(b), cnt);
        }
        mbar_init_fence();
        misc[M_COUNT] = 0;
        misc[M_ABORT] = 0;
        misc[M_OUT] = 0;
    }
    if (tid < kHI) reinterpret_cast<float *>(sp + OFF_W)[tid] = a.w[r * kHI + tid];
    if (tid < 128) { // the query's scale words in the copy layout (rows 64-127 zero)
        const int l = tid & 31, j = tid >> 5, h = l + 32 * j;
        reinterpret_cast<uint32_t *>(sp + OFF_SCL + kStages * 512)[4 * l + j] =
            h < kHI ? reinterpret_cast<const uint32_t *>(a.q4.scales)[r * kHI + h] : 0u;
    }
    fence_proxy_async_smem();
    if (warp == kMmaWarp) tmem_alloc(base + OFF_TMEM, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + OFF_TMEM);

    bool ok = true;
    if (warp == kProdWarp) {
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(B_QFULL), 4096u);
            tma_load_2d(base + OFF_Q, &maps.q, 0, (int32_t)(r * kHI), bar(B_QFULL));
        }
        const uint32_t *scales = reinterpret_cast<const uint32_t *>(a.k4.scales); // one word per key row
        for (int i = 0; i < ntiles && ok; ++i) {
            const uint32_t st = i % kStages;
            if (i >= kStages && !wwait(bar(B_EMPTY + st), ((i / kStages) - 1) & 1)) { ok = false; break; }
            const int64_t row0 = key0 + (int64_t)i * kKT;
            const int valid = n - i * kKT < kKT ? n - i * kKT : kKT; // keys of the chunk in this tile
            for (int j = lane; j < valid; j += 32)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(base + OFF_SCL + st * 512u +
                                                                          16u * (j & 31) + 4u * (j >> 5)),
                             "l"(scales + row0 + j)
                             : "memory");
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(B_FULL + st)) : "memory");
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(B_FULL + st), kTileCodes);
                tma_load_2d(base + OFF_ST + st * kTileCodes, &maps.k, 0, (int32_t)row0, bar(B_FULL + st));
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kMmaWarp) {
        const int quad = warp & 3, etid = tid - 32 * kEpiWarp0, grp = (warp - kEpiWarp0) >> 2;
        float w[kHI];
#pragma unroll
        for (int h = 0; h < kHI; ++h) w[h] = reinterpret_cast<const float *>(sp + OFF_W)[h];
        unsigned long long *buf = reinterpret_cast<unsigned long long *>(sp + OFF_BUF);
        unsigned long long *alt = buf + kCap;
        SelectSmem<uint32_t> *sel = reinterpret_cast<SelectSmem<uint32_t> *>(sp + OFF_SEL);
        unsigned long long theta = 0; // a key enters the buffer only above this
        const int npairs = (ntiles + 1) / 2;
        for (int p = 0; p < npairs; ++p) { // group g takes tile 2p + g; both groups pass the same barriers
            const int i = 2 * p + grp;
            const uint32_t db = i % kDBufs;
            const bool got = i >= ntiles || wwait(bar(B_DFULL + db), (i / kDBufs) & 1);
            if (i >= ntiles) {
            } else if (got) {
                tc_fence_after();
                uint32_t r0[32], r1[32];
                const uint32_t ta = tmem + db * 64u + ((uint32_t)(32 * quad) << 16);
                tmem_ld32(ta, r0);
                tmem_ld32(ta + 32, r1);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_DEMPTY + db));
                float acc[4] = {0.f, 0.f, 0.f, 0.f}; // four independent chains
#pragma unroll
                for (int h = 0; h < 32; ++h) acc[h & 3] = fmaf(w[h], fmaxf(__uint_as_float(r0[h]), 0.f), acc[h & 3]);
#pragma unroll
                for (int h = 0; h < 32; ++h)
                    acc[h & 3] = fmaf(w[32 + h], fmaxf(__uint_as_float(r1[h]), 0.f), acc[h & 3]);
                const float s = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                const int kc = i * kKT + 32 * quad + lane;
                const unsigned long long cv =
                    ((unsigned long long)float_key(s) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)(c0 + kc));
                const bool take = kc < n && cv > theta;
                const unsigned bal = __ballot_sync(0xffffffffu, take);
                if (bal) {
                    int pos = 0;
                    if (lane == 0) pos = atomicAdd(&misc[M_COUNT], __popc(bal));
                    pos = __shfl_sync(0xffffffffu, pos, 0);
                    if (take) buf[pos + __popc(bal & ((1u << lane) - 1u))] = cv;
                }
            } else if (lane == 0) {
                misc[M_ABORT] = 1;
            }
            if ((p + 1) % (kCheck / 2) != 0 && p + 1 != npairs) continue; // the buffer has room for kCheck tiles
            epi_sync();
            const bool abort = misc[M_ABORT] != 0;
            const int cnt = misc[M_COUNT];
            epi_sync(); // every warp has read the count before any appends the next tile's keys
            if (abort) { ok = false; break; }
            if (cnt > kCap - kCheck * kKT && cnt > a.k) { // cut the buffer back to the k best, raise the bar
                theta = block_kth64<kEpiThreads, kEpiBar>(cnt, a.k, [&](int j) { return buf[j]; }, sel, etid);
                if (etid == 0) misc[M_OUT] = 0;
                epi_sync();
                for (int j = etid; j < cnt; j += kEpiThreads) {
                    const unsigned long long v = buf[j];
                    if (v >= theta) alt[atomicAdd(&misc[M_OUT], 1)] = v;
                }
                epi_sync();
                for (int j = etid; j < a.k; j += kEpiThreads) buf[j] = alt[j];
                if (etid == 0) misc[M_COUNT] = a.k;
                epi_sync();
            }
        }
        if (ok) { // the chunk's exact top-min(k, n)
            const int cnt = misc[M_COUNT];
            if (cnt > a.k) {
                const unsigned long long thr =
                    block_kth64<kEpiThreads, kEpiBar>(cnt, a.k, [&](int j) { return buf[j]; }, sel, etid);
                if (etid == 0) misc[M_OUT] = 0;
                epi_sync();
                for (int j = etid; j < cnt; j += kEpiThreads) {
                    const unsigned long long v = buf[j];
                    if (v >= thr) out[atomicAdd(&misc[M_OUT], 1)] = v;
                }
                if (etid == 0) *out_count = a.k;
            } else {
                for (int j = etid; j < cnt; j += kEpiThreads) out[j] = buf[j];
                if (etid == 0) *out_count = cnt;
            }
        } else if (etid == 0) {
            *out_count = 0;
        }
    } else if (warp == kMmaWarp && lane == 0) {
        ok = mbar_wait(bar(B_QFULL), 0);
        if (ok) {
            tc_fence_after();
            tmem_cp_32x128b_x4(tmem + kColSfb, sdesc_plain(base + OFF_SCL + kStages * 512u, 128, 128));
        }
        for (int i = 0; i < ntiles && ok; ++i) {
            const uint32_t st = i % kStages, db = i % kDBufs;
            if (!mbar_wait(bar(B_FULL + st), (i / kStages) & 1)) { ok = false; break; }
            fence_proxy_async_smem(); // the cp.async scale words, read next by the tensor pipe
            if (i >= kDBufs && !mbar_wait(bar(B_DEMPTY + db), ((i / kDBufs) - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_tile = base + OFF_ST + st * kTileCodes;
            tmem_cp_32x128b_x4(tmem + kColSfa + 4u * st, sdesc_plain(base + OFF_SCL + st * 512u, 128, 128));
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) { // K = 0..63 (scale bytes 0-1), 64..127 (bytes 2-3)
                mma_mxf4(tmem + db * 64u, sdesc_sw64(a_tile + 32u * kh, 512), sdesc_sw64(base + OFF_Q + 32u * kh, 512),
                         idesc_mxf4(128, 64, 2u * kh, 2u * kh), tmem + kColSfa + 4u * st, tmem + kColSfb, kh);
            }
            mma_commit(bar(B_EMPTY + st));
            mma_commit(bar(B_DFULL + db));
        }
    }
    if (!ok) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    if (warp == kMmaWarp && lane == 0) {
        mma_commit(bar(B_FINAL));
        if (!mbar_wait(bar(B_FINAL), 0)) flag_error(a.err, CSA_DEVERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------------------------------
// kernel 2: exact top-k over the chunk candidates of one query
// ------------------------------------------------------------------------------------------
constexpr int kMergeThreads = 1024;

constexpr int kPivCap = 4096; // candidates above the sampled pivot that the merge selects from

// pivot: the union is first filtered by a pivot taken from every 16th candidate (the 1.5 k / 16-th
// best sample, which lies below the k-th best of the union with high probability), so the exact
// selection runs on about 1.5 k candidates; when the filter keeps fewer than k or more than
// kPivCap, the selection runs on the whole union.
__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(IndexerArgs a, int n_slots,
                                                                     const unsigned long long *cand,
                                                                     const int *cand_count, int pivot)
{
    extern __shared__ unsigned long long mv[];
    __shared__ SelectSmem<uint32_t> msel;
    __shared__ int s_cnt, s_off[64];
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const int k = a.k;
    if (tid == 0) {
        int o = 0;
        for (int s = 0; s < n_slots; ++s) {
            s_off[s] = o;
            o += cand_count[r * n_slots + s];
        }
        s_cnt = o;
    }
    __syncthreads();
    const int total = s_cnt;
    { // gather the chunk lists, 8 independent 8-byte loads per thread in flight
        const unsigned long long *src = cand + r * n_slots * k;
        const int span = n_slots * k;
        for (int e0 = tid; e0 < span; e0 += 8 * kMergeThreads) {
            unsigned long long v[8];
            int dst[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * kMergeThreads;
                dst[u] = -1;
                if (e < span) {
                    const int s = e / k, i = e - s * k;
                    if (i < cand_count[r * n_slots + s]) {
                        v[u] = src[e];
                        dst[u] = s_off[s] + i;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (dst[u] >= 0) mv[dst[u]] = v[u];
        }
    }
    __syncthreads();
    const int ke = total < k ? total : k;
    unsigned long long *buf = mv + total;                   // candidates above the pivot
    unsigned long long *sel = buf + (pivot ? kPivCap : 0);  // ke winners
    if (total > k) {
        bool done = false;
        const int ns = total >> 4, ks = (3 * k) >> 5;
        if (pivot && ks >= 1 && ns >= 2 * ks) {
            const unsigned long long piv =
                block_kth64<kMergeThreads>(ns, ks, [&](int i) { return mv[16 * i]; }, &msel);
            if (tid == 0) s_cnt = 0;
            __syncthreads();
            for (int i = tid; i < total; i += kMergeThreads) {
                const unsigned long long v = mv[i];
                if (v >= piv) {
                    const int p = atomicAdd(&s_cnt, 1);
                    if (p < kPivCap) buf[p] = v;
                }
            }
            __syncthreads();
            const int c = s_cnt;
            if (c >= k && c <= kPivCap) { // the k best of the union are all above the pivot
                const unsigned long long thr =
                    block_kth64<kMergeThreads>(c, k, [&](int i) { return buf[i]; }, &msel);
                __syncthreads();
                if (tid == 0) s_cnt = 0;
                __syncthreads();
                for (int i = tid; i < c; i += kMergeThreads) {
                    const unsigned long long v = buf[i];
                    if (v >= thr) sel[atomicAdd(&s_cnt, 1)] = v;
                }
                done = true;
            }
            __syncthreads();
        }
        if (!done) {
            const unsigned long long thr = block_kth64<kMergeThreads>(total, k, [&](int i) { return mv[i]; }, &msel);
            if (tid == 0) s_cnt = 0;
            __syncthreads();
            for (int i = tid; i < total; i += kMergeThreads) {
                const unsigned long long v = mv[i];
                if (v >= thr) {
                    const int p = atomicAdd(&s_cnt, 1);
                    if (p < ke) sel[p] = v;
                }
            }
        }
    } else {
        for (int i = tid; i < total; i += kMergeThreads) sel[i] = mv[i];
    }
    __syncthreads();
    int n2 = 1;
    while (n2 < ke) n2 <<= 1;
    for (int i = ke + tid; i < n2; i += kMergeThreads) sel[i] = 0ull;
    __syncthreads();
    for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < n2; i += kMergeThreads) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool desc = (i & size) == 0;
                    const unsigned long long x = sel[i], y = sel[j];
                    if (desc ? (x < y) : (x > y)) { sel[i] = y; sel[j] = x; }
                }
            }
            __syncthreads();
        }
    }
    for (int j = tid; j < k; j += kMergeThreads) {
        int32_t id = -1;
        float sc = -INFINITY;
        if (j < ke) {
            const unsigned long long v = sel[j];
            id = (int32_t)(0xffffffffu - (uint32_t)(v & 0xffffffffu));
            sc = key_float((uint32_t)(v >> 32));
        }
        a.idx_out[r * k + j] = id;
        if (a.score_out) a.score_out[r * k + j] = sc;
    }
}

} // namespace

// Chunking of the key lists: at most one CTA per SM of the B200's 148 (the CTAs of one launch fill
// a single wave: a 149th CTA would double the launch time), at most kChunk keys each.
static void decode_chunks(int64_t Nq, int64_t max_nvis, int *slots, int *chunk)
{
    int64_t want = 148 / (Nq > 0 ? Nq : 1);
    if (want < 1) want = 1;
    int64_t ch = (max_nvis + want - 1) / want;
    ch = (ch + kKT - 1) / kKT * kKT;
    if (ch > kChunk) ch = kChunk;
    if (ch < kKT) ch = kKT;
    *chunk = (int)ch;
    *slots = (int)((max_nvis + ch - 1) / ch);
    if (*slots < 1) *slots = 1;
}

// Workspace bytes of the decode path (candidates + counts).
size_t decode_indexer_workspace(int64_t Nq, int64_t max_nvis, int k)
{
    int slots, chunk;
    decode_chunks(Nq, max_nvis, &slots, &chunk);
    return (size_t)Nq * (size_t)slots * ((size_t)k * 8 + 4) + 256;
}

bool decode_indexer_eligible(const IndexerArgs &a)
{
    if (a.fmt != CSA_FP4 || a.H != kHI || a.d != kDI || a.Nq <= 0 || a.Nq > 65535 || a.max_nvis <= 0) return false;
    if (a.k > 2048 || a.k4.n >= (1ll << 31) || a.Nq * kHI >= (1ll << 31)) return false;
    int slots, chunk;
    decode_chunks(a.Nq, a.max_nvis, &slots, &chunk);
    if (slots > 64) return false;
    // merge kernel: candidates (slots * k) plus the padded winner array must fit in shared memory
    int n2 = 1;
    while (n2 < a.k) n2 <<= 1;
    return (size_t)(slots * a.k + n2) * 8 <= 200 * 1024;
}

cudaError_t launch_indexer_decode(const IndexerArgs &a, void *ws, cudaStream_t st)
{
    int slots, chunk;
    decode_chunks(a.Nq, a.max_nvis, &slots, &chunk);
    uintptr_t p = (reinterpret_cast<uintptr_t>(ws) + 255) / 256 * 256;
    unsigned long long *cand = reinterpret_cast<unsigned long long *>(p);
    int *cnt = reinterpret_cast<int *>(cand + (size_t)a.Nq * slots * a.k);
    Maps maps;
    memset(&maps, 0, sizeof(maps));
    const uint64_t key_rows = a.k4.n > 0 ? (uint64_t)a.k4.n : 1; // an empty key array is never read
    if (!tma::encode_u8_rows_sw64(&maps.q, a.q4.codes, (uint64_t)a.Nq * kHI, kDI / 2, kHI) ||
        !tma::encode_u8_rows_sw64(&maps.k, a.k4.codes, key_rows, kDI / 2, kKT))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(decode_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    decode_scan_kernel<<<dim3((unsigned)slots, (unsigned)a.Nq), kThreads, SMEM_ALLOC, st>>>(a, maps, slots, chunk, cand,
                                                                                           cnt);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int n2 = 1;
    while (n2 < a.k) n2 <<= 1;
    size_t msm = (size_t)(slots * a.k + n2) * 8;
    const int pivot = msm + (size_t)kPivCap * 8 <= 220 * 1024 ? 1 : 0;
    if (pivot) msm += (size_t)kPivCap * 8;
    e = cudaFuncSetAttribute(decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msm);
    if (e != cudaSuccess) return e;
    decode_merge_kernel<<<(unsigned)a.Nq, kMergeThreads, msm, st>>>(a, slots, cand, cnt, pivot);
    return cudaGetLastError();
}

} // namespace csa
