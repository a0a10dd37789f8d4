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
// Kernel 1 (one CTA per (query, key chunk)): each CTA streams its chunk of
// up to 16,384 keys in 128-key tiles through an 8-stage ring:
//   * producer warp: one lane issues the TMA load of the tile's codes (128 rows x 64 bytes,
//     64-byte swizzle, the MMA's K-major layout); the 32 lanes copy the tile's scale words
//     (4 bytes per key) with cp.async into the 32-row x 16-byte block the scale-factor copy
//     reads (row l holds the words of keys l, l+32, l+64, l+96);
//   * MMA lane: copies the tile's scale words into TMEM (tcgen05.cp 32x128b.warpx4), then two
//     M=128 (keys) x N=64 (heads) x K=64 block-scaled MMAs into one of four TMEM accumulators;
//   * 8 epilogue warps in two groups taking alternate tiles (one key per lane, a warp per TMEM
//     lane quadrant): score = w . ReLU(row of 64 head dot products), written to the score
//     buffer, and kept in the thread's own top-R list (registers, 64-bit keys
//     score key << 32 | ~entry, so equal scores order the lower entry first) when it beats the
//     list's last key.  No barrier inside the tile loop.
//   At the end of the chunk the lists (256 x R keys) are cut to about p = the chunk's share of k
//   (one radix digit, or an exact selection when that digit keeps too many) and published with
//   the chunk's bound theta_c: every key of the chunk that is not published is below theta_c
//   (theta_c = 0 when every key is published).
// Kernel 2 (one CTA per query): theta = the k-th largest published key is at most the query's
//   true k-th largest key (the k-th of a subset), so the exact top-k lies among the keys >= theta.
//   A chunk with theta_c <= theta published all of those; the others ("saturated", rare: a chunk
//   holding far more than its share of the winners) are re-read whole from the score buffer.  The
//   exact top-k of that set is then sorted by score descending, entry ascending.
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
constexpr int kR = 8;                         // keys kept per epilogue thread
constexpr int kMergeSmem = 200 * 1024;        // merge kernel: published lists + winners
constexpr int kShareMax = 512;                // most of k one chunk is expected to hold
constexpr int kProdWarp = 0, kEpiWarp0 = 1, kEpiWarps = 8, kMmaWarp = kEpiWarp0 + kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kEpiBar = 1;                    // named barrier of the 8 epilogue warps
constexpr uint32_t kTileCodes = kKT * kDI / 2; // 8192 B

constexpr uint32_t OFF_ST = 0;                              // 8 x 8 KB codes (64-byte swizzle)
constexpr uint32_t OFF_Q = OFF_ST + kStages * kTileCodes;    // query codes [64 x 64 B]
constexpr uint32_t OFF_SCL = OFF_Q + 4096;                   // 8 x 128 scale words, then the query's
constexpr uint32_t OFF_W = OFF_SCL + (kStages + 1) * 512;    // w [64] fp32
constexpr uint32_t OFF_BUF = OFF_W + 256;                    // the threads' lists, 256 x kR keys
constexpr uint32_t OFF_SEL = OFF_BUF + kEpiThreads * kR * 8; // selection scratch (< 2 KB)
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

enum { M_COUNT = 0, M_ABORT = 1, M_OUT = 2, M_RED = 4 }; // M_RED: 8 x u64 (one per warp)

struct Maps {
    CUtensorMap q, k, kp; // kp: key rows in boxes of one page (paged caches only)
    // Permuted tiles (see the scan kernel): every 4th key row (kq4: 32 rows a box, kq4p: a page's
    // share), the scale words as rows of 4 (sq: 32 rows a box, sqp: a page's share)
    CUtensorMap kq4, kq4p, sq, sqp;
    int perm; // the permuted maps exist (and, when paged, pages hold >= 32 rows)
};

__device__ __forceinline__ int64_t dec_nvis(const IndexerArgs &a, int64_t r)
{
    const int64_t t = a.q_pos ? a.q_pos[r] : r;
    int64_t nv = (t + 1) / a.m;
    if (nv > a.max_nvis) nv = a.max_nvis;
    if (a.pages) { // the page table bounds the entries
        const int64_t cap = (int64_t)a.max_pages * a.page_rows;
        return nv < 0 ? 0 : (nv > cap ? cap : nv);
    }
    const int64_t base = a.key_off ? a.key_off[r] : 0;
    if (base < 0) return 0;
    if (nv > a.n_keys - base) nv = a.n_keys - base;
    return nv < 0 ? 0 : nv;
}

// Query r's chunk size: its nv visible keys spread over all n_slots chunks (multiples of the
// 128-key tile), so every query's chunks hold about the same share of its k winners.
__host__ __device__ __forceinline__ int query_chunk(int64_t nv, int n_slots)
{
    int64_t ch = (nv + n_slots - 1) / n_slots;
    ch = (ch + kKT - 1) / kKT * kKT;
    return (int)(ch < kKT ? kKT : ch);
}

// Keys a chunk of query r publishes: about twice its share of k (at least 64), at most the list
// capacity and at most k.
__host__ __device__ __forceinline__ int query_keep(int64_t nv, int chunk, int k, int lcap)
{
    const int64_t ns = nv > 0 ? (nv + chunk - 1) / chunk : 1;
    const int64_t share = (k + ns - 1) / ns;
    int64_t keep = 2 * share + 32;
    keep = keep < 64 ? 64 : keep;
    keep = keep > k ? k : keep;
    return (int)(keep > lcap ? lcap : keep);
}

__device__ __forceinline__ bool wwait(uint32_t bar, uint32_t parity)
{
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync %0, %1;" ::"n"(kEpiBar), "n"(kEpiThreads) : "memory"); }

// ------------------------------------------------------------------------------------------
// kernel 1: FP4 key scan (tcgen05 kind::mxf4), every score stored, per-thread top-R lists
// ------------------------------------------------------------------------------------------

// Chunk output: list [lcap] 64-bit keys, count, theta_c (every unpublished key of the chunk is
// below theta_c; 0 when all are published).
struct ChunkOut {
    unsigned long long *list;   // [Nq, n_slots, lcap]
    int *count;                 // [Nq, n_slots]
    unsigned long long *theta;  // [Nq, n_slots]
    int n_slots, lcap;
};

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

// Largest of one value per epilogue thread (all 256 call it; returns the same on all).
__device__ __forceinline__ unsigned long long epi_max_u64(unsigned long long v, unsigned long long *red, int etid)
{
    v = warp_max_u64(v);
    if ((etid & 31) == 0) red[etid >> 5] = v;
    epi_sync();
    unsigned long long m = red[0];
#pragma unroll
    for (int w = 1; w < kEpiWarps; ++w) m = red[w] > m ? red[w] : m;
    epi_sync(); // red is read by every thread before it is reused
    return m;
}

__global__ void __launch_bounds__(kThreads, 1) decode_scan_kernel(IndexerArgs a, const __grid_constant__ Maps maps,
                                                                  ChunkOut co)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (base - raw);
    auto bar = [&](int b) { return base + OFF_BAR + 8u * (uint32_t)b; };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t r = (int64_t)blockIdx.x / co.n_slots; // query
    const int slot = (int)((int64_t)blockIdx.x % co.n_slots);
    const int64_t nv = dec_nvis(a, r);
    const int chunk = query_chunk(nv, co.n_slots);
    const int keep = query_keep(nv, chunk, a.k, co.lcap);
    const int64_t c0 = (int64_t)slot * chunk;
    const int n = (int)(nv - c0 < chunk ? (nv - c0 > 0 ? nv - c0 : 0) : chunk);
    const int64_t oslot = r * co.n_slots + slot;
    unsigned long long *out = co.list + oslot * co.lcap;
    if (n == 0) { // nothing visible in this chunk (CTA-uniform)
        if (tid == 0) {
            co.count[oslot] = 0;
            co.theta[oslot] = 0ull;
        }
        return;
    }
    const int64_t key0 = (a.key_off ? a.key_off[r] : 0) + c0; // first key row of the chunk
    const int ntiles = (n + kKT - 1) / kKT;
    // Permuted tiles: MMA row 32j + l holds key 4l + j of the tile, so that the scale words of the
    // keys on TMEM lane l (keys 4l .. 4l+3 in columns j = 0..3 of the block-scale layout) are 16
    // contiguous bytes, and a tile's 128 scale words arrive by TMA as they are stored.  The codes
    // come as four boxes of every 4th row.  Needs the chunk to start at a multiple of 4 rows.
    const bool perm = maps.perm && (a.pages || (key0 & 3) == 0);
    int *misc = reinterpret_cast<int *>(sp + OFF_MISC);
    unsigned long long *red = reinterpret_cast<unsigned long long *>(sp + OFF_MISC + 4 * M_RED);

    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            uint32_t cnt = 1;
            if (b >= B_FULL && b < B_FULL + kStages) cnt = perm ? 1 : 1 + 32; // expect_tx arrive (+ 32 cp.async arrivals)
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
            const int64_t e0 = c0 + (int64_t)i * kKT;                // the tile's first entry
            if (perm) { // codes and scale words by TMA only
                if (lane == 0) {
                    const uint32_t dst = base + OFF_ST + st * kTileCodes, sdst = base + OFF_SCL + st * 512u;
                    mbar_arrive_expect_tx(bar(B_FULL + st), kTileCodes + 512u);
                    if (!a.pages) {
                        const int32_t y0 = (int32_t)(row0 >> 2);
#pragma unroll
                        for (int j = 0; j < 4; ++j) tma_load_3d(dst + 2048u * j, &maps.kq4, 0, j, y0, bar(B_FULL + st));
                        tma_load_2d(sdst, &maps.sq, 0, y0, bar(B_FULL + st));
                    } else { // per page: its rows 4m + j and its scale words; a bad page reads page 0
                        const int pr4 = a.page_rows >> 2;
                        for (int u = 0; u * a.page_rows < kKT; ++u) {
                            const int64_t eu = e0 + (int64_t)u * a.page_rows;
                            int64_t prow = eu < c0 + n ? paged_row(a.pages, a.max_pages, a.page_rows, r, eu, 0) : 0;
                            if (prow < 0 || prow >= a.k4.n) prow = 0;
                            const int32_t y0 = (int32_t)(prow >> 2);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                tma_load_3d(dst + (uint32_t)(32 * j + pr4 * u) * 64u, &maps.kq4p, 0, j, y0, bar(B_FULL + st));
                            tma_load_2d(sdst + (uint32_t)(pr4 * u) * 16u, &maps.sqp, 0, y0, bar(B_FULL + st));
                        }
                    }
                }
                continue;
            }
            for (int j = lane; j < valid; j += 32) {
                const int64_t row = a.pages ? paged_row(a.pages, a.max_pages, a.page_rows, r, e0 + j, 0) : row0 + j;
                if (row >= 0 && row < a.k4.n) // a bad page leaves the word unset; the epilogue drops the key
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(base + OFF_SCL + st * 512u +
                                                                              16u * (j & 31) + 4u * (j >> 5)),
                                 "l"(scales + row)
                                 : "memory");
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(B_FULL + st)) : "memory");
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(B_FULL + st), kTileCodes);
                if (!a.pages) {
                    tma_load_2d(base + OFF_ST + st * kTileCodes, &maps.k, 0, (int32_t)row0, bar(B_FULL + st));
                } else { // one box per page; rows past the chunk or of a bad page read anything in range
                    for (int u = 0; u * a.page_rows < kKT; ++u) {
                        const int64_t eu = e0 + (int64_t)u * a.page_rows;
                        int64_t row = eu < c0 + n ? paged_row(a.pages, a.max_pages, a.page_rows, r, eu, 0) : 0;
                        if (row < 0 || row >= a.k4.n) row = 0;
                        tma_load_2d(base + OFF_ST + st * kTileCodes + (uint32_t)(u * a.page_rows) * 64u, &maps.kp, 0,
                                    (int32_t)row, bar(B_FULL + st));
                    }
                }
            }
        }
        // every cp.async of this warp has landed before the CTA can exit
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp >= kEpiWarp0 && warp < kMmaWarp) {
        const int quad = warp & 3, etid = tid - 32 * kEpiWarp0, grp = (warp - kEpiWarp0) >> 2;
        float w[kHI];
#pragma unroll
        for (int h = 0; h < kHI; ++h) w[h] = reinterpret_cast<const float *>(sp + OFF_W)[h];
        float *srow = a.scores + r * a.ld + c0; // this chunk's scores
        unsigned long long top[kR];             // this thread's best keys, descending (0 = empty)
#pragma unroll
        for (int j = 0; j < kR; ++j) top[j] = 0ull;
        for (int i = grp; i < ntiles; i += 2) { // group g takes tiles g, g + 2, ...
            const uint32_t db = i % kDBufs;
            if (!wwait(bar(B_DFULL + db), (i / kDBufs) & 1)) {
                ok = false;
                if (lane == 0) misc[M_ABORT] = 1;
                break;
            }
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
            const int kc = i * kKT + (perm ? 4 * lane + quad : 32 * quad + lane); // key of TMEM lane 32 quad + lane
            bool live = kc < n;
            if (live && a.pages) { // a key whose page is missing or out of range is dropped and reported
                const int64_t row = paged_row(a.pages, a.max_pages, a.page_rows, r, c0 + kc, 0);
                if (row < 0 || row >= a.k4.n) {
                    flag_error(a.err, CSA_DEVERR_INDEX);
                    srow[kc] = -INFINITY;
                    live = false;
                }
            }
            if (live) {
                srow[kc] = s;
                const unsigned long long cv =
                    ((unsigned long long)float_key(s) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)(c0 + kc));
                if (cv > top[kR - 1]) { // insert, keeping the list sorted
                    top[kR - 1] = cv;
#pragma unroll
                    for (int j = kR - 1; j > 0; --j) {
                        const unsigned long long x = top[j - 1], y = top[j];
                        top[j - 1] = y > x ? y : x;
                        top[j] = y > x ? x : y;
                    }
                }
            }
        }
        epi_sync();
        if (misc[M_ABORT] != 0) ok = false; // uniform over the epilogue warps
        if (ok) {
            // 1. the lists into shared memory, densely; tau = the largest last key of a full list
            unsigned long long *U = reinterpret_cast<unsigned long long *>(sp + OFF_BUF);
            int mine = 0;
#pragma unroll
            for (int j = 0; j < kR; ++j) mine += top[j] != 0ull ? 1 : 0;
            const int pos = atomicAdd(&misc[M_COUNT], mine);
#pragma unroll
            for (int j = 0; j < kR; ++j)
                if (j < mine) U[pos + j] = top[j];
            const unsigned long long tau = epi_max_u64(top[kR - 1], red, etid); // has a barrier: U complete
            const int nu = misc[M_COUNT];
            unsigned long long theta_c = tau;
            int cnt;
            if (nu <= keep) { // publish everything
                for (int j = etid; j < nu; j += kEpiThreads) out[j] = U[j];
                cnt = nu;
            } else {
                // 2. one radix digit of the high words keeps >= keep keys; an exact cut when it keeps too many
                SelectSmem<uint32_t> *sel = reinterpret_cast<SelectSmem<uint32_t> *>(sp + OFF_SEL);
                uint32_t kmin;
                int lead, n_ge;
                const int bin = top_bin32<kEpiThreads, kEpiBar>(
                    nu, keep, [&](int j) { return (uint32_t)(U[j] >> 32); }, sel, kmin, lead, n_ge, etid);
                unsigned long long thr = 0ull;
                if (n_ge > co.lcap)
                    thr = block_kth64<kEpiThreads, kEpiBar>(nu, keep, [&](int j) { return U[j]; }, sel, etid);
                unsigned long long mx = 0ull; // the largest key that is not published
                for (int j = etid; j < nu; j += kEpiThreads) {
                    const unsigned long long v = U[j];
                    const uint32_t hv = (uint32_t)(v >> 32) - kmin;
                    const bool keep = thr ? v >= thr : (lead >= 32 ? 0 : (int)((hv << lead) >> 24)) >= bin;
                    if (keep) out[atomicAdd(&misc[M_OUT], 1)] = v;
                    else mx = v > mx ? v : mx;
                }
                mx = epi_max_u64(mx, red, etid); // has a barrier: M_OUT complete
                cnt = misc[M_OUT];
                if (mx != 0ull && mx + 1 > theta_c) theta_c = mx + 1;
            }
            if (etid == 0) {
                co.count[oslot] = cnt;
                co.theta[oslot] = theta_c;
            }
        } else if (etid == 0) {
            co.count[oslot] = 0;
            co.theta[oslot] = ~0ull; // counts as saturated; the timeout flag marks the result invalid
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
// kernel 2: exact top-k of one query from the published lists (and saturated chunks' scores)
// ------------------------------------------------------------------------------------------
constexpr int kMergeThreads = 1024;
constexpr int kMaxSlots = 256; // list offsets: 8 per lane of one warp

__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(IndexerArgs a, ChunkOut co)
{
    extern __shared__ unsigned long long mv[];
    __shared__ SelectSmem<uint32_t> msel;
    __shared__ int s_cnt, s_nsat, s_off[kMaxSlots + 1], s_sat_off[kMaxSlots + 1], s_sat_slot[kMaxSlots];
    __shared__ unsigned long long s_theta[kMaxSlots];
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const int k = a.k, ns = co.n_slots;
    const int64_t nv = dec_nvis(a, r);
    const int chunk = query_chunk(nv, ns);
    const int lane = tid & 31, wid = tid >> 5;
    if (wid == 0) { // list offsets: lane l sums slots 8l .. 8l+7, then a warp scan
        int c[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int sl = 8 * lane + j;
            c[j] = sl < ns ? co.count[r * ns + sl] : 0;
            sum += c[j];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int o = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int sl = 8 * lane + j;
            if (sl < ns) s_off[sl] = o;
            o += c[j];
        }
        if (lane == 31) s_off[ns] = incl;
    }
    for (int sl = tid; sl < ns; sl += kMergeThreads) s_theta[sl] = co.theta[r * ns + sl];
    __syncthreads();
    const int total = s_off[ns];
    // 1. the published lists, one warp per list
    for (int sl = wid; sl < ns; sl += kMergeThreads / 32) {
        const unsigned long long *src = co.list + (r * ns + sl) * (int64_t)co.lcap;
        const int o = s_off[sl], c = s_off[sl + 1] - o;
        for (int i = lane; i < c; i += 32) mv[o + i] = src[i];
    }
    __syncthreads();
    // 2. theta = the k-th largest published key (0 when fewer than k are published), then the
    //    chunks that may hold unpublished keys >= theta
    const unsigned long long theta =
        total >= k ? block_kth64<kMergeThreads>(total, k, [&](int i) { return mv[i]; }, &msel) : 0ull;
    if (tid == 0) {
        int nsat = 0, o = 0;
        for (int sl = 0; sl < ns; ++sl) {
            if (s_theta[sl] > theta) {
                const int64_t n_s = nv - (int64_t)sl * chunk < chunk ? nv - (int64_t)sl * chunk : chunk;
                s_sat_slot[nsat] = sl;
                s_sat_off[nsat] = o;
                o += (int)(n_s > 0 ? n_s : 0);
                ++nsat;
            }
        }
        s_sat_off[nsat] = o;
        s_nsat = nsat;
        s_cnt = 0;
    }
    __syncthreads();
    const int nsat = s_nsat;
    unsigned long long *sel = mv + total; // the winners, padded to a power of two
    int ke;
    if (nsat == 0) { // every key >= theta is published: exactly min(k, total) of them
        ke = total < k ? total : k;
        for (int i = tid; i < total; i += kMergeThreads) {
            const unsigned long long v = mv[i];
            if (v >= theta) sel[atomicAdd(&s_cnt, 1)] = v;
        }
        __syncthreads();
    } else {
        // 3. saturated chunks join whole, from the stored scores (their published keys are dropped)
        for (int j = 0; j < nsat; ++j) {
            const int sl = s_sat_slot[j];
            for (int i = s_off[sl] + tid; i < s_off[sl + 1]; i += kMergeThreads) mv[i] = 0ull;
        }
        __syncthreads();
        const int nvirt = total + s_sat_off[nsat];
        const float *srow = a.scores + r * a.ld;
        auto get = [&](int i) -> unsigned long long {
            if (i < total) return mv[i];
            i -= total;
            int j = 0;
            while (j + 1 < nsat && i >= s_sat_off[j + 1]) ++j;
            const int64_t e = (int64_t)s_sat_slot[j] * chunk + (i - s_sat_off[j]);
            return ((unsigned long long)float_key(srow[e]) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)e);
        };
        int live = 0; // keys in the set (the dropped ones read 0)
        for (int i = tid; i < nvirt; i += kMergeThreads) live += get(i) != 0ull ? 1 : 0;
        for (int o = 16; o > 0; o >>= 1) live += __shfl_xor_sync(0xffffffffu, live, o);
        if ((tid & 31) == 0) atomicAdd(&s_cnt, live);
        __syncthreads();
        const int n_live = s_cnt;
        __syncthreads();
        ke = n_live < k ? n_live : k;
        // the k-th largest of the set (zeros sort below every key, so they never reach it)
        const unsigned long long thr =
            n_live > k ? block_kth64<kMergeThreads>(nvirt, k, get, &msel) : 1ull;
        if (tid == 0) s_cnt = 0;
        __syncthreads();
        for (int i = tid; i < nvirt; i += kMergeThreads) {
            const unsigned long long v = get(i);
            if (v != 0ull && v >= thr) {
                const int p = atomicAdd(&s_cnt, 1);
                if (p < ke) sel[p] = v;
            }
        }
        __syncthreads();
    }
    // 4. order the winners: score descending, then entry ascending (bitonic sort of the 64-bit keys)
    int n2 = 1;
    while (n2 < ke) n2 <<= 1;
    for (int i = ke + tid; i < n2; i += kMergeThreads) sel[i] = 0ull;
    __syncthreads();
    block_sort_desc64<kMergeThreads>(sel, n2);
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

// Chunking of the key lists: each query's keys are spread over n_slots chunks (query_chunk),
// enough that a chunk's expected share of k is at most kShareMax and that the launch fills the
// SMs; a chunk holds at most kChunk keys.  Every chunk publishes into a list of lcap slots, sized
// so that the merge holds all of a query's lists in shared memory.
struct Plan {
    int slots, lcap;
};

bool scan_plan(int64_t Nq, int64_t max_nvis, int k, int sms, Plan *p)
{
    int64_t want = sms / (Nq > 0 ? Nq : 1);
    const int64_t by_share = (k + kShareMax - 1) / kShareMax;
    if (want < by_share) want = by_share;
    if (want < 1) want = 1;
    int64_t ch = (max_nvis + want - 1) / want;
    ch = (ch + kKT - 1) / kKT * kKT;
    if (ch > kChunk) ch = kChunk;
    if (ch < kKT) ch = kKT;
    p->slots = (int)((max_nvis + ch - 1) / ch);
    if (p->slots < 1) p->slots = 1;
    int n2 = 1;
    while (n2 < k) n2 <<= 1;
    // a list needs room for its keep (largest for the query with the fewest chunks: at most k)
    // plus what one radix digit keeps above it; twice the keep is ample
    const int keep_max = query_keep(1, kKT, k, 1 << 30) > query_keep(max_nvis, query_chunk(max_nvis, p->slots), k, 1 << 30)
                             ? query_keep(1, kKT, k, 1 << 30)
                             : query_keep(max_nvis, query_chunk(max_nvis, p->slots), k, 1 << 30);
    int64_t lcap = 2 * (int64_t)keep_max;
    const int64_t room = (kMergeSmem - (int64_t)n2 * 8) / ((int64_t)p->slots * 8);
    if (lcap > room) lcap = room;
    if (lcap > kEpiThreads * kR) lcap = kEpiThreads * kR;
    p->lcap = (int)lcap;
    return p->slots <= kMaxSlots && p->lcap >= query_keep(max_nvis, query_chunk(max_nvis, p->slots), k, 1 << 30);
}

size_t lists_bytes(int64_t Nq, const Plan &p)
{
    return ((size_t)Nq * (size_t)p.slots * ((size_t)p.lcap * 8 + 8 + 4) + 255) / 256 * 256;
}

} // namespace

// Scratch of the decode path for this device: the chunk lists, counts and bounds, then every
// score ([Nq, ceil4(max_nvis)] fp32, re-read by the merge for saturated chunks).
size_t decode_indexer_need(int64_t Nq, int64_t max_nvis, int k)
{
    Plan p;
    scan_plan(Nq, max_nvis, k, device_sms(), &p);
    const size_t ld = (size_t)((max_nvis + 3) / 4 * 4);
    return lists_bytes(Nq, p) + (size_t)Nq * ld * 4 + 256;
}

// Workspace of the decode path on the current device (the chunking follows its SM count).
size_t decode_indexer_workspace(int64_t Nq, int64_t max_nvis, int k)
{
    return decode_indexer_need(Nq, max_nvis, k) + 256;
}

bool decode_indexer_eligible(const IndexerArgs &a)
{
    if (a.fmt != CSA_FP4 || a.H != kHI || a.d != kDI || a.Nq <= 0 || a.Nq > (1 << 24) || a.max_nvis <= 0) return false;
    if (a.pages && (a.page_rows < 8 || a.page_rows > kKT || (a.page_rows & (a.page_rows - 1)))) return false;
    if (a.k > 2048 || a.k4.n >= (1ll << 31) || a.Nq * kHI >= (1ll << 31)) return false;
    Plan p;
    return scan_plan(a.Nq, a.max_nvis, a.k, device_sms(), &p) && (int64_t)p.slots * a.Nq < (1ll << 31);
}

cudaError_t launch_indexer_decode(const IndexerArgs &a0, void *ws, cudaStream_t st)
{
    Plan p;
    if (!scan_plan(a0.Nq, a0.max_nvis, a0.k, device_sms(), &p)) return cudaErrorInvalidValue;
    uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + 255) / 256 * 256;
    ChunkOut co;
    co.list = reinterpret_cast<unsigned long long *>(base);
    co.theta = co.list + (size_t)a0.Nq * p.slots * p.lcap;
    co.count = reinterpret_cast<int *>(co.theta + (size_t)a0.Nq * p.slots);
    co.n_slots = p.slots;
    co.lcap = p.lcap;
    IndexerArgs a = a0;
    a.scores = reinterpret_cast<float *>(base + lists_bytes(a0.Nq, p));
    a.ld = (a0.max_nvis + 3) / 4 * 4;
    Maps maps;
    memset(&maps, 0, sizeof(maps));
    const uint64_t key_rows = a.k4.n > 0 ? (uint64_t)a.k4.n : 1; // an empty key array is never read
    if (!tma::encode_u8_rows_sw64(&maps.q, a.q4.codes, (uint64_t)a.Nq * kHI, kDI / 2, kHI) ||
        !tma::encode_u8_rows_sw64(&maps.k, a.k4.codes, key_rows, kDI / 2, kKT))
        return cudaErrorInvalidValue;
    if (a.pages && !tma::encode_u8_rows_sw64(&maps.kp, a.k4.codes, key_rows, kDI / 2, (uint32_t)a.page_rows))
        return cudaErrorInvalidValue;
    // permuted tiles when the key rows come in whole groups of 4 and the arrays are 16-byte aligned
    // (the encoder checks); otherwise every tile takes the natural order
    maps.perm = (key_rows % 4 == 0) && (!a.pages || a.page_rows >= 32) &&
                tma::encode_u8_rows_sw64_stride4(&maps.kq4, a.k4.codes, key_rows, kKT / 4) &&
                tma::encode_u32_quads(&maps.sq, a.k4.scales, key_rows, kKT / 4) &&
                (!a.pages || (tma::encode_u8_rows_sw64_stride4(&maps.kq4p, a.k4.codes, key_rows, (uint32_t)a.page_rows / 4) &&
                              tma::encode_u32_quads(&maps.sqp, a.k4.scales, key_rows, (uint32_t)a.page_rows / 4)))
                    ? 1
                    : 0;
    cudaError_t e = cudaFuncSetAttribute(decode_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    decode_scan_kernel<<<(unsigned)((int64_t)p.slots * a.Nq), kThreads, SMEM_ALLOC, st>>>(a, maps, co);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int n2 = 1;
    while (n2 < a.k) n2 <<= 1;
    const size_t msm = (size_t)p.slots * p.lcap * 8 + (size_t)n2 * 8;
    e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msm);
    if (e != cudaSuccess) return e;
    topk_merge_kernel<<<(unsigned)a.Nq, kMergeThreads, msm, st>>>(a, co);
    return cudaGetLastError();
}

} // namespace csa
