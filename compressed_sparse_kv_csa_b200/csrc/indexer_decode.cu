// indexer_decode.cu -- lightning-indexer scan + top-k for decode: few queries (one new token per
// sequence), very long key lists (262,144 FP4 keys per sequence at 1M context).
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 Eq. 16 and the Indexer listing (I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . K[s,:]) over
// s < N_vis(t), then the k best entries); the indexer's QK path runs in FP4 E2M1 with 32-element
// block scales (itsolotime.com Q&A essay on DeepSeek-V4, Question 4; "technical ledger" page).
//
// Kernel 1 (grid = key chunks x queries, about one CTA per SM): each CTA streams its chunk of up
// to 16,384 FP4 keys
//   * one lane issues bulk copies of 128-key tiles (8 KB of E2M1 codes + 512 B of E8M0 scales)
//     into a 4-stage ring;
//   * 8 converter warps turn a tile into f16 in the 128-byte-swizzled MMA layout with the
//     hardware E2M1x2 -> f16x2 conversion, folding each block's power-of-two scale in with one
//     f16x2 multiply (exact while the block's scale exponent lies in [-23, 13]; a non-zero block
//     outside that range sets CSA_DEVERR_RANGE, its scores are then approximate);
//   * one lane issues tcgen05 M=128 (keys) x N=64 (heads) x K=128 f16 MMAs against the query,
//     converted the same way once per CTA, into a double-buffered TMEM accumulator;
//   * 4 epilogue warps (one per TMEM lane quadrant) reduce w . ReLU(.) over the 64 heads per key
//     (one key per lane) into a shared-memory score array;
//   * finally all warps select the chunk's exact top-min(k, n) (radix select on order-preserving
//     score keys, equal scores to the lower entry) and write them as 64-bit candidates
//     (score key << 32 | ~entry) to the workspace.
// Kernel 2 (one CTA per query): the exact top-k of the union of its chunks' candidates (the
//   global top-k is contained in it), sorted by score descending then entry ascending.
// Every wait is bounded (%globaltimer); a timeout sets CSA_DEVERR_TIMEOUT and the CTA returns.
#include "common.cuh"
#include "tc_common.cuh"
#include "select.cuh"

namespace csa {

namespace {

using namespace tc;

constexpr int kHI = 64, kDI = 128, kKT = 128, kStages = 4;
constexpr int kChunk = 16384;                 // most keys per CTA (scores stay in shared memory)
constexpr int kConvWarps = 8;
constexpr int kProdWarp = 0, kConvWarp0 = 1, kEpiWarp0 = kConvWarp0 + kConvWarps, kMmaWarp = kEpiWarp0 + 4;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr uint32_t kStageCodes = kKT * kDI / 2;     // 8192 B
constexpr uint32_t kStageBytes = kStageCodes + kKT * (kDI / 32); // + 512 B scales

constexpr uint32_t OFF_SC = 0;                               // scores [16384] fp32 = 64 KB
constexpr uint32_t OFF_A = 65536;                            // 2 x [128 x 128] f16 = 64 KB
constexpr uint32_t OFF_B = OFF_A + 65536;                    // [64 x 128] f16 = 16 KB
constexpr uint32_t OFF_ST = OFF_B + 16384;                   // 4 x 8704 B staging
constexpr uint32_t OFF_W = OFF_ST + kStages * kStageBytes;   // w [64] fp32
constexpr uint32_t OFF_HIST = OFF_W + 256;                   // selection scratch (< 2 KB)
constexpr uint32_t OFF_MISC = OFF_HIST + 2048;               // counters
constexpr uint32_t OFF_BAR = OFF_MISC + 256;
constexpr uint32_t OFF_TMEM = OFF_BAR + 256;
constexpr uint32_t SMEM_USED = OFF_TMEM + 16;
constexpr uint32_t SMEM_ALLOC = ((SMEM_USED + 127) / 128) * 128 + 1024;

enum { B_STFULL = 0, B_STEMPTY = B_STFULL + kStages, B_AFULL = B_STEMPTY + kStages, B_AEMPTY = B_AFULL + 2,
       B_DFULL = B_AEMPTY + 2, B_DEMPTY = B_DFULL + 2, B_FINAL = B_DEMPTY + 2, NUM_BARS };

constexpr uint32_t IDESC = idesc_f16_f32(128, 64);

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

// f16 bits of 2^e for e in [-24, 15] (clamped outside)
__device__ __forceinline__ uint32_t f16_pow2x2(int e)
{
    uint32_t b;
    if (e >= -14) b = (uint32_t)((e > 15 ? 15 : e) + 15) << 10;
    else b = (e >= -24) ? (1u << (e + 24)) : 0u;
    return b | (b << 16);
}

// E2M1 magnitudes are m * 2^e with m in [0.5, 6]: in f16 exactly for block exponents e in
// [-23, 13] (the smallest, 0.5 * 2^-23, is f16's smallest subnormal; the largest, 6 * 2^13,
// is below 65504).  An all-zero block is exact for any scale.
__device__ __forceinline__ bool fp4_block_exact_f16(uint32_t scale_byte, uint4 codes)
{
    const bool zero = ((codes.x | codes.y | codes.z | codes.w) & 0x77777777u) == 0u;
    return zero || (scale_byte >= 127u - 23u && scale_byte <= 127u + 13u);
}

__device__ __forceinline__ uint32_t hmul2(uint32_t x, uint32_t y)
{
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
    return r;
}

// 32 E2M1 elements (16 bytes) scaled by 2^e -> 16 f16x2 words
__device__ __forceinline__ void e2m1x32_to_f16(uint4 codes, int e, uint32_t (&out)[16])
{
    const uint32_t s = f16_pow2x2(e);
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h0, h1, h2, h3;
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
            "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
            "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
            "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
            : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
            : "r"(w[i]));
        out[4 * i + 0] = hmul2(h0, s);
        out[4 * i + 1] = hmul2(h1, s);
        out[4 * i + 2] = hmul2(h2, s);
        out[4 * i + 3] = hmul2(h3, s);
    }
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Write 32 converted elements (block `blk` of row `row`) into a swizzled K-major f16 operand made
// of 64-element sub-tiles of `sub_bytes` bytes.
__device__ __forceinline__ void store_block(uint32_t op, uint32_t sub_bytes, int row, int blk, const uint32_t (&v)[16])
{
    const uint32_t sub = op + (uint32_t)(blk >> 1) * sub_bytes;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        sts128(sub + sw128_off(row, 32 * (blk & 1) + 8 * j), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ bool wwait(uint32_t bar, uint32_t parity)
{
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------------------------------------
// block-wide exact top-k of n (<= kChunk) scores in shared memory -> 64-bit candidates
// ------------------------------------------------------------------------------------------
template <int NT>
__device__ void chunk_topk(uint32_t sc_base, int n, int k, int64_t entry0, unsigned long long *out, int *out_count,
                           SelectSmem<uint32_t> *sel, int *misc)
{
    const int tid = threadIdx.x;
    auto score_key = [&](int i) {
        float f;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f) : "r"(sc_base + 4u * (uint32_t)i));
        return float_key(f);
    };
    auto cand = [&](uint32_t key, int i) {
        return ((unsigned long long)key << 32) | (unsigned long long)(0xffffffffu - (uint32_t)(entry0 + i));
    };
    if (n <= k) {
        for (int i = tid; i < n; i += NT) out[i] = cand(score_key(i), i);
        if (tid == 0) *out_count = n;
        return;
    }
    uint32_t thr;
    int n_gt;
    block_kth<NT, uint32_t>(n, k, score_key, sel, thr, n_gt);
    const int rem = k - n_gt;
    if (tid == 0) { misc[2] = 0; misc[3] = 0; }
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
        const uint32_t key = score_key(i);
        if (key > thr) {
            const int p = atomicAdd(&misc[2], 1);
            if (p < n_gt) out[p] = cand(key, i);
        }
    }
    __syncthreads();
    // equal to the threshold: lowest entries first (ordered block scan)
    int *warp_cnt = misc + 8;
    for (int base = 0; base < n; base += NT) {
        if (misc[3] >= rem) break; // read after a barrier: uniform
        const int i = base + tid;
        const bool eq = (i < n) && (score_key(i) == thr);
        const unsigned bal = __ballot_sync(0xffffffffu, eq);
        const int lane = tid & 31, wid = tid >> 5;
        if (lane == 0) warp_cnt[wid] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < NT / 32; ++w) {
            if (w < wid) before += warp_cnt[w];
            total += warp_cnt[w];
        }
        const int rank = misc[3] + before + __popc(bal & ((1u << lane) - 1u));
        if (eq && rank < rem) out[n_gt + rank] = cand(thr, i);
        __syncthreads();
        if (tid == 0) misc[3] += total;
        __syncthreads();
    }
    if (tid == 0) *out_count = k;
}

// ------------------------------------------------------------------------------------------
// kernel 1: FP4 key scan (tcgen05) + chunk top-k
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) decode_scan_kernel(IndexerArgs a, int n_slots, int chunk,
                                                                  unsigned long long *cand, int *cand_count)
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

    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            uint32_t cnt = 1;
            if ((b >= B_STEMPTY && b < B_STEMPTY + kStages) || (b >= B_AFULL && b < B_AFULL + 2))
                cnt = 32 * kConvWarps;
            if (b >= B_DEMPTY && b < B_DEMPTY + 2) cnt = 128;
            if (b >= B_STFULL && b < B_STFULL + kStages) cnt = 1 + 32; // expect_tx arrive + 32 cp.async arrivals
            mbar_init(bar(b), cnt);
        }
        mbar_init_fence();
    }
    if (warp == kMmaWarp) tmem_alloc(base + OFF_TMEM, 128);
    // query (64 heads x 128) -> f16 B operand with its block scales folded in; weights -> smem
    if (tid < 256) {
        const int h = tid >> 2, blk = tid & 3;
        const int64_t qr = r * kHI + h;
        const uint4 codes = *reinterpret_cast<const uint4 *>(a.q4.codes + qr * (kDI / 2) + 16 * blk);
        const uint32_t sb = a.q4.scales[qr * (kDI / 32) + blk];
        uint32_t v[16];
        e2m1x32_to_f16(codes, (int)sb - 127, v);
        if (!fp4_block_exact_f16(sb, codes)) flag_error(a.err, CSA_DEVERR_RANGE);
        store_block(base + OFF_B, 8192u, h, blk, v);
    } else if (tid < 256 + 64) {
        const int h = tid - 256;
        reinterpret_cast<float *>(sp + OFF_W)[h] = a.w[r * kHI + h];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + OFF_TMEM);

    bool ok = true;
    if (warp == kProdWarp) {
        // codes: one bulk copy per tile (row0 * 64 bytes is always 16-byte aligned); scales: 4-byte
        // cp.async per key row by the warp (a sequence's key offset need not be a multiple of 4
        // rows), each lane arriving on the stage barrier when its copies land
        for (int i = 0; i < ntiles && ok; ++i) {
            const uint32_t st = i % kStages;
            if (i >= kStages && !wwait(bar(B_STEMPTY + st), ((i / kStages) - 1) & 1)) { ok = false; break; }
            const int64_t row0 = key0 + (int64_t)i * kKT;
            const int64_t rows_left = a.k4.n - row0; // never read past the key array
            const uint32_t nr = (uint32_t)(rows_left < kKT ? rows_left : kKT);
            const uint32_t dst = base + OFF_ST + st * kStageBytes;
            for (uint32_t j = lane; j < nr; j += 32) // one 4-byte word of scales per key row
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst + kStageCodes + 4u * j),
                             "l"(a.k4.scales + (row0 + j) * (kDI / 32))
                             : "memory");
            asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(B_STFULL + st)) : "memory");
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(B_STFULL + st), nr * (kDI / 2));
                bulk_g2s(dst, a.k4.codes + row0 * (kDI / 2), nr * (kDI / 2), bar(B_STFULL + st));
            }
        }
    } else if (warp >= kConvWarp0 && warp < kEpiWarp0) {
        const int ct = tid - 32 * kConvWarp0; // 0 .. 32*kConvWarps-1
        bool out_of_range = false;            // a non-zero block whose scale f16 cannot carry exactly
        for (int i = 0; i < ntiles && ok; ++i) {
            const uint32_t st = i % kStages, ab = i & 1;
            if (!wwait(bar(B_STFULL + st), (i / kStages) & 1)) { ok = false; break; }
            if (i >= 2 && !wwait(bar(B_AEMPTY + ab), ((i >> 1) - 1) & 1)) { ok = false; break; }
            const uint32_t stb = base + OFF_ST + st * kStageBytes;
            const int valid = n - i * kKT; // keys of this tile inside the chunk
#pragma unroll 1
            for (int p = 0; p < 512 / (32 * kConvWarps); ++p) { // 128 keys x 4 blocks per tile
                const int key = (ct >> 2) + (8 * kConvWarps) * p, blk = ct & 3;
                uint32_t v[16];
                if (key < valid) {
                    uint4 codes;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(codes.x), "=r"(codes.y), "=r"(codes.z), "=r"(codes.w)
                                 : "r"(stb + (uint32_t)key * 64u + 16u * blk));
                    uint32_t sb;
                    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(sb) : "r"(stb + kStageCodes + (uint32_t)key * 4u + blk));
                    e2m1x32_to_f16(codes, (int)sb - 127, v);
                    out_of_range |= !fp4_block_exact_f16(sb, codes);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = 0u;
                }
                store_block(base + OFF_A + ab * 32768u, 16384u, key, blk, v);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(B_STEMPTY + st));
            mbar_arrive(bar(B_AFULL + ab));
        }
        if (out_of_range) flag_error(a.err, CSA_DEVERR_RANGE);
    } else if (warp >= kEpiWarp0 && warp < kMmaWarp) {
        const int quad = warp & 3;
        const float *wsm = reinterpret_cast<const float *>(sp + OFF_W);
        float *scs = reinterpret_cast<float *>(sp + OFF_SC);
        for (int i = 0; i < ntiles && ok; ++i) {
            const uint32_t db = i & 1;
            if (!wwait(bar(B_DFULL + db), (i >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            uint32_t r0[32], r1[32];
            const uint32_t ta = tmem + db * 64u + ((uint32_t)(32 * quad) << 16);
            tmem_ld32(ta, r0);
            tmem_ld32(ta + 32, r1);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(bar(B_DEMPTY + db));
            float s = 0.f;
#pragma unroll
            for (int h = 0; h < 32; ++h) s = fmaf(wsm[h], fmaxf(__uint_as_float(r0[h]), 0.f), s);
#pragma unroll
            for (int h = 0; h < 32; ++h) s = fmaf(wsm[32 + h], fmaxf(__uint_as_float(r1[h]), 0.f), s);
            const int key = i * kKT + 32 * quad + lane;
            if (key < n) scs[key] = s;
        }
    } else if (warp == kMmaWarp && lane == 0) {
        for (int i = 0; i < ntiles && ok; ++i) {
            const uint32_t ab = i & 1, db = i & 1;
            if (!mbar_wait(bar(B_AFULL + ab), (i >> 1) & 1)) { ok = false; break; }
            if (i >= 2 && !mbar_wait(bar(B_DEMPTY + db), ((i >> 1) - 1) & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = sdesc_sw128(base + OFF_A + ab * 32768u + 16384u * sub + 32u * kk, 16, 1024);
                    const uint64_t bd = sdesc_sw128(base + OFF_B + 8192u * sub + 32u * kk, 16, 1024);
                    mma_bf16(tmem + db * 64u, ad, bd, IDESC, (sub | kk) != 0); // same instruction; f16 formats in IDESC
                }
            }
            mma_commit(bar(B_AEMPTY + ab));
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
    if (warp == kMmaWarp) tmem_dealloc(tmem, 128);
    chunk_topk<kThreads>(base + OFF_SC, n, a.k, c0, out, out_count,
                         reinterpret_cast<SelectSmem<uint32_t> *>(sp + OFF_HIST), reinterpret_cast<int *>(sp + OFF_MISC));
}

// ------------------------------------------------------------------------------------------
// kernel 2: exact top-k over the chunk candidates of one query
// ------------------------------------------------------------------------------------------
constexpr int kMergeThreads = 1024;

__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(IndexerArgs a, int n_slots,
                                                                     const unsigned long long *cand,
                                                                     const int *cand_count)
{
    extern __shared__ unsigned long long mv[];
    __shared__ SelectSmem<unsigned long long> msel;
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
    for (int s = 0; s < n_slots; ++s) {
        const int c = cand_count[r * n_slots + s];
        for (int i = tid; i < c; i += kMergeThreads) mv[s_off[s] + i] = cand[(r * n_slots + s) * k + i];
    }
    __syncthreads();
    const int ke = total < k ? total : k;
    unsigned long long *sel = mv + total; // ke winners
    if (total > k) {
        // the k-th largest of the unique 64-bit keys
        unsigned long long thr64;
        int n_gt64;
        block_kth<kMergeThreads, unsigned long long>(total, k, [&](int i) { return mv[i]; }, &msel, thr64, n_gt64);
        if (tid == 0) s_cnt = 0;
        __syncthreads();
        const unsigned long long thr = thr64;
        for (int i = tid; i < total; i += kMergeThreads) {
            const unsigned long long v = mv[i];
            if (v >= thr) {
                const int p = atomicAdd(&s_cnt, 1);
                if (p < ke) sel[p] = v;
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
    cudaError_t e = cudaFuncSetAttribute(decode_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    decode_scan_kernel<<<dim3((unsigned)slots, (unsigned)a.Nq), kThreads, SMEM_ALLOC, st>>>(a, slots, chunk, cand, cnt);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int n2 = 1;
    while (n2 < a.k) n2 <<= 1;
    const size_t msm = (size_t)(slots * a.k + n2) * 8;
    e = cudaFuncSetAttribute(decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msm);
    if (e != cudaSuccess) return e;
    decode_merge_kernel<<<(unsigned)a.Nq, kMergeThreads, msm, st>>>(a, slots, cand, cnt);
    return cudaGetLastError();
}

} // namespace csa
