// select.cuh -- block-wide exact radix selection of the k-th largest key (32- or 64-bit,
// order-preserving), shared by the top-k kernels.
//
// The keys of one selection usually share their leading bits (scores of one query lie within a few
// binades), so the digits are taken from the bits that differ inside the group: keys are offset
// by the group minimum and left-aligned on the highest bit of (max - min) before 8-bit digit
// passes.  The crossing bin of each pass is found by a warp suffix scan over the 256 bins.
//
// A selection runs on a group of NT threads (local ids 0..NT-1).  BAR = 0 synchronises the whole
// block (__syncthreads, the group is the block); BAR > 0 uses named barrier BAR for a group that
// is part of a block (e.g. the epilogue warps of a warp-specialised kernel).
#pragma once

#include <stdint.h>

namespace csa {

template <typename K> struct KeyBits;
template <> struct KeyBits<uint32_t> { static constexpr int bits = 32; };
template <> struct KeyBits<unsigned long long> { static constexpr int bits = 64; };

template <typename K> __device__ __forceinline__ int clz_key(K x);
template <> __device__ __forceinline__ int clz_key<uint32_t>(uint32_t x) { return __clz(x); }
template <> __device__ __forceinline__ int clz_key<unsigned long long>(unsigned long long x) { return __clzll(x); }

template <typename K> __device__ __forceinline__ K warp_min_key(K v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const K w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w < v ? w : v;
    }
    return v;
}
template <typename K> __device__ __forceinline__ K warp_max_key(K v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const K w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

template <int NT, int BAR> __device__ __forceinline__ void group_sync()
{
    if constexpr (BAR == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// Scratch in shared memory for block_kth.
template <typename K> struct SelectSmem {
    int hist[256];
    K red[64];
    K kmin, kmax;
    int bin, rem;
    int cnt[32];
    uint32_t mn[32];
};

// Among the n keys get(i) (i < n), find thr = the k-th largest key (1 <= k <= n) and
// n_gt = the number of keys strictly greater than thr.  All NT threads of the group call it (ltid =
// the caller's id in the group) and all receive the result.
template <int NT, typename K, int BAR = 0, typename Get>
__device__ void block_kth(int n, int k, Get get, SelectSmem<K> *sm, K &thr, int &n_gt, int ltid = threadIdx.x)
{
    constexpr int KB = KeyBits<K>::bits;
    const int lane = ltid & 31, wid = ltid >> 5;
    // 1. range of the keys
    K lo = ~(K)0, hi = 0;
    for (int i = ltid; i < n; i += NT) {
        const K v = get(i);
        lo = v < lo ? v : lo;
        hi = v > hi ? v : hi;
    }
    lo = warp_min_key(lo);
    hi = warp_max_key(hi);
    if (lane == 0) { sm->red[wid] = lo; sm->red[32 + wid] = hi; }
    group_sync<NT, BAR>();
    if (ltid == 0) {
        K a = sm->red[0], b = sm->red[32];
        for (int w = 1; w < NT / 32; ++w) {
            a = sm->red[w] < a ? sm->red[w] : a;
            b = sm->red[32 + w] > b ? sm->red[32 + w] : b;
        }
        sm->kmin = a;
        sm->kmax = b;
    }
    group_sync<NT, BAR>();
    const K kmin = sm->kmin, range = sm->kmax - sm->kmin;
    if (range == 0) { // all keys equal
        thr = kmin;
        n_gt = 0;
        group_sync<NT, BAR>(); // kmin / kmax are read before anyone reuses the scratch
        return;
    }
    const int lead = clz_key<K>(range);      // left-align the significant bits
    const int nbits = KB - lead;
    const int passes = (nbits + 7) / 8;
    K prefix = 0, pmask = 0; // over the left-aligned relative keys
    int rem = k;
    for (int p = 0; p < passes; ++p) {
        const int shift = KB - 8 * (p + 1);
        for (int i = ltid; i < 256; i += NT) sm->hist[i] = 0;
        group_sync<NT, BAR>();
        for (int i = ltid; i < n; i += NT) {
            const K r = (get(i) - kmin) << lead;
            if ((r & pmask) == prefix) atomicAdd(&sm->hist[(int)((r >> shift) & 255)], 1);
        }
        group_sync<NT, BAR>();
        if (wid == 0) { // suffix scan from the top bin: lane l owns bins 255-8l .. 248-8l
            int c[8], s = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = sm->hist[255 - 8 * lane - j]; s += c[j]; }
            int incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - s;
            const bool cross = excl < rem && incl >= rem;
            const unsigned who = __ballot_sync(0xffffffffu, cross);
            if (cross && lane == __ffs(who) - 1) {
                int cum = excl, j = 0;
                for (; j < 7; ++j) {
                    if (cum + c[j] >= rem) break;
                    cum += c[j];
                }
                sm->bin = 255 - 8 * lane - j;
                sm->rem = rem - cum;
            }
        }
        group_sync<NT, BAR>();
        prefix |= (K)sm->bin << shift;
        pmask |= (K)255 << shift;
        rem = sm->rem;
        group_sync<NT, BAR>();
    }
    thr = (prefix >> lead) + kmin;
    n_gt = k - rem;
}

// One radix digit of a selection, for a cut that may keep a few more keys than asked: the n
// 32-bit keys get(i) (n >= 1) are offset by their minimum and left-aligned on the highest bit of
// their range, and binned by the top 8 bits of the result.  Returns the highest bin b such that
// at least `want` keys (1 <= want <= n) lie in bins >= b, with the bin rule in kmin / lead (a key
// v lies in bin ((v - kmin) << lead) >> 24; lead = 32 puts every key in bin 0 when all are equal)
// and the number of keys in bins >= b in n_ge.  Same calling rules as block_kth.
template <int NT, int BAR = 0, typename Get>
__device__ int top_bin32(int n, int want, Get get, SelectSmem<uint32_t> *sm, uint32_t &kmin, int &lead, int &n_ge,
                         int ltid = threadIdx.x)
{
    const int lane = ltid & 31, wid = ltid >> 5;
    uint32_t lo = 0xffffffffu, hi = 0;
    for (int i = ltid; i < n; i += NT) {
        const uint32_t v = get(i);
        lo = v < lo ? v : lo;
        hi = v > hi ? v : hi;
    }
    lo = warp_min_key(lo);
    hi = warp_max_key(hi);
    if (lane == 0) { sm->red[wid] = lo; sm->red[32 + wid] = hi; }
    for (int i = ltid; i < 256; i += NT) sm->hist[i] = 0;
    group_sync<NT, BAR>();
    uint32_t a = sm->red[0], b = sm->red[32];
    for (int w = 1; w < NT / 32; ++w) {
        a = sm->red[w] < a ? sm->red[w] : a;
        b = sm->red[32 + w] > b ? sm->red[32 + w] : b;
    }
    kmin = a;
    lead = (b == a) ? 32 : __clz(b - a);
    for (int i = ltid; i < n; i += NT) {
        const uint32_t v = get(i) - kmin;
        atomicAdd(&sm->hist[lead >= 32 ? 0 : (int)((v << lead) >> 24)], 1);
    }
    group_sync<NT, BAR>();
    if (wid == 0) { // suffix scan from the top bin: lane l owns bins 255-8l .. 248-8l
        int c[8], s = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { c[j] = sm->hist[255 - 8 * lane - j]; s += c[j]; }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int excl = incl - s;
        const bool cross = excl < want && incl >= want;
        const unsigned who = __ballot_sync(0xffffffffu, cross);
        if (cross && lane == __ffs(who) - 1) {
            int cum = excl, j = 0;
            for (; j < 7; ++j) {
                if (cum + c[j] >= want) break;
                cum += c[j];
            }
            sm->bin = 255 - 8 * lane - j;
            sm->rem = cum + c[j];
        }
    }
    group_sync<NT, BAR>();
    const int bin = sm->bin;
    n_ge = sm->rem;
    group_sync<NT, BAR>(); // the scratch is read before anyone reuses it
    return bin;
}

// The k-th largest of n unique 64-bit keys (1 <= k <= n): a 32-bit radix selection on the high
// words, then -- only when several keys share the threshold's high word and not all of them are
// needed -- a second one on the low words of those ties.  Same calling rules as block_kth.
template <int NT, int BAR = 0, typename Get>
__device__ unsigned long long block_kth64(int n, int k, Get get, SelectSmem<uint32_t> *sm, int ltid = threadIdx.x)
{
    uint32_t thr_hi;
    int n_gt;
    block_kth<NT, uint32_t, BAR>(n, k, [&](int i) { return (uint32_t)(get(i) >> 32); }, sm, thr_hi, n_gt, ltid);
    const int need = k - n_gt; // >= 1 keys with the threshold's high word
    // count the ties and find their smallest low word
    int cnt = 0;
    uint32_t mn = 0xffffffffu;
    for (int i = ltid; i < n; i += NT) {
        const unsigned long long v = get(i);
        if ((uint32_t)(v >> 32) == thr_hi) {
            ++cnt;
            mn = min(mn, (uint32_t)v);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    const int lane = ltid & 31, wid = ltid >> 5;
    if (lane == 0) { sm->cnt[wid] = cnt; sm->mn[wid] = mn; }
    group_sync<NT, BAR>();
    int tot = 0;
    uint32_t lo = 0xffffffffu;
    for (int w = 0; w < NT / 32; ++w) {
        tot += sm->cnt[w];
        lo = min(lo, sm->mn[w]);
    }
    group_sync<NT, BAR>();
    if (tot > need) { // select among the ties (non-ties map to 0, below every tie's low word)
        uint32_t thr_lo;
        int g;
        block_kth<NT, uint32_t, BAR>(n, need, [&](int i) {
            const unsigned long long v = get(i);
            return (uint32_t)(v >> 32) == thr_hi ? (uint32_t)v : 0u;
        }, sm, thr_lo, g, ltid);
        lo = thr_lo;
    }
    return ((unsigned long long)thr_hi << 32) | lo;
}

// Sorts a[0 .. n2) (n2 a power of two, 64-bit keys) into descending order with a bitonic network.
// The compare-exchange steps whose partners are less than 32 apart run in registers (element i is
// held by lane i % 32 of a warp, the partner's key comes by shuffle), so a barrier is taken only
// for the steps with partners 32 or more apart and once per merge size.  All NT threads of the
// group call it; the caller synchronises before (a[] complete) and may read a[] right after.
template <int NT, int BAR = 0>
__device__ void block_sort_desc64(unsigned long long *a, int n2, int ltid = threadIdx.x)
{
    static_assert(NT % 32 == 0, "whole warps");
    auto reg_steps = [&](int size_lo, int size_hi, int first_stride) {
        // sizes size_lo..size_hi (powers of two), strides < 32, first size starting at first_stride
        for (int i0 = 0; i0 < n2; i0 += NT) { // uniform trip count: every lane takes part in the shuffles
            const int i = i0 + ltid;
            const bool in = i < n2;
            unsigned long long v = in ? a[i] : 0ull;
            for (int size = size_lo; size <= size_hi; size <<= 1) {
                for (int st = (size == size_lo ? first_stride : size >> 1); st > 0; st >>= 1) {
                    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, st);
                    const bool keep_max = ((i & st) == 0) == ((i & size) == 0);
                    v = keep_max ? (w > v ? w : v) : (w < v ? w : v);
                }
            }
            if (in) a[i] = v;
        }
        group_sync<NT, BAR>();
    };
    if (n2 < 2) return;
    reg_steps(2, n2 < 32 ? n2 : 32, 1);
    for (int size = 64; size <= n2; size <<= 1) {
        for (int st = size >> 1; st >= 32; st >>= 1) {
            for (int i = ltid; i < n2; i += NT) {
                const int j = i ^ st;
                if (j > i) {
                    const bool desc = (i & size) == 0;
                    const unsigned long long x = a[i], y = a[j];
                    if (desc ? (x < y) : (x > y)) { a[i] = y; a[j] = x; }
                }
            }
            group_sync<NT, BAR>();
        }
        reg_steps(size, size, 16);
    }
}

} // namespace csa
