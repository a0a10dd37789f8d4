// select.cuh -- block-wide exact radix selection of the k-th largest key (32- or 64-bit,
// order-preserving), shared by the top-k kernels.
//
// The keys of one selection usually share their leading bits (scores of one query lie within a few
// binades), so the digits are taken from the bits that differ inside the block: keys are offset
// by the block minimum and left-aligned on the highest bit of (max - min) before 8-bit digit
// passes.  The crossing bin of each pass is found by a warp suffix scan over the 256 bins.
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

// Scratch in shared memory for block_kth.
template <typename K> struct SelectSmem {
    int hist[256];
    K red[64];
    K kmin, kmax;
    int bin, rem;
};

// Among the n keys get(i) (i < n), find thr = the k-th largest key (1 <= k <= n) and
// n_gt = the number of keys strictly greater than thr.  All NT threads of the block call it and
// all receive the result.
template <int NT, typename K, typename Get>
__device__ void block_kth(int n, int k, Get get, SelectSmem<K> *sm, K &thr, int &n_gt)
{
    constexpr int KB = KeyBits<K>::bits;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // 1. range of the keys
    K lo = ~(K)0, hi = 0;
    for (int i = tid; i < n; i += NT) {
        const K v = get(i);
        lo = v < lo ? v : lo;
        hi = v > hi ? v : hi;
    }
    lo = warp_min_key(lo);
    hi = warp_max_key(hi);
    if (lane == 0) { sm->red[wid] = lo; sm->red[32 + wid] = hi; }
    __syncthreads();
    if (tid == 0) {
        K a = sm->red[0], b = sm->red[32];
        for (int w = 1; w < NT / 32; ++w) {
            a = sm->red[w] < a ? sm->red[w] : a;
            b = sm->red[32 + w] > b ? sm->red[32 + w] : b;
        }
        sm->kmin = a;
        sm->kmax = b;
    }
    __syncthreads();
    const K kmin = sm->kmin, range = sm->kmax - sm->kmin;
    if (range == 0) { // all keys equal
        thr = kmin;
        n_gt = 0;
        return;
    }
    const int lead = clz_key<K>(range);      // left-align the significant bits
    const int nbits = KB - lead;
    const int passes = (nbits + 7) / 8;
    K prefix = 0, pmask = 0; // over the left-aligned relative keys
    int rem = k;
    for (int p = 0; p < passes; ++p) {
        const int shift = KB - 8 * (p + 1);
        for (int i = tid; i < 256; i += NT) sm->hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += NT) {
            const K r = (get(i) - kmin) << lead;
            if ((r & pmask) == prefix) atomicAdd(&sm->hist[(int)((r >> shift) & 255)], 1);
        }
        __syncthreads();
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
        __syncthreads();
        prefix |= (K)sm->bin << shift;
        pmask |= (K)255 << shift;
        rem = sm->rem;
        __syncthreads();
    }
    thr = (prefix >> lead) + kmin;
    n_gt = k - rem;
}

} // namespace csa
