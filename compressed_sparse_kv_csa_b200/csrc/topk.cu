// topk.cu -- per-query top-k selection over the indexer scores.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 Indexer listing: the k_eff = min(k, N_vis) best entries per query.  Ordering
// convention of this library: score descending, equal scores by lower entry index; unused slots
// hold -1.
//
// One CTA of 512 threads per query row; rows of at most TK_STAGE scores are staged in shared
// memory as order-preserving 32-bit keys.  Every entry has the unique 64-bit key
// (score key << 32 | ~index), so "the k largest keys" is exactly the wanted set.  Three passes
// over the row: (1) the range of the score keys (taken while staging); (2) a histogram of the top
// 11 bits of the keys offset by the minimum and left-aligned on the range (2,048 bins, shared-memory
// atomics), whose suffix sums give the bin b* that holds the k-th key; (3) keys in bins above b* are winners,
// keys in b* are candidates (warp-aggregated appends).  The few candidates are resolved by an
// exact 64-bit selection, and the k winners are sorted in shared memory (bitonic; the steps
// between elements less than 32 apart by warp shuffles).
#include "common.cuh"
#include "select.cuh"

namespace csa {

namespace {

constexpr int TK_THREADS = 512;
constexpr int TK_MAX = 2048;     // largest k
constexpr int TK_BINS = 2048;    // 11-bit first digit
constexpr int TK_CAND = 2048;    // candidates of the crossing bin kept in shared memory
constexpr int64_t TK_STAGE = 16384; // rows of at most this many scores are staged in shared memory

__device__ __forceinline__ int64_t tk_nvis(const IndexerArgs &a, int64_t r)
{
    const int64_t t = a.q_pos ? a.q_pos[r] : r;
    int64_t nv = (t + 1) / a.m;
    if (nv > a.max_nvis) nv = a.max_nvis;
    const int64_t base = a.key_off ? a.key_off[r] : 0;
    if (base < 0) return 0;
    if (nv > a.n_keys - base) nv = a.n_keys - base;
    return nv < 0 ? 0 : nv;
}

__device__ __forceinline__ unsigned long long key64(uint32_t k, int64_t i)
{
    return ((unsigned long long)k << 32) | (unsigned long long)(0xffffffffu - (uint32_t)i);
}

// Warp-aggregated append of the lanes with `take` to list[*count ...]; returns nothing.
__device__ __forceinline__ void warp_append(bool take, unsigned long long v, unsigned long long *list, int *count,
                                            int cap)
{
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (!m) return;
    const int lane = threadIdx.x & 31;
    int base = 0;
    if (lane == __ffs(m) - 1) base = atomicAdd(count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, __ffs(m) - 1);
    const int p = base + __popc(m & ((1u << lane) - 1u));
    if (take && p < cap) list[p] = v;
}

template <bool STAGED>
__global__ void __launch_bounds__(TK_THREADS) topk_kernel(IndexerArgs a)
{
    __shared__ unsigned long long sel[TK_MAX];
    __shared__ unsigned long long cand[TK_CAND];
    __shared__ int hist[TK_BINS];
    __shared__ SelectSmem<uint32_t> ssel;
    __shared__ uint32_t s_lo[TK_THREADS / 32], s_hi[TK_THREADS / 32];
    __shared__ int s_bin, s_above, s_nsel, s_ncand;
    extern __shared__ uint32_t skeys[]; // STAGED only

    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t nv = tk_nvis(a, r);
    const int k = a.k;
    const int ke = (int)(nv < k ? nv : k);
    const float *S = a.scores + r * a.ld;
    uint32_t lo = 0xffffffffu, hi = 0; // range of this thread's keys (the staging pass takes it)
    if (STAGED) { // rows are 16-byte aligned and padded to a multiple of 4 scores
        for (int64_t i4 = tid; 4 * i4 < nv; i4 += TK_THREADS) {
            const float4 v = *reinterpret_cast<const float4 *>(S + 4 * i4);
            const uint32_t k4[4] = {float_key(v.x), float_key(v.y), float_key(v.z), float_key(v.w)};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                skeys[4 * i4 + u] = k4[u];
                if (4 * i4 + u < nv) {
                    lo = k4[u] < lo ? k4[u] : lo;
                    hi = k4[u] > hi ? k4[u] : hi;
                }
            }
        }
    }
    if (tid == 0) {
        s_nsel = 0;
        s_ncand = 0;
    }
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    auto key = [&](int64_t i) -> uint32_t { return STAGED ? skeys[i] : float_key(S[i]); };

    if (nv <= k) { // every visible entry is a winner
        for (int64_t i = tid; i < nv; i += TK_THREADS) sel[i] = key64(key(i), i);
    } else {
        // 1. range of the score keys (already taken by the staging pass)
        if (!STAGED) {
            for (int64_t i = tid; i < nv; i += TK_THREADS) {
                const uint32_t v = key(i);
                lo = v < lo ? v : lo;
                hi = v > hi ? v : hi;
            }
        }
        lo = warp_min_key(lo);
        hi = warp_max_key(hi);
        if (lane == 0) {
            s_lo[wid] = lo;
            s_hi[wid] = hi;
        }
        __syncthreads();
        lo = s_lo[0];
        hi = s_hi[0];
        for (int w = 1; w < TK_THREADS / 32; ++w) {
            lo = s_lo[w] < lo ? s_lo[w] : lo;
            hi = s_hi[w] > hi ? s_hi[w] : hi;
        }
        const int lead = (hi == lo) ? 32 : __clz(hi - lo);
        auto bin_of = [&](uint32_t v) -> int { return lead >= 32 ? 0 : (int)(((v - lo) << lead) >> 21); };
        // 2. histogram of the 11-bit first digit (shared-memory atomics; the range-normalised bins
        //    spread a warp's keys, so lanes rarely collide)
        for (int64_t i = tid; i < nv; i += TK_THREADS) atomicAdd(&hist[bin_of(key(i))], 1);
        __syncthreads();
        if (wid == 0) { // suffix scan from the top bin: lane l owns bins 2047-64l .. 1984-64l
            int sum = 0;
            for (int j = 0; j < 64; ++j) sum += hist[TK_BINS - 1 - 64 * lane - j];
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = incl - sum;
            const bool cross = excl < k && incl >= k;
            const unsigned who = __ballot_sync(0xffffffffu, cross);
            if (cross && lane == __ffs(who) - 1) {
                int cum = excl, j = 0;
                for (; j < 63; ++j) {
                    const int c = hist[TK_BINS - 1 - 64 * lane - j];
                    if (cum + c >= k) break;
                    cum += c;
                }
                s_bin = TK_BINS - 1 - 64 * lane - j;
                s_above = cum; // keys in the bins above b*
            }
        }
        __syncthreads();
        const int bstar = s_bin, n_above = s_above, need = k - n_above;
        // 3. winners above b*, candidates in b*
        for (int64_t base = 0; base < nv; base += TK_THREADS) {
            const int64_t i = base + tid;
            const bool in = i < nv;
            const uint32_t v = in ? key(i) : 0u;
            const int b = in ? bin_of(v) : -1;
            warp_append(in && b > bstar, key64(v, i), sel, &s_nsel, TK_MAX);
            warp_append(in && b == bstar, key64(v, i), cand, &s_ncand, TK_CAND);
        }
        __syncthreads();
        const int n_cand = s_ncand; // >= need
        // 4. the `need` largest candidates join the winners
        if (n_cand <= TK_CAND) {
            const unsigned long long thr =
                n_cand > need ? block_kth64<TK_THREADS>(n_cand, need, [&](int j) { return cand[j]; }, &ssel) : 0ull;
            for (int j = tid; j < n_cand; j += TK_THREADS) {
                const unsigned long long v = cand[j];
                if (v >= thr) sel[atomicAdd(&s_nsel, 1)] = v; // s_nsel starts at n_above here
            }
        } else { // more candidates than shared memory holds (many equal scores): select over the row
            auto get = [&](int j) -> unsigned long long {
                const uint32_t v = key(j);
                return bin_of(v) == bstar ? key64(v, j) : 0ull;
            };
            const unsigned long long thr = block_kth64<TK_THREADS>((int)nv, need, get, &ssel);
            for (int64_t base = 0; base < nv; base += TK_THREADS) {
                const int64_t i = base + tid;
                const unsigned long long v = i < nv ? get((int)i) : 0ull;
                warp_append(v != 0ull && v >= thr, v, sel, &s_nsel, TK_MAX);
            }
        }
    }
    __syncthreads();
    // bitonic sort (descending) of the ke winners, padded with zeros to a power of two
    int n2 = 1;
    while (n2 < ke) n2 <<= 1;
    for (int i = ke + tid; i < n2; i += TK_THREADS) sel[i] = 0ull;
    __syncthreads();
    block_sort_desc64<TK_THREADS>(sel, n2);
    for (int j = tid; j < k; j += TK_THREADS) {
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

cudaError_t launch_topk(const IndexerArgs &a, cudaStream_t st)
{
    if (a.Nq == 0) return cudaSuccess;
    if (a.max_nvis <= TK_STAGE) {
        const size_t smem = (size_t)((a.max_nvis + 3) / 4 * 4) * sizeof(uint32_t);
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        topk_kernel<true><<<(unsigned)a.Nq, TK_THREADS, smem, st>>>(a);
    } else {
        topk_kernel<false><<<(unsigned)a.Nq, TK_THREADS, 0, st>>>(a);
    }
    return cudaGetLastError();
}

} // namespace csa

// ------------------------------------------------------------------------------------------
// merge of candidate lists (the last step of a top-k whose keys were scored in shards)
// ------------------------------------------------------------------------------------------
namespace csa {

namespace {

constexpr int TM_THREADS = 512;

// One CTA per query: the exact top-k of its n_lists x list_len (score, index) candidates, stored
// list-major ([n_lists, Nq, list_len]); list l's indices are offset by bases[l]; index < 0 is
// ignored.  Ordered by score descending then index ascending.  Candidate keys are staged in
// shared memory as 64-bit (score key << 32 | ~index) keys, unique when the indices are.
__global__ void __launch_bounds__(TM_THREADS) topk_merge_lists_kernel(const float *scores, const int32_t *idx,
                                                                     const int64_t *bases, int64_t Nq, int n_lists,
                                                                     int list_len, int k, int32_t *idx_out,
                                                                     float *score_out)
{
    const int n_cand = n_lists * list_len;
    extern __shared__ unsigned long long mk[];
    __shared__ SelectSmem<uint32_t> msel;
    __shared__ int s_n, s_w;
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_n = 0;
        s_w = 0;
    }
    __syncthreads();
    for (int j0 = 0; j0 < n_cand; j0 += TM_THREADS) {
        const int j = j0 + tid;
        const int l = j / list_len;
        const int64_t at = ((int64_t)l * Nq + r) * list_len + (j - l * list_len);
        const int32_t id = j < n_cand ? idx[at] : -1;
        const bool in = id >= 0;
        const unsigned long long v = in ? key64(float_key(scores[at]), (int64_t)id + (bases ? bases[l] : 0)) : 0ull;
        warp_append(in, v, mk, &s_n, n_cand);
    }
    __syncthreads();
    const int n = s_n;
    const int ke = n < k ? n : k;
    unsigned long long *sel = mk + n_cand;
    const unsigned long long thr = n > k ? block_kth64<TM_THREADS>(n, k, [&](int i) { return mk[i]; }, &msel) : 0ull;
    for (int i = tid; i < n; i += TM_THREADS) {
        const unsigned long long v = mk[i];
        if (v >= thr) {
            const int p = atomicAdd(&s_w, 1);
            if (p < ke) sel[p] = v;
        }
    }
    __syncthreads();
    int n2 = 1;
    while (n2 < ke) n2 <<= 1;
    for (int i = ke + tid; i < n2; i += TM_THREADS) sel[i] = 0ull;
    __syncthreads();
    block_sort_desc64<TM_THREADS>(sel, n2);
    for (int j = tid; j < k; j += TM_THREADS) {
        int32_t id = -1;
        float sc = -INFINITY;
        if (j < ke) {
            const unsigned long long v = sel[j];
            id = (int32_t)(0xffffffffu - (uint32_t)(v & 0xffffffffu));
            sc = key_float((uint32_t)(v >> 32));
        }
        idx_out[r * k + j] = id;
        if (score_out) score_out[r * k + j] = sc;
    }
}

} // namespace

cudaError_t launch_topk_merge_lists(const float *scores, const int32_t *idx, const int64_t *bases, int64_t Nq,
                                    int n_lists, int list_len, int k, int32_t *idx_out, float *score_out,
                                    cudaStream_t st)
{
    if (Nq == 0) return cudaSuccess;
    int n2 = 1;
    while (n2 < k) n2 <<= 1;
    const size_t smem = ((size_t)n_lists * list_len + (size_t)n2) * 8;
    cudaError_t e = cudaFuncSetAttribute(topk_merge_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_merge_lists_kernel<<<(unsigned)Nq, TM_THREADS, smem, st>>>(scores, idx, bases, Nq, n_lists, list_len, k,
                                                                    idx_out, score_out);
    return cudaGetLastError();
}

} // namespace csa
