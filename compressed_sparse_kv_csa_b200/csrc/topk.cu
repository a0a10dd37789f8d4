// topk.cu -- per-query top-k selection over the indexer scores.
//
// Method: "DeepSeek-V4: Towards Highly Efficient Million-Token Context Intelligence" paper notes,
// Sec. 2.3 Indexer listing: the k_eff = min(k, N_vis) best entries per query.  Ordering
// convention of this library: score descending, equal scores by lower entry index; unused slots
// hold -1.
//
// One CTA per query row.  Radix select over order-preserving 32-bit keys of the fp32 scores
// (8-bit digits over the bits that differ within the row, select.cuh) finds the exact k-th key; entries
// above it are taken unordered, entries equal to it are collected and the lowest-index ones kept
// (a second selection over the tie list), and the k_eff winners are then sorted in shared memory (bitonic, 64-bit keys
// (score key, inverted index)).
#include "common.cuh"
#include "select.cuh"

namespace csa {

namespace {

constexpr int TK_THREADS = 1024;
constexpr int TK_MAX = 2048;
constexpr int64_t TK_STAGE = 32768; // rows of at most this many scores are staged in shared memory

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

// STAGED: the row's scores (nv <= TK_STAGE) are first copied into shared memory as keys, so the
// selection passes read shared memory instead of the score buffer.
template <bool STAGED>
__global__ void __launch_bounds__(TK_THREADS) topk_kernel(IndexerArgs a)
{
    __shared__ unsigned long long sel[TK_MAX];
    __shared__ SelectSmem<uint32_t> ssel;
    __shared__ uint32_t ties[TK_MAX];
    __shared__ int s_cnt, s_eq, s_warp[TK_THREADS / 32], s_eq_taken;
    extern __shared__ uint32_t skeys[]; // STAGED only

    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t nv = tk_nvis(a, r);
    const int k = a.k;
    const int ke = (int)(nv < k ? nv : k);
    const float *S = a.scores + r * a.ld;
    if (STAGED) { // rows are 16-byte aligned and padded to a multiple of 4 scores
        for (int64_t i4 = tid; 4 * i4 < nv; i4 += TK_THREADS) {
            const float4 v = *reinterpret_cast<const float4 *>(S + 4 * i4);
            skeys[4 * i4 + 0] = float_key(v.x);
            skeys[4 * i4 + 1] = float_key(v.y);
            skeys[4 * i4 + 2] = float_key(v.z);
            skeys[4 * i4 + 3] = float_key(v.w);
        }
        __syncthreads();
    }
    auto key = [&](int64_t i) { return STAGED ? skeys[i] : float_key(S[i]); };

    uint32_t thr = 0;   // k-th largest key (only meaningful when nv > k)
    int n_gt = 0;       // number of keys strictly above thr
    if (nv > k) {
        block_kth<TK_THREADS, uint32_t>((int)nv, k, [&](int i) { return key(i); }, &ssel, thr, n_gt);
        const int need = k - n_gt; // entries equal to the threshold that are taken: the lowest indices
        if (tid == 0) { s_cnt = 0; s_eq = 0; s_eq_taken = 0; }
        __syncthreads();
        // strictly greater: unordered append; equal: their indices into the tie list
        for (int64_t s = tid; s < nv; s += TK_THREADS) {
            const uint32_t kv = key(s);
            if (kv > thr) {
                const int pos = atomicAdd(&s_cnt, 1);
                if (pos < n_gt) sel[pos] = ((unsigned long long)kv << 32) | (0xffffffffu - (uint32_t)s);
            } else if (kv == thr) {
                const int e = atomicAdd(&s_eq, 1);
                if (e < TK_MAX) ties[e] = (uint32_t)s;
            }
        }
        __syncthreads();
        const int n_eq = s_eq; // >= need
        const unsigned long long hi = (unsigned long long)thr << 32;
        if (n_eq <= TK_MAX) {
            uint32_t lim = 0; // take the ties whose inverted index is >= lim
            if (n_eq > need) {
                int g;
                block_kth<TK_THREADS, uint32_t>(n_eq, need, [&](int e) { return 0xffffffffu - ties[e]; }, &ssel, lim, g);
            }
            if (tid == 0) s_cnt = 0;
            __syncthreads();
            for (int e = tid; e < n_eq; e += TK_THREADS) {
                const uint32_t inv = 0xffffffffu - ties[e];
                if (inv >= lim) sel[n_gt + atomicAdd(&s_cnt, 1)] = hi | inv;
            }
        } else { // more ties than the list holds: ordered block scan from the lowest index
            for (int64_t base = 0; base < nv; base += TK_THREADS) {
                if (s_eq_taken >= need) break; // uniform: read after a barrier
                const int64_t s = base + tid;
                const bool eq = (s < nv) && (key(s) == thr);
                const unsigned bal = __ballot_sync(0xffffffffu, eq);
                const int lane = tid & 31, wid = tid >> 5;
                if (lane == 0) s_warp[wid] = __popc(bal);
                __syncthreads();
                int before = 0, total = 0;
                for (int w = 0; w < TK_THREADS / 32; ++w) {
                    if (w < wid) before += s_warp[w];
                    total += s_warp[w];
                }
                const int rank = s_eq_taken + before + __popc(bal & ((1u << lane) - 1u));
                if (eq && rank < need) sel[n_gt + rank] = hi | (0xffffffffu - (uint32_t)s);
                __syncthreads();
                if (tid == 0) s_eq_taken += total;
                __syncthreads();
            }
        }
    } else {
        for (int64_t s = tid; s < nv; s += TK_THREADS)
            sel[s] = ((unsigned long long)key(s) << 32) | (0xffffffffu - (uint32_t)s);
    }
    // bitonic sort (descending) of the ke winners, padded with zeros to a power of two
    int n2 = 1;
    while (n2 < ke) n2 <<= 1;
    for (int i = ke + tid; i < n2; i += TK_THREADS) sel[i] = 0ull;
    __syncthreads();
    for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < n2; i += TK_THREADS) {
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
