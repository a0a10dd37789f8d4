// noalloc.cu -- indexer_topk_static: the indexer scores + top-k entry point for callers that
// cannot allocate device memory.
//
// Some hosts of this library cannot call cudaMalloc when they call us: inference runtimes that
// reserve (nearly) all of the device memory for their own pools at start-up and hand plugins no
// allocator, or C callers embedded in processes whose allocator the library cannot reach.  For
// them the score scratch of indexer_topk lives in a file-scope device array that every GPU
// loading this library holds until the process exits.  The caller still passes every input and
// output; nothing else is allocated here (no cudaMalloc / cudaFree, no allocating library call).
#include <mutex>

#include "common.cuh"

namespace {

// 4 Mi fp32 scores (16 MiB) plus one alignment slot of the workspace carving.
constexpr size_t kStaticScores = size_t(4) << 20;
constexpr size_t kStaticBytes = kStaticScores * sizeof(float) + 256;

static __device__ __align__(256) unsigned char g_topk_scratch[kStaticBytes];

// Device address of g_topk_scratch for the current device, looked up once per device.  In host
// code the symbol name is only a host-side stand-in, never a device address.
void *scratch_for_current_device(cudaError_t *err)
{
    static std::mutex mu;
    static void *addr[64] = {nullptr};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_topk_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

} // namespace

extern "C" {

size_t indexer_topk_static_capacity(void) { return kStaticScores; }

int indexer_topk_static(const void *q, const float *w, const void *keys, int32_t fmt,
                        const int64_t *q_pos, const int64_t *key_off, int64_t n_keys, int64_t Nq,
                        int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis,
                        int32_t *idx_out, float *score_out, void *stream)
{
    if (Nq < 0 || max_nvis < 0) return CSA_ERR_INVALID_ARG;
    if (Nq == 0) // nothing to score: the arguments are still checked, no device is needed
        return indexer_topk(q, w, keys, fmt, q_pos, key_off, n_keys, Nq, H_I, d_I, m, k, max_nvis,
                            idx_out, score_out, nullptr, 0, stream);
    const size_t need = indexer_topk_workspace_size(Nq, max_nvis, k);
    if (need > kStaticBytes) return CSA_ERR_SCRATCH_CAPACITY;
    cudaError_t err = cudaSuccess;
    void *scratch = scratch_for_current_device(&err);
    if (!scratch) return CSA_ERR_CUDA;
    // The scores are written before they are read within one call, so nothing is cleared.
    return indexer_topk(q, w, keys, fmt, q_pos, key_off, n_keys, Nq, H_I, d_I, m, k, max_nvis, idx_out,
                        score_out, scratch, kStaticBytes, stream);
}

} // extern "C"
