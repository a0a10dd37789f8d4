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

// 16 MiB of scratch plus one alignment slot of the workspace carving.
constexpr size_t kStaticBytes = (size_t(16) << 20) + 256;

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

size_t indexer_topk_static_capacity(void) { return kStaticBytes; }

int indexer_topk_static(const void *q, const float *w, const void *keys, int32_t fmt,
                        const int64_t *q_pos, const int64_t *key_off, int64_t n_keys, int64_t Nq,
                        int32_t H_I, int32_t d_I, int32_t m, int32_t k, int64_t max_nvis,
                        int32_t *idx_out, float *score_out, void *stream)
{
    // The same checks and kernels as indexer_topk; the request is refused when the scratch of the
    // path it takes does not fit in the static array.  Every score is written before it is read
    // within one call, so nothing needs clearing between calls.
    return csa::indexer_topk_impl(q, w, keys, fmt, q_pos, key_off, n_keys, Nq, H_I, d_I, m, k, max_nvis, idx_out,
                                  score_out, nullptr, kStaticBytes, scratch_for_current_device, stream);
}

} // extern "C"
