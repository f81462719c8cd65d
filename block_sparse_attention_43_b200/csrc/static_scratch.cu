// static_scratch.cu -- msa_index_topk_static: the index branch with its
// block-score scratch in a fixed device array instead of a caller workspace.
//
// Some callers cannot hand the library a workspace: plugin hosts that give a
// kernel only its input and output buffers, processes whose device memory is
// entirely owned by another allocator, and latency-critical loops where a
// cudaMalloc would stall on an implicit device synchronisation.  For them the
// scratch lives in g_scratch below, a file-scope __device__ array that every
// GPU loading this library keeps for the life of the process.
#include <mutex>

#include "msa.h"
#include "msa_internal.h"

namespace {

// 256-byte header (device status word) + 4 MiB of block scores: enough for a
// decode batch with batch * index heads * ceil(max_kv_len / 128) <= 1,048,576
// (e.g. 4 sequences x 8 groups at 1M tokens, or 64 x 8 at 256k).  Prefill
// rows with bf16 keys use only the header.  The address of the array is
// looked up once per device and kept, so a primary-context reset between
// calls is not supported.
constexpr size_t kStaticScratchBytes = 256 + (size_t(4) << 20);

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_ptr[kMaxDevices];   // device address of g_scratch, per device

// Looks up g_scratch's device address on the current device once.  In host
// code the name g_scratch is only a host-side stand-in, never a device address.
msa_status_t scratch_ptr(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MSA_ERR_CUDA;
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
    return MSA_OK;
}

}  // namespace

extern "C" msa_status_t msa_index_topk_static(const msa_shape_t *shape, const void *q_idx,
                                              const void *k_idx, const int32_t *lens,
                                              const int64_t *kv_offsets, int32_t *block_ids,
                                              float *block_scores, msa_stream_t stream) {
    const size_t need = msa_index_topk_workspace_size(shape);
    if (need == 0 || (shape->index_key_format != MSA_INDEX_KEYS_BF16 &&
                      shape->index_key_format != MSA_INDEX_KEYS_BF16_SHARED))
        // rejected shape or key format: msa_index_topk reports which error, nothing is launched
        return msa_index_topk(shape, q_idx, k_idx, lens, kv_offsets, block_ids, block_scores,
                              nullptr, 0, stream);
    if (need > kStaticScratchBytes) return MSA_ERR_WORKSPACE;   // shape too large for g_scratch
    void *ws = nullptr;
    const msa_status_t st = scratch_ptr(&ws);
    if (st != MSA_OK) return st;
    // msa_index_topk clears the header and writes every score it later reads.
    return msa_index_topk(shape, q_idx, k_idx, lens, kv_offsets, block_ids, block_scores, ws,
                          kStaticScratchBytes, stream);
}
