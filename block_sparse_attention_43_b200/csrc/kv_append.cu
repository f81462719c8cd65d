// kv_append.cu -- writes the index keys, keys and values of new tokens into
// the caches right after each sequence's current length (packed or paged
// layout), the step before a decode call.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

// One warp per (sequence, new token, tensor): H x 256 contiguous bytes, H =
// H_idx for the index keys, H_kv for the keys and values.
__global__ void kv_append_kernel(const KvAppendArgs P) {
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long total = static_cast<long long>(P.B) * P.n_new * 3;
    if (warp >= total) return;
    const int which = static_cast<int>(warp % 3);
    const long long bt = warp / 3;
    const int b = static_cast<int>(bt / P.n_new), i = static_cast<int>(bt % P.n_new);
    const long long L = P.lens[b];
    const long long t = L + i;                       // position of the new token
    if (L < 0 || t >= P.max_kv_len || !kv_seq_ok(P.kv, b, t + 1)) {
        if (lane == 0 && i == 0 && which == 0) set_status(P.status, kStatusBadLens);
        return;
    }
    const long long row = kv_block_row(P.kv, b, static_cast<int>(t / kBlock), P.status) + t % kBlock;
    const int n16 = (which == 0 ? P.H_idx : P.H_kv) * kDim * 2 / 16;   // 16-byte chunks per token
    const uint4 *src = static_cast<const uint4 *>(P.src[which]) + bt * n16;
    uint4 *dst = static_cast<uint4 *>(P.dst[which]) + row * n16;
    for (int c = lane; c < n16; c += 32) dst[c] = src[c];
}

}  // namespace

cudaError_t launch_kv_append(const KvAppendArgs &a, cudaStream_t s) {
    const long long warps = static_cast<long long>(a.B) * a.n_new * 3;
    const long long blocks = (warps * 32 + 255) / 256;
    TraceScope trace(s, "kv_append");
    kv_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
