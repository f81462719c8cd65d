// topk.cu -- MSA top-k block selection per (query row, group).
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二: "Block Max Pool" then "Top-k" selection of
// the KV blocks; k = sparse_topk_blocks = 16 in the mlqm.cn MiniMax-M3 guide's
// configuration passage.  Readings fixed by this library: the query's own
// block is always kept; the other k-1 slots go to the best blocks j < own
// ranked by (score desc, id asc); with at most k visible blocks all are kept.
//
// Selection runs on 64-bit keys (order-preserving score bits, complemented
// id) so the order is total and the result is independent of the algorithm.
// Each warp finds its m = k-1 best keys by repeated warp argmax over per-lane
// register caches; long rows are split over the 8 warps of a CTA and the 8
// partial lists are merged the same way by warp 0.  Prefill rows select
// inside the tensor-core index kernel; this kernel serves decode.
#include "msa_device.cuh"
#include "msa_internal.h"
#include "topk_warp.cuh"

namespace msa {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ bool seq_valid(const TopkArgs &P, int b, int L) {
    return L >= P.Sq && L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
}

struct RowInfo {
    bool valid;
    int own;
};

__device__ __forceinline__ RowInfo row_info(const TopkArgs &P, long long row) {
    const int b = static_cast<int>(row / P.Sq);
    const int i = static_cast<int>(row % P.Sq);
    const int L = P.lens[b];
    RowInfo r;
    r.valid = seq_valid(P, b, L);
    r.own = r.valid ? (L - P.Sq + i) / kBlock : 0;
    return r;
}

// One warp per (row, group): rows with at most a few hundred candidates.
__global__ void __launch_bounds__(kWarps * 32) topk_warp_kernel(const TopkArgs P) {
    __shared__ unsigned long long keys[kWarps][kMaxK];
    __shared__ int sel[kWarps][kMaxK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long pair = static_cast<long long>(blockIdx.x) * kWarps + warp;
    const long long npairs = static_cast<long long>(P.B) * P.Sq * P.H_kv;
    if (pair >= npairs) return;
    const long long row = pair / P.H_kv;
    const int K = P.K;
    int32_t *ids_out = P.ids + pair * K;
    float *sc_out = P.out_scores + pair * K;
    const RowInfo ri = row_info(P, row);
    if (!ri.valid) {
        if (lane == 0 && (row % P.Sq) == 0) set_status(P.status, kStatusBadLens);
        for (int q = lane; q < K; q += 32) { ids_out[q] = -1; sc_out[q] = -INFINITY; }
        return;
    }
    const float *scores = P.scores + pair * P.nb_max;
    const int own = ri.own;
    int n = 0;
    if (own + 1 <= K) {
        for (int q = lane; q <= own; q += 32) sel[warp][q] = q;
        n = own + 1;
    } else {
        const int m = K - 1;
        warp_select([&](int j) { return topk_key(__ldg(scores + j), j); }, 0, own, m, lane,
                    keys[warp]);
        for (int q = lane; q < m; q += 32) sel[warp][q] = topk_key_id(keys[warp][q]);
        if (lane == 0) sel[warp][m] = own;
        n = K;
    }
    __syncwarp();
    emit_sorted(sel[warp], n, scores, K, lane, ids_out, sc_out);
}

// One CTA per (row, group): long rows (decode over long contexts).
__global__ void __launch_bounds__(kWarps * 32) topk_cta_kernel(const TopkArgs P) {
    __shared__ unsigned long long part[kWarps * kMaxK];
    __shared__ unsigned long long fin[kMaxK];
    __shared__ int sel[kMaxK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long pair = blockIdx.x;
    const long long row = pair / P.H_kv;
    const int K = P.K;
    int32_t *ids_out = P.ids + pair * K;
    float *sc_out = P.out_scores + pair * K;
    const RowInfo ri = row_info(P, row);
    if (!ri.valid) {
        if (warp == 0) {
            if (lane == 0 && (row % P.Sq) == 0) set_status(P.status, kStatusBadLens);
            for (int q = lane; q < K; q += 32) { ids_out[q] = -1; sc_out[q] = -INFINITY; }
        }
        return;
    }
    const float *scores = P.scores + pair * P.nb_max;
    const int own = ri.own;
    if (own + 1 <= K) {
        if (warp == 0) {
            for (int q = lane; q <= own; q += 32) sel[q] = q;
            __syncwarp();
            emit_sorted(sel, own + 1, scores, K, lane, ids_out, sc_out);
        }
        return;
    }
    const int m = K - 1;
    const int chunk = (own + kWarps - 1) / kWarps;
    const int lo = min(own, warp * chunk), hi = min(own, lo + chunk);
    warp_select([&](int j) { return topk_key(__ldg(scores + j), j); }, lo, hi, m, lane,
                part + warp * m);
    __syncthreads();
    if (warp == 0) {
        warp_select([&](int i) { return part[i]; }, 0, kWarps * m, m, lane, fin);
        for (int q = lane; q < m; q += 32) sel[q] = topk_key_id(fin[q]);
        if (lane == 0) sel[m] = own;
        __syncwarp();
        emit_sorted(sel, K, scores, K, lane, ids_out, sc_out);
    }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t s) {
    if (a.K < 1 || a.K > kMaxK) return cudaErrorInvalidValue;
    const long long npairs = static_cast<long long>(a.B) * a.Sq * a.H_kv;
    if (npairs <= 0) return cudaSuccess;
    TraceScope trace(s, "topk_select");
    // Few long rows: a CTA per row.  Many rows: a warp per row.
    if (a.nb_max > 512 && npairs < 4LL * 148 * kWarps) {
        topk_cta_kernel<<<static_cast<unsigned>(npairs), kWarps * 32, 0, s>>>(a);
    } else {
        const long long grid = (npairs + kWarps - 1) / kWarps;
        topk_warp_kernel<<<static_cast<unsigned>(grid), kWarps * 32, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace msa
