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
// Each warp finds its m = k-1 best keys by repeated warp argmax: every lane
// keeps the best key of its own candidates below the last winner, and only
// the winning lane rescans.  Long rows are split over the 8 warps of a CTA
// and the 8 partial lists are merged the same way by warp 0.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxK = 64;

// Best key < bound among scores[j] for j = lo + lane + 32 i, j < hi.
__device__ __forceinline__ unsigned long long lane_best(const float *scores, int lo, int hi,
                                                        int lane, unsigned long long bound) {
    unsigned long long best = 0;
    for (int j = lo + lane; j < hi; j += 32) {
        const unsigned long long k = topk_key(__ldg(scores + j), j);
        if (k < bound && k > best) best = k;
    }
    return best;
}

// Best key < bound among list[i], i = lane + 32 q < n.
__device__ __forceinline__ unsigned long long lane_best_list(const unsigned long long *list, int n,
                                                             int lane, unsigned long long bound) {
    unsigned long long best = 0;
    for (int i = lane; i < n; i += 32) {
        const unsigned long long k = list[i];
        if (k < bound && k > best) best = k;
    }
    return best;
}

// The m best keys of this warp's candidates, descending, written to out[0..m)
// (0 where the warp has fewer than m candidates).
template <typename Best>
__device__ __forceinline__ void warp_select(Best best_below, int m, int lane,
                                            unsigned long long *out) {
    unsigned long long mine = best_below(~0ull);
    for (int q = 0; q < m; ++q) {
        const unsigned long long top = warp_max_u64(mine);
        if (lane == 0) out[q] = top;
        if (top == 0) {
            for (int r = q + 1 + lane; r < m; r += 32) out[r] = 0;
            break;
        }
        if (mine == top) mine = best_below(top);   // keys are unique: one lane
        __syncwarp();
    }
    __syncwarp();
}

__device__ __forceinline__ bool seq_valid(int L, long long off, int Sq, int max_kv_len,
                                          long long cap) {
    return L >= Sq && L >= 1 && L <= max_kv_len && off >= 0 && off + L <= cap;
}

// Writes the ascending selection: ids sel[0..n) (unsorted), padded to K.
__device__ __forceinline__ void emit_sorted(const int *sel, int n, const float *scores, int K,
                                            int lane, int32_t *ids_out, float *sc_out) {
    for (int q = lane; q < n; q += 32) {
        const int id = sel[q];
        int rank = 0;
        for (int r = 0; r < n; ++r) rank += sel[r] < id;
        ids_out[rank] = id;
        sc_out[rank] = scores[id];
    }
    for (int q = n + lane; q < K; q += 32) {
        ids_out[q] = -1;
        sc_out[q] = -INFINITY;
    }
}

struct RowInfo {
    bool valid;
    int own;
};

__device__ __forceinline__ RowInfo row_info(const TopkArgs &P, long long row) {
    const int b = static_cast<int>(row / P.Sq);
    const int i = static_cast<int>(row % P.Sq);
    const int L = P.lens[b];
    const long long off = P.kv_offsets[b];
    RowInfo r;
    r.valid = seq_valid(L, off, P.Sq, P.max_kv_len, P.capacity);
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
        warp_select([&](unsigned long long bound) { return lane_best(scores, 0, own, lane, bound); },
                    m, lane, keys[warp]);
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
    warp_select([&](unsigned long long bound) { return lane_best(scores, lo, hi, lane, bound); }, m,
                lane, part + warp * m);
    __syncthreads();
    if (warp == 0) {
        warp_select(
            [&](unsigned long long bound) { return lane_best_list(part, kWarps * m, lane, bound); }, m,
            lane, fin);
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
