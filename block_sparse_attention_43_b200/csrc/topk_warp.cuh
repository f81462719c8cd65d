// topk_warp.cuh -- warp-level top-m selection on 64-bit keys (order-preserving
// score bits with the complemented block id, so the order is total and the
// selected set does not depend on the algorithm), shared by the top-k kernels
// and the fused decode kernel.
#pragma once
#include "msa_device.cuh"

namespace msa {

constexpr int kMaxK = 64;

// Keys are read once: every lane streams its candidates j = lo + lane + 32 i
// (coalesced) and keeps its own best kCache keys in registers.  The warp then
// takes its m best by repeated warp argmax over the lanes' heads; the winner
// pops its head and, in the rare case its cache runs dry while it still has
// candidates, rescans them below the last key it gave up.
constexpr int kCache = 4;

struct LaneTop {
    unsigned long long k[kCache];
    int popped;      // keys taken from this lane so far
};

template <typename Key>
__device__ __forceinline__ void lane_fill(LaneTop &t, Key key_at, int lo, int hi, int lane,
                                          unsigned long long bound) {
#pragma unroll
    for (int i = 0; i < kCache; ++i) t.k[i] = 0;
    // Eight independent loads in flight per round, then eight inserts.
    for (int base = lo + lane; base < hi; base += 32 * 8) {
        unsigned long long xs[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = base + 32 * u;
            xs[u] = j < hi ? key_at(j) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            unsigned long long x = xs[u];
            if (x >= bound || x <= t.k[kCache - 1]) continue;
#pragma unroll
            for (int i = 0; i < kCache; ++i) {
                const unsigned long long hi_k = t.k[i] > x ? t.k[i] : x;
                x = t.k[i] > x ? x : t.k[i];
                t.k[i] = hi_k;
            }
        }
    }
}

// The m best keys of the warp's candidates [lo, hi), descending, into out[0..m)
// (0 where there are fewer than m candidates).
template <typename Key>
__device__ __forceinline__ void warp_select(Key key_at, int lo, int hi, int m, int lane,
                                            unsigned long long *out) {
    LaneTop t;
    lane_fill(t, key_at, lo, hi, lane, ~0ull);
    const int mine_total = hi - lo > lane ? (hi - lo - lane + 31) / 32 : 0;
    int have = mine_total < kCache ? mine_total : kCache;   // cached keys not yet popped
    t.popped = 0;
    for (int q = 0; q < m; ++q) {
        const unsigned long long head = t.k[0];
        const unsigned long long top = warp_max_u64(head);
        if (lane == 0) out[q] = top;
        if (top == 0) {
            for (int r = q + 1 + lane; r < m; r += 32) out[r] = 0;
            break;
        }
        if (head == top) {                      // keys are unique: exactly one lane
#pragma unroll
            for (int i = 0; i < kCache - 1; ++i) t.k[i] = t.k[i + 1];
            t.k[kCache - 1] = 0;
            ++t.popped;
            --have;
            if (have == 0 && t.popped < mine_total) {
                lane_fill(t, key_at, lo, hi, lane, top);
                have = min(kCache, mine_total - t.popped);
            }
        }
        __syncwarp();
    }
    __syncwarp();
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

}  // namespace msa
