// decode_fused.cu -- the whole MSA decode step in one persistent launch:
// index scores + block max-pool, top-k per (sequence, group), and sparse
// attention over the kept blocks.
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 (index branch, Block Max Pool, top-k; exact
// attention over the kept blocks) and section 六 (the group's heads share its
// blocks); the step's cost is the index keys streamed from HBM (section 四).
//
// Why one launch: with separate kernels, top-k and attention of every
// sequence wait for the index scores of all sequences.  Here they overlap the
// index streaming of the later sequences:
//   - CTAs (one per SM, cooperative launch so all are resident) claim index
//     units (one 128-token block of one sequence, all groups) from a global
//     counter in sequence order, so sequences finish one after another;
//   - per unit the consumer warps hand the 16 row-slot maxima to a
//     bookkeeper warp, which stores the block scores and counts them with a
//     device-scope atomic, so no consumer ever waits on a global round trip;
//     the bookkeeper that counts a sequence's last score has the producer
//     queue that sequence's top-k (one consumer warp per group, the warp
//     selection of topk.cu), which publishes one attention item per group;
//   - between index units a CTA takes published attention items, one per
//     (sequence, group): the K/V tiles of its kept blocks (TMA, 128-byte
//     swizzle) stream through the same ring, S^T = K Q^T and O^T = V^T P^T
//     run on mma.sync for the group's heads (one n8 tile per 8 heads, groups
//     of up to 16) with a running softmax across the blocks, and the CTA
//     writes the group's output itself (no partial records, no merge across
//     CTAs).
// An attention item is claimed (one atomicAdd) only while the claim counter
// is below the published count; a claim that overtakes its publisher stays
// pending while the CTA streams more index units.  Once a CTA has no index
// unit left it waits for its claimed item, which the CTA whose bookkeeper
// counts that sequence's last score publishes; while it waits, its producer
// keeps queueing its own CTA's top-k requests, and it ends only after its
// bookkeeper has finished every unit it handed out, so no request is left
// behind.  Every wait is bounded.
#include <type_traits>

#include "msa_device.cuh"
#include "msa_internal.h"
#include "topk_warp.cuh"

namespace msa {
namespace {

constexpr int kWarps = 8;                     // consumer warps
constexpr int kConsumers = kWarps * 32;
constexpr int kProducerWarp = kWarps, kBookWarp = kWarps + 1;
constexpr int kThreads = kConsumers + 64;     // + producer warp + bookkeeper warp
constexpr int kRedQ = 4;                      // index units whose row maxima await the bookkeeper
constexpr int kFifo = 16;                     // top-k requests from the bookkeeper to the producer
constexpr int kStages = 5;
constexpr int kStageBytes = 32768;
constexpr int kQueue = 4;
constexpr int kMaxBatch = 4096;
constexpr float kLog2e = 1.4426950408889634f;

enum { kWorkIndex = 0, kWorkAttn = 1, kWorkTopk = 2, kWorkEnd = 3 };

struct Smem {
    uint8_t ring[kStages][kStageBytes];       // index-key stages / K and V tiles of a block
    float om[kWarps][8][kDim];                // attention: per-warp O^T; top-k scratch
    float mw[kWarps][8], lw[kWarps][8];
    uint64_t full[kStages], empty[kStages];
    uint64_t wq_full[kQueue], wq_empty[kQueue];
    uint64_t cbar;                            // consumer-wide sync (all 256 threads arrive)
    int4 wq[kQueue];                          // {kind, a, b, c}
    uint64_t red_full[kRedQ], red_empty[kRedQ];
    int prefix[kMaxBatch + 1];
    float red[kRedQ][16];                     // per index unit: max of each row slot
    int red_b[kRedQ], red_j[kRedQ];           // its (sequence, block); sequence -1 ends the stream
    int topk_fifo[kFifo];
    int topk_wr, topk_rd;
    int book_done;                            // index units the bookkeeper has finished
    int bcast[2];
    int total_attn;
    int abort_flag;
};

__device__ __forceinline__ bool seq_valid(const DecodeFusedArgs &P, int b, int L) {
    return L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
}

__device__ __forceinline__ int ld_volatile(const int *p) { return *reinterpret_cast<const volatile int *>(p); }

// Device-scope add that publishes this thread's earlier writes and, for the
// thread that sees the final count, acquires everyone else's.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Score rows padded to 32 floats: rows of different (sequence, group) never
// share a cache line, so no SM can hold a stale copy of a row it reads.
__host__ __device__ __forceinline__ int score_stride(int nb_max) { return (nb_max + 31) & ~31; }

// Largest b with prefix[b] <= u.
__device__ __forceinline__ void unit_of(const int *prefix, int B, int u, int &b, int &j) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= u) lo = mid; else hi = mid;
    }
    b = lo;
    j = u - prefix[lo];
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const DecodeFusedArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // H groups (attention items); HI index heads (scores, top-k), group g
    // reading index head g / (H / HI)
    const int H = P.H_kv, HI = P.n_idx, G = P.H_q / P.H_kv, K = P.K;
    const int nbs = score_stride(P.nb_max);
    volatile int *abort_flag = &S.abort_flag;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], kWarps);
        }
        for (int i = 0; i < kQueue; ++i) {
            mbar_init(&S.wq_full[i], 1);
            mbar_init(&S.wq_empty[i], kWarps);
        }
        mbar_init(&S.cbar, kConsumers);
        for (int i = 0; i < kRedQ; ++i) {
            mbar_init(&S.red_full[i], kWarps);
            mbar_init(&S.red_empty[i], 1);
        }
        S.topk_wr = S.topk_rd = S.book_done = 0;
        S.abort_flag = 0;
        fence_mbar_init();
    }
    // Units per sequence (exclusive prefix) and the number of attention items.
    if (warp == 0) {
        const int per = (P.B + 31) / 32;
        const int lo = lane * per, hi = min(P.B, lo + per);
        int sum = 0, items = 0;
        for (int b = lo; b < hi; ++b) {
            const int L = P.lens[b];
            if (seq_valid(P, b, L)) {
                const int nb = (L + kBlock - 1) / kBlock;
                sum += nb;
                items += H;
            } else if (blockIdx.x == 0) {
                // rejected sequence: -1 / -inf selection, NaN output, status word
                set_status(P.status, kStatusBadLens);
                for (int q = 0; q < HI * K; ++q) {
                    P.ids[static_cast<long long>(b) * HI * K + q] = -1;
                    P.out_scores[static_cast<long long>(b) * HI * K + q] = -INFINITY;
                }
                __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(P.out) + static_cast<long long>(b) * P.H_q * kDim;
                for (int e = 0; e < P.H_q * kDim; ++e) o[e] = __float2bfloat16(NAN);
            }
        }
        int incl = sum;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, m);
            if (lane >= m) incl += o;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) items += __shfl_xor_sync(0xffffffffu, items, m);
        int run = incl - sum;
        for (int b = lo; b < hi; ++b) {
            S.prefix[b] = run;
            const int L = P.lens[b];
            if (seq_valid(P, b, L)) run += (L + kBlock - 1) / kBlock;
        }
        if (lane == 31) S.prefix[P.B] = incl;
        if (lane == 0) S.total_attn = items;
    }
    __syncthreads();
    const int U = S.prefix[P.B];
    const int total_attn = S.total_attn;

    if (warp == kBookWarp) {
        // ------------------------------------------------ bookkeeper: block
        // scores and sequence completion, off the consumers' path.  Per index
        // unit: the max of the group's row slots is the block score (one lane
        // per group), stored and counted with a device-scope atomic; the lane
        // that counts a sequence's last score asks the producer (through a
        // shared-memory FIFO) to queue that sequence's top-k.
        const unsigned long long lim = wait_limit_ns(P.status);
        for (int k = 0;; ++k) {
            const int slot = k % kRedQ;
            bool have = !*abort_flag && mbar_wait(&S.red_full[slot], (k / kRedQ) & 1, P.status);
            have = __all_sync(0xffffffffu, have);
            if (!have) { *abort_flag = 1; break; }
            const int b = S.red_b[slot], j = S.red_j[slot];
            float m = -INFINITY;
            if (lane < HI)
                for (int r = lane; r < 16; r += HI) m = fmaxf(m, S.red[slot][r]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.red_empty[slot]);
            if (b < 0) break;                       // the consumers are done
            bool last = false;
            if (lane < HI) {
                P.scores[((long long)b * HI + lane) * nbs + j] = m;
                const int target = HI * ((P.lens[b] + kBlock - 1) / kBlock);
                last = atom_add_acq_rel_gpu(P.seq_done + b, 1) + 1 == target;
            }
            if (__any_sync(0xffffffffu, last) && lane == 0) {
                // at most kRedQ + kQueue units finish between two producer
                // polls, so the FIFO does not fill; the wait is a safety net
                const unsigned long long t0 = now_ns();
                while (S.topk_wr - ld_volatile(&S.topk_rd) >= kFifo) {
                    if (*abort_flag || now_ns() - t0 > lim) { set_status(P.status, kStatusTimeout); *abort_flag = 1; break; }
                    __nanosleep(64);
                }
                S.topk_fifo[S.topk_wr % kFifo] = b;
                __threadfence_block();
                *reinterpret_cast<volatile int *>(&S.topk_wr) = S.topk_wr + 1;
            }
            if (lane == 0) {
                __threadfence_block();              // the FIFO entry above comes first
                *reinterpret_cast<volatile int *>(&S.book_done) = k + 1;
            }
            __syncwarp();
        }
        return;
    }

    if (warp == kProducerWarp) {
        // ------------------------------------------------ producer: claims work,
        // publishes it to the consumers and issues its loads
        if (lane != 0) return;
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        const uint64_t pol = l2_policy_evict_first();
        const __nv_bfloat16 *kbase = static_cast<const __nv_bfloat16 *>(P.k_idx);
        const int tps = 128 / HI;                // tokens per index stage
        int n = 0, it = 0;                        // work entries pushed, stages issued
        bool index_left = true, ok = true;
        auto push = [&](int4 w) -> bool {
            const int slot = n % kQueue;
            if (n >= kQueue && (*abort_flag || !mbar_wait(&S.wq_empty[slot], ((n / kQueue) - 1) & 1, P.status)))
                return false;
            S.wq[slot] = w;
            mbar_arrive(&S.wq_full[slot]);
            ++n;
            return true;
        };
        auto stage = [&](int &slot) -> bool {
            slot = it % kStages;
            if (it >= kStages && (*abort_flag || !mbar_wait(&S.empty[slot], ((it / kStages) - 1) & 1, P.status)))
                return false;
            ++it;
            return true;
        };
        // Work claiming.  Attention items are claimed with one atomicAdd
        // (never a compare-and-swap loop, which a hundred polling CTAs turn
        // into a serial storm), and only while the claim counter is below the
        // published count; a claim may still overtake the publisher that
        // owns the item, so the item stays pending (this CTA goes on
        // streaming index units) until its flag is set.  The next index unit
        // and the counters are fetched one unit ahead, so their latency hides
        // behind the unit in flight.
        int *const c_unit = P.ctr, *const c_claim = P.ctr + 2 * kCtrStride;
        int *const c_pub = P.ctr + 3 * kCtrStride;
        int pending = -1, pending_flag = 0;
        bool attn_left = total_attn > 0;
        int u_next = atomicAdd(c_unit, 1);
        int seen_claim = 0, seen_pub = 0, units_pushed = 0;
        // queues the top-k of every sequence the bookkeeper has completed
        auto drain_topk = [&]() -> bool {
            while (S.topk_rd != ld_volatile(&S.topk_wr)) {
                __threadfence_block();
                const int b = S.topk_fifo[S.topk_rd % kFifo];
                if (!push(make_int4(kWorkTopk, b, 0, 0))) return false;
                *reinterpret_cast<volatile int *>(&S.topk_rd) = S.topk_rd + 1;
            }
            return true;
        };
        const unsigned long long lim = wait_limit_ns(P.status);
        // A test may make this CTA's first item wait on a word nothing writes.
        bool stall = (stall_mask(P.status) & kStallDecodeFused) != 0;
        unsigned long long t_idle = now_ns();   // start of the current idle spell
        while (ok) {
            if (!drain_topk()) { ok = false; break; }
            if (pending < 0 && attn_left) {
                if (!index_left) seen_claim = ld_volatile(c_claim);
                if (seen_claim >= total_attn) {
                    attn_left = false;
                } else if (!index_left || seen_claim < seen_pub) {
                    const int h = atomicAdd(c_claim, 1);
                    if (h >= total_attn) attn_left = false;
                    else { pending = h; pending_flag = 0; }
                    seen_claim = h + 1;
                }
            }
            if (pending >= 0 && (!index_left || pending_flag != 0)) {
                // Attention item: its flag is set, or will be once the index
                // units of its sequence are done.  While waiting, keep queueing
                // this CTA's top-k requests: the one that publishes the item
                // may be among them.
                const int item = pending;
                pending = -1;
                const int *flag = stall ? P.status + kCtlNeverWord : P.aq_flag + item;
                stall = false;
                const unsigned long long t0 = now_ns();   // this wait's own clock
                while (ld_volatile(flag) == 0) {
                    if (!drain_topk() || *abort_flag || now_ns() - t0 > lim) {
                        set_status(P.status, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    __nanosleep(128);
                }
                if (!ok) break;
                __threadfence();
                const int bg = __ldcg(P.aq_item + item);
                const int b = bg / H, g = bg % H;
                const int nb = (P.lens[b] + kBlock - 1) / kBlock;
                const int n_kept = min(K, nb);
                if (!push(make_int4(kWorkAttn, bg, n_kept, 0))) { ok = false; break; }
                // K and V tiles of every kept block, the next id loaded ahead
                const int32_t *idrow = P.ids + (static_cast<long long>(b) * HI + g / (H / HI)) * K;
                int jn = __ldcg(idrow);
                for (int sl = 0; sl < n_kept && ok; ++sl) {
                    const int j = jn;
                    if (sl + 1 < n_kept) jn = __ldcg(idrow + sl + 1);
                    const int tok = static_cast<int>(kv_block_row(P.kv, b, j, P.status));
                    int sk, sv;
                    if (!stage(sk)) { ok = false; break; }
                    mbar_arrive_expect_tx(&S.full[sk], kStageBytes);
                    tma_load_3d(S.ring[sk], &tmK, 0, g, tok, &S.full[sk]);
                    tma_load_3d(S.ring[sk] + 16384, &tmK, 64, g, tok, &S.full[sk]);
                    if (!stage(sv)) { ok = false; break; }
                    mbar_arrive_expect_tx(&S.full[sv], kStageBytes);
                    tma_load_3d(S.ring[sv], &tmV, 0, g, tok, &S.full[sv]);
                    tma_load_3d(S.ring[sv] + 16384, &tmV, 64, g, tok, &S.full[sv]);
                }
                t_idle = now_ns();
                continue;
            }
            if (index_left) {
                const int u = u_next;
                if (u >= U) { index_left = false; t_idle = now_ns(); continue; }
                u_next = atomicAdd(c_unit, 1);
                // read now, used at the next pass of the loop
                if (pending >= 0) pending_flag = ld_volatile(P.aq_flag + pending);
                else if (attn_left) { seen_claim = ld_volatile(c_claim); seen_pub = ld_volatile(c_pub); }
                int b, j;
                unit_of(S.prefix, P.B, u, b, j);
                const int L = P.lens[b];
                const int ntok = min(kBlock, L - j * kBlock);
                if (!push(make_int4(kWorkIndex, b, j, ntok))) { ok = false; break; }
                ++units_pushed;
                const long long t_first = kv_block_row(P.kv, b, j, P.status);
                for (int t0s = 0; t0s < ntok; t0s += tps) {
                    int slot;
                    if (!stage(slot)) { ok = false; break; }
                    const uint32_t bytes = static_cast<uint32_t>(min(tps, ntok - t0s)) * HI * kDim * 2;
                    mbar_arrive_expect_tx(&S.full[slot], bytes);
                    bulk_g2s(S.ring[slot], kbase + (t_first + t0s) * HI * kDim, bytes, &S.full[slot], pol);
                }
                t_idle = now_ns();
                continue;
            }
            if (!attn_left) break;
            // No work taken in this pass: an idle spell, bounded from its start.
            if (*abort_flag || now_ns() - t_idle > lim) { set_status(P.status, kStatusTimeout); ok = false; break; }
            continue;
        }
        // A top-k this CTA's bookkeeper has still to request must be queued
        // before the end: wait until it has finished every unit pushed here.
        const unsigned long long t_end = now_ns();
        while (ok && ld_volatile(&S.book_done) < units_pushed) {
            if (!drain_topk() || *abort_flag || now_ns() - t_end > lim) {
                set_status(P.status, kStatusTimeout);
                ok = false;
                break;
            }
            __nanosleep(64);
        }
        if (ok) ok = drain_topk();
        if (!ok) *abort_flag = 1;
        push(make_int4(kWorkEnd, 0, 0, 0));      // best effort: consumers also stop on abort
        // let every copy already issued land before the CTA can exit
        for (int k = max(0, it - kStages); k < it; ++k)
            mbar_wait(&S.full[k % kStages], (k / kStages) & 1, nullptr);
        return;
    }

    // ---------------------------------------------------- consumers
    // CTA-wide syncs among the consumers are a bounded mbarrier that every
    // consumer thread arrives on, so a warp that stops early cannot hang the
    // others: their wait gives up, raises the abort flag and they stop too.
    int cb = 0;
    auto cbar = [&]() {
        mbar_arrive(&S.cbar);
        if (!*abort_flag && !mbar_wait(&S.cbar, cb & 1, P.status)) *abort_flag = 1;
        ++cb;
    };
    const int c16 = tid & 15, r16 = tid >> 4;     // index rows: 16-byte chunk, row slot 0..15
    const int gi = r16 % HI;                       // index head of this thread's index rows
    const int gq = lane >> 2, tq = lane & 3;
    const int r0 = warp * 16;                      // attention: this warp's 16 tokens
    const int tps = 128 / HI;
    const float sl2 = P.softmax_scale * kLog2e;
    const __nv_bfloat16 *qibase = static_cast<const __nv_bfloat16 *>(P.q_idx);
    float qf[8];
    int cur_b = -1, it = 0, unit_iter = 0;
    auto wait_stage = [&](int &slot) -> bool {
        slot = it % kStages;
        bool have = !*abort_flag && mbar_wait(&S.full[slot], (it / kStages) & 1, P.status);
        have = __all_sync(0xffffffffu, have);
        ++it;
        if (!have) *abort_flag = 1;
        return have;
    };
    auto release_stage = [&](int slot) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[slot]);
    };

    // Top-k of sequence b for every group (warp per group), then one
    // attention item per group published to the global queue.
    auto topk_and_publish = [&](int b) {
        __threadfence();                           // other CTAs' scores of b are visible
        const int L = P.lens[b];
        const int nb = (L + kBlock - 1) / kBlock;
        const int own = nb - 1;                    // decode: the query is token L-1
        unsigned long long *keys = reinterpret_cast<unsigned long long *>(&S.om[warp][0][0]);
        int *sel = reinterpret_cast<int *>(&S.om[warp][2][0]);
        for (int g = warp; g < HI; g += kWarps) {   // index heads
            const long long bg = static_cast<long long>(b) * HI + g;
            const float *sc = P.scores + bg * nbs;
            int n = 0;
            if (nb <= K) {
                for (int q = lane; q < nb; q += 32) sel[q] = q;
                n = nb;
            } else {
                const int m = K - 1;
                warp_select([&](int jj) { return topk_key(__ldcg(sc + jj), jj); }, 0, own, m, lane, keys);
                for (int q = lane; q < m; q += 32) sel[q] = topk_key_id(keys[q]);
                if (lane == 0) sel[m] = own;
                n = K;
            }
            __syncwarp();
            emit_sorted(sel, n, sc, K, lane, P.ids + bg * K, P.out_scores + bg * K);
            __syncwarp();
        }
        __threadfence();
        cbar();
        const int count = H;                       // one attention item per group
        if (tid == 0) S.bcast[1] = atomicAdd(P.ctr + kCtrStride, count);
        cbar();
        const int base = S.bcast[1];
        for (int e = tid; e < count; e += kConsumers) P.aq_item[base + e] = b * H + e;
        __threadfence();
        for (int e = tid; e < count; e += kConsumers)
            *reinterpret_cast<volatile int *>(P.aq_flag + base + e) = 1;
        __threadfence();
        cbar();
        if (tid == 0) atomicAdd(P.ctr + 3 * kCtrStride, count);
    };

    // Hands one index unit's row-slot maxima (or, with b = -1, the end of the
    // stream) to the bookkeeper through the kRedQ-deep queue.
    auto hand_over = [&](int b, int j, float runmax) -> bool {
        const int slot = unit_iter % kRedQ;
        bool have = unit_iter < kRedQ ||
                    (!*abort_flag && mbar_wait(&S.red_empty[slot], ((unit_iter / kRedQ) - 1) & 1, P.status));
        have = __all_sync(0xffffffffu, have);
        ++unit_iter;
        if (!have) { *abort_flag = 1; return false; }
        if (c16 == 0) S.red[slot][r16] = runmax;
        if (tid == 0) { S.red_b[slot] = b; S.red_j[slot] = j; }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.red_full[slot]);
        return true;
    };

    for (int n = 0;; ++n) {
        const int wslot = n % kQueue;
        bool have = !*abort_flag && mbar_wait(&S.wq_full[wslot], (n / kQueue) & 1, P.status);
        have = __all_sync(0xffffffffu, have);
        if (!have) { *abort_flag = 1; break; }
        const int4 w = S.wq[wslot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.wq_empty[wslot]);
        if (w.x == kWorkEnd) break;
        if (w.x == kWorkTopk) {
            if (!*abort_flag) topk_and_publish(w.y);
            continue;
        }

        if (w.x == kWorkIndex) {
            // ---- index unit: block j of sequence b, every group
            const int b = w.y, j = w.z, ntok = w.w;
            if (b != cur_b) {
                const uint4 qv = *reinterpret_cast<const uint4 *>(qibase + ((long long)b * HI + gi) * kDim + c16 * 8);
                qf[0] = bf16lo(qv.x); qf[1] = bf16hi(qv.x);
                qf[2] = bf16lo(qv.y); qf[3] = bf16hi(qv.y);
                qf[4] = bf16lo(qv.z); qf[5] = bf16hi(qv.z);
                qf[6] = bf16lo(qv.w); qf[7] = bf16hi(qv.w);
                cur_b = b;
            }
            float runmax = -INFINITY;
            for (int t0 = 0; t0 < ntok; t0 += tps) {
                const int rows_valid = min(tps, ntok - t0) * HI;
                int slot;
                if (wait_stage(slot)) {
                    const uint8_t *sb = S.ring[slot];
#pragma unroll
                    for (int pass = 0; pass < 8; ++pass) {
                        const int row = r16 + 16 * pass;
                        const uint4 kv = *reinterpret_cast<const uint4 *>(sb + row * 256 + c16 * 16);
                        float d = qf[0] * bf16lo(kv.x);
                        d = fmaf(qf[1], bf16hi(kv.x), d);
                        d = fmaf(qf[2], bf16lo(kv.y), d);
                        d = fmaf(qf[3], bf16hi(kv.y), d);
                        d = fmaf(qf[4], bf16lo(kv.z), d);
                        d = fmaf(qf[5], bf16hi(kv.z), d);
                        d = fmaf(qf[6], bf16lo(kv.w), d);
                        d = fmaf(qf[7], bf16hi(kv.w), d);
                        d += __shfl_xor_sync(0xffffffffu, d, 8);
                        d += __shfl_xor_sync(0xffffffffu, d, 4);
                        d += __shfl_xor_sync(0xffffffffu, d, 2);
                        d += __shfl_xor_sync(0xffffffffu, d, 1);
                        if (row < rows_valid) runmax = fmaxf(runmax, d);
                    }
                    release_stage(slot);
                }
            }
            // Row-slot maxima to the bookkeeper, which finishes the unit.
            if (!hand_over(b, j, runmax)) break;
            continue;
        }

        // ---- attention item: every kept block of (sequence b, group g).
        // Warp w takes tokens 16w..16w+15 of each block, with a running
        // (max, sum, O^T) per head across the blocks; the blocks arrive in
        // ascending id order, so only the last one (the own block) is partial.
        // The group's heads sit on the 8-wide side of the products: NT = 1
        // n8 tile for groups of up to 8 heads, 2 for groups of 16.
        const int bg = w.y, n_kept = w.z;
        const int b = bg / H, g = bg % H;
        const int L = P.lens[b];
        const int last_valid = L - ((L - 1) / kBlock) * kBlock;
        auto attn_item = [&](auto ntc) {
            constexpr int NT = decltype(ntc)::value;
            uint32_t qb[NT][8][2];                  // Q^T of heads 8 nt + gq (zero past G)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int hq = nt * 8 + gq;
                const __nv_bfloat16 *qh = static_cast<const __nv_bfloat16 *>(P.q) +
                                          ((long long)b * P.H_q + (long long)g * G + hq) * kDim + tq * 2;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    qb[nt][kk][0] = hq < G ? *reinterpret_cast<const uint32_t *>(qh + kk * 16) : 0u;
                    qb[nt][kk][1] = hq < G ? *reinterpret_cast<const uint32_t *>(qh + kk * 16 + 8) : 0u;
                }
            }
            float m2[NT][2], l2[NT][2];
            float acc[NT][8][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                m2[nt][0] = m2[nt][1] = -INFINITY;
                l2[nt][0] = l2[nt][1] = 0.f;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;
            }
            for (int sl = 0; sl < n_kept; ++sl) {
                int sk, sv;
                const bool hk = wait_stage(sk);
                const bool hv = wait_stage(sv);
                if (!(hk && hv)) break;
                const int nvalid = sl == n_kept - 1 ? last_valid : kBlock;
                const uint32_t kb = smem_u32(S.ring[sk]), vb = smem_u32(S.ring[sv]);
                if (nvalid < r0 + 16) {
                    // value rows past the query: weight 0, but padding may hold NaN
                    for (int e = lane; e < 16 * 16; e += 32) {
                        const int r = r0 + (e >> 4), c = e & 15;
                        if (r >= nvalid)
                            *reinterpret_cast<uint4 *>(S.ring[sv] + (c >> 3) * 16384 + r * 128 + (c & 7) * 16) =
                                make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();      // before the next TMA write of this stage
                    __syncwarp();
                }
                float sv4[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) sv4[nt][0] = sv4[nt][1] = sv4[nt][2] = sv4[nt][3] = 0.f;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int chunk = ((kk & 3) << 1) | (lane >> 4);
                    uint32_t a4[4];
                    ldsm_x4(kb + (kk >> 2) * 16384 + swz128(r0 + (lane & 15), chunk), a4[0], a4[1], a4[2], a4[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sv4[nt], a4, qb[nt][kk][0], qb[nt][kk][1]);
                }
                uint32_t pb0[NT], pb1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float p[4];
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const float x0 = r0 + gq < nvalid ? sv4[nt][c] * sl2 : -INFINITY;
                        const float x1 = r0 + gq + 8 < nvalid ? sv4[nt][2 + c] * sl2 : -INFINITY;
                        float cm = fmaxf(x0, x1);
                        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 4));
                        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 8));
                        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 16));
                        const float mnew = fmaxf(m2[nt][c], cm);
                        const float mref = mnew == -INFINITY ? 0.f : mnew;
                        const float alpha = exp2f(m2[nt][c] - mref);
                        m2[nt][c] = mnew;
                        p[c] = exp2f(x0 - mref);
                        p[2 + c] = exp2f(x1 - mref);
                        l2[nt][c] = l2[nt][c] * alpha + p[c] + p[2 + c];
#pragma unroll
                        for (int mt = 0; mt < 8; ++mt) {
                            acc[nt][mt][c] *= alpha;
                            acc[nt][mt][2 + c] *= alpha;
                        }
                    }
                    pb0[nt] = movmatrix_t(pack_bf16x2(p[0], p[1]));
                    pb1[nt] = movmatrix_t(pack_bf16x2(p[2], p[3]));
                }
                const int mi = lane >> 3;
                const int r = r0 + ((mi >> 1) << 3) + (lane & 7);
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    const int d = mt * 16 + ((mi & 1) << 3);
                    uint32_t a4[4];
                    ldsm_x4_t(vb + (d >> 6) * 16384 + swz128(r, (d & 63) >> 3), a4[0], a4[1], a4[2], a4[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt][mt], a4, pb0[nt], pb1[nt]);
                }
                release_stage(sk);
                release_stage(sv);
            }
            // Per n8 tile: per-warp partials to shared memory (heads 2tq + c
            // of the tile), then the 8 warps merged and the heads written.
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float l = l2[nt][c];
                    l += __shfl_xor_sync(0xffffffffu, l, 4);
                    l += __shfl_xor_sync(0xffffffffu, l, 8);
                    l += __shfl_xor_sync(0xffffffffu, l, 16);
                    const int h = 2 * tq + c;
                    if (gq == 0) { S.mw[warp][h] = m2[nt][c]; S.lw[warp][h] = l; }
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        S.om[warp][h][mt * 16 + gq] = acc[nt][mt][c];
                        S.om[warp][h][mt * 16 + gq + 8] = acc[nt][mt][2 + c];
                    }
                }
                cbar();
                const int nh = min(8, G - nt * 8);            // heads of this tile
                if (!*abort_flag) {
                    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(P.out) +
                                         ((long long)b * P.H_q + (long long)g * G + nt * 8) * kDim;
                    for (int e = tid; e < nh * kDim; e += kConsumers) {
                        const int h = e / kDim, d = e % kDim;
                        float M = -INFINITY;
#pragma unroll
                        for (int w8 = 0; w8 < kWarps; ++w8) M = fmaxf(M, S.mw[w8][h]);
                        const float Mr = M == -INFINITY ? 0.f : M;
                        float o = 0.f, l = 0.f;
#pragma unroll
                        for (int w8 = 0; w8 < kWarps; ++w8) {
                            const float f = exp2f(S.mw[w8][h] - Mr);
                            o += S.om[w8][h][d] * f;
                            l += S.lw[w8][h] * f;
                        }
                        out[e] = __float2bfloat16(o / l);
                    }
                }
                cbar();                             // om, mw, lw and bcast are reused
            }
        };
        if (G > 8) attn_item(std::integral_constant<int, 2>{});
        else attn_item(std::integral_constant<int, 1>{});
    }
    hand_over(-1, 0, 0.f);                          // end of the bookkeeper's stream
}

}  // namespace

size_t decode_fused_layout(int B, int H_q, int H_kv, int n_idx, int K, int max_kv_len,
                           DecodeFusedLayout *L) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t nb_max = score_stride((max_kv_len + kBlock - 1) / kBlock);
    const size_t items = static_cast<size_t>(B) * H_kv;
    // Everything cleared per call sits right after the status header, so one
    // memset covers [0, zero_hi).
    size_t o = kWsHeaderBytes;
    L->zero_lo = o;
    L->ctr = o;      o += 4 * kCtrStride * 4;
    L->seq_done = o; o += up(static_cast<size_t>(B) * 4);
    L->aq_flag = o;  o += up(items * 4);
    L->zero_hi = o;
    L->scores = o;   o += up(static_cast<size_t>(B) * n_idx * nb_max * 4);
    L->aq_item = o;  o += up(items * 4);
    L->total = o;
    (void)H_q;
    (void)K;
    return o;
}

cudaError_t launch_decode_fused(const DecodeFusedArgs &a, cudaStream_t s) {
    static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory budget");
    CUtensorMap tk, tv;
    if (!encode_kv_tensor_map(&tk, a.k_cache, a.H_kv, a.kv.capacity) ||
        !encode_kv_tensor_map(&tv, a.v_cache, a.H_kv, a.kv.capacity))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope trace(s, "decode_fused_step");
    DecodeFusedArgs args = a;
    void *params[] = {&tk, &tv, &args};
    // Cooperative: every CTA resident at once (they hand work to each other).
    return cudaLaunchCooperativeKernel(reinterpret_cast<void *>(decode_fused_kernel),
                                       dim3(device_sm_count()), dim3(kThreads), params, smem, s);
}

}  // namespace msa
