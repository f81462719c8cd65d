// attn_prefill.cu -- MSA sparse branch for prefill (many query rows), on the
// fifth-generation tensor cores, organised around the KV blocks.
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 -- exact attention over the kept blocks
// only; section 六 -- the heads of a GQA group share the group's block set,
// so one K/V block tile serves every (row, head) of the group that kept it.
// The dev.to MiniMax-M3 summary describes the KV tile as the outer loop with
// each tile read once for every query that needs it; that is the organisation
// used here for every kept block except the query's own one.
//
// Exactness: softmax is invariant to the shift subtracted before exp, so the
// partial sums of different blocks can be added directly if they share one
// shift per (row, head).  The shift is the row's exact max over its own block
// (pass A) plus 4 (base 2).  Partial outputs are added in fp16: the adds at
// L2 cost bytes, not operations, so 16-bit partials halve the pass's bound,
// and fp16 keeps 11 significant bits (the bf16 output keeps 8).  A partial
// is checked before it is added: if any of its values exceeds 65504 / top_k
// (or is not finite), the sum of at most top_k partials could overflow, so
// that (row, head) is flagged instead, its partials are dropped, and the
// exact pass recomputes its output from scratch after the others (rare: a
// kept block would have to beat the own block's max by about 2^9 or more).
//
// Passes (one stream, no host synchronisation):
//   bucket_*   rows that kept block j (j != own) bucketed by (sequence, group,
//              8192-row range, j); buckets become work items of <= 256 rows
//   pass A     own block of every row (causal), query-outer: writes the
//              partial output (fp16), sum and shift
//   pass B     the other kept blocks, block-outer: partials added into the
//              accumulator with bulk fp16 reductions (cp.reduce.async.bulk)
//   finalize   out = accumulator / sum, bf16
//   exact      flagged (row, head) only: softmax over every kept key in fp32
//              on CUDA cores, written over finalize's output
//
// Passes A and B share one kernel: per 16-row tile, 16 rows x 8 heads = 128
// TMEM lanes; the tile's Q rows are gathered by TMA (one 8-head x 64-dim box
// per row and half), S = Q K^T and O = P V run as tcgen05.mma kind::f16
// (M=128, N=128, K=128).  S and O live in TMEM; the softmax writes P back to
// TMEM as bf16 pairs and the PV product reads it from there (V from shared
// memory, MN-major).  Roles: warp 0 TMA, warp 1 MMA issue, warp 2 TMEM owner,
// warps 4-11 softmax, warps 12-15 epilogue.  The epilogue stages each partial
// output in shared memory and hands it to the bulk-copy engine as one fp32
// add-reduction per row: the reductions, which bound pass B, then never sit
// in the SM's load/store queue in front of the softmax's memory operations.
// The accumulator interleaves the 8 heads of a row at 16-byte granularity
// (8 dims of one head per 16 bytes), so a row's partial output is one
// contiguous 2 KiB run.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 512;           // 4 control, 8 softmax and 4 epilogue warps
constexpr int kSoftWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kEpiWarp0 = 4 + kSoftWarps;    // first epilogue warp
constexpr int kG = 8;                      // heads per group handled by this path
constexpr int kTileRows = 128 / kG;        // query rows per 128-lane tile
constexpr int kRange = 8192;               // query rows per bucket range
constexpr int kItemRows = 256;             // max rows per pass-B work item
constexpr uint32_t kTmemCols = 512;        // S[2], P[2] and O
// TMEM columns: S[2] (2 x 128 fp32), P[2] (2 x 64 columns of bf16 pairs),
// O (128 fp32).  Two S buffers let the next tile's QK run while the softmax
// still works on this one; two P buffers let the softmax write a tile's P
// while the previous PV still reads the other; one O buffer suffices because
// the epilogue reads it while the next QK runs, before the next PV.
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kShiftPad = 4.f;           // shift = own-block max + this (base 2)

__device__ __forceinline__ bool seq_ok(const PrefillArgs &P, int b, int &L) {
    L = P.lens[b];
    return L >= P.Sq && L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
}

// A work item: one key block j of one (sequence, group) and the rows that
// use it.  Pass A: the rows whose own block is j (consecutive query rows
// from i_lo).  Pass B: a slice of the bucket of rows that kept j as a
// non-own block, entries rows_off .. rows_off + n - 1 of bucket_rows (and
// of bucket_shift).
struct Item {
    int b, g, j, n;         // n = number of rows; n <= 0: nothing to do
    int i_lo;               // pass A: first query row
    int rows_off;           // pass B: first bucket entry
    int L;
    int pad;
};

template <int MODE>
__device__ __forceinline__ Item item_at(const PrefillArgs &P, long long it) {
    Item x;
    x.i_lo = 0;
    x.rows_off = 0;
    x.pad = 0;
    if (MODE == 0) {
        const int nj = (P.Sq + 127) / 128 + 1;
        x.b = static_cast<int>(it / (static_cast<long long>(P.H_kv) * nj));
        const int rem = static_cast<int>(it % (static_cast<long long>(P.H_kv) * nj));
        x.g = rem / nj;
        const int jj = rem % nj;
        x.j = 0;
        if (!seq_ok(P, x.b, x.L)) { x.n = 0; return x; }
        const long long p0 = static_cast<long long>(x.L) - P.Sq;   // position of row 0
        x.j = static_cast<int>(p0 / 128) + jj;
        const long long plo = max(p0, static_cast<long long>(x.j) * 128);
        const long long phi = min(static_cast<long long>(x.L), static_cast<long long>(x.j) * 128 + 128);
        x.n = phi > plo ? static_cast<int>(phi - plo) : 0;
        x.i_lo = static_cast<int>(plo - p0);
    } else {
        // one 32-byte descriptor, written by item_table_kernel
        const int4 *d = reinterpret_cast<const int4 *>(P.item_desc) + 2 * it;
        const int4 a = d[0], c = d[1];
        x.b = a.x; x.g = a.y; x.j = a.z; x.n = a.w;
        x.rows_off = c.x; x.L = c.y;
    }
    return x;
}

// Flattened row (b*Sq + i) of row r of the item.
template <int MODE>
__device__ __forceinline__ long long tile_row(const PrefillArgs &P, const Item &x, int r) {
    return MODE == 1 ? static_cast<long long>(P.bucket_rows[x.rows_off + r])
                     : static_cast<long long>(x.b) * P.Sq + x.i_lo + r;
}

template <int MODE>
__device__ __forceinline__ long long n_items(const PrefillArgs &P) {
    if (MODE == 0) return static_cast<long long>(P.B) * P.H_kv * ((P.Sq + 127) / 128 + 1);
    return *P.item_total;
}

struct Smem {
    uint8_t kv[2][65536];                  // K lo, K hi, V lo, V hi (16 KiB each)
    uint8_t q[2][32768];                   // gathered Q tile, two swizzled halves
    uint8_t ostage[kEpiWarps][8192];       // epilogue: 4 rows x 128 dims x 8 heads fp16 per warp
    uint64_t kv_full[2], kv_empty[2], q_full[2], q_empty[2];
    uint64_t s_full[2], s_empty[2], o_full, o_empty;
    uint64_t p_full[2], p_empty[2];
    float xmax[2][128];                    // pass A: each softmax warp's half-row max
    uint64_t xbar[4];                      // pass A: the two softmax warps of a lane quarter
    uint64_t item_full[4], item_empty[4];  // work-item queue: producer -> MMA, softmax, epilogue
    Item item_q[4];                        // decoded items (n = -1: no more work)
    uint32_t tmem_base;
    int abort_flag;
};

// 227 KiB is the per-block shared-memory limit; 1 KiB more aligns the base.
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory over the per-block limit");

constexpr int kQueue = 4;
// Q loader warps: pass A one TMA thread (whole 16-row boxes), pass B two
// warps gathering rows with cp.async.
template <int MODE> constexpr int kLoaderWarps = MODE == 0 ? 1 : 2;
// MMA thread + one per loader, softmax and epilogue warp
template <int MODE> constexpr int kQueueReaders = 1 + kLoaderWarps<MODE> + kSoftWarps + kEpiWarps;

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// 2^x on the special-function unit (relative error ~2^-22, results below
// 2^-126 flushed to 0).  Probabilities are rounded to bf16 right after, and
// the shift keeps every kept term above 2^-64 of the row's largest one.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ16,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PrefillArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long total = n_items<MODE>(P);

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.kv_full[i], 1);
            mbar_init(&S.kv_empty[i], 1);
            // pass A: one expect-tx arrival (TMA); pass B: one arrival per
            // loader thread, made by the hardware once its copies have landed
            mbar_init(&S.q_full[i], MODE == 0 ? 1 : kLoaderWarps<MODE> * 32);
            mbar_init(&S.q_empty[i], 1);          // released by the MMA commit
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.s_empty[i], kSoftWarps);
            mbar_init(&S.p_full[i], kSoftWarps);
            mbar_init(&S.p_empty[i], 1);
        }
        mbar_init(&S.o_full, 1);
        mbar_init(&S.o_empty, kEpiWarps);
        for (int i = 0; i < 4; ++i) mbar_init(&S.xbar[i], 64);   // every lane of both warps
        for (int i = 0; i < kQueue; ++i) {
            mbar_init(&S.item_full[i], 1);
            mbar_init(&S.item_empty[i], kQueueReaders<MODE>);
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(&S.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    volatile int *abort_flag = &S.abort_flag;

    // Work items are claimed in order from one global counter, so every CTA
    // works on neighbouring items (the same row range): the accumulator and Q
    // rows of that range stay in L2.  Warp 0 claims, decodes and publishes
    // each item; the MMA thread, softmax and epilogue warps read it from the
    // queue.
    long long *counter = MODE == 0 ? P.item_next : P.item_next + 1;
    // n-th item for a reader, decoded by the producer; false on abort.
    // x.n < 0 marks the end of the work.
    auto next_item = [&](int n, bool warp_reader, Item &x) -> bool {
        const int slot = n % kQueue;
        bool ok = !*abort_flag && mbar_wait(&S.item_full[slot], (n / kQueue) & 1, P.status);
        if (warp_reader) ok = __all_sync(0xffffffffu, ok);
        if (!ok) return false;
        x = S.item_q[slot];
        if (warp_reader) __syncwarp();
        if (!warp_reader || lane == 0) mbar_arrive(&S.item_empty[slot]);
        return true;
    };

    if (warp == 0) {
        // ------------------------------------------------ producer (lane 0): claims
        // and decodes items, publishes them, loads each item's K and V block
        // lanes 1-31 go straight to the final barrier
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            int ki = 0;
            bool ok = true;
            for (int n = 0; ok; ++n) {
                const int slot = n % kQueue;
                if (n >= kQueue && (*abort_flag || !mbar_wait(&S.item_empty[slot], ((n / kQueue) - 1) & 1, P.status))) {
                    ok = false;
                    break;
                }
                // Decode once here; the other roles read the result.
                long long it = atomicAdd(reinterpret_cast<unsigned long long *>(counter), 1ull);
                Item x;
                if (it >= total) x.n = -1;
                else x = item_at<MODE>(P, it);
                S.item_q[slot] = x;
                mbar_arrive(&S.item_full[slot]);
                if (x.n < 0) break;
                if (x.n == 0) continue;
                const int kvs = ki & 1;
                if (ki >= 2 && (*abort_flag || !mbar_wait(&S.kv_empty[kvs], ((ki >> 1) - 1) & 1, P.status))) {
                    ok = false;
                    break;
                }
                const int tok = static_cast<int>(kv_block_row(P.kv, x.b, x.j, P.status));
                mbar_arrive_expect_tx(&S.kv_full[kvs], 65536);
                tma_load_3d(S.kv[kvs], &tmK, 0, x.g, tok, &S.kv_full[kvs]);
                tma_load_3d(S.kv[kvs] + 16384, &tmK, 64, x.g, tok, &S.kv_full[kvs]);
                tma_load_3d(S.kv[kvs] + 32768, &tmV, 0, x.g, tok, &S.kv_full[kvs]);
                tma_load_3d(S.kv[kvs] + 49152, &tmV, 64, x.g, tok, &S.kv_full[kvs]);
                ++ki;
            }
            if (!ok) *abort_flag = 1;
        }
    } else if (warp == 2 || (warp == 3 && MODE == 1)) {
        // ------------------------------------------------ Q loaders
        // Pass A: a tile is 16 consecutive query rows, two TMA boxes of
        // 16 rows x 8 heads x 64 dims.  Pass B: the tile's rows are scattered
        // (bucket entries), and one small TMA box per row would be bound by
        // the bulk engine's per-copy cost (shared with the reductions), so
        // two warps gather each 2 KiB (row, group) slice with 16-byte
        // cp.async copies straight into the 128-byte-swizzled layout the MMA
        // reads; the tile's barrier completes once every copy has landed.
        const int lw = warp - 2;
        int qt = 0, n = 0;
        bool ok = true;
        if (MODE == 0 && lane == 0) prefetch_tensormap(&tmQ16);
        Item x;
        while (ok) {
            if (!next_item(n++, true, x)) { ok = false; break; }
            if (x.n < 0) break;
            if (x.n == 0) continue;
            for (int t0 = 0; t0 < x.n; t0 += kTileRows, ++qt) {
                const int qs = qt & 1;
                int myrow = -1;                      // lane k < 8: row of this warp's k-th slot
                if (MODE == 1 && lane < 8 && t0 + lw + 2 * lane < x.n)
                    myrow = P.bucket_rows[x.rows_off + t0 + lw + 2 * lane];
                bool free_ = qt < 2 || (!*abort_flag && mbar_wait(&S.q_empty[qs], ((qt >> 1) - 1) & 1, P.status));
                free_ = __all_sync(0xffffffffu, free_);
                if (!free_) { ok = false; break; }
                if (MODE == 0) {
                    if (lane == 0) {
                        const int row0 = x.b * P.Sq + x.i_lo + t0;
                        mbar_arrive_expect_tx(&S.q_full[qs], 32768);
                        tma_load_3d(S.q[qs], &tmQ16, 0, x.g * kG, row0, &S.q_full[qs]);
                        tma_load_3d(S.q[qs] + 16384, &tmQ16, 64, x.g * kG, row0, &S.q_full[qs]);
                    }
                    __syncwarp();
                    continue;
                }
                const uint32_t qbase = smem_u32(S.q[qs]);
#pragma unroll 1
                for (int k = 0; k < 8; ++k) {
                    const int r = __shfl_sync(0xffffffffu, myrow, k);
                    if (r < 0) continue;
                    const int rr = lw + 2 * k;       // tile row
                    const uint8_t *src = static_cast<const uint8_t *>(P.q) +
                                         (static_cast<long long>(r) * P.H_q + x.g * kG) * (kDim * 2);
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        const int ch = lane + 32 * qq;   // 16-byte chunk of the 2 KiB slice
                        const int h = ch >> 4, c = ch & 15, m = rr * kG + h;
                        cp_async16(qbase + (c >> 3) * 16384 + m * 128 + (((c & 7) ^ (m & 7)) << 4),
                                   src + ch * 16);
                    }
                }
                // Each thread's arrival on the tile's barrier fires when its
                // copies have landed (tracked by the hardware; a software wait,
                // proxy fence and arrive let the MMA read stale rows).
                cp_async_arrive_noinc(&S.q_full[qs]);
            }
        }
        if (MODE == 1) cp_async_wait_all();          // nothing lands after the CTA ends
        if (!ok) *abort_flag = 1;
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc_qk = umma_idesc_bf16(128, 128);
        const uint32_t idesc_pv = umma_idesc_bf16(128, 128) | (1u << 16);   // B (V) MN-major
        int ki = 0, qt = 0;
        int pv_pending = -1, pv_kvs = 0, pv_last = 0;   // tile waiting for its PV
        bool ok = true;
        // O = P V: P (bf16) from TMEM, V from shared memory.
        // Descriptors are built once; a K step only moves the start address
        // field (bits 0-13, in 16-byte units), which never carries here.
        const uint64_t kv_desc0 = umma_desc(smem_u32(S.kv[0]), 16, 1024);
        const uint64_t kv_desc1 = umma_desc(smem_u32(S.kv[1]), 16, 1024);
        const uint64_t v_desc0 = umma_desc(smem_u32(S.kv[0] + 32768), 16384, 1024);
        const uint64_t v_desc1 = umma_desc(smem_u32(S.kv[1] + 32768), 16384, 1024);
        const uint64_t q_desc0 = umma_desc(smem_u32(S.q[0]), 16, 1024);
        const uint64_t q_desc1 = umma_desc(smem_u32(S.q[1]), 16, 1024);
        auto issue_pv = [&](int t, int kvs, int last_of_item) -> bool {
            const int pb = t & 1;
            if (*abort_flag || !mbar_wait(&S.p_full[pb], (t >> 1) & 1, P.status)) return false;
            // the epilogue has read the previous tile's O
            if (t >= 1 && (*abort_flag || !mbar_wait(&S.o_empty, (t - 1) & 1, P.status)))
                return false;
            tc_fence_after();
            const uint64_t vd = kvs ? v_desc1 : v_desc0;
            const uint32_t d = tmem + kColO, a = tmem + kColP + pb * 64;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma_bf16_ts(d, a + kk * 8, vd + static_cast<uint64_t>(kk * 128), idesc_pv, kk > 0 ? 1u : 0u);
            umma_commit(&S.o_full);
            umma_commit(&S.p_empty[pb]);
            if (last_of_item) umma_commit(&S.kv_empty[kvs]);
            return true;
        };
        for (int n = 0; ok; ++n) {
            Item x;
            if (!next_item(n, false, x)) { ok = false; break; }
            if (x.n < 0) break;
            if (x.n == 0) continue;
            const int kvs = ki & 1;
            if (*abort_flag || !mbar_wait(&S.kv_full[kvs], (ki >> 1) & 1, P.status)) { ok = false; break; }
            ++ki;
            const uint64_t kd = kvs ? kv_desc1 : kv_desc0;
            for (int t0 = 0; t0 < x.n; t0 += kTileRows, ++qt) {
                const int qs = qt & 1;
                if (*abort_flag || !mbar_wait(&S.q_full[qs], (qt >> 1) & 1, P.status)) { ok = false; break; }
                fence_proxy_async_smem();   // pass B's Q rows were written by cp.async
                // S[sb] is free once the softmax has read the tile two back.
                const int sb = qt & 1;
                if (qt >= 2 && (*abort_flag || !mbar_wait(&S.s_empty[sb], ((qt >> 1) - 1) & 1, P.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t qd = qs ? q_desc1 : q_desc0;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = static_cast<uint64_t>((kk >> 2) * 1024 + (kk & 3) * 2);
                    umma_bf16_ss(tmem + kColS + sb * 128, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(&S.s_full[sb]);
                umma_commit(&S.q_empty[qs]);
                // PV of the previous tile runs behind this tile's QK.
                if (pv_pending >= 0 && !issue_pv(pv_pending, pv_kvs, pv_last)) { ok = false; break; }
                pv_pending = qt;
                pv_kvs = kvs;
                pv_last = t0 + kTileRows >= x.n;
            }
        }
        if (ok && pv_pending >= 0 && !issue_pv(pv_pending, pv_kvs, pv_last)) ok = false;
        if (!ok) *abort_flag = 1;
        // Every MMA issued must finish before TMEM is released.
        if (qt > 0) mbar_wait(&S.s_full[(qt - 1) & 1], ((qt - 1) >> 1) & 1, nullptr);
        if (pv_pending >= 0) mbar_wait(&S.o_full, pv_pending & 1, nullptr);
    } else if (warp >= 4 && warp < kEpiWarp0) {
        // ------------------------------------------------ softmax
        // Warps 4-7 and 8-11 share the TMEM lanes of warp % 4 and split each
        // row's 128 columns: ch = 0 takes tokens 0-63, ch = 1 takes 64-127.
        // Each half-row sum goes to the row's running sum on its own, so the
        // two warps never wait for each other.  P goes back to TMEM as bf16
        // pairs (columns kColP + 32 ch ...), where the PV product reads it.
        const int ch = (warp - 4) >> 2;
        const int m = (warp & 3) * 32 + lane;          // TMEM lane = tile row x head
        const int ri = m / kG, h = m % kG;             // tile row, head in group
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const float sl2 = P.softmax_scale * kLog2e;
        int qt = 0;
        bool ok = true;
        int ki = 0;                                    // items seen (K/V ring position)
        // Each tile's row and (pass B) shift are loaded one tile ahead, so their
        // latency hides behind the previous tile's work; at an item's last tile
        // the next item is read from the queue early for that.
        int n = 0;
        auto fetch = [&](Item &it) -> bool {       // next non-empty item or the end
            do {
                if (!next_item(n++, true, it)) return false;
            } while (it.n == 0);
            return true;
        };
        auto load_tile = [&](const Item &it, int t0, long long &row, float &shift) {
            row = 0;
            shift = 0.f;
            if (t0 + ri < it.n) {
                row = tile_row<MODE>(P, it, t0 + ri);
                if (MODE == 1)
                    shift = P.bucket_shift[static_cast<long long>(it.rows_off + t0 + ri) * kG + h];
            }
        };
        Item x;
        long long row_nx = 0;
        float shift_nx = 0.f;
        if (!fetch(x)) ok = false;
        else if (x.n > 0) load_tile(x, 0, row_nx, shift_nx);
        while (ok && x.n > 0) {
            Item xn;
            xn.n = -1;
            const int kvs = ki & 1, kv_par = (ki >> 1) & 1;
            ++ki;
            // Pass A only: in a sequence's last, partial block the value rows
            // past its length may hold anything (padding of a paged pool);
            // they get weight 0, but 0 * NaN is NaN, so zero them before the
            // first PV of the item reads them (every softmax warp arrives on
            // p_full only after its share is written).
            const int nvalid_kv = MODE == 0 ? min(128, x.L - x.j * 128) : 128;
            bool zero_v = MODE == 0 && nvalid_kv < 128;
            for (int t0 = 0; t0 < x.n; t0 += kTileRows, ++qt) {
                const bool valid = t0 + ri < x.n;
                const long long row = row_nx;
                float shift = shift_nx;
                if (t0 + kTileRows < x.n) {
                    load_tile(x, t0 + kTileRows, row_nx, shift_nx);
                } else {
                    if (!fetch(xn)) { ok = false; break; }
                    if (xn.n > 0) load_tile(xn, 0, row_nx, shift_nx);
                }
                const int sb = qt & 1;
                bool have = !*abort_flag && mbar_wait(&S.s_full[sb], (qt >> 1) & 1, P.status);
                have = __all_sync(0xffffffffu, have);
                if (!have) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = lane_addr + kColS + sb * 128;
                int lim = 127;                         // last visible column of the row
                uint32_t a[32], b[32];
                tmem_ld32r(sa + ch * 64, a);
                tmem_ld32r(sa + ch * 64 + 32, b);
                tmem_wait_ld(a);
                tmem_tie(b);
                if (MODE == 0) {
                    // own block: causal mask t <= p, exact max of the visible
                    // logits.  Each warp of the pair takes the max of its own
                    // 64 columns and swaps it with its partner (same TMEM
                    // lanes, other half) through shared memory.
                    const long long p = static_cast<long long>(x.L) - P.Sq +
                                        (row - static_cast<long long>(x.b) * P.Sq);
                    // clamped: the row's position lies in this block when valid
                    lim = static_cast<int>(max(-1LL, min(127LL, p - static_cast<long long>(x.j) * 128)));
                    float mx = -INFINITY;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        if (ch * 64 + e <= lim) mx = fmaxf(mx, __uint_as_float(a[e]) * sl2);
                        if (ch * 64 + 32 + e <= lim) mx = fmaxf(mx, __uint_as_float(b[e]) * sl2);
                    }
                    // One buffer suffices: a warp writes the next tile's value
                    // only once S of that tile exists, i.e. after both warps
                    // of the pair arrived on s_empty below, after this read.
                    S.xmax[ch][m] = mx;
                    mbar_arrive(&S.xbar[warp & 3]);
                    bool xok = !*abort_flag && mbar_wait(&S.xbar[warp & 3], qt & 1, P.status);
                    xok = __all_sync(0xffffffffu, xok);
                    if (!xok) { ok = false; break; }
                    mx = fmaxf(mx, S.xmax[ch ^ 1][m]);
                    shift = valid ? mx + kShiftPad : 0.f;
                }
                // S is in registers: the next tile's QK may overwrite it.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.s_empty[sb]);
                float l = 0.f;
                uint32_t pk[32];                        // 64 probabilities as bf16 pairs
                if (MODE == 1) {
                    // every column is visible; a padding lane gets 2^-inf = 0
                    const float sh = valid ? shift : INFINITY;
                    // four independent sums: the adds are not one serial chain
                    float l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const uint32_t *src = e < 16 ? a : b;
                        const int k = (2 * e) & 31;
                        const float p0 = fast_exp2(fmaf(__uint_as_float(src[k]), sl2, -sh));
                        const float p1 = fast_exp2(fmaf(__uint_as_float(src[k + 1]), sl2, -sh));
                        const float p2 = fast_exp2(fmaf(__uint_as_float(src[k + 2]), sl2, -sh));
                        const float p3 = fast_exp2(fmaf(__uint_as_float(src[k + 3]), sl2, -sh));
                        l += p0;
                        l1 += p1;
                        l2 += p2;
                        l3 += p3;
                        pk[e] = pack_bf16x2(p0, p1);
                        pk[e + 1] = pack_bf16x2(p2, p3);
                    }
                    l = (l + l1) + (l2 + l3);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int c0 = ch * 64 + 2 * e;
                        const uint32_t *src = e < 16 ? a : b;
                        const int k = (2 * e) & 31;
                        float p0 = fast_exp2(__uint_as_float(src[k]) * sl2 - shift);
                        float p1 = fast_exp2(__uint_as_float(src[k + 1]) * sl2 - shift);
                        p0 = (valid && c0 <= lim) ? p0 : 0.f;
                        p1 = (valid && c0 + 1 <= lim) ? p1 : 0.f;
                        l += p0 + p1;
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                }
                // P[pb]'s columns are free once the PV two tiles back has read them.
                const int pb = qt & 1;
                bool pfree = !*abort_flag && (qt < 2 || mbar_wait(&S.p_empty[pb], ((qt >> 1) - 1) & 1, P.status));
                pfree = __all_sync(0xffffffffu, pfree);
                if (!pfree) { ok = false; break; }
                tc_fence_after();
                tmem_st32(lane_addr + kColP + pb * 64 + ch * 32, pk);
                if (zero_v) {
                    bool kok = !*abort_flag && mbar_wait(&S.kv_full[kvs], kv_par, P.status);
                    kok = __all_sync(0xffffffffu, kok);
                    if (!kok) { ok = false; break; }
                    // rows nvalid_kv..127 of V lo and V hi, 16 bytes per thread-step
                    const int tsw = (warp - 4) * 32 + lane;           // 0..255
                    for (int e = tsw; e < (128 - nvalid_kv) * 16; e += kSoftWarps * 32) {
                        const int rrow = nvalid_kv + e / 16, c16 = e % 16;
                        *reinterpret_cast<uint4 *>(S.kv[kvs] + 32768 + (c16 >> 3) * 16384 +
                                                   rrow * 128 + (c16 & 7) * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    zero_v = false;
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.p_full[pb]);
                if (valid) atomicAdd(P.l_acc + row * P.H_q + x.g * kG + h, l);
                if (MODE == 0 && ch == 0 && valid) P.m_arr[row * P.H_q + x.g * kG + h] = shift;
            }
            x = xn;
        }
        if (!ok) *abort_flag = 1;
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------ epilogue
        // Warp w owns the TMEM lanes of w % 4 (tile rows 4(w%4) .. +3, all 8
        // heads), one (tile row, head) per thread.  A tile's partial output
        // goes through the warp's 8 KiB staging slot in fp16, laid out as the
        // accumulator is (a row's 8 heads interleaved at 16-byte granularity),
        // and leaves as one 2 KiB bulk copy (pass A) or bulk fp16 add (pass
        // B) per row, issued by lane 0: the reductions run on the bulk-copy
        // engine.  A partial with a value above P.acc_limit (or not finite)
        // is not added: its (row, head) is flagged for the exact pass.
        const int w = warp & 3;
        const int m = w * 32 + lane;
        const int ri = m / kG, h = m % kG;
        const bool issuer = lane == 0;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(w * 32) << 16);
        uint8_t *stage = S.ostage[w] + (ri & 3) * 2048;
        uint8_t *stage0 = S.ostage[w];
        int qt = 0;
        bool ok = true;
        // Rows are loaded one tile ahead, as in the softmax warps.
        int n = 0;
        auto fetch = [&](Item &it) -> bool {
            do {
                if (!next_item(n++, true, it)) return false;
            } while (it.n == 0);
            return true;
        };
        auto load_row = [&](const Item &it, int t0) -> long long {
            return t0 + ri < it.n ? tile_row<MODE>(P, it, t0 + ri) : -1;
        };
        Item x;
        long long row_nx = -1;
        if (!fetch(x)) ok = false;
        else if (x.n > 0) row_nx = load_row(x, 0);
        while (ok && x.n > 0) {
            Item xn;
            xn.n = -1;
            for (int t0 = 0; t0 < x.n; t0 += kTileRows, ++qt) {
                const long long row = row_nx;
                const bool valid = row >= 0;
                if (t0 + kTileRows < x.n) {
                    row_nx = load_row(x, t0 + kTileRows);
                } else {
                    if (!fetch(xn)) { ok = false; break; }
                    if (xn.n > 0) row_nx = load_row(xn, 0);
                }
                __half *dst4[4];
#pragma unroll
                for (int r4 = 0; r4 < 4; ++r4) {
                    const long long rr = __shfl_sync(0xffffffffu, row, r4 * 8);
                    dst4[r4] = rr >= 0 ? P.o_acc + (rr * P.H_kv + x.g) * (kDim * kG) : nullptr;
                }
                bool have = !*abort_flag && mbar_wait(&S.o_full, qt & 1, P.status);
                have = __all_sync(0xffffffffu, have);
                if (!have) { ok = false; break; }
                tc_fence_after();
                // The slot is free once the bulk engine has read the last tile's rows.
                if (issuer) bulk_wait_read_all();
                __syncwarp();
                bool fits = true;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t a[32], b[32];
                    tmem_ld32r(lane_addr + kColO + half * 64, a);
                    tmem_ld32r(lane_addr + kColO + half * 64 + 32, b);
                    tmem_wait_ld(a);
                    tmem_tie(b);
                    if (half == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&S.o_empty);
                    }
                    if (valid) {
#pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8) {
                            const uint32_t *r = c8 < 4 ? a + 8 * c8 : b + 8 * (c8 - 4);
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float lo = __uint_as_float(r[2 * e]);
                                const float hi = __uint_as_float(r[2 * e + 1]);
                                fits = fits && fabsf(lo) <= P.acc_limit && fabsf(hi) <= P.acc_limit;
                                pk[e] = pack_f16x2(lo, hi);
                            }
                            *reinterpret_cast<uint4 *>(stage + ((half * 8 + c8) * kG + h) * 16) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
                if (valid && !fits) {
                    // Too large for the fp16 sum (or not finite): add zeros and
                    // leave this (row, head) to the exact pass.
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        *reinterpret_cast<uint4 *>(stage + (c * kG + h) * 16) = make_uint4(0, 0, 0, 0);
                    P.flags[row * P.H_q + x.g * kG + h] = 1;
                    atomicAdd(P.flag_count, 1);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (issuer) {
#pragma unroll
                    for (int r4 = 0; r4 < 4; ++r4) {
                        if (!dst4[r4]) continue;
                        if (MODE == 0) bulk_s2g(dst4[r4], stage0 + r4 * 2048, 2048);
                        else bulk_s2g_add_f16(dst4[r4], stage0 + r4 * 2048, 2048);
                    }
                    bulk_commit();
                }
            }
            x = xn;
        }
        // Staging must stay valid, and the adds land, before the CTA ends.
        if (issuer) bulk_wait_all();
        __syncwarp();
        if (!ok) *abort_flag = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- helpers
// Buckets of one (sequence, group, row range), built by one CTA: rows that
// kept block j (j != own) are counted, given offsets in the range's own
// region of bucket_rows, split into work items of <= item_rows rows, and
// scattered.  No grid-wide scan: each range owns fixed slices of the arrays.
constexpr int kBuildThreads = 512;

// Counters and cursors live in shared memory when nb_max <= this (64 KiB),
// else in the workspace.
constexpr int kBuildSmemBlocks = 8192;

__global__ void __launch_bounds__(kBuildThreads) bucket_build_kernel(const PrefillArgs P) {
    __shared__ int warp_c[kBuildThreads / 32], warp_i[kBuildThreads / 32];
    __shared__ int carry_c, carry_i;
    extern __shared__ int build_smem[];             // [2][nb_max] when it fits
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const long long r = blockIdx.x;
    const int rng = static_cast<int>(r % P.n_ranges);
    const int g = static_cast<int>((r / P.n_ranges) % P.H_kv);
    const int b = static_cast<int>(r / (static_cast<long long>(P.n_ranges) * P.H_kv));
    int L;
    if (!seq_ok(P, b, L)) {
        if (tid == 0) P.range_count[r] = 0;
        return;
    }
    const int i0 = rng * P.rows_per_range, i1 = min(P.Sq, i0 + P.rows_per_range);
    const long long n_e = static_cast<long long>(i1 - i0) * P.K;
    const bool in_smem = P.nb_max <= kBuildSmemBlocks;
    int *cnt = in_smem ? build_smem : P.bucket_cnt + r * P.nb_max;
    int *cur = in_smem ? build_smem + P.nb_max : P.bucket_cur + r * P.nb_max;
    if (in_smem) {
        for (int j = tid; j < 2 * P.nb_max; j += kBuildThreads) build_smem[j] = 0;
        __syncthreads();
    }
    const int32_t *ids = P.ids;
    auto entry = [&](long long e, long long &row) -> int {
        const int i = i0 + static_cast<int>(e / P.K);
        const int slot = static_cast<int>(e % P.K);
        row = static_cast<long long>(b) * P.Sq + i;
        const int j = ids[(row * P.n_idx + g / (P.H_kv / P.n_idx)) * P.K + slot];
        const long long p = static_cast<long long>(L) - P.Sq + i;
        return (j >= 0 && j < p / 128) ? j : -1;   // padding, own block, or out of range
    };
    for (long long e = tid; e < n_e; e += kBuildThreads) {
        long long row;
        const int j = entry(e, row);
        if (j >= 0) atomicAdd(cnt + j, 1);
    }
    if (tid == 0) { carry_c = 0; carry_i = 0; }
    __syncthreads();
    // Exclusive scans of row counts and item counts over j, 512 at a time.
    const long long region = r * static_cast<long long>(P.rows_per_range) * (P.K > 1 ? P.K - 1 : 1);
    for (int base = 0; base < P.nb_max; base += kBuildThreads) {
        const int j = base + tid;
        const int c = j < P.nb_max ? cnt[j] : 0;
        const int ni = (c + P.item_rows - 1) / P.item_rows;
        int ic = c, ii = ni;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int tc = __shfl_up_sync(0xffffffffu, ic, o), ti = __shfl_up_sync(0xffffffffu, ii, o);
            if (lane >= o) { ic += tc; ii += ti; }
        }
        if (lane == 31) { warp_c[wid] = ic; warp_i[wid] = ii; }
        __syncthreads();
        int pc = carry_c, pi = carry_i;
        for (int w = 0; w < wid; ++w) { pc += warp_c[w]; pi += warp_i[w]; }
        const int ex_c = pc + ic - c, ex_i = pi + ii - ni;
        if (j < P.nb_max) {
            const long long bk = r * P.nb_max + j;
            if (in_smem) P.bucket_cnt[bk] = c;       // read by item_table_kernel
            P.bucket_off[bk] = static_cast<int>(region + ex_c);
            P.item_off[bk] = ex_i;
            for (int q = 0; q < ni; ++q) P.item_bucket[r * P.items_per_range + ex_i + q] = j;
        }
        __syncthreads();
        if (tid == kBuildThreads - 1) { carry_c = ex_c + c; carry_i = ex_i + ni; }
        __syncthreads();
    }
    if (tid == 0) P.range_count[r] = carry_i;
    __syncthreads();
    __syncthreads();
    for (long long e = tid; e < n_e; e += kBuildThreads) {
        long long row;
        const int j = entry(e, row);
        if (j < 0) continue;
        const int pos = atomicAdd(cur + j, 1);
        P.bucket_rows[P.bucket_off[r * P.nb_max + j] + pos] = static_cast<int>(row);
    }
}

// Exclusive scan of the ranges' item counts -> global item numbering.
__global__ void __launch_bounds__(1024) range_scan_kernel(const PrefillArgs P) {
    __shared__ long long part[1024];
    const int tid = threadIdx.x;
    const long long n = P.n_ranges_total;
    const long long per = (n + 1023) / 1024;
    const long long lo = min(n, tid * per), hi = min(n, lo + per);
    long long sum = 0;
    for (long long k = lo; k < hi; ++k) sum += P.range_count[k];
    part[tid] = sum;
    __syncthreads();
    if (tid == 0) {
        long long a = 0;
        for (int t = 0; t < 1024; ++t) {
            const long long v = part[t];
            part[t] = a;
            a += v;
        }
        P.range_item_off[n] = a;
        *P.item_total = a;
    }
    __syncthreads();
    long long a = part[tid];
    for (long long k = lo; k < hi; ++k) {
        P.range_item_off[k] = a;
        a += P.range_count[k];
    }
}

// Flat table of pass-B work items: the descriptor of global item
// range_item_off[r] + li, for every range r and local item li, so that an item
// is decoded with one 32-byte load.  One CTA per range.
__global__ void item_table_kernel(const PrefillArgs P) {
    const long long r = blockIdx.x;
    const long long n = P.range_count[r];
    if (n == 0) return;                        // also every range of a rejected sequence
    const int g = static_cast<int>((r / P.n_ranges) % P.H_kv);
    const int b = static_cast<int>(r / (static_cast<long long>(P.n_ranges) * P.H_kv));
    const int L = P.lens[b];
    const long long base = P.range_item_off[r];
    for (long long li = threadIdx.x; li < n; li += blockDim.x) {
        const int j = P.item_bucket[r * P.items_per_range + li];
        const long long bk = r * P.nb_max + j;
        const int chunk = static_cast<int>(li) - P.item_off[bk];
        const int cnt = P.bucket_cnt[bk];
        int4 *d = reinterpret_cast<int4 *>(P.item_desc) + 2 * (base + li);
        d[0] = make_int4(b, g, j, min(P.item_rows, cnt - chunk * P.item_rows));
        d[1] = make_int4(P.bucket_off[bk] + chunk * P.item_rows, L, 0, 0);
    }
}

// The shift of every (bucket entry, head), copied from the per-(row, head)
// shifts once pass A and the fix-up have set them: pass B then reads a tile's
// shifts as one contiguous 512-byte run.  Two threads per entry (4 heads each).
__global__ void bucket_shift_kernel(const PrefillArgs P) {
    const long long total = *P.item_total * (kItemRows * 2);
    const int4 *desc = reinterpret_cast<const int4 *>(P.item_desc);
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long it = t / (kItemRows * 2);
        const int rr = static_cast<int>((t >> 1) % kItemRows), half = static_cast<int>(t & 1);
        const int4 a = desc[2 * it];            // b, g, j, n
        if (rr >= a.w) continue;
        const long long e = desc[2 * it + 1].x + rr;
        const long long row = P.bucket_rows[e];
        const float4 v = *reinterpret_cast<const float4 *>(P.m_arr + row * P.H_q + a.y * kG + half * 4);
        *reinterpret_cast<float4 *>(P.bucket_shift + e * kG + half * 4) = v;
    }
}

// out = accumulator / sum, bf16.  A thread takes 16-byte chunks of the fp16
// accumulator (8 dims of one head) in order, four at a time, so every warp
// reads 2 KiB contiguous and the loads of four chunks are in flight at once.
__global__ void __launch_bounds__(256) finalize_kernel(const PrefillArgs P) {
    const long long pairs = static_cast<long long>(P.B) * P.Sq * P.H_kv;
    const long long chunks = pairs * (kDim * kG / 8);        // 128 chunks per (row, group)
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const uint4 *acc = reinterpret_cast<const uint4 *>(P.o_acc);
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(P.out);
    for (long long c0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c0 < chunks;
         c0 += 4 * stride) {
        uint4 v[4];
        float l[4];
        bool ok[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const long long c = c0 + u * stride;
            ok[u] = c < chunks;
            if (!ok[u]) continue;
            const long long pair = c >> 7;
            const int q = static_cast<int>(c & 127), h = q & 7;
            const long long row = pair / P.H_kv;
            const int g = static_cast<int>(pair % P.H_kv);
            v[u] = acc[c];
            l[u] = P.l_acc[row * P.H_q + g * kG + h];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (!ok[u]) continue;
            const long long c = c0 + u * stride;
            const long long pair = c >> 7;
            const int q = static_cast<int>(c & 127), h = q & 7, cd = q >> 3;
            const long long row = pair / P.H_kv;
            const int g = static_cast<int>(pair % P.H_kv);
            const int b = static_cast<int>(row / P.Sq);
            int L;
            uint4 o;
            if (!seq_ok(P, b, L)) {
                const uint32_t nan2 = pack_bf16x2(NAN, NAN);
                o = make_uint4(nan2, nan2, nan2, nan2);
                if (P.lse && cd == 0) P.lse[row * P.H_q + g * kG + h] = NAN;
                // once per sequence: its first row's first chunk
                if (q == 0 && g == 0 && row == static_cast<long long>(b) * P.Sq)
                    set_status(P.status, kStatusBadLens);
            } else {
                const float inv = 1.f / l[u];
                if (P.lse && cd == 0)
                    P.lse[row * P.H_q + g * kG + h] = P.m_arr[row * P.H_q + g * kG + h] + log2f(l[u]);
                const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w4[e]));
                    o4[e] = pack_bf16x2(f.x * inv, f.y * inv);
                }
                o = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
            *reinterpret_cast<uint4 *>(out + (row * P.H_q + g * kG + h) * kDim + cd * 8) = o;
        }
    }
}

// Flagged (row, head) pairs (a partial too large for the fp16 sum): softmax
// over every kept key of the row, in fp32 on CUDA cores, written over the
// finalized output.  Exits at once when nothing was flagged.  One warp per
// (row, group); per flagged head a lane owns 4 output dims, each key's logit
// is a warp-reduced dot product.
__global__ void exact_rows_kernel(const PrefillArgs P) {
    if (*P.flag_count == 0) return;
    const int lane = threadIdx.x & 31;
    const long long total = static_cast<long long>(P.B) * P.Sq * P.H_kv;
    const float sl2 = P.softmax_scale * kLog2e;
    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(P.q);
    const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(P.k_cache);
    const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(P.v_cache);
    for (long long pair = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
         pair < total; pair += (static_cast<long long>(gridDim.x) * blockDim.x) >> 5) {
        const long long row = pair / P.H_kv;
        const int g = static_cast<int>(pair % P.H_kv);
        const int b = static_cast<int>(row / P.Sq), i = static_cast<int>(row % P.Sq);
        int L;
        if (!seq_ok(P, b, L)) continue;
        const long long p = static_cast<long long>(L) - P.Sq + i;
        const int own = static_cast<int>(p / 128);
        const int32_t *ids = P.ids + (row * P.n_idx + g / (P.H_kv / P.n_idx)) * P.K;
        for (int h = 0; h < kG; ++h) {
            const long long idx = row * P.H_q + g * kG + h;
            if (!P.flags[idx]) continue;
            float q4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) q4[e] = __bfloat162float(qb[idx * kDim + lane * 4 + e]);
            // logit of token t (row0 = first cache row of its block), warp-reduced
            auto logit = [&](long long krow) -> float {
                const __nv_bfloat16 *kt = kb + (krow * P.H_kv + g) * kDim + lane * 4;
                float d = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) d = fmaf(q4[e], __bfloat162float(kt[e]), d);
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                return d * sl2;
            };
            float mx = -INFINITY;
            for (int s = 0; s < P.K; ++s) {
                const int j = ids[s];
                if (j < 0 || j > own) continue;
                const long long row0 = kv_block_row(P.kv, b, j, P.status);
                const int nt = j == own ? static_cast<int>(p - 128LL * own) + 1 : 128;
                for (int t = 0; t < nt; ++t) mx = fmaxf(mx, logit(row0 + t));
            }
            float l = 0.f, o4[4] = {0.f, 0.f, 0.f, 0.f};
            for (int s = 0; s < P.K; ++s) {
                const int j = ids[s];
                if (j < 0 || j > own) continue;
                const long long row0 = kv_block_row(P.kv, b, j, P.status);
                const int nt = j == own ? static_cast<int>(p - 128LL * own) + 1 : 128;
                for (int t = 0; t < nt; ++t) {
                    const float w = exp2f(logit(row0 + t) - mx);
                    l += w;
                    const __nv_bfloat16 *vt = vb + ((row0 + t) * P.H_kv + g) * kDim + lane * 4;
#pragma unroll
                    for (int e = 0; e < 4; ++e) o4[e] = fmaf(w, __bfloat162float(vt[e]), o4[e]);
                }
            }
            __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(P.out) + idx * kDim + lane * 4;
            const float inv = 1.f / l;
            const uint2 wv = make_uint2(pack_bf16x2(o4[0] * inv, o4[1] * inv),
                                        pack_bf16x2(o4[2] * inv, o4[3] * inv));
            *reinterpret_cast<uint2 *>(out) = wv;
            if (P.lse && lane == 0) P.lse[idx] = mx + log2f(l);
        }
    }
}

template <int MODE>
cudaError_t launch_pass(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                        const PrefillArgs &a, cudaStream_t s, const char *name) {
    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope trace(s, name);
    attn_prefill_kernel<MODE><<<device_sm_count(), kThreads, smem, s>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

cudaError_t run_buckets(const PrefillArgs &a, const PrefillLayout &L, cudaStream_t s, const char *name) {
    TraceScope t(s, name);
    const size_t bsm = L.nb_max <= kBuildSmemBlocks ? static_cast<size_t>(2 * L.nb_max) * sizeof(int) : 0;
    cudaError_t e;
    if (bsm > 48 * 1024 &&
        (e = cudaFuncSetAttribute(bucket_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(bsm))) != cudaSuccess)
        return e;
    bucket_build_kernel<<<static_cast<unsigned>(L.n_ranges_total), kBuildThreads, bsm, s>>>(a);
    range_scan_kernel<<<1, 1024, 0, s>>>(a);
    item_table_kernel<<<static_cast<unsigned>(L.n_ranges_total), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool prefill_attention_supported(int H_q, int H_kv) { return H_q / H_kv == kG; }

size_t prefill_bucket_layout(int B, int Sq, int H_kv, int K, int max_kv_len, int item_rows,
                             int range_rows, size_t base, PrefillLayout *L) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    *L = PrefillLayout{};
    L->nb_max = (max_kv_len + 127) / 128;
    L->n_ranges = (Sq + range_rows - 1) / range_rows;
    L->n_ranges_total = static_cast<long long>(B) * H_kv * L->n_ranges;
    L->rows_per_range = Sq < range_rows ? Sq : range_rows;
    L->n_buckets = L->n_ranges_total * L->nb_max;
    const size_t per_range_rows = static_cast<size_t>(L->rows_per_range) * (K > 1 ? K - 1 : 1);
    L->item_rows = item_rows;
    L->items_per_range = static_cast<int>(L->nb_max + per_range_rows / item_rows + 1);
    size_t o = base;
    L->cnt = o;          o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->cur = o;          o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->zero_end = o;
    L->off = o;          o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->item_off = o;     o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->item_bucket = o;  o += up(static_cast<size_t>(L->n_ranges_total) * L->items_per_range * 4);
    L->range_count = o;  o += up(static_cast<size_t>(L->n_ranges_total) * 8);
    L->range_item_off = o; o += up(static_cast<size_t>(L->n_ranges_total + 1) * 8);
    L->rows = o;         o += up(static_cast<size_t>(L->n_ranges_total) * per_range_rows * 4);
    L->item_desc = o;    o += up(static_cast<size_t>(L->n_ranges_total) * L->items_per_range * 32);
    L->total = o;
    return o;
}

cudaError_t launch_prefill_buckets(PrefillArgs &a, uint8_t *ws, const PrefillLayout &L,
                                   long long *item_total, cudaStream_t s) {
    a.bucket_cnt = reinterpret_cast<int *>(ws + L.cnt);
    a.bucket_cur = reinterpret_cast<int *>(ws + L.cur);
    a.bucket_off = reinterpret_cast<int *>(ws + L.off);
    a.item_off = reinterpret_cast<int *>(ws + L.item_off);
    a.item_bucket = reinterpret_cast<int *>(ws + L.item_bucket);
    a.range_count = reinterpret_cast<long long *>(ws + L.range_count);
    a.range_item_off = reinterpret_cast<long long *>(ws + L.range_item_off);
    a.bucket_rows = reinterpret_cast<int *>(ws + L.rows);
    a.item_desc = reinterpret_cast<int *>(ws + L.item_desc);
    a.item_total = item_total;
    a.nb_max = L.nb_max;
    a.n_ranges = L.n_ranges;
    a.n_ranges_total = L.n_ranges_total;
    a.rows_per_range = L.rows_per_range;
    a.items_per_range = L.items_per_range;
    a.item_rows = L.item_rows;
    cudaError_t e = cudaMemsetAsync(ws + L.cnt, 0, L.zero_end - L.cnt, s);
    if (e != cudaSuccess) return e;
    return run_buckets(a, L, s, "backward_bucket");
}

size_t prefill_workspace_layout(int B, int Sq, int H_q, int H_kv, int K, int max_kv_len,
                                PrefillLayout *L) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const long long rows = static_cast<long long>(B) * Sq;
    L->nb_max = (max_kv_len + 127) / 128;
    L->n_ranges = (Sq + kRange - 1) / kRange;
    L->n_ranges_total = static_cast<long long>(B) * H_kv * L->n_ranges;
    L->rows_per_range = Sq < kRange ? Sq : kRange;
    L->n_buckets = L->n_ranges_total * L->nb_max;
    const size_t per_range_rows = static_cast<size_t>(L->rows_per_range) * (K > 1 ? K - 1 : 1);
    L->item_rows = kItemRows;
    L->items_per_range = static_cast<int>(L->nb_max + per_range_rows / kItemRows + 1);
    size_t o = kWsHeaderBytes;
    L->cnt = o;          o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->cur = o;          o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->l_acc = o;        o += up(static_cast<size_t>(rows) * H_q * 4);
    L->flags = o;        o += up(static_cast<size_t>(rows) * H_q);
    L->zero_end = o;                                  // [cnt, zero_end) is cleared per call
    L->off = o;          o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->item_off = o;     o += up(static_cast<size_t>(L->n_buckets) * 4);
    L->item_bucket = o;  o += up(static_cast<size_t>(L->n_ranges_total) * L->items_per_range * 4);
    L->range_count = o;  o += up(static_cast<size_t>(L->n_ranges_total) * 8);
    L->range_item_off = o; o += up(static_cast<size_t>(L->n_ranges_total + 1) * 8);
    L->rows = o;         o += up(static_cast<size_t>(L->n_ranges_total) * per_range_rows * 4);
    L->shift = o;        o += up(static_cast<size_t>(L->n_ranges_total) * per_range_rows * kG * 4);
    L->item_desc = o;    o += up(static_cast<size_t>(L->n_ranges_total) * L->items_per_range * 32);
    L->o_acc = o;        o += up(static_cast<size_t>(rows) * H_q * kDim * 2);
    L->m_arr = o;        o += up(static_cast<size_t>(rows) * H_q * 4);
    L->total = o;
    return o;
}

cudaError_t launch_prefill_attention(const PrefillArgs &a0, uint8_t *ws, const PrefillLayout &L,
                                     cudaStream_t s) {
    PrefillArgs a = a0;
    a.bucket_cnt = reinterpret_cast<int *>(ws + L.cnt);
    a.bucket_cur = reinterpret_cast<int *>(ws + L.cur);
    a.bucket_off = reinterpret_cast<int *>(ws + L.off);
    a.item_off = reinterpret_cast<int *>(ws + L.item_off);
    a.item_bucket = reinterpret_cast<int *>(ws + L.item_bucket);
    a.range_count = reinterpret_cast<long long *>(ws + L.range_count);
    a.range_item_off = reinterpret_cast<long long *>(ws + L.range_item_off);
    a.bucket_rows = reinterpret_cast<int *>(ws + L.rows);
    a.bucket_shift = reinterpret_cast<float *>(ws + L.shift);
    a.item_desc = reinterpret_cast<int *>(ws + L.item_desc);
    a.o_acc = reinterpret_cast<__half *>(ws + L.o_acc);
    a.l_acc = reinterpret_cast<float *>(ws + L.l_acc);
    a.m_arr = reinterpret_cast<float *>(ws + L.m_arr);
    a.flags = reinterpret_cast<uint8_t *>(ws + L.flags);
    a.flag_count = reinterpret_cast<int *>(ws + 4);
    a.item_total = reinterpret_cast<long long *>(ws + 8);
    a.item_next = reinterpret_cast<long long *>(ws + 16);   // [pass A, pass B]
    a.acc_limit = 65504.f / static_cast<float>(a.K > 0 ? a.K : 1);
    a.nb_max = L.nb_max;
    a.n_ranges = L.n_ranges;
    a.n_ranges_total = L.n_ranges_total;
    a.rows_per_range = L.rows_per_range;
    a.items_per_range = L.items_per_range;
    a.item_rows = L.item_rows;

    CUtensorMap tq, tk, tv;
    if (!encode_q_rows_map(&tq, a.q, a.H_q, static_cast<long long>(a.B) * a.Sq, kTileRows) ||
        !encode_kv_tensor_map(&tk, a.k_cache, a.H_kv, a.kv.capacity) ||
        !encode_kv_tensor_map(&tv, a.v_cache, a.H_kv, a.kv.capacity))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(ws + L.cnt, 0, L.zero_end - L.cnt, s);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    if ((e = run_buckets(a, L, s, "prefill_bucket")) != cudaSuccess) return e;
    if ((e = launch_pass<0>(tq, tk, tv, a, s, "prefill_attn_own_block")) != cudaSuccess) return e;
    {
        TraceScope t(s, "prefill_bucket_shift");
        bucket_shift_kernel<<<sms * 8, 256, 0, s>>>(a);
    }
    if ((e = launch_pass<1>(tq, tk, tv, a, s, "prefill_attn_kv_outer")) != cudaSuccess) return e;
    {
        TraceScope t(s, "prefill_finalize");
        finalize_kernel<<<sms * 16, 256, 0, s>>>(a);
    }
    {
        TraceScope t(s, "prefill_exact_rows");
        exact_rows_kernel<<<sms * 4, 256, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace msa
