// attn_bwd.cu -- backward of the MSA sparse branch (dQ, dK, dV over the kept
// blocks) on the fifth-generation tensor cores, organised around the KV
// blocks.
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 (exact attention over the kept blocks) and
// section 五 (MSA is trained natively).  The index branch's selection is
// piecewise constant, so only the sparse branch carries gradient.  For one
// (row, head) over its kept keys t, with P = softmax(scale q.k) and O the
// forward output:
//   dP_t = dO.v_t,  Delta = sum_t P_t dP_t = dO.O,  dS_t = P_t (dP_t - Delta),
//   dQ = scale sum_t dS_t k_t,  dK_t += scale dS_t q,  dV_t += P_t dO.
//
// Passes on one stream (the first is launched by the API entry point):
//   forward   the sparse branch's forward, recomputed, which also writes the
//             base-2 log-sum-exp of every (row, head)
//   prep      Delta = dO.O per (row, head); clears the fp32 dQ accumulator
//   buckets   rows that kept block j (j != own) as work items, built by the
//             forward's prefill bucket kernels (the forward's own items when
//             it ran the block-outer prefill path: groups of 8)
//   main      per work item -- one key block j of one (sequence, group) and
//             the rows that use it -- K_j and V_j are loaded once; per tile of
//             128/G rows x G heads = 128 (row, head) pairs:
//               S^T  = K_j Q^T                     tokens x pairs, TMEM
//               dP^T = V_j dO^T                    tokens x pairs, TMEM
//               P^T  = 2^(S^T scale log2 e - lse)  bf16, back into S^T's columns
//               dS^T = scale P^T (dP^T - Delta)    bf16, shared memory
//               dV  += P^T dO                      A from TMEM, summed over the item
//               dQ^T = K_j^T dS^T                  dims x pairs
//               dK^T += Q^T dS                     dims x tokens, summed over the item
//             (dQ and dK are formed transposed so that a warp's reduction
//             covers 32 consecutive dims of one row: whole 128-byte lines).
//             dQ of each tile is added to the accumulator with fp32
//             reductions; dK and dV leave TMEM once per item, not once per
//             (row, block); the next tile's S^T is issued ahead of the
//             current tile's dQ and dK
//   finalize  dq = accumulator, bf16
// The own block of each row is processed as items of the consecutive rows
// whose own block it is (causal mask); every product is tcgen05.mma
// kind::f16 with M = N = 128 (eight K = 16 steps), 40 MMAs per tile.
//
// Roles (512 threads): warp 0 lane 0 claims items and loads K_j and V_j by
// TMA; warp 1 lane 0 issues the MMAs; warps 2-3 gather each tile's Q and dO
// rows and statistics with cp.async (zero-filled past the item's rows);
// warps 4-11 compute P and dS, two warps per TMEM lane quarter with 64 pair
// columns each; warps 12-15 drain dQ per tile and dK, dV per item.  TMEM
// columns: S^T / P^T 0-127, dP^T / dQ^T 128-255, dV 256-383, dK^T 384-511.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 512;
constexpr int kLoaderWarps = 2;
constexpr int kSoftWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kEpiWarp0 = 4 + kSoftWarps;   // first epilogue warp
constexpr int kTilesPerItem = 16;           // bucket items hold up to 16 tiles of rows
#ifndef MSA_BWD_RANGE_ROWS
#define MSA_BWD_RANGE_ROWS 8192
#endif
// Bucket items are claimed range by range; a range's Q, dO and dQ
// accumulator rows (8 KiB per row and group) should stay in L2 meanwhile.
constexpr int kRangeRows = MSA_BWD_RANGE_ROWS;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kQueue = 4;
// MMA thread + one per loader, softmax and epilogue warp
constexpr int kQueueReaders = 1 + kLoaderWarps + kSoftWarps + kEpiWarps;

// A work item: key block j of one (sequence, group) and the rows that use it.
// Own items: the rows whose own block is j, consecutive from query row i_lo.
// Bucket items: entries rows_off .. rows_off + n - 1 of bucket_rows.
struct BItem {
    int b, g, j, n;         // n = rows; 0: nothing to do; < 0: no more work
    int i_lo, rows_off, L, own;
};

struct Smem {
    uint8_t kv[65536];                 // K lo, K hi, V lo, V hi: 128 tokens x 64 dims each
    uint8_t qdo[2][65536];             // per tile: Q lo, Q hi, dO lo, dO hi (128 pairs x 64 dims)
    uint8_t ds[32768];                 // dS^T: 128 tokens x 64 pairs, two halves
    float lse[2][128], dlt[2][128];    // per tile: each pair's log-sum-exp and Delta
    uint64_t kv_full, kv_empty, kv_ready;
    uint64_t qdo_full[2], qdo_empty[2];
    uint64_t s_full, dp_full, p_ready, dv_done, ds_ready, ds_empty, dq_full, dq_empty;
    uint64_t acc_full, acc_empty;
    uint64_t item_full[kQueue], item_empty[kQueue];
    BItem item_q[kQueue];
    uint32_t tmem_base;
    int abort_flag;
};
// Every buffer sits at a multiple of 1 KiB from the start (128-byte swizzle).
constexpr size_t kSmemLimit = 232448;
static_assert(sizeof(Smem) <= kSmemLimit, "shared memory over the per-block limit");

__device__ __forceinline__ bool seq_ok(const AttnBwdArgs &P, int b, int &L) {
    L = P.lens[b];
    return L >= P.Sq && L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
}

__device__ __forceinline__ long long n_own_items(const AttnBwdArgs &P) {
    return static_cast<long long>(P.B) * P.H_kv * ((P.Sq + 127) / 128 + 1);
}

// Items 0 .. n_own-1 are own-block items, one per (sequence, group, block the
// rows span); the rest are the bucket items.
__device__ BItem item_at(const AttnBwdArgs &P, long long it, long long n_own) {
    BItem x;
    x.i_lo = 0;
    x.rows_off = 0;
    x.own = 0;
    x.L = 0;
    if (it < n_own) {
        const int nj = (P.Sq + 127) / 128 + 1;
        x.own = 1;
        x.b = static_cast<int>(it / (static_cast<long long>(P.H_kv) * nj));
        const int rem = static_cast<int>(it % (static_cast<long long>(P.H_kv) * nj));
        x.g = rem / nj;
        x.j = 0;
        if (!seq_ok(P, x.b, x.L)) { x.n = 0; return x; }
        const long long p0 = static_cast<long long>(x.L) - P.Sq;      // position of row 0
        x.j = static_cast<int>(p0 / 128) + rem % nj;
        const long long plo = max(p0, static_cast<long long>(x.j) * 128);
        const long long phi = min(static_cast<long long>(x.L), static_cast<long long>(x.j) * 128 + 128);
        x.n = phi > plo ? static_cast<int>(phi - plo) : 0;
        x.i_lo = static_cast<int>(plo - p0);
    } else {
        const int4 *d = reinterpret_cast<const int4 *>(P.item_desc) + 2 * (it - n_own);
        const int4 a = d[0], c = d[1];
        x.b = a.x; x.g = a.y; x.j = a.z; x.n = a.w;
        x.rows_off = c.x; x.L = c.y;
    }
    return x;
}

// Flattened row (b * Sq + i) of row r of the item.
__device__ __forceinline__ long long item_row(const AttnBwdArgs &P, const BItem &x, int r) {
    return x.own ? static_cast<long long>(x.b) * P.Sq + x.i_lo + r
                 : static_cast<long long>(P.bucket_rows[x.rows_off + r]);
}

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Start-address step of K-major operand k-step kk (16 elements): four steps
// per 64-element swizzle atom, the next atom 16 KiB further.
__device__ __forceinline__ uint64_t kstep(int kk) {
    return static_cast<uint64_t>((kk >> 2) * 1024 + (kk & 3) * 2);
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void red_add_v4(float *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(__uint_as_float(a)),
                 "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
                 : "memory");
}

// 16-byte copy, or 16 zero bytes when !valid (nothing is read then).
__device__ __forceinline__ void cp_async16_zfill(uint32_t sdst, const void *gsrc, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sdst), "l"(gsrc),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_zfill(uint32_t sdst, const void *gsrc, bool valid) {
    if constexpr (N == 16) {
        cp_async16_zfill(sdst, gsrc, valid);
    } else {
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(sdst), "l"(gsrc), "n"(N),
                     "r"(valid ? N : 0)
                     : "memory");
    }
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const AttnBwdArgs P, uint32_t smem_bytes) {
    constexpr int TR = 128 / G;          // query rows per tile
    extern __shared__ uint8_t smem_raw[];
    const uintptr_t sbase = (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023);
    if (sbase + sizeof(Smem) > reinterpret_cast<uintptr_t>(smem_raw) + smem_bytes) {
        // The dynamic shared memory does not start on a 1 KiB boundary and
        // the 128-byte-swizzled buffers do not fit: nothing is computed.
        if (threadIdx.x == 0) set_status(P.status, kStatusTimeout);
        return;
    }
    Smem &S = *reinterpret_cast<Smem *>(sbase);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long n_own = n_own_items(P);
    const long long total = n_own + *P.item_total;

    if (tid == 0) {
        mbar_init(&S.kv_full, 1);
        mbar_init(&S.kv_empty, 1);
        mbar_init(&S.kv_ready, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.qdo_full[i], kLoaderWarps * 32);   // one hardware arrival per loader thread
            mbar_init(&S.qdo_empty[i], 1);
        }
        mbar_init(&S.s_full, 1);
        mbar_init(&S.dp_full, 1);
        mbar_init(&S.p_ready, kSoftWarps);
        mbar_init(&S.dv_done, 1);
        mbar_init(&S.ds_ready, kSoftWarps);
        mbar_init(&S.ds_empty, 1);
        mbar_init(&S.dq_full, 1);
        mbar_init(&S.dq_empty, kEpiWarps);
        mbar_init(&S.acc_full, 1);
        mbar_init(&S.acc_empty, kEpiWarps);
        for (int i = 0; i < kQueue; ++i) {
            mbar_init(&S.item_full[i], 1);
            mbar_init(&S.item_empty[i], kQueueReaders);
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

    // n-th item for a reader, decoded by the producer; false on abort.
    auto next_item = [&](int n, bool warp_reader, BItem &x) -> bool {
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
        // ------------------------------------------------ producer (lane 0)
        // Claims items in order from one global counter (neighbouring items
        // share a row range, so its dQ accumulator rows stay in L2), publishes
        // them, and loads each item's K and V block.  In a sequence's last,
        // partial block the key rows past its length may hold anything (the
        // padding of a cache); their dS is 0, but 0 * NaN is NaN in dQ = dS K,
        // so they are zeroed before the MMAs read them (kv_ready).
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            int ki = 0, last_issued = -1;
            bool ok = true;
            for (int n = 0; ok; ++n) {
                const int slot = n % kQueue;
                if (n >= kQueue &&
                    (*abort_flag || !mbar_wait(&S.item_empty[slot], ((n / kQueue) - 1) & 1, P.status))) {
                    ok = false;
                    break;
                }
                const long long it = static_cast<long long>(
                    atomicAdd(reinterpret_cast<unsigned long long *>(P.item_next), 1ull));
                BItem x;
                if (it >= total) x.n = -1;
                else x = item_at(P, it, n_own);
                S.item_q[slot] = x;
                mbar_arrive(&S.item_full[slot]);
                if (x.n < 0) break;
                if (x.n == 0) continue;
                if (ki >= 1 && (*abort_flag || !mbar_wait(&S.kv_empty, (ki - 1) & 1, P.status))) {
                    ok = false;
                    break;
                }
                const int tok = static_cast<int>(kv_block_row(P.kv, x.b, x.j, P.status));
                mbar_arrive_expect_tx(&S.kv_full, 65536);
                tma_load_3d(S.kv, &tmK, 0, x.g, tok, &S.kv_full);
                tma_load_3d(S.kv + 16384, &tmK, 64, x.g, tok, &S.kv_full);
                tma_load_3d(S.kv + 32768, &tmV, 0, x.g, tok, &S.kv_full);
                tma_load_3d(S.kv + 49152, &tmV, 64, x.g, tok, &S.kv_full);
                last_issued = ki;
                const int nvalid = x.L - x.j * 128;      // tokens of the block inside the sequence
                if (nvalid < 128) {
                    if (*abort_flag || !mbar_wait(&S.kv_full, ki & 1, P.status)) {
                        ok = false;
                        break;
                    }
                    for (int e = nvalid * 16; e < 128 * 16; ++e) {   // 16-byte pieces, both halves
                        const int r = e >> 4, c = e & 15;
                        *reinterpret_cast<uint4 *>(S.kv + (c >> 3) * 16384 + r * 128 + (c & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                mbar_arrive(&S.kv_ready);
                ++ki;
            }
            if (!ok) *abort_flag = 1;
            // The last K/V copy lands before the CTA can end, abort or not.
            if (last_issued >= 0) mbar_wait(&S.kv_full, last_issued & 1, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (lane 0)
        if (lane == 0) {
            const uint32_t id_kk = umma_idesc_bf16(128, 128);            // A, B K-major
            const uint32_t id_kb = id_kk | (1u << 16);                   // B MN-major
            const uint32_t id_mk = id_kk | (1u << 15);                   // A MN-major
            const uint32_t id_mm = id_kk | (1u << 15) | (1u << 16);      // A and B MN-major
            const uint32_t kv0 = smem_u32(S.kv), ds0 = smem_u32(S.ds);
            // Descriptors are built once; a k-step only moves the start address.
            const uint64_t k_kd = umma_desc(kv0, 16, 1024);              // K_j: tokens x dims
            const uint64_t k_mn = umma_desc(kv0, 16384, 1024);           // K_j^T: dims x tokens, transposed read
            const uint64_t v_kd = umma_desc(kv0 + 32768, 16, 1024);      // V_j: tokens x dims
            const uint64_t ds_kd = umma_desc(ds0, 16, 1024);             // dS: tokens (N) x pairs (K)
            const uint64_t ds_mn = umma_desc(ds0, 16384, 1024);          // dS^T: tokens (K) x pairs (N)
            // Stage 1's descriptors are stage 0's moved by 64 KiB (4096 16-byte units).
            const uint32_t qa = smem_u32(S.qdo[0]);
            const uint64_t q_kd0 = umma_desc(qa, 16, 1024), q_mn0 = umma_desc(qa, 16384, 1024);
            const uint64_t do_kd0 = umma_desc(qa + 32768, 16, 1024);
            const uint64_t do_mn0 = umma_desc(qa + 32768, 16384, 1024);
            int ki = 0, qt = 0;
            bool ok = true;
            auto wait = [&](uint64_t *bar, int parity) -> bool {
                return !*abort_flag && mbar_wait(bar, static_cast<uint32_t>(parity), P.status);
            };
            for (int n = 0; ok; ++n) {
                BItem x;
                if (!next_item(n, false, x)) { ok = false; break; }
                if (x.n < 0) break;
                if (x.n == 0) continue;
                if (!wait(&S.kv_full, ki & 1) || !wait(&S.kv_ready, ki & 1)) { ok = false; break; }
                const int ntile = (x.n + TR - 1) / TR;
                // S^T of tile q (Q from stage q & 1).  S^T's columns hold the
                // previous tile's P^T until that tile's dV is done.
                auto issue_s = [&](int q) -> bool {
                    const int sq = q & 1;
                    if (!wait(&S.qdo_full[sq], (q >> 1) & 1)) return false;
                    fence_proxy_async_smem();            // Q, dO rows were written by cp.async
                    if (q >= 1 && !wait(&S.dv_done, (q - 1) & 1)) return false;
                    tc_fence_after();
                    const uint64_t qk = q_kd0 + static_cast<uint64_t>(sq * 4096);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16_ss(tmem + kColS, k_kd + kstep(kk), qk + kstep(kk), id_kk, kk > 0 ? 1u : 0u);
                    umma_commit(&S.s_full);
                    return true;
                };
                if (!issue_s(qt)) { ok = false; break; }
                for (int t = 0; t < ntile; ++t, ++qt) {
                    const int st = qt & 1;
                    const uint64_t so = static_cast<uint64_t>(st * 4096);
                    const uint64_t q_mn = q_mn0 + so, do_kd = do_kd0 + so, do_mn = do_mn0 + so;
                    // dP^T's columns hold the previous tile's dQ^T until the epilogue has read it.
                    if (qt >= 1 && !wait(&S.dq_empty, (qt - 1) & 1)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16_ss(tmem + kColDP, v_kd + kstep(kk), do_kd + kstep(kk), id_kk, kk > 0 ? 1u : 0u);
                    umma_commit(&S.dp_full);
                    if (!wait(&S.p_ready, qt & 1)) { ok = false; break; }
                    // dV and dK restart with each item, once the last ones left TMEM.
                    if (t == 0 && ki >= 1 && !wait(&S.acc_empty, (ki - 1) & 1)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {     // P^T pairs 16kk..: columns 0-31 and 64-95
                        const uint32_t pa = tmem + kColS + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8);
                        umma_bf16_ts(tmem + kColDV, pa, do_mn + static_cast<uint64_t>(kk * 128), id_kb,
                                     (t > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&S.dv_done);
                    // The next tile's S^T goes ahead of this tile's dQ and dK, so
                    // the softmax warps start on it while those two run.
                    if (t + 1 < ntile && !issue_s(qt + 1)) { ok = false; break; }
                    if (!wait(&S.ds_ready, qt & 1)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)        // dQ^T = K_j^T dS^T, into dP^T's columns
                        umma_bf16_ss(tmem + kColDP, k_mn + static_cast<uint64_t>(kk * 128),
                                     ds_mn + static_cast<uint64_t>(kk * 128), id_mm, kk > 0 ? 1u : 0u);
                    umma_commit(&S.dq_full);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)        // dK^T += Q^T dS
                        umma_bf16_ss(tmem + kColDK, q_mn + static_cast<uint64_t>(kk * 128), ds_kd + kstep(kk),
                                     id_mk, (t > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&S.ds_empty);
                    umma_commit(&S.qdo_empty[st]);
                    if (t == ntile - 1) {
                        umma_commit(&S.acc_full);
                        umma_commit(&S.kv_empty);
                    }
                }
                ++ki;
            }
            if (!ok) *abort_flag = 1;
            // Every MMA issued must finish before TMEM is released.
            if (qt > 0) mbar_wait(&S.ds_empty, (qt - 1) & 1, nullptr);
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------ Q / dO / statistics loaders
        // Warp lw takes tile rows lw, lw + 2, ...; each (row, group) slice of Q
        // (and of dO) is G x 256 bytes, copied in 16-byte pieces straight into
        // the 128-byte-swizzled layout the MMAs read (pair m = row x G + head,
        // dims 0-63 then 64-127 in two halves).  Rows past the item's end are
        // zero-filled: their dS is 0, and 0 times stale data must not be NaN.
        const int lw = warp - 2;
        constexpr int CPR = 16 * G;                       // 16-byte pieces per slice
        constexpr int RPI = CPR >= 32 ? 1 : 32 / CPR;     // slices per warp step
        constexpr int CPL = CPR >= 32 ? CPR / 32 : 1;     // pieces per lane and slice
        constexpr int SB = 4 * G < 16 ? 4 * G : 16;       // statistics copy size
        constexpr int NSC = 4 * G / SB;                   // copies per row, each of lse and Delta
        int qt = 0, n = 0;
        bool ok = true;
        BItem x;
        while (ok) {
            if (!next_item(n++, true, x)) { ok = false; break; }
            if (x.n < 0) break;
            if (x.n == 0) continue;
            const int ntile = (x.n + TR - 1) / TR;
            for (int t = 0; t < ntile; ++t, ++qt) {
                const int st = qt & 1;
                long long rowv[2];                        // rows of slots k = lane, lane + 32
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int k = lane + 32 * u, r = t * TR + lw + 2 * k;
                    rowv[u] = (k < TR / 2 && r < x.n) ? item_row(P, x, r) : -1;
                }
                bool free_ = qt < 2 || (!*abort_flag && mbar_wait(&S.qdo_empty[st], ((qt >> 1) - 1) & 1, P.status));
                free_ = __all_sync(0xffffffffu, free_);
                if (!free_) { ok = false; break; }
                const uint32_t qb = smem_u32(S.qdo[st]);
                const int li = RPI > 1 ? lane % CPR : lane;   // lane within its slice
#pragma unroll 1
                for (int k0 = 0; k0 < TR / 2; k0 += RPI) {
                    const int k = k0 + (RPI > 1 ? lane / CPR : 0);
                    const long long row = __shfl_sync(0xffffffffu, k0 < 32 ? rowv[0] : rowv[1], k & 31);
                    const int rr = lw + 2 * k;            // tile row
                    const bool valid = row >= 0;
                    const long long pr = valid ? row * P.H_q + static_cast<long long>(x.g) * G : 0;
                    const uint8_t *qsrc = static_cast<const uint8_t *>(P.q) + pr * (kDim * 2);
                    const uint8_t *dsrc = static_cast<const uint8_t *>(P.dout) + pr * (kDim * 2);
#pragma unroll
                    for (int cq = 0; cq < CPL; ++cq) {
                        const int pc = li + 32 * cq;       // piece of the slice
                        const int hh = pc >> 4, c = pc & 15, m = rr * G + hh;
                        const uint32_t off = (c >> 3) * 16384 + m * 128 + (((c & 7) ^ (m & 7)) << 4);
                        cp_async16_zfill(qb + off, qsrc + (valid ? pc * 16 : 0), valid);
                        cp_async16_zfill(qb + 32768 + off, dsrc + (valid ? pc * 16 : 0), valid);
                    }
                    if (li < 2 * NSC) {
                        const bool isd = li >= NSC;
                        const int ci = isd ? li - NSC : li;
                        float *dstf = (isd ? S.dlt[st] : S.lse[st]) + rr * G + ci * (SB / 4);
                        const float *srcf = (isd ? P.delta : P.lse) + (valid ? pr + ci * (SB / 4) : 0);
                        cp_async_zfill<SB>(smem_u32(dstf), srcf, valid);
                    }
                }
                // Each thread's arrival fires once its copies have landed.
                cp_async_arrive_noinc(&S.qdo_full[st]);
            }
        }
        cp_async_wait_all();                              // nothing lands after the CTA ends
        if (!ok) *abort_flag = 1;
    } else if (warp >= 4 && warp < kEpiWarp0) {
        // ------------------------------------------------ P and dS
        // Warps 4-7 and 8-11 share the TMEM lanes of warp % 4 (lane = token
        // of the block) and split the 128 pair columns: ch = 0 takes pairs
        // 0-63, ch = 1 pairs 64-127.  P^T goes back to TMEM as bf16 pairs
        // over the warp's own first 32 columns of S^T (already read), where
        // the dV product takes it as its A operand; dS^T goes to shared
        // memory, row = token, half ch, 128-byte swizzle.
        const int ch = (warp - 4) >> 2;
        const int tok = (warp & 3) * 32 + lane;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const float sl2 = P.softmax_scale * kLog2e;
        const float scale = P.softmax_scale;
        uint8_t *ds_row = S.ds + ch * 16384 + tok * 128;
        int qt = 0, n = 0;
        bool ok = true;
        BItem x;
        auto wait_all = [&](uint64_t *bar, int parity) -> bool {
            const bool w = !*abort_flag && mbar_wait(bar, static_cast<uint32_t>(parity), P.status);
            return __all_sync(0xffffffffu, w);
        };
        while (ok) {
            if (!next_item(n++, true, x)) { ok = false; break; }
            if (x.n < 0) break;
            if (x.n == 0) continue;
            const int ntile = (x.n + TR - 1) / TR;
            for (int t = 0; t < ntile; ++t, ++qt) {
                const int st = qt & 1;
                const int nv = min(TR, x.n - t * TR);          // rows of this tile
                // Own items: token tok is visible to tile row r iff tok <= lim0 + r.
                const int lim0 = x.own ? (x.L - P.Sq + x.i_lo + t * TR) - x.j * 128 : (1 << 30);
                const bool masked = x.own || nv < TR;
                auto vis = [&](int c) -> bool {
                    const int r = c / G;
                    return r < nv && tok <= lim0 + r;
                };
                // The tile's statistics came with its Q rows (cp.async).
                if (!wait_all(&S.qdo_full[st], (qt >> 1) & 1)) { ok = false; break; }
                if (!wait_all(&S.s_full, qt & 1)) { ok = false; break; }
                tc_fence_after();
                uint32_t a[32], b[32];
                tmem_ld32r(lane_addr + kColS + ch * 64, a);
                tmem_ld32r(lane_addr + kColS + ch * 64 + 32, b);
                tmem_wait_ld(a);
                tmem_tie(b);
                const float *ls = S.lse[st] + ch * 64;
                uint32_t pk[32];                             // P of the 64 columns as bf16 pairs
#pragma unroll
                for (int e4 = 0; e4 < 16; ++e4) {
                    const float4 l4 = *reinterpret_cast<const float4 *>(ls + 4 * e4);
                    const uint32_t *src = e4 < 8 ? a : b;
                    const int k = (4 * e4) & 31;
                    float p0 = fast_exp2(fmaf(__uint_as_float(src[k]), sl2, -l4.x));
                    float p1 = fast_exp2(fmaf(__uint_as_float(src[k + 1]), sl2, -l4.y));
                    float p2 = fast_exp2(fmaf(__uint_as_float(src[k + 2]), sl2, -l4.z));
                    float p3 = fast_exp2(fmaf(__uint_as_float(src[k + 3]), sl2, -l4.w));
                    if (masked) {
                        const int c = ch * 64 + 4 * e4;
                        p0 = vis(c) ? p0 : 0.f;
                        p1 = vis(c + 1) ? p1 : 0.f;
                        p2 = vis(c + 2) ? p2 : 0.f;
                        p3 = vis(c + 3) ? p3 : 0.f;
                    }
                    pk[2 * e4] = pack_bf16x2(p0, p1);
                    pk[2 * e4 + 1] = pack_bf16x2(p2, p3);
                }
                tmem_st32(lane_addr + kColS + ch * 64, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.p_ready);

                if (!wait_all(&S.dp_full, qt & 1)) { ok = false; break; }
                tc_fence_after();
                tmem_ld32r(lane_addr + kColDP + ch * 64, a);
                tmem_ld32r(lane_addr + kColDP + ch * 64 + 32, b);
                tmem_wait_ld(a);
                tmem_tie(b);
                // The dS buffer is free once the previous tile's dQ and dK read it.
                if (qt >= 1 && !wait_all(&S.ds_empty, (qt - 1) & 1)) { ok = false; break; }
                const float *dl = S.dlt[st] + ch * 64;
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {                 // 8 pairs -> one 16-byte piece
                    uint32_t wv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int cc = c8 * 8 + 2 * e;            // column within the half
                        const uint32_t *src = cc < 32 ? a : b;
                        const int k = cc & 31;
                        const uint32_t pw = pk[cc >> 1];
                        const float2 dd = *reinterpret_cast<const float2 *>(dl + cc);
                        const float p0 = bf16lo(pw), p1 = bf16hi(pw);
                        float d0 = (p0 * scale) * (__uint_as_float(src[k]) - dd.x);
                        float d1 = (p1 * scale) * (__uint_as_float(src[k + 1]) - dd.y);
                        if (masked) {           // dP may be NaN where a key row is padding
                            d0 = p0 != 0.f ? d0 : 0.f;
                            d1 = p1 != 0.f ? d1 : 0.f;
                        }
                        wv[e] = pack_bf16x2(d0, d1);
                    }
                    *reinterpret_cast<uint4 *>(ds_row + ((c8 ^ (tok & 7)) << 4)) =
                        make_uint4(wv[0], wv[1], wv[2], wv[3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.ds_ready);
            }
        }
        if (!ok) *abort_flag = 1;
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------ epilogue
        // dQ^T (per tile) and dK^T (per item) have lane = dim, column = pair
        // or token: each column's 32 dims of a warp leave as one coalesced
        // 128-byte fp32 reduction (a full line; 16-byte pieces of separate
        // rows would each cost a whole 32-byte sector operation at L2).  dV
        // (per item) has lane = token and goes out as 16-byte vector
        // reductions along its row.  Pair p = tile row p / G, head p % G.
        constexpr int NRR = (TR + 31) / 32;                  // tile rows per lane
        const int w = warp & 3;
        const int d = w * 32 + lane;                          // dim (dQ^T, dK^T) or token (dV)
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(w * 32) << 16);
        int qt = 0, ki = 0, n = 0;
        bool ok = true;
        BItem x;
        auto wait_all = [&](uint64_t *bar, int parity) -> bool {
            const bool wt = !*abort_flag && mbar_wait(bar, static_cast<uint32_t>(parity), P.status);
            return __all_sync(0xffffffffu, wt);
        };
        auto red_row = [](float *dst, const uint32_t(&v)[32]) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) red_add_v4(dst + e, v[e], v[e + 1], v[e + 2], v[e + 3]);
        };
        // Accumulator row bases of tile rows lane, lane + 32, ... (0: no row).
        auto row_bases = [&](const BItem &it, int t, unsigned long long (&rb)[NRR]) {
#pragma unroll
            for (int i = 0; i < NRR; ++i) {
                const int rr = lane + 32 * i;
                rb[i] = 0;
                if (rr < TR && t * TR + rr < it.n)
                    rb[i] = reinterpret_cast<unsigned long long>(
                        P.dq_acc + (item_row(P, it, t * TR + rr) * P.H_q + static_cast<long long>(it.g) * G) * kDim);
            }
        };
        while (ok) {
            if (!next_item(n++, true, x)) { ok = false; break; }
            if (x.n < 0) break;
            if (x.n == 0) continue;
            const int ntile = (x.n + TR - 1) / TR;
            unsigned long long rb_nx[NRR];
            row_bases(x, 0, rb_nx);
            for (int t = 0; t < ntile; ++t, ++qt) {
                unsigned long long rb[NRR];
#pragma unroll
                for (int i = 0; i < NRR; ++i) rb[i] = rb_nx[i];
                if (t + 1 < ntile) row_bases(x, t + 1, rb_nx);
                if (!wait_all(&S.dq_full, qt & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t a[32], b[32];
                    tmem_ld32r(lane_addr + kColDP + half * 64, a);
                    tmem_ld32r(lane_addr + kColDP + half * 64 + 32, b);
                    tmem_wait_ld(a);
                    tmem_tie(b);
                    if (half == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&S.dq_empty);
                    }
#pragma unroll
                    for (int r2 = 0; r2 < 64 / G; ++r2) {        // the half's tile rows
                        const int rr = half * (64 / G) + r2;
                        const unsigned long long base = __shfl_sync(0xffffffffu, rb[rr / 32], rr % 32);
                        if (!base) continue;
                        float *dst = reinterpret_cast<float *>(base) + d;
#pragma unroll
                        for (int hh = 0; hh < G; ++hh) {
                            const int e = r2 * G + hh;
                            asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst + hh * kDim),
                                         "f"(__uint_as_float(e < 32 ? a[e] : b[e - 32]))
                                         : "memory");
                        }
                    }
                }
            }
            if (!ok) break;
            if (!wait_all(&S.acc_full, ki & 1)) { ok = false; break; }
            tc_fence_after();
            const long long trow0 = kv_block_row(P.kv, x.b, x.j, P.status);
            const int nvalid = x.L - x.j * 128;             // tokens inside the sequence
            {   // dV: lane = token d of the block
                float *dvp = P.dv + ((trow0 + d) * P.H_kv + x.g) * kDim;
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t a[32], b[32];
                    tmem_ld32r(lane_addr + kColDV + hf * 64, a);
                    tmem_ld32r(lane_addr + kColDV + hf * 64 + 32, b);
                    tmem_wait_ld(a);
                    tmem_tie(b);
                    if (d < nvalid) { red_row(dvp + hf * 64, a); red_row(dvp + hf * 64 + 32, b); }
                }
            }
            // dK^T: lane = dim d, column = token
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t a[32], b[32];
                tmem_ld32r(lane_addr + kColDK + hf * 64, a);
                tmem_ld32r(lane_addr + kColDK + hf * 64 + 32, b);
                tmem_wait_ld(a);
                tmem_tie(b);
                if (hf == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.acc_empty);
                }
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const int tk = hf * 64 + e;
                    if (tk < nvalid) {
                        float *dst = P.dk + ((trow0 + tk) * P.H_kv + x.g) * kDim + d;
                        asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst),
                                     "f"(__uint_as_float(e < 32 ? a[e] : b[e - 32]))
                                     : "memory");
                    }
                }
            }
            ++ki;
        }
        if (!ok) *abort_flag = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Delta = dO . O per (row, head), from the recomputed bf16 output, and the
// dQ accumulator cleared.  16 threads per (row, head), 8 dims each.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const AttnBwdArgs P) {
    const long long total = static_cast<long long>(P.B) * P.Sq * P.H_q * 16;
    const long long bound = (total + 31) & ~31LL;              // whole warps iterate together
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const uint4 *o = static_cast<const uint4 *>(P.o);
    const uint4 *d = static_cast<const uint4 *>(P.dout);
    float4 *acc = reinterpret_cast<float4 *>(P.dq_acc);
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < bound;
         t += stride) {
        float s = 0.f;
        if (t < total) {
            const uint4 ov = o[t], dv = d[t];
            const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                s = fmaf(bf16lo(ow[e]), bf16lo(dw[e]), fmaf(bf16hi(ow[e]), bf16hi(dw[e]), s));
            acc[2 * t] = make_float4(0.f, 0.f, 0.f, 0.f);
            acc[2 * t + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        s += __shfl_xor_sync(0xffffffffu, s, 8);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if (t < total && (t & 15) == 0) P.delta[t >> 4] = s;
    }
}

// dq = accumulator in bf16; NaN for sequences with bad lengths and after a
// wait gave up.
__global__ void __launch_bounds__(256) dq_finalize_kernel(const AttnBwdArgs P) {
    const bool aborted = (*reinterpret_cast<volatile const int *>(P.status) & kStatusTimeout) != 0;
    const long long total = static_cast<long long>(P.B) * P.Sq * P.H_q * 16;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const float4 *acc = reinterpret_cast<const float4 *>(P.dq_acc);
    uint4 *dq = static_cast<uint4 *>(P.dq);
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += stride) {
        const long long row = (t >> 4) / P.H_q;
        int L;
        uint4 v;
        if (aborted || !seq_ok(P, static_cast<int>(row / P.Sq), L)) {
            const uint32_t nan2 = pack_bf16x2(NAN, NAN);
            v = make_uint4(nan2, nan2, nan2, nan2);
        } else {
            const float4 x0 = acc[2 * t], x1 = acc[2 * t + 1];
            v = make_uint4(pack_bf16x2(x0.x, x0.y), pack_bf16x2(x0.z, x0.w), pack_bf16x2(x1.x, x1.y),
                           pack_bf16x2(x1.z, x1.w));
        }
        dq[t] = v;
    }
}

template <int G>
cudaError_t launch_blocks(const CUtensorMap &tk, const CUtensorMap &tv, const AttnBwdArgs &a,
                          cudaStream_t s) {
    // All of the opt-in shared memory: the buffers plus slack to align them.
    const uint32_t smem = static_cast<uint32_t>(kSmemLimit);
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    TraceScope t(s, "backward_blocks");
    attn_bwd_kernel<G><<<device_sm_count(), kThreads, smem, s>>>(tk, tv, a, smem);
    return cudaGetLastError();
}

}  // namespace

size_t attn_bwd_layout(int B, int Sq, int H_q, int H_kv, int K, int max_kv_len, size_t base,
                       const PrefillLayout *fwd, AttnBwdLayout *L) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t pairs = static_cast<size_t>(B) * Sq * H_q;
    size_t o = up(base);
    L->o = o;       o += up(pairs * kDim * 2);
    L->lse = o;     o += up(pairs * 4);
    L->delta = o;   o += up(pairs * 4);
    L->dq_acc = o;  o += up(pairs * kDim * 4);
    const int G = H_q / H_kv;
    const int item_rows = kTilesPerItem * (128 / G);
    L->reuse = fwd && fwd->item_rows == item_rows && fwd->rows_per_range == (Sq < kRangeRows ? Sq : kRangeRows);
    L->fwd_rows = L->reuse ? fwd->rows : 0;
    L->fwd_desc = L->reuse ? fwd->item_desc : 0;
    L->bk = PrefillLayout{};
    if (!L->reuse)
        o = prefill_bucket_layout(B, Sq, H_kv, K, max_kv_len, item_rows, kRangeRows, o, &L->bk);
    L->total = o;
    return o;
}

cudaError_t launch_attn_bwd(const AttnBwdArgs &a0, uint8_t *ws, const AttnBwdLayout &L,
                            cudaStream_t s) {
    AttnBwdArgs a = a0;
    a.o = ws + L.o;
    a.lse = reinterpret_cast<const float *>(ws + L.lse);
    a.delta = reinterpret_cast<float *>(ws + L.delta);
    a.dq_acc = reinterpret_cast<float *>(ws + L.dq_acc);
    // header bytes 32..47: the item count and the claim counter of this pass
    long long *hdr = reinterpret_cast<long long *>(ws + 32);
    PrefillArgs pb{};
    pb.q = a.q; pb.k_cache = a.k_cache; pb.v_cache = a.v_cache; pb.ids = a.ids; pb.lens = a.lens;
    pb.kv = a.kv; pb.status = a.status;
    pb.B = a.B; pb.Sq = a.Sq; pb.H_q = a.H_q; pb.H_kv = a.H_kv; pb.K = a.K;
    pb.max_kv_len = a.max_kv_len; pb.n_idx = a.n_idx; pb.softmax_scale = a.softmax_scale;
    CUtensorMap tk, tv;
    if (!encode_kv_tensor_map(&tk, a.k_cache, a.H_kv, a.kv.capacity) ||
        !encode_kv_tensor_map(&tv, a.v_cache, a.H_kv, a.kv.capacity))
        return cudaErrorInvalidValue;
    const int sms = device_sm_count();
    {
        TraceScope t(s, "backward_prep");
        bwd_prep_kernel<<<sms * 8, 256, 0, s>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (L.reuse) {
        // the forward's bucket items (same rows per item and range): its
        // item count sits in header bytes 8..15
        a.bucket_rows = reinterpret_cast<const int *>(ws + L.fwd_rows);
        a.item_desc = reinterpret_cast<const int *>(ws + L.fwd_desc);
        a.item_total = reinterpret_cast<const long long *>(ws + 8);
    } else {
        if ((e = launch_prefill_buckets(pb, ws, L.bk, hdr, s)) != cudaSuccess) return e;
        a.bucket_rows = pb.bucket_rows;
        a.item_desc = pb.item_desc;
        a.item_total = hdr;
    }
    a.item_next = hdr + 1;
    switch (a.H_q / a.H_kv) {
    case 1: e = launch_blocks<1>(tk, tv, a, s); break;
    case 2: e = launch_blocks<2>(tk, tv, a, s); break;
    case 4: e = launch_blocks<4>(tk, tv, a, s); break;
    case 8: e = launch_blocks<8>(tk, tv, a, s); break;
    case 16: e = launch_blocks<16>(tk, tv, a, s); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    {
        TraceScope t(s, "backward_dq");
        dq_finalize_kernel<<<sms * 8, 256, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace msa
