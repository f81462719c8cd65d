// index_decode.cu -- MSA index branch for decode: stream every index key of
// every sequence once from HBM, dot it with the group's index query and
// max-pool the scores over 128-token blocks.
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 -- one index query per GQA group, "Block Max
// Pool" over KV blocks before the top-k; section 四 -- decode is memory bound.
//
// Design: a persistent grid, one CTA per SM.  A work unit is one 128-token
// block of one sequence for all H_kv groups (H_kv * 32 KiB of contiguous
// index keys).  Warp 8 is the producer: one thread streams the unit as
// 32 KiB bulk copies (cp.async.bulk, evict-first L2 policy) into a 6-stage
// shared-memory ring.  Warps 0-7 consume: 16 threads per (token, group) row,
// each dotting 8 dims held in registers, a 4-step butterfly to finish the
// dot, a running max per thread, and one cross-warp max per unit.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kStages = 6;
constexpr int kStageBytes = 32768;          // 128 (token, group) rows x 256 bytes
constexpr int kMaxBatch = 4096;

struct Smem {
    uint8_t ring[kStages][kStageBytes];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t idle;                 // never arrived on: the test stall waits here
    int prefix[kMaxBatch + 1];
    float red[2][16];
    int abort_flag;
};

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}

__device__ __forceinline__ bool seq_valid(const IndexDecodeArgs &P, int b, int L) {
    return L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
}

__global__ void __launch_bounds__(kThreads, 1) index_decode_kernel(const IndexDecodeArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int H = P.H_kv;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], kConsumerWarps);
        }
        mbar_init(&S.idle, 1);
        S.abort_flag = 0;
        fence_mbar_init();
    }
    // Units per sequence (0 for an invalid sequence), exclusive prefix in warp 0.
    if (warp == 0) {
        const int per = (P.B + 31) / 32;
        const int lo = lane * per, hi = min(P.B, lo + per);
        int sum = 0;
        for (int b = lo; b < hi; ++b) {
            const int L = P.lens[b];
            if (seq_valid(P, b, L)) sum += (L + kBlock - 1) / kBlock;
            else if (blockIdx.x == 0) set_status(P.status, kStatusBadLens);
        }
        int incl = sum;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, m);
            if (lane >= m) incl += o;
        }
        int run = incl - sum;
        for (int b = lo; b < hi; ++b) {
            S.prefix[b] = run;
            const int L = P.lens[b];
            if (seq_valid(P, b, L)) run += (L + kBlock - 1) / kBlock;
        }
        if (lane == 31) S.prefix[P.B] = incl;
    }
    __syncthreads();
    const int U = S.prefix[P.B];
    const int tps = 128 / H;   // tokens per stage: 128 (token, group) rows

    auto unit_of = [&](int u, int &b, int &j) {
        int lo = 0, hi = P.B;              // largest b with prefix[b] <= u (skips empty ones)
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (S.prefix[mid] <= u) lo = mid; else hi = mid;
        }
        b = lo;
        j = u - S.prefix[lo];
    };

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            const __nv_bfloat16 *kbase = static_cast<const __nv_bfloat16 *>(P.k_idx);
            int it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
                int b, j;
                unit_of(u, b, j);
                const int L = P.lens[b];
                const long long t_first = kv_block_row(P.kv, b, j, P.status);
                const int ntok = min(kBlock, L - j * kBlock);
                for (int t0 = 0; t0 < ntok; t0 += tps, ++it) {
                    const int nt = min(tps, ntok - t0);
                    const int slot = it % kStages;
                    if (it >= kStages) {
                        if (*(volatile int *)&S.abort_flag ||
                            !mbar_wait(&S.empty[slot], ((it / kStages) - 1) & 1, P.status)) {
                            *(volatile int *)&S.abort_flag = 1;
                            ok = false;
                            break;
                        }
                    }
                    const uint32_t bytes = static_cast<uint32_t>(nt) * H * kDim * 2;
                    mbar_arrive_expect_tx(&S.full[slot], bytes);
                    bulk_g2s(S.ring[slot], kbase + (t_first + t0) * H * kDim, bytes, &S.full[slot],
                             pol);
                }
            }
            // Drain: every copy already issued lands before this thread
            // exits (after an abort the consumers may not wait for them).
            for (int k = max(0, it - kStages); k < it; ++k)
                mbar_wait(&S.full[k % kStages], (k / kStages) & 1, nullptr);
        }
        return;
    }

    // ---------------------------------------------------- consumers
    const int c = tid & 15;          // 16-byte chunk of the 256-byte row
    const int r0 = tid >> 4;         // row slot 0..15 within a pass of 16 rows
    const int g = r0 % H;            // group of every row this thread touches
    float qf[8];
    int cur_b = -1;
    int it = 0, unit_iter = 0;
    const __nv_bfloat16 *qbase = static_cast<const __nv_bfloat16 *>(P.q_idx);
    // A test may ask the consumers to wait once on a barrier nobody arrives
    // on: the wait gives up after the call's limit and the CTA aborts.
    if (stall_mask(P.status) & kStallIndexDecode) {
        if (!mbar_wait(&S.idle, 0, P.status)) *(volatile int *)&S.abort_flag = 1;
    }

    for (int u = blockIdx.x; u < U; u += gridDim.x, ++unit_iter) {
        int b, j;
        unit_of(u, b, j);
        const int L = P.lens[b];
        const int ntok = min(kBlock, L - j * kBlock);
        if (b != cur_b) {
            const uint4 qv = *reinterpret_cast<const uint4 *>(qbase + ((long long)b * H + g) * kDim + c * 8);
            qf[0] = bf16lo(qv.x); qf[1] = bf16hi(qv.x);
            qf[2] = bf16lo(qv.y); qf[3] = bf16hi(qv.y);
            qf[4] = bf16lo(qv.z); qf[5] = bf16hi(qv.z);
            qf[6] = bf16lo(qv.w); qf[7] = bf16hi(qv.w);
            cur_b = b;
        }
        float runmax = -INFINITY;
        for (int t0 = 0; t0 < ntok; t0 += tps, ++it) {
            const int rows_valid = min(tps, ntok - t0) * H;
            const int slot = it % kStages;
            bool have = false;
            if (!*(volatile int *)&S.abort_flag)
                have = mbar_wait(&S.full[slot], (it / kStages) & 1, P.status);
            have = __all_sync(0xffffffffu, have);   // warp-uniform before the shuffles
            if (!have) *(volatile int *)&S.abort_flag = 1;
            if (have) {
                const uint8_t *sb = S.ring[slot];
#pragma unroll
                for (int pass = 0; pass < 8; ++pass) {
                    const int row = r0 + 16 * pass;
                    const uint4 kv = *reinterpret_cast<const uint4 *>(sb + row * 256 + c * 16);
                    float s = qf[0] * bf16lo(kv.x);
                    s = fmaf(qf[1], bf16hi(kv.x), s);
                    s = fmaf(qf[2], bf16lo(kv.y), s);
                    s = fmaf(qf[3], bf16hi(kv.y), s);
                    s = fmaf(qf[4], bf16lo(kv.z), s);
                    s = fmaf(qf[5], bf16hi(kv.z), s);
                    s = fmaf(qf[6], bf16lo(kv.w), s);
                    s = fmaf(qf[7], bf16hi(kv.w), s);
                    s += __shfl_xor_sync(0xffffffffu, s, 8);
                    s += __shfl_xor_sync(0xffffffffu, s, 4);
                    s += __shfl_xor_sync(0xffffffffu, s, 2);
                    s += __shfl_xor_sync(0xffffffffu, s, 1);
                    if (row < rows_valid) runmax = fmaxf(runmax, s);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.empty[slot]);
            }
        }
        // Max over the row slots that hold group g.
        const int par = unit_iter & 1;
        if (c == 0) S.red[par][r0] = runmax;
        consumers_sync();
        if (tid < H && !*(volatile int *)&S.abort_flag) {
            float m = -INFINITY;
            for (int r = tid; r < 16; r += H) m = fmaxf(m, S.red[par][r]);
            P.scores[((long long)b * H + tid) * P.nb_max + j] = m;
        }
    }
}

}  // namespace

cudaError_t launch_index_decode(const IndexDecodeArgs &a, cudaStream_t s) {
    static_assert(sizeof(Smem) <= 227 * 1024, "shared memory budget");
    const size_t smem = sizeof(Smem) + 1024;  // + alignment slack
    cudaError_t e = cudaFuncSetAttribute(index_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    TraceScope trace(s, "index_score_maxpool_decode");
    index_decode_kernel<<<device_sm_count(), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
