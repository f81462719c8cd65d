// index_decode_variants.cu -- MSA decode index branch on the other index-key
// formats: keys shared by every index head (bf16 or FP8 E4M3), and one FP8
// E4M3 key per index head.
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 -- index score, "Block Max Pool" over KV
// blocks, top-k; the index-head count comes from the mlqm.cn guide's
// configuration ("sparse_num_index_heads").  Shared and FP8 keys cut the
// bytes decode must stream (the article's section 四: decode is bound by
// memory traffic); E4M3 values are decoded exactly and scaled per key row.
//
// Shared keys: per 128-token block the scores of all H index heads are the
// product K (128 tokens x 128 dims) . Q^T (128 x H), a small dense
// contraction, run on the tensor cores with mma.sync (S^T = K Q^T, tokens on
// M, index heads on N = 8 or 16).  A persistent grid streams one block per
// stage.  bf16 keys (index_shared_kernel) arrive as two 128-byte-swizzled TMA
// tiles; eight consumer warps take 16 tokens each and combine their block
// maxima in shared memory.  E4M3 keys (index_shared_fp8_kernel) arrive as one
// 16 KiB bulk copy per block; each warp takes whole blocks, widening its A
// operand words to bf16 in registers (exact: every E4M3 value is a bf16
// value) and scaling each token's scores by its row scale.
//
// Per-head FP8 keys (index_fp8_kernel): one dot per (token, head) row, 128
// bytes, as in the bf16 per-head kernel but with 8 threads per row (16 E4M3
// values each, widened to fp32 through f16 pairs) and the row's scale.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kWarps = 8;                  // consumer warps
constexpr int kConsumers = kWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + producer warp
constexpr int kMaxBatch = 4096;

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}

__device__ __forceinline__ bool seq_valid(const IndexDecodeVarArgs &P, int b, int L) {
    return L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
}

// Two E4M3 codes (low byte first) -> two f16 values, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
    return r;
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t h) {
    float2 f;
    asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
        : "=f"(f.x), "=f"(f.y)
        : "r"(h));
    return f;
}

// Units (128-token blocks) per sequence, exclusive prefix in shared memory;
// invalid sequences get none and raise the status word.  Warp 0 only.
__device__ void unit_prefix(const IndexDecodeVarArgs &P, int *prefix, int lane) {
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
        prefix[b] = run;
        const int L = P.lens[b];
        if (seq_valid(P, b, L)) run += (L + kBlock - 1) / kBlock;
    }
    if (lane == 31) prefix[P.B] = incl;
}

// Largest b with prefix[b] <= u (skips sequences with no units).
__device__ __forceinline__ void unit_of(const int *prefix, int B, int u, int &b, int &j) {
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= u) lo = mid; else hi = mid;
    }
    b = lo;
    j = u - prefix[lo];
}

// ------------------------------------------------------------ shared keys
constexpr int kRingBytes = 131072;             // 4 bf16 stages of 32 KiB or 8 E4M3 stages of 16 KiB

struct SharedSmem {
    uint8_t ring[kRingBytes];
    uint64_t full[8], empty[8];
    int prefix[kMaxBatch + 1];
    float red[2][kWarps][16];                  // per-warp block maxima, double-buffered
    int abort_flag;
};

// E4M3 pair (low byte first) -> bf16 pair, exact (every E4M3 value is a bf16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t v) {
    const float2 f = f16x2_to_float2(e4m3x2_to_f16x2(v));
    return pack_bf16x2(f.x, f.y);
}

// Shared bf16 index keys: the A operand (16 tokens x 16 dims per step) comes
// from the swizzled TMA tile by ldmatrix.
template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    index_shared_kernel(const __grid_constant__ CUtensorMap tmK, const IndexDecodeVarArgs P) {
    constexpr int kStageBytes = 32768;
    constexpr int kStages = kRingBytes / kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    SharedSmem &S = *reinterpret_cast<SharedSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                    ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = P.H;
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], kWarps);
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) unit_prefix(P, S.prefix, lane);
    __syncthreads();
    const int U = S.prefix[P.B];

    if (warp == kWarps) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            int it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < U && ok; u += gridDim.x, ++it) {
                int b, j;
                unit_of(S.prefix, P.B, u, b, j);
                const int L = P.lens[b];
                const int ntok = min(kBlock, L - j * kBlock);
                const int slot = it % kStages;
                uint8_t *dst = S.ring + slot * kStageBytes;
                if (it >= kStages && (*(volatile int *)&S.abort_flag ||
                                      !mbar_wait(&S.empty[slot], ((it / kStages) - 1) & 1, P.status))) {
                    *(volatile int *)&S.abort_flag = 1;
                    ok = false;
                    break;
                }
                const long long row0 = kv_block_row(P.kv, b, j, P.status);
                // Rows past the cache's end read as zeros; rows past the
                // sequence's length are masked below.
                mbar_arrive_expect_tx(&S.full[slot], 32768);
                tma_load_3d(dst, &tmK, 0, 0, static_cast<int>(row0), &S.full[slot]);
                tma_load_3d(dst + 16384, &tmK, 64, 0, static_cast<int>(row0), &S.full[slot]);
            }
            if (!ok)
                for (int k = max(0, it - kStages); k < it; ++k)
                    mbar_wait(&S.full[k % kStages], (k / kStages) & 1, nullptr);
        }
        return;
    }

    // ---------------------------------------------------- consumers
    const int tok0 = warp * 16;                      // this warp's 16 tokens of the block
    const int gq = lane >> 2, tq = lane & 3;
    const __nv_bfloat16 *qbase = static_cast<const __nv_bfloat16 *>(P.q_idx);
    uint32_t qf[8][NT][2];                           // Q^T fragments of the current sequence
    int cur_b = -1;
    int it = 0;
    for (int u = blockIdx.x; u < U; u += gridDim.x, ++it) {
        int b, j;
        unit_of(S.prefix, P.B, u, b, j);
        const int L = P.lens[b];
        const int ntok = min(kBlock, L - j * kBlock);
        const long long row0 = kv_block_row(P.kv, b, j, P.status);
        if (b != cur_b) {
            // B operand: B[k][n] = q_idx[b][n][k]; heads past H are zero.
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int h = nt * 8 + gq;
                    const __nv_bfloat16 *qh = qbase + ((long long)b * H + h) * kDim + kk * 16 + tq * 2;
                    qf[kk][nt][0] = h < H ? *reinterpret_cast<const uint32_t *>(qh) : 0u;
                    qf[kk][nt][1] = h < H ? *reinterpret_cast<const uint32_t *>(qh + 8) : 0u;
                }
            cur_b = b;
        }
        const int slot = it % kStages;
        const uint8_t *stage = S.ring + slot * kStageBytes;
        bool have = false;
        if (!*(volatile int *)&S.abort_flag) have = mbar_wait(&S.full[slot], (it / kStages) & 1, P.status);
        have = __all_sync(0xffffffffu, have);
        if (!have) *(volatile int *)&S.abort_flag = 1;
        float m[NT][2];                              // per head column pair: max of the warp's tokens
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = -INFINITY;
        if (have) {
            float s[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
            const uint32_t kbase = smem_u32(stage);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int chunk = ((kk & 3) << 1) | (lane >> 4);
                const int r = tok0 + (lane & 15);
                uint32_t a[4];
                ldsm_x4(kbase + (kk >> 2) * 16384 + swz128(r, chunk), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.empty[slot]);
            // s[nt][0..1]: token tok0+gq, heads nt*8 + 2tq + {0,1}; s[nt][2..3]: token +8.
            const bool v0 = tok0 + gq < ntok, v1 = tok0 + gq + 8 < ntok;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const float a0 = v0 ? s[nt][c] : -INFINITY;
                    const float a1 = v1 ? s[nt][2 + c] : -INFINITY;
                    m[nt][c] = fmaxf(a0, a1);
                }
        }
        // Max over the warp's 16 tokens: lanes with the same tq hold the same heads.
        const int par = it & 1;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float v = m[nt][c];
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                if (gq == 0) S.red[par][warp][nt * 8 + 2 * tq + c] = v;
            }
        // One barrier per block: red[par] is next written two blocks later,
        // after every reader of this block has passed the next barrier.
        consumers_sync();
        if (tid < H && !*(volatile int *)&S.abort_flag) {
            float v = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v = fmaxf(v, S.red[par][w][tid]);
            P.scores[((long long)b * H + tid) * P.nb_max + j] = v;
        }
    }
}

// m16n8k16 with f16 operands and fp32 accumulation (products of two f16
// values are exact in fp32, as those of two bf16 values are).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared E4M3 keys, one block per consumer warp: the widening makes each block
// worth ~1000 instructions per warp, so blocks are not split across warps
// (no cross-warp reduction, no CTA barrier); the CTA's k-th block goes to
// stage k % 8 and warp k % 8, so eight blocks are in flight per SM.
// Every E4M3 value is an f16 value, so when a sequence's index queries are f16
// values too (bf16 values inside f16's range, checked per warp and sequence),
// the products run on f16 operands and each pair of codes costs one
// conversion; otherwise the codes are widened to bf16 (three more steps).
template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    index_shared_fp8_kernel(const IndexDecodeVarArgs P) {
    constexpr int kStageBytes = 16384;
    constexpr int kStages = kWarps;
    extern __shared__ uint8_t smem_raw[];
    SharedSmem &S = *reinterpret_cast<SharedSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                    ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = P.H;
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], 1);
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) unit_prefix(P, S.prefix, lane);
    __syncthreads();
    const int U = S.prefix[P.B];

    if (warp == kWarps) {
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            const uint8_t *k8 = static_cast<const uint8_t *>(P.k_idx);
            int it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < U && ok; u += gridDim.x, ++it) {
                int b, j;
                unit_of(S.prefix, P.B, u, b, j);
                const int ntok = min(kBlock, P.lens[b] - j * kBlock);
                const int slot = it % kStages;
                if (it >= kStages && (*(volatile int *)&S.abort_flag ||
                                      !mbar_wait(&S.empty[slot], ((it / kStages) - 1) & 1, P.status))) {
                    *(volatile int *)&S.abort_flag = 1;
                    ok = false;
                    break;
                }
                const long long row0 = kv_block_row(P.kv, b, j, P.status);
                const uint32_t bytes = static_cast<uint32_t>(ntok) * kDim;
                mbar_arrive_expect_tx(&S.full[slot], bytes);
                bulk_g2s(S.ring + slot * kStageBytes, k8 + row0 * kDim, bytes, &S.full[slot], pol);
            }
            if (!ok)
                for (int k = max(0, it - kStages); k < it; ++k)
                    mbar_wait(&S.full[k % kStages], (k / kStages) & 1, nullptr);
        }
        return;
    }

    const int gq = lane >> 2, tq = lane & 3;
    const __nv_bfloat16 *qbase = static_cast<const __nv_bfloat16 *>(P.q_idx);
    uint32_t qf[8][NT][2];
    uint32_t qh16[8][NT][2];                    // the same queries as f16 pairs
    bool f16ok = false;
    int cur_b = -1;
    for (int it = warp;; it += kWarps) {
        const long long uu = blockIdx.x + static_cast<long long>(it) * gridDim.x;
        if (uu >= U) break;
        int b, j;
        unit_of(S.prefix, P.B, static_cast<int>(uu), b, j);
        const int ntok = min(kBlock, P.lens[b] - j * kBlock);
        const long long row0 = kv_block_row(P.kv, b, j, P.status);
        if (b != cur_b) {
            // The dot product does not depend on the order of the dims, so
            // step kk of thread (g, c) takes dims 32c + 4kk .. +3 of its two
            // tokens -- one 32-bit word per token, widened in registers -- as
            // its k slots (2c, 2c+1, 2c+8, 2c+9); the Q^T fragment holds the
            // same dims in the same slots.
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int h = nt * 8 + gq;
                    const __nv_bfloat16 *qh = qbase + ((long long)b * H + h) * kDim + 32 * tq + 4 * kk;
                    qf[kk][nt][0] = h < H ? *reinterpret_cast<const uint32_t *>(qh) : 0u;
                    qf[kk][nt][1] = h < H ? *reinterpret_cast<const uint32_t *>(qh + 2) : 0u;
                }
            bool exact = true;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float lo = bf16lo(qf[kk][nt][e]), hi = bf16hi(qf[kk][nt][e]);
                        const __half2 h2 = __floats2half2_rn(lo, hi);
                        exact = exact && __low2float(h2) == lo && __high2float(h2) == hi;
                        qh16[kk][nt][e] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
            f16ok = __all_sync(0xffffffffu, exact);
            cur_b = b;
        }
        // Row scales of this thread's 16 tokens (2 per 16-token tile).
        float sc[8][2];
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int tok = t * 16 + gq + 8 * e;
                sc[t][e] = tok < ntok ? __ldg(P.k_scale + row0 + tok) : 0.f;
            }
        const int slot = it % kStages;
        bool have = false;
        if (!*(volatile int *)&S.abort_flag) have = mbar_wait(&S.full[slot], (it / kStages) & 1, P.status);
        have = __all_sync(0xffffffffu, have);
        if (!have) { *(volatile int *)&S.abort_flag = 1; break; }
        const uint8_t *stage = S.ring + slot * kStageBytes;
        float m[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = -INFINITY;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int tok = t * 16 + gq;
            const uint4 *r0 = reinterpret_cast<const uint4 *>(stage + tok * kDim + tq * 32);
            const uint4 *r1 = reinterpret_cast<const uint4 *>(stage + (tok + 8) * kDim + tq * 32);
            const uint4 x0 = r0[0], x1 = r0[1], y0 = r1[0], y1 = r1[1];
            const uint32_t w0[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            const uint32_t w1[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
            float s[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
            if (f16ok) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t a[4];
                    a[0] = e4m3x2_to_f16x2(static_cast<uint16_t>(w0[kk] & 0xFFFFu));
                    a[1] = e4m3x2_to_f16x2(static_cast<uint16_t>(w1[kk] & 0xFFFFu));
                    a[2] = e4m3x2_to_f16x2(static_cast<uint16_t>(w0[kk] >> 16));
                    a[3] = e4m3x2_to_f16x2(static_cast<uint16_t>(w1[kk] >> 16));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(s[nt], a, qh16[kk][nt][0], qh16[kk][nt][1]);
                }
            } else {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t a[4];
                    a[0] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w0[kk] & 0xFFFFu));
                    a[1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w1[kk] & 0xFFFFu));
                    a[2] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w0[kk] >> 16));
                    a[3] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w1[kk] >> 16));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
                }
            }
            // rows past the length hold stale bytes: masked here
            const bool v0 = tok < ntok, v1 = tok + 8 < ntok;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if (v0) m[nt][c] = fmaxf(m[nt][c], s[nt][c] * sc[t][0]);
                    if (v1) m[nt][c] = fmaxf(m[nt][c], s[nt][2 + c] * sc[t][1]);
                }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[slot]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float v = m[nt][c];
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                const int h = nt * 8 + 2 * tq + c;
                if (gq == 0 && h < H && !*(volatile int *)&S.abort_flag)
                    P.scores[((long long)b * H + h) * P.nb_max + j] = v;
            }
    }
}

// ------------------------------------------------------------ per-head E4M3
constexpr int kFStages = 6;
constexpr int kFStageBytes = 32768;                  // 256 (token, head) rows x 128 bytes

struct Fp8Smem {
    uint8_t ring[kFStages][kFStageBytes];
    uint64_t full[kFStages], empty[kFStages];
    int prefix[kMaxBatch + 1];
    float red[2][kWarps * 4][16];
    int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1) index_fp8_kernel(const IndexDecodeVarArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Fp8Smem &S = *reinterpret_cast<Fp8Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = P.H;
    if (tid == 0) {
        for (int i = 0; i < kFStages; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], kWarps);
        }
        S.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) unit_prefix(P, S.prefix, lane);
    __syncthreads();
    const int U = S.prefix[P.B];
    const int tps = 256 / H;                         // tokens per stage

    if (warp == kWarps) {
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            const uint8_t *k8 = static_cast<const uint8_t *>(P.k_idx);
            int it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
                int b, j;
                unit_of(S.prefix, P.B, u, b, j);
                const int L = P.lens[b];
                const long long t_first = kv_block_row(P.kv, b, j, P.status);
                const int ntok = min(kBlock, L - j * kBlock);
                for (int t0 = 0; t0 < ntok; t0 += tps, ++it) {
                    const int nt = min(tps, ntok - t0);
                    const int slot = it % kFStages;
                    if (it >= kFStages && (*(volatile int *)&S.abort_flag ||
                                           !mbar_wait(&S.empty[slot], ((it / kFStages) - 1) & 1, P.status))) {
                        *(volatile int *)&S.abort_flag = 1;
                        ok = false;
                        break;
                    }
                    const uint32_t bytes = static_cast<uint32_t>(nt) * H * kDim;
                    mbar_arrive_expect_tx(&S.full[slot], bytes);
                    bulk_g2s(S.ring[slot], k8 + (t_first + t0) * H * kDim, bytes, &S.full[slot], pol);
                }
            }
            if (!ok)
                for (int k = max(0, it - kFStages); k < it; ++k)
                    mbar_wait(&S.full[k % kFStages], (k / kFStages) & 1, nullptr);
        }
        return;
    }

    // Consumers: 8 threads per 128-byte (token, head) row, 16 codes each;
    // 32 rows per pass, 8 passes per stage.
    const int c = tid & 7;
    const int r0 = tid >> 3;                         // 0..31
    const int g = r0 % H;                            // head of every row this thread touches
    float qf[16];
    int cur_b = -1;
    int it = 0, unit_iter = 0;
    const __nv_bfloat16 *qbase = static_cast<const __nv_bfloat16 *>(P.q_idx);
    for (int u = blockIdx.x; u < U; u += gridDim.x, ++unit_iter) {
        int b, j;
        unit_of(S.prefix, P.B, u, b, j);
        const int L = P.lens[b];
        const int ntok = min(kBlock, L - j * kBlock);
        const long long t_first = kv_block_row(P.kv, b, j, P.status);
        if (b != cur_b) {
            const uint4 *q4 = reinterpret_cast<const uint4 *>(qbase + ((long long)b * H + g) * kDim + c * 16);
            const uint4 qa = q4[0], qb = q4[1];
            const uint32_t w[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) { qf[2 * e] = bf16lo(w[e]); qf[2 * e + 1] = bf16hi(w[e]); }
            cur_b = b;
        }
        float runmax = -INFINITY;
        for (int t0 = 0; t0 < ntok; t0 += tps, ++it) {
            const int rows_valid = min(tps, ntok - t0) * H;
            const int slot = it % kFStages;
            // scales of this thread's rows (token-major, head-minor like the keys)
            float scl[8];
#pragma unroll
            for (int pass = 0; pass < 8; ++pass) {
                const int row = r0 + 32 * pass;
                scl[pass] = row < rows_valid ? __ldg(P.k_scale + (t_first + t0) * H + row) : 0.f;
            }
            bool have = false;
            if (!*(volatile int *)&S.abort_flag) have = mbar_wait(&S.full[slot], (it / kFStages) & 1, P.status);
            have = __all_sync(0xffffffffu, have);
            if (!have) *(volatile int *)&S.abort_flag = 1;
            if (have) {
                const uint8_t *sb = S.ring[slot];
#pragma unroll
                for (int pass = 0; pass < 8; ++pass) {
                    const int row = r0 + 32 * pass;
                    const uint4 kv = *reinterpret_cast<const uint4 *>(sb + row * kDim + c * 16);
                    const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
                    float s = 0.f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f0 = f16x2_to_float2(e4m3x2_to_f16x2(static_cast<uint16_t>(w[q] & 0xFFFFu)));
                        const float2 f1 = f16x2_to_float2(e4m3x2_to_f16x2(static_cast<uint16_t>(w[q] >> 16)));
                        s = fmaf(qf[4 * q], f0.x, s);
                        s = fmaf(qf[4 * q + 1], f0.y, s);
                        s = fmaf(qf[4 * q + 2], f1.x, s);
                        s = fmaf(qf[4 * q + 3], f1.y, s);
                    }
                    s += __shfl_xor_sync(0xffffffffu, s, 4);
                    s += __shfl_xor_sync(0xffffffffu, s, 2);
                    s += __shfl_xor_sync(0xffffffffu, s, 1);
                    if (row < rows_valid) runmax = fmaxf(runmax, s * scl[pass]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.empty[slot]);
            }
        }
        const int par = unit_iter & 1;
        if (c == 0) S.red[par][r0][0] = runmax;
        consumers_sync();
        if (tid < H && !*(volatile int *)&S.abort_flag) {
            float m = -INFINITY;
            for (int r = tid; r < 32; r += H) m = fmaxf(m, S.red[par][r][0]);
            P.scores[((long long)b * H + tid) * P.nb_max + j] = m;
        }
    }
}

}  // namespace

cudaError_t launch_index_decode_variant(const IndexDecodeVarArgs &a, cudaStream_t s) {
    TraceScope trace(s, "index_score_maxpool_decode_variant");
    if (a.KH == 1) {
        static_assert(sizeof(SharedSmem) + 1024 <= 232448, "shared memory budget");
        CUtensorMap tk;
        memset(&tk, 0, sizeof tk);
        if (!a.fp8 && !encode_kv_tensor_map(&tk, a.k_idx, 1, a.kv.capacity)) return cudaErrorInvalidValue;
        const size_t smem = sizeof(SharedSmem) + 1024;
        auto launch = [&](auto kern) -> cudaError_t {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            kern<<<device_sm_count(), kThreads, smem, s>>>(tk, a);
            return cudaGetLastError();
        };
        auto launch8 = [&](auto kern) -> cudaError_t {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            kern<<<device_sm_count(), kThreads, smem, s>>>(a);
            return cudaGetLastError();
        };
        if (a.fp8) return a.H <= 8 ? launch8(index_shared_fp8_kernel<1>) : launch8(index_shared_fp8_kernel<2>);
        return a.H <= 8 ? launch(index_shared_kernel<1>) : launch(index_shared_kernel<2>);
    }
    if (!a.fp8) return cudaErrorInvalidValue;       // per-head bf16 keys: index_decode_kernel
    static_assert(sizeof(Fp8Smem) + 1024 <= 232448, "shared memory budget");
    const size_t smem = sizeof(Fp8Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(index_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    index_fp8_kernel<<<device_sm_count(), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
