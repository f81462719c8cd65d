// attn_rows.cu -- MSA sparse branch, one CTA per (query row, group, split).
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 -- full attention over the top-k KV blocks
// only; section 六 -- every head of a GQA group shares the group's block set,
// so each kept block is brought on chip once and serves all of the group's
// heads.  Softmax over the kept keys is exact; split partials are merged with
// the online-softmax identity (FlashAttention lineage, dev.to MiniMax-M3
// summary, section on kernel/I-O optimisation).
//
// Design (decode and short prefill):
//   - warp 4 (one thread) TMA-loads each kept block's K and V tile of the
//     group (3-D tensor maps, 128-byte swizzle, 4 x 16 KiB) into a 1- or
//     2-stage ring (one stage when a CTA owns a single block, so three CTAs
//     share an SM); the tile is shared by the G = H_q/H_kv heads of the group;
//   - warps 0-3 each own 32 of the block's 128 tokens and run the swapped
//     products on mma.sync m16n8k16 bf16: S^T = K Q^T (tokens x heads, heads
//     fill N = 8) and O^T += V^T P^T, with P^T moved from the accumulator
//     layout to the operand layout by movmatrix; online softmax in fp32;
//   - warps merge in shared memory; with several splits each CTA writes a
//     partial (m, l, O) and the last CTA of the (row, group) to arrive merges
//     them and writes bf16 output.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kHalf = 16384;              // 128 tokens x 64 dims x bf16
constexpr int kStageBytes = 4 * kHalf;    // K lo/hi + V lo/hi
constexpr int kMaxK = 64;
constexpr float kLog2e = 1.4426950408889634f;

template <int NT, int kStages>
struct Smem {
    uint8_t ring[kStages][kStageBytes];   // reused as the merge area at the end
    __nv_bfloat16 q[NT * 8][kDim];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    int blocks[kMaxK];
    int nblk;
    int last;
    int abort_flag;
};

template <int NT>
struct Merge {
    float o[kConsumerWarps][NT * 8][kDim];
    float m[kConsumerWarps][NT * 8];
    float l[kConsumerWarps][NT * 8];
};

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

template <int NT, int kStages>
__global__ void __launch_bounds__(kThreads, kStages == 1 ? 3 : 1)
    attn_rows_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const AttnRowsArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Smem<NT, kStages> &S = *reinterpret_cast<Smem<NT, kStages> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = P.H_q / P.H_kv;
    const long long cta = blockIdx.x;
    const int split = static_cast<int>(cta % P.nsplit);
    const long long pair = cta / P.nsplit;          // row * H_kv + g
    const int g = static_cast<int>(pair % P.H_kv);
    const long long row = pair / P.H_kv;
    const int b = static_cast<int>(row / P.Sq);
    const int i = static_cast<int>(row % P.Sq);
    const int L = P.lens[b];
    const bool valid = L >= P.Sq && L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(P.out) + (row * P.H_q + (long long)g * G) * kDim;

    if (!valid) {
        if (split == 0) {
            for (int e = tid; e < G * kDim; e += kThreads) out[e] = __float2bfloat16(NAN);
            if (P.lse)
                for (int e = tid; e < G; e += kThreads) P.lse[row * P.H_q + static_cast<long long>(g) * G + e] = NAN;
            if (tid == 0 && i == 0 && g == 0) set_status(P.status, kStatusBadLens);
        }
        return;
    }
    const long long p = static_cast<long long>(L) - P.Sq + i;     // query position
    const int own = static_cast<int>(p / kBlock);
    const int bps = (P.K + P.nsplit - 1) / P.nsplit;

    if (tid == 0) {
        // Kept ids of this (row, group), -1 skipped, then this split's share;
        // the first blocks' TMA loads go out before anything else is set up.
        for (int st = 0; st < kStages; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], kConsumerWarps);
        }
        fence_mbar_init();
        S.abort_flag = 0;
        // the group's index head: contiguous sets of H_kv / n_idx groups
        const int32_t *ids = P.ids + (row * P.n_idx + g / (P.H_kv / P.n_idx)) * P.K;
        const int lo = split * bps, hi = lo + bps;
        int n = 0, bad = 0, nblk = 0;
        for (int q = 0; q < P.K; ++q) {
            const int j = __ldg(ids + q);
            if (j < 0) { bad |= (j != -1); continue; }
            if (j > own) { bad = 1; continue; }
            if (n >= lo && n < hi) {
                S.blocks[nblk] = j;
                if (nblk < kStages) {
                    const int tok = static_cast<int>(kv_block_row(P.kv, b, j, P.status));
                    uint8_t *dst = S.ring[nblk];
                    mbar_arrive_expect_tx(&S.full[nblk], kStageBytes);
                    tma_load_3d(dst, &tmK, 0, g, tok, &S.full[nblk]);
                    tma_load_3d(dst + kHalf, &tmK, 64, g, tok, &S.full[nblk]);
                    tma_load_3d(dst + 2 * kHalf, &tmV, 0, g, tok, &S.full[nblk]);
                    tma_load_3d(dst + 3 * kHalf, &tmV, 64, g, tok, &S.full[nblk]);
                }
                ++nblk;
            }
            ++n;
        }
        if (bad) set_status(P.status, kStatusBadLens);
        S.nblk = nblk;
    }
    // Q rows of the group's heads (zero rows pad G up to 8 * NT).
    {
        const __nv_bfloat16 *qrow = static_cast<const __nv_bfloat16 *>(P.q) +
                                    (row * P.H_q + (long long)g * G) * kDim;
        for (int e = tid; e < NT * 8 * kDim / 8; e += kThreads) {
            const int h = e / (kDim / 8), c = e % (kDim / 8);
            uint4 v = make_uint4(0, 0, 0, 0);
            if (h < G) v = *reinterpret_cast<const uint4 *>(qrow + h * kDim + c * 8);
            *reinterpret_cast<uint4 *>(&S.q[h][c * 8]) = v;
        }
    }
    __syncthreads();
    const int nblk = S.nblk;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer
        if (lane == 0 && nblk > kStages) {
            bool ok = true;
            int it = kStages;                      // the first stages were issued above
            for (; it < nblk; ++it) {
                const int st = it % kStages;
                if (it >= kStages &&
                    (*(volatile int *)&S.abort_flag ||
                     !mbar_wait(&S.empty[st], ((it / kStages) - 1) & 1, P.status))) {
                    *(volatile int *)&S.abort_flag = 1;
                    ok = false;
                    break;
                }
                const int tok = static_cast<int>(kv_block_row(P.kv, b, S.blocks[it], P.status));
                uint8_t *dst = S.ring[st];
                mbar_arrive_expect_tx(&S.full[st], kStageBytes);
                tma_load_3d(dst, &tmK, 0, g, tok, &S.full[st]);
                tma_load_3d(dst + kHalf, &tmK, 64, g, tok, &S.full[st]);
                tma_load_3d(dst + 2 * kHalf, &tmV, 0, g, tok, &S.full[st]);
                tma_load_3d(dst + 3 * kHalf, &tmV, 64, g, tok, &S.full[st]);
            }
            if (!ok)
                for (int k = max(0, it - kStages); k < it; ++k)
                    mbar_wait(&S.full[k % kStages], (k / kStages) & 1, nullptr);
        }
        return;
    }

    // ---------------------------------------------------- consumers
    const int gq = lane >> 2, tq = lane & 3;
    const int tok0 = warp * 32;
    const float sl2 = P.softmax_scale * kLog2e;

    uint32_t qf[8][NT][2];
#pragma unroll
    for (int kk = 0; kk < 8; kk += 2)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = nt * 8 + (lane & 7);
            const int col = (kk + (lane >> 4)) * 16 + ((lane >> 3) & 1) * 8;
            ldsm_x4(smem_u32(&S.q[h][col]), qf[kk][nt][0], qf[kk][nt][1], qf[kk + 1][nt][0],
                    qf[kk + 1][nt][1]);
        }

    float acc[8][NT][4];
    float mrun[NT][2], lrun[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) { mrun[nt][c] = -INFINITY; lrun[nt][c] = 0.f; }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
    }

    for (int it = 0; it < nblk; ++it) {
        const int st = it % kStages;
        bool have = false;
        if (!*(volatile int *)&S.abort_flag) have = mbar_wait(&S.full[st], (it / kStages) & 1, P.status);
        have = __all_sync(0xffffffffu, have);
        if (!have) { *(volatile int *)&S.abort_flag = 1; break; }
        const uint32_t kbase = smem_u32(S.ring[st]);
        const uint32_t vbase = kbase + 2 * kHalf;
        const int j = S.blocks[it];
        const long long nv_ll = p + 1 - (long long)j * kBlock;
        const int nvalid = nv_ll < kBlock ? static_cast<int>(nv_ll) : kBlock;

        if (nvalid < tok0 + 32) {
            // Zero the V rows of tokens past the query (they get weight 0; the
            // bytes may be padding of any value).
            uint8_t *vz = S.ring[st] + 2 * kHalf;
            for (int e = lane; e < 32 * 16; e += 32) {
                const int r = tok0 + (e >> 4), c = e & 15;
                if (r >= nvalid)
                    *reinterpret_cast<uint4 *>(vz + (c >> 3) * kHalf + r * 128 + (c & 7) * 16) =
                        make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }

        // S^T = K Q^T for this warp's 32 tokens.
        float s[2][NT][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[mt][nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int chunk = ((kk & 3) << 1) | (lane >> 4);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int r = tok0 + mt * 16 + (lane & 15);
                uint32_t a[4];
                ldsm_x4(kbase + (kk >> 2) * kHalf + swz128(r, chunk), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[mt][nt], a, qf[kk][nt][0], qf[kk][nt][1]);
            }
        }

        // Online softmax (base 2) per head column.
        uint32_t pb[2][NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float cmax = -INFINITY;
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int t = tok0 + mt * 16 + gq + 8 * hh;
                        float x = s[mt][nt][2 * hh + c] * sl2;
                        x = t < nvalid ? x : -INFINITY;
                        s[mt][nt][2 * hh + c] = x;
                        cmax = fmaxf(cmax, x);
                    }
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 4));
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 8));
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 16));
                const float mnew = fmaxf(mrun[nt][c], cmax);
                const float mref = mnew == -INFINITY ? 0.f : mnew;
                const float alpha = exp2f(mrun[nt][c] - mref);
                mrun[nt][c] = mnew;
                float psum = 0.f;
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const float pv = exp2f(s[mt][nt][2 * hh + c] - mref);
                        s[mt][nt][2 * hh + c] = pv;
                        psum += pv;
                    }
                lrun[nt][c] = lrun[nt][c] * alpha + psum;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    acc[mt][nt][c] *= alpha;
                    acc[mt][nt][2 + c] *= alpha;
                }
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                pb[mt][nt][0] = movmatrix_t(pack_bf16x2(s[mt][nt][0], s[mt][nt][1]));
                pb[mt][nt][1] = movmatrix_t(pack_bf16x2(s[mt][nt][2], s[mt][nt][3]));
            }
        }

        // O^T += V^T P^T.
#pragma unroll
        for (int kk2 = 0; kk2 < 2; ++kk2) {
            const int mi = lane >> 3;
            const int r = tok0 + kk2 * 16 + ((mi >> 1) << 3) + (lane & 7);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int d = mt * 16 + ((mi & 1) << 3);
                uint32_t a[4];
                ldsm_x4_t(vbase + (d >> 6) * kHalf + swz128(r, (d & 63) >> 3), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[mt][nt], a, pb[kk2][nt][0], pb[kk2][nt][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[st]);
    }

    // ------------------------------------------------ merge the 4 warps
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float l = lrun[nt][c];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            lrun[nt][c] = l;
        }
    consumers_sync();   // every warp is done with the ring before it is reused
    Merge<NT> &M = *reinterpret_cast<Merge<NT> *>(S.ring[0]);
    const bool aborted = *(volatile int *)&S.abort_flag;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int h = nt * 8 + 2 * tq + c;
            if (gq == 0) { M.m[warp][h] = mrun[nt][c]; M.l[warp][h] = lrun[nt][c]; }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                M.o[warp][h][mt * 16 + gq] = acc[mt][nt][c];
                M.o[warp][h][mt * 16 + gq + 8] = acc[mt][nt][2 + c];
            }
        }
    }
    consumers_sync();

    // Thread -> (head, 8 dims); heads beyond G are padding and skipped.
    const int nthr = kConsumerWarps * 32;
    const int rec = attn_partial_floats(G);         // floats per split partial
    const int ooff = attn_partial_o_offset(G);
    float *part = P.partials + (pair * P.nsplit) * rec;
    for (int e = tid; e < G * (kDim / 8); e += nthr) {
        const int h = e / (kDim / 8), d0 = (e % (kDim / 8)) * 8;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, M.m[w][h]);
        const float mref = mx == -INFINITY ? 0.f : mx;
        float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float wt = exp2f(M.m[w][h] - mref);
            l += wt * M.l[w][h];
#pragma unroll
            for (int x = 0; x < 8; ++x) o[x] += wt * M.o[w][h][d0 + x];
        }
        if (P.nsplit == 1) {
            const float inv = aborted ? NAN : 1.f / l;
            uint4 v;
            v.x = pack_bf16x2(o[0] * inv, o[1] * inv);
            v.y = pack_bf16x2(o[2] * inv, o[3] * inv);
            v.z = pack_bf16x2(o[4] * inv, o[5] * inv);
            v.w = pack_bf16x2(o[6] * inv, o[7] * inv);
            *reinterpret_cast<uint4 *>(out + h * kDim + d0) = v;
            if (P.lse && d0 == 0)
                P.lse[row * P.H_q + static_cast<long long>(g) * G + h] = aborted ? NAN : mref + log2f(l);
        } else {
            float *pr = part + split * rec;
            if (d0 == 0) { pr[h] = mx; pr[G + h] = aborted ? NAN : l; }
#pragma unroll
            for (int x = 0; x < 8; ++x) pr[ooff + h * kDim + d0 + x] = o[x];
        }
    }
    if (P.nsplit == 1) return;

    // ------------------------------------------------ last CTA merges splits
    consumers_sync();                     // every partial of this CTA is written
    if (tid == 0) {
        __threadfence();                  // ... and visible before the ticket
        const int t = atomicAdd(P.tickets + pair, 1);
        S.last = (t == P.nsplit - 1);
        if (S.last) P.tickets[pair] = 0;
    }
    consumers_sync();
    if (!S.last) return;
    __threadfence();
    // Splits are read eight at a time with every load issued before its use.
    for (int e = tid; e < G * (kDim / 8); e += nthr) {
        const int h = e / (kDim / 8), d0 = (e % (kDim / 8)) * 8;
        float mx = -INFINITY;
        for (int s0 = 0; s0 < P.nsplit; s0 += 8) {
            float mv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                mv[u] = s0 + u < P.nsplit ? __ldcg(part + (s0 + u) * rec + h) : -INFINITY;
#pragma unroll
            for (int u = 0; u < 8; ++u) mx = fmaxf(mx, mv[u]);
        }
        const float mref = mx == -INFINITY ? 0.f : mx;
        float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float l = 0.f;
        for (int s0 = 0; s0 < P.nsplit; s0 += 8) {
            float mv[8], lv[8];
            float4 ov[8][2];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool in = s0 + u < P.nsplit;
                const float *pr = part + (in ? s0 + u : 0) * rec;
                mv[u] = in ? __ldcg(pr + h) : -INFINITY;
                lv[u] = __ldcg(pr + G + h);
                ov[u][0] = __ldcg(reinterpret_cast<const float4 *>(pr + ooff + h * kDim + d0));
                ov[u][1] = __ldcg(reinterpret_cast<const float4 *>(pr + ooff + h * kDim + d0 + 4));
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float wt = exp2f(mv[u] - mref);          // 0 for splits past the end
                l += wt * lv[u];
                o[0] += wt * ov[u][0].x; o[1] += wt * ov[u][0].y;
                o[2] += wt * ov[u][0].z; o[3] += wt * ov[u][0].w;
                o[4] += wt * ov[u][1].x; o[5] += wt * ov[u][1].y;
                o[6] += wt * ov[u][1].z; o[7] += wt * ov[u][1].w;
            }
        }
        const float inv = 1.f / l;
        uint4 v;
        v.x = pack_bf16x2(o[0] * inv, o[1] * inv);
        v.y = pack_bf16x2(o[2] * inv, o[3] * inv);
        v.z = pack_bf16x2(o[4] * inv, o[5] * inv);
        v.w = pack_bf16x2(o[6] * inv, o[7] * inv);
        *reinterpret_cast<uint4 *>(out + h * kDim + d0) = v;
        if (P.lse && d0 == 0) P.lse[row * P.H_q + static_cast<long long>(g) * G + h] = mref + log2f(l);
    }
}

template <int NT, int STAGES>
cudaError_t launch_nt(const AttnRowsArgs &a, cudaStream_t s) {
    static_assert(sizeof(Merge<NT>) <= STAGES * kStageBytes, "merge area fits in the ring");
    static_assert(sizeof(Smem<NT, STAGES>) + 1024 <= 227 * 1024, "shared memory budget");
    CUtensorMap tk, tv;
    if (!encode_kv_tensor_map(&tk, a.k_cache, a.H_kv, a.kv.capacity) ||
        !encode_kv_tensor_map(&tv, a.v_cache, a.H_kv, a.kv.capacity))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(Smem<NT, STAGES>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_rows_kernel<NT, STAGES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long ctas = static_cast<long long>(a.B) * a.Sq * a.H_kv * a.nsplit;
    TraceScope trace(s, "sparse_attention_rows");
    attn_rows_kernel<NT, STAGES><<<static_cast<unsigned>(ctas), kThreads, smem, s>>>(tk, tv, a);
    return cudaGetLastError();
}

}  // namespace

int attn_rows_nsplit(long long rows_x_groups, int top_k) {
    // Few kept blocks in total (decode of a modest batch): one block per CTA,
    // single-stage CTAs of ~70 KiB so three fit on an SM and every block's
    // load is in flight at once.
    if (rows_x_groups * top_k <= 1536) return top_k;
    // Otherwise aim at two CTAs per SM of a 148-SM part.
    long long want = (2 * 148 + rows_x_groups - 1) / rows_x_groups;
    if (want < 1) want = 1;
    if (want > top_k) want = top_k;
    const int bps = static_cast<int>((top_k + want - 1) / want);
    return (top_k + bps - 1) / bps;
}

cudaError_t launch_attn_rows(const AttnRowsArgs &a, cudaStream_t s) {
    const int G = a.H_q / a.H_kv;
    const bool one = (a.K + a.nsplit - 1) / a.nsplit == 1;   // one block per CTA
    if (G <= 8) return one ? launch_nt<1, 1>(a, s) : launch_nt<1, 2>(a, s);
    if (G <= 16) return one ? launch_nt<2, 1>(a, s) : launch_nt<2, 2>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace msa
