// attn_bwd.cu -- backward of the MSA sparse branch: dQ, dK, dV over the kept
// blocks, one CTA per (query row, group).
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 (exact attention over the kept blocks) and
// section 五 (MSA is trained natively; the index branch supplies the
// selection, the sparse branch computes exactly on it).  The selection is
// piecewise constant, so only the sparse branch carries gradient.  For one
// (row, head) over its kept keys: P = softmax(scale q.k), dP_t = dO.v_t,
// Delta = sum_t P_t dP_t, dZ_t = P_t (dP_t - Delta), dQ = scale sum_t dZ_t k_t,
// dK_t += scale dZ_t q, dV_t += P_t dO.
//
// Design (a first, row-oriented path): warp 8 streams the kept blocks' K and V
// tiles (TMA, 128-byte swizzle, 64 KiB per block) twice through a 2-stage
// ring; warps 0-7 own 16 of a block's 128 tokens each and run every product
// on mma.sync m16n8k16 bf16 with the group's heads on the 8-wide side:
//   pass 1  S^T = K Q^T and dP^T = V dO^T; per head an online max, sum and
//           delta = sum_t p_t dP_t; warps merge three scalars per head;
//   pass 2  the same two products again, P and dZ from the merged statistics,
//           dV = P^T dO and dK = scale dZ^T Q (16 tokens x 128 dims per warp,
//           added to fp32 dK/dV with red.global.add.v2.f32), and
//           dQ^T += scale K^T dZ^T kept in registers, merged across warps at
//           the end and written as bf16.
// Keys and values past the query (or padding) are zeroed in shared memory and
// masked by selection.  Every (row, kept block) adds a full 128 x 128 block of
// dK and dV, so this path is bound by those reductions at large sizes; a
// block-outer kernel that sums a block's rows on chip is the next step.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kWarps = 8;                  // consumer warps, 16 tokens each
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kHalf = 16384;               // 128 tokens x 64 dims x bf16
constexpr int kStageBytes = 4 * kHalf;     // K lo/hi + V lo/hi
constexpr int kMaxK = 64;
constexpr float kLog2e = 1.4426950408889634f;

struct Smem {
    uint8_t ring[2][kStageBytes];          // reused for the dQ merge at the end
    __nv_bfloat16 q[16][kDim];             // the group's heads, zero past G
    __nv_bfloat16 dout[16][kDim];
    float m1[kWarps][16], l1[kWarps][16], d1[kWarps][16];   // pass-1 per-warp statistics
    float mh[16], lh[16], dh[16];          // merged: max (base 2), sum, Delta
    uint64_t full[2], empty[2];
    int blocks[kMaxK];
    int nblk;
    int abort_flag;
};

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
}

__device__ __forceinline__ void red_add_v2(float *p, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

// A operand (16 tokens x 16 heads) from the accumulator layout of S^T-shaped
// fragments: rows gq / gq+8 and heads 2tq, 2tq+1 of n-tile 0 (k 0-7) and n-tile
// 1 (k 8-15; zero with one n-tile).
template <int NT>
__device__ __forceinline__ void tokens_by_heads_operand(const float (&x)[NT][4], uint32_t (&a)[4]) {
    a[0] = pack_bf16x2(x[0][0], x[0][1]);
    a[1] = pack_bf16x2(x[0][2], x[0][3]);
    a[2] = NT > 1 ? pack_bf16x2(x[NT - 1][0], x[NT - 1][1]) : 0u;
    a[3] = NT > 1 ? pack_bf16x2(x[NT - 1][2], x[NT - 1][3]) : 0u;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const AttnBwdArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = P.H_q / P.H_kv;
    const long long pair = blockIdx.x;            // row * H_kv + g
    const int g = static_cast<int>(pair % P.H_kv);
    const long long row = pair / P.H_kv;
    const int b = static_cast<int>(row / P.Sq);
    const int i = static_cast<int>(row % P.Sq);
    const int L = P.lens[b];
    const bool valid = L >= P.Sq && L >= 1 && L <= P.max_kv_len && kv_seq_ok(P.kv, b, L);
    __nv_bfloat16 *dq = static_cast<__nv_bfloat16 *>(P.dq) + (row * P.H_q + (long long)g * G) * kDim;
    if (!valid) {
        for (int e = tid; e < G * kDim; e += kThreads) dq[e] = __float2bfloat16(NAN);
        if (tid == 0 && i == 0 && g == 0) set_status(P.status, kStatusBadLens);
        return;
    }
    const long long p = static_cast<long long>(L) - P.Sq + i;     // query position
    const int own = static_cast<int>(p / kBlock);

    if (tid == 0) {
        for (int st = 0; st < 2; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], kWarps);
        }
        fence_mbar_init();
        S.abort_flag = 0;
        const int32_t *ids = P.ids + (row * P.n_idx + g / (P.H_kv / P.n_idx)) * P.K;
        int n = 0, bad = 0;
        for (int q = 0; q < P.K; ++q) {
            const int j = __ldg(ids + q);
            if (j < 0) { bad |= (j != -1); continue; }
            if (j > own) { bad = 1; continue; }
            S.blocks[n++] = j;
        }
        if (bad) set_status(P.status, kStatusBadLens);
        S.nblk = n;
    }
    // Q and dO rows of the group's heads (zero rows pad G up to 16).
    {
        const __nv_bfloat16 *qrow = static_cast<const __nv_bfloat16 *>(P.q) + (row * P.H_q + (long long)g * G) * kDim;
        const __nv_bfloat16 *drow = static_cast<const __nv_bfloat16 *>(P.dout) + (row * P.H_q + (long long)g * G) * kDim;
        for (int e = tid; e < 16 * kDim / 8; e += kThreads) {
            const int h = e / (kDim / 8), c = e % (kDim / 8);
            uint4 vq = make_uint4(0, 0, 0, 0), vd = make_uint4(0, 0, 0, 0);
            if (h < G) {
                vq = *reinterpret_cast<const uint4 *>(qrow + h * kDim + c * 8);
                vd = *reinterpret_cast<const uint4 *>(drow + h * kDim + c * 8);
            }
            *reinterpret_cast<uint4 *>(&S.q[h][c * 8]) = vq;
            *reinterpret_cast<uint4 *>(&S.dout[h][c * 8]) = vd;
        }
    }
    __syncthreads();
    const int nblk = S.nblk;

    if (warp == kWarps) {
        // ------------------------------------------------ producer: both passes
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            bool ok = true;
            int it = 0;
            for (; it < 2 * nblk; ++it) {
                const int st = it & 1;
                if (it >= 2 && (*(volatile int *)&S.abort_flag ||
                                !mbar_wait(&S.empty[st], ((it >> 1) - 1) & 1, P.status))) {
                    *(volatile int *)&S.abort_flag = 1;
                    ok = false;
                    break;
                }
                const int tok = static_cast<int>(kv_block_row(P.kv, b, S.blocks[it % nblk], P.status));
                uint8_t *dst = S.ring[st];
                mbar_arrive_expect_tx(&S.full[st], kStageBytes);
                tma_load_3d(dst, &tmK, 0, g, tok, &S.full[st]);
                tma_load_3d(dst + kHalf, &tmK, 64, g, tok, &S.full[st]);
                tma_load_3d(dst + 2 * kHalf, &tmV, 0, g, tok, &S.full[st]);
                tma_load_3d(dst + 3 * kHalf, &tmV, 64, g, tok, &S.full[st]);
            }
            if (!ok)
                for (int k = max(0, it - 2); k < it; ++k) mbar_wait(&S.full[k & 1], (k >> 1) & 1, nullptr);
        }
        return;
    }

    // ---------------------------------------------------- consumers
    const int gq = lane >> 2, tq = lane & 3;
    const int r0 = warp * 16;                        // this warp's tokens of a block
    const float sl2 = P.softmax_scale * kLog2e;
    // Q^T and dO^T as B operands (k = dims, n = heads) for S^T and dP^T.
    uint32_t qf[8][NT][2], of[8][NT][2];
#pragma unroll
    for (int kk = 0; kk < 8; kk += 2)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = nt * 8 + (lane & 7);
            const int col = (kk + (lane >> 4)) * 16 + ((lane >> 3) & 1) * 8;
            ldsm_x4(smem_u32(&S.q[h][col]), qf[kk][nt][0], qf[kk][nt][1], qf[kk + 1][nt][0], qf[kk + 1][nt][1]);
            ldsm_x4(smem_u32(&S.dout[h][col]), of[kk][nt][0], of[kk][nt][1], of[kk + 1][nt][0], of[kk + 1][nt][1]);
        }

    // Waits for block `it` of the stream, zeroes this warp's K and V rows past
    // the query (padding may hold anything), returns the block's valid count.
    auto acquire = [&](int it, int &nvalid) -> bool {
        const int st = it & 1;
        bool have = !*(volatile int *)&S.abort_flag && mbar_wait(&S.full[st], (it >> 1) & 1, P.status);
        have = __all_sync(0xffffffffu, have);
        if (!have) { *(volatile int *)&S.abort_flag = 1; return false; }
        const int j = S.blocks[it % nblk];
        const long long nv = p + 1 - static_cast<long long>(j) * kBlock;
        nvalid = nv < kBlock ? static_cast<int>(nv) : kBlock;
        if (nvalid < r0 + 16) {
            for (int e = lane; e < 16 * 16; e += 32) {
                const int r = r0 + (e >> 4), c = e & 15;
                if (r >= nvalid) {
                    const int off = (c >> 3) * kHalf + r * 128 + (c & 7) * 16;
                    *reinterpret_cast<uint4 *>(S.ring[st] + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(S.ring[st] + 2 * kHalf + off) = make_uint4(0, 0, 0, 0);
                }
            }
            __syncwarp();
        }
        return true;
    };
    auto release = [&](int it) {
        fence_proxy_async_smem();                    // generic zeroing before the next TMA write
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[it & 1]);
    };
    // S^T = K Q^T and dP^T = V dO^T for this warp's 16 tokens.
    auto products = [&](int st, float (&s)[NT][4], float (&dp)[NT][4]) {
        const uint32_t kbase = smem_u32(S.ring[st]), vbase = kbase + 2 * kHalf;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int chunk = ((kk & 3) << 1) | (lane >> 4);
            const int r = r0 + (lane & 15);
            uint32_t a[4], v[4];
            ldsm_x4(kbase + (kk >> 2) * kHalf + swz128(r, chunk), a[0], a[1], a[2], a[3]);
            ldsm_x4(vbase + (kk >> 2) * kHalf + swz128(r, chunk), v[0], v[1], v[2], v[3]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(s[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
                mma_bf16_16816(dp[nt], v, of[kk][nt][0], of[kk][nt][1]);
            }
        }
    };

    // ---- pass 1: per-head max (base 2), sum and delta over this warp's tokens
    float mrun[NT][2], lrun[NT][2], drun[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) { mrun[nt][c] = -INFINITY; lrun[nt][c] = 0.f; drun[nt][c] = 0.f; }
    bool ok = true;
    for (int it = 0; it < nblk && ok; ++it) {
        int nvalid;
        if (!acquire(it, nvalid)) { ok = false; break; }
        float s[NT][4], dp[NT][4];
        products(it & 1, s, dp);
        release(it);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float x0 = r0 + gq < nvalid ? s[nt][c] * sl2 : -INFINITY;
                float x1 = r0 + gq + 8 < nvalid ? s[nt][2 + c] * sl2 : -INFINITY;
                float cmax = fmaxf(x0, x1);
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 4));
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 8));
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 16));
                const float mnew = fmaxf(mrun[nt][c], cmax);
                const float mref = mnew == -INFINITY ? 0.f : mnew;
                const float alpha = exp2f(mrun[nt][c] - mref);
                const float p0 = exp2f(x0 - mref), p1 = exp2f(x1 - mref);
                mrun[nt][c] = mnew;
                lrun[nt][c] = lrun[nt][c] * alpha + p0 + p1;
                // p0/p1 are 0 on masked tokens; their dP may be anything finite
                drun[nt][c] = drun[nt][c] * alpha + (p0 > 0.f ? p0 * dp[nt][c] : 0.f) +
                              (p1 > 0.f ? p1 * dp[nt][2 + c] : 0.f);
            }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float l = lrun[nt][c], d = drun[nt][c];
#pragma unroll
            for (int o = 4; o <= 16; o <<= 1) {
                l += __shfl_xor_sync(0xffffffffu, l, o);
                d += __shfl_xor_sync(0xffffffffu, d, o);
            }
            if (gq == 0) {
                const int h = nt * 8 + 2 * tq + c;
                S.m1[warp][h] = mrun[nt][c];
                S.l1[warp][h] = l;
                S.d1[warp][h] = d;
            }
        }
    consumers_sync();
    if (tid < NT * 8) {
        float m = -INFINITY;
        for (int w = 0; w < kWarps; ++w) m = fmaxf(m, S.m1[w][tid]);
        const float mref = m == -INFINITY ? 0.f : m;
        float l = 0.f, d = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            const float f = exp2f(S.m1[w][tid] - mref);
            l += S.l1[w][tid] * f;
            d += S.d1[w][tid] * f;
        }
        S.mh[tid] = mref;
        S.lh[tid] = l;
        S.dh[tid] = l > 0.f ? d / l : 0.f;             // Delta = sum_t P_t dP_t
    }
    consumers_sync();

    // ---- pass 2: P, dZ; dV, dK to global; dQ^T in registers
    float mh[NT][2], rl[NT][2], dl[NT][2];
    bool hv[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int h = nt * 8 + 2 * tq + c;
            mh[nt][c] = S.mh[h];
            rl[nt][c] = S.lh[h] > 0.f ? 1.f / S.lh[h] : 0.f;
            dl[nt][c] = S.dh[h];
            hv[nt][c] = h < G;                        // padding heads carry no gradient
        }
    float dqa[8][NT][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) dqa[mt][nt][e] = 0.f;
    const float scale = P.softmax_scale;
    for (int it = nblk; it < 2 * nblk && ok; ++it) {
        int nvalid;
        if (!acquire(it, nvalid)) { ok = false; break; }
        const int st = it & 1;
        float s[NT][4], dp[NT][4];
        products(st, s, dp);
        float ps[NT][4], dz[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = e & 1;
                const bool tv = r0 + gq + (e >> 1) * 8 < nvalid;
                const bool on = tv && hv[nt][c];
                const float pv = on ? exp2f(s[nt][e] * sl2 - mh[nt][c]) * rl[nt][c] : 0.f;
                ps[nt][e] = pv;
                dz[nt][e] = on ? pv * (dp[nt][e] - dl[nt][c]) : 0.f;
            }
        // dQ^T += K^T dZ^T (K rows past the query are zero in shared memory).
        {
            const uint32_t kbase = smem_u32(S.ring[st]);
            uint32_t zb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                zb[nt][0] = movmatrix_t(pack_bf16x2(dz[nt][0], dz[nt][1]));
                zb[nt][1] = movmatrix_t(pack_bf16x2(dz[nt][2], dz[nt][3]));
            }
            const int mi = lane >> 3;
            const int r = r0 + ((mi >> 1) << 3) + (lane & 7);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int d = mt * 16 + ((mi & 1) << 3);
                uint32_t a[4];
                ldsm_x4_t(kbase + (d >> 6) * kHalf + swz128(r, (d & 63) >> 3), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(dqa[mt][nt], a, zb[nt][0], zb[nt][1]);
            }
        }
        release(it);
        // dV = P^T dO and dK = scale dZ^T Q: 16 tokens x 128 dims, in two
        // halves of 64 dims; the B operand (k = heads, n = dims) comes from
        // the row-major head tiles by transposed ldmatrix.
        const int j = S.blocks[it % nblk];
        const long long krow = kv_block_row(P.kv, b, j, P.status);
        const int t0 = r0 + gq, t1 = t0 + 8;
        float *dv0 = P.dv + ((krow + t0) * P.H_kv + g) * kDim;
        float *dv1 = P.dv + ((krow + t1) * P.H_kv + g) * kDim;
        float *dk0 = P.dk + ((krow + t0) * P.H_kv + g) * kDim;
        float *dk1 = P.dk + ((krow + t1) * P.H_kv + g) * kDim;
        uint32_t ap[4], az[4];
        tokens_by_heads_operand<NT>(ps, ap);
        tokens_by_heads_operand<NT>(dz, az);
        const int hrow = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const __nv_bfloat16 (*src)[kDim] = which == 0 ? S.dout : S.q;
            const uint32_t(&a)[4] = which == 0 ? ap : az;
            const float mul = which == 0 ? 1.f : scale;
            float *o0 = which == 0 ? dv0 : dk0;
            float *o1 = which == 0 ? dv1 : dk1;
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
                float acc[8][4];
#pragma unroll
                for (int n = 0; n < 8; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
#pragma unroll
                for (int j2 = 0; j2 < 4; ++j2) {
                    const int d0 = hd * 64 + j2 * 16;
                    uint32_t bb[4];
                    ldsm_x4_t(smem_u32(&src[hrow][d0 + (lane >> 4) * 8]), bb[0], bb[1], bb[2], bb[3]);
                    mma_bf16_16816(acc[2 * j2], a, bb[0], bb[1]);
                    mma_bf16_16816(acc[2 * j2 + 1], a, bb[2], bb[3]);
                }
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const int d = hd * 64 + n * 8 + 2 * tq;
                    if (t0 < nvalid) red_add_v2(o0 + d, acc[n][0] * mul, acc[n][1] * mul);
                    if (t1 < nvalid) red_add_v2(o1 + d, acc[n][2] * mul, acc[n][3] * mul);
                }
            }
        }
    }

    // ---- merge dQ^T over the 8 warps (the ring is free once every warp is done)
    consumers_sync();
    float(*M)[16][kDim] = reinterpret_cast<float(*)[16][kDim]>(S.ring[0]);   // [warp][head][dim]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int h = nt * 8 + 2 * tq + c;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                M[warp][h][mt * 16 + gq] = dqa[mt][nt][c];
                M[warp][h][mt * 16 + gq + 8] = dqa[mt][nt][2 + c];
            }
        }
    consumers_sync();
    const bool aborted = *(volatile int *)&S.abort_flag;
    for (int e = tid; e < G * kDim; e += kWarps * 32) {
        const int h = e / kDim, d = e % kDim;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += M[w][h][d];
        dq[e] = __float2bfloat16(aborted ? NAN : v * scale);
    }
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnBwdArgs &a, cudaStream_t s) {
    static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory budget");
    static_assert(kWarps * 16 * kDim * 4 <= 2 * kStageBytes, "dQ merge area fits the ring");
    CUtensorMap tk, tv;
    if (!encode_kv_tensor_map(&tk, a.k_cache, a.H_kv, a.kv.capacity) ||
        !encode_kv_tensor_map(&tv, a.v_cache, a.H_kv, a.kv.capacity))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(Smem) + 1024;
    const long long ctas = static_cast<long long>(a.B) * a.Sq * a.H_kv;
    TraceScope trace(s, "sparse_attention_backward");
    auto go = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<static_cast<unsigned>(ctas), kThreads, smem, s>>>(tk, tv, a);
        return cudaGetLastError();
    };
    return a.H_q / a.H_kv <= 8 ? go(attn_bwd_kernel<1>) : go(attn_bwd_kernel<2>);
}

}  // namespace msa
