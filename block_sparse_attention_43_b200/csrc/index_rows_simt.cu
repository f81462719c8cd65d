// index_rows_simt.cu -- MSA index branch for several query rows per sequence
// (prefill), on CUDA cores: block max-pooled causal index scores.
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 -- one index query per GQA group dotted with
// the index keys, "Block Max Pool" per KV block.  Causal: a query at position
// p sees tokens t <= p, so its own block is pooled over t <= p only.
//
// One CTA per (sequence, group, 64 query rows).  For each visible key block
// the CTA stages the block's 128 index keys in shared memory as fp32, every
// thread forms a 4-row x 8-token tile of dot products over the 128 dims, and
// a 16-lane max gives each row's block score.  This kernel is the simple
// path; the tensor-core kernel (index_rows_tc.cu) computes the same values.
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kRows = 64;
constexpr int kThreads = 256;

struct Smem {
    float q[kDim][kRows];      // transposed index queries of the tile
    float k[kDim][kBlock];     // transposed index keys of one block
};

__global__ void __launch_bounds__(kThreads) index_rows_simt_kernel(const IndexRowsArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x;
    const int tiles = (P.Sq + kRows - 1) / kRows;
    const int tile = blockIdx.x % tiles;
    const int g = (blockIdx.x / tiles) % P.H_kv;
    const int b = blockIdx.x / (tiles * P.H_kv);
    const int H = P.H_kv;
    const int L = P.lens[b];
    const long long off = P.kv_offsets[b];
    if (!(L >= P.Sq && L >= 1 && L <= P.max_kv_len && off >= 0 && off + L <= P.capacity)) {
        if (tid == 0 && tile == 0 && g == 0) set_status(P.status, kStatusBadLens);
        return;
    }
    const int i0 = tile * kRows;
    const int nrows = min(kRows, P.Sq - i0);
    const long long p_first = static_cast<long long>(L) - P.Sq + i0;
    const long long p_last = p_first + nrows - 1;
    const int jmax = static_cast<int>(p_last / kBlock);

    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(P.q_idx);
    const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(P.k_idx);
    for (int e = tid; e < kRows * (kDim / 8); e += kThreads) {
        const int r = e % kRows, c = e / kRows;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < nrows)
            v = *reinterpret_cast<const uint4 *>(qb + (((long long)b * P.Sq + i0 + r) * H + g) * kDim + c * 8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            S.q[c * 8 + 2 * x][r] = bf16lo(w[x]);
            S.q[c * 8 + 2 * x + 1][r] = bf16hi(w[x]);
        }
    }

    const int rg = tid >> 4, tg = tid & 15;   // rows rg*4..+3, tokens tg*4..+3 and 64+tg*4..+3
    for (int j = 0; j <= jmax; ++j) {
        __syncthreads();
        for (int e = tid; e < kBlock * (kDim / 8); e += kThreads) {
            const int t = e % kBlock, c = e / kBlock;
            const long long tok = (long long)j * kBlock + t;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (tok < L) v = *reinterpret_cast<const uint4 *>(kb + ((off + tok) * H + g) * kDim + c * 8);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                S.k[c * 8 + 2 * x][t] = bf16lo(w[x]);
                S.k[c * 8 + 2 * x + 1][t] = bf16hi(w[x]);
            }
        }
        __syncthreads();
        float acc[4][8];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[r][x] = 0.f;
#pragma unroll 4
        for (int d = 0; d < kDim; ++d) {
            const float4 qv = *reinterpret_cast<const float4 *>(&S.q[d][rg * 4]);
            const float4 k0 = *reinterpret_cast<const float4 *>(&S.k[d][tg * 4]);
            const float4 k1 = *reinterpret_cast<const float4 *>(&S.k[d][64 + tg * 4]);
            const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
            const float ka[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int x = 0; x < 8; ++x) acc[r][x] = fmaf(qa[r], ka[x], acc[r][x]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int row = rg * 4 + r;
            const long long p = p_first + row;
            float m = -INFINITY;
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const long long t = (long long)j * kBlock + (x < 4 ? tg * 4 + x : 64 + tg * 4 + x - 4);
                if (t <= p) m = fmaxf(m, acc[r][x]);
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            if (tg == 0 && row < nrows && j <= p / kBlock)
                P.scores[(((long long)b * P.Sq + i0 + row) * H + g) * P.nb_max + j] = m;
        }
    }
}

}  // namespace

cudaError_t launch_index_rows_simt(const IndexRowsArgs &a, cudaStream_t s) {
    const size_t smem = sizeof(Smem) + 128;
    cudaError_t e = cudaFuncSetAttribute(index_rows_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long tiles = (a.Sq + kRows - 1) / kRows;
    const long long grid = tiles * a.H_kv * a.B;
    TraceScope trace(s, "index_score_maxpool_rows_simt");
    index_rows_simt_kernel<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
