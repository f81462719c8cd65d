// index_rows_tc.cu -- MSA index branch for prefill on the fifth-generation
// tensor cores: block max-pooled causal index scores as a tiled bf16 GEMM.
//
// Method: "百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快"
// (cloud.tencent.com), section 二 -- one index query per GQA group dotted with
// the index keys of every visible token, "Block Max Pool" per 128-token KV
// block.  For q_len query rows this is, per (sequence, group), the causal
// product Q_idx (rows x 128) . K_idx^T (128 x tokens) reduced by a max over
// each 128-column block: a real dense contraction, so it runs on tcgen05.
//
// Tiling: a work unit is (sequence, group, 128 query rows).  The unit's index
// queries (32 KiB) sit in shared memory; its visible key blocks stream through
// a 2-stage ring two blocks (64 KiB) at a time.  One thread issues
// tcgen05.mma kind::f16 M=128, N=256 (or 128 for a lone last block), K=128 as
// eight K=16 steps into one of two 256-column fp32 TMEM accumulators, and
// commits to mbarriers.  Four epilogue warps (one TMEM lane = one query row
// per thread) read the accumulator with tcgen05.ld, apply the causal mask
// where the block reaches past the row's position and write one block score
// per (row, block) into a running top-k list the thread keeps in registers
// (candidate blocks arrive in increasing order, so the list needs no
// scores buffer and no second pass).  At the end of the unit each thread
// writes its row's kept ids ascending, the own block last.  Units are dealt
// to a persistent grid in snake order of decreasing length.
//
// Roles: warp 0 = TMA producer, warp 1 = MMA issuer, warp 2 = TMEM owner,
// warps 4-7 and 8-11 = two epilogue warpgroups on alternate accumulator
// buffers (warp % 4 selects a warp's 32 TMEM lanes).
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 384;               // 4 control warps + 2 epilogue warpgroups
constexpr int kStages = 2;
constexpr int kQBytes = 2 * 16384;          // 128 rows x 128 dims, two swizzled halves
constexpr int kStageBytes = 2 * 32768;      // two key blocks: [256 rows x 128 B] per half
constexpr uint32_t kTmemCols = 512;         // two 256-column accumulators

template <int LIST>
struct Smem {
    uint8_t q[kQBytes];
    uint8_t ring[kStages][kStageBytes];
    unsigned long long xkeys[LIST][128];        // warpgroup 1's list, handed to warpgroup 0
    float xown[128];
    int xhas[128];
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t q_full, q_empty;
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};

struct Unit {
    int b, g, i0, nrows, L;
    long long p_first;
    int jmax;        // last visible key block of the tile
    bool valid;
};

__device__ __forceinline__ Unit unit_at(const IndexRowsArgs &P, long long u, int ntiles) {
    // Unit u -> (query tile, counted from the last one, sequence, group).
    Unit x;
    const long long per_tile = static_cast<long long>(P.B) * P.H_kv;
    const int t = ntiles - 1 - static_cast<int>(u / per_tile);
    const int rem = static_cast<int>(u % per_tile);
    x.b = rem / P.H_kv;
    x.g = rem % P.H_kv;
    x.i0 = t * 128;
    x.nrows = min(128, P.Sq - x.i0);
    x.L = P.lens[x.b];
    x.valid = x.L >= P.Sq && x.L >= 1 && x.L <= P.max_kv_len && kv_seq_ok(P.kv, x.b, x.L);
    x.p_first = static_cast<long long>(x.L) - P.Sq + x.i0;
    x.jmax = x.valid ? static_cast<int>((x.p_first + x.nrows - 1) / kBlock) : -1;
    return x;
}

// The r-th unit of this CTA in snake order over rounds of gridDim.x units.
__device__ __forceinline__ long long unit_index(int r) {
    const long long G = gridDim.x;
    const long long c = (r & 1) ? (G - 1 - blockIdx.x) : blockIdx.x;
    return static_cast<long long>(r) * G + c;
}

// Running top-(k-1) list of one query row: LIST keys sorted descending.
// The first LIST-(k-1) slots hold a sentinel larger than any key, so the
// smallest kept key is always L[LIST-1] and every index is static.
template <int LIST>
struct TopList {
    unsigned long long L[LIST];
    __device__ __forceinline__ void reset(int keep) {
#pragma unroll
        for (int i = 0; i < LIST; ++i) L[i] = (i < LIST - keep) ? ~0ull : 0ull;
    }
    __device__ __forceinline__ void offer(unsigned long long key) {
        if (key <= L[LIST - 1]) return;
        unsigned long long x = key;
#pragma unroll
        for (int i = 0; i < LIST; ++i) {
            const unsigned long long hi = L[i] > x ? L[i] : x;
            x = L[i] > x ? x : L[i];
            L[i] = hi;
        }
    }
};

__device__ __forceinline__ float key_score(unsigned long long key) {
    const uint32_t u = static_cast<uint32_t>(key >> 32);
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// E4M3 -> bf16, 16 codes per thread-step (every E4M3 value is a bf16 value).
__global__ void widen_e4m3_kernel(const uint4 *src, uint4 *dst, long long n16) {
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const uint4 w = src[i];
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t f16;
                const uint16_t pair = static_cast<uint16_t>(in[q] >> (16 * h));
                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(f16) : "h"(pair));
                float lo, hi;
                asm("{\n\t.reg .f16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
                    : "=f"(lo), "=f"(hi) : "r"(f16));
                o[2 * q + h] = pack_bf16x2(lo, hi);
            }
        }
        dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

template <int LIST, bool SCALED>
__global__ void __launch_bounds__(kThreads, 1)
    index_rows_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK, const IndexRowsArgs P) {
    extern __shared__ uint8_t smem_raw[];
    Smem<LIST> &S = *reinterpret_cast<Smem<LIST> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                    ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = (P.Sq + 127) / 128;
    const long long nunits = static_cast<long long>(ntiles) * P.B * P.H_kv;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.k_full[s], 1);
            mbar_init(&S.k_empty[s], 1);
        }
        mbar_init(&S.q_full, 1);
        mbar_init(&S.q_empty, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S.acc_full[a], 1);
            mbar_init(&S.acc_empty[a], 4);          // the four warps of the owning warpgroup
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

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        int itk = 0, nq = 0;
        bool ok = true;
        for (int r = 0; ok; ++r) {
            const long long u = unit_index(r);
            if (u >= nunits) break;
            const Unit x = unit_at(P, u, ntiles);
            const int kh = P.KH == 1 ? 0 : x.g;   // shared index keys: one row per token
            if (!x.valid) {
                if (x.i0 == 0 && x.g == 0) set_status(P.status, kStatusBadLens);
                continue;
            }
            if (nq > 0 && (*abort_flag || !mbar_wait(&S.q_empty, (nq - 1) & 1, P.status))) {
                ok = false;
                break;
            }
            const int qrow = x.b * P.Sq + x.i0;
            mbar_arrive_expect_tx(&S.q_full, kQBytes);
            tma_load_3d(S.q, &tmQ, 0, x.g, qrow, &S.q_full);
            tma_load_3d(S.q + 16384, &tmQ, 64, x.g, qrow, &S.q_full);
            ++nq;
            for (int j = 0; j <= x.jmax; j += 2, ++itk) {
                const int s = itk % kStages;
                if (itk >= kStages &&
                    (*abort_flag || !mbar_wait(&S.k_empty[s], ((itk / kStages) - 1) & 1, P.status))) {
                    ok = false;
                    break;
                }
                const int nb = min(2, x.jmax - j + 1);
                mbar_arrive_expect_tx(&S.k_full[s], nb * 32768);
                for (int jj = 0; jj < nb; ++jj) {
                    const int tok = static_cast<int>(kv_block_row(P.kv, x.b, j + jj, P.status));
                    tma_load_3d(S.ring[s] + jj * 16384, &tmK, 0, kh, tok, &S.k_full[s]);
                    tma_load_3d(S.ring[s] + 32768 + jj * 16384, &tmK, 64, kh, tok, &S.k_full[s]);
                }
            }
        }
        if (!ok) *abort_flag = 1;
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        int itk = 0, ita = 0, nq = 0;
        bool ok = true;
        for (int r = 0; ok; ++r) {
            const long long u = unit_index(r);
            if (u >= nunits) break;
            const Unit x = unit_at(P, u, ntiles);
            if (!x.valid) continue;
            if (*abort_flag || !mbar_wait(&S.q_full, nq & 1, P.status)) { ok = false; break; }
            ++nq;
            tc_fence_after();
            const uint32_t qa = smem_u32(S.q);
            for (int j = 0; j <= x.jmax; j += 2, ++itk, ++ita) {
                const int s = itk % kStages, a = ita & 1;
                if (*abort_flag || !mbar_wait(&S.k_full[s], (itk / kStages) & 1, P.status)) {
                    ok = false;
                    break;
                }
                if (ita >= 2 && (*abort_flag || !mbar_wait(&S.acc_empty[a], ((ita >> 1) - 1) & 1,
                                                           P.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nb = min(2, x.jmax - j + 1);
                const uint32_t idesc = umma_idesc_bf16(128, nb * 128);
                const uint32_t kb = smem_u32(S.ring[s]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = umma_desc_sw128(qa + (kk >> 2) * 16384 + (kk & 3) * 32);
                    const uint64_t bd = umma_desc_sw128(kb + (kk >> 2) * 32768 + (kk & 3) * 32);
                    umma_bf16_ss(tmem + a * 256, ad, bd, idesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&S.k_empty[s]);
                umma_commit(&S.acc_full[a]);
                if (j + 2 > x.jmax) umma_commit(&S.q_empty);
            }
        }
        if (!ok) {
            *abort_flag = 1;
            // Let every MMA already issued finish before TMEM is released.
            if (ita > 0) mbar_wait(&S.acc_full[(ita - 1) & 1], ((ita - 1) >> 1) & 1, nullptr);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ epilogue
        // Two warpgroups take alternate accumulator buffers (pairs of key
        // blocks).  Each keeps its own running list per row; at the end of a
        // unit warpgroup 1 hands its list to warpgroup 0, which merges and
        // writes the row's selection.  A warpgroup that hits a timeout keeps
        // stepping through the unit-end barriers so the other never waits on it.
        const int wg = (warp - 4) >> 2;
        const int r = (warp & 3) * 32 + lane;        // TMEM lane = tile row
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const int keep = P.K - 1;                    // non-own blocks kept per row
        TopList<LIST> top;
        int ita = 0;
        bool ok = true;
        for (int rr = 0;; ++rr) {
            const long long u = unit_index(rr);
            if (u >= nunits) break;
            const Unit x = unit_at(P, u, ntiles);
            const bool row_ok = r < x.nrows;
            const long long out_off =
                ((static_cast<long long>(x.b) * P.Sq + x.i0 + r) * P.H_kv + x.g) * P.K;
            if (!x.valid) {
                if (row_ok && wg == 0)
                    for (int q = 0; q < P.K; ++q) {
                        P.ids[out_off + q] = -1;
                        P.out_scores[out_off + q] = -INFINITY;
                    }
                continue;
            }
            const long long p = x.p_first + r;        // this row's query position
            const int own = static_cast<int>(p / kBlock);
            float s_own = -INFINITY;
            bool has_own = false;
            top.reset(keep);
            for (int j = 0; j <= x.jmax; j += 2, ++ita) {
                const int a = ita & 1;
                if (a != wg) continue;
                if (ok) {
                    bool have = !*abort_flag && mbar_wait(&S.acc_full[a], (ita >> 1) & 1, P.status);
                    have = __all_sync(0xffffffffu, have);
                    if (!have) { ok = false; *abort_flag = 1; }
                }
                if (ok) {
                    tc_fence_after();
                    const int nb = min(2, x.jmax - j + 1);
                    for (int jj = 0; jj < nb; ++jj) {
                        const int J = j + jj;
                        const long long t0 = static_cast<long long>(J) * kBlock;
                        const bool full = t0 + kBlock - 1 <= x.p_first;   // no masking for any row
                        float m = -INFINITY;
                        if (SCALED) {
                            // E4M3 keys (widened exactly to bf16 for the MMA): each
                            // token's score is its row scale times the dot.
                            const long long krow = kv_block_row(P.kv, x.b, J, P.status);
                            const float *sc = P.k_scale + krow * P.KH + (P.KH == 1 ? 0 : x.g);
#pragma unroll
                            for (int c = 0; c < 4; c += 2) {
                                uint32_t va[32], vb[32];
                                tmem_ld32r(lane_addr + a * 256 + jj * 128 + c * 32, va);
                                tmem_ld32r(lane_addr + a * 256 + jj * 128 + c * 32 + 32, vb);
                                tmem_wait_ld(va);
                                tmem_tie(vb);
#pragma unroll
                                for (int e = 0; e < 32; ++e) {
                                    const int c0 = c * 32 + e, c1 = c0 + 32;
                                    if (t0 + c0 <= p) m = fmaxf(m, __uint_as_float(va[e]) * __ldg(sc + c0 * P.KH));
                                    if (t0 + c1 <= p) m = fmaxf(m, __uint_as_float(vb[e]) * __ldg(sc + c1 * P.KH));
                                }
                            }
                        } else
#pragma unroll
                        for (int c = 0; c < 4; c += 2) {
                            uint32_t va[32], vb[32];
                            tmem_ld32r(lane_addr + a * 256 + jj * 128 + c * 32, va);
                            tmem_ld32r(lane_addr + a * 256 + jj * 128 + c * 32 + 32, vb);
                            tmem_wait_ld(va);
                            tmem_tie(vb);
                            if (full) {
                                // four independent max chains instead of one serial one
                                float m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
                                for (int e = 0; e < 32; e += 4) {
                                    m = fmax3(m, __uint_as_float(va[e]), __uint_as_float(vb[e]));
                                    m1 = fmax3(m1, __uint_as_float(va[e + 1]), __uint_as_float(vb[e + 1]));
                                    m2 = fmax3(m2, __uint_as_float(va[e + 2]), __uint_as_float(vb[e + 2]));
                                    m3 = fmax3(m3, __uint_as_float(va[e + 3]), __uint_as_float(vb[e + 3]));
                                }
                                m = fmax3(m, m1, fmaxf(m2, m3));
                            } else {
#pragma unroll
                                for (int e = 0; e < 32; ++e) {
                                    if (t0 + c * 32 + e <= p) m = fmaxf(m, __uint_as_float(va[e]));
                                    if (t0 + c * 32 + 32 + e <= p) m = fmaxf(m, __uint_as_float(vb[e]));
                                }
                            }
                        }
                        if (J < own) top.offer(topk_key(m, J));
                        else if (J == own) { s_own = m; has_own = true; }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.acc_empty[a]);
            }
            // Warpgroup 1 hands over its list; warpgroup 0 merges and writes.
            if (wg == 1) {
#pragma unroll
                for (int i = 0; i < LIST; ++i) S.xkeys[i][r] = top.L[i];
                S.xown[r] = s_own;
                S.xhas[r] = has_own;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (wg == 0) {
#pragma unroll
                for (int i = 0; i < LIST; ++i) {
                    const unsigned long long k2 = S.xkeys[i][r];
                    if (k2 != 0ull && k2 != ~0ull) top.offer(k2);
                }
                if (S.xhas[r]) s_own = S.xown[r];
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (wg != 0 || !ok || !row_ok) continue;
            // Kept non-own blocks (all ids < own) ascending, then the own block.
            // They sit in slots [LIST - keep, LIST - keep + n_other), best first.
            const int n_other = min(own, keep);
            const int lo = LIST - keep, hi = LIST - keep + n_other;
            int32_t *ids_out = P.ids + out_off;
            float *sc_out = P.out_scores + out_off;
#pragma unroll
            for (int i = 0; i < LIST; ++i) {
                if (i < lo || i >= hi) continue;
                const int id = topk_key_id(top.L[i]);
                int rank = 0;
#pragma unroll
                for (int k2 = 0; k2 < LIST; ++k2)
                    if (k2 >= lo && k2 < hi && topk_key_id(top.L[k2]) < id) ++rank;
                ids_out[rank] = id;
                sc_out[rank] = key_score(top.L[i]);
            }
            ids_out[n_other] = own;
            sc_out[n_other] = s_own;
            for (int q = n_other + 1; q < P.K; ++q) {
                ids_out[q] = -1;
                sc_out[q] = -INFINITY;
            }
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

}  // namespace

cudaError_t launch_widen_e4m3(const void *src, void *dst, long long rows, cudaStream_t s) {
    const long long n16 = rows * (kDim / 16);
    TraceScope trace(s, "index_widen_e4m3");
    widen_e4m3_kernel<<<device_sm_count() * 8, 256, 0, s>>>(static_cast<const uint4 *>(src),
                                                            static_cast<uint4 *>(dst), n16);
    return cudaGetLastError();
}

cudaError_t launch_index_rows_tc(const IndexRowsArgs &a, cudaStream_t s) {
    static_assert(sizeof(Smem<16>) + 1024 <= 227 * 1024, "shared memory budget");
    static_assert(sizeof(Smem<32>) + 1024 <= 227 * 1024, "shared memory budget");
    static_assert(sizeof(Smem<64>) + 1024 <= 227 * 1024, "shared memory budget");
    CUtensorMap tq, tk;
    if (!encode_kv_tensor_map(&tq, a.q_idx, a.H_kv, static_cast<long long>(a.B) * a.Sq) ||
        !encode_kv_tensor_map(&tk, a.k_idx, a.KH, a.kv.capacity))
        return cudaErrorInvalidValue;
    const long long ntiles = (a.Sq + 127) / 128;
    const long long units = ntiles * a.B * a.H_kv;
    const long long grid = units < device_sm_count() ? units : device_sm_count();
    auto go = [&](auto kern, size_t smem) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        TraceScope trace(s, "index_score_maxpool_topk_rows_tc");
        kern<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(tq, tk, a);
        return cudaGetLastError();
    };
    // E4M3 keys (row scales on the scores) get their own instantiation so the
    // bf16 kernels keep their register allocation.
    if (a.k_scale) {
        if (a.K <= 16) return go(index_rows_tc_kernel<16, true>, sizeof(Smem<16>) + 1024);
        if (a.K <= 32) return go(index_rows_tc_kernel<32, true>, sizeof(Smem<32>) + 1024);
        if (a.K <= 64) return go(index_rows_tc_kernel<64, true>, sizeof(Smem<64>) + 1024);
    }
    if (a.K <= 16) return go(index_rows_tc_kernel<16, false>, sizeof(Smem<16>) + 1024);
    if (a.K <= 32) return go(index_rows_tc_kernel<32, false>, sizeof(Smem<32>) + 1024);
    if (a.K <= 64) return go(index_rows_tc_kernel<64, false>, sizeof(Smem<64>) + 1024);
    return cudaErrorInvalidValue;
}

}  // namespace msa
