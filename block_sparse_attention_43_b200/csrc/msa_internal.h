// msa_internal.h -- host-side launchers of the MSA kernels (not exported).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "msa.h"

namespace msa {

// Where the tokens of a sequence live in the [capacity, H_kv, 128] caches:
// packed (sequence b starts at row offsets[b]) or paged (block j of sequence
// b is the 128-row page pages[b * pages_per_seq + j]).
struct KvMap {
    const int64_t *offsets;   // packed layout, or nullptr
    const int32_t *pages;     // paged layout, or nullptr
    int pages_per_seq;
    long long capacity;       // rows in the caches
};

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Records a CUDA event pair around the kernel launched in its scope when the
// trace is enabled (msa_trace_enable); a no-op otherwise.
class TraceScope {
  public:
    TraceScope(cudaStream_t s, const char *name);
    ~TraceScope();

  private:
    cudaStream_t stream_;
    int slot_;
};

// Block max-pooled index scores for decode (one query row per sequence):
// scores[b][g][j] = max over tokens t of block j (t < lens[b]) of
// dot(q_idx[b][0][g], k_idx[kv_offsets[b] + t][g]).
struct IndexDecodeArgs {
    const void *q_idx;
    const void *k_idx;
    const int32_t *lens;
    KvMap kv;
    float *scores;          // [B][H_kv][nb_max]
    int *status;
    int B, H_kv, nb_max, max_kv_len;
};
cudaError_t launch_index_decode(const IndexDecodeArgs &a, cudaStream_t s);

// Decode index branch on the other index-key formats (index_decode_variants.cu):
// keys shared by the H index heads ([T][1][128], bf16 or E4M3) or one E4M3 key
// per index head ([T][H][128]); E4M3 rows carry an fp32 scale (k_scale [T][KH]).
struct IndexDecodeVarArgs {
    const void *q_idx;      // [B][H][128] bf16
    const void *k_idx;      // [T][KH][128] bf16 or E4M3
    const float *k_scale;   // [T][KH] (E4M3 only)
    const int32_t *lens;
    KvMap kv;
    float *scores;          // [B][H][nb_max]
    int *status;
    int B, H, KH, nb_max, max_kv_len;
    int fp8;
};
cudaError_t launch_index_decode_variant(const IndexDecodeVarArgs &a, cudaStream_t s);

// Index branch for q_len >= 1 query rows per sequence (prefill), causal:
// block max-pooled scores of every visible block and the top-k selection,
// written straight to ids / out_scores [B*Sq][H_kv][K].
struct IndexRowsArgs {
    const void *q_idx;      // [B][Sq][H_kv][128]
    const void *k_idx;
    const int32_t *lens;
    KvMap kv;
    int32_t *ids;
    float *out_scores;
    int *status;
    int B, Sq, H_kv, K, max_kv_len;   // H_kv here: index heads
    int KH;                           // index-key rows per token: H_kv, or 1 (shared)
    const float *k_scale;             // E4M3 keys (widened to bf16 in k_idx): row scales [T][KH]
};
// E4M3 codes [rows][128] -> bf16 [rows][128], exact (index_rows_tc.cu).
cudaError_t launch_widen_e4m3(const void *src, void *dst, long long rows, cudaStream_t s);
// tcgen05 tensor-core kernel (index_rows_tc.cu).
cudaError_t launch_index_rows_tc(const IndexRowsArgs &a, cudaStream_t s);

// Top-k block selection per (row, group) from a block-score buffer.
struct TopkArgs {
    const float *scores;    // [B*Sq][H_kv][nb_max]
    const int32_t *lens;
    KvMap kv;
    int32_t *ids;           // [B*Sq][H_kv][K]
    float *out_scores;      // [B*Sq][H_kv][K]
    int *status;
    int B, Sq, H_kv, nb_max, K, max_kv_len;
};
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t s);

// Sparse attention, one CTA per (row, group, split) over the kept blocks.
struct AttnRowsArgs {
    const void *q;          // [B][Sq][H_q][128]
    const void *k_cache;
    const void *v_cache;
    const int32_t *ids;     // [B*Sq][H_kv][K]
    const int32_t *lens;
    KvMap kv;
    void *out;              // [B][Sq][H_q][128]
    float *lse;             // optional [rows][H_q]: base-2 log-sum-exp (as PrefillArgs)
    float *partials;        // [B*Sq][H_kv][nsplit][attn_partial_floats(G)]
    int *tickets;           // [B*Sq][H_kv]
    int *status;
    int B, Sq, H_q, H_kv, K, nsplit, max_kv_len;
    int n_idx;              // index heads: group g reads ids of g / (H_kv / n_idx)
    float softmax_scale;
};
cudaError_t launch_attn_rows(const AttnRowsArgs &a, cudaStream_t s);
// Splits used by launch_attn_rows for this shape (workspace sizing too).
int attn_rows_nsplit(long long rows_x_groups, int top_k);
// Floats of one split partial for G heads: m[G], l[G], padding to 16 bytes,
// then o[G][128] (so the o rows can be read as float4).
__host__ __device__ inline int attn_partial_floats(int G) { return ((2 * G + 3) & ~3) + G * 128; }
__host__ __device__ inline int attn_partial_o_offset(int G) { return (2 * G + 3) & ~3; }

// Prefill sparse attention organised around the KV blocks (attn_prefill.cu).
struct PrefillArgs {
    const void *q;          // [B][Sq][H_q][128]
    const void *k_cache;
    const void *v_cache;
    const int32_t *ids;     // [B*Sq][H_kv][K]
    const int32_t *lens;
    KvMap kv;
    void *out;
    int *status;
    int B, Sq, H_q, H_kv, K, max_kv_len;
    int n_idx;              // index heads: group g reads ids of g / (H_kv / n_idx)
    float softmax_scale;
    float *lse;             // optional [rows][H_q]: base-2 log-sum-exp of the
                            // scaled logits (p = 2^(s * scale * log2 e - lse))
    int item_rows;          // max rows per bucket work item
    // workspace views (filled by launch_prefill_attention)
    int *bucket_cnt, *bucket_cur, *bucket_off, *bucket_rows;  // per (range, block j)
    int *item_off;          // first item of each bucket, counted inside its range
    int *item_bucket;       // [range][item] -> block j
    int *item_desc;         // [item] {b, g, j, n}, {first bucket entry, L, 0, 0}
    float *bucket_shift;    // [bucket entry][8 heads] softmax shift of the entry's row
    long long *range_count, *range_item_off;
    long long *item_total;
    long long *item_next;   // claim counters of pass A and pass B (zeroed per call)
    __half *o_acc;          // [rows][H_kv][128 dims x 8 heads] fp16, heads interleaved per 8 dims
    float *l_acc, *m_arr;   // [rows][H_q] softmax sums and shifts (base 2)
    uint8_t *flags;         // [rows][H_q] 1: recomputed by the exact pass
    int *flag_count;
    float acc_limit;        // largest partial value added in fp16: 65504 / top_k
    int nb_max, n_ranges, rows_per_range, items_per_range;
    long long n_ranges_total;
};
struct PrefillLayout {
    size_t cnt, cur, l_acc, flags, zero_end, off, item_off, item_bucket, range_count,
        range_item_off, rows, shift, item_desc, o_acc, m_arr, total;
    int nb_max, n_ranges, rows_per_range, items_per_range, item_rows;
    long long n_ranges_total, n_buckets;
};
bool prefill_attention_supported(int H_q, int H_kv);
size_t prefill_workspace_layout(int B, int Sq, int H_q, int H_kv, int K, int max_kv_len,
                                PrefillLayout *L);
cudaError_t launch_prefill_attention(const PrefillArgs &a, uint8_t *ws, const PrefillLayout &L,
                                     cudaStream_t s);
// Buckets alone (rows that kept block j != own, per range of range_rows
// query rows, as work items of at most item_rows rows), laid out from byte
// `base` of a workspace; returns the end.  The item count lands in
// *item_total, the 32-byte descriptors in item_desc.
size_t prefill_bucket_layout(int B, int Sq, int H_kv, int K, int max_kv_len, int item_rows,
                             int range_rows, size_t base, PrefillLayout *L);
cudaError_t launch_prefill_buckets(PrefillArgs &a, uint8_t *ws, const PrefillLayout &L,
                                   long long *item_total, cudaStream_t s);
// 3-D map over q [rows, H_q, 128] with a box of 64 dims x 8 heads x box_rows
// rows, 128-byte swizzle.
bool encode_q_rows_map(CUtensorMap *map, const void *q, int H_q, long long rows, int box_rows);

// Appends n_new tokens per sequence after its current length (kv_append.cu):
// src[i] [B][n_new][H_kv][128] -> dst[i] at rows of tokens lens[b] .. + n_new - 1.
// Whole decode step in one persistent launch (decode_fused.cu): index
// scores, top-k per (sequence, index head) and sparse attention.
constexpr int kCtrStride = 32;
struct DecodeFusedArgs {
    const void *q_idx;      // [B][n_idx][128]
    const void *k_idx;      // [T][n_idx][128]
    const void *q;          // [B][H_q][128]
    const void *k_cache;
    const void *v_cache;
    const int32_t *lens;
    KvMap kv;
    int32_t *ids;           // [B][n_idx][K]
    float *out_scores;      // [B][n_idx][K]
    void *out;              // [B][H_q][128]
    int *status;
    // workspace views
    float *scores;          // [B][n_idx][nb_max] block scores
    int *seq_done;          // [B] index units finished
    int *aq_item;           // [B*H_kv] published attention items (b*H_kv + g)
    int *aq_flag;           // [B*H_kv] 1 once the item above is published
    int *ctr;               // one 128-byte line each (stride kCtrStride ints): next index unit,
                            // allocated items, next item claimed, items published
    int B, H_q, H_kv, K, nb_max, max_kv_len;
    int n_idx;              // index heads; group g reads the selection of g / (H_kv / n_idx)
    float softmax_scale;
};
struct DecodeFusedLayout {
    size_t scores, ctr, seq_done, aq_item, aq_flag, zero_lo, zero_hi, total;
};
size_t decode_fused_layout(int B, int H_q, int H_kv, int n_idx, int K, int max_kv_len,
                           DecodeFusedLayout *L);
cudaError_t launch_decode_fused(const DecodeFusedArgs &a, cudaStream_t s);

// Backward of the sparse branch (attn_bwd.cu), organised around the KV
// blocks.  The caller has run the forward into o and lse (the workspace
// regions of AttnBwdLayout) on the same stream.
struct AttnBwdArgs {
    const void *q;          // [B][Sq][H_q][128]
    const void *k_cache;
    const void *v_cache;
    const void *dout;       // [B][Sq][H_q][128]
    const int32_t *ids;     // [B*Sq][n_idx][K]
    const int32_t *lens;
    KvMap kv;
    void *dq;               // [B][Sq][H_q][128] bf16, written
    float *dk, *dv;         // [capacity][H_kv][128] fp32, added to
    int *status;
    int B, Sq, H_q, H_kv, n_idx, K, max_kv_len;
    float softmax_scale;
    // workspace views (filled by launch_attn_bwd)
    const void *o;          // [rows][H_q][128] bf16: the recomputed forward output
    const float *lse;       // [rows][H_q] base-2 log-sum-exp of the scaled logits
    float *delta;           // [rows][H_q] dO . O
    float *dq_acc;          // [rows][H_q][128] fp32, already scaled
    const int *bucket_rows; // bucket entries -> flattened row
    const int *item_desc;   // bucket work items (32 bytes each)
    const long long *item_total;
    long long *item_next;   // claim counter
};
struct AttnBwdLayout {
    size_t o, lse, delta, dq_acc, total;
    PrefillLayout bk;       // the backward's own buckets (unless reused)
    bool reuse;             // the forward's prefill buckets are the same items
    size_t fwd_rows, fwd_desc;
};
// Lays the backward's regions out from byte `base` of the workspace (the
// forward's layout ends there); returns the total size.  fwd: the forward's
// prefill layout when it ran the block-outer path (its bucket items are
// reused when they are the backward's), else nullptr.
size_t attn_bwd_layout(int B, int Sq, int H_q, int H_kv, int K, int max_kv_len, size_t base,
                       const PrefillLayout *fwd, AttnBwdLayout *L);
cudaError_t launch_attn_bwd(const AttnBwdArgs &a, uint8_t *ws, const AttnBwdLayout &L,
                            cudaStream_t s);

struct KvAppendArgs {
    const void *src[3];
    void *dst[3];
    const int32_t *lens;
    KvMap kv;
    int *status;
    int B, n_new, H_kv, max_kv_len;
    int H_idx;              // index-key rows per token (src[0] / dst[0])
};
cudaError_t launch_kv_append(const KvAppendArgs &a, cudaStream_t s);

// Encodes a [capacity, H_kv, 128] bf16 cache as a 3-D TMA tensor map whose
// box is (64 dims, 1 group, 128 tokens) with 128-byte swizzling.
bool encode_kv_tensor_map(CUtensorMap *map, const void *base, int H_kv, long long capacity);

}  // namespace msa
