/*
 * msa.h -- C ABI of the B200 (sm_100a) MiniMax Sparse Attention library.
 *
 * MiniMax Sparse Attention (MSA) runs attention in two stages:
 *
 *   index branch  ("百万token上下文提速近10倍，MiniMax M3的稀疏注意力凭什么这么快",
 *                 cloud.tencent.com, section 二): one lightweight index query
 *                 per GQA group is dotted with a per-token index key; the
 *                 scores are max-pooled over each 128-token KV block ("Block
 *                 Max Pool") and the top-k blocks are kept ("Top-k").
 *   sparse branch (same section): full softmax attention runs over the kept
 *                 blocks only.  Every query head of a GQA group uses the
 *                 group's one block set (same article, section 六).
 *
 * Block size 128, top-k 16 and index dimension 128 are the configuration the
 * mlqm.cn MiniMax-M3 guide prints ("sparse_block_size", "sparse_topk_blocks",
 * "sparse_index_dim").  The pages give no formula; this library fixes:
 *   - index score s[t] = dot(q_idx[b,i,g,:], k_idx[t,g,:]), no scale, for
 *     index head g (one per GQA group unless num_index_heads says fewer);
 *   - block score S[j] = max of s[t] over the tokens t of block j with
 *     t <= p, where p = lens[b] - q_len + i is the query's position;
 *   - the query's own block floor(p/128) is always kept; the other k-1 slots
 *     go to the highest block scores among blocks j < own, ties to the lower
 *     block id; with at most k visible blocks all are kept;
 *   - sparse branch: softmax(softmax_scale * q.k) over the keys t <= p of the
 *     kept blocks, applied to v; head h belongs to group h / (H_q / H_kv).
 *
 * Index-branch variants.  The guide's configuration also prints
 * "sparse_num_index_heads: 4", which one index query per group cannot match;
 * the pages say nothing more, so this library reads it as Hi index heads that
 * partition the groups into contiguous sets: group g uses index head
 * g / (H_kv / Hi) (Hi = H_kv is the default, one per group).  Index keys may
 * be one row per (token, index head) or one row per token shared by every
 * index head, in bf16 or in FP8 E4M3 with one fp32 scale per key row (score
 * = scale * dot(q_idx, decoded key)); see index_key_format.
 *
 * Layouts (all row-major, head dim innermost, bf16 = IEEE bfloat16 bits):
 *   q_idx  [B, q_len, Hi, index_dim]       q   [B, q_len, H_q, head_dim]
 *   k_cache, v_cache: packed [kv_capacity, H_kv, dim]; k_idx: packed
 *          [kv_capacity, KH, index_dim] with KH = Hi, or 1 for shared index
 *          keys; sequence b owns rows kv_offsets[b] .. kv_offsets[b] +
 *          lens[b] - 1 (a padded cache is the case kv_offsets[b] = b * stride).
 *   block_ids [B, q_len, Hi, top_k] int32, ascending, -1 padded
 *   block_scores: same shape, float32, -inf padded
 *   out    [B, q_len, H_q, head_dim] bf16 (round to nearest even)
 *
 * Ownership: every pointer is caller-owned device memory (lens and
 * kv_offsets included) and stays caller-owned; the library allocates no
 * device memory and keeps no pointer after a call returns.  Work is enqueued
 * on the caller's stream; no call synchronises except
 * msa_read_device_status.  The workspace must hold at least the bytes the
 * matching *_workspace_size call returns, 256-byte aligned, and must not be
 * shared by calls that may run concurrently.
 *
 * Errors: problems visible on the host (null pointers, unsupported sizes, a
 * short or misaligned workspace, misaligned tensors) return a status before
 * anything is launched.  A failed launch returns MSA_ERR_CUDA.  Problems that
 * only the device can see (lens[b] < q_len, lens[b] > max_kv_len, a sequence
 * that runs past kv_capacity, a bounded wait that gave up) set a status word
 * inside the workspace: the affected outputs are written as -1 / -inf / NaN,
 * nothing outside the caller's buffers is touched, and
 * msa_read_device_status reports the word.  The library never traps.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st *msa_stream_t;

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, H_q % H_kv != 0 */
    MSA_ERR_UNSUPPORTED = 2,    /* a size this library does not handle (see below) */
    MSA_ERR_WORKSPACE = 3,      /* workspace missing, too small or not 256-byte aligned */
    MSA_ERR_CUDA = 4,           /* a CUDA call or kernel launch failed */
    MSA_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait gave up (device status) */
    MSA_ERR_BAD_LENS = 6,       /* lens/kv_offsets out of range (device status) */
    MSA_ERR_MISALIGNED = 7      /* a tensor pointer is not 16-byte aligned */
} msa_status_t;

/* Layout of the index keys (msa_shape_t.index_key_format). */
typedef enum {
    MSA_INDEX_KEYS_BF16 = 0,        /* bf16 [kv_capacity, Hi, index_dim]: one key per index head */
    MSA_INDEX_KEYS_BF16_SHARED = 1, /* bf16 [kv_capacity, 1, index_dim]: one key per token */
    MSA_INDEX_KEYS_FP8 = 2,         /* E4M3 [kv_capacity, Hi, index_dim] + fp32 scale [kv_capacity, Hi] */
    MSA_INDEX_KEYS_FP8_SHARED = 3   /* E4M3 [kv_capacity, 1, index_dim] + fp32 scale [kv_capacity, 1] */
} msa_index_key_format_t;

/* Problem shape.  Supported by this library: head_dim == index_dim == 128,
 * block_size == 128, 1 <= top_k <= 64, num_kv_heads in {1, 2, 4, 8, 16},
 * num_q_heads / num_kv_heads in {1, 2, 4, 8, 16}, index heads in {1, 2, 4,
 * 8, 16} dividing num_kv_heads, batch <= 4096, max_kv_len <= 2^27,
 * batch * ceil(max_kv_len / 128) < 2^31, kv_capacity < 2^31. */
typedef struct {
    int32_t batch;        /* B */
    int32_t q_len;        /* query rows per sequence: 1 = decode, lens[b] = full prefill */
    int32_t max_kv_len;   /* upper bound on every lens[b] */
    int32_t num_q_heads;  /* H_q */
    int32_t num_kv_heads; /* H_kv = number of GQA groups */
    int32_t head_dim;     /* D */
    int32_t index_dim;    /* d_idx */
    int32_t block_size;   /* tokens per KV block */
    int32_t top_k;        /* blocks kept per (query row, index head), own block included */
    int64_t kv_capacity;  /* rows in the packed k_idx / k_cache / v_cache */
    int32_t num_index_heads;  /* Hi; 0 means num_kv_heads (one index head per group) */
    int32_t index_key_format; /* msa_index_key_format_t; 0 = bf16, one key per index head */
} msa_shape_t;

/* Bytes of workspace msa_index_topk needs for this shape (0 on bad shape). */
MSA_API size_t msa_index_topk_workspace_size(const msa_shape_t *shape);

/* Index branch: block max-pooled index scores and the top-k block ids of
 * every (query row, index head).  See the header comment for the definition.
 *   q_idx        device bf16 [B, q_len, Hi, index_dim]
 *   k_idx        device bf16 [kv_capacity, KH, index_dim] (KH = Hi, or 1 for
 *                MSA_INDEX_KEYS_BF16_SHARED; the FP8 formats take
 *                msa_index_topk_fp8 and return MSA_ERR_UNSUPPORTED here)
 *   lens         device int32 [B], each in [q_len, max_kv_len]
 *   kv_offsets   device int64 [B], row of token 0 of sequence b
 *   block_ids    device int32 [B, q_len, Hi, top_k]   (written)
 *   block_scores device float [B, q_len, Hi, top_k]   (written)
 *   workspace    device, >= msa_index_topk_workspace_size(shape) bytes */
MSA_API msa_status_t msa_index_topk(const msa_shape_t *shape, const void *q_idx, const void *k_idx,
                            const int32_t *lens, const int64_t *kv_offsets,
                            int32_t *block_ids, float *block_scores,
                            void *workspace, size_t workspace_bytes, msa_stream_t stream);

/* Index branch on FP8 E4M3 index keys (index_key_format MSA_INDEX_KEYS_FP8
 * or MSA_INDEX_KEYS_FP8_SHARED): the score of token t for index head g is
 * k_idx_scale[t, kh] * dot(q_idx[b,i,g,:], decoded k_idx_fp8[t, kh, :]),
 * kh = g (or 0 when shared), accumulated in fp32.  E4M3 is the OCP 8-bit
 * format with bias 7 and no infinities.  For q_len > 1 the workspace also
 * holds an exact bf16 copy of all kv_capacity key rows (see
 * msa_index_topk_workspace_size).
 *   k_idx_fp8    device uint8 [kv_capacity, KH, index_dim] (E4M3 codes)
 *   k_idx_scale  device float [kv_capacity, KH]
 * Other arguments, layouts, results and errors are those of msa_index_topk. */
MSA_API msa_status_t msa_index_topk_fp8(const msa_shape_t *shape, const void *q_idx,
                                        const void *k_idx_fp8, const float *k_idx_scale,
                                        const int32_t *lens, const int64_t *kv_offsets,
                                        int32_t *block_ids, float *block_scores, void *workspace,
                                        size_t workspace_bytes, msa_stream_t stream);

/* Bytes of workspace msa_sparse_attention needs for this shape (0 on bad shape). */
MSA_API size_t msa_sparse_attention_workspace_size(const msa_shape_t *shape);

/* Sparse branch: exact softmax attention of every query head over the keys
 * of its group's kept blocks (ids as written by msa_index_topk; -1 entries
 * are skipped; every id must be a visible block, the own block included).
 * Group g takes the ids of index head g / (H_kv / Hi).
 *   q            device bf16 [B, q_len, H_q, head_dim]
 *   k_cache      device bf16 [kv_capacity, H_kv, head_dim]
 *   v_cache      device bf16 [kv_capacity, H_kv, head_dim]
 *   block_ids    device int32 [B, q_len, Hi, top_k]
 *   softmax_scale  multiplies q.k before the softmax (1/sqrt(head_dim) usual)
 *   out          device bf16 [B, q_len, H_q, head_dim]  (written)
 *   workspace    device, >= msa_sparse_attention_workspace_size(shape) bytes */
MSA_API msa_status_t msa_sparse_attention(const msa_shape_t *shape, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *block_ids,
                                  const int32_t *lens, const int64_t *kv_offsets,
                                  float softmax_scale, void *out,
                                  void *workspace, size_t workspace_bytes, msa_stream_t stream);

/* Backward of the sparse branch (training; the pages say MSA is trained
 * natively, "百万token上下文提速近10倍..." section 五).  The index branch's
 * selection is piecewise constant and passes no gradient, so block_ids are an
 * input, as in the forward.  For each (row, head) over its kept keys t:
 *   P = softmax(softmax_scale * q.k_t), dP_t = d_out.v_t,
 *   Delta = sum_t P_t dP_t, dZ_t = P_t (dP_t - Delta),
 *   dq = softmax_scale * sum_t dZ_t k_t,
 *   dk_t += softmax_scale * dZ_t q,   dv_t += P_t d_out.
 * The forward is recomputed inside the call (no saved statistics are
 * needed): its output gives Delta = d_out . out, and it also yields each
 * (row, head)'s log-sum-exp.  The products then run around the kept blocks:
 * each block's dk and dv are summed on chip over all rows that kept it and
 * added once per work item; dq is summed in an fp32 workspace buffer.
 *   q, k_cache, v_cache, block_ids, lens, kv_offsets: as msa_sparse_attention
 *   d_out        device bf16 [B, q_len, H_q, head_dim], gradient of out
 *   dq           device bf16 [B, q_len, H_q, head_dim]  (written; NaN for
 *                sequences with bad lengths and after a device timeout)
 *   dk, dv       device float [kv_capacity, H_kv, head_dim]: the gradients of
 *                this call are ADDED (fp32 atomics, so their summation order
 *                and last bits vary by run); start them at zero.  Keys that
 *                no row reaches are not written.
 *   workspace    >= msa_sparse_attention_backward_workspace_size bytes
 *                (the forward's workspace, then the recomputed output, two
 *                floats per (row, head), the fp32 dq sum and work lists:
 *                about rows x H_q x 776 bytes beyond the forward's) */
MSA_API size_t msa_sparse_attention_backward_workspace_size(const msa_shape_t *shape);
MSA_API msa_status_t msa_sparse_attention_backward(const msa_shape_t *shape, const void *q,
                                                   const void *k_cache, const void *v_cache,
                                                   const int32_t *block_ids, const int32_t *lens,
                                                   const int64_t *kv_offsets, float softmax_scale,
                                                   const void *d_out, void *dq, float *dk,
                                                   float *dv, void *workspace,
                                                   size_t workspace_bytes, msa_stream_t stream);

/* One whole decode step in a single persistent launch: the index branch
 * (scores, block max-pool, top-k with the own block forced) and the sparse
 * branch over the kept blocks, for q_len == 1.  Results are those of
 * msa_index_topk followed by msa_sparse_attention on the same inputs (same
 * selection; the output within the attention tolerance, its partial sums
 * being combined in another order).  The top-k and attention work of a
 * sequence starts as soon as its own index scores are done, overlapping the
 * index streaming of the later sequences (MSA's decode cost is that
 * streaming: "百万token上下文提速近10倍..." section 四).
 * Requirements on top of the shape rules: q_len == 1, bf16 index keys with
 * one row per index head (index_key_format BF16; any num_index_heads the
 * shape allows, group g using the selection of index head
 * g / (num_kv_heads / num_index_heads)), and num_q_heads / num_kv_heads <= 16;
 * otherwise MSA_ERR_UNSUPPORTED (shared and E4M3 index keys go through
 * msa_index_topk / msa_index_topk_fp8 and msa_sparse_attention).  The
 * launch is cooperative (one CTA per SM, all resident); it is not meant to
 * share the GPU with another kernel running at the same time.
 *   q_idx, k_idx, lens, kv_offsets, block_ids, block_scores: as msa_index_topk
 *   q, k_cache, v_cache, softmax_scale, out: as msa_sparse_attention
 *   workspace    device, >= msa_decode_step_workspace_size(shape) bytes,
 *                256-byte aligned; its first word is the device status word */
MSA_API size_t msa_decode_step_workspace_size(const msa_shape_t *shape);
MSA_API msa_status_t msa_decode_step(const msa_shape_t *shape, const void *q_idx,
                                     const void *k_idx, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *lens,
                                     const int64_t *kv_offsets, float softmax_scale,
                                     int32_t *block_ids, float *block_scores, void *out,
                                     void *workspace, size_t workspace_bytes,
                                     msa_stream_t stream);

/* msa_decode_step on paged caches (the layout described below): index keys,
 * keys and values in pools of 128-token pages, block j of sequence b in page
 * page_table[b * pages_per_seq + j].  Same requirements, results, workspace
 * size and errors as msa_decode_step, plus the paged checks below; the
 * results equal msa_decode_step's on a packed copy of the same tokens, bit for
 * bit (the kernel's summation order does not depend on where a block lives). */
MSA_API msa_status_t msa_decode_step_paged(const msa_shape_t *shape, const void *q_idx,
                                           const void *k_idx_pool, const void *q,
                                           const void *k_pool, const void *v_pool,
                                           const int32_t *lens, const int32_t *page_table,
                                           int32_t pages_per_seq, float softmax_scale,
                                           int32_t *block_ids, float *block_scores, void *out,
                                           void *workspace, size_t workspace_bytes,
                                           msa_stream_t stream);

/* Paged caches (a block-table layout for serving): the index keys, keys and
 * values of all sequences live in pools of 128-token pages, [kv_capacity,
 * H_kv, dim] with page p = rows p*128 .. p*128+127, and block j of sequence b
 * (tokens 128j .. 128j+127) is page page_table[b * pages_per_seq + j].  The
 * MSA block and the page are the same 128 tokens, so a kept block is one
 * page.  Requirements: kv_capacity a multiple of 128, pages_per_seq * 128 >=
 * max_kv_len, page_table device int32 [B, pages_per_seq].  A page number
 * outside the pool sets MSA_ERR_BAD_LENS in the device status word; the
 * outputs of that sequence are then unspecified, and nothing outside the
 * pools is read.  Everything else is as for the packed calls above; the
 * results are the same as on a packed copy of the same tokens. */
MSA_API msa_status_t msa_index_topk_paged(const msa_shape_t *shape, const void *q_idx,
                                          const void *k_idx_pool, const int32_t *lens,
                                          const int32_t *page_table, int32_t pages_per_seq,
                                          int32_t *block_ids, float *block_scores,
                                          void *workspace, size_t workspace_bytes,
                                          msa_stream_t stream);
MSA_API msa_status_t msa_sparse_attention_paged(const msa_shape_t *shape, const void *q,
                                                const void *k_pool, const void *v_pool,
                                                const int32_t *block_ids, const int32_t *lens,
                                                const int32_t *page_table, int32_t pages_per_seq,
                                                float softmax_scale, void *out, void *workspace,
                                                size_t workspace_bytes, msa_stream_t stream);

/* Appends n_new tokens to every sequence: new_k, new_v are device bf16
 * [B, n_new, H_kv, 128], new_k_idx device bf16 [B, n_new, KH, 128] (bf16
 * index-key formats only; the FP8 formats return MSA_ERR_UNSUPPORTED); token
 * i of sequence b is written at position
 * lens[b] + i of the packed (kv_offsets) or paged (page_table, pages_per_seq)
 * caches -- pass exactly one of kv_offsets / page_table.  lens is not
 * changed; the caller advances it.  A token that would land at or past
 * max_kv_len or outside the layout is not written and ORs MSA_ERR_BAD_LENS's
 * bit (1) into *device_status when device_status is not null.  This is the
 * step before a decode call (the new token attends to itself). */
MSA_API msa_status_t msa_kv_append(const msa_shape_t *shape, int32_t n_new, const void *new_k_idx,
                                   const void *new_k, const void *new_v, const int32_t *lens,
                                   const int64_t *kv_offsets, const int32_t *page_table,
                                   int32_t pages_per_seq, void *k_idx_cache, void *k_cache,
                                   void *v_cache, int32_t *device_status, msa_stream_t stream);

/* msa_index_topk without a workspace argument, for callers that cannot
 * allocate device memory or hand over a workspace (plugin hosts that pass a
 * kernel only its inputs and outputs, processes whose device memory belongs
 * to another allocator, loops that must not stall on cudaMalloc).  The paper
 * has no counterpart; this is a library convenience.
 *   Scratch: a file-scope device array of 256 B + 4 MiB that every GPU which
 *   loads the library holds until the process exits.  What a call needs of
 *   it depends on the rows:
 *     - decode (q_len == 1): the 256 B header plus one fp32 block score per
 *       (sequence, index head, block), so batch * index heads *
 *       ceil(max_kv_len / 128) may be at most 1,048,576 (e.g. 4 sequences x
 *       8 index heads at 1M tokens, or 64 x 8 at 256k); larger shapes are
 *       rejected with MSA_ERR_WORKSPACE before anything is launched;
 *     - prefill (q_len > 1): the selection happens inside the tensor-core
 *       kernel, so only the 256 B header is used and no shape is refused
 *       for its size.
 *   Only the bf16 index-key formats are accepted (the E4M3 formats return
 *   MSA_ERR_UNSUPPORTED, as msa_index_topk does).
 *   Set-up: the first call on each device looks up the array's device
 *   address with cudaGetSymbolAddress (that device must be current) and
 *   keeps it for later calls; make that first call before any stream
 *   capture.  Tearing down a device's primary context between calls
 *   (cudaDeviceReset) is not supported: the kept address would be stale.
 *   Sharing: every call on a device uses the same array and it keeps the last
 *   call's contents; calls that may overlap on the GPU (different streams,
 *   no ordering) race on it and must be serialised by the caller.
 *   Device-detected errors leave -1 / -inf in the outputs; the status word
 *   stays inside the library's array and is not reported by this call.
 * Other arguments, layouts and results are those of msa_index_topk. */
MSA_API msa_status_t msa_index_topk_static(const msa_shape_t *shape, const void *q_idx,
                                           const void *k_idx, const int32_t *lens,
                                           const int64_t *kv_offsets, int32_t *block_ids,
                                           float *block_scores, msa_stream_t stream);

/* Waits for `stream`, then returns the device status word that the last call
 * using this workspace left (MSA_OK, MSA_ERR_BAD_LENS or
 * MSA_ERR_DEVICE_TIMEOUT), or MSA_ERR_CUDA if the wait or copy failed.  Every
 * call clears the word when it starts. */
MSA_API msa_status_t msa_read_device_status(const void *workspace, msa_stream_t stream);

/* Kernels that msa_set_wait_controls can make wait on something that never
 * happens (bits of stall_mask). */
typedef enum {
    MSA_STALL_NONE = 0,
    MSA_STALL_INDEX_DECODE = 1, /* decode index kernel of msa_index_topk (bf16 keys, one per
                                   index head): its consumer warps wait once on an mbarrier
                                   nobody arrives on */
    MSA_STALL_DECODE_STEP = 2   /* msa_decode_step: each CTA's first attention item waits on
                                   a flag nobody sets */
} msa_stall_t;

/* Testing aid for the bounded device waits; production code never needs it.
 * Every wait inside the kernels (an mbarrier phase, a flag another CTA sets)
 * gives up after a limit, measured from the start of that wait, records
 * MSA_ERR_DEVICE_TIMEOUT in the workspace's status word, lets the copies it
 * already issued land, frees what it holds and returns.  This call sets, for
 * the whole process and every later call until it is called again:
 *   wait_limit_ns  the limit (0 = the default, 2 s);
 *   stall_mask     msa_stall_t bits: the named kernels wait once on something
 *                  that never happens, so their give-up path runs.  The call
 *                  still returns MSA_OK; msa_read_device_status then reports
 *                  MSA_ERR_DEVICE_TIMEOUT and that call's outputs are
 *                  unspecified (no memory outside the caller's buffers and
 *                  the workspace is touched).  Clear the mask and the next
 *                  call works normally on the same workspace.
 * The values travel to the device in the workspace header (bytes 128..143),
 * which every call fills right after clearing it.  Not meant to be changed
 * while other threads are issuing calls.  Returns MSA_OK. */
MSA_API msa_status_t msa_set_wait_controls(uint64_t wait_limit_ns, uint32_t stall_mask);

/* Kernel timing trace (off by default).  After msa_trace_enable(1), every
 * call records a pair of CUDA events around each kernel it launches, on that
 * call's stream, from a pool of events created by msa_trace_enable (up to
 * 4096 kernels between reads; later launches go unrecorded).
 * msa_trace_read waits for the recorded events, copies out up to
 * max_entries records in launch order (kernel name, milliseconds between the
 * pair) and forgets every record; it returns the number copied, or -1 if a
 * CUDA call failed.  Names are static strings.  msa_trace_enable(0) stops
 * recording and drops unread records. */
MSA_API msa_status_t msa_trace_enable(int on);
MSA_API int msa_trace_read(const char **names, float *ms, int max_entries);

/* Static, human-readable name of a status code. */
MSA_API const char *msa_status_string(msa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
