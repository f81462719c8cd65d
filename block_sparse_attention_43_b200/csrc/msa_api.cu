// msa_api.cu -- the C ABI declared in include/msa.h: argument checks,
// workspace layout, launch sequence and the device status word.
#include <string.h>

#include <atomic>
#include <mutex>

#include "msa.h"
#include "msa_device.cuh"
#include "msa_internal.h"

namespace msa {

int device_sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool encode_kv_tensor_map(CUtensorMap *map, const void *base, int H_kv, long long capacity) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(H_kv),
                                static_cast<cuuint64_t>(capacity)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDim) * 2,
                                   static_cast<cuuint64_t>(kDim) * 2 * H_kv};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kBlock)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_q_rows_map(CUtensorMap *map, const void *q, int H_q, long long rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(H_q),
                                static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDim) * 2,
                                   static_cast<cuuint64_t>(kDim) * 2 * H_q};
    const cuuint32_t box[3] = {64, 8, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace msa

using namespace msa;

namespace {

constexpr size_t kAlign = 256;

// Wait controls set by msa_set_wait_controls, copied into every workspace
// header a call clears (bytes 128..143; see msa_device.cuh).
struct WaitControls {
    unsigned long long limit_ns;
    unsigned stall;
    unsigned never;     // stays 0: the word a stalled wait polls
};
std::mutex g_ctl_mu;
WaitControls g_ctl = {0, 0, 0};
std::atomic<bool> g_ctl_on{false};

// Clears the first `bytes` of a workspace (header first) and writes the
// wait controls into its header when a test has set them.
cudaError_t clear_header(void *ws, size_t bytes, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(ws, 0, bytes, s);
    if (e != cudaSuccess || !g_ctl_on.load(std::memory_order_acquire)) return e;
    WaitControls c;
    {
        std::lock_guard<std::mutex> lock(g_ctl_mu);
        c = g_ctl;
    }
    // From pageable memory: the source is staged before this returns.
    return cudaMemcpyAsync(static_cast<uint8_t *>(ws) + kCtlLimitWord * 4, &c, sizeof(c),
                           cudaMemcpyHostToDevice, s);
}

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool pow2_le16(int x) { return x == 1 || x == 2 || x == 4 || x == 8 || x == 16; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Index heads (0 in the shape: one per group), index-key rows per token, key dtype.
int index_heads(const msa_shape_t *s) {
    return s->num_index_heads > 0 ? s->num_index_heads : s->num_kv_heads;
}
int key_heads(const msa_shape_t *s) {
    return (s->index_key_format == MSA_INDEX_KEYS_BF16_SHARED ||
            s->index_key_format == MSA_INDEX_KEYS_FP8_SHARED)
               ? 1
               : index_heads(s);
}
bool key_fp8(const msa_shape_t *s) {
    return s->index_key_format == MSA_INDEX_KEYS_FP8 || s->index_key_format == MSA_INDEX_KEYS_FP8_SHARED;
}

// Shape checks shared by both calls.
msa_status_t check_shape(const msa_shape_t *s) {
    if (!s) return MSA_ERR_INVALID_ARG;
    if (s->batch < 1 || s->q_len < 1 || s->max_kv_len < 1 || s->num_q_heads < 1 ||
        s->num_kv_heads < 1 || s->top_k < 1 || s->kv_capacity < 1 || s->head_dim < 1 ||
        s->index_dim < 1 || s->block_size < 1)
        return MSA_ERR_INVALID_ARG;
    if (s->num_q_heads % s->num_kv_heads) return MSA_ERR_INVALID_ARG;
    if (s->num_index_heads < 0 || s->index_key_format < MSA_INDEX_KEYS_BF16 ||
        s->index_key_format > MSA_INDEX_KEYS_FP8_SHARED)
        return MSA_ERR_INVALID_ARG;
    if (s->num_kv_heads % index_heads(s)) return MSA_ERR_INVALID_ARG;
    if (s->q_len > s->max_kv_len) return MSA_ERR_INVALID_ARG;
    if (s->head_dim != kDim || s->index_dim != kDim || s->block_size != kBlock)
        return MSA_ERR_UNSUPPORTED;
    if (s->top_k > 64 || !pow2_le16(s->num_kv_heads) || !pow2_le16(index_heads(s)) ||
        !pow2_le16(s->num_q_heads / s->num_kv_heads))
        return MSA_ERR_UNSUPPORTED;
    if (s->batch > 4096 || s->max_kv_len > (1 << 27) || s->kv_capacity >= (1LL << 31))
        return MSA_ERR_UNSUPPORTED;
    // Work units (one 128-token block of one sequence) are counted in 32 bits;
    // sequences may share cache rows, so bound the count by batch x blocks.
    if (static_cast<long long>(s->batch) * ((s->max_kv_len + kBlock - 1) / kBlock) >= (1LL << 31))
        return MSA_ERR_UNSUPPORTED;
    return MSA_OK;
}

long long rows_of(const msa_shape_t *s) { return static_cast<long long>(s->batch) * s->q_len; }

int nb_max_of(const msa_shape_t *s) { return (s->max_kv_len + kBlock - 1) / kBlock; }

// Decode keeps one fp32 score per (sequence, index head, block) for the top-k
// pass; prefill selects inside the tensor-core kernel and needs only the
// header, plus a bf16 copy of E4M3 index keys for the MMA.
size_t index_ws_bytes(const msa_shape_t *s) {
    if (s->q_len > 1)
        return kWsHeaderBytes + (key_fp8(s) ? round_up(static_cast<size_t>(s->kv_capacity) *
                                                       key_heads(s) * kDim * 2)
                                            : 0);
    return kWsHeaderBytes +
           round_up(static_cast<size_t>(rows_of(s)) * index_heads(s) * nb_max_of(s) * sizeof(float));
}

// Prefill rows with groups of 8 heads run the block-outer tensor-core path;
// decode rows (and other group sizes) run one CTA per (row, group, split).
bool use_prefill_path(const msa_shape_t *s) {
    return s->q_len > 1 && prefill_attention_supported(s->num_q_heads, s->num_kv_heads);
}

struct AttnLayout {
    int nsplit;
    size_t tickets_off, tickets_bytes, partials_off, total;
    PrefillLayout pre;
};

AttnLayout attn_layout(const msa_shape_t *s) {
    AttnLayout L;
    if (use_prefill_path(s)) {
        L.nsplit = 1;
        L.tickets_off = L.partials_off = kWsHeaderBytes;
        L.tickets_bytes = 0;
        L.total = prefill_workspace_layout(s->batch, s->q_len, s->num_q_heads, s->num_kv_heads,
                                           s->top_k, s->max_kv_len, &L.pre);
        return L;
    }
    const long long pairs = rows_of(s) * s->num_kv_heads;
    L.nsplit = attn_rows_nsplit(pairs, s->top_k);
    const int G = s->num_q_heads / s->num_kv_heads;
    L.tickets_off = kWsHeaderBytes;
    L.tickets_bytes = L.nsplit > 1 ? round_up(static_cast<size_t>(pairs) * sizeof(int)) : 0;
    L.partials_off = L.tickets_off + L.tickets_bytes;
    const size_t part =
        L.nsplit > 1 ? static_cast<size_t>(pairs) * L.nsplit * attn_partial_floats(G) * 4 : 0;
    L.total = L.partials_off + round_up(part);
    return L;
}

msa_status_t check_ws(void *ws, size_t have, size_t need) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) || have < need)
        return MSA_ERR_WORKSPACE;
    return MSA_OK;
}

}  // namespace

extern "C" {

size_t msa_index_topk_workspace_size(const msa_shape_t *shape) {
    if (check_shape(shape) != MSA_OK) return 0;
    return index_ws_bytes(shape);
}

size_t msa_sparse_attention_workspace_size(const msa_shape_t *shape) {
    if (check_shape(shape) != MSA_OK) return 0;
    return attn_layout(shape).total;
}

}  // extern "C"

namespace {

// Paged caches: the pool holds whole 128-row pages and every sequence's
// blocks fit its page-table row.
msa_status_t check_paged(const msa_shape_t *s, const int32_t *page_table, int32_t pages_per_seq) {
    if (!page_table || pages_per_seq < 1) return MSA_ERR_INVALID_ARG;
    if (s->kv_capacity % kBlock) return MSA_ERR_INVALID_ARG;
    if (static_cast<long long>(pages_per_seq) * kBlock < s->max_kv_len) return MSA_ERR_INVALID_ARG;
    return MSA_OK;
}

msa_status_t index_topk_impl(const msa_shape_t *shape, const void *q_idx, const void *k_idx,
                             const float *k_scale, const int32_t *lens, const KvMap &kv,
                             int32_t *block_ids, float *block_scores, void *workspace,
                             size_t workspace_bytes, msa_stream_t stream) {
    if (!q_idx || !k_idx || !lens || !block_ids || !block_scores) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx)) return MSA_ERR_MISALIGNED;
    const bool fp8 = key_fp8(shape);
    if (fp8 && !k_scale) return MSA_ERR_INVALID_ARG;
    if (fp8 && (reinterpret_cast<uintptr_t>(k_scale) & 3)) return MSA_ERR_MISALIGNED;
    const int hi = index_heads(shape), kh = key_heads(shape);
    msa_status_t st = check_ws(workspace, workspace_bytes, index_ws_bytes(shape));
    if (st != MSA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws);
    float *scores = reinterpret_cast<float *>(ws + kWsHeaderBytes);
    const int nb_max = nb_max_of(shape);

    if (clear_header(ws, kWsHeaderBytes, s) != cudaSuccess) return MSA_ERR_CUDA;
    if (shape->q_len > 1) {
        IndexRowsArgs a;
        a.q_idx = q_idx; a.k_idx = k_idx; a.lens = lens; a.kv = kv; a.k_scale = nullptr;
        if (fp8) {
            // E4M3 keys widened exactly to bf16 in the workspace; the kernel
            // applies the row scales to the scores.
            void *wide = ws + kWsHeaderBytes;
            if (launch_widen_e4m3(k_idx, wide, static_cast<long long>(shape->kv_capacity) * kh, s) !=
                cudaSuccess)
                return MSA_ERR_CUDA;
            a.k_idx = wide;
            a.k_scale = k_scale;
        }
        a.ids = block_ids; a.out_scores = block_scores; a.status = status;
        a.B = shape->batch; a.Sq = shape->q_len; a.H_kv = hi; a.K = shape->top_k;
        a.max_kv_len = shape->max_kv_len; a.KH = kh;
        return launch_index_rows_tc(a, s) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
    }
    if (!fp8 && kh == hi) {
        // one bf16 key per index head
        IndexDecodeArgs a;
        a.q_idx = q_idx; a.k_idx = k_idx; a.lens = lens; a.kv = kv;
        a.scores = scores; a.status = status;
        a.B = shape->batch; a.H_kv = hi; a.nb_max = nb_max;
        a.max_kv_len = shape->max_kv_len;
        if (launch_index_decode(a, s) != cudaSuccess) return MSA_ERR_CUDA;
    } else {
        IndexDecodeVarArgs a;
        a.q_idx = q_idx; a.k_idx = k_idx; a.k_scale = k_scale; a.lens = lens; a.kv = kv;
        a.scores = scores; a.status = status;
        a.B = shape->batch; a.H = hi; a.KH = kh; a.nb_max = nb_max;
        a.max_kv_len = shape->max_kv_len; a.fp8 = fp8 ? 1 : 0;
        if (launch_index_decode_variant(a, s) != cudaSuccess) return MSA_ERR_CUDA;
    }
    TopkArgs t;
    t.scores = scores; t.lens = lens; t.kv = kv; t.ids = block_ids;
    t.out_scores = block_scores; t.status = status;
    t.B = shape->batch; t.Sq = shape->q_len; t.H_kv = hi; t.nb_max = nb_max;
    t.K = shape->top_k; t.max_kv_len = shape->max_kv_len;
    if (launch_topk(t, s) != cudaSuccess) return MSA_ERR_CUDA;
    return MSA_OK;
}

msa_status_t sparse_attention_impl(const msa_shape_t *shape, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *block_ids,
                                   const int32_t *lens, const KvMap &kv, float softmax_scale,
                                   void *out, void *workspace, size_t workspace_bytes,
                                   msa_stream_t stream, float *lse = nullptr) {
    if (!q || !k_cache || !v_cache || !block_ids || !lens || !out) return MSA_ERR_INVALID_ARG;
    if (!(softmax_scale == softmax_scale) || softmax_scale == INFINITY || softmax_scale == -INFINITY)
        return MSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return MSA_ERR_MISALIGNED;
    const AttnLayout L = attn_layout(shape);
    msa_status_t st = check_ws(workspace, workspace_bytes, L.total);
    if (st != MSA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (clear_header(ws, kWsHeaderBytes + L.tickets_bytes, s) != cudaSuccess)
        return MSA_ERR_CUDA;
    if (use_prefill_path(shape)) {
        PrefillArgs p;
        p.q = q; p.k_cache = k_cache; p.v_cache = v_cache; p.ids = block_ids; p.lens = lens;
        p.kv = kv; p.out = out; p.status = reinterpret_cast<int *>(ws);
        p.B = shape->batch; p.Sq = shape->q_len; p.H_q = shape->num_q_heads;
        p.H_kv = shape->num_kv_heads; p.K = shape->top_k; p.max_kv_len = shape->max_kv_len;
        p.n_idx = index_heads(shape);
        p.softmax_scale = softmax_scale;
        p.lse = lse;
        return launch_prefill_attention(p, ws, L.pre, s) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
    }
    AttnRowsArgs a;
    a.q = q; a.k_cache = k_cache; a.v_cache = v_cache; a.ids = block_ids; a.lens = lens;
    a.kv = kv; a.out = out; a.lse = lse;
    a.partials = reinterpret_cast<float *>(ws + L.partials_off);
    a.tickets = reinterpret_cast<int *>(ws + L.tickets_off);
    a.status = reinterpret_cast<int *>(ws);
    a.B = shape->batch; a.Sq = shape->q_len; a.H_q = shape->num_q_heads;
    a.H_kv = shape->num_kv_heads; a.K = shape->top_k; a.nsplit = L.nsplit;
    a.max_kv_len = shape->max_kv_len;
    a.n_idx = index_heads(shape);
    a.softmax_scale = softmax_scale;
    if (launch_attn_rows(a, s) != cudaSuccess) return MSA_ERR_CUDA;
    return MSA_OK;
}

KvMap packed_map(const msa_shape_t *s, const int64_t *kv_offsets) {
    KvMap m;
    m.offsets = kv_offsets; m.pages = nullptr; m.pages_per_seq = 0; m.capacity = s->kv_capacity;
    return m;
}

KvMap paged_map(const msa_shape_t *s, const int32_t *pages, int32_t pps) {
    KvMap m;
    m.offsets = nullptr; m.pages = pages; m.pages_per_seq = pps; m.capacity = s->kv_capacity;
    return m;
}

}  // namespace

extern "C" {

msa_status_t msa_index_topk(const msa_shape_t *shape, const void *q_idx, const void *k_idx,
                            const int32_t *lens, const int64_t *kv_offsets, int32_t *block_ids,
                            float *block_scores, void *workspace, size_t workspace_bytes,
                            msa_stream_t stream) {
    msa_status_t st = check_shape(shape);
    if (st != MSA_OK) return st;
    if (!kv_offsets) return MSA_ERR_INVALID_ARG;
    if (key_fp8(shape)) return MSA_ERR_UNSUPPORTED;   // msa_index_topk_fp8
    return index_topk_impl(shape, q_idx, k_idx, nullptr, lens, packed_map(shape, kv_offsets),
                           block_ids, block_scores, workspace, workspace_bytes, stream);
}

msa_status_t msa_index_topk_fp8(const msa_shape_t *shape, const void *q_idx,
                                const void *k_idx_fp8, const float *k_idx_scale,
                                const int32_t *lens, const int64_t *kv_offsets,
                                int32_t *block_ids, float *block_scores, void *workspace,
                                size_t workspace_bytes, msa_stream_t stream) {
    msa_status_t st = check_shape(shape);
    if (st != MSA_OK) return st;
    if (!kv_offsets || !key_fp8(shape)) return MSA_ERR_INVALID_ARG;
    return index_topk_impl(shape, q_idx, k_idx_fp8, k_idx_scale, lens,
                           packed_map(shape, kv_offsets), block_ids, block_scores, workspace,
                           workspace_bytes, stream);
}

msa_status_t msa_index_topk_paged(const msa_shape_t *shape, const void *q_idx,
                                  const void *k_idx_pool, const int32_t *lens,
                                  const int32_t *page_table, int32_t pages_per_seq,
                                  int32_t *block_ids, float *block_scores, void *workspace,
                                  size_t workspace_bytes, msa_stream_t stream) {
    msa_status_t st = check_shape(shape);
    if (st != MSA_OK) return st;
    if ((st = check_paged(shape, page_table, pages_per_seq)) != MSA_OK) return st;
    if (key_fp8(shape)) return MSA_ERR_UNSUPPORTED;
    return index_topk_impl(shape, q_idx, k_idx_pool, nullptr, lens,
                           paged_map(shape, page_table, pages_per_seq), block_ids, block_scores,
                           workspace, workspace_bytes, stream);
}

msa_status_t msa_sparse_attention(const msa_shape_t *shape, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *block_ids,
                                  const int32_t *lens, const int64_t *kv_offsets,
                                  float softmax_scale, void *out, void *workspace,
                                  size_t workspace_bytes, msa_stream_t stream) {
    msa_status_t st = check_shape(shape);
    if (st != MSA_OK) return st;
    if (!kv_offsets) return MSA_ERR_INVALID_ARG;
    return sparse_attention_impl(shape, q, k_cache, v_cache, block_ids, lens,
                                 packed_map(shape, kv_offsets), softmax_scale, out, workspace,
                                 workspace_bytes, stream);
}

msa_status_t msa_sparse_attention_paged(const msa_shape_t *shape, const void *q,
                                        const void *k_pool, const void *v_pool,
                                        const int32_t *block_ids, const int32_t *lens,
                                        const int32_t *page_table, int32_t pages_per_seq,
                                        float softmax_scale, void *out, void *workspace,
                                        size_t workspace_bytes, msa_stream_t stream) {
    msa_status_t st = check_shape(shape);
    if (st != MSA_OK) return st;
    if ((st = check_paged(shape, page_table, pages_per_seq)) != MSA_OK) return st;
    return sparse_attention_impl(shape, q, k_pool, v_pool, block_ids, lens,
                                 paged_map(shape, page_table, pages_per_seq), softmax_scale, out,
                                 workspace, workspace_bytes, stream);
}

msa_status_t msa_kv_append(const msa_shape_t *shape, int32_t n_new, const void *new_k_idx,
                           const void *new_k, const void *new_v, const int32_t *lens,
                           const int64_t *kv_offsets, const int32_t *page_table,
                           int32_t pages_per_seq, void *k_idx_cache, void *k_cache,
                           void *v_cache, int32_t *device_status, msa_stream_t stream) {
    msa_status_t st = check_shape(shape);
    if (st != MSA_OK) return st;
    if (n_new < 1 || !lens || !new_k_idx || !new_k || !new_v || !k_idx_cache || !k_cache ||
        !v_cache || (!kv_offsets) == (!page_table))
        return MSA_ERR_INVALID_ARG;
    if (key_fp8(shape)) return MSA_ERR_UNSUPPORTED;
    if (page_table && (st = check_paged(shape, page_table, pages_per_seq)) != MSA_OK) return st;
    if (!aligned16(new_k_idx) || !aligned16(new_k) || !aligned16(new_v) ||
        !aligned16(k_idx_cache) || !aligned16(k_cache) || !aligned16(v_cache))
        return MSA_ERR_MISALIGNED;
    KvAppendArgs a;
    a.src[0] = new_k_idx; a.src[1] = new_k; a.src[2] = new_v;
    a.dst[0] = k_idx_cache; a.dst[1] = k_cache; a.dst[2] = v_cache;
    a.lens = lens;
    a.kv = page_table ? paged_map(shape, page_table, pages_per_seq) : packed_map(shape, kv_offsets);
    a.status = device_status;
    a.B = shape->batch; a.n_new = n_new; a.H_kv = shape->num_kv_heads;
    a.H_idx = key_heads(shape);
    a.max_kv_len = shape->max_kv_len;
    return launch_kv_append(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MSA_OK
                                                                                     : MSA_ERR_CUDA;
}

// The backward's workspace: the forward's (recomputed first, from byte 0),
// then the output, statistics, dQ accumulator and buckets of the backward.
static size_t bwd_layout(const msa_shape_t *s, AttnBwdLayout *L) {
    const AttnLayout F = attn_layout(s);
    return attn_bwd_layout(s->batch, s->q_len, s->num_q_heads, s->num_kv_heads, s->top_k,
                           s->max_kv_len, F.total, use_prefill_path(s) ? &F.pre : nullptr, L);
}

size_t msa_sparse_attention_backward_workspace_size(const msa_shape_t *shape) {
    if (check_shape(shape) != MSA_OK) return 0;
    AttnBwdLayout L;
    return bwd_layout(shape, &L);
}

msa_status_t msa_sparse_attention_backward(const msa_shape_t *shape, const void *q,
                                           const void *k_cache, const void *v_cache,
                                           const int32_t *block_ids, const int32_t *lens,
                                           const int64_t *kv_offsets, float softmax_scale,
                                           const void *d_out, void *dq, float *dk, float *dv,
                                           void *workspace, size_t workspace_bytes,
                                           msa_stream_t stream) {
    msa_status_t st = check_shape(shape);
    if (st != MSA_OK) return st;
    if (!q || !k_cache || !v_cache || !block_ids || !lens || !kv_offsets || !d_out || !dq || !dk ||
        !dv)
        return MSA_ERR_INVALID_ARG;
    if (!(softmax_scale == softmax_scale) || softmax_scale == INFINITY || softmax_scale == -INFINITY)
        return MSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(d_out) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return MSA_ERR_MISALIGNED;
    AttnBwdLayout L;
    const size_t need = bwd_layout(shape, &L);
    if ((st = check_ws(workspace, workspace_bytes, need)) != MSA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // The forward, recomputed: its output and log-sum-exp go to the backward's
    // regions (it clears the header and owns bytes 4..31 of it).
    const KvMap kv = packed_map(shape, kv_offsets);
    if ((st = sparse_attention_impl(shape, q, k_cache, v_cache, block_ids, lens, kv, softmax_scale,
                                    ws + L.o, workspace, workspace_bytes, stream,
                                    reinterpret_cast<float *>(ws + L.lse))) != MSA_OK)
        return st;
    AttnBwdArgs a;
    a.q = q; a.k_cache = k_cache; a.v_cache = v_cache; a.dout = d_out; a.ids = block_ids;
    a.lens = lens; a.kv = packed_map(shape, kv_offsets); a.dq = dq; a.dk = dk; a.dv = dv;
    a.status = static_cast<int *>(workspace);
    a.B = shape->batch; a.Sq = shape->q_len; a.H_q = shape->num_q_heads;
    a.H_kv = shape->num_kv_heads; a.n_idx = index_heads(shape); a.K = shape->top_k;
    a.max_kv_len = shape->max_kv_len; a.softmax_scale = softmax_scale;
    return launch_attn_bwd(a, ws, L, s) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

// The fused decode step takes bf16 index keys, one row per index head (any
// index-head count the shape allows), q_len 1 and groups of at most 16 heads
// (one or two n8 tiles of the attention products).
static msa_status_t check_decode_step(const msa_shape_t *s) {
    msa_status_t st = check_shape(s);
    if (st != MSA_OK) return st;
    if (s->q_len != 1 || s->index_key_format != MSA_INDEX_KEYS_BF16 ||
        s->num_q_heads / s->num_kv_heads > 16)
        return MSA_ERR_UNSUPPORTED;
    return MSA_OK;
}

static DecodeFusedLayout decode_step_layout(const msa_shape_t *s) {
    DecodeFusedLayout L;
    decode_fused_layout(s->batch, s->num_q_heads, s->num_kv_heads, index_heads(s), s->top_k,
                        s->max_kv_len, &L);
    return L;
}

size_t msa_decode_step_workspace_size(const msa_shape_t *shape) {
    if (check_decode_step(shape) != MSA_OK) return 0;
    return decode_step_layout(shape).total;
}

static msa_status_t decode_step_impl(const msa_shape_t *shape, const void *q_idx,
                                     const void *k_idx, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *lens, const KvMap &kv,
                                     float softmax_scale, int32_t *block_ids, float *block_scores,
                                     void *out, void *workspace, size_t workspace_bytes,
                                     msa_stream_t stream) {
    if (!q_idx || !k_idx || !q || !k_cache || !v_cache || !lens || !block_ids || !block_scores ||
        !out)
        return MSA_ERR_INVALID_ARG;
    if (!(softmax_scale == softmax_scale) || softmax_scale == INFINITY || softmax_scale == -INFINITY)
        return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q) || !aligned16(k_cache) ||
        !aligned16(v_cache) || !aligned16(out))
        return MSA_ERR_MISALIGNED;
    const DecodeFusedLayout L = decode_step_layout(shape);
    msa_status_t st = check_ws(workspace, workspace_bytes, L.total);
    if (st != MSA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // status word, claim counters and per-call flags: one contiguous range
    if (clear_header(ws, L.zero_hi, s) != cudaSuccess) return MSA_ERR_CUDA;
    DecodeFusedArgs a;
    a.q_idx = q_idx; a.k_idx = k_idx; a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
    a.lens = lens; a.kv = kv;
    a.ids = block_ids; a.out_scores = block_scores; a.out = out;
    a.status = reinterpret_cast<int *>(ws);
    a.ctr = reinterpret_cast<int *>(ws + L.ctr);
    a.scores = reinterpret_cast<float *>(ws + L.scores);
    a.seq_done = reinterpret_cast<int *>(ws + L.seq_done);
    a.aq_item = reinterpret_cast<int *>(ws + L.aq_item);
    a.aq_flag = reinterpret_cast<int *>(ws + L.aq_flag);
    a.B = shape->batch; a.H_q = shape->num_q_heads; a.H_kv = shape->num_kv_heads;
    a.K = shape->top_k; a.nb_max = nb_max_of(shape); a.max_kv_len = shape->max_kv_len;
    a.n_idx = index_heads(shape);
    a.softmax_scale = softmax_scale;
    return launch_decode_fused(a, s) == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

msa_status_t msa_decode_step(const msa_shape_t *shape, const void *q_idx, const void *k_idx,
                             const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *lens, const int64_t *kv_offsets, float softmax_scale,
                             int32_t *block_ids, float *block_scores, void *out, void *workspace,
                             size_t workspace_bytes, msa_stream_t stream) {
    msa_status_t st = check_decode_step(shape);
    if (st != MSA_OK) return st;
    if (!kv_offsets) return MSA_ERR_INVALID_ARG;
    return decode_step_impl(shape, q_idx, k_idx, q, k_cache, v_cache, lens,
                            packed_map(shape, kv_offsets), softmax_scale, block_ids, block_scores,
                            out, workspace, workspace_bytes, stream);
}

msa_status_t msa_decode_step_paged(const msa_shape_t *shape, const void *q_idx,
                                   const void *k_idx_pool, const void *q, const void *k_pool,
                                   const void *v_pool, const int32_t *lens,
                                   const int32_t *page_table, int32_t pages_per_seq,
                                   float softmax_scale, int32_t *block_ids, float *block_scores,
                                   void *out, void *workspace, size_t workspace_bytes,
                                   msa_stream_t stream) {
    msa_status_t st = check_decode_step(shape);
    if (st != MSA_OK) return st;
    if ((st = check_paged(shape, page_table, pages_per_seq)) != MSA_OK) return st;
    return decode_step_impl(shape, q_idx, k_idx_pool, q, k_pool, v_pool, lens,
                            paged_map(shape, page_table, pages_per_seq), softmax_scale, block_ids,
                            block_scores, out, workspace, workspace_bytes, stream);
}

msa_status_t msa_read_device_status(const void *workspace, msa_stream_t stream) {
    if (!workspace) return MSA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MSA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MSA_ERR_CUDA;
    if (word & kStatusTimeout) return MSA_ERR_DEVICE_TIMEOUT;
    if (word & kStatusBadLens) return MSA_ERR_BAD_LENS;
    return MSA_OK;
}

msa_status_t msa_set_wait_controls(uint64_t wait_limit_ns, uint32_t stall_mask) {
    {
        std::lock_guard<std::mutex> lock(g_ctl_mu);
        g_ctl.limit_ns = wait_limit_ns;
        g_ctl.stall = stall_mask;
        g_ctl.never = 0;
    }
    g_ctl_on.store(wait_limit_ns != 0 || stall_mask != 0, std::memory_order_release);
    return MSA_OK;
}

const char *msa_status_string(msa_status_t status) {
    switch (status) {
        case MSA_OK: return "MSA_OK";
        case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG: null pointer or invalid size";
        case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED: size not handled by this library";
        case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE: workspace missing, short or misaligned";
        case MSA_ERR_CUDA: return "MSA_ERR_CUDA: a CUDA call or launch failed";
        case MSA_ERR_DEVICE_TIMEOUT: return "MSA_ERR_DEVICE_TIMEOUT: a device wait gave up";
        case MSA_ERR_BAD_LENS: return "MSA_ERR_BAD_LENS: lens, offsets or block ids out of range";
        case MSA_ERR_MISALIGNED: return "MSA_ERR_MISALIGNED: tensor not 16-byte aligned";
    }
    return "MSA_ERR_UNKNOWN";
}

}  // extern "C"
