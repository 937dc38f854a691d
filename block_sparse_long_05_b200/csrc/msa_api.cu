// msa_api.cu -- the C ABI of libmsa (declared in include/msa.h): argument
// validation, workspace layout, TMA tensor maps and kernel dispatch.  No
// computation happens here; every step of the path runs in the kernels.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "../../include/msa.h"
#include "kernels.h"
#include "msa_common.cuh"

using namespace msa;

namespace {

// Host-side validation shared by the entry points.  `need_attn` adds the
// attention sizes (Hq, Hkv, d); `need_index` adds d_idx.
msa_status validate(int Bt, int n_q, int T, int Hq, int Hkv, int d, int d_idx, int block, int K,
                    bool need_index, bool need_attn, Shape *out) {
    if (Bt < 1 || n_q < 1 || T < 1 || n_q > T || block < 1 || K < 1) return MSA_ERR_INVALID_ARG;
    if (need_attn && (Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv != 0)) return MSA_ERR_INVALID_ARG;
    if (need_index && d_idx < 1) return MSA_ERR_INVALID_ARG;
    if (K > kMaxK) return MSA_ERR_UNSUPPORTED;
    if (!(block == 32 || block == 64 || block % 128 == 0)) return MSA_ERR_UNSUPPORTED;
    if (need_index && !(d_idx == 64 || d_idx == 128)) return MSA_ERR_UNSUPPORTED;
    if (need_attn && !(d == 64 || d == 128)) return MSA_ERR_UNSUPPORTED;
    const long long N = (static_cast<long long>(T) + block - 1) / block;
    if (static_cast<long long>(Bt) * T >= (1ll << 31)) return MSA_ERR_UNSUPPORTED;
    if (static_cast<long long>(Bt) * n_q * K >= (1ll << 31)) return MSA_ERR_UNSUPPORTED;
    if (N > kMaxBlocksPrefill) return MSA_ERR_UNSUPPORTED;
    if (need_attn && static_cast<long long>(Bt) * n_q * Hq * d >= (1ll << 34)) return MSA_ERR_UNSUPPORTED;
    int G = 1;
    if (need_attn) {
        G = Hq / Hkv;
        if (128 % G != 0) return MSA_ERR_UNSUPPORTED;
    }
    out->Bt = Bt;
    out->n_q = n_q;
    out->T = T;
    out->Hq = Hq;
    out->Hkv = Hkv;
    out->d = d;
    out->d_idx = d_idx;
    out->block = block;
    out->K = K;
    out->N = static_cast<int>(N);
    out->G = G;
    return MSA_OK;
}

// Prefill partial bytes when kv_group kv heads are attended per launch.
size_t prefill_partial_bytes(const Shape &sh, int kv_group) {
    const size_t prow = static_cast<size_t>(sh.Bt) * sh.n_q * sh.K * kv_group * sh.G;
    return align_up(prow * sh.d * 2, 256) + align_up(prow * 4, 256);
}

// Largest divisor of Hkv whose partials fit in `budget` bytes (at least 1).
int kv_group_within(const Shape &sh, size_t budget) {
    int best = 1;
    for (int g = 1; g <= sh.Hkv; ++g)
        if (sh.Hkv % g == 0 && prefill_partial_bytes(sh, g) <= budget) best = g;
    return best;
}

// kv_group: prefill kv heads per attention launch (0: all of them).
WsLayout layout_for(const Shape &sh, bool with_attn, int kv_group = 0) {
    WsLayout L;
    size_t off = 256;  // status word + padding
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const long long pairs = static_cast<long long>(sh.Bt) * sh.N;
    L.n_chunks = (sh.n_q + kInvRows - 1) / kInvRows;
    L.rows_per_item = with_attn ? prefill_attn_rows_per_item(sh.G) : 128;
    L.max_items = static_cast<int>((static_cast<long long>(sh.Bt) * sh.n_q * sh.K + L.rows_per_item - 1) /
                                       L.rows_per_item +
                                   pairs);
    L.decode_splits = (sh.block + kDecodeKeys - 1) / kDecodeKeys;
    L.block_scores = take(static_cast<size_t>(pairs) * 4);
    L.chunk_counts = take(static_cast<size_t>(sh.Bt) * L.n_chunks * sh.N * 4);
    L.pair_totals = take(static_cast<size_t>(pairs) * 4);
    L.row_ptr = take(static_cast<size_t>(pairs + 1) * 4);
    L.entries = take(static_cast<size_t>(sh.Bt) * sh.n_q * sh.K * 4);
    L.item_ptr = take(static_cast<size_t>(pairs + 1) * 4);
    L.items = take(static_cast<size_t>(L.max_items) * sizeof(AttnItem));
    L.counters = take(static_cast<size_t>(2 * sh.Hkv) * 4);  // (items, cursor) per launch
    if (with_attn && sh.n_q > 1 && sh.block > 128) {  // the own-block pass's work list
        L.max_own_items = static_cast<int>((static_cast<long long>(sh.Bt) * sh.n_q + L.rows_per_item - 1) /
                                               L.rows_per_item + pairs);
        L.own_totals = take(static_cast<size_t>(pairs) * 4);
        L.own_row_ptr = take(static_cast<size_t>(pairs + 1) * 4);
        L.own_item_ptr = take(static_cast<size_t>(pairs + 1) * 4);
        L.own_items = take(static_cast<size_t>(L.max_own_items) * sizeof(AttnItem));
        L.own_counters = take(static_cast<size_t>(2 * sh.Hkv) * 4);
    }
    if (with_attn) {
        if (sh.n_q == 1) {
            const size_t prow = static_cast<size_t>(sh.Bt) * sh.K * L.decode_splits;
            L.part_o = take(prow * sh.Hq * sh.d * 4);
            L.part_lse = take(prow * sh.Hq * 4);
        } else {
            L.kv_group = kv_group > 0 ? kv_group : sh.Hkv;
            const size_t prow = static_cast<size_t>(sh.Bt) * sh.n_q * sh.K * L.kv_group * sh.G;
            L.part_o = take(prow * sh.d * 2);
            L.part_lse = take(prow * 4);
        }
    }
    L.total = off;
    return L;
}

msa_status check_ws(void *ws, size_t bytes, const WsLayout &L) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MSA_ERR_WORKSPACE;
    if (bytes < L.total) return MSA_ERR_WORKSPACE;
    return MSA_OK;
}

template <typename T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

msa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

int num_sms_current() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn load_encode() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeTiledFn>(fn);
}

EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = load_encode();  // thread-safe one-time init
    return fn;
}

// Tensor map (bf16 by default, or bytes) with 128-byte swizzle (or 64-byte
// for 64-byte box rows); dims/strides innermost first (strides in bytes for
// dims 1..rank-1).
bool make_tmap(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
               const cuuint64_t *strides, const cuuint32_t *box,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

// Record the start/stop event of stage i (if the caller supplied one).
void mark(const msa_stage_events *ev, int i, bool start, cudaStream_t st) {
    if (!ev) return;
    void *e = start ? ev->start[i] : ev->stop[i];
    if (e) cudaEventRecord(static_cast<cudaEvent_t>(e), st);
}

}  // namespace

extern "C" {

size_t msa_workspace_size(int Bt, int n_q, int T, int Hq, int Hkv, int d, int d_idx, int block,
                          int K) {
    Shape sh;
    if (validate(Bt, n_q, T, Hq, Hkv, d, d_idx, block, K, true, true, &sh) != MSA_OK) return 0;
    return layout_for(sh, true, kv_group_within(sh, kPartialBudget)).total;
}

size_t msa_workspace_size_kv_group(int Bt, int n_q, int T, int Hq, int Hkv, int d, int d_idx,
                                   int block, int K, int kv_group) {
    Shape sh;
    if (validate(Bt, n_q, T, Hq, Hkv, d, d_idx, block, K, true, true, &sh) != MSA_OK) return 0;
    if (kv_group < 1 || Hkv % kv_group != 0) return 0;
    return layout_for(sh, true, kv_group).total;
}

msa_status msa_index_topk(const void *q_idx, const void *k_idx, int32_t *ids, int Bt, int n_q,
                          int T, int d_idx, int block, int K, void *workspace,
                          size_t workspace_bytes, void *stream) {
    return msa_index_topk_ev(q_idx, k_idx, ids, Bt, n_q, T, d_idx, block, K, workspace,
                             workspace_bytes, stream, nullptr);
}

}  // extern "C"

namespace {

// Index branch for bf16 (elem_bytes 2) or signed 8-bit (elem_bytes 1) keys.
msa_status index_topk_impl(const void *q_idx, const void *k_idx, int32_t *ids, int Bt, int n_q,
                           int T, int d_idx, int block, int K, void *workspace,
                           size_t workspace_bytes, void *stream, const msa_stage_events *ev,
                           int elem_bytes) {
    if (!q_idx || !k_idx || !ids) return MSA_ERR_INVALID_ARG;
    Shape sh;
    msa_status s = validate(Bt, n_q, T, 1, 1, 64, d_idx, block, K, true, false, &sh);
    if (s != MSA_OK) return s;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned4(ids)) return MSA_ERR_INVALID_ARG;
    const WsLayout L = layout_for(sh, false);
    if ((s = check_ws(workspace, workspace_bytes, L)) != MSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int sms = num_sms_current();
    if (sms <= 0) return MSA_ERR_CUDA;
    int *status = at<int>(workspace, L.status);
    const bool s8 = elem_bytes == 1;
    if (n_q == 1) {
        float *scores = at<float>(workspace, L.block_scores);
        mark(ev, 0, true, st);
        if (launch_decode_scan(sh, q_idx, k_idx, scores, PageMap{}, status, sms, st, s8) !=
            cudaSuccess)
            return MSA_ERR_CUDA;
        mark(ev, 0, false, st);
        mark(ev, 1, true, st);
        if (launch_decode_select(sh, scores, ids, st, true) != cudaSuccess) return MSA_ERR_CUDA;
        mark(ev, 1, false, st);
        return MSA_OK;
    }
    // key rows of d_idx * elem_bytes bytes, loaded in boxes of at most 128
    // bytes (64-byte rows use the 64-byte swizzle)
    const cuuint32_t row_bytes = static_cast<cuuint32_t>(d_idx * elem_bytes);
    const cuuint32_t box_x = (row_bytes < 128 ? row_bytes : 128) / elem_bytes;
    const CUtensorMapDataType dt = s8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle swz = row_bytes < 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    CUtensorMap tq, tk;
    const cuuint64_t dq[2] = {static_cast<cuuint64_t>(d_idx), static_cast<cuuint64_t>(Bt) * n_q};
    const cuuint64_t dk[2] = {static_cast<cuuint64_t>(d_idx), static_cast<cuuint64_t>(Bt) * T};
    const cuuint64_t str[1] = {static_cast<cuuint64_t>(row_bytes)};
    const cuuint32_t qbox[2] = {box_x, 128};                                 // 128-query tile
    const cuuint32_t kbox[2] = {box_x, static_cast<cuuint32_t>(kIdxKeys)};  // key tile
    if (!make_tmap(&tq, q_idx, 2, dq, str, qbox, dt, swz) ||
        !make_tmap(&tk, k_idx, 2, dk, str, kbox, dt, swz))
        return MSA_ERR_CUDA;
    mark(ev, 0, true, st);
    const cudaError_t e = launch_prefill_index(sh, tq, tk, ids, status, sms, st, s8);
    mark(ev, 0, false, st);
    return cuda_status(e);
}

}  // namespace

extern "C" {

msa_status msa_index_topk_ev(const void *q_idx, const void *k_idx, int32_t *ids, int Bt, int n_q,
                             int T, int d_idx, int block, int K, void *workspace,
                             size_t workspace_bytes, void *stream, const msa_stage_events *ev) {
    return index_topk_impl(q_idx, k_idx, ids, Bt, n_q, T, d_idx, block, K, workspace,
                           workspace_bytes, stream, ev, 2);
}

msa_status msa_index_topk_i8(const int8_t *q_idx, const int8_t *k_idx, int32_t *ids, int Bt,
                             int n_q, int T, int d_idx, int block, int K, void *workspace,
                             size_t workspace_bytes, void *stream) {
    return msa_index_topk_i8_ev(q_idx, k_idx, ids, Bt, n_q, T, d_idx, block, K, workspace,
                                workspace_bytes, stream, nullptr);
}

msa_status msa_index_topk_i8_ev(const int8_t *q_idx, const int8_t *k_idx, int32_t *ids, int Bt,
                                int n_q, int T, int d_idx, int block, int K, void *workspace,
                                size_t workspace_bytes, void *stream,
                                const msa_stage_events *ev) {
    return index_topk_impl(q_idx, k_idx, ids, Bt, n_q, T, d_idx, block, K, workspace,
                           workspace_bytes, stream, ev, 1);
}

msa_status msa_select_invert(const int32_t *ids, int32_t *row_ptr, int32_t *entries, int Bt,
                             int n_q, int T, int block, int K, void *workspace,
                             size_t workspace_bytes, void *stream) {
    if (!ids || !row_ptr || !entries) return MSA_ERR_INVALID_ARG;
    Shape sh;
    msa_status s = validate(Bt, n_q, T, 1, 1, 64, 64, block, K, false, false, &sh);
    if (s != MSA_OK) return s;
    if (sh.N > kMaxBlocksPrefill) return MSA_ERR_UNSUPPORTED;
    if (!aligned4(ids) || !aligned4(row_ptr) || !aligned4(entries)) return MSA_ERR_INVALID_ARG;
    const WsLayout L = layout_for(sh, false);
    if ((s = check_ws(workspace, workspace_bytes, L)) != MSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(launch_invert(sh, ids, at<int>(workspace, L.chunk_counts),
                                     at<int>(workspace, L.pair_totals), row_ptr, entries, nullptr,
                                     nullptr, nullptr, L.rows_per_item, L.n_chunks,
                                     at<int>(workspace, L.status), st));
}

msa_status msa_sparse_attn(const void *q, const void *k, const void *v, const int32_t *ids,
                           float *out, float *lse, int Bt, int n_q, int T, int Hq, int Hkv, int d,
                           int block, int K, void *workspace, size_t workspace_bytes,
                           void *stream) {
    return msa_sparse_attn_ev(q, k, v, ids, out, lse, Bt, n_q, T, Hq, Hkv, d, block, K, workspace,
                              workspace_bytes, stream, nullptr);
}

msa_status msa_sparse_attn_ev(const void *q, const void *k, const void *v, const int32_t *ids,
                              float *out, float *lse, int Bt, int n_q, int T, int Hq, int Hkv,
                              int d, int block, int K, void *workspace, size_t workspace_bytes,
                              void *stream, const msa_stage_events *ev) {
    if (!q || !k || !v || !ids || !out || !lse) return MSA_ERR_INVALID_ARG;
    Shape sh;
    msa_status s = validate(Bt, n_q, T, Hq, Hkv, d, 64, block, K, false, true, &sh);
    if (s != MSA_OK) return s;
    // the combine writes out with 16-byte stores; ids and lse are read and
    // written as 4-byte words
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(ids) ||
        !aligned4(lse))
        return MSA_ERR_INVALID_ARG;
    // prefill: the fewest attention launches (largest kv-head groups) whose
    // partials fit in the workspace given
    int group = sh.Hkv;
    if (n_q > 1) {
        while (group > 1 && (sh.Hkv % group != 0 || layout_for(sh, true, group).total > workspace_bytes))
            --group;
    }
    const WsLayout L = layout_for(sh, true, group);
    if ((s = check_ws(workspace, workspace_bytes, L)) != MSA_OK) return s;
    // prefill kernels address a group's partial rows with 32-bit indices
    // (such a buffer could not fit in device memory anyway: 2^31 x 260 bytes)
    if (n_q > 1 && static_cast<long long>(Bt) * n_q * K * L.kv_group * sh.G >= (1ll << 31))
        return MSA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *status = at<int>(workspace, L.status);
    if (n_q == 1) {
        const int S = L.decode_splits;
        float *po = at<float>(workspace, L.part_o);
        float *pl = at<float>(workspace, L.part_lse);
        mark(ev, 1, true, st);
        cudaError_t e = launch_decode_attn(sh, q, k, v, ids, po, pl, S, PageMap{}, status, st, true);
        if (e != cudaSuccess) return MSA_ERR_CUDA;
        mark(ev, 1, false, st);
        mark(ev, 2, true, st);
        e = launch_combine(sh, po, false, pl, ids, out, lse, S, st, true);
        mark(ev, 2, false, st);
        return cuda_status(e);
    }
    const int sms = num_sms_current();
    if (sms <= 0) return MSA_ERR_CUDA;
    int32_t *rp = at<int32_t>(workspace, L.row_ptr);
    int32_t *ent = at<int32_t>(workspace, L.entries);
    AttnItem *items = at<AttnItem>(workspace, L.items);
    int *counters = at<int>(workspace, L.counters);
    const int n_launch = sh.Hkv / L.kv_group;
    // Blocks of several 128-key sub-tiles: hit lists without each row's own
    // block, whose rows get their own pass (causal: a chunk of consecutive
    // rows skips the sub-tiles past its last row).  A single-sub-tile block
    // has nothing to skip, and its own rows stay in the hit lists.
    const bool own_pass = block > 128;
    OwnWork own;
    own.totals = at<int>(workspace, L.own_totals);
    own.row_ptr = at<int>(workspace, L.own_row_ptr);
    own.item_ptr = at<int>(workspace, L.own_item_ptr);
    own.items = at<AttnItem>(workspace, L.own_items);
    own.counters = at<int>(workspace, L.own_counters);
    mark(ev, 0, true, st);
    cudaError_t e = launch_invert(sh, ids, at<int>(workspace, L.chunk_counts),
                                  at<int>(workspace, L.pair_totals), rp, ent,
                                  at<int>(workspace, L.item_ptr), items, counters,
                                  L.rows_per_item, L.n_chunks, status, st, n_launch,
                                  own_pass ? &own : nullptr);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    mark(ev, 0, false, st);
    const int NK = block < 128 ? block : 128;
    const cuuint64_t str[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(Hkv) * d * 2};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(NK)};
    void *po = at<void>(workspace, L.part_o);
    float *pl = at<float>(workspace, L.part_lse);
    // kv-head groups in turn: the hit-list pass attends the selected blocks
    // (all but the row's own one when there is an own-block pass), the
    // own-block pass the own blocks; both write per-slot partials (the
    // partial buffer holds one group), which the combine merges into out /
    // lse.  With
    // several groups, the attention stage's events span the combines of all
    // groups but the last, and the combine stage is the last group's.
    mark(ev, 1, true, st);
    for (int gi = 0; gi < n_launch; ++gi) {
        const int hk0 = gi * L.kv_group;
        // K/V tensor maps over this group's kv heads (row stride unchanged)
        CUtensorMap tk, tv;
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L.kv_group),
                                    static_cast<cuuint64_t>(Bt) * T};
        const size_t head_off = static_cast<size_t>(hk0) * d;  // elements
        if (!make_tmap(&tk, static_cast<const __nv_bfloat16 *>(k) + head_off, 3, dims, str, box) ||
            !make_tmap(&tv, static_cast<const __nv_bfloat16 *>(v) + head_off, 3, dims, str, box))
            return MSA_ERR_CUDA;
        e = launch_prefill_attn(sh, tk, tv, q, rp, ent, items, counters + 2 * gi, hk0,
                                L.kv_group, po, pl, status, sms, st);
        if (e != cudaSuccess) return MSA_ERR_CUDA;
        if (own_pass) {
            e = launch_prefill_attn(sh, tk, tv, q, own.row_ptr, ent, own.items,
                                    own.counters + 2 * gi, hk0, L.kv_group, po, pl, status, sms,
                                    st, ids);
            if (e != cudaSuccess) return MSA_ERR_CUDA;
        }
        if (gi + 1 == n_launch) {
            mark(ev, 1, false, st);
            mark(ev, 2, true, st);
        }
        e = launch_combine(sh, po, true, pl, ids, out, lse, 1, st, true, L.kv_group * sh.G,
                           hk0 * sh.G);
        if (e != cudaSuccess) return MSA_ERR_CUDA;
    }
    mark(ev, 2, false, st);
    return MSA_OK;
}

msa_status msa_index_topk_paged(const void *q_idx, const void *k_idx_pages,
                                const int32_t *page_table, int page_stride, int num_pages,
                                int32_t *ids, int Bt, int T, int d_idx, int block, int K,
                                void *workspace, size_t workspace_bytes, void *stream) {
    if (!q_idx || !k_idx_pages || !page_table || !ids) return MSA_ERR_INVALID_ARG;
    Shape sh;
    msa_status s = validate(Bt, 1, T, 1, 1, 64, d_idx, block, K, true, false, &sh);
    if (s != MSA_OK) return s;
    if (page_stride < sh.N || num_pages < 1) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx_pages) || !aligned4(page_table) || !aligned4(ids))
        return MSA_ERR_INVALID_ARG;
    const WsLayout L = layout_for(sh, false);
    if ((s = check_ws(workspace, workspace_bytes, L)) != MSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int sms = num_sms_current();
    if (sms <= 0) return MSA_ERR_CUDA;
    int *status = at<int>(workspace, L.status);
    float *scores = at<float>(workspace, L.block_scores);
    const PageMap pm{page_table, page_stride, num_pages};
    if (launch_decode_scan(sh, q_idx, k_idx_pages, scores, pm, status, sms, st) != cudaSuccess)
        return MSA_ERR_CUDA;
    return cuda_status(launch_decode_select(sh, scores, ids, st, true));
}

msa_status msa_sparse_attn_paged(const void *q, const void *k_pages, const void *v_pages,
                                 const int32_t *page_table, int page_stride, int num_pages,
                                 const int32_t *ids, float *out, float *lse, int Bt, int T,
                                 int Hq, int Hkv, int d, int block, int K, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    if (!q || !k_pages || !v_pages || !page_table || !ids || !out || !lse)
        return MSA_ERR_INVALID_ARG;
    Shape sh;
    msa_status s = validate(Bt, 1, T, Hq, Hkv, d, 64, block, K, false, true, &sh);
    if (s != MSA_OK) return s;
    if (page_stride < sh.N || num_pages < 1) return MSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) ||
        !aligned4(page_table) || !aligned4(ids) || !aligned4(lse))
        return MSA_ERR_INVALID_ARG;
    const WsLayout L = layout_for(sh, true);
    if ((s = check_ws(workspace, workspace_bytes, L)) != MSA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *status = at<int>(workspace, L.status);
    const int S = L.decode_splits;
    float *po = at<float>(workspace, L.part_o);
    float *pl = at<float>(workspace, L.part_lse);
    const PageMap pm{page_table, page_stride, num_pages};
    cudaError_t e = launch_decode_attn(sh, q, k_pages, v_pages, ids, po, pl, S, pm, status, st, true);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    return cuda_status(launch_combine(sh, po, false, pl, ids, out, lse, S, st, true));
}

msa_status msa_device_status(void *workspace, void *stream) {
    if (!workspace) return MSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MSA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MSA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return MSA_ERR_CUDA;
    if (h & kDevTimeout) return MSA_ERR_TIMEOUT;
    if (h & kDevBadIds) return MSA_ERR_BAD_IDS;
    return MSA_OK;
}

const char *msa_status_string(int status) {
    switch (status) {
        case MSA_OK: return "MSA_OK";
        case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
        case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
        case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE";
        case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
        case MSA_ERR_TIMEOUT: return "MSA_ERR_TIMEOUT";
        case MSA_ERR_BAD_IDS: return "MSA_ERR_BAD_IDS";
        default: return "unknown status";
    }
}

msa_status msa_selftest_umma(const void *A, const void *B, float *C, int N, int Kd,
                             int b_mn_major, int *status, void *stream) {
    if (!A || !B || !C || !status) return MSA_ERR_INVALID_ARG;
    if (!(N == 64 || N == 128 || N == 256) || Kd < 64 || Kd > 256 || Kd % 64 != 0)
        return MSA_ERR_UNSUPPORTED;
    const int b_mn = b_mn_major & 1;
    CUtensorMap ta, tb;
    const cuuint64_t da[2] = {static_cast<cuuint64_t>(Kd), 128};
    const cuuint64_t sa[1] = {static_cast<cuuint64_t>(Kd) * 2};
    const cuuint32_t ba[2] = {64, 128};
    if (!make_tmap(&ta, A, 2, da, sa, ba)) return MSA_ERR_CUDA;
    if (b_mn) {
        const cuuint64_t db[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(Kd)};
        const cuuint64_t sb[1] = {static_cast<cuuint64_t>(N) * 2};
        const cuuint32_t bb[2] = {64, static_cast<cuuint32_t>(Kd)};
        if (!make_tmap(&tb, B, 2, db, sb, bb)) return MSA_ERR_CUDA;
    } else {
        const cuuint64_t db[2] = {static_cast<cuuint64_t>(Kd), static_cast<cuuint64_t>(N)};
        const cuuint64_t sb[1] = {static_cast<cuuint64_t>(Kd) * 2};
        const cuuint32_t bb[2] = {64, static_cast<cuuint32_t>(N)};
        if (!make_tmap(&tb, B, 2, db, sb, bb)) return MSA_ERR_CUDA;
    }
    return cuda_status(launch_selftest_umma(ta, tb, C, N, Kd, b_mn_major & 1, (b_mn_major >> 1) & 1,
                                            status, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
