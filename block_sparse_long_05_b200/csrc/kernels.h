// kernels.h -- internal launchers of libmsa (host side).  Not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "msa_common.cuh"

namespace msa {

// SIMT kernels (kernels_simt.cu)
// pm: paged k_idx / K / V (pm.table == nullptr: contiguous); bad page ids
// are skipped and reported in *status
cudaError_t launch_decode_scan(const Shape &sh, const void *q_idx, const void *k_idx,
                               float *block_scores, const PageMap &pm, int *status, int num_sms,
                               cudaStream_t st, bool int8_keys = false);
// pdl: allow programmatic dependent launch after the previous kernel in st
// (the kernel waits for it before reading its results)
cudaError_t launch_decode_select(const Shape &sh, const float *block_scores, int32_t *ids,
                                 cudaStream_t st, bool pdl);
size_t decode_attn_smem_bytes(const Shape &sh);
cudaError_t launch_decode_attn(const Shape &sh, const void *q, const void *k, const void *v,
                               const int32_t *ids, float *part_o, float *part_lse, int S,
                               const PageMap &pm, int *status, cudaStream_t st, bool pdl);
// Merges the partials of query heads [h_off, h_off + Hp) (Hp heads per
// partial row) into those heads of out / lse.  Decode: Hp = Hq, h_off = 0.
cudaError_t launch_combine(const Shape &sh, const void *part_o, bool part_bf16,
                           const float *part_lse, const int32_t *ids, float *out, float *lse,
                           int S, cudaStream_t st, bool pdl, int Hp = 0, int h_off = 0);
// counters: n_cursors pairs (items per kv head, a zeroed work cursor), one
// per attention launch.  own != nullptr: the hit lists leave out each row's
// own block, and own receives the work list of the own-block pass.
cudaError_t launch_invert(const Shape &sh, const int32_t *ids, int *chunk_counts,
                          int *pair_totals, int32_t *row_ptr, int32_t *entries, int *item_ptr,
                          AttnItem *items, int *counters, int rows_per_item, int n_chunks,
                          int *status, cudaStream_t st, int n_cursors = 1,
                          const OwnWork *own = nullptr);

// tcgen05 kernels (kernels_tc.cu)
size_t selftest_smem_bytes(int N, int Kd);
cudaError_t launch_selftest_umma(const CUtensorMap &tm_a, const CUtensorMap &tm_b, float *C,
                                 int N, int Kd, int b_mn_major, int a_tmem, int *status,
                                 cudaStream_t st);
size_t prefill_index_smem_bytes(int d_idx, int elem_bytes);
// int8_keys: q_idx / k_idx are signed 8-bit integers (tcgen05 kind::i8)
// instead of bf16 (kind::f16)
cudaError_t launch_prefill_index(const Shape &sh, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                 int32_t *ids, int *status, int num_sms, cudaStream_t st,
                                 bool int8_keys);
size_t prefill_attn_smem_bytes(const Shape &sh);
int prefill_attn_rows_per_item(int G);
// One launch attends kv heads [hk0, hk0 + nhk) (and their query heads); its
// partials [rows][K][nhk * G][d] go to part_o / part_lse.  tm_k / tm_v must
// start at kv head hk0; counters: this launch's pair (items per kv head, a
// zeroed work cursor).
// own_ids != nullptr: the own-block pass instead (items: the own rows of each
// pair): attends each row's own block and writes the partial of the slot
// that holds it (own_ids: the selection, searched for that slot).
cudaError_t launch_prefill_attn(const Shape &sh, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                                const void *q, const int32_t *row_ptr, const int32_t *entries,
                                const AttnItem *items, int *counters, int hk0, int nhk,
                                void *part_o, float *part_lse, int *status, int num_sms,
                                cudaStream_t st, const int32_t *own_ids = nullptr);

}  // namespace msa
