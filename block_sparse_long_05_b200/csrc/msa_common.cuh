// msa_common.cuh -- definitions shared by the kernels and the host side of
// libmsa: device status bits, problem descriptor, workspace layout.
#pragma once

#include <cstddef>
#include <cstdint>

namespace msa {

// Device status word bits (OR-ed by kernels, read by msa_device_status).
constexpr int kDevTimeout = 1;
constexpr int kDevBadIds = 2;

constexpr int kMaxK = 32;          // top-K capacity of the register lists
constexpr int kMaxBlocksPrefill = 8192;  // N limit (inversion histograms, decode select)
constexpr int kInvRows = 128;      // query rows per inversion chunk (4 warps x 32)
constexpr int kDecodeKeys = 64;    // keys per split of the decode attention kernel
constexpr int kIdxKeys = 256;      // keys per tile of the prefill index kernel (one MMA N)

// Problem sizes of one call (host-validated).
struct Shape {
    int Bt, n_q, T, Hq, Hkv, d, d_idx, block, K;
    int N;  // number of blocks = ceil(T / block)
    int G;  // Hq / Hkv
};

// Paged KV for decode: logical block j of sequence b is physical page
// table[b * stride + j] of a store of `count` pages of `block` rows each
// (k_idx pages [count][block][d_idx], K/V pages [count][block][Hkv][d]).
// table == nullptr: contiguous [Bt][T] rows.
struct PageMap {
    const int32_t *table = nullptr;
    int stride = 0;
    int count = 0;
};

// One unit of work of the prefill attention kernel: the hit list of one
// (sequence, block) pair, rows [start, start + count) of that list.
struct AttnItem {
    int pair;   // b * N + j
    int start;  // offset inside the pair's list
    int count;  // number of list entries (query rows) in this item
    int pad;
};

inline __host__ __device__ size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Work list of the own-block pass of the prefill attention: per (sequence,
// block) pair, the query rows whose own block it is, cut into items like the
// hit lists (same scans).
struct OwnWork {
    int *totals;     // [Bt*N] own rows per pair
    int *row_ptr;    // [Bt*N + 1] (scan of totals; scratch)
    int *item_ptr;   // [Bt*N + 1]
    AttnItem *items; // [max own items]
    int *counters;   // per attention launch: (items, cursor)
};

// Workspace layout.  Offsets are in bytes from the workspace base; every
// region is 256-byte aligned.  Status word at offset 0.
struct WsLayout {
    size_t status = 0;
    // decode index
    size_t block_scores = 0;  // fp32 [Bt][N]
    // inversion
    size_t chunk_counts = 0;  // int32 [Bt][n_chunks][N]
    size_t pair_totals = 0;   // int32 [Bt*N]
    size_t row_ptr = 0;       // int32 [Bt*N + 1]
    size_t entries = 0;       // int32 [Bt*n_q*K]
    size_t item_ptr = 0;      // int32 [Bt*N + 1]
    size_t items = 0;         // AttnItem [max_items]
    size_t counters = 0;      // int32 [2 * launches]: (items per kv head, work cursor)
    // own-block pass (prefill): own rows per pair, scans, items, counters
    size_t own_totals = 0, own_row_ptr = 0, own_item_ptr = 0, own_items = 0, own_counters = 0;
    int max_own_items = 0;
    // attention partials
    size_t part_o = 0;        // prefill: bf16 [Bt*n_q][K][Hq][d]; decode: fp32 [Bt][K*S][Hq][d]
    size_t part_lse = 0;      // fp32 [Bt*n_q][K][Hq]; decode: [Bt][K*S][Hq]
    size_t total = 0;
    int n_chunks = 0;
    int max_items = 0;
    int rows_per_item = 0;
    int decode_splits = 0;    // S: splits per block in decode
    int kv_group = 0;         // prefill: kv heads per attention launch (partials hold their heads)
};

// Prefill partial buffer size that msa_workspace_size aims under: the kv
// heads are attended in groups whose partials fit (at least one kv head).
constexpr size_t kPartialBudget = static_cast<size_t>(4) << 30;

}  // namespace msa
