// kernels_tc.cu -- tcgen05 (5th-generation tensor core) kernels of the MSA
// hot path on sm_100a:
//   * prefill_index_kernel: index branch for many queries.  S = q_idx k_idx^T
//     tiles (128 queries x 128 keys) accumulate in tensor memory; the
//     epilogue warps max-pool each key block and keep a register top-K per
//     query row, so the n_q x T score matrix never exists.
//   * prefill_attn_kernel: sparse branch, KV-block-outer.  Each work item is
//     one (sequence, block, kv head) hit list (or a slice of it): the block's
//     K and V are TMA-loaded into shared memory once, the hit queries' G heads
//     are gathered as 128-row tiles, S = QK^T and O = PV run on tcgen05 with
//     the online softmax in between, and a normalised partial (O, lse) per
//     (query, slot, head) goes to the workspace for the log-sum-exp combine.
//   * selftest_umma_kernel: one 128 x N GEMM through the same TMA /
//     descriptor / MMA / TMEM code, for validating the building blocks.
//
// Method: "MiniMax M3模型算力成本大幅降低原因深度解析" (index branch: single-head
// key, block max-pool, top-K; sparse branch: GQA on the kept blocks, raw KV)
// and "MiniMax M3 深度实战", section 2.2 (KV outer gather Q, each KV block read
// once) and section 2.3 (local block always kept; softmax(QK^T/sqrt(d))V).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "kernels.h"
#include "msa_common.cuh"
#include "ptx_sm100.cuh"

namespace msa {

namespace {

constexpr float kLn2f = 0.6931471805599453f;
constexpr uint32_t kRegionBytes = 16384;  // 128 rows x 128 B (64 bf16) swizzled region

__device__ __forceinline__ unsigned char *align1024(unsigned char *p) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
}

// Bounded wait that ignores the abort flag: used only to drain copies that
// are still in flight when a kernel unwinds after an abort.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs / 4) break;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// ===========================================================================
// Self-test GEMM: C[128][N] = A[128][Kd] . B, one CTA of 128 threads.
// ===========================================================================
__global__ void __launch_bounds__(128, 1) selftest_umma_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    float *__restrict__ C, int N, int Kd, int b_mn_major, int a_tmem_cols, int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = align1024(smem_raw);
    unsigned char *a_s = base;                                  // Kd/64 regions x 16 KB
    unsigned char *b_s = a_s + (Kd / 64) * kRegionBytes;        // Kd*N*2 bytes
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(b_s + static_cast<size_t>(Kd) * N * 2);
    uint64_t *bar_mma = bar_ld + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid / 32;
    // accumulator columns [0, N); with A in tensor memory, A at [N, N + Kd/2)
    const int need = N + (a_tmem_cols ? Kd / 2 : 0);
    const uint32_t ncols = need <= 64 ? 64u : (need <= 128 ? 128u : (need <= 256 ? 256u : 512u));
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == 0) {
        const uint32_t bytes = static_cast<uint32_t>(128 * Kd * 2 + Kd * N * 2);
        mbar_arrive_expect_tx(bar_ld, bytes);
        for (int r = 0; r < Kd / 64; ++r) tma_load_2d(a_s + r * kRegionBytes, &tm_a, bar_ld, r * 64, 0);
        if (b_mn_major) {
            // B [Kd][N]: N/64 regions, each Kd rows x 128 B
            for (int r = 0; r < N / 64; ++r)
                tma_load_2d(b_s + static_cast<size_t>(r) * Kd * 128, &tm_b, bar_ld, r * 64, 0);
        } else {
            // B [N][Kd]: Kd/64 regions, each N rows x 128 B
            for (int r = 0; r < Kd / 64; ++r)
                tma_load_2d(b_s + static_cast<size_t>(r) * N * 128, &tm_b, bar_ld, r * 64, 0);
        }
    }
    bool ok = mbar_wait(bar_ld, 0, abort_flag, status);
    if (ok && a_tmem_cols) {
        // A operand from tensor memory: each thread copies its row of A from
        // the swizzled shared tile into TMEM columns [N, N + Kd/2), packed
        // two bf16 per column, even k in the low half.
        const int row = tid;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        for (int c0 = 0; c0 < Kd; c0 += 32) {  // 32 elements = 16 columns per store
            uint32_t w[16];
            for (int q = 0; q < 4; ++q) {  // four 16-byte pieces of 8 elements
                const int k = c0 + q * 8;
                const uint4 u = *reinterpret_cast<const uint4 *>(
                    a_s + (k / 64) * kRegionBytes + sw128_offset(row, (k % 64) / 8));
                w[q * 4 + 0] = u.x;
                w[q * 4 + 1] = u.y;
                w[q * 4 + 2] = u.z;
                w[q * 4 + 3] = u.w;
            }
            tmem_st16(tmem + lane_base + N + c0 / 2, w);
        }
        tmem_wait_st();
        tc_fence_before();
    }
    __syncthreads();
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, N, b_mn_major != 0);
        for (int kk = 0; kk < Kd / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(smem_addr(a_s + (kk / 4) * kRegionBytes + (kk % 4) * 32), 16, 1024);
            uint64_t bd;
            if (b_mn_major)
                bd = sdesc_sw128(smem_addr(b_s + kk * 16 * 128), static_cast<uint32_t>(Kd) * 128, 1024);
            else
                bd = sdesc_sw128(smem_addr(b_s + static_cast<size_t>(kk / 4) * N * 128 + (kk % 4) * 32), 16, 1024);
            if (a_tmem_cols)
                umma_bf16_tmem_a(tmem, tmem + N + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
            else
                umma_bf16(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_mma);
    }
    ok = ok && mbar_wait(bar_mma, 0, abort_flag, status);
    __syncwarp();
    tc_fence_after();
    if (__all_sync(0xFFFFFFFFu, ok)) {
        const int row = warp * 32 + (tid % 32);
        for (int c = 0; c < N / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c * 32, v);
            tmem_wait_ld();
            for (int e = 0; e < 32; ++e) C[static_cast<size_t>(row) * N + c * 32 + e] = __uint_as_float(v[e]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

// ===========================================================================
// Prefill index kernel.
//   warp 0: TMA producer (q tile once per item, kIdxKeys-key k tiles through
//           a kIdxStages-stage ring), warp 1: MMA issuer (TMEM owner: two
//           accumulators of kIdxKeys columns), warps 2-5: epilogue
//           (row = 32*(warp%4) + lane; block max-pool + top-K).
// Work item = (sequence b, 128-query tile qt); items ordered by decreasing
// cost and dealt to CTAs in a snake order.
// ===========================================================================
struct IndexParams {
    int32_t *ids;
    int *status;
    int Bt, n_q, T, block, K, n_qt, n_items;
};

constexpr int kIdxStages = 3;

__device__ __forceinline__ int snake_item(int it, int cta, int ncta) {
    return (it & 1) ? it * ncta + (ncta - 1 - cta) : it * ncta + cta;
}

template <int CAP>
__device__ __forceinline__ void topk_insert(float (&ts)[CAP], int (&tj)[CAP], float s, int j) {
    if (!(s > ts[CAP - 1])) return;
    bool ins = false;
#pragma unroll
    for (int p = 0; p < CAP; ++p) {
        const bool take = ins || s > ts[p];
        if (take) {
            const float fs = ts[p];
            const int ij = tj[p];
            ts[p] = s;
            tj[p] = j;
            s = fs;
            j = ij;
            ins = true;
        }
    }
}

// Index keys as bf16 (kind::f16, fp32 accumulation, K = 16 per MMA) or as
// signed 8-bit integers (kind::i8, s32 accumulation, K = 32 per MMA: twice
// the tensor-core rate, and exact for any int8 keys).  A key row of
// D_IDX * EB bytes is stored as NREG swizzled regions of RP-byte rows:
// 128-byte swizzle for 128-byte rows, 64-byte swizzle for 64-byte rows.
template <int D_IDX, int EB>
struct IndexTile {
    static constexpr int RB = D_IDX * EB;                  // bytes per key row
    static constexpr int RP = RB < 128 ? RB : 128;         // bytes per region row
    static constexpr int NREG = RB / RP;                   // regions per row
    static constexpr uint32_t QREG = 128u * RP;            // one region of the Q tile
    static constexpr uint32_t TILE = NREG * QREG;          // Q tile: 128 rows
    static constexpr uint32_t KREG = kIdxKeys * RP;        // one region of a key tile
    static constexpr uint32_t KTILE = NREG * KREG;         // key tile: kIdxKeys rows
    static constexpr int KSTEPS = RB / 32;                 // MMAs per tile (32 bytes of K each)
    __device__ static uint64_t desc(uint32_t saddr) {
        return RP == 128 ? sdesc_sw128(saddr, 16, 1024) : sdesc_sw64(saddr);
    }
};

template <int D_IDX, int CAP, int EB>
__global__ void __launch_bounds__(192, 1) prefill_index_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    IndexParams p) {
    using TL = IndexTile<D_IDX, EB>;
    constexpr int NREG = TL::NREG;
    constexpr uint32_t TILE = TL::TILE;                    // Q tile: 128 rows
    constexpr uint32_t KREG = TL::KREG;                    // one region of a key tile
    constexpr uint32_t KTILE = TL::KTILE;                  // key tile: kIdxKeys rows
    constexpr int XB = TL::RP / EB;                        // TMA box width (elements)
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = align1024(smem_raw);
    unsigned char *q_s = base;
    unsigned char *k_s = base + TILE;  // kIdxStages key tiles
    uint64_t *bars = reinterpret_cast<uint64_t *>(k_s + kIdxStages * KTILE);
    uint64_t *kfull = bars;
    uint64_t *kempty = bars + kIdxStages;
    uint64_t *qfull = bars + 2 * kIdxStages;
    uint64_t *qempty = qfull + 1;
    uint64_t *tfull = qfull + 2;   // [2]
    uint64_t *tempty = qfull + 4;  // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(qfull + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    if (tid == 0) {
        for (int s = 0; s < kIdxStages; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(kempty + s, 1);
        }
        mbar_init(qfull, 1);
        mbar_init(qempty, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 128);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * kIdxKeys);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int B = p.block;
    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            uint32_t n = 0;
            bool ok = true;
            int armed[kIdxStages];
            for (int s = 0; s < kIdxStages; ++s) armed[s] = -1;
            for (int it = 0; ok; ++it) {
                const int idx = snake_item(it, blockIdx.x, gridDim.x);
                if (idx >= p.n_items) break;
                const int qt = p.n_qt - 1 - idx / p.Bt, b = idx % p.Bt;
                const int i_last = min(qt * 128 + 127, p.n_q - 1);
                const int own_max = (p.T - p.n_q + i_last) / B;
                const int n_sub = (own_max * B + kIdxKeys - 1) / kIdxKeys;
                if (!mbar_wait(qempty, (it & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
                mbar_arrive_expect_tx(qfull, TILE);
                for (int r = 0; r < NREG; ++r)
                    tma_load_2d(q_s + r * TL::QREG, &tm_q, qfull, r * XB, b * p.n_q + qt * 128);
                for (int s = 0; s < n_sub; ++s, ++n) {
                    const uint32_t st = n % kIdxStages, rd = n / kIdxStages;
                    if (!mbar_wait(kempty + st, (rd & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
                    mbar_arrive_expect_tx(kfull + st, KTILE);
                    armed[st] = static_cast<int>(rd & 1);
                    for (int r = 0; r < NREG; ++r)
                        tma_load_2d(k_s + st * KTILE + r * KREG, &tm_k, kfull + st, r * XB,
                                    b * p.T + s * kIdxKeys);
                }
            }
            if (*abort_flag) {  // drain this CTA's copies still in flight
                for (int s = 0; s < kIdxStages; ++s)
                    if (armed[s] >= 0) mbar_drain(kfull + s, static_cast<uint32_t>(armed[s]));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = EB == 1 ? idesc_s8_s32(128, kIdxKeys)
                                           : idesc_bf16_f32(128, kIdxKeys, false);
            uint32_t n = 0, acc_n = 0;
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int idx = snake_item(it, blockIdx.x, gridDim.x);
                if (idx >= p.n_items) break;
                const int qt = p.n_qt - 1 - idx / p.Bt;
                const int i_last = min(qt * 128 + 127, p.n_q - 1);
                const int own_max = (p.T - p.n_q + i_last) / B;
                const int n_sub = (own_max * B + kIdxKeys - 1) / kIdxKeys;
                if (!mbar_wait(qfull, it & 1, abort_flag, p.status)) break;
                for (int s = 0; s < n_sub; ++s, ++n, ++acc_n) {
                    const uint32_t st = n % kIdxStages, rd = n / kIdxStages;
                    const uint32_t acc = acc_n & 1, ar = acc_n >> 1;
                    if (!mbar_wait(kfull + st, rd & 1, abort_flag, p.status)) { ok = false; break; }
                    if (!mbar_wait(tempty + acc, (ar & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t qa = smem_addr(q_s), ka = smem_addr(k_s + st * KTILE);
                    constexpr int SPR = TL::RP / 32;  // K steps per region row
#pragma unroll
                    for (int kk = 0; kk < TL::KSTEPS; ++kk) {
                        const uint32_t koff = (kk % SPR) * 32;
                        const uint64_t ad = TL::desc(qa + (kk / SPR) * TL::QREG + koff);
                        const uint64_t bd = TL::desc(ka + (kk / SPR) * KREG + koff);
                        if (EB == 1)
                            umma_i8(tmem + acc * kIdxKeys, ad, bd, idesc, kk > 0 ? 1u : 0u);
                        else
                            umma_bf16(tmem + acc * kIdxKeys, ad, bd, idesc, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(kempty + st);
                    umma_commit(tfull + acc);
                }
                umma_commit(qempty);
            }
        }
    } else {
        // epilogue warps 2..5
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t acc_n = 0;
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int idx = snake_item(it, blockIdx.x, gridDim.x);
            if (idx >= p.n_items) break;
            const int qt = p.n_qt - 1 - idx / p.Bt, b = idx % p.Bt;
            const int i_last = min(qt * 128 + 127, p.n_q - 1);
            const int own_max = (p.T - p.n_q + i_last) / B;
            const int n_sub = (own_max * B + kIdxKeys - 1) / kIdxKeys;
            const int i = qt * 128 + row;
            const bool valid = i < p.n_q;
            const int own = valid ? (p.T - p.n_q + i) / B : 0;
            float ts[CAP];
            int tj[CAP];
#pragma unroll
            for (int q = 0; q < CAP; ++q) {
                ts[q] = -FLT_MAX;
                tj[q] = 0x7FFFFFFF;
            }
            float bm = -FLT_MAX;
            for (int s = 0; s < n_sub; ++s, ++acc_n) {
                const uint32_t acc = acc_n & 1, ar = acc_n >> 1;
                if (!mbar_wait(tfull + acc, ar & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                // two halves of 128 columns: four loads in flight, one wait each
                // (a wait covers every load of the thread), so the load latency
                // is paid twice per tile rather than once per 32 columns
#pragma unroll 1
                for (int h = 0; h < kIdxKeys / 128; ++h) {
                    uint32_t v[128];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        tmem_ld32(tmem + lane_addr + acc * kIdxKeys + h * 128 + c4 * 32,
                                  *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c4));
                    tmem_wait_ld();
                    if (h == kIdxKeys / 128 - 1) {  // the accumulator has been read: refill it
                        tc_fence_before();
                        mbar_arrive(tempty + acc);
                    }
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        // block >= 32 and 32 | block: a 32-column chunk lies in one block
                        float m;
                        if (EB == 1) {  // s32 accumulators: integer maximum, then exact to fp32
                            // three independent chains of three-input maxima, as below
                            auto iv = [&](int e) { return static_cast<int>(v[32 * c4 + e]); };
                            int g3[3] = {iv(0), iv(1), iv(2)};
#pragma unroll
                            for (int e = 3; e + 5 < 32; e += 6) {
                                g3[0] = __vimax3_s32(g3[0], iv(e), iv(e + 3));
                                g3[1] = __vimax3_s32(g3[1], iv(e + 1), iv(e + 4));
                                g3[2] = __vimax3_s32(g3[2], iv(e + 2), iv(e + 5));
                            }
                            // columns 27..31 remain
                            int im = __vimax3_s32(__vimax3_s32(g3[0], g3[1], g3[2]), iv(27), iv(28));
                            im = __vimax3_s32(im, iv(29), max(iv(30), iv(31)));
                            m = static_cast<float>(im);
                        } else {
                            float g3[3] = {__uint_as_float(v[32 * c4]), __uint_as_float(v[32 * c4 + 1]),
                                           __uint_as_float(v[32 * c4 + 2])};
#pragma unroll
                            for (int e = 3; e + 5 < 32; e += 6) {
                                g3[0] = fmax3(g3[0], __uint_as_float(v[32 * c4 + e]), __uint_as_float(v[32 * c4 + e + 3]));
                                g3[1] = fmax3(g3[1], __uint_as_float(v[32 * c4 + e + 1]), __uint_as_float(v[32 * c4 + e + 4]));
                                g3[2] = fmax3(g3[2], __uint_as_float(v[32 * c4 + e + 2]), __uint_as_float(v[32 * c4 + e + 5]));
                            }
                            // columns 27..31 remain
                            m = fmax3(fmax3(g3[0], g3[1], g3[2]), __uint_as_float(v[32 * c4 + 27]),
                                      __uint_as_float(v[32 * c4 + 28]));
                            m = fmax3(m, __uint_as_float(v[32 * c4 + 29]),
                                      fmaxf(__uint_as_float(v[32 * c4 + 30]), __uint_as_float(v[32 * c4 + 31])));
                        }
                        bm = fmaxf(bm, m);
                        const int col_end = s * kIdxKeys + h * 128 + c4 * 32 + 32;
                        if (col_end % B == 0) {
                            const int j = col_end / B - 1;
                            if (j < own) topk_insert<CAP>(ts, tj, bm, j);
                            bm = -FLT_MAX;
                        }
                    }
                }
            }
            if (!ok) break;
            if (valid) {
                const int m = min(p.K, own + 1) - 1;
                int a[CAP + 1];
#pragma unroll
                for (int q = 0; q < CAP; ++q) a[q] = q < m ? tj[q] : 0x7FFFFFFF;
                a[CAP] = own;
                // odd-even transposition sort, ascending
#pragma unroll
                for (int r = 0; r < CAP + 1; ++r) {
#pragma unroll
                    for (int q = (r & 1); q + 1 < CAP + 1; q += 2) {
                        const int lo = min(a[q], a[q + 1]), hi = max(a[q], a[q + 1]);
                        a[q] = lo;
                        a[q + 1] = hi;
                    }
                }
                int32_t *dst = p.ids + (static_cast<long long>(b) * p.n_q + i) * p.K;
#pragma unroll
                for (int q = 0; q < CAP + 1; ++q)
                    if (q < p.K) dst[q] = a[q] == 0x7FFFFFFF ? -1 : a[q];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 2 * kIdxKeys);
}

// ===========================================================================
// Prefill attention (KV-block-outer).
//
// A work item is (kv head hk, sequence b, block j, slice of the block's hit
// list): the queries that selected block j, each with its G heads of kv head
// hk.  The list is cut into 128-row chunks (128/G tokens x G heads); every
// chunk yields, per row, the softmax partial over the keys of block j (keys
// after the query position masked):
//   S = Q K^T          (tcgen05, S in tensor memory)
//   P = 2^(S*c - m)    (registers; bf16 P written back over S)
//   O = P V            (tcgen05, A operand read from tensor memory)
//   partial row: O / l in bf16, lse = ln(l) + m  (per query, slot and head)
// and a later kernel merges the K partials of each row by their lse.  Blocks
// of at most 128 keys keep K_j and V_j resident per item (resident kernel);
// longer blocks stream them in 128-key sub-tiles (streamed kernel).  Work
// items are taken from a global queue by persistent CTAs, one per SM.
// ===========================================================================
struct AttnParams {
    const __nv_bfloat16 *q;
    const int32_t *row_ptr;
    const int32_t *entries;
    const AttnItem *items;
    int *counters;  // this launch's pair: [0] items per kv head, [1] work cursor
    __nv_bfloat16 *part_o;
    float *part_lse;
    int *status;
    int Hq;  // query heads of q (its row stride in heads)
    int n_q, T;
    int Hp;  // heads per partial row: this launch's kv heads x G
    int Hkv, G, block, K, N;
    int NK;      // keys per sub-tile (min(block, 128))
    int NS;      // sub-tiles per block
    int TOK;     // tokens per 128-row chunk = 128 / G
    int log2G;
    float scale_log2;
};

// Token table of one work item (at most kItemTokens hit-list entries),
// built once per item in shared memory.
constexpr int kItemTokens = 2048;
struct ItemRows {
    int qo16[kItemTokens];        // offset of the token's head group hk in q, 16-byte units (0 if none)
    int entry[kItemTokens];       // list entry = partial row (b*n_q + i)*K + slot, or -1
    int t[kItemTokens];           // query position, or -1
};

// Parameters of the own-block pass: the rows of each block whose own block
// it is (consecutive queries, causal within the block).  Each row's partial
// goes to the slot of its selection that holds the own block, as the
// hit-list pass would have written it; the hit lists leave those entries out.
struct OwnAttnParams : AttnParams {
    const int32_t *ids;  // [rows][K] selection (finds the own slot of each row)
};

// Token table entry of the own-block pass for token k of the own rows of
// block j: the entry (query row * K + the slot holding j) and position t, or
// -1 / -1 for a row whose selection does not hold its own block; q offset as
// in the hit-list pass.
template <int D>
__device__ __forceinline__ void own_token(const OwnAttnParams &p, int b, int j, int hk, int k,
                                          int &e, int &t, int &qo16) {
    const int t0 = max(j * p.block, p.T - p.n_q);
    const int qrow = b * p.n_q + (t0 + k - (p.T - p.n_q));
    int s_own = -1;
    for (int s = 0; s < p.K; ++s)
        if (p.ids[static_cast<long long>(qrow) * p.K + s] == j) s_own = s;
    e = s_own >= 0 ? qrow * p.K + s_own : -1;
    t = s_own >= 0 ? t0 + k : -1;
    qo16 = static_cast<int>((static_cast<long long>(qrow) * p.Hq + static_cast<long long>(hk) * p.G) * (D / 8));
}

// ===========================================================================
// Prefill attention, K/V block resident (block <= 128): warp-specialised.
//   warps 0-3 / 4-7: softmax warpgroups SG0 / SG1.  Each takes alternate
//     128-row chunks of the item: wait for S (which releases the Q tile),
//     softmax (S -> P in tensor memory), store the rows' lse, hand 1/l to
//     the epilogue warpgroup, issue PV, then S of its next chunk right
//     behind it (the MMAs of one thread execute in issue order, so S does
//     not overwrite P before PV has read it).  One elected thread per warpgroup issues that warpgroup's
//     tcgen05.mma.
//   warps 8-11: epilogue warpgroup.  For every chunk in order: read O from
//     tensor memory (which frees it for the next PV), scale by 1/l, stage
//     the bf16 partial rows token-major in one of two staging buffers and
//     write each token's G rows with one bulk copy.
//   warps 12-15: producers.  Thread 0 of them TMA-loads K_j and V_j once per
//     item; all gather the Q rows of chunks 0, 1, 2, ... into the owning
//     softmax warpgroup's Q tile: rows are loaded into registers (not
//     allocated in L1) before the tile is known to be free, then stored in
//     the 128-byte-swizzled layout.
// Every handshake is an mbarrier per softmax warpgroup; each side waits for
// the other's previous phase, so no signaller runs two phases ahead.
// Tensor memory: SG w owns columns [256w, 256w+256): S/P at +0, O at +128.
// ===========================================================================
constexpr int kResidentThreads = 512;

template <int D>
__global__ void __launch_bounds__(kResidentThreads, 1) prefill_attn_resident_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    AttnParams p) {
    constexpr int DREG = D / 64;
    constexpr uint32_t QT = DREG * kRegionBytes;   // Q tile
    constexpr uint32_t STB = QT + 2048;            // staging: 16-byte pad per token
    constexpr int PPR = D / 8;        // 16-byte pieces per row
    constexpr int NPROD = 128;        // producer threads (warps 12-15)
    constexpr int NLD = PPR;          // pieces per producer thread per chunk
    constexpr int RSTEP = NPROD / PPR;
    const int NK = p.NK;
    const uint32_t kv_tile = static_cast<uint32_t>(NK) * 128u * DREG;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = align1024(smem_raw);
    unsigned char *kv_s = base;                        // K tile, V tile
    unsigned char *q_s = kv_s + 2 * kv_tile;           // Q tile [sg]
    unsigned char *st_s = q_s + 2 * QT;                // staging [2]
    float2 *ml_s = reinterpret_cast<float2 *>(st_s + 2 * STB);  // (m, l) [sg][row]
    ItemRows *tab = reinterpret_cast<ItemRows *>(ml_s + 2 * 128);
    uint64_t *kvfull = reinterpret_cast<uint64_t *>(tab + 1);
    uint64_t *bar_s = kvfull + 1;      // [sg] S complete
    uint64_t *bar_o = kvfull + 3;      // [sg] PV complete
    uint64_t *q_ready = kvfull + 5;    // [sg] Q tile gathered
    uint64_t *q_free = kvfull + 7;     // [sg] Q tile read by S
    uint64_t *ml_ready = kvfull + 9;   // [sg] row statistics written
    uint64_t *o_free = kvfull + 11;    // [sg] O read by the epilogue warpgroup
    int *sh_item = reinterpret_cast<int *>(kvfull + 13);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sh_item + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid / 32;
    const int role = warp >> 2;        // 0, 1: softmax; 2: epilogue; 3: producers
    const int wg = role & 1, wtid = tid & 127;
    const uint32_t role_bar = 1 + role;
    if (tid == 0) {
        mbar_init(kvfull, 1);
        for (int w = 0; w < 2; ++w) {
            mbar_init(bar_s + w, 1);
            mbar_init(bar_o + w, 1);
            mbar_init(q_ready + w, 1);
            mbar_init(q_free + w, 1);
            mbar_init(ml_ready + w, 1);
            mbar_init(o_free + w, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_s = tmem_base + static_cast<uint32_t>(wg * 256);
    const uint32_t tmem_o = tmem_s + 128;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint64_t pol_first = l2_policy_evict_first(), pol_last = l2_policy_evict_last();

    const int n_items = p.counters[0];
    const int total = n_items * p.Hkv;
    const int G = p.G, TOK = p.TOK, K = p.K;
    const int row = wtid;
    const int tok = row >> p.log2G, g = row & (G - 1);

    // phase counters (each thread keeps those of its own role)
    uint32_t s_n = 0, pv_n = 0, qr_n = 0, item_n = 0;  // softmax warpgroup
    uint32_t eo_n[2] = {0, 0}, ec_n = 0;                // epilogue: per-sg chunks, all chunks
    uint32_t pf[2] = {0, 0};                            // producers: q_free phases
    int kv_armed = -1;
    bool aborted = false;
    int cur_j = 0, cur_hk = 0;

    // bounded wait of the role's thread 0, outcome shared by the role's 128 threads
    auto wait_role = [&](uint64_t *bar, uint32_t parity) -> bool {
        bool ok = true;
        if (wtid == 0) ok = mbar_wait(bar, parity, abort_flag, p.status);
        return !named_barrier_or(role_bar, 128, !ok || *abort_flag);
    };
    const uint32_t idesc_s = idesc_bf16_f32(128, NK, false);
    const uint32_t idesc_o = idesc_bf16_f32(128, D, true);
    // S = Q K^T for the warpgroup's Q tile (elected thread)
    auto issue_s = [&]() {
        tc_fence_after();
        const uint32_t qa = smem_addr(q_s + wg * QT), ka = smem_addr(kv_s);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
            umma_bf16(tmem_s, sdesc_sw128(qa + (kk / 4) * kRegionBytes + (kk % 4) * 32, 16, 1024),
                      sdesc_sw128(ka + (kk / 4) * NK * 128 + (kk % 4) * 32, 16, 1024), idesc_s,
                      kk > 0 ? 1u : 0u);
        umma_commit(bar_s + wg);
    };
    // O = P V with P (bf16) in tensor memory (elected thread)
    auto issue_pv = [&]() {
        tc_fence_after();
        const uint32_t va = smem_addr(kv_s + kv_tile);
        for (int kk = 0; kk < NK / 16; ++kk)
            umma_bf16_tmem_a(tmem_o, tmem_s + kk * 8,
                             sdesc_sw128(va + kk * 16 * 128, static_cast<uint32_t>(NK) * 128, 1024),
                             idesc_o, kk > 0 ? 1u : 0u);
        umma_commit(bar_o + wg);
    };

    // Softmax of this thread's row in one pass over tensor memory, 32 columns
    // at a time.  P = 2^(s*c - m_ref) with m_ref the first group's maximum;
    // a later group whose maximum exceeds m_ref by more than 8 (log2 units)
    // raises m_ref and rescales the P columns already written and the sum
    // (rare; any m_ref gives the same O / l and lse, it only has to keep the
    // terms in range).  P is written as bf16 over the S columns already read.
    // Rows away from the diagonal block skip the causal mask (warp-uniform).
    auto softmax_tile = [&](int c, float &m_run, float &l_run) {
        tc_fence_after();
        const int t = tab->t[c * TOK + tok];
        const int lim = t - cur_j * p.block;  // valid key columns: <= lim
        const bool wmask = __any_sync(0xffffffffu, lim < NK - 1);
        const float sc = p.scale_log2;
        const uint64_t sc2 = f2_pack(sc, sc);
        float mref = -INFINITY;
        float lsum = 0.f;
        for (int cc = 0; cc < NK / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem_s + lane_addr + cc * 32, v);
            tmem_wait_ld();
            if (wmask) {
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    if (cc * 32 + x > lim) v[x] = __float_as_uint(-INFINITY);
            }
            float g4[4] = {__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]), __uint_as_float(v[3])};
#pragma unroll
            for (int x = 4; x < 32; x += 8) {
                g4[0] = fmax3(g4[0], __uint_as_float(v[x]), __uint_as_float(v[x + 4]));
                g4[1] = fmax3(g4[1], __uint_as_float(v[x + 1]), __uint_as_float(v[x + 5]));
                g4[2] = fmax3(g4[2], __uint_as_float(v[x + 2]), __uint_as_float(v[x + 6]));
                g4[3] = fmax3(g4[3], __uint_as_float(v[x + 3]), __uint_as_float(v[x + 7]));
            }
            const float gm = fmaxf(fmax3(g4[0], g4[1], g4[2]), g4[3]) * sc;
            if (__any_sync(0xffffffffu, gm > mref + 8.f)) {
                const float mnew = fmaxf(mref, gm);
                // factor for what was accumulated with the old reference
                const float f = (mref == -INFINITY || mnew == -INFINITY) ? 0.f : ex2_approx(mref - mnew);
                if (cc > 0) tmem_wait_st();  // the P groups written so far are readable
                for (int g = 0; g < cc; ++g) {  // warp-collective; f = 1 leaves a row unchanged
                    uint32_t w16[16];
                    tmem_ld16(tmem_s + lane_addr + g * 16, w16);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w16[x]);
                        w16[x] = pack_bf16x2(__low2float(h) * f, __high2float(h) * f);
                    }
                    tmem_st16(tmem_s + lane_addr + g * 16, w16);
                }
                lsum *= f;
                mref = mnew;
            }
            const float mr = mref == -INFINITY ? 0.f : mref;
            const uint64_t nm2 = f2_pack(-mr, -mr);
            uint64_t ls2a = f2_pack(0.f, 0.f), ls2b = ls2a;
            uint32_t w16[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                float a0, a1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * x]), __uint_as_float(v[2 * x + 1])), sc2, nm2), a0, a1);
                const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);  // masked (-inf) columns give 0
                if (x & 1)
                    ls2b = f2_add(ls2b, f2_pack(p0, p1));
                else
                    ls2a = f2_add(ls2a, f2_pack(p0, p1));
                w16[x] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tmem_s + lane_addr + cc * 16, w16);
            float la0, la1, lb0, lb1;
            f2_unpack(ls2a, la0, la1);
            f2_unpack(ls2b, lb0, lb1);
            lsum += (la0 + la1) + (lb0 + lb1);
        }
        m_run = mref;
        l_run = lsum;
        tmem_wait_st();
        tc_fence_before();
    };

    // lse of this thread's row of chunk c (softmax warpgroup), natural log
    auto store_lse = [&](int c, float m_run, float l_run) {
        const int e = tab->entry[c * TOK + tok];
        if (e >= 0) {
            const long long prow = static_cast<long long>(e) * p.Hp + static_cast<long long>(cur_hk) * G + g;
            p.part_lse[prow] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2f : -INFINITY;
        }
    };
    // epilogue warpgroup, chunk c of softmax warpgroup w: partial rows of O
    // scaled by 1/l, as bf16, staged token-major (16-byte pad per token), one
    // bulk copy per token.  Returns false on abort.
    auto epilogue = [&](int c, int w) -> bool {
        if (!wait_role(bar_o + w, eo_n[w] & 1) || !wait_role(ml_ready + w, eo_n[w] & 1)) return false;
        ++eo_n[w];
        const float inv_l = ml_s[w * 128 + row].y;  // 1 / l, or 0 for a row without keys
        unsigned char *stage = st_s + (ec_n & 1) * STB;
        ++ec_n;
        // the bulk copies that last read this staging buffer (two chunks ago) are done
        if (g == 0) bulk_wait_read_1();
        if (G <= 32)
            __syncwarp();
        else
            named_barrier(role_bar, 128);
        tc_fence_after();
        const uint32_t to = tmem_base + static_cast<uint32_t>(w * 256 + 128);
        const uint64_t il2 = f2_pack(inv_l, inv_l);
        const uint32_t tok_bytes = static_cast<uint32_t>(G * D * 2 + 16);
        unsigned char *srow = stage + tok * tok_bytes + g * (D * 2);
        // 16-byte piece q of this head row is stored at q ^ prot (the partial
        // layout the combine reads), so a phase's 8 lanes hit 8 bank groups
        const int prot = (g * (G >= 8 ? 1 : 8 / G)) & 7;
#pragma unroll
        for (int c64 = 0; c64 < D; c64 += 64) {
            uint32_t v[64];
            tmem_ld32(to + lane_addr + c64, *reinterpret_cast<uint32_t(*)[32]>(v));
            tmem_ld32(to + lane_addr + c64 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                uint32_t wv[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    float a0, a1;
                    f2_unpack(f2_mul(f2_pack(__uint_as_float(v[q4 * 8 + 2 * x]), __uint_as_float(v[q4 * 8 + 2 * x + 1])), il2), a0, a1);
                    wv[x] = pack_bf16x2(a0, a1);
                }
                *reinterpret_cast<uint4 *>(srow + ((c64 / 8 + q4) ^ prot) * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        }
        // O and the row statistics have been read: the warpgroup may issue its next PV
        tc_fence_before();
        named_barrier(role_bar, 128);
        if (wtid == 0) mbar_arrive(o_free + w);
        const int e = tab->entry[c * TOK + tok];
        fence_proxy_async_smem();
        if (G <= 32)
            __syncwarp();
        else
            named_barrier(role_bar, 128);
        if (g == 0) {
            if (e >= 0) {
                const long long prow0 = static_cast<long long>(e) * p.Hp + static_cast<long long>(cur_hk) * G;
                bulk_store_hint(p.part_o + prow0 * D, stage + tok * tok_bytes, static_cast<uint32_t>(G * D * 2), pol_first);
            }
            bulk_commit();  // one group per chunk (possibly empty) keeps the count in step
        }
        return true;
    };

    while (true) {
        if (tid == 0) *sh_item = atomicAdd(p.counters + 1, 1);
        __syncthreads();
        const int w = *sh_item;
        if (w >= total || *abort_flag) break;
        const int hk = w / n_items;
        const AttnItem item = p.items[w - hk * n_items];
        const int b = item.pair / p.N, j = item.pair - b * p.N;
        cur_j = j;
        cur_hk = hk;
        const int list_base = p.row_ptr[item.pair] + item.start;
        const int ntok = item.count;
        const int n_chunks = (ntok + TOK - 1) / TOK;

        if (role == 3 && wtid == 0) {
            mbar_arrive_expect_tx(kvfull, 2 * kv_tile);
            kv_armed = static_cast<int>(item_n & 1);
            const int z = b * p.T + j * p.block;
            for (int r = 0; r < DREG; ++r) {
                tma_load_3d(kv_s + r * NK * 128, &tm_k, kvfull, r * 64, hk, z);
                tma_load_3d(kv_s + kv_tile + r * NK * 128, &tm_v, kvfull, r * 64, hk, z);
            }
        }
        for (int i = tid; i < n_chunks * TOK; i += blockDim.x) {
            int e = -1, t = -1;
            int qo16 = 0;
            if (i < ntok) {
                e = p.entries[list_base + i];
                const int qrow = e >= 0 ? e / K : -1;
                const int bi = qrow >= 0 ? qrow / p.n_q : -1;
                if (e < 0 || bi != b) {
                    atomicOr(p.status, kDevBadIds);
                    e = -1;
                } else {
                    t = p.T - p.n_q + (qrow - bi * p.n_q);
                    qo16 = static_cast<int>((static_cast<long long>(qrow) * p.Hq + static_cast<long long>(hk) * G) * (D / 8));
                }
            }
            tab->entry[i] = e;
            tab->t[i] = t;
            tab->qo16[i] = qo16;
        }
        __syncthreads();

        if (role == 3) {
            // ---- producers
            const int cc = wtid % PPR, r0 = wtid / PPR;
            const uint4 *qcol = reinterpret_cast<const uint4 *>(p.q) + cc;
            for (int c = 0; c < n_chunks; ++c) {
                const int x = c & 1, ci = c >> 1;
                uint4 v[NLD];
#pragma unroll
                for (int k = 0; k < NLD; ++k) {  // padding rows read row 0 (their output is dropped)
                    const int r = r0 + k * RSTEP;
                    v[k] = ld_nc_na_16_hint(qcol + tab->qo16[c * TOK + (r >> p.log2G)] + (r & (G - 1)) * PPR, pol_last);
                }
                if (ci >= 1) {  // S of the warpgroup's chunk ci - 1 has read the tile
                    if (!wait_role(q_free + x, pf[x] & 1)) {
                        aborted = true;
                        break;
                    }
                    ++pf[x];
                }
                unsigned char *dst = q_s + x * QT + (cc / 8) * kRegionBytes;
#pragma unroll
                for (int k = 0; k < NLD; ++k)
                    *reinterpret_cast<uint4 *>(dst + sw128_offset(r0 + k * RSTEP, cc % 8)) = v[k];
                fence_proxy_async_smem();
                named_barrier(role_bar, 128);
                if (wtid == 0) mbar_arrive(q_ready + x);
            }
            // the K/V copies have landed before the item ends (returns at once
            // when a warpgroup already saw them; bounded otherwise)
            if (wtid == 0 && kv_armed >= 0) mbar_drain(kvfull, static_cast<uint32_t>(kv_armed));
            kv_armed = -1;
        } else if (role == 2) {
            // ---- epilogue warpgroup: every chunk of the item in order
            for (int c = 0; c < n_chunks; ++c)
                if (!epilogue(c, c & 1)) {
                    aborted = true;
                    break;
                }
        } else {
            // ---- softmax warpgroup: its chunks c = wg, wg + 2, ...
            const int n = (n_chunks + 1 - wg) / 2;
            if (n > 0) {
                if (!wait_role(kvfull, item_n & 1) || !wait_role(q_ready + wg, qr_n & 1)) {
                    aborted = true;
                } else {
                    ++qr_n;
                    if (wtid == 0) issue_s();
                }
            }
            for (int ci = 0; ci < n && !aborted; ++ci) {
                const int c = wg + 2 * ci;
                if (!wait_role(bar_s + wg, s_n & 1)) { aborted = true; break; }
                ++s_n;
                if (wtid == 0 && ci + 1 < n) mbar_arrive(q_free + wg);
                float m_run, l_run;
                softmax_tile(c, m_run, l_run);
                store_lse(c, m_run, l_run);
                // the epilogue warpgroup has read O and 1/l of the previous PV
                if (pv_n > 0 && !wait_role(o_free + wg, (pv_n - 1) & 1)) { aborted = true; break; }
                ml_s[wg * 128 + row] = make_float2(m_run, l_run > 0.f ? 1.f / l_run : 0.f);
                named_barrier(role_bar, 128);
                if (wtid == 0) {
                    mbar_arrive(ml_ready + wg);
                    issue_pv();
                }
                ++pv_n;
                if (ci + 1 < n) {
                    // S of the next chunk overwrites the P that the PV just
                    // issued reads: tcgen05.mma of one thread execute in
                    // issue order, so it needs only the next Q tile
                    if (!wait_role(q_ready + wg, qr_n & 1)) {
                        aborted = true;
                        break;
                    }
                    ++qr_n;
                    if (wtid == 0) issue_s();
                }
            }
        }
        ++item_n;
        if (__syncthreads_or(aborted)) {
            aborted = true;
            break;
        }
    }
    __syncthreads();
    bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}

// ===========================================================================
// Prefill attention, K/V block streamed (block > 128): warp-specialised.
// A block of NS * 128 keys is streamed as NS sub-tiles; each chunk of 128
// tile rows sees all of them in order, with O accumulated in tensor memory.
//   warps 0-3 / 4-7: softmax warpgroups SG0 / SG1, alternate chunks (SG0
//     takes chunk 2r, SG1 chunk 2r + 1 of round r).  Per sub-tile: wait for
//     S, softmax against the chunk's running reference maximum (a rise by
//     more than 8 rescales the P columns written so far, the running sum
//     and, past the first sub-tile, O), hand P to the MMA thread; after the
//     last sub-tile hand (m, l) to the epilogue warpgroup.
//   warps 8-11: epilogue warpgroup, as in the resident kernel (one staging
//     buffer).
//   warp 12 (one thread): streams K and V sub-tiles through a ring of three
//     tile slots (TMA) and issues every tcgen05.mma: S(x, r, s) once K_s and
//     (for s = 0) Q of the chunk are in -- it may follow PV(x, r, s - 1) at
//     once, since the MMAs of one thread execute in issue order;
//     PV(x, r, s) once P is in tensor memory and V_s is in.  A slot is
//     refilled when every reader of its tile has completed (commit).
//   warps 13-15: producers, gathering each chunk's Q rows (two halves per
//     tile, registers, evict-last) into the owning warpgroup's Q tile.
// Tensor memory: SG w owns columns [256w, 256w+256): S/P at +0, O at +128.
// With OwnAttnParams (the own-block pass) the items are each block's own
// rows, consecutive queries; a chunk attends only the sub-tiles up to the one
// holding its last row, and a round loads as many as its later chunk needs.
// ===========================================================================
constexpr int kStreamedThreads = 512;
constexpr int kKvSlots = 3;

template <int D, typename PT>
__global__ void __launch_bounds__(kStreamedThreads, 1) prefill_attn_streamed_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    PT p) {
    // PT = OwnAttnParams: the own-block pass (own rows of each block)
    constexpr bool OWN = std::is_same<PT, OwnAttnParams>::value;
    constexpr int DREG = D / 64;
    constexpr uint32_t QT = DREG * kRegionBytes;   // Q tile
    constexpr uint32_t STB = QT + 2048;            // staging: 16-byte pad per token
    constexpr int PPR = D / 8;                     // 16-byte pieces per row
    constexpr int NPROD = 96;                      // producer threads (warps 13-15)
    constexpr int RSTEP = NPROD / PPR;             // rows between a thread's pieces
    constexpr int NLDH = (64 + RSTEP - 1) / RSTEP; // pieces per thread per half tile
    const int NK = p.NK, NS = p.NS;
    const uint32_t kv_tile = static_cast<uint32_t>(NK) * 128u * DREG;  // one K or V sub-tile

    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = align1024(smem_raw);
    unsigned char *kv_s = base;                             // kKvSlots tile slots
    unsigned char *q_s = kv_s + kKvSlots * kv_tile;         // Q tile [sg]
    unsigned char *st_s = q_s + 2 * QT;                     // staging
    float2 *ml_s = reinterpret_cast<float2 *>(st_s + STB);  // (m, l) [sg][row]
    ItemRows *tab = reinterpret_cast<ItemRows *>(ml_s + 2 * 128);
    uint64_t *kvfull = reinterpret_cast<uint64_t *>(tab + 1);  // [slot] tile landed
    uint64_t *slot_free = kvfull + 3;  // [slot] every reader of the slot's tile completed
    uint64_t *bar_s = kvfull + 6;      // [sg] S complete
    uint64_t *bar_pv = kvfull + 8;     // [sg] a PV complete
    uint64_t *bar_o = kvfull + 10;     // [sg] last PV of a chunk complete
    uint64_t *q_ready = kvfull + 12;   // [sg] Q tile gathered
    uint64_t *q_free = kvfull + 14;    // [sg] Q tile read by the chunk's last S
    uint64_t *ml_ready = kvfull + 16;  // [sg] row statistics written
    uint64_t *o_free = kvfull + 18;    // [sg] O read by the epilogue warpgroup
    uint64_t *p_ready = kvfull + 20;   // [sg] P in tensor memory
    int *sh_item = reinterpret_cast<int *>(kvfull + 22);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sh_item + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid & 31;
    // 0, 1: softmax; 2: epilogue; 3: MMA / K-V thread; 4: producers
    const int role = warp < 12 ? (warp >> 2) : (warp == 12 ? 3 : 4);
    const int wg = role & 1, wtid = tid & 127;
    const int ptid = tid - 13 * 32;    // producer thread index
    const uint32_t role_bar = 1 + role;
    const uint32_t role_threads = role == 4 ? NPROD : 128;
    if (tid == 0) {
        for (int sl = 0; sl < kKvSlots; ++sl) {
            mbar_init(kvfull + sl, 1);
            mbar_init(slot_free + sl, 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(bar_s + w, 1);
            mbar_init(bar_pv + w, 1);
            mbar_init(bar_o + w, 1);
            mbar_init(q_ready + w, 1);
            mbar_init(q_free + w, 1);
            mbar_init(ml_ready + w, 1);
            mbar_init(o_free + w, 1);
            mbar_init(p_ready + w, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_s = tmem_base + static_cast<uint32_t>(wg * 256);
    const uint32_t tmem_o = tmem_s + 128;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint64_t pol_first = l2_policy_evict_first(), pol_last = l2_policy_evict_last();

    const int n_items = p.counters[0];
    const int total = n_items * p.Hkv;
    const int G = p.G, TOK = p.TOK, K = p.K;
    const int row = wtid;
    const int tok = row >> p.log2G, g = row & (G - 1);

    // phase counters (each thread keeps those of its own role)
    uint32_t s_n = 0, pv_n = 0, och = 0, item_n = 0;  // softmax warpgroup
    uint32_t eo_n[2] = {0, 0};                         // epilogue
    uint32_t mq[2] = {0, 0}, mp[2] = {0, 0}, gt = 0;   // MMA thread: S rounds, PVs, tiles loaded
    uint32_t pf[2] = {0, 0};                           // producers
    bool aborted = false;
    int cur_j = 0, cur_hk = 0;

    auto wait_role = [&](uint64_t *bar, uint32_t parity) -> bool {
        bool ok = true;
        if ((role == 4 ? ptid : wtid) == 0) ok = mbar_wait(bar, parity, abort_flag, p.status);
        return !named_barrier_or(role_bar, role_threads, !ok || *abort_flag);
    };
    const uint32_t idesc_s = idesc_bf16_f32(128, NK, false);
    const uint32_t idesc_o = idesc_bf16_f32(128, D, true);

    // Softmax of sub-tile s of chunk c for this thread's row, one pass of 32
    // columns at a time against the chunk's reference maximum mref (log2
    // units).  A group more than 8 above mref raises it: P columns already
    // written in this sub-tile, the running sum and (s > 0) O are scaled by
    // 2^(old - new) (O once PV of the previous sub-tile has completed).
    auto softmax_sub = [&](int c, int s, float &mref, float &lsum) -> bool {
        tc_fence_after();
        const int t = tab->t[c * TOK + tok];
        const int lim = t - (cur_j * p.block + s * NK);  // valid key columns: <= lim
        const bool wmask = __any_sync(0xffffffffu, lim < NK - 1);
        const float sc = p.scale_log2;
        const uint64_t sc2 = f2_pack(sc, sc);
        bool ok = true;
        float oscale = 1.f;  // factor owed by O (the earlier sub-tiles) after reference rises
        for (int cc = 0; cc < NK / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem_s + lane_addr + cc * 32, v);
            tmem_wait_ld();
            if (wmask) {
#pragma unroll
                for (int x = 0; x < 32; ++x)
                    if (cc * 32 + x > lim) v[x] = __float_as_uint(-INFINITY);
            }
            float g4[4] = {__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]), __uint_as_float(v[3])};
#pragma unroll
            for (int x = 4; x < 32; x += 8) {
                g4[0] = fmax3(g4[0], __uint_as_float(v[x]), __uint_as_float(v[x + 4]));
                g4[1] = fmax3(g4[1], __uint_as_float(v[x + 1]), __uint_as_float(v[x + 5]));
                g4[2] = fmax3(g4[2], __uint_as_float(v[x + 2]), __uint_as_float(v[x + 6]));
                g4[3] = fmax3(g4[3], __uint_as_float(v[x + 3]), __uint_as_float(v[x + 7]));
            }
            const float gm = fmaxf(fmax3(g4[0], g4[1], g4[2]), g4[3]) * sc;
            if (__any_sync(0xffffffffu, gm > mref + 8.f)) {
                const float mnew = fmaxf(mref, gm);
                const float f = (mref == -INFINITY || mnew == -INFINITY) ? 0.f : ex2_approx(mref - mnew);
                if (cc > 0) tmem_wait_st();  // the P groups written so far are readable
                for (int gq = 0; gq < cc; ++gq) {  // warp-collective; f = 1 leaves a row unchanged
                    uint32_t w16[16];
                    tmem_ld16(tmem_s + lane_addr + gq * 16, w16);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w16[x]);
                        w16[x] = pack_bf16x2(__low2float(h) * f, __high2float(h) * f);
                    }
                    tmem_st16(tmem_s + lane_addr + gq * 16, w16);
                }
                lsum *= f;
                oscale *= f;
                mref = mnew;
            }
            const float mr = mref == -INFINITY ? 0.f : mref;
            const uint64_t nm2 = f2_pack(-mr, -mr);
            uint64_t ls2a = f2_pack(0.f, 0.f), ls2b = ls2a;
            uint32_t w16[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                float a0, a1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * x]), __uint_as_float(v[2 * x + 1])), sc2, nm2), a0, a1);
                const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);  // masked (-inf) columns give 0
                if (x & 1)
                    ls2b = f2_add(ls2b, f2_pack(p0, p1));
                else
                    ls2a = f2_add(ls2a, f2_pack(p0, p1));
                w16[x] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tmem_s + lane_addr + cc * 16, w16);
            float la0, la1, lb0, lb1;
            f2_unpack(ls2a, la0, la1);
            f2_unpack(ls2b, lb0, lb1);
            lsum += (la0 + la1) + (lb0 + lb1);
        }
        if (s > 0 && __any_sync(0xffffffffu, oscale != 1.f)) {
            // O holds the earlier sub-tiles: once their last PV has completed,
            // scale it to the new reference (warp-collective; 1 leaves a row)
            bool okw = true;
            if (lane == 0) okw = mbar_wait(bar_pv + wg, (pv_n - 1) & 1, abort_flag, p.status);
            okw = __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
            if (!okw) ok = false;
            tc_fence_after();
            for (int c16 = 0; c16 < D && okw; c16 += 16) {
                uint32_t o[16];
                tmem_ld16(tmem_o + lane_addr + c16, o);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 16; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * oscale);
                tmem_st16(tmem_o + lane_addr + c16, o);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        return ok;
    };

    // epilogue warpgroup, chunk c of softmax warpgroup w (as in the resident
    // kernel, one staging buffer).  Returns false on abort.
    auto epilogue = [&](int c, int w) -> bool {
        if (!wait_role(bar_o + w, eo_n[w] & 1) || !wait_role(ml_ready + w, eo_n[w] & 1)) return false;
        ++eo_n[w];
        const float2 ml = ml_s[w * 128 + row];
        const float m_run = ml.x, l_run = ml.y;
        // the bulk copies of the previous chunk have read the staging rows
        if (g == 0) bulk_wait_read_all();
        if (G <= 32)
            __syncwarp();
        else
            named_barrier(role_bar, 128);
        tc_fence_after();
        const uint32_t to = tmem_base + static_cast<uint32_t>(w * 256 + 128);
        const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
        const uint64_t il2 = f2_pack(inv_l, inv_l);
        const uint32_t tok_bytes = static_cast<uint32_t>(G * D * 2 + 16);
        unsigned char *srow = st_s + tok * tok_bytes + g * (D * 2);
        // 16-byte piece q of this head row is stored at q ^ prot (the partial
        // layout the combine reads), so a phase's 8 lanes hit 8 bank groups
        const int prot = (g * (G >= 8 ? 1 : 8 / G)) & 7;
#pragma unroll
        for (int c64 = 0; c64 < D; c64 += 64) {
            uint32_t v[64];
            tmem_ld32(to + lane_addr + c64, *reinterpret_cast<uint32_t(*)[32]>(v));
            tmem_ld32(to + lane_addr + c64 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                uint32_t wv[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    float a0, a1;
                    f2_unpack(f2_mul(f2_pack(__uint_as_float(v[q4 * 8 + 2 * x]), __uint_as_float(v[q4 * 8 + 2 * x + 1])), il2), a0, a1);
                    wv[x] = pack_bf16x2(a0, a1);
                }
                *reinterpret_cast<uint4 *>(srow + ((c64 / 8 + q4) ^ prot) * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        }
        // O and the row statistics have been read: the next chunk's PV may overwrite O
        tc_fence_before();
        named_barrier(role_bar, 128);
        if (wtid == 0) mbar_arrive(o_free + w);
        const int e = tab->entry[c * TOK + tok];
        if (e >= 0) {
            const long long prow = static_cast<long long>(e) * p.Hp + static_cast<long long>(cur_hk) * G + g;
            p.part_lse[prow] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2f : -INFINITY;
        }
        fence_proxy_async_smem();
        if (G <= 32)
            __syncwarp();
        else
            named_barrier(role_bar, 128);
        if (g == 0) {
            if (e >= 0) {
                const long long prow0 = static_cast<long long>(e) * p.Hp + static_cast<long long>(cur_hk) * G;
                bulk_store_hint(p.part_o + prow0 * D, st_s + tok * tok_bytes, static_cast<uint32_t>(G * D * 2), pol_first);
            }
            bulk_commit();
        }
        return true;
    };

    while (true) {
        if (tid == 0) *sh_item = atomicAdd(p.counters + 1, 1);
        __syncthreads();
        const int w = *sh_item;
        if (w >= total || *abort_flag) break;
        const int hk = w / n_items;
        const AttnItem item = p.items[w - hk * n_items];
        const int b = item.pair / p.N, j = item.pair - b * p.N;
        cur_j = j;
        cur_hk = hk;
        const int list_base = p.row_ptr[item.pair] + item.start;
        const int ntok = item.count;
        const int n_chunks = (ntok + TOK - 1) / TOK;
        // sub-tiles chunk c attends: all NS, or in the own-block pass those up
        // to the one holding its last row's position (later keys are masked
        // for every row of the chunk); non-decreasing in c
        const int own_off = OWN ? max(j * p.block, p.T - p.n_q) - j * p.block + item.start : 0;
        auto n_sub = [&](int c) -> int {
            if constexpr (OWN)
                return min(NS, (own_off + min((c + 1) * TOK, ntok) - 1) / NK + 1);
            else
                return NS;
        };

        for (int i = tid; i < n_chunks * TOK; i += blockDim.x) {
            int e = -1, t = -1;
            int qo16 = 0;
            if constexpr (OWN) {
                if (i < ntok) own_token<D>(p, b, j, hk, item.start + i, e, t, qo16);
            } else if (i < ntok) {
                e = p.entries[list_base + i];
                const int qrow = e >= 0 ? e / K : -1;
                const int bi = qrow >= 0 ? qrow / p.n_q : -1;
                if (e < 0 || bi != b) {
                    atomicOr(p.status, kDevBadIds);
                    e = -1;
                } else {
                    t = p.T - p.n_q + (qrow - bi * p.n_q);
                    qo16 = static_cast<int>((static_cast<long long>(qrow) * p.Hq + static_cast<long long>(hk) * G) * (D / 8));
                }
            }
            tab->entry[i] = e;
            tab->t[i] = t;
            tab->qo16[i] = qo16;
        }
        __syncthreads();

        if (role == 4) {
            // ---- producers: chunk c goes to softmax warpgroup c & 1, two halves per tile
            const int cc = ptid % PPR, r0 = ptid / PPR;
            const uint4 *qcol = reinterpret_cast<const uint4 *>(p.q) + cc;
            for (int c = 0; c < n_chunks && !aborted; ++c) {
                const int x = c & 1, ci = c >> 1;
                unsigned char *dst = q_s + x * QT + (cc / 8) * kRegionBytes;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    uint4 v[NLDH];
#pragma unroll
                    for (int k = 0; k < NLDH; ++k) {
                        const int r = 64 * h + r0 + k * RSTEP;
                        if (k < NLDH - 1 || r < 64 * h + 64)  // padding rows read row 0 (output dropped)
                            v[k] = ld_nc_na_16_hint(qcol + tab->qo16[c * TOK + (r >> p.log2G)] + (r & (G - 1)) * PPR,
                                                    pol_last);
                    }
                    if (h == 0 && ci >= 1) {  // the last S of the warpgroup's previous chunk has read the tile
                        if (!wait_role(q_free + x, pf[x] & 1)) {
                            aborted = true;
                            break;
                        }
                        ++pf[x];
                    }
#pragma unroll
                    for (int k = 0; k < NLDH; ++k) {
                        const int r = 64 * h + r0 + k * RSTEP;
                        if (k < NLDH - 1 || r < 64 * h + 64)
                            *reinterpret_cast<uint4 *>(dst + sw128_offset(r, cc % 8)) = v[k];
                    }
                    asm volatile("" ::: "memory");  // one half's registers at a time
                }
                if (aborted) break;
                fence_proxy_async_smem();
                named_barrier(role_bar, NPROD);
                if (ptid == 0) mbar_arrive(q_ready + x);
            }
        } else if (role == 3) {
            // ---- K/V streaming and MMA issue (one thread)
            if (lane == 0) {
                const int R = (n_chunks + 1) / 2;              // rounds (chunk pairs)
                const int nr[2] = {R, n_chunks / 2};           // rounds with a chunk, per warpgroup
                // K_0 V_0 K_1 V_1 ... per round, as many sub-tiles as the
                // round's later chunk attends
                int ntiles = R * NS * 2;
                if constexpr (OWN) {
                    ntiles = 0;
                    for (int r = 0; r < R; ++r) ntiles += 2 * n_sub(min(2 * r + 1, n_chunks - 1));
                }
                int fr = 0, fs = 0;    // own-block pass: round and sub-tile of the next tile
                int tb[2] = {0, 0};    // own-block pass: first tile of each warpgroup's round
                const uint32_t t0 = gt;                        // first tile of the item (global count)
                int tl = 0;                                    // tiles of the item issued
                int readers[kKvSlots] = {0, 0, 0};
                int rr[2] = {0, 0}, ss[2] = {0, 0}, act[2] = {0, 0};  // act: 0 = S next, 1 = PV next
                bool ok = true;
                uint64_t tw = global_timer_ns();
                auto tile_in = [&](int ti) -> bool {  // tile ti of the item has landed
                    if (ti >= tl) return false;
                    const uint32_t gg = t0 + static_cast<uint32_t>(ti);
                    return mbar_test(kvfull + gg % kKvSlots, (gg / kKvSlots) & 1);
                };
                auto release = [&](int ti) {  // one reader of tile ti has issued its MMA
                    const uint32_t sl = (t0 + static_cast<uint32_t>(ti)) % kKvSlots;
                    if (--readers[sl] == 0) umma_commit(slot_free + sl);
                };
                while (ok && (rr[0] < nr[0] || rr[1] < nr[1])) {
                    bool progress = false;
                    // refill: the next tile once its slot's previous tile is released
                    if (tl < ntiles) {
                        const uint32_t gg = t0 + static_cast<uint32_t>(tl);
                        const uint32_t sl = gg % kKvSlots;
                        if (gg < kKvSlots || mbar_test(slot_free + sl, ((gg / kKvSlots) - 1) & 1)) {
                            int s;
                            if constexpr (OWN) {
                                s = fs;
                                readers[sl] = (fs < n_sub(2 * fr) ? 1 : 0) + (2 * fr + 1 < n_chunks ? 1 : 0);
                            } else {
                                const int pair = tl >> 1, r = pair / NS;
                                s = pair % NS;
                                readers[sl] = (2 * r + 1 < n_chunks) ? 2 : 1;
                            }
                            unsigned char *dst = kv_s + sl * kv_tile;
                            mbar_arrive_expect_tx(kvfull + sl, kv_tile);
                            const int z = b * p.T + j * p.block + s * NK;
                            for (int rg = 0; rg < DREG; ++rg)
                                tma_load_3d(dst + rg * NK * 128, (tl & 1) ? &tm_v : &tm_k, kvfull + sl, rg * 64, hk, z);
                            ++tl;
                            if constexpr (OWN) {
                                if (!(tl & 1) && ++fs == n_sub(min(2 * fr + 1, n_chunks - 1))) {
                                    fs = 0;
                                    ++fr;
                                }
                            }
                            progress = true;
                        }
                    }
                    for (int x = 0; x < 2; ++x) {
                        if (rr[x] >= nr[x]) continue;
                        const int tK = OWN ? tb[x] + 2 * ss[x] : (rr[x] * NS + ss[x]) * 2;
                        const int nsx = n_sub(2 * rr[x] + x);
                        const uint32_t ts = tmem_base + static_cast<uint32_t>(x * 256);
                        if (act[x] == 0) {
                            if (!tile_in(tK)) continue;
                            if (ss[x] == 0 && !mbar_test(q_ready + x, mq[x] & 1)) continue;
                            // S overwrites the P that this warpgroup's previous PV
                            // reads: that PV was issued earlier by this thread, and
                            // tcgen05.mma of one thread execute in issue order
                            tc_fence_after();
                            const uint32_t qa = smem_addr(q_s + x * QT);
                            const uint32_t ka = smem_addr(kv_s + ((t0 + tK) % kKvSlots) * kv_tile);
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                umma_bf16(ts, sdesc_sw128(qa + (kk / 4) * kRegionBytes + (kk % 4) * 32, 16, 1024),
                                          sdesc_sw128(ka + (kk / 4) * NK * 128 + (kk % 4) * 32, 16, 1024),
                                          idesc_s, kk > 0 ? 1u : 0u);
                            umma_commit(bar_s + x);
                            release(tK);
                            if (ss[x] == 0) ++mq[x];
                            act[x] = 1;
                        } else {
                            if (!mbar_test(p_ready + x, mp[x] & 1)) continue;
                            if (!tile_in(tK + 1)) continue;
                            tc_fence_after();
                            const uint32_t va = smem_addr(kv_s + ((t0 + tK + 1) % kKvSlots) * kv_tile);
                            for (int kk = 0; kk < NK / 16; ++kk)
                                umma_bf16_tmem_a(ts + 128, ts + kk * 8,
                                                 sdesc_sw128(va + kk * 16 * 128, static_cast<uint32_t>(NK) * 128, 1024),
                                                 idesc_o, (ss[x] > 0 || kk > 0) ? 1u : 0u);
                            umma_commit(bar_pv + x);
                            if (ss[x] == nsx - 1) umma_commit(bar_o + x);
                            release(tK + 1);
                            ++mp[x];
                            act[x] = 0;
                            if (++ss[x] == nsx) {
                                ss[x] = 0;
                                if constexpr (OWN) tb[x] += 2 * n_sub(min(2 * rr[x] + 1, n_chunks - 1));
                                ++rr[x];
                            }
                        }
                        progress = true;
                    }
                    if (progress) {
                        tw = global_timer_ns();
                    } else if (*abort_flag) {
                        ok = false;
                    } else if (global_timer_ns() - tw > kWaitLimitNs) {
                        *abort_flag = 1;
                        atomicOr(p.status, kDevTimeout);
                        ok = false;
                    }
                }
                if (!ok) {
                    aborted = true;
                    // copies still in flight land before the CTA moves on
                    for (int ti = tl > kKvSlots ? tl - kKvSlots : 0; ti < tl; ++ti) {
                        const uint32_t gg = t0 + static_cast<uint32_t>(ti);
                        mbar_drain(kvfull + gg % kKvSlots, (gg / kKvSlots) & 1);
                    }
                }
                gt = t0 + static_cast<uint32_t>(tl);
            }
        } else if (role == 2) {
            // ---- epilogue warpgroup: every chunk of the item in order
            for (int c = 0; c < n_chunks; ++c)
                if (!epilogue(c, c & 1)) {
                    aborted = true;
                    break;
                }
        } else {
            // ---- softmax warpgroup: chunks c = wg + 2r, every sub-tile of each
            const int n = (n_chunks + 1 - wg) / 2;
            for (int r = 0; r < n && !aborted; ++r) {
                const int c = wg + 2 * r;
                float mref = -INFINITY, lsum = 0.f;
                const int nsc = n_sub(c);
                for (int s = 0; s < nsc; ++s) {
                    if (!wait_role(bar_s + wg, s_n & 1)) { aborted = true; break; }
                    ++s_n;
                    if (wtid == 0 && s == nsc - 1 && r + 1 < n) mbar_arrive(q_free + wg);
                    const bool sok = softmax_sub(c, s, mref, lsum);
                    // the epilogue warpgroup has read O of this warpgroup's previous chunk
                    if (s == 0 && och > 0 && !wait_role(o_free + wg, (och - 1) & 1)) { aborted = true; break; }
                    if (s == nsc - 1) ml_s[wg * 128 + row] = make_float2(mref, lsum);
                    if (named_barrier_or(role_bar, 128, !sok)) { aborted = true; break; }
                    if (wtid == 0) {
                        if (s == nsc - 1) mbar_arrive(ml_ready + wg);
                        mbar_arrive(p_ready + wg);
                    }
                    ++pv_n;
                }
                ++och;
            }
        }
        ++item_n;
        if (__syncthreads_or(aborted)) {
            aborted = true;
            break;
        }
    }
    __syncthreads();
    bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}


}  // namespace

// ------------------------------------------------------------------ launchers
size_t selftest_smem_bytes(int N, int Kd) {
    return 1024 + static_cast<size_t>(Kd / 64) * kRegionBytes + static_cast<size_t>(Kd) * N * 2 + 64;
}

cudaError_t launch_selftest_umma(const CUtensorMap &tm_a, const CUtensorMap &tm_b, float *C,
                                 int N, int Kd, int b_mn_major, int a_tmem, int *status,
                                 cudaStream_t st) {
    const size_t smem = selftest_smem_bytes(N, Kd);
    cudaFuncSetAttribute(selftest_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    selftest_umma_kernel<<<1, 128, smem, st>>>(tm_a, tm_b, C, N, Kd, b_mn_major, a_tmem, status);
    return cudaGetLastError();
}

size_t prefill_index_smem_bytes(int d_idx, int elem_bytes) {
    const size_t rb = static_cast<size_t>(d_idx) * elem_bytes;  // bytes per key row
    return 1024 + 128 * rb + kIdxStages * kIdxKeys * rb + 256;
}

template <int D_IDX, int CAP, int EB>
static cudaError_t launch_index_t(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                  const IndexParams &ip, int grid, cudaStream_t st) {
    const size_t smem = prefill_index_smem_bytes(D_IDX, EB);
    cudaFuncSetAttribute(prefill_index_kernel<D_IDX, CAP, EB>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    prefill_index_kernel<D_IDX, CAP, EB><<<grid, 192, smem, st>>>(tm_q, tm_k, ip);
    return cudaGetLastError();
}

template <int EB>
static cudaError_t launch_index_eb(const Shape &sh, const CUtensorMap &tm_q,
                                   const CUtensorMap &tm_k, const IndexParams &ip, int grid,
                                   cudaStream_t st) {
    if (sh.d_idx == 128) {
        if (sh.K <= 8) return launch_index_t<128, 7, EB>(tm_q, tm_k, ip, grid, st);
        if (sh.K <= 16) return launch_index_t<128, 15, EB>(tm_q, tm_k, ip, grid, st);
        return launch_index_t<128, 31, EB>(tm_q, tm_k, ip, grid, st);
    }
    if (sh.K <= 8) return launch_index_t<64, 7, EB>(tm_q, tm_k, ip, grid, st);
    if (sh.K <= 16) return launch_index_t<64, 15, EB>(tm_q, tm_k, ip, grid, st);
    return launch_index_t<64, 31, EB>(tm_q, tm_k, ip, grid, st);
}

cudaError_t launch_prefill_index(const Shape &sh, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                 int32_t *ids, int *status, int num_sms, cudaStream_t st,
                                 bool int8_keys) {
    IndexParams ip;
    ip.ids = ids;
    ip.status = status;
    ip.Bt = sh.Bt;
    ip.n_q = sh.n_q;
    ip.T = sh.T;
    ip.block = sh.block;
    ip.K = sh.K;
    ip.n_qt = (sh.n_q + 127) / 128;
    ip.n_items = ip.n_qt * sh.Bt;
    const int grid = ip.n_items < num_sms ? ip.n_items : num_sms;
    return int8_keys ? launch_index_eb<1>(sh, tm_q, tm_k, ip, grid, st)
                     : launch_index_eb<2>(sh, tm_q, tm_k, ip, grid, st);
}

size_t prefill_attn_smem_bytes(const Shape &sh) {
    const int NK = sh.block < 128 ? sh.block : 128;
    const int NS = sh.block / NK;
    const size_t kv_tile = static_cast<size_t>(NK) * 128 * (sh.d / 64);
    const size_t q = static_cast<size_t>(sh.d / 64) * kRegionBytes + 2048;
    if (NS == 1)  // resident kernel: K/V, two Q tiles, two staging buffers, row statistics
        return 1024 + 2 * kv_tile + 2 * (q - 2048) + 2 * q + 2 * 128 * 8 + sizeof(ItemRows) + 160 + 32;
    // streamed kernel: K/V tile slots, two Q tiles, one staging buffer, row statistics
    return 1024 + kKvSlots * kv_tile + 2 * (q - 2048) + q + 2 * 128 * 8 + sizeof(ItemRows) + 192 + 32;
}

int prefill_attn_rows_per_item(int G) {
    const int tok = 128 / G;
    return 64 * tok < kItemTokens ? 64 * tok : kItemTokens;
}

cudaError_t launch_prefill_attn(const Shape &sh, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                                const void *q, const int32_t *row_ptr, const int32_t *entries,
                                const AttnItem *items, int *counters, int hk0, int nhk,
                                void *part_o, float *part_lse, int *status, int num_sms,
                                cudaStream_t st, const int32_t *own_ids) {
    AttnParams ap;
    // the kernel indexes heads within the launch's group: q starts at the
    // group's first head (the K/V tensor maps start there too), Hkv counts
    // the group's kv heads
    ap.q = static_cast<const __nv_bfloat16 *>(q) + static_cast<size_t>(hk0) * sh.G * sh.d;
    ap.row_ptr = row_ptr;
    ap.entries = entries;
    ap.items = items;
    ap.counters = counters;
    ap.part_o = static_cast<__nv_bfloat16 *>(part_o);
    ap.part_lse = part_lse;
    ap.status = status;
    ap.Hp = nhk * sh.G;
    ap.n_q = sh.n_q;
    ap.T = sh.T;
    ap.Hq = sh.Hq;
    ap.Hkv = nhk;
    ap.G = sh.G;
    ap.block = sh.block;
    ap.K = sh.K;
    ap.N = sh.N;
    ap.NK = sh.block < 128 ? sh.block : 128;
    ap.NS = sh.block / ap.NK;
    ap.TOK = 128 / sh.G;
    ap.log2G = 0;
    while ((1 << ap.log2G) < sh.G) ++ap.log2G;
    ap.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(sh.d));
    const size_t smem = prefill_attn_smem_bytes(sh);
#define MSA_LAUNCH(KERNEL, THREADS, PARAMS)                                                      \
    do {                                                                                         \
        cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize,                \
                             static_cast<int>(smem));                                            \
        KERNEL<<<num_sms, THREADS, smem, st>>>(tm_k, tm_v, PARAMS);                              \
    } while (0)
    if (own_ids) {  // the own-block pass
        OwnAttnParams op;
        static_cast<AttnParams &>(op) = ap;
        op.ids = own_ids;
        if (ap.NS == 1) return cudaErrorInvalidValue;  // blocks of one sub-tile have no own pass
        if (sh.d == 128) MSA_LAUNCH((prefill_attn_streamed_kernel<128, OwnAttnParams>), kStreamedThreads, op);
        else MSA_LAUNCH((prefill_attn_streamed_kernel<64, OwnAttnParams>), kStreamedThreads, op);
        return cudaGetLastError();
    }
    if (ap.NS == 1) {
        if (sh.d == 128) MSA_LAUNCH(prefill_attn_resident_kernel<128>, kResidentThreads, ap);
        else MSA_LAUNCH(prefill_attn_resident_kernel<64>, kResidentThreads, ap);
    } else {
        if (sh.d == 128) MSA_LAUNCH((prefill_attn_streamed_kernel<128, AttnParams>), kStreamedThreads, ap);
        else MSA_LAUNCH((prefill_attn_streamed_kernel<64, AttnParams>), kStreamedThreads, ap);
    }
#undef MSA_LAUNCH
    return cudaGetLastError();
}

}  // namespace msa
