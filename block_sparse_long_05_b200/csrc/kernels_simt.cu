// kernels_simt.cu -- the HBM-bound and integer kernels of the MSA hot path:
//   * decode index scan + top-K select  (index branch, one query per sequence)
//   * split-K decode attention           (sparse branch, one query per sequence)
//   * log-sum-exp combine of partials    (prefill and decode)
//   * selection inversion (CSR of hit queries per KV block)
//
// Method: "MiniMax M3模型算力成本大幅降低原因深度解析" (index branch: single-head
// index key, block max-pool, top-K; sparse branch: GQA over the kept blocks)
// and "MiniMax M3 深度实战", sections 2.2 (KV outer gather Q: per-block hit
// lists), 2.3 (softmax(QK^T/sqrt(d))V over gathered keys) and 3.3 (decode).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "kernels.h"
#include "msa_common.cuh"

namespace msa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Total order on (score desc, block asc) packed into 64 bits: larger key
// ranks first.  Scores are finite.
__device__ __forceinline__ uint64_t rank_key(float s, int j) {
    uint32_t u = __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(0x7FFFFFFF - j);
}

// Warp-wide maximum of 64-bit keys in two reductions: the largest high word,
// then the largest low word among the lanes that hold it.
__device__ __forceinline__ uint64_t warp_max_key(uint64_t key) {
    const uint32_t hi = static_cast<uint32_t>(key >> 32), lo = static_cast<uint32_t>(key);
    const uint32_t mhi = __reduce_max_sync(0xFFFFFFFFu, hi);
    const uint32_t mlo = __reduce_max_sync(0xFFFFFFFFu, hi == mhi ? lo : 0u);
    return (static_cast<uint64_t>(mhi) << 32) | mlo;
}

// ------------------------------------------------------------------------
// Decode index scan: block_scores[b][j] = max_{i in block j} q_idx[b].k_idx[b][i]
// for j < own = (T-1)/block.  One CTA of 8 warps per (b, j); the warps split
// the block's rows; D_IDX/8 lanes per key row with 16-byte streaming loads,
// 16 loads in flight per warp.  fp32 accumulation (exact for integer keys).
// ------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream16(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Dot product of one 16-byte piece of a key row with this lane's piece of the
// query: 8 bf16 products in fp32, or 16 signed 8-bit products in exact
// integer arithmetic (dp4a).
struct ScanBf16 {
    static constexpr int EPL = 8;  // elements per 16-byte load
    float q[8];
    __device__ void load_q(const void *p) { bf16x8_to_f32(*reinterpret_cast<const uint4 *>(p), q); }
    __device__ float dot(const uint4 &u) const {
        float kf[8];
        bf16x8_to_f32(u, kf);
        float sc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) sc = fmaf(q[e], kf[e], sc);
        return sc;
    }
};
struct ScanS8 {
    static constexpr int EPL = 16;
    uint4 q;
    __device__ void load_q(const void *p) { q = *reinterpret_cast<const uint4 *>(p); }
    __device__ float dot(const uint4 &u) const {
        int acc = __dp4a(static_cast<int>(u.x), static_cast<int>(q.x), 0);
        acc = __dp4a(static_cast<int>(u.y), static_cast<int>(q.y), acc);
        acc = __dp4a(static_cast<int>(u.z), static_cast<int>(q.z), acc);
        acc = __dp4a(static_cast<int>(u.w), static_cast<int>(q.w), acc);
        return static_cast<float>(acc);  // |partial| <= 16 * 2^14: exact
    }
};

template <int D_IDX, typename SC>
__global__ void __launch_bounds__(256) decode_index_scan_kernel(
    const void *__restrict__ q_idx_v, const void *__restrict__ k_idx_v,
    float *__restrict__ block_scores, int Bt, int T, int block, int own, int N, int rw, int bpc,
    PageMap pm, int *__restrict__ status) {
    // rw: rows per warp (a warp's rows lie in one block); bpc: blocks per CTA
    constexpr int EB = 16 / SC::EPL;  // bytes per element
    constexpr int LPR = D_IDX / SC::EPL;  // lanes per key row
    constexpr int RPL = 32 / LPR;   // key rows per warp load
    constexpr int UNR = 16;         // loads in flight per warp
    __shared__ float wmax[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / LPR, part = lane % LPR;
    const int wpb = 8 / bpc;                         // warps per block
    const long long item = static_cast<long long>(blockIdx.x) * bpc + warp / wpb;
    bool active = item < static_cast<long long>(Bt) * own;
    float best = -FLT_MAX;
    long long row0 = 0;  // first k_idx row of the block in the (paged or contiguous) store
    if (active) {
        const int b = static_cast<int>(item / own), j = static_cast<int>(item % own);
        if (pm.table) {
            const int phys = pm.table[static_cast<long long>(b) * pm.stride + j];
            if (phys < 0 || phys >= pm.count) {  // skipped (scores -FLT_MAX) and reported
                active = false;
                if (lane == 0 && warp % (8 / bpc) == 0) atomicOr(status, kDevBadIds);
            }
            row0 = static_cast<long long>(phys) * block;
        } else {
            row0 = static_cast<long long>(b) * T + static_cast<long long>(j) * block;
        }
    }
    if (active) {
        const int b = static_cast<int>(item / own);
        const unsigned char *q_idx = static_cast<const unsigned char *>(q_idx_v);
        const unsigned char *k_idx = static_cast<const unsigned char *>(k_idx_v);
        SC qv;
        qv.load_q(q_idx + (static_cast<long long>(b) * D_IDX + part * SC::EPL) * EB);
        // the wpb warps of block j interleave over its row groups
        const int wi = warp % wpb;
        const uint4 *base = reinterpret_cast<const uint4 *>(k_idx + row0 * D_IDX * EB);
        const int groups = rw / RPL;  // row groups per warp
        for (int g0 = 0; g0 < groups; g0 += UNR) {
            uint4 ku[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int gi = wi + wpb * (g0 + u);
                ku[u] = g0 + u < groups ? ld_stream16(base + (gi * RPL + sub) * LPR + part)
                                        : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                float sc = qv.dot(ku[u]);
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1) sc += __shfl_xor_sync(0xFFFFFFFFu, sc, o);
                if (g0 + u < groups) best = fmaxf(best, sc);
            }
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) best = fmaxf(best, __shfl_xor_sync(0xFFFFFFFFu, best, o));
    }
    if (lane == 0) wmax[warp] = best;
    __syncthreads();
    if (threadIdx.x < bpc) {
        const long long it = static_cast<long long>(blockIdx.x) * bpc + threadIdx.x;
        if (it < static_cast<long long>(Bt) * own) {
            float m = -FLT_MAX;
            for (int w = threadIdx.x * wpb; w < (threadIdx.x + 1) * wpb; ++w) m = fmaxf(m, wmax[w]);
            block_scores[(it / own) * N + it % own] = m;
        }
    }
}

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start before the previous kernel in its
// stream has finished; this waits until that kernel has completed and its
// writes are visible.  A no-op for kernels launched the ordinary way.
__device__ __forceinline__ void grid_dep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------------------
// Decode select: one CTA of 1024 threads per sequence; a thread holds up to 8
// strided candidates as 64-bit keys (score desc, block asc).  m =
// min(K, own+1)-1 winners: every warp first extracts its own m best keys with
// warp max-reductions (redux.sync on the high, then the low word), then warp 0
// merges the 32 sorted lists (m rounds of a warp arg-max over the list
// heads).  own is added; each id is written at its rank (ascending).
// ------------------------------------------------------------------------
constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(kSelThreads) decode_select_kernel(
    const float *__restrict__ block_scores, int32_t *__restrict__ ids, int N, int own, int K) {
    grid_dep_wait();  // inputs come from the previous kernel in the stream
    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ uint64_t wtop[32 * kMaxK];  // per warp: its best keys, descending
    __shared__ int sel[kMaxK + 1];
    const float *sc = block_scores + static_cast<long long>(b) * N;
    const int m = min(K, own + 1) - 1;
    // candidates of this thread: j = tid, tid + 1024, ...  (own <= 8192 -> <= 8)
    uint64_t mine[8];
    int nm = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int j = tid + q * kSelThreads;
        mine[q] = j < own ? rank_key(sc[j], j) : 0;
        nm += j < own;
    }
    // stage 1: every warp takes its own m best keys, in order, with warp
    // reductions only (keys are unique, so a winner has one owner)
    for (int p = 0; p < m; ++p) {
        uint64_t best = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) best = mine[q] > best ? mine[q] : best;
        best = warp_max_key(best);
        if (best != 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (mine[q] == best) mine[q] = 0;
        }
        if (lane == 0) wtop[warp * kMaxK + p] = best;  // 0: the warp has no more candidates
    }
    __syncthreads();
    // stage 2: warp 0 merges the 32 descending lists, m rounds of a warp arg-max
    // over the list heads; the winning list advances
    if (warp == 0) {
        int ptr = 0;
        for (int p = 0; p < m; ++p) {
            const uint64_t head = ptr < m ? wtop[lane * kMaxK + ptr] : 0;
            const uint64_t best = warp_max_key(head);
            if (head == best && best != 0) ++ptr;
            if (lane == 0) sel[p] = 0x7FFFFFFF - static_cast<int>(static_cast<uint32_t>(best));
        }
        if (lane == 0) sel[m] = own;
    }
    __syncthreads();
    (void)nm;
    // ids ascending: each of the n = m + 1 distinct winners is written at its
    // rank; the slots after them get -1
    const int n = m + 1;
    if (tid < K) {
        int v = -1, slot = tid;
        if (tid < n) {
            v = sel[tid];
            slot = 0;
            for (int c = 0; c < n; ++c) slot += sel[c] < v;
        }
        ids[static_cast<long long>(b) * K + slot] = v;
    }
}

// ------------------------------------------------------------------------
// Split-K decode attention on mma.sync (m16n8k16, bf16 in, fp32 accumulate).
// One CTA of 4 warps per (b, kv head, slot, split of kDecodeKeys keys); warp
// w owns keys [16w, 16w+16) of the split.  K/V rows are staged in shared
// memory by 16-byte cp.async (coalesced 2*d-byte rows, padded by 16 bytes so
// ldmatrix reads are conflict-free; rows past the split's end are zero).  The
// G query heads of the kv head are processed 16 at a time (heads past G are
// zero rows): S = Q K^T (16 heads x 16 keys), softmax per head in the log2
// domain, O = P V with P taken straight from the S fragments; the four
// warps' partials are merged in shared memory.  Writes a normalised fp32
// partial and its natural-log lse (-inf when the split has no key).
// ------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <int D>
__global__ void __launch_bounds__(128) decode_attn_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, const int32_t *__restrict__ ids,
    float *__restrict__ part_o, float *__restrict__ part_lse, int T, int Hq, int Hkv, int block,
    int K, int S, int N, float scale_log2, PageMap pm, int *__restrict__ status) {
    grid_dep_wait();  // inputs come from the previous kernel in the stream
    constexpr int KS = kDecodeKeys;  // 64 keys = 4 warps x 16
    constexpr int STR = D + 8;       // padded row (bf16 elements)
    constexpr int PIECES = D / 8;    // 16-byte pieces per row
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __nv_bfloat16 *Ks = reinterpret_cast<__nv_bfloat16 *>(smem_raw);  // [KS][STR]
    __nv_bfloat16 *Vs = Ks + KS * STR;                                  // [KS][STR]
    __nv_bfloat16 *Qs = Vs + KS * STR;                                  // [16][STR]
    __nv_bfloat16 *Ps = Qs + 16 * STR;                                  // [16][KS + 8]
    float *mw = reinterpret_cast<float *>(Ps + 16 * (KS + 8));          // [4][16]
    float *lw = mw + 64;                                                // [4][16]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;  // mma fragment coordinates
    int idx = blockIdx.x;
    const int sp = idx % S;
    idx /= S;
    const int s = idx % K;
    idx /= K;
    const int hk = idx % Hkv;
    const int b = idx / Hkv;
    const int G = Hq / Hkv;
    const long long prow = (static_cast<long long>(b) * K + s) * S + sp;  // partial row
    const int t = T - 1;
    const int j = ids[static_cast<long long>(b) * K + s];
    int nk = 0;
    long long k0 = 0, row0 = 0;  // first key (logical position) and its row in the store
    if (j >= N || j < -1) {
        if (tid == 0) atomicOr(status, kDevBadIds);
    } else if (j >= 0) {
        k0 = static_cast<long long>(j) * block + static_cast<long long>(sp) * KS;
        long long k1 = k0 + KS;
        const long long blk_end = static_cast<long long>(j + 1) * block;
        if (k1 > blk_end) k1 = blk_end;
        if (k1 > T) k1 = T;
        if (k1 > t + 1) k1 = t + 1;
        nk = k1 > k0 ? static_cast<int>(k1 - k0) : 0;
        if (pm.table) {
            const int phys = pm.table[static_cast<long long>(b) * pm.stride + j];
            if (phys < 0 || phys >= pm.count) {  // skipped and reported
                if (tid == 0) atomicOr(status, kDevBadIds);
                nk = 0;
            }
            row0 = static_cast<long long>(phys) * block + static_cast<long long>(sp) * KS;
        } else {
            row0 = static_cast<long long>(b) * T + k0;
        }
    }
    if (nk == 0) {
        for (int g = tid; g < G; g += blockDim.x) part_lse[prow * Hq + hk * G + g] = -INFINITY;
        return;
    }
    // stage K and V rows (zero past nk)
    const __nv_bfloat16 *kbase = k + (row0 * Hkv + hk) * D;
    const __nv_bfloat16 *vbase = v + (row0 * Hkv + hk) * D;
    for (int e = tid; e < KS * PIECES; e += blockDim.x) {
        const int r = e / PIECES, c = e % PIECES;
        const bool ok = r < nk;
        const long long goff = ok ? static_cast<long long>(r) * Hkv * D + c * 8 : 0;
        const uint32_t bytes = ok ? 16u : 0u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(Ks + r * STR + c * 8))),
                     "l"(kbase + goff), "r"(bytes)
                     : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(Vs + r * STR + c * 8))),
                     "l"(vbase + goff), "r"(bytes)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const int key0 = warp * 16;  // this warp's keys

    for (int g0 = 0; g0 < G; g0 += 16) {
        // Q rows g0..g0+15 of this kv head group (zero past G), bf16
        const __nv_bfloat16 *qrow = q + (static_cast<long long>(b) * Hq + hk * G + g0) * D;
        for (int e = tid; e < 16 * PIECES; e += blockDim.x) {
            const int r = e / PIECES, c = e % PIECES;
            uint4 u = make_uint4(0, 0, 0, 0);
            if (g0 + r < G) u = *reinterpret_cast<const uint4 *>(qrow + r * D + c * 8);
            *reinterpret_cast<uint4 *>(Qs + r * STR + c * 8) = u;
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();

        // ---- S = Q K^T: 16 heads x 16 keys (two n-tiles of 8 keys)
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t af[4], bf[4];
            ldmatrix_x4(af, Qs + ((mi & 1) * 8 + ri) * STR + kk * 16 + (mi >> 1) * 8);
            ldmatrix_x4(bf, Ks + (key0 + (mi >> 1) * 8 + ri) * STR + kk * 16 + (mi & 1) * 8);
            mma_bf16_16816(acc[0], af, bf[0], bf[1]);
            mma_bf16_16816(acc[1], af, bf[2], bf[3]);
        }
        // ---- row max over the 64 keys (per-warp partials through shared memory)
        float x[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = key0 + nt * 8 + 2 * tq + (e & 1);
                x[nt][e] = key < nk ? acc[nt][e] * scale_log2 : -INFINITY;
            }
        float m0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        float m1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, o));
            m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, o));
        }
        if (tq == 0) {
            mw[warp * 16 + gq] = m0;
            mw[warp * 16 + gq + 8] = m1;
        }
        __syncthreads();
        float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            M0 = fmaxf(M0, mw[w * 16 + gq]);
            M1 = fmaxf(M1, mw[w * 16 + gq + 8]);
        }
        // key 0 of the split is always valid, so M0 and M1 are finite
        float pr[2][4];
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            pr[nt][0] = exp2f(x[nt][0] - M0);
            pr[nt][1] = exp2f(x[nt][1] - M0);
            pr[nt][2] = exp2f(x[nt][2] - M1);
            pr[nt][3] = exp2f(x[nt][3] - M1);
            l0 += pr[nt][0] + pr[nt][1];
            l1 += pr[nt][2] + pr[nt][3];
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, o);
            l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, o);
        }
        if (tq == 0) {
            lw[warp * 16 + gq] = l0;
            lw[warp * 16 + gq + 8] = l1;
        }
        // P (16 heads x 64 keys, bf16) to shared memory, row stride PSTR
        constexpr int PSTR = KS + 8;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = key0 + nt * 8 + 2 * tq;
            *reinterpret_cast<uint32_t *>(Ps + gq * PSTR + col) = bf16x2_bits(pr[nt][0], pr[nt][1]);
            *reinterpret_cast<uint32_t *>(Ps + (gq + 8) * PSTR + col) = bf16x2_bits(pr[nt][2], pr[nt][3]);
        }
        __syncthreads();
        // ---- O[:, 32w .. 32w+31] = P V over all 64 keys (4 k-steps x 4 n-tiles)
        constexpr int CW = D / 4;  // output columns per warp
        constexpr int NTW = CW / 8;
        float o[NTW][4];
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS / 16; ++kk) {
            uint32_t pa[4];
            ldmatrix_x4(pa, Ps + ((mi & 1) * 8 + ri) * PSTR + kk * 16 + (mi >> 1) * 8);
#pragma unroll
            for (int nt = 0; nt < NTW; nt += 2) {
                uint32_t vf[4];
                ldmatrix_x4_trans(vf, Vs + (kk * 16 + (mi & 1) * 8 + ri) * STR + warp * CW + (nt + (mi >> 1)) * 8);
                mma_bf16_16816(o[nt], pa, vf[0], vf[1]);
                mma_bf16_16816(o[nt + 1], pa, vf[2], vf[3]);
            }
        }
        const float L0 = lw[gq] + lw[16 + gq] + lw[32 + gq] + lw[48 + gq];
        const float L1 = lw[gq + 8] + lw[24 + gq] + lw[40 + gq] + lw[56 + gq];
        const float i0 = 1.f / L0, i1 = 1.f / L1;
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
            const int col = warp * CW + nt * 8 + 2 * tq;
            if (g0 + gq < G)
                *reinterpret_cast<float2 *>(part_o + (prow * Hq + hk * G + g0 + gq) * D + col) =
                    make_float2(o[nt][0] * i0, o[nt][1] * i0);
            if (g0 + gq + 8 < G)
                *reinterpret_cast<float2 *>(part_o + (prow * Hq + hk * G + g0 + gq + 8) * D + col) =
                    make_float2(o[nt][2] * i1, o[nt][3] * i1);
        }
        if (warp == 0 && tq == 0) {
            if (g0 + gq < G) part_lse[prow * Hq + hk * G + g0 + gq] = (M0 + log2f(L0)) * kLn2;
            if (g0 + gq + 8 < G) part_lse[prow * Hq + hk * G + g0 + gq + 8] = (M1 + log2f(L1)) * kLn2;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------
// Log-sum-exp combine.  One CTA per (query row, group of HG heads).  The P =
// K*S partials of each head are merged as LSE = log sum_p exp(lse_p) and
// out = sum_p exp(lse_p - LSE) o_p.  Weights are computed once into shared
// memory; the partial rows are then streamed with 16-byte loads (several in
// flight per thread).  Partial p = (slot s, split sp) is valid when
// 0 <= ids[row][s] < N and its lse is finite; invalid partials are never used
// (their memory may hold a previous call's data: the attention kernels write
// no partial for an id outside [0, N)).
// ------------------------------------------------------------------------
template <typename PT, int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(
    const PT *__restrict__ part_o, const float *__restrict__ part_lse,
    const int32_t *__restrict__ ids, float *__restrict__ out, float *__restrict__ lse_out, int Hq,
    int K, int S, int HG, int G, int N, int Hp, int h_off) {
    // partial rows hold Hp heads (query heads h_off .. h_off + Hp - 1 of out)
    grid_dep_wait();  // inputs come from the previous kernel in the stream
    constexpr int VEC = 16 / sizeof(PT);  // elements per 16-byte load
    constexpr int NV = D / VEC;           // 16-byte loads per head row
    extern __shared__ float wsm[];        // [P][HG] weights, then [HG] LSE
    const long long row = blockIdx.x;
    const int h0 = blockIdx.y * HG;
    const int P = K * S;
    float *Lsm = wsm + P * HG;
    const int tid = threadIdx.x;
    for (int e = tid; e < P * HG; e += blockDim.x) {
        const int pp = e / HG, hh = e % HG;
        const int s = pp / S;
        float l = -INFINITY;
        const int j = ids[row * K + s];
        if (j >= 0 && j < N) l = part_lse[((row * K + s) * S + pp % S) * Hp + h0 + hh];
        wsm[e] = l;
    }
    __syncthreads();
    for (int hh = tid; hh < HG; hh += blockDim.x) {
        float mx = -INFINITY;
        for (int pp = 0; pp < P; ++pp) mx = fmaxf(mx, wsm[pp * HG + hh]);
        float L = -INFINITY;
        if (mx != -INFINITY) {
            float sum = 0.f;
            for (int pp = 0; pp < P; ++pp) {
                const float l = wsm[pp * HG + hh];
                if (l != -INFINITY) sum += exp2f((l - mx) * kLog2e);
            }
            L = mx + log2f(sum) * kLn2;
        }
        for (int pp = 0; pp < P; ++pp) {
            const float l = wsm[pp * HG + hh];
            wsm[pp * HG + hh] = (l == -INFINITY) ? 0.f : exp2f((l - L) * kLog2e);
        }
        Lsm[hh] = L;
        lse_out[row * Hq + h_off + h0 + hh] = L;
    }
    __syncthreads();
    for (int e = tid; e < HG * NV; e += blockDim.x) {
        const int hh = e / NV, c = (e % NV) * VEC;
        float acc[VEC];
#pragma unroll
        for (int x = 0; x < VEC; ++x) acc[x] = 0.f;
        // G > 0: the prefill kernels store 16-byte piece q of a head row with
        // head index g inside its kv group at q ^ ((g * max(1, 8 / G)) & 7)
        const int gh = G > 0 ? ((h0 + hh) & (G - 1)) : 0;
        const int rot = G > 0 ? (gh * (G >= 8 ? 1 : 8 / G)) & 7 : 0;
        const int cr = ((c / VEC) ^ rot) * VEC;
        const PT *src = part_o + ((row * K) * S * Hp + h0 + hh) * static_cast<long long>(D) + cr;
        const long long pstride = static_cast<long long>(Hp) * D;  // between consecutive partials
#pragma unroll 4
        for (int pp = 0; pp < P; ++pp) {
            const float wgt = wsm[pp * HG + hh];
            const uint4 u = *reinterpret_cast<const uint4 *>(src + pp * pstride);
            if (sizeof(PT) == 2) {
                float f[8];
                bf16x8_to_f32(u, f);
#pragma unroll
                for (int x = 0; x < VEC; ++x) acc[x] += wgt != 0.f ? wgt * f[x] : 0.f;
            } else {
                const float f[4] = {__uint_as_float(u.x), __uint_as_float(u.y),
                                    __uint_as_float(u.z), __uint_as_float(u.w)};
#pragma unroll
                for (int x = 0; x < VEC; ++x) acc[x] += wgt != 0.f ? wgt * f[x] : 0.f;
            }
        }
        float *dst = out + (row * Hq + h_off + h0 + hh) * static_cast<long long>(D) + c;
#pragma unroll
        for (int x = 0; x < VEC; x += 4)
            *reinterpret_cast<float4 *>(dst + x) = make_float4(acc[x], acc[x + 1], acc[x + 2], acc[x + 3]);
    }
}

// Few query rows (decode): one CTA of NW warps per (row, head); warp w
// merges partials p = w, w+NW, ... of that head and the warps' sums are added
// in shared memory.  Same arithmetic as lse_combine_kernel.  NW = 8 while the
// grid fits the GPU in one wave of 8-warp CTAs, else 4 (smaller CTAs: one
// wave for twice the grid).
template <typename PT, int D, int NW>
__global__ void __launch_bounds__(32 * NW) lse_combine_split_kernel(
    const PT *__restrict__ part_o, const float *__restrict__ part_lse,
    const int32_t *__restrict__ ids, float *__restrict__ out, float *__restrict__ lse_out, int Hq,
    int K, int S, int N) {
    grid_dep_wait();  // inputs come from the previous kernel in the stream
    constexpr int PER = D / 32;  // elements per lane
    extern __shared__ float wsm[];                // [P] weights, then [NW][D] sums
    const long long row = blockIdx.x;
    const int h = blockIdx.y;
    const int P = K * S;
    float *acc_s = wsm + ((P + 3) & ~3);
    __shared__ float L_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int pp = tid; pp < P; pp += blockDim.x) {
        const int si = pp / S;
        float l = -INFINITY;
        const int j = ids[row * K + si];
        if (j >= 0 && j < N) l = part_lse[((row * K + si) * S + pp % S) * Hq + h];
        wsm[pp] = l;
    }
    __syncthreads();
    if (warp == 0) {
        float mx = -INFINITY;
        for (int pp = lane; pp < P; pp += 32) mx = fmaxf(mx, wsm[pp]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        float sum = 0.f;
        for (int pp = lane; pp < P; pp += 32) {
            const float l = wsm[pp];
            if (l != -INFINITY) sum += exp2f((l - mx) * kLog2e);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        const float L = mx == -INFINITY ? -INFINITY : mx + log2f(sum) * kLn2;
        __syncwarp();
        for (int pp = lane; pp < P; pp += 32) {
            const float l = wsm[pp];
            wsm[pp] = (l == -INFINITY) ? 0.f : exp2f((l - L) * kLog2e);
        }
        if (lane == 0) L_s = L;
    }
    __syncthreads();
    float acc[PER];
#pragma unroll
    for (int x = 0; x < PER; ++x) acc[x] = 0.f;
    const long long pstride = static_cast<long long>(Hq) * D;
    const PT *src = part_o + (row * K * S * Hq + h) * static_cast<long long>(D) + lane * PER;
#pragma unroll 4
    for (int pp = warp; pp < P; pp += NW) {
        const float wgt = wsm[pp];
        const PT *sp = src + pp * pstride;
        float f[PER];
        if (sizeof(PT) == 4 && PER == 4) {
            const float4 u = *reinterpret_cast<const float4 *>(sp);
            f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
        } else {
#pragma unroll
            for (int x = 0; x < PER; ++x) f[x] = static_cast<float>(sp[x]);
        }
#pragma unroll
        for (int x = 0; x < PER; ++x) acc[x] += wgt != 0.f ? wgt * f[x] : 0.f;
    }
#pragma unroll
    for (int x = 0; x < PER; ++x) acc_s[warp * D + lane * PER + x] = acc[x];
    __syncthreads();
    for (int c = tid; c < D; c += blockDim.x) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) a += acc_s[w * D + c];
        out[(row * Hq + h) * static_cast<long long>(D) + c] = a;
    }
    if (tid == 0) lse_out[row * Hq + h] = L_s;
}

// ------------------------------------------------------------------------
// Inversion.  Chunks of kInvRows query rows; warp w of a chunk owns rows
// [32w, 32w+32).  Per-warp histograms live in shared memory [4][N].
// ------------------------------------------------------------------------
// skip_own > 0 (the block size): leave out the entries of each row's own
// block (own(t) = t / block, t = T - n_q + i), which the own-block pass
// attends instead.
__device__ __forceinline__ void warp_histogram(const int32_t *__restrict__ ids, int *hist_w,
                                               int b, int n_q, int K, int N, int row0,
                                               int *status, int T, int skip_own) {
    const int lane = threadIdx.x % 32;
    const int i = row0 + lane;
    if (i < n_q) {
        const int32_t *r = ids + (static_cast<long long>(b) * n_q + i) * K;
        const int own = skip_own > 0 ? (T - n_q + i) / skip_own : -2;
        for (int s = 0; s < K; ++s) {
            const int j = r[s];
            if (j >= 0 && j < N) {
                if (j != own) atomicAdd(hist_w + j, 1);
            } else if (j != -1 && status) {
                atomicOr(status, kDevBadIds);
            }
        }
    }
}

__global__ void __launch_bounds__(128) inv_count_kernel(const int32_t *__restrict__ ids,
                                                         int *__restrict__ chunk_counts, int n_q,
                                                         int K, int N, int n_chunks,
                                                         int *__restrict__ status, int T,
                                                         int skip_own) {
    extern __shared__ int hist[];  // [4][N]
    const int chunk = blockIdx.x, b = blockIdx.y;
    for (int e = threadIdx.x; e < 4 * N; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int w = threadIdx.x / 32;
    warp_histogram(ids, hist + w * N, b, n_q, K, N, chunk * kInvRows + 32 * w, status, T, skip_own);
    __syncthreads();
    int *dst = chunk_counts + (static_cast<long long>(b) * n_chunks + chunk) * N;
    for (int j = threadIdx.x; j < N; j += blockDim.x)
        dst[j] = hist[j] + hist[N + j] + hist[2 * N + j] + hist[3 * N + j];
}

// Exclusive scan of one (b, j) column over the chunks, in place; total out.
__global__ void __launch_bounds__(256) inv_colscan_kernel(int *__restrict__ chunk_counts,
                                                           int *__restrict__ pair_totals, int N,
                                                           int n_chunks) {
    const int j = blockIdx.x, b = blockIdx.y;
    int *col = chunk_counts + static_cast<long long>(b) * n_chunks * N + j;
    __shared__ int warp_sums[8];
    const int per = (n_chunks + blockDim.x - 1) / blockDim.x;
    const int c0 = threadIdx.x * per;
    int local = 0;
    for (int c = c0; c < min(c0 + per, n_chunks); ++c) local += col[static_cast<long long>(c) * N];
    // block exclusive scan of `local`
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int warp_off = 0;
    for (int x = 0; x < warp; ++x) warp_off += warp_sums[x];
    int run = warp_off + incl - local;
    for (int c = c0; c < min(c0 + per, n_chunks); ++c) {
        const long long o = static_cast<long long>(c) * N;
        const int v = col[o];
        col[o] = run;
        run += v;
    }
    if (threadIdx.x == blockDim.x - 1) {
        int tot = 0;
        for (int x = 0; x < static_cast<int>(blockDim.x / 32); ++x) tot += warp_sums[x];
        pair_totals[static_cast<long long>(b) * N + j] = tot;
    }
}

// Single-CTA exclusive scans: row_ptr over pair totals; item_ptr over
// ceil(total / rows_per_item) (when items != nullptr); for each attention
// launch c < n_cursors, counters[2c] = items and counters[2c + 1] = 0 (its
// work cursor).
__global__ void __launch_bounds__(1024) inv_rowptr_kernel(const int *__restrict__ pair_totals,
                                                           int *__restrict__ row_ptr,
                                                           int *__restrict__ item_ptr,
                                                           int *__restrict__ counters, int n_pairs,
                                                           int rows_per_item, int n_cursors) {
    __shared__ int ws_a[32], ws_b[32];
    const int per = (n_pairs + blockDim.x - 1) / blockDim.x;
    const int p0 = threadIdx.x * per;
    int la = 0, lb = 0;
    for (int p = p0; p < min(p0 + per, n_pairs); ++p) {
        la += pair_totals[p];
        if (item_ptr) lb += (pair_totals[p] + rows_per_item - 1) / rows_per_item;
    }
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int ia = la, ib = lb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xFFFFFFFFu, ia, o);
        const int yb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
        if (lane >= o) {
            ia += ya;
            ib += yb;
        }
    }
    if (lane == 31) {
        ws_a[warp] = ia;
        ws_b[warp] = ib;
    }
    __syncthreads();
    int oa = 0, ob = 0;
    for (int x = 0; x < warp; ++x) {
        oa += ws_a[x];
        ob += ws_b[x];
    }
    int ra = oa + ia - la, rb = ob + ib - lb;
    for (int p = p0; p < min(p0 + per, n_pairs); ++p) {
        row_ptr[p] = ra;
        ra += pair_totals[p];
        if (item_ptr) {
            item_ptr[p] = rb;
            rb += (pair_totals[p] + rows_per_item - 1) / rows_per_item;
        }
    }
    if (threadIdx.x == blockDim.x - 1) {
        int ta = 0, tb = 0;
        for (int x = 0; x < static_cast<int>(blockDim.x / 32); ++x) {
            ta += ws_a[x];
            tb += ws_b[x];
        }
        row_ptr[n_pairs] = ta;
        if (item_ptr) {
            item_ptr[n_pairs] = tb;
            for (int c = 0; c < n_cursors; ++c) {
                counters[2 * c] = tb;
                counters[2 * c + 1] = 0;
            }
        }
    }
}

__global__ void __launch_bounds__(128) inv_scatter_kernel(
    const int32_t *__restrict__ ids, const int *__restrict__ chunk_prefix,
    const int *__restrict__ row_ptr, int32_t *__restrict__ entries, int n_q, int K, int N,
    int n_chunks, int *__restrict__ status, int T, int skip_own) {
    extern __shared__ int hist[];  // [4][N] counts, then cursors
    const int chunk = blockIdx.x, b = blockIdx.y;
    for (int e = threadIdx.x; e < 4 * N; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
    // bad ids were already reported by the count pass
    warp_histogram(ids, hist + w * N, b, n_q, K, N, chunk * kInvRows + 32 * w, nullptr, T,
                   skip_own);
    (void)status;
    __syncthreads();
    const int *pre = chunk_prefix + (static_cast<long long>(b) * n_chunks + chunk) * N;
    for (int j = threadIdx.x; j < N; j += blockDim.x) {
        int base = row_ptr[static_cast<long long>(b) * N + j] + pre[j];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int c = hist[x * N + j];
            hist[x * N + j] = base;
            base += c;
        }
    }
    __syncthreads();
    int *cursor = hist + w * N;
    const int row0 = chunk * kInvRows + 32 * w;
    for (int r = 0; r < 32; ++r) {
        const int i = row0 + r;
        if (i >= n_q) break;
        const long long row = static_cast<long long>(b) * n_q + i;
        const int own = skip_own > 0 ? (T - n_q + i) / skip_own : -2;
        if (lane < K) {
            const int j = ids[row * K + lane];
            if (j >= 0 && j < N && j != own) {
                const int pos = atomicAdd(cursor + j, 1);
                entries[pos] = static_cast<int32_t>(row * K + lane);
            }
        }
        __syncwarp();
    }
}

// Rows of each (sequence, block) pair whose own block it is: the queries
// t = T - n_q + i in [j * block, (j + 1) * block).
__global__ void __launch_bounds__(256) own_totals_kernel(int *__restrict__ own_totals, int n_q,
                                                          int T, int block, int N, int n_pairs) {
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= n_pairs) return;
    const int j = p % N;
    const long long lo = max(static_cast<long long>(j) * block, static_cast<long long>(T - n_q));
    const long long hi = min(static_cast<long long>(j + 1) * block, static_cast<long long>(T));
    own_totals[p] = hi > lo ? static_cast<int>(hi - lo) : 0;
}

__global__ void __launch_bounds__(256) attn_items_kernel(const int *__restrict__ pair_totals,
                                                          const int *__restrict__ item_ptr,
                                                          AttnItem *__restrict__ items,
                                                          int n_pairs, int rows_per_item) {
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= n_pairs) return;
    const int tot = pair_totals[p];
    int o = item_ptr[p];
    for (int s = 0; s < tot; s += rows_per_item) {
        AttnItem it;
        it.pair = p;
        it.start = s;
        it.count = min(rows_per_item, tot - s);
        it.pad = 0;
        items[o++] = it;
    }
}

}  // namespace

// ------------------------------------------------------------------ launchers
// Launch `kernel`; with pdl the kernel may be scheduled while the previous
// kernel in the stream drains (it calls grid_dep_wait before reading that
// kernel's results), which hides the launch gap between dependent kernels.
template <typename... KArgs, typename... Args>
static cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

cudaError_t launch_decode_scan(const Shape &sh, const void *q_idx, const void *k_idx,
                               float *block_scores, const PageMap &pm, int *status, int num_sms,
                               cudaStream_t st, bool int8_keys) {
    (void)num_sms;
    const int own = (sh.T - 1) / sh.block;
    if (own > 0) {
        // 8 warps per CTA; a warp scans at most 64 rows of one block (128
        // rows of int8 keys: the same bytes); small blocks are packed several
        // to a CTA
        const int rmax = int8_keys ? 128 : 64;
        int rw, bpc;
        if (sh.block <= 64) {
            rw = sh.block;
            bpc = 8;
        } else if (sh.block <= 8 * rmax && (8 * rmax) % sh.block == 0) {
            rw = rmax;
            bpc = 8 * rmax / sh.block;
        } else {
            rw = sh.block / 8;
            bpc = 1;
        }
        const long long items = static_cast<long long>(sh.Bt) * own;
        const long long grid = (items + bpc - 1) / bpc;
        const dim3 g(static_cast<unsigned>(grid));
#define MSA_SCAN(DI, SCT)                                                                      \
    decode_index_scan_kernel<DI, SCT><<<g, 256, 0, st>>>(q_idx, k_idx, block_scores, sh.Bt,   \
                                                        sh.T, sh.block, own, sh.N, rw, bpc, pm, \
                                                        status)
        if (int8_keys) {
            if (sh.d_idx == 128) MSA_SCAN(128, ScanS8); else MSA_SCAN(64, ScanS8);
        } else {
            if (sh.d_idx == 128) MSA_SCAN(128, ScanBf16); else MSA_SCAN(64, ScanBf16);
        }
#undef MSA_SCAN
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_select(const Shape &sh, const float *block_scores, int32_t *ids,
                                 cudaStream_t st, bool pdl) {
    const int own = (sh.T - 1) / sh.block;
    return launch_ex(decode_select_kernel, dim3(sh.Bt), dim3(kSelThreads), 0, st, pdl, block_scores,
                     ids, sh.N, own, sh.K);
}

size_t decode_attn_smem_bytes(const Shape &sh) {
    const size_t str = static_cast<size_t>(sh.d) + 8;
    return (2 * kDecodeKeys + 16) * str * 2 + static_cast<size_t>(16) * (kDecodeKeys + 8) * 2 + 128 * 4;
}

cudaError_t launch_decode_attn(const Shape &sh, const void *q, const void *k, const void *v,
                               const int32_t *ids, float *part_o, float *part_lse, int S,
                               const PageMap &pm, int *status, cudaStream_t st, bool pdl) {
    const long long grid = static_cast<long long>(sh.Bt) * sh.Hkv * sh.K * S;
    const size_t smem = decode_attn_smem_bytes(sh);
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(sh.d));
    const auto *qb = static_cast<const __nv_bfloat16 *>(q);
    const auto *kb = static_cast<const __nv_bfloat16 *>(k);
    const auto *vb = static_cast<const __nv_bfloat16 *>(v);
    if (sh.d == 128) {
        cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
        return launch_ex(decode_attn_kernel<128>, dim3(static_cast<unsigned>(grid)), dim3(128), smem, st,
                         pdl, qb, kb, vb, ids, part_o, part_lse, sh.T, sh.Hq, sh.Hkv, sh.block, sh.K,
                         S, sh.N, scale_log2, pm, status);
    } else {
        cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
        return launch_ex(decode_attn_kernel<64>, dim3(static_cast<unsigned>(grid)), dim3(128), smem, st,
                         pdl, qb, kb, vb, ids, part_o, part_lse, sh.T, sh.Hq, sh.Hkv, sh.block, sh.K,
                         S, sh.N, scale_log2, pm, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_combine(const Shape &sh, const void *part_o, bool part_bf16,
                           const float *part_lse, const int32_t *ids, float *out, float *lse,
                           int S, cudaStream_t st, bool pdl, int Hp, int h_off) {
    const long long rows = static_cast<long long>(sh.Bt) * sh.n_q;
    if (Hp <= 0) Hp = sh.Hq;
    if (rows * sh.Hq < 4096 && !part_bf16 && Hp == sh.Hq) {
        // few rows: split the partials of each (row, head) across the warps of a CTA
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const bool wide = rows * sh.Hq <= static_cast<long long>(sms) * 8;  // one wave of 8-warp CTAs
        const int nw = wide ? 8 : 4;
        const int P = sh.K * S;
        const size_t smem = (static_cast<size_t>((P + 3) & ~3) + static_cast<size_t>(nw) * sh.d) *
                            sizeof(float);
        const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(sh.Hq));
        const auto *po = static_cast<const float *>(part_o);
#define MSA_COMBINE_SPLIT(DD, NWW)                                                                \
    do {                                                                                          \
        cudaFuncSetAttribute(lse_combine_split_kernel<float, DD, NWW>,                            \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)); \
        return launch_ex(lse_combine_split_kernel<float, DD, NWW>, grid, dim3(32 * NWW), smem, st, \
                         pdl, po, part_lse, ids, out, lse, sh.Hq, sh.K, S, sh.N);                  \
    } while (0)
        if (sh.d == 128) {
            if (wide) MSA_COMBINE_SPLIT(128, 8);
            MSA_COMBINE_SPLIT(128, 4);
        }
        if (wide) MSA_COMBINE_SPLIT(64, 8);
        MSA_COMBINE_SPLIT(64, 4);
#undef MSA_COMBINE_SPLIT
    }
    // heads per CTA: all of them when there are many rows, else fewer so the
    // grid still covers the SMs a few times
    int HG = Hp;
    while (HG > 1 && HG % 2 == 0 && rows * (Hp / HG) < 1024) HG /= 2;
    const int vec = part_bf16 ? 8 : 4;
    int threads = HG * sh.d / vec;
    threads = threads > 256 ? 256 : ((threads + 31) / 32) * 32;
    const int P = sh.K * S;
    const size_t smem = static_cast<size_t>(P * HG + HG) * sizeof(float);
    const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(Hp / HG));
#define MSA_COMBINE(PT, DD)                                                                      \
    do {                                                                                         \
        cudaFuncSetAttribute(lse_combine_kernel<PT, DD>,                                         \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)); \
        e = launch_ex(lse_combine_kernel<PT, DD>, grid, dim3(threads), smem, st, pdl,             \
                      static_cast<const PT *>(part_o), part_lse, ids, out, lse, sh.Hq, sh.K, S,   \
                      HG, part_bf16 ? sh.G : 0, sh.N, Hp, h_off);                                 \
    } while (0)
    cudaError_t e = cudaSuccess;
    if (part_bf16) {
        if (sh.d == 128) MSA_COMBINE(__nv_bfloat16, 128); else MSA_COMBINE(__nv_bfloat16, 64);
    } else {
        if (sh.d == 128) MSA_COMBINE(float, 128); else MSA_COMBINE(float, 64);
    }
#undef MSA_COMBINE
    return e;
}

cudaError_t launch_invert(const Shape &sh, const int32_t *ids, int *chunk_counts,
                          int *pair_totals, int32_t *row_ptr, int32_t *entries, int *item_ptr,
                          AttnItem *items, int *counters, int rows_per_item, int n_chunks,
                          int *status, cudaStream_t st, int n_cursors, const OwnWork *own) {
    const int skip_own = own ? sh.block : 0;
    const size_t hist_bytes = static_cast<size_t>(4) * sh.N * sizeof(int);
    cudaFuncSetAttribute(inv_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(hist_bytes));
    cudaFuncSetAttribute(inv_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(hist_bytes));
    const dim3 cgrid(n_chunks, sh.Bt);
    inv_count_kernel<<<cgrid, 128, hist_bytes, st>>>(ids, chunk_counts, sh.n_q, sh.K, sh.N,
                                                      n_chunks, status, sh.T, skip_own);
    inv_colscan_kernel<<<dim3(sh.N, sh.Bt), 256, 0, st>>>(chunk_counts, pair_totals, sh.N,
                                                           n_chunks);
    const int n_pairs = sh.Bt * sh.N;
    inv_rowptr_kernel<<<1, 1024, 0, st>>>(pair_totals, row_ptr, item_ptr, counters, n_pairs,
                                          rows_per_item, n_cursors);
    inv_scatter_kernel<<<cgrid, 128, hist_bytes, st>>>(ids, chunk_counts, row_ptr, entries,
                                                        sh.n_q, sh.K, sh.N, n_chunks, status,
                                                        sh.T, skip_own);
    if (items)
        attn_items_kernel<<<(n_pairs + 255) / 256, 256, 0, st>>>(pair_totals, item_ptr, items,
                                                                  n_pairs, rows_per_item);
    if (own) {  // the own-block pass: items over each pair's own rows
        own_totals_kernel<<<(n_pairs + 255) / 256, 256, 0, st>>>(own->totals, sh.n_q, sh.T,
                                                                  sh.block, sh.N, n_pairs);
        inv_rowptr_kernel<<<1, 1024, 0, st>>>(own->totals, own->row_ptr, own->item_ptr,
                                              own->counters, n_pairs, rows_per_item, n_cursors);
        attn_items_kernel<<<(n_pairs + 255) / 256, 256, 0, st>>>(own->totals, own->item_ptr,
                                                                  own->items, n_pairs,
                                                                  rows_per_item);
    }
    return cudaGetLastError();
}

}  // namespace msa
