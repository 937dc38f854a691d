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

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
    uint32_t lo = static_cast<uint32_t>(v), hi = static_cast<uint32_t>(v >> 32);
    lo = __shfl_xor_sync(0xFFFFFFFFu, lo, m);
    hi = __shfl_xor_sync(0xFFFFFFFFu, hi, m);
    return (static_cast<uint64_t>(hi) << 32) | lo;
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

template <int D_IDX>
__global__ void __launch_bounds__(256) decode_index_scan_kernel(
    const __nv_bfloat16 *__restrict__ q_idx, const __nv_bfloat16 *__restrict__ k_idx,
    float *__restrict__ block_scores, int T, int block, int own, int N) {
    constexpr int LPR = D_IDX / 8;  // lanes per key row
    constexpr int RPL = 32 / LPR;   // key rows per warp load
    constexpr int UNR = 16;         // loads in flight per warp
    __shared__ float wmax[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / LPR, part = lane % LPR;
    const int b = blockIdx.x / own, j = blockIdx.x % own;
    float qv[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4 *>(q_idx + static_cast<long long>(b) * D_IDX + part * 8), qv);
    const uint4 *base = reinterpret_cast<const uint4 *>(
        k_idx + (static_cast<long long>(b) * T + static_cast<long long>(j) * block) * D_IDX);
    // rows of this warp: r = (warp + 8 * it) * RPL + sub
    const int groups = block / RPL;  // row groups of RPL rows
    float best = -FLT_MAX;
    for (int g0 = warp; g0 < groups; g0 += 8 * UNR) {
        uint4 ku[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int gi = g0 + 8 * u;
            ku[u] = gi < groups ? ld_stream16(base + (gi * RPL + sub) * LPR + part) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            float kf[8];
            bf16x8_to_f32(ku[u], kf);
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(qv[e], kf[e], s);
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
            if (g0 + 8 * u < groups) best = fmaxf(best, s);
        }
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) best = fmaxf(best, __shfl_xor_sync(0xFFFFFFFFu, best, o));
    if (lane == 0) wmax[warp] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = wmax[0];
        for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
        block_scores[static_cast<long long>(b) * N + j] = m;
    }
}

// ------------------------------------------------------------------------
// Decode select: one CTA of 1024 threads per sequence.  Each thread keeps the
// best of its strided candidates (key = score desc, block asc, packed in 64
// bits); min(K, own+1)-1 rounds of block arg-max pick the winners (the owner
// of a winner advances to its next best); own is added, ids written ascending.
// ------------------------------------------------------------------------
constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(kSelThreads) decode_select_kernel(
    const float *__restrict__ block_scores, int32_t *__restrict__ ids, int N, int own, int K) {
    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ uint64_t wbest[32];
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
    for (int p = 0; p < m; ++p) {
        uint64_t best = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) best = mine[q] > best ? mine[q] : best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t other = shfl_xor_u64(best, o);
            best = other > best ? other : best;
        }
        if (lane == 0) wbest[warp] = best;
        __syncthreads();
        if (warp == 0) {
            uint64_t v = wbest[lane];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const uint64_t other = shfl_xor_u64(v, o);
                v = other > v ? other : v;
            }
            if (lane == 0) wbest[0] = v;
        }
        __syncthreads();
        const uint64_t win = wbest[0];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (mine[q] == win) mine[q] = 0;  // keys are unique: one owner
        if (tid == 0) sel[p] = 0x7FFFFFFF - static_cast<int>(static_cast<uint32_t>(win));
        __syncthreads();
    }
    (void)nm;
    if (tid == 0) {
        sel[m] = own;
        const int n = m + 1;
        for (int a = 1; a < n; ++a) {  // insertion sort, ascending
            const int x = sel[a];
            int c = a - 1;
            while (c >= 0 && sel[c] > x) {
                sel[c + 1] = sel[c];
                --c;
            }
            sel[c + 1] = x;
        }
        for (int s = 0; s < K; ++s) ids[static_cast<long long>(b) * K + s] = s < n ? sel[s] : -1;
    }
}

// ------------------------------------------------------------------------
// Split-K decode attention.  One CTA of 128 threads per (b, kv head, slot,
// split of kDecodeKeys keys).  K/V rows are staged in shared memory by
// 16-byte cp.async (coalesced 2*d-byte rows); the G query heads share them.
// Scores: thread (key = tid/2, half = tid%2) holds its half K row in
// registers and reads q (pre-scaled, fp32) as broadcast float4; the two
// halves are summed by a shuffle.  Softmax in the log2 domain, one warp per
// head.  PV: thread per output column (and key half when d = 64), p read as
// float4 over heads.  Writes a normalised fp32 partial and its natural-log
// lse (-inf when the split has no key).
// ------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) decode_attn_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, const int32_t *__restrict__ ids,
    float *__restrict__ part_o, float *__restrict__ part_lse, int T, int Hq, int Hkv, int block,
    int K, int S, int N, float scale_log2, int *__restrict__ status) {
    constexpr int KS = kDecodeKeys;
    constexpr int KSTR = D + 8;       // padded K row (bf16) to spread banks
    constexpr int HALF = D / 2;       // elements of a half row
    constexpr int NH = 128 / D;       // key halves in the PV phase
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int G = Hq / Hkv;
    const int GP = (G + 3) & ~3;      // heads padded to a float4
    float *qs = reinterpret_cast<float *>(smem_raw);   // [G][D]
    float *ps = qs + G * D;                             // [KS][GP]
    float *ms = ps + KS * GP;                           // [G]
    float *ls = ms + G;                                 // [G]
    float *red = ls + G;                                // [NH-1][G][D] (d = 64 only)
    __nv_bfloat16 *Ks = reinterpret_cast<__nv_bfloat16 *>(
        (reinterpret_cast<uintptr_t>(red + (NH - 1) * G * D) + 15) & ~static_cast<uintptr_t>(15));
    __nv_bfloat16 *Vs = Ks + KS * KSTR;                 // [KS][D]

    const int tid = threadIdx.x;
    int idx = blockIdx.x;
    const int sp = idx % S;
    idx /= S;
    const int s = idx % K;
    idx /= K;
    const int hk = idx % Hkv;
    const int b = idx / Hkv;
    const long long prow = (static_cast<long long>(b) * K + s) * S + sp;  // partial row
    const int t = T - 1;
    const int j = ids[static_cast<long long>(b) * K + s];
    int nk = 0;
    long long k0 = 0;
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
    }
    if (nk == 0) {
        for (int g = tid; g < G; g += blockDim.x) part_lse[prow * Hq + hk * G + g] = -INFINITY;
        return;
    }
    constexpr int PIECES = D / 8;  // 16-byte pieces per row
    const __nv_bfloat16 *kbase = k + ((static_cast<long long>(b) * T + k0) * Hkv + hk) * D;
    const __nv_bfloat16 *vbase = v + ((static_cast<long long>(b) * T + k0) * Hkv + hk) * D;
    for (int e = tid; e < nk * PIECES; e += blockDim.x) {
        const int r = e / PIECES, c = e % PIECES;
        const long long goff = static_cast<long long>(r) * Hkv * D + c * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(Ks + r * KSTR + c * 8))),
                     "l"(kbase + goff)
                     : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(Vs + r * D + c * 8))),
                     "l"(vbase + goff)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const __nv_bfloat16 *qrow = q + (static_cast<long long>(b) * Hq + hk * G) * D;
    for (int e = tid; e < G * D; e += blockDim.x) qs[e] = __bfloat162float(qrow[e]) * scale_log2;
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    // ---- scores: ps[key][g] (log2 domain)
    {
        const int key = tid >> 1, half = tid & 1;
        const bool kv_ok = key < nk;
        uint4 kr[HALF / 8];
#pragma unroll
        for (int c = 0; c < HALF / 8; ++c)
            kr[c] = kv_ok ? *reinterpret_cast<const uint4 *>(Ks + key * KSTR + half * HALF + c * 8)
                          : make_uint4(0, 0, 0, 0);
        for (int g0 = 0; g0 < G; g0 += 8) {
            float acc[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = 0.f;
#pragma unroll
            for (int c = 0; c < HALF / 8; ++c) {
                float kf[8];
                bf16x8_to_f32(kr[c], kf);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    if (g0 + x < G) {
                        const float4 *qp = reinterpret_cast<const float4 *>(qs + (g0 + x) * D + half * HALF + c * 8);
                        const float4 qa = qp[0], qb = qp[1];
                        acc[x] = fmaf(qa.x, kf[0], acc[x]);
                        acc[x] = fmaf(qa.y, kf[1], acc[x]);
                        acc[x] = fmaf(qa.z, kf[2], acc[x]);
                        acc[x] = fmaf(qa.w, kf[3], acc[x]);
                        acc[x] = fmaf(qb.x, kf[4], acc[x]);
                        acc[x] = fmaf(qb.y, kf[5], acc[x]);
                        acc[x] = fmaf(qb.z, kf[6], acc[x]);
                        acc[x] = fmaf(qb.w, kf[7], acc[x]);
                    }
                }
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] += __shfl_xor_sync(0xFFFFFFFFu, acc[x], 1);
            if (half == 0) {
#pragma unroll
                for (int x = 0; x < 8; ++x)
                    if (g0 + x < G) ps[key * GP + g0 + x] = kv_ok ? acc[x] : -INFINITY;
            }
        }
    }
    __syncthreads();
    // ---- per-head max and sum (one warp per head), p in place
    const int warp = tid / 32, lane = tid % 32;
    for (int g = warp; g < G; g += blockDim.x / 32) {
        float mx = -INFINITY;
        for (int key = lane; key < nk; key += 32) mx = fmaxf(mx, ps[key * GP + g]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        float sum = 0.f;
        for (int key = lane; key < KS; key += 32) {
            const float pv = key < nk ? exp2f(ps[key * GP + g] - mx) : 0.f;
            ps[key * GP + g] = pv;
            sum += pv;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (lane == 0) {
            ms[g] = mx;
            ls[g] = sum;
        }
    }
    __syncthreads();
    // ---- out[g][c] = sum_key p[key][g] * V[key][c] / l[g]
    {
        const int c = tid % D, kh = tid / D;  // column, key half (NH halves)
        const int kb = kh * (KS / NH), ke = min(nk, kb + KS / NH);
        for (int g0 = 0; g0 < G; g0 += 8) {
            float acc[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = 0.f;
            for (int key = kb; key < ke; ++key) {
                const float vv = __bfloat162float(Vs[key * D + c]);
                const float4 pa = *reinterpret_cast<const float4 *>(ps + key * GP + g0);
                acc[0] = fmaf(pa.x, vv, acc[0]);
                acc[1] = fmaf(pa.y, vv, acc[1]);
                acc[2] = fmaf(pa.z, vv, acc[2]);
                acc[3] = fmaf(pa.w, vv, acc[3]);
                if (g0 + 4 < GP) {
                    const float4 pb = *reinterpret_cast<const float4 *>(ps + key * GP + g0 + 4);
                    acc[4] = fmaf(pb.x, vv, acc[4]);
                    acc[5] = fmaf(pb.y, vv, acc[5]);
                    acc[6] = fmaf(pb.z, vv, acc[6]);
                    acc[7] = fmaf(pb.w, vv, acc[7]);
                }
            }
            if (NH > 1 && kh > 0) {
#pragma unroll
                for (int x = 0; x < 8; ++x)
                    if (g0 + x < G) red[((kh - 1) * G + g0 + x) * D + c] = acc[x];
            }
            if (NH > 1) __syncthreads();
            if (kh == 0) {
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const int g = g0 + x;
                    if (g < G) {
                        float a = acc[x];
                        for (int h2 = 1; h2 < NH; ++h2) a += red[((h2 - 1) * G + g) * D + c];
                        part_o[(prow * Hq + hk * G + g) * D + c] = a / ls[g];
                    }
                }
            }
            if (NH > 1) __syncthreads();
        }
    }
    for (int g = tid; g < G; g += blockDim.x)
        part_lse[prow * Hq + hk * G + g] = (ms[g] + log2f(ls[g])) * kLn2;
}

// ------------------------------------------------------------------------
// Log-sum-exp combine.  One CTA per (query row, group of HG heads).  The P =
// K*S partials of each head are merged as LSE = log sum_p exp(lse_p) and
// out = sum_p exp(lse_p - LSE) o_p.  Weights are computed once into shared
// memory; the partial rows are then streamed with 16-byte loads (several in
// flight per thread).  Partial p = (slot s, split sp) is valid when
// ids[row][s] >= 0 and its lse is finite; invalid partials are never used
// (their memory may hold a previous call's data).
// ------------------------------------------------------------------------
template <typename PT, int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(
    const PT *__restrict__ part_o, const float *__restrict__ part_lse,
    const int32_t *__restrict__ ids, float *__restrict__ out, float *__restrict__ lse_out, int Hq,
    int K, int S, int HG) {
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
        if (ids[row * K + s] >= 0) l = part_lse[((row * K + s) * S + pp % S) * Hq + h0 + hh];
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
        lse_out[row * Hq + h0 + hh] = L;
    }
    __syncthreads();
    for (int e = tid; e < HG * NV; e += blockDim.x) {
        const int hh = e / NV, c = (e % NV) * VEC;
        float acc[VEC];
#pragma unroll
        for (int x = 0; x < VEC; ++x) acc[x] = 0.f;
        const PT *src = part_o + ((row * K) * S * Hq + h0 + hh) * static_cast<long long>(D) + c;
        const long long pstride = static_cast<long long>(Hq) * D;  // between consecutive partials
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
        float *dst = out + (row * Hq + h0 + hh) * static_cast<long long>(D) + c;
#pragma unroll
        for (int x = 0; x < VEC; x += 4)
            *reinterpret_cast<float4 *>(dst + x) = make_float4(acc[x], acc[x + 1], acc[x + 2], acc[x + 3]);
    }
}

// Few query rows (decode): one CTA of 8 warps per (row, head); warp w merges
// partials p = w, w+8, ... of that head and the warps' sums are added in
// shared memory.  Same arithmetic as lse_combine_kernel.
template <typename PT, int D>
__global__ void __launch_bounds__(256) lse_combine_split_kernel(
    const PT *__restrict__ part_o, const float *__restrict__ part_lse,
    const int32_t *__restrict__ ids, float *__restrict__ out, float *__restrict__ lse_out, int Hq,
    int K, int S) {
    constexpr int PER = D / 32;  // elements per lane
    extern __shared__ float wsm[];                // [P] weights, then [8][D] sums
    const long long row = blockIdx.x;
    const int h = blockIdx.y;
    const int P = K * S;
    float *acc_s = wsm + ((P + 3) & ~3);
    __shared__ float L_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int pp = tid; pp < P; pp += blockDim.x) {
        const int si = pp / S;
        float l = -INFINITY;
        if (ids[row * K + si] >= 0) l = part_lse[((row * K + si) * S + pp % S) * Hq + h];
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
    for (int pp = warp; pp < P; pp += 8) {
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
        for (int w = 0; w < 8; ++w) a += acc_s[w * D + c];
        out[(row * Hq + h) * static_cast<long long>(D) + c] = a;
    }
    if (tid == 0) lse_out[row * Hq + h] = L_s;
}

// ------------------------------------------------------------------------
// Inversion.  Chunks of kInvRows query rows; warp w of a chunk owns rows
// [32w, 32w+32).  Per-warp histograms live in shared memory [4][N].
// ------------------------------------------------------------------------
__device__ __forceinline__ void warp_histogram(const int32_t *__restrict__ ids, int *hist_w,
                                               int b, int n_q, int K, int N, int row0,
                                               int *status) {
    const int lane = threadIdx.x % 32;
    const int i = row0 + lane;
    if (i < n_q) {
        const int32_t *r = ids + (static_cast<long long>(b) * n_q + i) * K;
        for (int s = 0; s < K; ++s) {
            const int j = r[s];
            if (j >= 0 && j < N)
                atomicAdd(hist_w + j, 1);
            else if (j != -1 && status)
                atomicOr(status, kDevBadIds);
        }
    }
}

__global__ void __launch_bounds__(128) inv_count_kernel(const int32_t *__restrict__ ids,
                                                         int *__restrict__ chunk_counts, int n_q,
                                                         int K, int N, int n_chunks,
                                                         int *__restrict__ status) {
    extern __shared__ int hist[];  // [4][N]
    const int chunk = blockIdx.x, b = blockIdx.y;
    for (int e = threadIdx.x; e < 4 * N; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int w = threadIdx.x / 32;
    warp_histogram(ids, hist + w * N, b, n_q, K, N, chunk * kInvRows + 32 * w, status);
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
// ceil(total / rows_per_item) (when items != nullptr); counters[0] = items,
// counters[1] = 0 (work cursor of the attention kernel).
__global__ void __launch_bounds__(1024) inv_rowptr_kernel(const int *__restrict__ pair_totals,
                                                           int *__restrict__ row_ptr,
                                                           int *__restrict__ item_ptr,
                                                           int *__restrict__ counters, int n_pairs,
                                                           int rows_per_item) {
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
            counters[0] = tb;
            counters[1] = 0;
        }
    }
}

__global__ void __launch_bounds__(128) inv_scatter_kernel(
    const int32_t *__restrict__ ids, const int *__restrict__ chunk_prefix,
    const int *__restrict__ row_ptr, int32_t *__restrict__ entries, int n_q, int K, int N,
    int n_chunks, int *__restrict__ status) {
    extern __shared__ int hist[];  // [4][N] counts, then cursors
    const int chunk = blockIdx.x, b = blockIdx.y;
    for (int e = threadIdx.x; e < 4 * N; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
    // bad ids were already reported by the count pass
    warp_histogram(ids, hist + w * N, b, n_q, K, N, chunk * kInvRows + 32 * w, nullptr);
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
        if (lane < K) {
            const int j = ids[row * K + lane];
            if (j >= 0 && j < N) {
                const int pos = atomicAdd(cursor + j, 1);
                entries[pos] = static_cast<int32_t>(row * K + lane);
            }
        }
        __syncwarp();
    }
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
cudaError_t launch_decode_scan(const Shape &sh, const void *q_idx, const void *k_idx,
                               float *block_scores, int num_sms, cudaStream_t st) {
    (void)num_sms;
    const int own = (sh.T - 1) / sh.block;
    if (own > 0) {
        const long long grid = static_cast<long long>(sh.Bt) * own;
        const auto *qi = static_cast<const __nv_bfloat16 *>(q_idx);
        const auto *ki = static_cast<const __nv_bfloat16 *>(k_idx);
        if (sh.d_idx == 128)
            decode_index_scan_kernel<128><<<static_cast<unsigned>(grid), 256, 0, st>>>(
                qi, ki, block_scores, sh.T, sh.block, own, sh.N);
        else
            decode_index_scan_kernel<64><<<static_cast<unsigned>(grid), 256, 0, st>>>(
                qi, ki, block_scores, sh.T, sh.block, own, sh.N);
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_select(const Shape &sh, const float *block_scores, int32_t *ids,
                                 cudaStream_t st) {
    const int own = (sh.T - 1) / sh.block;
    decode_select_kernel<<<sh.Bt, kSelThreads, 0, st>>>(block_scores, ids, sh.N, own, sh.K);
    return cudaGetLastError();
}

size_t decode_attn_smem_bytes(const Shape &sh) {
    const int G = sh.G;
    const int GP = (G + 3) & ~3;
    const int NH = 128 / sh.d;
    size_t f = static_cast<size_t>(G) * sh.d + static_cast<size_t>(kDecodeKeys) * GP + 2 * G +
               static_cast<size_t>(NH - 1) * G * sh.d;
    size_t bytes = align_up(f * 4, 16);
    bytes += static_cast<size_t>(kDecodeKeys) * (sh.d + 8) * 2 + static_cast<size_t>(kDecodeKeys) * sh.d * 2;
    return bytes;
}

cudaError_t launch_decode_attn(const Shape &sh, const void *q, const void *k, const void *v,
                               const int32_t *ids, float *part_o, float *part_lse, int S,
                               int *status, cudaStream_t st) {
    const long long grid = static_cast<long long>(sh.Bt) * sh.Hkv * sh.K * S;
    const size_t smem = decode_attn_smem_bytes(sh);
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(sh.d));
    const auto *qb = static_cast<const __nv_bfloat16 *>(q);
    const auto *kb = static_cast<const __nv_bfloat16 *>(k);
    const auto *vb = static_cast<const __nv_bfloat16 *>(v);
    if (sh.d == 128) {
        cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
        decode_attn_kernel<128><<<static_cast<unsigned>(grid), 128, smem, st>>>(
            qb, kb, vb, ids, part_o, part_lse, sh.T, sh.Hq, sh.Hkv, sh.block, sh.K, S, sh.N,
            scale_log2, status);
    } else {
        cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
        decode_attn_kernel<64><<<static_cast<unsigned>(grid), 128, smem, st>>>(
            qb, kb, vb, ids, part_o, part_lse, sh.T, sh.Hq, sh.Hkv, sh.block, sh.K, S, sh.N,
            scale_log2, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_combine(const Shape &sh, const void *part_o, bool part_bf16,
                           const float *part_lse, const int32_t *ids, float *out, float *lse,
                           int S, cudaStream_t st) {
    const long long rows = static_cast<long long>(sh.Bt) * sh.n_q;
    if (rows * sh.Hq < 4096 && !part_bf16) {
        // few rows: split the partials of each (row, head) across 8 warps
        const int P = sh.K * S;
        const size_t smem = (static_cast<size_t>((P + 3) & ~3) + 8 * sh.d) * sizeof(float);
        const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(sh.Hq));
        const auto *po = static_cast<const float *>(part_o);
        if (sh.d == 128) {
            cudaFuncSetAttribute(lse_combine_split_kernel<float, 128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            lse_combine_split_kernel<float, 128><<<grid, 256, smem, st>>>(po, part_lse, ids, out,
                                                                         lse, sh.Hq, sh.K, S);
        } else {
            cudaFuncSetAttribute(lse_combine_split_kernel<float, 64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            lse_combine_split_kernel<float, 64><<<grid, 256, smem, st>>>(po, part_lse, ids, out,
                                                                        lse, sh.Hq, sh.K, S);
        }
        return cudaGetLastError();
    }
    // heads per CTA: all of them when there are many rows, else fewer so the
    // grid still covers the SMs a few times
    int HG = sh.Hq;
    while (HG > 1 && HG % 2 == 0 && rows * (sh.Hq / HG) < 1024) HG /= 2;
    const int vec = part_bf16 ? 8 : 4;
    int threads = HG * sh.d / vec;
    threads = threads > 256 ? 256 : ((threads + 31) / 32) * 32;
    const int P = sh.K * S;
    const size_t smem = static_cast<size_t>(P * HG + HG) * sizeof(float);
    const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(sh.Hq / HG));
#define MSA_COMBINE(PT, DD)                                                                      \
    do {                                                                                         \
        cudaFuncSetAttribute(lse_combine_kernel<PT, DD>,                                         \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)); \
        lse_combine_kernel<PT, DD><<<grid, threads, smem, st>>>(                                 \
            static_cast<const PT *>(part_o), part_lse, ids, out, lse, sh.Hq, sh.K, S, HG);       \
    } while (0)
    if (part_bf16) {
        if (sh.d == 128) MSA_COMBINE(__nv_bfloat16, 128); else MSA_COMBINE(__nv_bfloat16, 64);
    } else {
        if (sh.d == 128) MSA_COMBINE(float, 128); else MSA_COMBINE(float, 64);
    }
#undef MSA_COMBINE
    return cudaGetLastError();
}

cudaError_t launch_invert(const Shape &sh, const int32_t *ids, int *chunk_counts,
                          int *pair_totals, int32_t *row_ptr, int32_t *entries, int *item_ptr,
                          AttnItem *items, int *counters, int rows_per_item, int n_chunks,
                          int *status, cudaStream_t st) {
    const size_t hist_bytes = static_cast<size_t>(4) * sh.N * sizeof(int);
    cudaFuncSetAttribute(inv_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(hist_bytes));
    cudaFuncSetAttribute(inv_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(hist_bytes));
    const dim3 cgrid(n_chunks, sh.Bt);
    inv_count_kernel<<<cgrid, 128, hist_bytes, st>>>(ids, chunk_counts, sh.n_q, sh.K, sh.N,
                                                      n_chunks, status);
    inv_colscan_kernel<<<dim3(sh.N, sh.Bt), 256, 0, st>>>(chunk_counts, pair_totals, sh.N,
                                                           n_chunks);
    const int n_pairs = sh.Bt * sh.N;
    inv_rowptr_kernel<<<1, 1024, 0, st>>>(pair_totals, row_ptr, item_ptr, counters, n_pairs,
                                          rows_per_item);
    inv_scatter_kernel<<<cgrid, 128, hist_bytes, st>>>(ids, chunk_counts, row_ptr, entries,
                                                        sh.n_q, sh.K, sh.N, n_chunks, status);
    if (items)
        attn_items_kernel<<<(n_pairs + 255) / 256, 256, 0, st>>>(pair_totals, item_ptr, items,
                                                                  n_pairs, rows_per_item);
    return cudaGetLastError();
}

}  // namespace msa
