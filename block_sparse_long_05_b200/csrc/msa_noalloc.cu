// msa_noalloc.cu -- decode attention for callers that cannot allocate device
// memory.  It runs the same split-K decode attention and log-sum-exp combine
// kernels as msa_sparse_attn with n_q == 1, but takes its scratch (the per
// split partials) from a file-scope static __device__ array instead of a
// caller-provided workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/msa.h"
#include "kernels.h"
#include "msa_common.cuh"

using namespace msa;

namespace {

constexpr size_t kScratchBytes = MSA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch.  Its first 256 bytes hold a status word (used when the caller
// passes no status pointer); the partials follow.  In host code this name is
// only a host-side stand-in: the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, resolved once per
// device (the first call on a device does it).
msa_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MSA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MSA_OK;
}

}  // namespace

extern "C" {

msa_status msa_sparse_attn_decode_noalloc(const void *q, const void *k, const void *v,
                                          const int32_t *ids, float *out, float *lse, int Bt,
                                          int T, int Hq, int Hkv, int d, int block, int K,
                                          int *status, void *stream) {
    if (!q || !k || !v || !ids || !out || !lse) return MSA_ERR_INVALID_ARG;
    if (Bt < 1 || T < 1 || Hq < 1 || Hkv < 1 || d < 1 || block < 1 || K < 1 || Hq % Hkv != 0)
        return MSA_ERR_INVALID_ARG;
    if (K > kMaxK || !(d == 64 || d == 128) || !(block == 32 || block == 64 || block % 128 == 0) ||
        128 % (Hq / Hkv) != 0 || static_cast<long long>(Bt) * T >= (1ll << 31))
        return MSA_ERR_UNSUPPORTED;
    // q, k, v are read and out is written with 16-byte accesses; ids and lse
    // as 4-byte words
    const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
    if ((mis & 15) || ((reinterpret_cast<uintptr_t>(ids) | reinterpret_cast<uintptr_t>(lse)) & 3))
        return MSA_ERR_INVALID_ARG;

    Shape sh;
    sh.Bt = Bt;
    sh.n_q = 1;
    sh.T = T;
    sh.Hq = Hq;
    sh.Hkv = Hkv;
    sh.d = d;
    sh.d_idx = 64;
    sh.block = block;
    sh.K = K;
    sh.N = static_cast<int>((static_cast<long long>(T) + block - 1) / block);
    sh.G = Hq / Hkv;

    // Scratch needed: a 256-byte status word, fp32 partials
    // [Bt][K][S][Hq][d] and their lse [Bt][K][S][Hq].
    const int S = (block + kDecodeKeys - 1) / kDecodeKeys;
    const size_t prow = static_cast<size_t>(Bt) * K * S;
    const size_t o_bytes = align_up(prow * Hq * d * 4, 256);
    const size_t l_bytes = align_up(prow * Hq * 4, 256);
    if (256 + o_bytes + l_bytes > kScratchBytes) return MSA_ERR_WORKSPACE;

    void *base = nullptr;
    msa_status s = scratch_address(&base);
    if (s != MSA_OK) return s;
    unsigned char *b = static_cast<unsigned char *>(base);
    float *part_o = reinterpret_cast<float *>(b + 256);
    float *part_lse = reinterpret_cast<float *>(b + 256 + o_bytes);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *dev_status = status;
    if (!dev_status) {
        // the internal status word keeps the last call's value: clear it
        dev_status = reinterpret_cast<int *>(b);
        if (cudaMemsetAsync(dev_status, 0, sizeof(int), st) != cudaSuccess) return MSA_ERR_CUDA;
    }
    if (launch_decode_attn(sh, q, k, v, ids, part_o, part_lse, S, PageMap{}, dev_status, st, false) !=
        cudaSuccess)
        return MSA_ERR_CUDA;
    if (launch_combine(sh, part_o, false, part_lse, ids, out, lse, S, st, true) != cudaSuccess)
        return MSA_ERR_CUDA;
    return MSA_OK;
}

}  // extern "C"
