// Speculative commit: the accepted prefix of a verify pass back into the state pools.
//
// A pure copy, bound by HBM bandwidth.  For a request that accepted a >= 1 of
// its draft tokens, the checkpoints that the verify pass wrote after token a-1
// (the fp32 state of every value head, and the conv window) replace the
// request's pool slot; the pool then holds what an extend over the accepted
// tokens would have left.  The checkpoint layouts are the ones verify writes,
// so each copy is one contiguous span per (request, value head) and one per
// request for the conv window.

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kCommitThreads = 256;
constexpr int kVecPerThread = 4;  // 16-byte vectors in flight per thread

// n16 16-byte vectors from src to dst; each thread issues its loads before its stores
__device__ __forceinline__ void copy16(uint4* __restrict__ dst, const uint4* __restrict__ src, size_t n16) {
    for (size_t base = threadIdx.x; base < n16; base += (size_t)kCommitThreads * kVecPerThread) {
        uint4 v[kVecPerThread];
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
            const size_t e = base + (size_t)u * kCommitThreads;
            if (e < n16) v[u] = __ldcs(src + e);  // checkpoints are read once
        }
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
            const size_t e = base + (size_t)u * kCommitThreads;
            if (e < n16) dst[e] = v[u];
        }
    }
}

// grid (B, HV + 1): block (i, h < HV) copies value head h's state of request i, block (i, HV) its
// conv window
__global__ void __launch_bounds__(kCommitThreads) commit_kernel(CommitArgs p) {
    const int i = blockIdx.x, h = blockIdx.y;
    const int slot = p.slots[i], acc = p.accepted[i];
    if (slot < 0) return;  // padding
    if (slot >= p.P) {
        if (h == 0 && threadIdx.x == 0) raise_error(p.hdr, GDN_DEVERR_SLOT_RANGE);
        return;
    }
    if (acc < 0 || acc > p.D) {
        if (h == 0 && threadIdx.x == 0) raise_error(p.hdr, GDN_DEVERR_ACCEPT_RANGE);
        return;
    }
    if (acc == 0) return;  // nothing accepted: the slot keeps the state verify started from
    const size_t ck = (size_t)i * p.D + (acc - 1);  // checkpoint after the last accepted token
    if (h < p.d.HV) {
        const size_t n = (size_t)p.d.dk * p.d.dv;  // floats of one head's state
        copy16(reinterpret_cast<uint4*>(p.ssm_state + ((size_t)slot * p.d.HV + h) * n),
               reinterpret_cast<const uint4*>(p.state_ckpt + (ck * p.d.HV + h) * n), n / 4);
    } else if (p.conv_ckpt) {
        const size_t bytes = (size_t)p.d.conv_dim * (kConvK - 1) * p.conv_elem;  // a multiple of 16
        copy16(reinterpret_cast<uint4*>(static_cast<char*>(p.conv_state) + (size_t)slot * bytes),
               reinterpret_cast<const uint4*>(static_cast<const char*>(p.conv_ckpt) + ck * bytes), bytes / 16);
    }
}

}  // namespace

cudaError_t launch_commit(const CommitArgs& p, cudaStream_t s) {
    mark_launch(s, 0);
    commit_kernel<<<dim3(p.B, p.d.HV + 1), kCommitThreads, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    mark_launch(s, 1);
    return e;
}

}  // namespace gdn
