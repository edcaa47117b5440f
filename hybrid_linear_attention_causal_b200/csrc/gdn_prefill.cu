// EXTEND (chunked prefill) kernels of the GDN layer (sm_100a).
//
// Chunked WY / UT form of the gated delta rule, chunk length C = 64.  Inside a
// chunk of n rows that starts from state S0, with gamma_r = sum_{s<=r} g_s:
//   A[r,s] = beta_r e^{gamma_r - gamma_s} (k_r . k_s)  for s < r
//   (I + A) [W | U] = [diag(beta e^gamma) K | diag(beta) V]     (forward substitution)
//   V'    = U - W S0                                   (the per-row delta values)
//   o_r   = e^{gamma_r} q_r^T S0 + sum_{s<=r} e^{gamma_r - gamma_s} (q_r . k_s) V'_s
//   S_end = e^{gamma_n} S0 + sum_s e^{gamma_n - gamma_s} k_s V'_s^T
// (q carries the output scale).  Decay factors are always formed from
// differences of gamma inside one chunk, so they never overflow.
//
// Launch sequence (all stream-ordered, no host synchronisation):
//   1. chunk_map:  validates cu_seqlens and lays out the chunk table
//   2. prep:       conv1d + SiLU, L2 norm, gates -> fp32 q, k, v, (g, beta)
//   3. conv_tail:  writes each sequence's new conv window into its slot
//   4. intra:      per (chunk, qk head) on tensor cores: gamma, A, T, W, U and
//                  the masked decayed q.k of each value head (gdn_intra_tc.cu)
//   5. state:      per (sequence, value head) on tensor cores: the serial chunk
//                  pass V' = U - W S, the outputs and S <- e^{gamma_n} S + K~^T V'
//                  (gdn_state_tc.cu)
// Every intermediate is fp32 and every tensor-core operand is rounded to tf32
// (round to nearest): the parity bar leaves no room for bf16 rounding of q, k,
// v, W, U or V', and truncating to tf32 instead of rounding fails it too.

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;

// ---------------------------------------------------------------- 1. chunk map

__global__ void __launch_bounds__(1024) chunk_map_kernel(ExtendArgs p) {
    __shared__ int s_bad;
    __shared__ int s_scan[1024];
    __shared__ int s_base;
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_bad = (p.cu[0] != 0 || p.cu[p.N] != p.T) ? 1 : 0;
        s_base = 0;
    }
    __syncthreads();
    for (int n = tid; n < p.N; n += 1024)
        if (p.cu[n + 1] < p.cu[n]) atomicOr(&s_bad, 1);
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            raise_error(p.hdr, GDN_DEVERR_SEQLENS);
            p.hdr[kHdrNumChunks] = 0;
        }
        return;
    }
    for (int base = 0; base < p.N; base += 1024) {
        const int n = base + tid;
        int nc = 0;
        if (n < p.N) nc = (p.cu[n + 1] - p.cu[n] + C - 1) / C;
        s_scan[tid] = nc;
        __syncthreads();
        for (int off = 1; off < 1024; off <<= 1) {
            const int v = tid >= off ? s_scan[tid - off] : 0;
            __syncthreads();
            s_scan[tid] += v;
            __syncthreads();
        }
        if (n < p.N) p.seq_chunk0[n] = s_base + s_scan[tid] - nc;
        __syncthreads();
        if (tid == 1023) s_base += s_scan[1023];
        __syncthreads();
    }
    if (tid == 0) {
        p.seq_chunk0[p.N] = s_base;
        p.hdr[kHdrNumChunks] = s_base;
    }
    __threadfence_block();
    __syncthreads();
    const int total = s_base;
    for (int id = tid; id < total; id += 1024) {
        int lo = 0, hi = p.N - 1;  // last sequence whose first chunk id <= id
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.seq_chunk0[mid] <= id) lo = mid; else hi = mid - 1;
        }
        const int c = id - p.seq_chunk0[lo];
        const int len = p.cu[lo + 1] - p.cu[lo];
        p.chunk_tab[id] = make_int4(lo, p.cu[lo] + c * C, min(C, len - c * C), c);
    }
}

// ---------------------------------------------------------------- 2. prep

__device__ __forceinline__ int seq_of_row(const int32_t* cu, int N, int t) {
    int lo = 0, hi = N - 1;  // last n with cu[n] <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// One CTA per packed row.  Warps take whole heads: the 2*HK q/k heads are
// normalised with a warp reduction, the HV value heads are stored as is.
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256) prep_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    const LayerDims& d = p.d;
    const int t = blockIdx.x, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n = seq_of_row(p.cu, p.N, t);
    const int slot = p.slots[n];
    if (slot < 0 || slot >= p.P) return;
    const int pos = t - p.cu[n];
    const bool init = p.has_init ? p.has_init[n] != 0 : true;
    const T* x = reinterpret_cast<const T*>(p.x);
    const T* w = reinterpret_cast<const T*>(p.conv_w);
    const T* bias = reinterpret_cast<const T*>(p.conv_b);
    const T* cs = reinterpret_cast<const T*>(p.conv_state) + (size_t)slot * d.conv_dim * 3;

    auto conv = [&](int c) -> float {
        float acc = bias ? to_f(bias[c]) : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int src = pos - 3 + j;
            float xv;
            if (src >= 0) xv = to_f(x[(size_t)(t - 3 + j) * d.conv_dim + c]);
            else xv = init ? to_f(cs[c * 3 + 3 + src]) : 0.f;
            acc = fmaf(to_f(w[c * 4 + j]), xv, acc);
        }
        return silu_f(acc);
    };

    const int units = 2 * d.HK + d.HV;
    for (int u = warp; u < units; u += 8) {
        if (u < 2 * d.HK) {
            const bool isq = u < d.HK;
            const int hk = isq ? u : u - d.HK;
            const int c0 = isq ? hk * DK : d.HK * DK + hk * DK;
            float vals[DK / 32];
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < DK / 32; ++i) {
                vals[i] = conv(c0 + lane * (DK / 32) + i);
                ss += vals[i] * vals[i];
            }
            ss = warp_sum(ss);
            const float r = rsqrtf(ss + d.eps) * (isq ? d.scale : 1.0f);
            float* dst = (isq ? p.qn : p.kn) + ((size_t)t * d.HK + hk) * DK + lane * (DK / 32);
#pragma unroll
            for (int i = 0; i < DK / 32; ++i) dst[i] = vals[i] * r;
        } else {
            const int h = u - 2 * d.HK;
            const int c0 = 2 * d.HK * DK + h * DV;
            float* dst = p.vv + ((size_t)t * d.HV + h) * DV + lane * (DV / 32);
#pragma unroll
            for (int i = 0; i < DV / 32; ++i) dst[i] = conv(c0 + lane * (DV / 32) + i);
        }
    }
    for (int h = threadIdx.x; h < d.HV; h += 256) {
        const float av = to_f(reinterpret_cast<const T*>(p.a)[(size_t)t * d.HV + h]);
        const float bv = to_f(reinterpret_cast<const T*>(p.b)[(size_t)t * d.HV + h]);
        const float g = -expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]);
        p.gb[(size_t)t * d.HV + h] = make_float2(g, sigmoid_f(bv));
    }
}

// ---------------------------------------------------------------- 3. conv tail

template <typename T>
__global__ void __launch_bounds__(256) conv_tail_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    const int n = blockIdx.x;
    const int c = blockIdx.y * 256 + threadIdx.x;
    const int CD = p.d.conv_dim;
    if (c >= CD) return;
    const int len = p.cu[n + 1] - p.cu[n];
    const int slot = p.slots[n];
    if (len == 0 || slot < 0 || slot >= p.P) return;
    const bool init = p.has_init ? p.has_init[n] != 0 : true;
    T* cs = reinterpret_cast<T*>(p.conv_state) + ((size_t)slot * CD + c) * 3;
    const T* x = reinterpret_cast<const T*>(p.x);
    const T old0 = cs[0], old1 = cs[1], old2 = cs[2];
    const T zero = from_f<T>(0.f);
    T nv[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int pos = len + i;  // position in (old window | rows)
        if (pos < 3) nv[i] = init ? (pos == 0 ? old0 : pos == 1 ? old1 : old2) : zero;
        else nv[i] = x[(size_t)(p.cu[n] + pos - 3) * CD + c];
    }
    cs[0] = nv[0]; cs[1] = nv[1]; cs[2] = nv[2];
}

// ---------------------------------------------------------------- 4. intra
// on tensor cores, in gdn_intra_tc.cu

// ---------------------------------------------------------------- 5. state pass
// on tensor cores, in gdn_state_tc.cu

template <typename T, int DK, int DV>
cudaError_t launch_extend_t(const ExtendArgs& p, cudaStream_t s) {
    cudaError_t e;
    mark_launch(s, 0);
    chunk_map_kernel<<<1, 1024, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark_launch(s, 1);
    prep_kernel<T, DK, DV><<<p.T, 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark_launch(s, 2);
    conv_tail_kernel<T><<<dim3(p.N, (p.d.conv_dim + 255) / 256), 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark_launch(s, 3);
    if ((e = launch_intra<DK, DV>(p, s)) != cudaSuccess) return e;
    mark_launch(s, 4);
    if ((e = launch_state<T, DK, DV>(p, s)) != cudaSuccess) return e;
    mark_launch(s, 5);
    return cudaSuccess;
}

}  // namespace

size_t extend_workspace_bytes(const LayerDims& d, int max_N, int max_T, int* max_chunks_out) {
    const size_t mc = (size_t)max_T / C + (size_t)max_N + 1;
    if (max_chunks_out) *max_chunks_out = (int)mc;
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    const size_t per = mc * d.HV * sizeof(float);
    size_t off = kHeaderBytes;
    off += al(mc * sizeof(int4));
    off += al(((size_t)max_N + 1) * sizeof(int32_t));
    off += al((size_t)max_T * d.HK * d.dk * sizeof(float)) * 2;
    off += al((size_t)max_T * d.HV * d.dv * sizeof(float));
    off += al((size_t)max_T * d.HV * sizeof(float2));
    off += al(per * 2 * C * d.dk);
    off += al(per * C * C);
    off += al(per * d.dk * C);
    off += al(per * C * d.dv);
    off += al(per * C);
    return off;
}

void carve_extend_workspace(ExtendArgs& e, void* ws, int max_N, int max_T) {
    const LayerDims& d = e.d;
    int mc = 0;
    extend_workspace_bytes(d, max_N, max_T, &mc);
    e.max_chunks = mc;
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    const size_t per = (size_t)mc * d.HV * sizeof(float);
    char* base = static_cast<char*>(ws);
    e.hdr = reinterpret_cast<int32_t*>(base);
    size_t off = kHeaderBytes;
    e.chunk_tab = reinterpret_cast<int4*>(base + off); off += al((size_t)mc * sizeof(int4));
    e.seq_chunk0 = reinterpret_cast<int32_t*>(base + off); off += al(((size_t)max_N + 1) * sizeof(int32_t));
    e.qn = reinterpret_cast<float*>(base + off); off += al((size_t)max_T * d.HK * d.dk * sizeof(float));
    e.kn = reinterpret_cast<float*>(base + off); off += al((size_t)max_T * d.HK * d.dk * sizeof(float));
    e.vv = reinterpret_cast<float*>(base + off); off += al((size_t)max_T * d.HV * d.dv * sizeof(float));
    e.gb = reinterpret_cast<float2*>(base + off); off += al((size_t)max_T * d.HV * sizeof(float2));
    e.WQ = reinterpret_cast<float*>(base + off); off += al(per * 2 * C * d.dk);
    e.AQ = reinterpret_cast<float*>(base + off); off += al(per * C * C);
    e.KT = reinterpret_cast<float*>(base + off); off += al(per * d.dk * C);
    e.U = reinterpret_cast<float*>(base + off); off += al(per * C * d.dv);
    e.gam = reinterpret_cast<float*>(base + off);
}

cudaError_t launch_extend(const ExtendArgs& p, int dtype, cudaStream_t s) {
    if (dtype == GDN_DTYPE_BF16) GDN_DISPATCH_DIMS(__nv_bfloat16, launch_extend_t, p, s);
    GDN_DISPATCH_DIMS(float, launch_extend_t, p, s);
}

}  // namespace gdn
