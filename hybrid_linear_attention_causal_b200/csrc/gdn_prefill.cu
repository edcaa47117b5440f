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
//   4. intra:      per (chunk, value head): gamma, A, W, U, masked decayed q.k
//   5. state:      per (sequence, value head, dv tile): the serial chunk pass
//                  V' = U - W S, the outputs and S <- e^{gamma_n} S + K~^T V'
// Every intermediate is fp32: the parity bar leaves no room for bf16 rounding
// of q, k, v, W, U or V' (each alone adds ~1.7e-3 relative error).

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;

__device__ __forceinline__ bool batch_rejected(const ExtendArgs& p) { return p.hdr[kHdrNumChunks] == 0; }

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

template <int DK, int DV>
struct IntraSmem {
    float K[C][DK + 1];
    float Q[C][DK + 1];
    float X[C][DK + DV + 1];
    float A[C][C + 1];
    float gam[C];
    float beta[C];
};

template <int DK, int DV>
__global__ void __launch_bounds__(256) intra_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    const int id = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (id >= p.hdr[kHdrNumChunks]) return;
    const int4 ch = p.chunk_tab[id];
    const int slot = p.slots[ch.x];
    if (slot < 0 || slot >= p.P) return;
    const LayerDims& d = p.d;
    const int hk = h / d.G, t0 = ch.y, n = ch.z;
    extern __shared__ float4 smem4[];
    IntraSmem<DK, DV>& sm = *reinterpret_cast<IntraSmem<DK, DV>*>(smem4);

    for (int e = tid; e < C * DK; e += 256) {
        const int r = e / DK, i = e % DK;
        const bool live = r < n;
        sm.K[r][i] = live ? p.kn[((size_t)(t0 + r) * d.HK + hk) * DK + i] : 0.f;
        sm.Q[r][i] = live ? p.qn[((size_t)(t0 + r) * d.HK + hk) * DK + i] : 0.f;
    }
    for (int e = tid; e < C * DV; e += 256) {
        const int r = e / DV, j = e % DV;
        sm.X[r][DK + j] = r < n ? p.vv[((size_t)(t0 + r) * d.HV + h) * DV + j] : 0.f;
    }
    if (tid < 32) {  // inclusive scan of g over the chunk (two rows per lane)
        float2 gb0 = tid * 2 < n ? p.gb[(size_t)(t0 + tid * 2) * d.HV + h] : make_float2(0.f, 0.f);
        float2 gb1 = tid * 2 + 1 < n ? p.gb[(size_t)(t0 + tid * 2 + 1) * d.HV + h] : make_float2(0.f, 0.f);
        float pair = gb0.x + gb1.x;
        float incl = pair;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, incl, o);
            if (tid >= o) incl += v;
        }
        const float excl = incl - pair;
        sm.gam[tid * 2] = excl + gb0.x;
        sm.gam[tid * 2 + 1] = incl;
        sm.beta[tid * 2] = gb0.y;
        sm.beta[tid * 2 + 1] = gb1.y;
    }
    __syncthreads();

    // k.k (s < r) and q.k (s <= r): thread owns row r = tid/4 and columns s = tid%4 + 4m
    {
        const int r = tid >> 2, s0 = tid & 3;
        float kk[16], qk[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) { kk[m] = 0.f; qk[m] = 0.f; }
        for (int i = 0; i < DK; ++i) {
            const float kr = sm.K[r][i], qr = sm.Q[r][i];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float ks = sm.K[s0 + 4 * m][i];
                kk[m] = fmaf(kr, ks, kk[m]);
                qk[m] = fmaf(qr, ks, qk[m]);
            }
        }
        const float gr = sm.gam[r], br = sm.beta[r];
        float* aq = p.Aqk + (((size_t)id * d.HV + h) * C + r) * C;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int s = s0 + 4 * m;
            const bool valid = r < n && s < n;
            const float dec = valid && s <= r ? expf(gr - sm.gam[s]) : 0.f;
            sm.A[r][s] = (s < r) ? br * dec * kk[m] : 0.f;
            aq[s] = dec * qk[m];
        }
    }
    // right-hand sides: rows of diag(beta e^gamma) K and diag(beta) V
    for (int e = tid; e < C * DK; e += 256) {
        const int r = e / DK, i = e % DK;
        sm.X[r][i] = sm.beta[r] * expf(sm.gam[r]) * sm.K[r][i];
    }
    for (int e = tid; e < C * DV; e += 256) {
        const int r = e / DV, j = e % DV;
        sm.X[r][DK + j] *= sm.beta[r];
    }
    __syncthreads();
    // forward substitution, one column per thread: X[r] -= sum_{s<r} A[r,s] X[s]
    for (int col = tid; col < DK + DV; col += 256) {
        for (int r = 1; r < n; ++r) {
            float acc = sm.X[r][col];
            for (int s = 0; s < r; ++s) acc = fmaf(-sm.A[r][s], sm.X[s][col], acc);
            sm.X[r][col] = acc;
        }
    }
    __syncthreads();
    float* Wd = p.W + ((size_t)id * d.HV + h) * C * DK;
    float* Ud = p.U + ((size_t)id * d.HV + h) * C * DV;
    for (int e = tid; e < C * DK; e += 256) Wd[e] = sm.X[e / DK][e % DK];
    for (int e = tid; e < C * DV; e += 256) Ud[e] = sm.X[e / DV][DK + e % DV];
    if (tid < C) p.gam[((size_t)id * d.HV + h) * C + tid] = sm.gam[tid];
}

// ---------------------------------------------------------------- 5. state pass

template <int DK, int DT>
struct StateSmem {
    float S[DK][DT];
    float W[C][DK];
    float Q[C][DK];
    float K[C][DK];
    float Aqk[C][C];
    float U[C][DT];
    float Vn[C][DT];
    float gam[C];
};

template <typename T, int DK, int DV, int DT>
__global__ void __launch_bounds__(256) state_kernel(ExtendArgs p) {
    static_assert(DT == 32, "one warp spans the dv tile");
    if (batch_rejected(p)) return;
    const int nseq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * DT, tid = threadIdx.x;
    const LayerDims& d = p.d;
    const int hk = h / d.G;
    const int len = p.cu[nseq + 1] - p.cu[nseq];
    if (len == 0) return;
    const int slot = p.slots[nseq];
    T* out = reinterpret_cast<T*>(p.out);
    if (slot < 0 || slot >= p.P) {
        if (slot >= p.P && tid == 0 && h == 0 && blockIdx.z == 0) raise_error(p.hdr, GDN_DEVERR_SLOT_RANGE);
        for (int e = tid; e < len * DT; e += 256) {
            const int r = e / DT, j = e % DT;
            out[((size_t)(p.cu[nseq] + r) * d.HV + h) * DV + j0 + j] = from_f<T>(0.f);
        }
        return;
    }
    extern __shared__ float4 smem4[];
    StateSmem<DK, DT>& sm = *reinterpret_cast<StateSmem<DK, DT>*>(smem4);
    const bool init = p.has_init ? p.has_init[nseq] != 0 : true;
    float* Sg = p.ssm_state + ((size_t)slot * d.HV + h) * DK * DV;
    for (int e = tid; e < DK * DT; e += 256) {
        const int i = e / DT, j = e % DT;
        sm.S[i][j] = init ? Sg[(size_t)i * DV + j0 + j] : 0.f;
    }
    const int lane = tid & 31, wg = tid >> 5;  // lane = column j, warp = row group
    const int c_begin = p.seq_chunk0[nseq], c_end = p.seq_chunk0[nseq + 1];
    for (int id = c_begin; id < c_end; ++id) {
        const int4 ch = p.chunk_tab[id];
        const int t0 = ch.y, n = ch.z;
        const float* Wg = p.W + ((size_t)id * d.HV + h) * C * DK;
        const float* Ug = p.U + ((size_t)id * d.HV + h) * C * DV;
        const float* Ag = p.Aqk + ((size_t)id * d.HV + h) * C * C;
        for (int e = tid; e < C * DK / 4; e += 256) {
            const int r = (e * 4) / DK, i = (e * 4) % DK;
            reinterpret_cast<float4*>(&sm.W[r][i])[0] = reinterpret_cast<const float4*>(Wg)[e];
            const bool live = r < n;
            const size_t qo = ((size_t)(t0 + r) * d.HK + hk) * DK + i;
            reinterpret_cast<float4*>(&sm.Q[r][i])[0] =
                live ? *reinterpret_cast<const float4*>(p.qn + qo) : make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4*>(&sm.K[r][i])[0] =
                live ? *reinterpret_cast<const float4*>(p.kn + qo) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int e = tid; e < C * C / 4; e += 256)
            reinterpret_cast<float4*>(&sm.Aqk[0][0])[e] = reinterpret_cast<const float4*>(Ag)[e];
        for (int e = tid; e < C * DT; e += 256) {
            const int r = e / DT, j = e % DT;
            sm.U[r][j] = Ug[(size_t)r * DV + j0 + j];
        }
        if (tid < C) sm.gam[tid] = p.gam[((size_t)id * d.HV + h) * C + tid];
        __syncthreads();
        // V' = U - W S   (rows r = wg + 8m)
        {
            float acc[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[m] = sm.U[wg + 8 * m][lane];
            for (int i = 0; i < DK; ++i) {
                const float sv = sm.S[i][lane];
#pragma unroll
                for (int m = 0; m < 8; ++m) acc[m] = fmaf(-sm.W[wg + 8 * m][i], sv, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) sm.Vn[wg + 8 * m][lane] = acc[m];
        }
        __syncthreads();
        // outputs: e^{gamma_r} q_r^T S + sum_{s<=r} Aqk[r,s] V'_s
        {
            float acc[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[m] = 0.f;
            for (int i = 0; i < DK; ++i) {
                const float sv = sm.S[i][lane];
#pragma unroll
                for (int m = 0; m < 8; ++m) acc[m] = fmaf(sm.Q[wg + 8 * m][i], sv, acc[m]);
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int r = wg + 8 * m;
                float o = expf(sm.gam[r]) * acc[m];
                for (int s = 0; s <= r; ++s) o = fmaf(sm.Aqk[r][s], sm.Vn[s][lane], o);
                if (r < n) out[((size_t)(t0 + r) * d.HV + h) * DV + j0 + lane] = from_f<T>(o);
            }
        }
        // S <- e^{gamma_n} S + sum_r e^{gamma_n - gamma_r} k_r V'_r^T   (rows i = wg + 8m)
        {
            const float gl = sm.gam[n - 1];
            float acc[DK / 8];
#pragma unroll
            for (int m = 0; m < DK / 8; ++m) acc[m] = expf(gl) * sm.S[wg + 8 * m][lane];
            for (int r = 0; r < n; ++r) {
                const float vr = sm.Vn[r][lane] * expf(gl - sm.gam[r]);
#pragma unroll
                for (int m = 0; m < DK / 8; ++m) acc[m] = fmaf(sm.K[r][wg + 8 * m], vr, acc[m]);
            }
            __syncthreads();
#pragma unroll
            for (int m = 0; m < DK / 8; ++m) sm.S[wg + 8 * m][lane] = acc[m];
        }
        __syncthreads();
    }
    for (int e = tid; e < DK * DT; e += 256) {
        const int i = e / DT, j = e % DT;
        Sg[(size_t)i * DV + j0 + j] = sm.S[i][j];
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_extend_t(const ExtendArgs& p, cudaStream_t s) {
    constexpr int DT = 32;
    const size_t shm_intra = sizeof(IntraSmem<DK, DV>);
    const size_t shm_state = sizeof(StateSmem<DK, DT>);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(intra_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)shm_intra)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(state_kernel<T, DK, DV, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)shm_state)) != cudaSuccess)
        return e;
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
    intra_kernel<DK, DV><<<dim3(p.max_chunks, p.d.HV), 256, shm_intra, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark_launch(s, 4);
    state_kernel<T, DK, DV, DT><<<dim3(p.N, p.d.HV, DV / DT), 256, shm_state, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark_launch(s, 5);
    return cudaSuccess;
}

}  // namespace

size_t extend_workspace_bytes(const LayerDims& d, int max_N, int max_T, int* max_chunks_out) {
    const size_t mc = (size_t)max_T / C + (size_t)max_N + 1;
    if (max_chunks_out) *max_chunks_out = (int)mc;
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    size_t off = kHeaderBytes;
    off += al(mc * sizeof(int4));
    off += al(((size_t)max_N + 1) * sizeof(int32_t));
    off += al((size_t)max_T * d.HK * d.dk * sizeof(float)) * 2;
    off += al((size_t)max_T * d.HV * d.dv * sizeof(float));
    off += al((size_t)max_T * d.HV * sizeof(float2));
    off += al(mc * d.HV * C * d.dk * sizeof(float));
    off += al(mc * d.HV * C * d.dv * sizeof(float));
    off += al(mc * d.HV * C * C * sizeof(float));
    off += al(mc * d.HV * C * sizeof(float));
    return off;
}

void carve_extend_workspace(ExtendArgs& e, void* ws, int max_N, int max_T) {
    const LayerDims& d = e.d;
    int mc = 0;
    extend_workspace_bytes(d, max_N, max_T, &mc);
    e.max_chunks = mc;
    auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
    char* base = static_cast<char*>(ws);
    e.hdr = reinterpret_cast<int32_t*>(base);
    size_t off = kHeaderBytes;
    e.chunk_tab = reinterpret_cast<int4*>(base + off); off += al((size_t)mc * sizeof(int4));
    e.seq_chunk0 = reinterpret_cast<int32_t*>(base + off); off += al(((size_t)max_N + 1) * sizeof(int32_t));
    e.qn = reinterpret_cast<float*>(base + off); off += al((size_t)max_T * d.HK * d.dk * sizeof(float));
    e.kn = reinterpret_cast<float*>(base + off); off += al((size_t)max_T * d.HK * d.dk * sizeof(float));
    e.vv = reinterpret_cast<float*>(base + off); off += al((size_t)max_T * d.HV * d.dv * sizeof(float));
    e.gb = reinterpret_cast<float2*>(base + off); off += al((size_t)max_T * d.HV * sizeof(float2));
    e.W = reinterpret_cast<float*>(base + off); off += al((size_t)mc * d.HV * C * d.dk * sizeof(float));
    e.U = reinterpret_cast<float*>(base + off); off += al((size_t)mc * d.HV * C * d.dv * sizeof(float));
    e.Aqk = reinterpret_cast<float*>(base + off); off += al((size_t)mc * d.HV * C * C * sizeof(float));
    e.gam = reinterpret_cast<float*>(base + off);
}

cudaError_t launch_extend(const ExtendArgs& p, int dtype, cudaStream_t s) {
    if (dtype == GDN_DTYPE_BF16) GDN_DISPATCH_DIMS(__nv_bfloat16, launch_extend_t, p, s);
    GDN_DISPATCH_DIMS(float, launch_extend_t, p, s);
}

}  // namespace gdn
