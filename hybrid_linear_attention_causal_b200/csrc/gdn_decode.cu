// DECODE and TARGET_VERIFY kernels of the GDN layer (sm_100a).
//
// Both modes are bound by HBM traffic on the fp32 state: decode reads and
// writes each named slot's [HV, dk, dv] state once; verify reads it once and
// writes D checkpoints.  No tensor cores: the per-token work is two length-dk
// reductions per state column and a rank-1 update.
//
// One CTA serves one (request, qk head) pair, i.e. the G = HV/HK value heads
// that share that qk head.  That keeps every conv channel of the request owned
// by exactly one thread of one CTA, so the in-place conv-state update needs no
// cross-CTA ordering.  Inside the CTA each thread holds a float4 column group
// of RPT state rows in registers: coalesced 128-bit loads, both reductions
// (k^T S and q^T S) from one pass, cross-warp combination through shared
// memory, then the rank-1 update in registers and 128-bit stores.
//
// Per token and value head (the gated delta rule, fp32):
//   a = S^T k,  c = S^T q            (q already carries the output scale)
//   u = beta (v - e^g a)
//   o = e^g c + (q . k) u            (= scale * S_new^T q)
//   S <- e^g S + k u^T

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kNT = 256;
constexpr int kNW = kNT / 32;

// conv channel index of the i-th channel a (request, qk head hk) CTA owns:
// [q of hk (dk) | k of hk (dk) | v of heads hk*G .. hk*G+G-1 (G*dv)]
template <int DK, int DV>
__device__ __forceinline__ int owned_channel(const LayerDims& d, int hk, int i) {
    if (i < DK) return hk * DK + i;
    if (i < 2 * DK) return d.HK * DK + hk * DK + (i - DK);
    return 2 * d.HK * DK + hk * d.G * DV + (i - 2 * DK);
}

// L2-normalise q (times scale) and k of each token held in y[t][0 .. 2*DK),
// then store q.k per token in qk[t].  Warps take (token, q|k) pairs.
template <int DK>
__device__ __forceinline__ void normalise_qk(float* y, int nch, int D, const LayerDims& d, float* qk) {
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int pi = warp; pi < 2 * D; pi += kNW) {
        float* v = y + (pi >> 1) * nch + (pi & 1) * DK;
        float ss = 0.f;
        for (int i = lane; i < DK; i += 32) ss += v[i] * v[i];
        ss = warp_sum(ss);
        float r = rsqrtf(ss + d.eps) * ((pi & 1) ? 1.0f : d.scale);
        for (int i = lane; i < DK; i += 32) v[i] *= r;
    }
    __syncthreads();
    for (int t = warp; t < D; t += kNW) {
        const float* v = y + t * nch;
        float s = 0.f;
        for (int i = lane; i < DK; i += 32) s += v[i] * v[DK + i];
        s = warp_sum(s);
        if (lane == 0) qk[t] = s;
    }
}

// The per-token state step on register-held state.  Returns nothing; writes
// u to shared memory and the output column values through `emit`.
template <int DK, int DV, int RPT, int RSTEP, int CG, typename Emit>
__device__ __forceinline__ void state_step(float4 (&s)[RPT], const float* qv, const float* kv, const float* vv,
                                           float eg, float beta, float qk, float* red, float* usm, Emit emit) {
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int cg = tid % CG, r0 = tid / CG;
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pc = pa;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const int r = r0 + k * RSTEP;
        const float kr = kv[r], qr = qv[r];
        pa.x = fmaf(kr, s[k].x, pa.x); pa.y = fmaf(kr, s[k].y, pa.y);
        pa.z = fmaf(kr, s[k].z, pa.z); pa.w = fmaf(kr, s[k].w, pa.w);
        pc.x = fmaf(qr, s[k].x, pc.x); pc.y = fmaf(qr, s[k].y, pc.y);
        pc.z = fmaf(qr, s[k].z, pc.z); pc.w = fmaf(qr, s[k].w, pc.w);
    }
#pragma unroll
    for (int o = CG; o < 32; o <<= 1) {
        pa.x += __shfl_xor_sync(0xffffffffu, pa.x, o); pa.y += __shfl_xor_sync(0xffffffffu, pa.y, o);
        pa.z += __shfl_xor_sync(0xffffffffu, pa.z, o); pa.w += __shfl_xor_sync(0xffffffffu, pa.w, o);
        pc.x += __shfl_xor_sync(0xffffffffu, pc.x, o); pc.y += __shfl_xor_sync(0xffffffffu, pc.y, o);
        pc.z += __shfl_xor_sync(0xffffffffu, pc.z, o); pc.w += __shfl_xor_sync(0xffffffffu, pc.w, o);
    }
    if (lane < CG) {
        reinterpret_cast<float4*>(red + warp * DV)[lane] = pa;
        reinterpret_cast<float4*>(red + (kNW + warp) * DV)[lane] = pc;
    }
    __syncthreads();
    if (tid < DV) {
        float a = 0.f, c = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
            a += red[w * DV + tid];
            c += red[(kNW + w) * DV + tid];
        }
        const float u = beta * (vv[tid] - eg * a);
        usm[tid] = u;
        emit(tid, fmaf(eg, c, qk * u));
    }
    __syncthreads();
    const float4 u4 = reinterpret_cast<const float4*>(usm)[cg];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const float kr = kv[r0 + k * RSTEP];
        s[k].x = fmaf(eg, s[k].x, kr * u4.x); s[k].y = fmaf(eg, s[k].y, kr * u4.y);
        s[k].z = fmaf(eg, s[k].z, kr * u4.z); s[k].w = fmaf(eg, s[k].w, kr * u4.w);
    }
}

// The states of value heads h0 .. h0 + nh - 1 of a slot (contiguous in the pool) into L2, one
// 128-byte line per prefetch spread over the CTA, so that the state read overlaps work that does not
// need it yet (the conv, norm and gate phase; the previous head's tokens).
template <int DK, int DV>
__device__ __forceinline__ void prefetch_states_l2(const float* pool, int slot, int HV, int h0, int nh, int tid) {
    const char* base = reinterpret_cast<const char*>(pool + ((size_t)slot * HV + (size_t)h0) * DK * DV);
    const int lines = nh * DK * DV * 4 / 128;
    for (int l = tid; l < lines; l += kNT) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + (size_t)l * 128));
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kNT) decode_kernel(DecodeArgs p) {
    constexpr int CG = DV / 4, RSTEP = kNT / CG, RPT = DK / RSTEP;
    static_assert(DK % RSTEP == 0, "row split");
    extern __shared__ float4 smem4[];
    float* smem = reinterpret_cast<float*>(smem4);
    const LayerDims& d = p.d;
    const int req = blockIdx.x, hk = blockIdx.y, tid = threadIdx.x, G = d.G;
    const int nch = 2 * DK + G * DV;
    float* y = smem;                         // [nch]
    float* red = y + ((nch + 3) & ~3);       // [2*kNW*DV]
    float* usm = red + 2 * kNW * DV;         // [DV]
    float* misc = usm + DV;                  // qk, then (e^g, beta) per head
    T* out = reinterpret_cast<T*>(p.out) + ((size_t)req * d.HV + (size_t)hk * G) * DV;

    const int slot = p.slots[req];
    if (slot < 0 || slot >= p.P) {
        if (slot >= p.P && tid == 0 && hk == 0) raise_error(p.hdr, GDN_DEVERR_SLOT_RANGE);
        for (int i = tid; i < G * DV; i += kNT) out[i] = from_f<T>(0.f);
        return;
    }
    prefetch_states_l2<DK, DV>(p.ssm_state, slot, d.HV, hk * G, G, tid);
    // conv window update + SiLU for every owned channel
    {
        const T* x = reinterpret_cast<const T*>(p.x) + (size_t)req * d.conv_dim;
        T* cs = reinterpret_cast<T*>(p.conv_state) + (size_t)slot * d.conv_dim * 3;
        const T* w = reinterpret_cast<const T*>(p.conv_w);
        const T* bias = reinterpret_cast<const T*>(p.conv_b);
        for (int i = tid; i < nch; i += kNT) {
            const int c = owned_channel<DK, DV>(d, hk, i);
            const T s0 = cs[c * 3 + 0], s1 = cs[c * 3 + 1], s2 = cs[c * 3 + 2], xr = x[c];
            float acc = bias ? to_f(bias[c]) : 0.f;
            acc = fmaf(to_f(w[c * 4 + 0]), to_f(s0), acc);
            acc = fmaf(to_f(w[c * 4 + 1]), to_f(s1), acc);
            acc = fmaf(to_f(w[c * 4 + 2]), to_f(s2), acc);
            acc = fmaf(to_f(w[c * 4 + 3]), to_f(xr), acc);
            y[i] = silu_f(acc);
            cs[c * 3 + 0] = s1;
            cs[c * 3 + 1] = s2;
            cs[c * 3 + 2] = xr;
        }
    }
    if (tid < G) {
        const int h = hk * G + tid;
        const float av = to_f(reinterpret_cast<const T*>(p.a)[(size_t)req * d.HV + h]);
        const float bv = to_f(reinterpret_cast<const T*>(p.b)[(size_t)req * d.HV + h]);
        const float g = -expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]);
        misc[1 + 2 * tid] = expf(g);
        misc[2 + 2 * tid] = sigmoid_f(bv);
    }
    __syncthreads();
    normalise_qk<DK>(y, nch, 1, d, misc);
    __syncthreads();

    const int cg = tid % CG, r0 = tid / CG;
    for (int j = 0; j < G; ++j) {
        const int h = hk * G + j;
        float* Sp = p.ssm_state + ((size_t)slot * d.HV + h) * DK * DV;
        float4 s[RPT];
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            s[k] = __ldcs(reinterpret_cast<const float4*>(Sp + (size_t)(r0 + k * RSTEP) * DV) + cg);
        T* orow = out + j * DV;
        state_step<DK, DV, RPT, RSTEP, CG>(s, y, y + DK, y + 2 * DK + j * DV, misc[1 + 2 * j], misc[2 + 2 * j],
                                           misc[0], red, usm,
                                           [&](int col, float o) { orow[col] = from_f<T>(o); });
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            __stcs(reinterpret_cast<float4*>(Sp + (size_t)(r0 + k * RSTEP) * DV) + cg, s[k]);
    }
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kNT) verify_kernel(DecodeArgs p) {
    constexpr int CG = DV / 4, RSTEP = kNT / CG, RPT = DK / RSTEP;
    extern __shared__ float4 smem4[];
    float* smem = reinterpret_cast<float*>(smem4);
    const LayerDims& d = p.d;
    const int req = blockIdx.x, hk = blockIdx.y, tid = threadIdx.x, G = d.G, D = p.D;
    const int nch = 2 * DK + G * DV;
    const int nchp = (nch + 3) & ~3;
    float* y = smem;                        // [D][nchp]
    float* red = y + D * nchp;              // [2*kNW*DV]
    float* usm = red + 2 * kNW * DV;        // [DV]
    float* qk = usm + DV;                   // [D]
    float* gate = qk + kMaxVerifyDraft;     // [D][G] x (e^g, beta)
    __shared__ int par[kMaxVerifyDraft];    // draft-tree parent of each token (-1 = the slot)
    __shared__ int tree_bad;

    // the draft tree: a chain (parent t-1) unless parents are given; every parent must precede its token
    if (tid == 0) tree_bad = 0;
    __syncthreads();
    if (tid < D) {
        const int pt = p.parents ? p.parents[(size_t)req * D + tid] : tid - 1;
        par[tid] = pt;
        if (pt < -1 || pt >= tid) atomicOr(&tree_bad, 1);
    }
    __syncthreads();
    const int slot = p.slots[req];
    T* out0 = reinterpret_cast<T*>(p.out);
    if (slot < 0 || slot >= p.P || tree_bad) {
        if (slot >= p.P && tid == 0 && hk == 0) raise_error(p.hdr, GDN_DEVERR_SLOT_RANGE);
        if (tree_bad && slot >= 0 && tid == 0 && hk == 0) raise_error(p.hdr, GDN_DEVERR_TREE);
        for (int t = 0; t < D; ++t) {
            T* o = out0 + (((size_t)req * D + t) * d.HV + (size_t)hk * G) * DV;
            for (int i = tid; i < G * DV; i += kNT) o[i] = from_f<T>(0.f);
        }
        return;
    }
    // the first value head's state at the start; each next one while the previous head's tokens run
    // (measured faster than all of them at the start)
    prefetch_states_l2<DK, DV>(p.ssm_state, slot, d.HV, hk * G, 1, tid);
    {
        const T* cs = reinterpret_cast<const T*>(p.conv_state) + (size_t)slot * d.conv_dim * 3;
        const T* w = reinterpret_cast<const T*>(p.conv_w);
        const T* bias = reinterpret_cast<const T*>(p.conv_b);
        T* cck = reinterpret_cast<T*>(p.conv_ckpt);
        const T* xq = reinterpret_cast<const T*>(p.x) + (size_t)req * D * d.conv_dim;
        for (int i = tid; i < nch; i += kNT) {
            const int c = owned_channel<DK, DV>(d, hk, i);
            const float w0 = to_f(w[c * 4 + 0]), w1 = to_f(w[c * 4 + 1]), w2 = to_f(w[c * 4 + 2]),
                        w3 = to_f(w[c * 4 + 3]);
            const float bc = bias ? to_f(bias[c]) : 0.f;
            for (int t = 0; t < D; ++t) {
                // the 3 raw rows before token t, newest first: its ancestors' rows, then the slot's
                // window from its newest row back (on a chain these are rows t-1, t-2, t-3)
                T win[3];
                int nd = par[t], sk = 2;
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    if (nd >= 0) {
                        win[q] = xq[(size_t)nd * d.conv_dim + c];
                        nd = par[nd];
                    } else {
                        win[q] = cs[c * 3 + sk];
                        --sk;
                    }
                }
                const T xr = xq[(size_t)t * d.conv_dim + c];
                float acc = fmaf(w0, to_f(win[2]), bc);
                acc = fmaf(w1, to_f(win[1]), acc);
                acc = fmaf(w2, to_f(win[0]), acc);
                acc = fmaf(w3, to_f(xr), acc);
                y[t * nchp + i] = silu_f(acc);
                if (cck) {  // the window after token t, oldest first
                    T* dst = cck + (((size_t)req * D + t) * d.conv_dim + c) * 3;
                    dst[0] = win[1]; dst[1] = win[0]; dst[2] = xr;
                }
            }
        }
    }
    for (int i = tid; i < D * G; i += kNT) {
        const int t = i / G, j = i % G, h = hk * G + j;
        const size_t row = (size_t)req * D + t;
        const float av = to_f(reinterpret_cast<const T*>(p.a)[row * d.HV + h]);
        const float bv = to_f(reinterpret_cast<const T*>(p.b)[row * d.HV + h]);
        const float g = -expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]);
        gate[2 * i] = expf(g);
        gate[2 * i + 1] = sigmoid_f(bv);
    }
    __syncthreads();
    normalise_qk<DK>(y, nchp, D, d, qk);
    __syncthreads();

    const int cg = tid % CG, r0 = tid / CG;
    for (int j = 0; j < G; ++j) {
        const int h = hk * G + j;
        const float* Sp = p.ssm_state + ((size_t)slot * d.HV + h) * DK * DV;
        float4 s[RPT];
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            s[k] = __ldcs(reinterpret_cast<const float4*>(Sp + (size_t)(r0 + k * RSTEP) * DV) + cg);
        if (j + 1 < G) prefetch_states_l2<DK, DV>(p.ssm_state, slot, d.HV, h + 1, 1, tid);
        int cur = -1;  // the tree node whose state the registers hold
        for (int t = 0; t < D; ++t) {
            if (par[t] != cur) {  // a branch: continue from the parent's checkpoint (or the slot), which
                                  // this very thread wrote (or read) element for element
                const float* src =
                    par[t] < 0 ? Sp : p.state_ckpt + (((size_t)req * D + par[t]) * d.HV + h) * DK * DV;
#pragma unroll
                for (int k = 0; k < RPT; ++k)
                    s[k] = reinterpret_cast<const float4*>(src + (size_t)(r0 + k * RSTEP) * DV)[cg];
            }
            cur = t;
            const float* yt = y + t * nchp;
            T* orow = out0 + (((size_t)req * D + t) * d.HV + h) * DV;
            state_step<DK, DV, RPT, RSTEP, CG>(s, yt, yt + DK, yt + 2 * DK + j * DV, gate[2 * (t * G + j)],
                                               gate[2 * (t * G + j) + 1], qk[t], red, usm,
                                               [&](int col, float o) { orow[col] = from_f<T>(o); });
            float* ck = p.state_ckpt + (((size_t)req * D + t) * d.HV + h) * DK * DV;
#pragma unroll
            for (int k = 0; k < RPT; ++k)
                __stcs(reinterpret_cast<float4*>(ck + (size_t)(r0 + k * RSTEP) * DV) + cg, s[k]);
        }
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_decode_t(const DecodeArgs& p, cudaStream_t s) {
    const int nch = 2 * DK + p.d.G * DV;
    const size_t shm = sizeof(float) * (((nch + 3) & ~3) + 2 * kNW * DV + DV + 4 + 2 * p.d.G);
    auto k = decode_kernel<T, DK, DV>;
    if (shm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
        if (e != cudaSuccess) return e;
    }
    mark_launch(s, 0);
    k<<<dim3(p.B, p.d.HK), kNT, shm, s>>>(p);
    cudaError_t e = cudaGetLastError();
    mark_launch(s, 1);
    return e;
}

template <typename T, int DK, int DV>
cudaError_t launch_verify_t(const DecodeArgs& p, cudaStream_t s) {
    static_assert(kMaxVerifyDraft <= kNT, "one thread per draft token reads the tree");
    const int nchp = (2 * DK + p.d.G * DV + 3) & ~3;
    const size_t shm =
        sizeof(float) * ((size_t)p.D * nchp + 2 * kNW * DV + DV + kMaxVerifyDraft + 2 * (size_t)p.D * p.d.G);
    auto k = verify_kernel<T, DK, DV>;
    if (shm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
        if (e != cudaSuccess) return e;
    }
    mark_launch(s, 0);
    k<<<dim3(p.B, p.d.HK), kNT, shm, s>>>(p);
    cudaError_t e = cudaGetLastError();
    mark_launch(s, 1);
    return e;
}


}  // namespace

cudaError_t launch_decode(const DecodeArgs& p, int dtype, cudaStream_t s) {
    if (dtype == GDN_DTYPE_BF16) GDN_DISPATCH_DIMS(__nv_bfloat16, launch_decode_t, p, s);
    GDN_DISPATCH_DIMS(float, launch_decode_t, p, s);
}

cudaError_t launch_verify(const DecodeArgs& p, int dtype, cudaStream_t s) {
    if (dtype == GDN_DTYPE_BF16) GDN_DISPATCH_DIMS(__nv_bfloat16, launch_verify_t, p, s);
    GDN_DISPATCH_DIMS(float, launch_verify_t, p, s);
}

}  // namespace gdn
