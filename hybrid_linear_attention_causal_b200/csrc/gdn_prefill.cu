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
//   2. chunk:      per (chunk, qk head) on tensor cores: conv1d + SiLU, L2 norm,
//                  gates, A, T, W, U and the masked decayed q.k of each value
//                  head (gdn_chunk_tc.cu), segment by segment
//   3. state:      per (sequence, value head) on tensor cores: the serial chunk
//                  pass V' = U - W S, the outputs and S <- e^{gamma_n} S + K~^T V'
//                  (gdn_state_tc.cu), segment by segment on a second stream
//   4. conv_tail:  writes each sequence's new conv window into its slot, once
//                  every chunk has read the windows it started from
// Every tensor-core operand is rounded to fp16 (round to nearest) with fp32
// accumulation; the state, A, T and the gates stay fp32.

#include <cuda_fp16.h>

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;

// ---------------------------------------------------------------- 1. chunk map

__global__ void __launch_bounds__(1024) chunk_map_kernel(ExtendArgs p) {
    __shared__ int s_bad;
    __shared__ int s_scan[1024];
    __shared__ int s_base;
    __shared__ int s_rank[1024], s_off[1024];  // (N <= 1024) rank of each sequence; list offset by rank
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
    // Longest sequences first (rank by chunk count, ties by index; more than 1024 sequences keep
    // their order).  This is the state pass's launch order and the order of chunk_list, which holds
    // the chunks rank by rank; rank_off[r] is the list position of rank r's first chunk.
    const bool small = p.N <= 1024;
    if (small) {
        const int nc_t = tid < p.N ? p.seq_chunk0[tid + 1] - p.seq_chunk0[tid] : 0;
        if (tid < p.N) s_scan[tid] = nc_t;
        __syncthreads();
        if (tid < p.N) {
            int rank = 0;
            for (int j = 0; j < p.N; ++j) {
                const int o = s_scan[j];
                rank += (o > nc_t || (o == nc_t && j < tid)) ? 1 : 0;
            }
            p.seq_order[rank] = tid;
            s_rank[tid] = rank;
            s_off[rank] = nc_t;
        }
        __syncthreads();
        // exclusive scan of the chunk counts in rank order
        const int own = tid < p.N ? s_off[tid] : 0;
        for (int off = 1; off < 1024; off <<= 1) {
            const int v = tid >= off ? s_off[tid - off] : 0;
            __syncthreads();
            if (tid < p.N) s_off[tid] += v;
            __syncthreads();
        }
        if (tid < p.N) {
            s_off[tid] -= own;
            p.rank_off[tid] = s_off[tid];
        }
    } else {
        for (int i = tid; i < p.N; i += 1024) {
            p.seq_order[i] = i;
            p.rank_off[i] = p.seq_chunk0[i];
        }
    }
    if (tid == 0) p.rank_off[p.N] = total;
    __threadfence_block();
    __syncthreads();
    // Segments: the list cut into nseg pieces growing by kSegGrowth.  The state pass of segment k takes,
    // for each sequence, its chunks inside piece k, continuing from the state the previous piece left.
    if (tid < kMaxSegments) {
        const int k = tid, lo = seg_bound(k, p.nseg, total), hi = k < p.nseg ? seg_bound(k + 1, p.nseg, total) : lo;
        p.hdr[kHdrSegOff + k] = lo;
        p.hdr[kHdrSegCnt + k] = hi - lo;
        p.hdr[kHdrItemNext + k] = 0;
        int first = p.N, last = p.N - 1;
        if (lo < hi) {  // ranks holding list positions lo and hi - 1
            int a = 0, b = p.N - 1;
            while (a < b) {
                const int m = (a + b + 1) >> 1;
                if (p.rank_off[m] <= lo) a = m; else b = m - 1;
            }
            first = a;
            b = p.N - 1;
            while (a < b) {
                const int m = (a + b + 1) >> 1;
                if (p.rank_off[m] <= hi - 1) a = m; else b = m - 1;
            }
            last = a;
        }
        p.hdr[kHdrSegRank + k] = first;
        p.hdr[kHdrSegSeqs + k] = last - first + 1;
    }
    if (tid == 0) p.hdr[kHdrSegLen] = seg_bound(p.nseg, p.nseg, total) - seg_bound(p.nseg - 1, p.nseg, total);
    for (int id = tid; id < total; id += 1024) {
        int lo = 0, hi = p.N - 1;  // last sequence whose first chunk id <= id
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.seq_chunk0[mid] <= id) lo = mid; else hi = mid - 1;
        }
        const int c = id - p.seq_chunk0[lo];
        const int len = p.cu[lo + 1] - p.cu[lo];
        p.chunk_tab[id] = make_int4(lo, p.cu[lo] + c * C, min(C, len - c * C), c);
        p.chunk_list[(small ? s_off[s_rank[lo]] : p.seq_chunk0[lo]) + c] = id;
    }
}

// ---------------------------------------------------------------- conv tail

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

// A second stream (at the device's greatest priority) with one fork event per
// segment and a join event, per host thread and device, created by the first
// extend call there and kept until the process exits.  Inside a stream
// capture the fork / join events make it part of the captured graph.
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t seg[kMaxSegments] = {};
    cudaEvent_t join = nullptr;
};

constexpr int kMaxSideDevices = 64;

cudaError_t side_stream(SideStream** out) {
    thread_local SideStream per_device[kMaxSideDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
    SideStream& ss = per_device[dev];
    if (!ss.s) {
        SideStream n;
        int least = 0, greatest = 0;
        if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) == cudaSuccess)
            e = cudaStreamCreateWithPriority(&n.s, cudaStreamNonBlocking, greatest);
        for (int k = 0; k < kMaxSegments && e == cudaSuccess; ++k)
            e = cudaEventCreateWithFlags(&n.seg[k], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming);
        if (e != cudaSuccess) {  // nothing half-made is kept
            for (int k = 0; k < kMaxSegments; ++k)
                if (n.seg[k]) cudaEventDestroy(n.seg[k]);
            if (n.s) cudaStreamDestroy(n.s);
            return e;
        }
        ss = n;
    }
    *out = &ss;
    return cudaSuccess;
}

// ---------------------------------------------------------------- state checkpoints

// The conv window at each sequence's checkpoint boundary: the K-1 raw rows before it, reaching into
// the sequence's starting conv window (launched before the conv-state update overwrites that).
// Raises GDN_DEVERR_CKPT_RANGE for a boundary outside its sequence or a row out of range.
template <typename T>
__global__ void __launch_bounds__(256) ckpt_conv_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    const int n = blockIdx.x;
    const int slot = p.slots[n];
    if (slot < 0 || slot >= p.P) return;  // padded sequences capture nothing
    int row = 0;
    const int t = ckpt_offset(p, n, &row);
    if (t == -2 && blockIdx.y == 0 && threadIdx.x == 0) raise_error(p.hdr, GDN_DEVERR_CKPT_RANGE);
    if (t < 0 || !p.ck_conv) return;
    const int cd = p.d.conv_dim;
    const int c = blockIdx.y * 256 + threadIdx.x;
    if (c >= cd) return;
    const bool init = p.has_init ? p.has_init[n] != 0 : true;
    const int t0 = p.cu[n], bnd = t0 + t;
    const T* x = reinterpret_cast<const T*>(p.x);
    const T* cs = reinterpret_cast<const T*>(p.conv_state) + ((size_t)slot * cd + c) * (kConvK - 1);
    T* dst = reinterpret_cast<T*>(p.ck_conv) + ((size_t)row * cd + c) * (kConvK - 1);
#pragma unroll
    for (int j = 0; j < kConvK - 1; ++j) {
        const int r = bnd - (kConvK - 1) + j;  // window entry j (0 oldest)
        dst[j] = r >= t0 ? x[(size_t)r * cd + c] : (init ? cs[kConvK - 1 + (r - t0)] : from_f<T>(0.f));
    }
}

// The state at each checkpoint boundary that does not sit on a chunk edge.  The state pass stored
// the state S_c entering the boundary's chunk; the m rows of that chunk before the boundary add
//   S_m = e^{gamma_{m-1}} S_c + sum_{s<m} e^{gamma_{m-1} - gamma_s} k_s v'_s^T,   v'_s = u_s - S_c^T w_s,
// where u_s and w_s are rows of the chunk's U and W: those rows depend only on the chunk's rows up
// to s (T = (I + A)^{-1} is lower triangular), so cutting the chunk at the boundary leaves them as
// they are.  fp32 on CUDA cores, from the fp16 tiles the prefill already holds.  One CTA per
// (sequence, value head, quarter of the dv columns); a sequence with no rows gets the state it
// started from.
constexpr int kCkptSplit = 4;  // CTAs per (sequence, value head), one group of dv columns each

template <int DK, int DV>
__global__ void __launch_bounds__(256) ckpt_finish_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    constexpr int DVS = DV / kCkptSplit;  // this CTA's columns j0 .. j0 + DVS - 1
    const int n = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * DVS, tid = threadIdx.x;
    const int slot = p.slots[n];
    if (slot < 0 || slot >= p.P) return;
    int row = 0;
    const int t = ckpt_offset(p, n, &row);
    if (t < 0) return;
    const LayerDims& d = p.d;
    float* dst = p.ck_states + ((size_t)row * d.HV + h) * DK * DV;
    const int len = p.cu[n + 1] - p.cu[n];
    if (len == 0) {
        const bool init = p.has_init ? p.has_init[n] != 0 : true;
        const float* src = p.ssm_state + ((size_t)slot * d.HV + h) * DK * DV;
        for (int e = tid; e < DK * DVS; e += 256) {
            const size_t o = (size_t)(e / DVS) * DV + j0 + e % DVS;
            dst[o] = init ? src[o] : 0.f;
        }
        return;
    }
    const int cl = min(t / C, (len + C - 1) / C - 1), m = t - C * cl;
    if (m == 0) return;  // on a chunk edge: the state pass stored it
    const size_t id = (size_t)p.seq_chunk0[n] + cl;
    extern __shared__ __align__(16) float fsm[];
    float* Sc = fsm;            // [DK][DVS] this CTA's columns of S_c
    float* Wf = Sc + DK * DVS;  // [C][DK] rows s < m of W
    float* Kf = Wf + C * DK;    // [C][DK] rows s < m of K
    float* Vp = Kf + C * DK;    // [C][DVS] v'_s, this CTA's columns
    float* coef = Vp + C * DVS; // [C] e^{gamma_{m-1} - gamma_s}
    const char* Wg = reinterpret_cast<const char*>(p.W + (id * d.HV + h) * (C * DK));
    const char* KQg = reinterpret_cast<const char*>(p.KQ + (id * d.HK + h / d.G) * (2 * C * DK));
    const char* Ug = reinterpret_cast<const char*>(p.U + (id * d.HV + h) * (DV * C));
    const float* gam = reinterpret_cast<const float*>(p.GV + (id * d.HV + h) * C) + 2 * C;  // gamma
    auto h2f = [](const char* q) { return __half2float(*reinterpret_cast<const __half*>(q)); };
    for (int e = tid; e < DK * DVS / 4; e += 256) {
        const int f = e / (DVS / 4), j4 = e % (DVS / 4);
        reinterpret_cast<float4*>(Sc)[e] = reinterpret_cast<const float4*>(dst + (size_t)f * DV + j0)[j4];
    }
    for (int e = tid; e < m * DK; e += 256) {
        const int sr = e / DK, f = e % DK;
        Wf[e] = h2f(Wg + tc::sw128_off(f, sr, DK));  // the tile holds W^T
        Kf[e] = h2f(KQg + tc::sw128_off(sr, f, 2 * C));
    }
    if (tid < m) coef[tid] = expf(gam[m - 1] - gam[tid]);
    __syncthreads();
    for (int e = tid; e < m * DVS; e += 256) {  // v'_s[j] = u_s[j] - sum_f w_s[f] S_c[f][j]
        const int sr = e / DVS, jl = e % DVS;
        float acc = h2f(Ug + tc::sw128_off(j0 + jl, sr, DV));
#pragma unroll 8
        for (int f = 0; f < DK; ++f) acc = fmaf(-Wf[sr * DK + f], Sc[f * DVS + jl], acc);
        Vp[e] = acc;
    }
    __syncthreads();
    const float eg = expf(gam[m - 1]);
    for (int e = tid; e < DK * DVS; e += 256) {
        const int f = e / DVS, jl = e % DVS;
        float acc = eg * Sc[e];
        for (int sr = 0; sr < m; ++sr) acc = fmaf(coef[sr] * Kf[sr * DK + f], Vp[sr * DVS + jl], acc);
        dst[(size_t)f * DV + j0 + jl] = acc;
    }
}

template <int DK, int DV>
constexpr size_t ckpt_finish_smem() {
    return sizeof(float) * ((size_t)DK * (DV / kCkptSplit) + 2 * (size_t)C * DK + (size_t)C * (DV / kCkptSplit) + C);
}

template <typename T, int DK, int DV>
cudaError_t launch_extend_t(const ExtendArgs& p, cudaStream_t s) {
    cudaError_t e;
    mark_launch(s, 0);
    chunk_map_kernel<<<1, 1024, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark_launch(s, 1);
    if (p.ck_idx) {  // the conv windows at the checkpoint boundaries, before the conv-state update
        ckpt_conv_kernel<T><<<dim3(p.N, (p.d.conv_dim + 255) / 256), 256, 0, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // segment by segment: the per-chunk step on `s`; the state pass of segment k on the side stream
    // once the per-chunk step has finished segment k, alongside the per-chunk step of segment k+1
    SideStream* side = nullptr;
    if ((e = side_stream(&side)) != cudaSuccess) return e;
    for (int k = 0; k < p.nseg; ++k) {
        if ((e = launch_chunk<T, DK, DV>(p, k, s)) != cudaSuccess) return e;
        if ((e = cudaEventRecord(side->seg[k], s)) != cudaSuccess) return e;
        if ((e = cudaStreamWaitEvent(side->s, side->seg[k], 0)) != cudaSuccess) return e;
        if (k == 0) mark_launch(side->s, 6);
        if ((e = launch_state<T, DK, DV>(p, k, side->s)) != cudaSuccess) return e;
    }
    mark_launch(s, 2);
    // the new conv windows, once every chunk has staged the windows its sequence started from
    conv_tail_kernel<T><<<dim3(p.N, (p.d.conv_dim + 255) / 256), 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark_launch(s, 3);
    mark_launch(side->s, 7);
    if (p.ck_idx) {  // the checkpoint states off the chunk edges, once the state pass stored the edges
        constexpr size_t shm = ckpt_finish_smem<DK, DV>();
        if ((e = cudaFuncSetAttribute(ckpt_finish_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)shm)) != cudaSuccess)
            return e;
        ckpt_finish_kernel<DK, DV><<<dim3(p.N, p.d.HV, kCkptSplit), 256, shm, side->s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if ((e = cudaEventRecord(side->join, side->s)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(s, side->join, 0)) != cudaSuccess) return e;
    mark_launch(s, 5);
    return cudaSuccess;
}

}  // namespace

namespace {

// One walk over the extend workspace: the total size, and with `e` set the carved pointers.
size_t walk_extend_workspace(const LayerDims& d, int max_N, int max_T, char* base, ExtendArgs* e) {
    const size_t mc = (size_t)max_T / C + (size_t)max_N + 1;  // chunk capacity
    const size_t units = mc * d.HV;                           // (chunk, value head) units
    size_t off = kHeaderBytes;
    auto take = [&](size_t bytes) {
        char* ptr = base ? base + off : nullptr;
        off += (bytes + 255) & ~(size_t)255;
        return ptr;
    };
    char* chunk_tab = take(mc * sizeof(int4));
    char* seq_chunk0 = take(((size_t)max_N + 1) * sizeof(int32_t));
    char* seq_order = take((size_t)max_N * sizeof(int32_t));
    char* rank_off = take(((size_t)max_N + 1) * sizeof(int32_t));
    char* chunk_list = take(mc * sizeof(int32_t));
    char* kq = take(mc * d.HK * 2 * C * d.dk * sizeof(uint16_t));
    char* w = take(units * C * d.dk * sizeof(uint16_t));
    char* u = take(units * d.dv * C * sizeof(uint16_t));
    char* aq = take(units * C * C * sizeof(uint16_t));
    char* gv = take(units * C * sizeof(float4));
    if (e) {
        e->max_chunks = (int)mc;
        e->hdr = reinterpret_cast<int32_t*>(base);
        e->chunk_tab = reinterpret_cast<int4*>(chunk_tab);
        e->seq_chunk0 = reinterpret_cast<int32_t*>(seq_chunk0);
        e->seq_order = reinterpret_cast<int32_t*>(seq_order);
        e->rank_off = reinterpret_cast<int32_t*>(rank_off);
        e->chunk_list = reinterpret_cast<int32_t*>(chunk_list);
        e->KQ = reinterpret_cast<uint16_t*>(kq);
        e->W = reinterpret_cast<uint16_t*>(w);
        e->U = reinterpret_cast<uint16_t*>(u);
        e->AQ = reinterpret_cast<uint16_t*>(aq);
        e->GV = reinterpret_cast<float4*>(gv);
    }
    return off;
}

}  // namespace

size_t extend_workspace_bytes(const LayerDims& d, int max_N, int max_T, int* max_chunks_out) {
    if (max_chunks_out) *max_chunks_out = (int)((size_t)max_T / C + (size_t)max_N + 1);
    return walk_extend_workspace(d, max_N, max_T, nullptr, nullptr);
}

void carve_extend_workspace(ExtendArgs& e, void* ws, int max_N, int max_T) {
    walk_extend_workspace(e.d, max_N, max_T, static_cast<char*>(ws), &e);
}

cudaError_t launch_extend(const ExtendArgs& p, int dtype, cudaStream_t s) {
    if (dtype == GDN_DTYPE_BF16) GDN_DISPATCH_DIMS(__nv_bfloat16, launch_extend_t, p, s);
    GDN_DISPATCH_DIMS(float, launch_extend_t, p, s);
}

}  // namespace gdn
