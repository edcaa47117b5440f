// Serial inter-chunk state pass of the chunked GDN prefill on tcgen05 tensor
// cores (sm_100a), with the chunk outputs.
//
// One CTA per (sequence, value head), looping over the sequence's chunks.  The
// products are formed transposed, with the value dimension (dv) as the MMA's
// M, so that every shared-memory operand is K-major and every accumulator row
// belongs to one thread:
//
//   [X^T | O^T]  = S^T [W ; Qg]^T           M=dv N=128 K=dk   (X = W S, O = Qg S)
//   V'^T         = U^T - X^T                 CUDA cores, per thread row j
//   O^T         += V'^T Aqk^T                M=dv N=64  K=64
//   S^T         <- e^{gamma_n} S^T + V'^T K~ M=dv N=dk  K=64  (K~ = diag(e^{gamma_n-gamma}) K)
//
// where Qg = diag(e^gamma) Q (q carries the output scale).  The fp32 state
// S^T lives in tensor memory (the MMA accumulates onto it in fp32); a tf32
// copy in shared memory is the operand of the next chunk.  Eight warps: the
// two warps of a TMEM sub-partition share its 32 accumulator rows and take
// one half of the columns each.  The intra-chunk
// kernel wrote [W ; Qg], Aqk and K~^T already as tf32 tiles in the tensor
// core's shared-memory layout; they arrive by asynchronous bulk copies, each
// reissued for the next chunk as soon as the MMA that reads it has finished,
// so the copies overlap the rest of the chunk.  U (fp32) is read per thread.

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;  // 8 warps: two per TMEM sub-partition, each taking half of the columns

template <int DK, int DV>
struct StateTcSmem {
    float st[DV * DK];     // S^T tile, K-major: DV rows x DK (tf32 copy of the state)
    float wq[2 * C * DK];  // [W ; Qg] tile (bulk copy), K-major: 128 rows x DK
    float aq[C * C];       // Aqk tile (bulk copy), K-major: C rows (r) x C (s)
    float kt[DK * C];      // K~^T tile (bulk copy), K-major: DK rows (i) x C (s)
    float vt[DV * C];      // V'^T tile, K-major: DV rows (j) x C (s)
    float gam[C];
    unsigned long long bar_mma, bar_wq, bar_ak;
    uint32_t tmem_base;
};

__device__ __forceinline__ void store_f4(float* tile, uint32_t off, float4 v) {
    *reinterpret_cast<float4*>(reinterpret_cast<char*>(tile) + off) = v;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Writes 16 consecutive fp32 values of S^T row j (columns c0..c0+15) into the
// K-major tf32 operand tile.
template <int DK, int DV>
__device__ __forceinline__ void put_st_row(float* st, int j, int c0, const float (&v)[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
        store_f4(st, tc::kmajor_off(j, c0 + 4 * q, DV),
                 make_float4(tc::round_tf32(v[4 * q]), tc::round_tf32(v[4 * q + 1]), tc::round_tf32(v[4 * q + 2]),
                             tc::round_tf32(v[4 * q + 3])));
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, 1) state_tc_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    const LayerDims& d = p.d;
    const int HV = d.HV;
    // all heads of the longest sequence first, then the next longest, ...
    const int h = blockIdx.x % HV, nseq = p.seq_order[blockIdx.x / HV];
    const int len = p.cu[nseq + 1] - p.cu[nseq];
    if (len == 0) return;
    const int slot = p.slots[nseq];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    T* out = reinterpret_cast<T*>(p.out);
    if (slot < 0 || slot >= p.P) {
        if (slot >= p.P && tid == 0 && h == 0) raise_error(p.hdr, GDN_DEVERR_SLOT_RANGE);
        for (int e = tid; e < len * DV; e += NT)
            out[((size_t)(p.cu[nseq] + e / DV) * HV + h) * DV + e % DV] = from_f<T>(0.f);
        return;
    }
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StateTcSmem<DK, DV>& sm = *reinterpret_cast<StateTcSmem<DK, DV>*>(smem_raw);
    const uint32_t bar_mma = tc::smem_u32(&sm.bar_mma), bar_wq = tc::smem_u32(&sm.bar_wq),
                   bar_ak = tc::smem_u32(&sm.bar_ak);
    constexpr uint32_t WQ_BYTES = 2 * C * DK * 4, AQ_BYTES = C * C * 4, KT_BYTES = DK * C * 4;
    const int c_begin = p.seq_chunk0[nseq], c_end = p.seq_chunk0[nseq + 1];
    auto fetch_wq = [&](int id) {
        tc::mbar_expect_tx(bar_wq, WQ_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.wq), p.WQ + ((size_t)id * HV + h) * (2 * C * DK), WQ_BYTES, bar_wq);
    };
    auto fetch_ak = [&](int id) {
        tc::mbar_expect_tx(bar_ak, AQ_BYTES + KT_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.aq), p.AQ + ((size_t)id * HV + h) * (C * C), AQ_BYTES, bar_ak);
        tc::bulk_g2s(tc::smem_u32(sm.kt), p.KT + ((size_t)id * HV + h) * (DK * C), KT_BYTES, bar_ak);
    };
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 256);
    if (tid == 0) {
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_wq, 1);
        tc::mbar_init(bar_ak, 1);
        tc::fence_mbar_init();
        fetch_wq(c_begin);
        fetch_ak(c_begin);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    const uint32_t tXO = tm, tS = tm + 128;  // [X^T | O^T] (128 columns), S^T (DK columns)
    const int sp = warp & 3, half = warp >> 2;  // TMEM sub-partition, column half
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    // this thread's accumulator row j (the value-dimension index)
    const bool rowv = DV == 128 || lane < 16;
    const int j = DV == 128 ? sp * 32 + lane : sp * 16 + lane;

    // initial state: S^T row j = column j of S
    const bool init = p.has_init ? p.has_init[nseq] != 0 : true;
    float* Sg = p.ssm_state + ((size_t)slot * HV + h) * DK * DV;
#pragma unroll
    for (int cc = 0; cc < DK / 2; cc += 16) {
        const int c0 = half * (DK / 2) + cc;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = (init && rowv) ? Sg[(size_t)(c0 + i) * DV + j] : 0.f;
        tmem_st16(tS + lane_base + c0, v);
        if (rowv) put_st_row<DK, DV>(sm.st, j, c0, v);
    }
    tmem_st_wait();
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    uint32_t ph_mma = 0;
    bool ok = true;
    // gamma of the next chunk, loaded one chunk ahead so no global load sits before an MMA issue
    float g_next = tid < C ? p.gam[((size_t)c_begin * HV + h) * C + tid] : 0.f;
    for (int id = c_begin; id < c_end; ++id) {
        const uint32_t ph_ld = (uint32_t)(id - c_begin) & 1u;
        const int4 ch = p.chunk_tab[id];
        const int t0 = ch.y, n = ch.z;
        const size_t ch_h = (size_t)id * HV + h;
        if (tid < C) {
            sm.gam[tid] = g_next;
            if (id + 1 < c_end) g_next = p.gam[(ch_h + HV) * C + tid];
        }
        // U column j of this chunk, rows of this warp's half (consumed after the first MMA)
        float u[C / 2];
        {
            const float* Ug = p.U + ch_h * (C * DV) + (size_t)half * (C / 2) * DV;
#pragma unroll
            for (int s = 0; s < C / 2; ++s) u[s] = rowv ? Ug[(size_t)s * DV + j] : 0.f;
        }
        bool okw = true;
        if (tid == 0) {
            okw = tc::mbar_wait(bar_wq, ph_ld);
            if (okw) {  // [X^T | O^T] = S^T [W ; Qg]^T
                const uint32_t a = tc::smem_u32(sm.st), b = tc::smem_u32(sm.wq);
                constexpr uint32_t idesc = tc::idesc_tf32(DV, 128);
#pragma unroll
                for (int s = 0; s < DK / 8; ++s)
                    tc::mma_tf32(tXO, tc::desc_kmajor(a, DV, s), tc::desc_kmajor(b, 2 * C, s), idesc, s > 0);
                tc::mma_commit(bar_mma);
            }
        }
        ok = __syncthreads_and(okw);
        if (!ok) break;
        ok = __syncthreads_and(tc::mbar_wait(bar_mma, ph_mma));
        ph_mma ^= 1;
        if (!ok) break;
        tc::fence_after_sync();
        if (tid == 0 && id + 1 < c_end) fetch_wq(id + 1);  // the [W ; Qg] tile is free again
        const float egl = expf(sm.gam[n - 1]);
        // V'^T row j = U^T row j - X^T row j; the fp32 state is scaled by e^{gamma_n}
#pragma unroll
        for (int cc = 0; cc < C / 2; cc += 16) {
            const int c0 = half * (C / 2) + cc;
            float x[16];
            tc::tmem_ld16(tXO + lane_base + c0, x);
            tc::tmem_ld_wait();
            if (rowv)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    store_f4(sm.vt, tc::kmajor_off(j, c0 + 4 * q, DV),
                             make_float4(tc::round_tf32(u[cc + 4 * q] - x[4 * q]),
                                         tc::round_tf32(u[cc + 4 * q + 1] - x[4 * q + 1]),
                                         tc::round_tf32(u[cc + 4 * q + 2] - x[4 * q + 2]),
                                         tc::round_tf32(u[cc + 4 * q + 3] - x[4 * q + 3])));
        }
#pragma unroll
        for (int cc = 0; cc < DK / 2; cc += 16) {
            const int c0 = half * (DK / 2) + cc;
            float v[16];
            tc::tmem_ld16(tS + lane_base + c0, v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= egl;
            tmem_st16(tS + lane_base + c0, v);
        }
        tmem_st_wait();
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        bool oka = true;
        if (tid == 0) {
            oka = tc::mbar_wait(bar_ak, ph_ld);
            if (oka) {  // O^T += V'^T Aqk^T ;  S^T += V'^T K~
                const uint32_t av = tc::smem_u32(sm.vt), bq = tc::smem_u32(sm.aq), bk = tc::smem_u32(sm.kt);
                constexpr uint32_t io = tc::idesc_tf32(DV, 64), is = tc::idesc_tf32(DV, DK);
#pragma unroll
                for (int s = 0; s < C / 8; ++s)
                    tc::mma_tf32(tXO + 64, tc::desc_kmajor(av, DV, s), tc::desc_kmajor(bq, C, s), io, true);
#pragma unroll
                for (int s = 0; s < C / 8; ++s)
                    tc::mma_tf32(tS, tc::desc_kmajor(av, DV, s), tc::desc_kmajor(bk, DK, s), is, true);
                tc::mma_commit(bar_mma);
            }
        }
        ok = __syncthreads_and(oka);
        if (!ok) break;
        ok = __syncthreads_and(tc::mbar_wait(bar_mma, ph_mma));
        ph_mma ^= 1;
        if (!ok) break;
        tc::fence_after_sync();
        if (tid == 0 && id + 1 < c_end) fetch_ak(id + 1);  // the Aqk and K~^T tiles are free again
        // outputs: O^T row j is staged as column j of O [C][DV] in the (now free) V'^T tile, then the
        // chunk's rows leave as 16-byte vectors
        T* ostage = reinterpret_cast<T*>(sm.vt);
#pragma unroll
        for (int cc = 0; cc < C / 2; cc += 16) {
            const int c0 = half * (C / 2) + cc;
            float o[16];
            tc::tmem_ld16(tXO + lane_base + 64 + c0, o);
            tc::tmem_ld_wait();
            if (rowv)
#pragma unroll
                for (int i = 0; i < 16; ++i) ostage[(c0 + i) * DV + j] = from_f<T>(o[i]);
        }
#pragma unroll
        for (int cc = 0; cc < DK / 2; cc += 16) {
            const int c0 = half * (DK / 2) + cc;
            float v[16];
            tc::tmem_ld16(tS + lane_base + c0, v);
            tc::tmem_ld_wait();
            if (rowv) put_st_row<DK, DV>(sm.st, j, c0, v);
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        {
            constexpr int VPR = DV * (int)sizeof(T) / 16;  // 16-byte vectors per output row
            for (int e = tid; e < n * VPR; e += NT) {
                const int r = e / VPR, v = e % VPR;
                reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * HV + h) * DV)[v] =
                    reinterpret_cast<const uint4*>(ostage + r * DV)[v];
            }
        }
    }
    if (ok) {  // final state: column j of S
#pragma unroll
        for (int cc = 0; cc < DK / 2; cc += 16) {
            const int c0 = half * (DK / 2) + cc;
            float v[16];
            tc::tmem_ld16(tS + lane_base + c0, v);
            tc::tmem_ld_wait();
            if (rowv)
#pragma unroll
                for (int i = 0; i < 16; ++i) Sg[(size_t)(c0 + i) * DV + j] = v[i];
        }
    } else if (tid == 0) {
        raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
        // let copies already in flight land before the CTA's shared memory goes away
        tc::mbar_wait(bar_wq, 0, 100000000ull);
        tc::mbar_wait(bar_wq, 1, 100000000ull);
        tc::mbar_wait(bar_ak, 0, 100000000ull);
        tc::mbar_wait(bar_ak, 1, 100000000ull);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 256);
}

}  // namespace

template <typename T, int DK, int DV>
cudaError_t launch_state_head(const ExtendArgs& p, cudaStream_t s) {
    const size_t shm = sizeof(StateTcSmem<DK, DV>);
    cudaError_t e =
        cudaFuncSetAttribute(state_tc_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    state_tc_kernel<T, DK, DV><<<(unsigned)p.N * (unsigned)p.d.HV, NT, shm, s>>>(p);
    return cudaGetLastError();
}

// One CTA per (sequence, head) runs each head's chunks with the whole value
// dimension; the sliced kernel spends four times the MMA instructions on the
// same work (a tcgen05 MMA costs about the same few dozen cycles whatever its
// N), so it only pays when the per-head grid leaves most SMs idle: when the
// sliced grid still fits in one wave, the slices shorten each sequence's
// serial chain instead.
template <typename T, int DK, int DV>
cudaError_t launch_state(const ExtendArgs& p, cudaStream_t s) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if ((long long)p.N * p.d.HV * kStateSlices <= (long long)sms) return launch_state_slice<T, DK, DV>(p, s);
    return launch_state_head<T, DK, DV>(p, s);
}

#define GDN_STATE_INST(T)                                                        \
    template cudaError_t launch_state<T, 64, 64>(const ExtendArgs&, cudaStream_t);   \
    template cudaError_t launch_state<T, 64, 128>(const ExtendArgs&, cudaStream_t);  \
    template cudaError_t launch_state<T, 128, 64>(const ExtendArgs&, cudaStream_t);  \
    template cudaError_t launch_state<T, 128, 128>(const ExtendArgs&, cudaStream_t);
GDN_STATE_INST(float)
GDN_STATE_INST(__nv_bfloat16)

}  // namespace gdn
