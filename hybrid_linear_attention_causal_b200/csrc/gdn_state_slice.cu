// Serial inter-chunk state pass of the chunked GDN prefill on tcgen05 tensor
// cores (sm_100a), with the chunk outputs: the variant for few, long sequences.
//
// The columns of the state S [dk x dv] evolve independently: column j of
// V' = U - W S, of O = Qg S + Aqk V' and of the update S <- e^{gamma_n} S +
// K~^T V' only involve column j of S.  So the value dimension is cut into
// slices of SW columns and each CTA runs one (sequence, value head, slice)
// through the sequence's chunks; a long sequence then keeps dv/SW SMs busy
// instead of one, and each chunk's serial latency shrinks with the slice.
//
//   [X ; O]  = [W ; Qg] S_sl               M=128 N=SW K=dk   (X = W S, O = Qg S)
//   V'       = U_sl - X                     CUDA cores, thread t owns row t
//   Snew     = K~^T V'                      M=dk  N=SW K=C    (fresh accumulator)
//   O       += Aqk V'                       M=128 N=SW K=C    (rows 64..127 of the [X ; O] tile)
//   S_sl    <- e^{gamma_n} S_sl + Snew      CUDA cores, thread i owns row i, fp32 in registers
//
// where Qg = diag(e^gamma) Q (q carries the output scale) and
// K~ = diag(e^{gamma_n - gamma}) K.  The fp32 state slice lives in registers
// (one row of S per thread); its tf32 copy, written transposed into shared
// memory, is the B operand of the next chunk's first product.  The
// intra-chunk kernel wrote [W ; Qg], Aqk and K~^T as tf32 tiles in the tensor
// core's shared-memory layout; they arrive by asynchronous bulk copies, each
// reissued for the next chunk as soon as the products that read it have
// finished.  Every CTA of a (chunk, head) reads the same tiles, so the slices
// of one head are launched next to each other and share them through L2.
//
// The Aqk product needs its result in rows 64..127 of the M=128 accumulator
// that holds O.  Its A operand is described as a 128-row K-major tile that
// starts 1 KB (one K group of the 64-row Aqk tile) before Aqk: rows 64..127
// of that view are exactly Aqk, rows 0..63 alias the previous K group (or the
// [W ; Qg] tile just before Aqk) and only land in the X rows, which are dead
// by then and overwritten by the next chunk's first product.

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NT = 128;

template <int DK, int SW>
struct StateSliceSmem {
    float wq[2 * C * DK];  // [W ; Qg] tile (bulk copy), K-major: 128 rows x DK; must precede aq
    float aq[C * C];       // Aqk tile (bulk copy), K-major: C rows (r) x C (s)
    float kt[DK * C];      // K~^T tile (bulk copy), K-major: DK rows (i) x C (s)
    float st[SW * DK];     // S_sl^T, K-major: SW rows (slice column c) x DK (i), tf32
    float vt[SW * C];      // V'^T,   K-major: SW rows (slice column c) x C (t), tf32
    unsigned long long bar_x, bar_s, bar_o, bar_wq, bar_ak;
    uint32_t tmem_base;
};

// TMEM columns: two [X ; O] accumulators (alternating chunks) and Snew
template <int SW>
__host__ __device__ constexpr uint32_t tmem_cols() {
    return 3 * SW <= 32 ? 32u : 3 * SW <= 64 ? 64u : 3 * SW <= 128 ? 128u : 256u;
}

// Writes tf32(v[c]) at (row c, column k) of a K-major tile with SW rows, for
// every c.  Thread k holds a column, so a plain loop over c would put the 32
// lanes of a warp on 4 banks; each group of 4 lanes starts its 8-column blocks
// at a different column instead (a rotation by (k/4) mod 8 done with selects),
// which spreads one store instruction over all 32 banks.
template <int SW>
__device__ __forceinline__ void put_col(float* tile, int k, const float (&v)[SW]) {
    const int g = (k >> 2) & 7;
    char* base = reinterpret_cast<char*>(tile) + (k >> 2) * (SW / 8) * 128 + (k & 3) * 4;
#pragma unroll
    for (int b = 0; b < SW / 8; ++b) {
        float r[8], t[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) r[m] = tc::round_tf32(v[8 * b + m]);
#pragma unroll
        for (int m = 0; m < 8; ++m) t[m] = (g & 1) ? r[(m + 1) & 7] : r[m];
#pragma unroll
        for (int m = 0; m < 8; ++m) r[m] = (g & 2) ? t[(m + 2) & 7] : t[m];
#pragma unroll
        for (int m = 0; m < 8; ++m) t[m] = (g & 4) ? r[(m + 4) & 7] : r[m];
        // now t[m] holds column 8b + ((m + g) & 7)
#pragma unroll
        for (int m = 0; m < 8; ++m) *reinterpret_cast<float*>(base + b * 128 + ((m + g) & 7) * 16) = t[m];
    }
}

// SW consecutive TMEM columns of this warp's 32 lanes
template <int SW>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[SW]) {
#pragma unroll
    for (int c0 = 0; c0 < SW; c0 += 16) {
        float x[16];
        tc::tmem_ld16(taddr + c0, x);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[c0 + i] = x[i];
    }
    tc::tmem_ld_wait();
}

// SW consecutive values of one output row, as 16-byte vectors
template <typename T, int SW>
__device__ __forceinline__ void store_row(T* dst, const float (&v)[SW]) {
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int q = 0; q < SW / 4; ++q)
            reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
        for (int q = 0; q < SW / 8; ++q) {
            uint4 w;
            uint32_t* pw = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 pr = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
                pw[e] = *reinterpret_cast<const uint32_t*>(&pr);
            }
            reinterpret_cast<uint4*>(dst)[q] = w;
        }
    }
}

template <int SW>
__device__ __forceinline__ void load_row(const float* src, float (&v)[SW]) {
#pragma unroll
    for (int q = 0; q < SW / 4; ++q) {
        const float4 x = reinterpret_cast<const float4*>(src)[q];
        v[4 * q] = x.x;
        v[4 * q + 1] = x.y;
        v[4 * q + 2] = x.z;
        v[4 * q + 3] = x.w;
    }
}

template <typename T, int DK, int DV, int SW>
__global__ void __launch_bounds__(NT, 1) state_slice_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    constexpr int NSL = DV / SW;
    const LayerDims& d = p.d;
    const int HV = d.HV;
    // slices of one head are adjacent in launch order, so they run together and share the tiles in L2
    const int sl = blockIdx.x % NSL, h = (blockIdx.x / NSL) % HV, nseq = p.seq_order[blockIdx.x / (NSL * HV)];
    const int j0 = sl * SW;
    const int len = p.cu[nseq + 1] - p.cu[nseq];
    if (len == 0) return;
    const int slot = p.slots[nseq];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    T* out = reinterpret_cast<T*>(p.out);
    if (slot < 0 || slot >= p.P) {
        if (slot >= p.P && tid == 0 && h == 0 && sl == 0) raise_error(p.hdr, GDN_DEVERR_SLOT_RANGE);
        for (int e = tid; e < len * SW; e += NT)
            out[((size_t)(p.cu[nseq] + e / SW) * HV + h) * DV + j0 + e % SW] = from_f<T>(0.f);
        return;
    }
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StateSliceSmem<DK, SW>& sm = *reinterpret_cast<StateSliceSmem<DK, SW>*>(smem_raw);
    const uint32_t bar_x = tc::smem_u32(&sm.bar_x), bar_s = tc::smem_u32(&sm.bar_s),
                   bar_o = tc::smem_u32(&sm.bar_o), bar_wq = tc::smem_u32(&sm.bar_wq),
                   bar_ak = tc::smem_u32(&sm.bar_ak);
    constexpr uint32_t WQ_BYTES = 2 * C * DK * 4, AQ_BYTES = C * C * 4, KT_BYTES = DK * C * 4;
    constexpr uint32_t TCOLS = tmem_cols<SW>();
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
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, TCOLS);
    if (tid == 0) {
        tc::mbar_init(bar_x, 1);
        tc::mbar_init(bar_s, 1);
        tc::mbar_init(bar_o, 1);
        tc::mbar_init(bar_wq, 1);
        tc::mbar_init(bar_ak, 1);
        tc::fence_mbar_init();
        fetch_wq(c_begin);
        fetch_ak(c_begin);
    }

    // This thread's row i of the state: i = tid for dk = 128 (M=128
    // accumulator layout: row r in TMEM lane r), i = 16 warp + lane on the
    // first 16 lanes for dk = 64 (M=64 layout: rows 16w..16w+15 in lanes 0..15
    // of sub-partition w).
    const bool own = DK == 128 || lane < 16;
    const int i_row = DK == 128 ? tid : warp * 16 + lane;
    const bool init = p.has_init ? p.has_init[nseq] != 0 : true;
    float* Sg = p.ssm_state + ((size_t)slot * HV + h) * DK * DV + j0;
    float s[SW];
    if (init && own) {
        load_row<SW>(Sg + (size_t)i_row * DV, s);
    } else {
#pragma unroll
        for (int c = 0; c < SW; ++c) s[c] = 0.f;
    }
    if (own) put_col<SW>(sm.st, i_row, s);
    // threads 0..C-1 own row t of X and V'; U row t (column t of the U^T tile), this slice's
    // columns, is loaded one chunk ahead
    float u[SW];
    auto load_u = [&](int id) {
        const char* Ut = reinterpret_cast<const char*>(p.U + ((size_t)id * HV + h) * (DV * C));
#pragma unroll
        for (int c = 0; c < SW; ++c) u[c] = *reinterpret_cast<const float*>(Ut + tc::kmajor_off(j0 + c, tid, DV));
    };
    if (tid < C) load_u(c_begin);
    int4 ch = p.chunk_tab[c_begin];
    float gl = p.gam[((size_t)c_begin * HV + h) * C + ch.z - 1];  // gamma_n of this chunk
    int4 ch_nx = c_begin + 1 < c_end ? p.chunk_tab[c_begin + 1] : ch;
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    const uint32_t tS = tm + 2 * SW;  // Snew accumulator
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    bool ok = true;
    int prev_t0 = 0, prev_n = 0;  // rows of the chunk whose outputs are still in TMEM
    for (int id = c_begin; id < c_end; ++id) {
        const uint32_t ph = (uint32_t)(id - c_begin) & 1u;
        const uint32_t tXO = tm + ph * SW;  // [X ; O] accumulator of this chunk
        // one chunk ahead: the next chunk's total decay; two ahead: the table entry
        float gl_nx = 0.f;
        int4 ch_nx2 = ch_nx;
        if (id + 1 < c_end) gl_nx = p.gam[((size_t)(id + 1) * HV + h) * C + ch_nx.z - 1];
        if (id + 2 < c_end) ch_nx2 = p.chunk_tab[id + 2];
        bool okl = true;
        if (tid == 0) {
            okl = tc::mbar_wait(bar_wq, ph);
            if (okl) {  // [X ; O] = [W ; Qg] S_sl
                const uint32_t a = tc::smem_u32(sm.wq), b = tc::smem_u32(sm.st);
                constexpr uint32_t idesc = tc::idesc_tf32(2 * C, SW);
#pragma unroll
                for (int k = 0; k < DK / 8; ++k)
                    tc::mma_tf32(tXO, tc::desc_kmajor(a, 2 * C, k), tc::desc_kmajor(b, SW, k), idesc, k > 0);
                tc::mma_commit(bar_x);
            }
        }
        // the previous chunk's outputs leave while this chunk's first product runs
        if (warp >= 2 && id > c_begin) {
            okl = __all_sync(0xffffffffu, tc::mbar_wait(bar_o, ph ^ 1u) && okl);
            if (okl) {
                tc::fence_after_sync();
                float o[SW];
                tmem_ld_cols<SW>(tm + (ph ^ 1u) * SW + lane_base, o);
                const int r = tid - C;
                if (r < prev_n) store_row<T, SW>(out + ((size_t)(prev_t0 + r) * HV + h) * DV + j0, o);
            }
        }
        okl = __all_sync(0xffffffffu, okl && tc::mbar_wait(bar_x, ph));
        tc::fence_after_sync();
        if (tid == 0 && okl && id + 1 < c_end) fetch_wq(id + 1);  // the [W ; Qg] tile is free again
        if (warp < 2 && okl) {  // V' row t = U row t - X row t
            float x[SW];
            tmem_ld_cols<SW>(tXO + lane_base, x);
#pragma unroll
            for (int c = 0; c < SW; ++c) x[c] = u[c] - x[c];
            put_col<SW>(sm.vt, tid, x);
            if (id + 1 < c_end) load_u(id + 1);
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        ok = __syncthreads_and(okl);
        if (!ok) break;
        tc::fence_after_sync();
        if (tid == 0) {
            okl = tc::mbar_wait(bar_ak, ph);
            if (okl) {
                const uint32_t aq = tc::smem_u32(sm.aq), ak = tc::smem_u32(sm.kt), bv = tc::smem_u32(sm.vt);
                {  // Snew = K~^T V'
                    constexpr uint32_t is = tc::idesc_tf32(DK, SW);
#pragma unroll
                    for (int k = 0; k < C / 8; ++k)
                        tc::mma_tf32(tS, tc::desc_kmajor(ak, DK, k), tc::desc_kmajor(bv, SW, k), is, k > 0);
                    tc::mma_commit(bar_s);
                }
                {  // O += Aqk V', through the 128-row view that starts one K group before Aqk
                    constexpr uint32_t io = tc::idesc_tf32(2 * C, SW);
                    constexpr uint32_t LBO = (C / 8) * 128;
#pragma unroll
                    for (int k = 0; k < C / 8; ++k)
                        tc::mma_tf32(tXO, tc::make_desc(aq - LBO + 2 * k * LBO, LBO, 128),
                                     tc::desc_kmajor(bv, SW, k), io, true);
                    tc::mma_commit(bar_o);
                }
            }
        }
        okl = __all_sync(0xffffffffu, okl && tc::mbar_wait(bar_s, ph));
        if (okl) {  // S_sl <- e^{gamma_n} S_sl + Snew
            tc::fence_after_sync();
            float acc[SW];
            tmem_ld_cols<SW>(tS + lane_base, acc);
            const float egl = expf(gl);
#pragma unroll
            for (int c = 0; c < SW; ++c) s[c] = fmaf(egl, s[c], acc[c]);
            if (own) put_col<SW>(sm.st, i_row, s);
        }
        if (tid == 0 && okl) {  // Aqk, K~^T and V' are free once the output product is done
            okl = tc::mbar_wait(bar_o, ph);
            if (okl && id + 1 < c_end) fetch_ak(id + 1);
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        ok = __syncthreads_and(okl);
        if (!ok) break;
        tc::fence_after_sync();
        prev_t0 = ch.y;
        prev_n = ch.z;
        ch = ch_nx;
        ch_nx = ch_nx2;
        gl = gl_nx;
    }
    if (ok) {
        if (warp >= 2) {  // the last chunk's outputs
            const uint32_t ph = (uint32_t)(c_end - 1 - c_begin) & 1u;
            const bool okw = __all_sync(0xffffffffu, tc::mbar_wait(bar_o, ph));
            if (okw) {
                tc::fence_after_sync();
                float o[SW];
                tmem_ld_cols<SW>(tm + ph * SW + lane_base, o);
                const int r = tid - C;
                if (r < prev_n) store_row<T, SW>(out + ((size_t)(prev_t0 + r) * HV + h) * DV + j0, o);
            } else if (lane == 0) {
                raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
            }
        }
        if (own) {  // final state slice
#pragma unroll
            for (int q = 0; q < SW / 4; ++q)
                reinterpret_cast<float4*>(Sg + (size_t)i_row * DV)[q] =
                    make_float4(s[4 * q], s[4 * q + 1], s[4 * q + 2], s[4 * q + 3]);
        }
    } else if (tid == 0) {
        raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
        // let copies and products already in flight finish before the CTA's
        // shared and tensor memory go away
        tc::mbar_wait(bar_wq, 0, 100000000ull);
        tc::mbar_wait(bar_wq, 1, 100000000ull);
        tc::mbar_wait(bar_ak, 0, 100000000ull);
        tc::mbar_wait(bar_ak, 1, 100000000ull);
        tc::mbar_wait(bar_o, 0, 100000000ull);
        tc::mbar_wait(bar_o, 1, 100000000ull);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, TCOLS);
}

}  // namespace

template <typename T, int DK, int DV>
cudaError_t launch_state_slice(const ExtendArgs& p, cudaStream_t s) {
    constexpr int SW = DV / kStateSlices;
    const size_t shm = sizeof(StateSliceSmem<DK, SW>);
    cudaError_t e = cudaFuncSetAttribute(state_slice_kernel<T, DK, DV, SW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)p.N * (unsigned)p.d.HV * (unsigned)(DV / SW);
    state_slice_kernel<T, DK, DV, SW><<<grid, NT, shm, s>>>(p);
    return cudaGetLastError();
}

#define GDN_STATE_INST(T)                                                        \
    template cudaError_t launch_state_slice<T, 64, 64>(const ExtendArgs&, cudaStream_t);   \
    template cudaError_t launch_state_slice<T, 64, 128>(const ExtendArgs&, cudaStream_t);  \
    template cudaError_t launch_state_slice<T, 128, 64>(const ExtendArgs&, cudaStream_t);  \
    template cudaError_t launch_state_slice<T, 128, 128>(const ExtendArgs&, cudaStream_t);
GDN_STATE_INST(float)
GDN_STATE_INST(__nv_bfloat16)

}  // namespace gdn
