// Mamba2 SSD chunk scan (page "flashinfer.mamba.ssd_combined_fwd") on tcgen05
// tensor cores (sm_100a): one CTA per (sequence, head) walks the sequence in
// chunks of up to C = 64 rows, carrying the state h (P x N, fp32) in registers.
//
// In a chunk with processed steps d_r, gamma_r = sum_{q<=r} d_q A (rows r of the
// chunk) and the state h_in it starts from:
//
//     y_r   = sum_{s<=r} e^{gamma_r - gamma_s} d_s (C_r . B_s) x_s + e^{gamma_r} h_in C_r
//     h_out = e^{gamma_last} h_in + sum_s e^{gamma_last - gamma_s} d_s x_s B_s^T
//
// evaluated with four fp16 products, fp32 accumulators in tensor memory:
//
//   Gm     = C B^T             M=64 (r)  N=64 (s)  K=N   C and B rows K-major
//   Z      = C h_in^T          M=64 (r)  N=P       K=N   h^T rows read MN-major
//   Hnew^T = B^T Xw            M=N       N=P       K=64  B and Xw rows read MN-major
//            (Xw = diag(d e^{gamma_last - gamma}) X)
//   Y      = Lm X              M=64 (r)  N=P       K=64  X rows read MN-major
//            (Lm[r,s] = e^{gamma_r - gamma_s} d_s Gm[r,s] for s <= r, else 0)
//
// (C and B are exact in fp16, so Gm is exact up to fp32 accumulation; the step
// d enters only through the rounded Lm and Xw.)
//
// then h_out^T = e^{gamma_last} h_in^T + Hnew^T in registers (thread row n of
// h^T) and y_r = Y_r + e^{gamma_r} Z_r, plus the skip term D x_r and the gate
// silu(z_r) (staged in fp32 with the chunk's rows).  Decays are powers of two
// of base-2 cumulative sums (ex2.approx).  The first three products depend only on the chunk's inputs and
// on h_in, so they are issued together; Y follows once Lm is formed.
//
// A state checkpoint inside a chunk is taken by ending the chunk at the
// boundary: chunks are cut at every 64 rows and at the checkpoint row, so the
// state after the boundary's chunk is the checkpoint.
//
// The M = 64 accumulators keep row r in lane 16 (r / 16) + r % 16 of
// sub-partition r / 16, i.e. lanes 0-15 of each warp's 32.

#include <cuda_fp16.h>

#include "../../include/ssd.h"
#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int SC = 64;   // chunk rows
constexpr int SP = 64;   // head dim P
constexpr int SNT = 128; // threads: four warps, one per tensor-memory sub-partition

struct SsdArgs {
    int H, G, T, Nseq;
    int softplus, d_per_dim;
    float dt_lo, dt_hi;
    const __nv_bfloat16* x;
    const __nv_bfloat16* dt;
    const float* A;
    const __nv_bfloat16* B;
    const __nv_bfloat16* C;
    const __nv_bfloat16* D;
    const __nv_bfloat16* z;
    const float* dt_bias;
    const int32_t* cu;
    const int32_t* order;  // sequences, longest first
    const void* init;
    void* fin;
    const int32_t* ck_idx;
    const int32_t* ck_row;
    void* ck;
    int num_ck;
    __nv_bfloat16* out;
    int32_t* hdr;
};

template <int N>
struct SsdSmem {
    uint16_t ct[SC * N];   // C rows r x N, 16-bit K-major layout (R = 64)
    uint16_t bt[SC * N];   // B rows s x N, same layout
    uint16_t xt[SC * SP];  // X rows s x P
    uint16_t xw[SC * SP];  // Xw rows s x P
    uint16_t lm[SC * SC];  // Lm rows r x s
    uint16_t ht[N * SP];   // fp16 copy of h^T: rows n x P (R = N)
    __nv_bfloat16 xs[SC][SP + 8];  // the chunk's x rows (bf16) and gates silu(z) (fp32), rows padded by
    float zs[SC][SP + 4];          // 16 bytes so that the threads reading one row each spread over the banks
    // per chunk, double-buffered (the next chunk's are formed while this one's products run):
    float g2[2][SC];       // gamma_r log2(e) (rows past the chunk repeat the last row's)
    float dd[2][SC];       // processed step d_r (0 past the chunk)
    float wl[2][SC];       // d_s e^{gamma_last - gamma_s}
    unsigned long long bar1, bar2;
    uint32_t tmem_base;
};

__device__ __forceinline__ float ld_state(const float* p) { return *p; }
__device__ __forceinline__ float ld_state(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld_state(const __half* p) { return __half2float(*p); }
__device__ __forceinline__ void st_state(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_state(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void st_state(__half* p, float v) { *p = __float2half_rn(v); }

// eight bf16 (one 16-byte vector) as floats
__device__ __forceinline__ void bf16x8(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 f16x8(const float* f) {
    return make_uint4(tc::pack_f16(f[0], f[1]), tc::pack_f16(f[2], f[3]), tc::pack_f16(f[4], f[5]),
                      tc::pack_f16(f[6], f[7]));
}

__device__ __forceinline__ uint4 bf16x8_out(const float* f) {
    uint4 r;
    uint32_t* w = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return r;
}

__device__ __forceinline__ void st16(uint16_t* tile, uint32_t off, const uint4& v) {
    *reinterpret_cast<uint4*>(reinterpret_cast<char*>(tile) + off) = v;
}

// processed step of a raw step dt of head h: clamp(softplus?(dt + dt_bias), lo, hi)
__device__ __forceinline__ float ssd_step(const SsdArgs& p, float dt, int h) {
    float v = dt + (p.dt_bias ? p.dt_bias[h] : 0.f);
    if (p.softplus) v = v > 20.f ? v : log1pf(expf(v));
    return fminf(fmaxf(v, p.dt_lo), p.dt_hi);
}

template <typename TS, int N>
__global__ void __launch_bounds__(SNT, 2) ssd_scan_kernel(SsdArgs p) {
    const int seq = p.order[blockIdx.x / p.H], h = blockIdx.x % p.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = h / (p.H / p.G);
    const int s0 = p.cu[seq], s1 = p.cu[seq + 1];
    if (s0 < 0 || s1 < s0 || s1 > p.T) {
        if (tid == 0 && h == 0) raise_error(p.hdr, GDN_DEVERR_SEQLENS);
        return;
    }
    constexpr size_t SS = (size_t)SP * N;  // elements of one state
    int ck_b = -1;                         // this sequence's checkpoint boundary (absolute row), or -1
    TS* ck_dst = nullptr;
    if (p.ck_idx) {
        const int b = p.ck_idx[seq], r = p.ck_row[seq];
        if (b >= 0 && r >= 0) {
            if (b < s0 || b > s1 || r >= p.num_ck) {
                if (tid == 0 && h == 0) raise_error(p.hdr, GDN_DEVERR_CKPT_RANGE);
            } else {
                ck_b = b;
                ck_dst = reinterpret_cast<TS*>(p.ck) + ((size_t)r * p.H + h) * SS;
            }
        }
    }
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SsdSmem<N>& sm = *reinterpret_cast<SsdSmem<N>*>(smem_raw);
    const uint32_t bar1 = tc::smem_u32(&sm.bar1), bar2 = tc::smem_u32(&sm.bar2);
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 256);
    if (tid == 0) {
        tc::mbar_init(bar1, 1);
        tc::mbar_init(bar2, 1);
        tc::fence_mbar_init();
    }
    // this thread's row n of h^T (all 128 lanes when N = 128; lanes 0-15 of each warp in the
    // M = 64 layout when N = 64) and row r of the M = 64 accumulators (lanes 0-15)
    const bool srow = N == 128 || lane < 16;
    const int n = N == 128 ? tid : 16 * warp + (lane & 15);
    const int r_own = 16 * warp + (lane & 15);
    float hs[SP];
    {
        const TS* ini = p.init ? reinterpret_cast<const TS*>(p.init) + ((size_t)seq * p.H + h) * SS : nullptr;
#pragma unroll
        for (int q = 0; q < SP; ++q) hs[q] = (ini && srow) ? ld_state(ini + (size_t)q * N + n) : 0.f;
    }
    auto put_ht = [&]() {  // fp16 copy of row n of h^T, the B operand of the next Z
        if (srow)
#pragma unroll
            for (int q = 0; q < SP; q += 8) st16(sm.ht, tc::kmajor_off16(n, q, N), f16x8(&hs[q]));
    };
    auto put_state = [&](TS* dst) {  // column n of h into a [P, N] state
        if (srow)
#pragma unroll
            for (int q = 0; q < SP; ++q) st_state(dst + (size_t)q * N + n, hs[q]);
    };
    if (ck_b == s0) put_state(ck_dst);
    put_ht();
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    const uint32_t tG = tm, tZ = tm + 64, tS = tm + 128, tY = tm + 192;  // 64 columns each
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float Ah2 = p.A[h] * 1.4426950408889634f;  // A log2(e): decays are formed as powers of two
    const float Dh = (p.D && !p.d_per_dim) ? __bfloat162float(p.D[h]) : 0.f;
    constexpr uint32_t iG = tc::idesc_f16(SC, SC), iZ = tc::idesc_f16(SC, SP) | tc::kTransposeB,
                       iH = tc::idesc_f16(N, SP) | tc::kTransposeA | tc::kTransposeB;

    // the next chunk's rows, fetched into registers one chunk ahead: thread j of each group of eight
    // takes row 8 rg + j of one 16-byte column block, so that a warp reads 64 contiguous bytes of
    // each of 8 rows and eight consecutive threads later store one 128-byte core-matrix block
    constexpr int NBX = SP / 8, NBB = N / 8, KX = SC * NBX / SNT, KB = SC * NBB / SNT;
    uint4 rx[KX], rz[KX], rb[KB], rc[KB];
    // (warp 0) raw steps of rows lane and lane + 32, held as loaded (nothing waits for the loads until
    // the next chunk's step phase)
    __nv_bfloat16 rdt0 = __float2bfloat16(0.f), rdt1 = __float2bfloat16(0.f);
    auto chunk_len = [&](int t0) {  // up to 64 rows, cut at the checkpoint boundary
        int len = min(SC, s1 - t0);
        if (ck_b > t0 && ck_b < t0 + len) len = ck_b - t0;
        return len;
    };
    auto fetch = [&](int t0, int len) {
#pragma unroll
        for (int k = 0; k < KX; ++k) {
            const int e = tid + k * SNT, j = e & 7, cb = (e >> 3) % NBX, r = ((e >> 3) / NBX) * 8 + j;
            rx[k] = rz[k] = make_uint4(0u, 0u, 0u, 0u);
            if (r < len) {
                const size_t o = ((size_t)(t0 + r) * p.H + h) * SP + cb * 8;
                rx[k] = __ldcs(reinterpret_cast<const uint4*>(p.x + o));
                if (p.z) rz[k] = __ldcs(reinterpret_cast<const uint4*>(p.z + o));
            }
        }
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            const int e = tid + k * SNT, j = e & 7, cb = (e >> 3) % NBB, r = ((e >> 3) / NBB) * 8 + j;
            rb[k] = rc[k] = make_uint4(0u, 0u, 0u, 0u);
            if (r < len) {  // B and C rows are shared by the group's heads: kept in L2
                const size_t o = ((size_t)(t0 + r) * p.G + g) * N + cb * 8;
                rb[k] = __ldg(reinterpret_cast<const uint4*>(p.B + o));
                rc[k] = __ldg(reinterpret_cast<const uint4*>(p.C + o));
            }
        }
        if (warp == 0) {
            if (lane < len) rdt0 = p.dt[(size_t)(t0 + lane) * p.H + h];
            if (lane + 32 < len) rdt1 = p.dt[(size_t)(t0 + lane + 32) * p.H + h];
        }
    };
    // (warp 0) processed steps and in-chunk cumulative decay of a chunk of `ln` rows (rows lane and
    // lane + 32) into step buffer sb, from the raw steps fetched with its rows
    auto form_steps = [&](int sb, int ln) {
        const float d0 = lane < ln ? ssd_step(p, __bfloat162float(rdt0), h) : 0.f;
        const float d1 = lane + 32 < ln ? ssd_step(p, __bfloat162float(rdt1), h) : 0.f;
        float c0 = d0 * Ah2, c1 = d1 * Ah2;  // base-2 exponents
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v0 = __shfl_up_sync(0xffffffffu, c0, o), v1 = __shfl_up_sync(0xffffffffu, c1, o);
            if (lane >= o) {
                c0 += v0;
                c1 += v1;
            }
        }
        c1 += __shfl_sync(0xffffffffu, c0, 31);
        const float gl = __shfl_sync(0xffffffffu, c1, 31);  // rows past the chunk add nothing
        sm.g2[sb][lane] = c0;
        sm.g2[sb][lane + 32] = c1;
        sm.dd[sb][lane] = d0;
        sm.dd[sb][lane + 32] = d1;
        sm.wl[sb][lane] = d0 * tc::ex2_approx(gl - c0);
        sm.wl[sb][lane + 32] = d1 * tc::ex2_approx(gl - c1);
    };
    int len = s0 < s1 ? chunk_len(s0) : 0;
    if (len > 0) fetch(s0, len);
    if (len > 0 && warp == 0) form_steps(0, len);

    bool ok = true, okw = true;
    uint32_t ph = 0;
    for (int t0 = s0; t0 < s1; ph ^= 1u) {
        const int cur = (int)ph;  // this chunk's step buffer
        ok = __syncthreads_and(okw) != 0;  // (also: the previous chunk's outputs are all read)
        if (!ok) break;
        // ---- the fetched rows into the fp16 operand tiles (zero past the chunk) and the bf16
        // staging rows of x and z for the outputs
#pragma unroll
        for (int k = 0; k < KX; ++k) {
            const int e = tid + k * SNT, j = e & 7, cb = (e >> 3) % NBX, r = ((e >> 3) / NBX) * 8 + j;
            float f[8];
            bf16x8(rx[k], f);
            const uint32_t off = tc::kmajor_off16(r, cb * 8, SC);
            st16(sm.xt, off, f16x8(f));
            const float w = sm.wl[cur][r];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] *= w;
            st16(sm.xw, off, f16x8(f));
            *reinterpret_cast<uint4*>(&sm.xs[r][cb * 8]) = rx[k];
            if (p.z) {  // the gate silu(z) = z / (1 + e^{-z})
                bf16x8(rz[k], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fdividef(f[i], 1.f + __expf(-f[i]));
                *reinterpret_cast<float4*>(&sm.zs[r][cb * 8]) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4*>(&sm.zs[r][cb * 8 + 4]) = make_float4(f[4], f[5], f[6], f[7]);
            }
        }
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            const int e = tid + k * SNT, j = e & 7, cb = (e >> 3) % NBB, r = ((e >> 3) / NBB) * 8 + j;
            float f[8];
            const uint32_t off = tc::kmajor_off16(r, cb * 8, SC);
            bf16x8(rb[k], f);
            st16(sm.bt, off, f16x8(f));
            bf16x8(rc[k], f);
            st16(sm.ct, off, f16x8(f));
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0) {  // Gm = C B^T, Z = C h_in^T, Hnew^T = B^T Xw
            const uint32_t ct = tc::smem_u32(sm.ct), bt = tc::smem_u32(sm.bt), xw = tc::smem_u32(sm.xw),
                           ht = tc::smem_u32(sm.ht);
#pragma unroll
            for (int k = 0; k < N / 16; ++k)
                tc::mma_f16(tG, tc::desc_kmajor(ct, SC, k), tc::desc_kmajor(bt, SC, k), iG, k > 0);
#pragma unroll
            for (int k = 0; k < N / 16; ++k)
                tc::mma_f16(tZ, tc::desc_kmajor(ct, SC, k), tc::desc_mnmajor16(ht, N, k), iZ, k > 0);
#pragma unroll
            for (int k = 0; k < SC / 16; ++k)
                tc::mma_f16(tS, tc::desc_mnmajor16(bt, SC, k), tc::desc_mnmajor16(xw, SC, k), iH, k > 0);
            tc::mma_commit(bar1);
        }
        // the next chunk's rows load (into the registers this chunk's staging has just emptied) while
        // this chunk's products, state update and outputs run; warp 0 forms its steps meanwhile
        const int t0n = t0 + len, lenn = t0n < s1 ? chunk_len(t0n) : 0;
        if (lenn > 0) fetch(t0n, lenn);
        if (lenn > 0 && warp == 0) form_steps(cur ^ 1, lenn);
        okw = tc::mbar_wait(bar1, ph);
        tc::fence_after_sync();
        {  // h^T <- e^{gamma_last} h^T + Hnew^T
            const float egl = tc::ex2_approx(sm.g2[cur][SC - 1]);
#pragma unroll
            for (int c0 = 0; c0 < SP; c0 += 16) {
                float v[16];
                tc::tmem_ld16(tS + lane_base + c0, v);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) hs[c0 + i] = fmaf(egl, hs[c0 + i], v[i]);
            }
        }
        put_ht();
        {  // Lm row r_own: e^{gamma_r - gamma_s} d_s Gm[r, s] for s <= r
            const float gr = sm.g2[cur][r_own];
            const bool rv = lane < 16 && r_own < len;
#pragma unroll
            for (int c0 = 0; c0 < SC; c0 += 16) {
                float v[16];
                tc::tmem_ld16(tG + lane_base + c0, v);
                tc::tmem_ld_wait();
                if (lane < 16)
#pragma unroll
                    for (int q = 0; q < 16; q += 8) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int s = c0 + q + i;
                            f[i] = (rv && s <= r_own) ? v[q + i] * sm.dd[cur][s] * tc::ex2_approx(gr - sm.g2[cur][s]) : 0.f;
                        }
                        st16(sm.lm, tc::kmajor_off16(r_own, c0 + q, SC), f16x8(f));
                    }
            }
        }
        if (ck_b == t0 + len && okw) put_state(ck_dst);
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        ok = __syncthreads_and(okw) != 0;
        if (!ok) break;
        tc::fence_after_sync();
        if (tid == 0) {  // Y = Lm X
            const uint32_t lm = tc::smem_u32(sm.lm), xt = tc::smem_u32(sm.xt);
#pragma unroll
            for (int k = 0; k < SC / 16; ++k)
                tc::mma_f16(tY, tc::desc_kmajor(lm, SC, k), tc::desc_mnmajor16(xt, SC, k), iZ, k > 0);
            tc::mma_commit(bar2);
        }
        okw = tc::mbar_wait(bar2, ph);
        tc::fence_after_sync();
        {  // y_r = Y_r + e^{gamma_r} Z_r, skip term, gate
            const bool live = okw && lane < 16 && r_own < len;
            const float eg = tc::ex2_approx(sm.g2[cur][r_own]);
            const size_t row = ((size_t)(t0 + r_own) * p.H + h) * SP;
#pragma unroll
            for (int c0 = 0; c0 < SP; c0 += 16) {
                float yv[16], zv[16];
                tc::tmem_ld16(tY + lane_base + c0, yv);
                tc::tmem_ld16(tZ + lane_base + c0, zv);
                tc::tmem_ld_wait();
                if (live)
#pragma unroll
                    for (int q = 0; q < 16; q += 8) {
                        float o[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) o[i] = fmaf(eg, zv[q + i], yv[q + i]);
                        if (p.D) {
                            float xv[8], dv[8];
                            bf16x8(*reinterpret_cast<const uint4*>(&sm.xs[r_own][c0 + q]), xv);
                            if (p.d_per_dim) bf16x8(*reinterpret_cast<const uint4*>(p.D + (size_t)h * SP + c0 + q), dv);
#pragma unroll
                            for (int i = 0; i < 8; ++i) o[i] = fmaf(p.d_per_dim ? dv[i] : Dh, xv[i], o[i]);
                        }
                        if (p.z) {
                            const float4 g0 = *reinterpret_cast<const float4*>(&sm.zs[r_own][c0 + q]),
                                         g1 = *reinterpret_cast<const float4*>(&sm.zs[r_own][c0 + q + 4]);
                            o[0] *= g0.x; o[1] *= g0.y; o[2] *= g0.z; o[3] *= g0.w;
                            o[4] *= g1.x; o[5] *= g1.y; o[6] *= g1.z; o[7] *= g1.w;
                        }
                        __stcs(reinterpret_cast<uint4*>(p.out + row + c0 + q), bf16x8_out(o));
                    }
            }
        }
        t0 = t0n;
        len = lenn;
    }
    ok = __syncthreads_and(ok && okw) != 0;
    if (ok) {
        if (p.fin) put_state(reinterpret_cast<TS*>(p.fin) + ((size_t)seq * p.H + h) * SS);
    } else if (tid == 0) {
        raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
        // products still in flight finish before the tensor memory is released
        for (uint32_t par = 0; par < 2; ++par) {
            tc::mbar_wait(bar1, par, 100000000ull);
            tc::mbar_wait(bar2, par, 100000000ull);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 256);
}

// order[rank] = sequence: sequences by decreasing length (ties by index), so that the longest chains
// start first; a sequence with invalid bounds counts as empty
__global__ void ssd_order_kernel(const int32_t* cu, int nseq, int T, int32_t* order) {
    __shared__ int lens[1024];
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    auto len_of = [&](int j) {
        const int a = cu[j], b = cu[j + 1];
        return (a < 0 || b < a || b > T) ? 0 : b - a;
    };
    const int li = i < nseq ? len_of(i) : 0;
    int rank = 0;
    for (int j0 = 0; j0 < nseq; j0 += 1024) {
        __syncthreads();
        for (int j = threadIdx.x; j < 1024 && j0 + j < nseq; j += blockDim.x) lens[j] = len_of(j0 + j);
        __syncthreads();
        const int m = min(1024, nseq - j0);
        if (i < nseq)
            for (int j = 0; j < m; ++j) {
                const int lj = lens[j];
                rank += (lj > li) || (lj == li && j0 + j < i);
            }
    }
    if (i < nseq) order[rank] = i;
}

template <typename TS, int N>
cudaError_t launch_ssd(const SsdArgs& a, cudaStream_t s) {
    // at most two CTAs per SM, whose 256 tensor-memory columns each fill the SM's 512
    const size_t shm = sizeof(SsdSmem<N>) > 80 * 1024 ? sizeof(SsdSmem<N>) : 80 * 1024;
    cudaError_t e = cudaFuncSetAttribute(ssd_scan_kernel<TS, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    ssd_order_kernel<<<(a.Nseq + 255) / 256, 256, 0, s>>>(a.cu, a.Nseq, a.T, const_cast<int32_t*>(a.order));
    ssd_scan_kernel<TS, N><<<(unsigned)(a.Nseq * a.H), SNT, shm, s>>>(a);
    return cudaGetLastError();
}

template <typename TS>
cudaError_t launch_ssd_n(const SsdArgs& a, int dstate, cudaStream_t s) {
    return dstate == 128 ? launch_ssd<TS, 128>(a, s) : launch_ssd<TS, 64>(a, s);
}

bool al16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

}  // namespace
}  // namespace gdn

extern "C" GDN_API size_t ssd_workspace_size(const ssd_config_t* cfg, int32_t max_N, int32_t max_T) {
    if (!cfg || max_N < 0 || max_T < 0) return 0;
    return (size_t)gdn::kHeaderBytes + (((size_t)max_N * 4 + 15) & ~(size_t)15);  // header + sequence order
}

extern "C" GDN_API int ssd_combined_fwd(const ssd_config_t* cfg, const void* x, const void* dt, const float* A,
                                        const void* B, const void* C, const void* D, const void* z,
                                        const float* dt_bias, const int32_t* cu_seqlens, int32_t N, int32_t T,
                                        const void* initial_states, void* final_states,
                                        const int32_t* ckpt_token_indices, const int32_t* ckpt_state_slots,
                                        void* ckpt_states, int32_t num_ckpt, void* out, void* workspace,
                                        size_t workspace_bytes, gdn_stream_t stream) {
    using gdn::al16;
    if (!cfg || N < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    if (cfg->nheads <= 0 || cfg->ngroups <= 0 || cfg->nheads % cfg->ngroups != 0) return GDN_ERR_INVALID_ARG;
    if (cfg->headdim <= 0 || cfg->dstate <= 0) return GDN_ERR_INVALID_ARG;
    if (!(cfg->dt_min <= cfg->dt_max)) return GDN_ERR_INVALID_ARG;
    if (cfg->headdim != 64 || (cfg->dstate != 64 && cfg->dstate != 128)) return GDN_ERR_UNSUPPORTED;
    const int sd = cfg->state_dtype;
    if (sd != GDN_DTYPE_F32 && sd != GDN_DTYPE_BF16 && sd != GDN_DTYPE_F16) return GDN_ERR_UNSUPPORTED;
    const bool any_ck = ckpt_token_indices || ckpt_state_slots || ckpt_states;
    const bool all_ck = ckpt_token_indices && ckpt_state_slots && ckpt_states;
    if (any_ck && (!all_ck || num_ckpt < 0)) return GDN_ERR_INVALID_ARG;
    if (!workspace || !al16(workspace)) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < ssd_workspace_size(cfg, N, T)) return GDN_ERR_WORKSPACE;
    if (N == 0) return GDN_OK;
    if (!cu_seqlens || !A || !al16(cu_seqlens) || !al16(A)) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!x || !dt || !B || !C || !out)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt, B, C, D, z, dt_bias, initial_states, final_states, ckpt_token_indices,
                          ckpt_state_slots, ckpt_states, out};
    for (const void* q : ptrs)
        if (q && !al16(q)) return GDN_ERR_INVALID_ARG;
    if ((long long)N * cfg->nheads > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    gdn::SsdArgs a;
    a.H = cfg->nheads;
    a.G = cfg->ngroups;
    a.T = T;
    a.Nseq = N;
    a.softplus = cfg->dt_softplus != 0;
    a.d_per_dim = cfg->d_per_dim != 0;
    a.dt_lo = cfg->dt_min;
    a.dt_hi = cfg->dt_max;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.dt = static_cast<const __nv_bfloat16*>(dt);
    a.A = A;
    a.B = static_cast<const __nv_bfloat16*>(B);
    a.C = static_cast<const __nv_bfloat16*>(C);
    a.D = static_cast<const __nv_bfloat16*>(D);
    a.z = static_cast<const __nv_bfloat16*>(z);
    a.dt_bias = dt_bias;
    a.cu = cu_seqlens;
    a.order = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + gdn::kHeaderBytes);
    a.init = initial_states;
    a.fin = final_states;
    a.ck_idx = ckpt_token_indices;
    a.ck_row = ckpt_state_slots;
    a.ck = ckpt_states;
    a.num_ck = num_ckpt;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.hdr = static_cast<int32_t*>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (sd == GDN_DTYPE_F32) e = gdn::launch_ssd_n<float>(a, cfg->dstate, s);
    else if (sd == GDN_DTYPE_BF16) e = gdn::launch_ssd_n<__nv_bfloat16>(a, cfg->dstate, s);
    else e = gdn::launch_ssd_n<__half>(a, cfg->dstate, s);
    return e == cudaSuccess ? GDN_OK : gdn::record_cuda_failure(e);
}
