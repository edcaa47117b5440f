// Intra-chunk step of the chunked GDN prefill on tcgen05 tensor cores (sm_100a).
//
// One CTA per (chunk, qk head); it serves the G value heads that share the qk
// head.  For a chunk of n <= 64 rows with normalised k_r, q_r (q carries the
// output scale), gates g_r, beta_r and gamma_r = sum_{s<=r} g_s:
//
// The prep kernel's [K ; Q] tile and the V^T tiles and gates of the value
// heads arrive by asynchronous bulk copies (two value heads in flight).
//
//   D1  = [K; Q] K^T                          (tf32 MMA, M=128 N=64 K=dk)
//   A   = beta_r e^{gamma_r-gamma_s} (k_r.k_s)        s < r   (strictly lower)
//   Aqk = e^{gamma_r-gamma_s} (q_r.k_s)               s <= r
//   T   = (I + A)^{-1}                        (fp32, 32x32 blocks: forward substitution + block products)
//   W   = T diag(beta e^gamma) K, U = T diag(beta) V   (tf32 MMAs, M=64 K=64)
//
// Both products share the A operand T diag(beta): W takes (diag(e^gamma) K)^T
// and U the V^T tile as delivered.  K^T is transposed once per CTA from the
// [K ; Q] tile and serves every value head through column scalings.
//
// (the WY/UT form of the gated delta rule).  For the serial state pass it
// writes, per (chunk, value head): the tile [W ; diag(e^gamma) Q], the Aqk
// tile and the tile (diag(e^{gamma_n-gamma}) K)^T -- tf32, already in the
// tensor core's shared-memory layout so the state pass bulk-copies them --
// plus U (fp32) and gamma.  Operands are staged in shared memory as K-major
// no-swizzle tiles rounded to tf32 (round to nearest); accumulators live in
// tensor memory.  One thread issues the MMAs; the eight warps read their
// sub-partition's 32-lane slice of tensor memory (two warps per slice, one
// half of the columns each) for the CUDA-core steps.

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;  // 8 warps; warp w reads TMEM sub-partition w % 4

template <int DK, int DV>
struct IntraTcSmem {
    float kq[2 * C * DK];  // [K ; Q*scale] tile from the prep kernel (bulk copy), K-major, 128 rows
    float kt[DK * C];      // K^T, K-major, DK rows x C (built once, shared by the value heads)
    float kte[DK * C];     // (diag(e^gamma) K)^T of the current head, same layout
    float bv[DV * C];      // V^T tile of the current head (bulk copy), K-major, DV rows x C
    float t[C * C];        // T diag(beta) as a K-major tile, C rows x C
    float a[C][C + 1];     // A (fp32)
    float tf[C][C + 1];    // T (fp32)
    float m[32][33];       // A21 T11
    float2 gb[2][C];       // (g, beta) of the two heads in flight
    float gam[C], beta[C], eg[C];
    float fkt[C];          // e^{gamma_n - gamma_s} (0 past the chunk end): column factor of K~^T
    unsigned long long bar_mma, bar_kq, bar_v, bar_g[2];
    uint32_t tmem_base;
};

__device__ __forceinline__ void store_f4(float* tile, uint32_t off, float4 v) {
    *reinterpret_cast<float4*>(reinterpret_cast<char*>(tile) + off) = v;
}
__device__ __forceinline__ float load_f(const float* tile, uint32_t off) {
    return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(tile) + off);
}

// idx -> (row, first column) of a K-major tile with R rows, chosen so that the
// 32 lanes of a warp cover 8 consecutive rows x 4 column quads: each group of
// 8 lanes then touches one contiguous 128-byte core matrix.
template <int R>
__device__ __forceinline__ void tile_coord(int idx, int& r, int& k4) {
    const int rr = idx & 7, cc = (idx >> 3) & 3, rest = idx >> 5;
    const int rg = rest % (R / 8), cg = rest / (R / 8);
    r = 8 * rg + rr;
    k4 = 4 * (4 * cg + cc);
}

template <int DK, int DV>
__global__ void __launch_bounds__(NT, 1) intra_tc_kernel(ExtendArgs p) {
    if (batch_rejected(p)) return;
    const LayerDims& d = p.d;
    const int G = d.G, HV = d.HV, HK = d.HK;
    // work items (chunk, qk head) in order; CTA b takes items b, b + gridDim.x, ... skipping padded requests
    const int nitems = p.hdr[kHdrNumChunks] * HK;
    auto next_item = [&](int it) {
        for (; it < nitems; it += gridDim.x) {
            const int sl = p.slots[p.chunk_tab[it / HK].x];
            if (sl >= 0 && sl < p.P) break;
        }
        return it;
    };
    int item = next_item(blockIdx.x);
    if (item >= nitems) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    IntraTcSmem<DK, DV>& sm = *reinterpret_cast<IntraTcSmem<DK, DV>*>(smem_raw);
    const uint32_t bar = tc::smem_u32(&sm.bar_mma), bar_kq = tc::smem_u32(&sm.bar_kq);
    constexpr uint32_t KQ_BYTES = 2 * C * DK * 4, VT_BYTES = DV * C * 4, GB_BYTES = C * 8;
    const uint32_t bar_v = tc::smem_u32(&sm.bar_v);
    auto kq_src = [&](int it) { return p.KQ + (size_t)it * (2 * C * DK); };  // item = chunk * HK + hk
    auto head_row = [&](int it, int jj) { return (size_t)(it / HK) * HV + (it % HK) * G + jj; };
    auto fetch_kq = [&](int it) {
        tc::mbar_expect_tx(bar_kq, KQ_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.kq), kq_src(it), KQ_BYTES, bar_kq);
    };
    auto fetch_v = [&](int it, int jj) {  // V^T tile of value head jj of the item's group
        tc::mbar_expect_tx(bar_v, VT_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.bv), p.VT + head_row(it, jj) * (DV * C), VT_BYTES, bar_v);
    };
    auto fetch_g = [&](int it, int jj) {  // gates of value head jj of the item's group into buffer jj & 1
        const uint32_t bg = tc::smem_u32(&sm.bar_g[jj & 1]);
        tc::mbar_expect_tx(bg, GB_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.gb[jj & 1]), p.GB + head_row(it, jj) * C, GB_BYTES, bg);
    };
    auto prefetch_l2 = [&](int it) {  // the next item's inputs, while this one computes
        tc::bulk_prefetch_l2(kq_src(it), KQ_BYTES);
        for (int jj = 0; jj < G; ++jj) {
            tc::bulk_prefetch_l2(p.VT + head_row(it, jj) * (DV * C), VT_BYTES);
            tc::bulk_prefetch_l2(p.GB + head_row(it, jj) * C, GB_BYTES);
        }
    };

    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 512);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(bar_kq, 1);
        tc::mbar_init(bar_v, 1);
        tc::mbar_init(tc::smem_u32(&sm.bar_g[0]), 1);
        tc::mbar_init(tc::smem_u32(&sm.bar_g[1]), 1);
        tc::fence_mbar_init();
        fetch_kq(item);
        fetch_g(item, 0);
        if (G > 1) fetch_g(item, 1);
        fetch_v(item, 0);
    }
    // the upper off-diagonal block of T is zero for every head
    for (int e = tid; e < 32 * 32; e += NT) sm.tf[e >> 5][32 + (e & 31)] = 0.f;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    const uint32_t tD1 = tm, tW = tm + 64, tU = tm + 64 + DK;  // D1: 64 cols; W, U: M = 64 layout
    const int sp = warp & 3, half = warp >> 2;  // TMEM sub-partition, column half
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    // completed uses of each barrier so far, identical in every thread (parity = count & 1)
    uint32_t n_kq = 0, n_v = 0, n_g[2] = {0u, 0u}, ph_mma = 0;
    bool ok = true;
    while (ok && item < nitems) {
    const int nxt = next_item(item + gridDim.x);
    const int id = item / HK, hk = item % HK;
    const int n = p.chunk_tab[id].z;
    if (tid == 0 && nxt < nitems) prefetch_l2(nxt);
    if (tid == 0) {
        ok = tc::mbar_wait(bar_kq, n_kq & 1u);
        if (ok) {  // D1 = [K ; Q] K^T
            const uint32_t base = tc::smem_u32(sm.kq);
            constexpr uint32_t idesc = tc::idesc_tf32(128, 64);
#pragma unroll
            for (int s = 0; s < DK / 8; ++s)
                tc::mma_tf32(tD1, tc::desc_kmajor(base, 2 * C, s), tc::desc_kmajor(base, 2 * C, s), idesc, s > 0);
            tc::mma_commit(bar);
        }
    }
    // K^T (feature rows) from the k rows of the [K ; Q] tile, once for all value heads.  A warp reads
    // one 128-byte core matrix of the tile (8 rows s x 4 features f): no bank conflicts.
    ok = ok && tc::mbar_wait(bar_kq, n_kq & 1u);
    ++n_kq;
    if (ok)
        for (int idx = tid; idx < DK * C; idx += NT) {
            const int s = (idx & 7) + 8 * ((idx >> 5) & 7), f = ((idx >> 3) & 3) + 4 * (idx >> 8);
            *reinterpret_cast<float*>(reinterpret_cast<char*>(sm.kt) + tc::kmajor_off(f, s, DK)) =
                load_f(sm.kq, tc::kmajor_off(s, f, 2 * C));
        }
    ok = __syncthreads_and(ok);

    for (int j = 0; j < G && ok; ++j) {
        const int h = hk * G + j, b = j & 1;
        const size_t ch_h = (size_t)id * HV + h;
        char* WQg = reinterpret_cast<char*>(p.WQ + ch_h * (2 * C * DK));
        char* AQg = reinterpret_cast<char*>(p.AQ + ch_h * (C * C));
        char* KTg = reinterpret_cast<char*>(p.KT + ch_h * (DK * C));
        float* Ug = p.U + ch_h * (C * DV);
        bool okv = tc::mbar_wait(tc::smem_u32(&sm.bar_g[b]), n_g[b] & 1u);
        ++n_g[b];
        if (okv && warp == 0) {  // inclusive scan of g over the chunk, two rows per lane
            const float2 g0 = sm.gb[b][2 * lane], g1 = sm.gb[b][2 * lane + 1];
            const float pair = g0.x + g1.x;
            float incl = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const float gA = incl - pair + g0.x;
            sm.gam[2 * lane] = gA;
            sm.gam[2 * lane + 1] = incl;
            sm.beta[2 * lane] = g0.y;
            sm.beta[2 * lane + 1] = g1.y;
            sm.eg[2 * lane] = __expf(gA);
            sm.eg[2 * lane + 1] = __expf(incl);
            const float gn = __shfl_sync(0xffffffffu, (n - 1) & 1 ? incl : gA, (n - 1) >> 1);
            sm.fkt[2 * lane] = 2 * lane < n ? __expf(gn - gA) : 0.f;
            sm.fkt[2 * lane + 1] = 2 * lane + 1 < n ? __expf(gn - incl) : 0.f;
        }
        if (j == 0) {
            okv = okv && tc::mbar_wait(bar, ph_mma);
            ph_mma ^= 1;
        }
        ok = __syncthreads_and(okv);
        if (!ok) break;
        tc::fence_after_sync();
        const float gl = sm.gam[n - 1];
        {  // A (sub-partitions 0-1: k.k rows) and the masked decayed q.k tile (2-3: q.k rows) from D1;
           // the two warps of a sub-partition take one half of the 64 columns each
            const int r = (sp & 1) * 32 + lane, c0 = 32 * half;
            float row[32];
#pragma unroll
            for (int c = 0; c < 32; c += 16) {
                float v[16];
                tc::tmem_ld16(tD1 + lane_base + c0 + c, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) row[c + i] = v[i];
            }
            tc::tmem_ld_wait();
            const float gr = sm.gam[r], br = sm.beta[r];
            if (sp < 2) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int s = c0 + i;
                    sm.a[r][s] = (s < r && r < n) ? br * __expf(gr - sm.gam[s]) * row[i] : 0.f;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float o[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int s = c0 + i + u;
                        o[u] = (s <= r && r < n) ? tc::round_tf32(__expf(gr - sm.gam[s]) * row[i + u]) : 0.f;
                    }
                    store_f4(reinterpret_cast<float*>(AQg), tc::kmajor_off(r, c0 + i, C), make_float4(o[0], o[1], o[2], o[3]));
                }
            }
        }
        __syncthreads();
        // T = (I + A)^{-1} in 32-row blocks: T = [[T11, 0], [T21, T22]], T21 = -T22 (A21 T11).
        // Warps 0-1 invert the diagonal blocks, one column per lane held in registers, by forward
        // substitution (t_r = [r == c] - sum_{s<r} A_rs t_s; the s = r-1 term goes last so that only
        // one FMA per row sits on the dependent chain).  Meanwhile warps 2-7 write what needs only the
        // gates: (diag(e^gamma) K)^T for W, the state pass's (diag(e^{gamma_n-gamma}) K)^T and the
        // rows Qg = diag(e^gamma) Q of the [W ; Qg] tile.
        if (warp < 2) {
            const int o = 32 * warp;
            float t[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const float* arow = &sm.a[o + r][o];
                float acc[4] = {r == lane ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s = 0; s + 1 < r; ++s) acc[s & 3] = fmaf(-arow[s], t[s], acc[s & 3]);
                const float base = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                t[r] = r > 0 ? fmaf(-arow[r - 1], t[r - 1], base) : base;
            }
#pragma unroll
            for (int r = 0; r < 32; ++r) sm.tf[o + r][o + lane] = t[r];
        } else {
            constexpr int NW = NT - 64;
            const int wt = tid - 64;
            for (int idx = wt; idx < DK * C / 4; idx += NW) {
                int f, s4;
                tile_coord<DK>(idx, f, s4);
                const uint32_t off = tc::kmajor_off(f, s4, DK);
                const float4 k = *reinterpret_cast<const float4*>(reinterpret_cast<const char*>(sm.kt) + off);
                store_f4(sm.kte, off,
                         make_float4(tc::round_tf32(k.x * sm.eg[s4]), tc::round_tf32(k.y * sm.eg[s4 + 1]),
                                     tc::round_tf32(k.z * sm.eg[s4 + 2]), tc::round_tf32(k.w * sm.eg[s4 + 3])));
                store_f4(reinterpret_cast<float*>(KTg), off,
                         make_float4(tc::round_tf32(k.x * sm.fkt[s4]), tc::round_tf32(k.y * sm.fkt[s4 + 1]),
                                     tc::round_tf32(k.z * sm.fkt[s4 + 2]), tc::round_tf32(k.w * sm.fkt[s4 + 3])));
            }
            for (int idx = wt; idx < C * DK / 4; idx += NW) {  // same tile offsets as the q rows of [K ; Q]
                int r, k4;
                tile_coord<C>(idx, r, k4);
                const uint32_t off = tc::kmajor_off(C + r, k4, 2 * C);
                const float4 q = *reinterpret_cast<const float4*>(reinterpret_cast<const char*>(sm.kq) + off);
                const float e = sm.eg[r];
                store_f4(reinterpret_cast<float*>(WQg), off,
                         make_float4(tc::round_tf32(q.x * e), tc::round_tf32(q.y * e), tc::round_tf32(q.z * e),
                                     tc::round_tf32(q.w * e)));
            }
            if (wt < C) p.gam[ch_h * C + wt] = sm.gam[wt];
        }
        __syncthreads();
        {  // P = A21 T11 (T11 lower triangular): thread -> row r, columns c, c + 8, c + 16, c + 24
            const int r = tid >> 3, c = tid & 7;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int s = 0; s < 32; ++s) {
                const float av = sm.a[32 + r][s];
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] = fmaf(av, sm.tf[s][c + 8 * k], acc[k]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) sm.m[r][c + 8 * k] = acc[k];
        }
        __syncthreads();
        {  // T21 = -T22 P (T22 lower triangular)
            const int r = tid >> 3, c = tid & 7;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int s = 0; s < 32; ++s) {
                const float tv = sm.tf[32 + r][32 + s];
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] = fmaf(tv, sm.m[s][c + 8 * k], acc[k]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) sm.tf[32 + r][c + 8 * k] = -acc[k];
        }
        __syncthreads();
        // T diag(beta) -> K-major tf32 tile
        for (int idx = tid; idx < C * C / 4; idx += NT) {
            int r, s4;
            tile_coord<C>(idx, r, s4);
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = (s4 + u <= r) ? tc::round_tf32(sm.tf[r][s4 + u] * sm.beta[s4 + u]) : 0.f;
            store_f4(sm.t, tc::kmajor_off(r, s4, C), make_float4(v[0], v[1], v[2], v[3]));
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        bool okm = true;
        if (tid == 0) {  // W = (T diag(beta)) (diag(e^gamma) K),  U = (T diag(beta)) V   (M = 64)
            okm = tc::mbar_wait(bar_v, n_v & 1u);
            if (okm) {
                const uint32_t bt = tc::smem_u32(sm.t), bkk = tc::smem_u32(sm.kte), bvv = tc::smem_u32(sm.bv);
                constexpr uint32_t iw = tc::idesc_tf32(64, DK), iu = tc::idesc_tf32(64, DV);
#pragma unroll
                for (int s = 0; s < C / 8; ++s)
                    tc::mma_tf32(tW, tc::desc_kmajor(bt, C, s), tc::desc_kmajor(bkk, DK, s), iw, s > 0);
#pragma unroll
                for (int s = 0; s < C / 8; ++s)
                    tc::mma_tf32(tU, tc::desc_kmajor(bt, C, s), tc::desc_kmajor(bvv, DV, s), iu, s > 0);
                tc::mma_commit(bar);
            }
        }
        ++n_v;
        ok = okm && tc::mbar_wait(bar, ph_mma);  // okm is false only on tid 0, if the V tile never came
        ph_mma ^= 1;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        if (tid == 0) {  // the V^T tile and gate buffer b are free again; after the last head, so is [K ; Q]
            if (j + 1 < G) fetch_v(item, j + 1);
            if (j + 2 < G) fetch_g(item, j + 2);
            if (j == G - 1 && nxt < nitems) {  // the next item's tiles land during this epilogue
                fetch_kq(nxt);
                fetch_g(nxt, 0);
                if (G > 1) fetch_g(nxt, 1);
                fetch_v(nxt, 0);
            }
        }
        {  // W rows -> [W ; Qg] tile rows 0..63 (tf32, K-major); U rows -> fp32 row-major.
           // M = 64 layout: lanes 0-15 of sub-partition sp hold rows 16 sp .. 16 sp + 15;
           // the two warps of a sub-partition take one half of the columns each
            const bool valid = lane < 16;
            const int r = sp * 16 + lane;
#pragma unroll
            for (int c0 = half * (DK / 2); c0 < (half + 1) * (DK / 2); c0 += 16) {
                float v[16];
                tc::tmem_ld16(tW + lane_base + c0, v);
                tc::tmem_ld_wait();
                if (valid)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        store_f4(reinterpret_cast<float*>(WQg), tc::kmajor_off(r, c0 + 4 * q, 2 * C),
                                 make_float4(tc::round_tf32(v[4 * q]), tc::round_tf32(v[4 * q + 1]),
                                             tc::round_tf32(v[4 * q + 2]), tc::round_tf32(v[4 * q + 3])));
            }
#pragma unroll
            for (int c0 = half * (DV / 2); c0 < (half + 1) * (DV / 2); c0 += 16) {
                float v[16];
                tc::tmem_ld16(tU + lane_base + c0, v);
                tc::tmem_ld_wait();
                if (valid)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4*>(Ug + (size_t)r * DV + c0 + 4 * q) =
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    }
    item = nxt;
    }
    if (!ok && tid == 0) {
        raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
        // let copies already in flight land before the CTA's shared memory goes away
        for (int b = 0; b < 2; ++b)
            for (uint32_t par = 0; par < 2; ++par) tc::mbar_wait(tc::smem_u32(&sm.bar_g[b]), par, 100000000ull);
        for (uint32_t par = 0; par < 2; ++par) tc::mbar_wait(bar_v, par, 100000000ull);
        for (uint32_t par = 0; par < 2; ++par) tc::mbar_wait(bar_kq, par, 100000000ull);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 512);
}

}  // namespace

template <int DK, int DV>
cudaError_t launch_intra(const ExtendArgs& p, cudaStream_t s) {
    const size_t shm = sizeof(IntraTcSmem<DK, DV>);
    cudaError_t e = cudaFuncSetAttribute(intra_tc_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // persistent: one CTA per SM walks the (chunk, qk head) items
    const long long items = (long long)p.max_chunks * p.d.HK;
    const int grid = (int)(items < sms ? items : sms);
    intra_tc_kernel<DK, DV><<<grid, NT, shm, s>>>(p);
    return cudaGetLastError();
}

template cudaError_t launch_intra<64, 64>(const ExtendArgs&, cudaStream_t);
template cudaError_t launch_intra<64, 128>(const ExtendArgs&, cudaStream_t);
template cudaError_t launch_intra<128, 64>(const ExtendArgs&, cudaStream_t);
template cudaError_t launch_intra<128, 128>(const ExtendArgs&, cudaStream_t);

}  // namespace gdn
