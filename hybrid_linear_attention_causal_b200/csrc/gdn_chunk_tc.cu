// Per-chunk step of the chunked GDN prefill on tcgen05 tensor cores (sm_100a):
// the chunk's conv1d + SiLU, L2 norm and gates fused with the intra-chunk
// WY/UT products, so no intermediate of the chunk goes through global memory
// before the tiles the serial state pass reads.
//
// One (chunk, qk head) item at a time; an item serves the G value heads that
// share the qk head.  For a chunk of n <= 64 rows starting at packed row t0:
//
//   rows t0-3 .. t0+n-1 of the item's channels are staged in shared memory
//   (the 3 rows before the chunk come from the previous chunk of the same
//   sequence, or from the conv-state slot for a sequence's first chunk);
//   y = SiLU(conv1d(x)), q and k L2-normalised (q carries the output scale),
//   g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b), gamma_r = sum_{s<=r} g_s;
//
//   D1  = [K; Q] K^T                          (fp16 MMA, M=128 N=64 K=dk)
//   A   = beta_r e^{gamma_r-gamma_s} (k_r.k_s)        s < r   (strictly lower)
//   Aqk = e^{gamma_r-gamma_s} (q_r.k_s)               s <= r
//   T   = (I + A)^{-1}                        (fp32: 16x16 forward substitution + block products)
//   W   = T diag(beta e^gamma) K              (fp16 MMA, M=64 N=dk K=64; K read MN-major)
//   U^T = V^T (T diag(beta))^T                (fp16 MMA, M=dv N=64 K=64)
//
// (the WY/UT form of the gated delta rule, Gated DeltaNet, Yang, Kautz and
// Hatamizadeh, ICLR 2025).  The item writes, as fp16 tiles in the tensor
// core's 128-byte swizzled shared-memory layout (so the state pass copies
// them verbatim): [K ; Q] once per (chunk, qk head), and per (chunk, value
// head) W, U^T and the masked decayed q.k; plus gamma in fp32.  Rows past the
// end of a ragged chunk are zero in every tile.  One thread issues the MMAs;
// the eight warps read their sub-partition's 32-lane slice of tensor memory
// (two warps per slice, one group of columns each) for the CUDA-core steps.
// Two CTAs share an SM (half of its tensor memory and shared memory each), so
// one CTA's barrier waits are covered by the other.

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;        // 8 warps; warp w reads TMEM sub-partition w % 4
constexpr int kCtasPerSm = 2;
constexpr int NCG = NT / 128;  // warps per TMEM sub-partition, each taking one group of columns
constexpr uint32_t kTmemCols = 256;  // D1 (64 columns) + W (DK) + U^T (64), a half of tensor memory
constexpr int kInvBarrier = 1;       // named barrier of warps 0-3, which take levels 1 and 2 of the inverse
constexpr int kItemsPerCta = 2;
constexpr float kLog2e = 1.4426950408889634f;  // log2(e)

template <typename T, int DK, int DV>
struct ChunkShape {
    static constexpr int PADE = 16 / (int)sizeof(T);     // staged-row padding (one 16-byte vector)
    static constexpr int LDQK = 2 * DK + PADE;           // staged q,k row: k channels, then q channels
    static constexpr int LDV = DV + PADE;                // staged v row
    static constexpr size_t XQK = (size_t)(C + 3) * LDQK * sizeof(T);
    static constexpr size_t XV = (size_t)(C + 3) * LDV * sizeof(T);
};

template <typename T, int DK, int DV>
struct ChunkSmem {
    using S = ChunkShape<T, DK, DV>;
    // fp16 operand tiles in the 128-byte swizzled layout; each starts on a 1024-byte boundary
    uint16_t kq[2 * C * DK];  // [K ; Q*scale], 128 rows x DK: D1's operands, W's B (K rows read MN-major)
    uint16_t bv[DV * C];      // V^T of the current value head, DV rows x C
    uint16_t t[C * C];        // T diag(beta), C rows x C: U's operand
    uint16_t te[C * C];       // T diag(beta e^gamma), same layout: W's operand
    struct Inv {
        float a[C][C + 1];     // A (fp32)
        float tf[2][32][36];   // T (fp32) in its two 32x32 diagonal blocks: what the next levels read
        float m[32][36];       // A21 T11
        float y[2][16][20];    // A21 D1 inside each 32x32 diagonal block (rows 16-byte aligned)
    };
    // raw rows (q,k of the item, then v of one value head), or the inverse's fp32 work space
    static constexpr size_t XMAX = S::XQK > S::XV ? S::XQK : S::XV;
    static constexpr size_t UBYTES = XMAX > sizeof(Inv) ? XMAX : sizeof(Inv);
    alignas(16) unsigned char u[UBYTES];
    float2 gb[C];          // (g, beta) of the current value head
    float gam[C], gam2[C], beta[C], bge[C];  // gamma, gamma log2(e), beta, beta e^gamma
    unsigned long long bar_mma;
    uint32_t tmem_base;
    int next_item;
};

template <typename T, int DK, int DV>
constexpr size_t chunk_smem_bytes() {
    return sizeof(ChunkSmem<T, DK, DV>) + 1024;  // + room to align the tiles on 1024 bytes
}

__device__ __forceinline__ void bar_sync_n(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// 4 consecutive staged elements -> 4 floats (8-byte load for bf16, 16-byte for fp32)
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* v) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const float* p, float* v) {
    const float4 w = *reinterpret_cast<const float4*>(p);
    v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
}

// SiLU with the fast exponential and division: their error (a few ulp) is far below the fp16
// rounding every conv output goes through
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// 8 floats -> 8 fp16 (one 16-byte store) at byte offset `off` of a tile in global memory
__device__ __forceinline__ void store_h8_global(char* tile, uint32_t off, const float* v) {
    *reinterpret_cast<uint4*>(tile + off) = make_uint4(tc::pack_f16(v[0], v[1]), tc::pack_f16(v[2], v[3]),
                                                       tc::pack_f16(v[4], v[5]), tc::pack_f16(v[6], v[7]));
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, kCtasPerSm) chunk_tc_kernel(ExtendArgs p, int seg) {
    using S = ChunkShape<T, DK, DV>;
    using Sm = ChunkSmem<T, DK, DV>;
    if (batch_rejected(p)) return;
    const LayerDims& d = p.d;
    const int G = d.G, HV = d.HV, HK = d.HK;
    // This segment's (chunk, qk head) items, handed out dynamically from one counter: CTAs that start
    // late (while the other stream's state pass holds SMs) still find work.  An item is named by
    // chunk * HK + hk; padded requests are skipped; -1 = none left.
    const int base = p.hdr[kHdrSegOff + seg];
    const int nlist = p.hdr[kHdrSegCnt + seg] * HK;
    int* next_ctr = p.hdr + kHdrItemNext + seg;
    auto grab = [&]() -> int {
        while (true) {
            const int li = atomicAdd(next_ctr, 1);
            if (li >= nlist) return -1;
            const int cid = p.chunk_list[base + li / HK];
            const int sl = p.slots[p.chunk_tab[cid].x];
            if (sl >= 0 && sl < p.P) return cid * HK + li % HK;
        }
    };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    extern __shared__ unsigned char smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    if (tid == 0) sm.next_item = grab();
    __syncthreads();
    int item = sm.next_item;
    if (item < 0) return;
    const uint32_t bar = tc::smem_u32(&sm.bar_mma);
    const T* x = reinterpret_cast<const T*>(p.x);
    const T* w = reinterpret_cast<const T*>(p.conv_w);
    const T* cbias = reinterpret_cast<const T*>(p.conv_b);
    T* xs = reinterpret_cast<T*>(sm.u);
    typename Sm::Inv& inv = *reinterpret_cast<typename Sm::Inv*>(sm.u);

    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
    }
    // blocks of T above the diagonal are zero for every head: in the tiles, and in the two 16x16
    // corners of the 32x32 diagonal blocks that the inverse reads back
    for (int e = tid; e < C * C; e += NT) sm.t[e] = sm.te[e] = 0;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    // D1: 64 columns; W: M = 64 layout, DK columns; U^T: M = DV, 64 columns
    const uint32_t tD1 = tm, tW = tm + 64, tU = tm + 64 + DK;
    const int sp = warp & 3, cg = warp >> 2;  // TMEM sub-partition, column group
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    uint32_t ph_mma = 0;
    bool ok = true;
    int done = 0;
    while (ok && item >= 0) {
        int nxt = -1;
        // At most kItemsPerCta items, then the CTA ends: its SM goes to whatever waits, first of all a
        // state-pass CTA of the previous segment (its stream has the higher priority).
        if (tid == 0 && ++done < kItemsPerCta) nxt = grab();
        const int id = item / HK, hk = item % HK;
        const int4 ch = p.chunk_tab[id];
        const int seq = ch.x, t0 = ch.y, n = ch.z, cidx = ch.w;
        const int slot = p.slots[seq];
        const bool init = p.has_init ? p.has_init[seq] != 0 : true;
        const int ck0 = d.HK * DK + hk * DK, cq0 = hk * DK;  // first k / q channel
        if (tid == 0 && nxt >= 0) {  // the next item's rows into L2 while this one computes
            const int4 chn = p.chunk_tab[nxt / HK];
            const int hkn = nxt % HK;
            const int r0 = chn.w > 0 ? chn.y - 3 : chn.y;
            for (int r = r0; r < chn.y + chn.z; ++r) {
                const T* row = x + (size_t)r * d.conv_dim;
                tc::bulk_prefetch_l2(row + hkn * DK, DK * sizeof(T));
                tc::bulk_prefetch_l2(row + d.HK * DK + hkn * DK, DK * sizeof(T));
                tc::bulk_prefetch_l2(row + 2 * d.HK * DK + hkn * G * DV, G * DV * sizeof(T));
            }
        }
        // ---- stage the q,k rows: staged row i <-> packed row t0 - 3 + i; columns k then q
        {
            constexpr int VE = 16 / (int)sizeof(T);  // elements per 16-byte vector
            constexpr int VPR = 2 * DK / VE;         // vectors per staged row
            const int nv = n * VPR;
            for (int b0 = 0; b0 < nv; b0 += NT * 4) {
                uint4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = b0 + u * NT + tid;
                    if (e < nv) {
                        const int r = e / VPR, c = (e % VPR) * VE;
                        const int gc = c < DK ? ck0 + c : cq0 + (c - DK);
                        v[u] = *reinterpret_cast<const uint4*>(x + (size_t)(t0 + r) * d.conv_dim + gc);
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = b0 + u * NT + tid;
                    if (e < nv) {
                        const int r = e / VPR, c = (e % VPR) * VE;
                        *reinterpret_cast<uint4*>(xs + (size_t)(r + 3) * S::LDQK + c) = v[u];
                    }
                }
            }
            const T* cs = reinterpret_cast<const T*>(p.conv_state) + (size_t)slot * d.conv_dim * 3;
            for (int e = tid; e < 3 * 2 * DK; e += NT) {
                const int i = e / (2 * DK), c = e % (2 * DK);
                const int gc = c < DK ? ck0 + c : cq0 + (c - DK);
                T v;
                if (cidx > 0) v = x[(size_t)(t0 - 3 + i) * d.conv_dim + gc];
                else v = init ? cs[(size_t)gc * 3 + i] : from_f<T>(0.f);
                xs[(size_t)i * S::LDQK + c] = v;
            }
        }
        __syncthreads();
        // ---- conv + SiLU + L2 norm of k (tile rows 0..63) and q*scale (rows 64..127): warp w takes
        // rows 8w .. 8w+7; lane (rr, cc) row 8w + rr and the column quads 16 c + 4 cc; a row's four
        // lanes hold all DK channels, so the norm reduces over them
        {
            const int rr = lane & 7, cc = lane >> 3;
            const int r = 8 * warp + rr;
            char* kqb = reinterpret_cast<char*>(sm.kq);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int gc0 = part == 0 ? ck0 : cq0;
                float y[DK / 16][4];
                float ss = 0.f;
#pragma unroll
                for (int c16 = 0; c16 < DK / 16; ++c16) {
                    const int cl = 16 * c16 + 4 * cc;  // first of 4 channels, within the part
                    float acc[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int gc = gc0 + cl + u;
                        acc[u] = cbias ? to_f(cbias[gc]) : 0.f;
                    }
                    if (r < n) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float xv[4];
                            load4(xs + (size_t)(r + j) * S::LDQK + part * DK + cl, xv);
#pragma unroll
                            for (int u = 0; u < 4; ++u) acc[u] = fmaf(to_f(w[(size_t)(gc0 + cl + u) * 4 + j]), xv[u], acc[u]);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        y[c16][u] = r < n ? silu_fast(acc[u]) : 0.f;
                        ss = fmaf(y[c16][u], y[c16][u], ss);
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 8);
                ss += __shfl_xor_sync(0xffffffffu, ss, 16);
                const float sc = r < n ? rsqrtf(ss + d.eps) * (part ? d.scale : 1.f) : 0.f;
                const int tr = part * C + r;  // tile row
#pragma unroll
                for (int c16 = 0; c16 < DK / 16; ++c16) {
                    const int cl = 16 * c16 + 4 * cc;
                    *reinterpret_cast<uint2*>(kqb + tc::sw128_off(tr, cl, 2 * C)) =
                        make_uint2(tc::pack_f16(y[c16][0] * sc, y[c16][1] * sc), tc::pack_f16(y[c16][2] * sc, y[c16][3] * sc));
                }
            }
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0) {  // D1 = [K ; Q] K^T; the [K ; Q] tile leaves for the state pass by a bulk copy
            const uint32_t kqs = tc::smem_u32(sm.kq);
            constexpr uint32_t idesc = tc::idesc_f16(128, 64);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                tc::mma_f16(tD1, tc::desc_sw128_k(kqs, 2 * C, s), tc::desc_sw128_k(kqs, 2 * C, s), idesc, s > 0);
            tc::mma_commit(bar);
            tc::bulk_s2g(p.KQ + ((size_t)id * HK + hk) * (2 * C * DK), kqs, 2 * C * DK * 2);
            tc::bulk_commit();
        }

        for (int j = 0; j < G && ok; ++j) {
            const int h = hk * G + j;
            const size_t ch_h = (size_t)id * HV + h;
            // ---- stage this value head's v rows (the q,k rows are no longer needed), and its gates
            {
                const int cv0 = 2 * d.HK * DK + h * DV;
                constexpr int VE = 16 / (int)sizeof(T);
                constexpr int VPR = DV / VE;
                const int nv = n * VPR;
                for (int b0 = 0; b0 < nv; b0 += NT * 4) {
                    uint4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = b0 + u * NT + tid;
                        if (e < nv)
                            v[u] = *reinterpret_cast<const uint4*>(x + (size_t)(t0 + e / VPR) * d.conv_dim + cv0 +
                                                                   (e % VPR) * VE);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = b0 + u * NT + tid;
                        if (e < nv) *reinterpret_cast<uint4*>(xs + (size_t)(e / VPR + 3) * S::LDV + (e % VPR) * VE) = v[u];
                    }
                }
                const T* cs = reinterpret_cast<const T*>(p.conv_state) + (size_t)slot * d.conv_dim * 3;
                for (int e = tid; e < 3 * DV; e += NT) {
                    const int i = e / DV, c = e % DV;
                    T v;
                    if (cidx > 0) v = x[(size_t)(t0 - 3 + i) * d.conv_dim + cv0 + c];
                    else v = init ? cs[(size_t)(cv0 + c) * 3 + i] : from_f<T>(0.f);
                    xs[(size_t)i * S::LDV + c] = v;
                }
                if (tid >= NT - C) {  // gates of the chunk's rows (zero past the end)
                    const int r = tid - (NT - C);
                    float2 gb = make_float2(0.f, 0.f);
                    if (r < n) {
                        const size_t row = (size_t)(t0 + r) * HV + h;
                        const float av = to_f(reinterpret_cast<const T*>(p.a)[row]);
                        const float bv2 = to_f(reinterpret_cast<const T*>(p.b)[row]);
                        gb = make_float2(-expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]), sigmoid_f(bv2));
                    }
                    sm.gb[r] = gb;
                }
            }
            __syncthreads();
            // ---- V^T tile: thread (f, 4 consecutive rows) from a sliding window of 7 staged rows; warp 0
            // also scans the gates
            {
                char* bvb = reinterpret_cast<char*>(sm.bv);
                for (int idx = tid; idx < DV * (C / 4); idx += NT) {
                    const int ff = idx & 7, cq = (idx >> 3) & 3, rest = idx >> 5;
                    const int fg = rest % (DV / 8), rg = rest / (DV / 8);
                    const int f = 8 * fg + ff, r4 = 4 * (4 * rg + cq);
                    const int gcv = 2 * d.HK * DK + h * DV + f;
                    float wc[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) wc[q] = to_f(w[(size_t)gcv * 4 + q]);
                    const float b0 = cbias ? to_f(cbias[gcv]) : 0.f;
                    float xw[7];
#pragma unroll
                    for (int i = 0; i < 7; ++i) xw[i] = to_f(xs[(size_t)(r4 + i) * S::LDV + f]);
                    float yv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        float acc = fmaf(wc[0], xw[u], b0);
                        acc = fmaf(wc[1], xw[u + 1], acc);
                        acc = fmaf(wc[2], xw[u + 2], acc);
                        acc = fmaf(wc[3], xw[u + 3], acc);
                        yv[u] = r4 + u < n ? silu_fast(acc) : 0.f;
                    }
                    *reinterpret_cast<uint2*>(bvb + tc::sw128_off(f, r4, DV)) =
                        make_uint2(tc::pack_f16(yv[0], yv[1]), tc::pack_f16(yv[2], yv[3]));
                }
                if (warp == 0) {  // inclusive scan of g over the chunk, two rows per lane
                    const float2 g0 = sm.gb[2 * lane], g1 = sm.gb[2 * lane + 1];
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
                    sm.gam2[2 * lane] = gA * kLog2e;
                    sm.gam2[2 * lane + 1] = incl * kLog2e;
                    sm.beta[2 * lane] = g0.y;
                    sm.beta[2 * lane + 1] = g1.y;
                    sm.bge[2 * lane] = g0.y * __expf(gA);
                    sm.bge[2 * lane + 1] = g1.y * __expf(incl);
                }
            }
            bool okv = true;
            if (j == 0) okv = tc::mbar_wait(bar, ph_mma);  // D1
            ok = __syncthreads_and(okv);
            if (!ok) break;
            if (j == 0) {
                ph_mma ^= 1;
                tc::fence_after_sync();
            }
            // ---- A (sub-partitions 0-1: k.k rows) into shared memory and the masked decayed q.k tile
            // (2-3: q.k rows) straight to global memory, from D1; the warps of a sub-partition take one
            // group of C / NCG columns each.  The exponents are formed without branches (a masked entry
            // gets -inf, whose exponential is 0); a block wholly above the diagonal only gets zeros.
            {
                char* AQg = reinterpret_cast<char*>(p.AQ + ch_h * (C * C));
                constexpr int NC = C / NCG;
                static_assert(NC % 16 == 0, "16-column loads");
                const int r = (sp & 1) * 32 + lane;
                const bool qrow = sp >= 2;
#pragma unroll
                for (int c0 = NC * cg; c0 < NC * (cg + 1); c0 += 16) {
                    const bool live = c0 <= (sp & 1) * 32 + 31;  // warp-uniform
                    float v[16], e[16];
                    if (live) {
                        tc::tmem_ld16(tD1 + lane_base + c0, v);
                        tc::tmem_ld_wait();
                        const int lim = r < n ? r - c0 + (qrow ? 1 : 0) : 0;
                        const float gr = sm.gam2[r];
#pragma unroll
                        for (int q = 0; q < 16; q += 4) {
                            const float4 gs = *reinterpret_cast<const float4*>(&sm.gam2[c0 + q]);
                            const float gq[4] = {gs.x, gs.y, gs.z, gs.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                e[q + u] = q + u < lim ? gr - gq[u] : __int_as_float(0xff800000u);  // -inf
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) e[i] = tc::ex2_approx(e[i]) * v[i];
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) e[i] = 0.f;
                    }
                    if (!qrow) {
                        const float br = sm.beta[r];
#pragma unroll
                        for (int i = 0; i < 16; ++i) inv.a[r][c0 + i] = br * e[i];
                    } else {
                        store_h8_global(AQg, tc::sw128_off(r, c0, C), e);
                        store_h8_global(AQg, tc::sw128_off(r, c0 + 8, C), e + 8);
                    }
                }
            }
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            // T = (I + A)^{-1}, by blocks.  Every final entry goes straight into the fp16 tiles of
            // T diag(beta) and T diag(beta e^gamma) (the A operands of U and W); the fp32 copy tf holds
            // what the next level reads.
            //   level 1: the four diagonal 16x16 blocks by forward substitution, one column per lane held
            //            in registers (t_r = [r == c] - sum_{s<r} A_rs t_s; the s = r-1 term goes last so
            //            one FMA per row sits on the dependent chain); the other warps write gamma.
            //   level 2: within each 32x32 diagonal block, X = -D2 (A21 D1).
            //   level 3: T21 = -T22 (A21 T11) for the lower-left 32x32 block.
            char* tb = reinterpret_cast<char*>(sm.t);
            char* teb = reinterpret_cast<char*>(sm.te);
            auto put_t = [&](int r, int c, float v) {  // T entry (r, c) into both operand tiles
                const uint32_t off = tc::sw128_off(r, c, C);
                const uint32_t wv = tc::pack_f16(v * sm.beta[c], v * sm.bge[c]);
                *reinterpret_cast<uint16_t*>(tb + off) = (uint16_t)(wv & 0xffffu);
                *reinterpret_cast<uint16_t*>(teb + off) = (uint16_t)(wv >> 16);
            };
            auto fma4 = [](float4& acc, float a, const float4& b) {
                acc.x = fmaf(a, b.x, acc.x);
                acc.y = fmaf(a, b.y, acc.y);
                acc.z = fmaf(a, b.z, acc.z);
                acc.w = fmaf(a, b.w, acc.w);
            };
            if (warp < 4) {
                if (lane < 16) {
                    const int o = 16 * warp, c = lane;
                    float t[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        const float* arow = &inv.a[o + r][o];
                        float acc[2] = {r == c ? 1.f : 0.f, 0.f};
#pragma unroll
                        for (int s = 0; s + 1 < r; ++s) acc[s & 1] = fmaf(-arow[s], t[s], acc[s & 1]);
                        const float b2 = acc[0] + acc[1];
                        t[r] = r > 0 ? fmaf(-arow[r - 1], t[r - 1], b2) : b2;
                    }
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        inv.tf[warp >> 1][16 * (warp & 1) + r][16 * (warp & 1) + c] = t[r];
                        put_t(o + r, o + c, t[r]);
                    }
                } else if ((warp & 1) == 0) {  // the 16x16 corner above the diagonal of 32x32 block warp / 2
                    float4* row = reinterpret_cast<float4*>(&inv.tf[warp >> 1][lane - 16][16]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) row[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                bar_sync_n(kInvBarrier, 128);
                {  // level 2 (threads 0..127): 32-block bb, row r, columns c4 .. c4 + 3
                    const int bb = tid >> 6, r = (tid >> 2) & 15, c4 = 4 * (tid & 3);
                    const int o0 = 32 * bb, o1 = o0 + 16;
                    {
                        float4 yv = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (int s = 0; s < 16; ++s)  // Y = A21 D1
                            fma4(yv, inv.a[o1 + r][o0 + s], *reinterpret_cast<const float4*>(&inv.tf[bb][s][c4]));
                        *reinterpret_cast<float4*>(&inv.y[bb][r][c4]) = yv;
                    }
                    bar_sync_n(kInvBarrier, 128);
                    {
                        float4 xq = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (int s = 0; s < 16; ++s)  // X = -D2 Y
                            fma4(xq, inv.tf[bb][16 + r][16 + s], *reinterpret_cast<const float4*>(&inv.y[bb][s][c4]));
                        xq = make_float4(-xq.x, -xq.y, -xq.z, -xq.w);
                        *reinterpret_cast<float4*>(&inv.tf[bb][16 + r][c4]) = xq;
                        put_t(o1 + r, o0 + c4, xq.x);
                        put_t(o1 + r, o0 + c4 + 1, xq.y);
                        put_t(o1 + r, o0 + c4 + 2, xq.z);
                        put_t(o1 + r, o0 + c4 + 3, xq.w);
                    }
                }
            } else if (tid - 128 < C) {  // the state pass's per-row gate vector
                const int r = tid - 128;
                const float gr = sm.gam[r], gn = sm.gam[n - 1];
                p.GV[ch_h * C + r] = make_float4(__expf(gr), r < n ? __expf(gn - gr) : 0.f, gr, __expf(gn));
            }
            __syncthreads();
            // Level 3 reads one operand as a warp-wide broadcast and skips the zero blocks of the
            // triangular factors: T11[s][c] = 0 for s < c and T22[r][s] = 0 for s > r.
            static_assert(NT / 32 == 8, "level 3 maps 8 column groups, then row groups, onto the warps");
            {  // level 3a: P = A21 T11; warp w takes columns 4w .. 4w + 3, lane = row
                const int r = lane, c4 = 4 * warp;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
                for (int s = c4; s < 32; ++s)
                    fma4(acc, inv.a[32 + r][s], *reinterpret_cast<const float4*>(&inv.tf[0][s][c4]));
                *reinterpret_cast<float4*>(&inv.m[r][c4]) = acc;
            }
            __syncthreads();
            {  // level 3b: T21 = -T22 P; warp w takes 4 consecutive rows of the block, lane = column
                constexpr int RPW = 4;
                const int r0 = RPW * warp, c = lane;
                float acc[RPW];
#pragma unroll
                for (int i = 0; i < RPW; ++i) acc[i] = 0.f;
                for (int s4 = 0; s4 < r0 + RPW; s4 += 4) {
                    const float p0 = inv.m[s4][c], p1 = inv.m[s4 + 1][c], p2 = inv.m[s4 + 2][c], p3 = inv.m[s4 + 3][c];
#pragma unroll
                    for (int i = 0; i < RPW; ++i) {
                        const float4 t = *reinterpret_cast<const float4*>(&inv.tf[1][r0 + i][s4]);
                        acc[i] = fmaf(t.x, p0, fmaf(t.y, p1, fmaf(t.z, p2, fmaf(t.w, p3, acc[i]))));
                    }
                }
#pragma unroll
                for (int i = 0; i < RPW; ++i) put_t(32 + r0 + i, c, -acc[i]);
            }
            tc::fence_smem_to_async();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            if (tid == 0) {  // W = (T diag(beta e^gamma)) K (M = 64, K read MN-major from the [K ; Q] tile),
                             // U^T = V^T (T diag(beta))^T (M = DV)
                const uint32_t bt = tc::smem_u32(sm.t), bte = tc::smem_u32(sm.te), bkq = tc::smem_u32(sm.kq);
                const uint32_t bvv = tc::smem_u32(sm.bv);
                constexpr uint32_t iw = tc::idesc_f16(64, DK) | tc::kTransposeB, iu = tc::idesc_f16(DV, 64);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    tc::mma_f16(tW, tc::desc_sw128_k(bte, C, s), tc::desc_sw128_mn(bkq, 2 * C, s), iw, s > 0);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    tc::mma_f16(tU, tc::desc_sw128_k(bvv, DV, s), tc::desc_sw128_k(bt, C, s), iu, s > 0);
                tc::mma_commit(bar);
            }
            ok = __syncthreads_and(tc::mbar_wait(bar, ph_mma));
            ph_mma ^= 1;
            if (!ok) break;
            tc::fence_after_sync();
            {  // W rows -> the W tile; U -> the U^T tile (both fp16, swizzled, straight to global memory).
               // M = 64 layout: lanes 0-15 of sub-partition sp hold rows 16 sp .. 16 sp + 15; the warps
               // of a sub-partition take one group of columns each
                char* Wg = reinterpret_cast<char*>(p.W + ch_h * (C * DK));
                char* Ug = reinterpret_cast<char*>(p.U + ch_h * (DV * C));
                const bool valid = lane < 16;
                const int r = sp * 16 + lane;
#pragma unroll
                for (int c0 = cg * (DK / NCG); c0 < (cg + 1) * (DK / NCG); c0 += 16) {
                    float v[16];
                    tc::tmem_ld16(tW + lane_base + c0, v);
                    tc::tmem_ld_wait();
                    if (valid) {
                        store_h8_global(Wg, tc::sw128_off(r, c0, C), v);
                        store_h8_global(Wg, tc::sw128_off(r, c0 + 8, C), v + 8);
                    }
                }
                const bool vj = DV == 128 || lane < 16;
                const int jr = DV == 128 ? sp * 32 + lane : sp * 16 + lane;
#pragma unroll
                for (int c0 = cg * (C / NCG); c0 < (cg + 1) * (C / NCG); c0 += 16) {
                    float v[16];
                    tc::tmem_ld16(tU + lane_base + c0, v);
                    tc::tmem_ld_wait();
                    if (vj) {
                        store_h8_global(Ug, tc::sw128_off(jr, c0, DV), v);
                        store_h8_global(Ug, tc::sw128_off(jr, c0 + 8, DV), v + 8);
                    }
                }
            }
            tc::fence_before_sync();
            __syncthreads();  // tensor memory and the staging space are free for the next head
            tc::fence_after_sync();
        }
        if (tid == 0) tc::bulk_wait_read_all();  // the [K ; Q] tile has left before the next item rewrites it
        if (tid == 0) sm.next_item = nxt;
        __syncthreads();
        item = sm.next_item;
    }
    if (!ok && tid == 0) raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
    if (tid == 0) tc::bulk_wait_read_all();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, kTmemCols);
}

}  // namespace

template <typename T, int DK, int DV>
cudaError_t launch_chunk(const ExtendArgs& p, int seg, cudaStream_t s) {
    constexpr size_t shm = chunk_smem_bytes<T, DK, DV>();
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    // CTAs of up to kItemsPerCta (chunk, qk head) items each, enough for the most a segment can hold
    const long long items = ((long long)p.max_chunks + p.nseg - 1) / p.nseg * p.d.HK;
    const int grid = (int)((items + kItemsPerCta - 1) / kItemsPerCta);
    chunk_tc_kernel<T, DK, DV><<<grid, NT, shm, s>>>(p, seg);
    return cudaGetLastError();
}

#define GDN_CHUNK_INST(T)                                                              \
    template cudaError_t launch_chunk<T, 64, 64>(const ExtendArgs&, int, cudaStream_t);  \
    template cudaError_t launch_chunk<T, 64, 128>(const ExtendArgs&, int, cudaStream_t); \
    template cudaError_t launch_chunk<T, 128, 64>(const ExtendArgs&, int, cudaStream_t); \
    template cudaError_t launch_chunk<T, 128, 128>(const ExtendArgs&, int, cudaStream_t);
GDN_CHUNK_INST(float)
GDN_CHUNK_INST(__nv_bfloat16)

}  // namespace gdn
