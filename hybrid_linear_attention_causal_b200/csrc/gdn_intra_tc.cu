// Intra-chunk step of the chunked GDN prefill on tcgen05 tensor cores (sm_100a).
//
// One (chunk, qk head) item at a time; an item serves the G value heads that
// share the qk head.  For a chunk of n <= 64 rows with normalised k_r, q_r (q
// carries the output scale), gates g_r, beta_r and gamma_r = sum_{s<=r} g_s:
//
//   D1  = [K; Q] K^T                          (fp16 MMA, M=128 N=64 K=dk)
//   A   = beta_r e^{gamma_r-gamma_s} (k_r.k_s)        s < r   (strictly lower)
//   Aqk = e^{gamma_r-gamma_s} (q_r.k_s)               s <= r
//   T   = (I + A)^{-1}                        (fp32: 16x16 forward substitution + block products)
//   W   = T diag(beta e^gamma) K              (fp16 MMA, M=64 N=dk K=64; K read MN-major
//                                              straight from the [K ; Q] tile)
//   U^T = V^T (T diag(beta))^T                (fp16 MMA, M=dv N=64 K=64)
//
// (the WY/UT form of the gated delta rule).  The prep kernel's [K ; Q] tile and
// the V^T tiles and gates of the value heads arrive by asynchronous bulk copies.
// For the serial state pass it writes, per (chunk, value head), fp16 tiles in
// the tensor core's shared-memory layout, so the state pass bulk-copies them:
// [W ; diag(e^gamma) Q], Aqk, K~ = diag(e^{gamma_n-gamma}) K (rows s; read
// MN-major) and U^T; plus gamma.  Operands are staged in shared memory as
// no-swizzle tiles rounded to fp16; accumulators live in tensor memory.  One
// thread issues the MMAs; the eight warps read their sub-partition's 32-lane
// slice of tensor memory (two warps per slice, one group of columns each) for
// the CUDA-core steps.  Two CTAs share an SM (half of its tensor memory and
// shared memory each), so one CTA's barrier waits are covered by the other.

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;        // 8 warps; warp w reads TMEM sub-partition w % 4
constexpr int kCtasPerSm = 2;  // two CTAs share an SM: one's barrier waits are the other's issue slots
constexpr int NCG = NT / 128;  // warps per TMEM sub-partition, each taking one group of columns
constexpr uint32_t kTmemCols = 256;  // D1 (64 columns) + W (DK) + U^T (64), a half of tensor memory
constexpr int kInvBarrier = 1;       // named barrier of warps 0-3, which take levels 1 and 2 of the inverse
constexpr int kItemsPerCta = 2;
constexpr float kLog2e = 1.4426950408889634f;  // log2(e)

template <int DK, int DV>
struct IntraTcSmem {
    // fp16 operand tiles (16-bit K-major layout)
    uint16_t kq[2 * C * DK];  // [K ; Q*scale] tile from the prep kernel (bulk copy), 128 rows; its
                              // K rows are also W's B operand, read MN-major
    uint16_t bv[DV * C];      // V^T tile of the current head (bulk copy), DV rows x C
    uint16_t t[C * C];        // T diag(beta), C rows x C: U's operand
    uint16_t te[C * C];       // T diag(beta e^gamma), same layout: W's operand
    float a[C][C + 1];     // A (fp32)
    float tf[2][32][36];   // T (fp32) in its two 32x32 diagonal blocks: what the next levels read
    float m[32][36];       // A21 T11
    float y[2][16][20];    // A21 D1 inside each 32x32 diagonal block (rows 16-byte aligned)
    float2 gb[2][C];       // (g, beta) of the two heads in flight
    // per-row gate quantities of a value head, double-buffered by head parity: the tiles that need
    // only head j's gates are written while head j + 1's gates are scanned
    float gam[2][C], beta[2][C], eg[2][C];
    float gam2[2][C];      // gamma * log2(e): the exponents of the decay factors in base 2
    float bge[2][C];       // beta e^gamma: the column factor of W's operand
    float fkt[2][C];       // e^{gamma_n - gamma_s} (0 past the chunk end): row factor of K~
    unsigned long long bar_mma, bar_kq, bar_v, bar_g[2];
    uint32_t tmem_base;
    int next_item;         // thread 0's latest grab, for the other threads
};

__device__ __forceinline__ void bar_sync_n(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// idx -> (row, first column) of an 8-column group of a 16-bit K-major tile with R rows: 8
// consecutive lanes take 8 consecutive rows, i.e. one 128-byte core matrix
template <int R>
__device__ __forceinline__ void tile_coord8(int idx, int& r, int& k8) {
    const int rr = idx & 7, rest = idx >> 3;
    r = 8 * (rest % (R / 8)) + rr;
    k8 = 8 * (rest / (R / 8));
}

// 8 fp16 at byte offset `off` of a 16-bit tile (one 16-byte load) -> 8 floats
__device__ __forceinline__ void load_h8(const void* tile, uint32_t off, float* v) {
    const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(tile) + off);
    const float2 a = tc::unpack_f16(w.x), b = tc::unpack_f16(w.y), c = tc::unpack_f16(w.z), e = tc::unpack_f16(w.w);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y; v[4] = c.x; v[5] = c.y; v[6] = e.x; v[7] = e.y;
}

// 8 floats -> 8 fp16 at byte offset `off` of a 16-bit tile (one 16-byte store)
__device__ __forceinline__ void store_h8(void* tile, uint32_t off, const float* v) {
    *reinterpret_cast<uint4*>(reinterpret_cast<char*>(tile) + off) =
        make_uint4(tc::pack_f16(v[0], v[1]), tc::pack_f16(v[2], v[3]), tc::pack_f16(v[4], v[5]),
                   tc::pack_f16(v[6], v[7]));
}


template <int DK, int DV>
__global__ void __launch_bounds__(NT, kCtasPerSm) intra_tc_kernel(ExtendArgs p, int seg) {
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
    extern __shared__ __align__(16) unsigned char smem_raw[];
    IntraTcSmem<DK, DV>& sm = *reinterpret_cast<IntraTcSmem<DK, DV>*>(smem_raw);
    if (tid == 0) sm.next_item = grab();
    __syncthreads();
    int item = sm.next_item;
    if (item < 0) return;
    const uint32_t bar = tc::smem_u32(&sm.bar_mma), bar_kq = tc::smem_u32(&sm.bar_kq);
    constexpr uint32_t KQ_BYTES = 2 * C * DK * 2, VT_BYTES = DV * C * 2, GB_BYTES = C * 8;
    const uint32_t bar_v = tc::smem_u32(&sm.bar_v);
    auto kq_src = [&](int it) { return p.KQ + (size_t)it * (2 * C * DK); };  // [K ; Q] tiles are [chunk][hk]
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

    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
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
    // blocks of T above the diagonal are zero for every head: in the tile, and in the two 16x16
    // corners of the 32x32 diagonal blocks that the inverse reads back
    for (int e = tid; e < C * C; e += NT) sm.t[e] = sm.te[e] = 0;
    for (int e = tid; e < 2 * 256; e += NT) sm.tf[e >> 8][(e >> 4) & 15][16 + (e & 15)] = 0.f;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    // D1: 64 columns; W: M = 64 layout, DK columns; U^T: M = DV, 64 columns
    const uint32_t tD1 = tm, tW = tm + 64, tU = tm + 64 + DK;
    const int sp = warp & 3, cg = warp >> 2;  // TMEM sub-partition, column group
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    // completed uses of each barrier so far, identical in every thread (parity = count & 1)
    uint32_t n_kq = 0, n_v = 0, n_g[2] = {0u, 0u}, ph_mma = 0;
    bool ok = true;
    int done = 0;
    while (ok && item >= 0) {
    int nxt = -1;
    // At most kItemsPerCta items, then the CTA ends: its SM goes to whatever waits, first of all a
    // state-pass CTA of the previous segment (its stream has the higher priority).
    if (tid == 0 && ++done < kItemsPerCta) nxt = grab();
    if (tid == 0) sm.next_item = nxt;  // read by every thread after the barrier below
    const int id = item / HK, hk = item % HK;
    const int n = p.chunk_tab[id].z;
    if (tid == 0 && nxt >= 0) prefetch_l2(nxt);
    if (tid == 0) {
        ok = tc::mbar_wait(bar_kq, n_kq & 1u);
        if (ok) {  // D1 = [K ; Q] K^T
            const uint32_t base = tc::smem_u32(sm.kq);
            constexpr uint32_t idesc = tc::idesc_f16(128, 64);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                tc::mma_f16(tD1, tc::desc_kmajor(base, 2 * C, s), tc::desc_kmajor(base, 2 * C, s), idesc, s > 0);
            tc::mma_commit(bar);
        }
    }
    // every thread reads the [K ; Q] tile below
    ok = ok && tc::mbar_wait(bar_kq, n_kq & 1u);
    ++n_kq;
    ok = __syncthreads_and(ok);
    nxt = sm.next_item;

    // W and U^T of value head jj (accumulators in tensor memory) -> their workspace tiles
    auto epilogue = [&](int jj) {
        const size_t hrow = (size_t)id * HV + hk * G + jj;
        char* WQg = reinterpret_cast<char*>(p.WQ + hrow * (2 * C * DK));
        char* Ug = reinterpret_cast<char*>(p.U + hrow * (DV * C));  // U^T, K-major tile: DV rows (j) x C
        {  // W rows -> [W ; Qg] tile rows 0..63 (tf32, K-major); U -> U^T tile (fp32, K-major).
           // M = 64 layout: lanes 0-15 of sub-partition sp hold rows 16 sp .. 16 sp + 15;
           // the warps of a sub-partition take one group of columns each
            const bool valid = lane < 16;
            const int r = sp * 16 + lane;
#pragma unroll
            for (int c0 = cg * (DK / NCG); c0 < (cg + 1) * (DK / NCG); c0 += 16) {
                float v[16];
                tc::tmem_ld16(tW + lane_base + c0, v);
                tc::tmem_ld_wait();
                if (valid) {
                    store_h8(WQg, tc::kmajor_off16(r, c0, 2 * C), v);
                    store_h8(WQg, tc::kmajor_off16(r, c0 + 8, 2 * C), v + 8);
                }
            }
            {  // U^T row j (M = DV layout), the warp's group of C / NCG columns r
                const bool vj = DV == 128 || lane < 16;
                const int jr = DV == 128 ? sp * 32 + lane : sp * 16 + lane;
#pragma unroll
                for (int c0 = cg * (C / NCG); c0 < (cg + 1) * (C / NCG); c0 += 16) {
                    float v[16];
                    tc::tmem_ld16(tU + lane_base + c0, v);
                    tc::tmem_ld_wait();
                    if (vj) {
                        store_h8(Ug, tc::kmajor_off16(jr, c0, DV), v);
                        store_h8(Ug, tc::kmajor_off16(jr, c0 + 8, DV), v + 8);
                    }
                }
            }
        }
    };
    // warp 0: wait for value head jj's gates and scan them (warp-uniform result)
    auto scan_gates = [&](int jj) -> bool {
        const int bb = jj & 1;
        bool okg = tc::mbar_wait(tc::smem_u32(&sm.bar_g[bb]), n_g[bb] & 1u);
        ++n_g[bb];
        okg = __all_sync(0xffffffffu, okg);
        if (okg) {  // inclusive scan of g over the chunk, two rows per lane
            const float2 g0 = sm.gb[bb][2 * lane], g1 = sm.gb[bb][2 * lane + 1];
            const float pair = g0.x + g1.x;
            float incl = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const float gA = incl - pair + g0.x;
            sm.gam[bb][2 * lane] = gA;
            sm.gam[bb][2 * lane + 1] = incl;
            sm.gam2[bb][2 * lane] = gA * kLog2e;
            sm.gam2[bb][2 * lane + 1] = incl * kLog2e;
            sm.beta[bb][2 * lane] = g0.y;
            sm.beta[bb][2 * lane + 1] = g1.y;
            sm.eg[bb][2 * lane] = __expf(gA);
            sm.eg[bb][2 * lane + 1] = __expf(incl);
            sm.bge[bb][2 * lane] = g0.y * sm.eg[bb][2 * lane];
            sm.bge[bb][2 * lane + 1] = g1.y * sm.eg[bb][2 * lane + 1];
            const float gn = __shfl_sync(0xffffffffu, (n - 1) & 1 ? incl : gA, (n - 1) >> 1);
            sm.fkt[bb][2 * lane] = 2 * lane < n ? __expf(gn - gA) : 0.f;
            sm.fkt[bb][2 * lane + 1] = 2 * lane + 1 < n ? __expf(gn - incl) : 0.f;
        }
        return okg;
    };
    for (int j = 0; j < G && ok; ++j) {
        const int h = hk * G + j, hb = j & 1;
        const size_t ch_h = (size_t)id * HV + h;
        char* WQg = reinterpret_cast<char*>(p.WQ + ch_h * (2 * C * DK));
        char* AQg = reinterpret_cast<char*>(p.AQ + ch_h * (C * C));
        char* KTg = reinterpret_cast<char*>(p.KT + ch_h * (DK * C));
        if (j == 0) {  // head 0's gates, and D1; later heads' gates are scanned during the previous head's MMA
            bool okv = warp == 0 ? scan_gates(0) : true;
            okv = okv && tc::mbar_wait(bar, ph_mma);
            ph_mma ^= 1;
            ok = __syncthreads_and(okv);
            if (!ok) break;
            tc::fence_after_sync();
        }
        {  // A (sub-partitions 0-1: k.k rows) and the masked decayed q.k tile (2-3: q.k rows) from D1;
           // the warps of a sub-partition take one group of C / NCG columns each.  The exponents are
           // formed without branches (a masked entry gets -inf, whose exponential is 0) so the
           // sixteen exponentials of a 16-column block issue back to back; a block that lies wholly
           // above the diagonal only gets zeros.
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
                    // entry i is kept when column c0 + i lies below the diagonal (on it, for q.k) of a
                    // row inside the chunk
                    const int lim = r < n ? r - c0 + (qrow ? 1 : 0) : 0;
                    const float gr = sm.gam2[hb][r];
#pragma unroll
                    for (int q = 0; q < 16; q += 4) {
                        const float4 gs = *reinterpret_cast<const float4*>(&sm.gam2[hb][c0 + q]);
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
                    const float br = sm.beta[hb][r];
#pragma unroll
                    for (int i = 0; i < 16; ++i) sm.a[r][c0 + i] = br * e[i];
                } else {
                    store_h8(AQg, tc::kmajor_off16(r, c0, C), e);
                    store_h8(AQg, tc::kmajor_off16(r, c0 + 8, C), e + 8);
                }
            }
        }
        if (j > 0) epilogue(j - 1);  // the previous head's W and U^T, from other tensor-memory columns
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        // T = (I + A)^{-1}, by blocks.  Every final entry goes straight into the K-major fp16 tile of
        // T diag(beta) (the A operand of W and U); the fp32 copy tf holds what the next level reads.
        //   level 1: the four diagonal 16x16 blocks by forward substitution, one column per lane held
        //            in registers (t_r = [r == c] - sum_{s<r} A_rs t_s; the s = r-1 term goes last so
        //            one FMA per row sits on the dependent chain); the other warps meanwhile write the
        //            tiles that need only the gates: the state pass's K~ = diag(e^{gamma_n-gamma}) K
        //            and the rows Qg = diag(e^gamma) Q of [W ; Qg], and gamma.
        //   level 2: within each 32x32 diagonal block, X = -D2 (A21 D1).
        //   level 3: T21 = -T22 (A21 T11) for the lower-left 32x32 block.
        auto put_t = [&](int r, int c, float v) {  // T entry (r, c) into both operand tiles
            const uint32_t off = tc::kmajor_off16(r, c, C);
            const uint32_t w = tc::pack_f16(v * sm.beta[hb][c], v * sm.bge[hb][c]);
            *reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(sm.t) + off) = (uint16_t)(w & 0xffffu);
            *reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(sm.te) + off) = (uint16_t)(w >> 16);
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
                    const float* arow = &sm.a[o + r][o];
                    float acc[2] = {r == c ? 1.f : 0.f, 0.f};
#pragma unroll
                    for (int s = 0; s + 1 < r; ++s) acc[s & 1] = fmaf(-arow[s], t[s], acc[s & 1]);
                    const float base = acc[0] + acc[1];
                    t[r] = r > 0 ? fmaf(-arow[r - 1], t[r - 1], base) : base;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    sm.tf[warp >> 1][16 * (warp & 1) + r][16 * (warp & 1) + c] = t[r];
                    put_t(o + r, o + c, t[r]);
                }
            }
            // levels 1 -> 2 synchronise warps 0-3 only: the other warps keep writing the gate-only
            // tiles meanwhile
            bar_sync_n(kInvBarrier, 128);
            // Level 2 tiles the outputs in registers: a thread takes four consecutive columns of one
            // row, so each step of a dot product is one (broadcast) load of the left factor and one
            // 16-byte load of the right one for four FMAs; the shared-memory pipe, not the FMAs,
            // bounds these small products.
            {  // level 2 (threads 0..127): 32-block bb, row r, columns c4 .. c4 + 3
                const int bb = tid >> 6, r = (tid >> 2) & 15, c4 = 4 * (tid & 3);
                const int o0 = 32 * bb, o1 = o0 + 16;
                {
                    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int s = 0; s < 16; ++s)  // Y = A21 D1
                        fma4(y, sm.a[o1 + r][o0 + s], *reinterpret_cast<const float4*>(&sm.tf[bb][s][c4]));
                    *reinterpret_cast<float4*>(&sm.y[bb][r][c4]) = y;
                }
                bar_sync_n(kInvBarrier, 128);
                {
                    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int s = 0; s < 16; ++s)  // X = -D2 Y
                        fma4(x, sm.tf[bb][16 + r][16 + s], *reinterpret_cast<const float4*>(&sm.y[bb][s][c4]));
                    x = make_float4(-x.x, -x.y, -x.z, -x.w);
                    *reinterpret_cast<float4*>(&sm.tf[bb][16 + r][c4]) = x;
                    put_t(o1 + r, o0 + c4, x.x);
                    put_t(o1 + r, o0 + c4 + 1, x.y);
                    put_t(o1 + r, o0 + c4 + 2, x.z);
                    put_t(o1 + r, o0 + c4 + 3, x.w);
                }
            }
        } else {  // row scalings of the [K ; Q] tile, 8 features per 16-byte vector
            constexpr int NW = NT - 128;
            for (int idx = tid - 128; idx < 2 * C * DK / 8; idx += NW) {
                int r, k8;
                tile_coord8<2 * C>(idx, r, k8);  // a warp's 32 rows lie in one half of the tile
                const uint32_t off = tc::kmajor_off16(r, k8, 2 * C);
                float v[8];
                load_h8(sm.kq, off, v);
                const float e = r < C ? sm.fkt[hb][r] : sm.eg[hb][r - C];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] *= e;
                if (r < C)
                    store_h8(KTg, tc::kmajor_off16(r, k8, C), v);  // K~: a tile of C rows s
                else
                    store_h8(WQg, off, v);  // rows Qg: same offsets in [W ; Qg]
            }
            if (tid - 128 < C) p.gam[ch_h * C + tid - 128] = sm.gam[hb][tid - 128];
        }
        __syncthreads();
        // Level 3 reads one operand as a warp-wide broadcast and skips the zero blocks of the
        // triangular factors: T11[s][c] = 0 for s < c and T22[r][s] = 0 for s > r.
        static_assert(NT / 32 >= 8 && 32 % (NT / 32) == 0, "level 3 maps 8 column groups, then row groups, onto the warps");
        if (warp < 8) {  // level 3a: P = A21 T11; warp w takes columns 4w .. 4w + 3, lane = row
            const int r = lane, c4 = 4 * warp;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int s = c4; s < 32; ++s)
                fma4(acc, sm.a[32 + r][s], *reinterpret_cast<const float4*>(&sm.tf[0][s][c4]));
            *reinterpret_cast<float4*>(&sm.m[r][c4]) = acc;
        }
        __syncthreads();
        {  // level 3b: T21 = -T22 P; warp w takes RPW consecutive rows of the block, lane = column
            constexpr int RPW = 32 / (NT / 32);
            const int r0 = RPW * warp, c = lane;
            float acc[RPW];
#pragma unroll
            for (int i = 0; i < RPW; ++i) acc[i] = 0.f;
            for (int s4 = 0; s4 < r0 + RPW; s4 += 4) {
                const float p0 = sm.m[s4][c], p1 = sm.m[s4 + 1][c], p2 = sm.m[s4 + 2][c], p3 = sm.m[s4 + 3][c];
#pragma unroll
                for (int i = 0; i < RPW; ++i) {
                    const float4 t = *reinterpret_cast<const float4*>(&sm.tf[1][r0 + i][s4]);
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
        bool okm = true;
        if (tid == 0) {  // W = (T diag(beta e^gamma)) K (M = 64, K read MN-major from the [K ; Q] tile),
                         // U^T = V^T (T diag(beta))^T (M = DV)
            okm = tc::mbar_wait(bar_v, n_v & 1u);
            if (okm) {
                const uint32_t bt = tc::smem_u32(sm.t), bte = tc::smem_u32(sm.te), bkq = tc::smem_u32(sm.kq);
                const uint32_t bvv = tc::smem_u32(sm.bv);
                constexpr uint32_t iw = tc::idesc_f16(64, DK) | tc::kTransposeB, iu = tc::idesc_f16(DV, 64);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    tc::mma_f16(tW, tc::desc_kmajor(bte, C, s), tc::desc_mnmajor16(bkq, 2 * C, s), iw, s > 0);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    tc::mma_f16(tU, tc::desc_kmajor(bvv, DV, s), tc::desc_kmajor(bt, C, s), iu, s > 0);
                tc::mma_commit(bar);
            }
        }
        bool okn = true;
        if (warp == 0 && j + 1 < G) okn = scan_gates(j + 1);  // into the other gate buffer
        ++n_v;
        ok = okm && okn && tc::mbar_wait(bar, ph_mma);  // okm is false only on tid 0, if the V tile never came
        ph_mma ^= 1;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        if (tid == 0) {  // the V^T tile and gate buffer b are free again; after the last head, so is [K ; Q]
                         // (the last head's epilogue reads only tensor memory)
            if (j + 1 < G) fetch_v(item, j + 1);
            if (j + 2 < G) fetch_g(item, j + 2);
            if (j == G - 1 && nxt >= 0) {  // the next item's tiles land during this epilogue
                fetch_kq(nxt);
                fetch_g(nxt, 0);
                if (G > 1) fetch_g(nxt, 1);
                fetch_v(nxt, 0);
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    }
    if (ok) {
        epilogue(G - 1);
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
    if (warp == 0) tc::tmem_dealloc(tm, kTmemCols);
}

}  // namespace

template <int DK, int DV>
cudaError_t launch_intra(const ExtendArgs& p, int seg, cudaStream_t s) {
    const size_t shm = sizeof(IntraTcSmem<DK, DV>);
    cudaError_t e = cudaFuncSetAttribute(intra_tc_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // CTAs of up to kItemsPerCta (chunk, qk head) items each, enough for the most a segment can hold
    (void)sms;
    const long long items = ((long long)p.max_chunks + p.nseg - 1) / p.nseg * p.d.HK;
    const int grid = (int)((items + kItemsPerCta - 1) / kItemsPerCta);
    intra_tc_kernel<DK, DV><<<grid, NT, shm, s>>>(p, seg);
    return cudaGetLastError();
}

template cudaError_t launch_intra<64, 64>(const ExtendArgs&, int, cudaStream_t);
template cudaError_t launch_intra<64, 128>(const ExtendArgs&, int, cudaStream_t);
template cudaError_t launch_intra<128, 64>(const ExtendArgs&, int, cudaStream_t);
template cudaError_t launch_intra<128, 128>(const ExtendArgs&, int, cudaStream_t);

}  // namespace gdn
