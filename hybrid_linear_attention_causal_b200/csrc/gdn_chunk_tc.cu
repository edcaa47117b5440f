// Per-chunk step of the chunked GDN prefill on tcgen05 tensor cores (sm_100a):
// the chunk's conv1d + SiLU, L2 norm and gates fused with the intra-chunk
// WY/UT products, so no intermediate of the chunk goes through global memory
// before the tiles the serial state pass reads.
//
// One (chunk, qk head) item at a time; an item serves the G value heads that
// share the qk head.  For a chunk of n <= 64 rows starting at packed row t0:
//
//   rows t0-3 .. t0+n-1 of the item's channels and their conv weights are
//   staged in shared memory (the 3 rows before the chunk come from the
//   previous chunk of the same sequence, or from the conv-state slot for a
//   sequence's first chunk); y = SiLU(conv1d(x)), q and k L2-normalised (q
//   carries the output scale), g = -exp(A_log) softplus(a + dt_bias),
//   beta = sigmoid(b), gamma_r = sum_{s<=r} g_s;
//
//   D1  = [K; Q] K^T                          (fp16 MMA, M=128 N=64 K=dk)
//   A   = beta_r e^{gamma_r-gamma_s} (k_r.k_s)        s < r   (strictly lower)
//   Aqk = e^{gamma_r-gamma_s} (q_r.k_s)               s <= r
//   T   = (I + A)^{-1}
//   W^T = K^T (T diag(beta e^gamma))^T        (fp16 MMA, M=dk N=64 K=64; K read MN-major)
//   U^T = V^T (T diag(beta))^T                (fp16 MMA, M=dv N=64 K=64; V read MN-major)
//
// (the WY/UT form of the gated delta rule, Gated DeltaNet, Yang, Kautz and
// Hatamizadeh, ICLR 2025).  The triangular inverse runs in two stages: the
// four 16x16 diagonal blocks of I + A by forward substitution in fp32 on the
// CUDA cores (D = their inverses, block diagonal), then, with L the strictly
// block-lower part of A and E = D L (nilpotent: E^4 = 0),
//   T = (I + E)^{-1} D = (I + E^2)(I - E) D
// in three rounds of fp16 products on the tensor core (E; E^2 and
// Q = (I - E) D together; T = (I + E^2) Q), each result rounded to fp16 once
// on its way back to shared memory.  T's diagonal blocks are D itself and E's entries are L's scaled by
// D, so these roundings add nothing measurable to the fp16 rounding of
// T diag(beta) that W and U need anyway.
//
// The item writes, as fp16 tiles in the tensor core's 128-byte swizzled
// shared-memory layout (so the state pass copies them verbatim): [K ; Q] once
// per (chunk, qk head), and per (chunk, value head) W^T, U^T and the masked
// decayed q.k; plus a per-row gate vector in fp32.  The chunk's rows past the
// end of a ragged chunk are zero in every tile.  The rows of the next value
// head and of the next item are copied into shared memory asynchronously while
// the current one computes.  One thread issues the MMAs; the eight
// warps read their sub-partition's 32-lane slice of tensor memory (two warps
// per slice, one group of columns each) for the CUDA-core steps.  Two CTAs
// share an SM (half of its tensor memory and shared memory each), so one
// CTA's barrier waits are covered by the other.

#include <cuda_fp16.h>

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;        // 8 warps; warp w reads TMEM sub-partition w % 4
constexpr int kCtasPerSm = 2;
constexpr uint32_t kTmemCols = 256;  // D1, X1 / W^T, X2 / U^T: 64 columns each, a half of tensor memory
constexpr int kItemsPerCta = 2;
constexpr float kLog2e = 1.4426950408889634f;  // log2(e)

template <typename T, int DK, int DV>
struct ChunkShape {
    static constexpr int PADE = 16 / (int)sizeof(T);     // staged-row padding (one 16-byte vector)
    static constexpr int LDQK = 2 * DK + PADE;           // staged q,k row: k channels, then q channels
    static constexpr int LDV = DV + PADE;                // staged v row
    static constexpr size_t XQK = (size_t)(C + 3) * LDQK * sizeof(T);
};

template <typename T, int DK, int DV>
struct ChunkSmem {
    using S = ChunkShape<T, DK, DV>;
    // fp16 operand tiles in the 128-byte swizzled layout; each starts on a 1024-byte boundary
    uint16_t kq[2 * C * DK];  // [K ; Q*scale], 128 rows x DK: D1's operands, W's B (K rows read MN-major)
    uint16_t vr[C * DV];      // V of the current value head, C rows x DV: U's A (read MN-major)
    // the inverse's tiles (64 x 64 fp16 each) and fp32 diagonal blocks, or the raw rows being staged
    struct Inv {
        uint16_t tile[4][C * C];  // roles rotate: D | L | E | I - E, then I + E^2 in L's, P in E's, and
                                  // finally T diag(beta) in D's and T diag(beta e^gamma) in I - E's
        float dg[4][16][20];      // the diagonal 16x16 blocks of A (fp32), rows padded
    };
    static constexpr size_t UBYTES = S::XQK > sizeof(Inv) ? S::XQK : sizeof(Inv);
    alignas(1024) unsigned char u[UBYTES];
    alignas(16) T xv[(C + 3) * S::LDV];  // the staged v rows of one value head
    alignas(16) T wq[2 * DK * 4];  // conv taps of the item's k then q channels
    alignas(16) T wv[DV * 4];      // conv taps of the current value head's channels
    float2 gb[C];                  // (g, beta) of the current value head
    // gamma, gamma log2(e) (read as float4), beta, beta e^gamma
    alignas(16) float gam[C];
    alignas(16) float gam2[C];
    alignas(16) float beta[C];
    alignas(16) float bge[C];
    unsigned long long bar_mma;
    uint32_t tmem_base;
    int next_item;
    int prefetch_item;        // the item after the current one, or -1
};

template <typename T, int DK, int DV>
constexpr size_t chunk_smem_bytes() {
    return sizeof(ChunkSmem<T, DK, DV>) + 1024;  // + room to align the tiles on 1024 bytes
}

// 4 consecutive elements -> 4 floats (8-byte load for bf16, 16-byte for fp32)
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

// 8 floats -> 8 fp16 (one 16-byte store) at byte offset `off` of a tile
__device__ __forceinline__ void store_h8(char* tile, uint32_t off, const float* v) {
    *reinterpret_cast<uint4*>(tile + off) = make_uint4(tc::pack_f16(v[0], v[1]), tc::pack_f16(v[2], v[3]),
                                                       tc::pack_f16(v[4], v[5]), tc::pack_f16(v[6], v[7]));
}

// two fp32 lanes at once: d = a * b + c and d = a * b, each lane rounded exactly as fmaf / __fmul_rn
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}
// SiLU of two values: SiLU(x) = x sigmoid(x) = h + h tanh(h), h = x / 2, with the hardware tanh (one
// MUFU operation; its error is below the fp16 rounding every conv output goes through)
__device__ __forceinline__ float2 silu2(float2 x) {
    const float2 h = fmul2(make_float2(0.5f, 0.5f), x);
    float2 t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.x) : "f"(h.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.y) : "f"(h.y));
    return ffma2(h, t, h);
}

// conv1d (K = 4) + SiLU of 8 consecutive output rows r0 .. r0+7 (rows >= n give 0) of 4 consecutive
// channels, from staged rows r0 .. r0+10 (staged row i holds packed row t0 - 3 + i) with a sliding
// window; `xs` points at the first of the 4 channels in staged row 0, `w` at their 16 taps.  Channels
// go in pairs through the two-lane FMA, each channel's taps accumulated in the same order as one
// fmaf chain would.
template <typename T>
__device__ __forceinline__ void conv8x4(const T* xs, int ld, const T* w, const T* bias, int r0, int n,
                                        float (&y)[8][4]) {
    float wt[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) load4(w + 4 * u, wt[u]);
    float2 w01[4], w23[4];  // tap j of channels (0, 1) and (2, 3)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        w01[jj] = make_float2(wt[0][jj], wt[1][jj]);
        w23[jj] = make_float2(wt[2][jj], wt[3][jj]);
    }
    float b[4] = {0.f, 0.f, 0.f, 0.f};
    if (bias) load4(bias, b);
    float win[4][4];
#pragma unroll
    for (int i = 0; i < 3; ++i) load4(xs + (size_t)(r0 + i) * ld, win[i]);
#pragma unroll
    for (int o = 0; o < 8; ++o) {
        load4(xs + (size_t)(r0 + o + 3) * ld, win[(o + 3) & 3]);
        float2 a01 = make_float2(b[0], b[1]), a23 = make_float2(b[2], b[3]);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const float* wr = win[(o + jj) & 3];
            a01 = ffma2(w01[jj], make_float2(wr[0], wr[1]), a01);
            a23 = ffma2(w23[jj], make_float2(wr[2], wr[3]), a23);
        }
        if (r0 + o < n) {
            a01 = silu2(a01);
            a23 = silu2(a23);
        } else {
            a01 = a23 = make_float2(0.f, 0.f);
        }
        y[o][0] = a01.x;
        y[o][1] = a01.y;
        y[o][2] = a23.x;
        y[o][3] = a23.y;
    }
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, kCtasPerSm) chunk_tc_kernel(ExtendArgs p, int seg) {
    using S = ChunkShape<T, DK, DV>;
    using Sm = ChunkSmem<T, DK, DV>;
    static_assert(DK % 32 == 0 && DV % 32 == 0, "channel groups of 4 per lane");
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
    char* tiles = reinterpret_cast<char*>(inv.tile);
    auto tile_b = [&](int i) { return tiles + (size_t)i * C * C * 2; };
    auto tile_s = [&](int i) { return tc::smem_u32(tiles) + (uint32_t)i * C * C * 2; };

    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    // D1 at tm; the inverse's accumulators X1, X2 (M = 64 layout) at tm + 64 and tm + 128, then W^T
    // (M = DK) and U^T (M = DV) in their places: 64 columns each
    const uint32_t tD1 = tm, tX1 = tm + 64, tX2 = tm + 128, tW = tm + 64, tU = tm + 128;
    static_assert(192 <= (int)kTmemCols, "tensor-memory layout");
    const int sp = warp & 3, cg = warp >> 2;  // TMEM sub-partition, column group
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    uint32_t ph_mma = 0;
    bool ok = true;
    int done = 0;
    float amax = 0.f;  // largest magnitude this thread rounded to fp16 among v, T's tiles, W and U
    // all threads wait for the tensor core's latest commit
    auto wait_mma = [&]() -> bool {
        const bool r = __syncthreads_and(tc::mbar_wait(bar, ph_mma));
        ph_mma ^= 1;
        tc::fence_after_sync();
        return r;
    };
    // an M = 64 accumulator (rows 16 sp + lane in lanes 0-15 of sub-partition sp) -> 32 columns of this
    // warp's group for row m: `f(m, c0, v16)` per 16 columns
    auto read64 = [&](uint32_t t0, auto&& f) {
#pragma unroll
        for (int c0 = 32 * cg; c0 < 32 * cg + 32; c0 += 16) {
            float v[16];
            tc::tmem_ld16(t0 + lane_base + c0, v);
            tc::tmem_ld_wait();
            if (lane < 16) f(sp * 16 + lane, c0, v);
        }
    };

    constexpr int VE = 16 / (int)sizeof(T);  // elements per 16-byte vector
    // where an item's rows are: packed row t0 .. t0+n-1 of sequence seq, chunk cidx of it
    struct Pos {
        int id, hk, t0, n, cidx;
        bool init;
        const T* cs;  // the sequence's conv-state slot
    };
    auto pos_of = [&](int it) {
        Pos q;
        q.id = it / HK;
        q.hk = it % HK;
        const int4 ch = p.chunk_tab[q.id];
        q.t0 = ch.y;
        q.n = ch.z;
        q.cidx = ch.w;
        q.init = p.has_init ? p.has_init[ch.x] != 0 : true;
        q.cs = reinterpret_cast<const T*>(p.conv_state) + (size_t)p.slots[ch.x] * d.conv_dim * 3;
        return q;
    };
    // Staging: packed rows t0-3 .. t0+n-1 of some channels into shared rows of stride `ld` (staged row i
    // <-> packed row t0 - 3 + i), vector v (VE elements) of a row from global channel chan(v), by
    // asynchronous 16-byte copies; for a sequence's first chunk the 3 rows before it come from the
    // conv-state slot (channel-major there, so element by element, synchronously).
    auto stage_rows = [&](T* dst, int ld, int vpr, const Pos& q, auto&& chan) {
        const int r_lo = q.cidx > 0 ? 0 : 3;
        const int nv = (q.n + 3 - r_lo) * vpr;
        for (int e = tid; e < nv; e += NT) {
            const int i = r_lo + e / vpr, v = e % vpr;
            tc::cp_async16(dst + (size_t)i * ld + v * VE, x + (size_t)(q.t0 - 3 + i) * d.conv_dim + chan(v));
        }
        if (q.cidx == 0)
            for (int e = tid; e < 3 * vpr * VE; e += NT) {
                const int i = e / (vpr * VE), c = e % (vpr * VE);
                dst[(size_t)i * ld + c] = q.init ? q.cs[(size_t)(chan(c / VE) + c % VE) * 3 + i] : from_f<T>(0.f);
            }
    };
    // the q,k rows (columns k then q) and their taps
    auto stage_qk = [&](const Pos& q) {
        const int ck0 = d.HK * DK + q.hk * DK, cq0 = q.hk * DK;
        constexpr int VPR = 2 * DK / VE, VK = DK / VE;
        stage_rows(xs, S::LDQK, VPR, q, [&](int v) { return v < VK ? ck0 + v * VE : cq0 + (v - VK) * VE; });
        constexpr int WV = DK * 4 / VE;  // vectors of one part's taps
        for (int e = tid; e < 2 * WV; e += NT)
            tc::cp_async16(sm.wq + (e < WV ? 0 : DK * 4) + (e % WV) * VE,
                           w + (size_t)(e < WV ? ck0 : cq0) * 4 + (e % WV) * VE);
    };
    // value head h's rows and taps
    auto stage_v = [&](const Pos& q, int h) {
        const int cv0 = 2 * d.HK * DK + h * DV;
        stage_rows(sm.xv, S::LDV, DV / VE, q, [&](int v) { return cv0 + v * VE; });
        for (int e = tid; e < DV * 4 / VE; e += NT) tc::cp_async16(sm.wv + e * VE, w + (size_t)cv0 * 4 + e * VE);
    };
    // the raw gate inputs of value head h (threads NT-C .. NT-1, one row each), held in registers as
    // loaded (nothing waits for the loads) until commit_gates turns them into (g, beta) in shared memory
    T ga = from_f<T>(0.f), gbv = from_f<T>(0.f);
    auto load_gates = [&](const Pos& q, int h) {
        if (tid >= NT - C) {
            const int r = tid - (NT - C);
            if (r < q.n) {
                const size_t row = (size_t)(q.t0 + r) * HV + h;
                ga = reinterpret_cast<const T*>(p.a)[row];
                gbv = reinterpret_cast<const T*>(p.b)[row];
            }
        }
    };
    auto commit_gates = [&](int n, int h) {  // zero past the end of the chunk
        if (tid >= NT - C) {
            const int r = tid - (NT - C);
            sm.gb[r] = r < n ? make_float2(-expf(p.A_log[h]) * softplus_f(to_f(ga) + p.dt_bias[h]), sigmoid_f(to_f(gbv)))
                             : make_float2(0.f, 0.f);
        }
    };
    {
        const Pos q = pos_of(item);
        stage_qk(q);
        stage_v(q, q.hk * G);
        load_gates(q, q.hk * G);
    }

    while (ok && item >= 0) {
        int nxt = -1;
        // At most kItemsPerCta items, then the CTA ends: its SM goes to whatever waits, first of all a
        // state-pass CTA of the previous segment (its stream has the higher priority).
        if (tid == 0 && ++done < kItemsPerCta) nxt = grab();
        if (tid == 0) sm.prefetch_item = nxt;  // read by every thread after the staging barrier
        const Pos q = pos_of(item);
        const int id = q.id, hk = q.hk, n = q.n;
        const int ck0 = d.HK * DK + hk * DK, cq0 = hk * DK;  // first k / q channel
        // the item's rows and the first value head's, staged by the copies issued before
        commit_gates(n, hk * G);
        tc::cp_async_wait_all();
        __syncthreads();
        {  // the next item's rows into L2 while this one computes: one 128-byte line per prefetch, spread
           // over every thread (its q, k and v pieces of each row: 2 DK + G DV elements)
            const int pi = sm.prefetch_item;
            if (pi >= 0) {
                const int4 chn = p.chunk_tab[pi / HK];
                const int hkn = pi % HK;
                const int r0 = chn.w > 0 ? chn.y - 3 : chn.y, nr = chn.y + chn.z - r0;
                constexpr int LQ = DK * (int)sizeof(T) / 128, LV = DV * (int)sizeof(T) / 128;  // lines per piece
                const int lpr = 2 * LQ + G * LV;                                                 // lines per row
                for (int e = tid; e < nr * lpr; e += NT) {
                    const int r = r0 + e / lpr, l = e % lpr;
                    const T* row = x + (size_t)r * d.conv_dim;
                    const T* a_ = l < LQ ? row + hkn * DK + l * (128 / sizeof(T))
                                : l < 2 * LQ ? row + d.HK * DK + hkn * DK + (l - LQ) * (128 / sizeof(T))
                                             : row + 2 * d.HK * DK + hkn * G * DV + (l - 2 * LQ) * (128 / sizeof(T));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(a_));
                }
                // and its gate inputs: rows t0 .. t0+n-1 of a and b are one contiguous span each
                const char* ga0 = reinterpret_cast<const char*>(reinterpret_cast<const T*>(p.a) + (size_t)chn.y * HV);
                const char* gb0 = reinterpret_cast<const char*>(reinterpret_cast<const T*>(p.b) + (size_t)chn.y * HV);
                const int glines = (int)(((size_t)chn.z * HV * sizeof(T) + 127) / 128);
                for (int e = tid; e < 2 * glines; e += NT)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"((e < glines ? ga0 : gb0) + (size_t)(e % glines) * 128));
            }
        }
        // ---- conv + SiLU + L2 norm of k (tile rows 0..63) and q*scale (rows 64..127).  A task is 8 rows
        // of one part; its DK / 4 lanes take 4 channels each, so a row's norm reduces over them.
        {
            constexpr int LPP = DK / 4, PPW = 32 / LPP;  // lanes per part, parts per warp
            const int l = lane % LPP;
            char* kqb = reinterpret_cast<char*>(sm.kq);
            for (int task = warp * PPW + lane / LPP; task < 2 * (C / 8); task += 8 * PPW) {
                const int part = task & 1, r0 = 8 * (task >> 1);
                const int gc0 = part == 0 ? ck0 : cq0;
                float y[8][4];
                conv8x4(xs + part * DK + 4 * l, S::LDQK, sm.wq + (part * DK + 4 * l) * 4,
                        cbias ? cbias + gc0 + 4 * l : nullptr, r0, n, y);
#pragma unroll
                for (int o = 0; o < 8; ++o) {
                    float ss = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) ss = fmaf(y[o][u], y[o][u], ss);
#pragma unroll
                    for (int m = LPP / 2; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                    const float sc = r0 + o < n ? rsqrtf(ss + d.eps) * (part ? d.scale : 1.f) : 0.f;
                    *reinterpret_cast<uint2*>(kqb + tc::sw128_off(part * C + r0 + o, 4 * l, 2 * C)) =
                        make_uint2(tc::pack_f16(y[o][0] * sc, y[o][1] * sc), tc::pack_f16(y[o][2] * sc, y[o][3] * sc));
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
            const int cv0 = 2 * d.HK * DK + h * DV;  // first v channel of this head
            // ---- V rows (conv + SiLU) into the V tile: a task is 8 rows of DV / 4 lanes; warp 0 also
            // scans the gates
            {
                constexpr int LPV = DV / 4, VPW = 32 / LPV;
                const int l = lane % LPV;
                char* vrb = reinterpret_cast<char*>(sm.vr);
                for (int task = warp * VPW + lane / LPV; task < C / 8; task += 8 * VPW) {
                    const int r0 = 8 * task;
                    float y[8][4];
                    conv8x4(sm.xv + 4 * l, S::LDV, sm.wv + 16 * l, cbias ? cbias + cv0 + 4 * l : nullptr, r0, n, y);
#pragma unroll
                    for (int o = 0; o < 8; ++o) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) amax = fmaxf(amax, fabsf(y[o][u]));
                        *reinterpret_cast<uint2*>(vrb + tc::sw128_off(r0 + o, 4 * l, C)) =
                            make_uint2(tc::pack_f16(y[o][0], y[o][1]), tc::pack_f16(y[o][2], y[o][3]));
                    }
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
            if (j == 0) {
                ok = wait_mma();  // D1, and the barrier that publishes the gates
            } else {
                __syncthreads();
            }
            if (!ok) break;
            if (j + 1 < G) {  // the next value head's rows, taps and gates, while this one computes
                stage_v(q, h + 1);
                load_gates(q, h + 1);
            }
            // ---- from D1: A's diagonal 16x16 blocks (fp32) and its strictly block-lower part L (fp16 tile
            // 1) from the k.k rows (sub-partitions 0-1), the masked decayed q.k tile straight to global
            // memory from the q.k rows (2-3); the warps of a sub-partition take one group of 32 columns
            // each.  The exponents are formed without branches (a masked entry gets -inf, whose
            // exponential is 0); a block wholly above the diagonal only gets zeros.
            {
                char* AQg = reinterpret_cast<char*>(p.AQ + ch_h * (C * C));
                char* Lt = tile_b(1);
                const int r = (sp & 1) * 32 + lane;
                const bool qrow = sp >= 2;
                float v[32];
                const bool live0 = 32 * cg <= (sp & 1) * 32 + 31, live1 = 32 * cg + 16 <= (sp & 1) * 32 + 31;
                if (live0) tc::tmem_ld16(tD1 + lane_base + 32 * cg, *reinterpret_cast<float(*)[16]>(v));
                if (live1) tc::tmem_ld16(tD1 + lane_base + 32 * cg + 16, *reinterpret_cast<float(*)[16]>(v + 16));
                tc::tmem_ld_wait();
                const float gr = sm.gam2[r];
                const float br = qrow ? 1.f : sm.beta[r];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int c0 = 32 * cg + 16 * hh;
                    const bool live = hh == 0 ? live0 : live1;  // warp-uniform
                    float e[16];
                    if (live) {
                        const int lim = r < n ? r - c0 + (qrow ? 1 : 0) : 0;
#pragma unroll
                        for (int qq = 0; qq < 16; qq += 4) {
                            const float4 gs = *reinterpret_cast<const float4*>(&sm.gam2[c0 + qq]);
                            const float gq[4] = {gs.x, gs.y, gs.z, gs.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                e[qq + u] = qq + u < lim ? gr - gq[u] : __int_as_float(0xff800000u);  // -inf
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) e[i] = tc::ex2_approx(e[i]) * v[16 * hh + i] * br;
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) e[i] = 0.f;
                    }
                    if (!qrow) {
                        if (c0 == 16 * (r >> 4)) {  // the diagonal block: fp32, and zeros in L
#pragma unroll
                            for (int qq = 0; qq < 16; qq += 4)
                                *reinterpret_cast<float4*>(&inv.dg[r >> 4][r & 15][qq]) =
                                    make_float4(e[qq], e[qq + 1], e[qq + 2], e[qq + 3]);
#pragma unroll
                            for (int i = 0; i < 16; ++i) e[i] = 0.f;
                        }
                        store_h8(Lt, tc::sw128_off(r, c0, C), e);
                        store_h8(Lt, tc::sw128_off(r, c0 + 8, C), e + 8);
                    } else {
                        store_h8(AQg, tc::sw128_off(r, c0, C), e);
                        store_h8(AQg, tc::sw128_off(r, c0 + 8, C), e + 8);
                    }
                }
            }
            __syncthreads();
            if (j + 1 < G) commit_gates(n, h + 1);  // the scan of this head's gates is done
            // ---- D = the inverses of A's diagonal 16x16 blocks, by forward substitution in fp32 (warps
            // 0-1: lane (block, column c), t_r = [r == c] - sum_{s<r} A_rs t_s), into fp16 tile 0, whose
            // other blocks warps 2-7 clear; warps 4-5 also write the state pass's gate vectors
            if (warp < 2) {
                const int bk = 2 * warp + (lane >> 4), c = lane & 15;
                float t[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const float* arow = inv.dg[bk][r];
                    float acc[2] = {r == c ? 1.f : 0.f, 0.f};
#pragma unroll
                    for (int s = 0; s + 1 < r; ++s) acc[s & 1] = fmaf(-arow[s], t[s], acc[s & 1]);
                    const float b2 = acc[0] + acc[1];
                    t[r] = r > 0 ? fmaf(-arow[r - 1], t[r - 1], b2) : b2;
                }
                char* Dt = tile_b(0);
#pragma unroll
                for (int r = 0; r < 16; ++r)
                    *reinterpret_cast<__half*>(Dt + tc::sw128_off(16 * bk + r, 16 * bk + c, C)) = __float2half_rn(t[r]);
            } else {
                // the chunks of tile 0 outside the diagonal blocks: in row r, every 16-byte chunk but the
                // two that hold columns 16 (r / 16) .. 16 (r / 16) + 15
                char* Dt = tile_b(0);
                for (int e = tid - 64; e < C * 6; e += NT - 64) {
                    const int r = e / 6, k = e % 6;
                    const int c8 = k < 2 * (r >> 4) ? k : k + 2;
                    *reinterpret_cast<uint4*>(Dt + tc::sw128_off(r, 8 * c8, C)) = make_uint4(0u, 0u, 0u, 0u);
                }
                if (warp >= 4 && warp < 6) {  // the state pass's gate vectors: e^gamma, f, gamma, e^{gamma_n}
                    const int r = tid - 128;
                    const float gr = sm.gam[r], gn = sm.gam[n - 1];
                    float* gv = reinterpret_cast<float*>(p.GV + ch_h * C);
                    gv[r] = __expf(gr);
                    gv[C + r] = r < n ? __expf(gn - gr) : 0.f;
                    gv[2 * C + r] = gr;
                    gv[3 * C + r] = __expf(gn);
                }
            }
            tc::fence_smem_to_async();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            // ---- T = (I + E)^{-1} D = (I + E^2)(I - E) D with E = D L, in three rounds of fp16 products
            // (E; then E^2 and (I - E) D together; then T), each result rounded once
            constexpr uint32_t i64 = tc::idesc_f16(64, 64) | tc::kTransposeB;
            // a 64 x 64 x 64 product of tile `a` (K-major) and tile `b` (read MN-major) into `acc` (thread 0)
            auto issue = [&](uint32_t acc, int a, int b) {
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    tc::mma_f16(acc, tc::desc_sw128_k(tile_s(a), C, s), tc::desc_sw128_mn(tile_s(b), C, s), i64, s > 0);
            };
            auto publish = [&]() {  // the tiles written above are complete and visible to the tensor core
                tc::fence_smem_to_async();
                tc::fence_before_sync();
                __syncthreads();
                tc::fence_after_sync();
            };
            if (tid == 0) {  // E = D L
                issue(tX1, 0, 1);
                tc::mma_commit(bar);
            }
            if (!(ok = wait_mma())) break;
            read64(tX1, [&](int m, int c0, const float* v) {  // E -> tile 2, I - E -> tile 3
                float ne[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) ne[i] = (c0 + i == m ? 1.f : 0.f) - v[i];
                store_h8(tile_b(2), tc::sw128_off(m, c0, C), v);
                store_h8(tile_b(2), tc::sw128_off(m, c0 + 8, C), v + 8);
                store_h8(tile_b(3), tc::sw128_off(m, c0, C), ne);
                store_h8(tile_b(3), tc::sw128_off(m, c0 + 8, C), ne + 8);
            });
            publish();
            if (tid == 0) {  // E^2 = E E and Q = (I - E) D
                issue(tX2, 2, 2);
                issue(tX1, 3, 0);
                tc::mma_commit(bar);
            }
            if (!(ok = wait_mma())) break;
            read64(tX2, [&](int m, int c0, const float* v) {  // I + E^2 -> tile 1 (L is no longer needed)
                float pe[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pe[i] = (c0 + i == m ? 1.f : 0.f) + v[i];
                store_h8(tile_b(1), tc::sw128_off(m, c0, C), pe);
                store_h8(tile_b(1), tc::sw128_off(m, c0 + 8, C), pe + 8);
            });
            read64(tX1, [&](int m, int c0, const float* v) {  // Q -> tile 2 (E is no longer needed)
                store_h8(tile_b(2), tc::sw128_off(m, c0, C), v);
                store_h8(tile_b(2), tc::sw128_off(m, c0 + 8, C), v + 8);
            });
            publish();
            if (tid == 0) {  // T = (I + E^2) Q
                issue(tX2, 1, 2);
                tc::mma_commit(bar);
            }
            if (!(ok = wait_mma())) break;
            read64(tX2, [&](int m, int c0, const float* v) {  // T diag(beta) -> tile 0, T diag(beta e^gamma) -> 3
                float tb[16], te[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    tb[i] = v[i] * sm.beta[c0 + i];
                    te[i] = v[i] * sm.bge[c0 + i];
                    amax = fmaxf(amax, fmaxf(fabsf(tb[i]), fabsf(te[i])));
                }
                store_h8(tile_b(0), tc::sw128_off(m, c0, C), tb);
                store_h8(tile_b(0), tc::sw128_off(m, c0 + 8, C), tb + 8);
                store_h8(tile_b(3), tc::sw128_off(m, c0, C), te);
                store_h8(tile_b(3), tc::sw128_off(m, c0 + 8, C), te + 8);
            });
            publish();
            if (tid == 0) {  // W^T = K^T (T diag(beta e^gamma))^T (M = DK, K read MN-major from the [K ; Q]
                             // tile), U^T = V^T (T diag(beta))^T (M = DV, V read MN-major)
                const uint32_t bkq = tc::smem_u32(sm.kq), bvr = tc::smem_u32(sm.vr);
                constexpr uint32_t iw = tc::idesc_f16(DK, 64) | tc::kTransposeA;
                constexpr uint32_t iu = tc::idesc_f16(DV, 64) | tc::kTransposeA;
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    tc::mma_f16(tW, tc::desc_sw128_mn(bkq, 2 * C, s), tc::desc_sw128_k(tile_s(3), C, s), iw, s > 0);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    tc::mma_f16(tU, tc::desc_sw128_mn(bvr, C, s), tc::desc_sw128_k(tile_s(0), C, s), iu, s > 0);
                tc::mma_commit(bar);
            }
            if (!(ok = wait_mma())) break;
            if (j + 1 == G && sm.prefetch_item >= 0) {
                // the next item's rows (into the staging space, which the inverse's tiles have just left)
                // and its first value head's, while this head's W and U leave
                const Pos qn = pos_of(sm.prefetch_item);
                stage_qk(qn);
                stage_v(qn, qn.hk * G);
                load_gates(qn, qn.hk * G);
            }
            {  // W^T and U^T -> their tiles (fp16, swizzled, straight to global memory).  A row per lane
               // (M = 64: lanes 0-15 of each sub-partition); the warps of a sub-partition take one group of
               // 32 columns each
                char* Wg = reinterpret_cast<char*>(p.W + ch_h * (C * DK));
                char* Ug = reinterpret_cast<char*>(p.U + ch_h * (DV * C));
                float wv_[32], uv[32];
                tc::tmem_ld16(tW + lane_base + 32 * cg, *reinterpret_cast<float(*)[16]>(wv_));
                tc::tmem_ld16(tW + lane_base + 32 * cg + 16, *reinterpret_cast<float(*)[16]>(wv_ + 16));
                tc::tmem_ld16(tU + lane_base + 32 * cg, *reinterpret_cast<float(*)[16]>(uv));
                tc::tmem_ld16(tU + lane_base + 32 * cg + 16, *reinterpret_cast<float(*)[16]>(uv + 16));
                tc::tmem_ld_wait();
                if (DK == 128 || lane < 16) {
                    const int ir = DK == 128 ? sp * 32 + lane : sp * 16 + lane;
#pragma unroll
                    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(wv_[i]));
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) store_h8(Wg, tc::sw128_off(ir, 32 * cg + 8 * c8, DK), wv_ + 8 * c8);
                }
                if (DV == 128 || lane < 16) {
                    const int jr = DV == 128 ? sp * 32 + lane : sp * 16 + lane;
#pragma unroll
                    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(uv[i]));
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) store_h8(Ug, tc::sw128_off(jr, 32 * cg + 8 * c8, DV), uv + 8 * c8);
                }
            }
            if (j + 1 < G) tc::cp_async_wait_all();  // the next value head's rows
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
    report_f16_range(p.hdr, amax);
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
    const long long items = seg_max_piece(p.max_chunks, p.nseg) * p.d.HK;
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
