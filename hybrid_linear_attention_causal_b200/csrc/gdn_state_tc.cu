// Serial inter-chunk state pass of the chunked GDN prefill on tcgen05 tensor
// cores (sm_100a), with the chunk outputs.
//
// One CTA per (sequence, value head), looping over the sequence's chunks.  The
// products are formed transposed, with the value dimension (dv) as the MMA's
// M, so that every accumulator row belongs to one thread.  Per chunk, from the
// tiles the per-chunk step wrote ([K ; Q], W^T, U^T, Aqk and the gate vectors):
//
//   X^T     = S^T W^T                       M=dv N=64 K=dk   (on the chain)
//   Oi^T    = S^T Q^T                       M=dv N=64 K=dk   (off the chain)
//   V'^T    = U^T - X^T,  Vs'^T = V'^T diag(f),  f_s = e^{gamma_n - gamma_s}
//   Snew^T  = Vs'^T K                       M=dv N=dk K=64   (K read MN-major; on the chain)
//   S^T    <- e^{gamma_n} S^T + Snew^T      CUDA cores, fp32 in registers
//   Oq^T    = V'^T Aqk^T                    M=dv N=64 K=64   (off the chain)
//   o_r     = e^{gamma_r} Oi_r + Oq_r
//
// (the chunked WY/UT form of the gated delta rule; q carries the output scale).
// The chain from one chunk's state to the next is X, V', the state product and
// the update, and every step of it is cut in two so the next one starts on the
// first half:
//   - the state update writes the fp16 copy of S^T (the A operand of X and Oi,
//     in tensor memory) in two column halves, each released on its own
//     barrier once every compute warp has written its part of it, so the next
//     chunk's X issues its first k-steps while the second half is updated;
//   - V' is formed in two halves of the chunk's rows the same way, so the
//     state product issues its first k-steps while the second half is formed;
//   - the output products run on the tensor core while the CUDA cores form V'
//     and update the state, and four output warps (one per TMEM
//     sub-partition) read, scale, stage and store each chunk's outputs once
//     its products complete, handing the accumulators back to the next output
//     products on a barrier, so no output work sits on the chain.
// A ninth warp only issues MMAs, from descriptors formed once per buffer; a
// tenth issues every bulk copy, refilling each double-buffered tile as soon as
// its last reader releases it and prefetching tiles into L2 a few chunks ahead.
// The two compute warps of a TMEM sub-partition share its 32 accumulator rows
// and take one quarter of the columns each in either half, the first half
// first.

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NCW = 8;                  // compute warps 0-7
constexpr int ISSUER = NCW * 32;        // lane 0 of the ninth warp
constexpr int OW0 = NCW + 2;            // output warps OW0 .. OW0 + NOW - 1
constexpr int NOW = 4;
constexpr int NT = (OW0 + NOW) * 32;
constexpr int kCwBarrier = 1;           // named barrier of the compute warps
constexpr int kOwBarrier = 2;           // named barrier of the output warps
constexpr int kPrefetchAhead = 4;       // chunks between a tile's L2 prefetch and its use

// bf16 outputs are staged in shared memory and leave as 16-byte vectors; fp32 outputs (whose
// staging tiles would not fit) are stored by each thread
template <typename T>
constexpr bool kStageOut = sizeof(T) == 2;

template <typename T, int DK, int DV>
struct StateSmem {
    // fp16 operand tiles in the 128-byte swizzled layout (1024-byte aligned), double-buffered and
    // copied two chunks ahead
    uint16_t kq[2][2 * C * DK];  // [K ; Q]: K rows (MN-major B of Snew), Q rows (B of Oi)
    uint16_t w[2][C * DK];       // W^T (B of X, read MN-major)
    uint16_t ut[2][DV * C];      // U^T
    uint16_t aq[2][C * C];       // Aqk (B of Oq)
    uint16_t vt[DV * C];         // V'^T: A of Oq
    uint16_t vs[DV * C];         // Vs'^T: A of Snew
    T ostage[kStageOut<T> ? 2 : 1][kStageOut<T> ? C * DV : 1];  // a chunk's outputs O [C][DV]
    alignas(16) float gv[2][4][C];  // per row: e^{gamma_r}, f_r, gamma_r, e^{gamma_n} (a bulk-copy target)
    alignas(16) float eg[2][C];     // e^{gamma_r} of a chunk, the output warps' copy
    unsigned long long full_kq[2], full_w[2], full_u[2], full_aq[2];
    unsigned long long free_kq[2], free_w[2], free_u[2], free_aq[2];
    unsigned long long bar_x, bar_s, bar_o[2], bar_vp[2], bar_sa[2], out_free[2];
    uint32_t tmem_base;
};

template <typename T, int DK, int DV>
constexpr size_t state_smem_bytes() {
    return sizeof(StateSmem<T, DK, DV>) + 1024;  // + room to align the tiles on 1024 bytes
}
static_assert(state_smem_bytes<__nv_bfloat16, 128, 128>() <= 227 * 1024, "state pass shared memory");
using StateSmemF32 = StateSmem<float, 64, 64>;
static_assert(offsetof(StateSmemF32, gv) % 16 == 0 && offsetof(StateSmemF32, eg) % 16 == 0,
              "bulk-copy and vector targets stay 16-byte aligned whatever the output type");
static_assert(state_smem_bytes<float, 128, 128>() <= 227 * 1024, "state pass shared memory");

// barrier among `nthreads` threads on named barrier `id`; true when `pred` holds in all of them
__device__ __forceinline__ bool group_and(bool pred, int id, int nthreads) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool cw_and(bool pred) { return group_and(pred, kCwBarrier, NCW * 32); }
__device__ __forceinline__ bool ow_and(bool pred) { return group_and(pred, kOwBarrier, NOW * 32); }

// fp16 copy of 16 consecutive values of S^T row j (this thread's lane) into 8 columns of the
// tensor-memory A operand: two fp16 per column, the even column of S^T in the low half
__device__ __forceinline__ void put_sa16(uint32_t taddr, const float* v) {
    uint32_t wv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) wv[i] = tc::pack_f16(v[2 * i], v[2 * i + 1]);
    tc::tmem_st8(taddr, wv);
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, 1) state_tc_kernel(ExtendArgs p, int seg) {
    using Sm = StateSmem<T, DK, DV>;
    if (batch_rejected(p)) return;
    const LayerDims& d = p.d;
    const int HV = d.HV;
    // the ranks holding chunks of this segment's piece of the chunk list (all heads of the longer
    // sequence first); each CTA takes its sequence's chunks inside the piece
    const int rk = p.hdr[kHdrSegRank + seg] + (int)(blockIdx.x / HV);
    if (rk >= p.N) return;
    const int h = blockIdx.x % HV, hk = h / d.G, nseq = p.seq_order[rk];
    const int lo = p.hdr[kHdrSegOff + seg], hi = lo + p.hdr[kHdrSegCnt + seg];
    const int ro = p.rank_off[rk];
    const int a = max(lo, ro), b = min(hi, p.rank_off[rk + 1]);
    if (a >= b) return;
    const int c_first = p.seq_chunk0[nseq];
    const int c_begin = c_first + (a - ro), c_end = c_begin + (b - a);
    const int slot = p.slots[nseq];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    T* out = reinterpret_cast<T*>(p.out);
    if (slot < 0 || slot >= p.P) {
        if (slot >= p.P && tid == 0 && h == 0 && a == ro) raise_error(p.hdr, GDN_DEVERR_SLOT_RANGE);
        const int r0 = p.cu[nseq] + (c_begin - c_first) * C, r1 = min(p.cu[nseq + 1], r0 + (c_end - c_begin) * C);
        for (int e = tid; e < (r1 - r0) * DV; e += NT)
            out[((size_t)(r0 + e / DV) * HV + h) * DV + e % DV] = from_f<T>(0.f);
        return;
    }
    extern __shared__ unsigned char smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    constexpr uint32_t KQ_BYTES = 2 * C * DK * 2, W_BYTES = C * DK * 2, U_BYTES = DV * C * 2, AQ_BYTES = C * C * 2,
                       GV_BYTES = C * 16;
    auto bar = [](unsigned long long& m) { return tc::smem_u32(&m); };
    auto src_kq = [&](int id) { return p.KQ + ((size_t)id * d.HK + hk) * (2 * C * DK); };
    auto src_w = [&](int id) { return p.W + ((size_t)id * HV + h) * (C * DK); };
    auto src_u = [&](int id) { return p.U + ((size_t)id * HV + h) * (DV * C); };
    auto src_gv = [&](int id) { return p.GV + ((size_t)id * HV + h) * C; };
    auto src_aq = [&](int id) { return p.AQ + ((size_t)id * HV + h) * (C * C); };
    auto fetch = [&](int id) {  // every tile of chunk id into its buffers, on their "full" barriers
        const int bb = (id - c_begin) & 1;
        tc::mbar_expect_tx(bar(sm.full_kq[bb]), KQ_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.kq[bb]), src_kq(id), KQ_BYTES, bar(sm.full_kq[bb]));
        tc::mbar_expect_tx(bar(sm.full_w[bb]), W_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.w[bb]), src_w(id), W_BYTES, bar(sm.full_w[bb]));
        tc::mbar_expect_tx(bar(sm.full_u[bb]), U_BYTES + GV_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.ut[bb]), src_u(id), U_BYTES, bar(sm.full_u[bb]));
        tc::bulk_g2s(tc::smem_u32(sm.gv[bb]), src_gv(id), GV_BYTES, bar(sm.full_u[bb]));
        tc::mbar_expect_tx(bar(sm.full_aq[bb]), AQ_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.aq[bb]), src_aq(id), AQ_BYTES, bar(sm.full_aq[bb]));
    };
    auto prefetch = [&](int id) {  // chunk id's tiles into L2
        tc::bulk_prefetch_l2(src_kq(id), KQ_BYTES);
        tc::bulk_prefetch_l2(src_w(id), W_BYTES);
        tc::bulk_prefetch_l2(src_u(id), U_BYTES);
        tc::bulk_prefetch_l2(src_gv(id), GV_BYTES);
        tc::bulk_prefetch_l2(src_aq(id), AQ_BYTES);
    };
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 512);
    if (tid == ISSUER) {
        for (int bb = 0; bb < 2; ++bb) {
            tc::mbar_init(bar(sm.full_kq[bb]), 1);
            tc::mbar_init(bar(sm.full_w[bb]), 1);
            tc::mbar_init(bar(sm.full_u[bb]), 1);
            tc::mbar_init(bar(sm.full_aq[bb]), 1);
            tc::mbar_init(bar(sm.free_kq[bb]), 1);
            tc::mbar_init(bar(sm.free_w[bb]), 1);
            tc::mbar_init(bar(sm.free_u[bb]), NCW + NOW);  // V' formed + the output warps' copy of e^gamma
            tc::mbar_init(bar(sm.free_aq[bb]), 1);          // the output product's commit
            tc::mbar_init(bar(sm.bar_vp[bb]), NCW);
            tc::mbar_init(bar(sm.bar_sa[bb]), NCW);
            tc::mbar_init(bar(sm.out_free[bb]), NOW);
            tc::mbar_init(bar(sm.bar_o[bb]), 1);
        }
        tc::mbar_init(bar(sm.bar_x), 1);
        tc::mbar_init(bar(sm.bar_s), 1);
        tc::fence_mbar_init();
        for (int id = c_begin; id < c_end && id < c_begin + 2; ++id) fetch(id);
        for (int id = c_begin + 2; id < c_end && id < c_begin + kPrefetchAhead; ++id) prefetch(id);
    }

    // compute warps: thread (sp, hw, lane) owns row j of S^T and, in each half of its columns, the
    // quarter hw: columns q * DK/2 + hw * DK/4 .. + DK/4 for q = 0, 1 (register s[q * DK/4 + i]).
    // Every compute warp finishes its part of the first half before it starts on the second, so
    // each half's barrier completes half-way through the phase and the products waiting on it start
    // while the second half is formed.  (V'^T's chunk rows are shared out the same way.)
    const int sp = warp & 3, hw = (warp >> 2) & 1;
    constexpr int QW = DK / 4;
    auto col_of = [&](int i) { return (i / QW) * (DK / 2) + hw * QW + i % QW; };
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    const bool rowv = warp < NCW && (DV == 128 || lane < 16);
    const int j = DV == 128 ? sp * 32 + lane : sp * 16 + lane;
    // a range after the sequence's first chunk continues from the state the previous piece left
    const bool init = a > ro || (p.has_init ? p.has_init[nseq] != 0 : true);
    float* Sg = p.ssm_state + ((size_t)slot * HV + h) * DK * DV;
    float s[DK / 2];
#pragma unroll
    for (int i = 0; i < DK / 2; ++i) s[i] = (init && rowv) ? Sg[(size_t)col_of(i) * DV + j] : 0.f;
    // a state checkpoint of this sequence: the state entering the chunk that holds its boundary is
    // stored when that chunk comes up (a boundary at the very end belongs to the last chunk); the
    // rows of that chunk before the boundary are added afterwards, off the chain
    int ck_chunk = -1;
    float* ck_dst = nullptr;
    {
        int row = 0;
        const int t = ckpt_offset(p, nseq, &row);
        const int len = p.cu[nseq + 1] - p.cu[nseq];
        if (t >= 0 && len > 0) {
            ck_chunk = c_first + min(t / C, (len + C - 1) / C - 1);
            ck_dst = p.ck_states + ((size_t)row * HV + h) * DK * DV;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    // tensor memory: the fp16 copy of S^T (DK / 2 columns) at tm, X^T at tm + 64, Oi^T and Oq^T
    // double-buffered at tm + 128 + 64 b and tm + 256 + 64 b, Snew^T (DK columns) at tm + 384
    const uint32_t tA = tm, tX = tm + 64, tSn = tm + 384;
    auto tOi = [&](int bb) { return tm + 128 + 64 * bb; };
    auto tOq = [&](int bb) { return tm + 256 + 64 * bb; };
    static_assert(DK <= 128 && DV <= 128, "tensor-memory layout");
    // S^T column c of row j sits in tensor-memory column c / 2 of lane j's row of the A operand
    auto tA_at = [&](int i) { return tA + lane_base + (uint32_t)(col_of(i) / 2); };
    if (warp < NCW) {  // the starting state's fp16 copy, released as both halves of the first chunk's X
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
            for (int cc = 0; cc < QW; cc += 16) put_sa16(tA_at(q * QW + cc), &s[q * QW + cc]);
            tc::tmem_st_wait();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(sm.bar_sa[q]));
        }
    }

    bool ok = true;
    if (warp == NCW + 1) {
        // ---- the copier: each buffer is refilled for the chunk two ahead as soon as its readers have
        // released it (W after X, U^T and the gate vectors once V' has been formed, [K ; Q] after the
        // state product, Aqk once its product is done).  The next release of a buffer
        // needs the copy issued here, so none of these barriers can complete twice before this lane
        // has seen the first.
        if (lane == 0) {
            for (int id = c_begin; id + 2 < c_end && ok; ++id) {
                const int it = id - c_begin, bb = it & 1;
                const uint32_t pb = (uint32_t)(it >> 1) & 1u;
                if (id + kPrefetchAhead < c_end) prefetch(id + kPrefetchAhead);
                const int nx = id + 2, nb = bb;  // the chunk two ahead lands in this chunk's buffers
                ok = tc::mbar_wait(bar(sm.free_w[bb]), pb);
                if (ok) {
                    tc::mbar_expect_tx(bar(sm.full_w[nb]), W_BYTES);
                    tc::bulk_g2s(tc::smem_u32(sm.w[nb]), src_w(nx), W_BYTES, bar(sm.full_w[nb]));
                }
                if (ok) ok = tc::mbar_wait(bar(sm.free_u[bb]), pb);
                if (ok) {
                    tc::mbar_expect_tx(bar(sm.full_u[nb]), U_BYTES + GV_BYTES);
                    tc::bulk_g2s(tc::smem_u32(sm.ut[nb]), src_u(nx), U_BYTES, bar(sm.full_u[nb]));
                    tc::bulk_g2s(tc::smem_u32(sm.gv[nb]), src_gv(nx), GV_BYTES, bar(sm.full_u[nb]));
                }
                if (ok) ok = tc::mbar_wait(bar(sm.free_kq[bb]), pb);
                if (ok) {
                    tc::mbar_expect_tx(bar(sm.full_kq[nb]), KQ_BYTES);
                    tc::bulk_g2s(tc::smem_u32(sm.kq[nb]), src_kq(nx), KQ_BYTES, bar(sm.full_kq[nb]));
                }
                if (ok) ok = tc::mbar_wait(bar(sm.free_aq[bb]), pb);
                if (ok) {
                    tc::mbar_expect_tx(bar(sm.full_aq[nb]), AQ_BYTES);
                    tc::bulk_g2s(tc::smem_u32(sm.aq[nb]), src_aq(nx), AQ_BYTES, bar(sm.full_aq[nb]));
                }
            }
        }
    } else if (warp == NCW) {
        // ---- the MMA issuer, from descriptors formed once per buffer and advanced by constant offsets
        if (lane == 0) {
            // buffer 1's descriptors are buffer 0's advanced by the buffer stride
            const uint64_t dW0 = tc::desc_sw128_mn(tc::smem_u32(sm.w[0]), DK, 0);  // W^T, read MN-major
            const uint64_t dQ0 = tc::desc_sw128_k(tc::smem_u32(sm.kq[0]) + C * 128, 2 * C, 0);  // Q: rows C .. 2C-1
            const uint64_t dK0 = tc::desc_sw128_mn(tc::smem_u32(sm.kq[0]), 2 * C, 0);
            const uint64_t dA0 = tc::desc_sw128_k(tc::smem_u32(sm.aq[0]), C, 0);
            constexpr uint32_t kW1 = C * DK * 2, kKQ1 = 2 * C * DK * 2, kA1 = C * C * 2;
            const uint64_t dVs = tc::desc_sw128_k(tc::smem_u32(sm.vs), DV, 0);
            const uint64_t dVt = tc::desc_sw128_k(tc::smem_u32(sm.vt), DV, 0);
            constexpr uint32_t ix = tc::idesc_f16(DV, 64), ixw = ix | tc::kTransposeB,
                               is = tc::idesc_f16(DV, DK) | tc::kTransposeB;
            for (int id = c_begin; id < c_end && ok; ++id) {
                const int it = id - c_begin, bb = it & 1;
                const uint32_t ph = (uint32_t)it & 1u, pb = (uint32_t)(it >> 1) & 1u;
                const uint64_t dWb = tc::desc_add(dW0, bb * kW1), dQb = tc::desc_add(dQ0, bb * kKQ1),
                               dKb = tc::desc_add(dK0, bb * kKQ1), dAb = tc::desc_add(dA0, bb * kA1);
                ok = tc::mbar_wait(bar(sm.full_w[bb]), pb) && tc::mbar_wait(bar(sm.full_kq[bb]), pb);
                // X^T = S^T W^T, each half of S^T's columns as soon as the update has written it
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    if (ok) ok = tc::mbar_wait(bar(sm.bar_sa[hh]), ph);
                    tc::fence_after_sync();
                    if (ok)
#pragma unroll
                        for (int k = hh * (DK / 32); k < (hh + 1) * (DK / 32); ++k)
                            tc::mma_f16_ta(tX, tA + 8 * k, tc::desc_add(dWb, 2048u * k), ixw, k > 0);
                }
                if (!ok) break;
                tc::mma_commit(bar(sm.bar_x));
                tc::mma_commit(bar(sm.free_w[bb]));
                // Oi^T = S^T Q^T, once the outputs two chunks back have left its accumulator
                if (it >= 2) ok = tc::mbar_wait(bar(sm.out_free[bb]), (uint32_t)((it >> 1) - 1) & 1u);
                if (!ok) break;
#pragma unroll
                for (int k = 0; k < DK / 16; ++k)
                    tc::mma_f16_ta(tOi(bb), tA + 8 * k, tc::desc_add(dQb, tc::sw128_kstep(2 * C, k)), ix, k > 0);
                // Snew^T = Vs'^T K (K read MN-major) and Oq^T = V'^T Aqk^T, each half of the chunk's rows as
                // soon as it is formed: the state product's k-steps of a half first, then Oq's (off the
                // chain), so that Oq's first half fills the wait for V's second half and only its second
                // half sits between the state product and the next chunk's X
                ok = tc::mbar_wait(bar(sm.full_aq[bb]), pb);
#pragma unroll
                for (int hh = 0; hh < 2 && ok; ++hh) {
                    ok = tc::mbar_wait(bar(sm.bar_vp[hh]), ph);
                    tc::fence_after_sync();
                    if (!ok) break;
#pragma unroll
                    for (int k = 2 * hh; k < 2 * hh + 2; ++k)
                        tc::mma_f16(tSn, tc::desc_add(dVs, tc::sw128_kstep(DV, k)), tc::desc_add(dKb, 2048u * k), is,
                                    k > 0);
                    if (hh == 1) {
                        tc::mma_commit(bar(sm.bar_s));
                        tc::mma_commit(bar(sm.free_kq[bb]));
                    }
#pragma unroll
                    for (int k = 2 * hh; k < 2 * hh + 2; ++k)
                        tc::mma_f16(tOq(bb), tc::desc_add(dVt, tc::sw128_kstep(DV, k)),
                                    tc::desc_add(dAb, tc::sw128_kstep(C, k)), ix, k > 0);
                }
                if (!ok) break;
                tc::mma_commit(bar(sm.bar_o[bb]));
                tc::mma_commit(bar(sm.free_aq[bb]));
            }
        }
    } else if (warp < NCW) {
        // ---- the compute warps.  Every wait is bounded; a failed one skips the work that needed it,
        // and the compute warps agree on the outcome at one barrier per chunk, so they stop together.
        float amax = 0.f;  // largest magnitude this thread rounded to fp16 among V', f V' and S's copy
#pragma unroll
        for (int i = 0; i < DK / 2; ++i) amax = fmaxf(amax, fabsf(s[i]));  // the starting state's copy
        // row j's 16-byte chunk c of a swizzled DV x 64 tile (U^T, V'^T, Vs'^T)
        const uint32_t jrow = (uint32_t)j * 128, jx = (uint32_t)(j & 7);
        auto uoff = [&](int c) { return jrow + ((((uint32_t)c >> 3) ^ jx) << 4); };
        for (int id = c_begin; id < c_end; ++id) {
            const int it = id - c_begin, bb = it & 1;
            const uint32_t ph = (uint32_t)it & 1u, pb = (uint32_t)(it >> 1) & 1u;
            if (id == ck_chunk && rowv)  // the state entering the checkpoint's chunk: column j of S
#pragma unroll
                for (int i = 0; i < DK / 2; ++i) ck_dst[(size_t)col_of(i) * DV + j] = s[i];
            // V'^T row j = U^T row j - X^T row j and Vs'^T = V'^T diag(f), over this warp's quarter hw of
            // each half of the chunk's rows, the first half first
            bool okl = __all_sync(0xffffffffu, tc::mbar_wait(bar(sm.bar_x), ph) && tc::mbar_wait(bar(sm.full_u[bb]), pb));
            float egn = 0.f;
            if (okl) {
                tc::fence_after_sync();
                char* vtb = reinterpret_cast<char*>(sm.vt);
                char* vsb = reinterpret_cast<char*>(sm.vs);
                const char* utb = reinterpret_cast<const char*>(sm.ut[bb]);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
#pragma unroll
                    for (int cc = 0; cc < C / 4; cc += 8) {  // 8 fp16 values per 16-byte vector
                        const int c0 = q * (C / 2) + hw * (C / 4) + cc;
                        float xv[8], f[8];
                        tc::tmem_ld8(tX + lane_base + c0, xv);
#pragma unroll
                        for (int k4 = 0; k4 < 8; k4 += 4)
                            *reinterpret_cast<float4*>(f + k4) = *reinterpret_cast<const float4*>(&sm.gv[bb][1][c0 + k4]);
                        tc::tmem_ld_wait();
                        if (rowv) {
                            const uint32_t off = uoff(c0);
                            const uint4 u = *reinterpret_cast<const uint4*>(utb + off);
                            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
                            uint32_t vw[4], sw[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 uu = tc::unpack_f16(uw[e]);
                                const float v0 = uu.x - xv[2 * e], v1 = uu.y - xv[2 * e + 1];
                                amax = fmaxf(amax, fmaxf(fabsf(v0), fabsf(v1)));  // |f| <= 1: covers f V' too
                                vw[e] = tc::pack_f16(v0, v1);
                                sw[e] = tc::pack_f16(v0 * f[2 * e], v1 * f[2 * e + 1]);
                            }
                            *reinterpret_cast<uint4*>(vtb + off) = make_uint4(vw[0], vw[1], vw[2], vw[3]);
                            *reinterpret_cast<uint4*>(vsb + off) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
                        }
                    }
                    tc::fence_smem_to_async();
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(sm.bar_vp[q]));
                }
                egn = sm.gv[bb][3][0];  // e^{gamma_n}
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(sm.free_u[bb]));
            }
            // S^T <- e^{gamma_n} S^T + Snew^T, and its fp16 copy for the next chunk, the first half first
            if (okl) okl = __all_sync(0xffffffffu, tc::mbar_wait(bar(sm.bar_s), ph));
            if (okl) {
                tc::fence_after_sync();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
#pragma unroll
                    for (int cc = 0; cc < QW; cc += 16) {
                        const int i0 = q * QW + cc;
                        float v[16];
                        tc::tmem_ld16(tSn + lane_base + col_of(i0), v);
                        tc::tmem_ld_wait();
                        uint32_t wv[8];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            s[i0 + i] = fmaf(egn, s[i0 + i], v[i]);
                            amax = fmaxf(amax, fabsf(s[i0 + i]));
                        }
#pragma unroll
                        for (int i = 0; i < 8; ++i) wv[i] = tc::pack_f16(s[i0 + 2 * i], s[i0 + 2 * i + 1]);
                        tc::tmem_st8(tA_at(i0), wv);
                    }
                    tc::tmem_st_wait();
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(sm.bar_sa[q]));
                }
            }
            ok = cw_and(okl);
            if (!ok) break;
        }
        if (ok && rowv)  // final state: column j of S
#pragma unroll
            for (int i = 0; i < DK / 2; ++i) Sg[(size_t)col_of(i) * DV + j] = s[i];
        if (!rowv) amax = 0.f;  // lanes past a 64-row tile hold no row
        report_f16_range(p.hdr, amax);
    } else {
        // ---- the output warps: warp OW0 + w reads sub-partition (OW0 + w) % 4, a row j of Oi^T and
        // Oq^T with all of the chunk's 64 columns.  Per chunk: the chunk's e^{gamma_r} is copied while
        // its gate vector is in (then released to the copier); once the output products complete,
        // o = e^{gamma_r} Oi + Oq is staged (bf16) or stored (fp32) and the accumulators are handed
        // back; the staged rows then leave as 16-byte vectors.
        const int osp = warp & 3, ot = tid - OW0 * 32;
        const uint32_t olane = (uint32_t)(osp * 32) << 16;
        const bool orow = DV == 128 || lane < 16;
        const int oj = DV == 128 ? osp * 32 + lane : osp * 16 + lane;
        for (int id = c_begin; id < c_end && ok; ++id) {
            const int it = id - c_begin, bb = it & 1;
            const uint32_t pb = (uint32_t)(it >> 1) & 1u;
            const int4 ch = p.chunk_tab[id];
            const int t0 = ch.y, n = ch.z;
            bool okl = __all_sync(0xffffffffu, tc::mbar_wait(bar(sm.full_u[bb]), pb));
            if (okl) {
                if (ot < C) sm.eg[bb][ot] = sm.gv[bb][0][ot];
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(sm.free_u[bb]));
            }
            okl = ow_and(okl);  // the copy of e^gamma is complete
            if (okl) okl = __all_sync(0xffffffffu, tc::mbar_wait(bar(sm.bar_o[bb]), pb));
            if (okl) {
                tc::fence_after_sync();
#pragma unroll
                for (int c0 = 0; c0 < C; c0 += 16) {
                    float oi[16], oq[16], eg[16];
                    tc::tmem_ld16(tOi(bb) + olane + c0, oi);
                    tc::tmem_ld16(tOq(bb) + olane + c0, oq);
#pragma unroll
                    for (int q = 0; q < 16; q += 4)
                        *reinterpret_cast<float4*>(eg + q) = *reinterpret_cast<const float4*>(&sm.eg[bb][c0 + q]);
                    tc::tmem_ld_wait();
                    if (orow)
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float o = fmaf(eg[i], oi[i], oq[i]);
                            if constexpr (kStageOut<T>) sm.ostage[bb][(c0 + i) * DV + oj] = from_f<T>(o);
                            else if (c0 + i < n) out[((size_t)(t0 + c0 + i) * HV + h) * DV + oj] = from_f<T>(o);
                        }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(sm.out_free[bb]));
            }
            ok = ow_and(okl);  // the staged rows are complete
            if (ok) {
                if constexpr (kStageOut<T>) {
                    constexpr int VPR = DV * (int)sizeof(T) / 16;  // vectors per row
                    for (int e = ot; e < n * VPR; e += NOW * 32) {
                        const int r = e / VPR, v = e % VPR;
                        reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * HV + h) * DV)[v] =
                            reinterpret_cast<const uint4*>(sm.ostage[bb] + r * DV)[v];
                    }
                }
            }
        }
    }
    ok = __syncthreads_and(ok);  // the chain, the issuer, the copier, the output warps and the idle lanes agree
    if (!ok && tid == ISSUER) {
        raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
        // let copies and products already in flight finish before the CTA's shared and tensor
        // memory go away
        for (uint32_t par = 0; par < 2; ++par) {
            for (int bb = 0; bb < 2; ++bb) {
                tc::mbar_wait(bar(sm.full_kq[bb]), par, 100000000ull);
                tc::mbar_wait(bar(sm.full_w[bb]), par, 100000000ull);
                tc::mbar_wait(bar(sm.full_u[bb]), par, 100000000ull);
                tc::mbar_wait(bar(sm.full_aq[bb]), par, 100000000ull);
            }
            tc::mbar_wait(bar(sm.bar_o[0]), par, 100000000ull);
            tc::mbar_wait(bar(sm.bar_o[1]), par, 100000000ull);
        }
    }
    if (ok && tid == ISSUER) {  // the releases nobody waited for, so that none lands after the CTA is gone
        const int n = c_end - c_begin;
        for (int it = max(0, n - 2); it < n; ++it) {
            tc::mbar_wait(bar(sm.free_w[it & 1]), (uint32_t)(it >> 1) & 1u);
            tc::mbar_wait(bar(sm.free_kq[it & 1]), (uint32_t)(it >> 1) & 1u);
            tc::mbar_wait(bar(sm.free_aq[it & 1]), (uint32_t)(it >> 1) & 1u);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 512);
}

}  // namespace

template <typename T, int DK, int DV>
cudaError_t launch_state(const ExtendArgs& p, int seg, cudaStream_t s) {
    constexpr size_t shm = state_smem_bytes<T, DK, DV>();
    cudaError_t e =
        cudaFuncSetAttribute(state_tc_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    // a piece of P chunks touches at most P + 1 sequences
    const long long piece = seg_max_piece(p.max_chunks, p.nseg);
    const long long seqs = piece + 1 < p.N ? piece + 1 : p.N;
    state_tc_kernel<T, DK, DV><<<(unsigned)(seqs * p.d.HV), NT, shm, s>>>(p, seg);
    return cudaGetLastError();
}

#define GDN_STATE_INST(T)                                                        \
    template cudaError_t launch_state<T, 64, 64>(const ExtendArgs&, int, cudaStream_t);   \
    template cudaError_t launch_state<T, 64, 128>(const ExtendArgs&, int, cudaStream_t);  \
    template cudaError_t launch_state<T, 128, 64>(const ExtendArgs&, int, cudaStream_t);  \
    template cudaError_t launch_state<T, 128, 128>(const ExtendArgs&, int, cudaStream_t);
GDN_STATE_INST(float)
GDN_STATE_INST(__nv_bfloat16)

}  // namespace gdn
