// Serial inter-chunk state pass of the chunked GDN prefill on tcgen05 tensor
// cores (sm_100a), with the chunk outputs.
//
// One CTA per (sequence, value head), looping over the sequence's chunks.  The
// products are formed transposed, with the value dimension (dv) as the MMA's
// M, so that every accumulator row belongs to one thread; K~ is read MN-major
// (its rows s run along the product's K), every other operand K-major:
//
//   [X^T | O^T]  = S^T [W ; Qg]^T           M=dv N=128 K=dk   (X = W S, O = Qg S)
//   V'^T         = U^T - X^T                 CUDA cores, per thread row j
//   Snew^T       = V'^T K~                   M=dv N=dk  K=64  (K~ = diag(e^{gamma_n-gamma}) K)
//   S^T         <- e^{gamma_n} S^T + Snew^T  CUDA cores, fp32 in registers
//   O^T         += V'^T Aqk^T                M=dv N=64  K=64
//
// where Qg = diag(e^gamma) Q (q carries the output scale).  The chain from one
// chunk's state to the next runs through the first product, V', the state
// product and the update; everything else is kept off it:
//   - a ninth warp only issues the MMAs, so the eight compute warps never
//     wait behind an issue loop; it queues the output product right behind
//     the state product (the tensor core runs them in order) and never waits
//     for it;
//   - a tenth warp issues every bulk copy: each tile buffer has a "free"
//     barrier that the product reading it signals on completion (or the
//     compute warps, for U^T), and the copier refills the buffer as soon as
//     it completes, so no copy issue or wait sits on the chain;
//   - the fp32 state lives in registers (each thread holds one half of row j
//     of S^T), the state product goes to a fresh accumulator and the update
//     is one FMA per element, written straight into the fp16 copy of S^T that
//     the first product reads from tensor memory (so that product reads only
//     [W ; Qg] from shared memory);
//   - [X^T | O^T] is double-buffered in tensor memory: a chunk's outputs are
//     read and stored while the next chunk's first product runs;
//   - [W ; Qg] and K~ are double-buffered and copied two chunks ahead;
//   - the tiles [W ; Qg], K~ and Aqk (written by the intra-chunk kernel as
//     fp16 in the tensor core's layout) each have their own barrier and are
//     refetched as soon as the product that reads them completes;
//   - the intra-chunk kernel writes U^T in the layout of the V'^T operand
//     tile; it lands in a tile of its own, so the next chunk's copy starts
//     as soon as V' has been formed from it.
// The two compute warps of a TMEM sub-partition share its 32 accumulator rows
// and take one half of the columns each.

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

constexpr int C = kChunk;
constexpr int NCW = 8;                  // compute warps
constexpr int NCHAIN = (NCW + 1) * 32;  // + the issuing warp: the threads on the state chain
constexpr int ISSUER = NCW * 32;        // its lane 0
constexpr int COPIER = NCHAIN;          // lane 0 of a tenth warp, which issues every bulk copy
constexpr int NT = NCHAIN + 32;
constexpr int kChainBarrier = 1;        // named barrier of the chain threads

// barrier among the `n` threads of named barrier `id`; true when `pred` holds in all of them
__device__ __forceinline__ bool bar_and(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// bf16 outputs are staged in shared memory and leave as 16-byte vectors while
// the next state product runs; fp32 outputs (whose staging tile would not fit)
// are stored by each thread
template <typename T>
constexpr bool kStageOut = sizeof(T) == 2;

template <typename T, int DK, int DV>
struct StateTcSmem {
    // fp16 operand tiles (16-bit K-major layout); [W ; Qg] and K~ are double-buffered and copied
    // two chunks ahead
    uint16_t wq[2][2 * C * DK];  // [W ; Qg] tiles (bulk copy): 128 rows x DK
    uint16_t kt[2][C * DK];      // K~ tiles (bulk copy): C rows (s) x DK (i), the MN-major B of Snew^T
    uint16_t aq[C * C];       // Aqk tile (bulk copy): C rows (r) x C (s)
    uint16_t ut[DV * C];      // U^T tile (bulk copy): DV rows (j) x C (s)
    uint16_t vt[DV * C];      // V'^T = U^T - X^T, same layout: the A operand of the state and output products
    T ostage[kStageOut<T> ? C * DV : 1];  // a chunk's outputs O [C][DV] on their way out
    unsigned long long bar_x, bar_s, bar_o, bar_wq[2], bar_kt[2], bar_aq, bar_u;
    // the copier's signals that a tile buffer is free again: the product reading it has completed
    // (tensor-core commits), or V' has read U^T (one arrival per compute warp)
    unsigned long long free_wq[2], free_kt[2], free_aq, free_u;
    uint32_t tmem_base;
};


// fp16 copy of 32 consecutive values of S^T row j (this thread's lane) into 16 columns of the
// tensor-memory A operand: two fp16 per column, the even column of S^T in the low half
__device__ __forceinline__ void put_sa32(uint32_t taddr, const float* v) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = tc::pack_f16(v[2 * i], v[2 * i + 1]);
    tc::tmem_st16(taddr, w);
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(NT, 1) state_tc_kernel(ExtendArgs p, int seg) {
    if (batch_rejected(p)) return;
    const LayerDims& d = p.d;
    const int HV = d.HV;
    // the ranks holding chunks of this segment's piece of the chunk list (all heads of the longer
    // sequence first); each CTA takes its sequence's chunks inside the piece
    const int r = p.hdr[kHdrSegRank + seg] + (int)(blockIdx.x / HV);
    if (r >= p.N) return;
    const int h = blockIdx.x % HV, nseq = p.seq_order[r];
    const int lo = p.hdr[kHdrSegOff + seg], hi = lo + p.hdr[kHdrSegCnt + seg];
    const int ro = p.rank_off[r];
    const int a = max(lo, ro), b = min(hi, p.rank_off[r + 1]);
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
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StateTcSmem<T, DK, DV>& sm = *reinterpret_cast<StateTcSmem<T, DK, DV>*>(smem_raw);
    const uint32_t bar_x = tc::smem_u32(&sm.bar_x), bar_s = tc::smem_u32(&sm.bar_s),
                   bar_o = tc::smem_u32(&sm.bar_o), bar_aq = tc::smem_u32(&sm.bar_aq),
                   bar_u = tc::smem_u32(&sm.bar_u);
    constexpr uint32_t WQ_BYTES = 2 * C * DK * 2, AQ_BYTES = C * C * 2, KT_BYTES = DK * C * 2, U_BYTES = DV * C * 2;
    // buffer b = (id - c_begin) & 1 of the double-buffered tiles; its barrier completes once every
    // other chunk, so a chunk waits on parity ((id - c_begin) >> 1) & 1
    auto bar_wq = [&](int b) { return tc::smem_u32(&sm.bar_wq[b]); };
    auto bar_kt = [&](int b) { return tc::smem_u32(&sm.bar_kt[b]); };
    auto fetch_wq = [&](int id) {
        const int b = (id - c_begin) & 1;
        tc::mbar_expect_tx(bar_wq(b), WQ_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.wq[b]), p.WQ + ((size_t)id * HV + h) * (2 * C * DK), WQ_BYTES, bar_wq(b));
    };
    auto fetch_kt = [&](int id) {
        const int b = (id - c_begin) & 1;
        tc::mbar_expect_tx(bar_kt(b), KT_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.kt[b]), p.KT + ((size_t)id * HV + h) * (DK * C), KT_BYTES, bar_kt(b));
    };
    auto u_src = [&](int id) { return p.U + ((size_t)id * HV + h) * (DV * C); };
    auto fetch_u = [&](int id) {
        tc::mbar_expect_tx(bar_u, U_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.ut), u_src(id), U_BYTES, bar_u);
    };
    auto fetch_aq = [&](int id) {
        tc::mbar_expect_tx(bar_aq, AQ_BYTES);
        tc::bulk_g2s(tc::smem_u32(sm.aq), p.AQ + ((size_t)id * HV + h) * (C * C), AQ_BYTES, bar_aq);
    };
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, 512);
    if (tid == ISSUER) {
        tc::mbar_init(bar_x, 1);
        tc::mbar_init(bar_s, 1);
        tc::mbar_init(bar_o, 1);
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar_wq(b), 1);
            tc::mbar_init(bar_kt(b), 1);
        }
        tc::mbar_init(bar_aq, 1);
        tc::mbar_init(bar_u, 1);
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(tc::smem_u32(&sm.free_wq[b]), 1);
            tc::mbar_init(tc::smem_u32(&sm.free_kt[b]), 1);
        }
        tc::mbar_init(tc::smem_u32(&sm.free_aq), 1);
        tc::mbar_init(tc::smem_u32(&sm.free_u), NCW);
        tc::fence_mbar_init();
        for (int id = c_begin; id < c_end && id < c_begin + 2; ++id) {
            fetch_wq(id);
            fetch_kt(id);
        }
        fetch_aq(c_begin);
        fetch_u(c_begin);
    }

    // compute warps: thread (sp, half, lane) owns row j of S^T, columns half * DK/2 .. + DK/2
    const int sp = warp & 3, half = (warp >> 2) & 1;
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    const bool rowv = warp < NCW && (DV == 128 || lane < 16);
    const int j = DV == 128 ? sp * 32 + lane : sp * 16 + lane;
    // a range after the sequence's first chunk continues from the state the previous piece left
    const bool init = a > ro || (p.has_init ? p.has_init[nseq] != 0 : true);
    float* Sg = p.ssm_state + ((size_t)slot * HV + h) * DK * DV;
    float s[DK / 2];
#pragma unroll
    for (int i = 0; i < DK / 2; ++i) s[i] = (init && rowv) ? Sg[(size_t)(half * (DK / 2) + i) * DV + j] : 0.f;
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
    int4 ch = p.chunk_tab[c_begin];
    float gl = p.gam[((size_t)c_begin * HV + h) * C + ch.z - 1];  // gamma_n of this chunk
    int4 ch_nx = c_begin + 1 < c_end ? p.chunk_tab[c_begin + 1] : ch;
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tm = sm.tmem_base;
    // [X^T | O^T] double buffer at tm, tm + 128; Snew^T (DK columns) at tm + 256; the fp16 copy of
    // S^T, the A operand of the first product (DK / 2 columns), at tm + 384
    const uint32_t tS = tm + 256, tA = tm + 384;
    static_assert(DK <= 128, "tensor-memory layout");
    // this thread's DK / 2 state columns of row j into the A operand (lanes past the rows of a
    // 64-row tile hold values no product reads)
    const uint32_t tA_row = tA + lane_base + half * (DK / 4);
    if (warp < NCW) {
#pragma unroll
        for (int cc = 0; cc < DK / 2; cc += 32) put_sa32(tA_row + cc / 2, &s[cc]);
        tc::tmem_st_wait();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    // rows t < n of O (chunk at row t0), this thread's column j and half of the rows, from the
    // O^T half of an [X^T | O^T] buffer: into the staging tile, or straight to global memory
    auto put_out = [&](uint32_t tXO, int t0, int n) {
#pragma unroll
        for (int cc = 0; cc < C / 2; cc += 16) {
            const int c0 = half * (C / 2) + cc;
            float o[16];
            tc::tmem_ld16(tXO + lane_base + 64 + c0, o);
            tc::tmem_ld_wait();
            if (rowv)
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if constexpr (kStageOut<T>) sm.ostage[(c0 + i) * DV + j] = from_f<T>(o[i]);
                    else if (c0 + i < n) out[((size_t)(t0 + c0 + i) * HV + h) * DV + j] = from_f<T>(o[i]);
                }
        }
    };
    // (compute warps) the staged rows t < n leave as 16-byte vectors
    auto send_out = [&](int t0, int n) {
        if constexpr (kStageOut<T>) {
            constexpr int VPR = DV * (int)sizeof(T) / 16;  // vectors per row
            for (int e = tid; e < n * VPR; e += NCW * 32) {
                const int r = e / VPR, v = e % VPR;
                reinterpret_cast<uint4*>(out + ((size_t)(t0 + r) * HV + h) * DV)[v] =
                    reinterpret_cast<const uint4*>(sm.ostage + r * DV)[v];
            }
        }
    };

    bool ok = true;
    int prev_t0 = 0, prev_n = 0;  // the chunk whose outputs are still in tensor memory
    if (warp > NCW) {
        // ---- the copier: each tile buffer is refilled as soon as the chain frees it, in the order
        // the chain frees them ([W ; Qg] after the first product, U^T after V', K~ after the state
        // product, Aqk after the output product).  The next release of a buffer needs the copy issued
        // here, so none of these barriers can complete twice before this lane has seen the first.
        if (tid == COPIER) {
            for (int id = c_begin; id < c_end && ok; ++id) {
                const int it = id - c_begin, bb = it & 1;
                const uint32_t ph = (uint32_t)it & 1u, pb = (uint32_t)(it >> 1) & 1u;
                if (id + 2 < c_end) {  // tiles two chunks ahead into L2, so their copies wait on L2 only
                    const size_t nx = (size_t)(id + 2) * HV + h;
                    tc::bulk_prefetch_l2(p.WQ + nx * (2 * C * DK), WQ_BYTES);
                    tc::bulk_prefetch_l2(p.KT + nx * (DK * C), KT_BYTES);
                    tc::bulk_prefetch_l2(p.AQ + nx * (C * C), AQ_BYTES);
                    tc::bulk_prefetch_l2(u_src(id + 2), U_BYTES);
                }
                if (id + 2 < c_end) {
                    ok = tc::mbar_wait(tc::smem_u32(&sm.free_wq[bb]), pb);
                    if (ok) fetch_wq(id + 2);
                }
                if (ok && id + 1 < c_end) {
                    ok = tc::mbar_wait(tc::smem_u32(&sm.free_u), ph);
                    if (ok) fetch_u(id + 1);
                }
                if (ok && id + 2 < c_end) {
                    ok = tc::mbar_wait(tc::smem_u32(&sm.free_kt[bb]), pb);
                    if (ok) fetch_kt(id + 2);
                }
                if (ok && id + 1 < c_end) {
                    ok = tc::mbar_wait(tc::smem_u32(&sm.free_aq), ph);
                    if (ok) fetch_aq(id + 1);
                }
            }
        }
    } else
    for (int id = c_begin; id < c_end; ++id) {
        const uint32_t ph = (uint32_t)(id - c_begin) & 1u;
        const uint32_t tXO = tm + ph * 128;
        // loads one chunk ahead: the next chunk's gamma_n; two ahead: its table entry
        float gl_nx = 0.f;
        int4 ch_nx2 = ch_nx;
        if (id + 1 < c_end) gl_nx = p.gam[((size_t)(id + 1) * HV + h) * C + ch_nx.z - 1];
        if (id + 2 < c_end) ch_nx2 = p.chunk_tab[id + 2];
        bool okl = true;
        const int bb = (id - c_begin) & 1;
        const uint32_t pb = (uint32_t)((id - c_begin) >> 1) & 1u;
        if (tid == ISSUER) {
            okl = tc::mbar_wait(bar_wq(bb), pb);
            if (okl) {  // [X^T | O^T] = S^T [W ; Qg]^T, S^T from tensor memory
                const uint32_t b = tc::smem_u32(sm.wq[bb]);
                constexpr uint32_t idesc = tc::idesc_f16(DV, 128);
#pragma unroll
                for (int k = 0; k < DK / 16; ++k)
                    tc::mma_f16_ta(tXO, tA + 8 * k, tc::desc_kmajor(b, 2 * C, k), idesc, k > 0);
                tc::mma_commit(bar_x);
                tc::mma_commit(tc::smem_u32(&sm.free_wq[bb]));
            }
        } else if (warp < NCW) {
            if (id == ck_chunk && rowv)  // the state entering the checkpoint's chunk: column j of S
#pragma unroll
                for (int i = 0; i < DK / 2; ++i) ck_dst[(size_t)(half * (DK / 2) + i) * DV + j] = s[i];
            if (id > c_begin) {  // the previous chunk's outputs leave while this chunk's first product runs
                okl = __all_sync(0xffffffffu, tc::mbar_wait(bar_o, ph ^ 1u));
                if (okl) {
                    tc::fence_after_sync();
                    put_out(tm + (ph ^ 1u) * 128, prev_t0, prev_n);
                }
            }
            okl = __all_sync(0xffffffffu, okl && tc::mbar_wait(bar_x, ph) && tc::mbar_wait(bar_u, ph));
            tc::fence_after_sync();
            if (okl) {  // V'^T row j = U^T row j - X^T row j
#pragma unroll
                for (int cc = 0; cc < C / 2; cc += 16) {
                    const int c0 = half * (C / 2) + cc;
                    float x[16];
                    tc::tmem_ld16(tXO + lane_base + c0, x);
                    tc::tmem_ld_wait();
                    if (rowv)
#pragma unroll
                        for (int q = 0; q < 2; ++q) {  // 8 fp16 values per 16-byte vector
                            const uint32_t off = tc::kmajor_off16(j, c0 + 8 * q, DV);
                            uint4* pv = reinterpret_cast<uint4*>(reinterpret_cast<char*>(sm.vt) + off);
                            const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(sm.ut) + off);
                            const float2 u0 = tc::unpack_f16(u.x), u1 = tc::unpack_f16(u.y), u2 = tc::unpack_f16(u.z),
                                         u3 = tc::unpack_f16(u.w);
                            const float* xq = x + 8 * q;
                            *pv = make_uint4(tc::pack_f16(u0.x - xq[0], u0.y - xq[1]), tc::pack_f16(u1.x - xq[2], u1.y - xq[3]),
                                             tc::pack_f16(u2.x - xq[4], u2.y - xq[5]), tc::pack_f16(u3.x - xq[6], u3.y - xq[7]));
                        }
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tc::smem_u32(&sm.free_u));  // this warp has read its U^T rows
        }
        tc::fence_smem_to_async();
        tc::fence_before_sync();
        ok = bar_and(kChainBarrier, NCHAIN, okl);
        if (!ok) break;
        tc::fence_after_sync();
        if (tid == ISSUER) {
            okl = tc::mbar_wait(bar_kt(bb), pb);
            if (okl) {  // Snew^T = V'^T K~, K~ (rows s) read MN-major
                const uint32_t av = tc::smem_u32(sm.vt), bk = tc::smem_u32(sm.kt[bb]);
                constexpr uint32_t is = tc::idesc_f16(DV, DK) | tc::kTransposeB;
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    tc::mma_f16(tS, tc::desc_kmajor(av, DV, k), tc::desc_mnmajor16(bk, C, k), is, k > 0);
                tc::mma_commit(bar_s);
                tc::mma_commit(tc::smem_u32(&sm.free_kt[bb]));
            }
            if (okl) okl = tc::mbar_wait(bar_aq, ph);
            if (okl) {  // O^T += V'^T Aqk^T: queued behind the state product, off the state chain; the
                        // next chunk's first product waits for it (the tensor core runs them in order)
                const uint32_t av = tc::smem_u32(sm.vt), bq = tc::smem_u32(sm.aq);
                constexpr uint32_t io = tc::idesc_f16(DV, 64);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    tc::mma_f16(tXO + 64, tc::desc_kmajor(av, DV, k), tc::desc_kmajor(bq, C, k), io, true);
                tc::mma_commit(bar_o);
                tc::mma_commit(tc::smem_u32(&sm.free_aq));
            }
        } else if (warp < NCW) {
            if (id > c_begin) send_out(prev_t0, prev_n);  // staged before the middle barrier; the
                                                          // state product runs meanwhile
            okl = __all_sync(0xffffffffu, tc::mbar_wait(bar_s, ph));
            if (okl) {  // S^T <- e^{gamma_n} S^T + Snew^T, and its fp16 copy for the next chunk
                tc::fence_after_sync();
                const float egl = expf(gl);
#pragma unroll
                for (int cc = 0; cc < DK / 2; cc += 32) {
                    const int c0 = half * (DK / 2) + cc;
                    float v[32];
                    tc::tmem_ld16(tS + lane_base + c0, *reinterpret_cast<float(*)[16]>(v));
                    tc::tmem_ld16(tS + lane_base + c0 + 16, *reinterpret_cast<float(*)[16]>(v + 16));
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[cc + i] = fmaf(egl, s[cc + i], v[i]);
                    put_sa32(tA_row + cc / 2, &s[cc]);
                }
                tc::tmem_st_wait();
            }
        }
        tc::fence_before_sync();
        ok = bar_and(kChainBarrier, NCHAIN, okl);
        if (!ok) break;
        tc::fence_after_sync();
        prev_t0 = ch.y;
        prev_n = ch.z;
        ch = ch_nx;
        ch_nx = ch_nx2;
        gl = gl_nx;
    }
    ok = __syncthreads_and(ok);  // the chain, the copier and the idle lanes agree
    if (ok) {
        if (warp < NCW) {
            const uint32_t ph = (uint32_t)(c_end - 1 - c_begin) & 1u;
            const bool okw = __all_sync(0xffffffffu, tc::mbar_wait(bar_o, ph));
            if (okw) {  // the last chunk's outputs
                tc::fence_after_sync();
                put_out(tm + ph * 128, prev_t0, prev_n);
            } else if (lane == 0) {
                raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
            }
            if (rowv)  // final state: column j of S
#pragma unroll
                for (int i = 0; i < DK / 2; ++i) Sg[(size_t)(half * (DK / 2) + i) * DV + j] = s[i];
        }
        if (tid == ISSUER) {  // the releases nobody waited for, so that none lands after the CTA is gone
            const int n = c_end - c_begin;
            for (int it = max(0, n - 2); it < n; ++it) {
                tc::mbar_wait(tc::smem_u32(&sm.free_wq[it & 1]), (uint32_t)(it >> 1) & 1u);
                tc::mbar_wait(tc::smem_u32(&sm.free_kt[it & 1]), (uint32_t)(it >> 1) & 1u);
            }
            tc::mbar_wait(tc::smem_u32(&sm.free_aq), (uint32_t)(n - 1) & 1u);
        }
        if constexpr (kStageOut<T>) {
            __syncthreads();
            if (warp < NCW) send_out(prev_t0, prev_n);
        }
    } else if (tid == ISSUER) {
        raise_error(p.hdr, GDN_DEVERR_TIMEOUT);
        // (the copier has stopped issuing: its loop ends at its first failed wait, and every
        // wait of the chain threads above has returned)
        // let copies and products already in flight finish before the CTA's shared and tensor
        // memory go away
        for (uint32_t par = 0; par < 2; ++par) {
            for (int b = 0; b < 2; ++b) {
                tc::mbar_wait(bar_wq(b), par, 100000000ull);
                tc::mbar_wait(bar_kt(b), par, 100000000ull);
            }
            tc::mbar_wait(bar_aq, par, 100000000ull);
            tc::mbar_wait(bar_o, par, 100000000ull);
            tc::mbar_wait(bar_u, par, 100000000ull);
            for (int b = 0; b < 2; ++b) {
                tc::mbar_wait(tc::smem_u32(&sm.free_wq[b]), par, 100000000ull);
                tc::mbar_wait(tc::smem_u32(&sm.free_kt[b]), par, 100000000ull);
            }
            tc::mbar_wait(tc::smem_u32(&sm.free_aq), par, 100000000ull);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tm, 512);
}

}  // namespace

template <typename T, int DK, int DV>
cudaError_t launch_state(const ExtendArgs& p, int seg, cudaStream_t s) {
    const size_t shm = sizeof(StateTcSmem<T, DK, DV>);
    cudaError_t e =
        cudaFuncSetAttribute(state_tc_kernel<T, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    // a piece of P chunks touches at most P + 1 sequences
    const long long piece = ((long long)p.max_chunks + p.nseg - 1) / p.nseg;
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
