// Internal declarations shared by the kernels and the C-ABI layer of libgdn.
// Not part of the public interface (include/gdn.h is).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

constexpr int kChunk = 64;          // prefill chunk length C
constexpr int kConvK = 4;           // conv width K
constexpr int kHeaderBytes = 512;   // workspace header (error word + counters)
constexpr int kMaxVerifyDraft = 16; // D limit of gdn_verify

// header layout (int32 words)
constexpr int kHdrError = 0;        // sticky GDN_DEVERR_* bits
constexpr int kHdrNumChunks = 1;    // chunk count of the current extend batch
constexpr int kMaxSegments = 16;    // segments of an extend batch (see below)
constexpr int kHdrSegLen = 2;       // chunks in the largest segment
constexpr int kHdrSegOff = 3;       // [kMaxSegments]: first chunk_list entry of segment k
constexpr int kHdrSegCnt = kHdrSegOff + kMaxSegments;    // [kMaxSegments]: chunks in segment k
constexpr int kHdrSegSeqs = kHdrSegCnt + kMaxSegments;   // [kMaxSegments]: sequences with chunks in segment k
constexpr int kHdrItemNext = kHdrSegSeqs + kMaxSegments; // [kMaxSegments]: next per-chunk item of segment k
constexpr int kHdrSegRank = kHdrItemNext + kMaxSegments; // [kMaxSegments]: first rank with chunks in segment k
static_assert((kHdrSegRank + kMaxSegments) * 4 <= kHeaderBytes, "header too small");

// An extend batch is cut into S segments (S chosen by the host, at most
// kMaxSegments): the chunks, listed longest sequence first, in S pieces of
// consecutive list entries.  The per-chunk step runs segment by segment on the
// caller's stream; the state pass of segment k runs on a second stream once
// the per-chunk step has finished segment k, taking each sequence's chunks
// inside the piece and continuing from the state the previous piece left in
// its slot, alongside the per-chunk step of segment k+1.  A piece holds few sequences, so its state
// pass needs few SMs; the shortest sequences come last.
//
// The pieces grow geometrically by kSegGrowth: the chain cannot start before
// the first piece's per-chunk step ends, and the per-chunk step runs a little
// faster per chunk than the chain, so a short first piece starts the chain
// early while each later piece is still ready before the chain reaches it.
// Piece k holds list entries [seg_bound(k), seg_bound(k + 1)).
constexpr double kSegGrowth = 1.12;

__host__ __device__ inline int seg_bound(int k, int nseg, int total) {
    if (k <= 0) return 0;
    if (k >= nseg) return total;
    double rk = 1.0, rn = 1.0;
    for (int i = 0; i < nseg; ++i) {
        if (i < k) rk *= kSegGrowth;
        rn *= kSegGrowth;
    }
    const int b = (int)((double)total * (rk - 1.0) / (rn - 1.0));
    return b < 0 ? 0 : (b > total ? total : b);
}

// an upper bound on the entries of the largest piece of a list of at most `chunks` entries
__host__ inline long long seg_max_piece(long long chunks, int nseg) {
    if (nseg <= 1) return chunks;
    double rn = 1.0;
    for (int i = 0; i < nseg; ++i) rn *= kSegGrowth;
    return (long long)((double)chunks * (rn / kSegGrowth) * (kSegGrowth - 1.0) / (rn - 1.0)) + 2;
}

struct LayerDims {
    int HK, HV, dk, dv, G;  // G = HV / HK
    int conv_dim;           // 2*HK*dk + HV*dv
    float scale;            // resolved (> 0)
    float eps;
};

// ---- element access -------------------------------------------------------

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// SiLU, softplus and sigmoid in fp32 from the CUDA math library's expf/log1pf.
__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }
__device__ __forceinline__ float softplus_f(float x) { return x > 20.0f ? x : log1pf(expf(x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void raise_error(int32_t* hdr, int bits) {
    if (hdr) atomicOr(reinterpret_cast<int*>(hdr) + kHdrError, bits);
}

// Largest finite fp16 magnitude.  The prefill rounds its tensor-core operands to fp16; a kernel keeps
// the largest magnitude it rounded in a register (amax) and reports any above this bound once per warp.
constexpr float kF16Max = 65504.0f;
__device__ __forceinline__ void report_f16_range(int32_t* hdr, float amax) {
    if (__any_sync(0xffffffffu, !(amax <= kF16Max)) && (threadIdx.x & 31) == 0) raise_error(hdr, GDN_DEVERR_FP16_RANGE);
}

// ---- launch argument blocks ----------------------------------------------

struct DecodeArgs {
    LayerDims d;
    const float* A_log;
    const float* dt_bias;
    const void* conv_w;
    const void* conv_b;
    const void* x;      // [B*D, conv_dim]
    const void* a;      // [B*D, HV]
    const void* b;      // [B*D, HV]
    const int32_t* slots;
    int B, D, P;
    void* conv_state;   // decode: read/write; verify: read only
    float* ssm_state;   // decode: read/write; verify: read only
    float* state_ckpt;  // verify only
    void* conv_ckpt;    // verify only, nullable
    const int32_t* parents;  // verify only: [B, D] draft-tree parents (-1 = slot), nullable = a chain
    void* out;          // [B*D, HV, dv]
    int32_t* hdr;       // workspace header (error word)
};

struct CommitArgs {
    LayerDims d;
    const int32_t* slots;     // [B]
    const int32_t* accepted;  // [B], 0..D
    int B, D, P;
    const float* state_ckpt;  // [B, D, HV, dk, dv]
    const void* conv_ckpt;    // [B, D, conv_dim, K-1], nullable
    void* conv_state;         // [P, conv_dim, K-1]
    float* ssm_state;         // [P, HV, dk, dv]
    size_t conv_elem;         // bytes per conv element
    int32_t* hdr;             // workspace header (error word)
};

struct ExtendArgs {
    LayerDims d;
    const float* A_log;
    const float* dt_bias;
    const void* conv_w;
    const void* conv_b;
    const void* x;      // [T, conv_dim]
    const void* a;      // [T, HV]
    const void* b;      // [T, HV]
    const int32_t* cu;  // [N+1]
    const int32_t* slots;
    const int32_t* has_init;  // nullable
    int N, T, P;
    int max_chunks;     // upper bound on sum_n ceil(L_n / C)
    void* conv_state;
    float* ssm_state;
    void* out;          // [T, HV, dv]
    // optional state checkpoints, one per sequence (all null when not asked for)
    const int32_t* ck_idx;  // [N] exclusive absolute packed-row boundary; < 0 disables
    const int32_t* ck_row;  // [N] row of ck_states; < 0 disables
    float* ck_states;       // [num_ck, HV, dk, dv]
    void* ck_conv;          // [num_ck, conv_dim, K-1] (cfg dtype), nullable
    int num_ck;
    // workspace carve-out
    int32_t* hdr;
    int4* chunk_tab;    // [max_chunks] {seq, first row, length, chunk index within seq}
    int32_t* seq_chunk0;// [N+1] first chunk id of each sequence
    int32_t* seq_order; // [N] sequences by decreasing chunk count (the state pass's launch order)
    int32_t* rank_off;  // [N+1] chunk_list position of each rank's first chunk
    int32_t* chunk_list;// [max_chunks] chunk ids, rank by rank (longest sequence first)
    int nseg;           // S
    // per chunk, written by the per-chunk step (conv + SiLU, L2 norm, gates and the intra-chunk
    // products) and read by the state pass; the tiles are fp16 values already in the tensor core's
    // 128-byte swizzled shared-memory layout, so the state pass copies them verbatim.  Rows past the
    // end of a ragged chunk are zero.
    uint16_t* KQ;       // [max_chunks, HK, 2*C*dk]  [K ; Q*scale] (L2-normalised), 128 rows x dk
    uint16_t* W;        // [max_chunks, HV, dk*C]    W^T, W = T diag(beta e^gamma) K: dk rows x C
    uint16_t* U;        // [max_chunks, HV, dv*C]    U^T = (T diag(beta) V)^T, dv rows x C
    uint16_t* AQ;       // [max_chunks, HV, C*C]     masked decayed q.k, C rows x C
    float4* GV;         // [max_chunks, HV, C]       gate vectors, each block of C float4 read as
                        //                           float[4][C]: e^{gamma_r}, f_r = e^{gamma_n - gamma_r}
                        //                           (0 past the chunk end), gamma_r, e^{gamma_n}
};

// Dispatch on the supported (dk, dv) pairs; expects a LayerDims `p.d` in scope.
#define GDN_DISPATCH_DIMS(T, FN, ...)                                                   \
    do {                                                                                \
        if (p.d.dk == 128 && p.d.dv == 128) return FN<T, 128, 128>(__VA_ARGS__);        \
        if (p.d.dk == 128 && p.d.dv == 64) return FN<T, 128, 64>(__VA_ARGS__);          \
        if (p.d.dk == 64 && p.d.dv == 128) return FN<T, 64, 128>(__VA_ARGS__);          \
        if (p.d.dk == 64 && p.d.dv == 64) return FN<T, 64, 64>(__VA_ARGS__);            \
        return cudaErrorInvalidValue;                                                   \
    } while (0)

// True when chunk_map rejected the batch (it then publishes zero chunks).
__device__ __forceinline__ bool batch_rejected(const ExtendArgs& p) { return p.hdr[kHdrNumChunks] == 0; }

// The state checkpoint of sequence n: its boundary's offset inside the sequence (with *row set),
// -1 when none is asked for, -2 when the boundary lies outside the sequence or the row is out of range.
__device__ __forceinline__ int ckpt_offset(const ExtendArgs& p, int n, int* row) {
    if (!p.ck_idx) return -1;
    const int b = p.ck_idx[n], r = p.ck_row[n];
    if (b < 0 || r < 0) return -1;
    if (b < p.cu[n] || b > p.cu[n + 1] || r >= p.num_ck) return -2;
    *row = r;
    return b - p.cu[n];
}

// Per-chunk step on tensor cores (gdn_chunk_tc.cu) for the chunks of one
// segment: conv + SiLU, L2 norm, gates and the intra-chunk products of
// (chunk, qk head) items, taken dynamically by persistent CTAs.
template <typename T, int DK, int DV>
cudaError_t launch_chunk(const ExtendArgs& p, int seg, cudaStream_t s);

// Serial state pass + outputs on tensor cores (gdn_state_tc.cu) for one
// segment: one CTA per (sequence, value head), longest sequences first.
template <typename T, int DK, int DV>
cudaError_t launch_state(const ExtendArgs& p, int seg, cudaStream_t s);

// Records the calling thread's i-th profiling event on `s` if one is set
// (see gdn_set_launch_events); a no-op otherwise.
void mark_launch(cudaStream_t s, int i);

// Records a CUDA failure for gdn_last_cuda_error and returns GDN_ERR_CUDA.
int record_cuda_failure(cudaError_t e);

size_t extend_workspace_bytes(const LayerDims& d, int max_N, int max_T, int* max_chunks_out);

// Host checks of an extend call's arguments other than its workspace (configuration, parameters,
// sizes, required pointers, alignment).  Returns GDN_OK or the GDN_ERR_* code gdn_extend returns for
// them; *nothing is set when the batch is empty (N == 0 or T == 0), in which case the pointers are
// not checked.
int check_extend_args(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
                      const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T, const int32_t* state_indices,
                      const int32_t* has_initial_state, const void* conv_state, const float* ssm_state, int32_t P,
                      const void* out, LayerDims* d, bool* nothing);
void carve_extend_workspace(ExtendArgs& e, void* ws, int max_N, int max_T);

cudaError_t launch_decode(const DecodeArgs& args, int dtype, cudaStream_t s);
cudaError_t launch_verify(const DecodeArgs& args, int dtype, cudaStream_t s);
cudaError_t launch_commit(const CommitArgs& args, cudaStream_t s);
cudaError_t launch_extend(const ExtendArgs& args, int dtype, cudaStream_t s);

}  // namespace gdn
