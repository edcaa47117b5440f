/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet layer library (libgdn.so).
 *
 * The library runs the linear-attention half of a hybrid full-attention + GDN
 * model: the call that page "pymllm.layers.attention.hybrid_backend" shows as
 * HybridAttnBackend.forward_gdn(layer, forward_batch, mixed_qkv, a, b), with
 * the per-layer parameters that `layer` carries (A_log, dt_bias, conv weight)
 * passed explicitly.  The forward modes of page "SGLang GDN hybrid linear
 * attention test matrix" (section on the forward-mode contract: decode/idle,
 * extend and target-verify are the legal modes) map onto three entry points:
 *
 *   gdn_extend  EXTEND / MIXED / DRAFT_EXTEND: ragged packed-varlen prefill
 *               (gdn_extend_checkpoints: the same, also capturing each
 *               sequence's state at one token boundary, for prefix caching)
 *   gdn_decode  DECODE / IDLE: one token per request (IDLE = zero requests)
 *   gdn_verify  TARGET_VERIFY: D draft tokens per request, state checkpoints
 *               (gdn_verify_tree: the draft tokens form a tree given by parent indices)
 *   gdn_commit  the accepted prefix of a verify pass back into the pools
 *
 * The same library also exports the Mamba2 SSD chunk scan (ssd_combined_fwd),
 * declared in ssd.h, which shares this header's conventions and error codes.
 *
 * What every mode computes, per request and value head h (qk head h / (HV/HK)):
 *   conv:  y_t = SiLU(sum_{j<K} w[c,j] x_{t-K+1+j}[c] (+ bias[c])) per channel c,
 *          rows before the request's first new row come from its conv-state slot;
 *   split: y = [q (HK*dk) | k (HK*dk) | v (HV*dv)], head-major, dim-minor;
 *   norm:  q <- q / sqrt(|q|^2 + l2_eps), likewise k;
 *   gates: g = -exp(A_log[h]) * softplus(a_t[h] + dt_bias[h]), beta = sigmoid(b_t[h]);
 *   rule:  S_t = exp(g_t) (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *          o_t = scale * S_t^T q_t   (S in R^{dk x dv}, fp32),
 * which is the gated delta rule of Gated DeltaNet (Yang, Kautz, Hatamizadeh,
 * ICLR 2025).  scale <= 0 selects 1/sqrt(dk), the default of page
 * "pymllm.layers.attention.radix_attention" (RadixAttention, `scaling`).
 *
 * Conventions shared by all calls
 *   - Every pointer argument is DEVICE memory owned by the caller unless its
 *     comment says host.  The library allocates no device memory.  The state
 *     it does keep: per host thread and device, a second stream with its fork
 *     and join events (created by that thread's first extend call on the
 *     device, kept until the process exits; see gdn_extend); per host thread,
 *     the profiling events set by gdn_set_launch_events; and, per device, the
 *     one scratch array behind gdn_extend_static_scratch.  Calls on different
 *     streams with disjoint outputs and workspaces may run concurrently, with
 *     one exception: gdn_extend_static_scratch calls share that array, so
 *     calls of it that overlap on the GPU race (see there).
 *   - Every call is asynchronous and stream-ordered on `stream` (a
 *     cudaStream_t; NULL is the legacy default stream).  No call synchronises
 *     the host, so decode and verify can be captured in a CUDA graph, and so
 *     can extend for a fixed (N, T).
 *   - dtype GDN_DTYPE_BF16 or GDN_DTYPE_F32 applies to mixed_qkv, a, b, out,
 *     conv_weight, conv_bias and the conv-state pool.  A_log, dt_bias and the
 *     ssm-state pool (and verify checkpoints) are always fp32.
 *   - Pool layouts: conv_state [P, conv_dim, K-1] (the K-1 most recent raw rows
 *     of each channel, index 0 oldest), ssm_state [P, HV, dk, dv] (dv fastest),
 *     conv_dim = 2*HK*dk + HV*dv.
 *   - state_indices[i] names request i's pool slot.  A negative entry marks a
 *     padded request: its output rows are written as zeros and nothing else is
 *     touched.  An entry >= P is a caller error detected on the device: the
 *     request is treated as padded and GDN_DEVERR_SLOT_RANGE is raised in the
 *     workspace error word.  Slots not named by any request are never read or
 *     written.  Two live requests naming the same slot race (undefined).
 *   - Supported shapes: dk, dv in {64, 128}; HV % HK == 0; K == 4.  Every
 *     pointer must be 16-byte aligned.
 *   - Return value: GDN_OK, or a GDN_ERR_* code with nothing launched.
 *     Launch failures return GDN_ERR_CUDA; gdn_last_cuda_error() gives the
 *     CUDA error string of the most recent one on the calling thread.
 *   - Workspace: caller-allocated device memory of at least the size the
 *     matching *_workspace_size() returns.  Its first 512 bytes are a header
 *     whose first int32 is a sticky device error word: kernels OR GDN_DEVERR_*
 *     bits into it and never clear it.  Zero it once after allocation with
 *     gdn_reset_device_error() (or cudaMemset) and read it with
 *     gdn_get_device_error().
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

typedef struct CUstream_st* gdn_stream_t; /* same type as cudaStream_t */

/* return codes */
#define GDN_OK 0
#define GDN_ERR_INVALID_ARG 1 /* null required pointer, bad shape, misalignment, negative size */
#define GDN_ERR_UNSUPPORTED 2 /* well-formed but outside the supported set (dk/dv/K/dtype) */
#define GDN_ERR_WORKSPACE 3   /* workspace too small for (N, T) or (B, D) */
#define GDN_ERR_CUDA 4        /* a kernel launch failed */

/* device error bits (sticky word at the start of the workspace) */
#define GDN_DEVERR_SLOT_RANGE 0x1 /* a state index >= P was skipped */
#define GDN_DEVERR_SEQLENS 0x2    /* cu_seqlens not non-decreasing from 0 to T; the batch was skipped */
#define GDN_DEVERR_TIMEOUT 0x4    /* a tensor-core wait gave up after its time limit; results are invalid */
#define GDN_DEVERR_ACCEPT_RANGE 0x8 /* a commit's accepted count was outside 0..D; that request was skipped */
#define GDN_DEVERR_CKPT_RANGE 0x10  /* a checkpoint boundary outside its sequence or a row >= num_ckpt; skipped */
#define GDN_DEVERR_TREE 0x20        /* a draft tree parent outside -1 .. t-1; that request was treated as padded */
#define GDN_DEVERR_FP16_RANGE 0x40  /* a prefill value staged as an fp16 tensor-core operand exceeded 65504 in
                                       magnitude (see gdn_extend); that batch's results are invalid */

/* element types */
#define GDN_DTYPE_F32 0
#define GDN_DTYPE_BF16 1
#define GDN_DTYPE_F16 2 /* fp16: a state storage type of ssd.h only */

typedef struct {
    int32_t num_qk_heads; /* HK */
    int32_t num_v_heads;  /* HV, multiple of HK */
    int32_t head_k_dim;   /* dk: 64 or 128 */
    int32_t head_v_dim;   /* dv: 64 or 128 */
    int32_t conv_kernel;  /* K: 4 */
    int32_t dtype;        /* GDN_DTYPE_* */
    float scale;          /* <= 0: 1/sqrt(dk) */
    float l2_eps;         /* L2-norm epsilon, e.g. 1e-6 */
} gdn_config_t;

typedef struct {
    const float* A_log;      /* [HV] fp32 */
    const float* dt_bias;    /* [HV] fp32 */
    const void* conv_weight; /* [conv_dim, K], cfg dtype */
    const void* conv_bias;   /* [conv_dim], cfg dtype, or NULL for no bias */
} gdn_params_t;

/*
 * Workspace bytes for gdn_extend over at most max_N sequences and max_T
 * packed tokens: the chunk table, and per chunk of 64 rows the fp16 tiles the
 * per-chunk step hands the serial state pass ([K ; Q] per qk head; W^T, U^T and
 * the decayed q.k per value head) plus a 16-byte fp32 gate vector per row and
 * value head.  Returns 0 for an invalid configuration.
 */
GDN_API size_t gdn_extend_workspace_size(const gdn_config_t* cfg, int32_t max_N, int32_t max_T);

/*
 * EXTEND (prefill): sequence n owns rows cu_seqlens[n] .. cu_seqlens[n+1]-1
 * of the packed inputs and continues from pool slot state_indices[n].
 *
 *   mixed_qkv          [T, conv_dim] raw (pre-conv) rows, cfg dtype
 *   a, b               [T, HV] gate pre-activations, cfg dtype
 *   cu_seqlens         [N+1] int32 device, 0 = cu[0] <= cu[1] <= ... <= cu[N] = T
 *   state_indices      [N] int32 device, see the conventions above
 *   has_initial_state  [N] int32 device or NULL (= all 1); 0 reads the slot's
 *                      conv and ssm contents as zeros (they are overwritten)
 *   conv_state, ssm_state  pools of P slots, read and written in place
 *   out                [T, HV, dv] cfg dtype
 * Zero-length sequences are no-ops.  N == 0 or T == 0 returns GDN_OK with
 * nothing launched.  The final state of each sequence is written to its slot,
 * and the conv slot receives the K-1 most recent raw rows of (old conv state |
 * the sequence's rows).
 *
 * All work is ordered after earlier work on `stream` and complete before
 * later work on it.  Internally the call also uses a second stream of the
 * library (one per host thread and device, at the device's greatest stream
 * priority) that forks from and joins back into `stream`, so it is captured
 * along with `stream` into a CUDA graph; the first call on a device from a
 * host thread creates that stream and its two events, so make it before any
 * capture.
 */
GDN_API int gdn_extend(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
               const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T, const int32_t* state_indices,
               const int32_t* has_initial_state, void* conv_state, float* ssm_state, int32_t P, void* out,
               void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_extend that also captures, for prefix caching, each sequence's state at
 * one token boundary.  ckpt_token_indices [N] (device int32) holds an
 * exclusive ABSOLUTE packed-row boundary b_i with cu_seqlens[i] <= b_i <=
 * cu_seqlens[i+1]: the captured state is the one after rows
 * cu_seqlens[i] .. b_i - 1 (b_i == cu_seqlens[i] gives the state the sequence
 * started from, b_i == cu_seqlens[i+1] its final state).  ckpt_state_slots [N]
 * names the row of ckpt_states [num_ckpt, HV, dk, dv] (fp32) that receives it;
 * ckpt_conv [num_ckpt, conv_dim, K-1] (cfg dtype, or NULL) receives the conv
 * window at the boundary, the K-1 raw rows before it (reaching into the
 * sequence's starting conv window).  A negative boundary or row disables the
 * capture of that sequence, and padded sequences capture nothing; a boundary
 * outside its sequence or a row >= num_ckpt raises GDN_DEVERR_CKPT_RANGE and
 * skips it.  Two sequences naming the same row race.  Outputs and pools are
 * exactly those of gdn_extend, with the same workspace size.  Page
 * "flashinfer ... ssd_combined": checkpoint_token_indices (one exclusive
 * boundary per sequence, absolute for packed varlen, negative disables),
 * checkpoint_state_slots, checkpoint_states [num_checkpoints, nheads, headdim,
 * dstate]; and the tracked-state checkpoints of the prefill test on page
 * "SGLang GDN hybrid linear attention test matrix".
 */
GDN_API int gdn_extend_checkpoints(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv,
                                   const void* a, const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T,
                                   const int32_t* state_indices, const int32_t* has_initial_state, void* conv_state,
                                   float* ssm_state, int32_t P, void* out, const int32_t* ckpt_token_indices,
                                   const int32_t* ckpt_state_slots, float* ckpt_states, void* ckpt_conv,
                                   int32_t num_ckpt, void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/* Size of the fixed device scratch behind gdn_extend_static_scratch. */
#define GDN_EXTEND_STATIC_SCRATCH_BYTES (64u << 20)

/*
 * EXTEND for callers that cannot allocate device memory.  The paper has no
 * counterpart to this entry point; it exists for callers such as engine
 * plugins whose enqueue step may not allocate (the host framework's allocator
 * owns device memory), latency-critical paths that cannot take the device
 * synchronisation cudaMalloc/cudaFree may cause, and hosts that pass the
 * layer only its inputs and outputs.
 *
 * Same arguments and results as gdn_extend, minus the workspace: the scratch
 * comes from a fixed GDN_EXTEND_STATIC_SCRATCH_BYTES (64 MiB) array in the
 * library's own device memory, which every GPU that loads the library holds
 * until the process exits.  Nothing is allocated: no cudaMalloc, no cudaFree,
 * no allocating library routine.
 *   - Sizes whose gdn_extend_workspace_size(cfg, N, T) exceeds
 *     GDN_EXTEND_STATIC_SCRATCH_BYTES are rejected with GDN_ERR_WORKSPACE and
 *     nothing is launched (one sequence of up to 2175 tokens for the
 *     16/32-head, dk = dv = 128 layer; 15807 for the 4/8-head, 64 layer).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it, and,
 *     like gdn_extend, creates the library's second stream and its two
 *     events for the calling host thread (no device memory); make that first
 *     call outside any stream capture.  A failure there returns
 *     GDN_ERR_CUDA with the cause left in the CUDA runtime's last error.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; each call clears the part that must start at zero
 *     before its kernels run.  Calls whose work overlaps on the GPU (other
 *     streams, other host threads) race on the array: order them.
 *   - Device-detected argument errors are handled as in gdn_extend (the
 *     request or batch is skipped), but their error bits are not readable.
 */
GDN_API int gdn_extend_static_scratch(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv,
                                      const void* a, const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T,
                                      const int32_t* state_indices, const int32_t* has_initial_state,
                                      void* conv_state, float* ssm_state, int32_t P, void* out, gdn_stream_t stream);

/* Workspace bytes for gdn_decode (the error header only). */
GDN_API size_t gdn_decode_workspace_size(const gdn_config_t* cfg, int32_t max_B);

/*
 * DECODE: request i has one new row (row i of mixed_qkv [B, conv_dim], a and
 * b [B, HV]) and continues from slot state_indices[i]; its conv and ssm slots
 * are updated in place and out [B, HV, dv] receives the outputs.  B == 0
 * (IDLE) returns GDN_OK with nothing launched.
 */
GDN_API int gdn_decode(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
               const void* b, const int32_t* state_indices, int32_t B, void* conv_state, float* ssm_state,
               int32_t P, void* out, void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/* Workspace bytes for gdn_verify (the error header only). */
GDN_API size_t gdn_verify_workspace_size(const gdn_config_t* cfg, int32_t max_B, int32_t D);

/*
 * TARGET_VERIFY: request i has D draft rows (rows i*D .. i*D+D-1 of
 * mixed_qkv [B*D, conv_dim], a and b [B*D, HV]) and runs them in order from
 * slot state_indices[i].  Both pools are read only.  state_ckpt
 * [B, D, HV, dk, dv] fp32 receives the state after every draft token;
 * conv_ckpt [B, D, conv_dim, K-1] (cfg dtype, or NULL) the conv window after
 * every token; out [B*D, HV, dv] the outputs.  Checkpoints of padded requests
 * are left untouched.  1 <= D <= 16.  This is the speculative Mamba-state
 * buffer that the target-verify path of page "SGLang GDN hybrid linear
 * attention test matrix" (verification conventions) fills; committing an
 * accepted prefix back into the pool is a separate step.
 */
GDN_API int gdn_verify(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
               const void* b, const int32_t* state_indices, int32_t B, int32_t D, const void* conv_state,
               const float* ssm_state, int32_t P, float* state_ckpt, void* conv_ckpt, void* out, void* workspace,
               size_t workspace_bytes, gdn_stream_t stream);

/*
 * TARGET_VERIFY over a draft TREE (EAGLE topk > 1): as gdn_verify, except that
 * draft token t of request i continues from its parent parents[i*D + t]
 * (device int32 [B, D]) instead of from token t-1: -1 is the slot state, any
 * other parent must be an earlier token (0 <= parent < t).  Each token's
 * state, output, state_ckpt and conv_ckpt entries are those of the path from
 * the root to it; the conv window of a token is made of its ancestors' rows,
 * then the slot's window.  parents[i*D + t] == t-1 for every t is exactly
 * gdn_verify.  A parent outside -1 .. t-1 raises GDN_DEVERR_TREE and the
 * request is treated as padded.  Same workspace as gdn_verify.  The EAGLE
 * tree verification (topk = 2) of page "SGLang GDN hybrid linear attention
 * test matrix".
 */
GDN_API int gdn_verify_tree(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv,
                            const void* a, const void* b, const int32_t* state_indices, const int32_t* parents,
                            int32_t B, int32_t D, const void* conv_state, const float* ssm_state, int32_t P,
                            float* state_ckpt, void* conv_ckpt, void* out, void* workspace, size_t workspace_bytes,
                            gdn_stream_t stream);

/* Workspace bytes for gdn_commit (the error header only). */
GDN_API size_t gdn_commit_workspace_size(const gdn_config_t* cfg, int32_t max_B);

/*
 * Speculative commit, the step after gdn_verify: request i accepted accepted[i]
 * of its D draft tokens (accepted: device int32 [B]).  For accepted[i] >= 1
 * its pool slot state_indices[i] receives the checkpoints of its last accepted
 * token: ssm_state[slot] = state_ckpt[i, accepted[i] - 1] and, when conv_ckpt
 * is non-NULL, conv_state[slot] = conv_ckpt[i, accepted[i] - 1] (layouts as
 * gdn_verify writes them: state_ckpt [B, D, HV, dk, dv] fp32, conv_ckpt
 * [B, D, conv_dim, K-1] in the cfg dtype).  The pool then holds what
 * gdn_extend over the accepted tokens would have left.  accepted[i] == 0 leaves
 * the slot untouched (verify never writes the pool).  A negative slot is
 * padding and is skipped; a slot >= P raises GDN_DEVERR_SLOT_RANGE and an
 * accepted count outside 0..D raises GDN_DEVERR_ACCEPT_RANGE, and that request
 * is skipped.  1 <= D <= 16.  This is the accept step that follows the
 * target-verify pass of page "SGLang GDN hybrid linear attention test matrix"
 * (verification conventions: the speculative state buffer is committed for
 * the accepted draft prefix).
 */
GDN_API int gdn_commit(const gdn_config_t* cfg, const int32_t* state_indices, const int32_t* accepted, int32_t B,
                       int32_t D, const float* state_ckpt, const void* conv_ckpt, void* conv_state, float* ssm_state,
                       int32_t P, void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * Reads the sticky device error word of `workspace` into *err_out (host).
 * Enqueues a device-to-host copy on `stream` and waits for that stream, so it
 * must not be called during stream capture.  Returns GDN_ERR_CUDA on failure.
 */
GDN_API int gdn_get_device_error(const void* workspace, int32_t* err_out, gdn_stream_t stream);

/* Clears the device error word of `workspace` (an async memset on `stream`). */
GDN_API int gdn_reset_device_error(void* workspace, gdn_stream_t stream);

/*
 * Self-check of the failure path that keeps a stuck tensor-core kernel from
 * hanging the GPU.  Every wait of the prefill and SSD kernels on an mbarrier
 * phase (a tensor-core product, a bulk copy, another warp's hand-off) gives up
 * after a time limit, raises GDN_DEVERR_TIMEOUT in the workspace error word,
 * lets its copies in flight land and returns.  This call runs that same wait
 * in a one-thread kernel on `stream`: on an mbarrier the kernel completes
 * itself before waiting (arrive != 0: the wait succeeds at once) or that
 * nothing ever completes (arrive == 0: the wait runs out after limit_ns
 * nanoseconds, 0 < limit_ns <= 1e9, the bit is raised and the kernel
 * returns).  Read the result with gdn_get_device_error.  The workspace is
 * any buffer of at least 512 bytes (a decode workspace will do); the call is
 * asynchronous.  GDN_ERR_INVALID_ARG for a limit outside that range or a
 * null or misaligned workspace, GDN_ERR_WORKSPACE for one under 512 bytes.
 */
GDN_API int gdn_check_bounded_wait(int32_t arrive, int64_t limit_ns, void* workspace, size_t workspace_bytes,
                                   gdn_stream_t stream);

/*
 * Profiling aid (off by default).  With n > 0, the calling thread's later
 * gdn_extend / gdn_decode / gdn_verify / gdn_commit calls record events[i] (each a
 * cudaEvent_t created by the caller) at fixed points of the call; indices
 * >= n are not recorded.  n == 0 turns recording off.
 *   decode, verify, commit: 0 before the kernel, 1 after it (on `stream`).
 *   extend: on `stream`: 0 start, 1 after the chunk table, 2 after the
 *     last per-chunk segment (conv + SiLU, L2 norm, gates and the intra-chunk
 *     products), 3 after the conv-state update, 5 end (second stream
 *     joined); index 4 is not recorded; on the library's second stream: 6
 *     before the first and 7 after the last state-pass segment.  The batch is
 *     processed in segments of chunks (about one per 16384 packed rows, at
 *     most 16): the state pass of segment k runs on the second stream
 *     alongside the per-chunk step of segment k+1, so the two spans overlap.
 * Returns GDN_ERR_INVALID_ARG for n < 0, n > 16 or events == NULL with n > 0.
 */
GDN_API int gdn_set_launch_events(void* const* events, int32_t n);

/* Static description of a return code. */
GDN_API const char* gdn_strerror(int code);

/* CUDA error string of the most recent GDN_ERR_CUDA on the calling thread ("" if none). */
GDN_API const char* gdn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
