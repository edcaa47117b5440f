/*
 * ssd.h -- C ABI of the Mamba2 SSD chunk-scan layer in libgdn.so (sm_100a).
 *
 * The operation is the one page "flashinfer.mamba.ssd_combined_fwd" lists as
 * ssd_combined_fwd(x, dt, A, B, C, D, z, dt_bias, dt_softplus, dt_limit,
 * initial_states, ..., checkpoint_token_indices, checkpoint_state_slots,
 * checkpoint_states, return_final_states) in packed-varlen mode: the Mamba2
 * selective state-space scan (Dao and Gu, "Transformers are SSMs", the SSD
 * layer).  Per sequence n and head h, with group g = h / (H / G), step
 * dt'_t = clamp(softplus?(dt_t + dt_bias_h), dt_min, dt_max) and the state
 * h_t in R^{P x N} (headdim x dstate):
 *
 *     h_t = exp(dt'_t A_h) h_{t-1} + dt'_t x_t B_t^T
 *     y_t = (h_t C_t + D_h x_t) * (z_t * sigmoid(z_t))     (D and z optional)
 *
 * Sequences are given by cu_seqlens, so the page's seq_idx, chunk_indices and
 * chunk_offsets (metadata derived from the packing) are not taken.  Outputs
 * are token-major [T, H, P]; the page's chunk-major output storage is not
 * reproduced.
 *
 * Conventions (as in gdn.h): every pointer is device memory owned by the
 * caller and 16-byte aligned unless marked host; calls are asynchronous on
 * `stream`, allocate nothing, keep no state and may be captured into a CUDA
 * graph; the workspace starts with the sticky device error word read by
 * gdn_get_device_error() and cleared by gdn_reset_device_error().
 */
#ifndef SSD_H
#define SSD_H

#include "gdn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t nheads;      /* H, multiple of ngroups */
    int32_t headdim;     /* P: 64 */
    int32_t dstate;      /* N: 64 or 128 */
    int32_t ngroups;     /* G */
    int32_t state_dtype; /* GDN_DTYPE_F32, GDN_DTYPE_BF16 or GDN_DTYPE_F16: initial, final and checkpoint states */
    int32_t dt_softplus; /* 1: softplus(dt + dt_bias); 0: dt + dt_bias */
    int32_t d_per_dim;   /* 1: D is [H, P]; 0: D is [H] */
    float dt_min;        /* inclusive limits on the processed step (0 and +inf: none) */
    float dt_max;
} ssd_config_t;

/* Bytes of workspace ssd_combined_fwd needs for up to max_N sequences (the device error header and
 * the order in which the sequences are scanned, longest first). */
GDN_API size_t ssd_workspace_size(const ssd_config_t* cfg, int32_t max_N, int32_t max_T);

/*
 * The scan over N packed sequences of T rows in total.
 *   x [T, H, P] bf16; dt [T, H] bf16; A [H] fp32; B, C [T, G, N] bf16;
 *   D bf16 [H] or [H, P] (d_per_dim), or NULL; z [T, H, P] bf16 or NULL;
 *   dt_bias [H] fp32 or NULL; cu_seqlens [N + 1] int32, non-decreasing from 0 to T;
 *   initial_states [N, H, P, N] (state_dtype) or NULL for zero states;
 *   final_states [N, H, P, N] (state_dtype) or NULL: each sequence's last state;
 *   ckpt_token_indices, ckpt_state_slots [N] int32 and ckpt_states
 *   [num_ckpt, H, P, N] (state_dtype): all three NULL, or all given.  As in
 *   gdn_extend_checkpoints, boundary b_i is an exclusive absolute packed row with
 *   cu_seqlens[i] <= b_i <= cu_seqlens[i+1] and the captured state is the one
 *   after rows cu_seqlens[i] .. b_i - 1; a negative boundary or slot disables
 *   it, and an out-of-range one raises GDN_DEVERR_CKPT_RANGE and is skipped;
 *   out [T, H, P] bf16.
 * States are carried in fp32 and rounded to nearest even into state_dtype when
 * stored.  Returns GDN_OK, GDN_ERR_INVALID_ARG (null or misaligned pointer,
 * negative size, H % G != 0, dt_min > dt_max, checkpoint arguments given in
 * part), GDN_ERR_UNSUPPORTED (headdim, dstate or state_dtype outside the
 * supported set), GDN_ERR_WORKSPACE or GDN_ERR_CUDA.  A sequence whose bounds
 * are not 0 <= cu[i] <= cu[i+1] <= T raises GDN_DEVERR_SEQLENS and is skipped.
 */
GDN_API int ssd_combined_fwd(const ssd_config_t* cfg, const void* x, const void* dt, const float* A, const void* B,
                             const void* C, const void* D, const void* z, const float* dt_bias,
                             const int32_t* cu_seqlens, int32_t N, int32_t T, const void* initial_states,
                             void* final_states, const int32_t* ckpt_token_indices, const int32_t* ckpt_state_slots,
                             void* ckpt_states, int32_t num_ckpt, void* out, void* workspace, size_t workspace_bytes,
                             gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H */
