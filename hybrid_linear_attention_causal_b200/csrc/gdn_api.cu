// C ABI of libgdn: argument validation, workspace sizing and kernel dispatch.
// The operations and their contracts are documented in include/gdn.h.

#include <math.h>
#include <stdio.h>
#include <string.h>

#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace {

thread_local char g_cuda_err[256] = "";

constexpr int kMaxEvents = 16;
thread_local cudaEvent_t g_events[kMaxEvents];
thread_local int g_num_events = 0;

int cuda_fail(cudaError_t e) {
    snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return GDN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the configuration and fills the resolved layer dimensions.
int check_cfg(const gdn_config_t* cfg, gdn::LayerDims* d) {
    if (!cfg) return GDN_ERR_INVALID_ARG;
    if (cfg->num_qk_heads <= 0 || cfg->num_v_heads <= 0 || cfg->num_v_heads % cfg->num_qk_heads != 0)
        return GDN_ERR_INVALID_ARG;
    if (cfg->head_k_dim <= 0 || cfg->head_v_dim <= 0 || cfg->conv_kernel <= 0) return GDN_ERR_INVALID_ARG;
    if (!(cfg->l2_eps >= 0.0f) || isnan(cfg->scale)) return GDN_ERR_INVALID_ARG;
    if ((cfg->head_k_dim != 64 && cfg->head_k_dim != 128) || (cfg->head_v_dim != 64 && cfg->head_v_dim != 128))
        return GDN_ERR_UNSUPPORTED;
    if (cfg->conv_kernel != gdn::kConvK) return GDN_ERR_UNSUPPORTED;
    if (cfg->dtype != GDN_DTYPE_F32 && cfg->dtype != GDN_DTYPE_BF16) return GDN_ERR_UNSUPPORTED;
    const long long cd = 2LL * cfg->num_qk_heads * cfg->head_k_dim + (long long)cfg->num_v_heads * cfg->head_v_dim;
    if (cd > (1LL << 24)) return GDN_ERR_UNSUPPORTED;
    if (d) {
        d->HK = cfg->num_qk_heads;
        d->HV = cfg->num_v_heads;
        d->dk = cfg->head_k_dim;
        d->dv = cfg->head_v_dim;
        d->G = d->HV / d->HK;
        d->conv_dim = (int)cd;
        d->scale = cfg->scale > 0.0f ? cfg->scale : 1.0f / sqrtf((float)cfg->head_k_dim);
        d->eps = cfg->l2_eps;
    }
    return GDN_OK;
}

int check_params(const gdn_params_t* p) {
    if (!p || !p->A_log || !p->dt_bias || !p->conv_weight) return GDN_ERR_INVALID_ARG;
    if (!aligned16(p->A_log) || !aligned16(p->dt_bias) || !aligned16(p->conv_weight)) return GDN_ERR_INVALID_ARG;
    if (p->conv_bias && !aligned16(p->conv_bias)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

template <typename... P>
bool all_aligned(P... ptrs) {
    return (aligned16(ptrs) && ...);
}

}  // namespace

namespace gdn {
int record_cuda_failure(cudaError_t e) { return cuda_fail(e); }

namespace {
// The bounded mbarrier wait of the tensor-core kernels, on a barrier that this thread completes itself
// (arrive) or that nothing completes; a wait that gives up raises GDN_DEVERR_TIMEOUT and returns.
__global__ void bounded_wait_check_kernel(int32_t* hdr, int arrive, unsigned long long limit_ns) {
    __shared__ __align__(8) unsigned long long bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = tc::smem_u32(&bar);
    tc::mbar_init(b, 1);
    tc::fence_mbar_init();
    if (arrive) tc::mbar_arrive(b);
    if (!tc::mbar_wait(b, 0, limit_ns)) raise_error(hdr, GDN_DEVERR_TIMEOUT);
}
}  // namespace


int check_extend_args(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
                      const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T, const int32_t* state_indices,
                      const int32_t* has_initial_state, const void* conv_state, const float* ssm_state, int32_t P,
                      const void* out, LayerDims* d, bool* nothing) {
    *nothing = false;
    int rc = check_cfg(cfg, d);
    if (rc != GDN_OK) return rc;
    if ((rc = check_params(params)) != GDN_OK) return rc;
    if (N < 0 || T < 0 || P < 0) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens) return GDN_ERR_INVALID_ARG;
    if (N == 0 || T == 0) {
        *nothing = true;
        return GDN_OK;
    }
    if (!mixed_qkv || !a || !b || !state_indices || !conv_state || !ssm_state || !out) return GDN_ERR_INVALID_ARG;
    if (!all_aligned(mixed_qkv, a, b, cu_seqlens, state_indices, conv_state, ssm_state, out))
        return GDN_ERR_INVALID_ARG;
    if (has_initial_state && !aligned16(has_initial_state)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

}  // namespace gdn


void gdn::mark_launch(cudaStream_t s, int i) {
    if (i < g_num_events) cudaEventRecord(g_events[i], s);
}

extern "C" {

int gdn_set_launch_events(void* const* events, int32_t n) {
    if (n < 0 || n > kMaxEvents || (n > 0 && !events)) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) g_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_num_events = n;
    return GDN_OK;
}

const char* gdn_strerror(int code) {
    switch (code) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument (null pointer, bad shape, misalignment or negative size)";
        case GDN_ERR_UNSUPPORTED: return "unsupported configuration (dk/dv must be 64 or 128, K 4, dtype f32/bf16)";
        case GDN_ERR_WORKSPACE: return "workspace too small for the requested sizes";
        case GDN_ERR_CUDA: return "CUDA launch failure (see gdn_last_cuda_error)";
        default: return "unknown error code";
    }
}

const char* gdn_last_cuda_error(void) { return g_cuda_err; }

size_t gdn_extend_workspace_size(const gdn_config_t* cfg, int32_t max_N, int32_t max_T) {
    gdn::LayerDims d;
    if (check_cfg(cfg, &d) != GDN_OK || max_N < 0 || max_T < 0) return 0;
    return gdn::extend_workspace_bytes(d, max_N, max_T, nullptr);
}

size_t gdn_decode_workspace_size(const gdn_config_t* cfg, int32_t max_B) {
    if (check_cfg(cfg, nullptr) != GDN_OK || max_B < 0) return 0;
    return gdn::kHeaderBytes;
}

size_t gdn_verify_workspace_size(const gdn_config_t* cfg, int32_t max_B, int32_t D) {
    if (check_cfg(cfg, nullptr) != GDN_OK || max_B < 0 || D < 1 || D > gdn::kMaxVerifyDraft) return 0;
    return gdn::kHeaderBytes;
}

namespace {

// gdn_extend and gdn_extend_checkpoints: `ck` carries the checkpoint arguments (all null for none)
int extend_impl(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
                const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T, const int32_t* state_indices,
                const int32_t* has_initial_state, void* conv_state, float* ssm_state, int32_t P, void* out,
                const gdn::ExtendArgs& ck, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn::LayerDims d;
    bool nothing = false;
    int rc = gdn::check_extend_args(cfg, params, mixed_qkv, a, b, cu_seqlens, N, T, state_indices, has_initial_state,
                                    conv_state, ssm_state, P, out, &d, &nothing);
    if (rc != GDN_OK) return rc;
    if (!workspace) return GDN_ERR_INVALID_ARG;
    if (nothing) return GDN_OK;
    if (!aligned16(workspace)) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < gdn::extend_workspace_bytes(d, N, T, nullptr)) return GDN_ERR_WORKSPACE;

    gdn::ExtendArgs e{};
    e.d = d;
    e.A_log = params->A_log;
    e.dt_bias = params->dt_bias;
    e.conv_w = params->conv_weight;
    e.conv_b = params->conv_bias;
    e.x = mixed_qkv;
    e.a = a;
    e.b = b;
    e.cu = cu_seqlens;
    e.slots = state_indices;
    e.has_init = has_initial_state;
    e.N = N;
    e.T = T;
    e.P = P;
    e.conv_state = conv_state;
    e.ssm_state = ssm_state;
    e.out = out;
    e.ck_idx = ck.ck_idx;
    e.ck_row = ck.ck_row;
    e.ck_states = ck.ck_states;
    e.ck_conv = ck.ck_conv;
    e.num_ck = ck.num_ck;
    // about one segment per 16384 packed rows (measured best on B200 among 4096 .. 40000; 8192 and
    // 4096 again slower on the 8-sequence 32768-row batch with the fused per-chunk step): a
    // segment's per-chunk work then hides the previous segment's state pass, and each launch's
    // ramp-up and tail stay small against its work
    e.nseg = T / 16384 < 1 ? 1 : (T / 16384 > gdn::kMaxSegments ? gdn::kMaxSegments : T / 16384);
    gdn::carve_extend_workspace(e, workspace, N, T);
    cudaError_t err = gdn::launch_extend(e, cfg->dtype, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : cuda_fail(err);
}

}  // namespace

int gdn_extend(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
               const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T, const int32_t* state_indices,
               const int32_t* has_initial_state, void* conv_state, float* ssm_state, int32_t P, void* out,
               void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    const gdn::ExtendArgs none{};
    return extend_impl(cfg, params, mixed_qkv, a, b, cu_seqlens, N, T, state_indices, has_initial_state, conv_state,
                       ssm_state, P, out, none, workspace, workspace_bytes, stream);
}

int gdn_extend_checkpoints(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
                           const void* b, const int32_t* cu_seqlens, int32_t N, int32_t T,
                           const int32_t* state_indices, const int32_t* has_initial_state, void* conv_state,
                           float* ssm_state, int32_t P, void* out, const int32_t* ckpt_token_indices,
                           const int32_t* ckpt_state_slots, float* ckpt_states, void* ckpt_conv, int32_t num_ckpt,
                           void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (num_ckpt < 0 || !ckpt_token_indices || !ckpt_state_slots || !ckpt_states) return GDN_ERR_INVALID_ARG;
    if (!all_aligned(ckpt_token_indices, ckpt_state_slots, ckpt_states)) return GDN_ERR_INVALID_ARG;
    if (ckpt_conv && !aligned16(ckpt_conv)) return GDN_ERR_INVALID_ARG;
    gdn::ExtendArgs ck{};
    ck.ck_idx = ckpt_token_indices;
    ck.ck_row = ckpt_state_slots;
    ck.ck_states = ckpt_states;
    ck.ck_conv = ckpt_conv;
    ck.num_ck = num_ckpt;
    return extend_impl(cfg, params, mixed_qkv, a, b, cu_seqlens, N, T, state_indices, has_initial_state, conv_state,
                       ssm_state, P, out, ck, workspace, workspace_bytes, stream);
}

int gdn_decode(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
               const void* b, const int32_t* state_indices, int32_t B, void* conv_state, float* ssm_state,
               int32_t P, void* out, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn::LayerDims d;
    int rc = check_cfg(cfg, &d);
    if (rc != GDN_OK) return rc;
    if ((rc = check_params(params)) != GDN_OK) return rc;
    if (B < 0 || P < 0) return GDN_ERR_INVALID_ARG;
    if (!workspace) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!mixed_qkv || !a || !b || !state_indices || !conv_state || !ssm_state || !out) return GDN_ERR_INVALID_ARG;
    if (!all_aligned(mixed_qkv, a, b, state_indices, conv_state, ssm_state, out, workspace))
        return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < (size_t)gdn::kHeaderBytes) return GDN_ERR_WORKSPACE;
    gdn::DecodeArgs p{};
    p.d = d;
    p.A_log = params->A_log;
    p.dt_bias = params->dt_bias;
    p.conv_w = params->conv_weight;
    p.conv_b = params->conv_bias;
    p.x = mixed_qkv;
    p.a = a;
    p.b = b;
    p.slots = state_indices;
    p.B = B;
    p.D = 1;
    p.P = P;
    p.conv_state = conv_state;
    p.ssm_state = ssm_state;
    p.out = out;
    p.hdr = static_cast<int32_t*>(workspace);
    cudaError_t err = gdn::launch_decode(p, cfg->dtype, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : cuda_fail(err);
}

namespace {

int verify_impl(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
                const void* b, const int32_t* state_indices, const int32_t* parents, int32_t B, int32_t D,
                const void* conv_state, const float* ssm_state, int32_t P, float* state_ckpt, void* conv_ckpt,
                void* out, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn::LayerDims d;
    int rc = check_cfg(cfg, &d);
    if (rc != GDN_OK) return rc;
    if ((rc = check_params(params)) != GDN_OK) return rc;
    if (B < 0 || P < 0 || D < 1 || D > gdn::kMaxVerifyDraft) return GDN_ERR_INVALID_ARG;
    if (!workspace) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!mixed_qkv || !a || !b || !state_indices || !conv_state || !ssm_state || !state_ckpt || !out)
        return GDN_ERR_INVALID_ARG;
    if (!all_aligned(mixed_qkv, a, b, state_indices, conv_state, ssm_state, state_ckpt, out, workspace))
        return GDN_ERR_INVALID_ARG;
    if (conv_ckpt && !aligned16(conv_ckpt)) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < (size_t)gdn::kHeaderBytes) return GDN_ERR_WORKSPACE;
    gdn::DecodeArgs p{};
    p.d = d;
    p.A_log = params->A_log;
    p.dt_bias = params->dt_bias;
    p.conv_w = params->conv_weight;
    p.conv_b = params->conv_bias;
    p.x = mixed_qkv;
    p.a = a;
    p.b = b;
    p.slots = state_indices;
    p.B = B;
    p.D = D;
    p.P = P;
    p.conv_state = const_cast<void*>(conv_state);
    p.ssm_state = const_cast<float*>(ssm_state);
    p.state_ckpt = state_ckpt;
    p.conv_ckpt = conv_ckpt;
    p.parents = parents;
    p.out = out;
    p.hdr = static_cast<int32_t*>(workspace);
    cudaError_t err = gdn::launch_verify(p, cfg->dtype, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : cuda_fail(err);
}

}  // namespace

int gdn_verify(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
               const void* b, const int32_t* state_indices, int32_t B, int32_t D, const void* conv_state,
               const float* ssm_state, int32_t P, float* state_ckpt, void* conv_ckpt, void* out, void* workspace,
               size_t workspace_bytes, gdn_stream_t stream) {
    return verify_impl(cfg, params, mixed_qkv, a, b, state_indices, nullptr, B, D, conv_state, ssm_state, P,
                       state_ckpt, conv_ckpt, out, workspace, workspace_bytes, stream);
}

int gdn_verify_tree(const gdn_config_t* cfg, const gdn_params_t* params, const void* mixed_qkv, const void* a,
                    const void* b, const int32_t* state_indices, const int32_t* parents, int32_t B, int32_t D,
                    const void* conv_state, const float* ssm_state, int32_t P, float* state_ckpt, void* conv_ckpt,
                    void* out, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    if (!parents || !aligned16(parents)) return GDN_ERR_INVALID_ARG;
    return verify_impl(cfg, params, mixed_qkv, a, b, state_indices, parents, B, D, conv_state, ssm_state, P,
                       state_ckpt, conv_ckpt, out, workspace, workspace_bytes, stream);
}

size_t gdn_commit_workspace_size(const gdn_config_t* cfg, int32_t max_B) {
    if (check_cfg(cfg, nullptr) != GDN_OK || max_B < 0) return 0;
    return gdn::kHeaderBytes;
}

int gdn_commit(const gdn_config_t* cfg, const int32_t* state_indices, const int32_t* accepted, int32_t B, int32_t D,
               const float* state_ckpt, const void* conv_ckpt, void* conv_state, float* ssm_state, int32_t P,
               void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn::LayerDims d;
    int rc = check_cfg(cfg, &d);
    if (rc != GDN_OK) return rc;
    if (B < 0 || P < 0 || D < 1 || D > gdn::kMaxVerifyDraft) return GDN_ERR_INVALID_ARG;
    if (!workspace) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!state_indices || !accepted || !state_ckpt || !ssm_state) return GDN_ERR_INVALID_ARG;
    if (conv_ckpt && !conv_state) return GDN_ERR_INVALID_ARG;
    if (!all_aligned(state_indices, accepted, state_ckpt, ssm_state, workspace)) return GDN_ERR_INVALID_ARG;
    if (conv_ckpt && (!aligned16(conv_ckpt) || !aligned16(conv_state))) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < (size_t)gdn::kHeaderBytes) return GDN_ERR_WORKSPACE;
    gdn::CommitArgs p{};
    p.d = d;
    p.slots = state_indices;
    p.accepted = accepted;
    p.B = B;
    p.D = D;
    p.P = P;
    p.state_ckpt = state_ckpt;
    p.conv_ckpt = conv_ckpt;
    p.conv_state = conv_state;
    p.ssm_state = ssm_state;
    p.conv_elem = cfg->dtype == GDN_DTYPE_BF16 ? 2 : 4;
    p.hdr = static_cast<int32_t*>(workspace);
    cudaError_t err = gdn::launch_commit(p, reinterpret_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? GDN_OK : cuda_fail(err);
}

int gdn_check_bounded_wait(int32_t arrive, int64_t limit_ns, void* workspace, size_t workspace_bytes,
                           gdn_stream_t stream) {
    if (limit_ns <= 0 || limit_ns > 1000000000LL || !workspace || !aligned16(workspace)) return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < (size_t)gdn::kHeaderBytes) return GDN_ERR_WORKSPACE;
    gdn::bounded_wait_check_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<int32_t*>(workspace), arrive != 0, (unsigned long long)limit_ns);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

int gdn_get_device_error(const void* workspace, int32_t* err_out, gdn_stream_t stream) {
    if (!workspace || !err_out) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(err_out, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

int gdn_reset_device_error(void* workspace, gdn_stream_t stream) {
    if (!workspace) return GDN_ERR_INVALID_ARG;
    cudaError_t e = cudaMemsetAsync(workspace, 0, gdn::kHeaderBytes, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

}  // extern "C"
