"""Thin ctypes binding of libgdn.so (include/gdn.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch supplies device memory and the current stream.  If the
library has not been built, every call raises; there is no other code path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_WORKSPACE = 3
GDN_ERR_CUDA = 4
GDN_DEVERR_SLOT_RANGE = 0x1
GDN_DEVERR_SEQLENS = 0x2
GDN_DEVERR_TIMEOUT = 0x4
GDN_DEVERR_ACCEPT_RANGE = 0x8
GDN_DEVERR_CKPT_RANGE = 0x10
GDN_DEVERR_TREE = 0x20
GDN_DEVERR_FP16_RANGE = 0x40
GDN_DTYPE_F32 = 0
GDN_DTYPE_BF16 = 1
GDN_DTYPE_F16 = 2
HEADER_BYTES = 512
MAX_VERIFY_DRAFT = 16

_DTYPES = {torch.float32: GDN_DTYPE_F32, torch.bfloat16: GDN_DTYPE_BF16}


class GdnConfigC(ctypes.Structure):
    _fields_ = [
        ("num_qk_heads", ctypes.c_int32),
        ("num_v_heads", ctypes.c_int32),
        ("head_k_dim", ctypes.c_int32),
        ("head_v_dim", ctypes.c_int32),
        ("conv_kernel", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("l2_eps", ctypes.c_float),
    ]


class SsdConfigC(ctypes.Structure):
    _fields_ = [
        ("nheads", ctypes.c_int32),
        ("headdim", ctypes.c_int32),
        ("dstate", ctypes.c_int32),
        ("ngroups", ctypes.c_int32),
        ("state_dtype", ctypes.c_int32),
        ("dt_softplus", ctypes.c_int32),
        ("d_per_dim", ctypes.c_int32),
        ("dt_min", ctypes.c_float),
        ("dt_max", ctypes.c_float),
    ]


class GdnParamsC(ctypes.Structure):
    _fields_ = [
        ("A_log", ctypes.c_void_p),
        ("dt_bias", ctypes.c_void_p),
        ("conv_weight", ctypes.c_void_p),
        ("conv_bias", ctypes.c_void_p),
    ]


class GdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = f"{where}: {strerror(code)} (code {code})"
        if code == GDN_ERR_CUDA:
            msg += f": {last_cuda_error()}"
        super().__init__(msg)
        self.code = code


@dataclass(frozen=True)
class GdnConfig:
    num_qk_heads: int
    num_v_heads: int
    head_k_dim: int
    head_v_dim: int
    dtype: torch.dtype = torch.bfloat16
    conv_kernel: int = 4
    scale: float = 0.0
    l2_eps: float = 1e-6

    @property
    def conv_dim(self) -> int:
        return 2 * self.num_qk_heads * self.head_k_dim + self.num_v_heads * self.head_v_dim

    def c(self) -> GdnConfigC:
        return GdnConfigC(self.num_qk_heads, self.num_v_heads, self.head_k_dim, self.head_v_dim, self.conv_kernel,
                          _DTYPES.get(self.dtype, -1), self.scale, self.l2_eps)

    @staticmethod
    def from_spec(spec) -> "GdnConfig":
        return GdnConfig(spec.HK, spec.HV, spec.dk, spec.dv, dtype=spec.dtype, conv_kernel=spec.K)


_lib_handle = None


def lib() -> ctypes.CDLL:
    """The loaded libgdn.so; raises if it has not been built."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libgdn.so not found at {LIB_PATH}: build it with "
                "`python -m hybrid_linear_attention_causal_b200.build` (there is no fallback path)"
            )
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        cfg_p, par_p = ctypes.POINTER(GdnConfigC), ctypes.POINTER(GdnParamsC)
        L.gdn_extend_workspace_size.argtypes = [cfg_p, i32, i32]
        L.gdn_extend_workspace_size.restype = sz
        L.gdn_decode_workspace_size.argtypes = [cfg_p, i32]
        L.gdn_decode_workspace_size.restype = sz
        L.gdn_verify_workspace_size.argtypes = [cfg_p, i32, i32]
        L.gdn_verify_workspace_size.restype = sz
        L.gdn_extend.argtypes = [cfg_p, par_p, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, i32, vp, vp, sz, vp]
        L.gdn_extend.restype = ctypes.c_int
        L.gdn_extend_checkpoints.argtypes = [cfg_p, par_p, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp,
                                             vp, vp, i32, vp, sz, vp]
        L.gdn_extend_checkpoints.restype = ctypes.c_int
        L.gdn_extend_static_scratch.argtypes = [cfg_p, par_p, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, i32, vp, vp]
        L.gdn_extend_static_scratch.restype = ctypes.c_int
        L.gdn_decode.argtypes = [cfg_p, par_p, vp, vp, vp, vp, i32, vp, vp, i32, vp, vp, sz, vp]
        L.gdn_decode.restype = ctypes.c_int
        L.gdn_verify.argtypes = [cfg_p, par_p, vp, vp, vp, vp, i32, i32, vp, vp, i32, vp, vp, vp, vp, sz, vp]
        L.gdn_verify.restype = ctypes.c_int
        L.gdn_verify_tree.argtypes = [cfg_p, par_p, vp, vp, vp, vp, vp, i32, i32, vp, vp, i32, vp, vp, vp, vp, sz, vp]
        L.gdn_verify_tree.restype = ctypes.c_int
        L.gdn_commit_workspace_size.argtypes = [cfg_p, i32]
        L.gdn_commit_workspace_size.restype = sz
        L.gdn_commit.argtypes = [cfg_p, vp, vp, i32, i32, vp, vp, vp, vp, i32, vp, sz, vp]
        L.gdn_commit.restype = ctypes.c_int
        ssd_p = ctypes.POINTER(SsdConfigC)
        L.ssd_workspace_size.argtypes = [ssd_p, i32, i32]
        L.ssd_workspace_size.restype = sz
        L.ssd_combined_fwd.argtypes = [ssd_p, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, vp, i32,
                                       vp, vp, sz, vp]
        L.ssd_combined_fwd.restype = ctypes.c_int
        L.gdn_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), vp]
        L.gdn_get_device_error.restype = ctypes.c_int
        L.gdn_reset_device_error.argtypes = [vp, vp]
        L.gdn_reset_device_error.restype = ctypes.c_int
        L.gdn_check_bounded_wait.argtypes = [i32, ctypes.c_int64, vp, sz, vp]
        L.gdn_check_bounded_wait.restype = ctypes.c_int
        L.gdn_set_launch_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
        L.gdn_set_launch_events.restype = ctypes.c_int
        L.gdn_strerror.argtypes = [ctypes.c_int]
        L.gdn_strerror.restype = ctypes.c_char_p
        L.gdn_last_cuda_error.argtypes = []
        L.gdn_last_cuda_error.restype = ctypes.c_char_p
        _lib_handle = L
    return _lib_handle


def strerror(code: int) -> str:
    return lib().gdn_strerror(int(code)).decode()


def last_cuda_error() -> str:
    return lib().gdn_last_cuda_error().decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libgdn takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("libgdn takes contiguous tensors only")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _params(params: dict) -> GdnParamsC:
    return GdnParamsC(_ptr(params["A_log"]), _ptr(params["dt_bias"]), _ptr(params["conv_w"]),
                      _ptr(params.get("conv_b")))


def _check(rc: int, where: str):
    if rc != GDN_OK:
        raise GdnError(rc, where)


def gdn_extend_workspace_size(cfg: GdnConfig, max_N: int, max_T: int) -> int:
    return int(lib().gdn_extend_workspace_size(ctypes.byref(cfg.c()), max_N, max_T))


def gdn_decode_workspace_size(cfg: GdnConfig, max_B: int) -> int:
    return int(lib().gdn_decode_workspace_size(ctypes.byref(cfg.c()), max_B))


def gdn_verify_workspace_size(cfg: GdnConfig, max_B: int, D: int) -> int:
    return int(lib().gdn_verify_workspace_size(ctypes.byref(cfg.c()), max_B, D))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed workspace (the zeroed header is the cleared error word)."""
    return torch.zeros(max(int(nbytes), HEADER_BYTES), dtype=torch.uint8, device=device)


def gdn_extend(cfg: GdnConfig, params: dict, mixed_qkv, a, b, cu_seqlens, state_indices, has_initial_state,
               conv_state, ssm_state, out, workspace, stream=None) -> None:
    N = int(state_indices.shape[0])
    T = int(mixed_qkv.shape[0])
    P = int(ssm_state.shape[0])
    rc = lib().gdn_extend(
        ctypes.byref(cfg.c()), ctypes.byref(_params(params)), _ptr(mixed_qkv), _ptr(a), _ptr(b), _ptr(cu_seqlens),
        N, T, _ptr(state_indices), _ptr(has_initial_state), _ptr(conv_state), _ptr(ssm_state), P, _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(rc, "gdn_extend")


def gdn_extend_checkpoints(cfg: GdnConfig, params: dict, mixed_qkv, a, b, cu_seqlens, state_indices,
                           has_initial_state, conv_state, ssm_state, out, ckpt_token_indices, ckpt_state_slots,
                           ckpt_states, ckpt_conv, workspace, stream=None) -> None:
    """gdn_extend that also captures each sequence's state (and conv window) at one exclusive absolute
    packed-row boundary into row ckpt_state_slots[i] of ckpt_states / ckpt_conv (see include/gdn.h)."""
    N = int(state_indices.shape[0])
    T = int(mixed_qkv.shape[0])
    P = int(ssm_state.shape[0])
    rc = lib().gdn_extend_checkpoints(
        ctypes.byref(cfg.c()), ctypes.byref(_params(params)), _ptr(mixed_qkv), _ptr(a), _ptr(b), _ptr(cu_seqlens),
        N, T, _ptr(state_indices), _ptr(has_initial_state), _ptr(conv_state), _ptr(ssm_state), P, _ptr(out),
        _ptr(ckpt_token_indices), _ptr(ckpt_state_slots), _ptr(ckpt_states), _ptr(ckpt_conv),
        int(ckpt_states.shape[0]), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(rc, "gdn_extend_checkpoints")


EXTEND_STATIC_SCRATCH_BYTES = 64 << 20


def gdn_extend_static_scratch(cfg: GdnConfig, params: dict, mixed_qkv, a, b, cu_seqlens, state_indices,
                              has_initial_state, conv_state, ssm_state, out, stream=None) -> None:
    """gdn_extend for callers that cannot allocate: the scratch is the library's
    fixed 64 MiB device array (see include/gdn.h); calls must not overlap on the GPU."""
    N = int(state_indices.shape[0])
    T = int(mixed_qkv.shape[0])
    P = int(ssm_state.shape[0])
    rc = lib().gdn_extend_static_scratch(
        ctypes.byref(cfg.c()), ctypes.byref(_params(params)), _ptr(mixed_qkv), _ptr(a), _ptr(b), _ptr(cu_seqlens),
        N, T, _ptr(state_indices), _ptr(has_initial_state), _ptr(conv_state), _ptr(ssm_state), P, _ptr(out),
        _stream(stream),
    )
    _check(rc, "gdn_extend_static_scratch")


def gdn_decode(cfg: GdnConfig, params: dict, mixed_qkv, a, b, state_indices, conv_state, ssm_state, out, workspace,
               stream=None) -> None:
    B = int(state_indices.shape[0])
    P = int(ssm_state.shape[0])
    rc = lib().gdn_decode(
        ctypes.byref(cfg.c()), ctypes.byref(_params(params)), _ptr(mixed_qkv), _ptr(a), _ptr(b),
        _ptr(state_indices), B, _ptr(conv_state), _ptr(ssm_state), P, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(rc, "gdn_decode")


def gdn_verify(cfg: GdnConfig, params: dict, mixed_qkv, a, b, state_indices, D: int, conv_state, ssm_state,
               state_ckpt, conv_ckpt, out, workspace, stream=None) -> None:
    B = int(state_indices.shape[0])
    P = int(ssm_state.shape[0])
    rc = lib().gdn_verify(
        ctypes.byref(cfg.c()), ctypes.byref(_params(params)), _ptr(mixed_qkv), _ptr(a), _ptr(b),
        _ptr(state_indices), B, int(D), _ptr(conv_state), _ptr(ssm_state), P, _ptr(state_ckpt), _ptr(conv_ckpt),
        _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(rc, "gdn_verify")


def gdn_commit_workspace_size(cfg: GdnConfig, max_B: int) -> int:
    return int(lib().gdn_commit_workspace_size(ctypes.byref(cfg.c()), max_B))


def gdn_commit(cfg: GdnConfig, state_indices, accepted, D: int, state_ckpt, conv_ckpt, conv_state, ssm_state,
               workspace, stream=None) -> None:
    """Write the checkpoints of each request's last accepted draft token into its pool slot."""
    B = int(state_indices.shape[0])
    P = int(ssm_state.shape[0])
    rc = lib().gdn_commit(
        ctypes.byref(cfg.c()), _ptr(state_indices), _ptr(accepted), B, int(D), _ptr(state_ckpt), _ptr(conv_ckpt),
        _ptr(conv_state), _ptr(ssm_state), P, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream),
    )
    _check(rc, "gdn_commit")


def gdn_verify_tree(cfg: GdnConfig, params: dict, mixed_qkv, a, b, state_indices, parents, D: int, conv_state,
                    ssm_state, state_ckpt, conv_ckpt, out, workspace, stream=None) -> None:
    """gdn_verify over a draft tree: parents [B, D] int32, -1 = the slot state, else an earlier token."""
    B = int(state_indices.shape[0])
    P = int(ssm_state.shape[0])
    rc = lib().gdn_verify_tree(
        ctypes.byref(cfg.c()), ctypes.byref(_params(params)), _ptr(mixed_qkv), _ptr(a), _ptr(b),
        _ptr(state_indices), _ptr(parents), B, int(D), _ptr(conv_state), _ptr(ssm_state), P, _ptr(state_ckpt),
        _ptr(conv_ckpt), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(rc, "gdn_verify_tree")


def gdn_get_device_error(workspace, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().gdn_get_device_error(_ptr(workspace), ctypes.byref(v), _stream(stream)), "gdn_get_device_error")
    return int(v.value)


def gdn_reset_device_error(workspace, stream=None) -> None:
    _check(lib().gdn_reset_device_error(_ptr(workspace), _stream(stream)), "gdn_reset_device_error")


def gdn_check_bounded_wait(arrive: bool, limit_ns: int, workspace, stream=None) -> None:
    """Runs the kernels' bounded mbarrier wait once on the device (see include/gdn.h): on a barrier
    that completes (arrive=True) or that nothing completes (arrive=False: GDN_DEVERR_TIMEOUT after
    limit_ns nanoseconds).  Asynchronous; read the outcome with gdn_get_device_error."""
    _check(lib().gdn_check_bounded_wait(1 if arrive else 0, int(limit_ns), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream)),
           "gdn_check_bounded_wait")


def gdn_set_launch_events(events) -> None:
    """Profiling aid: record these torch.cuda.Event objects around each kernel
    the following calls launch (see include/gdn.h); [] turns it off."""
    n = len(events)
    for e in events:
        if not e.cuda_event:  # torch creates the underlying cudaEvent_t on first record
            e.record()
    arr = (ctypes.c_void_p * max(n, 1))(*[e.cuda_event for e in events])
    _check(lib().gdn_set_launch_events(arr if n else None, n), "gdn_set_launch_events")


_STATE_DTYPES = {torch.float32: GDN_DTYPE_F32, torch.bfloat16: GDN_DTYPE_BF16, torch.float16: GDN_DTYPE_F16}


@dataclass(frozen=True)
class SsdConfig:
    """Shape and options of the Mamba2 SSD scan (include/ssd.h, ssd_config_t)."""
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    state_dtype: torch.dtype = torch.bfloat16
    dt_softplus: bool = True
    d_per_dim: bool = False
    dt_limit: tuple = (0.0, float("inf"))

    def c(self) -> SsdConfigC:
        return SsdConfigC(self.nheads, self.headdim, self.dstate, self.ngroups, _STATE_DTYPES[self.state_dtype],
                          int(self.dt_softplus), int(self.d_per_dim), float(self.dt_limit[0]),
                          float(self.dt_limit[1]))


def ssd_workspace_size(cfg: SsdConfig, max_N: int, max_T: int) -> int:
    return int(lib().ssd_workspace_size(ctypes.byref(cfg.c()), max_N, max_T))


def ssd_combined_fwd(cfg: SsdConfig, x, dt, A, B, C, cu_seqlens, out, workspace, D=None, z=None, dt_bias=None,
                     initial_states=None, final_states=None, ckpt_token_indices=None, ckpt_state_slots=None,
                     ckpt_states=None, stream=None) -> None:
    """The Mamba2 SSD scan over packed sequences (include/ssd.h): out [T, H, P] and, when given,
    final_states / ckpt_states [.., H, P, N] in cfg.state_dtype."""
    N = int(cu_seqlens.shape[0]) - 1
    T = int(x.shape[0])
    num_ck = int(ckpt_states.shape[0]) if ckpt_states is not None else 0
    rc = lib().ssd_combined_fwd(
        ctypes.byref(cfg.c()), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        _ptr(cu_seqlens), N, T, _ptr(initial_states), _ptr(final_states), _ptr(ckpt_token_indices),
        _ptr(ckpt_state_slots), _ptr(ckpt_states), num_ck, _ptr(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream),
    )
    _check(rc, "ssd_combined_fwd")
