"""fp64 CPU oracle for the Mamba2 SSD chunk-scan layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` and the CPU-baseline leg of ``bench.py`` import this module.
The product package never imports it and shares no code with it.  The
arithmetic lives in ``ssd_oracle.c`` (plain C, fp64, OpenMP over (sequence,
head)); this file builds that library with gcc and marshals numpy arrays.

Every floating-point input is decoded to float64 exactly (bf16, fp16 and fp32
values are exactly representable), so the oracle sees the values the GPU path
reads.  Outputs are float64 and never rounded here.  See ``ssd_oracle.c`` for
what is computed and which page it follows.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

from .oracle import _f64, _i32, _p, _dbl_p, _i32_p

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32),
        ("P", ctypes.c_int32),
        ("N", ctypes.c_int32),
        ("G", ctypes.c_int32),
        ("dt_softplus", ctypes.c_int32),
        ("dt_lo", ctypes.c_double),
        ("dt_hi", ctypes.c_double),
        ("d_per_dim", ctypes.c_int32),
    ]


@dataclass(frozen=True)
class SsdCfg:
    H: int      # heads
    P: int      # head dim
    N: int      # state dim
    G: int      # groups of B / C
    dt_softplus: bool = True
    dt_limit: tuple = (0.0, math.inf)
    d_per_dim: bool = False

    def _c(self) -> _Cfg:
        return _Cfg(self.H, self.P, self.N, self.G, int(self.dt_softplus), float(self.dt_limit[0]),
                    float(self.dt_limit[1]), int(self.d_per_dim))


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c into libssd_oracle.so next to it (gcc, -O3, OpenMP).

    SSD_ORACLE_LIB, when set, names an already built library to load instead
    (the mutation tests load deliberately broken copies through it)."""
    override = os.environ.get("SSD_ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-march=native", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.ssd_dt.restype = ctypes.c_double
        lib.ssd_dt.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_double, ctypes.c_double]
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_L().ssd_num_threads())


def step_size(cfg: SsdCfg, dt: float, bias: float = 0.0) -> float:
    """The processed step of one (token, head): clamp(softplus?(dt + bias), lo, hi)."""
    c = cfg._c()
    return float(_L().ssd_dt(ctypes.byref(c), float(dt), float(bias)))


def _args(cfg, x, dt, A, B, C, D, z, dt_bias, cu_seqlens, init):
    x, dt, A, B, C = (_f64(t) for t in (x, dt, A, B, C))
    D, z, dt_bias, init = (_f64(t) for t in (D, z, dt_bias, init))
    cu = _i32(cu_seqlens)
    T, Nseq = x.shape[0], cu.shape[0] - 1
    assert x.shape == (T, cfg.H, cfg.P) and dt.shape == (T, cfg.H) and A.shape == (cfg.H,)
    assert B.shape == (T, cfg.G, cfg.N) and C.shape == B.shape
    if z is not None:
        assert z.shape == x.shape
    if init is not None:
        assert init.shape == (Nseq, cfg.H, cfg.P, cfg.N)
    return x, dt, A, B, C, D, z, dt_bias, cu, init, T, Nseq


def scan(cfg: SsdCfg, x, dt, A, B, C, cu_seqlens, D=None, z=None, dt_bias=None, init=None,
         ck_idx=None, ck_row=None, num_ck: int = 0, return_rc: bool = False):
    """Token-by-token scan.  Returns (y [T,H,P], final [Nseq,H,P,N], ck [num_ck,H,P,N] or None)."""
    x, dt, A, B, C, D, z, dt_bias, cu, init, T, Nseq = _args(cfg, x, dt, A, B, C, D, z, dt_bias, cu_seqlens, init)
    y = np.zeros((T, cfg.H, cfg.P))
    fin = np.zeros((Nseq, cfg.H, cfg.P, cfg.N))
    ci, cr = _i32(ck_idx), _i32(ck_row)
    ck = np.zeros((max(num_ck, 1), cfg.H, cfg.P, cfg.N)) if ci is not None else None
    c = cfg._c()
    rc = _L().ssd_scan(ctypes.byref(c), T, Nseq, _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D), _p(z), _p(dt_bias),
                       _p(cu, _i32_p), _p(init), _p(y), _p(fin), _p(ci, _i32_p), _p(cr, _i32_p), int(num_ck),
                       _p(ck))
    out = (y, fin, ck[:num_ck] if ck is not None else None)
    return out + (rc,) if return_rc else out


def scan_chunked(cfg: SsdCfg, x, dt, A, B, C, cu_seqlens, chunk: int, D=None, z=None, dt_bias=None, init=None):
    """The chunked form with chunks of `chunk` rows.  Returns (y, final)."""
    x, dt, A, B, C, D, z, dt_bias, cu, init, T, Nseq = _args(cfg, x, dt, A, B, C, D, z, dt_bias, cu_seqlens, init)
    y = np.zeros((T, cfg.H, cfg.P))
    fin = np.zeros((Nseq, cfg.H, cfg.P, cfg.N))
    c = cfg._c()
    rc = _L().ssd_scan_chunked(ctypes.byref(c), T, Nseq, int(chunk), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D),
                               _p(z), _p(dt_bias), _p(cu, _i32_p), _p(init), _p(y), _p(fin))
    assert rc == 0
    return y, fin
