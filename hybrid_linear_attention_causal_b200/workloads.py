"""Seeded synthetic inputs for the GDN layer.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic, so both the CUDA path and the fp64 oracle can be fed from
it.  Every tensor is produced by a ``torch.Generator`` seeded per workload and
drawn in the fixed order written in each function.

Distributions (the layer description's workloads): mixed_qkv, a, b ~ N(0, 1);
A_log ~ U(0, 1.5); dt_bias ~ U(-1, 1); conv weight ~ N(0, 0.25) read as
N(mean, variance), i.e. std 0.5; random initial states ~ N(0, 0.02) (std
sqrt(0.02)); random conv states ~ N(0, 1); slow-decay workloads draw
a ~ N(-2, 1).

Pools not named by a request are filled with a sentinel bit pattern so that a
test can check, byte for byte, that the library left them alone.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class LayerSpec:
    """Shape of one GDN layer."""

    HK: int  # qk heads
    HV: int  # value heads (HV % HK == 0)
    dk: int
    dv: int
    K: int = 4  # conv width
    dtype: torch.dtype = torch.bfloat16  # mixed_qkv, a, b, out, conv weight and conv state

    @property
    def conv_dim(self) -> int:
        return 2 * self.HK * self.dk + self.HV * self.dv


@dataclass
class Workload:
    """One synthetic batch.  Tensors live on ``device``; nothing is computed here."""

    name: str
    spec: LayerSpec
    params: dict  # A_log [HV] f32, dt_bias [HV] f32, conv_w [conv_dim, K] spec.dtype, conv_b or None
    x: torch.Tensor  # [T, conv_dim] spec.dtype
    a: torch.Tensor  # [T, HV] spec.dtype
    b: torch.Tensor  # [T, HV] spec.dtype
    cu_seqlens: torch.Tensor  # [N+1] int32
    state_indices: torch.Tensor  # [N] int32
    has_initial_state: torch.Tensor | None  # [N] int32
    conv_state: torch.Tensor  # [P, conv_dim, K-1] spec.dtype
    ssm_state: torch.Tensor  # [P, HV, dk, dv] f32
    extra: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.x.shape[0])

    @property
    def N(self) -> int:
        return int(self.state_indices.shape[0])

    @property
    def P(self) -> int:
        return int(self.ssm_state.shape[0])


SENTINEL_F32 = 0x7F7F_5A5A  # a finite float32 bit pattern (about 3.4e38 with a marked mantissa)
SENTINEL_16 = 0x5A5A  # a finite 16-bit pattern for bf16 / fp16 pools


def sentinel_fill_(t: torch.Tensor) -> torch.Tensor:
    """Fill ``t`` in place with the sentinel bit pattern of its dtype."""
    if t.dtype == torch.float32:
        t.view(torch.int32).fill_(SENTINEL_F32)
    elif t.element_size() == 2:
        t.view(torch.int16).fill_(SENTINEL_16)
    else:
        raise TypeError(f"no sentinel for {t.dtype}")
    return t


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_params(spec: LayerSpec, gen: torch.Generator, device) -> dict:
    """Per-layer parameters, drawn in the order A_log, dt_bias, conv weight."""
    A_log = torch.rand(spec.HV, generator=gen, device=device, dtype=torch.float32) * 1.5
    dt_bias = torch.rand(spec.HV, generator=gen, device=device, dtype=torch.float32) * 2.0 - 1.0
    conv_w = (torch.randn(spec.conv_dim, spec.K, generator=gen, device=device, dtype=torch.float32) * 0.5).to(
        spec.dtype
    )
    return {"A_log": A_log, "dt_bias": dt_bias, "conv_w": conv_w, "conv_b": None}


def make_tokens(spec: LayerSpec, T: int, gen: torch.Generator, device, a_mean: float = 0.0):
    """mixed_qkv [T, conv_dim], a [T, HV], b [T, HV], drawn in that order."""
    x = torch.randn(T, spec.conv_dim, generator=gen, device=device, dtype=torch.float32).to(spec.dtype)
    a = (torch.randn(T, spec.HV, generator=gen, device=device, dtype=torch.float32) + a_mean).to(spec.dtype)
    b = torch.randn(T, spec.HV, generator=gen, device=device, dtype=torch.float32).to(spec.dtype)
    return x, a, b


def make_pools(spec: LayerSpec, P: int, device):
    """Sentinel-filled conv and ssm pools."""
    conv_state = sentinel_fill_(torch.empty(P, spec.conv_dim, spec.K - 1, dtype=spec.dtype, device=device))
    ssm_state = sentinel_fill_(torch.empty(P, spec.HV, spec.dk, spec.dv, dtype=torch.float32, device=device))
    return conv_state, ssm_state


def fill_slots_random_(spec: LayerSpec, conv_state, ssm_state, slots, gen, device, ssm_var=0.02, conv_var=1.0):
    """Random initial contents for the named slots: ssm ~ N(0, ssm_var), conv ~ N(0, conv_var)."""
    slots = [int(s) for s in slots]
    n = len(slots)
    s = torch.randn(n, spec.HV, spec.dk, spec.dv, generator=gen, device=device, dtype=torch.float32)
    c = torch.randn(n, spec.conv_dim, spec.K - 1, generator=gen, device=device, dtype=torch.float32)
    idx = torch.tensor(slots, device=device, dtype=torch.long)
    ssm_state[idx] = s * math.sqrt(ssm_var)
    conv_state[idx] = (c * math.sqrt(conv_var)).to(conv_state.dtype)


def cu_from_lengths(lengths, device) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def loguniform_lengths(n: int, lo: int, hi: int, total: int, gen: torch.Generator) -> list[int]:
    """n lengths log-uniform in [lo, hi], rescaled and rounded so that they sum to
    ``total``; the last one absorbs the rounding remainder and every length is
    clamped to [lo, hi] (remainders that clamping leaves are spread over the others)."""
    u = torch.rand(n, generator=gen, device=gen.device, dtype=torch.float64).cpu()
    raw = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    scaled = raw * (total / float(raw.sum()))
    lens = [min(hi, max(lo, int(round(float(v))))) for v in scaled[:-1]]
    last = total - sum(lens)
    lens.append(last)
    # spread any excess so that every length stays inside [lo, hi]
    i = 0
    while not (lo <= lens[-1] <= hi) and i < 10 * n:
        j = i % (n - 1)
        if lens[-1] > hi and lens[j] < hi:
            d = min(hi - lens[j], lens[-1] - hi)
            lens[j] += d
            lens[-1] -= d
        elif lens[-1] < lo and lens[j] > lo:
            d = min(lens[j] - lo, lo - lens[-1])
            lens[j] -= d
            lens[-1] += d
        i += 1
    assert sum(lens) == total
    return lens


# ---------------------------------------------------------------------------
# the five workloads of the layer description
# ---------------------------------------------------------------------------

SPEC_TINY = LayerSpec(HK=2, HV=2, dk=64, dv=64, dtype=torch.float32)
SPEC_RAGGED = LayerSpec(HK=4, HV=8, dk=64, dv=64, dtype=torch.bfloat16)
SPEC_LARGE = LayerSpec(HK=16, HV=32, dk=128, dv=128, dtype=torch.bfloat16)


def tiny_fp32(device="cpu", seed: int = 0) -> Workload:
    """Tiny layer, fp32: one sequence of 64 tokens then 8 single-token decode steps,
    2/2 heads, dk = dv = 64, zero initial state, pool of 8 slots with the request
    at slot 3.  extra['decode'] holds the 8 decode tokens as (x, a, b) rows."""
    spec = SPEC_TINY
    g = _gen(seed, device)
    params = make_params(spec, g, device)
    x, a, b = make_tokens(spec, 64, g, device)
    xd, ad, bd = make_tokens(spec, 8, g, device)
    conv_state, ssm_state = make_pools(spec, 8, device)
    return Workload(
        "tiny_fp32_T64_decode8", spec, params, x, a, b, cu_from_lengths([64], device),
        torch.tensor([3], dtype=torch.int32, device=device), torch.tensor([0], dtype=torch.int32, device=device),
        conv_state, ssm_state, extra={"decode": (xd, ad, bd)},
    )


def ragged_varlen(device="cpu", seed: int = 1) -> Workload:
    """Ragged EXTEND, bf16 in / fp32 state: 6 requests, cached prefix lengths
    ~U{0..300}, extend lengths ~U{1..200}, slots = first 6 of a random permutation
    of a 64-slot pool, 4/8 heads, dk = dv = 64.

    The prefix rows are drawn too (extra['prefix'] = (x, a, b, cu_seqlens)) so that
    a caller can build each slot's state by running the layer over its prefix from
    zero; x/a/b/cu_seqlens here are the extend part only.  has_initial_state is 1
    where the prefix is non-empty."""
    spec = SPEC_RAGGED
    g = _gen(seed, device)
    params = make_params(spec, g, device)
    prefix = torch.randint(0, 301, (6,), generator=g, device=device).tolist()
    ext = torch.randint(1, 201, (6,), generator=g, device=device).tolist()
    perm = torch.randperm(64, generator=g, device=device)[:6].to(torch.int32)
    xp, ap, bp = make_tokens(spec, sum(prefix), g, device)
    x, a, b = make_tokens(spec, sum(ext), g, device)
    conv_state, ssm_state = make_pools(spec, 64, device)
    has_init = torch.tensor([1 if p > 0 else 0 for p in prefix], dtype=torch.int32, device=device)
    return Workload(
        "ragged_varlen_6req", spec, params, x, a, b, cu_from_lengths(ext, device), perm, has_init, conv_state,
        ssm_state, extra={"prefix": (xp, ap, bp, cu_from_lengths(prefix, device)), "prefix_lens": prefix,
                          "extend_lens": ext},
    )


def large_prefill(device="cpu", seed: int = 2, total: int = 32768, nseq: int = 8) -> Workload:
    """Large packed prefill, bf16: 16/32 heads, dk = dv = 128, 8 sequences with
    lengths log-uniform in [512, 16384] summing to 32768, zero initial states
    (has_initial_state = 0), slots = first 8 of a random permutation of a
    16-slot pool."""
    spec = SPEC_LARGE
    g = _gen(seed, device)
    params = make_params(spec, g, device)
    lens = loguniform_lengths(nseq, 512, 16384, total, g)
    P = 2 * nseq
    perm = torch.randperm(P, generator=g, device=device)[:nseq].to(torch.int32)
    x, a, b = make_tokens(spec, total, g, device)
    conv_state, ssm_state = make_pools(spec, P, device)
    return Workload(
        f"large_prefill_{nseq}seq_{total}tok", spec, params, x, a, b, cu_from_lengths(lens, device), perm,
        torch.zeros(nseq, dtype=torch.int32, device=device), conv_state, ssm_state, extra={"lens": lens},
    )


def decode_verify(device="cpu", seed: int = 3, B: int = 256, P: int = 1024, D: int = 4) -> Workload:
    """Batched DECODE + speculative verify, bf16 in / fp32 state: pool of P=1024
    slots [1024, 32, 128, 128], B=256 requests at the first 256 slots of a random
    permutation, one token each; the named slots hold ssm ~ N(0, 0.02) and conv
    ~ N(0, 1).  extra['verify'] holds (x, a, b) for D=4 draft tokens per request
    (rows i*D .. i*D+D-1 belong to request i)."""
    spec = SPEC_LARGE
    g = _gen(seed, device)
    params = make_params(spec, g, device)
    perm = torch.randperm(P, generator=g, device=device)[:B].to(torch.int32)
    conv_state, ssm_state = make_pools(spec, P, device)
    fill_slots_random_(spec, conv_state, ssm_state, perm.tolist(), g, device)
    x, a, b = make_tokens(spec, B, g, device)
    xv, av, bv = make_tokens(spec, B * D, g, device)
    return Workload(
        f"decode_{B}req_pool{P}", spec, params, x, a, b, cu_from_lengths([1] * B, device), perm, None, conv_state,
        ssm_state, extra={"verify": (xv, av, bv), "D": D},
    )


def long_prefill(device="cpu", seed: int = 4, T: int = 262144) -> Workload:
    """Long-context prefill, bf16: one sequence of 262144 tokens continuing from a
    random state ~N(0, 0.02) and a random conv state, 16/32 heads, dk = dv = 128,
    a ~ N(-2, 1) (slow decay), b ~ N(0, 1).  Pool of 4 slots, request at slot 1."""
    spec = SPEC_LARGE
    g = _gen(seed, device)
    params = make_params(spec, g, device)
    conv_state, ssm_state = make_pools(spec, 4, device)
    fill_slots_random_(spec, conv_state, ssm_state, [1], g, device)
    x, a, b = make_tokens(spec, T, g, device, a_mean=-2.0)
    return Workload(
        f"long_prefill_1seq_{T}tok", spec, params, x, a, b, cu_from_lengths([T], device),
        torch.tensor([1], dtype=torch.int32, device=device), torch.ones(1, dtype=torch.int32, device=device),
        conv_state, ssm_state,
    )


def random_case(spec: LayerSpec, lengths, P: int, seed: int, device="cpu", init_random: bool = True,
                a_mean: float = 0.0, has_init=None, slots=None) -> Workload:
    """A small seeded case of any shape for edge-case tests.  Slots default to
    the first len(lengths) entries of a random permutation of P; a negative slot
    in ``slots`` marks a padded request."""
    g = _gen(seed, device)
    params = make_params(spec, g, device)
    N = len(lengths)
    if slots is None:
        slots = torch.randperm(P, generator=g, device=device)[:N].to(torch.int32)
    else:
        slots = torch.tensor(list(slots), dtype=torch.int32, device=device)
    conv_state, ssm_state = make_pools(spec, P, device)
    live = [int(s) for s in slots.tolist() if 0 <= s < P]
    if init_random and live:
        fill_slots_random_(spec, conv_state, ssm_state, live, g, device)
    x, a, b = make_tokens(spec, sum(int(n) for n in lengths), g, device, a_mean=a_mean)
    hi = None if has_init is None else torch.tensor(list(has_init), dtype=torch.int32, device=device)
    return Workload(
        f"case_{spec.HK}x{spec.HV}_d{spec.dk}x{spec.dv}_{'_'.join(map(str, lengths))}", spec, params, x, a, b,
        cu_from_lengths(lengths, device), slots, hi, conv_state, ssm_state,
    )


# ---------------------------------------------------------------------------
# Mamba2 SSD chunk-scan workloads
# ---------------------------------------------------------------------------
#
# x, z, B, C and the raw steps dt ~ N(0, 1) in bf16; A = -U(a_lo, a_hi) (fp32;
# the Mamba2 initialisation draws -A from U(1, 16)); dt_bias ~ U(-4, -1) (fp32),
# so that softplus(dt + dt_bias) lies mostly in (0.005, 1); D ~ N(0, 1) in bf16
# per head (or per head and dim); random initial states ~ N(0, 0.02) in the
# state dtype.


@dataclass(frozen=True)
class SsdSpec:
    """Shape of one Mamba2 SSD layer."""

    H: int  # heads
    P: int  # head dim
    N: int  # state dim
    G: int  # groups of B / C
    state_dtype: torch.dtype = torch.bfloat16


@dataclass
class SsdWorkload:
    name: str
    spec: SsdSpec
    x: torch.Tensor       # [T, H, P] bf16
    dt: torch.Tensor      # [T, H] bf16
    A: torch.Tensor       # [H] fp32
    B: torch.Tensor       # [T, G, N] bf16
    C: torch.Tensor       # [T, G, N] bf16
    D: torch.Tensor | None
    z: torch.Tensor | None
    dt_bias: torch.Tensor | None
    cu: torch.Tensor      # [Nseq + 1] int32
    init: torch.Tensor | None  # [Nseq, H, P, N] state dtype
    lengths: list = field(default_factory=list)

    @property
    def T(self) -> int:
        return int(self.x.shape[0])

    def to(self, device) -> "SsdWorkload":
        mv = lambda t: None if t is None else t.to(device)
        return SsdWorkload(self.name, self.spec, mv(self.x), mv(self.dt), mv(self.A), mv(self.B), mv(self.C),
                           mv(self.D), mv(self.z), mv(self.dt_bias), mv(self.cu), mv(self.init), list(self.lengths))


def ssd_case(spec: SsdSpec, lengths, seed: int, device="cpu", with_D: bool = True, d_per_dim: bool = False,
             with_z: bool = True, with_bias: bool = True, init_random: bool = True, a_range=(1.0, 16.0)) -> SsdWorkload:
    """A seeded SSD case; tensors drawn in the order x, z, B, C, dt, A, dt_bias, D, init."""
    g = _gen(seed, device)
    T, H, P, N, G = sum(int(n) for n in lengths), spec.H, spec.P, spec.N, spec.G
    bf = torch.bfloat16
    x = torch.randn(T, H, P, generator=g, device=device).to(bf)
    z = torch.randn(T, H, P, generator=g, device=device).to(bf)
    B = torch.randn(T, G, N, generator=g, device=device).to(bf)
    C = torch.randn(T, G, N, generator=g, device=device).to(bf)
    dt = torch.randn(T, H, generator=g, device=device).to(bf)
    A = -(a_range[0] + (a_range[1] - a_range[0]) * torch.rand(H, generator=g, device=device))
    dt_bias = -4.0 + 3.0 * torch.rand(H, generator=g, device=device)
    D = torch.randn((H, P) if d_per_dim else (H,), generator=g, device=device).to(bf)
    init = (math.sqrt(0.02) * torch.randn(len(lengths), H, P, N, generator=g, device=device)).to(spec.state_dtype)
    return SsdWorkload(
        f"ssd_{H}h_p{P}_n{N}_g{G}_{'_'.join(map(str, lengths))}", spec, x, dt, A.float(), B, C,
        D if with_D else None, z if with_z else None, dt_bias.float() if with_bias else None,
        cu_from_lengths(lengths, device), init if init_random else None, list(lengths),
    )


SPEC_SSD = SsdSpec(H=128, P=64, N=128, G=8)


def ssd_prefill(device="cpu", seed: int = 5, total: int = 32768, nseq: int = 8) -> SsdWorkload:
    """The SSD bench workload: a Mamba2 layer of 128 heads (head dim 64, state 128, 8 groups) over
    nseq packed sequences with lengths log-uniform in [512, 16384] summing to ``total`` (the same
    length recipe as the large GDN prefill), bf16 states continuing from random initial states."""
    g = _gen(seed, device)
    lens = loguniform_lengths(nseq, 512, 16384, total, g)
    w = ssd_case(SPEC_SSD, lens, seed + 1000, device=device)
    w.name = f"ssd_prefill_{nseq}seq_{total}tok"
    return w
