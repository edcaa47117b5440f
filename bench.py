#!/usr/bin/env python
"""Benchmark of the GDN layer on B200: one step = one gdn_extend over the
prefill workload + one gdn_decode over the decode batch + one gdn_verify over
the verify batch + one gdn_commit of each verify request's accepted prefix
(every mode of the layer), on synthetic inputs already resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill262k|prefill32k]
    python bench.py --impl reference ...      # the fp64 CPU oracle on a bounded sample

The default prefill workload is the long-context one (one sequence of 262144
tokens continuing from a random state, 16/32 heads, d = 128): the largest
configuration that fits one GPU.  The 32768-token packed batch (8 sequences)
is timed beside it.  Prints one JSON line (rank 0).  `value` is prefill
tokens/s over all ranks, from the device time of the gdn_extend launches
inside the timed steps; decode, verify and commit report their own
state-traffic figures.  Multi-GPU runs are independent replicas (weak
scaling): every rank runs its own batch, no collective touches the data path;
the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "GDN prefill tokens/s + decode state GB/s (frac. of roofline), 1×B200"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# The prefill's tensor-core products are kind::f16 MMAs (fp16 operands, fp32 accumulation): their
# peak is the dense fp16 rate, which equals the bf16 rate the peaks file measures.
C = 64


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=["prefill262k", "prefill32k"], default="prefill262k")
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--e2e-piece", type=int, default=16384, help="rows per call of the end-to-end pipeline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-ssd", action="store_true", help="skip the Mamba2 SSD scan timing")
    p.add_argument("--no-side", action="store_true", help="skip the prefill timings outside the step")
    p.add_argument("--cpu-sample-tokens", type=int, default=16384)
    p.add_argument("--ref-sample-tokens", type=int, default=4096)
    p.add_argument("--profile", choices=["extend", "decode", "verify", "ssd"], default=None,
                   help="run only this call on a reduced case (an ncu target); prints timings, not the bench line")
    p.add_argument("--profile-tokens", type=int, default=8192, help="prefill rows of the --profile extend case")
    p.add_argument("--profile-seqs", type=int, default=4, help="sequences of the --profile extend case")
    p.add_argument("--profile-requests", type=int, default=64, help="requests of the --profile decode/verify case")
    return p.parse_args()


# ------------------------------------------------------------------ plumbing


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    try:
        d = json.load(open(PEAKS_FILE))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def source_digest(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    if there is none or the kernel's source changed since it was taken."""
    try:
        d = json.load(open(TRAFFIC_FILE))[kernel]
    except Exception:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src) or source_digest(src) != d["source_sha256_16"]:
        return None
    return float(d["bytes_per_launch"]) * float(d.get("scale_to_bench", 1.0))


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        self.file.flush()
        rows = []
        for line in open(self.file.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        smax = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.5 * smax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ algorithmic work


def prefill_work(spec, T):
    """Algorithmic FLOPs and bytes of one prefill of T tokens (per value head and
    chunk of C rows: intra 4C^2 d / G (q.k, k.k shared by the G value heads)
    + 4C^2 d (W, U) + C^3/3 (triangular solve); state pass 6 C d^2 (W S, q^T S,
    K^T V') + 2 C^2 d (decayed q.k times V'))."""
    d, G, HV = spec.dk, spec.HV // spec.HK, spec.HV
    per_chunk_intra = 4 * C * C * d / G + 4 * C * C * d + C ** 3 / 3
    per_chunk_state = 6 * C * d * d + 2 * C * C * d
    chunks = T / C
    flops_intra = per_chunk_intra * chunks * HV
    flops_state = per_chunk_state * chunks * HV
    es = 2 if spec.dtype == torch.bfloat16 else 4
    bytes_tok = spec.conv_dim * es + 2 * HV * es + HV * spec.dv * es
    return {"flops_intra": flops_intra, "flops_state": flops_state, "flops": flops_intra + flops_state,
            "bytes": bytes_tok * T, "bytes_per_token": bytes_tok}


def decode_bytes(spec, B):
    es = 2 if spec.dtype == torch.bfloat16 else 4
    state = 2 * spec.HV * spec.dk * spec.dv * 4 * B
    conv = 2 * spec.conv_dim * 3 * es * B
    io = (spec.conv_dim + 2 * spec.HV + spec.HV * spec.dv) * es * B
    return state, state + conv + io


def commit_bytes(spec, accepted):
    """Bytes one commit moves: for every request with a >= 1 accepted tokens, its checkpoint
    (every head's fp32 state and the conv window) read and written into the slot."""
    es = 2 if spec.dtype == torch.bfloat16 else 4
    n = int((accepted > 0).sum())
    state = 2 * spec.HV * spec.dk * spec.dv * 4 * n
    return state, state + 2 * spec.conv_dim * 3 * es * n


def verify_bytes(spec, B, D):
    es = 2 if spec.dtype == torch.bfloat16 else 4
    state = (1 + D) * spec.HV * spec.dk * spec.dv * 4 * B
    conv = (1 + D) * spec.conv_dim * 3 * es * B
    io = (spec.conv_dim + 2 * spec.HV + spec.HV * spec.dv) * es * B * D
    return state, state + conv + io


# ------------------------------------------------------------------ reference arm


def oracle_sample(pre, ntok):
    """The first `ntok` packed rows of the prefill batch (whole sequences, then
    a cut of the next one), all heads, from the batch's initial slot contents."""
    from oracle import oracle as O

    spec = pre.spec
    cu = pre.cu_seqlens.cpu().tolist()
    n = min(ntok, cu[-1])
    lens = []
    for i in range(len(cu) - 1):
        take = min(cu[i + 1], n) - cu[i]
        if take <= 0:
            break
        lens.append(take)
    N = len(lens)
    cfg = O.OracleCfg(HK=spec.HK, HV=spec.HV, dk=spec.dk, dv=spec.dv)
    slots = pre.state_indices[:N].cpu()
    cs = pre.conv_state.cpu()
    ss = pre.ssm_state.cpu()
    cu_s = torch.tensor([0] + [sum(lens[:i + 1]) for i in range(N)], dtype=torch.int32)
    args = (cfg, {k: (None if v is None else v.cpu()) for k, v in pre.params.items()}, pre.x[:n].cpu(),
            pre.a[:n].cpu(), pre.b[:n].cpu(), cu_s, slots, cs, ss)
    hi = None if pre.has_initial_state is None else pre.has_initial_state[:N].cpu()

    def run():
        O.extend(*args, has_initial_state=hi)

    workers = min(O.num_threads(), N * spec.HV)
    return run, n, workers


def ssd_oracle_sample(w, nrows):
    """The fp64 SSD oracle on the first `nrows` packed rows of SSD workload w (the leading sequences,
    the last one cut), all heads.  Returns (run, rows, workers)."""
    from oracle import ssd as OS

    s = w.spec
    lens, n = [], 0
    for L in w.lengths:
        take = min(int(L), nrows - n)
        if take <= 0:
            break
        lens.append(take)
        n += take
    cu = torch.tensor([0] + [sum(lens[:i + 1]) for i in range(len(lens))], dtype=torch.int32)
    cpu = lambda t: None if t is None else t[:n].cpu() if t.dim() >= 2 and t.shape[0] == w.T else t.cpu()
    cfg = OS.SsdCfg(H=s.H, P=s.P, N=s.N, G=s.G)
    init = None if w.init is None else w.init[:len(lens)].cpu()
    args = (cfg, cpu(w.x), cpu(w.dt), w.A.cpu(), cpu(w.B), cpu(w.C), cu)
    kw = dict(D=None if w.D is None else w.D.cpu(), z=cpu(w.z), dt_bias=None if w.dt_bias is None else w.dt_bias.cpu(),
              init=init)

    def run():
        OS.scan(*args, **kw)

    return run, n, min(OS.num_threads(), len(lens) * s.H)


def run_reference(args, rank, world):
    if rank != 0:
        return
    from hybrid_linear_attention_causal_b200 import workloads as W

    pre = W.large_prefill(device="cpu") if args.workload == "prefill32k" else W.long_prefill(device="cpu", T=8192)
    run, n, workers = oracle_sample(pre, args.ref_sample_tokens)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    val = n / dt
    sample = f"first {n} packed rows of the {pre.name} batch, all {pre.spec.HV} value heads, per step"
    ssd = None
    if not args.no_ssd:  # the SSD scan's oracle on a bounded sample of its workload, timed once
        sw = W.ssd_prefill(device="cpu")
        srun, sn, sworkers = ssd_oracle_sample(sw, args.ref_sample_tokens // 4)
        srun()
        t1 = time.perf_counter()
        srun()
        sdt = time.perf_counter() - t1
        ssd = {"value": sn / sdt, "unit": "rows/s", "cores": sworkers, "kind": "oracle", "workload": sw.name,
               "sample": f"first {sn} packed rows of the {sw.name} batch, all {sw.spec.H} heads"}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(pre, args),
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": workers, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "ssd": ssd,
    }), flush=True)


def workload_config(pre, args):
    s = pre.spec
    return {"workload": pre.name, "prefill_tokens": pre.T, "prefill_seqs": pre.N,
            "heads_qk_v": [s.HK, s.HV], "dk_dv": [s.dk, s.dv], "chunk": C, "io_dtype": str(s.dtype).split(".")[-1],
            "decode_requests": 256, "decode_pool_slots": 1024, "verify_draft_tokens": 4,
            "l2": "inputs larger than L2 (prefill input 512 MiB+, decode state 1 GiB touched per step)"}


# gdn_extend's profiling marks (gdn_set_launch_events): 0 start, 1 chunk table, 2 after the last
# per-chunk segment, 3 conv-state update, 5 end; on the library's second stream 6 / 7 bracket the
# state-pass segments, which run alongside the per-chunk segments after the first
EXT_EV = 8
EXT_K = ["chunk_map", "chunk", "conv_tail", "state"]


def extend_kernel_ms(ev):
    sp = lambda i, j: ev[i].elapsed_time(ev[j])
    return {"chunk_map": sp(0, 1), "chunk": sp(1, 2), "conv_tail": sp(2, 3), "state": sp(6, 7), "extend": sp(0, 5)}


def prefill_kernel_roofline(spec, T, chunks, kms, hbm, f16):
    """Per-kernel rooflines of one extend: the per-chunk step against the larger of its input read
    (the bf16 rows and gates: the algorithmic bytes it must move) at the HBM peak and the intra-chunk
    FLOPs at the tensor peak; the state pass against its FLOPs (the chain products and outputs)
    at the tensor peak."""
    pw = prefill_work(spec, T)
    es = 2 if spec.dtype == torch.bfloat16 else 4
    in_bytes = T * (spec.conv_dim + 2 * spec.HV) * es
    out = {}
    t_in, t_fi = in_bytes / (hbm * 1e9), pw["flops_intra"] / (f16 * 1e12)
    if t_in >= t_fi:
        out["chunk"] = {"bound": "hbm", "work": in_bytes, "unit": "GB/s", "peak": hbm}
    else:
        out["chunk"] = {"bound": "tensor", "work": pw["flops_intra"], "unit": "TFLOP/s", "peak": f16}
    out["state"] = {"bound": "tensor", "work": pw["flops_state"], "unit": "TFLOP/s", "peak": f16}
    for name, k in out.items():
        t = kms[name] * 1e-3
        scale = 1e12 if k["unit"] == "TFLOP/s" else 1e9
        k["ms"] = kms[name]
        k["achieved"] = k["work"] / t / scale
        k["frac"] = k["achieved"] / k["peak"]
    return out, pw


def prefill_summary(spec, T, chunks, ms, kms, hbm, f16, world):
    pw = prefill_work(spec, T)
    t_floor = max(pw["flops"] / (f16 * 1e12), pw["bytes"] / (hbm * 1e9))
    return {"ms": ms, "tokens_per_s": world * T / (ms * 1e-3), "chunks": chunks,
            "tflops": pw["flops"] / (ms * 1e-3) / 1e12, "gbs_algorithmic": pw["bytes"] / (ms * 1e-3) / 1e9,
            "roofline": {"floor_ms": t_floor * 1e3,
                         "bound": "tensor" if pw["flops"] / (f16 * 1e12) >= pw["bytes"] / (hbm * 1e9) else "hbm",
                         "frac": t_floor / (ms * 1e-3), "tensor_frac": pw["flops"] / (ms * 1e-3) / (f16 * 1e12),
                         "hbm_frac": pw["bytes"] / (ms * 1e-3) / (hbm * 1e9)},
            "kernel_ms": {k: kms[k] for k in EXT_K}}


# ------------------------------------------------------------------ our arm


def ssd_work(w):
    """Algorithmic bytes and FLOPs of one Mamba2 SSD scan over workload w (chunks of C rows).
    Bytes: x, z, out (H P bf16 each), B and C (G N bf16 each) and dt (H bf16) per row, plus the
    initial and final states once per sequence.  FLOPs per row and head: the group's C B^T shared
    by its H / G heads (2 C N / (H / G)), the intra product Lm X (2 C P), and the state's read-out
    C h^T and update B^T Xw (2 N P each)."""
    s = w.spec
    T, H, P, N, G = w.T, s.H, s.P, s.N, s.G
    esz = torch.tensor([], dtype=s.state_dtype).element_size()
    nseq = len(w.lengths)
    byts = T * (3 * H * P * 2 + 2 * G * N * 2 + H * 2) + 2 * nseq * H * P * N * esz
    flops = T * H * (2 * C * N / (H // G) + 2 * C * P + 4 * N * P)
    return byts, flops


def ssd_call(w, gdn, dev):
    s = w.spec
    cfg = gdn.SsdConfig(nheads=s.H, headdim=s.P, dstate=s.N, ngroups=s.G, state_dtype=s.state_dtype)
    ws = gdn.alloc_workspace(gdn.ssd_workspace_size(cfg, len(w.lengths), w.T), dev)
    out = torch.empty((w.T, s.H, s.P), dtype=torch.bfloat16, device=dev)
    fin = torch.empty((len(w.lengths), s.H, s.P, s.N), dtype=s.state_dtype, device=dev)
    call = lambda: gdn.ssd_combined_fwd(cfg, w.x, w.dt, w.A, w.B, w.C, w.cu, out, ws, D=w.D, z=w.z,
                                        dt_bias=w.dt_bias, initial_states=w.init, final_states=fin)
    return call, ws


def run_profile_case(args, dev):
    """A reduced case of one call, for ncu captures: `--profile extend` runs the
    prefill layer (16/32 heads, d=128) on --profile-tokens rows in 4 sequences;
    decode/verify run --profile-requests requests on a pool of twice as many
    slots.  Inputs stay larger than L2 for the default sizes."""
    import hybrid_linear_attention_causal_b200 as gdn
    from hybrid_linear_attention_causal_b200 import workloads as W

    if args.profile == "ssd":
        w = W.ssd_prefill(device=dev, total=args.profile_tokens, nseq=4)
        call, ws = ssd_call(w, gdn, dev)
        w.cu_seqlens, w.N = w.cu, len(w.lengths)
    elif args.profile == "extend":
        w = W.large_prefill(device=dev, total=args.profile_tokens, nseq=args.profile_seqs)
        cfg = gdn.GdnConfig.from_spec(w.spec)
        ws = gdn.alloc_workspace(gdn.gdn_extend_workspace_size(cfg, w.N, w.T), dev)
        out = torch.empty(w.T, w.spec.HV, w.spec.dv, dtype=w.spec.dtype, device=dev)
        call = lambda: gdn.gdn_extend(cfg, w.params, w.x, w.a, w.b, w.cu_seqlens, w.state_indices,
                                      w.has_initial_state, w.conv_state, w.ssm_state, out, ws)
    else:
        Bn = args.profile_requests
        w = W.decode_verify(device=dev, B=Bn, P=2 * Bn)
        cfg = gdn.GdnConfig.from_spec(w.spec)
        if args.profile == "decode":
            ws = gdn.alloc_workspace(gdn.gdn_decode_workspace_size(cfg, Bn), dev)
            out = torch.empty(Bn, w.spec.HV, w.spec.dv, dtype=w.spec.dtype, device=dev)
            call = lambda: gdn.gdn_decode(cfg, w.params, w.x, w.a, w.b, w.state_indices, w.conv_state,
                                          w.ssm_state, out, ws)
        else:
            D = w.extra["D"]
            xv, av, bv = w.extra["verify"]
            ws = gdn.alloc_workspace(gdn.gdn_verify_workspace_size(cfg, Bn, D), dev)
            out = torch.empty(Bn * D, w.spec.HV, w.spec.dv, dtype=w.spec.dtype, device=dev)
            ck = torch.empty(Bn, D, w.spec.HV, w.spec.dk, w.spec.dv, device=dev)
            call = lambda: gdn.gdn_verify(cfg, w.params, xv, av, bv, w.state_indices, D, w.conv_state,
                                          w.ssm_state, ck, None, out, ws)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(args.steps):
        call()
    s1.record()
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_error(ws) == 0
    cu = w.cu_seqlens.cpu().tolist() if args.profile in ("extend", "ssd") else list(range(w.N + 1))
    chunks = sum((cu[i + 1] - cu[i] + C - 1) // C for i in range(len(cu) - 1))
    rec = {"profile": args.profile, "workload": w.name, "chunks": chunks,
           "ms_per_call": s0.elapsed_time(s1) / args.steps}
    if args.profile == "extend":  # kernel spans of one more call (one segment below 16384 rows: the
        # state pass then starts after the per-chunk step, so its span is the serial chain alone)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(EXT_EV)]
        gdn.gdn_set_launch_events(ev)
        call()
        gdn.gdn_set_launch_events([])
        torch.cuda.synchronize()
        rec["kernel_ms"] = extend_kernel_ms(ev)
        longest = max((cu[i + 1] - cu[i] + C - 1) // C for i in range(len(cu) - 1))
        rec["state_us_per_chunk_of_longest"] = rec["kernel_ms"]["state"] * 1e3 / longest
    print(json.dumps(rec))


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        init_dist(world, "gloo")
        run_reference(args, rank, world)
        return
    import hybrid_linear_attention_causal_b200 as gdn
    from hybrid_linear_attention_causal_b200 import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.profile:
        return run_profile_case(args, dev)
    init_dist(world, "nccl")

    seed_off = 1000 * rank  # every rank runs its own independent batch
    if args.workload == "prefill32k":
        pre = W.large_prefill(device=dev, seed=2 + seed_off)
    else:
        pre = W.long_prefill(device=dev, seed=4 + seed_off)
    dv = W.decode_verify(device=dev, seed=3 + seed_off)
    spec, dspec = pre.spec, dv.spec
    cfg, dcfg = gdn.GdnConfig.from_spec(spec), gdn.GdnConfig.from_spec(dspec)
    D = dv.extra["D"]
    xv, av, bv = dv.extra["verify"]
    Bn = dv.N
    cu_list = pre.cu_seqlens.cpu().tolist()
    chunks = sum((cu_list[i + 1] - cu_list[i] + C - 1) // C for i in range(pre.N))

    ws_pre = gdn.alloc_workspace(gdn.gdn_extend_workspace_size(cfg, pre.N, pre.T), dev)
    out_pre = torch.empty(pre.T, spec.HV, spec.dv, dtype=spec.dtype, device=dev)
    ws_d = gdn.alloc_workspace(gdn.gdn_decode_workspace_size(dcfg, Bn), dev)
    out_d = torch.empty(Bn, dspec.HV, dspec.dv, dtype=dspec.dtype, device=dev)
    ws_v = gdn.alloc_workspace(gdn.gdn_verify_workspace_size(dcfg, Bn, D), dev)
    out_v = torch.empty(Bn * D, dspec.HV, dspec.dv, dtype=dspec.dtype, device=dev)
    ck = torch.empty(Bn, D, dspec.HV, dspec.dk, dspec.dv, dtype=torch.float32, device=dev)
    cck = torch.empty(Bn, D, dspec.conv_dim, 3, dtype=dspec.dtype, device=dev)
    ws_c = gdn.alloc_workspace(gdn.gdn_commit_workspace_size(dcfg, Bn), dev)
    # accepted draft tokens per request: seeded, 0 .. D
    acc_h = torch.from_numpy(np.random.default_rng(5 + seed_off).integers(0, D + 1, Bn).astype(np.int32))
    acc = acc_h.to(dev)

    def extend(x=pre.x, a=pre.a, b=pre.b, out=out_pre):
        gdn.gdn_extend(cfg, pre.params, x, a, b, pre.cu_seqlens, pre.state_indices, pre.has_initial_state,
                       pre.conv_state, pre.ssm_state, out, ws_pre)

    def decode(x=dv.x, a=dv.a, b=dv.b, out=out_d):
        gdn.gdn_decode(dcfg, dv.params, x, a, b, dv.state_indices, dv.conv_state, dv.ssm_state, out, ws_d)

    def verify(x=xv, a=av, b=bv, out=out_v):
        gdn.gdn_verify(dcfg, dv.params, x, a, b, dv.state_indices, D, dv.conv_state, dv.ssm_state, ck, cck, out,
                       ws_v)

    def commit():
        gdn.gdn_commit(dcfg, dv.state_indices, acc, D, ck, cck, dv.conv_state, dv.ssm_state, ws_c)

    n_ev = EXT_EV + 2 + 2 + 2

    def make_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]

    def step(ev=None):
        if ev is not None:
            gdn.gdn_set_launch_events(ev[:EXT_EV])
        extend()
        if ev is not None:
            gdn.gdn_set_launch_events(ev[EXT_EV:EXT_EV + 2])
        decode()
        if ev is not None:
            gdn.gdn_set_launch_events(ev[EXT_EV + 2:EXT_EV + 4])
        verify()
        if ev is not None:
            gdn.gdn_set_launch_events(ev[EXT_EV + 4:])
        commit()
        if ev is not None:
            gdn.gdn_set_launch_events([])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_error(ws_pre) == 0 and gdn.gdn_get_device_error(ws_d) == 0
    assert gdn.gdn_get_device_error(ws_v) == 0 and gdn.gdn_get_device_error(ws_c) == 0

    evs = [make_events() for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for k in range(args.steps):
            step(evs[k])
        end.record()
        torch.cuda.synchronize()
    barrier(world)
    clocks = clk.summary()
    total_ms = max_over_ranks(start.elapsed_time(end), world, dev)
    ms_step = total_ms / args.steps

    def mean_span(i, j):
        return statistics.mean(evs[k][i].elapsed_time(evs[k][j]) for k in range(args.steps))

    ek = [extend_kernel_ms(evs[k][:EXT_EV]) for k in range(args.steps)]
    kern_ms = {name: statistics.mean(e[name] for e in ek) for name in EXT_K}
    kern_ms["decode"] = mean_span(EXT_EV, EXT_EV + 1)
    kern_ms["verify"] = mean_span(EXT_EV + 2, EXT_EV + 3)
    kern_ms["commit"] = mean_span(EXT_EV + 4, EXT_EV + 5)
    ext_ms = max_over_ranks(statistics.mean(e["extend"] for e in ek), world, dev)
    dec_ms = max_over_ranks(kern_ms["decode"], world, dev)
    ver_ms = max_over_ranks(kern_ms["verify"], world, dev)
    com_ms = max_over_ranks(kern_ms["commit"], world, dev)

    hbm, bf16, bf16_sus, peak_src = peaks()
    f16 = bf16
    f16_src = f"{peak_src} bf16 burst {bf16:.1f} TFLOP/s (fp16 and bf16 share the dense tensor rate)"
    st_dec, by_dec = decode_bytes(dspec, Bn)
    st_ver, by_ver = verify_bytes(dspec, Bn, D)
    st_com, by_com = commit_bytes(dspec, acc_h)
    value = world * pre.T / (ext_ms * 1e-3)

    kernels, pw = prefill_kernel_roofline(spec, pre.T, chunks, kern_ms, hbm, f16)
    kernels["decode"] = {"bound": "hbm", "work": by_dec, "unit": "GB/s", "peak": hbm}
    kernels["verify"] = {"bound": "hbm", "work": by_ver, "unit": "GB/s", "peak": hbm}
    kernels["commit"] = {"bound": "hbm", "work": by_com, "unit": "GB/s", "peak": hbm}
    for name in ("decode", "verify", "commit"):
        k = kernels[name]
        k["ms"] = kern_ms[name]
        k["achieved"] = k["work"] / (kern_ms[name] * 1e-3) / 1e9
        k["frac"] = k["achieved"] / k["peak"]
    dom = max(kernels, key=lambda n: kernels[n]["ms"])
    dk = kernels[dom]
    roofline = {"kernel": dom, "bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"],
                "unit": dk["unit"], "frac": dk["frac"], "traffic": ncu_traffic(f"{dom}@{pre.name}"),
                "peak_source": (f16_src if dk["unit"] == "TFLOP/s" else f"{peak_src} copy {hbm:.1f} GB/s")
                + (" (of measured)" if peak_src == "measured" else " (of fallback)")}
    prefill = prefill_summary(spec, pre.T, chunks, ext_ms, kern_ms, hbm, f16, world)
    prefill["state_chain_us_per_chunk"] = kern_ms["state"] * 1e3 / max(1, max(
        (cu_list[i + 1] - cu_list[i] + C - 1) // C for i in range(pre.N)))
    prefill["kernel_roofline"] = {k: {kk: kernels[k][kk] for kk in ("bound", "ms", "achieved", "peak", "unit", "frac")}
                                  for k in ("chunk", "state")}

    # The other prefill workload (the 8-sequence packed batch, or the long one when it is the headline's
    # alternative), outside the timed step: its own inputs, workspace and pools
    other = None
    if not args.no_side:
        alt = W.large_prefill(device=dev, seed=2 + seed_off) if args.workload == "prefill262k" else \
            W.long_prefill(device=dev, seed=4 + seed_off)
        acu = alt.cu_seqlens.cpu().tolist()
        achunks = sum((acu[i + 1] - acu[i] + C - 1) // C for i in range(alt.N))
        acfg = gdn.GdnConfig.from_spec(alt.spec)
        aws = gdn.alloc_workspace(gdn.gdn_extend_workspace_size(acfg, alt.N, alt.T), dev)
        aout = torch.empty(alt.T, alt.spec.HV, alt.spec.dv, dtype=alt.spec.dtype, device=dev)

        def alt_extend():
            gdn.gdn_extend(acfg, alt.params, alt.x, alt.a, alt.b, alt.cu_seqlens, alt.state_indices,
                           alt.has_initial_state, alt.conv_state, alt.ssm_state, aout, aws)

        for _ in range(3):
            alt_extend()
        aev = [make_events()[:EXT_EV] for _ in range(5)]
        for ev in aev:
            gdn.gdn_set_launch_events(ev)
            alt_extend()
        gdn.gdn_set_launch_events([])
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_error(aws) == 0
        aek = [extend_kernel_ms(ev) for ev in aev]
        akms = {name: statistics.mean(e[name] for e in aek) for name in EXT_K}
        a_ms = max_over_ranks(statistics.mean(e["extend"] for e in aek), world, dev)
        other = prefill_summary(alt.spec, alt.T, achunks, a_ms, akms, hbm, f16, world)
        other["workload"] = alt.name
        akern, _ = prefill_kernel_roofline(alt.spec, alt.T, achunks, akms, hbm, f16)
        other["kernel_roofline"] = {k: {kk: akern[k][kk] for kk in ("bound", "ms", "achieved", "peak", "unit", "frac")}
                                    for k in akern}
        other["note"] = "timed outside the step: 5 calls after 3 warm-up calls, CUDA events"
        del aws, aout, alt

    # Prefill state checkpoints (prefix caching), outside the timed step: the same batch with one
    # checkpoint per sequence at a boundary three fifths into it (mid chunk in general)
    cu_h = pre.cu_seqlens.to("cpu").to(torch.int64)
    ck_idx = (cu_h[:-1] + (cu_h[1:] - cu_h[:-1]) * 3 // 5).to(torch.int32).to(dev)
    ck_rows = torch.arange(pre.N, dtype=torch.int32, device=dev)
    ck_states = torch.empty(pre.N, spec.HV, spec.dk, spec.dv, dtype=torch.float32, device=dev)
    ck_conv = torch.empty(pre.N, spec.conv_dim, 3, dtype=spec.dtype, device=dev)

    def extend_ck():
        gdn.gdn_extend_checkpoints(cfg, pre.params, pre.x, pre.a, pre.b, pre.cu_seqlens, pre.state_indices,
                                   pre.has_initial_state, pre.conv_state, pre.ssm_state, out_pre, ck_idx, ck_rows,
                                   ck_states, ck_conv, ws_pre)

    for _ in range(2):
        extend_ck()
    ck_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(3)]
    for e0, e1 in ck_ev:
        e0.record()
        extend_ck()
        e1.record()
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_error(ws_pre) == 0
    ck_ms = max_over_ranks(statistics.mean(e0.elapsed_time(e1) for e0, e1 in ck_ev), world, dev)

    # Draft-tree verify (EAGLE topk 2), outside the timed step: the verify batch with each request's D
    # draft tokens as a tree whose parents are [-1, 0, 0, 1, ...] (two children per node)
    tree = torch.tensor([-1] + [(t - 1) // 2 for t in range(1, D)], dtype=torch.int32)
    parents = tree.repeat(Bn, 1).contiguous().to(dev)

    def verify_tree():
        gdn.gdn_verify_tree(dcfg, dv.params, xv, av, bv, dv.state_indices, parents, D, dv.conv_state, dv.ssm_state,
                            ck, cck, out_v, ws_v)

    for _ in range(2):
        verify_tree()
    tr_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
    for e0, e1 in tr_ev:
        e0.record()
        verify_tree()
        e1.record()
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_error(ws_v) == 0
    tr_ms = max_over_ranks(statistics.mean(e0.elapsed_time(e1) for e0, e1 in tr_ev), world, dev)
    # the tree's algorithmic bytes are verify's: a parent checkpoint it reloads was written by the same
    # thread moments before and is not counted as HBM traffic
    by_tree = by_ver

    # Mamba2 SSD scan (the second workload), outside the timed step: its inputs (1.8 GB) exceed L2
    ssd = None
    if not args.no_ssd:
        sw = W.ssd_prefill(device=dev)
        ssd_run, ssd_ws = ssd_call(sw, gdn, dev)
        for _ in range(3):
            ssd_run()
        sd_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
        for e0, e1 in sd_ev:
            e0.record()
            ssd_run()
            e1.record()
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_error(ssd_ws) == 0
        sd_ms = max_over_ranks(statistics.mean(e0.elapsed_time(e1) for e0, e1 in sd_ev), world, dev)
        sb, sf = ssd_work(sw)
        floor_ms = max(sb / (hbm * 1e9), sf / (bf16 * 1e12)) * 1e3
        ssd = {"ms": sd_ms, "tokens_per_s": world * sw.T / (sd_ms * 1e-3), "workload": sw.name,
               "config": {"heads": sw.spec.H, "headdim": sw.spec.P, "dstate": sw.spec.N, "groups": sw.spec.G,
                          "lengths": sw.lengths, "state_dtype": "bf16", "D": True, "z": True},
               "roofline": {"bound": "hbm", "achieved": sb / (sd_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                            "frac": sb / (sd_ms * 1e-3) / 1e9 / hbm, "floor_ms": floor_ms,
                            "algorithmic_bytes": sb, "tensor_frac": sf / (sd_ms * 1e-3) / 1e12 / bf16,
                            "traffic": ncu_traffic("ssd")},
               "note": "timed outside the step; one ssd_combined_fwd per timing"}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            orun, on, oworkers = ssd_oracle_sample(sw, 1024)
            t0 = time.perf_counter()
            orun()
            odt = time.perf_counter() - t0
            ssd["cpu_baseline"] = {"value": on / odt, "unit": "rows/s", "cores": oworkers, "kind": "oracle",
                                   "sample": f"fp64 oracle, first {on} packed rows of the batch, all {sw.spec.H} heads"}
        del ssd_run, ssd_ws

    # End to end through the public API with pinned host buffers.  The layer is causal per sequence,
    # so the step cuts every sequence into pieces of --e2e-piece rows and calls gdn_extend once per
    # piece, each piece continuing from the state and conv window the previous one left in the slot
    # (prefix-then-extend equals the whole sequence); the host -> device copy of piece i + 1 and the
    # device -> host copy of piece i - 1 overlap the call for piece i (two copy streams, events
    # between them): the same bytes and the same work as one call over the whole batch.
    e2e = None
    if args.e2e_steps > 0:
        hx, ha, hb = (t.cpu().pin_memory() for t in (pre.x, pre.a, pre.b))
        dx, da, db = torch.empty_like(pre.x), torch.empty_like(pre.a), torch.empty_like(pre.b)
        hout = torch.empty(out_pre.shape, dtype=out_pre.dtype).pin_memory()
        hi_h = pre.has_initial_state.cpu()
        pieces = []  # (row range, host metadata [cu, slot, flag] pinned, device copies)
        for i in range(pre.N):
            r0, r1 = int(cu_h[i]), int(cu_h[i + 1])
            for q0 in range(r0, r1, args.e2e_piece):
                q1 = min(r1, q0 + args.e2e_piece)
                flag = hi_h[i:i + 1].clone() if q0 == r0 else torch.ones(1, dtype=torch.int32)
                hm = [torch.tensor([0, q1 - q0], dtype=torch.int32).pin_memory(),
                      pre.state_indices[i:i + 1].cpu().pin_memory(), flag.pin_memory()]
                pieces.append((q0, q1, hm, [torch.empty_like(t, device=dev) for t in hm]))
        ws_e2e = gdn.alloc_workspace(gdn.gdn_extend_workspace_size(cfg, 1, args.e2e_piece), dev)
        h2d = sum(t.numel() * t.element_size() for t in (hx, ha, hb)) + \
            sum(t.numel() * t.element_size() for g in pieces for t in g[2])
        d2h = hout.numel() * hout.element_size()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in pieces]
        ev_out = [torch.cuda.Event() for _ in pieces]

        def e2e_step():
            cur = torch.cuda.current_stream()
            s_in.wait_stream(cur)
            s_out.wait_stream(cur)
            with torch.cuda.stream(s_in):
                for k, (r0, r1, hm, dm) in enumerate(pieces):
                    for h, d_ in zip((hx[r0:r1], ha[r0:r1], hb[r0:r1], *hm), (dx[r0:r1], da[r0:r1], db[r0:r1], *dm)):
                        d_.copy_(h, non_blocking=True)
                    ev_in[k].record(s_in)
            for k, (r0, r1, hm, dm) in enumerate(pieces):
                cur.wait_event(ev_in[k])
                gdn.gdn_extend(cfg, pre.params, dx[r0:r1], da[r0:r1], db[r0:r1], dm[0], dm[1], dm[2],
                               pre.conv_state, pre.ssm_state, out_pre[r0:r1], ws_e2e)
                ev_out[k].record(cur)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_out[k])
                    hout[r0:r1].copy_(out_pre[r0:r1], non_blocking=True)
            cur.wait_stream(s_out)

        e2e_step()
        torch.cuda.synchronize()
        assert gdn.gdn_get_device_error(ws_e2e) == 0
        barrier(world)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(args.e2e_steps):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(s0.elapsed_time(s1) / args.e2e_steps, world, dev)
        e2e = {"value": world * pre.T / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "what": f"pinned host buffers; per piece of {args.e2e_piece} rows: host -> device copy of its "
                       "inputs, gdn_extend continuing from the slot, device -> host copy of its out, "
                       "pipelined across pieces on two copy streams"}
        del hx, ha, hb, dx, da, db, hout, ws_e2e

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        run, n, workers = oracle_sample(pre, args.cpu_sample_tokens)
        t0 = time.perf_counter()
        run()
        dt = time.perf_counter() - t0
        cpu_baseline = {"value": n / dt, "unit": "tokens/s", "cores": workers, "kind": "oracle",
                        "sample": f"fp64 oracle, first {n} packed rows of the {pre.name} batch, "
                                  f"all {spec.HV} value heads"}

    if rank == 0:
        nseg = min(16, max(1, pre.T // 16384))
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16/f32", "data": "synthetic",
            "config": workload_config(pre, args),
            "roofline": roofline,
            "cpu_baseline": cpu_baseline,
            "e2e": e2e,
            # extend: chunk table, the per-chunk step and the state pass per segment, conv-state update;
            # decode; verify; commit
            "gpu_launches": args.steps * (2 + 2 * nseg + 3),
            "clocks": clocks,
            "prefill": prefill,
            "prefill_other": other,
            "decode": {"ms": dec_ms, "requests_per_s": world * Bn / (dec_ms * 1e-3),
                       "state_gbs": world * st_dec / (dec_ms * 1e-3) / 1e9,
                       "total_gbs": world * by_dec / (dec_ms * 1e-3) / 1e9,
                       "frac_of_8tbs_state": st_dec / (dec_ms * 1e-3) / 8e12,
                       "frac_of_measured_hbm": by_dec / (dec_ms * 1e-3) / 1e9 / hbm},
            "verify": {"ms": ver_ms, "state_gbs": world * st_ver / (ver_ms * 1e-3) / 1e9,
                       "total_gbs": world * by_ver / (ver_ms * 1e-3) / 1e9,
                       "frac_of_8tbs_state": st_ver / (ver_ms * 1e-3) / 8e12,
                       "frac_of_measured_hbm": by_ver / (ver_ms * 1e-3) / 1e9 / hbm},
            "commit": {"ms": com_ms, "accepted_requests": int((acc_h > 0).sum()),
                       "total_gbs": world * by_com / (com_ms * 1e-3) / 1e9,
                       "frac_of_measured_hbm": by_com / (com_ms * 1e-3) / 1e9 / hbm},
            "verify_tree": {"ms": tr_ms, "parents": tree.tolist(), "total_gbs": world * by_tree / (tr_ms * 1e-3) / 1e9,
                            "frac_of_measured_hbm": by_tree / (tr_ms * 1e-3) / 1e9 / hbm,
                            "note": "timed outside the step; bytes counted as verify's (parent reloads not counted)"},
            "ssd": ssd,
            "prefill_checkpoints": {"ms": ck_ms, "checkpoints": pre.N, "vs_prefill": ck_ms / ext_ms,
                                    "note": "one state checkpoint per sequence, mid chunk; timed outside the step"},
            "kernels": {k: {kk: v[kk] for kk in ("bound", "ms", "achieved", "peak", "unit", "frac")}
                        for k, v in kernels.items()},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
