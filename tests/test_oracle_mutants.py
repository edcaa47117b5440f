"""The oracle's pins must catch plausible mistakes.  Each case compiles a copy
of the oracle source with one planted mistake (on the CPU, into a temporary
directory), loads it through GDN_ORACLE_LIB in a child pytest run of the pin
suite, and expects that run to fail."""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.c")

MUTANTS = {
    "delta_sign": ("u[j] = beta[t] * (vt[j] - kS);", "u[j] = beta[t] * (vt[j] + kS);"),
    "no_decay": ("for (int i = 0; i < dk * dv; ++i) S[i] *= decay;", "(void)decay;"),
    "write_with_query": ("S[(int64_t)i * dv + j] += kt[i] * u[j];", "S[(int64_t)i * dv + j] += qt[i] * u[j];"),
    "no_scale": ("o[(int64_t)t * dv + j] = scale * acc;\n        }\n        if (states)",
                 "o[(int64_t)t * dv + j] = acc;\n        }\n        if (states)"),
    "conv_reversed": ("acc += w[(int64_t)c * K + j] * xv;", "acc += w[(int64_t)c * K + (K - 1 - j)] * xv;"),
    "softplus_no_one": ("log1p(exp(x))", "log(exp(x))"),
    "gqa_interleaved": ("int hk = h / G;", "int hk = h % HK;"),
    "l2_eps_outside": ("double inv = 1.0 / sqrt(ss + eps);", "double inv = 1.0 / (sqrt(ss) + eps);"),
    "chunk_no_beta_in_A": ("val = bb[r] * exp(gam[r] - gam[s]) * kk;", "val = exp(gam[r] - gam[s]) * kk;"),
    "chunk_decay_sign": ("intra += exp(gam[r] - gam[s]) * qk", "intra += exp(gam[s] - gam[r]) * qk"),
    "conv_tail_shift": ("int64_t pos = (int64_t)L + i;", "int64_t pos = (int64_t)L + i - 1;"),
    "verify_ckpt_window": ("int src = t + 1 - (K - 1) + j;", "int src = t - (K - 1) + j;"),
    "ckpt_one_token_early": ("if (bnd > cu[n]) memcpy(dst, st + (bnd - 1) * sslot, sizeof(double) * sslot);",
                             "if (bnd > cu[n] + 1) memcpy(dst, st + (bnd - 2) * sslot, sizeof(double) * sslot);"),
    "commit_off_by_one": ("const int64_t t = (int64_t)i * D + (acc[i] - 1);", "const int64_t t = (int64_t)i * D + acc[i] % D;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/present"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mut.c")
        so = os.path.join(d, "libmut.so")
        open(c, "w").write(src.replace(old, new))
        subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so, c, "-lm"], check=True)
        env = dict(os.environ, GDN_ORACLE_LIB=so)
        r = subprocess.run(
            [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
             os.path.join(ROOT, "tests", "test_oracle_pins.py")],
            cwd=ROOT, env=env, capture_output=True, text=True, timeout=600,
        )
        assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"


SSD_SRC = os.path.join(ROOT, "oracle", "ssd_oracle.c")

SSD_MUTANTS = {
    "ssd_exclusive_output": ("acc += v * Ct[i];", "acc += (v - d * xt[p] * Bt[i]) * Ct[i];"),
    "ssd_decay_sign": ("const double decay = exp(d * A[h]);", "const double decay = exp(-d * A[h]);"),
    "ssd_group_interleaved": ("h / hpg;\n            double* S = (double*)malloc(sizeof(double) * ss);\n            if (init)",
                              "h % G;\n            double* S = (double*)malloc(sizeof(double) * ss);\n            if (init)"),
    "ssd_gate_no_silu": ("v *= zt[p] * ssd_sigmoid(zt[p]);", "v *= ssd_sigmoid(zt[p]);"),
    "ssd_bias_after_softplus": ("double v = dt + bias;\n    if (c->dt_softplus) v = ssd_softplus(v);",
                                "double v = dt;\n    if (c->dt_softplus) v = ssd_softplus(v);\n    v += bias;"),
    "ssd_input_without_step": ("+ d * xt[p] * Bt[i];", "+ xt[p] * Bt[i];"),
    "ssd_ckpt_one_token_late": ("t + 1 - cu[n] == ck", "t - cu[n] == ck"),
    "ssd_skip_index": ("D[(int64_t)h * c->P + p]", "D[(int64_t)p * c->H + h]"),
    "ssd_chunk_state_decay": ("const double w = exp(gl - gam[s]) * dd[s];", "const double w = exp(gl) * dd[s];"),
    "ssd_chunk_carry_undecayed": ("yr[p] = exp(gam[r]) * inter;", "yr[p] = inter;"),
}


@pytest.mark.parametrize("name", sorted(SSD_MUTANTS))
def test_ssd_pins_catch_planted_mistake(name):
    old, new = SSD_MUTANTS[name]
    src = open(SSD_SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/present"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mut.c")
        so = os.path.join(d, "libmut.so")
        open(c, "w").write(src.replace(old, new))
        subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so, c, "-lm"], check=True)
        env = dict(os.environ, SSD_ORACLE_LIB=so)
        r = subprocess.run(
            [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
             os.path.join(ROOT, "tests", "test_ssd_oracle_pins.py")],
            cwd=ROOT, env=env, capture_output=True, text=True, timeout=600,
        )
        assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
