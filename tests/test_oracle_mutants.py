"""Plant plausible mistakes in a copy of the oracle's C source and check that
the pins catch every one of them (CPU only).

Each mutant is a one-token edit of the kind a careful reader could still miss:
a dropped term, a wrong sign, a wrong index, operands swapped.  The edited
copy is compiled into a temporary directory and routed to with
``oracle.using_library``; the default oracle build is never touched.
"""
import os
import subprocess

import pytest

import oracle
import oracle_checks

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")

MUTANTS = {
    "drop_D_term": ("yt[p] = acc + Dh * xt[p];", "yt[p] = acc;"),
    "decay_sign": ("const double a = exp(dt * A);", "const double a = exp(-dt * A);"),
    "decay_missing_dt": ("const double a = exp(dt * A);", "const double a = exp(A);"),
    "input_missing_dt": ("row[n] = a * row[n] + dt * xt[p] * Bt[n];", "row[n] = a * row[n] + xt[p] * Bt[n];"),
    "output_before_update": (
        "row[n] = a * row[n] + dt * xt[p] * Bt[n];\n                acc += Ct[n] * row[n];",
        "acc += Ct[n] * row[n];\n                row[n] = a * row[n] + dt * xt[p] * Bt[n];"),
    "B_C_swapped": ("acc += Ct[n] * row[n];", "acc += Bt[n] * row[n];"),
    "group_map_modulo": ("const int64_t g = h / (H / G);", "const int64_t g = h % G;"),
    "softplus_no_abs": ("log1p(exp(-fabs(v)))", "log1p(exp(-v))"),
    "dt_bias_ignored": ("J->dt_raw[(bi * L + t) * H + h] + bias", "J->dt_raw[(bi * L + t) * H + h]"),
    "init_state_ignored": ("if (J->init_state) memcpy", "if (0) memcpy"),
    "silu_sign": ("return v / (1.0 + exp(-v));", "return v / (1.0 + exp(v));"),
    "conv_taps_reversed": ("acc += w[c * k + j] * hist[(t - k + 1 + j) + k];",
                           "acc += w[c * k + (k - 1 - j)] * hist[(t - k + 1 + j) + k];"),
    "conv_off_by_one": ("acc += w[c * k + j] * hist[(t - k + 1 + j) + k];",
                        "acc += w[c * k + j] * hist[(t - k + j) + k];"),
    "conv_cache_shift": ("conv_state[(bi * conv_dim + c) * k + j] = hist[L + j];",
                         "conv_state[(bi * conv_dim + c) * k + j] = hist[L + j - (j > 0)];"),
    "conv_bias_dropped": ("double acc = bias ? bias[c] : 0.0;", "double acc = 0.0;"),
    # backward pass
    "bwd_output_term_dropped": ("g[p * N + n] += dyt[p] * Ct[n];", "g[p * N + n] += 0.0 * Ct[n];"),
    "bwd_dC_from_previous_state": ("acc += dyt[p] * ht[p * N + n];", "acc += dyt[p] * hprev[p * N + n];"),
    "bwd_dB_missing_dt": ("dBt[n] += dt * acc;", "dBt[n] += acc;"),
    "bwd_ddt_decay_term_dropped": ("const double ddt = xgb + A * a * gh;", "const double ddt = xgb;"),
    "bwd_sigmoid_sign": ("const double dv = ddt * sigmoid(v);", "const double dv = ddt * sigmoid(-v);"),
    "bwd_dA_missing_dt": ("dA += dt * a * gh;", "dA += a * gh;"),
    "bwd_state_gradient_not_decayed": ("for (int64_t i = 0; i < PN; ++i) g[i] *= a;",
                                       "for (int64_t i = 0; i < PN; ++i) g[i] *= 1.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique in oracle source"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib_path = str(tmp_path / "libmutant.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           str(mutated), "-o", lib_path, "-lm"])
    lib = oracle.open_library(lib_path)
    caught = []
    with oracle.using_library(lib):
        for check in oracle_checks.ALL_CHECKS:
            try:
                check()
            except AssertionError:
                caught.append(check.__name__)
    assert caught, f"planted mistake {name!r} passed every pin"


def _carry_state_across_sequences(x, B, C, dt_raw, A, cu_seqlens, dt_bias=None, D=None, init_state=None,
                                  nthreads=None):
    """Planted mistake: every sequence after the first starts from the
    previous sequence's final state instead of its own initial state."""
    import numpy as np
    y, fs = _REAL_VARLEN(x, B, C, dt_raw, A, [0, int(cu_seqlens[-1])], dt_bias, D,
                         None if init_state is None else init_state[:1], nthreads)
    n = len(cu_seqlens) - 1
    return y, np.repeat(fs, n, axis=0)


def _ignore_initial_states(x, B, C, dt_raw, A, cu_seqlens, dt_bias=None, D=None, init_state=None,
                           nthreads=None):
    """Planted mistake: the per-sequence initial states are dropped."""
    return _REAL_VARLEN(x, B, C, dt_raw, A, cu_seqlens, dt_bias, D, None, nthreads)


_REAL_VARLEN = oracle.selective_scan_varlen


@pytest.mark.parametrize("mutant", [_carry_state_across_sequences, _ignore_initial_states],
                         ids=lambda f: f.__name__)
def test_pins_catch_planted_ragged_mistake(mutant, monkeypatch):
    monkeypatch.setattr(oracle, "selective_scan_varlen", mutant)
    with pytest.raises(AssertionError):
        oracle_checks.check_varlen_matches_each_sequence_alone()


# Planted mistakes in the mixer around the path (gated RMSNorm and the two
# projections, written in numpy in oracle/__init__.py): the edited module is
# executed apart and its mixer functions are routed to for the checks.
PY_SRC = os.path.join(os.path.dirname(oracle.__file__), "__init__.py")

MIXER_MUTANTS = {
    "gate_sigmoid_not_silu": ("return v / (1.0 + np.exp(-v))", "return 1.0 / (1.0 + np.exp(-v))"),
    "norm_sum_not_mean": ("ms = np.mean(gs * gs, axis=-1, keepdims=True)", "ms = np.sum(gs * gs, axis=-1, keepdims=True)"),
    "norm_groups_interleaved": ("gs = g.reshape(*shp[:-1], groups, d // groups)",
                                "gs = g.reshape(*shp[:-1], d // groups, groups).swapaxes(-1, -2)"),
    "norm_eps_outside_sqrt": ("return (gs / np.sqrt(ms + eps)).reshape(shp)",
                              "return (gs / (np.sqrt(ms) + eps)).reshape(shp)"),
    "dt_from_the_front": ("dt_raw = np.ascontiguousarray(zxbcdt[..., d_inner + conv_dim:])",
                          "dt_raw = np.ascontiguousarray(zxbcdt[..., :H])"),
    "xBC_offset_by_z": ("xBC = np.ascontiguousarray(zxbcdt[..., d_inner:d_inner + conv_dim])",
                        "xBC = np.ascontiguousarray(zxbcdt[..., :conv_dim])"),
    "in_proj_not_transposed": ("zxbcdt = hidden @ W_in.T", "zxbcdt = hidden @ W_in"),
    "out_proj_not_transposed": ("out = n @ _f64(W_out).T", "out = n @ _f64(W_out)"),
}


@pytest.mark.parametrize("name", sorted(MIXER_MUTANTS))
def test_pins_catch_planted_mixer_mistake(name, monkeypatch):
    old, new = MIXER_MUTANTS[name]
    src = open(PY_SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique in the oracle module"
    ns = {"__name__": "oracle_mutant", "__file__": PY_SRC}
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), ns)
    for fn in ("silu", "rmsnorm_gated", "mixer_forward"):
        monkeypatch.setattr(oracle, fn, ns[fn])
    caught = []
    for check in oracle_checks.ALL_CHECKS:
        try:
            check()
        except Exception:   # a wrong value, or a shape that no longer fits
            caught.append(check.__name__)
    assert caught, f"planted mistake {name!r} passed every pin"
