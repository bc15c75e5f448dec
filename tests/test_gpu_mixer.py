"""GPU parity of the Mamba-2 mixer around the path: the tensor-core linear
layer (ssd_linear_bf16) against float64 products of the same bf16 operands,
and the whole mixer (ssd_mixer_fwd: in_proj, conv1d+SiLU, chunked scan,
gated RMSNorm, out_proj) against the fp64 oracle (oracle.mixer_forward) on
identical seeded inputs, called through the C ABI.

Bounds: a linear layer's output is its fp32 sum rounded to bf16, so each
element is held to 2^-8 of its own size plus 1e-3 of the output's scale.
The mixer's outputs carry the bf16 rounding of every intermediate (in_proj
output, conv output, y, the normed y), so they take the bf16 bound of the
other parity tests, 2e-2 normalised max-abs; so do the conv cache (copies
of the bf16 in_proj output, which the oracle keeps in float64) and the final
state."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import TOL_BF16_NMA, cuda, f64, norm_max_abs
from ssd_selective_scan_b200 import layer, synth

pytestmark = pytest.mark.gpu


def _check_linear(y, ref, what):
    y = f64(y)
    scale = float(np.max(np.abs(ref)))
    err = np.abs(y - ref) - (2.0 ** -8) * np.abs(ref)
    assert float(np.max(err)) <= 1e-3 * scale, f"{what}: worst excess {float(np.max(err)):.3e} (scale {scale:.3e})"


@pytest.mark.parametrize("M,N,K", [(300, 520, 200), (128, 256, 64), (5, 8, 8), (1000, 7208, 2560)])
def test_linear_matches_fp64(M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    y = layer.linear(cuda(x), cuda(w))
    torch.cuda.synchronize()
    _check_linear(y, f64(x) @ f64(w).T, f"linear {M}x{N}x{K}")


def test_linear_strided_rows():
    """x and y as column ranges of wider rows (the layouts in_proj and the
    mixer's workspace use)."""
    g = torch.Generator().manual_seed(5)
    xw = torch.randn(300, 200, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(264, 120, generator=g) / 11.0).to(torch.bfloat16).cuda()
    yw = torch.zeros(300, 400, dtype=torch.bfloat16, device="cuda")
    x = xw[:, 40:160]
    layer.linear(x, w, y=yw[:, 64:328])
    torch.cuda.synchronize()
    _check_linear(yw[:, 64:328], f64(x) @ f64(w).T, "strided linear")
    assert torch.count_nonzero(yw[:, :64]) == 0 and torch.count_nonzero(yw[:, 328:]) == 0


def test_linear_in_proj_shape_sampled_rows():
    """The 3B layer's in_proj at full size (16384 tokens x 2560 -> 7208),
    checked on 96 sampled rows computed one by one in float64."""
    M, N, K = 16384, 7208, 2560
    g = torch.Generator().manual_seed(11)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    y = layer.linear(cuda(x), cuda(w))
    torch.cuda.synchronize()
    rows = torch.randperm(M, generator=g)[:96].sort().values
    _check_linear(y[rows.cuda()], f64(x[rows]) @ f64(w).T, "in_proj sampled rows")


def _run_mixer(s, d_model, inp, **kw):
    d = {k: cuda(v) for k, v in inp.items()}
    out, fs = layer.mixer_forward(d["hidden"], d["W_in"], d["conv_w"], d["dt_bias"], d["A"], d["D"], d["norm_w"],
                                  d["W_out"], s.H, s.P, s.G, s.N, conv_bias=d["conv_bias"],
                                  conv_state=d["conv_state"], init_state=d["init_state"], Q=s.Q, **kw)
    return out, fs, d["conv_state"]


def _oracle_mixer(s, inp, **kw):
    f = lambda t: None if t is None else f64(t)
    return oracle.mixer_forward(f(inp["hidden"]), f(inp["W_in"]), f(inp["conv_w"]), f(inp["conv_bias"]),
                                f(inp["dt_bias"]), f(inp["A"]), f(inp["D"]), f(inp["norm_w"]), f(inp["W_out"]),
                                s.H, s.P, s.G, s.N, conv_state=f(inp["conv_state"]),
                                init_state=f(inp["init_state"]), **kw)


MIXER = {
    # a short layer with a ragged last chunk, cache, conv bias and initial state
    "small_all_inputs": (synth.CONFIGS[1].with_(b=2, L=300, H=8, G=2), 256,
                         dict(conv_bias=True, conv_state=True, init_state=True), {}),
    # grouped gate norm (one slice per B/C group)
    "grouped_norm": (synth.CONFIGS[1].with_(b=1, L=257, H=16, G=4), 512, dict(conv_state=True), dict(norm_groups=4)),
}


@pytest.mark.parametrize("name", sorted(MIXER))
def test_mixer_matches_oracle(name):
    s, d_model, ikw, kw = MIXER[name]
    inp = synth.mixer_inputs(s, d_model, 71000 + len(name), **ikw)
    out, fs, cs = _run_mixer(s, d_model, inp, **kw)
    out_ref, fs_ref, cs_ref = _oracle_mixer(s, inp, **kw)
    torch.cuda.synchronize()
    e = norm_max_abs(out, out_ref)
    assert e <= TOL_BF16_NMA, f"{name}: out normalised error {e:.3e}"
    es = norm_max_abs(fs, fs_ref)
    assert es <= TOL_BF16_NMA, f"{name}: final state normalised error {es:.3e}"
    if cs is not None:
        ec = norm_max_abs(cs, cs_ref)
        assert ec <= TOL_BF16_NMA, f"{name}: conv cache normalised error {ec:.3e}"
    assert torch.isfinite(out.float()).all()


def test_mixer_full_3b_layer_matches_oracle():
    """The FRANKENSTALLM-H 3B mixer at full size: 8 x 2048 tokens, d_model
    2560, 40 heads x 64, d_state 128, 8 groups, element by element."""
    s = synth.CONFIGS[1]
    d_model = 2560
    inp = synth.mixer_inputs(s, d_model, synth.config_seed(1))
    out, fs, _ = _run_mixer(s, d_model, inp)
    out_ref, fs_ref, _ = _oracle_mixer(s, inp)
    torch.cuda.synchronize()
    e = norm_max_abs(out, out_ref)
    assert e <= TOL_BF16_NMA, f"out normalised error {e:.3e}"
    es = norm_max_abs(fs, fs_ref)
    assert es <= TOL_BF16_NMA, f"final state normalised error {es:.3e}"


def test_mixer_is_deterministic_and_status_clean():
    s = synth.CONFIGS[1].with_(b=2, L=300, H=8, G=2)
    inp = synth.mixer_inputs(s, 256, 72000)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    a, fa, _ = _run_mixer(s, 256, inp, status=st)
    b, fb, _ = _run_mixer(s, 256, inp)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(a, b) and torch.equal(fa, fb)
