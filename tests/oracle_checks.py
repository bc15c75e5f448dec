"""Checks that pin the fp64 oracle to things other than itself.

Each ``check_*`` function raises AssertionError when the oracle currently
routed by ``oracle`` (the default build, or a planted-mistake build selected
with ``oracle.using_library``) disagrees with:

* closed forms (dt -> 0 gives y = D x; scalar geometric series; a hand-worked
  case with softplus(0) = ln 2 and exp(-ln 2) = 1/2; SiLU through an identity
  conv tap);
* library routines for special cases (``np.convolve`` for the causal conv,
  ``np.logaddexp`` for softplus);
* the brute-force L x L state-space-duality matrix M[t,s] = (C_t.B_s)
  exp(sum_{r=s+1..t} dt_r A) dt_s ("Hybrid Architectures ..." summary page,
  section 2: state space duality recasts the scan as a matrix product;
  appendix O: Mamba's implicit attention matrix);
* an independent chunked evaluation of the same operator at several chunk
  lengths (chunk-size invariance; chunk length 1 is the recurrence itself and
  chunk length L is the full matrix);
* invariants: linearity of y - D x in x, causality, state hand-off between
  calls, prefill(L) + one decode step = prefill(L + 1), conv-state hand-off;
* the Mamba cache-size formula of the same page's appendix C, which fixes the
  element counts of the conv state and the SSM state;
* for the backward pass: central finite differences of the forward oracle for
  every input element (brute force on a tiny problem), the closed form of dD,
  the dt -> 0 limit, linearity in the output gradients, and independence of
  the thread count;
* for the mixer around the path (in_proj, the path, gated RMSNorm, out_proj):
  a hand-worked gated norm, SiLU against the library logistic function,
  the unit mean square and scale invariance of the norm, the slice-wise
  definition of a grouped norm, and the wiring of both projections against
  explicit index loops on a tiny layer.

All inputs are small and seeded so the whole set runs in seconds on a CPU.
"""
from __future__ import annotations

import math

import numpy as np

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3e}"


def _random_scan_inputs(rng, b=2, L=48, H=4, P=5, N=6, G=2, init=True, a_lo=0.05, a_hi=2.0):
    x = rng.standard_normal((b, L, H, P))
    B = rng.standard_normal((b, L, G, N)) / math.sqrt(N)
    C = rng.standard_normal((b, L, G, N)) / math.sqrt(N)
    dt_raw = rng.uniform(-4.0, 1.0, (b, L, H))
    dt_bias = rng.standard_normal(H) * 0.5
    A = -np.exp(rng.uniform(math.log(a_lo), math.log(a_hi), H))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((b, H, P, N)) * 0.3 if init else None
    return dict(x=x, B=B, C=C, dt_raw=dt_raw, dt_bias=dt_bias, A=A, D=D, init_state=h0)


def _scan(inp):
    return oracle.selective_scan(inp["x"], inp["B"], inp["C"], inp["dt_raw"], inp["A"],
                                 inp["dt_bias"], inp["D"], inp["init_state"], nthreads=2)


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------

def check_dt_to_zero():
    """dt_raw -> -40 makes dt = softplus(-40) ~ 4e-18: the state keeps its
    initial value and y_t = C_t.h0 + D x_t (with h0 = 0: y = D x)."""
    inp = _random_scan_inputs(_rng(1))
    inp["dt_raw"] = np.full_like(inp["dt_raw"], -40.0)
    inp["dt_bias"] = np.zeros_like(inp["dt_bias"])
    y, fs = _scan(inp)
    _close(fs, inp["init_state"], 1e-14, "dt->0 final state")
    H, G = inp["x"].shape[2], inp["B"].shape[2]
    g_of_h = np.arange(H) // (H // G)
    Cg = inp["C"][:, :, g_of_h, :]                               # [b,L,H,N]
    expect = np.einsum("blhn,bhpn->blhp", Cg, inp["init_state"]) + inp["D"][None, None, :, None] * inp["x"]
    _close(y, expect, 1e-13, "dt->0 output")
    inp["init_state"] = None
    y0, fs0 = _scan(inp)
    _close(y0, inp["D"][None, None, :, None] * inp["x"], 1e-15, "dt->0, zero state: y = D x")
    assert np.all(np.abs(fs0) < 1e-15), "dt->0, zero state: final state must stay 0"


def check_geometric_series():
    """Constant dt, B, C, x and one head: h_t = a h_{t-1} + dt x B gives
    h_t = a^{t+1} h0 + dt x B (1 - a^{t+1}) / (1 - a), a = exp(dt A)."""
    L, P, N = 40, 3, 4
    rng = _rng(2)
    Bv = rng.standard_normal(N)
    Cv = rng.standard_normal(N)
    xv = rng.standard_normal(P)
    h0 = rng.standard_normal((P, N))
    v, A, D = -0.7, -0.9, 0.25
    dt = math.log1p(math.exp(v))
    a = math.exp(dt * A)
    x = np.broadcast_to(xv, (1, L, 1, P)).copy()
    B = np.broadcast_to(Bv, (1, L, 1, N)).copy()
    C = np.broadcast_to(Cv, (1, L, 1, N)).copy()
    y, fs = oracle.selective_scan(x, B, C, np.full((1, L, 1), v), np.array([A]),
                                  None, np.array([D]), h0[None, None])
    t = np.arange(L)[:, None]
    geo = (1.0 - a ** (t + 1)) / (1.0 - a)                       # [L,1]
    expect = (a ** (t + 1)) * (h0 @ Cv)[None, :] + dt * (Cv @ Bv) * geo * xv[None, :] + D * xv[None, :]
    _close(y[0, :, 0, :], expect, 1e-13, "geometric series y")
    fs_expect = a ** L * h0 + dt * np.outer(xv, Bv) * (1.0 - a ** L) / (1.0 - a)
    _close(fs[0, 0], fs_expect, 1e-13, "geometric series final state")


def check_hand_worked():
    """dt_raw = 0, A = -1, B = C = x = 1, D = 3, one state: dt = softplus(0) =
    ln 2 and exp(dt A) = 1/2, so h_t = ln2 (2 - 2^-t) and y_t = h_t + 3."""
    L = 12
    ones = np.ones((1, L, 1, 1))
    y, fs = oracle.selective_scan(ones, ones, ones, np.zeros((1, L, 1)), np.array([-1.0]),
                                  None, np.array([3.0]))
    expect = [math.log(2.0) * (2.0 - 2.0 ** (-t)) + 3.0 for t in range(L)]
    _close(y[0, :, 0, 0], expect, 1e-15, "hand-worked y")
    _close(fs.reshape(-1), [math.log(2.0) * (2.0 - 2.0 ** (-(L - 1)))], 1e-15, "hand-worked state")


def check_conv_identity_tap():
    """Taps (0,..,0,1) and no bias reduce the conv to the identity, so
    u = SiLU(xBC) = xBC / (1 + exp(-xBC)); SiLU(0) = 0."""
    rng = _rng(3)
    xbc = rng.standard_normal((2, 9, 7)) * 3.0
    xbc[0, 0, 0] = 0.0
    k = 4
    w = np.zeros((7, k))
    w[:, k - 1] = 1.0
    st = rng.standard_normal((2, 7, k))
    u, _ = oracle.conv1d_silu(xbc, w, None, st)
    _close(u, xbc / (1.0 + np.exp(-xbc)), 1e-15, "identity tap = SiLU")
    assert u[0, 0, 0] == 0.0


# ----------------------------------------------------------------------------
# library routines for special cases
# ----------------------------------------------------------------------------

def check_conv_matches_np_convolve():
    """Causal depthwise conv with a cached left context equals np.convolve of
    the extended sequence with the reversed taps (valid part), then SiLU;
    the new cache is the last k inputs of the extended sequence."""
    rng = _rng(4)
    for (b, L, cd, k) in [(2, 11, 5, 4), (1, 2, 3, 4), (3, 1, 4, 4), (1, 7, 2, 3)]:
        xbc = rng.standard_normal((b, L, cd))
        w = rng.standard_normal((cd, k)) * 0.5
        bias = rng.standard_normal(cd) * 0.3
        st = rng.standard_normal((b, cd, k))
        u, st2 = oracle.conv1d_silu(xbc, w, bias, st)
        for bi in range(b):
            for c in range(cd):
                ext = np.concatenate([st[bi, c, :], xbc[bi, :, c]])           # times -k .. L-1
                pre = np.convolve(ext[1:], w[c, ::-1], mode="valid") + bias[c]  # starts at time -k+1
                _close(u[bi, :, c], pre / (1.0 + np.exp(-pre)), 1e-14, f"conv vs np.convolve {b,L,cd,k}")
                _close(st2[bi, c, :], ext[-k:], 0.0, "conv new cache")
        u0, none = oracle.conv1d_silu(xbc, w, bias, None)
        assert none is None
        for bi in range(b):
            for c in range(cd):
                ext = np.concatenate([np.zeros(k - 1), xbc[bi, :, c]])
                pre = np.convolve(ext, w[c, ::-1], mode="valid") + bias[c]
                _close(u0[bi, :, c], pre / (1.0 + np.exp(-pre)), 1e-14, "conv, zero left context")


def _softplus(v):
    return np.logaddexp(0.0, v)


def check_matrix_form():
    """Brute-force L x L SSD matrix with the initial-state term:
    y_t = sum_{s<=t} (C_t.B_s) exp(sum_{r=s+1..t} dt_r A) dt_s x_s
          + exp(sum_{r=0..t} dt_r A) C_t.h0 + D x_t,
    with dt = np.logaddexp(0, dt_raw + dt_bias) and head h on group h/(H/G)."""
    inp = _random_scan_inputs(_rng(5), b=2, L=37, H=4, P=3, N=5, G=2)
    y, fs = _scan(inp)
    x, B, C = inp["x"], inp["B"], inp["C"]
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            dt = _softplus(inp["dt_raw"][bi, :, h] + inp["dt_bias"][h])
            lg = dt * inp["A"][h]
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    M[t, s] = (C[bi, t, g] @ B[bi, s, g]) * math.exp(lg[s + 1: t + 1].sum()) * dt[s]
            h0 = inp["init_state"][bi, h]
            decay0 = np.exp(np.cumsum(lg))                                   # exp(sum_{r<=t})
            y_ref = M @ x[bi, :, h, :] + decay0[:, None] * (C[bi, :, g, :] @ h0.T) + inp["D"][h] * x[bi, :, h, :]
            _close(y[bi, :, h, :], y_ref, 1e-12, f"matrix form y (b={bi}, h={h})")
            # final state: h_L = exp(sum lg) h0 + sum_s exp(sum_{r>s} lg) dt_s x_s B_s^T
            w_s = np.array([math.exp(lg[s + 1:].sum()) * dt[s] for s in range(L)])
            fs_ref = decay0[-1] * h0 + (x[bi, :, h, :] * w_s[:, None]).T @ B[bi, :, g, :]
            _close(fs[bi, h], fs_ref, 1e-12, f"matrix form final state (b={bi}, h={h})")


def chunked_ssd(inp, Q):
    """Chunked evaluation of the same operator (independent of the oracle):
    intra-chunk masked (C B^T o L) X, inter-chunk state passing, C.h_prev."""
    x, B, C = inp["x"], inp["B"], inp["C"]
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros_like(x)
    fs = np.zeros((b, H, P, N))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            dt = _softplus(inp["dt_raw"][bi, :, h] + inp["dt_bias"][h])
            a = dt * inp["A"][h]
            hs = np.zeros((P, N)) if inp["init_state"] is None else inp["init_state"][bi, h].copy()
            for s0 in range(0, L, Q):
                s1 = min(L, s0 + Q)
                cum = np.cumsum(a[s0:s1])
                seg = cum[:, None] - cum[None, :]
                Lm = np.where(np.tril(np.ones_like(seg)) > 0, np.exp(np.minimum(seg, 0.0)), 0.0)
                Xc, Bc, Cc = x[bi, s0:s1, h, :], B[bi, s0:s1, g, :], C[bi, s0:s1, g, :]
                Gm = Cc @ Bc.T
                y_diag = (Gm * Lm * dt[None, s0:s1]) @ Xc
                y_off = np.exp(cum)[:, None] * (Cc @ hs.T)
                y[bi, s0:s1, h, :] = y_diag + y_off + inp["D"][h] * Xc
                wj = np.exp(cum[-1] - cum) * dt[s0:s1]
                hs = math.exp(cum[-1]) * hs + (Xc * wj[:, None]).T @ Bc
            fs[bi, h] = hs
    return y, fs


def check_chunk_size_invariance():
    """The chunked form at chunk 1, 8, 64 and L (incl. a ragged last chunk)
    equals the oracle's token-by-token recurrence to rounding."""
    inp = _random_scan_inputs(_rng(6), b=1, L=200, H=2, P=4, N=8, G=1)
    y, fs = _scan(inp)
    for Q in (1, 8, 64, 200, 256):
        yc, fc = chunked_ssd(inp, Q)
        _close(y, yc, 1e-11, f"chunked Q={Q} y")
        _close(fs, fc, 1e-11, f"chunked Q={Q} final state")


# ----------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------

def check_linearity_in_x():
    """For fixed dt, B, C and zero initial state, y - D x is linear in x."""
    rng = _rng(7)
    inp = _random_scan_inputs(rng, init=False)
    x1 = inp["x"]
    x2 = rng.standard_normal(x1.shape)
    Dx = lambda x: inp["D"][None, None, :, None] * x
    f = lambda x: _scan(dict(inp, x=x))[0] - Dx(x)
    _close(f(x1 + 2.5 * x2), f(x1) + 2.5 * f(x2), 1e-12, "linearity")


def check_causality():
    """Changing any input at time >= t0 leaves y[:t0] bit-identical."""
    rng = _rng(8)
    inp = _random_scan_inputs(rng)
    y, _ = _scan(inp)
    t0 = 21
    pert = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
    for key in ("x", "B", "C", "dt_raw"):
        pert[key][:, t0:] += rng.standard_normal(pert[key][:, t0:].shape)
    y2, _ = _scan(pert)
    assert np.array_equal(y[:, :t0], y2[:, :t0]), "causality"
    assert not np.allclose(y[:, t0:], y2[:, t0:]), "later outputs must change"


def check_state_handoff():
    """scan(0..L) equals scan(0..t) followed by scan(t..L) started from the
    first call's final state."""
    inp = _random_scan_inputs(_rng(9), L=50)
    y, fs = _scan(inp)
    t = 17
    first = {k: (v[:, :t] if k in ("x", "B", "C", "dt_raw") else v) for k, v in inp.items()}
    ya, fa = _scan(first)
    second = {k: (v[:, t:] if k in ("x", "B", "C", "dt_raw") else v) for k, v in inp.items()}
    second["init_state"] = fa
    yb, fb = _scan(second)
    _close(np.concatenate([ya, yb], axis=1), y, 1e-13, "hand-off y")
    _close(fb, fs, 1e-13, "hand-off final state")


def check_decode_step_extends_prefill():
    """prefill(L) then one decode step equals prefill(L+1)."""
    inp = _random_scan_inputs(_rng(10), L=30)
    y, fs = _scan(inp)
    L = 29
    pre = {k: (v[:, :L] if k in ("x", "B", "C", "dt_raw") else v) for k, v in inp.items()}
    _, f_pre = _scan(pre)
    yd, fd = oracle.state_update(f_pre, inp["x"][:, L], inp["B"][:, L], inp["C"][:, L],
                                 inp["dt_raw"][:, L], inp["A"], inp["dt_bias"], inp["D"])
    _close(yd, y[:, L], 1e-13, "decode y")
    _close(fd, fs, 1e-13, "decode state")


def check_conv_state_handoff():
    """conv over [0, L) equals conv over [0, t) then [t, L) carrying the cache,
    including calls shorter than the conv width."""
    rng = _rng(11)
    b, L, cd, k = 2, 13, 6, 4
    xbc = rng.standard_normal((b, L, cd))
    w = rng.standard_normal((cd, k))
    bias = rng.standard_normal(cd)
    st0 = rng.standard_normal((b, cd, k))
    u, st = oracle.conv1d_silu(xbc, w, bias, st0)
    cur = st0
    pieces = []
    for (s0, s1) in [(0, 2), (2, 3), (3, 9), (9, 13)]:
        part, cur = oracle.conv1d_silu(xbc[:, s0:s1], w, bias, cur)
        pieces.append(part)
    _close(np.concatenate(pieces, axis=1), u, 1e-15, "conv hand-off output")
    _close(cur, st, 0.0, "conv hand-off cache")


def check_cache_size_formula():
    """Appendix C: a Mamba layer caches d_ssm*d_state + N_conv*(2*d_state + d_ssm)
    values (one group).  The oracle's SSM state [H,P,N] and conv cache
    [conv_dim, k] per sequence must hold exactly that many."""
    H, P, N, G, k = 3, 4, 5, 1, 4
    inp = _random_scan_inputs(_rng(12), b=1, L=3, H=H, P=P, N=N, G=G)
    _, fs = _scan(inp)
    cd = H * P + 2 * G * N
    _, cs = oracle.conv1d_silu(np.zeros((1, 2, cd)), np.zeros((cd, k)), None, np.zeros((1, cd, k)))
    d_ssm, d_state = H * P, N
    assert fs[0].size + cs[0].size == d_ssm * d_state + k * (2 * d_state + d_ssm)


def check_varlen_matches_each_sequence_alone():
    """A ragged batch (lengths 13, 0, 40, 1, 7, 0: empty sequences inside and
    at the end) equals the independent chunked evaluation of each sequence
    alone from its own initial state; an empty sequence's final state is its
    initial state."""
    rng = _rng(21)
    lens = [13, 0, 40, 1, 7, 0]
    T, H, P, N, G = sum(lens), 4, 3, 5, 2
    inp = _random_scan_inputs(rng, b=1, L=T, H=H, P=P, N=N, G=G, init=False)
    x, B, C, dt_raw = inp["x"][0], inp["B"][0], inp["C"][0], inp["dt_raw"][0]
    h0 = rng.standard_normal((len(lens), H, P, N)) * 0.3
    cu = np.concatenate([[0], np.cumsum(lens)])
    y, fs = oracle.selective_scan_varlen(x, B, C, dt_raw, inp["A"], cu, inp["dt_bias"], inp["D"], h0,
                                         nthreads=2)
    for s in range(len(lens)):
        a, b = int(cu[s]), int(cu[s + 1])
        if a == b:
            assert np.array_equal(fs[s], h0[s]), f"empty sequence {s}: final state is not its initial state"
            continue
        one = dict(x=x[None, a:b], B=B[None, a:b], C=C[None, a:b], dt_raw=dt_raw[None, a:b],
                   dt_bias=inp["dt_bias"], A=inp["A"], D=inp["D"], init_state=h0[s:s + 1])
        yr, fr = chunked_ssd(one, Q=8)
        _close(y[a:b], yr[0], 1e-12, f"ragged y (sequence {s})")
        _close(fs[s], fr[0], 1e-12, f"ragged final state (sequence {s})")


def check_varlen_chunked_prefill():
    """A sequence prefilled as two ragged calls, the second from the first
    call's final state, equals one call on the whole sequence."""
    rng = _rng(22)
    L, t = 50, 23
    inp = _random_scan_inputs(rng, b=1, L=L)
    x, B, C, dt_raw, h0 = inp["x"][0], inp["B"][0], inp["C"][0], inp["dt_raw"][0], inp["init_state"]
    y, fs = oracle.selective_scan_varlen(x, B, C, dt_raw, inp["A"], [0, L], inp["dt_bias"], inp["D"], h0)
    ya, fa = oracle.selective_scan_varlen(x[:t], B[:t], C[:t], dt_raw[:t], inp["A"], [0, t], inp["dt_bias"],
                                          inp["D"], h0)
    yb, fb = oracle.selective_scan_varlen(x[t:], B[t:], C[t:], dt_raw[t:], inp["A"], [0, L - t],
                                          inp["dt_bias"], inp["D"], fa)
    _close(np.concatenate([ya, yb]), y, 1e-13, "chunked prefill y")
    _close(fb, fs, 1e-13, "chunked prefill final state")


# ----------------------------------------------------------------------------
# backward pass
# ----------------------------------------------------------------------------

def _loss(inp, dy, dfinal):
    y, fs = oracle.selective_scan(inp["x"], inp["B"], inp["C"], inp["dt_raw"], inp["A"], inp["dt_bias"],
                                  inp["D"], inp["init_state"], nthreads=1)
    return float(np.sum(dy * y) + np.sum(dfinal * fs))


def _bwd(inp, dy, dfinal, nthreads=2):
    return oracle.selective_scan_bwd(inp["x"], inp["B"], inp["C"], inp["dt_raw"], inp["A"], dy,
                                     inp["dt_bias"], inp["D"], inp["init_state"], dfinal, nthreads=nthreads)


def check_bwd_finite_differences():
    """Every gradient element against a central difference of the forward
    oracle's loss sum(dy * y) + sum(dfinal * final_state), step 1e-6 (error
    O(1e-12) from the step, O(1e-10) from rounding)."""
    rng = _rng(31)
    inp = _random_scan_inputs(rng, b=2, L=7, H=4, P=3, N=4, G=2)
    y, fs = _scan(inp)
    dy = rng.standard_normal(y.shape)
    dfinal = rng.standard_normal(fs.shape)
    grads = _bwd(inp, dy, dfinal)
    names = {"x": "dx", "B": "dB", "C": "dC", "dt_raw": "ddt_raw", "A": "dA", "D": "dD",
             "dt_bias": "ddt_bias", "init_state": "dinit"}
    eps = 1e-6
    for key, gname in names.items():
        base = inp[key]
        fd = np.empty_like(base)
        for i in np.ndindex(base.shape):
            orig = base[i]
            base[i] = orig + eps
            lp = _loss(inp, dy, dfinal)
            base[i] = orig - eps
            lm = _loss(inp, dy, dfinal)
            base[i] = orig
            fd[i] = (lp - lm) / (2 * eps)
        _close(grads[gname], fd, 1e-7, f"gradient {gname} vs finite differences")


def check_bwd_dD_closed_form():
    """y depends on D only through D x: dLoss/dD_h = sum over (b, t, p) of dy x."""
    rng = _rng(32)
    inp = _random_scan_inputs(rng, b=2, L=20, H=4, P=5, N=6, G=2)
    dy = rng.standard_normal(inp["x"].shape)
    g = _bwd(inp, dy, None)
    _close(g["dD"], np.einsum("blhp,blhp->h", dy, inp["x"]), 1e-12, "dD closed form")


def check_bwd_dt_to_zero():
    """dt -> 0: the state stays h0, so dx = D dy, dB = 0,
    dC_t[g] = sum over the group's heads of h0^T dy_t, and dinit = dfinal +
    sum_t C_t dy_t^T."""
    rng = _rng(33)
    inp = _random_scan_inputs(rng, b=1, L=9, H=4, P=3, N=5, G=2)
    inp["dt_raw"] = np.full_like(inp["dt_raw"], -40.0)
    inp["dt_bias"] = np.zeros_like(inp["dt_bias"])
    dy = rng.standard_normal(inp["x"].shape)
    dfinal = rng.standard_normal(inp["init_state"].shape)
    g = _bwd(inp, dy, dfinal)
    H, G = 4, 2
    grp = np.arange(H) // (H // G)
    _close(g["dx"], inp["D"][None, None, :, None] * dy, 1e-12, "dt->0 dx")
    _close(g["dB"], np.zeros_like(g["dB"]), 1e-12, "dt->0 dB")
    dC = np.zeros_like(g["dC"])
    for h in range(H):
        dC[:, :, grp[h], :] += np.einsum("blp,bpn->bln", dy[:, :, h, :], inp["init_state"][:, h])
    _close(g["dC"], dC, 1e-12, "dt->0 dC")
    Cg = inp["C"][:, :, grp, :]
    _close(g["dinit"], dfinal + np.einsum("blhp,blhn->bhpn", dy, Cg), 1e-12, "dt->0 dinit")


def check_bwd_linear_in_output_gradients():
    """The gradients are linear in (dy, dfinal)."""
    rng = _rng(34)
    inp = _random_scan_inputs(rng, b=1, L=15, H=2, P=4, N=3, G=1)
    y, fs = _scan(inp)
    d1, d2 = rng.standard_normal(y.shape), rng.standard_normal(y.shape)
    f1, f2 = rng.standard_normal(fs.shape), rng.standard_normal(fs.shape)
    g1, g2 = _bwd(inp, d1, f1), _bwd(inp, d2, f2)
    g12 = _bwd(inp, 2.0 * d1 - 0.5 * d2, 2.0 * f1 - 0.5 * f2)
    for k in g1:
        _close(g12[k], 2.0 * g1[k] - 0.5 * g2[k], 1e-12, f"linearity {k}")


def _chunked_bwd(inp, dy, dfinal, Q):
    """The backward pass evaluated chunk by chunk in matrix form (state-space
    duality applied to the gradient; written independently of the oracle's
    token loop).  Per chunk with entering state h0 and incoming state
    gradient g_end, cum = inclusive cumsum of dt A, Lm[i, j] = exp(cum_i -
    cum_j) for j <= i:
      dC  = diag(e^cum) dY h0 + (Lm o dt_j o dY X^T) B
      gB  = diag(e^(cum_last - cum)) B g_end^T + (Lm^T o (C B^T)^T) dY      (g_j B_j per token)
      U   = diag(e^(cum_last - cum)) X g_end + (Lm^T o (dY X^T)^T) C         (g_j^T x_j per token)
      dX  = D dY + diag(dt) gB,   dB = diag(dt) U,   ddt_explicit_j = U_j . B_j
      <g_t, exp(dt_t A) h_{t-1}> = <g_t, h_t> - dt_t U_t . B_t with
      <g_t, h_t> = e^cum_last <g_end, h0> + sum_{j<=t} e^(cum_last - cum_j) dt_j x_j^T g_end B_j
                   + sum_{k>=t} e^cum_k dy_k^T h0 C_k + sum_{k>=t, j<=t} W[k, j],
      W = Lm o dt_j o (dY X^T) o (C B^T), the last sum by a running update
    and the entering state's gradient e^cum_last g_end + sum_k e^cum_k dy_k C_k^T
    becomes the previous chunk's g_end."""
    x, B, C, dt_raw, A, Dv = inp["x"], inp["B"], inp["C"], inp["dt_raw"], inp["A"], inp["D"]
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    grp = np.arange(H) // (H // G)
    v = dt_raw + inp["dt_bias"][None, None, :]
    dt = np.logaddexp(0.0, v)
    sig = 1.0 / (1.0 + np.exp(-v))
    out = dict(dx=np.zeros_like(x), dB=np.zeros_like(B), dC=np.zeros_like(C), ddt_raw=np.zeros_like(dt_raw),
               dA=np.zeros(H), dD=np.zeros(H), ddt_bias=np.zeros(H), dinit=np.zeros((b, H, P, N)))
    starts = list(range(0, L, Q))
    for bi in range(b):
        for h in range(H):
            g_ = grp[h]
            h0s = []
            hcur = inp["init_state"][bi, h].copy() if inp["init_state"] is not None else np.zeros((P, N))
            for s0 in starts:                          # forward: the state entering each chunk
                h0s.append(hcur)
                sl = slice(s0, min(L, s0 + Q))
                cum = np.cumsum(dt[bi, sl, h] * A[h])
                w = np.exp(cum[-1] - cum) * dt[bi, sl, h]
                hcur = np.exp(cum[-1]) * hcur + (x[bi, sl, h].T * w) @ B[bi, sl, g_]
            gend = dfinal[bi, h].copy() if dfinal is not None else np.zeros((P, N))
            for ci in reversed(range(len(starts))):   # backward over chunks
                sl = slice(starts[ci], min(L, starts[ci] + Q))
                h0 = h0s[ci]
                X, Bc, Cc, dY, dtc = x[bi, sl, h], B[bi, sl, g_], C[bi, sl, g_], dy[bi, sl, h], dt[bi, sl, h]
                cum = np.cumsum(dtc * A[h])
                q = len(dtc)
                Lm = np.tril(np.exp(cum[:, None] - cum[None, :]))
                YX = dY @ X.T
                CB = Cc @ Bc.T
                el = np.exp(cum[-1] - cum)
                dCc = np.exp(cum)[:, None] * (dY @ h0) + (Lm * dtc[None, :] * YX) @ Bc
                gB = el[:, None] * (Bc @ gend.T) + (Lm.T * CB.T) @ dY
                U = el[:, None] * (X @ gend) + (Lm.T * YX.T) @ Cc
                dX = Dv[h] * dY + dtc[:, None] * gB
                W = Lm * dtc[None, :] * YX * CB
                S = np.empty(q)
                run = 0.0
                for t in range(q):                     # sum over k >= t, j <= t of W[k, j]
                    run += W[t:, t].sum() - (W[t - 1, :t].sum() if t > 0 else 0.0)
                    S[t] = run
                t1 = np.exp(cum[-1]) * np.sum(gend * h0)
                t2 = np.cumsum(el * dtc * np.einsum("jp,pn,jn->j", X, gend, Bc))
                t3 = np.cumsum((np.exp(cum) * np.einsum("kp,pn,kn->k", dY, h0, Cc))[::-1])[::-1]
                ub = np.einsum("jn,jn->j", U, Bc)
                r = t1 + t2 + t3 + S - dtc * ub
                ddt = ub + A[h] * r
                out["dx"][bi, sl, h] = dX
                out["dB"][bi, sl, g_] += dtc[:, None] * U
                out["dC"][bi, sl, g_] += dCc
                out["ddt_raw"][bi, sl, h] = ddt * sig[bi, sl, h]
                out["dA"][h] += np.sum(dtc * r)
                out["dD"][h] += np.sum(dY * X)
                gend = np.exp(cum[-1]) * gend + (dY.T * np.exp(cum)) @ Cc
            out["dinit"][bi, h] = gend
    out["ddt_bias"] = out["ddt_raw"].sum(axis=(0, 1))
    return out


def check_bwd_chunked_matrix_form():
    """The oracle's token-loop gradients equal the chunked matrix form at
    chunk lengths 1, 3, 8 and L (the dual evaluation of the backward pass)."""
    rng = _rng(36)
    inp = _random_scan_inputs(rng, b=2, L=17, H=4, P=3, N=5, G=2)
    y, fs = _scan(inp)
    dy = rng.standard_normal(y.shape)
    dfinal = rng.standard_normal(fs.shape)
    ref = _bwd(inp, dy, dfinal)
    for Q in (1, 3, 8, 17):
        got = _chunked_bwd(inp, dy, dfinal, Q)
        for k in ref:
            _close(ref[k], got[k], 1e-11, f"chunk {Q}: {k}")


def check_bwd_thread_count_invariance():
    rng = _rng(35)
    inp = _random_scan_inputs(rng, b=3, L=11, H=4, P=3, N=4, G=2)
    dy = rng.standard_normal(inp["x"].shape)
    a, b = _bwd(inp, dy, None, nthreads=1), _bwd(inp, dy, None, nthreads=5)
    for k in a:
        assert np.array_equal(a[k], b[k]), f"{k} depends on the thread count"


# ----------------------------------------------------------------------------
# the mixer: gated RMSNorm and the two projections
# ----------------------------------------------------------------------------

def check_gated_norm_hand_worked():
    """y = (3, 4), z = (1, -1), weight (1, 2), eps 0:
    SiLU(1) = 1/(1 + e^-1), SiLU(-1) = -1/(1 + e); g = y SiLU(z);
    n = g / sqrt((g0^2 + g1^2) / 2) times the weight."""
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    sm1 = -1.0 / (1.0 + math.e)
    g0, g1 = 3.0 * s1, 4.0 * sm1
    r = math.sqrt((g0 * g0 + g1 * g1) / 2.0)
    want = np.array([g0 / r, 2.0 * g1 / r])
    got = oracle.rmsnorm_gated(np.array([3.0, 4.0]), np.array([1.0, -1.0]), np.array([1.0, 2.0]), 1, 0.0)
    _close(got, want, 1e-14, "gated norm, hand-worked")


def check_silu_matches_library_logistic():
    from scipy.special import expit
    v = np.linspace(-30.0, 30.0, 1201)
    _close(oracle.silu(v), v * expit(v), 1e-15, "SiLU vs v * expit(v)")


def check_gated_norm_invariants():
    rng = _rng(41)
    y = rng.standard_normal((3, 5, 24))
    z = rng.standard_normal((3, 5, 24))
    ones = np.ones(24)
    # unit mean square per slice (weight 1, eps 0), whatever the grouping
    for groups in (1, 3, 8):
        n = oracle.rmsnorm_gated(y, z, ones, groups, 0.0).reshape(3, 5, groups, 24 // groups)
        _close(np.mean(n * n, axis=-1), np.ones((3, 5, groups)), 1e-13, f"unit mean square, {groups} groups")
    # scale invariance in y (eps 0)
    w = rng.standard_normal(24)
    _close(oracle.rmsnorm_gated(7.5 * y, z, w, 4, 0.0), oracle.rmsnorm_gated(y, z, w, 4, 0.0), 1e-13,
           "scale invariance")
    # a grouped norm is the one-group norm of each slice, with the library norm
    g = y * oracle.silu(z)
    eps = 1e-2
    want = np.concatenate([g[..., k:k + 8] / np.sqrt(np.linalg.norm(g[..., k:k + 8], axis=-1, keepdims=True) ** 2 / 8
                                                        + eps) for k in range(0, 24, 8)], axis=-1) * w
    _close(oracle.rmsnorm_gated(y, z, w, 3, eps), want, 1e-13, "grouped norm vs slices")


def _tiny_mixer(rng, b=2, L=40, d_model=7, H=2, P=3, G=1, N=4, k=4):
    d_inner = H * P
    conv_dim = d_inner + 2 * G * N
    return dict(hidden=rng.standard_normal((b, L, d_model)),
                W_in=rng.standard_normal((d_inner + conv_dim + H, d_model)) / math.sqrt(d_model),
                conv_w=rng.standard_normal((conv_dim, k)) * 0.5, conv_bias=rng.standard_normal(conv_dim) * 0.3,
                dt_bias=rng.standard_normal(H) * 0.5 - 1.0, A=-np.exp(rng.uniform(0.0, 2.0, H)),
                D=rng.standard_normal(H), norm_w=rng.standard_normal(d_inner),
                W_out=rng.standard_normal((d_model, d_inner)) / math.sqrt(d_inner), H=H, P=P, G=G, N=N)


def check_mixer_projection_wiring():
    """in_proj with a permutation matrix must hand the path the permuted input
    columns (z, then xBC, then dt_raw, read by explicit indexing), and
    out_proj must be out[m] = sum_k n[k] W_out[m][k] (an explicit loop)."""
    rng = _rng(43)
    H, P, G, N = 2, 3, 1, 4
    d_inner, conv_dim = H * P, H * P + 2 * G * N
    dproj = d_inner + conv_dim + H
    t = _tiny_mixer(rng, d_model=dproj, H=H, P=P, G=G, N=N)
    perm = rng.permutation(dproj)
    W_in = np.zeros((dproj, dproj))
    W_in[np.arange(dproj), perm] = 1.0          # row j picks input column perm[j]
    t["W_in"] = W_in
    hid = t["hidden"]
    cs0 = rng.standard_normal((hid.shape[0], conv_dim, 4))
    zxbcdt = hid[..., perm]
    z, xBC, dt_raw = zxbcdt[..., :d_inner], zxbcdt[..., d_inner:d_inner + conv_dim], zxbcdt[..., -H:]
    y, fs, cs = oracle.layer_prefill(np.ascontiguousarray(xBC), t["conv_w"], t["conv_bias"], cs0,
                                     np.ascontiguousarray(dt_raw), t["A"], t["dt_bias"], t["D"], None, H, P, G, N)
    n = oracle.rmsnorm_gated(y.reshape(y.shape[0], y.shape[1], d_inner), z, t["norm_w"])
    want = np.zeros(hid.shape[:2] + (dproj,))
    for m in range(dproj):
        for kk in range(d_inner):
            want[..., m] += n[..., kk] * t["W_out"][m, kk]
    out, fs2, cs2 = oracle.mixer_forward(hid, W_in, t["conv_w"], t["conv_bias"], t["dt_bias"], t["A"], t["D"],
                                         t["norm_w"], t["W_out"], H, P, G, N, conv_state=cs0)
    _close(out, want, 1e-12, "mixer output vs explicit wiring")
    _close(fs2, fs, 1e-13, "mixer final state")
    _close(cs2, cs, 0.0, "mixer conv state")


ALL_CHECKS = [
    check_dt_to_zero,
    check_geometric_series,
    check_hand_worked,
    check_conv_identity_tap,
    check_conv_matches_np_convolve,
    check_matrix_form,
    check_chunk_size_invariance,
    check_linearity_in_x,
    check_causality,
    check_state_handoff,
    check_decode_step_extends_prefill,
    check_conv_state_handoff,
    check_cache_size_formula,
    check_varlen_matches_each_sequence_alone,
    check_varlen_chunked_prefill,
    check_bwd_finite_differences,
    check_bwd_dD_closed_form,
    check_bwd_dt_to_zero,
    check_bwd_linear_in_output_gradients,
    check_bwd_thread_count_invariance,
    check_bwd_chunked_matrix_form,
    check_gated_norm_hand_worked,
    check_silu_matches_library_logistic,
    check_gated_norm_invariants,
    check_mixer_projection_wiring,
]
