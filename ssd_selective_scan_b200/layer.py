"""Torch-facing calls over the libssd C ABI.

PyTorch is plumbing here: it allocates device memory and supplies the current
CUDA stream.  Each function checks tensor shapes, allocates the outputs,
passes raw pointers to the C entry point of the same name (``libssd``) and
raises ``SsdError`` on any non-OK status.  All arithmetic runs in the CUDA
kernels of libssd.so.
"""
from __future__ import annotations

import torch

from . import binding as libssd

_DT = {torch.float32: libssd.SSD_F32, torch.bfloat16: libssd.SSD_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported I/O dtype {t.dtype}; use float32 or bfloat16")
    return _DT[t.dtype]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _f32(t, name):
    if t is None:
        return None
    if t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    return t


def conv1d_silu(xBC: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None = None,
                conv_state: torch.Tensor | None = None, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """Causal depthwise conv1d + SiLU.  xBC [b, L, conv_dim]; w [conv_dim, k] f32;
    conv_state [b, conv_dim, k] (updated in place).  Returns out."""
    if xBC.dim() != 3 or not xBC.is_contiguous():
        raise ValueError("xBC must be a contiguous [b, L, conv_dim] tensor")
    b, L, cd = xBC.shape
    k = w.shape[1]
    if out is None:
        out = torch.empty_like(xBC)
    if conv_state is not None and (conv_state.shape != (b, cd, k) or conv_state.dtype != xBC.dtype
                                   or not conv_state.is_contiguous()):
        raise ValueError("conv_state must be a contiguous [b, conv_dim, k] tensor of xBC's dtype")
    st = libssd.ssd_conv1d_silu(_ptr(xBC), _ptr(out), _ptr(_f32(w, "w")), _ptr(_f32(bias, "bias")),
                                _ptr(conv_state), b, L, cd, k, _dtype_code(xBC), _stream(stream))
    libssd.check("ssd_conv1d_silu", st)
    return out


def _row_view_stride(t: torch.Tensor, name: str) -> int:
    """Row stride (elements between consecutive tokens) of a [b, L, heads, dim]
    view whose tokens are evenly spaced and whose inner dims are dense."""
    b, L, nh, d = t.shape
    s = t.stride()
    if s[3] != 1 or s[2] != d or (b > 1 and s[0] != L * s[1]):
        raise ValueError(f"{name}: expected inner-dense [b, L, {nh}, {d}] with uniform token stride")
    return s[1]


def chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, dtype: torch.dtype) -> int:
    return int(libssd.ssd_chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, _DT[dtype]))


def chunk_scan_fwd(x: torch.Tensor, B: torch.Tensor, C: torch.Tensor, dt_raw: torch.Tensor,
                   A: torch.Tensor, dt_bias: torch.Tensor | None = None,
                   D: torch.Tensor | None = None, init_state: torch.Tensor | None = None,
                   Q: int = 128, y: torch.Tensor | None = None,
                   final_state: torch.Tensor | bool | None = True,
                   workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                   stream=None):
    """Chunked SSD scan.  x [b, L, H, P], B/C [b, L, G, N] (views sharing one
    token stride, e.g. channel ranges of the conv output), dt_raw [b, L, H].
    Returns (y [b, L, H, P], final_state [b, H, P, N] f32 or None)."""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if b * L == 0:
        # no tokens: strides of empty views are meaningless; any valid one will do
        rs = -(-max(H * P, G * N) // 8) * 8
    else:
        rs = _row_view_stride(x, "x")
        if _row_view_stride(B, "B") != rs or _row_view_stride(C, "C") != rs:
            raise ValueError("x, B and C must share one token stride")
    if B.dtype != x.dtype or C.dtype != x.dtype or dt_raw.dtype != x.dtype:
        raise ValueError("x, B, C, dt_raw must share the I/O dtype")
    if dt_raw.shape != (b, L, H) or not dt_raw.is_contiguous():
        raise ValueError("dt_raw must be a contiguous [b, L, H] tensor")
    if y is None:
        y = torch.empty((b, L, H, P), dtype=x.dtype, device=x.device)
    if final_state is True:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=x.device)
    elif final_state is False:
        final_state = None
    need = chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, x.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = libssd.ssd_chunk_scan_fwd(
        _ptr(x), _ptr(B), _ptr(C), rs, _ptr(dt_raw), _ptr(_f32(dt_bias, "dt_bias")),
        _ptr(_f32(A, "A")), _ptr(_f32(D, "D")), _ptr(_f32(init_state, "init_state")), _ptr(y),
        _ptr(final_state), b, L, H, P, N, G, Q, _dtype_code(x), _ptr(workspace), ws_bytes,
        _ptr(status), _stream(stream))
    libssd.check("ssd_chunk_scan_fwd", st)
    return y, final_state


def chunk_scan_varlen_workspace_bytes(nseq, T, H, P, N, G, Q, dtype: torch.dtype) -> int:
    return int(libssd.ssd_chunk_scan_varlen_workspace_bytes(nseq, T, H, P, N, G, Q, _DT[dtype]))


def chunk_scan_fwd_varlen(x: torch.Tensor, B: torch.Tensor, C: torch.Tensor, dt_raw: torch.Tensor,
                          A: torch.Tensor, cu_seqlens: torch.Tensor, dt_bias: torch.Tensor | None = None,
                          D: torch.Tensor | None = None, init_state: torch.Tensor | None = None,
                          Q: int = 128, y: torch.Tensor | None = None,
                          final_state: torch.Tensor | bool | None = True,
                          workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                          stream=None):
    """Chunked SSD scan of a ragged batch packed along the token dimension.
    x [T, H, P], B/C [T, G, N] (views sharing one token stride), dt_raw
    [T, H]; cu_seqlens int32 [nseq + 1] on the device (sequence s is tokens
    cu_seqlens[s] .. cu_seqlens[s+1]-1); init_state [nseq, H, P, N] or None.
    Returns (y [T, H, P], final_state [nseq, H, P, N] f32 or None).  A bad
    cu_seqlens is reported in `status` (allocated here if not given), which
    the caller reads after synchronising."""
    T, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 vector")
    nseq = cu_seqlens.numel() - 1
    if T == 0:
        rs = -(-max(H * P, G * N) // 8) * 8
    else:
        rs = x.stride(0)
        if x.stride(2) != 1 or x.stride(1) != P:
            raise ValueError("x must be [T, H, P] with contiguous (H, P) rows")
        for t, name in ((B, "B"), (C, "C")):
            if t.stride(0) != rs or t.stride(2) != 1 or t.stride(1) != N:
                raise ValueError(f"{name} must share x's token stride with contiguous (G, N) rows")
    if B.dtype != x.dtype or C.dtype != x.dtype or dt_raw.dtype != x.dtype:
        raise ValueError("x, B, C, dt_raw must share the I/O dtype")
    if dt_raw.shape != (T, H) or not dt_raw.is_contiguous():
        raise ValueError("dt_raw must be a contiguous [T, H] tensor")
    if y is None:
        y = torch.empty((T, H, P), dtype=x.dtype, device=x.device)
    if final_state is True:
        final_state = torch.empty((nseq, H, P, N), dtype=torch.float32, device=x.device)
    elif final_state is False:
        final_state = None
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=x.device)
    need = chunk_scan_varlen_workspace_bytes(nseq, T, H, P, N, G, Q, x.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = libssd.ssd_chunk_scan_fwd_varlen(
        _ptr(x), _ptr(B), _ptr(C), rs, _ptr(dt_raw), _ptr(_f32(dt_bias, "dt_bias")),
        _ptr(_f32(A, "A")), _ptr(_f32(D, "D")), _ptr(_f32(init_state, "init_state")), _ptr(y),
        _ptr(final_state), _ptr(cu_seqlens), nseq, T, H, P, N, G, Q, _dtype_code(x), _ptr(workspace),
        ws_bytes, _ptr(status), _stream(stream))
    libssd.check("ssd_chunk_scan_fwd_varlen", st)
    return y, final_state


def state_update(state: torch.Tensor, x: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
                 dt_raw: torch.Tensor, A: torch.Tensor, dt_bias: torch.Tensor | None = None,
                 D: torch.Tensor | None = None, y: torch.Tensor | None = None, stream=None):
    """One decode token, state [b, H, P, N] f32 updated in place.  x [b, H, P],
    B/C [b, G, N] views sharing one batch stride (e.g. channel ranges of the
    conv output), dt_raw [b, H].  Returns y [b, H, P]."""
    b, H, P, N = state.shape
    G = B.shape[1]
    _f32(state, "state")
    rs = x.stride(0)
    for t, nm, d in ((x, "x", P), (B, "B", N), (C, "C", N)):
        if t.stride(-1) != 1 or t.stride(-2) != d or (b > 1 and t.stride(0) != rs):
            raise ValueError(f"{nm}: inner-dense view with the shared batch stride expected")
    if y is None:
        y = torch.empty((b, H, P), dtype=x.dtype, device=x.device)
    st = libssd.ssd_state_update(_ptr(state), _ptr(x), _ptr(B), _ptr(C), rs, _ptr(dt_raw),
                                 _ptr(_f32(dt_bias, "dt_bias")), _ptr(_f32(A, "A")),
                                 _ptr(_f32(D, "D")), _ptr(y), b, H, P, N, G, _dtype_code(x),
                                 _stream(stream))
    libssd.check("ssd_state_update", st)
    return y


def chunk_scan_bwd_workspace_bytes(b, L, H, P, N, G, dtype: torch.dtype) -> int:
    return int(libssd.ssd_chunk_scan_bwd_workspace_bytes(b, L, H, P, N, G, _DT[dtype]))


def chunk_scan_bwd(x: torch.Tensor, B: torch.Tensor, C: torch.Tensor, dt_raw: torch.Tensor,
                   A: torch.Tensor, dy: torch.Tensor, dt_bias: torch.Tensor | None = None,
                   D: torch.Tensor | None = None, init_state: torch.Tensor | None = None,
                   dfinal: torch.Tensor | None = None, want_dinit: bool = True,
                   workspace: torch.Tensor | None = None, stream=None) -> dict:
    """Gradients through chunk_scan_fwd.  x, B, C, dt_raw, A, dt_bias, D,
    init_state as for the forward call; dy [b, L, H, P] (I/O dtype), dfinal
    [b, H, P, N] f32 or None.  Returns dict(dx, dB, dC, ddt_raw, dA, dD,
    ddt_bias, dinit): dB, dC [b, L, G, N] and ddt_raw in the I/O dtype, the
    parameter gradients f32 [H], dinit f32 [b, H, P, N] (None if not wanted)."""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if b * L == 0:
        rs = -(-max(H * P, G * N) // 8) * 8
    else:
        rs = _row_view_stride(x, "x")
        if _row_view_stride(B, "B") != rs or _row_view_stride(C, "C") != rs:
            raise ValueError("x, B and C must share one token stride")
    if dy.shape != (b, L, H, P) or dy.dtype != x.dtype or not dy.is_contiguous():
        raise ValueError("dy must be a contiguous [b, L, H, P] tensor of x's dtype")
    if dt_raw.shape != (b, L, H) or dt_raw.dtype != x.dtype or not dt_raw.is_contiguous():
        raise ValueError("dt_raw must be a contiguous [b, L, H] tensor of x's dtype")
    dev, dt = x.device, x.dtype
    out = dict(dx=torch.empty((b, L, H, P), dtype=dt, device=dev),
               dB=torch.empty((b, L, G, N), dtype=dt, device=dev),
               dC=torch.empty((b, L, G, N), dtype=dt, device=dev),
               ddt_raw=torch.empty((b, L, H), dtype=dt, device=dev),
               dA=torch.empty(H, dtype=torch.float32, device=dev),
               dD=torch.empty(H, dtype=torch.float32, device=dev),
               ddt_bias=torch.empty(H, dtype=torch.float32, device=dev),
               dinit=torch.empty((b, H, P, N), dtype=torch.float32, device=dev) if want_dinit else None)
    need = chunk_scan_bwd_workspace_bytes(b, L, H, P, N, G, dt)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = libssd.ssd_chunk_scan_bwd(
        _ptr(x), _ptr(B), _ptr(C), rs, _ptr(dt_raw), _ptr(_f32(dt_bias, "dt_bias")), _ptr(_f32(A, "A")),
        _ptr(_f32(D, "D")), _ptr(_f32(init_state, "init_state")), _ptr(dy), _ptr(_f32(dfinal, "dfinal")),
        _ptr(out["dx"]), _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["ddt_raw"]), _ptr(out["dA"]),
        _ptr(out["dD"]), _ptr(out["ddt_bias"]), _ptr(out["dinit"]), b, L, H, P, N, G, _dtype_code(x),
        _ptr(workspace), ws_bytes, _stream(stream))
    libssd.check("ssd_chunk_scan_bwd", st)
    return out


def split_channels(u: torch.Tensor, H: int, P: int, G: int, N: int):
    """[.., conv_dim] -> views x [.., H, P], B [.., G, N], C [.., G, N]."""
    lead = u.shape[:-1]
    x = u[..., : H * P].unflatten(-1, (H, P))
    B = u[..., H * P: H * P + G * N].unflatten(-1, (G, N))
    C = u[..., H * P + G * N:].unflatten(-1, (G, N))
    assert x.shape[:-2] == lead
    return x, B, C


def conv_scan_workspace_bytes(b, L, H, P, N, G, Q, k, dtype: torch.dtype) -> int:
    return int(libssd.ssd_conv_scan_workspace_bytes(b, L, H, P, N, G, Q, k, _DT[dtype]))


def conv_scan_fwd(xBC: torch.Tensor, w: torch.Tensor, dt_raw: torch.Tensor, A: torch.Tensor,
                  H: int, P: int, G: int, N: int, *, bias: torch.Tensor | None = None,
                  conv_state: torch.Tensor | None = None, dt_bias: torch.Tensor | None = None,
                  D: torch.Tensor | None = None, init_state: torch.Tensor | None = None,
                  Q: int = 128, y: torch.Tensor | None = None,
                  final_state: torch.Tensor | bool | None = True,
                  workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                  stream=None):
    """The prefill layer in one call: conv1d+SiLU of xBC [b, L, conv_dim] into
    the workspace, then the chunked scan of its x | B | C channels.  w
    [conv_dim, k] f32; conv_state [b, conv_dim, k] (I/O dtype) is updated in
    place.  Returns (y [b, L, H, P], final_state [b, H, P, N] f32 or None)."""
    if xBC.dim() != 3 or not xBC.is_contiguous():
        raise ValueError("xBC must be a contiguous [b, L, conv_dim] tensor")
    b, L, cd = xBC.shape
    if cd != H * P + 2 * G * N:
        raise ValueError(f"xBC has {cd} channels, expected H*P + 2*G*N = {H * P + 2 * G * N}")
    k = w.shape[1]
    if w.shape != (cd, k):
        raise ValueError("w must be [conv_dim, k]")
    if conv_state is not None and (conv_state.shape != (b, cd, k) or conv_state.dtype != xBC.dtype
                                   or not conv_state.is_contiguous()):
        raise ValueError("conv_state must be a contiguous [b, conv_dim, k] tensor of xBC's dtype")
    if dt_raw.dtype != xBC.dtype or dt_raw.shape != (b, L, H) or not dt_raw.is_contiguous():
        raise ValueError("dt_raw must be a contiguous [b, L, H] tensor of xBC's dtype")
    if y is None:
        y = torch.empty((b, L, H, P), dtype=xBC.dtype, device=xBC.device)
    if final_state is True:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=xBC.device)
    elif final_state is False:
        final_state = None
    need = conv_scan_workspace_bytes(b, L, H, P, N, G, Q, k, xBC.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=xBC.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = libssd.ssd_conv_scan_fwd(
        _ptr(xBC), _ptr(_f32(w, "w")), _ptr(_f32(bias, "bias")), _ptr(conv_state), _ptr(dt_raw),
        _ptr(_f32(dt_bias, "dt_bias")), _ptr(_f32(A, "A")), _ptr(_f32(D, "D")),
        _ptr(_f32(init_state, "init_state")), _ptr(y), _ptr(final_state), b, L, H, P, N, G, Q, k,
        _dtype_code(xBC), _ptr(workspace), ws_bytes, _ptr(status), _stream(stream))
    libssd.check("ssd_conv_scan_fwd", st)
    return y, final_state


def layer_prefill(xBC, w, dt_raw, A, H, P, G, N, *, bias=None, conv_state=None, dt_bias=None,
                  D=None, init_state=None, Q=128, y=None, final_state=True, workspace=None,
                  stream=None):
    """The prefill layer (conv1d+SiLU, then the chunked scan) through the
    one-call entry point.  Returns (y, final_state); conv_state, if given, is
    updated in place."""
    return conv_scan_fwd(xBC, w, dt_raw, A, H, P, G, N, bias=bias, conv_state=conv_state,
                         dt_bias=dt_bias, D=D, init_state=init_state, Q=Q, y=y,
                         final_state=final_state, workspace=workspace, stream=stream)


def decode_step(xBC, w, conv_state, state, dt_raw, A, H, P, G, N, *, bias=None, dt_bias=None,
                D=None, y=None, workspace=None, stream=None):
    """One token per sequence in one kernel: conv-cache roll, conv + SiLU,
    then the state update.  xBC [b, conv_dim]; conv_state [b, conv_dim, k]
    and state [b, H, P, N] f32 updated in place.  Returns y [b, H, P].
    With `workspace` (int32, at least b * G elements, zero before its first
    use; the call leaves it zero) the step runs one CTA per (sequence, head)
    (ssd_decode_step_ws), else one per (sequence, group) (ssd_decode_step);
    the results are the same."""
    if xBC.dim() != 2 or not xBC.is_contiguous():
        raise ValueError("xBC must be a contiguous [b, conv_dim] tensor")
    b, cd = xBC.shape
    if cd != H * P + 2 * G * N:
        raise ValueError(f"xBC has {cd} channels, expected H*P + 2*G*N = {H * P + 2 * G * N}")
    k = w.shape[1]
    if w.shape != (cd, k):
        raise ValueError("w must be [conv_dim, k]")
    if conv_state.shape != (b, cd, k) or conv_state.dtype != xBC.dtype or not conv_state.is_contiguous():
        raise ValueError("conv_state must be a contiguous [b, conv_dim, k] tensor of xBC's dtype")
    if state.shape != (b, H, P, N):
        raise ValueError("state must be [b, H, P, N]")
    _f32(state, "state")
    if dt_raw.shape != (b, H) or dt_raw.dtype != xBC.dtype or not dt_raw.is_contiguous():
        raise ValueError("dt_raw must be a contiguous [b, H] tensor of xBC's dtype")
    if y is None:
        y = torch.empty((b, H, P), dtype=xBC.dtype, device=xBC.device)
    if workspace is not None:
        if workspace.dtype != torch.int32 or not workspace.is_contiguous() or workspace.device != xBC.device:
            raise ValueError("workspace must be a contiguous int32 tensor on xBC's device")
        st = libssd.ssd_decode_step_ws(_ptr(state), _ptr(conv_state), _ptr(xBC), _ptr(_f32(w, "w")),
                                       _ptr(_f32(bias, "bias")), _ptr(dt_raw), _ptr(_f32(dt_bias, "dt_bias")),
                                       _ptr(_f32(A, "A")), _ptr(_f32(D, "D")), _ptr(y), b, H, P, N, G, k,
                                       _dtype_code(xBC), _ptr(workspace), workspace.numel() * 4, _stream(stream))
        libssd.check("ssd_decode_step_ws", st)
        return y
    st = libssd.ssd_decode_step(_ptr(state), _ptr(conv_state), _ptr(xBC), _ptr(_f32(w, "w")),
                                _ptr(_f32(bias, "bias")), _ptr(dt_raw), _ptr(_f32(dt_bias, "dt_bias")),
                                _ptr(_f32(A, "A")), _ptr(_f32(D, "D")), _ptr(y), b, H, P, N, G, k,
                                _dtype_code(xBC), _stream(stream))
    libssd.check("ssd_decode_step", st)
    return y


def decode_step_workspace(b: int, G: int, device) -> torch.Tensor:
    """A zeroed workspace for decode_step(..., workspace=...)."""
    n = libssd.ssd_decode_step_workspace_bytes(b, G) // 4
    return torch.zeros(max(n, 1), dtype=torch.int32, device=device)


def linear(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None, status: torch.Tensor | None = None,
           stream=None) -> torch.Tensor:
    """y = x w^T on the tensor cores (bf16 in and out, fp32 accumulation).
    x [..., K] with a dense last dimension, w [N, K]; returns y [..., N]."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise TypeError("linear: bf16 operands expected")
    K = x.shape[-1]
    N = w.shape[0]
    if w.shape != (N, K) or w.stride(1) != 1 or x.stride(-1) != 1:
        raise ValueError("linear: x [..., K] and w [N, K] with contiguous rows expected")
    x2 = x.reshape(-1, K)
    M = x2.shape[0]
    if y is None:
        y = torch.empty((*x.shape[:-1], N), dtype=torch.bfloat16, device=x.device)
    y2 = y.view(-1, N)
    st = libssd.ssd_linear_bf16(_ptr(x2), x2.stride(0) if M else K, _ptr(w), w.stride(0), _ptr(y2),
                                y2.stride(0) if M else N, M, N, K, _ptr(status), _stream(stream))
    libssd.check("ssd_linear_bf16", st)
    return y


def mixer_workspace_bytes(b, L, d_model, H, P, N, G, Q, k) -> int:
    return int(libssd.ssd_mixer_workspace_bytes(b, L, d_model, H, P, N, G, Q, k, libssd.SSD_BF16))


def mixer_forward(hidden: torch.Tensor, W_in: torch.Tensor, conv_w: torch.Tensor, dt_bias: torch.Tensor | None,
                  A: torch.Tensor, D: torch.Tensor | None, norm_w: torch.Tensor, W_out: torch.Tensor,
                  H: int, P: int, G: int, N: int, *, conv_bias: torch.Tensor | None = None,
                  conv_state: torch.Tensor | None = None, init_state: torch.Tensor | None = None,
                  Q: int = 128, norm_groups: int = 1, eps: float = 1e-5, out: torch.Tensor | None = None,
                  final_state: torch.Tensor | bool | None = True, workspace: torch.Tensor | None = None,
                  status: torch.Tensor | None = None, stream=None):
    """The Mamba-2 mixer forward in one call (in_proj, conv1d+SiLU, chunked
    scan, gated RMSNorm, out_proj).  hidden [b, L, d_model] bf16; W_in
    [2HP + 2GN + H, d_model] bf16; conv_w [conv_dim, k] f32; norm_w [H P] f32;
    W_out [d_model, H P] bf16; conv_state [b, conv_dim, k] bf16 (updated in
    place).  Returns (out [b, L, d_model] bf16, final_state [b, H, P, N] f32
    or None)."""
    if hidden.dim() != 3 or not hidden.is_contiguous() or hidden.dtype != torch.bfloat16:
        raise ValueError("hidden must be a contiguous bf16 [b, L, d_model] tensor")
    b, L, d_model = hidden.shape
    d_inner = H * P
    conv_dim = d_inner + 2 * G * N
    k = conv_w.shape[1]
    if W_in.shape != (d_inner + conv_dim + H, d_model) or not W_in.is_contiguous():
        raise ValueError("W_in must be a contiguous [2HP + 2GN + H, d_model] tensor")
    if W_out.shape != (d_model, d_inner) or not W_out.is_contiguous():
        raise ValueError("W_out must be a contiguous [d_model, H P] tensor")
    if conv_state is not None and (conv_state.shape != (b, conv_dim, k) or conv_state.dtype != torch.bfloat16
                                   or not conv_state.is_contiguous()):
        raise ValueError("conv_state must be a contiguous bf16 [b, conv_dim, k] tensor")
    if out is None:
        out = torch.empty((b, L, d_model), dtype=torch.bfloat16, device=hidden.device)
    if final_state is True:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=hidden.device)
    elif final_state is False:
        final_state = None
    need = mixer_workspace_bytes(b, L, d_model, H, P, N, G, Q, k)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=hidden.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = libssd.ssd_mixer_fwd(
        _ptr(hidden), _ptr(W_in), _ptr(_f32(conv_w, "conv_w")), _ptr(_f32(conv_bias, "conv_bias")), _ptr(conv_state),
        _ptr(_f32(dt_bias, "dt_bias")), _ptr(_f32(A, "A")), _ptr(_f32(D, "D")), _ptr(_f32(norm_w, "norm_w")),
        _ptr(W_out), _ptr(_f32(init_state, "init_state")), _ptr(out), _ptr(final_state), b, L, d_model, H, P, N, G,
        Q, k, norm_groups, eps, libssd.SSD_BF16, _ptr(workspace), ws_bytes, _ptr(status), _stream(stream))
    libssd.check("ssd_mixer_fwd", st)
    return out, final_state
