"""C-ABI boundary on the host (no GPU needed): libssd.so loads, exports every
entry point include/ssd.h declares (and the binding covers exactly those), and
argument validation rejects bad calls before anything reaches the device.

Pointer arguments here are fake addresses that are never dereferenced: every
call below fails validation (or is empty work) before any CUDA call."""
import os
import re
import subprocess

import pytest

from ssd_selective_scan_b200 import build as ssd_build
from ssd_selective_scan_b200 import binding as libssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")

OK, INV, UNS = libssd.SSD_OK, libssd.SSD_ERR_INVALID_ARG, libssd.SSD_ERR_UNSUPPORTED
F32, BF16 = libssd.SSD_F32, libssd.SSD_BF16


@pytest.fixture(scope="module", autouse=True)
def built():
    ssd_build.build()
    libssd.load()


def declared_entry_points():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    assert declared_entry_points() == sorted([
        "ssd_abi_version", "ssd_chunk_scan_bwd", "ssd_chunk_scan_bwd_workspace_bytes",
        "ssd_chunk_scan_fwd", "ssd_chunk_scan_fwd_static",
        "ssd_chunk_scan_fwd_varlen", "ssd_chunk_scan_varlen_workspace_bytes",
        "ssd_chunk_scan_workspace_bytes", "ssd_conv1d_silu", "ssd_conv_scan_fwd",
        "ssd_conv_scan_workspace_bytes", "ssd_decode_step", "ssd_decode_step_workspace_bytes",
        "ssd_decode_step_ws", "ssd_linear_bf16", "ssd_mixer_fwd",
        "ssd_mixer_workspace_bytes", "ssd_selftest_bounded_wait", "ssd_state_update", "ssd_status_string"])


def test_library_exports_every_declared_symbol():
    out = subprocess.check_output(["nm", "-D", "--defined-only", libssd.LIB_PATH], text=True)
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = set(declared_entry_points()) - exported
    assert not missing, f"declared but not exported: {missing}"
    assert set(libssd.SIGNATURES) == set(declared_entry_points())
    lib = libssd.load()
    for name in declared_entry_points():
        assert hasattr(lib, name)


def test_version_and_status_strings():
    assert libssd.ssd_abi_version() == 1
    assert libssd.status_string(OK) == "SSD_OK"
    for s in (INV, UNS, libssd.SSD_ERR_CUDA, libssd.SSD_ERR_TIMEOUT):
        assert libssd.status_string(s).startswith("SSD_ERR_")
    assert libssd.status_string(99) == "SSD_ERR_UNKNOWN"


# fake, well-separated, 256-byte aligned device addresses (never dereferenced)
def fake(i, off=0):
    return 0x7f0000000000 + i * (1 << 32) + off


def conv(**kw):
    a = dict(xBC=fake(1), out=fake(2), w=fake(3), bias=None, conv_state=fake(4), b=2, L=16,
             conv_dim=64, k=4, dtype=BF16, stream=None)
    a.update(kw)
    return libssd.ssd_conv1d_silu(**a)


def test_conv_validation():
    assert conv(b=0) == OK and conv(L=0) == OK                      # empty work, no launch
    assert conv(xBC=None) == INV and conv(out=None) == INV and conv(w=None) == INV
    assert conv(b=0, xBC=None, out=None) == OK                       # empty work takes NULL
    assert conv(b=-1) == INV and conv(L=-1) == INV and conv(conv_dim=0) == INV
    assert conv(dtype=7) == INV
    assert conv(conv_dim=60) == INV                                  # not a multiple of 8 (bf16)
    assert conv(conv_dim=60, dtype=F32, b=0) == OK                   # multiple of 4 is fine for f32
    assert conv(xBC=fake(1, 8)) == INV and conv(conv_state=fake(4, 4)) == INV   # misaligned
    assert conv(out=fake(1, 64)) == INV                              # out overlaps xBC
    assert conv(conv_state=fake(2, 16)) == INV                       # cache overlaps out
    assert conv(k=5) == UNS and conv(k=1) == UNS


def scan(**kw):
    a = dict(x=fake(1), B=fake(1, 2560 * 2), C=fake(1, (2560 + 1024) * 2), row_stride=4608,
             dt_raw=fake(2), dt_bias=None, A=fake(3), D=fake(4), init_state=None, y=fake(5),
             final_state=fake(6), b=2, L=256, H=40, P=64, N=128, G=8, Q=128, dtype=BF16,
             workspace=None, workspace_bytes=0, status=None, stream=None)
    a.update(kw)
    if a["workspace"] is None and a["workspace_bytes"] == 0 and "workspace_bytes" not in kw:
        need = libssd.ssd_chunk_scan_workspace_bytes(a["b"], a["L"], a["H"], a["P"], a["N"],
                                                     a["G"], a["Q"], a["dtype"])
        if need:
            a["workspace"], a["workspace_bytes"] = fake(7), need
    return libssd.ssd_chunk_scan_fwd(**a)


def test_scan_validation():
    assert scan(b=0) == OK and scan(b=0, x=None, y=None, B=None, C=None, dt_raw=None) == OK
    for k in ("x", "B", "C", "dt_raw", "A", "y"):
        assert scan(**{k: None}) == INV, k
    assert scan(H=40, G=7) == INV                                    # H % G
    assert scan(P=60) == INV and scan(N=100) == INV                  # multiples of 8
    assert scan(Q=96) == INV and scan(Q=256) == INV
    assert scan(row_stride=4604) == INV                              # not a multiple of 8
    assert scan(row_stride=2048) == INV                              # shorter than H*P
    assert scan(x=fake(1, 2)) == INV and scan(y=fake(5, 8)) == INV   # misaligned
    assert scan(y=fake(1, 4096)) == INV                              # y overlaps x
    assert scan(final_state=fake(5, 1024)) == INV                    # final state overlaps y
    assert scan(init_state=fake(6, 512)) == INV                      # partial alias of final state
    assert scan(dtype=3) == INV and scan(L=-1) == INV and scan(H=0) == INV


def test_scan_workspace_query_and_check():
    # the shape of scan()'s defaults: every call below must fail validation
    need = libssd.ssd_chunk_scan_workspace_bytes(2, 256, 40, 64, 128, 8, 128, BF16)
    assert need > 0                                   # the tensor-core path takes scratch
    assert libssd.ssd_chunk_scan_workspace_bytes(2, 256, 4, 64, 16, 1, 64, F32) == 0
    assert libssd.ssd_chunk_scan_workspace_bytes(0, 256, 40, 64, 128, 8, 128, BF16) == 0
    if need:
        assert scan(workspace=None, workspace_bytes=need) == INV
        assert scan(workspace=fake(7), workspace_bytes=need - 1) == INV
        assert scan(workspace=fake(1, 64), workspace_bytes=need) == INV    # overlaps x


def su(**kw):
    a = dict(state=fake(1), x=fake(2), B=fake(2, 16384 * 2), C=fake(2, (16384 + 1024) * 2),
             row_stride=10240, dt_raw=fake(3), dt_bias=None, A=fake(4), D=fake(5), y=fake(6),
             b=4, H=128, P=64, N=128, G=8, dtype=BF16, stream=None)
    a.update(kw)
    return libssd.ssd_state_update(**a)


def test_state_update_validation():
    assert su(b=0) == OK
    for k in ("state", "x", "B", "C", "dt_raw", "A", "y"):
        assert su(**{k: None}) == INV, k
    assert su(G=3) == INV and su(N=6) == INV and su(P=0) == INV
    assert su(row_stride=100) == INV
    assert su(state=fake(1, 8)) == INV                               # state not 16-byte aligned
    assert su(x=fake(2, 1)) == INV                                   # x not element aligned
    assert su(y=fake(1, 64)) == INV                                  # y overlaps state
    assert su(state=fake(2, 64)) == INV                              # state overlaps x
    assert su(N=512) == UNS and su(N=12) == UNS                      # no kernel for these N


def test_selftest_validation():
    # rejected before any launch: no status word, or a limit out of range
    assert libssd.ssd_selftest_bounded_wait(None, 1000000, None) == libssd.SSD_ERR_INVALID_ARG
    assert libssd.ssd_selftest_bounded_wait(fake(1), 0, None) == libssd.SSD_ERR_INVALID_ARG
    assert libssd.ssd_selftest_bounded_wait(fake(1), 2_000_000_000, None) == libssd.SSD_ERR_INVALID_ARG


def varlen(**kw):
    a = dict(x=fake(1), B=fake(1, 5120), C=fake(1, 7168), row_stride=4608, dt_raw=fake(2), dt_bias=None,
             A=fake(3), D=None, init_state=None, y=fake(4), final_state=fake(5), cu_seqlens=fake(6), nseq=3,
             T=500, H=40, P=64, N=128, G=8, Q=128, dtype=BF16, workspace=fake(7), workspace_bytes=1 << 30,
             status=fake(8), stream=None)
    a.update(kw)
    return libssd.ssd_chunk_scan_fwd_varlen(**a)


def test_varlen_validation():
    # every call here fails validation (or does nothing) before any launch
    assert varlen(nseq=0, T=0) == OK                 # nothing to do
    assert varlen(nseq=0, T=10) == INV               # tokens without sequences
    assert varlen(status=None) == INV                # cu_seqlens errors need a status word
    assert varlen(cu_seqlens=None) == INV
    assert varlen(A=None) == INV and varlen(x=None) == INV and varlen(y=None) == INV
    assert varlen(dtype=7) == INV and varlen(G=7) == INV and varlen(Q=96) == INV
    assert varlen(nseq=-1) == INV and varlen(T=-1) == INV
    assert varlen(workspace_bytes=16) == INV and varlen(workspace=None) == INV
    assert varlen(cu_seqlens=fake(6, 2)) == INV      # misaligned
    assert varlen(y=fake(1, 64)) == INV              # y overlaps x
    assert varlen(final_state=fake(6)) == INV        # final state overlaps cu_seqlens
    assert varlen(H=256, row_stride=16384, T=(1 << 31) - 1) == UNS   # unit list would overflow
    ws = libssd.ssd_chunk_scan_varlen_workspace_bytes(3, 500, 40, 64, 128, 8, 128, BF16)
    assert ws > 0 and ws == libssd.ssd_chunk_scan_varlen_workspace_bytes(3, 500, 40, 64, 128, 8, 128, BF16)
    # the fp32 path needs only the unit table
    assert libssd.ssd_chunk_scan_varlen_workspace_bytes(3, 500, 4, 64, 16, 1, 64, F32) == 256 + 256 * 0 + 256
    assert libssd.ssd_chunk_scan_varlen_workspace_bytes(0, 0, 4, 64, 16, 1, 64, F32) == 0


def cs(**kw):
    a = dict(xBC=fake(1), w=fake(2), bias=None, conv_state=None, dt_raw=fake(3), dt_bias=None,
             A=fake(4), D=None, init_state=None, y=fake(5), final_state=fake(6), b=2, L=256, H=40,
             P=64, N=128, G=8, Q=128, k=4, dtype=BF16, workspace=fake(7), workspace_bytes=1 << 30,
             status=None, stream=None)
    a.update(kw)
    return libssd.ssd_conv_scan_fwd(**a)


def test_conv_scan_validation():
    # every call here fails validation (or is empty work) before any launch
    assert cs(b=0, xBC=None, y=None, dt_raw=None, final_state=None) == OK   # nothing to do
    for k in ("xBC", "w", "dt_raw", "A", "y"):
        assert cs(**{k: None}) == INV, k
    assert cs(workspace=None) == INV and cs(workspace_bytes=16) == INV
    assert cs(H=40, G=7) == INV and cs(P=60) == INV and cs(Q=96) == INV and cs(dtype=5) == INV
    assert cs(xBC=fake(1, 8)) == INV and cs(conv_state=fake(8, 4)) == INV   # misaligned
    assert cs(y=fake(1, 64)) == INV                                    # y overlaps xBC
    assert cs(conv_state=fake(5, 16)) == INV                           # cache overlaps y
    assert cs(workspace=fake(6)) == INV                                # workspace overlaps final state
    assert cs(final_state=fake(3, 64)) == INV                          # final state overlaps dt_raw
    assert cs(k=5) == UNS and cs(k=1) == UNS
    # the conv output (b L conv_dim elements, 256-byte rounded), then the scan's own
    scan = libssd.ssd_chunk_scan_workspace_bytes(2, 256, 40, 64, 128, 8, 128, BF16)
    assert libssd.ssd_conv_scan_workspace_bytes(2, 256, 40, 64, 128, 8, 128, 4, BF16) == \
        2 * 256 * 4608 * 2 + scan
    assert libssd.ssd_conv_scan_workspace_bytes(1, 256, 4, 64, 16, 1, 64, 4, F32) == 256 * 288 * 4
    assert libssd.ssd_conv_scan_workspace_bytes(0, 256, 4, 64, 16, 1, 64, 4, F32) == 0


def dec(**kw):
    a = dict(state=fake(1), conv_state=fake(2), xBC=fake(3), w=fake(4), bias=None, dt_raw=fake(5),
             dt_bias=None, A=fake(6), D=None, y=fake(7), b=256, H=128, P=64, N=128, G=8, k=4,
             dtype=BF16, stream=None)
    a.update(kw)
    return libssd.ssd_decode_step(**a)


def test_decode_step_validation():
    # every call here fails validation (or is empty work) before any launch
    assert dec(b=0) == OK
    for k in ("state", "conv_state", "xBC", "w", "dt_raw", "A", "y"):
        assert dec(**{k: None}) == INV, k
    assert dec(G=3) == INV and dec(N=6) == INV and dec(P=0) == INV and dec(dtype=9) == INV
    assert dec(state=fake(1, 8)) == INV                          # state not 16-byte aligned
    assert dec(xBC=fake(3, 1)) == INV                            # xBC not element aligned
    assert dec(y=fake(3, 64)) == INV                             # y overlaps xBC
    assert dec(conv_state=fake(1, 4096)) == INV                  # cache overlaps the state
    assert dec(k=5) == UNS and dec(k=1) == UNS and dec(N=512) == UNS


def dec_ws(**kw):
    a = dict(state=fake(1), conv_state=fake(2), xBC=fake(3), w=fake(4), bias=None, dt_raw=fake(5),
             dt_bias=None, A=fake(6), D=None, y=fake(7), b=256, H=128, P=64, N=128, G=8, k=4,
             dtype=BF16, workspace=fake(8), workspace_bytes=256 * 8 * 4, stream=None)
    a.update(kw)
    return libssd.ssd_decode_step_ws(**a)


def test_decode_step_ws_validation():
    # every call here fails validation (or is empty work) before any launch
    assert libssd.ssd_decode_step_workspace_bytes(256, 8) == 256 * 8 * 4
    assert libssd.ssd_decode_step_workspace_bytes(0, 8) == 0
    assert dec_ws(b=0) == OK
    for k in ("state", "conv_state", "xBC", "w", "dt_raw", "A", "y", "workspace"):
        assert dec_ws(**{k: None}) == INV, k
    assert dec_ws(workspace_bytes=256 * 8 * 4 - 4) == INV       # short
    assert dec_ws(workspace=fake(8, 2)) == INV                   # not 4-byte aligned
    assert dec_ws(workspace=fake(7, 64)) == INV                  # overlaps y
    assert dec_ws(G=3) == INV and dec_ws(N=6) == INV and dec_ws(dtype=9) == INV
    assert dec_ws(conv_state=fake(1, 4096)) == INV               # cache overlaps the state
    assert dec_ws(k=5) == UNS and dec_ws(N=512) == UNS and dec_ws(P=320, b=1) == UNS


def bwd(**kw):
    a = dict(x=fake(1), B=fake(1, 2560 * 2), C=fake(1, (2560 + 1024) * 2), row_stride=4608, dt_raw=fake(2),
             dt_bias=None, A=fake(3), D=None, init_state=None, dy=fake(4), dfinal=None, dx=fake(5), dB=fake(6),
             dC=fake(7), ddt_raw=fake(8), dA=fake(9), dD=fake(9, 256), ddt_bias=fake(9, 512), dinit=None,
             b=2, L=256, H=40, P=64, N=128, G=8, dtype=BF16, workspace=fake(10), workspace_bytes=1 << 33,
             stream=None)
    a.update(kw)
    return libssd.ssd_chunk_scan_bwd(**a)


def test_scan_bwd_validation():
    # every call here fails validation before any launch
    for k in ("x", "B", "C", "dt_raw", "A", "dy", "dx", "dB", "dC", "ddt_raw", "dA", "dD", "ddt_bias"):
        assert bwd(**{k: None}) == INV, k
    assert bwd(G=7) == INV and bwd(dtype=4) == INV and bwd(L=-1) == INV
    assert bwd(row_stride=100) == INV                          # shorter than H*P
    assert bwd(x=fake(1, 1)) == INV and bwd(dA=fake(9, 2)) == INV   # misaligned
    assert bwd(dx=fake(4, 64)) == INV                          # dx overlaps dy
    assert bwd(dD=fake(9, 64)) == INV                          # dD overlaps dA
    assert bwd(workspace=fake(5)) == INV                       # workspace overlaps dx
    assert bwd(workspace_bytes=100) == INV
    need = libssd.ssd_chunk_scan_bwd_workspace_bytes(2, 256, 40, 64, 128, 8, BF16)
    assert need > 2 * 40 * 8 * 64 * 128 * 4                    # the chunks' entering states, at least
    assert libssd.ssd_chunk_scan_bwd_workspace_bytes(0, 256, 40, 64, 128, 8, BF16) == 0
    assert bwd(N=1024, G=1, workspace_bytes=1 << 40) == UNS   # one CTA's shared memory would not fit


def test_linear_validation():
    P_ = 1 << 20   # any 16-byte aligned non-null address (nothing is launched)
    f = libssd.ssd_linear_bf16
    assert f(P_, 64, P_ + (1 << 16), 64, P_ + (1 << 18), 64, 0, 64, 64, None, None) == OK   # no rows
    assert f(P_, 64, P_ + (1 << 16), 64, P_ + (1 << 18), 64, -1, 64, 64, None, None) == INV
    assert f(None, 64, P_ + (1 << 16), 64, P_ + (1 << 18), 64, 4, 64, 64, None, None) == INV
    assert f(P_, 64, P_ + (1 << 16), 64, P_ + (1 << 18), 64, 4, 60, 64, None, None) == INV   # N % 8
    assert f(P_, 64, P_ + (1 << 16), 64, P_ + (1 << 18), 64, 4, 64, 60, None, None) == INV   # K % 8
    assert f(P_, 32, P_ + (1 << 16), 64, P_ + (1 << 18), 64, 4, 64, 64, None, None) == INV   # ldx < K
    assert f(P_ + 2, 64, P_ + (1 << 16), 64, P_ + (1 << 18), 64, 4, 64, 64, None, None) == INV   # alignment
    assert f(P_, 64, P_ + (1 << 16), 64, P_, 64, 4, 64, 64, None, None) == INV   # y overlaps x


def test_mixer_validation():
    P_ = 1 << 20
    ws = libssd.ssd_mixer_workspace_bytes(2, 300, 256, 8, 64, 128, 2, 128, 4, BF16)
    assert ws > 2 * 300 * (2 * 512 + 512 + 8) * 2   # in_proj output alone
    assert libssd.ssd_mixer_workspace_bytes(2, 300, 256, 8, 64, 128, 2, 128, 4, F32) == 0

    def call(**kw):
        a = dict(hidden=P_, W_in=P_ + (1 << 22), conv_w=P_ + (2 << 22), conv_bias=None, conv_state=None,
                 dt_bias=None, A=P_ + (3 << 22), D=None, norm_w=P_ + (4 << 22), W_out=P_ + (5 << 22),
                 init_state=None, out=P_ + (6 << 22), final_state=None, b=2, L=300, d_model=256, H=8, P=64,
                 N=128, G=2, Q=128, k=4, norm_groups=1, eps=1e-5, dtype=BF16, workspace=P_ + (8 << 22),
                 workspace_bytes=ws, status=None, stream=None)
        a.update(kw)
        return libssd.ssd_mixer_fwd(*a.values())
    assert call(d_model=250) == INV          # d_model % 8
    assert call(H=6, G=3) == UNS             # H % 8: the dt rows are not 16-byte rows
    assert call(dtype=F32) == UNS            # bf16 projections only
    assert call(norm_groups=3) == INV        # H*P not divisible
    assert call(eps=-1.0) == INV
    assert call(k=5) == UNS
    assert call(hidden=None) == INV
    assert call(workspace_bytes=ws - 256) == INV
    assert call(out=P_ + 16) == INV          # out overlaps hidden
