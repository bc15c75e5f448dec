"""The benchmark's algorithmic work per token and per step (CPU only): the
byte and FLOP counts behind every roofline fraction, checked against their
definitions worked out by hand for the bench workloads, and the seeded
prompt-length mix of the ragged block."""
import bench
from ssd_selective_scan_b200 import synth


def test_scan_bytes_and_flops_per_token():
    # e (2 H P + 2 G N + H): x and y, B and C, dt, bf16
    assert bench.scan_bytes_per_token(synth.CONFIGS[1]) == 2 * (2 * 40 * 64 + 2 * 8 * 128 + 40) == 14416
    assert bench.scan_bytes_per_token(synth.CONFIGS[2]) == 2 * (2 * 128 * 64 + 2 * 8 * 128 + 128) == 37120
    assert bench.scan_bytes_per_token(synth.CONFIGS[3]) == 2 * (2 * 64 * 64 + 2 * 8 * 128 + 64) == 20608
    # causal C B^T (G Q N) + causal (.)X (H Q P) + chunk state and C h (4 H P N)
    s = synth.CONFIGS[1]
    assert bench.scan_flops_per_token(s) == 8 * 128 * 128 + 40 * 128 * 64 + 4 * 40 * 64 * 128 == 1769472


def test_conv_and_decode_bytes():
    assert bench.conv_bytes_per_token(synth.CONFIGS[1]) == 2 * 2 * 4608
    d = synth.CONFIGS[4]
    state = 8 * 256 * 128 * 64 * 128                  # fp32 state read and written
    assert state == 2147483648
    assert bench.decode_state_update_bytes(d) == state + 2 * 256 * (128 * 64 + 2 * 8 * 128 + 128 + 128 * 64)
    # the one-kernel step adds the conv cache (k columns read and written) and the
    # whole xBC row instead of its already-convolved x, B, C
    assert bench.decode_step_bytes(d) == state + 2 * 256 * (2 * 4 * 10240 + 10240 + 128 + 128 * 64)


def test_peaks_fallback_is_labelled(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))   # no MEASURED_PEAKS.json there
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0


def test_ragged_length_mix():
    from ssd_selective_scan_b200 import synth
    a = synth.ragged_lengths(16384, 11)
    assert a == synth.ragged_lengths(16384, 11), "not reproducible from its seed"
    assert sum(a) == 16384 and len(a) > 1
    assert all(64 <= n < 4096 + 64 for n in a)
    assert synth.ragged_lengths(16384, 12) != a
    assert synth.ragged_lengths(100, 3) == [100]
