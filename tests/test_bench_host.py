"""Host-side logic of the benchmark: the algorithmic byte models used for the
roofline, the lookup of ncu-measured traffic keyed on kernel sources, and
the reference arm's JSON line (it runs the CPU oracle only)."""
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_decode_bytes_per_head():
    # snapshot d_v d_k + 4 d_v + 4 d_k + r (4 + 4 d_k) at d = 128, r = 4
    S = 128 * 128 + 4 * 128 + 4 * 128 + 4 * (4 + 4 * 128)
    assert bench.snapshot_bytes(128, 128, 4) == S == 19472
    rec = 4 * (1 + 128 + 128)
    assert bench.record_bytes(128, 128, "scalar") == rec
    # position t: snapshot, t - 1 records, bf16 q k v + alpha beta, bf16 o, the new record
    for t in (1, 8, 16):
        want = S + (t - 1) * rec + 2 * (2 * 128 + 128) + 8 + 2 * 128 + rec
        assert bench.decode_launch_bytes(128, 128, 4, "scalar", 2, t) == want
    # diagonal gate: d_k gate values per record and per token
    assert bench.record_bytes(128, 128, "diag") == 4 * (3 * 128)
    assert bench.decode_launch_bytes(128, 128, 8, "diag", 2, 1) == \
        bench.snapshot_bytes(128, 128, 8) + 2 * 384 + 4 * 128 + 4 + 2 * 128 + 4 * 384


def test_commit_bytes_per_head():
    assert bench.commit_launch_bytes(128, 128, 4, "scalar", 16) == 2 * 19472 + 16 * 1028


def test_profiled_traffic_requires_matching_sources(tmp_path):
    digest = bench.source_digest("decode")
    (tmp_path / "a.md").write_text(
        f"# x\ntraffic_key: decode:wl\nsource_sha1: {digest}\ntraffic_bytes_per_launch: 123.5e6\n")
    (tmp_path / "b.md").write_text(
        "traffic_key: commit:wl\nsource_sha1: 000000000000\ntraffic_bytes_per_launch: 9\n")
    assert bench.profiled_traffic("decode:wl", str(tmp_path)) == 123.5e6
    assert bench.profiled_traffic("commit:wl", str(tmp_path)) is None   # stale sources
    assert bench.profiled_traffic("decode:other", str(tmp_path)) is None
    assert bench.source_digest("decode") != bench.source_digest("commit")


def test_profile_key_names_overrides():
    """The headline workload keeps its plain key (its ncu summary applies);
    any override of W, r, smoothing or the code width gets its own key."""
    import dataclasses
    from linear_attention_recurrent_int8_b200 import synth

    class A:
        bits = 8

    wl = synth.WORKLOADS["gdn_256x32_d128_bf16"]
    assert bench.profile_key("decode", wl, A) == "decode:gdn_256x32_d128_bf16"
    A.bits = 4
    assert bench.profile_key("decode", wl, A) == "decode:gdn_256x32_d128_bf16_W16_r4_s1_b4"
    A.bits = 8
    w8 = dataclasses.replace(wl, window=8)
    assert bench.profile_key("commit", w8, A) == "commit:gdn_256x32_d128_bf16_W8_r4_s1_b8"
    A.comp_rule = "svd"
    assert bench.profile_key("decode", wl, A) == "decode:gdn_256x32_d128_bf16_svd"


def test_svd_rule_byte_model():
    """The SVD rule adds the r u_c vectors (4 d_v bytes each) to a snapshot."""
    assert bench.snapshot_bytes(128, 128, 4, 8, svd=True) == 19472 + 4 * 4 * 128
    assert bench.decode_launch_bytes(128, 128, 4, "scalar", 2, 1, 8, True) == \
        bench.decode_launch_bytes(128, 128, 4, "scalar", 2, 1, 8) + 4 * 4 * 128


def test_narrow_code_byte_models():
    # 4-bit codes: d_v d_k / 2 code bytes per head; 6-bit: one byte per code
    assert bench.snapshot_bytes(128, 128, 4, 4) == 19472 - 8192
    assert bench.snapshot_bytes(128, 128, 4, 6) == 19472
    assert bench.decode_launch_bytes(128, 128, 4, "scalar", 2, 8, 4) == \
        bench.decode_launch_bytes(128, 128, 4, "scalar", 2, 8) - 8192
    assert bench.commit_launch_bytes(128, 128, 4, "scalar", 16, 4) == 2 * 11280 + 16 * 1028


def test_bf16_state_byte_model():
    # BF16 residual: two bytes per value
    assert bench.snapshot_bytes(128, 128, 0, 16) == 2 * 128 * 128 + 4 * 128 + 4 * 128


@pytest.mark.parametrize("bits", [8, 4, 16])
def test_reference_arm_line_on_cpu(bits):
    """The reference arm (the oracle on the host cores) prints one JSON line
    with the contract's keys, on a tiny workload, at every state width."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "gdn_1x1_d64_fp32", "--steps", "1", "--warmup", "3",
                        "--ref-seconds", "0.05", "--bits", str(bits)],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["warmup"] >= 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["bits"] == bits


def test_l2_note_says_which():
    assert bench.l2_note(160e6).startswith("inputs larger than L2")
    assert "L2-resident" in bench.l2_note(28e6)


def test_secondary_workloads_are_known():
    """The default run's secondary entries name existing workloads and modes."""
    from linear_attention_recurrent_int8_b200 import synth
    assert bench.DEFAULT_WORKLOAD in synth.WORKLOADS
    for name, mode, workload, steps, warmup, flags in bench.SECONDARY:
        assert workload in synth.WORKLOADS, name
        assert mode in ("decode", "prefill", "ragged"), name
        assert steps >= 1 and warmup >= 3, name
        assert f"--steps {steps}" in flags and f"--warmup {warmup}" in flags, name
