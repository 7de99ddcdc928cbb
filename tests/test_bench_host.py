"""Host-side logic of the benchmark: the algorithmic byte models used for the
roofline, and the lookup of ncu-measured traffic keyed on kernel sources."""
import bench


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
