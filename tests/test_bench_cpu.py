"""Host-side logic of bench.py that needs no GPU: the DRAM-traffic record is
reported only while the kernel sources still hash to the value recorded at
capture time, and the algorithmic byte counts follow their definitions."""
import bench


def test_recorded_traffic_is_tied_to_the_sources(tmp_path, monkeypatch):
    f = tmp_path / "traffic.txt"
    good = bench.source_hash("decode")
    f.write_text("# comment\nfresh %s 123 one launch\nstale 0000000000000000 456 old\n" % good)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.measured_traffic("fresh", "decode") == 123.0
    assert bench.measured_traffic("stale", "decode") is None
    assert bench.measured_traffic("absent", "decode") is None


def test_source_hash_changes_with_the_sources(tmp_path, monkeypatch):
    a = tmp_path / "a.cu"
    a.write_text("x")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "probe", ["a.cu"])
    h1 = bench.source_hash("probe")
    a.write_text("y")
    assert bench.source_hash("probe") != h1


def test_algorithmic_bytes():
    # q, k, v bf16 in, out bf16, g and beta fp32, final state fp32 out
    T, H, d = 64, 2, 128
    per = (2 * d + d) * 2 + 8 + d * 2
    assert bench.prefill_bytes(T, H, d, d, 1, with_state_in=False) == T * H * per + H * d * d * 4
    assert bench.prefill_bytes(T, H, d, d, 1, with_state_in=True) == T * H * per + 2 * H * d * d * 4
    # decode: the state read and written once, one token in and out
    assert bench.decode_bytes(3, 2, d, d) == 3 * 2 * (2 * d * d * 4 + 3 * d * 2 + 8 + d * 2)
