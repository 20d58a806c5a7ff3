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


def test_committed_traffic_records_are_well_formed():
    """Every record names a key bench.py asks for, a 16-digit source hash,
    a byte count and the profile summary it comes from; every key bench.py
    asks for has a record."""
    import os
    import re
    src = open(os.path.join(bench.ROOT, "bench.py")).read()
    asked = set(re.findall(r'measured_traffic\("([a-z0-9_]+)", "([a-z]+)"\)', src))
    keys = {}
    with open(bench.TRAFFIC_FILE) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, h, nbytes, what = line.split(None, 3)
            assert re.fullmatch(r"[0-9a-f]{16}", h), line
            assert float(nbytes) > 0, line
            ref = re.search(r"\(([\w.]+\.md)\)\s*$", what)
            assert ref and os.path.exists(os.path.join(bench.ROOT, "profiles", ref.group(1))), line
            keys[key] = h
    for key, kind in asked:
        assert kind in bench.KERNEL_SOURCES, (key, kind)
        assert key in keys, key
