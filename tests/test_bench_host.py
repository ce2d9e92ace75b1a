"""Host logic of bench.py that needs no GPU: the committed ncu summaries are read only
while they were taken on the current kernel source, and their fields turn into the
traffic figures of the benchmark line."""
import os

import bench


def _profile(tmp_path, files, **fields):
    p = tmp_path / "profile.txt"
    lines = ["# comment: with a colon", f"source_sha256: {bench.source_sha(files)}"]
    lines += [f"{k}: {v}" for k, v in fields.items()]
    p.write_text("\n".join(lines) + "\n")
    return str(p)


def test_profile_fields_follow_the_source_hash(tmp_path):
    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    path = _profile(tmp_path, [str(src)], dram_bytes_read_per_launch=100, command="ncu --x a:b")
    kv = bench.profile_fields(path, [str(src)])
    assert kv["dram_bytes_read_per_launch"] == "100" and kv["command"] == "ncu --x a:b"
    src.write_text("// version 2\n")                      # the kernel changed: the figures no longer apply
    assert bench.profile_fields(path, [str(src)]) is None
    assert bench.profile_fields(str(tmp_path / "missing.txt"), [str(src)]) is None


def test_committed_summaries_parse_and_scale():
    """The committed summaries carry the fields the benchmark line uses; when they match
    the current source, the traffic figures are the recorded ones."""
    for path, files, key in ((bench.PROFILE_TRAFFIC, bench.SCORE_SRC, "dram_bytes_read_per_launch"),
                             (bench.PROFILE_GATHER, bench.GATHER_SRC, "pcie_read_bytes_per_payload_byte")):
        assert os.path.exists(path)
        text = open(path).read()
        assert "source_sha256:" in text and key + ":" in text and "--clock-control none" in text
    kv = bench.profile_fields(bench.PROFILE_GATHER, bench.GATHER_SRC)
    if kv is not None:
        ratio = float(kv["pcie_read_bytes_per_payload_byte"])
        assert 1.0 <= ratio < 1.5
        assert bench.gather_link_traffic(10 ** 9) == round(ratio * 10 ** 9)
    kv = bench.profile_fields(bench.PROFILE_TRAFFIC, bench.SCORE_SRC)
    if kv is not None:
        assert bench.traffic_per_launch() == (int(kv["dram_bytes_read_per_launch"]) +
                                              int(kv["dram_bytes_write_per_launch"]))
