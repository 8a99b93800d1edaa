"""bench.py reports a captured DRAM traffic figure only for the kernel
sources it was captured on."""
import bench


def test_traffic_is_reported_for_the_captured_sources_only(monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_SOURCES", bench.kernel_sources_digest())
    assert bench.traffic_for("glm52_layer_decode_b1", "decode") == bench.TRAFFIC[("glm52_layer_decode_b1", "decode")]
    assert bench.traffic_for("glm52_layer_decode_b64_zipf", "decode") is None     # never captured
    monkeypatch.setattr(bench, "TRAFFIC_SOURCES", "0" * 16)
    assert bench.traffic_for("glm52_layer_decode_b1", "decode") is None


def test_digest_covers_every_kernel_source(tmp_path, monkeypatch):
    import shutil
    src = tmp_path / "int4_routed_expert_renorm_b200" / "csrc"
    shutil.copytree(bench.os.path.join(bench.ROOT, "int4_routed_expert_renorm_b200", "csrc"), src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.kernel_sources_digest()
    f = sorted(src.iterdir())[0]
    f.write_bytes(f.read_bytes() + b"\n")
    assert bench.kernel_sources_digest() != d0
