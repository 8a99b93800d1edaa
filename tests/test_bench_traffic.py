"""bench.py reports a captured DRAM traffic figure only for the kernel
sources it was captured on."""
import bench


def test_traffic_is_reported_for_the_captured_sources_only(monkeypatch):
    monkeypatch.setattr(bench, "_SK_SOURCES", bench.kernel_sources_digest(bench._KERNEL_FILES["decode"]))
    monkeypatch.setitem(bench.TRAFFIC, ("glm52_layer_decode_b1", "decode"), (123.0, bench._SK_SOURCES))
    assert bench.traffic_for("glm52_layer_decode_b1", "decode") == 123.0
    assert bench.traffic_for("glm52_layer_decode_b64_zipf", "decode") is None     # never captured
    monkeypatch.setitem(bench.TRAFFIC, ("glm52_layer_decode_b1", "decode"), (123.0, "0" * 16))
    assert bench.traffic_for("glm52_layer_decode_b1", "decode") is None


def test_digest_covers_the_named_sources(tmp_path, monkeypatch):
    import shutil
    src = tmp_path / "int4_routed_expert_renorm_b200" / "csrc"
    shutil.copytree(bench.os.path.join(bench.ROOT, "int4_routed_expert_renorm_b200", "csrc"), src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    files = bench._KERNEL_FILES["decode"]
    d0, d_all = bench.kernel_sources_digest(files), bench.kernel_sources_digest()
    other = src / "k_ffn_prefill.cuh"
    other.write_bytes(other.read_bytes() + b"\n")
    assert bench.kernel_sources_digest(files) == d0 and bench.kernel_sources_digest() != d_all
    f = src / files[-1]
    f.write_bytes(f.read_bytes() + b"\n")
    assert bench.kernel_sources_digest(files) != d0
