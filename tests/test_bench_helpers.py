"""Host-side helpers of bench.py (CPU): the DRAM-traffic lookup in a committed
ncu summary, which must answer only for the kernel source it was taken on,
and the name of the product kernel the library's switches select."""
import os

import bench


def _summary(tmp_path, text):
    d = tmp_path / "profiles"
    d.mkdir()
    (d / "t.md").write_text(text)
    return str(tmp_path)


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    root = _summary(tmp_path, "# x\n\n- kernel_source_hash: `abc123`\n"
                              "- dram_bytes_per_full_launch: `1000`\n")
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.profiled_traffic("abc123", "t.md") == 1000.0
    assert bench.profiled_traffic("def456", "t.md") is None      # kernel changed since
    assert bench.profiled_traffic("abc123", "missing.md") is None


def test_traffic_needs_both_keys(tmp_path, monkeypatch):
    root = _summary(tmp_path, "- kernel_source_hash: `abc123`\n")
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.profiled_traffic("abc123", "t.md") is None


def test_committed_traffic_profile_parses():
    """The committed summary names a hash and a byte count; whether the hash
    is the current one decides only whether the bench reports it."""
    path = os.path.join(bench.ROOT, "profiles", "kq_quantize_stress_traffic.md")
    text = open(path).read()
    assert "- kernel_source_hash: `" in text
    assert "- dram_bytes_per_full_launch: `" in text
    h = [l for l in text.splitlines() if l.startswith("- kernel_source_hash:")][0]
    hval = h.split(":", 1)[1].strip().strip("`")
    assert bench.profiled_traffic(hval, "kq_quantize_stress_traffic.md") > 4e8


def test_gemm_kernel_name_follows_the_library_switches(monkeypatch):
    for var in ("KQ_GEMM_PAIR", "KQ_GEMM_PERSISTENT"):
        monkeypatch.delenv(var, raising=False)
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_persistent<")
    monkeypatch.setenv("KQ_GEMM_PAIR", "1")
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_pair<")
    monkeypatch.setenv("KQ_GEMM_PAIR", "00")                   # atoi("00") == 0
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_persistent<")
    monkeypatch.setenv("KQ_GEMM_PERSISTENT", "0")
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_kernel<")
    monkeypatch.setenv("KQ_GEMM_PERSISTENT", "x")              # atoi("x") == 0
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_kernel<")
