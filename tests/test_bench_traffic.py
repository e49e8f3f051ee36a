"""The benchmark's ncu traffic figure is tied to the GEMM kernel's code: a
comment-only edit keeps it, any change to the code makes it null (CPU only)."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_strip_comments_keeps_code_and_strings():
    import bench
    src = 'int a = 1;  // note\n/* block\n comment */ const char* s = "x // y";\n'
    assert bench._strip_c_comments(src) == 'inta=1;constchar*s="x // y";'
    assert bench._strip_c_comments("f('/');//z") == "f('/');"


def _copy_sources(tmp_path):
    import bench
    dst = tmp_path / "fine_grained_moe_router_b200" / "csrc"
    dst.mkdir(parents=True)
    for name in bench.TRAFFIC_SOURCES:
        shutil.copy(os.path.join(ROOT, "fine_grained_moe_router_b200", "csrc", name), dst / name)
    return dst


def test_fingerprint_ignores_comments_not_code(tmp_path, monkeypatch):
    import bench
    base = bench.kernel_code_fingerprint()
    dst = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_code_fingerprint() == base

    gemm = dst / "ffn_tc.cu"
    text = gemm.read_text()
    gemm.write_text("// an added comment line\n" + text.replace("\n", "\n\n", 3))
    assert bench.kernel_code_fingerprint() == base

    gemm.write_text(text + "\nstatic int kUnused = 0;\n")
    assert bench.kernel_code_fingerprint() != base


def test_traffic_reported_only_for_captured_workload():
    import bench
    m = bench.MEASURED_TRAFFIC
    wl = bench.mi.WORKLOADS[m["workload"]]
    current = bench.kernel_code_fingerprint() == m["kernel_code_sha256_16"]
    got = bench.measured_traffic(wl, m["T"])
    assert (got == m["bytes_per_step"] / 2.0) if current else got is None
    assert bench.measured_traffic(wl, m["T"] + 1) is None
