"""Host-side pieces of the benchmark that decide what its JSON line reports:
the fingerprint that ties the committed ncu DRAM-traffic figure to the GEMM
kernel's code, and the reading of that figure."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comment_stripper_keeps_code_and_literals():
    src = ('int a = 1; // trailing\n'
           '/* block\n comment */ const char *p = "//not /*a*/ comment";\n'
           "char q = '\"'; char r = '\\''; int b = a / 2; // x\n")
    out = bench._strip_comments(src)
    assert "trailing" not in out and "block" not in out and "// x" not in out
    assert '"//not /*a*/ comment"' in out
    assert "char q = '\"';" in out and "char r = '\\'';" in out
    assert "int b = a / 2;" in out


def test_fingerprint_ignores_comments_but_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "fp8_block_scaled_fp8bq_b200" / "csrc"
    csrc.mkdir(parents=True)
    names = ("gemm.cu", "gemm_promote.cuh", "device.cuh", "quant.cuh", "raster.cu")
    for n in names:
        (csrc / n).write_text("int f() { return 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_sha()
    (csrc / "device.cuh").write_text("// a new comment\nint f() { return 1; } /* and another */\n")
    assert bench.kernel_source_sha() == base
    (csrc / "device.cuh").write_text("int f() { return 2; }\n")
    assert bench.kernel_source_sha() != base


def test_committed_traffic_matches_the_current_code():
    """The committed summary names the code it was captured from; while that
    code is unchanged the benchmark reports its per-launch DRAM bytes."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic_llama8b_layer_M8192.txt")
    fields = dict(line.split(": ", 1) for line in open(path).read().splitlines()
                  if line.startswith(("source_sha: ", "dram_bytes_per_launch_step_avg: ")))
    t = bench.committed_traffic()
    if fields["source_sha"].strip() == bench.kernel_source_sha():
        assert t == int(fields["dram_bytes_per_launch_step_avg"])
    else:
        assert t is None
