"""Host-side pieces of bench.py that the reported numbers rest on (CPU only): the algorithmic
bytes per expert, and the ncu traffic figure that is only reported while the profiled kernel's
code is unchanged."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_expert_bytes_match_the_packed_layout():
    # one OLMoE-shaped expert: W13 (2I x H) and W2 (H x I) at half a byte per weight, plus one bf16
    # scale per 128 weights of a row: 3,145,728 B of codes + 98,304 B of scales
    H, I = 2048, 1024
    codes = (2 * I * H + H * I) // 2
    scales = (2 * I * (H // 128) + H * (I // 128)) * 2
    assert codes == 3_145_728 and scales == 98_304
    assert bench.expert_bytes(H, I) == codes + scales == 3_244_032


def test_code_of_drops_comments_and_blank_space():
    a = "int f(int x) {  // doubles\n  return 2 * x;   /* twice */\n}\n\n"
    b = "int f(int x) {\n return 2 * x;\n}"
    assert bench.code_of(a) == bench.code_of(b)
    assert bench.code_of(a) != bench.code_of(b.replace("2", "3"))


def test_profiled_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    import json
    # a record written for copies of the profiled sources is read back while they are unchanged
    copies = []
    for i, f in enumerate(bench.PROFILE_SOURCES):
        dst = tmp_path / f"src{i}"
        shutil.copyfile(os.path.join(ROOT, f), dst)
        copies.append(str(dst))
    monkeypatch.setattr(bench, "PROFILE_SOURCES", copies)
    record = tmp_path / "record.json"
    record.write_text(json.dumps({"source_hash": bench.source_hash(), "traffic_bytes_per_launch": 12345}))
    monkeypatch.setattr(bench, "PROFILE", str(record))
    assert bench.profiled_traffic() == 12345
    # a comment-only edit leaves the compiled kernel, and so the figure, as it was
    with open(copies[0], "a") as fh:
        fh.write("\n// edited\n/* and a block\n comment */\n")
    assert bench.profiled_traffic() == 12345
    # any change to the code drops the figure
    with open(copies[0], "a") as fh:
        fh.write("\nstatic int edited = 1;\n")
    assert bench.profiled_traffic() is None
    # so does a missing record
    monkeypatch.setattr(bench, "PROFILE", str(tmp_path / "missing.json"))
    assert bench.profiled_traffic() is None


def test_committed_profile_traffic_is_near_the_algorithmic_bytes():
    tr = bench.profiled_traffic()
    if tr is None:
        import pytest
        pytest.skip("the profiled kernel changed since its ncu summary was taken (traffic reported as null)")
    # DRAM traffic per launch within 1% of the algorithmic bytes of a top-8 OLMoE layer
    algo = 8 * bench.expert_bytes(2048, 1024)
    assert abs(tr - algo) <= 0.01 * algo
