"""The DRAM traffic record the bench line reports (profiles/traffic.json):
figures are used only while the kernels' code, without comments and blank
lines, still has the sha256 stored beside them."""
import json
import os
import shutil

import bench

CSRC = ("block_sparse_bidirectional_select_b200", "csrc")


def _tree(tmp_path):
    src = os.path.join(bench.ROOT, *CSRC)
    dst = tmp_path.joinpath(*CSRC)
    dst.mkdir(parents=True)
    for name in bench.LOSA_KERNEL_FILES:
        shutil.copy(os.path.join(src, name), dst / name)
    (tmp_path / "profiles").mkdir()
    return dst


def _record(tmp_path):
    rec = {"attn_kernels_sha256": bench.kernel_signature(),
           "c4_64k": {"attn_fwd_kernel<128,128,dense>": 123},
           "losa_kernels_sha256": bench.kernel_signature(bench.LOSA_KERNEL_FILES),
           "losa_32k": {"block_run": 456}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))


def test_signature_ignores_comments_and_blank_lines():
    code = "int a = 1;  // one\n\n// a line of comment\n  int b = 2;\n"
    assert bench.code_signature(code) == bench.code_signature("int a = 1;\nint b = 2;")
    assert bench.code_signature(code) != bench.code_signature("int a = 1;\nint b = 3;")


def test_record_used_only_while_the_kernels_are_unchanged(tmp_path, monkeypatch):
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _record(tmp_path)
    assert bench.load_traffic("c4_64k") == {"attn_fwd_kernel<128,128,dense>": 123}
    assert bench.load_traffic("losa_32k", "losa_kernels_sha256", bench.LOSA_KERNEL_FILES) == {"block_run": 456}
    # a comment added to a kernel keeps the record
    with open(csrc / "attn_list_kernel.cuh", "a") as f:
        f.write("\n// a note\n")
    assert bench.load_traffic("c4_64k") != {}
    # a change of code voids it; the block-wise record covers its own kernels too
    with open(csrc / "losa_kernels.cuh", "a") as f:
        f.write("\nstatic int unused_marker = 0;\n")
    assert bench.load_traffic("c4_64k") != {}
    assert bench.load_traffic("losa_32k", "losa_kernels_sha256", bench.LOSA_KERNEL_FILES) == {}
    with open(csrc / "attn_kernel.cuh", "a") as f:
        f.write("\nstatic int unused_marker2 = 0;\n")
    assert bench.load_traffic("c4_64k") == {}


def test_missing_record_gives_no_figures(tmp_path, monkeypatch):
    _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("c4_64k") == {}
