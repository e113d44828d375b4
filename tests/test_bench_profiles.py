"""CPU checks of how bench.py attaches ncu traffic to a bench line: the
DRAM bytes come from a committed summary only while the kernel family's
sources (its header and the headers it includes, comments and blank space
ignored) still hash to the value the summary records."""
import os
import shutil

import bench

KERNEL = "halo_fwd_tc4<16,14>"


def _summary(sha, nbytes=123456, workload="stage1_bf16"):
    return (f"# summary\n\n- workload: `{workload}`\n- kernel_source_sha: `{sha}`\n"
            f"- dram_bytes_per_launch: {nbytes}\n")


def test_traffic_only_while_the_sources_match(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    (tmp_path / "a.md").write_text(_summary(bench.kernel_source_hash(KERNEL)))
    assert bench.ncu_traffic("stage1_bf16", KERNEL) == 123456.0
    assert bench.ncu_traffic("deep_bf16", KERNEL) is None            # no summary for that workload
    (tmp_path / "a.md").write_text(_summary("0123456789abcdef"))
    assert bench.ncu_traffic("stage1_bf16", KERNEL) is None          # sources changed since the capture


def test_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "blocked_local_self_b200", "csrc")
    copy = tmp_path / "blocked_local_self_b200" / "csrc"
    shutil.copytree(src, copy)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_hash(KERNEL)
    hdr = copy / "halo_tc4.cuh"
    text = hdr.read_text()
    hdr.write_text(text + "\n// a comment only\n/* and a block comment */\n")
    assert bench.kernel_source_hash(KERNEL) == base
    hdr.write_text(text + "\nstatic_assert(true, \"\");\n")
    assert bench.kernel_source_hash(KERNEL) != base
    # an included header counts too
    hdr.write_text(text)
    sm = copy / "sm100.cuh"
    sm.write_text(sm.read_text() + "\nstatic_assert(true, \"\");\n")
    assert bench.kernel_source_hash(KERNEL) != base
    # another family's header does not
    sm.write_text((copy / "sm100.cuh").read_text().replace("\nstatic_assert(true, \"\");\n", ""))
    assert bench.kernel_source_hash(KERNEL) == base
    other = copy / "halo_tc3.cuh"
    other.write_text(other.read_text() + "\nstatic_assert(true, \"\");\n")
    assert bench.kernel_source_hash(KERNEL) == base


def test_committed_summaries_name_their_workload_and_kernel():
    import glob
    import re
    seen = set()
    for path in glob.glob(os.path.join(bench.PROFILES, "halo_fwd_*.md")):
        text = open(path).read()
        fields = dict(re.findall(r"^- (\w+): `?([^`\n]+?)`?\s*$", text, flags=re.M))
        assert "workload" in fields and "kernel_source_sha" in fields and "dram_bytes_per_launch" in fields, path
        assert re.search(r"ncu .*--clock-control none", text), path
        seen.add(fields["workload"])
    assert {"stage1_bf16", "deep_bf16", "stride2_bf16", "large_bf16"} <= seen
