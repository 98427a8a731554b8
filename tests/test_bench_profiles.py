"""bench.py reports a kernel's DRAM traffic from its ncu summary only while the
sources that kernel is built and launched from are those the summary records."""
import os
import shutil

import bench


def _summary(path, sources, nbytes):
    path.write_text(f"# summary\n\nkernel_source_hash: {bench.kernel_source_hash(sources)}\n"
                    f"dram_bytes_per_launch_full_size: {nbytes}\n")
    return str(path)


def test_each_kernel_hashes_only_its_own_sources():
    assert "pa_kernels.cuh" in bench.DECODE_SOURCES
    assert "pa_prefill_tc.cuh" not in bench.DECODE_SOURCES
    assert "pa_prefill_tc.cuh" in bench.PREFILL_SOURCES
    assert "pa_kernels.cuh" not in bench.PREFILL_SOURCES
    for f in bench.DECODE_SOURCES + bench.PREFILL_SOURCES:
        assert os.path.exists(os.path.join(bench.CSRC, f))


def test_a_source_change_voids_only_that_kernels_traffic(tmp_path, monkeypatch):
    csrc = tmp_path / "csrc"
    shutil.copytree(bench.CSRC, csrc)
    monkeypatch.setattr(bench, "CSRC", str(csrc))
    dec = _summary(tmp_path / "dec.md", bench.DECODE_SOURCES, 1000)
    pre = _summary(tmp_path / "pre.md", bench.PREFILL_SOURCES, 2000)
    assert bench.profiled_traffic(dec, bench.DECODE_SOURCES) == 1000
    assert bench.profiled_traffic(pre, bench.PREFILL_SOURCES) == 2000
    with open(csrc / "pa_prefill_tc.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.profiled_traffic(dec, bench.DECODE_SOURCES) == 1000
    assert bench.profiled_traffic(pre, bench.PREFILL_SOURCES) is None
    with open(csrc / "pa_kernels.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.profiled_traffic(dec, bench.DECODE_SOURCES) is None


def test_a_summary_without_the_fields_gives_none(tmp_path):
    p = tmp_path / "summary.md"
    p.write_text("# a summary\nno hash here\n")
    assert bench.profiled_traffic(str(p)) is None
    assert bench.profiled_traffic(str(tmp_path / "missing.md")) is None
