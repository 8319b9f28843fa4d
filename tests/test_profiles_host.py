"""Host-side checks of the committed ncu summaries and of how bench.py reads them
(no GPU): every summary gives the command that made it, with the clocks left
alone, and each full capture the source hash it was taken on; bench.py's
traffic lookup returns a positive byte count for a summary of the current
sources and None otherwise."""
import glob
import importlib.util
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def summaries():
    return sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def test_there_are_summaries():
    assert summaries()


@pytest.mark.parametrize("path", summaries(), ids=os.path.basename)
def test_summary_names_its_command_and_source(path):
    text = open(path).read()
    cmds = [line for line in text.splitlines() if line.strip().startswith("ncu ")]
    assert cmds, "no ncu command line"
    for line in cmds:
        assert "--clock-control none" in line
    # A full capture of a kernel records the sources it was taken on (a launch
    # list records shares only).
    if any("--set full" in line for line in cmds):
        assert re.search(r"source_sha256_16[^:]*:\s*[0-9a-f]{16}\b", text)
    # The profiled commands run committed files only.
    assert "_work" not in text


def test_source_sets_exist(bench):
    for names in (bench.GEMM_SOURCES, bench.DECODE_SOURCES):
        for name in names:
            assert os.path.exists(os.path.join(ROOT, "ternary_weight_linear_bitlinear_b200",
                                               "csrc", name)), name
        assert re.fullmatch(r"[0-9a-f]{16}", bench.source_sha(names))


def test_traffic_lookup(bench, tmp_path, monkeypatch):
    # A summary taken on the current sources yields its byte count; one taken on
    # other sources, or without the fields, yields None.
    sha = bench.source_sha(bench.GEMM_SOURCES)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "cur.md").write_text(
        "source_sha256_16: %s\ndram_bytes_per_launch: 1234\n" % sha)
    (tmp_path / "profiles" / "old.md").write_text(
        "source_sha256_16: 0000000000000000\ndram_bytes_per_launch: 1234\n")
    (tmp_path / "profiles" / "bare.md").write_text("nothing here\n")
    real_root = bench.ROOT
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # source_sha reads the kernel sources under ROOT: point it back at the repository.
    monkeypatch.setattr(bench, "source_sha", lambda names: _source_sha_at(real_root, names))
    assert bench.profile_traffic("cur.md", bench.GEMM_SOURCES) == 1234.0
    assert bench.profile_traffic("old.md", bench.GEMM_SOURCES) is None
    assert bench.profile_traffic("bare.md", bench.GEMM_SOURCES) is None
    assert bench.profile_traffic("missing.md", bench.GEMM_SOURCES) is None


def _source_sha_at(root, names):
    import hashlib
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(root, "ternary_weight_linear_bitlinear_b200", "csrc", name),
                  "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def test_committed_summaries_resolve(bench):
    # The summaries bench.py reads for its roofline lines exist and parse.
    for name, sources in (("gemm_tc_pair_prefill_2048x4096x11008.md", bench.GEMM_SOURCES),
                          ("decode_kernel_2560x6912_t1.md", bench.DECODE_SOURCES)):
        text = open(os.path.join(ROOT, "profiles", name)).read()
        m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
        assert m and float(m.group(1)) > 0
