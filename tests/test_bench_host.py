"""Host-side logic of bench.py: the code hash that keys the committed DRAM
traffic records, and the lookup that returns a record only while the kernel's
code is the one the counters were taken on."""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


SRC = """// header comment
#include "x.h"
/* block
   comment */
__device__ int f(int a) {  // trailing comment
  const char* s = "not // a comment";
  char c = '/';
  return a + 1;
}
"""


def test_code_sha1_ignores_comments_and_blank_lines(bench):
    edited = SRC.replace("// header comment", "// a different,\n// longer header comment\n")
    edited = edited.replace("/* block\n   comment */", "")
    edited = edited.replace("// trailing comment", "")
    assert bench.code_sha1(edited) == bench.code_sha1(SRC)


@pytest.mark.parametrize("change", [
    ("a + 1", "a + 2"),                          # arithmetic
    ('"not // a comment"', '"not // a Comment"'),  # inside a string that holds //
    ("'/'", "'*'"),                              # a character literal
    ("int a", "int  a"),                         # whitespace inside a code line
])
def test_code_sha1_sees_code_changes(bench, change):
    assert change[0] in SRC
    assert bench.code_sha1(SRC.replace(*change)) != bench.code_sha1(SRC)


def test_load_traffic_matches_only_the_recorded_code(bench, tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cuh").write_text(SRC)
    rec = {"kern": {"wl": {"bytes": 123.0, "code_sha1": bench.code_sha1(SRC), "source": "k.cuh"}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("kern", "wl") == 123.0
    assert bench.load_traffic("kern", "other") is None
    (tmp_path / "k.cuh").write_text("// comment edit only\n" + SRC)
    assert bench.load_traffic("kern", "wl") == 123.0
    (tmp_path / "k.cuh").write_text(SRC.replace("a + 1", "a - 1"))
    assert bench.load_traffic("kern", "wl") is None


def test_committed_traffic_records_name_existing_sources(bench):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    for kernel, per_wl in recs.items():
        if kernel.startswith("_"):
            continue
        for wl, rec in per_wl.items():
            assert os.path.isfile(os.path.join(ROOT, rec["source"])), (kernel, wl)
            assert len(rec["code_sha1"]) == 40 and rec["bytes"] > 0, (kernel, wl)
