"""Host-side logic of bench.py that needs no GPU: the kernel-source hash that
ties a profile's DRAM traffic to the code it was captured on."""
import os
import shutil

import bench


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1; // trailing\n'
           'const char *s = "x // y /* z */";  /* block\n   over lines */ int b;\n'
           "char q = '\"'; char e = '\\''; const char *t = \"say \\\"//\\\"\";\n"
           '/* only a comment */\n')
    out = bench.strip_comments(src)
    assert "trailing" not in out and "block" not in out and "only a comment" not in out
    assert '"x // y /* z */"' in out
    assert "char q = '\"';" in out and "char e = '\\'';" in out
    assert 'const char *t = "say \\"//\\"";' in out
    assert "int a = 1;" in out and "int b;" in out


def _hash_of_tree(monkeypatch, root):
    monkeypatch.setattr(bench, "ROOT", root)
    return bench.kernel_source_hash()


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    csrc = os.path.join(bench.ROOT, "head_sparse_decode_b200", "csrc")
    copy = tmp_path / "head_sparse_decode_b200" / "csrc"
    shutil.copytree(csrc, copy)
    base = _hash_of_tree(monkeypatch, str(tmp_path))

    target = copy / "sha_schedule.cuh"
    text = target.read_text()
    target.write_text("// a new comment line\n\n" + text.replace(
        "namespace sha {", "namespace sha {  /* reworded */", 1))
    assert _hash_of_tree(monkeypatch, str(tmp_path)) == base

    target.write_text(text.replace("constexpr int kMaxBlocks = 4096;",
                                   "constexpr int kMaxBlocks = 4095;", 1))
    assert _hash_of_tree(monkeypatch, str(tmp_path)) != base


def test_step_distribution_percentiles():
    # 41 graph replays with per-call times 100..140 us: p10/median/p90 by rank
    per_step = [1e-6 * x for x in range(140, 99, -1)]
    d = bench.step_distribution(per_step, 100)
    assert d == {"p10_us": 104.0, "median_us": 120.0, "p90_us": 136.0, "graph_replays": 41,
                 "calls_per_replay": 100}
    assert bench.step_distribution([], 100) is None
    one = bench.step_distribution([2.5e-4], 7)
    assert one["p10_us"] == one["median_us"] == one["p90_us"] == 250.0
    assert one["calls_per_replay"] == 7
