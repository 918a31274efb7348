"""Host logic of the offline sweep and of the compiled configuration table,
checked without a GPU: the winner rule (stream-K must win by a margin), the
table writer's output (it compiles as C++ and reads back the same rows), and
that the library's configuration choice honours every committed table row."""
import os
import re
import shutil
import subprocess

import pytest

from tensor_core_gemm_fp16_b200 import binding
from tensor_core_gemm_fp16_b200 import sweep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ROW = re.compile(r"^\s*\{(-?\d+), (-?\d+), (-?\d+), (-?\d+), (-?\d+), (-?\d+)\},")


def _row(cfg, split, ms, **kw):
    return {"config": cfg, "split": split, "ms": ms, "tflops": 1.0, **kw}


def test_pick_best_handicaps_stream_k():
    tiles = _row(3, 1, 1.00e-2)
    assert sweep.pick_best([tiles, _row(4, 2, 0.98e-2)])["config"] == 3     # 2% faster: not enough
    assert sweep.pick_best([tiles, _row(4, 2, 0.95e-2)])["config"] == 4     # 5% faster: wins
    assert sweep.pick_best([tiles, _row(5, 1, 0.99e-2)])["config"] == 5     # whole tiles: plain min
    assert sweep.pick_best([{"config": 1, "split": 1, "error": "x"}, tiles])["config"] == 3
    assert sweep.pick_best([{"config": 1, "split": 1, "error": "x"}]) is None


def _parse(path):
    rows = []
    with open(path) as f:
        for line in f:
            m = ROW.match(line)
            if m:
                rows.append(tuple(int(g) for g in m.groups()))
    return rows


def test_table_writer_round_trip(tmp_path):
    results = [
        {"shape": "a", "M": 64, "N": 128, "K": 256, "epilogue": 2, "best": 3, "best_split": 1,
         "rows": [_row(3, 1, 1e-2), _row(3, 2, 2e-2)]},
        {"shape": "b", "M": 7, "N": 9, "K": 11, "epilogue": 0, "best": 4, "best_split": 2,
         "rows": [_row(4, 2, 1e-3)]},
        {"shape": "none", "M": 1, "N": 1, "K": 1, "epilogue": 0, "best": None,
         "best_split": None, "rows": []},
    ]
    out = tmp_path / "t.inc"
    sweep.write_table(results, path=str(out))
    assert _parse(out) == [(64, 128, 256, 2, 3, 1), (7, 9, 11, 0, 4, 2), (-1, -1, -1, -1, -1, -1)]
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    src = tmp_path / "t.cc"
    src.write_text("#include <cstdint>\nstruct TableRow { int64_t M, N, K; int epilogue; "
                   "int config; int split; };\n#include \"t.inc\"\n"
                   "int main() { return kShapeTable[2].M == -1 ? 0 : 1; }\n")
    exe = tmp_path / "t"
    subprocess.run([cxx, "-std=c++17", "-Wall", "-Werror", "-I", str(tmp_path), str(src), "-o",
                    str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0


def test_committed_table_rows_are_what_the_library_picks():
    path = os.path.join(ROOT, "tensor_core_gemm_fp16_b200", "csrc", "tg_configs.inc")
    rows = _parse(path)
    assert rows and rows[-1] == (-1, -1, -1, -1, -1, -1)
    n_cfg = binding.tg_num_configs()
    for M, N, K, epi, cfg, split in rows[:-1]:
        assert 0 <= cfg < n_cfg and split in (1, 2)
        got = binding.tg_gemm_select_config(M, N, K, max(epi, 0))   # -1: any epilogue
        assert (got["id"], got["split"]) == (cfg, split), (M, N, K, epi)


def test_partial_sweep_keeps_the_other_rows(tmp_path):
    """A sweep of some shapes rewrites their rows and, with keep, leaves the
    table's other rows (and their comments) as they were."""
    committed = sweep.read_table()
    assert len(committed) >= 2 and all(len(r) == 7 for r in committed)
    first = committed[0]
    results = [{"shape": "new", "M": first[0], "N": first[1], "K": first[2],
                "epilogue": first[3], "best": 1, "best_split": 2,
                "rows": [_row(1, 2, 1e-2)]}]
    out = tmp_path / "t.inc"
    sweep.write_table(results, path=str(out), keep=committed)
    merged = sweep.read_table(str(out))
    assert merged[0][:6] == first[:4] + (1, 2)
    assert merged[1:] == committed[1:]
    sweep.write_table(results, path=str(out))
    assert len(sweep.read_table(str(out))) == 1


def test_cost_rule_is_close_to_the_sweep_on_shapes_outside_the_table():
    """Shapes missing from the table get the cost rule's choice.  On a set of
    such shapes swept on a B200 (offtable_sweep.json: every configuration and
    work division, timed), the rule's (configuration, split) must be within
    20% of the fastest, and within 8% on average."""
    import json
    path = os.path.join(ROOT, "tensor_core_gemm_fp16_b200", "offtable_sweep.json")
    with open(path) as f:
        shapes = json.load(f)["shapes"]
    assert len(shapes) >= 8
    ratios = []
    for s in shapes:
        assert (s["M"], s["N"], s["K"]) not in {(r[0], r[1], r[2]) for r in sweep.read_table()}
        best = min(r["us"] for r in s["rows"])
        c = binding.tg_gemm_select_config(s["M"], s["N"], s["K"], s["epilogue"], 148)
        mine = [r["us"] for r in s["rows"] if r["config"] == c["id"] and r["split"] == c["split"]]
        assert mine, f"{s['shape']}: the rule's choice was not swept"
        ratios.append(mine[0] / best)
        assert mine[0] <= 1.2 * best, f"{s['shape']}: rule {mine[0]} us vs best {best} us"
    assert sum(ratios) / len(ratios) <= 1.08, ratios
