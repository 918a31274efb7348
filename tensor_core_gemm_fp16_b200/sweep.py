"""Offline schedule sweep: time every compiled configuration, dealing out
whole tiles and with stream-K, on each shape and (optionally) rewrite
csrc/tg_configs.inc with the winners.

    python -m tensor_core_gemm_fp16_b200.sweep [--shapes all|offtable|NAME ...]
        [--reps 30] [--splits 1 2] [--context] [--write] [--json out.json]

The tutorial sweeps tile sizes, pipeline stages, thread counts and an L2
swizzle by hand on its 2048^3 GEMM and keeps the fastest that also passes
its relative-Frobenius check ("Designing High-Performance GPU Kernels with
TileLang", thecryptopost.io, section 3 "Knobs"), noting that the best
schedule depends on the architecture and the shape.  This tool does the
same over this library's compiled configurations on B200: every candidate
is checked against torch's fp32 matmul of the same fp16 inputs (relative
Frobenius error < 2e-2, as in the tutorial's sweep) before it is timed, and
it is timed with CUDA events (L2 flushed before each launch when the
operands fit in L2).  The events on B200 tick in steps of about 2 us, so a
single launch's time is quantised; the mean over many launches, whose start
falls at random within a tick, resolves finer than a tick, and a median would
not.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
TABLE = os.path.join(HERE, "csrc", "tg_configs.inc")
L2_BYTES = 126 * 1024 * 1024

DEFAULT_SHAPES = {
    # name: (M, N, K, epilogue)
    "gemm_256": (256, 256, 256, 0),
    "gemm_2048": (2048, 2048, 2048, 0),
    "fused_2048": (2048, 2048, 2048, 2),
    "ragged_fused": (3000, 1537, 2050, 2),
    "fused_8192": (8192, 8192, 8192, 2),
    "gemm_8192": (8192, 8192, 8192, 0),
    "fused_tanh_2048": (2048, 2048, 2048, 3),
    "softmax_8192x256x4096": (8192, 256, 4096, 4),
    "deepk_fused_1024x1024x8192": (1024, 1024, 8192, 2),
    "deepk_512x512x16384": (512, 512, 16384, 0),
}


# Shapes that are not in the table, swept to check the cost rule that
# chooses for them (tests/test_sweep_host.py reads the committed results in
# offtable_sweep.json): squares between the table's sizes, wide and tall
# panels, a deep-K shape and unaligned pitches.
OFF_TABLE_SHAPES = {
    "fused_1024": (1024, 1024, 1024, 2),
    "fused_4096": (4096, 4096, 4096, 2),
    "gemm_1536x3072x2048": (1536, 3072, 2048, 0),
    "bias_512x4096x1024": (512, 4096, 1024, 1),
    "fused_6144x2048x512": (6144, 2048, 512, 2),
    "gemm_768x768x4096": (768, 768, 4096, 0),
    "fused_2500x999x2998": (2500, 999, 2998, 2),
    "gemm_4096x512x8192": (4096, 512, 8192, 0),
}


def time_config(torch, binding, a, b, bias, c, M, N, K, epi, cfg, reps, warmup, flush, gm=0,
                split=0):
    stream = torch.cuda.current_stream()
    args = (a.data_ptr(), b.data_ptr(), bias.data_ptr() if bias is not None else None,
            c.data_ptr(), M, N, K, epi)

    def launch():
        st = binding.tg_gemm_ex(*args, config_id=cfg, stream=stream.cuda_stream, group_m=gm,
                                split=split)
        if st != binding.TG_OK:
            raise binding.TgError(st, f"config {cfg}")

    for _ in range(warmup):
        launch()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        launch()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    st = binding.tg_gemm_check_error(stream.cuda_stream)
    if st != binding.TG_OK:
        raise binding.TgError(st, f"config {cfg}")
    return statistics.fmean(times)


def time_library(torch, a, b, bias, epi, reps, warmup, flush):
    """torch.matmul (cuBLAS) plus the eager bias + erf-GELU, for context only."""
    F = torch.nn.functional

    def run():
        if epi == 0:
            return a @ b
        y = torch.addmm(bias, a, b)
        if epi == 2:
            return F.gelu(y)
        if epi == 3:
            return F.gelu(y, approximate="tanh")
        if epi == 4:
            return torch.softmax(y, dim=1)
        return y

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.fmean(times)


def sweep_shape(torch, binding, name, M, N, K, epi, reps, warmup, configs, group_ms=(0,),
                context=False, rounds=5, splits=(1, 2)):
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(1234)
    a = torch.randn(M, K, device=dev, generator=g).half()
    b = (torch.randn(K, N, device=dev, generator=g) / math.sqrt(K)).half()
    bias = torch.randn(N, device=dev, generator=g).half() if epi else None
    c = torch.empty(M, N, device=dev, dtype=torch.float16)
    ref = a.float() @ b.float()
    F = torch.nn.functional
    if epi == 1:
        ref = ref + bias.float()
    elif epi == 2:
        ref = F.gelu(ref + bias.float())
    elif epi == 3:
        ref = F.gelu(ref + bias.float(), approximate="tanh")
    elif epi == 4:
        ref = torch.softmax(ref + bias.float(), dim=1)
    small = 2 * (M * K + K * N + M * N) <= L2_BYTES
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if small else None
    rows = []
    candidates = []
    for cfg, gm, split in [(c, g, sp) for c in configs for g in group_ms for sp in splits]:
        info = dict(binding.tg_config_info(cfg))
        if epi == 4 and (info["epi_warps"] != 4 or info["block_n"] < N):
            continue   # the row softmax needs whole rows per epilogue thread
        if gm:
            info["group_m"] = gm
        st = binding.tg_gemm_ex(a.data_ptr(), b.data_ptr(),
                                bias.data_ptr() if bias is not None else None, c.data_ptr(),
                                M, N, K, epi, config_id=cfg, group_m=gm, split=split,
                                stream=torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        if st != binding.TG_OK:
            rows.append({"config": cfg, "split": split, "error": binding.tg_status_string(st)})
            continue
        rel = float((c.float() - ref).norm() / ref.norm())
        if not rel < 2e-2:
            rows.append({"config": cfg, "split": split,
                         "error": f"numerically wrong (rel {rel:.2e})"})
            continue
        candidates.append((cfg, gm, split, info, rel))
    # Interleaved rounds: every candidate (and the library context) is timed
    # once per round, so slow drifts of the GPU's clock (power, temperature)
    # touch all of them alike; each result is the median over rounds of the
    # per-round means.
    per_round = {i: [] for i in range(len(candidates))}
    lib_rounds = []
    per = max(1, reps // rounds)
    for _ in range(rounds):
        if context:
            lib_rounds.append(time_library(torch, a, b, bias, epi, per, warmup, flush))
        for i, (cfg, gm, split, info, rel) in enumerate(candidates):
            per_round[i].append(time_config(torch, binding, a, b, bias, c, M, N, K, epi, cfg,
                                            per, warmup, flush, gm, split))
    lib_ms = statistics.median(lib_rounds) if context else None
    for i, (cfg, gm, split, info, rel) in enumerate(candidates):
        ms = statistics.median(per_round[i])
        rows.append({"config": cfg, "group_m_override": gm, "split": split, "ms": ms,
                     "tflops": 2.0 * M * N * K / (ms * 1e-3) / 1e12,
                     "rel_err": rel, **{k: info[k] for k in ("block_m", "block_n", "stages",
                                                           "cta_pair", "group_m", "epi_warps")}})
    best = pick_best(rows)
    return {"shape": name, "M": M, "N": N, "K": K, "epilogue": epi, "rows": rows,
            "best": best["config"] if best else None,
            "best_split": best["split"] if best else None,
            "best_group_m": best["group_m"] if best else None, "l2_flushed": small,
            "library_ms": lib_ms}


# Stream-K must beat whole tiles by this factor to be recorded: the event
# timer's resolution makes near-ties common, and whole tiles need no
# workspace and no cross-CTA exchange.
STREAM_K_MARGIN = 1.03


def pick_best(rows):
    """The fastest timed row, with stream-K handicapped by STREAM_K_MARGIN."""
    ok = [r for r in rows if "ms" in r]
    if not ok:
        return None
    return min(ok, key=lambda r: r["ms"] * (STREAM_K_MARGIN if r.get("split") == 2 else 1.0))


_TABLE_ROW = re.compile(r"^\s*\{(-?\d+), (-?\d+), (-?\d+), (-?\d+), (-?\d+), (-?\d+)\},"
                        r"\s*(//.*)?$")


def read_table(path=TABLE):
    """The rows of a configuration table file, each (M, N, K, epilogue, config,
    split, comment), sentinel excluded."""
    rows = []
    with open(path) as f:
        for line in f:
            m = _TABLE_ROW.match(line)
            if m and int(m.group(1)) >= 0:
                rows.append(tuple(int(g) for g in m.groups()[:6]) + ((m.group(7) or "").strip(),))
    return rows


def write_table(results, path=TABLE, keep=()):
    """Write the table: one row per swept shape with a winner, then the rows
    of `keep` (from read_table) whose shape this sweep did not cover."""
    lines = [
        "// tg_configs.inc -- per-shape configuration table.",
        "//",
        "// Rows: {M, N, K, epilogue (-1 = any), config id, split (1 whole tiles,",
        "// 2 stream-K)}.  A row matches a problem of exactly that shape.  Rows are",
        "// the winners of the offline sweep (tensor_core_gemm_fp16_b200/sweep.py),",
        "// which rewrites this file; shapes it does not list fall back to the cost",
        "// rule in tg_gemm.cu.  The last row is a sentinel (M = -1).",
        "//",
        "// Written by the sweep on a B200; per row: ms and TFLOP/s of the winner.",
        "static const TableRow kShapeTable[] = {",
    ]
    for r in results:
        if r["best"] is None:
            continue
        w = next(x for x in r["rows"]
                 if x["config"] == r["best"] and x.get("split") == r["best_split"] and "ms" in x)
        lines.append(f"    {{{r['M']}, {r['N']}, {r['K']}, {r['epilogue']}, {r['best']}, "
                     f"{r['best_split']}}},"
                     f"  // {r['shape']}: {w['ms'] * 1e3:.1f} us, {w['tflops']:.0f} TFLOP/s")
    swept = {(r["M"], r["N"], r["K"], r["epilogue"]) for r in results}
    for M, N, K, epi, cfg, split, comment in keep:
        if (M, N, K, epi) not in swept:
            lines.append(f"    {{{M}, {N}, {K}, {epi}, {cfg}, {split}}},"
                         + (f"  {comment}" if comment else ""))
    lines += ["    {-1, -1, -1, -1, -1, -1},", "};", ""]
    with open(path, "w") as f:
        f.write("\n".join(lines))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--shapes", nargs="*", default=["all"])
    ap.add_argument("--reps", type=int, default=30, help="launches per candidate in total")
    ap.add_argument("--rounds", type=int, default=5,
                    help="interleaved rounds over all candidates (reps are split among them)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--configs", type=int, nargs="*", default=None)
    ap.add_argument("--group-m", type=int, nargs="*", default=[0],
                    help="rasterisation panel heights to try (0: the configuration's own)")
    ap.add_argument("--splits", type=int, nargs="*", default=[1, 2],
                    help="work divisions to try (1 whole tiles, 2 stream-K)")
    ap.add_argument("--context", action="store_true",
                    help="also time torch.matmul (+ eager bias/GELU) on each shape")
    ap.add_argument("--write", action="store_true", help="rewrite csrc/tg_configs.inc")
    ap.add_argument("--keep-others", action="store_true",
                    help="with --write or --from-json: keep the table's rows for shapes this "
                         "sweep did not cover")
    ap.add_argument("--json", default=None)
    ap.add_argument("--from-json", default=None,
                    help="rewrite the table from a saved sweep (no GPU needed)")
    args = ap.parse_args(argv)
    if args.from_json:
        with open(args.from_json) as f:
            results = json.load(f)
        for r in results:
            best = pick_best(r["rows"])
            r["best"] = best["config"] if best else None
            r["best_split"] = best["split"] if best else None
        write_table(results, keep=read_table() if args.keep_others else ())
        return 0
    sys.path.insert(0, os.path.dirname(HERE))
    import torch
    from tensor_core_gemm_fp16_b200 import binding

    shapes = dict(DEFAULT_SHAPES, **OFF_TABLE_SHAPES)
    if args.shapes == ["all"]:
        names = list(DEFAULT_SHAPES)
    elif args.shapes == ["offtable"]:
        names = list(OFF_TABLE_SHAPES)
    else:
        names = args.shapes
    configs = args.configs if args.configs is not None else list(range(binding.tg_num_configs()))
    results = []
    for name in names:
        M, N, K, epi = shapes[name]
        r = sweep_shape(torch, binding, name, M, N, K, epi, args.reps, args.warmup, configs,
                        tuple(args.group_m), args.context, args.rounds, tuple(args.splits))
        results.append(r)
        print(f"== {name} ({M}x{N}x{K}, epilogue {epi}) best config {r['best']} "
              f"split {r['best_split']} group_m {r['best_group_m']}")
        if r["library_ms"] is not None:
            print(f"   torch/cuBLAS (context) {r['library_ms'] * 1e3:9.1f} us  "
                  f"{2.0 * M * N * K / (r['library_ms'] * 1e-3) / 1e12:7.1f} TFLOP/s")
        for row in r["rows"]:
            if "ms" in row:
                print(f"   cfg {row['config']:2d} split{row['split']}  BM{row['block_m']:4d} "
                      f"BN{row['block_n']:4d} "
                      f"st{row['stages']} pair{row['cta_pair']} g{row['group_m']:2d} "
                      f"ew{row['epi_warps']}  {row['ms'] * 1e3:9.1f} us  "
                      f"{row['tflops']:7.1f} TFLOP/s")
            else:
                print(f"   cfg {row['config']:2d} split{row['split']}  {row['error']}")
        sys.stdout.flush()
    if args.json:
        with open(args.json, "w") as f:
            json.dump(results, f, indent=1)
    if args.write:
        write_table(results, keep=read_table() if args.keep_others else ())
    return 0


if __name__ == "__main__":
    sys.exit(main())
