"""The committed ncu summaries stay reproducible from committed files: every
summary gives its command, the command runs `python bench.py` with options
bench.py accepts (and a workload it defines), every ncu line keeps the
clocks unlocked (--clock-control none), profiles/ holds summaries only (no
raw reports), and every DRAM-traffic entry of profiles/traffic.json points at
a summary that exists and at kernel sources that exist. No GPU needed."""
import json
import os
import re
import shlex

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def summaries():
    return sorted(f for f in os.listdir(PROFILES) if f.endswith(".md"))


def command_block(path):
    text = open(path).read()
    m = re.search(r"```\n(.*?)```", text, flags=re.S)
    assert m, f"{path}: no command block"
    return m.group(1).replace("\\\n", " ")


@pytest.fixture(scope="module")
def bench_parser():
    import bench
    return bench


@pytest.mark.parametrize("name", summaries())
def test_summary_command_runs_committed_files(name, bench_parser):
    cmd = command_block(os.path.join(PROFILES, name))
    assert "_work" not in cmd and "run_case" not in cmd
    parts = [p.strip() for p in cmd.split("&&")]
    assert parts, name
    for part in parts:
        toks = shlex.split(part.split(">")[0])
        if toks and toks[0] == "ncu":
            assert "--clock-control" in toks and \
                toks[toks.index("--clock-control") + 1] == "none", name
            i = toks.index("python")
            toks = toks[i:]
        assert toks[:2] == ["python", "bench.py"], (name, part)
        args = toks[2:]
        if "--workload" in args:
            wl = args[args.index("--workload") + 1]
            assert wl in bench_parser.WORKLOADS, (name, wl)
        for a in args:
            if a.startswith("--"):
                assert a in ("--workload", "--fmt", "--n", "--k", "--batch",
                             "--steps", "--warmup", "--no-cpu-baseline",
                             "--planes", "--lut-rows", "--force-path",
                             "--gpus"), (name, a)


def test_profiles_hold_summaries_only():
    # raw reports (.ncu-rep, .nsys-rep) stay out of the repository
    for f in os.listdir(PROFILES):
        assert f.endswith((".md", ".txt", ".json")), f


def test_traffic_entries_point_at_existing_captures():
    table = json.load(open(os.path.join(PROFILES, "traffic.json")))
    assert table
    for key, e in table.items():
        cap = e["capture"].split(" ")[0]
        assert os.path.exists(os.path.join(ROOT, cap)), (key, cap)
        for f in e["files"]:
            assert os.path.exists(os.path.join(
                ROOT, "packed_weight_matmul_b200", "csrc", f)), (key, f)
        assert 0.9 < e["dram_bytes_per_unit"] < 2.0, key
        assert re.fullmatch(r"[0-9a-f]{16}", e["source_hash"]), key
