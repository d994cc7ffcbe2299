"""bench.py's JSON line on the CPU: the reference arm (the oracle on the host
cores) runs without a GPU, so its line is checked for the contract's keys."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_k2", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny_k2"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_flop_accounting_counts_valid_token_pairs():
    # effective FLOPs = 4 d x (number of (query token, selected key token) pairs
    # over valid tokens)
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    from oracle import vsa_oracle as vo
    from video_dit_block_vsa_b200 import workloads as wl
    w = wl.Workload("t", 2, 3, 16, (5, 6, 7), 3, 9, 0.5, False)
    counts = bench.cube_counts(w.grid)
    assert np.array_equal(counts, vo.cube_permutation(w.grid)[1])
    rng = np.random.default_rng(0)
    C = counts.shape[0]
    sel = np.stack([np.sort(rng.choice(C, w.topk, replace=False)) for _ in range(2 * 3 * C)])
    sel = sel.reshape(2, 3, C, w.topk)
    eff, issued, coarse = bench.flop_counts(w, counts, sel)
    pairs = 0
    for b in range(2):
        for h in range(3):
            for i in range(C):
                for j in sel[b, h, i]:
                    pairs += int(counts[i]) * int(counts[j])
    assert eff == 4.0 * w.head_dim * pairs
    # issued: 64 query rows x the packed key rows (a selected cube with more
    # than 16 valid tokens costs 64 key rows, one with at most 16 costs 16)
    rows = 0
    for b in range(2):
        for h in range(3):
            for i in range(C):
                rows += sum(64 if counts[j] > 16 else 16 for j in sel[b, h, i])
    assert issued == 4.0 * w.head_dim * 64 * rows
    assert coarse == 4.0 * w.head_dim * 2 * 3 * C * C
