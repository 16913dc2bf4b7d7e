"""Host logic of the benchmark that needs no GPU: the FLOPs accounting of the
layer and the rank of the FLOPs-matched static baseline ([DyRA] App. E.4:
a static low-rank layer of rank r + k + k' with the same FLOPs as DyRA)."""

import dataclasses
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from synth import CONFIGS  # noqa: E402


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_static_matched_rank(name):
    s = CONFIGS[name]
    rs = bench.static_matched_rank(s)
    _, _, dyra_flops, _ = bench.algorithmic(s)
    per_rank = 2.0 * s.N * (s.d_in + s.d_out)
    cap = min(s.d_in, s.d_out) // 8 * 8
    assert rs % 8 == 0
    # the static layer has at least the ranks DyRA applies (r static + k correction)
    assert s.r + s.k <= rs <= cap
    # the largest multiple of 8 whose FLOPs do not exceed DyRA's, unless capped
    if rs < cap:
        assert rs * per_rank <= dyra_flops < (rs + 8) * per_rank
    else:
        assert rs * per_rank <= dyra_flops or rs == cap


def test_algorithmic_counts_the_correction():
    """With k = 0 the layer's FLOPs are exactly the static part's."""
    s = dataclasses.replace(CONFIGS["vit_fc1"], k=0)
    flops, _, total, _ = bench.algorithmic(s)
    assert flops["gram"] == 0 and flops["solve"] == 0 and flops["rfactor"] == 0
    assert total == pytest.approx(2.0 * s.N * s.r * (s.d_in + s.d_out))


def _run_reference(env_extra, workload="tiny_f32"):
    import json
    import subprocess
    env = dict(os.environ, **env_extra)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", workload, "--steps", "3", "--warmup", "3"],
                         cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    return [json.loads(l) for l in lines]


def test_reference_arm_prints_the_contract_line():
    """The reference arm (the fp64 oracle on the host cores) prints one JSON
    line with the keys the benchmark contract names, on the workload asked."""
    (line,) = _run_reference({"RANK": "0", "WORLD_SIZE": "1"})
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 3
    assert line["config"]["workload"] == "tiny_f32" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_other_ranks_do_no_work():
    assert _run_reference({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_reference_arm_config_matches_the_gpu_arm():
    """Both arms build `config` from the same function, so the driver compares
    lines on identical configurations."""
    (line,) = _run_reference({"RANK": "0", "WORLD_SIZE": "1"})
    assert line["config"] == bench.config_of("tiny_f32", 1)


def test_vit_block_runs_the_four_block_linears_in_order():
    names = [s.name for s in bench.specs_of("vit_block")]
    assert names == ["vit_block_qkv", "vit_block_proj", "vit_block_fc1", "vit_block_fc2"]
    c = bench.config_of("vit_block", 1)
    assert [l["name"] for l in c["layers"]] == names and c["rows"] == 64 * 201
    assert "vit_block" in bench.workload_names()
    assert set(CONFIGS) < set(bench.workload_names())


def test_headline_is_the_largest_single_gpu_configuration():
    """The default workload is the configuration with the most dense FLOPs."""
    big = max(CONFIGS.values(), key=lambda s: s.N * s.d_in * s.d_out)
    assert bench.HEADLINE == big.name


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_parity_rows_are_valid_and_cover_whole_instances(name):
    s = CONFIGS[name]
    rows = bench.parity_rows(s)
    assert rows.ndim == 1 and len(rows) > 0
    assert rows.min() >= 0 and rows.max() < s.N and len(np.unique(rows)) == len(rows)
    if s.N <= 1024:
        assert len(rows) == s.N
    elif s.B > 1:
        # whole leading instances
        assert len(rows) % s.T == 0 and rows[-1] == len(rows) - 1
    else:
        # a single long instance: its first and last rows (the ragged tail) are checked
        assert rows[0] == 0 and rows[-1] == s.N - 1


def test_launch_count_per_forward():
    assert bench.launches_per_forward(CONFIGS["vit_fc1"]) == 5
    assert bench.launches_per_forward(dataclasses.replace(CONFIGS["vit_fc1"], k=0)) == 2
    assert bench.launches_per_forward(CONFIGS["tiny_f32"]) == 7
