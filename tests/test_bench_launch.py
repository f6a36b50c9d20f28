"""bench.py's multi-GPU plumbing on CPU: `--gpus 2` starts two ranks itself
(through torch.distributed.run) and the ranks' parts of every workload cover
each expert, row and calibration token exactly once; and a strong-scaling
step split over two gloo ranks (with a host stand-in for the four library
calls) gives the one-process results: the same per-group outputs for every
expert and row, the same imatrix after the all-reduce of the token shards,
and the same whole-matrix (num, den) after the all-reduce of the row shards."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import dist_workers
from test_dist_gloo import _port, _run

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_gpus_2_launches_two_ranks_that_cover_every_unit_once():
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--plan-only", "--scale", "0.05"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(line) == 1, r.stdout            # rank 0 alone prints
    d = json.loads(line[0])
    assert d["world"] == 2
    assert set(d["plan"]) == {"c0", "c1", "c2", "c3", "c4"}
    for name, p in d["plan"].items():
        assert p["covered_once"], name
        assert [g["rank"] for g in p["ranks"]] == [0, 1]
    # MoE stacks split by experts, dense matrices by rows with their tokens
    assert {pc[0] for g in d["plan"]["c4"]["ranks"] for pc in g["pieces"]} == {"experts"}
    assert {pc[0] for g in d["plan"]["c3"]["ranks"] for pc in g["pieces"]} == {"rows"}
    assert set(d["plan"]["c3"]["ranks"][0]["tokens"]) == {"qkv_in", "o_in", "gateup_in", "down_in"}


def test_gpus_must_match_the_launcher():
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--plan-only"], cwd=ROOT, capture_output=True,
                       text=True, timeout=120, env=dict(os.environ, WORLD_SIZE="3", CUDA_VISIBLE_DEVICES=""))
    assert r.returncode != 0 and "launcher started 3 ranks" in r.stderr


@pytest.mark.parametrize("config", ["c2", "c3"])
def test_sharded_step_equals_one_process(tmp_path, config):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    codes = _run(dist_workers.bench_sharded_step, (_port(), ROOT, str(tmp_path), config), world=2, timeout=240)
    assert codes == [0, 0]
    parts = [np.load(tmp_path / f"s{r}.npy", allow_pickle=True)[0] for r in range(2)]
    wl = synth.make(config, "cpu", seed=0, scale=0.05)
    step = bench.Step(dist_workers._HostStandIn(), wl, bench.make_sets(wl, 1))
    step(0)
    for k, u in enumerate(step.units):
        got_s, got_px = [], []
        for p in parts:
            axis, a, b, n = p["pieces"][k]
            got_s.append(p["scales"][k])
            got_px.append(p["px"][k])
        whole_s = step.res[k].scales.numpy()
        whole_px = np.stack([step.px[k][0].numpy(), step.px[k][1].numpy()])
        if axis == "experts":            # each rank owns whole experts: outputs concatenate along E
            assert np.array_equal(np.concatenate(got_s, axis=0), whole_s)
            assert np.array_equal(np.concatenate(got_px, axis=1), whole_px)
        else:                            # rows split: outputs concatenate along O; (num, den) all-reduced
            assert np.array_equal(np.concatenate(got_s, axis=1), whole_s)
            for g in got_px:            # m differs from the one-process m by fp32 rounding of the shard sums
                np.testing.assert_allclose(g, whole_px, rtol=1e-6)
    for site, m in step.m.items():
        for p in parts:
            if site in p["m"]:
                got = p["m"][site]
                if got.shape == m.shape:  # token-split site: every rank holds the all-reduced imatrix
                    np.testing.assert_allclose(got, m.numpy(), rtol=1e-6)
                else:                     # expert-split site: this rank's experts
                    assert got.shape[1] == m.shape[1]


def test_profile_table_rows_are_read_by_workload_and_kernel(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    got = bench.read_profile(os.path.join(ROOT, "profiles", "traffic.md"), "c2", "search int3_g64_sym")
    assert got["launches"] == 1 and got["traffic"] > 0 and got["ms"] > 0 and got["source"].endswith(".md")
    assert 0 < got["fp32_pipe_frac"] <= 1
    assert bench.read_profile(os.path.join(ROOT, "profiles", "traffic.md"), "c9", "k_proxy")["traffic"] is None
    t = tmp_path / "t.md"
    t.write_text("| c2 | k_proxy | 2 | 123 | 0.1 | - | x.md |\n")
    assert bench.read_profile(str(t), "c2", "k_proxy") == {"launches": 2, "traffic": 123, "ms": 0.1,
                                                          "fp32_pipe_frac": None, "source": "x.md"}


def test_config_dictionary_is_shared_by_both_arms():
    """The reference arm and the tq arm print the same config for the same
    workload, GPU count and scaling; weights and groups follow the shapes."""
    sys.path.insert(0, ROOT)
    import bench
    c = bench.config_dict("c2", 1.0, 1, "strong")
    assert c["weights"] == 64 * 2048 * 7168 and c["groups"] == 64 * 2048 * 112
    assert c["workload"].startswith("c2:") and "> 126 MiB L2" in c["l2"]
    assert bench.config_dict("c2", 1.0, 8, "strong")["weights"] == 64 * 2048 * 7168
    assert bench.config_dict("c2", 1.0, 8, "weak")["weights"] == 8 * 64 * 2048 * 7168
    assert bench.config_dict("c4", 1.0, 1, "strong")["groups"] == 128 * 1856 * 168
    assert bench.workload_weights("c3") == sum(o * i for _, o, i, _ in __import__("synth").C3_LINEARS)
