"""Benchmark command line (no GPU): workload selection and scaling, the
config block of the JSON line, and the help text."""
import argparse
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _args(**kw):
    base = dict(workload="glove", nq=None, leaves=None, n=None, num_leaves=None, lut_mode=0)
    base.update(kw)
    return argparse.Namespace(**base)


def test_default_workload_is_the_glove_configuration():
    w = bench.workload_spec(_args())
    assert (w.n, w.d, w.dims_per_block, w.num_leaves, w.num_leaves_to_search, w.nq, w.k, w.reorder_num) == \
        (1_000_000, 100, 2, 1000, 32, 1000, 10, 100)


def test_reduced_size_scales_partition_and_means():
    w = bench.workload_spec(_args(workload="openai", n=200_000, num_leaves=200, nq=2000))
    assert (w.n, w.num_leaves, w.nq, w.d, w.reorder_num) == (200_000, 200, 2000, 1536, 300)
    assert w.training_sample_size <= 200_000 and w.n_means == 200
    w = bench.workload_spec(_args(n=100_000))
    assert w.num_leaves == 100                       # scaled with n when not given


def test_config_block_names_the_workload():
    w = bench.workload_spec(_args(leaves=64))
    c = bench.config_dict(w, _args())
    assert c["num_leaves_to_search"] == 64 and c["lut_mode"] == "f32" and c["l2_flush_between_steps"]
    assert c["workload"].startswith("glove-shaped IVF-AH: n=1,000,000 d=100")
    assert "model" not in c


def test_traffic_only_for_the_default_batch():
    # the headline workload's scan traffic per step is at least the codes it reads
    # (384 MB for 2M points x 192 code bytes)
    assert ("openai", 0) in bench.SCAN_TRAFFIC_BYTES
    assert bench.SCAN_TRAFFIC_BYTES[("openai", 0)] > 384e6


def test_help_lists_the_modes():
    r = subprocess.run([sys.executable, "bench.py", "--help"], cwd=ROOT, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0
    for flag in ("--gpus", "--steps", "--warmup", "--impl", "--sweep", "--encode", "--kmeans", "--leaf-shards"):
        assert flag in r.stdout
