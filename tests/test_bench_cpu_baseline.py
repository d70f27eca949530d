"""bench.py's CPU baselines run without a GPU: the whole-workload oracle step and the bounded
per-layer sample return a positive throughput, the thread count, and a description of what was
timed (small workloads: config 0, and config 1 cut to two layers)."""
import dataclasses
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_whole_workload_baseline_on_the_small_config():
    import bench
    import synth
    cfg = synth.config(0)
    tps, threads, sample = bench.oracle_full_step_tokens_per_s(cfg, 2.0, "exact")
    assert tps > 0 and threads >= 1
    assert "whole workload" in sample and f"{cfg.layers} layers" in sample


def test_whole_workload_baseline_with_groups_and_v():
    import bench
    import synth
    cfg = dataclasses.replace(synth.config(1), layers=2, groups=2, tokens=128)
    tps, threads, sample = bench.oracle_full_step_tokens_per_s(cfg, 2.0, "sketch")
    assert tps > 0 and threads >= 1
    assert "2 layer groups" in sample


def test_per_layer_sample_is_bounded():
    import bench
    import synth
    cfg = dataclasses.replace(synth.config(1), layers=3, tokens=128)
    tps, threads, sample = bench.oracle_sample_tokens_per_s(cfg, 2.0, "sketch", budget_s=0.0, max_s=5.0)
    assert tps > 0 and threads >= 1
    assert "single-group plan" in sample
