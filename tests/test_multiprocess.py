"""The multi-rank plumbing of bench.py on CPU: two gloo ranks agree on the slowest rank's time,
and only rank 0 runs and prints the reference arm."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
import synth
from mp_workers import max_over_ranks_worker


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    values = [3.25, 7.5]
    mp.start_processes(max_over_ranks_worker, args=(2, free_port(), values, str(tmp_path)), nprocs=2,
                       join=True, start_method="spawn")
    for r in range(2):
        assert float(open(tmp_path / f"rank{r}.txt").read()) == max(values)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(1.5, 1) == 1.5


class Args:
    gpus, steps, warmup, seq = 2, 1, 0, 0


def test_reference_arm_only_rank0_prints(monkeypatch, capsys):
    w = synth.WORKLOADS["moe_t1_h1024_e32_k4_i256_int4"]
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(Args, w)
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(Args, w)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.metric_name(w)
    assert line["config"] == bench.base_config(w, 2) and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
