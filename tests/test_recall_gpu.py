"""The recall-over-horizon measurement (bench.py --recall) on a short
horizon: its FP32 probe leaves the state unchanged, its quantized and FP32
trajectories match the oracle's, and it reports every arm."""
import argparse
import json

import numpy as np
import pytest

import bench
from oracle import oracle as O
from ssm_decode_step_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_fp32_probe_leaves_state_unchanged():
    import torch
    from ssm_decode_step_b200 import qstate as Q
    w = W.get("recall")
    T, dk, dv = 16, w.dk, w.dv
    tiles = np.arange(T)
    kstar, vstar = W.probe(w, tiles)
    S0 = bench.plant(W.initial_state(w, tiles), kstar, vstar)
    cfg = Q.Config(T, dk, dv, 8, 32, 1, "scalar")
    S = torch.from_numpy(S0.copy()).cuda()
    o = torch.empty((T, dv), dtype=torch.float32, device="cuda")
    z = lambda *s: torch.zeros(s, dtype=torch.float32, device="cuda")
    Q.fp32_decode_step(cfg, S, torch.from_numpy(kstar).cuda(), z(T, dk), z(T, dv),
                       torch.ones(T, device="cuda"), z(T), o)
    assert np.array_equal(S.cpu().numpy(), S0)
    ocfg = O.OracleConfig(T, dk, dv, 8, 32, 1, "scalar", "persistent")
    ref = O.fp32_step(ocfg, S0.copy(), kstar, np.zeros((T, dk), np.float32),
                      np.zeros((T, dv), np.float32), np.ones(T, np.float32), np.zeros(T, np.float32))
    assert np.array_equal(o.cpu().numpy(), ref)
    # the planted association holds to float32 rounding
    assert np.abs(ref - vstar).max() < 1e-5 * np.abs(vstar).max()


def test_recall_measurement_runs(capsys):
    args = argparse.Namespace(recall_steps=16, pool=8, recall_tol=0.5, recall_lrb=4)
    bench.run_recall(args)
    line = capsys.readouterr().out.strip().splitlines()[-1]
    d = json.loads(line)
    assert d["checkpoints"] == [0, 1, 2, 4, 8, 16]
    names = {a.name for a in W.get("recall").arms}
    names |= {a.name + "+lrb4" for a in W.get("recall").arms if a.policy != "yoked"}
    assert set(d["arms"]) == names
    # a bypass arm's stored-state norm is taken at the ends of periods only
    assert d["arms"]["int4-g32-persistent+lrb4"]["norm_ratio_vs_fp32"][1] is None
    assert d["arms"]["int4-g32-persistent+lrb4"]["norm_ratio_vs_fp32"][3] is not None
    # at t = 0 every arm holds the planted state up to its quantization error
    assert d["fp32"]["recall_err_vs_vstar"][0] < 1e-5
    assert d["arms"]["int8-g32-dynamic"]["recall_err_vs_fp32"][0] < 0.05
    # the yoked arm's scale never feeds back on its codes: its norm tracks FP32
    assert abs(d["arms"]["int4-g32-yoked"]["norm_ratio_vs_fp32"][-1] - 1.0) < 0.2
