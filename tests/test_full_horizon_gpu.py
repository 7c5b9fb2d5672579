"""Full-horizon parity at full size: the CUDA decode step runs every tile of
each workload over its whole decode horizon, and the CPU oracle follows
independently (free run: the two never exchange state), on

* the Gated DeltaNet-, Mamba-2- and GLA-shaped workloads: every tile for the
  first 64 steps, and 16 seeded tiles (the last tile among them) over the
  full 2048 / 1024 / 4096 steps;
* the 24-layer stack: 8 seeded tiles over all 32768 steps, both arms.

Tiles are independent recurrences, so a sampled tile is an exact check of
that tile.  Inputs cycle a pool of 64 slots of the workload's draw, as the
benchmark's do.  The dynamic policy feeds the state back into its scale
("When Dynamic Scaling Fails", project page), so a single late rounding
difference would show as diverging codes; the expectation under the shared
fixed operation order is none: codes and the yoked shadow bit for bit at
every checkpoint, scales within 1e-6, readouts within 1e-4 of the tile's
largest at every step.

Cost on the GPU machine (16 host cores): the oracle runs about 14 ns per state
element and step per core; the largest part is the Mamba-2-shaped workload's
first 64 steps over all 16384 tiles (8.6e9 element-steps, under 10 s on 16
cores) and the stack's 8 tiles x 32768 steps x 2 arms (8.6e9, about 20 s on
8 cores); the GPU side is a few seconds per workload."""
import numpy as np
import pytest

from oracle import oracle as O
from ssm_decode_step_b200 import Config, workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

POOL = 64
ALL_TILE_STEPS = 64


def _checkpoints(H):
    return sorted({1, 8, ALL_TILE_STEPS, 128, 512, H // 2, H} & set(range(1, H + 1)))


def _full_horizon(wname, n_sample, all_tiles):
    w = W.get(wname)
    H = w.steps
    dev = torch.device("cuda")
    rng = np.random.default_rng(1000 + W.ORDER.index(wname))
    sample = np.sort(rng.choice(w.tiles, size=n_sample, replace=False))
    sample[-1] = w.tiles - 1
    host = W.pool(w, POOL)
    pool = [torch.from_numpy(a).to(dev) for a in host]
    sub = [np.ascontiguousarray(a[:, sample]) for a in host]
    S0 = W.initial_state(w)
    idx = torch.as_tensor(sample, device=dev)
    checks = _checkpoints(H)
    for arm in w.arms:
        cfg = Config(w.tiles, w.dk, w.dv, arm.bits, arm.group, w.delta, w.decay, arm.policy,
                     arm.rounding)
        label = f"{wname} {arm.name}"
        gpu = P.GpuRun(cfg, S0)
        ora_s = O.init(P.oracle_cfg(cfg, len(sample)), np.ascontiguousarray(S0[sample]))
        ora_a = O.init(P.oracle_cfg(cfg), S0) if all_tiles else None
        o = torch.empty((w.tiles, w.dv), dtype=torch.float32, device=dev)
        o_s = torch.empty((H, len(sample), w.dv), dtype=torch.float32, device=dev)
        refs = np.empty((H, len(sample), w.dv), np.float32)
        worst = 0.0
        for t in range(H):
            s = t % POOL
            gpu.st.step(pool[0][s], pool[1][s], pool[2][s], pool[3][s], pool[4][s], o)
            torch.index_select(o, 0, idx, out=o_s[t])
            refs[t] = O.step(ora_s, *(a[s] for a in sub))
            if ora_a is not None and t < ALL_TILE_STEPS:
                o_all = O.step(ora_a, *(a[s] for a in host))
                worst = max(worst, P.compare_readout(o.cpu().numpy(), o_all, f"{label} step {t} all tiles"))
                if t + 1 in checks:
                    c, sc, sh = gpu.state()
                    rep = P.compare_state(cfg, c, sc, ora_a, None, f"{label} step {t + 1} all tiles")
                    assert rep.code_flips == 0, rep
                    if sh is not None:
                        assert np.array_equal(sh, ora_a.shadow), f"{label} step {t + 1}: shadow"
            if t + 1 in checks:
                c, sc, sh = gpu.state(sample)
                rep = P.compare_state(cfg, c, sc, ora_s, None, f"{label} step {t + 1} sampled tiles")
                assert rep.code_flips == 0, rep
                if sh is not None:
                    assert np.array_equal(sh, ora_s.shadow), f"{label} step {t + 1}: shadow"
        # every step's readouts of the sampled tiles, gathered on the device
        got = o_s.cpu().numpy()
        for t in range(H):
            worst = max(worst, P.compare_readout(got[t], refs[t], f"{label} step {t} sampled tiles"))
        assert worst <= P.READOUT_REL
        del gpu
        torch.cuda.empty_cache()


@pytest.mark.parametrize("wname", ["gdn", "mamba2", "gla"])
def test_full_horizon_all_tiles_then_sampled(wname):
    _full_horizon(wname, 16, all_tiles=True)


def test_full_horizon_stack24():
    _full_horizon("stack24", 8, all_tiles=False)
