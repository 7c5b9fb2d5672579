"""GPU parity of the Low-Rank Bypass step (qstate_lrb_decode_step) against the
oracle's qo_lrb_step: codes bit-exact, scales, readouts, and the bypass
buffers (accumulated decay, decayed keys, coefficients) bit-exact, over more
than two periods, in lock-step and in free run."""
import numpy as np
import pytest

from oracle import oracle as O
from ssm_decode_step_b200 import Config
from tests import parity as P

pytestmark = pytest.mark.gpu

# (bits, dk, dv, group, delta, decay, policy, rounding, tiles, rank)
CASES = [
    (4, 128, 128, 32, 1, "scalar", "dynamic", "nearest", 67, 4),
    (4, 128, 128, 32, 1, "scalar", "persistent", "bdr", 33, 8),
    (4, 128, 64, 32, 0, "diagonal", "persistent", "bdr", 29, 3),
    (8, 128, 64, 64, 0, "scalar", "persistent", "nearest", 40, 16),
    (4, 128, 128, 32, 1, "scalar", "yoked", "nearest", 21, 5),
    (8, 64, 48, 32, 1, "diagonal", "dynamic", "bdr", 9, 2),
    (4, 64, 16, 64, 0, "scalar", "yoked", "bdr", 7, 6),
    (8, 128, 32, 128, 1, "diagonal", "yoked", "bdr", 5, 7),
    (4, 128, 16, 32, 1, "diagonal", "persistent", "nearest", 3, 12),
    (4, 128, 4096, 32, 1, "scalar", "persistent", "bdr", 2, 4),   # the largest Dv
]


def _id(c):
    b, dk, dv, g, de, dc, pol, r, T, R = c
    return f"int{b}-dk{dk}-dv{dv}-g{g}-{'delta' if de else 'linear'}-{dc}-{pol}-{r}-T{T}-R{R}"


def _run(case, lockstep):
    import torch
    from ssm_decode_step_b200 import qstate as Q
    b, dk, dv, g, de, dc, pol, r, T, R = case
    cfg = Config(T, dk, dv, b, g, de, dc, pol, r)
    rng = np.random.default_rng(sum(map(ord, _id(case))))
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    gpu = P.GpuRun(cfg, S0)
    buf = Q.LrbBuffers(cfg, R)
    ocfg = P.oracle_cfg(cfg)
    ora = O.init(ocfg, S0)
    obuf = O.LrbBuffers(ocfg, R)
    steps = P.random_steps(rng, T, dk, dv, dc, 2 * R + R // 2 + 1, scale=0.3)
    for t, (q, k, v, a, bb) in enumerate(steps):
        if lockstep:
            c, s, sh = gpu.state()
            ora = O.State(ocfg, O.unpack(b, c.reshape(-1, c.shape[-1]), dk).reshape(T, dv, dk), s, sh)
        o_ref, pre = O.lrb_step(ora, obuf, q, k, v, a, bb, want_pre=True)
        o = torch.empty((T, dv), dtype=torch.float32, device="cuda")
        buf.step(gpu.st, gpu.t(q), gpu.t(k), gpu.t(v), gpu.t(a), gpu.t(bb), o)
        c, s, sh = gpu.state()
        rep = P.compare_state(cfg, c, s, ora, pre, f"{_id(case)} step {t}")
        assert rep.code_flips == 0, rep
        if sh is not None:
            assert np.array_equal(sh, ora.shadow), f"step {t}: shadow"
        P.compare_readout(o.cpu().numpy(), o_ref, f"{_id(case)} step {t}")
        if buf.slot > 0:   # after a bypass step the buffers hold the period so far
            n = buf.slot
            assert np.array_equal(buf.A[buf.cur].cpu().numpy(), obuf.A), f"step {t}: A"
            assert np.array_equal(buf.K[buf.cur][:, :n].cpu().numpy(), obuf.K[:, :n]), f"step {t}: K"
            assert np.array_equal(buf.U[:, :, :n].cpu().numpy(), obuf.U[:, :, :n]), f"step {t}: U"


@pytest.mark.parametrize("case", CASES, ids=_id)
def test_lrb_lockstep(case):
    _run(case, lockstep=True)


@pytest.mark.parametrize("case", CASES[:4], ids=_id)
def test_lrb_free_run(case):
    _run(case, lockstep=False)


def test_lrb_rank1_is_the_plain_step():
    import torch
    from ssm_decode_step_b200 import qstate as Q
    rng = np.random.default_rng(5)
    T, dk, dv = 11, 128, 64
    cfg = Config(T, dk, dv, 4, 32, 1, "scalar", "dynamic", "bdr")
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    a, b = P.GpuRun(cfg, S0), P.GpuRun(cfg, S0)
    buf = Q.LrbBuffers(cfg, 1)
    for q, k, v, al, be in P.random_steps(rng, T, dk, dv, "scalar", 3):
        a.step(q, k, v, al, be)
        buf.step(b.st, b.t(q), b.t(k), b.t(v), b.t(al), b.t(be), None)
        ca, sa, _ = a.state()
        cb, sb, _ = b.state()
        assert np.array_equal(ca, cb) and np.array_equal(sa, sb)


def test_lrb_without_readout():
    """Bypass and merge steps with the readout off (o = NULL: q is neither
    read nor staged) leave the same state and buffers as the oracle's steps."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    rng = np.random.default_rng(17)
    T, dk, dv, R = 23, 128, 64, 5
    for bits, dc in ((4, "scalar"), (8, "diagonal")):
        cfg = Config(T, dk, dv, bits, 32, 1, dc, "persistent", "bdr")
        S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
        gpu = P.GpuRun(cfg, S0)
        buf = Q.LrbBuffers(cfg, R)
        ocfg = P.oracle_cfg(cfg)
        ora = O.init(ocfg, S0)
        obuf = O.LrbBuffers(ocfg, R)
        for t, (q, k, v, a, bb) in enumerate(P.random_steps(rng, T, dk, dv, dc, 2 * R + 1, scale=0.3)):
            O.lrb_step(ora, obuf, q, k, v, a, bb)
            buf.step(gpu.st, gpu.t(q), gpu.t(k), gpu.t(v), gpu.t(a), gpu.t(bb), None)
            torch.cuda.synchronize()
            c, s, _ = gpu.state()
            rep = P.compare_state(cfg, c, s, ora, None, f"no readout int{bits} {dc} step {t}")
            assert rep.code_flips == 0, rep
            if buf.slot > 0:
                n = buf.slot
                assert np.array_equal(buf.A[buf.cur].cpu().numpy(), obuf.A), f"step {t}: A"
                assert np.array_equal(buf.K[buf.cur][:, :n].cpu().numpy(), obuf.K[:, :n]), f"step {t}: K"
                assert np.array_equal(buf.U[:, :, :n].cpu().numpy(), obuf.U[:, :, :n]), f"step {t}: U"
