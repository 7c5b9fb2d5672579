"""GPU parity: the CUDA decode step (through the C ABI) against the CPU
oracle, element by element, on seeded inputs.

Sizes span several tiles per CTA (persistent grid) and a ragged tail; the
workloads' full sizes are covered on sampled tiles in the launch
configuration the benchmark times.
"""
import numpy as np
import pytest

from oracle import oracle as O
from ssm_decode_step_b200 import Config, workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

# (bits, dk, dv, group, delta, decay, policy, rounding, tiles)
CASES = [
    (4, 128, 128, 32, 1, "scalar", "persistent", "nearest", 333),
    (4, 128, 128, 32, 1, "scalar", "dynamic", "nearest", 301),
    (4, 128, 128, 32, 1, "scalar", "yoked", "nearest", 150),
    (8, 128, 64, 64, 0, "scalar", "persistent", "nearest", 300),
    (4, 128, 128, 32, 0, "diagonal", "persistent", "bdr", 151),
    (4, 128, 128, 32, 0, "diagonal", "dynamic", "bdr", 40),
    (4, 128, 128, 32, 1, "scalar", "persistent", "bdr", 40),
    (8, 128, 128, 32, 1, "scalar", "dynamic", "nearest", 40),
    (8, 64, 64, 64, 1, "scalar", "persistent", "nearest", 7),
    (4, 64, 48, 32, 1, "diagonal", "yoked", "bdr", 9),
    (8, 64, 16, 32, 0, "scalar", "dynamic", "bdr", 5),
    (4, 128, 16, 128, 1, "diagonal", "dynamic", "nearest", 11),
    (8, 128, 112, 128, 0, "diagonal", "yoked", "nearest", 13),
    (4, 64, 256, 64, 1, "scalar", "persistent", "bdr", 6),
    (8, 128, 32, 64, 1, "diagonal", "persistent", "nearest", 21),
    (4, 128, 80, 64, 0, "scalar", "yoked", "bdr", 17),
    (8, 64, 128, 32, 1, "diagonal", "dynamic", "bdr", 3),
    (4, 64, 64, 32, 0, "scalar", "dynamic", "nearest", 1),
]


def _id(c):
    b, dk, dv, g, de, dc, pol, r, T = c
    return f"int{b}-dk{dk}-dv{dv}-g{g}-{'delta' if de else 'linear'}-{dc}-{pol}-{r}-T{T}"


@pytest.mark.parametrize("case", CASES, ids=_id)
def test_lockstep(case):
    b, dk, dv, g, de, dc, pol, r, T = case
    cfg = Config(T, dk, dv, b, g, de, dc, pol, r)
    rng = np.random.default_rng(hash(_id(case)) % 2**32)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    steps = P.random_steps(rng, T, dk, dv, dc, 6, scale=0.5)
    rep = P.lockstep(cfg, S0, steps, label=_id(case))
    assert rep.code_flips == 0, rep
    # one more step without readout (o = NULL path)
    gpu = P.GpuRun(cfg, S0)
    ora = O.init(P.oracle_cfg(cfg), S0)
    q, k, v, a, bb = steps[0]
    gpu.step(None, k, v, a, bb, want_o=False)
    O.step(ora, q, k, v, a, bb, want_o=False)
    c, s, sh = gpu.state()
    P.compare_state(cfg, c, s, ora, None, "no readout")


def test_tiny_workload_full_horizon():
    """The tiny gated delta-rule workload, all tiles, all 256 steps, free-run:
    GPU and oracle never exchange state and must agree at every step."""
    w = W.get(0)
    arm = w.arms[0]
    cfg = Config(w.tiles, w.dk, w.dv, arm.bits, arm.group, w.delta, w.decay, arm.policy, arm.rounding)
    S0 = W.initial_state(w)
    steps = [W.slot(w, t) for t in range(w.steps)]
    rep = P.free_run(cfg, S0, steps, "tiny-gdn")
    assert rep.code_flips == 0
    assert rep.worst_o_rel <= P.READOUT_REL


@pytest.mark.parametrize("policy,rounding,bits", [("persistent", "bdr", 4), ("dynamic", "nearest", 4),
                                                  ("yoked", "nearest", 4), ("dynamic", "bdr", 8)])
def test_long_free_run(policy, rounding, bits):
    """A longer free run (512 steps) on a small gated delta-rule stack,
    including the dynamic policy whose scale feeds back on the state."""
    rng = np.random.default_rng(7)
    T, dk, dv = 12, 128, 64
    cfg = Config(T, dk, dv, bits, 32, 1, "scalar", policy, rounding)
    S0 = (rng.standard_normal((T, dv, dk)) / np.sqrt(dk)).astype(np.float32)
    steps = P.random_steps(rng, T, dk, dv, "scalar", 512)
    rep = P.free_run(cfg, S0, steps, f"long-{policy}-{rounding}")
    assert rep.code_flips == 0


@pytest.mark.parametrize("bits,dk,dv,group", [(4, 128, 128, 32), (8, 128, 64, 64), (4, 64, 64, 64),
                                              (8, 64, 32, 32)])
def test_readout_entry(bits, dk, dv, group):
    import torch
    from ssm_decode_step_b200 import qstate as Q
    rng = np.random.default_rng(bits * dk + dv)
    T = 157
    cfg = Config(T, dk, dv, bits, group, 1, "scalar", "persistent")
    S0 = (rng.standard_normal((T, dv, dk)) * 0.4).astype(np.float32)
    gpu = P.GpuRun(cfg, S0)
    q = rng.standard_normal((T, dk)).astype(np.float32)
    o = torch.empty((T, dv), dtype=torch.float32, device="cuda")
    Q.readout(cfg, gpu.st.codes, gpu.st.scales, gpu.t(q), o)
    ora = O.init(P.oracle_cfg(cfg), S0)
    ref = O.readout(ora, q)
    P.compare_readout(o.cpu().numpy(), ref, "readout")


def test_zero_tiles_is_a_noop():
    import torch
    from ssm_decode_step_b200 import qstate as Q
    cfg = Config(0, 128, 128, 4, 32, 1, "scalar", "persistent")
    e = torch.empty(0, device="cuda")
    Q.init(cfg, e, e, e)
    Q.decode_step(cfg, e, e, None, e, e, e, e, e, e)
    Q.readout(cfg, e, e, e, e)
    torch.cuda.synchronize()


def test_zero_state_and_zero_groups():
    """S0 = 0: every scale is 0 and every code 0 (zero-scale rule); the
    persistent state stays 0, the dynamic one picks up the first write."""
    rng = np.random.default_rng(3)
    T, dk, dv = 5, 128, 32
    S0 = np.zeros((T, dv, dk), np.float32)
    S0[1, :, 32:] = rng.standard_normal((dv, dk - 32)).astype(np.float32)   # one tile half zero
    steps = P.random_steps(rng, T, dk, dv, "scalar", 3)
    for pol in ("persistent", "dynamic", "yoked"):
        cfg = Config(T, dk, dv, 4, 32, 1, "scalar", pol, "bdr")
        P.lockstep(cfg, S0, steps, label=f"zero-{pol}")


def test_zero_update_keeps_persistent_codes():
    rng = np.random.default_rng(4)
    T, dk, dv = 9, 128, 128
    cfg = Config(T, dk, dv, 4, 32, 1, "scalar", "persistent")
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    gpu = P.GpuRun(cfg, S0)
    c0, s0, _ = gpu.state()
    q = rng.standard_normal((T, dk)).astype(np.float32)
    v = rng.standard_normal((T, dv)).astype(np.float32)
    gpu.step(q, np.zeros((T, dk), np.float32), v, np.ones(T, np.float32), np.full(T, 0.5, np.float32))
    c1, s1, _ = gpu.state()
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


def test_clipping_and_huge_updates():
    """Persistent and yoked scales clip; updates of millions of grid steps
    and overflowing values go through the clamping path.  The last step
    writes v = 3e38, so readouts overflow: the GPU must give NaN and
    infinities of the same sign exactly where the oracle does."""
    rng = np.random.default_rng(5)
    T, dk, dv = 6, 128, 64
    S0 = (rng.standard_normal((T, dv, dk)) * 1e-3).astype(np.float32)
    steps = P.random_steps(rng, T, dk, dv, "scalar", 3, scale=1.0)
    q, k, v, a, b = steps[1]
    steps[1] = (q, k, (v * 1e4).astype(np.float32), a, b)
    q, k, v, a, b = steps[2]
    steps[2] = (q, k, np.full_like(v, 3e38), a, np.ones_like(b))
    for pol in ("persistent", "yoked", "dynamic"):
        for rnd in ("nearest", "bdr"):
            cfg = Config(T, dk, dv, 8, 64, 0, "scalar", pol, rnd)
            P.lockstep(cfg, S0, steps, label=f"clip-{pol}-{rnd}")
            # the overflow step, free-run, with its readouts compared by pattern
            gpu = P.GpuRun(cfg, S0)
            ora = O.init(P.oracle_cfg(cfg), S0)
            for t, (q, k, v, a, b) in enumerate(steps):
                o = gpu.step(q, k, v, a, b)
                o_ref = O.step(ora, q, k, v, a, b)
                P.compare_readout(o, o_ref, f"clip-{pol}-{rnd} free step {t}")
            assert not np.all(np.isfinite(o_ref)), "the overflow step overflowed no readout"
            c, s_, sh = gpu.state()
            P.compare_state(cfg, c, s_, ora, None, f"clip-{pol}-{rnd} after the overflow step")


def _boundary_case(bits, T=4, dk=128, dv=64, group=32):
    """A state whose groups have power-of-two scales (one code of each group
    at qmax) and updates that put x / s' on half-integers (ties), on the
    range's edges and beyond it, under both update signs, with and without
    decay, then overflowing values."""
    qmax = 7 if bits == 4 else 127
    rng = np.random.default_rng(bits)
    e = 2.0 ** -3
    codes = rng.integers(-qmax, qmax + 1, size=(T, dv, dk))
    codes[:, :, ::group] = qmax                        # each group's maximum: s = 2^-3 exactly
    S0 = (codes * e).astype(np.float32)
    kpat = np.array([1.0, -1.0, 0.5, 0.0, -0.5, 2.0, -2.0, 0.25], np.float32)
    k = np.tile(kpat, (T, dk // 8))
    halves = np.arange(-(qmax + 3), qmax + 3) + 0.5    # ..., -q-2.5, ..., q+2.5
    far = np.array([-1e4, -3 * qmax, 3 * qmax, 1e4])
    h = np.concatenate([halves, far, -halves[::-1] * 2.0])
    v = np.resize(h, (T, dv)).astype(np.float64) * e
    q = rng.standard_normal((T, dk)).astype(np.float32)
    one, half = np.ones(T, np.float32), np.full(T, 0.5, np.float32)
    steps = [(q, k, v.astype(np.float32), one, one),
             (q, -k, (v[:, ::-1] * 0.75).astype(np.float32), half, one),
             (q, k, np.where(np.arange(dv) % 2 == 0, 3e38, -3e38)[None, :].repeat(T, 0).astype(np.float32),
              one, one)]
    return S0, steps


@pytest.mark.parametrize("bits", [4, 8])
def test_rounding_boundaries_and_saturation(bits):
    """Ties (x / s' on half-integers) round to even, values on and beyond
    the range's edges clamp to +-qmax (the INT4 saturating pack through the
    subnormal grid, the INT8 saturating pack), BDR steps toward the update
    on both sides, and overflowing updates: codes, scales and readouts
    against the oracle, in lock-step and free run."""
    S0, steps = _boundary_case(bits)
    T, dv, dk = S0.shape
    for pol in ("persistent", "dynamic"):
        for rnd in ("nearest", "bdr"):
            cfg = Config(T, dk, dv, bits, 32, 0, "scalar", pol, rnd)
            rep = P.lockstep(cfg, S0, steps, label=f"edges-int{bits}-{pol}-{rnd}")
            assert rep.code_flips == 0, rep
            gpu = P.GpuRun(cfg, S0)
            ora = O.init(P.oracle_cfg(cfg), S0)
            for t, (q, k, v, a, b) in enumerate(steps):
                o = gpu.step(q, k, v, a, b)
                o_ref = O.step(ora, q, k, v, a, b)
                P.compare_readout(o, o_ref, f"edges-int{bits}-{pol}-{rnd} free step {t}")
                c, s_, _ = gpu.state()
                rep = P.compare_state(cfg, c, s_, ora, None, f"edges-int{bits}-{pol}-{rnd} free step {t}")
                assert rep.code_flips == 0, rep


# Full-size workloads at the benchmark's launch configuration, on sampled
# tiles (tiles are independent, so a sampled tile is an exact check of that
# tile).
@pytest.mark.parametrize("wname", ["gdn", "mamba2", "gla", "stack24"])
def test_workload_full_size_sampled(wname):
    w = W.get(wname)
    rng = np.random.default_rng(99)
    tiles = np.sort(rng.choice(w.tiles, size=16, replace=False))
    tiles[-1] = w.tiles - 1          # always include the ragged last tile
    S0 = W.initial_state(w)
    steps = [W.slot(w, t) for t in range(4)]
    for arm in w.arms:
        cfg = Config(w.tiles, w.dk, w.dv, arm.bits, arm.group, w.delta, w.decay, arm.policy,
                     arm.rounding)
        rep = P.lockstep(cfg, S0, steps, tiles=tiles, label=f"{wname}-{arm.name}")
        assert rep.code_flips == 0, rep


@pytest.mark.parametrize("dk,dv,delta,decay,T", [(128, 128, 1, "scalar", 333), (128, 64, 0, "diagonal", 77),
                                                 (64, 64, 1, "diagonal", 5), (64, 48, 0, "scalar", 3),
                                                 (128, 16, 1, "scalar", 9)])
def test_fp32_state_step_matches_oracle_bit_for_bit(dk, dv, delta, decay, T):
    """The unquantized FP32 decode step (qstate_fp32_decode_step) against the
    oracle's FP32 recurrence: same fixed order, so states and readouts agree
    bit for bit over several steps."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    rng = np.random.default_rng(dk * 1000 + dv + T)
    cfg = Config(T, dk, dv, 8, 32, delta, decay)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    S_gpu = torch.from_numpy(S0.copy()).cuda()
    S_ref = S0.copy()
    ocfg = P.oracle_cfg(cfg)
    for t, (q, k, v, a, b) in enumerate(P.random_steps(rng, T, dk, dv, decay, 6)):
        o = torch.empty((T, dv), dtype=torch.float32, device="cuda")
        dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
        Q.fp32_decode_step(cfg, S_gpu, dev(q), dev(k), dev(v), dev(a), dev(b), o if t % 2 == 0 else None)
        o_ref = O.fp32_step(ocfg, S_ref, q, k, v, a, b)
        assert np.array_equal(S_gpu.cpu().numpy(), S_ref), f"state differs at step {t}"
        if t % 2 == 0:
            assert np.array_equal(o.cpu().numpy(), o_ref), f"readout differs at step {t}"


@pytest.mark.parametrize("bits,dk,dv,group,T", [(4, 128, 128, 32, 37), (8, 128, 64, 64, 300),
                                                (4, 64, 48, 64, 9), (8, 64, 16, 32, 5)])
def test_state_norms(bits, dk, dv, group, T):
    """qstate_state_sq_norms / qstate_fp32_sq_norms against the oracle's
    FP64 sums (same terms, summation order differs: relative 1e-12)."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    rng = np.random.default_rng(bits * 7 + dk + dv + T)
    cfg = Config(T, dk, dv, bits, group, 1, "scalar", "dynamic")
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    gpu = P.GpuRun(cfg, S0)
    ora = O.init(P.oracle_cfg(cfg), S0)
    for q, k, v, a, b in P.random_steps(rng, T, dk, dv, "scalar", 3):
        gpu.step(q, k, v, a, b)
        O.step(ora, q, k, v, a, b)
    c, s, _ = gpu.state()
    P.compare_state(cfg, c, s, ora, None, "before norms")
    out = torch.empty(T, dtype=torch.float64, device="cuda")
    Q.state_sq_norms(cfg, gpu.st.codes, gpu.st.scales, out)
    assert np.allclose(out.cpu().numpy(), O.sq_norms(ora), rtol=1e-12, atol=0.0)
    S = torch.from_numpy(S0).cuda()
    Q.fp32_sq_norms(cfg, S, out)
    assert np.allclose(out.cpu().numpy(), O.fp32_sq_norms(P.oracle_cfg(cfg), S0), rtol=1e-12, atol=0.0)


@pytest.mark.parametrize("bits,dk,policy,rounding", [(4, 128, "dynamic", "bdr"), (8, 64, "yoked", "nearest")])
def test_maximum_dv(bits, dk, policy, rounding):
    """The largest supported value dimension (Dv = 4096) on a few tiles."""
    rng = np.random.default_rng(bits + dk)
    T, dv = 3, 4096
    cfg = Config(T, dk, dv, bits, 32, 1, "scalar", policy, rounding)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    steps = P.random_steps(rng, T, dk, dv, "scalar", 2)
    rep = P.lockstep(cfg, S0, steps, label=f"dv4096-int{bits}-{policy}")
    assert rep.code_flips == 0


def test_many_tiles_sampled():
    """300,000 tiles (the row-block sequence far past one grid's worth of
    warps, ragged against it), checked on sampled tiles including the last."""
    rng = np.random.default_rng(17)
    T, dk, dv = 300_000, 64, 16
    cfg = Config(T, dk, dv, 4, 32, 1, "diagonal", "persistent", "bdr")
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    steps = P.random_steps(rng, T, dk, dv, "diagonal", 2)
    tiles = np.sort(rng.choice(T, size=24, replace=False))
    tiles[-1] = T - 1
    rep = P.lockstep(cfg, S0, steps, tiles=tiles, label="300k tiles")
    assert rep.code_flips == 0


@pytest.mark.parametrize("policy,bits,dv", [("dynamic", 4, 128), ("yoked", 4, 64), ("persistent", 8, 96)])
def test_back_to_back_steps_on_one_state(policy, bits, dv):
    """Steps on the same state launched one right after the other, with every
    input already on the device and nothing else in the stream between them:
    each launch may be scheduled while the previous one finishes
    (programmatic dependent launch) and must still read the state that
    launch wrote.  Free run against the oracle, every step's readout and the
    final state."""
    import torch
    from ssm_decode_step_b200 import QState
    rng = np.random.default_rng(23 + dv)
    T, dk, n = 300, 128, 24
    cfg = Config(T, dk, dv, bits, 32, 1, "scalar", policy, "nearest")
    S0 = (rng.standard_normal((T, dv, dk)) / np.sqrt(dk)).astype(np.float32)
    steps = P.random_steps(rng, T, dk, dv, "scalar", n)
    dev = torch.device("cuda")
    stack = [torch.from_numpy(np.ascontiguousarray(np.stack([s[i] for s in steps]))).to(dev)
             for i in range(5)]
    st = QState(cfg, dev).init(torch.from_numpy(S0).to(dev))
    o = torch.empty((n, T, dv), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    for t in range(n):
        st.step(stack[0][t], stack[1][t], stack[2][t], stack[3][t], stack[4][t], o[t])
    torch.cuda.synchronize()
    ora = O.init(P.oracle_cfg(cfg), S0)
    o_gpu = o.cpu().numpy()
    for t, (q, k, v, a, b) in enumerate(steps):
        o_ref = O.step(ora, q, k, v, a, b)
        P.compare_readout(o_gpu[t], o_ref, f"back-to-back {policy} step {t}")
    rep = P.compare_state(cfg, st.codes.cpu().numpy(), st.scales.cpu().numpy(), ora, None,
                          f"back-to-back {policy} final state")
    assert rep.code_flips == 0
    if st.shadow is not None:
        assert np.array_equal(st.shadow.cpu().numpy(), ora.shadow)
