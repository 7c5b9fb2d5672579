"""Helpers shared by the GPU parity tests: run the CUDA path (through the
C ABI binding) and the CPU oracle on the same seeded inputs and compare.

Tolerances (fixed for this step): packed codes bit-exact, except that at
most 1e-6 of the elements may differ by one code level, and only where the
oracle's pre-rounding value lies within 1e-6 (relative) of a half-step
boundary; scales within 1e-6 relative; readouts within 1e-4 * ||o_t||_inf
of the tile.  The FP32 shadow of the yoked policy must match bit for bit
(same operation order, element-wise arithmetic).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from oracle import oracle as O

CODE_FLIP_FRACTION = 1e-6
HALF_STEP_REL = 1e-6
SCALE_REL = 1e-6
READOUT_REL = 1e-4


def oracle_cfg(cfg, tiles: Optional[int] = None) -> O.OracleConfig:
    return O.OracleConfig(cfg.num_tiles if tiles is None else tiles, cfg.dk, cfg.dv, cfg.bits,
                          cfg.group, cfg.delta, cfg.decay, cfg.policy, cfg.rounding)


@dataclass
class Report:
    code_flips: int = 0
    elements: int = 0
    worst_scale_rel: float = 0.0
    worst_o_rel: float = 0.0

    def merge(self, other: "Report"):
        self.code_flips += other.code_flips
        self.elements += other.elements
        self.worst_scale_rel = max(self.worst_scale_rel, other.worst_scale_rel)
        self.worst_o_rel = max(self.worst_o_rel, other.worst_o_rel)


def compare_state(cfg, gpu_codes_packed: np.ndarray, gpu_scales: np.ndarray,
                  ora: O.State, prequant: Optional[np.ndarray], what: str) -> Report:
    rep = Report()
    g = O.unpack(cfg.bits, gpu_codes_packed.reshape(-1, gpu_codes_packed.shape[-1]), cfg.dk)
    g = g.reshape(ora.codes.shape)
    diff = g != ora.codes
    rep.elements = diff.size
    rep.code_flips = int(diff.sum())
    if rep.code_flips:
        assert prequant is not None, f"{what}: {rep.code_flips} codes differ"
        d = np.abs(g[diff].astype(np.int64) - ora.codes[diff])
        assert np.all(d == 1), f"{what}: codes differ by more than one level"
        pre = prequant[diff]
        dist = np.abs(np.abs(pre - np.floor(pre)) - 0.5)
        assert np.all(dist <= HALF_STEP_REL * np.abs(pre)), \
            f"{what}: {rep.code_flips} code flips away from a half-step boundary"
        assert rep.code_flips <= CODE_FLIP_FRACTION * rep.elements, \
            f"{what}: {rep.code_flips} code flips of {rep.elements}"
    # scales: non-finite ones (a group maximum that overflowed) by pattern,
    # NaN where the oracle has NaN and infinities of the same sign; the
    # relative bound on the finite ones
    s_ref = ora.scales.astype(np.float64)
    s_gpu = np.asarray(gpu_scales).astype(np.float64)
    assert np.array_equal(np.isnan(s_gpu), np.isnan(s_ref)), f"{what}: NaN scales differ"
    assert np.array_equal(np.isposinf(s_gpu), np.isposinf(s_ref)) and \
        np.array_equal(np.isneginf(s_gpu), np.isneginf(s_ref)), f"{what}: infinite scales differ"
    fin = np.isfinite(s_ref)
    rel = np.abs(s_gpu[fin] - s_ref[fin]) / np.maximum(np.abs(s_ref[fin]), 1e-38)
    rel[(s_ref[fin] == 0) & (s_gpu[fin] == 0)] = 0.0
    rep.worst_scale_rel = float(rel.max()) if rel.size else 0.0
    assert rep.worst_scale_rel <= SCALE_REL, f"{what}: scale rel err {rep.worst_scale_rel}"
    return rep


def compare_readout(gpu_o: np.ndarray, ora_o: np.ndarray, what: str) -> float:
    """Readouts within READOUT_REL * ||o||_inf of the tile's oracle readout.
    Non-finite values are compared by pattern first: NaN where the oracle
    has NaN and nowhere else, and infinities of the same sign at the same
    places.  The bound then applies to every tile whose oracle readout is
    finite throughout (a tile with an infinite readout has no finite
    ||o||_inf to bound against)."""
    g = gpu_o.astype(np.float64)
    ref = ora_o.astype(np.float64)
    assert g.shape == ref.shape, f"{what}: readout shapes {g.shape} vs {ref.shape}"
    assert np.array_equal(np.isnan(g), np.isnan(ref)), \
        f"{what}: NaN readouts at {int(np.isnan(g).sum())} places, oracle {int(np.isnan(ref).sum())}"
    assert np.array_equal(np.isposinf(g), np.isposinf(ref)) and \
        np.array_equal(np.isneginf(g), np.isneginf(ref)), f"{what}: infinite readouts differ"
    finite_row = np.all(np.isfinite(ref), axis=-1, keepdims=True)
    inf = np.where(finite_row, np.abs(np.where(np.isfinite(ref), ref, 0.0)).max(axis=-1, keepdims=True), 0.0)
    with np.errstate(invalid="ignore"):
        err = np.where(np.isfinite(ref), np.abs(g - ref), 0.0)
    bad = (err > READOUT_REL * inf) & finite_row
    assert not np.any(bad & (inf > 0)), f"{what}: readout error {err[bad].max()} vs {inf.max()}"
    assert not np.any((inf == 0) & (err > 0) & finite_row), f"{what}: nonzero readout where the oracle is 0"
    with np.errstate(invalid="ignore", divide="ignore"):
        r = np.where((inf > 0) & finite_row, err / np.where(inf > 0, inf, 1.0), 0.0)
    return float(r.max()) if r.size else 0.0


class GpuRun:
    """A quantized state on the GPU driven through the C ABI binding."""

    def __init__(self, cfg, S0: np.ndarray, device="cuda"):
        import torch
        from ssm_decode_step_b200 import QState
        self.torch = torch
        self.cfg = cfg
        self.dev = torch.device(device)
        self.st = QState(cfg, self.dev)
        self.st.init(torch.from_numpy(np.ascontiguousarray(S0, dtype=np.float32)).to(self.dev))

    def t(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a)).to(self.dev)

    def step(self, q, k, v, alpha, beta, want_o=True):
        o = self.torch.empty((self.cfg.num_tiles, self.cfg.dv), dtype=self.torch.float32,
                             device=self.dev) if want_o else None
        self.st.step(self.t(q) if q is not None else None, self.t(k), self.t(v), self.t(alpha),
                     self.t(beta), o)
        return None if o is None else o.cpu().numpy()

    def state(self, tiles=None):
        idx = None if tiles is None else self.torch.as_tensor(np.asarray(tiles), device=self.dev)
        c = self.st.codes if idx is None else self.st.codes.index_select(0, idx)
        s = self.st.scales if idx is None else self.st.scales.index_select(0, idx)
        sh = None
        if self.st.shadow is not None:
            sh = (self.st.shadow if idx is None else self.st.shadow.index_select(0, idx)).cpu().numpy()
        return c.cpu().numpy(), s.cpu().numpy(), sh

    def set_state(self, codes_packed, scales, shadow=None):
        self.st.codes.copy_(self.t(codes_packed))
        self.st.scales.copy_(self.t(scales))
        if shadow is not None:
            self.st.shadow.copy_(self.t(shadow))


def lockstep(cfg, S0, steps, tiles=None, want_o=True, label="") -> Report:
    """Drive GPU and oracle over the given step inputs; before each step the
    oracle starts from the GPU's state (so one flip cannot cascade), and the
    GPU result of the step is compared with the oracle's.  `tiles` selects
    which tiles the oracle evaluates (all when None)."""
    gpu = GpuRun(cfg, S0)
    sel = np.arange(cfg.num_tiles) if tiles is None else np.asarray(tiles)
    ocfg = oracle_cfg(cfg, len(sel))
    ini = O.init(ocfg, np.ascontiguousarray(S0[sel]))
    c, s, sh = gpu.state(sel)
    rep = compare_state(cfg, c, s, ini, None, f"{label} init")
    if sh is not None:
        assert np.array_equal(sh, ini.shadow), f"{label} init shadow"
    for t, (q, k, v, a, b) in enumerate(steps):
        c, s, sh = gpu.state(sel)
        ora = O.State(ocfg, O.unpack(cfg.bits, c.reshape(-1, c.shape[-1]), cfg.dk).reshape(len(sel), cfg.dv, cfg.dk), s, sh)
        o_ref, pre = O.step(ora, q[sel], k[sel], v[sel], a[sel], b[sel], want_o=True, want_pre=True)
        o = gpu.step(q, k, v, a, b, want_o)
        c, s, sh = gpu.state(sel)
        rep.merge(compare_state(cfg, c, s, ora, pre, f"{label} step {t}"))
        if sh is not None:
            assert np.array_equal(sh, ora.shadow), f"{label} step {t}: shadow differs"
        if want_o:
            rep.worst_o_rel = max(rep.worst_o_rel, compare_readout(o[sel], o_ref, f"{label} step {t}"))
    return rep


def free_run(cfg, S0, steps, label="") -> Report:
    """GPU and oracle run independently over all steps; everything must agree
    at every step (exact codes expected with the shared operation order)."""
    gpu = GpuRun(cfg, S0)
    ora = O.init(oracle_cfg(cfg), S0)
    rep = Report()
    for t, (q, k, v, a, b) in enumerate(steps):
        o_ref = O.step(ora, q, k, v, a, b)
        o = gpu.step(q, k, v, a, b)
        c, s, sh = gpu.state()
        r = compare_state(cfg, c, s, ora, None, f"{label} step {t}")
        rep.merge(r)
        if sh is not None:
            assert np.array_equal(sh, ora.shadow), f"{label} step {t}: shadow differs"
        rep.worst_o_rel = max(rep.worst_o_rel, compare_readout(o, o_ref, f"{label} step {t}"))
    return rep


def random_steps(rng, T, dk, dv, decay, n, unit_k=True, scale=1.0):
    out = []
    for _ in range(n):
        q = rng.standard_normal((T, dk)).astype(np.float32)
        k = rng.standard_normal((T, dk))
        if unit_k:
            k = k / np.linalg.norm(k, axis=-1, keepdims=True)
        k = k.astype(np.float32)
        v = (rng.standard_normal((T, dv)) * scale).astype(np.float32)
        a = rng.uniform(0.8, 1.0, size=(T, dk) if decay == "diagonal" else (T,)).astype(np.float32)
        b = rng.uniform(0.05, 1.0, size=(T,)).astype(np.float32)
        out.append((q, k, v, a, b))
    return out
