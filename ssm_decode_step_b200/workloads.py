"""Seeded synthetic workloads for the quantized-state decode step.

This module only draws random inputs with the shapes and value
distributions of the five workloads below.  It holds none of the method's
arithmetic (no recurrence, no quantization): the CUDA path and the CPU
oracle both take their inputs from here and nothing else is shared.

Shapes and distributions follow the workloads named for this step:
gated delta-rule (Gated DeltaNet-shaped), Mamba-2-shaped scalar-decay
linear write, GLA-shaped diagonal decay, and a 24-layer long-horizon stack.
The pages evaluate on trained models and natural text; these synthetic
draws stand in for both (no dataset item is reproduced).

Randomness layout (fixed, so that every consumer sees the same bytes):
* the initial state S0 of workload seed s comes from default_rng([s, 1]);
* the inputs of pool slot t come from default_rng([s, 2, t]), drawn in the
  order q, k, v, alpha, beta, so a slot does not depend on the pool size.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Callable, Dict, List, Optional, Tuple

import numpy as np


@dataclass(frozen=True)
class Arm:
    """One storage / scale / rounding choice for a workload."""
    bits: int
    group: int
    policy: str          # "dynamic" | "persistent" | "yoked"
    rounding: str = "nearest"   # "nearest" | "bdr"

    @property
    def name(self) -> str:
        r = "+bdr" if self.rounding == "bdr" else ""
        return f"int{self.bits}-g{self.group}-{self.policy}{r}"


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    layers: int
    batch: int
    heads: int
    dk: int
    dv: int
    steps: int
    delta: int
    decay: str                      # "scalar" | "diagonal"
    arms: Tuple[Arm, ...]
    seed: int
    layer_seeds: Optional[Tuple[int, ...]] = None   # one seed per layer (stack)
    s0_std: float = 0.1
    draw: str = "gdn"               # which input law to use (see _draw_slot)
    readout: bool = True
    tile_ids: Optional[Tuple[int, ...]] = None   # a shard: these tiles of the whole draw

    @property
    def all_tiles(self) -> int:
        return self.layers * self.batch * self.heads

    @property
    def tiles(self) -> int:
        return self.all_tiles if self.tile_ids is None else len(self.tile_ids)

    @property
    def tiles_per_layer(self) -> int:
        return self.batch * self.heads


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _softplus(x):
    return np.log1p(np.exp(-np.abs(x))) + np.maximum(x, 0.0)


def _unit_rows(g):
    n = np.sqrt(np.sum(g * g, axis=-1, keepdims=True))
    return g / np.maximum(n, 1e-30)


def _draw_slot(law: str, rng: np.random.Generator, T: int, dk: int, dv: int,
               decay: str):
    """q, k, v, alpha, beta for one decode step of T tiles."""
    if law == "tiny":           # tiny gated delta rule
        q = rng.standard_normal((T, dk))
        k = _unit_rows(rng.standard_normal((T, dk)))
        v = rng.standard_normal((T, dv))
        alpha = rng.uniform(0.9, 1.0, size=(T,))
        beta = rng.uniform(0.0, 1.0, size=(T,))
    elif law == "gdn":          # Gated DeltaNet-shaped
        q = rng.standard_normal((T, dk))
        k = _unit_rows(rng.standard_normal((T, dk)))
        v = rng.standard_normal((T, dv))
        alpha = _sigmoid(rng.normal(3.0, 1.0, size=(T,)))
        beta = _sigmoid(rng.standard_normal((T,)))
    elif law == "mamba2":       # Mamba-2-shaped scalar decay, linear write
        q = rng.standard_normal((T, dk))
        k = rng.standard_normal((T, dk))
        v = rng.standard_normal((T, dv))
        alpha = np.exp(-_softplus(rng.standard_normal((T,))) * 0.1)
        beta = _softplus(rng.standard_normal((T,)))
    elif law == "gla":          # GLA-shaped diagonal decay, beta = 1
        s = 1.0 / np.sqrt(128.0)
        q = rng.standard_normal((T, dk)) * s
        k = rng.standard_normal((T, dk)) * s
        v = rng.standard_normal((T, dv)) * s
        alpha = rng.uniform(0.8, 1.0, size=(T, dk))
        beta = np.ones((T,))
    elif law == "recall":       # distractor steps of the recall-over-horizon measurement
        q = rng.standard_normal((T, dk))
        k = _unit_rows(rng.standard_normal((T, dk)))
        v = rng.standard_normal((T, dv))
        alpha = rng.uniform(0.999, 1.0, size=(T,))
        beta = rng.uniform(0.0, 0.1, size=(T,))
    else:
        raise ValueError(law)
    if decay == "diagonal" and alpha.ndim == 1:
        alpha = np.repeat(alpha[:, None], dk, axis=1)
    if decay == "scalar" and alpha.ndim == 2:
        raise ValueError("scalar decay with a per-channel draw")
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)
    return f(q), f(k), f(v), f(alpha), f(beta)


WORKLOADS: Dict[str, Workload] = {}


def _reg(w: Workload):
    WORKLOADS[w.name] = w
    return w


TINY = _reg(Workload(
    name="tiny-gdn", description="tiny gated delta rule: B1 H4 Dk=Dv=64, 256 steps, "
    "INT8 G64 persistent, scalar alpha~U(0.9,1), beta~U(0,1), k unit-norm; seed 0",
    layers=1, batch=1, heads=4, dk=64, dv=64, steps=256, delta=1, decay="scalar",
    arms=(Arm(8, 64, "persistent"),), seed=0, s0_std=1.0 / 8.0, draw="tiny"))

GDN = _reg(Workload(
    name="gdn", description="Gated DeltaNet-shaped: B64 H16 Dk=Dv=128, 2048 steps, "
    "INT4 G32, dynamic / persistent / yoked; alpha=sigmoid(N(3,1)), "
    "beta=sigmoid(N(0,1)), k unit-norm; seed 1",
    layers=1, batch=64, heads=16, dk=128, dv=128, steps=2048, delta=1, decay="scalar",
    arms=(Arm(4, 32, "dynamic"), Arm(4, 32, "persistent"), Arm(4, 32, "yoked")),
    seed=1, s0_std=1.0 / np.sqrt(128.0), draw="gdn"))

MAMBA2 = _reg(Workload(
    name="mamba2", description="Mamba-2-shaped scalar-decay linear write: B256 H64 "
    "Dk=128 Dv=64, 1024 steps, INT8 G64 persistent; alpha=exp(-softplus(N(0,1))*0.1), "
    "beta=softplus(N(0,1)); seed 2",
    layers=1, batch=256, heads=64, dk=128, dv=64, steps=1024, delta=0, decay="scalar",
    arms=(Arm(8, 64, "persistent"),), seed=2, s0_std=2.5, draw="mamba2"))

GLA = _reg(Workload(
    name="gla", description="GLA-shaped diagonal decay: B128 H32 Dk=Dv=128, 4096 steps, "
    "INT4 G32 + BDR (persistent; dynamic as second arm); alpha_j~U(0.8,1), beta=1, "
    "q,k,v~N(0,1)/sqrt(128); seed 3",
    layers=1, batch=128, heads=32, dk=128, dv=128, steps=4096, delta=0, decay="diagonal",
    arms=(Arm(4, 32, "persistent", "bdr"), Arm(4, 32, "dynamic", "bdr")),
    seed=3, s0_std=0.02, draw="gla"))

STACK = _reg(Workload(
    name="stack24", description="24-layer x 16-head gated delta-rule stack: B32 "
    "Dk=Dv=128, 32768 steps, INT4 G32 persistent + BDR vs INT8 G32 dynamic, readout "
    "every step; GDN inputs with seed 4000+layer",
    layers=24, batch=32, heads=16, dk=128, dv=128, steps=32768, delta=1, decay="scalar",
    arms=(Arm(4, 32, "persistent", "bdr"), Arm(8, 32, "dynamic")),
    seed=4, layer_seeds=tuple(4000 + l for l in range(24)),
    s0_std=1.0 / np.sqrt(128.0), draw="gdn"))

RECALL = _reg(Workload(
    name="recall", description="recall over a decode horizon, gated delta rule: B16 H16 "
    "Dk=Dv=128, a probe association (k*, v*) planted in S0, then distractor steps with k "
    "unit-norm, v~N(0,1), alpha~U(0.999,1), beta~U(0,0.1); INT8/INT4 dynamic, INT4 persistent, "
    "yoked and BDR arms against the FP32 state; seed 5",
    layers=1, batch=16, heads=16, dk=128, dv=128, steps=32768, delta=1, decay="scalar",
    arms=(Arm(8, 32, "dynamic"), Arm(4, 32, "dynamic"), Arm(4, 32, "persistent"),
          Arm(4, 32, "yoked"), Arm(4, 32, "persistent", "bdr"), Arm(4, 32, "dynamic", "bdr")),
    seed=5, s0_std=1.0 / np.sqrt(128.0), draw="recall"))

# Index in the order the workloads are listed for this step (the recall
# measurement above is not one of them).

ORDER: List[str] = ["tiny-gdn", "gdn", "mamba2", "gla", "stack24"]


def get(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[ORDER[name_or_index]]
    return WORKLOADS[name_or_index]


def shard(w: Workload, rank: int, world: int) -> Workload:
    """Rank `rank`'s part of the workload on `world` GPUs: the contiguous
    tile range [rank T / world, (rank + 1) T / world) of the whole draw.
    Tiles are independent recurrences, so the shards need no exchange; a
    shard draws exactly the inputs and initial state that the whole
    workload gives those tiles (per-layer seeds included)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    T = w.all_tiles
    ids = tuple(range(rank * T // world, (rank + 1) * T // world))
    return replace(w, name=f"{w.name}[{rank}/{world}]", tile_ids=ids)


def _select(w: Workload, tiles: Optional[np.ndarray]) -> Optional[np.ndarray]:
    """Indices into the whole draw: the shard's tiles, then `tiles` within them."""
    if w.tile_ids is None:
        return tiles
    ids = np.asarray(w.tile_ids)
    return ids if tiles is None else ids[np.asarray(tiles)]


def _seeds(w: Workload) -> List[Tuple[int, int]]:
    """(seed, tiles) per layer block."""
    if w.layer_seeds is None:
        return [(w.seed, w.tiles)]
    return [(s, w.tiles_per_layer) for s in w.layer_seeds]


def initial_state(w: Workload, tiles: Optional[np.ndarray] = None) -> np.ndarray:
    """S0 [T][dv][dk] float32, iid N(0, s0_std^2) per element.  If tiles is
    given, only those tile indices are returned (same values as in the full
    draw)."""
    blocks = []
    for seed, T in _seeds(w):
        rng = np.random.default_rng([seed, 1])
        blocks.append(rng.standard_normal((T, w.dv, w.dk)) * w.s0_std)
    S0 = np.ascontiguousarray(np.concatenate(blocks, axis=0), dtype=np.float32)
    sel = _select(w, tiles)
    return S0 if sel is None else np.ascontiguousarray(S0[sel])


def slot(w: Workload, t: int, tiles: Optional[np.ndarray] = None):
    """(q, k, v, alpha, beta) of pool slot t for every tile (or the listed
    tiles)."""
    parts = [[] for _ in range(5)]
    for seed, T in _seeds(w):
        rng = np.random.default_rng([seed, 2, t])
        for p, a in zip(parts, _draw_slot(w.draw, rng, T, w.dk, w.dv, w.decay)):
            p.append(a)
    out = tuple(np.ascontiguousarray(np.concatenate(p, axis=0)) for p in parts)
    sel = _select(w, tiles)
    if sel is not None:
        out = tuple(np.ascontiguousarray(a[sel]) for a in out)
    return out


def pool(w: Workload, n_slots: int, tiles: Optional[np.ndarray] = None):
    """Stacked inputs of slots 0..n_slots-1: arrays with a leading slot axis."""
    slots = [slot(w, t, tiles) for t in range(n_slots)]
    return tuple(np.ascontiguousarray(np.stack([s[i] for s in slots])) for i in range(5))


def scaled_down(w: Workload, tiles_per_layer: int, layers: Optional[int] = None,
                steps: Optional[int] = None) -> Workload:
    """Same laws and arms with fewer tiles (for tests that must finish fast)."""
    L = w.layers if layers is None else layers
    seeds = None if w.layer_seeds is None else w.layer_seeds[:L]
    return replace(w, name=w.name + "-small", layers=L, batch=1, heads=tiles_per_layer,
                   layer_seeds=seeds, steps=w.steps if steps is None else steps)


def probe(w: Workload, tiles: Optional[np.ndarray] = None):
    """(k*, v*) of the recall measurement: per tile a unit-norm key and a
    N(0, 1) value, from default_rng([seed, 3]) (float32 [T][dk], [T][dv])."""
    rng = np.random.default_rng([w.seed, 3])
    k = _unit_rows(rng.standard_normal((w.all_tiles, w.dk)))
    v = rng.standard_normal((w.all_tiles, w.dv))
    sel = _select(w, tiles)
    f = lambda a: np.ascontiguousarray(a if sel is None else a[sel], dtype=np.float32)
    return f(k), f(v)
