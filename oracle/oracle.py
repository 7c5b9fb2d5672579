"""NumPy front end of the CPU oracle (test infrastructure only).

Only tests/, the smoke check and the benchmark's CPU-baseline leg load this
module.  It marshals NumPy arrays into oracle/liboracle.so; every number is
computed by the C code in qstate_oracle.c, whose header states the
element-level definition it follows (LinQuant eq. (1); the scale policies of
"When Dynamic Scaling Fails"; Bounded Directional Rounding of "Preserving
Updates in Low-Bit Recurrent State Quantization").
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

DECAY = {"scalar": 0, "diagonal": 1}
POLICY = {"dynamic": 0, "persistent": 1, "yoked": 2}
ROUNDING = {"nearest": 0, "bdr": 1}

FAULTS = {
    "none": 0, "drop_delta": 1, "write_sign": 2, "decay_skipped": 3,
    "read_k_for_q": 4, "group_index": 5, "bdr_reference": 6,
    "round_trunc": 7, "beta_on_v_only": 8, "diag_decay_row": 9,
    "persist_update": 10, "yoked_from_x": 11, "lrb_sign_last": 12,
}


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "tiles", "dk", "dv", "qmax", "group", "delta", "decay", "policy",
        "rounding")]


@dataclass(frozen=True)
class OracleConfig:
    tiles: int
    dk: int
    dv: int
    bits: int            # 4 or 8 for the packed layout; any >= 2 unpacked
    group: int
    delta: int
    decay: str = "scalar"
    policy: str = "persistent"
    rounding: str = "nearest"

    @property
    def qmax(self) -> int:
        return (1 << (self.bits - 1)) - 1

    @property
    def groups(self) -> int:
        return self.dk // self.group

    def c(self) -> _Cfg:
        return _Cfg(self.tiles, self.dk, self.dv, self.qmax, self.group,
                    self.delta, DECAY[self.decay], POLICY[self.policy],
                    ROUNDING[self.rounding])


_libs = {}
_active = None      # the mutation build while a mistake is planted, else None
_planted = "none"


def _load(path: str, mutations: bool) -> ctypes.CDLL:
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    C = ctypes.POINTER(_Cfg)
    for name, args in {
        "qo_check": [C],
        "qo_num_threads": [],
        "qo_pack": [ctypes.c_int, ctypes.c_int64, P, P],
        "qo_unpack": [ctypes.c_int, ctypes.c_int64, P, P],
        "qo_init": [C, P, P, P, P],
        "qo_step": [C, P, P, P, P, P, P, P, P, P, P],
        "qo_readout": [C, P, P, P, P],
        "qo_fp32_step": [C, P, P, P, P, P, P, P],
        "qo_sq_norms": [C, P, P, P],
        "qo_lrb_step": [C, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "qo_fp32_sq_norms": [C, P, P],
    }.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    L.qo_dot.argtypes = [P, P, ctypes.c_int]
    L.qo_dot.restype = ctypes.c_float
    if mutations:
        L.qo_set_fault.argtypes = [ctypes.c_int]
        L.qo_set_fault.restype = None
    return L


def lib() -> ctypes.CDLL:
    """The oracle library every call goes to: the oracle proper, or its
    mutation build while planted() is active."""
    if _active is not None:
        return _active
    if "plain" not in _libs:
        _libs["plain"] = _load(_build.build(), False)
    return _libs["plain"]


class planted:
    """Context manager that routes every oracle call to the mutation build
    with one mistake planted, and back to the oracle proper on exit (also on
    an exception)."""

    def __init__(self, fault: str):
        self.fault = fault

    def __enter__(self):
        global _active, _planted
        if "mut" not in _libs:
            _build.build()
            _libs["mut"] = _load(_build.MUT_LIB, True)
        _libs["mut"].qo_set_fault(FAULTS[self.fault])
        _active, _planted = _libs["mut"], self.fault
        return self

    def __exit__(self, *exc):
        global _active, _planted
        _libs["mut"].qo_set_fault(0)
        _active, _planted = None, "none"
        return False


def planted_fault() -> str:
    """The mistake planted right now ("none" outside planted())."""
    return _planted


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float32)


def _ok(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments")


def num_threads() -> int:
    return lib().qo_num_threads()


def dot(a, b) -> np.float32:
    a, b = _f32(a), _f32(b)
    assert a.shape == b.shape and a.ndim == 1
    return np.float32(lib().qo_dot(_p(a), _p(b), a.size))


def pack(bits: int, codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    n = codes.size
    out = np.empty(n if bits == 8 else n // 2, dtype=np.uint8)
    _ok(lib().qo_pack(bits, n, _p(codes), _p(out)), "pack")
    return out.reshape(codes.shape[:-1] + (-1,))


def unpack(bits: int, packed: np.ndarray, n_last: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n_rows = packed.size // (n_last if bits == 8 else n_last // 2)
    out = np.empty(n_rows * n_last, dtype=np.int32)
    _ok(lib().qo_unpack(bits, out.size, _p(packed), _p(out)), "unpack")
    return out.reshape(packed.shape[:-1] + (n_last,))


class State:
    """Quantized state held by the oracle: unpacked int32 codes, FP32 scales
    and (yoked only) the FP32 shadow."""

    def __init__(self, cfg: OracleConfig, codes, scales, shadow=None):
        self.cfg = cfg
        self.codes = np.ascontiguousarray(codes, dtype=np.int32)
        self.scales = np.ascontiguousarray(scales, dtype=np.float32)
        self.shadow = None if shadow is None else np.ascontiguousarray(shadow, dtype=np.float32)

    def copy(self) -> "State":
        return State(self.cfg, self.codes.copy(), self.scales.copy(),
                     None if self.shadow is None else self.shadow.copy())

    def packed(self) -> np.ndarray:
        return pack(self.cfg.bits, self.codes)

    def dequantized(self) -> np.ndarray:
        c = self.cfg
        s = np.repeat(self.scales, c.group, axis=-1)
        return (self.codes.astype(np.float32) * s).astype(np.float32)


def init(cfg: OracleConfig, S0) -> State:
    S0 = _f32(S0)
    assert S0.shape == (cfg.tiles, cfg.dv, cfg.dk)
    codes = np.empty(S0.shape, dtype=np.int32)
    scales = np.empty((cfg.tiles, cfg.dv, cfg.groups), dtype=np.float32)
    shadow = np.empty_like(S0) if cfg.policy == "yoked" else None
    cc = cfg.c()
    _ok(lib().qo_init(ctypes.byref(cc), _p(S0), _p(codes), _p(scales), _p(shadow)), "init")
    return State(cfg, codes, scales, shadow)


def step(st: State, q, k, v, alpha, beta, want_o=True, want_pre=False):
    """One decode step in place on st; returns o (or None) and, if asked, the
    exact pre-rounding values x * inv."""
    cfg = st.cfg
    q, k, v, alpha, beta = map(_f32, (q, k, v, alpha, beta))
    o = np.empty((cfg.tiles, cfg.dv), dtype=np.float32) if want_o else None
    pre = np.empty((cfg.tiles, cfg.dv, cfg.dk), dtype=np.float64) if want_pre else None
    cc = cfg.c()
    _ok(lib().qo_step(ctypes.byref(cc), _p(st.codes), _p(st.scales), _p(st.shadow),
                      _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(o), _p(pre)), "step")
    return (o, pre) if want_pre else o


def readout(st: State, q) -> np.ndarray:
    cfg = st.cfg
    q = _f32(q)
    o = np.empty((cfg.tiles, cfg.dv), dtype=np.float32)
    cc = cfg.c()
    _ok(lib().qo_readout(ctypes.byref(cc), _p(st.codes), _p(st.scales), _p(q), _p(o)), "readout")
    return o


def fp32_step(cfg: OracleConfig, S, q, k, v, alpha, beta, want_o=True):
    """Unquantized FP32 recurrence, in place on S ([tiles][dv][dk] float32)."""
    assert S.dtype == np.float32 and S.flags.c_contiguous
    q, k, v, alpha, beta = map(_f32, (q, k, v, alpha, beta))
    o = np.empty((cfg.tiles, cfg.dv), dtype=np.float32) if want_o else None
    cc = cfg.c()
    _ok(lib().qo_fp32_step(ctypes.byref(cc), _p(S), _p(q), _p(k), _p(v), _p(alpha),
                           _p(beta), _p(o)), "fp32_step")
    return o


def sq_norms(st: State) -> np.ndarray:
    """Squared Frobenius norm of each tile of the dequantized stored state (float64 [T])."""
    cfg = st.cfg
    out = np.empty(cfg.tiles, dtype=np.float64)
    cc = cfg.c()
    _ok(lib().qo_sq_norms(ctypes.byref(cc), _p(st.codes), _p(st.scales), _p(out)), "sq_norms")
    return out


def fp32_sq_norms(cfg: OracleConfig, S) -> np.ndarray:
    """Squared Frobenius norm of each tile of an FP32 state (float64 [T])."""
    S = _f32(S)
    out = np.empty(cfg.tiles, dtype=np.float64)
    cc = cfg.c()
    _ok(lib().qo_fp32_sq_norms(ctypes.byref(cc), _p(S), _p(out)), "fp32_sq_norms")
    return out


class LrbBuffers:
    """Low-Rank Bypass buffers of the oracle (see qo_lrb_step): accumulated
    column decay A, decayed keys K and write coefficients U of the current
    period, with the slot (position in the period) of the next step."""

    def __init__(self, cfg: OracleConfig, rank: int):
        self.rank = rank
        self.slot = 0
        self.A = np.ones((cfg.tiles, cfg.dk), np.float32)
        self.K = np.zeros((cfg.tiles, rank, cfg.dk), np.float32)
        self.U = np.zeros((cfg.tiles, cfg.dv, rank), np.float32)


def lrb_step(st: State, buf: LrbBuffers, q, k, v, alpha, beta, want_o=True, want_pre=False):
    """One Low-Rank Bypass step in place on (st, buf); returns o (and, if
    asked, the exact pre-rounding values at a merge step, else None)."""
    cfg = st.cfg
    q, k, v, alpha, beta = map(_f32, (q, k, v, alpha, beta))
    o = np.empty((cfg.tiles, cfg.dv), dtype=np.float32) if want_o else None
    merge = buf.slot == buf.rank - 1
    pre = np.full((cfg.tiles, cfg.dv, cfg.dk), np.nan) if (want_pre and merge) else None
    A_out = None if merge else np.empty_like(buf.A)
    K_out = None if merge else np.empty_like(buf.K)
    cc = cfg.c()
    _ok(lib().qo_lrb_step(ctypes.byref(cc), buf.rank, buf.slot, _p(st.codes), _p(st.scales),
                          _p(st.shadow), _p(buf.A), _p(A_out), _p(buf.K), _p(K_out), _p(buf.U),
                          _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(o), _p(pre)), "lrb_step")
    if merge:
        buf.slot = 0
        buf.A[:] = 1.0
        buf.K[:] = 0.0
        buf.U[:] = 0.0
    else:
        buf.A, buf.K = A_out, K_out
        buf.slot += 1
    return (o, pre) if want_pre else o
