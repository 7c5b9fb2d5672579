"""Python binding of the qstate C ABI (include/qstate.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libqstate.so.  Tensors are torch CUDA tensors (PyTorch supplies
device memory and streams); their data pointers and the current CUDA stream
are handed to the library.  There is no CPU fallback: if libqstate.so is
missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqstate.so")

DECAY = {"scalar": 0, "diagonal": 1}
POLICY = {"dynamic": 0, "persistent": 1, "yoked": 2}
ROUNDING = {"nearest": 0, "bdr": 1}

QS_OK, QS_ERR_INVALID_ARG, QS_ERR_UNSUPPORTED, QS_ERR_CUDA = 0, 1, 2, 3

# Every entry point that include/qstate.h declares.
EXPORTS = ("qstate_query_sizes", "qstate_init", "qstate_decode_step", "qstate_readout",
           "qstate_fp32_decode_step", "qstate_lrb_query_sizes", "qstate_lrb_decode_step",
           "qstate_prefill", "qstate_prefill_tf32", "qstate_prefill_tf32_timeouts",
           "qstate_prefill_tf32_wait_selfcheck",
           "qstate_pipeline_query_sizes", "qstate_pipeline_create", "qstate_pipeline_step",
           "qstate_pipeline_wait_stream", "qstate_pipeline_join", "qstate_pipeline_sync",
           "qstate_pipeline_destroy", "qstate_decode_step_host_static",
           "qstate_state_sq_norms", "qstate_fp32_sq_norms",
           "qstate_selfcheck", "qstate_status_string", "qstate_version")


class QStateError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class qs_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_tiles", "dk", "dv", "bits", "group", "delta", "decay", "policy", "rounding")]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libqstate.so (built by ssm_decode_step_b200/build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m ssm_decode_step_b200.build` "
                              "(or __graft_entry__.build()) first")
        L = ctypes.CDLL(LIB_PATH)
        P, C = ctypes.c_void_p, ctypes.POINTER(qs_config)
        sz = ctypes.POINTER(ctypes.c_size_t)
        L.qstate_query_sizes.argtypes = [C, sz, sz, sz]
        L.qstate_init.argtypes = [C, P, P, P, P, P]
        L.qstate_decode_step.argtypes = [C, P, P, P, P, P, P, P, P, P, P]
        L.qstate_readout.argtypes = [C, P, P, P, P, P]
        L.qstate_selfcheck.argtypes = [P, P]
        L.qstate_fp32_decode_step.argtypes = [C, P, P, P, P, P, P, P, P]
        L.qstate_lrb_query_sizes.argtypes = [C, ctypes.c_int, sz, sz, sz]
        L.qstate_lrb_decode_step.argtypes = [C, ctypes.c_int, ctypes.c_int] + [P] * 15
        L.qstate_prefill.argtypes = [C, ctypes.c_int] + [P] * 8
        L.qstate_prefill_tf32.argtypes = [C, ctypes.c_int] + [P] * 8
        L.qstate_prefill_tf32_timeouts.argtypes = [P]
        L.qstate_prefill_tf32_wait_selfcheck.argtypes = [ctypes.c_uint, P]
        L.qstate_pipeline_query_sizes.argtypes = [C, ctypes.c_int, sz, sz]
        L.qstate_pipeline_create.argtypes = [ctypes.c_int, C, ctypes.c_int, ctypes.POINTER(P)]
        L.qstate_pipeline_step.argtypes = [P, P, P, P, P, P, P]
        L.qstate_pipeline_wait_stream.argtypes = [P, P]
        L.qstate_pipeline_join.argtypes = [P, P]
        L.qstate_pipeline_sync.argtypes = [P]
        L.qstate_pipeline_destroy.argtypes = [P]
        L.qstate_decode_step_host_static.argtypes = [C, P, P, P, P, P, P]
        L.qstate_state_sq_norms.argtypes = [C, P, P, P, P]
        L.qstate_fp32_sq_norms.argtypes = [C, P, P, P]
        for f in (L.qstate_query_sizes, L.qstate_init, L.qstate_decode_step, L.qstate_readout,
                  L.qstate_selfcheck, L.qstate_fp32_decode_step, L.qstate_state_sq_norms,
                  L.qstate_fp32_sq_norms, L.qstate_lrb_query_sizes, L.qstate_lrb_decode_step,
                  L.qstate_prefill, L.qstate_prefill_tf32, L.qstate_prefill_tf32_timeouts,
                  L.qstate_prefill_tf32_wait_selfcheck, L.qstate_pipeline_query_sizes,
                  L.qstate_pipeline_create, L.qstate_pipeline_step, L.qstate_pipeline_wait_stream,
                  L.qstate_pipeline_join, L.qstate_pipeline_sync, L.qstate_pipeline_destroy,
                  L.qstate_decode_step_host_static):
            f.restype = ctypes.c_int
        L.qstate_status_string.argtypes = [ctypes.c_int]
        L.qstate_status_string.restype = ctypes.c_char_p
        L.qstate_version.argtypes = []
        L.qstate_version.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qstate_status_string(status).decode()


@dataclass(frozen=True)
class Config:
    """One family of quantized states (the fields of qs_config)."""
    num_tiles: int
    dk: int
    dv: int
    bits: int
    group: int
    delta: int
    decay: str = "scalar"
    policy: str = "persistent"
    rounding: str = "nearest"

    def c(self) -> qs_config:
        return qs_config(self.num_tiles, self.dk, self.dv, self.bits, self.group, self.delta,
                         DECAY[self.decay], POLICY[self.policy], ROUNDING[self.rounding])

    @property
    def groups(self) -> int:
        return self.dk // self.group


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str) -> None:
    if status != QS_OK:
        raise QStateError(status, what)


def query_sizes(cfg: Config):
    """(codes_bytes, scales_bytes, shadow_bytes) for cfg."""
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    cc = cfg.c()
    _check(lib().qstate_query_sizes(ctypes.byref(cc), ctypes.byref(a), ctypes.byref(b),
                                    ctypes.byref(c)), "qstate_query_sizes")
    return a.value, b.value, c.value


def init(cfg: Config, S0, codes, scales, shadow=None, stream=None) -> None:
    cc = cfg.c()
    _check(lib().qstate_init(ctypes.byref(cc), _ptr(S0), _ptr(codes), _ptr(scales), _ptr(shadow),
                             _stream(stream)), "qstate_init")


def decode_step(cfg: Config, codes, scales, shadow, q, k, v, alpha, beta, o=None,
                stream=None) -> None:
    cc = cfg.c()
    _check(lib().qstate_decode_step(ctypes.byref(cc), _ptr(codes), _ptr(scales), _ptr(shadow),
                                    _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                    _stream(stream)), "qstate_decode_step")


def readout(cfg: Config, codes, scales, q, o, stream=None) -> None:
    cc = cfg.c()
    _check(lib().qstate_readout(ctypes.byref(cc), _ptr(codes), _ptr(scales), _ptr(q), _ptr(o),
                                _stream(stream)), "qstate_readout")


def fp32_decode_step(cfg: Config, S, q, k, v, alpha, beta, o=None, stream=None) -> None:
    """The unquantized FP32 recurrence, in place on S (float32 [T, dv, dk])."""
    cc = cfg.c()
    _check(lib().qstate_fp32_decode_step(ctypes.byref(cc), _ptr(S), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(alpha), _ptr(beta), _ptr(o), _stream(stream)),
           "qstate_fp32_decode_step")


def lrb_query_sizes(cfg: Config, rank: int):
    """(decay_bytes, keys_bytes, coef_bytes) of the Low-Rank Bypass buffers."""
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    cc = cfg.c()
    _check(lib().qstate_lrb_query_sizes(ctypes.byref(cc), rank, ctypes.byref(a), ctypes.byref(b),
                                        ctypes.byref(c)), "qstate_lrb_query_sizes")
    return a.value, b.value, c.value


def lrb_decode_step(cfg: Config, rank: int, slot: int, codes, scales, shadow, A_in, A_out, K_in,
                    K_out, U, q, k, v, alpha, beta, o=None, stream=None) -> None:
    cc = cfg.c()
    _check(lib().qstate_lrb_decode_step(ctypes.byref(cc), rank, slot, _ptr(codes), _ptr(scales),
                                        _ptr(shadow), _ptr(A_in), _ptr(A_out), _ptr(K_in),
                                        _ptr(K_out), _ptr(U), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(alpha), _ptr(beta), _ptr(o), _stream(stream)),
           "qstate_lrb_decode_step")


class LrbBuffers:
    """Low-Rank Bypass buffers of one state family (qstate_lrb_decode_step):
    two copies of the accumulated decay A and of the buffered keys K (read one,
    write the other), the coefficients U, and the slot of the next step."""

    def __init__(self, cfg: Config, rank: int, device=None):
        import torch
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.cfg, self.rank, self.slot, self.cur = cfg, rank, 0, 0
        self.rpad = (rank + 3) // 4 * 4
        T = cfg.num_tiles
        z = lambda *shape: torch.zeros(shape, dtype=torch.float32, device=dev)
        self.A = [z(T, cfg.dk), z(T, cfg.dk)]
        self.K = [z(T, rank, cfg.dk), z(T, rank, cfg.dk)]
        self.U = z(T, cfg.dv, self.rpad)
        a, b, c = lrb_query_sizes(cfg, rank)
        assert a == 4 * self.A[0].numel() and b == 4 * self.K[0].numel() and c == 4 * self.U.numel()

    def step(self, st: "QState", q, k, v, alpha, beta, o=None, stream=None):
        i, j = self.cur, 1 - self.cur
        lrb_decode_step(self.cfg, self.rank, self.slot, st.codes, st.scales, st.shadow,
                        self.A[i], self.A[j], self.K[i], self.K[j], self.U, q, k, v, alpha, beta,
                        o, stream)
        if self.slot == self.rank - 1:
            self.slot = 0
        else:
            self.slot += 1
            self.cur = j
        return o


def prefill(cfg: Config, length: int, S, q, k, v, alpha, beta, o=None, stream=None) -> None:
    """Chunkwise prefill (delta = 0) of the FP32 state S [T][dv][dk] over
    `length` tokens: q, k [T][L][dk], v [T][L][dv], alpha [T][L] or
    [T][L][dk], beta [T][L]; o [T][L][dv] or None."""
    cc = cfg.c()
    _check(lib().qstate_prefill(ctypes.byref(cc), length, _ptr(S), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(alpha), _ptr(beta), _ptr(o), _stream(stream)),
           "qstate_prefill")


def prefill_tf32(cfg: Config, length: int, S, q, k, v, alpha, beta, o=None, stream=None,
                 check_timeouts: bool = True) -> None:
    """The same prefill on the tensor cores (TF32 operands, FP32 accumulators);
    S, q and k 16-byte aligned.  With check_timeouts (the default) the call
    synchronizes and raises if a CTA's bounded wait for the tensor cores gave
    up during it (S and o are then undefined); without it the call stays
    asynchronous and the caller compares prefill_tf32_timeouts() itself."""
    cc = cfg.c()
    before = prefill_tf32_timeouts() if check_timeouts else 0
    _check(lib().qstate_prefill_tf32(ctypes.byref(cc), length, _ptr(S), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(alpha), _ptr(beta), _ptr(o), _stream(stream)),
           "qstate_prefill_tf32")
    if check_timeouts:
        import torch
        torch.cuda.synchronize()
        gave_up = prefill_tf32_timeouts() - before
        if gave_up:
            raise RuntimeError(f"qstate_prefill_tf32: {gave_up} CTA(s) gave up waiting for the "
                               "tensor cores; S and o of this call are undefined")


def prefill_tf32_timeouts() -> int:
    """CTAs of prefill_tf32 whose bounded wait for the tensor cores gave up."""
    n = ctypes.c_uint(0)
    _check(lib().qstate_prefill_tf32_timeouts(ctypes.byref(n)), "qstate_prefill_tf32_timeouts")
    return n.value


def prefill_tf32_wait_selfcheck(polls: int = 1000) -> int:
    """Run the bounded-wait self-check of the tensor-core prefill; returns the
    number of CTAs that reported a timeout (1 when the mechanism works)."""
    n = ctypes.c_uint(0)
    _check(lib().qstate_prefill_tf32_wait_selfcheck(polls, ctypes.byref(n)),
           "qstate_prefill_tf32_wait_selfcheck")
    return n.value


def state_sq_norms(cfg: Config, codes, scales, out, stream=None) -> None:
    """out[t] (float64 [T]) = squared Frobenius norm of tile t of the stored state."""
    cc = cfg.c()
    _check(lib().qstate_state_sq_norms(ctypes.byref(cc), _ptr(codes), _ptr(scales), _ptr(out),
                                       _stream(stream)), "qstate_state_sq_norms")


def fp32_sq_norms(cfg: Config, S, out, stream=None) -> None:
    """out[t] (float64 [T]) = squared Frobenius norm of tile t of an FP32 state."""
    cc = cfg.c()
    _check(lib().qstate_fp32_sq_norms(ctypes.byref(cc), _ptr(S), _ptr(out), _stream(stream)),
           "qstate_fp32_sq_norms")


def selfcheck(stream=None):
    """Run qstate_selfcheck on the current GPU; returns the three mismatch
    counts (reciprocal, division by 7, division by 127), all expected 0."""
    import torch
    bad = torch.zeros(3, dtype=torch.int64, device="cuda")
    _check(lib().qstate_selfcheck(bad.data_ptr(), _stream(stream)), "qstate_selfcheck")
    torch.cuda.synchronize()
    return [int(x) for x in bad.cpu()]


class QState:
    """Device buffers of one quantized state family plus convenience calls.

    Buffers are torch tensors on the current CUDA device:
      codes  uint8 [T, dv, dk*bits/8], scales float32 [T, dv, dk/group],
      shadow float32 [T, dv, dk] (yoked only).
    """

    def __init__(self, cfg: Config, device=None):
        import torch
        self.cfg = cfg
        dev = torch.device("cuda") if device is None else torch.device(device)
        T, dv, dk = cfg.num_tiles, cfg.dv, cfg.dk
        self.codes = torch.empty((T, dv, dk * cfg.bits // 8), dtype=torch.uint8, device=dev)
        self.scales = torch.empty((T, dv, cfg.groups), dtype=torch.float32, device=dev)
        self.shadow = (torch.empty((T, dv, dk), dtype=torch.float32, device=dev)
                       if cfg.policy == "yoked" else None)
        cb, sb, hb = query_sizes(cfg)
        assert cb == self.codes.numel() and sb == 4 * self.scales.numel()
        assert hb == (0 if self.shadow is None else 4 * self.shadow.numel())
        # the C struct of cfg, built once: step() is called once per token
        self._cc = cfg.c()
        self._ccp = ctypes.byref(self._cc)

    def init(self, S0, stream=None) -> "QState":
        init(self.cfg, S0, self.codes, self.scales, self.shadow, stream)
        return self

    def step(self, q, k, v, alpha, beta, o=None, stream=None):
        _check(lib().qstate_decode_step(self._ccp, _ptr(self.codes), _ptr(self.scales),
                                        _ptr(self.shadow), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                        _ptr(beta), _ptr(o), _stream(stream)),
               "qstate_decode_step")
        return o

    def readout(self, q, o, stream=None):
        readout(self.cfg, self.codes, self.scales, q, o, stream)
        return o


def decode_step_host_static(cfg: Config, codes, scales, shadow, host_in, host_out=None,
                            stream=None) -> None:
    """qstate_decode_step_host_static: one decode step with inputs from host
    memory (the packed layout of pipeline_query_sizes with n = 1) and
    readouts back to host memory, staged through the library's static device
    array instead of any allocation.  host_in / host_out are host tensors
    (page-locked for asynchronous copies); read host_out after synchronizing
    with `stream`."""
    cc = cfg.c()
    _check(lib().qstate_decode_step_host_static(ctypes.byref(cc), _ptr(codes), _ptr(scales),
                                                _ptr(shadow), _ptr(host_in), _ptr(host_out),
                                                _stream(stream)),
           "qstate_decode_step_host_static")


def pipeline_query_sizes(cfg: Config, n: int):
    """(input bytes, output bytes) of one step of a host-buffer pipeline over
    n families of cfg's recurrence."""
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    cc = cfg.c()
    _check(lib().qstate_pipeline_query_sizes(ctypes.byref(cc), n, ctypes.byref(a), ctypes.byref(b)),
           "qstate_pipeline_query_sizes")
    return a.value, b.value


class HostPipeline:
    """Host-buffer decode pipeline (qstate_pipeline_*): step() takes one
    token's packed inputs from host memory (q | k | v | alpha | beta, float32,
    page-locked for asynchronous copies), runs the decode step of every state
    family on `stream`, and writes the readouts [n][T][dv] back to host
    memory; the copies run on the pipeline's own streams, `depth` steps deep.
    A step's host buffers may be reused, or its readouts read, once sync() has
    returned or the step `depth` calls later has been issued."""

    def __init__(self, states, depth: int = 3):
        self.cfgs = [st.cfg for st in states]
        n = len(self.cfgs)
        arr = (qs_config * n)(*[c.c() for c in self.cfgs])
        h = ctypes.c_void_p()
        _check(lib().qstate_pipeline_create(n, arr, depth, ctypes.byref(h)), "qstate_pipeline_create")
        self._h = h
        self.depth = depth
        self.in_bytes, self.out_bytes = pipeline_query_sizes(self.cfgs[0], n)
        self._default = tuple(states)
        self._arrays = {}

    def _state_arrays(self, states):
        key = tuple(id(st) for st in states)
        got = self._arrays.get(key)
        if got is None:
            if [st.cfg for st in states] != self.cfgs:
                raise ValueError("states do not match the pipeline's families")
            n = len(states)
            VP = ctypes.c_void_p
            got = (tuple(states),  # keeps the states (and their ids) alive with the entry
                   (VP * n)(*[_ptr(st.codes) for st in states]),
                   (VP * n)(*[_ptr(st.scales) for st in states]),
                   (VP * n)(*[_ptr(st.shadow) for st in states]))
            self._arrays[key] = got
        return got

    def step(self, host_in, host_out=None, stream=None, states=None):
        if host_in.numel() * host_in.element_size() < self.in_bytes:
            raise ValueError("host input smaller than one step's packed inputs")
        if host_out is not None and host_out.numel() * host_out.element_size() < self.out_bytes:
            raise ValueError("host output smaller than one step's readouts")
        _, codes, scales, shadow = self._state_arrays(self._default if states is None else states)
        _check(lib().qstate_pipeline_step(self._h, codes, scales, shadow, _ptr(host_in),
                                          _ptr(host_out), _stream(stream)), "qstate_pipeline_step")

    def wait_stream(self, stream=None):
        _check(lib().qstate_pipeline_wait_stream(self._h, _stream(stream)), "qstate_pipeline_wait_stream")

    def join(self, stream=None):
        _check(lib().qstate_pipeline_join(self._h, _stream(stream)), "qstate_pipeline_join")

    def sync(self):
        _check(lib().qstate_pipeline_sync(self._h), "qstate_pipeline_sync")

    def close(self):
        if self._h is not None:
            h, self._h = self._h, None
            _check(lib().qstate_pipeline_destroy(h), "qstate_pipeline_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
