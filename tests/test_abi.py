"""The C ABI library: it loads, exports every entry point include/*.h
declares, and rejects bad arguments before launching anything (so these
run without a GPU)."""
import ctypes
import glob
import os
import re

import pytest

from ssm_decode_step_b200 import qstate as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"QS_API\s+[\w\s\*]+?\b(qstate_\w+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    declared = _declared()
    assert declared, "no declarations found"
    lib = Q.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert set(Q.EXPORTS) >= set(declared)


def test_version_and_status_strings():
    assert Q.lib().qstate_version() >= 100
    for s in (0, 1, 2, 3):
        assert Q.status_string(s)


def _cfg(**kw):
    base = dict(num_tiles=4, dk=128, dv=128, bits=4, group=32, delta=1, decay="scalar",
                policy="persistent", rounding="nearest")
    base.update(kw)
    return Q.Config(**base)


def _raw(cfg):
    return cfg.c()


@pytest.mark.parametrize("field,value,status", [
    ("bits", 3, Q.QS_ERR_INVALID_ARG),
    ("bits", 16, Q.QS_ERR_INVALID_ARG),
    ("group", 48, Q.QS_ERR_INVALID_ARG),
    ("group", 16, Q.QS_ERR_UNSUPPORTED),
    ("dk", 96, Q.QS_ERR_UNSUPPORTED),
    ("dk", 256, Q.QS_ERR_UNSUPPORTED),
    ("dv", 24, Q.QS_ERR_UNSUPPORTED),
    ("dv", 4112, Q.QS_ERR_UNSUPPORTED),
    ("dv", 0, Q.QS_ERR_INVALID_ARG),
    ("num_tiles", -1, Q.QS_ERR_INVALID_ARG),
    ("delta", 2, Q.QS_ERR_INVALID_ARG),
    ("decay", 5, Q.QS_ERR_INVALID_ARG),
    ("policy", 3, Q.QS_ERR_INVALID_ARG),
    ("rounding", -1, Q.QS_ERR_INVALID_ARG),
])
def test_config_validation(field, value, status):
    c = _raw(_cfg())
    setattr(c, field, value)
    lib = Q.lib()
    assert lib.qstate_query_sizes(ctypes.byref(c), None, None, None) == status
    assert lib.qstate_decode_step(ctypes.byref(c), 16, 16, None, 16, 16, 16, 16, 16, None, None) == status


def test_null_config():
    lib = Q.lib()
    assert lib.qstate_query_sizes(None, None, None, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_init(None, 16, 16, 16, None, None) == Q.QS_ERR_INVALID_ARG


def test_sizes():
    assert Q.query_sizes(_cfg(num_tiles=1024)) == (1024 * 128 * 64, 1024 * 128 * 4 * 4, 0)
    assert Q.query_sizes(_cfg(num_tiles=3, bits=8, group=64, dv=64, policy="yoked")) == \
        (3 * 64 * 128, 3 * 64 * 2 * 4, 3 * 64 * 128 * 4)


# Fake device addresses: validation rejects these before any CUDA call.
A = 1 << 20


def _step(cfg, **ptrs):
    p = dict(codes=A, scales=2 * A, shadow=None, q=3 * A, k=4 * A, v=5 * A, alpha=6 * A,
             beta=7 * A, o=8 * A)
    p.update(ptrs)
    c = cfg.c()
    return Q.lib().qstate_decode_step(ctypes.byref(c), p["codes"], p["scales"], p["shadow"],
                                      p["q"], p["k"], p["v"], p["alpha"], p["beta"], p["o"], None)


@pytest.mark.parametrize("ptrs", [
    dict(codes=None), dict(scales=None), dict(k=None), dict(v=None), dict(alpha=None),
    dict(beta=None), dict(q=None),                         # o given without q
    dict(codes=A + 8), dict(codes=A + 16), dict(scales=2 * A + 4), dict(k=4 * A + 4), dict(q=3 * A + 8),
    dict(v=5 * A + 12), dict(beta=7 * A + 2), dict(o=8 * A + 1),
    dict(scales=A + 64),                                   # overlaps codes
    dict(o=4 * A),                                         # output overlaps an input
])
def test_pointer_validation(ptrs):
    assert _step(_cfg(), **ptrs) == Q.QS_ERR_INVALID_ARG


def test_yoked_needs_shadow_and_diag_alpha_alignment():
    assert _step(_cfg(policy="yoked")) == Q.QS_ERR_INVALID_ARG
    assert _step(_cfg(policy="yoked"), shadow=9 * A + 4) == Q.QS_ERR_INVALID_ARG
    assert _step(_cfg(policy="yoked"), shadow=9 * A + 16) == Q.QS_ERR_INVALID_ARG
    assert _step(_cfg(decay="diagonal"), alpha=6 * A + 4) == Q.QS_ERR_INVALID_ARG


def test_readout_validation():
    c = _cfg().c()
    lib = Q.lib()
    assert lib.qstate_readout(ctypes.byref(c), None, 2 * A, 3 * A, 8 * A, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_readout(ctypes.byref(c), A, 2 * A, 3 * A + 4, 8 * A, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_readout(ctypes.byref(c), A, 2 * A, 3 * A, A + 16, None) == Q.QS_ERR_INVALID_ARG


def test_norms_validation():
    # null, misaligned and overlapping arguments are rejected before any launch
    c = _cfg().c()
    lib = Q.lib()
    assert lib.qstate_state_sq_norms(ctypes.byref(c), None, 2 * A, 8 * A, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_state_sq_norms(ctypes.byref(c), A + 16, 2 * A, 8 * A, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_state_sq_norms(ctypes.byref(c), A, 2 * A, 8 * A + 4, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_state_sq_norms(ctypes.byref(c), A, 2 * A, A + 64, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_fp32_sq_norms(ctypes.byref(c), None, 8 * A, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_fp32_sq_norms(ctypes.byref(c), A + 4, 8 * A, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_fp32_sq_norms(ctypes.byref(c), A, A + 64, None) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_fp32_sq_norms(None, A, 8 * A, None) == Q.QS_ERR_INVALID_ARG


def _lrb(rank, slot, **ptrs):
    p = dict(codes=A, scales=2 * A, shadow=None, A_in=10 * A, A_out=11 * A, K_in=12 * A,
             K_out=13 * A, U=14 * A, q=3 * A, k=4 * A, v=5 * A, alpha=6 * A, beta=7 * A, o=8 * A)
    p.update(ptrs)
    c = _cfg().c()
    return Q.lib().qstate_lrb_decode_step(ctypes.byref(c), rank, slot, p["codes"], p["scales"],
                                          p["shadow"], p["A_in"], p["A_out"], p["K_in"], p["K_out"],
                                          p["U"], p["q"], p["k"], p["v"], p["alpha"], p["beta"],
                                          p["o"], None)


def test_lrb_validation():
    # rejected before any launch: unsupported rank, slot outside the period,
    # missing or misaligned buffers, buffers overlapping the state
    assert _lrb(0, 0) == Q.QS_ERR_UNSUPPORTED
    assert _lrb(17, 0) == Q.QS_ERR_UNSUPPORTED
    assert _lrb(4, 4) == Q.QS_ERR_INVALID_ARG
    assert _lrb(4, -1) == Q.QS_ERR_INVALID_ARG
    assert _lrb(4, 1, U=None) == Q.QS_ERR_INVALID_ARG
    assert _lrb(4, 1, A_in=None) == Q.QS_ERR_INVALID_ARG
    assert _lrb(4, 1, K_out=None) == Q.QS_ERR_INVALID_ARG
    assert _lrb(4, 1, U=14 * A + 4) == Q.QS_ERR_INVALID_ARG
    assert _lrb(4, 1, A_out=A + 64) == Q.QS_ERR_INVALID_ARG
    assert _lrb(4, 1, K_out=12 * A) == Q.QS_ERR_INVALID_ARG
    cfg = _cfg()
    assert Q.lrb_query_sizes(cfg, 6) == (4 * 128 * 4, 4 * 6 * 128 * 4, 4 * 128 * 8 * 4)


def test_prefill_validation():
    lib = Q.lib()
    pre = lambda cfg, L, **kw: lib.qstate_prefill(ctypes.byref(cfg.c()), L, kw.get("S", A), kw.get("q", 2 * A),
                                                  kw.get("k", 3 * A), kw.get("v", 4 * A), kw.get("a", 5 * A),
                                                  kw.get("b", 6 * A), kw.get("o", 7 * A), None)
    assert pre(_cfg(delta=0, dv=256), 8) == Q.QS_ERR_UNSUPPORTED
    assert pre(_cfg(delta=1, dv=256), 8) == Q.QS_ERR_UNSUPPORTED
    for d in (0, 1):  # the FP32 path takes the linear write and the delta rule
        assert pre(_cfg(delta=d), -1) == Q.QS_ERR_INVALID_ARG
        assert pre(_cfg(delta=d), 8, S=None) == Q.QS_ERR_INVALID_ARG
        assert pre(_cfg(delta=d), 8, o=A + 64) == Q.QS_ERR_INVALID_ARG
        assert pre(_cfg(delta=d), 0, S=None) == Q.QS_OK
    assert pre(_cfg(delta=2), 8) == Q.QS_ERR_INVALID_ARG


def test_prefill_tf32_validation():
    """The tensor-core prefill takes the same arguments as qstate_prefill and
    also needs S, q and k 16-byte aligned (rejected before any launch)."""
    lib = Q.lib()
    pre = lambda cfg, L, **kw: lib.qstate_prefill_tf32(
        ctypes.byref(cfg.c()), L, kw.get("S", A), kw.get("q", 2 * A), kw.get("k", 3 * A),
        kw.get("v", 4 * A), kw.get("a", 5 * A), kw.get("b", 6 * A), kw.get("o", 7 * A), None)
    assert pre(_cfg(delta=1), 8) == Q.QS_ERR_UNSUPPORTED
    assert pre(_cfg(delta=1), 0, S=None) == Q.QS_ERR_UNSUPPORTED
    assert pre(_cfg(delta=0, dv=256), 8) == Q.QS_ERR_UNSUPPORTED
    assert pre(_cfg(delta=0), -1) == Q.QS_ERR_INVALID_ARG
    assert pre(_cfg(delta=0), 8, S=None) == Q.QS_ERR_INVALID_ARG
    assert pre(_cfg(delta=0), 8, S=A + 4) == Q.QS_ERR_INVALID_ARG
    assert pre(_cfg(delta=0), 8, q=2 * A + 8) == Q.QS_ERR_INVALID_ARG
    assert pre(_cfg(delta=0), 8, k=3 * A + 4) == Q.QS_ERR_INVALID_ARG
    assert pre(_cfg(delta=0), 8, o=A + 64) == Q.QS_ERR_INVALID_ARG
    assert pre(_cfg(delta=0), 0, S=None) == Q.QS_OK
    with pytest.raises(Q.QStateError):
        lib_call = lib.qstate_prefill_tf32_timeouts(None)
        Q._check(lib_call, "qstate_prefill_tf32_timeouts")
    n = ctypes.c_uint(0)
    assert lib.qstate_prefill_tf32_wait_selfcheck(0, ctypes.byref(n)) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_prefill_tf32_wait_selfcheck(1 << 21, ctypes.byref(n)) == Q.QS_ERR_INVALID_ARG
    assert lib.qstate_prefill_tf32_wait_selfcheck(1000, None) == Q.QS_ERR_INVALID_ARG


def test_binding_raises():
    with pytest.raises(Q.QStateError):
        Q.query_sizes(_cfg(bits=5))


def test_pipeline_sizes_and_validation_without_a_gpu():
    """Host-buffer pipeline: sizes of one step's packed input and readouts,
    and every argument check that runs before a CUDA call."""
    L = Q.lib()
    cfg = _cfg(num_tiles=5, dv=64, decay="diagonal")
    inb, outb = Q.pipeline_query_sizes(cfg, 2)
    assert inb == 4 * 5 * (128 + 128 + 64 + 128 + 1)       # q, k, v, diagonal alpha, beta
    assert outb == 2 * 4 * 5 * 64
    inb1, _ = Q.pipeline_query_sizes(_cfg(num_tiles=5, dv=64), 1)
    assert inb1 == 4 * 5 * (128 + 128 + 64 + 1 + 1)         # scalar alpha
    h = ctypes.c_void_p()
    one = (Q.qs_config * 1)(_raw(cfg))
    assert L.qstate_pipeline_create(0, one, 3, ctypes.byref(h)) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_create(9, one, 3, ctypes.byref(h)) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_create(1, one, 1, ctypes.byref(h)) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_create(1, one, 9, ctypes.byref(h)) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_create(1, one, 3, None) == Q.QS_ERR_INVALID_ARG
    assert h.value is None
    # families must share the recurrence (tiles, dk, dv, delta, decay)
    for other in (_cfg(num_tiles=6, dv=64, decay="diagonal"), _cfg(num_tiles=5, dv=80, decay="diagonal"),
                  _cfg(num_tiles=5, dv=64, decay="scalar"), _cfg(num_tiles=5, dv=64, decay="diagonal", delta=0)):
        two = (Q.qs_config * 2)(_raw(cfg), _raw(other))
        assert L.qstate_pipeline_create(2, two, 3, ctypes.byref(h)) == Q.QS_ERR_INVALID_ARG
    # an unsupported family is reported as such
    two = (Q.qs_config * 2)(_raw(cfg), _raw(_cfg(num_tiles=5, dv=64, decay="diagonal", group=16)))
    assert L.qstate_pipeline_create(2, two, 3, ctypes.byref(h)) == Q.QS_ERR_UNSUPPORTED
    assert L.qstate_pipeline_step(None, None, None, None, None, None, None) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_sync(None) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_join(None, None) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_wait_stream(None, None) == Q.QS_ERR_INVALID_ARG
    assert L.qstate_pipeline_destroy(None) == Q.QS_OK


def test_host_pipeline_fails_loudly_without_a_device():
    """Creating a pipeline needs the device (memory, streams, events): with
    none, the binding raises the library's CUDA error; there is no fallback."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")

    class Fake:
        def __init__(self, cfg):
            self.cfg = cfg

    with pytest.raises(Q.QStateError) as e:
        Q.HostPipeline([Fake(_cfg()), Fake(_cfg(policy="yoked"))], depth=3)
    assert e.value.status == Q.QS_ERR_CUDA
    with pytest.raises(Q.QStateError) as e:
        Q.HostPipeline([Fake(_cfg()), Fake(_cfg(num_tiles=5))], depth=3)
    assert e.value.status == Q.QS_ERR_INVALID_ARG    # checked before any CUDA call
