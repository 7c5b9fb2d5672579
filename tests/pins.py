"""Pins of the CPU oracle: checks against what the pages and the mathematics
fix, each independent of the oracle's own code path.

Every pin is a plain function that raises AssertionError on failure, so that
test_oracle_pins.py runs them one by one and test_oracle_mutations.py can
run them all against the oracle's mutation build with a mistake planted in
it (oracle.planted) and require that some pin catches each mistake.

Sources:
* eq. (1) and its decay / delta / write-gate choices: "LinQuant: Functional
  Invariances for Low-Precision Linear Recurrences", Theoretical Foundation;
* invariances used as properties: same page, The Seven Functional
  Invariances, key-side rotation (1/7), key-side rescaling (2/7),
  value-side rescaling (4/7);
* policies: "When Dynamic Scaling Fails" project page (per-token dynamic,
  static/persistent, yoked to a full-precision reference);
* BDR: "Preserving Updates in Low-Bit Recurrent State Quantization",
  abstract.
"""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

F32 = np.float32


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(g):
    return g / np.linalg.norm(g, axis=-1, keepdims=True)


def _inputs(rng, T, dk, dv, decay, unit_k=True, alpha=None, beta=None):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if unit_k:
        k = _unit(k)
    v = rng.standard_normal((T, dv))
    if alpha is None:
        alpha = rng.uniform(0.8, 1.0, size=(T, dk) if decay == "diagonal" else (T,))
    if beta is None:
        beta = rng.uniform(0.1, 1.0, size=(T,))
    f = lambda a: np.ascontiguousarray(a, dtype=F32)
    return f(q), f(k), f(v), f(np.broadcast_to(alpha, (T, dk) if decay == "diagonal" else (T,))), \
        f(np.broadcast_to(beta, (T,)))


def _decay64(alpha, decay, dk):
    a = alpha.astype(np.float64)
    return a if decay == "diagonal" else np.repeat(a[:, None], dk, axis=1)


# --------------------------------------------------------------------------
# The FP32 recurrence (the oracle's unquantized step)
# --------------------------------------------------------------------------

def pin_linear_write_sum_of_outer_products():
    """delta = 0, Lambda = I, beta = 1, S0 = 0  =>  S_H = sum_t v_t k_t^T."""
    rng = _rng(10)
    for decay in ("scalar", "diagonal"):
        T, dk, dv, H = 3, 32, 5, 12
        cfg = O.OracleConfig(T, dk, dv, 8, 16, 0, decay)
        S = np.zeros((T, dv, dk), F32)
        acc = np.zeros((T, dv, dk))
        for _ in range(H):
            q, k, v, a, b = _inputs(rng, T, dk, dv, decay, unit_k=False,
                                    alpha=1.0, beta=1.0)
            O.fp32_step(cfg, S, q, k, v, a, b, want_o=False)
            acc += np.einsum("ti,tj->tij", v.astype(np.float64), k.astype(np.float64))
        err = np.abs(S - acc).max() / np.abs(acc).max()
        assert err < 1e-6, err


def pin_decay_closed_form():
    """delta = 0, S0 = 0:  S_H = sum_t beta_t v_t (k_t * prod_{s>t} a_s)^T
    for scalar and diagonal decay (the decay multiplies the key side)."""
    rng = _rng(11)
    for decay in ("scalar", "diagonal"):
        T, dk, dv, H = 2, 32, 3, 10
        cfg = O.OracleConfig(T, dk, dv, 8, 16, 0, decay)
        S = np.zeros((T, dv, dk), F32)
        steps = [_inputs(rng, T, dk, dv, decay, unit_k=False) for _ in range(H)]
        for q, k, v, a, b in steps:
            O.fp32_step(cfg, S, q, k, v, a, b, want_o=False)
        ref = np.zeros((T, dv, dk))
        for t, (q, k, v, a, b) in enumerate(steps):
            later = np.ones((T, dk))
            for s in range(t + 1, H):
                later *= _decay64(steps[s][3], decay, dk)
            ref += b.astype(np.float64)[:, None, None] * np.einsum(
                "ti,tj->tij", v.astype(np.float64), k.astype(np.float64) * later)
        err = np.abs(S - ref).max() / np.abs(ref).max()
        assert err < 1e-5, (decay, err)


def pin_delta_rule_key_recall():
    """delta = 1, ||k|| = 1:  S_t k_t = (1 - beta_t) S_{t-1} Lambda_t k_t + beta_t v_t,
    for any decay; with beta = 1 the key recalls its value exactly."""
    rng = _rng(12)
    for decay in ("scalar", "diagonal"):
        for beta_one in (False, True):
            T, dk, dv = 3, 32, 6
            cfg = O.OracleConfig(T, dk, dv, 8, 16, 1, decay)
            S = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
            for _ in range(8):
                q, k, v, a, b = _inputs(rng, T, dk, dv, decay,
                                        beta=1.0 if beta_one else None)
                prev = S.astype(np.float64).copy()
                O.fp32_step(cfg, S, q, k, v, a, b, want_o=False)
                k64 = k.astype(np.float64)
                lhs = np.einsum("tij,tj->ti", S.astype(np.float64), k64)
                Sd = prev * _decay64(a, decay, dk)[:, None, :]
                rhs = (1 - b.astype(np.float64))[:, None] * np.einsum("tij,tj->ti", Sd, k64) \
                    + b.astype(np.float64)[:, None] * v.astype(np.float64)
                scale = 1.0 + np.abs(rhs).max()
                assert np.abs(lhs - rhs).max() < 2e-5 * scale, (decay, beta_one)


def pin_readout_is_state_times_q():
    """o_t = S_t q_t with S_t the updated state (FP32 recurrence)."""
    rng = _rng(13)
    for delta in (0, 1):
        T, dk, dv = 2, 64, 4
        cfg = O.OracleConfig(T, dk, dv, 8, 16, delta, "scalar")
        S = (rng.standard_normal((T, dv, dk)) * 0.2).astype(F32)
        for _ in range(4):
            q, k, v, a, b = _inputs(rng, T, dk, dv, "scalar")
            o = O.fp32_step(cfg, S, q, k, v, a, b)
            ref = np.einsum("tij,tj->ti", S.astype(np.float64), q.astype(np.float64))
            assert np.abs(o - ref).max() < 1e-5 * (1 + np.abs(ref).max())


def pin_value_rescaling_exact():
    """v -> D_V v with D_V a positive diagonal of powers of two: the FP32
    state becomes D_V S bit for bit, and the quantized state keeps its codes
    while its scales take the factor (LinQuant 4/7, exact for powers of two)."""
    rng = _rng(14)
    T, dk, dv = 2, 32, 8
    d = (2.0 ** rng.integers(-3, 4, size=dv)).astype(F32)
    for delta in (0, 1):
        for decay in ("scalar", "diagonal"):
            cfg = O.OracleConfig(T, dk, dv, 8, 16, delta, decay)
            S = (rng.standard_normal((T, dv, dk)) * 0.2).astype(F32)
            S2 = (S * d[None, :, None]).astype(F32)
            for _ in range(5):
                q, k, v, a, b = _inputs(rng, T, dk, dv, decay)
                O.fp32_step(cfg, S, q, k, v, a, b, want_o=False)
                O.fp32_step(cfg, S2, q, k, (v * d[None, :]).astype(F32), a, b, want_o=False)
            assert np.array_equal(S2, (S * d[None, :, None]).astype(F32))
            for policy in ("dynamic", "persistent", "yoked"):
                for rounding in ("nearest", "bdr"):
                    qc = O.OracleConfig(T, dk, dv, 4, 16, delta, decay, policy, rounding)
                    S0 = (rng.standard_normal((T, dv, dk)) * 0.2).astype(F32)
                    A = O.init(qc, S0)
                    B = O.init(qc, (S0 * d[None, :, None]).astype(F32))
                    for _ in range(5):
                        q, k, v, a, b = _inputs(rng, T, dk, dv, decay)
                        O.step(A, q, k, v, a, b, want_o=False)
                        O.step(B, q, k, (v * d[None, :]).astype(F32), a, b, want_o=False)
                    assert np.array_equal(A.codes, B.codes), (policy, rounding)
                    assert np.array_equal(B.scales, (A.scales * d[None, :, None]).astype(F32))


def _rotation(rng, n):
    Q, R = np.linalg.qr(rng.standard_normal((n, n)))
    return Q * np.sign(np.diag(R))[None, :]


def pin_key_rotation():
    """(q, k) -> (R q, R k) with R orthogonal leaves the readout unchanged
    when R commutes with Lambda (no or scalar decay), also for the delta rule
    (LinQuant 1/7); diagonal decay breaks it."""
    rng = _rng(15)
    T, dk, dv, H = 2, 32, 4, 6
    R = _rotation(rng, dk)
    for decay, delta, should_hold in (("scalar", 0, True), ("scalar", 1, True),
                                      ("diagonal", 0, False)):
        cfg = O.OracleConfig(T, dk, dv, 8, 16, delta, decay)
        S = np.zeros((T, dv, dk), F32)
        Sr = np.zeros((T, dv, dk), F32)
        worst = 0.0
        for _ in range(H):
            q, k, v, a, b = _inputs(rng, T, dk, dv, decay)
            o = O.fp32_step(cfg, S, q, k, v, a, b)
            orot = O.fp32_step(cfg, Sr, (q @ R.T).astype(F32), (k @ R.T).astype(F32), v, a, b)
            worst = max(worst, np.abs(o - orot).max() / (1 + np.abs(o).max()))
        assert (worst < 1e-5) == should_hold, (decay, delta, worst)


def pin_key_rescaling():
    """(q, k) -> (D q, D^-1 k), D positive diagonal (powers of two): the
    readout is unchanged bit for bit for linear writes under scalar or
    diagonal decay; the delta rule does not preserve it (LinQuant 2/7)."""
    rng = _rng(16)
    T, dk, dv, H = 2, 32, 4, 6
    d = (2.0 ** rng.integers(-2, 3, size=dk)).astype(F32)
    for decay, delta, should_hold in (("scalar", 0, True), ("diagonal", 0, True),
                                      ("scalar", 1, False)):
        cfg = O.OracleConfig(T, dk, dv, 8, 16, delta, decay)
        S = np.zeros((T, dv, dk), F32)
        Sd = np.zeros((T, dv, dk), F32)
        same = True
        for _ in range(H):
            q, k, v, a, b = _inputs(rng, T, dk, dv, decay)
            o = O.fp32_step(cfg, S, q, k, v, a, b)
            od = O.fp32_step(cfg, Sd, (q * d).astype(F32), (k / d).astype(F32), v, a, b)
            same = same and np.array_equal(o, od)
        assert same == should_hold, (decay, delta)


# --------------------------------------------------------------------------
# Quantizer, policies, BDR
# --------------------------------------------------------------------------

def _x64(prev: "O.State", q, k, v, a, b, cfg):
    """Updated state x in float64 from the previous quantized state, written
    from eq. (1) with numpy (independent of the oracle's loops)."""
    d = prev.codes.astype(np.float64) * np.repeat(prev.scales.astype(np.float64), cfg.group, axis=-1)
    Sd = d * _decay64(a, cfg.decay, cfg.dk)[:, None, :]
    k64 = k.astype(np.float64)
    if cfg.delta:
        w = b.astype(np.float64)[:, None] * (v.astype(np.float64) - np.einsum("tij,tj->ti", Sd, k64))
    else:
        w = b.astype(np.float64)[:, None] * v.astype(np.float64)
    return Sd + w[:, :, None] * k64[:, None, :], Sd, w


def pin_quantizer_error_bound():
    """Quantize -> dequantize error is at most half a grid step per element,
    except where the persistent (or yoked) scale clips."""
    rng = _rng(17)
    T, dk, dv = 3, 64, 8
    for bits in (4, 8):
        for policy in ("dynamic", "persistent", "yoked"):
            cfg = O.OracleConfig(T, dk, dv, bits, 32, 1, "scalar", policy)
            S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
            st = O.init(cfg, S0)
            # init itself: |S0 - n s| <= s/2 (init uses the dynamic rule)
            deq = st.codes * np.repeat(st.scales, cfg.group, axis=-1).astype(np.float64)
            s_el = np.repeat(st.scales, cfg.group, axis=-1).astype(np.float64)
            assert np.all(np.abs(S0 - deq) <= 0.5 * s_el * (1 + 1e-6))
            for _ in range(6):
                q, k, v, a, b = _inputs(rng, T, dk, dv, "scalar")
                prev = st.copy()
                x64, _, _ = _x64(prev, q, k, v, a, b, cfg)
                O.step(st, q, k, v, a, b, want_o=False)
                s_el = np.repeat(st.scales, cfg.group, axis=-1).astype(np.float64)
                err = np.abs(x64 - st.codes * s_el)
                clipped = np.abs(st.codes) == cfg.qmax
                ok = err <= 0.5 * s_el * (1 + 1e-5) + 1e-6 * np.abs(x64)
                assert np.all(ok | (clipped & (policy != "dynamic"))), (bits, policy)


def pin_dynamic_scale_reaches_qmax():
    """Dynamic scale = group max|x| / qmax: every group with a nonzero entry
    has an element at code magnitude qmax, and the scale equals the group
    maximum of the float64 update over qmax to FP32 precision."""
    rng = _rng(18)
    T, dk, dv = 3, 64, 8
    for bits in (4, 8):
        cfg = O.OracleConfig(T, dk, dv, bits, 32, 1, "scalar", "dynamic")
        st = O.init(cfg, (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32))
        for _ in range(5):
            q, k, v, a, b = _inputs(rng, T, dk, dv, "scalar")
            x64, _, _ = _x64(st.copy(), q, k, v, a, b, cfg)
            O.step(st, q, k, v, a, b, want_o=False)
            m = np.abs(st.codes).reshape(T, dv, dk // 32, 32).max(axis=-1)
            assert np.all(m == cfg.qmax)
            gmax = np.abs(x64).reshape(T, dv, dk // 32, 32).max(axis=-1)
            assert np.allclose(st.scales, gmax / cfg.qmax, rtol=2e-6, atol=0)


def pin_persistent_zero_update():
    """A zero update (k = 0, alpha = 1) leaves persistent codes and scales
    bit-identical, for both write kinds."""
    rng = _rng(19)
    T, dk, dv = 3, 64, 8
    for bits in (4, 8):
        for delta in (0, 1):
            for rounding in ("nearest", "bdr"):
                cfg = O.OracleConfig(T, dk, dv, bits, 32, delta, "scalar", "persistent", rounding)
                st = O.init(cfg, (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32))
                before = st.copy()
                q, _, v, _, b = _inputs(rng, T, dk, dv, "scalar")
                O.step(st, q, np.zeros((T, dk), F32), v, np.ones(T, F32), b, want_o=False)
                assert np.array_equal(st.codes, before.codes)
                assert np.array_equal(st.scales, before.scales)


def pin_persistent_scales_fixed():
    """Persistent scales are those of the quantization start, forever."""
    rng = _rng(20)
    T, dk, dv = 2, 64, 8
    cfg = O.OracleConfig(T, dk, dv, 4, 32, 1, "scalar", "persistent")
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
    st = O.init(cfg, S0)
    s0 = st.scales.copy()
    for _ in range(10):
        O.step(st, *_inputs(rng, T, dk, dv, "scalar"), want_o=False)
    assert np.array_equal(st.scales, s0)
    # and they are max|S0| / qmax of each group
    gmax = np.abs(S0.astype(np.float64)).reshape(T, dv, 2, 32).max(axis=-1)
    assert np.allclose(s0, gmax / cfg.qmax, rtol=1e-6, atol=0)


def pin_zero_scale_group():
    """A group that is all zero at the quantization start has scale 0 and
    codes 0; under the persistent scale it stays 0."""
    rng = _rng(21)
    T, dk, dv = 1, 64, 4
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
    S0[0, 1, 32:64] = 0.0
    cfg = O.OracleConfig(T, dk, dv, 8, 32, 1, "scalar", "persistent")
    st = O.init(cfg, S0)
    assert st.scales[0, 1, 1] == 0.0 and np.all(st.codes[0, 1, 32:] == 0)
    for _ in range(3):
        O.step(st, *_inputs(rng, T, dk, dv, "scalar"), want_o=False)
    assert st.scales[0, 1, 1] == 0.0 and np.all(st.codes[0, 1, 32:] == 0)


def pin_bdr_bruteforce():
    """BDR against nearest rounding from the same state and inputs, element by
    element: with sigma = sign(w) sign(k_j) and d = c * s the element as
    stored before the step, BDR's own move is never against the update and
    never more than one code step (the chosen code is nearest or
    nearest + sigma, clamped); it equals nearest when sigma = 0 or when
    nearest does not move the stored element against sigma; and where
    nearest does, it is nearest + sigma unless that leaves [-qmax, qmax].
    With a fixed scale and no decay nearest never moves an element against
    its update, so BDR leaves every code alone; decay or a scale change are
    what make reversals (checked both ways below)."""
    rng = _rng(22)
    T, dk, dv = 8, 32, 4
    moved = 0
    for bits in (4, 8):
        for policy in ("persistent", "dynamic"):
            for decay_lo in (0.8, 1.0):
                qmax = (1 << (bits - 1)) - 1
                cN = O.OracleConfig(T, dk, dv, bits, 16, 0, "diagonal", policy, "nearest")
                cB = O.OracleConfig(T, dk, dv, bits, 16, 0, "diagonal", policy, "bdr")
                S0 = (rng.standard_normal((T, dv, dk)) * 0.5).astype(F32)
                B = O.init(cB, S0)
                for _ in range(8):
                    q, k, v, a, b = _inputs(rng, T, dk, dv, "diagonal")
                    if decay_lo == 1.0:
                        a = np.ones_like(a)
                    k[:, ::5] = 0.0          # some columns with no update
                    v[:, 0] = 0.0            # a row with no update
                    v = (v * 0.05).astype(F32)   # small updates: reversals are common
                    prev = B.copy()
                    Nst = O.State(cN, prev.codes.copy(), prev.scales.copy())
                    O.step(Nst, q, k, v, a, b, want_o=False)
                    O.step(B, q, k, v, a, b, want_o=False)
                    d = (prev.codes.astype(F32) * np.repeat(prev.scales, 16, axis=-1)).astype(F32)
                    w = (b[:, None] * v).astype(F32)
                    sigma = np.sign(w)[:, :, None] * np.sign(k)[:, None, :]
                    s_el = np.repeat(B.scales, 16, axis=-1)
                    n_near, n = Nst.codes, B.codes
                    assert np.array_equal(Nst.scales, B.scales)
                    step = n - n_near
                    assert np.all((step == 0) | (step == sigma))
                    dqn = (n_near.astype(F32) * s_el).astype(F32)
                    near_rev = (((sigma > 0) & (dqn < d)) | ((sigma < 0) & (dqn > d))) & (s_el > 0)
                    assert np.all(n[~near_rev] == n_near[~near_rev])
                    want = np.clip(n_near + sigma.astype(np.int64), -qmax, qmax)
                    assert np.array_equal(n[near_rev], want[near_rev])
                    if policy == "persistent" and decay_lo == 1.0:
                        assert not np.any(near_rev)
                    moved += int(np.count_nonzero(step))
    assert moved > 0


def pin_bdr_reversal_explained():
    """The specification's BDR invariant, its first clause (BDR never moves
    an element against its update), as it holds under the stored-value
    reading of the move ("Preserving Updates", abstract: BDR rounds the
    elements that moved opposite to their updates toward them).
    The move is measured from d = c * s, the element as stored before the
    step.  Without decay (Lambda = I) no element ends the step against its
    update, under a fixed or a changing scale.  With decay, an element can:
    the decay shrinks it before the write, and when the shrinkage exceeds
    what one code step can restore it stays on the wrong side of d.  The
    pin checks both directions and the bound: an element that ends against
    sigma after BDR has sigma (d - S') > s'/2 (S' the decayed element before
    the write) when its code is not at the clamp, and sigma (d - S') > 0
    when it is.  Derivation: x lies on the update's side of S', nearest puts
    n s' within s'/2 of x, and BDR's step adds s' when n s' was against d."""
    rng = _rng(28)
    T, dk, dv, G = 8, 32, 4, 16
    seen_against = 0
    for bits in (4, 8):
        qmax = (1 << (bits - 1)) - 1
        for policy in ("persistent", "dynamic"):
            for decay_lo in (1.0, 0.8):
                cfg = O.OracleConfig(T, dk, dv, bits, G, 0, "diagonal", policy, "bdr")
                st = O.init(cfg, (rng.standard_normal((T, dv, dk)) * 0.5).astype(F32))
                for _ in range(10):
                    q, k, v, a, b = _inputs(rng, T, dk, dv, "diagonal")
                    if decay_lo == 1.0:
                        a = np.ones_like(a)
                    v = (v * 0.05).astype(F32)
                    prev = st.copy()
                    O.step(st, q, k, v, a, b, want_o=False)
                    s_old = np.repeat(prev.scales, G, axis=-1)
                    d = (prev.codes.astype(F32) * s_old).astype(F32)
                    Sp = (prev.codes.astype(F32) * (s_old * a[:, None, :]).astype(F32)).astype(F32)
                    w = (b[:, None] * v).astype(F32)
                    sigma = np.sign(w)[:, :, None] * np.sign(k)[:, None, :]
                    s_new = np.repeat(st.scales, G, axis=-1)
                    val = (st.codes.astype(F32) * s_new).astype(F32)
                    against = (((sigma > 0) & (val < d)) | ((sigma < 0) & (val > d))) & (s_new > 0)
                    if decay_lo == 1.0:
                        assert not np.any(against), (bits, policy)
                        continue
                    seen_against += int(against.sum())
                    shrink = sigma * (d.astype(np.float64) - Sp)
                    slack = 1e-6 * (np.abs(d) + np.abs(Sp) + s_new)
                    clamped = np.abs(st.codes) == qmax
                    assert np.all(shrink[against & ~clamped] > 0.5 * s_new[against & ~clamped]
                                  - slack[against & ~clamped]), (bits, policy)
                    assert np.all(shrink[against & clamped] > -slack[against & clamped]), (bits, policy)
    assert seen_against > 0


def pin_yoked_shadow_is_fp32_run():
    """The yoked shadow follows the unquantized FP32 recurrence bit for bit
    (the full-precision reference run alongside)."""
    rng = _rng(23)
    T, dk, dv = 2, 64, 8
    for decay in ("scalar", "diagonal"):
        cfg = O.OracleConfig(T, dk, dv, 4, 32, 1, decay, "yoked")
        S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
        st = O.init(cfg, S0)
        S = S0.copy()
        for _ in range(6):
            inp = _inputs(rng, T, dk, dv, decay)
            O.step(st, *inp, want_o=False)
            O.fp32_step(cfg, S, *inp, want_o=False)
        assert np.array_equal(st.shadow, S)


def pin_yoked_scale_from_shadow_only():
    """Yoked scales are a function of the shadow trajectory alone: two runs
    that share the shadow but start from different codes get the same scales
    (the feedback loop from the quantized state to the scale is cut)."""
    rng = _rng(24)
    T, dk, dv = 2, 64, 8
    cfg = O.OracleConfig(T, dk, dv, 4, 32, 1, "scalar", "yoked")
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
    A = O.init(cfg, S0)
    B = A.copy()
    B.codes = np.clip(B.codes + rng.integers(-2, 3, size=B.codes.shape), -7, 7).astype(np.int32)
    for _ in range(4):
        inp = _inputs(rng, T, dk, dv, "scalar")
        O.step(A, *inp, want_o=False)
        O.step(B, *inp, want_o=False)
        assert np.array_equal(A.scales, B.scales)
    assert not np.array_equal(A.codes, B.codes)
    gmax = np.abs(A.shadow.astype(np.float64)).reshape(T, dv, 2, 32).max(axis=-1)
    assert np.allclose(A.scales, gmax / cfg.qmax, rtol=1e-6, atol=0)


def pin_high_bit_tracks_fp32():
    """With a 16-bit grid the quantized trajectory stays within ~1e-4 of the
    unquantized FP32 one: the quantized path is the same recurrence."""
    rng = _rng(25)
    T, dk, dv, H = 2, 64, 8, 20
    for decay in ("scalar", "diagonal"):
        for delta in (0, 1):
            for policy in ("dynamic", "yoked"):
                cfg = O.OracleConfig(T, dk, dv, 16, 32, delta, decay, policy)
                S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
                st = O.init(cfg, S0)
                S = S0.copy()
                for _ in range(H):
                    inp = _inputs(rng, T, dk, dv, decay)
                    oq = O.step(st, *inp)
                    o = O.fp32_step(cfg, S, *inp)
                    assert np.abs(oq - o).max() < 1e-3 * (1 + np.abs(o).max()), (decay, delta, policy)
                err = np.abs(st.dequantized() - S).max() / np.abs(S).max()
                assert err < 2e-4, (decay, delta, policy, err)


def pin_error_accumulation_bound():
    """Persistent scale, non-expansive steps (||k|| = 1, alpha <= 1,
    beta in (0, 1]): ||S^q_t - S_t||_F <= ||S^q_0 - S_0||_F + sum_tau ||eps_tau||_F
    where eps_tau is the rounding error of step tau (float64 closed-form
    check)."""
    rng = _rng(26)
    T, dk, dv, H = 2, 64, 8, 40
    for bits in (4, 8):
        for rounding in ("nearest", "bdr"):
            cfg = O.OracleConfig(T, dk, dv, bits, 32, 1, "scalar", "persistent", rounding)
            S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(F32)
            st = O.init(cfg, S0)
            S = S0.astype(np.float64)
            bound = np.linalg.norm((st.dequantized() - S).reshape(T, -1), axis=1)
            for _ in range(H):
                q, k, v, a, b = _inputs(rng, T, dk, dv, "scalar")
                x64, _, _ = _x64(st.copy(), q, k, v, a, b, cfg)
                O.step(st, q, k, v, a, b, want_o=False)
                eps = st.dequantized().astype(np.float64) - x64
                bound = bound + np.linalg.norm(eps.reshape(T, -1), axis=1)
                Sd = S * a.astype(np.float64)[:, None, None]
                k64 = k.astype(np.float64)
                w = b.astype(np.float64)[:, None] * (v - np.einsum("tij,tj->ti", Sd, k64))
                S = Sd + w[:, :, None] * k64[:, None, :]
                gap = np.linalg.norm((st.dequantized() - S).reshape(T, -1), axis=1)
                assert np.all(gap <= bound * (1 + 1e-4) + 1e-5), (bits, rounding)


# --------------------------------------------------------------------------
# Worked examples and layout / order fixtures
# --------------------------------------------------------------------------

def _dense(spec, n):
    out = np.zeros(n, F32)
    for key, val in spec.items():
        out[int(key)] = val
    return out


def pin_worked_steps():
    """The hand-worked steps of tests/golden/worked_steps.json."""
    with open(os.path.join(GOLDEN, "worked_steps.json")) as f:
        data = json.load(f)
    for case in data["cases"]:
        dk, dv = case["dk"], case["dv"]
        cfg = O.OracleConfig(1, dk, dv, case["bits"], case["group"], case["delta"],
                             case["decay"], case["policy"], case["rounding"])
        S0 = _dense(case["S0"], dk).reshape(1, 1, dk).repeat(dv, axis=1)
        st = O.init(cfg, S0)
        assert np.array_equal(st.codes[0, 0], _dense(case["init_codes"], dk).astype(np.int32)), case["name"]
        assert st.scales[0, 0, 0] == F32(case["init_scale"]), case["name"]
        alpha = np.full((1,), case["alpha"], F32) if case["decay"] == "scalar" else \
            np.full((1, dk), case["alpha"], F32)
        o = O.step(st, _dense(case["q"], dk)[None], _dense(case["k"], dk)[None],
                   np.array([case["v"]], F32), alpha, np.array([case["beta"]], F32))
        assert np.array_equal(st.codes[0, 0], _dense(case["codes"], dk).astype(np.int32)), case["name"]
        assert st.scales[0, 0, 0] == F32(case["scale"]), case["name"]
        assert np.array_equal(o[0], np.array(case["o"], F32)), case["name"]
        if "codes_nearest" in case:
            from dataclasses import replace
            c2 = replace(cfg, rounding="nearest")
            st2 = O.init(c2, S0)
            O.step(st2, _dense(case["q"], dk)[None], _dense(case["k"], dk)[None],
                   np.array([case["v"]], F32), alpha, np.array([case["beta"]], F32))
            assert np.array_equal(st2.codes[0, 0], _dense(case["codes_nearest"], dk).astype(np.int32))


def pin_pack_layout():
    with open(os.path.join(GOLDEN, "layout_and_order.json")) as f:
        data = json.load(f)
    for bits, key in ((4, "int4_pack"), (8, "int8_pack")):
        codes = np.array(data[key]["codes"], np.int32)
        packed = O.pack(bits, codes[None])[0]
        assert list(packed) == data[key]["bytes"]
        assert np.array_equal(O.unpack(bits, packed[None], codes.size)[0], codes)


def pin_dot_order():
    """The fixed dot-product order: eight interleaved chains within each
    32-column chunk, a fixed combine of the chains, pairwise tree over the
    chunks (worked examples in tests/golden/layout_and_order.json)."""
    with open(os.path.join(GOLDEN, "layout_and_order.json")) as f:
        data = json.load(f)
    for key in ("dot_order_chunks", "dot_order_combine", "dot_order_chain_sequence"):
        d = data[key]
        a = np.zeros(d["n"], F32)
        b = np.zeros(d["n"], F32)
        for idx, val in d["products"].items():
            a[int(idx)] = val
            b[int(idx)] = 1.0
        assert O.dot(a, b) == F32(d["expected"]), key
        # a left-to-right sum, where the fixture says so, gives another value
        acc = F32(0.0)
        for j in range(d["n"]):
            acc = F32(acc + F32(a[j] * b[j]))
        assert acc == F32(d["left_to_right"]), key
    # and within the error bound of the exact value on random data: every
    # product passes through at most 4 chain steps, 3 combine additions and
    # log2(n / 32) tree additions
    rng = _rng(27)
    for n in (32, 64, 128, 256):
        for _ in range(20):
            a = rng.standard_normal(n).astype(F32)
            b = rng.standard_normal(n).astype(F32)
            exact = float(np.dot(a.astype(np.float64), b.astype(np.float64)))
            bound = (4 + 3 + np.log2(n // 32) + 1) * 2.0 ** -24 * float(np.abs(a.astype(np.float64) * b).sum())
            assert abs(float(O.dot(a, b)) - exact) <= bound


def pin_sq_norms():
    """State norms (the quantity the dynamic-scale norm inflation is measured
    in): closed forms on constant and one-hot states, sign invariance, and
    agreement with the squared readouts against the unit vectors e_j (which
    return the dequantized columns exactly)."""
    T, dk, dv, G = 3, 64, 16, 32
    cfg = O.OracleConfig(T, dk, dv, 4, G, 1, "scalar", "persistent")
    codes = np.full((T, dv, dk), 3, np.int32)
    scales = np.full((T, dv, dk // G), 0.5, F32)
    st = O.State(cfg, codes, scales)
    assert np.array_equal(O.sq_norms(st), np.full(T, dv * dk * 2.25))
    codes = np.zeros((T, dv, dk), np.int32)
    codes[1, 5, 40] = -7
    scales = np.full((T, dv, dk // G), 0.25, F32)
    assert np.array_equal(O.sq_norms(O.State(cfg, codes, scales)), np.array([0.0, 3.0625, 0.0]))
    rng = _rng(31)
    codes = rng.integers(-7, 8, size=(T, dv, dk)).astype(np.int32)
    scales = rng.uniform(0.01, 2.0, size=(T, dv, dk // G)).astype(F32)
    st = O.State(cfg, codes, scales)
    n = O.sq_norms(st)
    assert np.array_equal(n, O.sq_norms(O.State(cfg, -codes, scales)))
    cols = np.zeros(T)
    for j in range(dk):
        e = np.zeros((T, dk), F32)
        e[:, j] = 1.0
        o = O.readout(st, e).astype(np.float64)
        cols += (o * o).sum(axis=1)
    assert np.allclose(n, cols, rtol=1e-12, atol=0.0)
    S = np.ones((T, dv, dk), F32)
    assert np.array_equal(O.fp32_sq_norms(cfg, S), np.full(T, float(dv * dk)))
    S = np.where(rng.integers(0, 2, size=(T, dv, dk)) == 1, F32(1.5), F32(-1.5)).astype(F32)
    assert np.array_equal(O.fp32_sq_norms(cfg, S), np.full(T, dv * dk * 2.25))


def pin_lrb_rank1_is_step():
    """Low-Rank Bypass with a period of one step merges at every step, so it
    must be the plain decode step bit for bit (codes, scales, shadow, o)."""
    rng = _rng(41)
    T, dk, dv = 4, 64, 16
    for policy in ("dynamic", "persistent", "yoked"):
        for rounding in ("nearest", "bdr"):
            for decay, delta in (("scalar", 1), ("diagonal", 0)):
                cfg = O.OracleConfig(T, dk, dv, 4, 32, delta, decay, policy, rounding)
                S0 = (rng.standard_normal((T, dv, dk)) * 0.4).astype(F32)
                a = O.init(cfg, S0)
                b = a.copy()
                buf = O.LrbBuffers(cfg, 1)
                for _ in range(4):
                    q, k, v, al, be = _inputs(rng, T, dk, dv, decay)
                    v = (v * 0.2).astype(F32)
                    oa = O.step(a, q, k, v, al, be)
                    ob = O.lrb_step(b, buf, q, k, v, al, be)
                    assert np.array_equal(oa, ob)
                    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales)
                    if a.shadow is not None:
                        assert np.array_equal(a.shadow, b.shadow)


def _lrb_effective(st, buf):
    """S' + sum_r U_r K_r^T of the LRB state, in float64 (stored codes times
    the accumulated decay, plus the buffered writes of the period)."""
    cfg = st.cfg
    d = st.codes.astype(np.float64) * np.repeat(st.scales.astype(np.float64), cfg.group, axis=-1)
    S = d * buf.A.astype(np.float64)[:, None, :]
    for r in range(buf.slot):
        S += np.einsum("ti,tj->tij", buf.U[:, :, r].astype(np.float64), buf.K[:, r].astype(np.float64))
    return S


def pin_lrb_bypass_tracks_fp32():
    """Between merges LRB quantizes nothing: the stored codes and scales stay
    fixed and the effective state (stored state with its accumulated decay
    plus the buffered rank-1 writes) follows the unquantized recurrence of
    LinQuant eq. (1) from the dequantized state, readouts included."""
    rng = _rng(42)
    T, dk, dv, R = 3, 64, 16, 6
    for decay, delta in (("scalar", 1), ("diagonal", 0), ("diagonal", 1)):
        cfg = O.OracleConfig(T, dk, dv, 8, 32, delta, decay, "dynamic", "nearest")
        st = O.init(cfg, (rng.standard_normal((T, dv, dk)) * 0.4).astype(F32))
        codes0, scales0 = st.codes.copy(), st.scales.copy()
        buf = O.LrbBuffers(cfg, R)
        ref = (st.codes.astype(np.float64) *
               np.repeat(st.scales.astype(np.float64), cfg.group, axis=-1))
        for _ in range(R - 1):
            q, k, v, al, be = _inputs(rng, T, dk, dv, decay)
            o = O.lrb_step(st, buf, q, k, v, al, be)
            a = _decay64(al, decay, dk)
            ref = ref * a[:, None, :]
            k64 = k.astype(np.float64)
            u = np.einsum("tij,tj->ti", ref, k64) if delta else 0.0
            w = be.astype(np.float64)[:, None] * (v.astype(np.float64) - u)
            ref = ref + np.einsum("ti,tj->tij", w, k64)
            o_ref = np.einsum("tij,tj->ti", ref, q.astype(np.float64))
            assert np.array_equal(st.codes, codes0) and np.array_equal(st.scales, scales0)
            eff = _lrb_effective(st, buf)
            scale = np.abs(ref).max()
            assert np.abs(eff - ref).max() <= 2e-6 * scale * (1 + buf.slot)
            assert np.abs(o - o_ref).max() <= 2e-5 * np.abs(o_ref).max() * (1 + buf.slot)


def pin_lrb_merge_closed_form():
    """With no decay, a linear write and a persistent scale, the merge at the
    end of a period requantizes the stored state plus the sum of the
    period's writes: codes = nearest(clamped) of (d + sum_t beta_t v_t k_t^T)/s,
    up to ties within FP32 rounding of a half step."""
    rng = _rng(43)
    T, dk, dv, R = 4, 64, 16, 5
    cfg = O.OracleConfig(T, dk, dv, 4, 32, 0, "scalar", "persistent", "nearest")
    st = O.init(cfg, (rng.standard_normal((T, dv, dk)) * 0.5).astype(F32))
    s_el = np.repeat(st.scales.astype(np.float64), 32, axis=-1)
    x = st.codes.astype(np.float64) * s_el
    buf = O.LrbBuffers(cfg, R)
    for _ in range(R):
        q, k, v, al, be = _inputs(rng, T, dk, dv, "scalar", alpha=1.0)
        v = (v * 0.1).astype(F32)
        O.lrb_step(st, buf, q, k, v, al, be)
        x += np.einsum("ti,tj->tij", be.astype(np.float64)[:, None] * v.astype(np.float64),
                       k.astype(np.float64))
    assert buf.slot == 0
    p = x / s_el
    want = np.clip(np.rint(p), -7, 7)
    near_tie = np.abs(np.abs(p - np.floor(p)) - 0.5) < 1e-4
    assert np.all((st.codes == want) | near_tie)
    assert np.count_nonzero(st.codes != want) <= np.count_nonzero(near_tie)


def pin_lrb_merge_bdr_follows_accumulated_update():
    """At a Low-Rank Bypass merge with rank > 1, BDR's direction is the sign
    of the period's accumulated update M = sum_r U_r K'_r^T + w k^T, not of the
    last write alone ("Preserving Updates...", abstract: the buffer merges
    before rounding, BDR acts at the rounding).  Checked element by element
    against the nearest-rounding merge of the same buffers, with M formed in
    float64 from the buffers; elements whose M is too close to 0 for its
    sign to be certain are skipped.  The case is built so that many
    reversed elements have sign(M) != sign(w k_j)."""
    rng = _rng(44)
    T, dk, dv, R, G = 16, 64, 16, 3, 32
    qmax = 7
    checked = differing = 0
    for period in range(3):
        cN = O.OracleConfig(T, dk, dv, 4, G, 0, "diagonal", "persistent", "nearest")
        cB = O.OracleConfig(T, dk, dv, 4, G, 0, "diagonal", "persistent", "bdr")
        stB = O.init(cB, (rng.standard_normal((T, dv, dk)) * 0.5).astype(F32))
        stN = O.State(cN, stB.codes.copy(), stB.scales.copy())
        bB, bN = O.LrbBuffers(cB, R), O.LrbBuffers(cN, R)
        for slot in range(R):
            q, k, v, a, b = _inputs(rng, T, dk, dv, "diagonal")
            v = (v * 0.05).astype(F32)
            if slot == R - 1:
                prev_codes, prev_scales = stB.codes.copy(), stB.scales.copy()
                a64 = a.astype(np.float64)
                M = np.einsum("tir,trj->tij", bB.U[:, :, :slot].astype(np.float64),
                              bB.K[:, :slot].astype(np.float64) * a64[:, None, :])
                w = (b[:, None] * v).astype(F32).astype(np.float64)
                M += w[:, :, None] * k.astype(np.float64)[:, None, :]
                lastsign = np.sign(w)[:, :, None] * np.sign(k)[:, None, :]
            O.lrb_step(stB, bB, q, k, v, a, b, want_o=False)
            O.lrb_step(stN, bN, q, k, v, a, b, want_o=False)
        s_el = np.repeat(prev_scales, G, axis=-1)
        d = (prev_codes.astype(F32) * s_el).astype(F32)
        n_near = stN.codes
        dq = (n_near.astype(F32) * s_el).astype(F32)
        mag = np.abs(M).max(axis=-1, keepdims=True)
        sure = np.abs(M) > 1e-5 * mag
        sigma = np.sign(M)
        rev = ((sigma > 0) & (dq < d)) | ((sigma < 0) & (dq > d))
        want = np.where(rev, np.clip(n_near + sigma.astype(np.int64), -qmax, qmax), n_near)
        assert np.array_equal(stB.codes[sure], want[sure])
        checked += int(sure.sum())
        differing += int((sure & rev & (sigma != lastsign)).sum())
    assert checked > 0 and differing > 0


def pin_lrb_preserves_small_writes():
    """The point of the bypass: a write of 0.3 code steps per step is rounded
    away by every per-step requantization (persistent scale, no decay), but
    survives when four of them accumulate in the buffer before one merge."""
    T, dk, dv, R = 2, 32, 4, 4
    cfg = O.OracleConfig(T, dk, dv, 8, 32, 0, "scalar", "persistent", "nearest")
    S0 = np.zeros((T, dv, dk), F32)
    S0[:, :, 0] = 127.0 / 64.0                      # scale 1/64 for every row
    plain = O.init(cfg, S0)
    lrb = plain.copy()
    buf = O.LrbBuffers(cfg, R)
    q = np.zeros((T, dk), F32)
    k = np.zeros((T, dk), F32)
    k[:, 5] = 1.0
    v = np.full((T, dv), 0.3 / 64.0, F32)           # 0.3 steps of the 1/64 grid
    one = np.ones(T, F32)
    for _ in range(R):
        O.step(plain, q, k, v, one, one, want_o=False)
        O.lrb_step(lrb, buf, q, k, v, one, one, want_o=False)
    assert np.all(plain.codes[:, :, 5] == 0)         # lost in rounding, every step
    assert np.all(lrb.codes[:, :, 5] == 1)           # 4 x 0.3 = 1.2 steps -> 1


ALL_PINS = [
    pin_linear_write_sum_of_outer_products,
    pin_decay_closed_form,
    pin_delta_rule_key_recall,
    pin_readout_is_state_times_q,
    pin_value_rescaling_exact,
    pin_key_rotation,
    pin_key_rescaling,
    pin_quantizer_error_bound,
    pin_dynamic_scale_reaches_qmax,
    pin_persistent_zero_update,
    pin_persistent_scales_fixed,
    pin_zero_scale_group,
    pin_bdr_bruteforce,
    pin_bdr_reversal_explained,
    pin_yoked_shadow_is_fp32_run,
    pin_yoked_scale_from_shadow_only,
    pin_high_bit_tracks_fp32,
    pin_error_accumulation_bound,
    pin_worked_steps,
    pin_pack_layout,
    pin_dot_order,
    pin_sq_norms,
    pin_lrb_rank1_is_step,
    pin_lrb_bypass_tracks_fp32,
    pin_lrb_merge_closed_form,
    pin_lrb_merge_bdr_follows_accumulated_update,
    pin_lrb_preserves_small_writes,
]
