"""The chunkwise regrouping that the prefill kernels implement, checked on
the CPU against the oracle's token-by-token FP32 recurrence.

Written here in float64 NumPy from the recurrence (no code shared with the
kernels or the oracle):
- linear write (delta = 0): per chunk, o_t = S (q_t e^{Lam_t}) +
  sum_{s <= t} (q_t . k_s e^{Lam_t - Lam_s}) beta_s v_s and
  S_new = S e^{Lam_C} + sum_s beta_s v_s (k_s e^{Lam_C - Lam_s})^T
  (LinQuant, Low-Precision Chunkwise Realization, with the decay per
  channel for diagonal decay);
- delta rule (delta = 1): the corrected values w_t = beta_t (v_t -
  S_{t-1} Lambda_t k_t) of a chunk solve (I + B) w = beta (v - S (k e^{Lam})),
  B_ts = beta_t (k_t . k_s e^{Lam_t - Lam_s}) for s < t, by forward
  substitution; then w replaces beta v in the linear write's formulas.
Agreement within 1e-5 of the magnitudes (the oracle runs in FP32; the
chunk form here in float64) pins the derivation itself, independently of
the GPU."""
import numpy as np
import pytest

from oracle import oracle as O


def chunk_form(S0, q, k, v, a, b, delta, decay, C, skip_solve=False):
    """Chunkwise prefill of one tile in float64: S0 [dv][dk]; q, k [L][dk];
    v [L][dv]; a [L] or [L][dk]; b [L].  Returns (S, o [L][dv]).
    skip_solve (a planted mistake) takes w = r without the substitution."""
    S = S0.astype(np.float64).copy()
    L = q.shape[0]
    dv = v.shape[1]
    o = np.zeros((L, dv))
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        qc, kc, vc, bc = (x[sl].astype(np.float64) for x in (q, k, v, b))
        ac = a[sl].astype(np.float64)
        lam = np.cumsum(np.log(ac), axis=0)            # [c] or [c][dk], inclusive
        if decay == "scalar":
            lam = np.repeat(lam[:, None], q.shape[1], axis=1)
        e_t = np.exp(lam)                               # e^{Lam_t} per channel
        n = qc.shape[0]
        # decay between s and t, per channel: e^{Lam_t - Lam_s}
        D = np.exp(lam[:, None, :] - lam[None, :, :])   # [t][s][dk]
        qk = np.einsum("tj,sj,tsj->ts", qc, kc, D)      # q_t . k_s e^{...}
        if delta:
            kk = np.einsum("tj,sj,tsj->ts", kc, kc, D)
            B = np.tril(bc[:, None] * kk, -1)
            r = bc[:, None] * (vc - (kc * e_t) @ S.T)   # beta_t (v_t - S (k_t e^{Lam_t}))
            w = np.zeros_like(r)
            for t in range(n):
                w[t] = r[t] if skip_solve else r[t] - B[t, :t] @ w[:t]
        else:
            w = bc[:, None] * vc
        A = np.tril(qk)
        o[sl] = (qc * e_t) @ S.T + A @ w
        kbar = kc * np.exp(lam[-1][None, :] - lam)      # k_s e^{Lam_C - Lam_s}
        S = S * np.exp(lam[-1])[None, :] + w.T @ kbar
    return S, o


@pytest.mark.parametrize("delta", [0, 1])
@pytest.mark.parametrize("decay", ["scalar", "diagonal"])
@pytest.mark.parametrize("L,C", [(75, 32), (64, 64), (1, 32)])
def test_chunk_form_matches_token_by_token(delta, decay, L, C):
    rng = np.random.default_rng(100 * delta + L + C + (decay == "diagonal"))
    T, dk, dv = 2, 32, 12
    f = lambda x: np.ascontiguousarray(x, dtype=np.float32)
    S0 = f(rng.standard_normal((T, dv, dk)) * 0.1)
    q = f(rng.standard_normal((T, L, dk)) / np.sqrt(dk))
    k = rng.standard_normal((T, L, dk))
    k = f(k / np.linalg.norm(k, axis=-1, keepdims=True))
    v = f(rng.standard_normal((T, L, dv)))
    a = f(rng.uniform(0.8, 1.0, size=(T, L, dk) if decay == "diagonal" else (T, L)))
    b = f(rng.uniform(0.05, 1.0, size=(T, L)))
    cfg = O.OracleConfig(T, dk, dv, 8, 32, delta, decay, "persistent")
    S = S0.copy()
    o_ref = np.empty((T, L, dv), np.float32)
    for t in range(L):
        o_ref[:, t] = O.fp32_step(cfg, S, q[:, t], k[:, t], v[:, t], a[:, t], b[:, t])
    for i in range(T):
        S_c, o_c = chunk_form(S0[i], q[i], k[i], v[i], a[i], b[i], delta, decay, C)
        sc = np.abs(S[i]).max()
        assert np.abs(S_c - S[i]).max() <= 1e-5 * sc, "state"
        oc = np.abs(o_ref[i]).max(axis=-1, keepdims=True)
        assert np.all(np.abs(o_c - o_ref[i]) <= 1e-5 * oc + 1e-30), "outputs"


def test_chunk_form_catches_a_wrong_solve():
    """The check has teeth: dropping the substitution (w = r) breaks the
    delta rule's agreement with the oracle by far more than the tolerance."""
    rng = np.random.default_rng(3)
    T, L, dk, dv = 1, 40, 32, 12
    f = lambda x: np.ascontiguousarray(x, dtype=np.float32)
    S0 = f(rng.standard_normal((T, dv, dk)) * 0.1)
    q = f(rng.standard_normal((T, L, dk)) / np.sqrt(dk))
    k = rng.standard_normal((T, L, dk))
    k = f(k / np.linalg.norm(k, axis=-1, keepdims=True))
    v = f(rng.standard_normal((T, L, dv)))
    a = f(rng.uniform(0.8, 1.0, size=(T, L)))
    b = f(rng.uniform(0.5, 1.0, size=(T, L)))
    cfg = O.OracleConfig(T, dk, dv, 8, 32, 1, "scalar", "persistent")
    S = S0.copy()
    for t in range(L):
        O.fp32_step(cfg, S, q[:, t], k[:, t], v[:, t], a[:, t], b[:, t], want_o=False)
    S_bad, _ = chunk_form(S0[0], q[0], k[0], v[0], a[0], b[0], 1, "scalar", 32, skip_solve=True)
    S_ok, _ = chunk_form(S0[0], q[0], k[0], v[0], a[0], b[0], 1, "scalar", 32)
    sc = np.abs(S[0]).max()
    assert np.abs(S_ok - S[0]).max() <= 1e-5 * sc
    assert np.abs(S_bad - S[0]).max() > 1e-3 * sc
