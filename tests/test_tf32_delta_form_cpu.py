"""Precision of the delta rule's chunk form with TF32 operands, emulated in
NumPy: the numerical check behind the planned tensor-core delta-rule
prefill, taken before that kernel is built.

Every operand a tensor-core contraction would take is rounded to TF32 (10
explicit mantissa bits, nearest, ties away from zero, as cvt.rna.tf32.f32);
products of TF32 values are exact in FP32 and are accumulated in FP32; the
chunk's inverse T = (I + B)^{-1} is formed in FP32 by forward substitution
and rounded to TF32 for its contraction W = T (beta (v - S k e^{Lam})).
The state is held pre-scaled by e^{Lam_m} as in the linear write's
tensor-core path.  Against the float64 chunk form (which
tests/test_chunk_form_cpu.py pins to the oracle's token-by-token
recurrence), on Gated DeltaNet-shaped sequences (unit-norm keys, alpha =
sigmoid(N(3,1)), beta = sigmoid(N(0,1)), 256 tokens, chunks of 64, Dk = Dv
= 128), the state must stay within 2^-8 of max|S| and every output within
2^-8 of max|o_t| (observed about 2^-10.5 and 2^-9.5)."""
import numpy as np
import pytest


def tf32(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000
    return b.astype(np.uint32).view(np.float32)


def mm32(a, b):
    return (a.astype(np.float32) @ b.astype(np.float32)).astype(np.float32)


def chunk_delta(S0, q, k, v, a, b, C, emulate_tf32):
    """Chunkwise delta rule, scalar decay; float64 when emulate_tf32 is False."""
    S = S0.astype(np.float32 if emulate_tf32 else np.float64).copy()
    L = q.shape[0]
    o = np.zeros((L, v.shape[1]))
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        qc, kc, vc, bc = q[sl], k[sl], v[sl], b[sl]
        lam = np.cumsum(np.log(a[sl].astype(np.float64)))
        n = len(lam)
        if not emulate_tf32:
            D = np.exp(lam[:, None] - lam[None, :])
            B = np.tril(bc[:, None] * (kc @ kc.T) * D, -1)
            r = bc[:, None] * (vc - (kc * np.exp(lam)[:, None]) @ S.T)
            w = np.zeros_like(r)
            for t in range(n):
                w[t] = r[t] - B[t, :t] @ w[:t]
            o[sl] = (qc * np.exp(lam)[:, None]) @ S.T + np.tril((qc @ kc.T) * D) @ w
            S = S * np.exp(lam[-1]) + w.T @ (kc * np.exp(lam[-1] - lam)[:, None])
            continue
        m = (n - 1) // 2
        fq = np.exp(lam - lam[m]).astype(np.float32)
        fk = np.exp(lam[m] - lam).astype(np.float32)
        P = (S * np.float32(np.exp(lam[m]))).astype(np.float32)
        Qs, Ks, Kq = tf32(qc * fq[:, None]), tf32(kc * fk[:, None]), tf32(kc * fq[:, None])
        Bm = np.tril(bc[:, None].astype(np.float32) * mm32(Kq, Ks.T), -1)
        R = mm32(tf32(P), Kq.T).T                       # S (k_t e^{Lam_t}), [t][i]
        X = (bc[:, None] * (vc - R)).astype(np.float32)
        T = np.eye(n, dtype=np.float32)
        for t in range(n):
            T[t, :t] = -(Bm[t, :t] @ T[:t, :t]).astype(np.float32)
        W = mm32(tf32(T), tf32(X))
        o[sl] = mm32(tf32(P), Qs.T).T + mm32(tf32(np.tril(mm32(Qs, Ks.T))), tf32(W))
        P = P + mm32(tf32(W).T, Ks)
        S = (P * np.float32(np.exp(lam[-1] - lam[m]))).astype(np.float32)
    return S, o


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_tf32_delta_chunk_form_within_bound(seed):
    rng = np.random.default_rng(seed)
    L, dk, dv, C = 256, 128, 128, 64
    q = rng.standard_normal((L, dk)).astype(np.float32)
    k = rng.standard_normal((L, dk))
    k = (k / np.linalg.norm(k, axis=1, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((L, dv)).astype(np.float32)
    a = (1 / (1 + np.exp(-rng.normal(3, 1, L)))).astype(np.float32)
    b = (1 / (1 + np.exp(-rng.normal(0, 1, L)))).astype(np.float32)
    S0 = np.zeros((dv, dk), np.float32)
    Se, oe = chunk_delta(S0, q, k, v, a, b, C, False)
    St, ot = chunk_delta(S0, q, k, v, a, b, C, True)
    assert np.abs(St - Se).max() <= 2.0 ** -8 * np.abs(Se).max()
    assert np.all(np.abs(ot - oe).max(axis=1) <= 2.0 ** -8 * np.abs(oe).max(axis=1))


def test_tf32_rounding_helper():
    """tf32 keeps 10 explicit mantissa bits, rounds to nearest, ties away."""
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -10)
    assert tf32(one + ulp)[()] == one + ulp
    assert tf32(one + ulp / 2)[()] == one + ulp          # tie: away from zero
    assert tf32(one + ulp / 4)[()] == one
    assert tf32(-(one + ulp / 2))[()] == -(one + ulp)
