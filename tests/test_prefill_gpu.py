"""GPU checks of the chunkwise prefill (qstate_prefill, linear write and
delta rule, and its tensor-core form qstate_prefill_tf32, linear write)
against the oracle's token-by-token FP32 recurrence (qo_fp32_step per token).

The chunkwise form regroups the same sums, so the two agree to FP32 rounding
rather than bit for bit.  Tolerance: every state element within 1e-4 of the
tile's largest state magnitude and every output within 1e-4 of the token's
largest output magnitude (the delta rule too: its chunk solve is a forward
substitution with unit diagonal and off-diagonal terms beta_t e^{...} k_t.k_s
of magnitude at most one here, and the recurrence it reproduces contracts,
so errors do not grow from chunk to chunk).  Derivation: a reordered FP32 sum of n terms is
within about n * 2^-24 of the sum of their magnitudes; per chunk n is at most
dk + 32 = 160 (1e-5), cancellation makes the error relative to the largest
result a few times that, and the decay factors come from exp of running log
sums instead of running products (a few ulp times |log decay|).  Observed
worst case over these inputs: 2.6e-5 (the Mamba-2-shaped law, unnormalized
keys); the assertion message reports it.

The tensor-core form rounds every operand to TF32 (relative error 2^-11 per
operand, 2^-10 for the state, which the state read takes at TF32 precision
by dropping mantissa bits), so each product carries at most about 2^-10 +
2^-11 + 2^-11 = 2^-9 of its magnitude, and the FP32 accumulation adds
n * 2^-24 (n <= 192).  Errors of the state carry into later chunks with the
decay and stay relative to the magnitudes.  Bound checked: every element
within 2^-8 of the same recurrence run on |S0|, |q|, |k|, |v| (the sum of
the magnitudes of its terms), twice the estimate."""
import numpy as np
import pytest

from oracle import oracle as O
from ssm_decode_step_b200 import Config, workloads as W

pytestmark = pytest.mark.gpu

TOL = 1e-4
TOL_TF32 = 2.0 ** -8

# (dk, dv, decay, tiles, length, with_o)
CASES = [
    (128, 64, "scalar", 13, 100, True),
    (128, 128, "diagonal", 7, 77, True),
    (64, 48, "scalar", 5, 32, True),
    (64, 16, "diagonal", 3, 1, True),
    (128, 32, "diagonal", 4, 33, False),
    (64, 64, "scalar", 2, 257, True),
]


def _id(c):
    dk, dv, dc, T, L, wo = c
    return f"dk{dk}-dv{dv}-{dc}-T{T}-L{L}{'' if wo else '-no-o'}"


def _inputs(rng, T, L, dk, dv, decay):
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)
    q = f(rng.standard_normal((T, L, dk)) / np.sqrt(dk))
    k = f(rng.standard_normal((T, L, dk)) / np.sqrt(dk))
    v = f(rng.standard_normal((T, L, dv)))
    a = f(rng.uniform(0.8, 1.0, size=(T, L, dk) if decay == "diagonal" else (T, L)))
    b = f(rng.uniform(0.0, 1.0, size=(T, L)))
    return q, k, v, a, b


def _reference(T, dk, dv, decay, S0, q, k, v, a, b, delta=0):
    cfg = O.OracleConfig(T, dk, dv, 8, 32, delta, decay, "persistent")
    S = S0.copy()
    o = np.empty((T, q.shape[1], dv), np.float32)
    for t in range(q.shape[1]):
        o[:, t] = O.fp32_step(cfg, S, q[:, t], k[:, t], v[:, t], a[:, t], b[:, t])
    return S, o


def _check(S_gpu, S_ref, o_gpu, o_ref):
    sc = np.abs(S_ref).max(axis=(1, 2), keepdims=True)
    err = np.abs(S_gpu - S_ref) / np.maximum(sc, 1e-30)
    assert err.max() <= TOL, f"state: worst relative error {err.max():.3g}"
    if o_gpu is not None:
        oc = np.abs(o_ref).max(axis=-1, keepdims=True)
        err = np.abs(o_gpu - o_ref) / np.maximum(oc, 1e-30)
        assert err.max() <= TOL, f"outputs: worst relative error {err.max():.3g}"


@pytest.mark.parametrize("case", CASES, ids=_id)
def test_prefill_matches_token_by_token(case):
    import torch
    from ssm_decode_step_b200 import qstate as Q
    dk, dv, decay, T, L, with_o = case
    rng = np.random.default_rng(dk + dv + T + L)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.1).astype(np.float32)
    q, k, v, a, b = _inputs(rng, T, L, dk, dv, decay)
    S_ref, o_ref = _reference(T, dk, dv, decay, S0, q, k, v, a, b)
    cfg = Config(T, dk, dv, 8, 32, 0, decay)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    o = torch.empty((T, L, dv), dtype=torch.float32, device="cuda") if with_o else None
    Q.prefill(cfg, L, S, dev(q), dev(k), dev(v), dev(a), dev(b), o)
    _check(S.cpu().numpy(), S_ref, None if o is None else o.cpu().numpy(), o_ref)


@pytest.mark.parametrize("wname", ["mamba2", "gla"])
def test_prefill_on_workload_laws(wname):
    """The Mamba-2- and GLA-shaped input laws (64 tiles, 256 tokens from a
    zero state): the state the decode path would start from."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    w = W.scaled_down(W.get(wname), 64)
    T, L = w.tiles, 256
    slots = [W.slot(w, t) for t in range(L)]
    q, k, v, a, b = (np.ascontiguousarray(np.stack([s[i] for s in slots], axis=1)) for i in range(5))
    S0 = np.zeros((T, w.dv, w.dk), np.float32)
    S_ref, o_ref = _reference(T, w.dk, w.dv, w.decay, S0, q, k, v, a, b)
    cfg = Config(T, w.dk, w.dv, 8, 32, 0, w.decay)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    o = torch.empty((T, L, w.dv), dtype=torch.float32, device="cuda")
    Q.prefill(cfg, L, S, dev(q), dev(k), dev(v), dev(a), dev(b), o)
    _check(S.cpu().numpy(), S_ref, o.cpu().numpy(), o_ref)


# (dk, dv, decay, tiles, length, with_o) for the delta rule
DELTA_CASES = [
    (128, 128, "scalar", 9, 100, True),
    (128, 64, "diagonal", 5, 77, True),
    (64, 48, "scalar", 4, 33, True),
    (64, 16, "diagonal", 3, 1, True),
    (128, 32, "scalar", 3, 64, False),
    (64, 64, "diagonal", 2, 257, True),
    (128, 128, "diagonal", 3, 70, True),   # the largest shared-memory configuration (212.6 KB)
]


@pytest.mark.parametrize("case", DELTA_CASES, ids=_id)
def test_prefill_delta_rule_matches_token_by_token(case):
    import torch
    from ssm_decode_step_b200 import qstate as Q
    dk, dv, decay, T, L, with_o = case
    rng = np.random.default_rng(3 * dk + dv + T + L)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.1).astype(np.float32)
    q, k, v, a, b = _inputs(rng, T, L, dk, dv, decay)
    S_ref, o_ref = _reference(T, dk, dv, decay, S0, q, k, v, a, b, delta=1)
    cfg = Config(T, dk, dv, 8, 32, 1, decay)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    o = torch.empty((T, L, dv), dtype=torch.float32, device="cuda") if with_o else None
    Q.prefill(cfg, L, S, dev(q), dev(k), dev(v), dev(a), dev(b), o)
    _check(S.cpu().numpy(), S_ref, None if o is None else o.cpu().numpy(), o_ref)


def test_prefill_delta_rule_on_gated_deltanet_laws():
    """The Gated DeltaNet-shaped law (unit-norm keys, alpha = sigmoid(N(3,1)),
    beta = sigmoid(N(0,1)); 64 tiles, 256 tokens from a zero state): the S_0
    its quantized decode starts from, prefilled instead of warmed up token by
    token."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    w = W.scaled_down(W.get("gdn"), 64)
    assert w.delta == 1
    T, L = w.tiles, 256
    slots = [W.slot(w, t) for t in range(L)]
    q, k, v, a, b = (np.ascontiguousarray(np.stack([s[i] for s in slots], axis=1)) for i in range(5))
    S0 = np.zeros((T, w.dv, w.dk), np.float32)
    S_ref, o_ref = _reference(T, w.dk, w.dv, w.decay, S0, q, k, v, a, b, delta=1)
    cfg = Config(T, w.dk, w.dv, 8, 32, 1, w.decay)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    o = torch.empty((T, L, w.dv), dtype=torch.float32, device="cuda")
    Q.prefill(cfg, L, S, dev(q), dev(k), dev(v), dev(a), dev(b), o)
    _check(S.cpu().numpy(), S_ref, o.cpu().numpy(), o_ref)


TF32_CASES = [
    (128, 64, "scalar", 13, 100, True),
    (128, 128, "diagonal", 7, 77, True),
    (64, 48, "scalar", 5, 32, True),
    (64, 16, "diagonal", 3, 1, True),
    (128, 32, "diagonal", 4, 33, False),
    (64, 64, "scalar", 2, 257, True),
    (128, 112, "scalar", 3, 64, True),
    (64, 128, "diagonal", 2, 65, True),
    (128, 128, "scalar", 300, 130, True),
    (64, 64, "scalar", 4, 1000, True),
    (128, 64, "diagonal", 3, 300, True),
]


def _check_bound(name, gpu, ref, mag):
    err = np.abs(gpu.astype(np.float64) - ref)
    bound = TOL_TF32 * mag.astype(np.float64) + 1e-30
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{name}: worst error / bound {worst:.3g} (bound 2^-8 of magnitudes)"
    return worst


@pytest.mark.parametrize("case", TF32_CASES, ids=_id)
def test_prefill_tf32_within_bound(case):
    import torch
    from ssm_decode_step_b200 import qstate as Q
    dk, dv, decay, T, L, with_o = case
    rng = np.random.default_rng(7 * dk + dv + T + L)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.1).astype(np.float32)
    q, k, v, a, b = _inputs(rng, T, L, dk, dv, decay)
    S_ref, o_ref = _reference(T, dk, dv, decay, S0, q, k, v, a, b)
    S_mag, o_mag = _reference(T, dk, dv, decay, np.abs(S0), np.abs(q), np.abs(k), np.abs(v), a, b)
    cfg = Config(T, dk, dv, 8, 32, 0, decay)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    o = torch.empty((T, L, dv), dtype=torch.float32, device="cuda") if with_o else None
    before = Q.prefill_tf32_timeouts()
    Q.prefill_tf32(cfg, L, S, dev(q), dev(k), dev(v), dev(a), dev(b), o)
    torch.cuda.synchronize()
    assert Q.prefill_tf32_timeouts() == before
    _check_bound("state", S.cpu().numpy(), S_ref, S_mag)
    if with_o:
        _check_bound("outputs", o.cpu().numpy(), o_ref, o_mag)


@pytest.mark.parametrize("wname", ["mamba2", "gla"])
def test_prefill_tf32_on_workload_laws(wname):
    """The Mamba-2- and GLA-shaped laws (64 tiles, 256 tokens from a zero
    state), the tensor-core form against the same bound."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    w = W.scaled_down(W.get(wname), 64)
    T, L = w.tiles, 256
    slots = [W.slot(w, t) for t in range(L)]
    q, k, v, a, b = (np.ascontiguousarray(np.stack([s[i] for s in slots], axis=1)) for i in range(5))
    S0 = np.zeros((T, w.dv, w.dk), np.float32)
    S_ref, o_ref = _reference(T, w.dk, w.dv, w.decay, S0, q, k, v, a, b)
    S_mag, o_mag = _reference(T, w.dk, w.dv, w.decay, S0, np.abs(q), np.abs(k), np.abs(v), a, b)
    cfg = Config(T, w.dk, w.dv, 8, 32, 0, w.decay)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    o = torch.empty((T, L, w.dv), dtype=torch.float32, device="cuda")
    Q.prefill_tf32(cfg, L, S, dev(q), dev(k), dev(v), dev(a), dev(b), o)
    torch.cuda.synchronize()
    _check_bound("state", S.cpu().numpy(), S_ref, S_mag)
    _check_bound("outputs", o.cpu().numpy(), o_ref, o_mag)


@pytest.mark.parametrize("wname", ["mamba2", "gla"])
def test_prompt_then_quantized_state(wname):
    """The path a prompt takes into decode: the tensor-core prefill leaves S,
    qstate_init quantizes it (dynamic rule, nearest) and qstate_readout reads
    it, against the oracle's token-by-token FP32 state S_ref.  Bound, element
    by element: |c s - S_ref| <= s/2 (rounding at the group's scale s, which
    the dynamic rule keeps in range) + 2^-8 * S_mag (the prefill's bound), and
    for the readout the same terms times |q_j| summed over j, plus the FP32
    rounding of that sum."""
    import torch
    from ssm_decode_step_b200 import QState, qstate as Q
    w = W.scaled_down(W.get(wname), 32)
    T, L = w.tiles, 200
    slots = [W.slot(w, t) for t in range(L)]
    q, k, v, a, b = (np.ascontiguousarray(np.stack([s[i] for s in slots], axis=1)) for i in range(5))
    S0 = np.zeros((T, w.dv, w.dk), np.float32)
    S_ref, _ = _reference(T, w.dk, w.dv, w.decay, S0, q, k, v, a, b)
    S_mag, _ = _reference(T, w.dk, w.dv, w.decay, S0, np.abs(q), np.abs(k), np.abs(v), a, b)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    Q.prefill_tf32(Config(T, w.dk, w.dv, 8, 32, 0, w.decay), L, S, dev(q), dev(k), dev(v), dev(a), dev(b))
    cfg = Config(T, w.dk, w.dv, 8, 32, 0, w.decay, "dynamic")
    st = QState(cfg).init(S)
    qr = np.random.default_rng(17).standard_normal((T, w.dk)).astype(np.float32)
    o = torch.empty((T, w.dv), dtype=torch.float32, device="cuda")
    st.readout(dev(qr), o)
    torch.cuda.synchronize()
    codes = st.codes.cpu().numpy().view(np.int8).astype(np.float32)   # INT8: one code per element
    scales = st.scales.cpu().numpy()                                     # [T][dv][dk/32]
    s_el = np.repeat(scales, 32, axis=2)
    deq = codes * s_el
    bound = 0.5 * s_el * (1 + 2.0 ** -20) + TOL_TF32 * S_mag + 1e-30
    err = np.abs(deq.astype(np.float64) - S_ref)
    assert (err <= bound).all(), f"dequantized state off by {float((err / bound).max()):.3g} x its bound"
    o_ref = np.einsum("tij,tj->ti", S_ref.astype(np.float64), qr.astype(np.float64))
    # plus the FP32 rounding of the readout's own sum (at most Dk * 2^-24 of
    # the sum of magnitudes, taken as 2^-16)
    o_bound = (np.einsum("tij,tj->ti", bound, np.abs(qr).astype(np.float64))
               + 2.0 ** -16 * np.einsum("tij,tj->ti", np.abs(deq).astype(np.float64), np.abs(qr).astype(np.float64)))
    o_err = np.abs(o.cpu().numpy().astype(np.float64) - o_ref)
    assert (o_err <= o_bound).all(), f"readout off by {float((o_err / o_bound).max()):.3g} x its bound"


def test_bounded_wait_gives_up_and_leaves_the_context_usable():
    """The tensor-core prefill's waits are bounded: a CTA launched so that its
    first wait cannot complete (nothing committed) gives up after the poll
    limit, counts one timeout, frees its tensor memory and returns; the next
    prefill on the same context runs normally and counts none."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    before = Q.prefill_tf32_timeouts()
    assert Q.prefill_tf32_wait_selfcheck(1000) == 1
    assert Q.prefill_tf32_timeouts() == before + 1
    dk, dv, decay, T, L = 128, 64, "scalar", 3, 70
    rng = np.random.default_rng(23)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.1).astype(np.float32)
    q, k, v, a, b = _inputs(rng, T, L, dk, dv, decay)
    S_ref, o_ref = _reference(T, dk, dv, decay, S0, q, k, v, a, b)
    S_mag, o_mag = _reference(T, dk, dv, decay, np.abs(S0), np.abs(q), np.abs(k), np.abs(v), a, b)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    S = dev(S0)
    o = torch.empty((T, L, dv), dtype=torch.float32, device="cuda")
    Q.prefill_tf32(Config(T, dk, dv, 8, 32, 0, decay), L, S, dev(q), dev(k), dev(v), dev(a), dev(b), o)
    torch.cuda.synchronize()
    assert Q.prefill_tf32_timeouts() == before + 1
    _check_bound("state", S.cpu().numpy(), S_ref, S_mag)
    _check_bound("outputs", o.cpu().numpy(), o_ref, o_mag)
