"""qstate_decode_step_host_static: the decode step for callers that may not
allocate device memory themselves (an engine whose memory manager owns the
device budget, a serving loop that cannot take cudaMalloc's device-wide
synchronization).  It stages each step through the library's static device
array instead of allocating, and must leave exactly the state and readouts
of the same step issued through qstate_decode_step with device buffers.

Checked on two calls in a row on the same state (the second call reuses the
array the first one left behind), through the C ABI binding, against the
existing entry point within the parity tolerances (codes and scales bit for
bit, readouts within 1e-4 of the tile's largest).  This file is collected
last, so that a run which stops at the first failure has run every other
test before it."""
import numpy as np
import pytest

from tests import parity as PR

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _packed(step):
    q, k, v, a, b = step
    flat = np.concatenate([x.reshape(-1) for x in (q, k, v, a, b)]).astype(np.float32)
    return torch.from_numpy(flat).pin_memory()


@pytest.mark.parametrize("case", [(150, 128, 64, 4, 32, 1, "scalar", "dynamic", "nearest"),
                                  (37, 128, 128, 4, 32, 0, "diagonal", "persistent", "bdr"),
                                  (21, 64, 48, 8, 64, 1, "scalar", "yoked", "nearest")],
                         ids=lambda c: f"T{c[0]}-dk{c[1]}-int{c[3]}-{c[7]}-{c[8]}")
def test_static_stage_step_matches_decode_step(case):
    from ssm_decode_step_b200 import Config, QState, qstate as Q
    T, dk, dv, bits, group, delta, decay, policy, rounding = case
    cfg = Config(T, dk, dv, bits, group, delta, decay, policy, rounding)
    dev = torch.device("cuda")
    rng = np.random.default_rng(T * 7 + dk + bits)
    S0 = (rng.standard_normal((T, dv, dk)) * 0.3).astype(np.float32)
    steps = PR.random_steps(rng, T, dk, dv, decay, 2, scale=0.5)
    S0d = torch.from_numpy(S0).to(dev)
    staged = QState(cfg, dev).init(S0d)
    direct = QState(cfg, dev).init(S0d)
    stream = torch.cuda.current_stream()
    in_bytes, out_bytes = Q.pipeline_query_sizes(cfg, 1)
    for t, step in enumerate(steps):
        host_in = _packed(step)
        assert host_in.numel() * 4 == in_bytes
        host_out = torch.full((T, dv), float("nan")).pin_memory()
        assert host_out.numel() * 4 == out_bytes
        Q.decode_step_host_static(cfg, staged.codes, staged.scales, staged.shadow, host_in, host_out,
                                  stream)
        q, k, v, a, b = (torch.from_numpy(x).to(dev) for x in step)
        o = torch.empty((T, dv), dtype=torch.float32, device=dev)
        direct.step(q, k, v, a, b, o)
        torch.cuda.synchronize()
        assert torch.equal(staged.codes, direct.codes), f"codes differ after call {t}"
        assert torch.equal(staged.scales, direct.scales), f"scales differ after call {t}"
        if staged.shadow is not None:
            assert torch.equal(staged.shadow, direct.shadow), f"shadow differs after call {t}"
        PR.compare_readout(host_out.numpy(), o.cpu().numpy(), f"static staging, call {t}")


def test_static_stage_rejects_steps_beyond_its_size():
    """A step whose inputs and readouts exceed the static array is refused
    before anything is enqueued; without readouts the same step may fit."""
    from ssm_decode_step_b200 import Config, QState, qstate as Q
    dev = torch.device("cuda")
    # 65536 tiles of Dk = Dv = 64: 50.3 MB of inputs, more than 32 MiB
    cfg = Config(65536, 64, 64, 4, 32, 1, "scalar", "dynamic", "nearest")
    in_bytes, out_bytes = Q.pipeline_query_sizes(cfg, 1)
    assert in_bytes > (32 << 20)
    st = QState(cfg, dev)
    host_in = torch.zeros(in_bytes // 4).pin_memory()
    with pytest.raises(Q.QStateError) as e:
        Q.decode_step_host_static(cfg, st.codes, st.scales, st.shadow, host_in, None)
    assert e.value.status == Q.QS_ERR_UNSUPPORTED
    torch.cuda.synchronize()
