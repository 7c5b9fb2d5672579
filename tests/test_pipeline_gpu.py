"""Host-buffer decode pipeline (qstate_pipeline_*): steps whose inputs come
from page-locked host memory and whose readouts go back there must leave
exactly the states and readouts of the same steps issued directly with
device buffers (the same kernels run on the same values), and its readouts
must agree with the oracle's.  Buffers wrap (more steps than the pipeline's
depth), families differ in bits, group, policy and rounding, and a step may
skip its readouts."""
import numpy as np
import pytest

from oracle import oracle as O
from tests import parity as PR

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _families(T, dv, decay):
    from ssm_decode_step_b200 import Config
    return [Config(T, 128, dv, 4, 32, 1, decay, "dynamic", "nearest"),
            Config(T, 128, dv, 8, 64, 1, decay, "persistent", "bdr"),
            Config(T, 128, dv, 4, 32, 1, decay, "yoked", "nearest")]


def _packed(step):
    q, k, v, a, b = step
    flat = np.concatenate([x.reshape(-1) for x in (q, k, v, a, b)]).astype(np.float32)
    return torch.from_numpy(flat).pin_memory()


@pytest.mark.parametrize("decay,depth,T", [("diagonal", 3, 37), ("scalar", 2, 150)])
def test_pipeline_matches_direct_steps(decay, depth, T):
    from ssm_decode_step_b200 import HostPipeline, QState
    dev = torch.device("cuda")
    dv = 64
    cfgs = _families(T, dv, decay)
    rng = np.random.default_rng(11)
    S0 = rng.standard_normal((T, dv, 128)).astype(np.float32)
    steps = PR.random_steps(rng, T, 128, dv, decay, 7)
    S0d = torch.from_numpy(S0).to(dev)
    piped = [QState(c, dev).init(S0d) for c in cfgs]
    direct = [QState(c, dev).init(S0d) for c in cfgs]
    torch.cuda.synchronize()

    pl = HostPipeline(piped, depth=depth)
    host_in = [_packed(s) for s in steps]
    host_out = [torch.full((len(cfgs), T, dv), float("nan")).pin_memory() for _ in steps]
    assert host_in[0].numel() * 4 == pl.in_bytes and host_out[0].numel() * 4 == pl.out_bytes
    stream = torch.cuda.current_stream()
    for t in range(len(steps)):
        # step 4 skips its readouts: the states must advance all the same
        pl.step(host_in[t], None if t == 4 else host_out[t], stream)
    pl.sync()

    # the same steps issued directly, with device buffers
    ora = [O.init(PR.oracle_cfg(c), S0) for c in cfgs]
    for t, (q, k, v, a, b) in enumerate(steps):
        dq, dk_, dv_, da, db = (torch.from_numpy(x).to(dev) for x in (q, k, v, a, b))
        for i, st in enumerate(direct):
            o = torch.empty((T, dv), dtype=torch.float32, device=dev)
            st.step(dq, dk_, dv_, da, db, o)
            o_ref = O.step(ora[i], q, k, v, a, b)
            if t == 4:
                assert torch.isnan(host_out[t][i]).all(), "a step without readouts wrote some"
                continue
            got = host_out[t][i].numpy()
            assert np.array_equal(got, o.cpu().numpy()), f"family {i} step {t}: readout differs"
            PR.compare_readout(got, o_ref, f"pipeline family {i} step {t}")
    for i, (a_, b_) in enumerate(zip(piped, direct)):
        assert torch.equal(a_.codes, b_.codes), f"family {i}: codes differ"
        assert torch.equal(a_.scales, b_.scales), f"family {i}: scales differ"
        if a_.shadow is not None:
            assert torch.equal(a_.shadow, b_.shadow), f"family {i}: shadow differs"
    pl.close()


def test_pipeline_join_orders_the_copies_before_the_stream():
    """An event recorded on a stream after join() completes only once every
    readout has reached host memory; wait_stream() orders the first input
    copy after an event recorded before it."""
    from ssm_decode_step_b200 import HostPipeline, QState
    dev = torch.device("cuda")
    T, dv = 64, 128
    cfgs = _families(T, dv, "scalar")
    rng = np.random.default_rng(5)
    S0 = torch.from_numpy(rng.standard_normal((T, dv, 128)).astype(np.float32)).to(dev)
    states = [QState(c, dev).init(S0) for c in cfgs]
    steps = PR.random_steps(rng, T, 128, dv, "scalar", 5)
    host_in = [_packed(s) for s in steps]
    host_out = [torch.full((len(cfgs), T, dv), float("nan")).pin_memory() for _ in steps]
    stream = torch.cuda.Stream()
    pl = HostPipeline(states, depth=2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    pl.wait_stream(stream)
    for t in range(len(steps)):
        pl.step(host_in[t], host_out[t], stream)
    pl.join(stream)
    e1.record(stream)
    e1.synchronize()
    for t in range(len(steps)):
        assert not torch.isnan(host_out[t]).any(), f"step {t}: readouts not in host memory at the event"
    assert e0.elapsed_time(e1) > 0
    pl.close()
