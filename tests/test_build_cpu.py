"""Register use of the built kernels, from ptxas's resource report of the
last build (no GPU needed).

The decode-step kernels the benchmark times for its workloads (the
streamed kernel for dynamic and persistent scales, the ring kernel for the
yoked one) must not spill; a few rarely used combinations at the register
cap (yoked or Low-Rank Bypass merges with Bounded Directional Rounding at
168 registers, four tensor-core prefill instances at 128) spill a few bytes
to local memory, and no kernel may spill more than 64 bytes."""
import re

from ssm_decode_step_b200 import build as B

# the ring kernel (yoked policy) and the streamed kernel (dynamic, persistent)
STEP = re.compile(r"_ZN2qs(?:11step_kernel|18stream_step_kernel)ILi(\d)ELi(\d+)ELi(\d)ELb(\d)ELb(\d)ELb(\d)E")


def _step_key(name):
    m = STEP.match(name)
    return None if m is None else tuple(int(x) for x in m.groups())


def _bench_arms():
    """(bits, dk, policy, bdr, delta, diag) of every arm the benchmark's workloads time."""
    from ssm_decode_step_b200 import workloads as W
    pol = {"dynamic": 0, "persistent": 1, "yoked": 2}
    out = set()
    for name in W.ORDER:
        w = W.get(name)
        for a in w.arms:
            out.add((a.bits, w.dk, pol[a.policy], int(a.rounding == "bdr"), w.delta,
                     int(w.decay == "diagonal")))
    return out


def test_benchmarked_kernels_do_not_spill():
    rep = B.ptxas_report()
    assert rep, "empty ptxas report"
    arms = _bench_arms()
    seen = set()
    for name, r in rep.items():
        key = _step_key(name)
        if key in arms:
            seen.add(key)
            assert r.get("spill_stores", 0) == 0 and r.get("spill_loads", 0) == 0, (name, r)
    assert seen == arms
    # the FP32 prefill (every instance) and the Mamba-2-shaped tensor-core prefill
    for name, r in rep.items():
        if name.startswith("_ZN2qs14prefill_kernel") or name.startswith("_ZN2qs17prefill_tc_kernelILi128ELi64ELb0E"):
            assert r.get("spill_stores", 0) == 0, (name, r)


def test_no_kernel_spills_more_than_a_few_bytes():
    for name, r in B.ptxas_report().items():
        assert r.get("spill_stores", 0) <= 64 and r.get("spill_loads", 0) <= 64, (name, r)
