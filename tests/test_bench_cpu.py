"""Host-side checks of bench.py (no GPU).

The roofline fraction of every bench line divides by the algorithmic bytes
of one launch (bench.arm_bytes); those are pinned here against the per-launch
figures tabulated independently from the layouts (codes read and written,
scales, q, k, v, alpha, beta, o, and the yoked shadow), to three significant
digits.  The reference arm (the oracle timed on the host) is run once with
one step and its JSON line checked against the contract: the same metric,
unit and direction as the GPU arm, impl "reference", a cpu_baseline of kind
"oracle", and an e2e entry that moves no bytes across PCIe."""
import json
import os
import subprocess
import sys

import pytest

import bench
from ssm_decode_step_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (workload, arm) -> algorithmic bytes per launch, three significant digits
TABLE = {
    ("tiny-gdn", "int8-g64-persistent"): 38.0e3,
    ("gdn", "int4-g32-dynamic"): 23.1e6,
    ("gdn", "int4-g32-persistent"): 21.0e6,
    ("gdn", "int4-g32-yoked"): 157e6,
    ("mamba2", "int8-g64-persistent"): 302e6,
    ("gla", "int4-g32-persistent+bdr"): 86.0e6,
    ("gla", "int4-g32-dynamic+bdr"): 94.4e6,
    ("stack24", "int4-g32-persistent+bdr"): 252e6,
    ("stack24", "int8-g32-dynamic"): 478e6,
}


def test_every_bench_arm_is_tabulated():
    arms = {(n, a.name) for n in W.ORDER for a in W.get(n).arms}
    assert arms == set(TABLE)


@pytest.mark.parametrize("key", sorted(TABLE), ids=lambda k: f"{k[0]}:{k[1]}")
def test_arm_bytes_match_table(key):
    w = W.get(key[0])
    arm = next(a for a in w.arms if a.name == key[1])
    got = bench.arm_bytes(w, arm)
    assert abs(got - TABLE[key]) <= 0.005 * TABLE[key], (got, TABLE[key])


def test_prefill_bytes_grow_with_tokens():
    """Per token: q, k, v, alpha, beta read and o written; per tile: the
    state read and written once."""
    for dk, dv, diag in ((128, 64, False), (128, 128, True), (64, 64, False)):
        b0 = bench.prefill_bytes(dk, dv, 0, diag)
        assert b0 == 2 * dv * dk * 4
        per_token = bench.prefill_bytes(dk, dv, 1, diag) - b0
        assert per_token == 4 * (2 * dk + dv + (dk if diag else 1) + 1 + dv)
        assert bench.prefill_bytes(dk, dv, 300, diag) == b0 + 300 * per_token


def test_reference_arm_contract():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference"
    assert line["metric"].startswith("quantized-state decode steps/sec")
    assert line["unit"] == "steps/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["n_gpus"] == 1 and line["steps"] == 1
    assert line["scaling"] == "weak"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_prefill_flops_of_the_delta_rule():
    """The delta rule adds, per chunk of c tokens, the keys' projection on the
    state (2 c dk dv), their scores (c^2 dk) and the forward substitution
    (c^2 dv) to the linear write's count."""
    for dk, dv, L in ((128, 128, 256), (64, 48, 33), (128, 64, 1)):
        extra = sum(2 * c * dk * dv + c * c * (dk + dv)
                    for c in (min(32, L - c0) for c0 in range(0, L, 32)))
        assert bench.prefill_flops(dk, dv, L, delta=1) - bench.prefill_flops(dk, dv, L) == extra
    # one full chunk of the linear write, term by term
    assert bench.prefill_flops(128, 64, 32) == 4 * 32 * 128 * 64 + 32 * 32 * (128 + 64) + 128 * 64
