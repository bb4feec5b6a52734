"""Times the fp64 oracle on every named workload on the host cores (a
reported CPU baseline, not a test of correctness).  Minutes of CPU work, so it
runs only when asked: ORACLE_TIMING=1 python -m pytest tests/test_oracle_timing.py -s -q
prints one JSON line per (workload, mask).  The whole workload is timed for
the small ones, two heads extrapolated to all heads for the long-sequence one
(heads are independent), and the single-head workload also on one core."""
from __future__ import annotations

import json
import os
import time

import pytest

import oracle
from io_aware_tiled_b200.configs import WORKLOADS
from io_aware_tiled_b200.inputs import attention_inputs


@pytest.mark.skipif(os.environ.get("ORACLE_TIMING") != "1", reason="set ORACLE_TIMING=1 to time the oracle")
def test_time_the_oracle_on_every_workload():
    cores = oracle.num_threads()
    try:
        for w in WORKLOADS.values():
            heads = w.B * w.H
            timed_heads = 2 if w.N >= 16384 else heads
            q, k, v, do = attention_inputs(1, timed_heads, w.N, w.d, seed=w.seed, sigma_qk=w.sigma_qk)
            args = [t.double().numpy() for t in (q, k, v, do)]
            for causal in w.causal_modes:
                for threads in ((cores, 1) if heads == 1 else (cores,)):
                    oracle.set_num_threads(threads)
                    t0 = time.perf_counter()
                    if w.backward:
                        oracle.backward(*args, causal, w.scale)
                    else:
                        oracle.forward(*args[:3], causal, w.scale)
                    dt = (time.perf_counter() - t0) * heads / timed_heads
                    flops = w.fwd_flops(causal) + (w.bwd_flops(causal) if w.backward else 0.0)
                    assert dt > 0
                    print(json.dumps({"oracle": w.name, "causal": causal, "pass": "fwd+bwd" if w.backward else "fwd",
                                      "seconds": dt, "tflops": flops / dt / 1e12, "cores": threads,
                                      "timed_heads": timed_heads, "heads": heads,
                                      "extrapolated": timed_heads != heads}), flush=True)
    finally:
        oracle.set_num_threads(cores)
