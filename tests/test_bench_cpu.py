"""The benchmark's CPU baseline runs the oracle on every host core (worker processes over
(head, query-block chunk), results gathered in shared memory).  It must compute what the
oracle computes serially: the same O and LSE and, up to the order of the fp64 additions of
the chunks' dK/dV contributions, the same gradients."""
import numpy as np
import pytest

import bench
from oracle import llsa_oracle as orc
from synthetic import WORKLOADS, make_config_inputs, to_f32_numpy, to_f64_numpy


@pytest.mark.parametrize("name", ["tiny-f32"])
def test_oracle_pool_matches_serial_oracle(name):
    cfg = WORKLOADS[name]
    host = make_config_inputs(cfg, with_do=True)
    pool = bench.OraclePool(cfg, host, dict(log_bias=False, all_top=False, level1=False), cores=3)
    try:
        pool.step(backward=True)
        from multiprocessing import shared_memory  # noqa: F401  (the pool keeps its blocks)
        B, H, N, D = cfg.B, cfg.H, cfg.N, cfg.D
        got = {k: np.ndarray((B, H, N, D), dtype=np.float64, buffer=pool.shm[k].buf).copy()
               for k in ("o", "dq", "dk", "dv")}
        got["lse"] = np.ndarray((B, H, N), dtype=np.float64, buffer=pool.shm["lse"].buf).copy()
    finally:
        pool.close()
    q32, k32, v32 = (to_f32_numpy(host[x]) for x in ("q", "k", "v"))
    ref = orc.llsa_step(to_f64_numpy(host["q"]), to_f64_numpy(host["k"]), to_f64_numpy(host["v"]),
                        to_f64_numpy(host["do"]), cfg.levels, cfg.topk)
    np.testing.assert_array_equal(got["o"], ref["o"])
    np.testing.assert_array_equal(got["lse"], ref["lse"])
    np.testing.assert_array_equal(got["dq"], ref["dq"])
    np.testing.assert_allclose(got["dk"], ref["dk"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["dv"], ref["dv"], rtol=0, atol=1e-12)


def test_reference_arm_prints_whole_measured_steps():
    """`bench.py --impl reference` times whole oracle steps inside its own run: the line says
    so, and steps x ms_per_step fits in the run's wall clock."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
                          "tiny-f32", "--steps", "2", "--warmup", "3", "--ref-cores", "2"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3
    assert line["cpu_baseline"]["cores"] == 2 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    c = line["consistency"]
    assert c["fits_in_driver_run"] and not c["extrapolated"]
    assert abs(c["timed_seconds"] - 2 * line["ms_per_step"] / 1000.0) < 1e-2
    assert line["config"]["heads_per_step"] == 2   # tiny-f32 has 2 heads: whole steps, no sample
