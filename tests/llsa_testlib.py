"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and compare with
the CPU oracle on identical seeded inputs.

Protocol (selection near-ties): the pyramid must be bit-identical; the GPU's selection is
checked level by level against the oracle's fp64 scores (a row passes if it is the
oracle's Top-K, or a valid Top-K within the tie window); then attention outputs and
gradients are compared with the oracle re-run on the GPU's checked indices ("replay").
"""
from __future__ import annotations

import numpy as np
import torch

from log_linear_hierarchical_b200 import api
from oracle import llsa_oracle as orc
from synthetic import make_inputs, to_f32_numpy, to_f64_numpy

# Tolerances stated for the path: max-abs 1e-4 (fp32) and 2e-2 (bf16) on O, dQ, dK, dV.
TOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def run_gpu(B, H, N, D, topk, levels, dtype, inputs, backward=True, device="cuda", log_bias=False, all_top=False,
            level1=False):
    """All five calls on one stream; returns CPU tensors of every output."""
    tdt = TORCH_DTYPE[dtype]
    shape = api.make_shape(B, H, N, D, topk, levels, tdt, log_bias=log_bias, all_top=all_top,
                           level1=level1)
    dev = {k: v.to(device) for k, v in inputs.items()}
    buf = api.LLSABuffers.allocate(shape, device, tdt)
    assert api.llsa_device_status() == 0
    api.llsa_forward_path(shape, dev["q"], dev["k"], dev["v"], buf)
    if backward:
        api.llsa_backward_path(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    else:
        api.llsa_index_transpose(shape, buf.idx, buf.row_ptr, buf.col, buf.ws_transpose)
    torch.cuda.synchronize()
    status = api.llsa_device_status()
    out = {
        "status": status,
        "q_pyr": [t.cpu().numpy() for t in buf.pyramid_levels(buf.q_pyr)],
        "k_pyr": [t.cpu().numpy() for t in buf.pyramid_levels(buf.k_pyr)],
        "v_pyr": [t.cpu().numpy() for t in buf.pyramid_levels(buf.v_pyr)],
        "idx": [t.cpu().numpy() for t in buf.idx_levels()],
        "row_ptr": [t.cpu().numpy() for t in buf.csr_levels()[0]],
        "col": [t.cpu().numpy() for t in buf.csr_levels()[1]],
        "o": buf.o.float().cpu().numpy(),
        "lse": buf.lse.cpu().numpy(),
    }
    if backward:
        out["dq"] = buf.dq.float().cpu().numpy()
        out["dk"] = buf.dk.float().cpu().numpy()
        out["dv"] = buf.dv.float().cpu().numpy()
    return out


def check_pyramid_bitexact(inputs, gpu, levels):
    for name in ("q", "k", "v"):
        ref = orc.build_pyramid(to_f32_numpy(inputs[name]), levels)
        for lev in range(levels):
            got = gpu[f"{name}_pyr"][lev]
            assert got.shape == ref[lev].shape
            if not np.array_equal(got.view(np.uint32), ref[lev].view(np.uint32)):
                bad = np.argwhere(got.view(np.uint32) != ref[lev].view(np.uint32))[:3]
                raise AssertionError(f"{name} pyramid level {lev + 1} differs at {bad.tolist()}")


def check_selection(gpu, topk):
    res = orc.check_selection(gpu["q_pyr"], gpu["k_pyr"], gpu["idx"], topk)
    assert res["bad"] == 0, res
    return res


def check_transpose_bitexact(gpu):
    rps, cols = orc.index_transpose_all(gpu["idx"])
    for lev, (rp, cl) in enumerate(zip(rps, cols)):
        assert np.array_equal(gpu["row_ptr"][lev], rp), f"row_ptr level {lev + 1}"
        assert np.array_equal(gpu["col"][lev], cl), f"col level {lev + 1}"


def replay(inputs, gpu, backward=True, heads=None, log_bias=False, all_top=False, level1=False):
    """Oracle forward (and backward) on the GPU's indices; ``heads`` = (b, h slice) subset."""
    def sl(x):
        return x if heads is None else x[heads[0]:heads[0] + 1, heads[1]]
    q, k, v = (sl(to_f64_numpy(inputs[n])) for n in ("q", "k", "v"))
    kp = [sl(x) for x in gpu["k_pyr"]]
    vp = [sl(x) for x in gpu["v_pyr"]]
    idx = [sl(x) for x in gpu["idx"]]
    o, lse = orc.forward(q, k, v, kp, vp, idx, log_bias=log_bias, all_top=all_top, level1=level1)
    out = {"o": o, "lse": lse}
    if backward:
        do = sl(to_f64_numpy(inputs["do"]))
        out["dq"], out["dk"], out["dv"] = orc.backward(q, k, v, o, lse, do, kp, vp, idx, log_bias=log_bias,
                                                           all_top=all_top, level1=level1)
    return out


def max_err(a, b):
    return float(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)).max())


def bf16_half_ulp(x):
    """Half a unit in the last place of bf16 (8 significant bits) at |x|: the error of
    storing an exact value in the output format alone, bounded by |x| * 2^-8."""
    return np.abs(np.asarray(x, np.float64)) * 2.0 ** -8


def compare_outputs(gpu, ref, dtype, names, heads=None):
    """Element-wise check: |gpu - ref| <= tol (+ the bf16 output half-ulp of ref for bf16
    outputs, since a bf16 store alone errs by up to |ref| * 2^-8, more than 2e-2 once
    |ref| > 5).  LSE is fp32 in both dtypes."""
    tol = TOL[dtype]
    report = {}
    for n in names:
        g = np.asarray(gpu[n] if heads is None else gpu[n][heads[0]:heads[0] + 1, heads[1]], np.float64)
        r = np.asarray(ref[n], np.float64)
        err = np.abs(g - r)
        if n == "lse":
            lim = np.full_like(r, 1e-4 if dtype == "f32" else 1e-2)
        elif dtype == "bf16":
            lim = tol + bf16_half_ulp(r)
        else:
            lim = np.full_like(r, tol)
        worst = np.unravel_index(np.argmax(err - lim), err.shape)
        report[n] = dict(max_abs=float(err.max()), max_ref=float(np.abs(r).max()),
                         worst_excess=float((err - lim)[worst]), ok=bool(np.all(err <= lim)))
    for n, rep in report.items():
        assert rep["ok"], f"{n}: error exceeds tolerance by {rep['worst_excess']:.3g}; all: {report}"
    return report


def inputs_for(B, H, N, D, dtype, qk_kind, seed):
    return make_inputs(B, H, N, D, dtype, qk_kind, seed)
