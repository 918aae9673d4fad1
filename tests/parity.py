"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI on
seeded inputs and compare with the fp64 oracle element by element.

Tolerances (stated for the fused forward with 16-bit inputs and fp32
accumulation): max |O_gpu - O_ref| <= 2e-2 and max |LSE_gpu - LSE_ref| <= 1e-3."""
import json
import os

import numpy as np
import torch

import attention_forward_18_b200 as af
import oracle
from workloads import make_qkv

O_TOL = 2e-2
LSE_TOL = 1e-3


def run_gpu(q, k, v, causal, scale, stream=None, with_lse=True):
    """q, k, v: CPU 16-bit tensors.  Returns (O, LSE) as CPU float64 numpy arrays."""
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = af.attention(dq, dk, dv, causal=causal, scale=scale, with_lse=with_lse,
                          stream=stream)
    torch.cuda.synchronize()
    assert af.attn_fwd_status() == 0
    return (o.double().cpu().numpy(),
            lse.double().cpu().numpy() if lse is not None else None)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Element-wise comparison; returns a dict with the max / mean errors and the
    worst element, and asserts the tolerances."""
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite O"
    do = np.abs(o_gpu - o_ref)
    worst = np.unravel_index(np.argmax(do), do.shape)
    rep = {"max_dO": float(do.max()), "mean_dO": float(do.mean()), "worst": tuple(map(int, worst)),
           "|O| at worst": float(abs(o_ref[worst]))}
    if lse_gpu is not None:
        assert np.isfinite(lse_gpu).all(), f"{what}: non-finite LSE"
        dl = np.abs(lse_gpu - lse_ref)
        rep["max_dLSE"] = float(dl.max())
        assert rep["max_dLSE"] <= LSE_TOL, f"{what}: {rep}"
    assert rep["max_dO"] <= O_TOL, f"{what}: {rep}"
    return rep


def record(what, rep):
    """Append a comparison report to the JSON-lines file named by ATTN_PARITY_REPORT
    (when set), so a run can keep the measured errors of its full-size checks."""
    path = os.environ.get("ATTN_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": what, **rep}) + "\n")


def check_full(B, H, Sq, Sk, D, dtype, causal, seed, k_scale=1.0, scale=None):
    scale = (1.0 / np.sqrt(D)) if scale is None else scale
    q, k, v = make_qkv(B, H, Sq, Sk, D, dtype, seed, k_scale)
    o, lse = run_gpu(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attn_ref(q.double().numpy(), k.double().numpy(),
                                     v.double().numpy(), causal, scale)
    what = f"B{B} H{H} Sq{Sq} Sk{Sk} D{D} {dtype} c{causal}"
    rep = compare(o, lse, o_ref, lse_ref, what)
    return rep
