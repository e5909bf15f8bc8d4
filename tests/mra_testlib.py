"""Helpers shared by the GPU parity tests (no test functions here).

The CUDA path is called only through the C ABI (ctypes binding); the oracle
gets the same host bytes, widened exactly to fp64.  Nothing computed by the
CUDA path is ever fed to the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import resolution_block_sparse_b200 as mra

# Output tolerances: bf16 inputs 2e-2, fp32 inputs 1e-4 (max-abs over all
# elements, padded rows included).
OUT_TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
# Selection keys: a GPU/oracle difference in the selected set is accepted only
# for blocks whose oracle key lies within TIE_TOL (+ twice the measured
# low-resolution logit error of the fp32 GPU keys) of the k-th oracle key.
TIE_TOL = 1e-6


def run_gpu(inputs, *, block_per_row, approx_mode, first_n=0, diag_n=0, want_intermediates=True):
    q, k, v, mask = inputs["q"], inputs["k"], inputs["v"], inputs["mask"]
    B, H, N, D = q.shape
    nbr = N // 32
    kk = min(nbr * block_per_row, nbr * nbr)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    md = None if mask is None else mask.to(dev)
    out = torch.empty_like(qd)
    res = {}
    if want_intermediates:
        sel = torch.full((B * H, kk), -1, dtype=torch.int32, device=dev)
        logit = torch.empty((B * H, nbr, nbr), dtype=torch.float32, device=dev)
        pooled = torch.empty((3, B * H, nbr, D), dtype=torch.float32, device=dev)
        mra.mra_attention_fwd_ex(qd, kd, vd, md, out, block_per_row, approx_mode, first_n, diag_n,
                                 sel_idx=sel, lowres_logit=logit, pooled=pooled)
        torch.cuda.synchronize()
        res.update(sel=sel.cpu().numpy(), logit=logit.cpu().numpy(), pooled=pooled.cpu().numpy())
    else:
        fn = mra.mra_attention_fwd if q.dtype == torch.bfloat16 else mra.mra_attention_fwd_f32
        fn(qd, kd, vd, md, out, block_per_row, approx_mode, first_n, diag_n)
    torch.cuda.synchronize()
    res["status"] = mra.mra_get_device_status()
    res["out"] = out.float().cpu().numpy()
    res["k"] = kk
    return res


def run_oracle(inputs, *, block_per_row, approx_mode, first_n=0, diag_n=0):
    q, k, v, mask = (inputs[x] for x in ("q", "k", "v", "mask"))
    res = oracle.forward(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                         None if mask is None else mask.double().numpy(),
                         block_per_row=block_per_row, approx_mode=approx_mode, first_n=first_n,
                         diag_n=diag_n)
    res["approx_mode"] = approx_mode
    return res


def compare(inputs, gpu, ora, *, check_intermediates=True, report=None):
    """Assert parity; return a dict of the measured errors."""
    dtype = inputs["q"].dtype
    tol = OUT_TOL[dtype]
    B, H, N, D = inputs["q"].shape
    nbr = N // 32
    kk = ora["k"]
    stats = {}
    assert gpu["status"] == 0, f"device status word {gpu['status']}"
    logit_err = 0.0
    if check_intermediates:
        # q-hat, k-hat; v-hat too in full mode (the pooled V of step four)
        planes = 3 if ora["approx_mode"] == 0 else 2
        pooled_err = float(np.max(np.abs(gpu["pooled"][:planes] - ora["pooled"][:planes])))
        stats["pooled_max_abs"] = pooled_err
        stats["pooled_planes"] = planes
        scale = 1.0 + float(np.max(np.abs(ora["pooled"][:planes])))
        assert pooled_err <= 1e-5 * scale, pooled_err
        logit_err = float(np.max(np.abs(gpu["logit"] - ora["logit"])))
        stats["logit_max_abs"] = logit_err
        lscale = 1.0 + float(np.max(np.abs(ora["logit"])))
        assert logit_err <= 2e-6 * lscale, logit_err
    # selection: per head, set equality except near-ties
    rows_differ = np.zeros((B * H, nbr), dtype=bool)
    mismatches = 0
    window = TIE_TOL + 2.0 * logit_err
    stats["tie_window"] = window
    stats["max_mismatch_gap"] = 0.0
    if check_intermediates:
        for bh in range(B * H):
            g = gpu["sel"][bh]
            o = ora["sel"][bh]
            assert np.all(np.diff(g) > 0), "GPU selection not strictly ascending"
            assert g.min() >= 0 and g.max() < nbr * nbr
            if np.array_equal(g, o):
                continue
            key = ora["key"][bh].reshape(-1)
            kth = np.sort(key)[::-1][kk - 1]
            diff = np.setxor1d(g, o)
            mismatches += diff.size
            stats["max_mismatch_gap"] = max(stats["max_mismatch_gap"],
                                            float(np.max(np.abs(key[diff] - kth))))
            # the band is 1e-6 (the stated tie tolerance) widened by twice
            # the measured fp32 error of the GPU's low-resolution logits
            bad = [int(i) for i in diff if abs(key[i] - kth) > window]
            assert not bad, f"head {bh}: blocks {bad[:8]} differ but are not near-ties"
            rows_differ[bh, np.unique(diff // nbr)] = True
    stats["sel_mismatches"] = mismatches
    # outputs on every query row whose block row has the same selection
    out_g = gpu["out"].reshape(B * H, nbr, 32, D)
    out_o = ora["out"].reshape(B * H, nbr, 32, D)
    same = ~rows_differ
    err = float(np.max(np.abs(out_g[same] - out_o[same]))) if same.any() else 0.0
    stats["out_max_abs"] = err
    stats["rows_compared"] = int(same.sum())
    assert np.all(np.isfinite(gpu["out"])), "non-finite output"
    assert err <= tol, f"max-abs output error {err} > {tol}"
    if report is not None:
        report.update(stats)
    return stats
