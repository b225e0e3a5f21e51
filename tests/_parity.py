"""Helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used by every parity test):
  * scale:  fp16 bits identical;
  * zero:   fp32 z_best within 1e-4 (code units) -- the canonical arithmetic is
            identical on both sides, so equality is expected; fp16 zero equal in
            value;
  * codes:  identical on >= 99.99 % of the weights (only rounding-boundary flips
            are tolerated; 100 % is expected);
  * l_p:    per-tensor sum |W - W_hat|^0.7 (fp64) within 1e-4 relative;
  * the solver's per-group binary32 error sums and accepted-iteration counts:
            identical (the arithmetic is the same op for op on both sides, so a
            one-ulp difference in an error sum is a defect even when it flips no
            early-stop decision);
  * dequantize: fp16 bits identical (both sides compute fp16((c - z) * s) in
            binary32 from the same stored values).
"""
from __future__ import annotations

import numpy as np

import oracle

ZERO_TOL = 1e-4
CODE_MATCH = 0.9999
LP_REL = 1e-4


def gpu_quantize(W_dev, nbits, group, **kw):
    import weight_only_quantization_b200 as hqq
    q = hqq.hqq_quantize_ex(W_dev, nbits=nbits, group=group, **kw)
    import torch
    torch.cuda.synchronize()
    return q


def to_np(q):
    return dict(packed=q.packed.cpu().numpy(),
                scale=q.scale.cpu().numpy().reshape(-1),
                zero=q.zero.cpu().numpy().reshape(-1),
                zero_f32=q.zero_f32.cpu().numpy().reshape(-1),
                err=q.err.cpu().numpy().reshape(-1),
                iters=q.iters.cpu().numpy().reshape(-1))


def compare_full(W_np, gq, ref, nbits, group, p=0.7, label=""):
    """Element-by-element comparison of a whole matrix; returns a stats dict."""
    n = W_np.size
    codes_gpu = oracle.unpack(gq["packed"], n, nbits)
    stats = {}
    assert np.array_equal(gq["scale"].view(np.uint16), ref["scale"].view(np.uint16)), \
        f"{label}: scale mismatch"
    dz = np.abs(gq["zero_f32"].astype(np.float64) - ref["zero_f32"].astype(np.float64))
    stats["max_dz"] = float(dz.max()) if dz.size else 0.0
    assert stats["max_dz"] <= ZERO_TOL, f"{label}: zero differs by {stats['max_dz']}"
    assert np.array_equal(gq["zero"].astype(np.float32), ref["zero"].astype(np.float32)), \
        f"{label}: fp16 zero mismatch"
    match = float(np.mean(codes_gpu == ref["codes"])) if n else 1.0
    stats["code_match"] = match
    assert match >= CODE_MATCH, f"{label}: code match {match}"
    if match == 1.0:
        assert np.array_equal(gq["packed"], ref["packed"]), f"{label}: packed bytes differ"
    stats["iters_equal"] = float(np.mean(gq["iters"] == ref["iters"])) if gq["iters"].size else 1.0
    # the solver's own binary32 error sums: identical arithmetic on both sides
    stats["err_equal"] = float(np.mean(gq["err"].view(np.uint32) == ref["err"].view(np.uint32))) \
        if gq["err"].size else 1.0
    assert stats["iters_equal"] == 1.0, f"{label}: accepted iterations differ"
    assert stats["err_equal"] == 1.0, f"{label}: solver error sums differ"
    Wh_g = oracle.dequantize(codes_gpu, gq["scale"], gq["zero"], group)
    Wh_r = oracle.dequantize(ref["codes"], ref["scale"], ref["zero"], group)
    # fp16 storage can overflow on groups spanning the whole fp16 range; such
    # elements must overflow on both sides and are left out of the error sum
    fin_g, fin_r = np.isfinite(Wh_g), np.isfinite(Wh_r)
    assert np.array_equal(fin_g, fin_r), f"{label}: non-finite reconstructions differ"
    Wf = np.asarray(W_np).reshape(-1)
    eg = oracle.lp_error(Wf[fin_g], Wh_g[fin_g], p)
    er = oracle.lp_error(Wf[fin_r], Wh_r[fin_r], p)
    stats["lp_rel"] = abs(eg - er) / max(er, 1e-300)
    assert stats["lp_rel"] <= LP_REL, f"{label}: l_p error differs by {stats['lp_rel']}"
    return stats


def group_codes(packed, nbits, group, g_idx):
    """Codes of the listed groups, read straight out of a packed buffer."""
    g_idx = np.asarray(g_idx, np.int64)
    out = np.empty((g_idx.size, group), np.uint8)
    for k, g in enumerate(g_idx):
        e0 = int(g) * group
        if nbits in (8, 4, 2, 1):                 # groups are whole bytes (8 | group)
            per = 8 // nbits
            b = packed[e0 // per:(e0 + group) // per]
            out[k] = oracle.unpack(b, group, nbits)
        else:
            w0, w1 = e0 // 10, (e0 + group - 1) // 10
            b = packed[4 * w0:4 * (w1 + 1)]
            allc = oracle.unpack(b, 10 * (w1 - w0 + 1), 3)
            out[k] = allc[e0 - 10 * w0:e0 - 10 * w0 + group]
    return out
