"""Shared test helpers: device copies of seeded inputs and oracle comparisons.

The oracle side gets numpy arrays from ``synthetic``; the CUDA side gets the
same bytes as torch tensors.  Neither side's arithmetic lives here.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synthetic as S

REL_TOL = 2e-3          # max|gpu - oracle| / max|oracle| on layer outputs
GATE_TOL = 1e-6         # absolute, on fp32 gates
TIE_EPS = 1e-5          # logit gap under which a selection difference is logged


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    return float(np.abs(gpu - ref).max() / (den if den > 0 else 1.0))


def dev_x(L: S.LayerInputs, device="cuda"):
    if L.cfg.x_dtype == "bf16":
        return torch.from_numpy(L.x_raw.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(L.x_raw).to(device)


def dev(a, device="cuda"):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)


def dev_pool(moe, L: S.LayerInputs, device="cuda"):
    return moe.ExpertPool(dev(L.gate, device), dev(L.up, device), dev(L.down, device),
                          L.cfg.qtype)


def dev_shared(moe, L: S.LayerInputs, device="cuda"):
    if L.shared is None:
        return None
    g, u, d = L.shared
    return moe.ExpertPool(dev(g, device), dev(u, device), dev(d, device), L.cfg.shared_qtype)


def oracle_route(L: S.LayerInputs):
    if L.logits is not None:
        logits = L.logits if L.bias is None else (L.logits + L.bias)
        ids, g = oracle.select(logits, L.cfg.k, L.cfg.renorm)
        return logits.astype(np.float32), ids, g
    return oracle.route(L.x, L.w_router, L.bias, L.cfg.k, L.cfg.renorm)


def gates_at(logits, ids, renorm=True):
    """Oracle gates (double) of an arbitrary selection ``ids`` of the
    oracle logits: softmax over the selected logits when renormalised."""
    Lg = np.asarray(logits, np.float64)
    sel = np.take_along_axis(Lg, ids.astype(np.int64), axis=1)
    m = Lg.max(axis=1, keepdims=True)
    p = np.exp(sel - m)
    if renorm:
        return p / p.sum(axis=1, keepdims=True)
    return p / np.exp(Lg - m).sum(axis=1, keepdims=True)


def check_ids(gpu_ids, ref_ids, ref_logits, k, log=None):
    """Exact match except on near-tie tokens, which are logged.  Returns
    the list of logged tokens."""
    gpu_ids = np.asarray(gpu_ids)
    diff = np.nonzero((gpu_ids != ref_ids).any(axis=1))[0]
    ties = set(oracle.near_tie_tokens(ref_logits, k, TIE_EPS).tolist())
    bad = [int(t) for t in diff if int(t) not in ties]
    assert not bad, f"routing mismatch on non-tie tokens {bad[:10]}"
    logged = [int(t) for t in diff]
    if log is not None and logged:
        log(f"near-tie tokens with a different selection: {logged}")
    return logged
