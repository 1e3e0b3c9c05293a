"""Shared helpers of the GPU parity tests: load a seeded model on both sides,
run the oracle on the same inputs, and compare with the stated tolerances.

Tolerances (from the round's parity bar):
  * bf16 model: |gpu - oracle| <= 1e-2 + 2e-2 |oracle| for attention outputs,
    K/V rows and logits.
  * fp32 model: relative 1e-4, as |gpu - oracle| <= 1e-4 (|oracle| + rms(oracle))
    (the rms term keeps near-zero entries, where fp32 rounding of a dot
    product is relative to its summands rather than its result, from
    reading as relative noise).
  * tokens: teacher-forced -- the oracle walks with the GPU's previous token,
    and wherever the oracle's top-1 minus top-2 margin exceeds 1e-2 the GPU
    token must equal the oracle's.
  * confidences: |delta| <= 1e-3, with the GPU's tokens as the previous tokens.

The cache rows are compared with the oracle's fp64 K/V; the round itself is
compared with the oracle run on the K/V as the cache stores them (fp16 rows
for a bf16 model, fp32 for fp32: dspark_kv_dtype).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import dspark as O
from synthetic import make_weights

MARGIN = 1e-2
CONF_TOL = 1e-3


def to_device(tensors, device="cuda"):
    return {k: v.to(device) for k, v in tensors.items()}


def build(shape, seed, **kw):
    import block_draft_model_dspark_b200 as dsp
    cpu = make_weights(shape, seed, **kw)
    gpu = to_device(cpu)
    model = dsp.DsparkModel(shape, gpu)
    return cpu, O.OracleWeights(cpu, shape), model


def assert_close(got, want, dtype: str, what: str):
    g = np.asarray(got, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    if dtype == "fp32":
        scale = np.sqrt(np.mean(w * w)) if w.size else 0.0
        tol = 1e-4 * (np.abs(w) + scale)
    else:
        tol = 1e-2 + 2e-2 * np.abs(w)
    err = np.abs(g - w)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {bad.sum()}/{bad.size} outside tolerance; worst at {i}: "
                             f"gpu {g[i]:.6g} oracle {w[i]:.6g} (tol {tol[i]:.3g})")


def check_tokens(W, U_oracle, anchors, gpu_tokens, what="tokens"):
    """Teacher-forced token parity; returns (checked steps, total steps)."""
    toks, margins = O.teacher_forced_walk(W, U_oracle, anchors, gpu_tokens)
    decisive = margins > MARGIN
    mism = decisive & (toks != gpu_tokens)
    if mism.any():
        b, k = np.argwhere(mism)[0]
        raise AssertionError(f"{what}: gpu token {gpu_tokens[b, k]} != oracle {toks[b, k]} at row {b} step {k} "
                             f"(margin {margins[b, k]:.4g}); {mism.sum()} mismatches")
    return int(decisive.sum()), int(decisive.size)


def cache_store(dtype: str) -> str:
    """Storage type of a model's K/V cache: fp16 rows for a bf16 model (dspark_kv_dtype), fp32 for fp32."""
    return "fp16" if dtype == "bf16" else dtype


def as_stored(kv_rows, dtype: str):
    """The oracle's fp64 context K/V as the cache of a `dtype` model stores them."""
    store = cache_store(dtype)
    return [[(O.store_rounded(k, store), O.store_rounded(v, store)) for (k, v) in row] for row in kv_rows]


def ensure_built():
    from block_draft_model_dspark_b200 import build as b
    b.build()
