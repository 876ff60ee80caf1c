"""Tune tau (the threshold's beta) per workload so the oracle's routing hits a target sparsity.

Writes ``block_sparse_attention_sum_b200/tuned_tau.json``.  Sparsity is the fraction of
(query-block, key-block) pairs that are NOT exact, forced blocks (adjacent, sink) counted as exact.
The search starts from the Gaussian calibration rho_G(beta) = 1 - Phi(beta) (Sol-Attn paper,
section 3.1, "Threshold-Based Routing") and bisects on the oracle's own mask.

Usage: python oracle/tune_tau.py [workload ...]
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_sparse_attention_sum_b200.workloads import TUNED_TAU_PATH, WORKLOADS, load_tuned_tau  # noqa: E402
from oracle import sol_attn_oracle as orc  # noqa: E402


def head_routing(q, k, sink_flags):
    B, N, H, _ = q.shape
    out = []
    for b in range(B):
        for h in range(H):
            qb = orc.head_slice(q, b, h)
            kb = orc.head_slice(k, b, h)
            shat = orc.proxy_scores(orc.block_means(qb), orc.block_means(kb))
            out.append(shat)
    return out, sink_flags


def sparsity_at(tau, shats, sink_flags):
    exact = 0
    total = 0
    for shat in shats:
        _, _, thr = orc.threshold(shat, tau)
        m = orc.exact_mask(shat, thr, sink_flags)
        exact += int(m.sum())
        total += m.size
    return 1.0 - exact / total


def tune(w, tol=2e-4):
    from scipy.stats import norm

    t0 = time.time()
    q, k, _ = w.make_inputs("cpu")
    sink = orc.sink_block_flags(w.N, w.sink_start, w.sink_tokens)
    shats, _ = head_routing(q, k, sink)
    target = w.target_sparsity
    # forced blocks reduce the achievable sparsity; start from the Gaussian calibration
    lo, hi = -6.0, 12.0
    tau = float(norm.ppf(target))
    s = sparsity_at(tau, shats, sink)
    for _ in range(60):
        if abs(s - target) <= tol:
            break
        if s < target:
            lo = tau
        else:
            hi = tau
        tau = 0.5 * (lo + hi)
        s = sparsity_at(tau, shats, sink)
    print(f"{w.name}: tau={tau:.6f} sparsity={s:.5f} target={target} ({time.time() - t0:.1f}s)", flush=True)
    return dict(tau=tau, sparsity=s, target=target, workload=w.name)


def main(names):
    tuned = load_tuned_tau()
    for name in names:
        w = WORKLOADS[name]
        if w.target_sparsity is None:
            continue
        tuned[w.input_key()] = tune(w)
        with open(TUNED_TAU_PATH, "w") as f:
            json.dump(tuned, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or ["s32k_80", "s32k_85", "s32k_90", "s64k", "s128k"])
