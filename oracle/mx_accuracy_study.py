"""Accuracy study of the MXFP8 emulation (test infrastructure, CPU only).

    python -m oracle.mx_accuracy_study [--threads N]

Prints two markdown tables.

1. Cosine similarity to the exact fp64 oracle of O, dQ, dK, dV for the MXFP8
   emulation as the method defines it (FLAMIA page, sec. "FLAMIA Mimarisi ve
   Temel Tasarim Ilkeleri": MXFP8 operands, token-block scaling, leak guards)
   and with one quantisation taken out at a time (inputs Q, K, V, dO; the
   computed P~/P~T; the computed dS~/dS~T), with the OCP scale rule, and with
   the symmetric diagonal guard, and for the mixed NVFP4/FP8 path (scores
   from NVFP4 Q and K, decode scales 1).  Workloads: the 16384-token outlier-channel
   workload (all 16 heads) and the first documents of the 32768-token
   log-normal workload (KV heads 0-7).
2. The leak test T3 at document-local token positions t that are not the end
   of a 32-token block: with dO = 0 after t in both runs and Q, K, V
   randomised after t, the number of dK and dV elements at positions <= t that
   differ (and the largest difference relative to the RMS of dK or dV), for
   the method's reading (Q and dO in token-block form in every query block of
   dK = dS^T Q and dV = P^T dO) and for the symmetric guard (per-token Q and dO
   on the diagonal query block).
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from causal_flash_attention_packed_b200 import workloads as W  # noqa: E402  (seeded inputs only)

VARIANTS = [
    ("method (RCEIL)", oracle.MX_QUANT_P),
    ("inputs unquantised", oracle.MX_QUANT_P | oracle.MX_KEEP_INPUTS),
    ("P~, P~T unquantised", oracle.MX_QUANT_P | oracle.MX_KEEP_P),
    ("dS~, dS~T unquantised", oracle.MX_QUANT_P | oracle.MX_KEEP_DS),
    ("only inputs quantised", oracle.MX_QUANT_P | oracle.MX_KEEP_P | oracle.MX_KEEP_DS),
    ("OCP scale rule", oracle.MX_QUANT_P | oracle.MX_RULE_OCP),
    ("symmetric diagonal guard", oracle.MX_QUANT_P | oracle.MX_SYM_GUARD),
    ("mixed NVFP4/FP8 (NVFP4 scores)", None),
]


def _cos(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def _subset(w, max_tokens, kv_heads):
    q, k, v, do = w.tensors()
    cu = w.cu
    n = 1
    while n < w.n_docs and cu[n + 1] <= max_tokens:
        n += 1
    T = int(cu[n])
    G = w.Hq // w.Hkv
    hq = slice(0, kv_heads * G)
    hk = slice(0, kv_heads)
    arrs = (q[:T, hq], k[:T, hk], v[:T, hk], do[:T, hq])
    return [a.double().numpy() for a in arrs], cu[: n + 1].astype(np.int32), n, T


def cosine_table():
    rows = []
    cases = [("16K outlier channels, 16 heads", W.config(3, 0), 16384, 16),
             ("32K log-normal, first documents, KV heads 0-7", W.config(4, 0), 6000, 8)]
    for title, w, max_tokens, kvh in cases:
        args, cu, n, T = _subset(w, max_tokens, kvh)
        ex = oracle.attn_bwd(*args, cu, w.scale)
        for name, flags in VARIANTS:
            if flags is None:
                em = oracle.nvmx_attn_bwd(*args, cu, w.scale, flags=oracle.MX_QUANT_P)
            else:
                em = oracle.mx_attn_bwd(*args, cu, w.scale, flags=flags)
            rows.append((f"{title} ({n} docs, {T} tokens)", name,
                         *(_cos(em[key], ex[key]) for key in ("o", "dq", "dk", "dv"))))
    out = ["| workload | emulation | O | dQ | dK | dV |", "|---|---|---|---|---|---|"]
    out += [f"| {r[0]} | {r[1]} | " + " | ".join(f"{c:.5f}" for c in r[2:]) + " |" for r in rows]
    return "\n".join(out)


def t3_table():
    w = W.custom([300, 513, 200], Hq=2, Hkv=2, d=128, seed=74)
    q, k, v, do = (t.double().numpy() for t in w.tensors())
    rng = np.random.default_rng(10)
    out = ["| t (doc-local) | reading | dK elements differing | dV elements differing | max rel. diff dK | max rel. diff dV |",
           "|---|---|---|---|---|---|"]
    for t_rel in (13, 100, 200, 300, 450):
        t = 300 + t_rel
        do0 = do.copy()
        do0[t + 1:] = 0.0
        q2, k2, v2 = (x.copy() for x in (q, k, v))
        for x in (q2, k2, v2):
            x[t + 1:] = rng.standard_normal(x[t + 1:].shape) * 30
        for name, flags in (("method", oracle.MX_QUANT_P), ("symmetric guard", oracle.MX_QUANT_P | oracle.MX_SYM_GUARD)):
            a = oracle.mx_attn_bwd(q, k, v, do0, w.cu, w.scale, flags=flags)
            b = oracle.mx_attn_bwd(q2, k2, v2, do0, w.cu, w.scale, flags=flags)
            cells = []
            for key in ("dk", "dv"):
                x, y = a[key][: t + 1], b[key][: t + 1]
                cells.append((int(np.count_nonzero(x != y)), x.size,
                              float(np.max(np.abs(x - y)) / np.sqrt(np.mean(x * x)))))
            out.append(f"| {t_rel} | {name} | {cells[0][0]} of {cells[0][1]} | {cells[1][0]} of {cells[1][1]} | "
                       f"{cells[0][2]:.2e} | {cells[1][2]:.2e} |")
    return "\n".join(out)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--threads", type=int, default=len(os.sched_getaffinity(0)))
    a = ap.parse_args()
    oracle.set_threads(a.threads)
    print(cosine_table())
    print()
    print(t3_table())


if __name__ == "__main__":
    main()
