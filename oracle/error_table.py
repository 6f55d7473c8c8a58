"""Approximation error of the truncated series against the exact inverse.

TEST INFRASTRUCTURE (part of the oracle): runs the float64 oracle only, no
kernel.  For a sample of chunks of the B=4, H=16, T=4096, k=64 workload (bf16
K and V, as stored) it reports, per Neumann order N, band mask and residual
order S, the relative Frobenius error and the SNR of T and of W = T diag(b) K
against the exact inverse (forward substitution), the worst chunk, and the
largest entry of each masked power (the dynamic range the INT8 / INT16 codes
must cover), and the same errors for the INT8 and INT16 series.  "When Good
Enough Is Optimal", Études d'Ablation, reports these quantities per N and
mask on its own models; here they are measured on the synthetic inputs.

    python -m oracle.error_table [--chunks 256] [--gate-scale 1.0]
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from gated_deltanet_chunk_02_b200.inputs import Workload, as_f64_numpy, make_inputs  # noqa: E402
from oracle import gdn_oracle as o  # noqa: E402


def sample_chunks(n: int, gate_scale: float = 1.0, seed: int = 0):
    """``n`` chunks spread evenly over the heads of the B=4, H=16, T=4096 workload."""
    w = Workload(B=4, H=16, T=4096, k=64, dtype="bf16")
    inp = make_inputs(w, seed=seed, gate_scale=gate_scale)
    K = o.to_chunks(as_f64_numpy(inp["K"]), w.k)
    V = o.to_chunks(as_f64_numpy(inp["V"]), w.k)
    beta = o.to_chunks(as_f64_numpy(inp["beta"]), w.k)
    g = o.to_chunks(as_f64_numpy(inp["g"]), w.k)
    idx = np.linspace(0, w.n_chunks - 1, n).astype(np.int64)
    return K[idx], V[idx], beta[idx], g[idx]


def error_table(n_chunks: int = 256, gate_scale: float = 1.0, Ns=(1, 2, 3, 4), Ss=(0, 8)):
    K, V, beta, g = sample_chunks(n_chunks, gate_scale)
    A = o.build_A(K, beta, g)
    T_ex = o.invert_fwdsub(A)
    W_ex, _ = o.wy(T_ex, K, V, beta)
    rows = []
    for N in Ns:
        for mask in (True, False):
            for S in Ss:
                T = o.invert_neumann(A, N, mask, S)
                W, _ = o.wy(T, K, V, beta)
                per_chunk = [o.rel_fro(T[c], T_ex[c]) for c in range(len(T))]
                rows.append({"N": N, "mask": int(mask), "S": S,
                             "T_rel_fro": o.rel_fro(T, T_ex), "T_snr_db": o.snr_db(T, T_ex),
                             "T_worst_chunk": max(per_chunk),
                             "W_rel_fro": o.rel_fro(W, W_ex), "W_snr_db": o.snr_db(W, W_ex)})
    # the quantised series (S = 0): INT8 and INT16 codes with per-chunk scales,
    # from the float32 A both integer schemes start from
    A32 = A.astype(np.float32)
    quant = []
    for N in Ns:
        for mask in (True, False):
            T8 = o.int8_neumann(A32, N, mask)["T"]
            T16 = o.int16_neumann(A32, N, mask)["T"]
            Tf = o.invert_neumann(A, N, mask, 0)
            quant.append({"N": N, "mask": int(mask),
                          "float_rel_fro": o.rel_fro(Tf, T_ex),
                          "int8_rel_fro": o.rel_fro(T8, T_ex),
                          "int16_rel_fro": o.rel_fro(T16, T_ex),
                          "int8_vs_float": o.rel_fro(T8, Tf),
                          "int16_vs_float": o.rel_fro(T16, Tf)})
    # largest entry of the masked powers P_n = M (.) (P_{n-1} A), mean over chunks
    amax = {}
    k = A.shape[-1]
    for N in Ns:
        Mb = o.band_mask(k, N)
        P = A * Mb
        vals = [float(np.mean(np.max(np.abs(P), axis=(1, 2))))]
        for _ in range(2, N + 1):
            P = (P @ A) * Mb
            vals.append(float(np.mean(np.max(np.abs(P), axis=(1, 2)))))
        amax[N] = vals
    return {"chunks": n_chunks, "gate_scale": gate_scale, "rows": rows, "quantised": quant,
            "amax_masked_powers": amax}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--chunks", type=int, default=256)
    ap.add_argument("--gate-scale", type=float, default=1.0)
    ap.add_argument("--json", action="store_true", help="print one JSON object")
    args = ap.parse_args(argv)
    res = error_table(args.chunks, args.gate_scale)
    if args.json:
        print(json.dumps(res))
        return 0
    print(f"{res['chunks']} chunks, gate scale {res['gate_scale']}")
    print("| N | mask | S | T rel. Frobenius | T SNR (dB) | worst chunk | W rel. Frobenius | W SNR (dB) |")
    print("|---|---|---|---|---|---|---|---|")
    for r in res["rows"]:
        print(f"| {r['N']} | {'on' if r['mask'] else 'off'} | {r['S']} | {r['T_rel_fro']:.3e} | "
              f"{r['T_snr_db']:.1f} | {r['T_worst_chunk']:.3e} | {r['W_rel_fro']:.3e} | "
              f"{r['W_snr_db']:.1f} |")
    print()
    print("| N | mask | float64 series | INT8 | INT16 | INT8 vs float64 series | INT16 vs float64 series |")
    print("|---|---|---|---|---|---|---|")
    for r in res["quantised"]:
        print(f"| {r['N']} | {'on' if r['mask'] else 'off'} | {r['float_rel_fro']:.3e} | "
              f"{r['int8_rel_fro']:.3e} | {r['int16_rel_fro']:.3e} | {r['int8_vs_float']:.3e} | "
              f"{r['int16_vs_float']:.3e} |")
    print("max |P_n| (masked powers, mean over chunks):",
          {N: [f"{v:.3g}" for v in vals] for N, vals in res["amax_masked_powers"].items()})
    return 0


if __name__ == "__main__":
    sys.exit(main())
