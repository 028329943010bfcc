"""Prints the measured parity errors of the CUDA path against the fp64 oracle on
the five layer workloads, as a markdown table (needs a GPU):

    python tests/report_errors.py

The comparisons are those of test_gpu_configs.py.  C1 and C2 use the full
oracle.  C3, C4 and C5 use sampled query rows (O, LSE, dQ) and key columns
(dK, dV) of the first and last head, the first head only for C5.  C4 also
compares its shared-table gradients in full on a one-head copy of the shape.
The C5 forward is judged on its fp32 output.
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle as orc  # noqa: E402
from synth import make_workload  # noqa: E402
from relpos_harness import lse_err, maxabs, omap, relf, run_library, run_oracle  # noqa: E402


def _f64(t):
    return None if t is None else t.double().numpy()


def _rows(N, seed, k=24):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, N // 2, N - 129, N - 128, N - 2, N - 1]
    return np.unique(np.concatenate([fixed, rng.choice(N, size=k, replace=False)]))


def _table(t, h):
    return None if t is None else (t[h] if t.ndim == 3 else t)


def full(name):
    w = make_workload(name)
    got, want = run_library(w), run_oracle(w)
    r = {"O relF": relf(got["o"], want["o"]), "O maxabs": maxabs(got["o"], want["o"]),
         "LSE maxabs": lse_err(got["lse"], want["lse"])}
    for g in ("dq", "dk", "dv", "daq", "dak", "db"):
        if got.get(g) is not None:
            r[g + " relF"] = relf(got[g], want[g])
    return r


def sampled(name, heads, out_f32=False):
    w = make_workload(name)
    got = run_library(w, out_f32=out_f32)
    m = omap(w)
    q, k, v, do = (_f64(getattr(w, n)) for n in ("q", "k", "v", "do"))
    aq, ak, b = _f64(w.aq), _f64(w.ak), _f64(w.b)
    rows, cols = _rows(w.N, 1), _rows(w.N, 2)
    acc = {}
    for bi in range(w.B):
        for h in heads:
            ref = orc.head_grads_sampled(q[bi, h], k[bi, h], v[bi, h], do[bi, h], _table(aq, h), _table(ak, h),
                                         None if b is None else b[h], w.tau, m, w.causal, None, rows, cols)
            vals = {"O relF": relf(got["o"][bi, h][rows], ref["o"][rows]),
                    "O maxabs": maxabs(got["o"][bi, h][rows], ref["o"][rows]),
                    "LSE maxabs": lse_err(got["lse"][bi, h][rows], ref["lse"][rows]),
                    "dq relF": relf(got["dq"][bi, h][rows], ref["dq"]),
                    "dk relF": relf(got["dk"][bi, h][cols], ref["dk"]),
                    "dv relF": relf(got["dv"][bi, h][cols], ref["dv"])}
            for key, val in vals.items():
                acc[key] = max(acc.get(key, 0.0), val)
    return acc


def one_head_tables():
    w = make_workload("shaw_clip64_n8192", H=1)
    got = run_library(w)
    m = omap(w)
    f = lambda t: t[0, 0].double().numpy()
    g = orc.head_backward(f(w.q), f(w.k), f(w.v), f(w.do), w.aq.double().numpy(), w.ak.double().numpy(), None,
                          w.tau, orc.phi_matrix(m, w.N), np.ones((w.N, w.N), bool), orc.table_rows(m, w.N))
    return {"daq relF": relf(got["daq"], g["daq"]), "dak relF": relf(got["dak"], g["dak"])}


def main():
    res = {
        "C1 shaw_clip16_n256 (full)": full("shaw_clip16_n256"),
        "C2 deberta_log256_n2048 (full)": full("deberta_log256_n2048"),
        "C3 t5_bucket32_n8192 (sampled)": sampled("t5_bucket32_n8192", [0, 11]),
        "C4 shaw_clip64_n8192 (sampled)": sampled("shaw_clip64_n8192", [0, 11]),
        "C4 one head (tables in full)": one_head_tables(),
        "C5 txl_identity_causal_n16384 (sampled, fp32 O)": sampled("txl_identity_causal_n16384", [0], out_f32=True),
    }
    cols = ["O relF", "O maxabs", "LSE maxabs", "dq relF", "dk relF", "dv relF", "daq relF", "dak relF", "db relF"]
    print("| workload | " + " | ".join(cols) + " |")
    print("|---|" + "---|" * len(cols))
    print("| bar | 2e-3 | 5e-3 | 2e-3 | 1e-2 | 1e-2 | 1e-2 | 1e-2 | 1e-2 | 1e-2 |")
    for name, r in res.items():
        print(f"| {name} | " + " | ".join(f"{r[c]:.1e}" if c in r else "" for c in cols) + " |")


if __name__ == "__main__":
    main()
