"""Write the stored expected values under tests/golden/ (calls only the oracle).

wkv_tiny_decimal.txt: the "tiny" workload (B=1, T=8, C=4, seed 0, zero initial
state) evaluated by the direct sum of the wkv_t equation ("Linear attention
without writing a CUDA kernel", section "The recurrence") in 50-digit decimal
arithmetic. Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import oracle as O  # noqa: E402
from wkv_recurrence_b200 import inputs as I  # noqa: E402


def main():
    wl = I.WORKLOADS["tiny"]
    k, v = I.draw_kv(wl, seed=0)
    w, u = I.draw_w(wl, 0), I.draw_u(wl, 0)
    res = O.decimal_forward(k, v, w, u, digits=50)
    path = os.path.join(HERE, "wkv_tiny_decimal.txt")
    with open(path, "w") as f:
        f.write("# wkv_t by the direct sum of the equation in 'Linear attention without writing a\n")
        f.write("# CUDA kernel', section 'The recurrence'; 50-digit decimal arithmetic.\n")
        f.write("# workload tiny (B=1, T=8, C=4, seed 0), zero initial state. Written by make_golden.py.\n")
        f.write("# columns: b t c k v w u wkv   (k, v, w, u: the fp32 inputs, printed exactly)\n")
        for b in range(wl.B):
            for t in range(wl.T):
                for c in range(wl.C):
                    f.write(f"{b} {t} {c} {float(k[b, t, c])!r} {float(v[b, t, c])!r} "
                            f"{float(w[c])!r} {float(u[c])!r} {res[b][t][c]:.30e}\n")
    print("wrote", path)

    # the same tiny case with per-token decays w_t = exp(N(-1, 1)) and a
    # receptance gate r ~ N(0, 1) ("RWKV-v6 Architecture: Attention-Free Linear
    # Transformers", sections "2. Dynamic Data-Dependent Decay" and the gated
    # readout of "3. Matrix-Valued Hidden State")
    import numpy as np
    g = np.random.default_rng(2024)
    wt = np.exp(g.normal(-1.0, 1.0, k.shape)).astype(np.float32)
    r = g.normal(0.0, 1.0, k.shape).astype(np.float32)
    res = O.decimal_forward(k, v, w, u, digits=50, w_t=wt, r=r)
    path = os.path.join(HERE, "wkv_tiny_wt_gate_decimal.txt")
    with open(path, "w") as f:
        f.write("# sigmoid(r_t) * wkv_t by the direct sum of the equation in 'Linear attention without\n")
        f.write("# writing a CUDA kernel', section 'The recurrence', with the per-token decay w_t of\n")
        f.write("# 'RWKV-v6 Architecture', section '2. Dynamic Data-Dependent Decay' in place of w\n")
        f.write("# (token i reaches token t with exponent k_i - (w_{i+1} + ... + w_{t-1})); 50-digit\n")
        f.write("# decimal arithmetic. Workload tiny (B=1, T=8, C=4, seed 0), zero initial state;\n")
        f.write("# w_t = exp(N(-1, 1)), r ~ N(0, 1) from numpy seed 2024. Written by make_golden.py.\n")
        f.write("# columns: b t c k v w_t u r out   (inputs: the fp32 values, printed exactly)\n")
        for b in range(wl.B):
            for t in range(wl.T):
                for c in range(wl.C):
                    f.write(f"{b} {t} {c} {float(k[b, t, c])!r} {float(v[b, t, c])!r} "
                            f"{float(wt[b, t, c])!r} {float(u[c])!r} {float(r[b, t, c])!r} "
                            f"{res[b][t][c]:.30e}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
