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


if __name__ == "__main__":
    main()
