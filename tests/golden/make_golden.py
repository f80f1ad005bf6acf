"""Writes thm35_sigmoid.txt: the worked example of Theorem 3.5 in the Swimba paper notes
(papernotes.org NeurIPS 2026, Method, key design 3).  With two experts, T = 1, A = 0 and N = P = 1,
router logits (0, x) give the second expert the weight e^x / (1 + e^x) = sigma(x).
The values are that closed form evaluated with the standard library; nothing here calls the oracle
or the CUDA library.  Run:  python tests/golden/make_golden.py"""
import math
import os

XS = (-3.0, -0.25, 0.0, 1.5, 4.0)

here = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(here, "thm35_sigmoid.txt"), "w") as f:
    f.write("# Swimba paper notes (papernotes.org, NeurIPS 2026), Method, key design 3, Theorem 3.5:\n")
    f.write("# two experts, logits g = (0, x): weight of expert 1 = e^x / (1 + e^x) = sigma(x)\n")
    f.write("# columns: x  sigma(x)\n")
    for x in XS:
        f.write(f"{x!r} {math.exp(x) / (1.0 + math.exp(x))!r}\n")
