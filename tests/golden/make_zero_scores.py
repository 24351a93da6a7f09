"""Writes zero_scores.txt: log Z of one sequence with all-zero emissions,
transitions and duration bias, from the exact number of labelled segmentations.

With every score zero, exp Score(y) = 1 for every segmentation y, so Z is the
count of segmentations of [0, L) into segments of duration 1..K, each with one
of C labels:  N(0) = 1,  N(t) = C * sum_{d=1..min(K,t)} N(t-d),  Z = N(L).
(For K >= L this is C (1+C)^(L-1).)  Exact integer arithmetic; the log is taken
of the integer.  Pure combinatorics: nothing here comes from the oracle or the
CUDA path.  Run from the repository root:  python tests/golden/make_zero_scores.py
"""
import math
import os

# (L, K, C): the named workloads' label and duration counts at lengths the exact
# integers stay quick for
SHAPES = [(64, 8, 4), (512, 16, 17), (4000, 64, 128), (3000, 1000, 24), (5000, 200, 24), (1500, 512, 256)]


def count(L, K, C):
    N = [1] + [0] * L
    window = 1   # sum of N[t-d] for d = 1..min(K, t), kept incrementally
    for t in range(1, L + 1):
        N[t] = C * window
        window += N[t]
        if t - K >= 0:
            window -= N[t - K]
    return N[L]


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zero_scores.txt")
    with open(path, "w") as f:
        f.write("# L K C logZ  -- all-zero scores: log of the exact segmentation count (make_zero_scores.py)\n")
        for L, K, C in SHAPES:
            f.write(f"{L} {K} {C} {math.log(count(L, K, C))!r}\n")


if __name__ == "__main__":
    main()
