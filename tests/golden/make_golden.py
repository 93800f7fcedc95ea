"""Writes the hand-worked attention fixtures in this folder.

Every expected value here is a closed form derived by hand (the derivation is
stored with each case); this script only evaluates those closed forms with
Python's ``math`` module.  It calls neither the oracle nor the CUDA path.

Operator: scaled dot-product attention with an optional causal mask and
grouped-query heads, the workload the PipeThreader pages benchmark as
"FlashAttention" (papers.lqhl.me "PipeThreader-OSDI25", section 实验与结果,
paper Sec. 6.2 / Fig. 12).  The pages do not print the formula; the textbook
definition O = softmax(Q K^T / sqrt(D) + mask) V with LSE = ln sum exp of the
scaled logits is the reading used throughout.

Run:  python tests/golden/make_golden.py
"""
import json
import math
import os

CITE = ("Operator: scaled dot-product attention with an optional causal mask, benchmarked as "
        "'FlashAttention' on the PipeThreader pages (papers.lqhl.me 'PipeThreader-OSDI25', "
        "section '实验与结果', paper Sec. 6.2 / Fig. 12). The pages do not print the formula; the "
        "textbook definition O = softmax(QK^T/sqrt(D) + mask) V, LSE = log sum exp of the scaled "
        "logits, is used. Expected values are worked by hand below; decimals are those closed forms.")


def cases():
    r2, e = math.sqrt(2.0), math.e
    out = []
    out.append(dict(
        name="causal_s2_d1", causal=True, B=1, Hq=1, Hkv=1, S=2, D=1,
        derivation=["scale = 1/sqrt(1) = 1; q = [1, 1]; k = [0, ln 3]; v = [2, 6]",
                    "row 0 (causal) sees key 0 only: P = [1], O = v0 = 2, LSE = s00 = 0",
                    "row 1 sees keys 0,1: s = [0, ln 3], P = [1/4, 3/4], "
                    "O = 2/4 + 3*6/4 = 5, LSE = ln(1+3) = ln 4"],
        q=[1.0, 1.0], k=[0.0, math.log(3.0)], v=[2.0, 6.0], o=[2.0, 5.0],
        lse=[0.0, math.log(4.0)]))

    k = [[0.0, 0.0], [math.log(2.0), 1.0], [math.log(5.0), -1.0]]
    v = [[8.0, 0.0], [0.0, 8.0], [8.0, 8.0]]
    z1 = 1 + e + 1 / e
    z2 = 1 + 2 * e + 5 / e
    out.append(dict(
        name="noncausal_s3_d2", causal=False, B=1, Hq=1, Hkv=1, S=3, D=2,
        derivation=["scale = 1/sqrt(2); q rows (sqrt2,0), (0,sqrt2), (sqrt2,sqrt2) so "
                    "s_ij = k_j0, k_j1, k_j0+k_j1",
                    "k = [(0,0), (ln2,1), (ln5,-1)]; v = [(8,0), (0,8), (8,8)]",
                    "row 0: s = (0, ln2, ln5), P = (1,2,5)/8, O = (6,7), LSE = ln 8",
                    "row 1: s = (0, 1, -1), P = (1,e,1/e)/Z1 with Z1 = 1+e+1/e, "
                    "O = (8+8/e, 8e+8/e)/Z1, LSE = ln Z1",
                    "row 2: s = (0, ln2+1, ln5-1), P = (1,2e,5/e)/Z2 with Z2 = 1+2e+5/e, "
                    "O = (8+40/e, 16e+40/e)/Z2, LSE = ln Z2"],
        q=[[r2, 0.0], [0.0, r2], [r2, r2]], k=k, v=v,
        o=[[6.0, 7.0], [(8 + 8 / e) / z1, (8 * e + 8 / e) / z1],
           [(8 + 40 / e) / z2, (16 * e + 40 / e) / z2]],
        lse=[math.log(8.0), math.log(z1), math.log(z2)]))

    out.append(dict(
        name="causal_s3_d2", causal=True, B=1, Hq=1, Hkv=1, S=3, D=2,
        derivation=["scale = 1/sqrt(2); every q row = (sqrt2, 0) so s_ij = k_j0 = (0, ln2, ln5)",
                    "row 0 sees key 0: O = v0 = (8,0), LSE = 0",
                    "row 1 sees keys 0,1: P = (1,2)/3, O = (8/3, 16/3), LSE = ln 3",
                    "row 2 sees all: P = (1,2,5)/8, O = (6,7), LSE = ln 8"],
        q=[[r2, 0.0]] * 3, k=k, v=v, o=[[8.0, 0.0], [8 / 3, 16 / 3], [6.0, 7.0]],
        lse=[0.0, math.log(3.0), math.log(8.0)]))

    out.append(dict(
        name="gqa_s1_d1", causal=True, B=1, Hq=4, Hkv=2, S=1, D=1,
        derivation=["S=1: each query row sees one key, so P = [1], O = V[b,g,0], "
                    "LSE = q*k/sqrt(1)",
                    "grouped-query heads in contiguous groups: g = hq // (Hq/Hkv) = hq // 2",
                    "q = [1,2,3,4]; k = [0.5, -1]; v = [10, 20] -> O = [10,10,20,20], "
                    "LSE = [0.5, 1.0, -3, -4]"],
        q=[1.0, 2.0, 3.0, 4.0], k=[0.5, -1.0], v=[10.0, 20.0], o=[10.0, 10.0, 20.0, 20.0],
        lse=[0.5, 1.0, -3.0, -4.0]))
    return out


def main():
    here = os.path.dirname(os.path.abspath(__file__))
    for c in cases():
        c = dict(cite=CITE, **c)
        with open(os.path.join(here, c["name"] + ".json"), "w") as f:
            json.dump(c, f, indent=1)
            f.write("\n")


if __name__ == "__main__":
    main()
