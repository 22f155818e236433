"""Derive the hand-checkable schedule fixture ``schedule_case.json`` with exact fractions.

The case is small enough to check on paper: N_img = 4 image tokens in M = 2 patches of 2,
T = 1 text token, one head, head_dim 1, softmax scale 1, two diffusion steps.  Keys are
stored as natural logarithms of small integers, so a query value q gives the key of
integer a the weight a**q and every output is a rational number.

Which rows a patch sees follows "기술 요약: PipeFusion" (핵심 메커니즘 2, 시간적 중복성 활용)
and the micro-step order of 핵심 메커니즘 3: at step s, patch p sees this step's rows for
patches <= p and step s-1's rows for patches > p; step 0 sees step 0 everywhere.

This script uses exact rational arithmetic only; it does not import the oracle.
Run:  python tests/golden/derive_schedule_case.py > tests/golden/schedule_case.json
"""
import json
from fractions import Fraction

CASE = {
    "n_img": 4, "n_patches": 2, "n_txt": 1, "heads": 1, "head_dim": 1, "scale": 1.0,
    # per step: key integers (key value = ln(a)), values, text key integer, text value, queries
    "steps": [
        {"k_int": [1, 2, 3, 4], "v": [10, 20, 30, 40], "ktxt_int": 2, "vtxt": 6, "q": [1, 1, 2, 1]},
        {"k_int": [2, 1, 5, 1], "v": [12, 24, 36, 48], "ktxt_int": 3, "vtxt": 9, "q": [1, 2, 1, 2]},
    ],
}


def derive():
    plen = CASE["n_img"] // CASE["n_patches"]
    out = []
    for s, st in enumerate(CASE["steps"]):
        prev = CASE["steps"][s - 1] if s > 0 else st
        for p in range(CASE["n_patches"]):
            keys, vals, src = [], [], []
            for r in range(CASE["n_img"]):
                fresh = (r // plen) <= p
                use = st if fresh else prev
                keys.append(use["k_int"][r])
                vals.append(use["v"][r])
                src.append("now" if fresh or s == 0 else "prev")
            keys.append(st["ktxt_int"])
            vals.append(st["vtxt"])
            for i in range(plen):
                q = st["q"][p * plen + i]
                w = [Fraction(a) ** q for a in keys]
                o = sum(wi * v for wi, v in zip(w, vals)) / sum(w)
                out.append({"step": s, "patch": p, "row": i, "image_row_source": src,
                            "o_num": o.numerator, "o_den": o.denominator})
    return out


if __name__ == "__main__":
    doc = dict(CASE)
    doc["citation"] = ("기술 요약: PipeFusion -- 핵심 메커니즘 1 (패치 분할), 2 (stale reuse of step T+1), "
                       "3 (micro-step patch order); 주요 기여 (full attention)")
    doc["expected"] = derive()
    print(json.dumps(doc, indent=1, ensure_ascii=False))
