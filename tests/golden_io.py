"""Readers for the hand-derived fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                yield line.split()


def fp16_rounding():
    return [(float.fromhex(a), int(b, 16)) for a, b in _lines("fp16_rounding.txt")]


def quant_groups(G=128):
    """-> list of dicts: name, v (fp16 [G]), s bits, z, q [G], w {index: bits}."""
    cases, cur = [], None
    for tok in _lines("quant_groups.txt"):
        if tok[0] == "case":
            cur = {"name": tok[1], "set": {}, "q": {}, "w": {}}
        elif tok[0] == "fill":
            cur["fill"] = float.fromhex(tok[1])
        elif tok[0] == "set":
            cur["set"][int(tok[1])] = float.fromhex(tok[2])
        elif tok[0] == "s":
            cur["s"] = int(tok[1], 16)
        elif tok[0] == "z":
            cur["z"] = int(tok[1])
        elif tok[0] == "q":
            cur["q"][tok[1]] = int(tok[2])
        elif tok[0] == "w":
            cur["w"][tok[1]] = int(tok[2], 16)
        elif tok[0] == "end":
            v = np.full(G, cur["fill"], np.float64)
            for i, x in cur["set"].items():
                v[i] = x
            h = v.astype(np.float16)
            assert (h.astype(np.float64) == v).all(), cur["name"]  # fixtures hold exact fp16 values
            q = np.full(G, cur["q"].get("fill", -1), np.int64)
            for i, n in cur["q"].items():
                if i != "fill":
                    q[int(i)] = n
            w = {}
            for i, b in cur["w"].items():
                if i == "fill":
                    for j in range(G):
                        if j not in cur["set"]:
                            w[j] = b
                else:
                    w[int(i)] = b
            cases.append({"name": cur["name"], "v": h, "s": cur["s"], "z": cur["z"], "q": q, "w": w})
            cur = None
    return cases


def packed_words():
    """-> list of (N, K, n, k, qvalue, word_index, word_value, G); G is 128 where
    the line gives none."""
    out = []
    for t in _lines("packed_words.txt"):
        v = [int(x, 0) for x in t]
        out.append(tuple(v + [128] * (8 - len(v))))
    return out
