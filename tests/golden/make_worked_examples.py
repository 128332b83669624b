"""Writes the hand-derived worked examples in this folder.

The pages print no numeric example for Slim attention, so these fixtures are
closed forms derived by hand (the "derivation" field of each file) from the
definitions in the Slim Attention article, section "K-Cache is All You Need":
W_KV = W_K^(-1)·W_V, V = K·W_KV, and a generation step that scores q against
the cached K, takes a softmax and applies it to the values. Scores are chosen
to differ by ln 3 (softmax 3/4, 1/4) or to tie (1/2, 1/2), so every expected
value is a short rational number. Nothing here calls any implementation.
Run: python tests/golden/make_worked_examples.py
"""
import json
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
CITE = ("Slim Attention article (localbendi.com/xw/1329462), section 'K-Cache is All You Need': "
        "W_KV = W_K^(-1)*W_V, V = K*W_KV, generation step = scores of q against cached K, softmax, then values.")

ONE_HEAD = {
    "citation": CITE,
    "derivation": ("H=1, d=d_h=2. k0 = x0*W_K = [2,0], k1 = [0,1]. q = [ln(3)/sqrt(2), 0] so "
                   "scores/sqrt(d_h) = [ln 3, 0] and softmax = [3/4, 1/4]. v0 = x0*W_V = [1,2], "
                   "v1 = [3,4]. o = 3/4*v0 + 1/4*v1 = [3/2, 5/2]. W_KV = diag(1/2,1)*W_V = [[1/2,1],[3,4]]."),
    "H": 1,
    "X": [[1, 0], [0, 1]],
    "W_K": [[2, 0], [0, 1]],
    "W_V": [[1, 2], [3, 4]],
    "q": [math.log(3) / math.sqrt(2), 0.0],
    "expected_W_KV": [[0.5, 1.0], [3.0, 4.0]],
    "expected_softmax": [[0.75, 0.25]],
    "expected_o": [1.5, 2.5],
}

TWO_HEADS = {
    "citation": CITE,
    "derivation": ("H=2, d=4, d_h=2, head h owns columns [2h,2h+2). W_K = diag(2,1,1,1). k0 = [2,0,1,0], "
                   "k1 = [0,1,0,1]. Head 0: q[0:2] = [ln(3)/sqrt(2), 0] gives scaled scores [ln 3, 0], "
                   "softmax [3/4,1/4]. Head 1: q[2:4] = [1,1] gives scaled scores [1/sqrt(2), 1/sqrt(2)], "
                   "softmax [1/2,1/2]. W_V rows are 1..16 row-major; v0 = W_V[0]+W_V[2] = [10,12,14,16], "
                   "v1 = W_V[1]+W_V[3] = [18,20,22,24]. o[0:2] = 3/4*[10,12] + 1/4*[18,20] = [12,14]; "
                   "o[2:4] = ([14,16]+[22,24])/2 = [18,20]."),
    "H": 2,
    "X": [[1, 0, 1, 0], [0, 1, 0, 1]],
    "W_K": [[2, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 0], [0, 0, 0, 1]],
    "W_V": [[1, 2, 3, 4], [5, 6, 7, 8], [9, 10, 11, 12], [13, 14, 15, 16]],
    "q": [math.log(3) / math.sqrt(2), 0.0, 1.0, 1.0],
    "expected_W_KV": [[0.5, 1.0, 1.5, 2.0], [5, 6, 7, 8], [9, 10, 11, 12], [13, 14, 15, 16]],
    "expected_softmax": [[0.75, 0.25], [0.5, 0.5]],
    "expected_o": [12.0, 14.0, 18.0, 20.0],
}

if __name__ == "__main__":
    for name, obj in [("worked_two_rows_one_head.json", ONE_HEAD), ("worked_two_rows_two_heads.json", TWO_HEADS)]:
        with open(os.path.join(HERE, name), "w") as f:
            json.dump(obj, f, indent=1)
