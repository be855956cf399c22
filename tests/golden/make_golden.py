"""Write tests/golden/codebooks.json from the oracle alone.

The pages print no worked numeric example, so the stored values here are the oracle's own
Lloyd-Max codebooks (fp64, 17 significant digits) for every supported dimension and bit width.
They are pinned by tests/test_oracle_codebook.py and serve as a stable table that the library's
host-side codebook is compared with.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import codebook  # noqa: E402


def main():
    table = {}
    for d in (8, 16, 32, 64, 128, 256, 512, 1024):
        for b in (1, 2, 3, 4):
            c, t = codebook.codebook(d, b)
            table[f"{d}/{b}"] = {"centroids": [repr(float(v)) for v in c],
                                 "thresholds": [repr(float(v)) for v in t],
                                 "mse_per_coord": repr(codebook.mse_per_coord(d, c, t))}
    with open(os.path.join(HERE, "codebooks.json"), "w") as f:
        json.dump({"source": "oracle.codebook.lloyd_max (fp64); density from the juejin page "
                             "'谷歌 TurboQuant 深度拆解', 第六部分 '为什么随机旋转这么关键'",
                   "codebooks": table}, f, indent=1)


if __name__ == "__main__":
    main()
