"""Write tests/golden/tiny_wave.txt from the oracle alone.

Workload: the tiny wave (2 heads x 64, 3 chunks x 32 tokens laid out as
2 frames x 4 x 4, no history), seed 0, round 0, positions derived from the
round.  The file stores, for a fixed set of (row, head) pairs, the oracle's
attention output (fp64, %.17g) and log-sum-exp, plus the bf16 bits of the
appended q/k rows.  It is a regression fixture for the oracle: regenerate it
only with a change whose commit message names the passage that justifies it.

    python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from chunk_causal_dit_b200 import inputs as wi  # noqa: E402

ROWS = [0, 1, 31, 32, 33, 47, 63, 64, 80, 95]


def compute():
    w = wi.WORKLOADS["tiny"]
    x = wi.wave_inputs(w, seed=0)
    pos = oracle.positions(0, w.n_wave, w.F, w.gh, w.gw)
    qo, ko, vo = oracle.append(wi.bits(x.q), wi.bits(x.k), wi.bits(x.v), pos,
                               x.gamma_q.numpy(), x.gamma_k.numpy())
    cache = oracle.OracleCache(w.L)
    cache.put_wave(0, ko, vo)
    rows = np.repeat(ROWS, w.H)
    heads = np.tile(np.arange(w.H), len(ROWS))
    o, lse = oracle.round_attention(cache, 0, w.n_wave, w.n_hist, qo, rows, heads)
    return w, qo, ko, rows, heads, o, lse


def main(path=os.path.join(HERE, "tiny_wave.txt")):
    w, qo, ko, rows, heads, o, lse = compute()
    with open(path, "w") as f:
        f.write("# tiny wave, seed 0, round 0; written by tests/golden/make_golden.py (oracle only)\n")
        for n, h in ((0, 0), (40, 1), (95, 1)):
            f.write("qk %d %d %s %s\n" % (n, h, ",".join("%04x" % b for b in qo[n, h]),
                                          ",".join("%04x" % b for b in ko[n, h])))
        for i in range(len(rows)):
            f.write("o %d %d %.17g %s\n" % (rows[i], heads[i], lse[i],
                                            ",".join("%.17g" % t for t in o[i])))


if __name__ == "__main__":
    main()
