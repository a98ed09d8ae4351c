"""Write tests/golden/tiny_oracle.txt: the oracle's step outputs on the
seeded ``tiny`` workload (4 requests, cached lengths {17,64,100,255},
Hq 8 / Hkv 2, d 64, page 16, RoPE base 1e4).

Calls only the generator and ``oracle/``.  The fixture is a regression pin:
any later change to the oracle's arithmetic shows up as a diff here and has
to be justified by the passage it follows.

    python tests/golden/make_golden.py
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from tests._util import oracle_step  # noqa: E402
from paged_kv_flight_b200 import workloads  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.txt")


def rows():
    w = workloads.make("tiny")
    h, out, st = oracle_step(w)
    assert st == 0
    lines = []
    for b in range(w.batch):
        for hh in range(w.Hq):
            vals = " ".join(repr(float(v)) for v in out[b, hh, :4])
            lines.append(f"out {b} {hh} {vals}")
    for b, L in enumerate(w.seq_lens):
        page = int(w.block_tables[b, L // w.P])
        for kvh in range(w.Hkv):
            kb = " ".join(f"{int(x):04x}" for x in h["k_pool"][page, kvh, L % w.P, :8])
            lines.append(f"k {b} {kvh} {kb}")
    return lines


if __name__ == "__main__":
    with open(OUT, "w") as f:
        f.write("# oracle outputs on the seeded tiny workload, written by make_golden.py\n")
        f.write("# out b h <first 4 of d, fp64>; k b kvh <first 8 appended K bf16 bits>\n")
        f.write("\n".join(rows()) + "\n")
    print(OUT)
