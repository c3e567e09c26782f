"""Write tests/golden/oracle_small.txt: digests of the oracle's outputs on the
256x256 N(0,1) workload (seed 0), one line per call.

This script calls only the CPU oracle and the seeded input generator.  The file
it writes guards the oracle against unintended changes: a deliberate change of
the oracle's arithmetic regenerates it in the same commit.

    python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from nvfp4_microscaling_quantization_b200 import workloads  # noqa: E402

OUT = os.path.join(HERE, "oracle_small.txt")


def digest_lines():
    wl = workloads.small()
    x = workloads.bf16_bits(wl.tensors()["x"])
    lines = []
    calls = list(wl.calls) + [workloads.Call("x", 1, m, 128) for m in (0, 1, 2, 3, 4)] + \
        [workloads.Call("x", 0, 3, 0), workloads.Call("x", 0, 4, 0), workloads.Call("x", 0, 5, 0),
         workloads.Call("x", 1, 5, 128), workloads.Call("x", 0, 6, 0), workloads.Call("x", 1, 6, 128),
         workloads.Call("x", 0, 7, 0), workloads.Call("x", 1, 7, 128)] + \
        [workloads.Call("x", lay, m, g) for m in (8, 9, 10, 11) for lay, g in ((0, 0), (1, 128))]
    for c in calls:
        codes, scales, gs = oracle.quantize(x, c.layout, c.mode, c.rht_group, wl.seed)
        h = hashlib.sha256(codes.tobytes() + scales.tobytes()).hexdigest()
        lines.append(f"{c.name} gscale={gs.hex()} sha256={h}")
    return lines


if __name__ == "__main__":
    with open(OUT, "w") as f:
        f.write("# oracle digests, 256x256 N(0,1) seed 0; written by tests/golden/make_golden.py\n")
        for line in digest_lines():
            f.write(line + "\n")
    print(open(OUT).read())
