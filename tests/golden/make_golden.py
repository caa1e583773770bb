"""Write tests/golden/tiny_oracle.txt from the CPU oracle alone.

The pages print no worked numeric example for this operation, so the stored
values here are the oracle's own output on the seeded "tiny" workload (B=2,
Hq=8, Hkv=2, D=128, 16-token pages, lengths 37 and 300).  They guard the
oracle against unintended changes; they are not an independent pin (the pins
live in tests/oracle_pins.py).  Run:  python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from fp8_paged_decode_b200 import workloads as W  # noqa: E402


def main():
    wl = W.make_workload("tiny")
    out, lse = oracle.decode_workload(wl, threads=1)
    path = os.path.join(HERE, "tiny_oracle.txt")
    with open(path, "w") as f:
        f.write("# oracle output on the seeded tiny workload; written by make_golden.py\n")
        f.write(f"# k_scale={wl.k_scale!r} v_scale={wl.v_scale!r} sm_scale={wl.sm_scale!r}\n")
        f.write("# b h lse out[0] out[1] out[63] out[127] sum(out)\n")
        for b in range(wl.B):
            for h in range(wl.Hq):
                o = out[b, h]
                f.write(f"{b} {h} {float(lse[b, h])!r} {float(o[0])!r} {float(o[1])!r} {float(o[63])!r} {float(o[127])!r} {float(o.sum())!r}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
