"""Writes tests/golden/lloyd_max_n01.txt: the fixed codebooks, from the oracle only.

The 2-bit codebook is the 4-level Lloyd-Max quantiser of N(0,1), whose values
the OmniKVQuant workload description prints as +-0.4528, +-1.5104; the 4-bit one
is the 16-level quantiser of the same source (used for the K4/V4 setting of the
paper's bit-width sweep, paperpeel.com section 3.3, Table 5). Each level is
stored as the fp32 rounding of the fp64 fixed point, as 8 hex digits (the bit
pattern) followed by the decimal value.

Run:  python tests/golden/write_lloyd_max.py
"""
import os
import struct
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.codebook import lloyd_max_gaussian  # noqa: E402


def f32_bits(x: float) -> str:
    return "%08x" % struct.unpack("<I", struct.pack("<f", x))[0]


def main():
    lines = ["# Lloyd-Max levels for N(0,1), fp32; written by tests/golden/write_lloyd_max.py",
             "# levels <L>: then one line per level: <fp32 hex bits> <decimal>"]
    for L in (4, 16):
        lines.append("levels %d" % L)
        for c in lloyd_max_gaussian(L):
            c32 = struct.unpack("<f", struct.pack("<f", c))[0]
            lines.append("%s %.9g" % (f32_bits(c32), c32))
    with open(os.path.join(HERE, "lloyd_max_n01.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
