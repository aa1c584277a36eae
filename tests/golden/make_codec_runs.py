"""Write the oracle's FP8 encoding of every fp32 bit pattern as runs.

For each format the oracle encoder is evaluated on all 2^32 fp32 bit patterns
(0x00000000 .. 0xFFFFFFFF).  The output is stored run-length encoded: one line
``<first bit pattern, hex> <code, hex>`` wherever the code changes.  The files
let a GPU test compare the device codec with the oracle on every input without
re-running the (slow) oracle there.  Only ``oracle`` is called here.

Usage:  python tests/golden/make_codec_runs.py
"""
from __future__ import annotations

import os
import sys
from concurrent.futures import ThreadPoolExecutor

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

CHUNK = 1 << 24
NAMES = {oracle.E4M3: "e4m3", oracle.E5M2: "e5m2"}


def runs_of(fmt: int, threads: int) -> list:
    starts = list(range(0, 1 << 32, CHUNK))

    def one(first):
        c = oracle.encode_bits_range(fmt, first, CHUNK)
        change = np.flatnonzero(np.diff(c)) + 1
        return first, int(c[0]), [(first + int(i), int(c[i])) for i in change]

    out = []
    with ThreadPoolExecutor(threads) as ex:
        for first, c0, ch in ex.map(one, starts):
            if not out or out[-1][1] != c0:
                out.append((first, c0))
            out.extend(ch)
    return out


def path_for(fmt: int) -> str:
    return os.path.join(HERE, "codec_runs_%s.txt" % NAMES[fmt])


def main() -> None:
    threads = len(os.sched_getaffinity(0))
    for fmt in (oracle.E4M3, oracle.E5M2):
        runs = runs_of(fmt, threads)
        with open(path_for(fmt), "w") as f:
            f.write("# oracle encoding (RNE, satfinite, NaN->0x7F) of all 2^32 fp32 bit patterns,\n")
            f.write("# run-length encoded: <first bit pattern> <code>; written by make_codec_runs.py\n")
            for first, code in runs:
                f.write("%08x %02x\n" % (first, code))
        print(NAMES[fmt], len(runs), "runs")


if __name__ == "__main__":
    main()
