"""Philox4x32-10 words from Triton's own Philox implementation, run on the
CPU through Triton's interpreter.  Used only as an independent library
reference for the oracle's Philox; prints JSON to stdout.

usage: TRITON_INTERPRET=1 python philox_triton_ref.py '<json list of [seed, c0, c1, c2, c3]>'
"""
import json
import os
import sys

os.environ.setdefault("TRITON_INTERPRET", "1")

import torch  # noqa: E402
import triton  # noqa: E402
import triton.language as tl  # noqa: E402


@triton.jit
def _philox_kernel(out_ptr, ctr_ptr, seed):
    # counters are loaded as int32 bit patterns so that every word has the
    # same 32-bit type whatever its value
    o = tl.arange(0, 1)
    c0 = tl.load(ctr_ptr + 0 + o)
    c1 = tl.load(ctr_ptr + 1 + o)
    c2 = tl.load(ctr_ptr + 2 + o)
    c3 = tl.load(ctr_ptr + 3 + o)
    a, b, c, d = tl.philox(seed, c0, c1, c2, c3)
    tl.store(out_ptr + 0 + tl.arange(0, 1), a)
    tl.store(out_ptr + 1 + tl.arange(0, 1), b)
    tl.store(out_ptr + 2 + tl.arange(0, 1), c)
    tl.store(out_ptr + 3 + tl.arange(0, 1), d)


def main():
    cases = json.loads(sys.argv[1])
    res = []
    for seed, c0, c1, c2, c3 in cases:
        out = torch.zeros(4, dtype=torch.int32)
        ctr = torch.tensor([c0, c1, c2, c3], dtype=torch.int64).to(torch.int32)
        _philox_kernel[(1,)](out, ctr, seed)
        res.append([v & 0xFFFFFFFF for v in out.tolist()])
    print(json.dumps(res))


if __name__ == "__main__":
    main()
