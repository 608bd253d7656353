"""The kernels' native sm_100a conversions against the oracle's encoders,
written from the OCP format definitions, over EVERY binary32 bit pattern
(2^32 inputs per format; NaN inputs are left out of the e2m1 comparison: the
format has no NaN and the code a NaN takes is unspecified, which the oracle
marks with 0xFF).  This pins the hardware `cvt ... satfinite` used by
the dispatch and combine-backward kernels to the oracle bit for bit.  Formats
2 and 3 pin the kernels' division-free MX exponent (qmax 448 and 6) to the
oracle's frexp-based definition on every finite block maximum."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import combine_ep_dispatch_04_b200 as ep
import oracle

pytestmark = pytest.mark.gpu

CHUNK = 1 << 28


def _oracle_chunk(fmt, start, n):
    if fmt == 0:
        return oracle.e4m3_encode_bits(start, n)
    if fmt == 1:
        return oracle.e2m1_encode_bits(start, n)
    return oracle.mx_exponent_bits(start, n, 448.0 if fmt == 2 else 6.0)


@pytest.mark.parametrize("fmt", [0, 1, 2, 3], ids=["e4m3", "e2m1", "e8m0_448", "e8m0_6"])
def test_cvt_exhaustive(fmt):
    out = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
    pieces = 16
    with ThreadPoolExecutor(8) as pool:  # the oracle's C loops release the GIL
        for c in range(0, 1 << 32, CHUNK):
            futs = [pool.submit(_oracle_chunk, fmt, c + i * (CHUNK // pieces), CHUNK // pieces)
                    for i in range(pieces)]
            ep.ep_cvt_sweep(fmt, c, out)
            got = out.cpu().numpy()
            want = np.concatenate([f.result() for f in futs])
            if fmt >= 1:  # e2m1: NaN has no specified code; e8m0: non-finite
                got = np.where(want == 0xFF, 0xFF, got)  # patterns are not block maxima
            bad = np.nonzero(got != want)[0]
            assert bad.size == 0, [(hex(c + int(i)), int(got[i]), int(want[i])) for i in bad[:8]]
