"""Worker for the exhaustive fp32 -> binary16 rounding check (imported by
spawned processes: numpy and the oracle's encodings only)."""
import warnings

import numpy as np

from oracle import encodings as enc


def check_block(first: int, count: int):
    """Compare the oracle's rounding with numpy's float16 cast on the fp32 bit
    patterns first .. first + count - 1.  Returns (mismatches, first few)."""
    x = (np.arange(count, dtype=np.uint64) + np.uint64(first)).astype(np.uint32).view(np.float32)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")              # signalling NaN patterns
        want = x.astype(np.float16).view(np.uint16)
        xd = x.astype(np.float64)
    got = enc.rn16_bits(xd)
    nan = np.isnan(x)
    # NaN payloads are not specified: any binary16 NaN is accepted for a NaN input
    got_nan = ((got & 0x7C00) == 0x7C00) & ((got & 0x03FF) != 0)
    ok = np.where(nan, got_nan, got == want)
    bad = np.nonzero(~ok)[0]
    return int(bad.size), [(int(first + i), int(got[i]), int(want[i])) for i in bad[:4]]
