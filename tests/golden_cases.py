"""Loader for the hand-worked fixtures under tests/golden/."""
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def worked_example_v4():
    """Return (fixture dict, batch arrays) for tests/golden/worked_example_v4.json."""
    with open(os.path.join(GOLDEN, "worked_example_v4.json")) as f:
        fx = json.load(f)
    g, cases = fx["gamma"], fx["cases"]
    B = len(cases)
    tgt = np.log(np.array(fx["p"], dtype=np.float64)).astype(np.float32)
    dft = np.log(np.array(fx["q"], dtype=np.float64)).astype(np.float32)
    arrays = dict(
        target=np.ascontiguousarray(np.broadcast_to(tgt, (B,) + tgt.shape)),
        draft=np.ascontiguousarray(np.broadcast_to(dft, (B,) + dft.shape)),
        draft_tokens=np.array([c["draft_tokens"] for c in cases], np.int32).reshape(B, g),
        temperature=np.array([c["T"] for c in cases], np.float32),
        u_accept=np.array([c["u_accept"] for c in cases], np.float32).reshape(B, g),
        u_resample=np.array([c["u_resample"] for c in cases], np.float32),
    )
    return fx, arrays
