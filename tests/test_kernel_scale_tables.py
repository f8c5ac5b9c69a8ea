"""The quantizer kernels take a BF16 group's scale s = fl32(amax/448) and its reciprocal
fl32(1/s) from two 128-entry tables indexed by amax's 7-bit mantissa, scaled by a power
of two. This test re-derives the tables from their definition, checks the literals in
the kernel source against them, and proves the identity for every normal BF16 amax with
exponent >= -71 (smaller amax take the division path in the kernel)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "fp8_block_scaled_08_b200", "csrc", "fp8q_quant.cu")


def _table(name):
    txt = open(SRC).read()
    body = re.search(r"__constant__ float %s\[128\] = \{(.*?)\};" % name, txt, re.S).group(1)
    vals = [float.fromhex(t.strip().rstrip("f")) for t in body.split(",") if t.strip()]
    return np.array(vals, np.float32)


def test_tables_match_their_definition():
    ts = _table("kScaleMant")
    tr = _table("kRecipMant")
    assert ts.shape == (128,) and tr.shape == (128,)
    for i in range(128):
        want = np.float32(np.float32(1 + i / 128.0) / np.float32(7.0))
        assert ts[i] == want, i
        assert tr[i] == np.float32(np.float32(1.0) / want), i


def test_power_of_two_scaling_identity_all_bf16():
    ts = _table("kScaleMant").view(np.uint32).astype(np.int64)
    tr = _table("kRecipMant").view(np.uint32).astype(np.int64)
    b = np.arange(0x0080, 0x7F80, dtype=np.int64)          # normal positive BF16
    e = ((b >> 7) & 0xFF) - 127
    b = b[e > -72]
    e = e[e > -72]
    i = b & 0x7F
    amax = (b.astype(np.uint32) << 16).view(np.float32)
    s_true = (amax / np.float32(448.0)).astype(np.float32)
    r_true = (np.float32(1.0) / s_true).astype(np.float32)
    s_tab = (ts[i] + ((e - 6) << 23)).astype(np.uint32).view(np.float32)
    r_tab = (tr[i] + ((6 - e) << 23)).astype(np.uint32).view(np.float32)
    assert np.array_equal(s_tab.view(np.uint32), s_true.view(np.uint32))
    assert np.array_equal(r_tab.view(np.uint32), r_true.view(np.uint32))
    assert len(b) > 25000
