"""GPU unit test of the tensor-core kernel's four matrix products.

gla_selftest_mma runs each product with the kernel's own shared-memory
layouts, descriptors and TMEM read-back; the result must equal a float64
matmul of the same operands rounded to the operand type.  A layout or
descriptor error shows up here as a permuted or garbled D long before it
would be visible through the full operator.
"""
import ctypes

import numpy as np
import pytest

from recurrent_vision_backbone_only_b200 import build, gla

pytestmark = pytest.mark.gpu


def tf32_round(x):
    """Round-to-nearest to a 10-bit mantissa (tf32), as the bound for the check."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000
    return b.astype(np.uint32).view(np.float32)


CASES = {
    0: ((128, 64), (128, 64), (128, 128), "split", lambda a, b: a @ b.T),
    1: ((128, 64), (128, 64), (64, 64), "f16", lambda a, b: b.T @ a),
    2: ((128, 128), (128, 64), (128, 64), "f16", lambda a, b: a @ b),
    3: ((128, 64), (64, 64), (128, 64), "tf32", lambda a, b: a @ b.T),
}


@pytest.mark.parametrize("kind", [0, 1, 2, 3])
def test_selftest_mma(cuda_ok, kind):
    import torch
    build.build()
    lib = gla.load()
    lib.gla_selftest_mma.argtypes = [ctypes.c_int] + [ctypes.c_void_p] * 4
    lib.gla_selftest_mma.restype = ctypes.c_int
    sa, sb, sd, typ, ref = CASES[kind]
    rng = np.random.default_rng(kind)
    # structured values make index errors visible: row/column dependent magnitudes
    A = (rng.standard_normal(sa) * (1 + np.arange(sa[0])[:, None] / sa[0])).astype(np.float32)
    B = (rng.standard_normal(sb) * (1 + np.arange(sb[1])[None, :] / sb[1])).astype(np.float32)
    dA, dB = torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()
    dD = torch.full(sd, float("nan"), dtype=torch.float32, device="cuda")
    rc = lib.gla_selftest_mma(kind, dA.data_ptr(), dB.data_ptr(), dD.data_ptr(), None)
    assert rc == 0, gla.status_string(rc)
    torch.cuda.synchronize()
    D = dD.cpu().numpy().astype(np.float64)
    if typ == "f16":
        a64, b64 = A.astype(np.float16).astype(np.float64), B.astype(np.float16).astype(np.float64)
        expect = ref(a64, b64)
        np.testing.assert_allclose(D, expect, rtol=1e-5, atol=1e-4)
    elif typ == "split":
        # high + low tf32 parts, three products: ~2^-21 relative to the sum of |terms|
        expect = ref(A.astype(np.float64), B.astype(np.float64))
        scale = ref(np.abs(A).astype(np.float64), np.abs(B).astype(np.float64))
        assert np.max(np.abs(D - expect) / scale) < 2e-6, np.max(np.abs(D - expect) / scale)
    else:
        # operands are rounded to tf32 (nearest) before the product; products are exact in fp32
        expect = ref(tf32_round(A).astype(np.float64), tf32_round(B).astype(np.float64))
        np.testing.assert_allclose(D, expect, rtol=1e-5, atol=1e-4)
