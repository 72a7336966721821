"""GPU unit tests of the tensor-core kernel's matrix products and its TMA gather.

gla_selftest_chunk runs each product of the 64-token-chunk kernel with the kernel's own
shared-memory layouts, descriptors and TMEM accesses (M = 64 tiles in 16-lane halves,
16-bit operands packed in TMEM); the result must equal a float64 matmul of the same
operands rounded the way the kernel rounds them.  gla_selftest_gather fetches permuted
rows with the kernel's tile::gather4 path and returns the tile.  A layout, packing or
descriptor error shows up here as a permuted or garbled result before it can hide in the
full operator.
"""
import numpy as np
import pytest

from recurrent_vision_backbone_only_b200 import build, gla

pytestmark = pytest.mark.gpu


def bf16_round(x):
    """Round-to-nearest-even to bfloat16 (8-bit mantissa), returned as float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def split_bf16(x):
    hi = bf16_round(x)
    lo = bf16_round(x.astype(np.float32) - hi)
    return hi.astype(np.float64), lo.astype(np.float64)


def split_product(a, b, op):
    """The kernel's three-term split product: hi*hi + hi*lo + lo*hi (lo*lo dropped)."""
    ah, al = split_bf16(a)
    bh, bl = split_bf16(b)
    return op(ah, bh) + op(ah, bl) + op(al, bh)


def structured(rng, shape, axis):
    """Normal values whose magnitude grows along `axis`: index errors change the result."""
    ramp = 1 + np.arange(shape[axis]) / shape[axis]
    ramp = ramp[:, None] if axis == 0 else ramp[None, :]
    return (rng.standard_normal(shape) * ramp).astype(np.float32)


@pytest.fixture(scope="module")
def lib(cuda_ok):
    build.build()
    return gla.load()


@pytest.mark.parametrize("d,kind", [(d, k) for d in (64, 128) for k in range(4)] + [(64, 4)])
def test_selftest_chunk_products(lib, d, kind):
    import torch
    rng = np.random.default_rng(10 * kind + d)
    shapes = {0: ((64, d), (64, d), (64, 64)), 1: ((64, d), (64, d), (d, d)),
              2: ((64, 64), (64, d), (64, d)), 3: ((64, d), (d, d), (64, d)),
              4: ((64, 64), (64, d), (64, d))}
    sa, sb, sd = shapes[kind]
    A = structured(rng, sa, 0)
    B = structured(rng, sb, 1)
    dA, dB = torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()
    dD = torch.full(sd, float("nan"), dtype=torch.float32, device="cuda")
    rc = lib.gla_selftest_chunk(d, kind, dA.data_ptr(), dB.data_ptr(), dD.data_ptr(), None)
    assert rc == 0, gla.status_string(rc)
    torch.cuda.synchronize()
    D = dD.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(D))
    if kind in (1, 2, 4):
        a16 = A.astype(np.float16).astype(np.float64)
        b16 = B.astype(np.float16).astype(np.float64)
        expect = a16.T @ b16 if kind == 1 else a16 @ b16
        np.testing.assert_allclose(D, expect, rtol=1e-5, atol=1e-4)
    else:
        op = (lambda x, y: x @ y.T) if kind == 0 else (lambda x, y: x @ y)
        expect = split_product(A, B, op)
        scale = op(np.abs(A).astype(np.float64), np.abs(B).astype(np.float64))
        err = np.max(np.abs(D - expect) / scale)
        assert err < 1e-6, err


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("gh,gw,direction,chunk", [(5, 70, 0, 3), (5, 70, 1, 3), (70, 5, 2, 3),
                                                   (70, 5, 3, 1), (9, 7, 1, 8), (9, 7, 2, 6),
                                                   (9, 7, 3, 6)])
def test_selftest_load_chunk_tiles(lib, d, gh, gw, direction, chunk):
    # the five tiles of one chunk, fetched with the kernel's TMA boxes: tile row i must hold the
    # token at the spatial index the kernel reports for it (rows past the chunk are not checked)
    import torch
    B, H = 2, 3
    L = gh * gw
    rng = np.random.default_rng(gh * 100 + gw + direction)
    src = [rng.standard_normal((B, L, H, d)).astype(np.float16) for _ in range(5)]
    dsrc = [torch.from_numpy(x).cuda() for x in src]
    out = torch.full((5, 64, d), float("nan"), dtype=torch.float32, device="cuda")
    info = torch.full((65,), -2, dtype=torch.int32, device="cuda")
    rc = lib.gla_selftest_load(*[t.data_ptr() for t in dsrc], B, H, gh, gw, d, direction, chunk,
                               out.data_ptr(), info.data_ptr(), None)
    assert rc == 0, gla.status_string(rc)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    inf = info.cpu().numpy()
    n = int(inf[0])
    assert 0 < n <= 64
    spatial = inf[1:1 + n]
    assert np.all(spatial >= 0) and np.all(inf[1 + n:] == -1)
    # the chunk's positions, in scan order, are the direction's map of consecutive scan positions
    line_len = gw if direction < 2 else gh
    pieces = -(-line_len // 64)
    clen = -(-line_len // pieces)
    line, piece = divmod(chunk, pieces)
    pos = line * line_len + piece * clen + np.arange(n)
    if direction == 0:
        expect = (pos // gw) * gw + pos % gw
    elif direction == 1:
        expect = (pos // gw) * gw + gw - 1 - pos % gw
    elif direction == 2:
        expect = (pos % gh) * gw + pos // gh
    else:
        expect = (gh - 1 - pos % gh) * gw + pos // gh
    # tile rows hold the chunk in increasing spatial order; R->L and B->T scan them backwards
    np.testing.assert_array_equal(np.sort(expect), spatial)
    for x in range(5):
        np.testing.assert_array_equal(o[x, :n], src[x][0, spatial, 0].astype(np.float32))
