"""quant4_pack / quant4_unpack on the GPU against the oracle codec: codes and
scales bit for bit, for both codebooks (linear square and dynamic tree)."""
import numpy as np
import pytest
import torch

from oracle import shampoo4_oracle as O
from gpu_helpers import cuda_f32

pytestmark = pytest.mark.gpu


def _api():
    from bit_quantized_shampoo_b200 import api
    return api


BOOKS = {"linear_square": O.LINEAR_SQUARE, "dynamic_tree": O.DYNAMIC_TREE}


def _check(xs, book="linear_square"):
    api = _api()
    cbk = BOOKS[book]
    tx = [cuda_f32(x) for x in xs]
    codes, scales = api.quant4_pack(tx, codebook=book)
    torch.cuda.synchronize()
    for x, c, s in zip(xs, codes, scales):
        oc, os_ = O.quantize(x, codebook=cbk)
        gc, gs = c.cpu().numpy(), s.cpu().numpy()
        assert np.array_equal(gc, oc), (x.size, np.nonzero(gc != oc)[0][:8])
        assert np.array_equal(gs.view(np.uint32), os_.view(np.uint32)) or \
            np.array_equal(np.isnan(gs), np.isnan(os_)) and np.array_equal(gs[~np.isnan(gs)], os_[~np.isnan(os_)])
    back = api.quant4_unpack(codes, scales, [x.size for x in xs], codebook=book)
    torch.cuda.synchronize()
    for x, c, s, b in zip(xs, codes, scales, back):
        ref = O.dequantize(c.cpu().numpy(), s.cpu().numpy(), x.size, codebook=cbk)
        got = b.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)) or \
            (np.array_equal(np.isnan(got), np.isnan(ref)) and np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)]))


@pytest.mark.parametrize("book", list(BOOKS))
def test_ragged_sizes_one_batch(book):
    rng = np.random.default_rng(11)
    sizes = [1, 2, 7, 8, 63, 64, 65, 127, 128, 4095, 4096, 4097, 8193, 16383, 16384, 16385, 100003, 1 << 18]
    _check([rng.standard_normal(n).astype(np.float32) for n in sizes], book)


@pytest.mark.parametrize("book", list(BOOKS))
def test_eigenvector_shaped_inputs(book):
    from bit_quantized_shampoo_b200.workloads import u_like
    xs = [u_like(d, 100 + d)[0].ravel() for d in (64, 147, 576, 768, 1024)]
    _check(xs, book)


@pytest.mark.parametrize("book", list(BOOKS))
def test_special_values(book):
    rng = np.random.default_rng(12)
    t = O.thresholds_f32(BOOKS[book])
    blocks = []
    blocks.append(np.zeros(64, np.float32))                                   # zero block
    blocks.append((rng.standard_normal(64) * 1e-39).astype(np.float32))      # subnormal scale
    b = (rng.standard_normal(64) * 1e-30).astype(np.float32); b[0] = 1.0     # tiny quotients
    blocks.append(b)
    b = np.concatenate([t, -t, [1.0], np.zeros(64 - 31)]).astype(np.float32)  # exact ties, absmax 1
    blocks.append(b[:64])
    b = rng.standard_normal(64).astype(np.float32); b[5] = -np.abs(b).max(); b[9] = -b[5]   # +-absmax tie
    blocks.append(b)
    b = np.ones(64, np.float32); b[3] = np.nan; blocks.append(b)
    b = np.ones(64, np.float32); b[4] = np.inf; b[7] = -np.inf; blocks.append(b)
    b = (rng.standard_normal(64) * 3e38).astype(np.float32); blocks.append(b)   # near overflow
    b = (rng.standard_normal(64)).astype(np.float32) * np.float32(2.0 ** -126); blocks.append(b)
    _check([np.concatenate(blocks).astype(np.float32)], book)
    _check(blocks, book)


@pytest.mark.parametrize("book", list(BOOKS))
def test_shared_divisor_division_matches_ieee_over_exponent_range(book):
    rng = np.random.default_rng(13)
    xs = []
    for e in range(-140, 120, 7):
        x = rng.standard_normal(64 * 97).astype(np.float32) * np.float32(2.0 ** e)
        m = rng.integers(-60, 1, size=x.size).astype(np.float32)
        xs.append((x * np.exp2(m)).astype(np.float32))
    _check(xs, book)


@pytest.mark.parametrize("book", list(BOOKS))
def test_signed_bucket_path(book):
    """Whole warps (4 blocks of 64) with scales in [2^-60, 1] and no ragged
    end take the signed-bucket decision; one block out of range sends its
    warp to the general one.  Ties: thresholds times a power-of-two scale
    equal to the block's absmax."""
    rng = np.random.default_rng(16)
    t = O.thresholds_f32(BOOKS[book])
    xs = []
    for s in (1.0, 0.5, 2.0 ** -20, 2.0 ** -60, 2.0 ** -59, 0.7, 0.999999):
        x = (rng.uniform(-1, 1, 64 * 4 * 33) * s).astype(np.float32)
        x[::64] = np.float32(s)                               # absmax exactly s
        xs.append(x)
    for p in (0, -3, -40, -60):
        s = np.float32(2.0 ** p)
        blk = np.concatenate([t * s, -t * s, [s], np.zeros(64 - 31)]).astype(np.float32)[:64]
        xs.append(np.tile(blk, 4 * 9))
    x = (rng.uniform(-1, 1, 64 * 4 * 16) * 0.3).astype(np.float32)
    x[64 * 4 * 5 + 17] = 1.5                                  # one warp to the general path
    x[64 * 4 * 9 + 3] = np.float32(2.0 ** -61)                # below 2^-60: general path
    x[64 * 4 * 9 + 4:64 * 4 * 9 + 64] = 0.0
    x[64 * 4 * 9:64 * 4 * 9 + 3] = 0.0
    xs.append(x)
    _check(xs, book)
    _check([np.concatenate(xs)], book)


@pytest.mark.parametrize("book", list(BOOKS))
def test_large_tensor_unit_scale_sampled(book):
    """512 MiB with block scales below 1 (the signed-bucket path), sampled."""
    api = _api()
    n = (1 << 27) + 37
    g = torch.Generator(device="cuda").manual_seed(6)
    x = torch.randn(n, device="cuda", generator=g) * 0.125
    codes, scales = api.quant4_pack([x], codebook=book)
    torch.cuda.synchronize()
    rng = np.random.default_rng(17)
    nb = (n + 63) // 64
    for b in list(rng.integers(0, nb, 64)) + [nb - 1]:
        lo, hi = 64 * int(b), min(64 * int(b) + 64, n)
        oc, os_ = O.quantize(x[lo:hi].cpu().numpy(), codebook=BOOKS[book])
        assert scales[0][int(b)].item() == os_[0]
        assert np.array_equal(codes[0][lo // 2:(hi + 1) // 2].cpu().numpy(), oc)


def test_misaligned_pointers():
    api = _api()
    rng = np.random.default_rng(14)
    n = 1000
    x = rng.standard_normal(n + 3).astype(np.float32)
    tx = cuda_f32(x)[1:n + 1]                      # 4-byte but not 16-byte aligned
    cbuf = torch.empty(n // 2 + 3, dtype=torch.uint8, device="cuda")
    sbuf = torch.empty((n + 63) // 64 + 1, dtype=torch.float32, device="cuda")
    codes, scales = api.quant4_pack([tx], codes=[cbuf[1:1 + n // 2]], scales=[sbuf[1:]])
    torch.cuda.synchronize()
    oc, os_ = O.quantize(x[1:n + 1])
    assert np.array_equal(codes[0].cpu().numpy(), oc)
    assert np.array_equal(scales[0].cpu().numpy()[:os_.size], os_)


def test_large_tensor_sampled():
    api = _api()
    n = (1 << 27) + 37                            # 512 MiB of fp32, ragged tail
    g = torch.Generator(device="cuda").manual_seed(5)
    x = torch.randn(n, device="cuda", generator=g)
    codes, scales = api.quant4_pack([x])
    torch.cuda.synchronize()
    rng = np.random.default_rng(15)
    nb = (n + 63) // 64
    for b in list(rng.integers(0, nb, 64)) + [nb - 1]:
        lo, hi = 64 * int(b), min(64 * int(b) + 64, n)
        xb = x[lo:hi].cpu().numpy()
        oc, os_ = O.quantize(xb)
        assert scales[0][int(b)].item() == os_[0]
        gc = codes[0][lo // 2:(hi + 1) // 2].cpu().numpy()
        assert np.array_equal(gc, oc)
