"""Decode fused with y = W x (dfw_decode_gemv_lanes) against the oracle.

The GPU decodes the oracle's own encoding and multiplies each tensor of the
scope by its bf16 vector without writing the weights; the oracle decodes
bit-serially and forms y in float64.  The bound is the textbook one for any
order of floating-point summation of exact products (fp32: u = 2^-24):
|y_gpu - y_exact| <= gamma(cols) * sum_j |w_j x_j|, gamma(m) = m u / (1 - m u).
Repeated calls must give identical bits (the summation order is fixed).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import lossless_entropy_coded_canonical_b200 as dfw
import workloads

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dfw.lib()
    dfw.check()


def _encoded_from_oracle(oenc) -> dfw.Encoded:
    t = dfw.Table()
    t.version, t.cap, t.n = 1, 32, oenc.n
    t.total_bits = oenc.total_bits
    t.stream_bytes = oenc.stream.size
    for s in range(256):
        t.len[s] = int(oenc.lengths[s])
    if oenc.n and oenc.total_bits == 0:
        t.n_symbols, t.single_symbol = 1, oenc.single_symbol
    else:
        t.n_symbols = int(np.count_nonzero(oenc.lengths))
    mant = np.zeros(dfw.mant_bytes(oenc.n), np.uint8)
    mant[: oenc.n] = oenc.mant
    return dfw.Encoded(torch.from_numpy(oenc.stream.copy()), torch.from_numpy(mant), t)


def _normal_u16(rng, n, std):
    f = (rng.standard_normal(n) * std).astype(np.float32).view(np.uint32)
    return ((f + 0x7FFF + ((f >> 16) & 1)) >> 16).astype(np.uint16)  # round to nearest even


def gemv_parity(oracle, tensors, cols, seed=0, fast_bits=0):
    """tensors: list of uint16 arrays (row-major, len = rows * cols[i])."""
    rng = np.random.default_rng(seed)
    u = np.concatenate(tensors)
    offs = np.concatenate([[0], np.cumsum([t.size for t in tensors])]).astype(np.uint64)
    oenc = oracle.encode(u, 32)
    enc = _encoded_from_oracle(oenc)
    dl = dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc, fast_bits=fast_bits))
    xs = [_normal_u16(rng, c, 1.0) for c in cols]
    xs_dev = [torch.from_numpy(x.view(np.int16)).cuda() for x in xs]
    ys = dfw.decode_gemv_lanes(dl, xs_dev, cols, tensor_offsets=offs)
    dfw.check()
    ys2 = dfw.decode_gemv_lanes(dl, xs_dev, cols, tensor_offsets=offs)
    dfw.check()
    w_all = oracle.decode(oenc)
    assert np.array_equal(w_all, u)
    for i, c in enumerate(cols):
        rows = tensors[i].size // c
        w = w_all[int(offs[i]): int(offs[i + 1])]
        want = oracle.gemv(w, rows, c, xs[i])
        scale = oracle.gemv_abs(w, rows, c, xs[i])
        got = ys[i].cpu().numpy().astype(np.float64)
        gamma = c * U32 / (1 - c * U32)
        bad = np.nonzero(np.abs(got - want) > gamma * scale + 1e-30)[0]
        assert bad.size == 0, f"tensor {i}: {bad.size} rows off, first {bad[:3]}"
        assert torch.equal(ys[i].view(torch.int32), ys2[i].view(torch.int32)), "not reproducible"
    return ys


def test_gemv_one_matrix(oracle):
    rng = np.random.default_rng(1)
    gemv_parity(oracle, [_normal_u16(rng, 512 * 4096, 0.02)], [4096])


def test_gemv_llama3_block_shapes_scaled(oracle):
    """Seven tensors, one table: q, k, v, o, gate, up with 4096 columns and
    down with 14336, rows scaled down 16x; groups straddle tensor ends."""
    rng = np.random.default_rng(2)
    shapes = [(256, 4096), (64, 4096), (64, 4096), (256, 4096), (896, 4096), (896, 4096), (256, 14336)]
    ts = [_normal_u16(rng, r * c, 0.02) for r, c in shapes]
    gemv_parity(oracle, ts, [c for _, c in shapes], seed=3)


def test_gemv_narrow_and_mixed_columns(oracle):
    """64 and 128 columns put up to 32 rows in one warp's group."""
    rng = np.random.default_rng(4)
    shapes = [(333, 64), (77, 128), (5, 11008), (40, 192)]
    ts = [_normal_u16(rng, r * c, 0.03) for r, c in shapes]
    gemv_parity(oracle, ts, [c for _, c in shapes], seed=5, fast_bits=9)


def test_gemv_heavy_tails_and_zeros(oracle):
    u = np.concatenate([workloads.as_u16_numpy(t)
                        for t in workloads.generate_block(workloads.scaled(workloads.c2(), 1 << 21))])
    u = u[: (u.size // 4096) * 4096]
    gemv_parity(oracle, [u], [4096], seed=6)


def test_gemv_single_exponent(oracle):
    rng = np.random.default_rng(7)
    n = 96 * 1024
    u = ((rng.integers(0, 2, n) << 15) | (119 << 7) | rng.integers(0, 128, n)).astype(np.uint16)
    gemv_parity(oracle, [u], [1024], seed=8)


def test_gemv_rejects_bad_shapes():
    rng = np.random.default_rng(9)
    u = _normal_u16(rng, 64 * 100, 0.02)
    enc = dfw.encode(u)
    dl = dfw.DeviceLanes.upload(enc, dfw.plan_lanes(enc))
    x = torch.zeros(100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dfw.DfwError) as ei:
        dfw.decode_gemv_lanes(dl, [x], [100])  # columns not a multiple of 64
    assert ei.value.status == dfw.EINVAL
    x = torch.zeros(64 + 8, dtype=torch.bfloat16, device="cuda")[8:]  # 16-byte but not 32-byte aligned
    with pytest.raises(dfw.DfwError) as ei:
        dfw.decode_gemv_lanes(dl, [x], [64])
    assert ei.value.status == dfw.EALIGN


def test_gemv_full_size_llama3_block(oracle):
    """One Llama-3-8B-shaped transformer block at full size (218 M weights)."""
    blk = workloads.c5()[1]
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)]
    ts = [workloads.as_u16_numpy(t) for t in workloads.generate_block(blk, "cuda")]
    assert [t.size for t in ts] == [r * c for r, c in shapes]
    gemv_parity(oracle, ts, [c for _, c in shapes], seed=10)
