"""The streaming decode kernel's bit-level reading of packed weights, checked on
the CPU against the oracle's own encoders (no GPU): which bits of a 32-bit word
hold which code, and the byte arithmetic that turns codes into DP2A operands.
The kernel's operations are restated here in numpy (PRMT in its generic form,
IADD3, AND/shift planes); a change in either side's packing fails these tests.
"""
import re
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle

KERNEL = Path(__file__).resolve().parents[1] / "quantized_matmul_03_b200" / "csrc" / "gemv_fast.cu"

# Twice the E2M1 magnitudes of codes 0..7, as two little-endian PRMT table words.
E2M1_LO, E2M1_HI = 0x03020100, 0x0C080604


def test_the_kernel_uses_this_table():
    m = re.search(r"kE2m1Lo = 0x([0-9A-Fa-f]+)u, kE2m1Hi = 0x([0-9A-Fa-f]+)u", KERNEL.read_text())
    assert m and (int(m.group(1), 16), int(m.group(2), 16)) == (E2M1_LO, E2M1_HI)


def prmt(a, b, c):
    """PRMT generic form on uint32 arrays: byte n of the result is byte
    (c >> 4n) & 7 of {b:a}, or that byte's sign replicated when bit 3 of the
    selector nibble is set."""
    a, b, c = (np.asarray(t, dtype=np.uint64) for t in (a, b, c))
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    out = np.zeros(np.broadcast(a, b, c).shape, dtype=np.uint64)
    for n in range(4):
        nib = (c >> (4 * n)) & 0xF
        sel = nib & 7
        byte = np.zeros_like(out)
        for k in range(8):
            byte = np.where(sel == k, src[k], byte)
        byte = np.where(nib & 8, np.where(byte & 0x80, 0xFF, 0), byte).astype(np.uint64)
        out |= byte << np.uint64(8 * n)
    return out


def e2m1_word_to_u8(w):
    """The kernel's four-codes-to-bytes step: two PRMT lookups and one IADD3."""
    w = np.asarray(w, dtype=np.uint64)
    wn = w ^ 0x88888888
    m32 = 0xFFFFFFFF
    v0 = (prmt(E2M1_LO, E2M1_HI, w) + 0x80808080 - prmt(E2M1_LO, E2M1_HI, wn)) & m32
    v1 = (prmt(E2M1_LO, E2M1_HI, w >> 16) + 0x80808080 - prmt(E2M1_LO, E2M1_HI, wn >> 16)) & m32
    return v0, v1


def exact_e2m1_weight(rows, groups, gs, seed, scale_of):
    """A weight whose every group is E2M1 values times one scale, with +-6 in
    each group so that the encoder picks exactly that scale."""
    g = torch.Generator().manual_seed(seed)
    grid = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    e = grid[torch.randint(0, 8, (rows, groups, gs), generator=g)]
    e = e * torch.where(torch.rand(rows, groups, gs, generator=g) < 0.5, -1.0, 1.0)
    e[:, :, 0] = 6.0 * torch.where(torch.rand(rows, groups, generator=g) < 0.5, -1.0, 1.0)
    sc = scale_of(torch.randint(0, 6, (rows, groups, 1), generator=g))
    return (e * sc).reshape(rows, groups * gs), e.reshape(rows, groups * gs)


@pytest.mark.parametrize("mode,gs,scale_of", [
    ("mxfp4", 32, lambda k: torch.pow(2.0, k.double() - 3).float()),
    ("nvfp4", 16, lambda k: torch.tensor([0.25, 0.5, 1.0, 1.5, 3.0, 7.0])[k]),
])
def test_e2m1_bytes_from_the_oracles_packing(mode, gs, scale_of):
    """For words packed by the oracle, the kernel's bytes are 128 + 2e of the
    oracle's element values e, in code order, with no borrow between bytes."""
    w, e = exact_e2m1_weight(8, 8, gs, 3 if mode == "mxfp4" else 4, scale_of)
    wq, s, _ = oracle.quantize(w, gs, 4, mode)
    deq = oracle.dequantize(wq, s, None, gs, 4, mode, dtype=torch.float32)
    assert torch.equal(deq, w)                       # the groups are encoded exactly
    words = wq.numpy().astype(np.uint64).reshape(-1)
    v0, v1 = e2m1_word_to_u8(words)
    got = np.stack([(v0 >> (8 * i)) & 0xFF for i in range(4)] +
                   [(v1 >> (8 * i)) & 0xFF for i in range(4)], axis=-1).astype(np.int64)
    want = 128 + (2 * e).reshape(-1, 8).numpy().astype(np.int64)
    assert np.array_equal(got, want)
    assert got.min() >= 116 and got.max() <= 140


def test_negative_zero_codes_read_as_zero():
    """Code 8 (E2M1 -0) gives byte 128 like code 0."""
    v0, v1 = e2m1_word_to_u8(np.array([0x88888888, 0x08080808, 0x80808080], dtype=np.uint64))
    for v in (v0, v1):
        assert np.all(v == 0x80808080)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_affine_planes_hold_the_codes_the_kernel_pairs(bits):
    """Plane p of a word (w >> p*bits masked to the low bits of each byte) has
    code j*NP + p in byte j, NP = 8 / bits, for the oracle's packing."""
    w = torch.randn(4, 256)
    wq, s, b = oracle.quantize(w, 64, bits)
    codes = oracle.unpack_codes(wq, bits).numpy().reshape(-1, 32 // bits)
    words = wq.numpy().astype(np.uint64).reshape(-1)
    npl = 8 // bits
    mask = ((1 << bits) - 1) * 0x01010101
    for p in range(npl):
        plane = (words >> (p * bits)) & mask
        for j in range(4):
            assert np.array_equal((plane >> (8 * j)) & 0xFF, codes[:, j * npl + p])


def block_shift(amax):
    """sh with |x 2^sh| < 2^14 for |x| <= amax (the kernel's choice)."""
    ex = ((amax.view(np.uint32) >> 23) & 0xFF).astype(np.int64) - 126
    return np.clip(14 - ex, -126, 126)


@pytest.mark.parametrize("amax_factor", [1.0, 3.0, 1000.0])
def test_magic_rounding_gives_rint_of_the_scaled_activation(amax_factor):
    """x 2^sh + 1.5 * 2^23 in fp32 (exact product, one rounding) has
    rint(x 2^sh) (ties to even) in its low 16 bits, and |x_int| < 2^14, for
    every finite bf16 x and slice maxima at or above |x|."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    x = x[np.isfinite(x)]
    with np.errstate(over="ignore"):        # maxima past fp32's range are dropped
        amax = (np.abs(x) * np.float32(amax_factor)).astype(np.float32)
    keep = np.isfinite(amax)
    x, amax = x[keep], amax[keep]
    sh = block_shift(amax)
    up = np.ldexp(np.float32(1.0), sh).astype(np.float32)
    scaled = (x * up).astype(np.float32)               # exact: a power-of-two scale
    t = (scaled + np.float32(12582912.0)).astype(np.float32)
    low = (t.view(np.uint32) & 0xFFFF).astype(np.uint16).view(np.int16).astype(np.int64)
    want = np.rint(scaled.astype(np.float64)).astype(np.int64)
    assert np.array_equal(low, want)
    assert np.abs(want).max() < (1 << 14)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_packed_max_of_magnitude_bits_is_the_largest_magnitude(dtype):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(4096, 32, generator=g) * torch.logspace(-6, 4, 32)).to(dtype)
    raw = x.view(torch.int16).numpy().astype(np.uint16) & 0x7FFF
    got = raw.max(axis=1).astype(np.uint16).view(np.int16)
    want = x.abs().max(dim=1).values.view(torch.int16).numpy()
    assert np.array_equal(got, want)
