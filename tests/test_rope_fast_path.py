"""The RoPE kernels' fp32 fast path and its rounding test, on the host.

The kernels rotate each 16-byte chunk (4 channel pairs) in fp32 with exact
products of split table values and keep the result only when a rounding test
proves it is the bf16 rounding of the exact fp64 definition (UltraGen-ar
§2.ب; reading R1); otherwise they recompute the chunk in fp64.  Here that
same code (ug_rope_math.h), built for the host, is checked against the
oracle's definition (exact fp64 products, one fp64 rounding, the oracle's own
bf16 rounding), for the rotation and its transpose:
  * every accepted chunk equals the oracle's, on random inputs and on inputs
    built to land within a few fp32 ulps of a bf16 rounding midpoint, exactly
    on one, or after heavy cancellation;
  * the test rejects the cases it cannot decide (so the exact route runs),
    and accepts nearly every random chunk (the fast path is the common one);
  * the table split is exact and keeps 16 significant bits in the high part.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import hier_local_attn as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hostlib(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("no host C++ compiler")
    so = tmp_path_factory.mktemp("rope") / "rope_fast_host.so"
    subprocess.run(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                    "-I", os.path.join(ROOT, "block_sparse_local_raster_b200", "csrc"),
                    os.path.join(ROOT, "tests", "cpp", "rope_fast_host.cpp"), "-o", str(so)],
                   check=True)
    lib = ctypes.CDLL(str(so))
    P = ctypes.c_void_p
    lib.rope_chunks_fast.argtypes = [P, P, P, ctypes.c_int, P, P, ctypes.c_int64]
    lib.rope_split.argtypes = [P, P, P, ctypes.c_int64]
    return lib


@pytest.fixture(scope="module", params=[False, True], ids=["rotation", "transpose"])
def fast(hostlib, request):
    """run(xw, c, s) -> (out words, per-pair accepted): pairs are grouped in
    chunks of 4 (padded with the last pair); a pair counts as accepted when
    its chunk is."""
    transpose = request.param

    def run(xw, c, s):
        n = xw.size
        m = -(-n // 4) * 4
        pad = lambda a, dt: np.ascontiguousarray(np.concatenate([a, np.repeat(a[-1:], m - n)]), dt)
        w, cc, ss = pad(xw, np.uint32), pad(c, np.float32), pad(s, np.float32)
        out = np.zeros(m, np.uint32)
        ok = np.zeros(m // 4, np.uint8)
        hostlib.rope_chunks_fast(w.ctypes.data, cc.ctypes.data, ss.ctypes.data, int(transpose),
                                 out.ctypes.data, ok.ctypes.data, m // 4)
        return out[:n], np.repeat(ok.astype(bool), 4)[:n]
    run.transpose = transpose
    return run


def oracle_pair(xw, c, s, transpose=False):
    """The oracle's rotation (or its transpose: the sine negated) of the
    pairs, as two bf16 patterns packed like the kernels' output word (y0
    low)."""
    x0 = O.bf16_to_f64((xw & 0xFFFF).astype(np.uint16))
    x1 = O.bf16_to_f64((xw >> 16).astype(np.uint16))
    x = np.stack([x0, x1], axis=-1)
    sn = -s.astype(np.float64) if transpose else s.astype(np.float64)
    y = O.rope_rotate_f64(x, c.astype(np.float64)[:, None], sn[:, None])
    b = O.f64_to_bf16(y).astype(np.uint32)
    return b[:, 0] | (b[:, 1] << 16)


def bf16_bits(v):
    return O.f64_to_bf16(np.asarray(v, np.float64)).astype(np.uint32)


def check(fast, xw, c, s):
    got, ok = fast(xw, c, s)
    ref = oracle_pair(xw, c, s, fast.transpose)
    bad = ok & (got != ref)
    assert not bad.any(), (xw[bad][:4], c[bad][:4], s[bad][:4])
    return ok


def test_table_split_is_exact(hostlib):
    rng = np.random.default_rng(9)
    c = np.concatenate([np.cos(rng.uniform(0, 600, 100000)), [0.0, 1.0, -1.0, 1e-20]]).astype(np.float32)
    hi, lo = np.zeros_like(c), np.zeros_like(c)
    hostlib.rope_split(c.ctypes.data, hi.ctypes.data, lo.ctypes.data, c.size)
    assert (hi.astype(np.float64) + lo.astype(np.float64) == c.astype(np.float64)).all()
    assert (hi + lo == c).all()  # the fp32 sum the exact route uses is exact too
    assert ((hi.view(np.uint32) & 0xFF) == 0).all()  # 16 significant bits in hi
    nz = lo != 0
    assert (np.abs(lo[nz]) < np.abs(c[nz]) * 2.0 ** -15).all()


def test_random_chunks_agree_and_mostly_take_the_fast_path(fast):
    rng = np.random.default_rng(0)
    n = 400_000
    xw = bf16_bits(rng.standard_normal(n)) | (bf16_bits(rng.standard_normal(n)) << 16)
    ang = rng.uniform(0, 600, n)
    c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    ok = check(fast, xw, c, s)
    assert ok.mean() > 0.995, ok.mean()


def test_pairs_near_bf16_midpoints(fast):
    """x0 c - x1 s placed within +-8 fp32 ulps of a bf16 midpoint: x0, x1, c
    drawn, s solved so that the result hits the midpoint, then rounded to
    fp32 and nudged by a few ulps either way."""
    rng = np.random.default_rng(1)
    n = 200_000
    x0 = O.bf16_to_f64(bf16_bits(rng.standard_normal(n)).astype(np.uint16))
    x1 = O.bf16_to_f64(bf16_bits(rng.uniform(0.5, 2.0, n) * rng.choice([-1, 1], n)).astype(np.uint16))
    c = rng.uniform(-1, 1, n).astype(np.float32)
    # a bf16 midpoint near x0 c: the bf16 value below it plus half its ulp
    t = x0 * c.astype(np.float64) * rng.uniform(0.2, 1.5, n)
    lo = O.bf16_to_f64(O.f64_to_bf16(t))
    e = np.floor(np.log2(np.abs(lo)))
    mid = lo + np.sign(lo) * np.ldexp(1.0, (e - 8).astype(int))
    s = ((x0 * c - mid) / x1 * (-1.0 if fast.transpose else 1.0)).astype(np.float32)
    s = np.clip(s, -1, 1).astype(np.float32)
    k = rng.integers(-8, 9, n).astype(np.int32)
    s = (s.view(np.int32) + k).view(np.float32)
    s = np.clip(s, -1, 1).astype(np.float32)
    xw = bf16_bits(x0) | (bf16_bits(x1) << 16)
    ok = check(fast, xw, c, s)
    # most of these are too close to call: the exact route must take them
    assert ok.mean() < 0.95, ok.mean()


def test_exact_midpoints_and_cancellation(fast):
    """Results exactly on a bf16 midpoint (ties to even decide), exact zeros
    and heavy cancellation (x0 c almost equal to x1 s)."""
    rng = np.random.default_rng(2)
    n = 100_000
    # exact midpoints: x1 = 0, c = 1 - tiny so that x0 c is a midpoint? use x0 c
    # with c a power of two: x0 c is bf16-exact; add x1 s = half an ulp of it
    x0 = O.bf16_to_f64(bf16_bits(rng.standard_normal(n)).astype(np.uint16))
    c = np.ldexp(1.0, rng.integers(-3, 1, n)).astype(np.float32)
    p = x0 * c.astype(np.float64)
    e = np.floor(np.log2(np.abs(p)))
    half = np.ldexp(1.0, (e - 8).astype(int))  # half a bf16 ulp of p
    x1 = np.ones(n)
    s = (-half * rng.choice([-1, 1], n)).astype(np.float32)  # y0 = p - s = p +- half
    xw = bf16_bits(x0) | (bf16_bits(x1) << 16)
    ok = check(fast, xw, c, s)
    # p +- half is a midpoint unless it crossed into the binade below (where it
    # is a bf16 value): the midpoints are never decided by the fast path
    y0 = p + s.astype(np.float64) * (1.0 if fast.transpose else -1.0)
    is_mid = O.bf16_to_f64(O.f64_to_bf16(y0)) != y0
    assert is_mid.mean() > 0.9
    assert not ok[is_mid].any()
    # cancellation: x1 s equal to x0 c up to a few fp32 ulps
    x0 = O.bf16_to_f64(bf16_bits(rng.standard_normal(n)).astype(np.uint16))
    x1 = O.bf16_to_f64(bf16_bits(rng.standard_normal(n)).astype(np.uint16))
    c = rng.uniform(-1, 1, n).astype(np.float32)
    s = (x0 * c / x1).astype(np.float32)
    ok_s = np.abs(s) <= 1
    s = np.where(ok_s, s, 0.5).astype(np.float32)
    s = (s.view(np.int32) + rng.integers(-3, 4, n).astype(np.int32)).view(np.float32)
    xw = bf16_bits(x0) | (bf16_bits(x1) << 16)
    check(fast, xw, c, s)
    # zeros of both signs
    z = np.array([0x0000, 0x8000, 0x80000000, 0x80008000, 0x00008000], np.uint32)
    ok = check(fast, z, np.full(5, 0.3, np.float32), np.full(5, -0.7, np.float32))
    assert not ok.any()


def test_table_values_of_the_configs(fast):
    """The cos/sin values a kernel meets: every angle of the 8K config's
    tables (positions up to 512, both axes), with random bf16 pairs."""
    rng = np.random.default_rng(3)
    a = 64
    f = 10000.0 ** (-2.0 * np.arange(a // 2) / a)
    pos = np.concatenate([np.arange(512.0), 4.0 * np.arange(128.0)])
    ang = (pos[:, None] * f[None, :]).ravel()
    c = np.cos(ang).astype(np.float32)
    s = np.sin(ang).astype(np.float32)
    for rep in range(4):
        n = c.size
        xw = bf16_bits(rng.standard_normal(n)) | (bf16_bits(rng.standard_normal(n)) << 16)
        check(fast, xw, c, s)
        check(fast, xw, c, -s)  # the transposed rotation
