"""Bit-level helpers of the CUDA path, compiled as host code (they are
__host__ __device__): the order-preserving unsigned keys on which the routers'
warp top-k takes its maxima, and the bf16 round-to-nearest-even conversion,
against numpy and the oracle's own bf16 rounding."""

import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_E4M3 = {}  # the helper program's widening of all 256 codes (filled by the fixture)


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("helpers")
    exe = str(d / "helpers_check")
    subprocess.run([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
                    os.path.join(ROOT, "tests", "helpers_check.cu"), "-o", exe],
                   check=True, capture_output=True)
    rng = np.random.default_rng(5)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 1.0, -1.0, 1e-45, -1e-45, 1e-40, -1e-40,
                        np.finfo(np.float32).max, -np.finfo(np.float32).max,
                        np.finfo(np.float32).tiny, -np.finfo(np.float32).tiny], np.float32)
    bits = rng.integers(0, 2 ** 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = np.concatenate([special, bits.view(np.float32), rng.normal(size=20_000).astype(np.float32)])
    f = f[~np.isnan(f)]
    src, dst, e8 = str(d / "in.bin"), str(d / "out.bin"), str(d / "e4m3.bin")
    f.view(np.uint32).tofile(src)
    subprocess.run([exe, src, dst, e8], check=True)
    rec = np.fromfile(dst, dtype=np.uint32).reshape(-1, 5)
    _E4M3["scaled"] = np.fromfile(e8, dtype=np.uint32)
    return f, rec


def test_order_keys_sort_like_the_floats(results):
    f, rec = results
    key = rec[:, 0]
    o = np.argsort(f, kind="stable")
    fs, ks = f[o], key[o]
    # strictly increasing keys for strictly increasing values, equal for equal
    # values (-0 and +0 share one key)
    d_f, d_k = np.diff(fs.astype(np.float64)), np.diff(ks.astype(np.int64))
    assert np.all((d_f > 0) == (d_k > 0)) and np.all((d_f == 0) == (d_k == 0))
    # a key 0 (how the top-k marks removed entries) sorts below every float
    assert key.min() > 0


def test_key_value_inverts_order_key(results):
    f, rec = results
    back = rec[:, 1].view(np.float32)
    assert np.array_equal(back, f + np.float32(0.0))           # -0 comes back as +0
    assert not np.any(np.signbit(back[f == 0]))


def test_bf16_rounding_matches_the_oracle(results):
    f, rec = results
    finite = np.isfinite(f)
    want = oracle.bf16_from_double(f[finite].astype(np.float64))
    assert np.array_equal(rec[finite, 2].astype(np.uint16), want)


def test_bf16_pair_packing_round_trips(results):
    f, rec = results
    bf = rec[:, 2].astype(np.uint32)
    lo = rec[:, 3].view(np.float32)
    hi = rec[:, 4].view(np.float32)
    # the low half is the first value; widening a bf16 is exact (bits << 16)
    assert np.array_equal(lo.view(np.uint32), bf << 16)
    neg = np.isfinite(f)
    assert np.array_equal(hi[neg], -lo[neg])


def test_scaled_e4m3_widening_is_exact_for_every_code(results):
    """The FP8 GEMM widens e4m3 codes to bf16 with integer bit moves that give
    value * 2^-120 (then one bf16 multiply by 2^120 on the GPU). Every non-NaN
    code, normal, subnormal and both zeros, against the oracle's e4m3 decoding."""
    r = _E4M3["scaled"][:256]
    codes = np.arange(256)
    lo = (r & 0xFFFF).astype(np.uint16)
    hi = (r >> 16).astype(np.uint16)
    for half, code in ((lo, codes), (hi, 255 - codes)):
        got = oracle.double_from_bf16(half) * 2.0 ** 120
        want = oracle.double_from_e4m3(code.astype(np.uint8))
        ok = ~np.isnan(want)
        assert ok.sum() == 254
        assert np.array_equal(got[ok], want[ok])
        # signed zeros carry over
        assert np.array_equal(np.signbit(got[ok]), np.signbit(want[ok]))


def test_scaled_e2m1_widening_is_exact_for_every_byte(results):
    """The FP4 GEMM widens a byte of two E2M1 codes to a bf16 pair with integer
    moves that give value * 2^-126 (the GPU then multiplies by the block scale
    times 2^126). Every byte, both codes, against the oracle's E2M1 decoding."""
    r = _E4M3["scaled"][256:]
    b = np.arange(256, dtype=np.uint8)
    for half, nib in (((r & 0xFFFF), b & 0xF), ((r >> 16), b >> 4)):
        got = oracle.double_from_bf16(half.astype(np.uint16)) * 2.0 ** 126
        want = oracle.double_from_e2m1(nib.astype(np.uint8))
        assert np.array_equal(got, want)
        assert np.array_equal(np.signbit(got), np.signbit(want))
