"""Exhaustive device-side checks of the arithmetic shortcuts and conversion
helpers inside the quantizer kernels (libfos_check.so, include/fos_check.h).

The kernels replace IEEE divisions with reciprocal products plus one
correction step (r / 6 and a / S_t of the block-scale step), use an integer
form of the stochastic-rounding rule, and rely on the hardware E2M1/E4M3
conversions.  The parity tests only sample these on real data; here every
input of each helper's domain runs on the device (every binary32 pattern,
every bf16 pair, every (value, byte) pair), and the encoders and decoders
are compared with the CPU oracle.

Sources of the steps: Hugging Face transformers doc "Four Over Six",
introduction (block max mapped to 4 or 6); Ultralytics glossary "FP4",
"Como funciona FP4" (E4M3 block scale, FP32 tensor scale, E2M1 values) and
"Inferencia e Treinamento FP4" (stochastic rounding)."""
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_fos_b200 import build as fbuild

from helpers import require_gpu

pytestmark = pytest.mark.gpu

_L = None


def _lib():
    global _L
    if _L is None:
        path = fbuild.build_check()
        L = ctypes.CDLL(path)
        P, u64, i64, i32, u32, f32 = (ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_uint32, ctypes.c_float)
        sigs = {
            "fosck_div6": [P, P],
            "fosck_div_tscale_bf16": [f32, P, P],
            "fosck_div_tscale_random": [u64, u64, P, P],
            "fosck_sr_forms": [P, P],
            "fosck_philox_vs_curand": [u64, u64, P, P],
            "fosck_sr_codes": [P, P, i64, i32, P, P],
            "fosck_transitions": [i32, P, u32, P, P],
            "fosck_codes_at": [P, i64, i32, P, P],
            "fosck_e2m1_decode_words": [P, P, P],
            "fosck_e4m3_decode_all": [P, P],
            "fosck_hmax_abs": [P, P],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.restype = ctypes.c_int
            fn.argtypes = args
        _L = L
    return _L


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _run(name, *args):
    rc = getattr(_lib(), name)(*args, _stream())
    assert rc == 0, "%s launch failed: cudaError %d" % (name, rc)
    torch.cuda.synchronize()


def _counts(n=2):
    return torch.zeros(n, dtype=torch.int64, device=require_gpu())


def test_div6_every_finite_binary32():
    c = _counts()
    _run("fosck_div6", _p(c))
    assert c.tolist() == [0, 0], "r/6 shortcut: %d quotient mismatches, %d E4M3 code mismatches" % tuple(c.tolist())


@pytest.mark.parametrize("divisor", [1792.0, 2688.0])
def test_div_tscale_every_bf16_pair(divisor):
    c = _counts()
    _run("fosck_div_tscale_bf16", ctypes.c_float(divisor), _p(c))
    assert c.tolist() == [0, 0], "a/S_t shortcut: %d code mismatches, %d quotient mismatches" % tuple(c.tolist())


def test_div_tscale_random_binary32_pairs():
    c = _counts()
    _run("fosck_div_tscale_random", 12345, 1 << 30, _p(c))
    assert c.tolist() == [0, 0], "a/S_t shortcut: %d code mismatches, %d quotient mismatches" % tuple(c.tolist())


def test_philox_equals_curand():
    """The device Philox4x32-10 behind the SR bytes and the RHT signs equals
    cuRAND's curand_Philox4x32_10 on 2^24 random (counter, key) pairs."""
    c = _counts(1)
    _run("fosck_philox_vs_curand", 2024, 1 << 24, _p(c))
    assert c.item() == 0, "Philox differs from cuRAND in %d words" % c.item()


def test_sr_integer_and_pair_forms_equal_float_form_everywhere():
    c = _counts(1)
    _run("fosck_sr_forms", _p(c))
    assert c.item() == 0, "SR forms differ on %d (v, byte) pairs" % c.item()


def _sr_probe_values():
    """Values at and next to every threshold of the rule: for each grid
    interval [lo, hi) the points lo + (hi-lo)*k/512 (k = 0..511), one ulp on
    either side, the grid points, values >= 6, and random binary32 values."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    pts = []
    for lo, hi in zip(grid[:-1], grid[1:]):
        k = np.arange(512, dtype=np.float64)
        v = (lo + (hi - lo) * k / 512).astype(np.float32)
        pts += [v, np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(0))]
    pts.append(np.array([6.0, 6.5, 7.0, 1e30, np.inf], np.float32))
    rng = np.random.default_rng(7)
    pts.append(rng.uniform(0, 8, 1 << 14).astype(np.float32))
    v = np.concatenate(pts).astype(np.float32)
    v = v[np.isfinite(v) | np.isinf(v)]
    return np.abs(v)


def test_sr_rule_matches_oracle():
    dev = require_gpu()
    v = _sr_probe_values()
    vv = np.repeat(v, 256)
    bb = np.tile(np.arange(256, dtype=np.uint8), v.size)
    want = oracle.e2m1_sr(vv, bb)
    tv = torch.from_numpy(vv).to(dev)
    tb = torch.from_numpy(bb).to(dev)
    for form in (0, 1, 2):
        out = torch.empty(vv.size, dtype=torch.uint8, device=dev)
        _run("fosck_sr_codes", _p(tv), _p(tb), vv.size, form, _p(out))
        got = out.cpu().numpy()
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, "form %d: v=%r byte=%d gpu %d oracle %d" % (
            form, float(vv[bad[0]]), bb[bad[0]], got[bad[0]], want[bad[0]])


def _oracle_codes(bits, e4m3):
    v = np.asarray(bits, np.uint32).view(np.float32)
    return (oracle.e4m3_encode(v) if e4m3 else oracle.e2m1_encode(v)).astype(np.int64)


def _gpu_codes_at(bits, e4m3):
    dev = require_gpu()
    idx = torch.from_numpy(np.asarray(bits, np.uint32).view(np.int32).copy()).to(dev)
    out = torch.empty(idx.numel(), dtype=torch.int32, device=dev)
    _run("fosck_codes_at", _p(idx), idx.numel(), int(e4m3), _p(out))
    return out.cpu().numpy().view(np.uint32).astype(np.int64)


@pytest.mark.parametrize("e4m3", [0, 1], ids=["e2m1", "e4m3"])
def test_encoder_equals_oracle_on_every_binary32(e4m3):
    """The device encoder's code changes at exactly the patterns where the
    oracle's does.  The device returns every pattern i (non-NaN) whose code
    differs from that of pattern i-1; each segment between such patterns has
    one device code, and the oracle agrees at both ends of every segment.
    The oracle's code is a nearest-value search, monotone in |v| within each
    sign, so it is constant on the segment too: the two encoders agree on
    all 2^32 patterns but the NaNs.  A random sample double-checks."""
    dev = require_gpu()
    max_out = 4096
    out = torch.zeros(3 * max_out, dtype=torch.int32, device=dev)
    cnt = torch.zeros(1, dtype=torch.int32, device=dev)
    _run("fosck_transitions", int(e4m3), _p(out), max_out, _p(cnt))
    n = int(cnt.item())
    assert 0 < n <= max_out, n
    tr = out.cpu().numpy().view(np.uint32)[: 3 * n].reshape(n, 3).astype(np.int64)
    tr = tr[np.argsort(tr[:, 0])]
    assert not np.any(tr[:, 1:] == 0xFFFF), "the two lanes of the paired conversion disagree"
    expect = 2 * (7 if not e4m3 else 126)
    assert n == expect, "%d code changes, expected %d" % (n, expect)
    # both sides of every change
    assert np.array_equal(_oracle_codes(tr[:, 0] - 1, e4m3), tr[:, 1])
    assert np.array_equal(_oracle_codes(tr[:, 0], e4m3), tr[:, 2])
    # both ends of every segment, per sign half
    ends = []
    for lo, hi in ((0x00000000, 0x7F800000), (0x80000000, 0xFF800000)):
        cuts = [int(t) for t in tr[:, 0] if lo < t <= hi]
        starts = [lo] + cuts
        stops = [c - 1 for c in cuts] + [hi]
        ends += list(zip(starts, stops))
    s = np.array([a for a, _ in ends], np.uint64)
    e = np.array([b for _, b in ends], np.uint64)
    gs, ge = _gpu_codes_at(s, e4m3), _gpu_codes_at(e, e4m3)
    assert np.array_equal(gs, ge)
    assert np.array_equal(_oracle_codes(s, e4m3), gs)
    assert np.array_equal(_oracle_codes(e, e4m3), ge)
    rng = np.random.default_rng(3 + e4m3)
    sample = rng.integers(0, 1 << 32, 1 << 18, dtype=np.uint64).astype(np.uint32)
    sample = sample[(sample & 0x7FFFFFFF) <= 0x7F800000]
    assert np.array_equal(_gpu_codes_at(sample, e4m3), _oracle_codes(sample, e4m3))


def test_e2m1_decoder_every_word():
    dev = require_gpu()
    vals = np.array([oracle.e2m1_decode(c) for c in range(16)], np.float32)
    table = torch.from_numpy(vals.astype(np.float16).view(np.int16).copy()).to(dev)
    assert np.array_equal(vals.astype(np.float16).astype(np.float32), vals)
    c = _counts(1)
    _run("fosck_e2m1_decode_words", _p(table), _p(c))
    assert c.item() == 0, "%d decoded words differ" % c.item()


def test_e4m3_decoder_all_codes():
    dev = require_gpu()
    out = torch.empty(256, dtype=torch.float32, device=dev)
    _run("fosck_e4m3_decode_all", _p(out))
    got = out.cpu().numpy()
    want = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


def test_packed_bf16_magnitude_max_every_pair():
    c = _counts(1)
    _run("fosck_hmax_abs", _p(c))
    assert c.item() == 0, "%d bf16 pairs give a wrong magnitude maximum" % c.item()
