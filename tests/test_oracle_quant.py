"""Pins of the oracle's code tables and NF4 double quantisation (CPU only).

Each pin comes from outside the oracle: figures the pages print
(tests/golden/pages_figures.json), closed forms of the published table
constructions, brute force on tiny tensors, special cases that reduce to the
identity, and the error bound of nearest-entry quantisation.
"""
import io
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import account, bf16, codebooks, quant
from nf4_layer_streamed_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")))


# ----------------------------------------------------------------------------- code tables

def test_nf4_table_shape_and_ends():
    t = codebooks.nf4_table()
    assert t.dtype == np.float32 and t.size == GOLD["nf4_table_entries"]["value"]
    assert t[0] == -1.0 and t[-1] == 1.0
    assert t[7] == 0.0 and np.count_nonzero(t == 0.0) == 1
    assert np.all(np.diff(t.astype(np.float64)) > 0)
    assert np.count_nonzero(t > 0) == 8 and np.count_nonzero(t < 0) == 7


def _phi(x):
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def _phi_inv_bisect(p):
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_nf4_table_matches_normal_quantiles_via_erfc():
    # Independent route to the same quantiles: bisection on erfc instead of ndtri.
    delta = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    top = _phi_inv_bisect(delta)
    t = codebooks.nf4_table().astype(np.float64)
    pos = sorted(_phi_inv_bisect(delta + i * (0.5 - delta) / 8) / top for i in range(8))
    neg = sorted(-_phi_inv_bisect(delta + i * (0.5 - delta) / 7) / top for i in range(7))
    np.testing.assert_allclose(t[8:], pos, rtol=0, atol=2e-7)
    np.testing.assert_allclose(t[:7], neg, rtol=0, atol=2e-7)


def test_code8_table_closed_forms():
    t = codebooks.code8_table()
    assert t.dtype == np.float32 and t.size == GOLD["nested_table_entries"]["value"]
    assert np.all(np.diff(t.astype(np.float64)) > 0)
    assert np.count_nonzero(t == 0.0) == 1
    assert t.max() == 1.0
    assert t.min() == np.float32(-(1.0 - 0.9 / 128.0))
    assert t[t > 0].min() == np.float32(0.55e-6)
    # per decade level i there are 2^i values of each sign in [0.1, 1) * 10^(i-6)
    for i in range(7):
        lo, hi = 0.1 * 10.0 ** (i - 6), 10.0 ** (i - 6)
        pos = t[(t >= np.float32(lo) * 0.999) & (t < np.float32(hi) * 0.999)]
        neg = t[(t <= -np.float32(lo) * 0.999) & (t > -np.float32(hi) * 0.999)]
        assert pos.size == 2 ** i and neg.size == 2 ** i, i


def test_midpoint_rule_brute_force():
    rng = np.random.default_rng(0)
    for table in (codebooks.nf4_table(), codebooks.code8_table()):
        tt = table.astype(np.float64)
        u = rng.uniform(-1, 1, 4000).astype(np.float32)
        u = np.concatenate([u, codebooks.midpoints(table), table])
        idx = codebooks.nearest_index(u, table)
        mids = codebooks.midpoints(table).astype(np.float64)
        window = np.max(np.abs(mids - (tt[:-1] + tt[1:]) / 2))
        for ui, ii in zip(u.astype(np.float64), idx):
            dist = np.abs(tt - ui)
            assert dist[ii] <= dist.min() + 2 * window + 1e-12
        # exact ties at a midpoint go to the lower index
        m_idx = codebooks.nearest_index(codebooks.midpoints(table), table)
        assert np.array_equal(m_idx, np.arange(table.size - 1))


def test_codebook_hash_stable():
    assert codebooks.codebook_hash() == codebooks.codebook_hash()
    assert codebooks.fnv1a64(b"") == 0xCBF29CE484222325


# ----------------------------------------------------------------------------- bytes

def test_byte_identity_matches_quantizer_output():
    rng = np.random.default_rng(1)
    for n in (64, 64 * 256, 64 * 300, 576 * 192):
        w = bf16.round_f32(rng.normal(0, 0.02, n).astype(np.float32))
        q = quant.quantize(w)
        tb = quant.tensor_bytes(n)
        assert q["packed"].nbytes == tb["packed"] == n // 2
        assert q["q8"].nbytes == tb["q8"] == n // 64
        assert q["nested"].nbytes == tb["nested"] == 4 * math.ceil(n / 16384)


def test_bytes_per_param_and_store_sizes_from_pages():
    L8 = synth.LLAMA_8B
    b = account.layer_shard_bytes(L8)
    assert b == 112_513_052
    ratio = b / account.decoder_params(L8)
    assert round(ratio, 3) == GOLD["bytes_per_param"]["value"]
    assert round(account.store_bytes(L8, 32) / 1e9, 2) == GOLD["llama8b_pinned_store_gb"]["value"]
    S1 = synth.SMOLLM2_135M
    assert account.layer_shard_bytes(S1) == 1_825_668
    assert round(account.store_bytes(S1, 30) / 1e9, 3) == GOLD["smollm2_pinned_store_gb"]["value"]
    big = account.layer_shard_bytes(synth.QWEN_32B_CLASS)
    assert big / 2 ** 20 > GOLD["aliasing_layer_threshold_mib"]["value"]


# ----------------------------------------------------------------------------- quantiser

def _brute_quantize(w):
    """Pure-Python loops over blocks, elements and all table entries.  Also returns the
    fp32 ratios u = x / absmax and c / nested that each nearest-entry choice was made on."""
    nf4 = [float(v) for v in codebooks.nf4_table()]
    c8 = [float(v) for v in codebooks.code8_table()]
    x = [float(v) for v in np.asarray(w, np.float32)]
    nb = len(x) // 64
    absmax, codes, us = [], [], []
    for b in range(nb):
        blk = x[b * 64:(b + 1) * 64]
        am = max(abs(v) for v in blk)
        absmax.append(am)
        for v in blk:
            if am == 0.0:
                codes.append(nf4.index(0.0))
                us.append(None)
                continue
            u = float(np.float32(v) / np.float32(am))
            best = min(range(16), key=lambda j: (abs(u - nf4[j]), j))
            codes.append(best)
            us.append(u)
    tot = 0.0
    for am in absmax:
        tot += am
    offset = float(np.float32(tot / nb))
    cs = [float(np.float32(np.float32(am) - np.float32(offset))) for am in absmax]
    nested, q8, uus = [], [], []
    for g in range(0, nb, 256):
        grp = cs[g:g + 256]
        nm = max(abs(c) for c in grp)
        nested.append(nm)
        for c in grp:
            if nm == 0.0:
                q8.append(c8.index(0.0))
                uus.append(None)
                continue
            u = float(np.float32(c) / np.float32(nm))
            q8.append(min(range(256), key=lambda j: (abs(u - c8[j]), j)))
            uus.append(u)
    packed = [(codes[2 * j] << 4) | codes[2 * j + 1] for j in range(len(codes) // 2)]
    return packed, q8, nested, offset, codes, us, uus


def _check_choices(got, want, ratios, table):
    """Every choice equals the exact nearest entry, except where the ratio lies between
    the exact midpoint of two neighbouring entries and that midpoint rounded to fp32
    (the stated fp32-midpoint rule); there the two choices must be those neighbours."""
    t = [Fraction(float(v)) for v in table]
    got, want = np.asarray(got), np.asarray(want)
    for i in np.nonzero(got != want)[0]:
        a, b = sorted((int(got[i]), int(want[i])))
        assert b == a + 1, (i, got[i], want[i])
        exact_mid = (t[a] + t[b]) / 2
        f32_mid = Fraction(float(np.float32(float(exact_mid))))
        u = Fraction(ratios[i])
        assert min(exact_mid, f32_mid) <= u <= max(exact_mid, f32_mid), (i, float(u), float(exact_mid))
    return int(np.count_nonzero(got != want))


@pytest.mark.parametrize("n,seed", [(64 * 4, 0), (64 * 300, 1), (64 * 513, 2)])
def test_quantizer_brute_force(n, seed):
    rng = np.random.default_rng(seed)
    w = bf16.round_f32(rng.normal(0, 0.02, n).astype(np.float32))
    w[:64] = 0.0                       # a zero block
    q = quant.quantize(w)
    packed, q8, nested, offset, codes, us, uus = _brute_quantize(w)
    assert q["offset"] == np.float32(offset)
    np.testing.assert_array_equal(q["nested"], np.array(nested, np.float32))
    _check_choices(quant.unpack_codes(q["packed"]), codes, us, codebooks.nf4_table())
    _check_choices(q["q8"], q8, uus, codebooks.code8_table())


def test_quantizer_brute_force_at_midpoints():
    """Ratios placed exactly on, and one fp32 ulp either side of, every fp32 midpoint
    of the NF4 table: the oracle's choices differ from the exact nearest entry only
    inside the fp32-midpoint window, and an exact fp32 tie goes to the lower index."""
    nf4 = codebooks.nf4_table()
    mids = codebooks.midpoints(nf4)
    u = np.concatenate([mids, np.nextafter(mids, np.float32(2)), np.nextafter(mids, np.float32(-2))])
    u = np.concatenate([u, np.zeros((-u.size) % 64 + 64, np.float32)])
    u[63] = 1.0                                      # absmax 1 in the first block: x / absmax = x
    w = u.astype(np.float32)
    w[64:128] = np.where(np.arange(64) == 0, 1.0, w[64:128]).astype(np.float32)
    q = quant.quantize(w)
    _, _, _, _, codes, us, _ = _brute_quantize(w)
    _check_choices(quant.unpack_codes(q["packed"]), codes, us, nf4)
    got = quant.unpack_codes(q["packed"])[:mids.size]
    np.testing.assert_array_equal(got, np.arange(mids.size))   # on the fp32 midpoint: lower index


def test_nibble_order_high_first():
    nf4 = codebooks.nf4_table()
    A = np.float32(0.125)
    codes = np.array([15, 0] + [7] * 62, dtype=np.int64)
    w = bf16.round_f32(nf4[codes] * A)
    q = quant.quantize(w)
    assert q["packed"][0] == 0xF0
    assert q["packed"][1] == 0x77


def test_quant_dequant_identity_on_representable_tensor():
    # Every block holds +-A and table values times A with the same power-of-two A:
    # offset = A, nested = 0, s = A exactly, so dequant(quant(w)) == w bit for bit.
    rng = np.random.default_rng(3)
    nf4 = codebooks.nf4_table()
    A = np.float32(2.0 ** -5)
    codes = rng.integers(0, 16, 64 * 700)
    codes[0::64] = 15
    w = bf16.round_f32(nf4[codes] * A)
    q = quant.quantize(w)
    np.testing.assert_array_equal(quant.unpack_codes(q["packed"]), codes)
    np.testing.assert_array_equal(quant.dequantize_bits(q), bf16.f32_to_bf16_bits(w))


def test_dequant_error_bound_and_zero_block():
    rng = np.random.default_rng(4)
    n = 64 * 1000
    w = bf16.round_f32(rng.normal(0, 0.02, n).astype(np.float32))
    w[64 * 10:64 * 11] = 0.0
    q = quant.quantize(w)
    wh = quant.dequantize(q)
    nf4 = codebooks.nf4_table().astype(np.float64)
    c8 = codebooks.code8_table().astype(np.float64)
    g4 = np.max(np.diff(nf4)) / 2
    g8 = np.max(np.diff(c8)) / 2
    xb = w.astype(np.float64).reshape(-1, 64)
    absmax = np.abs(xb).max(axis=1)
    nested_max = float(q["nested"].max())
    bound = g4 * absmax[:, None] + g8 * nested_max + 2.0 ** -8 * np.abs(xb) + 1e-9
    assert np.all(np.abs(xb - wh.reshape(-1, 64)) <= bound)
    assert np.all(wh.reshape(-1, 64)[10] == 0.0)


def _multi_group_tensor():
    """3 full nested groups and a partial fourth (50 blocks) whose deviations of the
    block absmax from the mean are scaled by 1, 2^-8, 2^6 and 2^-4 (|d| below 2^-7,
    2^-15, 2^-1 and 2^-11).  Deviations come in +d / -d pairs of multiples of 2^-23
    around 1, so the fp32 absmax values are exact, their mean (the offset) is exactly
    1, and each group's nested absmax is exactly its largest |d|.  Each block holds
    its absmax once (with a random sign) and NF4 table values times it elsewhere."""
    rng = np.random.default_rng(21)
    scales = [1.0, 2.0 ** -8, 2.0 ** 6, 2.0 ** -4]
    sizes = [256, 256, 256, 50]
    nf4 = codebooks.nf4_table()
    absmax, nested = [], []
    for sc, nb in zip(scales, sizes):
        k = rng.integers(1, int(2 ** 16 * sc), nb // 2)  # |d| = k * 2^-23 < 2^-7 * scale
        d = np.concatenate([k, -k]).astype(np.float64) * 2.0 ** -23
        rng.shuffle(d)
        absmax.append(1.0 + d)
        nested.append(float(np.max(np.abs(d))))
    absmax = np.concatenate(absmax)
    assert np.all(absmax.astype(np.float32).astype(np.float64) == absmax)
    nb = absmax.size
    codes = rng.integers(0, 16, (nb, 64))
    top = rng.integers(0, 64, nb)
    codes[np.arange(nb), top] = np.where(rng.random(nb) < 0.5, 0, 15)     # the -1 or +1 entry
    w = (nf4[codes].astype(np.float64) * absmax[:, None]).astype(np.float32)
    # the fp32 product nf4[c] * absmax can round; the block's largest magnitude is exact
    assert np.all(np.abs(w).max(axis=1).astype(np.float64) == absmax)
    return w.reshape(-1), absmax, np.array(nested), np.array(sizes)


def test_dequant_across_nested_groups_with_different_scales():
    """Pins the nested-group indexing of the double quantisation and of the scale
    decode: the offset is exactly 1, each group's nested absmax is its own largest
    deviation (groups of 256 consecutive blocks, the last one partial), each decoded
    block scale is within half an 8-bit table gap times its OWN group's nested absmax
    of the true absmax (a wrong group would be off by up to 2^14 of that), and the
    dequantised weights equal a pure-Python per-element decode."""
    w, absmax, nested, sizes = _multi_group_tensor()
    q = quant.quantize(w)
    assert q["offset"] == np.float32(1.0)
    np.testing.assert_array_equal(q["nested"].astype(np.float64), nested)
    c8 = codebooks.code8_table().astype(np.float64)
    halfgap = np.max(np.diff(c8)) / 2
    group = np.repeat(np.arange(sizes.size), sizes)
    s = quant.block_scales(q).astype(np.float64)
    err = np.abs(s - absmax)
    # two fp32 roundings (the product and the sum with 1) add at most 2^-23 + 2^-24 each
    assert np.all(err <= halfgap * nested[group] + 2.0 ** -22), np.max(err / nested[group])
    # the smallest groups resolve far below the largest group's table gap
    assert np.max(err[group == 1]) < halfgap * nested[2] * 2.0 ** -10

    nf4 = [float(v) for v in codebooks.nf4_table()]
    c8f = [float(v) for v in codebooks.code8_table()]
    bits = quant.dequantize_bits(q)
    packed, q8, nst, off = list(q["packed"]), list(q["q8"]), list(q["nested"]), np.float32(q["offset"])
    for i in range(0, w.size, 7):                   # every 7th element, across all four groups
        b = i // 64
        g = b // 256
        c = (packed[i // 2] >> 4) if i % 2 == 0 else (packed[i // 2] & 15)
        sc = np.float32(np.float32(np.float32(c8f[q8[b]]) * np.float32(nst[g])) + off)
        val = np.float32(np.float32(nf4[c]) * sc)
        ref = int(torch.from_numpy(np.array([val], np.float32)).to(torch.bfloat16).view(torch.int16)[0]) & 0xFFFF
        assert int(bits[i]) == ref, (i, b, g)


def test_quantize_deterministic_and_roundtrip_through_bytes():
    w = synth.tensor_values((192, 576), seed=77, scale=0.02).float().numpy()
    q1, q2 = quant.quantize(w), quant.quantize(w)
    for k in ("packed", "q8", "nested"):
        assert np.array_equal(q1[k], q2[k])
    buf = io.BytesIO()
    np.savez(buf, **{k: q1[k] for k in ("packed", "q8", "nested")}, offset=q1["offset"])
    buf.seek(0)
    r = np.load(buf)
    assert np.array_equal(quant.dequantize_bits({**{k: r[k] for k in ("packed", "q8", "nested")},
                                                 "offset": r["offset"]}),
                          quant.dequantize_bits(q1))


# ----------------------------------------------------------------------------- properties
from hypothesis import given, settings, strategies as st  # noqa: E402


@st.composite
def _weight_blocks(draw):
    """1-9 blocks of 64 bf16 values: a per-block scale over 40 binades, some blocks all
    zero, some holding a single nonzero, signs mixed."""
    nb = draw(st.integers(1, 9))
    rng = np.random.default_rng(draw(st.integers(0, 2 ** 31 - 1)))
    w = np.empty(64 * nb, np.float32)
    for b in range(nb):
        kind = draw(st.sampled_from(["normal", "zero", "single", "uniform"]))
        scale = np.float32(2.0 ** draw(st.integers(-30, 10)))
        if kind == "zero":
            blk = np.zeros(64, np.float32)
        elif kind == "single":
            blk = np.zeros(64, np.float32)
            blk[draw(st.integers(0, 63))] = scale * draw(st.sampled_from([-1.0, 1.0, 0.37]))
        elif kind == "uniform":
            blk = (rng.uniform(-1, 1, 64) * scale).astype(np.float32)
        else:
            blk = (rng.normal(0, 1, 64) * scale).astype(np.float32)
        w[b * 64:(b + 1) * 64] = blk
    return bf16.round_f32(w)


@settings(max_examples=60, deadline=None)
@given(_weight_blocks())
def test_quantizer_properties(w):
    """What any correct blockwise NF4 quantiser with double-quantised absmax does,
    on blocks spanning 40 binades: each code is a nearest NF4 entry to x / absmax
    (up to the fp32 midpoint window); a block's largest magnitude maps to -1 or +1; an
    all-zero block gives the zero code and dequantises to exact zeros; the nested scale
    reproduces absmax within the 8-bit table's resolution."""
    q = quant.quantize(w)
    nf4 = codebooks.nf4_table().astype(np.float64)
    codes = quant.unpack_codes(q["packed"]).reshape(-1, 64)
    xb = w.astype(np.float64).reshape(-1, 64)
    am = np.abs(xb).max(axis=1)
    zero = codebooks.zero_index(nf4)
    for b in range(xb.shape[0]):
        if am[b] == 0.0:
            assert np.all(codes[b] == zero)
            continue
        u = xb[b] / am[b]
        dist = np.abs(u[:, None] - nf4[None, :])
        chosen = dist[np.arange(64), codes[b]]
        assert np.all(chosen <= dist.min(axis=1) + 1e-6)
        i = int(np.argmax(np.abs(xb[b])))
        assert nf4[codes[b][i]] == np.sign(xb[b][i])
    wh = quant.dequantize(q).reshape(-1, 64)
    assert np.all(wh[am == 0.0] == 0.0)
    s = quant.block_scales(q).astype(np.float64)
    c8 = codebooks.code8_table().astype(np.float64)
    gap = np.max(np.diff(c8)) / 2 * float(np.max(q["nested"])) + 1e-6 * am.max()
    assert np.all(np.abs(s - am) <= gap + 2.0 ** -20 * am)
