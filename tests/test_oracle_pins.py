"""Pins of the CPU oracle against what the pages and mathematics fix.

None of these compares the oracle with itself: each check uses an
independent route (numpy/torch number formats, brute force, closed forms,
hand-derived fixtures under tests/golden/, exact special cases).
"""
import itertools
import os

import numpy as np
import pytest
import torch

import oracle as orc
from quantized_gemv_group_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f16_bits(a):
    return np.asarray(a, np.float16).view(np.uint16)


def _f16_val(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------- number formats
def test_f16_decode_every_pattern_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.f16_decode(bits)
    ref = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(ours[m], ref[m])
    assert np.array_equal(np.signbit(ours[m]), np.signbit(ref[m]))


def test_bf16_decode_matches_torch():
    g = np.random.default_rng(1)
    bits = g.integers(0, 65536, 4000).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]           # finite only
    ours = orc.bf16_decode(bits)
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(ours, ref)


def _pred_f16(v):
    return np.nextafter(np.float16(v), np.float16(-np.inf))


def test_f32_to_f16_round_up_is_smallest_upper_bound():
    g = np.random.default_rng(2)
    vals = np.concatenate([
        g.standard_normal(3000) * 0.02,
        g.standard_normal(1000) * 1e-6,                    # fp16 subnormal range
        g.standard_normal(1000) * 3e4,
        _f16_val(g.integers(0, 0x7C00, 1000).astype(np.uint16)),   # exact fp16 values
        -_f16_val(g.integers(0, 0x7C00, 500).astype(np.uint16)),
        np.array([6.1e-5, 65504.0, 65504.5, 1e5, -1e5, 1e-30, -1e-30]),
    ]).astype(np.float32)
    out = orc.f32_to_f16_ru(vals)
    r = _f16_val(out)
    x = vals.astype(np.float64)
    big = x > 65504.0
    assert np.all(np.isposinf(r[big]))
    neg_big = x < -65504.0
    assert np.all(r[neg_big] == -65504.0)
    m = ~(big | neg_big)
    assert np.all(r[m] >= x[m])
    preds = np.array([_pred_f16(v) for v in r[m]], np.float64)
    assert np.all(preds < x[m])


# ---------------------------------------------------------------- packing
def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([p.strip() for p in line.split("|")])
    return rows


def test_canonical_pack_hand_bytes():
    for bits, codes, expect in _read_table("pack_hand.txt"):
        b = int(bits)
        c = np.array([[int(v) for v in codes.split()]], np.uint8)
        exp = bytes(int(v, 16) for v in expect.split())
        got = orc.pack(c, b).tobytes()
        assert got == exp, (bits, codes, got.hex(), exp.hex())
        assert np.array_equal(orc.unpack(np.frombuffer(exp, np.uint8), 1, c.shape[1], b), c)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("layout", [orc.LAYOUT_CANONICAL, orc.LAYOUT_KERNEL])
def test_pack_unpack_identity(bits, layout):
    g = np.random.default_rng(bits + 10 * layout)
    n, k = 48, 512
    codes = g.integers(0, 1 << bits, (n, k)).astype(np.uint8)
    p = orc.pack(codes, bits, layout)
    assert p.size == n * k * bits // 8
    assert np.array_equal(orc.unpack(p, n, k, bits, layout), codes)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
def test_kernel_layout_is_a_permutation_of_bits(bits):
    # same multiset of set bits per code width: popcount of the buffer equals
    # the total popcount of the codes
    g = np.random.default_rng(100 + bits)
    n, k = 32, 256
    codes = g.integers(0, 1 << bits, (n, k)).astype(np.uint8)
    p = orc.pack(codes, bits, orc.LAYOUT_KERNEL)
    pop = int(np.unpackbits(p).sum())
    assert pop == int(np.unpackbits(codes.reshape(-1, 1), axis=1)[:, 8 - bits:].sum())


def test_kernel_layout_hand_positions():
    for head, cell, pos in _read_table("kernel_layout_positions.txt"):
        b, n, k = (int(v) for v in head.split())
        row, col, code = (int(v) for v in cell.split())
        byte, bit = (int(v) for v in pos.split())
        codes = np.zeros((n, k), np.uint8)
        codes[row, col] = code
        p = orc.pack(codes, b, orc.LAYOUT_KERNEL)
        set_bits = np.flatnonzero(np.unpackbits(p, bitorder="little"))
        assert list(set_bits) == [8 * byte + bit], (head, cell, list(set_bits))


def test_sign_kernel_layout_hand_positions():
    for head, cell, pos in _read_table("sign_layout_positions.txt"):
        rows, cols = (int(v) for v in head.split())
        r, c = (int(v) for v in cell.split())
        byte, bit = (int(v) for v in pos.split())
        words = np.zeros((rows, cols // 32), np.uint32)
        words[r, c // 32] = np.uint32(1 << (c % 32))
        p = orc.pack_signs_kernel(words, rows, cols)
        assert p.size == rows * orc.sign_cols_pad(cols) // 8
        set_bits = np.flatnonzero(np.unpackbits(p, bitorder="little"))
        assert list(set_bits) == [8 * byte + bit], (head, cell, list(set_bits))


def test_sign_pack_roundtrip_and_canonical_bits():
    pm = synth.pm1(32, 96, seed=3).numpy()
    words = orc.pack_signs(pm)
    # canonical: element c at bit c%32 of word c/32, bit 1 = +1 (numpy unpackbits route)
    bits = np.unpackbits(words.view(np.uint8).reshape(32, -1), axis=1, bitorder="little")
    assert np.array_equal(bits.astype(np.int8) * 2 - 1, pm)
    kp = orc.pack_signs_kernel(words, 32, 96)
    assert np.array_equal(orc.unpack_signs_kernel(kp, 32, 96), words)


# ---------------------------------------------------------------- RTN quantizer
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("group", [32, 64, 128])
def test_rtn_grid_identity(bits, group):
    """Weights already on the grid w = 2^-6 (q - z), with q spanning [0, 2^b-1]
    in every group, come back exactly as (q, s = 2^-6, z)."""
    g = np.random.default_rng(bits * 1000 + group)
    n, k = 8, 4 * group
    qmax = (1 << bits) - 1
    G = k // group
    q = g.integers(0, qmax + 1, (n, k))
    q[:, ::group] = 0
    q[:, 1::group] = qmax
    z = g.integers(0, qmax + 1, (n, G))
    w = (q - np.repeat(z, group, axis=1)) * 2.0 ** -6
    codes, s, zz = orc.quantize_rtn(_f16_bits(w), bits, group)
    assert np.array_equal(codes, q)
    assert np.all(_f16_val(s) == 2.0 ** -6)
    assert np.array_equal(_f16_val(zz), z.astype(np.float64))


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("group", [32, 64, 128])
def test_rtn_error_bound_and_nearest_level(bits, group):
    W = synth.weight(24, 512, seed=bits + group)
    Wb = synth.bits_u16(W)
    codes, s_bits, z_bits = orc.quantize_rtn(Wb, bits, group)
    qmax = (1 << bits) - 1
    assert codes.max() <= qmax
    w = _f16_val(Wb)
    s = np.repeat(_f16_val(s_bits), group, axis=1)
    z = np.repeat(_f16_val(z_bits), group, axis=1)
    assert np.all(z == np.round(z)) and z.min() >= 0 and z.max() <= qmax
    wh = s * (codes - z)
    err = np.abs(w - wh)
    assert np.all(err <= s / 2 * (1 + 2.0 ** -20))
    # brute force: no other code is strictly nearer (ties allowed)
    best = np.full(w.shape, np.inf)
    for cand in range(qmax + 1):
        best = np.minimum(best, np.abs(w - s * (cand - z)))
    assert np.all(err <= best * (1 + 1e-9) + 1e-30)
    # scale: the smallest fp16 >= the fp32 step (hi - lo) / (2^b - 1), numpy route
    wg = w.reshape(w.shape[0], -1, group)
    lo = np.minimum(wg.min(axis=2), 0).astype(np.float32)
    hi = np.maximum(wg.max(axis=2), 0).astype(np.float32)
    step = (hi - lo) / np.float32(qmax)
    sv = _f16_val(s_bits)
    assert np.all(sv >= step)
    preds = np.array([_pred_f16(v) for v in sv.ravel()], np.float64).reshape(sv.shape)
    assert np.all(preds < step)


def test_rtn_all_zero_group_and_nonfinite():
    W = np.zeros((16, 64), np.float16)
    codes, s, z = orc.quantize_rtn(W.view(np.uint16), 4, 32)
    assert np.all(codes == 0) and np.all(_f16_val(s) == 1.0) and np.all(_f16_val(z) == 0)
    W[3, 5] = np.inf
    with pytest.raises(FloatingPointError):
        orc.quantize_rtn(W.view(np.uint16), 4, 32)


# ---------------------------------------------------------------- group GEMV
def _dequant_numpy(codes, s_bits, z_bits, group):
    s = np.repeat(_f16_val(s_bits), group, axis=1)
    z = np.repeat(_f16_val(z_bits), group, axis=1)
    return s * (codes.astype(np.float64) - z)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("layout", [orc.LAYOUT_CANONICAL, orc.LAYOUT_KERNEL])
def test_gemv_group_matches_numpy_matmul(bits, layout):
    n, k, group, M = 32, 512, 64, 3
    W = synth.weight(n, k, seed=7 * bits)
    x = synth.activations(M, k, seed=8)
    codes, s, z = orc.quantize_rtn(synth.bits_u16(W), bits, group)
    y = orc.gemv_group(synth.bits_u16(x), orc.pack(codes, bits, layout), s, z, n, k,
                       bits, group, layout=layout)
    ref = _f16_val(synth.bits_u16(x)) @ _dequant_numpy(codes, s, z, group).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    # row subset returns the same columns
    rows = np.array([5, 0, 31])
    ys = orc.gemv_group(synth.bits_u16(x), orc.pack(codes, bits, layout), s, z, n, k,
                        bits, group, layout=layout, rows=rows)
    assert np.array_equal(ys, y[:, rows])


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
def test_gemv_on_grid_weights_equals_dense(bits):
    """b-bit weights already on the grid: the group product is the dense x W^T."""
    g = np.random.default_rng(bits)
    n, k, group = 16, 256, 32
    qmax = (1 << bits) - 1
    q = g.integers(0, qmax + 1, (n, k))
    q[:, ::group] = 0
    q[:, 1::group] = qmax
    zg = g.integers(0, qmax + 1, (n, k // group))
    w = (q - np.repeat(zg, group, axis=1)) * 2.0 ** -6
    Wb = _f16_bits(w)
    x = synth.bits_u16(synth.activations(2, k, seed=bits))
    codes, s, z = orc.quantize_rtn(Wb, bits, group)
    for layout in (orc.LAYOUT_CANONICAL, orc.LAYOUT_KERNEL):
        y = orc.gemv_group(x, orc.pack(codes, bits, layout), s, z, n, k, bits, group, layout=layout)
        assert np.array_equal(y, orc.gemv_dense(x, Wb))


def test_gemv_bf16_activations():
    n, k = 16, 128
    W = synth.weight(n, k, seed=1)
    x = synth.activations(2, k, seed=2, dtype=torch.bfloat16)
    codes, s, z = orc.quantize_rtn(synth.bits_u16(W), 4, 128)
    y = orc.gemv_group(synth.bits_u16(x), orc.pack(codes, 4), s, z, n, k, 4, 128, x_is_bf16=True)
    ref = x.double().numpy() @ _dequant_numpy(codes, s, z, 128).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_single_code_change_moves_one_output_by_closed_form():
    """Positions of a 16x256 2-bit matrix, in both layouts: raising one code by 1
    changes only that row's output, by x[k] * s."""
    n, k, bits, group = 16, 256, 2, 32
    g = np.random.default_rng(5)
    codes = g.integers(0, 3, (n, k)).astype(np.uint8)          # room for +1
    s = _f16_bits(np.full((n, k // group), 0.5))
    z = _f16_bits(np.ones((n, k // group)))
    x = _f16_bits(g.standard_normal((1, k)))
    xv = _f16_val(x)[0]
    for layout in (orc.LAYOUT_CANONICAL, orc.LAYOUT_KERNEL):
        base = orc.gemv_group(x, orc.pack(codes, bits, layout), s, z, n, k, bits, group, layout=layout)
        for (i, kk) in [(0, 0), (15, 255), (7, 64), (9, 33), (3, 100), (12, 201)]:
            c2 = codes.copy()
            c2[i, kk] += 1
            y2 = orc.gemv_group(x, orc.pack(c2, bits, layout), s, z, n, k, bits, group, layout=layout)
            d = y2 - base
            assert abs(d[0, i] - 0.5 * xv[kk]) < 1e-12
            d[0, i] = 0
            assert np.all(np.abs(d) < 1e-12)


# ---------------------------------------------------------------- binary low-rank
def _signs_numpy(words, cols):
    b = np.unpackbits(np.ascontiguousarray(words).view(np.uint8).reshape(words.shape[0], -1),
                      axis=1, bitorder="little")[:, :cols]
    return b.astype(np.float64) * 2 - 1


def _binlr_case(d_out, d_in, r, M, seed):
    U = synth.words_u32(synth.sign_words(d_out, r, seed))
    Vt = synth.words_u32(synth.sign_words(r, d_in, seed + 1))
    s1 = synth.bits_u16(synth.channel_scales(d_out, seed + 2))
    s2 = synth.bits_u16(synth.channel_scales(d_in, seed + 3))
    x = synth.bits_u16(synth.activations(M, d_in, seed + 4))
    return x, U, Vt, s1, s2


def test_binlr_explicit_matches_numpy_and_factored():
    d_out, d_in, r, M = 48, 64, 32, 2
    x, U, Vt, s1, s2 = _binlr_case(d_out, d_in, r, M, 11)
    yd = orc.binlr_dense(x, U, Vt, s1, s2, d_out, d_in, r)
    yf = orc.binlr_factored(x, U, Vt, s1, s2, d_out, d_in, r)
    Wh = np.diag(_f16_val(s1)) @ _signs_numpy(U, r) @ _signs_numpy(Vt, d_in) @ np.diag(_f16_val(s2))
    ref = _f16_val(x) @ Wh.T
    assert np.allclose(yd, ref, rtol=1e-12, atol=1e-14)
    assert np.linalg.norm(yd - yf) <= 1e-12 * np.linalg.norm(yd)


def test_binlr_brute_force_python_loops():
    d_out, d_in, r = 2, 32, 32
    x, U, Vt, s1, s2 = _binlr_case(d_out, d_in, r, 1, 21)
    sU = [[1 if (int(U[i, j // 32]) >> (j % 32)) & 1 else -1 for j in range(r)] for i in range(d_out)]
    sV = [[1 if (int(Vt[j, c // 32]) >> (c % 32)) & 1 else -1 for c in range(d_in)] for j in range(r)]
    xs = _f16_val(x)[0]
    a, b = _f16_val(s1), _f16_val(s2)
    for i in range(d_out):
        tot = 0.0
        for c in range(d_in):
            wic = sum(sU[i][j] * sV[j][c] for j in range(r)) * a[i] * b[c]
            tot += xs[c] * wic
        y = orc.binlr_factored(x, U, Vt, s1, s2, d_out, d_in, r)[0, i]
        assert abs(y - tot) <= 1e-12 * max(1.0, abs(tot))


def test_binlr_all_plus_one_closed_form():
    d_out, d_in, r = 16, 64, 64
    U = np.full((d_out, r // 32), 0xFFFFFFFF, np.uint32)
    Vt = np.full((r, d_in // 32), 0xFFFFFFFF, np.uint32)
    _, _, _, s1, s2 = _binlr_case(d_out, d_in, r, 1, 31)
    x = synth.bits_u16(synth.activations(1, d_in, 32))
    y = orc.binlr_factored(x, U, Vt, s1, s2, d_out, d_in, r)[0]
    expect = r * _f16_val(s1) * float(np.dot(_f16_val(s2), _f16_val(x)[0]))
    assert np.allclose(y, expect, rtol=1e-12)


def test_binlr_single_sign_flip():
    d_out, d_in, r = 16, 64, 32
    x, U, Vt, s1, s2 = _binlr_case(d_out, d_in, r, 1, 41)
    y0, t0 = orc.binlr_factored(x, U, Vt, s1, s2, d_out, d_in, r, return_t=True)
    i, j = 5, 17
    U2 = U.copy()
    U2[i, j // 32] ^= np.uint32(1 << (j % 32))
    y1 = orc.binlr_factored(x, U2, Vt, s1, s2, d_out, d_in, r)
    old = 1.0 if (int(U[i, j // 32]) >> (j % 32)) & 1 else -1.0
    d = y1 - y0
    assert abs(d[0, i] - (-2 * old * _f16_val(s1)[i] * t0[0, j])) < 1e-12
    d[0, i] = 0
    assert np.all(d == 0)
    # flipping V^T[j, c] changes t_j by -2*sign*s2_c*x_c and y by s1*U[:,j]*dt
    c = 40
    Vt2 = Vt.copy()
    Vt2[j, c // 32] ^= np.uint32(1 << (c % 32))
    y2, t2 = orc.binlr_factored(x, U, Vt2, s1, s2, d_out, d_in, r, return_t=True)
    sv = 1.0 if (int(Vt[j, c // 32]) >> (c % 32)) & 1 else -1.0
    dt = -2 * sv * _f16_val(s2)[c] * _f16_val(x)[0, c]
    assert abs((t2 - t0)[0, j] - dt) < 1e-12
    uj = _signs_numpy(U, r)[:, j]
    assert np.allclose(y2 - y0, (_f16_val(s1) * uj * dt)[None, :], atol=1e-12)


def test_binlr_row_subset():
    d_out, d_in, r = 64, 64, 32
    x, U, Vt, s1, s2 = _binlr_case(d_out, d_in, r, 2, 51)
    y = orc.binlr_factored(x, U, Vt, s1, s2, d_out, d_in, r)
    rows = np.array([63, 2, 7])
    assert np.array_equal(orc.binlr_factored(x, U, Vt, s1, s2, d_out, d_in, r, rows=rows), y[:, rows])
