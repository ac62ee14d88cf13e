"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Codes, scales, zeros and packed bytes must match bit for bit; GEMV/GEMM
outputs must be within relative L2 error 1e-3 of the oracle's fp64 result
(fp32 accumulation, fp16/bf16 outputs).  Small shapes are compared in full
(spanning several tiles, split-K fixups and ragged row blocks); the
Llama-2-70B-shaped layers are compared on seeded samples of output rows.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from quantized_gemv_group_b200 import lbq, synth
from quantized_gemv_group_b200 import workloads as wl

pytestmark = pytest.mark.gpu

REL_TOL = 1e-3
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_gemv_group_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lbq.lib()


def _u16(t):
    return synth.bits_u16(t)


def _np(t):
    return t.detach().cpu().numpy()


def _rel(a, b):
    return orc.rel_l2(a, b)


def _quantize_both(W, bits, group):
    codes, s, z = lbq.lbq_quantize_rtn(W, bits, group)
    torch.cuda.synchronize()
    oc, os_, oz = orc.quantize_rtn(_u16(W), bits, group, w_is_bf16=(W.dtype == torch.bfloat16))
    return (codes, s, z), (oc, os_, oz)


# ---------------------------------------------------------------- quantize / pack
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_quantize_bit_exact(bits, group, dtype):
    W = synth.weight(96, 1024, seed=bits * 7 + group, device=DEV, dtype=dtype)
    (c, s, z), (oc, os_, oz) = _quantize_both(W, bits, group)
    assert np.array_equal(_np(c), oc)
    assert np.array_equal(_u16(s), os_)
    assert np.array_equal(_u16(z), oz)


def test_quantize_config0_and_degenerate_groups():
    # tiny correctness workload: 256x256 fp16, seed 0, INT4 group 32
    W = synth.weight(256, 256, seed=0, device=DEV)
    W[3, :32] = 0                               # all-zero group -> s = 1, z = 0
    W[4, 32:64] = 1e-7                          # subnormal-range step
    (c, s, z), (oc, os_, oz) = _quantize_both(W, 4, 32)
    assert np.array_equal(_np(c), oc) and np.array_equal(_u16(s), os_) and np.array_equal(_u16(z), oz)
    assert _np(s.float())[3, 0] == 1.0


def test_quantize_nonfinite_sets_device_error():
    assert lbq.lbq_last_device_error() == 0
    W = synth.weight(16, 64, seed=1, device=DEV)
    W[2, 7] = float("inf")
    lbq.lbq_quantize_rtn(W, 4, 32)
    assert lbq.lbq_last_device_error() & 1
    assert lbq.lbq_last_device_error() == 0       # read clears it


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("layout", [lbq.LAYOUT_CANONICAL, lbq.LAYOUT_KERNEL])
def test_pack_bit_exact(bits, layout):
    g = torch.Generator(device=DEV)
    g.manual_seed(bits)
    n, k = 48, 512
    codes = torch.randint(0, 1 << bits, (n, k), generator=g, device=DEV, dtype=torch.int32).to(torch.uint8)
    packed = lbq.lbq_pack(codes, bits, layout)
    ref = orc.pack(_np(codes), bits, layout)
    assert np.array_equal(_np(packed), ref)
    back = lbq.lbq_unpack(packed, n, k, bits, layout)
    assert torch.equal(back, codes)


@pytest.mark.parametrize("rows,cols", [(16, 256), (48, 96), (64, 800)])
def test_sign_pack_bit_exact(rows, cols):
    pm = synth.pm1(rows, cols, seed=rows + cols, device=DEV)
    canon = lbq.lbq_pack_signs(pm, lbq.LAYOUT_CANONICAL)
    ref = orc.pack_signs(_np(pm))
    assert np.array_equal(_np(canon).view(np.uint32).reshape(rows, cols // 32), ref)
    kern = lbq.lbq_pack_signs(pm, lbq.LAYOUT_KERNEL)
    kref = orc.pack_signs_kernel(ref, rows, cols)
    assert np.array_equal(_np(kern), kref)
    words = synth.sign_words(rows, cols, seed=5, device=DEV)
    rep = lbq.lbq_repack_signs(words, rows, cols)
    assert np.array_equal(_np(rep), orc.pack_signs_kernel(synth.words_u32(words), rows, cols))


# ---------------------------------------------------------------- group GEMV
def _group_case(n, k, bits, group, M, seed, xdtype=torch.float16):
    W = synth.weight(n, k, seed=seed, device=DEV)
    x = synth.activations(M, k, seed=seed + 1, device=DEV, dtype=xdtype)
    codes, s, z = lbq.lbq_quantize_rtn(W, bits, group)
    return W, x, codes, s, z


def _oracle_group(x, codes, s, z, n, k, bits, group, rows=None):
    return orc.gemv_group(_u16(x), orc.pack(_np(codes), bits), _u16(s), _u16(z), n, k, bits, group,
                          rows=rows, x_is_bf16=(x.dtype == torch.bfloat16))


def test_config0_group_gemv_int4_g32():
    n = k = 256
    W, x, codes, s, z = _group_case(n, k, 4, 32, 1, seed=0)
    ref = _oracle_group(x, codes, s, z, n, k, 4, 32)
    for layout in (lbq.LAYOUT_CANONICAL, lbq.LAYOUT_KERNEL):
        packed = lbq.lbq_pack(codes, 4, layout)
        y = lbq.lbq_gemv_group(x, packed, s, z, n, k, 4, 32, layout)
        assert _rel(_np(y.float()), ref) <= REL_TOL


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("layout", [lbq.LAYOUT_CANONICAL, lbq.LAYOUT_KERNEL])
@pytest.mark.parametrize("M", [1, 3, 9, 16])
def test_group_gemv_sweep(bits, group, layout, M):
    # 400 rows = 25 tiles (last 128-row block ragged); k = 1024 spans several superblocks
    n, k = 400, 1024
    W, x, codes, s, z = _group_case(n, k, bits, group, M, seed=100 * bits + group + M)
    ref = _oracle_group(x, codes, s, z, n, k, bits, group)
    packed = lbq.lbq_pack(codes, bits, layout)
    y = lbq.lbq_gemv_group(x, packed, s, z, n, k, bits, group, layout)
    assert _rel(_np(y.float()), ref) <= REL_TOL


@pytest.mark.parametrize("bits,group", [(4, 128), (4, 64), (2, 32), (6, 32)])
def test_group_gemv_bf16_activations(bits, group):
    n, k, M = 256, 2048, 5
    W, x, codes, s, z = _group_case(n, k, bits, group, M, seed=7, xdtype=torch.bfloat16)
    ref = _oracle_group(x, codes, s, z, n, k, bits, group)
    y = lbq.lbq_gemv_group(x, lbq.lbq_pack(codes, bits), s, z, n, k, bits, group)
    assert y.dtype == torch.float16                 # outputs are fp16 for either input type
    assert _rel(_np(y.float()), ref) <= REL_TOL


@pytest.mark.parametrize("bits,group,k", [(4, 64, 320), (2, 32, 384), (6, 64, 640), (4, 128, 1152), (3, 32, 96)])
@pytest.mark.parametrize("M", [1, 12])
def test_group_gemv_canonical_odd_shapes(bits, group, k, M):
    """Shapes outside the kernel layout (k not a multiple of 256, or k/group not a
    multiple of 8) run through the canonical layout; same parity bar."""
    n = 40
    W, x, codes, s, z = _group_case(n, k, bits, group, M, seed=k + bits)
    ref = _oracle_group(x, codes, s, z, n, k, bits, group)
    y = lbq.lbq_gemv_group(x, lbq.lbq_pack(codes, bits, lbq.LAYOUT_CANONICAL), s, z, n, k, bits, group,
                           lbq.LAYOUT_CANONICAL)
    assert _rel(_np(y.float()), ref) <= REL_TOL


def test_kernel_layout_rejects_unsupported_scale_stride():
    # k/group = 2 is not a multiple of 8: the kernel path refuses, launching nothing
    n, k = 32, 256
    W, x, codes, s, z = _group_case(n, k, 4, 128, 1, seed=3)
    packed = lbq.lbq_pack(codes, 4)
    with pytest.raises(lbq.LbqError) as ei:
        lbq.lbq_gemv_group(x, packed, s, z, n, k, 4, 128)
    assert ei.value.status == lbq.ERR_UNSUPPORTED


def test_group_gemv_deterministic_and_split_k():
    # n = 1024 (k/v-like): few row blocks, so every block is split across CTAs
    n, k = 1024, 8192
    W, x, codes, s, z = _group_case(n, k, 4, 64, 1, seed=11)
    packed = lbq.lbq_pack(codes, 4)
    y1 = lbq.lbq_gemv_group(x, packed, s, z, n, k, 4, 64).clone()
    y2 = lbq.lbq_gemv_group(x, packed, s, z, n, k, 4, 64).clone()
    assert torch.equal(y1, y2)
    ref = _oracle_group(x, codes, s, z, n, k, 4, 64)
    assert _rel(_np(y1.float()), ref) <= REL_TOL


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("bits,group", [(4, 64), (2, 32), (5, 32), (3, 128)])
def test_gemv_group_multi_matches_each_product(M, bits, group):
    """One grouped launch of heterogeneous products (the q/k/v pattern: shared x,
    different n; plus a product with its own x and k) equals the oracle per product."""
    shapes = [(400, 1024), (64, 1024), (64, 1024), (256, 2048)]
    xa = synth.activations(M, 1024, seed=5, device=DEV)
    xb = synth.activations(M, 2048, seed=6, device=DEV)
    probs, refs = [], []
    for i, (n, k) in enumerate(shapes):
        W = synth.weight(n, k, seed=50 + i + 10 * bits, device=DEV)
        codes, s, z = lbq.lbq_quantize_rtn(W, bits, group)
        x = xa if k == 1024 else xb
        y = torch.full((M, n), float("nan"), dtype=torch.float16, device=DEV)
        probs.append((x, lbq.lbq_pack(codes, bits), s, z, y, n, k))
        refs.append(_oracle_group(x, codes, s, z, n, k, bits, group))
    lbq.lbq_gemv_group_multi(probs, bits, group)
    for pr, ref in zip(probs, refs):
        assert _rel(_np(pr[4].float()), ref) <= REL_TOL


def test_gemv_group_multi_argument_errors():
    x = torch.zeros(1, 256, dtype=torch.float16, device=DEV)
    codes = torch.zeros(16, 256, dtype=torch.uint8, device=DEV)
    s = torch.ones(16, 8, dtype=torch.float16, device=DEV)
    z = torch.zeros(16, 8, dtype=torch.float16, device=DEV)
    y = torch.empty(1, 16, dtype=torch.float16, device=DEV)
    pr = (x, lbq.lbq_pack(codes, 4), s, z, y, 16, 256)
    with pytest.raises(lbq.LbqError):
        lbq.lbq_gemv_group_multi([pr] * 9, 4, 32)             # more than LBQ_MAX_GEMV_PROBLEMS
    with pytest.raises(lbq.LbqError):
        lbq.lbq_gemv_group_multi([pr], 7, 32)                  # bad bit width


def test_gemm_group_small_m_blocks():
    n, k, M = 256, 1024, 37                       # 16 + 16 + 5 tokens
    W, x, codes, s, z = _group_case(n, k, 4, 128, M, seed=21, xdtype=torch.bfloat16)
    ref = _oracle_group(x, codes, s, z, n, k, 4, 128)
    y = lbq.lbq_gemm_group(x, lbq.lbq_pack(codes, 4), s, z, n, k, 4, 128)
    assert _rel(_np(y.float()), ref) <= REL_TOL


# ---------------------------------------------------------------- batched GEMM on tcgen05 (M >= 64)
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("M", [64, 100, 200, 300])
def test_gemm_group_tc_sweep(bits, group, M):
    # 400 rows: three full 128-row blocks and a ragged 16-row block; M = 64 / 100 / 200 / 300
    # takes token tiles of 64, 128 (ragged), 256 (ragged) and two tiles of 256.
    n, k = 400, 1024
    xdtype = torch.bfloat16 if (bits + M) % 2 else torch.float16
    W, x, codes, s, z = _group_case(n, k, bits, group, M, seed=7 * bits + group + M, xdtype=xdtype)
    ref = _oracle_group(x, codes, s, z, n, k, bits, group)
    y = lbq.lbq_gemm_group(x, lbq.lbq_pack(codes, bits), s, z, n, k, bits, group)
    torch.cuda.synchronize()
    assert lbq.lbq_last_device_error() == 0
    assert _rel(_np(y.float()), ref) <= REL_TOL
    # each output element, not only the aggregate: fp16 weights and fp32 accumulation
    yf = _np(y.float()).astype(np.float64)
    scale = np.abs(ref).max()
    assert np.max(np.abs(yf - ref)) <= 2e-2 * scale


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 32), (6, 64)])
@pytest.mark.parametrize("M", [64, 200])
def test_gemm_group_tc_split_k(bits, group, M):
    # 2 row blocks with k = 4096 (16 superblocks): the tile count is far below the SM count,
    # so k is split in 4 slices whose fp32 partials are added by the last slice to finish
    n, k = 256, 4096
    W, x, codes, s, z = _group_case(n, k, bits, group, M, seed=11 * bits + M, xdtype=torch.bfloat16)
    ref = _oracle_group(x, codes, s, z, n, k, bits, group)
    packed = lbq.lbq_pack(codes, bits)
    y1 = lbq.lbq_gemm_group(x, packed, s, z, n, k, bits, group).clone()
    y2 = lbq.lbq_gemm_group(x, packed, s, z, n, k, bits, group).clone()
    torch.cuda.synchronize()
    assert lbq.lbq_last_device_error() == 0
    assert _rel(_np(y1.float()), ref) <= REL_TOL
    assert torch.equal(y1, y2)                     # fixed slice order: deterministic


def test_gemm_binlr_tc_split_k():
    d_out, d_in, r, M = 256, 4096, 64, 100
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, M, seed=77)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL, fn=lbq.lbq_gemm_binlr)
    torch.cuda.synchronize()
    assert lbq.lbq_last_device_error() == 0
    ref = _binlr_oracle(Uw, Vw, s1, s2, x, d_out, d_in, r)
    assert _rel(_np(y.float()), ref) <= REL_TOL


def test_gemm_group_tc_deterministic_and_matches_gemv_blocks():
    n, k, M = 256, 2048, 96
    W, x, codes, s, z = _group_case(n, k, 4, 64, M, seed=31)
    packed = lbq.lbq_pack(codes, 4)
    y1 = lbq.lbq_gemm_group(x, packed, s, z, n, k, 4, 64).clone()
    y2 = lbq.lbq_gemm_group(x, packed, s, z, n, k, 4, 64).clone()
    assert torch.equal(y1, y2)
    # the 16-token GEMV blocks compute the same product
    yb = torch.cat([lbq.lbq_gemv_group(x[m0:m0 + 16].contiguous(), packed, s, z, n, k, 4, 64)
                    for m0 in range(0, M, 16)])
    assert _rel(_np(y1.float()), _np(yb.float()).astype(np.float64)) <= REL_TOL


def test_group_gemv_empty_inputs():
    x = torch.zeros(0, 256, dtype=torch.float16, device=DEV)
    codes = torch.zeros(16, 256, dtype=torch.uint8, device=DEV)
    s = torch.ones(16, 8, dtype=torch.float16, device=DEV)
    z = torch.zeros(16, 8, dtype=torch.float16, device=DEV)
    y = lbq.lbq_gemv_group(x, lbq.lbq_pack(codes, 4), s, z, 16, 256, 4, 32)
    assert y.shape == (0, 16)


# ---------------------------------------------------------------- binary low-rank
def _binlr_case(d_out, d_in, r, M, seed, xdtype=torch.float16):
    Uw = synth.sign_words(d_out, r, seed, device=DEV)
    Vw = synth.sign_words(r, d_in, seed + 1, device=DEV)
    s1 = synth.channel_scales(d_out, seed + 2, device=DEV)
    s2 = synth.channel_scales(d_in, seed + 3, device=DEV)
    x = synth.activations(M, d_in, seed + 4, device=DEV, dtype=xdtype)
    return Uw, Vw, s1, s2, x


def _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, layout, fn=None):
    if layout == lbq.LAYOUT_KERNEL:
        U = lbq.lbq_repack_signs(Uw, d_out, r)
        Vt = lbq.lbq_repack_signs(Vw, r, d_in)
    else:
        U, Vt = Uw, Vw
    fn = fn or lbq.lbq_gemv_binlr
    return fn(x, U, Vt, s1, s2, d_out, d_in, r, layout)


def _binlr_oracle(Uw, Vw, s1, s2, x, d_out, d_in, r, rows=None):
    return orc.binlr_factored(_u16(x), synth.words_u32(Uw), synth.words_u32(Vw), _u16(s1), _u16(s2), d_out,
                              d_in, r, rows=rows, x_is_bf16=(x.dtype == torch.bfloat16))


@pytest.mark.parametrize("layout", [lbq.LAYOUT_CANONICAL, lbq.LAYOUT_KERNEL])
def test_config0_binlr(layout):
    d_out = d_in = 256
    r = 64
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, 1, seed=0)
    ref = orc.binlr_dense(_u16(x), synth.words_u32(Uw), synth.words_u32(Vw), _u16(s1), _u16(s2), d_out, d_in, r)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, layout)
    assert _rel(_np(y.float()), ref) <= REL_TOL


@pytest.mark.parametrize("layout", [lbq.LAYOUT_CANONICAL, lbq.LAYOUT_KERNEL])
@pytest.mark.parametrize("M", [1, 4, 5, 9, 16])
def test_binlr_sweep(layout, M):
    d_out, d_in, r = 400, 544, 96                 # padding of both K extents, ragged row blocks
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, M, seed=M)
    ref = _binlr_oracle(Uw, Vw, s1, s2, x, d_out, d_in, r)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, layout)
    assert _rel(_np(y.float()), ref) <= REL_TOL


def test_binlr_bf16_and_gemm_blocks():
    d_out, d_in, r, M = 256, 1024, 128, 21
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, M, seed=3, xdtype=torch.bfloat16)
    ref = _binlr_oracle(Uw, Vw, s1, s2, x, d_out, d_in, r)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL, fn=lbq.lbq_gemm_binlr)
    assert _rel(_np(y.float()), ref) <= REL_TOL


def test_binlr_deterministic():
    d_out, d_in, r = 1024, 8192, 736
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, 1, seed=9)
    y1 = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL).clone()
    y2 = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL).clone()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("shape", [(400, 288, 96), (256, 1024, 160), (128, 512, 256)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("M", [64, 100, 300])
def test_gemm_binlr_tc(shape, M):
    # d_in = 288 and r = 96 / 160 leave 256-column padding in the sign layout; r = 96 and
    # d_out = 400 leave ragged 128-row blocks; M = 100 / 300 leave ragged token tiles.
    d_out, d_in, r = shape
    xdtype = torch.bfloat16 if M == 100 else torch.float16
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, M, seed=d_out + r + M, xdtype=xdtype)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL, fn=lbq.lbq_gemm_binlr)
    torch.cuda.synchronize()
    assert lbq.lbq_last_device_error() == 0
    ref = _binlr_oracle(Uw, Vw, s1, s2, x, d_out, d_in, r)
    assert _rel(_np(y.float()), ref) <= REL_TOL
    # the 16-token GEMV blocks compute the same product
    yb = torch.cat([_binlr_run(Uw, Vw, s1, s2, x[m0:m0 + 16].contiguous(), d_out, d_in, r, lbq.LAYOUT_KERNEL)
                    for m0 in range(0, M, 16)])
    assert _rel(_np(yb.float()), ref) <= REL_TOL


def test_gemm_binlr_tc_all_plus_one():
    # U = V = all +1: y[m, i] = r * s1[i] * sum_k s2[k] x[m, k]
    d_out, d_in, r, M = 128, 256, 64, 64
    Uw = torch.full((d_out, r // 32), -1, dtype=torch.int32, device=DEV)
    Vw = torch.full((r, d_in // 32), -1, dtype=torch.int32, device=DEV)
    s1 = synth.channel_scales(d_out, 1, device=DEV)
    s2 = synth.channel_scales(d_in, 2, device=DEV)
    x = synth.activations(M, d_in, 3, device=DEV)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL, fn=lbq.lbq_gemm_binlr)
    xs = _np(x.float()).astype(np.float64) @ _np(s2.float()).astype(np.float64)
    ref = r * np.outer(xs, _np(s1.float()).astype(np.float64))
    assert _rel(_np(y.float()), ref) <= REL_TOL


# ---------------------------------------------------------------- full 70B shapes, sampled rows
def _sample_rows(n, count, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(count, n), replace=False))


@pytest.mark.parametrize("lin", wl.block_linears(), ids=lambda l: l.name)
def test_block_linears_int4_g64_sampled(lin):
    n, k = lin.d_out, lin.d_in
    seed = synth.tensor_seed(0, wl.PROJS.index(lin.name))
    W = synth.weight(n, k, seed=seed, device=DEV)
    x = synth.activations(1, k, seed=seed + 500, device=DEV)
    codes, s, z = lbq.lbq_quantize_rtn(W, 4, 64)
    rows = _sample_rows(n, 48, seed)
    # codes of the sampled rows are bit-exact with the oracle quantizer
    oc, os_, oz = orc.quantize_rtn(_u16(W[torch.from_numpy(rows).to(DEV)]), 4, 64)
    assert np.array_equal(_np(codes)[rows], oc)
    assert np.array_equal(_u16(s)[rows], os_) and np.array_equal(_u16(z)[rows], oz)
    packed = lbq.lbq_pack(codes, 4)
    y = lbq.lbq_gemv_group(x, packed, s, z, n, k, 4, 64)
    ref = orc.gemv_group(_u16(x), _np(packed), _u16(s), _u16(z), n, k, 4, 64, layout=orc.LAYOUT_KERNEL, rows=rows)
    assert _rel(_np(y.float())[:, rows], ref) <= REL_TOL


@pytest.mark.parametrize("M", [1, 3])
@pytest.mark.parametrize("bits,group", [(4, 64), (5, 32)], ids=["int4_g64_pairs", "int5_g32_tickets"])
def test_gemv_group_multi_qkv_full_grid_sampled(bits, group, M):
    """The grouped q/k/v launch at 70B shapes fills the grid: 16-warp shapes run as pairs of
    CTAs whose shared tile is finished across the cluster barrier, 8-warp shapes finish
    CTA-crossing tiles by ticket.  Sampled rows of every product match the oracle and a
    second launch gives the same bits."""
    shapes = [(8192, 8192), (1024, 8192), (1024, 8192)]
    x = synth.activations(M, 8192, seed=31, device=DEV)
    probs, rows_l, ref_l = [], [], []
    for i, (n, k) in enumerate(shapes):
        W = synth.weight(n, k, seed=300 + i, device=DEV)
        codes, s, z = lbq.lbq_quantize_rtn(W, bits, group)
        del W
        packed = lbq.lbq_pack(codes, bits)
        y = torch.full((M, n), float("nan"), dtype=torch.float16, device=DEV)
        probs.append((x, packed, s, z, y, n, k))
        rows = _sample_rows(n, 24, 40 + i)
        rows_l.append(rows)
        ref_l.append(orc.gemv_group(_u16(x), _np(packed), _u16(s), _u16(z), n, k, bits, group,
                                    layout=orc.LAYOUT_KERNEL, rows=rows))
    lbq.lbq_gemv_group_multi(probs, bits, group)
    first = [pr[4].clone() for pr in probs]
    lbq.lbq_gemv_group_multi(probs, bits, group)
    for pr, y1, rows, ref in zip(probs, first, rows_l, ref_l):
        assert torch.equal(pr[4], y1)
        assert not torch.isnan(pr[4].float()).any()
        assert _rel(_np(pr[4].float())[:, rows], ref) <= REL_TOL


@pytest.mark.parametrize("shape", [(28672, 8192), (8192, 28672)], ids=["gate_up", "down"])
@pytest.mark.parametrize("M", [4, 16])
def test_prefill_shapes_int4_g128_bf16_sampled(shape, M):
    n, k = shape
    W = synth.weight(n, k, seed=77, device=DEV)
    x = synth.activations(M, k, seed=78, device=DEV, dtype=torch.bfloat16)
    codes, s, z = lbq.lbq_quantize_rtn(W, 4, 128)
    packed = lbq.lbq_pack(codes, 4)
    y = lbq.lbq_gemm_group(x, packed, s, z, n, k, 4, 128)
    rows = _sample_rows(n, 32, 5)
    ref = orc.gemv_group(_u16(x), _np(packed), _u16(s), _u16(z), n, k, 4, 128, layout=orc.LAYOUT_KERNEL,
                         rows=rows, x_is_bf16=True)
    assert _rel(_np(y.float())[:, rows], ref) <= REL_TOL


@pytest.mark.parametrize("shape", [(28672, 8192), (8192, 28672)], ids=["gate_up", "down"])
@pytest.mark.parametrize("M", [64, 256, 1024])
def test_gemm_tc_70b_shapes_int4_g128_bf16_sampled(shape, M):
    n, k = shape
    W = synth.weight(n, k, seed=79, device=DEV)
    x = synth.activations(M, k, seed=80, device=DEV, dtype=torch.bfloat16)
    codes, s, z = lbq.lbq_quantize_rtn(W, 4, 128)
    packed = lbq.lbq_pack(codes, 4)
    y = lbq.lbq_gemm_group(x, packed, s, z, n, k, 4, 128)
    torch.cuda.synchronize()
    assert lbq.lbq_last_device_error() == 0
    rows = _sample_rows(n, 24, 6)
    ref = orc.gemv_group(_u16(x), _np(packed), _u16(s), _u16(z), n, k, 4, 128, layout=orc.LAYOUT_KERNEL,
                         rows=rows, x_is_bf16=True)
    assert _rel(_np(y.float())[:, rows], ref) <= REL_TOL


@pytest.mark.parametrize("shape,M", [((28672, 8192), 64), ((28672, 8192), 256), ((8192, 28672), 64)],
                         ids=["gate_up-64", "gate_up-256", "down-64"])
def test_gemm_binlr_tc_70b_shapes_sampled(shape, M):
    d_out, d_in = shape
    r = wl.binlr_rank(d_out, d_in, 0.8)
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, M, seed=d_out + 3 * d_in, xdtype=torch.bfloat16)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL, fn=lbq.lbq_gemm_binlr)
    torch.cuda.synchronize()
    assert lbq.lbq_last_device_error() == 0
    rows = _sample_rows(d_out, 32, 4)
    ref = _binlr_oracle(Uw, Vw, s1, s2, x, d_out, d_in, r, rows=rows)
    assert _rel(_np(y.float())[:, rows], ref) <= REL_TOL


@pytest.mark.parametrize("shape", wl.BINLR_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("M", [1, 16])
def test_binlr_70b_shapes_sampled(shape, M):
    d_out, d_in = shape
    r = wl.binlr_rank(d_out, d_in, 0.8)
    Uw, Vw, s1, s2, x = _binlr_case(d_out, d_in, r, M, seed=d_out + d_in)
    y = _binlr_run(Uw, Vw, s1, s2, x, d_out, d_in, r, lbq.LAYOUT_KERNEL)
    rows = _sample_rows(d_out, 64, 3)
    ref = _binlr_oracle(Uw, Vw, s1, s2, x, d_out, d_in, r, rows=rows)
    assert _rel(_np(y.float())[:, rows], ref) <= REL_TOL
