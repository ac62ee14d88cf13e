"""Closed-form pins of the host-side tables (shapes, bit schedule, sizes)
against the figures the pages print (tests/golden/closed_forms.txt)."""
import os

import pytest

from quantized_gemv_group_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    out = {}
    with open(os.path.join(GOLDEN, "closed_forms.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, val, tol, _src = [p.strip() for p in line.split("|")]
                out[key] = (float(val), float(tol))
    return out


G = _golden()


def _close(key, value):
    ref, tol = G[key]
    assert abs(value - ref) <= tol * abs(ref), (key, value, ref)


def test_llama2_70b_fp16_size_matches_page():
    _close("fp16_70b_bytes", wl.llama2_70b_params() * 2)


def test_page_compression_ratios():
    _close("nanoquant_ratio_v1", 138.04 / 5.35)
    _close("nanoquant_ratio_v3", 137.95 / 5.75)


def test_int4_and_layer_sizes():
    _close("int4_70b_bytes", 70e9 / 2)
    per_layer = sum(l.d_in * l.d_out for l in wl.block_linears()) * 2
    _close("fp16_layer_bytes", per_layer)


def test_group_overhead_bits():
    _close("group_overhead_bits_g32", wl.group_bpw(4, 32) - 4)
    _close("group_overhead_bits_g16", wl.group_bpw(4, 16) - 4)
    for bits in range(2, 7):
        for g in (32, 64, 128):
            n, k = 8192, 8192
            assert wl.group_packed_bytes(n, k, bits, g) * 8 == pytest.approx(n * k * wl.group_bpw(bits, g))


def test_bit_schedule_within_page_range():
    bpw = wl.schedule_code_bits_per_weight()
    assert G["schedule_bpw_min"][0] <= bpw <= G["schedule_bpw_max"][0]
    for layer in range(wl.N_LAYERS):
        for p in wl.PROJS:
            b = wl.schedule_bits(layer, p)
            assert (b in (5, 6)) if p in wl.ATTN else (b in (2, 3))
    # code bytes of the 80-layer sweep ~ 25.5 GB, plus 1 bpw of g32 scale/zero
    n_w = wl.N_LAYERS * sum(l.d_in * l.d_out for l in wl.block_linears())
    assert abs(n_w * bpw / 8 / 1e9 - 25.47) < 0.01
    tot = sum(wl.group_packed_bytes(l.d_out, l.d_in, wl.schedule_bits(ly, l.name), 32)
              for ly in range(wl.N_LAYERS) for l in wl.block_linears())
    assert abs(tot / 1e9 - (25.47 + 8.56)) < 0.02


def test_binlr_rank_hits_target_bpw():
    for d_out, d_in in wl.BINLR_SHAPES:
        for bpw in wl.BINLR_BPW:
            r = wl.binlr_rank(d_out, d_in, bpw)
            assert r % 32 == 0
            # rounding r to a multiple of 32 moves bpw by at most 16 (d_out+d_in)/(d_out d_in)
            assert abs(wl.binlr_bpw(d_out, d_in, r) - bpw) <= 16 * (d_out + d_in) / (d_out * d_in)


def test_disk_time_model():
    # seconds per token ~ model bytes / read bandwidth
    _close("nvme_gen4_s_per_token", 140e9 / 7e9)
    _close("sata_s_per_token", 140e9 / 0.5e9)
