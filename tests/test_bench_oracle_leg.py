"""Host checks of bench.py's oracle legs (cpu_baseline, --impl reference).

The legs quantize and pack only the 16-row tiles that hold the sampled rows.  That must
give exactly what the oracle gives on the whole matrix at the same rows, or the sampled
parity figure of the bench would compare against the wrong reference."""
import numpy as np
import torch

import bench
import oracle as orc
from quantized_gemv_group_b200 import synth, workloads as wl


def test_tile_subset_equals_full_matrix_oracle():
    dev = torch.device("cpu")
    (d,) = bench._oracle_block_inputs(dev, 8, only=["k_proj"])
    lin = wl.block_linears()[d["p"]]
    n, k = lin.d_out, lin.d_in
    W = synth.weight(n, k, seed=synth.tensor_seed(0, d["p"]), device=dev)
    codes, s, z = orc.quantize_rtn(synth.bits_u16(W), 4, 64)
    packed = orc.pack(codes, 4, layout=orc.LAYOUT_KERNEL)
    full = orc.gemv_group(d["xh"], packed, s, z, n, k, 4, 64, layout=orc.LAYOUT_KERNEL, rows=d["rows_global"])
    sub = orc.gemv_group(d["xh"], d["packed"], d["s"], d["z"], d["n_sub"], k, 4, 64, layout=orc.LAYOUT_KERNEL,
                         rows=d["rows"])
    assert len(d["rows_global"]) == n // 128
    assert np.array_equal(full, sub)


def test_reference_config_matches_block_workload_config():
    cfg = bench._block_config()
    assert cfg["shapes"] == [[l.d_out, l.d_in] for l in wl.block_linears()]
    assert cfg["bits"] == 4 and cfg["group"] == 64 and cfg["global_batch"] == 1
