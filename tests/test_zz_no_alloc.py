"""The group GEMV entry point that allocates nothing (lbq_gemv_group_noalloc).

Some callers cannot allocate device memory where they multiply (plugins handed no
workspace, code running after a pool allocator reserved all device memory, host
callbacks on a stream).  This entry point keeps its scratch in a fixed device array
owned by the library.  Its results must equal those of lbq_gemv_group, which takes
a caller-provided workspace, within the parity tolerance of the other GPU tests, on
two calls in a row (the second call finds the array as the first one left it).
This file is collected last so that a run stopping at the first failure has already
run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from quantized_gemv_group_b200 import lbq, synth

pytestmark = pytest.mark.gpu

REL_TOL = 1e-3


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_gemv_group_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lbq.lib()


@pytest.mark.parametrize("n,k,bits,group,M", [(1024, 8192, 4, 64, 1), (400, 1024, 3, 32, 5), (8192, 2048, 2, 128, 16)])
def test_noalloc_matches_workspace_entry_point(n, k, bits, group, M):
    dev = torch.device("cuda")
    W = synth.weight(n, k, seed=n + k, device=dev)
    codes, s, z = lbq.lbq_quantize_rtn(W, bits, group)
    packed = lbq.lbq_pack(codes, bits)
    ws = torch.zeros(lbq.lbq_workspace_bytes(lbq.OP_GEMV_GROUP, M, n, k), dtype=torch.uint8, device=dev)
    for call in range(2):
        x = synth.activations(M, k, seed=call + 7, device=dev)
        ref = lbq.lbq_gemv_group(x, packed, s, z, n, k, bits, group, ws=ws)
        y = lbq.lbq_gemv_group_noalloc(x, packed, s, z, n, k, bits, group)
        torch.cuda.synchronize()
        assert _rel(y, ref) <= REL_TOL, (call, _rel(y, ref))


def test_noalloc_rejects_problems_beyond_its_scratch():
    dev = torch.device("cuda")
    n, k, M = 16384 * 16, 256, 16             # 16384 tiles x 16 tokens of partial sums: far above 8 MiB
    x = torch.zeros(M, k, dtype=torch.float16, device=dev)
    packed = torch.zeros(n * k // 2, dtype=torch.uint8, device=dev)
    s = torch.ones(n, k // 32, dtype=torch.float16, device=dev)
    z = torch.zeros(n, k // 32, dtype=torch.float16, device=dev)
    with pytest.raises(lbq.LbqError) as ei:
        lbq.lbq_gemv_group_noalloc(x, packed, s, z, n, k, 4, 32)
    assert ei.value.status == lbq.ERR_SCRATCH_LIMIT
