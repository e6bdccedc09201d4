"""The decode-shaped GEMM for callers that cannot allocate device memory.

Callers that may not call cudaMalloc (code inside another framework's memory
pool, latency-critical paths that cannot afford cudaMalloc's implicit
synchronisation, plugin hosts that forbid allocation) use
fl_gemm_skinny_noalloc, whose split-K scratch is an array built into the
library.  It must give the same product as the same GEMM run with
caller-provided scratch (fl_test_gemm, swap_ab = 1), call after call, since
every call reuses the one array; shapes that do not fit the array are refused.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    from cross_loop_sparsity_b200 import build, flashloop as fl
    build.build()
    fl.lib()
    return torch, fl


def _operands(torch, m, n, k, seed):
    rng = np.random.default_rng(seed)
    A = torch.from_numpy(rng.standard_normal((m, k)).astype(np.float32)).to(torch.bfloat16).cuda()
    B = torch.from_numpy((rng.standard_normal((n, k)) * 0.05).astype(np.float32)).to(torch.bfloat16).cuda()
    return A, B


def test_no_alloc_gemm_matches_the_caller_scratch_gemm_on_two_calls(env):
    torch, fl = env
    # Both entry points run the same kernel with the same tile width, split
    # count and ordered ticket reduction, so the products must agree bit for bit.
    # Two calls in a row with different split counts: the second must not see
    # the first's tickets or partials.
    shapes = ((8, 3072, 2048, 1), (16, 2048, 5632, 2))
    ops = [_operands(torch, m, n, k, seed) for m, n, k, seed in shapes]
    wants = [fl.gemm(A, B, swap_ab=True) for A, B in ops]
    outs = [torch.empty((m, n), dtype=torch.float32, device="cuda") for m, n, _, _ in shapes]
    fl.gemm_noalloc(*ops[0], out=outs[0])      # first call on this device: looks up the array's address
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for (A, B), out, want in zip(ops, outs, wants):
        out.fill_(float("nan"))
        got = fl.gemm_noalloc(A, B, out=out)
        torch.cuda.synchronize()
        assert got.data_ptr() == out.data_ptr()
        assert torch.equal(got, want)
    # the calls allocated nothing: neither the device's free memory nor torch's pool moved
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_no_alloc_gemm_refuses_shapes_beyond_its_scratch(env):
    torch, fl = env
    A, B = _operands(torch, 64, 2048, 2048, 3)       # 9 splits x 16 tiles x 64 x 128 floats > 2 MiB
    with pytest.raises(fl.FlashLoopError) as exc:
        fl.gemm_noalloc(A, B)
    assert exc.value.status == 2
    assert "bytes of split-K scratch" in str(exc.value)
