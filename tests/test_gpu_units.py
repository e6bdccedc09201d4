"""GPU unit parity through the C ABI: top-k selection and the residual
quantiser bit-exact against the oracle on identical inputs; the tcgen05 GEMM
against a plain fp64 product of the same bf16 operands."""
import numpy as np
import pytest

from cross_loop_sparsity_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    from cross_loop_sparsity_b200 import build, flashloop as fl
    build.build()
    fl.lib()
    from oracle import flashloop_oracle as orc
    return torch, fl, orc


@pytest.mark.parametrize("n,k,kind", [(1, 1, "ties"), (7, 3, "ties"), (100, 25, "ties"), (1000, 1000, "ties"),
                                      (1000, 1500, "ties"), (4097, 256, "ties"), (4097, 256, "distinct"),
                                      (16384, 2458, "ties"), (16384, 512, "distinct"), (65537, 1024, "ties"),
                                      (65537, 1, "distinct"), (8, 1, "distinct")])
def test_topk_bit_exact(env, n, k, kind):
    torch, fl, orc = env
    n_seg = 3
    keys = np.stack([synth.make_keys(1000 + 17 * s + n, n, kind) for s in range(n_seg)])
    if kind == "ties":
        keys[0, : min(n, 5)] = np.float32(np.inf)
        keys[1, n // 2] = np.float32(np.nan)
    got = fl.topk(torch.from_numpy(keys).cuda(), k).cpu().numpy()
    for s in range(n_seg):
        assert np.array_equal(got[s], orc.select_top(keys[s], k))


@pytest.mark.parametrize("width,g,bits", [(128, 32, 4), (128, 64, 4), (128, 128, 4), (128, 64, 2), (128, 128, 2),
                                          (256, 64, 4), (64, 32, 4), (64, 64, 4), (64, 32, 2), (64, 64, 2)])
def test_quantize_bit_exact(env, width, g, bits):
    torch, fl, orc = env
    rows = 2000
    r = synth.make_residuals(7 + width + g + bits, rows, width)
    codes, scales = fl.quantize(torch.from_numpy(r).cuda(), g, bits)
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy().view(np.float16)
    want_c, want_s = orc.quantize_groups(r, bits, g)
    assert np.array_equal(scales.view(np.uint16), want_s.view(np.uint16))
    assert np.array_equal(codes, orc.pack_codes(want_c, bits))


def _tie_residuals(seed, rows, width, g, bits):
    """Rows whose quotients r/s sit exactly on, and one fp32 ulp either side
    of, half-integers: each group's first element is qmax * s0 for an fp16
    value s0 (so s = s0 exactly), the others (k + 1/2) * s0 nudged by -1, 0 or
    +1 ulp, or a random multiple of s0."""
    rng = np.random.default_rng(seed)
    qm = (1 << (bits - 1)) - 1
    s0 = (2.0 ** rng.integers(-14, 6, size=(rows, width // g, 1))
          * rng.integers(1024, 2048, size=(rows, width // g, 1)) / 1024.0).astype(np.float16).astype(np.float32)
    k = rng.integers(-qm, qm, size=(rows, width // g, g)).astype(np.float32)
    r = ((k + np.float32(0.5)) * s0).astype(np.float32)
    nudge = rng.integers(-1, 2, size=r.shape)
    r = np.where(nudge > 0, np.nextafter(r, np.float32(np.inf)),
                 np.where(nudge < 0, np.nextafter(r, np.float32(-np.inf)), r)).astype(np.float32)
    rand = rng.random(r.shape) < 0.3
    r[rand] = (rng.uniform(-qm, qm, size=r.shape).astype(np.float32) * s0 * np.ones_like(r))[rand]
    r[:, :, 0] = (qm * s0[:, :, 0]).astype(np.float32)
    r[rng.random(rows) < 0.02] = 0.0
    return r.reshape(rows, width).astype(np.float32)


@pytest.mark.parametrize("width,g,bits", [(128, 64, 4), (128, 32, 2), (64, 32, 4), (256, 128, 4)])
def test_quantize_ties_bit_exact(env, width, g, bits):
    """Quotients on and next to half-integers: rint ties to even of the correctly
    rounded quotient, as the oracle takes it."""
    torch, fl, orc = env
    r = _tie_residuals(3 + width + g + bits, 3000, width, g, bits)
    codes, scales = fl.quantize(torch.from_numpy(r).cuda(), g, bits)
    want_c, want_s = orc.quantize_groups(r, bits, g)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), want_s.view(np.uint16))
    assert np.array_equal(codes.cpu().numpy(), orc.pack_codes(want_c, bits))


@pytest.mark.parametrize("width,g,bits", [(128, 64, 4), (128, 32, 2), (64, 32, 4), (256, 128, 2)])
def test_quantize_residual_bit_exact(env, width, g, bits):
    # r = x - prev in IEEE fp32 (exact rounding on both sides), then the quantiser
    torch, fl, orc = env
    rows = 1500
    rng = np.random.default_rng(11 + width + g + bits)
    x = rng.standard_normal((rows, width)).astype(np.float32)
    prev = (x + 0.05 * rng.standard_normal((rows, width))).astype(np.float32)
    prev_bits = orc.bf16_round(prev.astype(np.float64)).astype(np.float32).view(np.uint32) >> 16
    prev_b = prev_bits.astype(np.uint16)
    r = x - prev_b.astype(np.uint32).__lshift__(16).view(np.float32)
    codes, scales = fl.quantize_residual(torch.from_numpy(x).cuda(), torch.from_numpy(prev_b.view(np.int16)).cuda(),
                                         g, bits)
    want_c, want_s = orc.quantize_groups(r, bits, g)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), want_s.view(np.uint16))
    assert np.array_equal(codes.cpu().numpy(), orc.pack_codes(want_c, bits))


def _bf16(torch, rng, shape, scale=1.0):
    x = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32))
    return x.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("m,n,k,swap", [(256, 384, 512, False), (200, 300, 688, False), (128, 128, 64, False),
                                        (1000, 2048, 2048, False), (1, 3072, 2048, True), (8, 2048, 2048, True),
                                        (16, 2048, 5632, True), (33, 700, 256, True), (64, 11008, 4096, True),
                                        (5, 32000, 2048, True), (8, 3072, 2048, False)])
def test_gemm_matches_fp64_product(env, m, n, k, swap):
    torch, fl, orc = env
    if not swap and m <= 64:
        pytest.skip("normal orientation is for m > 64")
    rng = np.random.default_rng(m * 7 + n + k)
    A = _bf16(torch, rng, (m, k))
    B = _bf16(torch, rng, (n, k), 0.05)
    D = fl.gemm(A, B, swap_ab=swap)
    ref = (A.double() @ B.double().T)
    bound = (A.double().abs() @ B.double().abs().T) * (k * 2.0 ** -23) + 1e-6
    err = (D.double() - ref).abs()
    assert torch.all(err <= bound), float((err / bound).max())
