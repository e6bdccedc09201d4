"""The variants around the looped core on the GPU, against the oracle.

Independent prelude and coda layers with their own one-pass KV, a learned loop
embedding added to each loop's input, and input injection of the state that
entered the loop stack ("从'堆层数'到'循环复用'：FlashLoop 到底在解决什么问题",
§3.1, §3.2 and §4.1; "Looped Transformer 教程", 第三步), on the lazy path (the
oracle's integer decisions handed over) and on the dense one.  Weights are
synthetic (no trained checkpoint exists here).
"""
import pytest

import e2e_common as E
from cross_loop_sparsity_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from cross_loop_sparsity_b200 import build
    build.build()


VARIANTS = {
    "prelude_coda": dict(n_prelude=2, n_coda=1),
    "loop_embedding": dict(loop_embed=1),
    "injection": dict(inject_scale=0.5),
    "all": dict(n_prelude=1, n_coda=2, loop_embed=1, inject_scale=0.3),
}


@pytest.mark.parametrize("name", list(VARIANTS))
def test_variants_lazy_prefill_then_decode_forced(name):
    cfg = synth.config("c1").with_(seed=101, n_loops=3, c_cols=24, **VARIANTS[name])
    E.check_all(E.run_calls(cfg, 2, [0, 0], [90], decode_after=2))


def test_variants_lazy_decode_over_context_forced():
    """Decode over a synthetic context whose prelude / coda layers hold their own KV."""
    cfg = synth.config("c2").with_(ctx_len=600, seed=103, **VARIANTS["all"])
    E.check_all(E.run_calls(cfg, 4, [600, 350, 77, 512], [], decode_after=1))


@pytest.mark.parametrize("name", ["prelude_coda", "all"])
def test_variants_dense_forced(name):
    cfg = synth.config("c1").with_(seed=107, n_loops=3, **VARIANTS[name])
    E.check_all(E.run_calls(cfg, 2, [40, 0], [60], dense=True, decode_after=1))
