"""Chunked prefill onto an existing cache, and the last_loop KV mode, on the GPU.

A prefill chunk continues sequences that already hold tokens -- a synthetic
context with residual levels, an earlier chunk of the same prompt, or decoded
tokens -- at positions len_b + t, with query tiles counted from the chunk's
first token ("Looped Transformer 教程", 第四步, and the lazy-update step of
"FlashLoop: Fast and Memory-Efficient Looped Transformers via Lazy Updates",
abstract).  The last_loop KV mode keeps one KV per layer that every loop
overwrites (第四步: recurrent_kv_cache_mode = "last_loop").  Hidden states and
logits must be within 2e-2 x RMS of the oracle's, with the oracle's integer
decisions handed over as in the other end-to-end tests.
"""
import pytest

import e2e_common as E
from cross_loop_sparsity_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from cross_loop_sparsity_b200 import build
    build.build()


def test_prefill_chunk_onto_a_residual_context_forced():
    """Ragged synthetic contexts that hold residual levels 2..K, then one chunk
    per sequence (tiles, columns and chains reach into the context)."""
    cfg = synth.config("c1").with_(seed=91, c_cols=24)
    E.check_all(E.run_calls(cfg, 2, [150, 40], [100]))


def test_prefill_chunk_long_block_onto_context_forced():
    cfg = synth.config("c3").with_(n_layers=2, n_loops=3, seed=93)
    E.check_all(E.run_calls(cfg, 1, [700], [300]))


def test_prompt_in_chunks_then_decode_forced():
    """A fresh prompt prefilled as two chunks, then two decode steps."""
    cfg = synth.config("c1").with_(seed=95, c_cols=20, n_loops=3)
    E.check_all(E.run_calls(cfg, 2, [0, 0], [70, 90], decode_after=2))


def test_dense_prompt_in_chunks_onto_context():
    cfg = synth.config("c1").with_(seed=97, n_loops=3)
    E.check_all(E.run_calls(cfg, 2, [60, 130], [50, 40], dense=True, decode_after=1))


@pytest.mark.parametrize("ctx_lens", [[0, 0], [90, 33]])
def test_last_loop_kv_mode_prefill_and_decode(ctx_lens):
    cfg = synth.config("c1").with_(seed=99, n_loops=3, kv_mode=1)
    E.check_all(E.run_calls(cfg, 2, ctx_lens, [64, 30], dense=True, decode_after=2))

