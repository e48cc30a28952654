"""mla_decode_attention_noalloc against mla_decode_attention.

The no-allocation entry point serves callers that cannot allocate device
memory when they call the library (inside a CUDA graph capture, under a
serving engine that owns all GPU memory, as a plugin under a foreign
allocator). It keeps the split-KV partial results in a fixed array inside the
library. This test runs the regular entry point (with a caller workspace) and
then the no-allocation one twice in a row, on a plan that splits sequences,
and requires the same outputs within the decode tolerance both times; it also
checks that a plan too large for the built-in array is refused.

The file name makes pytest collect it last.
"""

import math

import numpy as np
import pytest
import torch

import synth
from mla_latent_kv_32_b200 import build as build_mod
from mla_latent_kv_32_b200 import mla
from mla_latent_kv_32_b200.runtime import DecodeSession
from tests._util import assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    mla.load()
    return torch.device("cuda:0")


def test_noalloc_matches_workspace_entry_point(dev):
    lens = [3000, 2000, 77, 64, 5]
    w = synth.Workload("noalloc", B=len(lens), q_len=2, L=3000, n_h=128, seed=21)
    inp = synth.make_decode_inputs(w, lens=lens)
    sess = DecodeSession(inp, dev, num_ctas=74)
    assert sess.info.num_partials > 0, "the plan must split sequences to exercise the scratch"
    sess.append()
    sess.absorb()
    sess.attend()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    want_o = sess.o.float().cpu().numpy()
    want_lse = sess.lse.cpu().numpy()
    for call in range(2):
        o = torch.full_like(sess.o, float("nan"))
        lse = torch.full_like(sess.lse, float("nan"))
        mla.mla_decode_attention_noalloc(sess.q_full, sess.cache, sess.num_pages, sess.table,
                                         sess.max_pages, sess.B, sess.q_len, sess.n_h,
                                         sess.scale, sess.plan_host, sess.plan_dev, o, lse,
                                         sess.status)
        torch.cuda.synchronize()
        assert sess.read_status() == 0
        assert_parity(o.float().cpu().numpy(), want_o, f"o_latent, call {call + 1}")
        assert np.max(np.abs(lse.cpu().numpy() - want_lse)) <= 1e-3, f"lse, call {call + 1}"


def test_noalloc_rejects_plan_beyond_scratch(dev):
    lens = np.full(64, 131072, dtype=np.int32)
    plan, info = mla.mla_decode_plan(lens, 64, 2, 128, num_ctas=512)
    assert info.workspace_bytes > (48 << 20)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_attention_noalloc(16, 16, 1, 16, 4096, 64, 2, 128, 1.0 / math.sqrt(192),
                                         plan, 16, 16, None, None)
    assert e.value.status == mla.MLA_ERR_WORKSPACE_TOO_SMALL
