"""mla_decode_attention_noalloc against mla_decode_attention.

The no-allocation entry point serves callers that cannot hand the library
device memory of their own when they call it: a serving engine that reserved
nearly all of the GPU's memory for its own cache pool up front, or a plugin
running under another framework's allocator that must not grow the device
footprint behind that allocator's back. It keeps the split-KV partial results
in a fixed array inside the library instead of a caller workspace.

The test runs the regular entry point (with a caller workspace) and then the
no-allocation one twice, with a call on a different split plan (other lengths
and work-list count, so the shared array holds other partial results) in
between, and requires bit-identical outputs every time: both entry points run
the same kernels on the same plan, so any difference would be scratch
corruption. It also checks that a plan too large for the built-in array is
refused before anything is launched.

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

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    mla.load()
    return torch.device("cuda:0")


def _session(dev, lens, q_len, seed, num_ctas):
    w = synth.Workload("noalloc", B=len(lens), q_len=q_len, L=max(lens), n_h=128, seed=seed)
    inp = synth.make_decode_inputs(w, lens=lens)
    sess = DecodeSession(inp, dev, num_ctas=num_ctas)
    assert sess.info.num_partials > 0, "the plan must split sequences to exercise the scratch"
    sess.append()
    sess.absorb()
    torch.cuda.synchronize()
    return sess


def _noalloc(sess):
    o = torch.full_like(sess.o, float("nan"))
    lse = torch.full_like(sess.lse, float("nan"))
    mla.mla_decode_attention_noalloc(sess.q_full, sess.cache, sess.num_pages, sess.table,
                                     sess.max_pages, sess.B, sess.q_len, sess.n_h, sess.scale,
                                     sess.plan_host, sess.plan_dev, o, lse, sess.status)
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    return o, lse


def test_noalloc_matches_workspace_entry_point(dev):
    sess = _session(dev, [3000, 2000, 77, 64, 5], 2, 21, 74)
    other = _session(dev, [9000, 130, 4100], 1, 22, 37)
    sess.attend()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    want_o = sess.o.clone()
    want_lse = sess.lse.clone()
    for call in range(2):
        if call == 1:
            _noalloc(other)   # another plan's partial results now fill the array
        o, lse = _noalloc(sess)
        assert torch.equal(o.view(torch.int16), want_o.view(torch.int16)), \
            f"o_latent differs from the workspace entry point, call {call + 1}"
        assert torch.equal(lse, want_lse), f"lse differs, call {call + 1}"


def test_noalloc_rejects_plan_beyond_scratch(dev):
    lens = np.full(64, 131072, dtype=np.int32)
    plan, info = mla.mla_decode_plan(lens, 64, 2, 128, num_ctas=512)
    assert info.workspace_bytes > (48 << 20)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_attention_noalloc(16, 16, 1, 16, 4096, 64, 2, 128, 1.0 / math.sqrt(192),
                                         plan, 16, 16, None, None)
    assert e.value.status == mla.MLA_ERR_WORKSPACE_TOO_SMALL
