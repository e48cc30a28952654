"""Device-side failure detection of the decode kernel, without faulting the GPU.

Every barrier wait of the tensor-core decode kernel is bounded. The test hook
mla_debug_decode_wait shortens the bound and makes the producer of every CTA
pair skip its first arrival on the first stage barrier, so the MMA issuer's
wait can only end by running out: the kernel must report MLA_DEV_TIMEOUT in
the status word, stop, drain and exit, and the context must stay usable (the
next call, with the hook off, gives the oracle's result).
"""

import math
import time

import numpy as np
import pytest
import torch

import synth
from mla_latent_kv_32_b200 import build as build_mod
from mla_latent_kv_32_b200 import mla
from mla_latent_kv_32_b200.runtime import DecodeSession
from oracle import mla_oracle as O
from tests._util import assert_parity

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(192)


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    mla.load()
    return torch.device("cuda:0")


def test_bounded_wait_reports_timeout_and_recovers(dev):
    lens = [700, 64, 129]
    w = synth.Workload("timeout", B=len(lens), q_len=1, L=max(lens), n_h=128, seed=9)
    inp = synth.make_decode_inputs(w, lens=lens)
    table = O.rope_table(max(lens))
    sess = DecodeSession(inp, dev, rope_table=table)
    sess.append()
    sess.absorb()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    try:
        mla.mla_debug_decode_wait(0.02, 1)
        t0 = time.perf_counter()
        sess.attend()
        torch.cuda.synchronize()
        took = time.perf_counter() - t0
    finally:
        mla.mla_debug_decode_wait(1.0, 0)
    bits = sess.read_status()
    assert bits & mla.MLA_DEV_TIMEOUT, f"status 0x{bits:x}"
    assert took < 5.0   # a few 20 ms waits, not the default 1 s ones
    # the context still works and the next call is right
    sess.attend()
    sess.expand()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    u = sess.u.float().cpu().numpy().reshape(w.B, 1, 128, 128)
    got, ref = [], []
    for b in range(w.B):
        L = int(inp.lens[b])
        prefix = O.gather_rows(inp.pool, inp.table, b, L - 1)
        r = O.decode_sequence(prefix, inp.c_new[b], inp.k_new[b], inp.q_nope[b], inp.q_pe[b],
                              inp.w_uk, inp.w_uv, L, table, SCALE)
        got.append(u[b]); ref.append(r["u"])
    assert_parity(np.stack(got), np.stack(ref), "u after the timeout")
