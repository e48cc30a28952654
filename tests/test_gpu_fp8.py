"""GPU parity of the FP8 (E4M3) latent cache through the C ABI.

The cache contract is bit-exact: every slot of the FP8 pool (codes, the bf16
k^R bytes) and every per-token scale equals the oracle's quantization of the
same bf16 inputs (the prefix rows enter through the library's FP8 append, as
a prefill would write them; the step's new rows are appended by the step).
The attention outputs are compared with the oracle's attention over the
exactly dequantized rows within the decode tolerance.
"""

import math

import numpy as np
import pytest
import torch

import synth
from mla_latent_kv_32_b200 import build as build_mod
from mla_latent_kv_32_b200 import mla
from mla_latent_kv_32_b200.runtime import DecodeSession, FP8_FILL_CODE
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


def oracle_fp8_seq(inp, b, table, queries=None):
    """The oracle's FP8 rows of sequence b (prefix quantized from the bf16
    prefix rows at positions 0..) and its decode step."""
    w = inp.w
    L = int(inp.lens[b])
    n = L - w.q_len
    pref = (O.gather_rows(inp.pool, inp.table, b, n) if n > 0
            else np.zeros((0, 576), np.uint16))
    pb, ps = O.make_cache_row_fp8(pref[:, :512], pref[:, 512:], np.arange(n), table)
    r = O.decode_sequence_fp8(pb, ps, inp.c_new[b], inp.k_new[b], inp.q_nope[b], inp.q_pe[b],
                              inp.w_uk, inp.w_uv, L, table, SCALE, queries=queries)
    r["rows"] = np.concatenate([pb, r["new_rows"]], axis=0)
    r["scales"] = np.concatenate([ps, r["new_scales"]])
    return r


def check_fp8(sess, inp, seqs, table, whole_pool):
    w = inp.w
    q_len, n_h = w.q_len, w.n_h
    pool = sess.cache8.cpu().numpy()
    scales = sess.scales8.cpu().numpy()
    u = sess.u.float().cpu().numpy().reshape(w.B, q_len, n_h, 128)
    o = sess.o.float().cpu().numpy().reshape(w.B, q_len, n_h, 512)
    if whole_pool:
        want = np.zeros_like(pool)
        want[:, :, :512] = FP8_FILL_CODE
        want[:, :, 512:] = np.frombuffer(np.uint16(0x4280).tobytes() * 64, np.uint8)
        want_s = np.ones_like(scales)
    got_u, ref_u, got_o, ref_o = [], [], [], []
    for b in seqs:
        r = oracle_fp8_seq(inp, b, table)
        L = int(inp.lens[b])
        pages = inp.table[b, :(L + 63) // 64]
        gp = pool[pages].reshape(-1, 640)[:L]
        gs = scales[pages].reshape(-1)[:L]
        assert np.array_equal(gp, r["rows"]), f"FP8 rows of sequence {b}"
        assert np.array_equal(gs.astype(np.float64), r["scales"]), f"scales of sequence {b}"
        if whole_pool:
            for i, pg in enumerate(pages):
                k = min(64, L - 64 * i)
                want[pg, :k] = r["rows"][64 * i:64 * i + k]
                want_s[pg, :k] = r["scales"][64 * i:64 * i + k]
        got_u.append(u[b]); ref_u.append(r["u"])
        got_o.append(o[b]); ref_o.append(r["o"])
    if whole_pool:
        assert np.array_equal(pool, want), "FP8 pool differs outside the written rows"
        assert np.array_equal(scales, want_s), "scales differ outside the written rows"
    assert_parity(np.stack(got_u), np.stack(ref_u), "u (FP8 cache)")
    assert_parity(np.stack(got_o), np.stack(ref_o), "o_latent (FP8 cache)")


SMALL = [
    ("edges", [1, 63, 64, 65, 127, 200, 1000], 1, 128),
    ("mtp", [2, 64, 129, 3000], 2, 128),
    ("heads32", [700, 3, 4100], 1, 32),
    ("heads48_mtp4", [130, 4, 513], 4, 48),
]


@pytest.mark.parametrize("name,lens,q_len,n_h", SMALL, ids=[c[0] for c in SMALL])
def test_fp8_small(dev, name, lens, q_len, n_h):
    w = synth.Workload(name, B=len(lens), q_len=q_len, L=max(lens), n_h=n_h, seed=23)
    inp = synth.make_decode_inputs(w, lens=lens)
    table = O.rope_table(max(lens))
    sess = DecodeSession(inp, dev, rope_table=table, fp8=True)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    check_fp8(sess, inp, list(range(w.B)), table, whole_pool=True)


@pytest.mark.parametrize("num_ctas,max_split", [(1, 0), (74, 0), (5, 1)])
def test_fp8_split_invariance(dev, num_ctas, max_split):
    lens = [3000, 2000, 77, 64, 2]
    w = synth.Workload("fp8split", B=len(lens), q_len=2, L=3000, n_h=128, seed=29)
    inp = synth.make_decode_inputs(w, lens=lens)
    table = O.rope_table(max(lens))
    sess = DecodeSession(inp, dev, num_ctas=num_ctas, max_split=max_split, rope_table=table,
                         fp8=True)
    sess.workspace.fill_(0xFF)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    check_fp8(sess, inp, list(range(w.B)), table, whole_pool=False)


@pytest.mark.parametrize("name", ["v3", "ragged"])
def test_fp8_workload_full_size(dev, name):
    w = synth.WORKLOADS[name]
    inp = synth.make_decode_inputs(w)
    table = O.rope_table(int(inp.lens.max()))
    sess = DecodeSession(inp, dev, rope_table=table, fp8=True)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    check_fp8(sess, inp, synth.sample_sequences(w, inp.lens, 6), table, whole_pool=False)


@pytest.mark.parametrize("where", ["query", "latent"])
def test_fp8_range_reported(dev, where):
    # The FP8 decode computes in fp16: a query value beyond its range, or a
    # token whose scale exceeds 2^7 (a latent value beyond 448 * 2^7), sets
    # MLA_DEV_RANGE; in-range inputs leave the status clear (every other test)
    lens = [300, 129]
    w = synth.Workload("fp8range", B=len(lens), q_len=1, L=300, n_h=128, seed=31)
    inp = synth.make_decode_inputs(w, lens=lens)
    sess = DecodeSession(inp, dev, fp8=True)
    if where == "latent":
        sess.c_new[1, 7] = 1.0e5
    sess.append()
    sess.absorb()
    if where == "query":
        sess.q_full[0, 5, 11] = 1.0e5
    sess.attend()
    torch.cuda.synchronize()
    assert sess.read_status() & mla.MLA_DEV_RANGE
