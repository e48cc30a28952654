"""GPU parity of the decode path (through the C ABI) against the CPU oracle.

Every case runs the library's kernels on seeded synthetic inputs and compares
with the fp64 oracle on the same bf16 inputs:
  * cache contents bit-exact (the appended rows and every other slot);
  * decode outputs u (and the latent o, lse) within max|d| <= 2e-2 max|ref|,
    sum|d|/sum|ref| <= 5e-3 against the absorbed oracle, and against the
    non-absorbed (expanded K/V) oracle on a subset of heads.
Small cases cover every sequence; full-size workloads run in the launch
configuration of the benchmark and are checked on sampled sequences.
"""

import math

import numpy as np
import pytest
import torch

import synth
from mla_latent_kv_32_b200 import build as build_mod
from mla_latent_kv_32_b200 import mla
from mla_latent_kv_32_b200.runtime import DecodeSession, bf16_to_numpy_bits
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


def oracle_seq(inp, b, table, form="absorbed", heads=None):
    w = inp.w
    L = int(inp.lens[b])
    n_pref = L - w.q_len
    prefix = (O.gather_rows(inp.pool, inp.table, b, n_pref) if n_pref > 0
              else np.zeros((0, 576), np.uint16))
    return O.decode_sequence(prefix, inp.c_new[b], inp.k_new[b], inp.q_nope[b], inp.q_pe[b],
                             inp.w_uk, inp.w_uv, L, table, SCALE, form=form, heads=heads)


def check_session(sess, inp, seqs, table, nonabs=2, check_pool=False):
    """Compare sess outputs for sequences `seqs` with the oracle."""
    w = inp.w
    q_len, n_h = w.q_len, w.n_h
    u = sess.u.float().cpu().numpy().reshape(w.B, q_len, n_h, 128)
    o = sess.o.float().cpu().numpy().reshape(w.B, q_len, n_h, 512)
    lse = sess.lse.cpu().numpy().reshape(w.B, q_len, n_h)
    pool = bf16_to_numpy_bits(sess.cache)
    got_u, ref_u, got_o, ref_o, got_l, ref_l = [], [], [], [], [], []
    for k, b in enumerate(seqs):
        r = oracle_seq(inp, b, table)
        got_u.append(u[b]); ref_u.append(r["u"])
        got_o.append(o[b]); ref_o.append(r["o"])
        got_l.append(lse[b]); ref_l.append(r["lse"])
        # appended rows are bit-exact
        L = int(inp.lens[b])
        for j in range(q_len):
            p = L - q_len + j
            row = pool[inp.table[b, p // 64], p % 64]
            assert np.array_equal(row, r["new_rows"][j]), f"cache row of seq {b} pos {p}"
        if k < nonabs:
            heads = [0, n_h - 1]
            rn = oracle_seq(inp, b, table, form="nonabsorbed", heads=heads)
            assert_parity(u[b][:, heads], rn["u"], f"u vs non-absorbed oracle, seq {b}")
    assert_parity(np.stack(got_u), np.stack(ref_u), "u")
    assert_parity(np.stack(got_o), np.stack(ref_o), "o_latent")
    gl, rl = np.stack(got_l), np.stack(ref_l)
    assert np.max(np.abs(gl - rl)) <= 2e-2, "lse"
    if check_pool:
        want = inp.pool.copy()
        pos = inp.positions
        for b in range(w.B):
            for j in range(q_len):
                p = int(pos[b, j])
                want[inp.table[b, p // 64], p % 64] = O.make_cache_row(
                    inp.c_new[b, j], inp.k_new[b, j], [p], table)[0]
        assert np.array_equal(pool, want), "pool differs outside the appended rows"


SMALL = [
    ("edges", [1, 63, 64, 65, 127, 200], 1, 128),
    ("mtp", [2, 64, 65, 129, 1000], 2, 128),
    ("tiny_heads", [256], 1, 16),
    ("heads32", [5000, 3, 700], 1, 32),
    ("one", [1], 1, 128),
    ("mtp_min", [2, 3], 2, 64),
    # head counts that leave part of a CTA's 64 query rows (or all of the
    # second CTA's) empty
    ("heads48", [300, 64, 1], 1, 48),
    ("heads80_mtp", [130, 2, 513], 2, 80),
    ("heads96", [65, 4100], 1, 96),
    ("heads112_mtp", [257, 66], 2, 112),
    # multi-token-prediction verify depths beyond two (causal between them)
    ("mtp3", [3, 64, 66, 700], 3, 128),
    ("mtp4_heads32", [4, 130, 5000], 4, 32),
    ("mtp8", [8, 71, 640, 1000], 8, 128),
    ("mtp16", [16, 64, 300], 16, 64),
    # chunked prefill: every token of the chunk is a causal query
    ("prefill64", [64, 200, 65], 64, 128),
    ("prefill128_heads32", [128, 1000, 700], 128, 32),
]


@pytest.mark.parametrize("name,lens,q_len,n_h", SMALL, ids=[s[0] for s in SMALL])
def test_decode_small(dev, name, lens, q_len, n_h):
    w = synth.Workload(name, B=len(lens), q_len=q_len, L=max(lens), n_h=n_h, seed=7)
    inp = synth.make_decode_inputs(w, lens=lens)
    table = O.rope_table(max(lens))
    sess = DecodeSession(inp, dev, rope_table=table)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    check_session(sess, inp, list(range(w.B)), table, nonabs=w.B, check_pool=True)


def test_append_bit_exact_with_library_rope_table(dev):
    # The product path's own RoPE table (mla_rope_table, not the oracle's):
    # with that same table handed to the oracle, every appended row and every
    # other slot of the pool is bit-exact.
    lens = [1, 63, 64, 65, 4000, 300]
    w = synth.Workload("libtab", B=len(lens), q_len=2, L=max(lens), n_h=128, seed=17)
    inp = synth.make_decode_inputs(w, lens=[max(l, 2) for l in lens])
    sess = DecodeSession(inp, dev)                       # rope_table=None: the library's
    lib_table = mla.mla_rope_table(sess.max_pos)
    assert np.array_equal(sess.rope.cpu().numpy(), lib_table)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    check_session(sess, inp, list(range(w.B)), lib_table, nonabs=1, check_pool=True)


@pytest.mark.parametrize("num_ctas,max_split", [(1, 0), (5, 0), (74, 0), (148, 0), (74, 1)])
def test_split_invariance(dev, num_ctas, max_split):
    lens = [3000, 2000, 77, 64, 1]
    w = synth.Workload("split", B=len(lens), q_len=2 if max(lens) > 1 else 1, L=3000, n_h=128,
                       seed=11)
    lens = [max(l, w.q_len) for l in lens]
    inp = synth.make_decode_inputs(w, lens=lens)
    table = O.rope_table(max(lens))
    sess = DecodeSession(inp, dev, num_ctas=num_ctas, max_split=max_split, rope_table=table)
    # NaN in every workspace byte: a split unit may only read partial results
    # that this call wrote
    sess.workspace.fill_(0xFF)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    check_session(sess, inp, list(range(w.B)), table, nonabs=1)


def test_e2e_graphs_match_oracle(dev):
    # the benchmark's end-to-end loop: two sessions, each one CUDA graph of
    # upload + library calls + download, alternate steps on two streams;
    # every step's result read back to the host must be the oracle's
    from mla_latent_kv_32_b200.runtime import capture_io_step, run_e2e_graphs
    lens = [700, 64, 1, 129]
    w = synth.Workload("e2e", B=len(lens), q_len=1, L=max(lens), n_h=128, seed=5)
    inp = synth.make_decode_inputs(w, lens=lens)
    table = O.rope_table(max(lens))
    pair = [DecodeSession(inp, dev, rope_table=table) for _ in range(2)]
    ins, host_in, host_out0 = pair[0].pinned_step_buffers()   # the true inputs
    for s in pair:   # clobber the device inputs: the graphs must upload them
        for t in s.io_inputs():
            t.zero_()
    host_outs = [torch.full_like(host_out0, 7.0).pin_memory() for _ in range(2)]
    graphs = [capture_io_step(s, host_in, host_outs[i]) for i, s in enumerate(pair)]
    for s in pair:
        for t in s.io_inputs():
            t.zero_()
    for h in host_outs:
        h.fill_(7.0)
    run_e2e_graphs(graphs, [torch.cuda.Stream(), torch.cuda.Stream()], 5)
    torch.cuda.synchronize()
    for s in pair:
        assert s.read_status() == 0
    ref = np.stack([oracle_seq(inp, b, table)["u"] for b in range(w.B)])
    for h in host_outs:
        u = h.float().numpy().reshape(w.B, 1, 128, 128)
        assert_parity(u, ref, "u (e2e)")


def test_bad_page_sets_status(dev):
    lens = [300, 200]
    w = synth.Workload("bad", B=2, q_len=1, L=300, n_h=128, seed=3)
    inp = synth.make_decode_inputs(w, lens=lens)
    table = O.rope_table(300)
    sess = DecodeSession(inp, dev, rope_table=table)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    good_u1 = sess.u.float().cpu().numpy().reshape(2, 128, 128)[1].copy()
    # corrupt sequence 0's second page id, rerun attention only
    bad = sess.table.clone()
    bad[0, 1] = 10 ** 6
    sess.table.copy_(bad)
    sess.attend()
    sess.expand()
    torch.cuda.synchronize()
    bits = sess.read_status()
    assert bits & mla.MLA_DEV_BAD_PAGE
    u1 = sess.u.float().cpu().numpy().reshape(2, 128, 128)[1]
    assert np.array_equal(u1, good_u1), "an unaffected sequence changed"
    assert np.all(np.isfinite(sess.u.float().cpu().numpy()))


def test_prefill_full_size_sampled_queries(dev):
    # The chunked-prefill workload (4 sequences, 512-token chunks ending a
    # 4096-token context) in the bench's launch configuration; the oracle
    # evaluates a sample of each sequence's chunk queries (the first and last
    # among them), and every appended row is checked bit for bit.
    w = synth.WORKLOADS["prefill"]
    inp = synth.make_decode_inputs(w)
    table = O.rope_table(int(inp.lens.max()))
    sess = DecodeSession(inp, dev, rope_table=table)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    u = sess.u.float().cpu().numpy().reshape(w.B, w.q_len, w.n_h, 128)
    o = sess.o.float().cpu().numpy().reshape(w.B, w.q_len, w.n_h, 512)
    pool = bf16_to_numpy_bits(sess.cache)
    rng = np.random.default_rng(5)
    got_u, ref_u, got_o, ref_o = [], [], [], []
    for b in range(w.B):
        qs = sorted({0, 1, 63, 64, w.q_len - 1, *rng.choice(w.q_len, 6, replace=False).tolist()})
        L = int(inp.lens[b])
        prefix = O.gather_rows(inp.pool, inp.table, b, L - w.q_len)
        r = O.decode_sequence(prefix, inp.c_new[b], inp.k_new[b], inp.q_nope[b], inp.q_pe[b],
                              inp.w_uk, inp.w_uv, L, table, SCALE, queries=qs)
        got_u.append(u[b][qs]); ref_u.append(r["u"])
        got_o.append(o[b][qs]); ref_o.append(r["o"])
        for j in range(w.q_len):
            p = L - w.q_len + j
            assert np.array_equal(pool[inp.table[b, p // 64], p % 64], r["new_rows"][j])
    assert_parity(np.concatenate(got_u), np.concatenate(ref_u), "u (prefill)")
    assert_parity(np.concatenate(got_o), np.concatenate(ref_o), "o_latent (prefill)")


@pytest.mark.parametrize("name", ["v3", "ragged", "long_mtp", "mtp8"])
def test_workload_full_size(dev, name):
    w = synth.WORKLOADS[name]
    inp = synth.make_decode_inputs(w)
    table = O.rope_table(int(inp.lens.max()))
    sess = DecodeSession(inp, dev, rope_table=table)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    seqs = synth.sample_sequences(w, inp.lens, 8)
    check_session(sess, inp, seqs, table, nonabs=2)
    # every appended row of every sequence is bit-exact
    pool = bf16_to_numpy_bits(sess.cache)
    pos = inp.positions
    for b in range(w.B):
        for j in range(w.q_len):
            p = int(pos[b, j])
            want = O.make_cache_row(inp.c_new[b, j], inp.k_new[b, j], [p], table)[0]
            assert np.array_equal(pool[inp.table[b, p // 64], p % 64], want)


@pytest.mark.parametrize("lens,q_len,n_h,ctas", [
    ([700, 64, 1, 129, 2000], 1, 128, 74), ([300, 4100], 2, 128, 16), ([90, 33], 1, 48, 3)])
def test_tensor_core_vs_cuda_core(dev, lens, q_len, n_h, ctas):
    """Two independent GPU kernels on the same inputs and plan agree."""
    w = synth.Workload("diff", B=len(lens), q_len=q_len, L=max(lens), n_h=n_h, seed=13)
    inp = synth.make_decode_inputs(w, lens=[max(l, q_len) for l in lens])
    sess = DecodeSession(inp, dev, num_ctas=ctas)
    sess.append()
    sess.absorb()
    sess.attend()
    torch.cuda.synchronize()
    o_tc = sess.o.float().cpu().numpy()
    lse_tc = sess.lse.cpu().numpy()
    o_cc = torch.empty_like(sess.o)
    lse_cc = torch.empty_like(sess.lse)
    mla.mla_decode_attention_cudacore(sess.q_full, sess.cache, sess.num_pages, sess.table,
                                      sess.max_pages, sess.B, sess.q_len, sess.n_h, sess.scale,
                                      sess.plan_host, sess.plan_dev, sess.workspace, sess.ws_bytes,
                                      o_cc, lse_cc, sess.status)
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    assert_parity(o_tc, o_cc.float().cpu().numpy(), "o: tensor-core vs CUDA-core kernel")
    assert np.max(np.abs(lse_tc - lse_cc.cpu().numpy())) <= 1e-2
