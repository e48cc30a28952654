"""GPU parity of the whole decode layer (projections, RoPE, append, absorbed
attention, W_UV, W_O) against the fp64 oracle's layer, through the C ABI."""

import math

import numpy as np
import pytest
import torch

import synth
from mla_latent_kv_32_b200 import build as build_mod
from mla_latent_kv_32_b200 import mla
from mla_latent_kv_32_b200.runtime import LayerSession, bf16_to_numpy_bits
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


@pytest.mark.parametrize("name", ["tiny", "layer_v3"])
def test_layer(dev, name):
    w = synth.WORKLOADS[name]
    inp = synth.make_layer_inputs(w)
    sess = LayerSession(inp, dev)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    seqs = [0] if w.B == 1 else synth.sample_sequences(w, inp.lens, 6)
    ref = O.layer_decode(inp.h, inp.weights, w.n_h, w.q_len, inp.tok_seq, inp.tok_pos,
                         inp.query_tok, lambda b, n: synth.prefix_rows(w, b, n), inp.lens,
                         SCALE, seqs)
    rows = np.concatenate([np.arange(b * w.q_len, (b + 1) * w.q_len) for b in seqs])
    out = sess.out.cpu().numpy()[rows]
    u = sess.u.float().cpu().numpy()[rows].reshape(-1, w.n_h, 128)
    assert_parity(u, ref["u"], "u")
    assert_parity(out, ref["out"], "layer output")
    # the rows the layer appended, against the oracle's float64 chain (tolerance:
    # the GPU rounds the projection to bf16 before the RoPE, the oracle after)
    pool = bf16_to_numpy_bits(sess.cache)
    got = np.stack([pool[inp.table[inp.tok_seq[t], inp.tok_pos[t] // 64], inp.tok_pos[t] % 64]
                    for t in ref["new_tok"]])
    assert_parity(O.bf16_to_f64(got), O.bf16_to_f64(ref["new_rows"]), "appended rows")
    # ... and bit for bit: the GPU's own bf16 projections [c^KV | k^R_pre]
    # (a GEMM's bf16 output cannot be pinned to float64) through the oracle's
    # cache row (latent copied, float32 RoPE with the same table) must give
    # exactly the stored rows, for every token the layer appended
    kv = bf16_to_numpy_bits(sess.kv)
    table = mla.mla_rope_table(sess.max_pos)
    all_tok = np.arange(sess.T)
    want = O.make_cache_row(kv[:, :512], kv[:, 512:], inp.tok_pos[all_tok], table)
    got_all = np.stack([pool[inp.table[inp.tok_seq[t], inp.tok_pos[t] // 64],
                             inp.tok_pos[t] % 64] for t in all_tok])
    assert np.array_equal(got_all, want), "appended cache rows are not bit-exact"


@pytest.mark.parametrize("M,N,K,fp32", [
    (256, 576, 7168, 0), (256, 1536, 7168, 0), (7, 64, 512, 0), (256, 24576, 1536, 0),
    (256, 7168, 16384, 1), (100, 1100, 640, 1), (3, 2048, 1024, 0), (64, 24576, 512, 0),
    (48, 20000, 512, 0)])
def test_split_k_gemm_matches_fp32(dev, M, N, K, fp32):
    # C = X W^T with a workspace (split over K into partial sums when the tile
    # grid is below one wave; 256-row weight tiles from 1024 rows up, also
    # with narrow token tiles, 64 x 24576 and 48 x 20000 here, the latter
    # with a ragged last tile) and without one (fp32 outputs may split with
    # atomic adds), against a float64 product of the same bf16 inputs
    g = torch.Generator().manual_seed(M * 7 + N)
    X = (torch.randn(M, K, generator=g) / math.sqrt(K)).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    ref = (X.double() @ W.double().T).numpy()
    Xd, Wd = X.to(dev), W.to(dev)
    dt = torch.float32 if fp32 else torch.bfloat16
    C = torch.full((M, N), float("nan"), dtype=dt, device=dev)
    need = mla.mla_gemm_bf16_workspace_bytes(M, N, K)
    ws = torch.full((max(need, 256),), 0xFF, dtype=torch.uint8, device=dev)   # NaN-poisoned
    mla.mla_gemm_bf16_ws(Xd, K, Wd, K, C, N, fp32, M, N, K, ws, ws.numel())
    got = C.float().cpu().numpy()
    C2 = torch.full_like(C, float("nan"))
    mla.mla_gemm_bf16(Xd, K, Wd, K, C2, N, fp32, M, N, K)
    got2 = C2.float().cpu().numpy()
    for g_ in (got, got2):
        assert np.all(np.isfinite(g_))
        err = np.abs(g_ - ref)
        assert err.max() <= 2e-2 * np.abs(ref).max() and err.sum() <= 5e-3 * np.abs(ref).sum()


@pytest.mark.parametrize("name", ["tiny", "layer_v3"])
def test_layer_folded(dev, name):
    # The layer with folded weights (W~QK = W^UK^T W^UQ per head, W~O = W^O W^UV
    # per head, computed once by the library): the folds match the oracle's
    # float64 folds to bf16 rounding, and the layer output matches the
    # oracle's unfolded layer (the definition) within the decode tolerance.
    w = synth.WORKLOADS[name]
    inp = synth.make_layer_inputs(w)
    sess = LayerSession(inp, dev, folded=True)
    sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0
    W = inp.weights
    up = W["w_uq"] if w.q_lora else W["w_q"]
    wqk = bf16_to_numpy_bits(sess.w_qk_f)
    wof = bf16_to_numpy_bits(sess.w_o_f)
    for h in synth.sample_heads(w.n_h, 4):
        ref_qk = O.fold_qk(up[h * 128:(h + 1) * 128], W["w_uk"][h:h + 1], 1)
        ref_o = O.fold_o(W["w_o"][:, h * 128:(h + 1) * 128], W["w_uv"][h:h + 1], 1)
        assert_parity(O.bf16_to_f64(wqk[h * 512:(h + 1) * 512]), ref_qk, f"W~QK head {h}",
                      tol_max=4e-3, tol_mean=3e-3)
        assert_parity(O.bf16_to_f64(wof[:, h * 512:(h + 1) * 512]), ref_o, f"W~O head {h}",
                      tol_max=4e-3, tol_mean=3e-3)
    seqs = [0] if w.B == 1 else synth.sample_sequences(w, inp.lens, 6)
    ref = O.layer_decode(inp.h, inp.weights, w.n_h, w.q_len, inp.tok_seq, inp.tok_pos,
                         inp.query_tok, lambda b, n: synth.prefix_rows(w, b, n), inp.lens,
                         SCALE, seqs)
    rows = np.concatenate([np.arange(b * w.q_len, (b + 1) * w.q_len) for b in seqs])
    assert_parity(sess.out.cpu().numpy()[rows], ref["out"], "folded layer output")
    o = sess.o.float().cpu().numpy()[rows]
    assert_parity(o, ref["o"], "latent attention output (folded query)")
