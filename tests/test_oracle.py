"""Pins of the CPU fp64 oracle to things other than itself.

Each test checks the oracle against a brute-force loop written from the
definition, a closed form printed on the pages, a textbook invariant, or a
library routine (torch's bf16 cast, torch's scaled_dot_product_attention).
The comment on each test names the plausible oracle mistake it would catch.
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------- helpers ---

def brute_attention(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos):
    """Pure-Python loops over the non-absorbed definition: k^C_i = W^UK c_i,
    v_i = W^UV c_i, score = q^C.k^C + q^R.k^R, softmax over i <= q_pos."""
    J, H = len(q_nope), len(q_nope[0])
    L = len(rows)
    d_nope, d_c = len(w_uk[0]), len(w_uk[0][0])
    d_v = len(w_uv[0])
    d_r = len(q_rope[0][0])
    u = [[[0.0] * d_v for _ in range(H)] for _ in range(J)]
    for j in range(J):
        for h in range(H):
            scores = []
            for i in range(L):
                if i > q_pos[j]:
                    scores.append(None)
                    continue
                sc = 0.0
                for d in range(d_nope):
                    k_c = 0.0
                    for c in range(d_c):
                        k_c += w_uk[h][d][c] * rows[i][c]
                    sc += q_nope[j][h][d] * k_c
                for r in range(d_r):
                    sc += q_rope[j][h][r] * rows[i][d_c + r]
                scores.append(sc * scale)
            mx = max(s for s in scores if s is not None)
            ex = [0.0 if s is None else math.exp(s - mx) for s in scores]
            tot = sum(ex)
            for dv in range(d_v):
                acc = 0.0
                for i in range(L):
                    if scores[i] is None:
                        continue
                    v = 0.0
                    for c in range(d_c):
                        v += w_uv[h][dv][c] * rows[i][c]
                    acc += (ex[i] / tot) * v
                u[j][h][dv] = acc
    return np.array(u)


def rand_case(rng, J, H, L, d_c, d_r, d_nope, d_v):
    q_nope = rng.standard_normal((J, H, d_nope))
    q_rope = rng.standard_normal((J, H, d_r))
    rows = rng.standard_normal((L, d_c + d_r))
    w_uk = rng.standard_normal((H, d_nope, d_c)) / math.sqrt(d_c)
    w_uv = rng.standard_normal((H, d_v, d_c)) / math.sqrt(d_c)
    q_pos = np.arange(L - J, L)
    return q_nope, q_rope, rows, w_uk, w_uv, q_pos


# ----------------------------------------------------------- bf16 storage ---

def test_round_to_bf16_matches_torch_cast():
    # catches: truncation instead of round-to-nearest-even, wrong mantissa width
    rng = np.random.default_rng(5)
    x = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    # exact ties: bf16 value + half an ulp, representable in float32
    base = rng.standard_normal(2000).astype(np.float32)
    bits = base.view(np.uint32) & np.uint32(0xFFFF0000)
    ties = (bits | np.uint32(0x8000)).view(np.float32)
    tiny = np.array([1e-39, -3e-40, 2.0 ** -130, 1e-45], dtype=np.float32)
    big = np.array([3.0e38, -3.3e38, 65504.0, 1.0e30], dtype=np.float32)
    allx = np.concatenate([x, ties, tiny, big, np.float32([0.0, -0.0, 1.0])])
    want = torch.from_numpy(allx).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.round_to_bf16(allx.astype(np.float64))
    assert np.array_equal(got, want)
    assert np.array_equal(synth.f32_to_bf16_bits(allx), want)
    back = O.bf16_to_f64(want)
    assert np.array_equal(back, torch.from_numpy(want.view(np.int16)).view(torch.bfloat16)
                          .to(torch.float64).numpy())


# ------------------------------------------------------------------- RoPE ---

@pytest.mark.parametrize("pos", [0, 1, 7, 255, 8191, 131071])
def test_rope_unit_vectors_closed_form(pos):
    # catches: rotate-half pairing, wrong sign of the sine term, wrong frequency law
    d = 64
    e0 = np.zeros(d); e0[0] = 1
    e1 = np.zeros(d); e1[1] = 1
    e16 = np.zeros(d); e16[16] = 1       # pair j = 8: frequency 10000^(-16/64) = 1/10
    e32 = np.zeros(d); e32[32] = 1       # pair j = 16: frequency 10000^(-32/64) = 1/100
    y0 = O.rope_f64(e0, pos)
    y1 = O.rope_f64(e1, pos)
    y16 = O.rope_f64(e16, pos)
    y32 = O.rope_f64(e32, pos)
    want0 = np.zeros(d); want0[0], want0[1] = math.cos(pos), math.sin(pos)
    want1 = np.zeros(d); want1[0], want1[1] = -math.sin(pos), math.cos(pos)
    want16 = np.zeros(d); want16[16], want16[17] = math.cos(pos / 10), math.sin(pos / 10)
    want32 = np.zeros(d); want32[32], want32[33] = math.cos(pos / 100), math.sin(pos / 100)
    for got, want in ((y0, want0), (y1, want1), (y16, want16), (y32, want32)):
        assert np.allclose(got, want, atol=1e-12, rtol=0)


def test_rope_invariants():
    # catches: non-orthogonal rotation, position offsets, pair mix-ups across heads
    rng = np.random.default_rng(1)
    q = rng.standard_normal((5, 64))
    k = rng.standard_normal((5, 64))
    assert np.array_equal(O.rope_f64(q, 0), q)
    for m, n in [(3, 1), (1000, 17), (131071, 5), (64, 64)]:
        qm = O.rope_f64(q, m)
        assert np.allclose(np.linalg.norm(qm, axis=1), np.linalg.norm(q, axis=1), rtol=1e-13)
        lhs = np.sum(O.rope_f64(q, m) * O.rope_f64(k, n), axis=1)
        rhs = np.sum(O.rope_f64(q, m - n) * k, axis=1)
        assert np.allclose(lhs, rhs, rtol=1e-9, atol=1e-9)


def test_rope_table_closed_form():
    # catches: table built with the wrong base or exponent, cos/sin swapped
    t = O.rope_table(9000)
    assert t.dtype == np.float32 and t.shape == (9000, 32, 2)
    for p in [0, 1, 2, 100, 8191, 8999]:
        assert t[p, 0, 0] == np.float32(math.cos(p)) and t[p, 0, 1] == np.float32(math.sin(p))
        assert t[p, 8, 0] == np.float32(math.cos(p / 10.0))
        assert t[p, 16, 1] == np.float32(math.sin(p / 100.0))


def test_rope_fp32_cache_code_vs_exact():
    # catches: a cached k^R code that drifts from the exact rotation by more than
    # one bf16 rounding (wrong table entry, wrong pair, missing term)
    rng = np.random.default_rng(2)
    n = 4000
    x = synth.f32_to_bf16_bits(rng.standard_normal((n, 64)).astype(np.float32))
    pos = rng.integers(0, 131072, size=n)
    t = O.rope_table(131072)
    cs = t[pos]
    got = O.bf16_to_f64(O.rope_f32_to_bf16(x, cs[..., 0], cs[..., 1]))
    exact = O.rope_f64(O.bf16_to_f64(x), pos)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    assert np.all(np.abs(got - exact) <= ulp * 1.01)
    same = got == O.bf16_to_f64(O.round_to_bf16(exact))
    assert same.mean() > 0.99
    # position 0 is the identity on the stored bits
    cs0 = t[np.zeros(n, dtype=int)]
    assert np.array_equal(O.rope_f32_to_bf16(x, cs0[..., 0], cs0[..., 1]), x)


# ------------------------------------------------------------------ cache ---

def test_cache_append_placement_brute_force():
    # catches: wrong page/slot arithmetic, writes into other sequences' pages,
    # missing skip of out-of-range tokens
    rng = np.random.default_rng(3)
    n_pages, B = 11, 3
    pool0 = rng.integers(0, 2 ** 16, size=(n_pages, 64, 576), dtype=np.uint16)
    table = np.full((B, 4), -1, np.int32)
    perm = rng.permutation(n_pages).astype(np.int32)
    table[0, :4] = perm[:4]; table[1, :3] = perm[4:7]; table[2, :2] = perm[7:9]
    seq = np.array([0, 0, 1, 2, 2, 1, 0, 2, 5], np.int32)
    pos = np.array([0, 255, 130, 64, 127, 191, 63, 128, 0], np.int32)
    n = len(seq)
    c_kv = rng.integers(0, 2 ** 15, size=(n, 512), dtype=np.uint16)
    k_pe = synth.f32_to_bf16_bits(rng.standard_normal((n, 64)).astype(np.float32))
    tab = O.rope_table(300)
    pool, skipped = O.cache_append(pool0, table, seq, pos, c_kv, k_pe, tab)
    expect_skip = [False, False, False, False, False, False, False, True, True]
    assert skipped.tolist() == expect_skip
    written = {}
    for t in range(n):
        if expect_skip[t]:
            continue
        page = table[seq[t]][pos[t] // 64]
        written[(int(page), int(pos[t] % 64))] = t
    for page in range(n_pages):
        for slot in range(64):
            if (page, slot) in written:
                t = written[(page, slot)]
                assert np.array_equal(pool[page, slot, :512], c_kv[t])
                cs = tab[pos[t]]
                assert np.array_equal(pool[page, slot, 512:],
                                      O.rope_f32_to_bf16(k_pe[t], cs[:, 0], cs[:, 1]))
            else:
                assert np.array_equal(pool[page, slot], pool0[page, slot])


# -------------------------------------------------------------- attention ---

@pytest.mark.parametrize("L,J", [(1, 1), (2, 1), (5, 1), (2, 2), (5, 2)])
def test_attention_brute_force_tiny(L, J):
    # catches: transposed W_UK/W_UV, dropped RoPE term, wrong scale, mask off by one
    rng = np.random.default_rng(10 * L + J)
    args = rand_case(rng, J, H=2, L=L, d_c=8, d_r=4, d_nope=4, d_v=4)
    q_nope, q_rope, rows, w_uk, w_uv, q_pos = args
    scale = 1.0 / math.sqrt(4 + 4)
    want = brute_attention(q_nope.tolist(), q_rope.tolist(), rows.tolist(),
                           w_uk.tolist(), w_uv.tolist(), scale, q_pos.tolist())
    u1, _ = O.attend_nonabsorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos)
    u2, _, _ = O.attend_absorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos)
    assert np.allclose(u1, want, rtol=1e-12, atol=1e-13)
    assert np.allclose(u2, want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("J,H,L", [(1, 16, 256), (2, 4, 300), (1, 3, 1)])
def test_absorption_identity(J, H, L):
    # catches: any algebra slip between the two forms at the real widths
    rng = np.random.default_rng(J * 1000 + H * 10 + L)
    q_nope, q_rope, rows, w_uk, w_uv, q_pos = rand_case(rng, J, H, L, 512, 64, 128, 128)
    scale = O.default_scale()
    u1, att = O.attend_nonabsorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos)
    u2, o, lse = O.attend_absorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos)
    assert np.max(np.abs(u1 - u2)) <= 1e-11 * np.max(np.abs(u1))
    # softmax rows sum to one and masked keys carry zero weight
    assert np.allclose(att.sum(-1), 1.0, atol=1e-12)
    for j in range(J):
        assert np.all(att[j, :, q_pos[j] + 1:] == 0.0)


def test_default_scale_is_inverse_sqrt_192():
    # catches: scaling by 1/sqrt(d_h) or 1/sqrt(d_c) instead of 1/sqrt(d_h + d_R)
    assert O.default_scale() == 1.0 / math.sqrt(192)


def test_special_cases_closed_form():
    # catches: normalisation errors, wrong value expansion, wrong averaging
    rng = np.random.default_rng(4)
    H = 4
    q_nope, q_rope, rows, w_uk, w_uv, _ = rand_case(rng, 1, H, 7, 512, 64, 128, 128)
    scale = O.default_scale()
    # one cached token: u_h = W_UV[h] c_0 whatever the query
    u, o, lse = O.attend_absorbed(q_nope, q_rope, rows[:1], w_uk, w_uv, scale, np.array([0]))
    for h in range(H):
        assert np.allclose(u[0, h], w_uv[h] @ rows[0, :512], rtol=1e-13)
    # every latent equal: o = c, whatever the scores
    rows_eq = rows.copy(); rows_eq[:, :512] = rows[0, :512]
    u, o, lse = O.attend_absorbed(q_nope, q_rope, rows_eq, w_uk, w_uv, scale, np.array([6]))
    assert np.allclose(o[0], np.broadcast_to(rows[0, :512], (H, 512)), rtol=1e-13)
    # zero query: uniform weights, o = mean of the visible latents, lse = log L
    for J in (1, 2):
        zq1 = np.zeros((J, H, 128)); zq2 = np.zeros((J, H, 64))
        qp = np.arange(7 - J, 7)
        u, o, lse = O.attend_absorbed(zq1, zq2, rows, w_uk, w_uv, scale, qp)
        for j in range(J):
            n = qp[j] + 1
            assert np.allclose(o[j], rows[:n, :512].mean(0), rtol=1e-13)
            assert np.allclose(lse[j], math.log(n), rtol=1e-13)


@pytest.mark.parametrize("J", [1, 2])
def test_reduction_to_sdpa(J):
    # With no RoPE channel and W_UK = W_UV, MLA is single-KV attention per head:
    # compare with torch's scaled_dot_product_attention (float64, explicit mask).
    # catches: mask direction, softmax axis, scale placement
    rng = np.random.default_rng(20 + J)
    H, L, d_c, d = 3, 40, 32, 16
    q_nope = rng.standard_normal((J, H, d))
    q_rope = np.zeros((J, H, 0))
    rows = rng.standard_normal((L, d_c))
    w = rng.standard_normal((H, d, d_c)) / math.sqrt(d_c)
    scale = 0.37
    q_pos = np.arange(L - J, L)
    u, _, _ = O.attend_absorbed(q_nope, q_rope, rows, w, w, scale, q_pos)
    kv = torch.einsum("lc,hdc->hld", torch.from_numpy(rows), torch.from_numpy(w))
    q = torch.from_numpy(q_nope).permute(1, 0, 2)                  # [H, J, d]
    mask = torch.arange(L)[None, :] <= torch.from_numpy(q_pos)[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None], kv[None], kv[None], attn_mask=mask, scale=scale)[0]
    assert np.allclose(u, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_mtp_query0_equals_shorter_context():
    # the first of two causal queries must not see the second token:
    # its output equals a single-query decode over the first L-1 rows
    rng = np.random.default_rng(6)
    q_nope, q_rope, rows, w_uk, w_uv, q_pos = rand_case(rng, 2, 4, 70, 512, 64, 128, 128)
    scale = O.default_scale()
    u2, o2, l2 = O.attend_absorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos)
    u1, o1, l1 = O.attend_absorbed(q_nope[:1], q_rope[:1], rows[:69], w_uk, w_uv, scale,
                                   np.array([68]))
    assert np.allclose(u2[0], u1[0], rtol=1e-12)


# ------------------------------------------------------------ closed forms ---

def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(None, 1)
            val = rest.split("|")[0].strip()
            vals[key] = val
    return vals


def close_to_printed(x, printed):
    digits = len(printed.split(".")[1]) if "." in printed else 0
    return abs(x - float(printed)) <= 10.0 ** (-digits) + 1e-12


def _partial(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos, a, b):
    """Attention of every query over keys [a, b) only, through the oracle's
    unsplit attention on that slice; a query that sees none of them gets
    o = 0, lse = -inf."""
    J, H = q_nope.shape[:2]
    o = np.zeros((J, H, rows.shape[1] - q_rope.shape[-1]))
    lse = np.full((J, H), -np.inf)
    for j in range(J):
        qp = int(q_pos[j]) - a
        if qp < 0:
            continue
        _, oj, lj = O.attend_absorbed(q_nope[j:j + 1], q_rope[j:j + 1], rows[a:b], w_uk, w_uv,
                                      scale, [qp])
        o[j], lse[j] = oj[0], lj[0]
    return o, lse


@pytest.mark.parametrize("cuts", [[0, 64, 200], [0, 1, 63, 64, 129, 199, 200], [0, 137, 199, 200]])
def test_merge_partials_equals_unsplit_attention(cuts):
    # The split-KV merge (log-sum-exp identity) against the unsplit softmax on
    # the same keys, including a last range that query 0 cannot see.
    # Catches: a wrong sign in the weights exp(lse_s - lse), a missing
    # renormalisation, lse taken as a max instead of a log-sum-exp, an empty
    # range given weight.
    rng = np.random.default_rng(11)
    q_nope, q_rope, rows, w_uk, w_uv, q_pos = rand_case(rng, 2, 3, 200, 512, 64, 128, 128)
    scale = O.default_scale()
    _, o_ref, lse_ref = O.attend_absorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos)
    parts = [_partial(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos, a, b)
             for a, b in zip(cuts[:-1], cuts[1:])]
    if cuts[-2] == 199:
        assert np.isneginf(parts[-1][1][0]).all()      # query 0 sees no key of [199, 200)
    o, lse = O.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * np.max(np.abs(o_ref))
    assert np.max(np.abs(lse - lse_ref)) <= 1e-12 * np.max(np.abs(lse_ref))
    # the order of the parts does not matter
    rev = O.merge_partials([p[0] for p in parts[::-1]], [p[1] for p in parts[::-1]])
    assert np.max(np.abs(rev[0] - o)) <= 1e-13 * np.max(np.abs(o))


def test_merge_partials_edge_cases():
    rng = np.random.default_rng(12)
    o1 = rng.standard_normal((3, 4, 8))
    l1 = rng.standard_normal((3, 4))
    # one part: the identity, exactly
    o, lse = O.merge_partials([o1], [l1])
    assert np.array_equal(o, o1) and np.array_equal(lse, l1)
    # an empty part (lse = -inf, any o) changes nothing
    o, lse = O.merge_partials([o1, np.full_like(o1, 7.0)], [l1, np.full_like(l1, -np.inf)])
    assert np.allclose(o, o1, rtol=0, atol=1e-15) and np.allclose(lse, l1, rtol=0, atol=1e-15)
    # two equal halves of the same keys: same o, lse + log 2
    o, lse = O.merge_partials([o1, o1], [l1, l1])
    assert np.allclose(o, o1, rtol=1e-15, atol=1e-15)
    assert np.allclose(lse, l1 + math.log(2.0), rtol=0, atol=1e-14)
    # no visible key anywhere: o = 0, lse = -inf
    o, lse = O.merge_partials([o1, o1], [np.full_like(l1, -np.inf)] * 2)
    assert not o.any() and np.isneginf(lse).all()


def test_cache_footprint_closed_forms():
    g = read_golden("cache_footprint.txt")
    n_h, d_h = 128, 128
    mla = O.kv_cache_bytes(1) // 2
    mha = 2 * n_h * d_h
    gqa8 = 2 * 8 * d_h
    assert mla == int(g["mla_elements_per_token_layer"])
    assert mha == int(g["mha_elements_per_token_layer"])
    assert gqa8 == int(g["gqa8_elements_per_token_layer"])
    assert close_to_printed(100 * (1 - mla / mha), g["reduction_vs_mha_percent"])
    assert close_to_printed(100 * (1 - mla / gqa8), g["reduction_vs_gqa8_percent"])
    assert close_to_printed(O.kv_cache_bytes(1) / 1000, g["mla_kb_per_token_fp16"])
    assert close_to_printed(O.kv_cache_bytes(128 * 1024) / 1e9, g["mla_gb_128k_fp16"])
    assert close_to_printed(mha * 2 / 1000, g["mha_kb_per_token_fp16"])
    assert close_to_printed(100 * mla / mha, g["mla_relative_footprint_percent"])
    assert close_to_printed(mla / d_h, g["cache_over_dh_ratio"])
    pool = O.kv_cache_bytes(4 * 131072)
    assert pool == 603979776
    assert close_to_printed(pool / 1e6, g["long_mtp_pool_mb"] + ".0") or round(pool / 1e6) == 604


# ------------------------------------------------------------------ layer ---

def brute_layer(h, W, n_h, tok_pos, prefix_rows_f, q_tok, scale, base=10000.0):
    """Pure-Python layer for one sequence: projections, exact RoPE, bf16 cache
    rows, attention (brute_attention), output projection."""
    def mat(Wm, x):
        return [sum(Wm[o][i] * x[i] for i in range(len(x))) for o in range(len(Wm))]

    def rope(x, p):
        d = len(x)
        y = list(x)
        for j in range(d // 2):
            th = p / base ** (2 * j / d)
            y[2 * j] = x[2 * j] * math.cos(th) - x[2 * j + 1] * math.sin(th)
            y[2 * j + 1] = x[2 * j + 1] * math.cos(th) + x[2 * j] * math.sin(th)
        return y

    T = len(h)
    rows = [list(r) for r in prefix_rows_f]
    for t in range(T):
        ckv = mat(W["w_dkv"], h[t])
        kr = rope(mat(W["w_kr"], h[t]), tok_pos[t])
        stored = O.bf16_to_f64(O.round_to_bf16(np.array(ckv + kr))).tolist()
        rows.append(stored)
    x = h[q_tok]
    if "w_dq" in W:
        cq = mat(W["w_dq"], x)
        qc, qr = mat(W["w_uq"], cq), mat(W["w_qr"], cq)
    else:
        qc, qr = mat(W["w_q"], x), mat(W["w_qr"], x)
    d_nope = len(W["w_uk"][0])
    d_r = len(qr) // n_h
    q_nope = [[qc[hh * d_nope:(hh + 1) * d_nope] for hh in range(n_h)]]
    q_rope = [[rope(qr[hh * d_r:(hh + 1) * d_r], tok_pos[q_tok]) for hh in range(n_h)]]
    u = brute_attention(q_nope, q_rope, rows, W["w_uk"], W["w_uv"], scale,
                        [tok_pos[q_tok]])
    flat = u[0].reshape(-1).tolist()
    return np.array(mat(W["w_o"], flat))


@pytest.mark.parametrize("q_lora", [0, 5])
def test_layer_brute_force_tiny(q_lora):
    # catches: wrong head split of the projections, RoPE on the wrong slice,
    # missing bf16 storage of the new rows, wrong W_O orientation
    rng = np.random.default_rng(30 + q_lora)
    hid, n_h, d_nope, d_r, d_c, d_v = 6, 2, 3, 4, 4, 3
    T, n_pref = 3, 2
    L = n_pref + T

    def bf(shape, std=1.0):
        return synth.f32_to_bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))

    W = {}
    if q_lora:
        W["w_dq"] = bf((q_lora, hid)); W["w_uq"] = bf((n_h * d_nope, q_lora))
        W["w_qr"] = bf((n_h * d_r, q_lora))
    else:
        W["w_q"] = bf((n_h * d_nope, hid)); W["w_qr"] = bf((n_h * d_r, hid))
    W["w_dkv"] = bf((d_c, hid)); W["w_kr"] = bf((d_r, hid))
    W["w_uk"] = bf((n_h, d_nope, d_c)); W["w_uv"] = bf((n_h, d_v, d_c))
    W["w_o"] = bf((hid, n_h * d_v))
    h = bf((T, hid))
    prefix = bf((n_pref, d_c + d_r))
    tok_seq = np.zeros(T, np.int32)
    tok_pos = np.arange(n_pref, L, dtype=np.int32)
    scale = 0.41
    res = O.layer_decode(h, W, n_h, 1, tok_seq, tok_pos, np.array([T - 1]),
                         lambda b, n: prefix[:n], np.array([L]), scale)
    Wf = {k: O.bf16_to_f64(v).tolist() for k, v in W.items()}
    want = brute_layer(O.bf16_to_f64(h).tolist(), Wf, n_h, tok_pos.tolist(),
                       O.bf16_to_f64(prefix).tolist(), T - 1, scale)
    assert np.allclose(res["out"][0], want, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------------ synth ---

def test_synth_pool_layout():
    w = synth.Workload("t", B=5, q_len=2, L=300, n_h=4, lens="ragged")
    lens = synth.seq_lens(w)
    assert lens.min() >= 2 and lens.max() <= 300
    table = synth.block_table(w, lens)
    npg = synth.pages_needed(lens)
    ids = np.concatenate([table[b, :npg[b]] for b in range(w.B)])
    assert sorted(ids.tolist()) == list(range(int(npg.sum())))
    pool = synth.build_pool(w, lens, table)
    for b in range(w.B):
        rows = O.gather_rows(pool, table, b, int(lens[b]))
        want = synth.prefix_rows(w, b, int(lens[b]) - 2)
        assert np.array_equal(rows[: lens[b] - 2], want)
        assert np.all(rows[lens[b] - 2:] == synth.FILL_BITS)
    # same seed, same bits
    assert np.array_equal(pool, synth.build_pool(w, lens, table))


# ------------------------------------------------- decode_sequence (a step) ---

def _torch_rope_code(k_bits, cos32, sin32):
    """Cached k^R code through torch's float32 element-wise ops (each product
    and each sum its own IEEE float32 operation) and torch's bf16 cast."""
    x = torch.from_numpy(np.asarray(k_bits, np.uint16).view(np.int16)).view(torch.bfloat16)
    x = x.to(torch.float32)
    c = torch.from_numpy(np.asarray(cos32, np.float32))
    s = torch.from_numpy(np.asarray(sin32, np.float32))
    x0, x1 = x[..., 0::2], x[..., 1::2]
    a0, b0 = torch.mul(x0, c), torch.mul(x1, s)
    a1, b1 = torch.mul(x1, c), torch.mul(x0, s)
    y = torch.empty_like(x)
    y[..., 0::2] = torch.sub(a0, b0)
    y[..., 1::2] = torch.add(a1, b1)
    return y.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_rope_f32_code_bit_exact_vs_torch_float32():
    # The cached k^R code is a fixed function of the bf16 input and the fp32
    # table: pinned bit for bit to torch's float32 ops. Catches a fused
    # multiply-add, a rotation evaluated in float64, a pair or sign mix-up.
    rng = np.random.default_rng(41)
    n = 20000
    x = synth.f32_to_bf16_bits((rng.standard_normal((n, 64)) * 3).astype(np.float32))
    pos = rng.integers(0, 131072, size=n)
    t = O.rope_table(131072)
    cs = t[pos]
    got = O.rope_f32_to_bf16(x, cs[..., 0], cs[..., 1])
    want = _torch_rope_code(x, cs[..., 0], cs[..., 1])
    assert np.array_equal(got, want)
    # the pin separates the float32 contract from an exact (float64) rotation
    # rounded once: some codes differ between the two
    exact = O.round_to_bf16(O.rope_f64(O.bf16_to_f64(x), pos))
    assert (exact != want).any()


def _brute_rope(x, p, base=10000.0):
    d = len(x)
    y = list(x)
    for j in range(d // 2):
        th = p / base ** (2 * j / d)
        y[2 * j] = x[2 * j] * math.cos(th) - x[2 * j + 1] * math.sin(th)
        y[2 * j + 1] = x[2 * j + 1] * math.cos(th) + x[2 * j] * math.sin(th)
    return y


def _decode_sequence_case(seed=51, n_pref=3, q_len=2, H=1):
    """Inputs of a small decode step at the real widths (576-wide rows)."""
    rng = np.random.default_rng(seed)

    def bf(shape, std=1.0):
        return synth.f32_to_bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))

    L = n_pref + q_len
    prefix = bf((n_pref, 576))
    # the new tokens' latents are large so that the keys appended this step
    # carry most of the softmax weight
    c_new = bf((q_len, 512), 3.0)
    k_new = bf((q_len, 64), 3.0)
    q_nope = bf((q_len, H, 128))
    q_pe = bf((q_len, H, 64), 3.0)
    w_uk = bf((H, 128, 512), 1.0 / math.sqrt(512))
    w_uv = bf((H, 128, 512), 1.0 / math.sqrt(512))
    return dict(prefix=prefix, c_new=c_new, k_new=k_new, q_nope=q_nope, q_pe=q_pe, w_uk=w_uk,
                w_uv=w_uv, L=L)


def _decode_sequence_brute(cs):
    """Independent restatement of one decode step: the new rows built with
    torch float32 ops at positions L-q_len.., appended after the prefix, the
    query's RoPE rotated exactly at its own position, then the pure-Python
    non-absorbed attention."""
    L, q_len = cs["L"], cs["c_new"].shape[0]
    tab = O.rope_table(L)
    pos = np.arange(L - q_len, L)
    new_k = _torch_rope_code(cs["k_new"], tab[pos][..., 0], tab[pos][..., 1])
    rows_bits = np.concatenate([cs["prefix"], np.concatenate([cs["c_new"], new_k], 1)], 0)
    rows = O.bf16_to_f64(rows_bits)
    qn = O.bf16_to_f64(cs["q_nope"])
    qp = O.bf16_to_f64(cs["q_pe"])
    H = qn.shape[1]
    q_rope = [[_brute_rope(qp[j, h].tolist(), int(pos[j])) for h in range(H)]
              for j in range(q_len)]
    u = brute_attention(qn.tolist(), q_rope, rows.tolist(), O.bf16_to_f64(cs["w_uk"]).tolist(),
                        O.bf16_to_f64(cs["w_uv"]).tolist(), O.default_scale(), pos.tolist())
    return u, rows_bits


def _decode_sequence_error(mod, cs, want_u, want_rows):
    tab = O.rope_table(cs["L"] + 8)
    r = mod.decode_sequence(cs["prefix"], cs["c_new"], cs["k_new"], cs["q_nope"], cs["q_pe"],
                            cs["w_uk"], cs["w_uv"], cs["L"], tab, O.default_scale())
    err = np.max(np.abs(r["u"] - want_u)) / np.max(np.abs(want_u))
    return err, np.array_equal(r["rows"], want_rows)


@pytest.fixture(scope="module")
def decode_case():
    cs = _decode_sequence_case()
    want_u, want_rows = _decode_sequence_brute(cs)
    return cs, want_u, want_rows


def test_decode_sequence_brute_force(decode_case):
    # One attention-only decode step with two causal queries: append first,
    # then score ("DeepSeek-V3 MLA ... Guide", Step 3), q^R rotated at the
    # query's own position L-2 / L-1.
    cs, want_u, want_rows = decode_case
    err, rows_ok = _decode_sequence_error(O, cs, want_u, want_rows)
    assert rows_ok
    assert err <= 1e-12
    # the non-absorbed form of the same step agrees too
    tab = O.rope_table(cs["L"])
    r = O.decode_sequence(cs["prefix"], cs["c_new"], cs["k_new"], cs["q_nope"], cs["q_pe"],
                          cs["w_uk"], cs["w_uv"], cs["L"], tab, O.default_scale(),
                          form="nonabsorbed")
    assert np.max(np.abs(r["u"] - want_u)) <= 1e-12 * np.max(np.abs(want_u))


def _plant_score_before_append(monkeypatch):
    real = O.attend_absorbed

    def scored_on_prefix(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos):
        n = len(q_pos)
        return real(q_nope, q_rope, rows[:-n], w_uk, w_uv, scale,
                    np.minimum(np.asarray(q_pos), len(rows) - n - 1))
    monkeypatch.setattr(O, "attend_absorbed", scored_on_prefix)


def _plant_query_rope_at_last_position(monkeypatch):
    real = O.rope_f64

    def rope_last(x, pos, base=O.ROPE_BASE):
        p = np.asarray(pos)
        return real(x, np.full_like(p, p.max()), base)
    monkeypatch.setattr(O, "rope_f64", rope_last)


def _plant_append_one_position_late(monkeypatch):
    real = O.make_cache_row

    def late(c, k, pos, table):
        return real(c, k, np.asarray(pos) + 1, table)
    monkeypatch.setattr(O, "make_cache_row", late)


@pytest.mark.parametrize("plant", [_plant_score_before_append,
                                   _plant_query_rope_at_last_position,
                                   _plant_append_one_position_late])
def test_decode_sequence_pin_catches_planted_mistakes(decode_case, monkeypatch, plant):
    # Each plausible slip in the step's composition, planted in the oracle,
    # moves u far outside the 1e-12 pin (or changes the appended rows).
    cs, want_u, want_rows = decode_case
    plant(monkeypatch)
    err, rows_ok = _decode_sequence_error(O, cs, want_u, want_rows)
    assert err > 1e-4 or not rows_ok


# ---------------------------------------------------------------- folding ---

def test_fold_brute_force_tiny():
    # the two folds are plain per-head products: explicit triple loops.
    # Catches: a transposed W^UK or W^UV, heads mixed up, the wrong slice of
    # W^O or W^UQ.
    rng = np.random.default_rng(61)
    n_h, d_h, d_c, q_in, d_model = 3, 2, 5, 4, 6

    def bf(shape):
        return synth.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))

    w_up, w_uk = bf((n_h * d_h, q_in)), bf((n_h, d_h, d_c))
    w_o, w_uv = bf((d_model, n_h * d_h)), bf((n_h, d_h, d_c))
    U, K = O.bf16_to_f64(w_up), O.bf16_to_f64(w_uk)
    Wo, V = O.bf16_to_f64(w_o), O.bf16_to_f64(w_uv)
    fq = O.fold_qk(w_up, w_uk, n_h)
    fo = O.fold_o(w_o, w_uv, n_h)
    for h in range(n_h):
        for c in range(d_c):
            for i in range(q_in):
                want = sum(U[h * d_h + d, i] * K[h, d, c] for d in range(d_h))
                assert abs(fq[h * d_c + c, i] - want) <= 1e-13
            for f in range(d_model):
                want = sum(Wo[f, h * d_h + d] * V[h, d, c] for d in range(d_h))
                assert abs(fo[f, h * d_c + c] - want) <= 1e-13


@pytest.mark.parametrize("q_lora", [0, 5])
def test_folded_layer_equals_unfolded(q_lora):
    # Associativity: the layer through W~QK and W~O equals the layer through
    # q^C, W^UK, W^UV and W^O (the absorption identity carried into the
    # projections). Catches a fold applied to the wrong input (h instead of
    # c^Q) or the wrong side of the output projection.
    rng = np.random.default_rng(70 + q_lora)
    hid, n_h, d_c = 64, 2, 512
    T, n_pref = 3, 4
    L = n_pref + T

    def bf(shape, std=1.0):
        return synth.f32_to_bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))

    W = {}
    if q_lora:
        W["w_dq"] = bf((64, hid), 1 / 8); W["w_uq"] = bf((n_h * 128, 64), 1 / 8)
        W["w_qr"] = bf((n_h * 64, 64), 1 / 8)
    else:
        W["w_q"] = bf((n_h * 128, hid), 1 / 8); W["w_qr"] = bf((n_h * 64, hid), 1 / 8)
    W["w_dkv"] = bf((d_c, hid), 1 / 8); W["w_kr"] = bf((64, hid), 1 / 8)
    W["w_uk"] = bf((n_h, 128, d_c), 1 / 22.6); W["w_uv"] = bf((n_h, 128, d_c), 1 / 22.6)
    W["w_o"] = bf((hid, n_h * 128), 1 / 16)
    h = bf((T, hid))
    prefix = bf((n_pref, 576))
    args = (h, W, n_h, 1, np.zeros(T, np.int32), np.arange(n_pref, L, dtype=np.int32),
            np.array([T - 1]), lambda b, n: prefix[:n], np.array([L]), O.default_scale())
    ref = O.layer_decode(*args)
    fold = {"w_qk": O.fold_qk(W["w_uq"] if q_lora else W["w_q"], W["w_uk"], n_h),
            "w_o": O.fold_o(W["w_o"], W["w_uv"], n_h)}
    got = O.layer_decode(*args, fold=fold)
    assert np.max(np.abs(got["out"] - ref["out"])) <= 1e-11 * np.max(np.abs(ref["out"]))
    assert np.max(np.abs(got["o"] - ref["o"])) <= 1e-11 * np.max(np.abs(ref["o"]))


# -------------------------------------------------------- chunked prefill ---

def test_query_subset_matches_full_step():
    # decode_sequence(queries=...) evaluates only those queries, with every new
    # row appended: the same values as the full step's rows
    cs = _decode_sequence_case(seed=81, n_pref=20, q_len=6, H=2)
    tab = O.rope_table(cs["L"])
    args = (cs["prefix"], cs["c_new"], cs["k_new"], cs["q_nope"], cs["q_pe"], cs["w_uk"],
            cs["w_uv"], cs["L"], tab, O.default_scale())
    full = O.decode_sequence(*args)
    sub = O.decode_sequence(*args, queries=[5, 0, 3])
    assert np.array_equal(sub["rows"], full["rows"])
    assert np.array_equal(sub["u"], full["u"][[5, 0, 3]])
    assert np.array_equal(sub["lse"], full["lse"][[5, 0, 3]])


def test_chunked_prefill_equals_token_by_token_decode():
    # A chunk of C tokens attended causally in one step gives, for chunk token
    # j, what a one-token decode step gives after the tokens before it were
    # appended one by one: the causal mask inside the chunk, restated as
    # sequential decoding. Catches a chunk token that sees later chunk tokens,
    # or a query rotated at the wrong position.
    C, n_pref, H = 5, 9, 2
    cs = _decode_sequence_case(seed=83, n_pref=n_pref, q_len=C, H=H)
    L = n_pref + C
    tab = O.rope_table(L)
    chunk = O.decode_sequence(cs["prefix"], cs["c_new"], cs["k_new"], cs["q_nope"], cs["q_pe"],
                              cs["w_uk"], cs["w_uv"], L, tab, O.default_scale())
    for j in range(C):
        before = O.make_cache_row(cs["c_new"][:j], cs["k_new"][:j],
                                  np.arange(n_pref, n_pref + j), tab)
        prefix = np.concatenate([cs["prefix"], before], axis=0)
        one = O.decode_sequence(prefix, cs["c_new"][j:j + 1], cs["k_new"][j:j + 1],
                                cs["q_nope"][j:j + 1], cs["q_pe"][j:j + 1], cs["w_uk"],
                                cs["w_uv"], n_pref + j + 1, tab, O.default_scale())
        assert np.max(np.abs(chunk["u"][j] - one["u"][0])) <= 1e-12 * np.max(np.abs(one["u"]))


# -------------------------------------------------------------- FP8 cache ---

def test_e4m3_rounding_matches_torch_float8():
    # E4M3 rounding (nearest, ties to even, subnormals, signed zero) and the
    # bit layout, against torch's float8_e4m3fn cast (finite range only: torch
    # maps values >= 464 to NaN where the cache saturates at 448).
    rng = np.random.default_rng(90)
    v = np.concatenate([rng.standard_normal(200000) * 60, rng.standard_normal(20000) * 0.01,
                        np.array([0.0, -0.0, 448.0, 447.9, 2.0 ** -10, 3 * 2.0 ** -10,
                                  -(2.0 ** -9), 2.0 ** -6, 1.0625, 1.1875, -2.0 ** -11])])
    v = v[np.abs(v) < 464]
    got = O.e4m3_round(v)
    t = torch.from_numpy(v).to(torch.float8_e4m3fn)
    assert np.array_equal(got, t.to(torch.float64).numpy())
    assert np.array_equal(O.e4m3_bits(got), t.view(torch.uint8).numpy())
    codes = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], np.uint8)   # finite codes
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(O.e4m3_value(codes), want)
    assert O.e4m3_round(np.array([460.0, 1e6]))[0] == 448.0      # saturation


def test_fp8_scale_and_error_bound():
    # The per-token scale is the least power of two that brings max|c| to at
    # most 448 (so max|c|/scale is in (224, 448]); every dequantized value is
    # within one E4M3 rounding of the bf16 input.
    rng = np.random.default_rng(91)
    c = synth.f32_to_bf16_bits((rng.standard_normal((300, 512))
                                * np.exp(rng.uniform(-12, 12, (300, 1)))).astype(np.float32))
    codes, scale = O.quantize_latent_fp8(c)
    x = O.bf16_to_f64(c)
    amax = np.abs(x).max(1)
    assert np.all(np.log2(scale) == np.round(np.log2(scale)))
    r = amax / scale
    assert np.all(r <= 448.0) and np.all(r > 224.0)
    deq = O.e4m3_value(codes) * scale[:, None]
    normal = np.abs(x) / scale[:, None] >= 2.0 ** -6
    err = np.abs(deq - x)
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]))
    assert np.all(err[~normal] <= (2.0 ** -10 * np.broadcast_to(scale[:, None], x.shape))[~normal])
    zc, zs = O.quantize_latent_fp8(np.zeros((1, 512), np.uint16))
    assert zs[0] == 1.0 and not zc.any()


def test_fp8_decode_equals_bf16_decode_on_representable_rows():
    # When every latent value is an E4M3 value times a power of two, the FP8
    # cache is lossless: the FP8 step must equal the bf16 step on the same
    # inputs (the new rows' k^R code is the bf16 cache's code).
    rng = np.random.default_rng(92)
    L, q_len, H = 40, 2, 3
    lat = O.e4m3_round(rng.standard_normal((L, 512)) * 100) * 2.0 ** -7
    kr = rng.standard_normal((L, 64))
    rows_bits = np.concatenate([O.round_to_bf16(lat), O.round_to_bf16(kr)], axis=1)
    assert np.array_equal(O.bf16_to_f64(rows_bits[:, :512]), lat)
    prefix = rows_bits[:L - q_len]
    c_new, k_new = rows_bits[L - q_len:, :512], rows_bits[L - q_len:, 512:]
    q_nope = O.round_to_bf16(rng.standard_normal((q_len, H, 128)))
    q_pe = O.round_to_bf16(rng.standard_normal((q_len, H, 64)))
    w_uk = O.round_to_bf16(rng.standard_normal((H, 128, 512)) / 22.6)
    w_uv = O.round_to_bf16(rng.standard_normal((H, 128, 512)) / 22.6)
    tab = O.rope_table(L)
    ref = O.decode_sequence(prefix, c_new, k_new, q_nope, q_pe, w_uk, w_uv, L, tab,
                            O.default_scale())
    pb, ps = O.quantize_latent_fp8(prefix[:, :512])
    prefix8 = np.concatenate([pb, np.ascontiguousarray(prefix[:, 512:].astype("<u2"))
                              .view(np.uint8).reshape(-1, 128)], axis=1)
    got = O.decode_sequence_fp8(prefix8, ps, c_new, k_new, q_nope, q_pe, w_uk, w_uv, L, tab,
                                O.default_scale())
    assert np.max(np.abs(got["u"] - ref["u"])) <= 1e-12 * np.max(np.abs(ref["u"]))
    assert np.array_equal(got["new_rows"][:, 512:].view("<u2"), ref["new_rows"][:, 512:])
