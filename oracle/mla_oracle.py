"""CPU fp64 oracle for absorbed Multi-Head Latent Attention decode.

TEST INFRASTRUCTURE. Only the test suite, the package's ``smoke()`` check and
the benchmark's CPU-baseline / reference leg may import this module. The CUDA
product path never imports, links or calls it, and this module imports nothing
from the product package.

What it computes, and where the pages define it:

* Cache row per token: ``[c^KV (512) | k^R (64)]``, stored as bf16 -- "DeepSeek-V3
  MLA: Multi-Head Latent Attention Guide", section "4. Cache Footprint Math"
  (512 + 64 = 576 cached values, "fp8 / bf16" in the topology figure).
* Decoupled RoPE on k^R and q^R with interleaved pairs (2j, 2j+1) and angle
  ``pos / base^(2j/d_R)`` -- "Deconstructing DeepSeek V4 Pro ...", section
  "Hands-On PyTorch Implementation" (``apply_rope``); the key is rotated before
  it is cached -- "DeepSeek-V3 MLA ... Guide", section "3. The Decoupled RoPE
  Key" and "Step 3" of "Production Implementation".
* Non-absorbed attention (the definition): ``k_{j,i} = [W^UK_i c_j ; k^R_j]``,
  ``v_{j,i} = W^UV_i c_j``, ``q_i = [q^C_i ; q^R_i]``, score scaled by
  ``1/sqrt(d_h + d_R)``, softmax over the causal prefix, ``u_i = sum a v`` --
  "DeepSeek-V3 MLA ... Guide", sections "1. Low-Rank Key-Value Joint
  Compression", "3. The Decoupled RoPE Key" and "Step 2" (``forward_train``);
  "Deconstructing DeepSeek V4 Pro ...", "Mathematical Formulation".
* Absorbed attention: ``q~_i = (W^UK_i)^T q^C_i``; ``score_j = q~_i . c_j +
  q^R_i . k^R_j``; ``o_i = sum_j a_j c_j``; ``u_i = W^UV_i o_i`` --
  "DeepSeek-V3 MLA ... Guide", section "Inference Optimization: The Matrix
  Absorption Trick", parts 2 and 3, and "Step 3" (``forward_decode_absorbed``).
* Split-KV merge of partial results (``merge_partials``): the log-sum-exp
  identity; the pages have no split, so this is the plain reading of a
  combine that is exact in real arithmetic.
* FP8 latent cache (``quantize_latent_fp8``, ``make_cache_row_fp8``,
  ``dequant_fp8_rows``, ``decode_sequence_fp8``): E4M3 latent codes with a
  power-of-two per-token scale, bf16 k^R -- "Deconstructing DeepSeek V4 Pro
  ...", "Practical Deployment & Systems Engineering Takeaways"; the attention
  then runs on the exactly dequantized rows.
* Folded weights (``fold_qk``, ``fold_o``): W~QK_h = (W^UK_h)^T W^UQ_h and
  W~O = W^O W^UV per head, applied to the query input and to the latent
  outputs -- "DeepSeek-V3 MLA ... Guide", "The Matrix Absorption Trick",
  parts 2 and 3; equal to the unfolded layer in real arithmetic.
* Whole decode layer (query compression c^Q = W^DQ h, q^C = W^UQ c^Q,
  q^R = RoPE(W^QR c^Q); c^KV = W^DKV h; k^R = RoPE(W^KR h); output W^O u) --
  "DeepSeek-V3 MLA ... Guide", sections 1-3 of "Core Architecture &
  Mathematics"; without query compression, q^C = W_Q x and q^R = RoPE(W_QR x)
  -- "Deconstructing DeepSeek V4 Pro ...", "Hands-On PyTorch Implementation".

Readings where the pages are silent or disagree (each is listed with its
reason in the design notes of the repository):
  - weight views ``W_UK[h][d][c]``, ``W_UV[h][d][c]`` (the ``view(n_heads,
    d_head, d_c_kv)`` of "Step 3");
  - the new token(s) are appended before attention and attend to themselves;
    query j of a q_len-token step sits at position ``L - q_len + j`` and sees
    keys ``i <= L - q_len + j``;
  - no normalisation layers and no biases;
  - the rotation that produces a cached bf16 key is taken in float32 with a
    float32 cos/sin table (each product and sum rounded once, no fused
    multiply-add), because its result is a stored bf16 code that both sides
    must decide in the same precision; everything else is float64.

Arrays of bf16 values travel as uint16 bit patterns.
"""

from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

D_C = 512
D_R = 64
D_NOPE = 128
D_V = 128
ROW_ELEMS = D_C + D_R
BLOCK = 64
ROPE_BASE = 10000.0


# ---------------------------------------------------------------- storage ---

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to bf16 once (nearest, ties to even) -> uint16 bits.

    bf16 keeps 8 significant bits and float32's exponent range; below 2**-126
    the spacing is 2**-133.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    tiny = np.abs(x) < 2.0 ** -126
    r = np.where(tiny, np.rint(x * 2.0 ** 133) * 2.0 ** -133, r)
    with np.errstate(over="ignore"):
        r32 = r.astype(np.float32)
    return (r32.view(np.uint32) >> 16).astype(np.uint16)


def kv_cache_bytes(n_tokens: int, elem_bytes: int = 2, layers: int = 1) -> int:
    """Bytes the latent cache holds: (d_c + d_R) values per token per layer
    ("DeepSeek-V3 MLA ... Guide", "4. Cache Footprint Math")."""
    return int(n_tokens) * ROW_ELEMS * int(elem_bytes) * int(layers)


# ------------------------------------------------------------------- RoPE ---

def rope_angles(pos, d_r: int = D_R, base: float = ROPE_BASE) -> np.ndarray:
    """theta[..., j] = pos / base**(2j/d_r) in float64, j = 0..d_r/2-1."""
    j = np.arange(d_r // 2, dtype=np.float64)
    denom = base ** (2.0 * j / d_r)
    return np.asarray(pos, dtype=np.float64)[..., None] / denom


def rope_table(max_pos: int, d_r: int = D_R, base: float = ROPE_BASE) -> np.ndarray:
    """float32 [max_pos, d_r/2, 2] of (cos, sin), computed in float64 and
    rounded once to float32."""
    th = rope_angles(np.arange(max_pos), d_r, base)
    return np.stack([np.cos(th), np.sin(th)], axis=-1).astype(np.float32)


def rope_f64(x, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Exact (float64) rotation of interleaved pairs over the last axis:
    y[2j] = x[2j] cos - x[2j+1] sin,  y[2j+1] = x[2j+1] cos + x[2j] sin."""
    x = np.asarray(x, dtype=np.float64)
    th = rope_angles(pos, x.shape[-1], base)
    c, s = np.cos(th), np.sin(th)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x1 * c + x0 * s
    return y


def rope_f32_to_bf16(x_bits, cos32, sin32) -> np.ndarray:
    """Rotation that produces a cached k^R code: bf16 input widened to float32,
    each product and each sum a single float32 operation, the result rounded
    once to bf16. cos32/sin32 broadcast against x[..., 0::2]."""
    x = bf16_to_f64(x_bits).astype(np.float32)
    c = np.asarray(cos32, dtype=np.float32)
    s = np.asarray(sin32, dtype=np.float32)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = (x0 * c) - (x1 * s)
    y[..., 1::2] = (x1 * c) + (x0 * s)
    return round_to_bf16(y.astype(np.float64))


# ------------------------------------------------------------------ cache ---

def make_cache_row(c_kv_bits, k_pe_bits, pos, table) -> np.ndarray:
    """New cache rows [n, 576]: c^KV copied, k^R rotated at its position."""
    c_kv_bits = np.asarray(c_kv_bits, dtype=np.uint16).reshape(-1, D_C)
    k_pe_bits = np.asarray(k_pe_bits, dtype=np.uint16).reshape(-1, D_R)
    pos = np.asarray(pos, dtype=np.int64).reshape(-1)
    cs = table[pos]                                   # [n, 32, 2]
    kr = rope_f32_to_bf16(k_pe_bits, cs[..., 0], cs[..., 1])
    return np.concatenate([c_kv_bits, kr], axis=1)


def cache_append(pool, block_table, seq_idx, pos, c_kv_bits, k_pe_bits, table):
    """Write each new token's row into its page slot.

    Token t of sequence b at position p lands in page ``block_table[b][p // 64]``,
    slot ``p % 64``. A token whose page id, sequence, or table position is out
    of range is skipped and reported. Returns (new_pool, skipped[bool n]).
    """
    pool = np.array(pool, dtype=np.uint16, copy=True)
    seq_idx = np.asarray(seq_idx, dtype=np.int64).reshape(-1)
    pos = np.asarray(pos, dtype=np.int64).reshape(-1)
    n = seq_idx.shape[0]
    n_pages = pool.shape[0]
    B, max_pages = block_table.shape
    skipped = np.zeros(n, dtype=bool)
    ok = ((seq_idx >= 0) & (seq_idx < B) & (pos >= 0)
          & (pos // BLOCK < max_pages) & (pos < table.shape[0]))
    rows = np.zeros((n, ROW_ELEMS), dtype=np.uint16)
    if ok.any():
        rows[ok] = make_cache_row(np.asarray(c_kv_bits).reshape(-1, D_C)[ok],
                                  np.asarray(k_pe_bits).reshape(-1, D_R)[ok],
                                  pos[ok], table)
    for t in range(n):
        if not ok[t]:
            skipped[t] = True
            continue
        page = int(block_table[seq_idx[t], pos[t] // BLOCK])
        if page < 0 or page >= n_pages:
            skipped[t] = True
            continue
        pool[page, pos[t] % BLOCK] = rows[t]
    return pool, skipped


def gather_rows(pool, block_table, b: int, L: int) -> np.ndarray:
    """Logical rows 0..L-1 of sequence b (uint16 [L, 576])."""
    n_pages = (L + BLOCK - 1) // BLOCK
    pages = pool[block_table[b, :n_pages]].reshape(n_pages * BLOCK, ROW_ELEMS)
    return pages[:L]


# ------------------------------------------------------------ FP8 cache ---
# An 8-bit latent cache ("Deconstructing DeepSeek V4 Pro ...", "Practical
# Deployment & Systems Engineering Takeaways", quantization strategies: c^KV
# tolerates E4M3 / E5M2; "DeepSeek-V3 MLA ... Guide", "4. Cache Footprint
# Math", an FP8 cache). The pages fix no format; the reading taken here: the
# 512 latent values of a token are E4M3 codes with one power-of-two float32
# scale per token, the decoupled key k^R stays the bf16 code of the bf16 cache
# (its rotation carries the position), so a row is 512 + 128 bytes and the
# scale lives in a separate array.

E4M3_MAX = 448.0


def e4m3_round(v) -> np.ndarray:
    """Round float64 values to the nearest E4M3 value (ties to even),
    saturating at +-448. E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits;
    normals 2^-6 .. 448, subnormals multiples of 2^-9."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)                       # below 2^-6 the spacing stays 2^-9
    step = 2.0 ** (e - 3)
    r = np.rint(a / step) * step                  # rint: ties to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, v)


def e4m3_bits(v) -> np.ndarray:
    """Bit patterns (uint8) of values that are exactly E4M3 (see e4m3_round)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    sign = (v < 0) | ((v == 0) & np.signbit(v))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, e + 7, 0).astype(np.int64)
    mant = np.where(normal, a / 2.0 ** e - 1.0, a / 2.0 ** -6) * 8.0
    mant = np.rint(mant).astype(np.int64)
    return ((sign.astype(np.int64) << 7) | (exp_field << 3) | mant).astype(np.uint8)


def e4m3_value(bits) -> np.ndarray:
    """float64 value of E4M3 bit patterns (uint8), the finite codes."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    ef = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(ef == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (ef - 7.0))
    return s * val


def fp8_token_scale(amax) -> np.ndarray:
    """The power of two 2^k with the least k such that amax / 2^k <= 448
    (1 when amax is 0): the per-token scale of the FP8 cache."""
    amax = np.asarray(amax, dtype=np.float64)
    m, e = np.frexp(np.where(amax > 0, amax, 1.0))      # amax = m 2^e, m in [0.5, 1)
    k = np.where(m <= E4M3_MAX / 512.0, e - 9, e - 8)
    return np.where(amax > 0, np.ldexp(1.0, k), 1.0)


def quantize_latent_fp8(c_kv_bits):
    """Per token: scale = fp8_token_scale(max |c|), codes = E4M3(c / scale).
    Returns (codes uint8 [n, 512], scales float64 [n])."""
    c = bf16_to_f64(np.asarray(c_kv_bits, np.uint16).reshape(-1, D_C))
    scale = fp8_token_scale(np.abs(c).max(axis=1))
    codes = e4m3_bits(e4m3_round(c / scale[:, None]))   # division by 2^k is exact
    return codes, scale


def make_cache_row_fp8(c_kv_bits, k_pe_bits, pos, table):
    """New FP8 cache rows: (bytes uint8 [n, 640] = [512 E4M3 codes | k^R as
    the bf16 code of make_cache_row, little-endian], scales float64 [n])."""
    codes, scale = quantize_latent_fp8(c_kv_bits)
    kr = make_cache_row(c_kv_bits, k_pe_bits, pos, table)[:, D_C:]
    kr_bytes = np.ascontiguousarray(kr.astype("<u2")).view(np.uint8).reshape(-1, 2 * D_R)
    return np.concatenate([codes, kr_bytes], axis=1), scale


def dequant_fp8_rows(row_bytes, scales) -> np.ndarray:
    """float64 rows [n, 576] of FP8 cache rows: latent = code * scale (exact),
    k^R = the stored bf16 values."""
    row_bytes = np.asarray(row_bytes, np.uint8).reshape(-1, D_C + 2 * D_R)
    lat = e4m3_value(row_bytes[:, :D_C]) * np.asarray(scales, np.float64).reshape(-1, 1)
    kr = bf16_to_f64(np.ascontiguousarray(row_bytes[:, D_C:]).view("<u2"))
    return np.concatenate([lat, kr], axis=1)


# -------------------------------------------------------------- attention ---

def softmax_masked(s: np.ndarray, visible: np.ndarray):
    """Softmax over the last axis with invisible entries given weight 0.
    Returns (weights, max, sum) with max/sum over the visible entries."""
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=-1, keepdims=True)
    return e / l, m[..., 0], l[..., 0]


def causal_visible(q_pos, L: int) -> np.ndarray:
    """visible[j, i] = key i is in the causal prefix of the query at q_pos[j]."""
    return np.arange(L)[None, :] <= np.asarray(q_pos)[:, None]


def attend_nonabsorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos,
                       heads: Optional[Sequence[int]] = None):
    """The definition: expand keys and values per head and run softmax attention.

    q_nope [J, H, 128], q_rope [J, H, 64] (already rotated), rows [L, 576]
    (float64 values of the cached bf16 rows), w_uk/w_uv [H, 128, 512].
    Returns u [J, len(heads), 128] and the attention weights [J, len(heads), L].
    """
    q_nope = np.asarray(q_nope, np.float64)
    q_rope = np.asarray(q_rope, np.float64)
    rows = np.asarray(rows, np.float64)
    J, H = q_nope.shape[:2]
    L = rows.shape[0]
    d_c, d_v = w_uk.shape[-1], w_uv.shape[-2]
    heads = list(range(H)) if heads is None else list(heads)
    c, k_r = rows[:, :d_c], rows[:, d_c:]
    vis = causal_visible(q_pos, L)
    u = np.zeros((J, len(heads), d_v))
    att = np.zeros((J, len(heads), L))
    for n, h in enumerate(heads):
        k = np.concatenate([c @ np.asarray(w_uk[h], np.float64).T, k_r], axis=1)  # [L, 192]
        v = c @ np.asarray(w_uv[h], np.float64).T                                  # [L, 128]
        for j in range(J):
            q = np.concatenate([q_nope[j, h], q_rope[j, h]])                      # [192]
            a, _, _ = softmax_masked((k @ q) * scale, vis[j])
            att[j, n] = a
            u[j, n] = a @ v
    return u, att


def attend_latent(q_lat, q_rope, rows, scale, q_pos):
    """Scores on the latent rows and the softmax-weighted latent sum.

    q_lat [J, H, d_c] (the absorbed content query), q_rope [J, H, d_R],
    rows [L, d_c + d_R]: score_i = (q_lat . c_i + q^R . k^R_i) * scale over the
    causal prefix, o = sum_i a_i c_i. Returns o [J, H, d_c] and the
    natural-log sum-exp of the scaled scores lse [J, H].
    """
    q_lat = np.asarray(q_lat, np.float64)
    q_rope = np.asarray(q_rope, np.float64)
    rows = np.asarray(rows, np.float64)
    J, H, d_c = q_lat.shape
    d_r = q_rope.shape[-1]
    L = rows.shape[0]
    c, k_r = rows[:, :d_c], rows[:, d_c:]
    s = (q_lat.reshape(J * H, d_c) @ c.T
         + q_rope.reshape(J * H, d_r) @ k_r.T).reshape(J, H, L) * scale
    vis = causal_visible(q_pos, L)[:, None, :]
    a, m, l = softmax_masked(s, vis)
    o = (a.reshape(J * H, L) @ c).reshape(J, H, d_c)               # sum_j a_j c_j
    return o, m + np.log(l)


def attend_absorbed(q_nope, q_rope, rows, w_uk, w_uv, scale, q_pos):
    """Absorbed form over the latent rows.

    Returns u [J, H, 128], the latent output o [J, H, 512] and the natural-log
    sum-exp of the scaled scores lse [J, H].
    """
    q_nope = np.asarray(q_nope, np.float64)
    w_uk = np.asarray(w_uk, np.float64)
    w_uv = np.asarray(w_uv, np.float64)
    q_lat = np.einsum("jhd,hdc->jhc", q_nope, w_uk)                # (W^UK_i)^T q^C_i
    o, lse = attend_latent(q_lat, q_rope, rows, scale, q_pos)
    u = np.einsum("jhc,hdc->jhd", o, w_uv)                         # W^UV_i o_i
    return u, o, lse


def fold_qk(w_up_bits, w_uk_bits, n_h: int) -> np.ndarray:
    """Query-side fold, float64: W~QK[h*d_c + c][i] = sum_d W_up[h*d_h + d][i]
    W^UK[h][d][c], so that q~_h = W~QK_h x straight from the query input x
    (c^Q, or h without a query latent). W_up is W^UQ (or W_Q), [n_h*d_h, q_in]
    ("DeepSeek-V3 MLA ... Guide", "The Matrix Absorption Trick", part 2;
    "Deconstructing DeepSeek V4 Pro ...", "Practical Deployment & Systems
    Engineering Takeaways": the product computed once, offline)."""
    w_up = bf16_to_f64(w_up_bits)
    w_uk = bf16_to_f64(w_uk_bits)
    d_h, d_c = w_uk.shape[1], w_uk.shape[2]
    q_in = w_up.shape[1]
    out = np.empty((n_h * d_c, q_in))
    for h in range(n_h):
        out[h * d_c:(h + 1) * d_c] = w_uk[h].T @ w_up[h * d_h:(h + 1) * d_h]
    return out


def fold_o(w_o_bits, w_uv_bits, n_h: int) -> np.ndarray:
    """Output-side fold, float64: W~O[f][h*d_c + c] = sum_d W^O[f][h*d_v + d]
    W^UV[h][d][c], so that out = W~O [o_1; ...; o_H] straight from the latent
    attention outputs ("DeepSeek-V3 MLA ... Guide", "The Matrix Absorption
    Trick", part 3: W^UV pre-multiplied into the output projection)."""
    w_o = bf16_to_f64(w_o_bits)
    w_uv = bf16_to_f64(w_uv_bits)
    d_v, d_c = w_uv.shape[1], w_uv.shape[2]
    out = np.empty((w_o.shape[0], n_h * d_c))
    for h in range(n_h):
        out[:, h * d_c:(h + 1) * d_c] = w_o[:, h * d_v:(h + 1) * d_v] @ w_uv[h]
    return out


def merge_partials(o_parts, lse_parts):
    """Merge attention results taken over disjoint key ranges (split-KV).

    The pages have no split; this is the log-sum-exp identity that makes a
    split exact in real arithmetic. With lse_s the log of the sum of exp(score)
    over range s and o_s the softmax-weighted mean of range s's rows, the
    whole range has lse = log(sum_s exp(lse_s)) and o = sum_s exp(lse_s - lse)
    o_s. A range without a visible key (lse_s = -inf) gets weight 0.
    o_parts [S, ..., d], lse_parts [S, ...]; returns (o [..., d], lse [...]).
    """
    o_parts = np.asarray(o_parts, np.float64)
    lse_parts = np.asarray(lse_parts, np.float64)
    m = lse_parts.max(axis=0)
    m_ref = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - m_ref)                      # exp(-inf) = 0
    tot = w.sum(axis=0)
    lse = np.where(tot > 0, m_ref + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    o = (w[..., None] * o_parts).sum(axis=0) / np.where(tot > 0, tot, 1.0)[..., None]
    return o, lse


def default_scale(d_nope: int = D_NOPE, d_r: int = D_R) -> float:
    """1/sqrt(d_h + d_R), the score scale of both PyTorch modules on the pages."""
    return 1.0 / math.sqrt(d_nope + d_r)


# ------------------------------------------------------- attention step ----

def decode_sequence_fp8(prefix_bytes, prefix_scales, c_new_bits, k_new_bits, q_nope_bits,
                        q_pe_bits, w_uk_bits, w_uv_bits, L: int, table, scale: float,
                        queries=None):
    """One decode step over an FP8 cache: the new tokens are quantized and
    appended (make_cache_row_fp8), every row is dequantized exactly, then the
    absorbed attention of decode_sequence runs on those values."""
    q_len = np.asarray(q_nope_bits).shape[0]
    pos = np.arange(L - q_len, L)
    new_rows, new_scales = make_cache_row_fp8(c_new_bits, k_new_bits, pos, table)
    rows_b = np.concatenate([np.asarray(prefix_bytes, np.uint8).reshape(-1, D_C + 2 * D_R),
                             new_rows], axis=0)
    scales = np.concatenate([np.asarray(prefix_scales, np.float64).reshape(-1), new_scales])
    rows = dequant_fp8_rows(rows_b, scales)
    sel = np.arange(q_len) if queries is None else np.asarray(queries, dtype=np.int64)
    q_nope = bf16_to_f64(np.asarray(q_nope_bits)[sel])
    q_rope = rope_f64(bf16_to_f64(np.asarray(q_pe_bits)[sel]), pos[sel][:, None])
    u, o, lse = attend_absorbed(q_nope, q_rope, rows, bf16_to_f64(w_uk_bits),
                                bf16_to_f64(w_uv_bits), scale, pos[sel])
    return {"new_rows": new_rows, "new_scales": new_scales, "u": u, "o": o, "lse": lse}


def decode_sequence(prefix_bits, c_new_bits, k_new_bits, q_nope_bits, q_pe_bits,
                    w_uk_bits, w_uv_bits, L: int, table, scale: float,
                    form: str = "absorbed", heads=None, queries=None):
    """One attention-only decode step for one sequence of L tokens.

    prefix_bits: the first L-q_len cached rows (uint16 [L-q_len, 576]);
    c_new/k_new: the q_len new tokens' latent and pre-RoPE key (appended at
    positions L-q_len..L-1 before attention); q_nope/q_pe: [q_len, H, .] with
    q_pe pre-RoPE (rotated here exactly, at the query's position). A chunk of
    prefill is the same step with q_len = the chunk length.
    ``queries``: indices j of the query tokens to evaluate (default all; every
    new row is appended either way). Returns dict with the full row block and
    the outputs of the chosen form for those queries.
    """
    q_len = np.asarray(q_nope_bits).shape[0]
    pos = np.arange(L - q_len, L)
    new_rows = make_cache_row(c_new_bits, k_new_bits, pos, table)
    rows_bits = np.concatenate([np.asarray(prefix_bits, np.uint16).reshape(-1, ROW_ELEMS),
                                new_rows], axis=0)
    rows = bf16_to_f64(rows_bits)
    sel = np.arange(q_len) if queries is None else np.asarray(queries, dtype=np.int64)
    q_nope_bits = np.asarray(q_nope_bits)[sel]
    q_pe_bits = np.asarray(q_pe_bits)[sel]
    pos = pos[sel]
    q_nope = bf16_to_f64(q_nope_bits)
    q_rope = rope_f64(bf16_to_f64(q_pe_bits), pos[:, None])
    out = {"rows": rows_bits, "new_rows": new_rows}
    if form == "absorbed":
        u, o, lse = attend_absorbed(q_nope, q_rope, rows, bf16_to_f64(w_uk_bits),
                                    bf16_to_f64(w_uv_bits), scale, pos)
        out.update(u=u, o=o, lse=lse)
    else:
        u, att = attend_nonabsorbed(q_nope, q_rope, rows, bf16_to_f64(w_uk_bits),
                                    bf16_to_f64(w_uv_bits), scale, pos, heads)
        out.update(u=u, att=att)
    return out


# ------------------------------------------------------------ whole layer ---

def layer_project(h_bits, weights: Dict[str, np.ndarray], n_h: int, tok_pos):
    """Projections and RoPE of the tokens entering the layer (all float64).

    Returns dict: q_nope [T, H, 128], q_rope [T, H, 64] (rotated),
    c_kv [T, 512], k_r [T, 64] (rotated), all float64.
    """
    h = bf16_to_f64(h_bits)
    W = {k: bf16_to_f64(v) for k, v in weights.items()}
    T = h.shape[0]
    d_nope = W["w_uk"].shape[1]
    if "w_dq" in W:
        c_q = h @ W["w_dq"].T                      # c^Q = W^DQ h
        q_c = c_q @ W["w_uq"].T                    # q^C = W^UQ c^Q
        q_r = c_q @ W["w_qr"].T                    # W^QR c^Q (pre-RoPE)
        x_q = c_q
    else:
        q_c = h @ W["w_q"].T
        q_r = h @ W["w_qr"].T
        x_q = h
    c_kv = h @ W["w_dkv"].T                        # c^KV = W^DKV h
    k_r = h @ W["w_kr"].T                          # W^KR h (pre-RoPE)
    tok_pos = np.asarray(tok_pos)
    return {
        "x_q": x_q,
        "q_nope": q_c.reshape(T, n_h, d_nope),
        "q_rope": rope_f64(q_r.reshape(T, n_h, -1), tok_pos[:, None]),
        "c_kv": c_kv,
        "k_r": rope_f64(k_r, tok_pos),
    }


def layer_decode(h_bits, weights, n_h: int, q_len: int, tok_seq, tok_pos, query_tok,
                 prefix_of, lens, scale: float, seqs: Optional[Sequence[int]] = None,
                 fold: Optional[Dict[str, np.ndarray]] = None):
    """Whole decode layer in float64.

    prefix_of(b, n) -> uint16 [n, 576] returns the synthetic prefix rows of
    sequence b (rows whose tokens do not enter the layer this step). The rows
    computed from h are rounded to bf16 for storage (the cache is a bf16 cache)
    before attention. With ``fold`` = {"w_qk": W~QK, "w_o": W~O} (float64, see
    fold_qk / fold_o) the latent query is W~QK x and the output W~O o instead
    of going through q^C, W^UK, W^UV and W^O. Returns dict(out [B*q_len,
    hidden] for the chosen sequences' queries, u [.., H, 128], o, lse,
    new_rows).
    """
    tok_seq = np.asarray(tok_seq)
    tok_pos = np.asarray(tok_pos)
    query_tok = np.asarray(query_tok)
    B = len(lens)
    seqs = list(range(B)) if seqs is None else list(seqs)
    need = np.zeros(tok_seq.shape[0], dtype=bool)
    for b in seqs:
        need |= tok_seq == b
    idx = np.nonzero(need)[0]
    pr = layer_project(np.asarray(h_bits)[idx], weights, n_h, tok_pos[idx])
    new_rows = np.concatenate([round_to_bf16(pr["c_kv"]), round_to_bf16(pr["k_r"])], axis=1)
    local = {int(t): n for n, t in enumerate(idx)}
    w_uk = bf16_to_f64(weights["w_uk"])
    w_uv = bf16_to_f64(weights["w_uv"])
    w_o = bf16_to_f64(weights["w_o"])
    outs, us, os_, lses = [], [], [], []
    for b in seqs:
        L = int(lens[b])
        toks = idx[tok_seq[idx] == b]
        rows = np.zeros((L, new_rows.shape[1]), dtype=np.uint16)
        computed = np.zeros(L, dtype=bool)
        for t in toks:
            rows[tok_pos[t]] = new_rows[local[int(t)]]
            computed[tok_pos[t]] = True
        n_pref = int((~computed).sum())
        if n_pref:
            assert not computed[:n_pref].any() and computed[n_pref:].all()
            rows[:n_pref] = prefix_of(b, n_pref)
        qt = query_tok[b * q_len:(b + 1) * q_len]
        ql = np.array([local[int(t)] for t in qt])
        if fold is None:
            u, o, lse = attend_absorbed(pr["q_nope"][ql], pr["q_rope"][ql], bf16_to_f64(rows),
                                        w_uk, w_uv, scale, tok_pos[qt])
            outs.append(u.reshape(q_len, -1) @ w_o.T)               # W^O [u_1; ...; u_H]
        else:
            q_lat = (pr["x_q"][ql] @ fold["w_qk"].T).reshape(q_len, n_h, -1)
            o, lse = attend_latent(q_lat, pr["q_rope"][ql], bf16_to_f64(rows), scale,
                                   tok_pos[qt])
            u = np.einsum("jhc,hdc->jhd", o, w_uv)
            outs.append(o.reshape(q_len, -1) @ fold["w_o"].T)       # W~O [o_1; ...; o_H]
        us.append(u)
        os_.append(o)
        lses.append(lse)
    return {
        "out": np.concatenate(outs, axis=0),
        "u": np.concatenate(us, axis=0),
        "o": np.concatenate(os_, axis=0),
        "lse": np.concatenate(lses, axis=0),
        "new_rows": new_rows,
        "new_tok": idx,
    }
