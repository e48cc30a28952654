"""Seeded synthetic workloads for absorbed MLA decode over a paged latent cache.

The five workloads mirror the DeepSeek-V2/V3 attention shapes that the MLA
pages describe ("DeepSeek-V3 MLA: Multi-Head Latent Attention Guide", section
"Multi-Head Latent Attention (MLA): Core Architecture & Mathematics": d = 7168,
d_c = 512, d'_c = 1536, 128 heads of 128 dims, 64-dim decoupled RoPE key).

Everything here is input preparation only:
  * every tensor is drawn from its own numpy PCG64 stream, keyed by
    ``(seed, stream_id, index)``, so a single sequence's rows can be
    regenerated without drawing the rest of the pool;
  * normal draws are made in float32, scaled by the stated standard deviation
    and rounded to bf16 storage (round to nearest even);
  * the paged pool, the shuffled block table and the filler rows are laid out.

bf16 tensors are returned as ``uint16`` bit patterns.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

D_C = 512      # latent width of c^KV
D_R = 64       # decoupled RoPE key width k^R
D_NOPE = 128   # per-head content query/key width
D_V = 128      # per-head value width
ROW = D_C + D_R  # elements per cached token: [c^KV | k^R]
BLOCK = 64     # tokens per cache page

# Filler written into every pool slot that holds no prefix token: the slots of
# the new tokens before they are appended and the unused tail of each
# sequence's last page. It is finite (so a masked token times a zero weight is
# zero) and large (so a token that escapes the mask ruins the result).
FILL_BITS = np.uint16(0x4280)  # bf16 64.0

# Stream ids. Each tensor draws from default_rng([seed, stream_id, ...]).
S_CACHE, S_PERM, S_LENS, S_QNOPE, S_QPE, S_CNEW, S_KNEW, S_WUK, S_WUV = range(9)
S_H, S_WDQ, S_WUQ, S_WQR, S_WDKV, S_WKR, S_WO, S_WQ = range(9, 17)


def stream(seed: int, *ids: int) -> np.random.Generator:
    """Independent PCG64 stream for (seed, ids...)."""
    return np.random.default_rng([int(seed), *[int(i) for i in ids]])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) draws in float32, rounded to bf16 bits."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic MLA decode workload.

    lens: "uniform" (every sequence holds ``L`` tokens) or "ragged" (lengths
    drawn uniformly from the integers 1..L).
    layer: True when the workload runs the whole decode layer (projections,
    RoPE, append, absorbed attention, W_UV, W_O) from hidden states.
    """

    name: str
    B: int
    q_len: int
    L: int
    n_h: int
    lens: str = "uniform"
    layer: bool = False
    hidden: int = 0
    q_lora: int = 0          # 0 = no query compression (direct W_Q from h)
    synth_prefix: bool = True  # False = every cached token comes from h
    seed: int = 0


WORKLOADS: Dict[str, Workload] = {
    # Tiny decode layer: 1 sequence, the 256 tokens all appended from h.
    "tiny": Workload("tiny", B=1, q_len=1, L=256, n_h=16, layer=True,
                     hidden=1024, q_lora=0, synth_prefix=False),
    # DeepSeek-V3-shaped absorbed decode, uniform context.
    "v3": Workload("v3", B=64, q_len=1, L=4096, n_h=128),
    # Ragged context lengths 1..32768, exercises split-KV + combine.
    "ragged": Workload("ragged", B=128, q_len=1, L=32768, n_h=128, lens="ragged"),
    # Long context with two causal query tokens per sequence (MTP verify).
    "long_mtp": Workload("long_mtp", B=4, q_len=2, L=131072, n_h=128),
    # Full decode layer at V3 dims over an 8192-token context.
    "layer_v3": Workload("layer_v3", B=256, q_len=1, L=8192, n_h=128, layer=True,
                         hidden=7168, q_lora=1536),
    # Multi-token-prediction verify with eight draft tokens per sequence.
    "mtp8": Workload("mtp8", B=8, q_len=8, L=32768, n_h=128),
    # Chunked prefill: a 512-token chunk per sequence appended at the end of a
    # 4096-token context, every chunk token a causal query.
    "prefill": Workload("prefill", B=4, q_len=512, L=4096, n_h=128),
}


def seq_lens(w: Workload) -> np.ndarray:
    """Total tokens per sequence, including the q_len new ones (int32 [B])."""
    if w.lens == "uniform":
        return np.full(w.B, w.L, dtype=np.int32)
    lens = stream(w.seed, S_LENS).integers(1, w.L, size=w.B, endpoint=True)
    return np.maximum(lens, w.q_len).astype(np.int32)


def pages_needed(lens: np.ndarray) -> np.ndarray:
    return (np.asarray(lens, dtype=np.int64) + BLOCK - 1) // BLOCK


def block_table(w: Workload, lens: np.ndarray) -> np.ndarray:
    """Fisher-Yates-shuffled page ids; sequence b takes the next ceil(L_b/64).

    Unused table entries are -1. Returns int32 [B, max_pages].
    """
    npg = pages_needed(lens)
    total = int(npg.sum())
    perm = stream(w.seed, S_PERM).permutation(total).astype(np.int32)
    table = np.full((w.B, int(npg.max())), -1, dtype=np.int32)
    off = 0
    for b in range(w.B):
        table[b, : npg[b]] = perm[off: off + npg[b]]
        off += npg[b]
    return table


def prefix_rows(w: Workload, b: int, n_rows: int) -> np.ndarray:
    """The n_rows cached rows [c^KV | k^R] of sequence b, N(0,1) bf16 bits."""
    return normal_bf16(stream(w.seed, S_CACHE, b), (n_rows, ROW))


def build_pool(w: Workload, lens: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Paged pool uint16 [num_pages, 64, 576] before the new tokens are appended.

    Positions 0..L_b-q_len-1 of sequence b hold its synthetic prefix (when the
    workload has one); every other slot holds FILL_BITS.
    """
    npg = pages_needed(lens)
    pool = np.full((int(npg.sum()), BLOCK, ROW), FILL_BITS, dtype=np.uint16)
    if not w.synth_prefix:
        return pool
    for b in range(w.B):
        n_prefix = int(lens[b]) - w.q_len
        if n_prefix <= 0:
            continue
        rows = prefix_rows(w, b, n_prefix)
        full = n_prefix // BLOCK
        if full:
            pool[table[b, :full]] = rows[: full * BLOCK].reshape(full, BLOCK, ROW)
        rem = n_prefix - full * BLOCK
        if rem:
            pool[table[b, full], :rem] = rows[full * BLOCK:]
    return pool


@dataclasses.dataclass
class DecodeInputs:
    """Per-step inputs of an attention-only workload (bf16 as uint16 bits).

    The new tokens of sequence b sit at positions L_b-q_len .. L_b-1; their
    rows arrive pre-RoPE (c_new, k_new) and are appended before attention.
    q_pe is the pre-RoPE query side channel.
    """

    w: Workload
    lens: np.ndarray          # int32 [B]
    table: np.ndarray         # int32 [B, max_pages]
    pool: np.ndarray          # uint16 [pages, 64, 576]
    q_nope: np.ndarray        # uint16 [B, q_len, n_h, 128]
    q_pe: np.ndarray          # uint16 [B, q_len, n_h, 64]
    c_new: np.ndarray         # uint16 [B, q_len, 512]
    k_new: np.ndarray         # uint16 [B, q_len, 64]
    w_uk: np.ndarray          # uint16 [n_h, 128, 512]
    w_uv: np.ndarray          # uint16 [n_h, 128, 512]

    @property
    def positions(self) -> np.ndarray:
        """int32 [B, q_len] absolute positions of the new tokens."""
        j = np.arange(self.w.q_len, dtype=np.int32)
        return (self.lens[:, None] - self.w.q_len + j[None, :]).astype(np.int32)


def attention_weights(w: Workload):
    """W_UK, W_UV ~ N(0, 1/512) (fan_in = d_c), bf16 bits [n_h, 128, 512]."""
    std = 1.0 / math.sqrt(D_C)
    w_uk = normal_bf16(stream(w.seed, S_WUK), (w.n_h, D_NOPE, D_C), std)
    w_uv = normal_bf16(stream(w.seed, S_WUV), (w.n_h, D_V, D_C), std)
    return w_uk, w_uv


def make_decode_inputs(w: Workload, with_pool: bool = True, lens=None) -> DecodeInputs:
    """Inputs of workload w; ``lens`` overrides its sequence lengths."""
    lens = seq_lens(w) if lens is None else np.asarray(lens, dtype=np.int32)
    assert lens.shape == (w.B,) and lens.min() >= w.q_len
    table = block_table(w, lens)
    pool = build_pool(w, lens, table) if with_pool else None
    q_nope = normal_bf16(stream(w.seed, S_QNOPE), (w.B, w.q_len, w.n_h, D_NOPE))
    q_pe = normal_bf16(stream(w.seed, S_QPE), (w.B, w.q_len, w.n_h, D_R))
    c_new = normal_bf16(stream(w.seed, S_CNEW), (w.B, w.q_len, D_C))
    k_new = normal_bf16(stream(w.seed, S_KNEW), (w.B, w.q_len, D_R))
    w_uk, w_uv = attention_weights(w)
    return DecodeInputs(w, lens, table, pool, q_nope, q_pe, c_new, k_new, w_uk, w_uv)


@dataclasses.dataclass
class LayerInputs:
    """Inputs of a whole decode layer (bf16 as uint16 bits).

    h holds the hidden states of the tokens that enter the layer this step,
    ``tok_seq``/``tok_pos`` their sequence and position. Weights follow
    nn.Linear's [out_features, in_features] layout, N(0, 1/fan_in).
    When q_lora == 0 the content and RoPE queries come straight from h
    (w_q, w_qr over the hidden size); otherwise through c^Q (w_dq, w_uq, w_qr).
    """

    w: Workload
    lens: np.ndarray
    table: np.ndarray
    pool: np.ndarray
    h: np.ndarray             # uint16 [T, hidden]
    tok_seq: np.ndarray       # int32 [T]
    tok_pos: np.ndarray       # int32 [T]
    query_tok: np.ndarray     # int32 [B*q_len]: which rows of h are queries
    weights: Dict[str, np.ndarray]


def make_layer_inputs(w: Workload, with_pool: bool = True, lens=None) -> LayerInputs:
    """Inputs of layer workload w; ``lens`` overrides its sequence lengths."""
    assert w.layer
    lens = seq_lens(w) if lens is None else np.asarray(lens, dtype=np.int32)
    assert lens.shape == (w.B,) and lens.min() >= w.q_len
    table = block_table(w, lens)
    pool = build_pool(w, lens, table) if with_pool else None
    if w.synth_prefix:
        # one token per query enters the layer: the newest of each sequence
        tok_seq = np.repeat(np.arange(w.B, dtype=np.int32), w.q_len)
        tok_pos = (np.repeat(lens, w.q_len)
                   - w.q_len + np.tile(np.arange(w.q_len), w.B)).astype(np.int32)
        query_tok = np.arange(w.B * w.q_len, dtype=np.int32)
    else:
        # every token of every sequence enters the layer; the last q_len query
        tok_seq = np.concatenate([np.full(int(l), b, np.int32) for b, l in enumerate(lens)])
        tok_pos = np.concatenate([np.arange(int(l), dtype=np.int32) for l in lens])
        ends = np.cumsum(lens)
        query_tok = np.concatenate(
            [np.arange(int(e) - w.q_len, int(e), dtype=np.int32) for e in ends])
    T = tok_seq.shape[0]
    d, n_h = w.hidden, w.n_h
    h = normal_bf16(stream(w.seed, S_H), (T, d))

    def lin(sid, out_f, in_f):
        return normal_bf16(stream(w.seed, sid), (out_f, in_f), 1.0 / math.sqrt(in_f))

    wts: Dict[str, np.ndarray] = {}
    if w.q_lora:
        wts["w_dq"] = lin(S_WDQ, w.q_lora, d)
        wts["w_uq"] = lin(S_WUQ, n_h * D_NOPE, w.q_lora)
        wts["w_qr"] = lin(S_WQR, n_h * D_R, w.q_lora)
    else:
        wts["w_q"] = lin(S_WQ, n_h * D_NOPE, d)
        wts["w_qr"] = lin(S_WQR, n_h * D_R, d)
    wts["w_dkv"] = lin(S_WDKV, D_C, d)
    wts["w_kr"] = lin(S_WKR, D_R, d)
    wts["w_uk"], wts["w_uv"] = attention_weights(w)
    wts["w_o"] = lin(S_WO, d, n_h * D_V)
    return LayerInputs(w, lens, table, pool, h, tok_seq, tok_pos, query_tok, wts)


def sample_sequences(w: Workload, lens: np.ndarray, k: int, seed: int = 1) -> List[int]:
    """k sequence ids for sampled full-size checks: always the shortest and the
    longest, the rest drawn without replacement from the seeded stream."""
    order = np.argsort(lens, kind="stable")
    pick = {int(order[0]), int(order[-1])}
    rest = [b for b in stream(seed, 99).permutation(w.B).tolist() if b not in pick]
    for b in rest:
        if len(pick) >= min(k, w.B):
            break
        pick.add(int(b))
    return sorted(pick)


def sample_heads(n_h: int, k: int, seed: int = 2) -> List[int]:
    """k head ids: always 0 and n_h-1, the rest from the seeded stream."""
    pick = {0, n_h - 1}
    for h in stream(seed, 98).permutation(n_h).tolist():
        if len(pick) >= min(k, n_h):
            break
        pick.add(int(h))
    return sorted(pick)


__all__ = [
    "D_C", "D_R", "D_NOPE", "D_V", "ROW", "BLOCK", "FILL_BITS",
    "Workload", "WORKLOADS", "DecodeInputs", "LayerInputs",
    "stream", "f32_to_bf16_bits", "bf16_bits_to_f32", "normal_bf16",
    "seq_lens", "pages_needed", "block_table", "prefix_rows", "build_pool",
    "attention_weights", "make_decode_inputs", "make_layer_inputs",
    "sample_sequences", "sample_heads",
]
