"""CPU tests of the C-ABI library: it loads, exports every declared symbol,
validates arguments before touching the GPU, and its host planner and RoPE
table are correct. No test here launches a kernel."""

import ctypes
import glob
import os
import re

import numpy as np
import pytest

from mla_latent_kv_32_b200 import build as build_mod
from mla_latent_kv_32_b200 import mla
from oracle import mla_oracle as O
from tests._plan import parse_plan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return mla.load()


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"\b(mla_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert "mla_decode_attention" in names and len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    # the binding covers the same set
    for n in names:
        assert n in mla.SIGNATURES, f"{n} has no Python binding"


def test_invalid_arguments_rejected_before_launch(lib):
    with pytest.raises(mla.MlaError) as e:
        mla.mla_cache_append(None, 1, None, 1, 1, None, None, None, 512, None, 64, None, 1, 4,
                             stream=0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT
    with pytest.raises(mla.MlaError) as e:
        mla.mla_absorb_q(16, 2048, 16, 1024, 16, None, None, 0, 1, 24, 16, stream=0)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
    with pytest.raises(mla.MlaError) as e:
        mla.mla_gemm_bf16(16, 16, 16, 16, 8, 16, 0, 4, 4, 16, stream=0)   # C misaligned
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT
    # zero-sized calls are no-ops that succeed without a device
    mla.mla_cache_append(None, 1, None, 1, 1, None, None, None, 512, None, 64, None, 1, 0, stream=0)
    mla.mla_out_absorb(None, None, 0, 128, None, 16384, stream=0)


def test_empty_inputs_are_noops_without_a_device(lib):
    """Every entry point treats an empty problem (no sequences, tokens or rows)
    as a successful no-op that touches neither the GPU nor its pointers."""
    for q_len in (1, 2):
        plan, info = mla.mla_decode_plan(np.zeros(0, np.int32), 0, q_len, 128, num_ctas=8)
        assert info.num_items == 0 and info.num_partials == 0 and info.workspace_bytes == 0
        for fn in (mla.mla_decode_attention, mla.mla_decode_attention_cudacore):
            fn(None, None, 1, None, 1, 0, q_len, 128, 0.07, plan, plan, None, 0, None, stream=0)
        mla.mla_decode_attention_noalloc(None, None, 1, None, 1, 0, q_len, 128, 0.07, plan, plan,
                                         None, stream=0)
    mla.mla_absorb_q(None, 16384, None, 8192, None, None, None, 0, 0, 128, None, stream=0)
    mla.mla_gemm_bf16(None, 64, None, 64, None, 64, 0, 0, 64, 64, stream=0)      # M = 0
    mla.mla_gemm_bf16(None, 64, None, 64, None, 64, 1, 64, 0, 64, stream=0)      # N = 0
    mla.mla_gemm_bf16_ws(None, 64, None, 64, None, 64, 0, 0, 64, 64, None, 0, stream=0)
    assert mla.mla_gemm_bf16_workspace_bytes(0, 64, 64) == 0
    # the fused append + absorption with neither tokens to append nor queries
    mla.mla_append_absorb_q(None, 1, None, 1, 1, None, None, None, 576, None, 576, 0, None, 24576,
                            None, 24576, None, None, None, 1, 0, 128, None, stream=0)
    mla.mla_append_fp8_absorb_q(None, None, 1, None, 1, 1, None, None, None, 576, None, 576, 0,
                                None, 24576, None, 24576, None, None, None, 1, 0, 128, None,
                                stream=0)
    # the FP8 cache's entry points, the folds and the folded absorption
    mla.mla_cache_append_fp8(None, None, 1, None, 1, 1, None, None, None, 512, None, 64, None, 1,
                             0, stream=0)
    plan, _ = mla.mla_decode_plan(np.zeros(0, np.int32), 0, 1, 128, num_ctas=8)
    mla.mla_decode_attention_fp8(None, None, None, 1, None, 1, 0, 1, 128, 0.07, plan, plan, None,
                                 0, None, stream=0)
    mla.mla_fold_qk(None, 1536, 1536, None, 0, None, None, 0, stream=0)
    mla.mla_fold_o(None, 16384, 7168, None, 0, None, stream=0)
    mla.mla_absorb_q_folded(None, 1536, 1536, None, 8192, None, None, None, 1, 0, 128, None,
                            stream=0)


def test_fused_append_absorb_checks_both_halves(lib):
    """mla_append_absorb_q validates the append's and the absorption's
    arguments before launching anything: a NULL cache with tokens to append,
    or an unsupported head count with queries, fails on the host."""
    with pytest.raises(mla.MlaError) as e:
        mla.mla_append_absorb_q(None, 1, None, 1, 1, None, None, None, 576, None, 576, 4, None,
                                24576, None, 24576, None, None, None, 1, 0, 128, None, stream=0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT
    with pytest.raises(mla.MlaError) as e:
        mla.mla_append_absorb_q(None, 1, None, 1, 1, None, None, None, 576, None, 576, 0, 16,
                                2048, 16, 1024, 16, None, None, 0, 1, 24, 16, stream=0)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
    # the FP8 flavour: a NULL scale array with tokens to append
    with pytest.raises(mla.MlaError) as e:
        mla.mla_append_fp8_absorb_q(16, None, 1, 16, 1, 1, 16, 16, 16, 512, 16, 64, 4, 16, 16384,
                                    16, 8192, 16, None, 16, 1, 1, 128, 16, stream=0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT


def test_rope_table_matches_oracle(lib):
    got = mla.mla_rope_table(140000)
    want = O.rope_table(140000)
    # Both round a float64 cos/sin to float32. The float64 angles may differ in
    # their last bit (the two pow implementations differ), which flips the
    # float32 rounding when the value sits next to a rounding midpoint: the
    # tables then differ by one float32 ulp in a handful of entries.
    d = np.abs(got.astype(np.float64) - want.astype(np.float64))
    assert d.max() <= 2.0 ** -24 * 1.0001
    assert (got != want).mean() < 1e-4
    with pytest.raises(mla.MlaError):
        mla.mla_rope_table(0)


def check_plan(lens, q_len, num_ctas, max_split=0, n_h=128):
    lens = np.asarray(lens, np.int32)
    B = len(lens)
    buf, info = mla.mla_decode_plan(lens, B, q_len, n_h, num_ctas, max_split)
    p = parse_plan(buf)
    assert p["num_items"] == info.num_items and p["num_partials"] == info.num_partials
    assert p["num_items"] <= B * q_len + num_ctas
    cover = {}
    for it in p["items"]:
        key = (it["b"], it["j"])
        L = int(lens[it["b"]])
        assert it["L"] == L and it["qpos"] == L - q_len + it["j"]
        assert 0 <= it["page_begin"] < it["page_end"]
        cover.setdefault(key, []).append(it)
    assert len(cover) == B * q_len
    slots = set()
    for (b, j), its in cover.items():
        need = (int(lens[b]) - q_len + j + 1 + 63) // 64
        rng = sorted((i["page_begin"], i["page_end"]) for i in its)
        assert rng[0][0] == 0 and rng[-1][1] == need
        for a, c in zip(rng, rng[1:]):
            assert a[1] == c[0]
        if len(its) == 1:
            assert its[0]["slot"] == -1
        else:
            ss = sorted(i["slot"] for i in its)
            assert ss == list(range(ss[0], ss[0] + len(its)))
            slots.update(ss)
            ci = [c for c in p["combine"] if (c["b"], c["j"]) == (b, j)]
            assert len(ci) == 1 and ci[0]["first_slot"] == ss[0] and ci[0]["n_parts"] == len(its)
    assert len(slots) == p["num_partials"]
    # work lists partition the items
    cb = p["cta_begin"]
    assert cb[0] == 0 and cb[-1] == p["num_items"] and np.all(np.diff(cb) >= 0)
    loads = [sum(p["items"][k]["page_end"] - p["items"][k]["page_begin"]
                 for k in range(cb[c], cb[c + 1])) for c in range(p["num_ctas"])]
    total = sum(need for need in
                [(int(lens[b]) - q_len + j + 1 + 63) // 64 for b in range(B) for j in range(q_len)])
    assert sum(loads) == total
    return p, loads, total


@pytest.mark.parametrize("lens,q_len,ctas", [
    ([4096] * 64, 1, 74), ([1, 63, 64, 65, 127, 200], 1, 3), ([2, 131072, 5000, 64], 2, 74),
    ([1], 1, 74), ([300] * 7, 2, 1)])
def test_planner_contiguous_cuts(lens, q_len, ctas):
    p, loads, total = check_plan(lens, q_len, ctas, max_split=0)
    # cuts fall on 4-page tiles: a list exceeds its equal share by under a tile
    assert max(loads) <= -(-total // min(ctas, total)) + 3
    # every cut inside a unit is tile-aligned
    for it in p["items"]:
        assert it["page_begin"] % 4 == 0


def test_planner_ragged_workload_balanced():
    import synth
    w = synth.WORKLOADS["ragged"]
    lens = synth.seq_lens(w)
    p, loads, total = check_plan(lens, 1, 74, max_split=0)
    # the cut plan balances pages to within a tile of the equal share
    assert max(loads) <= -(-total // 74) + 3 and min(loads) >= total // 74 - 4


def test_planner_no_split_mode():
    p, loads, total = check_plan([4096] * 64, 1, 74, max_split=1)
    assert p["num_partials"] == 0 and p["num_items"] == 64
    assert max(loads) == 64


def test_planner_auto_picks_by_estimate():
    # equal lengths that fill most lists: one item per sequence, no combine
    p, loads, total = check_plan([4096] * 64, 1, 74, max_split=-1)
    assert p["num_partials"] == 0 and p["num_items"] == 64
    # a few very long sequences: cut, merged by the combine pass
    p, loads, total = check_plan([131072] * 4, 2, 74, max_split=-1)
    assert p["num_partials"] > 0 and max(loads) <= -(-total // 74) + 3


def test_planner_rejects_bad_input():
    with pytest.raises(mla.MlaError):
        mla.mla_decode_plan(np.array([1, 0], np.int32), 2, 1, 128, 8)    # L < q_len
    with pytest.raises(mla.MlaError):
        mla.mla_decode_plan(np.array([5, 2], np.int32), 2, 3, 128, 8)    # L < q_len 3
    with pytest.raises(mla.MlaError):
        mla.mla_decode_plan(np.array([5], np.int32), 1, 1, 100, 8)       # n_h 100
    buf, info = mla.mla_decode_plan(np.zeros(0, np.int32), 0, 1, 128, 8)
    assert info.num_items == 0


def test_debug_wait_cap_validated():
    # host-side validation of the failure-detection hook (no launch)
    with pytest.raises(mla.MlaError):
        mla.mla_debug_decode_wait(0.0, 0)
    with pytest.raises(mla.MlaError):
        mla.mla_debug_decode_wait(11.0, 0)
    mla.mla_debug_decode_wait(1.0, 0)


def test_q_len_range(lib):
    # MTP verify depths 1..MLA_MAX_Q_LEN are planned; beyond is unsupported,
    # below one is an invalid argument
    for q_len in (1, 3, 8, 16, 512, mla.MAX_Q_LEN):
        check_plan(np.array([max(40, q_len), q_len + 300], np.int32), q_len, 7)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_plan(np.array([100], np.int32), 1, mla.MAX_Q_LEN + 1, 128, num_ctas=4)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_plan(np.array([100], np.int32), 1, 0, 128, num_ctas=4)
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT


def test_plan_used_bytes_and_upload_checks(lib):
    lens = np.array([3000, 2000, 77], np.int32)
    plan, info = mla.mla_decode_plan(lens, 3, 2, 128, num_ctas=5, max_split=0)
    assert mla.mla_plan_used_bytes(plan) == info.plan_bytes <= plan.nbytes
    assert mla.mla_plan_used_bytes(np.zeros(64, np.uint8)) == 0
    with pytest.raises(mla.MlaError) as e:                       # device buffer too small
        mla.mla_plan_upload(plan, 256, info.plan_bytes - 16, stream=0)
    assert e.value.status == mla.MLA_ERR_WORKSPACE_TOO_SMALL
    with pytest.raises(mla.MlaError) as e:                       # misaligned device buffer
        mla.mla_plan_upload(plan, 258, info.plan_bytes, stream=0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT
    with pytest.raises(mla.MlaError) as e:
        mla.mla_reset_status(None, stream=0)
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT
