"""The tensor-core GEMM's tile planner, on the CPU (mla_debug_gemm_plan).

Every plan must cover the problem exactly once: the N and M tiles cover N
and M with no empty tile, the splits over K cover the k-chunks with no empty
split, the accumulators fit the 512 TMEM columns, partial-sum tiles appear
only for an fp32 output given a workspace (at most 8 splits, the workspace
sized for all of them), and atomic splits keep the grid within two waves.
The layer's projection shapes get the plans the measurements chose.
"""

import itertools

import pytest

from mla_latent_kv_32_b200 import mla

SHAPES = [(M, N, K, b) for M, N, K, b in itertools.product(
    (64, 128, 576, 1000, 1024, 1536, 7168, 24576), (1, 7, 64, 100, 256, 300),
    (64, 128, 640, 1536, 7168, 16384), (1, 16, 128))
    if M * N * b <= 24576 * 300 * 16]


@pytest.mark.parametrize("a_mn,c_fp32,fp32_part,atomic_split",
                         [(0, 0, 0, 0), (0, 0, 0, 1), (0, 1, 0, 1), (0, 1, 1, 0), (1, 0, 0, 0)])
def test_plan_covers_the_problem(a_mn, c_fp32, fp32_part, atomic_split):
    for M, N, K, batch in SHAPES:
        p = mla.mla_debug_gemm_plan(M, N, K, batch, a_mn, c_fp32, fp32_part, atomic_split, 148)
        kchunks = (K + 63) // 64
        rows = 128 * p["accumulators"]
        assert p["BN"] % 16 == 0 and 16 <= p["BN"] <= 256
        assert p["ntile"] * p["BN"] >= N > (p["ntile"] - 1) * p["BN"]
        assert p["mtile"] * rows >= M > (p["mtile"] - 1) * rows
        assert p["accumulators"] in (1, 2) and p["accumulators"] * p["BN"] <= 512
        if p["accumulators"] == 2:
            assert not a_mn and M >= 1024
        s, kc = p["splits"], p["k_chunks"]
        assert s * kc >= kchunks > (s - 1) * kc, (M, N, K, batch, p)
        if not (atomic_split or (c_fp32 and fp32_part)):
            assert s == 1
        if p["part"]:
            assert c_fp32 and fp32_part and 2 <= s <= 8
            need = (s * M * N * batch * 4 + 255) // 256 * 256
            assert p["part_bytes"] == min(need, 2 ** 31 - 1)
        else:
            assert p["part_bytes"] == 0
            if s > 1:
                assert p["ntile"] * p["mtile"] * batch * s <= 296


def test_layer_projection_plans():
    # W_O at 256 tokens (fp32 out, workspace): 256-row tiles, 5 partial-sum
    # splits; [W_UQ|W_QR]: 256-row tiles, no split; W_DQ and [W_DKV|W_KR]
    # (bf16 out, workspace): 128-row tiles split 16 ways with atomic sums; the
    # v3 absorption (W_UK read MN-major, 128 heads): 128-row tiles, no split
    p = mla.mla_debug_gemm_plan(7168, 256, 16384, 1, 0, 1, 1, 0, 148)
    assert (p["accumulators"], p["splits"], p["part"]) == (2, 5, 1)
    p = mla.mla_debug_gemm_plan(24576, 256, 1536, 1, 0, 0, 0, 1, 148)
    assert (p["accumulators"], p["mtile"], p["splits"]) == (2, 96, 1)
    for M in (1536, 576):
        p = mla.mla_debug_gemm_plan(M, 256, 7168, 1, 0, 0, 0, 1, 148)
        assert (p["accumulators"], p["splits"], p["part"]) == (1, 16, 0)
    p = mla.mla_debug_gemm_plan(512, 64, 128, 128, 1, 0, 0, 0, 148)
    assert (p["BN"], p["accumulators"], p["mtile"], p["splits"]) == (64, 1, 4, 1)


def test_plan_rejects_bad_sizes():
    with pytest.raises(mla.MlaError) as e:
        mla.mla_debug_gemm_plan(0, 64, 64)
    assert e.value.status == mla.MLA_ERR_INVALID_ARGUMENT
