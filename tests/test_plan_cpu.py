"""Host-side work planning of the GEMM (no GPU needed): tile size, split-K and the cluster
hand-off, through apex_debug_gemm_plan with an explicit SM count."""
import numpy as np
import pytest

import group_quantized_w4a4_b200 as apex

SMS = 148   # a B200


@pytest.fixture(scope="module", autouse=True)
def lib():
    apex.load_library()


def plan(M, N, K, sms=SMS, ws=True):
    return apex.apex_debug_gemm_plan(M, N, K, sms, ws)


def test_decode_splits_every_tile_over_a_two_cta_cluster():
    p = plan(16, 8192, 8192)
    assert p == {"bt": 16, "tiles": 64, "stages": 16, "ctas": 128, "split_k": 1, "cluster": 2}


@pytest.mark.parametrize("N,ways", [(4096, 4), (5120, 3), (8192, 2)])
def test_cluster_size_is_the_even_split(N, ways):
    p = plan(16, N, 8192)
    assert p["cluster"] == ways and p["ctas"] == ways * p["tiles"]


def test_32_token_tiles_cluster_up_to_two():
    assert plan(32, 8192, 8192)["cluster"] == 2
    p = plan(32, 4096, 8192)                   # four ways: parts go through global memory
    assert p["ctas"] == 4 * p["tiles"] and p["cluster"] == 1


def test_wide_splits_and_wide_tiles_use_global_memory():
    p = plan(16, 2048, 8192)                   # 9 CTAs per tile
    assert (p["ctas"], p["split_k"], p["cluster"]) == (144, 1, 1)
    assert plan(64, 8192, 8192)["cluster"] == 1   # 64-token parts do not fit the owner


def test_many_tiles_run_whole_tiles():
    p = plan(4096, 8192, 8192)
    assert (p["bt"], p["tiles"], p["ctas"], p["split_k"], p["cluster"]) == (128, 2048, SMS, 0, 1)


def test_no_workspace_means_no_split():
    p = plan(16, 8192, 8192, ws=False)
    assert (p["split_k"], p["cluster"], p["ctas"]) == (0, 1, 64)


def test_plan_invariants_over_random_shapes():
    rng = np.random.default_rng(7)
    for _ in range(400):
        M = int(rng.choice([1, 5, 16, 17, 32, 33, 64, 100, 128, 1000, 4096]))
        N = int(rng.integers(1, 40000))
        K = 128 * int(rng.integers(1, 256))
        sms = int(rng.choice([8, 64, 132, 148]))
        p = plan(M, N, K, sms)
        assert 1 <= p["ctas"] <= sms
        assert p["bt"] == next(b for b in (16, 32, 64, 128) if M <= b or b == 128)
        assert p["tiles"] == -(-N // 128) * -(-M // p["bt"])
        assert p["stages"] == -(-(K // 128) // (4 if p["bt"] <= 32 else 2))
        if p["split_k"] == 0:
            assert p["cluster"] == 1 and p["ctas"] == min(p["tiles"], sms)
        if p["cluster"] > 1:
            assert p["cluster"] <= {16: 4, 32: 2}[p["bt"]]
            assert p["ctas"] == p["cluster"] * p["tiles"]
            assert p["stages"] >= p["cluster"]       # every CTA of a cluster has work


def test_plan_argument_errors():
    with pytest.raises(apex.ApexError):
        apex.apex_debug_gemm_plan(16, 8192, 8192, 0)
    with pytest.raises(apex.ApexError):
        apex.apex_debug_gemm_plan(16, 8192, 100, SMS)
    with pytest.raises(apex.ApexError):
        apex.apex_debug_gemm_plan(0, 8192, 8192, SMS)
