"""Pins of the oracle's RAC steps: selection, special cases, products, and the
accuracy claim of the pages."""
import math

import numpy as np
import pytest

import oracle
from oracle import scalar
from oracle.nvfp4 import F32
from precision_rl_rollout_nvfp4_b200 import synthetic as S


@pytest.mark.parametrize("k,K,want", [(0, 2048, 0), (100, 2048, 2048), (50, 2048, 1024),
                                      (25, 2048, 512), (50, 11008, 5504), (12.5, 11008, 1376),
                                      (33.3, 1000, 332), (0.1, 1000, 1), (99.99, 64, 63)])
def test_n_selected(k, K, want):
    # 33.3 and 99.99 are not exact in fp32: floor of the exact value of the float
    assert oracle.n_selected(k, K) == want


def test_select_matches_rank_definition():
    """j is selected iff fewer than n_sel channels outrank it (higher score, or
    equal score and lower index) -- brute force O(K^2) on tiny K with ties."""
    rng = np.random.default_rng(7)
    for trial in range(40):
        K = int(rng.integers(1, 48))
        score = rng.integers(0, 6, K).astype(np.float64) * 0.25     # many ties
        n_sel = int(rng.integers(0, K + 1))
        sel, mask = oracle.select_channels(score, n_sel)
        for j in range(K):
            outrank = sum(1 for i in range(K) if score[i] > score[j] or (score[i] == score[j] and i < j))
            assert mask[j] == (outrank < n_sel)
        assert len(sel) == n_sel and np.all(np.diff(sel) > 0)
        assert np.array_equal(np.nonzero(mask)[0], sel)


def test_identical_channels_tie_to_lower_index():
    x = S.activations(40, 64, seed=2)
    xb = S.bf16_bits(x).copy()
    xb[:, 48:64] = xb[:, 0:16]       # block 3 repeats block 0: equal residuals
    qa = oracle.quantize_activations(xb)
    assert np.array_equal(qa["score"][48:64], qa["score"][0:16])
    order = np.lexsort((np.arange(64), -qa["score"]))
    pos10 = int(np.nonzero(order == 10)[0][0])
    assert order[pos10 + 1] == 58     # the twin comes right after, by index
    # choose n_sel so that exactly one of the pair fits
    sel, mask = oracle.select_channels(qa["score"], pos10 + 1)
    assert mask[10] == 1 and mask[58] == 0


def test_score_order_and_bound():
    x = S.activations(300, 32, seed=3)
    qa = oracle.quantize_activations(S.bf16_bits(x))
    a = np.abs(qa["dx"]).astype(np.float64)
    exact = np.array([math.fsum(a[:, j]) for j in range(32)])
    assert np.all(np.abs(qa["score"] - exact) <= 300 * 2.0 ** -52 * exact)
    assert np.array_equal(qa["res_colamax"], np.abs(qa["dx"]).max(axis=0))


def test_score_order_is_rows_then_chunks():
    """channel_score adds the rows of each 128-row chunk one by one in row
    order, then the chunk sums in chunk order, each addition rounded to the
    nearest fp64 (ties to even).  The columns below are built so that this
    order, a grouped order, a reversed order and the exactly rounded sum all
    give different fp64 results; the expected values follow from IEEE
    binary64 rounding alone (u = 2^-53 is half an ulp of 1.0):
      col 0: 1, then 127 x u           -> 1 + u is a tie, rounds to 1 each
                                          time: 1.0 (exact sum rounds to
                                          1 + 2^-46; groups of 4 give
                                          1 + 31 * 2^-51)
      col 1: 127 x u, then 1           -> 127 u is exact; 1 + 127 u =
                                          1 + 63.5 * 2^-52 ties to even:
                                          1 + 2^-46 (reversed order gives 1)
      col 2: 1 at row 0, u at rows 128 and 129
                                       -> chunk sums 1 and 2u = 2^-52:
                                          1 + 2^-52 (one sequential pass over
                                          all rows would give 1)
      col 3: 1, u, u in chunks 0, 1, 2  -> (1 + u) + u: 1.0 (adding the two
                                          small chunks first gives 1 + 2^-52)
    """
    u = 2.0 ** -53
    dx = np.zeros((3 * 128, 4), F32)
    dx[0, 0] = 1.0
    dx[1:128, 0] = u
    dx[0:127, 1] = u
    dx[127, 1] = 1.0
    dx[0, 2] = 1.0
    dx[128, 2] = u
    dx[129, 2] = u
    dx[0, 3] = 1.0
    dx[128, 3] = u
    dx[256, 3] = u
    score, colamax = oracle.channel_score(-dx)          # |dX|: the sign does not matter
    assert score[0] == 1.0
    assert score[1] == 1.0 + 2.0 ** -46
    assert score[2] == 1.0 + 2.0 ** -52
    assert score[3] == 1.0
    assert np.array_equal(colamax, np.array([1.0, 1.0, 1.0, 1.0], F32))
    # the other orders named above really differ on these columns
    assert math.fsum(dx[:, 0].astype(np.float64)) != score[0]
    assert math.fsum(dx[:, 1].astype(np.float64)) == 1.0 + 2.0 ** -46


def test_k0_is_plain_w4a4_and_k100_is_full_residual():
    x = S.activations(64, 128, seed=4)
    w = S.weights(96, 128, seed=4)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    r0 = oracle.rac_linear(xb, wb, 0.0)
    assert r0["n_sel"] == 0 and not r0["mask"].any()
    assert np.array_equal(r0["y"], r0["y_plain"])
    r100 = oracle.rac_linear(xb, wb, 100.0)
    assert np.array_equal(r100["sel"], np.arange(128))
    # W_sel == W, so its second-pass quantization equals Q(W) bit for bit
    assert np.array_equal(r100["ws_codes"], r100["wq"]["codes"])
    assert np.array_equal(r100["ws_scales"], r100["wq"]["scales"])
    assert r100["ws_st"] == r100["wq"]["s_t"]
    # dX_sel == dX, so Q(dX_sel) equals Q(dX) with dX's own tensor scale
    c, s, st = oracle.quantize_tensor(r100["dx"])
    assert np.array_equal(r100["r_codes"], c) and np.array_equal(r100["r_scales"], s)
    assert r100["r_st"] == st


def test_gemm_fp64_matches_plain_loop():
    rng = np.random.default_rng(9)
    M, N, K = 5, 7, 64
    ac = rng.integers(0, 16, (M, K)).astype(np.uint8)
    bc = rng.integers(0, 16, (N, K)).astype(np.uint8)
    asc = rng.integers(0, 0x7F, (M, K // 16)).astype(np.uint8)
    bsc = rng.integers(0, 0x7F, (N, K // 16)).astype(np.uint8)
    y = oracle.gemm_fp64(ac, asc, F32(0.75), bc, bsc, F32(1.5))
    for i in range(M):
        for j in range(N):
            acc = 0.0
            for k in range(K):
                acc += (oracle.e2m1_decode(ac[i, k]) * oracle.e4m3_decode(asc[i, k // 16])
                        * oracle.e2m1_decode(bc[j, k]) * oracle.e4m3_decode(bsc[j, k // 16]))
            assert abs(y[i, j] - 0.75 * 1.5 * acc) <= 1e-12 * max(1.0, abs(acc))


@pytest.mark.parametrize("M,K,N,k", [(5, 64, 3, 50.0), (9, 32, 4, 25.0), (130, 48, 2, 50.0),
                                     (3, 80, 2, 100.0), (4, 64, 2, 0.0)])
def test_scalar_restatement_agrees(M, K, N, k):
    x = S.activations(M, K, seed=M + K)
    w = S.weights(N, K, seed=N)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    r = oracle.rac_linear(xb, wb, k)
    s = scalar.rac_linear(xb.tolist(), wb.tolist(), k)
    assert np.array_equal(r["codes"], np.array(s["codes"], np.uint8))
    assert np.array_equal(r["scales"], np.array(s["scales"], np.uint8))
    assert np.array_equal(r["dx"], np.array(s["dx"], np.float32))
    assert np.array_equal(r["score"], np.array(s["score"]))
    assert r["sel"].tolist() == s["sel"]
    if r["n_sel"]:
        assert np.array_equal(r["r_codes"], np.array(s["r_codes"], np.uint8))
        assert np.array_equal(r["r_scales"], np.array(s["r_scales"], np.uint8))
        assert np.array_equal(r["ws_codes"], np.array(s["ws_codes"], np.uint8))
        assert r["r_st"] == s["r_st"] and r["ws_st"] == s["ws_st"]
    assert np.allclose(r["y"], np.array(s["y"]), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("M,K,N,seed", [(64, 512, 512, 0), (128, 256, 64, 1), (256, 1024, 128, 2)])
def test_rac_reduces_error_against_bf16_product(M, K, N, seed):
    """RAC brings the output closer to the BF16 reference (QUADS technical
    summary, section 2.2 B, "Doel"); removing it leaves an accuracy gap
    (section 4, ablation)."""
    x = S.activations(M, K, seed=seed)
    w = S.weights(N, K, seed=seed)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    ref = oracle.bf16_to_f32(xb).astype(np.float64) @ oracle.bf16_to_f32(wb).astype(np.float64).T
    wq = oracle.weight_qdq(wb)
    errs = {}
    for k in (0.0, 25.0, 50.0, 100.0):
        r = oracle.rac_linear(xb, wb, k, wq=wq)
        errs[k] = np.linalg.norm(r["y"] - ref)
    assert errs[50.0] <= errs[0.0]
    assert errs[100.0] <= errs[0.0]


def test_weight_qdq_on_grid_and_colamax():
    w = S.weights(64, 256, seed=5)
    wb = S.bf16_bits(w)
    q = oracle.weight_qdq(wb)
    dq = oracle.dequantize(q["codes"], q["scales"], q["s_t"])
    assert np.array_equal(q["w_out"], oracle.f32_to_bf16(dq))
    wf = oracle.bf16_to_f32(wb)
    assert np.array_equal(q["colamax"], np.abs(wf).max(axis=0))
    # fake quantization moves every weight by at most one grid half-gap
    s_dec = np.repeat(oracle.e4m3_decode(q["scales"]) * float(q["s_t"]), 16, axis=1)
    assert np.all(np.abs(oracle.bf16_to_f32(q["w_out"]) - wf) <= s_dec * 1.01 + 1e-30)


def test_moe_groups_are_independent_linears():
    rng = np.random.default_rng(1)
    E, N, K = 4, 32, 64
    counts = [70, 0, 130, 5]
    off = np.concatenate([[0], np.cumsum(counts)])
    x = S.activations(int(off[-1]), K, seed=6)
    w = S.weights(N, K, seed=6, batch=E)
    xb = S.bf16_bits(x)
    wb = S.bf16_bits(w).reshape(E, N, K)
    y, masks, per = oracle.moe_rac(xb, off, wb, 50.0)
    for e in range(E):
        if counts[e] == 0:
            assert masks[e].tolist() == [1] * 32 + [0] * 32
            continue
        r = oracle.rac_linear(xb[off[e]:off[e + 1]], wb[e], 50.0)
        assert np.array_equal(y[off[e]:off[e + 1]], r["y"])
        assert np.array_equal(masks[e], r["mask"])


@pytest.mark.parametrize("M,K,N,k", [(5, 64, 3, 50.0), (9, 32, 4, 25.0), (3, 80, 2, 100.0)])
def test_wsel_from_fp4_scalar_restatement_agrees(M, K, N, k):
    """The W_sel variant from Q(W) against the independent scalar
    restatement (codes, scales, tensor scale and Y)."""
    x = S.activations(M, K, seed=M + 2 * K)
    w = S.weights(N, K, seed=N + 7)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    r = oracle.rac_linear(xb, wb, k, wsel_source="fp4")
    s = scalar.rac_linear(xb.tolist(), wb.tolist(), k, wsel_source="fp4")
    assert np.array_equal(r["ws_codes"], np.array(s["ws_codes"], np.uint8))
    assert np.array_equal(r["ws_scales"], np.array(s["ws_scales"], np.uint8))
    assert r["ws_st"] == s["ws_st"]
    assert np.allclose(r["y"], np.array(s["y"]), rtol=1e-12, atol=1e-14)


def test_wsel_from_fp4_equals_bf16_source_on_grid_weights():
    """Weights already on the NVFP4 grid (W = DQ(Q(W0)), tensor scale a power
    of two so every value is exact in bf16) quantize back to themselves
    (Q(DQ(Q(w))) = Q(w)), so both sources of W_sel agree exactly."""
    rng = np.random.default_rng(11)
    N, K = 48, 256
    w0 = rng.standard_normal((N, K)).astype(np.float32) * 0.05
    amax = np.float32(2688.0 * 2.0 ** -10)                 # s_t = 2^-10 exactly
    w0[3, 7] = amax
    w0 = np.clip(w0, -amax, amax)
    c0, s0, st0 = oracle.quantize_tensor(w0)
    assert st0 == np.float32(2.0 ** -10)
    dq = oracle.dequantize(c0, s0, st0)
    wb = oracle.f32_to_bf16(dq)
    assert np.array_equal(oracle.bf16_to_f32(wb), dq)       # exact in bf16
    wq = oracle.weight_qdq(wb)
    assert np.array_equal(wq["codes"], c0) and np.array_equal(wq["scales"], s0)
    sel = np.sort(rng.choice(K, 100, replace=False)).astype(np.int32)
    width = oracle.padded_width(len(sel))
    a = oracle.weight_sel_from_fp4(wq["codes"], wq["scales"], wq["s_t"], sel, width)
    b = oracle.gather_quantize(oracle.bf16_to_f32(wb), sel, width, wq["colamax"][sel].max())
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_wsel_from_fp4_k0_is_plain_and_error_is_bounded():
    x = S.activations(32, 128, seed=4)
    w = S.weights(16, 128, seed=4)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    r0 = oracle.rac_linear(xb, wb, 0.0, wsel_source="fp4")
    assert np.array_equal(r0["y"], r0["y_plain"])
    # the FP4-sourced correction still reduces the error against bf16
    ref = oracle.bf16_to_f32(xb).astype(np.float64) @ oracle.bf16_to_f32(wb).astype(np.float64).T
    r50 = oracle.rac_linear(xb, wb, 50.0, wsel_source="fp4")
    assert np.linalg.norm(r50["y"] - ref) <= np.linalg.norm(r0["y"] - ref)


def test_reused_mask_equal_to_this_calls_mask_changes_nothing():
    """The mask-reuse variant with the selection this X would make itself is
    the per-call RAC linear, intermediate for intermediate."""
    x = S.bf16_bits(S.activations(96, 256, seed=21))
    w = S.bf16_bits(S.weights(64, 256, seed=21))
    a = oracle.rac_linear(x, w, 50.0)
    b = oracle.rac_linear(x, w, 50.0, sel=a["sel"])
    for key in ("mask", "sel", "r_codes", "r_scales", "ws_codes", "ws_scales"):
        assert np.array_equal(a[key], b[key]), key
    assert a["r_st"] == b["r_st"] and a["ws_st"] == b["ws_st"]
    assert np.array_equal(a["y"], b["y"])


def test_reused_mask_from_another_batch():
    """A mask kept from batch A applied to batch B: B's own residual (its
    tensor scale is the maximum over the kept channels of B's residual
    maxima), A's channels, and the plain W4A4 product when the mask is empty."""
    xa = S.bf16_bits(S.activations(64, 256, seed=22))
    xb = S.bf16_bits(S.activations(64, 256, seed=23))
    w = S.bf16_bits(S.weights(32, 256, seed=22))
    sel_a = oracle.rac_linear(xa, w, 25.0)["sel"]
    r = oracle.rac_linear(xb, w, 25.0, sel=sel_a)
    own = oracle.quantize_activations(xb)
    assert np.array_equal(r["sel"], sel_a)
    assert r["r_st"] == oracle.tensor_scale(own["res_colamax"][sel_a].max())
    codes, scales, st = oracle.gather_quantize(own["dx"], sel_a, r["width"], own["res_colamax"][sel_a].max())
    assert np.array_equal(r["r_codes"], codes) and np.array_equal(r["r_scales"], scales)
    empty = oracle.rac_linear(xb, w, 25.0, sel=np.zeros(0, np.int32))
    assert np.array_equal(empty["y"], empty["y_plain"])
    # the kept mask is not this batch's own choice, and RAC with it still helps
    assert not np.array_equal(sel_a, oracle.rac_linear(xb, w, 25.0)["sel"])
    ref = oracle.bf16_to_f32(xb).astype(np.float64) @ oracle.bf16_to_f32(w).astype(np.float64).T
    assert np.linalg.norm(r["y"] - ref) <= np.linalg.norm(r["y_plain"] - ref)
