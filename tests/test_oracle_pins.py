"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test checks the oracle against something the pages or the mathematics fix:
hand-worked fixtures (tests/golden), closed forms, brute-force enumeration on
tiny inputs, finite differences, special cases that reduce to a library
routine, and invariants.  They are chosen so that a dropped term, a wrong sign
or index, or a transposed operand in the oracle fails one of them.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import floats, ints, read_golden
from top_expert_selection_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore")


def _bf16_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------- dtype conversions


def test_bf16_conversions_match_torch_rne():
    g = torch.Generator().manual_seed(123)
    x = torch.randn(4000, generator=g) * 10.0
    # exact ties: fp32 values whose low 16 bits are 0x8000 (odd and even upper halves)
    ties = torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 3.0 + 2 ** -7], dtype=torch.float32)
    x = torch.cat([x, ties, torch.tensor([0.0, -0.0, 1e-40, 3.4e38])])
    ref = _bf16_bits(x.to(torch.bfloat16))
    got = oracle.f32_to_bf16(x.numpy())
    assert np.array_equal(got, ref)
    back = oracle.bf16_to_f32(ref)
    assert np.array_equal(back, x.to(torch.bfloat16).to(torch.float32).numpy())


def _exact_bf16_round(y: float) -> int:
    """Brute force: the bf16 value nearest to y (ties to even mantissa), by exact rationals."""
    f = np.float32(y)
    base = int(np.array(f, np.float32).view(np.uint32)) >> 16
    best = None
    for cand in range(max(base - 2, 0), base + 3):
        v = Fraction(float(np.array(cand << 16, np.uint32).view(np.float32)))
        d = abs(v - Fraction(y))
        key = (d, cand & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return best[1]


def test_f64_to_bf16_single_rounding_brute_force():
    rng = np.random.default_rng(5)
    ys = list(rng.uniform(0.5, 64.0, 300))
    # values just above / below bf16 ties, where rounding via fp32 would round twice
    for base in (1.0, 11.3125, 100.0):
        ulp = 2.0 ** (math.floor(math.log2(base)) - 7)
        for off in (0.5, 0.5 + 2 ** -30, 0.5 - 2 ** -30, 0.25, 0.75):
            ys.append(base + off * ulp)
    for y in ys:
        assert int(oracle.f64_to_bf16(np.array([y]))[0]) == _exact_bf16_round(float(y)), y


# --------------------------------------------------------------------------- bookkeeping


@pytest.mark.parametrize("case", read_golden("bookkeeping_handworked.txt"), ids=lambda c: c["case"])
def test_bookkeeping_handworked(case):
    ids = np.array([ints(r) for r in case["ids"].split("|")], np.int32)
    out = oracle.route_bookkeeping(ids, int(case["E"]), int(case["tile"]), int(case.get("local_offset", 0)),
                                   int(case["local_num"]) if "local_num" in case else None)
    for key in ("counts", "offsets", "e2p", "p2t", "tile_expert", "tile_mn_limit", "totals"):
        assert out[key].tolist() == ints(case[key]), key


@pytest.mark.parametrize("tile", [1, 4, 128])
@pytest.mark.parametrize("shards", [[(0, 4), (4, 4), (8, 4), (12, 4)], [(0, 5), (5, 6), (11, 5)], [(3, 1)]])
def test_bookkeeping_shards_match_the_global_bookkeeping(tile, shards):
    # an expert-parallel shard's bookkeeping is the global bookkeeping restricted to its experts
    # and shifted by the global offset of its first expert (slots, token map, tiles)
    rng = np.random.default_rng(tile + len(shards))
    T, E, k = 203, 16, 3
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    g = oracle.route_bookkeeping(ids, E, tile)
    owned = np.zeros(T * k, np.int32)
    for off, nl in shards:
        s = oracle.route_bookkeeping(ids, E, tile, off, nl)
        base = int(g["offsets"][off])
        assert np.array_equal(s["counts"], g["counts"][off:off + nl])
        assert np.array_equal(s["offsets"], g["offsets"][off:off + nl + 1] - base)
        loc = (ids.ravel() >= off) & (ids.ravel() < off + nl)
        owned += loc
        assert np.all(s["e2p"][~loc] == -1)
        assert np.array_equal(s["e2p"][loc], g["e2p"][loc] - base)
        P = int(s["totals"][0])
        assert P == int(g["offsets"][off + nl]) - base
        assert np.array_equal(s["p2t"], g["p2t"][base:base + P])
        t0, t1 = base // tile, (base + P) // tile
        assert np.array_equal(s["tile_expert"] + off, g["tile_expert"][t0:t1])
        assert np.array_equal(s["tile_mn_limit"], g["tile_mn_limit"][t0:t1] - base)
    if sum(nl for _, nl in shards) == E:
        assert np.all(owned == 1)  # every selection has exactly one owning shard


def _check_bookkeeping_invariants(ids, E, tile, bk):
    T, k = ids.shape
    counts, offsets, e2p, p2t = bk["counts"], bk["offsets"], bk["e2p"], bk["p2t"]
    P, ntiles = int(bk["totals"][0]), int(bk["totals"][1])
    assert counts.sum() == T * k
    assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
    assert offsets[0] == 0 and np.all(offsets % tile == 0) and offsets[-1] == P and P % tile == 0
    assert np.all(np.diff(offsets) >= counts) and np.all(np.diff(offsets) - counts < tile)
    assert ntiles == P // tile
    assert P <= bk["max_padded"] and ntiles <= bk["max_tiles"]
    # e2p is a bijection onto the non-padding slots, and p2t inverts it
    assert len(set(e2p.tolist())) == T * k
    filled = np.zeros(P, bool)
    filled[e2p] = True
    assert np.array_equal(filled, p2t >= 0)
    tok = np.repeat(np.arange(T), k)
    assert np.array_equal(p2t[e2p], tok)
    # the trtllm identity: the expert of slot p is the expert of tile p // tile
    assert np.array_equal(bk["tile_expert"][e2p // tile], ids.ravel())
    # slots of one expert follow token order
    for e in range(E):
        sl = e2p[ids.ravel() == e]
        assert np.all(np.diff(sl) == 1) and (sl.size == 0 or sl[0] == offsets[e])
    # each tile's limit is its last valid row + 1
    for c in range(ntiles):
        e = bk["tile_expert"][c]
        assert offsets[e] <= c * tile < offsets[e + 1]
        assert bk["tile_mn_limit"][c] == min((c + 1) * tile, offsets[e] + counts[e])


@pytest.mark.parametrize("tile", [1, 4, 8, 128])
def test_bookkeeping_invariants_random(tile):
    rng = np.random.default_rng(tile)
    T, E, k = 301, 16, 3
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    _check_bookkeeping_invariants(ids, E, tile, oracle.route_bookkeeping(ids, E, tile))


def test_bookkeeping_skewed_and_empty_experts():
    # one hot expert taking more than half the rows, several experts with no rows
    T, E, k = 257, 12, 2
    ids = np.zeros((T, k), np.int32)
    ids[:, 0] = 5
    ids[:, 1] = np.where(np.arange(T) % 3 == 0, 0, 9)
    bk = oracle.route_bookkeeping(ids, E, 8)
    _check_bookkeeping_invariants(ids, E, 8, bk)
    assert bk["counts"][5] == T and bk["counts"][1] == 0


def test_bookkeeping_rejects_non_power_of_two_tile():
    with pytest.raises(ValueError):
        oracle.route_bookkeeping(np.zeros((2, 1), np.int32), 2, 6)


# --------------------------------------------------------------------------- selection


@pytest.mark.parametrize("case", read_golden("selection_handworked.txt"), ids=lambda c: c["case"])
def test_selection_handworked(case):
    lg = np.array([floats(case["logits"])], np.float32)
    n_group = int(case["n_group"])
    out = oracle.route_select(lg, k=int(case["k"]), score_fn=W.SOFTMAX, softmax_before_topk=int(case["pre"]),
                              n_group=n_group, topk_group=int(case["topk_group"]), renormalize=1)
    assert out["ids"][0].tolist() == ints(case["ids"])
    if "group_scores" in case:
        assert out["group_scores"][0, :n_group].tolist() == floats(case["group_scores"])


def test_all_equal_logits_tie_break_and_weights():
    for k in (1, 2, 3, 8):
        for score_fn, pre in ((W.SOFTMAX, 1), (W.SOFTMAX, 0), (W.SIGMOID, 1)):
            lg = np.full((3, 16), 0.75, np.float32)
            out = oracle.route_select(lg, k=k, score_fn=score_fn, softmax_before_topk=pre, renormalize=1,
                                      scaling_factor=2.5)
            assert out["ids"].tolist() == [list(range(k))] * 3
            np.testing.assert_allclose(out["weights"], 2.5 / k, rtol=2e-7)


def test_te_usage_example_equals_plain_pre_softmax_top2():
    """TransformerEngine Fused Router, Usage Examples: topk=2, pre-softmax, num_groups=1,
    group_topk=0, scaling 1.0, softmax, zero expert bias == plain softmax + top-2."""
    g = torch.Generator().manual_seed(7)
    lg = torch.randn(64, 16, generator=g).numpy()
    out = oracle.route_select(lg, k=2, score_fn=W.SOFTMAX, softmax_before_topk=1, n_group=1, topk_group=0,
                              renormalize=0, scaling_factor=1.0, bias=np.zeros(16, np.float32))
    p = torch.softmax(torch.from_numpy(lg).double(), dim=-1).numpy()
    order = np.argsort(-p, axis=1, kind="stable")[:, :2]
    assert np.array_equal(out["ids"], order)
    np.testing.assert_allclose(out["weights"], np.take_along_axis(p, order, 1), rtol=2e-6)


def test_keys_match_float64_definitions():
    g = torch.Generator().manual_seed(11)
    lg = (torch.randn(32, 64, generator=g) * 2).numpy()
    b = (torch.rand(64, generator=g) * 0.2 - 0.1).numpy()
    sm = oracle.route_select(lg, k=4, score_fn=W.SOFTMAX, softmax_before_topk=1)
    ref = torch.softmax(torch.from_numpy(lg).double(), -1).numpy()
    np.testing.assert_allclose(sm["keys"], ref, rtol=2e-6, atol=0)
    sg = oracle.route_select(lg, k=4, score_fn=W.SIGMOID, bias=b)
    ref = 1.0 / (1.0 + np.exp(-lg.astype(np.float64))) + b.astype(np.float64)
    np.testing.assert_allclose(sg["keys"], ref, rtol=0, atol=3e-7)


def test_bias_selects_but_does_not_weight():
    """max.nn.moe.SigmoidTopKRouter steps 3-4: select on score + bias, weight by the unbiased score."""
    lg = np.array([[0.0, 2.0, -2.0, 1.0]], np.float32)
    bias = np.array([0.0, 0.0, 10.0, 0.0], np.float32)
    out = oracle.route_select(lg, k=1, score_fn=W.SIGMOID, renormalize=0, scaling_factor=1.0, bias=bias)
    assert out["ids"].tolist() == [[2]]
    assert abs(out["weights"][0, 0] - 1.0 / (1.0 + math.exp(2.0))) < 1e-7
    out = oracle.route_select(lg, k=2, score_fn=W.SIGMOID, renormalize=0, scaling_factor=3.0, bias=bias)
    assert out["ids"].tolist() == [[2, 1]]
    np.testing.assert_allclose(out["weights"][0], [3.0 / (1 + math.exp(2.0)), 3.0 / (1 + math.exp(-2.0))],
                               rtol=1e-6)


def test_post_softmax_closed_form():
    """Top-k on logits then softmax over the selected: logits (a, a + ln 3) -> weights (1/4, 3/4)."""
    a = 0.3
    lg = np.array([[a, -5.0, a + math.log(3.0), -4.0]], np.float32)
    out = oracle.route_select(lg, k=2, score_fn=W.SOFTMAX, softmax_before_topk=0, renormalize=0)
    assert out["ids"].tolist() == [[2, 0]]
    np.testing.assert_allclose(out["weights"][0], [0.75, 0.25], rtol=1e-6)
    # sigmoid renormalised with equal selected scores -> 1/k * scale
    lg = np.array([[1.5, 1.5, -3.0, 1.5]], np.float32)
    out = oracle.route_select(lg, k=3, score_fn=W.SIGMOID, renormalize=1, scaling_factor=2.0)
    np.testing.assert_allclose(out["weights"][0], [2.0 / 3] * 3, rtol=1e-6)


def test_renormalized_weights_sum_to_scale():
    g = torch.Generator().manual_seed(3)
    lg = (torch.randn(200, 64, generator=g) * 2).numpy()
    for score_fn in (W.SOFTMAX, W.SIGMOID):
        out = oracle.route_select(lg, k=6, score_fn=score_fn, renormalize=1, scaling_factor=2.5)
        np.testing.assert_allclose(out["weights"].astype(np.float64).sum(1), 2.5, rtol=3e-6)
        assert all(len(set(r)) == 6 for r in out["ids"].tolist())


def _best_subset(values, m):
    """Brute force: the m-subset with the largest exact sum; ties -> lexicographically smallest indices."""
    best = None
    for sub in itertools.combinations(range(len(values)), m):
        s = sum(Fraction(float(values[i])) for i in sub)
        key = (-s, sub)
        if best is None or key < best[0]:
            best = (key, sub)
    return set(best[1])


@pytest.mark.parametrize("E,n_group,topk_group,k,score_fn", [
    (16, 4, 2, 3, W.SIGMOID), (16, 8, 3, 4, W.SIGMOID), (12, 3, 2, 2, W.SOFTMAX), (16, 1, 0, 4, W.SOFTMAX),
    (8, 4, 4, 3, W.SIGMOID)])
def test_grouped_selection_brute_force(E, n_group, topk_group, k, score_fn):
    """Enumerate every group subset and every expert subset for E <= 16."""
    g = torch.Generator().manual_seed(E * 100 + k)
    lg = (torch.randn(40, E, generator=g) * 2).to(torch.bfloat16)
    bias = (torch.rand(E, generator=g) * 0.2 - 0.1)
    # include exact ties: duplicate a column
    lg[:, 1] = lg[:, 0]
    out = oracle.route_select(lg, k=k, score_fn=score_fn, n_group=n_group, topk_group=topk_group,
                              bias=bias if score_fn == W.SIGMOID else None)
    keys = out["keys"]
    grouped = n_group > 1 and topk_group > 0
    for t in range(lg.shape[0]):
        if grouped:
            gs = E // n_group
            gscore = []
            for gi in range(n_group):
                top2 = sorted(keys[t, gi * gs:(gi + 1) * gs].tolist(), reverse=True)[:2]
                gscore.append(np.float32(top2[0]) + np.float32(top2[1]))
            kept = _best_subset(gscore, min(topk_group, n_group))
            assert set(np.nonzero(out["group_kept"][t])[0].tolist()) == kept
            cand = [e for e in range(E) if e // gs in kept]
        else:
            cand = list(range(E))
        best = _best_subset([keys[t, e] for e in cand], k)
        assert set(out["ids"][t].tolist()) == {cand[i] for i in best}
        sel = out["ids"][t]
        for a, b in zip(sel[:-1], sel[1:]):
            assert keys[t, a] > keys[t, b] or (keys[t, a] == keys[t, b] and a < b)


def test_grouped_all_kept_equals_ungrouped():
    spec = W.DSV3_GROUPED_SIGMOID.with_(T=256)
    inp = W.route_inputs(spec)
    base = dict(k=8, score_fn=W.SIGMOID, renormalize=1, scaling_factor=2.5, bias=inp["bias"])
    a = oracle.route_select(inp["logits"], n_group=8, topk_group=8, **base)
    b = oracle.route_select(inp["logits"], n_group=0, topk_group=0, **base)
    assert np.array_equal(a["ids"], b["ids"]) and np.array_equal(a["weights"], b["weights"])


def test_grouped_workload_invariants():
    spec = W.DSV3_GROUPED_SIGMOID.with_(T=512)
    inp = W.route_inputs(spec)
    out = oracle.route_select(inp["logits"], k=8, score_fn=W.SIGMOID, n_group=8, topk_group=4,
                              renormalize=1, scaling_factor=2.5, bias=inp["bias"])
    ids = out["ids"]
    assert all(len(set(r)) == 8 for r in ids.tolist())
    # every selected expert lies in a kept group, exactly 4 groups kept
    assert np.all(out["group_kept"].sum(1) == 4)
    assert np.all(np.take_along_axis(out["group_kept"], ids // 32, 1) == 1)
    np.testing.assert_allclose(out["weights"].astype(np.float64).sum(1), 2.5, rtol=3e-6)
    bk = oracle.route_bookkeeping(ids, 256, 128)
    _check_bookkeeping_invariants(ids, 256, 128, bk)


# --------------------------------------------------------------------------- aux loss


def test_aux_uniform_closed_form():
    T, E, k, coeff = 512, 128, 8, 1e-2
    lg = np.zeros((T, E), np.float32)
    sc = oracle.aux_scores(lg, k)
    assert np.all(sc["probs"] == np.float32(1.0 / E))
    assert np.all(sc["routing_map"][:, :k] == 1) and np.all(sc["routing_map"][:, k:] == 0)
    assert sc["tokens_per_expert"].tolist() == [T] * k + [0] * (E - k)
    L = oracle.aux_loss_fwd(sc["probs"], sc["tokens_per_expert"], T, k, coeff)
    assert abs(L - coeff * T) <= 1e-6 * coeff * T
    # T_total differs from the rows given: L = coeff * T_rows^2 / T_total
    L2 = oracle.aux_loss_fwd(sc["probs"], sc["tokens_per_expert"], 4 * T, k, coeff)
    assert abs(L2 - coeff * T / 4) <= 1e-6 * coeff * T
    C = coeff * E / (T * k)
    gr = oracle.aux_loss_bwd(sc["probs"], sc["tokens_per_expert"], T, k, coeff, 1.0)
    exp = np.where(np.arange(E) < k, (C / E) * (T - k * T / E), -(C / E) * (k * T / E))
    np.testing.assert_allclose(gr["grad_logits"], np.broadcast_to(exp, (T, E)), rtol=1e-6)
    np.testing.assert_allclose(gr["grad_probs"], np.broadcast_to(C * sc["tokens_per_expert"], (T, E)), rtol=1e-7)
    assert np.abs(gr["grad_logits"].astype(np.float64).sum(1)).max() < 1e-9


def test_aux_one_hot_probs_closed_form():
    """Logits far apart make the fp32 softmax exactly one-hot; the loss is C * sum_t tpe[e(t)]."""
    T, E, k, coeff = 64, 16, 1, 0.5
    lg = np.full((T, E), -200.0, np.float32)
    e_of_t = (np.arange(T) * 7) % E
    lg[np.arange(T), e_of_t] = 0.0
    sc = oracle.aux_scores(lg, k)
    assert np.array_equal(sc["probs"], np.eye(E, dtype=np.float32)[e_of_t])
    tpe = np.arange(E, dtype=np.int32) * 3 + 1  # arbitrary constants (tpe is an input)
    L = oracle.aux_loss_fwd(sc["probs"], tpe, T, k, coeff)
    C = coeff * E / (T * k)
    assert abs(L - C * tpe[e_of_t].sum()) <= 1e-6 * abs(L)


def test_aux_backward_finite_differences():
    """grad_logits is d/dlogits of coeff*E/(T*k) * sum_t sum_e softmax(l_t)_e * tpe_e (tpe fixed)."""
    T, E, k, coeff = 6, 10, 3, 0.7
    rng = np.random.default_rng(0)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    sc = oracle.aux_scores(lg, k)
    tpe = sc["tokens_per_expert"]
    gr = oracle.aux_loss_bwd(sc["probs"], tpe, T, k, coeff, 1.7)

    def loss64(x):
        z = np.exp(x - x.max(1, keepdims=True))
        p = z / z.sum(1, keepdims=True)
        return 1.7 * coeff * E / (T * k) * float((p.sum(0) * tpe).sum())

    x0 = lg.astype(np.float64)
    h = 1e-6
    fd = np.zeros_like(x0)
    for t in range(T):
        for e in range(E):
            xp = x0.copy(); xp[t, e] += h
            xm = x0.copy(); xm[t, e] -= h
            fd[t, e] = (loss64(xp) - loss64(xm)) / (2 * h)
    np.testing.assert_allclose(gr["grad_logits"], fd, rtol=2e-5, atol=1e-7)


def test_aux_scores_backward_finite_differences():
    """aux_scores_bwd is the vector-Jacobian product of the softmax scores: for a fixed upstream
    gradient G, grad_logits = d/dlogits of sum_t sum_e softmax(l_t)_e * G[t,e] (central differences of a
    float64 softmax)."""
    T, E = 5, 12
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    G = rng.standard_normal((T, E)).astype(np.float32)
    probs = oracle.aux_scores(lg, 2)["probs"]
    gl = oracle.aux_scores_bwd(probs, G)

    def f64(x):
        z = np.exp(x - x.max(1, keepdims=True))
        return float(((z / z.sum(1, keepdims=True)) * G.astype(np.float64)).sum())

    x0 = lg.astype(np.float64)
    h = 1e-6
    fd = np.zeros_like(x0)
    for t in range(T):
        for e in range(E):
            xp = x0.copy(); xp[t, e] += h
            xm = x0.copy(); xm[t, e] -= h
            fd[t, e] = (f64(xp) - f64(xm)) / (2 * h)
    np.testing.assert_allclose(gl, fd, rtol=2e-5, atol=2e-7)


@pytest.mark.parametrize("score_fn,pre,renorm", [(W.SIGMOID, 1, 1), (W.SIGMOID, 1, 0), (W.SOFTMAX, 1, 1),
                                                 (W.SOFTMAX, 1, 0), (W.SOFTMAX, 0, 1), (W.SOFTMAX, 0, 0)])
def test_route_weights_backward_finite_differences(score_fn, pre, renorm):
    """route_weights_bwd is d/dlogits of sum_t sum_j G[t,j] * w[t,j] for a fixed selection, where the
    weights follow the forward's definition (score of the selected, optional renorm, times the scale);
    central differences of a float64 forward written here from that definition."""
    T, E, k, scale = 4, 10, 3, 2.5
    rng = np.random.default_rng(11 + score_fn + 2 * pre + 4 * renorm)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    G = rng.standard_normal((T, k)).astype(np.float32)
    got = oracle.route_weights_bwd(lg, ids, G, score_fn=score_fn, softmax_before_topk=pre, renormalize=renorm,
                                   scaling_factor=scale)

    def f64(x):
        tot = 0.0
        for t in range(T):
            if score_fn == W.SIGMOID:
                v = 1.0 / (1.0 + np.exp(-x[t, ids[t]]))
            elif pre:
                z = np.exp(x[t] - x[t].max())
                v = (z / z.sum())[ids[t]]
            else:
                z = np.exp(x[t, ids[t]] - x[t, ids[t]].max())
                v = z / z.sum()
            w = scale * v / v.sum() if renorm else scale * v
            tot += float((G[t].astype(np.float64) * w).sum())
        return tot

    x0 = lg.astype(np.float64)
    h = 1e-6
    fd = np.zeros_like(x0)
    for t in range(T):
        for e in range(E):
            xp = x0.copy(); xp[t, e] += h
            xm = x0.copy(); xm[t, e] -= h
            fd[t, e] = (f64(xp) - f64(xm)) / (2 * h)
    np.testing.assert_allclose(got, fd, rtol=2e-5, atol=2e-7)


def test_route_weights_backward_zero_off_selection():
    """Sigmoid and post-softmax weights depend only on the selected logits: the gradient is zero
    elsewhere; renormalised post-softmax weights are the softmax itself (sum 1), so renorm changes nothing."""
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((3, 8)).astype(np.float32)
    ids = np.array([[1, 5], [0, 7], [6, 2]], np.int32)
    G = rng.standard_normal((3, 2)).astype(np.float32)
    for sf, pre in ((W.SIGMOID, 1), (W.SOFTMAX, 0)):
        g = oracle.route_weights_bwd(lg, ids, G, score_fn=sf, softmax_before_topk=pre, renormalize=0)
        mask = np.zeros_like(g, dtype=bool)
        np.put_along_axis(mask, ids.astype(np.int64), True, axis=1)
        assert np.all(g[~mask] == 0)
    a = oracle.route_weights_bwd(lg, ids, G, score_fn=W.SOFTMAX, softmax_before_topk=0, renormalize=1)
    b = oracle.route_weights_bwd(lg, ids, G, score_fn=W.SOFTMAX, softmax_before_topk=0, renormalize=0)
    np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-9)


def test_aux_scores_backward_special_cases():
    """A constant upstream gradient moves no logit (softmax is shift-invariant); a one-hot upstream
    gradient on expert j gives p_j * (1 - p_j) at j; sigmoid scores are refused."""
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((4, 9)).astype(np.float32)
    probs = oracle.aux_scores(lg, 2)["probs"]
    z = oracle.aux_scores_bwd(probs, np.full_like(probs, 2.5))
    assert np.all(np.abs(z) <= 1e-6 * probs)
    onehot = np.zeros_like(probs)
    onehot[:, 3] = 1.0
    g1 = oracle.aux_scores_bwd(probs, onehot)
    np.testing.assert_allclose(g1[:, 3], probs[:, 3].astype(np.float64) * (1 - probs[:, 3]), rtol=1e-6)
    with pytest.raises(ValueError):
        oracle.aux_scores_bwd(probs, onehot, score_fn=W.SIGMOID)


@pytest.mark.parametrize("score_fn", [W.SOFTMAX, W.SIGMOID])
def test_aux_scores_backward_from_logits_finite_differences(score_fn):
    """aux_scores_bwd_logits is d/dlogits of sum_t sum_e p(l_t)_e * G[t,e], with p the softmax or the
    sigmoids over their row sum (central differences of a float64 forward written here from that
    definition)."""
    T, E = 4, 11
    rng = np.random.default_rng(21 + score_fn)
    lg = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    G = rng.standard_normal((T, E)).astype(np.float32)
    gl = oracle.aux_scores_bwd_logits(lg, G, score_fn=score_fn)

    def f64(x):
        if score_fn == W.SOFTMAX:
            z = np.exp(x - x.max(1, keepdims=True))
        else:
            z = 1.0 / (1.0 + np.exp(-x))
        return float(((z / z.sum(1, keepdims=True)) * G.astype(np.float64)).sum())

    x0 = lg.astype(np.float64)
    h = 1e-6
    fd = np.zeros_like(x0)
    for t in range(T):
        for e in range(E):
            xp = x0.copy(); xp[t, e] += h
            xm = x0.copy(); xm[t, e] -= h
            fd[t, e] = (f64(xp) - f64(xm)) / (2 * h)
    np.testing.assert_allclose(gl, fd, rtol=2e-5, atol=2e-7)


def test_aux_scores_backward_from_logits_special_cases():
    """Normalised scores sum to 1 for any logits, so a constant upstream gradient moves no logit and a
    single expert (E = 1) has no gradient; for softmax, the entry that recomputes the scores agrees with
    the one given the probs; saturated sigmoids (|x| = 30) leave finite gradients."""
    rng = np.random.default_rng(6)
    lg = rng.standard_normal((5, 10)).astype(np.float32)
    for sf in (W.SOFTMAX, W.SIGMOID):
        z = oracle.aux_scores_bwd_logits(lg, np.full_like(lg, -1.75), score_fn=sf)
        assert np.all(np.abs(z) <= 1e-7)
        one = oracle.aux_scores_bwd_logits(lg[:, :1].copy(), rng.standard_normal((5, 1)).astype(np.float32), sf)
        assert np.all(one == 0)
    G = rng.standard_normal(lg.shape).astype(np.float32)
    a = oracle.aux_scores_bwd_logits(lg, G, score_fn=W.SOFTMAX)
    b = oracle.aux_scores_bwd(oracle.aux_scores(lg, 2)["probs"], G)
    np.testing.assert_allclose(a, b, rtol=1e-5, atol=1e-7)
    sat = np.array([[30.0, -30.0, 0.0, 30.0]], np.float32)
    g = oracle.aux_scores_bwd_logits(sat, np.array([[1.0, 2.0, 3.0, 4.0]], np.float32), score_fn=W.SIGMOID)
    assert np.all(np.isfinite(g)) and abs(g[0, 1]) < 1e-12 and g[0, 2] != 0


def test_aux_sigmoid_scores_closed_forms():
    E = 8
    sc = oracle.aux_scores(np.zeros((2, E), np.float32), 2, score_fn=W.SIGMOID)
    assert np.all(sc["probs"] == np.float32(1.0 / E))
    lg = np.full((1, E), -200.0, np.float32)
    lg[0, 3] = 1.0
    sc = oracle.aux_scores(lg, 1, score_fn=W.SIGMOID)
    assert sc["probs"][0].tolist() == [0, 0, 0, 1.0, 0, 0, 0, 0]
    # exact sigmoids 1/2, 1, 0, 1/2 (saturated at +-100) normalise to 1/4, 1/2, 0, 1/4; the top-2
    # map takes expert 1, then expert 0 of the tied 1/4s (lower index)
    sc = oracle.aux_scores(np.array([[0.0, 100.0, -100.0, 0.0]], np.float32), 2, score_fn=W.SIGMOID)
    assert sc["probs"][0].tolist() == [0.25, 0.5, 0.0, 0.25]
    assert sc["routing_map"][0].tolist() == [1, 1, 0, 0]
    assert sc["tokens_per_expert"].tolist() == [1, 1, 0, 0]


# --------------------------------------------------------------------------- dispatch / combine


def test_dispatch_handworked():
    hidden = np.array([[1, 2, 3], [4, 5, 6]], np.uint16)
    ids = np.array([[1, 0], [1, 2]], np.int32)
    bk = oracle.route_bookkeeping(ids, 3, 2)  # counts [1,2,1] -> offsets [0,2,4,6]
    assert bk["e2p"].tolist() == [2, 0, 3, 4]
    out = oracle.dispatch(hidden, bk["e2p"], bk["p2t"], int(bk["totals"][0]), 8)
    assert out.tolist() == [[1, 2, 3], [0, 0, 0], [1, 2, 3], [4, 5, 6], [4, 5, 6], [0, 0, 0],
                            [0xFFFF] * 3, [0xFFFF] * 3]


def _bf(vals):
    return _bf16_bits(torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16))


def test_combine_closed_forms():
    eo = np.stack([_bf([1.0, 2.0, 1.0, 1.0]), _bf([3.0, 4.0, 1.0, 1.0])])
    e2p = np.array([0, 1], np.int32)
    # 0.25*1 + 0.75*3 = 2.5 ; 0.25*2 + 0.75*4 = 3.5 ; exact
    w = np.array([[0.25, 0.75]], np.float32)
    out = oracle.combine(eo, e2p, w, 2)
    assert out[0, :2].tolist() == _bf([2.5, 3.5]).tolist()
    # bf16 rounding ties: 1 + 2^-8 -> 1.0 (even), 1 + 3*2^-8 -> 1 + 2^-6 (even)
    w = np.array([[1.0, 2 ** -8]], np.float32)
    assert oracle.combine(eo, e2p, w, 2)[0, 2] == _bf([1.0])[0]
    w = np.array([[1.0, 3 * 2 ** -8]], np.float32)
    assert oracle.combine(eo, e2p, w, 2)[0, 2] == _bf([1.0 + 2 ** -6])[0]
    # fp32 accumulation (rounded product, rounded add): w0 = 1 + 2^-23, x = 1 + 2^-7 gives the
    # product 1 + 2^-7 + 2^-23 (the 2^-30 term is rounded away); adding -(1 + 2^-7) leaves 2^-23.
    # An exact (double) sum would give 2^-23 + 2^-30, a different bf16 value.
    x = _bf([1.0 + 2 ** -7])
    eo2 = np.stack([x, x])
    w = np.array([[np.float32(1.0 + 2 ** -23), -1.0]], np.float32)
    assert oracle.combine(eo2, e2p, w, 2)[0, 0] == _bf([2.0 ** -23])[0]
    # exact product second: a fused multiply-add would leave 2^-23 + 2^-30 = 2^-23 (1 + 2^-7), a bf16 value
    w = np.array([[-1.0, np.float32(1.0 + 2 ** -23)]], np.float32)
    assert oracle.combine(eo2, e2p, w, 2)[0, 0] == _bf([2.0 ** -23])[0]
    # k=1 with weight 1 is a copy; bf16 weights are read as bf16
    assert np.array_equal(oracle.combine(eo, np.array([1], np.int32), np.array([[1.0]], np.float32), 1), eo[1:2])
    wb = _bf([0.5, 0.5]).reshape(1, 2)
    assert oracle.combine(eo, e2p, wb, 2)[0, :2].tolist() == _bf([2.0, 3.0]).tolist()
    # another shard's selections (slot -1) add nothing: with the other slot weighted 1 the
    # result is that row; with every slot -1 it is zero
    w = np.array([[1.0, 0.75]], np.float32)
    assert np.array_equal(oracle.combine(eo, np.array([0, -1], np.int32), w, 2), eo[0:1])
    assert np.all(oracle.combine(eo, np.array([-1, -1], np.int32), w, 2) == 0)


def test_dispatch_skips_other_shards_selections():
    # dispatch of a shard: rows only for local slots; tokens whose selections are all elsewhere are
    # copied nowhere; padding rows zero; rows past P untouched
    hidden = np.stack([_bf([1.0, 2.0]), _bf([3.0, 4.0]), _bf([5.0, 6.0])])
    ids = np.array([[1, 0], [1, 2], [3, 0]], np.int32)  # experts 1, 2 local (offset 1, two experts)
    bk = oracle.route_bookkeeping(ids, 4, 4, 1, 2)
    P = int(bk["totals"][0])
    out = oracle.dispatch(hidden, bk["e2p"], bk["p2t"], P, P + 4, fill=0x7FBF)
    assert P == 8 and bk["e2p"].tolist() == [0, -1, 1, 4, -1, -1]
    assert out[0].tolist() == hidden[0].tolist() and out[1].tolist() == hidden[1].tolist()
    assert out[4].tolist() == hidden[1].tolist()
    assert np.all(out[[2, 3, 5, 6, 7]] == 0)
    assert np.all(out[P:] == 0x7FBF)


def test_combine_f32_rows_closed_forms():
    """fp32 expert rows -> fp32 token rows: the same slot-order fp32 accumulation (rounded product, rounded
    add), with no final rounding."""
    eo = np.array([[1.0, 2.0, -3.0], [3.0, 4.0, 0.5]], np.float32)
    e2p = np.array([0, 1], np.int32)
    out = oracle.combine(eo, e2p, np.array([[0.25, 0.75]], np.float32), 2)
    assert out.dtype == np.float32 and out[0].tolist() == [2.5, 3.5, -0.375]
    # a rounded product then a rounded add: (1 + 2^-23)(1 + 2^-7) rounds to 1 + 2^-7 + 2^-23, minus
    # (1 + 2^-7) leaves 2^-23; a fused multiply-add or an exact sum gives 2^-23 + 2^-30
    x = np.float32(1.0 + 2 ** -7)
    eo2 = np.array([[x], [x]], np.float32)
    w = np.array([[np.float32(1.0 + 2 ** -23), -1.0]], np.float32)
    assert oracle.combine(eo2, e2p, w, 2)[0, 0] == np.float32(2.0 ** -23)
    # the same with the exact product second, where a fused multiply-add would keep the 2^-30
    w = np.array([[-1.0, np.float32(1.0 + 2 ** -23)]], np.float32)
    assert oracle.combine(eo2, e2p, w, 2)[0, 0] == np.float32(2.0 ** -23)
    # slot order: 1 + 2^-24 + 2^-24 in slot order stays 1 (each add ties to even); the reverse order
    # would give 1 + 2^-23
    ones = np.ones((3, 1), np.float32)
    w3 = np.array([[1.0, 2 ** -24, 2 ** -24]], np.float32)
    assert oracle.combine(ones, np.array([0, 1, 2], np.int32), w3, 3)[0, 0] == np.float32(1.0)
    w3r = np.array([[2 ** -24, 2 ** -24, 1.0]], np.float32)
    assert oracle.combine(ones, np.array([0, 1, 2], np.int32), w3r, 3)[0, 0] == np.float32(1.0 + 2 ** -23)
    # bf16 weights read as bf16; another shard's slot adds nothing
    wb = _bf([0.5, 0.5]).reshape(1, 2)
    assert oracle.combine(eo, e2p, wb, 2)[0].tolist() == [2.0, 3.0, -1.25]
    assert oracle.combine(eo, np.array([-1, 1], np.int32), np.array([[9.0, 2.0]], np.float32), 2)[0].tolist() == \
        [6.0, 8.0, 1.0]


# --------------------------------------------------------------------------- decode fused


def test_decode_rmsnorm_special_cases():
    T, H, E = 2, 128, 8
    ones = _bf([1.0] * H)
    x = np.stack([ones, ones])
    Wm = np.zeros((H, E), np.uint16)
    out = oracle.rmsnorm_router_topk(x, ones, Wm, None, k=2, eps=1e-6)
    assert np.all(out["out_norm"] == _bf([1.0])[0])  # 1/sqrt(1 + 1e-6) rounds to 1.0 in bf16
    # one-hot row, eps = 0: xn = sign(a) * sqrt(H) * gamma = 11.3137... -> bf16 11.3125
    xr = np.zeros((1, H), np.uint16)
    xr[0, 5] = _bf([-3.0])[0]
    out = oracle.rmsnorm_router_topk(xr, ones, Wm[:, :2], None, k=1, eps=0.0)
    assert out["out_norm"][0, 5] == _bf([-11.3125])[0]
    assert np.all(np.delete(out["out_norm"][0], 5) == 0)
    # constant row a = 2^-10 with eps = 3 a^2: xn = a / sqrt(a^2 + 3 a^2) = 1/2 exactly
    xc = np.stack([_bf([2.0 ** -10] * H)])
    out = oracle.rmsnorm_router_topk(xc, ones, Wm, None, k=2, eps=3.0 * 2.0 ** -20)
    assert np.all(out["out_norm"] == _bf([0.5])[0])
    # power-of-two scaling of x leaves xn unchanged when eps = 0
    g = torch.Generator().manual_seed(1)
    xa = torch.randn(3, H, generator=g).to(torch.bfloat16)
    a = oracle.rmsnorm_router_topk(xa, ones, Wm, None, k=2, eps=0.0)
    b = oracle.rmsnorm_router_topk(xa * 4, ones, Wm, None, k=2, eps=0.0)
    assert np.array_equal(a["out_norm"], b["out_norm"])


def _bf16_round_fraction(y: Fraction) -> float:
    """The bf16 value nearest to the exact rational y (ties to even), as a float."""
    if y == 0:
        return 0.0
    f = np.float32(float(y))
    base = int(np.array(f, np.float32).view(np.uint32)) >> 16
    best = None
    for cand in range(max(base - 2, 0), base + 3):
        v = Fraction(float(np.array(cand << 16, np.uint32).view(np.float32)))
        key = (abs(v - y), cand & 1)
        if best is None or key < best[0]:
            best = (key, float(v))
    return best[1]


def _near_bf16_midpoint(y: Fraction, rel: float) -> bool:
    """True if y lies within rel (relative) of a point halfway between two bf16 values."""
    if y == 0:
        return False
    f = np.float32(float(y))
    base = int(np.array(f, np.float32).view(np.uint32)) >> 16
    for cand in range(max(base - 2, 0), base + 2):
        lo = Fraction(float(np.array(cand << 16, np.uint32).view(np.float32)))
        hi = Fraction(float(np.array((cand + 1) << 16, np.uint32).view(np.float32)))
        if abs((lo + hi) / 2 - y) <= abs(y) * Fraction(rel):
            return True
    return False


def test_decode_rmsnorm_gamma_per_hidden_index_exact():
    """out_norm[t,h] = bf16(x[t,h] * gamma[h] / sqrt(mean_h x[t,h]^2 + eps)) against exact rationals (the
    square root to 60 significant digits), with a gamma that differs on every h and has negative and zero
    entries: dropping gamma, indexing it by the token, or applying it twice fails this pin (NKI page,
    Parameters: gamma [1, H], and Background: RMSNorm before the router)."""
    import decimal
    T, H = 3, 256
    g = torch.Generator().manual_seed(11)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    gam = torch.randn(H, generator=g) * 0.7 + 0.2
    gam[::17] = 0.0
    gam[5::23] *= -3.0
    gam = gam.to(torch.bfloat16)
    eps = 1e-6
    out = oracle.rmsnorm_router_topk(x, gam, np.zeros((H, 8), np.uint16), None, k=2, eps=eps)
    xn = oracle.bf16_to_f32(out["out_norm"])
    xf, gf = x.float().numpy(), gam.float().numpy()
    assert len(set(gf.tolist())) > H // 2 and (gf < 0).any() and (gf == 0).any()
    ctx = decimal.Context(prec=60)
    eps_q = Fraction(float(np.float32(eps)))
    checked = 0
    for t in range(T):
        ms = sum(Fraction(float(v)) ** 2 for v in xf[t]) / H + eps_q
        root = ctx.sqrt(ctx.divide(decimal.Decimal(ms.numerator), decimal.Decimal(ms.denominator)))
        r = 1 / Fraction(root)  # 1/sqrt to ~60 digits
        for h in range(H):
            y = Fraction(float(xf[t, h])) * Fraction(float(gf[h])) * r
            if _near_bf16_midpoint(y, 1e-12):
                continue
            assert xn[t, h] == _bf16_round_fraction(y), (t, h, float(y), xn[t, h])
            checked += 1
    assert checked >= T * H - 4


def test_decode_one_hot_projection_and_affinity():
    """One-hot W columns copy normalised entries into the logits exactly; the affinities are
    sigmoid(logit) at the selected experts (ACT2: activation after top-k), 0 elsewhere."""
    T, H, E, k = 4, 256, 16, 3
    g = torch.Generator().manual_seed(2)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    gamma = (torch.randn(H, generator=g) * 0.1 + 1).to(torch.bfloat16)
    Wm = torch.zeros(H, E)
    cols = [(e * 13) % H for e in range(E)]
    for e, h in enumerate(cols):
        Wm[h, e] = 1.0
    bias = torch.zeros(E)
    bias[2] = 0.5
    out = oracle.rmsnorm_router_topk(x, gamma, Wm.to(torch.bfloat16), bias.to(torch.bfloat16), k=k)
    xn = oracle.bf16_to_f32(out["out_norm"])
    np.testing.assert_array_equal(out["logits"], xn[:, cols] + bias.numpy())
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-out["logits"][t, e], e))[:k]
        assert out["ids"][t].tolist() == order
        aff = oracle.bf16_to_f32(out["affinities"][t])
        for e in range(E):
            if e in order:
                ref = 1.0 / (1.0 + math.exp(-float(out["logits"][t, e])))
                assert abs(aff[e] - ref) <= 2 ** -8 * ref
            else:
                assert aff[e] == 0.0


def test_router_logits_alone_matches_fused_oracle():
    spec = W.DecodeSpec(T=4, H=256, E=32, k=4)
    inp = W.decode_inputs(spec)
    out = oracle.rmsnorm_router_topk(inp["hidden"], inp["gamma"], inp["W"], inp["bias"], k=4)
    assert np.array_equal(oracle.router_logits(out["out_norm"], inp["W"], inp["bias"]), out["logits"])


def test_decode_projection_matches_library_matmul():
    spec = W.DecodeSpec(T=8, H=512, E=64, k=8)
    inp = W.decode_inputs(spec)
    out = oracle.rmsnorm_router_topk(inp["hidden"], inp["gamma"], inp["W"], inp["bias"], k=8)
    xn = torch.from_numpy(oracle.bf16_to_f32(out["out_norm"])).double()
    ref = (xn @ inp["W"].double() + inp["bias"].double()).float().numpy()
    np.testing.assert_array_equal(out["logits"], ref)


def test_decode_rejects_page_constraints():
    x = np.zeros((129, 128), np.uint16)
    with pytest.raises(ValueError):
        oracle.rmsnorm_router_topk(x, np.zeros(128, np.uint16), np.zeros((128, 8), np.uint16), None, k=2)
    x = np.zeros((4, 100), np.uint16)
    with pytest.raises(ValueError):
        oracle.rmsnorm_router_topk(x, np.zeros(100, np.uint16), np.zeros((100, 8), np.uint16), None, k=2)


# --------------------------------------------------------------------------- expert-parallel regroup


def test_ep_regroup_handworked():
    # two ranks send to a rank owning two experts, tile 2: rank 0 sends one row for expert 0 and two for
    # expert 1, rank 1 one row for expert 1.  Receive order r0 (s0,e0), r1 r2 (s0,e1), r3 (s1,e1).
    # Expert 0: 1 row -> 2 padded rows; expert 1: 3 rows -> 4, ordered by source then token.
    counts = np.array([[1, 2], [0, 1]], np.int32)
    recv = np.array([[10, 11], [20, 21], [30, 31], [40, 41]], np.uint16)
    out = oracle.ep_regroup(counts, recv, 2)
    assert out["offsets"].tolist() == [0, 2, 6] and out["totals"].tolist() == [6, 3]
    assert out["padded_to_recv"].tolist() == [0, -1, 1, 2, 3, -1]
    assert out["padded"].tolist() == [[10, 11], [0, 0], [20, 21], [30, 31], [40, 41], [0, 0]]
    # no rows at all, and a rank that sends nothing
    e = oracle.ep_regroup(np.zeros((3, 2), np.int32), np.zeros((0, 8), np.float32), 4)
    assert e["offsets"].tolist() == [0, 0, 0] and e["totals"].tolist() == [0, 0]


def test_ep_regroup_equals_single_route_of_the_concatenation():
    """Rows sent by W ranks (each routed over all experts with tile 1 and dispatched) and regrouped by the
    receiving rank equal the shard bookkeeping + dispatch of all ranks' tokens concatenated in rank order:
    two definitions written separately (the shard route of the pages' local_expert_offset /
    local_num_experts, and the exchange) must agree."""
    rng = np.random.default_rng(7)
    W, E, k, H, tile = 3, 12, 3, 4, 4
    L = E // W
    Ts = [9, 0, 14]
    ids_r = [np.array([rng.choice(E, k, replace=False) for _ in range(T)], np.int32).reshape(T, k) for T in Ts]
    hid_r = [rng.integers(0, 60000, (T, H)).astype(np.uint16) for T in Ts]
    ids_all = np.concatenate(ids_r)
    hid_all = np.concatenate(hid_r)
    for d in range(W):
        # the sender side: tile-1 bookkeeping over all experts, dispatch, this destination's expert range
        counts = np.zeros((W, L), np.int32)
        parts = []
        for s in range(W):
            bk = oracle.route_bookkeeping(ids_r[s], E, 1)
            send = oracle.dispatch(hid_r[s], bk["e2p"], bk["p2t"], int(bk["totals"][0]), max(int(bk["totals"][0]), 1))
            lo, hi = int(bk["offsets"][d * L]), int(bk["offsets"][(d + 1) * L])
            parts.append(send[lo:hi])
            counts[s] = bk["counts"][d * L:(d + 1) * L]
        recv = np.concatenate(parts) if sum(p.shape[0] for p in parts) else np.zeros((0, H), np.uint16)
        got = oracle.ep_regroup(counts, recv, tile)
        ref_bk = oracle.route_bookkeeping(ids_all, E, tile, d * L, L)
        P = int(ref_bk["totals"][0])
        ref = oracle.dispatch(hid_all, ref_bk["e2p"], ref_bk["p2t"], P, P)
        assert got["offsets"].tolist() == ref_bk["offsets"].tolist()
        assert got["totals"].tolist() == ref_bk["totals"].tolist()
        assert np.array_equal(got["padded"], ref[:P])
        assert np.array_equal(got["padded_to_recv"] >= 0, ref_bk["p2t"] >= 0)


# --------------------------------------------------------------------------- fused shared experts


def test_fused_shared_experts_handworked():
    """Reading of num_fused_shared_experts (trtllm_gen_routing, Parameters): one shared expert (id E = 4)
    appended to every token after its k routed slots, weight 1.0, local on every shard after the shard's
    routed experts.  Hand-worked from T=3, k=2, E=4, tile 4, ids [[1,0],[1,2],[3,1]]."""
    ids, w = oracle.append_shared(np.array([[1, 0], [1, 2], [3, 1]], np.int32),
                                  np.array([[0.5, 0.25], [0.6, 0.4], [0.7, 0.3]], np.float32), 4, 1)
    assert ids.tolist() == [[1, 0, 4], [1, 2, 4], [3, 1, 4]]
    assert w[:, 2].tolist() == [1.0, 1.0, 1.0] and w[0, :2].tolist() == [0.5, 0.25]
    bk = oracle.route_bookkeeping(ids, 4, 4, num_shared=1)
    assert bk["counts"].tolist() == [1, 3, 1, 1, 3]
    assert bk["offsets"].tolist() == [0, 4, 8, 12, 16, 20]
    assert bk["e2p"].tolist() == [4, 0, 16, 5, 8, 17, 12, 6, 18]
    assert bk["p2t"].tolist() == [0, -1, -1, -1, 0, 1, 2, -1, 1, -1, -1, -1, 2, -1, -1, -1, 0, 1, 2, -1]
    assert bk["tile_expert"].tolist() == [0, 1, 2, 3, 4] and bk["tile_mn_limit"].tolist() == [1, 7, 9, 13, 19]
    assert bk["totals"].tolist() == [20, 5]
    # a shard owning experts 1 and 2: the shared expert is local there too, after them
    sh = oracle.route_bookkeeping(ids, 4, 4, 1, 2, num_shared=1)
    assert sh["counts"].tolist() == [3, 1, 3] and sh["offsets"].tolist() == [0, 4, 8, 12]
    assert sh["e2p"].tolist() == [0, -1, 8, 1, 4, 9, -1, 2, 10]
    assert sh["p2t"].tolist() == [0, 1, 2, -1, 1, -1, -1, -1, 0, 1, 2, -1]
    assert sh["tile_expert"].tolist() == [0, 1, 2] and sh["tile_mn_limit"].tolist() == [3, 5, 11]
    assert sh["totals"].tolist() == [12, 3]
