"""GPU parity of the aux-loss path (scores, loss forward, loss backward) against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from parity import near_tie_ok, to_np
from top_expert_selection_b200 import binding as B
from top_expert_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu
RTOL = 1e-5


def check_scores(logits, k, score_fn=W.SOFTMAX):
    T, E = logits.shape
    g = B.aux_scores(logits.cuda(), k, score_fn)
    torch.cuda.synchronize()
    o = oracle.aux_scores(logits, k, score_fn)
    probs = to_np(g["probs"])
    ref = o["probs"]
    assert np.all(np.abs(probs - ref) <= RTOL * np.abs(ref) + 1e-30), "probs off by more than 1e-5 relative"
    gm = to_np(g["routing_map"])
    om = o["routing_map"]
    flips = 0
    for t in np.nonzero((gm != om).any(1))[0]:
        gsel = np.nonzero(gm[t])[0]
        osel = sorted(np.nonzero(om[t])[0].tolist(), key=lambda e: (-ref[t, e], e))
        gsel = sorted(gsel.tolist(), key=lambda e: (-ref[t, e], e))
        assert near_tie_ok(ref[t], gsel, osel, k, False, 0, 0, None), f"token {t} routing map not a near tie"
        flips += 1
    assert flips <= max(1, T // 1000)
    assert np.all(gm.sum(1) == k)
    tpe = to_np(g["tokens_per_expert"])
    assert np.array_equal(tpe, gm.sum(0).astype(np.int32)), "tokens_per_expert != column sums of routing_map"
    if flips == 0:
        assert np.array_equal(tpe, o["tokens_per_expert"])
    return g, o, flips


def test_aux_workload_full_size():
    spec = W.QWEN3_AUX
    lg = W.aux_inputs(spec)["logits"]
    g, o, flips = check_scores(lg, spec.k)
    print("aux scores flips:", flips)
    # loss forward on the GPU's own probs / counts vs the oracle on the same inputs, and from scratch
    loss = B.aux_loss_fwd(g["probs"], g["tokens_per_expert"], spec.T, spec.k, spec.coeff)
    torch.cuda.synchronize()
    ref_same = oracle.aux_loss_fwd(to_np(g["probs"]), to_np(g["tokens_per_expert"]), spec.T, spec.k, spec.coeff)
    ref_scratch = oracle.aux_loss_fwd(o["probs"], o["tokens_per_expert"], spec.T, spec.k, spec.coeff)
    got = float(loss.item())
    assert abs(got - ref_same) <= RTOL * abs(ref_same)
    assert abs(got - ref_scratch) <= RTOL * abs(ref_scratch)
    # determinism of the reduction
    loss2 = B.aux_loss_fwd(g["probs"], g["tokens_per_expert"], spec.T, spec.k, spec.coeff)
    assert float(loss2.item()) == got
    # backward with upstream grad 1.0
    gl = torch.tensor([spec.grad_loss], dtype=torch.float32, device="cuda")
    gr = B.aux_loss_bwd(gl, g["probs"], g["tokens_per_expert"], spec.T, spec.k, spec.coeff)
    torch.cuda.synchronize()
    check_backward(to_np(g["probs"]), to_np(g["tokens_per_expert"]), spec.T, spec.k, spec.coeff, spec.grad_loss,
                   to_np(gr["grad_probs"]), to_np(gr["grad_logits"]))


def check_backward(p, tpe, T_total, k, coeff, grad, got_gp, got_gl):
    ref = oracle.aux_loss_bwd(p, tpe, T_total, k, coeff, grad)
    assert np.all(np.abs(got_gp - ref["grad_probs"]) <= RTOL * np.abs(ref["grad_probs"]) + 1e-30)
    # relative to the terms before cancellation: |p * g_e| + |p * sum_j p_j g_j|
    E = p.shape[1]
    C = coeff * E / (T_total * k)
    ge = grad * C * tpe.astype(np.float64)
    dot = (p.astype(np.float64) * ge).sum(1, keepdims=True)
    scale = np.abs(p * ge) + np.abs(p * dot)
    err = np.abs(got_gl.astype(np.float64) - ref["grad_logits"])
    assert np.all(err <= RTOL * scale + 1e-30), f"grad_logits err/scale max {np.max(err / (scale + 1e-30))}"


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (33, 64, 6), (1000, 128, 8), (257, 96, 4), (300, 256, 8),
                                   (129, 1024, 16), (77, 33, 3), (1, 64, 1), (5, 128, 8), (4097, 256, 7),
                                   (999, 64, 8), (2, 128, 3), (6, 256, 1)])
def test_aux_shapes(T, E, k):
    g = torch.Generator().manual_seed(T + E)
    lg = torch.randn(T, E, generator=g) * 1.5
    gg, o, _ = check_scores(lg, k)
    probs, tpe = gg["probs"], gg["tokens_per_expert"]
    for T_total in (T, 3 * T):
        loss = B.aux_loss_fwd(probs, tpe, T_total, k, 0.37)
        ref = oracle.aux_loss_fwd(to_np(probs), to_np(tpe), T_total, k, 0.37)
        assert abs(float(loss.item()) - ref) <= RTOL * abs(ref)
        gl = torch.tensor([0.75], dtype=torch.float32, device="cuda")
        gr = B.aux_loss_bwd(gl, probs, tpe, T_total, k, 0.37)
        check_backward(to_np(probs), to_np(tpe), T_total, k, 0.37, 0.75, to_np(gr["grad_probs"]),
                       to_np(gr["grad_logits"]))


@pytest.mark.parametrize("score_fn", [W.SOFTMAX, W.SIGMOID])
@pytest.mark.parametrize("E", [64, 128, 256])
def test_aux_scores_masked_and_tied_rows(E, score_fn):
    """Rows the per-lane top-3 threshold cannot settle alone: exact ties (all equal; a block of equal
    maxima wider than k; ties at zero probability after -inf logits), one dominant expert, and the top k
    held by one lane's experts.  The routing map equals the oracle's exactly (ties -> lower expert)."""
    k = 8
    rng = np.random.default_rng(E + score_fn)
    lg = rng.standard_normal((13, E)).astype(np.float32)
    lg[0] = 0.5                                    # all equal
    lg[1] = -np.inf
    lg[1, [5, 77 % E, 40]] = [1.0, 2.0, 0.5]       # three finite: then ties at 0 -> lowest experts
    lg[2] = 0.0
    lg[2, rng.permutation(E)[:20]] = 1.0           # 20 equal maxima
    lg[3] = 0.0
    lg[3, 9] = 100.0                               # one dominant expert, the rest equal
    lane_experts = [c * 32 + 4 * 2 + r for c in range(E // 32) for r in range(4)]
    lg[4, lane_experts] += 6.0                     # the top k all in one lane's experts
    if score_fn == W.SIGMOID:
        lg[1] = np.where(np.isinf(lg[1]), -30.0, lg[1])  # sigmoid(-inf) = 0 is a tie as well; keep finite
    g = B.aux_scores(torch.from_numpy(lg).cuda(), k, score_fn)
    torch.cuda.synchronize()
    o = oracle.aux_scores(lg, k, score_fn)
    assert np.array_equal(to_np(g["routing_map"]), o["routing_map"])
    assert np.array_equal(to_np(g["tokens_per_expert"]), o["tokens_per_expert"])
    ref = o["probs"]
    assert np.all(np.abs(to_np(g["probs"]) - ref) <= RTOL * np.abs(ref) + 1e-30)


def test_aux_scores_rows_with_non_finite_logits():
    """A NaN or +inf logit makes the row's score sum non-finite: that row is redone by the whole warp and
    still marks exactly k experts; the other rows of the same four-token group match the oracle."""
    T, E, k = 9, 128, 8
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[2, 17] = np.nan
    lg[5, 100] = np.inf
    g = B.aux_scores(torch.from_numpy(lg).cuda(), k)
    torch.cuda.synchronize()
    o = oracle.aux_scores(lg, k)
    gm = to_np(g["routing_map"])
    assert np.all(gm.sum(1) == k)
    assert np.array_equal(to_np(g["tokens_per_expert"]), gm.sum(0).astype(np.int32))
    ok = [t for t in range(T) if t not in (2, 5)]
    assert np.array_equal(gm[ok], o["routing_map"][ok])
    assert np.all(np.abs(to_np(g["probs"])[ok] - o["probs"][ok]) <= RTOL * np.abs(o["probs"][ok]) + 1e-30)


def test_aux_loss_fwd_unaligned_counts_and_ragged_rows():
    # counts that start off 16 bytes take the shared-memory column path; both paths agree with the oracle
    T, E, k = 1001, 128, 8
    g = torch.Generator().manual_seed(9)
    lg = torch.randn(T, E, generator=g)
    sc = B.aux_scores(lg.cuda(), k)
    big = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    big[1:] = sc["tokens_per_expert"]
    for tpe in (sc["tokens_per_expert"], big[1:]):
        loss = B.aux_loss_fwd(sc["probs"], tpe, 3 * T, k, 0.01)
        ref = oracle.aux_loss_fwd(to_np(sc["probs"]), to_np(sc["tokens_per_expert"]), 3 * T, k, 0.01)
        assert abs(float(loss.item()) - ref) <= RTOL * abs(ref)


def test_division_by_reciprocal_matches_ieee_quotient():
    """The aux-scores kernel divides a row's entries by their sum through one reciprocal and two fused
    multiply-add corrections (Markstein's method); that must give the IEEE quotient bit for bit.  Random
    pairs over the method's whole range, pairs whose first product is least accurate (numerator mantissa
    near 2, denominator mantissa near 1 and near 2), exact and near-exact multiples, and the softmax
    rows of the aux workload."""
    g = torch.Generator().manual_seed(17)
    n = 1 << 24

    def rand_float(lo_exp, hi_exp, mant=None):
        e = torch.randint(lo_exp, hi_exp + 1, (n,), generator=g).to(torch.float64)
        m = torch.rand(n, generator=g, dtype=torch.float64) + 1.0 if mant is None else mant
        return (m * torch.pow(2.0, e)).to(torch.float32)

    cases = []
    b = rand_float(-20, 19)
    cases.append((rand_float(-60, 19), b))                                   # anything in range
    cases.append((b * rand_float(-40, 0), b))                                # quotients <= 2
    near2 = 2.0 - torch.rand(n, generator=g, dtype=torch.float64) * 2.0 ** -10
    near1 = 1.0 + torch.rand(n, generator=g, dtype=torch.float64) * 2.0 ** -10
    cases.append((rand_float(-30, 0, near2), rand_float(-10, 10, near1)))
    cases.append((rand_float(-30, 0, near2), rand_float(-10, 10, near2)))
    cases.append((rand_float(-30, 0, near1), rand_float(-10, 10, near2)))
    k = torch.randint(1, 1 << 20, (n,), generator=g).to(torch.float32)
    cases.append((b * k, b))                                                 # exact multiples
    cases.append((torch.nextafter(b * k, torch.full_like(b, float("inf"))), b))
    lg = W.aux_inputs(W.QWEN3_AUX)["logits"]
    z = torch.exp(lg.double() - lg.double().max(1, keepdim=True).values).float()
    cases.append((z.reshape(-1), z.sum(1, keepdim=True).expand_as(z).reshape(-1).contiguous()))
    for a_, b_ in cases:
        assert B.debug_div_check(a_.contiguous().cuda(), b_.contiguous().cuda()) == 0


def test_aux_uniform_closed_form_on_gpu():
    T, E, k, coeff = 4096, 128, 8, 1e-2
    g = B.aux_scores(torch.zeros(T, E, device="cuda"), k)
    loss = B.aux_loss_fwd(g["probs"], g["tokens_per_expert"], T, k, coeff)
    assert abs(float(loss.item()) - coeff * T) <= 1e-6 * coeff * T
    assert to_np(g["tokens_per_expert"]).tolist() == [T] * k + [0] * (E - k)
    gr = B.aux_loss_bwd(torch.ones(1, device="cuda"), g["probs"], g["tokens_per_expert"], T, k, coeff)
    rs = gr["grad_logits"].double().sum(1).abs().max().item()
    assert rs < 1e-9


def test_aux_sigmoid_scores():
    g = torch.Generator().manual_seed(1)
    lg = torch.randn(500, 64, generator=g)
    check_scores(lg, 4, W.SIGMOID)


def test_aux_repeated_calls_reuse_workspace():
    g = torch.Generator().manual_seed(2)
    lg = (torch.randn(2000, 128, generator=g)).cuda()
    ws = B.aux_workspace(2000, 128, "cuda")
    a = B.aux_scores(lg, 8, ws=ws)
    b = B.aux_scores(lg, 8, ws=ws)
    assert torch.equal(a["tokens_per_expert"], b["tokens_per_expert"])
    l1 = B.aux_loss_fwd(a["probs"], a["tokens_per_expert"], 2000, 8, 0.01, ws=ws)
    l2 = B.aux_loss_fwd(a["probs"], a["tokens_per_expert"], 2000, 8, 0.01, ws=ws)
    assert torch.equal(l1, l2)
    assert B.status(ws) == B.MOE_OK


@pytest.mark.parametrize("T,E", [(1, 8), (77, 33), (1000, 128), (32768, 128), (129, 1024)])
def test_aux_scores_backward(T, E):
    """moe_aux_scores_bwd against the oracle's vector-Jacobian product of the softmax, relative to the
    terms before cancellation: |p_e*g_e| + |p_e| * sum_j |p_j*g_j| (the dot of a signed upstream
    gradient cancels, so its fp32 rounding scales with the sum of the magnitudes of its terms)."""
    g = torch.Generator().manual_seed(T * 7 + E)
    lg = torch.randn(T, E, generator=g) * 1.5
    G = torch.randn(T, E, generator=g)
    probs = oracle.aux_scores(lg, 2)["probs"]
    got = to_np(B.aux_scores_bwd(torch.from_numpy(probs).cuda(), G.cuda()))
    torch.cuda.synchronize()
    ref = oracle.aux_scores_bwd(probs, G)
    p64 = probs.astype(np.float64)
    terms = np.abs(p64 * G.double().numpy())
    scale = terms + p64 * terms.sum(1, keepdims=True)
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= RTOL * scale + 1e-30), f"err/scale max {np.max(err / (scale + 1e-30))}"


@pytest.mark.parametrize("score_fn", [W.SIGMOID, W.SOFTMAX])
@pytest.mark.parametrize("T,E", [(1, 8), (77, 33), (1000, 128), (32768, 128), (129, 1024), (300, 5)])
def test_aux_scores_backward_from_logits(score_fn, T, E):
    """moe_aux_scores_bwd_logits against the oracle's vector-Jacobian product of the scores recomputed from
    the logits, relative to the terms before cancellation: d_e * (|g_e| + sum_j p_j |g_j|), with
    d = p (softmax) or s (1 - s) / S (sigmoid over the row sum)."""
    g = torch.Generator().manual_seed(T * 11 + E + 3 * score_fn)
    lg = torch.randn(T, E, generator=g) * 2.0
    G = torch.randn(T, E, generator=g)
    got = to_np(B.aux_scores_bwd_logits(lg.cuda(), G.cuda(), score_fn=score_fn))
    torch.cuda.synchronize()
    ref = oracle.aux_scores_bwd_logits(lg, G, score_fn=score_fn)
    x = lg.double().numpy()
    if score_fn == W.SOFTMAX:
        z = np.exp(x - x.max(1, keepdims=True))
        p = z / z.sum(1, keepdims=True)
        d = p
    else:
        s = 1.0 / (1.0 + np.exp(-x))
        p = s / s.sum(1, keepdims=True)
        d = s * (1 - s) / s.sum(1, keepdims=True)
    ag = np.abs(G.double().numpy())
    scale = d * (ag + (p * ag).sum(1, keepdims=True))
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= RTOL * scale + 1e-30), f"err/scale max {np.max(err / (scale + 1e-30))}"


def test_aux_scores_backward_from_logits_unaligned_rows():
    # rows that start off 16 bytes (a view one element in) take the scalar loads, same values
    T, E = 64, 128
    g = torch.Generator().manual_seed(5)
    big = torch.randn(T * E + 1, generator=g).cuda()
    Gbig = torch.randn(T * E + 1, generator=g).cuda()
    lg, G = big[1:].view(T, E), Gbig[1:].view(T, E)
    out = torch.empty(T * E + 1, device="cuda")[1:].view(T, E)
    B.aux_scores_bwd_logits_into(lg, G, out, score_fn=W.SIGMOID)
    ref = B.aux_scores_bwd_logits(lg.contiguous().clone(), G.clone(), score_fn=W.SIGMOID)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_aux_scores_backward_sigmoid_unsupported():
    p = torch.full((4, 8), 0.125, device="cuda")
    with pytest.raises(Exception):
        B.aux_scores_bwd(p, p, score_fn=W.SIGMOID)
