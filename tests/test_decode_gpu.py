"""GPU parity of moe_rmsnorm_router_topk (fused RMSNorm + tcgen05 router projection + top-k)."""
import numpy as np
import pytest
import torch

import oracle
from parity import ULP_TOL, bf16_ulp_dist, to_np, ulp_dist
from top_expert_selection_b200 import binding as B
from top_expert_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu
LOGIT_RTOL = 1e-5


def run_decode(spec: W.DecodeSpec, inp=None):
    inp = W.decode_inputs(spec) if inp is None else inp
    x, gamma, Wm, bias = inp["hidden"], inp["gamma"], inp["W"], inp["bias"]
    g = B.rmsnorm_router_topk(x.cuda(), gamma.cuda(), Wm.cuda(), bias.cuda() if bias is not None else None,
                              k=spec.k, eps=spec.eps, act=spec.act, debug_logits=True)
    torch.cuda.synchronize()
    assert B.status(g["ws"]) == B.MOE_OK
    o = oracle.rmsnorm_router_topk(x, gamma, Wm, bias, k=spec.k, eps=spec.eps, act=spec.act)
    # normalised hidden states: <= 1 bf16 ulp
    d = bf16_ulp_dist(to_np(g["out_norm"]), o["out_norm"])
    assert d.max() <= 1, f"out_norm off by {d.max()} bf16 ulp"
    n_ulp = int((d > 0).sum())
    # logits: the projection of the GPU's own normalised states, within 1e-5 of sum_h |xn * W|
    # (the scale of the fp32 tensor-core accumulation); then against the oracle from scratch
    xn = oracle.bf16_to_f32(o["out_norm"]).astype(np.float64)
    wf = Wm.float().numpy().astype(np.float64)
    scale = np.abs(xn) @ np.abs(wf)
    gl = to_np(g["logits"])
    ref_same = oracle.router_logits(to_np(g["out_norm"]), Wm, bias)
    err = np.abs(gl.astype(np.float64) - ref_same)
    assert np.all(err <= LOGIT_RTOL * scale + 1e-30), f"logit err/scale max {np.max(err / (scale + 1e-30))}"
    if n_ulp == 0:
        err = np.abs(gl.astype(np.float64) - o["logits"])
        assert np.all(err <= LOGIT_RTOL * scale + 1e-30)
    # ids: the oracle's top-k on the GPU's own logits must equal the GPU ids exactly
    sel = oracle.route_select(gl, k=spec.k, score_fn=W.SIGMOID, softmax_before_topk=0, renormalize=0)
    gids = to_np(g["ids"])
    assert np.array_equal(gids, sel["ids"]), "GPU ids are not the top-k of the GPU logits"
    # against the oracle from scratch: flips only where the oracle's logit gap is within tolerance
    flips = 0
    for t in np.nonzero((gids != o["ids"]).any(1))[0]:
        for a_, b_ in zip(gids[t], o["ids"][t]):
            gap = abs(float(o["logits"][t, a_]) - float(o["logits"][t, b_]))
            tol = 2 * LOGIT_RTOL * max(scale[t, a_], scale[t, b_])
            assert gap <= tol or ulp_dist(o["logits"][t, a_], o["logits"][t, b_]) <= ULP_TOL
        flips += 1
    # affinities: on tokens whose ids agree, <= 1 bf16 ulp; zero off the selected experts
    aff = to_np(g["affinities"])
    same = ~((gids != o["ids"]).any(1))
    d = bf16_ulp_dist(aff[same], o["affinities"][same])
    assert d.max(initial=0) <= 1, f"affinities off by {d.max()} bf16 ulp"
    mask = np.zeros_like(aff, dtype=bool)
    np.put_along_axis(mask, gids.astype(np.int64), True, axis=1)
    assert np.all(aff[~mask] == 0)
    return {"flips": flips, "out_norm_elements_1ulp": n_ulp}, g


def test_decode_workload_full_size():
    rep, _ = run_decode(W.DECODE_FUSED)
    print("decode flips:", rep)


@pytest.mark.parametrize("T,H,E,k,act,bias", [
    (1, 128, 16, 1, W.SIGMOID, False), (7, 256, 64, 4, W.SIGMOID, True), (128, 7168, 256, 8, W.SOFTMAX, True),
    (33, 1024, 96, 6, W.SIGMOID, False), (128, 19200, 128, 8, W.SIGMOID, True), (64, 640, 48, 3, W.SOFTMAX, False),
    (100, 2048, 160, 6, W.SIGMOID, True), (65, 512, 256, 8, W.SIGMOID, True), (128, 32768, 64, 4, W.SIGMOID, True),
    (128, 7168, 384, 8, W.SIGMOID, True), (40, 2048, 272, 8, W.SOFTMAX, True), (128, 4096, 512, 8, W.SIGMOID, True),
    (17, 1024, 784, 6, W.SOFTMAX, False), (128, 2048, 1024, 8, W.SIGMOID, True)])
def test_decode_shapes(T, H, E, k, act, bias):
    # cluster sizes 2..16 (H/64 chunks), one or two 64-token groups, partial expert groups, slices
    # longer than the staging ring (H=19200, 32768), and 272 .. 1024 experts (two to four rounds of 256
    # in the top-k stage, the last one partial for 272 and 784)
    run_decode(W.DecodeSpec(T=T, H=H, E=E, k=k, act=act, has_bias=bias, seed=T + H + E))


def test_decode_all_ones_rows():
    spec = W.DecodeSpec(T=16, H=512, E=64, k=4, has_bias=False)
    inp = W.decode_inputs(spec)
    inp["hidden"] = torch.ones(16, 512).to(torch.bfloat16)
    inp["gamma"] = torch.ones(512).to(torch.bfloat16)
    _, g = run_decode(spec, inp)
    assert bool((g["out_norm"].float() == 1.0).all())


def test_decode_repeated_calls_deterministic():
    spec = W.DECODE_FUSED
    inp = W.decode_inputs(spec)
    args = (inp["hidden"].cuda(), inp["gamma"].cuda(), inp["W"].cuda(), inp["bias"].cuda())
    a = B.rmsnorm_router_topk(*args, k=8, debug_logits=True)
    b = B.rmsnorm_router_topk(*args, k=8, debug_logits=True, ws=a["ws"])
    for key in ("out_norm", "ids", "affinities", "logits"):
        assert torch.equal(a[key], b[key]), key
