"""GPU parity of moe_route against the CPU oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from parity import compare_route, to_np
from top_expert_selection_b200 import binding as B
from top_expert_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu

GUARD = 64
SENT = -123456789


def _guarded(n, dtype, dev):
    """A buffer of n elements with GUARD sentinel elements on each side; returns (full, view)."""
    full = torch.empty(n + 2 * GUARD, dtype=dtype, device=dev)
    if dtype == torch.int32:
        full.fill_(SENT)
    elif dtype == torch.bfloat16:
        full.view(torch.int16).fill_(0x7FC1)
    else:
        full.view(torch.int32).fill_(0x7FC00001)
    return full, full[GUARD:GUARD + n]


def _guards_intact(full, n):
    f = full.detach().cpu()
    if f.dtype == torch.bfloat16:
        f = f.view(torch.int16)
        sent = 0x7FC1
    elif f.dtype == torch.float32:
        f = f.view(torch.int32)
        sent = 0x7FC00001
    else:
        sent = SENT
    return bool((f[:GUARD] == sent).all() and (f[GUARD + n:] == sent).all())


def run_route(spec: W.RouteSpec, logits=None, bias=None):
    inp = W.route_inputs(spec)
    if logits is None:
        logits, bias = inp["logits"], inp["bias"]
    dev = torch.device("cuda")
    p = B.route_params(spec.T, spec.E, spec.k, score_fn=spec.score_fn, softmax_before_topk=spec.softmax_before_topk,
                       n_group=spec.n_group, topk_group=spec.topk_group, group_score_topn=spec.group_score_topn,
                       renormalize=spec.renormalize, scaling_factor=spec.scaling_factor,
                       tile_tokens_dim=spec.tile_tokens_dim, logits_dtype=spec.logits_dtype,
                       bias_dtype=spec.bias_dtype, weights_dtype=spec.weights_dtype,
                       local_expert_offset=spec.local_expert_offset, local_num_experts=spec.local_num_experts)
    max_padded, max_tiles = B.route_capacity(p)
    T, E, k = spec.T, spec.E, spec.k
    nl = spec.local_num_experts or E
    wdt = torch.bfloat16 if spec.weights_dtype == W.BF16 else torch.float32
    sizes = {"ids": (T * k, torch.int32), "weights": (T * k, wdt), "counts": (nl, torch.int32),
             "offsets": (nl + 1, torch.int32), "e2p": (T * k, torch.int32), "p2t": (max_padded, torch.int32),
             "tile_expert": (max_tiles, torch.int32), "tile_mn_limit": (max_tiles, torch.int32),
             "totals": (2, torch.int32)}
    fulls, views = {}, {}
    for name, (n, dt) in sizes.items():
        fulls[name], views[name] = _guarded(n, dt, dev)
    ws = B.make_workspace(B.route_workspace_bytes(p), dev)
    lg_d = logits.to(dev)
    b_d = bias.to(dev) if bias is not None else None
    B.route_into(p, lg_d, b_d, views, ws)
    torch.cuda.synchronize()
    assert B.status(ws) == B.MOE_OK
    for name, (n, _) in sizes.items():
        assert _guards_intact(fulls[name], n), f"guard zone of {name} overwritten"
    P = int(views["totals"][0])
    # rows of permuted_to_token at or past P are not written
    assert bool((views["p2t"][P:].cpu() == SENT).all())
    gpu = {n: v for n, v in views.items()}
    gpu["ids"] = views["ids"].view(T, k)
    gpu["weights"] = views["weights"].view(T, k)
    orc = oracle.route_select(logits, k=k, score_fn=spec.score_fn, softmax_before_topk=spec.softmax_before_topk,
                              n_group=spec.n_group, topk_group=spec.topk_group,
                              group_score_topn=spec.group_score_topn, renormalize=spec.renormalize,
                              scaling_factor=spec.scaling_factor, bias=bias)
    sp = {"k": k, "E": E, "tile": spec.tile_tokens_dim, "n_group": spec.n_group, "topk_group": spec.topk_group,
          "local_expert_offset": spec.local_expert_offset, "local_num_experts": spec.local_num_experts}
    rep = compare_route(sp, gpu, orc)
    return rep, gpu, (p, lg_d, b_d, ws, views)


def test_tiny_softmax_workload():
    rep, _, _ = run_route(W.TINY_SOFTMAX)
    assert rep["flips"] == 0


def test_dsv3_grouped_sigmoid_full_size():
    rep, gpu, _ = run_route(W.DSV3_GROUPED_SIGMOID)
    print("dsv3 grouped sigmoid:", rep)


def test_mixtral_route_full_size():
    rep, _, _ = run_route(W.MIXTRAL_ROUTE)
    print("mixtral route:", rep)


EDGE = []
for T in (1, 31, 33, 4097):
    EDGE.append(W.RouteSpec(T=T, E=8, k=2, tile_tokens_dim=4, seed=T))
    EDGE.append(W.RouteSpec(T=T, E=256, k=8, score_fn=W.SIGMOID, n_group=8, topk_group=4, renormalize=1,
                            scaling_factor=2.5, tile_tokens_dim=128, logits_dtype=W.BF16, weights_dtype=W.BF16,
                            has_bias=True, logit_std=2.0, seed=T + 1))
for E, k in ((4, 1), (16, 6), (64, 8), (72, 6), (128, 8), (160, 6), (384, 8), (1024, 32), (33, 2), (100, 3)):
    EDGE.append(W.RouteSpec(T=257, E=E, k=k, tile_tokens_dim=8, seed=E))
    EDGE.append(W.RouteSpec(T=257, E=E, k=k, score_fn=W.SIGMOID, has_bias=True, renormalize=0,
                            scaling_factor=1.5, tile_tokens_dim=1, seed=E + 7))
    EDGE.append(W.RouteSpec(T=129, E=E, k=k, softmax_before_topk=0, renormalize=0, logits_dtype=W.BF16,
                            tile_tokens_dim=4, seed=E + 9))
for E, ng, tg, k in ((64, 8, 4, 8), (128, 4, 2, 6), (160, 8, 3, 6), (256, 16, 4, 8), (16, 4, 2, 3), (384, 8, 3, 8),
                     (64, 32, 8, 4), (256, 8, 8, 8)):
    EDGE.append(W.RouteSpec(T=300, E=E, k=k, score_fn=W.SIGMOID, n_group=ng, topk_group=tg, has_bias=True,
                            logits_dtype=W.BF16, logit_std=2.0, tile_tokens_dim=8, seed=E + ng))
    EDGE.append(W.RouteSpec(T=300, E=E, k=k, score_fn=W.SOFTMAX, n_group=ng, topk_group=tg, group_score_topn=1,
                            tile_tokens_dim=16, seed=E + ng + 1))


@pytest.mark.parametrize("spec", EDGE, ids=lambda s: f"T{s.T}-E{s.E}-k{s.k}-sf{s.score_fn}-pre{s.softmax_before_topk}"
                         f"-g{s.n_group}.{s.topk_group}-tile{s.tile_tokens_dim}-dt{s.logits_dtype}")
def test_route_edge_sweep(spec):
    run_route(spec)


def test_all_equal_logits_tie_break():
    spec = W.RouteSpec(T=64, E=256, k=8, score_fn=W.SIGMOID, n_group=8, topk_group=4, tile_tokens_dim=8,
                       logits_dtype=W.BF16, weights_dtype=W.BF16)
    lg = torch.full((64, 256), 0.5).to(torch.bfloat16)
    rep, gpu, _ = run_route(spec, lg, None)
    assert rep["flips"] == 0
    assert to_np(gpu["ids"]).tolist() == [list(range(8))] * 64
    spec = W.RouteSpec(T=40, E=8, k=3, tile_tokens_dim=4)
    rep, gpu, _ = run_route(spec, torch.zeros(40, 8), None)
    assert to_np(gpu["ids"]).tolist() == [[0, 1, 2]] * 40


def test_bf16_logits_with_many_exact_ties():
    g = torch.Generator().manual_seed(9)
    lg = torch.randint(-3, 4, (500, 128), generator=g).float().to(torch.bfloat16)
    spec = W.RouteSpec(T=500, E=128, k=8, score_fn=W.SOFTMAX, tile_tokens_dim=8, logits_dtype=W.BF16)
    rep, _, _ = run_route(spec, lg, None)
    assert rep["flips"] == 0


def test_hot_expert_skew_and_empty_experts():
    spec = W.RouteSpec(T=4000, E=64, k=4, score_fn=W.SIGMOID, has_bias=True, tile_tokens_dim=128, seed=5)
    inp = W.route_inputs(spec)
    bias = inp["bias"].clone()
    bias[17] = 5.0     # every token picks expert 17
    bias[40:] = -5.0   # experts 40.. are never picked
    rep, gpu, _ = run_route(spec, inp["logits"], bias)
    counts = to_np(gpu["counts"])
    assert counts[17] == 4000 and counts[40:].sum() == 0


def test_grouped_all_kept_equals_ungrouped_on_gpu():
    base = W.DSV3_GROUPED_SIGMOID.with_(T=2048)
    _, a, _ = run_route(base.with_(topk_group=8))
    _, b, _ = run_route(base.with_(n_group=0, topk_group=0))
    assert torch.equal(a["ids"].cpu(), b["ids"].cpu()) and torch.equal(a["weights"].cpu(), b["weights"].cpu())


def test_repeated_calls_are_deterministic():
    spec = W.DSV3_GROUPED_SIGMOID
    _, gpu, (p, lg, b, ws, views) = run_route(spec)
    first = {n: v.clone() for n, v in views.items()}
    other = W.route_inputs(spec.with_(seed=77))
    B.route_into(p, other["logits"].cuda(), other["bias"].cuda(), views, ws)
    for _ in range(3):
        B.route_into(p, lg, b, views, ws)
    torch.cuda.synchronize()
    for n in first:
        assert torch.equal(first[n], views[n]), n


def test_one_workspace_across_shapes_and_paths():
    """One workspace reused by calls of different shapes, in both count-table
    formats (byte counts: tagged rows, no grid barrier; wider counts: the grid
    barrier), must give what a fresh workspace gives, call after call."""
    big = B.route_params(16384, 256, 8)
    ws = B.make_workspace(max(B.route_workspace_bytes(big),
                              B.route_workspace_bytes(B.route_params(65536, 8, 2))), "cuda")
    seq = [W.DSV3_GROUPED_SIGMOID, W.DSV3_GROUPED_SIGMOID.with_(T=3000, seed=5), W.MIXTRAL_ROUTE,
           W.DSV3_GROUPED_SIGMOID.with_(seed=6), W.DSV3_GROUPED_SIGMOID.with_(T=500, seed=7),
           W.DSV3_GROUPED_SIGMOID.with_(seed=6), W.MIXTRAL_ROUTE.with_(T=20000, seed=8)]
    for spec in seq:
        inp = W.route_inputs(spec)
        kw = dict(score_fn=spec.score_fn, n_group=spec.n_group, topk_group=spec.topk_group,
                  group_score_topn=spec.group_score_topn, renormalize=spec.renormalize,
                  softmax_before_topk=spec.softmax_before_topk, scaling_factor=spec.scaling_factor,
                  tile_tokens_dim=spec.tile_tokens_dim, logits_dtype=spec.logits_dtype, bias_dtype=spec.bias_dtype,
                  weights_dtype=spec.weights_dtype)
        p = B.route_params(spec.T, spec.E, spec.k, **kw)
        lg = inp["logits"].cuda()
        b = inp["bias"].cuda() if inp["bias"] is not None else None
        fresh = B.Router(p)
        ref = fresh(lg, b)
        shared = B.Router(p)
        B.route_into(p, lg, b, shared.out, ws)
        torch.cuda.synchronize()
        assert B.status(ws) == B.MOE_OK and B.status(fresh.ws) == B.MOE_OK
        P = int(ref["totals"][0])
        for n in ("ids", "weights", "counts", "offsets", "e2p", "totals"):
            assert torch.equal(ref[n], shared.out[n]), (spec, n)
        assert torch.equal(ref["p2t"][:P], shared.out["p2t"][:P]), spec


def test_zero_tokens():
    p = B.route_params(0, 16, 2, tile_tokens_dim=4)
    dev = torch.device("cuda")
    views = {"ids": None, "weights": None, "e2p": None, "p2t": None, "tile_expert": None, "tile_mn_limit": None,
             "counts": torch.full((16,), 5, dtype=torch.int32, device=dev),
             "offsets": torch.full((17,), 5, dtype=torch.int32, device=dev),
             "totals": torch.full((2,), 5, dtype=torch.int32, device=dev)}
    ws = B.make_workspace(B.route_workspace_bytes(p), dev)
    B.route_into(p, torch.empty(0, 16, device=dev), None, views, ws)
    torch.cuda.synchronize()
    assert views["counts"].sum().item() == 0 and views["offsets"].sum().item() == 0
    assert views["totals"].tolist() == [0, 0]


def test_bounded_wait_times_out_cleanly():
    """A bounded wait on a barrier that nothing completes (the kind of wait the kernels use for their
    bulk copies) gives up after its limit and records a timeout in the status word; the context stays
    usable and a wait that completes records nothing."""
    dev = torch.device("cuda")
    ws = B.make_workspace(64, dev)
    B.debug_wait_timeout(True, 20_000_000, ws)
    torch.cuda.synchronize()
    assert B.status(ws, clear=True) == B.MOE_ERR_DEVICE_TIMEOUT
    assert B.status(ws) == B.MOE_OK
    B.debug_wait_timeout(False, 20_000_000, ws)
    torch.cuda.synchronize()
    assert B.status(ws) == B.MOE_OK
    run_route(W.TINY_SOFTMAX)


def test_sigmoid_proxy_error_bound_exhaustive_bf16():
    """The fast path's half-precision proxy key 0.5 tanh(x/2) + (0.5 + b) is within the error bound it
    assumes of the exact fp32 key sigmoid(x) + b, for every finite bf16 logit under a sweep of biases
    (small ones like the grouped workload's, and large ones where f16 rounding grows); and for fp32
    logits (rounded to f16 first) at every f16 input of the tanh and on random inputs."""
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16).float()
    x = x[torch.isfinite(x)]
    biases = [float(v) for v in torch.linspace(-0.1, 0.1, 11)] + [-0.5, -0.49, 0.3, 0.7, -1.0, 1.0, -3.0, 3.0,
                                                                  10.0, -10.0, 100.0, 700.0]
    worst = 0.0
    for b in biases:
        err, delta = B.debug_sigmoid_proxy_error(x.cuda(), torch.full_like(x, b).cuda())
        ratio = (err.abs() / delta).max().item()
        worst = max(worst, ratio)
        assert ratio <= 1.0, f"bias {b}: |proxy - key| reaches {ratio:.3f} of the assumed bound"
    # fp32 logits: x = 2h for every finite f16 h reaches tanh.approx.f16 at every input it can see, plus
    # random fp32 logits (rounded to f16 first)
    h = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.float16).float()
    h = h[torch.isfinite(h)]
    g = torch.Generator().manual_seed(0)
    xf = torch.cat([2.0 * h, torch.randn(1 << 20, generator=g) * 8, torch.rand(1 << 20, generator=g) * 60 - 30])
    worst32 = 0.0
    for b in (-0.1, 0.0, 0.07, 0.5, -2.0, 30.0):
        err, delta = B.debug_sigmoid_proxy_error(xf.cuda(), torch.full_like(xf, b).cuda(), f32_logits=True)
        ratio = (err.abs() / delta).max().item()
        worst32 = max(worst32, ratio)
        assert ratio <= 1.0, f"fp32 logits, bias {b}: |proxy - key| reaches {ratio:.3f} of the assumed bound"
    print("worst |proxy - key| / bound: bf16", worst, "fp32", worst32)


def test_fast_path_group_ties_and_fallbacks():
    """Sigmoid fast path: exactly tied groups (slow path, lower group wins), k = 16 with 4 kept groups
    (candidate bound unavailable -> slow path), k = 1, and fp32 logits."""
    base = W.DSV3_GROUPED_SIGMOID.with_(T=1024, seed=21)
    inp = W.route_inputs(base)
    lg = inp["logits"].clone()
    lg[:, 3 * 32:4 * 32] = lg[:, 5 * 32:6 * 32]  # groups 3 and 5 identical logits
    bias = inp["bias"].clone()
    bias[3 * 32:4 * 32] = bias[5 * 32:6 * 32]
    run_route(base, lg, bias)
    run_route(base.with_(k=16, seed=22))
    run_route(base.with_(k=1, seed=23))
    run_route(base.with_(logits_dtype=W.F32, E=128, n_group=8, topk_group=3, k=6, seed=24))
    run_route(base.with_(n_group=0, topk_group=0, k=8, seed=25))
    # saturated sigmoids: many keys equal 1 + bias exactly
    run_route(base.with_(logit_std=40.0, seed=26))


def _weights_bwd_magnitude(lg64, ids, G, score_fn, pre, renorm, scale):
    """Error scale for the routed-weight backward: the same chain with every difference replaced by a
    sum of magnitudes (the terms before cancellation), float64."""
    T, E = lg64.shape
    k = ids.shape[1]
    mag = np.zeros((T, E))
    for t in range(T):
        x = lg64[t]
        if score_fn == W.SIGMOID:
            v = 1.0 / (1.0 + np.exp(-x[ids[t]]))
        elif pre:
            z = np.exp(x - x.max()); p = z / z.sum(); v = p[ids[t]]
        else:
            z = np.exp(x[ids[t]] - x[ids[t]].max()); v = z / z.sum()
        g = np.abs(G[t].astype(np.float64))
        gv = scale / v.sum() * (g + (g * v).sum() / v.sum()) if renorm else scale * g
        D = (v * gv).sum()
        if score_fn == W.SIGMOID:
            mag[t, ids[t]] = gv * v * (1 - v)
        elif pre:
            gp = np.zeros(E); gp[ids[t]] = gv
            mag[t] = p * (gp + D)
        else:
            mag[t, ids[t]] = v * (gv + D)
    return mag


@pytest.mark.parametrize("score_fn,pre,renorm,dtype,E,k", [
    (W.SIGMOID, 1, 1, W.BF16, 256, 8), (W.SIGMOID, 1, 0, W.F32, 64, 6), (W.SOFTMAX, 1, 1, W.F32, 128, 8),
    (W.SOFTMAX, 1, 0, W.BF16, 96, 4), (W.SOFTMAX, 0, 1, W.BF16, 8, 2), (W.SOFTMAX, 0, 0, W.F32, 33, 3),
    (W.SIGMOID, 1, 1, W.F32, 1024, 32)])
def test_route_weights_backward(score_fn, pre, renorm, dtype, E, k):
    """moe_route_weights_bwd against the oracle, relative to the terms before cancellation."""
    T, scale = 777, 2.5
    g = torch.Generator().manual_seed(E + k + 10 * pre + renorm)
    lg = torch.randn(T, E, generator=g) * 1.5
    lg = lg.to(torch.bfloat16) if dtype == W.BF16 else lg
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    G = torch.randn(T, k, generator=g)
    p = B.route_params(T, E, k, score_fn=score_fn, softmax_before_topk=pre, renormalize=renorm,
                       scaling_factor=scale, logits_dtype=dtype)
    ws = B.make_workspace(64, "cuda")
    got = to_np(B.route_weights_bwd(p, lg.cuda(), ids.cuda(), G.cuda(), ws=ws))
    torch.cuda.synchronize()
    assert B.status(ws) == B.MOE_OK
    lg32 = lg.float().numpy()
    ref = oracle.route_weights_bwd(lg32, ids.numpy(), G.numpy(), score_fn=score_fn, softmax_before_topk=pre,
                                   renormalize=renorm, scaling_factor=scale)
    mag = _weights_bwd_magnitude(lg32.astype(np.float64), ids.numpy(), G.numpy(), score_fn, pre, renorm, scale)
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= 1e-5 * mag + 1e-30), f"err/mag max {np.max(err / (mag + 1e-30))}"


def test_route_weights_backward_bad_id_recorded():
    """An id outside [0, E) is caught by the kernel's bounds check (clamped, status set)."""
    p = B.route_params(4, 16, 2, score_fn=W.SIGMOID)
    lg = torch.randn(4, 16, device="cuda")
    ids = torch.tensor([[0, 1], [2, 3], [4, 16], [5, 6]], dtype=torch.int32, device="cuda")
    ws = B.make_workspace(64, "cuda")
    B.route_weights_bwd(p, lg, ids, torch.ones(4, 2, device="cuda"), ws=ws)
    torch.cuda.synchronize()
    assert B.status(ws) == B.MOE_ERR_DEVICE_BOUNDS


# expert-parallel shards: selection global, bookkeeping of the local experts only
@pytest.mark.parametrize("spec", [
    W.DSV3_GROUPED_SIGMOID.with_(T=4096, local_expert_offset=64, local_num_experts=64),
    W.DSV3_GROUPED_SIGMOID.with_(T=777, local_expert_offset=0, local_num_experts=32),
    W.DSV3_GROUPED_SIGMOID.with_(T=777, local_expert_offset=255, local_num_experts=1),
    W.RouteSpec(T=5000, E=8, k=2, softmax_before_topk=0, renormalize=0, logits_dtype=W.BF16, tile_tokens_dim=128,
                local_expert_offset=2, local_num_experts=4, seed=3),
    W.RouteSpec(T=300, E=160, k=6, score_fn=W.SOFTMAX, n_group=8, topk_group=3, tile_tokens_dim=8,
                local_expert_offset=40, local_num_experts=40, seed=11),
    W.RouteSpec(T=129, E=16, k=3, tile_tokens_dim=4, local_expert_offset=5, local_num_experts=7, seed=12),
], ids=lambda s: f"T{s.T}-E{s.E}-local{s.local_expert_offset}+{s.local_num_experts}")
def test_route_expert_parallel_shard(spec):
    rep, gpu, _ = run_route(spec)
    e2p = to_np(gpu["e2p"]).reshape(spec.T, spec.k)
    ids = to_np(gpu["ids"])
    loc = (ids >= spec.local_expert_offset) & (ids < spec.local_expert_offset + spec.local_num_experts)
    assert np.all(e2p[~loc] == -1) and np.all(e2p[loc] >= 0)
    print(rep)


def test_route_expert_parallel_shard_bad_range():
    for off, nl in ((-1, 4), (6, 4), (3, -2), (2, 0)):
        p = B.route_params(16, 8, 2, local_expert_offset=off, local_num_experts=nl)
        with pytest.raises(B.MoeError):
            B.Router(p)(torch.randn(16, 8, device="cuda"))


@pytest.mark.parametrize("name,S,off,nl", [("dsv3", 1, 0, 0), ("dsv3", 2, 64, 64), ("mixtral", 2, 0, 0),
                                           ("e64", 1, 16, 16), ("e64", 3, 0, 0)])
def test_route_fused_shared_experts(name, S, off, nl):
    """num_fused_shared_experts (trtllm_gen_routing, Parameters): the routed slots equal the plain route's,
    each token's S appended slots hold experts E .. E+S-1 with weight 1.0, and the whole bookkeeping
    (routed local experts, then the shared ones) equals the oracle's on the GPU's ids, bit-exactly."""
    if name == "dsv3":
        spec = W.DSV3_GROUPED_SIGMOID.with_(T=3000, seed=77)
    elif name == "mixtral":
        spec = W.MIXTRAL_ROUTE.with_(T=999, seed=78)
    else:
        spec = W.RouteSpec(T=777, E=64, k=6, score_fn=W.SOFTMAX, softmax_before_topk=1, n_group=0, topk_group=0,
                           group_score_topn=2, renormalize=1, scaling_factor=1.0, tile_tokens_dim=16,
                           logits_dtype=W.F32, bias_dtype=W.F32, weights_dtype=W.F32, seed=79)
    inp = W.route_inputs(spec)
    kw = dict(score_fn=spec.score_fn, softmax_before_topk=spec.softmax_before_topk, n_group=spec.n_group,
              topk_group=spec.topk_group, group_score_topn=spec.group_score_topn, renormalize=spec.renormalize,
              scaling_factor=spec.scaling_factor, tile_tokens_dim=spec.tile_tokens_dim,
              logits_dtype=spec.logits_dtype, bias_dtype=spec.bias_dtype, weights_dtype=spec.weights_dtype,
              local_expert_offset=off, local_num_experts=nl)
    lg = inp["logits"].cuda()
    b = inp["bias"].cuda() if inp["bias"] is not None else None
    plain = B.Router(B.route_params(spec.T, spec.E, spec.k, **kw))(lg, b)
    plain = {n: v.clone() for n, v in plain.items()}
    r = B.Router(B.route_params(spec.T, spec.E, spec.k, num_fused_shared_experts=S, **kw))
    got = r(lg, b)
    torch.cuda.synchronize()
    assert B.status(r.ws) == B.MOE_OK
    k, E, T = spec.k, spec.E, spec.T
    ids = to_np(got["ids"]).reshape(T, k + S)
    w = got["weights"].float().cpu().numpy().reshape(T, k + S)
    assert np.array_equal(ids[:, :k], to_np(plain["ids"]).reshape(T, k))
    assert np.array_equal(w[:, :k], plain["weights"].float().cpu().numpy().reshape(T, k))
    assert np.all(ids[:, k:] == np.arange(E, E + S)) and np.all(w[:, k:] == 1.0)
    bk = oracle.route_bookkeeping(ids, E, spec.tile_tokens_dim, off, nl or E, num_shared=S)
    P, nt = int(bk["totals"][0]), int(bk["totals"][1])
    assert to_np(got["totals"]).tolist() == [P, nt]
    for name_, n in (("counts", (nl or E) + S), ("offsets", (nl or E) + S + 1), ("e2p", T * (k + S)),
                     ("p2t", P), ("tile_expert", nt), ("tile_mn_limit", nt)):
        assert np.array_equal(to_np(got[name_])[:n], bk[name_][:n]), f"{name_} differs from the oracle"
