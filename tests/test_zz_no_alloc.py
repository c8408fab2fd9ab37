"""moe_route_no_alloc: the allocation-free variant of moe_route for callers that cannot allocate device
memory (a serving runtime whose memory manager owns the GPU, a plugin interface that provides no workspace,
a plain C caller without a device allocator).  Its workspace is a static array inside the library; this
checks, through the C ABI, that two calls in a row give exactly what moe_route gives on the same inputs,
and that the static workspace's status word reports a recorded device-side error instead of losing it.

Collected last (file name) so that a run stopping at the first failure has run every other test first."""
import pytest
import torch

from top_expert_selection_b200 import binding as B
from top_expert_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu

NAMES = ("ids", "weights", "counts", "offsets", "e2p", "p2t", "tile_expert", "tile_mn_limit", "totals")


def _params(spec):
    return B.route_params(spec.T, spec.E, spec.k, score_fn=spec.score_fn, softmax_before_topk=spec.softmax_before_topk,
                          n_group=spec.n_group, topk_group=spec.topk_group, group_score_topn=spec.group_score_topn,
                          renormalize=spec.renormalize, scaling_factor=spec.scaling_factor,
                          tile_tokens_dim=spec.tile_tokens_dim, logits_dtype=spec.logits_dtype,
                          bias_dtype=spec.bias_dtype, weights_dtype=spec.weights_dtype)


def test_no_alloc_route_matches_route_on_two_calls_in_a_row():
    for spec in (W.DSV3_GROUPED_SIGMOID.with_(seed=41), W.DSV3_GROUPED_SIGMOID.with_(seed=42),
                 W.MIXTRAL_ROUTE.with_(T=4097, seed=43), W.TINY_SOFTMAX):
        p = _params(spec)
        inp = W.route_inputs(spec)
        lg = inp["logits"].cuda()
        b = inp["bias"].cuda() if inp["bias"] is not None else None
        ref = B.Router(p)(lg, b)
        got = {n: torch.full_like(v, -7) for n, v in ref.items()}
        B.route_no_alloc_into(p, lg, b, got)
        torch.cuda.synchronize()
        P, nt = ref["totals"].tolist()
        limits = {"p2t": P, "tile_expert": nt, "tile_mn_limit": nt}
        for n in NAMES:
            lim = limits.get(n)
            a_ = ref[n] if lim is None else ref[n][:lim]
            g_ = got[n] if lim is None else got[n][:lim]
            # deterministic kernels: identical results (stricter than the parity tolerances)
            assert torch.equal(a_, g_), f"{n} differs between moe_route_no_alloc and moe_route"
        assert B.route_no_alloc_status() == B.MOE_OK


def test_no_alloc_route_rejects_a_workspace_it_cannot_hold():
    # 65536 tokens of 1024 experts: 256 segments of 256 tokens, 2-byte counts -> a 512 KB table plus the
    # header, past the static array (rejected before anything is launched)
    p = B.route_params(65536, 1024, 8, tile_tokens_dim=8)
    dev = torch.device("cuda")
    out = {n: torch.zeros(1 << 16, dtype=torch.int32, device=dev) for n in NAMES}
    with pytest.raises(B.MoeError) as ei:
        B.route_no_alloc_into(p, torch.zeros(64, 1024, device=dev), None, out)
    assert ei.value.code == B.MOE_ERR_WORKSPACE


def test_no_alloc_status_survives_the_next_call():
    # a device-side error recorded in the static workspace (here by the test hook, as a kernel's bounds
    # check would) is still there after another moe_route_no_alloc call, and clears when read with clear=1
    spec = W.TINY_SOFTMAX
    p = _params(spec)
    lg = W.route_inputs(spec)["logits"].cuda()
    ref = B.Router(p)(lg)
    got = {n: torch.empty_like(v) for n, v in ref.items()}
    assert B.route_no_alloc_status() == B.MOE_OK
    B._check(B.lib().moe_debug_no_alloc_record(B.MOE_ERR_DEVICE_BOUNDS, B._stream(None)), "record")
    B.route_no_alloc_into(p, lg, None, got)
    assert B.route_no_alloc_status(clear=False) == B.MOE_ERR_DEVICE_BOUNDS
    assert B.route_no_alloc_status(clear=True) == B.MOE_ERR_DEVICE_BOUNDS
    assert B.route_no_alloc_status() == B.MOE_OK
    B.route_no_alloc_into(p, lg, None, got)
    torch.cuda.synchronize()
    assert torch.equal(got["ids"], ref["ids"]) and B.route_no_alloc_status() == B.MOE_OK
