"""GPU parity of moe_dispatch and moe_combine against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from parity import bf16_ulp_dist, to_np
from top_expert_selection_b200 import binding as B
from top_expert_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu
FILL = 0x7FBF  # bf16 NaN pattern marking rows that must stay untouched


def route_for(T, E, k, logits, tile, post=True):
    p = B.route_params(T, E, k, score_fn=W.SOFTMAX, softmax_before_topk=0 if post else 1, renormalize=0,
                       tile_tokens_dim=tile, logits_dtype=B._DT[logits.dtype], weights_dtype=W.F32)
    r = B.Router(p)
    out = r(logits.cuda())
    torch.cuda.synchronize()
    # the permutation must already be bit-exact with the oracle on the GPU's ids
    bk = oracle.route_bookkeeping(to_np(out["ids"]), E, tile)
    assert np.array_equal(to_np(out["e2p"]), bk["e2p"])
    return r, out, bk


def run_dispatch_combine(T, H, E, k, tile, dtype=torch.bfloat16, wdtype=torch.float32, seed=0, full=False):
    g = torch.Generator().manual_seed(seed)
    if full:
        inp = W.mixtral_inputs()
        logits, hidden, rows = inp["logits"], inp["hidden"], inp["expert_rows"]
    else:
        logits = torch.randn(T, E, generator=g).to(torch.bfloat16)
        hidden = torch.randn(T, H, generator=g).to(dtype)
        rows = torch.randn(T * k, H, generator=g).to(dtype)
    r, out, bk = route_for(T, E, k, logits, tile)
    P = int(bk["totals"][0])
    maxp = r.max_padded
    # ---- dispatch ----
    dev_out = torch.empty((maxp, H), dtype=dtype, device="cuda")
    if dtype == torch.bfloat16:
        dev_out.view(torch.int16).fill_(FILL)
    else:
        dev_out.view(torch.int32).fill_(0x7FC00001)
    hid_d = hidden.cuda()
    B.dispatch_into(hid_d, out["e2p"], out["p2t"], out["totals"], k, dev_out)
    torch.cuda.synchronize()
    got = to_np(dev_out)
    if dtype == torch.bfloat16:
        ref = oracle.dispatch(hidden, bk["e2p"], bk["p2t"], P, maxp, fill=FILL)
        assert np.array_equal(got, ref), "dispatch differs from the oracle (bit-exact copy expected)"
    else:
        h32 = hidden.numpy()
        assert np.array_equal(got[bk["e2p"]], np.repeat(h32, k, axis=0))
        pad = np.nonzero(bk["p2t"] < 0)[0]
        assert np.all(got[pad] == 0)
        assert np.all(got[P:].view(np.int32) == 0x7FC00001)
    # ---- combine: expert rows in permuted order, padding rows NaN (must never be read) ----
    eo = W.place_expert_rows(rows, torch.from_numpy(bk["p2t"]), P, maxp)
    w = out["weights"] if wdtype == torch.float32 else out["weights"].to(torch.bfloat16)
    res = torch.empty((T, H), dtype=dtype, device="cuda")
    ws = B.make_workspace(64, "cuda")
    B.combine_into(eo.cuda(), out["e2p"], w.contiguous(), k, res, ws=ws)
    torch.cuda.synchronize()
    assert B.status(ws) == B.MOE_OK
    got = to_np(res)
    assert np.all(np.isfinite(res.float().cpu().numpy())), "combine read a padding row"
    ref = oracle.combine(eo, bk["e2p"], to_np(w), k)
    if dtype == torch.bfloat16:
        d = bf16_ulp_dist(got, ref)
        assert d.max() <= 1, f"combine off by {d.max()} bf16 ulp"
        return int((d > 0).sum())
    # fp32 rows: the same slot-order fp32 sum, compared within 1e-5 of the terms before cancellation
    ew = np.abs(np.asarray(to_np(w), np.float64)).reshape(T, k)
    mag = np.zeros((T, H))
    for j in range(k):
        p = bk["e2p"].reshape(T, k)[:, j]
        v = p >= 0
        mag[v] += ew[v, j:j + 1] * np.abs(eo.numpy()[p[v]].astype(np.float64))
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= 1e-5 * mag), f"fp32 combine off by {(err / np.maximum(mag, 1e-30)).max()} (relative)"
    return int((got != ref).sum())


def test_mixtral_dispatch_combine_full_size():
    n1 = run_dispatch_combine(65536, W.MIXTRAL_HIDDEN, 8, 2, 128, full=True)
    print("combine elements 1 ulp from the oracle:", n1)


@pytest.mark.parametrize("T,H,E,k,tile", [(1, 8, 4, 1, 1), (33, 64, 8, 2, 4), (1000, 4096, 8, 2, 128),
                                          (257, 7168, 16, 8, 8), (500, 128, 64, 6, 16), (77, 24, 8, 3, 2)])
def test_dispatch_combine_shapes(T, H, E, k, tile):
    run_dispatch_combine(T, H, E, k, tile, seed=T + H)


def test_dispatch_combine_fp32_and_bf16_weights():
    n = run_dispatch_combine(300, 256, 8, 2, 8, dtype=torch.float32, seed=5)
    assert n == 0, f"{n} fp32 combine elements differ from the oracle's fp32 sum"
    run_dispatch_combine(300, 256, 8, 2, 8, wdtype=torch.bfloat16, seed=6)


def test_combine_fp32_mixtral_shape():
    # fp32 rows at a Mixtral-like shape (several tiles, a ragged tail): T=4099, H=4096, top-2 of 8
    n = run_dispatch_combine(4099, 4096, 8, 2, 128, dtype=torch.float32, seed=9)
    assert n == 0


def test_combine_skips_rows_past_the_buffer():
    # a stale map pointing past expert_out is skipped and recorded, never read
    T, H, k = 64, 64, 2
    eo = torch.randn(16, H, device="cuda")
    e2p = torch.tensor([[j % 16, 16 + j] if j % 3 == 0 else [j % 16, (j + 1) % 16] for j in range(T)],
                       dtype=torch.int32, device="cuda").reshape(-1)
    w = torch.ones(T, k, device="cuda")
    res = torch.empty(T, H, device="cuda")
    ws = B.make_workspace(64, "cuda")
    B.combine_into(eo, e2p, w, k, res, ws=ws)
    torch.cuda.synchronize()
    assert B.status(ws) == B.MOE_ERR_DEVICE_BOUNDS
    ref = oracle.combine(eo.cpu().numpy(), np.where(to_np(e2p) >= 16, -1, to_np(e2p)), w.cpu().numpy(), k)
    assert np.array_equal(to_np(res), ref)


@pytest.mark.parametrize("off,nl", [(2, 4), (0, 1), (7, 1)])
def test_dispatch_combine_expert_parallel_shard(off, nl):
    # one shard's route -> dispatch -> combine: only the local experts' rows are moved and summed;
    # the other shards' selections (expanded_to_permuted = -1) contribute nothing here
    T, H, E, k, tile = 700, 256, 8, 2, 16
    g = torch.Generator().manual_seed(off * 10 + nl)
    logits = torch.randn(T, E, generator=g).to(torch.bfloat16)
    hidden = torch.randn(T, H, generator=g).to(torch.bfloat16)
    p = B.route_params(T, E, k, score_fn=W.SOFTMAX, softmax_before_topk=0, renormalize=0, tile_tokens_dim=tile,
                       logits_dtype=W.BF16, weights_dtype=W.F32, local_expert_offset=off, local_num_experts=nl)
    r = B.Router(p)
    out = r(logits.cuda())
    torch.cuda.synchronize()
    bk = oracle.route_bookkeeping(to_np(out["ids"]), E, tile, off, nl)
    assert np.array_equal(to_np(out["e2p"]), bk["e2p"])
    P, maxp = int(bk["totals"][0]), r.max_padded
    dev_out = torch.empty((maxp, H), dtype=torch.bfloat16, device="cuda")
    dev_out.view(torch.int16).fill_(FILL)
    B.dispatch_into(hidden.cuda(), out["e2p"], out["p2t"], out["totals"], k, dev_out)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(dev_out), oracle.dispatch(hidden, bk["e2p"], bk["p2t"], P, maxp, fill=FILL))
    rows = torch.randn(int((bk["e2p"] >= 0).sum()), H, generator=g).to(torch.bfloat16)
    eo = W.place_expert_rows(rows, torch.from_numpy(bk["p2t"]), P, maxp)
    res = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    B.combine_into(eo.cuda(), out["e2p"], out["weights"].contiguous(), k, res)
    torch.cuda.synchronize()
    ref = oracle.combine(eo, bk["e2p"], to_np(out["weights"]), k)
    assert bf16_ulp_dist(to_np(res), ref).max() <= 1
