"""Comparison rules between the CUDA path and the CPU oracle.

* ids: compared position-wise.  A token whose ids differ is accepted only as a
  near tie: every position must carry an oracle key within 2 fp32 ulp of the
  oracle's own choice at that position, after allowing the kept-group set to
  differ only in groups whose oracle group scores lie within 2 ulp of the
  group cut.  Accepted tokens are counted and reported.
* bookkeeping (counts, offsets, maps, tile tables, totals): bit-exact against
  the oracle's bookkeeping re-run on the GPU's ids, and against the oracle from
  scratch whenever no token flipped.
* fp32 weights: |d| <= 1e-5 |ref|; bf16 weights: <= 1 bf16 ulp of the oracle's
  fp32 weight rounded to bf16.
"""
from __future__ import annotations

import itertools

import numpy as np
import torch

import oracle

ULP_TOL = 2
F32_RTOL = 1e-5


def ordered(x: np.ndarray) -> np.ndarray:
    """fp32 -> int64 whose order is the float order (adjacent floats differ by 1)."""
    u = np.asarray(x, np.float32).view(np.int32).astype(np.int64)
    return np.where(u < 0, -(u & 0x7FFFFFFF), u)


def ulp_dist(a, b) -> np.ndarray:
    return np.abs(ordered(a) - ordered(b))


def bf16_ulp_dist(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    def o(x):
        x = np.asarray(x, np.uint16).astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(o(a_bits) - o(b_bits))


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _topk_over(keys: np.ndarray, allowed: np.ndarray, k: int):
    idx = np.nonzero(allowed)[0]
    order = sorted(idx.tolist(), key=lambda e: (-float(keys[e]), e))
    return order[:k]


def near_tie_ok(keys: np.ndarray, gpu_ids, orc_ids, k: int, grouped: bool, n_group: int, topk_group: int,
                gscores: np.ndarray | None) -> bool:
    """Is the GPU's selection for one token a valid top-k under the oracle keys, up to 2-ulp ties?"""
    E = keys.shape[0]
    candidates_sets = []
    if grouped:
        gs = E // n_group
        kept = min(topk_group, n_group)
        order = sorted(range(n_group), key=lambda g: (-float(gscores[g]), g))
        cut = gscores[order[kept - 1]]
        # groups clearly in, and groups within 2 ulp of the cut (ambiguous)
        amb = [g for g in range(n_group) if ulp_dist(gscores[g], cut) <= ULP_TOL]
        sure = [g for g in order[:kept] if g not in amb]
        need = kept - len(sure)
        for extra in itertools.combinations(amb, need):
            allowed = np.zeros(E, bool)
            for g in list(sure) + list(extra):
                allowed[g * gs:(g + 1) * gs] = True
            candidates_sets.append(allowed)
    else:
        candidates_sets.append(np.ones(E, bool))
    gpu_ids = list(map(int, gpu_ids))
    if len(set(gpu_ids)) != k:
        return False
    for allowed in candidates_sets:
        if not all(allowed[e] for e in gpu_ids):
            continue
        ref = _topk_over(keys, allowed, k)
        # position-wise: same key up to 2 ulp at every slot, and the set must be a valid top-k:
        # every unselected allowed expert's key may exceed a selected one by at most 2 ulp
        if all(ulp_dist(keys[a], keys[b]) <= ULP_TOL for a, b in zip(gpu_ids, ref)):
            sel = np.zeros(E, bool)
            sel[gpu_ids] = True
            rest = allowed & ~sel
            if not rest.any():
                return True
            worst_in = keys[gpu_ids].min()
            best_out = keys[rest].max()
            if best_out <= worst_in or ulp_dist(best_out, worst_in) <= ULP_TOL:
                return True
    return False


def compare_route(spec: dict, gpu: dict, orc: dict, *, max_flip_frac: float = 1e-3) -> dict:
    """Compare GPU routing outputs with the oracle's.  Returns a report dict; raises AssertionError."""
    k = spec["k"]
    E = spec["E"]
    tile = spec["tile"]
    grouped = spec.get("n_group", 0) > 1 and spec.get("topk_group", 0) > 0
    g_ids = to_np(gpu["ids"]).astype(np.int32)
    o_ids = orc["ids"]
    T = o_ids.shape[0]
    diff_rows = np.nonzero((g_ids != o_ids).any(1))[0]
    flips = []
    for t in diff_rows:
        ok = near_tie_ok(orc["keys"][t], g_ids[t], o_ids[t], k, grouped, spec.get("n_group", 0),
                         spec.get("topk_group", 0), orc["group_scores"][t] if grouped else None)
        assert ok, f"token {t}: gpu ids {g_ids[t].tolist()} vs oracle {o_ids[t].tolist()} is not a near tie"
        flips.append(int(t))
    assert len(flips) <= max(1, int(max_flip_frac * T)), f"too many near-tie flips: {len(flips)} of {T}"

    # weights on tokens whose ids agree
    same = np.ones(T, bool)
    same[flips] = False
    w = to_np(gpu["weights"])
    if w.dtype == np.uint16:
        ref = oracle.f32_to_bf16(orc["weights"][same]) if same.any() else np.zeros((0, k), np.uint16)
        d = bf16_ulp_dist(w[same], ref)
        assert d.max(initial=0) <= 1, f"bf16 weights off by {d.max()} ulp"
    else:
        ref = orc["weights"][same]
        err = np.abs(w[same].astype(np.float64) - ref) - F32_RTOL * np.abs(ref)
        assert err.max(initial=-1) <= 0, f"fp32 weights rel err {np.max(np.abs(w[same] - ref) / np.abs(ref))}"

    # bookkeeping (of the local experts, all E by default): bit-exact vs the oracle re-run on the GPU's ids
    off = spec.get("local_expert_offset", 0)
    nl = spec.get("local_num_experts", 0) or E
    bk = oracle.route_bookkeeping(g_ids, E, tile, off, nl)
    P, nt = int(bk["totals"][0]), int(bk["totals"][1])
    got_totals = to_np(gpu["totals"]).tolist()
    assert got_totals == [P, nt], f"totals {got_totals} vs {[P, nt]}"
    for name, n in (("counts", nl), ("offsets", nl + 1), ("e2p", T * k), ("p2t", P), ("tile_expert", nt),
                    ("tile_mn_limit", nt)):
        got = to_np(gpu[name])[:n]
        assert np.array_equal(got, bk[name][:n]), f"{name} differs from the oracle on the GPU's ids"
    if not flips:
        bk0 = oracle.route_bookkeeping(o_ids, E, tile, off, nl)
        assert np.array_equal(bk0["e2p"], bk["e2p"]) and np.array_equal(bk0["p2t"], bk["p2t"])
    return {"tokens": T, "flips": len(flips), "flip_tokens": flips[:10], "P": P, "tiles": nt}
