"""Parity harness: the CUDA path (through the C ABI) against the fp64 oracle.

Acceptance (the method's tolerances; where selections may differ, only
inside the 1e-6 tie band below):
* ``assign`` and ``counts`` bit-exact;
* ``vsum`` within 1e-5 of the per-codeword sum of |V| (fp32 accumulation);
* ``selected``: every parent whose normalised oracle score lies more than
  1e-6 above the P-th score is selected, none lying more than 1e-6 below it
  is, and consecutive entries never invert the oracle's order by more than
  1e-6; a tile whose GPU set differs from the oracle's (only possible inside
  the band) is counted as a tie-band tile and its outputs are compared with
  the oracle re-run on the GPU's selection;
* ``O`` max-abs error <= 2e-3 (fp32 inputs) or 2e-2 (bf16 inputs).
"""
from __future__ import annotations

import numpy as np
import torch

from adaptive_vector_quantized_avq_b200 import binding as bd
from adaptive_vector_quantized_avq_b200 import synthetic as syn

BAND = 1e-6
O_TOL = {"f32": 2e-3, "bf16": 2e-2}
VSUM_REL = 1e-5


def to_device(arr: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(arr.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def from_device(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return syn.bf16_bits_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.cpu().numpy()


def run_gpu(wl: syn.Workload, inp: syn.Inputs, Ps, device="cuda"):
    """Both calls through the C ABI; also checks the device status words
    (no timeout, no range flag) and returns the fp64 re-decision counters."""
    dt = wl.dtype
    K, V, Q, cb = (to_device(getattr(inp, n), dt, device) for n in ("K", "V", "Q", "codebook"))
    shape = bd.make_shape(wl.B, wl.H, wl.N, wl.d, wl.M0, wl.C, K.dtype)
    ws_pre = bd.workspace(bd.avq_precompute_workspace_bytes(shape), K.device)
    assign, counts, vsum = bd.precompute(K, V, cb, wl.M0, wl.C, ws=ws_pre)
    torch.cuda.synchronize()
    diag = ws_pre[:16].view(torch.int32).cpu().numpy()
    st = bd.avq_device_status(ws_pre)
    assert st == 0, f"precompute device status {st}"
    att = {}
    for P in Ps:
        ws_att = bd.workspace(bd.avq_attention_workspace_bytes(shape, P, wl.tile), K.device)
        O, sel = bd.attention(Q, cb, counts, vsum, wl.M0, wl.C, P, wl.tile, wl.softmax_scale, ws=ws_att)
        st = bd.avq_device_status(ws_att)
        assert st == 0, f"attention device status {st} (P={P})"
        att[P] = (O, sel)
    torch.cuda.synchronize()
    return {"assign": assign.cpu().numpy(), "counts": counts.cpu().numpy(),
            "vsum": vsum.cpu().numpy(), "redecided": (int(diag[2]), int(diag[3])),
            "att": {P: (from_device(O), sel.cpu().numpy()) for P, (O, sel) in att.items()}}


class Report(dict):
    pass


def check_precompute(wl, inp, gpu, ora, oracle) -> Report:
    rep = Report()
    bad = np.nonzero(gpu["assign"] != ora["assign"])
    assert bad[0].size == 0, f"{wl.name}: {bad[0].size} assignments differ, first at {[b[0] for b in bad]}: " \
                             f"gpu {gpu['assign'][tuple(b[0] for b in bad)]} oracle {ora['assign'][tuple(b[0] for b in bad)]}"
    assert np.array_equal(gpu["counts"], ora["counts"]), f"{wl.name}: counts differ"
    # per-codeword sum of |V| from the oracle itself (same assignment rule)
    absV = np.abs(inp.f64("V"))
    abs_sum = oracle.precompute(inp.f64("K"), absV, inp.f64("codebook"), wl.M0, wl.C)["vsum"]
    err = np.abs(gpu["vsum"] - ora["vsum"])
    lim = VSUM_REL * abs_sum + 1e-30
    worst = float((err / np.maximum(abs_sum, 1e-30)).max()) if err.size else 0.0
    assert np.all(err <= lim), f"{wl.name}: vsum error {worst:.3g} of sum|V| exceeds {VSUM_REL}"
    rep["vsum_rel_err"] = worst
    rep["fp64_redecided_parent_child"] = gpu.get("redecided")
    return rep


def check_selection(sel_gpu, sel_ora, score, P):
    """Returns True when the GPU set equals the oracle's; raises outside the band."""
    if P == 0:
        return True
    kth = np.sort(score)[::-1][P - 1]
    g = set(int(x) for x in sel_gpu)
    assert len(g) == P and all(0 <= x < score.size for x in g), f"invalid selection {sel_gpu}"
    sure_in = set(np.nonzero(score > kth + BAND)[0].tolist())
    sure_out = set(np.nonzero(score < kth - BAND)[0].tolist())
    assert sure_in <= g, f"selection misses {sorted(sure_in - g)} (scores {score[list(sure_in - g)]}, kth {kth})"
    assert not (g & sure_out), f"selection takes {sorted(g & sure_out)} below the band"
    for a, b in zip(sel_gpu[:-1], sel_gpu[1:]):
        assert score[a] >= score[b] - BAND, f"order inverted: {a} ({score[a]}) before {b} ({score[b]})"
    return g == set(int(x) for x in sel_ora)


def check_attention(wl, inp, P, gpu_O, gpu_sel, counts, vsum, oracle, tile_ids=None) -> Report:
    """Compare all tiles (tile_ids None) or the listed global tile ids."""
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    T = wl.tile
    ntiles = wl.ntiles
    Q = inp.f64("Q")
    cb = inp.f64("codebook")
    ids = np.arange(B * H * ntiles) if tile_ids is None else np.asarray(tile_ids)
    ora = oracle.attention(Q, cb, counts, vsum, wl.M0, wl.C, P, T, wl.softmax_scale, tile_ids=ids)
    gsel = gpu_sel.reshape(B * H * ntiles, P)[ids] if P > 0 else np.zeros((ids.size, 0), np.int32)
    band_tiles = []
    for j in range(ids.size):
        if not check_selection(gsel[j], ora["selected"][j], ora["score"][j], P):
            band_tiles.append(j)
    O_ref = ora["O"].copy()
    if band_tiles:
        forced = oracle.attention(Q, cb, counts, vsum, wl.M0, wl.C, P, T, wl.softmax_scale,
                                  tile_ids=ids[band_tiles], forced=gsel[band_tiles])
        O_ref[band_tiles] = forced["O"]
    # gather the GPU rows of the listed tiles
    Og = gpu_O.reshape(B * H, N, d)
    err = 0.0
    for j, g in enumerate(ids):
        bh, t = divmod(int(g), ntiles)
        r0, r1 = t * T, min(N, (t + 1) * T)
        e = np.abs(Og[bh, r0:r1] - O_ref[j, : r1 - r0]).max() if r1 > r0 else 0.0
        err = max(err, float(e))
    tol = O_TOL[wl.dtype]
    assert err <= tol, f"{wl.name} P={P}: O max-abs error {err:.3g} > {tol}"
    assert np.isfinite(Og).all(), "non-finite output"
    return Report(O_maxabs=err, tiles=int(ids.size), tie_band_tiles=len(band_tiles))


def check_deep(wl_name, dtype, gpu_assign, gpu_counts, gpu_vsum, gpu_O, gpu_sel, Q, K, V, cb, M0, C, L, Ps, T,
               scale) -> Report:
    """A depth-L tree on the GPU against oracle/deep.py (fp64 inputs Q, K, V,
    cb as stored): assignments and counts bit-exact, value sums within 1e-5 of
    the per-node sum of |V|, per tile and level the expanded set and order
    equal to the oracle's outside the 1e-6 band of normalised scores (a tile
    whose selection differs inside the band is counted and its output not
    compared, since every later step depends on the selection), and O within
    the tolerance of the dtype."""
    from oracle import deep
    pre = deep.precompute(K, V, cb, M0, C, L)
    bad = int((gpu_assign != pre["assign"]).sum())
    assert bad == 0, f"{wl_name}: {bad} assignments differ"
    assert np.array_equal(gpu_counts, pre["counts"]), f"{wl_name}: counts differ"
    abs_sum = deep.precompute(K, np.abs(V), cb, M0, C, L)["vsum"]
    err = np.abs(gpu_vsum - pre["vsum"])
    worst = float((err / np.maximum(abs_sum, 1e-30)).max()) if err.size else 0.0
    assert np.all(err <= VSUM_REL * abs_sum + 1e-30), f"{wl_name}: vsum error {worst:.3g} of sum|V|"
    att = deep.attention(Q, cb, pre["counts"], pre["vsum"], M0, C, L, Ps, T, scale)
    B, H, N, d = Q.shape
    ntiles = (N + T - 1) // T
    gsel = gpu_sel.reshape(B * H * ntiles, -1)
    Og = gpu_O.reshape(B * H, N, d)
    Oref = att["O_full"].reshape(B * H, N, d)
    band_tiles, err_o = 0, 0.0
    for j in range(B * H * ntiles):
        off, same = 0, True
        for l in range(L - 1):
            p = len(att["selected"][j][l])
            g = [int(x) for x in gsel[j, off:off + p]]
            o = [int(x) for x in att["selected"][j][l]]
            off += Ps[l]
            if g == o:
                continue
            cand = [int(x) for x in att["candidates"][j][l]]
            score = dict(zip(cand, att["score"][j][l]))
            assert len(set(g)) == p and set(g) <= set(cand), f"{wl_name}: tile {j} level {l}: invalid {g}"
            kth = sorted(score.values(), reverse=True)[p - 1]
            sure_in = {c for c, v in score.items() if v > kth + BAND}
            sure_out = {c for c, v in score.items() if v < kth - BAND}
            assert sure_in <= set(g) and not (set(g) & sure_out), \
                f"{wl_name}: tile {j} level {l}: selection {g} differs from {o} outside the band"
            same = False
            break
        if not same:
            band_tiles += 1
            continue
        bh, t = divmod(j, ntiles)
        r0, r1 = t * T, min(N, (t + 1) * T)
        err_o = max(err_o, float(np.abs(Og[bh, r0:r1] - Oref[bh, r0:r1]).max()))
    tol = O_TOL[dtype]
    assert err_o <= tol, f"{wl_name}: O max-abs error {err_o:.3g} > {tol}"
    assert np.isfinite(Og).all(), "non-finite output"
    return Report(O_maxabs=err_o, tiles=B * H * ntiles, tie_band_tiles=band_tiles, vsum_rel_err=worst,
                  max_depth=int(pre["depth"].max()))
