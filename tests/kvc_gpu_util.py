"""Helpers shared by the GPU parity tests: drive the CUDA library and the oracle over
the same seeded stream and compare them."""
from __future__ import annotations

import math

import numpy as np
import torch

from kvc_streams import FrameStream, keyframe_schedule
from oracle import OracleConfig, StreamOracle

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
F32_MAX_ABS = 1e-4
U64 = 2.0 ** -53          # unit roundoff of fp64


def np64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to(torch.float64).cpu().numpy()


def sample_rows(T: int, n: int = 64, seed: int = 0) -> np.ndarray:
    """Seeded query rows, always including rows 0-4 and the last row."""
    rng = np.random.default_rng(seed)
    fixed = [r for r in (0, 1, 2, 3, 4, T - 1) if r < T]
    rest = [r for r in rng.permutation(T).tolist() if r not in fixed][: max(0, n - len(fixed))]
    return np.array(sorted(set(fixed + rest)))


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x| (the largest error of rounding x to bf16)."""
    _, e = np.frexp(np.abs(x))                 # |x| in [2^(e-1), 2^e): spacing 2^(e-8)
    return np.where(x == 0, 0.0, np.ldexp(1.0, np.maximum(e - 9, -134)))


def compare_out(got: np.ndarray, ref: np.ndarray, io_dtype: str, what: str = ""):
    """fp32 outputs: max-abs <= 1e-4. bf16 outputs: mean-abs <= 2e-3 and max-abs <= 2e-2,
    where for |ref| >= 4 the bound applies to the error beyond the rounding of the exact
    value to the bf16 output format (half a bf16 ulp: 1/64 on [4, 8), and more than 2e-2
    itself from 8 on); below 4 the bound applies to the plain error. Returns the plain
    max-abs and mean-abs errors."""
    err = np.abs(got - ref)
    if io_dtype == "f32":
        assert err.max() <= F32_MAX_ABS, f"{what}: max abs {err.max():.3e} > {F32_MAX_ABS}"
        return float(err.max()), float(err.mean())
    allow = np.where(np.abs(ref) >= 4.0, bf16_half_ulp(ref), 0.0)
    beyond = err - allow
    assert beyond.max() <= BF16_MAX_ABS, \
        f"{what}: max abs {err.max():.3e} ({beyond.max():.3e} beyond bf16 output rounding where |O| >= 4) > {BF16_MAX_ABS}"
    assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs {err.mean():.3e} > {BF16_MEAN_ABS}"
    return float(err.max()), float(err.mean())


def run_parity(kvc, wl, frames, *, check_frames=None, rows=None, seed=0, layers=None, kv_splits=0,
               check_pages=False, record=None, batched_append=False, transform=None, joint=0, joint_rows=None):
    """Stream `frames` frames through the library and the oracle; compare page tables at
    every step and outputs on `check_frames` (all if None) for `rows` (all if None).
    `transform(t, layer, q, k, v) -> (q, k, v)` edits a frame's inputs for both sides.
    `joint` = n > 0 runs frames 0..n-1 as the joint scale-frame phase first (its output
    compared on `joint_rows`, all if None), then the stream continues causally."""
    dev = torch.device("cuda")
    cfg = kvc.config_from_workload(wl, kv_splits=kv_splits)
    h = kvc.kvc_create(cfg)
    try:
        st = FrameStream(wl, seed=seed, device=dev)
        orc = StreamOracle(OracleConfig.from_workload(wl))
        layers = range(wl.num_layers) if layers is None else layers
        T, H, D = wl.tokens_per_frame, wl.num_heads, wl.head_dim
        out = torch.empty((T, H, D), dtype=q_dtype(wl), device=dev)
        stats = []
        if joint:
            oj = torch.empty((joint * T, H, D), dtype=q_dtype(wl), device=dev)
            for l in layers:
                fr = [st.frame(l, t) for t in range(joint)]
                Q, K, V = (torch.cat([x[i] for x in fr]) for i in range(3))
                kvc.kvc_scale_phase(h, l, joint, Q, K, V, oj)
                ref = orc.scale_phase(l, joint, np64(Q), np64(K), np64(V), rows=joint_rows)
                torch.cuda.synchronize()
                got = np64(oj) if joint_rows is None else np64(oj)[joint_rows]
                stats.append((-1, l) + compare_out(got, ref, wl.io_dtype, f"joint phase layer {l}"))
                pt, info = kvc.kvc_page_table(h, l)
                assert np.array_equal(pt, orc.page_table(l)), f"page table differs after the joint phase, layer {l}"
                assert info["device_error"] == 0
        for t in range(joint, frames):
            key = keyframe_schedule(t, wl.scale_frames, wl.keyframe_interval)
            qkv = {l: st.frame(l, t) for l in layers}
            if transform is not None:
                qkv = {l: transform(t, l, *qkv[l]) for l in layers}
            if batched_append:
                kvc.kvc_append_frame_all(h, t, [qkv[l][1] for l in layers], [qkv[l][2] for l in layers], key)
            for l in layers:
                q, k, v = qkv[l]
                if not batched_append:
                    kvc.kvc_append_frame(h, l, t, k, v, key)
                kvc.kvc_attend(h, l, q, out)
                orc.append(l, t, np64(k), np64(v), key)
                do_check = check_frames is None or t in check_frames
                if do_check:
                    ref = orc.attend(l, np64(q), rows=rows)
                else:
                    orc.commit(l)
                if do_check:
                    torch.cuda.synchronize()
                    got = np64(out)
                    got = got if rows is None else got[rows]
                    stats.append((t, l) + compare_out(got, ref, wl.io_dtype, f"frame {t} layer {l}"))
                pt, info = kvc.kvc_page_table(h, l)
                want = orc.page_table(l)
                assert np.array_equal(pt, want), f"page table differs at frame {t} layer {l}"
                assert info["device_error"] == 0
                if check_pages and do_check:
                    check_page_bytes(kvc, h, l, wl, orc)
            if record is not None:
                record(t, h, orc)
        return stats
    finally:
        kvc.kvc_destroy(h)


def q_dtype(wl):
    return torch.float32 if wl.io_dtype == "f32" else torch.bfloat16


def check_page_bytes(kvc, h, layer, wl, orc):
    """Stored pages are bit-exact: bf16/f32 values equal the inputs (zeros in masked
    slots); FP8 codes and scales equal the oracle's."""
    pt = orc.page_table(layer)
    n = len(pt)
    H, P, D = wl.num_heads, wl.page_size, wl.head_dim
    fp8 = wl.kv_dtype == "fp8_e4m3"
    elem = 1 if fp8 else (4 if wl.kv_dtype == "f32" else 2)
    kb, vb, ks, vs = kvc.kvc_export_pages(h, layer, 0, n, H * P * D * elem, H, fp8)
    if fp8:
        kc, vc, kso, vso = orc.fp8_pages(layer)
        assert np.array_equal(kb.reshape(n, H, P, D), kc), "FP8 K codes differ"
        assert np.array_equal(vb.reshape(n, H, P, D), vc), "FP8 V codes differ"
        assert np.array_equal(ks.astype(np.float64), kso), "FP8 K scales differ"
        assert np.array_equal(vs.astype(np.float64), vso), "FP8 V scales differ"
        if getattr(wl, "fp8_dim_adaptive", 0):
            kc_g, vt_g = kvc.kvc_export_fp8_group_scales(h, layer, 0, n, H, D, P)
            kc_o, vt_o = orc.fp8_da_scales(layer)
            assert np.array_equal(kc_g.astype(np.float64), kc_o), "FP8 K channel scales differ"
            assert np.array_equal(vt_g.astype(np.float64), vt_o), "FP8 V token scales differ"
    else:
        dt = torch.float32 if elem == 4 else torch.bfloat16
        L = orc.layers[layer]
        for i, (pid, owner, g, nv) in enumerate(L.entries):
            pg = L.pages[pid]
            kk = torch.from_numpy(kb[i].copy()).view(dt).view(H, P, D).to(torch.float64).numpy()
            vv = torch.from_numpy(vb[i].copy()).view(dt).view(H, P, D).to(torch.float64).numpy()
            assert np.array_equal(kk[:, :nv], pg.k[:, :nv]) and np.array_equal(vv[:, :nv], pg.v[:, :nv])
            assert not kk[:, nv:].any() and not vv[:, nv:].any(), "masked slots must be zero"


def raw_score_choices(r: np.ndarray, s_gpu: np.ndarray) -> dict:
    """Check the GPU's raw scores s = fp32(|r_i|) against the exact norms and return the
    slots where the GPU took the other fp32 neighbour legitimately.

    The squares of fp32 residuals are exact in fp64, so any order of the R - 1 additions
    is within (R - 1) u of the exact sum, and the square root adds half that plus u; the
    oracle's exactly rounded sum is within 1.5 u. A token whose interval
    |r_i| (1 +- (R + 8) u) holds an fp32 rounding boundary may be rounded either way; every
    other token must be bit-equal to the oracle's rounding.
    """
    r = np.asarray(r, np.float64)
    R = r.shape[1]
    exact = np.sqrt(np.array([math.fsum(row * row) for row in r]))
    want = exact.astype(np.float32)
    d = (R + 8) * U64
    lo = (exact * (1 - d)).astype(np.float32)
    hi = (exact * (1 + d)).astype(np.float32)
    amb = lo != hi
    got = np.asarray(s_gpu, np.float32)
    bad = (~amb) & (got != want)
    assert not bad.any(), f"raw scores differ at slots {np.nonzero(bad)[0][:8]}"
    choice = {}
    for i in np.nonzero(amb & (got != want))[0]:
        assert got[i] in (lo[i], hi[i]), f"slot {i}: raw score outside its rounding interval"
        choice[int(i)] = float(got[i])
    return choice


def rolling_score_bound(Kc: np.ndarray) -> np.ndarray:
    """Per candidate, a bound on the difference of two fp64 evaluations of the diversity
    score -cos(k_i, mu) in any summation order (the GPU's blocked sums against the
    oracle's numpy ones), from first-order error analysis with u = 2^-53:
    k_hat within (D/2 + 5) u of k/|k| per component; each mu_d within (N + D/2 + 5) u of
    its exact sum times A_d = sum_i |k_hat_id|; the dot within D u relative plus the
    inputs' errors; |mu| likewise. Both sides' errors are added and the result doubled."""
    Kc = np.asarray(Kc, np.float64)
    N, D = Kc.shape
    nrm = np.linalg.norm(Kc, axis=1)
    nz = nrm > 0
    kh = np.zeros_like(Kc)
    kh[nz] = Kc[nz] / nrm[nz, None]
    mu = kh.sum(axis=0)
    mn = np.linalg.norm(mu)
    if mn == 0.0:
        return np.full(N, 1e-12)
    A = np.abs(kh).sum(axis=0)
    dmu = (N + D / 2 + 5) * U64 * A
    akh = np.abs(kh)
    ddot = akh @ dmu + (1.5 * D + 5) * U64 * (akh @ np.abs(mu))
    dmn = (np.abs(mu) @ dmu) / mn + (D / 2 + 3) * U64 * mn
    sc = np.abs(kh @ mu) / mn
    one_side = ddot / mn + sc * dmn / mn + 4 * U64
    return 2.0 * 2.0 * one_side


def top_k_valid(got_ids, want_ids, cand_ids, scores, bound, k) -> bool:
    """True when the GPU's kept set equals the oracle's; when they differ, assert that the
    difference lies among candidates whose scores are within their bounds of the K-th best
    score (a Top-K that rounding may decide either way) and return False."""
    got, want = set(int(x) for x in got_ids), set(int(x) for x in want_ids)
    if got == want:
        return True
    cand = [int(x) for x in cand_ids]
    assert len(got) == len(want) and got <= set(cand), "kept set of the wrong size or not from the candidates"
    order = sorted(range(len(cand)), key=lambda i: (-scores[i], cand[i]))
    theta = scores[order[min(k, len(cand)) - 1]]
    E = float(np.max(bound))
    amb = {cand[i] for i in range(len(cand)) if abs(scores[i] - theta) <= bound[i] + E}
    assert (want - amb) <= got and (got - want) <= amb, "kept sets differ beyond the rounding of the scores"
    return False
