"""The allocation-free attention entry point (for callers that cannot allocate device
memory) against the cache's own kvc_attend, through the C ABI, on two calls in a row.

This file sorts last so that a stop-at-first-failure run has run every other test first;
it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from kvc_streams import WORKLOADS, FrameStream

pytestmark = pytest.mark.gpu


def test_noalloc_attention_matches_kvc_attend_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import transformer_kv_cache_b200 as kvc
    wl = WORKLOADS["vggt_518x378"].replace(tokens_per_frame=300, num_heads=4, window_frames=4, scale_frames=1)
    T, H, D, P = wl.tokens_per_frame, wl.num_heads, wl.head_dim, wl.page_size
    dev = torch.device("cuda")
    st = FrameStream(wl, seed=21, device=dev)
    h = kvc.kvc_create(kvc.config_from_workload(wl, kv_splits=3))
    frames = []
    o_ref = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    for t in range(7):
        q, k, v = st.frame(0, t)
        frames.append((q, k, v))
        kvc.kvc_append_frame(h, 0, t, k, v, True)
        kvc.kvc_attend(h, 0, q, o_ref)
    torch.cuda.synchronize()
    kvc.kvc_destroy(h)
    # frame 6 attended the first S = 1 and last W = 4 committed frames plus itself
    attended = [0, 2, 3, 4, 5, 6]
    ppf = -(-T // P)
    n_pages = len(attended) * ppf
    kp = torch.zeros((n_pages, H, P, D), dtype=torch.bfloat16, device=dev)
    vp = torch.zeros_like(kp)
    rows = []
    for i, f in enumerate(attended):
        _, k, v = frames[f]
        for src, dst in ((k, kp), (v, vp)):
            pad = torch.zeros((ppf * P, H, D), dtype=torch.bfloat16, device=dev)
            pad[:T] = src
            dst[i * ppf:(i + 1) * ppf] = pad.view(ppf, P, H, D).permute(0, 2, 1, 3)
        for g in range(ppf):
            rows.append([i * ppf + g, 0, 0, min(P, T - g * P)])
    table = torch.tensor(rows, dtype=torch.int32, device=dev)
    q6 = frames[6][0]
    outs = []
    for call in range(2):
        o = torch.full((T, H, D), float("nan"), dtype=torch.bfloat16, device=dev)
        kvc.kvc_attend_paged_noalloc(q6, o, kp, vp, n_pages, table, n_pages, T, H, D, P, wl.softmax_scale,
                                     kv_splits=3)
        torch.cuda.synchronize()
        err = (o.double() - o_ref.double()).abs()
        assert torch.isfinite(o.float()).all()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3, (call, err.max().item())
        outs.append(o)
    assert torch.equal(outs[0], outs[1])
    # a split count whose partials exceed the fixed scratch is rejected before anything is
    # launched; the buffers have the declared shape (8,032 queries, 16 heads, a 4,096-row
    # table of valid entries on a one-page pool), so a guard that let the call through would
    # compute a wrong answer rather than read or write out of bounds
    Tb, Hb, nb = 1004 * 8, 16, 4096
    qb = torch.zeros((Tb, Hb, D), dtype=torch.bfloat16, device=dev)
    ob = torch.empty_like(qb)
    kb = torch.zeros((1, Hb, P, D), dtype=torch.bfloat16, device=dev)
    vb = torch.zeros_like(kb)
    tb = torch.tensor([[0, 0, 0, P]] * nb, dtype=torch.int32, device=dev)
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_attend_paged_noalloc(qb, ob, kb, vb, 1, tb, nb, Tb, Hb, D, P, 0.125, kv_splits=8)
    assert e.value.status_name == "KVC_ERR_ARG"
