"""The multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1 run the same
functions the N-GPU bench uses (independent per-rank streams, max over ranks, whole-job
rate), and the reference arm's non-zero ranks exit without work."""
import os
import socket
import sys
from datetime import timedelta

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from kvc_streams import WORKLOADS, FrameStream
        m = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        rate = bench.job_rate(world, 20, m)
        st = FrameStream(WORKLOADS["tiny_f32"], seed=bench.rank_seed(rank))
        k = st.frame(0, 0)[1]
        ks = [torch.zeros_like(k) for _ in range(world)]
        dist.all_gather(ks, k)
        q.put((rank, m, rate, bool(torch.equal(ks[0], ks[1]))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_independent_streams():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, rate, same in res:
        assert m == 15.0                      # the slower rank's time, on every rank
        assert rate == pytest.approx(2 * 20 / 0.015)
        assert not same                       # replicas stream different frames


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_rate(1, 10, 100.0) == pytest.approx(100.0)


def test_reference_arm_nonzero_rank_exits_without_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"steps": 3, "warmup": 3, "gpus": 2})()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def _sharded_worker(rank, world, port, results):
    """Each rank computes its heads of one stream with the fp64 oracle (heads are
    independent), then bench.gather_heads assembles the full output."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from kvc_streams import WORKLOADS, FrameStream, keyframe_schedule
        from oracle import OracleConfig, StreamOracle
        wl = WORKLOADS["tiny_f32"].replace(num_heads=4)
        h0, h1 = bench.head_range(rank, world, wl.num_heads)
        st = FrameStream(wl, seed=bench.rank_seed(0))
        mine = StreamOracle(OracleConfig.from_workload(wl.replace(num_heads=h1 - h0)))
        full = StreamOracle(OracleConfig.from_workload(wl))
        worst = 0.0
        for t in range(8):
            key = keyframe_schedule(t, wl.scale_frames, wl.keyframe_interval)
            qf, kf, vf = (x.to(torch.float64).numpy() for x in st.frame(0, t))
            mine.append(0, t, kf[:, h0:h1], vf[:, h0:h1], key)
            o_local = torch.from_numpy(mine.attend(0, qf[:, h0:h1]))
            o_all = bench.gather_heads(o_local, world)
            full.append(0, t, kf, vf, key)
            ref = full.attend(0, qf)
            worst = max(worst, float(np.abs(o_all.numpy() - ref).max()))
        results.put((rank, (h0, h1), worst))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_sharded_step_reassembles_the_full_output():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [(0, 2), (2, 4)]
    assert all(r[2] <= 1e-12 for r in res)          # heads are independent: the same answer
    import bench
    with pytest.raises(ValueError):
        bench.head_range(0, 3, 4)


def test_profile_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    """The bench's roofline `traffic` comes from the committed ncu summary of the attention
    kernel, and only while the kernel source hashes to the one that summary names."""
    sys.path.insert(0, ROOT)
    import bench
    txt = open(bench.PROFILE_ATTN).read()
    assert "source_sha256:" in txt and "traffic_bytes_per_launch:" in txt
    t = bench.profile_traffic()
    assert t is not None, "the attention source changed since its ncu summary was taken"
    assert 2.9e8 < t < 3.5e8                 # about the 298.7 MB algorithmic bytes of a launch
    changed = tmp_path / "kvc_attn_tc.cu"
    changed.write_bytes(open(bench.ATTN_SRC, "rb").read() + b"\n")
    monkeypatch.setattr(bench, "ATTN_SRC", str(changed))
    assert bench.profile_traffic() is None


@pytest.mark.parametrize("text,kind,hbm,bf16", [
    ('{"hbm_gbs": 7000.5, "bf16_tflops": 1650, "bf16_tflops_sustained": 1420}', "measured", 7000.5, 1650.0),
    ('{"hbm": {"hbm_gbs": 7001}, "gemm": {"bf16_tflops": {"value": 1640.0}}}', "measured", 7001.0, 1640.0),
    ('{"hbm_gbs": 7002, "bf16_tflops": 1630}', "measured", 7002.0, 1630.0),
    ('{"hbm_gbs": 7003}', "fallback", 6650.0, 1590.0),
    ('{"hbm_gbs": "fast", "bf16_tflops": -1}', "fallback", 6650.0, 1590.0),
    ("not json", "fallback", 6650.0, 1590.0),
])
def test_peaks_file_read_or_fallback(tmp_path, text, kind, hbm, bf16):
    """The roofline denominators come from the peaks file when it holds the HBM and bf16
    figures (flat, in sections, or as {"value": x}); otherwise every figure falls back."""
    sys.path.insert(0, ROOT)
    import bench
    f = tmp_path / "peaks.json"
    f.write_text(text)
    peaks, k = bench.load_peaks(str(f))
    assert (k, peaks["hbm_gbs"], peaks["bf16_tflops"]) == (kind, hbm, bf16)
    assert peaks["bf16_tflops_sustained"] > 0
    assert bench.load_peaks(str(tmp_path / "absent.json"))[1] == "fallback"
