"""Host logic of bench.py's multi-rank (replica) mode on CPU: two gloo ranks
in child processes, the max-over-ranks time, the whole-job rate and the
reference arm's rank-0-only rule."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world, cuda=False)
        ms = 2.0 + 3.0 * rank  # rank 1 is the slow one
        rate, ms_max = bench.job_rate(1, ms, world, device="cpu")

        class A:
            pass
        args = A()
        ref = bench.run_reference(args, world, rank) if rank != 0 else "skipped"
        q.put((rank, rate, ms_max, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_sum_units():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, rate, ms_max, ref = q.get(timeout=120)
        out[r] = (rate, ms_max, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time; the rate counts both ranks' units
    assert out[0][1] == out[1][1] == pytest.approx(5.0)
    assert out[0][0] == out[1][0] == pytest.approx(2 * 1000.0 / 5.0)
    # only rank 0 runs the reference arm
    assert out[1][2] is None


def test_single_rank_rate_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    rate, ms = bench.job_rate(4, 2.0, 1)
    assert ms == 2.0 and rate == pytest.approx(2000.0)


def test_cpu_oracle_rate_scales_to_the_whole_stack():
    # the sampled layers' time per layer is charged for every layer of the stack
    sys.path.insert(0, ROOT)
    import bench
    from routed_expert_layer_route_b200 import synth

    class SmallStack:
        wl = {"T": 1, "layers": 3}

        def __init__(self):
            self.layers = [synth.make_layer(1, 64, 8, 32, seed=0, layer=l, device="cpu")
                           for l in range(3)]

        def down_hf(self, L, e):
            return synth.to_numpy(L.w_down[e])

    st = SmallStack()
    r_own, n_own, _, _ = bench.cpu_oracle_rate(st, 2, 4, budget_s=0.3)
    r_48, n_48, _, _ = bench.cpu_oracle_rate(st, 2, 4, budget_s=0.3, stack_layers=48)
    assert n_own > 10 and n_48 > 10
    assert r_48 < r_own / 4  # 16x fewer tokens/s for a 16x deeper stack, within timing noise


def test_reference_arm_inputs_leave_the_product_library_unloaded():
    # the oracle arm builds its layers from the seeded generators alone
    import subprocess
    code = ("import sys; sys.path.insert(0, %r); import bench\n"
            "wl = dict(bench.WORKLOADS['decode_b1']); wl.update(d=64, E=8, I=32, layers=2)\n"
            "st = bench.OracleLayers(wl, 0, 'cpu')\n"
            "assert st.down_hf(st.layers[0], 3).shape == (64, 32)\n"
            "assert 'routed_expert_layer_route_b200.moe' not in sys.modules\n"
            "print('ok')" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stderr


def test_both_arms_report_the_same_config():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, T, layers, k1, k2 = "decode_b1", 0, 0, 0, 0
        cascade = channel_keep = skip = router_std = None
    wl, sweep = bench.workload_of(A())
    c = bench.line_config(A(), wl, sweep[0], 1)
    assert c["workload"].startswith("decode_b1: 48 layers, d=2048, E=128, I=768, T=1")
    assert (c["k1"], c["k2"]) == (4, 16)
    assert "us_per_layer" not in c  # measured values stay out of the shared config


def test_few_token_workload_config():
    # --cm: the small-batch workload on the channel-major down matrix (the few-token
    # decode kernel); the default run times T = 2 / 4 / 8 that way after the others
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, T, layers, k1, k2, cm = "decode_small_batch", 4, 0, 4, 16, True
        cascade = channel_keep = skip = router_std = None
    wl, sweep = bench.workload_of(A())
    assert wl["cm"] == 1 and wl["T"] == 4 and sweep == [(4, 16)]
    c = bench.line_config(A(), wl, sweep[0], 1)
    assert c["w_down_layout"].startswith("channel-major")
    keys = [name + "".join("_%s%d" % kv for kv in sorted(over.items()))
            for name, over in bench.EXTRA_WORKLOADS]
    assert keys[-3:] == ["decode_small_batch_T2_cm1", "decode_small_batch_T4_cm1",
                         "decode_small_batch_T8_cm1"]
    assert keys[0] == "prefill"
    # the grouped GEMMs at the same batch sizes, for the comparison
    assert {"decode_small_batch_T2", "decode_small_batch_T4", "decode_small_batch_T8"} <= set(keys)
