"""Host-side logic of bench.py (CPU only): algorithmic byte / FLOP counts (top-k,
decode step, sparse attention), the clock-log summary, the phase-stamp table,
the replay spread and input rotation, and the max-over-ranks reduction with two
gloo ranks."""

import os
import socket

import numpy as np
import torch.multiprocessing as mp

import bench


def test_topk_bytes():
    # 64 rows x 129280 float32 read once; k (index + value) written per row
    assert bench.topk_bytes(64, 129280, 1024) == 64 * 129280 * 4 + 64 * 1024 * 8
    assert bench.topk_bytes(4, 8192, 512, elem=2) == 4 * 8192 * 2 + 4 * 512 * 6


def test_decode_bytes_and_flops():
    vl = np.array([4096, 32768, 10000], dtype=np.int32)
    b, f = bench.decode_bytes_flops(vl, 64, 128, 1024)
    assert f == 2 * 64 * 128 * int(vl.sum())
    assert b == 32768 * 256 + 3 * 64 * 128 * 2 + 3 * 64 * 4 + 3 * 4 + 3 * 1024 * 4


def test_attention_bytes_and_flops_decode_workload():
    # 8 rows x (1024 selected + 128 window) rows of 512 bf16 channels, read once;
    # q read and out written (8 x 128 x 512 bf16 each), lse, slots, sink, win_len
    idx = np.arange(8 * 1024, dtype=np.int32).reshape(8, 1024)
    b, f = bench.attention_bytes_flops(idx, 32768, np.full(8, 128), 128, 512, 1024)
    assert b == 9437184 + 2097152 + 4096 + 32768 + 512 + 32 == 11571744
    assert f == 4 * 128 * 512 * 9216


def test_attention_bytes_skip_invalid_slots():
    # -1 padding and slots at or past T attend nothing and read no row
    idx = np.array([[0, -1, 5, 9], [10, 3, -1, -1]], dtype=np.int32)
    b, f = bench.attention_bytes_flops(idx, 9, np.array([2, 0]), 4, 64, 4)
    rows = 2 + 1 + 2                      # T = 9: (0, 5) and (3) valid; 2 window rows
    assert f == 4 * 4 * 64 * rows
    assert b == rows * 64 * 2 + 2 * 2 * 4 * 64 * 2 + 2 * 4 * 4 + 2 * 4 * 4 + 4 * 4 + 2 * 4


def test_clock_summary_flags_throttle_reasons():
    s = bench.ClockSampler(None)
    s.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
    ]
    out = s.summary()
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    r, ws = bench.dist_setup("gloo")
    got = bench.max_over_ranks([float(rank + 1), 10.0 - rank], "cpu")
    bench.barrier()
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, ws, got))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, ws, got in res:
        assert ws == 2
        assert got == [2.0, 10.0]


def test_stamp_table_medians_after_the_first_start():
    import numpy as np
    # two CTAs that started 1000 ns apart; the second never reached the leader
    # phases (0 = not reached); unused rows (start 0) are ignored
    st = np.zeros((4, 10), dtype=np.uint64)
    st[0, :6] = [5000, 6000, 7000, 8000, 9000, 10000]
    st[0, 6:] = [11000, 12000, 13000, 14000]
    st[1, :6] = [6000, 7000, 8000, 9000, 10000, 11000]
    t = bench.stamp_table(st)
    assert t["ctas"] == 2
    m = t["median_us_after_start"]
    assert m["start"] == 0.5 and m["prologue"] == 1.5 and m["merged"] == 5.5
    assert m["leader: stash counted"] == 6.0 and m["leader: emission written"] == 9.0


def test_spread_and_rotation():
    s = bench.spread([3.0, 1.0, 2.0])
    assert s == {"median": 2.0, "min": 1.0, "max": 3.0, "replays": 3}
    # copies whose cycle reads more than 2x L2 between two uses of one copy
    r = bench.rotation(33_095_680)
    assert (r - 1) * 33_095_680 > 2 * bench.L2_BYTES
    assert bench.rotation(1) == 4096  # capped
