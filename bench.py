"""Benchmark of the sparse-attention selection step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole selection path over one batch of synthetic,
seeded input:
  * top-k of the sampling workload (64 rows x 129280 float32 logits ~ N(0, 9)
    with 20 planted +15 outliers per row) at k = 1024 and at k = 64, values
    and indices, unsorted;
  * the decode indexer + top-k (8 query rows x 64 heads x 128 bf16 against one
    bf16 key cache of 32768 positions, valid_len ~ U{4096..32768}, k = 1024).
Reported beside it, in "configs", every workload of the selection step, each
timed over repeated CUDA-graph replays (median and spread) with its oracle
time on one host core: the standalone top-k (4 x 8192 bf16, k = 512), the
sampling top-k, the indexer-style top-k (bf16, 1/8/64 rows x 32768/131072,
k = 2048, and the same rows sorted ascending), the decode and the prefill
indexer + top-k.  Also beside it: the sparse attention that consumes the
selection (8 tokens x 128 heads x 512 over k = 1024 selected rows plus a
window of 128, rotating slot sets); and the indexer query projection that
feeds the scorer (8 tokens, width 1536 -> 64 x 128 queries and 64 weights),
alone and chained in front of the decode indexer + top-k.
The headline value is the top-k effective HBM bandwidth (algorithmic bytes /
device time, GB/s); the decode indexer + top-k time is reported in
microseconds per decode step beside it.  Inputs rotate through enough copies
(> 2x the 126 MB L2) that every call reads HBM.  With N > 1 (torchrun, one
process per GPU) every rank processes its own batch (weak scaling, no data
collective); the value is the total over ranks divided by the slowest rank's
time.

``--impl reference`` times the CPU oracle (float64, single thread) on a bounded
sample of the same workload and prints the same line with "impl": "reference".
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "top-k effective HBM GB/s (% of peak); indexer+top-k µs per decode step"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024

SAMPLING = dict(batch=64, n=129280, ks=(1024, 64))
# ds_topk runs the one-pass stash kernel for >= 64 rows (the cluster kernel below)
TOPK_KERNEL = "topk_stash_kernel<F32Keys, 1024>"
DECODE = dict(batch=8, heads=64, d=128, S=32768, k=1024)
PREFILL = dict(k=2048)
ATTENTION = dict(batch=8, heads=128, d=512, T=32768, k=1024, W=128)
ATTN_CALLS = 40
QPROJ = dict(T=8, d_in=1536, heads=64)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def topk_bytes(batch, n, k, elem=4, values=True):
    """Algorithmic bytes of one top-k call: read every score once, write k
    int32 indices (and k values) per row."""
    return batch * n * elem + batch * k * (4 + (elem if values else 0))


def decode_bytes_flops(vl, heads, d, k):
    """Algorithmic bytes and FLOPs of one decode indexer + top-k call."""
    maxvl = int(np.max(vl))
    B = len(vl)
    bytes_ = maxvl * d * 2 + B * heads * d * 2 + B * heads * 4 + B * 4 + B * k * 4
    flops = 2 * heads * d * int(np.sum(vl))
    return bytes_, flops


def attention_bytes_flops(idx, T, win_len, heads, d, k):
    """Algorithmic bytes and FLOPs of one sparse-attention call: every attended
    row read once (it is both key and value), queries read and outputs (bf16
    out, float32 lse) written once, the slots and the sink read once; two
    products of 2 * heads * d FLOPs per attended row."""
    idx = np.asarray(idx)
    rows = int(((idx >= 0) & (idx < T)).sum()) + int(np.sum(win_len))
    B = idx.shape[0]
    bytes_ = rows * d * 2 + 2 * B * heads * d * 2 + B * heads * 4 + B * k * 4 + heads * 4 + B * 4
    flops = 4.0 * heads * d * rows
    return bytes_, flops


def graph_time_us(fn_of_i, count, reps=3):
    """Device time per call of fn_of_i(0..count-1), captured as one CUDA graph
    (host launch cost off the device timeline) and replayed `reps` times after
    one warm replay; CUDA events on the current stream."""
    import torch
    stream = torch.cuda.current_stream()
    for i in range(count):          # warm-up, and the first-use set-up of each input set
        fn_of_i(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(count):
            fn_of_i(i)
    g.replay()
    torch.cuda.synchronize()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) * 1e3 / (count * reps)


def graph_times_us(fn_of_i, count, reps=5):
    """Per-call device times of fn_of_i(0..count-1), captured as one CUDA graph
    and replayed `reps` times (after one warm replay), each replay timed alone
    with CUDA events: the list of µs per call."""
    import torch
    stream = torch.cuda.current_stream()
    for i in range(min(count, 3)):
        fn_of_i(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(count):
            fn_of_i(i)
    g.replay()
    torch.cuda.synchronize()
    barrier()
    out = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        out.append(a.elapsed_time(b) * 1e3 / count)
    del g
    return out


def spread(us):
    """Median and range of repeated timings, µs."""
    return {"median": round(statistics.median(us), 3), "min": round(min(us), 3), "max": round(max(us), 3),
            "replays": len(us)}


def rotation(nbytes, cap=4096):
    """Copies of an input of `nbytes` such that, cycling through them, more than
    2x L2 is read between two uses of one copy (at most `cap`)."""
    return int(min(cap, max(3, -(-2 * L2_BYTES // max(nbytes, 1)) + 1)))


def topk_config(us, batch, n, k, elem, values, hbm_gbs):
    """The figures of one top-k workload from its per-call times."""
    med = statistics.median(us)
    nbytes = topk_bytes(batch, n, k, elem, values)
    gbs = nbytes / (med * 1e-6) / 1e9
    return {"us_per_call": spread(us), "rows_per_s": round(batch / (med * 1e-6), 1),
            "algorithmic_bytes": int(nbytes), "achieved_gbs": round(gbs, 1),
            "pct_of_measured_hbm": round(100 * gbs / hbm_gbs, 1), "pct_of_nominal_8tbs": round(100 * gbs / NOMINAL_HBM_GBS, 1),
            "roofline_us": round(nbytes / (hbm_gbs * 1e9) * 1e6, 3)}


def measure_configs(ds, inputs, dev, rank, hbm_gbs, tflops, reps=5):
    """Every top-k workload of the selection step beside the headline: the
    standalone rows and the indexer-style rows (inputs rotate through copies
    totalling more than 2x L2, so every call reads HBM).  The indexer-style
    rows are made by this library's scorer from seeded factors and rounded to
    bfloat16 (round to nearest even), as their config prescribes."""
    import torch
    res = {}
    # 1: standalone, 4 x 8192 bf16 ~ N(0, 1), k = 512, values + indices
    x = inputs.standalone(seed=inputs.SEED_STANDALONE + rank)
    B, n, k = x.shape[0], x.shape[1], 512
    R = rotation(x.nbytes)
    xb = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev).unsqueeze(0).repeat(R, 1, 1)
    oi = torch.empty((B, k), dtype=torch.int32, device=dev)
    ov = torch.empty((B, k), dtype=torch.bfloat16, device=dev)
    us = graph_times_us(lambda i: ds.ds_topk(xb[i % R], k, return_value=True, out_idx=oi, out_val=ov), R, reps)
    res["standalone_4x8192_bf16_k512"] = dict(topk_config(us, B, n, k, 2, True, hbm_gbs), rotation=R,
                                              bound="launch latency (64 KiB per call)")
    del xb
    # 3: indexer-style rows, bf16, k = 2048, indices only; and the ascending variant
    rows3 = {}
    for nn in (32768, 131072):
        q, kc, w = inputs.indexer_factors(seed=inputs.SEED_INDEXER + rank, batch=64, n=nn)
        to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        sc = ds.ds_indexer_score(to(q), to(kc), torch.from_numpy(w).to(dev))
        rows3[nn] = sc.to(torch.bfloat16)
        del sc
    for nn in (32768, 131072):
        for bb in (1, 8, 64):
            for variant in ("random", "ascending"):
                r = rows3[nn][:bb]
                if variant == "ascending":
                    r = torch.sort(r, dim=1).values
                R = rotation(r.numel() * 2)
                buf = r.unsqueeze(0).repeat(R, 1, 1)
                oi = torch.empty((bb, 2048), dtype=torch.int32, device=dev)
                us = graph_times_us(lambda i: ds.ds_topk(buf[i % R], 2048, return_value=False, out_idx=oi), R, reps)
                res[f"indexer_style_{bb}x{nn}_bf16_k2048_{variant}"] = dict(
                    topk_config(us, bb, nn, 2048, 2, False, hbm_gbs), rotation=R)
                del buf
    status = ds.ds_get_device_status()
    if status != ds.DS_OK:
        raise RuntimeError(f"device status after the configs: {ds.strerror(status)}")
    return res


def oracle_configs(seconds=1.5):
    """The CPU oracle (float64, one thread) on a bounded sample of every
    top-k workload: µs per row, and the implied µs per call."""
    from threadpoolctl import threadpool_limits
    import oracle
    from sparse_attention_top_ds_b200 import inputs
    out = {}

    def per_row(fn, rows):
        t0, done = time.perf_counter(), 0
        while done < rows and (done == 0 or time.perf_counter() - t0 < seconds):
            fn(done)
            done += 1
        return (time.perf_counter() - t0) / done * 1e6, done

    with threadpool_limits(limits=1):
        x = inputs.standalone()
        us, dn = per_row(lambda r: oracle.topk_rows(x[r:r + 1], "bf16", 512), x.shape[0])
        out["standalone_4x8192_bf16_k512"] = {"us_per_row": round(us, 1), "us_per_call": round(us * 4, 1),
                                             "rows_timed": dn}
        for nn in (32768, 131072):
            q, kc, w = inputs.indexer_factors(batch=2, n=nn)
            us, dn = per_row(lambda r: oracle.indexer_topk(q[r:r + 1], kc, w[r:r + 1], 2048), 2)
            out[f"indexer_style_rows_n{nn}"] = {"us_per_row": round(us, 1), "rows_timed": dn,
                                                 "what": "float64 score row + stable sort (the top-k alone is a "
                                                         "fraction of it)"}
        pq, pkc, pw, pvl = inputs.prefill()
        sub = inputs.sample_rows(inputs.SEED_PREFILL, pq.shape[0], 4)
        us, dn = per_row(lambda r: oracle.indexer_topk(pq[sub[r]:sub[r] + 1], pkc, pw[sub[r]:sub[r] + 1], 2048,
                                                       pvl[sub[r]:sub[r] + 1]), 4)
        out["prefill_4096x64x128_vs_32768_k2048"] = {"us_per_row": round(us, 1), "rows_timed": dn,
                                                    "us_per_call_extrapolated": round(us * pq.shape[0], 1)}
    return out


def measure_attention(ds, inputs, dev, stream, rank, hbm_gbs, tflops, calls, warmup=3):
    """Sparse attention over the selected rows (the step that consumes the
    selection): 8 tokens x 128 heads x d = 512 against a 32768-row cache per
    batch row, k = 1024 slots plus a window of 128.  Calls rotate through 24
    slot sets, each with its own copy of the queries and the window, so that
    between two uses of a set the other sets have touched more than 2x L2 of
    rows: every call gathers its rows from HBM, as after the selection step."""
    import torch
    A = ATTENTION
    R = 24
    aa = inputs.attention(seed=inputs.SEED_ATTENTION + rank, batch=A["batch"], heads=A["heads"], d=A["d"],
                          T=A["T"], k=A["k"], W=A["W"])
    to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    a_kv = to(aa["kv"])
    q0, w0 = to(aa["q"]), to(aa["win"])
    a_q = [q0.clone() for _ in range(R)]
    a_win = [w0.clone() for _ in range(R)]
    idx_sets = [aa["idx"]] + [inputs.attention_slots(inputs.SEED_ATTENTION + 1000 * (rank + 1) + r, batch=A["batch"],
                                                     T=A["T"], k=A["k"]) for r in range(1, R)]
    a_idx = [torch.from_numpy(i).to(dev) for i in idx_sets]
    a_wl = torch.from_numpy(aa["win_len"]).to(dev)
    a_sink = torch.from_numpy(aa["sink"]).to(dev)
    a_out = torch.empty((A["batch"], A["heads"], A["d"]), dtype=torch.bfloat16, device=dev)
    a_lse = torch.empty((A["batch"], A["heads"]), dtype=torch.float32, device=dev)

    def call(i):
        r = i % R
        ds.ds_sparse_attention(a_q[r], a_kv, a_idx[r], win=a_win[r], win_len=a_wl, sink=a_sink, out=a_out, lse=a_lse)

    attn_us = graph_time_us(call, R, reps=max(1, calls // R))
    (attn_us,) = max_over_ranks([attn_us], dev)
    status = ds.ds_get_device_status()
    if status != ds.DS_OK:
        raise RuntimeError(f"device status after attention: {ds.strerror(status)}")
    ab = [attention_bytes_flops(i, A["T"], aa["win_len"], A["heads"], A["d"], A["k"]) for i in idx_sets]
    abytes = sum(x[0] for x in ab) / R
    aflops = sum(x[1] for x in ab) / R
    a_t_hbm = abytes / (hbm_gbs * 1e9) * 1e6
    a_t_tc = aflops / (tflops * 1e12) * 1e6
    return {
        "workload": "8 tokens x 128 heads x d=512 bf16 queries; per-row bf16 cache of 32768 x 512; k=1024 "
                    "selected rows + window of 128 + per-head sink; out bf16 + lse f32; 24 rotating slot sets "
                    "(> 2x L2 of rows between reuses)",
        "us_per_call": round(attn_us, 2),
        "roofline_us": round(max(a_t_hbm, a_t_tc), 3),
        "bound": "hbm" if a_t_hbm >= a_t_tc else "tensor",
        "frac_of_roofline": round(max(a_t_hbm, a_t_tc) / attn_us, 3),
        "achieved_gbs": round(abytes / (attn_us * 1e-6) / 1e9, 1),
        "achieved_tflops": round(aflops / (attn_us * 1e-6) / 1e12, 1),
        "algorithmic_bytes": int(abytes), "flops": int(aflops),
        "peaks": {"hbm_gbs": hbm_gbs, "bf16_tflops": tflops, "kind": "burst"},
    }


def measure_qproj(ds, inputs, dev, stream, rank, hbm_gbs, calls, warmup=3):
    """The indexer query projection of a decode step (8 tokens, width 1536,
    64 heads x 128 + 64 per-head weights), alone and chained in front of the
    decode indexer + top-k.  Calls rotate through 11 copies of the 25.5 MB of
    weights (and 33 copies of the 8 MB key cache for the chained step), more
    than 2x L2 between reuses, so the weights come from HBM."""
    import torch
    Q = QPROJ
    x, wq, ww = inputs.qproj(seed=inputs.SEED_QPROJ + rank, T=Q["T"], d_in=Q["d_in"], heads=Q["heads"])
    to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    xd = to(x)
    Rw = max(3, -(-2 * L2_BYTES // (wq.nbytes + ww.nbytes)) + 1)
    wq0, ww0 = to(wq), to(ww)
    wqs = [wq0] + [wq0.clone() for _ in range(Rw - 1)]
    wws = [ww0] + [ww0.clone() for _ in range(Rw - 1)]
    q_out = torch.empty((Q["T"], Q["heads"], 128), dtype=torch.bfloat16, device=dev)
    w_out = torch.empty((Q["T"], Q["heads"]), dtype=torch.float32, device=dev)
    _, kc, _, vl = inputs.decode(seed=inputs.SEED_DECODE + rank)
    Rk = max(3, -(-2 * L2_BYTES // kc.nbytes) + 1)
    kc0 = to(kc)
    kcs = [kc0] + [kc0.clone() for _ in range(Rk - 1)]
    vld = torch.from_numpy(vl).to(dev)
    idx = torch.empty((Q["T"], DECODE["k"]), dtype=torch.int32, device=dev)

    def proj(i):
        ds.ds_indexer_qproj(xd, wqs[i % Rw], wws[i % Rw], q_out=q_out, w_out=w_out)

    def step(i):
        proj(i)
        ds.ds_indexer_topk(q_out, kcs[i % Rk], w_out, DECODE["k"], valid_len=vld, out_idx=idx)

    proj_us = graph_time_us(proj, Rw, reps=max(1, calls // Rw))
    step_us = graph_time_us(step, Rk, reps=max(1, calls // Rk))
    proj_us, step_us = max_over_ranks([proj_us, step_us], dev)
    status = ds.ds_get_device_status()
    if status != ds.DS_OK:
        raise RuntimeError(f"device status after the projection: {ds.strerror(status)}")
    nbytes = wq.nbytes + ww.nbytes + x.nbytes + q_out.numel() * 2 + w_out.numel() * 4
    roof_us = nbytes / (hbm_gbs * 1e9) * 1e6
    return {
        "workload": f"8 tokens x width 1536 bf16 -> 64 heads x 128 bf16 queries + 64 f32 weights "
                    f"(Wq 8192 x 1536, Ww 64 x 1536 bf16); {Rw} rotating weight copies (> 2x L2 between reuses)",
        "us_per_call": round(proj_us, 2), "roofline_us": round(roof_us, 3), "bound": "hbm",
        "frac_of_roofline": round(roof_us / proj_us, 3),
        "achieved_gbs": round(nbytes / (proj_us * 1e-6) / 1e9, 1), "algorithmic_bytes": int(nbytes),
        "decode_step_with_projection_us": round(step_us, 2),
    }


def measure_compress(ds, inputs, dev, rank):
    """The compressor's 4:1 fold of a decode step: 8 batch rows, 4 new rows of
    the attention's width 512 each, folded into position 0 of a compressed
    cache.  A few KiB per call: latency bound, so the number is µs per call
    (CUDA-graph replays of 64 calls over 4 rotating input copies)."""
    import torch
    rows, gate = inputs.compress(seed=inputs.SEED_COMPRESS + rank, batch=8, D=512)
    to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    rs = [to(rows) for _ in range(4)]
    gd = to(gate)
    cache = torch.empty((8, 64, 512), dtype=torch.bfloat16, device=dev)
    us = graph_time_us(lambda i: ds.ds_compress_fold(rs[i % 4], gd, out=cache[:, i % 64, :]), 64, reps=3)
    (us,) = max_over_ranks([us], dev)
    return {"workload": "8 batch rows x 4 rows x 512 bf16 -> 8 folded rows written into a [8, 64, 512] cache",
            "us_per_call": round(us, 2), "bound": "latency",
            "bytes_per_call": int(rows.nbytes + gate.nbytes + 8 * 512 * 2)}


ONLY_WORKLOADS = {
    "decode": "decode indexer + top-k: 8 rows x 64 heads x 128 bf16 vs 32768 keys, valid_len ~ U{4096..32768}, "
              "k = 1024, scores returned",
    "sampling": "top-k of 64 x 129280 float32 sampling rows, k = 1024, values and indices",
    "indexer-rows": "top-k of 64 x 131072 bfloat16 indexer-style rows, k = 2048, indices only",
    "prefill": "prefill indexer + top-k: 4096 rows x 64 heads x 128 bf16 vs 32768 keys, causal valid_len, k = 2048",
    "floor": "read-only passes over the sampling rows (64 x 129280 float32, 8 copies rotating): 64, 128 and 256 "
             "CTAs of 1024 threads",
    "stash-phases": "phase stamps of the stash top-k kernel (needs DS_TOPK_LIB = libdstopk_debug.so): one call "
                    "each of the sampling workload at k = 1024 and 64 and of 64 x 131072 bfloat16 rows at k = 2048",
}

STAMP_NAMES = ("start", "prologue", "sample counted", "threshold", "streamed", "merged", "leader: stash counted",
               "leader: bin of the k-th key", "leader: bin resolved", "leader: emission written")


def stamp_table(st):
    """Median over CTAs of each phase stamp, µs after the first CTA's start."""
    st = st.astype(np.float64)
    used = st[:, 0] > 0
    st = st[used]
    t0 = st[:, 0].min()
    out = {}
    for j, nm in enumerate(STAMP_NAMES):
        col = st[:, j]
        col = col[col > 0]
        if len(col):
            out[nm] = round(float(np.median(col - t0)) / 1000.0, 2)
    return {"ctas": int(used.sum()), "median_us_after_start": out}


def run_only(args):
    """`--only <part>`: one part of the step alone, for profiling (the commands
    the profiles are taken with): the sparse attention, the query projection,
    or one workload of the selection step timed over `steps` plain calls
    (one input, so the times of inputs smaller than L2 are L2-warm)."""
    import torch
    import sparse_attention_top_ds_b200 as ds
    from sparse_attention_top_ds_b200 import inputs
    rank, ws = dist_setup("nccl")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    hbm_gbs, tflops, _, _ = load_peaks()
    stream = torch.cuda.current_stream()
    if args.only == "qproj":
        key, a = "qproj", measure_qproj(ds, inputs, dev, stream, rank, hbm_gbs, args.steps, warmup=args.warmup)
    elif args.only == "attention":
        key, a = "sparse_attention", measure_attention(ds, inputs, dev, stream, rank, hbm_gbs, tflops, args.steps,
                                                       warmup=args.warmup)
    else:
        to = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        if args.only in ("decode", "prefill"):
            if args.only == "decode":
                q, kc, w, vl = inputs.decode(seed=inputs.SEED_DECODE + rank)
                k = DECODE["k"]
            else:
                q, kc, w, vl = inputs.prefill(seed=inputs.SEED_PREFILL + rank)
                k = PREFILL["k"]
            qd, kd, wd, vd = to(q), to(kc), torch.from_numpy(w).to(dev), torch.from_numpy(vl).to(dev)
            oi = torch.empty((q.shape[0], k), dtype=torch.int32, device=dev)
            osc = torch.empty((q.shape[0], k), dtype=torch.float32, device=dev)
            fn = lambda: ds.ds_indexer_topk(qd, kd, wd, k, valid_len=vd, return_score=True, out_idx=oi, out_score=osc)
        elif args.only == "floor":
            x = torch.from_numpy(inputs.sampling(seed=inputs.SEED_SAMPLING + rank)[0]).to(dev)
            xs = [x.clone() for _ in range(8)]
            res = {}
            for ctas in (64, 128, 256):
                us = graph_times_us(lambda i: ds.ds_read_floor(xs[i % 8], ctas), 40, reps=5)
                res[f"{ctas}_ctas"] = {"us_per_call": spread(us),
                                       "gbs": round(x.numel() * 4 / (statistics.median(us) * 1e-6) / 1e9, 1)}
            if rank == 0:
                print(json.dumps({"floor": {"workload": ONLY_WORKLOADS["floor"], **res}}), flush=True)
            return
        elif args.only == "stash-phases":
            if not ds.ds_debug_build():
                raise RuntimeError("--only stash-phases needs DS_TOPK_LIB pointing at libdstopk_debug.so")
            res = {}
            samp = torch.from_numpy(inputs.sampling(seed=inputs.SEED_SAMPLING + rank)[0]).to(dev)
            q, kc, w = inputs.indexer_factors(seed=inputs.SEED_INDEXER + rank, batch=64, n=131072)
            rows = ds.ds_indexer_score(to(q), to(kc), torch.from_numpy(w).to(dev)).to(torch.bfloat16)
            for name, xx, k in (("sampling_k1024", samp, 1024), ("sampling_k64", samp, 64),
                                ("bf16_64x131072_k2048", rows, 2048)):
                for _ in range(3):
                    ds.ds_topk(xx, k, return_value=True)
                torch.cuda.synchronize()
                ds.ds_debug_stash_stamps(1024)  # clears
                ds.ds_topk(xx, k, return_value=True)
                torch.cuda.synchronize()
                res[name] = stamp_table(ds.ds_debug_stash_stamps(1024))
            if rank == 0:
                print(json.dumps({"stash_phases": {"workload": ONLY_WORKLOADS["stash-phases"], **res}}), flush=True)
            return
        elif args.only == "sampling":
            x = torch.from_numpy(inputs.sampling(seed=inputs.SEED_SAMPLING + rank)[0]).to(dev)
            oi = torch.empty((x.shape[0], 1024), dtype=torch.int32, device=dev)
            ov = torch.empty((x.shape[0], 1024), dtype=torch.float32, device=dev)
            fn = lambda: ds.ds_topk(x, 1024, return_value=True, out_idx=oi, out_val=ov)
        else:  # indexer-rows
            q, kc, w = inputs.indexer_factors(seed=inputs.SEED_INDEXER + rank, batch=64, n=131072)
            x = ds.ds_indexer_score(to(q), to(kc), torch.from_numpy(w).to(dev)).to(torch.bfloat16)
            oi = torch.empty((64, 2048), dtype=torch.int32, device=dev)
            fn = lambda: ds.ds_topk(x, 2048, return_value=False, out_idx=oi)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a0, b0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            fn()
        b0.record(stream)
        torch.cuda.synchronize()
        status = ds.ds_get_device_status()
        if status != ds.DS_OK:
            raise RuntimeError(f"device status: {ds.strerror(status)}")
        key, a = args.only, {"workload": ONLY_WORKLOADS[args.only],
                             "us_per_call": round(a0.elapsed_time(b0) * 1e3 / max(1, args.steps), 2)}
    if rank == 0:
        print(json.dumps({key: a, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup}), flush=True)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_uuid(dev):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# ------------------------------------------------------------------ CPU oracle leg

def oracle_sample(seconds=10.0, decode_rows=8):
    """Time the CPU oracle (single thread) on a bounded sample of the workload.

    Top-k: whole rows of the sampling workload at k = 1024 and 64, as many as
    fit in `seconds`.  Decode: the float64 indexer score + top-k of the decode
    workload's rows.  Returns a dict with GB/s, rows and microseconds."""
    from threadpoolctl import threadpool_limits
    import oracle
    from sparse_attention_top_ds_b200 import inputs
    x, _ = inputs.sampling()
    q, kc, w, vl = inputs.decode()
    with threadpool_limits(limits=1):
        done_bytes, rows, t0 = 0, 0, time.perf_counter()
        while time.perf_counter() - t0 < seconds and rows < 2 * x.shape[0]:
            t = rows % x.shape[0]
            k = SAMPLING["ks"][(rows // x.shape[0]) % 2]
            oracle.topk_rows(x[t:t + 1], "f32", k)
            done_bytes += topk_bytes(1, x.shape[1], k)
            rows += 1
        t_topk = time.perf_counter() - t0
        t1 = time.perf_counter()
        oracle.indexer_topk(q[:decode_rows], kc, w[:decode_rows], DECODE["k"], vl[:decode_rows])
        t_dec = time.perf_counter() - t1
    return {"topk_gbs": done_bytes / t_topk / 1e9, "topk_rows": rows, "topk_s": t_topk,
            "decode_us": t_dec * 1e6 * (DECODE["batch"] / decode_rows), "decode_rows": decode_rows}


# ------------------------------------------------------------------ distributed helpers

def dist_setup(backend):
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return (dist.get_rank() if dist.is_initialized() else 0), ws


def max_over_ranks(values, device):
    """Element-wise max of a list of floats over all ranks."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ arms

def run_reference(args):
    rank, ws = dist_setup("gloo")
    if rank != 0:
        return
    r = oracle_sample(seconds=max(3.0, min(20.0, 0.2 * args.steps)))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(r["topk_gbs"], 6), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "decode_us_per_step": round(r["decode_us"], 1),
        "config": {"workload": "sampling top-k 64x129280 f32 k in {1024,64} + decode indexer 8x64x128 vs 32768 "
                               "k=1024 (bounded oracle sample)"},
        "cpu_baseline": {"value": round(r["topk_gbs"], 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{r['topk_rows']} sampling rows (k=1024/64) + {r['decode_rows']} decode rows"},
        "e2e": {"value": round(r["topk_gbs"], 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import sparse_attention_top_ds_b200 as ds
    from sparse_attention_top_ds_b200 import inputs

    rank, ws = dist_setup("nccl")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    hbm_gbs, tflops, tflops_sus, peak_src = load_peaks()

    # ---- inputs (each rank its own seeded batch), resident in HBM
    x_host, _ = inputs.sampling(seed=inputs.SEED_SAMPLING + rank)
    xb = x_host.nbytes
    R = max(3, -(-2 * L2_BYTES // xb) + 1)
    xs = [torch.from_numpy(x_host).to(dev) for _ in range(R)]
    xs2 = [torch.from_numpy(x_host).to(dev) for _ in range(R)]   # the k=64 phase rotates its own copies
    q, kc, w, vl = inputs.decode(seed=inputs.SEED_DECODE + rank)
    q_d = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).to(dev)
    w_d = torch.from_numpy(w).to(dev)
    vl_d = torch.from_numpy(vl).to(dev)
    kcb = kc.nbytes
    Rk = max(3, -(-2 * L2_BYTES // kcb) + 1)
    kcs = [torch.from_numpy(kc.view(np.int16)).view(torch.bfloat16).to(dev) for _ in range(Rk)]
    B, n = x_host.shape
    k1, k2 = SAMPLING["ks"]
    idx1 = torch.empty((B, k1), dtype=torch.int32, device=dev)
    val1 = torch.empty((B, k1), dtype=torch.float32, device=dev)
    idx2 = torch.empty((B, k2), dtype=torch.int32, device=dev)
    val2 = torch.empty((B, k2), dtype=torch.float32, device=dev)
    didx = torch.empty((DECODE["batch"], DECODE["k"]), dtype=torch.int32, device=dev)

    # Each phase of a step is captured G times in a CUDA graph (one replay =
    # G calls, inputs rotating), so host launch overhead stays off the device
    # timeline.  A step is one call of each phase.
    def phase_a(i):
        ds.ds_topk(xs[i % R], k1, return_value=True, out_idx=idx1, out_val=val1)

    def phase_b(i):
        ds.ds_topk(xs2[i % R], k2, return_value=True, out_idx=idx2, out_val=val2)

    def phase_c(i):
        ds.ds_indexer_topk(q_d, kcs[i % Rk], w_d, DECODE["k"], valid_len=vl_d, out_idx=didx)

    phases = (phase_a, phase_b, phase_c)
    # clocks and throttle reasons from the warm-up through the last section
    sampler = ClockSampler(gpu_uuid(dev))
    sampler.start()
    for i in range(args.warmup):
        for ph in phases:
            ph(i)
    torch.cuda.synchronize()
    status = ds.ds_get_device_status()
    if status != ds.DS_OK:
        raise RuntimeError(f"device status after warm-up: {ds.strerror(status)}")

    G = min(args.steps, 200)
    chunks = [G] * (args.steps // G) + ([args.steps % G] if args.steps % G else [])

    def capture(ph, count, first):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(count):
                ph(first + i)
        return g

    graphs = {}
    for c in sorted(set(chunks)):
        graphs[c] = [capture(ph, c, 0) for ph in phases]
    for c in graphs:                       # warm the graphs once
        for g in graphs[c]:
            g.replay()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in chunks]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for ci, c in enumerate(chunks):
        ga, gb, gc = graphs[c]
        evs[ci][0].record(stream)
        ga.replay()
        evs[ci][1].record(stream)
        gb.replay()
        evs[ci][2].record(stream)
        gc.replay()
        evs[ci][3].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    total_ms = t_start.elapsed_time(t_end)
    ph_ms = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])] for e in evs])
    t_k1, t_k2, t_dec = (ph_ms.sum(axis=0) / args.steps).tolist()        # ms per call
    total_ms, t_k1, t_k2, t_dec = max_over_ranks([total_ms, t_k1, t_k2, t_dec], dev)
    status = ds.ds_get_device_status()
    if status != ds.DS_OK:
        raise RuntimeError(f"device status after timing: {ds.strerror(status)}")

    # the same phase graphs replayed again, each replay alone: the spread
    rep_ms = {"k1024": [], "k64": [], "decode": []}
    c0 = chunks[0]
    for _ in range(5):
        for key, g in zip(("k1024", "k64", "decode"), graphs[c0]):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            rep_ms[key].append(e0.elapsed_time(e1) / c0)

    b1, b2 = topk_bytes(B, n, k1), topk_bytes(B, n, k2)
    topk_gbs = ws * (b1 + b2) / ((t_k1 + t_k2) * 1e-3) / 1e9
    per_launch_gbs = ((b1 + b2) / 2) / (((t_k1 + t_k2) / 2) * 1e-3) / 1e9
    dbytes, dflops = decode_bytes_flops(vl, DECODE["heads"], DECODE["d"], DECODE["k"])
    dec_roof_us = max(dbytes / (hbm_gbs * 1e9), dflops / (tflops * 1e12)) * 1e6

    # ---- end to end: pinned host logits in, selection back to host, every step
    x_pin = torch.from_numpy(x_host).pin_memory()
    x_dev = torch.empty_like(xs[0])
    out_pin = [torch.empty((B, k), dtype=torch.int32).pin_memory() for k in (k1, k2)]
    val_pin = [torch.empty((B, k), dtype=torch.float32).pin_memory() for k in (k1, k2)]
    e2e_steps = max(3, min(args.steps, 200))

    def e2e_step():
        x_dev.copy_(x_pin, non_blocking=True)
        for j, (k, oi, ov) in enumerate(((k1, idx1, val1), (k2, idx2, val2))):
            ds.ds_topk(x_dev, k, return_value=True, out_idx=oi, out_val=ov)
            out_pin[j].copy_(oi, non_blocking=True)
            val_pin[j].copy_(ov, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], dev)
    e2e_gbs = ws * (b1 + b2) / (e2e_ms * 1e-3) / 1e9
    h2d = xb
    d2h = B * (k1 + k2) * 8

    # ---- end to end, the decode step: queries, weights and valid lengths from
    # pinned host memory, the selection back to pinned host memory, every step
    q_pin = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).pin_memory()
    w_pin = torch.from_numpy(w).pin_memory()
    vl_pin = torch.from_numpy(vl).pin_memory()
    q_e, w_e, vl_e = torch.empty_like(q_d), torch.empty_like(w_d), torch.empty_like(vl_d)
    didx_pin = torch.empty((DECODE["batch"], DECODE["k"]), dtype=torch.int32).pin_memory()

    def e2e_dec(i):
        q_e.copy_(q_pin, non_blocking=True)
        w_e.copy_(w_pin, non_blocking=True)
        vl_e.copy_(vl_pin, non_blocking=True)
        ds.ds_indexer_topk(q_e, kcs[i % Rk], w_e, DECODE["k"], valid_len=vl_e, out_idx=didx)
        didx_pin.copy_(didx, non_blocking=True)

    for i in range(3):
        e2e_dec(i)
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_dec(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    (e2e_dec_us,) = max_over_ranks([e0.elapsed_time(e1) * 1e3 / e2e_steps], dev)
    e2e_dec_h2d = q_pin.numel() * 2 + w_pin.numel() * 4 + vl_pin.numel() * 4
    e2e_dec_d2h = didx_pin.numel() * 4

    # ---- prefill, reported beside the headline: 4096 query rows x 64 heads
    # against 32768 keys, causal valid_len, k = 2048 (indexer + top-k per call,
    # and the scorer alone for its tensor-pipe fraction)
    pq, pkc, pw, pvl = inputs.prefill(seed=inputs.SEED_PREFILL + rank)
    pq_d = torch.from_numpy(pq.view(np.int16)).view(torch.bfloat16).to(dev)
    pkc_d = torch.from_numpy(pkc.view(np.int16)).view(torch.bfloat16).to(dev)
    pw_d = torch.from_numpy(pw).to(dev)
    pvl_d = torch.from_numpy(pvl).to(dev)
    T = pq.shape[0]
    pidx = torch.empty((T, PREFILL["k"]), dtype=torch.int32, device=dev)
    pscore = torch.empty((T, pkc.shape[0]), dtype=torch.float32, device=dev)

    def time_calls(fn, calls=3):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(calls):
                fn()
        g.replay()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / calls

    pre_ms = time_calls(lambda: ds.ds_indexer_topk(pq_d, pkc_d, pw_d, PREFILL["k"], valid_len=pvl_d, out_idx=pidx))
    pre_score_ms = time_calls(lambda: ds.ds_indexer_score(pq_d, pkc_d, pw_d, valid_len=pvl_d, out=pscore))
    pre_ms, pre_score_ms = max_over_ranks([pre_ms, pre_score_ms], dev)
    del pscore
    pre_flops = 2.0 * pq.shape[1] * pq.shape[2] * float(np.sum(pvl.astype(np.int64)))
    status = ds.ds_get_device_status()
    if status != ds.DS_OK:
        raise RuntimeError(f"device status after prefill: {ds.strerror(status)}")

    # the floor under the top-k: a read-only pass over the same rows, launched
    # the same way (2 CTAs of 1024 threads per row), rotating the same copies
    floor_us = graph_times_us(lambda i: ds.ds_read_floor(xs[i % R], 2 * B), R, reps=5)
    (floor_med,) = max_over_ranks([statistics.median(floor_us)], dev)
    configs = measure_configs(ds, inputs, dev, rank, hbm_gbs, tflops)
    attention = measure_attention(ds, inputs, dev, stream, rank, hbm_gbs, tflops, ATTN_CALLS)
    qproj = measure_qproj(ds, inputs, dev, stream, rank, hbm_gbs, ATTN_CALLS)
    compress = measure_compress(ds, inputs, dev, rank)

    # DRAM bytes per launch of the dominant kernel from one ncu capture; null
    # once the kernel's source has changed since that capture
    traffic = None
    prof = os.path.join(ROOT, "profiles", "topk_traffic.json")
    try:
        import hashlib
        with open(prof) as f:
            pj = json.load(f)
        src = open(os.path.join(ROOT, "sparse_attention_top_ds_b200", "csrc", pj["kernel_source"]), "rb").read()
        if pj.get("kernel_source_sha256") == hashlib.sha256(src).hexdigest():
            traffic = pj.get("dram_bytes_per_launch")
    except Exception:
        traffic = None

    sampler.stop()
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        r = oracle_sample(seconds=10.0)
        cpu = {"value": round(r["topk_gbs"], 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
               "host_cpus": os.cpu_count(),
               "sample": f"{r['topk_rows']} whole sampling rows (k=1024 then 64), single thread; "
                         f"decode oracle {r['decode_us']:.0f} us/step on {r['decode_rows']} rows",
               "decode_us_per_step": round(r["decode_us"], 1),
               "per_config": oracle_configs()}

    clocks = sampler.summary()
    dflops_mean = dflops
    configs["sampling_64x129280_f32_k1024"] = dict(topk_config([m * 1e3 for m in rep_ms["k1024"]], B, n, k1, 4, True,
                                                               hbm_gbs), timed_steps_us=round(t_k1 * 1e3, 3))
    configs["sampling_64x129280_f32_k64"] = dict(topk_config([m * 1e3 for m in rep_ms["k64"]], B, n, k2, 4, True,
                                                             hbm_gbs), timed_steps_us=round(t_k2 * 1e3, 3))
    dec_med = statistics.median(rep_ms["decode"]) * 1e3
    configs["decode_8x64x128_vs_32768_k1024"] = {
        "us_per_step": spread([m * 1e3 for m in rep_ms["decode"]]), "timed_steps_us": round(t_dec * 1e3, 3),
        "rows_per_s": round(DECODE["batch"] / (dec_med * 1e-6), 1), "roofline_us": round(dec_roof_us, 3),
        "frac_of_roofline": round(dec_roof_us / dec_med, 3),
        "achieved_tflops": round(dflops_mean / (dec_med * 1e-6) / 1e12, 1), "algorithmic_bytes": int(dbytes),
        "e2e_us_per_step": round(e2e_dec_us, 2), "e2e_h2d_bytes": int(e2e_dec_h2d), "e2e_d2h_bytes": int(e2e_dec_d2h)}
    configs["prefill_4096x64x128_vs_32768_k2048"] = {
        "ms_per_call": round(pre_ms, 4), "rows_per_s": round(T / (pre_ms * 1e-3), 1),
        "scorer_ms_per_call": round(pre_score_ms, 4),
        "roofline_ms": round(pre_flops / (tflops * 1e12) * 1e3, 4),
        "frac_of_roofline": round(pre_flops / (tflops * 1e12) * 1e3 / pre_ms, 3)}
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(topk_gbs, 2), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "sampling top-k 64x129280 f32 (N(0,9) + 20 planted +15/row), k=1024 and k=64, "
                                   "values+indices, unsorted; plus decode indexer+top-k 8x64x128 bf16 vs 32768 "
                                   "bf16 keys, valid_len~U{4096..32768}, k=1024",
                       "global_batch": ws * B, "seq_len": n, "parallelism": f"replicas{ws}",
                       "l2": f"inputs rotate through 2x{R} logit copies and {Rk} key caches (> 2x L2 between reuses)"},
            "topk_pct_of_peak": round(100 * per_launch_gbs / hbm_gbs, 1),
            "topk_pct_of_nominal_8tbs": round(100 * per_launch_gbs / NOMINAL_HBM_GBS, 1),
            "topk_rows_per_s": round(2 * B / ((t_k1 + t_k2) * 1e-3), 1),
            "topk_us_per_call": {"k1024": round(t_k1 * 1e3, 2), "k64": round(t_k2 * 1e3, 2)},
            "topk_read_floor_us": {"us_per_call": round(floor_med, 2), "replays": spread(floor_us),
                                   "what": "a kernel that only reads the same 33.1 MB of rows, 128 CTAs x 1024 "
                                           "threads, 16-byte loads (ds_read_floor)"},
            "decode_us_per_step": round(t_dec * 1e3, 2),
            "decode_roofline_us": round(dec_roof_us, 3),
            "decode_frac_of_roofline": round(dec_roof_us / (t_dec * 1e3), 3),
            "prefill": {"workload": "4096 x 64 x 128 bf16 queries vs 32768 bf16 keys, causal valid_len, k=2048",
                        "ms_per_call": round(pre_ms, 4), "scorer_ms_per_call": round(pre_score_ms, 4),
                        "useful_tflop": round(pre_flops / 1e12, 4),
                        "scorer_tflops": round(pre_flops / (pre_score_ms * 1e-3) / 1e12, 1),
                        "scorer_frac_of_bf16_peak": round(pre_flops / (pre_score_ms * 1e-3) / 1e12 / tflops, 3),
                        "bf16_peak_tflops": tflops, "peak_kind": "burst (the scorer is timed alone, 3 calls)"},
            "configs": configs,
            "sparse_attention": attention,
            "qproj": qproj,
            "compress_fold": compress,
            "roofline": {"bound": "hbm", "achieved": round(per_launch_gbs, 1), "peak": hbm_gbs, "unit": "GB/s",
                         "frac": round(per_launch_gbs / hbm_gbs, 4), "traffic": traffic,
                         "kernel": TOPK_KERNEL, "peak_source": peak_src},
            "e2e": {"value": round(e2e_gbs, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["all", "attention", "qproj"] + list(ONLY_WORKLOADS), default="all",
                    help="time one part of the step alone (profiling): the sparse attention, the query "
                         "projection, or one selection workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only != "all":
        run_only(args)
    else:
        run_ours(args)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
