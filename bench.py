"""Benchmark of the FVAttn single-GPU hot path on B200.

One step = one attention layer through the C ABI: reorder Q, K, V into
spatio-temporal tiles -> route (block mean-pooling, block scores, Top-p with
a Top-k floor) -> block-sparse attention -> inverse reorder.  Inputs are the
seeded synthetic 720p-shaped layer (B=1, 40 heads, d=128, 21x45x80 latent,
2x8x8 blocks, p=0.9, k=16) already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fvattn|reference]

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs an
independent replica layer with its own seed: there is no exchange step in
this path, so scaling is weak and no collective touches the data.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
import types

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn TFLOPS on executed blocks (% of bf16 peak) + end-to-end ms per layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD = "720p"

# DRAM bytes (read + write) of one sparse_attn_kernel<128, 0> launch on the 720p layer: an ncu capture
# of the same layer restricted to 4 heads read 383.7 MB and wrote 75.6 MB; K/V reuse stays inside a
# head, so traffic scales with the head count (x10 for 40 heads).
ATTN_TRAFFIC_720P = {"bytes": (383.733504e6 + 75.581184e6) * 10,
                     "how": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the 4-head 720p layer, x10 heads"}
# The CFG 720p layer (B=2, 64-token blocks) restricted to 4 heads: 627.3 MB read, 152.1 MB written.
ATTN_TRAFFIC_CFG720P = {"bytes": (627.297792e6 + 152.127744e6) * 10,
                        "how": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the 4-head CFG 720p layer, "
                               "x10 heads"}
ATTN_TRAFFIC = {"720p": ATTN_TRAFFIC_720P, "cfg720p": ATTN_TRAFFIC_CFG720P}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w, g):
    return {
        "workload": f"{w.name}-shaped layer: B={w.B}, H={w.H}, D={w.D}, latent {w.F}x{w.Hs}x{w.Ws} "
                    f"= {w.N} tokens, {w.tf}x{w.th}x{w.tw} = {g.bs}-token blocks (nb={g.nb}), "
                    f"p={w.p}, k={w.k}",
        "global_batch": w.B, "seq_len": w.N, "heads": w.H, "head_dim": w.D,
        "block": f"{w.tf}x{w.th}x{w.tw}", "nb": g.nb, "p": w.p, "k_floor": w.k,
        "block_order": getattr(w, "order", "raster"),
        "l2": (f"no flush: every input tensor ({w.B * w.N * w.H * w.D * 2 / 1e6:.0f} MB raster) is larger "
               "than the 126 MB L2") if w.B * w.N * w.H * w.D * 2 > 126e6 else
              "small layer: inputs fit in L2 (no flush; not a bandwidth measurement)",
        "parallelism": "replicas (independent layer per GPU)",
    }


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)

def oracle_sample_time(w, qt, kt, vt, q_raster, kv_idx_full, kv_cnt_full, heads=8, items_per_head=16):
    """Time the oracle, as it stands, on a bounded sample of one layer and
    extrapolate to the whole layer.

    Sample: reorder of one raster tensor; routing (pool, scores, select) of
    `heads` heads; masked attention on `items_per_head` query blocks of each
    of those heads.  Extrapolation: reorder x4 (Q, K, V, inverse O), routing
    x H/heads, attention x (executed block pairs of the layer / of the
    sample).  Returns (seconds for the full layer, description, threads)."""
    import numpy as np
    from oracle import oracle as orc
    from block_sparse_attention_aware_b200 import synth
    orc.build_oracle()
    threads = orc.num_threads()
    t0 = time.perf_counter()
    orc.reorder(synth.bf16_bits(q_raster), w)
    t_reorder = time.perf_counter() - t0
    sub = synth.custom_workload(**{**w.as_dict(), "H": heads, "name": "sample"})
    hsel = list(range(heads))
    qb = synth.bf16_bits(qt[:, hsel].contiguous())
    kb = synth.bf16_bits(kt[:, hsel].contiguous())
    vb = synth.bf16_bits(vt[:, hsel].contiguous())
    t0 = time.perf_counter()
    _, _, _, idx, cnt, _, _ = orc.route(qb, kb, sub, w.p, w.k, 1.0 / math.sqrt(w.D))
    t_route = time.perf_counter() - t0
    nb = idx.shape[-1]
    items = []
    for h in range(heads):
        order = np.argsort(-cnt[0, h], kind="stable")
        picks = [int(order[(i * len(order)) // items_per_head]) for i in range(items_per_head)]
        items += [h * nb + i for i in picks]
    t0 = time.perf_counter()
    orc.attention(qb, kb, vb, idx, cnt, items, sub, 1.0 / math.sqrt(w.D))
    t_attn = time.perf_counter() - t0
    sample_pairs = int(sum(cnt.reshape(-1)[i] for i in items))
    layer_pairs = int(kv_cnt_full.sum())
    full = 4 * t_reorder + t_route * (w.H * w.B / heads) + t_attn * layer_pairs / max(sample_pairs, 1)
    desc = (f"oracle on {threads} host threads: reorder of 1 raster tensor (x4), routing of {heads} of "
            f"{w.B * w.H} heads (x{w.B * w.H / heads:g}), masked attention on {len(items)} query blocks "
            f"({sample_pairs} block pairs, scaled to the layer's {layer_pairs}); measured "
            f"{t_reorder + t_route + t_attn:.1f} s, extrapolated to {full:.1f} s per layer")
    return full, desc, threads, t_reorder + t_route + t_attn


def oracle_mask_parity(w, g, layer, q, k, e2e_heads=4):
    """Mask parity of the benchmarked step, checked by the oracle after the
    timed region (same leg as the CPU baseline, rank 0 only).

    One more pass of the step's routing call, with its debug logits output,
    gives the kv lists and the fp32 logits they were selected from.  The
    oracle's selection on those logits must give the same kept set in every
    row except rows it flags as near ties (cumulative mass within 1e-5 of p);
    all three counts are returned.  End-to-end mode: on `e2e_heads` heads the
    oracle also pools and scores the tiles itself and selects on its own
    logits; the rows whose kept set then differs are counted (not graded:
    logit rounding can move rows that sit near the p boundary)."""
    import numpy as np
    import torch
    from oracle import oracle as orc
    from block_sparse_attention_aware_b200 import fvattn, synth
    dev = q.device
    routed = fvattn.RouteOut(kv_idx=torch.empty_like(layer.routed.kv_idx),
                             kv_cnt=torch.empty_like(layer.routed.kv_cnt),
                             logits=torch.empty((g.B, g.H, g.nb, g.nb), dtype=torch.float32, device=dev))
    if layer.fused_route:
        fvattn.reorder_route(layer.g, q, k, layer.p, layer.k, layer.scale, out=routed, qt=layer.qt, kt=layer.kt,
                             workspace=layer.route_ws)
    else:
        fvattn.route(layer.g, layer.qt, layer.kt, layer.p, layer.k, layer.scale, out=routed,
                     workspace=layer.route_ws)
    torch.cuda.synchronize()
    same_as_step = bool(torch.equal(routed.kv_cnt, layer.routed.kv_cnt))
    nb = g.nb
    cnt_g = routed.kv_cnt.cpu().numpy().reshape(-1)
    idx_g = routed.kv_idx.cpu().numpy().reshape(-1, nb)
    t0 = time.perf_counter()
    idx_o, cnt_o, _, tie = orc.select(routed.logits.cpu().numpy().reshape(-1, nb), w.p, w.k)

    def differing(ig, cg, io, co):
        bad = set(np.nonzero(cg != co)[0].tolist())
        for r in np.nonzero(cg == co)[0]:
            if not np.array_equal(ig[r, :cg[r]], io[r, :co[r]]):
                bad.add(int(r))
        return sorted(bad)

    bad = differing(idx_g, cnt_g, idx_o, cnt_o)
    unexcused = [r for r in bad if not tie[r]]
    BH = g.B * g.H
    heads = sorted({0, BH // 2, BH - 1} | set(synth.sample_items(BH, max(e2e_heads - 3, 0), seed=11)))
    sub = synth.custom_workload(**{**w.as_dict(), "B": 1, "H": len(heads), "name": "sample"})
    sel = torch.tensor(heads, device=dev)
    qb = synth.bf16_bits(layer.qt.view(BH, g.Npad, g.D)[sel].unsqueeze(0))
    kb = synth.bf16_bits(layer.kt.view(BH, g.Npad, g.D)[sel].unsqueeze(0))
    _, _, _, idx_e, cnt_e, _, _ = orc.route(qb, kb, sub, w.p, w.k, layer.scale)
    hs = np.array(heads)
    e2e_bad = differing(idx_g.reshape(BH, nb, nb)[hs].reshape(-1, nb), cnt_g.reshape(BH, nb)[hs].reshape(-1),
                        idx_e.reshape(-1, nb), cnt_e.reshape(-1))
    return {"rows": int(len(cnt_g)), "near_tie_rows": int(tie.sum()), "mismatched_rows": len(bad),
            "unexcused": len(unexcused), "near_tie_band": orc.TIE_BAND,
            "kv_lists_equal_timed_step": same_as_step,
            "how": "oracle selection on the GPU's own fp32 logits, every row of the layer",
            "e2e": {"heads": heads, "rows": int(len(hs) * nb), "mismatched_rows": len(e2e_bad),
                    "how": "oracle pools, scores and selects the tiles of these heads by itself"},
            "oracle_seconds": time.perf_counter() - t0}


def run_reference(args):
    """The oracle timed as the reference arm (rank 0; other ranks exit)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    from block_sparse_attention_aware_b200 import synth
    w = synth.WORKLOADS[WORKLOAD]
    q, k, v, _ = synth.make_qkv(w, device="cpu")
    from oracle import oracle as orc
    orc.build_oracle()
    qt = torch.from_numpy(orc.reorder(synth.bf16_bits(q), w).view("int16")).view(torch.bfloat16)
    kt = torch.from_numpy(orc.reorder(synth.bf16_bits(k), w).view("int16")).view(torch.bfloat16)
    vt = torch.from_numpy(orc.reorder(synth.bf16_bits(v), w).view("int16")).view(torch.bfloat16)
    # full-layer routing counts (needed for the executed-pair total)
    _, _, _, _, cnt_full, _, _ = orc.route(synth.bf16_bits(qt), synth.bf16_bits(kt), w, w.p, w.k,
                                           1.0 / math.sqrt(w.D))
    geo = orc.geometry(w)
    flops = 4.0 * geo["bs"] * geo["bs"] * w.D * float(cnt_full.sum())
    times, descs = [], []
    for i in range(args.warmup + args.steps):
        full, desc, threads, _ = oracle_sample_time(w, qt, kt, vt, q, None, cnt_full)
        if i >= args.warmup:
            times.append(full)
            descs.append(desc)
    t = statistics.mean(times)
    val = flops / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded, CPU generator)",
        "config": workload_config(w, types.SimpleNamespace(bs=geo["bs"], nb=geo["nb"])),
        "cpu_baseline": {"kind": "oracle", "value": val, "unit": "TFLOP/s", "cores": threads,
                         "sample": descs[-1]},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ranks

def aggregate_over_ranks(t_local: float, work_local: float, world: int, device):
    """Whole-job figures of a replicated step: the slowest rank's time (the
    job finishes when it does) and the work of all ranks.  Every rank calls
    this with its own values; with one rank it returns them unchanged."""
    import torch
    if world <= 1:
        return float(t_local), float(work_local)
    import torch.distributed as dist
    t = torch.tensor([t_local], dtype=torch.float64, device=device)
    wk = torch.tensor([work_local], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(wk, op=dist.ReduceOp.SUM)
    return float(t.item()), float(wk.item())


# ---------------------------------------------------------------- GPU arm

NOMINAL_DENSE_BF16_TFLOPS = 2250.0   # NVIDIA's B200 dense bf16 figure (context only)


def block_real_counts(g, tile_of_block=None):
    """Real (non-padding) tokens of each block: the tile's clipped extent.
    tile_of_block: the block -> raster tile table (Hilbert order), or None."""
    counts = []
    for blk in range(g.nb):
        t = blk if tile_of_block is None else int(tile_of_block[blk])
        bx, by, bf = t % g.nbx, (t // g.nbx) % g.nby, t // (g.nbx * g.nby)
        counts.append(min(g.tf, g.F - bf * g.tf) * min(g.th, g.Hs - by * g.th) * min(g.tw, g.Ws - bx * g.tw))
    return counts


def valid_token_flops(g, kv_idx, kv_cnt, counts, rows_per_chunk=64):
    """Attention FLOPs over real tokens only: 4 * D * sum over (b, h, i) of
    n_i * sum of n_j over the kept blocks j (entries past kv_cnt ignored)."""
    import torch
    nb = g.nb
    n = torch.as_tensor(counts, dtype=torch.float64, device=kv_idx.device)
    idx = kv_idx.reshape(-1, nb, nb)
    cnt = kv_cnt.reshape(-1, nb)
    pos = torch.arange(nb, device=kv_idx.device)
    total = 0.0
    for r0 in range(0, idx.shape[0], rows_per_chunk):
        i = idx[r0:r0 + rows_per_chunk].long().clamp(0, nb - 1)
        used = pos[None, None, :] < cnt[r0:r0 + rows_per_chunk, :, None]
        kept = torch.where(used, n[i], torch.zeros((), dtype=torch.float64, device=n.device)).sum(dim=-1)
        total += float((kept * n[None, :]).sum())
    return 4.0 * g.D * total


def _imbalance(layer, nsm):
    import numpy as np
    st = layer.sm_stats.cpu().numpy().astype(np.float64)
    busy = st[:nsm]
    used = busy > 0
    return float(busy[used].max() / busy[used].mean()) if used.any() else None


def p_sweep(layer, w, g, nsm, stream):
    """Route + attend at each p of the workload's sweep; per-head kept blocks
    and the SM busy-time imbalance of the attention kernel."""
    import torch
    out = []
    for p in w.p_sweep:
        layer.p = p
        layer.route()
        layer.attend(stats=True)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        layer.route()
        e1.record(stream)
        layer.attend(stats=True)
        e2.record(stream)
        torch.cuda.synchronize()
        cnt = layer.routed.kv_cnt
        pairs = int(cnt.sum())
        per_head = cnt.view(g.B * g.H, g.nb).sum(dim=1).cpu().tolist()
        ms = e1.elapsed_time(e2)
        out.append({"p": p, "density": pairs / float(g.B * g.H * g.nb * g.nb), "executed_block_pairs": pairs,
                    "route_ms": e0.elapsed_time(e1), "attention_ms": ms,
                    "attention_tflops": 4.0 * g.bs * g.bs * g.D * pairs / (ms / 1e3) / 1e12,
                    "sm_imbalance_max_over_mean": _imbalance(layer, nsm),
                    "head_blocks": per_head,
                    "head_blocks_max_over_mean": max(per_head) / (sum(per_head) / len(per_head))})
    return out


def layer_stack(layer, w, g, dev, stream, barrier):
    """Every seeded layer of the workload once: inputs drawn (untimed), then
    one whole layer step timed with CUDA events; the stack time is the sum."""
    import torch
    from block_sparse_attention_aware_b200 import synth
    per_layer, flops = [], 0.0
    for li in range(w.layers):
        q, k, v, _ = synth.make_qkv(w, layer=li, device=dev)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer(q, k, v)
        e1.record(stream)
        torch.cuda.synchronize()
        per_layer.append(e0.elapsed_time(e1))
        flops += 4.0 * g.bs * g.bs * g.D * float(layer.routed.kv_cnt.sum())
        del q, k, v
    total = sum(per_layer)
    return {"layers": w.layers, "total_ms": total, "per_layer_ms": per_layer,
            "tflops_executed_blocks": flops / (total / 1e3) / 1e12,
            "note": "each layer step timed alone (inputs of 40 layers do not fit in HBM together)"}


def run_fvattn(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    from block_sparse_attention_aware_b200 import fvattn, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    fvattn.load()
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        w = synth.custom_workload(**{**w.as_dict(), "H": args.heads, "name": f"{w.name}-h{args.heads}"})
    if args.order != w.order:
        w = synth.custom_workload(**{**w.as_dict(), "order": args.order})
    g = fvattn.geom_of(w)
    dev = torch.device("cuda", local)
    # each rank: its own seeded replica layer
    q, k, v, _ = synth.make_qkv(w, layer=rank, device=dev)
    fused = not args.unfused_route
    layer = fvattn.Layer(g, w.p, w.k, device=dev, order=args.order, fused_route=fused)
    g = layer.g
    stream = torch.cuda.current_stream(dev)
    nsm = fvattn.num_sms()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        layer(q, k, v, stats=True)
    torch.cuda.synchronize()
    assert fvattn.get_status() == 0, "device status after warm-up"

    # timed region: K full steps, CUDA events per stage on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    start.record(stream)
    for i in range(args.steps):
        e = ev[i]
        e[0].record(stream)
        if fused:
            layer.reorder_route(q, k)
            e[1].record(stream)
            layer.reorder_v(v)
        else:
            layer.reorder_qkv(q, k, v)
            e[1].record(stream)
            layer.route()
        e[2].record(stream)
        layer.attend(stats=True)
        e[3].record(stream)
        layer.restore()
        e[4].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    barrier()
    status = fvattn.get_status()
    assert status == 0, f"device status {status}"
    t_total = start.elapsed_time(end) / 1e3
    cnt = layer.routed.kv_cnt
    pairs = int(cnt.sum())
    flops = 4.0 * g.bs * g.bs * g.D * pairs
    t_max, flops_all = aggregate_over_ranks(t_total, flops, world, dev)

    names = (("reorder_route_qk", "reorder_v") if fused else ("reorder_qkv", "route")) + \
        ("attention", "inverse_reorder")
    stage = {n: [] for n in names}
    for e in ev:
        for j, n in enumerate(names):
            stage[n].append(e[j].elapsed_time(e[j + 1]))
    ms = {kk: statistics.mean(vv) for kk, vv in stage.items()}
    if fused:
        # routing alone (pooling from the tiles, scoring, selection) on the tiles the step wrote,
        # for its own bandwidth figure; the same kv lists come out
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        layer.route()
        r0.record(stream)
        for _ in range(args.steps):
            layer.route()
        r1.record(stream)
        torch.cuda.synchronize()
        ms["route_alone"] = r0.elapsed_time(r1) / args.steps
    peaks, peak_src = load_peaks()
    raster_bytes = g.B * g.N * g.H * g.D * 2
    tiled_bytes = g.B * g.H * g.Npad * g.D * 2
    attn_s = ms["attention"] / 1e3
    attn_tflops = flops / attn_s / 1e12
    kv_bytes = 4 * pairs + 4 * cnt.numel()
    route_bytes = 2 * tiled_bytes * (g.N / g.Npad) + kv_bytes
    route_gbs = route_bytes / (ms["route_alone" if fused else "route"] / 1e3) / 1e9
    inverse_gbs = (raster_bytes + tiled_bytes) / (ms["inverse_reorder"] / 1e3) / 1e9
    gbs = {"route": route_gbs, "inverse_reorder": inverse_gbs,
           "route_pct_of_hbm": 100.0 * route_gbs / peaks["hbm_gbs"]}
    if fused:
        # fused stage: raster Q, K read once, their tiles and the kv lists written
        fr_bytes = 2 * (raster_bytes + tiled_bytes) + kv_bytes
        gbs["reorder_route_qk"] = fr_bytes / (ms["reorder_route_qk"] / 1e3) / 1e9
        gbs["reorder_route_qk_pct_of_hbm"] = 100.0 * gbs["reorder_route_qk"] / peaks["hbm_gbs"]
        gbs["reorder_v"] = (raster_bytes + tiled_bytes) / (ms["reorder_v"] / 1e3) / 1e9
    else:
        gbs["reorder_qkv"] = 3 * (raster_bytes + tiled_bytes) / (ms["reorder_qkv"] / 1e3) / 1e9
    st = layer.sm_stats.cpu().numpy().astype(np.float64)
    busy, blocks = st[:nsm], st[nsm:2 * nsm]
    used = busy > 0
    imb = float(busy[used].max() / busy[used].mean()) if used.any() else None
    imb_pred = float(blocks[used].max() / blocks[used].mean()) if used.any() else None
    per_head = cnt.view(g.B * g.H, g.nb).sum(dim=1).double().cpu().numpy()
    sustained = peaks["bf16_tflops_sustained"]
    table = layer.order_table[: g.nb].cpu().tolist() if layer.order_table is not None else None
    vflops = valid_token_flops(g, layer.routed.kv_idx, cnt, block_real_counts(g, table))

    line = {
        "metric": METRIC,
        "value": flops_all / (t_max / args.steps) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_max / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": (f"synthetic: seeded Gaussian Wan2.2 {w.name}-shaped Q/K/V (seed {w.seed}+rank), "
                 + {"loguniform": "per-head log-uniform Q scales in [0.25, 4]",
                    "skew": "Q scale 4 on heads 0-19 and 0.25 on heads 20-39",
                    "fixed": f"fixed per-head Q scales {list(w.qscale_values)}"}[w.qscale]
                 + (", shared rank-8 spatio-temporal component" if w.lowrank else "")),
        "config": workload_config(w, g),
        "value_note": "executed-block attention FLOPs of all ranks / (max-over-ranks time of one whole "
                      "layer step: " + ("reorder+route of Q/K in one pass + reorder V" if fused else
                                        "reorder x3 + route") + " + attention + inverse reorder)",
        "attention": {
            "tflops_executed_blocks": attn_tflops,
            "pct_of_bf16_peak_burst": 100.0 * attn_tflops / peaks["bf16_tflops"],
            "pct_of_bf16_peak_sustained": 100.0 * attn_tflops / sustained,
            "pct_of_nominal_dense_bf16": 100.0 * attn_tflops / NOMINAL_DENSE_BF16_TFLOPS,
            "tflops_valid_tokens": vflops / attn_s / 1e12,
            "valid_token_flop_fraction": vflops / flops,
            "ms": ms["attention"], "density": pairs / float(g.B * g.H * g.nb * g.nb),
            "executed_block_pairs": pairs,
            "sm_imbalance_max_over_mean": imb, "sm_imbalance_predicted_from_blocks": imb_pred,
            "head_blocks_max_over_mean": float(per_head.max() / per_head.mean()),
        },
        "stages_ms": ms,
        "stages_gbs": gbs,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": sustained, "unit": "TFLOP/s",
                     "frac": attn_tflops / sustained,
                     "traffic": ATTN_TRAFFIC[w.name]["bytes"] if (w.name in ATTN_TRAFFIC and not args.heads) else None,
                     "traffic_how": ATTN_TRAFFIC[w.name]["how"] if (w.name in ATTN_TRAFFIC and not args.heads) else None,
                     "algorithmic_bytes_per_launch": 4 * tiled_bytes,
                     "kernel": f"sparse_attn_kernel<{g.D}, {int(g.bs < 128)}>",
                     "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside back-to-back steps)",
                     "algorithmic_flops_per_launch": flops},
        "gpu_launches": layer.kernel_launches() * args.steps,
        "clocks": clock_info,
    }

    # the same step with the inverse reorder fused into the attention epilogue
    ef0, ef1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    layer(q, k, v, fused_inverse=True)
    ef0.record(stream)
    for _ in range(args.steps):
        layer(q, k, v, fused_inverse=True)
    ef1.record(stream)
    torch.cuda.synchronize()
    line["fused_inverse_step_ms"] = ef0.elapsed_time(ef1) / args.steps

    # the step with the other routing path (separate reorders and routing, or the fused call)
    layer.fused_route = not fused
    layer(q, k, v)
    ef0.record(stream)
    for _ in range(args.steps):
        layer(q, k, v)
    ef1.record(stream)
    torch.cuda.synchronize()
    line["unfused_route_step_ms" if fused else "fused_route_step_ms"] = ef0.elapsed_time(ef1) / args.steps
    layer.fused_route = fused

    # p sweep (load-skew workload): per p, one routed + attended step after one warm-up
    if w.p_sweep:
        line["sweep"] = p_sweep(layer, w, g, nsm, stream)
        layer.p = w.p

    # full-depth stack: every seeded layer once (inputs drawn outside the timed region)
    if w.layers > 1 and args.stack:
        line["stack"] = layer_stack(layer, w, g, dev, stream, barrier)

    # end to end through the public API from pinned host buffers: the head-group pipeline
    # (uploads, compute and downloads of different head groups overlap)
    if args.e2e_steps > 0:
        qh = q.cpu().pin_memory()
        kh = k.cpu().pin_memory()
        vh = v.cpu().pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        groups = args.e2e_groups or fvattn.default_head_group_sizes(g.H)
        pipe = fvattn.HostPipeline(fvattn.geom_of(w), w.p, w.k, groups=groups, device=dev, order=args.order,
                                   fused_route=fused)
        pipe(qh, kh, vh, oh)
        torch.cuda.synchronize()
        barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.e2e_steps):
            pipe(qh, kh, vh, oh)
        s1.record(stream)
        torch.cuda.synchronize()
        te, _ = aggregate_over_ranks(s0.elapsed_time(s1) / 1e3, 0.0, world, dev)
        te /= args.e2e_steps
        line["e2e"] = {"value": flops_all / te / 1e12, "unit": "TFLOP/s", "ms_per_step": te * 1e3,
                       "h2d_bytes_per_step": 3 * raster_bytes, "d2h_bytes_per_step": raster_bytes,
                       "steps": args.e2e_steps, "head_groups": pipe.sizes,
                       "how": "fvattn.HostPipeline: per head group, 2-D H2D copies of Q/K/V, the layer's calls "
                              "(Q/K reorder + routing in one pass, V reorder, attention, inverse reorder), "
                              "2-D D2H copy of O; groups overlap on two copy streams and the compute stream"}

    # oracle leg (rank 0, one GPU, after every timed region): the CPU baseline and the mask parity
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["mask_parity"] = oracle_mask_parity(w, g, layer, q, k)
        full, desc, threads, spent = oracle_sample_time(
            w, layer.qt.cpu(), layer.kt.cpu(), layer.vt.cpu(), q.cpu(), None, cnt.cpu().numpy())
        line["cpu_baseline"] = {"value": flops / full / 1e12, "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "sample": desc, "sample_seconds": spent}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="fvattn", choices=["fvattn", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle leg (CPU baseline timing and mask parity)")
    ap.add_argument("--workload", default=WORKLOAD, help="named workload of synth.WORKLOADS")
    ap.add_argument("--order", default="raster", choices=["raster", "hilbert"],
                    help="block order of the tiles (raster tile order or the 3-D Hilbert curve)")
    ap.add_argument("--stack", action="store_true",
                    help="also time every seeded layer of a multi-layer workload once (cfg720p: 40 layers)")
    ap.add_argument("--e2e-groups", type=int, default=0,
                    help="equal head groups of the end-to-end pipeline (uploads, compute and downloads "
                         "overlap); 0: fvattn.default_head_group_sizes (two heads a group, one in the first "
                         "and the last: 21 groups for 40 heads)")
    ap.add_argument("--unfused-route", action="store_true",
                    help="time the step with separate reorders and routing instead of the fused call")
    ap.add_argument("--heads", type=int, default=0,
                    help="profiling-size variant: the same layer with fewer heads (0 = all)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_fvattn(args)


if __name__ == "__main__":
    main()
