"""Benchmark: decode step of IsoQuant compressed-space attention on B200.

Workload (default): GQA decode, batch 16, 32 query / 4 KV heads, d = 128,
context 32768 (bf16 heavy-tailed K/V compressed into a paged 3-bit cache
with 256-token pages and a shuffled page table).  One step = append one new
token per sequence and rotate the queries (isoquant_decode_prep, one
launch), then split-context attention over the packed codes with the merge
of the splits and the inverse rotation (isoquant_attend_decode: the partial
and combine kernels): every row of the hot path.  The kernels are
programmatic dependent launches, so each one's launch overlaps the tail of
the one before.  The end-to-end figure drives the same step through the
one-call isoquant_decode_step.

Metric: KV-token x KV-head pairs attended per second (sum over sequences of
the context length times the KV heads, per step), and the achieved HBM
bandwidth of the attention kernel on the 108 compressed bytes per KV
token-head, against the measured copy bandwidth of this GPU.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 it is launched with torchrun, one rank per GPU; every rank runs its
own shard (weak scaling) and rank 0 prints the line.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention KV-token·heads/s on packed 3-bit KV; achieved HBM GB/s vs ~8 TB/s"
UNIT = "KV-token·heads/s"
DEFAULT_WORKLOAD = "gqa_b16_q32_kv4_L32768_paged"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            mp = json.load(f)
        return float(mp["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peak():
    """Measured sustained dense bf16 tensor throughput (TFLOP/s): the fp16
    products run at the same rate, in a step that keeps them busy for
    seconds."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            mp = json.load(f)
        return float(mp["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        return 1400.0, "fallback (sustained)"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stage_layout(tensors, align=256):
    """Byte layout of one pinned staging row holding the given tensors back to
    back: a list of (offset, bytes, dtype, shape) with every offset a multiple
    of `align`, and the row's total size."""
    layout, row_bytes = [], 0
    for t in tensors:
        n = t.numel() * t.element_size()
        layout.append((row_bytes, n, t.dtype, t.shape))
        row_bytes += (n + align - 1) // align * align
    return layout, row_bytes


def profiled_traffic(kernel_src, bytes_per_launch):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    summary, scaled from the captured launch to this one by the algorithmic
    bytes (traffic grows in proportion to the pages streamed), or None when
    the kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "attend_partial_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("source_hash") != source_hash(*kernel_src):
        return None
    return d["traffic_bytes_per_launch"] * bytes_per_launch / d["algorithmic_bytes_per_launch"]


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons, n = [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                except ValueError:
                    continue
                n += 1
                for nm, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": n}


def clocks_or_resample(clocks, uuid, run_once, dev, seconds=0.5):
    """The clocks sampled over a timed region, or, when that region was too
    short for nvidia-smi to take a sample (it polls every 50 ms), the clocks
    over untimed repeats of the same step run right after it, said so."""
    if clocks.get("samples", 0) > 0:
        return clocks
    import torch
    sampler = ClockSampler(uuid)
    sampler.start()
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        run_once()
        torch.cuda.synchronize(dev)
    c = sampler.stop()
    c["note"] = "sampled over untimed repeats of the step right after the timed region (too short to sample)"
    return c


GRAPH_STEPS = 32  # decode steps (or attention calls) per CUDA graph under --graph


# ---------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    import compressed_space_decode_b200 as csd
    from compressed_space_decode_b200 import multi, synthetic
    from compressed_space_decode_b200.workload import DecodeState

    rank, local_rank, world = multi.env_rank()
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)

    wl = multi.shard_workload(synthetic.workloads()[args.workload], rank, world)
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    # tokens each step appends per sequence: one for decode; a causal chunk
    # of nq query positions (verification) appends its nq tokens
    adv = wl.nq if wl.causal else 1
    growth = (args.warmup + args.steps + e2e_steps + 2) * adv
    st = DecodeState(wl, growth=growth, device=dev, bits=args.bits)
    bytes_per_token_head = 2 * (csd.WORDS_FOR[args.bits] * 4 + 2)
    B, H, Hq, nq = st.B, st.H, st.Hq, wl.nq
    if args.graph:
        # graphs are captured on a side stream (not the legacy default one),
        # which then stays the current stream for the whole run
        torch.cuda.synchronize(dev)
        torch.cuda.set_stream(torch.cuda.Stream(device=dev))
    stream = torch.cuda.current_stream(dev)

    # per-step inputs, generated up front (device-resident for the kernel metric)
    n_total = args.warmup + args.steps
    lens0 = list(st.seq_lens)
    # step s appends tokens lens0[b] + s adv + a (a < adv) of every sequence b,
    # ordered (a, b) like their slots
    k_all = torch.empty((n_total, adv, B, H, 128), dtype=torch.bfloat16, device=dev)
    v_all = torch.empty_like(k_all)
    for b in range(B):
        k, v = st.kv_tokens(b, lens0[b], lens0[b] + n_total * adv)
        k_all[:, :, b] = k.view(n_total, adv, H, 128)
        v_all[:, :, b] = v.view(n_total, adv, H, 128)
    k_all = k_all.view(n_total, adv * B, H, 128)
    v_all = v_all.view(n_total, adv * B, H, 128)
    q_all = synthetic.gaussian(wl.seed, 20_000_000, (n_total, B * nq, Hq, 128), device=dev, dtype=torch.bfloat16)
    slots_all = st.slot_matrix(lens0, n_total * adv).reshape(n_total, adv * B)
    lens_all = torch.tensor([[L + (s + 1) * adv for L in lens0] for s in range(n_total)], dtype=torch.int32,
                            device=dev)
    q_rot = torch.empty((B, nq, Hq, 128), dtype=torch.float32, device=dev)
    out = torch.empty_like(q_rot)
    ws = csd.alloc_workspace(st.ctx, B, nq, Hq, device=dev)
    launches = [0]

    def step(s, k, v, q, slots, lens):
        # append + rotate q (one launch), then attention (partial + combine):
        # the launches of isoquant_decode_step, issued as its two halves so
        # that events can bracket the attention
        csd.isoquant_decode_prep(st.ctx, st.cache, k, v, slots, q, q_rot.view(B * nq, Hq, 128), stream=stream)
        launches[0] += csd.isoquant_last_launch_count(st.ctx)
        ev = attn_events.get(s) if attn_events is not None else None
        if ev is not None:
            ev[0].record(stream)
        csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, lens, ws, out, causal=wl.causal,
                                   stream=stream)
        launches[0] += csd.isoquant_last_launch_count(st.ctx)
        if ev is not None:
            ev[1].record(stream)

    attn_events = None
    for s in range(args.warmup):
        step(s, k_all[s], v_all[s], q_all[s], slots_all[s], lens_all[s])
    torch.cuda.synchronize(dev)

    # the attention call's own duration, from events around it on every 8th
    # timed step (events between the launches of every step would break the
    # programmatic launch overlap of the whole run)
    attn_events = {s: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for s in range(args.warmup, n_total, 8)}
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    launches[0] = 0
    graphs = []
    if args.graph:
        # --graph: the timed steps are captured up front as CUDA graphs of
        # GRAPH_STEPS consecutive steps each (every step its own inputs, so
        # the context grows as without graphs) and replayed in order, so the
        # host's per-call cost is off the timed path
        attn_events = {}
        for c0 in range(args.warmup, n_total, GRAPH_STEPS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for s in range(c0, min(c0 + GRAPH_STEPS, n_total)):
                    step(s, k_all[s], v_all[s], q_all[s], slots_all[s], lens_all[s])
            graphs.append(g)
    multi.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    if args.graph:
        for g in graphs:
            g.replay()
    else:
        for s in range(args.warmup, n_total):
            step(s, k_all[s], v_all[s], q_all[s], slots_all[s], lens_all[s])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    multi.barrier()
    ms_local = t_start.elapsed_time(t_end)
    kernel_launches = launches[0]
    attn_ms = [e0.elapsed_time(e1) for e0, e1 in attn_events.values()]
    attn_avg_ms = sum(attn_ms) / len(attn_ms) if attn_ms else ms_local / args.steps

    units_local = sum(int(lens_all[s].sum().item()) * H for s in range(args.warmup, n_total))
    ms = multi.max_over_ranks(ms_local, device=dev)
    units = multi.sum_over_ranks(units_local, device=dev)
    value = units / (ms / 1e3)

    # the attention call alone, repeated for >= --attn-seconds so that the
    # roofline rests on thousands of launches and the clock sampler sees
    # them: CUDA events around every call on the launching stream (median),
    # over the cache as the timed loop left it (larger than L2)
    lens_last = lens_all[n_total - 1]
    n_attn = max(200, int(math.ceil(args.attn_seconds * 1e3 / max(attn_avg_ms, 1e-3))))
    attn_launches = 0
    if args.graph:
        # the attention call GRAPH_STEPS times in one graph; events around
        # each replay, per-call time = replay time / GRAPH_STEPS
        ga = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ga, stream=stream):
            for _ in range(GRAPH_STEPS):
                csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, lens_last, ws, out,
                                           causal=wl.causal, stream=stream)
        n_attn = GRAPH_STEPS * max(1, n_attn // GRAPH_STEPS)
    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_attn // GRAPH_STEPS if args.graph else n_attn)]
    multi.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(uuid)
    sampler.start()
    for ea, eb in attn_ev:
        ea.record(stream)
        if args.graph:
            ga.replay()
        else:
            csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, lens_last, ws, out, causal=wl.causal,
                                       stream=stream)
            attn_launches += csd.isoquant_last_launch_count(st.ctx)
        eb.record(stream)
    torch.cuda.synchronize(dev)
    clocks_attn = sampler.stop()
    multi.barrier()
    per_call = GRAPH_STEPS if args.graph else 1
    loop_ms = sorted(ea.elapsed_time(eb) / per_call for ea, eb in attn_ev)
    attn_med_ms = loop_ms[len(loop_ms) // 2]

    # roofline of the attention kernel: algorithmic bytes per launch / duration
    bytes_per_launch = bytes_per_token_head * int(lens_last.sum().item()) * H
    bytes_in_step = bytes_per_token_head * units_local / args.steps
    achieved = bytes_per_launch / (attn_med_ms / 1e3) / 1e9
    # (under --graph no events sit between a step's launches: no in-step figure)
    achieved_in_step = bytes_in_step / (attn_avg_ms / 1e3) / 1e9 if attn_ms else None
    peak, peak_kind = peaks()
    # the profiled traffic is that of the 3-bit mma.sync kernel
    traffic = None  # set below once the kernel is known

    # end to end through the public API from pinned host buffers
    attn_events = None
    st.seq_lens = [L + n_total * adv for L in lens0]
    base = n_total * adv
    # a step's inputs (k | v | q | slots | lens) sit in one pinned staging row
    # and cross to the device in one transfer, as a serving loop would stage them
    kd, vd = torch.empty_like(k_all[0]), torch.empty_like(v_all[0])
    qd, sd, ld = torch.empty_like(q_all[0]), torch.empty_like(slots_all[0]), torch.empty_like(lens_all[0])
    layout, row_bytes = stage_layout((kd, vd, qd, sd, ld))
    # two device staging rows and two outputs, so that a step's copies overlap
    # the neighbouring steps' kernels
    stage_ds = [torch.empty(row_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dviews = [[sd_[o:o + n].view(dt).view(shp) for o, n, dt, shp in layout] for sd_ in stage_ds]
    outs = [out, torch.empty_like(out)]
    stage_h = torch.zeros((e2e_steps, row_bytes), dtype=torch.uint8).pin_memory()
    host_views = [[stage_h[s, o:o + n].view(dt).view(shp) for o, n, dt, shp in layout] for s in range(e2e_steps)]
    lens_e2e = [[L + base + (s + 1) * adv for L in lens0] for s in range(e2e_steps)]
    for b in range(B):
        k, v = st.kv_tokens(b, lens0[b] + base, lens0[b] + base + e2e_steps * adv)
        k, v = k.cpu().view(e2e_steps, adv, H, 128), v.cpu().view(e2e_steps, adv, H, 128)
        for s in range(e2e_steps):
            host_views[s][0].view(adv, B, H, 128)[:, b] = k[s]
            host_views[s][1].view(adv, B, H, 128)[:, b] = v[s]
    slots_h = st.slot_matrix([L + base for L in lens0], e2e_steps * adv).reshape(e2e_steps, adv * B).cpu()
    for s in range(e2e_steps):
        host_views[s][2].copy_(q_all[s].cpu())
        host_views[s][3].copy_(slots_h[s])
        host_views[s][4].copy_(torch.tensor(lens_e2e[s], dtype=torch.int32))
    out_h = torch.empty((e2e_steps, B, nq, Hq, 128), dtype=torch.float32).pin_memory()
    h2d = sum(n for _, n, _, _ in layout)
    d2h = out.numel() * 4
    ws_step = csd.alloc_step_workspace(st.ctx, B, nq, Hq, device=dev)
    # copies on their own streams, one per direction (the link is full
    # duplex): step s + 1's inputs go in while step s computes, step s's
    # output comes back while step s + 1 computes; events order each buffer's
    # reuse (inputs of step s + 2 after step s's kernels, its output after
    # step s's read-back).  For steps of a few KB the extra stream and event
    # calls cost the host more than the copies take, so those run in line.
    overlap = h2d + d2h >= 65536
    if overlap:
        h2d_stream, d2h_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    else:
        h2d_stream = d2h_stream = stream
    ev_in = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_out = [torch.cuda.Event() for _ in range(e2e_steps)]

    def copy_in(s):
        if s >= 2:
            h2d_stream.wait_event(ev_done[s - 2])
        with torch.cuda.stream(h2d_stream):
            stage_ds[s % 2].copy_(stage_h[s], non_blocking=True)
        ev_in[s].record(h2d_stream)

    def step_in_line(s):
        kd, vd, qd, sd, ld = dviews[s % 2]
        stage_ds[s % 2].copy_(stage_h[s], non_blocking=True)
        csd.isoquant_decode_step(st.ctx, st.cache, kd, vd, sd, qd.view(B, nq, Hq, 128), st.page_table, ld, ws_step,
                                 outs[s % 2], causal=wl.causal, stream=stream)
        out_h[s].copy_(outs[s % 2], non_blocking=True)

    # --graph with in-line copies: the e2e steps, copies included, captured
    # as graphs of GRAPH_STEPS steps and replayed
    e2e_graphs = []
    if args.graph and not overlap:
        for c0 in range(0, e2e_steps, GRAPH_STEPS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for s in range(c0, min(c0 + GRAPH_STEPS, e2e_steps)):
                    step_in_line(s)
            e2e_graphs.append(g)
    multi.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if overlap:
        h2d_stream.wait_event(e0)
        d2h_stream.wait_event(e0)
        copy_in(0)
    for g in e2e_graphs:
        g.replay()
    for s in range(e2e_steps if not e2e_graphs else 0):
        kd, vd, qd, sd, ld = dviews[s % 2]
        if overlap:
            if s + 1 < e2e_steps:
                copy_in(s + 1)
            stream.wait_event(ev_in[s])
            if s >= 2:
                stream.wait_event(ev_out[s - 2])
        else:
            step_in_line(s)
            continue
        # the one-call public API of a decode step
        csd.isoquant_decode_step(st.ctx, st.cache, kd, vd, sd, qd.view(B, nq, Hq, 128), st.page_table, ld, ws_step,
                                 outs[s % 2], causal=wl.causal, stream=stream)
        if overlap:
            ev_done[s].record(stream)
            d2h_stream.wait_event(ev_done[s])
            with torch.cuda.stream(d2h_stream):
                out_h[s].copy_(outs[s % 2], non_blocking=True)
            ev_out[s].record(d2h_stream)
    if overlap:
        stream.wait_event(ev_out[e2e_steps - 1])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    # the overlapped steps against the same steps run one at a time on one
    # stream (the kernels are deterministic: a race between the copies and
    # the kernels would show as a difference)
    e2e_checked = sorted({0, e2e_steps // 2, e2e_steps - 1})
    e2e_identical = True
    for s in e2e_checked:
        stage_ds[0].copy_(stage_h[s])
        kd, vd, qd, sd, ld = dviews[0]
        csd.isoquant_decode_step(st.ctx, st.cache, kd, vd, sd, qd.view(B, nq, Hq, 128), st.page_table, ld, ws_step,
                                 outs[0], causal=wl.causal, stream=stream)
        torch.cuda.synchronize(dev)
        e2e_identical = e2e_identical and bool(torch.equal(outs[0].cpu(), out_h[s]))
    e2e_ms = multi.max_over_ranks(e0.elapsed_time(e1), device=dev)
    e2e_units = multi.sum_over_ranks(sum(sum(lens_e2e[s]) * H for s in range(e2e_steps)), device=dev)
    e2e_value = e2e_units / (e2e_ms / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, budget_s=args.cpu_seconds, bits=args.bits, st=st, dev=dev)
    # the library's kernel choice: mma.sync below 64 query rows per KV head
    # (or with pages under 64 tokens), tcgen05 from there
    rows = wl.nq * (Hq // H)
    partial_kernel = ("k_attend_partial" if rows < 64 or st.ps < 64 else
                      "k_attend_wide" if rows >= 128 else "k_attend_tiles")
    if partial_kernel == "k_attend_partial" and args.bits == 3:
        # the ncu capture behind this figure is of the 3-bit mma.sync kernel
        traffic = profiled_traffic(["compressed_space_decode_b200/csrc/attend.cu",
                                    "compressed_space_decode_b200/csrc/isoquant_internal.cuh"], bytes_per_launch)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": (f"f32 accumulate ({args.bits}-bit codes -> f16 centroids, hi/lo f16 queries on mma.sync)"
                  if partial_kernel == "k_attend_partial" else
                  f"f32 accumulate ({args.bits}-bit codes -> f16 centroids, hi/lo f16 queries and weights on tcgen05)"),
        "data": "synthetic (seeded bf16 Student-t(4) K/V, log-uniform channel scales, x20 outliers)",
        "config": {"workload": wl.name.split("@")[0], "batch": B, "q_heads": Hq, "kv_heads": H, "head_dim": 128,
                   "context_start": lens0[0], "page_size": st.ps, "page_table": "shuffled",
                   "step": f"decode_prep (append {adv} token(s)/seq + rotate q, one launch) + attend_decode (split-K attention + combine); programmatic launches",
                   "launch": (f"CUDA graphs of {GRAPH_STEPS} steps, replayed" if args.graph else
                              "one library call per half step from the host"),
                   "l2": f"packed cache {bytes_per_launch / 1e6:.0f} MB > 126 MB L2; no flush",
                   "parallelism": f"dp{world} (independent shards)", "code_bits": args.bits,
                   "bytes_per_kv_token_head": bytes_per_token_head},
        # the same rate per query head (each KV token-head serves G = Hq / H query heads)
        "value_q_head_equivalent": {"value": value * (Hq // H), "unit": "KV-token·q-heads/s", "group": Hq // H},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "api": "isoquant_decode_step",
                "copies": ("pinned host <-> device every step, each direction on its own stream, overlapping the "
                           "neighbouring steps' kernels (double-buffered inputs and outputs)" if overlap else
                           "pinned host <-> device every step, in line on the launching stream" +
                           (f"; steps and copies replayed as CUDA graphs of {GRAPH_STEPS}" if e2e_graphs else "")),
                "serial_recheck": {"steps": e2e_checked, "identical": e2e_identical}},
        "roofline": {"bound": "hbm", "kernel": f"isoquant_attend_decode ({partial_kernel} + k_attend_combine)",
                     "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                     "bytes_per_launch": bytes_per_launch, "avg_launch_ms": attn_med_ms,
                     "launches_timed": n_attn, "launch_ms_p10_p90": [loop_ms[len(loop_ms) // 10],
                                                                     loop_ms[(9 * len(loop_ms)) // 10]],
                     "loop": (f"{n_attn} attention calls back to back in graphs of {GRAPH_STEPS}, CUDA events "
                              f"around each replay (median per call); clocks sampled over the loop" if args.graph else
                              f"{n_attn} attention calls back to back, CUDA events around each (median); "
                              f"clocks sampled over the loop"),
                     "clocks": clocks_attn,
                     "achieved_in_step": achieved_in_step, "in_step_launches_timed": len(attn_ms),
                     "frac_of_8TBps": achieved / 8000.0},
        "gpu_launches": kernel_launches,
        # the timed steps are often too short for nvidia-smi to sample (it
        # polls every 50 ms); then the clocks of the attention loop that
        # follows them on the same GPU stand in, and say so
        "clocks": clocks if clocks.get("samples", 0) > 0 else
        dict(clocks_attn, note="sampled over the attention-only loop right after the timed steps "
                               "(the timed steps ended before the first sample)"),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line))


def oracle_sample(wl, b, h, bits=3, device="cuda"):
    """Oracle state for one (sequence, KV head) of workload `wl`: its own
    codes of the context, the tokens a step appends (one, or the nq of a
    causal chunk) and the step's query rows (every position of the chunk,
    each seeing the tokens up to its own), and how many context coordinates
    lie within 1e-6 of a decision threshold.  Inputs come from the seeded
    generators only."""
    import oracle
    from compressed_space_decode_b200 import synthetic
    L = wl.seq_lens[b]
    G = wl.group
    adv = wl.nq if wl.causal else 1
    k, v = synthetic.workload_kv_tokens(wl, b, 0, L + adv, device=device)
    signs, quats = synthetic.rotation_params(wl.seed, wl.kv_heads)
    s, qt = signs[h].numpy(), quats[h].numpy()
    kc, kn, zk, _ = oracle.compress(s, qt, k[:L, h].double().cpu().numpy(), want_z=True, bits=bits)
    vc, vn, zv, _ = oracle.compress(s, qt, v[:L, h].double().cpu().numpy(), want_z=True, bits=bits)
    near = [int(oracle.near_boundary(z, 1e-6, bits=bits).sum()) for z in (zk, zv)]
    newk = k[L:L + adv, h].double().cpu().numpy()
    newv = v[L:L + adv, h].double().cpu().numpy()
    nq = adv
    q = synthetic.workload_queries(wl, 0, device=device)[b, :nq, h * G:(h + 1) * G]
    q = q.reshape(nq * G, 128).double().cpu().numpy()  # rows (position, head)
    lims = [L + i + 1 for i in range(nq) for _ in range(G)]
    return dict(s=s, qt=qt, kc=kc, kn=kn, vc=vc, vn=vn, newk=newk, newv=newv, q=q, L=L, G=G, bits=bits, b=b, h=h,
                near=near, adv=adv, nq=nq, lims=lims, causal=bool(wl.causal))


def oracle_step(o):
    """One step of the oracle for one (sequence, KV head): compress the
    appended K/V tokens, then attend (position i of the step's chunk over the
    first L + i + 1 tokens)."""
    import numpy as np

    import oracle
    kc1, kn1, _, _ = oracle.compress(o["s"], o["qt"], o["newk"], bits=o["bits"])
    vc1, vn1, _, _ = oracle.compress(o["s"], o["qt"], o["newv"], bits=o["bits"])
    kc = np.concatenate([o["kc"], kc1])
    kn = np.concatenate([o["kn"], kn1])
    vc = np.concatenate([o["vc"], vc1])
    vn = np.concatenate([o["vn"], vn1])
    return oracle.attend(o["s"], o["qt"], o["q"], kc, kn, vc, vn, o["lims"], bits=o["bits"])


def host_cores():
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _oracle_worker(job):
    """One host process of the all-core oracle leg: wait for the common
    start, then run whole oracle decode steps until the budget is spent."""
    sample, start_at, budget_s, max_steps = job
    while time.time() < start_at:
        time.sleep(0.001)
    n, t0 = 0, time.perf_counter()
    while n < max_steps and (budget_s is None or time.perf_counter() - t0 < budget_s):
        oracle_step(sample)
        n += 1
    return n, time.perf_counter() - t0


def _compress_worker(job):
    """One host process of the all-core bulk-compression leg: compress the
    sample's vectors with the oracle until the budget is spent; returns the
    vectors compressed and the time taken."""
    import oracle
    sample, start_at, budget_s, max_steps = job
    while time.time() < start_at:
        time.sleep(0.001)
    n, t0 = 0, time.perf_counter()
    while n < max_steps and (budget_s is None or time.perf_counter() - t0 < budget_s):
        oracle.compress(sample["s"], sample["qt"], sample["x"], bits=sample["bits"])
        n += 1
    return n * len(sample["x"]), time.perf_counter() - t0


class OraclePool:
    """`cores` spawned host processes, each running the oracle's decode step
    (or, with `worker=_compress_worker`, its bulk compression) on the sample
    (processes, not threads: the oracle is single-threaded C behind ctypes;
    spawned, not forked, since the parent holds a CUDA context)."""

    def __init__(self, sample, cores, worker=None):
        import multiprocessing as mp
        self.sample, self.cores = sample, cores
        self.worker = worker or _oracle_worker
        self.pool = mp.get_context("spawn").Pool(cores)

    def run(self, budget_s=None, steps=1):
        start_at = time.time() + 0.5
        res = self.pool.map(self.worker, [(self.sample, start_at, budget_s, steps if budget_s is None else 1 << 40)]
                            * self.cores, chunksize=1)
        return sum(r[0] for r in res), max(r[1] for r in res)

    def close(self):
        self.pool.close()
        self.pool.join()


def parity_sample(st, o, dev):
    """The oracle sample's (sequence, KV head) against the GPU path: its
    context's codes and norms as the library wrote them (mismatches, and
    coordinates within 1e-6 of a threshold), and one attention call over the
    same L + 1 tokens with the sample's query rows (max row-normwise error)."""
    import numpy as np
    import torch

    import compressed_space_decode_b200 as csd
    import oracle
    from compressed_space_decode_b200 import synthetic
    b, h, L, G, bits = o["b"], o["h"], o["L"], o["G"], o["bits"]
    res = {"pair": f"sequence {b}, KV head {h}", "vectors": 2 * L, "coords": 2 * L * 128,
           "near_boundary_1e-6": sum(o["near"])}
    mism_codes = mism_norms = 0
    for kv, (oc, on) in enumerate(((o["kc"], o["kn"]), (o["vc"], o["vn"]))):
        gc, gn = st.gather(b, h, kv, 0, L)
        gc = gc.numpy().astype(np.uint32)
        gn = gn.numpy().astype(np.uint16)
        diff = (gc != oc).any(axis=1)
        if diff.any():
            mism_codes += int((oracle.unpack(gc[diff], bits=bits) != oracle.unpack(oc[diff], bits=bits)).sum())
        mism_norms += int((gn != on).sum())
    res["code_mismatches"] = mism_codes
    res["norm_mismatches"] = mism_norms
    wl = st.wl
    nq = o["nq"]
    q = synthetic.workload_queries(wl, 0, device=dev)[b:b + 1, :nq].contiguous()
    q_rot = torch.empty(q.shape, dtype=torch.float32, device=dev)
    csd.isoquant_rotate_q(st.ctx, q.view(-1, st.Hq, 128), q_rot.view(-1, st.Hq, 128))
    out = torch.empty_like(q_rot)
    lens = torch.tensor([L + o["adv"]], dtype=torch.int32, device=dev)
    ws = csd.alloc_workspace(st.ctx, 1, nq, st.Hq, page_size=st.ps, device=dev)
    csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table[b:b + 1].contiguous(), lens, ws, out,
                               causal=o["causal"])
    torch.cuda.synchronize(dev)
    got = out[0, :, h * G:(h + 1) * G].reshape(nq * G, 128).double().cpu().numpy()
    ref = oracle_step(o)
    err = np.abs(got - ref).max(axis=1) / np.abs(ref).max(axis=1)
    res["max_row_rel_err"] = float(err.max())
    res["tolerance"] = 2e-3
    return res


def cpu_baseline(wl, budget_s=12.0, bits=3, st=None, dev=None):
    """The fp64 oracle, as it stands, on the host cores: a bounded sample of
    the same decode step (one (sequence, KV head) unit, repeated), on one
    core and on every core (one spawned process per core), plus the sample's
    parity against the GPU path."""
    o = oracle_sample(wl, 0, 0, bits)
    units, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        oracle_step(o)
        units += o["L"] + o["adv"]
    dt = time.perf_counter() - t0
    one = {"value": units / dt, "unit": UNIT, "cores": 1,
           "sample": f"{units // (o['L'] + o['adv'])} steps in {dt:.1f} s"}
    cores = host_cores()
    pool = OraclePool(o, cores)
    pool.run(steps=1)  # start-up, untimed
    n, dt_all = pool.run(budget_s=budget_s)
    pool.close()
    line = {"value": n * (o["L"] + o["adv"]) / dt_all, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"sequence 0, KV head 0 of the workload (context {o['L'] + o['adv']}, {len(o['lims'])} "
                      f"query rows): compress the {o['adv']} appended token(s) + attend; {cores} host processes "
                      f"ran {n} steps in {dt_all:.1f} s",
            "single_core": one}
    if st is not None:
        line["parity_sample"] = parity_sample(st, o, dev)
    return line


# ---------------------------------------------------------- reference arm
def run_reference(args):
    """The fp64 oracle as the reference arm (there is no reference code to
    install: the pages describe the method only).  Rank 0 only."""
    rank, local_rank, world = (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
                               int(os.environ.get("WORLD_SIZE", "1")))
    if rank != 0:
        return
    import torch

    from compressed_space_decode_b200 import synthetic
    torch.cuda.set_device(local_rank)
    wl = synthetic.workloads()[args.workload]
    if args.workload.startswith("prefill_attend"):
        ostep, oflops, text = prefill_oracle_sample(wl, bits=args.bits)
        for _ in range(args.warmup):
            ostep()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            ostep()
        dt = time.perf_counter() - t0
        value = args.steps * oflops / dt / 1e12
        print(json.dumps({
            "impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "q_heads": wl.q_heads, "kv_heads": wl.kv_heads,
                       "head_dim": 128, "prompt": wl.seq_lens[0], "query_positions": wl.nq, "causal": True},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: {text}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return
    o = oracle_sample(wl, 0, 0, args.bits)
    cores = host_cores()
    pool = OraclePool(o, cores)
    pool.run(steps=args.warmup)
    # each step: every host process runs one oracle decode step
    _, dt = pool.run(steps=args.steps)  # the slowest process's own time
    pool.close()
    units = args.steps * cores * (o["L"] + o["adv"])
    value = units / dt
    sample = (f"each step: {cores} host processes each run sequence 0, KV head 0 of {wl.name} (context "
              f"{o['L'] + o['adv']}, {len(o['lims'])} query rows): compress the {o['adv']} appended token(s) "
              f"+ attend")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "q_heads": wl.q_heads, "kv_heads": wl.kv_heads,
                   "head_dim": 128, "context_start": wl.seq_lens[0], "page_size": wl.page_size,
                   "code_bits": args.bits},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------ causal prefill attention
PREFILL_METRIC = "causal prefill attention TFLOP/s over packed 3-bit KV (4*128 flop per visible query-key pair per q head)"


def causal_pairs(wl):
    """Visible (query position, key) pairs per q head: query i of a sequence
    of L tokens with nq query positions sees min(L, max(0, L - nq + i + 1))."""
    import numpy as np
    i = np.arange(wl.nq, dtype=np.int64)
    return int(sum(np.clip(L - wl.nq + i + 1, 0, L).sum() for L in wl.seq_lens))


def prefill_oracle_sample(wl, rows=32, bits=3):
    """The oracle on a bounded sample of the prefill attention: KV head 0 of
    sequence 0, its own codes of the whole prompt, and the last rows / G
    query positions of its G query heads.  Returns (step, flops, text)."""
    import numpy as np

    import oracle
    from compressed_space_decode_b200 import synthetic
    L, G, nq = wl.seq_lens[0], wl.group, wl.nq
    k, v = synthetic.workload_kv_tokens(wl, 0, 0, L, device="cuda")
    signs, quats = synthetic.rotation_params(wl.seed, wl.kv_heads)
    s, qt = signs[0].numpy(), quats[0].numpy()
    kc, kn, _, _ = oracle.compress(s, qt, k[:, 0].double().cpu().numpy(), bits=bits)
    vc, vn, _, _ = oracle.compress(s, qt, v[:, 0].double().cpu().numpy(), bits=bits)
    npos = max(1, rows // G)
    q = synthetic.workload_queries(wl, 0, device="cuda")[0, nq - npos:, 0:G].double().cpu().numpy()
    q = q.reshape(npos * G, 128)
    lim = [max(0, min(L, L - nq + i + 1)) for i in range(nq - npos, nq) for _ in range(G)]
    flops = 4 * 128 * sum(lim)

    def step():
        return oracle.attend(s, qt, q, kc, kn, vc, vn, lim, bits=bits)
    text = (f"sequence 0, KV head 0 of {wl.name}: the last {npos} query positions x {G} q heads "
            f"({npos * G} rows over up to {L} tokens)")
    return step, flops, text


def run_prefill_attend(args):
    """Causal prefill attention over the packed cache: every step compresses
    the prompt's K/V into the paged cache and rotates its queries
    (isoquant_decode_prep, one launch), then runs the split attention with
    its combine and inverse rotation (isoquant_attend_decode).  With 128 or
    more query rows per KV head the partial kernel is the warp-specialised
    tcgen05 one, each 128-row stream walking only the pages inside its
    causal horizon.  Reported as useful TFLOP/s (4*128 flop per visible
    query-key pair per q head); the tensor cores issue twice that (fp16 high
    and low parts of the queries and of the softmax weights)."""
    import torch

    import compressed_space_decode_b200 as csd
    from compressed_space_decode_b200 import synthetic
    from compressed_space_decode_b200.workload import DecodeState

    wl = synthetic.workloads()[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    st = DecodeState(wl, device=dev, fill=False, bits=args.bits)
    B, H, Hq, nq = st.B, st.H, st.Hq, wl.nq
    kv = [st.kv_tokens(b, 0, wl.seq_lens[b]) for b in range(B)]
    ks = torch.cat([k for k, _ in kv]).contiguous()
    vs = torch.cat([v for _, v in kv]).contiguous()
    slots = torch.cat([st.slots(b, 0, wl.seq_lens[b]) for b in range(B)]).contiguous()
    qs = [st.queries(i) for i in range(2)]  # two query sets of 268 MB, alternating (> L2)
    q_rot = torch.empty((B, nq, Hq, 128), dtype=torch.float32, device=dev)
    out = torch.empty_like(q_rot)
    ws = csd.alloc_workspace(st.ctx, B, nq, Hq, device=dev)
    launches = [0]
    ev = {}

    def step(i, timed):
        csd.isoquant_decode_prep(st.ctx, st.cache, ks, vs, slots, qs[i % 2].view(B * nq, Hq, 128),
                                 q_rot.view(B * nq, Hq, 128), stream=stream)
        launches[0] += csd.isoquant_last_launch_count(st.ctx)
        if timed:
            ev[i] = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[i][0].record(stream)
        csd.isoquant_attend_partial(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, causal=True,
                                    stream=stream)
        launches[0] += csd.isoquant_last_launch_count(st.ctx)
        if timed:
            ev[i][1].record(stream)
        csd.isoquant_attend_combine(st.ctx, B, nq, Hq, st.seq_lens_dev, st.ps, ws, out, stream=stream)
        launches[0] += csd.isoquant_last_launch_count(st.ctx)

    for i in range(args.warmup):
        step(i, False)
    torch.cuda.synchronize(dev)
    assert csd.isoquant_get_status(st.ctx) == 0
    launches[0] = 0
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(i, True)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1) / args.steps
    part_ms = sum(a.elapsed_time(b) for a, b in ev.values()) / len(ev)
    timed_launches = launches[0]
    clocks = clocks_or_resample(clocks, uuid, lambda: step(0, False), dev)
    flops = 4 * 128 * Hq * causal_pairs(wl)
    value = flops / (ms / 1e3) / 1e12
    achieved = flops / (part_ms / 1e3) / 1e12
    peak, peak_kind = tensor_peak()

    # end to end: the one-call step from pinned host buffers (prompt K/V,
    # queries, slots, lengths in; the attention output back)
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    kh, vh = ks.cpu().pin_memory(), vs.cpu().pin_memory()
    qh = qs[0].cpu().pin_memory()
    sh = slots.cpu().pin_memory()
    lh = st.seq_lens_dev.cpu().pin_memory()
    oh = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    # two sets of device inputs and outputs: a step's copies (each direction
    # on its own stream) overlap the neighbouring steps' kernels
    bufs = [(torch.empty_like(ks), torch.empty_like(vs), torch.empty_like(qs[0]), torch.empty_like(slots),
             torch.empty_like(st.seq_lens_dev), torch.empty_like(out)) for _ in range(2)]
    ws_step = csd.alloc_step_workspace(st.ctx, B, nq, Hq, device=dev)
    kd, vd, qd, sd, ld, _ = bufs[0]
    h2d = (kd.numel() + vd.numel() + qd.numel()) * 2 + sd.numel() * 8 + ld.numel() * 4
    d2h = out.numel() * 4
    del ws
    h2d_stream, d2h_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_out = [torch.cuda.Event() for _ in range(e2e_steps)]

    def copy_in(i):
        if i >= 2:
            h2d_stream.wait_event(ev_done[i - 2])
        with torch.cuda.stream(h2d_stream):
            for dst, src in zip(bufs[i % 2][:5], (kh, vh, qh, sh, lh)):
                dst.copy_(src, non_blocking=True)
        ev_in[i].record(h2d_stream)

    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)
    d2h_stream.wait_event(e0)
    copy_in(0)
    for i in range(e2e_steps):
        if i + 1 < e2e_steps:
            copy_in(i + 1)
        kd, vd, qd, sd, ld, od = bufs[i % 2]
        stream.wait_event(ev_in[i])
        if i >= 2:
            stream.wait_event(ev_out[i - 2])
        csd.isoquant_decode_step(st.ctx, st.cache, kd, vd, sd, qd, st.page_table, ld, ws_step, od, causal=True,
                                 stream=stream)
        ev_done[i].record(stream)
        d2h_stream.wait_event(ev_done[i])
        with torch.cuda.stream(d2h_stream):
            oh.copy_(od, non_blocking=True)
        ev_out[i].record(d2h_stream)
    stream.wait_event(ev_out[e2e_steps - 1])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    assert csd.isoquant_get_status(st.ctx) == 0

    line = {
        "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 accumulate (fp16 high + low parts of queries and softmax weights on tcgen05)",
        "data": "synthetic (seeded bf16 Student-t(4) K/V, log-uniform channel scales, x20 outliers; N(0,1) queries)",
        "config": {"workload": wl.name, "batch": B, "q_heads": Hq, "kv_heads": H, "head_dim": 128,
                   "prompt": wl.seq_lens[0], "query_positions": nq, "causal": True, "page_size": st.ps,
                   "code_bits": args.bits,
                   "step": "decode_prep (compress the prompt's K/V + rotate its queries, one launch) + "
                           "attend_partial (tcgen05, causal horizon per 128-row stream) + attend_combine",
                   "l2": "two query sets of 268 MB alternate; no flush"},
        "e2e": {"value": flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "api": "isoquant_decode_step",
                "copies": "pinned host <-> device every step, each direction on its own stream, overlapping the "
                          "neighbouring steps' kernels (double-buffered inputs and outputs)"},
        "roofline": {"bound": "tensor", "kernel": "isoquant_attend_partial (k_attend_wide)", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": None, "avg_launch_ms": part_ms, "flops_per_launch": flops,
                     "tensor_issued_tflops": 2 * achieved},
        "gpu_launches": timed_launches, "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        ostep, oflops, text = prefill_oracle_sample(wl, bits=args.bits)
        n, c0 = 0, time.perf_counter()
        while time.perf_counter() - c0 < args.cpu_seconds:
            ostep()
            n += 1
        dt = time.perf_counter() - c0
        line["cpu_baseline"] = {"value": n * oflops / dt / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                                "sample": f"{text}, repeated {n}x in {dt:.1f} s"}
    print(json.dumps(line))


def compress_cpu_baseline(wl, cache, k, budget_s, n_vec=2048):
    """The fp64 oracle's bulk compression, as it stands, on the host cores: a
    bounded sample (the K vectors of the first n_vec tokens of KV head 0 of
    layer 0, compressed again and again for budget_s) on one core and on
    every core; plus the sample's codes and norms against the ones the GPU
    wrote into layer 0's cache (mismatches, and coordinates within 1e-6 of a
    threshold)."""
    import numpy as np
    import torch

    import oracle
    from compressed_space_decode_b200 import synthetic
    signs, quats = synthetic.rotation_params(wl.seed, wl.kv_heads)
    sample = {"s": signs[0].numpy(), "qt": quats[0].numpy(), "x": k[:n_vec, 0].double().cpu().numpy(), "bits": 3}
    reps, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        oracle.compress(sample["s"], sample["qt"], sample["x"])
        reps += 1
    dt = time.perf_counter() - t0
    one = {"value": reps * n_vec / dt, "unit": "vectors/s", "cores": 1, "sample": f"{reps} x {n_vec} vectors in {dt:.1f} s"}
    cores = host_cores()
    pool = OraclePool(sample, cores, worker=_compress_worker)
    pool.run(steps=1)  # start-up, untimed
    n, dt_all = pool.run(budget_s=budget_s)
    pool.close()
    oc, on, z, _ = oracle.compress(sample["s"], sample["qt"], sample["x"], want_z=True)
    t = torch.arange(n_vec, device=cache.codes.device)
    gc = cache.codes[t // 256, 0, 0, :, t % 256].to(torch.int64).cpu().numpy().astype(np.uint32)
    gn = cache.norms[t // 256, 0, 0, t % 256].view(torch.int16).cpu().numpy().astype(np.uint16)
    diff = (gc != oc).any(axis=1)
    mism = int((oracle.unpack(gc[diff]) != oracle.unpack(oc[diff])).sum()) if diff.any() else 0
    return {"value": n / dt_all, "unit": "vectors/s", "cores": cores, "kind": "oracle",
            "sample": f"K vectors of tokens 0..{n_vec - 1}, KV head 0, layer 0 (bf16 in, 3-bit codes out); "
                      f"{cores} host processes compressed {n} vectors in {dt_all:.1f} s",
            "single_core": one,
            "parity_sample": {"vectors": n_vec, "coords": n_vec * 128,
                              "near_boundary_1e-6": int(oracle.near_boundary(z, 1e-6).sum()),
                              "code_mismatches": mism, "norm_mismatches": int((gn != on).sum())}}


def run_prefill(args):
    """Bulk compression of a long prompt: 32768 tokens x 8 KV heads x 48
    layers, K and V (isoquant_compress_kv per layer, one context per layer).
    Reported as vectors/s and achieved HBM GB/s on bf16 in + packed out."""
    import torch

    import compressed_space_decode_b200 as csd
    from compressed_space_decode_b200 import synthetic

    wl = synthetic.workloads()[args.workload]
    T, H, layers = wl.seq_lens[0], wl.kv_heads, wl.layers
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    ctxs = []
    for layer in range(layers):
        signs, quats = synthetic.rotation_params(wl.seed + 1000 * layer, H)
        ctxs.append(csd.isoquant_init(signs, quats))
    pages = (T + 255) // 256
    caches = [csd.PagedCache.allocate(H, pages, 256, device=dev) for _ in range(layers)]
    scales = synthetic.workload_scales(wl)
    n_inputs = 3  # distinct inputs rotated over the layers: 3 x 134 MB > L2
    inputs = []
    for i in range(n_inputs):
        k, v = synthetic.workload_kv_tokens(wl, i, 0, T, device=dev, scales=scales)
        inputs.append((k.contiguous(), v.contiguous()))
    slots = torch.arange(T, dtype=torch.int64, device=dev)

    def step():
        for layer in range(layers):
            k, v = inputs[layer % n_inputs]
            csd.isoquant_compress_kv(ctxs[layer], caches[layer], k, v, slots, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    clocks = clocks_or_resample(clocks, uuid, step, dev)
    cpu = None if args.no_cpu_baseline else compress_cpu_baseline(wl, caches[0], inputs[0][0], args.cpu_seconds)
    vectors = 2 * T * H * layers
    bytes_moved = vectors * (128 * 2 + 13 * 4 + 2)
    peak, peak_kind = peaks()
    gbs = bytes_moved / (ms / 1e3) / 1e9
    print(json.dumps({
        "metric": "bulk KV compression vectors/s (rotate + quantize + pack into the paged cache)",
        "value": vectors / (ms / 1e3), "unit": "vectors/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 rotation (f64 norm and near-threshold re-check), bf16 in",
        "data": "synthetic", "config": {"workload": wl.name, "tokens": T, "kv_heads": H, "layers": layers,
                                         "l2": f"{n_inputs} distinct inputs of {2 * T * H * 256 / 1e6:.0f} MB"},
        "roofline": {"bound": "hbm", "kernel": "isoquant_compress_kv", "achieved": gbs, "peak": peak,
                     "unit": "GB/s", "frac": gbs / peak, "peak_kind": peak_kind,
                     "bytes_per_step": bytes_moved},
        "gpu_launches": layers * args.steps, "clocks": clocks, "cpu_baseline": cpu}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1, help="GPUs (ranks) of the run; N > 1 under torchrun, one shard per rank")
    ap.add_argument("--steps", type=int, default=5000, help="timed steps")
    ap.add_argument("--warmup", type=int, default=20, help="untimed warm-up steps (at least 3)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours",
                    help="ours: the CUDA library; reference: the fp64 oracle on the host")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="decode workload name, prefill_attend_* for causal prefill, prefill_32768_kv8_layers48 for compression")
    ap.add_argument("--e2e-steps", type=int, default=500, help="steps of the end-to-end (host buffers) measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="time budget of each CPU-oracle baseline leg (one core, then all cores)")
    ap.add_argument("--attn-seconds", type=float, default=1.0,
                    help="length of the attention-only loop behind the roofline figure")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--graph", action="store_true",
                    help="capture the timed decode steps (and the attention loop) as CUDA graphs and replay them")
    ap.add_argument("--bits", type=int, default=3, choices=[2, 3, 4],
                    help="code width of the decode workload (3: the method's; 2 and 4: other widths)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload.startswith("prefill_attend"):
        run_prefill_attend(args)
    elif args.workload.startswith("prefill"):
        run_prefill(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
