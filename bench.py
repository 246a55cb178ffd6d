"""Benchmark of the hybrid compressed-attention decode hot path (CSA + HCA layer pair).

One step = one decode query per sequence through one CSA layer (append, lightning-indexer
top-k, sparse attention with the window branch) and one HCA layer (append, dense attention
with the window branch), for the whole batch, on seeded synthetic caches resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode1m|decode128k]
                    [--impl ours|reference]

Timing: K steps are replayed from a CUDA graph, rotating over 3 replicas of every cache so
that no step finds its data in L2 from the step before; CUDA events on the launching stream,
synchronize + barrier on both sides, max over ranks.  The step time comes from a graph without
instrumentation (its launches keep their programmatic early-launch edges); a second capture of
the same launches with event records between the kernels gives the per-kernel times and the
roofline of the dominant kernel.  `--impl reference` times the float64 CPU oracle instead
(on rank 0 only), on a bounded sample of the same workload.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode queries/s & HBM GB/s (% of 8 TB/s) for CSA+HCA attention at 128K–1M ctx"
UNIT = "decode queries/s"
REPLICAS = 3
# kernels one step launches: 2 x append_kernel, indexer_topk_coop_kernel,
# 2 x (attention_tc_partial_kernel + attention_merge_kernel)
LAUNCHES_PER_STEP = 7


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=6)
    p.add_argument("--workload", default="decode1m", choices=["decode1m", "decode128k"])
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--profile", action="store_true",
                   help="run a few eager steps on one cache replica (for ncu captures); prints no JSON")
    return p.parse_args()


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ------------------------------------------------------------------------------------------
# Clock sampling during the timed region.
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# Our implementation.
# ------------------------------------------------------------------------------------------
def algorithmic_bytes(wl):
    """Bytes the method must move per step (whole batch), by operation."""
    B = wl.batch
    return {
        "indexer": B * wl.csa_entries * 40,                          # 32 B codes + 8 B scales / entry
        "csa_attention": B * (wl.topk + wl.window) * 576,
        "hca_attention": B * (wl.hca_entries + wl.window) * 576,
        "append": 2 * B * (1024 + 576) + B * 4 * 1024 // 4,          # token in, window entry out, tail reads
    }


# ncu summaries under profiles/: DRAM read+write bytes per launch, valid only while the kernel's
# sources hash to the value recorded with the capture (a changed kernel reports null).
PROFILES = {
    "indexer": ("indexer_topk_decode1m.md", "indexer.cu", ""),
    "csa_attention": ("attention_tc_partial_decode1m.md", "attention_tc.cu", " (CSA)"),
    "hca_attention": ("attention_tc_partial_decode1m.md", "attention_tc.cu", " (HCA)"),
}


def kernel_source_hash(cu):
    """sha256[:16] of the kernel's source file followed by every shared header (sorted)."""
    import hashlib
    d = os.path.join(ROOT, "compressed_sparse_long_decode_b200", "csrc")
    h = hashlib.sha256()
    for f in [cu] + sorted(x for x in os.listdir(d) if x.endswith(".cuh")):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel on this workload,
    or None when there is none or the kernel changed since it was taken."""
    if kernel not in PROFILES or workload != "decode1m":
        return None
    md, cu, tag = PROFILES[kernel]
    try:
        with open(os.path.join(ROOT, "profiles", md)) as fh:
            text = fh.read()
    except OSError:
        return None
    want_hash, traffic = None, None
    for line in text.splitlines():
        if line.startswith("source_sha256[:16]"):
            want_hash = line.rsplit(":", 1)[1].strip()
        if line.startswith(f"traffic_bytes_per_launch{tag}:"):
            traffic = int(line.rsplit(":", 1)[1].strip())
    if want_hash is None or traffic is None or want_hash != kernel_source_hash(cu):
        return None
    return traffic


def max_over_ranks(ms, device):
    """The slowest rank's time: every rank contributes its device-timed milliseconds and all
    of them get the maximum back (a no-op without a process group)."""
    import torch
    import torch.distributed as td
    if not (td.is_available() and td.is_initialized()) or td.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, ms_max, world):
    """Whole-job rate: the units all ranks processed (each rank processes the same number:
    independent sequences, weak scaling) over the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def run_ours(args, rank, world, local_rank):
    import torch
    import compressed_sparse_long_decode_b200 as csld
    import synth
    global REPLICAS
    if args.profile:
        REPLICAS = 1

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = synth.WORKLOADS[args.workload]
    B, W, k = wl.batch, wl.window, wl.topk
    scale = 1.0 / math.sqrt(512.0)
    g = synth.gen(1234 + rank, dev)

    # --- caches: REPLICAS independent copies of the CSA and the HCA layer ------------------
    inp = synth.prefill_inputs(8, seed=rank)
    layers = []
    for r in range(REPLICAS):
        csa = csld.LayerCache(B, wl.csa_cap, wl.csa_ratio, W, inp["bias4"], inp["w_idx"], device=dev)
        hca = csld.LayerCache(B, wl.hca_cap, wl.hca_ratio, W, inp["bias128"], device=dev)
        for c, n_ent in ((csa, wl.csa_entries), (hca, wl.hca_entries)):
            c.comp_kv[:, :n_ent] = synth.random_entries((B, n_ent), g, dev)
            c.win_kv[:] = synth.random_entries((B, W), g, dev)
            c.tail_kv.normal_(generator=g)
            c.seq_len.fill_(wl.context)
        ik, isc = synth.random_ikeys(B, csa.capacity, g, dev, heavy_frac=wl.heavy_frac, n_valid=wl.csa_entries)
        csa.ikeys.copy_(synth.ikeys_swap_halves(ik))   # the cache's stored layout
        csa.iscales.copy_(isc)
        del ik, isc
        layers.append((csa, hca))
    torch.cuda.synchronize()

    n_total = args.warmup + args.steps
    # --- per-step inputs, resident in HBM --------------------------------------------------
    toks = synth.decode_tokens(B * (n_total + REPLICAS), seed=100 + rank, device=dev)
    qs = synth.decode_queries(B * REPLICAS, seed=200 + rank, device=dev)
    x_all = toks["kv"].view(-1, B, 512)
    z_all = toks["gate"].view(-1, B)
    q_all = qs["q"].view(REPLICAS, B, 16, 512)
    qi_all = qs["q_idx"].view(REPLICAS, B, 4, 64)
    hw_all = qs["head_w"].view(REPLICAS, B, 4)
    sel = torch.empty((REPLICAS, B, k), dtype=torch.int32, device=dev)
    out_csa = torch.empty((REPLICAS, B, 16, 512), dtype=torch.float32, device=dev)
    out_hca = torch.empty_like(out_csa)
    lse_csa = torch.empty((REPLICAS, B, 16), dtype=torch.float32, device=dev)
    lse_hca = torch.empty_like(lse_csa)
    ws_idx = [csld.indexer_workspace(B, wl.csa_cap + (wl.csa_cap & 1), k, dev) for _ in range(REPLICAS)]
    ws_att = csld.attention_workspace(B, max(wl.csa_cap, wl.hca_cap), k, W, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    x_slot = torch.empty((REPLICAS, B, 512), dtype=torch.bfloat16, device=dev)
    z_slot = torch.empty((REPLICAS, B), dtype=torch.float32, device=dev)

    ev = {name: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * REPLICAS)]
          for name in ("indexer", "csa_attention", "hca_attention")}

    def step(r, timed_events):
        csa, hca = layers[r]
        csld.kv_cache_append(csa, x_slot[r], z_slot[r], err)
        if timed_events:
            ev["indexer"][2 * r].record()
        csld.indexer_topk(csa.ikeys, csa.iscales, csa.seq_len, 4, qi_all[r], hw_all[r], k, out=sel[r],
                          ws=ws_idx[r], err=err)
        if timed_events:
            ev["indexer"][2 * r + 1].record()
            ev["csa_attention"][2 * r].record()
        csld.hybrid_decode_attention(q_all[r], csa.comp_kv, 4, sel[r], csa.win_kv, W, csa.seq_len, scale,
                                     out=out_csa[r], lse=lse_csa[r], ws=ws_att, err=err)
        if timed_events:
            ev["csa_attention"][2 * r + 1].record()
        csld.kv_cache_append(hca, x_slot[r], z_slot[r], err)
        if timed_events:
            ev["hca_attention"][2 * r].record()
        csld.hybrid_decode_attention(q_all[r], hca.comp_kv, 128, None, hca.win_kv, W, hca.seq_len, scale,
                                     out=out_hca[r], lse=lse_hca[r], ws=ws_att, err=err)
        if timed_events:
            ev["hca_attention"][2 * r + 1].record()

    # eager warm-up of every replica (also sets kernel attributes outside capture)
    for r in range(REPLICAS):
        x_slot[r].copy_(x_all[r])
        z_slot[r].copy_(z_all[r])
        step(r, False)
    torch.cuda.synchronize()
    if args.profile:
        for _ in range(args.steps):
            step(0, False)
        torch.cuda.synchronize()
        assert err.item() == 0
        print(f"profile run ok: {args.steps} eager steps of {wl.name} on one replica", flush=True)
        return None

    # graph = one step on each replica.  Two captures of the same launches: one with event
    # records between the kernels (the per-kernel breakdown) and one without, whose launches keep
    # their programmatic (early-launch) edges to each other (the step time).
    def capture(timed_events):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for r in range(REPLICAS):
                    step(r, timed_events)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        return g

    graph = capture(True)
    graph_plain = capture(False)

    rounds_w = max(1, math.ceil(args.warmup / REPLICAS))
    rounds_t = max(1, math.ceil(args.steps / REPLICAS))
    steps_timed = rounds_t * REPLICAS
    for _ in range(rounds_w):
        graph.replay()
        graph_plain.replay()
    torch.cuda.synchronize()

    dist = world > 1
    if dist:
        import torch.distributed as td
        td.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record()
    per = {name: 0.0 for name in ev}
    for _ in range(rounds_t):
        graph.replay()
        torch.cuda.synchronize()
        for name, evs in ev.items():
            per[name] += sum(evs[2 * r].elapsed_time(evs[2 * r + 1]) for r in range(REPLICAS))
    t1.record()
    torch.cuda.synchronize()
    ms_total = t0.elapsed_time(t1)
    # the per-round synchronize and the event records above add gaps; time the device work
    # without them too
    t2 = torch.cuda.Event(enable_timing=True)
    t3 = torch.cuda.Event(enable_timing=True)
    if dist:
        td.barrier()
    torch.cuda.synchronize()
    t2.record()
    for _ in range(rounds_t):
        graph_plain.replay()
    t3.record()
    torch.cuda.synchronize()
    ms_dev = t2.elapsed_time(t3)
    clk = clocks.stop()
    ms = max_over_ranks(min(ms_total, ms_dev), dev)
    assert err.item() == 0, f"device error word {err.item()}"

    # --- end to end: host (pinned) inputs -> device -> step -> host outputs -----------------
    e2e = run_e2e(csld, torch, layers, wl, dev, k, W, scale, ws_idx, ws_att, err, rounds_t, world)

    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    bytes_ = algorithmic_bytes(wl)
    avg = {n: per[n] / steps_timed for n in per}            # ms per launch (one call per step)
    dominant = max(avg, key=avg.get)
    achieved = bytes_[dominant] / (avg[dominant] * 1e-3) / 1e9
    step_bytes = sum(bytes_.values())
    ms_step = ms / steps_timed
    value = job_throughput(B * steps_timed, ms, world)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": steps_timed,
        "warmup": rounds_w * REPLICAS, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16 KV, e2m1 indexer keys; tcgen05 e2m1, e4m3 and bf16 MMA, fp32 accumulate",
        "data": "synthetic (seeded)",
        "config": {"workload": wl.name, "batch_per_gpu": B, "context": wl.context, "csa_entries": wl.csa_entries,
                   "hca_entries": wl.hca_entries, "topk": k, "window": W, "heads": 16, "dim": 512,
                   "l2": f"{REPLICAS} rotating cache replicas per step ({REPLICAS}x "
                         f"{(layers[0][0].comp_kv.numel() + layers[0][1].comp_kv.numel()) / 1e9:.2f} GB); "
                         f"each step touches {step_bytes / 1e6:.1f} MB not left in L2 by the step before",
                   "parallelism": f"replicas x{world} (independent sequences per GPU, no collective)"},
        "hbm": {"algorithmic_bytes_per_step": step_bytes,
                "gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
                "frac_of_measured_peak": round(step_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak, 4),
                "frac_of_8tbs": round(step_bytes / (ms_step * 1e-3) / 1e9 / 8000.0, 4)},
        "kernels_ms_per_step": {n: round(v, 5) for n, v in avg.items()},
        "roofline": {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": profiled_traffic(dominant, wl.name),
                     "algorithmic_bytes_per_launch": bytes_[dominant]},
        "roofline_all": {n: {"achieved_gbs": round(bytes_[n] / (avg[n] * 1e-3) / 1e9, 1),
                             "frac": round(bytes_[n] / (avg[n] * 1e-3) / 1e9 / hbm_peak, 4)} for n in avg},
        "clocks": clk,
        "gpu_launches": LAUNCHES_PER_STEP * steps_timed,
        "e2e": e2e,
    }
    return res


def run_e2e(csld, torch, layers, wl, dev, k, W, scale, ws_idx, ws_att, err, rounds, world):
    """Same step through the public API with the step's inputs copied from pinned host memory
    and both layers' outputs copied back, inside the timed region (graph-replayed)."""
    B = wl.batch
    import synth
    tok = synth.decode_tokens(B, seed=999)
    qq = synth.decode_queries(B, seed=998)
    # The step's inputs (token, indexer query, head weights, attention query) are packed in one
    # pinned host buffer and brought to the device by one staging kernel (csld_stage: a kernel
    # node chains to the append behind it, where a copy-engine transfer between kernels costs a
    # round trip through the copy engine).  The CSA output goes back by a copy on a second stream
    # under the HCA layer; the HCA attention writes its output straight into pinned host memory.
    # Every transfer is inside the timed region; the step ends when the HCA output is on the host.
    host = {"x": tok["kv"], "z": tok["gate"], "qi": qq["q_idx"], "w": qq["head_w"], "q": qq["q"]}
    offs, total = {}, 0
    for n, t in host.items():
        offs[n] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_in = torch.zeros(total, dtype=torch.uint8).pin_memory()
    for n, t in host.items():
        nb = t.numel() * t.element_size()
        h_in[offs[n]:offs[n] + nb].copy_(t.contiguous().view(-1).view(torch.uint8))
    d_in = torch.empty_like(h_in, device=dev)
    d = {n: d_in[offs[n]:offs[n] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
         for n, t in host.items()}
    o1 = torch.empty((B, 16, 512), dtype=torch.float32, device=dev)
    h_out = torch.empty((REPLICAS, 2, B, 16, 512), dtype=torch.float32).pin_memory()
    h_lse = torch.empty((REPLICAS, B, 16), dtype=torch.float32).pin_memory()
    sel = torch.empty((B, k), dtype=torch.int32, device=dev)
    h2d = h_in.numel()
    d2h = h_out[0].numel() * 4
    side = torch.cuda.Stream(device=dev)
    ev = [[torch.cuda.Event() for _ in range(2)] for _ in range(REPLICAS)]

    def step(r):
        csa, hca = layers[r]
        main = torch.cuda.current_stream()
        e_o1, e_d1 = ev[r]
        csld.stage(d_in, h_in)
        csld.kv_cache_append(csa, d["x"], d["z"], err)
        csld.indexer_topk(csa.ikeys, csa.iscales, csa.seq_len, 4, d["qi"], d["w"], k, out=sel, ws=ws_idx[r], err=err)
        csld.hybrid_decode_attention(d["q"], csa.comp_kv, 4, sel, csa.win_kv, W, csa.seq_len, scale, out=o1,
                                     ws=ws_att, err=err)
        e_o1.record(main)
        side.wait_event(e_o1)
        with torch.cuda.stream(side):
            h_out[r, 0].copy_(o1, non_blocking=True)
            e_d1.record(side)
        csld.kv_cache_append(hca, d["x"], d["z"], err)
        csld.hybrid_decode_attention(d["q"], hca.comp_kv, 128, None, hca.win_kv, W, hca.seq_len, scale,
                                     out=h_out[r, 1], lse=h_lse[r], ws=ws_att, err=err)
        main.wait_event(e_d1)

    for r in range(REPLICAS):
        step(r)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            for r in range(REPLICAS):
                step(r)
    torch.cuda.current_stream().wait_stream(s)
    graph.replay()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(rounds):
        graph.replay()
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    n_steps = rounds * REPLICAS
    assert torch.isfinite(h_out).all()
    return {"value": round(job_throughput(B * n_steps, ms, world), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms / n_steps, 5)}


# ------------------------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and the reference arm).
# ------------------------------------------------------------------------------------------
def oracle_sample(wl, n_seq, seed=7):
    """Host copies of n_seq sequences' caches and one step's queries (seeded, synthetic)."""
    import torch
    import synth
    g = synth.gen(seed)
    ik, isc = synth.random_ikeys(n_seq, wl.csa_cap + (wl.csa_cap & 1), g, heavy_frac=wl.heavy_frac,
                                 n_valid=wl.csa_entries)
    return {
        "ikeys": ik.numpy(), "iscales": isc.numpy(),
        "csa": synth.random_entries((n_seq, wl.csa_cap), g).numpy(),
        "hca": synth.random_entries((n_seq, wl.hca_cap), g).numpy(),
        "win": synth.random_entries((n_seq, wl.window), g).numpy(),
        "seq": torch.full((n_seq,), wl.context, dtype=torch.int32).numpy(),
        "q": synth.bits16(synth.decode_queries(n_seq, seed=seed + 1)["q"]),
        "q_idx": synth.decode_queries(n_seq, seed=seed + 1)["q_idx"].numpy(),
        "head_w": synth.decode_queries(n_seq, seed=seed + 1)["head_w"].numpy(),
    }


def oracle_step(oracle, wl, smp):
    scale = 1.0 / math.sqrt(512.0)
    sel = oracle.indexer_topk_batch(smp["ikeys"], smp["iscales"], smp["seq"], 4, smp["q_idx"], smp["head_w"], wl.topk)
    oracle.attention_batch(smp["q"], smp["csa"], 4, sel, smp["win"], smp["seq"], scale)
    oracle.attention_batch(smp["q"], smp["hca"], 128, None, smp["win"], smp["seq"], scale)


def cpu_baseline(wl, n_seq=2, reps=1):
    import oracle
    smp = oracle_sample(wl, n_seq)
    oracle_step(oracle, wl, smp)   # warm (page-in)
    t = time.perf_counter()
    for _ in range(reps):
        oracle_step(oracle, wl, smp)
    dt = time.perf_counter() - t
    return {"value": round(n_seq * reps / dt, 3), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n_seq} sequences x {reps} decode step(s) of {wl.name}: indexer over {wl.csa_entries} FP4 "
                      f"keys + top-{wl.topk}, CSA attention over {wl.topk}+{wl.window} entries, HCA attention over "
                      f"{wl.hca_entries}+{wl.window} entries, float64 C with OpenMP"}


def run_reference(args, wl):
    import oracle
    smp = oracle_sample(wl, 1)
    for _ in range(args.warmup):
        oracle_step(oracle, wl, smp)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(oracle, wl, smp)
    dt = time.perf_counter() - t
    v = round(args.steps / dt, 3)
    cb = {"value": v, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
          "sample": f"1 sequence per step of {wl.name} (the batch of {wl.batch} is not run: each step is a "
                    f"bounded sample), float64 C with OpenMP"}
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": wl.name, "batch_per_gpu": 1, "context": wl.context, "topk": wl.topk,
                       "window": wl.window},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    import synth
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return
    if args.warmup < 3:
        args.warmup = 3
    if world > 1:
        import datetime
        import torch
        import torch.distributed as td
        torch.cuda.set_device(local_rank)
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                              device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if res is None:
            return
        if rank == 0 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as td
            td.destroy_process_group()


if __name__ == "__main__":
    main()
