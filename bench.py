"""Benchmark of the hybrid compressed-attention decode hot path (CSA + HCA).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode1m|decode128k|prefill128k|sweep61] [--extra decode128k|none]

Workloads (seeded synthetic data resident in HBM; see synth/__init__.py):
  decode1m / decode128k  one step = one decode query per sequence through one CSA layer (append,
                         lightning-indexer top-k, sparse attention with the window branch) and one
                         HCA layer (append, dense attention with the window branch), whole batch.
                         The default run times decode1m and adds decode128k's figures under
                         "extra" in the same JSON line.
  prefill128k            one step = 131,072 raw tokens compressed by one CSA layer (ratio 4, with
                         FP4 indexer keys) and one HCA layer (ratio 128).
  sweep61                one step = one decode token per sequence through a 61-layer stack (layers
                         0-1 HCA, then CSA / HCA alternating), swept over context x batch; the
                         line's value is the 1M-token, batch-8 point, every point is under "sweep".
  mtp1m                  one step = Q = 4 query tokens per sequence (a multi-token-prediction or
                         speculative draft) at the decode1m shape: the multi-query indexer (one
                         pass over the FP4 keys for all 4), multi-query sparse CSA attention and
                         multi-query dense HCA attention.

Timing: exactly K steps are replayed from CUDA graphs (graphs of one step per cache replica, the
replicas rotating so that no step finds its data in L2 from the step before), between a
synchronize + barrier on both sides, timed with CUDA events on the launching stream; the job time
is the max over ranks.  Without --steps, K is chosen so the timed region lasts about 1.2 s.  The
kernels of the timed graphs keep their programmatic (early-launch) edges; a second capture of the
same launches with event records between the kernels gives the per-kernel times inside the
step, and a graph of each operation's calls alone (rotating over cache copies, so no launch finds
its data in L2) gives the per-launch durations behind the roofline of the dominant kernel.  `--impl reference` times the float64 CPU oracle instead (on
rank 0 only), on a bounded sample of the same workload.
"""
import argparse
import gc
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
TARGET_TIMED_S = 1.2
# kernels one decode step launches: 2 x append_kernel, indexer_topk_coop_kernel,
# 2 x (attention_tc_partial_kernel + attention_merge_kernel)
LAUNCHES_PER_STEP = 7


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default: as many as fill about 1.2 s; 10 for the reference arm)")
    p.add_argument("--warmup", type=int, default=6)
    p.add_argument("--workload", default="decode1m",
                   choices=["decode1m", "decode128k", "prefill128k", "sweep61", "mtp1m"])
    p.add_argument("--extra", default="decode128k", help="decode workloads reported under 'extra' ('none')")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--sweep-contexts", default=None, help="comma list (sweep61)")
    p.add_argument("--sweep-batches", default=None, help="comma list (sweep61)")
    p.add_argument("--profile", action="store_true",
                   help="run a few eager steps on one cache replica (for ncu captures); prints no JSON")
    return p.parse_args(argv)


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
            time.sleep(0.3)   # the first sample lands before the timed region starts
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def mark(self):
        return time.perf_counter()

    def stop(self, t0=None, t1=None):
        """Median SM clock over the samples taken between t0 and t1 (host times of the timed
        region; all samples when not given) and every throttle reason seen in them."""
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
        for ts, line in self.lines:
            if t0 is not None and not (t0 <= ts <= t1 + 0.15):
                continue
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
# Bookkeeping shared by every workload.
# ------------------------------------------------------------------------------------------
def algorithmic_bytes(wl):
    """Bytes the method must move per decode step (whole batch), by operation."""
    B = wl.batch
    return {
        "indexer": B * wl.csa_entries * 40,                          # 32 B codes + 8 B scales / entry
        "csa_attention": B * (wl.topk + wl.window) * 576,
        "hca_attention": B * (wl.hca_entries + wl.window) * 576,
        "append": 2 * B * (1024 + 576) + B * 4 * 1024 // 4,          # token in, window entry out, tail reads
    }


def prefill_bytes(T):
    """Bytes one prefill step moves: raw bf16 [T,512] + gates in, entries (+ FP4 keys) out."""
    return {"csa_compress": T * 1024 + T * 4 + (T // 4) * (576 + 40),
            "hca_compress": T * 1024 + T * 4 + (T // 128) * 576}


# ncu summaries under profiles/: DRAM read+write bytes per launch, valid only while the kernel's
# sources hash to the value recorded with the capture (a changed kernel reports null).
PROFILES = {
    ("indexer", "decode1m"): ("indexer_topk_decode1m.md", "indexer.cu", ""),
    ("csa_attention", "decode1m"): ("attention_tc_partial_decode1m.md", "attention_tc.cu", " (CSA)"),
    ("hca_attention", "decode1m"): ("attention_tc_partial_decode1m.md", "attention_tc.cu", " (HCA)"),
    ("attention", "decode1m"): ("attention_tc_partial_decode1m.md", "attention_tc.cu", " (CSA+HCA)"),
    ("csa_compress", "prefill128k"): ("compress_prefill128k.md", "compress.cu", " (CSA)"),
    ("hca_compress", "prefill128k"): ("compress_prefill128k.md", "compress.cu", " (HCA)"),
    ("indexer", "mtp1m"): ("indexer_multi_mtp1m.md", "indexer_multi.cu", ""),
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
    if (kernel, workload) not in PROFILES:
        return None
    md, cu, tag = PROFILES[(kernel, workload)]
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


def barrier(world):
    if world > 1:
        import torch.distributed as td
        td.barrier()


def capture(torch, dev, fn):
    """A CUDA graph of whatever fn() launches on the current stream."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def replay_steps(rounds_graph, single_graphs, n):
    """Replays exactly n steps: n // R replays of the R-step graph, then n % R one-step graphs."""
    R = len(single_graphs)
    for _ in range(n // R):
        rounds_graph.replay()
    for r in range(n % R):
        single_graphs[r].replay()


def time_steps(torch, dev, world, rounds_graph, single_graphs, n, clocks=None):
    """Device time (ms, max over ranks) of exactly n steps, bracketed by synchronize + barrier."""
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    h0 = time.perf_counter()
    t0.record()
    replay_steps(rounds_graph, single_graphs, n)
    t1.record()
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    barrier(world)
    return max_over_ranks(t0.elapsed_time(t1), dev), (h0, h1)


def auto_steps(torch, rounds_graph, single_graphs, R, lo=60, hi=None):
    """Steps that fill about TARGET_TIMED_S, from a short timing of the R-step graph."""
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(5):
        rounds_graph.replay()
    t1.record()
    torch.cuda.synchronize()
    per_step_s = t0.elapsed_time(t1) * 1e-3 / (5 * R)
    n = max(lo, int(math.ceil(TARGET_TIMED_S / per_step_s)))
    return min(n, hi) if hi else n


# ------------------------------------------------------------------------------------------
# Decode workloads (decode1m, decode128k): one CSA + one HCA layer.
# ------------------------------------------------------------------------------------------
def run_decode(args, wl, rank, world, local_rank, steps=None, with_e2e=True):
    import torch
    import compressed_sparse_long_decode_b200 as csld
    import synth
    n_rep = 1 if args.profile else REPLICAS
    dev = torch.device("cuda", local_rank)
    B, W, k = wl.batch, wl.window, wl.topk
    scale = 1.0 / math.sqrt(512.0)
    g = synth.gen(1234 + rank, dev)

    # --- caches: n_rep independent copies of the CSA and the HCA layer ---------------------
    inp = synth.prefill_inputs(8, seed=rank)
    layers = []
    for r in range(n_rep):
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

    # --- per-step inputs, resident in HBM --------------------------------------------------
    toks = synth.decode_tokens(B * n_rep, seed=100 + rank, device=dev)
    qs = synth.decode_queries(B * n_rep, seed=200 + rank, device=dev)
    x_slot = toks["kv"].view(n_rep, B, 512)
    z_slot = toks["gate"].view(n_rep, B)
    q_all = qs["q"].view(n_rep, B, 16, 512)
    qi_all = qs["q_idx"].view(n_rep, B, 4, 64)
    hw_all = qs["head_w"].view(n_rep, B, 4)
    sel = torch.empty((n_rep, B, k), dtype=torch.int32, device=dev)
    out_csa = torch.empty((n_rep, B, 16, 512), dtype=torch.float32, device=dev)
    out_hca = torch.empty_like(out_csa)
    lse_csa = torch.empty((n_rep, B, 16), dtype=torch.float32, device=dev)
    lse_hca = torch.empty_like(lse_csa)
    ws_idx = [csld.indexer_workspace(B, layers[0][0].capacity, k, dev) for _ in range(n_rep)]
    ws_att = csld.attention_workspace(B, max(wl.csa_cap, wl.hca_cap), k, W, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    names = ("indexer", "csa_attention", "hca_attention")
    ev = {n: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * n_rep)] for n in names}

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
    for r in range(n_rep):
        step(r, False)
    torch.cuda.synchronize()
    if args.profile:
        for _ in range(args.steps or 3):
            step(0, False)
        torch.cuda.synchronize()
        assert err.item() == 0
        print(f"profile run ok: {args.steps or 3} eager steps of {wl.name} on one replica", flush=True)
        return None

    # graphs: one step per replica, and one round (a step on every replica), without
    # instrumentation (the timed ones), and one instrumented round (per-kernel times)
    singles = [capture(torch, dev, lambda r=r: step(r, False)) for r in range(n_rep)]
    rounds = capture(torch, dev, lambda: [step(r, False) for r in range(n_rep)])
    instr = capture(torch, dev, lambda: [step(r, True) for r in range(n_rep)])

    replay_steps(rounds, singles, max(3, args.warmup))
    torch.cuda.synchronize()
    if steps is None:
        steps = auto_steps(torch, rounds, singles, n_rep)
    clocks = ClockSampler(local_rank)
    clocks.start()
    ms, (h0, h1) = time_steps(torch, dev, world, rounds, singles, steps)
    clk = clocks.stop(h0, h1)
    assert err.item() == 0, f"device error word {err.item()}"

    # per-kernel times from the instrumented graph (event records break the early-launch edges,
    # so these include each kernel's launch gap)
    n_instr = 20
    per = {n: 0.0 for n in names}
    for _ in range(n_instr):
        instr.replay()
        torch.cuda.synchronize()
        for n, evs in ev.items():
            per[n] += sum(evs[2 * r].elapsed_time(evs[2 * r + 1]) for r in range(n_rep))
    avg = {n: per[n] / (n_instr * n_rep) for n in per}             # ms per launch (one call per step)

    # Each operation alone, graph-replayed with its early-launch edges kept: the attention calls
    # (CSA on the selections of the last step, HCA) rotating over 8 HCA cache copies so a round
    # touches ~350 MB before any data comes round again, and the indexer calls over the 3
    # replicas (252 MB per round).  These give the per-launch durations of the roofline.
    n_hca = 8
    hca_copies = [layers[r % n_rep][1].comp_kv if r < n_rep else layers[r % n_rep][1].comp_kv.clone()
                  for r in range(n_hca)]

    def att_round():
        for r in range(n_hca):
            csa, hca = layers[r % n_rep]
            csld.hybrid_decode_attention(q_all[r % n_rep], csa.comp_kv, 4, sel[r % n_rep], csa.win_kv, W, csa.seq_len,
                                         scale, out=out_csa[r % n_rep], lse=lse_csa[r % n_rep], ws=ws_att, err=err)
            csld.hybrid_decode_attention(q_all[r % n_rep], hca_copies[r], 128, None, hca.win_kv, W, hca.seq_len,
                                         scale, out=out_hca[r % n_rep], lse=lse_hca[r % n_rep], ws=ws_att, err=err)

    def idx_round():
        for r in range(n_rep):
            csa = layers[r][0]
            csld.indexer_topk(csa.ikeys, csa.iscales, csa.seq_len, 4, qi_all[r], hw_all[r], k, out=sel[r],
                              ws=ws_idx[r], err=err)

    op_ms = {}
    for name, fn, per_round in (("attention", att_round, n_hca), ("indexer", idx_round, n_rep)):
        g_op = capture(torch, dev, fn)
        g_op.replay()
        n_op = max(20, int(0.3 / max(1e-6, avg["csa_attention" if name == "attention" else "indexer"] * 1e-3 *
                                       per_round)))
        ms_op, _ = time_steps(torch, dev, world, g_op, [g_op], n_op)
        op_ms[name] = ms_op / (n_op * per_round)                    # ms per step (one call of each layer)
        del g_op
    del hca_copies
    assert err.item() == 0, f"device error word {err.item()}"

    e2e = run_decode_e2e(csld, torch, layers, wl, dev, k, W, scale, ws_idx, ws_att, err, steps, world) \
        if with_e2e else None

    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    bytes_ = algorithmic_bytes(wl)
    step_bytes = sum(bytes_.values())
    ms_step = ms / steps
    att_bytes = bytes_["csa_attention"] + bytes_["hca_attention"]
    att_ms = op_ms["attention"]
    # the dominant kernel of the step, and its per-launch duration from its own graph
    dom_ms = {"indexer": op_ms["indexer"], "attention": att_ms}
    dom_bytes = {"indexer": bytes_["indexer"], "attention": att_bytes}
    dominant = max(dom_ms, key=dom_ms.get)
    achieved = dom_bytes[dominant] / (dom_ms[dominant] * 1e-3) / 1e9
    return {
        "value": round(job_throughput(B * steps, ms, world), 1), "steps": steps, "ms_per_step": round(ms_step, 5),
        "config": {"workload": wl.name, "batch_per_gpu": B, "context": wl.context, "csa_entries": wl.csa_entries,
                   "hca_entries": wl.hca_entries, "topk": k, "window": W, "heads": 16, "dim": 512,
                   "l2": f"{n_rep} rotating cache replicas ({n_rep}x "
                         f"{(layers[0][0].comp_kv.numel() + layers[0][1].comp_kv.numel()) / 1e9:.2f} GB); "
                         f"each step touches {step_bytes / 1e6:.1f} MB not left in L2 by the step before",
                   "parallelism": f"replicas x{world} (independent sequences per GPU, no collective)"},
        "hbm": {"algorithmic_bytes_per_step": step_bytes,
                "gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
                "frac_of_peak": round(step_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak, 4),
                "frac_of_8tbs": round(step_bytes / (ms_step * 1e-3) / 1e9 / 8000.0, 4)},
        "kernels_ms_per_step": {n: round(v, 5) for n, v in avg.items()},
        "roofline": {"kernel": "indexer_topk" if dominant == "indexer" else
                     "hybrid_decode_attention (CSA + HCA calls)", "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": profiled_traffic(dominant, wl.name),
                     "algorithmic_bytes_per_launch": dom_bytes[dominant],
                     "ms_per_launch": round(dom_ms[dominant], 5),
                     "timing": "the operation's calls alone, graph-replayed with early-launch edges, CUDA events"},
        "roofline_in_step": {n: {"achieved_gbs": round(bytes_[n] / (avg[n] * 1e-3) / 1e9, 1),
                                 "frac": round(bytes_[n] / (avg[n] * 1e-3) / 1e9 / hbm_peak, 4)} for n in avg},
        "attention": {"bytes_per_step": att_bytes, "ms_per_step": round(att_ms, 5),
                      "gbs": round(att_bytes / (att_ms * 1e-3) / 1e9, 1),
                      "frac": round(att_bytes / (att_ms * 1e-3) / 1e9 / hbm_peak, 4),
                      "timing": "CSA + HCA hybrid_decode_attention calls alone, graph-replayed over 8 HCA cache "
                                "copies (early-launch edges kept)"},
        "indexer": {"bytes_per_step": bytes_["indexer"], "ms_per_step": round(op_ms["indexer"], 5),
                    "gbs": round(bytes_["indexer"] / (op_ms["indexer"] * 1e-3) / 1e9, 1),
                    "frac": round(bytes_["indexer"] / (op_ms["indexer"] * 1e-3) / 1e9 / hbm_peak, 4)},
        "clocks": clk,
        "gpu_launches": LAUNCHES_PER_STEP * steps,
        "e2e": e2e,
    }


def run_decode_e2e(csld, torch, layers, wl, dev, k, W, scale, ws_idx, ws_att, err, steps, world):
    """Same step through the public API with the step's inputs copied from pinned host memory
    and both layers' outputs copied back, inside the timed region (graph-replayed)."""
    B = wl.batch
    n_rep = len(layers)
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
    h_out = torch.empty((n_rep, 2, B, 16, 512), dtype=torch.float32).pin_memory()
    h_lse = torch.empty((n_rep, B, 16), dtype=torch.float32).pin_memory()
    sel = torch.empty((B, k), dtype=torch.int32, device=dev)
    h2d = h_in.numel()
    d2h = h_out[0].numel() * 4 + h_lse[0].numel() * 4
    side = torch.cuda.Stream(device=dev)
    ev = [[torch.cuda.Event() for _ in range(2)] for _ in range(n_rep)]

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

    for r in range(n_rep):
        step(r)
    torch.cuda.synchronize()
    singles = [capture(torch, dev, lambda r=r: step(r)) for r in range(n_rep)]
    rounds = capture(torch, dev, lambda: [step(r) for r in range(n_rep)])
    replay_steps(rounds, singles, 3)
    ms, _ = time_steps(torch, dev, world, rounds, singles, steps)
    assert torch.isfinite(h_out).all()
    return {"value": round(job_throughput(B * steps, ms, world), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms / steps, 5), "steps": steps}


# ------------------------------------------------------------------------------------------
# Prefill compression (prefill128k): one CSA layer and one HCA layer compress 128K tokens.
# ------------------------------------------------------------------------------------------
def run_prefill(args, rank, world, local_rank):
    import torch
    import compressed_sparse_long_decode_b200 as csld
    import synth
    T = synth.PREFILL_TOKENS
    n_rep = 1 if args.profile else REPLICAS
    dev = torch.device("cuda", local_rank)
    inp = synth.prefill_inputs(8, seed=rank, device=dev)
    g = synth.gen(4321 + rank, dev)
    # distinct raw K/V for the CSA and the HCA layer of every replica (3 x 2 x 134 MB)
    raw = [[synth.bf16_normal((T, 512), g, dev) for _ in range(2)] for _ in range(n_rep)]
    gate = [[torch.randn(T, generator=g, device=dev) for _ in range(2)] for _ in range(n_rep)]
    kv4 = [torch.empty((T // 4, 576), dtype=torch.uint8, device=dev) for _ in range(n_rep)]
    ik = [torch.empty((T // 4, 32), dtype=torch.uint8, device=dev) for _ in range(n_rep)]
    isc = [torch.empty((T // 4, 2), dtype=torch.float32, device=dev) for _ in range(n_rep)]
    kv128 = [torch.empty((T // 128, 576), dtype=torch.uint8, device=dev) for _ in range(n_rep)]
    names = ("csa_compress", "hca_compress")
    ev = {n: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * n_rep)] for n in names}

    def step(r, timed_events):
        if timed_events:
            ev["csa_compress"][2 * r].record()
        csld.csa_compress(raw[r][0], gate[r][0], inp["bias4"], inp["w_idx"], kv4[r], ik[r], isc[r])
        if timed_events:
            ev["csa_compress"][2 * r + 1].record()
            ev["hca_compress"][2 * r].record()
        csld.hca_compress(raw[r][1], gate[r][1], inp["bias128"], kv128[r])
        if timed_events:
            ev["hca_compress"][2 * r + 1].record()

    for r in range(n_rep):
        step(r, False)
    torch.cuda.synchronize()
    if args.profile:
        for _ in range(args.steps or 3):
            step(0, False)
        torch.cuda.synchronize()
        print(f"profile run ok: {args.steps or 3} eager prefill steps on one replica", flush=True)
        return None
    singles = [capture(torch, dev, lambda r=r: step(r, False)) for r in range(n_rep)]
    rounds = capture(torch, dev, lambda: [step(r, False) for r in range(n_rep)])
    instr = capture(torch, dev, lambda: [step(r, True) for r in range(n_rep)])
    replay_steps(rounds, singles, max(3, args.warmup))
    steps = args.steps or auto_steps(torch, rounds, singles, n_rep, lo=30)
    clocks = ClockSampler(local_rank)
    clocks.start()
    ms, (h0, h1) = time_steps(torch, dev, world, rounds, singles, steps)
    clk = clocks.stop(h0, h1)
    n_instr = 10
    per = {n: 0.0 for n in names}
    for _ in range(n_instr):
        instr.replay()
        torch.cuda.synchronize()
        for n, evs in ev.items():
            per[n] += sum(evs[2 * r].elapsed_time(evs[2 * r + 1]) for r in range(n_rep))
    avg = {n: per[n] / (n_instr * n_rep) for n in per}

    # Each compressor alone, graph-replayed over the replicas (every launch reads 134 MB of raw
    # K/V that the launch before it did not, above the 126 MB L2): the per-launch durations of the
    # roofline, without the event nodes that the instrumented step puts between the kernels.
    def op_round(name):
        for r in range(n_rep):
            if name == "csa_compress":
                csld.csa_compress(raw[r][0], gate[r][0], inp["bias4"], inp["w_idx"], kv4[r], ik[r], isc[r])
            else:
                csld.hca_compress(raw[r][1], gate[r][1], inp["bias128"], kv128[r])

    alone = {}
    for n in names:
        g_op = capture(torch, dev, lambda n=n: op_round(n))
        g_op.replay()
        n_op = max(20, int(0.3 / max(1e-6, avg[n] * 1e-3 * n_rep)))
        ms_op, _ = time_steps(torch, dev, world, g_op, [g_op], n_op)
        alone[n] = ms_op / (n_op * n_rep)
        del g_op

    # end to end: the raw K/V and gates of both layers from pinned host memory, the entries and
    # keys back, every step (copy-engine transfers: a prefill moves 268 MB in)
    h_raw = [t.cpu().pin_memory() for t in raw[0]]
    h_gate = [t.cpu().pin_memory() for t in gate[0]]
    h_out = [torch.empty_like(t, device="cpu").pin_memory() for t in (kv4[0], ik[0], isc[0], kv128[0])]

    def e2e_step():
        raw[0][0].copy_(h_raw[0], non_blocking=True)
        gate[0][0].copy_(h_gate[0], non_blocking=True)
        raw[0][1].copy_(h_raw[1], non_blocking=True)
        gate[0][1].copy_(h_gate[1], non_blocking=True)
        step(0, False)
        for h, d in zip(h_out, (kv4[0], ik[0], isc[0], kv128[0])):
            h.copy_(d, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    eg = capture(torch, dev, e2e_step)
    eg.replay()
    n_e2e = max(10, min(steps, 200))
    ms_e2e, _ = time_steps(torch, dev, world, eg, [eg], n_e2e)
    h2d = sum(t.numel() * t.element_size() for t in h_raw + h_gate)
    d2h = sum(t.numel() * t.element_size() for t in h_out)

    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    bytes_ = prefill_bytes(T)
    dominant = max(alone, key=alone.get)
    achieved = bytes_[dominant] / (alone[dominant] * 1e-3) / 1e9
    step_bytes = sum(bytes_.values())
    ms_step = ms / steps
    proj_flop = 2 * (T // 4) * 512 * 64
    return {
        "metric": "prefill compression tokens/s & HBM GB/s (one CSA + one HCA layer, 128K tokens)",
        "value": round(job_throughput(T * steps, ms, world), 1), "unit": "prefill tokens/s", "n_gpus": world,
        "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 raw K/V -> e4m3+bf16 entries, e2m1 indexer keys; fp32 pooling, bf16 projection",
        "data": "synthetic (seeded)",
        "config": {"workload": "prefill128k", "tokens": T, "csa_entries": T // 4, "hca_entries": T // 128,
                   "l2": f"{n_rep} rotating replicas, distinct raw K/V per layer ({2 * T * 1024 / 1e6:.0f} MB "
                         "of raw reads per step, above the 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "hbm": {"algorithmic_bytes_per_step": step_bytes, "gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
                "frac_of_peak": round(step_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak, 4)},
        "kernels_ms_per_step": {n: round(v, 5) for n, v in avg.items()},
        "kernels_ms_alone": {n: round(v, 5) for n, v in alone.items()},
        "roofline": {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": profiled_traffic(dominant, "prefill128k"),
                     "algorithmic_bytes_per_launch": bytes_[dominant], "ms_per_launch": round(alone[dominant], 5),
                     "timing": "the kernel's calls alone, graph-replayed over the replicas, CUDA events"},
        "roofline_all": {n: {"achieved_gbs": round(bytes_[n] / (alone[n] * 1e-3) / 1e9, 1),
                             "frac": round(bytes_[n] / (alone[n] * 1e-3) / 1e9 / hbm_peak, 4),
                             "in_step_frac": round(bytes_[n] / (avg[n] * 1e-3) / 1e9 / hbm_peak, 4)} for n in alone},
        "projection": {"flop_per_step": proj_flop,
                       "tflops": round(proj_flop / (alone["csa_compress"] * 1e-3) / 1e12, 2)},
        "clocks": clk,
        "gpu_launches": 2 * steps,
        "e2e": {"value": round(job_throughput(T * n_e2e, ms_e2e, world), 1), "unit": "prefill tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e / n_e2e, 5),
                "steps": n_e2e},
    }


# ------------------------------------------------------------------------------------------
# Multi-query decode (mtp1m): Q draft tokens per sequence at the decode1m shape.
# ------------------------------------------------------------------------------------------
MTP_Q = 4


def run_mtp(args, rank, world, local_rank):
    import torch
    import compressed_sparse_long_decode_b200 as csld
    import synth
    wl = synth.WORKLOADS["decode1m"]
    Q = MTP_Q
    B, W, k = wl.batch, wl.window, wl.topk
    n_rep = 1 if args.profile else REPLICAS
    dev = torch.device("cuda", local_rank)
    scale = 1.0 / math.sqrt(512.0)
    g = synth.gen(4242 + rank, dev)
    W_ring = W + Q - 1
    reps = []
    for r in range(n_rep):
        csa_kv = synth.random_entries((B, wl.csa_cap), g, dev)
        hca_kv = synth.random_entries((B, wl.hca_cap), g, dev)
        ring_c = synth.random_entries((B, W_ring), g, dev)
        ring_h = synth.random_entries((B, W_ring), g, dev)
        ik, isc = synth.random_ikeys(B, wl.csa_cap, g, dev, heavy_frac=wl.heavy_frac, n_valid=wl.csa_entries)
        reps.append(dict(csa=csa_kv, hca=hca_kv, ring_c=ring_c, ring_h=ring_h, ik=synth.ikeys_swap_halves(ik), isc=isc,
                         ws=csld.indexer_multi_workspace(B, Q, wl.csa_cap, dev)))
        del ik
    seq = torch.full((B,), wl.context, dtype=torch.int32, device=dev)
    qd = synth.decode_queries(B * Q * n_rep, seed=300 + rank, device=dev)
    q_all = qd["q"].view(n_rep, B, Q, 16, 512)
    qgen = synth.gen(301 + rank, dev)
    qi_all = torch.randn((n_rep, B, Q, 4, 64), generator=qgen, device=dev)
    hw_all = torch.randn((n_rep, B, Q, 4), generator=qgen, device=dev).abs()
    sel = torch.empty((n_rep, B, Q, k), dtype=torch.int32, device=dev)
    out_c = torch.empty((n_rep, B, Q, 16, 512), dtype=torch.float32, device=dev)
    out_h = torch.empty_like(out_c)
    ws_att = csld.attention_workspace(B * Q, max(wl.csa_cap, wl.hca_cap), k, W, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ev = {n: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * n_rep)]
          for n in ("indexer", "csa_attention", "hca_attention")}

    def step(r, timed):
        x = reps[r]
        if timed:
            ev["indexer"][2 * r].record()
        csld.indexer_topk_multi(x["ik"], x["isc"], seq, 4, qi_all[r], hw_all[r], k, out=sel[r], ws=x["ws"], err=err)
        if timed:
            ev["indexer"][2 * r + 1].record()
            ev["csa_attention"][2 * r].record()
        csld.hybrid_decode_attention_multi(q_all[r], x["csa"], 4, sel[r], x["ring_c"], W, seq, scale, out=out_c[r],
                                           ws=ws_att, err=err)
        if timed:
            ev["csa_attention"][2 * r + 1].record()
            ev["hca_attention"][2 * r].record()
        csld.hybrid_decode_attention_multi(q_all[r], x["hca"], 128, None, x["ring_h"], W, seq, scale, out=out_h[r],
                                           ws=ws_att, err=err)
        if timed:
            ev["hca_attention"][2 * r + 1].record()

    for r in range(n_rep):
        step(r, False)
    torch.cuda.synchronize()
    if args.profile:
        for _ in range(args.steps or 3):
            step(0, False)
        torch.cuda.synchronize()
        assert err.item() == 0
        print(f"profile run ok: {args.steps or 3} eager steps of mtp1m on one replica", flush=True)
        return None
    singles = [capture(torch, dev, lambda r=r: step(r, False)) for r in range(n_rep)]
    rounds = capture(torch, dev, lambda: [step(r, False) for r in range(n_rep)])
    instr = capture(torch, dev, lambda: [step(r, True) for r in range(n_rep)])
    replay_steps(rounds, singles, max(3, args.warmup))
    steps = args.steps or auto_steps(torch, rounds, singles, n_rep)
    clocks = ClockSampler(local_rank)
    clocks.start()
    ms, (h0, h1) = time_steps(torch, dev, world, rounds, singles, steps)
    clk = clocks.stop(h0, h1)
    per = {n: 0.0 for n in ev}
    for _ in range(10):
        instr.replay()
        torch.cuda.synchronize()
        for n, evs in ev.items():
            per[n] += sum(evs[2 * r].elapsed_time(evs[2 * r + 1]) for r in range(n_rep))
    avg = {n: per[n] / (10 * n_rep) for n in per}
    assert err.item() == 0, f"device error word {err.item()}"
    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    bytes_ = {"indexer": B * wl.csa_entries * 40 + 2 * B * Q * wl.csa_entries * 4,   # keys once; score keys out and in
              "csa_attention": B * Q * (k + W) * 576,
              "hca_attention": B * (wl.hca_entries + W + Q - 1) * 576}              # the cache once per step
    dominant = max(avg, key=avg.get)
    achieved = bytes_[dominant] / (avg[dominant] * 1e-3) / 1e9
    ms_step = ms / steps
    return {
        "metric": METRIC, "value": round(job_throughput(B * Q * steps, ms, world), 1), "unit": UNIT,
        "n_gpus": world, "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3+bf16 KV, e2m1 indexer keys; tcgen05 e2m1, e4m3 and bf16 MMA, fp32 accumulate",
        "data": "synthetic (seeded)",
        "config": {"workload": "mtp1m", "batch_per_gpu": B, "queries_per_sequence": Q, "context": wl.context,
                   "topk": k, "window": W,
                   "l2": f"{n_rep} rotating cache replicas", "parallelism": f"replicas x{world}"},
        "kernels_ms_per_step": {n: round(v, 5) for n, v in avg.items()},
        "indexer_keys_gbs": round(B * wl.csa_entries * 40 / (avg["indexer"] * 1e-3) / 1e9, 1),
        "roofline": {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": profiled_traffic(dominant, "mtp1m"), "algorithmic_bytes_per_launch": bytes_[dominant]},
        "clocks": clk, "gpu_launches": steps * 7,   # indexer: score, gather, select; 2 x attention: partial, merge
    }


# ------------------------------------------------------------------------------------------
# The 61-layer stack (sweep61).
# ------------------------------------------------------------------------------------------
def stack_bytes_per_step(kinds, B, context, topk, window):
    """Bytes one decode step of the stack must move (whole batch): per CSA layer the indexer's
    40 B per visible entry and (k + W) entries of attention, per HCA layer every visible entry
    plus the window, 576 B each."""
    b_idx = b_att = 0
    for kind in kinds:
        if kind == "csa":
            b_idx += B * (context // 4) * 40
            b_att += B * (topk + window) * 576
        else:
            b_att += B * (context // 128 + window) * 576
    return b_idx, b_att


def stack_cache_bytes(B, n_csa, n_hca, csa_cap, hca_cap, window):
    return B * (n_csa * (csa_cap * (576 + 40) + window * 576 + 4 * (1024 + 4)) +
                n_hca * (hca_cap * 576 + window * 576 + 128 * (1024 + 4)))


def sweep_e2e(torch, dev, world, csld, stack, kinds, kv_new, gate_new, q, q_idx, head_w, out, scale, B, n):
    """The stack's decode step end to end: every layer's inputs (new token, gate, attention query,
    indexer query, head weights) from pinned host memory and every layer's output back, inside
    the timed region (copy-engine transfers around the graph-replayed layers)."""
    h_in = [t.cpu().pin_memory() for t in (kv_new, gate_new, q, q_idx, head_w)]
    d_in = (kv_new, gate_new, q, q_idx, head_w)
    h_out = torch.empty_like(out, device="cpu").pin_memory()

    def step():
        for d, h in zip(d_in, h_in):
            d.copy_(h, non_blocking=True)
        stack.step(kv_new, gate_new, q, q_idx, head_w, scale, out)
        h_out.copy_(out, non_blocking=True)

    step()
    torch.cuda.synchronize()
    g = capture(torch, dev, step)
    g.replay()
    ms, _ = time_steps(torch, dev, world, g, [g], n)
    assert not stack.err.item(), f"device error word {stack.err.item()}"
    return {"value": round(job_throughput(B * n, ms, world), 1), "unit": UNIT,
            "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_in),
            "d2h_bytes_per_step": h_out.numel() * 4, "ms_per_step": round(ms / n, 4), "steps": n}


def run_sweep(args, rank, world, local_rank):
    import torch
    import compressed_sparse_long_decode_b200 as csld
    import synth
    dev = torch.device("cuda", local_rank)
    scale = 1.0 / math.sqrt(512.0)
    kinds = csld.layer_pattern(synth.SWEEP_LAYERS)
    L = len(kinds)
    n_csa, n_hca = kinds.count("csa"), kinds.count("hca")
    k, W = synth.SWEEP_TOPK, synth.SWEEP_WINDOW
    contexts = [int(x) for x in args.sweep_contexts.split(",")] if args.sweep_contexts else list(synth.SWEEP_CONTEXTS)
    batches = [int(x) for x in args.sweep_batches.split(",")] if args.sweep_batches else list(synth.SWEEP_BATCHES)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    inp = synth.prefill_inputs(8, seed=rank, device=dev)
    points, head = [], None
    for ctx in contexts:
        for B in batches:
            slack = 8192 if ctx < 1048576 else 1024   # tokens appended while timing (capacity margin)
            csa_cap = (ctx + slack) // 4 + ((ctx + slack) // 4 & 1)
            hca_cap = (ctx + slack) // 128
            b_idx, b_att = stack_bytes_per_step(kinds, B, ctx, k, W)
            step_bytes = b_idx + b_att
            one = stack_cache_bytes(B, n_csa, n_hca, csa_cap, hca_cap, W)
            n_rep = max(1, math.ceil(3 * l2 / step_bytes))
            torch.cuda.empty_cache()
            free = torch.cuda.mem_get_info(dev)[0]
            io = L * B * (16 * 512 * (2 + 4 * 2) + 512 * 2 + 4 + 64 * 4 + 16 + 16 * 4)
            budget = 0.90 * free - 2 ** 30
            while n_rep > 1 and n_rep * one + io > budget:
                n_rep -= 1
            pt = {"context": ctx, "batch": B, "cache_gb": round(one / 1e9, 2)}
            if one + io > budget:
                pt["skipped"] = f"does not fit: {one / 1e9:.1f} GB of caches, {free / 1e9:.1f} GB free"
                points.append(pt)
                continue
            stacks = [csld.DecodeStack(B, kinds, csa_cap, hca_cap, W, k, inp["bias4"], inp["bias128"],
                                       inp["w_idx"], device=dev) for _ in range(n_rep)]
            g = synth.gen(777 + ctx + B, dev)
            # one random CSA and one random HCA layer; every other layer gets a copy of its kind
            src = {}
            for kind, lay in zip(kinds, stacks[0].layers):
                if kind in src:
                    continue
                n_ent = ctx // lay.ratio
                lay.comp_kv[:, :n_ent] = synth.random_entries((B, n_ent), g, dev)
                lay.win_kv[:] = synth.random_entries((B, W), g, dev)
                lay.tail_kv.normal_(generator=g)
                if lay.has_indexer:
                    ikk, iss = synth.random_ikeys(B, lay.capacity, g, dev, n_valid=n_ent)
                    lay.ikeys.copy_(synth.ikeys_swap_halves(ikk))
                    lay.iscales.copy_(iss)
                    del ikk, iss
                src[kind] = lay
            for st in stacks:
                for kind, lay in zip(kinds, st.layers):
                    s_ = src[kind]
                    if lay is not s_:
                        for a in ("comp_kv", "win_kv", "tail_kv", "tail_gate", "ikeys", "iscales"):
                            if getattr(lay, a) is not None:
                                getattr(lay, a).copy_(getattr(s_, a))
                    lay.seq_len.fill_(ctx)
            torch.cuda.synchronize()
            toks = synth.decode_tokens(n_rep * L * B, seed=5 + B, device=dev)
            qs = synth.decode_queries(n_rep * L * B, seed=6 + B, device=dev)
            kv_new = toks["kv"].view(n_rep, L, B, 512)
            gate_new = toks["gate"].view(n_rep, L, B)
            q = qs["q"].view(n_rep, L, B, 16, 512)
            q_idx = qs["q_idx"].view(n_rep, L, B, 4, 64)
            head_w = qs["head_w"].view(n_rep, L, B, 4)
            out = torch.empty((n_rep, L, B, 16, 512), dtype=torch.float32, device=dev)
            sel_all = torch.full((n_rep, L, B, k), -1, dtype=torch.int32, device=dev)
            ev_idx = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * L)] for _ in range(n_rep)]
            ev_att = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * L)] for _ in range(n_rep)]

            def step(r, timed):
                st = stacks[r]
                for i, lay in enumerate(st.layers):
                    csld.kv_cache_append(lay, kv_new[r, i], gate_new[r, i], st.err)
                    if lay.has_indexer:
                        if timed:
                            ev_idx[r][2 * i].record()
                        csld.indexer_topk(lay.ikeys, lay.iscales, lay.seq_len, 4, q_idx[r, i], head_w[r, i], k,
                                          out=sel_all[r, i], ws=st.ws_idx, err=st.err)
                        if timed:
                            ev_idx[r][2 * i + 1].record()
                            ev_att[r][2 * i].record()
                        csld.hybrid_decode_attention(q[r, i], lay.comp_kv, 4, sel_all[r, i], lay.win_kv, W,
                                                     lay.seq_len, scale, out=out[r, i], ws=st.ws_att, err=st.err)
                    else:
                        if timed:
                            ev_att[r][2 * i].record()
                        csld.hybrid_decode_attention(q[r, i], lay.comp_kv, 128, None, lay.win_kv, W, lay.seq_len,
                                                     scale, out=out[r, i], ws=st.ws_att, err=st.err)
                    if timed:
                        ev_att[r][2 * i + 1].record()

            for r in range(n_rep):
                step(r, False)
            torch.cuda.synchronize()
            singles = [capture(torch, dev, lambda r=r: step(r, False)) for r in range(n_rep)]
            rounds = capture(torch, dev, lambda: [step(r, False) for r in range(n_rep)])
            instr = capture(torch, dev, lambda: [step(r, True) for r in range(n_rep)])
            replay_steps(rounds, singles, max(3, args.warmup))
            is_head = (ctx, B) == (1048576, 8)
            steps = args.steps if (args.steps and is_head) else auto_steps(
                torch, rounds, singles, n_rep, lo=10, hi=n_rep * (slack - 64))
            steps = min(steps, n_rep * (slack - 64))
            clocks = ClockSampler(local_rank)
            clocks.start()
            ms, (h0, h1) = time_steps(torch, dev, world, rounds, singles, steps)
            clk = clocks.stop(h0, h1)
            n_instr = max(2, min(20, int(0.3e3 / (ms / steps * n_rep))))
            t_idx = t_att = 0.0
            for _ in range(n_instr):
                instr.replay()
                torch.cuda.synchronize()
                for r in range(n_rep):
                    for i, kind in enumerate(kinds):
                        t_att += ev_att[r][2 * i].elapsed_time(ev_att[r][2 * i + 1])
                        if kind == "csa":
                            t_idx += ev_idx[r][2 * i].elapsed_time(ev_idx[r][2 * i + 1])
            t_att /= n_instr * n_rep
            t_idx /= n_instr * n_rep
            # each operation alone over all layers (early-launch edges kept): attention calls on
            # the selections of the last step, and the indexer calls
            def att_only():
                for r in range(n_rep):
                    st = stacks[r]
                    for i, lay in enumerate(st.layers):
                        csld.hybrid_decode_attention(q[r, i], lay.comp_kv, lay.ratio,
                                                     sel_all[r, i] if lay.has_indexer else None, lay.win_kv, W,
                                                     lay.seq_len, scale, out=out[r, i], ws=st.ws_att, err=st.err)

            def idx_only():
                for r in range(n_rep):
                    st = stacks[r]
                    for i, lay in enumerate(st.layers):
                        if lay.has_indexer:
                            csld.indexer_topk(lay.ikeys, lay.iscales, lay.seq_len, 4, q_idx[r, i], head_w[r, i], k,
                                              out=sel_all[r, i], ws=st.ws_idx, err=st.err)

            op_ms = {}
            for name, fn, guess in (("attention", att_only, t_att), ("indexer", idx_only, t_idx)):
                g_op = capture(torch, dev, fn)
                g_op.replay()
                n_op = max(5, int(0.3 / max(1e-6, guess * 1e-3 * n_rep)))
                ms_op, _ = time_steps(torch, dev, world, g_op, [g_op], n_op)
                op_ms[name] = ms_op / (n_op * n_rep)
                del g_op
            errs = [int(st.err.item()) for st in stacks]
            assert not any(errs), f"device error words {errs}"
            ms_step = ms / steps
            kv_seq = stacks[0].kv_bytes_per_sequence(ctx)
            gqa8 = L * ctx * 4096
            pt.update({
                "replicas": n_rep, "steps": steps, "step_ms": round(ms_step, 4),
                "us_per_token": round(ms_step * 1e3 / B, 3),
                "value": round(job_throughput(B * steps, ms, world), 1),
                "bytes_per_step": step_bytes, "hbm_gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
                "attention": {"bytes_per_step": b_att, "ms_per_step": round(op_ms["attention"], 4),
                              "gbs": round(b_att / (op_ms["attention"] * 1e-3) / 1e9, 1),
                              "frac": round(b_att / (op_ms["attention"] * 1e-3) / 1e9 / hbm_peak, 4),
                              "us_per_layer_call": round(op_ms["attention"] * 1e3 / L, 2),
                              "in_step_ms": round(t_att, 4)},
                "indexer": {"bytes_per_step": b_idx, "ms_per_step": round(op_ms["indexer"], 4),
                            "gbs": round(b_idx / (op_ms["indexer"] * 1e-3) / 1e9, 1),
                            "frac": round(b_idx / (op_ms["indexer"] * 1e-3) / 1e9 / hbm_peak, 4),
                            "in_step_ms": round(t_idx, 4)},
                "kv_bytes_per_sequence": kv_seq, "gqa8_bf16_bytes_per_sequence": gqa8,
                "kv_frac_of_gqa8": round(kv_seq / gqa8, 5), "clocks": clk,
            })
            if is_head:
                pt["e2e"] = sweep_e2e(torch, dev, world, csld, stacks[0], kinds, kv_new[0], gate_new[0], q[0],
                                      q_idx[0], head_w[0], out[0], scale, B, min(steps, 200))
            points.append(pt)
            del stacks, singles, rounds, instr, out, toks, qs, sel_all, step, att_only, idx_only, src, lay, st, s_
            torch.cuda.synchronize()
            gc.collect()
            torch.cuda.empty_cache()
    measured = [p for p in points if "skipped" not in p]
    assert measured, "no sweep point fits"
    head = next((p for p in measured if (p["context"], p["batch"]) == (1048576, 8)),
                max(measured, key=lambda p: (p["context"], p["batch"])))
    dom = "attention" if head["attention"]["ms_per_step"] >= head["indexer"]["ms_per_step"] else "indexer"
    calls = L if dom == "attention" else n_csa
    per_launch_ms = head[dom]["ms_per_step"] / calls
    per_launch_bytes = head[dom]["bytes_per_step"] / calls
    return {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": head["steps"],
        "warmup": max(3, args.warmup), "ms_per_step": head["step_ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3+bf16 KV, e2m1 indexer keys; tcgen05 e2m1, e4m3 and bf16 MMA, fp32 accumulate",
        "data": "synthetic (seeded)",
        "config": {"workload": "sweep61", "layers": L, "csa_layers": n_csa, "hca_layers": n_hca,
                   "context": head["context"], "batch_per_gpu": head["batch"], "topk": k, "window": W,
                   "l2": "61 distinct layer caches per step; small points rotate replicas so that a step "
                         "touches more than 3 x L2 before its data comes round again",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "hybrid_decode_attention (all layers)" if dom == "attention" else
                     "indexer_topk (all CSA layers)", "bound": "hbm",
                     "achieved": round(per_launch_bytes / (per_launch_ms * 1e-3) / 1e9, 1), "peak": hbm_peak,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(per_launch_bytes / (per_launch_ms * 1e-3) / 1e9 / hbm_peak, 4),
                     "traffic": None, "algorithmic_bytes_per_launch": int(per_launch_bytes)},
        "clocks": head["clocks"],
        "gpu_launches": head["steps"] * (4 * n_csa + 3 * n_hca),
        "e2e": head.get("e2e"),
        "sweep": points,
    }


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
    qd = synth.decode_queries(n_seq, seed=seed + 1)
    return {
        "ikeys": ik.numpy(), "iscales": isc.numpy(),
        "csa": synth.random_entries((n_seq, wl.csa_cap), g).numpy(),
        "hca": synth.random_entries((n_seq, wl.hca_cap), g).numpy(),
        "win": synth.random_entries((n_seq, wl.window), g).numpy(),
        "seq": torch.full((n_seq,), wl.context, dtype=torch.int32).numpy(),
        "q": synth.bits16(qd["q"]), "q_idx": qd["q_idx"].numpy(), "head_w": qd["head_w"].numpy(),
    }


def oracle_step(oracle, wl, smp):
    scale = 1.0 / math.sqrt(512.0)
    sel = oracle.indexer_topk_batch(smp["ikeys"], smp["iscales"], smp["seq"], 4, smp["q_idx"], smp["head_w"], wl.topk)
    oracle.attention_batch(smp["q"], smp["csa"], 4, sel, smp["win"], smp["seq"], scale)
    oracle.attention_batch(smp["q"], smp["hca"], 128, None, smp["win"], smp["seq"], scale)


def timed_reps(fn, budget_s, min_reps=3):
    """Runs fn at least min_reps times and until budget_s has passed; returns (reps, seconds)."""
    reps, t = 0, time.perf_counter()
    while reps < min_reps or time.perf_counter() - t < budget_s:
        fn()
        reps += 1
    return reps, time.perf_counter() - t


def cpu_baseline(wl, n_seq=2, budget_s=10.0):
    import oracle
    smp = oracle_sample(wl, n_seq)
    oracle_step(oracle, wl, smp)   # warm (page-in)
    reps, dt = timed_reps(lambda: oracle_step(oracle, wl, smp), budget_s)
    return {"value": round(n_seq * reps / dt, 3), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n_seq} sequences x {reps} decode steps of {wl.name} ({dt:.1f} s): indexer over "
                      f"{wl.csa_entries} FP4 keys + top-{wl.topk}, CSA attention over {wl.topk}+{wl.window} "
                      f"entries, HCA attention over {wl.hca_entries}+{wl.window} entries, float64 C with OpenMP"}


def cpu_baseline_prefill(budget_s=10.0, T=16384):
    import oracle
    import synth
    inp = synth.prefill_inputs(T, seed=3)
    bits = synth.bits16(inp["raw"])
    gate = inp["gate"].numpy()

    def run():
        oracle.compress(bits, gate, inp["bias4"].numpy(), 4, inp["w_idx"].numpy())
        oracle.compress(bits, gate, inp["bias128"].numpy(), 128)

    run()
    reps, dt = timed_reps(run, budget_s)
    return {"value": round(T * reps / dt, 1), "unit": "prefill tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{T} tokens x {reps} repetitions ({dt:.1f} s) compressed at ratio 4 (with indexer keys) "
                      f"and at ratio 128, float64 C"}


def cpu_baseline_sweep(context=65536, budget_s=10.0):
    """The oracle on one sequence of one CSA and one HCA layer at `context`, scaled to a token
    through the 61-layer stack (30 CSA + 31 HCA layers)."""
    import oracle
    import synth
    wl = synth.DecodeWorkload("sweep-sample", batch=1, context=context, topk=synth.SWEEP_TOPK, slack_tokens=0)
    smp = oracle_sample(wl, 1)
    scale = 1.0 / math.sqrt(512.0)

    def csa():
        sel = oracle.indexer_topk_batch(smp["ikeys"], smp["iscales"], smp["seq"], 4, smp["q_idx"], smp["head_w"],
                                        wl.topk)
        oracle.attention_batch(smp["q"], smp["csa"], 4, sel, smp["win"], smp["seq"], scale)

    def hca():
        oracle.attention_batch(smp["q"], smp["hca"], 128, None, smp["win"], smp["seq"], scale)

    csa(), hca()
    rc, tc = timed_reps(csa, budget_s / 2)
    rh, th = timed_reps(hca, budget_s / 2)
    per_token = 30 * tc / rc + 31 * th / rh
    return {"value": round(1.0 / per_token, 4), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"one sequence at {context} tokens: {rc} CSA-layer calls and {rh} HCA-layer calls "
                      f"({tc + th:.1f} s), scaled to 30 CSA + 31 HCA layers per token, float64 C"}


def run_reference(args):
    import oracle
    import synth
    steps = args.steps or 10
    if args.workload == "prefill128k":
        T = 16384
        inp = synth.prefill_inputs(T, seed=3)
        bits, gate = synth.bits16(inp["raw"]), inp["gate"].numpy()

        def one():
            oracle.compress(bits, gate, inp["bias4"].numpy(), 4, inp["w_idx"].numpy())
            oracle.compress(bits, gate, inp["bias128"].numpy(), 128)

        for _ in range(args.warmup):
            one()
        t = time.perf_counter()
        for _ in range(steps):
            one()
        dt = time.perf_counter() - t
        v = round(T * steps / dt, 1)
        unit = "prefill tokens/s"
        metric = "prefill compression tokens/s & HBM GB/s (one CSA + one HCA layer, 128K tokens)"
        sample = f"{T} of the 131072 tokens per step, compressed at ratios 4 and 128, float64 C"
        config = {"workload": "prefill128k", "tokens": T}
    else:
        wl = synth.WORKLOADS["decode1m" if args.workload in ("sweep61", "mtp1m") else args.workload]
        smp = oracle_sample(wl, 1)
        for _ in range(args.warmup):
            oracle_step(oracle, wl, smp)
        t = time.perf_counter()
        for _ in range(steps):
            oracle_step(oracle, wl, smp)
        dt = time.perf_counter() - t
        v = round(steps / dt, 3)
        unit, metric = UNIT, METRIC
        sample = (f"1 sequence per step of {wl.name} (the batch of {wl.batch} is not run: each step is a bounded "
                  f"sample), float64 C with OpenMP")
        config = {"workload": wl.name, "batch_per_gpu": 1, "context": wl.context, "topk": wl.topk,
                  "window": wl.window}
    cb = {"value": v, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle", "sample": sample}
    return {"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": args.gpus, "steps": steps,
            "warmup": args.warmup, "ms_per_step": round(dt / steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "config": config,
            "cpu_baseline": cb, "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def decode_line(args, rank, world, local_rank):
    import synth
    wl = synth.WORKLOADS[args.workload]
    r = run_decode(args, wl, rank, world, local_rank, steps=args.steps)
    if r is None:
        return None
    res = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": r["steps"],
           "warmup": max(3, args.warmup), "ms_per_step": r["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None,
           "dtype": "e4m3+bf16 KV, e2m1 indexer keys; tcgen05 e2m1, e4m3 and bf16 MMA, fp32 accumulate",
           "data": "synthetic (seeded)"}
    res.update({k: v for k, v in r.items() if k not in ("value", "steps", "ms_per_step")})
    extras = [] if args.extra in ("", "none") else [x for x in args.extra.split(",") if x != args.workload]
    if extras:
        import torch
        res["extra"] = {}
        for name in extras:
            torch.cuda.empty_cache()
            e = run_decode(args, synth.WORKLOADS[name], rank, world, local_rank, steps=None)
            res["extra"][name] = {k: e[k] for k in ("value", "steps", "ms_per_step", "config", "hbm",
                                                    "kernels_ms_per_step", "roofline", "roofline_in_step",
                                                    "attention", "indexer", "clocks", "e2e")}
            res["gpu_launches"] += e["gpu_launches"]
    return res


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.warmup < 3:
        args.warmup = 3
    import torch
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        import torch.distributed as td
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                              device_id=torch.device("cuda", local_rank))
    try:
        if args.workload == "prefill128k":
            res = run_prefill(args, rank, world, local_rank)
            baseline = cpu_baseline_prefill
        elif args.workload == "sweep61":
            res = run_sweep(args, rank, world, local_rank)
            baseline = cpu_baseline_sweep
        elif args.workload == "mtp1m":
            res = run_mtp(args, rank, world, local_rank)
            baseline = lambda: None   # noqa: E731
        else:
            import synth
            res = decode_line(args, rank, world, local_rank)
            baseline = lambda: cpu_baseline(synth.WORKLOADS[args.workload])   # noqa: E731
        if res is None:
            return
        if rank == 0 and not args.no_cpu_baseline:
            cb = baseline()
            if cb is not None:
                res["cpu_baseline"] = cb
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as td
            td.destroy_process_group()


if __name__ == "__main__":
    main()
