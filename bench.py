"""GSA hot-path benchmark: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gsa|reference] [--workload NAME]

A step is one GSA decode step (score every completed gist -> top-k ->
unfold + attend) for the whole batch of the workload, through the C ABI of
libgsa.so.  The default workload is the Llama-3.2-1B-shaped decode at 8x
compression (16 sequences x 32 query heads / 8 kv heads, d=64, 32K raw
context, chunk 8 -> 4096 gists, top-64).  Inputs are seeded synthetic
tensors resident in HBM; L2 is flushed between timed steps (a 2x-L2 buffer
is written, then another 2x-L2 buffer is read so the dirty lines are written
back before the step) and the flush is outside the timed events.

With --gpus N (launched under torch.distributed.run) every rank runs its own
batch (different seed): decode rows are independent, so the work shards with
no collective on the data path (weak scaling).  Step time is the maximum
over ranks of the device-measured time.

--impl reference times the float64 CPU oracle instead (rank 0 only), on a
bounded sample of rows per step, with the same metric and workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "GSA decode head-queries/s"
UNIT = "head-queries/s"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="gsa", choices=["gsa", "reference"])
    p.add_argument("--workload", default="llama1b_8x")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--main-only", action="store_true", help="skip the other workloads")
    p.add_argument("--extra-only", action="store_true",
                   help="run only the --extra workloads (no headline line; for profiler captures of one workload)")
    p.add_argument("--extra", default="qwen7b_16x,qwen7b_16x_excl,hgsa_32x,hgsa2_32x,prefill_32k,prefill_llama1b_32k,llama1b_8x_topp,llama1b_8x_bwd,qwen7b_16x_bwd,llama1b_8x_giststep,kvreuse_qwen7b",
                   help="comma-separated other workloads to measure after the headline one")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline")
    p.add_argument("--sweep", action="store_true",
                   help="context-length sweep of flat, one-level and two-level H-GSA decode (bytes and time per "
                        "step); one JSON line per point, then a summary line")
    return p.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------ helpers
def peaks():
    f = ROOT / "MEASURED_PEAKS.json"
    if f.exists():
        d = json.loads(f.read_text())
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,clocks.mem,clocks.max.mem")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return None
        rows = []
        for line in Path(self.file.name).read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mem = (float(parts[9]), float(parts[10])) if len(parts) >= 11 else None
            except ValueError:
                mem = None
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9], mem))
            except ValueError:
                continue
        os.unlink(self.file.name)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags, _ in rows for i, f in enumerate(flags) if f.lower() == "active"})
        out = {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
               "reasons": reasons, "samples": len(rows)}
        mem = [r[3] for r in rows if r[3] is not None]
        if mem:  # a memory clock below its maximum caps HBM bandwidth
            out["mem_mhz"] = statistics.median(m[0] for m in mem)
            out["mem_max_mhz"] = max(m[1] for m in mem)
        return out


def algorithmic_bytes(cfg, x, sel):
    """Bytes the method must move for one step: every gist key (+ value in
    the default set), the raw K/V rows of the union of selected chunks per
    (b, kv head), selected gist values in exclude mode, own rows, q and out."""
    e = 2 if cfg.dtype == "bf16" else 4
    B, hq, hkv, d, c = cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.chunk
    G = hq // hkv
    N = cfg.n_gists
    gist = B * hkv * N * d * e * (1 if cfg.exclude else 2)
    s = sel.reshape(B, hkv, G, -1).cpu()
    union = 0
    for b in range(B):
        for kv in range(hkv):
            u = torch.unique(s[b, kv])
            union += int((u >= 0).sum())
    raw = union * c * d * e * 2
    gsel = union * d * e if cfg.exclude else 0
    own = B * hkv * 1 * d * e * 2
    qo = B * hq * d * e + B * hq * d * 4
    return {"gist": gist, "raw_union": raw, "gist_sel": gsel, "own": own, "q_out": qo,
            "total": gist + raw + gsel + own + qo, "union_chunks": union}


def score_kernel_bytes(cfg):
    e = 2 if cfg.dtype == "bf16" else 4
    return cfg.batch * cfg.hkv * cfg.n_gists * cfg.d * e * (1 if cfg.exclude else 2)


# --------------------------------------------------------------- CPU oracle
def oracle_rate(x_host, cfg, rows_per_call, target_s, max_calls=1000):
    """Time the float64 oracle on repeated calls of `rows_per_call` rows."""
    import oracle
    o = oracle.get()
    n_rows = cfg.batch * cfg.hq
    rows = np.arange(rows_per_call) % n_rows
    t0 = time.perf_counter()
    calls = 0
    while True:
        o.decode(x_host["q"], x_host["gist_k"], x_host["gist_v"], x_host["raw_k"], x_host["raw_v"],
                 x_host["n_gists"], x_host["own_len"], chunk=cfg.chunk, topk=cfg.topk, exclude=cfg.exclude,
                 rows=rows)
        calls += 1
        el = time.perf_counter() - t0
        if el >= target_s or calls >= max_calls:
            break
    return calls * rows_per_call / el, calls, el, o.default_threads()


def host_copy(x):
    from long_context_gsa_b200.workloads import to_oracle
    return {k: to_oracle(v) for k, v in x.items() if k in ("q", "gist_k", "gist_v", "raw_k", "raw_v", "n_gists",
                                                           "own_len")}


# ---------------------------------------------------------------- GSA arm
class Flusher:
    """Write a 2x-L2 buffer, then read another one, so the written lines are
    evicted (written back) before the next timed step starts."""

    def __init__(self, dev):
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        n = max(2 * l2, 256 << 20)
        self.w = torch.empty(n, dtype=torch.uint8, device=dev)
        self.r = torch.ones(n // 4, dtype=torch.int32, device=dev)
        self.sink = torch.empty((), dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.amax(self.r, dim=0, out=self.sink)


def timed_steps(step, steps, flush, n_marks=1):
    """Run `steps` steps, L2 flushed before each; step(evs) records events
    evs[0..n_marks] on the current stream.  Returns [steps, n_marks] ms."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks + 1)] for _ in range(steps)]
    for s in range(steps):
        flush()
        step(ev[s])
    torch.cuda.synchronize()
    return np.array([[ev[s][i].elapsed_time(ev[s][i + 1]) for i in range(n_marks)] for s in range(steps)])


def pipelined_e2e(G, x, desc, out, sel, ssc, ws, steps):
    """A serving loop through gsa_decode: step s's query goes host -> device
    on one copy stream while step s-1 computes, and step s's output comes
    back device -> host on a second copy stream while step s+1 computes
    (two buffers each way).  Every step copies its input in and its result
    out inside the timed region.  The loop runs back to back: its inputs
    (gist and raw K/V) are larger than L2, so no flush runs between steps.
    Returns the loop's total time in ms (events on the compute stream)."""
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    q_host = [x["q"].cpu().pin_memory() for _ in range(2)]
    q_dev = [torch.empty_like(x["q"]) for _ in range(2)]
    out_dev = [torch.empty_like(out) for _ in range(2)]
    out_host = [torch.empty_like(out, device="cpu").pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for i in range(2):
        ev_comp[i].record(comp)
        ev_out[i].record(comp)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(comp)
    for s in range(steps):
        i = s & 1
        h2d.wait_event(ev_comp[i])  # step s-2 no longer reads q_dev[i]
        with torch.cuda.stream(h2d):
            q_dev[i].copy_(q_host[i], non_blocking=True)
        ev_in[i].record(h2d)
        comp.wait_event(ev_in[i])
        comp.wait_event(ev_out[i])  # step s-2's result has left out_dev[i]
        G.gsa_decode(desc, q_dev[i], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                     out_dev[i], None, sel, ssc, ws)
        ev_comp[i].record(comp)
        d2h.wait_event(ev_comp[i])
        with torch.cuda.stream(d2h):
            out_host[i].copy_(out_dev[i], non_blocking=True)
        ev_out[i].record(d2h)
    for i in range(2):
        comp.wait_event(ev_out[i])  # every result is on the host
    t1.record(comp)
    t1.synchronize()
    return t0.elapsed_time(t1)


def decode_setup(G, W, cfg, dev, seed):
    x = W.decode_inputs(cfg, device=dev, seed=seed)
    B, hq, d = x["q"].shape
    n_max, t_max = x["gist_k"].shape[2], x["raw_k"].shape[2]
    dt = G.GSA_BF16 if cfg.dtype == "bf16" else G.GSA_F32
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, n_max, t_max, cfg.topk, cfg.exclude, 0.0, dt, G.GSA_F32)
    return x, desc


def measure_flat(G, W, cfg, dev, args, flush, seed, e2e=False, clock_index=None):
    x, desc = decode_setup(G, W, cfg, dev, seed)
    B, hq, d = x["q"].shape
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device=dev)
    ssc = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device=dev)
    scores = torch.empty((B, hq, x["gist_k"].shape[2]), dtype=torch.float32, device=dev)
    prior = G.GSA_PRIOR_NONE if cfg.exclude else G.GSA_PRIOR_GISTS

    def fused():
        G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                     out, None, sel, ssc, ws)

    def step_fused(evs):
        evs[0].record()
        fused()
        evs[1].record()

    def step_split(evs):
        """The fused step's kernels one call at a time: (bf16) scoring with
        the selection in its tail, then the unfold; (fp32) scoring,
        selection, unfold."""
        evs[0].record()
        if cfg.dtype == "bf16":
            G.gsa_score_select(desc, x["q"], x["gist_k"], None if cfg.exclude else x["gist_v"], x["n_gists"], scores,
                               sel, ssc, ws)
            evs[1].record()
        else:
            G.gsa_score_gists(desc, x["q"], x["gist_k"], None if cfg.exclude else x["gist_v"], x["n_gists"], scores,
                              ws)
            evs[1].record()
            G.gsa_topk_select(desc, scores, x["n_gists"], sel, ssc, ws)
        evs[2].record()
        G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"], sel, ssc,
                            prior, out, None, ws)
        evs[3].record()

    for _ in range(args.warmup):
        flush()
        fused()
    torch.cuda.synchronize()
    clk = ClockSampler(clock_index) if clock_index is not None else None
    if clk:
        clk.__enter__()
    step_ms = timed_steps(step_fused, args.steps, flush)[:, 0]
    if clk:
        clk.__exit__()
    kern_ms = timed_steps(step_split, args.steps, flush, 3)
    res = {"x": x, "sel": sel, "step_ms": step_ms, "kern_ms": kern_ms, "clocks": clk.summary() if clk else None,
           "ws": ws}
    if e2e:
        q_host = x["q"].cpu().pin_memory()
        out_host = torch.empty_like(out, device="cpu").pin_memory()

        def step_e2e(evs):
            evs[0].record()
            x["q"].copy_(q_host, non_blocking=True)
            fused()
            out_host.copy_(out, non_blocking=True)
            evs[1].record()

        res["e2e_seq_ms"] = timed_steps(step_e2e, args.steps, flush)[:, 0]
        res["e2e_pipe_ms"] = pipelined_e2e(G, x, desc, out, sel, ssc, ws, args.steps)
        res["h2d"] = int(x["q"].numel() * x["q"].element_size())
        res["d2h"] = int(out.numel() * out.element_size())
    assert G.gsa_workspace_status(ws) == 0, "device status flags set"
    return res


def flat_summary(cfg, m, hbm):
    ms = float(np.mean(m["step_ms"]))
    ab = algorithmic_bytes(cfg, m["x"], m["sel"])
    k = m["kern_ms"].mean(0)
    return {"metric": "GSA decode head-queries/s", "value": round(cfg.head_queries / (ms / 1e3), 1),
            "unit": UNIT, "ms_per_step": round(ms, 5),
            "step_hbm": {"alg_bytes": ab["total"], "achieved_gbs": round(ab["total"] / (ms / 1e3) / 1e9, 1),
                         "frac": round(ab["total"] / (ms / 1e3) / 1e9 / hbm, 4)},
            "kernels_us": kernel_times(cfg, k),
            "score_gists_gbs": round(score_kernel_bytes(cfg) / (k[0] / 1e3) / 1e9, 1),
            "unfold_gbs": round((ab["raw_union"] + ab["gist_sel"] + ab["own"] + ab["q_out"]) / (k[2] / 1e3) / 1e9, 1)}


def kernel_times(cfg, k):
    """Per-call event times (us) of the split step: bf16 runs two kernels
    (scoring + selection; unfold), fp32 three."""
    if cfg.dtype == "bf16":
        return {"score_select": round(float(k[0]) * 1e3, 2), "unfold_attend": round(float(k[2]) * 1e3, 2)}
    return {"score_gists": round(float(k[0]) * 1e3, 2), "topk_select": round(float(k[1]) * 1e3, 2),
            "unfold_attend": round(float(k[2]) * 1e3, 2)}


def measure_hgsa(G, W, cfg, dev, args, flush, hbm):
    x = W.decode_inputs(cfg, device=dev)
    B, hq, d = x["q"].shape
    hkv, n_max, t_max, m_max = x["gist_k"].shape[1], x["gist_k"].shape[2], x["raw_k"].shape[2], x["meta_k"].shape[2]
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, n_max, t_max, cfg.topk, cfg.exclude, 0.0, G.GSA_BF16, G.GSA_F32)
    hd = G.make_hdesc(cfg.group, cfg.topk_meta, m_max)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_HGSA, hd), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    mi = torch.empty((B, hq, cfg.topk_meta), dtype=torch.int32, device=dev)
    si = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device=dev)
    ss = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device=dev)

    def fused(evs=None):
        if evs:
            evs[0].record()
        G.hgsa_decode(desc, hd, x["q"], x["meta_k"], x["meta_v"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"],
                      x["n_gists"], x["own_len"], out, None, mi, si, ss, ws)
        if evs:
            evs[1].record()

    def split(evs):
        evs[0].record()
        G.hgsa_select(desc, hd, x["q"], x["meta_k"], x["meta_v"], x["gist_k"], x["gist_v"], x["n_gists"], mi, si, ss,
                      ws)
        evs[1].record()
        G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"], si, ss,
                            G.GSA_PRIOR_HGSA, out, None, ws)
        evs[2].record()

    for _ in range(args.warmup):
        flush()
        fused()
    step_ms = timed_steps(fused, args.steps, flush)[:, 0]
    k = timed_steps(split, args.steps, flush, 2).mean(0)
    assert G.gsa_workspace_status(ws) == 0
    # algorithmic bytes: meta K+V, K+V of the chosen groups' children (union per
    # (b, kv head)), raw K/V of the chosen chunks (union), own rows, q and out
    e, G_ = 2, hq // hkv
    M = cfg.n_gists // cfg.group
    meta = B * hkv * M * d * e * 2
    mic, sic = mi.reshape(B, hkv, G_, -1).cpu(), si.reshape(B, hkv, G_, -1).cpu()
    ug = sum(int((torch.unique(mic[b, kv]) >= 0).sum()) for b in range(B) for kv in range(hkv))
    uc = sum(int((torch.unique(sic[b, kv]) >= 0).sum()) for b in range(B) for kv in range(hkv))
    total = meta + ug * cfg.group * d * e * 2 + uc * cfg.chunk * d * e * 2 + B * hkv * d * e * 2 + B * hq * d * (e + 4)
    ms = float(np.mean(step_ms))
    return {"metric": "GSA decode head-queries/s", "value": round(cfg.head_queries / (ms / 1e3), 1), "unit": UNIT,
            "ms_per_step": round(ms, 5),
            "step_hbm": {"alg_bytes": total, "achieved_gbs": round(total / (ms / 1e3) / 1e9, 1),
                         "frac": round(total / (ms / 1e3) / 1e9 / hbm, 4)},
            "kernels_us": {"hgsa_select": round(float(k[0]) * 1e3, 2), "unfold_attend": round(float(k[1]) * 1e3, 2)}}


def measure_hgsa2(G, W, cfg, dev, args, flush, hbm):
    """H-GSA with two meta levels: the fused step (hgsa2_decode), the select
    and unfold halves, and the step's algorithmic bytes (all level-2
    meta-gists, the level-1 candidates under the chosen level-2 groups, the
    gist candidates under the chosen level-1 meta-gists -- unions per (b, kv
    head) -- the chosen chunks' raw rows, own rows, q and out)."""
    x = W.decode_inputs(cfg, device=dev)
    B, hq, d = x["q"].shape
    hkv, n_max, t_max = x["gist_k"].shape[1], x["gist_k"].shape[2], x["raw_k"].shape[2]
    m1_max, m2_max = x["meta_k"].shape[2], x["meta2_k"].shape[2]
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, n_max, t_max, cfg.topk, cfg.exclude, 0.0, G.GSA_BF16, G.GSA_F32)
    h2 = G.make_h2desc(G.make_hdesc(cfg.group, cfg.topk_meta, m1_max), G.make_hdesc(cfg.group2, cfg.topk_meta2, m2_max))
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_HGSA2, h2), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    m2 = torch.empty((B, hq, cfg.topk_meta2), dtype=torch.int32, device=dev)
    m1 = torch.empty((B, hq, cfg.topk_meta), dtype=torch.int32, device=dev)
    si = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device=dev)
    ss = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device=dev)
    args_ = (x["q"], x["meta2_k"], x["meta2_v"], x["meta_k"], x["meta_v"], x["gist_k"], x["gist_v"])

    def fused(evs=None):
        if evs:
            evs[0].record()
        G.hgsa2_decode(desc, h2, *args_, x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"], out, None, m2, m1, si,
                       ss, ws)
        if evs:
            evs[1].record()

    def split(evs):
        evs[0].record()
        G.hgsa2_select(desc, h2, *args_, x["n_gists"], m2, m1, si, ss, ws)
        evs[1].record()
        G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"], si, ss,
                            G.GSA_PRIOR_HGSA2, out, None, ws)
        evs[2].record()

    for _ in range(args.warmup):
        flush()
        fused()
    step_ms = timed_steps(fused, args.steps, flush)[:, 0]
    k = timed_steps(split, args.steps, flush, 2).mean(0)
    assert G.gsa_workspace_status(ws) == 0
    e, G_ = 2, hq // hkv
    M1 = cfg.n_gists // cfg.group
    M2 = M1 // cfg.group2

    def union(t):
        t = t.reshape(B, hkv, G_, -1).cpu()
        return sum(int((torch.unique(t[b, kv]) >= 0).sum()) for b in range(B) for kv in range(hkv))

    meta2 = B * hkv * M2 * d * e * 2
    u2, u1, u0 = union(m2), union(m1), union(si)
    trail1 = B * hkv * (M1 - M2 * cfg.group2)  # level-1 meta-gists of an incomplete level-2 group
    trail0 = B * hkv * (cfg.n_gists - M1 * cfg.group)
    total = (meta2 + (u2 * cfg.group2 + trail1) * d * e * 2 + (u1 * cfg.group + trail0) * d * e * 2
             + u0 * cfg.chunk * d * e * 2 + B * hkv * d * e * 2 + B * hq * d * (e + 4))
    one_level_meta = B * hkv * M1 * d * e * 2  # what scoring every level-1 meta-gist would read
    ms = float(np.mean(step_ms))
    return {"metric": "GSA decode head-queries/s", "value": round(cfg.head_queries / (ms / 1e3), 1), "unit": UNIT,
            "ms_per_step": round(ms, 5),
            "step_hbm": {"alg_bytes": total, "achieved_gbs": round(total / (ms / 1e3) / 1e9, 1),
                         "frac": round(total / (ms / 1e3) / 1e9 / hbm, 4)},
            "level_bytes": {"level2_meta": meta2, "level1_candidates": (u2 * cfg.group2 + trail1) * d * e * 2,
                            "gist_candidates": (u1 * cfg.group + trail0) * d * e * 2,
                            "one_level_meta_read_instead": one_level_meta},
            "kernels_us": {"hgsa2_select": round(float(k[0]) * 1e3, 2), "unfold_attend": round(float(k[1]) * 1e3, 2)}}


def measure_prefill(G, W, cfg, dev, args, flush, bf16_peak):
    x = W.prefill_inputs(cfg, device=dev)
    B, hq, L, d = x["q_raw"].shape
    hkv, N = x["k_raw"].shape[1], x["k_gist"].shape[2]
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, N, L, cfg.topk, cfg.exclude, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_PREFILL), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out_raw = torch.empty((B, hq, L, d), dtype=torch.float32, device=dev)
    out_gist = torch.empty((B, hq, N, d), dtype=torch.float32, device=dev)
    sel = torch.empty((B, hq, L, cfg.topk), dtype=torch.int32, device=dev)
    ssc = torch.empty((B, hq, L, cfg.topk), dtype=torch.float32, device=dev)

    def split(evs):
        evs[0].record()
        G.gsa_prefill_score(desc, x["q_raw"], x["q_gist"], x["k_gist"], sel, ssc, ws)
        evs[1].record()
        G.gsa_prefill_attend(desc, x["q_raw"], x["k_raw"], x["v_raw"], x["q_gist"], x["k_gist"], x["v_gist"], sel,
                             ssc, out_raw, out_gist, ws)
        evs[2].record()

    steps = max(3, min(args.steps, 10))
    for _ in range(max(1, min(args.warmup, 3))):
        flush()
        split([torch.cuda.Event(enable_timing=True) for _ in range(3)])
    k = timed_steps(split, steps, flush, 2).mean(0)
    assert G.gsa_workspace_status(ws) == 0
    # scoring FLOPs: raw position in chunk m scores m gists (2*d FLOP each)
    flops = B * hq * 2 * d * cfg.chunk * N * (N - 1) / 2
    tf = flops / (k[0] / 1e3) / 1e12
    tokens = B * (L + N)
    return {"metric": "GSA prefill scoring TFLOP/s", "value": round(tf, 1), "unit": "TFLOP/s",
            "scoring_ms": round(float(k[0]), 4), "attend_ms": round(float(k[1]), 4),
            "prefill_tokens_per_s": round(tokens / ((k[0] + k[1]) / 1e3), 1), "scoring_alg_flops": flops,
            "tensor_frac": round(tf / bf16_peak, 4), "steps": steps}


def measure_topp(G, W, cfg, dev, args, flush, hbm, top_p):
    """A decode step with top-p selection (score -> top-p -> unfold): the
    selection is variable-length, so the step's bytes follow the actual
    union of chosen chunks."""
    x, desc = decode_setup(G, W, cfg, dev, cfg.seed)
    B, hq, d = x["q"].shape
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device=dev)
    ssc = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device=dev)
    cnt = torch.empty((B, hq), dtype=torch.int32, device=dev)
    scores = torch.empty((B, hq, x["gist_k"].shape[2]), dtype=torch.float32, device=dev)

    def step(evs):
        evs[0].record()
        G.gsa_score_gists(desc, x["q"], x["gist_k"], x["gist_v"], x["n_gists"], scores, ws)
        evs[1].record()
        G.gsa_topp_select(desc, scores, x["n_gists"], top_p, sel, ssc, cnt, ws)
        evs[2].record()
        G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"], sel, ssc,
                            G.GSA_PRIOR_GISTS, out, None, ws)
        evs[3].record()

    for _ in range(args.warmup):
        flush()
        step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    k = timed_steps(step, args.steps, flush, 3)
    assert G.gsa_workspace_status(ws) == 0, "device status flags set"
    ms = float(k.sum(1).mean())
    ab = algorithmic_bytes(cfg, x, sel)
    c = cnt.float()
    return {"metric": "GSA decode head-queries/s", "value": round(cfg.head_queries / (ms / 1e3), 1), "unit": UNIT,
            "top_p": top_p, "ms_per_step": round(ms, 5),
            "chunks_selected": {"mean": round(float(c.mean()), 2), "min": int(c.min()), "max": int(c.max()),
                                "cap": cfg.topk},
            "step_hbm": {"alg_bytes": ab["total"], "achieved_gbs": round(ab["total"] / (ms / 1e3) / 1e9, 1),
                         "frac": round(ab["total"] / (ms / 1e3) / 1e9 / hbm, 4)},
            "kernels_us": {"score_gists": round(float(k[:, 0].mean()) * 1e3, 2),
                           "topp_select": round(float(k[:, 1].mean()) * 1e3, 2),
                           "unfold_attend": round(float(k[:, 2].mean()) * 1e3, 2)}}


def backward_bytes(cfg, x, sel):
    """Bytes the decode backward must move: every attended key / value row
    read once (bf16 or fp32) and its fp32 key / value gradient rows read and
    written once (the gradients accumulate), plus q, out, d_out, lse and the
    d_q read-modify-write per query head.  The attended rows per (b, kv head)
    are the gists (all, or the union of the selected ones with exclude), the
    union of the selected chunks' raw rows and the own rows."""
    e = 2 if cfg.dtype == "bf16" else 4
    B, hq, hkv, d, c = cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.chunk
    s = sel.reshape(B, hkv, hq // hkv, -1).cpu()
    union = sum(int((torch.unique(s[b, kv]) >= 0).sum()) for b in range(B) for kv in range(hkv))
    own = int(x["own_len"].sum()) * hkv
    rows = (union if cfg.exclude else B * hkv * cfg.n_gists) + union * c + own
    return rows * d * (2 * e + 2 * 4 * 2) + B * hq * d * (e + 4 + 4 + 2 * 4) + B * hq * 4


def measure_backward(G, W, cfg, dev, args, flush, hbm):
    """The backward of a decode step for the forward's selection
    (gsa_decode_backward alone; the forward runs once, untimed, to give the
    selection, output and lse).  The fp32 gradient buffers accumulate over
    the timed calls, as in gradient accumulation."""
    x, desc = decode_setup(G, W, cfg, dev, cfg.seed)
    B, hq, d = x["q"].shape
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    lse = torch.empty((B, hq), dtype=torch.float32, device=dev)
    sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device=dev)
    ssc = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device=dev)
    G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"], out, lse,
                 sel, ssc, ws)
    gen = torch.Generator(device=dev).manual_seed(cfg.seed + 7)
    d_out = torch.randn((B, hq, d), generator=gen, dtype=torch.float32, device=dev)
    grads = [torch.zeros((B, hq, d), dtype=torch.float32, device=dev)] + \
        [torch.zeros(x[k].shape, dtype=torch.float32, device=dev) for k in ("gist_k", "gist_v", "raw_k", "raw_v")]

    def step(evs):
        evs[0].record()
        G.gsa_decode_backward(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"],
                              x["own_len"], sel, out, lse, d_out, *grads)
        evs[1].record()

    for _ in range(args.warmup):
        flush()
        step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    k = timed_steps(step, args.steps, flush, 1)
    assert G.gsa_workspace_status(ws) == 0, "device status flags set"
    ms = float(k[:, 0].mean())
    ab = backward_bytes(cfg, x, sel)
    del grads
    return {"metric": "GSA decode backward head-queries/s", "value": round(cfg.head_queries / (ms / 1e3), 1),
            "unit": UNIT, "ms_per_step": round(ms, 5),
            "roofline": {"bound": "hbm", "alg_bytes": ab, "achieved_gbs": round(ab / (ms / 1e3) / 1e9, 1),
                         "peak_gbs": hbm, "frac": round(ab / (ms / 1e3) / 1e9 / hbm, 4)}}


def measure_gist_step(G, W, cfg, dev, args, flush, hbm):
    """The gist-position step at chunk completion (gsa_gist_step) for every
    sequence of the workload: append the new gist, attend gists 0..N and the
    completed chunk's raw rows, advance the counts.  The counts are put back
    before each step, outside the timed region."""
    x = W.gist_step_inputs(cfg, device=dev)
    B, hq, d = x["q"].shape
    n_max, t_max = x["gist_k"].shape[2], x["raw_k"].shape[2]
    dt = G.GSA_BF16 if cfg.dtype == "bf16" else G.GSA_F32
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, n_max, t_max, 0, False, 0.0, dt, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_GIST_STEP), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    n0, o0 = x["n_gists"].clone(), x["own_len"].clone()

    def step(evs):
        x["n_gists"].copy_(n0)
        x["own_len"].copy_(o0)
        evs[0].record()
        G.gsa_gist_step(desc, x["q"], x["k_new"], x["v_new"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"],
                        x["n_gists"], x["own_len"], out, None, ws)
        evs[1].record()

    for _ in range(args.warmup):
        flush()
        step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    k = timed_steps(step, args.steps, flush, 1)
    assert G.gsa_workspace_status(ws) == 0, "device status flags set"
    ms = float(k[:, 0].mean())
    e = 2 if cfg.dtype == "bf16" else 4
    # gists 0..N and the chunk's raw rows (key + value), the new gist read and
    # written, q in and fp32 out
    rows = int(n0.sum()) * cfg.hkv + B * cfg.hkv + int(o0.sum()) * cfg.hkv
    ab = rows * d * e * 2 + B * cfg.hkv * d * e * 2 * 2 + B * hq * d * (e + 4)
    return {"metric": "GSA gist-position steps (head-queries)/s", "value": round(cfg.head_queries / (ms / 1e3), 1),
            "unit": UNIT, "ms_per_step": round(ms, 5),
            "roofline": {"bound": "hbm", "alg_bytes": ab, "achieved_gbs": round(ab / (ms / 1e3) / 1e9, 1),
                         "peak_gbs": hbm, "frac": round(ab / (ms / 1e3) / 1e9 / hbm, 4)}}


def measure_multiquery(G, W, cfg, dev, args, flush, bf16):
    """Multi-query scoring against one shared gist cache (KV reuse): every
    query row of every head scores all N gists on the tensor cores and
    keeps its top k (gsa_multiquery_select)."""
    x = W.multiquery_inputs(cfg, device=dev)
    B, hq, Q, d = x["q"].shape
    desc = G.make_desc(B, hq, cfg.hkv, d, 1, cfg.n_gists, Q, cfg.topk, False, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_MULTIQUERY), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    sel = torch.empty((B, hq, Q, cfg.topk), dtype=torch.int32, device=dev)
    ssc = torch.empty((B, hq, Q, cfg.topk), dtype=torch.float32, device=dev)

    def step(evs):
        evs[0].record()
        G.gsa_multiquery_select(desc, x["q"], x["gist_k"], sel, ssc, ws)
        evs[1].record()

    for _ in range(args.warmup):
        flush()
        step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    k = timed_steps(step, args.steps, flush, 1)
    assert G.gsa_workspace_status(ws) == 0, "device status flags set"
    ms = float(k[:, 0].mean())
    tf = cfg.flops / (ms / 1e3) / 1e12
    return {"metric": "GSA multi-query routing queries/s", "value": round(B * hq * Q / (ms / 1e3), 1),
            "unit": "query-rows/s", "ms_per_step": round(ms, 5),
            "roofline": {"bound": "tensor", "flops": cfg.flops, "achieved_tflops": round(tf, 1), "peak_tflops": bf16,
                         "frac": round(tf / bf16, 4)}}


def rank_seed(cfg, rank):
    """Each rank draws its own batch of the workload (weak scaling: disjoint
    rows, no data-path exchange)."""
    return cfg.seed + 1000 * rank


def max_over_ranks(values, world, device):
    """Per-rank timed totals -> the maximum over ranks (the job's time)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def job_rate(units_per_rank_step, world, steps, total_ms):
    """Whole-job throughput: the units all ranks processed / the max-over-ranks time."""
    return units_per_rank_step * world * steps / (total_ms / 1e3)


def measure_extra(G, W, args, dev, flush, hbm, bf16):
    """The --extra workloads, each against its own roofline (rank 0, one GPU)."""
    extra = {}
    for name in [n for n in args.extra.split(",") if n]:
        if name.endswith("_giststep"):  # <decode workload>_giststep: chunk completion for every sequence
            extra[name] = measure_gist_step(G, W, W.CONFIGS[name[:-len("_giststep")]], dev, args, flush, hbm)
            torch.cuda.empty_cache()
            continue
        if name.endswith("_bwd"):  # <decode workload>_bwd: the backward of that decode step
            extra[name] = measure_backward(G, W, W.CONFIGS[name[:-len("_bwd")]], dev, args, flush, hbm)
            torch.cuda.empty_cache()
            continue
        if name.endswith("_topp"):  # <decode workload>_topp: the same step with top-p selection, p = 0.1
            # (the softmax over thousands of gists is flat: p = 0.1 keeps from a few chunks up to the cap)
            c = W.CONFIGS[name[:-len("_topp")]]
            extra[name] = measure_topp(G, W, c, dev, args, flush, hbm, 0.1)
            torch.cuda.empty_cache()
            continue
        c = W.CONFIGS[name]
        if name.startswith("kvreuse"):
            extra[name] = measure_multiquery(G, W, c, dev, args, flush, bf16)
            torch.cuda.empty_cache()
            continue
        if name.startswith("prefill"):
            extra[name] = measure_prefill(G, W, c, dev, args, flush, bf16)
        elif c.group2:
            extra[name] = measure_hgsa2(G, W, c, dev, args, flush, hbm)
        elif c.group:
            extra[name] = measure_hgsa(G, W, c, dev, args, flush, hbm)
        else:
            m = measure_flat(G, W, c, dev, args, flush, c.seed)
            extra[name] = flat_summary(c, m, hbm)
            del m
        torch.cuda.empty_cache()
    return extra


SWEEP_CONTEXTS = (131072, 524288, 2097152)


def sweep_config(context, levels):
    """The H-GSA workload shape (32 query / 8 kv heads, d = 128, chunks of 32,
    top-64) at one context length and batch 1: flat (levels 0), one meta
    level (16 gists per meta-gist, keep 32) or two (16 meta-gists per level-2
    meta-gist, keep 8)."""
    import long_context_gsa_b200.workloads as W
    kw = dict(group=16, topk_meta=32) if levels >= 1 else {}
    if levels == 2:
        kw.update(group2=16, topk_meta2=8)
    return W.DecodeConfig(f"hgsa_sweep_{context // 1024}k_l{levels}", 1, 32, 8, 128, 32, context, 64, "bf16",
                          seed=20260100 + levels, **kw)


def run_sweep(args):
    """How bytes and time per decode step grow with the context (the pages'
    O(log n) claim for H-GSA): flat GSA reads every gist key and value; one
    meta level reads every meta-gist and the chosen groups' children; two
    levels read every level-2 meta-gist, the chosen level-1 candidates and
    their gist children."""
    import long_context_gsa_b200 as G
    import long_context_gsa_b200.workloads as W
    G.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = Flusher(dev)
    hbm, _, _ = peaks()
    points = []
    for ctx in SWEEP_CONTEXTS:
        for levels in (0, 1, 2):
            cfg = sweep_config(ctx, levels)
            if levels == 0:
                m = measure_flat(G, W, cfg, dev, args, flush, cfg.seed)
                r = flat_summary(cfg, m, hbm)
                del m
            elif levels == 1:
                r = measure_hgsa(G, W, cfg, dev, args, flush, hbm)
            else:
                r = measure_hgsa2(G, W, cfg, dev, args, flush, hbm)
            torch.cuda.empty_cache()
            pt = {"sweep": "hgsa_levels", "context": ctx, "n_gists": cfg.n_gists, "meta_levels": levels,
                  "ms_per_step": r["ms_per_step"], "alg_bytes": r["step_hbm"]["alg_bytes"],
                  "hbm_frac": r["step_hbm"]["frac"], "head_queries_per_s": r["value"]}
            points.append(pt)
            print(json.dumps(pt), flush=True)
    summary = {"sweep": "hgsa_levels", "contexts": list(SWEEP_CONTEXTS), "points": len(points)}
    for levels in (0, 1, 2):
        ps = [p for p in points if p["meta_levels"] == levels]
        # growth per 4x context: bytes and time ratio between consecutive contexts
        summary[f"l{levels}_bytes_x4"] = [round(b["alg_bytes"] / a["alg_bytes"], 3) for a, b in zip(ps, ps[1:])]
        summary[f"l{levels}_time_x4"] = [round(b["ms_per_step"] / a["ms_per_step"], 3) for a, b in zip(ps, ps[1:])]
    print(json.dumps(summary), flush=True)


def run_gsa(args, world, rank, local):
    import long_context_gsa_b200 as G
    import long_context_gsa_b200.workloads as W

    G.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    cfg = W.CONFIGS[args.workload]
    flush = Flusher(dev)
    hbm, bf16, peak_kind = peaks()

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    barrier()
    if getattr(args, "extra_only", False) and world == 1:
        if rank == 0:
            print(json.dumps({"note": "extra workloads only", "workloads": measure_extra(G, W, args, dev, flush, hbm, bf16)}))
        return None
    main = measure_flat(G, W, cfg, dev, args, flush, rank_seed(cfg, rank), e2e=True, clock_index=local)
    barrier()
    total_ms, total_e2e_ms, total_seq_ms = max_over_ranks(
        [np.sum(main["step_ms"]), main["e2e_pipe_ms"], np.sum(main["e2e_seq_ms"])], world, dev)

    extra = {}
    if rank == 0 and world == 1 and not args.main_only:
        extra = measure_extra(G, W, args, dev, flush, hbm, bf16)

    result = None
    if rank == 0:
        s = flat_summary(cfg, main, hbm)
        value = job_rate(cfg.head_queries, world, args.steps, total_ms)
        k = main["kern_ms"].mean(0)
        ab = algorithmic_bytes(cfg, main["x"], main["sel"])
        if cfg.dtype == "bf16":  # two kernels: scoring + selection; unfold
            names = ["score_select", "unfold_attend"]
            k = np.array([k[0], k[2]])
            kbytes = [score_kernel_bytes(cfg), ab["raw_union"] + ab["gist_sel"] + ab["own"] + ab["q_out"]]
        else:
            names = ["score_gists", "topk_select", "unfold_attend"]
            kbytes = [score_kernel_bytes(cfg), 0, ab["raw_union"] + ab["gist_sel"] + ab["own"] + ab["q_out"]]
        dom = int(np.argmax(k))
        ach = kbytes[dom] / (k[dom] / 1e3) / 1e9 if kbytes[dom] else None
        rec = recorded_kernel(names[dom], cfg.name)
        roof = {"bound": "hbm", "kernel": names[dom], "achieved": round(ach, 1) if ach else None, "peak": hbm,
                "unit": "GB/s", "frac": round(ach / hbm, 4) if ach else None,
                "traffic": rec.get("bytes"), "peak_kind": peak_kind,
                "event_us": round(float(k[dom]) * 1e3, 2), "ncu_us": rec.get("duration_us")}
        # The other workloads come first and the headline's own figures last,
        # so a reader that keeps only the end of this long line keeps them.
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "batch_per_gpu": cfg.batch, "hq": cfg.hq, "hkv": cfg.hkv, "d": cfg.d,
                       "context": cfg.context, "chunk": cfg.chunk, "n_gists": cfg.n_gists, "topk": cfg.topk,
                       "exclude_unselected": cfg.exclude,
                       "l2": "flushed between timed steps (2x-L2 buffer written, then another 2x-L2 buffer read "
                             "so no dirty lines remain)",
                       "parallelism": f"dp{world} (independent rows per GPU)"},
            "gpu_launches": launches_per_step(cfg) * args.steps,
            "workloads": extra,
            "clocks": main["clocks"],
            "e2e": {"value": round(job_rate(cfg.head_queries, world, args.steps, total_seq_ms), 1), "unit": UNIT,
                    "h2d_bytes_per_step": main["h2d"], "d2h_bytes_per_step": main["d2h"],
                    "mode": "each step timed alone: its query copied in, the decode, its output copied out, in "
                            "sequence on one stream, L2 flushed between steps",
                    "pipelined_value": round(job_rate(cfg.head_queries, world, args.steps, total_e2e_ms), 1),
                    "pipelined_mode": "serving loop, steps back to back without L2 flushes: each step's query "
                                      "copied in on one stream while the previous step computes, its output copied "
                                      "out on another while the next computes"},
            "kernels_us": s["kernels_us"],
            "step_hbm": s["step_hbm"],
            "roofline": roof,
        }
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        xh = host_copy(main["x"])
        rate, calls, el, cores = oracle_rate(xh, cfg, cfg.head_queries, args.cpu_seconds)
        result["cpu_baseline"] = {"value": round(rate, 2), "unit": UNIT, "cores": cores, "kind": "oracle",
                                  "sample": f"{calls} full steps of {cfg.head_queries} head-queries ({el:.1f} s)"}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return result


def recorded_kernel(kernel, workload):
    """The committed ncu record of a kernel on a workload (DRAM bytes per
    launch, and its ncu duration when recorded), if it was taken on the
    current source of that kernel; otherwise an empty dict."""
    f = ROOT / "profiles" / "traffic.json"
    if not f.exists():
        return {}
    try:
        rec = json.loads(f.read_text()).get(f"{kernel}/{workload}")
    except ValueError:
        return {}
    if not rec:
        return {}
    import hashlib
    sources = rec["source"] if isinstance(rec["source"], list) else [rec["source"]]
    h = hashlib.sha256()
    for name in sources:  # every source file the kernel is built from
        src = ROOT / "long_context_gsa_b200" / "csrc" / name
        if not src.exists():
            return {}
        h.update(src.read_bytes())
    if h.hexdigest()[:16] != rec["sha"]:
        return {}
    return rec


def launches_per_step(cfg):
    """Kernels of this library one fused decode step launches (bf16: scoring,
    then selection + unfold; fp32: scoring, selection, unfold)."""
    if cfg.dtype == "bf16":
        return 2
    return 3 if cfg.topk > 0 else 2


# ---------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return None
    import long_context_gsa_b200.workloads as W
    cfg = W.CONFIGS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = W.decode_inputs(cfg, device=dev)
    xh = host_copy(x)
    del x
    rows_per_step = min(cfg.head_queries, 64)
    import oracle
    o = oracle.get()
    rows = np.arange(rows_per_step)

    def one():
        o.decode(xh["q"], xh["gist_k"], xh["gist_v"], xh["raw_k"], xh["raw_v"], xh["n_gists"], xh["own_len"],
                 chunk=cfg.chunk, topk=cfg.topk, exclude=cfg.exclude, rows=rows)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    value = args.steps * rows_per_step / el
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "batch_per_gpu": cfg.batch, "hq": cfg.hq, "hkv": cfg.hkv, "d": cfg.d,
                   "context": cfg.context, "chunk": cfg.chunk, "topk": cfg.topk},
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": o.default_threads(), "kind": "oracle",
                         "sample": f"each step = {rows_per_step} of the {cfg.head_queries} head-queries"},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world, rank, local = dist_env()
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        res = run_reference(args, world, rank)
    else:
        res = run_gsa(args, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
