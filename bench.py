"""Benchmark: generated tokens/s of Block Transformer inference on B200.

One step = the two runs of the Pythia-160M-scale Block Transformer workload
(d_model 768, 12 heads, V 50304, L_B 4, 6 + 6 layers, prefix 1, bf16,
random-init weights, Zipf(1.1) token ids), on one model instance:
  prefill-heavy  batch 64, prompt 2048, 128 generated tokens;
  decode-heavy   batch 64, prompt 128, 2048 generated tokens.
Each run is a prefill plus greedy decode steps through the C-ABI (G tokens
generated per sequence = 1 prefill + G - 1 decode calls). value = generated
tokens of both runs / their device time, summed over ranks (replicas).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). --impl reference times the CPU oracle on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

RUNS = ("pythia160m_prefill_heavy", "pythia160m_decode_heavy")
METRIC = "generated tokens/s at 1 B200 (prefill- & decode-heavy); % HBM roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def allreduce_max(values, device: str = "cuda"):
    """Element-wise max of per-rank timings over all ranks (identity when
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank generates the same tokens per step;
    the job lasts as long as the slowest rank."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


def build(rank: int):
    import torch
    from hierarchical_global_local_b200.loader import build_model
    wl = synth.WORKLOADS[RUNS[0]]
    w = synth.make_weights(wl)
    max_seq = max(synth.WORKLOADS[r].max_seq for r in RUNS)
    B = max(synth.WORKLOADS[r].batch for r in RUNS)
    model = build_model(wl.shape, w, B, max_seq)
    prompts = {}
    for r in RUNS:
        x = synth.WORKLOADS[r]
        toks = synth.make_tokens(x, seed=x.token_seed + 100 * rank)
        prompts[r] = torch.from_numpy(np.ascontiguousarray(toks[:, :x.prompt_len])).cuda()
    return model, prompts


def generate(model, prompt, G, out):
    """Prefill + G - 1 greedy decode calls; generated ids land in out [G, B]."""
    model.prefill(prompt, next_tokens=out[0])
    for i in range(1, G):
        model.decode(None, next_tokens=out[i])


def run_ours(args):
    import torch
    import torch.distributed as dist
    from hierarchical_global_local_b200 import costmodel as cm
    from hierarchical_global_local_b200 import native

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    model, prompts = build(rank)
    gens = {r: torch.empty(synth.WORKLOADS[r].gen_len, synth.WORKLOADS[r].batch,
                           dtype=torch.int32, device="cuda") for r in RUNS}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def barrier():
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def one_step(times):
        for r in RUNS:
            x = synth.WORKLOADS[r]
            flush.fill_(rank & 0xFF)          # L2 flush between timed runs (untimed)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            generate(model, prompts[r], x.gen_len, gens[r])
            b.record(stream)
            times.append((r, a, b))

    for _ in range(args.warmup):
        one_step([])
    model.sync()
    k0 = native.lib().bt_kernel_launches(model._h)
    times = []
    barrier()
    with ClockSampler(local) as clk:
        torch.cuda.nvtx.range_push("timed")      # ncu --nvtx-include timed/
        for _ in range(args.steps):
            one_step(times)
        barrier()
        torch.cuda.nvtx.range_pop()
    k1 = native.lib().bt_kernel_launches(model._h)
    model.sync()
    per_run = {r: 0.0 for r in RUNS}
    for r, a, b in times:
        per_run[r] += a.elapsed_time(b)
    total_ms = sum(per_run.values())
    tmax = allreduce_max([total_ms] + [per_run[r] for r in RUNS])
    total_ms = tmax[0]
    per_run_max = {r: tmax[1 + i] for i, r in enumerate(RUNS)}
    tokens_per_step = sum(synth.WORKLOADS[r].batch * synth.WORKLOADS[r].gen_len for r in RUNS)
    value = job_throughput(tokens_per_step, args.steps, ws, total_ms)

    # ---- end to end through the public API, host buffers -------------------
    e2e = None
    if not args.no_e2e:
        host_prompts = {r: prompts[r].cpu().pin_memory() for r in RUNS}
        host_out = {r: torch.empty_like(gens[r], device="cpu").pin_memory() for r in RUNS}
        dev_prompts = {r: torch.empty_like(prompts[r]) for r in RUNS}
        e_times = []
        barrier()
        for _ in range(args.steps):
            for r in RUNS:
                x = synth.WORKLOADS[r]
                flush.fill_(1)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                dev_prompts[r].copy_(host_prompts[r], non_blocking=True)
                generate(model, dev_prompts[r], x.gen_len, gens[r])
                host_out[r].copy_(gens[r], non_blocking=True)
                b.record(stream)
                e_times.append((a, b))
        barrier()
        e_ms = allreduce_max([sum(a.elapsed_time(b) for a, b in e_times)])[0]
        h2d = sum(int(prompts[r].numel()) * 4 for r in RUNS)
        d2h = sum(int(gens[r].numel()) * 4 for r in RUNS)
        e2e = {"value": job_throughput(tokens_per_step, args.steps, ws, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # ---- profiled pass: event pair around every kernel of one step ---------
    hbm, tf_burst, tf_sus, peak_src = _peaks()
    prof = profile_step(model, prompts, gens, flush) if not args.no_profile else None

    # ---- bytes / FLOPs roofline of the whole generate runs ------------------
    s = cm.Shape.of(synth.WORKLOADS[RUNS[0]].shape)
    roof = {}
    for r in RUNS:
        x = synth.WORKLOADS[r]
        g = cm.generate(s, x.batch, x.prompt_len, x.gen_len)
        t_roof = g.roofline_seconds(hbm, tf_sus)
        t_meas = per_run_max[r] / args.steps / 1e3
        roof[r] = {"ms": per_run_max[r] / args.steps, "tokens_per_s": ws * x.batch * x.gen_len / t_meas,
                   "roofline_ms": t_roof * 1e3, "frac_of_roofline": t_roof / t_meas,
                   "decode_bytes_per_step_GB": g.decode.bytes / 1e9,
                   "prefill_tflop": g.prefill.flops / 1e12}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "pythia160m-scale Block Transformer L_B=4 6+6 layers P=1: "
                               "prefill-heavy B64 2048/128 + decode-heavy B64 128/2048",
                   "global_batch": 64 * ws, "seq_len": 2176, "parallelism": f"replicas{ws}",
                   "l2": "flushed (256 MiB write) before each timed run; weights + KV > L2",
                   "tokens": "Zipf(1.1) ids, greedy generation"},
        "runs": roof,
        "gpu_launches": int(k1 - k0),
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if prof:
        line["roofline"] = prof["dominant"]
        line["roofline_decode_attention"] = prof.get("attn_decode")
        line["roofline_decode_attention_n300"] = prof.get("attn_decode_n300")
        if line["roofline_decode_attention_n300"] is not None and ws == 1:
            line["roofline_decode_attention_n300"]["graph_replay"] = decode_attention_replay(hbm)
        line["roofline_decode_gemm"] = prof.get("gemm_decode")
        line["kernel_time_shares"] = prof["shares"]
        line["roofline"]["peak_source"] = peak_src
    if ws == 1 and not args.no_extra:
        with ClockSampler(local) as clk_x:
            line["runs_extra"] = run_extras(flush, hbm, tf_sus)
            line["runs_extra"]["batch_sweep"] = run_batch_sweep(flush, hbm, tf_sus, cap=args.max_batch_cap)
        line["runs_extra"]["clocks"] = clk_x.summary()
        line["runs_extra"]["note"] = ("timed once each after an untimed run, outside value; the pages "
                                      "report 10-20x Block Transformer throughput over vanilla models of "
                                      "equal perplexity on H100 (context only: different sizes, trained "
                                      "weights)")
    if rank == 0 and ws == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    if ws > 1:
        dist.barrier()
    if rank == 0:
        print(json.dumps(line), flush=True)
    model.close()
    if ws > 1:
        dist.destroy_process_group()


# DRAM bytes (read + write) per launch of a kernel class on this workload,
# measured by an ncu capture, with the SHA-256 prefix of the kernel's source
# file at the time of the capture. The bench reports the figure only while
# the source is unchanged; after a change the traffic is null until it is
# captured again.
NCU_TRAFFIC = {
    "token_step": {"bytes": 171.34e6, "source": "hierarchical_global_local_b200/csrc/decode_step.cu",
                   "sha16": "88745d49660d9d00"},
}


def ncu_traffic(kind: str):
    """Measured DRAM bytes per launch of `kind`, or None when there is no
    capture of the current kernel source."""
    import hashlib
    e = NCU_TRAFFIC.get(kind)
    if not e:
        return None
    try:
        with open(os.path.join(ROOT, e["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return e["bytes"] if sha == e["sha16"] else None


def decode_attention_replay(hbm: float, ns=(300, 420, 545)):
    """The block decoder's decode attention alone at the decode-heavy
    workload's shapes (B 64, H 12, d_head 64, bf16, cache capacity 576):
    32 launches per n, captured in one CUDA graph, cycling through 8 K/V
    sets (8 x 113 MB, past L2) so that every launch reads its cache from
    HBM; CUDA events around the replays. Unlike the in-model figure (an
    event pair around every launch, which also times each launch's start
    without the overlap programmatic dependent launch gives inside the
    decode graphs) this is the kernel's duration in a launch sequence."""
    import torch
    from hierarchical_global_local_b200 import native
    shape = synth.WORKLOADS["pythia160m_decode_heavy"].shape
    B, H, d, cap, R = 64, shape.n_heads, shape.d_model // shape.n_heads, 576, 8
    g = torch.Generator(device="cuda").manual_seed(3)
    qs = [torch.randn(B, H * d, device="cuda", generator=g).bfloat16() for _ in range(R)]
    ks = [torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16() for _ in range(R)]
    vs = [torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16() for _ in range(R)]
    out = torch.empty(B, H * d, device="cuda", dtype=torch.bfloat16)
    scr = native.decode_attention_scratch(native.BT_BF16, B, H, d, cap)
    st = torch.cuda.Stream()
    res, tot_b, tot_us = {}, 0.0, 0.0
    with torch.cuda.stream(st):
        for n in ns:
            for i in range(R):
                native.decode_attention(qs[i], ks[i], vs[i], n, out=out, scratch=scr)
            st.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=st):
                for _ in range(4):
                    for i in range(R):
                        native.decode_attention(qs[i], ks[i], vs[i], n, out=out, scratch=scr)
            for _ in range(3):
                gr.replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            st.synchronize()
            a.record(st)
            for _ in range(5):
                gr.replay()
            b.record(st)
            st.synchronize()
            us = a.elapsed_time(b) * 1e3 / (5 * 4 * R)
            by = B * H * (2.0 * n * d * 2 + 2.0 * d * 2)
            res[str(n)] = {"us": us, "GB/s": by / us / 1e3, "frac": by / us / 1e3 / hbm}
            tot_b += by
            tot_us += us
            del gr
    ach = tot_b / tot_us / 1e3
    del qs, ks, vs
    torch.cuda.empty_cache()
    return {"kernel": "attn_decode", "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
            "frac": ach / hbm, "per_n": res,
            "case": f"B {B} H {H} d {d} bf16, n {list(ns)}, 8 K/V sets past L2, CUDA-graph replay"}


def profile_step(model, prompts, gens, flush):
    """One step with an event pair around every kernel; per-kind time shares
    and the roofline of the dominant kernel class."""
    import torch
    from hierarchical_global_local_b200 import native
    L = native.lib()
    cap = 400000
    _check = native._check
    _check(L.bt_profile_begin(model._h, cap), "bt_profile_begin")
    for r in RUNS:
        flush.fill_(2)
        generate(model, prompts[r], synth.WORKLOADS[r].gen_len, gens[r])
    recs = (native_record() * cap)()
    n = native.ctypes.c_int32()
    _check(L.bt_profile_end(model._h, native.ctypes.cast(recs, native.ctypes.c_void_p), cap,
                           native.ctypes.byref(n)), "bt_profile_end")
    hbm, tf_burst, tf_sus, _ = _peaks()
    kinds = {0: "gemm", 1: "attn_decode", 2: "attn_prefill", 3: "attn_local", 4: "layernorm",
             5: "rope_append", 6: "embed", 7: "argmax", 8: "other", 9: "token_step", 10: "block_step"}
    shape0 = synth.WORKLOADS[RUNS[0]].shape
    D = shape0.d_model
    Nt = shape0.n_token_layers if shape0.use_token_decoder else 0
    Nb = shape0.n_block_layers
    cls = {}
    for i in range(n.value):
        rc = recs[i]
        k = kinds.get(rc.kind, "other")
        if k == "gemm":
            k = "gemm_decode" if rc.m <= 256 else "gemm_prefill"
        c = cls.setdefault(k, {"ms": 0.0, "launches": 0, "bytes": 0.0, "flops": 0.0})
        c["ms"] += rc.ms
        c["launches"] += 1
        if k.startswith("gemm"):
            # output: bf16 q|k|v|GELU(fc1); fp32 residual read + write; fp32 logits / prefix rows
            out_b = 2 if rc.n == 7 * D else (8 if rc.k == 5 * D else 4)
            c["bytes"] += 2.0 * (rc.n * rc.k + rc.m * rc.k) + out_b * rc.m * rc.n
            c["flops"] += 2.0 * rc.m * rc.n * rc.k
        elif k == "attn_decode":
            c["bytes"] += rc.m * (2.0 * rc.n * rc.k * 2 + 2.0 * rc.k * 2)
            if rc.n >= 300:
                # launches over caches of >= 300 entries, on their own
                cl = cls.setdefault("attn_decode_n300", {"ms": 0.0, "launches": 0, "bytes": 0.0, "flops": 0.0})
                cl["ms"] += rc.ms
                cl["launches"] += 1
                cl["bytes"] += rc.m * (2.0 * rc.n * rc.k * 2 + 2.0 * rc.k * 2)
        elif k == "block_step":
            # block-decoder, prefix, token-decoder and LM-head weights (the
            # block KV read is not in the record and is left out)
            c["bytes"] += 2.0 * ((Nb + Nt) * 12 * rc.k * rc.k + rc.k * rc.k + rc.n * rc.k)
            c["flops"] += 2.0 * rc.m * ((Nb + Nt) * 12 * rc.k * rc.k + rc.k * rc.k + rc.n * rc.k)
        elif k == "token_step":
            # every token-decoder weight (q|k|v|fc1 and o|fc2: 12 D^2 per layer)
            # and the LM head, once per launch; activations stay in L2
            c["bytes"] += 2.0 * (Nt * 12 * rc.k * rc.k + rc.n * rc.k)
            c["flops"] += 2.0 * rc.m * (Nt * 12 * rc.k * rc.k + rc.n * rc.k)
    long_attn = cls.pop("attn_decode_n300", None)
    total = sum(c["ms"] for c in cls.values())
    shares = {k: round(c["ms"] / total, 4) for k, c in sorted(cls.items(), key=lambda kv: -kv[1]["ms"])}
    dom_name = max(cls, key=lambda k: cls[k]["ms"])

    def roof(k):
        c = cls[k]
        per = c["ms"] / c["launches"] / 1e3
        if k == "gemm_prefill":
            ach = c["flops"] / c["launches"] / per / 1e12
            return {"kernel": k, "bound": "tensor", "achieved": ach, "peak": tf_sus, "unit": "TFLOP/s",
                    "frac": ach / tf_sus, "traffic": None, "launches": c["launches"],
                    "avg_launch_us": per * 1e6}
        ach = c["bytes"] / c["launches"] / per / 1e9
        return {"kernel": k, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                "frac": ach / hbm, "traffic": ncu_traffic(k), "launches": c["launches"],
                "avg_launch_us": per * 1e6}

    out = {"dominant": roof(dom_name) if dom_name in ("gemm_decode", "gemm_prefill", "attn_decode", "token_step",
                                                     "block_step")
           else {"kernel": dom_name, "bound": "hbm", "achieved": None, "peak": hbm, "unit": "GB/s",
                 "frac": None, "traffic": None},
           "shares": shares}
    if "attn_decode" in cls:
        out["attn_decode"] = roof("attn_decode")
    if long_attn is not None:
        cls["attn_decode_n300"] = long_attn
        out["attn_decode_n300"] = roof("attn_decode_n300")
    if "gemm_decode" in cls:
        out["gemm_decode"] = roof("gemm_decode")
    return out


EXTRA_RUNS = (
    # (key, workload, what it is)
    ("vanilla_lb1", "lb_sweep_L1", "vanilla 24-layer model (L_B = 1, no token decoder), same kernels"),
    ("lb2", "lb_sweep_L2", "L_B = 2, 12 + 12 layers"),
    ("lb4", "lb_sweep_L4", "L_B = 4, 12 + 12 layers"),
    ("lb8", "lb_sweep_L8", "L_B = 8, 12 + 12 layers"),
    ("pythia410m_decode_heavy", "pythia410m_decode_heavy", "pythia410m-scale, B 256, prompt 128, 2048 generated"),
    ("long_context", "long_context", "d_model 2048, d_head 128, B 32, prompt 8192, 512 generated"),
)


def run_extras(flush, hbm: float, tf_sus: float):
    """The other workloads of the method's evaluation, each timed once after
    one untimed run (graph capture), outside the benchmark's timed value:
    the L_B sweep with the vanilla L_B = 1 model built from the same kernels,
    the pythia410m-scale decode-heavy run and the long-context run. Greedy
    generation through the C-ABI; L2 flushed before each timed run."""
    import torch
    from hierarchical_global_local_b200 import costmodel as cm
    from hierarchical_global_local_b200.loader import build_model
    out = {}
    stream = torch.cuda.current_stream()
    for key, name, what in EXTRA_RUNS:
        wl = synth.WORKLOADS[name]
        t_build = time.perf_counter()
        model = build_model(wl.shape, synth.make_weights(wl), wl.batch, wl.max_seq)
        toks = synth.make_tokens(wl)
        prompt = torch.from_numpy(np.ascontiguousarray(toks[:, :wl.prompt_len])).cuda()
        gen = torch.empty(wl.gen_len, wl.batch, dtype=torch.int32, device="cuda")
        generate(model, prompt, wl.gen_len, gen)
        model.sync()
        flush.fill_(3)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        generate(model, prompt, wl.gen_len, gen)
        b.record(stream)
        model.sync()
        ms = a.elapsed_time(b)
        g = cm.generate(cm.Shape.of(wl.shape), wl.batch, wl.prompt_len, wl.gen_len)
        t_roof = g.roofline_seconds(hbm, tf_sus)
        out[key] = {"workload": what, "batch": wl.batch, "prompt": wl.prompt_len, "generated": wl.gen_len,
                    "ms": ms, "tokens_per_s": wl.batch * wl.gen_len / (ms / 1e3),
                    "roofline_ms": t_roof * 1e3, "frac_of_roofline": t_roof / (ms / 1e3),
                    "wall_s_incl_build": time.perf_counter() - t_build}
        model.close()
        del model, prompt, gen
        torch.cuda.empty_cache()
    if "vanilla_lb1" in out:
        v = out["vanilla_lb1"]["tokens_per_s"]
        for k in ("lb2", "lb4", "lb8"):
            if k in out:
                out[k]["vs_vanilla"] = out[k]["tokens_per_s"] / v
    return out


SWEEP_RUNS = ("pythia160m_prefill_heavy", "pythia160m_decode_heavy")
SWEEP_BATCHES = (1, 32, 256)
SWEEP_MEMORY_FRACTION = 0.85  # of the device memory free when the sweep starts


def run_batch_sweep(flush, hbm: float, tf_sus: float, cap: int = 0):
    """Batch-size sensitivity and the maximum-throughput setting of the
    method's evaluation: the pythia160m-scale prefill-heavy and decode-heavy
    runs at batch 1, 32, 256 and the largest batch the device holds (every
    model at its own memory-maximising batch, FlexGen's "maximum throughput"),
    each timed once after an untimed run, plus memory per sample of the
    Block Transformer against the vanilla L_B = 1 model. The largest batch is
    the planner's (loader.max_batch_by_memory) for SWEEP_MEMORY_FRACTION of
    the free device memory; cap > 0 bounds it."""
    import torch
    from hierarchical_global_local_b200 import costmodel as cm
    from hierarchical_global_local_b200 import loader
    stream = torch.cuda.current_stream()
    free, total = torch.cuda.mem_get_info()
    budget = int(free * SWEEP_MEMORY_FRACTION)
    wl0 = synth.WORKLOADS[SWEEP_RUNS[0]]
    shape, max_seq = wl0.shape, max(synth.WORKLOADS[r].max_seq for r in SWEEP_RUNS)
    per_sample = loader.memory_per_sample(shape, max_seq)
    ws1 = loader.workspace_bytes(shape, 1, max_seq)
    b_mem = int((budget - ws1) // per_sample) + 1 if budget > ws1 else 0
    b_max = loader.max_batch_by_memory(shape, max_seq, budget)
    if cap > 0:
        b_max = min(b_max, cap)
    batches = sorted({b for b in SWEEP_BATCHES if b <= b_max} | {b_max})
    out = {"budget_GB": budget / 1e9, "device_total_GB": total / 1e9,
           "memory_per_sample_MB": per_sample / 1e6,
           "max_batch_by_memory": b_mem,
           "max_batch_run": b_max,
           "max_batch_bound": "memory" if b_max >= b_mem else
                              ("cap" if cap > 0 and b_max == cap else
                               "32-bit buffer indexing (bt_config.max_batch)"),
           "runs": {}}
    model = loader.build_model(shape, synth.make_weights(wl0), b_max, max_seq)
    for r in SWEEP_RUNS:
        wl = synth.WORKLOADS[r]
        toks = synth.make_tokens(wl, batch=b_max)
        res = {}
        for bs in batches:
            prompt = torch.from_numpy(np.ascontiguousarray(toks[:bs, :wl.prompt_len])).cuda()
            gen = torch.empty(wl.gen_len, bs, dtype=torch.int32, device="cuda")
            generate(model, prompt, wl.gen_len, gen)
            model.sync()
            flush.fill_(4)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            generate(model, prompt, wl.gen_len, gen)
            b.record(stream)
            model.sync()
            ms = a.elapsed_time(b)
            t_roof = cm.generate(cm.Shape.of(shape), bs, wl.prompt_len, wl.gen_len).roofline_seconds(hbm, tf_sus)
            res[str(bs)] = {"ms": ms, "tokens_per_s": bs * wl.gen_len / (ms / 1e3),
                            "roofline_ms": t_roof * 1e3, "frac_of_roofline": t_roof / (ms / 1e3)}
            del prompt, gen
        out["runs"][r] = res
    model.close()
    del model
    torch.cuda.empty_cache()
    # memory per sample across L_B at equal width and depth (the L_B sweep
    # family, prompt 2,048 + 512 generated): L_B = 1 is the vanilla model
    mem = {}
    for lb in (1, 2, 4, 8):
        w = synth.WORKLOADS[f"lb_sweep_L{lb}"]
        mem[f"L_B={lb}"] = loader.memory_per_sample(w.shape, w.max_seq) / 1e6
    out["lb_sweep_memory_per_sample_MB"] = mem
    out["vanilla_over_lb4_memory_per_sample"] = mem["L_B=1"] / mem["L_B=4"]
    return out


def native_record():
    from hierarchical_global_local_b200 import native
    import ctypes

    class Rec(ctypes.Structure):
        _fields_ = [("kind", ctypes.c_int32), ("m", ctypes.c_int32), ("n", ctypes.c_int32),
                    ("k", ctypes.c_int32), ("ms", ctypes.c_float)]
    return Rec


# --------------------------------------------------------------------------
# oracle on the host cores (baseline / reference arm)
# --------------------------------------------------------------------------

def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(budget_s: float = 20.0):
    """The oracle (fp64 numpy), as it stands, on a bounded sample of the same
    workload: 1 sequence of each run, the full prompt, and as many generated
    tokens as fit in the time budget (split between the runs)."""
    from oracle.model import BlockTransformerOracle
    wl = synth.WORKLOADS[RUNS[0]]
    w = synth.make_weights(wl)
    params = {n: w.values(n) for n in w.names()}
    o = BlockTransformerOracle(wl.shape, params)
    gen_total, t_total, parts = 0, 0.0, []
    for r in RUNS:
        x = synth.WORKLOADS[r]
        toks = synth.make_tokens(x, batch=1)
        sess = o.session()
        t0 = time.perf_counter()
        z = sess.prefill(toks[:, :x.prompt_len])
        g = 1
        while g < x.gen_len and time.perf_counter() - t0 < budget_s / len(RUNS):
            z = sess.decode(z.argmax(-1))
            g += 1
        dt = time.perf_counter() - t0
        gen_total += g
        t_total += dt
        parts.append(f"{r}: 1 sequence, prompt {x.prompt_len}, {g} of {x.gen_len} tokens, {dt:.1f}s")
    return {"value": gen_total / t_total, "unit": UNIT, "cores": _threads(), "kind": "oracle",
            "sample": "; ".join(parts), "seconds": t_total}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    # each step: a bounded sample of the workload (--ref-seconds over all steps)
    per_step = []
    budget = max(2.0, args.ref_seconds / max(1, args.warmup + args.steps))
    for _ in range(args.warmup + args.steps):
        per_step.append(cpu_baseline(budget_s=budget))
    timed = per_step[args.warmup:]
    v = statistics.mean(s["value"] for s in timed)
    ms = 1e3 * statistics.mean(s["seconds"] for s in timed)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "pythia160m-scale Block Transformer L_B=4 6+6 layers P=1: "
                                   "prefill-heavy B64 2048/128 + decode-heavy B64 128/2048",
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": timed[0]["cores"], "kind": "oracle",
                             "sample": timed[0]["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_decode_case(args):
    """A bounded decode-only case for profiler captures: the decode-heavy
    model and batch, its 128-token prompt, then --case-steps greedy decode
    calls (every L_B-th a block step). Prints the mean ms per decode call."""
    import torch
    torch.cuda.set_device(0)
    model, prompts = build(0)
    r = RUNS[1]
    x = synth.WORKLOADS[r]
    out = torch.empty(args.case_steps + 1, x.batch, dtype=torch.int32, device="cuda")
    model.prefill(prompts[r], next_tokens=out[0])
    model.sync()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(1, args.case_steps + 1):
        model.decode(None, next_tokens=out[i])
    b.record()
    model.sync()
    print(json.dumps({"case": "decode", "workload": r, "steps": args.case_steps,
                      "ms_per_decode_call": a.elapsed_time(b) / args.case_steps}), flush=True)
    model.close()


def run_variants_case(args):
    """A bounded case for profiler captures of the context-injection variants'
    kernels: pythia160m-scale models with summation injection and with a
    window of w = 3 context embeddings, batch 64, a 130-token prompt (two
    trailing tokens inside the current block), then --case-steps greedy
    decode calls each."""
    import dataclasses
    import torch
    from hierarchical_global_local_b200.loader import build_model
    torch.cuda.set_device(0)
    base = synth.WORKLOADS[RUNS[1]]
    for variant in ({"injection": "sum"}, {"context_window": 3}):
        shape = dataclasses.replace(base.shape, **variant)
        T = 130
        model = build_model(shape, synth.make_weights(shape, seed=base.weight_seed), base.batch,
                            T + args.case_steps + 1)
        toks = synth.make_tokens(base, length=T)
        out = torch.empty(args.case_steps + 1, base.batch, dtype=torch.int32, device="cuda")
        model.prefill(torch.from_numpy(np.ascontiguousarray(toks)).cuda(), next_tokens=out[0])
        for i in range(1, args.case_steps + 1):
            model.decode(None, next_tokens=out[i])
        model.sync()
        model.close()
        print(json.dumps({"case": "variants", "variant": variant, "prompt": T, "decode_calls": args.case_steps}),
              flush=True)


def run_prefill_case(args):
    """A bounded prefill-only case for profiler captures: --case-steps
    prefills of the prefill-heavy run (batch 64, prompt 2048)."""
    import torch
    torch.cuda.set_device(0)
    model, prompts = build(0)
    r = RUNS[0]
    x = synth.WORKLOADS[r]
    nxt = torch.empty(x.batch, dtype=torch.int32, device="cuda")
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.case_steps):
        model.prefill(prompts[r], next_tokens=nxt)
    b.record()
    model.sync()
    print(json.dumps({"case": "prefill", "workload": r, "calls": args.case_steps,
                      "ms_per_prefill": a.elapsed_time(b) / args.case_steps}), flush=True)
    model.close()


def run_lb_sweep(args):
    """The L_B sweep configurations (d_model 1024, 16 heads, 12 + 12 layers,
    batch 128, prompt 2,048, 512 generated; L_B = 1 is the vanilla 24-layer
    model without a token decoder, built from the same kernels): one untimed
    generate run (graph capture), then one timed run each. One JSON line per
    configuration; --case-steps > 0 shortens the generated length."""
    import torch
    from hierarchical_global_local_b200.loader import build_model
    torch.cuda.set_device(0)
    for lb in (1, 2, 4, 8):
        wl = synth.WORKLOADS[f"lb_sweep_L{lb}"]
        model = build_model(wl.shape, synth.make_weights(wl), wl.batch, wl.max_seq)
        toks = synth.make_tokens(wl)
        prompt = torch.from_numpy(np.ascontiguousarray(toks[:, :wl.prompt_len])).cuda()
        G = min(args.case_steps, wl.gen_len) if args.case_steps > 0 else wl.gen_len
        out = torch.empty(G, wl.batch, dtype=torch.int32, device="cuda")
        generate(model, prompt, G, out)
        model.sync()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        generate(model, prompt, G, out)
        b.record()
        model.sync()
        ms = a.elapsed_time(b)
        print(json.dumps({"case": "lb_sweep", "workload": wl.name, "block_len": lb,
                          "vanilla": not wl.shape.use_token_decoder, "batch": wl.batch,
                          "prompt": wl.prompt_len, "generated": G, "ms": ms,
                          "tokens_per_s": wl.batch * G / (ms / 1e3)}), flush=True)
        model.close()
        del model
        torch.cuda.empty_cache()


def run_kernel_case(args):
    """One op of the path through the op-level C-ABI, a few launches, for
    profiler captures: decode attention (B, H, d, n), the tensor-core
    prefill attention (B, H, d, n: causal over n block rows per sequence) or
    a dense projection (M, N, K) on the tensor-core path."""
    import torch
    from hierarchical_global_local_b200 import native
    torch.cuda.set_device(0)
    dims = [int(v) for v in args.case_shape.split(",")]
    g = torch.Generator(device="cuda").manual_seed(7)
    if args.case == "decode_attention":
        B, H, d, n = dims
        q = torch.randn(B, H * d, device="cuda", generator=g).bfloat16()
        k = torch.randn(B, H, n, d, device="cuda", generator=g).bfloat16()
        v = torch.randn(B, H, n, d, device="cuda", generator=g).bfloat16()
        out = torch.empty(B, H * d, device="cuda", dtype=torch.bfloat16)
        scr = native.decode_attention_scratch(native.BT_BF16, B, H, d, n)
        run = lambda: native.decode_attention(q, k, v, n, out=out, scratch=scr)  # noqa: E731
    elif args.case == "prefill_attention":
        B, H, d, n = dims
        q = torch.randn(B * n, H * d, device="cuda", generator=g).bfloat16()
        k = torch.randn(B, H, n, d, device="cuda", generator=g).bfloat16()
        v = torch.randn(B, H, n, d, device="cuda", generator=g).bfloat16()
        out = torch.empty(B * n, H * d, device="cuda", dtype=torch.bfloat16)
        run = lambda: native.prefill_attention_tc(q, k, v, n, out=out)  # noqa: E731
    else:
        M, N, K = dims
        x = torch.randn(M, K, device="cuda", generator=g).bfloat16()
        w = torch.randn(N, K, device="cuda", generator=g).bfloat16()
        out = torch.empty(M, N, device="cuda")
        scr = torch.zeros(native.lib().bt_op_linear_scratch_bytes(M, N), dtype=torch.uint8, device="cuda")
        run = lambda: native.linear(x, w, None, path=2, out=out, scratch=scr)  # noqa: E731
    for _ in range(args.case_steps):
        run()
    torch.cuda.synchronize()
    print(json.dumps({"case": args.case, "shape": dims, "launches": args.case_steps}), flush=True)


def relaunch_distributed(n: int):
    """One process per GPU: run this script again under torch.distributed.run
    with n ranks on this node (rendezvous on 127.0.0.1)."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    os.execv(sys.executable, cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-profile", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip runs_extra (L_B sweep incl. vanilla, pythia410m-scale, long context)")
    ap.add_argument("--max-batch-cap", type=int, default=0,
                    help="bound on the largest batch of the batch sweep (0: the planner's, memory and "
                         "buffer indexing only)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="time budget of the cpu_baseline leg of our arm")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: oracle time budget over all warm-up and timed steps")
    ap.add_argument("--case", default=None, choices=["decode", "prefill", "decode_attention", "prefill_attention",
                                                     "linear", "lb_sweep",
                                                     "batch_sweep", "variants"],
                    help="instead of the benchmark, run a bounded case for profiler captures: decode "
                         "calls of the decode-heavy workload, or one op of the path")
    ap.add_argument("--case-steps", type=int, default=None,
                    help="decode calls / launches of the case (default 8); lb_sweep: generated "
                         "tokens (default: the configured 512)")
    ap.add_argument("--case-shape", default="128,16,64,640",
                    help="decode_attention, prefill_attention: B,H,d,n; linear: M,N,K")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.case is None:
        relaunch_distributed(args.gpus)
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws != args.gpus and args.case is None:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={ws}; timing {ws} rank(s)", file=sys.stderr)
    if args.case == "lb_sweep":
        args.case_steps = args.case_steps or 0
        run_lb_sweep(args)
        return
    if args.case == "batch_sweep":
        import torch
        torch.cuda.set_device(0)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        hbm, _, tf_sus, _ = _peaks()
        print(json.dumps({"case": "batch_sweep",
                          **run_batch_sweep(flush, hbm, tf_sus, cap=args.max_batch_cap)}), flush=True)
        return
    if args.case is not None and args.case_steps is None:
        args.case_steps = 8
    if args.case == "decode":
        run_decode_case(args)
        return
    if args.case == "prefill":
        run_prefill_case(args)
        return
    if args.case == "variants":
        run_variants_case(args)
        return
    if args.case in ("decode_attention", "prefill_attention", "linear"):
        run_kernel_case(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
