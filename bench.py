"""Throughput of the GPT-2 124M forward pass (B=4, T=1024, bf16) on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one full forward pass through the C ABI (gpt2_forward_loss):
embedding, 12 Pre-LN blocks, ln_f, the tied lm_head writing fp32 logits
[4, 1024, 50257], and the shifted cross-entropy. Inputs are resident in HBM
when the timed region starts; `e2e` repeats the measurement with the ids and
targets copied from pinned host memory and the loss read back every step
(the copies on a second stream, overlapping the neighbouring steps;
`serial_value`: the same with every copy between the steps).
Under torchrun (N > 1) every rank runs its own batch of 4 sequences (weak
scaling, data-parallel replicas); the only exchange is an all-reduce of the
loss numerator and count. Rank 0 prints one JSON line.

--impl reference times the CPU oracle (fp64 NumPy, the plain definition of
the forward pass) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

WL = synthetic.WORKLOADS[1]          # GPT-2 124M, B=4, T=1024, bf16
METRIC = "GPT-2 124M fwd tokens/s (B4,T1024,bf16), 1 B200; % of BF16 tensor peak"
UNIT = "tokens/s"


def n_params(wl) -> int:
    C, V, L = wl.n_embd, wl.vocab, wl.n_layer
    per_layer = 2 * C + 3 * C * C + 3 * C + C * C + C + 2 * C + 4 * C * C + 4 * C + 4 * C * C + C
    return V * C + wl.n_ctx * C + L * per_layer + 2 * C


def model_flops(wl, tokens_per_seq=None, seqs=None) -> float:
    """2 * params * tokens over the parameters that multiply (every parameter
    but the position table, which is gathered: the blocks, ln_f and the tied
    wte as the lm_head), plus causal attention 2 * C * T * (T + 1) per layer
    and sequence (QK^T and PV over the lower triangle with its diagonal)."""
    T = tokens_per_seq or wl.seq
    Bn = seqs or wl.batch
    return 2.0 * (n_params(wl) - wl.n_ctx * wl.n_embd) * Bn * T + wl.n_layer * Bn * 2.0 * wl.n_embd * T * (T + 1)


def lmhead_flops(wl, M) -> float:
    return 2.0 * M * wl.vocab * wl.n_embd


LMHEAD_SOURCES = ("transformer_decoder_lm_b200/csrc/gemm_tc.cu", "transformer_decoder_lm_b200/csrc/common.cuh",
                  "transformer_decoder_lm_b200/csrc/kernels.h")
LMHEAD_PROFILE = "profiles/lm_head_tcgen05_124M.md"


def lmhead_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in LMHEAD_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def lmhead_traffic():
    """DRAM bytes (read + write) per lm_head launch from the committed ncu
    summary, or None if the summary is missing or was taken on other kernel
    sources than the ones built now."""
    import re
    p = os.path.join(ROOT, LMHEAD_PROFILE)
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m_hash = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != lmhead_source_hash():
        return None
    return int(m_bytes.group(1))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 6:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[2:6]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline(budget_s: float = 12.0):
    """Time the CPU oracle (as it stands) on a bounded sample of the workload:
    whole 1024-token sequences of the 124M model, forward + shifted loss,
    repeated until ~budget_s of CPU work. Returns the dict for the JSON line."""
    from oracle import gpt2_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1
    W = synthetic.make_weights(WL)
    ids = synthetic.make_ids(WL)
    done, tokens, elapsed = 0, 0, 0.0
    while done == 0 or (elapsed < budget_s and done < WL.batch):   # at least one whole sequence
        x = ids[done:done + 1]
        t0 = time.perf_counter()
        z = O.forward(W, x, WL.n_head)
        O.shifted_cross_entropy(z, x)
        elapsed += time.perf_counter() - t0
        tokens += x.size
        done += 1
    return {"value": tokens / elapsed, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"{done} of {WL.batch} sequences x {WL.seq} tokens of the 124M workload, fp64 NumPy forward "
                      f"+ shifted cross-entropy, {elapsed:.1f} s"}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the host cores. Each
    step is a bounded sample of the 124M workload - the forward + shifted loss
    of a prefix of one of its sequences (causal, so a prefix is a valid
    forward), its length chosen so that the whole warm-up + timed run takes
    about two minutes whatever --steps and --warmup are."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import gpt2_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1
    W = synthetic.make_weights(WL)
    ids = synthetic.make_ids(WL)

    def sample(k, n):
        x = ids[k % WL.batch:k % WL.batch + 1, :n]
        t0 = time.perf_counter()
        O.shifted_cross_entropy(O.forward(W, x, WL.n_head), x)
        return time.perf_counter() - t0

    per_token = sample(0, 128) / 128.0   # calibration (not timed)
    budget = max(0.25, 120.0 / max(1, args.steps + args.warmup))
    n = int(min(WL.seq, max(16, budget / max(per_token, 1e-9))) // 16 * 16)
    for k in range(args.warmup):
        sample(k, n)
    elapsed = sum(sample(args.warmup + k, n) for k in range(args.steps))
    v = args.steps * n / elapsed
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * elapsed / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WL.name, "global_batch": WL.batch * args.gpus, "seq_len": WL.seq,
                   "parallelism": f"dp{args.gpus}", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": int(cores), "kind": "oracle",
                         "sample": f"per step the first {n} tokens of one 1024-token sequence of the 124M workload, "
                                   f"fp64 NumPy forward + shifted cross-entropy ({elapsed:.1f} s over {args.steps} steps); "
                                   f"ms_per_step is the time of one such {n}-token step; a whole {WL.batch}x{WL.seq} "
                                   f"batch would take {WL.batch * WL.seq / n:.1f} times as long"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import transformer_decoder_lm_b200 as G

    W = synthetic.make_weights(WL)
    ids_np = synthetic.make_ids(WL)
    if world > 1:   # each rank its own sequences (same distribution, rank-offset draw)
        ids_np = np.random.default_rng(1501 + 7919 * rank).integers(0, WL.vocab, size=ids_np.shape).astype(np.int32)
    tg_np = synthetic.next_token_targets(ids_np)
    model = G.GPT2Model.from_workload(WL, W)
    stream = torch.cuda.current_stream()
    ids = torch.from_numpy(ids_np).cuda()
    tg = torch.from_numpy(tg_np).cuda()
    M = WL.batch * WL.seq
    logits = torch.empty(WL.batch, WL.seq, WL.vocab, dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    n_valid = float((tg_np >= 0).sum())

    from transformer_decoder_lm_b200 import dist as gdist

    def step(i_ids, i_tg, o_loss=None):
        o_loss = loss if o_loss is None else o_loss
        G.gpt2_forward_loss(model.handle, i_ids, i_tg, WL.batch, WL.seq, logits, o_loss, None, stream)
        if world > 1:   # the one exchange of the data-parallel forward: the loss mean
            o_loss.copy_(gdist.global_mean_loss(o_loss, int(n_valid)))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step(ids, tg)
    barrier()
    rc = model.status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {G.gpt2_error_string(rc)}")

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    launches0 = G.gpt2_launch_count(model.handle)
    barrier()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            step(ids, tg)
        t1.record(stream)
        barrier()
    launches = G.gpt2_launch_count(model.handle) - launches0
    ms = t0.elapsed_time(t1)

    # The dominant kernel (lm_head + fused log-sum-exp) on a separate pass of
    # the same steps, with CUDA events recorded around its launch on the
    # launching stream (events between two kernels break their programmatic
    # overlap, so they stay out of the step timing above).
    lm_steps = min(args.steps, 50)
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(lm_steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(lm_steps)]
    for ev in ev_b + ev_e:   # creates the underlying CUDA events before their handles are passed on
        ev.record(stream)
    barrier()
    for i in range(lm_steps):
        G.gpt2_set_timing_events(model.handle, G.binding.GPT2_TIMED_LMHEAD, ev_b[i], ev_e[i])
        step(ids, tg)
    G.gpt2_set_timing_events(model.handle, G.binding.GPT2_TIMED_LMHEAD, None, None)
    barrier()
    lm_ms = float(np.mean([b.elapsed_time(e) for b, e in zip(ev_b, ev_e)]))
    rc = model.status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {G.gpt2_error_string(rc)}")
    if world > 1:
        ms = gdist.max_over_ranks(ms, "cuda")
    ms_step = ms / args.steps
    tokens_all = M * world
    value = tokens_all / (ms_step / 1000.0)

    # The same forward without the logits output: loss only (lm_head with the
    # fused log-sum-exp, no logits written) and the trunk only (ln_f output
    # left in the workspace, no lm_head), timed the same way.
    def timed_variant(fn):
        for _ in range(3):
            fn()
        barrier()
        v0 = torch.cuda.Event(enable_timing=True)
        v1 = torch.cuda.Event(enable_timing=True)
        v0.record(stream)
        for _ in range(args.steps):
            fn()
        v1.record(stream)
        barrier()
        vms = v0.elapsed_time(v1)
        if world > 1:
            vms = gdist.max_over_ranks(vms, "cuda")
        return {"ms_per_step": vms / args.steps, "tokens_per_s": M * world / (vms / args.steps / 1000.0)}

    variants = {
        "loss_only": timed_variant(lambda: G.gpt2_forward_loss(model.handle, ids, tg, WL.batch, WL.seq, None, loss,
                                                               None, stream)),
        "trunk_only": timed_variant(lambda: G.gpt2_forward(model.handle, ids, WL.batch, WL.seq, None, stream)),
    }
    rc = model.status()
    if rc != 0:
        raise RuntimeError(f"device status after the variants: {G.gpt2_error_string(rc)}")

    # e2e: host buffers, copies inside the timed region: every step copies
    # its ids and targets from pinned host memory and reads its loss back.
    # As a production loop does, the copies run on a second stream, double
    # buffered: step i+1's inputs go up while step i computes, and step i's
    # loss comes back while step i+1 runs; the timed region ends after the
    # last loss has reached the host. The same loop with every copy on the
    # compute stream, between the steps, is reported as e2e_serial.
    h_ids = torch.from_numpy(ids_np).pin_memory()
    h_tg = torch.from_numpy(tg_np).pin_memory()
    h_loss = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(2)]
    d_ids = [torch.empty_like(ids) for _ in range(2)]
    d_tg = [torch.empty_like(tg) for _ in range(2)]
    d_loss = [torch.empty(1, dtype=torch.float32, device="cuda") for _ in range(2)]
    cs = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]

    def e2e_pipelined(n):
        with torch.cuda.stream(cs):
            d_ids[0].copy_(h_ids, non_blocking=True)
            d_tg[0].copy_(h_tg, non_blocking=True)
            ev_in[0].record(cs)
        for i in range(n):
            b = i & 1
            if i + 1 < n:   # the next step's inputs, once step i-1 no longer reads that buffer
                with torch.cuda.stream(cs):
                    if i >= 1:
                        cs.wait_event(ev_done[b ^ 1])
                    d_ids[b ^ 1].copy_(h_ids, non_blocking=True)
                    d_tg[b ^ 1].copy_(h_tg, non_blocking=True)
                    ev_in[b ^ 1].record(cs)
            stream.wait_event(ev_in[b])
            if i >= 2:   # step i-2's loss has been read out of this buffer
                stream.wait_event(ev_read[b])
            step(d_ids[b], d_tg[b], d_loss[b])
            ev_done[b].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(ev_done[b])
                h_loss[b].copy_(d_loss[b], non_blocking=True)
                ev_read[b].record(cs)
        stream.wait_stream(cs)

    def e2e_serial(n):
        for _ in range(n):
            d_ids[0].copy_(h_ids, non_blocking=True)
            d_tg[0].copy_(h_tg, non_blocking=True)
            step(d_ids[0], d_tg[0], d_loss[0])
            h_loss[0].copy_(d_loss[0], non_blocking=True)

    def timed_e2e(run):
        run(3)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(args.steps)
        e1.record(stream)
        barrier()
        t = e0.elapsed_time(e1)
        if world > 1:
            t = gdist.max_over_ranks(t, "cuda")
        return tokens_all / (t / args.steps / 1000.0)

    e2e_value = timed_e2e(e2e_pipelined)
    e2e_serial_value = timed_e2e(e2e_serial)
    if not math.isfinite(float(h_loss[0].item())) or abs(float(h_loss[0].item()) - float(loss.item())) > 1e-5:
        raise RuntimeError("the loss read back in the end-to-end loop differs from the device-timed one")

    hbm, tf_burst, tf_sust, peak_kind = peaks()
    lm_tflops = lmhead_flops(WL, M) / (lm_ms / 1000.0) / 1e12
    total_tflops = model_flops(WL) * world / (ms_step / 1000.0) / 1e12
    clk = clocks.summary()
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded random init, uniform ids)",
        "config": {"workload": WL.name, "model": "GPT-2 124M (L12 H12 C768 V50257)", "global_batch": WL.batch * world,
                   "seq_len": WL.seq, "parallelism": f"dp{world}", "outputs": "fp32 logits + shifted CE loss",
                   "l2": "no flush: per-step working set > L2 (weights 249 MB read, logits 823 MB written)"},
        "tflops": total_tflops,
        "frac_of_bf16_peak": total_tflops / tf_burst,
        "peak_note": f"{peak_kind} bf16 {tf_burst} TF/s burst, {tf_sust} sustained",
        "roofline": {"kernel": "lm_head tcgen05 GEMM + fused log-sum-exp (gemm_tc_kernel EPI_LMHEAD)",
                     "bound": "tensor", "achieved": lm_tflops, "peak": tf_burst, "unit": "TFLOP/s",
                     "frac": lm_tflops / tf_burst, "traffic": lmhead_traffic(),
                     "flops_per_launch": lmhead_flops(WL, M), "ms_per_launch": lm_ms,
                     "launches_timed": lm_steps,
                     "peak_kind": f"{peak_kind} burst (the timed region lasts tens of milliseconds)"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h_ids.numel() * 4 + h_tg.numel() * 4),
                "d2h_bytes_per_step": 4, "copies": "second stream, double buffered",
                "serial_value": e2e_serial_value},
        "gpu_launches": int(launches),
        "variants": variants,
        "clocks": clk,
        "loss": float(loss.item()),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(out), flush=True)
    model.close()
    if world > 1:
        dist.destroy_process_group()


def run_kernel(args):
    """Run one step of the forward pass on its own, at the 124M workload's
    shapes, through the single-step C entry points (for per-kernel timing and
    profiler captures). Prints the mean CUDA-event time per launch."""
    import torch
    import transformer_decoder_lm_b200 as G

    torch.cuda.set_device(0)
    rng = np.random.default_rng(0)
    M, C, V, H = WL.batch * WL.seq, WL.n_embd, WL.vocab, WL.n_head
    bf = torch.bfloat16

    def rnd(*shape, scale=1.0, dtype=bf):
        return (torch.from_numpy(rng.standard_normal(shape).astype(np.float32)) * scale).to("cuda", dtype)

    k = args.kernel
    if k in ("lmhead", "lmhead_ce"):
        hf, wte = rnd(M, C), rnd(V, C, scale=0.02)
        tg = torch.from_numpy(rng.integers(0, V, size=M).astype(np.int32)).cuda()
        logits = torch.empty(M, V, dtype=torch.float32, device="cuda") if k == "lmhead" else None
        loss = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.empty(G.gpt2_op_lmhead_ce_workspace_bytes(G.GPT2_BF16, M, V), dtype=torch.uint8, device="cuda")
        fn = lambda: G.gpt2_op_lmhead_ce(G.GPT2_BF16, hf, wte, tg, M, C, V, logits, None, loss, ws)
        flops = lmhead_flops(WL, M)
    elif k in ("c_attn", "attn_proj", "c_fc", "mlp_proj"):
        N, K, epi = {"c_attn": (3 * C, C, 0), "attn_proj": (C, C, 2), "c_fc": (4 * C, C, 1),
                     "mlp_proj": (C, 4 * C, 2)}[k]
        A, W, b = rnd(M, K), rnd(N, K, scale=0.02), rnd(N, scale=0.01)
        out = torch.zeros(M, N, dtype=torch.float32 if epi == 2 else bf, device="cuda")
        fn = lambda: G.gpt2_op_linear(G.GPT2_BF16, epi, A, W, b, M, N, K, out)
        flops = 2.0 * M * N * K
    elif k == "attention":
        qkv, y = rnd(M, 3 * C), torch.empty(M, C, dtype=bf, device="cuda")
        fn = lambda: G.gpt2_op_attention(G.GPT2_BF16, qkv, WL.batch, WL.seq, H, C, y)
        flops = WL.batch * 2.0 * C * WL.seq * (WL.seq + 1)
    elif k == "embed_ln":
        ids = torch.from_numpy(rng.integers(0, V, size=M).astype(np.int32)).cuda()
        wte, wpe = rnd(V, C, scale=0.02), rnd(WL.n_ctx, C, scale=0.02)
        g, be = rnd(C), rnd(C)
        x = torch.empty(M, C, dtype=torch.float32, device="cuda")
        h = torch.empty(M, C, dtype=bf, device="cuda")
        fn = lambda: G.gpt2_op_embed_layernorm(ids, wte, wpe, M, WL.seq, C, V, g, be, x, h)
        flops = 0.0
    elif k == "embed":
        ids = torch.from_numpy(rng.integers(0, V, size=M).astype(np.int32)).cuda()
        wte, wpe = rnd(V, C, scale=0.02), rnd(WL.n_ctx, C, scale=0.02)
        x = torch.empty(M, C, dtype=torch.float32, device="cuda")
        fn = lambda: G.gpt2_op_embed(G.GPT2_BF16, ids, wte, wpe, M, WL.seq, C, V, x)
        flops = 0.0
    elif k == "layernorm":
        x, g, b = rnd(M, C, dtype=torch.float32), rnd(C), rnd(C)
        out = torch.empty(M, C, dtype=bf, device="cuda")
        fn = lambda: G.gpt2_op_layernorm(G.GPT2_BF16, x, g, b, M, C, out)
        flops = 0.0
    elif k == "train":
        # one training step's forward and backward of the 124M model at B 4,
        # T 1024 (gpt2_forward_backward: loss and every weight's gradient)
        model = G.GPT2Model.from_workload(WL, synthetic.make_weights(WL))
        grads = model.new_grads()
        tws = model.new_train_workspace()
        ids_np = synthetic.make_ids(WL)
        ids = torch.from_numpy(ids_np).cuda()
        tg = torch.from_numpy(synthetic.next_token_targets(ids_np)).cuda()
        loss = torch.empty(1, dtype=torch.float32, device="cuda")
        fn = lambda: model.forward_backward(ids, tg, grads, tws, loss_out=loss)
        flops = 3.0 * model_flops(WL)   # forward, then about twice its work for the gradients
    elif k == "attn_bwd":
        # the attention gradient of one layer (gpt2_op_attention_backward: Dv,
        # the tcgen05 kernel, the dq scaling) after one training forward
        qkv, dy = rnd(M, 3 * C), rnd(M, C)
        y = torch.empty(M, C, dtype=bf, device="cuda")
        lse2 = torch.empty(WL.batch, H, WL.seq, dtype=torch.float32, device="cuda")
        G.gpt2_op_attention_train(qkv, WL.batch, WL.seq, H, C, y, lse2)
        ws = torch.empty(G.gpt2_op_attention_backward_workspace_bytes(WL.batch, WL.seq, H, C), dtype=torch.uint8,
                         device="cuda")
        dqkv = torch.empty(M, 3 * C, dtype=bf, device="cuda")
        fn = lambda: G.gpt2_op_attention_backward(qkv, y, dy, lse2, WL.batch, WL.seq, H, C, dqkv, ws)
        flops = 2.5 * WL.batch * 2.0 * C * WL.seq * (WL.seq + 1)
    elif k == "decode":
        # one incremental decoding step of the 124M model for 4 sequences at
        # position 1023 (context 1024), after a prefill of positions 0..1022
        model = G.GPT2Model.from_workload(WL, synthetic.make_weights(WL))
        cache = model.new_kv_cache()
        ids = torch.from_numpy(synthetic.make_ids(WL)).cuda()
        pos = WL.seq - 1
        model.prefill(ids[:, :pos].contiguous(), cache, want_logits=False)
        new = ids[:, pos].contiguous()
        dlog = torch.empty(WL.batch, V, dtype=torch.float32, device="cuda")
        fn = lambda: model.decode_step(new, pos, cache, logits=dlog)
        flops = 0.0
        es = 2
        n_block = WL.n_layer * (12 * C * C + 13 * C)   # Linear weights + biases + LN of the blocks
        decode_bytes = es * (n_block + V * C) + es * WL.n_layer * WL.batch * WL.seq * 2 * C
    else:
        raise SystemExit(f"unknown kernel {k}")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    # Replay the launches from a captured CUDA graph so that the host-side
    # cost of each binding call does not hide the GPU time of short kernels.
    per_graph = 20
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()                                   # first call on this stream outside the capture
        stream.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(per_graph):
                fn()
    torch.cuda.synchronize()
    reps = max(1, args.steps // per_graph)
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * per_graph)
    line = {"kernel": k, "ms_per_launch": ms, "tflops": flops / (ms / 1e3) / 1e12 if flops else None,
            "launches": reps * per_graph, "timing": "CUDA graph replay"}
    if k == "decode":
        hbm = peaks()[0]
        line.update({"tokens_per_s": WL.batch / (ms / 1e3), "context": WL.seq,
                     "min_bytes_per_step": decode_bytes, "gbs": decode_bytes / (ms / 1e3) / 1e9,
                     "hbm_frac": decode_bytes / (ms / 1e3) / 1e9 / hbm})
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default=None,
                    help="run one step alone: lmhead, lmhead_ce (no logits), c_attn, attn_proj, c_fc, mlp_proj, "
                         "attention, attn_bwd (attention gradient), embed, embed_ln (with the first ln_1), layernorm, "
                         "train (forward + backward), "
                         "decode (one key/value-cache decoding step, B 4, context 1024)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.kernel:
        run_kernel(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
