"""Benchmark of the S3R per-round hot path on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload qwen3-8b]

A step is one whole S3R round over the batch of the chosen synthetic workload (default:
the Qwen3-8B-shaped single attention layer, 32 requests with contexts uniform in
[8192, 24576], k = 6, s = 0.05, vocabulary 151936): select, k x (sparse draft attention +
draft sampling), dense verify with score capture, speculative sampling and commit, every
step in libs3r.so. Each step starts from the workload's committed lengths (the lengths are
restored by a 4-byte-per-request device copy), so every timed step is the same workload.
Inputs (KV cache 2.1 GB, logits 0.25 GB per round) are larger than the 126 MB L2.

Rank 0 prints one JSON line. `--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "accepted tokens/s per draft+verify round"
UNIT = "tokens/s"


# ------------------------------------------------------------------------ helpers -------
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(
        os.environ.get("LOCAL_RANK", 0))


def reduce_results(elapsed_ms: float, tokens: int, group=None):
    """Max of elapsed time and sum of tokens over ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return elapsed_ms, tokens
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    n = torch.tensor([tokens], dtype=torch.int64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(n, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), int(n.item())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


VERIFY_SOURCES = ["sparse_dense_kv_b200/csrc/verify_tc.cu", "sparse_dense_kv_b200/csrc/verify.cu",
                  "sparse_dense_kv_b200/csrc/attention.cuh", "sparse_dense_kv_b200/csrc/common.cuh",
                  "sparse_dense_kv_b200/csrc/kernels.h"]


def verify_traffic_per_launch(workload: str):
    """DRAM bytes per verify launch from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "verify_attn_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash(VERIFY_SOURCES):
        return None
    return d.get("per_launch_bytes", {}).get(workload)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self, t0, t1):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r for t, r in self.rows if t0 - 0.15 <= t <= t1 + 0.15] or [r for _, r in self.rows]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# -------------------------------------------------------------------- GPU workload ------
def build_workload(spec, rank, device):
    import torch
    lens = synth.make_lengths(spec)
    k = spec.k
    cache = synth.build_cache(spec, lens, extra_tokens=k + 1 + 16, device=device,
                              seed=spec.data_seed + 7919 * rank)
    NR, Hq, Hkv, d, V = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.vocab
    s = 100 + 13 * rank
    inp = dict(
        q=synth.randn_bf16((NR, k + 1, Hq, d), s, device),
        k=synth.randn_bf16((NR, k + 1, Hkv, d), s + 1, device),
        v=synth.randn_bf16((NR, k + 1, Hkv, d), s + 2, device),
        p=synth.randn_f32((NR, k + 1, V), s + 3, device, scale=spec.logit_std),
    )
    inp["qlog"] = (inp["p"][:, :k] + synth.randn_f32((NR, k, V), s + 4, device,
                                                      scale=spec.draft_noise_std)).contiguous()
    seq = torch.as_tensor(lens, dtype=torch.int32, device=device)
    return lens, cache, seq, inp


def algorithmic_bytes(spec, lens, sel_counts=None):
    """KV bytes per launch: verify reads (L+k+1) positions, draft step i reads n+i+1 positions
    (+4 B per selected index), 2*d*2 bytes per position and KV head. sel_counts [NR][Hkv]
    (the set sizes the select kernel wrote) replaces the token budget n when given."""
    from sparse_dense_kv_b200.engine import budget_count
    Hkv, d, k = spec.num_kv_heads, spec.head_dim, spec.k
    per_pos = 2 * d * 2 * Hkv
    verify = int(sum((L + k + 1) for L in lens)) * per_pos
    draft = []
    for i in range(k):
        tot = 0
        for r, L in enumerate(lens):
            if sel_counts is None:
                ns = [budget_count(int(L), spec.budget_bp, spec.window)] * Hkv
            else:
                ns = [int(x) for x in sel_counts[r]]
            tot += sum((n + i + 1) * 2 * d * 2 + 4 * n for n in ns)
        draft.append(tot)
    G = spec.num_q_heads // Hkv
    scores = int(sum(lens)) * Hkv * G * (k + 1) * 4
    return verify, draft, scores


def projection_logits_round(eng, spec, inp, seq, seq0, o_prefill):
    """Fill inp["p"] / inp["qlog"] from a round whose logits are gamma * (head-concatenated
    attention output) @ W, W the workload's seeded bf16 projection; gamma is one scalar
    calibrated on the prefill outputs so that dense logits have standard deviation sqrt(2).
    Returns (gamma, the round's emitted-token count)."""
    import math as _m
    import torch
    NR, k = spec.num_requests, spec.k
    W = synth.projection_matrix(spec, seq.device).float()
    gamma = float(_m.sqrt(2.0) / (o_prefill.float().reshape(NR, -1) @ W).std().item())

    def draft_fn(i, out, q_logits):
        q_logits[:, i] = gamma * (out.float().reshape(NR, -1) @ W)

    def target_fn(vout, p_logits):
        p_logits.copy_((gamma * (vout.float().reshape(NR * (k + 1), -1) @ W)).view(NR, k + 1, -1))

    seq.copy_(seq0)
    before = int(eng.buf.stats[0].item())
    eng.round(inp["q"], inp["k"], inp["v"], inp["p"], inp["qlog"], draft_logits_fn=draft_fn,
              target_logits_fn=target_fn)
    torch.cuda.synchronize()
    return gamma, int(eng.buf.stats[0].item()) - before


def boundary_cases(eng, k, margin=1e-5, tight=1e-7):
    """Decisions of the last round whose margin to their boundary (as the samplers computed
    it) is below `margin` (the stated 1e-5) and below `tight` (about the rounding of the
    samplers' fp32 cumulative sums, the margins that can flip a decision): draft draws, and
    the accept tests and final draws of the speculative sampler (min(n_out, k) + 1 decisions
    per request). With a 151936-token vocabulary the mean cell of a draw is 6.6e-6 wide, so
    most draws lie within 1e-5 of a cell edge."""
    dm = eng.buf.draft_margins.cpu().numpy()
    sm = eng.buf.spec_margins.cpu().numpy()
    n_out = eng.buf.n_out.cpu().numpy()
    spec_dec = [sm[r, : min(int(n_out[r]), k) + 1] for r in range(len(n_out))]
    n_spec = int(sum(x.size for x in spec_dec))
    count = lambda th: {"draft_draws": int((dm < th).sum()),  # noqa: E731
                        "spec_decisions": int(sum((x < th).sum() for x in spec_dec))}
    return {"threshold": margin, **count(margin), "draft_of": int(dm.size), "spec_of": n_spec,
            "tight_threshold": tight, "tight": count(tight),
            "note": "counted from the samplers' margin outputs of the last timed round"}


def round_bytes(spec, lens, vb, db, sb, greedy=False):
    """Algorithmic HBM bytes of one round: verify K/V reads and score-logit writes, the
    selection's score-logit reads and its per-position score array (written, read), the
    draft K/V and index reads, and the samplers' logit reads (draft sampling: one row per
    request and step, whose normaliser the speculative sampling reuses; speculative sampling:
    the k+1 target rows, plus the drawn row's target and draft rows again; greedy: the k+1
    target rows)."""
    NR, Hkv, V, k = spec.num_requests, spec.num_kv_heads, spec.vocab, spec.k
    pos = int(sum(lens))
    select = sb + 2 * 4 * pos * Hkv
    draft_sampling = k * NR * V * 4
    spec_sampling = NR * (k + 1) * V * 4 + (0 if greedy else NR * V * 4 * 2)
    parts = {"verify_kv": int(vb), "verify_scores": int(sb), "select": int(select),
             "draft_kv": int(sum(db)), "draft_sampling": int(draft_sampling),
             "spec_sampling": int(spec_sampling)}
    return {"total": int(sum(parts.values())), "parts": parts}


def run_ours(args, spec):
    import torch
    import torch.distributed as dist
    import sparse_dense_kv_b200 as s3r

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    lens, cache, seq, inp = build_workload(spec, rank, dev)
    k = spec.k
    eng = s3r.S3REngine(cache.k_pool, cache.v_pool, cache.page_table, seq, spec.num_q_heads,
                        k=k, budget_bp=spec.budget_bp, window=spec.window, vocab=spec.vocab,
                        seed=spec.sample_seed + rank, page_select=args.select == "pages",
                        greedy=args.greedy)
    seq0 = seq.clone()
    o0 = eng.prefill(inp["q"][:, :1].contiguous(), inp["k"][:, :1].contiguous(), inp["v"][:, :1].contiguous())
    stream = torch.cuda.current_stream()

    def step(ev=None, x=inp):
        rec = (lambda name, i=None: (ev[name] if i is None else ev[name][i]).record(stream)) \
            if ev is not None else (lambda name, i=None: None)
        seq.copy_(seq0, non_blocking=True)
        rec("s0")
        eng.select()
        for i in range(k):
            rec("d0", i)
            eng.draft_attn(i, x["q"], x["k"], x["v"])
            rec("dm", i)
            eng.draft_sample(i, x["qlog"])
            rec("d1", i)
        rec("v0")
        eng.verify(x["q"], x["k"], x["v"])
        rec("v1")
        eng.sample_and_commit(x["p"], x["qlog"])
        rec("c1")

    for _ in range(args.warmup):
        step()
    assert eng.check_errors() == 0, "device error during warm-up"
    gamma = None
    if spec.projection_logits:
        # the logits of the round come from a seeded bf16 projection of the attention outputs
        # (the rest of the model, off the timed path): one round from the committed lengths,
        # in the steady state the warm-up reached, computes them; the timed rounds replay the
        # same round with these logits, so acceptance follows draft / verify fidelity
        gamma, _ = projection_logits_round(eng, spec, inp, seq, seq0, o0)
        assert eng.check_errors() == 0, "device error in the projection round"

    # the round as one CUDA graph: the same launches on the same buffers, no host work per
    # launch; the timed steps are graph replays
    graph, launches_per_step = eng.capture(step)
    for _ in range(2):
        graph.replay()
    assert eng.check_errors() == 0, "device error in the captured round"

    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    start, end = E(), E()
    tok0 = int(eng.buf.stats[0].item())
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    for _ in range(args.steps):
        graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop(t0, t1)
    launches = launches_per_step * args.steps
    ms = start.elapsed_time(end)
    tokens = int(eng.buf.stats[0].item()) - tok0
    assert eng.check_errors() == 0, "device error in the timed region"
    ms_max, tokens_all = reduce_results(ms, tokens)
    boundary = boundary_cases(eng, k)

    # per-kernel device times: eager steps with events between the library calls, each
    # enqueued behind a sleeping kernel so that the host is ahead and the kernels run back to
    # back as in the graph; the roofline of the dominant kernel (verify) comes from these
    nb = max(3, min(args.steps, 10))
    evs = [dict(s0=E(), d0=[E() for _ in range(k)], dm=[E() for _ in range(k)],
                d1=[E() for _ in range(k)], v0=E(), v1=E(), c1=E()) for _ in range(nb)]
    for e in evs:
        torch.cuda._sleep(30_000_000)
        step(e)
    torch.cuda.synchronize()
    assert eng.check_errors() == 0, "device error in the per-kernel pass"
    avg = lambda a, b: sum(a(e).elapsed_time(b(e)) for e in evs) / nb  # noqa: E731
    v_ms = avg(lambda e: e["v0"], lambda e: e["v1"])
    d_ms = [avg(lambda e: e["d0"][i], lambda e: e["dm"][i]) for i in range(k)]
    ds_ms = [avg(lambda e: e["dm"][i], lambda e: e["d1"][i]) for i in range(k)]
    sel_ms = avg(lambda e: e["s0"], lambda e: e["d0"][0])
    spec_ms = avg(lambda e: e["v1"], lambda e: e["c1"])
    # the verify call without score capture (score_logits = NULL): its K/V stream alone
    evn = [(E(), E()) for _ in range(nb)]
    for a_, b_ in evn:
        torch.cuda._sleep(30_000_000)
        a_.record(stream)
        s3r.s3r_verify_attn(eng.cache, eng.batch, k, inp["q"], inp["k"], inp["v"], eng.buf.verify_out,
                            eng.buf.lse, None, eng.ws)
        b_.record(stream)
    torch.cuda.synchronize()
    assert eng.check_errors() == 0, "device error in the no-capture verify pass"
    vn_ms = sum(a_.elapsed_time(b_) for a_, b_ in evn) / nb
    vb, db, sb = algorithmic_bytes(spec, lens, eng.buf.sel_count.cpu().numpy())
    peak, peak_kind = measured_peaks()
    v_gbs = vb / (v_ms * 1e-3) / 1e9
    d_gbs = sum(db) / (sum(d_ms) * 1e-3) / 1e9
    rb = round_bytes(spec, lens, vb, db, sb, greedy=args.greedy)

    # end to end through the public API: pinned host inputs in, tokens out, every round. The
    # inputs are double-buffered: while the graph of round s runs on the compute stream, the
    # copy stream brings round s+1's inputs into the other buffer set (its own graph)
    e2e = None
    if args.e2e_steps > 0:
        host = {n: t.cpu().pin_memory() for n, t in inp.items()}
        out_h = torch.empty((spec.num_requests, k + 1), dtype=torch.int32).pin_memory()
        n_h = torch.empty((spec.num_requests,), dtype=torch.int32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = out_h.numel() * 4 + n_h.numel() * 4
        inp_b = {n: t.clone() for n, t in inp.items()}
        graph_b, _ = eng.capture(lambda: step(x=inp_b))
        graphs, bufs = (graph, graph_b), (inp, inp_b)
        copy_stream = torch.cuda.Stream()
        ready = [torch.cuda.Event(), torch.cuda.Event()]
        free = [torch.cuda.Event(), torch.cuda.Event()]
        for ev_ in free:
            ev_.record(stream)
        e0, e1 = E(), E()
        tok_e = int(eng.buf.stats[0].item())
        torch.cuda.synchronize()
        e0.record(stream)
        copy_stream.wait_event(e0)
        for st_ in range(args.e2e_steps):
            b = st_ & 1
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(free[b])
                for n_, t in host.items():
                    bufs[b][n_].copy_(t, non_blocking=True)
                ready[b].record(copy_stream)
            stream.wait_event(ready[b])
            graphs[b].replay()
            free[b].record(stream)
            out_h.copy_(eng.buf.out_tokens, non_blocking=True)
            n_h.copy_(eng.buf.n_out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        tok_e = int(eng.buf.stats[0].item()) - tok_e
        ems, etok = reduce_results(e0.elapsed_time(e1), tok_e)
        e2e = {"value": etok / (ems * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "overlap": "inputs double-buffered, copy stream overlaps the previous round"}
        del graph_b
    del graph

    st = eng.buf.stats.cpu().numpy()
    acc = [float(st[2 + j] / max(st[2 + s3r.MAX_K + j], 1)) for j in range(k)]
    result = {
        "metric": METRIC, "value": tokens_all / (ms_max * 1e-3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{spec.name}: {spec.num_requests} requests, "
                               f"L {spec.lengths}, {spec.num_q_heads}/{spec.num_kv_heads} heads, "
                               f"d {spec.head_dim}, k {k}, s {spec.budget_bp / 1e4}, window {spec.window}, "
                               f"vocab {spec.vocab}",
                   "requests_per_gpu": spec.num_requests, "parallelism": f"replicas x{world}",
                   "selection": args.select,
                   "scores": "the next selection's position scores on a second stream, beside "
                             "speculative sampling and the commit",
                   "verification": "greedy" if args.greedy else "speculative sampling",
                   "l2": "inputs larger than L2 (KV 2.1 GB, logits 0.25 GB per round)"},
        "roofline": {"bound": "hbm", "achieved": v_gbs, "peak": peak, "unit": "GB/s",
                     "frac": v_gbs / peak, "traffic": verify_traffic_per_launch(spec.name),
                     "kernel": "s3r_verify_attn", "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": vb},
        "kernels": {"verify_ms": v_ms, "verify_kv_gbs": v_gbs,
                    "verify_gbs_with_scores": (vb + sb) / (v_ms * 1e-3) / 1e9,
                    "verify_no_capture_ms": vn_ms,
                    "verify_no_capture_kv_gbs": vb / (vn_ms * 1e-3) / 1e9,
                    "verify_no_capture_frac": vb / (vn_ms * 1e-3) / 1e9 / peak,
                    "draft_attn_ms_per_step": sum(d_ms) / k, "draft_kv_gbs": d_gbs,
                    "draft_sample_ms_per_step": sum(ds_ms) / k, "select_ms": sel_ms,
                    "spec_sample_commit_ms": spec_ms,
                    "frac_of_8tbs": {"verify": v_gbs / 8000.0, "draft": d_gbs / 8000.0}},
        "round_roofline": {"bytes": rb["total"], "parts": rb["parts"],
                           "ms_at_peak": rb["total"] / (peak * 1e9) * 1e3,
                           "achieved_gbs": rb["total"] / (ms_max / args.steps * 1e-3) / 1e9,
                           "frac": rb["total"] / (ms_max / args.steps * 1e-3) / 1e9 / peak},
        "boundary_cases": boundary,
        "tau": float(st[0] / max(st[1], 1)), "acceptance_by_position": acc,
        "gpu_launches": int(launches), "launches_per_step": int(launches_per_step),
        "execution": "CUDA graph of one round, replayed per step", "clocks": clocks, "e2e": e2e,
    }
    if spec.projection_logits:
        result["config"]["logits"] = (f"seeded bf16 projection (vocab {spec.vocab}) of the attention "
                                      f"outputs, gamma {gamma:.3f}, computed off the timed path")
        result["config"]["l2"] = "inputs larger than L2 (KV 3.2 GB)"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(spec, lens, cache, inp, budget_s=args.cpu_seconds,
                                              mode=oracle_mode(args))
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ----------------------------------------------------------- mixed-phase ragged batch ----
def run_ragged(args, spec):
    """The high-concurrency ragged workload: requests at mixed round phases over shuffled
    page tables. A step is one iteration of the mixed-phase schedule: the requests in the
    middle of a round draft their next token (one draft-attention and one draft-sampling
    launch over their ids, each request at its own step) and the others verify, sample,
    commit and select their next set (one launch each over their ids); k+1 steps give every
    request one round. The k+1 iteration patterns repeat, so each is captured once as a
    CUDA graph and the timed steps replay them in order; the drafting requests' current
    q/k/v rows (the model's output in a real system) are gathered per pattern outside the
    timed region. value = tokens emitted by the steps' commits / device time."""
    import torch
    import torch.distributed as dist
    import sparse_dense_kv_b200 as s3r

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    k, NR = spec.k, spec.num_requests
    # iterations the cache must absorb: warm-up, the capture's eager pass, timed steps, the
    # per-kernel pass and the end-to-end steps, each advancing a request by <= k+1 tokens a round
    iters = args.warmup + 2 * (k + 1) + args.steps + (k + 1) + args.e2e_steps
    extra = (iters // (k + 1) + 3) * (k + 1) + 16
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=extra, device=dev, seed=spec.data_seed + 7919 * rank)
    Hq, Hkv, d, V = spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.vocab
    s0 = 100 + 13 * rank
    inp = dict(q=synth.randn_bf16((NR, k + 1, Hq, d), s0, dev), k=synth.randn_bf16((NR, k + 1, Hkv, d), s0 + 1, dev),
               v=synth.randn_bf16((NR, k + 1, Hkv, d), s0 + 2, dev),
               p=synth.randn_f32((NR, k + 1, V), s0 + 3, dev, scale=spec.logit_std))
    inp["qlog"] = (inp["p"][:, :k] + synth.randn_f32((NR, k, V), s0 + 4, dev, scale=spec.draft_noise_std)).contiguous()
    seq = torch.as_tensor(lens, dtype=torch.int32, device=dev)
    eng = s3r.S3REngine(cache.k_pool, cache.v_pool, cache.page_table, seq, Hq, k=k, budget_bp=spec.budget_bp,
                        window=spec.window, vocab=V, seed=spec.sample_seed + rank,
                        page_select=args.select == "pages", greedy=args.greedy)
    eng.prefill(inp["q"][:, :1].contiguous(), inp["k"][:, :1].contiguous(), inp["v"][:, :1].contiguous())
    drv = s3r.MixedPhaseDriver(eng, synth.initial_phases(spec, seed=spec.data_seed + rank))
    drv.start(inp["q"], inp["k"], inp["v"], inp["qlog"])
    its = drv.cycle(inp["q"], inp["k"], inp["v"], inp["p"], inp["qlog"])
    n = len(its)
    stream = torch.cuda.current_stream()
    for w in range(args.warmup):
        its[w % n]()
    # finish the cycle, so the graphs are captured (each after one eager pass of its own
    # iteration) in cycle order from pattern 0
    for w in range(args.warmup, -(-args.warmup // n) * n):
        its[w % n]()
    assert eng.check_errors() == 0, "device error during warm-up"
    graphs, lpi = [], []
    for it in its:
        g, nl = eng.capture(it)
        graphs.append(g)
        lpi.append(nl)

    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    start, end = E(), E()
    tok0 = int(eng.buf.stats[0].item())
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    for st_ in range(args.steps):
        graphs[st_ % n].replay()
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop(t0, t1)
    ms = start.elapsed_time(end)
    tokens = int(eng.buf.stats[0].item()) - tok0
    assert eng.check_errors() == 0, "device error in the timed region"
    ms_max, tokens_all = reduce_results(ms, tokens)
    launches = sum(lpi[st_ % n] for st_ in range(args.steps))
    boundary = boundary_cases(eng, k)
    # the timed steps end on a cycle boundary only if steps % n == 0: finish the cycle so the
    # per-kernel pass starts at pattern 0
    for st_ in range(args.steps, -(-args.steps // n) * n):
        graphs[st_ % n].replay()

    # per-kernel device times over one eager cycle, behind a sleeping kernel; the lengths and
    # set sizes each iteration saw are copied aside on the device for the byte counts
    evs = [{n_: E() for n_ in ("d0", "dm", "d1", "v0", "v1", "c1", "s1")} for _ in range(n)]
    L_hist = torch.empty((n, NR), dtype=torch.int32, device=dev)
    C_hist = torch.empty((n, NR, Hkv), dtype=torch.int32, device=dev)
    torch.cuda._sleep(60_000_000)
    for c, it in enumerate(its):
        L_hist[c].copy_(eng.seq_lens)
        C_hist[c].copy_(eng.buf.sel_count)
        it(evs[c])
    torch.cuda.synchronize()
    assert eng.check_errors() == 0, "device error in the per-kernel pass"
    L_hist, C_hist = L_hist.cpu().numpy().astype(np.int64), C_hist.cpu().numpy().astype(np.int64)
    per_pos = 2 * d * 2 * Hkv
    v_ms = d_ms = ds_ms = sp_ms = sel_ms = 0.0
    vb = db = 0
    for c, it in enumerate(its):
        e = evs[c]
        d_ms += e["d0"].elapsed_time(e["dm"])
        ds_ms += e["dm"].elapsed_time(e["d1"])
        v_ms += e["v0"].elapsed_time(e["v1"])
        sp_ms += e["v1"].elapsed_time(e["c1"])
        sel_ms += e["c1"].elapsed_time(e["s1"])
        info = it.info
        vb += int(sum(L_hist[c, r] + k + 1 for r in info["v_ids"])) * per_pos
        for r in info["d_ids"]:
            i = int(info["steps"][r])
            db += int(sum((C_hist[c, r, h] + i + 1) * 2 * d * 2 + 4 * C_hist[c, r, h] for h in range(Hkv)))
    peak, peak_kind = measured_peaks()
    v_gbs = vb / (v_ms * 1e-3) / 1e9
    d_gbs = db / (d_ms * 1e-3) / 1e9

    # end to end: every step copies the rows its launches read from pinned host memory
    # (drafting requests: their current q/k/v rows and draft-logit row; verifying requests:
    # their q/k/v blocks, target and draft logits) and reads the emitted tokens back
    e2e = None
    if args.e2e_steps > 0:
        hp = {n_: t.cpu().pin_memory() for n_, t in inp.items()}
        plan = []
        for it in its:
            info = it.info
            di = torch.as_tensor(info["d_ids"], dtype=torch.long)
            vi = torch.as_tensor(info["v_ids"], dtype=torch.long)
            st_h = torch.as_tensor(info["steps"], dtype=torch.long)[di]
            host = {"qc": it.info["qc"].cpu()[di].pin_memory(), "kc": it.info["kc"].cpu()[di].pin_memory(),
                    "vc": it.info["vc"].cpu()[di].pin_memory(), "qd": hp["qlog"][di, st_h].pin_memory()}
            for n_ in ("q", "k", "v", "p", "qlog"):
                host["v_" + n_] = hp[n_][vi].pin_memory()
            devb = {n_: torch.empty_like(t, device=dev) for n_, t in host.items()}
            plan.append((di.to(dev), vi.to(dev), st_h.to(dev), host, devb))
        out_h = torch.empty((NR, k + 1), dtype=torch.int32).pin_memory()
        n_h = torch.empty((NR,), dtype=torch.int32).pin_memory()
        h2d = d2h = 0
        e0, e1 = E(), E()
        tok_e = int(eng.buf.stats[0].item())
        torch.cuda.synchronize()
        e0.record(stream)
        for st_ in range(args.e2e_steps):
            c = st_ % n
            di, vi, st_d, host, devb = plan[c]
            for n_, t in host.items():
                devb[n_].copy_(t, non_blocking=True)
                h2d += t.numel() * t.element_size()
            it = its[c].info
            it["qc"].index_copy_(0, di, devb["qc"])
            it["kc"].index_copy_(0, di, devb["kc"])
            it["vc"].index_copy_(0, di, devb["vc"])
            inp["qlog"][di, st_d] = devb["qd"]
            for n_ in ("q", "k", "v", "p", "qlog"):
                inp[n_].index_copy_(0, vi, devb["v_" + n_])
            graphs[c].replay()
            out_h.copy_(eng.buf.out_tokens, non_blocking=True)
            n_h.copy_(eng.buf.n_out, non_blocking=True)
            d2h += out_h.numel() * 4 + n_h.numel() * 4
        e1.record(stream)
        torch.cuda.synchronize()
        tok_e = int(eng.buf.stats[0].item()) - tok_e
        ems, etok = reduce_results(e0.elapsed_time(e1), tok_e)
        e2e = {"value": etok / (ems * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d // args.e2e_steps,
               "d2h_bytes_per_step": d2h // args.e2e_steps, "steps": args.e2e_steps,
               "overlap": "none: each step's rows are copied, scattered into place, then the step runs"}
    del graphs

    st = eng.buf.stats.cpu().numpy()
    acc = [float(st[2 + j] / max(st[2 + s3r.MAX_K + j], 1)) for j in range(k)]
    result = {
        "metric": METRIC, "value": tokens_all / (ms_max * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{spec.name}: {NR} requests, L {spec.lengths}, {Hq}/{Hkv} heads, d {d}, k {k}, "
                               f"s {spec.budget_bp / 1e4}, window {spec.window}, vocab {V}, mixed round phases, "
                               "shuffled page tables",
                   "step": "one iteration of the mixed-phase schedule (k+1 iterations = one round per request)",
                   "requests_per_gpu": NR, "parallelism": f"replicas x{world}", "selection": args.select,
                   "verification": "greedy" if args.greedy else "speculative sampling",
                   "l2": "inputs larger than L2 (KV 5.8 GB, logits 2.0 GB)"},
        "roofline": {"bound": "hbm", "achieved": v_gbs, "peak": peak, "unit": "GB/s", "frac": v_gbs / peak,
                     "traffic": None, "kernel": "s3r_verify_attn", "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": vb // n},
        "kernels": {"verify_ms_per_cycle": v_ms, "verify_kv_gbs": v_gbs, "draft_attn_ms_per_cycle": d_ms,
                    "draft_kv_gbs": d_gbs, "draft_sample_ms_per_cycle": ds_ms,
                    "spec_sample_commit_ms_per_cycle": sp_ms, "select_ms_per_cycle": sel_ms,
                    "frac_of_8tbs": {"verify": v_gbs / 8000.0, "draft": d_gbs / 8000.0},
                    "draft_frac": d_gbs / peak},
        "boundary_cases": boundary,
        "tau": float(st[0] / max(st[1], 1)), "acceptance_by_position": acc,
        "gpu_launches": int(launches), "launches_per_step": float(sum(lpi)) / n,
        "execution": f"{n} CUDA graphs (one per iteration pattern), replayed in order", "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline_ragged(spec, lens, cache, inp, budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cpu_baseline_ragged(spec, lens, cache, inp, budget_s=15.0):
    """The oracle's rounds of the first requests of the ragged workload (each request's round
    is what one cycle of iterations computes for it), on this host's cores."""
    base = cpu_baseline(spec.with_(mixed_phases=False), lens, cache, inp, budget_s=budget_s)
    base["sample"] += "; the oracle runs whole rounds (a cycle of k+1 iterations per request)"
    return base


# ---------------------------------------------------------------- admission scheduler ----


def run_sched(args):
    """KV-aware AIMD admission against offloading or recomputing at a fixed concurrency of
    256, on one synthetic rollout replica per rank (512 requests, 42,000 KV pages, a
    memory-pressure event taking a quarter of the pages for 1,000 iterations): transferred
    pages per 1,000 generated tokens and tokens per unit of modelled time. The library's
    host scheduler runs the replicas; the oracle is timed beside it on the same replica."""
    import torch.distributed as dist
    from datetime import timedelta
    from sparse_dense_kv_b200.replicas import simulate_replicas

    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group("gloo", timeout=timedelta(seconds=120))
    spec = synth.RolloutSpec(num_requests=512 * world)
    p, r, tau = synth.make_rollouts(spec)
    pressure = np.zeros(4000, dtype=np.int32)
    pressure[3000:4000] = 42000 // 4
    base = dict(capacity=42000, pressure=pressure)
    runs = {}
    for name, kw in [("aimd", dict(policy="aimd", cap0=16)),
                     ("fixed256_offload", dict(policy="fixed", cap0=256)),
                     ("fixed256_recompute", dict(policy="fixed", cap0=256, evict="recompute"))]:
        t0 = time.perf_counter()
        tot = simulate_replicas(p, r, tau, **base, **kw)
        wall = time.perf_counter() - t0
        runs[name] = dict(pages_per_1k_tokens=1000.0 * tot["transferred"] / max(tot["tokens"], 1),
                          recomputed_per_1k_tokens=1000.0 * tot["recomputed"] / max(tot["tokens"], 1),
                          tokens_per_time=tot["tokens"] / max(tot["time"], 1e-9), evictions=tot["evictions"],
                          iterations=tot["iterations"], done=tot["done"], stalled=tot["stalled"],
                          wall_s=wall)
    a, f = runs["aimd"], runs["fixed256_offload"]
    out = {"metric": "transferred KV pages per 1000 generated tokens (admission scheduler model)",
           "value": a["pages_per_1k_tokens"], "unit": "pages/1k tokens", "n_gpus": world,
           "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
           "data": "synthetic", "steps": 1, "warmup": 0,
           "config": {"workload": f"rollout replicas x{world}: 512 requests each, prompts U[200, 600], "
                                  "responses log-normal (median 6000, clip 24576), 1 + capped geometric "
                                  "tokens per round (k 6, accept 0.9), 42000 KV pages, pressure event",
                      "costs": "c0 10, c_kv 0.00074, c_xfer 0.094, c_rec 0.5, c_pre 0.5 per iteration / page"},
           "runs": runs,
           "aimd_vs_fixed_offload": {"pages_ratio": a["pages_per_1k_tokens"] / max(f["pages_per_1k_tokens"], 1e-9),
                                     "throughput_ratio": a["tokens_per_time"] / f["tokens_per_time"]},
           "gpu_launches": 0, "execution": "host C++ (libs3r.so s3r_sched_simulate), one replica per rank"}
    if rank == 0 and world == 1:
        from oracle import kv_sched_oracle as K
        t0 = time.perf_counter()
        K.simulate(p, r, tau, policy="aimd", cap0=16, **base)
        out["cpu_baseline"] = {"kind": "oracle", "cores": 1, "sample": "the AIMD replica",
                               "value": time.perf_counter() - t0, "unit": "s per replica",
                               "library_s": runs["aimd"]["wall_s"]}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ adaptive horizon ----


def run_adaptive(args, spec):
    """Rounds whose draft length an AdaptiveHorizon controller picks every --interval rounds
    from the measured acceptance by position, against the same procedure at the fixed k of
    the workload. Each length has its own CUDA graph: k draft steps, verify, speculative
    sampling, commit, and the selection of the next round from this verify's scores (so a
    graph never reads scores of another length); lengths grow from round to round. The
    controller prices a round at each length by replaying that length's graph (the line
    fitted to the replays of k = 3 .. k_max is reported beside it)."""
    import torch
    import sparse_dense_kv_b200 as s3r

    rank, world, local = dist_env()
    if world > 1:
        raise SystemExit("--adaptive runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    k_max, k0 = args.k_max, spec.k
    rounds_total = 2 * (args.warmup + args.steps) + 40
    spec_m = spec.with_(k=k_max)
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec_m, lens, extra_tokens=rounds_total * (k_max + 1) + 16, device=dev,
                              seed=spec.data_seed)
    NR, Hq, Hkv, d, V = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.vocab
    base = dict(q=synth.randn_bf16((NR, k_max + 1, Hq, d), 100, dev),
                k=synth.randn_bf16((NR, k_max + 1, Hkv, d), 101, dev),
                v=synth.randn_bf16((NR, k_max + 1, Hkv, d), 102, dev),
                p=synth.randn_f32((NR, k_max + 1, V), 103, dev, scale=spec.logit_std))
    noise = synth.randn_f32((NR, k_max, V), 104, dev, scale=1.0)
    if args.falling_acceptance:
        # draft noise growing with the draft position, so acceptance falls from about 0.96 at
        # the first position to about 0.68 at the sixth (the 8B model's 95.8% -> 67.9% that
        # [Wispaper] reports by draft position); std 0.11 + 0.142 (i - 1) at position i
        std = torch.tensor([0.11 + 0.142 * i for i in range(k_max)], device=dev).view(1, k_max, 1)
    else:
        std = spec.draft_noise_std
    base["qlog"] = base["p"][:, :k_max] + noise * std
    inputs = {k: dict(q=base["q"][:, : k + 1].contiguous(), k=base["k"][:, : k + 1].contiguous(),
                      v=base["v"][:, : k + 1].contiguous(), p=base["p"][:, : k + 1].contiguous(),
                      qlog=base["qlog"][:, :k].contiguous()) for k in range(1, k_max + 1)}
    seq0 = torch.as_tensor(lens, dtype=torch.int32, device=dev)

    def fresh_engine():
        seq = seq0.clone()
        eng = s3r.S3REngine(cache.k_pool, cache.v_pool, cache.page_table, seq, Hq, k=k0,
                            budget_bp=spec.budget_bp, window=max(spec.window, k_max + 1),
                            vocab=V, seed=spec.sample_seed, k_max=k_max)
        x = inputs[k_max]
        eng.prefill(x["q"][:, :1].contiguous(), x["k"][:, :1].contiguous(), x["v"][:, :1].contiguous())
        eng.select()
        graphs = {}
        for k in range(1, k_max + 1):
            eng.set_k(k)
            xk = inputs[k]

            def step(xk=xk, k=k):
                for i in range(k):
                    eng.draft_attn(i, xk["q"], xk["k"], xk["v"])
                    eng.draft_sample(i, xk["qlog"])
                eng.verify(xk["q"], xk["k"], xk["v"])
                eng.sample_and_commit(xk["p"], xk["qlog"])
                eng.select()
            graphs[k], _ = eng.capture(step)
        return eng, graphs

    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def replay_ms(graphs, k, n=8):
        a, b = E(), E()
        a.record()
        for _ in range(n):
            graphs[k].replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    def run(adaptive: bool):
        eng, graphs = fresh_engine()
        eng.set_k(k0)
        for _ in range(args.warmup):
            graphs[k0].replay()
        # costs per round: t(k) = c_verify + k c_draft, a least-squares line through the
        # replayed graphs of k = 3 .. k_max (one verify configuration: 32-row tiles at G = 4)
        round_ms = [replay_ms(graphs, k) for k in range(1, k_max + 1)]
        kk = np.arange(min(3, k_max), k_max + 1, dtype=np.float64)
        tt = np.array([round_ms[int(k) - 1] for k in kk])
        if kk.size >= 2:
            c_draft, c_verify = (float(x) for x in np.polyfit(kk, tt, 1))
        else:
            c_draft, c_verify = tt[0] / 2, tt[0] / 2
        c_draft, c_verify = max(c_draft, 1e-4), max(c_verify, 1e-4)
        ctl = s3r.AdaptiveHorizon(eng, decay=args.decay, round_costs=round_ms, stale_counts=True) \
            if adaptive else None
        assert eng.check_errors() == 0, "device error in warm-up"
        tok0 = int(eng.buf.stats[0].item())
        ks = []
        torch.cuda.synchronize()
        a, b = E(), E()
        a.record()
        k = k0
        for st_ in range(args.steps):
            if ctl is not None and st_ % args.interval == 0:
                k = ctl.step()
            ks.append(k)
            graphs[k].replay()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        tokens = int(eng.buf.stats[0].item()) - tok0
        assert eng.check_errors() == 0, "device error in the timed rounds"
        st = eng.buf.stats.cpu().numpy()
        acc = [float(st[2 + j] / max(st[2 + s3r.MAX_K + j], 1)) for j in range(k_max)]
        del graphs
        return dict(ms=ms, tokens=tokens, ks=ks, c_draft=c_draft, c_verify=c_verify, acc=acc, round_ms=round_ms)

    fixed = run(False)
    adapt = run(True)
    hist = {str(k): adapt["ks"].count(k) for k in range(1, k_max + 1) if k in adapt["ks"]}
    value = adapt["tokens"] / (adapt["ms"] * 1e-3)
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": adapt["ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{spec.name}: {NR} requests, L {spec.lengths} growing "
                               f"by the emitted tokens, {Hq}/{Hkv} heads, d {d}, s {spec.budget_bp / 1e4}, "
                               f"vocab {V}, adaptive draft length in 1..{k_max}"
                               + (", draft noise growing with the position" if args.falling_acceptance else ""),
                   "requests_per_gpu": NR, "parallelism": "replicas x1", "horizon": "adaptive",
                   "interval": args.interval, "decay": args.decay},
        "adaptive": {"k_histogram": hist, "round_cost_ms": adapt["round_ms"],
                     "c_draft_ms": adapt["c_draft"], "c_verify_ms": adapt["c_verify"],
                     "acceptance_by_position": adapt["acc"][:k_max],
                     "tau": adapt["tokens"] / max(1, args.steps * NR)},
        "fixed_k": {"k": k0, "value": fixed["tokens"] / (fixed["ms"] * 1e-3), "ms_per_step": fixed["ms"] / args.steps,
                    "tau": fixed["tokens"] / max(1, args.steps * NR)},
        "execution": "one CUDA graph per draft length, chosen on the host every interval rounds",
    }
    print(json.dumps(result), flush=True)


# -------------------------------------------------------------------------- sweep -------
def run_sweep(args):
    """Budget / draft-length sweep on the 32 x 24576 Qwen3-8B-shaped workload. Logits come
    from a seeded bf16 projection of the head-concatenated attention outputs (computed by a
    torch matmul between the library calls, outside the kernel timings), so acceptance
    follows how closely the sparse draft attention tracks the dense verify. One JSON line
    per (s, k) point: acceptance by draft position, tau, draft and verify KV GB/s."""
    import torch
    import sparse_dense_kv_b200 as s3r
    from sparse_dense_kv_b200.engine import budget_count
    spec = synth.WORKLOADS["sweep"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lens = synth.make_lengths(spec)
    kmax = max(spec.sweep_ks)
    rounds = args.sweep_rounds
    cache = synth.build_cache(spec, lens, extra_tokens=(kmax + 1) * (rounds + 4) + 16, device=dev)
    NR, Hq, Hkv, d, V = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.vocab
    W = synth.projection_matrix(spec, dev).float()
    seq0 = torch.as_tensor(lens, dtype=torch.int32, device=dev)
    per_pos = 2 * d * 2 * Hkv
    x0 = [synth.randn_bf16((NR, 1, Hq, d), 900 + j, dev) for j in range(3)]
    gamma = None
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for bp in spec.sweep_budgets_bp:
        for k in spec.sweep_ks:
            seq = seq0.clone()
            eng = s3r.S3REngine(cache.k_pool, cache.v_pool, cache.page_table, seq, Hq, k=k,
                                budget_bp=bp, window=spec.window, vocab=V, seed=spec.sample_seed)
            o0 = eng.prefill(x0[0], x0[1][:, :, :Hkv].contiguous(), x0[2][:, :, :Hkv].contiguous())
            if gamma is None:   # one scalar for all points: dense logits with std sqrt(2)
                gamma = float(math.sqrt(2.0) / (o0.float().reshape(NR, -1) @ W).std().item())
            pl = torch.empty((NR, k + 1, V), dtype=torch.float32, device=dev)
            ql = torch.empty((NR, k, V), dtype=torch.float32, device=dev)
            t_draft = t_verify = 0.0
            kv_draft = kv_verify = 0
            timed = 0
            for rnd in range(rounds + 1):
                s0 = 1000 * rnd + 10 * k + bp
                q = synth.randn_bf16((NR, k + 1, Hq, d), s0, dev)
                kb = synth.randn_bf16((NR, k + 1, Hkv, d), s0 + 1, dev)
                vb = synth.randn_bf16((NR, k + 1, Hkv, d), s0 + 2, dev)
                Lh = eng.seq_lens.cpu().numpy()
                if rnd == 1:
                    eng.buf.stats.zero_()
                eng.select()
                for i in range(k):
                    e0, e1 = E(), E()
                    e0.record()
                    eng.draft_attn(i, q, kb, vb)
                    e1.record()
                    ql[:, i] = gamma * (eng.buf.draft_out.float().reshape(NR, -1) @ W)
                    eng.draft_sample(i, ql)
                    if rnd:
                        torch.cuda.synchronize()
                        t_draft += e0.elapsed_time(e1)
                        kv_draft += sum((budget_count(int(L), bp, spec.window) + i + 1) * per_pos for L in Lh)
                e0, e1 = E(), E()
                e0.record()
                eng.verify(q, kb, vb)
                e1.record()
                pl.copy_((gamma * (eng.buf.verify_out.float().reshape(NR * (k + 1), -1) @ W))
                         .view(NR, k + 1, V))
                eng.sample_and_commit(pl, ql)
                if rnd:
                    torch.cuda.synchronize()
                    t_verify += e0.elapsed_time(e1)
                    kv_verify += sum((int(L) + k + 1) * per_pos for L in Lh)
                    timed += 1
            assert eng.check_errors() == 0
            st = eng.buf.stats.cpu().numpy()
            acc = [float(st[2 + j] / max(st[2 + s3r.MAX_K + j], 1)) for j in range(k)]
            print(json.dumps({
                "sweep_point": {"budget": bp / 1e4, "k": k}, "workload": spec.name,
                "rounds": timed, "requests": NR, "context": int(lens[0]),
                "acceptance_by_position": acc, "tau": float(st[0] / max(st[1], 1)),
                "draft_kv_gbs": kv_draft / (t_draft * 1e-3) / 1e9,
                "verify_kv_gbs": kv_verify / (t_verify * 1e-3) / 1e9,
                "gamma": gamma, "data": "synthetic"}), flush=True)
            del eng


# ------------------------------------------------------------------------- oracle -------
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return 1


def oracle_mode(args):
    """Keyword arguments of the oracle's round for the bench's selection / verification."""
    return {"page": 16 if args.select == "pages" else 1, "greedy": bool(args.greedy)}


def oracle_round_sample(spec, lens, pools, page_table, inp_host, reqs, mode=None, timings=None,
                        dtype=np.float64):
    """Oracle rounds for the requests `reqs` (dense copies built outside the timing);
    `timings` accumulates the seconds of each step of the round; `dtype` is the oracle's
    attention arithmetic (float64, or the float32 timing variant)."""
    from oracle import s3r_oracle as O
    k = spec.k
    kp, vp = pools
    prepared = []
    for r in reqs:
        L = int(lens[r])
        H = spec.num_kv_heads
        K = np.stack([O.gather_positions(kp, page_table[r], h, np.arange(L + k + 1)) for h in range(H)])
        V = np.stack([O.gather_positions(vp, page_table[r], h, np.arange(L + k + 1)) for h in range(H)])
        st = O.RequestState(K, V, L, dtype=dtype)
        q = inp_host["q"][r].astype(dtype)
        O.prefill_scores(st, q[0], inp_host["k"][r][0], inp_host["v"][r][0])
        prepared.append((r, st))
    t0 = time.perf_counter()
    tokens = 0
    for r, st in prepared:
        res = O.run_round(st, r, spec.sample_seed, k, spec.budget_bp, spec.window,
                          inp_host["q"][r], inp_host["k"][r], inp_host["v"][r],
                          inp_host["qlog"][r], inp_host["p"][r], timings=timings, **(mode or {}))
        tokens += res["n_out"]
    return tokens, time.perf_counter() - t0


def host_inputs(inp, reqs):
    return {n: {r: t[r].float().cpu().numpy() for r in reqs} for n, t in inp.items()}


def cpu_baseline(spec, lens, cache, inp, budget_s=15.0, mode=None):
    """The oracle on this host's cores on a bounded sample of the same workload, with the
    seconds of each step of its rounds, and the first sampled request's round again with
    the BLAS thread pool limited to one thread."""
    reqs, tokens, secs = [], 0, 0.0
    pt_all = cache.page_table.cpu().numpy()
    timings = {}

    def request_pools(r):
        # the request's own pages only (its page-table row renumbered), in float32 on the host
        import torch
        ids = pt_all[r][pt_all[r] >= 0]
        idx = torch.as_tensor(ids, dtype=torch.long, device=cache.k_pool.device)
        kp = cache.k_pool.index_select(0, idx).float().cpu().numpy()
        vp = cache.v_pool.index_select(0, idx).float().cpu().numpy()
        pt = np.full_like(pt_all, -1)
        pt[r, : ids.size] = np.arange(ids.size)
        return (kp, vp), pt

    r = 0
    while secs < budget_s and r < spec.num_requests:
        hi = host_inputs(inp, [r])
        pools, pt = request_pools(r)
        t, s = oracle_round_sample(spec, lens, pools, pt, hi, [r], mode, timings)
        tokens, secs = tokens + t, secs + s
        reqs.append(r)
        r += 1
    one = None
    try:
        from threadpoolctl import threadpool_limits
        hi = host_inputs(inp, [reqs[0]])
        pools, pt = request_pools(reqs[0])
        with threadpool_limits(limits=1):
            t1, s1 = oracle_round_sample(spec, lens, pools, pt, hi, [reqs[0]], mode)
        one = {"value": t1 / s1, "unit": UNIT, "cores": 1, "sample": f"one round of request {reqs[0]}",
               "seconds": s1}
    except ImportError:
        pass
    # the same sample with the oracle's attention in float32 (its samplers stay float64)
    t32, s32, timings32 = 0, 0.0, {}
    for r in reqs:
        hi = host_inputs(inp, [r])
        pools, pt = request_pools(r)
        t, s_ = oracle_round_sample(spec, lens, pools, pt, hi, [r], mode, timings32, dtype=np.float32)
        t32, s32 = t32 + t, s32 + s_
    fp32 = {"value": t32 / s32, "unit": UNIT, "cores": oracle_threads(), "seconds": round(s32, 3),
            "sample": "the same requests, attention in float32 numpy",
            "step_seconds": {n_: round(v_, 4) for n_, v_ in timings32.items()}}
    return {"value": tokens / secs, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"one round of requests {reqs[0]}..{reqs[-1]} ({len(reqs)} of "
                      f"{spec.num_requests}), float64 numpy, {secs:.1f} s",
            "step_seconds": {n_: round(v_, 4) for n_, v_ in timings.items()},
            "single_thread": one, "float32": fp32}


def run_reference(args, spec):
    """The CPU oracle as the reference arm: each step = one round of one request."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch
    sub = spec.with_(num_requests=max(1, min(spec.num_requests, 4)))
    lens = synth.make_lengths(spec)[: sub.num_requests]
    cache = synth.build_cache(sub.with_(lengths=("fixed", tuple(int(x) for x in lens))), lens,
                              extra_tokens=spec.k + 1 + 16, device="cpu")
    k = spec.k
    NR = sub.num_requests
    inp = dict(q=synth.randn_bf16((NR, k + 1, spec.num_q_heads, spec.head_dim), 100),
               k=synth.randn_bf16((NR, k + 1, spec.num_kv_heads, spec.head_dim), 101),
               v=synth.randn_bf16((NR, k + 1, spec.num_kv_heads, spec.head_dim), 102),
               p=synth.randn_f32((NR, k + 1, spec.vocab), 103, scale=spec.logit_std))
    inp["qlog"] = inp["p"][:, :k] + synth.randn_f32((NR, k, spec.vocab), 104, scale=spec.draft_noise_std)
    pools = (cache.k_pool.float().numpy(), cache.v_pool.float().numpy())
    pt = cache.page_table.numpy()
    tok, secs = 0, 0.0
    for s in range(args.warmup + args.steps):
        r = s % NR
        hi = host_inputs(inp, [r])
        t, dt = oracle_round_sample(spec, lens, pools, pt, hi, [r], oracle_mode(args))
        if s >= args.warmup:
            tok, secs = tok + t, secs + dt
    v = tok / secs
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {"workload": f"{spec.name}, one request-round per step",
                      "requests_sampled": NR, "selection": args.select,
                      "verification": "greedy" if args.greedy else "speculative sampling"},
           "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                            "sample": f"{args.steps} request-rounds over {NR} requests of the workload"},
           "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    del torch


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3-8b", choices=["tiny", "qwen3-1.7b", "qwen3-8b", "ragged", "sweep"],
                    help="synthetic workload (ragged: mixed-phase iterations; sweep: one (s, k) point of the "
                         "budget / draft-length sweep, --budget-bp / --k)")
    ap.add_argument("--budget-bp", type=int, default=0, help="sparse budget s in 1e-4 units (sweep point)")
    ap.add_argument("--k", type=int, default=0, help="draft length (sweep point)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--requests", type=int, default=0,
                    help="override the workload's request count (small cases for profiling)")
    ap.add_argument("--sweep", action="store_true",
                    help="budget / draft-length sweep (one JSON line per point)")
    ap.add_argument("--sweep-rounds", type=int, default=3)
    ap.add_argument("--select", choices=["positions", "pages"], default="positions",
                    help="selection unit: positions, or whole 16-position pages")
    ap.add_argument("--greedy", action="store_true",
                    help="temperature 0: argmax drafts and greedy verification")
    ap.add_argument("--adaptive", action="store_true",
                    help="draft length chosen from the measured acceptance (one line, with the fixed-k run)")
    ap.add_argument("--k-max", type=int, default=7,
                    help="largest adaptive draft length")
    ap.add_argument("--interval", type=int, default=4)
    ap.add_argument("--falling-acceptance", action="store_true",
                    help="with --adaptive: draft noise growing with the position (acceptance 0.96 -> 0.68)")
    ap.add_argument("--decay", type=float, default=0.8)
    ap.add_argument("--sched", action="store_true",
                    help="KV-aware admission scheduler model (host; one line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.sweep:
        run_sweep(args)
        return
    if args.sched:
        run_sched(args)
        return
    spec = synth.WORKLOADS[args.workload]
    if args.requests > 0:
        spec = spec.with_(num_requests=args.requests,
                          lengths=spec.lengths if spec.lengths[0] != "fixed"
                          else ("fixed", spec.lengths[1][: args.requests]))
    if args.budget_bp > 0 or args.k > 0:
        if not spec.projection_logits:
            raise SystemExit("--budget-bp / --k choose a point of the sweep workload")
        spec = spec.with_(budget_bp=args.budget_bp or spec.budget_bp, k=args.k or spec.k)
    if args.impl == "reference":
        run_reference(args, spec)
    elif args.adaptive:
        run_adaptive(args, spec)
    elif spec.mixed_phases:
        run_ragged(args, spec)
    else:
        run_ours(args, spec)


if __name__ == "__main__":
    main()
