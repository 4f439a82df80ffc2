"""Benchmark of the speculative-decoding verification step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload b256] [--variant auto|split|fused]

One step = one call of the library (row statistics, accept scan, race) over one
batch of synthetic logits already resident in HBM.  Workload (default): B=256
requests, D=7 drafts, V=128256, bf16 logits, target N(0, 3^2), draft = target +
N(0, 0.75^2), draft tokens sampled from q, T=1, stochastic mode.  Its inputs
(985 MB) exceed the 126 MB L2, so no flush is needed between steps; smaller
workloads rotate over copies of their inputs that together exceed twice the L2.

Multi-GPU (launched by torchrun): requests shard with no exchange, so every
rank verifies its own batch of the same shape (weak scaling, no data-path
collective); the step time is the max over ranks.

Prints one JSON line on rank 0.  `--impl reference` times the CPU oracle (the
plain double-precision restatement of the rule) on the host cores instead.
"""
import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified rows/s (B×(D+1)) and achieved HBM GB/s vs B200 peak, 1 GPU"
SPEC_HBM_GBS = 8000.0
KEV_EVERY = 8  # kernel-timing events on one step in 8 of the timed region
L2_ROTATE_BYTES = 2 * 126 * 1000 * 1000  # inputs below twice the L2 rotate over copies
MAX_INPUT_COPIES = 8192
FALLBACK_HBM_GBS = 6650.0


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_desc(w):
    m = w.meta
    if hasattr(w, "parents"):
        return (f"{w.name}: B={w.B}, draft tree with branching {tuple(m['branching'])} "
                f"({w.N} nodes), V={w.V}, {'bf16' if w.dtype == 1 else 'fp32'} logits, target "
                f"N(0,{m['target_sd']}^2), draft = target + N(0,{m['draft_sd']}^2), candidates drawn "
                f"from q at their parent, T={w.temperature}, "
                f"{['stochastic', 'greedy', 'saguaro'][w.mode]}")
    return (f"{w.name}: B={w.B}, D={w.D_max}, V={w.V}, "
            f"{'bf16' if w.dtype == 1 else 'fp32'} logits, target N(0,{m['target_sd']}^2), "
            f"draft = target + N(0,{m['draft_sd']}^2), draft tokens sampled from q, T={w.temperature}, "
            f"{['stochastic', 'greedy', 'saguaro'][w.mode]}")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.active = False
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            if self.active:
                self.samples.append([s.strip() for s in line.split(",")])

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for s in self.samples:
            try:
                sm.append(float(s[1]))
                mx.append(float(s[2]))
            except Exception:
                continue
            for name, v in zip(names, s[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def tail_items(w, sms):
    """Whether the library races a batch of this shape as items spread over the
    GPU (three split launches) rather than one CTA per request (two)."""
    seg_tokens = 4096 if w.dtype == 1 else 2048
    nseg = -(-w.V // seg_tokens)
    return 5 * w.B < 4 * sms and w.B * nseg > sms


def early_exit_bounds(D_max):
    """The position rounds of SV_VARIANT_EARLY_EXIT (the library's rule, in
    include/specverify.h): position 0, then 1-2, then 3 to D_max."""
    return [0] + [p for p in (1, 3) if p < D_max + 1] + [D_max + 1]


def early_exit_rows(accept_len, row_D, modes, D_max):
    """Rows the early-exit rounds read for outcomes accept_len (n = AL - 1): a
    request listed in a round reads every row of the round's positions up to
    D_b (draft rows only for sampling requests), plus the race's row."""
    bounds = early_exit_bounds(D_max)
    rows = 0
    for al, Db, m in zip(accept_len, row_D, modes):
        n = al - 1
        if n < 0:
            continue  # a parameter error: nothing read
        end = next(p1 for p0, p1 in zip(bounds, bounds[1:]) if p0 <= n < p1)
        last = min(end - 1, Db)
        rows += (last + 1) + (0 if m == 1 else min(end, Db) + 1)  # target, draft + race row
    return rows


def input_copies(in_bytes):
    """How many copies of a step's inputs the timed loop rotates over: enough
    that together they are at least twice the L2 (at most MAX_INPUT_COPIES),
    or 1 when the inputs alone are that large."""
    if in_bytes >= L2_ROTATE_BYTES:
        return 1
    return min(MAX_INPUT_COPIES, -(-L2_ROTATE_BYTES // max(1, in_bytes)))


def traffic_record(kernel_name, sources, alg_bytes):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source and on a launch of the same algorithmic bytes (the
    same workload), else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for s in sources:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    sha = h.hexdigest()[:16]
    rec = {}
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 5 and parts[0] == kernel_name and int(parts[4]) == alg_bytes:
                rec[parts[1]] = (float(parts[2]), int(parts[3]))  # sha -> (bytes per launch, units)
    return rec.get(sha)


def cpu_baseline(w, target_seconds=10.0, single_seconds=5.0):
    """The oracle, as it stands, on the host cores over the same host copy of the
    inputs: the whole batch repeated on all cores (OpenMP over requests) until
    about `target_seconds` pass, and the plain single-threaded loop on the first
    requests of the batch for about `single_seconds`."""
    import oracle
    cores = os.cpu_count() or 1
    if hasattr(w, "parents"):
        return tree_cpu_baseline(w, target_seconds, single_seconds, cores)
    h = w.host_arrays()

    def run(sl, nthreads):
        oracle.verify(h["target"][sl], h["draft"][sl], h["tokens"][sl],
                      None if h["row_D"] is None else h["row_D"][sl], temperature=w.temperature,
                      mode=w.mode, seed=w.seed,
                      temperature_per_req=None if h["temperature_per_req"] is None
                      else h["temperature_per_req"][sl],
                      mode_per_req=None if h["mode_per_req"] is None else h["mode_per_req"][sl],
                      saguaro_k=w.saguaro_k, saguaro_c=w.saguaro_c, nthreads=nthreads,
                      request_offset=sl.start)

    reps, t0 = 0, time.perf_counter()
    while True:
        run(slice(0, w.B), cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_seconds or reps >= 50:
            break
    rows = reps * w.verified_rows()
    D = w.row_D_list()
    # single core: requests one at a time until the budget is spent
    n1, t1 = 0, time.perf_counter()
    while n1 < w.B:
        run(slice(n1, n1 + 1), 1)
        n1 += 1
        if time.perf_counter() - t1 >= single_seconds:
            break
    el1 = time.perf_counter() - t1
    rows1 = sum(d + 1 for d in D[:n1])
    return {"value": rows / el, "unit": "rows/s", "cores": cores, "kind": "oracle",
            "sample": f"the whole {w.name} batch ({w.B} requests, {w.verified_rows()} verified rows) "
                      f"x {reps} repetitions, {el:.1f} s, OpenMP over requests on {cores} threads",
            "single_core": {"value": rows1 / el1, "unit": "rows/s", "cores": 1,
                            "sample": f"the first {n1} requests ({rows1} verified rows), "
                                      f"{el1:.1f} s, the plain single-threaded loop"}}


def tree_cpu_baseline(w, target_seconds, single_seconds, cores):
    """cpu_baseline for a tree workload: the oracle's tree walk."""
    import numpy as np
    import oracle

    def host(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch_int16()).numpy().view(np.uint16) if w.dtype == 1 else t.numpy()
    tgt, dft = host(w.target), host(w.draft)
    tok, par = w.tokens.cpu().numpy(), w.parents.cpu().numpy()

    def run(sl, nthreads):
        oracle.verify_tree(tgt[sl], dft[sl], tok[sl], par[sl], temperature=w.temperature,
                           mode=w.mode, seed=0, request_offset=sl.start, nthreads=nthreads)

    reps, t0 = 0, time.perf_counter()
    while True:
        run(slice(0, w.B), cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_seconds or reps >= 50:
            break
    n1, t1 = 0, time.perf_counter()
    while n1 < w.B:
        run(slice(n1, n1 + 1), 1)
        n1 += 1
        if time.perf_counter() - t1 >= single_seconds:
            break
    el1 = time.perf_counter() - t1
    per_req = w.verified_rows() // w.B
    return {"value": reps * w.verified_rows() / el, "unit": "rows/s", "cores": cores,
            "kind": "oracle",
            "sample": f"the whole {w.name} batch ({w.B} requests) x {reps} repetitions, {el:.1f} s, "
                      f"OpenMP over requests on {cores} threads",
            "single_core": {"value": n1 * per_req / el1, "unit": "rows/s", "cores": 1,
                            "sample": f"the first {n1} requests, {el1:.1f} s, single-threaded"}}


def torch_int16():
    import torch
    return torch.int16


def acceptance_stats(sv, w, variant, nseeds, stream):
    """Mean accepted length and the AL histogram (AL = 1 .. D_max+1) of the
    workload's stochastic requests over `nseeds` verifier seeds, from the
    library's own outputs; for requests that rejected a draft, the share whose
    correction token is among the draft row's k largest logits (what saguaro
    concentrates the residual on)."""
    import torch
    stoch = torch.tensor([m != sv.SV_GREEDY for m in w.modes()], device=w.target.device)
    hist = torch.zeros(w.D_max + 2, dtype=torch.int64, device=w.target.device)
    in_top = rejected = hits = 0
    k = min(w.saguaro_k, w.V)
    Db = torch.tensor(w.row_D_list(), device=w.target.device)
    # the speculation cache of speculative speculative decoding: keys (d + 1, each of the
    # draft's top-k at position d) for d < D, looked up with the verified outcome
    dev = w.target.device
    keys_tok = torch.topk(w.draft.float(), k, dim=-1).indices.to(torch.int32).reshape(w.B, -1)
    keys_al = (torch.arange(w.D_max, device=dev, dtype=torch.int32) + 1).repeat_interleave(k)
    keys_al = keys_al[None].repeat(w.B, 1).contiguous()
    keys_tok = keys_tok.contiguous()
    hit = torch.empty(w.B, dtype=torch.int32, device=dev)
    out = None
    for seed in range(nseeds):
        out = sv.verify_workload(w, seed=7000 + seed, variant=variant, stream=stream, out=out)
        sv._check(sv.sv_ssd_lookup(out["tokens"], out["accept_len"], w.B, w.D_max, keys_al, keys_tok,
                                   keys_al.shape[1], None, 0, hit, stream=stream))
        hits += int(((hit >= 0) & stoch).sum())
        al = out["accept_len"].long()
        hist += torch.bincount(al[stoch], minlength=w.D_max + 2)
        n = al - 1
        rej = stoch & (n < Db)
        if bool(rej.any()):
            b = torch.nonzero(rej).flatten()
            rows = w.draft[b, n[b]].float()
            top = torch.topk(rows, k, dim=-1).indices
            tok = out["tokens"][b, n[b]].long()
            in_top += int((top == tok[:, None]).any(dim=1).sum())
            rejected += int(b.numel())
    hist = hist.cpu().tolist()
    total = sum(hist)
    return {"mean_al": sum(i * c for i, c in enumerate(hist)) / max(1, total),
            "al_hist": hist[1:], "requests": total,
            "rejections": rejected,
            f"correction_in_draft_top{k}": in_top / max(1, rejected),
            f"speculation_cache_hit_rate_top{k}": hits / max(1, total)}


def run_reference(args):
    """--impl reference: the oracle on the host cores, timed per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch  # noqa: F401  (workload generation)
    from speculative_decoding_verification_lse_b200 import workloads
    w = workloads.make(args.workload, "cpu")
    import oracle
    h = w.host_arrays()
    cores = os.cpu_count() or 1

    def run(sl):
        oracle.verify(h["target"][sl], h["draft"][sl], h["tokens"][sl],
                      None if h["row_D"] is None else h["row_D"][sl], temperature=w.temperature,
                      mode=w.mode, seed=w.seed,
                      temperature_per_req=None if h["temperature_per_req"] is None
                      else h["temperature_per_req"][sl],
                      mode_per_req=None if h["mode_per_req"] is None else h["mode_per_req"][sl],
                      saguaro_k=w.saguaro_k, saguaro_c=w.saguaro_c, nthreads=cores,
                      request_offset=sl.start)

    # a bounded sample per step: one request per core, repeated so that all
    # warm-up and timed steps together take about `ref_seconds`
    t0 = time.perf_counter()
    run(slice(0, 1))
    t_req = time.perf_counter() - t0
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    waves = max(1, int(per_step / max(t_req, 1e-6)))
    nreq = max(1, min(w.B, cores * waves))
    sl = slice(0, nreq)
    rows = sum(d + 1 for d in w.row_D_list()[:nreq])

    def step():
        run(sl)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = rows * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "B": w.B, "D": w.D_max, "V": w.V},
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {nreq} of {w.B} requests ({rows} verified rows) per step"},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    import speculative_decoding_verification_lse_b200 as sv
    from speculative_decoding_verification_lse_b200 import workloads
    from speculative_decoding_verification_lse_b200.sharding import max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    sv.load()
    variant = {"auto": sv.SV_VARIANT_AUTO, "split": sv.SV_VARIANT_SPLIT,
               "split-items": sv.SV_VARIANT_SPLIT | sv.SV_TAIL_ITEMS,
               "split-per-request": sv.SV_VARIANT_SPLIT | sv.SV_TAIL_PER_REQUEST,
               "fused": sv.SV_VARIANT_FUSED, "cluster": sv.SV_VARIANT_CLUSTER,
               "early-exit": sv.SV_VARIANT_EARLY_EXIT}[args.variant]

    # every rank verifies its own batch (its own seed and request range)
    tree = args.workload in workloads.TREE_CONFIGS
    if tree:
        w = workloads.make_tree(args.workload, dev,
                                seed=workloads.TREE_CONFIGS[args.workload]["seed"] + 97 * rank)
    else:
        w = workloads.make(args.workload, dev,
                           seed=workloads.CONFIGS[args.workload]["seed"] + 97 * rank)
    offset = rank * w.B
    stream = torch.cuda.current_stream(dev)
    out = dict(tokens=torch.empty((w.B, w.D_max + 1), dtype=torch.int32, device=dev),
               accept_len=torch.empty((w.B,), dtype=torch.int32, device=dev),
               flags=torch.empty((w.B,), dtype=torch.int32, device=dev))

    def barrier():
        if world > 1:
            dist.barrier()

    # inputs that fit in L2 rotate over copies whose total is at least twice the
    # L2, so that every timed step reads its logits from HBM
    in_bytes = sum(t.numel() * t.element_size() for t in (w.target, w.draft, w.tokens))
    ncopies = input_copies(in_bytes)
    copies = [w]
    if ncopies > 1:
        big = [t.unsqueeze(0).repeat((ncopies,) + (1,) * t.dim()) for t in (w.target, w.draft, w.tokens)]
        copies = [dataclasses.replace(w, target=big[0][c], draft=big[1][c], tokens=big[2][c])
                  for c in range(ncopies)]

    if tree:
        out = None

    def step(i, ev=None):
        if tree:
            c = copies[i % ncopies]
            sv.verify_tree(c.target, c.draft, c.tokens, c.parents, temperature=c.temperature,
                           mode=c.mode, seed=1000 + i, request_offset=offset, stream=stream,
                           timing_events=ev)
            return
        sv.verify_workload(copies[i % ncopies], seed=1000 + i, request_offset=offset,
                           variant=variant, stream=stream, out=out, timing_events=ev)

    # clocks are sampled from the start of the warm-up to the end of a window of
    # untimed steps after the timed region, every step the same call, so that a
    # short timed region still has samples around it
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    clocks.active = True
    t_window = time.perf_counter()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    status = sv.sv_get_device_status(stream)
    if status & sv.SV_FLAG_ERRORS:
        raise RuntimeError(f"device status {status:#x} during warm-up")
    extra = 0
    while time.perf_counter() - t_window < args.clock_window / 2:  # untimed, before
        for _ in range(16):
            step(args.warmup + args.steps + extra)
            extra += 1
        torch.cuda.synchronize()

    # dominant-kernel timing events on every KEV_EVERY-th step of the timed region
    # (a pair on every step would add its own recording cost to the step time)
    kev_steps = list(range(0, args.steps, KEV_EVERY))
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in kev_steps]
    for a_ev, b_ev in kev:  # torch creates the CUDA event on first record
        a_ev.record(stream)
        b_ev.record(stream)
    torch.cuda.synchronize()
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, kev[i // KEV_EVERY] if i % KEV_EVERY == 0 else None)
    t_stop.record(stream)
    torch.cuda.synchronize()
    t_after = time.perf_counter()
    while time.perf_counter() - t_after < args.clock_window / 2:  # untimed, after
        for _ in range(16):
            step(args.warmup + args.steps + extra)
            extra += 1
        torch.cuda.synchronize()
    clocks.active = False
    window_s = time.perf_counter() - t_window
    barrier()
    clocks.stop()
    ms = max_over_ranks(t_start.elapsed_time(t_stop), dev)
    k_list = [a.elapsed_time(b) for a, b in kev]
    k_ms = statistics.mean(k_list)
    k_med = statistics.median(k_list)
    ms_per_step = ms / args.steps
    rows_total = w.verified_rows() * args.steps * world
    graph = None
    if args.graph > 0 and not tree:
        # the same steps captured in a CUDA graph (one per input copy and seed,
        # args.graph of them) and replayed: the per-launch host and dependency
        # costs a decode loop saves by capturing its calls
        K = args.graph
        ws = torch.empty(sv.sv_workspace_bytes(w.B, w.D_max, w.V, w.dtype), dtype=torch.uint8,
                         device=dev)
        gs = torch.cuda.Stream(dev)
        with torch.cuda.stream(gs):
            sv.verify_workload(copies[0], seed=999, out=out, workspace=ws, stream=gs,
                               variant=variant)
        torch.cuda.synchronize()
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=gs):
            for i in range(K):
                sv.verify_workload(copies[i % ncopies], seed=1000 + i, out=out, workspace=ws,
                                   stream=gs, variant=variant)
        reps = max(1, args.steps // K)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(gs):
            for _ in range(3):
                cg.replay()
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            g0.record(gs)
            for _ in range(reps):
                cg.replay()
            g1.record(gs)
        torch.cuda.synchronize()
        gms = max_over_ranks(g0.elapsed_time(g1), dev)
        graph = {"ms_per_step": gms / (reps * K), "steps_per_graph": K, "replays": reps,
                 "value": w.verified_rows() * reps * K * world / (gms / 1e3), "unit": "rows/s"}
        del cg
    ee_rows = None
    if args.variant == "early-exit" and not tree:
        # the rows the timed steps read, from their outcomes (each step again,
        # untimed: the same inputs and seeds give the same outcomes)
        ee_rows = 0
        for i in range(args.steps):
            step(args.warmup + i)
            ee_rows += early_exit_rows(out["accept_len"].cpu().tolist(), w.row_D_list(),
                                       w.modes(), w.D_max)
        ee_rows /= args.steps
    value = rows_total / (ms / 1e3)

    # acceptance: mean AL and its histogram (for saguaro next to the plain rule
    # on the same logits, its draft tokens drawn from q instead of q')
    acceptance = None
    if args.al_seeds > 0 and not tree:
        acceptance = acceptance_stats(sv, w, variant, args.al_seeds, stream)
        if w.mode == sv.SV_SAGUARO:
            wp = workloads.make(args.workload, dev, mode=sv.SV_STOCHASTIC,
                                seed=workloads.CONFIGS[args.workload]["seed"] + 97 * rank)
            acceptance = {"saguaro": acceptance,
                          "plain_rule_same_logits": acceptance_stats(sv, wp, variant, args.al_seeds,
                                                                     stream)}
            del wp

    # end to end through the same call with host buffers: pinned H2D of the
    # step's inputs, the call, D2H of the step's outputs, all in the timed region
    e2e = None
    if args.e2e_steps > 0 and not tree:
        h_t = torch.empty(w.target.shape, dtype=w.target.dtype, pin_memory=True)
        h_q = torch.empty(w.draft.shape, dtype=w.draft.dtype, pin_memory=True)
        h_x = torch.empty(w.tokens.shape, dtype=w.tokens.dtype, pin_memory=True)
        h_t.copy_(w.target)
        h_q.copy_(w.draft)
        h_x.copy_(w.tokens)
        o_t = torch.empty(out["tokens"].shape, dtype=torch.int32, pin_memory=True)
        o_a = torch.empty(out["accept_len"].shape, dtype=torch.int32, pin_memory=True)
        d_t, d_q, d_x = torch.empty_like(w.target), torch.empty_like(w.draft), torch.empty_like(w.tokens)
        # the per-request inputs (ragged draft lengths, modes, temperatures) travel too
        small = {k: getattr(w, k) for k in ("row_D", "temperature_per_req", "mode_per_req")
                 if getattr(w, k) is not None}
        h_small = {k: v.cpu().pin_memory() for k, v in small.items()}
        d_small = {k: torch.empty_like(v) for k, v in small.items()}

        def e2e_step(i):
            d_t.copy_(h_t, non_blocking=True)
            d_q.copy_(h_q, non_blocking=True)
            d_x.copy_(h_x, non_blocking=True)
            for k in d_small:
                d_small[k].copy_(h_small[k], non_blocking=True)
            sv.verify(d_t, d_q, d_x, d_small.get("row_D"), temperature=w.temperature, mode=w.mode,
                      seed=5000 + i, temperature_per_req=d_small.get("temperature_per_req"),
                      mode_per_req=d_small.get("mode_per_req"), saguaro_k=w.saguaro_k,
                      saguaro_c=w.saguaro_c, request_offset=offset, variant=variant, stream=stream,
                      out=out)
            o_t.copy_(out["tokens"], non_blocking=True)
            o_a.copy_(out["accept_len"], non_blocking=True)

        e2e_step(0)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.e2e_steps):
            e2e_step(1 + i)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        h2d = (h_t.numel() * h_t.element_size() + h_q.numel() * h_q.element_size() + h_x.numel() * 4
               + sum(v.numel() * v.element_size() for v in h_small.values()))
        d2h = o_t.numel() * 4 + o_a.numel() * 4
        e2e = {"value": w.verified_rows() * args.e2e_steps * world / (ems / 1e3), "unit": "rows/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / args.e2e_steps}

    status = sv.sv_get_device_status(stream)
    if status & sv.SV_FLAG_ERRORS:
        raise RuntimeError(f"device status {status:#x} after the timed region")

    if rank == 0:
        peak, peak_kind = measured_peak()
        step_bytes = w.algorithmic_bytes()
        used_variant = args.variant if args.variant != "auto" else "split"
        if ee_rows is not None:
            # the bytes the rounds read (the rows up to each request's outcome)
            # and the race's rows; the rounds are the timed kernels
            step_bytes = int(ee_rows * w.V * (2 if w.dtype == 1 else 4))
            kname = "early_exit_rounds"
            kbytes = int((ee_rows - sum(m != 1 for m in w.modes())) * w.V * (2 if w.dtype == 1 else 4))
            ksrc = ["speculative_decoding_verification_lse_b200/csrc/early_exit.cu"]
        elif used_variant in ("fused", "cluster"):
            main = "fused_verify.cu" if used_variant == "fused" else "cluster_verify.cu"
            kname, kbytes = main[:-3], step_bytes
            ksrc = ["speculative_decoding_verification_lse_b200/csrc/" + f
                    for f in (main, "tail_device.cuh", "race_device.cuh", "scan_device.cuh",
                              "stats_device.cuh", "sv_common.cuh", "philox.cuh")]
        else:
            # the statistics pass reads every needed logit row once
            rows_read = 0
            if tree:
                rows_read = w.B * ((w.N + 1) + (0 if w.mode == 1 else len(set(w.parent_list()))))
            for d, m in ([] if tree else zip(w.row_D_list(), w.modes())):
                rows_read += (d + 1) + (0 if m == 1 else d)
            kname, kbytes = "row_stats", rows_read * w.V * (2 if w.dtype == 1 else 4)
            ksrc = ["speculative_decoding_verification_lse_b200/csrc/row_stats.cu",
                    "speculative_decoding_verification_lse_b200/csrc/stats_device.cuh",
                    "speculative_decoding_verification_lse_b200/csrc/sv_common.cuh"]
        achieved = kbytes / (k_ms / 1e3) / 1e9
        tr = traffic_record(kname, ksrc, kbytes)
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "rows/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if w.dtype == 1 else "f32",
            "data": "synthetic",
            "config": {
                "workload": workload_desc(w),
                "B": w.B, "D": w.D_max, "V": w.V,
                "variant": used_variant,
                "l2": (f"inputs {in_bytes / 1e6:.0f} MB > 126 MB L2: no flush between steps"
                       if ncopies == 1 else
                       f"inputs {in_bytes / 1e6:.3f} MB rotated over {ncopies} copies "
                       f"({ncopies * in_bytes / 1e6:.0f} MB >= twice the 126 MB L2): no flush"),
                "parallelism": f"replicas x{world} (request-sharded, no collective)",
            },
            "hbm": {
                "algorithmic_bytes_per_step": step_bytes,
                "achieved_gbs": step_bytes / (ms_per_step / 1e3) / 1e9,
                "frac_of_spec_8000": step_bytes / (ms_per_step / 1e3) / 1e9 / SPEC_HBM_GBS,
                f"frac_of_{peak_kind}_{peak:.0f}": step_bytes / (ms_per_step / 1e3) / 1e9 / peak,
            },
            "roofline": {
                "bound": "hbm",
                "kernel": kname,
                "achieved": achieved,
                "peak": peak,
                "peak_kind": peak_kind,
                "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": None if tr is None else tr[0],
                "algorithmic_bytes_per_launch": kbytes,
                "launch_ms": k_ms,
                "launch_ms_median": k_med,
                "launches_timed": len(k_list),
            },
            "clocks": dict(clocks.summary(), window=(
                f"{window_s:.2f} s from the first warm-up step to {args.clock_window / 2:.2f} s of "
                f"untimed steps after the timed region, every step the same call")),
            # fused: one launch; split: statistics, then one kernel per request or
            # the scan and the race items (the library's rule, in include/specverify.h)
            "gpu_launches": (2 * (len(early_exit_bounds(w.D_max)) - 1) + (
                                 2 if tail_items(w, torch.cuda.get_device_properties(dev).multi_processor_count)
                                 else 1) if ee_rows is not None else
                             2 if tree else 1 if used_variant in ("fused", "cluster") else
                             3 if (used_variant == "split-items" or (used_variant == "split" and tail_items(
                                 w, torch.cuda.get_device_properties(dev).multi_processor_count)))
                             else 2) * args.steps,
            "e2e": e2e,
            "acceptance": acceptance,
        }
        if graph is not None:
            line["graph"] = graph
        if args.cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="b256")
    ap.add_argument("--variant", choices=["auto", "split", "split-items", "split-per-request",
                                          "fused", "cluster", "early-exit"], default="auto")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--graph", type=int, default=0,
                    help="also time the steps captured K at a time in a CUDA graph")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0)
    ap.add_argument("--clock-window", type=float, default=0.8,
                    help="seconds of same-call steps around the timed region while clocks are sampled")
    ap.add_argument("--al-seeds", type=int, default=40,
                    help="verifier seeds for the acceptance statistics (0: skip)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
