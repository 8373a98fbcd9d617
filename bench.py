#!/usr/bin/env python
"""Benchmark of the Muon optimizer step on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--impl ours|reference]

One step = one muon_step call over the whole matrix set of the workload: momentum +
norm pass, five Newton-Schulz steps (Gram, polynomial, update launches) and the
apply pass, on seeded synthetic gradients with the shapes of the 3.8B Llama-style
model (168 matrices, 2.82B parameters; inputs larger than L2).  Rank 0 prints one
JSON line.

value      algorithmic Newton-Schulz TFLOP (one triangle of the symmetric products)
           per step x steps, summed over ranks, / the slowest rank's device time of
           the whole steps (CUDA events on the launch stream).
e2e        the same metric when every step also copies the gradients in from pinned
           host memory and the updated weights back out; the step is issued as eight
           calls over layer runs so the copies overlap compute (--e2e-chunks).
roofline   the kernel with the largest share of device time, from per-launch CUDA
           events the library records on its stream during the timed steps.
cpu_baseline  the float64 CPU oracle on a bounded sample of the same workload.
--gpus N>1 runs N independent replicas of the full set (weak scaling): the step has no
data exchange, so there is no collective on the data path.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Muon step ms & NS TFLOP/s (fraction of bf16 tensor peak) per model matrix set, 1 B200"
UNIT = "TFLOP/s"
LR, MU, EPS, NS_STEPS = 0.02, 0.95, 1e-7, 5
E2E_CHUNKS = 8  # calls per step in the end-to-end pipeline (transfers overlap within a step)
WORKLOAD_TEXT = {
    1: "d8: depth-8 GPT, d_model 512, MLP 2048, 48 bf16 matrices",
    2: "d12: depth-12 GPT, d_model 768, MLP 3072, 72 bf16 matrices",
    3: "d24: depth-24 GPT, d_model 1536, MLP 6144, 144 bf16 matrices, heavy-tailed gradient spectrum",
    4: ("llama3p8b: 168 matrices of the 3.8B Llama-style model (28 layers: Wq 3072x3072, Wk/Wv 1024x3072, "
        "Wo 3072x3072, W_fc 12288x3072, W_proj 3072x12288), bf16 params and grads, fp32 momentum"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=4, choices=[1, 2, 3, 4])
    ap.add_argument("--layers", type=int, default=0,
                    help="keep only the first N layers of the set (profiling captures); 0 = all")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--shard", action="store_true",
                    help="split the matrices across ranks (strong scaling, one all-gather of the new "
                         "weights per step) instead of running one replica per rank")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of one captured step (CUDA graph) instead of eager calls; "
                         "per-kernel times then come from an eager pass after the timed region")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=E2E_CHUNKS,
                    help="calls per step in the end-to-end pipeline; with 1 (one call for the whole set) "
                         "the weights' download must end before the next step starts")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lerp", action="store_true", help="interpolation-form momentum (muon_step_ex)")
    ap.add_argument("--weight-decay", type=float, default=0.0, help="decoupled weight decay (muon_step_ex)")
    ap.add_argument("--cautious", action="store_true", help="decay only where update and weight agree in sign")
    ap.add_argument("--normuon", action="store_true",
                    help="NorMuon rescaling of the orthogonalised update (muon_step_ex, beta2 0.95)")
    ap.add_argument("--launch-mode", default="auto", choices=["auto", "phases", "persistent"],
                    help="Newton-Schulz launch form: one launch per phase and step, one persistent launch "
                         "for all steps, or the library's choice by problem size")
    ap.add_argument("--mode", default="bf16", choices=["bf16", "fp32", "fp32_simt"],
                    help="arithmetic of the Newton-Schulz steps: bf16 tensor cores (the method's mode), fp32 "
                         "validation on tensor cores (3xTF32), or fp32 validation on CUDA cores")
    ap.add_argument("--cpu-sample-seconds", type=float, default=15.0)
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def measured_traffic(config, layers):
    """DRAM bytes per launch of each kernel kind from the committed ncu summary, or {}
    when the kernel sources have changed since the capture (or for another workload)."""
    import glob
    import hashlib
    path = os.path.join(ROOT, "profiles", "ncu_traffic_llama3p8b.json")
    if config != 4 or layers or not os.path.exists(path):
        return {}
    with open(path) as f:
        t = json.load(f)
    files = sorted(glob.glob(os.path.join(ROOT, "muon_newton_schulz_06_b200", "csrc", "*.cu")) +
                   glob.glob(os.path.join(ROOT, "muon_newton_schulz_06_b200", "csrc", "*.cuh")) +
                   glob.glob(os.path.join(ROOT, "muon_newton_schulz_06_b200", "csrc", "*.h")))
    h = hashlib.sha256()
    for fn in files:
        h.update(os.path.basename(fn).encode())
        with open(fn, "rb") as fh:
            h.update(fh.read())
    return t["per_full_launch_bytes"] if h.hexdigest() == t.get("csrc_sha256") else {}


# ------------------------------------------------------------------ clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd.insert(1, f"--id={self.gpu_id}")
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle timing

def oracle_sample(config, seconds, device_data=None):
    """Times the float64 oracle step on matrices of layer 0 (then further layers) of the
    workload until `seconds` of CPU time have passed.  Returns (flops, time, names, cores)."""
    import numpy as np

    import oracle
    import synth
    from muon_newton_schulz_06_b200 import cost

    try:
        from threadpoolctl import threadpool_info
        cores = max([int(i.get("num_threads", 1)) for i in threadpool_info() if i.get("user_api") == "blas"] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    specs = synth.config_shapes(config)
    flops, spent, names = 0, 0.0, []
    for idx, spec in enumerate(specs):
        if device_data is not None and idx < len(device_data["G"]):
            g = device_data["G"][idx].float().cpu().numpy()
            m = device_data["M"][idx].cpu().numpy()
            w = device_data["W"][idx].float().cpu().numpy()
        else:
            d = synth.make_matrix_set(config, device="cpu", indices=[idx])
            g, m, w = d["G"][0].float().numpy(), d["M"][0].numpy(), d["W"][0].float().numpy()
        t0 = time.perf_counter()
        oracle.muon_step_matrix(w.astype(np.float64), g, m, lr=LR, mu=MU, nesterov=True, eps=EPS)
        spent += time.perf_counter() - t0
        flops += cost.ns_flops([(spec.rows, spec.cols)], NS_STEPS)["algorithmic"]
        names.append(spec.name)
        if spent >= seconds:
            break
    return flops, spent, names, cores


def run_reference(args):
    rank, _, _ = dist_env()
    if rank != 0:
        return
    import synth
    from muon_newton_schulz_06_b200 import cost
    cfg = args.config
    # each step: the oracle on one Wk-shaped matrix of layer 0 (a bounded sample of the set)
    specs = synth.config_shapes(cfg)
    pick = min(range(len(specs)), key=lambda i: specs[i].rows * specs[i].cols)
    import numpy as np

    import oracle
    d = synth.make_matrix_set(cfg, device="cpu", indices=[pick])
    g, m, w = d["G"][0].float().numpy(), d["M"][0].numpy(), d["W"][0].float().numpy().astype(np.float64)
    for _ in range(args.warmup):
        oracle.muon_step_matrix(w, g, m, lr=LR, mu=MU, nesterov=True, eps=EPS)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        w, m, _ = oracle.muon_step_matrix(w, g, m, lr=LR, mu=MU, nesterov=True, eps=EPS)
    dt = time.perf_counter() - t0
    spec = specs[pick]
    flops = cost.ns_flops([(spec.rows, spec.cols)], NS_STEPS)["algorithmic"] * args.steps
    value = flops / dt / 1e12
    try:
        from threadpoolctl import threadpool_info
        cores = max([int(i.get("num_threads", 1)) for i in threadpool_info() if i.get("user_api") == "blas"] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    sample = f"one {spec.rows}x{spec.cols} matrix ({spec.name}) of the set per step, float64 NumPy oracle"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD_TEXT[cfg], "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ multi-rank plumbing

def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 process if absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank passes its own device time, all get the max."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(work_per_step, steps, world, ms_max):
    """Whole-job rate of `world` replicas that each did `steps` steps of `work_per_step`
    (weak scaling), timed by the slowest rank; in work units per second / 1e12."""
    return work_per_step * steps * world / (ms_max / 1e3) / 1e12


# ------------------------------------------------------------------ our arm

def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    import muon_newton_schulz_06_b200 as mb
    import synth
    from muon_newton_schulz_06_b200 import cost

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    cfg = args.config
    data = synth.make_matrix_set(cfg, device=dev, layers=list(range(args.layers)) if args.layers else None)
    W, G, M = data["W"], data["G"], data["M"]
    shapes = [(s.rows, s.cols) for s in data["specs"]]
    fl = cost.ns_flops(shapes, NS_STEPS)
    eb = cost.elementwise_bytes(shapes)
    torch.cuda.synchronize()

    h = mb.muon_init(local)
    mb.muon_set_launch_mode(h, args.launch_mode)
    stream = torch.cuda.current_stream(dev)
    options, nstate = False, None
    if args.shard:
        from muon_newton_schulz_06_b200.sharded import ShardedMuon
        sm = ShardedMuon(W, device=dev, handle=h)
        W = sm.params
        del M

        def step(grads=G, st=None):
            sm.step(grads, lr=LR, momentum=MU, nesterov=True, ns_steps=NS_STEPS, eps=EPS, mode=args.mode,
                    stream=st or stream)
    else:
        sm = None

        options = args.lerp or args.weight_decay or args.cautious or args.normuon
        nstate = [torch.zeros(min(w.shape), device=dev) for w in W] if args.normuon else None

        def step(grads=G, st=None):
            if options:
                mb.muon_step_ex(h, W, grads, M, lr=LR, momentum=MU, nesterov=True, ns_steps=NS_STEPS, eps=EPS,
                                momentum_form="lerp" if args.lerp else "sgd", weight_decay=args.weight_decay,
                                cautious=args.cautious, normuon_state=nstate, mode=args.mode, stream=st or stream)
            else:
                mb.muon_step(h, W, grads, M, lr=LR, momentum=MU, nesterov=True, ns_steps=NS_STEPS, eps=EPS,
                             mode=args.mode, stream=st or stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    mb.muon_sync(h)
    launches_per_step = mb.muon_last_launch_count(h)

    def barrier():
        if world > 1:
            dist.barrier()

    graph = None
    if args.graph and args.shard:
        raise SystemExit("--graph is for single-replica timing; it is not combined with --shard")
    if args.graph:
        mb.muon_sync(h)
        cap = torch.cuda.Stream(dev)  # capture needs a non-default stream
        cap.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            step(st=cap)
        graph.replay()  # one untimed replay (part of warm-up), on the current stream
        torch.cuda.synchronize()

    # ---------------- device-timed region
    mb.muon_profile_enable(h, graph is None)
    mb.muon_profile_read(h)
    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if gpu_uuid and not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        gpu_uuid = None
    sampler = ClockSampler(gpu_uuid)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    mb.muon_sync(h)
    ms = e0.elapsed_time(e1)
    if graph is not None:
        # per-kernel times from eager steps (library events cannot sit inside the graph)
        mb.muon_profile_enable(h, True)
        mb.muon_profile_read(h)
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
    prof = mb.muon_profile_read(h)
    mb.muon_profile_enable(h, False)
    ms_max = max_over_ranks(ms, world, dev)
    # replicas: every rank does the whole set; sharded: the ranks share one set
    value = replica_throughput(fl["algorithmic"], args.steps, 1 if args.shard else world, ms_max)

    # ---------------- end to end: pinned host gradients in, updated weights out, every step
    # The step is issued as E2E_CHUNKS calls over contiguous runs of matrices of about
    # equal work (one library handle each, as a training loop would bucket its layers),
    # so transfers overlap compute within a step as well as across steps: chunk c's
    # gradients are uploaded on a copy stream while earlier chunks compute (two device
    # gradient buffers alternate between steps), and chunk c's updated weights are
    # downloaded on a second copy stream while later chunks compute.  Chunk c of the next
    # step starts only after that download has read the weights.  Every step still moves
    # its full gradients in and its full weights out inside the timed region.
    e2e = None
    if not args.no_e2e:
        n_chunks = 1 if args.shard else max(1, min(args.e2e_chunks, len(W)))
        bounds = cost.contiguous_chunks(shapes, n_chunks, NS_STEPS)
        hc = [h] if n_chunks == 1 else [mb.muon_init(local) for _ in bounds]
        for x in hc:
            mb.muon_set_launch_mode(x, args.launch_mode)
        g_host = [g.cpu().pin_memory() for g in G]
        w_host = [torch.empty(w.shape, dtype=w.dtype, pin_memory=True) for w in W]
        g_dev = [G, [torch.empty_like(g) for g in G]]
        h2d_bytes = sum(x.numel() * x.element_size() for x in g_host)
        d2h_bytes = sum(x.numel() * x.element_size() for x in w_host)
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        g_ready = [[ev() for _ in bounds] for _ in range(2)]
        g_free = [[ev() for _ in bounds] for _ in range(2)]
        done = [ev() for _ in bounds]
        fetched = [ev() for _ in bounds]

        def chunk_step(c, grads, st):
            a, b = bounds[c]
            if args.shard:
                step(grads, st=st)
            elif options:
                mb.muon_step_ex(hc[c], W[a:b], grads[a:b], M[a:b], lr=LR, momentum=MU, nesterov=True,
                                ns_steps=NS_STEPS, eps=EPS, momentum_form="lerp" if args.lerp else "sgd",
                                weight_decay=args.weight_decay, cautious=args.cautious,
                                normuon_state=nstate[a:b] if nstate is not None else None, mode=args.mode,
                                stream=st)
            else:
                mb.muon_step(hc[c], W[a:b], grads[a:b], M[a:b], lr=LR, momentum=MU, nesterov=True,
                             ns_steps=NS_STEPS, eps=EPS, mode=args.mode, stream=st)

        def upload(k, c):
            a, b = bounds[c]
            with torch.cuda.stream(up):
                for gd, gh in zip(g_dev[k % 2][a:b], g_host[a:b]):
                    gd.copy_(gh, non_blocking=True)
                g_ready[k % 2][c].record(up)

        def download(c):
            a, b = bounds[c]
            with torch.cuda.stream(down):
                down.wait_event(done[c])
                for wh, wd in zip(w_host[a:b], W[a:b]):
                    wh.copy_(wd, non_blocking=True)
                fetched[c].record(down)

        # untimed pass of the chunked step (plans and workspaces of the chunk handles)
        for c in range(n_chunks):
            chunk_step(c, G, stream)
        torch.cuda.synchronize()

        e2 = torch.cuda.Event(enable_timing=True)
        e3 = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e2.record(stream)
        up.wait_event(e2)
        down.wait_event(e2)
        for c in range(n_chunks):
            fetched[c].record(down)
            upload(0, c)
        for k in range(args.steps):
            b = k % 2
            for c in range(n_chunks):
                if k + 1 < args.steps:
                    if k >= 1:
                        up.wait_event(g_free[(k + 1) % 2][c])
                    upload(k + 1, c)
                stream.wait_event(g_ready[b][c])
                stream.wait_event(fetched[c])  # the previous step's weights of this chunk are out
                chunk_step(c, g_dev[b], stream)
                g_free[b][c].record(stream)
                done[c].record(stream)
                download(c)
        for c in range(n_chunks):
            stream.wait_event(fetched[c])
        e3.record(stream)
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e2.elapsed_time(e3), world, dev)
        e2e = {"value": replica_throughput(fl["algorithmic"], args.steps, 1 if args.shard else world, ms_e2e),
               "unit": UNIT, "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
               "ms_per_step": ms_e2e / args.steps, "chunks": n_chunks,
               "overlap": "per chunk of matrices: upload ahead on one copy stream, download right after "
                          "on another, both overlapping the other chunks' compute and the next step"}
        for x in hc:
            if x is not h:
                mb.muon_destroy(x)
        del g_host, w_host, g_dev

    # ---------------- per-kernel roofline
    pk = peaks()
    traffic = measured_traffic(cfg, args.layers)
    kernels = {}
    for kind, (kms, n) in prof.items():
        if n == 0:
            continue
        avg_ms = kms / n
        if kind in ("gram", "poly", "update", "update_apply", "ns_persistent"):
            work = (fl["algorithmic"] if kind == "ns_persistent"
                    else fl["per_launch"]["update" if kind == "update_apply" else kind])
            ach = work / (avg_ms / 1e3) / 1e12
            kernels[kind] = {"bound": "tensor", "ms_per_launch": avg_ms, "launches": n, "achieved": ach,
                             "unit": "TFLOP/s", "work_per_launch": work,
                             "frac": ach / pk["bf16_tflops_sustained"]}
        else:
            work = eb[kind]
            ach = work / (avg_ms / 1e3) / 1e9
            kernels[kind] = {"bound": "hbm", "ms_per_launch": avg_ms, "launches": n, "achieved": ach,
                             "unit": "GB/s", "work_per_launch": work, "frac": ach / pk["hbm_gbs"]}
        kernels[kind]["share"] = kms / max(sum(v[0] for v in prof.values()), 1e-9)
        kernels[kind]["traffic"] = traffic.get(kind)
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    dk = kernels[dom]
    roofline = {"bound": dk["bound"], "kernel": dom, "achieved": dk["achieved"],
                "peak": pk["bf16_tflops_sustained"] if dk["bound"] == "tensor" else pk["hbm_gbs"],
                "peak_kind": ("sustained bf16 (kernel timed inside a long loop), " if dk["bound"] == "tensor"
                              else "copy bandwidth, ") + pk["source"],
                "unit": dk["unit"], "frac": dk["frac"], "traffic": dk["traffic"],
                "traffic_note": "DRAM bytes per launch (ncu, first layer x 28 layers); null if the kernels "
                                "changed since the capture"}
    ns_ms = sum(prof[k][0] for k in ("gram", "poly", "update", "update_apply", "ns_persistent")) / args.steps
    ns_tflops = fl["algorithmic"] / (ns_ms / 1e3) / 1e12 if ns_ms > 0 else None

    # ---------------- CPU oracle on a bounded sample (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops_s, secs, names, cores = oracle_sample(cfg, args.cpu_sample_seconds, data)
        cpu = {"value": flops_s / secs / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"float64 NumPy oracle step on {len(names)} matrices of the set ({', '.join(names)}), "
                         f"{secs:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "strong" if args.shard else "weak", "vs_baseline": None,
            "dtype": "bf16" if args.mode == "bf16" else "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT[cfg] + (f" (first {args.layers} layers only)" if args.layers
                                                          else ""), "matrices": len(shapes),
                       "params": int(eb["numel"]), "ns_steps": NS_STEPS,
                       "coeffs": "quintic (3.4445, -4.7750, 2.0315) every step", "lr": LR, "momentum": MU,
                       **({"options": {"momentum_form": "lerp" if args.lerp else "sgd",
                                       "weight_decay": args.weight_decay, "cautious": args.cautious,
                                       "normuon": args.normuon}} if options else {}),
                       "nesterov": True, "eps": EPS, "launch_mode": args.launch_mode, "mode": args.mode,
                       "l2": "no flush: inputs larger than L2 (%.1f GB of gradients per step)" % (
                           sum(g.numel() * g.element_size() for g in G) / 1e9),
                       "parallelism": ("matrix-sharded, all-gather of new weights" if args.shard else
                                       "replicas" if world > 1 else "single GPU")},
            "ns_tflops_algorithmic": ns_tflops,
            "ns_frac_of_sustained_peak": ns_tflops / pk["bf16_tflops_sustained"] if ns_tflops else None,
            "ns_frac_of_burst_peak": ns_tflops / pk["bf16_tflops"] if ns_tflops else None,
            "ns_tflop_per_step_algorithmic": fl["algorithmic"] / 1e12,
            "ns_tflop_per_step_dense_equivalent": fl["dense_equivalent"] / 1e12,
            "matrices_per_s": len(shapes) * args.steps * (1 if args.shard else world) / (ms_max / 1e3),
            "kernels": kernels, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
            "timing": "CUDA graph replays of one captured step" if graph is not None else "eager calls",
        }
        print(json.dumps(line), flush=True)
    graph = None
    mb.muon_destroy(h)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
