"""Throughput of the Attamba layer forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole prefill hot path on one batch of the inference-mask
workload (B=4, n=4096, d_model=1024, 16 heads x 64, N=16, P=8, L=64, M_test,
bf16): chunk index -> KV-SSM scan (K and V) -> chunk-masked attention, three
C-ABI calls on inputs already resident in HBM.  L2 is flushed between steps
(a 256 MiB write, outside the per-step events).  Each rank runs its own batch
(weak scaling, no collective on the data path); the time is the max over ranks.
``--gpus N`` with N > 1 runs one rank per GPU: started without a launcher, the
script relaunches itself under torch.distributed.run with N processes on this
node (rendezvous on 127.0.0.1); under a launcher, WORLD_SIZE must equal N.
Each timed step is bracketed by two CUDA events on the launching stream (the
scan and the attention are programmatic dependent launches, so nothing is
recorded between the calls); a second pass of the same steps with events
between the calls gives each kernel's time for the roofline.

--impl reference times the CPU oracle (float64 numpy, test infrastructure) on
this host's cores: each step is one head of sequence 0 of the same workload at
its full length (both scans over that head's channels and its dense n x n
attention), the heads taken in turn.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from ssm_compressed_chunked_b200 import workloads as W  # noqa: E402

METRIC = "Attamba layer fwd tokens/s at n=4096,P=8,L=64 bf16"
UNIT = "tokens/s"
CFG = W.BF16_TEST_P8_L64
L2_FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def config_block(cfg, extra=None):
    c = {"workload": cfg.name, "batch": cfg.B, "seq_len": cfg.n, "d_model": cfg.D, "heads": cfg.H,
         "head_dim": cfg.dh, "ssm_state": cfg.N, "chunk": cfg.P, "offset": cfg.offset, "leading_tokens": cfg.L,
         "mask": "M_" + cfg.mode, "seed": cfg.seed, "l2": "flushed between steps (256 MiB write)"}
    if extra:
        c.update(extra)
    return c


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every ~0.5 ms in a thread.

    mark() opens the window whose samples are reported (the timed region)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, gpu_index):
        import threading
        self.samples, self.t_mark = [], None
        self.stop_evt = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            try:  # NVML indexes physical devices: find ours by PCI address
                pr = torch.cuda.get_device_properties(gpu_index)
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: no clock record
            self.nv = None
            return
        self.th = threading.Thread(target=self._run, daemon=True)
        self.th.start()

    def _run(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.0005)

    def mark(self):
        self.t_mark = time.perf_counter()

    def stop(self):
        if self.nv is None:
            return None
        self.stop_evt.set()
        self.th.join(timeout=2)
        win = [x for x in self.samples if self.t_mark is None or x[0] >= self.t_mark]
        if len(win) < 8:  # a very short timed region: widen to the last 0.5 s before it
            win = [x for x in self.samples if self.t_mark is None or x[0] >= self.t_mark - 0.5]
        if not win:
            return None
        reasons = sorted(k for k, bit in self.REASONS.items() if any(r & bit for _, _, r in win))
        return {"sm_mhz": statistics.median(m for _, m, _ in win), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(win), "source": "NVML, 0.5 ms period"}


class nvtx:
    """An NVTX range (torch's binding) around a block, so a timeline tool shows each C-ABI call by name."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()


def source_sha(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "ssm_compressed_chunked_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d or d.get("source_sha") != source_sha(d["sources"]):
        return None
    return d["bytes_per_launch_full"]


def setup_dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_config(cfg, ws, rank):
    """Each rank runs its own batch of the workload (weak scaling): same shapes, its own seed."""
    return W.shrink(cfg, seed=cfg.seed + 1000 * rank) if ws > 1 else cfg


def job_throughput(ws, tokens_per_rank, max_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return ws * tokens_per_rank / (max_ms * 1e-3)


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle (reference arm / baseline)
def oracle_sample(inp, b=0, heads=None):
    """The oracle on the whole of sequence b (all n tokens) for the heads ``heads`` (None: all):
    the float64 scans of K and V over those heads' channels (channels are independent) and the dense
    n x n M_test softmax attention of those heads."""
    from oracle import attention as OA, chunks as OC, mask as OM, ssm as OS
    cfg = inp["cfg"]
    n, dh = cfg.n, cfg.dh
    heads = list(range(cfg.H)) if heads is None else list(heads)
    ch = np.concatenate([np.arange(h * dh, (h + 1) * dh) for h in heads])
    f = lambda t: t.detach().to(torch.float64).numpy()
    st = OC.uniform_starts(n, cfg.P, cfg.offset)
    is_start = OC.is_start_mask(st, n)
    x = f(inp["x"][b])[:, ch]
    K, _ = OS.selective_scan(x, f(inp["dt_k"][b])[:, ch], f(inp["bias_k"])[ch], f(inp["A_k"])[ch],
                             f(inp["B_k"][b]), f(inp["C_k"][b]), is_start)
    V, _ = OS.selective_scan(x, f(inp["dt_v"][b])[:, ch], f(inp["bias_v"])[ch], f(inp["A_v"])[ch],
                             f(inp["B_v"][b]), f(inp["C_v"][b]), is_start)
    M = OM.dense_mask(n, st, cfg.L, cfg.mode)
    hn = len(heads)
    OA.masked_attention(f(inp["q"][b])[:, heads], K.reshape(n, hn, dh), V.reshape(n, hn, dh), M, inp["scale"])


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, ws, rank):
    """Each step is one head of sequence 0 at its full length (n tokens: that head's channels of
    both scans and its dense n x n attention), the heads taken in turn; a step counts n / H tokens."""
    if rank != 0:
        return
    inp = W.make_layer(CFG)
    H = CFG.H
    for k in range(args.warmup):
        oracle_sample(inp, heads=[k % H])
    t0, c0 = time.perf_counter(), time.process_time()
    for k in range(args.steps):
        oracle_sample(inp, heads=[k % H])
    wall, cpu = time.perf_counter() - t0, time.process_time() - c0
    dt = wall / args.steps
    v = (CFG.n / H) / dt
    sample = (f"sequence 0 of the workload at its full length ({CFG.n} tokens), one of its {H} heads per step "
              f"(heads in turn): float64 scans of K and V over that head's {CFG.dh} channels + the dense "
              f"{CFG.n}x{CFG.n} M_test softmax attention of that head; a step counts {CFG.n}/{H} tokens")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(CFG),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": effective_threads(cpu, wall),
                         "cores_available": cpu_cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def effective_threads(cpu_s, wall_s):
    """Average number of host threads busy over a timed region (process CPU time over wall time)."""
    return max(1, int(round(cpu_s / wall_s))) if wall_s > 0 else 1


def cpu_baseline():
    inp = W.make_layer(CFG)
    t0, c0 = time.perf_counter(), time.process_time()
    oracle_sample(inp)
    dt, cpu = time.perf_counter() - t0, time.process_time() - c0
    return {"value": CFG.n / dt, "unit": UNIT, "cores": effective_threads(cpu, dt),
            "cores_available": cpu_cores(), "kind": "oracle",
            "sample": f"sequence 0 of the workload at its full length ({CFG.n} tokens), all {CFG.H} heads, one "
                      f"pass (float64 scans of K and V + dense {CFG.n}x{CFG.n} M_test attention), {dt:.1f} s; "
                      f"tokens/s of one sequence (the batch's {CFG.B} sequences take {CFG.B}x as long)"}


# ------------------------------------------------------------------ decode row
def decode_cache_from_prefill(cfg, dec, g, dev):
    """The decode workload's cache as the library leaves it after a prefill: a synthetic prefill of
    ctx tokens per sequence (keys, values and scan inputs ~ N(0, 1), drawn on the device from a seeded
    generator) handed into a cache of the workload's capacity by attamba_cache_from_prefill.
    Returns the cache's arrays by name."""
    from ssm_compressed_chunked_b200 import attamba as A
    gen = torch.Generator(device=dev).manual_seed(cfg.seed)
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    B, n0, H, dh, N, L = cfg.B, cfg.ctx, cfg.H, cfg.dh, cfg.N, cfg.L
    D = H * dh
    cap = dec["cap"]
    rnd = lambda *shape: torch.randn(*shape, generator=gen, device=dev, dtype=bf)  # noqa: E731
    K, V = rnd(B, n0, H, dh), rnd(B, n0, H, dh)
    x, dtk, dtv = rnd(B * n0, D), rnd(B * n0, D), rnd(B * n0, D)
    bc = [rnd(B * n0, N) for _ in range(4)]
    arrs = {"state": torch.empty(2, B, N, D, dtype=f32, device=dev),
            "Kb": torch.empty(B, H, cap, dh, dtype=bf, device=dev), "Vb": torch.empty(B, H, cap, dh, dtype=bf, device=dev),
            "bpos": torch.zeros(B, cap, dtype=i32, device=dev),
            "Kr": torch.empty(B, H, L, dh, dtype=bf, device=dev), "Vr": torch.empty(B, H, L, dh, dtype=bf, device=dev),
            "nb": torch.zeros(B, dtype=i32, device=dev), "pos": torch.zeros(B, dtype=i32, device=dev)}
    cache = A.Cache(*(arrs[k] for k in ("state", "Kb", "Vb", "bpos", "Kr", "Vr", "nb", "pos")), cfg.P, cfg.offset)
    status = torch.zeros(1, dtype=i32, device=dev)
    A.cache_from_prefill(cache, K, V, x, dtk, dtv, g["bias_k"], g["bias_v"], g["A_k"], g["A_v"], *bc, n0, status)
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item()}"
    del K, V, x, dtk, dtv, bc
    return arrs


def decode_bench(dev, reps=3, batch=None):
    """128 decode steps of the decode workload (B=32, 16384 compressed tokens of context, P=8, L=64)
    on the cache a prefill of the context leaves: tokens/s and the HBM fraction of the whole step
    (cached K/V read + SSM state read/write).  ``batch`` runs the same workload with another batch
    size (a smaller case for profiler captures)."""
    from ssm_compressed_chunked_b200 import attamba as A
    cfg = W.DECODE_CONFIG if batch is None else W.shrink(W.DECODE_CONFIG, B=batch)
    dec = W.make_decode(cfg)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in dec.items()}
    names = ("state", "Kb", "Vb", "bpos", "Kr", "Vr", "nb", "pos")
    pristine = decode_cache_from_prefill(cfg, dec, g, dev)
    torch.cuda.empty_cache()
    work = {k: pristine[k].clone() for k in names}
    cache = A.Cache(*(work[k] for k in names), cfg.P, cfg.offset)
    ws_buf = torch.empty(A.decode_workspace_size(cache), dtype=torch.uint8, device=dev)
    o = torch.empty(cfg.B, cfg.H, cfg.dh, dtype=torch.bfloat16, device=dev)

    def steps():
        for st in range(cfg.steps):
            with nvtx("attamba_decode_step"):
                A.decode_step(cache, g["q"][st], g["x"][st], g["dt_k"][st], g["dt_v"][st], g["bias_k"],
                              g["bias_v"], g["A_k"], g["A_v"], g["B_k"][st], g["C_k"][st], g["B_v"][st], g["C_v"][st],
                              dec["scale"], o, ws_buf)

    times = []
    for rep in range(reps + 1):
        for k in names:
            work[k].copy_(pristine[k])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        steps()
        e1.record()
        torch.cuda.synchronize()
        if rep > 0:
            times.append(e0.elapsed_time(e1))
    ms = float(np.median(times))
    # keys read per step: chunk ends below the window plus the window, for t = ctx .. ctx + steps - 1
    keys = sum((t - cfg.L + 1) // cfg.P + cfg.L for t in range(cfg.ctx, cfg.ctx + cfg.steps)) / cfg.steps
    D = cfg.H * cfg.dh
    step_bytes = cfg.B * cfg.H * keys * cfg.dh * 2 * 2 + 2 * 2 * cfg.B * cfg.N * D * 4
    hbm, _, _, src = peaks()
    per_step = ms / cfg.steps
    gbs = step_bytes / (per_step * 1e-3) / 1e9
    return {"workload": cfg.name, "tokens_per_s": cfg.B * cfg.steps / (ms * 1e-3), "ms_per_step": per_step,
            "steps": cfg.steps, "batch": cfg.B, "context": cfg.ctx, "bytes_per_step": step_bytes,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "peak_source": f"{src} HBM copy", "traffic": ncu_traffic("decode_attn_kernel"),
                         "traffic_kernel": "decode_attn_kernel"},
            "gpu_launches_per_step": 2}


def next_rows_bench(cfg, g, inp, pf, nch, dev, flush, scan_exps, reps=10):
    """The rows built after the hot path, timed on the bench workload's shapes (L2 flushed before each
    launch, median of CUDA-event times on the launching stream): the projection GEMMs, the kept-projection
    scan (one input per SSM), the scan at the pages' state size N = 32, the prefill -> decode handoff, and
    the whole layer with its projections (device-resident x, then x in and y out through pinned host
    memory)."""
    import math
    from ssm_compressed_chunked_b200 import attamba as A

    stream = torch.cuda.current_stream(dev)
    exp_peak = 16 * 148 * 1.965e9
    hbm = peaks()[0]

    def timed(fn):
        ts = []
        for _ in range(reps + 2):
            flush.fill_(3)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(np.median(ts[2:]))  # ms

    T, D, H, dh = cfg.B * cfg.n, cfg.D, cfg.H, cfg.dh
    flat = lambda t: t.reshape(T, -1)
    K2, V2 = torch.empty_like(pf.K), torch.empty_like(pf.V)
    Kc2, Vc2 = torch.empty_like(pf.Kc), torch.empty_like(pf.Vc)
    rows = {}
    # f3: the values SSM reads a second [T, D] input (q's memory stands in for x W_V)
    ms = timed(lambda: A.kv_ssm_scan_u(flat(g["x"]), flat(g["q"]), flat(g["dt_k"]), flat(g["dt_v"]), g["bias_k"],
                                       g["bias_v"], g["A_k"], g["A_v"], flat(g["B_k"]), flat(g["C_k"]), flat(g["B_v"]),
                                       flat(g["C_v"]), pf.index.cu, nch, K2, V2, Kc2, Vc2, pf.status))
    rows["f3_scan_kept_projection"] = {"us": ms * 1e3, "Gexp_s": scan_exps / (ms * 1e-3) / 1e9,
                                       "frac_of_exp_unit": scan_exps / (ms * 1e-3) / exp_peak}
    # f4: N = 32, B / C ~ N(0, 1) and A = -exp(U(log 1, log 16)) like the workload's, drawn here
    gen = torch.Generator().manual_seed(32)
    N2 = 32
    bc = [torch.randn(T, N2, generator=gen).to(torch.bfloat16).to(dev) for _ in range(4)]
    A32 = [(-torch.exp(torch.rand(D, N2, generator=gen) * math.log(16.0))).to(dev) for _ in range(2)]
    ms = timed(lambda: A.kv_ssm_scan(flat(g["x"]), flat(g["dt_k"]), flat(g["dt_v"]), g["bias_k"], g["bias_v"],
                                     A32[0], A32[1], bc[0], bc[1], bc[2], bc[3], pf.index.cu, nch, K2, V2, Kc2, Vc2,
                                     pf.status))
    exps32 = 2.0 * T * D * N2
    rows["f4_scan_N32"] = {"us": ms * 1e3, "Gexp_s": exps32 / (ms * 1e-3) / 1e9,
                           "frac_of_exp_unit": exps32 / (ms * 1e-3) / exp_peak}
    # f2: the cache a prefill of the whole sequence leaves (uniform chunks; L leading tokens)
    L = max(1, cfg.L)
    cap = cfg.n // cfg.P + 2
    bf = torch.bfloat16
    cache = A.Cache(torch.zeros(2, cfg.B, cfg.N, D, device=dev), torch.zeros(cfg.B, H, cap, dh, dtype=bf, device=dev),
                    torch.zeros(cfg.B, H, cap, dh, dtype=bf, device=dev),
                    torch.zeros(cfg.B, cap, dtype=torch.int32, device=dev),
                    torch.zeros(cfg.B, H, L, dh, dtype=bf, device=dev), torch.zeros(cfg.B, H, L, dh, dtype=bf, device=dev),
                    torch.zeros(cfg.B, dtype=torch.int32, device=dev), torch.zeros(cfg.B, dtype=torch.int32, device=dev),
                    cfg.P, cfg.offset)
    Kv, Vv = pf.K.view(cfg.B, cfg.n, H, dh), pf.V.view(cfg.B, cfg.n, H, dh)
    ms = timed(lambda: A.cache_from_prefill(cache, Kv, Vv, flat(g["x"]), flat(g["dt_k"]), flat(g["dt_v"]), g["bias_k"],
                                            g["bias_v"], g["A_k"], g["A_v"], flat(g["B_k"]), flat(g["C_k"]),
                                            flat(g["B_v"]), flat(g["C_v"]), cfg.n, pf.status))
    nb = int(cache.nb[0].item())
    hbytes = cfg.B * ((nb + min(L, cfg.n)) * 2 * D * 2 * 2 + 2 * cfg.N * D * 4 + cfg.P * (3 * D * 2 + 4 * cfg.N * 2))
    rows["f2_cache_from_prefill"] = {"us": ms * 1e3, "bytes": hbytes, "GB_s": hbytes / (ms * 1e-3) / 1e9,
                                     "frac_of_hbm": hbytes / (ms * 1e-3) / 1e9 / hbm,
                                     "note": "launch-bound at this size (a few MB)"}
    # f1: the layer's seven input projections as one GEMM (q | dt_K | dt_V | B_K | C_K | B_V | C_V, random-init
    # weights of the workload's shapes), and the output projection
    tf_burst = peaks()[1]
    widths = [H * dh, D, D, cfg.N, cfg.N, cfg.N, cfg.N]
    W_in = (torch.randn(sum(widths), D, generator=gen) / math.sqrt(D)).to(bf).to(dev)
    outs, c = [], 0
    for w in widths:
        outs.append((torch.empty(T, w, dtype=bf, device=dev), c))
        c += w
    ms_in = timed(lambda: A.proj_gemm(flat(g["x"]), W_in, outs, pf.status))
    W_O = (torch.randn(D, H * dh, generator=gen) / math.sqrt(D)).to(bf).to(dev)
    y = torch.empty(T, D, dtype=bf, device=dev)
    ms_o = timed(lambda: A.proj_gemm(pf.O.view(T, H * dh), W_O, [(y, 0)], pf.status))
    fl_in, fl_o = 2.0 * T * sum(widths) * D, 2.0 * T * D * H * dh
    rows["f1_projection_gemm"] = {
        "inputs": {"us": ms_in * 1e3, "TFLOP_s": fl_in / (ms_in * 1e-3) / 1e12,
                   "frac_of_bf16_burst": fl_in / (ms_in * 1e-3) / 1e12 / tf_burst},
        "output": {"us": ms_o * 1e3, "TFLOP_s": fl_o / (ms_o * 1e-3) / 1e12,
                   "frac_of_bf16_burst": fl_o / (ms_o * 1e-3) / 1e12 / tf_burst},
        "traffic_inputs": ncu_traffic("proj_gemm_kernel")}

    # the layer with its projections: x -> the seven input projections (one GEMM) -> chunk_index,
    # kv_ssm_scan, chunk_attn_fwd -> W_O.  Timed with x resident, then end to end with x copied in from
    # pinned host memory and y copied back every step (copies on streams of their own, two x buffers,
    # so step k + 1's x crosses PCIe while step k computes)
    from ssm_compressed_chunked_b200 import layer
    weights = {name: blk for name, blk in zip(layer.INPUT_PROJECTIONS, torch.split(W_in, widths, dim=0))}
    weights.update(W_O=W_O, bias_k=g["bias_k"], bias_v=g["bias_v"], A_k=g["A_k"], A_v=g["A_v"])
    lay = layer.Layer(cfg.B, cfg.n, D, H, dh, cfg.N, weights, cfg.P, cfg.offset, cfg.L, layer.mode_code(cfg.mode),
                      inp["scale"], device=dev)
    y = lay.y

    def layer_fwd(xs):
        lay.forward(xs)

    ms_layer = timed(lambda: layer_fwd(flat(g["x"])))
    h_x = inp["x"].reshape(T, D).pin_memory()
    h_y = torch.empty(T, D, dtype=bf).pin_memory()
    xs = [flat(g["x"]), torch.empty_like(flat(g["x"]))]
    cp_in, cp_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def layer_e2e(n_steps):
        ev_comp = [torch.cuda.Event() for _ in range(n_steps)]
        ev_out = [torch.cuda.Event() for _ in range(n_steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(cp_in)
        for k in range(n_steps):
            if k >= 2:
                cp_in.wait_event(ev_comp[k - 2])
            with torch.cuda.stream(cp_in):
                xs[k & 1].copy_(h_x, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(cp_in)
            stream.wait_event(ev_in)
            if k >= 1:
                stream.wait_event(ev_out[k - 1])
            layer_fwd(xs[k & 1])
            ev_comp[k].record(stream)
            cp_out.wait_event(ev_comp[k])
            with torch.cuda.stream(cp_out):
                h_y.copy_(y, non_blocking=True)
            ev_out[k].record(cp_out)
        t1.record(cp_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n_steps

    layer_e2e(2)
    ms_e2e = layer_e2e(reps)
    rows["layer_incl_projections"] = {
        "us": ms_layer * 1e3, "tokens_per_s": T / (ms_layer * 1e-3),
        "e2e_tokens_per_s": T / (ms_e2e * 1e-3), "h2d_bytes_per_step": T * D * 2, "d2h_bytes_per_step": T * D * 2,
        "note": "x in, y = O W_O out; random-init projection weights of the workload's shapes"}
    assert pf.status.item() == 0 and lay.status.item() == 0, \
        f"device status {pf.status.item()}, layer {lay.status.item()}"
    return rows


# ------------------------------------------------------------------ CUDA path
def run_ours(args, ws, rank, local):
    from ssm_compressed_chunked_b200 import attamba as A, layer

    dev = torch.device("cuda", local)
    cfg = rank_config(CFG, ws, rank)
    inp = W.make_layer(cfg)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    nch = layer.n_chunks_of(cfg)
    pf = layer.Prefill(cfg.B, cfg.n, cfg.D, cfg.H, cfg.dh, cfg.N, nch, torch.bfloat16, dev)
    mode = layer.mode_code(cfg.mode)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(events=None, src=None):
        """One step: chunk_index, kv_ssm_scan, chunk_attn_fwd on the inputs `src` (default: the
        resident set).  Two events bracket the step; four also split it per call (an event between two
        calls keeps the second call's launch from overlapping the first call's tail, so the split sums
        to a little more than the step).  Each C-ABI call sits in an NVTX range of its name."""
        src = g if src is None else src
        if events:
            events[0].record(stream)
        with nvtx("attamba_chunk_index"):
            pf.index_step(None, cfg.P, cfg.offset, cfg.L, mode)
        if events and len(events) == 4:
            events[1].record(stream)
        with nvtx("attamba_kv_ssm_scan"):
            pf.scan_step(src["x"], src["dt_k"], src["dt_v"], g["bias_k"], g["bias_v"], g["A_k"], g["A_v"],
                         src["B_k"], src["C_k"], src["B_v"], src["C_v"])
        if events and len(events) == 4:
            events[2].record(stream)
        with nvtx("attamba_chunk_attn_fwd"):
            pf.attn_step(src["q"], inp["scale"])
        if events:
            events[-1].record(stream)

    sampler = ClockSampler(local) if rank == 0 else None
    t_w = time.perf_counter()
    nw = 0
    while nw < max(3, args.warmup) or (time.perf_counter() - t_w) * 1e3 < args.min_warmup_ms:
        flush.fill_(1)
        step()
        nw += 1
        if nw % 16 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()

    # algorithmic work of one step
    T, D, N, H, dh = cfg.B * cfg.n, cfg.D, cfg.N, cfg.H, cfg.dh
    ls = pf.index.ls.cpu().numpy().astype(np.int64)
    nbb = pf.index.nbb.cpu().numpy().astype(np.int64)
    i = np.tile(np.arange(cfg.n), cfg.B)
    keys = int((nbb + np.maximum(0, i - ls + 1)).sum())
    attn_flops = 4.0 * dh * H * keys
    scan_bytes = T * (5 * D * 2 + 4 * N * 2) + 2 * nch * D * 2
    scan_exps = 2.0 * T * D * N
    index_bytes = T * 8 + nch * 8

    # timed region: K steps, each bracketed by two events on the launching stream (the L2 flush
    # between steps lies outside them)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        step(evs[k])
    torch.cuda.synchronize()
    barrier(ws)
    clocks = sampler.stop() if sampler else None
    step_ms = np.array([evs[k][0].elapsed_time(evs[k][1]) for k in range(args.steps)])
    ms = max_over_ranks(float(step_ms.mean()), ws)
    value = job_throughput(ws, T, ms)

    # per-call split (roofline of each kernel): the same K steps again with events between the calls
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        step(evk[k])
    torch.cuda.synchronize()
    per = np.array([[evk[k][j].elapsed_time(evk[k][j + 1]) for j in range(3)] for k in range(args.steps)])  # ms

    # end to end through the public API with host buffers: every step copies its activations in from
    # pinned host memory and its output back.  The copies run on streams of their own and two device
    # input sets alternate, so step k + 1's inputs cross PCIe while step k computes and its output
    # returns (the order a serving loop runs them in); the time is from the first copy in to the last
    # copy out.
    names = ["x", "q", "dt_k", "dt_v", "B_k", "C_k", "B_v", "C_v"]
    host = {k: inp[k].pin_memory() for k in names}
    h_out = torch.empty(pf.O.shape, dtype=pf.O.dtype).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = h_out.numel() * h_out.element_size()
    sets = [{k: g[k] for k in names}, {k: torch.empty_like(g[k]) for k in names}]
    cp_in, cp_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n_steps):
        ev_in = [torch.cuda.Event() for _ in range(n_steps)]
        ev_comp = [torch.cuda.Event() for _ in range(n_steps)]
        ev_out = [torch.cuda.Event() for _ in range(n_steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(cp_in)
        for k in range(n_steps):
            src = sets[k & 1]
            if k >= 2:
                cp_in.wait_event(ev_comp[k - 2])     # step k - 2 has finished reading this input set
            with torch.cuda.stream(cp_in):
                for n_ in names:
                    src[n_].copy_(host[n_], non_blocking=True)
            ev_in[k].record(cp_in)
            stream.wait_event(ev_in[k])
            if k >= 1:
                stream.wait_event(ev_out[k - 1])     # step k - 1's output has been copied out
            step(src=src)
            ev_comp[k].record(stream)
            cp_out.wait_event(ev_comp[k])
            with torch.cuda.stream(cp_out):
                h_out.copy_(pf.O, non_blocking=True)
            ev_out[k].record(cp_out)
        t1.record(cp_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(2)
    e2e_steps = max(3, min(args.steps, 10))
    barrier(ws)
    e2e_ms = max_over_ranks(e2e_run(e2e_steps) / e2e_steps, ws)
    e2e_value = job_throughput(ws, T, e2e_ms)
    # the last output matches the resident-input step's (same inputs, same kernels)
    o_e2e = h_out.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(o_e2e, pf.O.cpu()), "end-to-end output differs from the resident-input step"

    assert pf.status.item() == 0, f"device status {pf.status.item()}"
    if rank != 0:
        return

    hbm, tf_burst, _, src = peaks()
    mean = per.mean(axis=0)  # ms per launch: index, scan, attention
    kernels = {
        "chunk_index": {"ms": mean[0], "bytes": index_bytes},
        "kv_ssm_scan": {"ms": mean[1], "bytes": scan_bytes, "exps": scan_exps},
        "chunk_attn_fwd": {"ms": mean[2], "flops": attn_flops},
    }
    for k, d in kernels.items():
        d["share"] = d["ms"] / mean.sum()
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    d = kernels[dom]
    exp_peak = 16 * 148 * 1.965e9  # ex2 per second: 16 per clock per SM, 148 SMs, 1965 MHz
    if dom == "kv_ssm_scan":
        ach = d["exps"] / (d["ms"] * 1e-3) / 1e9
        roof = {"bound": "alu", "achieved": ach, "peak": exp_peak / 1e9, "unit": "Gexp/s", "frac": ach / (exp_peak / 1e9),
                "peak_source": "multi-function unit: 16 ex2/clk/SM x 148 SMs x 1965 MHz (derived; 15.9/clk/SM measured)",
                "hbm_frac": d["bytes"] / (d["ms"] * 1e-3) / 1e9 / hbm}
        roof["traffic"] = ncu_traffic("kv_ssm_scan_kernel")
    elif dom == "chunk_attn_fwd":
        ach = d["flops"] / (d["ms"] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tf_burst, "unit": "TFLOP/s", "frac": ach / tf_burst,
                "peak_source": f"{src} bf16 burst"}
        roof["traffic"] = ncu_traffic("chunk_attn_bf16_kernel")
    else:
        ach = d["bytes"] / (d["ms"] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "peak_source": f"{src} HBM copy"}
        roof["traffic"] = ncu_traffic("kv_ssm_scan_kernel" if dom == "kv_ssm_scan" else "chunk_index_kernel")
    roof["kernel"] = dom
    scan = kernels["kv_ssm_scan"]
    # each kernel's binding bound: the slowest of its algorithmic bytes at the HBM copy rate, its
    # exponentials at 16/clk/SM, its FMA-pipe work at 128 lanes/clk/SM (3 per scan exponential) and
    # its tensor flops at the bf16 burst peak; the hot path's fraction is their sum over the step
    fma_rate = 128 * 148 * 1.965e9
    attn_bytes = T * D * 2 * 4 + 2 * nch * D * 2   # q, K, V read and O written once, chunk-end rows Kc, Vc
    limits = {
        "chunk_index": {"hbm": index_bytes / (hbm * 1e9)},
        "kv_ssm_scan": {"hbm": scan_bytes / (hbm * 1e9), "exp": scan_exps / exp_peak, "fma": 3 * scan_exps / fma_rate},
        "chunk_attn_fwd": {"hbm": attn_bytes / (hbm * 1e9), "exp": attn_flops / (4 * dh) / exp_peak,
                           "tensor": attn_flops / (tf_burst * 1e12)},
    }
    hot = {}
    for k, lim in limits.items():
        b = max(lim, key=lim.get)
        hot[k] = {"bound": b, "bound_us": round(lim[b] * 1e6, 2), "measured_us": round(kernels[k]["ms"] * 1e3, 2),
                  "frac": round(lim[b] / (kernels[k]["ms"] * 1e-3), 4)}
    sum_bound = sum(v["bound_us"] for v in hot.values())
    hot_path = {"kernels": hot, "sum_bound_us": round(sum_bound, 2), "step_us": round(ms * 1e3, 2),
                "frac": round(sum_bound / (ms * 1e3), 4)}
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) input, random-init projections)",
        "config": config_block(cfg, {"parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"}),
        "roofline": roof,
        "kernels": {k: {"ms": round(v["ms"], 5), "share": round(v["share"], 4)} for k, v in kernels.items()},
        "scan_exp_rate": {"achieved_Gexp_s": scan["exps"] / (scan["ms"] * 1e-3) / 1e9,
                          "mufu_peak_Gexp_s": exp_peak / 1e9,
                          "frac": scan["exps"] / (scan["ms"] * 1e-3) / exp_peak,
                          "hbm_frac": scan["bytes"] / (scan["ms"] * 1e-3) / 1e9 / hbm},
        "attn_tensor": {"achieved_TFLOP_s": attn_flops / (mean[2] * 1e-3) / 1e12,
                        "frac_of_burst": attn_flops / (mean[2] * 1e-3) / 1e12 / tf_burst},
        "hot_path_bound": hot_path,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if ws == 1 and not args.no_decode:
        out["decode"] = decode_bench(dev, batch=args.decode_batch)
        torch.cuda.empty_cache()   # the decode caches go back to the driver before the next rows
    if ws == 1 and not args.no_next_rows:
        out["next_rows"] = next_rows_bench(cfg, g, inp, pf, nch, dev, flush, scan_exps)
    if ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    print(json.dumps(out), flush=True)


def relaunch_ranks(n):
    """Run this script as n ranks on this node (torch.distributed.run, rendezvous on 127.0.0.1 at a
    free port); returns the launcher's exit status."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-row measurement")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip timing the rows built after the hot path (kept projections, N = 32, handoff)")
    ap.add_argument("--min-warmup-ms", type=float, default=500.0,
                    help="keep warming up at least this long so clocks have ramped (0 under a profiler)")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode row and print it (a profiler capture of the decode kernels)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="batch size of the decode row (default: the workload's 32)")
    args = ap.parse_args()
    if args.gpus < 1:
        raise SystemExit("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: run this same command under torch.distributed.run with N ranks
        sys.exit(relaunch_ranks(args.gpus))
    if int(os.environ.get("WORLD_SIZE", "1")) != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={os.environ.get('WORLD_SIZE')}: launch one rank per GPU")
    if args.decode_only:
        torch.cuda.set_device(0)
        print(json.dumps({"decode": decode_bench(torch.device("cuda", 0), batch=args.decode_batch)}), flush=True)
        return
    if args.impl == "reference":
        # the CPU oracle needs no process group: rank 0 times it, other ranks exit without work
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    ws, rank, local = setup_dist()
    try:
        run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
