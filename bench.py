"""Benchmark: SALA hybrid-attention prefill throughput (tokens/s) at 128K tokens.

One step = one prefill pass of the 8-layer hybrid attention stack (Lightning
layers 0,1,3,4,5,7; sparse layers 2,6), B=1, T=131072, 32 heads (2 KV heads in
the sparse layers), head_dim 128, bf16, through the libsala C ABI:
    Lightning layer: sala_lightning_prefill (chunk 128, fresh zero state)
    sparse layer:    sala_sparse_select (block 64, top-64 + 1 init + 2 local) then
                     sala_sparse_attn (gated)
Inputs are synthetic N(0,1) per layer (seed 1005 + layer), all resident in HBM
(about 39 GB, far larger than L2, so no flush is needed between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU.  Run as is with ``--gpus N`` (N > 1), bench.py
starts the N ranks itself through torch.distributed.run; under torchrun, WORLD_SIZE
must equal N.  Every rank runs its own independent sequence (weak scaling, no
data-path collective); the step time is the max over ranks; value = tokens processed
by all ranks / that time.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only) and reports the whole-step throughput extrapolated from it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Hybrid-attn prefill tokens/s at 128K (lightning+sparse); % of roofline"
# DRAM read + write bytes per launch of a kernel, by T (see the comment where it is used)
NCU_TRAFFIC = {131072: {"attn": 8369097472 + 1124515072}}
B, H, HKV, D = 1, 32, 2, 128
CHUNK, BLOCK, TOPK, N_INIT, N_LOCAL = 128, 64, 64, 1, 2
SPARSE_LAYERS = (2, 6)
NUM_LAYERS = 8


def source_digest() -> str:
    """First 12 hex digits of the sha256 of the CUDA sources and the C header the library
    is built from (the GPU host gets no git history, so this identifies the build)."""
    import glob
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    files = sorted(glob.glob(os.path.join(root, "sparse_attention_long_lightning_b200", "csrc",
                                          "*.cu*")))
    files.append(os.path.join(root, "include", "sala.h"))
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]),
                "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, dist.get_rank(), ws
    torch.cuda.set_device(0)
    return None, 0, 1


def max_over_ranks(dist, seconds, device):
    """Step time of the whole job: the slowest rank's device-timed seconds."""
    if dist is None:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world, tokens_per_rank, seconds_max):
    """Whole-job tokens/s: every rank processes its own sequence of tokens_per_rank."""
    return world * tokens_per_rank / seconds_max


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [s for s in sm if mx is None or s >= 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


class Layer:
    pass


def make_layers(T, device, seed=1005, share=False):
    """The 8 layers with their seeded inputs, outputs and scratch.  With share=True the
    Lightning layers all use the first Lightning layer's buffers and the sparse layers the
    first sparse layer's: at T=1048576 fresh per-layer buffers would need ~310 GB, and the
    kernels' time does not depend on which N(0,1) draw they read."""
    from sparse_attention_long_lightning_b200 import inputs
    import sparse_attention_long_lightning_b200 as sala
    layers = []
    first = {}
    for l in range(NUM_LAYERS):
        kind = l in SPARSE_LAYERS
        if share and kind in first:
            L = Layer()
            L.__dict__.update(first[kind].__dict__)
            L.index = l
            layers.append(L)
            continue
        x = inputs.hybrid_layer_inputs(l, T, B, H, HKV, D, device=device, seed=seed)
        L = Layer()
        L.index, L.sparse = l, l in SPARSE_LAYERS
        L.q, L.k, L.v, L.g = x.q, x.k, x.v, x.g
        L.o = torch.empty_like(x.q)
        if L.sparse:
            L.idx = torch.empty((B, HKV, T, N_INIT + TOPK + N_LOCAL), dtype=torch.int32,
                                device=device)
            # one scratch serves both calls (selection, then the fp16 copy of v)
            L.ws = torch.empty(max(sala.sparse_select_workspace(B, T, H, HKV, D, BLOCK, TOPK),
                                   sala.sparse_attn_workspace(B, T, HKV, D)),
                               dtype=torch.uint8, device=device)
        else:
            L.state = torch.empty((B, H, D, D), dtype=torch.float32, device=device)
            n = sala.lightning_prefill_workspace(B, T, H, D, CHUNK, torch.bfloat16)
            L.ws = torch.empty(max(n, 1), dtype=torch.uint8, device=device)
        first[kind] = L
        layers.append(L)
    return layers


def resident_bytes(layers):
    """Device bytes held by the layers' distinct buffers."""
    seen, n = set(), 0
    for L in layers:
        for t in L.__dict__.values():
            if isinstance(t, torch.Tensor) and t.data_ptr() not in seen:
                seen.add(t.data_ptr())
                n += t.numel() * t.element_size()
    return n


def run_layer(L, sala, events=None):
    """One layer of the stack through the C ABI; optional per-op CUDA events."""
    if L.sparse:
        if events is not None:
            events["sel"][0].record()
        sala.sparse_select(L.q, L.k, topk=TOPK, n_init=N_INIT, n_local=N_LOCAL, block=BLOCK,
                           out=L.idx, workspace=L.ws)
        if events is not None:
            events["sel"][1].record()
            events["attn"][0].record()
        sala.sparse_attn(L.q, L.k, L.v, L.idx, L.g, block=BLOCK, out=L.o, workspace=L.ws)
        if events is not None:
            events["attn"][1].record()
    else:
        if events is not None:
            events["light"][0].record()
        # fresh zero initial state each pass (state=None semantics via init_zero)
        sala.lightning_prefill(L.q, L.k, L.v, L.g, None, chunk=CHUNK, out=L.o, workspace=L.ws)
        if events is not None:
            events["light"][1].record()


def step(layers, sala, ev=None):
    for L in layers:
        run_layer(L, sala, ev)


def sparse_attn_flops(L):
    """Algorithmic flops of one sparse-attention launch: 4*D per (query head, attended key)."""
    T = L.q.shape[1]
    idx = L.idx.long()
    t = torch.arange(T, device=idx.device).view(1, 1, T, 1)
    valid = (idx >= 0) & (idx * BLOCK <= t)
    keys = torch.clamp(t - idx * BLOCK + 1, max=BLOCK)
    keys = torch.where(valid, keys, torch.zeros_like(keys))
    n = keys.sum().item()  # over (b, hk, t): keys per row, shared by the group
    return 4.0 * D * n * (H // HKV)


def count_launches(layers, sala):
    """Kernels of libsala launched by one step (profiled once, outside the timed region)."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        step(layers, sala)
        torch.cuda.synchronize()
    n = 0
    for e in prof.events():
        if e.device_type.name == "CUDA" and "sala::" in e.name:
            n += 1
    return n


ORACLE_SAMPLE = {"light_heads": 16, "light_tokens": 1024, "sparse_rows": 128}


class OracleSample:
    """A bounded, stratified sample of one step for the fp64 oracle on the host cores:
    Lightning over `light_heads` heads x `light_tokens` tokens, and selection + attention
    of the sparse layer for `sparse_rows` rows evenly spaced over [0, T) (both KV heads).
    The inputs are drawn once; time() runs the oracle on the sample and scales each
    part by its share of the full step (6 Lightning layers x 32 heads x T tokens, 2 sparse
    layers x T rows).  The in-bench cpu_baseline and `--impl reference` use this same
    sample."""

    def __init__(self, T):
        from sparse_attention_long_lightning_b200 import inputs
        self.T = T
        nh, nt, nr = (ORACLE_SAMPLE[k] for k in ("light_heads", "light_tokens", "sparse_rows"))
        x = inputs.lightning_inputs(1, nt, nh, D, seed=1005)
        self.light = [t.double().numpy() for t in (x.q, x.k, x.v, x.g)]
        s = inputs.sparse_inputs(1, T, H, HKV, D, seed=1007, gate=True)
        self.k64, self.v64 = s.k.double().numpy(), s.v.double().numpy()
        self.rows = np.unique(np.linspace(0, T - 1, nr).astype(np.int64))
        self.q_rows = s.q[:, self.rows].double().numpy()
        self.g_rows = s.g[:, self.rows].double().numpy()
        self.light_units = nh * nt                  # token-heads in the sample
        self.sparse_units = len(self.rows)          # rows in the sample
        self.light_factor = 6 * H * T / self.light_units
        self.sparse_factor = 2 * T / self.sparse_units
        self.cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
        self.description = (f"Lightning: {nh} heads x {nt} tokens (x{self.light_factor:.0f} to "
                            f"6 layers x {H} heads x {T} tokens); sparse: {len(self.rows)} rows "
                            f"evenly spaced over T={T}, select+attention, 2 KV heads "
                            f"(x{self.sparse_factor:.0f} to 2 layers x {T} rows)")

    def time(self):
        """(seconds the sample took, extrapolated seconds of one full step)."""
        import oracle
        t0 = time.perf_counter()
        oracle.lightning_recurrent(*self.light)
        t1 = time.perf_counter()
        idx, _ = oracle.sparse_select(self.q_rows, self.k64, rows=self.rows, T=self.T)
        oracle.attention(self.q_rows, self.k64, self.v64, self.g_rows, idx=idx, rows=self.rows)
        t2 = time.perf_counter()
        full = (t1 - t0) * self.light_factor + (t2 - t1) * self.sparse_factor
        return t2 - t0, full

    def info(self):
        return {"kind": "oracle", "cores": self.cores, "sample": self.description,
                "extrapolated": True,
                "factor": {"lightning": self.light_factor, "sparse": self.sparse_factor}}


def cpu_baseline(T):
    """Time the fp64 oracle once on the bounded sample and scale it to tokens/s of the
    whole 8-layer stack.  Returns (tok/s, info)."""
    smp = OracleSample(T)
    _, full = smp.time()
    return T / full, smp.info()


def run_reference(args):
    """--impl reference: the fp64 CPU oracle, as it stands, on the bounded sample of the
    workload (rank 0 only; other ranks exit without work).  Each step times the sample
    once; `steps` counts the samples timed and `ms_per_step` is their measured time.  The
    value is the whole-step throughput extrapolated from the sample (marked as such)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    T = args.T
    smp = OracleSample(T)
    sample_s, full_s = [], []
    for i in range(args.warmup + args.steps):
        a, b = smp.time()
        if i >= args.warmup:
            sample_s.append(a)
            full_s.append(b)
    full = float(np.mean(full_s))
    value = T / full
    info = smp.info()
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean(sample_s)) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "extrapolated": {"value_from": "sample", "sample": info["sample"],
                             "factor": info["factor"],
                             "full_step_ms_estimate": full * 1e3,
                             "ms_per_step_is": "measured time of one sample"},
            "config": {"workload": f"SALA hybrid attention prefill, 8 layers (Lightning 0,1,3,4,5,7;"
                                   f" sparse 2,6), B1 T{T} H32 Hkv2 D128",
                       "global_batch": B, "seq_len": T, "parallelism": "cpu"},
            "cpu_baseline": dict(info, value=value, unit="tokens/s"),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def launch_ranks(args):
    """`--gpus N` with N > 1 outside torchrun: start N ranks on this node through
    torch.distributed.run (one process per GPU, rendezvous on 127.0.0.1) and return its
    exit status.  Inside torchrun, WORLD_SIZE must equal N."""
    ws = os.environ.get("WORLD_SIZE")
    if ws is not None:
        if int(ws) != args.gpus:
            sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={ws}\n")
            return 2
        return None
    if args.gpus <= 1:
        return None
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def e2e_measure(layers, sala, steps, stream):
    """Same step through the public API with inputs in pinned host memory: every step
    copies each layer's inputs host->device and its output device->host.  Copies run on
    their own streams, so layer l+1's inputs cross PCIe while layer l computes and layer
    l-1's output comes back; each layer's device buffers are reused only after their
    previous copies and kernels have finished (events)."""
    host_light = [t.cpu().pin_memory() for t in (layers[0].q, layers[0].k, layers[0].v,
                                                 layers[0].g)]
    sp = layers[SPARSE_LAYERS[0]]
    host_sparse = [t.cpu().pin_memory() for t in (sp.q, sp.k, sp.v, sp.g)]
    host_out = [torch.empty_like(L.o, device="cpu").pin_memory() for L in layers]
    h2d = sum(sum(t.numel() * t.element_size() for t in (L.q, L.k, L.v, L.g)) for L in layers)
    d2h = sum(L.o.numel() * L.o.element_size() for L in layers)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(layers)
    ev = lambda: torch.cuda.Event()
    computed = [ev() for _ in range(n)]   # layer l's kernels finished (its inputs are free)
    copied_out = [ev() for _ in range(n)]  # layer l's output is on the host (o is free)
    first = [True]

    def one():
        for l, L in enumerate(layers):
            arrived = ev()
            with torch.cuda.stream(s_in):
                if not first[0]:
                    s_in.wait_event(computed[l])
                src = host_sparse if L.sparse else host_light
                for dst, h in zip((L.q, L.k, L.v, L.g), src):
                    dst.copy_(h, non_blocking=True)
                arrived.record(s_in)
            stream.wait_event(arrived)
            if not first[0]:
                stream.wait_event(copied_out[l])
            with torch.cuda.stream(stream):
                run_layer(L, sala)
                computed[l].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[l])
                host_out[l].copy_(L.o, non_blocking=True)
                copied_out[l].record(s_out)
        first[0] = False

    one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for _ in range(steps):
        one()
    stream.wait_stream(s_out)
    stream.wait_stream(s_in)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps / 1e3, h2d, d2h


def decode_components(dev, hbm):
    """One-token decode steps, timed outside the hybrid-prefill region: the Lightning layer
    (B64 H32 D128, the fp32 state read and written) and the sparse layer (B64 sequences with
    131072-token KV caches, 32q/2kv D128).  Both move far more than L2 per step."""
    import sparse_attention_long_lightning_b200 as sala
    from sparse_attention_long_lightning_b200 import inputs

    def timed(fn, iters=50, warmup=5):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters  # ms

    out = {}
    Bd = 64
    S = inputs.decode_state(Bd, H, D, seed=1003, device=dev)
    q, k, v, g = inputs.decode_tokens(Bd, H, D, seed=1003, step=0, device=dev)
    pos = torch.full((Bd,), 131072, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    ms = timed(lambda: sala.lightning_decode(q, k, v, g, S, pos, out=o))
    nbytes = Bd * H * (2 * D * D * 4 + 5 * D * 2)
    out["lightning_decode_b64"] = {"us": ms * 1e3, "GB/s": nbytes / ms / 1e6,
                                   "frac_hbm": nbytes / ms / 1e6 / hbm}
    del S, q, k, v, g, o
    Tc = 131072
    gen = inputs.generator(1006, dev)
    kc = inputs.randn((Bd, Tc, HKV, D), gen, device=dev)
    vc = inputs.randn((Bd, Tc, HKV, D), gen, device=dev)
    qd = inputs.randn((Bd, H, D), gen, device=dev)
    gd = inputs.randn((Bd, H, D), gen, device=dev)
    kbar = sala.sparse_block_means(kc)
    p_l = [Tc - 1 - 13 * b for b in range(Bd)]
    posd = torch.tensor(p_l, dtype=torch.int32, device=dev)
    n_sel = N_INIT + TOPK + N_LOCAL
    ws = torch.empty(sala.sparse_decode_workspace(Bd, Tc, H, HKV, D, n_sel), dtype=torch.uint8,
                     device=dev)
    od = torch.empty_like(qd)
    ms = timed(lambda: sala.sparse_decode(qd, kc, vc, kbar, posd, gd, topk=TOPK, n_init=N_INIT,
                                          n_local=N_LOCAL, out=od, workspace=ws))
    cand = sum(max(0, p // BLOCK - N_LOCAL - N_INIT + 1) for p in p_l)
    nbytes = cand * HKV * D * 4 + Bd * HKV * n_sel * BLOCK * D * 2 * 2 + 3 * Bd * H * D * 2
    out["sparse_decode_b64_128k"] = {"us": ms * 1e3, "GB/s": nbytes / ms / 1e6,
                                     "frac_hbm": nbytes / ms / 1e6 / hbm}
    err = sala.get_device_error()
    if err:
        raise RuntimeError(f"device error in the decode components: {sala.status_string(err)}")
    return out


def projection_components(dev, hbm, tf_burst):
    """The fused projection GEMM of a Lightning layer (x [16384, 4096] times W [16384,
    4096]^T, QK-norm / RoPE / sigmoid epilogue) against the bf16 tensor peak, and the
    Lightning prefill on prepared operands at T=131072 against HBM (same bytes as the raw
    prefill: qh, kh, gate (fp16) and v read, o written).  Timed alone, outside the hybrid
    step."""
    import sparse_attention_long_lightning_b200 as sala
    from sparse_attention_long_lightning_b200 import inputs

    def timed(fn, iters=10, warmup=3):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters  # ms

    out = {}
    Tp, hidden = 16384, 4096
    gen = inputs.generator(1008, dev)
    x = inputs.randn((1, Tp, hidden), gen, device=dev)
    w = inputs.randn((4 * H * D, hidden), gen, device=dev, scale=hidden ** -0.5)
    outs = sala.lightning_projection(x, w, heads=H, head_dim=D)
    ms = timed(lambda: sala.lightning_projection(x, w, heads=H, head_dim=D, out=outs))
    flops = 2.0 * Tp * hidden * 4 * H * D
    out["lightning_projection_t16k"] = {"ms": ms, "TFLOP/s": flops / ms / 1e9,
                                        "frac_tensor": flops / ms / 1e9 / tf_burst,
                                        "peak": "bf16_tflops (burst, timed alone)"}
    del x, w, outs
    T = 131072
    qh = inputs.randn((1, T, H, D), gen, torch.float16, dev)
    kh = inputs.randn((1, T, H, D), gen, torch.float16, dev)
    v = inputs.randn((1, T, H, D), gen, device=dev)
    gate = inputs.randn((1, T, H, D), gen, device=dev).sigmoid().to(torch.float16)
    o = torch.empty_like(v)
    ws = torch.empty(sala.lightning_prefill_workspace(1, T, H, D, CHUNK), dtype=torch.uint8,
                     device=dev)
    ms = timed(lambda: sala.lightning_prefill_prepared(qh, kh, v, gate, None, out=o,
                                                       workspace=ws))
    nbytes = 5 * T * H * D * 2 + H * D * D * 4
    out["lightning_prefill_prepared"] = {"ms": ms, "GB/s": nbytes / ms / 1e6,
                                         "frac_hbm": nbytes / ms / 1e6 / hbm}
    err = sala.get_device_error()
    if err:
        raise RuntimeError(f"device error in the projection components: {sala.status_string(err)}")
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--T", type=int, default=131072)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the e2e, CPU-baseline and launch-count legs")
    ap.add_argument("--share-buffers", action="store_true",
                    help="one input/output set per layer type (implied for T > 131072)")
    args = ap.parse_args()
    rc = launch_ranks(args)
    if rc is not None:
        return rc
    if args.impl == "reference":
        return run_reference(args)

    import sparse_attention_long_lightning_b200 as sala
    sala.load_library()
    dist, rank, world = _dist()
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm, tf_burst, tf_sust, peak_src = _peaks()
    T = args.T
    shared_bufs = args.share_buffers or T > 131072
    layers = make_layers(T, dev, seed=1005 + 1000 * rank, share=shared_bufs)
    gb = resident_bytes(layers) / 1e9
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        step(layers, sala)
    torch.cuda.synchronize()
    err = sala.get_device_error()
    if err:
        raise RuntimeError(f"device error after warm-up: {sala.status_string(err)}")

    per_op = {k: [] for k in ("light", "sel", "attn")}
    n_ops = {"light": 6, "sel": 2, "attn": 2}

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        start.record(stream)
        for _ in range(args.steps):
            for L in layers:
                if L.sparse:
                    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    run_layer(L, sala, {"sel": (s0, s1), "attn": (a0, a1)})
                    per_op["sel"].append((s0, s1))
                    per_op["attn"].append((a0, a1))
                else:
                    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    run_layer(L, sala, {"light": (l0, l1)})
                    per_op["light"].append((l0, l1))
        end.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    sec = max_over_ranks(dist, start.elapsed_time(end) / 1e3 / args.steps, dev)
    err = sala.get_device_error()
    if err:
        raise RuntimeError(f"device error in timed region: {sala.status_string(err)}")

    op_ms = {k: float(np.mean([a.elapsed_time(b) for a, b in v])) for k, v in per_op.items()}
    value = weak_scaling_value(world, T, sec)

    # roofline of the dominant kernel and component figures
    light_bytes = 5 * B * T * H * D * 2 + B * H * D * D * 4
    sel_bytes = B * T * H * D * 2 + B * T * HKV * D * 2 + B * HKV * T * (N_INIT + TOPK + N_LOCAL) * 4
    attn_flops = sparse_attn_flops(layers[SPARSE_LAYERS[0]])
    comps = {
        "lightning_prefill": {"ms": op_ms["light"], "GB/s": light_bytes / op_ms["light"] / 1e6,
                              "frac_hbm": light_bytes / op_ms["light"] / 1e6 / hbm},
        "sparse_select": {"ms": op_ms["sel"], "GB/s": sel_bytes / op_ms["sel"] / 1e6,
                          "frac_hbm": sel_bytes / op_ms["sel"] / 1e6 / hbm},
        "sparse_attn": {"ms": op_ms["attn"], "TFLOP/s": attn_flops / op_ms["attn"] / 1e9,
                        "frac_tensor": attn_flops / op_ms["attn"] / 1e9 / tf_sust},
    }
    # DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
    # dominant kernels, each from a capture of that one kernel alone (profile_case.py,
    # `-k` one kernel, `-c` a few launches, a few GB on the device), summarised under
    # profiles/.  Set to None when a kernel changes until it is captured again.
    ncu_traffic = NCU_TRAFFIC.get(T, {})
    share = {k: n_ops[k] * op_ms[k] for k in op_ms}
    dom = max(share, key=share.get)
    if dom == "attn":
        roof = {"kernel": "sparse_attn_kernel", "bound": "tensor",
                "achieved": attn_flops / op_ms["attn"] / 1e9, "peak": tf_sust, "unit": "TFLOP/s",
                "traffic": ncu_traffic.get("attn"),
                "peak_source": f"bf16_tflops_sustained ({peak_src})",
                "per_launch": f"{attn_flops:.4e} flop"}
    elif dom == "light":
        roof = {"kernel": "lightning_prefill", "bound": "hbm",
                "achieved": light_bytes / op_ms["light"] / 1e6, "peak": hbm, "unit": "GB/s",
                "traffic": ncu_traffic.get("light"), "peak_source": f"hbm_gbs ({peak_src})",
                "per_launch": f"{light_bytes:.4e} bytes"}
    else:
        roof = {"kernel": "sparse_select", "bound": "hbm",
                "achieved": sel_bytes / op_ms["sel"] / 1e6, "peak": hbm, "unit": "GB/s",
                "traffic": ncu_traffic.get("sel"), "peak_source": f"hbm_gbs ({peak_src})",
                "per_launch": f"{sel_bytes:.4e} bytes"}
    roof["frac"] = roof["achieved"] / roof["peak"]

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "SALA hybrid attention prefill, 8 layers (Lightning 0,1,3,4,5,7; "
                                   f"sparse 2,6), B1 T{T} H32 (sparse: 32q/2kv) D128 bf16",
                       "global_batch": B * world, "seq_len": T,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs (~{gb:.0f} GB resident) far exceed L2; no flush",
                       "buffers": ("one set per layer type, shared by the layers of that type"
                                   if shared_bufs else "fresh seeded inputs per layer"),
                       "chunk": CHUNK, "block": BLOCK, "topk": TOPK, "n_init": N_INIT,
                       "n_local": N_LOCAL},
            "roofline": roof, "components": comps, "clocks": clk.summary(),
            "build": {"sources_sha256": source_digest(), "library": sala.version()}}

    if not args.no_extras:
        line["gpu_launches"] = count_launches(layers, sala) * args.steps
        e2e_sec, h2d, d2h = e2e_measure(layers, sala, args.e2e_steps, stream)
        e2e_sec = max_over_ranks(dist, e2e_sec, dev)
        line["e2e"] = {"value": weak_scaling_value(world, T, e2e_sec), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e2e_sec * 1e3}
        line["components"].update(decode_components(dev, hbm))
        line["components"].update(projection_components(dev, hbm, tf_burst))
        if rank == 0 and world == 1:
            tps, info = cpu_baseline(T)
            line["cpu_baseline"] = dict(info, value=tps, unit="tokens/s")
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
