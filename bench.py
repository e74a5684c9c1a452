"""Benchmark of the decode hot path: GQA attention over the static KV cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config ragged|single|long2048|long1024|prefill] [--mode aware|masked]

A step is one pass of the whole decode path over one batch: for each of the
36 layers, RoPE on the new q/k rows with the delta write into that layer's
static cache, then split-KV decode attention (with its log-sum-exp merge).
The default workload is the ragged decode batch: 32 requests, T = 512,
valid lengths uniform in [40, 511] before the append (41..512 rows read),
K/V with 1% x8 row outliers, 36 independent layers (604 MB of caches, larger
than the 126 MB L2, so every step streams from HBM).

Timing: W untimed warm-up steps, then exactly K steps replayed from one CUDA
graph, bracketed by a barrier and a device synchronisation, timed with CUDA
events on the launching stream; max over ranks.  Rank 0 prints one JSON line.
Multi-GPU runs are independent replicas (weak scaling, no collective on the
data path).

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (the oracle is the only reference implementation there is).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attn KV GB/s & tokens·layers/s (1×B200); % of HBM roofline"
FALLBACK_HBM_GBS = 6650.0
N_LAYERS = 36

# Per-launch DRAM traffic of the decode kernel from an ncu capture, keyed by the
# sha256 of the kernel source it was taken on; reported as null once the source
# has changed.
DECODE_TRAFFIC = {
    # ncu, one call of the ragged decode workload: decode_kernel (--set full) plus
    # merge_kernel (dram bytes), read + write (see profiles/)
    "79d6a2dbdddefa6947b568ea05b6e92b19c54f1d75f952faafdef48dae35a988":
        329.755392e6 + 4.086016e6 + 13.198848e6 + 0,
}


# Per-launch DRAM traffic of the prefill kernel (one layer of the coalesced
# prefill workload) from an ncu --set full capture, keyed the same way.
PREFILL_TRAFFIC = {
    # one 16-layer launch of the coalesced prefill (read 332.35 MB + write 185.23 MB) / 16
    "2c8173635d520a21840a02bbb4ccc3d051ffc242c7595b1d02691730f9a13e6c": (332.350976e6 + 185.234688e6) / 16,
}


# Per-launch DRAM traffic of the projection kernel (one layer) from ncu --set full
# captures of the two projection workloads, keyed by source hash and workload.
QKV_TRAFFIC = {
    # the 3-stage instantiation (many tiles); the 6-stage split-K instantiation used for a decode
    # step has not been captured since it changed, so that workload reports null
    ("cde2e14ac2c31091a231005ee3800a1c5b6ed3f7342cfb4061ca0ee650e6b0ef", "qkv_prefill"): 36.077568e6 + 0.54272e6,
}


# Per-launch DRAM traffic of the encoder attention kernel (one layer of the encoder batch)
# from an ncu --set full capture, keyed the same way.
ENCODER_TRAFFIC = {
    "c9a95e526155cc2b96648ff6961d41d4db8aa6cb1fc2d46f91b176f748b1f761": 64.04736e6 + 2.65472e6,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="ragged",
                    choices=["ragged", "single", "long2048", "long1024", "prefill", "encoder", "qkv_decode",
                             "qkv_prefill"])
    ap.add_argument("--mode", default="aware", choices=["aware", "masked"])
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="cache format of the decode configurations: bf16, or fp8 E4M3 codes with per-head scales")
    ap.add_argument("--max-splits", type=int, default=8)
    ap.add_argument("--per-layer", action="store_true",
                    help="issue the single-layer calls layer by layer instead of the layer-batched calls")
    ap.add_argument("--rope-on-load", action="store_true",
                    help="prefill: K/V-only append, RoPE applied by the prefill kernel as it loads q")
    ap.add_argument("--layers", type=int, default=None,
                    help="encoder / qkv: layers per step (default 32 / 36; fewer only for profiler captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def make_workload(name: str, layers: int, device: str):
    from gqa_attention_static_b200 import workloads as W
    if name == "ragged":
        b = W.cfg_ragged_decode(layers=layers, device=device)
        desc = "ragged decode B=32 T=512 kv_len U[41,512] 1% x8 K/V row outliers, 36 layers"
    elif name == "single":
        b = W.cfg_single_decode(layers=layers, device=device)
        desc = "single decode B=1 T=512 kv_len 65, 36 layers"
    elif name == "long2048":
        b = W.cfg_long_decode(layers=layers, T=2048, device=device)
        desc = "long decode B=32 T=2048 kv_len U[1501,2048], 36 layers"
    else:
        b = W.cfg_long_decode(layers=layers, T=1024, device=device)
        desc = "long decode B=32 T=1024 full (kv_len 1024), 36 layers"
    return b, desc


def algorithmic_bytes(kv_len, B: int, kv: str = "bf16") -> int:
    """Decode attention per layer: K+V rows read (1024 B per position for the
    2 KV heads, 512 B for an fp8 cache) + q read (4096 B) + o written (4096 B),
    per request."""
    per_pos = 512 if kv == "fp8" else 1024
    return int(sum(int(x) for x in kv_len) * per_pos + B * 8192)


def fp8_cache_for(batch, mode: str):
    """fp8 caches (e4m3 codes, per-head scales) for a decode workload: valid
    rows before each request's cache_position, garbage after it (NaN codes for
    the length-aware mode, large finite codes for the masked one)."""
    from gqa_attention_static_b200 import workloads as W
    return W.make_fp8_cache(1000 + batch.B, batch.B, batch.T, batch.pos0, layers=batch.layers,
                            garbage="big" if mode == "masked" else "nan")


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's device time: every rank runs the same replica
    workload, so the job takes as long as its slowest GPU."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job GB/s of N independent replicas (weak scaling): the bytes all
    ranks processed over the slowest rank's time."""
    return bytes_per_rank * world / (ms_max * 1e-3) / 1e9


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def src_hash(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
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
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


class OracleRunner:
    """The fp64 oracle (as it stands) on this host's cores: whole decode
    layer-steps (RoPE + delta write + attention) over a bounded sample of the
    workload's layers.  OpenMP threads = all host cores."""

    def __init__(self, workload: str, mode: str, layers: int = 4, kv: str = "bf16"):
        import numpy as np
        import torch
        cores = os.cpu_count() or 1
        os.environ.setdefault("OMP_NUM_THREADS", str(cores))
        import oracle
        oracle.build()
        self.oracle = oracle
        self.cores = oracle.num_threads()
        batch, self.desc = make_workload(workload, layers, "cpu")

        def bits(x):
            return x.contiguous().view(torch.int16).numpy().view(np.uint16)

        self.fp8 = (kv == "fp8")
        if self.fp8:
            fc = fp8_cache_for(batch, mode)
            self.inputs = [(bits(batch.q[l]), bits(batch.k_new[l]), bits(batch.v_new[l]),
                            fc.cache_k[l].numpy(), fc.cache_v[l].numpy(), fc.k_scale[l].numpy(),
                            fc.v_scale[l].numpy()) for l in range(layers)]
            self.desc = self.desc.replace(" 1% x8 K/V row outliers", "") + ", fp8 E4M3 cache"
        else:
            self.inputs = [(bits(batch.q[l]), bits(batch.k_new[l]), bits(batch.v_new[l]),
                            bits(batch.cache_k[l]), bits(batch.cache_v[l])) for l in range(layers)]
        self.pos0 = batch.pos0.numpy()
        self.n_new = batch.n_new.numpy()
        self.kv = batch.kv_len.numpy()
        self.B = batch.B
        self.static = (mode == "masked")
        self.bytes_per_layer = algorithmic_bytes(self.kv, self.B, kv)
        self.i = 0

    def layer_step(self):
        x = self.inputs[self.i % len(self.inputs)]
        self.i += 1
        if self.fp8:
            q, kn, vn, ck, cv, ks, vs = x
            qr, ck2, cv2, _ = self.oracle.append_rope_fp8(q, kn, vn, ck, cv, ks, vs, self.pos0, self.n_new)
            self.oracle.decode_fp8(qr, ck2, cv2, ks, vs, self.kv, 1.0 / math.sqrt(128), static_mode=self.static)
            return
        q, kn, vn, ck, cv = x
        qr, ck2, cv2, _ = self.oracle.append_rope(q, kn, vn, ck, cv, self.pos0, self.n_new)
        self.oracle.decode(qr, ck2, cv2, self.kv, 1.0 / math.sqrt(128), static_mode=self.static)

    def timed(self, seconds: float = 0.0, min_layers: int = 1):
        n = 0
        t0 = time.perf_counter()
        while True:
            self.layer_step()
            n += 1
            el = time.perf_counter() - t0
            if n >= min_layers and el >= seconds:
                return n, el


def cpu_baseline(workload: str, seconds: float, mode: str, kv: str = "bf16"):
    r = OracleRunner(workload, mode, kv=kv)
    r.timed(0.0, 1)   # warm
    n, el = r.timed(seconds, 1)
    return {"value": r.bytes_per_layer * n / el / 1e9, "unit": "GB/s", "cores": r.cores, "kind": "oracle",
            "sample": f"{n} layer-steps (4 distinct layers of: {r.desc}) in {el:.1f} s; fp64; OpenMP over "
                      f"(request, head); GB/s by the same algorithmic-byte count as the GPU line",
            "tokens_layers_per_s": r.B * n / el}


class EncoderOracleRunner:
    """The fp64 oracle's encoder attention on this host's cores over a bounded
    sample: one clip of the encoder batch per step (clips cycled, 4 layers)."""

    def __init__(self, layers: int = 4):
        import numpy as np
        import torch
        cores = os.cpu_count() or 1
        os.environ.setdefault("OMP_NUM_THREADS", str(cores))
        import oracle
        from gqa_attention_static_b200 import workloads as W
        oracle.build()
        self.oracle = oracle
        self.cores = oracle.num_threads()
        e = W.cfg_encoder(layers=layers)
        bits = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
        self.items = [(bits(e.q[l][b:b + 1]), bits(e.k[l][b:b + 1]), bits(e.v[l][b:b + 1]),
                       e.length[b:b + 1].numpy()) for l in range(layers) for b in range(e.B)]
        self.scale = 1.0 / math.sqrt(W.ENC_HEAD_DIM)
        self.i = 0
        self.flops = 0

    def step(self):
        q, k, v, n = self.items[self.i % len(self.items)]
        self.i += 1
        self.oracle.attention_bidir(q, k, v, n, self.scale)
        self.flops += encoder_flops(n.tolist())


def run_reference_encoder(args):
    r = EncoderOracleRunner()
    r.step()
    r.flops = 0
    for _ in range(max(0, args.warmup - 1)):
        r.step()
    r.flops = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r.step()
    el = time.perf_counter() - t0
    v = r.flops / el / 1e12
    sample = (f"each step = encoder attention of ONE clip (all 20 heads) of one layer of the encoder batch "
              f"(8 clips x 4 layers cycled); fp64 oracle; TFLOP/s by the GPU line's FLOP count")
    line = {"impl": "reference", "metric": "encoder attention TFLOP/s (1xB200); % of bf16 tensor roofline",
            "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "encoder attention B=8 clips of 150..1500 frames (S=1500), 20 heads x 64, "
                                   "32 layers"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": r.cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_qkv(args):
    """The oracle's projection + RoPE + delta write on the host cores: each step is
    one layer over a bounded sample of the workload's live token rows (all 32 of a
    decode step; 64 of the prefill batch), layers cycled."""
    import numpy as np
    import torch
    cores = os.cpu_count() or 1
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    import oracle
    from gqa_attention_static_b200 import workloads as W
    oracle.build()
    bits = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
    if args.config == "qkv_decode":
        base = W.cfg_ragged_decode(layers=1)
        rows = [(b, 0) for b in range(base.B)]
        desc = "decode step B=32 (ragged batch), hidden 2048 -> 16+2+2 heads x 128, 36 layers"
    else:
        base = W.cfg_prefill(layers=1)
        live = [(b, t) for b in range(base.B) for t in range(int(base.n_new[b]))]
        rng = np.random.default_rng(0)
        rows = [live[i] for i in rng.choice(len(live), 64, replace=False)]
        desc = "coalesced prefill B=16 L U[20,387] S=387, hidden 2048 -> 16+2+2 heads x 128, 36 layers"
    B, S, T = base.B, base.q[0].shape[1], base.T
    pos = np.array([int(base.pos0[b]) + t for b, t in rows], np.int32)
    layers = []
    for l in range(4):
        w, bias = W.make_qkv_weights(1000 + l)
        x = bits(W.make_hidden(2000 + l, B, S))
        xs = np.stack([x[b, t] for b, t in rows])[:, None, :]
        layers.append((xs, bits(w), bits(bias)))
    ck = np.zeros((len(rows), T, 2, 128), np.uint16)
    cv = np.zeros((len(rows), T, 2, 128), np.uint16)
    ones = np.ones(len(rows), np.int32)

    def step(i):
        xs, w, bias = layers[i % len(layers)]
        oracle.qkv_rope_append(xs, w, bias, ck, cv, pos, ones, 16, 2)

    for i in range(max(1, args.warmup)):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    v = len(rows) * args.steps / el
    sample = (f"each step = projection + RoPE + delta write of ONE layer over {len(rows)} live token rows of: "
              f"{desc} (4 distinct layers cycled); fp64 oracle; token-layers/s")
    line = {"impl": "reference",
            "metric": "fused Q/K/V projection + RoPE + delta write, token-layers/s (1xB200); % of roofline",
            "value": v, "unit": "token-layers/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (random-init weights)", "config": {"workload": desc},
            "cpu_baseline": {"value": v, "unit": "token-layers/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "token-layers/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    if args.config == "encoder":
        run_reference_encoder(args)
        return
    if args.config in ("qkv_decode", "qkv_prefill"):
        run_reference_qkv(args)
        return
    r = OracleRunner(args.config, args.mode, kv=args.kv)
    for _ in range(max(1, args.warmup)):
        r.layer_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r.layer_step()          # one step = one layer of the workload (bounded sample)
    el = time.perf_counter() - t0
    v = r.bytes_per_layer * args.steps / el / 1e9
    sample = (f"each step = RoPE + delta write + decode attention of ONE of the 36 layers of: {r.desc} "
              f"(4 distinct layers cycled); fp64 oracle; GB/s by the GPU line's algorithmic-byte count")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": r.desc, "mode": args.mode, "kv_cache": args.kv},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": r.cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def prefill_bytes_flops(n_new):
    """Causal prefill per layer: 9216 B per prompt row (q read 4096, o written
    4096, K/V row 1024) and 4096 * L * (L + 1) FLOPs per request of L rows
    (QK^T and PV over the causal half, 16 heads, head dim 128)."""
    rows = sum(int(x) for x in n_new)
    return rows * 9216, sum(4096 * int(x) * (int(x) + 1) for x in n_new)


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def run_prefill(args):
    """Coalesced prefill: 16 prompts of 20..387 rows, 36 layers.  A step is
    RoPE + delta write of all prompt rows of all layers, then the causal
    prefill of every layer."""
    import torch
    from gqa_attention_static_b200 import ops
    from gqa_attention_static_b200 import workloads as W
    from gqa_attention_static_b200.step import PrefillStep

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    ops.load()
    batch = W.cfg_prefill(layers=N_LAYERS)
    L = batch.layers
    step = PrefillStep([x.to(dev) for x in batch.q], [x.to(dev) for x in batch.k_new],
                       [x.to(dev) for x in batch.v_new], [x.to(dev) for x in batch.cache_k],
                       [x.to(dev) for x in batch.cache_v], batch.pos0.to(dev), batch.n_new.to(dev),
                       fused_rope=args.rope_on_load)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step.run(s)
    torch.cuda.synchronize()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=s):
        step.run(s)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
    g_inst = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_inst, stream=s):
        ev[0].record(s)
        step.append(s)
        ev[1].record(s)
        step.attention(s)
        ev[2].record(s)
    torch.cuda.synchronize()
    for _ in range(max(3, args.warmup)):
        g_step.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(args.steps):
            g_step.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms_step = e0.elapsed_time(e1) / args.steps
    with torch.cuda.stream(s):
        g_inst.replay()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms_prefill = ev[1].elapsed_time(ev[2]) / L          # per layer: the layer-batched prefill call / L
    ms_append = ev[0].elapsed_time(ev[1])
    if int(step.status.item()) != 0:
        print(f"device status word set: {int(step.status.item())}", file=sys.stderr)
    nb, nf = prefill_bytes_flops(batch.n_new.tolist())
    hbm, hbm_kind = measured_peaks()
    tc, tc_kind = measured_tensor_peak()
    t_bytes = nb / (hbm * 1e9)
    t_flops = nf / (tc * 1e12)
    bound = "hbm" if t_bytes >= t_flops else "tensor"
    achieved_gbs = nb / (ms_prefill * 1e-3) / 1e9
    achieved_tf = nf / (ms_prefill * 1e-3) / 1e12
    roof = {"kernel": "prefill_kernel (ark_attn_prefill%s_layers, per layer)" % ("_rope" if args.rope_on_load else ""),
            "bound": bound,
            "achieved": achieved_gbs if bound == "hbm" else achieved_tf,
            "peak": hbm if bound == "hbm" else tc, "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": (t_bytes if bound == "hbm" else t_flops) / (ms_prefill * 1e-3),
            "peak_kind": hbm_kind if bound == "hbm" else tc_kind,
            "traffic": PREFILL_TRAFFIC.get(src_hash("gqa_attention_static_b200/csrc/prefill.cu")),
            "launch_ms": ms_prefill, "algorithmic_bytes_per_launch": nb, "flops_per_launch": nf,
            "achieved_tflops": achieved_tf, "tensor_peak_tflops": tc,
            "append_ms_per_step": ms_append}
    value = nb * L / (ms_step * 1e-3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "coalesced causal prefill B=16 L U[20,387] S=387 T=512, 36 layers",
                       "layers": L, "rows": int(batch.n_new.sum()),
                       "l2": "q/o of 36 layers (1.8 GB) larger than L2",
                       "path": ("layer-batched K/V append + layer-batched prefill rotating q as it loads it"
                                if args.rope_on_load else "layer-batched append + layer-batched prefill") +
                               " (16 layers per launch), replayed from one CUDA graph"},
            "tokens_layers_per_s": int(batch.n_new.sum()) * L / (ms_step * 1e-3),
            "roofline": roof, "gpu_launches": step.launches_per_step() * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)


def encoder_flops(lengths, H: int = 20, D: int = 64) -> int:
    """Encoder attention per layer: 4 * D FLOPs per (query frame, key frame)
    pair of a clip (QK^T and PV), len^2 pairs per clip and head."""
    return sum(4 * D * H * int(n) * int(n) for n in lengths)


def run_encoder(args):
    """The audio encoder's bidirectional attention: 8 clips of 3..30 s (150..1500
    frames, padded to 1500), 20 heads of 64 dims, 32 layers; a step is the
    attention of all 32 layers (one launch each), replayed from a CUDA graph."""
    import torch
    from gqa_attention_static_b200 import ops
    from gqa_attention_static_b200 import workloads as W

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    ops.load()
    e = W.cfg_encoder(layers=args.layers or W.ENC_LAYERS)
    L = len(e.q)
    q = [x.to(dev) for x in e.q]
    k = [x.to(dev) for x in e.k]
    v = [x.to(dev) for x in e.v]
    length = e.length.to(dev)
    o = [torch.empty_like(x) for x in q]
    lse = [torch.empty((e.B, x.shape[2], e.S), dtype=torch.float32, device=dev) for x in q]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(W.ENC_HEAD_DIM)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())

    def step():
        for l in range(L):
            ops.ark_attn_encoder(q[l], k[l], v[l], length, o[l], lse[l], scale, status, stream=s)

    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    torch.cuda.synchronize()
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(args.steps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    if int(status.item()) != 0:
        print(f"device status word set: {int(status.item())}", file=sys.stderr)
    nf = encoder_flops(e.length.tolist())
    tc, tc_kind = measured_tensor_peak()
    ms_launch = ms_step / L
    achieved = nf / (ms_launch * 1e-3) / 1e12
    roof = {"kernel": "encoder_attn_kernel (ark_attn_encoder, one layer per launch)", "bound": "tensor",
            "achieved": achieved, "peak": tc, "unit": "TFLOP/s", "frac": achieved / tc, "peak_kind": tc_kind,
            "traffic": ENCODER_TRAFFIC.get(src_hash("gqa_attention_static_b200/csrc/encoder.cu")),
            "launch_ms": ms_launch, "flops_per_launch": nf}
    value = achieved
    line = {"metric": "encoder attention TFLOP/s (1xB200); % of bf16 tensor roofline", "value": value,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "encoder attention B=8 clips of 150..1500 frames (S=1500), 20 heads x 64, "
                                   f"{L} layers", "lengths": e.length.tolist(),
                       "l2": "q/k/v/o of 32 layers (3.9 GB) larger than L2"},
            "roofline": roof, "gpu_launches": L * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_qkv(args):
    """The projection step in front of the attention, fused with RoPE and the
    delta write (ark_attn_qkv_rope_append), for 36 layers each with its own
    synthetic weights [2560, 2048] (+ bias).  qkv_decode: one decode step of the
    ragged batch (32 token rows); qkv_prefill: the coalesced prefill batch
    (16 prompts of 20..387 rows, padded to 387)."""
    import torch
    from gqa_attention_static_b200 import ops
    from gqa_attention_static_b200 import workloads as W

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    ops.load()
    L = args.layers or N_LAYERS
    if args.config == "qkv_decode":
        base = W.cfg_ragged_decode(layers=1)
        desc = "decode step B=32 (ragged batch), hidden 2048 -> 16+2+2 heads x 128, 36 layers"
    else:
        base = W.cfg_prefill(layers=1)
        desc = "coalesced prefill B=16 L U[20,387] S=387, hidden 2048 -> 16+2+2 heads x 128, 36 layers"
    B, S, T = base.B, base.q[0].shape[1], base.T
    pos0, n_new = base.pos0.to(dev), base.n_new.to(dev)
    ws, bs, xs, qs, cks, cvs = [], [], [], [], [], []
    for l in range(L):
        w, b = W.make_qkv_weights(1000 + l)
        ws.append(w.to(dev))
        bs.append(b.to(dev))
        xs.append(W.make_hidden(2000 + l, B, S).to(dev))
        qs.append(torch.empty((B, S, 16, 128), dtype=torch.bfloat16, device=dev))
        cks.append(torch.zeros((B, T, 2, 128), dtype=torch.bfloat16, device=dev))
        cvs.append(torch.zeros((B, T, 2, 128), dtype=torch.bfloat16, device=dev))
    table = ops.rope_table(T, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())

    def step():
        for l in range(L):
            ops.ark_attn_qkv_rope_append(xs[l], ws[l], bs[l], pos0, n_new, table, qs[l], cks[l], cvs[l], status,
                                         stream=s)

    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    torch.cuda.synchronize()
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(args.steps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    if int(status.item()) != 0:
        print(f"device status word set: {int(status.item())}", file=sys.stderr)
    rows = int(base.n_new.sum())
    N, K = 2560, 2048
    # algorithmic bytes per layer: W + bias, the live x rows, the q / k / v rows written
    nbytes = N * K * 2 + N * 2 + rows * K * 2 + rows * N * 2
    nflops = 2 * rows * K * N
    ms_launch = ms_step / L
    hbm, hbm_kind = measured_peaks()
    tc, tc_kind = measured_tensor_peak()
    t_bytes = nbytes / (hbm * 1e9)
    t_flops = nflops / (tc * 1e12)
    bound = "hbm" if t_bytes >= t_flops else "tensor"
    achieved = (nbytes / 1e9 if bound == "hbm" else nflops / 1e12) / (ms_launch * 1e-3)
    roof = {"kernel": "qkv_proj_kernel (ark_attn_qkv_rope_append, one layer per launch)", "bound": bound,
            "achieved": achieved, "peak": hbm if bound == "hbm" else tc, "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": (t_bytes if bound == "hbm" else t_flops) / (ms_launch * 1e-3),
            "peak_kind": hbm_kind if bound == "hbm" else tc_kind,
            "traffic": QKV_TRAFFIC.get((src_hash("gqa_attention_static_b200/csrc/qkv_proj.cu"), args.config)),
            "launch_ms": ms_launch,
            "algorithmic_bytes_per_launch": nbytes, "flops_per_launch": nflops,
            "achieved_gbs": nbytes / (ms_launch * 1e-3) / 1e9, "achieved_tflops": nflops / (ms_launch * 1e-3) / 1e12}
    value = rows * L / (ms_step * 1e-3)
    line = {"metric": "fused Q/K/V projection + RoPE + delta write, token-layers/s (1xB200); % of roofline",
            "value": value, "unit": "token-layers/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (random-init weights)",
            "config": {"workload": desc.replace("36 layers", f"{L} layers"), "rows": rows,
                       "l2": "weights of %d layers (%.0f MB) larger than L2" % (L, L * N * K * 2 / 1e6)},
            "roofline": roof, "gpu_launches": L * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.config == "prefill":
        run_prefill(args)
        return
    if args.config == "encoder":
        run_encoder(args)
        return
    if args.config in ("qkv_decode", "qkv_prefill"):
        run_qkv(args)
        return
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = f"cuda:{local}"

    from gqa_attention_static_b200 import ops
    from gqa_attention_static_b200.step import DecodeStep

    ops.load()
    mode = ops.ARK_MASKED_STATIC if args.mode == "masked" else ops.ARK_LENGTH_AWARE
    batch, desc = make_workload(args.config, N_LAYERS, "cpu")
    B, T = batch.B, batch.T
    L = batch.layers

    # device buffers: one packed input buffer (q | k_new | v_new) and one packed output (o | lse)
    qsz = B * 16 * 128
    ksz = B * 2 * 128
    in_elems = L * (qsz + 2 * ksz)
    d_in = torch.empty(in_elems, dtype=torch.bfloat16, device=dev)
    qv = d_in[:L * qsz].view(L, B, 1, 16, 128)
    kv_ = d_in[L * qsz:L * (qsz + ksz)].view(L, B, 1, 2, 128)
    vv = d_in[L * (qsz + ksz):].view(L, B, 1, 2, 128)
    for l in range(L):
        qv[l].copy_(batch.q[l])
        kv_[l].copy_(batch.k_new[l])
        vv[l].copy_(batch.v_new[l])
    fp8 = (args.kv == "fp8")
    ks = vs = None
    if fp8:
        fc = fp8_cache_for(batch, args.mode)
        ck = [x.to(dev) for x in fc.cache_k]
        cv = [x.to(dev) for x in fc.cache_v]
        ks = [x.to(dev) for x in fc.k_scale]
        vs = [x.to(dev) for x in fc.v_scale]
        desc = desc.replace(" 1% x8 K/V row outliers", "") + ", fp8 E4M3 cache (per-head scales)"
    else:
        ck = [x.to(dev) for x in batch.cache_k]
        cv = [x.to(dev) for x in batch.cache_v]
    pos0 = batch.pos0.to(dev)
    n_new = batch.n_new.to(dev)
    kv_len = batch.kv_len.to(dev)
    step = DecodeStep([qv[l] for l in range(L)], [kv_[l] for l in range(L)], [vv[l] for l in range(L)],
                      ck, cv, pos0, n_new, kv_len, max_splits=args.max_splits, mode=mode,
                      batched=not args.per_layer, k_scale=ks, v_scale=vs)
    # outputs packed for the device->host read of the e2e leg
    osz = B * 16 * 128
    d_out_o = torch.empty(L * osz, dtype=torch.bfloat16, device=dev)
    d_out_lse = torch.empty(L * B * 16, dtype=torch.float32, device=dev)
    step.o = [d_out_o[l * osz:(l + 1) * osz].view(B, 1, 16, 128) for l in range(L)]
    step.lse = [d_out_lse[l * B * 16:(l + 1) * B * 16].view(B, 16) for l in range(L)]

    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step.run(s)                 # eager run before capture (loads kernels, sets attributes)
    torch.cuda.synchronize()
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=s):
        step.run(s)
    # The same steps with event-record nodes around each kernel group, to read
    # per-launch kernel durations from inside the timed stream.
    U = 8 if step.batched else 2
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(U)]
    g_inst = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_inst, stream=s):
        for u in range(U):
            ev[u][0].record(s)
            step.append(s)
            ev[u][1].record(s)
            step.attention(s)
            ev[u][2].record(s)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, K):
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(K):
                fn()
            e1.record(s)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    for _ in range(max(3, args.warmup)):
        g_step.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms_total = timed(g_step.replay, args.steps)
    # kernel durations: the instrumented graph, replayed right after, same stream
    reps = max(1, args.steps // U)
    timed(g_inst.replay, reps)
    clk = clocks.stop()
    ms_step = ms_total / args.steps
    if int(step.status.item()) != 0:
        print(f"device status word set: {int(step.status.item())}", file=sys.stderr)
    attn_ms = [ev[u][1].elapsed_time(ev[u][2]) for u in range(U)]
    app_ms = [ev[u][0].elapsed_time(ev[u][1]) for u in range(U)]
    calls_per_group = 1 if step.batched else L          # decode launches per attention group
    per_launch_ms = sum(attn_ms) / len(attn_ms) / calls_per_group

    kvl = batch.kv_len.tolist()
    bytes_layer = algorithmic_bytes(kvl, B, args.kv)
    step_bytes = bytes_layer * L
    value = job_throughput(step_bytes, world, ms_step)
    tl = B * L * world / (ms_step * 1e-3)
    bytes_launch = bytes_layer * (L if step.batched else 1)
    peak, peak_kind = measured_peaks()
    achieved = bytes_launch / (per_launch_ms * 1e-3) / 1e9
    h = src_hash("gqa_attention_static_b200/csrc/decode.cu")
    # the capture is of the default workload's batched launch
    traffic = (DECODE_TRAFFIC.get(h) if (not args.per_layer and args.config == "ragged" and args.mode == "aware"
                                         and not fp8) else None)

    e2e = None
    if not args.no_e2e:
        # End to end through the public calls: every step copies its q/k_new/v_new
        # from pinned host memory and reads o/lse back.  Two buffer sets let the
        # copy engines work on step i+1's inputs and step i-1's outputs while the
        # kernels run step i (three streams, events between them).
        h_in = torch.empty(in_elems, dtype=torch.bfloat16, pin_memory=True)
        h_in.copy_(d_in.cpu())
        sets = []
        for k in range(2):
            di = d_in if k == 0 else torch.empty_like(d_in)
            do = d_out_o if k == 0 else torch.empty_like(d_out_o)
            dl = d_out_lse if k == 0 else torch.empty_like(d_out_lse)
            if k == 0:
                st_k, g_k = step, g_step
            else:
                q2 = di[:L * qsz].view(L, B, 1, 16, 128)
                k2 = di[L * qsz:L * (qsz + ksz)].view(L, B, 1, 2, 128)
                v2 = di[L * (qsz + ksz):].view(L, B, 1, 2, 128)
                st_k = DecodeStep([q2[l] for l in range(L)], [k2[l] for l in range(L)], [v2[l] for l in range(L)],
                                  ck, cv, pos0, n_new, kv_len, max_splits=args.max_splits, mode=mode,
                                  batched=not args.per_layer, k_scale=ks, v_scale=vs)
                st_k.o = [do[l * osz:(l + 1) * osz].view(B, 1, 16, 128) for l in range(L)]
                st_k.lse = [dl[l * B * 16:(l + 1) * B * 16].view(B, 16) for l in range(L)]
                with torch.cuda.stream(s):
                    st_k.run(s)
                torch.cuda.synchronize()
                g_k = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g_k, stream=s):
                    st_k.run(s)
            ho = torch.empty(L * osz, dtype=torch.bfloat16, pin_memory=True)
            hl = torch.empty(L * B * 16, dtype=torch.float32, pin_memory=True)
            sets.append((di, do, dl, g_k, ho, hl))
        s_h2d = torch.cuda.Stream(device=dev)
        s_d2h = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for k in range(2):
            ev_comp[k].record(s)
            ev_out[k].record(s)
        torch.cuda.synchronize()

        def run_e2e(K):
            for i in range(K):
                k = i % 2
                di, do, dl, g_k, ho, hl = sets[k]
                s_h2d.wait_event(ev_comp[k])          # step i-2 no longer reads this input set
                with torch.cuda.stream(s_h2d):
                    di.copy_(h_in, non_blocking=True)
                ev_in[k].record(s_h2d)
                s.wait_event(ev_in[k])
                s.wait_event(ev_out[k])                # step i-2's outputs were read back
                with torch.cuda.stream(s):
                    g_k.replay()
                ev_comp[k].record(s)
                s_d2h.wait_event(ev_comp[k])
                with torch.cuda.stream(s_d2h):
                    ho.copy_(do, non_blocking=True)
                    hl.copy_(dl, non_blocking=True)
                ev_out[k].record(s_d2h)

        run_e2e(4)
        K2 = max(10, args.steps // 2)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_h2d)
        run_e2e(K2)
        s_h2d.wait_stream(s_d2h)
        e1.record(s_h2d)
        barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / K2, world, dev)
        e2e = {"value": job_throughput(step_bytes, world, ms_e2e), "unit": "GB/s",
               "h2d_bytes_per_step": in_elems * 2, "d2h_bytes_per_step": L * osz * 2 + L * B * 16 * 4,
               "ms_per_step": ms_e2e,
               "how": "pinned host buffers, H2D of the step inputs and D2H of o/lse every step, "
                      "double-buffered on separate copy streams"}

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(args.config, args.cpu_seconds, args.mode, args.kv)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 cache, f16 MMA" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": desc, "batch": B, "max_total_len": T, "layers": L, "kv_cache": args.kv,
                       "mode": "masked-static" if args.mode == "masked" else "length-aware",
                       "max_splits": args.max_splits, "min_tiles_per_warp": step.min_tiles,
                       "l2": "inputs larger than L2 (%.0f MB of caches streamed per step)" %
                             (2 * L * B * T * 2 * 128 * (1 if fp8 else 2) / 1e6),
                       "parallelism": f"replicas x{world}",
                       "path": ("per-layer calls" if args.per_layer else "layer-batched calls") +
                               " replayed from one CUDA graph"},
            "tokens_layers_per_s": tl,
            "roofline": {"kernel": "decode_kernel + merge_kernel (one ark_attn_decode%s call)" %
                                   ("" if args.per_layer else "_layers"),
                         "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                         "launch_ms": per_launch_ms, "algorithmic_bytes_per_launch": bytes_launch,
                         "append_ms_per_step": sum(app_ms) / len(app_ms)},
            "cpu_baseline": cb,
            "e2e": e2e,
            "gpu_launches": step.launches_per_step() * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        del g_step, g_inst
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
