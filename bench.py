"""Benchmark of the decode hot path: GQA attention over the static KV cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config ragged|single|long2048|long1024|sweep|prefill|encoder|qkv_decode|qkv_prefill]
                    [--mode aware|masked] [--kv bf16|fp8]

A step is one pass of the whole decode path over one batch: for each of the
36 layers, RoPE on the new q/k rows with the delta write into that layer's
static cache, then split-KV decode attention (with its log-sum-exp merge).
The default workload is the ragged decode batch: 32 requests, T = 512,
valid lengths uniform in [40, 511] before the append (41..512 rows read),
K/V with 1% x8 row outliers, 36 independent layers (604 MB of caches, larger
than the 126 MB L2, so every step streams from HBM).

The default run (N = 1) also measures the other workloads of the decoder's
attention and reports them under "configs" in the same JSON line: the single
decode step (B = 1), the batch-1 autoregressive sweep (50-row prefill, then
461 decode steps), the coalesced prefill (16 prompts of 20..387 rows), and the
long-cache batches (T = 2048 ragged, T = 1024 full) in the length-aware and
masked-static modes side by side.  Each of them can also be run alone with
--config.

Timing: W untimed warm-up steps, then exactly K steps replayed from one CUDA
graph, bracketed by a barrier and a device synchronisation, timed with CUDA
events on the launching stream; max over ranks.  Rank 0 prints one JSON line.
Multi-GPU runs are independent replicas (weak scaling, no collective on the
data path).  Roofline fractions are given against the measured copy
bandwidth (MEASURED_PEAKS.json) and against the 8 TB/s HBM3e figure.

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
SPEC_HBM_GBS = 8000.0          # B200 HBM3e figure the decode target is stated against
N_LAYERS = 36
DECODE_CONFIGS = ("ragged", "single", "long2048", "long1024")

# Per-launch DRAM traffic of the decode kernel from an ncu capture, keyed by the
# sha256 of the kernel source it was taken on; reported as null once the source
# has changed.
DECODE_TRAFFIC = {
    # ncu dram bytes, one call of the ragged decode workload: decode_kernel plus
    # merge_kernel, read + write (see profiles/)
    "09c8f33c6fa5b1855d6c89b8aca0676a6d501d7e5059e7b4c2d4dd0dfb6ba281":
        329.766656e6 + 3.29088e6 + 13.198336e6 + 0,
}
# The same for the fp8 cache (the ragged workload with --kv fp8).
DECODE_TRAFFIC_FP8 = {
    "09c8f33c6fa5b1855d6c89b8aca0676a6d501d7e5059e7b4c2d4dd0dfb6ba281":
        167.267072e6 + 3.617536e6 + 13.19808e6 + 0,
}


# Per-launch DRAM traffic of the prefill kernel (one layer of the coalesced
# prefill workload) from an ncu --set full capture, keyed the same way.
PREFILL_TRAFFIC = {
    # ncu --set full of one 4-layer launch of the workload (RoPE on load), read + write, / 4:
    # reads 17.92 MB per layer (q rows, K/V rows); most of o is still in L2 when the kernel
    # ends, so DRAM writes (2.93 MB per layer) stay below the 13.5 MB written (see profiles/)
    "3ba101752de68b41be5d43962949cc44d37ede4c00e20bccf4cb897a3b498984": (71.671552e6 + 11.726848e6) / 4,
}


# Per-launch DRAM traffic of the projection kernel (one layer) from ncu --set full
# captures of the two projection workloads, keyed by source hash and workload.
QKV_TRAFFIC = {
    # the 3-stage instantiation (many tiles) for the prompt rows (dram bytes); the narrow form
    # (token rows on the MMA's N, K split 8 ways) for a decode step (--set full)
    ("dbafa3a02e382f7a7a073b2e97a78056853bc297e8293e2f1726c646a5e573b9", "qkv_prefill"): 36.077824e6 + 0.27904e6,
    ("dbafa3a02e382f7a7a073b2e97a78056853bc297e8293e2f1726c646a5e573b9", "qkv_decode"): 10.684928e6 + 0,
}


# Per-launch DRAM traffic of the encoder attention kernel (one layer of the encoder batch)
# from an ncu --set full capture, keyed the same way.
ENCODER_TRAFFIC = {
    "80df227913d295a8609e6a3f910c9fec15f5022b9b6a5ccd51b8841d3da00579": 64.049152e6 + 2.81856e6,
}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="ragged",
                    choices=list(DECODE_CONFIGS) + ["sweep", "prefill", "encoder", "qkv_decode", "qkv_prefill"])
    ap.add_argument("--mode", default="aware", choices=["aware", "masked"])
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="cache format of the decode configurations: bf16, or fp8 E4M3 codes with per-head scales")
    ap.add_argument("--max-splits", type=int, default=8)
    ap.add_argument("--per-layer", action="store_true",
                    help="issue the single-layer calls layer by layer instead of the layer-batched calls")
    ap.add_argument("--two-call-prefill", action="store_true",
                    help="prefill: rotate q in the append (q read and written) instead of in the prefill kernel")
    ap.add_argument("--layers", type=int, default=None,
                    help="encoder / qkv / prefill: layers per step (default 32 / 36 / 36; fewer only for profiler "
                         "captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="default run: skip the other workloads reported under \"configs\"")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


WORKLOAD_DESC = {
    "ragged": "ragged decode B=32 T=512 kv_len U[41,512] 1% x8 K/V row outliers, 36 layers",
    "single": "single decode B=1 T=512 kv_len 65, 36 layers",
    "long2048": "long decode B=32 T=2048 kv_len U[1501,2048], 36 layers",
    "long1024": "long decode B=32 T=1024 full (kv_len 1024), 36 layers",
    "sweep": "autoregressive sweep B=1 T=512: prefill of 50 rows (37 audio + 13 text), then 461 decode steps "
             "(positions 50..510), fresh q/k/v per step, 36 layers",
    "prefill": "coalesced causal prefill B=16 L U[20,387] S=387 T=512, 36 layers",
}


def make_workload(name: str, layers: int, device: str):
    from gqa_attention_static_b200 import workloads as W
    if name == "ragged":
        b = W.cfg_ragged_decode(layers=layers, device=device)
    elif name == "single":
        b = W.cfg_single_decode(layers=layers, device=device)
    elif name == "long2048":
        b = W.cfg_long_decode(layers=layers, T=2048, device=device)
    elif name == "long1024":
        b = W.cfg_long_decode(layers=layers, T=1024, device=device)
    else:
        raise ValueError(f"not a decode workload: {name}")
    return b, WORKLOAD_DESC[name]


def decode_config(name: str, B: int, T: int, L: int, kv: str, mode: str, world: int) -> dict:
    """The `config` of a decode workload's JSON line, the same for both arms."""
    desc = WORKLOAD_DESC[name]
    if kv == "fp8":
        desc = desc.replace(" 1% x8 K/V row outliers", "") + ", fp8 E4M3 cache (per-head scales)"
    return {"workload": desc, "batch": B, "max_total_len": T, "layers": L, "kv_cache": kv,
            "mode": "masked-static" if mode == "masked" else "length-aware",
            "l2": "inputs larger than L2 (%.0f MB of caches per step)" %
                  (2 * L * B * T * 2 * 128 * (1 if kv == "fp8" else 2) / 1e6),
            "parallelism": f"replicas x{world}"}


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


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def hbm_roofline(achieved_gbs: float) -> dict:
    """An HBM-bound kernel's fractions: of the measured copy bandwidth (or the
    fallback when no measurement is present) and of the 8 TB/s HBM3e figure."""
    peak, kind = measured_peaks()
    return {"bound": "hbm", "achieved": achieved_gbs, "peak": peak, "unit": "GB/s", "frac": achieved_gbs / peak,
            "peak_kind": kind, "spec_peak": SPEC_HBM_GBS, "frac_spec": achieved_gbs / SPEC_HBM_GBS}


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


def encoder_config(L: int, lengths) -> dict:
    return {"workload": "encoder attention B=8 clips of 150..1500 frames (S=1500), 20 heads x 64, %d layers" % L,
            "lengths": list(lengths), "l2": "q/k/v/o of the layers (%.1f GB) larger than L2" % (L * 0.123)}


def qkv_config(desc: str, rows: int, L: int) -> dict:
    return {"workload": desc.replace("36 layers", f"{L} layers"), "rows": rows,
            "l2": "weights of %d layers (%.0f MB) larger than L2" % (L, L * 2560 * 2048 * 2 / 1e6)}


# ------------------------------------------------------------ the oracle arms ----
# The fp64 oracle (test infrastructure) timed as it stands on this host's cores:
# the cpu_baseline of the GPU line and the --impl reference arm.  Nothing here
# runs on the GPU.

def _bits(x):
    import numpy as np
    import torch
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle():
    cores = os.cpu_count() or 1
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    import oracle
    oracle.build()
    return oracle


class OracleRunner:
    """The fp64 oracle (as it stands) on this host's cores: whole decode
    layer-steps (RoPE + delta write + attention) over a bounded sample of the
    workload's layers.  OpenMP threads = all host cores."""

    def __init__(self, workload: str, mode: str, layers: int = 4, kv: str = "bf16"):
        self.oracle = _oracle()
        self.cores = self.oracle.num_threads()
        batch, self.desc = make_workload(workload, layers, "cpu")
        self.fp8 = (kv == "fp8")
        if self.fp8:
            from gqa_attention_static_b200 import workloads as W
            fc = fp8_cache_for(batch, mode)
            # the oracle takes caches in [B,T,Hkv,D] order; the library's fp8 cache is head-major
            self.inputs = [(_bits(batch.q[l]), _bits(batch.k_new[l]), _bits(batch.v_new[l]),
                            W.to_btkd(fc.cache_k[l]).contiguous().numpy(),
                            W.to_btkd(fc.cache_v[l]).contiguous().numpy(), fc.k_scale[l].numpy(),
                            fc.v_scale[l].numpy()) for l in range(layers)]
            self.desc = self.desc.replace(" 1% x8 K/V row outliers", "") + ", fp8 E4M3 cache"
        else:
            self.inputs = [(_bits(batch.q[l]), _bits(batch.k_new[l]), _bits(batch.v_new[l]),
                            _bits(batch.cache_k[l]), _bits(batch.cache_v[l])) for l in range(layers)]
        self.pos0 = batch.pos0.numpy()
        self.n_new = batch.n_new.numpy()
        self.kv = batch.kv_len.numpy()
        self.B, self.T = batch.B, batch.T
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


def _reference_line(args, metric, value, unit, el, config, sample, cores, dtype="f64", data="synthetic"):
    return {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": data,
            "config": config,
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference_decode(args):
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
    cfg = decode_config(args.config, r.B, r.T, N_LAYERS, args.kv, args.mode, args.gpus)
    print(json.dumps(_reference_line(args, METRIC, v, "GB/s", el, cfg, sample, r.cores)), flush=True)


def run_reference_prefill(args):
    """The oracle's RoPE + delta write + causal prefill on the host cores: each
    step is one request of the coalesced prefill batch in one layer (requests
    and 4 layers cycled); GB/s by the GPU line's prefill byte count."""
    import numpy as np
    from gqa_attention_static_b200 import workloads as W
    oracle = _oracle()
    batch = W.cfg_prefill(layers=4)
    items = []
    for l in range(4):
        for b in range(batch.B):
            n = int(batch.n_new[b])
            items.append((_bits(batch.q[l][b:b + 1]), _bits(batch.k_new[l][b:b + 1]), _bits(batch.v_new[l][b:b + 1]),
                          _bits(batch.cache_k[l][b:b + 1]), _bits(batch.cache_v[l][b:b + 1]), n))
    scale = 1.0 / math.sqrt(128)
    zero = np.zeros(1, np.int32)
    state = {"i": 0, "bytes": 0}

    def step():
        q, kn, vn, ck, cv, n = items[state["i"] % len(items)]
        state["i"] += 1
        nn = np.array([n], np.int32)
        qr, ck2, cv2, _ = oracle.append_rope(q, kn, vn, ck, cv, zero, nn)
        oracle.prefill(qr, ck2, cv2, zero, nn, scale)
        state["bytes"] += 9216 * n

    for _ in range(max(1, args.warmup)):
        step()
    state["bytes"] = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    v = state["bytes"] / el / 1e9
    sample = (f"each step = RoPE + delta write + causal prefill of ONE request (all 16 heads) of one layer of: "
              f"{WORKLOAD_DESC['prefill']} (16 requests x 4 layers cycled); fp64 oracle; GB/s by the GPU line's "
              f"prefill byte count (9216 B per prompt row)")
    cfg = prefill_config(N_LAYERS, int(batch.n_new.sum()), args.gpus)
    print(json.dumps(_reference_line(args, PREFILL_METRIC, v, "GB/s", el, cfg, sample, oracle.num_threads())),
          flush=True)


def run_reference_sweep(args):
    """The oracle's sweep on the host cores: each step is the whole sweep of ONE
    layer (prefill of the 50-row prompt, then 461 decode steps, each with its
    RoPE + delta write); tokens·layers/s."""
    import numpy as np
    from gqa_attention_static_b200 import workloads as W
    oracle = _oracle()
    pre = W.cfg_sweep_prefill(layers=1)
    L0 = pre.S
    nsteps = pre.T - 1 - L0
    qa, ka, va = W.sweep_all_step_inputs(2, nsteps, 1)
    scale = 1.0 / math.sqrt(128)
    one = np.ones(1, np.int32)

    def sweep():
        qr, ck, cv, _ = oracle.append_rope(_bits(pre.q[0]), _bits(pre.k_new[0]), _bits(pre.v_new[0]),
                                           _bits(pre.cache_k[0]), _bits(pre.cache_v[0]), pre.pos0.numpy(),
                                           pre.n_new.numpy())
        oracle.prefill(qr, ck, cv, pre.pos0.numpy(), pre.n_new.numpy(), scale)
        for i in range(nsteps):
            p = L0 + i
            qd, ck, cv, _ = oracle.append_rope(_bits(qa[i, 0]), _bits(ka[i, 0]), _bits(va[i, 0]), ck, cv,
                                               np.array([p], np.int32), one)
            oracle.decode(qd, ck, cv, np.array([p + 1], np.int32), scale)

    for _ in range(max(1, args.warmup)):
        sweep()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sweep()
    el = time.perf_counter() - t0
    v = (L0 + nsteps) * args.steps / el
    sample = (f"each step = the whole sweep of ONE layer (of the 36) of: {WORKLOAD_DESC['sweep']}; fp64 oracle; "
              f"tokens·layers/s")
    cfg = {"workload": WORKLOAD_DESC["sweep"], "batch": 1, "max_total_len": pre.T, "layers": N_LAYERS,
           "prompt_rows": L0, "decode_steps": nsteps, "parallelism": f"replicas x{args.gpus}"}
    print(json.dumps(_reference_line(args, SWEEP_METRIC, v, "tokens·layers/s", el, cfg, sample,
                                     oracle.num_threads())), flush=True)


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
        self.lengths = e.length.tolist()
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
            "config": encoder_config(32, [int(x) for x in r.lengths]),
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
            "dtype": "f64", "data": "synthetic (random-init weights)", "config": qkv_config(desc, int(base.n_new.sum()) if args.config == "qkv_prefill" else base.B, N_LAYERS),
            "cpu_baseline": {"value": v, "unit": "token-layers/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "token-layers/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)




# ---------------------------------------------------------------- the GPU arm ----

PREFILL_METRIC = "coalesced causal prefill GB/s (1×B200); % of HBM roofline"
SWEEP_METRIC = "autoregressive sweep tokens·layers/s (1×B200)"


def _capture(fn, s):
    """A CUDA graph of fn(s) (run once eagerly first: loads kernels, sets attributes)."""
    import torch
    with torch.cuda.stream(s):
        fn(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn(s)
    torch.cuda.synchronize()
    return g


def _replay_ms(g, s, n: int) -> float:
    """Device time per replay of graph g, n replays back to back on stream s,
    CUDA events on s with a synchronisation on both sides."""
    import torch
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(n):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def _instrumented(append_fn, attn_fn, s, U: int):
    """A graph of U steps with event-record nodes around each step's two kernel
    groups, so per-launch durations are read on the launching stream."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(U)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for u in range(U):
            ev[u][0].record(s)
            append_fn(s)
            ev[u][1].record(s)
            attn_fn(s)
            ev[u][2].record(s)
    torch.cuda.synchronize()
    return g, ev


def _launch_times(g, ev, s, U: int, step_ms: float, min_calls: int = 200, min_s: float = 0.5):
    """Replay the instrumented graph for at least min_calls calls and min_s
    seconds; mean (append ms, attention ms) per call over the last replay's U
    calls (every replay overwrites the same events)."""
    import torch
    reps = max(-(-min_calls // U), int(math.ceil(min_s * 1e3 / max(step_ms * U, 1e-3))))
    with torch.cuda.stream(s):
        for _ in range(reps):
            g.replay()
    torch.cuda.synchronize()
    app = [ev[u][0].elapsed_time(ev[u][1]) for u in range(U)]
    att = [ev[u][1].elapsed_time(ev[u][2]) for u in range(U)]
    return sum(app) / U, sum(att) / U, reps * U


def decode_measure(name: str, mode_name: str, dev: str, s, steps: int, batched: bool = True, max_splits: int = 8,
                   kv: str = "bf16"):
    """One decode workload on this GPU: step time (graph replays), the decode
    call's duration (instrumented graph), algorithmic GB/s and roofline
    fractions.  Inputs are generated on the device."""
    import torch
    from gqa_attention_static_b200 import ops
    from gqa_attention_static_b200.step import DecodeStep
    batch, desc = make_workload(name, N_LAYERS, dev)
    mode = ops.ARK_MASKED_STATIC if mode_name == "masked" else ops.ARK_LENGTH_AWARE
    ks = vs = None
    if kv == "fp8":
        fc = fp8_cache_for(batch, mode_name)
        ck, cv = [x.to(dev) for x in fc.cache_k], [x.to(dev) for x in fc.cache_v]
        ks, vs = [x.to(dev) for x in fc.k_scale], [x.to(dev) for x in fc.v_scale]
    else:
        ck, cv = batch.cache_k, batch.cache_v
    step = DecodeStep(batch.q, batch.k_new, batch.v_new, ck, cv, batch.pos0, batch.n_new, batch.kv_len,
                      max_splits=max_splits, mode=mode, batched=batched, k_scale=ks, v_scale=vs)
    g = _capture(step.run, s)
    for _ in range(3):
        g.replay()
    ms_step = _replay_ms(g, s, steps)
    U = 8 if batched else 2
    gi, ev = _instrumented(step.append, step.attention, s, U)
    app_ms, attn_ms, calls = _launch_times(gi, ev, s, U, ms_step)
    per_call = attn_ms / (1 if batched else N_LAYERS)
    L = batch.layers
    bytes_layer = algorithmic_bytes(batch.kv_len.tolist(), batch.B, kv)
    bytes_call = bytes_layer * (L if batched else 1)
    out = {"workload": desc, "mode": "masked-static" if mode_name == "masked" else "length-aware",
           "ms_per_step": ms_step, "gbs": bytes_layer * L / (ms_step * 1e-3) / 1e9,
           "tokens_layers_per_s": batch.B * L / (ms_step * 1e-3),
           "decode_call_us": per_call * 1e3, "append_us_per_step": app_ms * 1e3,
           "algorithmic_bytes_per_step": bytes_layer * L, "timed_calls": calls,
           "status": int(step.status.item())}
    out.update({"decode_" + k: v for k, v in hbm_roofline(bytes_call / (per_call * 1e-3) / 1e9).items()
                if k in ("achieved", "frac", "frac_spec", "peak", "peak_kind")})
    return out, step, batch, g, ms_step, per_call, bytes_layer


def sweep_measure(dev: str, s, reps: int = 3, fused_rope: bool = True):
    """The batch-1 autoregressive sweep over 36 layers: prefill of the 50-row
    prompt, then 461 decode steps at positions 50..510, each appending its fresh
    k/v row and attending to every valid row.  The prefill and the 461 steps
    are each one CUDA graph (the decode graph holds 461 x 3 launches)."""
    import torch
    from gqa_attention_static_b200 import ops
    from gqa_attention_static_b200 import workloads as W
    from gqa_attention_static_b200.step import DecodeStep, PrefillStep
    L = N_LAYERS
    pre = W.cfg_sweep_prefill(layers=L, device=dev)
    L0, T = pre.S, pre.T
    nsteps = T - 1 - L0
    ps = PrefillStep(pre.q, pre.k_new, pre.v_new, pre.cache_k, pre.cache_v, pre.pos0, pre.n_new,
                     fused_rope=fused_rope)
    qa, ka, va = W.sweep_all_step_inputs(2, nsteps, L, device=dev)
    pos_all = torch.arange(L0, L0 + nsteps, dtype=torch.int32, device=dev)
    kv_all = pos_all + 1
    one = torch.ones(1, dtype=torch.int32, device=dev)
    ws = ops.decode_workspace(1, 16, 128, T, 8, device=dev, layers=L)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    o = [torch.empty(1, 1, 16, 128, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    lse = [torch.empty(1, 16, dtype=torch.float32, device=dev) for _ in range(L)]
    steps = [DecodeStep([qa[i, l] for l in range(L)], [ka[i, l] for l in range(L)], [va[i, l] for l in range(L)],
                        pre.cache_k, pre.cache_v, pos_all[i:i + 1], one, kv_all[i:i + 1], table=ps.table,
                        workspace=ws, status=status, o=o, lse=lse) for i in range(nsteps)]

    def decode_all(st):
        for x in steps:
            x.run(st)

    g_pre = _capture(ps.run, s)
    g_dec = _capture(decode_all, s)
    for _ in range(2):
        g_pre.replay()
        g_dec.replay()
    torch.cuda.synchronize()
    ms_pre = _replay_ms(g_pre, s, max(3, reps))
    ms_dec = _replay_ms(g_dec, s, reps)
    # the whole sweep: prefill then decode, back to back
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(reps):
            g_pre.replay()
            g_dec.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms_sweep = e0.elapsed_time(e1) / reps
    positions = sum(range(L0 + 1, L0 + nsteps + 1))
    dec_bytes = (positions * 1024 + nsteps * 8192) * L
    st = int(status.item()) | int(ps.status.item())
    res = {"workload": WORKLOAD_DESC["sweep"], "ms_per_sweep": ms_sweep,
           "tokens_layers_per_s": (L0 + nsteps) * L / (ms_sweep * 1e-3),
           "prefill_ms": ms_pre, "decode_ms": ms_dec, "decode_us_per_step": ms_dec * 1e3 / nsteps,
           "decode_tokens_layers_per_s": nsteps * L / (ms_dec * 1e-3),
           "decode_kv_gbs": dec_bytes / (ms_dec * 1e-3) / 1e9, "decode_algorithmic_bytes": dec_bytes,
           "prefill_path": "K/V append + prefill rotating q on load" if fused_rope else "append + prefill",
           "launches_per_sweep": ps.launches_per_step() + 3 * nsteps, "status": st}
    return res, ps.launches_per_step() + 3 * nsteps


def prefill_bytes_flops(n_new):
    """Causal prefill per layer: 9216 B per prompt row (q read 4096, o written
    4096, K/V row 1024) and 4096 * L * (L + 1) FLOPs per request of L rows
    (QK^T and PV over the causal half, 16 heads, head dim 128)."""
    rows = sum(int(x) for x in n_new)
    return rows * 9216, sum(4096 * int(x) * (int(x) + 1) for x in n_new)


def prefill_config(L: int, rows: int, world: int) -> dict:
    return {"workload": WORKLOAD_DESC["prefill"].replace("36 layers", f"{L} layers"), "layers": L, "rows": rows,
            "l2": "q/o of the layers (%.1f GB) larger than L2" % (L * 16 * 387 * 16 * 128 * 2 * 2 / 1e9),
            "parallelism": f"replicas x{world}"}


def prefill_measure(dev: str, s, steps: int, fused_rope: bool = True, layers: int = N_LAYERS):
    """Coalesced prefill: 16 prompts of 20..387 rows, 36 layers.  A step is the
    K/V append (RoPE on k, delta write) of every prompt row of every layer, then
    the causal prefill of every layer (rotating q as it loads it); with
    fused_rope False the append also rotates q in place."""
    import torch
    from gqa_attention_static_b200 import workloads as W
    from gqa_attention_static_b200.step import PrefillStep
    batch = W.cfg_prefill(layers=layers, device=dev)
    L = batch.layers
    step = PrefillStep(batch.q, batch.k_new, batch.v_new, batch.cache_k, batch.cache_v, batch.pos0, batch.n_new,
                       fused_rope=fused_rope)
    g = _capture(step.run, s)
    for _ in range(3):
        g.replay()
    ms_step = _replay_ms(g, s, steps)
    U = 4
    gi, ev = _instrumented(step.append, step.attention, s, U)
    ms_append, ms_attn, calls = _launch_times(gi, ev, s, U, ms_step, min_calls=40, min_s=0.3)
    ms_layer = ms_attn / L
    nb, nf = prefill_bytes_flops(batch.n_new.tolist())
    tc, tc_kind = measured_tensor_peak()
    hb = hbm_roofline(nb / (ms_layer * 1e-3) / 1e9)
    achieved_tf = nf / (ms_layer * 1e-3) / 1e12
    roof = dict(hb)
    roof.update({"kernel": "prefill_kernel (ark_attn_prefill%s_layers: one launch of 36 layers), per layer" %
                           ("_rope" if fused_rope else ""),
                 "traffic": PREFILL_TRAFFIC.get(src_hash("gqa_attention_static_b200/csrc/prefill.cu")),
                 "launch_ms_per_layer": ms_layer, "algorithmic_bytes_per_layer": nb, "flops_per_layer": nf,
                 "achieved_tflops": achieved_tf, "tensor_peak_tflops": tc, "tensor_peak_kind": tc_kind,
                 "frac_tensor": achieved_tf / tc, "append_ms_per_step": ms_append, "timed_calls": calls})
    res = {"workload": WORKLOAD_DESC["prefill"], "ms_per_step": ms_step, "gbs": nb * L / (ms_step * 1e-3) / 1e9,
           "tokens_layers_per_s": int(batch.n_new.sum()) * L / (ms_step * 1e-3),
           "prefill_ms_per_layer": ms_layer, "append_ms_per_step": ms_append,
           "frac": hb["frac"], "frac_spec": hb["frac_spec"], "frac_tensor": achieved_tf / tc,
           "path": ("K/V-only append + prefill rotating q as it loads it" if fused_rope else
                    "append rotating q in place + prefill"),
           "status": int(step.status.item())}
    return res, roof, step, batch, ms_step


E2E_SETS = 4


def e2e_measure(step_factory, d_in, d_out_o, d_out_lse, g_step, step, s, dev, steps: int):
    """End to end through the public calls: every step copies its inputs
    (q/k_new/v_new of all layers) from pinned host memory and reads o/lse back
    into pinned host memory.  E2E_SETS buffer sets let the copy engines move
    later steps' inputs and earlier steps' outputs while the kernels run step i
    (three streams, events between them; the kernels of a step replay its CUDA
    graph); with more than two sets the input copy of step i+E2E_SETS waits only
    for step i's compute, so both copy directions can stream back to back (four
    sets: 0.172 ms per step against 0.217 with two; the two directions together
    then move ~62 GB/s over PCIe, against ~53 GB/s for one alone).  Timed over at
    least `steps` steps and 0.3 s; the copies alone and the compute alone are
    timed too, for the breakdown."""
    import torch
    NS = E2E_SETS
    sets = []
    for k in range(NS):
        if k == 0:
            di, do, dl, g_k = d_in, d_out_o, d_out_lse, g_step
        else:
            di, do, dl = torch.empty_like(d_in), torch.empty_like(d_out_o), torch.empty_like(d_out_lse)
            g_k = _capture(step_factory(di, do, dl).run, s)
        ho = torch.empty(do.numel(), dtype=do.dtype, pin_memory=True)
        hl = torch.empty(dl.numel(), dtype=dl.dtype, pin_memory=True)
        sets.append((di, do, dl, g_k, ho, hl))
    h_in = torch.empty(d_in.numel(), dtype=d_in.dtype, pin_memory=True)
    h_in.copy_(d_in.cpu())
    s_h2d = torch.cuda.Stream(device=dev)
    s_d2h = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(NS)]
    ev_comp = [torch.cuda.Event() for _ in range(NS)]
    ev_out = [torch.cuda.Event() for _ in range(NS)]
    for k in range(NS):
        ev_comp[k].record(s)
        ev_out[k].record(s)
    torch.cuda.synchronize()

    def run_e2e(K):
        for i in range(K):
            k = i % NS
            di, do, dl, g_k, ho, hl = sets[k]
            s_h2d.wait_event(ev_comp[k])          # step i-NS no longer reads this input set
            with torch.cuda.stream(s_h2d):
                di.copy_(h_in, non_blocking=True)
            ev_in[k].record(s_h2d)
            s.wait_event(ev_in[k])
            s.wait_event(ev_out[k])                # step i-NS's outputs were read back
            with torch.cuda.stream(s):
                g_k.replay()
            ev_comp[k].record(s)
            s_d2h.wait_event(ev_comp[k])
            with torch.cuda.stream(s_d2h):
                ho.copy_(do, non_blocking=True)
                hl.copy_(dl, non_blocking=True)
            ev_out[k].record(s_d2h)

    run_e2e(8)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    run_e2e(10)
    s_h2d.wait_stream(s_d2h)
    e1.record(s_h2d)
    torch.cuda.synchronize()
    ms10 = e0.elapsed_time(e1) / 10
    K = max(steps, int(math.ceil(300.0 / max(ms10, 1e-3))))
    e0.record(s_h2d)
    run_e2e(K)
    s_h2d.wait_stream(s_d2h)
    e1.record(s_h2d)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / K
    # breakdown: the copies alone, the compute alone
    ho, hl = sets[0][4], sets[0][5]

    def h2d_only(st):
        d_in.copy_(h_in, non_blocking=True)

    def d2h_only(st):
        ho.copy_(d_out_o, non_blocking=True)
        hl.copy_(d_out_lse, non_blocking=True)

    g_h = _capture(h2d_only, s)
    g_d = _capture(d2h_only, s)
    ms_h2d = _replay_ms(g_h, s, 20)
    ms_d2h = _replay_ms(g_d, s, 20)
    ms_comp = _replay_ms(g_step, s, 20)
    h2d_bytes = d_in.numel() * d_in.element_size()
    d2h_bytes = d_out_o.numel() * d_out_o.element_size() + d_out_lse.numel() * d_out_lse.element_size()
    return {"ms_per_step": ms_e2e, "timed_steps": K, "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes,
            "breakdown_ms": {"h2d": ms_h2d, "compute": ms_comp, "d2h": ms_d2h,
                             "h2d_gbs": h2d_bytes / (ms_h2d * 1e-3) / 1e9, "d2h_gbs": d2h_bytes / (ms_d2h * 1e-3) / 1e9},
            "how": "pinned host buffers, H2D of the step inputs and D2H of o/lse every step, %d buffer sets on "
                   "separate copy streams, the step's kernels replayed from its CUDA graph" % NS}


def run_decode(args):
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

    def views(di):
        qv = di[:L * qsz].view(L, B, 1, 16, 128)
        kv_ = di[L * qsz:L * (qsz + ksz)].view(L, B, 1, 2, 128)
        vv = di[L * (qsz + ksz):].view(L, B, 1, 2, 128)
        return [qv[l] for l in range(L)], [kv_[l] for l in range(L)], [vv[l] for l in range(L)]

    qv, kv_, vv = views(d_in)
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
    else:
        ck = [x.to(dev) for x in batch.cache_k]
        cv = [x.to(dev) for x in batch.cache_v]
    pos0 = batch.pos0.to(dev)
    n_new = batch.n_new.to(dev)
    kv_len = batch.kv_len.to(dev)
    osz = B * 16 * 128
    d_out_o = torch.empty(L * osz, dtype=torch.bfloat16, device=dev)
    d_out_lse = torch.empty(L * B * 16, dtype=torch.float32, device=dev)

    def make_step(di, do, dl):
        q_, k_, v_ = views(di)
        return DecodeStep(q_, k_, v_, ck, cv, pos0, n_new, kv_len, max_splits=args.max_splits, mode=mode,
                          batched=not args.per_layer, k_scale=ks, v_scale=vs,
                          o=[do[l * osz:(l + 1) * osz].view(B, 1, 16, 128) for l in range(L)],
                          lse=[dl[l * B * 16:(l + 1) * B * 16].view(B, 16) for l in range(L)])

    step = make_step(d_in, d_out_o, d_out_lse)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    g_step = _capture(step.run, s)
    U = 8 if step.batched else 2
    g_inst, ev = _instrumented(step.append, step.attention, s, U)

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
    ms_step = ms_total / args.steps
    # kernel durations: the instrumented graph, replayed right after on the same stream, for at
    # least 200 decode calls and 0.5 s whatever --steps is
    app_ms, attn_ms, inst_calls = _launch_times(g_inst, ev, s, U, ms_step)
    clk = clocks.stop()
    if int(step.status.item()) != 0:
        print(f"device status word set: {int(step.status.item())}", file=sys.stderr)
    calls_per_group = 1 if step.batched else L          # decode launches per attention group
    per_launch_ms = attn_ms / calls_per_group

    kvl = batch.kv_len.tolist()
    bytes_layer = algorithmic_bytes(kvl, B, args.kv)
    step_bytes = bytes_layer * L
    value = job_throughput(step_bytes, world, ms_step)
    tl = B * L * world / (ms_step * 1e-3)
    bytes_launch = bytes_layer * (L if step.batched else 1)
    achieved = bytes_launch / (per_launch_ms * 1e-3) / 1e9
    h = src_hash("gqa_attention_static_b200/csrc/decode.cu")
    # the capture is of the default workload's batched launch
    traffic = ((DECODE_TRAFFIC_FP8 if fp8 else DECODE_TRAFFIC).get(h)
               if (not args.per_layer and args.config == "ragged" and args.mode == "aware") else None)
    roof = {"kernel": "decode_kernel + merge_kernel (one ark_attn_decode%s call)" % ("" if args.per_layer else
                                                                                     "_layers")}
    roof.update(hbm_roofline(achieved))
    roof.update({"traffic": traffic, "launch_ms": per_launch_ms, "algorithmic_bytes_per_launch": bytes_launch,
                 "timed_calls": inst_calls, "append_ms_per_step": app_ms})

    e2e = None
    if not args.no_e2e:
        r = e2e_measure(make_step, d_in, d_out_o, d_out_lse, g_step, step, s, dev, max(100, args.steps))
        ms_e2e = max_over_ranks(r["ms_per_step"], world, dev)
        e2e = {"value": job_throughput(step_bytes, world, ms_e2e), "unit": "GB/s",
               "h2d_bytes_per_step": r["h2d_bytes_per_step"], "d2h_bytes_per_step": r["d2h_bytes_per_step"],
               "ms_per_step": ms_e2e, "timed_steps": r["timed_steps"], "breakdown_ms": r["breakdown_ms"],
               "how": r["how"]}

    extras = None
    if (world == 1 and not args.no_extras and args.config == "ragged" and args.mode == "aware" and not fp8
            and not args.per_layer):
        del g_step, g_inst
        extras = measure_extras(dev, s, args)

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(args.config, args.cpu_seconds, args.mode, args.kv)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 cache, f16 MMA" if fp8 else "bf16", "data": "synthetic",
            "config": decode_config(args.config, B, T, L, args.kv, args.mode, world),
            "impl_details": {"max_splits": args.max_splits, "min_tiles_per_warp": step.min_tiles,
                             "path": ("per-layer calls" if args.per_layer else "layer-batched calls") +
                                     " replayed from one CUDA graph"},
            "tokens_layers_per_s": tl,
            "roofline": roof,
            "cpu_baseline": cb,
            "e2e": e2e,
            "gpu_launches": step.launches_per_step() * args.steps,
            "clocks": clk,
        }
        if extras is not None:
            line["configs"] = extras
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_extras(dev, s, args):
    """The decoder's other attention workloads, each measured on this GPU in a
    few seconds (inputs generated on the device, freed after each)."""
    import torch
    out = {}
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    for name, mode in (("single", "aware"), ("ragged", "masked"), ("long2048", "aware"), ("long2048", "masked"),
                       ("long1024", "aware"), ("long1024", "masked")):
        r = decode_measure(name, mode, dev, s, 50)[0]
        out[f"{name}_{mode}"] = r
        torch.cuda.empty_cache()
    out["single_aware"]["us_per_step"] = out["single_aware"]["ms_per_step"] * 1e3
    for T in ("long2048", "long1024"):
        a, m = out[f"{T}_aware"], out[f"{T}_masked"]
        m["masked_over_aware_time"] = m["ms_per_step"] / a["ms_per_step"]
    sw, _ = sweep_measure(dev, s, reps=3, fused_rope=not args.two_call_prefill)
    out["sweep"] = sw
    torch.cuda.empty_cache()
    pr = prefill_measure(dev, s, 20, fused_rope=not args.two_call_prefill)[0]
    out["prefill"] = pr
    torch.cuda.empty_cache()
    out["clocks"] = clocks.stop()
    return out


def run_sweep(args):
    import torch
    from gqa_attention_static_b200 import ops
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    ops.load()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    res, launches = sweep_measure(dev, s, reps=max(3, args.steps), fused_rope=not args.two_call_prefill)
    clk = clocks.stop()
    if res["status"]:
        print(f"device status word set: {res['status']}", file=sys.stderr)
    roof = {"kernel": "decode_kernel + merge_kernel, one call per sweep position (latency-bound at B=1)"}
    roof.update(hbm_roofline(res["decode_kv_gbs"]))
    line = {"metric": SWEEP_METRIC, "value": res["tokens_layers_per_s"], "unit": "tokens·layers/s", "n_gpus": world,
            "steps": max(3, args.steps), "warmup": 2, "ms_per_step": res["ms_per_sweep"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC["sweep"], "batch": 1, "max_total_len": 512, "layers": N_LAYERS,
                       "prompt_rows": 50, "decode_steps": 461, "parallelism": f"replicas x{world}"},
            "sweep": res, "roofline": roof, "gpu_launches": launches * max(3, args.steps), "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_prefill(args):
    import torch
    from gqa_attention_static_b200 import ops
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    ops.load()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    res, roof, step, batch, ms_step = prefill_measure(dev, s, args.steps, fused_rope=not args.two_call_prefill,
                                                      layers=args.layers or N_LAYERS)
    clk = clocks.stop()
    if res["status"]:
        print(f"device status word set: {res['status']}", file=sys.stderr)
    L = batch.layers
    nb, _ = prefill_bytes_flops(batch.n_new.tolist())
    line = {"metric": PREFILL_METRIC, "value": nb * L * world / (ms_step * 1e-3) / 1e9, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": prefill_config(L, int(batch.n_new.sum()), world),
            "impl_details": {"path": res["path"] + " (one launch of 36 layers), replayed from one CUDA graph"},
            "tokens_layers_per_s": res["tokens_layers_per_s"], "prefill": res, "roofline": roof,
            "gpu_launches": step.launches_per_step() * args.steps, "clocks": clk}
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
            "config": encoder_config(L, e.length.tolist()),
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
    kname = "qkv_proj_narrow_kernel" if args.config == "qkv_decode" else "qkv_proj_kernel"
    roof = {"kernel": kname + " (ark_attn_qkv_rope_append, one layer per launch)", "bound": bound,
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
            "config": qkv_config(desc, rows, L),
            "roofline": roof, "gpu_launches": L * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)




def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    if args.config == "encoder":
        run_reference_encoder(args)
    elif args.config in ("qkv_decode", "qkv_prefill"):
        run_reference_qkv(args)
    elif args.config == "prefill":
        run_reference_prefill(args)
    elif args.config == "sweep":
        run_reference_sweep(args)
    else:
        run_reference_decode(args)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.config == "prefill":
        run_prefill(args)
    elif args.config == "sweep":
        run_sweep(args)
    elif args.config == "encoder":
        run_encoder(args)
    elif args.config in ("qkv_decode", "qkv_prefill"):
        run_qkv(args)
    else:
        run_decode(args)


if __name__ == "__main__":
    main()
