"""Benchmark of the Codec-Gauge KV codec round trip on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--bits 4] [--impl cg|reference]

One step = fused gauge + quantize + pack encode (cg_encode) followed by fused
unpack + dequantize + inverse-gauge decode (cg_decode) of a Llama-3-8B-shaped
GQA cache: 32 layers x {K, V} x 8 KV heads x 4096 tokens x d_head 128, batch 1,
bf16 (268,435,456 values, 0.537 GB), gauge groups g = 16, block-uniform ranges
of 16 tokens x 16 channels.  Inputs are seeded synthetic caches (AR(1) keys with
lognormal channel scales and outlier channels, AR(1) values); the gauge is
built on the device from A ~ N(0, 0.1^2) by cg_gauge_build before timing.

Metric: KV GB/s = bf16 KV bytes (2 N) carried through encode + decode per
second, summed over GPUs (each GPU runs its own replica: the codec has no
cross-GPU exchange, so scaling is weak).  Per-kernel rates and the HBM roofline
fraction of the dominant kernel come with it.  The working set (0.54 GB in,
0.13 GB codes, 0.54 GB out) is far larger than the 126 MB L2, so no flush is
needed between steps.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L, B, H, T, D = 32, 1, 8, 4096, 128
G_GROUP = 16


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
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
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings over all ranks of the process group
    (the values unchanged on a single process).  Every rank must call it, in the same
    order, with as many values."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_gbs(world_size, bytes_per_rank, ms):
    """Whole-job throughput: the bytes all ranks processed over the slowest rank's time."""
    return world_size * bytes_per_rank / (ms * 1e-3) / 1e9


def run_cg(args):
    import torch
    import torch.distributed as dist
    from quantization_cg_encode_b200 import cg, synth

    ws, rank, local = _dist()
    if ws > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)

    L = args.layers
    kvd = cg.kv_desc(L, B, H, T, D)
    codec = cg.codec_desc(g=G_GROUP, bits=args.bits)
    n_values = L * 2 * B * H * T * D
    kv_bytes = 2 * n_values

    with torch.cuda.stream(stream):
        kv = synth.kv_cache(L, B, H, T, D, seed=rank, device=dev, n_outliers=4)
        A = synth.gauge_params(L, H, D // G_GROUP, G_GROUP, sigma=0.1, seed=rank).to(dev)
        G = torch.empty_like(A)
        cg.cg_gauge_build(A, G, stream=stream)
        codes, scales, zeros = cg.alloc_encoded(kvd, codec, device=dev)
        out = torch.empty_like(kv)
    stream.synchronize()

    def step():
        cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros, None, stream=stream)
        cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out, stream=stream)

    for _ in range(args.warmup):
        step()
    cg.cg_sync_status(stream)

    # --- timed region: K steps, events on the launching stream --------------------------
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for e0, e1, e2 in ev:
            e0.record(stream)
            cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros, None, stream=stream)
            e1.record(stream)
            cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out, stream=stream)
            e2.record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    cg.cg_sync_status(stream)
    total_ms = t_start.elapsed_time(t_end)
    enc_ms = [e0.elapsed_time(e1) for e0, e1, _ in ev]
    dec_ms = [e1.elapsed_time(e2) for _, e1, e2 in ev]

    rows = {} if args.no_rows else measure_rows(args, cg, synth, torch, kv, G, stream, dev, rank)

    # The chain-exact tensor-core encoder checks every value it re-evaluates against the
    # accumulation bound its decisions assume; run it once on the benchmark cache (outside
    # any timed region) and record whether the bound held.
    chain_bound_ok = None
    if not args.no_rows:
        codec_ct = cg.codec_desc(g=16, bits=args.bits, engine=cg.ENGINE_CHAIN_TENSOR)
        cg.cg_encode(kvd, codec_ct, kv, G, 0, T, codes, scales, zeros, None, stream=stream)
        try:
            cg.cg_sync_status(stream)
            chain_bound_ok = True
        except cg.CgError as err:
            if err.status != cg.CG_ERR_BOUND:
                raise
            chain_bound_ok = False

    # --- end to end through the C ABI with host buffers -------------------------------------
    # cg_roundtrip_host: the cache from pinned host memory, its codes on the device, the
    # decoded cache back in pinned host memory, pipelined by layer inside the call.
    kv_host = kv.cpu().pin_memory()
    out_host = torch.empty(kv.shape, dtype=kv.dtype, pin_memory=True)
    ws_rt = torch.empty(cg.cg_roundtrip_workspace_size(kvd), dtype=torch.uint8, device=dev)

    def e2e_step():
        cg.cg_roundtrip_host(kvd, codec, kv_host, G, codes, scales, zeros, out_host, ws_rt, stream=stream)

    e2e_steps = max(2, min(args.steps, 5))
    with torch.cuda.stream(stream):
        if args.no_e2e:
            e2e_steps = 0
        e2e_step() if e2e_steps else None
        stream.synchronize()
        if ws > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        s1.record(stream)
        stream.synchronize()
    e2e_ms = s0.elapsed_time(s1) / e2e_steps if e2e_steps else float("nan")

    # --- max over ranks -----------------------------------------------------------------------
    total_ms, enc_avg, dec_avg, e2e_ms = max_over_ranks(
        [total_ms, statistics.mean(enc_ms), statistics.mean(dec_ms), e2e_ms], dev)
    if ws > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None

    ms_step = total_ms / args.steps
    hbm_peak, peak_kind = _peaks()
    bpv = 2.0 + args.bits / 8.0 + 4.0 / (16 * G_GROUP)       # algorithmic bytes per value, encode and decode
    alg_bytes = bpv * n_values
    enc_gbs = alg_bytes / (enc_avg * 1e-3) / 1e9
    dec_gbs = alg_bytes / (dec_avg * 1e-3) / 1e9
    dominant = "cg_encode" if enc_avg >= dec_avg else "cg_decode"
    dom_ms = max(enc_avg, dec_avg)
    achieved = alg_bytes / (dom_ms * 1e-3) / 1e9
    traffic = _traffic_record(dominant, args.bits)
    value = job_gbs(ws, kv_bytes, ms_step)
    line = {
        "metric": "KV GB/s for fused gauge+quant encode/decode at %d bits; %% of HBM roofline" % args.bits,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 in/out, fp32 arithmetic, %d-bit codes" % args.bits,
        "data": "synthetic (seeded AR(1) KV cache, lognormal channel scales, 4 outlier key channels per head)",
        "config": {"workload": "Llama-3-8B-shaped GQA KV cache 32x2x8x4096x128 bf16, g=16 gauge, block-uniform "
                               "16x16 ranges, %d bits: encode + decode" % args.bits,
                   "kv_bytes": kv_bytes, "parallelism": "replicas (dp%d, no collective)" % ws,
                   "l2": "inputs 0.54 GB > 126 MB L2, no flush"},
        "encode": {"ms": round(enc_avg, 4), "alg_GBps": round(enc_gbs, 1), "frac": round(enc_gbs / hbm_peak, 4),
                   "kv_GBps": round(kv_bytes / (enc_avg * 1e-3) / 1e9, 1)},
        "decode": {"ms": round(dec_avg, 4), "alg_GBps": round(dec_gbs, 1), "frac": round(dec_gbs / hbm_peak, 4),
                   "kv_GBps": round(kv_bytes / (dec_avg * 1e-3) / 1e9, 1)},
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1), "peak": hbm_peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": traffic, "alg_bytes_per_value": bpv},
        "e2e": None if args.no_e2e else {"value": round(job_gbs(ws, kv_bytes, e2e_ms), 2), "unit": "GB/s",
                                         "h2d_bytes_per_step": kv_bytes, "d2h_bytes_per_step": kv_bytes,
                                         "api": "cg_roundtrip_host (pinned host in/out, layer-pipelined)"},
        "gpu_launches": 2 * args.steps,
        "rows": rows,
        "chain_tensor_bound_ok": chain_bound_ok,
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.bits, budget_s=args.cpu_seconds)
    return line


def _time(fn, stream, reps=5, warm=2):
    import torch
    for _ in range(warm):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_rows(args, cg, synth, torch, kv, G16, stream, dev, rank):
    """Per-row kernel timings on the 8B-shaped cache (every other hot-path row), each
    as ms per call, GB/s of algorithmic traffic and the fraction of the HBM peak."""
    hbm, _ = _peaks()
    Lc = kv.shape[0]
    n = kv.numel()
    kvd = cg.kv_desc_of(kv)
    out = torch.empty_like(kv)
    rows = {}

    def rec(name, ms, bytes_per_value, flops_per_value=None):
        gbs = bytes_per_value * n / (ms * 1e-3) / 1e9
        rows[name] = {"ms": round(ms, 4), "alg_GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                      "kv_GBps": round(2 * n / (ms * 1e-3) / 1e9, 1)}
        if flops_per_value:
            rows[name]["TFLOPs"] = round(flops_per_value * n / (ms * 1e-3) / 1e12, 1)

    with torch.cuda.stream(stream):
        for bits in (3, 6):
            codec = cg.codec_desc(g=16, bits=bits)
            c, sc, z = cg.alloc_encoded(kvd, codec, device=dev)
            bpv = 2 + bits / 8 + 4 / 256
            rec("encode_g16_b%d" % bits, _time(lambda: cg.cg_encode(kvd, codec, kv, G16, 0, T, c, sc, z, None, stream=stream), stream), bpv)
            rec("decode_g16_b%d" % bits, _time(lambda: cg.cg_decode(kvd, codec, c, sc, z, G16, 0, T, out, stream=stream), stream), bpv)
        # full-head gauge, G = exp(A - A^T), A ~ N(0, 0.05^2)
        A = synth.gauge_params(Lc, H, 1, 128, sigma=0.05, seed=rank + 5).to(dev)
        G128 = torch.empty_like(A)
        cg.cg_gauge_build(A, G128, stream=stream)
        codec = cg.codec_desc(g=128, bits=4, range_cols=128)
        c, sc, z = cg.alloc_encoded(kvd, codec, device=dev)
        bpv = 2 + 4 / 8 + 4 / (16 * 128)
        rec("fullhead_encode_b4", _time(lambda: cg.cg_encode(kvd, codec, kv, G128, 0, T, c, sc, z, None, stream=stream), stream), bpv, 256)
        rec("fullhead_decode_b4", _time(lambda: cg.cg_decode(kvd, codec, c, sc, z, G128, 0, T, out, stream=stream), stream), bpv, 256)
        # KIVI-style, 3 bits, g = 16 fused
        codec = cg.codec_desc(g=16, bits=3, mode=cg.KIVI)
        c, sc, z = cg.alloc_encoded(kvd, codec, device=dev)
        bpv = 2 + 3 / 8 + 4 / 32
        rec("kivi_encode_b3", _time(lambda: cg.cg_encode(kvd, codec, kv, G16, 0, T, c, sc, z, None, stream=stream), stream), bpv)
        rec("kivi_decode_b3", _time(lambda: cg.cg_decode(kvd, codec, c, sc, z, G16, 0, T, out, stream=stream), stream), bpv)
        # append: one 128-token chunk of every head (a decode step of the rolling cache)
        rec("kivi_append_128tok", _time(lambda: cg.cg_encode(kvd, codec, kv, G16, T - 128, 128, c, sc, z, None, stream=stream), stream, reps=20), bpv * 128 / T)
        # spectral statistics of one 4096-token window: forward, and forward + dL/dG
        st = cg.StatsDesc(16, 16, 0, 1.0, 0.02, 0.04)
        nblk = n // (16 * 128)
        lf = torch.empty(nblk, dtype=torch.float32, device=dev)
        lr = torch.empty_like(lf)
        tot = torch.empty(4, dtype=torch.float64, device=dev)
        dG = torch.empty_like(G16)
        ws = torch.empty(max(cg.cg_spectral_workspace_size(kvd, st, True), 16), dtype=torch.uint8, device=dev)
        rec("stats_fwd", _time(lambda: cg.cg_spectral_stats(kvd, st, kv, G16, lf, lr, tot, None, ws, stream=stream), stream), 2.0, 2 * 144 + 32)
        rec("stats_fwd_bwd", _time(lambda: cg.cg_spectral_stats(kvd, st, kv, G16, lf, lr, tot, dG, ws, stream=stream), stream), 4.0, 2 * 288 + 96)
        # the same window as fp32 already-gauged tensors (G NULL): 4 B per value in
        x32 = kv.float()
        st32 = cg.StatsDesc(16, 0, 1, 1.0, 0.02, 0.04)
        rec("stats_fwd_fp32_gauged", _time(lambda: cg.cg_spectral_stats(kvd, st32, x32, None, lf, lr, tot, None, ws, stream=stream), stream), 4.0, 2 * 144 + 32)
        del x32
        # decode-step attention from the 4-bit cache: every layer, 32 query heads, all 4096 tokens
        codec = cg.codec_desc(g=16, bits=4)
        c, sc, z = cg.alloc_encoded(kvd, codec, device=dev)
        cg.cg_encode(kvd, codec, kv, G16, 0, T, c, sc, z, None, stream=stream)
        at = cg.attn_desc(32, T, 0, Lc, d_head=D)
        q = torch.randn((Lc, B, 32, D), device=dev).to(torch.bfloat16)
        o = torch.empty((Lc, B, 32, D), dtype=torch.float32, device=dev)
        aws = torch.empty(cg.cg_decode_attention_workspace_size(kvd, at), dtype=torch.uint8, device=dev)
        rec("decode_attention_b4", _time(lambda: cg.cg_decode_attention(kvd, codec, at, q, c, sc, z, G16, o, aws, stream=stream), stream), 4 / 8 + 4 / 256)
        # gauge training: dL/dA of every g = 16 gauge, AdamW, and one whole step on this 4096-token window
        from quantization_cg_encode_b200.train import GaugeTrainer
        A = synth.gauge_params(Lc, H, D // 16, 16, sigma=0.1, seed=rank).to(dev)
        dA = torch.empty_like(A)
        m0, v0 = torch.zeros_like(A), torch.zeros_like(A)
        hp = cg.adamw_desc()
        ms = _time(lambda: cg.cg_gauge_grad(A, dG, dA, stream=stream), stream)
        rows["gauge_grad_g16"] = {"ms": round(ms, 4), "matrices": A.numel() // 256}
        A2 = A.clone()
        ms = _time(lambda: cg.cg_adamw_step(A2, dA, m0, v0, hp, 1, stream=stream), stream)
        rows["adamw_g16"] = {"ms": round(ms, 4), "params": A.numel()}
        tr = GaugeTrainer(A.clone(), kv.shape, stream=stream)
        ms = _time(lambda: tr.step(kv), stream, reps=3, warm=1)
        rows["train_step_4096tok_window"] = {"ms": round(ms, 4), "windows_per_s": round(1e3 / ms, 1)}
        gram = torch.empty((Lc, 2, H, D // 16, 16, 16), dtype=torch.float64, device=dev)
        rec("group_gram_g16", _time(lambda: cg.cg_group_gram(kvd, 16, kv, gram, stream=stream), stream), 2.0)
    cg.cg_sync_status(stream)
    rows["controls_nrmse_b4"] = control_nrmse(cg, synth, torch, kv, G16, stream, dev, rank)
    return rows


def control_nrmse(cg, synth, torch, kv, G16, stream, dev, rank):
    """Round-trip NRMSE ||x_hat - x|| / ||x|| of the 4-bit g = 16 codec (same rate for
    every gauge) under the coordinate controls: identity, Haar-random, DCT-II,
    Hadamard, PCA/KLT of this cache, the random exp(A) gauge, and the gauge after 16
    training steps on this window (lr 1e-2)."""
    from quantization_cg_encode_b200 import controls
    from quantization_cg_encode_b200.train import GaugeTrainer
    Lc, H = kv.shape[0], kv.shape[3]
    kvd = cg.kv_desc_of(kv)
    codec = cg.codec_desc(g=16, bits=4)
    c, sc, z = cg.alloc_encoded(kvd, codec, device=dev)
    out = torch.empty_like(kv)
    with torch.cuda.stream(stream):
        tr = GaugeTrainer(synth.gauge_params(Lc, H, D // 16, 16, sigma=0.1, seed=rank).to(dev), kv.shape,
                          hp=cg.adamw_desc(lr=1e-2), stream=stream)
        for _ in range(16):
            tr.step(kv)
        gauges = {"identity": synth.identity_gauge(Lc, H, D // 16, 16, device=dev),
                  "haar": synth.haar_gauge(Lc, H, D // 16, 16, seed=rank, device=dev),
                  "dct": synth.dct_gauge(Lc, H, D // 16, 16, device=dev),
                  "hadamard": controls.hadamard_gauge(Lc, H, D // 16, 16, device=dev),
                  "klt": controls.klt_gauge(kv, 16, stream=stream),
                  "random_exp": G16,
                  "trained_16_steps": tr.gauge().clone()}
        res = {}
        x = kv.float()
        nx = torch.linalg.vector_norm(x)
        for name, G in gauges.items():
            cg.cg_encode(kvd, codec, kv, G, 0, T, c, sc, z, None, stream=stream)
            cg.cg_decode(kvd, codec, c, sc, z, G, 0, T, out, stream=stream)
            res[name] = round(float(torch.linalg.vector_norm(out.float() - x) / nx), 5)
    cg.cg_sync_status(stream)
    return res


def _traffic_record(kernel, bits):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
    committed ncu record, or None when there is none for this kernel or its source
    has changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)["%s_b%d" % (kernel, bits)]
        with open(os.path.join(ROOT, "quantization_cg_encode_b200", "csrc", rec["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != rec["sha256"]:
                return None
        return int(rec["traffic"])
    except Exception:
        return None


# ---------------------------------------------------------------------------------------------
# CPU baseline / reference arm: the oracle, as it stands, on a bounded sample of the workload.

def _oracle_slice_roundtrip(x, G, bits):
    from oracle import codec as oc
    enc = oc.encode_block_uniform(x, G, bits)
    oc.decode_block_uniform(enc["codes"], enc["z"], enc["s"], G, bits)


def _oracle_inputs(seed):
    import numpy as np
    from oracle import gauge as og
    from quantization_cg_encode_b200 import synth
    kv = synth.kv_cache(1, B, 1, T, D, seed=seed, n_outliers=4)      # one (layer, head) of the cache
    A = synth.gauge_params(1, 1, D // G_GROUP, G_GROUP, sigma=0.1, seed=seed)
    G = og.gauge_from_A(A.numpy().astype(np.float64)).astype(np.float32).astype(np.float64)
    return kv.float().numpy().astype(np.float64), G


def _cpu_task(task):
    """One oracle unit of work on one host core (runs in a spawned worker)."""
    kind, seed, bits = task
    import numpy as np
    if kind == "warm":  # start-up: imports and one input, outside every timing
        _oracle_inputs(seed)
        return 0.0, 0
    x, G = _oracle_inputs(seed)
    t0 = time.perf_counter()
    if kind == "codec":
        _oracle_slice_roundtrip(x, G, bits)
    elif kind == "fullhead":
        from oracle import codec as oc
        from oracle import gauge as og
        from quantization_cg_encode_b200 import synth
        A = synth.gauge_params(1, 1, 1, 128, sigma=0.05, seed=seed)
        G1 = og.gauge_from_A(A.numpy().astype(np.float64)).astype(np.float32).astype(np.float64)
        enc = oc.encode_block_uniform(x, G1, bits, w=128, full_head_bf16=True)
        oc.decode_block_uniform(enc["codes"], enc["z"], enc["s"], G1, bits, w=128, full_head_bf16=True)
    else:  # stats: forward and dL/dG of one (layer, K/V, head) slice
        from oracle import spectral as sp
        sp.spectral_stats(x, G, want_grad=True)
    return time.perf_counter() - t0, int(x.size)


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _pool():
    import multiprocessing as mp
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = "1"  # one thread per worker: the pool supplies the parallelism
    n = os.cpu_count() or 1
    return mp.get_context("spawn").Pool(n), n


def cpu_baseline(bits, budget_s=15.0):
    """The oracle on every host core (a spawned process pool, one numpy thread per
    worker), each worker on whole (layer, head) slices of the 8B-shaped cache:
    encode + decode (the metric), plus a full-head leg and a statistics leg
    (forward + dL/dG of one slice); values per second of wall time."""
    pool, n = _pool()
    try:
        pool.map(_cpu_task, [("warm", i, bits) for i in range(n)])
        legs = {}
        for kind, share in (("codec", 0.6), ("fullhead", 0.2), ("stats", 0.2)):
            done_vals, rounds, t0 = 0, 0, time.perf_counter()
            while True:
                res = pool.map(_cpu_task, [(kind, rounds * n + i, bits) for i in range(n)])
                done_vals += sum(v for _, v in res)
                rounds += 1
                if time.perf_counter() - t0 > share * budget_s:
                    break
            el = time.perf_counter() - t0
            legs[kind] = {"values_per_s": round(done_vals / el, 1), "kv_GBps": round(2 * done_vals / el / 1e9, 6),
                          "slices": rounds * n, "seconds": round(el, 2)}
    finally:
        pool.close()
        pool.join()
    return {"value": legs["codec"]["kv_GBps"], "unit": "GB/s", "cores": n, "kind": "oracle",
            "cpu_model": _cpu_model(),
            "sample": "%d (layer, K+V, head) slices of 2x4096x128 values, encode + decode, %d worker processes with "
                      "one numpy thread each (%.1f s); full-head and statistics legs alongside"
                      % (legs["codec"]["slices"], n, legs["codec"]["seconds"]),
            "legs": legs}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return None
    pool, n = _pool()
    try:
        pool.map(_cpu_task, [("warm", i, args.bits) for i in range(n)])
        task = [("codec", i, args.bits) for i in range(n)]
        for _ in range(max(0, min(args.warmup, 1))):
            pool.map(_cpu_task, task)
        t0 = time.perf_counter()
        vals = 0
        for k in range(args.steps):
            vals += sum(v for _, v in pool.map(_cpu_task, [("codec", k * n + i, args.bits) for i in range(n)]))
        el = time.perf_counter() - t0
    finally:
        pool.close()
        pool.join()
    gbs = 2 * vals / el / 1e9
    ms = el / args.steps * 1e3
    line = {
        "impl": "reference",
        "metric": "KV GB/s for fused gauge+quant encode/decode at %d bits; %% of HBM roofline" % args.bits,
        "value": round(gbs, 5), "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 oracle (fp32-exact codec steps)", "data": "synthetic",
        "config": {"workload": "Llama-3-8B-shaped GQA KV cache 32x2x8x4096x128 bf16, g=16, 4-bit block-uniform; "
                               "each step a bounded sample: one (layer, head) K+V slice per host core"},
        "cpu_baseline": {"value": round(gbs, 5), "unit": "GB/s", "cores": n, "kind": "oracle",
                         "cpu_model": _cpu_model(),
                         "sample": "%d slices of 2x4096x128 values per step (one per worker process)" % n},
        "e2e": {"value": round(gbs, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--impl", default="cg", choices=["cg", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--layers", type=int, default=L, help="fewer layers for a small profiling case")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row kernel timings")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "cg":
        args.warmup = 3
    line = run_reference(args) if args.impl == "reference" else run_cg(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
