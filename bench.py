#!/usr/bin/env python
"""Benchmark of the batch-invariant, error-compensated decode layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one step): one decode_layer call -- RMSNorm, compensated QKV GEMM,
rotary embedding + INT16 quantisation into the cache, fixed-split attention
over a 2048-token INT16 KV cache, compensated output GEMM + residual,
RMSNorm, compensated gate/up GEMM, SwiGLU, compensated down GEMM + residual --
for B = 128 sequences of a 7B-like layer (hidden 4096, 32 query / 8 KV heads
of 128, MLP 11008).  Weights are random N(0, 0.02) fp32 packed once into the
hi/lo binary16 image; the KV cache holds 2047 synthetic tokens per sequence
and every step decodes position 2047 (2048 keys).  The rows come in a seeded
shuffled order of the cache slots.

Reported: tokens/s of the whole job (value: the step replayed as a CUDA graph
of the decode_layer call, inputs resident), the device-resident step time,
an end-to-end figure through the C ABI with host buffers (H2D of the step's
inputs and D2H of its output inside the timed region), per-kernel times from
CUDA events recorded around every kernel inside the timed region, the
roofline of the dominant kernel, SM clocks sampled during the run, and the
CPU oracle timed on a bounded sample of the same workload.  Components: the
compensated GEMM at the GEMM-sweep shapes, the decode attention at the
ragged-length shape and RMSNorm at 128 and 8192 rows, each against its
roofline.

Multi-GPU: replicas only -- every rank runs the full per-GPU workload on its
own device (weak scaling); the only cross-rank traffic is a barrier and the
max of the timings.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

H, HQ, HKV, D, F = 4096, 32, 8, 128, 11008
BATCH, KV_LEN = 128, 2048
REFERENCE_SECONDS = 60.0  # timed oracle work of the reference arm, at most
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_FP16_TFLOPS = 2250.0  # dense fp16/bf16 tensor-core figure of the B200 specification (context)
# Per-launch timings: after the L2 flush the GPU runs a fixed spin of this many
# clock cycles (~100 us) before the start event, so that the host's enqueue of
# the timed call (argument checks, tensor maps, launches) overlaps it and the
# events bracket the call's kernels only.
HOST_GAP_CYCLES = 200_000


def host_gap(torch) -> None:
    """The fixed GPU spin before a per-launch start event (skipped if this
    PyTorch build has no spin kernel)."""
    spin = getattr(torch.cuda, "_sleep", None)
    if spin is not None:
        spin(HOST_GAP_CYCLES)
# DRAM traffic per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)
# of the step's kernels, recorded by a capture of this benchmark's workload in
# profiles/dram_traffic.txt together with the SHA-256 of the kernel's source
# file at capture time: a record whose source has changed since is not used.
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.txt")
KERNEL_SOURCES = {"comp_gemm_kernel": "comp_gemm.cu", "qkv_attn_kernel": "comp_gemm.cu",
                  "attn_split_kernel": "attention.cu"}


def captured_traffic(kernel: str, workload: str, record: str = TRAFFIC_RECORD,
                     src_dir: str = os.path.join(ROOT, "invariant_numerics_b200", "csrc")):
    """(bytes per launch, note) from the capture record, or (None, why)."""
    import hashlib
    try:
        with open(record) as f:
            rec = json.load(f).get(kernel)
    except Exception:
        return None, "no capture record"
    if not rec or rec.get("workload") != workload:
        return None, "no capture of this workload"
    src = os.path.join(src_dir, KERNEL_SOURCES[kernel])
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if sha != rec.get("source_sha256"):
        return None, "kernel source changed since the capture"
    return rec["dram_bytes_per_launch"], rec.get("command", "")


def _numeric_leaves(obj, path=()):
    if isinstance(obj, dict):
        for k, v in obj.items():
            yield from _numeric_leaves(v, path + (str(k).lower(),))
    elif isinstance(obj, (int, float)) and not isinstance(obj, bool):
        yield "/".join(path), float(obj)


def load_peaks(path: str = os.path.join(ROOT, "MEASURED_PEAKS.json")):
    """Measured peaks of this GPU model (HBM copy GB/s, dense bf16 TFLOP/s as
    a burst and sustained), read from MEASURED_PEAKS.json at the repository
    root whatever its nesting: each figure is the first numeric entry whose
    key path names it.  A figure the file lacks (or a missing file) takes the
    fallback value, and the returned kind says which."""
    try:
        with open(path) as f:
            leaves = list(_numeric_leaves(json.load(f)))
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"
    want = {
        "hbm_gbs": lambda k: "hbm" in k and ("gbs" in k or "gb/s" in k or "gb_s" in k),
        "bf16_tflops": lambda k: "bf16" in k and "tflop" in k and "sustain" not in k,
        "bf16_tflops_sustained": lambda k: "bf16" in k and "tflop" in k and "sustain" in k,
    }
    peaks, found = {}, []
    for name, match in want.items():
        hit = next((v for k, v in leaves if match(k) and v > 0), None)
        peaks[name] = hit if hit is not None else PEAKS_FALLBACK[name]
        if hit is not None:
            found.append(name)
    if len(found) == len(want):
        return peaks, "measured"
    return peaks, "measured " + ",".join(found) + "; fallback for the rest" if found else "fallback"


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        busy = [r for r in rows if (num(r[9]) or 0) > 0] or rows
        sm = [num(r[1]) for r in busy if num(r[1]) is not None]
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in busy:
            for name, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][2]),
                "reasons": sorted(reasons), "samples": len(busy),
                "power_w_max": max((num(r[3]) or 0) for r in busy)}


# ------------------------------------------------------------ distributed --

from invariant_numerics_b200 import replicas  # noqa: E402


def cpu_cores_used() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------------ oracle --

def oracle_sample_inputs(rows: int, seed: int = 0):
    """Host inputs for the CPU oracle: the layer's weights and `rows` sequences
    with a (KV_LEN - 1)-token cache each."""
    from invariant_numerics_b200 import synth
    from oracle import reference as ref
    p = host_layer_params(seed)
    cache = ref.KVCache.empty(rows, HKV, KV_LEN, D)
    for b in range(rows):
        k = synth.kv_tensor(KV_LEN - 1, HKV, D, seed=seed + 100, stream=b)
        v = synth.kv_tensor(KV_LEN - 1, HKV, D, seed=seed + 200, stream=b)
        pos = np.arange(KV_LEN - 1)
        cache.write("k", k, np.full(KV_LEN - 1, b), pos)
        cache.write("v", v, np.full(KV_LEN - 1, b), pos)
    x = synth.normal((rows, H), seed=seed + 300)
    return p, cache, x


_PARAMS = {}


def host_layer_params(seed: int = 0):
    if seed in _PARAMS:
        return _PARAMS[seed]
    from invariant_numerics_b200 import synth
    from oracle import reference as ref
    s = lambda i, shape: synth.normal(shape, seed=seed, stream=i, std=0.02)
    p = ref.LayerParams(wq=s(1, (H, HQ * D)), wk=s(2, (H, HKV * D)), wv=s(3, (H, HKV * D)), wo=s(4, (HQ * D, H)),
                        w_gate=s(5, (H, F)), w_up=s(6, (H, F)), w_down=s(7, (F, H)),
                        g_attn=synth.uniform(H, seed=seed, stream=8, lo=0.5, hi=1.5),
                        g_mlp=synth.uniform(H, seed=seed, stream=9, lo=0.5, hi=1.5),
                        n_heads=HQ, n_kv_heads=HKV, head_dim=D)
    _PARAMS[seed] = p
    return p


def time_oracle(rows: int, min_seconds: float, max_calls: int = 1000):
    """Run the oracle decode layer on `rows` sequences until min_seconds pass."""
    from oracle import reference as ref
    p, cache, x = oracle_sample_inputs(rows)
    slot = np.arange(rows)
    pos = np.full(rows, KV_LEN - 1)
    calls, t0 = 0, time.perf_counter()
    while True:
        ref.decode_layer(p, cache, x, slot, pos)
        calls += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or calls >= max_calls:
            break
    return rows * calls / el, el, calls


def host_layer_params_threaded(seed: int, threads: int = 8):
    """host_layer_params with the seven weight matrices drawn in parallel
    threads (the same synth streams, so the same values)."""
    from concurrent.futures import ThreadPoolExecutor

    from invariant_numerics_b200 import synth
    from oracle import reference as ref
    shapes = {1: (H, HQ * D), 2: (H, HKV * D), 3: (H, HKV * D), 4: (HQ * D, H), 5: (H, F), 6: (H, F), 7: (F, H)}
    with ThreadPoolExecutor(threads) as ex:
        mats = dict(zip(shapes, ex.map(lambda i: synth.normal(shapes[i], seed=seed, stream=i, std=0.02), shapes)))
    return ref.LayerParams(wq=mats[1], wk=mats[2], wv=mats[3], wo=mats[4], w_gate=mats[5], w_up=mats[6],
                           w_down=mats[7], g_attn=synth.uniform(H, seed=seed, stream=8, lo=0.5, hi=1.5),
                           g_mlp=synth.uniform(H, seed=seed, stream=9, lo=0.5, hi=1.5),
                           n_heads=HQ, n_kv_heads=HKV, head_dim=D)


def _rowwise_err(got, want):
    got = np.asarray(got, np.float64).reshape(len(got), -1)
    want = np.asarray(want, np.float64).reshape(len(want), -1)
    return np.abs(got - want).max(axis=1) / np.maximum(np.abs(want).max(axis=1), 1e-300)


def stack_divergence(inv, torch, device, n_layers=32, vocab=32000, T=8192, prefix=512, n_dec=16, n_sample=64,
                     seed=5000, threads=8):
    """Per-layer divergence of the layer stack from the float64 CPU oracle,
    at the size of the chunked-prefill workload (32 layers, vocab 32000, an
    8192-token random prompt), by the two reduced oracle runs a full float64
    stack over 8192 tokens would be too slow for:

    * teacher-forced: the GPU prefills the whole prompt one shot, layer by
      layer; for every layer l the oracle takes the GPU's input to layer l at
      all 8192 positions, computes every position's K/V into its own INT16
      cache, and evaluates the rest of layer l at n_sample positions
      (oracle.reference.decode_layer_at).  Reported: max over those positions
      of the normwise error of the GPU's layer-l output -- each layer's own
      error, not accumulated.
    * free-running: the oracle runs its own float64 stack (hidden states
      rounded to fp32 between layers) over the first `prefix` prompt tokens
      followed by the n_dec tokens the GPU decoded greedily after that prefix.
      Reported: per layer, the max normwise distance between the GPU's and the
      oracle's hidden states (accumulated over depth), and how many of the
      GPU's greedy ids the oracle's argmax reproduces.

    Weights: synth N(0, 0.02) per layer (seed + 1 + l), embedding and LM head
    N(0, 0.02), final gain U(0.5, 1.5), prompt ids U{0..vocab-1}."""
    from concurrent.futures import ThreadPoolExecutor

    from invariant_numerics_b200 import synth
    from oracle import reference as ref
    t0 = time.perf_counter()
    cfg = inv.LayerConfig(hidden=H, n_heads=HQ, n_kv_heads=HKV, ffn=F, max_pos=T)
    rope = inv.rope_tables(T, device=device)
    embed = synth.normal((vocab, H), seed=seed, stream=100, std=0.02)
    g_final = synth.uniform(H, seed=seed, stream=101, lo=0.5, hi=1.5)
    lm_head = synth.normal((H, vocab), seed=seed, stream=102, std=0.02)
    prompt = synth.token_ids(T, vocab, seed=seed, stream=103)
    # sampled positions: split edges, the prefix edge, the ends, and random others
    fixed = np.unique(np.array([0, 1, 2, 255, 256, 257, prefix - 1, prefix, T // 2, T - 1]))
    fixed = fixed[(fixed >= 0) & (fixed < T)]
    others = [q for q in synth.permutation(T, seed=seed, stream=104) if q not in set(fixed.tolist())]
    sample = np.sort(np.concatenate([fixed, np.array(others[:max(0, n_sample - len(fixed))], np.int64)]))
    tdev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)

    params, gpu_w = [], []
    for l in range(n_layers):
        p = host_layer_params_threaded(seed + 1 + l, threads)
        params.append(p)
        gpu_w.append(inv.LayerWeights(cfg, tdev(p.wq), tdev(p.wk), tdev(p.wv), tdev(p.wo), tdev(p.w_gate),
                                      tdev(p.w_up), tdev(p.w_down), tdev(p.g_attn), tdev(p.g_mlp), rope=rope))
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    t_gen = time.perf_counter() - t0

    # GPU: one-shot prefill of the prompt, every layer's input kept on the host
    embed_d, gf_d = tdev(embed), tdev(g_final)
    lm_P, lm_e = inv.heal_pack_weight(tdev(lm_head))
    caches = [inv.KVCache(n_slots=1, n_kv_heads=HKV, max_len=T, device=device) for _ in range(n_layers)]
    x = inv.embed_gather(embed_d, tdev(prompt))
    X = [x.cpu().numpy()]
    for l in range(n_layers):
        x = inv.prefill_layer(cfg, gpu_w[l], caches[l], x, 0, 0)
        X.append(x.cpu().numpy())

    def head(rows):
        hi, lo = inv.rmsnorm_bi(rows, gf_d, 1e-6, want_y=False, want_split=True)
        return inv.argmax_rows(inv.comp_gemm(hi, lo, lm_P, lm_e))

    # GPU: n_dec greedy decode steps after the prefix (positions prefix ..; the
    # prompt run's cache entries there are no longer needed)
    ids = [int(head(x[prefix - 1:prefix].contiguous())[0])]
    dec = np.zeros((n_dec, n_layers, H), np.float32)
    zero = torch.zeros(1, dtype=torch.int32, device=device)
    for t in range(n_dec):
        xd = inv.embed_gather(embed_d, torch.tensor([ids[-1]], dtype=torch.int32, device=device))
        pos = torch.tensor([prefix + t], dtype=torch.int32, device=device)
        for l in range(n_layers):
            xd = inv.decode_layer(cfg, gpu_w[l], caches[l], xd, zero, pos)
            dec[t, l] = xd[0].cpu().numpy()
        ids.append(int(head(xd)[0]))
    st = inv.inv_get_device_status()
    if st != inv.INV_OK:
        raise RuntimeError(f"device status {inv.status_string(st)}")
    del gpu_w, caches, x, lm_P
    torch.cuda.empty_cache()
    t_gpu = time.perf_counter() - t0 - t_gen

    # oracle, teacher-forced at the sampled positions of every layer
    def teacher_forced(l):
        cache = ref.KVCache.empty(1, HKV, T, D)
        out = ref.decode_layer_at(params[l], cache, X[l], np.zeros(T, np.int64), np.arange(T), sample)
        return float(_rowwise_err(X[l + 1][sample], out).max())
    with ThreadPoolExecutor(threads) as ex:
        tf = list(ex.map(teacher_forced, range(n_layers)))
    t_tf = time.perf_counter() - t0 - t_gen - t_gpu

    # oracle, free-running over the prefix and the GPU's decoded tokens
    n = prefix + n_dec
    tokens = np.concatenate([prompt[:prefix], np.array(ids[:n_dec], np.int32)])
    sp = ref.StackParams(embed=embed, layers=params, g_final=g_final, lm_head=lm_head)
    ocaches = [ref.KVCache.empty(1, HKV, (n + 63) // 64 * 64, D) for _ in range(n_layers)]
    _, oids, ohidden = ref.stack_forward(sp, ocaches, tokens, np.zeros(n, np.int64), np.arange(n),
                                         return_hidden=True)
    fr = [float(_rowwise_err(np.concatenate([X[l + 1][:prefix], dec[:, l]]), ohidden[l]).max())
          for l in range(n_layers)]
    agree = int(np.sum(oids[prefix - 1:prefix - 1 + n_dec] == np.array(ids[:n_dec])))
    return {
        "layers": n_layers, "prompt_tokens": T, "vocab": vocab,
        "teacher_forced": {"positions": int(len(sample)), "per_layer_max_normwise": [float("%.3e" % e) for e in tf],
                           "max": float("%.3e" % max(tf))},
        "free_running": {"prefix_tokens": prefix, "decode_steps": n_dec,
                         "per_layer_max_normwise": [float("%.3e" % e) for e in fr], "max": float("%.3e" % max(fr)),
                         "greedy_ids_reproduced_by_oracle": f"{agree}/{n_dec}"},
        "seconds": {"weights": round(t_gen, 1), "gpu": round(t_gpu, 1), "oracle_teacher_forced": round(t_tf, 1),
                    "oracle_free_running": round(time.perf_counter() - t0 - t_gen - t_gpu - t_tf, 1)},
        "oracle_threads": threads,
    }


# ------------------------------------------------------------------- ours --

def build_gpu_layer(inv, torch, device, max_pos=0):
    p = host_layer_params(0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    cfg = inv.LayerConfig(hidden=H, n_heads=HQ, n_kv_heads=HKV, ffn=F, max_pos=max(KV_LEN, 8192, max_pos))
    w = inv.LayerWeights(cfg, t(p.wq), t(p.wk), t(p.wv), t(p.wo), t(p.w_gate), t(p.w_up), t(p.w_down),
                         t(p.g_attn), t(p.g_mlp))
    return cfg, w


def fill_cache(inv, torch, cache, n_tokens: int, seed: int):
    """Synthetic K/V for positions 0..n_tokens-1 of every slot, quantised by
    kv_quant_int16 (K/V ~ N(0,1) times a per-channel LogUniform(0.1, 10) factor)."""
    from invariant_numerics_b200 import synth
    dev = cache.k.device
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    scale = torch.from_numpy(synth.channel_scale(HKV, D, seed=seed)).to(dev)
    chunk = 512
    for s in range(cache.n_slots):
        for p0 in range(0, n_tokens, chunk):
            n = min(chunk, n_tokens - p0)
            slot = torch.full((n,), s, dtype=torch.int32, device=dev)
            pos = torch.arange(p0, p0 + n, dtype=torch.int32, device=dev)
            for which in ("k", "v"):
                x = torch.randn((n, HKV, D), generator=g, device=dev) * scale
                inv.kv_quant_int16(x.contiguous(), slot, pos, cache, which)


def layer_bytes(B, L):
    """Algorithmic HBM bytes of one decode-layer step and of its kernels."""
    Nqkv = (HQ + 2 * HKV) * D
    gemm = {  # packed weights (4 B / weight) + A hi/lo (4 B / element) + y fp32 (+ residual fp32)
        # QKV: its epilogue writes rotated q (fp32), the new K/V rows of the
        # cache (INT16 codes + fp32 scale) and reads the rows' rotary tables
        "gemm_qkv_rope_quant": 4 * H * Nqkv + 4 * B * H + 4 * B * HQ * D + B * 2 * HKV * (2 * D + 4) + B * 2 * 64 * 4,
        "gemm_o": 4 * HQ * D * H + 4 * B * HQ * D + 8 * B * H,
        "gemm_gate_up_swiglu": 4 * H * 2 * F + 4 * B * H + 4 * B * F,
        "gemm_down": 4 * F * H + 4 * B * F + 8 * B * H,
    }
    S = (L + 255) // 256
    attn_split = B * L * HKV * (2 * 2 * D + 2 * 4) + B * HQ * D * 4 + B * HQ * S * (D + 2) * 4
    return gemm, attn_split


def run_ours(args, rank, world, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    from invariant_numerics_b200 import build as _b
    if rank == 0:
        _b.build()
    if replicas.init("nccl", device=device):
        replicas.barrier()
        _b.build()  # no-op once rank 0 has built
    from invariant_numerics_b200 import invnum as inv
    from invariant_numerics_b200 import synth

    peaks, peak_kind = load_peaks()
    cfg, w = build_gpu_layer(inv, torch, device)
    cache = inv.KVCache(n_slots=BATCH, n_kv_heads=HKV, max_len=KV_LEN, device=device)
    fill_cache(inv, torch, cache, KV_LEN - 1, seed=replicas.replica_seed(1, rank))
    x = torch.from_numpy(synth.normal((BATCH, H), seed=replicas.replica_seed(2, rank))).to(device)
    slot = torch.from_numpy(synth.permutation(BATCH, seed=replicas.replica_seed(3, rank)).astype(np.int32)).to(device)
    pos = torch.full((BATCH,), KV_LEN - 1, dtype=torch.int32, device=device)
    y = torch.empty_like(x)
    call = inv.DecodeLayerCall(cfg, w, cache, x, slot, pos, y)
    stream = torch.cuda.current_stream()
    assert inv.inv_get_device_status() == inv.INV_OK

    barrier = replicas.barrier

    def max_over_ranks(v: float) -> float:
        return replicas.max_over_ranks(v, device=device)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()

    # ----- the step as a CUDA graph: one decode_layer call (8 kernels) captured
    # once; every launch argument (buffers, tensor maps) is fixed for the run
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        call()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.perf_counter()
    g0.record(stream)
    for k in range(args.steps):
        graph.replay()
    g1.record(stream)
    g1.synchronize()
    t_wall = time.perf_counter() - t_wall0
    # a short timed region (small --steps) gives the 100 ms clock sampler too
    # few points: keep replaying the same step, untimed, until 1.5 s have passed
    while time.perf_counter() - t_wall0 < 1.5:
        graph.replay()
        torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = max_over_ranks(g0.elapsed_time(g1) / args.steps)

    # ----- the same call without the graph, every kernel traced with CUDA events
    K = args.steps
    nk = inv.DECODE_LAYER_KERNELS
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for k in range(K):  # create the events outside the timed region
        for e in evs[k]:
            e.record()
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for k in range(K):
        inv.inv_trace_events(evs[k])
        call()
    end.record(stream)
    end.synchronize()
    inv.inv_trace_events(None)
    ms_traced = max_over_ranks(start.elapsed_time(end) / K)
    st = inv.inv_get_device_status()
    if st != inv.INV_OK:
        raise RuntimeError(f"device status {inv.status_string(st)}")
    kern_ms = {name: statistics.fmean(evs[k][2 * i].elapsed_time(evs[k][2 * i + 1]) for k in range(K))
               for i, name in enumerate(inv.DECODE_LAYER_KERNEL_NAMES)}

    # ----- end to end through the C ABI with host buffers: every step uploads
    # its inputs from pinned host memory and downloads its output.  Two buffer
    # sets alternate so that step k+1's upload and step k's download (on their
    # own copy streams) overlap step k's compute; all copies are inside the
    # timed region.
    x_host = x.cpu().pin_memory()
    slot_host = slot.cpu().pin_memory()
    pos_host = pos.cpu().pin_memory()
    y_hosts = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
    xs, ss, ps, ys = [x, torch.empty_like(x)], [slot, torch.empty_like(slot)], [pos, torch.empty_like(pos)], \
        [y, torch.empty_like(y)]
    graphs = [graph, torch.cuda.CUDAGraph()]
    call1 = inv.DecodeLayerCall(cfg, w, cache, xs[1], ss[1], ps[1], ys[1])
    xs[1].copy_(x)
    ss[1].copy_(slot)
    ps[1].copy_(pos)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call1()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graphs[1]):
        call1()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    calls = [call, call1]

    def e2e_run(step):
        """K steps of `step(buffer set)` with every step's upload and download
        inside the timed region; returns ms per step (max over ranks)."""
        up_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        down_done = [torch.cuda.Event() for _ in range(2)]
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_event(e0)
        down.wait_event(e0)
        for k in range(K):
            bi = k & 1
            up.wait_event(comp_done[bi])        # step k-2 has finished reading this input set
            with torch.cuda.stream(up):
                xs[bi].copy_(x_host, non_blocking=True)
                ss[bi].copy_(slot_host, non_blocking=True)
                ps[bi].copy_(pos_host, non_blocking=True)
                up_done[bi].record(up)
            stream.wait_event(up_done[bi])
            stream.wait_event(down_done[bi])    # step k-2's output has left this set
            step(bi)
            comp_done[bi].record(stream)
            down.wait_event(comp_done[bi])
            with torch.cuda.stream(down):
                y_hosts[bi].copy_(ys[bi], non_blocking=True)
                down_done[bi].record(down)
        stream.wait_event(down_done[0])
        stream.wait_event(down_done[1])
        e1.record(stream)
        e1.synchronize()
        assert torch.equal(y_hosts[(K - 1) & 1], ys[(K - 1) & 1].cpu())
        return max_over_ranks(e0.elapsed_time(e1) / K)

    # the public call every step (host validation, tensor maps, launches), and
    # the same call captured once as a CUDA graph and replayed
    e2e_ms = e2e_run(lambda bi: calls[bi](stream))
    e2e_graph_ms = e2e_run(lambda bi: graphs[bi].replay())
    h2d = x_host.numel() * 4 + slot_host.numel() * 4 + pos_host.numel() * 4
    d2h = y_hosts[0].numel() * 4

    # ----- rooflines: per kernel function, its share of the traced step; the
    # largest is the line's `roofline`, the next `roofline_second`
    gemm_b, attn_b = layer_bytes(BATCH, KV_LEN)
    hbm = peaks["hbm_gbs"]
    kernels = {}
    for name, t in kern_ms.items():
        ent = {"us": round(t * 1e3, 2)}
        byts = gemm_b.get(name, attn_b if name == "attn_split" else None)
        if byts is not None:
            ent["algorithmic_bytes"] = byts
            ent["gbs"] = round(byts / (t * 1e-3) / 1e9, 1)
            ent["frac_hbm"] = round(ent["gbs"] / hbm, 3)
        kernels[name] = ent
    traced_us = sum(kern_ms.values()) * 1e3
    workload = f"decode_layer H{H} Hq{HQ} Hkv{HKV} D{D} F{F} B{BATCH} kv{KV_LEN}"

    def roofline_of(kernel, names, byts_per_step):
        us = sum(kern_ms[n] for n in names) * 1e3
        launches = len(names)
        achieved = byts_per_step / (us * 1e-6) / 1e9
        traffic, src = captured_traffic(kernel, workload)
        return {"kernel": kernel, "launches_per_step": launches, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "traffic": round(traffic) if traffic is not None else None, "traffic_source": src,
                "algorithmic_bytes_per_launch": round(byts_per_step / launches),
                "us_per_launch": round(us / launches, 2), "share_of_traced_step": round(us / traced_us, 4),
                "peak_source": f"{peak_kind} hbm_gbs"}
    # kernel functions: comp_gemm_kernel (o, gate/up + SwiGLU, down), the QKV
    # GEMM with the fused rotary/quantise epilogue (qkv_attn_kernel), the
    # attention split kernel
    plain = [n for n in gemm_b if n != "gemm_qkv_rope_quant"]
    lines = sorted([roofline_of("comp_gemm_kernel", plain, sum(gemm_b[n] for n in plain)),
                    roofline_of("qkv_attn_kernel", ["gemm_qkv_rope_quant"], gemm_b["gemm_qkv_rope_quant"]),
                    roofline_of("attn_split_kernel", ["attn_split"], attn_b)],
                   key=lambda r: -r["share_of_traced_step"])
    step_bytes = sum(gemm_b.values()) + attn_b
    result = {
        "metric": "batch-invariant decode-layer tokens/s",
        "value": round(replicas.job_throughput(BATCH, world, ms), 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16 hi/lo products, f32 accumulate; int16 KV",
        "data": "synthetic",
        "config": {"workload": workload,
                   "global_batch": BATCH * world, "seq_len": KV_LEN, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (708.8 MB packed weights + 1.09 GB INT16 KV per step)"},
        "roofline": lines[0],
        "roofline_second": lines[1],
        "roofline_others": lines[2:],
        "step_roofline": {"bytes": step_bytes, "hbm_bound_ms": round(step_bytes / (hbm * 1e9) * 1e3, 4),
                          "frac": round(step_bytes / (hbm * 1e9) * 1e3 / ms, 4)},
        "kernels": kernels,
        "ms_per_step_without_graph": round(ms_traced, 4),
        "e2e": {"value": round(replicas.job_throughput(BATCH, world, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "call": "decode_layer through the C ABI every step (host validation and launches inside the region)"},
        "e2e_graph": {"value": round(replicas.job_throughput(BATCH, world, e2e_graph_ms), 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_graph_ms, 4),
                      "call": "the same decode_layer call captured once in a CUDA graph, replayed every step"},
        "gpu_launches": K * len(kern_ms),
        "clocks": clocks,
        "wall_s_timed": round(t_wall, 3),
    }

    if not args.no_components and rank == 0:
        result["components"] = bench_components(inv, torch, device, peaks, peak_kind)
        result["components"]["prefill"] = bench_prefill(inv, torch, device, cfg, w)
        result["components"]["decode_batch_sweep"] = bench_batch_sweep(inv, torch, cfg, w, cache, x, slot, pos,
                                                                      peaks)
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        # CPU-oracle leg (after every timed region): the oracle's own speed,
        # and the stack's divergence from it at the chunked-prefill size
        if not args.no_stack_divergence:
            result["stack_divergence"] = stack_divergence(inv, torch, device)
        v, el, ncalls = time_oracle(args.oracle_rows, args.oracle_seconds)
        result["cpu_baseline"] = {"value": round(v, 4), "unit": "tokens/s", "cores": cpu_cores_used(),
                                  "kind": "oracle",
                                  "sample": f"{args.oracle_rows} sequences x {ncalls} oracle decode_layer calls "
                                            f"(same layer shape, kv {KV_LEN}), {el:.1f} s"}
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                v1, el1, calls1 = time_oracle(args.oracle_rows, args.oracle_seconds / 2)
            result["cpu_baseline"]["value_1thread"] = round(v1, 4)
            result["cpu_baseline"]["sample_1thread"] = (f"{args.oracle_rows} sequences x {calls1} calls with the "
                                                        f"BLAS pool limited to 1 thread, {el1:.1f} s")
        except ImportError:
            result["cpu_baseline"]["value_1thread"] = None
    replicas.barrier()
    del graph, graphs
    replicas.finalize()
    if rank == 0:
        print(json.dumps(result), flush=True)


def bench_components(inv, torch, device, peaks, peak_kind):
    """Compensated GEMM (K 4096, N 4096/11008, M 1..1024), decode attention
    (32/8 heads, ragged lengths U(128, 8192), B 64 and its first 1..32 rows)
    and RMSNorm (hidden 4096, 128 and 8192 rows), each timed per launch with
    CUDA events, L2 flushed between launches."""
    from invariant_numerics_b200 import synth
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    tc_peak = peaks["bf16_tflops"]

    def timed(fn, reps=5):
        ts = []
        for r in range(reps + 2):
            flush.zero_()
            host_gap(torch)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            if r >= 2:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    K = 4096
    A = torch.from_numpy(synth.normal_with_outliers((1024, K), seed=10)).to(device)
    hi, lo = inv.heal_split(A)
    gem = {}
    for N in (4096, 11008):
        W = torch.from_numpy(synth.normal((K, N), seed=11, std=0.02)).to(device)
        P, e = inv.heal_pack_weight(W)
        del W
        for M in (1, 3, 17, 64, 256, 1024):
            a_hi, a_lo = hi[:M].contiguous(), lo[:M].contiguous()
            y = torch.empty((M, N), dtype=torch.float32, device=device)
            t = timed(lambda: inv.comp_gemm(a_hi, a_lo, P, e, out=y))
            useful = 2.0 * M * N * K / (t * 1e-3) / 1e12
            byts = 4 * N * K + 4 * M * K + 4 * M * N
            gbs = byts / (t * 1e-3) / 1e9
            gem[f"M{M}_N{N}"] = {"us": round(t * 1e3, 2), "useful_tflops": round(useful, 2),
                                 "frac_of_peak_over_3": round(useful / (tc_peak / 3), 4),
                                 "frac_of_nominal_over_3": round(useful / (NOMINAL_FP16_TFLOPS / 3), 4),
                                 "gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    out["comp_gemm"] = {"shapes": gem, "peak_tflops": tc_peak, "peak_source": f"{peak_kind} bf16_tflops (fp16 = bf16 rate)",
                        "nominal_tflops": NOMINAL_FP16_TFLOPS,
                        "target": ">= 0.5 x peak / 3 useful at M 256, 1024"}

    B = 64
    lens = synth.ragged_lengths(B, seed=40)
    cache = inv.KVCache(n_slots=B, n_kv_heads=HKV, max_len=8192, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(41)
    for b in range(B):
        L = int(lens[b])
        sl = torch.full((L,), b, dtype=torch.int32, device=device)
        ps = torch.arange(L, dtype=torch.int32, device=device)
        for which in ("k", "v"):
            inv.kv_quant_int16(torch.randn((L, HKV, D), generator=g, device=device), sl, ps, cache, which)
    q = torch.from_numpy(synth.normal((B, HQ, D), seed=42)).to(device)
    slot = torch.arange(B, dtype=torch.int32, device=device)
    lens_d = torch.from_numpy(lens).to(device)
    o = torch.empty_like(q)
    ws = torch.empty(inv.attn_decode_workspace_size(B, HQ, 8192), dtype=torch.uint8, device=device)
    t = timed(lambda: inv.attn_decode_fixedsplit(q, cache, slot, lens_d, 0.08838834764831845, out=o, workspace=ws))
    def attn_bytes(ls):
        S = (ls.astype(np.int64) + 255) // 256
        return int(ls.astype(np.int64).sum()) * HKV * 520 + len(ls) * HQ * D * 4 * 2 + int(S.sum()) * HQ * (D + 2) * 4 * 2
    byts = attn_bytes(lens)
    gbs = byts / (t * 1e-3) / 1e9
    # the same call on the first Bs sequences of the cache
    sweep = {}
    for Bs in (1, 2, 4, 8, 16, 32, 64):
        qs, ss, ls, os_ = q[:Bs].contiguous(), slot[:Bs].contiguous(), lens_d[:Bs].contiguous(), o[:Bs]
        ts = timed(lambda: inv.attn_decode_fixedsplit(qs, cache, ss, ls, 0.08838834764831845, out=os_, workspace=ws))
        bs = attn_bytes(lens[:Bs])
        sweep[f"B{Bs}"] = {"mean_len": float(lens[:Bs].mean()), "us": round(ts * 1e3, 2), "bytes": bs,
                           "gbs": round(bs / (ts * 1e-3) / 1e9, 1),
                           "frac_hbm": round(bs / (ts * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    out["attention_batch_sweep"] = sweep
    # LAMP variant on the same workload: time, recompute rate, distance from the plain call
    lamp = {}
    for tau in (0.01, 0.1, 1.0):
        tl = timed(lambda: inv.attn_decode_lamp(q, cache, slot, lens_d, 0.08838834764831845, tau, out=o,
                                                workspace=ws))
        ol, rec = inv.attn_decode_lamp(q, cache, slot, lens_d, 0.08838834764831845, tau, want_recompute=True,
                                       workspace=ws)
        plain = inv.attn_decode_fixedsplit(q, cache, slot, lens_d, 0.08838834764831845, workspace=ws)
        valid = torch.arange(rec.shape[2], device=device)[None, None, :] < lens_d[:, None, None]
        rate = float(rec[valid.expand_as(rec)].float().mean())
        dist = float(((ol - plain).abs().amax(-1) / plain.abs().amax(-1)).max())
        lamp[f"tau{tau}"] = {"us": round(tl * 1e3, 2), "gbs": round(byts / (tl * 1e-3) / 1e9, 1),
                             "recompute_rate": round(rate, 5), "max_normwise_distance_from_plain": dist}
    out["attention_lamp"] = lamp
    out["attention"] = {"B": B, "mean_len": float(lens.mean()), "us": round(t * 1e3, 2), "gbs": round(gbs, 1),
                        "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "bytes": byts,
                        "note": "one attn_decode_fixedsplit call (split kernel + ordered combine kernel), "
                                "L2 flushed between launches"}
    # RMSNorm at hidden 4096: the decode step's 128 rows and a prompt's 8192
    # rows, with the layer's binary16 hi/lo output and with fp32 output as well;
    # bytes = x read + outputs written (gamma is 16 KB and stays in L2)
    Hn = 4096
    gamma = torch.from_numpy(synth.uniform((Hn,), seed=50, lo=0.5, hi=1.5)).to(device)
    norm = {}
    for rows in (128, 8192):
        xn = torch.from_numpy(synth.normal((rows, Hn), seed=51)).to(device)
        for want_y, tag in ((False, "split"), (True, "y_and_split")):
            t = timed(lambda: inv.rmsnorm_bi(xn, gamma, 1e-6, want_y=want_y, want_split=True))
            byts = rows * Hn * (4 + 4 + (4 if want_y else 0))
            gbs = byts / (t * 1e-3) / 1e9
            norm[f"rows{rows}_{tag}"] = {"us": round(t * 1e3, 2), "bytes": byts, "gbs": round(gbs, 1),
                                         "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        del xn
    out["rmsnorm"] = {"shapes": norm, "note": "one rmsnorm_bi call (one CTA per row, fixed reduction order), "
                                              "L2 flushed between launches"}
    assert inv.inv_get_device_status() == inv.INV_OK
    return out


def bench_prefill(inv, torch, device, cfg, w, T=8192, chunk=512):
    """One layer over a T-token prompt of one sequence: prefill_layer one shot
    and in chunks (each attention split is loaded once per chunk)."""
    from invariant_numerics_b200 import synth
    max_len = (T + 63) // 64 * 64
    pcfg = inv.LayerConfig(hidden=cfg.hidden, n_heads=cfg.n_heads, n_kv_heads=cfg.n_kv_heads, ffn=cfg.ffn,
                           max_pos=cfg.max_pos)
    if pcfg.max_pos < max_len:
        return {"skipped": f"rotary tables cover {pcfg.max_pos} positions < {T}"}
    x = torch.from_numpy(synth.normal((T, cfg.hidden), seed=77)).to(device)
    out = {}
    for name, step in (("one_shot", T), (f"chunk{chunk}", chunk)):
        cache = inv.KVCache(n_slots=1, n_kv_heads=cfg.n_kv_heads, max_len=max_len, device=device)
        y = torch.empty_like(x)

        def run():
            for a in range(0, T, step):
                inv.prefill_layer(pcfg, w, cache, x[a:a + step], 0, a, out=y[a:a + step])
        run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        e1.synchronize()
        ms = e0.elapsed_time(e1)
        out[name] = {"ms": round(ms, 3), "tokens_per_s": round(T / (ms * 1e-3), 1)}
    assert inv.inv_get_device_status() == inv.INV_OK
    out["tokens"] = T
    return out


def bench_batch_sweep(inv, torch, cfg, w, cache, x, slot, pos, peaks, batches=(1, 8, 32), reps=300):
    """The same decode step at smaller batches (the first B sequences of the
    bench cache), each replayed as a CUDA graph: tokens/s and the fraction of
    the step's HBM roofline (weights + KV + activations at the measured copy
    bandwidth)."""
    out = {}
    L = KV_LEN
    for B in batches:
        if B > x.shape[0]:
            continue
        xb, sb, pb = x[:B].clone(), slot[:B].clone(), pos[:B].clone()
        yb = torch.empty_like(xb)
        call = inv.DecodeLayerCall(cfg, w, cache, xb, sb, pb, yb)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            call()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        ms = e0.elapsed_time(e1) / reps
        gemm, attn = layer_bytes(B, L)
        total = sum(gemm.values()) + attn
        bound_ms = total / (peaks["hbm_gbs"] * 1e9) * 1e3
        out[f"B{B}"] = {"ms_per_step": round(ms, 4), "tokens_per_s": round(B / (ms * 1e-3), 1),
                        "hbm_roofline_frac": round(bound_ms / ms, 4)}
        del g
    assert inv.inv_get_device_status() == inv.INV_OK
    return out


# -------------------------------------------------------------- reference --

def run_reference(args, rank, world):
    """The CPU oracle as it stands, on a bounded sample of the same workload."""
    if rank != 0:
        return
    rows = args.oracle_rows
    times = []
    from oracle import reference as ref
    p, cache, x = oracle_sample_inputs(rows)
    slot = np.arange(rows)
    pos = np.full(rows, KV_LEN - 1)
    # One step is one oracle decode_layer call on `rows` sequences (~0.1-0.3 s
    # each).  So that the run stays within a few minutes whatever --steps is,
    # warm-up is capped at 3 calls and the timed calls stop after ~60 s of
    # oracle time; the line reports how many calls were timed.
    warm = min(args.warmup, 3)
    for _ in range(warm):
        ref.decode_layer(p, cache, x, slot, pos)
    t_start = time.perf_counter()
    for _ in range(args.steps):
        t0 = time.perf_counter()
        ref.decode_layer(p, cache, x, slot, pos)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start > REFERENCE_SECONDS:
            break
    ms = statistics.fmean(times) * 1e3
    v = rows / (ms * 1e-3)
    sample = (f"{len(times)} timed float64 oracle decode_layer calls of {rows} sequences (kv {KV_LEN}) "
              f"for {args.steps} requested steps, {warm} warm-up calls")
    print(json.dumps({
        "impl": "reference", "metric": "batch-invariant decode-layer tokens/s", "value": round(v, 4),
        "unit": "tokens/s", "n_gpus": world, "steps": len(times), "steps_requested": args.steps,
        "warmup": warm,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"decode_layer H{H} Hq{HQ} Hkv{HKV} D{D} F{F} B{BATCH} kv{KV_LEN}",
                   "global_batch": BATCH * world, "seq_len": KV_LEN, "parallelism": "cpu oracle, rank 0"},
        "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s", "cores": cpu_cores_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_gemm_only(args, local):
    """One compensated GEMM shape, timed with CUDA events (inputs larger than L2
    are flushed by a 256 MB write before every launch)."""
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    from invariant_numerics_b200 import build as _b
    _b.build()
    from invariant_numerics_b200 import invnum as inv
    from invariant_numerics_b200 import synth
    M, N, K = args.gemm
    A = torch.from_numpy(synth.normal_with_outliers((M, K), seed=10)).to(device)
    W = torch.from_numpy(synth.normal((K, N), seed=11, std=0.02)).to(device)
    hi, lo = inv.heal_split(A)
    P, e = inv.heal_pack_weight(W)
    y = torch.empty((M, N), dtype=torch.float32, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    ts = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        host_gap(torch)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        inv.comp_gemm(hi, lo, P, e, out=y)
        b.record()
        b.synchronize()
        if i >= args.warmup:
            ts.append(a.elapsed_time(b))
    st = inv.inv_get_device_status()
    if st != inv.INV_OK:
        raise RuntimeError(f"device status {inv.status_string(st)}")
    peaks, kind = load_peaks()
    us = statistics.median(ts) * 1e3
    tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
    print(json.dumps({"metric": "comp_gemm useful TFLOP/s", "value": round(tf, 2), "unit": "TFLOP/s",
                      "config": {"workload": f"comp_gemm M{M} N{N} K{K}"}, "us": round(us, 2),
                      "frac_of_peak_over_3": round(tf / (peaks["bf16_tflops"] / 3.0), 4),
                      "steps": args.steps, "warmup": args.warmup}))


def run_rmsnorm_only(args, local):
    """One rmsnorm_bi shape (rows x hidden, binary16 hi/lo output as the layer
    uses it), timed with CUDA events after a 256 MB write that flushes L2."""
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    from invariant_numerics_b200 import build as _b
    _b.build()
    from invariant_numerics_b200 import invnum as inv
    from invariant_numerics_b200 import synth
    rows, hidden = args.rmsnorm, args.hidden
    x = torch.from_numpy(synth.normal((rows, hidden), seed=51)).to(device)
    gamma = torch.from_numpy(synth.uniform((hidden,), seed=50, lo=0.5, hi=1.5)).to(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    ts = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        host_gap(torch)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        inv.rmsnorm_bi(x, gamma, 1e-6, want_y=False, want_split=True)
        b.record()
        b.synchronize()
        if i >= args.warmup:
            ts.append(a.elapsed_time(b))
    st = inv.inv_get_device_status()
    if st != inv.INV_OK:
        raise RuntimeError(f"device status {inv.status_string(st)}")
    peaks, kind = load_peaks()
    us = statistics.median(ts) * 1e3
    byts = rows * hidden * 8   # fp32 x read, binary16 hi and lo written
    gbs = byts / (us * 1e-6) / 1e9
    print(json.dumps({"metric": "rmsnorm_bi GB/s", "value": round(gbs, 1), "unit": "GB/s",
                      "config": {"workload": f"rmsnorm_bi rows{rows} hidden{hidden} hi/lo out"}, "us": round(us, 2),
                      "bytes": byts, "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "peak_source": kind,
                      "steps": args.steps, "warmup": args.warmup}))


def run_prefill_only(args, local):
    """prefill_layer over one T-token sequence (one layer), one shot, timed with
    CUDA events per call; one JSON line (for profiling the prefill kernels)."""
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    from invariant_numerics_b200 import build as _b
    _b.build()
    from invariant_numerics_b200 import invnum as inv
    from invariant_numerics_b200 import synth
    T = args.prefill
    cfg, w = build_gpu_layer(inv, torch, device, max_pos=T)
    x = torch.from_numpy(synth.normal((T, H), seed=77)).to(device)
    y = torch.empty_like(x)
    cache = inv.KVCache(n_slots=1, n_kv_heads=HKV, max_len=(T + 63) // 64 * 64, device=device)
    ts = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        inv.prefill_layer(cfg, w, cache, x, 0, 0, out=y)
        b.record()
        b.synchronize()
        if i >= args.warmup:
            ts.append(a.elapsed_time(b))
    st = inv.inv_get_device_status()
    if st != inv.INV_OK:
        raise RuntimeError(f"device status {inv.status_string(st)}")
    ms = statistics.median(ts)
    print(json.dumps({"metric": "prefill_layer tokens/s", "value": round(T / (ms * 1e-3), 1), "unit": "tokens/s",
                      "config": {"workload": f"prefill_layer H{H} Hq{HQ} Hkv{HKV} D{D} F{F} T{T} one-shot"},
                      "ms": round(ms, 3), "steps": args.steps, "warmup": args.warmup}))


def main():
    global BATCH, KV_LEN, H, HQ, HKV, F
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stack-divergence", action="store_true",
                    help="skip the 32-layer divergence-from-oracle report of the CPU-oracle leg")
    ap.add_argument("--hidden", type=int, default=H)
    ap.add_argument("--heads", type=int, default=HQ)
    ap.add_argument("--kv-heads", type=int, default=HKV)
    ap.add_argument("--ffn", type=int, default=F)
    ap.add_argument("--batch", type=int, default=BATCH, help="sequences per GPU (profiling of smaller cases)")
    ap.add_argument("--kv", type=int, default=KV_LEN, help="KV length per sequence, multiple of 64")
    ap.add_argument("--oracle-rows", type=int, default=2)
    ap.add_argument("--oracle-seconds", type=float, default=10.0)
    ap.add_argument("--gemm", type=int, nargs=3, metavar=("M", "N", "K"),
                    help="time one compensated GEMM shape only (one JSON line; for profiling)")
    ap.add_argument("--prefill", type=int, metavar="T",
                    help="time prefill_layer over one T-token sequence only (one JSON line; for profiling)")
    ap.add_argument("--rmsnorm", type=int, metavar="ROWS",
                    help="time rmsnorm_bi over ROWS x hidden only (one JSON line; for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    BATCH, KV_LEN = args.batch, args.kv
    H, HQ, HKV, F = args.hidden, args.heads, args.kv_heads, args.ffn
    if KV_LEN % 64 != 0 or KV_LEN < 64:
        raise SystemExit("--kv must be a positive multiple of 64")
    rank, world, local = replicas.env_ranks()
    if world > 1 and world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.gemm:
        run_gemm_only(args, local)
    elif args.prefill:
        run_prefill_only(args, local)
    elif args.rmsnorm:
        run_rmsnorm_only(args, local)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
