#!/usr/bin/env python
"""Decode-attention throughput over a packed 3-bit (2+1) KV cache.

Workload (default): Llama-3.1-8B-shaped GQA decode - 32 layers, batch 16,
32 query heads over 8 KV heads, head_dim 128, 32768 cached tokens per
sequence, bf16 heavy-tailed K/V (N(0,1) + 4 outlier channels x20 per
(layer, kv-head)), 2-bit Lloyd-Max codes + 1-bit QJL (m = 128).

One step = one decode step of the whole model's attention: for every layer,
one tq_decode_attention_append call quantizes the new token's K and V into
record T-1 of each sequence in the same launch as the query preparation,
then scores the query against all T cached tokens (split-KV kernel, merge).  The packed cache (15 GB) is far larger than L2, so no flush is
needed between steps.

Metric: cached tokens scored per second, one unit = one (layer, sequence,
kv-head, token) K+V record pair scored for all 4 query heads of its group.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs an independent replica of the
workload (the path shards by sequence with no exchange: weak scaling), the
elapsed device time is the max over ranks and rank 0 prints the JSON line.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOAD = "llama31_8b_gqa_decode"
METRIC = "cached tokens scored/s (decode attn, 3-bit KV); % of B200 HBM roofline"
UNIT = "tokens/s"


# ncu dram__bytes_read.sum + dram__bytes_write.sum of decode_split_kernel<2,4>
# per cached token (235,720,704 + 5,453,056 B over 16*8*16384 tokens), or None
# when the kernel has changed since that capture.
SPLIT_TRAFFIC_PER_TOKEN = (235_720_704 + 5_453_056) / (16 * 8 * 16384)

EXTRAS = ("encode_70b_slice", "decode_70b_slice", "encoder_esm2_layer", "search_1m_d1536", "decode_llama8b_layer_3p1",
          "decode_llama8b_layer_window", "tiny_d128_t1024", "encode_esm2_33_layers", "memory_esm2",
          "decode_llama8b_layer_nsn")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--bits", type=int, default=2, help="Lloyd-Max code bits (QJL adds 1)")
    ap.add_argument("--layers", type=int, default=None, help="override layer count (testing only)")
    ap.add_argument("--context", type=int, default=None, help="override context length (testing only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the secondary workload measurements")
    ap.add_argument("--extra", action="append", choices=EXTRAS, default=None,
                    help="run only this secondary workload (repeatable) and print its measurement")
    ap.add_argument("--slice-tokens", type=int, default=None,
                    help="context of the 70B-shaped slice for --extra runs (default 2^20)")
    ap.add_argument("--search-rows", type=int, default=None,
                    help="database rows of the search workload for --extra runs (default 10^6)")
    ap.add_argument("--esm-layers", type=int, default=None,
                    help="layers of the ESM-2-shaped cache encode for --extra runs (default 33)")
    return ap.parse_args()


def shape(args):
    c = dict(__import__("synth").CONFIGS[WORKLOAD])
    if args.layers:
        c["layers"] = args.layers
    if args.context:
        c["tokens"] = args.context
    return c


def config_json(c, args, world):
    return {"workload": WORKLOAD, "layers": c["layers"], "batch": c["batch"], "q_heads": c["q_heads"],
            "kv_heads": c["kv_heads"], "head_dim": c["head_dim"], "context": c["tokens"],
            "bits": f"{args.bits}+1", "qjl_m": c["head_dim"], "kv_dtype_in": "bf16",
            "cache_bytes_per_step": c["layers"] * c["batch"] * c["kv_heads"] * c["tokens"] * 2 * rec_bytes(c, args),
            "l2": "inputs > L2, no flush",
            "parallelism": f"replicas x{world} (weak)" if world > 1 else "single GPU"}


def rec_bytes(c, args):
    d = c["head_dim"]
    return args.bits * d // 8 + d // 8 + 8


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------- oracle baseline
def oracle_baseline(c, args, budget_s=12.0, max_steps=None):
    """Time the oracle decode on a bounded sample: one (layer, sequence,
    kv-head) slice of the workload per step, on the host cores."""
    import synth
    from oracle import attention as at
    from oracle import codec, rotation as ro
    d, T, G = c["head_dim"], c["tokens"], c["q_heads"] // c["kv_heads"]
    rk = ro.build_rotation(d, args.bits, synth.rotation_randomness(d, c["seed"]), rope_base=c["rope_base"])
    rv = ro.build_rotation(d, args.bits, synth.rotation_randomness(d, c["seed"] + 7777))
    k = synth.heavy_tailed((1, 1, T, d), [c["seed"], 1]).reshape(T, d)
    v = synth.heavy_tailed((1, 1, T, d), [c["seed"], 2]).reshape(T, d)
    q = synth.heavy_tailed((1, G, d), [c["seed"], 3])

    def packed(rot, x, pos):
        e = codec.encode(rot, x, pos)
        return (codec.pack_planes(e["codes"], rot.bits)[None, None], codec.pack_bits(e["signs"])[None, None],
                np.stack([e["norm"], e["rnorm"]], 1).astype(np.float32)[None, None])

    kc, vc = packed(rk, k, np.arange(T)), packed(rv, v, None)
    times = []
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        at.decode_attention(rk, rv, q, [T - 1], kc, vc, 1 / np.sqrt(d))
        times.append(time.perf_counter() - t0)
        if (max_steps and len(times) >= max_steps) or (not max_steps and time.perf_counter() - t_start > budget_s):
            break
    per = float(np.mean(times[1:] if len(times) > 1 else times))
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    return {"value": T / per, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"1 layer x 1 seq x 1 kv-head ({T} tokens, {G} q-heads) per step, {len(times)} steps"}, \
        len(times), per



def _oracle_rate(fn, units, min_s=1.5):
    """Units per second of fn on the host cores: at least one call and min_s."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= min_s:
            return units * n / el, n, el / n


def oracle_extra_baselines(select):
    """The oracle as it stands timed beside each secondary line, on a bounded
    sample of that line's workload (same laws and sizes per unit), in that
    line's unit."""
    import synth
    from oracle import attention as at
    from oracle import codec, rotation as ro
    from oracle import search as osearch
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    out = {}

    def base(value, unit, sample):
        return {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample}

    def packed(rot, x, pos):
        e = codec.encode(rot, x, pos)
        return (codec.pack_planes(e["codes"], rot.bits)[None, None], codec.pack_bits(e["signs"])[None, None],
                np.stack([e["norm"], e["rnorm"]], 1).astype(np.float32)[None, None])

    d = 128
    if select & {"encode_70b_slice", "decode_70b_slice"}:
        c = synth.CONFIGS["llama31_70b_long_slice"]
        n = 8192
        rk = ro.build_rotation(d, 2, synth.rotation_randomness(d, [c["seed"], 1]), rope_base=c["rope_base"])
        rv = ro.build_rotation(d, 2, synth.rotation_randomness(d, [c["seed"], 2]))
        k = synth.heavy_tailed((1, 1, n, d), [c["seed"], 91]).reshape(n, d)
        v = synth.heavy_tailed((1, 1, n, d), [c["seed"], 92]).reshape(n, d)
        if "encode_70b_slice" in select:
            ne = 4096
            r, calls, per = _oracle_rate(lambda: (codec.encode(rk, k[:ne], np.arange(ne)), codec.encode(rv, v[:ne])),
                                         2 * ne)
            out["encode_70b_slice"] = base(r, "vectors/s", f"{ne} keys (RoPE) + {ne} values, d 128, 2+1 bits; "
                                                           f"{calls} calls, {per:.2f} s each")
        if "decode_70b_slice" in select:
            G = c["q_heads"] // c["kv_heads"]
            kc, vc = packed(rk, k, np.arange(n)), packed(rv, v, None)
            q = synth.heavy_tailed((1, G, d), [c["seed"], 93])
            r, calls, per = _oracle_rate(lambda: at.decode_attention(rk, rv, q, [n - 1], kc, vc, 1 / np.sqrt(d)), n)
            out["decode_70b_slice"] = base(r, "tokens/s", f"one KV head with its {G} query heads over {n} cached "
                                                          f"tokens (the slice has 2^20; the oracle's time is linear "
                                                          f"in tokens); {calls} calls, {per:.2f} s each")
    if "encoder_esm2_layer" in select:
        c = synth.CONFIGS["esm2_650m_encoder"]
        T, de = c["tokens"], c["head_dim"]
        rk = ro.build_rotation(de, 2, synth.rotation_randomness(de, [c["seed"], 1]), rope_base=c["rope_base"])
        rv = ro.build_rotation(de, 2, synth.rotation_randomness(de, [c["seed"], 2]))
        x = synth.lognormal_channels((1, 3, T, de), [c["seed"], 94])
        kc, vc = packed(rk, x[0, 0], np.arange(T)), packed(rv, x[0, 1], None)
        q = x[:, 2:3]
        flops = 2 * T * T * 2 * (de + de)
        r, calls, per = _oracle_rate(lambda: at.encoder_attention(rk, rv, q, kc, vc, 1 / np.sqrt(de)), flops / 1e12)
        out["encoder_esm2_layer"] = base(r, "TFLOP/s", f"one head of the layer (S = T = {T}, d {de}, 2+1 bits; the "
                                                       f"layer has {c['batch'] * c['heads']}); {calls} calls, "
                                                       f"{per:.2f} s each")
    for key, bits in (("search_1m_d1536", 1), ("search_1m_d1536_3p1", 3)):
        if "search_1m_d1536" not in select:
            break
        c = synth.CONFIGS["vector_search_d1536"]
        N, ds, nq = 4096, c["dim"], 4
        rot = ro.build_rotation(ds, bits, synth.rotation_randomness(ds, c["seed"] + bits, dense=True), "dense")
        basis = synth.haar_basis(ds, c["seed"])
        db = synth.anisotropic(N, ds, [c["seed"], 95], basis)
        qs = synth.anisotropic(nq, ds, [c["seed"], 96], basis)
        e = codec.encode(rot, db)
        codes, signs = e["codes"], e["signs"]
        norms = np.stack([e["norm"], e["rnorm"]], 1)

        def run():
            sc = osearch.search_scores(rot, qs, codes, signs, norms)
            for row in sc:
                osearch.topk_desc(row, c["top_k"])
        r, calls, per = _oracle_rate(run, nq * N / c["n_db"])
        out[key] = base(r, "queries/s", f"{nq} queries over {N} of the {c['n_db']} database vectors, d {ds}, "
                                        f"{bits}+1 bits, top-{c['top_k']}, scaled to the full database; "
                                        f"{calls} calls, {per:.2f} s each")
    if "tiny_d128_t1024" in select:
        c = synth.CONFIGS["tiny_d128_t1024"]
        T, seed = c["tokens"], c["seed"]
        rk = ro.build_rotation(d, 2, synth.rotation_randomness(d, [seed, 9, 1]), rope_base=c["rope_base"])
        rv = ro.build_rotation(d, 2, synth.rotation_randomness(d, [seed, 9, 2]))
        k = synth.heavy_tailed((1, 1, T, d), [seed, 9, 3]).reshape(T, d)
        v = synth.heavy_tailed((1, 1, T, d), [seed, 9, 4]).reshape(T, d)
        q = synth.heavy_tailed((1, 1, d), [seed, 9, 5])
        t0 = time.perf_counter()
        kc, vc = packed(rk, k, np.arange(T)), packed(rv, v, None)
        t_enc = time.perf_counter() - t0
        _, calls, per = _oracle_rate(lambda: at.decode_attention(rk, rv, q, [T - 1], kc, vc, 1 / np.sqrt(d)), 1)
        out["tiny_d128_t1024"] = {"value": per * 1e6, "unit": "decode us", "encode_us": t_enc * 1e6, "cores": cores,
                                  "kind": "oracle",
                                  "sample": f"the whole workload: encode of {T} keys + {T} values once, decode "
                                            f"{calls} times ({per * 1e3:.1f} ms each)"}
    if "encode_esm2_33_layers" in select:
        c = synth.CONFIGS["esm2_650m_encoder"]
        de, ne = c["head_dim"], 8192
        rk = ro.build_rotation(de, 2, synth.rotation_randomness(de, [c["seed"], 9, 1]), rope_base=c["rope_base"])
        rv = ro.build_rotation(de, 2, synth.rotation_randomness(de, [c["seed"], 9, 2]))
        x = synth.lognormal_channels((1, 2, ne, de), [c["seed"], 9, 6])
        pos = np.arange(ne) % c["tokens"]
        r, calls, per = _oracle_rate(lambda: (codec.encode(rk, x[0, 0], pos), codec.encode(rv, x[0, 1])), 2 * ne)
        out["encode_esm2_33_layers"] = base(r, "vectors/s", f"{ne} keys (RoPE) + {ne} values, d {de}, 2+1 bits; "
                                                            f"{calls} calls, {per:.2f} s each")
    if "decode_llama8b_layer_nsn" in select:
        c = synth.CONFIGS["llama31_8b_gqa_decode"]
        T, G = 8192, c["q_heads"] // c["kv_heads"]
        rk = ro.build_rotation(d, 2, synth.rotation_randomness(d, [c["seed"], 11, 1]), rope_base=c["rope_base"])
        rv = ro.build_rotation(d, 2, synth.rotation_randomness(d, [c["seed"], 11, 2]))
        k = synth.heavy_tailed((1, 1, T, d), [c["seed"], 11, 3]).reshape(T, d)
        v = synth.heavy_tailed((1, 1, T, d), [c["seed"], 11, 4]).reshape(T, d)
        q = synth.heavy_tailed((1, G, d), [c["seed"], 11, 5])
        ek, ev = codec.nsn_encode(rk, k, np.arange(T)), codec.nsn_encode(rv, v)
        rec = lambda e, rot: (codec.pack_planes(e["codes"], rot.bits)[None, None],
                              codec.pack_bits(e["signs"])[None, None],
                              np.stack([e["norm"], e["rnorm"]], 1).astype(np.float32)[None, None])
        kc, vc = rec(ek, rk), rec(ev, rv)
        fn = lambda: at.decode_attention_nsn(rk, rv, q, [T - 1], kc, vc, ek["s1"][None, None], ek["o"][None, None],
                                             ev["s1"][None, None], ev["o"][None, None], 1 / np.sqrt(d))
        r, calls, per = _oracle_rate(fn, T)
        out["decode_llama8b_layer_nsn"] = base(r, "tokens/s", f"one (sequence, KV head), {T} of the layer's "
                                                              f"{c['tokens']} NSN records, {G} query heads, 2+1 bits; "
                                                              f"{calls} calls, {per:.2f} s each")
    if select & {"decode_llama8b_layer_3p1", "decode_llama8b_layer_window"}:
        c = synth.CONFIGS["llama31_8b_gqa_decode"]
        T, G = 8192, c["q_heads"] // c["kv_heads"]
        for key, bits, R in (("decode_llama8b_layer_3p1", 3, 0), ("decode_llama8b_layer_window", 2, 128)):
            if key not in select:
                continue
            rk = ro.build_rotation(d, bits, synth.rotation_randomness(d, [c["seed"], 97]), rope_base=c["rope_base"])
            rv = ro.build_rotation(d, bits, synth.rotation_randomness(d, [c["seed"], 98]))
            k = synth.heavy_tailed((1, 1, T, d), [c["seed"], 99]).reshape(T, d)
            v = synth.heavy_tailed((1, 1, T, d), [c["seed"], 100]).reshape(T, d)
            q = synth.heavy_tailed((1, G, d), [c["seed"], 101])
            Tp = T - R
            kc, vc = packed(rk, k[:Tp], np.arange(Tp)), packed(rv, v[:Tp], None)
            if R:
                kw, vw = k[None, None, Tp:], v[None, None, Tp:]
                fn = lambda: at.decode_attention_window(rk, rv, q, [T - 1], kc, vc, kw, vw, 1 / np.sqrt(d))
            else:
                fn = lambda: at.decode_attention(rk, rv, q, [T - 1], kc, vc, 1 / np.sqrt(d))
            r, calls, per = _oracle_rate(fn, T)
            out[key] = base(r, "tokens/s", f"one (sequence, KV head), {T} of the layer's {c['tokens']} tokens"
                                           f"{f' ({R} in the window)' if R else ''}, {G} query heads, {bits}+1 bits "
                                           f"(the oracle's time is linear in tokens); {calls} calls, {per:.2f} s each")
    return out


# --------------------------------------------------------------------------- secondary workloads
def _time_ms(fn, reps=3, warm=2):
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def run_extras(dev, peak_gbs, select=None, slice_tokens=None, search_rows=None, cpu=True, esm_layers=None):
    """Device-timed measurements of the other rows of the path, each on its
    own workload: encode and decode on the Llama-3.1-70B-shaped 1M-token
    slice, one ESM-2-650M encoder layer, and 1M-vector d=1536 search.
    `select` restricts the run to some of them; `slice_tokens` shrinks the
    70B-shaped slice (profiling runs)."""
    import torch
    import synth
    from vector_quantization_b200 import tq
    out = {}
    select = set(select or EXTRAS)
    g = torch.Generator(device=dev)
    # 70B-shaped slice: 1 layer, 8 KV heads, 64 query heads, 2^20 tokens, 2+1 bits
    c = synth.CONFIGS["llama31_70b_long_slice"]
    Hkv, Hq, d, T, seed = c["kv_heads"], c["q_heads"], c["head_dim"], c["tokens"], c["seed"]
    T = slice_tokens or T
    runs = [({"encode_70b_slice", "decode_70b_slice"},
             lambda: _extras_70b(dev, peak_gbs, select, Hkv, Hq, d, T, seed, c)),
            ({"encoder_esm2_layer"}, lambda: _extra_encoder(dev, g)),
            ({"search_1m_d1536"}, lambda: _extra_search(dev, g, search_rows)),
            ({"decode_llama8b_layer_3p1"}, lambda: _extra_decode_3p1(dev, peak_gbs)),
            ({"decode_llama8b_layer_window"}, lambda: _extra_decode_window(dev, peak_gbs)),
            ({"tiny_d128_t1024"}, lambda: _extra_tiny(dev)),
            ({"encode_esm2_33_layers"}, lambda: _extra_encode_esm2(dev, peak_gbs, g, esm_layers)),
            ({"decode_llama8b_layer_nsn"}, lambda: _extra_decode_nsn(dev, peak_gbs))]
    for names, run in runs:
        if not names & select:
            continue
        try:   # one line failing leaves the others (and the headline) in place
            out.update(run())
        except Exception as exc:
            out[sorted(names & select)[0]] = {"error": f"{type(exc).__name__}: {exc}"}
        torch.cuda.empty_cache()
    if cpu and not slice_tokens and not esm_layers:
        try:
            for key, b in oracle_extra_baselines(select).items():
                if key in out and "error" not in out[key]:
                    out[key]["cpu"] = float(f"{b['value']:.4g}")   # the oracle, same unit as "value"
        except Exception as exc:
            out["cpu_baseline_error"] = f"{type(exc).__name__}: {exc}"
    if "memory_esm2" in select:
        try:
            out["memory_esm2"] = memory_ratio_esm2()
        except Exception as exc:
            out["memory_esm2"] = {"error": f"{type(exc).__name__}: {exc}"}
    return out


def _extras_70b(dev, peak_gbs, select, Hkv, Hq, d, T, seed, c):
    import torch
    import synth
    from vector_quantization_b200 import tq
    out = {}
    rk = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 2]))
    k = synth.heavy_tailed_torch((1, Hkv, T, d), [seed, 3], dev)
    v = synth.heavy_tailed_torch((1, Hkv, T, d), [seed, 4], dev)
    kc, vc = tq.empty_records(rk, (1, Hkv, T), dev), tq.empty_records(rv, (1, Hkv, T), dev)
    def enc():
        tq.quantize_kv(rk, k, apply_rope=True, pos_period=T, out=kc)
        tq.quantize_kv(rv, v, out=vc)
    ms = _time_ms(enc)
    nvec = 2 * Hkv * T
    byts = nvec * (2 * d + rec_bytes({"head_dim": d}, argparse.Namespace(bits=2)))
    if "encode_70b_slice" in select:
        out["encode_70b_slice"] = {"value": nvec / ms * 1e3, "unit": "vectors/s", "ms": round(ms, 4),
                                   "GB_s": round(byts / ms / 1e6, 1), "frac_hbm": round(byts / ms / 1e6 / peak_gbs, 4)}
        # the same slice in sign-residual records (same record sizes)
        rks = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 1]), rope_base=c["rope_base"], rope_max_pos=T,
                          residual="sign")
        rvs = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 2]), residual="sign")
        def enc_sign():
            tq.quantize_kv(rks, k, apply_rope=True, pos_period=T, out=kc)
            tq.quantize_kv(rvs, v, out=vc)
        out["encode_70b_slice"]["ms_sign"] = round(_time_ms(enc_sign), 4)
        enc()   # the QJL records again for the decode line
    del k, v
    if "decode_70b_slice" not in select:
        return out
    q = synth.heavy_tailed_torch((1, Hq, d), [seed, 5], dev)
    qpos = torch.full((1,), T - 1, dtype=torch.int64, device=dev)
    ws = tq.alloc_workspace(tq.decode_workspace_size(rk, rv, 1, Hq, Hkv, T), dev)
    o = torch.empty((1, Hq, d), dtype=torch.float32, device=dev)
    ms = _time_ms(lambda: tq.decode_attention(rk, rv, q, qpos, kc, vc, T, out=o, workspace=ws), reps=10)
    byts = Hkv * T * 2 * rec_bytes({"head_dim": d}, argparse.Namespace(bits=2))
    out["decode_70b_slice"] = {"value": Hkv * T / ms * 1e3, "unit": "tokens/s", "ms": round(ms, 4),
                               "GB_s": round(byts / ms / 1e6, 1), "frac_hbm": round(byts / ms / 1e6 / peak_gbs, 4)}
    return out


def _extra_encoder(dev, g):
    import torch
    import synth
    from vector_quantization_b200 import tq
    out = {}
    # ESM-2-650M encoder layer: [8, 20, 1024, 64] bf16, 2+1 bits, bidirectional attention
    c = synth.CONFIGS["esm2_650m_encoder"]
    B, H, T, d, seed = c["batch"], c["heads"], c["tokens"], c["head_dim"], c["seed"]
    rk = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 2]))
    g.manual_seed(seed)
    mk = lambda: torch.randn((B, H, T, d), generator=g, device=dev).to(torch.bfloat16)
    k, v, q = mk(), mk(), mk()
    kc, vc = tq.quantize_kv(rk, k, apply_rope=True, pos_period=T), tq.quantize_kv(rv, v)
    o = torch.empty((B, H, T, d), dtype=torch.float32, device=dev)
    ws = tq.alloc_workspace(tq._lib.tq_encoder_workspace_size(rk.handle, B, H, T), dev)
    ms = _time_ms(lambda: tq.encoder_attention(rk, rv, q, kc, vc, T, out=o, workspace=ws))
    flops = 2 * B * H * T * T * 2 * (d + d)
    out["encoder_esm2_layer"] = {"value": round(flops / ms / 1e9, 1), "unit": "TFLOP/s", "ms": round(ms, 4)}
    return out


def _extra_search(dev, g, rows=None, recall_queries=100):
    """1M x 1536 search at 1+1 and 3+1 bits: encode of the database, top-10
    of 1000 queries, and recall@10 of the first `recall_queries` queries
    against exact float64 brute-force inner-product search."""
    import torch
    import synth
    from vector_quantization_b200 import tq
    out = {}
    # x = U (lambda^1/2 g), lambda_i = i^-0.8, U the workload's seeded Haar basis
    c = synth.CONFIGS["vector_search_d1536"]
    N, d, nq, kk, seed = c["n_db"], c["dim"], c["n_queries"], c["top_k"], c["seed"]
    N = rows or N
    U = torch.from_numpy(synth.haar_basis(d, seed)).to(dev)
    Uf = U.float()
    g.manual_seed(seed)
    lam = (torch.arange(1, d + 1, device=dev, dtype=torch.float32) ** -0.4)
    db = torch.empty((N, d), dtype=torch.float32, device=dev)
    for s0 in range(0, N, 131072):
        n = min(N, s0 + 131072) - s0
        db[s0:s0 + n] = (torch.randn((n, d), generator=g, device=dev) * lam) @ Uf.T
    qs = (torch.randn((nq, d), generator=g, device=dev) * lam) @ Uf.T
    # exact float64 top-10 of the recall subset
    nr = min(recall_queries, nq)
    qd = qs[:nr].double()
    best_s = torch.full((nr, kk), -float("inf"), dtype=torch.float64, device=dev)
    best_i = torch.zeros((nr, kk), dtype=torch.int64, device=dev)
    for s0 in range(0, N, 131072):
        sc = qd @ db[s0:s0 + 131072].double().T
        cat_s = torch.cat([best_s, sc], 1)
        cat_i = torch.cat([best_i, torch.arange(s0, s0 + sc.shape[1], device=dev).expand(nr, -1)], 1)
        top = cat_s.topk(kk, dim=1)
        best_s, best_i = top.values, cat_i.gather(1, top.indices)
    exact = best_i.cpu().numpy()
    del U, Uf
    wsd = None
    for bits, key in ((1, "search_1m_d1536"), (3, "search_1m_d1536_3p1")):
        rot = tq.Rotation(d, bits, synth.rotation_randomness(d, [seed, bits], dense=True), kind="dense")
        if wsd is None:
            wsd = tq.alloc_workspace(tq._lib.tq_quantize_dense_workspace_size(rot.handle, N), dev)
        packed = tq.empty_records(rot, (N,), dev)
        ms_enc = _time_ms(lambda: tq.quantize_dense(rot, db, out=packed, workspace=wsd), reps=1, warm=1)
        wss = tq.alloc_workspace(tq.search_workspace_size(rot, nq, N, kk), dev)
        ms = _time_ms(lambda: tq.search_topk(rot, qs, packed, kk, workspace=wss), reps=2, warm=1)
        _, ids = tq.search_topk(rot, qs[:nr], packed, kk)
        ids = ids.cpu().numpy()
        recall = float(np.mean([len(set(ids[i].tolist()) & set(exact[i].tolist())) / kk for i in range(nr)]))
        flops = 2 * nq * N * (d + d)
        out[key] = {"value": nq / ms * 1e3, "unit": "queries/s", "ms": round(ms, 3),
                    "TFLOP_s": round(flops / ms / 1e9, 1), "recall10": round(recall, 4), "recall_q": nr,
                    "enc_ms": round(ms_enc, 3)}
        del packed, wss
    return out


def memory_ratio_esm2():
    """Cache bytes of the ESM-2-650M-shaped encoder (33 layers, 20 heads,
    d 64, 1024 tokens, batch 1) at 2+1 bits against float32 K and V, from the
    library's record geometry (tq_rotation_dims), next to the page's quoted
    330 MB -> 47 MB (7.1x)."""
    import ctypes
    import synth
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["esm2_650m_encoder"]
    L, H, T, d = c["layers"], c["heads"], c["tokens"], c["head_dim"]
    rot = tq.Rotation(d, 2, 0)
    cb, sb = ctypes.c_int64(), ctypes.c_int64()
    tq._lib.tq_rotation_dims(rot.handle, None, None, None, ctypes.byref(cb), ctypes.byref(sb))
    rec = cb.value + sb.value + 8
    vecs = 2 * L * H * T
    fp32 = vecs * d * 4
    return {"fp32_MiB": round(fp32 / 2**20, 2), "packed_MiB": round(vecs * rec / 2**20, 3),
            "ratio": round(fp32 / (vecs * rec), 3), "page": "330 MB -> 47 MB, 7.1x"}


def _extra_decode_3p1(dev, peak_gbs):
    """One layer of the Llama-3.1-8B-shaped decode (B16, Hq32, Hkv8, T32768)
    at 4-bit (3+1): the split kernel's time and bandwidth."""
    import torch
    import synth
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["llama31_8b_gqa_decode"]
    B, Hq, Hkv, d, T, seed = c["batch"], c["q_heads"], c["kv_heads"], c["head_dim"], c["tokens"], c["seed"]
    rk = tq.Rotation(d, 3, synth.rotation_randomness(d, [seed, 7, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(d, 3, synth.rotation_randomness(d, [seed, 7, 2]))
    kc, vc = tq.empty_records(rk, (B, Hkv, T), dev), tq.empty_records(rv, (B, Hkv, T), dev)
    x = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, 7, 3], dev)
    tq.quantize_kv(rk, x, apply_rope=True, pos_period=T, out=kc)
    x = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, 7, 4], dev)
    tq.quantize_kv(rv, x, out=vc)
    del x
    q = synth.heavy_tailed_torch((B, Hq, d), [seed, 7, 5], dev)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    ws = tq.alloc_workspace(tq.decode_workspace_size(rk, rv, B, Hq, Hkv, T), dev)
    o = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(8)]
    for i in range(11):
        if i >= 3:
            tq.profile_next_decode(*ev[i - 3])
        tq.decode_attention(rk, rv, q, qpos, kc, vc, T, out=o, workspace=ws)
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    byts = B * Hkv * T * 2 * rec_bytes({"head_dim": d}, argparse.Namespace(bits=3))
    return {"decode_llama8b_layer_3p1": {"value": B * Hkv * T / ms * 1e3, "unit": "tokens/s", "split_ms": round(ms, 4),
                                         "GB_s": round(byts / ms / 1e6, 1),
                                         "frac_hbm": round(byts / ms / 1e6 / peak_gbs, 4)}}

def _extra_decode_window(dev, peak_gbs, R=128):
    """One layer of the Llama-3.1-8B-shaped decode (B16, Hq32, Hkv8, 2+1 bits)
    whose 32768 cached tokens are 32768 - R packed ones plus a bf16
    full-precision window of the R most recent, against the same layer with
    all 32768 packed.  Whole-call device time of both (four launches, and
    five with the window); the cache (470 MB) is larger than L2."""
    import torch
    import synth
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["llama31_8b_gqa_decode"]
    B, Hq, Hkv, d, T, seed = c["batch"], c["q_heads"], c["kv_heads"], c["head_dim"], c["tokens"], c["seed"]
    rk = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 8, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 8, 2]))
    kc, vc = tq.empty_records(rk, (B, Hkv, T), dev), tq.empty_records(rv, (B, Hkv, T), dev)
    xk = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, 8, 3], dev)
    tq.quantize_kv(rk, xk, apply_rope=True, pos_period=T, out=kc)
    kw = xk[:, :, T - R:].to(torch.bfloat16).contiguous()
    del xk
    xv = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, 8, 4], dev)
    tq.quantize_kv(rv, xv, out=vc)
    vw = xv[:, :, T - R:].to(torch.bfloat16).contiguous()
    del xv
    q = synth.heavy_tailed_torch((B, Hq, d), [seed, 8, 5], dev)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    o = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = tq.alloc_workspace(tq.decode_window_workspace_size(rk, rv, B, Hq, Hkv, T - R, R), dev)
    ws2 = tq.alloc_workspace(tq.decode_workspace_size(rk, rv, B, Hq, Hkv, T), dev)
    ms_w = _time_ms(lambda: tq.decode_attention_window(rk, rv, q, qpos, kc, vc, T - R, kw, vw, R, out=o,
                                                       workspace=ws), reps=20, warm=3)
    ms_p = _time_ms(lambda: tq.decode_attention(rk, rv, q, qpos, kc, vc, T, out=o, workspace=ws2), reps=20, warm=3)
    byts = B * Hkv * (T - R) * 2 * rec_bytes({"head_dim": d}, argparse.Namespace(bits=2)) + 2 * kw.numel() * 2
    # the flush when the window is full: its R tokens of every sequence into
    # records T - R .. T - 1 (keys with RoPE at those positions), one launch
    rows = torch.arange(B * Hkv, device=dev, dtype=torch.int64).repeat_interleave(R) * T + \
        torch.arange(T - R, T, device=dev, dtype=torch.int64).repeat(B * Hkv)
    fpos = torch.arange(T - R, T, device=dev, dtype=torch.int64).repeat(B * Hkv)
    flat = lambda cache: tuple(a.view(B * Hkv * T, -1) for a in cache)
    ms_f = _time_ms(lambda: tq.quantize_kv_pair_scatter(rk, kw.view(-1, d), rv, vw.view(-1, d), rows, flat(kc),
                                                        flat(vc), pos=fpos, apply_rope=True), reps=20, warm=3)
    return {"decode_llama8b_layer_window": {"value": B * Hkv * T / ms_w * 1e3, "unit": "tokens/s",
                                            "ms": round(ms_w, 4), "ms_all_packed": round(ms_p, 4),
                                            "frac_hbm": round(byts / ms_w / 1e6 / peak_gbs, 4),
                                            "flush_ms": round(ms_f, 4), "flush_rows": 2 * B * Hkv * R}}

def _extra_decode_nsn(dev, peak_gbs):
    """One layer of the Llama-3.1-8B-shaped decode (B16, Hq32, Hkv8, 2+1
    bits, T 32768) over NSN records ([NSNQuant] §1): the NSN encode of the
    layer's keys (RoPE) and values (tq_nsn_shift, then the codec on the
    shifted rows) and the decode with the s1 and o terms, against the plain
    decode of the same records.  The s1 arrays add 4 B per record to the
    112 B of the record pair."""
    import torch
    import synth
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["llama31_8b_gqa_decode"]
    B, Hq, Hkv, d, T, seed = c["batch"], c["q_heads"], c["kv_heads"], c["head_dim"], c["tokens"], c["seed"]
    rk = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 11, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 11, 2]))
    xk = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, 11, 3], dev)
    kc, ks1, ko = tq.quantize_kv_nsn(rk, xk, apply_rope=True)
    enc_k = _time_ms(lambda: tq.quantize_kv_nsn(rk, xk, apply_rope=True, out=kc), reps=3, warm=1)
    del xk
    xv = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, 11, 4], dev)
    vc, vs1, vo = tq.quantize_kv_nsn(rv, xv)
    enc_v = _time_ms(lambda: tq.quantize_kv_nsn(rv, xv, out=vc), reps=3, warm=1)
    del xv
    q = synth.heavy_tailed_torch((B, Hq, d), [seed, 11, 5], dev)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    o = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = tq.alloc_workspace(tq.decode_workspace_size(rk, rv, B, Hq, Hkv, T), dev)
    ms = _time_ms(lambda: tq.decode_attention_nsn(rk, rv, q, qpos, kc, vc, ks1, ko, vs1, vo, T, out=o, workspace=ws),
                  reps=20, warm=3)
    ms_p = _time_ms(lambda: tq.decode_attention(rk, rv, q, qpos, kc, vc, T, out=o, workspace=ws), reps=20, warm=3)
    byts = B * Hkv * T * 2 * (rec_bytes({"head_dim": d}, argparse.Namespace(bits=2)) + 4)
    return {"decode_llama8b_layer_nsn": {"value": B * Hkv * T / ms * 1e3, "unit": "tokens/s", "ms": round(ms, 4),
                                         "ms_plain": round(ms_p, 4), "frac_hbm": round(byts / ms / 1e6 / peak_gbs, 4),
                                         "encode_ms": round(enc_k + enc_v, 4)}}


def _extra_tiny(dev):
    """The tiny workload (1 head, d 128, 1024 fp32 tokens, heavy-tailed with
    4 outlier channels x20, RoPE on K, 2+1 bits, one fp32 query): encode of
    its K and V and one decode, as absolute latencies (the data fit in L2)."""
    import torch
    import synth
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["tiny_d128_t1024"]
    T, d, seed = c["tokens"], c["head_dim"], c["seed"]
    rk = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 9, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 9, 2]))
    k = torch.from_numpy(synth.heavy_tailed((1, 1, T, d), [seed, 9, 3])).to(dev)
    v = torch.from_numpy(synth.heavy_tailed((1, 1, T, d), [seed, 9, 4])).to(dev)
    q = torch.from_numpy(synth.heavy_tailed((1, 1, d), [seed, 9, 5])).to(dev)
    kc, vc = tq.empty_records(rk, (1, 1, T), dev), tq.empty_records(rv, (1, 1, T), dev)

    def enc():
        tq.quantize_kv(rk, k, apply_rope=True, pos_period=T, out=kc)
        tq.quantize_kv(rv, v, out=vc)
    us_enc = _time_ms(enc, reps=50, warm=5) * 1e3
    qpos = torch.full((1,), T - 1, dtype=torch.int64, device=dev)
    ws = tq.alloc_workspace(tq.decode_workspace_size(rk, rv, 1, 1, 1, T), dev)
    o = torch.empty((1, 1, d), dtype=torch.float32, device=dev)
    us_dec = _time_ms(lambda: tq.decode_attention(rk, rv, q, qpos, kc, vc, T, out=o, workspace=ws),
                      reps=50, warm=5) * 1e3
    return {"tiny_d128_t1024": {"value": round(us_dec, 2), "unit": "decode us", "encode_us": round(us_enc, 2)}}


def _extra_encode_esm2(dev, peak_gbs, g, layers=None):
    """Encode of the whole ESM-2-650M-shaped cache: 33 layers x [8, 20, 1024,
    64] bf16 keys (RoPE at positions 0..1023) and values, 2+1 bits, one call
    each: 2 x 5.4M vectors.  N(0, 1) bf16 rows stand in for the log-normal
    channel law (the encode does the same work whatever the values)."""
    import torch
    import synth
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["esm2_650m_encoder"]
    L, B, H, T, d, seed = c["layers"], c["batch"], c["heads"], c["tokens"], c["head_dim"], c["seed"]
    L = layers or L
    n = L * B * H * T
    rk = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 9, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(d, 2, synth.rotation_randomness(d, [seed, 9, 2]))
    g.manual_seed(seed + 9)
    k = torch.randn((n, d), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((n, d), generator=g, device=dev).to(torch.bfloat16)
    kc, vc = tq.empty_records(rk, (n,), dev), tq.empty_records(rv, (n,), dev)

    def enc():
        tq.quantize_kv(rk, k, apply_rope=True, pos_period=T, out=kc)
        tq.quantize_kv(rv, v, out=vc)
    ms = _time_ms(enc, reps=5, warm=2)
    nvec = 2 * n
    byts = nvec * (2 * d + rec_bytes({"head_dim": d}, argparse.Namespace(bits=2)))
    return {"encode_esm2_33_layers": {"value": nvec / ms * 1e3, "unit": "vectors/s", "ms": round(ms, 4),
                                      "GB_s": round(byts / ms / 1e6, 1),
                                      "frac_hbm": round(byts / ms / 1e6 / peak_gbs, 4)}}


# --------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    c = shape(args)
    steps, warm = args.steps, args.warmup
    base, n, per = oracle_baseline(c, args, max_steps=steps + warm)
    line = {"metric": METRIC, "value": base["value"], "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": warm, "ms_per_step": per * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_json(c, args, world), "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- rank plumbing
def max_over_ranks(value, dist, device):
    """The largest `value` over all ranks (every rank receives it); the
    value itself with a single process (dist None)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, units_per_step_per_rank, steps, slowest_ms):
    """Units all ranks processed per second, timed by the slowest rank
    (weak scaling: every rank processes the same number of units)."""
    return world * units_per_step_per_rank * steps / (slowest_ms / 1e3)


# --------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import synth
    from vector_quantization_b200 import tq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    c = shape(args)
    L, B, Hq, Hkv, d, T = c["layers"], c["batch"], c["q_heads"], c["kv_heads"], c["head_dim"], c["tokens"]
    seed = c["seed"] + 100 * rank
    bits = args.bits
    # ---- build: per-layer handles and packed caches ------------------------
    rks, rvs, kcs, vcs, qs, nks, nvs = [], [], [], [], [], [], []
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    for layer in range(L):
        rk = tq.Rotation(d, bits, synth.rotation_randomness(d, [seed, layer, 1]), rope_base=c["rope_base"],
                         rope_max_pos=T)
        rv = tq.Rotation(d, bits, synth.rotation_randomness(d, [seed, layer, 2]))
        kc = tq.empty_records(rk, (B, Hkv, T), dev)
        vc = tq.empty_records(rv, (B, Hkv, T), dev)
        x = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, layer, 3], dev)
        tq.quantize_kv(rk, x, apply_rope=True, pos_period=T, out=kc)
        del x
        x = synth.heavy_tailed_torch((B, Hkv, T, d), [seed, layer, 4], dev)
        tq.quantize_kv(rv, x, out=vc)
        del x
        rks.append(rk)
        rvs.append(rv)
        kcs.append(kc)
        vcs.append(vc)
        qs.append(synth.heavy_tailed_torch((B, Hq, d), [seed, layer, 5], dev))
        nks.append(synth.heavy_tailed_torch((B, Hkv, 1, d), [seed, layer, 6], dev).view(B * Hkv, d))
        nvs.append(synth.heavy_tailed_torch((B, Hkv, 1, d), [seed, layer, 7], dev).view(B * Hkv, d))
    ws = tq.alloc_workspace(tq.decode_workspace_size(rks[0], rvs[0], B, Hq, Hkv, T), dev)
    outs = [torch.empty((B, Hq, d), dtype=torch.float32, device=dev) for _ in range(L)]
    torch.cuda.synchronize()

    def step(prof=None, src=None):
        # per layer: the new token's K and V appended at record T - 1 (RoPE at
        # position T - 1) in the same launch as the query preparation, then
        # attention over all T records
        for layer in range(L):
            nk = nks[layer] if src is None else src[0][layer]
            nv = nvs[layer] if src is None else src[1][layer]
            q = qs[layer] if src is None else src[2][layer]
            if prof is not None:
                tq.profile_next_decode(*prof[layer])
            tq.decode_attention_append(rks[layer], rvs[layer], q, qpos, nk, nv, kcs[layer], vcs[layer], T,
                                       out=outs[layer], workspace=ws)

    launches_per_step = L * 3
    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- device-timed region -------------------------------------------------
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    prof = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L)]
            for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("bench_timed")
    e0.record()
    for s in range(args.steps):
        step(prof[s])
    e1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    elapsed_ms = e0.elapsed_time(e1)
    split_ms = [a.elapsed_time(b) for row in prof for (a, b) in row]
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)
    tokens_per_step = L * B * Hkv * T
    value = whole_job_rate(world, tokens_per_step, args.steps, elapsed_ms)

    # ---- end-to-end through the public API with host buffers ----------------
    host_in = ([torch.empty_like(x, device="cpu").pin_memory().copy_(x.cpu()) for x in nks],
               [torch.empty_like(x, device="cpu").pin_memory().copy_(x.cpu()) for x in nvs],
               [torch.empty_like(x, device="cpu").pin_memory().copy_(x.cpu()) for x in qs])
    host_out = [torch.empty((B, Hq, d), dtype=torch.float32).pin_memory() for _ in range(L)]
    dev_in = ([torch.empty_like(x) for x in nks], [torch.empty_like(x) for x in nvs], [torch.empty_like(x) for x in qs])
    h2d = sum(x.numel() * x.element_size() for group in host_in for x in group)
    d2h = sum(x.numel() * x.element_size() for x in host_out)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(args.steps):
        for g in range(3):
            for a, b in zip(dev_in[g], host_in[g]):
                a.copy_(b, non_blocking=True)
        step(src=dev_in)
        for a, b in zip(host_out, outs):
            a.copy_(b, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = f0.elapsed_time(f1)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    e2e_value = whole_job_rate(world, tokens_per_step, args.steps, e2e_ms)

    if rank != 0:
        return
    peak, peak_kind = measured_peaks()
    bytes_per_launch = B * Hkv * T * 2 * rec_bytes(c, args)
    split_avg_s = float(np.mean(split_ms)) / 1e3
    achieved = bytes_per_launch / split_avg_s / 1e9
    # DRAM bytes per launch of the split kernel, from one ncu capture of the
    # T = 16384 case (read + write = 241.71 MB), scaled by the token count to
    # the launch timed here; traffic grows in proportion to the tokens streamed.
    # Must be reset to None whenever decode_split_kernel changes.
    traffic = SPLIT_TRAFFIC_PER_TOKEN * B * Hkv * T if SPLIT_TRAFFIC_PER_TOKEN and args.bits == 2 else None
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "kernel": "decode_split_kernel (one launch per layer)",
                "algorithmic_bytes_per_launch": bytes_per_launch, "peak_source": peak_kind,
                "launch_ms_avg": round(split_avg_s * 1e3, 4)}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_json(c, args, world),
            "roofline": roofline, "gpu_launches": launches_per_step * args.steps,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "clocks": clk}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_baseline(c, args)[0]
    if world == 1 and not args.no_extras:
        del kcs, vcs
        torch.cuda.empty_cache()
        try:
            line["extras"] = run_extras(dev, peak, cpu=not args.no_cpu_baseline)
        except Exception as exc:   # the headline line is printed whatever a secondary line does
            line["extras"] = {"error": f"{type(exc).__name__}: {exc}"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.extra:
        import torch
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        print(json.dumps({"extras": run_extras(dev, measured_peaks()[0], args.extra, args.slice_tokens,
                                               args.search_rows, cpu=not args.no_cpu_baseline,
                                               esm_layers=args.esm_layers)}), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
