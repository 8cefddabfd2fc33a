"""Benchmark: compressed decode attention over a TurboQuant KV cache.

Default workload (one step): a Llama-3-8B-shaped decode step over 32
attention layers, each with its own compressed cache -- batch 1, 32 query
heads, 8 KV heads (GQA 4), d = 128, 32768 cached tokens, K 4-bit / V 2-bit.
Per layer the step appends one new token (quantise-append of its K and V)
and runs decode attention over the whole cache (32769+ tokens).  Inputs are
seeded synthetic bf16 data (log-normal per-channel scales, sigma 1); the 32
distinct caches (839 MB) are far larger than L2, so every layer's cache
comes from HBM.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle on the same workload instead (bounded sample per step).
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

LAYERS, BATCH, HQ, HKV, D, CONTEXT = 32, 1, 32, 8, 128, 32768
K_BITS, V_BITS = 4, 2
SEED = 1234
WORKLOAD = "llama3-8b-shaped decode step: 32 layers x (append 1 token + decode attention), B=1, Hq=32, Hkv=8, " \
           "d=128, context 32768, K4/V2 packed cache"
METRIC = "compressed decode-attn KV tokens/s"


def bytes_per_token_head(k_bits=K_BITS, v_bits=V_BITS, d=D):
    """Algorithmic bytes one decode step reads per cached token and kv head."""
    return d * k_bits // 8 + 2 + d * v_bits // 8 + 2


def rank_seed(rank):
    """Input seed of one replica: every rank draws its own layers and queries."""
    return SEED + 7919 * rank


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x, world):
    if world == 1:
        return x
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        with open(self.file.name) as fh:
            rows = [r.split(",") for r in fh.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip() == "Active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


# DRAM traffic per kernel from ncu captures, machine-read from
# profiles/traffic.json: for each kernel the bytes (dram__bytes_read.sum +
# dram__bytes_write.sum) of one captured launch, the units of work that launch
# processed, and the sha256 of the sources it was built from.  A figure applies
# only while those sources are unchanged.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "bit_kv_cache_tq_b200", "csrc")


def sources_sha256(names):
    import hashlib
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(CSRC, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(kernel, units):
    """DRAM bytes of one launch of `kernel` over `units` units of work, scaled
    from the captured launch; None when no capture of the current sources is
    recorded."""
    try:
        with open(TRAFFIC_FILE, encoding="utf-8") as fh:
            rec = json.load(fh)[kernel]
        if rec["sources_sha256"] != sources_sha256(rec["sources"]):
            return None
        return float(rec["dram_bytes_per_launch"]) * units / float(rec["units_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ------------------------------------------------------------------ oracle leg
class OracleDecode:
    """The fp64 CPU oracle on a bounded sample of the decode step.  One unit
    of work = one (kv head) of one layer: encode the appended token, dequantise
    the unit's cached tokens and attend with its 4 query heads.  The cache
    contents (prefill) are built once, untimed."""

    def __init__(self, context=CONTEXT, units=2):
        from oracle import codebook as ocb, quantize as oq, rng as orng
        from bit_kv_cache_tq_b200 import inputs
        self.oq = oq
        self.context = context
        self.kc, self.kt = ocb.lloyd_max(D, K_BITS)
        self.vc, self.vt = ocb.lloyd_max(D, V_BITS)
        self.signs = orng.rotation_signs(SEED, D)
        k = inputs.lognormal_kv(1, context + 1, units, D, seed=SEED, layer=0, which=inputs.K).float().numpy()
        v = inputs.lognormal_kv(1, context + 1, units, D, seed=SEED, layer=0, which=inputs.V).float().numpy()
        self.q = inputs.queries(1, HQ, D, seed=SEED).float().numpy().astype(np.float64)
        self.new = [(k[0, context:, h], v[0, context:, h]) for h in range(units)]
        self.caches = [(oq.encode_turbo(k[0, :context, h], self.signs, self.kc, self.kt, K_BITS),
                        oq.encode_turbo(v[0, :context, h], self.signs, self.vc, self.vt, V_BITS))
                       for h in range(units)]
        self.done = 0

    def unit(self):
        from oracle import attention as oatt
        oq, h = self.oq, self.done % len(self.caches)
        ek, ev = self.caches[h]
        nk = oq.encode_turbo(self.new[h][0], self.signs, self.kc, self.kt, K_BITS)
        nv = oq.encode_turbo(self.new[h][1], self.signs, self.vc, self.vt, V_BITS)
        khat = oq.dequantize_turbo(np.concatenate([ek["codes"], nk["codes"]]),
                                   np.concatenate([ek["norm16"], nk["norm16"]]), self.signs, self.kc)
        vhat = oq.dequantize_turbo(np.concatenate([ev["codes"], nv["codes"]]),
                                   np.concatenate([ev["norm16"], nv["norm16"]]), self.signs, self.vc)
        g = HQ // HKV
        oatt.decode_attention(self.q[:, h * g:(h + 1) * g], khat[None, None], vhat[None, None], [self.context + 1])
        self.done += 1

    def tokens_per_unit(self):
        return (self.context + 1) / HKV  # a layer token spans all 8 kv heads

    @staticmethod
    def cores():
        try:
            from threadpoolctl import threadpool_info
            return max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
        except Exception:
            return os.cpu_count()


def oracle_sample(seconds_target=12.0):
    """(tokens/s, cpu_baseline dict) of the oracle over ~seconds_target of work."""
    w = OracleDecode()
    w.unit()  # warm-up
    n = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds_target:
        w.unit()
        n += 1
    dt = time.perf_counter() - t0
    val = n * w.tokens_per_unit() / dt
    return val, {"kind": "oracle", "cores": w.cores(), "value": val, "unit": "tokens/s",
                 "sample": "%d (kv head) units of one layer, each: encode 1 appended token, dequantise %d cached "
                           "tokens, 4-head attention (fp64 numpy); %.1f s; a layer token = 8 kv-head vectors"
                           % (n, CONTEXT, dt)}


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = OracleDecode()
    for _ in range(args.warmup):
        w.unit()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        w.unit()
    dt = time.perf_counter() - t0
    value = args.steps * w.tokens_per_unit() / dt
    info = {"kind": "oracle", "cores": w.cores(), "value": value, "unit": "tokens/s",
            "sample": "each step: one (kv head) unit of one layer (encode 1 appended token, dequantise 32768 "
                      "cached tokens, 4-head attention), fp64 numpy; a layer token = 8 kv-head vectors"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": BATCH, "seq_len": CONTEXT + 1, "parallelism": "none"},
            "cpu_baseline": info,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU leg
BULK_TOKENS, BULK_HEADS, BULK_LAYERS = 262144, 8, 32
BULK_INT8_LAYERS = (0, 1, 30, 31)  # the first two and last two layers keep int8 (per-vector absmax)


def bulk_quantize(dev, d, reps=3):
    """Bulk prefill quantise at full size: one bf16 input slab of 262144 tokens x
    8 kv heads (K and V) quantised into 32 distinct layer caches with the
    layer policy (int8 boundary layers, K4/V3 turbo codes elsewhere).  Returns
    GB/s of (input read + codes and norms written) for the whole 32-layer
    sweep and per layer kind, timed with CUDA events (inputs and outputs far
    larger than L2)."""
    from bit_kv_cache_tq_b200 import inputs, tq
    k = inputs.lognormal_kv(1, BULK_TOKENS, BULK_HEADS, d, SEED, 2, inputs.K, device=dev)
    v = inputs.lognormal_kv(1, BULK_TOKENS, BULK_HEADS, d, SEED, 2, inputs.V, device=dev)
    turbo = tq.make_params(d, BULK_HEADS, BULK_HEADS, k_bits=4, v_bits=3, seed=SEED)
    int8 = tq.make_params(d, BULK_HEADS, BULK_HEADS, k_mode=tq.TQ_MODE_INT8, v_mode=tq.TQ_MODE_INT8, seed=SEED)
    kcb, vcb = tq.tq_codebook_init(d, 4), tq.tq_codebook_init(d, 3)
    params = [int8 if l in BULK_INT8_LAYERS else turbo for l in range(BULK_LAYERS)]
    caches = [tq.alloc_cache(p, 1, BULK_TOKENS, device=dev) for p in params]
    pos = torch.zeros(1, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    in_bytes = 2 * k.numel() * k.element_size()

    def out_bytes(p):
        return sum(tq.tq_cache_bytes(p, 1, BULK_TOKENS))

    def layer(l):
        tq.tq_quantize_append(params[l], kcb, vcb, k, v, pos, caches[l], err)

    for l in range(BULK_LAYERS):  # warm-up: every layer once
        layer(l)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * BULK_LAYERS + 2)]
    best = None
    for _ in range(reps):
        ev[0].record()
        for l in range(BULK_LAYERS):
            ev[1 + 2 * l].record()
            layer(l)
            ev[2 + 2 * l].record()
        ev[-1].record()
        ev[-1].synchronize()
        sweep = ev[0].elapsed_time(ev[-1])
        if best is None or sweep < best[0]:
            best = (sweep, [ev[1 + 2 * l].elapsed_time(ev[2 + 2 * l]) for l in range(BULK_LAYERS)])
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_OK, ("bulk quantise", st, word)
    sweep_ms, per = best
    t_us = statistics.median([per[l] for l in range(BULK_LAYERS) if l not in BULK_INT8_LAYERS]) * 1e3
    i_us = statistics.median([per[l] for l in BULK_INT8_LAYERS]) * 1e3
    total = sum(in_bytes + out_bytes(p) for p in params)
    res = {"sweep_ms": sweep_ms, "sweep_gbs": total / (sweep_ms * 1e-3) / 1e9,
           "turbo_layer_us": t_us, "turbo_layer_gbs": (in_bytes + out_bytes(turbo)) / (t_us * 1e-6) / 1e9,
           "int8_layer_us": i_us, "int8_layer_gbs": (in_bytes + out_bytes(int8)) / (i_us * 1e-6) / 1e9,
           "input_only_gbs": BULK_LAYERS * in_bytes / (sweep_ms * 1e-3) / 1e9}
    del caches, k, v
    torch.cuda.empty_cache()
    return {key: round(val, 2) for key, val in res.items()}


def bf16_sdpa_baseline(dev, reps=20):
    """Uncompressed comparison arm (library code, not this path): torch's
    scaled_dot_product_attention over bf16 K/V of the same decode shape (B=1,
    Hq=32, Hkv=8, d=128, 32769 tokens), 32 distinct layer caches (4.3 GB,
    larger than L2), timed with CUDA events; 512 B per token and kv head."""
    import torch.nn.functional as F
    from bit_kv_cache_tq_b200 import inputs
    seq = CONTEXT + 1
    ks = [inputs.lognormal_kv(BATCH, seq, HKV, D, SEED, l, inputs.K, device=dev).transpose(1, 2).contiguous()
          for l in range(LAYERS)]
    vs = [inputs.lognormal_kv(BATCH, seq, HKV, D, SEED, l, inputs.V, device=dev).transpose(1, 2).contiguous()
          for l in range(LAYERS)]
    q = inputs.queries(BATCH, HQ, D, SEED, device=dev).view(BATCH, HQ, 1, D)

    def sweep():
        for l in range(LAYERS):
            F.scaled_dot_product_attention(q, ks[l], vs[l], enable_gqa=True)

    for _ in range(3):
        sweep()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        sweep()
    e1.record()
    e1.synchronize()
    us = 1000.0 * e0.elapsed_time(e1) / (reps * LAYERS)
    bytes_layer = 2 * BATCH * HKV * seq * D * 2
    del ks, vs
    torch.cuda.empty_cache()
    return {"kernel": "torch.nn.functional.scaled_dot_product_attention (bf16, enable_gqa, default backend)",
            "us_per_layer": round(us, 2), "kv_tokens_per_s": round(BATCH * seq / (us * 1e-6)),
            "gbs": round(bytes_layer / (us * 1e-6) / 1e9, 1), "bytes_per_layer": bytes_layer}


def decode_configs(dev, reps=10):
    """The decode kernel on the other full-size decode workloads, timed with
    CUDA events over `reps` calls (caches larger than L2, or cycled copies):
    batched ragged (B=16, Hq=32, Hkv=8, lengths uniform in [2048, 8192], K3/V2,
    4 cache copies), 70B-shaped long context (B=4, Hq=64, Hkv=8, 131072
    tokens, K3 + 64-bit QJL / V2, Sparse V at 1e-6), and the Llama-3-8B-shaped
    layer (B=1, 32768 tokens, 4 cache copies) with int8 keys and 2-bit values
    (the mixed setting) and as an int8 boundary layer (int8 keys and values),
    the latter also with 64 query heads (groups of 8).
    A kb of 8 below stands for int8 (one byte per channel, fp16 scale)."""
    from bit_kv_cache_tq_b200 import inputs, tq
    res = {}
    cases = [("batched_ragged_b16_k3v2", 16, 32, 8192, 3, 2, 0, 0.0, 4),
             ("long_context_b4_hq64_128k_k3qjl_v2_sparse", 4, 64, 131072, 3, 2, 64, 1e-6, 1),
             ("llama8b_32k_int8k_v2", 1, 32, 32768, 8, 2, 0, 0.0, 4),
             ("llama8b_32k_int8k_int8v", 1, 32, 32768, 8, 8, 0, 0.0, 4),
             ("hq64_32k_int8k_int8v", 1, 64, 32768, 8, 8, 0, 0.0, 4)]
    for name, bsz, hq, tmax, kb, vb, m, tau, copies in cases:
        modes = dict(k_mode=tq.TQ_MODE_INT8 if kb == 8 else tq.TQ_MODE_TURBO,
                     v_mode=tq.TQ_MODE_INT8 if vb == 8 else tq.TQ_MODE_TURBO,
                     k_bits=4 if kb == 8 else kb, v_bits=2 if vb == 8 else vb)
        p = tq.make_params(D, hq, HKV, qjl_dims=m, seed=SEED, sparse_v_threshold=tau, **modes)
        kcb, vcb = tq.tq_codebook_init(D, modes["k_bits"]), tq.tq_codebook_init(D, modes["v_bits"])
        if bsz == 16:
            lens = inputs.ragged_lengths(bsz, 2048, 8192, seed=0).tolist()
        else:
            lens = [tmax] * bsz
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        pos = torch.zeros(bsz, dtype=torch.int32, device=dev)
        caches = []
        for c in range(copies):
            cache = tq.alloc_cache(p, bsz, tmax, device=dev)
            k = inputs.lognormal_kv(bsz, tmax, HKV, D, SEED, 40 + c, inputs.K, device=dev)
            v = inputs.lognormal_kv(bsz, tmax, HKV, D, SEED, 40 + c, inputs.V, device=dev)
            tq.tq_quantize_append(p, kcb, vcb, k, v, pos, cache, err)
            del k, v
            caches.append(cache)
        q = inputs.queries(bsz, hq, D, SEED, device=dev)
        lens_t = torch.tensor(lens, dtype=torch.int32, device=dev)
        ws = torch.zeros(tq.tq_decode_workspace_bytes(p, bsz, tmax), dtype=torch.uint8, device=dev)
        out = torch.empty(bsz, hq, D, dtype=torch.float32, device=dev)
        for c in range(copies):
            tq.tq_decode_attention(p, kcb, vcb, q, caches[c], lens_t, tmax, out, ws, err)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for r in range(reps):
            tq.tq_decode_attention(p, kcb, vcb, q, caches[r % copies], lens_t, tmax, out, ws, err)
        e1.record()
        e1.synchronize()
        st, word = tq.tq_read_device_error(err)
        assert st == tq.TQ_OK, (name, st, word)
        us = 1000.0 * e0.elapsed_time(e1) / reps
        extra = {}
        if tau > 0:  # Sparse V's effect: the same call without skipping, and the positions it dropped
            dense = tq.make_params(D, hq, HKV, qjl_dims=m, seed=SEED, **modes)
            out_d = torch.empty_like(out)
            mask = torch.zeros(bsz, hq, (tmax + 31) // 32, dtype=torch.int32, device=dev)
            tq.tq_decode_attention(p, kcb, vcb, q, caches[0], lens_t, tmax, out, ws, err, skip_mask=mask)
            words = mask.cpu().numpy().astype(np.uint32)
            dropped = int(np.unpackbits(words.view(np.uint8)).sum())
            extra["skip_fraction"] = dropped / float(hq * sum(lens))
            tq.tq_decode_attention(dense, kcb, vcb, q, caches[0], lens_t, tmax, out_d, ws, err)
            rel = ((out - out_d).norm(dim=-1) / out_d.norm(dim=-1)).max().item()
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d0.record()
            for r in range(reps):
                tq.tq_decode_attention(dense, kcb, vcb, q, caches[r % copies], lens_t, tmax, out_d, ws, err)
            d1.record()
            d1.synchronize()
            extra.update({"max_rel_l2_vs_no_skip": rel,
                          "us_without_sparse_v": round(1000.0 * d0.elapsed_time(d1) / reps, 2)})
        per_tok = D * kb // 8 + 2 + (m // 8 + 2 if m else 0) + D * vb // 8 + 2
        nbytes = sum(lens) * HKV * per_tok
        res[name] = {"us_per_call": round(us, 2), "kv_tokens_per_s": round(sum(lens) / (us * 1e-6)),
                     "gbs": round(nbytes / (us * 1e-6) / 1e9, 1), "algorithmic_bytes": nbytes,
                     "bytes_per_token_kv_head": per_tok, **extra}
        del caches, ws
        torch.cuda.empty_cache()
    return res


def paged_decode(dev, reps=10, copies=4):
    """The Llama-3-8B-shaped layer (B=1, 32768 tokens, K4/V2) read through a
    block table (blocks in a random order over the pool), block sizes 16 and
    256 tokens; 4 pools cycled so the reads come from HBM."""
    from bit_kv_cache_tq_b200 import inputs, tq
    p = tq.make_params(D, HQ, HKV, K_BITS, V_BITS, seed=SEED)
    kcb, vcb = tq.tq_codebook_init(D, K_BITS), tq.tq_codebook_init(D, V_BITS)
    n = CONTEXT
    res = {}
    for bs in (16, 256):
        max_blocks = (n + bs - 1) // bs
        gen = torch.Generator().manual_seed(SEED + bs)
        pools, tables = [], []
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        for c in range(copies):
            pool = tq.alloc_cache(p, max_blocks, bs, device=dev)
            table = torch.randperm(max_blocks, generator=gen).to(torch.int32).view(1, max_blocks).to(dev)
            k = inputs.lognormal_kv(1, n, HKV, D, SEED, 60 + c, inputs.K, device=dev)
            v = inputs.lognormal_kv(1, n, HKV, D, SEED, 60 + c, inputs.V, device=dev)
            tq.tq_quantize_append_paged(p, kcb, vcb, k, v, torch.zeros(1, dtype=torch.int32, device=dev), pool,
                                        table, err)
            del k, v
            pools.append(pool)
            tables.append(table)
        q = inputs.queries(1, HQ, D, SEED, device=dev)
        lens_t = torch.tensor([n], dtype=torch.int32, device=dev)
        ws = torch.zeros(tq.tq_decode_workspace_bytes(p, 1, n), dtype=torch.uint8, device=dev)
        out = torch.empty(1, HQ, D, dtype=torch.float32, device=dev)
        for c in range(copies):
            tq.tq_decode_attention_paged(p, kcb, vcb, q, pools[c], tables[c], lens_t, n, out, ws, err)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for r in range(reps):
            tq.tq_decode_attention_paged(p, kcb, vcb, q, pools[r % copies], tables[r % copies], lens_t, n, out, ws,
                                         err)
        e1.record()
        e1.synchronize()
        st, word = tq.tq_read_device_error(err)
        assert st == tq.TQ_OK, (bs, st, word)
        us = 1000.0 * e0.elapsed_time(e1) / reps
        nbytes = n * HKV * bytes_per_token_head()
        res["block_%d" % bs] = {"us_per_call": round(us, 2), "kv_tokens_per_s": round(n / (us * 1e-6)),
                                "gbs": round(nbytes / (us * 1e-6) / 1e9, 1), "algorithmic_bytes": nbytes}
        del pools, tables, ws
        torch.cuda.empty_cache()
    return res


PREFILL_CHUNK = 512


def oracle_prefill_sample(seconds_target=8.0):
    """The fp64 CPU oracle on a bounded sample of the prefill workload: one kv
    head of the Llama-3-8B-shaped layer, 32768 cached tokens; each unit
    encodes a 4-token chunk, dequantises the cache and runs the causal
    attention of the chunk's 4 tokens x 4 query heads.  Returns a cpu_baseline
    dict in attention GFLOP/s (4 d FLOPs per query head and visible key)."""
    from oracle import attention as oatt
    w = OracleDecode(units=1)
    oq, c = w.oq, 4
    from bit_kv_cache_tq_b200 import inputs
    kn = inputs.lognormal_kv(1, c, 1, D, seed=SEED, layer=9, which=inputs.K).float().numpy()[0, :, 0]
    vn = inputs.lognormal_kv(1, c, 1, D, seed=SEED, layer=9, which=inputs.V).float().numpy()[0, :, 0]
    g = HQ // HKV
    q = inputs.queries(1, c * g, D, seed=SEED, layer=9).float().numpy().astype(np.float64).reshape(1, c, g, D)
    ek, ev = w.caches[0]

    def unit():
        nk = oq.encode_turbo(kn, w.signs, w.kc, w.kt, K_BITS)
        nv = oq.encode_turbo(vn, w.signs, w.vc, w.vt, V_BITS)
        khat = oq.dequantize_turbo(np.concatenate([ek["codes"], nk["codes"]]),
                                   np.concatenate([ek["norm16"], nk["norm16"]]), w.signs, w.kc)
        vhat = oq.dequantize_turbo(np.concatenate([ev["codes"], nv["codes"]]),
                                   np.concatenate([ev["norm16"], nv["norm16"]]), w.signs, w.vc)
        oatt.prefill_attention(q, khat[None, None], vhat[None, None], [w.context])

    unit()  # warm-up
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds_target:
        unit()
        n += 1
    dt = time.perf_counter() - t0
    flops = 4.0 * D * g * sum(w.context + j + 1 for j in range(c))
    val = n * flops / dt / 1e9
    return {"kind": "oracle", "cores": w.cores(), "value": round(val, 3), "unit": "GFLOP/s",
            "sample": "%d units, each: encode a %d-token chunk of one kv head, dequantise its %d cached tokens, "
                      "causal attention of %d queries x %d heads (fp64 numpy); %.1f s" % (n, c, w.context, c, g, dt)}


def prefill_chunk(dev, reps=100, warmup=10, smaller=(128, 32)):
    """Chunked prefill from the compressed cache (tq_prefill_attention): the
    Llama-3-8B-shaped layer (B=1, Hq=32, Hkv=8, d=128, K4/V2) with 32768
    cached tokens and a 512-token chunk appended and attended causally.
    Reports the call (append kernel + attention kernel) and the attention's
    algorithmic tensor work: 4 d FLOPs per (query, head, visible key) for
    Q K^T and P V, against the measured dense bf16 peak, burst (the call is
    timed alone) and sustained (fp16 operands have the same nominal rate).
    The smaller chunks after the same 32768 tokens (fewer units of 128 query
    rows than SMs) are reported beside it."""
    from bit_kv_cache_tq_b200 import inputs, tq
    p = tq.make_params(D, HQ, HKV, K_BITS, V_BITS, seed=SEED)
    kcb, vcb = tq.tq_codebook_init(D, K_BITS), tq.tq_codebook_init(D, V_BITS)
    start = CONTEXT
    cache = tq.alloc_cache(p, 1, start + PREFILL_CHUNK, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    k = inputs.lognormal_kv(1, start, HKV, D, SEED, 70, inputs.K, device=dev)
    v = inputs.lognormal_kv(1, start, HKV, D, SEED, 70, inputs.V, device=dev)
    tq.tq_quantize_append(p, kcb, vcb, k, v, torch.zeros(1, dtype=torch.int32, device=dev), cache, err)
    del k, v

    def timed(n_new):
        # (each call appends the chunk at the same slots, then attends)
        kn = inputs.lognormal_kv(1, n_new, HKV, D, SEED, 70, inputs.K, device=dev, token_offset_seed=3)
        vn = inputs.lognormal_kv(1, n_new, HKV, D, SEED, 70, inputs.V, device=dev, token_offset_seed=3)
        q = inputs.queries(1, n_new * HQ, D, SEED, layer=70, device=dev).view(1, n_new, HQ, D)
        pos = torch.full((1,), start, dtype=torch.int32, device=dev)
        out = torch.empty(1, n_new, HQ, D, dtype=torch.float32, device=dev)
        ws = torch.zeros(tq.tq_prefill_workspace_bytes(p, 1, n_new), dtype=torch.uint8, device=dev)
        for _ in range(warmup):
            tq.tq_prefill_attention(p, kcb, vcb, kn, vn, q, pos, cache, out, ws, err)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            tq.tq_prefill_attention(p, kcb, vcb, kn, vn, q, pos, cache, out, ws, err)
        e1.record()
        e1.synchronize()
        st, word = tq.tq_read_device_error(err)
        assert st == tq.TQ_OK, ("prefill", n_new, st, word)
        us = 1000.0 * e0.elapsed_time(e1) / reps
        keys = sum(start + j + 1 for j in range(n_new))  # visible keys per (query, head), summed over the chunk
        flops = 4.0 * D * HQ * keys
        return us, flops, flops / (us * 1e-6) / 1e12

    us, flops, tflops = timed(PREFILL_CHUNK)
    small = []
    for n in smaller:
        su, _, st = timed(n)
        small.append({"chunk": n, "us_per_call": round(su, 2), "attention_tflops": round(st, 1)})
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            peaks = json.load(fh)
        peak_tf, peak_kind = float(peaks["bf16_tflops"]), "measured bf16 burst"
        sustained_tf = float(peaks["bf16_tflops_sustained"])
    except (OSError, KeyError, ValueError):
        peak_tf, peak_kind, sustained_tf = 1590.0, "fallback", 1400.0
    del cache
    torch.cuda.empty_cache()
    return {"workload": "llama3-8b-shaped layer, %d cached tokens + a %d-token chunk, K4/V2, causal"
                        % (start, PREFILL_CHUNK),
            "us_per_call": round(us, 2), "tokens_per_s": round(PREFILL_CHUNK / (us * 1e-6)),
            "attention_tflops": round(tflops, 1), "peak_tflops": peak_tf, "peak_kind": peak_kind,
            "frac_of_peak": round(tflops / peak_tf, 4), "sustained_peak_tflops": sustained_tf,
            "frac_of_sustained_peak": round(tflops / sustained_tf, 4), "algorithmic_flops": flops,
            "traffic": profiled_traffic("prefill_kernel", 1),
            "timing": "%d calls after %d warm-up calls, CUDA events" % (reps, warmup),
            "smaller_chunks": small,
            "kernels": "tq_prefill_attention: quantise-append of the chunk, then the tcgen05 attention kernel "
                       "(one block per SM sharing all units' key tiles), then the merge kernel for units split "
                       "between blocks"}


class EagerWork:
    """Stands in for a captured CUDA graph: replay() enqueues the work."""

    def __init__(self, fn):
        self.fn = fn

    def replay(self):
        self.fn()


def run_tq(args, world, rank, local):
    from bit_kv_cache_tq_b200 import inputs, tq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    steps, warmup = args.steps, args.warmup
    total_steps = steps + warmup
    # a capacity that is a multiple of 8 lets the kernel stage norms beside the codes
    cap = (CONTEXT + total_steps + 1 + 7) // 8 * 8
    gen_seed = rank_seed(rank)
    kcb, vcb = tq.tq_codebook_init(D, K_BITS), tq.tq_codebook_init(D, V_BITS)
    # each layer's kernel follows another layer's on the stream, which never
    # writes this layer's cache: the decode may start streaming it early
    params = [tq.make_params(D, HQ, HKV, K_BITS, V_BITS, seed=gen_seed + l, flags=tq.TQ_PARAM_PREFETCH_EARLY)
              for l in range(LAYERS)]
    caches = [tq.alloc_cache(p, BATCH, cap, device=dev) for p in params]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    zero_pos = torch.zeros(BATCH, dtype=torch.int32, device=dev)
    # prefill: quantise the 32768-token context of every layer on the GPU (set-up)
    for l in range(LAYERS):
        k = inputs.lognormal_kv(BATCH, CONTEXT, HKV, D, gen_seed, l, inputs.K, device=dev)
        v = inputs.lognormal_kv(BATCH, CONTEXT, HKV, D, gen_seed, l, inputs.V, device=dev)
        tq.tq_quantize_append(params[l], kcb, vcb, k, v, zero_pos, caches[l], err)
        del k, v
    # per-step inputs, resident in HBM: new K/V tokens and queries per layer
    k_new = [inputs.lognormal_kv(BATCH, total_steps, HKV, D, gen_seed, l, inputs.K, device=dev, token_offset_seed=1)
             for l in range(LAYERS)]
    v_new = [inputs.lognormal_kv(BATCH, total_steps, HKV, D, gen_seed, l, inputs.V, device=dev, token_offset_seed=1)
             for l in range(LAYERS)]
    qs = [[inputs.queries(BATCH, HQ, D, gen_seed, layer=l, step=i, device=dev) for i in range(total_steps)]
          for l in range(LAYERS)]
    positions = torch.arange(CONTEXT, CONTEXT + total_steps, dtype=torch.int32, device=dev).view(total_steps, 1)
    lens = positions + 1
    outs = torch.empty(LAYERS, BATCH, HQ, D, dtype=torch.float32, device=dev)
    ws = torch.zeros(tq.tq_decode_workspace_bytes(params[0], BATCH, cap), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_OK, ("prefill", st, word)

    stream = torch.cuda.Stream(device=dev)

    def enqueue_step(i, decode_only=False):
        for l in range(LAYERS):
            if decode_only:
                tq.tq_decode_attention(params[l], kcb, vcb, qs[l][i], caches[l], lens[i], cap, outs[l], ws, err,
                                       stream=stream)
            else:  # append the step's token and attend, one launch per layer
                tq.tq_append_decode_attention(params[l], kcb, vcb, k_new[l][:, i:i + 1], v_new[l][:, i:i + 1],
                                              qs[l][i], caches[l], lens[i], cap, outs[l], ws, err, stream=stream)

    # one CUDA graph per step (the pointers of step i are baked in); --eager
    # enqueues the same launches directly instead (for profilers that cannot
    # follow graph kernel nodes)
    graphs = []
    with torch.cuda.stream(stream):
        for i in range(total_steps):
            if args.eager:
                graphs.append(EagerWork(lambda i=i: enqueue_step(i)))
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                enqueue_step(i)
            graphs.append(g)
        if args.eager:
            g_decode = EagerWork(lambda: enqueue_step(total_steps - 1, decode_only=True))
        else:
            g_decode = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_decode, stream=stream):
                enqueue_step(total_steps - 1, decode_only=True)
    torch.cuda.synchronize()

    for i in range(warmup):
        graphs[i].replay()
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        with torch.cuda.stream(stream):
            start.record(stream)
            for i in range(warmup, total_steps):
                graphs[i].replay()
            end.record(stream)
        end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    ms = max_over_ranks(ms, world)
    tokens_per_step = sum(LAYERS * BATCH * (CONTEXT + i + 1) for i in range(warmup, total_steps)) / steps
    value = world * tokens_per_step * steps / (ms / 1000.0)
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_OK, ("timed steps", st, word)

    # dominant kernel: decode attention alone, 32 layers per graph replay
    reps = 20
    with torch.cuda.stream(stream):
        g_decode.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g_decode.replay()
        e1.record(stream)
    e1.synchronize()
    decode_us = 1000.0 * e0.elapsed_time(e1) / (reps * LAYERS)
    seq = CONTEXT + total_steps
    alg_bytes = BATCH * HKV * seq * bytes_per_token_head()
    achieved = alg_bytes / (decode_us * 1e-6) / 1e9
    peak, peak_kind = measured_peaks()

    # end to end through the C ABI with host buffers: every step, the step's
    # inputs (each layer's new K and V rows and queries, staged in one pinned
    # slab) go in with one copy, and the outputs come back with one copy
    kv_elems, q_elems = BATCH * HKV * D, BATCH * HQ * D
    per_layer = 2 * kv_elems + q_elems  # bf16 elements: k row, v row, queries

    def layer_views(slab):
        ks, vs, qv = [], [], []
        for l in range(LAYERS):
            o = l * per_layer
            ks.append(slab[o:o + kv_elems].view(BATCH, 1, HKV, D))
            vs.append(slab[o + kv_elems:o + 2 * kv_elems].view(BATCH, 1, HKV, D))
            qv.append(slab[o + 2 * kv_elems:o + per_layer].view(BATCH, HQ, D))
        return ks, vs, qv

    h_in = torch.empty(LAYERS * per_layer, dtype=torch.bfloat16).pin_memory()
    h_k, h_v, h_q = layer_views(h_in)
    for l in range(LAYERS):
        h_k[l].copy_(k_new[l][:, -1:])
        h_v[l].copy_(v_new[l][:, -1:])
        h_q[l].copy_(qs[l][-1])
    # Two sets of device inputs and outputs (one CUDA graph each) so that the
    # copies overlap the kernels: step i's inputs go up on one copy stream
    # while step i - 1 computes, its outputs come down on another while step
    # i + 1 computes.  Every step still moves its own inputs and outputs
    # inside the timed region.
    h_out = [torch.empty(LAYERS, BATCH, HQ, D, dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in = [torch.empty(LAYERS * per_layer, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    outs_e = [torch.empty(LAYERS, BATCH, HQ, D, dtype=torch.float32, device=dev) for _ in range(2)]
    views = [layer_views(x) for x in s_in]
    last = total_steps - 1

    def e2e_layers(k):
        s_k, s_v, s_q = views[k]
        for l in range(LAYERS):
            tq.tq_append_decode_attention(params[l], kcb, vcb, s_k[l], s_v[l], s_q[l], caches[l], lens[last], cap,
                                          outs_e[k][l], ws, err, stream=stream)

    g_e2e = []
    for k in range(2):
        if args.eager:
            g_e2e.append(EagerWork(lambda k=k: e2e_layers(k)))
        else:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    e2e_layers(k)
            g_e2e.append(g)
    torch.cuda.synchronize()
    h2d = h_in.numel() * h_in.element_size()
    d2h = h_out[0].numel() * h_out[0].element_size()
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    fetched = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = steps
    for it in range(warmup + e2e_steps):
        k = it % 2
        if it == warmup:
            torch.cuda.synchronize()
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            up.wait_event(f0)
        up.wait_event(computed[k])  # step it - 2 has read this input set
        with torch.cuda.stream(up):
            s_in[k].copy_(h_in, non_blocking=True)
            in_ready[k].record(up)
        stream.wait_event(in_ready[k])
        stream.wait_event(fetched[k])  # step it - 2's outputs have left this output set
        with torch.cuda.stream(stream):  # a graph replays on the current stream
            g_e2e[k].replay()
        computed[k].record(stream)
        down.wait_event(computed[k])
        with torch.cuda.stream(down):
            h_out[k].copy_(outs_e[k], non_blocking=True)
            fetched[k].record(down)
    stream.wait_event(fetched[(warmup + e2e_steps - 1) % 2])
    f1.record(stream)
    f1.synchronize()
    # the same steps with every copy serialised with the kernels on one stream
    # (reported beside the pipelined figure)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for it in range(e2e_steps):
            s_in[0].copy_(h_in, non_blocking=True)
            g_e2e[0].replay()
            h_out[0].copy_(outs_e[0], non_blocking=True)
        g1.record(stream)
    g1.synchronize()
    serial_ms = max_over_ranks(g0.elapsed_time(g1), world)
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
    e2e_value = world * LAYERS * BATCH * (last + CONTEXT + 1) * e2e_steps / (e2e_ms / 1000.0)

    launches_per_step = LAYERS  # one fused append + decode-attention kernel per layer
    if rank == 0:
        cpu_info = oracle_sample(seconds_target=12.0)[1] if (world == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16-in/fp16-mma/fp32-acc", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": BATCH * world, "seq_len": CONTEXT + 1,
                       "layers": LAYERS, "parallelism": "replicas%d" % world if world > 1 else "none",
                       "l2": "inputs larger than L2: 32 distinct layer caches, %.0f MB" %
                             (LAYERS * HKV * seq * bytes_per_token_head() / 1e6),
                       "graphs": ("eager launches (--eager): " if args.eager else "one CUDA graph per step: ") +
                                 "32 x tq_append_decode_attention (append + attend, one kernel per layer)"},
            "hbm_gbs": alg_bytes * LAYERS / (ms / steps * 1e-3) / 1e9,
            "pct_of_8tbs": 100.0 * alg_bytes * LAYERS / (ms / steps * 1e-3) / 8e12,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": profiled_traffic("decode_mma_kernel", seq),
                         "peak_kind": peak_kind,
                         "kernel": "decode kernel timed alone (tq_decode_attention, no append), %.2f us per launch, %d B algorithmic"
                                   % (decode_us, alg_bytes)},
            "cpu_baseline": cpu_info,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "every step uploads its inputs (one copy) and downloads its outputs (one copy) inside "
                              "the timed region, on two copy streams that overlap the previous and next steps' "
                              "kernels (two sets of device buffers)",
                    "serial_value": world * LAYERS * BATCH * (last + CONTEXT + 1) * e2e_steps / (serial_ms / 1000.0)},
            "gpu_launches": launches_per_step * steps,
            "clocks": clocks.summary(),
        }
        if not args.quick and world == 1:  # the other workloads: single-GPU runs only (N GPUs stay held meanwhile)
            line["bf16_baseline"] = bf16_sdpa_baseline(dev)
            line["decode_configs"] = decode_configs(dev)
            line["paged_decode"] = {"workload": "llama3-8b-shaped layer, 32768 tokens, K4/V2, through a block "
                                                "table (blocks in random order)", **paged_decode(dev)}
            line["prefill"] = prefill_chunk(dev)
            if not args.no_cpu_baseline:
                line["prefill"]["cpu_baseline"] = oracle_prefill_sample()
            peak_gbs = measured_peaks()[0]
            q = {"workload": "bulk prefill quantise: 262144 tokens x 8 kv heads, bf16, 32 layers (0, 1, 30, 31 "
                             "int8 per-vector absmax, others K4/V3 turbo), one input slab, 32 distinct outputs",
                 "unit": "GB/s (input read + codes and norms written)"}
            for d in (128, 256):
                q["d%d" % d] = bulk_quantize(dev, d)
                q["d%d" % d]["frac_of_peak"] = round(q["d%d" % d]["sweep_gbs"] / peak_gbs, 4)
            line["quantize"] = q
        print(json.dumps(line), flush=True)
    del graphs, g_decode, g_e2e


def run_profile_case(args):
    """A small case for ncu: one Llama-3-8B-shaped layer (26 MB cache) and a
    few eager launches of one kernel; prints nothing worth timing."""
    from bit_kv_cache_tq_b200 import inputs, tq
    dev = torch.device("cuda", 0)
    params = tq.make_params(D, HQ, HKV, K_BITS, V_BITS, seed=SEED)
    kcb, vcb = tq.tq_codebook_init(D, K_BITS), tq.tq_codebook_init(D, V_BITS)
    cap = CONTEXT + 8
    cache = tq.alloc_cache(params, BATCH, cap, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pos = torch.zeros(BATCH, dtype=torch.int32, device=dev)
    k = inputs.lognormal_kv(BATCH, CONTEXT + 1, HKV, D, SEED, 0, inputs.K, device=dev)
    v = inputs.lognormal_kv(BATCH, CONTEXT + 1, HKV, D, SEED, 0, inputs.V, device=dev)
    if args.profile == "quantize":
        for _ in range(args.warmup + args.steps):
            tq.tq_quantize_append(params, kcb, vcb, k, v, pos, cache, err)
    elif args.profile == "prefill":
        # a 512-token chunk after 32768 cached tokens (the prefill workload)
        pcache = tq.alloc_cache(params, BATCH, CONTEXT + PREFILL_CHUNK, device=dev)
        tq.tq_quantize_append(params, kcb, vcb, k[:, :CONTEXT].contiguous(), v[:, :CONTEXT].contiguous(), pos,
                              pcache, err)
        kn = inputs.lognormal_kv(BATCH, PREFILL_CHUNK, HKV, D, SEED, 0, inputs.K, device=dev, token_offset_seed=3)
        vn = inputs.lognormal_kv(BATCH, PREFILL_CHUNK, HKV, D, SEED, 0, inputs.V, device=dev, token_offset_seed=3)
        q = inputs.queries(BATCH, PREFILL_CHUNK * HQ, D, SEED, device=dev).view(BATCH, PREFILL_CHUNK, HQ, D)
        start = torch.full((BATCH,), CONTEXT, dtype=torch.int32, device=dev)
        out = torch.empty(BATCH, PREFILL_CHUNK, HQ, D, dtype=torch.float32, device=dev)
        ws = torch.zeros(tq.tq_prefill_workspace_bytes(params, BATCH, PREFILL_CHUNK), dtype=torch.uint8, device=dev)
        for _ in range(args.warmup + args.steps):
            tq.tq_prefill_attention(params, kcb, vcb, kn, vn, q, start, pcache, out, ws, err)
    elif args.profile == "split":
        # the split-and-combine decode kernels: d = 256 heads (B=1, Hq=32,
        # Hkv=8, K4/V2), 8192 cached tokens
        p256 = tq.make_params(256, HQ, HKV, K_BITS, V_BITS, seed=SEED)
        kc2, vc2 = tq.tq_codebook_init(256, K_BITS), tq.tq_codebook_init(256, V_BITS)
        t256 = 8192
        c256 = tq.alloc_cache(p256, 1, t256 + 8, device=dev)
        k2 = inputs.lognormal_kv(1, t256, HKV, 256, SEED, 0, inputs.K, device=dev)
        v2 = inputs.lognormal_kv(1, t256, HKV, 256, SEED, 0, inputs.V, device=dev)
        tq.tq_quantize_append(p256, kc2, vc2, k2, v2, pos[:1], c256, err)
        q2 = inputs.queries(1, HQ, 256, SEED, device=dev)
        lens2 = torch.full((1,), t256, dtype=torch.int32, device=dev)
        ws2 = torch.zeros(tq.tq_decode_workspace_bytes(p256, 1, t256 + 8), dtype=torch.uint8, device=dev)
        out2 = torch.empty(1, HQ, 256, dtype=torch.float32, device=dev)
        for _ in range(args.warmup + args.steps):
            tq.tq_decode_attention(p256, kc2, vc2, q2, c256, lens2, t256 + 8, out2, ws2, err)
    elif args.profile == "dequantize":
        # dequantise one sequence's 32768 cached tokens (all kv heads, K and V)
        tq.tq_quantize_append(params, kcb, vcb, k, v, pos, cache, err)
        ko = torch.empty(CONTEXT, HKV, D, dtype=torch.float32, device=dev)  # token-major
        vo = torch.empty(CONTEXT, HKV, D, dtype=torch.float32, device=dev)
        for _ in range(args.warmup + args.steps):
            tq.tq_dequantize(params, kcb, vcb, cache, 0, 0, CONTEXT, ko, vo)
    else:
        tq.tq_quantize_append(params, kcb, vcb, k, v, pos, cache, err)
        q = inputs.queries(BATCH, HQ, D, SEED, device=dev)
        lens = torch.full((BATCH,), CONTEXT + 1, dtype=torch.int32, device=dev)
        ws = torch.zeros(tq.tq_decode_workspace_bytes(params, BATCH, cap), dtype=torch.uint8, device=dev)
        out = torch.empty(BATCH, HQ, D, dtype=torch.float32, device=dev)
        for _ in range(args.warmup + args.steps):
            tq.tq_decode_attention(params, kcb, vcb, q, cache, lens, cap, out, ws, err)
    torch.cuda.synchronize()
    st, word = tq.tq_read_device_error(err)
    assert st == tq.TQ_OK, (st, word)
    print(json.dumps({"profile_case": args.profile, "launches": args.warmup + args.steps + (args.profile == "decode")}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="enqueue each step's launches directly instead of replaying CUDA graphs")
    ap.add_argument("--quick", action="store_true",
                    help="skip the bf16 baseline and the bulk prefill quantise measurement")
    ap.add_argument("--profile", choices=["decode", "quantize", "prefill", "split", "dequantize"], default=None,
                    help="run a small one-layer case for ncu instead of the benchmark")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_tq(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
