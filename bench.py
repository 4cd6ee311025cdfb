"""Benchmark of the KV-vector quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload (default): 65,536 KV vectors, d = 128, fp16, rows = Gaussian direction
x LogNormal(0, 0.5) norm with 4 outlier channels x10 (seeded synthetic data,
one independent shard per rank). One step runs the fused quantize+dequantize
roundtrip for RotorQuant (and TurboQuant-mse when built) at b = 2, 3, 4 over
the batch. The headline `value` is the RotorQuant b = 3 roundtrip throughput
in million vectors per second, summed over ranks (weak scaling, no
collective on the data path). Step k runs on batch set k mod 8 (8 independent
batches, ~306 MB with their outputs: over twice L2, so no launch finds its inputs
in L2); each leg's K launches are captured into a CUDA graph and replayed back to
back between two CUDA events on the launching stream, and the max over ranks is
taken.

`--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_VEC = 65536
NSETS = 8  # independent batches the timed steps rotate over (inputs and outputs over twice L2)
D = 128
BITS = (2, 3, 4)
HEADLINE_BITS = 3
LARGE_ROWS = 4194304  # 1 GiB of fp16 input at d = 128


def rq_bytes_per_vector(d, bits, in_bytes=2, out_bytes=2):
    """Algorithmic bytes of the fused roundtrip: x in, packed codes + norm out, x_hat out."""
    G = -(-d // 3)
    W = -(-(3 * G * bits) // 32)
    return d * in_bytes + 4 * W + 4 + d * out_bytes


def leg_name(leg):
    """JSON key of a leg: rq_b3, tq_b2, ... and pq_4222 (PolarQuant's four levels of 4, 2, 2, 2 bits)."""
    kind, b = leg
    return "pq_4222" if kind == "pq" else "%s_b%d" % (kind, b)


def pq_bytes_per_vector(d=128, in_bytes=2, out_bytes=2):
    """PolarQuant fused roundtrip at d = 128: x in, 496 bits of angle codes and fp16 radii out, x_hat out."""
    return d * in_bytes + 62 + d * out_bytes


def tq_bytes_per_vector(d, bits, in_bytes=2, out_bytes=2):
    """TurboQuant-mse fused roundtrip: x in, d codes of b bits + norm out, x_hat out."""
    return d * in_bytes + 4 * (-(-(d * bits) // 32)) + 4 + d * out_bytes


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j.get("hbm_gbs"), "measured"
    return 6650.0, "fallback"


def kernel_source_hash(spec):
    """SHA-256 prefix of a kernel's source: `file#ns` hashes the text of `namespace ns { ... }  // namespace ns`
    in that file together with the device headers it includes (helpers and the bisection quantizer); a plain
    path hashes the whole file."""
    import hashlib

    path, _, ns = spec.partition("#")
    src = os.path.join(ROOT, path)
    if not os.path.exists(src):
        return None
    text = open(src, "rb").read()
    if ns:
        a = text.find(("namespace %s {" % ns).encode())
        b = text.find(("}  // namespace %s" % ns).encode())
        if a < 0 or b < a:
            return None
        text = text[a:b]
        for hdr in ("kvrq_device.cuh", "bisect.cuh"):
            text += open(os.path.join(os.path.dirname(src), hdr), "rb").read()
    return hashlib.sha256(text).hexdigest()[:16]


def build_identity():
    """What was measured: the git commit when the tree has its history (a snapshot copied without .git has
    none), and a SHA-256 prefix of the library's sources, the public header and this script, which names
    the build either way."""
    import hashlib
    import subprocess

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_vector_rq_b200", "csrc")
    files = sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh", ".h", ".cpp")))
    files += [os.path.join(ROOT, "include", "kvrq.h"), os.path.abspath(__file__)]
    for f in files:
        h.update(os.path.relpath(f, ROOT).encode() + b"\0" + open(f, "rb").read())
    sha = None
    try:
        out = subprocess.run(["git", "-C", ROOT, "rev-parse", "HEAD"], capture_output=True, text=True, timeout=10)
        if out.returncode == 0:
            sha = out.stdout.strip() or None
    except (OSError, subprocess.SubprocessError):
        sha = None
    return {"git_sha": sha, "source_sha256": h.hexdigest()[:16]}


def recorded_traffic(kernel):
    """Per-launch DRAM bytes of `kernel` from profiles/traffic.txt, or None when that record is missing or the
    kernel's source changed since the counters were taken (the record keeps a SHA-256 prefix of the source)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        if line.startswith("#") or "|" not in line:
            continue
        f = [x.strip() for x in line.split("|")]
        if f[0] != kernel:
            continue
        if kernel_source_hash(f[1]) != f[2]:
            return None
        return int(f[4]) + int(f[5])
    return None


def measured_tensor_peak():
    """Dense fp16/bf16 tensor-core peak in TFLOP/s: the measured cuBLAS bf16 burst figure (fp16 runs at the same
    nominal rate), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f).get("bf16_tflops", 1590.0))
    return 1590.0


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_oracle_rate(n_sample, bits=HEADLINE_BITS, seed=0):
    """Vectors/s of the oracle's RQ roundtrip on one host core (bounded sample; numpy's BLAS held to one
    thread, so that one core is what it uses)."""
    from threadpoolctl import threadpool_limits

    from kv_cache_vector_rq_b200 import synth
    from oracle import codebook, params, rq

    x = synth.lognormal(n_sample, D, seed=seed).float().numpy().astype(np.float64)
    rot = params.rotors(D, 1)
    c, _, _ = codebook.lloyd_max(D, bits)
    with threadpool_limits(1):
        t0 = time.perf_counter()
        rq.roundtrip(x, rot, c, bits)
        dt = time.perf_counter() - t0
    return n_sample / dt, dt


def boundary_ties(kind, bits, x_rows, gpu_words, rot, pi, centroids):
    """Sampled oracle comparison of one leg's packed codes: (coordinates within 1e-5 of a decision boundary,
    codes that differ from the oracle's, codes that differ away from a boundary). The parameters are the
    device's rounded values as float64 numbers."""
    from oracle import codes as ocodes, polar, rq, tq

    c = np.asarray(centroids, dtype=np.float64)
    if kind == "pq":
        books = [c[:16], c[16:20], c[20:24], c[24:28]]
        ref = polar.quantize(x_rows, pi, books)
        gw = np.asarray(gpu_words, dtype=np.uint32)
        near = diff = far_ = 0
        for lv, (w0, w1, b) in enumerate([(0, 8, 4), (8, 10, 2), (10, 11, 2), (11, 12, 2)]):
            g = ocodes.unpack(gw[:, w0:w1], 64 >> lv, b)
            t = 0.5 * (books[lv][:-1] + books[lv][1:])
            if lv == 0:
                t = np.concatenate([[0.0, 2.0 * np.pi], t])
            dist = np.min(np.abs(np.asarray(ref["angles"][lv])[..., None] - t), axis=-1)
            d_ = g != ref["codes"][lv]
            near += int((dist < 1e-5).sum())
            diff += int(d_.sum())
            far_ += int((d_ & ~(dist < 1e-5)).sum())
        return near, diff, far_
    if kind == "rq":
        ref = rq.quantize(x_rows, rot, c, bits)
        n_codes = 3 * (-(-D // 3))
    else:
        ref = tq.mse_quantize(x_rows, pi, c, bits)
        n_codes = D
    g = ocodes.unpack(np.asarray(gpu_words, dtype=np.uint32), n_codes, bits)
    t = 0.5 * (c[:-1] + c[1:])
    near = np.min(np.abs(ref["y"][..., None] - t), axis=-1) < 1e-5
    diff = g != ref["codes"]
    return int(near.sum()), int(diff.sum()), int((diff & ~near).sum())


def _oracle_worker(job):
    n, seed = job
    return cpu_oracle_rate(n, seed=seed)[1]


def cpu_oracle_all_cores(n_per_worker, max_workers=32):
    """(vectors/s, workers): the same oracle on every host core at once, one single-threaded worker per core
    (a spawn pool: a forked child of a process that holds a CUDA context would hang), each on its own rows.
    The rate is all rows over the slowest worker's oracle time."""
    import multiprocessing

    workers = max(1, min(max_workers, len(os.sched_getaffinity(0))))
    with multiprocessing.get_context("spawn").Pool(workers) as pool:
        pool.map(_oracle_worker, [(32, 100 + i) for i in range(workers)])  # imports and set-up
        dts = pool.map(_oracle_worker, [(n_per_worker, 200 + i) for i in range(workers)])
    return workers * n_per_worker / max(dts), workers


def max_over_ranks(v, world, dist=None, device=None):
    """The largest of every rank's v (times: the slowest rank sets the step), by one all-reduce."""
    if world == 1:
        return v
    import torch

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Units per second over all ranks: every rank processes its own shard of units_per_rank (weak scaling)."""
    return units_per_rank * world / (ms * 1e-3)


def shard_seed(rank):
    """Seed of a rank's input shard: ranks draw different vectors."""
    return 1000 + rank


def run_reference(args, rank, world):
    if rank != 0:
        return
    sample = 2048
    for _ in range(args.warmup):
        cpu_oracle_rate(256)
    times = []
    for k in range(args.steps):
        rate, dt = cpu_oracle_rate(sample, seed=k)
        times.append(dt)
    t = sum(times) / len(times)
    value = sample / t / 1e6
    line = {
        "impl": "reference", "metric": "quantize+dequantize Mvec/s at d=128 3-bit", "value": value,
        "unit": "Mvec/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "65536 x d128 fp16 KV vectors (LogNormal norms, 4 outlier channels x10), "
                               "RotorQuant 3-bit quantize+dequantize", "sample_rows_per_step": sample},
        "cpu_baseline": {"value": value, "unit": "Mvec/s", "cores": 1, "kind": "oracle",
                         "sample": "%d rows of the workload per step, float64 numpy oracle" % sample},
        "e2e": {"value": value, "unit": "Mvec/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def decode_step_c4(kvrq, synth, torch, dev, batch, steps, warmup, layers=36, kv_heads=2, group=8,
                   cached=131072):
    """Qwen2.5-3B-shaped decode step: append one K (TurboQuant-prod 3-bit) and one V
    (RotorQuant 3-bit) per (layer, batch, KV head), then score all 16 query heads over
    cached + 1 tokens straight from the packed keys. Returns timings and traffic."""
    heads = layers * kv_heads * batch
    t_max = cached + 1
    bits_k, bits_v = 3, 3
    pi = torch.from_numpy(kvrq.tq_rotation_init(D, 2)).to(torch.float16).to(dev)
    T = torch.from_numpy(kvrq.qjl_matrix_init(D, D, 3)).to(torch.float16).to(dev)
    rot = torch.from_numpy(kvrq.rq_rotors_init(D, 1).astype(np.float32)).to(dev)
    ck = torch.from_numpy(kvrq.tq_codebook_init(D, bits_k - 1)[0].astype(np.float32)).to(dev)
    cv = torch.from_numpy(kvrq.tq_codebook_init(D, bits_v)[0].astype(np.float32)).to(dev)
    Wk, Wv = kvrq.packed_words(D, bits_k - 1), kvrq.packed_words(129, bits_v)
    k_codes = torch.empty((heads, t_max, Wk), dtype=torch.int32, device=dev)
    k_signs = torch.empty((heads, t_max, D // 32), dtype=torch.int32, device=dev)
    k_norms = torch.empty((heads, t_max), dtype=torch.float32, device=dev)
    k_gam = torch.empty((heads, t_max), dtype=torch.float32, device=dev)
    v_codes = torch.empty((heads, t_max, Wv), dtype=torch.int32, device=dev)
    v_norms = torch.empty((heads, t_max), dtype=torch.float32, device=dev)
    # prefill (untimed): the cached tokens, quantized in chunks of heads
    chunk = max(1, (1 << 22) // cached)
    for h0 in range(0, heads, chunk):
        h1 = min(heads, h0 + chunk)
        rows = (h1 - h0) * t_max
        kx = synth.lognormal(rows, D, seed=5000 + h0, dtype=torch.float16, device=dev)
        kvrq.tq_quantize_prod(kx, pi, T, ck, bits_k, codes=k_codes[h0:h1].view(rows, Wk),
                              norms=k_norms[h0:h1].reshape(rows), signs=k_signs[h0:h1].view(rows, D // 32),
                              gammas=k_gam[h0:h1].reshape(rows))
        vx = synth.gaussian(rows, D, seed=7000 + h0, dtype=torch.float16, device=dev)
        kvrq.rq_quantize(vx, rot, cv, bits_v, codes=v_codes[h0:h1].view(rows, Wv), norms=v_norms[h0:h1].reshape(rows))
        del kx, vx
    torch.cuda.synchronize()
    q = synth.gaussian(heads * group, D, seed=9, dtype=torch.float16, device=dev).view(heads, group, D)
    new_k = synth.lognormal(heads, D, seed=10, dtype=torch.float16, device=dev)
    new_v = synth.gaussian(heads, D, seed=11, dtype=torch.float16, device=dev)
    scores = torch.empty((heads, group, t_max), dtype=torch.float32, device=dev)
    # the calls take the current stream at call time: the capture stream while a graph is recorded
    def append():
        st = torch.cuda.current_stream()
        kvrq.kv_cache_append(kvrq.TQ_PROD, new_k, cached, bits_k, ck, k_codes, k_norms, pi=pi, T=T, signs=k_signs,
                             gammas=k_gam, stream=st)
        kvrq.kv_cache_append(kvrq.RQ_MSE, new_v, cached, bits_v, cv, v_codes, v_norms, rotors=rot, stream=st)

    def score():
        kvrq.kv_score_packed(kvrq.TQ_PROD, q, k_codes, k_norms, bits_k, t_max, ck, pi=pi, T=T, signs=k_signs,
                             gammas=k_gam, scores=scores, stream=torch.cuda.current_stream())

    for _ in range(warmup):
        append()
        score()
    torch.cuda.synchronize()
    kvrq.device_status()
    # the appends and the scores each captured into a CUDA graph: replays run their launches back to back
    # on the device, so the host cost of the calls stays out of the timed region
    g_app, g_sc = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_app):
        append()
    with torch.cuda.graph(g_sc):
        score()
    stream = torch.cuda.current_stream()
    g_app.replay()
    g_sc.replay()
    torch.cuda.synchronize()
    tot, sc = [], []
    for _ in range(steps):
        s, m, e = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        s.record(stream)
        g_app.replay()
        m.record(stream)
        g_sc.replay()
        e.record(stream)
        e.synchronize()
        tot.append(s.elapsed_time(e))
        sc.append(m.elapsed_time(e))
    del g_app, g_sc
    kvrq.device_status()
    ms, ms_score = sum(tot) / len(tot), sum(sc) / len(sc)
    keys = heads * t_max
    score_bytes = keys * (4 * Wk + 4 * (D // 32) + 8) + keys * group * 4
    out = {"batch": batch, "layers": layers, "kv_heads": kv_heads, "query_heads_per_kv": group, "tokens": t_max,
           "timing": "CUDA events around graph replays of the appends and of the scores", "ms_per_step": ms, "ms_score": ms_score, "keys_scored_per_s": keys / (ms_score * 1e-3),
           "score_GB_s": score_bytes / (ms_score * 1e-3) / 1e9, "score_bytes_per_step": score_bytes}
    del k_codes, k_signs, k_norms, k_gam, v_codes, v_norms, scores
    torch.cuda.empty_cache()
    return out


def decode_attention_c4(kvrq, synth, torch, dev, batch, steps, warmup, layers=36, kv_heads=2, group=8,
                        cached=131072):
    """Qwen2.5-3B-shaped decode attention: for every (layer, batch, KV head), the 8 query heads
    of its group attend over cached + 1 tokens of a packed cache (keys TurboQuant-prod 3-bit,
    values RotorQuant 3-bit), softmax(q k_hat / sqrt(d)) v_hat straight from the codes. The
    cache is 4x L2 or more, so every call streams it from HBM."""
    heads = layers * kv_heads * batch
    t_max = cached + 1
    # capacity in whole 16-token blocks, as a cache allocator (or a page pool) gives it: every head's
    # rows then start 16-byte aligned, which the kernel's bulk copies need for 52-byte value rows
    cap = -(-t_max // 16) * 16
    pi = torch.from_numpy(kvrq.tq_rotation_init(D, 2)).to(torch.float16).to(dev)
    T = torch.from_numpy(kvrq.qjl_matrix_init(D, D, 3)).to(torch.float16).to(dev)
    rot = torch.from_numpy(kvrq.rq_rotors_init(D, 1).astype(np.float32)).to(dev)
    ck = torch.from_numpy(kvrq.tq_codebook_init(D, 2)[0].astype(np.float32)).to(dev)
    cv = torch.from_numpy(kvrq.tq_codebook_init(D, 3)[0].astype(np.float32)).to(dev)
    Wk, Wv = kvrq.packed_words(D, 2), kvrq.packed_words(129, 3)
    k_codes = torch.empty((heads, cap, Wk), dtype=torch.int32, device=dev)
    k_signs = torch.empty((heads, cap, D // 32), dtype=torch.int32, device=dev)
    k_norms = torch.empty((heads, cap), dtype=torch.float32, device=dev)
    k_gam = torch.empty((heads, cap), dtype=torch.float32, device=dev)
    v_codes = torch.empty((heads, cap, Wv), dtype=torch.int32, device=dev)
    v_norms = torch.empty((heads, cap), dtype=torch.float32, device=dev)
    chunk = max(1, (1 << 22) // cap)
    for h0 in range(0, heads, chunk):  # prefill (untimed)
        h1 = min(heads, h0 + chunk)
        rows = (h1 - h0) * cap
        kx = synth.lognormal(rows, D, seed=5000 + h0, dtype=torch.float16, device=dev)
        kvrq.tq_quantize_prod(kx, pi, T, ck, 3, codes=k_codes[h0:h1].view(rows, Wk),
                              norms=k_norms[h0:h1].reshape(rows), signs=k_signs[h0:h1].view(rows, D // 32),
                              gammas=k_gam[h0:h1].reshape(rows))
        vx = synth.gaussian(rows, D, seed=7000 + h0, dtype=torch.float16, device=dev)
        kvrq.rq_quantize(vx, rot, cv, 3, codes=v_codes[h0:h1].view(rows, Wv), norms=v_norms[h0:h1].reshape(rows))
        del kx, vx
    q = synth.gaussian(heads * group, D, seed=9, dtype=torch.float16, device=dev).view(heads, group, D)
    out = torch.empty((heads, group, D), dtype=torch.float32, device=dev)
    ws = torch.empty(kvrq.attention_workspace_bytes(heads, group, t_max) // 4 + 4, dtype=torch.float32, device=dev)
    # the current stream at call time: the capture stream while the graph below is recorded
    fn = lambda: kvrq.kv_attention_packed(kvrq.TQ_PROD, q, k_codes, k_norms, 3, v_codes, v_norms, 3, t_max, ck, rot,
                                          cv, pi=pi, T=T, k_signs=k_signs, k_gammas=k_gam, out=out, workspace=ws,
                                          stream=torch.cuda.current_stream())
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    kvrq.device_status()
    # one call (its three launches) captured into a CUDA graph: a replay runs them back to back on the
    # device, so the host cost of the call (binding, argument checks) stays out of the timed region
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    stream = torch.cuda.current_stream()
    g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        g.replay()
        e.record(stream)
        e.synchronize()
        ts.append(s.elapsed_time(e))
    del g
    kvrq.device_status()
    ms = sum(ts) / len(ts)
    tokens = heads * t_max
    cache_bytes = tokens * (4 * Wk + 4 * (D // 32) + 8 + 4 * Wv + 4)  # keys 56 B + values 56 B per token
    res = {"batch": batch, "layers": layers, "kv_heads": kv_heads, "query_heads_per_kv": group, "tokens": t_max,
           "capacity": cap,
           "ms_per_call": ms, "tokens_per_s": tokens / (ms * 1e-3), "cache_bytes": cache_bytes,
           "cache_GB_s": cache_bytes / (ms * 1e-3) / 1e9, "launches_per_call": 3}
    del k_codes, k_signs, k_norms, k_gam, v_codes, v_norms, ws
    torch.cuda.empty_cache()
    return res


def kv_stack_c3(kvrq, synth, torch, dev, steps, layers=32, kv_heads=8, tokens=32768):
    """Llama-3.1-8B-shaped KV stack: keys from a rank-16 factor model with 4 outlier channels,
    values N(0,1), both bf16 [layers][KV heads][tokens][128]; keys compressed with TurboQuant-prod
    3-bit (2-bit codes + 1-bit QJL, m = 128), values with RotorQuant 3-bit. Each timed step compresses
    the whole stack (8,388,608 keys and as many values, 4 GiB of input)."""
    n = layers * kv_heads * tokens
    k = synth.factor_keys(layers, kv_heads, tokens, D, seed=21, dtype=torch.bfloat16, device=dev).view(n, D)
    v = synth.gaussian(n, D, seed=22, dtype=torch.bfloat16, device=dev)
    pi = torch.from_numpy(kvrq.tq_rotation_init(D, 2)).to(torch.bfloat16).to(dev)
    T = torch.from_numpy(kvrq.qjl_matrix_init(D, D, 3)).to(torch.float16).to(dev)
    rot = torch.from_numpy(kvrq.rq_rotors_init(D, 1).astype(np.float32)).to(dev)
    ck = torch.from_numpy(kvrq.tq_codebook_init(D, 2)[0].astype(np.float32)).to(dev)
    cv = torch.from_numpy(kvrq.tq_codebook_init(D, 3)[0].astype(np.float32)).to(dev)
    kc, ks, kg, kn = kvrq.tq_quantize_prod(k, pi, T, ck, 3)
    vc, vn = kvrq.rq_quantize(v, rot, cv, 3)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    tk, tv = [], []
    for i in range(steps + 2):
        a, b, c = ev(), ev(), ev()
        a.record(stream)
        kvrq.tq_quantize_prod(k, pi, T, ck, 3, codes=kc, signs=ks, gammas=kg, norms=kn, stream=stream)
        b.record(stream)
        kvrq.rq_quantize(v, rot, cv, 3, codes=vc, norms=vn, stream=stream)
        c.record(stream)
        c.synchronize()
        if i >= 2:
            tk.append(a.elapsed_time(b))
            tv.append(b.elapsed_time(c))
    kvrq.device_status()
    mk, mv = sum(tk) / len(tk), sum(tv) / len(tv)
    bk = 2 * D + 4 * kvrq.packed_words(D, 2) + 4 * (D // 32) + 8  # 312 B per key
    bv = 2 * D + 4 * kvrq.packed_words(129, 3) + 4                  # 312 B per value
    out = {"vectors_each": n, "keys_ms": mk, "values_ms": mv, "ms_per_step": mk + mv,
           "keys_Gvec_s": n / mk / 1e6, "values_Gvec_s": n / mv / 1e6,
           "keys_GB_s": n * bk / mk / 1e6, "values_GB_s": n * bv / mv / 1e6,
           "stack_GB_s": n * (bk + bv) / (mk + mv) / 1e6,
           "keys_TFLOP_s": n * 4.0 * D * D / mk / 1e9}
    del k, v, kc, ks, kg, kn, vc, vn
    torch.cuda.empty_cache()
    return out


def run_leg_only(args):
    """One kernel leg on args.rows seeded vectors: a warm-up call, then args.iters timed calls."""
    import torch

    import kv_cache_vector_rq_b200 as kvrq
    from kv_cache_vector_rq_b200 import synth

    dev = torch.device("cuda", 0)
    if args.leg.startswith("score"):
        # packed-key scores (TurboQuant-prod 3-bit keys, 72 KV heads x 8 query heads), args.rows keys in total
        heads, group = 72, 8
        t = max(1, args.rows // heads)
        pi = torch.from_numpy(kvrq.tq_rotation_init(D, 2)).to(torch.float16).to(dev)
        T = torch.from_numpy(kvrq.qjl_matrix_init(D, D, 3)).to(torch.float16).to(dev)
        ck = torch.from_numpy(kvrq.tq_codebook_init(D, 2)[0].astype(np.float32)).to(dev)
        kx = synth.lognormal(heads * t, D, seed=3, dtype=torch.float16, device=dev)
        codes, signs, gam, norms = kvrq.tq_quantize_prod(kx, pi, T, ck, 3)
        del kx
        q = synth.gaussian(heads * group, D, seed=4, dtype=torch.float16, device=dev).view(heads, group, D)
        sc = torch.empty((heads, group, t), dtype=torch.float32, device=dev)
        fn = lambda: kvrq.kv_score_packed(kvrq.TQ_PROD, q, codes.view(heads, t, -1), norms.view(heads, t), 3, t, ck,
                                          pi=pi, T=T, signs=signs.view(heads, t, -1), gammas=gam.view(heads, t),
                                          scores=sc)
        rows = heads * t
    else:
        fn, rows = None, None
    if args.leg in ("pq_qdq", "pq_dq"):  # PolarQuant at d = 128 (levels of 4, 2, 2, 2 bits): roundtrip, dequantize
        x = synth.lognormal(args.rows, D, seed=1, dtype=torch.float16, device=dev)
        pi = torch.from_numpy(kvrq.tq_rotation_init(D, 2)).to(torch.float16).to(dev)
        pc = torch.from_numpy(kvrq.pq_codebooks()).to(dev)
        codes = torch.empty((args.rows, kvrq.PQ_WORDS), dtype=torch.int32, device=dev)
        xh = torch.empty_like(x)
        if args.leg == "pq_qdq":
            fn = lambda: kvrq.pq_quantize_dequantize(x, pi, pc, codes=codes, xhat=xh)
        else:
            kvrq.pq_quantize_dequantize(x, pi, pc, codes=codes, xhat=xh)
            fn = lambda: kvrq.pq_dequantize(codes, D, pi, pc, xhat=xh)
        rows = args.rows
    if fn is not None:
        return time_fn(fn, rows, args, torch, kvrq)
    kind, b = args.leg.rsplit("_", 1)[0], args.leg.rsplit("_", 1)[1]
    mode, b = b.rstrip("0123456789"), int(b.lstrip("qdmpro"))
    rows = args.rows
    dd = args.dim
    x = synth.lognormal(rows, dd, seed=1, dtype=torch.float16, device=dev, outliers=() if dd != D else
                        synth.OUTLIER_CHANNELS)
    xh = torch.empty_like(x)
    if kind == "rq":
        rot = torch.from_numpy(kvrq.rq_rotors_init(dd, 1).astype(np.float32)).to(dev)
        cb = torch.from_numpy(kvrq.tq_codebook_init(dd, b)[0].astype(np.float32)).to(dev)
        codes, norms = kvrq.rq_quantize(x, rot, cb, b)
        calls = {"q": lambda: kvrq.rq_quantize(x, rot, cb, b, codes=codes, norms=norms),
                 "dq": lambda: kvrq.rq_dequantize(codes, norms, dd, rot, cb, b, xhat=xh),
                 "qdq": lambda: kvrq.rq_quantize_dequantize(x, rot, cb, b, codes=codes, norms=norms, xhat=xh)}
    else:
        D_ = dd
        pi = torch.from_numpy(kvrq.tq_rotation_init(D_, 2)).to(torch.float16).to(dev)
        T = torch.from_numpy(kvrq.qjl_matrix_init(D_, D_, 3)).to(torch.float16).to(dev)
        prod = mode in ("prod", "dqp")
        cb = torch.from_numpy(kvrq.tq_codebook_init(D_, b - 1 if prod else b)[0].astype(np.float32)).to(dev)
        ws = kvrq.tq_workspace(rows, D_, dev, max_bytes=1 << 30) if kvrq.tq_needs_workspace(D_, x.dtype) else None
        if prod:
            codes, signs, gam, norms = kvrq.tq_quantize_prod(x, pi, T, cb, b)
        else:
            codes, norms = kvrq.tq_quantize_mse(x, pi, cb, b)
        calls = {"q": lambda: kvrq.tq_quantize_mse(x, pi, cb, b, codes=codes, norms=norms),
                 "qdq": lambda: kvrq.tq_quantize_dequantize_mse(x, pi, cb, b, codes=codes, norms=norms, xhat=xh),
                 "dqm": lambda: kvrq.tq_dequantize(codes, norms, D_, pi, cb, b, xhat=xh)}
        if prod:
            calls["prod"] = lambda: kvrq.tq_quantize_prod(x, pi, T, cb, b, codes=codes, norms=norms, signs=signs,
                                                          gammas=gam, workspace=ws)
            calls["dqp"] = lambda: kvrq.tq_dequantize(codes, norms, D_, pi, cb, b, signs=signs, gammas=gam, T=T,
                                                      xhat=xh, workspace=ws)
    return time_fn(calls[mode], rows, args, torch, kvrq)


def run_attention(args):
    """Decode attention at batch 1 and 16 (the packed caches of 151M tokens at batch 16 take
    about 17 GB); one JSON line with the per-call time and the cache bytes streamed per second."""
    import torch

    import kv_cache_vector_rq_b200 as kvrq
    from kv_cache_vector_rq_b200 import synth

    dev = torch.device("cuda", 0)
    peak, kind = measured_peaks()
    res = {"leg": "decode_attention_c4", "timing": "CUDA events around a CUDA graph replay of one call",
           "hbm_peak_gbs": peak,
           "peak_kind": kind}
    for b in [int(v) for v in args.attn_batches.split(",")]:
        r = decode_attention_c4(kvrq, synth, torch, dev, b, args.steps, args.warmup, cached=args.attn_tokens)
        r["frac_of_hbm_peak"] = r["cache_GB_s"] / peak
        res["batch%d" % b] = r
    print(json.dumps(res), flush=True)


def run_dim_sweep(args):
    """Config-5 sweep: 1 GiB of fp16 rows (N(0,1) directions, LogNormal(0, 0.5) norms, no outlier
    channels) per d; each cell timed over args.iters calls after a warm-up call (inputs >> L2)."""
    import torch

    import kv_cache_vector_rq_b200 as kvrq
    from kv_cache_vector_rq_b200 import synth

    dev = torch.device("cuda", 0)
    peak, peak_kind = measured_peaks()
    tflops_peak = measured_tensor_peak()
    clk = ClockSampler(0)
    clk.__enter__()
    cells = []
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        s, e = ev(), ev()
        s.record()
        for _ in range(args.iters):
            fn()
        e.record()
        torch.cuda.synchronize()
        kvrq.device_status()
        return s.elapsed_time(e) / args.iters

    for d in (128, 256, 1536, 4096):
        rows = (1 << 30) // (2 * d)
        x = synth.lognormal(rows, d, seed=5 + d, dtype=torch.float16, device=dev, outliers=())
        xh = torch.empty_like(x)
        rot = torch.from_numpy(kvrq.rq_rotors_init(d, 1).astype(np.float32)).to(dev)
        pi = torch.from_numpy(kvrq.tq_rotation_init(d, 2)).to(torch.float16).to(dev)
        T = torch.from_numpy(kvrq.qjl_matrix_init(d, d, 3)).to(torch.float16).to(dev)
        ws = kvrq.tq_workspace(rows, d, dev) if kvrq.tq_needs_workspace(d, x.dtype) else None
        for b in (2, 3, 4):
            cb = torch.from_numpy(kvrq.tq_codebook_init(d, b)[0].astype(np.float32)).to(dev)
            rc, rn = kvrq.rq_quantize(x, rot, cb, b)
            ms = timed(lambda: kvrq.rq_quantize_dequantize(x, rot, cb, b, codes=rc, norms=rn, xhat=xh))
            bpv = rq_bytes_per_vector(d, b)
            cells.append({"d": d, "b": b, "path": "rq_roundtrip", "rows": rows, "ms": ms,
                          "Mvec_s": rows / ms / 1e3, "GB_s": bpv * rows / ms / 1e6,
                          "frac_hbm": bpv * rows / ms / 1e6 / peak})
            del rc, rn
            cp = torch.from_numpy(kvrq.tq_codebook_init(d, b - 1)[0].astype(np.float32)).to(dev)
            codes, signs, gam, norms = kvrq.tq_quantize_prod(x, pi, T, cp, b, workspace=ws)
            msq = timed(lambda: kvrq.tq_quantize_prod(x, pi, T, cp, b, codes=codes, norms=norms, signs=signs,
                                                      gammas=gam, workspace=ws))
            msd = timed(lambda: kvrq.tq_dequantize(codes, norms, d, pi, cp, b, signs=signs, gammas=gam, T=T,
                                                   xhat=xh, workspace=ws))
            flops_q = 2.0 * d * d * 2  # y = Pi x, z = T r (m = d)
            bq = 2 * d + 4 * kvrq.packed_words(d, b - 1) + 4 * (d // 32) + 8
            for path, t, by in (("tq_prod_quantize", msq, bq), ("tq_prod_dequantize", msd, bq),
                                ("tq_prod_roundtrip", msq + msd, 2 * bq)):
                fl = flops_q * (2 if path == "tq_prod_roundtrip" else 1)
                cells.append({"d": d, "b": b, "path": path, "rows": rows, "ms": t, "Mvec_s": rows / t / 1e3,
                              "GB_s": by * rows / t / 1e6, "TFLOP_s": fl * rows / t / 1e9,
                              "frac_tensor": fl * rows / t / 1e9 / tflops_peak})
            del codes, signs, gam, norms
        del x, xh, ws
        torch.cuda.empty_cache()
    clk.__exit__(None, None, None)
    print(json.dumps({"sweep": "config5", "input": "1 GiB fp16 per d", "peak_GB_s": peak, "peak_kind": peak_kind,
                      "tensor_peak_TFLOP_s": tflops_peak, "cells": cells, "clocks": clk.summary()}), flush=True)


def time_fn(fn, rows, args, torch, kvrq):
    """args.iters calls timed on the device. The calls are captured once into a CUDA graph and the graph is
    replayed, so the host cost of a call (binding, tensor-map encoding) does not pace small launches."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(args.iters):
            fn()
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    g.replay()
    e.record()
    torch.cuda.synchronize()
    kvrq.device_status()
    ms = s.elapsed_time(e) / args.iters
    print(json.dumps({"leg": args.leg, "rows": rows, "ms": ms, "Mvec_s": rows / ms / 1e3, "timing": "graph replay"}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvrq", choices=["kvrq", "reference"])
    ap.add_argument("--no-large", action="store_true", help="skip the 1 GiB HBM-roofline leg")
    ap.add_argument("--leg", default=None,
                    help="time one kernel leg (rq_q3, rq_dq3, rq_qdq3, tq_q3, tq_qdq3, tq_prod3, tq_dqm3, tq_dqp3, "
                         "any b; score_prod3; pq_qdq, pq_dq) on --rows vectors instead of the workload; used for profiler "
                         "captures")
    ap.add_argument("--rows", type=int, default=1 << 20)
    ap.add_argument("--dim", type=int, default=D, help="head dimension of --leg (the tiled TurboQuant path "
                                                       "and the general RotorQuant kernel run d != 128)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--c5", action="store_true",
                    help="dimension sweep at 1 GiB fp16 input: d in {128, 256, 1536, 4096}, b in {2, 3, 4}, "
                         "RotorQuant roundtrip vs TurboQuant-prod quantize + dequantize; one JSON line")
    ap.add_argument("--attn", action="store_true",
                    help="decode attention from the packed cache at the Qwen2.5-3B decode shape (batch 1 and 16); "
                         "one JSON line")
    ap.add_argument("--attn-batches", default="1,16", help="batches of --attn (comma separated)")
    ap.add_argument("--attn-tokens", type=int, default=131072, help="cached tokens of --attn (one more is appended)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.leg:
        run_leg_only(args)
        return
    if args.c5:
        run_dim_sweep(args)
        return
    if args.attn:
        run_attention(args)
        return

    import torch
    import torch.distributed as dist

    import kv_cache_vector_rq_b200 as kvrq
    from kv_cache_vector_rq_b200 import synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def ranks_max(v):
        return max_over_ranks(v, world, dist, dev)

    # ---------------------------------------------------------------- inputs and parameters
    # NSETS independent batches of the workload (inputs and outputs ~306 MB, over twice L2): step k runs on
    # set k mod NSETS, so no launch finds its inputs in L2 (the previous NSETS - 1 launches streamed ~268 MB)
    xs = [synth.lognormal(N_VEC, D, seed=shard_seed(rank) * 16 + k, dtype=torch.float16, device=dev)
          for k in range(NSETS)]
    x = xs[0]
    rot = torch.from_numpy(kvrq.rq_rotors_init(D, 1).astype(np.float32)).to(dev)
    cbs = {b: torch.from_numpy(kvrq.tq_codebook_init(D, b)[0].astype(np.float32)).to(dev) for b in BITS}
    W = {b: kvrq.packed_words(3 * kvrq.rq_groups(D), b) for b in BITS}
    WMAX = max(max(W.values()), max(kvrq.packed_words(D, b) for b in BITS))
    codes_all = [torch.empty((N_VEC, WMAX), dtype=torch.int32, device=dev) for _ in range(NSETS)]
    norms_all = [torch.empty(N_VEC, dtype=torch.float32, device=dev) for _ in range(NSETS)]
    xhats = [torch.empty_like(x) for _ in range(NSETS)]
    codes = {b: codes_all[0][:, :W[b]] for b in BITS}
    norms, xhat = norms_all[0], xhats[0]
    stream = torch.cuda.current_stream()

    pi = torch.from_numpy(kvrq.tq_rotation_init(D, 2)).to(torch.float16).to(dev)
    tq_codes = {b: codes_all[0][:, :kvrq.packed_words(D, b)] for b in BITS}
    pq_c = torch.from_numpy(kvrq.pq_codebooks()).to(dev)
    legs = [("rq", b) for b in BITS] + [("tq", b) for b in BITS] + [("pq", 4)]

    def run_leg(leg, k=0):
        kind, b = leg
        st = torch.cuda.current_stream()  # the capture stream while a graph is recorded
        if kind == "rq":
            kvrq.rq_quantize_dequantize(xs[k], rot, cbs[b], b, codes=codes_all[k][:, :W[b]], norms=norms_all[k],
                                        xhat=xhats[k], stream=st)
        elif kind == "pq":
            kvrq.pq_quantize_dequantize(xs[k], pi, pq_c, codes=codes_all[k][:, :kvrq.PQ_WORDS], xhat=xhats[k],
                                        stream=st)
        else:
            kvrq.tq_quantize_dequantize_mse(xs[k], pi, cbs[b], b, codes=codes_all[k][:, :kvrq.packed_words(D, b)],
                                            norms=norms_all[k], xhat=xhats[k], stream=st)

    # ---------------------------------------------------------------- warm-up
    # clocks are sampled from the warm-up through the timed region and the 1 GiB leg
    clk = ClockSampler(local)
    clk.__enter__()
    time.sleep(0.3)
    for i in range(args.warmup):
        for leg in legs:
            for k in range(NSETS):
                run_leg(leg, k)
    torch.cuda.synchronize()
    kvrq.device_status()
    # Each leg's K launches of the timed region, step k on set k mod NSETS, are captured once into a CUDA
    # graph: a replay issues them back to back on the device, so neither the host cost of a call (binding,
    # tensor-map encoding) nor an event pair per launch enters the time of a launch.
    graphs = {}
    for leg in legs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for k in range(args.steps):
                run_leg(leg, k % NSETS)
        graphs[leg] = g
    for leg in legs:
        graphs[leg].replay()  # one untimed replay (the warm-up of the captured launches)
    torch.cuda.synchronize()
    kvrq.device_status()

    # ---------------------------------------------------------------- timed region
    ev = {}
    launches = 0
    barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for leg in legs:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        graphs[leg].replay()
        e.record(stream)
        ev[leg] = (s, e)
        launches += args.steps
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - t_wall
    kvrq.device_status()
    del graphs

    leg_ms = {leg: ranks_max(ev[leg][0].elapsed_time(ev[leg][1]) / args.steps) for leg in legs}
    step_ms = sum(leg_ms.values())
    head = ("rq", HEADLINE_BITS)
    head_ms = leg_ms[head]
    value = whole_job_rate(N_VEC, world, head_ms) / 1e6

    peak, peak_kind = measured_peaks()
    bpv = rq_bytes_per_vector(D, HEADLINE_BITS)
    achieved = bpv * N_VEC / (head_ms * 1e-3) / 1e9
    legs_out = {}
    for (kind, b), ms in leg_ms.items():
        bpv_leg = (rq_bytes_per_vector(D, b) if kind == "rq" else
                   pq_bytes_per_vector(D) if kind == "pq" else tq_bytes_per_vector(D, b))
        legs_out[leg_name((kind, b))] = {
            "ms": ms, "Mvec_s": N_VEC / (ms * 1e-3) / 1e6, "GB_s": bpv_leg * N_VEC / (ms * 1e-3) / 1e9}

    # every leg's codes for the boundary-tie count (rank 0 compares sampled rows with the oracle below)
    tie_rows = np.unique(np.concatenate([np.random.default_rng(1).choice(N_VEC, 1024, replace=False), [0, N_VEC - 1]]))
    tie_data = {}
    if rank == 0:
        idx = torch.as_tensor(tie_rows, device=dev)
        for leg in legs:
            run_leg(leg)
            kind, b = leg
            cw = (codes[b] if kind == "rq" else codes_all[0][:, :kvrq.PQ_WORDS] if kind == "pq" else tq_codes[b])[idx]
            tie_data[leg] = cw.cpu().numpy().astype(np.int64).astype(np.uint32)
        tie_x = x[idx].double().cpu().numpy()
        tie_params = (rot.double().cpu().numpy(), pi.double().cpu().numpy(),
                      dict({b: cbs[b].double().cpu().numpy() for b in BITS}, pq=pq_c.double().cpu().numpy()))

    # ---------------------------------------------------------------- end to end through the public API
    x_host = x.to("cpu").pin_memory()
    codes_h = torch.empty((N_VEC, W[HEADLINE_BITS]), dtype=torch.int32).pin_memory()
    norms_h = torch.empty(N_VEC, dtype=torch.float32).pin_memory()
    xhat_h = torch.empty_like(x_host).pin_memory()
    # the host-buffer call: chunks of 16,384 rows whose copy-in, kernel and copy-out overlap (smaller chunks pay
    # the fixed cost of each copy more often: 4,096-row chunks measured 0.82 ms a step, 16,384-row ones 0.62 ms)
    ws = torch.empty(kvrq.host_workspace_bytes(D, HEADLINE_BITS, torch.float16, 16384), dtype=torch.uint8, device=dev)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        kvrq.rq_quantize_dequantize_host(x_host, rot, cbs[HEADLINE_BITS], HEADLINE_BITS, ws, codes=codes_h,
                                         norms=norms_h, xhat=xhat_h, stream=stream)
        e.record(stream)
        e.synchronize()
        if i >= args.warmup:
            e2e_ms.append(s.elapsed_time(e))
    e2e = ranks_max(sum(e2e_ms) / len(e2e_ms))
    h2d = x_host.numel() * 2
    d2h = codes_h.numel() * 4 + norms_h.numel() * 4 + xhat_h.numel() * 2

    # ---------------------------------------------------------------- 1 GiB leg (HBM roofline, inputs >> L2)
    large = None
    if not args.no_large:
        del xs, xhats, codes_all, norms_all
        torch.cuda.empty_cache()
        xl = synth.lognormal(LARGE_ROWS, D, seed=2000 + rank, dtype=torch.float16, device=dev)
        cl = torch.empty((LARGE_ROWS, W[HEADLINE_BITS]), dtype=torch.int32, device=dev)
        nl = torch.empty(LARGE_ROWS, dtype=torch.float32, device=dev)
        ol = torch.empty_like(xl)
        for _ in range(3):
            kvrq.rq_quantize_dequantize(xl, rot, cbs[HEADLINE_BITS], HEADLINE_BITS, codes=cl, norms=nl, xhat=ol)
        torch.cuda.synchronize()
        ts = []
        for _ in range(10):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            kvrq.rq_quantize_dequantize(xl, rot, cbs[HEADLINE_BITS], HEADLINE_BITS, codes=cl, norms=nl, xhat=ol)
            e.record(stream)
            ts.append((s, e))
        torch.cuda.synchronize()
        lms = ranks_max(sum(s.elapsed_time(e) for s, e in ts) / len(ts))
        gbs = bpv * LARGE_ROWS / (lms * 1e-3) / 1e9
        large = {"rows": LARGE_ROWS, "ms": lms, "Mvec_s": LARGE_ROWS / (lms * 1e-3) / 1e6, "GB_s": gbs,
                 "frac_of_peak": gbs / peak, "frac_of_8TBs": gbs / 8000.0}
        del xl, cl, nl, ol
        torch.cuda.empty_cache()

    decode = None
    stack = None
    if not args.no_large:
        decode = {"b1": decode_step_c4(kvrq, synth, torch, dev, 1, max(args.steps, 5), args.warmup),
                  "b16": decode_step_c4(kvrq, synth, torch, dev, 16, 5, 3)}
        stack = kv_stack_c3(kvrq, synth, torch, dev, 5)
    clk.__exit__(None, None, None)
    cpu = None
    if rank == 0:
        rate, dt = cpu_oracle_rate(1024)
        n_s = int(min(N_VEC, max(1024, rate * 10)))  # about 10 s of work, at most the whole workload
        rate, dt = cpu_oracle_rate(n_s)
        cpu = {"value": rate / 1e6, "unit": "Mvec/s", "cores": 1, "kind": "oracle",
               "sample": "%d rows of the workload, RotorQuant 3-bit roundtrip, float64 numpy oracle (%.1f s)" % (
                   n_s, dt)}
        per_w = int(min(8192, max(256, rate * 4)))
        rate_all, workers = cpu_oracle_all_cores(per_w)
        cpu["all_cores"] = {"value": rate_all / 1e6, "unit": "Mvec/s", "cores": workers,
                            "sample": "%d rows per worker, one single-threaded oracle per core" % per_w}
        ties = {"rows": int(len(tie_rows)), "margin": 1e-5}
        for (kind, b), words in tie_data.items():
            cb_leg = tie_params[2]["pq"] if kind == "pq" else tie_params[2][b]
            near, diff, far = boundary_ties(kind, b, tie_x, words, tie_params[0], tie_params[1], cb_leg)
            ties[leg_name((kind, b))] = {"coords_within_margin": near, "codes_differing": diff,
                                          "codes_differing_off_boundary": far}

    if rank == 0:
        line = {
            "metric": "quantize+dequantize Mvec/s at d=128 3-bit", "value": value, "unit": "Mvec/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "65536 x d128 fp16 KV vectors (LogNormal(0,0.5) norms, 4 outlier channels x10), "
                                   "fused quantize+dequantize, RotorQuant and TurboQuant-mse b=2,3,4, PolarQuant "
                                   "4-2-2-2; headline RotorQuant b=3",
                       "n_vectors_per_gpu": N_VEC, "d": D, "io_dtype": "fp16",
                       "l2": "inputs larger than L2: step k runs on batch set k mod %d (%d independent batches, "
                             "%.0f MB with outputs); each leg's K launches replayed back to back from a CUDA graph"
                             % (NSETS, NSETS, NSETS * N_VEC * (4 * D + 4 * 17 + 4) / 1e6), "parallelism": "independent shard per GPU (weak scaling)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": recorded_traffic("rq_row_kernel<__half,3,RQ_QDQ>"),
                         "traffic_unit": "bytes per launch", "peak_kind": peak_kind,
                         "kernel": "rq_row_kernel<__half, 3, RQ_QDQ>", "bytes_per_vector": bpv},
            "legs": legs_out,
            "hbm_1gib": large,
            "decode_c4": decode,
            "kv_stack_c3": stack,
            "e2e": {"value": whole_job_rate(N_VEC, world, e2e) / 1e6, "unit": "Mvec/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms": e2e},
            "gpu_launches": launches,
            "build": build_identity(),
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "boundary_ties": ties if rank == 0 else None,
            "wall_s_timed_region": wall,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
