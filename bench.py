"""Benchmark of the PhaseQuant / multiplication-free complex product path on B200.

Default run (the contract line): one step is one pass of the whole path on the
LLaMA-2-7B-shaped Fairy2i block (seven real layers q,k,v,o 4096x4096,
gate,up 4096->11008, down 11008->4096; 2 residual stages; U and W):
  1. widely-linear conversion of the seven real layers        (7 launches)
  2. 2-stage PhaseQuant + pack of the 14 complex tensors      (2 stage + 2 reduction launches)
  3. L2 flush (256 MiB memset), then decode GEMV at B = 1     (1 launch, all 7 layers)
  4. prefill GEMM at M = 2048 tokens                          (7 launches)
Inputs are resident in HBM when the timed region starts; the metric value is
the decode GEMV's algorithmic HBM bytes over its CUDA-event time; the prefill
GEMM's equivalent TOP/s (8 M N K per stage and branch) is reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --case gemv|gemm|quant|convert ...   (single-kernel cases for ncu)

Multi-GPU (torchrun, one process per GPU): each rank runs an independent
replica of the block (weak scaling, no data-path collective); timing is the
max over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bit_complex_quantized_b200 as Q  # noqa: E402
from bit_complex_quantized_b200 import workloads as W  # noqa: E402

METRIC = "decode GEMV HBM GB/s (% of peak); prefill GEMM equiv TOP/s at M=2048"
WORKLOAD = "Fairy2i LLaMA-2-7B-shaped block (7 real layers -> 14 U/W tensors, 2 stages): conversion + " \
           "PhaseQuant + decode GEMV B=1 + prefill GEMM M=2048"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.1)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def source_hash(name):
    with open(os.path.join(ROOT, "bit_complex_quantized_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel_file, kernel, workload):
    """dram bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {})
    if e.get("source_sha256_16") != source_hash(kernel_file) or e.get("workload") != workload:
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- the block
class Block:
    """Device-resident state of the 7B-shaped block: real weights, planes, codes, activations."""

    def __init__(self, dev, gemm_M=2048, decode_B=1):
        self.cfg = W.config("llama7b")
        self.cfg4 = W.config("llama7b_prefill")
        self.T = self.cfg.T
        self.dev = dev
        self.R = []
        self.planes = []
        for i, spec in enumerate(self.cfg.layers):
            self.R.append(torch.from_numpy(W.real_weight(self.cfg, i)).to(dev))
            self.planes.append([torch.empty((spec.N, spec.K), dtype=torch.float32, device=dev) for _ in range(4)])
        self.codes = []
        for i, spec in enumerate(self.cfg.layers):
            for _ in range(2):
                self.codes.append((torch.empty((self.T, spec.N, spec.K // 4), dtype=torch.uint8, device=dev),
                                   torch.empty((self.T, 2), dtype=torch.float32, device=dev)))
        self.qt = []
        for i in range(len(self.cfg.layers)):
            p = self.planes[i]
            self.qt.append((p[0], p[1], *self.codes[2 * i]))
            self.qt.append((p[2], p[3], *self.codes[2 * i + 1]))
        self.ws = torch.empty(Q.ifq_quantize_workspace_bytes(self.qt, self.T), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.B, self.M = decode_B, gemm_M
        self.gemv_layers = self._layers(self.cfg, self.B)
        self.gemv_ws = torch.zeros(max(16, Q.ifq_gemv_workspace_bytes(self.gemv_layers, self.T, self.B)),
                                   dtype=torch.uint8, device=dev)
        self.gemm_layers = self._layers(self.cfg4, self.M)
        # the same conversion and quantization as one fused call per block (next-row measurement)
        self.wl_layers = []
        for i in range(len(self.cfg.layers)):
            p = self.planes[i]
            (cu, su), (cw, sw) = self.codes[2 * i], self.codes[2 * i + 1]
            self.wl_layers.append(dict(R=self.R[i], U_re=p[0], U_im=p[1], W_re=p[2], W_im=p[3],
                                       codes_u=cu, scales_u=su, codes_w=cw, scales_w=sw))
        self.wl_ws = torch.empty(Q.ifq_widely_linear_quantize_workspace_bytes(self.wl_layers, self.T),
                                 dtype=torch.uint8, device=dev)

    def _layers(self, cfg, rows):
        out = []
        for i, spec in enumerate(cfg.layers):
            xr, xi = W.activations(cfg, i, rows)
            (cu, su), (cw, sw) = self.codes[2 * i], self.codes[2 * i + 1]
            out.append(dict(codes_u=cu, scales_u=su, codes_w=cw, scales_w=sw, N=spec.N, K=spec.K,
                            x_re=xr.to(self.dev), x_im=xi.to(self.dev),
                            y_re=torch.empty((rows, spec.N), dtype=torch.float32, device=self.dev),
                            y_im=torch.empty((rows, spec.N), dtype=torch.float32, device=self.dev)))
        return out

    # algorithmic bytes / flops
    def convert_bytes(self):
        return sum(32 * l.N * l.K for l in self.cfg.layers)

    def quant_bytes(self):
        # pass t reads w (8 B) and t earlier code bytes (t/4 B... per stage), writes 1/4 B, per complex entry
        T = self.T
        per_entry = 8 * T + sum(t / 4 for t in range(T)) + T / 4
        return int(2 * sum(l.N * l.K for l in self.cfg.layers) * per_entry)

    def fused_bytes(self):
        # stage 1 fused with the conversion: R read (16 B), U and W written (16 B), two code bytes/4 written;
        # stage t >= 2: U and W read (16 B), 2 (t-1)/4 earlier code bytes read, 2/4 written
        T = self.T
        per_pos = 32.5 + sum(16 + 0.5 * (t - 1) + 0.5 for t in range(2, T + 1))
        return int(per_pos * sum(l.N * l.K for l in self.cfg.layers))

    def gemv_bytes(self, B):
        codes = W.code_bytes(self.cfg)
        return codes + sum(4 * B * l.K + 8 * B * l.N for l in self.cfg.layers) + 2 * len(self.cfg.layers) * 8 * self.T

    def gemm_flops(self):
        return sum(8 * self.M * l.N * l.K * 2 * self.T for l in self.cfg.layers)

    def step(self, ev=None):
        s = torch.cuda.current_stream()
        if ev:
            ev[0].record(s)
        for i in range(len(self.cfg.layers)):
            Q.ifq_widely_linear_from_real(self.R[i], *self.planes[i])
        if ev:
            ev[1].record(s)
        Q.ifq_quantize_pack(self.qt, self.T, self.ws, dev_status=self.status)
        if ev:
            ev[2].record(s)
        self.flush.zero_()
        if ev:
            ev[3].record(s)
        Q.ifq_gemv(self.gemv_layers, self.T, self.B, workspace=self.gemv_ws, dev_status=self.status)
        if ev:
            ev[4].record(s)
        Q.ifq_gemm(self.gemm_layers, self.T, self.M, dev_status=self.status)
        if ev:
            ev[5].record(s)

    def launches_per_step(self):
        """Our kernels per step (the L2-flush memset is not counted): conversion, quantizer (a stage
        kernel and a reduction kernel per stage), GEMV, GEMM."""
        gemv = 2  # activation digits (prep) + product
        gemm = 1  # one persistent launch over all layers
        return len(self.cfg.layers) + 2 * self.T + gemv + gemm


def oracle_sample_layers(rows_per_layer):
    """A row sample of the block for the fp64 oracle: codes from the C oracle's quantizer on the
    sampled rows (setup, untimed), and the block's activations."""
    import oracle as O
    from oracle import cref
    cfg = W.config("llama7b")
    rng = np.random.default_rng(123)
    layers = []
    for i, spec in enumerate(cfg.layers):
        rows = np.sort(rng.choice(spec.N, size=rows_per_layer, replace=False))
        R = W.real_weight(cfg, i)
        n = spec.N
        Rs = np.concatenate([R[rows], R[n + rows]], axis=0)
        del R
        ur, ui, wr, wi = O.widely_linear_planes_fp32(Rs)
        cu, su = cref.quantize_tensor(ur, ui, cfg.T)
        cw, sw = cref.quantize_tensor(wr, wi, cfg.T)
        xr, xi = W.activations(cfg, i, 1)
        layers.append((cu, su, cw, sw, W.bf16_to_f32_numpy(xr), W.bf16_to_f32_numpy(xi)))
    nbytes = sum(2 * cfg.T * rows_per_layer * l.K // 4 for l in cfg.layers)
    return layers, nbytes


def oracle_decode_time(layers, nbytes, rows_per_layer, seconds_budget):
    """Times the fp64 oracle's decode product on the sample for about `seconds_budget` (CPU)."""
    import oracle as O
    reps, t0 = 0, time.perf_counter()
    while True:
        for (cu, su, cw, sw, xr, xi) in layers:
            O.product(cu, su, cw, sw, xr, xi)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds_budget:
            break
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        cores = 1
    return {"value": nbytes * reps / el / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 NumPy oracle decode product, B=1, {rows_per_layer} sampled rows of each of the 7 "
                      f"layers, U+W, T=2 ({nbytes / 1e6:.2f} MB of codes per rep), {reps} reps in {el:.1f} s"}


def oracle_decode_sample(seconds_budget=12.0, rows_per_layer=256):
    layers, nbytes = oracle_sample_layers(rows_per_layer)
    return oracle_decode_time(layers, nbytes, rows_per_layer, seconds_budget)


def host_info():
    """BLAS vendor of NumPy and the CPU model of this host."""
    blas = None
    try:
        cfg = np.show_config(mode="dicts")
        b = cfg.get("Build Dependencies", {}).get("blas", {})
        blas = f"{b.get('name')} {b.get('version', '')}".strip()
    except Exception:  # noqa: BLE001
        pass
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"blas": blas, "cpu_model": model, "affinity_cores": len(os.sched_getaffinity(0))}


def _time_budget(fn, seconds):
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return reps, el


def oracle_steps(seconds_each=3.0, rows=128, gemm_rows=32, M=2048):
    """The fp64 oracle's other steps, each timed on a bounded row sample of the block's gate layer
    (real 11008 x 4096 -> complex 5504 x 2048): the widely-linear conversion, the T-stage quantization
    of U and W (NumPy, every stage over the sample) and the prefill product of M = 2048 tokens."""
    import oracle as O
    cfg = W.config("llama7b")
    spec = cfg.layers[4]
    R = W.real_weight(cfg, 4)
    rng = np.random.default_rng(7)
    sel = np.sort(rng.choice(spec.N, size=rows, replace=False))
    Rs = np.concatenate([R[sel], R[spec.N + sel]], axis=0)
    del R
    out = {}
    reps, el = _time_budget(lambda: O.widely_linear_planes_fp32(Rs), seconds_each)
    out["convert"] = {"GBps": 32 * rows * spec.K * reps / el / 1e9, "sample": f"{rows} complex rows of gate"}
    ur, ui, wr, wi = O.widely_linear_planes_fp32(Rs)
    per_entry = 8 * cfg.T + sum(t / 4 for t in range(cfg.T)) + cfg.T / 4
    reps, el = _time_budget(lambda: (O.quantize_tensor(ur, ui, cfg.T), O.quantize_tensor(wr, wi, cfg.T)),
                            seconds_each)
    out["quantize"] = {"GBps": 2 * rows * spec.K * per_entry * reps / el / 1e9,
                       "sample": f"U and W of {rows} rows of gate, T = {cfg.T}"}
    cu, su, _ = O.quantize_tensor(ur[:gemm_rows], ui[:gemm_rows], cfg.T)
    cw, sw, _ = O.quantize_tensor(wr[:gemm_rows], wi[:gemm_rows], cfg.T)
    xr, xi = W.activations(W.config("llama7b_prefill"), 4, M)
    xr, xi = W.bf16_to_f32_numpy(xr), W.bf16_to_f32_numpy(xi)
    reps, el = _time_budget(lambda: O.product(cu, su, cw, sw, xr, xi), seconds_each)
    out["prefill_product"] = {"TOPs_equiv": 8 * M * gemm_rows * spec.K * 2 * cfg.T * reps / el / 1e12,
                              "sample": f"{gemm_rows} output rows of gate, U+W, T = {cfg.T}, M = {M}"}
    return out


def near_boundary_counts(block):
    """Later-stage codes of the block's 14 tensors that differ from the oracle's rule applied to the
    residuals rebuilt from the GPU's own earlier codes and scales (the C restatement of one stage), with
    how many of those lie within 1e-6 of a decision boundary; the acceptance rule allows only those."""
    from oracle import cref
    names = [f"{spec.name}.{br}" for spec in block.cfg.layers for br in ("U", "W")]
    res = {}
    for name, (wr, wi, codes, scales) in zip(names, block.qt):
        w_re, w_im = wr.cpu().numpy(), wi.cpu().numpy()
        c = codes.cpu().numpy().reshape(block.T, -1)
        sc = scales.cpu().numpy()
        per_stage = []
        for t in range(block.T):
            want, _, near = cref.stage(w_re, w_im, t, c[:t], sc[:t], want_near=t > 0)
            diff = np.nonzero(c[t] != want)[0]
            total = near_ok = 0
            for q in diff:
                for e in range(4):
                    if ((c[t][q] >> (2 * e)) & 3) != ((want[q] >> (2 * e)) & 3):
                        total += 1
                        near_ok += int(near[4 * q + e]) if near is not None else 0
            per_stage.append({"stage": t + 1, "mismatches": total, "near_boundary": near_ok})
        res[name] = per_stage
    return res


# ---------------------------------------------------------------- decode at B = 16
def decode_batch(block, B, reps=20):
    """The block's decode product at batch B (B <= 2: the integer path; B >= 3: bf16 mma.sync), after
    an L2 flush, through the same grouped call; reported beside the step, not part of it."""
    layers = Q.LayerSet(block._layers(block.cfg, B))
    nws = Q.ifq_gemv_workspace_bytes(layers, block.T, B)
    ws = torch.zeros(max(16, nws), dtype=torch.uint8, device=block.dev)
    times = []
    for i in range(reps + 3):
        block.flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        Q.ifq_gemv(layers, block.T, B, workspace=ws, dev_status=block.status)
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            times.append(a.elapsed_time(b) * 1e-3)
    t = statistics.median(times)
    nbytes = block.gemv_bytes(B)
    gbs = nbytes / t / 1e9
    return {"B": B, "us": t * 1e6, "algorithmic_bytes": nbytes, "GBps": gbs,
            "frac_of_hbm": gbs / float(peaks()[0]["hbm_gbs"]),
            "path": "int8 mma.sync (bit planes)" if B <= 2 else "bf16 mma.sync (K segments)"}


def decode_b16(block, reps=20):
    return decode_batch(block, 16, reps)


# ---------------------------------------------------------------- decode on the other workloads
def workload_codes(name, dev, seed=11):
    """Device-resident codes and scales of a workload's layers, made by the library: the complex
    weights of layer256 / block1024 from the seeded generators, the real weights of llama70b drawn on
    the device with torch's seeded generator (same N(0, sigma) distribution; 3.4 GB of weights that the
    NumPy generator would take long to draw), converted and quantized with the workload's T stages."""
    cfg = W.config(name)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    out = []
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for i, spec in enumerate(cfg.layers):
        if spec.kind == "complex":
            wr, wi = W.complex_weights(cfg, i)
            ws = [(torch.from_numpy(wr).to(dev), torch.from_numpy(wi).to(dev))]
        else:
            R = spec.sigma * torch.randn(spec.real_shape, device=dev, generator=g)
            pl = [torch.empty((spec.N, spec.K), device=dev) for _ in range(4)]
            Q.ifq_widely_linear_from_real(R, *pl)
            del R
            ws = [(pl[0], pl[1]), (pl[2], pl[3])]
        qt = [(wr, wi, torch.empty((cfg.T, spec.N, spec.K // 4), dtype=torch.uint8, device=dev),
               torch.empty((cfg.T, 2), device=dev)) for wr, wi in ws]
        wsb = torch.empty(Q.ifq_quantize_workspace_bytes(qt, cfg.T), dtype=torch.uint8, device=dev)
        Q.ifq_quantize_pack(qt, cfg.T, wsb, dev_status=st)
        torch.cuda.synchronize()
        out.append([(c, s_) for _, _, c, s_ in qt])
        del ws, qt, wsb
    assert int(st.item()) == 0, f"device status set while quantizing {name}"
    return cfg, out


def decode_workload(name, dev, flush, batches, hot=False, reps=20):
    """The grouped decode call over all layers of a workload at each batch in `batches`, timed with
    CUDA events after an L2 flush (and, with hot=True, also back to back without one: the codes of the
    small workloads fit in L2).  Algorithmic bytes: codes + bf16 x + float32 y + scales."""
    cfg, codes = workload_codes(name, dev)
    res = []
    for B in batches:
        layers = []
        for i, spec in enumerate(cfg.layers):
            xr, xi = W.activations(cfg, i, B)
            cw = codes[i][1] if len(codes[i]) > 1 else (None, None)
            layers.append(dict(codes_u=codes[i][0][0], scales_u=codes[i][0][1], codes_w=cw[0], scales_w=cw[1],
                               N=spec.N, K=spec.K, x_re=xr.to(dev), x_im=xi.to(dev),
                               y_re=torch.empty((B, spec.N), device=dev), y_im=torch.empty((B, spec.N), device=dev)))
        ls = Q.LayerSet(layers)
        gws = torch.zeros(max(16, Q.ifq_gemv_workspace_bytes(ls, cfg.T, B)), dtype=torch.uint8, device=dev)
        nbytes = W.code_bytes(cfg) + sum(4 * B * l.K + 8 * B * l.N for l in cfg.layers) + \
            sum(8 * cfg.T * (2 if cfg.conj else 1) for _ in cfg.layers)
        entry = {"workload": name, "B": B, "algorithmic_bytes": int(nbytes)}
        for label, do_flush in (("flushed", True), ("l2_hot", False)) if hot else (("flushed", True),):
            times = []
            for k in range(reps + 3):
                if do_flush:
                    flush.zero_()
                else:
                    # keep the GPU busy while the host enqueues the call, so that the events time the
                    # kernels and not the host's launch work (the flush does this in the other mode)
                    torch.cuda._sleep(100000)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                Q.ifq_gemv(ls, cfg.T, B, workspace=gws)
                b.record()
                torch.cuda.synchronize()
                if k >= 3:
                    times.append(a.elapsed_time(b) * 1e-3)
            t = statistics.median(times)
            gbs = nbytes / t / 1e9
            entry[label] = {"us": t * 1e6, "GBps": gbs, "frac_of_hbm": gbs / float(peaks()[0]["hbm_gbs"])}
        res.append(entry)
        del ls, layers, gws
    del codes
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- dense comparator
def dequantize_block(block, reps=10):
    """bf16 dequantized weights of the block's 14 tensors (the forward weights of quantization-aware
    training), one ifq_dequantize call, CUDA events; reads T/4 B of codes and writes 4 B of bf16 per
    complex entry (910 MB of writes: larger than L2)."""
    ts = []
    for (cu, su), spec in zip(block.codes, [l for l in block.cfg.layers for _ in range(2)]):
        ts.append((cu, su, torch.empty((spec.N, spec.K), dtype=torch.int16, device=block.dev),
                   torch.empty((spec.N, spec.K), dtype=torch.int16, device=block.dev)))
    times = []
    for k in range(reps + 3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        Q.ifq_dequantize(ts, block.T)
        b.record()
        torch.cuda.synchronize()
        if k >= 3:
            times.append(a.elapsed_time(b) * 1e-3)
    t = statistics.median(times)
    entries = 2 * sum(l.N * l.K for l in block.cfg.layers)
    nbytes = entries * (block.T / 4 + 4)
    gbs = nbytes / t / 1e9
    del ts
    return {"us": t * 1e6, "algorithmic_bytes": int(nbytes), "GBps": gbs,
            "frac_of_hbm": gbs / float(peaks()[0]["hbm_gbs"])}


def decode_rope(block, reps=20):
    """The block's decode product at B = 1 with the complex rotary code applied in the epilogue of the
    q and k projections (layers 0 and 1; rot = e^{i pos omega_n}), after an L2 flush, through the C ABI.
    Reported beside the plain decode time: the rotation adds 8 bytes read per rotated output."""
    layers = [dict(d) for d in block.gemv_layers]
    pos = 1234
    for i in (0, 1):
        N = layers[i]["N"]
        omega = 10000.0 ** (-torch.arange(N, dtype=torch.float64) / N)
        layers[i]["rot_re"] = torch.cos(pos * omega).to(torch.float32).reshape(1, N).to(block.dev)
        layers[i]["rot_im"] = torch.sin(pos * omega).to(torch.float32).reshape(1, N).to(block.dev)
    ls = Q.LayerSet(layers)
    times = []
    for k in range(reps + 3):
        block.flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        Q.ifq_gemv(ls, block.T, 1, workspace=block.gemv_ws, dev_status=block.status)
        b.record()
        torch.cuda.synchronize()
        if k >= 3:
            times.append(a.elapsed_time(b) * 1e-3)
    assert int(block.status.item()) == 0, "device status set by the rotated decode"
    t = statistics.median(times)
    return {"us": t * 1e6, "rotated_layers": ["q", "k"], "GBps": block.gemv_bytes(1) / t / 1e9}


def fused_convert_quantize(block, reps=10):
    """Conversion fused with stage 1 of the quantizer (one call for the block's seven layers), timed
    with CUDA events; its inputs (3.2 GB of R) are far larger than L2.  Reported beside the two-pass
    conversion + quantizer times of the step, which compute the same outputs bit for bit."""
    times = []
    for k in range(reps + 3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        Q.ifq_widely_linear_quantize_pack(block.wl_layers, block.T, block.wl_ws, dev_status=block.status)
        b.record()
        torch.cuda.synchronize()
        if k >= 3:
            times.append(a.elapsed_time(b) * 1e-3)
    assert int(block.status.item()) == 0, "device status set by the fused call"
    t = statistics.median(times)
    hbm = float(peaks()[0]["hbm_gbs"])
    gbs = block.fused_bytes() / t / 1e9
    return {"us": t * 1e6, "algorithmic_bytes": block.fused_bytes(), "GBps": gbs, "frac_of_hbm": gbs / hbm,
            "launches": 2 * block.T, "bytes_per_complex_position": block.fused_bytes() /
            sum(l.N * l.K for l in block.cfg.layers)}


def _stacked_uw(U_re, U_im, W_re, W_im):
    """The unquantized widely-linear layer as two real bf16 matrices acting on [x_re; x_im]:
    U x -> [[U_re, -U_im], [U_im, U_re]] and W conj(x) -> [[W_re, W_im], [W_im, -W_re]]."""
    AU = torch.cat([torch.cat([U_re, -U_im], 1), torch.cat([U_im, U_re], 1)], 0).to(torch.bfloat16)
    AW = torch.cat([torch.cat([W_re, W_im], 1), torch.cat([W_im, -W_re], 1)], 0).to(torch.bfloat16)
    return AU, AW


def _timed(fn, flush, reps):
    times = []
    for i in range(reps + 3):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            times.append(a.elapsed_time(b) * 1e-3)
    return statistics.median(times)


def _dense_pair(Rs, UWs, dev, flush, M, reps):
    """cuBLAS bf16 (torch.matmul) times of the original real layers R and of the unquantized U, W:
    decode at B = 1 after an L2 flush, and prefill at M tokens when M > 0."""
    xs1 = [torch.randn((1, R.shape[1]), device=dev, dtype=torch.bfloat16) for R in Rs]
    out = {"decode_R_us": _timed(lambda: [torch.matmul(x, R.t()) for x, R in zip(xs1, Rs)], flush, reps) * 1e6,
           "decode_UW_us": _timed(lambda: [torch.addmm(torch.matmul(x, AU.t()), x, AW.t())
                                           for x, (AU, AW) in zip(xs1, UWs)], flush, reps) * 1e6,
           "R_weight_bytes": sum(R.numel() * 2 for R in Rs),
           "UW_weight_bytes": sum(AU.numel() * 2 + AW.numel() * 2 for AU, AW in UWs)}
    if M > 0:
        xsM = [torch.randn((M, R.shape[1]), device=dev, dtype=torch.bfloat16) for R in Rs]
        out["prefill_R_us"] = _timed(lambda: [torch.matmul(x, R.t()) for x, R in zip(xsM, Rs)], None, reps) * 1e6
        out["prefill_UW_us"] = _timed(lambda: [torch.addmm(torch.matmul(x, AU.t()), x, AW.t())
                                               for x, (AU, AW) in zip(xsM, UWs)], None, reps) * 1e6
        out["prefill_R_TFLOPs"] = sum(2 * M * R.shape[0] * R.shape[1] for R in Rs) / (out["prefill_R_us"] * 1e-6) / 1e12
        del xsM
    return out


def dense_comparator(block, reps=20):
    """Context, not the product: cuBLAS bf16 (torch.matmul) of the block's original real layers R and of
    the unquantized widely-linear U, W (two real-stacked products per layer, twice R's bytes), decode at
    B = 1 after an L2 flush and prefill at the block's M."""
    Rs = [R.to(torch.bfloat16) for R in block.R]
    UWs = [_stacked_uw(*pl) for pl in block.planes]
    out = _dense_pair(Rs, UWs, block.dev, block.flush, block.M, reps)
    out["what"] = ("cuBLAS bf16 of the 7B-shaped block: the original real layers (y = R x) and the unquantized "
                   "U, W (y = U x + W conj(x) as two real-stacked products); decode B = 1 after an L2 flush, "
                   "prefill M = %d" % block.M)
    del Rs, UWs
    torch.cuda.empty_cache()
    return out


def dense_comparator_70b(dev, flush, reps=10):
    """The same comparators on the 70B-shaped layer set (decode B = 1 only), on weights drawn on the
    device with torch's seeded generator."""
    cfg = W.config("llama70b")
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    Rs, UWs = [], []
    for spec in cfg.layers:
        R = spec.sigma * torch.randn(spec.real_shape, device=dev, generator=g)
        pl = [torch.empty((spec.N, spec.K), device=dev) for _ in range(4)]
        Q.ifq_widely_linear_from_real(R, *pl)
        Rs.append(R.to(torch.bfloat16))
        UWs.append(_stacked_uw(*pl))
        del R, pl
    out = _dense_pair(Rs, UWs, dev, flush, 0, reps)
    out["what"] = "cuBLAS bf16 of the 70B-shaped layer set: R and the unquantized U, W; decode B = 1 after an L2 flush"
    del Rs, UWs
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- e2e
def e2e_decode(block, steps, warmup):
    """Decode GEMV through the public API with host buffers, per step, as a prepared call
    (ifq_gemv_prepare once, ifq_gemv_run per step).  Two ways of moving the step's inputs and result:
    - "pinned host buffers": x and y live in pinned host memory, which the kernels address directly
      (unified addressing): the prep kernel reads x over PCIe and the product writes y over PCIe,
      inside the timed region, overlapping the rest of the work;
    - "explicit copies": one host -> device copy of every x (packed in one pinned buffer) before the
      call and one device -> host copy of every y after it.
    The first is the reported e2e value (the integer path reads x once, in its prep kernel); both give
    the same y bit for bit, which is checked here."""
    dev = block.dev
    xs = [t for L in block.gemv_layers for t in (L["x_re"], L["x_im"])]
    ys = [t for L in block.gemv_layers for t in (L["y_re"], L["y_im"])]

    def views(buf, like):
        out, off = [], 0
        for t in like:
            out.append(buf[off:off + t.numel()].view(t.shape))
            off += t.numel()
        return out

    def layers_on(xv, yv):
        out = []
        for i, L in enumerate(block.gemv_layers):
            d = dict(L)
            d["x_re"], d["x_im"], d["y_re"], d["y_im"] = xv[2 * i], xv[2 * i + 1], yv[2 * i], yv[2 * i + 1]
            out.append(d)
        return out

    def timed(one):
        times = []
        for i in range(warmup + steps):
            block.flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            one()
            b.record()
            torch.cuda.synchronize()
            if i >= warmup:
                times.append(a.elapsed_time(b) * 1e-3)
        return statistics.mean(times)

    x_src = torch.cat([t.flatten().cpu() for t in xs])
    ny = sum(t.numel() for t in ys)
    h2d = x_src.numel() * x_src.element_size()
    d2h = ny * 4
    # explicit copies
    x_dev = torch.empty(x_src.numel(), dtype=torch.bfloat16, device=dev)
    y_dev = torch.empty(ny, dtype=torch.float32, device=dev)
    plan_c = Q.GemvPlan(layers_on(views(x_dev, xs), views(y_dev, ys)), block.T, block.B, workspace=block.gemv_ws,
                        dev_status=block.status)
    x_host = x_src.clone().pin_memory()
    y_host = torch.empty(ny, dtype=torch.float32).pin_memory()

    def one_copies():
        x_dev.copy_(x_host, non_blocking=True)
        plan_c.run()
        y_host.copy_(y_dev, non_blocking=True)
    t_copies = timed(one_copies)

    def copies_only():
        x_dev.copy_(x_host, non_blocking=True)
        y_host.copy_(y_dev, non_blocking=True)
    t_copies_only = timed(copies_only)
    # pinned host buffers addressed by the kernels
    x_map = x_src.clone().pin_memory()
    y_map = torch.empty(ny, dtype=torch.float32).pin_memory()
    plan_m = Q.GemvPlan(layers_on(views(x_map, xs), views(y_map, ys)), block.T, block.B, workspace=block.gemv_ws,
                        dev_status=block.status)
    t_mapped = timed(plan_m.run)
    assert torch.equal(y_map.view(torch.int32), y_host.view(torch.int32)), "host-buffer decode differs from the copies"
    return {"value": block.gemv_bytes(block.B) / t_mapped / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": t_mapped * 1e3, "mode": "pinned host buffers read and written by the kernels",
            "explicit_copies": {"value": block.gemv_bytes(block.B) / t_copies / 1e9, "ms_per_step": t_copies * 1e3,
                                "copies_only_ms": t_copies_only * 1e3}}


def bench_config(ws, B, M, T):
    """The workload of a bench line; both arms report the same one."""
    return {"workload": WORKLOAD, "decode_batch": B, "prefill_M": M, "stages": T,
            "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
            "l2": "256 MiB L2 flush before the GEMV in every step; conversion/quantizer inputs (1.6 GB) exceed L2"}


def max_over_ranks(values, device):
    """Element-wise max of every rank's values (times in seconds); a no-op on one rank."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_rate(world, units_per_rank, seconds):
    """Whole-job throughput of `world` replicas that each processed `units_per_rank` in at most `seconds`."""
    return world * units_per_rank / seconds


# ---------------------------------------------------------------- main arm
def run_ours(args):
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    block = Block(dev)
    for _ in range(args.warmup):
        block.step()
    torch.cuda.synchronize()
    assert int(block.status.item()) == 0, "device status set during warm-up"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    clocks = Clocks(local)
    clocks.start()
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for k in range(args.steps):
        block.step(evs[k])
    end.record()
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    total_s = start.elapsed_time(end) * 1e-3
    per = {name: statistics.mean(e[a].elapsed_time(e[b]) * 1e-3 for e in evs)
           for name, a, b in (("convert", 0, 1), ("quant", 1, 2), ("gemv", 3, 4), ("gemm", 4, 5))}
    assert int(block.status.item()) == 0, "device status set during timing"

    # max over ranks of every time
    total_s, t_conv, t_quant, t_gemv, t_gemm = max_over_ranks(
        [total_s, per["convert"], per["quant"], per["gemv"], per["gemm"]], dev)

    pk, pk_src = peaks()
    hbm = float(pk["hbm_gbs"])
    tf_sus = float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
    # The GEMM is timed inside a step of a few ms with the SM clock at its maximum, so its denominator is
    # the burst bf16 figure (measured over a short loop), not the power-capped seconds-long one.
    tf_burst = float(pk["bf16_tflops"])
    gemv_bytes = block.gemv_bytes(block.B)
    gemv_gbs = gemv_bytes / t_gemv / 1e9
    gemm_tops = block.gemm_flops() / t_gemm / 1e12
    conv_gbs = block.convert_bytes() / t_conv / 1e9
    quant_gbs = block.quant_bytes() / t_quant / 1e9
    e2e = None
    if rank == 0:
        e2e = e2e_decode(block, steps=max(args.steps, 5), warmup=3)
    cpu = None
    if rank == 0 and ws == 1 and not args.skip_cpu_baseline:
        cpu = oracle_decode_sample(seconds_budget=args.cpu_seconds)
        cpu["steps"] = oracle_steps()
        cpu["host"] = host_info()
    nbc = near_boundary_counts(block) if rank == 0 and not args.skip_cpu_baseline else None
    others = None
    if rank == 0 and not args.skip_other_workloads:
        others = (decode_workload("layer256", dev, block.flush, [1], hot=True) +
                  decode_workload("block1024", dev, block.flush, [1, 8], hot=True) +
                  decode_workload("llama70b", dev, block.flush, [1, 8]))
    b16 = decode_b16(block) if rank == 0 else None
    batched = [decode_batch(block, B) for B in (2, 4, 8)] if rank == 0 else None
    fused = fused_convert_quantize(block) if rank == 0 else None
    rope = decode_rope(block) if rank == 0 else None
    dq = dequantize_block(block) if rank == 0 else None
    if rope is not None:
        rope["plain_decode_us"] = t_gemv * 1e6
    if fused is not None:
        fused["two_pass_us"] = (t_conv + t_quant) * 1e6
        fused["speedup_over_two_pass"] = (t_conv + t_quant) / (fused["us"] * 1e-6)
    if b16 is not None:
        b16["frac_of_hbm"] = b16["GBps"] / float(peaks()[0]["hbm_gbs"])
    dense = dense70 = None
    if rank == 0 and not args.skip_dense:
        dense = dense_comparator(block)
        dense["decode_quantized_us"] = t_gemv * 1e6
        dense["decode_ratio_quantized_to_R"] = t_gemv / (dense["decode_R_us"] * 1e-6)
        dense["decode_ratio_quantized_to_UW"] = t_gemv / (dense["decode_UW_us"] * 1e-6)
        dense["prefill_quantized_us"] = t_gemm * 1e6
        dense["prefill_ratio_quantized_to_R"] = t_gemm / (dense["prefill_R_us"] * 1e-6)
        dense["prefill_ratio_quantized_to_UW"] = t_gemm / (dense["prefill_UW_us"] * 1e-6)
        dense70 = dense_comparator_70b(dev, block.flush)
        if others:
            q70 = [e for e in others if e["workload"] == "llama70b" and e["B"] == 1]
            if q70:
                dense70["decode_quantized_us"] = q70[0]["flushed"]["us"]
                dense70["decode_ratio_quantized_to_R"] = q70[0]["flushed"]["us"] / dense70["decode_R_us"]
                dense70["decode_ratio_quantized_to_UW"] = q70[0]["flushed"]["us"] / dense70["decode_UW_us"]
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    kernels = {
        "gemv": {"bound": "hbm", "achieved": gemv_gbs, "peak": hbm, "unit": "GB/s", "frac": gemv_gbs / hbm,
                 "us": t_gemv * 1e6, "algorithmic_bytes": gemv_bytes,
                 "traffic": recorded_traffic("gemv_i8.cu", "gemv", "llama7b_b1")},
        "gemm": {"bound": "tensor", "achieved": gemm_tops, "peak": tf_burst, "unit": "TFLOP/s",
                 "frac": gemm_tops / tf_burst, "us": t_gemm * 1e6, "equiv_flops": block.gemm_flops(),
                 "traffic": recorded_traffic("gemm.cu", "gemm", "llama7b_prefill_m2048")},
        "quantize": {"bound": "hbm", "achieved": quant_gbs, "peak": hbm, "unit": "GB/s", "frac": quant_gbs / hbm,
                     "us": t_quant * 1e6, "algorithmic_bytes": block.quant_bytes()},
        "convert": {"bound": "hbm", "achieved": conv_gbs, "peak": hbm, "unit": "GB/s", "frac": conv_gbs / hbm,
                    "us": t_conv * 1e6, "algorithmic_bytes": block.convert_bytes()},
    }
    dominant = max(("gemv", "gemm", "quantize", "convert"), key=lambda k: kernels[k]["us"])
    rl = dict(kernels[dominant])
    line = {
        "metric": METRIC,
        "value": job_rate(ws, gemv_bytes, t_gemv) / 1e9,
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_s / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 activations x 2-bit codes, f32 accumulate; f64 scale reduction",
        "data": "synthetic: seeded N(0,0.02) real weights, N(0,1) bf16 activations",
        "config": bench_config(ws, block.B, block.M, block.T),
        "prefill_gemm": {"value": job_rate(ws, block.gemm_flops(), t_gemm) / 1e12, "unit": "TOP/s (equivalent dense, 8 M N K per stage and branch)",
                         "frac_of_burst_bf16": gemm_tops / tf_burst, "frac_of_sustained_bf16": gemm_tops / tf_sus},
        "roofline": {"kernel": dominant, "bound": rl["bound"], "achieved": rl["achieved"], "peak": rl["peak"],
                     "unit": rl["unit"], "frac": rl["frac"], "traffic": rl.get("traffic"),
                     "peak_source": f"{pk_src} ({'bf16_tflops' if rl['bound'] == 'tensor' else 'hbm_gbs'})"},
        "roofline_decode": {"kernel": "gemv", "bound": "hbm", "achieved": gemv_gbs, "peak": hbm, "unit": "GB/s",
                            "frac": gemv_gbs / hbm, "traffic": kernels["gemv"]["traffic"],
                            "peak_source": f"{pk_src} (hbm_gbs)"},
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "decode_b16": b16,
        "decode_batched": batched,
        "fused_convert_quantize": fused,
        "decode_rope": rope,
        "dequantize_bf16": dq,
        "dense_bf16_comparator": dense,
        "dense_bf16_comparator_llama70b": dense70,
        "decode_other_workloads": others,
        "near_boundary_mismatches": nbc,
        "gpu_launches": block.launches_per_step() * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line))


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    reps = []
    rows = 128
    layers, nbytes = oracle_sample_layers(rows)
    for i in range(args.warmup + args.steps):  # each step: a bounded sample of the block's decode product
        r = oracle_decode_time(layers, nbytes, rows, seconds_budget=min(5.0, 60.0 / max(1, args.steps)))
        if i >= args.warmup:
            reps.append(r)
    v = statistics.mean(r["value"] for r in reps)
    cpu = dict(reps[-1])
    cpu["value"] = v
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": bench_config(ws, 1, 2048, 2),
            "cpu_baseline": cpu,
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ---------------------------------------------------------------- single-kernel cases (ncu)
def run_case(args):
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    if args.case == "gemv":
        # 7B-shaped block (llama7b, 50.6 MB of codes) or 70B-shaped layer set (llama70b, 321 MB,
        # larger than L2), random codes: the kernel's work does not depend on code values.  The L2 is
        # flushed before every timed call.
        cfg = W.config(args.workload)
        layers = []
        for i, spec in enumerate(cfg.layers):
            def rnd(shape):
                return torch.randint(0, 256, shape, dtype=torch.uint8, device=dev, generator=g)
            sc = lambda: torch.full((cfg.T, 2), 0.01, dtype=torch.float32, device=dev)  # noqa: E731
            xr, xi = W.activations(cfg, i, args.batch)
            layers.append(dict(codes_u=rnd((cfg.T, spec.N, spec.K // 4)), scales_u=sc(),
                               codes_w=rnd((cfg.T, spec.N, spec.K // 4)), scales_w=sc(), N=spec.N, K=spec.K,
                               x_re=xr.to(dev), x_im=xi.to(dev),
                               y_re=torch.empty((args.batch, spec.N), device=dev),
                               y_im=torch.empty((args.batch, spec.N), device=dev)))
        nbytes = W.code_bytes(cfg)
        gws = torch.zeros(max(16, Q.ifq_gemv_workspace_bytes(layers, cfg.T, args.batch)), dtype=torch.uint8,
                          device=dev)

        def fn():
            Q.ifq_gemv(layers, cfg.T, args.batch, workspace=gws)
        label = f"gemv {args.workload} B={args.batch}"
    elif args.case == "gemm":
        cfg = W.config("llama7b_prefill")
        spec = cfg.layers[4]  # gate: N = 5504, K = 2048
        M = 2048

        def rnd(shape):
            return torch.randint(0, 256, shape, dtype=torch.uint8, device=dev, generator=g)
        xr, xi = W.activations(cfg, 4, M)
        L = dict(codes_u=rnd((2, spec.N, spec.K // 4)), scales_u=torch.full((2, 2), 0.01, device=dev),
                 codes_w=rnd((2, spec.N, spec.K // 4)), scales_w=torch.full((2, 2), 0.01, device=dev),
                 N=spec.N, K=spec.K, x_re=xr.to(dev), x_im=xi.to(dev),
                 y_re=torch.empty((M, spec.N), device=dev), y_im=torch.empty((M, spec.N), device=dev))
        nbytes = 8 * M * spec.N * spec.K * 4  # equiv flops

        def fn():
            Q.ifq_gemm([L], 2, M)
        label = "gemm llama7b gate M=2048"
    elif args.case == "quant":
        cfg = W.config("llama7b")
        spec = cfg.layers[4]
        ts = []
        for _ in range(2):
            wr = 0.02 * torch.randn((spec.N, spec.K), device=dev, generator=g)
            wi = 0.02 * torch.randn((spec.N, spec.K), device=dev, generator=g)
            ts.append((wr, wi, torch.empty((2, spec.N, spec.K // 4), dtype=torch.uint8, device=dev),
                       torch.empty((2, 2), device=dev)))
        wsb = torch.empty(Q.ifq_quantize_workspace_bytes(ts, 2), dtype=torch.uint8, device=dev)
        nbytes = 2 * spec.N * spec.K * 16.75

        def fn():
            Q.ifq_quantize_pack(ts, 2, wsb)
        label = "quantize llama7b gate U+W T=2"
    elif args.case == "wlq":
        cfg = W.config("llama7b")
        spec = cfg.layers[4]
        R = 0.02 * torch.randn(spec.real_shape, device=dev, generator=g)
        f = lambda: torch.empty((spec.N, spec.K), device=dev)  # noqa: E731
        cb = lambda: torch.empty((2, spec.N, spec.K // 4), dtype=torch.uint8, device=dev)  # noqa: E731
        wl = [dict(R=R, U_re=f(), U_im=f(), W_re=f(), W_im=f(), codes_u=cb(), scales_u=torch.empty((2, 2), device=dev),
                   codes_w=cb(), scales_w=torch.empty((2, 2), device=dev))]
        wsb = torch.empty(Q.ifq_widely_linear_quantize_workspace_bytes(wl, 2), dtype=torch.uint8, device=dev)
        nbytes = 49.5 * spec.N * spec.K

        def fn():
            Q.ifq_widely_linear_quantize_pack(wl, 2, wsb)
        label = "fused convert + quantize llama7b gate T=2"
    elif args.case == "dequant":
        cfg = W.config("llama7b")
        spec = cfg.layers[4]
        cb = torch.randint(0, 256, (2, spec.N, spec.K // 4), dtype=torch.uint8, device=dev, generator=g)
        sc = torch.full((2, 2), 0.01, device=dev)
        outp = [torch.empty((spec.N, spec.K), dtype=torch.int16, device=dev) for _ in range(2)]
        nbytes = spec.N * spec.K * (2 / 4 + 4)

        def fn():
            Q.ifq_dequantize([(cb, sc, outp[0], outp[1])], 2)
        label = "dequantize bf16 llama7b gate T=2"
    elif args.case == "convert":
        cfg = W.config("llama7b")
        spec = cfg.layers[4]
        R = 0.02 * torch.randn(spec.real_shape, device=dev, generator=g)
        planes = [torch.empty((spec.N, spec.K), device=dev) for _ in range(4)]
        nbytes = 32 * spec.N * spec.K

        def fn():
            Q.ifq_widely_linear_from_real(R, *planes)
        label = "convert llama7b gate"
    else:
        raise SystemExit("unknown case")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e-3)
    t = statistics.median(times)
    unit = "TOP/s" if args.case == "gemm" else "GB/s"
    print(json.dumps({"case": label, "median_us": t * 1e6, "min_us": min(times) * 1e6,
                      "rate": nbytes / t / (1e12 if args.case == "gemm" else 1e9), "unit": unit}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--case", choices=["gemv", "gemm", "quant", "convert", "wlq", "dequant"], default=None)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--workload", choices=["llama7b", "llama70b"], default="llama70b", help="layer set of --case gemv")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-dense", action="store_true", help="skip the cuBLAS bf16 dense comparator")
    ap.add_argument("--skip-other-workloads", action="store_true",
                    help="skip the decode timings of layer256, block1024 and llama70b")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.case:
        run_case(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
