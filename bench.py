"""Benchmark: MoE-FFN decode / verify tokens/s and achieved HBM GB/s on B200.

Workload (default): one full-size MoE layer (H=4096, I=2048, 256 routed experts
top-6 + 1 shared; routed gate/up ROCmFP2, down ROCmFP3, shared ROCmFP4, 2.3 GB
packed) in decode at q=1 over 1000 seeded tokens with Zipf(s=1.1) routing
bias.  A step is one pass of the whole hot path for one batch: router top-k +
softmax, expert grouping, fused dequant gate/up GEMV + SwiGLU, down GEMV and
weighted combine.  The same layer in speculative verify at q=4 is reported
beside it.  Weights are synthetic (seeded) and stay resident in HBM; 8 copies
of the layer are rotated so that every step reads its weights from DRAM
(inputs larger than L2).

Beside the headline the same JSON line carries (each skippable by a flag):
the q = 2, 3, 5 and uniform-routing sweep; the layer as a ROCmFPX MIX (a
format per expert chosen by routing heat) at q = 1 and 4; the standalone
quantised GEMV in each format at q = 1 and 4; the router projection + top-k;
the prefill grouped GEMM at T = 2048 and 8192; the 43-layer stack at q = 1
and 4 (98.7 GB of distinct layers resident); and the oracle timed on the
host cores on a bounded sample.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun) every rank runs an independent replica of the workload
(the path is one GPU's work; nothing is exchanged) and rank 0 prints one JSON
line with the whole-job throughput over the max-over-ranks device time.
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
sys.path.insert(0, ROOT)

METRIC = "MoE-FFN decode tokens/s & achieved HBM GB/s (% of ~8 TB/s) at q=1 and q=4"
H, I, E, K_TOP = 4096, 2048, 256, 6
ZIPF_S = 1.1
NTOK = 1000
COPIES = 8
SEED = 0
CSRC = os.path.join(ROOT, "block_quantized_moe_rocmfpx_b200", "csrc")
KERNEL_SOURCES = {
    "moe_decode": ("moe_decode.cu", "moe_decode.h", "rfx_tile.cuh", "rfx_device.cuh", "rfx_layout.h"),
    "prefill": ("prefill.cu", "prefill.h", "tc.cuh", "rfx_tile.cuh", "rfx_device.cuh", "rfx_layout.h"),
}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch from
# one ncu capture: (kernel, workload) -> (digest of the kernel's sources when
# it was captured, bytes, algorithmic bytes of that launch).  Reported scaled
# to the run's mean algorithmic bytes per launch (the traffic grows with the
# union of experts), and only while the sources still have that digest; after
# any change the key reads null until the kernel is captured again.
TRAFFIC = {
    ("moe_decode", "q1"): ("557fce27bf9ab819", 67_082_240 + 866_816, 66_872_368),
    ("moe_decode", "q4"): ("557fce27bf9ab819", 111_705_856 + 3_130_368, 111_513_792),
    # both pf_gemm launches of one T = 2048 step (gate/up + down), token batch 0
    ("prefill", "T2048"): ("ab522f207f7dd16d", 751_524_096 + 42_337_024 + 522_533_120 + 3_903_232, 1_070_858_240),
}


def source_digest(kernel: str) -> str:
    import hashlib
    h = hashlib.sha1()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic(kernel: str, workload: str, algo_bytes: float):
    ent = TRAFFIC.get((kernel, workload))
    if not ent or ent[0] != source_digest(kernel):
        return None
    return ent[1] * algo_bytes / ent[2]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--copies", type=int, default=COPIES, help="rotating layer copies (>= 8 keeps steps L2-cold)")
    ap.add_argument("--only-q1", action="store_true", help="skip the q=4 verify measurement")
    ap.add_argument("--stack-only", action="store_true", help="time only the 43-layer stack")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill grouped-GEMM measurement")
    ap.add_argument("--prefill-only", action="store_true", help="time only the prefill (T = 2048 and 8192)")
    ap.add_argument("--prefill-steps", type=int, default=20)
    ap.add_argument("--no-router-proj", action="store_true", help="skip the router projection measurement")
    ap.add_argument("--no-sweep", action="store_true", help="skip the q = 2, 3, 5 and uniform-routing decode sweep")
    ap.add_argument("--router-proj-only", action="store_true", help="time only the router projection + top-k")
    ap.add_argument("--no-stack", action="store_true", help="skip the 43-layer stack measurement")
    ap.add_argument("--no-mix", action="store_true", help="skip the ROCmFPX MIX (format per expert) measurement")
    ap.add_argument("--no-gemv", action="store_true", help="skip the standalone quantised GEMV measurement")
    return ap.parse_args()


def max_over_ranks(v: float, world: int, device) -> float:
    """The largest of every rank's value (device time of the timed region):
    the job is as slow as its slowest replica.  Every rank must call it."""
    if world == 1:
        return float(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, units_per_rank: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (each rank runs an independent replica of the same work)."""
    return world * units_per_rank / (ms_max / 1e3)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            P = json.load(f)
        return float(P["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ----------------------------------------------------------------- clocks ---

class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        import torch
        try:
            self.index = "GPU-" + str(torch.cuda.get_device_properties(index).uuid)
        except Exception:
            self.index = str(index)
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# ----------------------------------------------------------------- oracle ---

def cpu_baseline(n_tokens: int, q: int, budget_s: float = 20.0):
    """The fp64 oracle as it stands, on the host cores, on a bounded sample of
    the same workload (tokens of the same layer and routing): the router and
    the expert FFNs of each token column, until about ``budget_s`` seconds of
    oracle time.  Codes are regenerated outside the timed region (a small
    cache of recently used experts keeps host memory bounded)."""
    import collections
    import numpy as np
    import oracle
    import synth

    L = synth.logits(SEED, 0, 0, n_tokens * q, E, ZIPF_S)
    xb = synth.x_bf16(SEED, 0, n_tokens * q, H)
    idx, w = oracle.router_topk(L, K_TOP)
    mats = collections.OrderedDict()

    def get(kind, e, bits, r, c):
        key_ = (kind, e)
        if key_ in mats:
            mats.move_to_end(key_)
        else:
            s = synth.MatrixSpec(SEED, 0, kind, e, bits, r, c)
            mats[key_] = oracle.Mat(bits, s.codes(), s.scales())
            if len(mats) > 60:
                mats.popitem(last=False)
        return mats[key_]

    xf = synth.bf16_to_f64(xb)
    done, t_oracle = 0, 0.0
    for t in range(n_tokens * q):
        shared = tuple(get(k, 0, 4, r, c) for k, (r, c) in zip((3, 4, 5), ((I, H), (I, H), (H, I))))
        ex = [tuple(get(k, int(e), b, r, c) for k, b, (r, c) in zip((0, 1, 2), (2, 2, 3), ((I, H), (I, H), (H, I))))
              for e in idx[t]]
        t0 = time.perf_counter()
        oracle.router_topk(L[t:t + 1], K_TOP)
        oracle.moe_token(ex, w[t], shared, xf[t])
        t_oracle += time.perf_counter() - t0
        done += 1
        if t_oracle > budget_s:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": done / t_oracle, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} token columns of the q={q} workload (router + 6 routed experts + shared, fp64), "
                      f"{t_oracle:.1f} s of oracle time"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    base = cpu_baseline(max(args.steps, 20), 1, budget_s=max(10.0, min(60.0, 2.0 * args.steps)))
    line = {"impl": "reference", "metric": METRIC, "value": base["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / base["value"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "one full-size MoE layer decode q=1 (H=4096, I=2048, 256 experts top-6 + 1 shared, "
                                   "FP2 gate/up, FP3 down, FP4 shared), Zipf(1.1) routing", "global_batch": 1,
                       "seq_len": 1, "parallelism": "replicas"},
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- GPU ---

class Workload:
    """C rotating copies of one synthetic full-size layer plus seeded inputs."""

    def __init__(self, q: int, ntok: int, dev, copies: int = COPIES, zipf_s: float = ZIPF_S, mix=None):
        import torch
        import numpy as np
        import synth
        from synth.layers import SynthLayer
        self.q, self.dev = q, dev
        base = SynthLayer(SEED, 0, H, I, E, K_TOP, device=dev, mix=mix)
        self.base = base
        self.layers = [base.moe_layer(max_T=q)]
        self._keep = [base]
        self.copies = copies
        for c in range(1, copies):
            bufs = [b.clone() for b in base.bufs]
            sh = [b.clone() for b in base.shared]
            self._keep.append((bufs, sh))
            self.layers.append(base.moe_layer(max_T=q, bufs=bufs, shared=sh))
        torch.cuda.synchronize()
        self.ntok = ntok
        nb = ntok * q
        self.logits_h = synth.logits(SEED, 0, 0, nb, E, zipf_s)
        self.x_h = synth.x_bf16(SEED, 0, nb, H)
        self.logits = torch.from_numpy(self.logits_h).to(dev).view(ntok, q, E)
        self.x = torch.from_numpy(self.x_h).view(torch.bfloat16).to(dev).view(ntok, q, H)
        self.idx = torch.empty((ntok, q, K_TOP), dtype=torch.int32, device=dev)
        self.w = torch.empty((ntok, q, K_TOP), dtype=torch.float32, device=dev)
        self.y = torch.empty((copies, q, H), dtype=torch.float32, device=dev)

    def step(self, t: int, route: bool = True, ffn: bool = True):
        import block_quantized_moe_rocmfpx_b200 as rfx
        s = t % self.ntok
        if route:
            rfx.moe_router_topk(self.logits[s], K_TOP, self.idx[s], self.w[s])
        if ffn:
            self.layers[t % self.copies].forward(self.x[s], self.idx[s], self.w[s], self.y[t % self.copies])

    def algo_bytes(self, tokens) -> float:
        """Bytes one pass must move: packed blocks of the union of routed
        experts + the shared expert, plus activations in/out."""
        import numpy as np
        idx = self.idx.cpu().numpy()
        tot = 0.0
        for t in tokens:
            s = t % self.ntok
            tot += self.base.union_bytes(idx[s].ravel())
            tot += self.q * (2 * H + 8 * K_TOP + 4 * H + 4 * E)
        return tot


STACK_LAYERS = 43


def measure_stack(qs, steps: int, warmup: int, dev):
    """The 43-layer stack: distinct seeded full-size layers resident in HBM,
    each token step one moe_stack_forward call (one router launch for all
    layers, then one MoE FFN kernel per layer, each next layer applying the
    unit-RMS bf16 chaining while it stages its input), captured in one CUDA
    graph."""
    import time
    import numpy as np
    import torch
    import synth
    import block_quantized_moe_rocmfpx_b200 as rfx
    from synth.layers import SynthLayer
    t0 = time.time()
    layers = [SynthLayer(SEED, l, H, I, E, K_TOP, device=dev) for l in range(STACK_LAYERS)]
    gen_s = time.time() - t0
    out = {"layers": STACK_LAYERS, "resident_gb": sum(
        E * sum(l.strides) + sum(b.numel() for b in l.shared) for l in layers) / 1e9, "generate_s": gen_s}
    stream = torch.cuda.Stream(device=dev)
    for q in qs:
        mls = [l.moe_layer(max_T=q) for l in layers]
        ntok = 64
        logits_h = np.stack([np.stack([synth.logits(SEED, l, t * q, q, E, ZIPF_S) for l in range(STACK_LAYERS)])
                             for t in range(ntok)])                                  # [tok][L][q][E]
        x_h = np.stack([synth.x_bf16(SEED, t * q, q, H) for t in range(ntok)])       # [tok][q][H]
        logits = torch.from_numpy(logits_h).to(dev)
        x = torch.from_numpy(x_h).view(torch.bfloat16).to(dev)
        y = torch.empty((q, H), dtype=torch.float32, device=dev)
        ws = torch.empty(rfx.moe_stack_workspace_bytes(mls, q), dtype=torch.uint8, device=dev)
        rfx.rfx_ws_init(ws)
        # bytes one step must move: each layer's union of routed experts + shared + activations
        nbytes = 0.0
        for t in range(ntok):
            for l in range(STACK_LAYERS):
                idx_o = np.argsort(-logits_h[t, l], axis=-1, kind="stable")[:, :K_TOP]
                nbytes += layers[l].union_bytes(idx_o.ravel()) + q * (2 * H + 8 * K_TOP + 4 * H + 4 * E)
        per_step = nbytes / ntok
        with torch.cuda.stream(stream):
            def step(t):
                rfx.moe_stack_forward(mls, logits[t % ntok], x[t % ntok], y, ws, stream)
            for t in range(3):
                step(t)
            torch.cuda.synchronize()
            g = graph_of(step, steps, stream)
            gw = graph_of(step, max(3, warmup), stream)
            gw.replay()
            torch.cuda.synchronize()
            ms = time_graph(g, stream)
            del g, gw
        st = rfx_status_of(ws)
        peak, _ = peaks()
        gbs = per_step * steps / (ms / 1e3) / 1e9
        out[f"q{q}"] = {"value": q * steps / (ms / 1e3), "unit": "tokens/s", "ms_per_token_step": ms / steps,
                        "us_per_layer": ms / steps / STACK_LAYERS * 1e3, "achieved_gbs": gbs, "frac": gbs / peak,
                        "bytes_per_step": per_step, "launches_per_step": 1 + STACK_LAYERS, "steps": steps,
                        "device_status": st}
        del mls
    return out


PREFILL_TS = (2048, 8192)
PREFILL_BATCHES = 2


def measure_prefill(T: int, steps: int, warmup: int, dev, layer=None, exact=False):
    """Prefill of one full-size layer: T tokens, Zipf(1.1)-skewed top-6 routing,
    each step = router top-k + moe_ffn_prefill (grouping, gather, gate/up
    tcgen05 GEMM + SwiGLU, down tcgen05 GEMM + combine), captured in a graph.
    Two seeded token batches alternate (x is T x 8 KB; the touched experts'
    packed weights, about 1 GB, are larger than L2)."""
    import numpy as np
    import torch
    import synth
    import block_quantized_moe_rocmfpx_b200 as rfx
    from synth.layers import SynthLayer
    lay = layer if layer is not None else SynthLayer(SEED, 0, H, I, E, K_TOP, device=dev)
    ml = lay.moe_layer()
    nb = PREFILL_BATCHES
    logits_h = [synth.logits(SEED, 0, 100000 + b * T, T, E, ZIPF_S) for b in range(nb)]
    x_h = [synth.x_bf16(SEED, 100000 + b * T, T, H) for b in range(nb)]
    logits = [torch.from_numpy(a).to(dev) for a in logits_h]
    x = [torch.from_numpy(a).view(torch.bfloat16).to(dev) for a in x_h]
    idx = [torch.empty((T, K_TOP), dtype=torch.int32, device=dev) for _ in range(nb)]
    w = [torch.empty((T, K_TOP), dtype=torch.float32, device=dev) for _ in range(nb)]
    y = [torch.empty((T, H), dtype=torch.float32, device=dev) for _ in range(nb)]
    stream = torch.cuda.Stream(device=dev)

    def step(t):
        b = t % nb
        rfx.moe_router_topk(logits[b], K_TOP, idx[b], w[b], stream)
        ml.prefill(x[b], idx[b], w[b], y[b], stream, exact=exact)

    with torch.cuda.stream(stream):
        for t in range(3):
            step(t)
        torch.cuda.synchronize()
        gw = graph_of(step, max(3, warmup), stream)
        g = graph_of(step, steps, stream)
        gw.replay()
        torch.cuda.synchronize()
        ms = time_graph(g, stream)
        del g, gw
    st = ml.prefill_status()
    # algorithmic work: 2 flops per multiply-add of the real (unpadded) rows;
    # bytes: packed blocks of the touched experts + the shared expert, x and y
    flops = 2.0 * T * (K_TOP + 1) * 3 * H * I
    # the exact variant's tensor work: gate/up 2 MMAs per product, down 4
    tflops_work = flops * ((2 * 2 + 4) / 3.0 if exact else 1.0)
    nbytes = []
    for b in range(nb):
        top = np.argsort(-logits_h[b], axis=-1, kind="stable")[:, :K_TOP]
        nbytes.append(lay.union_bytes(top.ravel()) + T * (2 * H + 4 * H))
    per_step_bytes = sum(nbytes) / nb
    t_step = ms / steps / 1e3
    peak_tf, peak_gbs = peaks_tensor(), peaks()[0]
    t_min = max(tflops_work / (peak_tf * 1e12), per_step_bytes / (peak_gbs * 1e9))
    return {"T": T, "precision": "exact (bf16 hi/lo weights, h1 + h2)" if exact else "bf16 operands",
            "ms_per_step": ms / steps, "value": T / t_step, "unit": "tokens/s",
            "tflops": flops / t_step / 1e12, "flops_per_step": flops, "tensor_flops_per_step": tflops_work,
            "bytes_per_step": per_step_bytes,
            "roofline": {"bound": "tensor" if tflops_work / (peak_tf * 1e12) >= per_step_bytes / (peak_gbs * 1e9)
                         else "hbm", "peak_tflops": peak_tf, "peak_gbs": peak_gbs, "t_min_ms": t_min * 1e3,
                         "frac": t_min / t_step, "peak_kind": "bf16_tflops_sustained of measured",
                         "traffic": None if exact else traffic("prefill", f"T{T}", per_step_bytes)},
            "device_status": st, "steps": steps}


ROUTER_PROJ_COPIES = 80   # 80 x 2 MB of router weights rotate: every call reads them from DRAM
ROUTER_PROJ_TS = (1, 4, 2048)


def measure_router_proj(T: int, steps: int, warmup: int, dev):
    """Router projection + top-k (moe_router_project_topk: logits = W_router x +
    bias, bf16 W [256][4096], then top-6) for T token columns, captured in a
    graph; ROUTER_PROJ_COPIES weight copies rotate so that W is read from DRAM.
    Roofline (HBM): W + x + bias read, logits written, by the projection kernel."""
    import torch
    import synth
    import block_quantized_moe_rocmfpx_b200 as rfx
    nc = ROUTER_PROJ_COPIES
    W0 = torch.from_numpy(synth.router_weight_bf16(SEED, 0, E, H).view("int16")).to(dev)
    Ws = [W0] + [W0.clone() for _ in range(nc - 1)]
    b = torch.from_numpy(synth.router_bias_f32(SEED, 0, E, ZIPF_S)).to(dev)
    x = torch.from_numpy(synth.x_bf16(SEED, 300000, T, H).view("int16")).to(dev)
    lg = torch.empty((T, E), dtype=torch.float32, device=dev)
    idx = torch.empty((T, K_TOP), dtype=torch.int32, device=dev)
    w = torch.empty((T, K_TOP), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(t):
        rfx.moe_router_project_topk(Ws[t % nc], b, x, K_TOP, lg, idx, w, stream)

    with torch.cuda.stream(stream):
        for t in range(3):
            step(t)
        torch.cuda.synchronize()
        gw = graph_of(step, max(3, warmup), stream)
        g = graph_of(step, steps, stream)
        gw.replay()
        torch.cuda.synchronize()
        ms = time_graph(g, stream)
        del g, gw
    us = ms * 1e3 / steps
    nbytes = E * H * 2 + T * H * 2 + E * 4 + T * E * 4
    peak, peak_kind = peaks()
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"T": T, "us_per_call": us, "bytes_per_call": nbytes, "achieved_gbs": gbs,
            "roofline": {"bound": "hbm", "peak_gbs": peak, "frac": gbs / peak, "peak_kind": peak_kind,
                         "t_min_us": nbytes / (peak * 1e9) * 1e6},
            "launches_per_call": 1 if T <= 8 else 2, "steps": steps}


GEMV_N, GEMV_K = 131072, 4096   # one matrix larger than L2 in every format (168 to 285 MB packed)


def measure_gemv(fmt: int, q: int, steps: int, warmup: int, dev):
    """Standalone quantised GEMV (rfx_gemv_q): y[q][N] = W x for a packed
    N x K matrix in one format, q bf16 columns, captured in a graph.  W is an
    8192-row seeded slice packed once and repeated (the packed layout is
    row-group after row-group), larger than L2 as a whole.  Roofline (HBM):
    packed W + x read, y written."""
    import torch
    import synth
    import block_quantized_moe_rocmfpx_b200 as rfx
    N, K, R = GEMV_N, GEMV_K, 8192
    spec = synth.MatrixSpec(SEED, 0, 0, 0, fmt, R, K)
    sl = torch.from_numpy(rfx.rfx_pack(fmt, spec.codes(), spec.scales())).to(dev)
    W = torch.empty(sl.numel() * (N // R), dtype=torch.uint8, device=dev)
    for i in range(N // R):
        W[i * sl.numel():(i + 1) * sl.numel()].copy_(sl)
    x = torch.from_numpy(synth.x_bf16(SEED, 400000, q, K)).view(torch.bfloat16).to(dev)
    y = torch.empty((q, N), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(t):
        rfx.rfx_gemv_q(fmt, W, N, K, x, y, stream)

    with torch.cuda.stream(stream):
        for t in range(3):
            step(t)
        torch.cuda.synchronize()
        gw = graph_of(step, max(3, warmup), stream)
        g = graph_of(step, steps, stream)
        gw.replay()
        torch.cuda.synchronize()
        ms = time_graph(g, stream)
        del g, gw
    us = ms * 1e3 / steps
    nbytes = rfx.rfx_packed_bytes(fmt, N, K) + q * K * 2 + q * N * 4
    peak, peak_kind = peaks()
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"fmt": fmt, "q": q, "N": N, "K": K, "us_per_call": us, "bytes_per_call": nbytes, "achieved_gbs": gbs,
            "frac": gbs / peak, "peak_kind": peak_kind, "steps": steps}


def peaks_tensor() -> float:
    """Measured sustained dense bf16 TFLOP/s (a kernel timed inside a long step)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return 1400.0


def rfx_status_of(ws) -> int:
    import block_quantized_moe_rocmfpx_b200 as rfx
    return rfx.rfx_ws_status(ws)


def graph_of(fn, n, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for t in range(n):
            fn(t)
    return g


def time_graph(g, stream):
    """Device time of one replay: events recorded on the stream the graph is launched on."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def measure(q: int, steps: int, warmup: int, dev, rank, world, want_clocks: bool, want_e2e: bool, copies: int,
            zipf_s: float = ZIPF_S, mix=None):
    import torch
    import torch.distributed as dist
    wl = Workload(q, NTOK, dev, copies, zipf_s, mix)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for t in range(3):            # eager warm-up (kernel attributes, lazy loading)
            wl.step(t)
        torch.cuda.synchronize()
        off = warmup
        g_warm = graph_of(lambda t: wl.step(t), warmup, stream)
        g_main = graph_of(lambda t: wl.step(off + t), steps, stream)
        g_ffn = graph_of(lambda t: wl.step(off + t, route=False), steps, stream)
    # warm-up
    with torch.cuda.stream(stream):
        g_warm.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = None
    with (Clocks(torch.cuda.current_device()) if want_clocks else _Null()) as ck:
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = time_graph(g_main, stream)
        if world > 1:
            dist.barrier()
        clk = ck.summary() if want_clocks else None
    # dominant kernel alone (routing already in HBM from the timed pass)
    ms_ffn = time_graph(g_ffn, stream)
    status = max(ml.status() for ml in wl.layers[:1])
    abytes = wl.algo_bytes(range(off, off + steps))
    idx_all = wl.idx.cpu().numpy()
    union = sum(len(set(idx_all[(off + t) % wl.ntok].ravel().tolist())) for t in range(steps)) / steps
    res = {"ms": ms, "ms_ffn": ms_ffn, "bytes": abytes, "clocks": clk, "status": status, "union": union}
    if want_e2e:
        res["e2e"] = e2e(wl, steps, stream)
    del g_warm, g_main, g_ffn
    return res


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass

    def summary(self):
        return None


def e2e(wl, steps, stream):
    """Same workload through the C-ABI call with host buffers
    (moe_ffn_forward_host): per step, the token's x and router logits go
    host->device from pinned memory, the router and the MoE FFN run, and y comes
    back device->host, all enqueued by one call."""
    import torch
    import block_quantized_moe_rocmfpx_b200 as rfx
    q = wl.q
    n = min(steps, wl.ntok)
    xh = torch.from_numpy(wl.x_h).view(torch.bfloat16).view(wl.ntok, q, H).pin_memory()
    lh = torch.from_numpy(wl.logits_h).view(wl.ntok, q, E).pin_memory()
    yh = torch.empty((n, q, H), dtype=torch.float32).pin_memory()

    def one(t):
        wl.layers[t % wl.copies].forward_host(xh[t], lh[t], yh[t], stream)

    with torch.cuda.stream(stream):
        for t in range(5):
            one(t)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for t in range(n):
            one(t)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return {"value": n * q / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": q * (2 * H + 4 * E),
            "d2h_bytes_per_step": q * 4 * H, "steps": n}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import __graft_entry__
    if rank == 0 or world == 1:
        __graft_entry__.build()
    if world > 1:
        dist.barrier()
    if args.stack_only:
        st = measure_stack((1, 4), min(args.steps, 200), max(3, args.warmup), dev)
        peak, peak_kind = peaks()
        if rank == 0:
            print(json.dumps({"metric": "43-layer MoE-FFN stack decode tokens/s (FFN only)", "stack": st,
                              "peak_gbs": peak, "peak_kind": peak_kind}), flush=True)
        return
    if args.router_proj_only:
        rp = [measure_router_proj(T, min(args.steps, 400), max(3, args.warmup), dev) for T in ROUTER_PROJ_TS]
        if rank == 0:
            print(json.dumps({"metric": "router projection + top-k (W_router x + bias, top-6) us per call",
                              "router_projection": rp}), flush=True)
        return
    if args.prefill_only:
        pf = [measure_prefill(T, args.prefill_steps, max(3, args.warmup), dev) for T in PREFILL_TS]
        if rank == 0:
            print(json.dumps({"metric": "MoE-FFN prefill grouped GEMM tokens/s and TFLOP/s", "prefill": pf}),
                  flush=True)
        return
    r1 = measure(1, args.steps, max(3, args.warmup), dev, rank, world, True, not args.no_e2e, args.copies)
    r4 = r1 if args.only_q1 else measure(4, args.steps, max(3, args.warmup), dev, rank, world, False, False,
                                         args.copies)

    def reduce_max(v):
        return max_over_ranks(v, world, dev)

    ms1, ms4 = reduce_max(r1["ms"]), reduce_max(r4["ms"])
    ms1f, ms4f = reduce_max(r1["ms_ffn"]), reduce_max(r4["ms_ffn"])
    e2e_v = None
    if "e2e" in r1:
        e2e_ms = reduce_max(r1["e2e"]["steps"] / r1["e2e"]["value"] * 1e3)
        e2e_v = dict(r1["e2e"])
        e2e_v["value"] = world * r1["e2e"]["steps"] / (e2e_ms / 1e3)
    sweep = None
    if not args.no_sweep:
        # verify widths and routing modes beside the headline (Zipf q=1 / q=4): the
        # same layer, fewer steps; the kernel-only time and the measured union size
        peak_s, _ = peaks()
        sweep = []
        for q, zs in ((2, ZIPF_S), (3, ZIPF_S), (5, ZIPF_S), (1, 0.0), (4, 0.0)):
            n = min(args.steps, 200)
            r = measure(q, n, max(3, args.warmup), dev, rank, world, False, False, args.copies, zs)
            ms_f = reduce_max(r["ms_ffn"])
            gbs = r["bytes"] / (ms_f / 1e3) / 1e9
            sweep.append({"q": q, "routing": "zipf(1.1)" if zs > 0 else "uniform", "steps": n,
                          "kernel_us": ms_f * 1e3 / n, "tokens_per_s_step": world * q * n / (reduce_max(r["ms"]) / 1e3),
                          "achieved_gbs": gbs, "frac": gbs / peak_s, "union_experts": r["union"],
                          "algo_bytes_per_launch": r["bytes"] / n, "device_status": r["status"]})
    mix = None
    if not args.no_mix:
        # ROCmFPX MIX: the same layer with a format per expert chosen by routing heat
        from synth.layers import heat_mix
        peak_s, _ = peaks()
        hm = heat_mix(SEED, 0, E, ZIPF_S)
        mix = {"assignment": "hottest 1/8 of experts FP4/FP4, next 3/8 FP3/FP3, rest FP2/FP3 (gate-up/down); "
                             "shared FP4", "experts_per_format": {f"fp{f}": sum(1 for m in hm if m[0] == f)
                                                                 for f in (2, 3, 4)}}
        for q in (1, 4):
            n = min(args.steps, 200)
            r = measure(q, n, max(3, args.warmup), dev, rank, world, False, False, args.copies, ZIPF_S, hm)
            ms_f = reduce_max(r["ms_ffn"])
            gbs = r["bytes"] / (ms_f / 1e3) / 1e9
            mix[f"q{q}"] = {"tokens_per_s_step": world * q * n / (reduce_max(r["ms"]) / 1e3),
                            "kernel_us": ms_f * 1e3 / n, "achieved_gbs": gbs, "frac": gbs / peak_s,
                            "algo_bytes_per_launch": r["bytes"] / n, "bytes_per_token": r["bytes"] / n / q,
                            "union_experts": r["union"], "steps": n, "device_status": r["status"]}
    gemv = None
    if not args.no_gemv:
        gemv = [measure_gemv(f, q, min(args.steps, 200), max(3, args.warmup), dev) for f in (2, 3, 4) for q in (1, 4)]
    rp = None
    if not args.no_router_proj:
        rp = [measure_router_proj(T, min(args.steps, 400), max(3, args.warmup), dev) for T in ROUTER_PROJ_TS]
    pf = None
    if not args.no_prefill:
        pf = [measure_prefill(T, args.prefill_steps, max(3, args.warmup), dev) for T in PREFILL_TS]
        pf.append(measure_prefill(2048, args.prefill_steps, max(3, args.warmup), dev, exact=True))
    stack = None
    if not args.no_stack:
        import gc
        import torch
        gc.collect()
        torch.cuda.empty_cache()
        stack = measure_stack((1, 4), min(args.steps, 100), max(3, args.warmup), dev)
    if world > 1:
        dist.barrier()
    if rank == 0:
        peak, peak_kind = peaks()
        gbs1 = r1["bytes"] / (r1["ms_ffn"] / 1e3) / 1e9
        gbs4 = r4["bytes"] / (r4["ms_ffn"] / 1e3) / 1e9
        value = whole_job_value(world, args.steps, ms1)
        base = None if args.no_cpu_baseline else cpu_baseline(200, 1, budget_s=15.0)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms1 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "one full-size MoE layer decode q=1 (H=4096, I=2048, 256 experts top-6 + 1 shared, "
                                   "FP2 gate/up, FP3 down, FP4 shared; 2.30 GB packed), 1000 seeded tokens, "
                                   "Zipf(1.1) routing", "global_batch": world, "seq_len": 1,
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": f"inputs larger than L2: {args.copies} rotating copies of the layer",
                       "graph": "CUDA graph of all timed steps"},
            "roofline": {"bound": "hbm", "achieved": gbs1, "peak": peak, "unit": "GB/s", "frac": gbs1 / peak,
                         "traffic": traffic("moe_decode", "q1", r1["bytes"] / args.steps),
                         "kernel": "moe_decode_kernel",
                         "peak_kind": peak_kind, "algo_bytes_per_launch": r1["bytes"] / args.steps,
                         "kernel_us": r1["ms_ffn"] * 1e3 / args.steps,
                         "q4": {"achieved": gbs4, "frac": gbs4 / peak, "kernel_us": r4["ms_ffn"] * 1e3 / args.steps,
                                "algo_bytes_per_launch": r4["bytes"] / args.steps,
                                "traffic": traffic("moe_decode", "q4", r4["bytes"] / args.steps)}},
            "q4": {"value": world * 4 * args.steps / (ms4 / 1e3), "unit": "tokens/s", "ms_per_step": ms4 / args.steps,
                   "union_experts": r4["union"],
                   "achieved_gbs": gbs4, "frac": gbs4 / peak, "kernel_us": r4["ms_ffn"] * 1e3 / args.steps,
                   "algo_bytes_per_launch": r4["bytes"] / args.steps},
            "cpu_baseline": base,
            "e2e": e2e_v,
            "gpu_launches": 2 * args.steps,
            "clocks": r1["clocks"],
            "device_status": {"q1": r1["status"], "q4": r4["status"]},
            "prefill": pf,
            "router_projection": rp,
            "q_sweep": sweep,
            "mix": mix,
            "gemv": gemv,
            "stack": stack,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
