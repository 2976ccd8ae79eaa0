"""Benchmark of the OrbitQuant hot path on B200: one step = RPBH rotate +
Lloyd-Max quantize of the activations, then the codebook W4A4 GEMM with the
norm-rescale + bias epilogue, on the FLUX-like attention projection
(X[4608 x 3072] bf16, fused QKV W[9216 x 3072], block 128, W4A4).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The value is timed over K steps with events only at the ends of the region;
the per-kernel split behind the roofline fields comes from a second region of K
steps with events around each kernel (those events keep the two kernels from
overlapping, so that region runs slower; its step time is reported too).

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun, one rank per GPU): every
rank runs its own copy of the workload (the path is row-parallel with no
exchange), timing is the max over ranks, value is the whole-job throughput.
`--impl reference` times the CPU oracle (plain fp64 NumPy) on a bounded sample
of the same workload; it is the deliberately slow program the ratio divides by.
"""

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RPBH+Lloyd-Max act-quant GB/s (frac of HBM); codebook W4A4 linear TFLOP/s"
UNIT = "TFLOP/s"
WORKLOAD = dict(workload="flux_attention_qkv_projection", M=4608, K=3072, N=9216, block=128, bits_w=4, bits_a=4,
                seed=0, bias=True, out="bf16")
N_SETS = 4
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def algorithmic(M, K, N, ba, bw):
    """Per-launch algorithmic work: act-quant bytes (read bf16 X, write codes and
    fp32 norms) and GEMM flops 2MNK."""
    aq_bytes = M * K * 2 + M * K * ba / 8 + 4 * M
    gemm_flops = 2.0 * M * N * K
    return aq_bytes, gemm_flops


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def profiled_traffic(kernel_files, summary_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of that kernel (sha256 of its source files, concatenated
    in the order given, matching the summary's source_sha256), else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", summary_name)
    srcs = [os.path.join(ROOT, "calibration_free_rotated_b200", "csrc", f) for f in kernel_files]
    if not (os.path.exists(path) and all(os.path.exists(s) for s in srcs)):
        return None
    sha = hashlib.sha256(b"".join(open(s, "rb").read() for s in srcs)).hexdigest()
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip().strip("-* ").lower()] = v.strip().strip("`")
    if vals.get("source_sha256") != sha:
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _poll(self):
        nv = self._nv
        while True:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._started.set()
            if self._stop.wait(0.001):
                break

    def __enter__(self):
        if self._nv is not None:
            self._started = threading.Event()
            self._t = threading.Thread(target=self._poll, daemon=True)
            self._t.start()
            self._started.wait(1.0)  # polling before the timed work is enqueued
            self.samples.clear()
        return self

    def __exit__(self, *exc):
        if self._nv is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(values, world):
    """Max over ranks of a list of floats (identity when world == 1)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def whole_job_value(units_per_rank, world, max_seconds):
    return units_per_rank * world / max_seconds


# ---------------------------------------------------------------------------
# CPU oracle arm (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def oracle_sample(rows, W_state=None):
    """Times the oracle on `rows` activation rows of the workload: act-quant +
    fp64 linear against precomputed oracle weight codes (offline step, untimed)."""
    from calibration_free_rotated_b200 import inputs
    from oracle import codebook as ocb
    from oracle import linear as olin
    from oracle import quantize as oqz
    from oracle import rpbh as orpbh
    w = WORKLOAD
    M, K, N, h = w["M"], w["K"], w["N"], w["block"]
    if W_state is None:
        perm, signs = orpbh.draw_permutation_and_signs(w["seed"], K)
        cb = ocb.lloyd_max(K, 4)
        Wb = inputs.weights(2, inputs.T_W, N, K)
        cw, r16, _, _ = oqz.quantize_weight_rows(inputs.bf16_bits_to_f64(Wb), perm, signs, h, cb["centroids"])
        bias = inputs.bf16_bits_to_f64(inputs.bias(2, N))
        W_state = dict(perm=perm, signs=signs, cb=cb, cw=cw, r16=r16, bias=bias)
    X = inputs.bf16_bits_to_f64(inputs.activations(2, M, K, rows=(0, rows)))
    st = W_state
    t0 = time.perf_counter()
    ca, s, _ = oqz.quantize_rows(X, st["perm"], st["signs"], h, st["cb"]["centroids"])
    y = olin.linear_from_codes(ca, s, st["cw"], st["r16"], st["cb"]["centroids"], st["cb"]["centroids"], K,
                               bias=st["bias"])
    dt = time.perf_counter() - t0
    assert np.isfinite(y).all()
    return dt, W_state


def parity_report(oq, cb, bufs, w_norm, W_state, K, bias):
    """Parity of one bench set's outputs against the oracle on sampled rows.

    Codes: the kernel's codes of the sampled rows against the oracle's
    nearest-centroid codes; mismatches are counted with the entries whose t lies
    within 1e-5 of a decision boundary (the band the parity rule forgives).
    Norms: max relative error of s.  Linear: relative Frobenius error of the
    GEMM's fp32 output (one extra launch on the same codes) and of the bench's
    bf16 output against the oracle's fp64 layer on its own codes."""
    import torch
    from calibration_free_rotated_b200 import inputs
    from oracle import linear as olin
    from oracle import quantize as oqz
    w = WORKLOAD
    M, h = w["M"], w["block"]
    rows = np.unique(np.concatenate([np.linspace(0, M - 1, 64).astype(int), [M - 1]]))
    st = W_state
    X = inputs.bf16_bits_to_f64(inputs.activations(2, M, K)[rows])
    ca, s, T = oqz.quantize_rows(X, st["perm"], st["signs"], h, st["cb"]["centroids"])
    got = oqz.unpack_codes(bufs["codes"].cpu().numpy()[rows], 4, K)
    mism = got != ca
    band = oqz.boundary_distance(T, st["cb"]["boundaries"]) < 1e-5
    s_gpu = bufs["norms"].cpu().numpy()[rows].astype(np.float64)
    ref = olin.linear_from_codes(ca, s, st["cw"], st["r16"], st["cb"]["centroids"], st["cb"]["centroids"], K,
                                 bias=st["bias"])
    y32, _ = oq.linear_codes(K, cb, cb, bufs["codes"], bufs["norms"], bufs["wc"], w_norm, bias=bias)
    torch.cuda.synchronize()
    y32 = y32.double().cpu().numpy()[rows]
    y16 = bufs["Y"].double().cpu().numpy()[rows]
    rel = lambda y: float(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    return {"rows_sampled": int(len(rows)), "codes_checked": int(mism.size), "code_mismatches": int(mism.sum()),
            "in_band": int(band.sum()), "mismatches_outside_band": int((mism & ~band).sum()), "band": 1e-5,
            "norm_max_rel": float(np.max(np.abs(s_gpu - s) / np.maximum(s, 1e-300))),
            "rel_fro_f32": rel(y32), "rel_fro_bf16_out": rel(y16), "tol": 2e-3,
            "weights": "oracle-quantized weights for the reference; the GPU's own weight codes for the GEMM"}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count()


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = WORKLOAD
    rows = 256
    _, flops = algorithmic(rows, w["K"], w["N"], w["bits_a"], w["bits_w"])
    dt, st = oracle_sample(rows)
    for _ in range(max(0, args.warmup - 1)):
        oracle_sample(rows, st)
    times = [oracle_sample(rows, st)[0] for _ in range(args.steps)]
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = f"{rows} of {w['M']} activation rows per step (act-quant + fp64 linear vs all {w['N']} outputs)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": dict(w, l2="n/a (CPU)", sample_rows=rows),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import inputs
    from calibration_free_rotated_b200 import orbitquant as oq

    w = WORKLOAD
    M, K, N, h = w["M"], w["K"], w["N"], w["block"]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    r = oq.Rpbh(w["seed"], K, h)
    cb = oq.Codebook(K, 4)

    def dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    X0 = dev_bf16(inputs.activations(2, M, K))
    W0 = dev_bf16(inputs.weights(2, inputs.T_W, N, K))
    bias = dev_bf16(inputs.bias(2, N))
    # offline weight quantization (not part of the step)
    wc0, wn = oq.quantize_weight(r, cb, W0)
    del W0
    sets = []
    for i in range(N_SETS):
        sets.append(dict(
            X=X0.clone(), wc=wc0.clone(),
            codes=torch.empty((M, K * 4 // 8), dtype=torch.uint8, device=dev),
            norms=torch.empty((M,), dtype=torch.float32, device=dev),
            Y=torch.empty((M, N), dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()

    def step(i, ev=None):
        s = sets[i % N_SETS]
        if ev is not None:
            ev[0].record(stream)
        oq.quantize_act(r, cb, s["X"], s["codes"], s["norms"], stream=stream)
        if ev is not None:
            ev[1].record(stream)
        oq.linear_codes(K, cb, cb, s["codes"], s["norms"], s["wc"], wn, bias=bias, out_bf16=s["Y"],
                        want_f32=False, want_bf16=True, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    oq.device_status()

    # Two timed regions of K steps each.  (1) The value: events only at its two
    # ends, so consecutive kernels stay adjacent in the stream (a user's layer
    # sequence; programmatic dependent launch overlaps them).  (2) The kernel
    # split for the roofline: an event before, between and after the two
    # kernels of every step (which serialises them).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start2, end2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(i)
        end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        start2.record(stream)
        for i in range(args.steps):
            step(i, evs[i])
        end2.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    oq.device_status()
    total_s = start.elapsed_time(end) / 1e3
    split_s = start2.elapsed_time(end2) / 1e3
    k1 = [e[0].elapsed_time(e[1]) / 1e3 for e in evs]
    k2 = [e[1].elapsed_time(e[2]) / 1e3 for e in evs]
    total_s, split_s, k1_avg, k2_avg = reduce_max([total_s, split_s, sum(k1) / len(k1), sum(k2) / len(k2)], world)
    pct = lambda v: {q: 1e3 * sorted(v)[round(f * (len(v) - 1))] for q, f in (("p10", 0.1), ("median", 0.5), ("p90", 0.9))}
    k1_pct, k2_pct = pct(k1), pct(k2)  # this rank's spread

    aq_bytes, flops = algorithmic(M, K, N, 4, 4)
    value = whole_job_value(flops * args.steps, world, total_s) / 1e12

    # end to end through the public oq_linear call with host buffers: every step
    # uploads its X from pinned host memory and reads its Y back.  Steps are
    # pipelined the way a caller would: upload of step i+1 and download of step
    # i-1 run on their own copy streams while step i computes (two device
    # buffer sets; events order each step's copy -> compute -> copy).
    n_e2e = 2
    Xh = [torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True) for _ in range(n_e2e)]
    Yh = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(n_e2e)]
    for xh in Xh:
        xh.copy_(X0.cpu())
    ws = [torch.empty((oq.workspace_bytes(M, K, 4),), dtype=torch.uint8, device=dev) for _ in range(n_e2e)]
    Xd = [torch.empty_like(X0) for _ in range(n_e2e)]
    Yd = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(n_e2e)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n_e2e)]
    ev_done = [torch.cuda.Event() for _ in range(n_e2e)]
    ev_out = [torch.cuda.Event() for _ in range(n_e2e)]
    for e in ev_out:
        e.record(s_out)

    def e2e_step(i):
        b = i % n_e2e
        s_in.wait_event(ev_done[b])  # device X buffer b is free once step i-2 has computed
        with torch.cuda.stream(s_in):
            Xd[b].copy_(Xh[b], non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])  # Y buffer b has been read back (step i-2)
        oq.linear(r, cb, cb, Xd[b], wc0, wn, bias=bias, out_bf16=Yd[b], want_f32=False, want_bf16=True,
                  workspace=ws[b], stream=stream)
        ev_done[b].record(stream)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            Yh[b].copy_(Yd[b], non_blocking=True)
        ev_out[b].record(s_out)

    for e in ev_done:
        e.record(stream)
    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)  # the first upload starts the timed region
    for i in range(args.steps):
        e2e_step(i)
    e1.record(s_out)  # the last download ends it
    torch.cuda.synchronize()
    e2e_s = reduce_max([e0.elapsed_time(e1) / 1e3], world)[0]
    oq.device_status()
    e2e_value = whole_job_value(flops * args.steps, world, e2e_s) / 1e12

    peaks, peak_kind = load_peaks()
    gemm_tflops = flops / k2_avg / 1e12
    aq_gbs = aq_bytes / k1_avg / 1e9
    gemm_traffic = profiled_traffic(["oq_cbgemm.cu"], "cbgemm_flux_qkv_w4a4.md")
    aq_traffic = profiled_traffic(["oq_rotq.cuh", "oq_rotq.cu"], "rotq_flux_qkv_act_w4.md")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16 (tensor operands, f32 accumulate; f32 rotate)",
        "data": "synthetic",
        "config": dict(w, parallelism=f"replicated weights, rows per rank (dp{world})",
                       l2=f"{N_SETS} rotating input/weight/output sets (~{N_SETS * 127} MB) > 126 MB L2"),
        "roofline": {"bound": "tensor", "kernel": "cbgemm_kernel", "achieved": gemm_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": gemm_tflops / peaks["bf16_tflops"],
                     "traffic": gemm_traffic, "peak_source": f"{peak_kind} bf16 burst (f16 same rate)",
                     "algorithmic_per_launch": flops},
        "roofline_act_quant": {"bound": "hbm", "kernel": "rotq_kernel", "achieved": aq_gbs,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": aq_gbs / peaks["hbm_gbs"],
                               "traffic": aq_traffic, "peak_source": f"{peak_kind} copy bandwidth",
                               "algorithmic_per_launch": aq_bytes},
        "kernel_ms": {"rotq_kernel": 1e3 * k1_avg, "cbgemm_kernel": 1e3 * k2_avg,
                      "rotq_kernel_spread": k1_pct, "cbgemm_kernel_spread": k2_pct,
                      "region": "a second timed region of K steps with an event before, between and after the two "
                                "kernels of every step (means, max over ranks; spreads of rank 0's K steps)",
                      "ms_per_step_with_kernel_events": 1e3 * split_s / args.steps},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2},
        "gpu_launches": 2 * args.steps,
        "timing": "value: K steps between two events (kernels adjacent in the stream); kernel_ms: a second region of "
                  "K steps with per-kernel events",
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the host-side oracle leg: the timed CPU baseline, and (untimed) the
        # parity of this run's own outputs -- sampled rows of set 0 (codes,
        # norms and Y from the timed steps) against the oracle, with the
        # boundary ties counted
        rows = 2048
        _, st = oracle_sample(8)
        if not args.no_parity:
            line["parity"] = parity_report(oq, cb, sets[0], wn, st, K, bias)
        dt, _ = oracle_sample(rows, st)
        _, sflops = algorithmic(rows, K, N, 4, 4)
        line["cpu_baseline"] = {"value": sflops / dt / 1e12, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"{rows} of {M} activation rows (act-quant + fp64 linear vs all {N} "
                                          "outputs); weights quantized beforehand, untimed"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_profile_case(args):
    """Launches one kernel on a given shape, for ncu captures (prints a short JSON,
    not the contract line).  Data: device-side random bf16 rows / random codes."""
    import torch
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant as oq
    torch.manual_seed(0)
    M, d, N = args.rows, args.d, args.n
    if args.profile == "rotq":
        r = oq.Rpbh(0, d, args.block, rounds=args.rounds)
        cb = oq.Codebook(d, args.bits_a)
        X = torch.randn(M, d, device="cuda").to(torch.bfloat16)
        codes, norms = oq.quantize_act(r, cb, X)
        run = lambda: oq.quantize_act(r, cb, X, codes, norms)
    elif args.profile == "flatness":
        X = torch.randn(M, d, device="cuda").to(torch.bfloat16)
        r3, ri, bm = oq.row_flatness(X)
        run = lambda: oq.row_flatness(X, r3, ri, bm)
    else:
        cba, cbw = oq.Codebook(d, args.bits_a), oq.Codebook(d, args.bits_w)
        a = torch.randint(0, 256, (M, d * args.bits_a // 8), dtype=torch.uint8, device="cuda")
        w = torch.randint(0, 256, (N, d * args.bits_w // 8), dtype=torch.uint8, device="cuda")
        an = torch.rand(M, device="cuda")
        wn = torch.rand(N, device="cuda").to(torch.bfloat16)
        y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
        run = lambda: oq.linear_codes(d, cba, cbw, a, an, w, wn, epilogue=args.epilogue, out_bf16=y, want_f32=False,
                                      want_bf16=True)
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):  # back to back: inputs smaller than L2 stay cached
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    oq.device_status()
    ms = statistics.median(times) if times else float("nan")
    out = {"profile": args.profile, "rows": M, "d": d, "n": N, "launches": args.warmup + args.steps,
           "median_ms": ms}
    if args.profile == "rotq":
        out["GB/s"] = algorithmic(M, d, N, args.bits_a, args.bits_w)[0] / ms / 1e6
    elif args.profile == "flatness":
        out["GB/s"] = (2.0 * M * d + 8.0 * M + 8) / ms / 1e6
    else:
        out["TFLOP/s"] = algorithmic(M, d, N, args.bits_a, args.bits_w)[1] / ms / 1e9
    print(json.dumps(out))
    return 0


def run_ablation(args):
    """Rotation ablation ([OQ] "Rotation Ablation (Table 3)", latency column):
    times oq_quantize_act (4-bit) under RPBH, Block-RHT (no permutation) and Full
    RHT (d's largest power-of-two block) on N(0,1) bf16 rows, and the composed
    RPBH of 2 and 3 rounds ([RHT] Methodology).  L2 is flushed
    (L2Flush: a 256 MB write, then a 256 MB read) before every timed launch;
    CUDA events bracket the launch alone.  Prints one JSON line per (shape, rotation); not the contract line."""
    import torch
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant as oq
    peaks, src = load_peaks()
    torch.manual_seed(0)
    flush = L2Flush()
    d = args.d
    for M in (args.rows, 32768):
        X = torch.randn(M, d, device="cuda").to(torch.bfloat16)
        codes = torch.empty(M, d // 2, dtype=torch.uint8, device="cuda")
        norms = torch.empty(M, dtype=torch.float32, device="cuda")
        cb = oq.Codebook(d, 4)
        for kind, block, rounds in (("rpbh", args.block, 1), ("block_rht", args.block, 1), ("full_rht", 0, 1),
                                    ("rpbh", args.block, 2), ("rpbh", args.block, 3)):
            r = oq.Rpbh(0, d, block, kind=kind, rounds=rounds)
            for _ in range(args.warmup):
                oq.quantize_act(r, cb, X, codes, norms)
            times = []
            for _ in range(args.steps):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                oq.quantize_act(r, cb, X, codes, norms)
                e1.record()
                e1.synchronize()
                times.append(e0.elapsed_time(e1))
            oq.device_status()
            ms = statistics.median(times)
            gbs = algorithmic(M, d, 1, 4, 4)[0] / ms / 1e6
            print(json.dumps({"ablation": "rotation", "kind": kind, "rounds": rounds, "block": r.block, "rows": M,
                              "d": d, "bits": 4,
                              "median_us": 1e3 * ms, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                              "peak_source": src}), flush=True)
    return 0


def run_ablation_steps(args):
    """Back-to-back steps of the bench workload (act-quant + GEMM, bf16 out) with
    CUDA events only at the two ends of the timed region, so that consecutive
    kernels stay adjacent in the stream and programmatic dependent launch can
    overlap them (the contract line's per-kernel events serialise them).  Run it
    once as is and once with OQ_NO_PDL=1 to compare.  One JSON line."""
    import torch
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import inputs
    from calibration_free_rotated_b200 import orbitquant as oq
    w = WORKLOAD
    M, K, N, h = w["M"], w["K"], w["N"], w["block"]
    dev = torch.device("cuda")
    bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)
    r, cb = oq.Rpbh(w["seed"], K, h), oq.Codebook(K, 4)
    X0 = bf(inputs.activations(2, M, K))
    wc0, wn = oq.quantize_weight(r, cb, bf(inputs.weights(2, inputs.T_W, N, K)))
    bias = bf(inputs.bias(2, N))
    sets = [dict(X=X0.clone(), wc=wc0.clone(), codes=torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                 norms=torch.empty((M,), device=dev), Y=torch.empty((M, N), dtype=torch.bfloat16, device=dev))
            for _ in range(N_SETS)]
    stream = torch.cuda.current_stream()

    def step(i):
        s = sets[i % N_SETS]
        oq.quantize_act(r, cb, s["X"], s["codes"], s["norms"], stream=stream)
        oq.linear_codes(K, cb, cb, s["codes"], s["norms"], s["wc"], wn, bias=bias, out_bf16=s["Y"], want_f32=False,
                        want_bf16=True, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    oq.device_status()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"ablation": "steps", "pdl": os.environ.get("OQ_NO_PDL", "0") != "1", "ms_per_step": ms,
                      "TFLOP/s": 2.0 * M * N * K / ms / 1e9, "steps": args.steps}), flush=True)
    return 0


class L2Flush:
    """Leaves L2 cold and clean before a timed launch: a 256 MB write (the
    flush), then a 256 MB read of another buffer, which evicts the written
    lines, so their write-back to HBM happens here and not inside the timed
    window (a write alone leaves up to the whole L2 dirty, and an HBM-bound
    kernel timed after it shares the bus with that write-back)."""

    def __init__(self, device="cuda"):
        import torch
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.clean = torch.ones(64 << 20, dtype=torch.float32, device=device)

    def __call__(self):
        self.buf.zero_()
        self.clean.sum()


def _flush_and_time(fn, flush, steps, warmup):
    """Median CUDA-event time (ms) of fn() with an L2 flush (L2Flush) before each call."""
    import torch
    for _ in range(warmup):
        fn()
    times = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def _flush_and_time_many(fns, flush, steps, warmup):
    """Median CUDA-event times (ms) of several launches, each timed alone after
    an L2 flush, taken round-robin (one of each per repetition) so that a clock
    change during the run affects them alike."""
    import torch
    for fn in fns:
        for _ in range(warmup):
            fn()
    times = [[] for _ in fns]
    for _ in range(steps):
        for i, fn in enumerate(fns):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            times[i].append(e0.elapsed_time(e1))
    return [statistics.median(t) for t in times]


def oracle_workload_sample(workload, rows):
    """The oracle on `rows` tokens of a two-layer workload or the W3A3
    projection, timed on the host cores (the cpu_baseline of the workload
    lines).  Weights are quantized beforehand, untimed; the timed part is what
    the GPU times: act-quant, linear (+ GELU, bf16 rounding of the hidden
    layer, act-quant, linear).  Returns (seconds, flops of the sample)."""
    from calibration_free_rotated_b200 import inputs
    from oracle import codebook as ocb
    from oracle import linear as olin
    from oracle import quantize as oqz
    from oracle import rpbh as orpbh
    h = 128
    f64 = inputs.bf16_bits_to_f64
    if workload == "flux_qkv_w3a3":
        d, N, b = 3072, 9216, 3
        perm, signs = orpbh.draw_permutation_and_signs(0, d)
        cb = ocb.lloyd_max(d, b)
        cw, r16, _, _ = oqz.quantize_weight_rows(f64(inputs.weights(2, inputs.T_W, N, d)), perm, signs, h,
                                                 cb["centroids"])
        bias = f64(inputs.bias(2, N))
        X = f64(inputs.activations(2, 4608, d, rows=(0, rows)))
        t0 = time.perf_counter()
        ca, s, _ = oqz.quantize_rows(X, perm, signs, h, cb["centroids"])
        y = olin.linear_from_codes(ca, s, cw, r16, cb["centroids"], cb["centroids"], d, bias=bias)
        dt = time.perf_counter() - t0
        assert np.isfinite(y).all()
        return dt, 2.0 * rows * N * d
    wl, M, d1, d2, bw, ba = {"flux_mlp": (3, 4608, 3072, 12288, 2, 4),
                             "wan_ffn": (4, 32760, 1536, 8960, 4, 6)}[workload]
    p1, s1 = orpbh.draw_permutation_and_signs(0, d1)
    p2, s2 = orpbh.draw_permutation_and_signs(0, d2)
    ca1, cw1, ca2, cw2 = (ocb.lloyd_max(d1, ba)["centroids"], ocb.lloyd_max(d1, bw)["centroids"],
                          ocb.lloyd_max(d2, ba)["centroids"], ocb.lloyd_max(d2, bw)["centroids"])
    w1c, w1r, _, _ = oqz.quantize_weight_rows(f64(inputs.weights(wl, inputs.T_W, d2, d1)), p1, s1, h, cw1)
    w2c, w2r, _, _ = oqz.quantize_weight_rows(f64(inputs.weights(wl, inputs.T_W2, d1, d2)), p2, s2, h, cw2)
    X = f64(inputs.activations(wl, M, d1, rows=(0, rows)))
    t0 = time.perf_counter()
    a1, n1, _ = oqz.quantize_rows(X, p1, s1, h, ca1)
    y1 = oqz.bf16_round(olin.linear_from_codes(a1, n1, w1c, w1r, ca1, cw1, d1, gelu=True))
    a2, n2, _ = oqz.quantize_rows(y1, p2, s2, h, ca2)
    y2 = olin.linear_from_codes(a2, n2, w2c, w2r, ca2, cw2, d2)
    dt = time.perf_counter() - t0
    assert np.isfinite(y2).all()
    return dt, 4.0 * rows * d1 * d2


def _workload_cpu_baseline(args, rows):
    if getattr(args, "no_cpu_baseline", False):
        return None
    dt, flops = oracle_workload_sample(args.workload, rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{rows} tokens through the timed launches; weights quantized beforehand, untimed"}


def run_workload(args):
    """Per-kernel times of the two-layer workloads (one JSON line each; not the
    contract line).  flux_mlp: X[4608 x 3072] -> fc1 [12288 x 3072] + GELU ->
    fc2 [3072 x 12288], W2A4, block 128.  wan_ffn: X[32760 x 1536] Student-t(3)
    -> fc1 [8960 x 1536] + GELU -> fc2 [1536 x 8960], W4A6, block 128.
    flux_qkv_w3a3: the FLUX-like QKV projection (X[4608 x 3072] -> W[9216 x 3072]
    + bias) at W3A3 ([OQ] Experiments, Qualitative Results).  Every launch is
    timed alone after an L2 flush (L2Flush), the launches round-robin; the SM
    clock is sampled meanwhile."""
    import torch
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import inputs
    from calibration_free_rotated_b200 import orbitquant as oq
    peaks, src = load_peaks()
    h = 128
    dev = torch.device("cuda")
    bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)
    flush = L2Flush(dev)
    if args.workload == "flux_qkv_w3a3":
        M, d, N, b = 4608, 3072, 9216, 3
        r, cb = oq.Rpbh(0, d, h), oq.Codebook(d, b)
        X = bf(inputs.activations(2, M, d))
        wc, wn = oq.quantize_weight(r, cb, bf(inputs.weights(2, inputs.T_W, N, d)))
        bias = bf(inputs.bias(2, N))
        ac, an = oq.quantize_act(r, cb, X)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        with ClockSampler(torch.cuda.current_device()) as clk:
            ms_q, ms_g = _flush_and_time_many(
                [lambda: oq.quantize_act(r, cb, X, ac, an),
                 lambda: oq.linear_codes(d, cb, cb, ac, an, wc, wn, bias=bias, out_bf16=Y, want_f32=False,
                                         want_bf16=True)], flush, args.steps, args.warmup)
        oq.device_status()
        gbs, tfs = algorithmic(M, d, N, b, b)[0] / ms_q / 1e6, 2.0 * M * N * d / ms_g / 1e9
        print(json.dumps({"workload": args.workload, "M": M, "d": d, "N": N, "bits_w": b, "bits_a": b, "block": h,
                          "kernels": {"act_quant": {"ms": ms_q, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]},
                                      "qkv": {"ms": ms_g, "TFLOP/s": tfs, "frac": tfs / peaks["bf16_tflops"]}},
                          "peak_source": src, "step_ms": ms_q + ms_g,
                          "TFLOP/s": 2.0 * M * N * d / (ms_q + ms_g) / 1e9, "clocks": clk.summary(),
                          "cpu_baseline": _workload_cpu_baseline(args, 2048)}), flush=True)
        return 0
    wl, M, d1, d2, bw, ba = {"flux_mlp": (3, 4608, 3072, 12288, 2, 4),
                             "wan_ffn": (4, 32760, 1536, 8960, 4, 6)}[args.workload]
    X = bf(inputs.activations(wl, M, d1))
    r1, r2 = oq.Rpbh(0, d1, h), oq.Rpbh(0, d2, h)
    ca1, cw1, ca2, cw2 = oq.Codebook(d1, ba), oq.Codebook(d1, bw), oq.Codebook(d2, ba), oq.Codebook(d2, bw)
    W1 = bf(inputs.weights(wl, inputs.T_W, d2, d1))
    w1c, w1n = oq.quantize_weight(r1, cw1, W1)
    w2c, w2n = oq.quantize_weight(r2, cw2, bf(inputs.weights(wl, inputs.T_W2, d1, d2)))
    # fc2's permutation folded into fc1 (offline): W1's rows in the order pi_2,
    # so fc1 emits P_2 GELU(.) and fc2's act-quant needs only blkdiag(H D_2),
    # the Block-RHT handle of the same seed (same signs, no permutation)
    perm2 = torch.from_numpy(r2.export()[0].astype(np.int64)).to(dev)
    w1fc, w1fn = oq.quantize_weight(r1, cw1, W1[perm2].contiguous())
    del W1
    r2b = oq.Rpbh(0, d2, h, kind="block_rht")
    a1c, a1n = oq.quantize_act(r1, ca1, X)
    Y1 = torch.empty((M, d2), dtype=torch.bfloat16, device=dev)
    Y1f = torch.empty((M, d2), dtype=torch.bfloat16, device=dev)
    a2c = torch.empty((M, d2 * ba // 8), dtype=torch.uint8, device=dev)
    a2n = torch.empty((M,), dtype=torch.float32, device=dev)
    Y2 = torch.empty((M, d1), dtype=torch.bfloat16, device=dev)
    steps = [
        ("act_quant_1", lambda: oq.quantize_act(r1, ca1, X, a1c, a1n), "hbm", algorithmic(M, d1, d2, ba, bw)[0]),
        ("fc1_gelu", lambda: oq.linear_codes(d1, ca1, cw1, a1c, a1n, w1c, w1n, epilogue="gelu", out_bf16=Y1,
                                             want_f32=False, want_bf16=True), "tensor", 2.0 * M * d1 * d2),
        ("act_quant_2", lambda: oq.quantize_act(r2, ca2, Y1, a2c, a2n), "hbm", algorithmic(M, d2, d1, ba, bw)[0]),
        ("fc2", lambda: oq.linear_codes(d2, ca2, cw2, a2c, a2n, w2c, w2n, out_bf16=Y2, want_f32=False,
                                        want_bf16=True), "tensor", 2.0 * M * d1 * d2),
        ("fc1_gelu_folded", lambda: oq.linear_codes(d1, ca1, cw1, a1c, a1n, w1fc, w1fn, epilogue="gelu",
                                                    out_bf16=Y1f, want_f32=False, want_bf16=True),
         "tensor", 2.0 * M * d1 * d2),
        ("act_quant_2_folded", lambda: oq.quantize_act(r2b, ca2, Y1f, a2c, a2n), "hbm",
         algorithmic(M, d2, d1, ba, bw)[0]),
    ]
    out = {"workload": args.workload, "M": M, "d_in": d1, "d_hidden": d2, "bits_w": bw, "bits_a": ba, "block": h,
           "kernels": {}, "peak_source": src}
    total = 0.0
    folded = 0.0
    with ClockSampler(torch.cuda.current_device()) as clk:
        all_ms = _flush_and_time_many([fn for _, fn, _, _ in steps], flush, args.steps, args.warmup)
    for (name, fn, bound, work), ms in zip(steps, all_ms):
        if name in ("act_quant_1", "fc2") or name.endswith("_folded"):
            folded += ms
        if not name.endswith("_folded"):
            total += ms
        if bound == "hbm":
            ach = work / ms / 1e6
            out["kernels"][name] = {"ms": ms, "GB/s": ach, "frac": ach / peaks["hbm_gbs"]}
        else:
            ach = work / ms / 1e9
            out["kernels"][name] = {"ms": ms, "TFLOP/s": ach, "frac": ach / peaks["bf16_tflops"]}
    oq.device_status()
    out["step_ms"] = total
    out["TFLOP/s"] = 4.0 * M * d1 * d2 / total / 1e9
    out["step_ms_folded_permutation"] = folded
    out["TFLOP/s_folded_permutation"] = 4.0 * M * d1 * d2 / folded / 1e9
    out["clocks"] = clk.summary()
    out["cpu_baseline"] = _workload_cpu_baseline(args, 1024)
    print(json.dumps(out), flush=True)
    return 0


def run_flatness(args):
    """The flatness check ([RHT] Key contribution 4: rho3 and rhoinf of every
    row, and the batch maxima) timed alone after an L2 flush (L2Flush), with per-row
    outputs and with the batch maxima only, on N(0,1) bf16 rows.  Algorithmic
    bytes: the rows once (2 M d) plus 8 bytes per row written (4 per measure)
    and the maxima.  One JSON line per shape; not the contract line."""
    import torch
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import orbitquant as oq
    peaks, src = load_peaks()
    torch.manual_seed(0)
    flush = L2Flush()
    for M, d in ((4608, 3072), (32768, 3072), (32760, 8960), (16384, 12288)):
        X = torch.randn(M, d, device="cuda").to(torch.bfloat16)
        r3 = torch.empty(M, device="cuda")
        ri = torch.empty(M, device="cuda")
        bm = torch.empty(2, device="cuda")
        ms_rows = _flush_and_time(lambda: oq.row_flatness(X, r3, ri, bm), flush, args.steps, args.warmup)
        ms_batch = _flush_and_time(lambda: oq.row_flatness(X, batch_max=bm, want_rows=False), flush, args.steps,
                                   args.warmup)
        oq.device_status()
        byt_rows, byt_batch = 2.0 * M * d + 8.0 * M + 8, 2.0 * M * d + 8
        out = {"flatness": "row_flatness", "M": M, "d": d, "peak_source": src,
               "with_rows": {"us": 1e3 * ms_rows, "GB/s": byt_rows / ms_rows / 1e6,
                             "frac_hbm": byt_rows / ms_rows / 1e6 / peaks["hbm_gbs"]},
               "batch_only": {"us": 1e3 * ms_batch, "GB/s": byt_batch / ms_batch / 1e6,
                              "frac_hbm": byt_batch / ms_batch / 1e6 / peaks["hbm_gbs"]}}
        print(json.dumps(out), flush=True)
        del X
    return 0


def _sylvester(h, device):
    import torch
    H = torch.ones((1, 1), dtype=torch.float64, device=device)
    while H.shape[0] < h:
        H = torch.cat([torch.cat([H, H], 1), torch.cat([H, -H], 1)], 0)
    return H


def rotate_rows_f64(U, tables, h):
    """The (composed) RPBH rotation of fp64 rows U [n, d] for the sweep's error
    measurement: per round (round 1 first), gather by the round's permutation,
    multiply by its signs, then each block of h by the normalised Sylvester
    Hadamard matrix.  tables: [(perm int64 [d], sign float64 [d]), ...]."""
    n, d = U.shape
    H = _sylvester(h, U.device) / math.sqrt(h)
    for perm_t, sign in tables:
        U = ((U[:, perm_t] * sign).view(n, d // h, h) @ H.T).view(n, d)
    return U


def run_sweep(args):
    """The standalone rotate+quantize sweep: M in {1k, 16k, 64k} x d in {1536,
    3072, 12288} x block {64, 128, 256} x bits {2, 4, 6} on N(0,1) rows whose
    last M/8 are one-hot / k-sparse (one zero row).  Per run: the kernel's time
    (L2 flushed, CUDA events), GB/s against the measured HBM copy rate, and the
    empirical per-row squared error ||t - c[code]||^2 of the unit rotated rows
    (dense rows and sparse rows apart, up to 4096 of each) next to the Lloyd-Max
    distortion d * D(d, b) of the codebook.  The error is measured with a
    separate torch rotation (fp64) of the exported permutation and signs; the
    codes are the kernel's.  One JSON line per run."""
    import torch
    from calibration_free_rotated_b200 import build
    build.build()
    from calibration_free_rotated_b200 import inputs
    from calibration_free_rotated_b200 import orbitquant as oq
    peaks, src = load_peaks()
    dev = torch.device("cuda")
    flush = L2Flush(dev)
    Ms = [int(x) for x in args.sweep_rows.split(",")]
    for d in (1536, 3072, 12288):
        for M in Ms:
            X = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
            for r0 in range(0, M, 8192):  # generated in row blocks to bound host memory
                r1 = min(M, r0 + 8192)
                Xb = inputs.sweep_activations(M, d, rows=(r0, r1))
                X[r0:r1] = torch.from_numpy(np.ascontiguousarray(Xb).view(np.int16)).to(dev).view(torch.bfloat16)
            n_adv = M // 8
            rows_dense = torch.arange(0, min(4096, M - n_adv), device=dev)
            rows_adv = torch.arange(M - n_adv, min(M - 1, M - n_adv + 4096), device=dev)  # not the zero row
            # the flatness check's batch maxima ([RHT] Key contribution 4) of each row set
            flat = {k: oq.row_flatness(X[rows].contiguous(), want_rows=False)[2].tolist()
                    for k, rows in (("dense", rows_dense), ("adversarial", rows_adv))}
            for h in (64, 128, 256):
                r = oq.Rpbh(0, d, h, rounds=args.rounds)
                tables = []
                for k in range(1, args.rounds + 1):
                    perm, sbits = r.export_round(k)
                    sign = torch.tensor([-1.0 if (sbits[j >> 5] >> (j & 31)) & 1 else 1.0 for j in range(d)],
                                        dtype=torch.float64, device=dev)
                    tables.append((torch.from_numpy(perm.astype(np.int64)).to(dev), sign))
                def unit_rotated(rows):
                    u = rotate_rows_f64(X[rows].double(), tables, h)
                    return u / u.norm(dim=1, keepdim=True).clamp_min(1e-300)

                T = {"dense": unit_rotated(rows_dense), "adversarial": unit_rotated(rows_adv)}
                for bits in (2, 4, 6):
                    cb = oq.Codebook(d, bits)
                    ex = cb.export()
                    c, D = ex["centroids"], ex["distortion"]
                    codes = torch.empty((M, d * bits // 8), dtype=torch.uint8, device=dev)
                    norms = torch.empty((M,), dtype=torch.float32, device=dev)
                    ms = _flush_and_time(lambda: oq.quantize_act(r, cb, X, codes, norms), flush, args.steps,
                                         args.warmup)
                    gbs = algorithmic(M, d, 1, bits, bits)[0] / ms / 1e6
                    cent = torch.from_numpy(np.asarray(c, dtype=np.float64)).to(dev)
                    line = {"sweep": "rotate_quantize", "M": M, "d": d, "block": h, "rounds": args.rounds, "bits": bits,
                            "median_us": 1e3 * ms,
                            "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"], "peak_source": src,
                            "mse_theory": d * D}
                    for key, rows in (("dense", rows_dense), ("adversarial", rows_adv)):
                        k = _unpack_codes_torch(codes[rows], bits, d)
                        err = ((T[key] - cent[k]) ** 2).sum(dim=1)
                        line["mse_" + key] = float(err.mean())
                        line["rho3_max_" + key], line["rhoinf_max_" + key] = flat[key]
                    print(json.dumps(line), flush=True)
            del X
    oq.device_status()
    return 0


def _unpack_codes_torch(packed, bits, d):
    """Little-endian bit stream [rows, d*bits/8] -> int64 codes [rows, d]."""
    import torch
    b = packed.to(torch.int64)
    bitpos = torch.arange(d, device=packed.device) * bits
    byte, sh = bitpos // 8, bitpos % 8
    lo = b[:, byte]
    hi = b[:, torch.clamp(byte + 1, max=packed.shape[1] - 1)]
    return ((lo | (hi << 8)) >> sh) & ((1 << bits) - 1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parity", action="store_true", help="skip the sampled-row parity check of the bench line")
    ap.add_argument("--profile", choices=["rotq", "gemm", "flatness"], help="launch one kernel only (for ncu captures)")
    ap.add_argument("--ablation", choices=["rotation", "steps"],
                    help="rotation: the rotation variants of the ablation table; steps: back-to-back steps without "
                         "per-kernel events (programmatic dependent launch on, or off with OQ_NO_PDL=1)")
    ap.add_argument("--workload", choices=["flux_mlp", "wan_ffn", "flux_qkv_w3a3"],
                    help="per-kernel times of a layer workload")
    ap.add_argument("--sweep", action="store_true", help="the rotate+quantize sweep with empirical MSE")
    ap.add_argument("--flatness", action="store_true", help="time the flatness check (rho3, rhoinf per row)")
    ap.add_argument("--sweep-rows", default="1024,16384,65536")
    ap.add_argument("--rounds", type=int, default=1, help="composed RPBH rounds for --sweep and --profile rotq (1, 2 or 3)")
    ap.add_argument("--rows", type=int, default=4608)
    ap.add_argument("--d", type=int, default=3072)
    ap.add_argument("--n", type=int, default=9216)
    ap.add_argument("--block", type=int, default=128)
    ap.add_argument("--bits-a", type=int, default=4)
    ap.add_argument("--bits-w", type=int, default=4)
    ap.add_argument("--epilogue", choices=["none", "gelu"], default="none", help="GEMM epilogue for --profile gemm")
    args = ap.parse_args()
    if args.profile:
        return run_profile_case(args)
    if args.ablation == "steps":
        return run_ablation_steps(args)
    if args.ablation:
        return run_ablation(args)
    if args.workload:
        return run_workload(args)
    if args.sweep:
        return run_sweep(args)
    if args.flatness:
        return run_flatness(args)
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
