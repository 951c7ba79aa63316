#!/usr/bin/env python
"""Benchmark of the activation-sparse ReLU FFN forward pass (TwELL) on B200.

One step = one whole layer forward through the C ABI, twell_ffn_forward (fused
up-projection + ReLU + TwELL packing, then the sparse down-projection; the
phase split comes from a second loop of twell_up_pack + twell_spmm) on
the 1.5B-scale layer (M=4096 tokens, d_model=2048, d_ff=8192, bf16, weights
N(0, 1/fan_in), bias set for the target activation density, tile_w=128, ell_w
from the 99th-percentile rule).  Synthetic, seeded inputs; no dataset.

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun): tokens are independent, so
every rank runs its own 4096-token batch with replicated weights and no
data-path collective ("scaling": "weak"); value = all ranks' tokens / the
slowest rank's device time.

--impl reference times the CPU oracle (fp64 NumPy) on the host cores on a
bounded sample of the same workload; nothing else exists to compare against.
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
sys.path.insert(0, ROOT)

METRIC = "sparse FFN tokens/s per layer vs activation density; % of roofline (HBM/TC)"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return dict(hbm_gbs=float(j["hbm_gbs"]), tc_tflops=float(j["bf16_tflops"]),
                    tc_tflops_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, tc_tflops=1590.0, tc_tflops_sustained=1400.0, source="fallback")


def _kernel_source_hash(path):
    with open(os.path.join(ROOT, path), "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def _ncu_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, only if it was taken on the current source of the kernel (else null)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        j = json.load(fh)
    e = j.get(workload, {}).get(kernel)
    if not e or e.get("source_sha256_16") != _kernel_source_hash(
            os.path.join("activation_sparse_ffn_twell_b200", "csrc", e["source"])):
        return None
    return float(e["dram_bytes_per_launch"])


# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            self.h = N.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        N = self.N
        names = {
            "gpu_idle": getattr(N, "nvmlClocksEventReasonGpuIdle", 0x1),
            "sw_power_cap": getattr(N, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(N, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(N, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(N, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(N, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
                try:
                    r = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = N.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for k, bit in names.items():
                    if r & bit and k != "gpu_idle":
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()
        return False

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(s)}


# ---------------------------------------------------------------------------
WORKLOADS = ("relu_15b", "gated_2b", "heavy_tail", "decode32", "decode128", "decode256", "tiny")


def _workload(density, M, seed, name="relu_15b"):
    """The synthetic layer for `name` (default: the 1.5B-scale ReLU layer)."""
    import twell_synth as S
    if name == "relu_15b":
        return S.relu_15b(density=density, M=M, seed=seed)
    if name == "gated_2b":
        return S.gated_2b(density=density, seed=seed)
    if name == "heavy_tail":
        return S.heavy_tail(seed=seed)
    if name.startswith("decode"):
        return S.decode(M=int(name[len("decode"):]), seed=seed)
    if name == "tiny":
        return S.tiny_relu(seed)
    raise SystemExit(f"unknown workload {name}")


def _roofline_layer(L, nnz_total, touched_rows, peaks):
    """North-star roofline of the whole layer: max(useful FLOP / TC peak,
    unavoidable bytes / HBM BW).  Useful FLOP = dense up (x2 if gated) + 2*nnz*d;
    unavoidable bytes = x + W_up (+W_gate) + b + touched W_down rows + y."""
    M, d, f = L.M, L.d_model, L.d_ff
    flop = 2.0 * M * d * f * (2 if L.gated else 1) + 2.0 * nnz_total * d
    byts = 2.0 * (M * d + f * d * (2 if L.gated else 1) + f + touched_rows * d + M * d)
    t_tc = flop / (peaks["tc_tflops"] * 1e12)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    return dict(t_s=max(t_tc, t_hbm), bound="tensor" if t_tc >= t_hbm else "hbm",
                useful_flop=flop, unavoidable_bytes=byts)


def run_ours(args):
    import torch
    import activation_sparse_ffn_twell_b200 as T
    from activation_sparse_ffn_twell_b200 import dist as D

    rank, local, world = D.init("nccl" if args.gpus > 1 else "gloo")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = _peaks()

    def to_dev(bits):
        import numpy as np
        return None if bits is None else torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    L = _workload(args.density, args.M, args.seed + rank, args.workload)   # own batch per rank
    x, wu, b, wd = to_dev(L.x), to_dev(L.w_up), to_dev(L.b), to_dev(L.w_down)
    wg = to_dev(L.w_gate)
    M, d, f, tw, E = L.M, L.d_model, L.d_ff, L.tile_w, L.ell_w
    T_tiles = f // tw
    a = T.TwELL.allocate(M, f, tw, E, T.default_ovf_capacity(M, T_tiles), device=dev)
    y = torch.empty((M, d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fused():
        T.twell_ffn_forward(x, wu, b, wd, tile_w=tw, ell_w=E, W_gate=wg, mode=args.mode, out=a, y=y)

    def split():
        T.twell_up_pack(x, wu, b, wg, tile_w=tw, ell_w=E, out=a)
        T.twell_spmm(a, wd, mode=args.mode, y=y)

    # warm-up: the timed call itself (W steps), then the phase calls of the
    # second loop, so neither loop's first step pays for first use
    for _ in range(args.warmup):
        flush.zero_()
        fused()
    for _ in range(3):
        flush.zero_()
        split()
    code, n_ovf = T.read_status(a)
    if code != 0:
        raise SystemExit(f"status {T.STATUS[code]} after warm-up")
    nnz = a.nnz_u16()
    nnz_total = int(nnz.sum().item())
    # W_down rows any token touches (hidden units active for at least one token)
    # are counted from the packed output with a tiny torch reduction off the timed path.
    touched = int(_touched_rows(a, torch).item())
    density = nnz_total / float(M * f)

    # ------------------------------------------------ timed region (device events)
    # A step is the user-facing fused call twell_ffn_forward (its kernels chain
    # as dependent launches).  A second timed loop of the same length runs the
    # two calls separately, with events between them, for the phase split.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    evp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    D.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()                      # evict L2 between steps (inputs < 126 MB)
            e0, e1 = ev[i]
            e0.record(stream)
            fused()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
        for i in range(args.steps):
            flush.zero_()
            e0, e1, e2 = evp[i]
            e0.record(stream)
            T.twell_up_pack(x, wu, b, wg, tile_w=tw, ell_w=E, out=a)
            e1.record(stream)
            T.twell_spmm(a, wd, mode=args.mode, y=y)
            e2.record(stream)
        torch.cuda.synchronize(dev)
    D.barrier(dev)
    # the step time is the median of the K per-step event intervals (robust to a
    # stray slow step); the mean is reported beside it
    step_all = [e0.elapsed_time(e1) for e0, e1 in ev]
    step_ms = _median(step_all)
    step_mean = sum(step_all) / len(step_all)
    up_ms = [e0.elapsed_time(e1) for e0, e1, _ in evp]
    down_ms = [e1.elapsed_time(e2) for _, e1, e2 in evp]
    step_ms_max = D.max_over_ranks(step_ms, dev if world > 1 and args.gpus > 1 else None)
    code, n_ovf2 = T.read_status(a)
    if code != 0:
        raise SystemExit(f"status {T.STATUS[code]} in timed region")

    tokens_s = world * M / (step_ms_max * 1e-3)
    up_s = _median(up_ms) * 1e-3
    down_s = _median(down_ms) * 1e-3
    rl = _roofline_layer(L, nnz_total, touched, peaks)
    # Per-phase rooflines from algorithmic work: each phase is bound by the
    # slower of its FLOPs at the tensor peak and its unavoidable bytes at the HBM
    # peak.  Up: 2*M*d*f FLOP (x2 gated); x + W_up (+W_gate) + b read, packed
    # TwELL written.  Down: 2*nnz*d FLOP; the W_down rows any token touches,
    # the packed TwELL and y.  (The tensor-core down path executes the dense
    # 2*M*d*f on h tiles rebuilt from TwELL: reported as executed_tflops.)
    dec_up, dec_down = _decode_paths(M, f, tw, args.mode)
    packed = M * T_tiles * (3 * E + 2) + n_ovf * (4 + 2 * tw)
    up_flop = 2.0 * M * d * f * (2 if L.gated else 1)
    up_bytes = 2.0 * (M * d + f * d * (2 if L.gated else 1) + f) + packed
    down_flop = 2.0 * nnz_total * d
    down_bytes = 2.0 * touched * d + packed + 2.0 * M * d
    wkey = f"relu_15b_rho{args.density:g}" if args.workload == "relu_15b" else args.workload

    def phase(kernel, desc, flop, byts, sec):
        t_tc, t_hbm = flop / (peaks["tc_tflops"] * 1e12), byts / (peaks["hbm_gbs"] * 1e9)
        if t_tc >= t_hbm:
            bound, ach, unit, peak = "tensor", flop / sec / 1e12, "TFLOP/s", peaks["tc_tflops"]
        else:
            bound, ach, unit, peak = "hbm", byts / sec / 1e9, "GB/s", peaks["hbm_gbs"]
        return {"kernel": f"{kernel} ({desc})", "ms": sec * 1e3, "bound": bound, "achieved": ach,
                "unit": unit, "peak": peak, "frac": ach / peak, "roofline_ms": max(t_tc, t_hbm) * 1e3,
                "algorithmic_flop": flop, "algorithmic_bytes": byts,
                "traffic": _ncu_traffic(kernel, wkey)}

    if dec_up:
        up_k = ("k_up_pack_dec", "decode batch: tokens on MMA N, ballot/prefix TwELL epilogue")
    else:
        up_k = ("k_up_pack", "fused up-GEMM + ReLU + TwELL pack, CTA pairs")
    if args.mode == "gather":
        down_k = ("k_spmm_gather", "CUDA-core gather of W_down rows per nonzero")
    elif dec_down and _decode_touched(M, f):
        down_k = ("k_spmm_dec_touched", "decode batch: touched W_down rows only, split-K clusters")
    elif dec_down:
        down_k = ("k_spmm_dec", "decode batch: split-K clusters, DSMEM reduction")
    elif args.mode == "sparse" and _sparse_ok(M, f, tw, E):
        down_k = ("k_spmm_sp", "2:4 sparse tensor cores on tiles rebuilt from TwELL + excess on CUDA cores")
    else:
        down_k = ("k_spmm_mma", "tensor cores on h tiles rebuilt from TwELL")
    phases = {"up": phase(*up_k, up_flop, up_bytes, up_s),
              "down": phase(*down_k, down_flop, down_bytes, down_s)}
    phases["down"]["executed_tflops"] = 2.0 * M * d * f / down_s / 1e12
    # the executed (dense-rate) work against the tensor peak, next to the algorithmic frac
    phases["down"]["executed_frac_of_tensor_peak"] = phases["down"]["executed_tflops"] / peaks["tc_tflops"]
    dom = max(phases, key=lambda k: phases[k]["ms"])
    P_ = phases[dom]
    result = {
        "metric": METRIC, "value": tokens_s, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
        "ms_per_step_stat": f"median of {args.steps} CUDA-event step intervals",
        "ms_per_step_mean": step_mean, "ms_per_step_min": min(step_all),
        "phase_sum_ms": (up_s + down_s) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1/fan_in) weights, bias for target density)",
        "config": {"workload": {"relu_15b": "relu_ffn_layer_1.5b"}.get(args.workload, args.workload),
                   "M": M, "d_model": d, "d_ff": f,
                   "target_density": L.target_density, "measured_density": density,
                   "tile_w": tw, "ell_w": E, "gated": bool(L.gated), "down_mode": args.mode,
                   "n_ovf": n_ovf, "l2": "flushed: 256 MiB write between timed steps",
                   "parallelism": f"token-sharded x{world} (weights replicated, no collective)"},
        "roofline": {"bound": P_["bound"], "kernel": P_["kernel"], "phase": dom,
                     "achieved": P_["achieved"], "peak": P_["peak"], "unit": P_["unit"],
                     "frac": P_["frac"],
                     "peak_source": f"{peaks['source']} " + ("bf16 burst" if P_["bound"] == "tensor"
                                                              else "HBM copy"),
                     "traffic": P_["traffic"],
                     "interval": "CUDA events around the phase's C-ABI call on the launching stream"},
        "phases": phases,
        "roofline_layer": {"bound": rl["bound"], "roofline_ms": rl["t_s"] * 1e3,
                           "frac": rl["t_s"] * 1e3 / step_ms_max,
                           "useful_flop": rl["useful_flop"],
                           "unavoidable_bytes": rl["unavoidable_bytes"],
                           "touched_w_down_rows": touched, "peaks": peaks["source"]},
        "gpu_launches": args.steps * _kernels_per_step(args.mode, dec_down, d, _sparse_ok(M, f, tw, E),
                                                       dec_down and _decode_touched(M, f), M),
        "wall_s_timed_region": wall,
    }
    result["clocks"] = clk.summary()

    if not args.quick:
        result["dense_ffn"] = _dense_baseline(x, wu, b, wd, args, flush, stream, dev, wg)
        result["e2e"] = _e2e(T, L, x, wu, b, wd, a, y, args, dev, stream, world)
        if args.workload == "relu_15b":
            # fused layer against the dense cuBLAS FFN at every density of the
            # 1.5B-layer workload (--sweep adds the forced gather / MMA paths)
            result["density_sweep"] = _sweep(T, args, dev, peaks,
                                             modes=("auto", "gather", "mma") if args.sweep else ("auto",))
    if args.backward and not L.gated and M % 128 == 0:
        result["backward"] = _backward(T, x, wu, b, wd, a, args, flush, stream, dev)
    if args.token_overflow:
        result["token_overflow"] = _token_overflow(T, a, wd, y, args, flush, stream, dev, n_ovf)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = _cpu_baseline(L, seconds=args.cpu_seconds)
    if args.workload != "relu_15b":
        result["note"] = "extra workload (not the headline configuration)"
    if rank == 0:
        print(json.dumps(result), flush=True)
    del a
    D.finish()


def _median(v):
    s = sorted(v)
    n = len(s)
    return s[n // 2] if n % 2 else 0.5 * (s[n // 2 - 1] + s[n // 2])


def _touched_rows(a, torch):
    # a hidden unit j is touched if any token has it among its packed nonzeros
    # (ELL slots of non-overflowing pairs, or nonzeros of a backup segment)
    M, T_, E = a.vals.shape
    tw = a.tile_w
    nnz = a.nnz_u16()
    live = torch.arange(E, device=a.vals.device)[None, None, :] < torch.minimum(nnz, torch.tensor(E, device=nnz.device))[:, :, None]
    live = live & (nnz[:, :, None] <= E)
    cols = (torch.arange(T_, device=a.vals.device)[None, :, None] * tw + a.idx.to(torch.int64))
    touched = torch.zeros(a.d_ff, dtype=torch.bool, device=a.vals.device)
    touched[cols[live]] = True
    n = int(a.n_ovf.item())
    if n:
        pos = a.ovf_pos[:n].to(torch.int64)
        t = pos % T_
        seg = a.ovf_dense[:n].view(torch.int16) & 0x7FFF
        jj = torch.nonzero(seg != 0)
        touched[t[jj[:, 0]] * tw + jj[:, 1]] = True
    return touched.sum()


def _decode_paths(M, f, tw, mode):
    """Which kernels the library picks (the dispatch rule of twell_up_pack and
    twell_spmm): decode-size batches (M <= 256) use the token-on-N kernels."""
    return (M <= 256 and tw <= 128 and f % 128 == 0), (M <= 256 and mode != "gather")


def _decode_touched(M, f):
    """Decode-size batches whose down-projection takes the touched-unit kernel
    (the library's rule: up to 32 tokens, d_ff <= 65536; TWELL_DECODE_TOUCHED=0
    turns it off, =all extends it to every decode-size batch)."""
    import os
    sel = os.environ.get("TWELL_DECODE_TOUCHED", "")
    if sel.startswith("0") or f > 65536:
        return False
    if not sel.startswith("a"):
        return M <= 32
    # every decode-size batch whose stage ring leaves room for the gather's
    # lag of 4 stages (the library's check, with the largest unit list)
    np_ = 16 if M <= 16 else (M + 15) // 16 * 16
    tables = 8 * (f // 32 + 1) + 2 * ((f + 63) // 64) * 64
    return M <= 256 and (225 * 1024 - 1536 - tables) // (16384 + np_ * 128) > 4


def _kernels_per_step(mode, dec_down=False, d_model=0, sparse_ok=False, dec_touched=False, M=4096):
    # up_pack: k_pack_reset + the producer + k_ovf_row_scan + k_ovf_scatter (up to
    # 256 tokens the scan and the scatter are one kernel, k_ovf_finalize_small).
    # spmm in sparse mode, where the 2:4 path applies: k_sp_prep, k_sp_decide,
    # k_spmm_sp and k_spmm_mma, each tensor kernel taking its own token groups.
    # Otherwise auto: k_block_path, gather and k_spmm_mma; mma runs
    # k_block_path too when the split schedule is possible (d_model > 256: it
    # zeroes the arrival counters); the decode-size down path is one kernel.
    up = 3 if M <= 256 else 4
    if dec_down:
        return up + (2 if dec_touched else 1)   # k_dec_touch before the touched-unit kernel
    if sparse_ok and mode == "sparse":
        return up + 4   # k_sp_prep, k_sp_decide, k_spmm_sp, k_spmm_mma
    if mode == "auto":
        return up + 3
    if mode in ("mma", "sparse"):
        return up + (2 if d_model > 256 else 1)
    return up + 1


def _sparse_ok(M, f, tw, E):
    """Shapes the library's 2:4 down path takes (its host-side eligibility rule)."""
    return tw in (64, 128) and E % 8 == 0 and E <= 32 and f < 65536 and M > 256


def _dense_baseline(x, wu, b, wd, args, flush, stream, dev, wg=None):
    """Same-shape dense bf16 FFN through cuBLAS (torch.matmul), same run, same timing."""
    import torch
    import torch.nn.functional as F

    def dense():
        if wg is not None:   # gated: ReLU(x W_g^T + b) * (x W_u^T)
            h = torch.relu(F.linear(x, wg, b)) * F.linear(x, wu)
        else:
            h = torch.relu(F.linear(x, wu, b))
        return torch.matmul(h, wd)
    for _ in range(max(3, args.warmup)):
        dense()
    ts = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        dense()
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize(dev)
    ms = _median([a.elapsed_time(b) for a, b in ts])
    return {"ms_per_step": ms, "tokens_s": x.shape[0] / (ms * 1e-3),
            "impl": "torch.matmul bf16 (cuBLAS): relu(x W_up^T + b) W_down"}


def _backward(T, x, wu, b, wd, a, args, flush, stream, dev):
    """Backward pass through the hybrid form (twell_ffn_backward, given the
    forward's TwELL) next to the same-shape dense backward through cuBLAS
    (dH = dY W_down^T, ReLU mask, dX = dZ W_up, dW_up = dZ^T x, db, dW_down = h^T dY),
    same run, same timing (L2 flushed between steps)."""
    import torch
    g = torch.Generator(device=dev).manual_seed(1)
    dy = torch.randn(x.shape, generator=g, device=dev).to(torch.bfloat16)
    M, f = x.shape[0], wu.shape[0]
    cap_t = max(4096, f * (M // 128) // 8)

    def ours():
        return T.twell_ffn_backward(x, wu, wd, a, dy, ovf_capacity_t=cap_t)

    h = torch.relu(torch.nn.functional.linear(x, wu, b))   # the dense forward's saved h

    def dense():
        dz = torch.matmul(dy, wd.t()) * (h > 0)
        return torch.matmul(dz, wu), torch.matmul(dz.t(), x), dz.float().sum(0), torch.matmul(h.t(), dy)

    out = {}
    for name, fn in (("ms", ours), ("dense_ms", dense)):
        for _ in range(max(3, args.warmup)):
            fn()
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            ts.append((e0, e1))
        torch.cuda.synchronize(dev)
        out[name] = sum(p.elapsed_time(q) for p, q in ts) / len(ts)
    code, _ = T.read_status(a)
    out["status"] = T.STATUS[code]
    out["impl"] = ("twell_ffn_backward: SDDMM dZ on tensor cores at the forward's pattern, dX / "
                   "dW_down / dW_up through the sparse down-projection on transposed TwELL; dense: "
                   "torch.matmul bf16 (cuBLAS) from the dense forward's saved h")
    out["ovf_capacity_t"] = cap_t
    return out


def _token_overflow(T, a, wd, y, args, flush, stream, dev, n_ovf):
    """The two readings of the dense backup on the same packed data: per (token,
    tile) pair (the library's form) against whole tokens (twell_spmm_token_overflow:
    tokens with any over-full tile run as a small dense product).  Backup bytes and
    down-projection time of each."""
    import torch
    _, n_tok = T.twell_spmm_token_overflow(a, wd, cap_tok=a.M)
    torch.cuda.synchronize(dev)
    nt = int(n_tok.item())
    cap = max(128, (nt + 127) // 128 * 128)
    T_ = a.d_ff // a.tile_w
    out = {"n_overflow_pairs": n_ovf, "n_overflow_tokens": nt, "cap_tok": cap,
           "backup_bytes_pairs": n_ovf * (4 + 2 * a.tile_w),
           "backup_bytes_tokens_dense_rows": nt * (4 + 2 * a.d_ff),
           "backup_bytes_tokens_as_stored": nt * T_ * (3 * a.tile_w + 2) + 4 * nt}
    for name, fn in (("ms_pairs", lambda: T.twell_spmm(a, wd, y=y)),
                     ("ms_tokens", lambda: T.twell_spmm_token_overflow(a, wd, cap_tok=cap, y=y))):
        for _ in range(max(3, args.warmup)):
            fn()
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            ts.append((e0, e1))
        torch.cuda.synchronize(dev)
        out[name] = sum(p.elapsed_time(q) for p, q in ts) / len(ts)
    code, _ = T.read_status(a)
    out["status"] = T.STATUS[code]
    return out


def _e2e(T, L, x, wu, b, wd, a, y, args, dev, stream, world):
    """End to end through the public API with host buffers: each step copies its
    tokens from pinned host memory to the device, runs twell_ffn_forward and copies
    y back to pinned host memory, all inside the timed region.  As in a serving
    pipeline the three run on their own streams with double-buffered device x / y
    and host y: step i+1's upload and step i-1's download overlap step i's layer
    (stream events order every reuse of a buffer)."""
    import numpy as np
    import torch
    from activation_sparse_ffn_twell_b200 import dist as D
    xh = torch.from_numpy(L.x.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = [torch.empty((L.M, L.d_model), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(x) for _ in range(2)]
    yd = [torch.empty_like(y) for _ in range(2)]
    wg = None if L.w_gate is None else torch.from_numpy(L.w_gate.view(np.int16)).view(torch.bfloat16).to(dev)
    s_up, s_cmp, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run(n):
        done_cmp = [None, None]   # compute of the step that last used buffer j
        done_dn = [None, None]    # download of the step that last used buffer j
        last = None
        for i in range(n):
            j = i & 1
            with torch.cuda.stream(s_up):
                if done_cmp[j] is not None:
                    s_up.wait_event(done_cmp[j])
                xd[j].copy_(xh, non_blocking=True)
                up = torch.cuda.Event()
                up.record(s_up)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(up)
                if done_dn[j] is not None:
                    s_cmp.wait_event(done_dn[j])
                T.twell_ffn_forward(xd[j], wu, b, wd, tile_w=L.tile_w, ell_w=L.ell_w, W_gate=wg,
                                    mode=args.mode, out=a, y=yd[j], stream=s_cmp)
                c = torch.cuda.Event()
                c.record(s_cmp)
                done_cmp[j] = c
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(c)
                yh[j].copy_(yd[j], non_blocking=True)
                dn = torch.cuda.Event()
                dn.record(s_dn)
                done_dn[j] = dn
                last = dn
        return last

    run(3)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    s_cmp.wait_stream(s_up)
    s_dn.wait_stream(s_up)
    last = run(args.steps)
    s_dn.wait_event(last)
    e1.record(s_dn)
    torch.cuda.synchronize(dev)
    # the downloaded result is the layer's output for these tokens
    T.twell_ffn_forward(x, wu, b, wd, tile_w=L.tile_w, ell_w=L.ell_w, W_gate=wg, mode=args.mode,
                        out=a, y=y)
    torch.cuda.synchronize(dev)
    if not torch.equal(yh[(args.steps - 1) & 1].view(torch.int16), y.cpu().view(torch.int16)):
        raise SystemExit("e2e: the downloaded y differs from the device result")
    ms = e0.elapsed_time(e1) / args.steps
    ms = D.max_over_ranks(ms, dev if world > 1 else None)
    return {"value": world * L.M / (ms * 1e-3), "unit": UNIT,
            "h2d_bytes_per_step": int(L.M * L.d_model * 2),
            "d2h_bytes_per_step": int(L.M * L.d_model * 2),
            "ms_per_step": ms,
            "note": ("weights resident; x in / y out through pinned host memory every step, "
                     "upload / layer / download pipelined on three streams")}


SWEEP_DENSITIES = (0.20, 0.10, 0.05, 0.02, 0.01)
# --sweep: the forced gather / MMA paths beside auto, with the low densities
# where the per-block crossover between them lies
SWEEP_DENSITIES_FINE = (0.20, 0.10, 0.05, 0.03, 0.02, 0.01, 0.005, 0.0025)


def _sweep(T, args, dev, peaks, modes=("auto",)):
    """The 1.5B-scale layer at each target density: the fused twell_ffn_forward
    (per down mode in `modes`) and the same-shape dense cuBLAS FFN, timed in the
    same run the same way (median of CUDA-event step intervals, L2 flushed
    between steps), with the layer roofline and the margin over dense."""
    import numpy as np
    import torch
    import torch.nn.functional as F
    out = []
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    n_steps = max(10, min(args.steps, 30))

    def timed(fn):
        for _ in range(3):
            flush.zero_()
            fn()
        evs = []
        for _ in range(n_steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            evs.append((e0, e1))
        torch.cuda.synchronize(dev)
        return _median([p.elapsed_time(q) for p, q in evs])

    for rho in (SWEEP_DENSITIES_FINE if len(modes) > 1 else SWEEP_DENSITIES):
        L = _workload(rho, args.M, args.seed)
        tb = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        x, wu, b, wd = tb(L.x), tb(L.w_up), tb(L.b), tb(L.w_down)
        T_tiles = L.d_ff // L.tile_w
        a = T.TwELL.allocate(L.M, L.d_ff, L.tile_w, L.ell_w, T.default_ovf_capacity(L.M, T_tiles),
                             device=dev)
        y = torch.empty((L.M, L.d_model), dtype=torch.bfloat16, device=dev)
        row = {"target_density": rho, "ell_w": L.ell_w, "steps": n_steps}
        for mode in modes:
            row[f"{mode}_ms"] = timed(lambda: T.twell_ffn_forward(x, wu, b, wd, tile_w=L.tile_w,
                                                                  ell_w=L.ell_w, mode=mode, out=a, y=y))
        T.twell_ffn_forward(x, wu, b, wd, tile_w=L.tile_w, ell_w=L.ell_w, mode="auto", out=a, y=y)
        code, n_ovf = T.read_status(a)
        if code != 0:
            raise SystemExit(f"sweep {rho}: status {T.STATUS[code]}")
        nnz_total = int(a.nnz_u16().sum().item())
        row["measured_density"] = nnz_total / float(L.M * L.d_ff)
        row["n_ovf"] = n_ovf
        rl = _roofline_layer(L, nnz_total, int(_touched_rows(a, torch).item()), peaks)
        row["roofline_ms"] = rl["t_s"] * 1e3
        row["frac_roofline_auto"] = rl["t_s"] * 1e3 / row["auto_ms"]
        row["tokens_s_auto"] = L.M / (row["auto_ms"] * 1e-3)
        row["dense_ms"] = timed(lambda: torch.matmul(torch.relu(F.linear(x, wu, b)), wd))
        row["speedup_vs_dense_auto"] = row["dense_ms"] / row["auto_ms"]
        row["margin_vs_dense_auto"] = 1.0 - row["auto_ms"] / row["dense_ms"]
        out.append(row)
        del a, x, wu, b, wd, y
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def _oracle_rate(L, seconds, sample_tokens, max_reps=64):
    """Tokens/s of the oracle forward over repeated `sample_tokens`-token slices
    of the batch (full weights) until ~`seconds` elapse.  Returns (rate, reps, s)."""
    import oracle as O
    done, reps, t0 = 0, 0, time.perf_counter()
    while True:
        r0 = (reps * sample_tokens) % L.M
        rows = slice(r0, r0 + sample_tokens)
        O.ffn_forward(L.x[rows], L.w_up, L.b, L.w_down, L.tile_w, L.ell_w, L.w_gate)
        done += min(sample_tokens, L.M - r0)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or reps >= max_reps:
            return done / el, reps, el


def _cpu_baseline(L, seconds=10.0, sample_tokens=256):
    """The oracle, as it stands, on the host cores over a bounded token sample of
    the same layer (full weights): the whole forward on every BLAS thread, the
    same on one core, and the reference packer alone."""
    import oracle as O
    threads = _blas_threads()
    rate, reps, el = _oracle_rate(L, seconds, sample_tokens)
    out = {"value": rate, "unit": UNIT, "cores": int(threads), "kind": "oracle",
           "sample": f"{reps} x {sample_tokens}-token slices of the {L.M}-token batch, full "
                     f"{L.d_model}x{L.d_ff} weights, fp64 NumPy, {el:.1f} s"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            r1, reps1, el1 = _oracle_rate(L, max(1.0, seconds / 4), 64, max_reps=16)
        out["value_1core"] = r1
        out["sample_1core"] = f"{reps1} x 64-token slices on 1 core, {el1:.1f} s"
    except Exception as e:   # threadpoolctl missing: say so rather than guess
        out["value_1core"] = None
        out["sample_1core"] = f"unavailable: {type(e).__name__}"
    # packer alone: the reference TwELL packer on the sample's (untimed) h
    h = O.hidden(L.x[:sample_tokens], L.w_up, L.b, L.w_gate)
    n, t0 = 0, time.perf_counter()
    while True:
        O.twell_pack(h, L.tile_w, L.ell_w)
        n += 1
        el = time.perf_counter() - t0
        if el >= max(0.5, seconds / 8) or n >= 64:
            break
    out["pack_tokens_s"] = n * h.shape[0] / el
    out["sample_pack"] = f"{n} packs of a {h.shape[0]}-token h, {el:.1f} s"
    return out


def run_reference(args):
    """--impl reference: the CPU oracle timed on the host cores (rank 0 only).
    Each step is the oracle forward over a `ref_tokens`-token sample of the
    batch; ms_per_step is that step's measured time (not scaled to the batch)."""
    from activation_sparse_ffn_twell_b200 import dist as D
    rank, _, world = D.env_rank_world()
    if rank != 0:
        return
    import oracle as O
    L = _workload(args.density, args.M, args.seed)
    n = args.ref_tokens

    def one(r0):
        rows = slice(r0 % L.M, r0 % L.M + n)
        t0 = time.perf_counter()
        O.ffn_forward(L.x[rows], L.w_up, L.b, L.w_down, L.tile_w, L.ell_w, L.w_gate)
        return time.perf_counter() - t0

    for i in range(args.warmup):
        one(i * n)
    per = [one((args.warmup + i) * n) for i in range(args.steps)]
    ms = _median(per) * 1e3
    value = n / (ms * 1e-3)
    cores = _blas_threads()
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "impl": "reference",
        "device": "cpu (host cores)", "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "ms_per_step_stat": f"median of {args.steps} measured steps",
        "total_timed_s": sum(per), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "relu_ffn_layer_1.5b", "M": L.M, "tokens_per_step": n,
                   "d_model": L.d_model, "d_ff": L.d_ff, "target_density": args.density,
                   "tile_w": L.tile_w, "ell_w": L.ell_w},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: the oracle forward over {n} tokens of the "
                                   f"{L.M}-token batch (full weights); ms_per_step is that time"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--density", type=float, default=0.05)
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--mode", default="auto", choices=["auto", "gather", "mma", "sparse"])
    ap.add_argument("--workload", default="relu_15b", choices=WORKLOADS,
                    help="default: the 1.5B-scale layer the headline metric is quoted on")
    ap.add_argument("--sweep", action="store_true",
                    help="density sweep 20%% .. 0.25%% with the forced gather / MMA paths beside auto")
    ap.add_argument("--token-overflow", action="store_true",
                    help="add the whole-token reading of the backup next to the per-pair one")
    ap.add_argument("--backward", action="store_true",
                    help="add the backward pass (twell_ffn_backward) next to a dense cuBLAS backward")
    ap.add_argument("--quick", action="store_true", help="skip dense/e2e legs (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-tokens", type=int, default=128)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
