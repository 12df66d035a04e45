"""Benchmark of the N:M sparsity hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload linear_4096|mlp_pair|decode_T16|decode_T64|decode_T256|decode_T1024|ties_mask|
                               srste|saliency_mask|transposable_mask|transposable_24|pairs_12|int8_24]

One step is one pass of every step of the path over one batch of synthetic
input.  Default: the MLP pair, bf16 W_up 14336x4096 and W_down 4096x14336
pruned 2:4 along K, X 4096x8192 (8192 tokens), 20 timed repetitions; on each
weight
    nm_mask (2:4) -> nm_compress (that mask) -> nm_mask_compress (fused)
    -> nm_meta_to_sm100 -> nm_decompress,
then nm_spmm up (H = W_up' X) and down (Y = W_down' H), bf16 out.
`value` is the dense-equivalent TFLOP/s of the whole step (2*R*K*T flops of
both products per step over the device time of the full step); the
per-kernel breakdown, the roofline of the dominant kernel (the longer
product, sparse tensor peak) and the bandwidth kernels' GB/s against HBM are
reported beside it.

Timing: W untimed warm-up steps, then exactly K steps, each bracketed by CUDA
events on the launching stream, with L2 flushed between steps outside the
events (a 256 MiB write, then a 256 MiB read that evicts the written lines,
so no write-back of the flush lands in a timed region); barrier + synchronize
around the loop; the max over ranks.  The per-kernel breakdown times every
launch on its own with the same flush before each.  N > 1 runs one
independent copy of the workload per GPU (the path has no exchange step;
weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nm_inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Integer (ALU) pipe of a B200 SM: 16 lanes per clock in each of its 4 sub-partitions
# (ncu shows the ALU pipe busy for two issue cycles per warp instruction), 148 SMs at the
# 1965 MHz maximum clock.
ALU_PEAK_TOPS = 148 * 64 * 1.965e9 / 1e12


def transposable_int_ops(M: int) -> float:
    """Integer operations the greedy transposable mask needs per M x M block: two
    (max and min) per comparator of Batcher's network on the padded key count, seven per
    greedy step (position, row and column test, two count updates, record), two per
    key (pack magnitude and position)."""
    P = 1
    while P < M * M:
        P *= 2
    comps, p = 0, 1
    while p < P:
        k = p
        while k >= 1:
            j = k % p
            while j + k < P:
                comps += sum(1 for i in range(k) if i + j + k < P and (i + j) // (2 * p) == (i + j + k) // (2 * p))
                j += 2 * k
            k //= 2
        p *= 2
    return 2.0 * comps + 7.0 * M * M + 2.0 * M * M
SPARSE_RATIO = 2.0   # 2:4 sparse tensor peak = 2x dense (dense-equivalent flops)
PEER_WAIT_NS = 2_000_000_000   # limit of the row-split step's wait for every GPU's rows of H
IPC_MAPPINGS = []              # (address, offset) of every other GPU's buffer this process mapped
# dense throughput of the int8 and tf32 tensor-core kinds relative to bf16 (nominal B200 figures:
# 4.5 POPS int8, 1.1 PFLOPS tf32 against 2.25 PFLOPS bf16); applied to the measured bf16 peak
KIND_RATIO = {"int8": 2.0, "pairs": 0.5}
KIND_NOTE = {"int8": " x 2 (nominal int8/bf16 ratio)", "pairs": " x 0.5 (nominal tf32/bf16 ratio)"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ncu summaries that carry a per-launch DRAM traffic figure for the dominant
# kernel of a workload; the figure is reported only while the kernel source is
# unchanged since the capture (its sha256 is recorded in the summary).
TRAFFIC_PROFILES = {
    ("linear_4096", "nm_spmm"): "profiles/spmm_pair_linear_4096.md",
    ("mlp_pair", "nm_spmm_up"): "profiles/spmm_pair_mlp_up.md",
    ("mlp_pair", "nm_spmm_down"): "profiles/spmm_pair_mlp_down.md",
    ("int8_24", "nm_spmm_s8"): "profiles/spmm_pair_int8_decode_28672x8192x1024.md",
    ("pairs_12", "nm_spmm12"): "profiles/spmm_pair_tf32_8192x8192x4096.md",
}


def compute_dtype(wl, kind: str) -> str:
    """The arithmetic type of the step's dominant work: the product's operand
    type where the step has a product (TF32 for the 1:2 product on fp32 W),
    else the element type the masks and compressors read."""
    if kind == "pairs":
        return "tf32"
    return {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32", torch.int8: "s8"}[wl["W"].dtype]


def profiled_traffic(workload: str, kernel: str):
    import hashlib
    rel = TRAFFIC_PROFILES.get((workload, kernel))
    if rel is None or not os.path.exists(os.path.join(ROOT, rel)):
        return None
    fields = {}
    with open(os.path.join(ROOT, rel)) as f:
        for line in f:
            if ":" in line and line.split(":")[0] in ("traffic_bytes_per_launch", "source_sha256", "source_file"):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    try:
        with open(os.path.join(ROOT, fields["source_file"]), "rb") as fh:
            src = fh.read()
        if hashlib.sha256(src).hexdigest() != fields["source_sha256"]:
            return None
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, OSError, ValueError):
        return None


# ----------------------------------------------------------------- workloads
def make_workload(name: str):
    """-> dict(W, X, R, K, T, desc) with CPU tensors."""
    if name == "linear_4096":
        W, X = nm_inputs.linear_4096()
        desc = "transformer linear: bf16 W 4096x4096 ~N(0,0.02) 2:4 along K; X bf16 4096x4096 ~N(0,1)"
    elif name.startswith("decode_T"):
        T = int(name[len("decode_T"):])
        W, X = nm_inputs.decode_skinny_W(), nm_inputs.decode_skinny_X(T)
        desc = "decode-like skinny: bf16 W 28672x8192 ~N(0,0.02) 2:4; X bf16 8192x%d ~N(0,1)" % T
    elif name == "mlp_pair":
        W_up, W_down, X = nm_inputs.mlp_pair()
        return {"W": W_up, "W2": W_down, "X": X, "R": W_up.shape[0], "K": W_up.shape[1], "T": X.shape[1],
                "desc": "MLP pair: bf16 W_up 14336x4096, W_down 4096x14336 ~N(0,0.02) 2:4; X bf16 4096x8192 ~N(0,1);"
                        " up then down"}
    elif name == "srste":
        W, _ = nm_inputs.linear_4096()
        return {"W": W, "G": nm_inputs.srste_grad(), "X": None, "R": 4096, "K": 4096, "T": 0,
                "desc": "SR-STE step: bf16 W 4096x4096 ~N(0,0.02) and bf16 gradient ~N(0,1e-3); 2:4, decay 0.0002"}
    elif name == "saliency_mask":
        W = nm_inputs.decode_skinny_W()
        return {"W": W, "D": nm_inputs.saliency_d(W.shape[1]), "X": None, "R": W.shape[0], "K": W.shape[1], "T": 0,
                "desc": "saliency-scored 2:4 mask: bf16 W 28672x8192 ~N(0,0.02); d = diag of the upper Cholesky factor"
                        " of the inverse of a damped synthetic Gram matrix (512 calibration rows ~N(0,1))"}
    elif name == "int8_24":
        W = nm_inputs.int8_decode()
        X = nm_inputs.decode_X_int8(1024)
        return {"W": W, "I8": True, "X": X, "R": W.shape[0], "K": W.shape[1], "T": X.shape[1],
                "desc": "int8 2:4: the 28672x8192 decode weight quantised to int8, X its 8192x1024 activations"
                        " quantised to int8; mask 2:4, fused mask+compress, .kind::i8 image, decompress, int8"
                        " sparse product with exact int32 output"}
    elif name == "pairs_12":
        W = nm_inputs.fp32_linear()
        X = nm_inputs.fp32_linear_X(4096)
        return {"W": W, "P12": True, "X": X, "R": W.shape[0], "K": W.shape[1], "T": X.shape[1],
                "desc": "1:2 pattern (sparse TF32): fp32 W 8192x8192 ~N(0,0.02), X fp32 8192x4096 ~N(0,1); mask 1:2,"
                        " compress under it, fused mask+compress, .kind::tf32 image, decompress, TF32 sparse product"}
    elif name == "transposable_mask":
        W, _ = nm_inputs.linear_4096()
        return {"W": W, "TM": (4, 8), "X": None, "R": 4096, "K": 4096, "T": 0,
                "desc": "greedy transposable 4:8 mask over 8x8 blocks: bf16 W 4096x4096 ~N(0,0.02)"}
    elif name == "transposable_24":
        W, X = nm_inputs.linear_4096()
        return {"W": W, "X": X, "DY": nm_inputs.linear_4096_grad(), "T24": True, "R": 4096, "K": 4096, "T": 4096,
                "desc": "transposable 2:4 training step of the transformer linear: bf16 W 4096x4096 ~N(0,0.02), "
                        "X 4096x4096 and dY 4096x4096 ~N(0,1); greedy transposable 2:4 mask (4x4 blocks), "
                        "compress W and W^T under it, Y = W X and dX = W^T dY on the sparse tensor cores"}
    elif name == "ties_mask":
        W = nm_inputs.ties_fp32()
        return {"W": W, "X": None, "R": 8192, "K": 8192, "T": 0,
                "desc": "mask-only: fp32 W 8192x8192 = k/100, k ~ U{-8..7}; 1:4, 2:4, 4:8, 2:8"}
    else:
        raise SystemExit("unknown workload " + name)
    return {"W": W, "X": X, "R": W.shape[0], "K": W.shape[1], "T": X.shape[1], "desc": desc}


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", "nm_clocks_%d_%d.csv" % (os.getpid(), index))

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            if getattr(self, "fh", None) is not None:
                self.fh.close()
        self.t0 = time.time()

    def mark(self, what: str):
        setattr(self, what, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        import datetime
        sm, smax, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t_lo = getattr(self, "t_begin", 0.0) - 0.05
        t_hi = getattr(self, "t_end", 1e30) + 0.05
        samples = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    samples.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        inside = [x for x in samples if t_lo <= x[0] <= t_hi]
        if not inside and samples:   # region shorter than the sampling period: nearest sample
            mid = 0.5 * (t_lo + t_hi)
            inside = [min(samples, key=lambda x: abs(x[0] - mid))]
        for ts, mhz, mx, flags in inside:
            sm.append(mhz)
            smax = mx
            n += 1
            for name, v in zip(names, flags):
                if v.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": n}


# ----------------------------------------------------------------- GPU arm
def _dev_x(X: torch.Tensor, dev, mult: int = 8) -> torch.Tensor:
    """X on the device in a buffer whose rows are 16-byte aligned (mult elements)."""
    K, T = X.shape
    buf = torch.zeros((K, (T + mult - 1) // mult * mult), dtype=X.dtype, device=dev)
    buf[:, :T].copy_(X)
    return buf[:, :T]


class Step:
    """Device buffers and the launch sequence of one step of the path."""

    def __init__(self, nm, wl, dev):
        self.nm, self.wl, self.dev = nm, wl, dev
        R, K, T = wl["R"], wl["K"], wl["T"]
        self.kind = "srste" if "G" in wl else "scored" if "D" in wl else "transposable" if "TM" in wl else \
            "trans24" if "T24" in wl else \
            "pairs" if "P12" in wl else "int8" if "I8" in wl else \
            ("ties" if wl["X"] is None else ("mlp" if "W2" in wl else "linear"))
        self.W = wl["W"].to(dev)
        if self.kind == "int8":
            self.X = _dev_x(wl["X"], dev, 16)
            self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
            self.values, self.meta, _ = nm.alloc_compressed(R, K, self.W.dtype, dev, sm100=False)
            self.img = torch.empty((nm.nm_meta_s8_image_bytes(R, K),), dtype=torch.uint8, device=dev)
            self.Wd = torch.empty_like(self.W)
            self.Y = torch.empty((R, T), dtype=torch.int32, device=dev)
            G = R * K
            self.names = ["nm_mask_s8", "nm_mask_compress_s8", "nm_meta_to_sm100_s8", "nm_decompress_s8",
                          "nm_spmm_s8"]
            self.bytes = {"nm_mask_s8": G * 2, "nm_mask_compress_s8": G * (1 + 0.5 + 0.125),
                          "nm_meta_to_sm100_s8": G * 0.25, "nm_decompress_s8": G * (0.5 + 0.125 + 1),
                          "nm_spmm_s8": G * (0.5 + 0.125) + K * T + R * T * 4}
            self.flop_k = {"nm_spmm_s8": 2.0 * R * K * T}
            self.flops = self.flop_k["nm_spmm_s8"]
            return
        if self.kind == "pairs":
            self.X = _dev_x(wl["X"], dev, 4)
            self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
            self.v1, self.m1 = nm.alloc_compressed12(R, K, self.W.dtype, dev)
            self.v2, self.m2 = nm.alloc_compressed12(R, K, self.W.dtype, dev)
            self.img = torch.empty((nm.nm_meta12_image_bytes(R, K),), dtype=torch.uint8, device=dev)
            self.Wd = torch.empty_like(self.W)
            self.Y = torch.empty((R, T), dtype=torch.float32, device=dev)
            es = self.W.element_size()
            G = R * K
            self.names = ["nm_mask_1:2", "nm_compress12", "nm_mask_compress12", "nm_meta12_to_sm100",
                          "nm_decompress12", "nm_spmm12"]
            self.bytes = {"nm_mask_1:2": G * (es + 1), "nm_compress12": G * (es + 1 + es / 2 + 1 / 16),
                          "nm_mask_compress12": G * (es + es / 2 + 1 / 16), "nm_meta12_to_sm100": G * (1 / 16 + 1 / 8),
                          "nm_decompress12": G * (es / 2 + 1 / 16 + es),
                          "nm_spmm12": G * (es / 2 + 1 / 8) + K * T * es + R * T * 4}
            self.flop_k = {"nm_spmm12": 2.0 * R * K * T}
            self.flops = self.flop_k["nm_spmm12"]
            return
        if self.kind == "transposable":
            self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
            self.names = ["nm_mask_transposable"]
            self.bytes = {"nm_mask_transposable": R * K * (self.W.element_size() + 1)}
            self.flops = 0
            return
        if self.kind == "scored":
            self.D = wl["D"].to(dev)
            self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
            self.names = ["nm_mask_scored"]
            self.bytes = {"nm_mask_scored": R * K * (self.W.element_size() + 1) + K * 4}
            self.flops = 0
            return
        if self.kind == "srste":
            self.G = wl["G"].to(dev)
            self.WS = torch.empty_like(self.W)
            self.GO = torch.empty_like(self.W)
            self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
            self.names = ["nm_srste_step"]
            es = self.W.element_size()
            self.bytes = {"nm_srste_step": R * K * (4 * es + 1)}
            self.flops = 0
            return
        if self.kind == "ties":
            self.masks = [torch.empty((R, K), dtype=torch.uint8, device=dev) for _ in range(4)]
            self.names = ["nm_mask_1:4", "nm_mask_2:4", "nm_mask_4:8", "nm_mask_2:8"]
            G = R * K
            self.bytes = {n: G * (4 + 1) for n in self.names}
            self.flops = 0
            return
        self.X = _dev_x(wl["X"], dev)
        v, m, img = nm.alloc_compressed(R, K, self.W.dtype, dev)
        self.values, self.meta, self.img = v, m, img
        if self.kind == "trans24":
            self.DY = _dev_x(wl["DY"], dev)
            self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
            self.v_t, self.m_t, self.img_t = nm.alloc_compressed(K, R, self.W.dtype, dev)
            self.Y = torch.empty((R, T), dtype=torch.bfloat16, device=dev)
            self.DX = torch.empty((K, T), dtype=torch.bfloat16, device=dev)
            # the two products run concurrently in the captured step: one scratch buffer each
            ws_f = nm.nm_spmm_workspace_bytes(self.W.dtype, R, K, T)
            ws_b = nm.nm_spmm_workspace_bytes(self.W.dtype, K, R, T)
            self.ws = torch.empty((ws_f,), dtype=torch.uint8, device=dev) if ws_f else None
            self.ws_t = torch.empty((ws_b,), dtype=torch.uint8, device=dev) if ws_b else None
            self.names = ["nm_mask_transposable_2:4", "nm_compress", "nm_compress_t", "nm_spmm_fwd", "nm_spmm_bwd"]
            G = R * K
            es = self.W.element_size()
            self.bytes = {"nm_mask_transposable_2:4": G * (es + 1), "nm_compress": G * (es + 1 + es / 2 + 0.25),
                          "nm_compress_t": G * (es + 1 + es / 2 + 0.25),
                          "nm_spmm_fwd": G * (es / 2 + 0.125) + K * T * es + R * T * 2,
                          "nm_spmm_bwd": G * (es / 2 + 0.125) + R * T * es + K * T * 2}
            self.flop_k = {"nm_spmm_fwd": 2.0 * R * K * T, "nm_spmm_bwd": 2.0 * R * K * T}
            self.flops = sum(self.flop_k.values())
            return
        if self.kind == "mlp":
            # every row of the path on both weights, then the two products
            self.W2 = wl["W2"].to(dev)
            R2, K2 = self.W2.shape
            es = self.W.element_size()
            self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
            self.mask2 = torch.empty((R2, K2), dtype=torch.uint8, device=dev)
            self.v_c, self.m_c, self.img_c = nm.alloc_compressed(R, K, self.W.dtype, dev)
            self.v2_c, self.m2_c, self.img2_c = nm.alloc_compressed(R2, K2, self.W2.dtype, dev)
            self.v2, self.m2, self.img2 = nm.alloc_compressed(R2, K2, self.W2.dtype, dev)
            self.img_r = torch.empty_like(self.img)
            self.img2_r = torch.empty_like(self.img2)
            self.Wd = torch.empty_like(self.W)
            self.W2d = torch.empty_like(self.W2)
            Tp = (T + 7) // 8 * 8
            self.gather = wl.get("gather")
            self.fused = self.gather is not None and wl.get("gather_mode") == "fused"
            if self.gather is None:
                self.H = torch.empty((R, Tp), dtype=torch.bfloat16, device=dev)[:, :T]
                self.H_down = self.H
            elif self.fused:
                self._init_fused_gather(nm, wl, Tp, dev)
            else:
                # the up product writes this rank's rows into a slice-sized buffer; the
                # all-gather assembles every rank's rows; the down product reads them all
                dist_, per, R_full = self.gather
                world_ = dist_.get_world_size()
                self.H_local = torch.zeros((per, Tp), dtype=torch.bfloat16, device=dev)
                self.H_all = torch.empty((world_ * per, Tp), dtype=torch.bfloat16, device=dev)
                self.H = self.H_local[:R, :T]
                self.H_down = self.H_all[:R_full, :T]
            self.Y = torch.empty((R2, T), dtype=torch.bfloat16, device=dev)
            ws = max(nm.nm_spmm_workspace_bytes(self.W.dtype, R, K, T),
                     nm.nm_spmm_workspace_bytes(self.W2.dtype, R2, K2, T))
            # the two products run one after the other (down reads H), so they may share scratch
            self.ws = torch.empty((ws,), dtype=torch.uint8, device=dev) if ws else None
            self.names, self.bytes = [], {}
            for tag, G in (("up", R * K), ("down", R2 * K2)):
                self.names += ["nm_mask_" + tag, "nm_compress_" + tag, "nm_mask_compress_" + tag,
                               "nm_meta_to_sm100_" + tag, "nm_decompress_" + tag]
                self.bytes.update({"nm_mask_" + tag: G * (es + 1), "nm_compress_" + tag: G * (es + 1 + es / 2 + 0.25),
                                   "nm_mask_compress_" + tag: G * (es + es / 2 + 0.25),
                                   "nm_meta_to_sm100_" + tag: G * 0.25,
                                   "nm_decompress_" + tag: G * (es / 2 + 0.125 + es)})
            exchange = (["peer_signal", "peer_wait"] if self.fused else ["all_gather_H"]) if self.gather else []
            self.names += ["nm_spmm_up"] + exchange + ["nm_spmm_down"]
            n_dest = len(self.peer_H[0]) if self.fused else 1     # the up product's output copies
            self.bytes.update({"nm_spmm_up": R * K * (es / 2 + 0.125) + K * T * es + n_dest * R * T * 2,
                               "nm_spmm_down": R2 * K2 * (es / 2 + 0.125) + K2 * T * es + R2 * T * 2})
            if self.fused:
                self.bytes.update({"peer_signal": 8 * n_dest, "peer_wait": 8 * n_dest})
            elif self.gather:
                self.bytes["all_gather_H"] = self.H_all.numel() * self.H_all.element_size()
            self.flop_k = {"nm_spmm_up": 2.0 * R * K * T, "nm_spmm_down": 2.0 * R2 * K2 * T}
            self.flops = sum(self.flop_k.values())
            return
        self.mask = torch.empty((R, K), dtype=torch.uint8, device=dev)
        self.v_c, self.m_c, self.img_c = nm.alloc_compressed(R, K, self.W.dtype, dev)
        self.img_r = torch.empty_like(self.img)
        self.Wd = torch.empty_like(self.W)
        self.Y = torch.empty((R, T), dtype=torch.bfloat16, device=dev)
        ws = nm.nm_spmm_workspace_bytes(self.W.dtype, R, K, T)
        self.ws = torch.empty((max(ws, 1),), dtype=torch.uint8, device=dev) if ws else None
        self.names = ["nm_mask", "nm_compress", "nm_mask_compress", "nm_meta_to_sm100", "nm_decompress", "nm_spmm"]
        G = R * K
        es = self.W.element_size()
        self.bytes = {"nm_mask": G * (es + 1), "nm_compress": G * (es + 1 + es / 2 + 0.25),
                      "nm_mask_compress": G * (es + es / 2 + 0.25), "nm_meta_to_sm100": G * 0.25,
                      "nm_decompress": G * (es / 2 + 0.125 + es),
                      "nm_spmm": G * (es / 2 + 0.125) + K * T * es + R * T * 2}
        self.flop_k = {"nm_spmm": 2.0 * R * K * T}
        self.flops = self.flop_k["nm_spmm"]

    def _init_fused_gather(self, nm, wl, Tp, dev):
        """The exchange of the row-split MLP pair without a collective library:
        every rank's up product stores its rows of H straight into every rank's
        H (nm_spmm_peers over CUDA IPC mappings), raises its flag on every rank
        (nm_peer_signal) and waits for all flags (nm_peer_wait) before the down
        product.  H is double-buffered by step parity: a rank that runs ahead
        writes step s+1's rows into the buffer its peers last read at step s-1,
        which they finished before signalling step s."""
        dist_, per, R_full = self.gather
        world_, rank_ = dist_.get_world_size(), dist_.get_rank()
        T = wl["T"]
        self.rank, self.epoch, self.row0, self.ldh = rank_, 0, wl["rows"][0], Tp
        self.H_bufs = [torch.zeros((world_ * per, Tp), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.flags = torch.zeros(world_, dtype=torch.int64, device=dev)
        mine = [nm.nm_ipc_handle(t) for t in (self.H_bufs[0], self.H_bufs[1], self.flags)]
        if self.flags.is_cuda:
            torch.cuda.synchronize()              # zeroed before any peer can write
        every = [None] * world_
        dist_.all_gather_object(every, mine)
        self.peer_H, self.peer_F = [[], []], []
        for j in range(world_):
            if j == rank_:
                self.peer_H[0].append(self.H_bufs[0])
                self.peer_H[1].append(self.H_bufs[1])
                self.peer_F.append(self.flags)
                continue
            addrs = []
            for h, off in every[j]:
                addrs.append(nm.nm_ipc_open(h, off))
                IPC_MAPPINGS.append((addrs[-1], off))
            self.peer_H[0].append(addrs[0])
            self.peer_H[1].append(addrs[1])
            self.peer_F.append(addrs[2])
        self.H = self.H_bufs[0][self.row0:self.row0 + wl["R"], :T]
        self.H_down = self.H_bufs[0][:R_full, :T]
        dist_.barrier()                           # every rank has mapped every buffer

    def _up_fused(self):
        nm = self.nm
        self.epoch += 1
        b = self.epoch % 2
        R_full, T = self.gather[2], self.wl["T"]
        self.H_down = self.H_bufs[b][:R_full, :T]
        nm.nm_spmm_peers(self.values, self.img, self.X, self.peer_H[b], self.row0, self.ldh)

    def launches(self):
        return len(self.names)

    def own_launches(self):
        """Launches of the library's own kernels per step (a collective library's are not counted)."""
        return len([n for n in self.names if n != "all_gather_H"])

    def calls(self):
        """The step's launches, in the order of self.names, as zero-argument callables."""
        nm = self.nm
        if self.kind == "srste":
            return [lambda: nm.nm_srste_step(self.W, self.G, 2, 4, 0.0002, W_sparse=self.WS, grad_out=self.GO,
                                             mask=self.mask)]
        if self.kind == "scored":
            return [lambda: nm.nm_mask_scored(self.W, self.D, 2, 4, mask=self.mask)]
        if self.kind == "transposable":
            return [lambda: nm.nm_mask_transposable(self.W, *self.wl["TM"], mask=self.mask)]
        if self.kind == "int8":
            R, K = self.wl["R"], self.wl["K"]
            return [lambda: nm.nm_mask(self.W, 2, 4, mask=self.mask),
                    lambda: nm.nm_mask_compress(self.W, self.values, self.meta, None, sm100=False),
                    lambda: nm.nm_meta_to_sm100_s8(self.meta, R, K, out=self.img),
                    lambda: nm.nm_decompress(self.values, self.meta, K, out=self.Wd),
                    lambda: nm.nm_spmm(self.values, self.img, self.X, Y=self.Y)]
        if self.kind == "pairs":
            R, K = self.wl["R"], self.wl["K"]
            return [lambda: nm.nm_mask(self.W, 1, 2, mask=self.mask),
                    lambda: nm.nm_compress12(self.W, self.mask, self.v1, self.m1),
                    lambda: nm.nm_mask_compress12(self.W, self.v2, self.m2),
                    lambda: nm.nm_meta12_to_sm100(self.m2, R, K, out=self.img),
                    lambda: nm.nm_decompress12(self.v2, self.m2, K, out=self.Wd),
                    lambda: nm.nm_spmm12(self.v2, self.img, self.X, Y=self.Y)]
        if self.kind == "ties":
            return [(lambda i=i, N=N, M=M: nm.nm_mask(self.W, N, M, mask=self.masks[i]))
                    for i, (N, M) in enumerate([(1, 4), (2, 4), (4, 8), (2, 8)])]
        if self.kind == "trans24":
            return [lambda: nm.nm_mask_transposable(self.W, 2, 4, mask=self.mask),
                    lambda: nm.nm_compress(self.W, self.mask, self.values, self.meta, self.img),
                    lambda: nm.nm_compress_t(self.W, self.mask, self.v_t, self.m_t, self.img_t),
                    lambda: nm.nm_spmm(self.values, self.img, self.X, Y=self.Y, workspace=self.ws),
                    lambda: nm.nm_spmm(self.v_t, self.img_t, self.DY, Y=self.DX, workspace=self.ws_t)]
        if self.kind == "mlp":
            K, K2 = self.wl["K"], self.W2.shape[1]
            R, R2 = self.wl["R"], self.W2.shape[0]
            return [lambda: nm.nm_mask(self.W, 2, 4, mask=self.mask),
                    lambda: nm.nm_compress(self.W, self.mask, self.v_c, self.m_c, self.img_c),
                    lambda: nm.nm_mask_compress(self.W, self.values, self.meta, self.img),
                    lambda: nm.nm_meta_to_sm100(self.meta, R, K, out=self.img_r),
                    lambda: nm.nm_decompress(self.values, self.meta, K, out=self.Wd),
                    lambda: nm.nm_mask(self.W2, 2, 4, mask=self.mask2),
                    lambda: nm.nm_compress(self.W2, self.mask2, self.v2_c, self.m2_c, self.img2_c),
                    lambda: nm.nm_mask_compress(self.W2, self.v2, self.m2, self.img2),
                    lambda: nm.nm_meta_to_sm100(self.m2, R2, K2, out=self.img2_r),
                    lambda: nm.nm_decompress(self.v2, self.m2, K2, out=self.W2d)] + \
                ([self._up_fused,
                  lambda: nm.nm_peer_signal(self.peer_F, self.rank, self.epoch),
                  lambda: nm.nm_peer_wait(self.flags, self.epoch, timeout_ns=PEER_WAIT_NS)] if self.fused else
                 [lambda: nm.nm_spmm(self.values, self.img, self.X, Y=self.H, workspace=self.ws)] +
                 ([lambda: gather_rows(self.gather[0], self.H_all, self.H_local)] if self.gather else [])) + \
                [lambda: nm.nm_spmm(self.v2, self.img2, self.H_down, Y=self.Y, workspace=self.ws)]
        K = self.wl["K"]
        return [lambda: nm.nm_mask(self.W, 2, 4, mask=self.mask),
                lambda: nm.nm_compress(self.W, self.mask, self.v_c, self.m_c, self.img_c),
                lambda: nm.nm_mask_compress(self.W, self.values, self.meta, self.img),
                lambda: nm.nm_meta_to_sm100(self.meta, self.wl["R"], K, out=self.img_r),
                lambda: nm.nm_decompress(self.values, self.meta, K, out=self.Wd),
                lambda: nm.nm_spmm(self.values, self.img, self.X, Y=self.Y, workspace=self.ws)]

    def run(self):
        for fn in self.calls():
            fn()

    def deps(self):
        """For each launch of calls(), the earlier launches whose outputs it reads."""
        n = self.launches()
        if self.kind == "linear":     # mask -> compress; fused -> {image, decompress, product}
            return [[], [0], [], [2], [2], [2]]
        if self.kind == "mlp":        # per weight: mask -> compress; fused -> {image, decompress}; then
            #                               up product after the fused up call, down after fused down and up
            #                               (split by rows: up -> all-gather of H -> down)
            if self.fused:            # up (peer stores) -> signal -> wait -> down
                return [[], [0], [], [2], [2], [], [5], [], [7], [7], [2], [10], [11], [7, 12]]
            if self.gather:
                return [[], [0], [], [2], [2], [], [5], [], [7], [7], [2], [10], [7, 11]]
            return [[], [0], [], [2], [2], [], [5], [], [7], [7], [2], [7, 10]]
        if self.kind == "trans24":    # mask -> {compress -> forward, compress_t -> backward}
            return [[], [0], [0], [1], [2]]
        if self.kind == "ties":       # four masks of the same W
            return [[] for _ in range(n)]
        if self.kind == "int8":       # mask; fused -> {image -> product, decompress}
            return [[], [], [1], [1], [1, 2]]
        if self.kind == "pairs":      # mask -> compress; fused -> {image -> product, decompress}
            return [[], [0], [], [2], [2], [2, 3]]
        return [[i - 1] if i else [] for i in range(n)]

    def capture(self):
        """CUDA graphs captured once after warm-up: the whole step as its
        dependency graph (a launch waits only for the launches whose outputs it
        reads; independent chains run on forked streams), the same step as one
        sequential chain, and each launch alone.  Replaying them issues the same
        kernels with the same arguments without the host's per-launch latency."""
        calls, deps = self.calls(), self.deps()
        pool = [torch.cuda.Stream() for _ in range(4)]
        dag = torch.cuda.CUDAGraph()
        with torch.cuda.graph(dag):
            cap = torch.cuda.current_stream()
            start = torch.cuda.Event()
            start.record(cap)
            done, where, last_on, used = [None] * len(calls), [None] * len(calls), {}, []
            for i, fn in enumerate(calls):
                # continue a dependency's chain when it is the last launch on its stream
                st = next((where[j] for j in deps[i] if last_on.get(where[j]) == j), None)
                if st is None:
                    st = next(k for k in range(len(pool)) if k not in last_on or k == len(pool) - 1)
                stream = pool[st]
                if st not in used:
                    stream.wait_event(start)
                    used.append(st)
                for j in deps[i]:
                    if where[j] != st:
                        stream.wait_event(done[j])
                with torch.cuda.stream(stream):
                    fn()
                    ev = torch.cuda.Event()
                    ev.record(stream)
                done[i], where[i], last_on[st] = ev, st, i
            for st in used:
                cap.wait_event(done[last_on[st]])
        seq = torch.cuda.CUDAGraph()
        with torch.cuda.graph(seq):
            for fn in calls:
                fn()
        per = []
        for fn in calls:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            per.append(g)
        torch.cuda.synchronize()
        return dag, per, seq

    def result(self):
        if self.kind == "srste":
            return self.GO
        if self.kind in ("scored", "transposable"):
            return self.mask
        if self.kind == "trans24":
            return self.DX
        return self.masks[1] if self.kind == "ties" else self.Y


class L2Flush:
    """Evicts L2 between timed iterations, outside the events: a 256 MiB write
    (twice the L2) and then a 256 MiB read of a second buffer.  The read pushes
    the written lines out (their write-back happens here, not in the next timed
    kernel) and leaves L2 holding clean, unrelated lines, so the timed work
    starts cold and pays only for its own traffic."""

    def __init__(self, dev):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(32 << 20, dtype=torch.int64, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def timed_steps(step: Step, steps: int, flush, graphs=None):
    """-> per-step ms over exactly `steps` steps (graph replays when captured)."""
    s = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()                            # evict L2 between steps (outside the events)
        ev[i][0].record(s)
        if graphs is not None:
            graphs[0].replay()
        else:
            step.run()
        ev[i][1].record(s)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def kernel_breakdown(step: Step, steps: int, flush, graphs=None):
    """-> per-kernel ms lists: each launch of the step timed on its own, L2
    flushed before every launch (outside its events), so every kernel starts
    cold and its figure counts only its own traffic."""
    s = torch.cuda.current_stream()
    n = step.launches()
    calls = step.calls()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
          for _ in range(steps)]
    for i in range(steps):
        for j in range(n):
            flush()
            ev[i][j][0].record(s)
            if graphs is not None:
                graphs[1][j].replay()
            else:
                calls[j]()
            ev[i][j][1].record(s)
    torch.cuda.synchronize()
    return {name: [ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(steps)] for j, name in enumerate(step.names)}


def event_floor_us(reps: int, flush) -> float:
    """Context for the per-kernel figures: the median CUDA-event time of a
    one-element torch kernel, timed the way each launch is (L2 flushed before,
    outside the events).  A tiny launch cannot read below this."""
    s = torch.cuda.current_stream()
    t = torch.empty(1, dtype=torch.int32, device=s.device)
    ts = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        t.zero_()
        b.record(s)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return 1e3 * float(np.median(ts))


def dense_context(step: Step, reps: int, flush):
    """Context only: the same products as dense bf16 GEMMs in cuBLAS (torch.matmul)
    on the decompressed weights, timed like the step (L2 flushed before each rep).
    -> {name: ms} for the product launches of the step, or None."""
    if step.kind not in ("linear", "mlp", "trans24", "int8", "pairs"):
        return None
    nm = step.nm
    s = torch.cuda.current_stream()
    mm = torch.matmul
    if step.kind == "int8":          # cuBLAS int8 GEMM with int32 output
        Wd = nm.nm_decompress(step.values, step.meta, step.wl["K"])
        jobs = {"nm_spmm_s8": (Wd, step.X.contiguous())}
        mm = torch._int_mm
    elif step.kind == "pairs":       # cuBLAS fp32 GEMM on the TF32 tensor cores
        Wd = nm.nm_decompress12(step.v2, step.m2, step.wl["K"])
        jobs = {"nm_spmm12": (Wd, step.X.contiguous())}
    elif step.kind == "linear":
        Wd = nm.nm_decompress(step.values, step.meta, step.wl["K"])
        jobs = {"nm_spmm": (Wd, step.X)}
    elif step.kind == "trans24":
        Wd = nm.nm_decompress(step.values, step.meta, step.wl["K"])
        jobs = {"nm_spmm_fwd": (Wd, step.X), "nm_spmm_bwd": (Wd.t().contiguous(), step.DY)}
    else:
        Wu = nm.nm_decompress(step.values, step.meta, step.wl["K"])
        Wdn = nm.nm_decompress(step.v2, step.m2, step.W2.shape[1])
        jobs = {"nm_spmm_up": (Wu, step.X), "nm_spmm_down": (Wdn, step.H_down)}
    out = {}
    tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = step.kind == "pairs"
    try:
        for name, (A, B) in jobs.items():
            cdt = torch.int32 if step.kind == "int8" else (torch.float32 if step.kind == "pairs" else torch.bfloat16)
            C = torch.empty((A.shape[0], B.shape[1]), dtype=cdt, device=A.device)
            for _ in range(3):
                mm(A, B, out=C)
            ts = []
            for _ in range(reps):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(s)
                mm(A, B, out=C)
                b.record(s)
                b.synchronize()
                ts.append(a.elapsed_time(b))
            out[name] = float(np.median(ts))
    finally:
        torch.backends.cuda.matmul.allow_tf32 = tf32
    return out


def e2e_steps(step: Step, steps: int, nm, wl, dev):
    """The step through the public API with host buffers, pipelined over two
    replicas of the device buffers: step i+1's inputs copy in (pinned H2D on
    one stream) while step i runs (the public calls, on a second stream) and
    step i-1's result copies out (D2H on a third).  Every step copies all of
    its inputs in and its result out.
    -> (device ms of the whole run, H2D bytes per step, D2H bytes per step)"""
    reps = [step, Step(nm, wl, dev)]
    names = [k for k in ("W", "X", "W2", "G", "D", "DY") if wl.get(k) is not None]
    host = {k: wl[k].pin_memory() for k in names}
    outs = [torch.empty(r.result().shape, dtype=r.result().dtype).pin_memory() for r in reps]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = outs[0].numel() * outs[0].element_size()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in reps]
    ev_run = [torch.cuda.Event() for _ in reps]
    ev_out = [torch.cuda.Event() for _ in reps]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(s_in)
    for i in range(steps):
        b = i % 2
        r = reps[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_run[b])       # step i-2 has finished reading these inputs
            for k in names:
                getattr(r, k).copy_(host[k], non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[b])
            if i >= 2:
                s_run.wait_event(ev_out[b])      # step i-2's result has been copied out
            r.run()
            ev_run[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[b])
            outs[b].copy_(r.result(), non_blocking=True)
            ev_out[b].record(s_out)
    end.record(s_out)                            # after the last copy-out, which follows everything
    torch.cuda.synchronize()
    return start.elapsed_time(end), h2d, d2h


# ----------------------------------------------------------------- CPU oracle (baseline / reference arm)
def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_step(wl, rows: int, threads: int):
    """The oracle doing the step's work on the first `rows` rows of W.
    -> (seconds, units) with units in the metric's unit (dense-eq flops or bytes)."""
    import oracle
    if "G" in wl:                 # SR-STE step
        Wb = _u16(wl["W"][:rows].contiguous())
        Gb = _u16(wl["G"][:rows].contiguous())
        t0 = time.perf_counter()
        oracle.srste(Wb, Gb, 2, 4, 0.0002, dtype=oracle.BF16)
        return time.perf_counter() - t0, float(rows * wl["K"] * 9)
    if "T24" in wl:               # transposable 2:4 training step (whole 4-row blocks)
        rows = max(4, rows - rows % 8)
        Wb = _u16(wl["W"][:rows].contiguous())
        X, DY = _u16(wl["X"]), _u16(wl["DY"][:rows].contiguous())
        t0 = time.perf_counter()
        mask = oracle.mask_transposable(Wb, 2, 4, dtype=oracle.BF16)
        v, m = oracle.compress24(Wb, mask, dtype=oracle.BF16)
        vt, mt = oracle.compress24(np.ascontiguousarray(Wb.T), np.ascontiguousarray(mask.T), dtype=oracle.BF16)
        oracle.spmm(v, m, X, oracle.BF16, threads=threads)                  # Y rows = W rows . X
        oracle.spmm(vt, mt, DY, oracle.BF16, threads=threads)               # dX = W^T dY over those rows
        return time.perf_counter() - t0, 2 * 2.0 * rows * wl["K"] * wl["T"]
    if "TM" in wl:                # transposable mask (whole M-row blocks)
        rows = max(wl["TM"][1], rows - rows % wl["TM"][1])
        Wb = _u16(wl["W"][:rows].contiguous())
        t0 = time.perf_counter()
        oracle.mask_transposable(Wb, *wl["TM"], dtype=oracle.BF16)
        return time.perf_counter() - t0, float(rows * wl["K"] * 3)
    if "I8" in wl:                # int8 2:4 with its product
        W = wl["W"][:rows].contiguous().numpy()
        X = wl["X"].numpy()
        t0 = time.perf_counter()
        mask = oracle.mask_rank(W, 2, 4)
        v, m = oracle.compress24(W, mask)
        oracle.meta_sm100_s8(m, rows, wl["K"])
        oracle.decompress24(v, m, wl["K"])
        oracle.spmm(v, m, X, oracle.S8, threads=threads)
        return time.perf_counter() - t0, 2.0 * rows * wl["K"] * wl["T"]
    if "P12" in wl:               # 1:2 family on fp32 with the TF32 product
        W = wl["W"][:rows].contiguous().numpy()
        X = wl["X"].numpy()
        t0 = time.perf_counter()
        mask = oracle.mask_rank(W, 1, 2)
        oracle.compress12(W, mask)
        v, m = oracle.compress12(W, mask)
        oracle.meta12_sm100(m, rows, wl["K"])
        oracle.decompress12(v, m, wl["K"])
        oracle.spmm12(v, m, X, threads=threads)
        return time.perf_counter() - t0, 2.0 * rows * wl["K"] * wl["T"]
    if "D" in wl:                 # saliency-scored mask
        Wb = _u16(wl["W"][:rows].contiguous())
        d = wl["D"].numpy()
        t0 = time.perf_counter()
        oracle.mask_scored(Wb, d, 2, 4, dtype=oracle.BF16)
        return time.perf_counter() - t0, float(rows * wl["K"] * 3)
    if wl["X"] is None:           # mask-only workload
        W = wl["W"][:rows].contiguous().numpy()
        t0 = time.perf_counter()
        for N, M in [(1, 4), (2, 4), (4, 8), (2, 8)]:
            oracle.rows_parallel(0, W, N, M, oracle.F32, threads)
        return time.perf_counter() - t0, 4.0 * rows * W.shape[1] * 5
    code = oracle.BF16
    X = _u16(wl["X"])
    K, T = wl["K"], wl["T"]

    def six_calls(Wfull, Kw):
        """mask, compress under it, fused mask+compress, image, decompress on the
        first `rows` rows of one weight -> (values, meta) of the fused call"""
        Wb = _u16(Wfull[:rows].contiguous())
        mask, _, _ = oracle.rows_parallel(0, Wb, 2, 4, code, threads)
        oracle.compress24(Wb, mask, dtype=code)
        _, values, meta = oracle.rows_parallel(1, Wb, 2, 4, code, threads)
        oracle.meta_sm100(meta, rows, Kw)
        oracle.decompress24(values, meta, Kw, dtype=code)
        return values, meta

    t0 = time.perf_counter()
    values, meta = six_calls(wl["W"], K)
    oracle.spmm(values, meta, X, code, threads=threads)                     # product
    units = 2.0 * rows * K * T
    if "W2" in wl:
        # the same rows of W_down, then its product; its input H (W_up's output,
        # 14336 x T) is a zero stand-in of that shape, which costs the oracle the same
        K2 = wl["W2"].shape[1]
        v2, m2 = six_calls(wl["W2"], K2)
        H = np.zeros((K2, T), dtype=np.uint16)
        oracle.spmm(v2, m2, H, code, threads=threads)
        units += 2.0 * rows * K2 * T
    return time.perf_counter() - t0, units


def size_oracle_sample(wl, threads: int, target_s: float):
    """Rows of W whose oracle step takes about target_s seconds (probe on 8 rows)."""
    probe = 8
    t, _ = oracle_step(wl, probe, threads)
    per_row = max(t / probe, 1e-6)
    rows = int(max(probe, min(wl["R"], target_s / per_row)))
    return rows


def cpu_baseline(wl, target_s: float = 15.0):
    threads = os.cpu_count() or 1
    rows = size_oracle_sample(wl, threads, target_s)
    secs, units = oracle_step(wl, rows, threads)
    scale, unit = ((1e12, "TOP/s" if "I8" in wl else "TFLOP/s") if wl["X"] is not None else (1e9, "GB/s"))
    what = ("SR-STE step (mask, masked weight, decay gradient)" if "G" in wl else
            "saliency-scored 2:4 mask" if "D" in wl else
            "greedy transposable 4:8 mask" if "TM" in wl else
            "transposable 2:4 mask, compress W and W^T, fp64 forward and backward products" if "T24" in wl else
            "1:2 mask, compress, fused compress, image, decompress, fp64 1:2 product" if "P12" in wl else
            "int8 2:4 mask, compress, image, decompress, exact int8 product" if "I8" in wl else
            "mask at 1:4, 2:4, 4:8, 2:8" if wl["X"] is None else
            "whole step on the sampled rows of both weights (mask, compress, fused mask+compress, image, "
            "decompress, fp64 product; the down product's input is a zero stand-in of H's shape)" if "W2" in wl else
            "whole step (mask, compress, fused mask+compress, image, decompress, fp64 product)")
    return {"value": units / secs / scale, "unit": unit, "cores": threads, "kind": "oracle",
            "sample": "first %d of %d rows of W, %s, %.1f s" % (rows, wl["R"], what, secs)}


def run_reference(args, wl, metric):
    """The oracle as it stands on the host cores, `steps` bounded samples."""
    threads = os.cpu_count() or 1
    per_step_s = max(0.5, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    rows = size_oracle_sample(wl, threads, per_step_s)
    for _ in range(args.warmup):
        oracle_step(wl, rows, threads)
    tot_s, tot_u = 0.0, 0.0
    for _ in range(args.steps):
        s, u = oracle_step(wl, rows, threads)
        tot_s += s
        tot_u += u
    scale, unit = ((1e12, "TOP/s" if "I8" in wl else "TFLOP/s") if wl["X"] is not None else (1e9, "GB/s"))
    value = tot_u / tot_s / scale
    sample = "first %d of %d rows of W per step, whole step on the CPU oracle" % (rows, wl["R"])
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "data": "synthetic",
            # the oracle's arithmetic: fp64 product, binary32 decay term / scores, integer magnitude keys
            "dtype": ("int64" if "I8" in wl else "f64") if wl["X"] is not None else
                     ("f32" if ("G" in wl or "D" in wl) else "u32"),
            "config": {"workload": args.workload, "desc": wl["desc"], "R": wl["R"], "K": wl["K"], "T": wl["T"]},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- main
METRIC = "nm_spmm dense-equiv TFLOP/s + mask/compress GB/s, % of B200 roofline"


def max_over_ranks(pg, values, device):
    """Element-wise maximum of a list of floats over every rank of the process
    group (the slowest rank's time is the job's time); identity without one."""
    if pg is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def shard_rows(R: int, world: int, rank: int, align: int = 256):
    """Rows [lo, hi) of an R-row weight that `rank` holds when the rows are split
    over `world` ranks in slices of one common size `per` (a multiple of `align`,
    so every slice is whole CTA-pair tiles); the last slices may be short or
    empty.  -> (lo, hi, per)"""
    per = -(-R // world)
    per = -(-per // align) * align
    lo = min(R, rank * per)
    return lo, min(R, lo + per), per


def gather_rows(dist, out: torch.Tensor, local: torch.Tensor):
    """All-gather of equal row slices: rank i's `local` (per x T) lands in rows
    [i*per, (i+1)*per) of `out` (world*per x T) on every rank.  NCCL gathers into
    the tensor directly; other backends (gloo, in the CPU tests) through a list."""
    if dist.get_backend() == "nccl":
        dist.all_gather_into_tensor(out, local)
    else:
        parts = list(out.split(local.shape[0]))
        dist.all_gather(parts, local.contiguous())
        for dst, src in zip(out.split(local.shape[0]), parts):
            if dst.data_ptr() != src.data_ptr():
                dst.copy_(src)


def split_workload(wl, world: int, rank: int, dist, gather: str = "nccl"):
    """The rank's share of a product workload split by output rows: its rows of
    W (and of W_down for the MLP pair), all of X.  The MLP pair's hidden
    activation H = W_up X is row-split too and gathered on every rank before
    the down product, the path's one exchange: an NCCL all-gather ("nccl"), or
    the up product's own stores into every rank's H followed by completion
    flags ("fused").  The transformer linear needs none."""
    lo, hi, per = shard_rows(wl["R"], world, rank)
    out = dict(wl)
    out["W"] = wl["W"][lo:hi]
    out["R"] = hi - lo
    out["rows"] = (lo, hi)
    if "W2" in wl:
        R2 = wl["W2"].shape[0]
        lo2, hi2, _ = shard_rows(R2, world, rank)
        out["W2"] = wl["W2"][lo2:hi2]
        out["rows2"] = (lo2, hi2)
        out["gather"] = (dist, per, wl["R"])       # H slices of `per` rows, R_up rows in all
        out["gather_mode"] = gather
    return out


def whole_job_rate(world: int, units_per_step: float, steps: int, ms: float, scale: float) -> float:
    """Units every rank processed (each rank runs the full step) per second,
    divided by `scale` (1e12 for TFLOP/s, 1e9 for GB/s)."""
    return world * units_per_step * steps / (ms * 1e-3) / scale


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)       # the MLP-pair workload's 20 timed repetitions
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="nm", choices=["nm", "reference"])
    ap.add_argument("--workload", default="mlp_pair")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", default="replicas", choices=["replicas", "rows"],
                    help="N > 1: an independent replica of the workload per GPU (weak scaling), or one problem "
                         "split by output rows over the GPUs (strong scaling; linear_4096 and mlp_pair)")
    ap.add_argument("--gather", default="nccl", choices=["nccl", "fused"],
                    help="--split rows, mlp_pair: assemble H with an NCCL all-gather, or by the up product's "
                         "own stores into every GPU's H (CUDA IPC) and completion flags")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, make_workload(args.workload), METRIC)
        return

    warmup = max(3, args.warmup)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    import structured_sparsity_prune_b200 as nm
    nm.load()                                    # fails loudly without the CUDA library
    wl_full = make_workload(args.workload)
    split = args.split == "rows" and world > 1
    if split and args.workload not in ("linear_4096", "mlp_pair"):
        raise SystemExit("--split rows applies to the product workloads linear_4096 and mlp_pair")
    if args.gather == "fused" and not (split and args.workload == "mlp_pair"):
        raise SystemExit("--gather fused applies to --split rows of mlp_pair on more than one GPU")
    wl = split_workload(wl_full, world, rank, pg, args.gather) if split else wl_full
    step = Step(nm, wl, dev)
    # work of the whole job per step: every rank's replica, or the one split problem
    full_flops = 2.0 * wl_full["R"] * wl_full["K"] * wl_full["T"] + \
        (2.0 * wl_full["W2"].shape[0] * wl_full["W2"].shape[1] * wl_full["T"] if "W2" in wl_full else 0.0)
    flush = L2Flush(dev)

    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    if nm.nm_last_device_status() != 0:
        raise SystemExit("device status reports a timed-out wait")
    try:
        if split:   # the all-gather stays outside CUDA graphs: the split step is timed as eager launches
            raise RuntimeError("row-split step with a collective, timed eagerly")
        eager = step.result().clone()
        graphs = step.capture()
        launch_mode = ("CUDA graph of the step as its dependency graph (independent launches on forked "
                       "streams), captured once after warm-up and replayed")
        for g in (graphs[0], graphs[2]):
            for _ in range(warmup):
                g.replay()
            torch.cuda.synchronize()
            if not torch.equal(step.result(), eager):
                raise SystemExit("graph replay of the step differs from the eager step")
    except SystemExit:
        raise
    except Exception as exc:   # capture unavailable: time eager launches instead
        graphs = None
        launch_mode = "eager launches (graph capture failed: %s)" % str(exc).splitlines()[0][:120]

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.5)                              # let the sampler start emitting
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    clocks.mark("t_begin")
    tot = timed_steps(step, args.steps, flush, graphs)
    torch.cuda.synchronize()
    clocks.mark("t_end")
    if pg:
        pg.barrier()
    clk = clocks.stop()
    per = kernel_breakdown(step, args.steps, flush, graphs)
    # the same step as one sequential chain, for comparison (not the timed region)
    seq_ms = float(np.mean(timed_steps(step, args.steps, flush, (graphs[2],) if graphs else None)))
    floor_us = event_floor_us(50, flush)

    total_ms = float(np.sum(tot))
    e2e_ms, h2d, d2h = e2e_steps(step, args.steps, nm, wl, dev)
    total_ms, e2e_ms = max_over_ranks(pg, [total_ms, e2e_ms], dev)
    if nm.nm_last_device_status() != 0:
        raise SystemExit("device status reports a timed-out wait")

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    # Tensor peak: the dense burst figure for kernels that ran at full clock;
    # the sustained (power-capped) figure when the clock record of the timed
    # region shows the power cap, i.e. the kernels ran inside a long, capped step.
    capped = "sw_power_cap" in (clk.get("reasons") or [])
    dense_key = "bf16_tflops_sustained" if capped and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    sparse_peak = float(peaks[dense_key]) * SPARSE_RATIO
    kernels = {}
    for name in step.names:
        ms = float(np.mean(per[name]))
        k = {"us": 1e3 * ms, "GB/s": step.bytes[name] / (ms * 1e-3) / 1e9,
             "hbm_frac": step.bytes[name] / (ms * 1e-3) / 1e9 / hbm}
        if hasattr(step, "flop_k") and name in step.flop_k:
            tf = step.flop_k[name] / (ms * 1e-3) / 1e12
            k.update({"TFLOP/s": tf, "tensor_frac": tf / sparse_peak})
        kernels[name] = k

    if step.kind in ("ties", "srste", "scored", "transposable"):
        units_per_step = sum(step.bytes.values())
        value = whole_job_rate(world, units_per_step, args.steps, total_ms, 1e9)
        unit = "GB/s"
        dom = {"ties": "nm_mask_2:4", "srste": "nm_srste_step", "scored": "nm_mask_scored",
               "transposable": "nm_mask_transposable"}[step.kind]
        if step.kind == "transposable":
            N_, M_ = wl["TM"]
            ops = transposable_int_ops(M_) * (wl["R"] // M_) * (wl["K"] // M_)
            tops = ops / (kernels[dom]["us"] * 1e-6) / 1e12
            roof = {"bound": "alu", "achieved": tops, "peak": ALU_PEAK_TOPS, "unit": "Tint-op/s",
                    "frac": tops / ALU_PEAK_TOPS, "kernel": dom, "algorithmic_int_ops_per_launch": ops,
                    "algorithmic_bytes_per_launch": step.bytes[dom], "achieved_GB/s": kernels[dom]["GB/s"]}
        else:
            roof = {"bound": "hbm", "achieved": kernels[dom]["GB/s"], "peak": hbm, "unit": "GB/s",
                    "frac": kernels[dom]["GB/s"] / hbm, "kernel": dom,
                    "algorithmic_bytes_per_launch": step.bytes[dom]}
        e2e_value = whole_job_rate(world, units_per_step, args.steps, e2e_ms, 1e9)
    else:
        value = (full_flops * args.steps / (total_ms * 1e-3) / 1e12 if split
                 else whole_job_rate(world, step.flops, args.steps, total_ms, 1e12))
        unit = "TOP/s" if step.kind == "int8" else "TFLOP/s"
        dom = max(step.flop_k, key=lambda n: np.mean(per[n]))
        # the product's own tensor peak: 2:4 (or 1:2) sparse = 2 x dense of its
        # operand type; int8 and tf32 dense taken as the measured bf16 figure
        # times the nominal B200 ratios (int8 2x, tf32 0.5x bf16)
        ratio = KIND_RATIO.get(step.kind, 1.0)
        peak = sparse_peak * ratio
        roof = {"bound": "tensor", "achieved": kernels[dom]["TFLOP/s"], "peak": peak, "unit": unit,
                "frac": kernels[dom]["TFLOP/s"] / peak, "kernel": dom,
                "algorithmic_flops_per_launch": step.flop_k[dom]}
        kernels[dom]["tensor_frac"] = kernels[dom]["TFLOP/s"] / peak
        e2e_value = (full_flops * args.steps / (e2e_ms * 1e-3) / 1e12 if split
                     else whole_job_rate(world, step.flops, args.steps, e2e_ms, 1e12))
    roof["peak_source"] = ("%s: 2 x dense bf16 %s%s" % (peak_src, "sustained (power cap seen in the timed region)"
                                                        if dense_key.endswith("sustained") else "burst",
                                                        KIND_NOTE.get(step.kind, ""))
                           if roof["bound"] == "tensor" else
                           "derived: 148 SMs x 64 integer lanes x 1965 MHz" if roof["bound"] == "alu" else
                           "%s: HBM copy" % peak_src)
    # the committed DRAM counters were taken on the whole problem on one GPU
    roof["traffic"] = None if split else profiled_traffic(args.workload, dom)

    dense = dense_context(step, 20, flush)
    dense_line = None
    if dense:
        dense_line = {"what": "context only: the dense cuBLAS GEMM of the same operand type on decompress(W) "
                              "(bf16 torch.matmul; int8 torch._int_mm; fp32 torch.matmul on the TF32 tensor cores), "
                              "same shapes, L2 flushed, median of 20",
                      "kernels": {}}
        for name, ms in dense.items():
            tf = step.flop_k[name] / (ms * 1e-3) / 1e12
            dense_line["kernels"][name] = {"dense_us": 1e3 * ms, "dense_TFLOP/s": tf,
                                           "sparse_over_dense_speedup": ms / float(np.mean(per[name]))}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
                "warmup": warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "strong" if split else "weak", "vs_baseline": None,
                "dtype": compute_dtype(wl, step.kind),
                "data": "synthetic",
                "config": {"workload": args.workload, "desc": wl["desc"], "R": wl_full["R"], "K": wl["K"], "T": wl["T"],
                           "sparsity": {"ties": "N:M along K (1:4, 2:4, 4:8, 2:8)", "pairs": "1:2 along K",
                                        "transposable": "4:8 transposable (8x8 blocks)",
                                        "trans24": "2:4 transposable (4x4 blocks)"}.get(step.kind, "2:4 along K"),
                           "l2": "flushed between timed steps, outside the events: a 256 MiB write, then a 256 MiB read "
                                 "that evicts the written lines",
                           "launch": launch_mode,
                           "step_sequential_ms": seq_ms,
                           "event_floor_us": floor_us,
                           "parallelism": ("rows of W split over the GPUs, X replicated%s" %
                                           ((", H gathered by the up product's stores into every GPU's H "
                                             "(CUDA IPC) and completion flags before the down product"
                                             if args.gather == "fused" else
                                             ", H all-gathered (NCCL) before the down product")
                                            if step.kind == "mlp" else ", no exchange")) if split else
                                          ("independent replica per GPU" if world > 1 else "single GPU")},
                "roofline": roof, "cpu_baseline": cpu, "dense_context": dense_line,
                "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                        "method": "public calls with pinned host buffers; H2D, step and D2H of consecutive steps "
                                  "overlapped on three streams over two buffer replicas"},
                "gpu_launches": step.own_launches() * args.steps,
                "clocks": clk, "kernels": kernels}
        print(json.dumps(line), flush=True)
    if pg:
        torch.cuda.synchronize()
        pg.barrier()                # no rank's kernels touch another GPU's buffers any more
        while IPC_MAPPINGS:
            nm.nm_ipc_close(*IPC_MAPPINGS.pop())
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
