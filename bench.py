"""Benchmark: one BitNet a4.8 decoder layer's BitLinear forward path, 7B shapes.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--afmt int4|fp4]

A step is one pass of the whole hot path over one batch of M = 8 x 4096 tokens
(hidden 4096, 32 heads x 128, FFN 11008), all on the GPU through the C ABI:

  pack_ternary x5      latent fp32 W -> ternary int8 operand + alpha (Eq. 2),
                       re-ternarized every pass as in the paper's forward
  quant_a4(X_attn)     INT4 absmean (Eq. 6-7) or FP4 E2M1 (Eq. 8-9)
  gemm  QKV            [M x 4096] x [12288 x 4096]^T
  kv_quant3  K, V      3-bit post-RoPE KV, position 0 at 4 bits
  sparsify_a8(X_o)     Top-K 50% + INT8 (Eq. 1)
  gemm  O              [M x 4096] x [4096 x 4096]^T
  quant_a4(X_ffn)
  gemm  Up|Gate        [M x 4096] x [22016 x 4096]^T, one alpha per tensor
  relu2_glu            up * relu(gate)^2 (Eq. 5) + Top-K 50% + INT8
  gemm  Down           [M x 11008] x [4096 x 11008]^T

Attention itself is outside the path; its output (the O-projection input) is a
seeded heavy-tailed tensor.  Inputs are seeded synthetic data larger than L2.
With --gpus N (torchrun) every rank runs an independent replica on its own
tokens (weak scaling, no data-path collective); the time is the max over ranks.

--impl reference times the CPU oracle on the host (rank 0 only) on a bounded
token sample of the same workload, scaled to tokens/s.
"""
from __future__ import annotations

import argparse
import functools
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "BitLinear GEMM TOPS & tokens/s (7B layer shapes) vs B200 INT8/FP4 peak; quant GB/s"
SHAPE = synth.L7B
EPS = 1e-5
# measured B200 peaks of this machine (generated file), else the documented fallback
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
INT8_PER_BF16 = 2.0   # nominal dense int8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
FP4_PER_BF16 = 4.0    # nominal dense fp4 : bf16 (9 : 2.25 PFLOP/s)
# DRAM bytes (read + write) of one launch of each of the step's four GEMM shapes at
# 16384 tokens (`--profile-case gemm / gemm_o / gemm_upgate / gemm_down`, ncu
# dram__bytes_read.sum + dram__bytes_write.sum, second launch), doubled for the
# step's 32768 tokens: A and Y grow with the token count, the 202 MB of weights do
# not, so the doubling overstates by at most 0.2 GB.  Algorithmic bytes of the same
# launches at 32768 tokens: 3.75 GB (A and W read once, Y written once).
GEMM_TRAFFIC_16K = {"qkv": 269529088 + 358346496, "o": 103798016 + 91663360,
                    "upgate": 436135936 + 679412736, "down": 627190016 + 121038336}
GEMM_STEP_DRAM_BYTES = 2 * sum(GEMM_TRAFFIC_16K.values())


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def workload_config(afmt: str, m: int):
    s = SHAPE
    return {
        "workload": f"BitNet a4.8 7B-shape decoder layer, BitLinear forward, prefill 8x4096 tokens",
        "hidden": s.hidden, "heads": s.heads, "head_dim": s.head_dim, "ffn": s.ffn, "tokens_per_gpu": m,
        "activations": ("INT4 absmean" if afmt == "int4" else "FP4 E2M1 MinMax") +
                       " for QKV/Up/Gate inputs; Top-K 50% + INT8 for O and Down inputs",
        "weights": "ternary, re-quantized from fp32 latent weights every step",
        "kv_cache": "3-bit, BOS position at 4 bits",
        "l2": "inputs larger than L2 (each activation tensor 268 MB)",
    }


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.bus_id:
            cmd.insert(1, f"--id={self.bus_id}")
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.reader.join(timeout=2)
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
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# multi-rank timing: every rank runs its own replica; the job's time is the
# slowest rank's, and the job's throughput counts every rank's tokens
# ---------------------------------------------------------------------------
def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (a collective used for timing only)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_throughput(world: int, tokens_per_rank: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (elapsed_ms / 1e3)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
class Layer:
    """Device buffers and the launch sequence of one layer step."""

    def __init__(self, torch, tba, dev, m: int, afmt: str, seed: int):
        self.torch, self.tba, self.dev = torch, tba, dev
        s = SHAPE
        d, f, H, Dh = s.hidden, s.ffn, s.heads, s.head_dim
        self.m, self.d, self.f, self.H, self.Dh = m, d, f, H, Dh
        self.afmt = afmt
        T = torch
        u8, i8, f32, i16, i32 = T.uint8, T.int8, T.float32, T.int16, T.int32

        def dev_from(a):
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:
                a = a.view(np.int16)
            return T.from_numpy(a).to(dev)

        # latent weights (fp32, resident) and their ternary int8 operands
        wts = synth.layer_weights(SHAPE, seed=3)
        self.w_lat = {k: dev_from(v) for k, v in wts.items()}
        del wts
        # QKV and Up|Gate take the INT4 inputs' int8 operand, or with FP4 inputs E2M1-coded weights
        # (kind::mxf4 GEMM); O and Down always take the Top-K INT8 inputs and int8 weights
        fp4 = afmt == "fp4"
        kq = d // 2 if fp4 else d
        self.wfmt_q = tba.BL_W_E2M1 if fp4 else tba.BL_W_I8
        self.afmt_q = tba.BL_A_E2M1 if fp4 else tba.BL_A_I8
        self.store_q = tba.BL_STORE_PACKED if fp4 else tba.BL_STORE_BYTES
        self.w8 = {"qkv": T.empty((3 * d, kq), dtype=u8, device=dev), "o": T.empty((d, d), dtype=u8, device=dev),
                   "upgate": T.empty((2 * f, kq), dtype=u8, device=dev), "down": T.empty((d, f), dtype=u8, device=dev)}
        self.alpha = T.zeros((8,), dtype=f32, device=dev)   # qkv, o, up, gate, down
        self.ws = T.empty((tba.workspace_size("pack_ternary") // 8,), dtype=T.int64, device=dev)

        # activations: host copies (pinned, for the end-to-end leg) and device copies
        x_attn, x_o, x_ffn = synth.layer_activations(SHAPE, seed=seed, tokens=m)
        self.h_in = [T.from_numpy(a.view(np.int16)).pin_memory() for a in (x_attn, x_o, x_ffn)]
        del x_attn, x_o, x_ffn
        # two device sets of the step's inputs and outputs, so the end-to-end
        # leg can copy one step's data while another step computes
        self.x_sets = [[h.to(dev) for h in self.h_in] for _ in range(2)]
        self.x = self.x_sets[0]

        # BL_STORE_BYTES: one int8 per element; FP4: packed E2M1 nibbles
        self.qa = T.empty((m, kq), dtype=u8, device=dev)
        self.qa_s = T.empty((m,), dtype=f32, device=dev)
        self.qf = T.empty((m, kq), dtype=u8, device=dev)
        self.qf_s = T.empty((m,), dtype=f32, device=dev)
        self.o8 = T.empty((m, d), dtype=i8, device=dev)
        self.o8_s = T.empty((m,), dtype=f32, device=dev)
        self.h8 = T.empty((m, f), dtype=i8, device=dev)
        self.h8_s = T.empty((m,), dtype=f32, device=dev)
        self.y_qkv = T.empty((m, 3 * d), dtype=i16, device=dev)
        self.y_ug = T.empty((m, 2 * f), dtype=i16, device=dev)
        self.out_sets = []
        for _ in range(2):
            self.out_sets.append([T.empty((m, d), dtype=i16, device=dev),                 # O projection output
                                  T.empty((m, d), dtype=i16, device=dev),                 # down projection output
                                  T.empty((2, m, H, Dh * 3 // 8), dtype=u8, device=dev),  # 3-bit K and V codes
                                  T.empty((2, m, H), dtype=f32, device=dev),              # their scales
                                  T.empty((2, H, Dh // 2), dtype=u8, device=dev)])        # 4-bit BOS rows
        self.use_set(0)
        self.h_out = [T.empty(o.shape, dtype=o.dtype).pin_memory() for o in self.outputs]

        # algorithmic work per step
        N_K = {"qkv": (3 * d, d), "o": (d, d), "upgate": (2 * f, d), "down": (d, f)}
        self.gemm_ops = {k: 2.0 * m * n * kk for k, (n, kk) in N_K.items()}
        self.weights = sum(n * kk for n, kk in N_K.values())
        # kernels of this library per step: exact-sum + pack for each of the five weight
        # tensors (each call also enqueues a 2 KiB workspace memset, not counted), two
        # quantizers, four GEMMs, two KV quantizers, sparsify, ReLU^2-GLU
        self.launches_per_step = 5 * 2 + 2 + 4 + 2 + 1 + 1

    def alg_gemm_ops(self):
        """2 N nnz(A) per step: QKV and Up|Gate dense, O and Down with the
        Top-K survivors (k_keep of K per token)."""
        m, d, f = self.m, self.d, self.f
        keep_o, keep_d = synth.k_keep(d, SHAPE.topk_pct_o), synth.k_keep(f, SHAPE.topk_pct_down)
        return (self.gemm_ops["qkv"] + self.gemm_ops["upgate"] + 2.0 * m * d * keep_o + 2.0 * m * d * keep_d)

    # kernel-by-kernel bytes each launch must move (algorithmic, per the formulas
    # of the path: read inputs once, write outputs once)
    def kernel_bytes(self):
        m, d, f, H, Dh = self.m, self.d, self.f, self.H, self.Dh
        kv_one = m * H * (2 * Dh + Dh * 3 // 8 + 4)
        fp4 = self.afmt == "fp4"
        qout = m * d // 2 if fp4 else m * d
        wq = 4.5 if fp4 else 5      # fp32 read + E2M1 nibble or int8 written per weight
        return {
            "quant_a4": 2 * (m * d * 2 + qout + 4 * m),
            "sparsify_a8": m * d * 2 + m * d + 4 * m,
            "relu2_glu": m * f * 4 + m * f + 4 * m,
            "kv_quant3": 2 * kv_one,
            "pack_ternary": int(sum(n * kk * c for (n, kk), c in [((3 * d, d), wq), ((d, d), 5), ((2 * f, d), wq),
                                                                  ((d, f), 5)])),
        }

    def step(self, ev=None):
        """Enqueue one step on the current stream; ev (optional) collects
        (name, start_event, end_event) around every library call."""
        tba, T = self.tba, self.torch
        d, f, m, H, Dh = self.d, self.f, self.m, self.H, self.Dh
        fp4 = self.afmt == "fp4"

        def timed(name, fn):
            if ev is None:
                fn()
                return
            a = T.cuda.Event(enable_timing=True)
            b = T.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            ev.append((name, a, b))

        W, w8, al = self.w_lat, self.w8, self.alpha
        ws = self.ws
        wq, aq, sq = self.wfmt_q, self.afmt_q, self.store_q
        timed("pack_ternary", lambda: tba.pack_ternary(W["qkv"], al[0:1], w8["qkv"], wq, ws, eps=EPS))
        timed("pack_ternary", lambda: tba.pack_ternary(W["o"], al[1:2], w8["o"], tba.BL_W_I8, ws, eps=EPS))
        timed("pack_ternary", lambda: tba.pack_ternary(W["up"], al[2:3], w8["upgate"][:f], wq, ws, eps=EPS))
        timed("pack_ternary", lambda: tba.pack_ternary(W["gate"], al[3:4], w8["upgate"][f:], wq, ws, eps=EPS))
        timed("pack_ternary", lambda: tba.pack_ternary(W["down"], al[4:5], w8["down"], tba.BL_W_I8, ws, eps=EPS))
        q = tba.BL_QUANT_FP4_E2M1 if fp4 else tba.BL_QUANT_INT4
        x_attn, x_o, x_ffn = self.x
        # attention block
        timed("quant_a4", lambda: tba.bitlinear_quant_a4(x_attn, self.qa, self.qa_s, q, sq, EPS))
        timed("gemm_qkv", lambda: tba.bitlinear_gemm(self.qa, self.qa_s, w8["qkv"], al[0:1], m, 3 * d, d,
                                                     y=self.y_qkv, afmt=aq, wfmt=wq))
        for i, off in enumerate((d, 2 * d)):     # K and V slices of the QKV output
            timed("kv_quant3", lambda off=off, i=i: tba.kv_quant3(self.y_qkv[:, off:], m, H, Dh, self.kv_codes[i],
                                                                  self.kv_scale[i], self.kv_bos[i], bits=3,
                                                                  bos_pos=0, eps=EPS, ldt=3 * d))
        timed("sparsify_a8", lambda: tba.bitlinear_sparsify_a8(x_o, synth.k_keep(d, SHAPE.topk_pct_o), self.o8,
                                                               self.o8_s, None, EPS))
        timed("gemm_o", lambda: tba.bitlinear_gemm(self.o8, self.o8_s, w8["o"], al[1:2], m, d, d, y=self.y_o))
        # FFN block
        timed("quant_a4", lambda: tba.bitlinear_quant_a4(x_ffn, self.qf, self.qf_s, q, sq, EPS))
        timed("gemm_upgate", lambda: tba.bitlinear_gemm(self.qf, self.qf_s, w8["upgate"], al[2:4], m, 2 * f, d,
                                                        y=self.y_ug, alpha_group=f, afmt=aq, wfmt=wq))
        timed("relu2_glu", lambda: tba.relu2_glu(self.y_ug[:, f:], self.y_ug[:, :f],
                                                 synth.k_keep(f, SHAPE.topk_pct_down), self.h8, self.h8_s, None,
                                                 EPS, M=m, F=f, ld=2 * f))
        timed("gemm_down", lambda: tba.bitlinear_gemm(self.h8, self.h8_s, w8["down"], al[4:5], m, d, f,
                                                      y=self.y_down))

    def use_set(self, i: int):
        """Point the step at input/output buffer set i."""
        self.x = self.x_sets[i]
        self.outputs = self.out_sets[i]
        self.y_o, self.y_down, self.kv_codes, self.kv_scale, self.kv_bos = self.outputs

    def h2d(self):
        for h, dv in zip(self.h_in, self.x):
            dv.copy_(h, non_blocking=True)

    def d2h(self):
        for o, h in zip(self.outputs, self.h_out):
            h.copy_(o, non_blocking=True)

    def run_e2e(self, steps: int):
        """`steps` end-to-end steps: per step, H2D of the inputs from pinned host
        memory, the step, D2H of the outputs.  Copies run on their own streams
        and overlap the neighbouring steps' compute; buffer sets alternate, and
        events keep each set's copy-in, compute and copy-out in order.
        Returns (start_event, end_event)."""
        T = self.torch
        comp = T.cuda.current_stream()
        s_in = T.cuda.Stream()
        s_out = T.cuda.Stream()
        ev = lambda: T.cuda.Event()
        inputs_free = [ev(), ev()]     # compute finished reading set i's inputs
        inputs_ready = [ev(), ev()]
        outputs_ready = [ev(), ev()]
        outputs_free = [ev(), ev()]    # set i's outputs copied out
        start = T.cuda.Event(enable_timing=True)
        end = T.cuda.Event(enable_timing=True)
        for e in inputs_free + outputs_free:
            e.record(comp)
        start.record(comp)
        s_in.wait_event(start)
        for i in range(steps):
            p = i & 1
            self.use_set(p)
            with T.cuda.stream(s_in):
                s_in.wait_event(inputs_free[p])
                self.h2d()
                inputs_ready[p].record(s_in)
            comp.wait_event(inputs_ready[p])
            comp.wait_event(outputs_free[p])
            self.step()
            inputs_free[p].record(comp)
            outputs_ready[p].record(comp)
            with T.cuda.stream(s_out):
                s_out.wait_event(outputs_ready[p])
                self.d2h()
                outputs_free[p].record(s_out)
        comp.wait_stream(s_out)
        end.record(comp)
        self.use_set(0)
        return start, end

    def io_bytes(self):
        return (sum(h.numel() * h.element_size() for h in self.h_in),
                sum(h.numel() * h.element_size() for h in self.h_out))


def zero_fractions(torch, layer) -> dict:
    """Per projection, the fraction of zero codes in its quantized input after
    the last step, and the fraction of gate pre-activations that ReLU^2 zeroes:
    the sparsity the paper tabulates per projection (here of synthetic data)."""
    def frac(is_zero):
        return round(float(is_zero.sum().item()) / is_zero.numel(), 4)
    out = {"o_input": frac(layer.o8 == 0), "down_input": frac(layer.h8 == 0),
           "gate_relu_zero": frac(layer.y_ug[:, layer.f:].view(torch.bfloat16) <= 0)}
    # what a sparse Down GEMM could skip: K columns that are zero in every row of a
    # 128-row tile (the tensor-core GEMM's M tile), and groups of four codes with
    # more than two nonzeros (which break the 2:4 pattern of a structured-sparse MMA)
    nz = layer.h8 != 0
    rows = (nz.shape[0] // 128) * 128
    if rows:
        tile_any = nz[:rows].view(rows // 128, 128, nz.shape[1]).any(dim=1)
        out["down_all_zero_k_columns_per_128_rows"] = frac(~tile_any)
    if nz.shape[1] % 4 == 0:
        out["down_groups_over_2of4"] = frac(nz.view(nz.shape[0], -1, 4).sum(dim=-1) > 2)
    del nz
    if layer.afmt == "int4":   # byte layout: one code per byte
        out["qkv_input"] = frac(layer.qa == 0)
        out["upgate_input"] = frac(layer.qf == 0)
    return out


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import ternary_bit_activation_b200 as tba

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    distributed = world > 1
    if distributed:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    tba.lib()
    m = SHAPE.tokens
    layer = Layer(torch, tba, dev, m, args.afmt, seed=SHAPE.tokens + 17 * rank)
    tba.sync_status()

    def barrier():
        if distributed:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        layer.step()
    tba.sync_status()

    props = torch.cuda.get_device_properties(dev)
    bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    clocks = ClockSampler(bus)
    clocks.start()
    time.sleep(0.3)
    events = []
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        layer.step(events)
    t1.record()
    barrier()
    clk = clocks.stop()
    tba.sync_status()
    elapsed_ms = t0.elapsed_time(t1)
    per_kernel = {}
    for name, a, b in events:
        per_kernel.setdefault(name, []).append(a.elapsed_time(b))

    # end to end through the C ABI with host buffers: every step copies its
    # inputs in from pinned host memory and its outputs back out
    layer.run_e2e(max(2, args.warmup))
    barrier()
    e0, e1 = layer.run_e2e(args.steps)
    barrier()
    e2e_ms = e0.elapsed_time(e1)

    if distributed:
        elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], dev)

    if rank == 0:
        peaks = load_peaks()
        ms_step = elapsed_ms / args.steps
        value = weak_scaling_throughput(world, m, args.steps, elapsed_ms)
        gemm_names = [k for k in per_kernel if k.startswith("gemm_")]
        gemm_ms = sum(sum(per_kernel[k]) for k in gemm_names)
        gemm_ops = sum(layer.gemm_ops[k[5:]] for k in gemm_names) * args.steps
        tops = gemm_ops / (gemm_ms / 1e3) / 1e12
        # burst peak when the SM clock held its maximum through the timed region (a
        # step of a few ms stays below the power cap), else the sustained one
        burst = (clk.get("sm_mhz") or 0) >= 0.95 * (clk.get("sm_max_mhz") or 1e9)
        basis = "bf16_tflops" if burst else "bf16_tflops_sustained"
        peak_int8 = peaks[basis] * INT8_PER_BF16
        if args.afmt == "fp4":
            # QKV and Up|Gate run as kind::mxf4 (nominal dense fp4 = 2 x int8): the step's peak is
            # the ops-weighted harmonic combination of the two rates
            ops_f4 = layer.gemm_ops["qkv"] + layer.gemm_ops["upgate"]
            ops_i8 = layer.gemm_ops["o"] + layer.gemm_ops["down"]
            peak_int8 = (ops_f4 + ops_i8) / (ops_f4 / (2 * peak_int8) + ops_i8 / peak_int8)
        kb = layer.kernel_bytes()
        kernels = {}
        for k, v in per_kernel.items():
            per_step = sum(v) / args.steps
            entry = {"ms_per_step": round(per_step, 4), "launches_per_step": len(v) // args.steps}
            if k.startswith("gemm_"):
                entry["tops_dense"] = round(layer.gemm_ops[k[5:]] / (per_step / 1e3) / 1e12, 1)
            elif k in kb:
                entry["gbs"] = round(kb[k] / (per_step / 1e3) / 1e9, 1)
                entry["hbm_frac"] = round(entry["gbs"] / peaks["hbm_gbs"], 3)
            kernels[k] = entry
        # algorithmic ops: 2 N nnz(A) -- the INT4 / FP4 inputs are dense, the
        # Top-K inputs of O and Down keep k_keep of their K values per token
        alg_ops = layer.alg_gemm_ops() * args.steps
        alg_tops = alg_ops / (gemm_ms / 1e3) / 1e12
        h2d, d2h = layer.io_bytes()
        line = {
            "metric": METRIC,
            "value": round(value, 1),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "int8" if args.afmt == "int4" else "fp4(e2m1)+int8",
            "data": "synthetic (seeded; Gaussian QKV/FFN inputs, Student-t nu=3 O input, N(0,0.02) latent weights)",
            "config": dict(workload_config(args.afmt, m), parallelism=f"replicas x{world}"),
            "roofline": {
                "bound": "tensor",
                "kernel": "gemm_tc2_kernel (tcgen05 kind::i8, CTA pairs)" if args.afmt == "int4" else
                          "gemm_tc2_kernel (tcgen05 kind::mxf4 for QKV/Up|Gate, kind::i8 for O/Down, CTA pairs)",
                "achieved": round(tops, 1),
                "peak": round(peak_int8, 1),
                "unit": "TFLOP/s",
                "frac": round(tops / peak_int8, 4),
                "achieved_algorithmic": round(alg_tops, 1),
                "frac_algorithmic": round(alg_tops / peak_int8, 4),
                "traffic": GEMM_STEP_DRAM_BYTES if args.afmt == "int4" else None,
                "traffic_note": "DRAM read+write bytes of the 4 GEMM shapes, each captured by ncu at 16384 "
                                "tokens (--profile-case) and doubled for the step's 32768 (the weights do not "
                                "double: overstates by <= 0.2e9); algorithmic 3.75e9",
                "peak_note": f"int8 = {INT8_PER_BF16:g} x {peaks['source']} {'burst' if burst else 'sustained'} "
                             f"bf16 cuBLAS ({peaks[basis]} TFLOP/s; nominal dense int8:bf16 ratio)" +
                             ("; fp4 = 2 x int8, combined by the ops of each kind" if args.afmt == "fp4" else ""),
                "work": "achieved / frac: dense-equivalent 2*M*N*K over the 4 GEMM launches of a step / their "
                        "summed event time; achieved_algorithmic / frac_algorithmic: 2*N*nnz(A), the O and Down "
                        "inputs counted with their k_keep survivors per token",
            },
            "gemm": {"tops_dense": round(tops, 1), "tops_algorithmic": round(alg_tops, 1),
                     "ms_per_step": round(gemm_ms / args.steps, 4)},
            # the same step with the ternary weights packed once beforehand (as at
            # inference): the step's time less its pack_ternary launches
            "value_weights_packed_once": round(weak_scaling_throughput(
                world, m, args.steps, elapsed_ms - sum(per_kernel.get("pack_ternary", []))), 1),
            "kernels": kernels,
            "e2e": {"value": round(world * m * args.steps / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms / args.steps, 4)},
            "gpu_launches": layer.launches_per_step * args.steps,
            "clocks": clk,
            "zero_fraction": zero_fractions(torch, layer),
        }
        if not args.no_extras and world == 1:
            # the decode sweep (7B shapes, 1-256 tokens) and the FP4 variant's two
            # GEMMs, on this GPU, after the timed regions
            dec = decode_sweep(torch, tba, dev, synth.DECODE_TOKENS, steps=20, warmup=3, w_lat=layer.w_lat,
                               variants=False)
            line["decode"] = {"unit": "us per layer",
                              "workload": f"M tokens through the BitLinear path (quantizers, Top-K, ReLU^2-GLU "
                                          f"and the four GEMMs on 2-bit weights) of {DECODE_LAYERS} 7B-shape layers "
                                          f"with their own weight buffers (together larger than L2); CUDA-graph "
                                          f"replay; hbm_frac_layer = weight bytes / layer time / HBM peak",
                              **dec}
            f4 = fp4_gemm_key(torch, tba, layer, reps=10)
            f4_peak = FP4_PER_BF16 * peaks[basis]
            for v in f4.values():
                v["frac"] = round(v["tops_dense"] / f4_peak, 4)
            line["fp4"] = {"unit": "TFLOP/s", "peak": round(f4_peak, 1),
                           "peak_note": f"fp4 = {FP4_PER_BF16:g} x {peaks['source']} "
                                        f"{'burst' if burst else 'sustained'} bf16 cuBLAS (nominal dense 9 : 2.25 "
                                        f"PFLOP/s)",
                           "workload": "QKV [32768 x 4096] x [12288 x 4096]^T and Up|Gate [32768 x 4096] x "
                                       "[22016 x 4096]^T, packed E2M1 activations x E2M1-coded ternary weights, "
                                       "tcgen05 kind::mxf4; median of 10 launches",
                           **f4}
            line["attention"] = attention_key(torch, tba, dev, peaks["hbm_gbs"])
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(args.afmt, args.cpu_tokens_per_core, args.cpu_tokens)
        print(json.dumps(line), flush=True)
    if distributed:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# CPU oracle arm
# ---------------------------------------------------------------------------
def host_cores() -> int:
    """Host CPU threads this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


@functools.lru_cache(maxsize=1)
def _oracle_weights():
    """The layer's latent weights for the CPU oracle, generated once."""
    return synth.layer_weights(SHAPE, seed=3)


def oracle_sample_seconds(afmt: str, tokens: int, threads: int = 1):
    """Time the CPU oracle over the same step on `tokens` rows: the ternary
    quantization of all latent weights (the five tensors side by side), then
    the per-token work (quantizers, the four products, ReLU^2-GLU, KV) with the
    token rows split over `threads` threads.  The oracle's loops are C called
    through ctypes, which releases the GIL, so the threads run in parallel.
    Returns (pack seconds, token seconds), wall clock; input generation is
    outside both."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    oracle.build()
    s = SHAPE
    d, f = s.hidden, s.ffn
    wts = _oracle_weights()
    x_attn, x_o, x_ffn = synth.layer_activations(s, seed=99, tokens=tokens)
    keep_o, keep_d = synth.k_keep(d, s.topk_pct_o), synth.k_keep(f, s.topk_pct_down)
    with ThreadPoolExecutor(max_workers=max(threads, 1)) as pool:
        t0 = time.perf_counter()
        packed = dict(zip(wts, pool.map(lambda w: oracle.ternary_quantize(w, EPS), wts.values())))
        t_pack = time.perf_counter() - t0
        tq = {k: v[0] for k, v in packed.items()}
        al = {k: v[1] for k, v in packed.items()}

        def quant4(x):
            if afmt == "fp4":
                _, q, _, sc = oracle.quant_fp4(x)
                return q, (sc / 2).astype(np.float32)
            q, _, sc = oracle.quant_int4(x, EPS)
            return q, sc

        def rows(sl):
            n = sl.stop - sl.start
            qa, s_a = quant4(x_attn[sl])
            _, y_qkv = oracle.gemm(qa, s_a, tq["qkv"], al["qkv"])
            kvin = np.ascontiguousarray(y_qkv[:, d:].reshape(n, 2, s.heads, s.head_dim).transpose(1, 0, 2, 3))
            for i in range(2):
                oracle.kv_quant(kvin[i], bits=3, bos_pos=0, eps=EPS)
            c8, _, _, s8 = oracle.sparsify_a8(x_o[sl], keep_o, EPS)
            oracle.gemm(c8, s8, tq["o"], al["o"])
            qf, s_f = quant4(x_ffn[sl])
            _, y_up = oracle.gemm(qf, s_f, tq["up"], al["up"])
            _, y_gate = oracle.gemm(qf, s_f, tq["gate"], al["gate"])
            h8, _, _, sh = oracle.relu2_glu(y_gate, y_up, keep_d, EPS)
            oracle.gemm(h8, sh, tq["down"], al["down"])

        bounds = np.linspace(0, tokens, max(threads, 1) + 1).astype(int)
        slices = [slice(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
        t0 = time.perf_counter()
        list(pool.map(rows, slices))
        t_tok = time.perf_counter() - t0
    return t_pack, t_tok


def cpu_baseline(afmt: str, tokens_per_core: int, one_core_tokens: int):
    """The oracle on all host cores (token rows split over one thread per core,
    the five weight tensors quantized side by side) and on one core, each over
    a bounded token sample scaled linearly to the step's token count."""
    m = SHAPE.tokens
    cores = host_cores()
    n_all = tokens_per_core * cores
    p_all, t_all = oracle_sample_seconds(afmt, n_all, threads=cores)
    p_one, t_one = oracle_sample_seconds(afmt, one_core_tokens, threads=1)
    v_all = m / (p_all + t_all * (m / n_all))
    v_one = m / (p_one + t_one * (m / one_core_tokens))
    return {"value": round(v_all, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "value_1core": round(v_one, 2),
            "sample": f"all cores: {n_all} tokens ({tokens_per_core} per thread, {cores} threads) of the 7B-shape "
                      f"layer through every step of the path, plus the ternary quantization of all 202M latent "
                      f"weights (five tensors side by side): pack {p_all:.2f} s, tokens {t_all:.2f} s wall; one "
                      f"core: {one_core_tokens} tokens, pack {p_one:.2f} s, tokens {t_one:.2f} s; per-token time "
                      f"scaled linearly to {m} tokens (extrapolated); C oracle via ctypes"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    m = SHAPE.tokens
    cores = host_cores()
    n_tok = args.cpu_tokens_ref * cores
    for _ in range(args.warmup):
        oracle_sample_seconds(args.afmt, n_tok, threads=cores)
    wall, full = 0.0, 0.0
    for _ in range(args.steps):
        t_pack, t_tok = oracle_sample_seconds(args.afmt, n_tok, threads=cores)
        wall += t_pack + t_tok
        full += t_pack + t_tok * (m / n_tok)
    value = args.steps * m / full
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * wall / args.steps, 1),
        "extrapolated": True, "ms_per_step_full_workload": round(1e3 * full / args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8" if args.afmt == "int4" else "fp4(e2m1)+int8", "data": "synthetic (seeded)",
        "config": dict(workload_config(args.afmt, m), parallelism=f"replicas x{world}"),
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: the ternary quantization of all latent weights plus {n_tok} tokens "
                                   f"({args.cpu_tokens_ref} per thread, {cores} threads) of the 7B-shape layer "
                                   f"through the whole path; ms_per_step is that sample's wall time, and value scales "
                                   f"its per-token time linearly to {m} tokens (extrapolated)"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# decode: M tokens through the BitLinear path of DECODE_LAYERS distinct 7B-shape
# layers (2-bit weights packed once, as at inference); the layers' weights
# together exceed L2, so every layer streams its weights from HBM.  Activations
# are INT4 / Top-K INT8 codes one byte each; the GEMM runs on the dp4a GEMV for
# 1-2 tokens, the warp-MMA GEMV for 3-16 and the tensor cores beyond.
# ---------------------------------------------------------------------------
DECODE_LAYERS = 4   # 4 x 50.6 MB of 2-bit weights > the 126 MB L2


def decode_gemm_kernel(m: int) -> str:
    if m <= 2:
        return "CUDA-core GEMV (dp4a on offset codes)"
    if m <= 16:
        return "warp-MMA GEMV (m16n8k32 u8 x s8)"
    return "tcgen05 (2-bit weights widened into TMEM)"


def run_quant_variants(args):
    """The 4-bit activation quantizer with each bl_quant variant (INT4 absmean,
    FP4 E2M1, and the ablation variants INT4 absmax, INT4 absmean with beta =
    2 mean|x|, FP4 E1M2) on the 7B QKV input, M = 32768 x K = 4096 bf16 (268 MB,
    larger than L2), byte-layout codes; CUDA events around each launch."""
    import torch

    import ternary_bit_activation_b200 as tba
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    s = SHAPE
    m, k = s.tokens, s.hidden
    x = torch.from_numpy(synth.gaussian_bf16(synth.rng(500), (m, k)).view(np.int16)).to(dev)   # Gaussian QKV input
    codes = torch.empty((m, k), dtype=torch.int8, device=dev)
    scale = torch.empty((m,), dtype=torch.float32, device=dev)
    peaks = load_peaks()
    nbytes = m * (2 * k + k + 4)
    variants = [("int4_absmean", tba.BL_QUANT_INT4), ("fp4_e2m1", tba.BL_QUANT_FP4_E2M1),
                ("int4_absmax", tba.BL_QUANT_INT4_ABSMAX), ("int4_absmean_2beta", tba.BL_QUANT_INT4_ABSMEAN2),
                ("fp4_e1m2", tba.BL_QUANT_FP4_E1M2)]
    gnorm = (1.0 + 0.3 * torch.randn((k,), device=dev)).float()
    beta = torch.empty((1,), dtype=torch.float32, device=dev)
    ws = torch.empty((tba.workspace_size("quant_a4_per_tensor") // 8,), dtype=torch.int64, device=dev)
    calls = [(name, (lambda q=q: tba.bitlinear_quant_a4(x, codes, scale, q, tba.BL_STORE_BYTES, EPS)))
             for name, q in variants]
    # RMSNorm fused in front of INT4 (one read of x), and INT4 with one scale for the
    # tensor (a pass for the exact mean |x|, then the quantizer: x is read twice)
    calls.append(("rmsnorm_int4", lambda: tba.bitlinear_rmsnorm_quant_a4(x, codes, scale, gamma=gnorm, eps_norm=1e-6,
                                                                         store=tba.BL_STORE_BYTES, eps=EPS)))
    calls.append(("int4_per_tensor", lambda: tba.bitlinear_quant_a4_per_tensor(x, codes, scale, beta, ws,
                                                                              store=tba.BL_STORE_BYTES, eps=EPS)))
    results = []
    for name, fn in calls:
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record()
            fn()
            b_.record()
            torch.cuda.synchronize()
            ts.append(a_.elapsed_time(b_))
        tba.sync_status()
        ms = sorted(ts)[len(ts) // 2]
        gbs = nbytes / (ms / 1e3) / 1e9
        r = {"variant": name, "us": round(ms * 1e3, 1), "gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 3)}
        if name == "int4_per_tensor":
            moved = nbytes + m * 2 * k        # x is read by both passes
            r["hbm_frac_bytes_moved"] = round(moved / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 3)
        results.append(r)
    line = {"metric": "4-bit activation quantizer GB/s per variant (7B QKV input)", "unit": "GB/s",
            "workload": f"X bf16 [{m} x {k}] -> int8 codes + fp32 scale per token (median of {args.steps} launches)",
            "algorithmic_bytes": nbytes, "hbm_peak_gbs": peaks["hbm_gbs"], "results": results}
    print(json.dumps(line), flush=True)


def decode_sweep(torch, tba, dev, tokens_list, steps, warmup, w_lat=None, variants=True):
    """Per M in tokens_list: CUDA-graph replay of M tokens through the BitLinear
    path of DECODE_LAYERS distinct 7B-shape layers (2-bit weights packed once,
    as at inference; together they exceed L2, so every layer streams its weights
    from HBM).  w_lat: latent fp32 weights on the device to pack into each
    layer's own buffers (else seeded weights per layer).  variants adds the
    fused-quantizer and conditional-Up timings."""
    s = SHAPE
    d, f = s.hidden, s.ffn
    T = torch
    shapes = {"qkv": (3 * d, d), "o": (d, d), "upgate": (2 * f, d), "down": (d, f)}
    layers = []
    ws = T.empty((tba.workspace_size("pack_ternary") // 8,), dtype=T.int64, device=dev)
    for li in range(DECODE_LAYERS):
        wts = w_lat if w_lat is not None else {k: T.from_numpy(v).to(dev)
                                                for k, v in synth.layer_weights(s, seed=3 + li).items()}
        w2 = {k: T.empty((n, kk // 4), dtype=T.uint8, device=dev) for k, (n, kk) in shapes.items()}
        alpha = T.zeros((8,), dtype=T.float32, device=dev)
        for key, dst, ai in (("qkv", w2["qkv"], 0), ("o", w2["o"], 1), ("up", w2["upgate"][:f], 2),
                             ("gate", w2["upgate"][f:], 3), ("down", w2["down"], 4)):
            tba.pack_ternary(wts[key], alpha[ai:ai + 1], dst, tba.BL_W_T2, ws)
        del wts
        layers.append((w2, alpha))
    weight_bytes = sum(n * kk // 4 for n, kk in shapes.values())
    peaks = load_peaks()
    results = []
    for m in tokens_list:
        x_attn, x_o, x_ffn = [T.from_numpy(a.view(np.int16)).to(dev)
                              for a in synth.layer_activations(s, seed=500 + m, tokens=m)]
        qa = T.empty((m, d), dtype=T.int8, device=dev)
        qa_s = T.empty((m,), dtype=T.float32, device=dev)
        o8 = T.empty((m, d), dtype=T.int8, device=dev)
        o8_s = T.empty((m,), dtype=T.float32, device=dev)
        h8 = T.empty((m, f), dtype=T.int8, device=dev)
        h8_s = T.empty((m,), dtype=T.float32, device=dev)
        y_qkv = T.empty((m, 3 * d), dtype=T.int16, device=dev)
        y_o = T.empty((m, d), dtype=T.int16, device=dev)
        y_ug = T.empty((m, 2 * f), dtype=T.int16, device=dev)
        y_down = T.empty((m, d), dtype=T.int16, device=dev)
        qg_ws = T.empty((tba.workspace_size("quant_gemm", m, 2 * f, d) // 8 + 1,), dtype=T.int64, device=dev)

        def layer(w2, alpha, gemms=True, others=True, fused=False, gated=False):
            # fused: the INT4 quantizer of the QKV and Up|Gate inputs runs inside
            # the GEMM call (bitlinear_quant_gemm)
            if fused:
                tba.bitlinear_quant_gemm(x_attn, w2["qkv"], alpha[0:1], m, 3 * d, d, y=y_qkv, eps=EPS,
                                         workspace=qg_ws)
            if others and not fused:
                tba.bitlinear_quant_a4(x_attn, qa, qa_s, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
            if gemms and not fused:
                tba.bitlinear_gemm(qa, qa_s, w2["qkv"], alpha[0:1], m, 3 * d, d, y=y_qkv, wfmt=tba.BL_W_T2)
            if others:
                tba.bitlinear_sparsify_a8(x_o, synth.k_keep(d, s.topk_pct_o), o8, o8_s, None, EPS)
            if gemms:
                tba.bitlinear_gemm(o8, o8_s, w2["o"], alpha[1:2], m, d, d, y=y_o, wfmt=tba.BL_W_T2)
            if fused:
                tba.bitlinear_quant_gemm(x_ffn, w2["upgate"], alpha[2:4], m, 2 * f, d, y=y_ug, eps=EPS,
                                         alpha_group=f, workspace=qg_ws)
            if others and not fused:
                tba.bitlinear_quant_a4(x_ffn, qa, qa_s, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES, EPS)
            if gemms and not fused and not gated:
                tba.bitlinear_gemm(qa, qa_s, w2["upgate"], alpha[2:4], m, 2 * f, d, y=y_ug, wfmt=tba.BL_W_T2,
                                   alpha_group=f)
            if gemms and gated:
                # conditional Up: Gate rows first, Up rows only for channels with a positive gate
                tba.bitlinear_gemm_gated(qa, qa_s, w2["upgate"], alpha[2:4], m, f, d, y_ug)
            if others:
                tba.relu2_glu(y_ug[:, f:], y_ug[:, :f], synth.k_keep(f, s.topk_pct_down), h8, h8_s, None, EPS,
                              M=m, F=f, ld=2 * f)
            if gemms:
                tba.bitlinear_gemm(h8, h8_s, w2["down"], alpha[4:5], m, d, f, y=y_down, wfmt=tba.BL_W_T2)

        def all_layers(**kw):
            return lambda: [layer(w2, alpha, **kw) for w2, alpha in layers]

        for _ in range(warmup):
            all_layers()()
        tba.sync_status()
        torch.cuda.synchronize()

        # decode launches are a few microseconds each: capture the layers in CUDA
        # graphs and time graph replays
        def capture(fn):
            side = T.cuda.Stream()
            side.wait_stream(T.cuda.current_stream())
            with T.cuda.stream(side):
                fn()
            T.cuda.current_stream().wait_stream(side)
            graph = T.cuda.CUDAGraph()
            with T.cuda.graph(graph):
                fn()
            return graph

        def time_graph(graph):
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            a_, b_ = T.cuda.Event(enable_timing=True), T.cuda.Event(enable_timing=True)
            a_.record()
            for _ in range(steps):
                graph.replay()
            b_.record()
            torch.cuda.synchronize()
            return a_.elapsed_time(b_) / (steps * DECODE_LAYERS)

        graphs = {"step": capture(all_layers()), "gemm": capture(all_layers(others=False))}
        if variants:
            graphs["fused"] = capture(all_layers(fused=True))
            if m <= 2:
                graphs["gated"] = capture(all_layers(gated=True))
        ms = {k: time_graph(g) for k, g in graphs.items()}
        tba.sync_status()
        del graphs
        gbs = weight_bytes / (ms["gemm"] / 1e3) / 1e9
        r = {"tokens": m, "us_per_layer": round(1e3 * ms["step"], 2), "tokens_per_s": round(m / (ms["step"] / 1e3), 1),
             "us_gemm_per_layer": round(1e3 * ms["gemm"], 2), "gemm_kernel": decode_gemm_kernel(m),
             "weight_stream_gbs": round(gbs, 1), "hbm_frac_gemm": round(gbs / peaks["hbm_gbs"], 3),
             "hbm_frac_layer": round(weight_bytes / (ms["step"] / 1e3) / 1e9 / peaks["hbm_gbs"], 3)}
        if "fused" in ms:
            r["fused_quant_us_per_layer"] = round(1e3 * ms["fused"], 2)
        if "gated" in ms:
            r["conditional_up_us_per_layer"] = round(1e3 * ms["gated"], 2)
        results.append(r)
    return {"weight_bytes_per_layer": weight_bytes, "layers": DECODE_LAYERS, "hbm_peak_gbs": peaks["hbm_gbs"],
            "results": results}


def run_decode(args):
    import torch

    import ternary_bit_activation_b200 as tba
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    sweep = decode_sweep(torch, tba, dev, args.decode_tokens, args.steps, args.warmup)
    line = {"metric": "decode BitLinear layer latency (7B shapes, 2-bit weights; CUDA-graph replay)",
            "unit": "us per layer",
            "workload": f"7B-shape decoder layers, decode of M tokens through all four BitLinear matrices of "
                        f"each of {DECODE_LAYERS} distinct layers (weights exceed L2), separate quantizer and GEMM "
                        f"calls; fused_quant_us_per_layer: the QKV and Up|Gate INT4 quantizers fused into their "
                        f"GEMMs (bitlinear_quant_gemm); conditional_up_us_per_layer (1-2 tokens): the Up|Gate GEMM as "
                        f"Gate first and Up only on channels with a positive gate (bitlinear_gemm_gated)",
            "steps": args.steps, "warmup": args.warmup, **sweep}
    print(json.dumps(line), flush=True)


def fp4_gemm_key(torch, tba, layer, reps: int):
    """The FP4 activation variant's two tensor-core GEMMs at the step's size:
    packed E2M1 activations (the step's QKV and FFN inputs, quantized) x
    E2M1-coded ternary weights (the step's latent Q|K|V and Up|Gate weights) on
    tcgen05 kind::mxf4; CUDA events around each launch, median of reps."""
    T = torch
    dev = layer.dev
    m, d, f = layer.m, layer.d, layer.f
    W = layer.w_lat
    wq = T.empty((3 * d, d // 2), dtype=T.uint8, device=dev)
    wug = T.empty((2 * f, d // 2), dtype=T.uint8, device=dev)
    al = T.zeros((4,), dtype=T.float32, device=dev)
    tba.pack_ternary(W["qkv"], al[0:1], wq, tba.BL_W_E2M1, layer.ws, eps=EPS)
    tba.pack_ternary(W["up"], al[1:2], wug[:f], tba.BL_W_E2M1, layer.ws, eps=EPS)
    tba.pack_ternary(W["gate"], al[2:3], wug[f:], tba.BL_W_E2M1, layer.ws, eps=EPS)
    qa = T.empty((m, d // 2), dtype=T.uint8, device=dev)
    qf = T.empty((m, d // 2), dtype=T.uint8, device=dev)
    sa = T.empty((m,), dtype=T.float32, device=dev)
    sf = T.empty((m,), dtype=T.float32, device=dev)
    tba.bitlinear_quant_a4(layer.x[0], qa, sa, tba.BL_QUANT_FP4_E2M1, tba.BL_STORE_PACKED, EPS)
    tba.bitlinear_quant_a4(layer.x[2], qf, sf, tba.BL_QUANT_FP4_E2M1, tba.BL_STORE_PACKED, EPS)
    runs = {"qkv": (lambda: tba.bitlinear_gemm(qa, sa, wq, al[0:1], m, 3 * d, d, y=layer.y_qkv,
                                                afmt=tba.BL_A_E2M1, wfmt=tba.BL_W_E2M1), 3 * d),
            "upgate": (lambda: tba.bitlinear_gemm(qf, sf, wug, al[1:3], m, 2 * f, d, y=layer.y_ug, alpha_group=f,
                                                   afmt=tba.BL_A_E2M1, wfmt=tba.BL_W_E2M1), 2 * f)}
    out = {}
    for name, (fn, n) in runs.items():
        for _ in range(2):
            fn()
        ts = []
        for _ in range(reps):
            a_, b_ = T.cuda.Event(enable_timing=True), T.cuda.Event(enable_timing=True)
            a_.record()
            fn()
            b_.record()
            T.cuda.synchronize()
            ts.append(a_.elapsed_time(b_))
        ms = sorted(ts)[len(ts) // 2]
        out[name] = {"us": round(1e3 * ms, 1), "tops_dense": round(2.0 * m * n * d / (ms / 1e3) / 1e12, 1)}
    tba.sync_status()
    return out


ATTN_SHAPE = (32768, 32, 128)   # positions x heads x head_dim of the 7B decode cache
ATTN_CACHES = 4                 # 4 x 109 MB of codes and scales > the 126 MB L2


def attention_key(torch, tba, dev, hbm_peak: float, queries=(1, 2, 4, 8), reps: int = 10):
    """attention_lowbit in the 7B decode context: M 4-bit queries over a
    32768-position cache of 32 heads of 128 (3-bit K and V, the BOS position at
    4 bits).  ATTN_CACHES caches with their own buffers (together larger than L2)
    are visited in turn, so every call streams its cache from HBM; CUDA events
    around `reps` passes over the caches.  Algorithmic bytes per call: the K and
    V codes and scales, 2 * T * H * (3 D / 8 + 4)."""
    T = torch
    Tn, H, D = ATTN_SHAPE
    g = T.Generator(device=dev)
    g.manual_seed(11)

    def quant(x, bits, bos):
        n = x.shape[0]
        c = T.empty((n, H, D * bits // 8), dtype=T.uint8, device=dev)
        sc = T.empty((n, H), dtype=T.float32, device=dev)
        b = T.empty((H, D // 2), dtype=T.uint8, device=dev)
        tba.kv_quant3(x, n, H, D, c, sc, bos_codes=b, bits=bits, bos_pos=bos, eps=EPS)
        return c, sc, b

    caches = []
    for _ in range(ATTN_CACHES):
        kx = T.randn((Tn, H * D), generator=g, device=dev).to(T.bfloat16).view(T.int16)
        kc, ks, kb = quant(kx, 3, 0)
        del kx
        vx = T.randn((Tn, H * D), generator=g, device=dev).to(T.bfloat16).view(T.int16)
        vc, vs, vb = quant(vx, 3, 0)
        del vx
        caches.append((kc, ks, kb, vc, vs, vb))
    nbytes = 2 * Tn * H * (3 * D // 8 + 4)
    results = []
    for m in queries:
        qx = T.randn((m, H * D), generator=g, device=dev).to(T.bfloat16).view(T.int16)
        qc, qs, _ = quant(qx, 4, -1)
        out = T.empty((m, H * D), dtype=T.int16, device=dev)
        ws = T.empty((tba.workspace_size("attention_lowbit", m, H, D) // 4,), dtype=T.float32, device=dev)

        def one_pass():
            for kc, ks, kb, vc, vs, vb in caches:
                tba.attention_lowbit(qc, qs, m, kc, ks, vc, vs, Tn, H, D, out, ws, k_bos=kb, v_bos=vb, kv_bits=3,
                                     bos_pos=0)

        for _ in range(3):
            one_pass()
        a_, b_ = T.cuda.Event(enable_timing=True), T.cuda.Event(enable_timing=True)
        T.cuda.synchronize()
        a_.record()
        for _ in range(reps):
            one_pass()
        b_.record()
        T.cuda.synchronize()
        us = 1e3 * a_.elapsed_time(b_) / (reps * ATTN_CACHES)
        gbs = nbytes / (us * 1e-6) / 1e9
        results.append({"queries": m, "us": round(us, 2), "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm_peak, 3)})
    tba.sync_status()
    return {"unit": "us per call", "workload": f"attention_lowbit: M 4-bit queries over a {Tn}-position cache of {H} "
                                               f"heads x {D} (3-bit K and V, BOS position at 4 bits); "
                                               f"{ATTN_CACHES} caches visited in turn (larger than L2)",
            "algorithmic_bytes": nbytes, "hbm_peak_gbs": hbm_peak, "results": results}


# ---------------------------------------------------------------------------
# single-kernel cases for profiler captures (small enough for ncu's replays;
# inputs still larger than L2)
# ---------------------------------------------------------------------------
PROFILE_CASES = {
    "gemm": "tcgen05 GEMM, int8 A [16384 x 4096] x ternary int8 W [12288 x 4096]",
    "gemm_o": "tcgen05 GEMM, int8 A [16384 x 4096] x ternary int8 W [4096 x 4096]",
    "gemm_upgate": "tcgen05 GEMM, int8 A [16384 x 4096] x ternary int8 W [22016 x 4096]",
    "gemm_down": "tcgen05 GEMM, int8 A [16384 x 11008] x ternary int8 W [4096 x 11008]",
    "quant_a4": "INT4 quantizer, X bf16 [32768 x 4096]",
    "rmsnorm_quant_a4": "RMSNorm (with a weight) fused into the INT4 quantizer, X bf16 [32768 x 4096]",
    "sparsify_a8": "Top-K 50% + INT8, X bf16 [32768 x 4096]",
    "relu2_glu": "ReLU^2-GLU + Top-K 50% + INT8, gate/up bf16 [16384 x 11008]",
    "kv_quant3": "3-bit KV, K bf16 [32768 x 32 x 128]",
    "attention": "low-bit attention, 1 4-bit query over a 3-bit cache [32768 x 32 x 128]",
    "pack_ternary": "ternary pack to int8, W fp32 [22016 x 4096]",
    "gemm_decode": "CUDA-core GEMV, 2-bit W [12288 x 4096], 1 token",
    "gemm_decode_mma": "warp-MMA GEMV, 2-bit W [12288 x 4096], 8 tokens",
    "gemm_decode_stream": "streaming GEMV, 2-bit W [4096 x 11008] (Down), 1 token",
    "gemm_decode_tc": "tcgen05 GEMM, 2-bit W [12288 x 4096] widened into TMEM, 16 tokens",
}


def run_profile_case(name: str, launches: int):
    import torch

    import ternary_bit_activation_b200 as tba
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(7)

    def bf16(m, k, scale=1.0):
        return (torch.randn((m, k), generator=g, device=dev) * scale).to(torch.bfloat16).view(torch.int16)

    if name in ("gemm", "gemm_o", "gemm_upgate", "gemm_down"):
        M, N, K = {"gemm": (16384, 12288, 4096), "gemm_o": (16384, 4096, 4096), "gemm_upgate": (16384, 22016, 4096),
                   "gemm_down": (16384, 4096, 11008)}[name]
        a = torch.randint(-8, 8, (M, K), generator=g, device=dev, dtype=torch.int8)
        w = torch.randint(-1, 2, (N, K), generator=g, device=dev, dtype=torch.int8)
        s = torch.rand((M,), generator=g, device=dev)
        al = torch.full((1,), 0.0173, device=dev)
        y = torch.empty((M, N), dtype=torch.int16, device=dev)
        fn = lambda: tba.bitlinear_gemm(a, s, w, al, M, N, K, y=y)
    elif name in ("gemm_decode", "gemm_decode_mma", "gemm_decode_stream"):
        M, N, K = {"gemm_decode": (1, 12288, 4096), "gemm_decode_mma": (8, 12288, 4096),
                   "gemm_decode_stream": (1, 4096, 11008)}[name]
        a = torch.randint(-8, 8, (M, K), generator=g, device=dev, dtype=torch.int8)
        w = torch.randint(0, 256, (N, K // 4), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
        s = torch.rand((M,), generator=g, device=dev)
        al = torch.full((1,), 0.0173, device=dev)
        y = torch.empty((M, N), dtype=torch.int16, device=dev)
        fn = lambda: tba.bitlinear_gemm(a, s, w, al, M, N, K, y=y, wfmt=tba.BL_W_T2)
    elif name == "gemm_decode_tc":
        M, N, K = 16, 12288, 4096
        a = torch.randint(-8, 8, (M, K), generator=g, device=dev, dtype=torch.int8)
        w = torch.randint(0, 256, (N, K // 4), generator=g, device=dev, dtype=torch.int32).to(torch.uint8)
        s = torch.rand((M,), generator=g, device=dev)
        al = torch.full((1,), 0.0173, device=dev)
        y = torch.empty((M, N), dtype=torch.int16, device=dev)
        fn = lambda: tba.bitlinear_gemm(a, s, w, al, M, N, K, y=y, wfmt=tba.BL_W_T2)
    elif name == "quant_a4":
        x = bf16(32768, 4096)
        c = torch.empty((32768, 4096), dtype=torch.uint8, device=dev)
        s = torch.empty((32768,), device=dev)
        fn = lambda: tba.bitlinear_quant_a4(x, c, s, tba.BL_QUANT_INT4, tba.BL_STORE_BYTES)
    elif name == "rmsnorm_quant_a4":
        x = bf16(32768, 4096)
        c = torch.empty((32768, 4096), dtype=torch.uint8, device=dev)
        s = torch.empty((32768,), device=dev)
        gn = (1.0 + 0.3 * torch.randn((4096,), generator=g, device=dev)).float()
        fn = lambda: tba.bitlinear_rmsnorm_quant_a4(x, c, s, gamma=gn, store=tba.BL_STORE_BYTES)
    elif name == "sparsify_a8":
        x = bf16(32768, 4096)
        c = torch.empty((32768, 4096), dtype=torch.int8, device=dev)
        s = torch.empty((32768,), device=dev)
        fn = lambda: tba.bitlinear_sparsify_a8(x, 2048, c, s, None)
    elif name == "relu2_glu":
        M, F = 16384, 11008
        ug = bf16(M, 2 * F)
        c = torch.empty((M, F), dtype=torch.int8, device=dev)
        s = torch.empty((M,), device=dev)
        fn = lambda: tba.relu2_glu(ug[:, F:], ug[:, :F], F // 2, c, s, None, M=M, F=F, ld=2 * F)
    elif name == "kv_quant3":
        T, H, D = 32768, 32, 128
        kv = bf16(T, H * D)
        c = torch.empty((T, H, D * 3 // 8), dtype=torch.uint8, device=dev)
        s = torch.empty((T, H), device=dev)
        b = torch.empty((H, D // 2), dtype=torch.uint8, device=dev)
        fn = lambda: tba.kv_quant3(kv, T, H, D, c, s, b, bits=3, bos_pos=0)
    elif name == "attention":
        T_, H, D = 32768, 32, 128

        def quant(x, n, bits, bos):
            c = torch.empty((n, H, D * bits // 8), dtype=torch.uint8, device=dev)
            s = torch.empty((n, H), device=dev)
            b = torch.empty((H, D // 2), dtype=torch.uint8, device=dev)
            tba.kv_quant3(x, n, H, D, c, s, b, bits=bits, bos_pos=bos)
            return c, s, b

        kc, ks, kb = quant(bf16(T_, H * D), T_, 3, 0)
        vc, vs, vb = quant(bf16(T_, H * D), T_, 3, 0)
        qc, qs, _ = quant(bf16(1, H * D), 1, 4, -1)
        out = torch.empty((1, H * D), dtype=torch.int16, device=dev)
        ws = torch.empty((tba.workspace_size("attention_lowbit", 1, H, D) // 4,), device=dev)
        fn = lambda: tba.attention_lowbit(qc, qs, 1, kc, ks, vc, vs, T_, H, D, out, ws, k_bos=kb, v_bos=vb,
                                          kv_bits=3, bos_pos=0)
    elif name == "pack_ternary":
        w = torch.randn((22016, 4096), generator=g, device=dev) * 0.02
        o = torch.empty((22016, 4096), dtype=torch.uint8, device=dev)
        al = torch.empty((1,), device=dev)
        ws = torch.empty((256,), dtype=torch.int64, device=dev)
        fn = lambda: tba.pack_ternary(w, al, o, tba.BL_W_I8, ws)
    else:
        raise SystemExit(f"unknown profile case {name}; one of {sorted(PROFILE_CASES)}")
    for _ in range(launches):
        fn()
    tba.sync_status()
    print(f"profile case {name}: {PROFILE_CASES[name]}, {launches} launches OK")


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--afmt", choices=["int4", "fp4"], default="int4")
    ap.add_argument("--cpu-tokens", type=int, default=16, help="token sample of the one-core CPU baseline")
    ap.add_argument("--cpu-tokens-per-core", type=int, default=4, help="tokens per thread of the all-core CPU baseline")
    ap.add_argument("--cpu-tokens-ref", type=int, default=2, help="tokens per thread and step of --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the decode and FP4 keys of the prefill line")
    ap.add_argument("--workload", choices=["prefill", "decode", "quant-variants", "attention"], default="prefill",
                    help="prefill: the headline step; decode: per-token-batch latency sweep; "
                         "quant-variants: the 4-bit quantizer and its ablation variants at the 7B prefill input; "
                         "attention: low-bit attention over the 7B decode cache")
    ap.add_argument("--decode-tokens", type=int, nargs="+", default=synth.DECODE_TOKENS)
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES), help="run one kernel's small case and exit")
    ap.add_argument("--launches", type=int, default=3, help="launches of --profile-case")
    args = ap.parse_args(argv)
    if args.profile_case:
        run_profile_case(args.profile_case, args.launches)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "decode":
        run_decode(args)
    elif args.workload == "quant-variants":
        run_quant_variants(args)
    elif args.workload == "attention":
        import torch

        import ternary_bit_activation_b200 as tba
        torch.cuda.set_device(0)
        print(json.dumps(attention_key(torch, tba, torch.device("cuda", 0), load_peaks()["hbm_gbs"])), flush=True)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
