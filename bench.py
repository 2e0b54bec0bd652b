#!/usr/bin/env python
"""Benchmark of the tensor-parallel block on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sq4096|tiny|mlp70b|mlp70b_w8|attn70b|mlp405b] [--tp T]

Default workload: the largest block of the measured set, the 405B-shaped MLP
in prefill (x[8192, 16384], W1 [53248, 16384] split by columns into t = 8
shards, GeLU, W2 [16384, 53248] split by rows with the fused 8-shard sum).  One
step = one pass of the whole block over one batch: the column-parallel GEMM and
the row-parallel GEMM with its on-chip all-reduce, 8192 tokens.  The other
workloads are available with --workload: sq4096 (the pages' TP=2 square
projection at decode batches T = 1, 8, 64), mlp70b (the 70B-shaped MLP decode),
mlp70b_w8 (the same with 8-bit E4M3 weights and per-row scales), attn70b (the
70B-shaped attention projections in prefill) and tiny.

Timing: W warm-up steps, then exactly K steps captured in CUDA graphs and
bracketed by a barrier + synchronize on both sides, timed with CUDA events on
the launching stream; the max over ranks is taken.  Weights are rotated over
enough copies that each call reads weights not touched for >= 4x the L2 size
(or the weights alone exceed L2).  Multi-GPU runs are independent replicas
(the block has no cross-GPU step here): value = all ranks' tokens / max time.

--impl reference times the fp64 CPU oracle (the only reference this block
has) on a bounded sample of the same workload on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "TP-block tokens/s; % of HBM roofline (decode) and bf16 TC peak (prefill)"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
# device sources whose change invalidates a kernel's recorded ncu traffic
KERNEL_SOURCES = {
    "stream_gemm_kernel": ["csrc/ptx.cuh", "csrc/stream_kernel.cuh"],
    "tiled_gemm_kernel": ["csrc/ptx.cuh", "csrc/tiled_kernel.cuh"],
    "pair_gemm_kernel": ["csrc/ptx.cuh", "csrc/tiled_kernel.cuh", "csrc/pair_kernel.cuh"],
    "attn_decode_kernel": ["csrc/ptx.cuh", "csrc/attn_kernel.cuh"],
    "attn_prefill2_kernel": ["csrc/ptx.cuh", "csrc/attn_kernel.cuh", "csrc/attn_prefill_kernel.cuh"],
    "add_rmsnorm_kernel": ["csrc/ptx.cuh", "csrc/norm_kernel.cuh"],
}
LAUNCH_OPTIONS = {"none": 0, "pdl": 1, "pdl+static_weights": 3}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# default (timed steps, warm-up steps) per workload: about a second of timed work
DEFAULT_STEPS = {"mlp405b": (40, 5), "attn70b": (1000, 20), "attn70b_decode": (5000, 50),
                 "attn70b_prefill": (2000, 20),
                 "mlp70b_bwd": (100, 5),
                 "sp405b": (2000, 20),
                 "mlp70b": (2000, 50),
                 "mlp70b_w8": (2000, 50), "sq4096": (20000, 200), "tiny": (20000, 200)}


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a float over ranks (identity for one rank)."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    dev = device if (device is not None and dist.get_backend() == "nccl") else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(tokens_per_step: float, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput of `world` independent replicas timed by the slowest rank."""
    return tokens_per_step * world / (ms_per_step_max / 1000.0)


# ---------------------------------------------------------------- peaks, clocks, provenance

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel.split("<")[0].split(":")[0]]:
        with open(os.path.join(ROOT, "tensor_transformer_linear_column_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if taken on this kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(f"{kernel}:{workload}")
        if e and e.get("source_hash") == kernel_source_hash(kernel):
            return e.get("dram_bytes_per_launch")
    except Exception:
        return None
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clk", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- workloads

class Workload:
    """Device-resident inputs of one workload and its step as C-ABI calls."""

    def __init__(self, name: str, tp_degree, device, rotate=True, tokens=None):
        import tensor_transformer_linear_column_b200 as tp
        self.tp = tp
        self.name = name
        self.cfg = workloads.CONFIGS[name]
        self.dev = device
        cfg = self.cfg
        if name == "sq4096":
            self.t = tp_degree or cfg.tp_degrees[0]
            self.Ts = list(tokens or cfg.tokens)
            w = workloads.proj_inputs(cfg, 1)["w"]
            self.weight_bytes = w.numel() * 2
            self.xs = {T: workloads.normal_bf16((T, cfg.k), 1.0, 0, workloads.x_index(T))
                       for T in self.Ts}
            self.hidden_in, self.hidden_out = cfg.k, cfg.n
            self.weights = [w.to(device)]
            self.bias = None
        elif name in ("tiny", "mlp70b", "mlp405b"):
            self.t = tp_degree or cfg.tp_degrees[-1]
            self.Ts = list(tokens or cfg.tokens)
            d = workloads.mlp_inputs(cfg, self.Ts[0])
            self.xs = {T: workloads.mlp_x(cfg, T) for T in self.Ts}
            self.weight_bytes = (d["w1"].numel() + d["w2"].numel()) * 2
            self.hidden_in = self.hidden_out = cfg.hidden
            self.weights = [(d["w1"].to(device), d["w2"].to(device))]
            self.bias = (None if d["b1"] is None else d["b1"].to(device),
                         None if d["b2"] is None else d["b2"].to(device))
            self.ws = torch.empty(max(tp.tp_mlp_workspace_bytes(T, cfg.ffn) for T in self.Ts),
                                  dtype=torch.uint8, device=device)
        elif name == "mlp70b_w8":
            self.t = tp_degree or cfg.tp_degrees[-1]
            self.Ts = list(tokens or cfg.tokens)
            d = workloads.mlp_inputs(cfg, self.Ts[0])
            self.xs = {T: workloads.mlp_x(cfg, T) for T in self.Ts}
            q1, s1 = workloads.quantize_e4m3_rows(d["w1"])
            q2, s2 = workloads.quantize_e4m3_rows(d["w2"])
            self.weight_bytes = q1.numel() + q2.numel() + 4 * (s1.numel() + s2.numel())
            self.hidden_in = self.hidden_out = cfg.hidden
            self.weights = [tuple(a.to(device) for a in (q1, s1, q2, s2))]
            self.bias = (None, None)
            self.ws = torch.empty(max(tp.tp_mlp_workspace_bytes(T, cfg.ffn) for T in self.Ts),
                                  dtype=torch.uint8, device=device)
        elif name == "attn70b":
            self.t = tp_degree or cfg.tp_degrees[0]
            self.Ts = list(tokens or cfg.tokens)
            d = workloads.attn_inputs(cfg, self.Ts[0])
            self.xs = {self.Ts[0]: d["x"]}
            self.ctx = d["ctx"].to(device)
            self.weight_bytes = (d["w_qkv"].numel() + d["w_o"].numel()) * 2
            self.hidden_in = self.hidden_out = cfg.hidden
            self.weights = [(d["w_qkv"].to(device), d["w_o"].to(device))]
            nqkv = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
            self.qkv = torch.empty((self.Ts[0], nqkv), dtype=torch.bfloat16, device=device)
        elif name == "attn70b_prefill":
            self.t = tp_degree or cfg.tp_degrees[0]
            self.Ts = list(tokens or cfg.tokens)
            self.xs = {T: workloads.attn_decode_qkv(cfg, T) for T in self.Ts}
            d = cfg.head_dim
            self.max_len = cfg.past + max(self.Ts)
            kc = torch.empty((cfg.n_kv_heads, self.max_len, d), dtype=torch.bfloat16, device=device)
            self.weights = [(kc, torch.empty_like(kc))]
            # the caches each call writes and then reads (rotated like weights)
            self.weight_bytes = 2 * cfg.n_kv_heads * self.max_len * d * 2
            self.hidden_in = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * d
            self.hidden_out = cfg.n_q_heads * d
        elif name == "attn70b_decode":
            self.t = tp_degree or cfg.tp_degrees[0]
            self.Ts = list(tokens or cfg.tokens)
            self.xs = {T: workloads.attn_decode_qkv(cfg, T) for T in self.Ts}
            k, v = workloads.attn_decode_cache(cfg)
            d = cfg.head_dim
            self.max_len = cfg.past + max(self.Ts)
            kc = torch.empty((cfg.n_kv_heads, self.max_len, d), dtype=torch.bfloat16, device=device)
            vc = torch.empty_like(kc)
            kc[:, :cfg.past].copy_(k)
            vc[:, :cfg.past].copy_(v)
            self.weights = [(kc, vc)]
            self.weight_bytes = 2 * k.numel() * 2  # the cache read by every call
            self.hidden_in = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * d
            self.hidden_out = cfg.n_q_heads * d
            self.ws = torch.empty(max(tp.tp_attn_decode_workspace_bytes(
                T, cfg.past, cfg.n_q_heads, cfg.n_kv_heads, d) for T in self.Ts),
                dtype=torch.uint8, device=device)
        elif name == "mlp70b_bwd":
            self.t = tp_degree or cfg.tp_degrees[-1]
            self.Ts = list(tokens or cfg.tokens)
            d = workloads.mlp_inputs(cfg, self.Ts[0])
            self.xs = {T: workloads.mlp_x(cfg, T) for T in self.Ts}
            self.dy = {T: workloads.mlp_dy(cfg, T).to(device) for T in self.Ts}
            self.weight_bytes = (d["w1"].numel() + d["w2"].numel()) * 2
            self.hidden_in = self.hidden_out = cfg.hidden
            self.weights = [(d["w1"].to(device), d["w2"].to(device))]
            F, H = cfg.ffn, cfg.hidden
            self.grads = {T: {"dw1": torch.empty((F, H), dtype=torch.bfloat16, device=device),
                              "dw2": torch.empty((H, F), dtype=torch.bfloat16, device=device),
                              "db1": torch.empty((F,), dtype=torch.bfloat16, device=device),
                              "db2": torch.empty((H,), dtype=torch.bfloat16, device=device)}
                          for T in self.Ts}
            self.ws = torch.empty(max(tp.tp_mlp_backward_workspace_bytes(T, F) for T in self.Ts),
                                  dtype=torch.uint8, device=device)
        elif name == "sp405b":
            self.t = tp_degree or cfg.tp_degrees[0]
            self.Ts = list(tokens or cfg.tokens)
            ds = {T: workloads.sp_norm_inputs(cfg, T) for T in self.Ts}
            self.xs = {T: d["y"] for T, d in ds.items()}
            self.res = {T: d["residual"].to(device) for T, d in ds.items()}
            self.weights = [ds[self.Ts[0]]["gamma"].to(device)]
            self.weight_bytes = cfg.hidden * 2
            self.hidden_in = self.hidden_out = cfg.hidden
            self.r_out = {T: torch.empty((T, cfg.hidden), dtype=torch.bfloat16, device=device)
                          for T in self.Ts}
        else:
            raise ValueError(name)
        self.xd = {T: x.to(device) for T, x in self.xs.items()}
        self.outs = {T: torch.empty((T, self.hidden_out), dtype=torch.bfloat16, device=device)
                     for T in self.Ts}
        # rotate weight copies so each step reads weights evicted from L2
        assert tokens or self.weight_bytes == workload_weight_bytes(name)
        # (the sequence-parallel region streams activations only, all larger than L2)
        self.rot = rotation_copies(self.weight_bytes) if rotate and name != "sp405b" else 1
        if self.rot > 1:
            base = self.weights[0]
            for _ in range(self.rot - 1):
                if isinstance(base, tuple):
                    self.weights.append(tuple(b.clone() for b in base))
                else:
                    self.weights.append(base.clone())
        self.tokens_per_step = sum(self.Ts)
        self.launches_per_step = len(self.Ts) * {"sq4096": 1, "attn70b_decode": 3,
                                                 "attn70b_prefill": 2,
                                                 "sp405b": 1, "mlp70b_bwd": 7}.get(name, 2)

    def step(self, i: int, xs=None, outs=None):
        tp = self.tp
        xs = xs or self.xd
        outs = outs or self.outs
        for j, T in enumerate(self.Ts):
            # every call of every step reads a weight copy not touched for
            # rot - 1 calls, so weights come from HBM, never from L2
            w = self.weights[(i * len(self.Ts) + j) % self.rot]
            if self.name == "sq4096":
                tp.tp_colpar_gemm_gelu(xs[T], w, None, self.t, "none", out=outs[T])
            elif self.name == "mlp70b_w8":
                tp.tp_mlp_forward_w8(xs[T], w[0], w[1], None, w[2], w[3], None, self.t,
                                     self.cfg.act, out=outs[T], workspace=self.ws)
            elif self.name == "mlp70b_bwd":
                gr = self.grads[T]
                st = tp.load().tp_mlp_backward(
                    xs[T].data_ptr(), w[0].data_ptr(), None, w[1].data_ptr(),
                    self.dy[T].data_ptr(), T, self.cfg.hidden, self.cfg.ffn, self.t,
                    tp.ACTS[self.cfg.act], outs[T].data_ptr(), gr["dw1"].data_ptr(),
                    gr["db1"].data_ptr(), gr["dw2"].data_ptr(), gr["db2"].data_ptr(),
                    self.ws.data_ptr(), self.ws.numel(), torch.cuda.current_stream().cuda_stream)
                if st != tp.TP_OK:
                    raise tp.TPError(st, "tp_mlp_backward")
            elif self.name == "sp405b":
                tp.tp_sp_add_rmsnorm(xs[T], self.res[T], w, self.t, 1e-5, r_out=self.r_out[T],
                                     n_out=outs[T])
            elif self.name == "attn70b_prefill":
                c = self.cfg
                tp.tp_attn_prefill(xs[T], w[0], w[1], c.past, c.n_q_heads, c.n_kv_heads,
                                   c.head_dim, self.t, ctx=outs[T])
            elif self.name == "attn70b_decode":
                c = self.cfg
                tp.tp_attn_decode(xs[T], w[0], w[1], c.past, c.n_q_heads, c.n_kv_heads,
                                  c.head_dim, self.t, ctx=outs[T], workspace=self.ws)
            elif self.name == "attn70b":
                tp.tp_attn_proj_forward(xs[T], w[0], None, self.ctx, w[1], None,
                                        self.cfg.n_q_heads, self.cfg.n_kv_heads,
                                        self.cfg.head_dim, self.t, qkv_out=self.qkv, out=outs[T])
            else:
                tp.tp_mlp_forward(xs[T], w[0], self.bias[0], w[1], self.bias[1], self.t,
                                  self.cfg.act, out=outs[T], workspace=self.ws)

    # algorithmic work of one step (for the roofline)
    def step_bytes(self):
        """Weights once per call + activations in and out (decode roofline)."""
        b = 0
        for T in self.Ts:
            b += self.weight_bytes + 2 * T * (self.hidden_in + self.hidden_out)
            if self.name == "attn70b_decode":
                # the new tokens' keys and values: written to the cache, then read
                b += 2 * 2 * 2 * T * self.cfg.n_kv_heads * self.cfg.head_dim
            if self.name == "sp405b":
                b += 2 * 2 * T * self.cfg.hidden  # the residual read and r written
            if self.name in ("tiny", "mlp70b", "mlp70b_w8", "mlp405b"):
                b += 2 * 2 * T * self.cfg.ffn  # h written and read once
        return b

    def step_flops(self):
        """2 T per weight element (bf16 weights: 2 bytes per element); the
        backward pass makes five GEMMs of the layer's size per step.  Causal
        attention: 4 d flops (q.k and p v) per query head and visible key."""
        if self.name == "attn70b_prefill":
            c = self.cfg
            return sum(4 * c.head_dim * c.n_q_heads * (T * (T + 1) // 2 + c.past * T)
                       for T in self.Ts)
        f = 0
        for T in self.Ts:
            f += 2 * T * self.weight_bytes // 2
        return f * 5 // 2 if self.name == "mlp70b_bwd" else f

    def bound(self):
        if self.name == "sp405b":
            return "hbm"
        return "tensor" if max(self.Ts) > 256 else "hbm"

    def hbm_kernel(self):
        return {"attn70b_decode": "attn_decode_kernel",
                "sp405b": "add_rmsnorm_kernel"}.get(self.name, "stream_gemm_kernel")


class _OracleRunner:
    _cache = {}

    @classmethod
    def get(cls, name, t):
        key = (name, t)
        if key not in cls._cache:
            cls._cache[key] = cls(name, t)
        return cls._cache[key]

    def __init__(self, name, t):
        cfg = workloads.CONFIGS[name]
        self.name = name
        self.cfg = cfg
        if name == "mlp70b_bwd":
            self.t = t or cfg.tp_degrees[-1]
            T0 = cfg.tokens[0]
            d = workloads.mlp_inputs(cfg, T0)
            rows = workloads.sample_rows(T0, cfg.sample_rows)
            self.x, self.dy = d["x"][rows], workloads.mlp_dy(cfg, T0)[rows]
            self.w1, self.w2 = d["w1"], d["w2"]
            self.n_out = cfg.hidden
        elif name == "sp405b":
            self.t = t or cfg.tp_degrees[0]
            T0 = cfg.tokens[0]
            d = workloads.sp_norm_inputs(cfg, T0)
            rows = workloads.sample_rows(T0, 64)
            self.y, self.res, self.gamma = d["y"][rows], d["residual"][rows], d["gamma"]
            self.n_out = cfg.hidden
        elif name == "attn70b_decode":
            self.t = t or cfg.tp_degrees[0]
            self.xs = {T: workloads.attn_decode_qkv(cfg, T) for T in cfg.tokens}
            self.k, self.v = workloads.attn_decode_cache(cfg)
            self.n_out = cfg.n_q_heads * cfg.head_dim
        elif name == "attn70b_prefill":
            # 8 seeded tokens of the prompt, every query head of each (tokens
            # are independent given the keys and values they see)
            self.t = t or cfg.tp_degrees[0]
            T0 = cfg.tokens[0]
            self.qkv = workloads.attn_decode_qkv(cfg, T0)
            self.rows = workloads.sample_rows(T0, 8)
            self.n_out = cfg.n_q_heads * cfg.head_dim
        elif name == "sq4096":
            self.t = t or cfg.tp_degrees[0]
            self.w = workloads.proj_inputs(cfg, 1)["w"]
            self.xs = {T: workloads.normal_bf16((T, cfg.k), 1.0, 0, workloads.x_index(T))
                       for T in cfg.tokens}
            self.n_out = cfg.n
        elif name == "attn70b":
            self.t = t or cfg.tp_degrees[0]
            d = workloads.attn_inputs(cfg, cfg.tokens[0])
            rows = workloads.sample_rows(cfg.tokens[0], cfg.sample_rows)
            self.x = d["x"][rows]
            self.ctx = d["ctx"][rows]
            self.w_qkv, self.w_o = d["w_qkv"], d["w_o"]
            self.n_out = cfg.hidden
        else:
            self.t = t or cfg.tp_degrees[-1]
            T0 = cfg.tokens[0]
            d = workloads.mlp_inputs(cfg, T0)
            self.w1, self.w2, self.b1, self.b2 = d["w1"], d["w2"], d["b1"], d["b2"]
            if cfg.weights == "e4m3":
                import oracle
                self.w1 = oracle.E4M3Weight(*workloads.quantize_e4m3_rows(d["w1"]))
                self.w2 = oracle.E4M3Weight(*workloads.quantize_e4m3_rows(d["w2"]))
            if cfg.sample_rows:
                rows = workloads.sample_rows(T0, cfg.sample_rows)
                self.xs = {T0: d["x"][rows]}
            else:
                self.xs = {T: workloads.mlp_x(cfg, T) for T in cfg.tokens}
            self.n_out = cfg.hidden

    def full_tokens(self):
        """Tokens a full oracle step covers (the sampled rows for prefill workloads)."""
        if self.name == "attn70b":
            return self.x.shape[0]
        if self.name == "sp405b":
            return self.y.shape[0]
        if self.name == "attn70b_prefill":
            return len(self.rows)
        if self.name == "mlp70b_bwd":
            return self.x.shape[0]
        return sum(x.shape[0] for x in self.xs.values())

    def run(self, fraction, offset):
        """Compute the step on output-feature block [offset, offset + fraction * n_out)."""
        import oracle
        if self.name == "mlp70b_bwd":
            # the backward pass of 64 seeded tokens (weight gradients over them)
            oracle.mlp_block_backward(self.x, self.w1, None, self.w2, self.dy, self.t,
                                      self.cfg.act)
            return 1.0
        if self.name == "sp405b":
            # 64 seeded token rows (rows are independent); one token shard
            oracle.sp_residual_norm([oracle.to_f64(self.y)], None, self.res, self.gamma, 1)
            return 1.0
        if self.name == "attn70b_prefill":
            # each sampled token i against the keys and values 0 .. i of its
            # key-value head, for all query heads
            c = self.cfg
            d, nq, nkv = c.head_dim, c.n_q_heads, c.n_kv_heads
            G = nq // nkv
            for i in self.rows:
                i = int(i)
                kv = oracle.to_f64(self.qkv[:i + 1, nq * d:])
                q = oracle.to_f64(self.qkv[i:i + 1, :nq * d])
                for h in range(nq):
                    g = h // G
                    oracle.attend_head(q[:, h * d:(h + 1) * d], kv[:, g * d:(g + 1) * d],
                                       kv[:, (nkv + g) * d:(nkv + g + 1) * d], i)
            return 1.0
        if self.name == "attn70b_decode":
            # every new token needs the whole cache: the sample is whole calls
            c = self.cfg
            kh = c.n_kv_heads // self.t
            cache = [(self.k[s * kh:(s + 1) * kh], self.v[s * kh:(s + 1) * kh])
                     for s in range(self.t)]
            for T, qkv in self.xs.items():
                oracle.attn_core(qkv, c.n_q_heads, c.n_kv_heads, c.head_dim, self.t, cache)
            return 1.0
        n = self.n_out
        cnt = max(64, int(round(fraction * n)) // 64 * 64)
        j0 = (offset * cnt) % n
        j1 = min(n, j0 + cnt)
        if self.name == "sq4096":
            for T, x in self.xs.items():
                oracle.linear(x, self.w[j0:j1])
        elif self.name == "attn70b":
            nqkv = self.w_qkv.shape[0]
            oracle.linear(self.x, self.w_qkv[j0 * nqkv // n:j1 * nqkv // n])
            oracle.rowpar_linear(self.ctx, self.w_o[j0:j1], None, self.t)
        else:
            for T, x in self.xs.items():
                # the first layer is needed in full for any output feature
                h = oracle.colpar_linear(x, self.w1, self.b1, self.t, self.cfg.act) \
                    if fraction >= 1.0 or not hasattr(self, "_h") else self._h[T]
                if fraction < 1.0:
                    self._h = getattr(self, "_h", {})
                    self._h[T] = h
                oracle.rowpar_linear(h, self.w2[j0:j1], None if self.b2 is None else self.b2[j0:j1],
                                     self.t)
        return (j1 - j0) / n


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def time_oracle(wl_name, t, budget_s=12.0):
    """Oracle tokens/s on a bounded sample: whole steps while they fit the budget."""
    runner = _OracleRunner.get(wl_name, t)
    toks = runner.full_tokens()
    t0 = time.perf_counter()
    runner.run(1.0, 0)
    one = time.perf_counter() - t0
    steps, elapsed = 1, one
    while elapsed + one <= budget_s:
        t1 = time.perf_counter()
        runner.run(1.0, 0)
        elapsed += time.perf_counter() - t1
        steps += 1
    return toks * steps / elapsed, steps, elapsed, toks


# ---------------------------------------------------------------- arms

def run_reference(args, world, rank):
    if rank != 0:
        return 0
    name = args.workload
    runner = _OracleRunner.get(name, args.tp)
    toks = runner.full_tokens()
    # calibrate the fraction of output features per step so the run stays short
    t0 = time.perf_counter()
    runner.run(1.0 / 16, 0)
    per16 = time.perf_counter() - t0
    total = args.steps + args.warmup
    budget = 120.0
    frac = min(1.0, max(1.0 / 64, (budget / max(total, 1)) / max(per16 * 16, 1e-9)))
    for i in range(args.warmup):
        runner.run(frac, i)
    t0 = time.perf_counter()
    covered = 0.0
    for i in range(args.steps):
        covered += runner.run(frac, i)
    el = time.perf_counter() - t0
    value = toks * covered / el
    cores = blas_threads()
    sample = (f"fp64 numpy oracle; each step covers {frac:.4f} of the output features of "
              f"{toks} tokens ({name}); tokens/s counts full-token equivalents")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(name, runner.t, args.options),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_weight_bytes(name):
    """Bytes of the weights one step reads per call (same count as Workload)."""
    cfg = workloads.CONFIGS[name]
    if name == "sq4096":
        return cfg.k * cfg.n * 2
    if name == "attn70b":
        nqkv = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
        return (nqkv + cfg.n_q_heads * cfg.head_dim) * cfg.hidden * 2
    if name == "mlp70b_w8":
        return 2 * cfg.hidden * cfg.ffn + 4 * (cfg.hidden + cfg.ffn)
    if name == "attn70b_decode":
        return 2 * cfg.n_kv_heads * cfg.past * cfg.head_dim * 2
    if name == "attn70b_prefill":
        return 2 * cfg.n_kv_heads * (cfg.past + max(cfg.tokens)) * cfg.head_dim * 2
    if name == "sp405b":
        return cfg.hidden * 2
    return 2 * cfg.hidden * cfg.ffn * 2


def rotation_copies(weight_bytes):
    """Weight copies rotated per call so each call reads weights evicted from L2."""
    if weight_bytes < 4 * L2_BYTES:
        return int(math.ceil(4 * L2_BYTES / weight_bytes))
    return 1


def workload_config(name, t, options, tokens=None):
    cfg = workloads.CONFIGS[name]
    desc = {
        "sq4096": "column-parallel projection W[4096,4096] bf16, t=2 column shards, decode T=1,8,64",
        "tiny": "MLP block H=256 F=1024, t=2, GeLU, biases, T=8",
        "mlp70b": "Llama-3-70B-shaped MLP decode H=8192 F=28672, GeLU, T=1,16,64",
        "mlp70b_w8": "Llama-3-70B-shaped MLP decode H=8192 F=28672, GeLU, T=1,16,64, "
                     "8-bit weights (FP8 E4M3 codes, one fp32 scale per row)",
        "attn70b": "Llama-3-70B-shaped attention projections prefill T=4096, QKV 8192->10240 "
                   "split by 64q/8kv heads, O-proj 8192->8192 row-split",
        "attn70b_decode": "attention core decode, 64 query / 8 key-value heads of 128 (t=8), "
                          "65536 cached tokens, T=1,2,4 new tokens per call",
        "attn70b_prefill": "attention core prefill, 64 query / 8 key-value heads of 128 (t=8), "
                           "a T=4096-token prompt, causal, its keys and values appended to "
                           "the per-head caches",
        "mlp70b_bwd": "backward pass of the Llama-3-70B-shaped MLP block H=8192 F=28672, GeLU, "
                      "t=8, T=4096 tokens: dx (fused backward shard sum), dW1, dW2, db1, db2",
        "sp405b": "sequence-parallel region of the 405B-shaped block: residual add + RMSNorm "
                  "of T=8192 token rows of H=16384 in 8 token shards",
        "mlp405b": "405B-shaped MLP prefill H=16384 F=53248, GeLU, T=8192, column-parallel "
                   "up-projection + row-parallel down-projection with the fused 8-shard sum",
    }[name]
    wb = workload_weight_bytes(name)
    rot = rotation_copies(wb) if name != "sp405b" else 1
    what = "KV caches" if name in ("attn70b_decode", "attn70b_prefill") else "weights"
    if tokens:
        desc += f" (token counts overridden: {list(tokens)})"
    if name == "attn70b_prefill":
        T0 = cfg.tokens[0]
        nqkv = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
        l2 = (f"KV caches rotated per call over {rot} copies ({rot * wb / 1e6:.0f} MB); qkv "
              f"{T0 * nqkv * 2 / 1e6:.0f} MB read and ctx {T0 * cfg.n_q_heads * cfg.head_dim * 2 / 1e6:.0f}"
              f" MB written per call: {(T0 * nqkv * 2 + T0 * cfg.n_q_heads * cfg.head_dim * 2 + wb) / 1e6:.0f}"
              f" MB per call > 126 MB L2")
    elif name == "sp405b":
        l2 = (f"y, residual, r, n: {cfg.tokens[0] * cfg.hidden * 2 / 1e6:.0f} MB each > 126 MB "
              f"L2, each read or written once per step")
    else:
        l2 = (f"{what} rotated per call over {rot} copies ({rot * wb / 1e6:.0f} MB >= 4x "
              f"the 126 MB L2): every call reads cold {what}" if rot > 1 else
              f"{what} {wb / 1e6:.0f} MB > 126 MB L2, read once per step")
    return {"workload": desc, "name": name, "tp_degree": t, "tokens": list(tokens or cfg.tokens),
            "parallelism": "replicas (per-GPU block, t logical shards on chip)",
            "l2": l2,
            "launch_options": options}


def run_ours(args, world, rank, local):
    import tensor_transformer_linear_column_b200 as tp
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    tp.load()
    tp.tp_set_launch_options(LAUNCH_OPTIONS[args.options])
    if args.decode_max_tokens is not None:
        tp.tp_set_decode_max_tokens(args.decode_max_tokens)
    wl = Workload(args.workload, args.tp, dev, rotate=True, tokens=args.tokens)
    stream = torch.cuda.Stream(device=dev)
    K, W = args.steps, args.warmup

    # graphs: one per rotation index (single step) and one of a full rotation
    use_graph = not args.no_graph
    g_single, g_rot = [], None
    with torch.cuda.stream(stream):
        for i in range(min(3, wl.rot) + 1):  # eager warm-up of each path
            wl.step(i)
    torch.cuda.synchronize()
    if use_graph:
        for i in range(wl.rot):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                wl.step(i)
            g_single.append(g)
        if wl.rot > 1:
            g_rot = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rot, stream=stream):
                for i in range(wl.rot):
                    wl.step(i)

    def run_steps(n, start=0):
        i = start
        if not use_graph:
            for _ in range(n):
                wl.step(i)
                i += 1
            return
        while n > 0:
            if g_rot is not None and i % wl.rot == 0 and n >= wl.rot:
                g_rot.replay()
                i += wl.rot
                n -= wl.rot
            else:
                g_single[i % wl.rot].replay()
                i += 1
                n -= 1

    with torch.cuda.stream(stream):
        run_steps(W)
    torch.cuda.synchronize()
    if tp.tp_device_error_check() != tp.TP_OK:
        raise RuntimeError("device-side timeout during warm-up")

    clk = ClockSampler(local)
    clk.start()
    barrier(world, dev)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        run_steps(K, start=W)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world, dev)
    clocks = clk.stop()
    ms = e0.elapsed_time(e1)
    ms_per_step = reduce_max(ms / K, world, dev)
    value = replica_value(wl.tokens_per_step, world, ms_per_step)
    if tp.tp_device_error_check() != tp.TP_OK:
        raise RuntimeError("device-side timeout during the timed region")

    # kernel attribution: each kernel type of the step timed alone (same inputs)
    power_capped = bool(clocks and "sw_power_cap" in clocks.get("reasons", []))
    roof = roofline(wl, ms_per_step, stream, use_graph, power_capped)
    if args.tokens:
        roof["traffic"] = None  # recorded captures are per launch of the workload's own sizes

    # end to end through the public API with host buffers (pinned)
    e2e = end_to_end(wl, stream, max(3, min(K, args.e2e_steps)), world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.tokens:
        v, steps, el, toks = time_oracle(args.workload, args.tp, budget_s=args.cpu_budget)
        cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{steps} full oracle step(s) of {toks} tokens in {el:.1f} s "
                         f"(fp64 numpy, {args.workload})"}

    if rank == 0:
        config = workload_config(args.workload, wl.t, args.options, args.tokens)
        if args.decode_max_tokens is not None:
            config["decode_max_tokens"] = args.decode_max_tokens
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0, sigma) bf16 inputs of the workload's shapes)",
            "config": config,
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": wl.launches_per_step * K,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    del g_single, g_rot
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def roofline(wl, ms_per_step, stream, use_graph, power_capped=False):
    peaks, src = load_peaks()
    if wl.bound() == "hbm":
        # the step is nothing but the streaming kernel(s); bytes are weights +
        # activations read once, duration = the timed region's average per step
        achieved = wl.step_bytes() / (ms_per_step / 1000.0) / 1e9
        peak = float(peaks["hbm_gbs"])
        unit = "GB/s"
        launches = wl.launches_per_step
        kernel = wl.hbm_kernel()
        traffic = recorded_traffic(kernel, wl.name)
        return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": traffic,
                "kernel": kernel, "launches_per_step": launches,
                "bytes_per_step": wl.step_bytes(), "peak_source": f"{src} hbm_gbs"}
    # tensor-bound: time each kernel of the step alone with events on the stream
    per_kernel = kernel_durations(wl, stream)
    name, (ms, flops) = max(per_kernel.items(), key=lambda kv: kv[1][0])
    achieved = flops / (ms / 1000.0) / 1e12
    # the sustained figure is the one measured under the power cap; use it when
    # the timed region ran power-capped, the burst figure otherwise
    key = "bf16_tflops_sustained" if power_capped else "bf16_tflops"
    peak = float(peaks.get(key, FALLBACK_PEAKS[key]))
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": recorded_traffic(name, wl.name),
            "kernel": name, "kernel_ms": ms, "flops_per_launch": flops,
            "peak_source": f"{src} {key}",
            "per_kernel_ms": {k: v[0] for k, v in per_kernel.items()}}


def kernel_durations(wl, stream, reps=5):
    """Average duration of each kernel of a prefill step, each launch between its
    own events (T > 128: both GEMMs run on the CTA-pair kernel)."""
    tp = wl.tp
    T = wl.Ts[0]
    out = {}
    if wl.name == "attn70b_prefill":
        # one call: the cache append (a copy of 2 nkv d values per token, about
        # 1 % of the time) and the attention kernel
        calls = {"attn_prefill2_kernel": (lambda: wl.step(0), wl.step_flops())}
    elif wl.name == "mlp70b_bwd":
        # one backward pass: z recompute, dz and h, dx with the shard sum, dW1,
        # dW2 (five CTA-pair GEMMs) and the two column sums, as one call
        calls = {"pair_gemm_kernel<backward>:five_gemms": (lambda: wl.step(0), wl.step_flops())}
    elif wl.name == "attn70b":
        cfg = wl.cfg
        wq, wo = wl.weights[0]
        nctx = cfg.n_q_heads * cfg.head_dim
        calls = {
            "pair_gemm_kernel<colpar>:qkv": (
                lambda: tp.tp_colpar_gemm_gelu(wl.xd[T], wq, None, wl.t, "none", out=wl.qkv),
                2 * T * cfg.hidden * wq.shape[0]),
            "pair_gemm_kernel<rowpar>:o_proj": (
                lambda: tp.tp_rowpar_gemm_reduce(wl.ctx, wo, None, wl.t, out=wl.outs[T]),
                2 * T * nctx * cfg.hidden),
        }
    else:
        w1, w2 = wl.weights[0]
        F, H = wl.cfg.ffn, wl.cfg.hidden
        h = torch.empty((T, F), dtype=torch.bfloat16, device=wl.dev)
        calls = {
            "pair_gemm_kernel<colpar>:up_gelu": (
                lambda: tp.tp_colpar_gemm_gelu(wl.xd[T], w1, wl.bias[0], wl.t, wl.cfg.act, out=h),
                2 * T * H * F),
            "pair_gemm_kernel<rowpar>:down_sum": (
                lambda: tp.tp_rowpar_gemm_reduce(h, w2, wl.bias[1], wl.t, out=wl.outs[T]),
                2 * T * F * H),
        }
    # the kernels of the step are timed interleaved (a, b, a, b, ...), each
    # between its own events, so both see the same clocks and power state
    names = list(calls)
    with torch.cuda.stream(stream):
        for name in names:
            calls[name][0]()
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)] for _ in names]
        for r in range(reps):
            for i, name in enumerate(names):
                ev[i][r][0].record(stream)
                calls[name][0]()
                ev[i][r][1].record(stream)
    torch.cuda.synchronize()
    for i, name in enumerate(names):
        ms = sum(a.elapsed_time(b) for a, b in ev[i]) / reps
        out[name] = (ms, calls[name][1])
    return out


def end_to_end(wl, stream, steps, world, dev):
    """Same metric through the public API with host (pinned) inputs and outputs.

    Every step copies its inputs host -> device and its output device -> host
    inside the timed region, pipelined as a serving loop runs them: the copy in
    of step i + 1 and the copy out of step i - 1 run on their own streams while
    step i computes, with the device inputs and outputs double-buffered and
    ordered by events (a buffer is refilled only after the step that read it,
    and rewritten only after its copy out)."""
    hx = {T: wl.xs[T].pin_memory() for T in wl.Ts}
    hy = {T: torch.empty_like(wl.outs[T], device="cpu").pin_memory() for T in wl.Ts}
    h2d = sum(x.numel() * x.element_size() for x in hx.values())
    d2h = sum(y.numel() * y.element_size() for y in hy.values())
    dx = [{T: torch.empty_like(wl.xd[T]) for T in wl.Ts} for _ in range(2)]
    dy = [{T: torch.empty_like(wl.outs[T]) for T in wl.Ts} for _ in range(2)]
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)]
          for k in ("x_ready", "x_free", "y_ready", "y_free")}
    used = [False, False]

    def run(n, start):
        for i in range(start, start + n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(ev["x_free"][b])
                for T in wl.Ts:
                    dx[b][T].copy_(hx[T], non_blocking=True)
                ev["x_ready"][b].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(ev["x_ready"][b])
                if used[b]:
                    stream.wait_event(ev["y_free"][b])
                wl.step(i, xs=dx[b], outs=dy[b])
                ev["x_free"][b].record(stream)
                ev["y_ready"][b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["y_ready"][b])
                for T in wl.Ts:
                    hy[T].copy_(dy[b][T], non_blocking=True)
                ev["y_free"][b].record(s_out)
            used[b] = True
        # the region ends when the last outputs are on the host
        for b in range(2):
            if used[b]:
                stream.wait_event(ev["y_free"][b])

    run(3, 0)
    torch.cuda.synchronize()
    barrier(world, dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    # nothing of the timed steps starts before e0
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    run(steps, 3)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(e0.elapsed_time(e1) / steps, world, dev)
    barrier(world, dev)
    return {"value": replica_value(wl.tokens_per_step, world, ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": steps, "pipelined": "copy in of step i+1 and copy out of step i-1 "
                                         "overlap step i (double-buffered device x and y)"}


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about a second of work for the workload)")
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mlp405b", choices=sorted(workloads.CONFIGS))
    ap.add_argument("--tp", type=int, default=None, help="tp degree (default: the workload's)")
    ap.add_argument("--options", choices=sorted(LAUNCH_OPTIONS), default="pdl+static_weights",
                    help="library launch options: the workload's weights are loaded once and "
                         "never written, so kernels may prefetch them under PDL")
    ap.add_argument("--tokens", type=int, nargs="+", default=None,
                    help="override the workload's token counts (smaller captures for ncu); "
                         "not a headline configuration")
    ap.add_argument("--decode-max-tokens", type=int, default=None,
                    help="token count up to which calls take the weight-streaming kernel "
                         "(the library's default is 128)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    args = ap.parse_args(argv)
    steps, warmup = DEFAULT_STEPS.get(args.workload, (200, 10))
    if args.steps is None:
        args.steps = steps
    if args.warmup is None:
        args.warmup = warmup
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    return args


def main(argv=None):
    args = parse(argv)
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
