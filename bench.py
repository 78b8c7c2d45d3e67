#!/usr/bin/env python
"""Benchmark of the sparse-attention layer (IndexPool append -> 32-head
indexer -> top-512 blocks -> sparse MLA attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl spx|reference]
                    [--workload 1m|mid|dense|tiny|prefill]

Default workload: 1M-token decode, 4 sequences per GPU, 64 MLA heads, 600
planted needle blocks per sequence.  One step = one fused decode call for the
whole batch: append the new token's indexer key, score all 262,144 pooled
blocks of every sequence, keep the top 512, attend over the 2,051 gathered
latent rows.  Prints one JSON line (rank 0).

Multi-GPU (torchrun): every rank runs its own 4 sequences (weak scaling, no
data-path collective); the timed region is bracketed by barriers and the
reported time is the max over ranks.

--impl reference times the fp64 CPU oracle on this machine's host cores on
the same workload (each step one query), rank 0 only.
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
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "index_score_traffic.json")
SCORE_SRC = os.path.join(ROOT, "long_context_decode_indexpool_b200", "csrc", "index_score.cu")

GEN_CHUNK_TOKENS = 1 << 18  # tokens per device generation chunk


def spx_module():
    import long_context_decode_indexpool_b200 as spx
    return spx


# ---------------------------------------------------------------------------
# device-side workload construction (shared with the GPU tests)
# ---------------------------------------------------------------------------
class DecodeState:
    """Caches and step inputs of a decode workload on one device.

    Sequences b_offset .. b_offset+B-1 of the workload recipe.  The pooled
    cache holds the first L-1 tokens (built with spx_pool_append), the tail
    the last 3 of them; each step appends token L-1 and queries with n = L.
    keys="int8" keeps the pooled keys in the INT8 cache (int8 codes plus one
    scale per block, spx_pool_append_i8 / spx_decode_fused_i8).
    """

    def __init__(self, w: synth.Workload, device, b_offset: int = 0, B: int | None = None,
                 build_latent: bool = True, keys: str = "bf16"):
        spx = spx_module()
        self.w = w
        self.device = device
        self.b_offset = b_offset
        self.B = B = w.B if B is None else B
        self.L = L = w.L
        self.H = w.heads
        self.d = spx.dims(w.heads, w.sm_scale)
        self.pool_w = w.pool_weights().astype(np.float32)
        self.cap_blk = L // synth.POOL
        self.cap_tok = L
        bf16 = torch.bfloat16
        assert keys in ("bf16", "int8")
        self.keys = keys
        self.i8 = keys == "int8"
        self.pooled = torch.zeros(B, self.cap_blk, synth.IDX_DIM,
                                  dtype=torch.int8 if self.i8 else bf16, device=device)
        self.k_scale = (torch.zeros(B, self.cap_blk, dtype=torch.float32, device=device)
                        if self.i8 else None)
        self.tail = torch.zeros(B, synth.POOL - 1, synth.IDX_DIM, dtype=bf16, device=device)
        self.needles = {}
        for b in range(B):
            bg = b_offset + b
            if w.needles:
                self.needles[b] = torch.as_tensor(w.needle_blocks(bg), device=device)
            t = 0
            while t < L - 1:
                t1 = min(L - 1, t + GEN_CHUNK_TOKENS)
                raw = w.raw_keys_t(bg, t, t1, device, self.needles.get(b)).view(bf16)
                ln = torch.tensor([t], dtype=torch.int64, device=device)
                if self.i8:
                    spx.spx_pool_append_i8(self.d, 1, raw.reshape(1, t1 - t, synth.IDX_DIM),
                                           t1 - t, self.pool_w, self.tail[b:b + 1],
                                           self.pooled[b:b + 1], self.k_scale[b:b + 1],
                                           self.cap_blk, ln, t1)
                else:
                    spx.spx_pool_append(self.d, 1, raw.reshape(1, t1 - t, synth.IDX_DIM), t1 - t,
                                        self.pool_w, self.tail[b:b + 1], self.pooled[b:b + 1],
                                        self.cap_blk, ln, t1)
                t = t1
        self.latent = None
        if build_latent:
            self.latent = torch.empty(B, L, synth.LATENT, dtype=bf16, device=device)
            for b in range(B):
                for t in range(0, L, GEN_CHUNK_TOKENS):
                    t1 = min(L, t + GEN_CHUNK_TOKENS)
                    self.latent[b, t:t1].view(torch.int16).copy_(
                        w.latent_t(b_offset + b, t, t1, device))
        rows = np.arange(b_offset, b_offset + B)
        self.raw_new = torch.stack([
            w.raw_keys_t(b_offset + b, L - 1, L, device, self.needles.get(b)).view(bf16)
            for b in range(B)])  # [B, 1, 128]
        self.q_idx = torch.from_numpy(w.q_idx_np(rows).view(np.int16)).to(device).view(bf16)
        self.w_head = torch.from_numpy(w.w_head_np(rows)).to(device)
        self.q = torch.from_numpy(w.q_np(rows).view(np.int16)).to(device).view(bf16)
        self.len_dev = torch.full((B,), L - 1, dtype=torch.int64, device=device)
        self.max_len = L
        self.out = torch.empty(B, self.H, synth.LATENT, dtype=bf16, device=device)
        self.lse = torch.empty(B, self.H, dtype=torch.float32, device=device)
        self.idx = torch.empty(B, synth.TOPK_BLOCKS, dtype=torch.int32, device=device)
        self.count = torch.empty(B, dtype=torch.int32, device=device)
        self.ws = spx.workspace(spx.spx_decode_workspace_size(self.d, B, L), device)
        self._call = None
        torch.cuda.synchronize(device)

    def step(self, timing=None, raw_new=None, q_idx=None, w_head=None, q=None, out=None,
             stream=None):
        spx = spx_module()
        if self._call is None:  # device pointers and host arguments, resolved once
            self._call = dict(
                pool_w=spx.pool_weights(self.pool_w), tail=self.tail.data_ptr(),
                pooled=self.pooled.data_ptr(), len_dev=self.len_dev.data_ptr(),
                latent=self.latent.data_ptr(), lse=self.lse.data_ptr(), idx=self.idx.data_ptr(),
                count=self.count.data_ptr(), ws=self.ws.data_ptr(),
                ws_bytes=self.ws.numel() * self.ws.element_size(),
                stream=torch.cuda.current_stream(self.device).cuda_stream)
        c = self._call
        raw_new = self.raw_new if raw_new is None else raw_new
        q_idx = self.q_idx if q_idx is None else q_idx
        w_head = self.w_head if w_head is None else w_head
        q = self.q if q is None else q
        out = self.out if out is None else out
        if self.i8:
            spx.spx_decode_fused_i8(
                self.d, self.B, raw_new, c["pool_w"], c["tail"], c["pooled"], self.k_scale,
                self.cap_blk, c["len_dev"], q_idx, w_head, q, c["latent"], self.cap_tok,
                self.max_len, out, c["lse"], c["idx"], c["count"], c["ws"], ws_bytes=c["ws_bytes"],
                timing=timing, stream=c["stream"] if stream is None else stream)
        else:
            spx.spx_decode_fused(
                self.d, self.B, raw_new, c["pool_w"], c["tail"], c["pooled"], self.cap_blk,
                c["len_dev"], q_idx, w_head, q, c["latent"], self.cap_tok, self.max_len, out,
                c["lse"], c["idx"], c["count"], c["ws"], ws_bytes=c["ws_bytes"], timing=timing,
                stream=c["stream"] if stream is None else stream)

    # ---- host copies of what the oracle needs (generator output) ----
    def raw_keys_host(self, b: int) -> np.ndarray:
        """All L raw keys of local sequence b, bf16 bits [L, 128]."""
        out = np.empty((self.L, synth.IDX_DIM), dtype=np.uint16)
        for t in range(0, self.L, GEN_CHUNK_TOKENS):
            t1 = min(self.L, t + GEN_CHUNK_TOKENS)
            out[t:t1] = self.w.raw_keys_t(self.b_offset + b, t, t1, self.device,
                                          self.needles.get(b)).cpu().numpy().view(np.uint16)
        return out

    def latent_rows_host(self, b: int, positions) -> np.ndarray:
        return self.w.latent_np(self.b_offset + b, positions)


class PrefillState:
    """Caches and inputs of a chunked-prefill workload (batch 1): a cache of
    pos0 tokens built with spx_pool_append (spx_pool_append_i8 with
    keys="int8": int8 codes plus one scale per block), then T new tokens."""

    def __init__(self, w: synth.Workload, device, pos0: int | None = None, T: int | None = None,
                 keys: str = "bf16"):
        spx = spx_module()
        self.w = w
        self.i8 = keys == "int8"
        self.device = device
        self.pos0 = pos0 = w.L if pos0 is None else pos0
        self.T = T = w.T if T is None else T
        self.H = w.heads
        self.d = spx.dims(w.heads, w.sm_scale)
        self.pool_w = w.pool_weights().astype(np.float32)
        total = pos0 + T
        self.cap_blk = (total + 3) // 4
        self.cap_tok = total
        bf16 = torch.bfloat16
        self.pooled = torch.zeros(1, self.cap_blk, synth.IDX_DIM,
                                  dtype=torch.int8 if self.i8 else bf16, device=device)
        self.k_scale = (torch.zeros(1, self.cap_blk, dtype=torch.float32, device=device)
                        if self.i8 else None)
        self.tail = torch.zeros(1, 3, synth.IDX_DIM, dtype=bf16, device=device)
        t = 0
        while t < pos0:
            t1 = min(pos0, t + GEN_CHUNK_TOKENS)
            raw = w.raw_keys_t(0, t, t1, device).view(bf16)
            ln = torch.tensor([t], dtype=torch.int64, device=device)
            if self.i8:
                spx.spx_pool_append_i8(self.d, 1, raw.reshape(1, t1 - t, synth.IDX_DIM), t1 - t,
                                       self.pool_w, self.tail, self.pooled, self.k_scale,
                                       self.cap_blk, ln, t1)
            else:
                spx.spx_pool_append(self.d, 1, raw.reshape(1, t1 - t, synth.IDX_DIM), t1 - t,
                                    self.pool_w, self.tail, self.pooled, self.cap_blk, ln, t1)
            t = t1
        self.latent = torch.empty(total, synth.LATENT, dtype=bf16, device=device)
        for t in range(0, total, GEN_CHUNK_TOKENS):
            t1 = min(total, t + GEN_CHUNK_TOKENS)
            self.latent[t:t1].view(torch.int16).copy_(w.latent_t(0, t, t1, device))
        rows = np.arange(pos0, pos0 + T)
        self.raw_k = w.raw_keys_t(0, pos0, total, device).view(bf16)
        self.q_idx = torch.from_numpy(w.q_idx_np(rows).view(np.int16)).to(device).view(bf16)
        self.w_head = torch.from_numpy(w.w_head_np(rows)).to(device)
        self.q = torch.from_numpy(w.q_np(rows).view(np.int16)).to(device).view(bf16)
        self.out = torch.empty(T, self.H, synth.LATENT, dtype=bf16, device=device)
        self.lse = torch.empty(T, self.H, dtype=torch.float32, device=device)
        self.idx = torch.empty(T, synth.TOPK_BLOCKS, dtype=torch.int32, device=device)
        self.count = torch.empty(T, dtype=torch.int32, device=device)
        self.ws = spx.workspace(spx.spx_prefill_workspace_size(self.d, T, pos0), device)
        torch.cuda.synchronize(device)

    def step(self, timing=None):
        spx = spx_module()
        if self.i8:
            spx.spx_prefill_chunk_i8(self.d, self.T, self.raw_k, self.pool_w, self.tail,
                                     self.pooled, self.k_scale, self.cap_blk, self.pos0,
                                     self.q_idx, self.w_head, self.q, self.latent, self.cap_tok,
                                     self.out, self.lse, self.idx, self.count, self.ws,
                                     timing=timing)
            return
        spx.spx_prefill_chunk(self.d, self.T, self.raw_k, self.pool_w, self.tail, self.pooled,
                              self.cap_blk, self.pos0, self.q_idx, self.w_head, self.q,
                              self.latent, self.cap_tok, self.out, self.lse, self.idx, self.count,
                              self.ws, timing=timing)

    def raw_keys_host(self) -> np.ndarray:
        total = self.pos0 + self.T
        out = np.empty((total, synth.IDX_DIM), dtype=np.uint16)
        for t in range(0, total, GEN_CHUNK_TOKENS):
            t1 = min(total, t + GEN_CHUNK_TOKENS)
            out[t:t1] = self.w.raw_keys_t(0, t, t1, self.device).cpu().numpy().view(np.uint16)
        return out


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------
def measured_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def recorded_traffic(kernel_key: str):
    """ncu DRAM bytes per launch recorded for the current scoring-kernel source, or None."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        sha = hashlib.sha256(open(SCORE_SRC, "rb").read()).hexdigest()
        e = rec.get(kernel_key)
        if e and e.get("source_sha256") == sha:
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clock and throttle-reason samples while the timed region runs.

    NVML is polled from a host thread every ~0.2 ms, so that even a timed
    region of a millisecond or two holds several samples; nvidia-smi (one
    sample per 50 ms) is the fallback when NVML is not importable."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int, period_s: float = 2e-4):
        self.samples = []  # (sm_mhz, sm_max_mhz, set of reason names)
        self.period = period_s
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.source = None
        self.gpu_id = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu_id = None
        self.nvml = None
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.handle = (pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id) if self.gpu_id
                           else pynvml.nvmlDeviceGetHandleByIndex(device_index))
            self.nvml = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.reason_bits = (
                ("hw_slowdown", pynvml.nvmlClocksEventReasonHwSlowdown),
                ("hw_thermal_slowdown", pynvml.nvmlClocksEventReasonHwThermalSlowdown),
                ("sw_thermal_slowdown", pynvml.nvmlClocksEventReasonSwThermalSlowdown),
                ("sw_power_cap", pynvml.nvmlClocksEventReasonSwPowerCap))
        except Exception:
            self.nvml = None

    def _nvml_sample(self):
        n = self.nvml
        mhz = float(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
        bits = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        return (mhz, self.max_mhz, {name for name, b in self.reason_bits if bits & b})

    def _smi_cmd(self, loop: bool):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        if loop:
            cmd += ["-lms", "50"]
        return cmd

    @classmethod
    def _parse_smi(cls, line):
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            return None
        try:
            sm, smax = float(parts[1]), float(parts[2])
        except ValueError:
            return None
        return (sm, smax, {n for n, v in zip(cls.NAMES, parts[5:9]) if v.lower() in ("active", "1")})

    def start(self):
        self.samples = []
        self.stop_flag.clear()
        if self.nvml is not None:
            self.source = "nvml"

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        self.samples.append(self._nvml_sample())
                    except Exception:
                        pass
                    time.sleep(self.period)
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 2.0:
                time.sleep(1e-4)
            self.samples.clear()  # keep only samples taken once the region has started
            return
        self.source = "nvidia-smi"
        try:
            self.proc = subprocess.Popen(self._smi_cmd(True), stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return

        def reader():
            for line in self.proc.stdout:
                r = self._parse_smi(line)
                if r:
                    self.samples.append(r)
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)
        self.samples.clear()

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if not self.samples:  # region shorter than one sampling period
            try:
                if self.nvml is not None:
                    self.samples = [self._nvml_sample()]
                else:
                    out = subprocess.run(self._smi_cmd(False), capture_output=True, text=True,
                                         timeout=20)
                    self.samples = [r for r in map(self._parse_smi, out.stdout.splitlines()) if r]
            except Exception:
                pass

    def summary(self):
        sm = [x[0] for x in self.samples]
        smax = self.samples[-1][1] if self.samples else None
        reasons = set()
        for x in self.samples:
            reasons |= x[2]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "sm_mhz_min": min(sm) if sm else None, "source": self.source}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a per-rank value (the slowest rank's time) over the process group."""
    if world == 1:
        return value
    if torch.distributed.get_backend() == "gloo":
        device = torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def shard_offset(rank: int, per_rank: int) -> int:
    """First sequence of a rank: ranks take disjoint, consecutive sequences."""
    return rank * per_rank


def score_algorithmic_bytes(nblk_per_row, rows: int, keys: str = "bf16") -> int:
    """Bytes the scoring kernel must read (the step's own accounting, which
    leaves out the scores it materialises): every pooled key once (256 B;
    INT8 cache: 128 B of codes + a 4 B scale), plus each query row (8 KiB;
    INT8: 4 KiB of codes) and its head weights (128 B)."""
    if keys == "int8":
        per_blk, per_row = synth.IDX_DIM + 4, synth.IDX_HEADS * synth.IDX_DIM + synth.IDX_HEADS * 4
    else:
        per_blk, per_row = synth.IDX_DIM * 2, synth.IDX_HEADS * synth.IDX_DIM * 2 + synth.IDX_HEADS * 4
    return int(sum(nblk_per_row)) * per_blk + rows * per_row


def score_write_bytes(nblk_per_row) -> int:
    """Bytes of fp32 scores the scoring kernel writes (overhead outside the
    algorithmic accounting)."""
    return int(sum(nblk_per_row)) * 4


def step_algorithmic_bytes(B: int, L: int, heads: int, keys: str = "bf16") -> int:
    """Bytes one decode step must move for B queries that see L tokens each:
    pooled keys, the selected latent rows (512 blocks of 4 tokens plus the
    partial tail, 1 KiB each), the indexer query and head weights, the MLA
    query and the output."""
    nblk = L // synth.POOL
    S = min(nblk, synth.TOPK_BLOCKS) * synth.POOL + L % synth.POOL
    per_q = (score_algorithmic_bytes([nblk], 1, keys) + S * synth.LATENT * 2
             + 2 * heads * synth.LATENT * 2)
    return B * per_q


def attention_flops_prefill(pos0: int, T: int, heads: int) -> int:
    """QK^T and PV flops of a prefill chunk: 4 H D per attended token."""
    tot = 0
    for t in range(T):
        n = pos0 + t + 1
        tot += min(n // synth.POOL, synth.TOPK_BLOCKS) * synth.POOL + n % synth.POOL
    return 4 * heads * synth.LATENT * tot


def score_algorithmic_flops_prefill(pos0: int, T: int) -> int:
    tot = 0
    for t in range(T):
        tot += (pos0 + t + 1) // 4
    return 2 * synth.IDX_HEADS * synth.IDX_DIM * tot


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
class OracleDecodeSample:
    """Host inputs of decode queries and a timed oracle step per query."""

    def __init__(self, w: synth.Workload, device, b_offset=0):
        import oracle
        self.oracle = oracle
        self.w = w
        self.pw = w.pool_weights()
        self.L = w.L
        self.device = device
        self.b_offset = b_offset
        self.cache = {}

    def prepare(self, b):
        if b in self.cache:
            return self.cache[b]
        w = self.w
        bg = self.b_offset + b
        needle = torch.as_tensor(w.needle_blocks(bg), device=self.device) if w.needles else None
        raw = np.empty((self.L, synth.IDX_DIM), dtype=np.uint16)
        for t in range(0, self.L, GEN_CHUNK_TOKENS):
            t1 = min(self.L, t + GEN_CHUNK_TOKENS)
            if self.device is not None:
                raw[t:t1] = w.raw_keys_t(bg, t, t1, self.device, needle).cpu().numpy().view(np.uint16)
            else:
                raw[t:t1] = w.raw_keys_np(bg, t, t1)
        # the cache as earlier steps left it: pooled keys of every complete block
        # before the new token (untimed set-up)
        pooled = self.oracle.pool(raw[: self.L - 1], self.pw)
        rows = np.array([bg])
        item = dict(raw=raw, pooled=pooled, q_idx=w.q_idx_np(rows)[0],
                    w_head=w.w_head_np(rows)[0].astype(np.float64), q=w.q_np(rows)[0])
        self.cache[b] = item
        return item

    def run_query(self, b, nthreads=0):
        """One decode step of sequence b in the oracle; returns (seconds, result)."""
        o = self.oracle
        it = self.prepare(b)
        bg = self.b_offset + b
        t0 = time.perf_counter()
        last = o.pool(it["raw"][self.L - 4: self.L], self.pw)  # the block the new token completes
        pooled = np.concatenate([it["pooled"], last], axis=0)
        s, idx, pos = o.select_query(it["q_idx"], it["w_head"], pooled, self.L, nthreads=nthreads)
        t1 = time.perf_counter()
        rows = self.w.latent_np(bg, pos)  # gather (input generation, not timed)
        t2 = time.perf_counter()
        out, lse = o.attention(it["q"], rows, self.w.sm_scale)
        t3 = time.perf_counter()
        return (t1 - t0) + (t3 - t2), dict(scores=s, idx=idx, positions=pos, out=out, lse=lse)


def cpu_baseline(w, device, budget_s=12.0):
    import oracle
    samp = OracleDecodeSample(w, device)
    nthreads = oracle.threads(0)
    total_t, n = 0.0, 0
    for b in range(w.B):
        dt, _ = samp.run_query(b, nthreads)
        total_t += dt
        n += 1
        if total_t >= budget_s:
            break
    return {"value": n / total_t, "unit": "queries/s", "cores": nthreads, "kind": "oracle",
            "sample": f"{n} of the {w.B} decode queries of {w.name} (full 1M-token scoring, "
                      f"top-512, attention over the gathered rows), fp64, {total_t:.2f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = synth.workload(args.workload)
    if w.kind != "decode":
        print(json.dumps({"impl": "reference", "unavailable": "reference arm implemented for decode workloads"}))
        return 0
    device = torch.device("cuda", 0) if torch.cuda.is_available() else None
    samp = OracleDecodeSample(w, device)
    nthreads = oracle.threads(0)
    for i in range(args.warmup):
        samp.run_query(i % w.B, nthreads)
    tot = 0.0
    for i in range(args.steps):
        dt, _ = samp.run_query(i % w.B, nthreads)
        tot += dt
    value = args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
        "config": decode_config(w, w.B, w.L, w.heads, max(1, args.gpus), args.keys == "int8"),
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"one query of {w.name} per step (a bounded sample of its "
                                   f"{w.B} queries; value = queries / oracle time)"},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


METRIC = "sparse-attn decode queries/s at 1M ctx; achieved HBM GB/s vs 8 TB/s peak"


def decode_config(w, B: int, L: int, heads: int, world: int, i8: bool = False) -> dict:
    """The `config` of a decode line; both arms (this library and the oracle)
    report the same dict for the same workload."""
    return {"workload": w.name, "batch_per_gpu": B, "context": L, "heads": heads,
            "indexer": "32 heads x 128, pool 4, top-512 blocks", "latent": 512,
            "pooled_keys": "int8 codes + fp32 scale per block" if i8 else "bf16",
            "parallelism": f"dp{world} (independent sequences)",
            "l2": "inputs larger than L2 (pooled keys + 4 GiB latent per GPU)"}


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def run_decode(args, world, rank, local):
    spx = spx_module()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.workload(args.workload)
    st = DecodeState(w, device, b_offset=shard_offset(rank, w.B), keys=args.keys)
    B, L = st.B, st.L
    stream = torch.cuda.current_stream(device)

    for _ in range(args.warmup):
        st.step()
    torch.cuda.synchronize(device)
    if spx.spx_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    K = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device.index)
    clocks.start()
    n0 = spx.spx_launch_count()
    ev0.record(stream)
    for _ in range(K):
        st.step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    launches = spx.spx_launch_count() - n0
    clocks.stop()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world, device)
    score_avg = time_scoring_launches(st, stream, max(8, min(K, 64)))

    # ---- end to end: host buffers in, host result out, every step ----------
    e2e_ms, h2d, d2h, e2e_mode = run_e2e(st, stream, K, args.warmup, world, device)
    if spx.spx_device_error() != 0:
        raise RuntimeError("device error during the timed region")

    if rank != 0:
        return None
    hbm, bf16, bf16s, src = measured_peaks()
    nblk = [L // synth.POOL] * B
    alg = score_algorithmic_bytes(nblk, B, args.keys)
    achieved = alg / (score_avg * 1e-3) / 1e9
    step_bytes = step_algorithmic_bytes(B, L, st.H, args.keys)
    step_gbs = step_bytes / (ms_max / K * 1e-3) / 1e9
    queries = B * world * K
    i8 = args.keys == "int8"
    line = {
        "metric": METRIC,
        "value": queries / (ms_max * 1e-3),
        "unit": "queries/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_max / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8 indexer keys and queries (s32 dots), bf16 attention" if i8 else "bf16",
        "data": "synthetic (seeded generator; int-valued indexer keys, dyadic pool weights, "
                "600 needles/seq, N(0,1) latent)",
        "config": decode_config(w, B, L, st.H, world, i8),
        "roofline": {"bound": "hbm",
                     "kernel": "k_index_score (decode scoring" + (", INT8 cache)" if i8 else ")"),
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_source": f"{src} hbm_gbs",
                     "traffic": None if i8 else recorded_traffic("decode_1m"),
                     "algorithmic_bytes_per_launch": alg,
                     "score_write_bytes_per_launch": score_write_bytes(nblk),
                     "avg_launch_us": score_avg * 1e3,
                     "timed": "separate pass after the timed region, events around the launch",
                     "vs_8tbs": achieved / 8000.0},
        "roofline_step": {"bound": "hbm", "algorithmic_bytes_per_step": step_bytes,
                          "achieved": step_gbs, "unit": "GB/s", "peak": hbm,
                          "frac": step_gbs / hbm, "peak_source": f"{src} hbm_gbs",
                          "frac_of_8tbs": step_gbs / 8000.0},
        "e2e": {"value": queries / (e2e_ms * 1e-3), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "launch": e2e_mode},
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
    }
    return line


def run_e2e(st, stream, K: int, warmup: int, world: int, device):
    """K decode steps through the public call with host buffers: every step
    copies its inputs (new raw key, indexer query and weights, MLA query:
    one packed pinned buffer, one copy) to the device, runs the fused call,
    and copies the output back to pinned host memory; the host waits for
    every step's output, one step behind (it enqueues step k, then waits for
    step k-1).  The copies run on two more streams, one per direction, into
    two alternating device buffers, so step k+1's inputs and step k-1's output
    move while step k computes; the fused call of each buffer pair is replayed
    from a captured CUDA graph (eager calls if capture is unavailable).
    Timed by the host
    clock from the first copy to the last output in host memory (max over
    ranks).  Returns (ms, h2d bytes per step, d2h bytes per step, mode)."""
    ins = (st.raw_new, st.q_idx, st.w_head, st.q)
    sizes = [t.numel() * t.element_size() for t in ins]
    offs = [0]
    for n in sizes[:-1]:
        offs.append(offs[-1] + (n + 255) // 256 * 256)
    total = offs[-1] + sizes[-1]
    h_in = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    for t, o, n in zip(ins, offs, sizes):
        h_in[o:o + n].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
    d_in = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]
    views = [tuple(d[o:o + n].view(t.dtype).view(t.shape) for t, o, n in zip(ins, offs, sizes))
             for d in d_in]
    d_out = [torch.empty_like(st.out) for _ in range(2)]
    h_out = [torch.empty(st.out.shape, dtype=st.out.dtype, pin_memory=True) for _ in range(2)]
    d2h = h_out[0].numel() * h_out[0].element_size()

    def compute(i, s):
        raw, qi, wh, q = views[i]
        st.step(raw_new=raw, q_idx=qi, w_head=wh, q=q, out=d_out[i], stream=s.cuda_stream)

    graphs = None
    try:
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            compute(0, cap)  # (warms the library's per-device caches on this stream)
        cap.synchronize()
        graphs = []
        for i in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                compute(i, cap)
            graphs.append(g)
        stream.wait_stream(cap)
    except Exception:
        graphs = None
    # one stream per direction: an input copy must not queue behind the
    # previous step's output copy, which waits for that step's compute
    h2d, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    in_ready, used, out_home = ([ev(), ev()] for _ in range(3))

    def run(n):
        for k in range(n):
            i = k & 1
            with torch.cuda.stream(h2d):
                if k >= 2:
                    h2d.wait_event(used[i])  # step k-2 has finished with d_in[i]
                d_in[i].copy_(h_in, non_blocking=True)
                in_ready[i].record(h2d)
            stream.wait_event(in_ready[i])
            if k >= 2:
                stream.wait_event(out_home[i])  # step k-2's output has left d_out[i]
            if graphs is not None:
                graphs[i].replay()
            else:
                compute(i, stream)
            used[i].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(used[i])
                h_out[i].copy_(d_out[i], non_blocking=True)
                out_home[i].record(d2h_s)
            if k >= 1:
                out_home[i ^ 1].synchronize()  # the host has step k-1's output
        out_home[(n - 1) & 1].synchronize()

    run(max(warmup, 2))
    barrier(world)
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    run(K)
    ms = (time.perf_counter() - t0) * 1e3
    torch.cuda.synchronize(device)
    return (max_over_ranks(ms, world, device), total, d2h,
            "graph replay" if graphs is not None else "eager")


def time_scoring_launches(st, stream, n: int) -> float:
    """Average duration (ms) of the decode scoring kernel, from CUDA events
    the fused call records on its stream around that launch, over n extra
    steps run after the timed region (an event between two launches stops
    the next one from starting early, so the timed steps carry none)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:  # torch creates its events on first record
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for ev in evs:
        st.step(timing=ev)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / n


def run_indexshare(args, world, rank, local):
    """IndexShare decode ([W3] "IndexShare는 관련 토큰을 찾는 비용을 낮춘다": one
    indexer per group of sparse layers): per step, layer 0 runs the whole path
    (append, scores, top-512, attention) and the other N-1 layers run only the
    attention on layer 0's selection, each with its own query and latent cache.
    Reports amortised queries/s per layer."""
    spx = spx_module()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.workload(args.workload)
    st = DecodeState(w, device, b_offset=shard_offset(rank, w.B))
    B, L, H, N = st.B, st.L, st.H, args.indexshare
    g = torch.Generator(device=device).manual_seed(1234 + rank)
    lat = [torch.randn(B, st.cap_tok, synth.LATENT, generator=g, device=device).to(torch.bfloat16)
           for _ in range(N - 1)]
    qs = [(torch.randn(B, H, synth.LATENT, generator=g, device=device) * synth.MLA_Q_SCALE)
          .to(torch.bfloat16) for _ in range(N - 1)]
    outs = [torch.empty_like(st.out) for _ in range(N - 1)]
    n_vis = torch.full((B,), L, dtype=torch.int64, device=device)  # after the append
    ws_a = spx.workspace(spx.spx_attn_workspace_size(st.d, B, L), device)
    stream = torch.cuda.current_stream(device)

    def step():
        st.step()
        for l in range(N - 1):
            spx.spx_sparse_mla_attn(st.d, B, qs[l], lat[l], st.cap_tok * synth.LATENT, st.cap_tok,
                                    st.idx, st.count, n_vis, L, outs[l], None, ws_a)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    K = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(device)
    ev0.record(stream)
    for _ in range(K):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    if spx.spx_device_error() != 0:
        raise RuntimeError("device error during the timed region")
    if rank != 0:
        return None
    per_layer_ms = ms / K / N
    return {"metric": f"IndexShare decode: amortised per-layer queries/s, one indexer per {N} layers",
            "value": B * world / (per_layer_ms * 1e-3), "unit": "queries/s per layer",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_layer": per_layer_ms,
            "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "dtype": "bf16",
            "data": "synthetic (layer 0 as the decode workload; other layers N(0,1) latent, "
                    "N(0,1)/sqrt(512) queries)",
            "config": {"workload": w.name, "layers_per_indexer": N, "batch_per_gpu": B,
                       "context": L, "heads": H}}


def run_host_latent(args, world, rank, local):
    """Decode with the latent cache in pinned host memory ([W3] "HiSparse는 전체
    이력을 GPU 밖으로 옮긴다": the full history lives off the GPU and only the
    selected rows are fetched); pooled keys stay in HBM.  Two ways are timed:
    (1) the fused call reading the 2048 selected rows per query straight from
    host memory every step; (2) a device working set of --ws-slots 4-token
    blocks per sequence (spx_sparse_mla_attn_ws), where a step fetches only
    the selected blocks not already resident.  The indexer query cycles over
    four different queries, so that consecutive steps select partly
    different blocks; the hit rate is reported."""
    spx = spx_module()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.workload(args.workload)
    st = DecodeState(w, device, b_offset=shard_offset(rank, w.B))
    B, L = st.B, st.L
    host_lat = st.latent.cpu().pin_memory()
    st.latent = None  # the device copy is released; the calls read the host rows
    torch.cuda.empty_cache()
    st.latent = host_lat  # step() passes its data_ptr (mapped under unified addressing)
    st._call = None
    stream = torch.cuda.current_stream(device)
    g = torch.Generator(device=device).manual_seed(99 + rank)
    qs = [st.q_idx] + [torch.randint(-4, 5, st.q_idx.shape, generator=g, device=device)
                       .to(torch.bfloat16) for _ in range(3)]
    K = args.steps

    def timed(fn):
        for i in range(args.warmup):
            fn(i)
        torch.cuda.synchronize(device)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(device)
        ev0.record(stream)
        for i in range(K):
            fn(args.warmup + i)
        ev1.record(stream)
        torch.cuda.synchronize(device)
        if spx.spx_device_error() != 0:
            raise RuntimeError("device error during the timed region")
        return max_over_ranks(ev0.elapsed_time(ev1), world, device)

    # (1) zero-copy: the fused call reads the selected rows from host memory
    ms_zc = timed(lambda i: st.step(q_idx=qs[i % 4]))

    # (2) working set: pooled-key append, scores and top-k on the device, then
    # attention through the slot pool
    nslots = args.ws_slots
    cap_blk = L // synth.POOL
    pool = torch.zeros(B, nslots + 1, 4, synth.LATENT, dtype=torch.bfloat16, device=device)
    slot_blk = torch.full((B, nslots), -1, dtype=torch.int32, device=device)
    blk_slot = torch.full((B, cap_blk), -1, dtype=torch.int32, device=device)
    stamp = torch.full((B, nslots), -1, dtype=torch.int32, device=device)
    hand = torch.zeros(B, dtype=torch.int32, device=device)
    stats = torch.zeros(B, 2, dtype=torch.int64, device=device)
    ws = spx.workspace(spx.spx_ws_workspace_size(st.d, B, nslots), device)
    ws_t = spx.workspace(spx.spx_topk_workspace_size(st.d, B, L), device)
    n_vis = torch.full((B,), L, dtype=torch.int64, device=device)
    stride = (L // synth.POOL + 3) // 4 * 4
    scores = torch.empty(B, stride, device=device)

    def ws_step(i):
        spx.spx_pool_append(st.d, B, st.raw_new, 1, st.pool_w, st.tail, st.pooled, st.cap_blk,
                            st.len_dev, L)
        spx.spx_index_score(st.d, B, qs[i % 4], st.w_head, st.pooled, st.cap_blk, n_vis, L,
                            scores, stride)
        spx.spx_topk_blocks(st.d, B, scores, stride, n_vis, L, st.idx, st.count, ws_t)
        spx.spx_sparse_mla_attn_ws(st.d, B, st.q, host_lat.data_ptr(), L * synth.LATENT, L, st.idx,
                                   st.count, n_vis, L, pool, nslots, slot_blk, blk_slot, stamp,
                                   hand, i, stats, st.out, st.lse, ws)

    ms_ws = timed(ws_step)
    hits, fetched = (int(x) for x in stats.sum(dim=0).tolist())
    if rank != 0:
        return None
    rows_bytes = st.B * (synth.TOPK_BLOCKS * synth.POOL) * synth.LATENT * 2
    return {"metric": "decode queries/s with the latent cache in pinned host memory",
            "value": st.B * world * K / (ms_ws * 1e-3), "unit": "queries/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_ws / K, "higher_is_better": True,
            "scaling": "weak", "dtype": "bf16", "data": "synthetic (indexer query cycling over 4)",
            "working_set": {"slots_per_sequence": nslots, "tokens_per_sequence": nslots * 4,
                            "hit_rate": hits / max(1, hits + fetched),
                            "fetched_blocks_per_step": fetched / max(1, args.warmup + K) / st.B},
            "zero_copy": {"ms_per_step": ms_zc / K, "queries_per_s": st.B * world * K / (ms_zc * 1e-3),
                          "host_rows_gbs": rows_bytes / (ms_zc / K * 1e-3) / 1e9},
            "config": {"workload": w.name, "latent": "pinned host memory",
                       "batch_per_gpu": st.B, "context": st.L}}


def measure_prefill(device, steps: int, warmup: int, world: int = 1, keys: str = "bf16"):
    """Times the chunked-prefill workload (4096 new tokens on a 131,072-token
    cache, one fused call per step) and its scoring kernel; returns the
    per-rank numbers and the state (for the oracle sample)."""
    spx = spx_module()
    w = synth.workload("prefill")
    st = PrefillState(w, device, keys=keys)
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        st.step()
    torch.cuda.synchronize(device)
    if spx.spx_device_error() != 0:
        raise RuntimeError("device error during the prefill warm-up")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device.index)
    clocks.start()
    n0 = spx.spx_launch_count()
    ev0.record(stream)
    for _ in range(steps):
        st.step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    launches = spx.spx_launch_count() - n0
    clocks.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    # the scoring kernel, in a separate pass (events around its launch)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(max(3, min(steps, 10)))]
    for a, b in evs:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize(device)
    for ev in evs:
        st.step(timing=ev)
    torch.cuda.synchronize(device)
    if spx.spx_device_error() != 0:
        raise RuntimeError("device error during the prefill timing")
    score_ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    return st, dict(ms=ms, steps=steps, score_ms=score_ms, launches=int(launches),
                    clocks=clocks.summary())


def prefill_summary(st, m, world: int = 1):
    """The prefill numbers against the tensor roofline (measured bf16 peaks)."""
    hbm, bf16, bf16s, src = measured_peaks()
    # the INT8 cache scores on kind::i8 (twice the bf16 rate, nominally)
    sc_peak, sc_peak_s = (2 * bf16, 2 * bf16s) if st.i8 else (bf16, bf16s)
    ms_step = m["ms"] / m["steps"]
    f_idx = score_algorithmic_flops_prefill(st.pos0, st.T)
    f_att = attention_flops_prefill(st.pos0, st.T, st.H)
    step_tf = (f_idx + f_att) / (ms_step * 1e-3) / 1e12
    score_tf = f_idx / (m["score_ms"] * 1e-3) / 1e12
    return {
        "workload": st.w.name, "ms_per_step": ms_step,
        "queries_per_s": st.T * world / (ms_step * 1e-3),
        "flops_per_step": {"indexer": f_idx, "attention": f_att},
        "step_tflops": step_tf, "step_frac_of_burst": step_tf / bf16,
        "step_frac_of_sustained": step_tf / bf16s,
        "scoring_kernel": {"avg_launch_us": m["score_ms"] * 1e3, "tflops": score_tf,
                           "frac_of_burst": score_tf / sc_peak,
                           "frac_of_sustained": score_tf / sc_peak_s,
                           "peak_dtype": "int8 (2 x bf16)" if st.i8 else "bf16"},
        "peak": {"bf16_burst_tflops": bf16, "bf16_sustained_tflops": bf16s, "source": src},
        "gpu_launches_per_step": m["launches"] / m["steps"],
        "clocks": m["clocks"],
    }


def prefill_cpu_baseline(st, nq: int = 256):
    """The oracle (as it stands) on a stratified sample of the prefill
    chunk's queries: each query scores every visible pooled block, keeps
    the top 512 and attends over the gathered rows.  Queries run in
    parallel, one host thread each; inputs are prepared untimed."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    pw = st.w.pool_weights()
    pooled = oracle.pool(st.raw_keys_host(), pw)
    sub = stratified_prefill_queries(st.T, nq)
    rows = st.pos0 + np.asarray(sub)
    q_idx, w_head, q = st.w.q_idx_np(rows), st.w.w_head_np(rows).astype(np.float64), st.w.q_np(rows)
    sels = [None] * len(sub)
    nthreads = oracle.threads(0)

    def select(i):
        sels[i] = oracle.select_query(q_idx[i], w_head[i], pooled, st.pos0 + sub[i] + 1, nthreads=1)[1]

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        list(ex.map(select, range(len(sub))))
    t_sel = time.perf_counter() - t0
    lat = [st.w.latent_np(0, oracle.token_set(sels[i], st.pos0 + sub[i] + 1)) for i in range(len(sub))]

    def attend(i):
        oracle.attention(q[i], lat[i], st.w.sm_scale)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        list(ex.map(attend, range(len(sub))))
    t_att = time.perf_counter() - t0
    tot = t_sel + t_att
    return {"value": len(sub) / tot, "unit": "queries/s", "cores": nthreads, "kind": "oracle",
            "sample": f"{len(sub)} stratified queries of the {st.T}-token prefill chunk on a "
                      f"{st.pos0}-token cache (scoring, top-512, attention), fp64, {tot:.2f} s"}


def stratified_prefill_queries(T: int, n: int = 256, seed: int = 5) -> list:
    """A stratified subset of a prefill chunk's queries: the first and last
    ones, every phase of the partial tail block (t % 4), both sides of the
    edges of the scoring kernel's 8-query groups and of 128-block key tiles,
    then seeded random queries up to n."""
    qs = set(range(min(12, T))) | set(range(max(0, T - 8), T))
    for g in (1, 2, 3, 64, 127, 128, 255, 256, 383, 511):
        for t in (8 * g - 1, 8 * g):
            if 0 <= t < T:
                qs.add(t)
    for k in range(1, 9):
        for t in (512 * k - 4, 512 * k - 1, 512 * k):
            if 0 <= t < T:
                qs.add(t)
    rng = np.random.default_rng(seed)
    while len(qs) < min(n, T):
        qs.add(int(rng.integers(0, T)))
    return sorted(qs)[:n]


def run_prefill(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    st, m = measure_prefill(device, args.steps, args.warmup, world, keys=args.keys)
    if rank != 0:
        return None
    summ = prefill_summary(st, m, world)
    line = {
        "metric": "sparse-attn chunked prefill queries/s; % of bf16 tensor peak",
        "value": summ["queries_per_s"], "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": summ["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": st.w.name, "pos0": st.pos0, "T": st.T,
                                        "heads": st.H, "pooled_keys": args.keys},
        "roofline": {"bound": "tensor", "kernel": "k_index_score<8> (prefill scoring)",
                     "achieved": summ["scoring_kernel"]["tflops"],
                     "peak": summ["scoring_kernel"]["tflops"] / summ["scoring_kernel"]["frac_of_burst"],
                     "unit": "TFLOP/s",
                     "frac": summ["scoring_kernel"]["frac_of_burst"],
                     "peak_source": f"{summ['peak']['source']} bf16_tflops (burst)"
                                    + (" x 2 for int8" if st.i8 else ""),
                     "traffic": None, "avg_launch_us": summ["scoring_kernel"]["avg_launch_us"]},
        "roofline_step": {"bound": "tensor", "achieved": summ["step_tflops"], "unit": "TFLOP/s",
                          "frac_of_burst": summ["step_frac_of_burst"],
                          "frac_of_sustained": summ["step_frac_of_sustained"]},
        "gpu_launches": m["launches"], "clocks": m["clocks"],
    }
    if world == 1 and not args.no_cpu_baseline and not st.i8:
        line["cpu_baseline"] = prefill_cpu_baseline(st)
    return line


def run_score_only(args, world, rank, local):
    """The decode scoring kernel alone on the 1M workload's pooled cache
    (no latent cache is built): for kernel profiling."""
    spx = spx_module()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.workload(args.workload)
    st = DecodeState(w, device, b_offset=shard_offset(rank, w.B), build_latent=False)
    B, L = st.B, st.L
    stride = L // synth.POOL
    n_vis = torch.full((B,), L, dtype=torch.int64, device=device)
    spx.spx_pool_append(st.d, B, st.raw_new, 1, st.pool_w, st.tail, st.pooled, st.cap_blk,
                        st.len_dev, L)
    scores = torch.empty(B, stride, device=device)

    def launch():
        spx.spx_index_score(st.d, B, st.q_idx, st.w_head, st.pooled, st.cap_blk, n_vis, L, scores,
                            stride)

    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    stream = torch.cuda.current_stream(device)
    for a, b in evs:
        a.record(stream)
        launch()
        b.record(stream)
    torch.cuda.synchronize(device)
    us = [a.elapsed_time(b) * 1e3 for a, b in evs]
    hbm = measured_peaks()[0]
    alg = score_algorithmic_bytes([L // synth.POOL] * B, B)
    avg = sum(us) / len(us)
    return {"mode": "score-only", "workload": w.name, "avg_us": avg, "min_us": min(us),
            "achieved_gbs": alg / (avg * 1e-6) / 1e9, "frac_of_measured_hbm": alg / (avg * 1e-6) / 1e9 / hbm,
            "algorithmic_bytes": alg}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("spx", "reference"), default="spx")
    ap.add_argument("--workload", default="1m", choices=synth.WORKLOADS)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="leave the nested prefill measurement out of the decode line")
    ap.add_argument("--host-latent", action="store_true",
                    help="decode with the latent cache in pinned host memory")
    ap.add_argument("--ws-slots", type=int, default=8192,
                    help="device working-set slots (4-token blocks) per sequence, --host-latent")
    ap.add_argument("--indexshare", type=int, default=0, metavar="N",
                    help="IndexShare decode: one indexer per N layers (reports per-layer rate)")
    ap.add_argument("--keys", choices=("bf16", "int8"), default="bf16",
                    help="pooled-key cache format (decode and prefill workloads)")
    ap.add_argument("--score-only", action="store_true",
                    help="time the decode scoring kernel alone (profiling aid)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    world, rank, local = dist_setup()
    try:
        if args.score_only:
            line = run_score_only(args, world, rank, local)
        elif args.indexshare > 1:
            line = run_indexshare(args, world, rank, local)
        elif args.host_latent:
            line = run_host_latent(args, world, rank, local)
        elif args.workload == "prefill":
            line = run_prefill(args, world, rank, local)
        else:
            line = run_decode(args, world, rank, local)
        if rank == 0 and line is not None:
            plain_decode = (args.workload != "prefill" and not args.score_only
                            and args.indexshare <= 1 and not args.host_latent)
            if (world == 1 and not args.no_cpu_baseline and plain_decode
                    and args.keys == "bf16"):
                line["cpu_baseline"] = cpu_baseline(synth.workload(args.workload),
                                                    torch.device("cuda", local))
            if plain_decode and args.workload == "1m" and not args.no_prefill:
                # the second target of the layer: chunked prefill on the tensor cores
                dev = torch.device("cuda", local)
                torch.cuda.empty_cache()
                st, m = measure_prefill(dev, 10, 3)
                pre = prefill_summary(st, m)
                if world == 1 and not args.no_cpu_baseline:
                    pre["cpu_baseline"] = prefill_cpu_baseline(st)
                line["prefill"] = pre
                del st
            print(json.dumps(line))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
