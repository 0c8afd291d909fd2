"""Benchmark: hybrid sparse attention prefill, one HCA layer + one MLA-DSA layer per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-decode]

Step = the whole hot path over one batch of synthetic input (L = 32768 tokens):
  HCA layer : hca_compress_kv (K, V -> 128:1 entries) + hca_attn_fwd (16 query heads, 1 K/V
              head, d = 512, window 128)
  DSA layer : dsa_index_topk (int8 indexer, 4 heads x 64, top-2048) + dsa_sparse_attn_fwd
              (64 heads, shared K/V head, d = 256)
value = tokens per second through both layers, summed over ranks (each rank runs its own
sequence: weak scaling, no data-path collective).  Inputs (Q alone is 1.5 GiB) are larger
than the 126 MB L2, so no flush is needed between steps.  A decode block (batch 32 at
position 1,048,575) is measured after the timed loop and reported beside the headline.

--impl reference times the CPU oracle (the only reference this method has) on a bounded
row sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L = 32768
HCA = synth.HCA_32K
DSA = synth.DSA_32K
DEC = synth.DECODE_1M
METRIC = "prefill attention tokens/s and TFLOP/s (% of B200 BF16 peak) per HCA / DSA layer"
WORKLOAD = "hca_prefill_L32768_hq16_hkv1_d512 + dsa_prefill_L32768_h64_d256_k2048 (B=1 per rank)"


# ----------------------------------------------------------------------------- work accounting

def hca_visible_keys_per_head(L, W=128, blk=128):
    tot = 0
    for t in range(L):
        s = t - W + 1
        tot += (s // blk if s > 0 else 0) + (t - max(0, s) + 1)
    return tot


def dsa_keys_per_head(L, k=2048):
    return sum(min(t + 1, k) for t in range(L))


HCA_KEYS = hca_visible_keys_per_head(L)                   # 8,331,711
DSA_KEYS = dsa_keys_per_head(L)                           # 65,012,736
HCA_FLOP = 4.0 * HCA.d * HCA.Hq * HCA_KEYS                # algorithmic: QK^T + PV
DSA_FLOP = 4.0 * DSA.d * DSA.Hq * DSA_KEYS
COMPRESS_BYTES = 2 * (L * HCA.Hkv * HCA.d * 2) + 2 * ((L // 128) * HCA.Hkv * HCA.d * 2) + 128 * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def kernel_source_hash(name):
    p = os.path.join(ROOT, "sparse_attention_hca_b200", "csrc", name)
    h = hashlib.sha256()
    for f in (p, os.path.join(ROOT, "sparse_attention_hca_b200", "csrc", "ptx.cuh")):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(summary_file, source_file):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel is unchanged since."""
    p = os.path.join(ROOT, "profiles", summary_file)
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != kernel_source_hash(source_file):
        return None
    return float(m.group(1))


# ----------------------------------------------------------------------------- multi-rank plumbing

def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """Max of a per-rank scalar (device time in ms) over all ranks; identity on one rank."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ms_per_step_max: float, world: int, tokens_per_rank: int = None) -> float:
    """Whole-job tokens/s: every rank runs its own sequence (weak scaling), so the job moves
    world * tokens_per_rank tokens per step, paced by the slowest rank."""
    tokens = L if tokens_per_rank is None else tokens_per_rank
    return world * tokens / (ms_per_step_max * 1e-3)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi every 20 ms with host timestamps; stop() keeps the samples taken inside the
    window marked by begin()/end() (the timed region)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.t0 = self.t1 = None
        import tempfile

        fd, self.path = tempfile.mkstemp(prefix=f"hcadsa_clocks_gpu{device_index}_", suffix=".csv")
        os.close(fd)

    def start(self, ready_timeout_s=5.0):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t_end = time.time() + ready_timeout_s  # the first sample is there before timing starts
        while time.time() < t_end and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    @staticmethod
    def _stamp(text):
        import datetime

        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(text, fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                rows.append((self._stamp(f[0]), float(f[2]), float(f[3]), f[6:10]))
            except ValueError:
                continue
        if not rows:
            return None
        window = "timed region"
        inside = [r for r in rows if r[0] is not None and self.t0 is not None and self.t1 is not None
                  and self.t0 - 0.02 <= r[0] <= self.t1 + 0.02]
        if not inside and self.t0 is not None and self.t1 is not None:
            # no sample fell inside (a very short region): the two samples nearest to it in time
            window = "nearest samples to the timed region"
            stamped = [r for r in rows if r[0] is not None]
            dist = lambda r: max(self.t0 - r[0], r[0] - self.t1, 0.0)  # noqa: E731
            inside = sorted(stamped, key=dist)[:2]
        if not inside:
            return None
        reasons = set()
        for r in inside:
            for n, v in zip(names, r[3]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "samples": len(inside), "window": window, "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- our arm

class _Draw:
    """Seeded draws on the device with torch's generator (same laws as synth, other values);
    each tensor has its own id, so a layer's inputs do not depend on which others are drawn."""

    def __init__(self, device, seed):
        self.device, self.seed = device, seed
        self.g = torch.Generator(device=device)

    def normal(self, shape, sigma, tid):
        self.g.manual_seed(self.seed * 1000 + tid)
        return (torch.randn(*shape, generator=self.g, device=self.device) * sigma).to(torch.bfloat16)

    def ints(self, shape, lo, hi, tid, dtype):
        self.g.manual_seed(self.seed * 1000 + tid)
        return torch.randint(lo, hi + 1, shape, generator=self.g, device=self.device, dtype=torch.int64).to(dtype)

    def uniform(self, n, hi, tid):
        self.g.manual_seed(self.seed * 1000 + tid)
        return torch.rand(n, generator=self.g, device=self.device) * hi


def make_hca_inputs(device, seed):
    d, sh = _Draw(device, seed), 1 / math.sqrt(HCA.d)
    return {"hQ": d.normal((1, L, HCA.Hq, HCA.d), sh, 1), "hK": d.normal((1, L, HCA.Hkv, HCA.d), sh, 2),
            "hV": d.normal((1, L, HCA.Hkv, HCA.d), sh, 3), "w": d.uniform(HCA.blk, 2.0 / HCA.blk, 4)}


def make_dsa_inputs(device, seed):
    d, sd = _Draw(device, seed), 1 / math.sqrt(DSA.d)
    return {"dQ": d.normal((1, L, DSA.Hq, DSA.d), sd, 11), "dK": d.normal((1, L, DSA.d), sd, 12),
            "dV": d.normal((1, L, DSA.d), sd, 13),
            "q_idx": d.ints((1, L, 4, 64), -8, 8, 15, torch.int8), "k_idx": d.ints((1, L, 64), -8, 8, 16, torch.int8),
            "w_idx": d.ints((4,), 1, 4, 17, torch.int32)}


def make_inputs(device, seed):
    """Bench inputs of both layers (see _Draw)."""
    return {**make_hca_inputs(device, seed), **make_dsa_inputs(device, seed)}


class Step:
    """Pre-allocated outputs/workspace; run() enqueues the 5 kernels of one step."""

    N_KERNELS = 5

    def __init__(self, hd, x, device):
        self.hd, self.x = hd, x
        self.Kc = torch.empty((1, L // 128, 1, HCA.d), dtype=torch.bfloat16, device=device)
        self.Vc = torch.empty_like(self.Kc)
        self.hO = torch.empty_like(x["hQ"])
        self.dO = torch.empty_like(x["dQ"])
        self.idx = torch.empty((1, L, DSA.k), dtype=torch.int32, device=device)
        ws = hd.dsa_index_topk_workspace_size(1, L, 0, L, DSA.k)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        hws = hd.lib().hca_attn_fwd_workspace_size(1, L, 0, HCA.Hq, HCA.Hkv, HCA.d, L // 128, 128, 128)
        self.hws = torch.empty(max(hws, 16), dtype=torch.uint8, device=device)

    def run(self, ev=None):
        hd, x = self.hd, self.x
        if ev: ev[0].record()
        hd.hca_compress_kv(x["hK"], x["hV"], x["w"], 128, Kc=self.Kc, Vc=self.Vc)
        if ev: ev[1].record()
        hd.hca_attn_fwd(x["hQ"], self.Kc, self.Vc, x["hK"], x["hV"], O=self.hO, workspace=self.hws)
        if ev: ev[2].record()
        hd.dsa_index_topk(x["q_idx"], x["k_idx"], x["w_idx"], DSA.k, idx=self.idx, workspace=self.ws)
        if ev: ev[3].record()
        hd.dsa_sparse_attn_fwd(x["dQ"], x["dK"], x["dV"], self.idx, O=self.dO)
        if ev: ev[4].record()


def run_decode(hd, device, iters=20):
    """Batch 32 single-token queries at t = 1,048,575: HCA layer and DSA layer, HBM-bound."""
    B, t = DEC.B, DEC.t
    g = torch.Generator(device=device)
    g.manual_seed(777)
    n_c = DEC.n_c
    Kc = torch.randn(B, n_c, 1, 512, generator=g, device=device).to(torch.bfloat16)
    Vc = torch.randn(B, n_c, 1, 512, generator=g, device=device).to(torch.bfloat16)
    Kw = torch.randn(B, DEC.W, 1, 512, generator=g, device=device).to(torch.bfloat16)
    Vw = torch.randn(B, DEC.W, 1, 512, generator=g, device=device).to(torch.bfloat16)
    hQ = torch.randn(B, 1, 16, 512, generator=g, device=device).to(torch.bfloat16)
    Lk = t + 1
    k_idx = torch.randint(-8, 9, (B, Lk, 64), generator=g, device=device, dtype=torch.int8)
    q_idx = torch.randint(-8, 9, (B, 1, 4, 64), generator=g, device=device, dtype=torch.int8)
    w_idx = torch.randint(1, 5, (4,), generator=g, device=device, dtype=torch.int32)
    K = torch.empty(B, Lk, 256, dtype=torch.bfloat16, device=device)
    V = torch.empty(B, Lk, 256, dtype=torch.bfloat16, device=device)
    for b in range(B):
        K[b].normal_(generator=g)
        V[b].normal_(generator=g)
    dQ = torch.randn(B, 1, 64, 256, generator=g, device=device).to(torch.bfloat16)
    hO = torch.empty_like(hQ)
    dO = torch.empty_like(dQ)
    idx = torch.empty(B, 1, DEC.k, dtype=torch.int32, device=device)
    ws = torch.empty(hd.dsa_index_topk_workspace_size(B, 1, t, Lk, DEC.k), dtype=torch.uint8, device=device)
    ws_start = t - DEC.W + 1
    hws = hd.lib().hca_attn_fwd_workspace_size(B, 1, t, 16, 1, 512, n_c, 128, DEC.W)
    hws = torch.empty(max(hws, 16), dtype=torch.uint8, device=device)
    # the DSA attention of 32 tokens splits each token's key tiles over several CTAs
    dws = torch.empty(max(hd.lib().dsa_sparse_attn_fwd_workspace_size(B, 1, DEC.k), 16), dtype=torch.uint8,
                      device=device)

    def step(ev=None):
        if ev: ev[0].record()
        hd.hca_attn_fwd(hQ, Kc, Vc, Kw, Vw, win_start=ws_start, q_offset=t, O=hO, workspace=hws)
        if ev: ev[1].record()
        hd.dsa_index_topk(q_idx, k_idx, w_idx, DEC.k, q_offset=t, idx=idx, workspace=ws)
        if ev: ev[2].record()
        hd.dsa_sparse_attn_fwd(dQ, K, V, idx, O=dO, workspace=dws)
        if ev: ev[3].record()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(iters)]
    for i in range(iters):
        step(evs[i])
    torch.cuda.synchronize()
    hca_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    idx_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    att_ms = statistics.median(e[2].elapsed_time(e[3]) for e in evs)
    hca_bytes = B * ((n_c + DEC.W) * 512 * 2 * 2 + 16 * 512 * 2 * 2)
    dsa_idx_bytes = B * Lk * 64
    dsa_att_bytes = B * (DEC.k * 256 * 2 * 2 + 64 * 256 * 2 * 2)
    out = {
        "workload": "decode_B32_t1048575 (HCA 16h d512 over 8191 entries + 128 window; DSA 64h d256 top-2048 of 1M)",
        "hca_us": hca_ms * 1e3, "hca_gbs": hca_bytes / hca_ms / 1e6,
        "dsa_index_topk_us": idx_ms * 1e3, "dsa_index_gbs": dsa_idx_bytes / idx_ms / 1e6,
        "dsa_attn_us": att_ms * 1e3, "dsa_attn_gbs": dsa_att_bytes / att_ms / 1e6,
        "step_us": (hca_ms + idx_ms + att_ms) * 1e3,
    }
    del Kc, Vc, K, V, k_idx, ws
    torch.cuda.empty_cache()
    return out


def csa_keys_per_head(L, k=2048, blk=4):
    return sum(min(k, (t + 1) // blk) for t in range(L))


def run_csa(hd, device, peaks, iters=10):
    """The CSA layer (compressed sparse attention, the pages' comparison point) at the MLA-DSA
    layer's size: B = 1, L = 32768, K/V compressed 4:1 (8192 entries, d = 256), indexer + top-2048
    over the complete blocks, sparse attention of 64 heads over the selected entries.  CUDA events
    per kernel, median of `iters` after 3 warm-up runs."""
    Lc, blk, k = L, 4, DSA.k
    n_c = Lc // blk
    d = _Draw(device, synth.SEED)
    sd = 1 / math.sqrt(DSA.d)
    Q = d.normal((1, Lc, DSA.Hq, DSA.d), sd, 31)
    K = d.normal((1, Lc, 1, DSA.d), sd, 32)
    V = d.normal((1, Lc, 1, DSA.d), sd, 33)
    w4 = d.uniform(blk, 2.0 / blk, 34)
    q_idx = d.ints((1, Lc, 4, 64), -8, 8, 35, torch.int8)
    kc_idx = d.ints((1, n_c, 64), -8, 8, 36, torch.int8)
    w_idx = d.ints((4,), 1, 4, 37, torch.int32)
    Kc = torch.empty((1, n_c, 1, DSA.d), dtype=torch.bfloat16, device=device)
    Vc = torch.empty_like(Kc)
    idx = torch.empty((1, Lc, k), dtype=torch.int32, device=device)
    ws = torch.empty(max(hd.lib().csa_index_topk_workspace_size(1, Lc, 0, n_c, k, blk), 16), dtype=torch.uint8,
                     device=device)
    O = torch.empty_like(Q)

    def step(ev=None):
        if ev: ev[0].record()
        hd.hca_compress_kv(K, V, w4, blk, Kc=Kc, Vc=Vc)
        if ev: ev[1].record()
        hd.csa_index_topk(q_idx, kc_idx, w_idx, k, blk, idx=idx, workspace=ws)
        if ev: ev[2].record()
        hd.dsa_sparse_attn_fwd(Q, Kc.view(1, n_c, DSA.d), Vc.view(1, n_c, DSA.d), idx, O=O)
        if ev: ev[3].record()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(iters)]
    for i in range(iters):
        step(evs[i])
    torch.cuda.synchronize()
    ms = [statistics.median(e[i].elapsed_time(e[i + 1]) for e in evs) for i in range(3)]
    flop = 4.0 * DSA.d * DSA.Hq * csa_keys_per_head(Lc, k, blk)
    comp_bytes = 2 * (Lc * DSA.d * 2) + 2 * (n_c * DSA.d * 2) + blk * 4
    tf = flop / (ms[2] * 1e-3) / 1e12
    del Q, K, V, O, idx, Kc, Vc
    torch.cuda.empty_cache()
    return {"workload": "csa_prefill_L32768_h64_d256_blk4_k2048 (B=1; 8192 entries)", "iters": iters,
            "compress_us": ms[0] * 1e3, "compress_gbs": comp_bytes / (ms[0] * 1e-3) / 1e9,
            "index_topk_ms": ms[1], "attn_ms": ms[2], "attn_tflops": tf, "attn_pct_bf16": 100 * tf / peaks["bf16_tflops"],
            "algorithmic_flop": flop, "layer_tokens_per_s": Lc / (sum(ms) * 1e-3)}


def run_gate_vha(hd, device, peaks, iters=10, H=16, dv=512, rq=1024, r=4):
    """The fused output gate + virtual-head mix on the HCA layer's output (L = 32768, 16 heads of
    512, query latent 1024, mix rank 4): a tensor-core GEMM (M = tokens, N = H * dv, K = rq) with
    the epilogue reading O and writing Y.  CUDA events, median of `iters` after 3 warm-up runs."""
    d = _Draw(device, synth.SEED)
    O = d.normal((1, L, H, dv), 0.05, 41)
    cq = d.normal((1, L, rq), 1.0, 42)
    Wg = d.normal((H * dv, rq), 1 / math.sqrt(rq), 43)
    U = d.uniform(H * r, 0.5, 44).view(H, r) - 0.25
    V = d.uniform(H * r, 0.5, 45).view(H, r) - 0.25
    Y = torch.empty_like(O)
    for _ in range(3):
        hd.attn_gate_vha_fwd(O, cq, Wg, U, V, Y=Y)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
    for i in range(iters):
        evs[i][0].record()
        hd.attn_gate_vha_fwd(O, cq, Wg, U, V, Y=Y)
        evs[i][1].record()
    torch.cuda.synchronize()
    ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    flop = 2.0 * L * H * dv * rq
    hbm = 2 * (2 * L * H * dv) + 2 * L * rq + 2 * H * dv * rq
    tf = flop / (ms * 1e-3) / 1e12
    del O, cq, Wg, Y
    torch.cuda.empty_cache()
    return {"workload": f"gate_vha_L{L}_h{H}_dv{dv}_rq{rq}_r{r} (B=1)", "iters": iters, "ms": ms,
            "tflops": tf, "pct_bf16": 100 * tf / peaks["bf16_tflops"], "gbs": hbm / (ms * 1e-3) / 1e9,
            "pct_hbm": 100 * hbm / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "algorithmic_flop": flop,
            "algorithmic_bytes": hbm}


def run_hca_latent(hd, device, peaks, iters=10):
    """HCA layer prefill with FlashMask-4's head shape (qk 576 / v 512, values = the latent part of
    the keys) at L = 32768, 16 query heads on one K/V head: compression of the 576-wide keys and
    the attention, CUDA events, median of `iters` after 3 warm-up runs."""
    dqk, dv = 576, 512
    d = _Draw(device, synth.SEED)
    sh = 1 / math.sqrt(dqk)
    Q = d.normal((1, L, HCA.Hq, dqk), sh, 51)
    K = d.normal((1, L, HCA.Hkv, dqk), sh, 52)
    w = d.uniform(HCA.blk, 2.0 / HCA.blk, 54)
    Kc = torch.empty((1, L // 128, 1, dqk), dtype=torch.bfloat16, device=device)
    O = torch.empty((1, L, HCA.Hq, dv), dtype=torch.bfloat16, device=device)
    nb = hd.lib().hca_attn_fwd_latent_workspace_size(1, L, 0, HCA.Hq, HCA.Hkv, dqk, dv, L // 128, 128, 128)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)

    def step(ev=None):
        if ev: ev[0].record()
        hd.hca_compress_kv(K, K, w, 128, Kc=Kc, Vc=Kc)
        if ev: ev[1].record()
        hd.hca_attn_fwd_latent(Q, Kc, K, O=O, workspace=ws)
        if ev: ev[2].record()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(iters)]
    for i in range(iters):
        step(evs[i])
    torch.cuda.synchronize()
    comp_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    flop = 2.0 * (dqk + dv) * HCA.Hq * hca_visible_keys_per_head(L)
    tf = flop / (attn_ms * 1e-3) / 1e12
    del Q, K, O, ws
    torch.cuda.empty_cache()
    return {"workload": f"hca_prefill_L{L}_hq16_hkv1_dqk576_dv512 (B=1, values = latent part of the keys)",
            "iters": iters, "compress_us": comp_ms * 1e3, "attn_ms": attn_ms, "attn_tflops": tf,
            "attn_pct_bf16": 100 * tf / peaks["bf16_tflops"], "algorithmic_flop": flop}


def run_backward(hd, device, peaks, iters=5):
    """Backward kernels at the layer sizes of the step (L = 32768): the DSA sparse attention
    backward (dQ, dK, dV from the forward's O and lse over the top-2048 selection of the step's
    indexer), the HCA compressor's adjoint (dX, dw for 512-wide keys, blocks of 128) and the HCA
    attention backward (dQ, entry and window dK / dV; 5 * 2 * 512 flop per visible (row, key)).  CUDA
    events, median of `iters` after 3 warm-up runs.  Algorithmic units: 5 * 2 * 256 flop per
    (query, head, selected key) (S, dP, dV, dK, dQ) and 2 KB of fp32 reductions into dK / dV per
    (query, selected key)."""
    x = make_dsa_inputs(device, synth.SEED)
    idx = hd.dsa_index_topk(x["q_idx"], x["k_idx"], x["w_idx"], DSA.k)
    O, lse = hd.dsa_sparse_attn_fwd(x["dQ"], x["dK"], x["dV"], idx, return_lse=True)
    gO = _Draw(device, synth.SEED).normal(tuple(O.shape), 0.1, 61)
    dK = torch.zeros((1, L, DSA.d), dtype=torch.float32, device=device)
    dV = torch.zeros_like(dK)
    for _ in range(3):
        hd.dsa_sparse_attn_bwd(x["dQ"], x["dK"], x["dV"], idx, O, gO, lse, dK=dK, dV=dV)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
    for i in range(iters):
        evs[i][0].record()
        hd.dsa_sparse_attn_bwd(x["dQ"], x["dK"], x["dV"], idx, O, gO, lse, dK=dK, dV=dV)
        evs[i][1].record()
    torch.cuda.synchronize()
    ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    keys = int((idx >= 0).sum().item())  # selected (query, key) pairs
    del x, idx, O, lse, gO, dK, dV
    torch.cuda.empty_cache()
    flop = 10.0 * DSA.d * DSA.Hq * keys
    red_bytes = 2.0 * 4 * DSA.d * keys
    tf = flop / (ms * 1e-3) / 1e12
    # compressor adjoint: X (bf16) read, dX (fp32) read + written, dXc (fp32) read
    Xk = _Draw(device, synth.SEED).normal((1, L, HCA.Hkv, HCA.d), 1 / math.sqrt(HCA.d), 62)
    w = _Draw(device, synth.SEED).uniform(HCA.blk, 2.0 / HCA.blk, 63)
    dXc = _Draw(device, synth.SEED).normal((1, L // HCA.blk, HCA.Hkv, HCA.d), 1.0, 64).float()
    dX = torch.zeros((1, L, HCA.Hkv, HCA.d), dtype=torch.float32, device=device)
    dw = torch.zeros(HCA.blk, dtype=torch.float32, device=device)
    for _ in range(3):
        hd.hca_compress_bwd(Xk, w, dXc, HCA.blk, dX=dX, dw=dw)
    torch.cuda.synchronize()
    cevs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
    for i in range(iters):
        cevs[i][0].record()
        hd.hca_compress_bwd(Xk, w, dXc, HCA.blk, dX=dX, dw=dw)
        cevs[i][1].record()
    torch.cuda.synchronize()
    cms = statistics.median(e[0].elapsed_time(e[1]) for e in cevs)
    cbytes = L * HCA.Hkv * HCA.d * (2 + 4 + 4) + (L // HCA.blk) * HCA.Hkv * HCA.d * 4
    del Xk, dXc, dX, dw
    torch.cuda.empty_cache()
    # HCA attention backward (prep, score blocks, dQ, dK/dV: four launches)
    h = make_hca_inputs(device, synth.SEED)
    Kc = torch.empty((1, L // HCA.blk, HCA.Hkv, HCA.d), dtype=torch.bfloat16, device=device)
    Vc = torch.empty_like(Kc)
    hd.hca_compress_kv(h["hK"], h["hV"], h["w"], HCA.blk, Kc=Kc, Vc=Vc)
    hO, hlse = hd.hca_attn_fwd(h["hQ"], Kc, Vc, h["hK"], h["hV"], return_lse=True)
    hgO = _Draw(device, synth.SEED).normal(tuple(hO.shape), 0.1, 65)
    hws = torch.empty(hd.lib().hca_attn_bwd_workspace_size(1, L, 0, HCA.Hq, HCA.Hkv, HCA.d, L // HCA.blk, HCA.blk,
                                                           HCA.W), dtype=torch.uint8, device=device)
    grads = {}

    def hbwd():
        return hd.hca_attn_bwd(h["hQ"], Kc, Vc, h["hK"], h["hV"], hO, hgO, hlse, workspace=hws, **grads)

    out = hbwd()
    grads.update(dKc=out[1], dVc=out[2], dKw=out[3], dVw=out[4])
    for _ in range(2):
        hbwd()
    torch.cuda.synchronize()
    hevs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
    for i in range(iters):
        hevs[i][0].record()
        hbwd()
        hevs[i][1].record()
    torch.cuda.synchronize()
    hms = statistics.median(e[0].elapsed_time(e[1]) for e in hevs)
    hflop = 10.0 * HCA.d * HCA.Hq * hca_visible_keys_per_head(L)
    htf = hflop / (hms * 1e-3) / 1e12
    del h, Kc, Vc, hO, hlse, hgO, hws, grads, out
    torch.cuda.empty_cache()
    return {"workload": f"dsa_bwd_L{L}_h64_d256_k2048 + compress_bwd_L{L}_d512_blk128 + hca_bwd_L{L}_hq16_hkv1_d512 "
                        "(B=1)", "iters": iters,
            "dsa_bwd_ms": ms, "dsa_bwd_tflops": tf, "dsa_bwd_pct_bf16": 100 * tf / peaks["bf16_tflops"],
            "dsa_bwd_reduce_gbs": red_bytes / (ms * 1e-3) / 1e9, "dsa_bwd_algorithmic_flop": flop,
            "dsa_bwd_reduce_bytes": red_bytes,
            "compress_bwd_us": cms * 1e3, "compress_bwd_gbs": cbytes / (cms * 1e-3) / 1e9,
            "compress_bwd_pct_hbm": 100 * cbytes / (cms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "compress_bwd_bytes": cbytes,
            "hca_bwd_ms": hms, "hca_bwd_tflops": htf, "hca_bwd_pct_bf16": 100 * htf / peaks["bf16_tflops"],
            "hca_bwd_algorithmic_flop": hflop}


def run_hca_131k(hd, device, peaks, iters=10):
    """The HCA long-context prefill configuration (B = 1, L = 131072, 16 query heads on one K/V
    head, d = 512, 1024 compressed entries): compression and attention timed with CUDA events
    after 3 warm-up runs (median of `iters`), with its own clock record."""
    Lh = synth.HCA_131K.L
    d = _Draw(device, synth.SEED)
    sh = 1 / math.sqrt(HCA.d)
    Q = d.normal((1, Lh, HCA.Hq, HCA.d), sh, 21)
    K = d.normal((1, Lh, HCA.Hkv, HCA.d), sh, 22)
    V = d.normal((1, Lh, HCA.Hkv, HCA.d), sh, 23)
    w = d.uniform(HCA.blk, 2.0 / HCA.blk, 24)
    Kc = torch.empty((1, Lh // 128, 1, HCA.d), dtype=torch.bfloat16, device=device)
    Vc = torch.empty_like(Kc)
    O = torch.empty_like(Q)
    nb = hd.lib().hca_attn_fwd_workspace_size(1, Lh, 0, HCA.Hq, HCA.Hkv, HCA.d, Lh // 128, 128, 128)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)

    def step(ev=None):
        if ev: ev[0].record()
        hd.hca_compress_kv(K, V, w, 128, Kc=Kc, Vc=Vc)
        if ev: ev[1].record()
        hd.hca_attn_fwd(Q, Kc, Vc, K, V, O=O, workspace=ws)
        if ev: ev[2].record()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(device.index or 0)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(iters)]
    clocks.begin()
    for i in range(iters):
        step(evs[i])
    torch.cuda.synchronize()
    clocks.end()
    clk = clocks.stop()
    comp_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    flop = 4.0 * HCA.d * HCA.Hq * hca_visible_keys_per_head(Lh)
    comp_bytes = 2 * (Lh * HCA.Hkv * HCA.d * 2) + 2 * ((Lh // 128) * HCA.Hkv * HCA.d * 2) + 128 * 4
    tf = flop / (attn_ms * 1e-3) / 1e12
    gbs = comp_bytes / (comp_ms * 1e-3) / 1e9
    del Q, K, V, O, ws
    torch.cuda.empty_cache()
    return {"workload": "hca_prefill_L131072_hq16_hkv1_d512 (B=1)", "iters": iters,
            "compress_us": comp_ms * 1e3, "compress_gbs": gbs, "compress_pct_hbm": 100 * gbs / peaks["hbm_gbs"],
            "attn_ms": attn_ms, "attn_tflops": tf, "attn_pct_bf16": 100 * tf / peaks["bf16_tflops"],
            "algorithmic_flop": flop, "tokens_per_s": Lh / ((comp_ms + attn_ms) * 1e-3), "clocks": clk}


def e2e_measure(hd, x, device, steps):
    """Same step through the C ABI with host buffers: every step copies all of its inputs from
    pinned host memory to the device and both layer outputs back, inside the timed region.  The
    steps are pipelined on three streams (host-to-device copies, compute, device-to-host
    copies) over two sets of device buffers, so step i+1's inputs and step i-1's outputs cross
    PCIe while step i computes; the timed region runs from the first input copy to the last
    output copy."""
    host = {k: v.cpu().pin_memory() for k, v in x.items()}
    bufs = []
    for _ in range(2):
        dev = {k: torch.empty_like(v) for k, v in x.items()}
        bufs.append((dev, Step(hd, dev, device)))
    outs = [(torch.empty(x["hQ"].shape, dtype=torch.bfloat16).pin_memory(),
             torch.empty(x["dQ"].shape, dtype=torch.bfloat16).pin_memory()) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = outs[0][0].numel() * 2 + outs[0][1].numel() * 2
    s_in, s_cmp, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev(), ev()]    # inputs of buffer b landed
    cmp_done = [ev(), ev()]   # step on buffer b finished (inputs free, outputs ready)
    out_done = [ev(), ev()]   # outputs of buffer b copied to the host

    def run(n, e_start=None, e_end=None):
        for i in range(n):
            b = i & 1
            dev, stp = bufs[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(cmp_done[b])  # step i-2 no longer reads these inputs
                if i == 0 and e_start is not None:
                    e_start.record(s_in)
                for k in host:
                    dev[k].copy_(host[k], non_blocking=True)
                in_done[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_done[b])
                if i >= 2:
                    s_cmp.wait_event(out_done[b])  # step i-2's outputs are on the host
                stp.run()
                cmp_done[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[b])
                outs[b][0].copy_(stp.hO, non_blocking=True)
                outs[b][1].copy_(stp.dO, non_blocking=True)
                out_done[b].record(s_out)
        if e_end is not None:
            s_out.wait_stream(s_in)
            s_out.wait_stream(s_cmp)
            e_end.record(s_out)

    run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, e0, e1)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del bufs
    torch.cuda.empty_cache()
    return ms, h2d, d2h


def cpu_sample(n_hca=12288, n_dsa=3072):
    """Times the oracle (plain C, OpenMP over query rows) on a bounded sample of the workload:
    full compression, HCA attention for n_hca query tokens and DSA top-k + attention for
    n_dsa query tokens, positions spread evenly over [0, L).  Each function runs once over all
    its sampled rows, so OpenMP spreads them over the host cores.  Returns tokens/s through
    both layers (inverse of the mean per-token cost)."""
    import numpy as np

    import oracle

    oracle.build()
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    hx = synth.hca_inputs(HCA)                   # same shapes and laws as the GPU workload
    Kh, Vh, Qh = bits(hx["K"]), bits(hx["V"]), bits(hx["Q"])
    w = hx["w"].numpy()
    t0 = time.perf_counter()
    Kc, Vc = oracle.hca_compress(Kh, w, HCA.blk), oracle.hca_compress(Vh, w, HCA.blk)
    t_comp = time.perf_counter() - t0
    rows_h = np.linspace(0, L - 1, n_hca).astype(np.int64)
    t0 = time.perf_counter()
    oracle.hca_attn(Qh, Kc, Vc, Kh, Vh, blk=HCA.blk, W=HCA.W, rows=rows_h)
    t_hca = time.perf_counter() - t0
    dc = synth.DsaConfig("s", B=1, L=L, Hq=1)    # indexer inputs and K/V (Q drawn per sample)
    di = synth.dsa_inputs(dc)
    rows_d = np.linspace(0, L - 1, n_dsa).astype(np.int64)
    Qd = bits(synth.normal_bf16((1, n_dsa, DSA.Hq, DSA.d), 1 / math.sqrt(DSA.d), synth.SEED, "Q"))
    t0 = time.perf_counter()
    idx = oracle.dsa_topk(di["q_idx"].numpy(), di["k_idx"].numpy(), di["w_idx"].numpy(), DSA.k, rows=rows_d)
    oracle.dsa_attn(Qd, bits(di["K"]), bits(di["V"]), idx)
    t_dsa = time.perf_counter() - t0
    per_token = t_comp / L + t_hca / n_hca + t_dsa / n_dsa
    cores = int(os.environ.get("OMP_NUM_THREADS", "0")) or (
        len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())
    return {
        "value": 1.0 / per_token, "unit": "tokens/s", "cores": cores, "kind": "oracle",
        "sample": (f"full compression of the L={L} sequence; HCA attention (16 heads) for {n_hca} and DSA "
                   f"top-{DSA.k} + attention (64 heads) for {n_dsa} query tokens spread evenly over [0, {L}); "
                   f"tokens/s extrapolated from the sample's per-token cost = 1 / (compress/L + HCA per row "
                   f"+ DSA per row)"),
        "extrapolated": True,
        "sample_seconds": t_comp + t_hca + t_dsa,
    }


def ours(args):
    import sparse_attention_hca_b200 as hd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    hd.lib()
    x = make_inputs(device, seed=synth.SEED + rank)
    st = Step(hd, x, device)
    for _ in range(args.warmup):
        st.run()
    torch.cuda.synchronize()
    hd.hcadsa_check_device_error()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()  # waits for its first sample, so it runs before the barrier that opens timing
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.begin()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        st.run(evs[i])
    t_end.record()
    torch.cuda.synchronize()
    clocks.end()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    hd.hcadsa_check_device_error()
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dist, device)
    ms_step = ms_total / args.steps
    k_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i in range(4)]
    comp_ms, hca_ms, idx_ms, dsa_ms = k_ms
    peaks = load_peaks()
    hca_tf = HCA_FLOP / (hca_ms * 1e-3) / 1e12
    dsa_tf = DSA_FLOP / (dsa_ms * 1e-3) / 1e12
    # The timed region is well under a second at full clock, so the denominator is the burst
    # peak (a cuBLAS bf16 GEMM timed alone); the sustained figure was taken over seconds under
    # the power cap at ~1.34 GHz and is reported beside it for context only.
    peak_b = peaks["bf16_tflops"]
    peak_s = peaks["bf16_tflops_sustained"]

    decode = None
    e2e = None
    hca131 = None
    if rank == 0 and not args.no_decode:
        decode = run_decode(hd, device)
        hd.hcadsa_check_device_error()
    if rank == 0 and not args.no_131k:
        hca131 = run_hca_131k(hd, device, peaks)
        hd.hcadsa_check_device_error()
    csa = None
    if rank == 0 and not args.no_csa:
        csa = run_csa(hd, device, peaks)
        hd.hcadsa_check_device_error()
    gate = None
    if rank == 0 and not args.no_gate:
        gate = run_gate_vha(hd, device, peaks)
        hd.hcadsa_check_device_error()
    latent = None
    if rank == 0 and not args.no_latent:
        latent = run_hca_latent(hd, device, peaks)
        hd.hcadsa_check_device_error()
    bwd = None
    if rank == 0 and not args.no_bwd:
        bwd = run_backward(hd, device, peaks)
        hd.hcadsa_check_device_error()
    e2e_ms, h2d, d2h = e2e_measure(hd, x, device, steps=max(4, min(args.steps, 8)))
    e2e_ms = max_over_ranks(e2e_ms, dist, device)
    e2e = {"value": job_throughput(e2e_ms, world), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_sample()
    traffic = profiled_traffic("dsa_sparse_attn_fwd_L32768.md", "dsa_attn.cu")
    line = {
        "metric": METRIC,
        "value": job_throughput(ms_step, world),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; Q/K/V ~N(0,1)/sqrt(d) bf16, int8 indexer U[-8,8], weights U[1,4], w~U(0,2/128))",
        "config": bench_config(world),
        "layers": {
            "hca": {"compress_us": comp_ms * 1e3, "compress_gbs": COMPRESS_BYTES / (comp_ms * 1e-3) / 1e9,
                    "compress_pct_hbm": 100 * COMPRESS_BYTES / (comp_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "attn_ms": hca_ms, "attn_tflops": hca_tf, "attn_pct_bf16": 100 * hca_tf / peak_b,
                    "layer_tokens_per_s": L / ((comp_ms + hca_ms) * 1e-3)},
            "dsa": {"index_topk_ms": idx_ms, "attn_ms": dsa_ms, "attn_tflops": dsa_tf,
                    "attn_pct_bf16": 100 * dsa_tf / peak_b,
                    "layer_tokens_per_s": L / ((idx_ms + dsa_ms) * 1e-3)},
            "algorithmic_flop": {"hca_attn": HCA_FLOP, "dsa_attn": DSA_FLOP},
            "peak_note": f"percentages of the burst bf16 peak {peak_b} TFLOP/s and of {peaks['hbm_gbs']} GB/s "
                         f"({peaks['src']})",
        },
        "roofline": {"kernel": "dsa_sparse_attn_fwd", "bound": "tensor", "achieved": dsa_tf,
                     "peak": peak_b, "unit": "TFLOP/s", "frac": dsa_tf / peak_b,
                     "peak_kind": f"bf16_tflops, burst ({peaks['src']}): the kernel runs for ~10 ms at a time "
                                  "inside a sub-second timed region at full clock",
                     "frac_of_sustained_peak": dsa_tf / peak_s, "traffic": traffic,
                     "units_per_launch": f"{DSA_KEYS} visible keys x 64 heads x 4*256 flop"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": Step.N_KERNELS * args.steps,
        "clocks": clk,
        "decode": decode,
        "hca_131k": hca131,
        "csa": csa,
        "gate_vha": gate,
        "hca_latent_576": latent,
        "backward": bwd,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def bench_config(world):
    """The workload description both arms print (the reference arm runs the same workload)."""
    return {"workload": WORKLOAD, "global_batch": world, "seq_len": L, "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2 (1.5 GiB of Q per step), no flush"}


def reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per, secs = [], []
    cpu = None
    for _ in range(args.warmup):
        cpu_sample(n_hca=256, n_dsa=32)
    for _ in range(args.steps):
        cpu = cpu_sample(n_hca=1024, n_dsa=128)
        per.append(cpu["value"])
        secs.append(cpu["sample_seconds"])
    v = statistics.median(per)
    cpu["value"] = v
    # Each timed step is the bounded row sample (what ms_per_step reports); value is the tokens/s
    # of the whole workload extrapolated from the sample's per-token cost.
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
        "ms_per_full_step_extrapolated": 1e3 * L / v, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same laws as the GPU arm); value extrapolated from a bounded row sample",
        "config": bench_config(world),
        "cpu_baseline": cpu,
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def only_kernel(args):
    """Runs one library kernel alone at sequence length --seq-len (profiling mode): W warm-up
    and K timed launches; prints a small JSON record (not the benchmark contract line).
    --only decode runs the decode step instead; --only csa / gate_vha the CSA layer / the output
    gate block at --seq-len."""
    global L
    import sparse_attention_hca_b200 as hd

    if args.only == "decode":
        out = run_decode(hd, torch.device("cuda", 0), iters=max(1, args.steps))
        hd.hcadsa_check_device_error()
        print(json.dumps(out))
        return
    if args.only in ("csa", "gate_vha", "hca_latent", "backward"):
        L = args.seq_len
        run = {"csa": run_csa, "gate_vha": run_gate_vha, "hca_latent": run_hca_latent,
               "backward": run_backward}[args.only]
        out = run(hd, torch.device("cuda", 0), load_peaks(), iters=max(1, args.steps))
        hd.hcadsa_check_device_error()
        print(json.dumps(out))
        return

    L = args.seq_len
    device = torch.device("cuda", 0)
    # only the selected kernel's layer is allocated (a profiled launch should hold a few GB at most)
    if args.only in ("compress", "hca_attn"):
        x = make_hca_inputs(device, seed=synth.SEED)
        Kc = torch.empty((1, L // 128, 1, HCA.d), dtype=torch.bfloat16, device=device)
        Vc = torch.empty_like(Kc)
        hd.hca_compress_kv(x["hK"], x["hV"], x["w"], 128, Kc=Kc, Vc=Vc)
        if args.only == "compress":
            fn = lambda: hd.hca_compress_kv(x["hK"], x["hV"], x["w"], 128, Kc=Kc, Vc=Vc)  # noqa: E731
        else:
            hO = torch.empty_like(x["hQ"])
            nb = hd.lib().hca_attn_fwd_workspace_size(1, L, 0, HCA.Hq, HCA.Hkv, HCA.d, L // 128, 128, 128)
            hws = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)
            fn = lambda: hd.hca_attn_fwd(x["hQ"], Kc, Vc, x["hK"], x["hV"], O=hO, workspace=hws)  # noqa: E731
    else:
        x = make_dsa_inputs(device, seed=synth.SEED)
        idx = torch.empty((1, L, DSA.k), dtype=torch.int32, device=device)
        ws = torch.empty(hd.dsa_index_topk_workspace_size(1, L, 0, L, DSA.k), dtype=torch.uint8, device=device)
        hd.dsa_index_topk(x["q_idx"], x["k_idx"], x["w_idx"], DSA.k, idx=idx, workspace=ws)
        if args.only == "index_topk":
            fn = lambda: hd.dsa_index_topk(x["q_idx"], x["k_idx"], x["w_idx"], DSA.k, idx=idx,  # noqa: E731
                                           workspace=ws)
        else:
            torch.cuda.synchronize()
            del ws  # the attention needs only the index rows
            torch.cuda.empty_cache()
            dO = torch.empty_like(x["dQ"])
            fn = lambda: hd.dsa_sparse_attn_fwd(x["dQ"], x["dK"], x["dV"], idx, O=dO)  # noqa: E731
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    hd.hcadsa_check_device_error()
    print(json.dumps({"kernel": args.only, "seq_len": L, "ms_per_launch": e0.elapsed_time(e1) / max(1, args.steps)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-131k", action="store_true", help="skip the L = 131072 HCA block")
    ap.add_argument("--no-csa", action="store_true", help="skip the CSA layer block")
    ap.add_argument("--no-gate", action="store_true", help="skip the output gate + head mix block")
    ap.add_argument("--no-latent", action="store_true", help="skip the qk 576 / v 512 HCA block")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward block")
    ap.add_argument("--only", choices=["compress", "hca_attn", "index_topk", "dsa_attn", "decode", "csa", "gate_vha",
                                       "hca_latent", "backward"],
                    help="profiling mode: run one kernel alone at --seq-len, or the decode step "
                         "(B = 32 at t = 1,048,575; --steps timed steps after 3 warm-up steps)")
    ap.add_argument("--seq-len", type=int, default=L)
    args = ap.parse_args()
    if args.only:
        return only_kernel(args)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
