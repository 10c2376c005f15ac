"""Benchmark of the MLA absorbed-decode step on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: query absorption + RoPE, the
split-KV decode attention over the latent cache (plan, split kernel, combine), and the W_UV
up-projection, through the C ABI. The K timed steps are replayed from a CUDA graph of the
same calls (`value`). `e2e` runs the step through the public API with the inputs copied
from pinned host memory and the output copied back every step: `value` as a serving loop
would (per-step CUDA graphs, copies on side branches), `eager_value` as plain calls (the
host path of every C-ABI call inside the timed region). Inputs are resident in HBM before
the timed region; every step reads a different one of several cache copies whose total
exceeds L2 four times, so no step finds its cache in L2.

The headline workload is the largest single-GPU configuration (64 ragged sequences, paged);
`workloads` reports the other four the same way. Multi-GPU (one process per GPU; started
under torchrun, or `--gpus N` relaunches itself under torchrun): every rank runs its own
replica of the workload (sequences are independent; no data-path collective), the timing is
the max over ranks, and `value` counts the tokens of all ranks (weak scaling).

--impl reference times the fp64 CPU oracle on the host cores (rank 0 only), each step one
sample unit of the same workload (8 heads of one sequence, the non-absorbed definition),
the same unit `cpu_baseline` repeats for about 15 s.
--profile runs W warm-up steps and then K eager steps of the hot path alone (no graphs, no
extra measurements, no JSON line): the command the committed ncu summaries were taken on.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_latent_kv_28_b200 import workloads as wl  # noqa: E402

METRIC = "MLA decode tokens/s & latent-KV GB/s on 1 B200; % of binding roofline"
DEFAULT_WORKLOAD = "ragged_paged_b64"
L2_BYTES = 126 * 2**20
ROW_BYTES = 576 * 2
KERNEL_SOURCES = ["decode_split.cu", "sm100.cuh"]


# --------------------------------------------------------------------------- ranks
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, local: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def max_over_ranks(x: float, world: int, device) -> float:
    """The max of x over all ranks (the timing rule for multi-GPU numbers)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, local: int, cuda: bool):
    if world > 1:
        import torch.distributed as dist
        if cuda:
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


def replica_seed(rank: int) -> int:
    """Each rank draws its own replica of the workload."""
    return rank


def job_tokens_per_s(world: int, batch: int, ms_max: float) -> float:
    """Whole-job throughput: every rank decodes one token for each of its `batch` sequences
    per step, and a step takes the slowest rank's time."""
    return world * batch / (ms_max * 1e-3)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML every few ms on a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.ok = False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.err = repr(e)
        self.period = period_s
        self.t = threading.Thread(target=self._run, daemon=True)

    def _handle(self, idx):
        nv = self.nv
        try:
            p = torch.cuda.get_device_properties(idx)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                idx = int(vis.split(",")[idx])
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = int(self._reasons(self.h))
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t.start()

    def stop(self):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        win = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-3:]
        reasons = set()
        for _, _, rs in win:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(win)}


# --------------------------------------------------------------------------- roofline
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def sustained_tensor_peak():
    """bf16 dense TFLOP/s for a kernel timed inside a long loop: the measured sustained figure,
    else the fallback (about 1.4 PFLOP/s under the power cap)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured bf16_tflops_sustained"
    return 1400.0, "fallback 1400 TFLOP/s"


def kernel_sources_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_latent_kv_28_b200", "csrc")
    for name in KERNEL_SOURCES:
        p = os.path.join(csrc, name)
        if os.path.exists(p):
            with open(p, "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"decode_attn_{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_sources_sha") != kernel_sources_sha():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------------- CPU oracle
def _np(t):
    """torch tensor -> numpy; bf16 as uint16 bit patterns (the oracle widens them)."""
    import numpy as np
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def workload_np(w):
    return dict(q_c=_np(w.q_c), q_r=_np(w.q_r), w_uk=_np(w.w_uk), w_uv=_np(w.w_uv),
                cache=_np(w.cache), kv_lens=_np(w.kv_lens),
                page_table=None if w.page_table is None else _np(w.page_table),
                page_size=w.page_size)


HEADS_PER_UNIT = 8


class OracleSample:
    """The fp64 oracle as it stands (the non-absorbed definition) on sample units of a
    workload. A unit is HEADS_PER_UNIT heads of one sequence; unit k is head group
    k // batch of sequence k % batch, so consecutive units spread over the sequences (and,
    in the ragged workload, over its length mix). The weights and queries are cut to each
    unit's heads before any timing, so a call widens only what it reads. The reference arm
    and `cpu_baseline` both time these units."""

    def __init__(self, w):
        import numpy as np
        import oracle
        self.oracle = oracle
        self.w = w
        self.a = workload_np(w)
        self.scale = oracle.default_scale()
        self.groups = [list(range(i, min(i + HEADS_PER_UNIT, w.n_heads)))
                       for i in range(0, w.n_heads, HEADS_PER_UNIT)]
        a = self.a
        self.cut = []
        for hs in self.groups:
            idx = np.array(hs)
            self.cut.append((a["q_c"][:, idx], a["q_r"][:, idx], a["w_uk"][idx], a["w_uv"][idx]))

    def describe(self) -> str:
        return (f"units of {HEADS_PER_UNIT} heads of one sequence (non-absorbed fp64), "
                f"sequence k mod {self.w.batch}, head group k div {self.w.batch}")

    def run(self, k: int) -> float:
        """Unit k; returns the decode tokens it is worth (heads / n_heads)."""
        b = k % self.w.batch
        gi = (k // self.w.batch) % len(self.groups)
        q_c, q_r, w_uk, w_uv = self.cut[gi]
        a = self.a
        n = len(self.groups[gi])
        self.oracle.mla_decode_nonabsorbed(q_c, q_r, w_uk, w_uv, a["cache"], a["kv_lens"],
                                           self.scale, self.w.rope_base, a["page_table"],
                                           a["page_size"], pairs=[(b, i) for i in range(n)])
        return n / self.w.n_heads


def oracle_tokens_per_s(w, budget_s: float = 15.0):
    """cpu_baseline: oracle sample units, one after another, until the budget is spent.
    Returns (tokens/s, units, seconds, sample description)."""
    s = OracleSample(w)
    s.run(0)   # warm-up (BLAS threads, page faults)
    tokens, k, t0 = 0.0, 0, time.perf_counter()
    while True:
        tokens += s.run(1 + k)
        k += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return tokens / dt, k, dt, s.describe()


def blas_threads() -> int:
    try:
        import numpy  # noqa: F401
        from threadpoolctl import threadpool_info
        n = [d["num_threads"] for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return 0
    w = wl.config_workload(args.workload, seed=0)
    s = OracleSample(w)
    for k in range(args.warmup):
        s.run(k)
    tokens, t0 = 0.0, time.perf_counter()
    for k in range(args.steps):
        tokens += s.run(args.warmup + k)
    dt = time.perf_counter() - t0
    value = tokens / dt
    cores = blas_threads()
    sample = f"{args.steps} sample units of {args.workload}, one per step: {s.describe()}"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.workload, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- ours
def cache_copies(w) -> tuple[int, int]:
    """(copies, bytes per copy): enough copies of the cache that their total exceeds L2 four
    times, so a step that reads the next copy finds none of it in L2."""
    alloc = w.cache.numel() * w.cache.element_size()
    return max(1, math.ceil(4 * L2_BYTES / alloc)), alloc


def workload_config(w, name, world: int = 1):
    lens = w.kv_lens
    copies, alloc = cache_copies(w)
    return {"workload": name, "batch": w.batch, "n_heads": w.n_heads,
            "kv_len": int(lens[0]) if bool((lens == lens[0]).all()) else
            f"ragged {int(lens.min())}..{int(lens.max())}",
            "cached_tokens_per_gpu": w.cached_tokens,
            "layout": f"paged {w.page_size}" if w.page_size else "contiguous",
            "rope_base": w.rope_base, "d_c": 512, "d_rope": 64, "d_head": 128,
            "l2": f"inputs larger than L2: {copies} rotating cache copies of "
                  f"{alloc / 1e6:.0f} MB per GPU, one per step",
            "parallelism": f"replicas x{world} (one per GPU, no data-path collective)"}


def append_kv_measure(h, w, g, caches, copies, stream, args, world, local, dev,
                      d_model: int = 5120):
    """The cache write of the step's new tokens (mla_append_kv) on the same workload, timed
    alone from a graph of K calls. It is the step before the decode step, measured beside it
    and not counted in the step's tokens/s. Its inputs rotate over enough weight copies that
    they do not stay in L2 from one call to the next."""
    inp = {k: v.to(dev) for k, v in wl.draw_append_inputs(w.batch, d_model, seed=7).items()}
    wbytes = (inp["w_dkv"].numel() + inp["w_kr"].numel()) * 2
    n_w = max(1, math.ceil(4 * L2_BYTES / wbytes))
    weights = [(inp["w_dkv"], inp["w_kr"])] + [(inp["w_dkv"].clone(), inp["w_kr"].clone())
                                               for _ in range(n_w - 1)]

    def call(k):
        wd, wr = weights[k % n_w]
        h.append_kv(inp["hidden"], wd, wr, inp["gamma"], caches[k % copies], g.kv_lens,
                    g.page_table, stream=stream)

    ms = graph_ms(call, stream, args, world, local, dev)
    h.check_device_errors(stream)
    # algorithmic bytes: the two weights, the hidden states, gamma, the rows written
    algo = wbytes + w.batch * d_model * 2 + 512 * 2 + w.batch * ROW_BYTES
    hbm_gbs, _, peak_kind = measured_peaks()
    gbs = algo / (ms * 1e-3) / 1e9
    return {"us": ms * 1e3, "d_model": d_model, "batch": w.batch, "algorithmic_bytes": algo,
            "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm_gbs, "peak_source": f"{peak_kind} hbm_gbs",
            "l2": f"{n_w} rotating weight copies of {wbytes / 1e6:.1f} MB",
            "kernels": "kv_down_tc + kv_finalize", "gpu_launches": 2 * args.steps}


def graph_ms(fn, stream, args, world, local, dev):
    """Device time of fn(k), k = 0..K-1, replayed from one CUDA graph after W eager calls."""
    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            fn(k)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for k in range(args.steps):
            fn(k)
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, local, True)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, local, True)
    del graph
    return max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)


def multi_token_measure(w, g, caches, copies, stream, args, world, local, dev,
                        n_heads: int = 16, q_len: int = 8):
    """Several new tokens per sequence on the same cache: 16 heads x 8 new tokens (128
    attention rows, e.g. one tensor-parallel shard of the 128 heads verifying 8 draft tokens),
    the attention call alone, timed like the step. Every token's rows come from the cache
    once for all its tokens, so the cache bytes per call are those of one-token decode."""
    from mla_latent_kv_28_b200 import binding
    hm = binding.MlaDecode(n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                           rope_base=w.rope_base, q_len=q_len)
    qa = wl.draw_q_abs(w.batch, n_heads * q_len, seed=9).view(w.batch, q_len, n_heads, 576).to(dev)
    lat = torch.empty((w.batch, q_len, n_heads, 512), dtype=torch.bfloat16, device=dev)
    ms = graph_ms(lambda k: hm.decode_attn(qa, caches[k % copies], g.kv_lens, g.page_table, lat,
                                           None, want_lse=False, stream=stream),
                  stream, args, world, local, dev)
    hm.check_device_errors(stream)
    hm.close()
    cache_bytes = w.cached_tokens * ROW_BYTES
    hbm_gbs, _, peak_kind = measured_peaks()
    gbs = cache_bytes / (ms * 1e-3) / 1e9
    return {"n_heads": n_heads, "q_len": q_len, "attn_us": ms * 1e3,
            "query_tokens_per_s": world * w.batch * q_len / (ms * 1e-3),
            "kv_gbs": gbs, "frac_of_hbm": gbs / hbm_gbs, "peak_source": f"{peak_kind} hbm_gbs",
            "gpu_launches": 3 * args.steps}


def quantise_cache_e4m3(cache: torch.Tensor):
    """Input preparation for the quantised-cache measurement: every row as E4M3 codes and the
    smallest power-of-two scale 2^e with max|row| / 2^e <= 448 (rows that are not part of a
    sequence, NaN in the workload, get code 0 and e = 0)."""
    rows = cache.float().reshape(-1, cache.shape[-1])
    finite = torch.isfinite(rows).all(dim=1)
    rows = torch.where(finite[:, None], rows, torch.zeros_like(rows))
    amax = rows.abs().amax(dim=1).double()
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax))
    e = e + (amax / torch.exp2(e) > 448.0).double()
    e = e - ((amax > 0) & (amax / torch.exp2(e - 1) <= 448.0)).double()
    codes = (rows.double() / torch.exp2(e)[:, None]).float().to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.view(cache.shape), e.to(torch.int8).view(cache.shape[:2])


def fp8_cache_measure(h, w, g, stream, args, world, local, dev):
    """The attention call over the same rows held as a quantised cache (E4M3 codes + one
    power-of-two scale per row: 577 bytes per token instead of 1152), timed like the step,
    with as many rotating copies as keep every call's reads out of L2."""
    codes, exps = quantise_cache_e4m3(w.cache)
    codes, exps = codes.to(dev), exps.to(dev)
    per_copy = codes.numel() + exps.numel()
    n_copies = max(1, math.ceil(4 * L2_BYTES / per_copy))
    copies8 = [(codes, exps)] + [(codes.clone(), exps.clone()) for _ in range(n_copies - 1)]
    qa = wl.draw_q_abs(w.batch, w.n_heads, seed=11).to(dev)
    lat = torch.empty((w.batch, w.n_heads, 512), dtype=torch.bfloat16, device=dev)
    ms = graph_ms(lambda k: h.decode_attn_fp8(qa, copies8[k % n_copies][0], copies8[k % n_copies][1],
                                              g.kv_lens, g.page_table, lat, None, want_lse=False,
                                              stream=stream),
                  stream, args, world, local, dev)
    h.check_device_errors(stream)
    del copies8
    algo = w.cached_tokens * (576 + 1)
    hbm_gbs, _, peak_kind = measured_peaks()
    gbs = algo / (ms * 1e-3) / 1e9
    return {"attn_us": ms * 1e3, "bytes_per_token": 577, "algorithmic_bytes": algo,
            "kv_gbs": gbs, "frac_of_hbm": gbs / hbm_gbs, "peak_source": f"{peak_kind} hbm_gbs",
            "l2": f"{n_copies} rotating copies of {per_copy / 1e6:.0f} MB",
            "gpu_launches": 3 * args.steps}


def quantise_weight_e4m3(w: torch.Tensor):
    """Input preparation for the FP8-weight measurement: a bf16 weight [n_h, 128, 512] as E4M3
    codes [n_h * 128, 512] and one power-of-two exponent per 1 x 128 tile [n_h * 128, 4] (the
    smallest e with max|tile| / 2^e <= 448; codes by torch's float8_e4m3fn cast)."""
    rows = w.detach().double().reshape(-1, 4, 128)
    amax = rows.abs().amax(dim=2)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax))
    e = e + (amax / torch.exp2(e) > 448.0).double()
    e = e - ((amax > 0) & (amax / torch.exp2(e - 1) <= 448.0)).double()
    codes = (rows / torch.exp2(e)[:, :, None]).float().to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.reshape(-1, 512).contiguous(), e.to(torch.int8).contiguous()


def head_gemm_measure(b, args, world, local, dev):
    """The two head projections alone (absorb + RoPE, and W_UV), bf16 and FP8 weights, each
    timed from a graph of K calls over rotating weight copies (4x L2 in total, so every call
    reads its weights from HBM). Algorithmic bytes: the weights (bf16: 2 B per element; FP8:
    1 B + one exponent byte per 128) plus the call's inputs and outputs."""
    w, g, h, stream = b.w, b.g, b.h, b.stream
    B, H = w.batch, w.n_heads
    hbm_gbs, _, peak_kind = measured_peaks()
    q_abs = torch.empty((B, H, 576), dtype=torch.bfloat16, device=dev)
    latent = wl.draw_latent(B, H, seed=12).to(dev)
    out = torch.empty((B, H, 128), dtype=torch.bfloat16, device=dev)
    res = {}
    for kind in ("bf16", "fp8"):
        if kind == "bf16":
            wk, wv = g.w_uk, g.w_uv
            wbytes = wk.numel() * 2
        else:
            wk, wv = quantise_weight_e4m3(g.w_uk), quantise_weight_e4m3(g.w_uv)
            wbytes = wk[0].numel() + wk[1].numel()
        n = max(1, math.ceil(4 * L2_BYTES / wbytes))
        clone = (lambda t: t.clone()) if kind == "bf16" else (lambda t: (t[0].clone(), t[1].clone()))
        wks = [wk] + [clone(wk) for _ in range(n - 1)]
        wvs = [wv] + [clone(wv) for _ in range(n - 1)]
        if kind == "bf16":
            fa = lambda k: h.absorb_q(g.q_c, g.q_r, wks[k % n], g.kv_lens, q_abs, stream)
            fv = lambda k: h.apply_wuv(latent, wvs[k % n], out, stream)
        else:
            fa = lambda k: h.absorb_q_fp8(g.q_c, g.q_r, wks[k % n][0], wks[k % n][1], g.kv_lens, q_abs, stream)
            fv = lambda k: h.apply_wuv_fp8(latent, wvs[k % n][0], wvs[k % n][1], out, stream)
        ms_a = graph_ms(fa, stream, args, world, local, dev)
        ms_v = graph_ms(fv, stream, args, world, local, dev)
        h.check_device_errors(stream)
        io_a = B * H * (128 + 64 + 576) * 2
        io_v = B * H * (512 + 128) * 2
        for name, ms, io in (("absorb", ms_a, io_a), ("wuv", ms_v, io_v)):
            algo = wbytes + io
            gbs = algo / (ms * 1e-3) / 1e9
            res[f"{name}_{kind}"] = {"us": ms * 1e3, "algorithmic_bytes": algo, "achieved_gbs": gbs,
                                     "frac_of_hbm": gbs / hbm_gbs}
        del wks, wvs
    res["peak_source"] = f"{peak_kind} hbm_gbs"
    res["l2"] = "rotating weight copies, 4x L2 in total"
    res["gpu_launches"] = 8 * args.steps
    return res


def fp8_weight_step_ms(b, args, world, local, dev):
    """The whole step (absorb, attention, W_UV) with FP8 W_UK / W_UV, timed like the step."""
    g, h, stream, bufs = b.g, b.h, b.stream, b.bufs
    uk, uv = quantise_weight_e4m3(g.w_uk), quantise_weight_e4m3(g.w_uv)

    def step(k):
        q_abs = h.absorb_q_fp8(g.q_c, g.q_r, uk[0], uk[1], g.kv_lens, bufs["q_abs"], stream)
        h.decode_attn(q_abs, b.caches[k % b.copies], g.kv_lens, g.page_table, bufs["latent"],
                      None, want_lse=False, stream=stream)
        h.apply_wuv_fp8(bufs["latent"], uv[0], uv[1], bufs["out"], stream)

    ms = graph_ms(step, stream, args, world, local, dev)
    h.check_device_errors(stream)
    return {"ms_per_step": ms, "tokens_per_s": job_tokens_per_s(world, b.w.batch, ms),
            "weights": "E4M3 codes + one power-of-two scale per 1 x 128 tile", "gpu_launches": 5 * args.steps}


def prefill_measure(args, world, local, dev, T: int = 2048, n_heads: int = 128):
    """Prefill: one prompt of T new tokens (the whole cache: kv_len = T) through
    mla_prefill_attn, timed from a graph of K calls. Its work is a contraction (each cache row
    is read by 128 rows of one head at once and stays in L2), so it is reported against the
    tensor peak: FLOPs = sum over tokens of visible rows x n_h x 2 x (576 + 512)."""
    from mla_latent_kv_28_b200 import binding
    w = wl.make_workload(1, n_heads, [T], seed=13)
    g = w.to(dev)
    q = wl.draw_q_abs(T, n_heads, seed=14).view(1, T, n_heads, 576).to(dev)
    h = binding.MlaDecode(n_heads, 1, T, q_len=T)
    lat = torch.empty((1, T, n_heads, 512), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)
    ms = graph_ms(lambda k: h.prefill_attn(q, g.cache, g.kv_lens, None, lat, None, want_lse=False,
                                           stream=stream), stream, args, world, local, dev)
    h.check_device_errors(stream)
    h.close()
    flops = sum(t + 1 for t in range(T)) * n_heads * 2 * (576 + 512)
    peak_s, kind = sustained_tensor_peak()
    tflops = flops / (ms * 1e-3) / 1e12
    return {"prompt_tokens": T, "n_heads": n_heads, "us": ms * 1e3,
            "tokens_per_s": world * T / (ms * 1e-3), "tflops": tflops,
            "tensor_frac": tflops / peak_s, "peak_source": kind,
            "flops": flops, "gpu_launches": args.steps}


class DecodeBench:
    """One workload on this GPU: its inputs in HBM, the rotating cache copies, a handle, and
    the timings of the step, of the attention call alone, and of the step end to end."""

    def __init__(self, name, args, world, local, dev, rank):
        from mla_latent_kv_28_b200 import binding
        self.name, self.args, self.world, self.local, self.dev = name, args, world, local, dev
        self.w = wl.config_workload(name, seed=replica_seed(rank))
        self.g = self.w.to(dev)
        self.copies, self.alloc_bytes = cache_copies(self.w)
        self.caches = [self.g.cache] + [self.g.cache.clone() for _ in range(self.copies - 1)]
        w = self.w
        self.h = binding.MlaDecode(w.n_heads, w.batch, w.max_kv_len, page_size=w.page_size,
                                   rope_base=w.rope_base)
        B, H = w.batch, w.n_heads
        self.bufs = {"q_abs": torch.empty((B, H, 576), dtype=torch.bfloat16, device=dev),
                     "latent": torch.empty((B, H, 512), dtype=torch.bfloat16, device=dev),
                     "out": torch.empty((B, H, 128), dtype=torch.bfloat16, device=dev)}
        self.stream = torch.cuda.Stream(dev)   # a capturable stream for the graphs below

    def step(self, k):
        """One decode step through the public call a user makes (MlaDecode.step: absorption
        with the work plan beside it, split-KV attention, combine, W_UV; four launches)."""
        g = self.g
        self.h.step(g.q_c, g.q_r, g.w_uk, g.w_uv, self.caches[k % self.copies], g.kv_lens,
                    g.page_table, self.stream, self.bufs)

    def step_calls(self, k):
        """The same step as the three calls (absorb, attention with its own plan launch, W_UV;
        five launches): every kernel of the path in a launch of its own, for the profiles."""
        h, g, b, s = self.h, self.g, self.bufs, self.stream
        q_abs = h.absorb_q(g.q_c, g.q_r, g.w_uk, g.kv_lens, b["q_abs"], s)
        h.decode_attn(q_abs, self.caches[k % self.copies], g.kv_lens, g.page_table, b["latent"],
                      None, want_lse=False, stream=s)
        h.apply_wuv(b["latent"], g.w_uv, b["out"], s)

    def attn(self, k):
        h, g, b = self.h, self.g, self.bufs
        h.decode_attn(b["q_abs"], self.caches[k % self.copies], g.kv_lens, g.page_table,
                      b["latent"], None, want_lse=False, stream=self.stream)

    def device_times(self, clocks=None):
        """(step ms, attention ms, wall window of the step's timed region), each from a CUDA
        graph of K calls (no host launch time between kernels; the kernels are the launches
        the eager calls make), max over ranks."""
        args, stream, dev = self.args, self.stream, self.dev
        with torch.cuda.stream(stream):
            for k in range(args.warmup):
                self.step(k)
        self.h.check_device_errors(stream)
        step_graph, attn_graph = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(step_graph, stream=stream):
            for k in range(args.steps):
                self.step(k)
        with torch.cuda.graph(attn_graph, stream=stream):
            for k in range(args.steps):
                self.attn(k)
        with torch.cuda.stream(stream):
            step_graph.replay()
            attn_graph.replay()
        torch.cuda.synchronize(dev)
        self.h.check_device_errors(stream)

        def timed(graph):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier(self.world, self.local, True)
            torch.cuda.synchronize(dev)
            with torch.cuda.stream(stream):
                e0.record(stream)
                graph.replay()
                e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier(self.world, self.local, True)
            return e0.elapsed_time(e1) / args.steps

        w0 = time.perf_counter()
        ms = timed(step_graph)
        w1 = time.perf_counter()
        attn_ms = timed(attn_graph)
        self.h.check_device_errors(stream)
        del step_graph, attn_graph
        return (max_over_ranks(ms, self.world, dev), max_over_ranks(attn_ms, self.world, dev),
                (w0, w1))

    def e2e_times(self):
        """(graph ms, eager ms, h2d bytes, d2h bytes) per step, end to end through the public
        API: every step uploads its inputs (q^C, q^R, kv_len) from pinned host memory and
        downloads its head outputs to pinned host memory.

        Graph: as a serving loop would, the step runs as a CUDA graph with the copies on their
        own branches: graph k computes step k from the inputs graph k-1 uploaded, while
        uploading step k+1's inputs and downloading step k-1's outputs, so the copies overlap
        the kernels and one graph launch is all the host does per step. The graphs are
        captured from the public calls (MlaDecode.step and tensor copies); the timed region
        covers the first upload, K graphs, and the last download.
        Eager: the same step issued call by call from the host every step (no graph), so the
        host path of every C-ABI call (argument checks, tensor-map encodes, launches) and of
        the copies is inside the timed region."""
        args, stream, dev, g, h = self.args, self.stream, self.dev, self.g, self.h
        B, H = self.w.batch, self.w.n_heads
        hq_c = g.q_c.cpu().pin_memory()
        hq_r = g.q_r.cpu().pin_memory()
        hlens = g.kv_lens.cpu().pin_memory()
        hout = [torch.empty((B, H, 128), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        din = [(torch.empty_like(g.q_c), torch.empty_like(g.q_r), torch.empty_like(g.kv_lens))
               for _ in range(2)]
        dout = [torch.empty((B, H, 128), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        h2d = hq_c.numel() * 2 + hq_r.numel() * 2 + hlens.numel() * 4
        d2h = hout[0].numel() * 2
        copy = torch.cuda.Stream(dev)       # uploads
        copy_out = torch.cuda.Stream(dev)   # downloads, on another copy engine
        copies = self.copies

        def upload(slot):
            for d, hsrc in zip(din[slot], (hq_c, hq_r, hlens)):
                d.copy_(hsrc, non_blocking=True)

        def e2e_step(k):
            slot = k % 2
            fork = torch.cuda.Event()
            fork.record(stream)
            copy.wait_event(fork)
            copy_out.wait_event(fork)
            with torch.cuda.stream(copy):
                upload(1 - slot)                                        # inputs of step k+1
                join_in = torch.cuda.Event()
                join_in.record(copy)
            with torch.cuda.stream(copy_out):
                hout[1 - slot].copy_(dout[1 - slot], non_blocking=True)  # outputs of step k-1
                join_out = torch.cuda.Event()
                join_out.record(copy_out)
            dq_c, dq_r, dlens = din[slot]
            h.step(dq_c, dq_r, g.w_uk, g.w_uv, self.caches[k % copies], dlens, g.page_table,
                   stream, dict(self.bufs, out=dout[slot]))
            stream.wait_event(join_in)
            stream.wait_event(join_out)

        n_graphs = 2 * copies // math.gcd(2, copies)   # input slot and cache copy both cycle
        with torch.cuda.stream(stream):
            upload(0)
            for k in range(max(args.warmup, n_graphs)):
                e2e_step(k)
        torch.cuda.synchronize(dev)
        e2e_graphs = []
        for k in range(n_graphs):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                e2e_step(k)
            e2e_graphs.append(gr)
        with torch.cuda.stream(stream):
            upload(0)
            for k in range(n_graphs):
                e2e_graphs[k].replay()
        torch.cuda.synchronize(dev)
        h.check_device_errors(stream)
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(self.world, self.local, True)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e_start.record(stream)
            upload(0)
            for k in range(args.steps):
                e2e_graphs[k % n_graphs].replay()
            hout[(args.steps - 1) % 2].copy_(dout[(args.steps - 1) % 2], non_blocking=True)
            e_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(self.world, self.local, True)
        h.check_device_errors(stream)
        del e2e_graphs
        graph_ms_ = max_over_ranks(e_start.elapsed_time(e_end) / args.steps, self.world, dev)

        # eager: the same step (copies on their own streams, overlapping the kernels), issued
        # call by call from the host every step instead of replayed from a graph
        with torch.cuda.stream(stream):
            upload(0)
            for k in range(args.warmup):
                e2e_step(k)
        torch.cuda.synchronize(dev)
        barrier(self.world, self.local, True)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e_start.record(stream)
            upload(0)
            for k in range(args.steps):
                e2e_step(k)
            hout[(args.steps - 1) % 2].copy_(dout[(args.steps - 1) % 2], non_blocking=True)
            e_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(self.world, self.local, True)
        h.check_device_errors(stream)
        eager_ms = max_over_ranks(e_start.elapsed_time(e_end) / args.steps, self.world, dev)
        return graph_ms_, eager_ms, h2d, d2h

    def roofline(self, attn_ms):
        hbm_gbs, bf16_tf, peak_kind = measured_peaks()
        cache_bytes = self.w.cached_tokens * ROW_BYTES
        achieved = cache_bytes / (attn_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved / hbm_gbs, "traffic": profiled_traffic(self.name),
                "kernel": "mla_decode_attn (plan + split-KV + combine)",
                "peak_source": f"{peak_kind} hbm_gbs", "algorithmic_bytes": cache_bytes,
                "tensor_frac_of_measured": (self.w.cached_tokens * 2 * 1088 * self.w.n_heads)
                / (attn_ms * 1e-3) / (bf16_tf * 1e12)}

    def close(self):
        self.h.close()
        del self.caches, self.g


def run_profile(args):
    """W warm-up steps, then K eager steps of the hot path of one workload, issued as the three
    calls (every kernel in a launch of its own, the plan kernel included): nothing else runs,
    so an ncu capture of this command sees only the step's kernels."""
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    bench = DecodeBench(args.workload, args, 1, local, dev, rank)
    with torch.cuda.stream(bench.stream):
        for k in range(args.warmup + args.steps):
            bench.step_calls(k)
    torch.cuda.synchronize(dev)
    bench.h.check_device_errors(bench.stream)
    bench.close()
    return 0


def run_ours(args):
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, local, "nccl")

    main = DecodeBench(args.workload, args, world, local, dev, rank)
    w = main.w
    clocks = ClockSampler(local)
    clocks.start()
    ms_max, attn_ms, (w0, w1) = main.device_times()
    e2e_ms, eager_ms, h2d, d2h = main.e2e_times()
    clocks.stop()

    append = append_kv_measure(main.h, w, main.g, main.caches, main.copies, main.stream, args,
                               world, local, dev)
    tokens = multi_token_measure(w, main.g, main.caches, main.copies, main.stream, args, world,
                                 local, dev)
    fp8 = fp8_cache_measure(main.h, w, main.g, main.stream, args, world, local, dev)
    heads = head_gemm_measure(main, args, world, local, dev)
    prefill = prefill_measure(args, world, local, dev)
    fp8w = fp8_weight_step_ms(main, args, world, local, dev)
    roof = main.roofline(attn_ms)
    main.close()
    del main
    torch.cuda.empty_cache()

    # the other workloads, timed the same way (one at a time, each with its own cache copies)
    others = {}
    for name in sorted(wl.CONFIGS):
        if name == args.workload or args.headline_only:
            continue
        o = DecodeBench(name, args, world, local, dev, rank)
        o_ms, o_attn, _ = o.device_times()
        o_e2e, o_eager, _, _ = o.e2e_times()
        others[name] = {"tokens_per_s": job_tokens_per_s(world, o.w.batch, o_ms),
                        "ms_per_step": o_ms, "attn_us": o_attn * 1e3,
                        "cached_tokens_per_gpu": o.w.cached_tokens,
                        "roofline": o.roofline(o_attn),
                        "e2e": {"value": job_tokens_per_s(world, o.w.batch, o_e2e),
                                "eager_value": job_tokens_per_s(world, o.w.batch, o_eager),
                                "unit": "tokens/s"},
                        "config": workload_config(o.w, name, world),
                        "gpu_launches": 4 * args.steps}
        o.close()
        del o
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, units, secs, desc = oracle_tokens_per_s(w)
        cpu = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{units} sample units of {args.workload} in {secs:.1f} s: {desc}"}

    cache_bytes = w.cached_tokens * ROW_BYTES
    B = w.batch
    line = {
        "metric": METRIC, "value": job_tokens_per_s(world, B, ms_max), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; workload shapes of the DeepSeek-V2 MLA layer)",
        "config": workload_config(w, args.workload, world),
        "kv_gbs": world * cache_bytes / (ms_max * 1e-3) / 1e9,
        "attn_us": attn_ms * 1e3,
        "roofline": roof,
        "e2e": {"value": job_tokens_per_s(world, B, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "eager_value": job_tokens_per_s(world, B, eager_ms),
                "how": "value: per-step CUDA graphs of MlaDecode.step with the copies on side "
                       "branches; eager_value: the same step issued call by call, no graphs"},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks.summary(w0, w1),
    }
    line["append_kv"] = append
    line["multi_token"] = tokens
    line["fp8_cache"] = fp8
    line["head_gemms"] = heads
    line["prefill"] = prefill
    line["fp8_weights"] = fp8w
    if others:
        line["workloads"] = others
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def relaunch_under_torchrun(argv, gpus: int) -> int:
    """`--gpus N` (N > 1) started without torchrun: start N ranks through torchrun on this
    node (rendezvous on 127.0.0.1) and return its exit status."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only --workload (no `workloads` key)")
    ap.add_argument("--profile", action="store_true",
                    help="run W + K eager steps of --workload and nothing else (for ncu)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    rank, world, _ = dist_env()
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return relaunch_under_torchrun(argv, args.gpus)
    if world != args.gpus:
        print(f"error: --gpus {args.gpus} but WORLD_SIZE {world}: launch one process per GPU "
              f"(torchrun --nproc-per-node {args.gpus}) or drop torchrun", file=sys.stderr)
        return 2
    if args.profile:
        return run_profile(args)
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
