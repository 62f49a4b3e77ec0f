"""Benchmark of block-sparse video self-attention on B200.

One step = one whole attention call over one batch of synthetic inputs:
layout -> permute Q, K, V -> pool -> top-k select -> sparse attention ->
unpermute, all through libbsa.so on one stream.  Default workload: the 720p
121-frame clip (B=2 CFG pair, 24 heads of 128, 32x48x80 = 122,880 tokens,
fixed 4x4x4 blocks, sparsity 0.75 = keep 480 of 1,920).  Metric: effective
TFLOP/s counted on kept 64x64 tiles only (4*64*64*d FLOP per tile), plus
ms per call and the fraction of the measured bf16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 720p|720p_dyn|ref_prefix|lowres|sweep] [--keep-ratio r]
                    [--block-mode 0|1]
                    [--sweep]   # keep-ratio sweep on the 1152x640 grid instead

N > 1 runs under torchrun: each rank processes its own independent call
(its own seeded inputs; the (batch, head) problems share nothing), no
collective on the data path; `value` = all ranks' kept-tile FLOPs / the
slowest rank's time (weak scaling).

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (one (batch, head), a seeded subset of query
blocks per step) and reports the same metric for that sample.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gen import SWEEP_KEEP_RATIOS, config, derived_sizes, make_qkv  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per sparse-attention launch from one ncu capture
# of a B=1 x 4-head launch of the 720p grid (2.119 GB read + 0.126 GB
# written), scaled by the number of (batch, head) problems.  Valid only for
# the kernel source it was measured on and the 720p keep-480 fixed-block
# workload on the permuted path; null otherwise.
ATTN_TRAFFIC = {"sha256": "4d2c4962edb62dac8bee4b4d4b3f9ff60c58d586771bb1c8242ce43d2a543feb",
                "bytes_per_bh": (1.943522e9 + 0.124784e9) / 4, "workload": ("720p", 0.25, 0)}


def attn_traffic(cfg, keep_ratio):
    import hashlib
    src = os.path.join(ROOT, "block_sparse_attention_47_b200", "csrc", "attention.cu")
    try:
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    if digest != ATTN_TRAFFIC["sha256"]:
        return None
    if (cfg.get("name"), keep_ratio, cfg["block_mode"]) != ATTN_TRAFFIC["workload"]:
        return None
    if PATH["path"] != "perm" or PATH.get("windows") is not None:
        return None
    return ATTN_TRAFFIC["bytes_per_bh"] * cfg["B"] * cfg["heads"]
METRIC = "ms/call & effective TFLOP/s (kept tiles) at 122,880 tok, s=0.75; % BF16 peak"


# ----------------------------------------------------------------------------
def peaks():
    """The measured peaks where the file gives them, each missing number
    taken from the fallback figures; the kind says which the sustained bf16
    figure (the roofline's denominator) is."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    p = dict(FALLBACK_PEAKS)
    try:
        with open(path) as f:
            got = json.load(f)
    except (OSError, ValueError):
        return p, "fallback"
    if not isinstance(got, dict):
        return p, "fallback"
    for key in FALLBACK_PEAKS:
        if isinstance(got.get(key), (int, float)) and got[key] > 0:
            p[key] = float(got[key])
    measured = isinstance(got.get("bf16_tflops_sustained"), (int, float))
    return p, "measured" if measured else "fallback"


# tcgen05 dense bf16 rate per SM and clock (4,096 multiply-adds; measured
# back-to-back with M=128, N>=128) and the SM count of a B200
MMA_FLOP_PER_CLK_SM = 8192
N_SM = 148


def mma_rate_frac(tflops, clocks):
    """The kernel's rate over the tensor cores' rate at the SM clock sampled
    during the timed region (both sides at the same clock)."""
    if not clocks or not clocks.get("sm_mhz"):
        return None
    return tflops / (MMA_FLOP_PER_CLK_SM * N_SM * clocks["sm_mhz"] * 1e6 / 1e12)


def kept_tiles(cfg, keep):
    """64x64 tiles attention touches: video query blocks keep every prefix
    block plus `keep` video blocks; prefix query blocks keep every block."""
    s = derived_sizes(cfg)
    per_bh = s["nbv"] * (s["nbp"] + keep) + s["nbp"] * s["nb"]
    return cfg["B"] * cfg["heads"] * per_bh


def dense_tiles(cfg):
    s = derived_sizes(cfg)
    return cfg["B"] * cfg["heads"] * s["nb"] * s["nb"]


def tile_flops(cfg):
    return 4 * 64 * 64 * cfg["head_dim"]


def stage_bandwidth(cfg, stage_ms):
    """Achieved GB/s of the memory-bound stages: algorithmic bytes (one bf16
    [B, N, heads, d] tensor is R bytes) over each stage's time.  permute
    (with the pooling fused in) reads and writes Q, K, V (6R), a separate
    pool would read permuted Q and K (2R), unpermute reads and writes O (2R),
    the dynamic layout reads K (R); the pooled outputs and index lists are
    small and not counted."""
    s = derived_sizes(cfg)
    R = cfg["B"] * s["N"] * cfg["heads"] * cfg["head_dim"] * 2
    if PATH["path"] == "raster":
        nbytes = {"pool": 2 * R}   # pool_raster reads raster Q and K
    else:
        nbytes = {"permute": 6 * R, "unpermute": 2 * R}
    if cfg["block_mode"] == 1:
        nbytes["layout"] = R
    return {k: round(v / (stage_ms[k] * 1e-3) / 1e9, 1)
            for k, v in nbytes.items() if stage_ms.get(k, 0) > 0}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.tmp = None
        self.target = self._gpu_id(device_index)

    @staticmethod
    def _gpu_id(i):
        try:
            u = str(torch.cuda.get_device_properties(i).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return str(i)

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.target, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[3:7]))
                except ValueError:
                    continue
        os.unlink(self.tmp.name)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
def dist_setup(want_gpus):
    """Rank, world size and local rank from the torchrun environment; for
    N > 1 one process group over NCCL (gloo on a host without CUDA, where
    only the host-side plumbing and the oracle arm can run)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != want_gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (want_gpus, world))
    if world > 1:
        import datetime
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout,
                                                 device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group("gloo", timeout=timeout)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """The largest x over all ranks (every rank gets it)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank):
    """Each rank draws its own inputs: independent calls, nothing shared."""
    return 42002 + 1000 * rank


def whole_job_tflops(world, flops_per_rank, ms_slowest):
    """Weak scaling: every rank does the same work; the job's throughput is
    all ranks' FLOPs over the slowest rank's time."""
    return world * flops_per_rank / (ms_slowest / 1e3) / 1e12


# ----------------------------------------------------------------------------
STAGES = ("layout", "permute", "pool", "select", "attention", "unpermute")


# "perm" (permuted copies) or "raster" (permute-free); the learned-gate
# matrices (select_topk_gated) and the window heads (window attention) when
# those modes are timed
PATH = {"path": "perm", "row_pad": 0, "gate": None, "windows": None}

# window-head patterns for --windows (w_t, w_y, w_x), negative = unbounded: a
# spatial head sees +-1 latent frame, a temporal head +-2 latent pixels
WINDOW_PATTERNS = {"spatial": [(1, -1, -1)], "temporal": [(-1, 2, 2)],
                   "mixed": [(1, -1, -1), (-1, 2, 2)]}


def run_step(bsa, attn, q, k, v, out, ev):
    """One call; ev (list of 7 events or None) brackets the six stages.  The
    permute-free path has no permute and unpermute stages (0 ms); window
    heads have no pool and select stages either."""
    p, L = attn.prob, attn.layout_buf
    raster = PATH["path"] == "raster"
    windows = PATH["windows"]
    if ev:
        ev[0].record()
    bsa.layout(p, k, L)
    if ev:
        ev[1].record()
    if not raster:
        # the permutes and the pooling in one pass (its time is the
        # "permute" stage; "pool" stays empty)
        bsa.permute_pool(p, L, q, k, v, attn.qp, attn.kp, attn.vp, attn.q_pool, attn.k_pool)
    if ev:
        ev[2].record()
    if windows is None and raster:
        bsa.pool_raster(p, L, q, k, attn.q_pool, attn.k_pool)
    if ev:
        ev[3].record()
    if windows is not None:
        pass
    elif PATH["gate"] is not None:
        bsa.select_topk_gated(p, attn.q_pool, attn.k_pool, PATH["gate"], attn.idx, attn.cnt)
    else:
        bsa.select_topk(p, attn.q_pool, attn.k_pool, attn.idx, attn.cnt)
    if ev:
        ev[4].record()
    if windows is not None:
        bsa.window_attn_fwd_raster(p, L, q, k, v, windows, out, attn.status)
    elif raster:
        bsa.sparse_attn_fwd_raster(p, L, q, k, v, attn.idx, attn.cnt, out, attn.status)
    else:
        bsa.sparse_attn_fwd(p, L, attn.qp, attn.kp, attn.vp, attn.idx, attn.cnt, attn.op,
                            attn.status)
    if ev:
        ev[5].record()
    if not raster:
        bsa.unpermute(p, L, attn.op, out)
    if ev:
        ev[6].record()


def launches_per_step(cfg):
    layout = 2 if cfg["block_mode"] == 1 else 1
    if PATH["windows"] is not None:
        return layout + 1
    if PATH["path"] == "raster":
        return layout + 1 + 1 + 1
    return layout + 1 + 1 + 1 + 1


def window_heads(cfg, pattern):
    """Per-head windows of a pattern, cycling over the heads."""
    pat = WINDOW_PATTERNS[pattern]
    return [pat[h % len(pat)] for h in range(cfg["heads"])]


def window_tiles(cfg, wins):
    """64x64 tiles the window heads visit on the fixed 4x4x4 layout: every
    prefix row and column, plus the video block pairs whose boxes come within
    the window on every axis (two blocks d apart along an axis have a gap of
    4|d| - 3 tokens).  The axes are independent, so the video count of a head
    is the product of the per-axis counts."""
    s = derived_sizes(cfg)
    n = {"t": cfg["T"] // 4, "y": cfg["H"] // 4, "x": cfg["W"] // 4}
    per_b = 0
    for w3 in wins:
        video = 1
        for w, ax in zip(w3, ("t", "y", "x")):
            a = np.arange(n[ax])
            gap = np.maximum(0, 4 * np.abs(a[:, None] - a[None, :]) - 3)
            video *= int(((gap <= w) | (w < 0)).sum())
        per_b += video + s["nbp"] * s["nb"] + s["nbv"] * s["nbp"]
    return cfg["B"] * per_b


def measure(cfg, keep, steps, warmup, world, rank, local, do_e2e, do_dense):
    import block_sparse_attention_47_b200 as bsa
    from block_sparse_attention_47_b200 import build
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    prob = bsa.Problem.make(**dict(cfg, keep_blocks=keep))
    q, k, v = make_qkv(cfg, rank_seed(rank), pad_fill=0.0, device=dev)
    if PATH.get("row_pad"):
        # the same tensors in rows of heads*d + row_pad elements (a wider token
        # stride, as in a fused projection's output buffer)
        def padded(x):
            B, N, h, d = x.shape
            buf = torch.zeros((B, N, h * d + PATH["row_pad"]), dtype=x.dtype, device=x.device)
            buf[..., :h * d] = x.reshape(B, N, h * d)
            return buf[..., :h * d].view(B, N, h, d)
        q, k, v = padded(q), padded(k), padded(v)
    attn = bsa.BlockSparseAttention(prob, device=dev)
    out = torch.empty_like(q)
    wins = None
    if PATH.get("window_pattern"):
        wins = window_heads(cfg, PATH["window_pattern"])
        PATH["windows"] = torch.tensor(wins, dtype=torch.int32, device=dev)
    if PATH.get("gate_seed") is not None:
        from gen import make_gate
        PATH["gate"] = make_gate(cfg["heads"], cfg["head_dim"], PATH["gate_seed"], device=dev)
    torch.cuda.synchronize()

    flops = (window_tiles(cfg, wins) if wins else kept_tiles(cfg, keep)) * tile_flops(cfg)
    for _ in range(warmup):
        run_step(bsa, attn, q, k, v, out, None)
    torch.cuda.synchronize()
    attn.check_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        run_step(bsa, attn, q, k, v, out, evs[i])
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    attn.check_status()
    ms_total = t0.elapsed_time(t1)
    ms_step = max_over_ranks(ms_total / steps, world)
    stage_ms = {}
    for si, name in enumerate(STAGES):
        stage_ms[name] = statistics.median(e[si].elapsed_time(e[si + 1]) for e in evs)
    attn_ms = statistics.mean(e[4].elapsed_time(e[5]) for e in evs)

    res = dict(ms_step=ms_step, flops=flops, stage_ms=stage_ms, attn_ms=attn_ms, clocks=clocks)

    if do_dense:
        o = torch.empty_like(attn.op)
        bsa.dense_attn_fwd(prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, o, attn.status)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(2):
            bsa.dense_attn_fwd(prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, o, attn.status)
        b_.record()
        torch.cuda.synchronize()
        res["dense_ms"] = a.elapsed_time(b_) / 2
        res["dense_flops"] = dense_tiles(cfg) * tile_flops(cfg)
        del o

    if PATH.get("backward") and PATH["path"] == "perm":
        # the training step's attention: forward with row statistics, then
        # the backward (dQ, dK, dV) over the same kept tiles
        n_tok = attn.sizes.n_tokens
        lse = torch.empty((cfg["B"], cfg["heads"], n_tok), dtype=torch.float32, device=dev)
        o = torch.empty_like(attn.op)
        dout = torch.randn(attn.op.shape, device=dev).to(torch.bfloat16)
        grads = [torch.empty_like(attn.op) for _ in range(3)]
        ws = torch.empty(bsa.bwd_workspace_bytes(prob), dtype=torch.uint8, device=dev)

        def fwd():
            bsa.sparse_attn_fwd_lse(prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, attn.idx,
                                    attn.cnt, o, lse, attn.status)

        def bwd():
            bsa.sparse_attn_bwd(prob, attn.layout_buf, attn.qp, attn.kp, attn.vp, o, dout, lse,
                                attn.idx, attn.cnt, *grads, ws, attn.status)
        for _ in range(warmup):
            fwd()
            bwd()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        fms, bms = [], []
        for _ in range(steps):
            ev[0].record()
            fwd()
            ev[1].record()
            bwd()
            ev[2].record()
            torch.cuda.synchronize()
            fms.append(ev[0].elapsed_time(ev[1]))
            bms.append(ev[1].elapsed_time(ev[2]))
        attn.check_status()
        res["backward"] = dict(fwd_lse_ms=statistics.median(fms), bwd_ms=statistics.median(bms))
        del lse, o, dout, grads, ws

    if do_e2e:
        # the call a user with host tensors makes: bsa_forward_host moves
        # every input to the device and the output back, overlapped with the
        # computation by groups of heads
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        hout = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hg = bsa.default_heads_per_group(cfg["heads"])

        def e2e_step():
            attn.host_call(hq, hk, hv, out=hout, heads_per_group=hg,
                           raster=PATH["path"] == "raster")

        for _ in range(max(1, min(warmup, 2))):
            e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(2, min(steps, 5))
        barrier(world)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n_e2e):
            e2e_step()
        b_.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(a.elapsed_time(b_) / n_e2e, world)
        nbytes = q.numel() * q.element_size()
        res["e2e"] = dict(ms=e2e_ms, h2d=3 * nbytes, d2h=nbytes, heads_per_group=hg)
        attn.check_status()
        del hq, hk, hv, hout
    return res


# ----------------------------------------------------------------------------
def oracle_sample(cfg, keep, n_query_blocks, seed, inputs=None):
    """Run the fp64 oracle on one (batch, head) of the workload for a seeded
    sample of query blocks; returns (seconds, kept tiles processed)."""
    from oracle import bsa_oracle as O
    geo = O.Geometry(cfg)
    if inputs is None:
        q, k, v = make_qkv(dict(cfg, B=1, heads=1), seed, pad_fill=0.0)
        inputs = [t[0, :, 0].float().numpy().astype(np.float64) for t in (q, k, v)]
    qn, kn, vn = inputs
    rng = np.random.default_rng(seed)
    blocks = sorted(set(rng.choice(geo.nb, size=min(n_query_blocks, geo.nb), replace=False).tolist()))
    t0 = time.perf_counter()
    if cfg["block_mode"] == 0:
        perm = O.fixed_perm(geo)
    else:
        kk = kn[None, :, None, :] if kn.ndim == 2 else kn
        v_ = O.region_variation(geo, kk[0])
        perm = O.dynamic_perm(geo, [O.shape_code(v_[r], cfg["dyn_tau"]) for r in range(len(v_))])
    qp, kp, vp = (O.permute(geo, perm, x) for x in (qn, kn, vn))
    lists = O.select(geo, O.pool(geo, perm, qp), O.pool(geo, perm, kp), keep, rows=blocks)
    O.block_sparse_attention(geo, perm, qp, kp, vp, lists, 1 / math.sqrt(geo.d), blocks)
    secs = time.perf_counter() - t0
    return secs, sum(len(lists[i]) for i in blocks), inputs


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, keep, budget_s=15.0):
    n = 32
    secs, tiles, inputs = oracle_sample(cfg, keep, n, 4242)
    # grow the sample to roughly the time budget (one more run)
    if secs < budget_s / 3:
        n = int(n * min(budget_s / max(secs, 1e-3), 16))
        secs, tiles, _ = oracle_sample(cfg, keep, n, 4243, inputs)
    tflops = tiles * tile_flops(cfg) / secs / 1e12
    full = kept_tiles(cfg, keep)
    return {"value": tflops, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "extrapolated_full_call_s": secs * full / tiles,
            "sample": "fp64 numpy oracle, one (batch, head) of %s: layout, permute, pool, full "
                      "block scores, top-k and attention for %d seeded query blocks (%d kept "
                      "tiles) in %.1f s; value = kept-tile FLOPs / wall time.  The oracle "
                      "loops over query blocks in one Python thread; only its numpy matrix "
                      "products use the %d BLAS threads counted as cores.  "
                      "extrapolated_full_call_s scales the sample linearly in kept tiles to "
                      "the whole call (%d tiles)"
                      % (cfg.get("name", "?"), n, tiles, secs, cpu_threads(), full)}


# ----------------------------------------------------------------------------
def reference_arm(args, cfg, keep, world, rank):
    if rank != 0:
        return
    n_blocks = 48
    _, _, inputs = oracle_sample(cfg, keep, 1, 7)
    for i in range(args.warmup):
        oracle_sample(cfg, keep, n_blocks, 100 + i, inputs)
    tiles = 0
    secs = 0.0
    for i in range(args.steps):
        s, t, _ = oracle_sample(cfg, keep, n_blocks, 200 + i, inputs)
        secs += s
        tiles += t
    value = tiles * tile_flops(cfg) / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, keep, args),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(),
                             "kind": "oracle",
                             "sample": "per step: one (batch, head), %d seeded query blocks of "
                                       "the workload through the fp64 oracle" % n_blocks},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def workload_config(cfg, keep, args):
    s = derived_sizes(cfg)
    return {"workload": "%s: B=%d heads=%d d=%d grid %dx%dx%d%s = %d tokens, %d blocks, keep %d "
                        "(%s blocks)" % (cfg.get("name"), cfg["B"], cfg["heads"], cfg["head_dim"],
                                         cfg["T"], cfg["H"], cfg["W"],
                                         " + prefix %s" % (list(cfg["prefix"]),) if cfg["prefix"] else "",
                                         s["N"], s["nb"], keep,
                                         "dynamic 8x8x8" if cfg["block_mode"] else "fixed 4x4x4"),
            "global_batch": cfg["B"] * args.gpus, "seq_len": s["N"], "keep_blocks": keep,
            "keep_ratio": cfg["keep_ratio"], "parallelism": "independent calls per GPU (dp%d)" % args.gpus,
            "path": PATH["path"],
            "selection": ("window heads (%s: %s)" % (PATH["window_pattern"],
                                                     WINDOW_PATTERNS[PATH["window_pattern"]])
                          if PATH.get("window_pattern") else
                          "learned gate (synthetic seeded matrices)" if PATH.get("gate_seed")
                          else "pooled-mean top-k"),
            "l2": "inputs larger than L2 (Q, K, V %.2f GB each); no flush" %
                  (cfg["B"] * s["N"] * cfg["heads"] * cfg["head_dim"] * 2 / 1e9)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--config", default="720p")
    ap.add_argument("--keep-ratio", type=float, default=None)
    ap.add_argument("--heads", type=int, default=None, help="override heads (profiling runs)")
    ap.add_argument("--batch", type=int, default=None, help="override B (profiling runs)")
    ap.add_argument("--block-mode", type=int, default=None, choices=(0, 1),
                    help="override the block mode (0 fixed 4x4x4, 1 dynamic 8x8x8)")
    ap.add_argument("--path", default="perm", choices=("raster", "perm"),
                    help="perm: permute -> attention -> unpermute; raster: tiles read straight "
                         "from the raster tensors (no permuted copies)")
    ap.add_argument("--row-pad", type=int, default=0,
                    help="extra elements per raster token row (a wider token stride)")
    ap.add_argument("--backward", action="store_true",
                    help="also time the training step's attention: forward with row "
                         "statistics and the backward (permuted path)")
    ap.add_argument("--gate", action="store_true",
                    help="learned-gate selection with seeded synthetic gate matrices")
    ap.add_argument("--windows", default=None, choices=sorted(WINDOW_PATTERNS),
                    help="window heads instead of top-k selection (raster path, fixed blocks); "
                         "the metric counts the tiles the windows visit")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="keep-ratio sweep on the 1152x640 grid")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    PATH["path"] = args.path
    PATH["row_pad"] = args.row_pad
    PATH["gate_seed"] = 42010 if args.gate else None
    PATH["window_pattern"] = args.windows
    PATH["backward"] = args.backward
    if args.windows:
        PATH["path"] = "raster"

    cfg = config(args.config)
    if args.keep_ratio is not None:
        cfg["keep_ratio"] = args.keep_ratio
    if args.heads is not None:
        cfg["heads"] = args.heads
    if args.batch is not None:
        cfg["B"] = args.batch
    if args.block_mode is not None:
        cfg["block_mode"] = args.block_mode
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            # the oracle arm shares nothing with the CUDA path: the keep count
            # comes from the oracle and the product library is never loaded
            from oracle import bsa_oracle as O
            reference_arm(args, cfg, O.keep_count(derived_sizes(cfg)["nbv"], cfg["keep_ratio"]),
                          world, rank)
            return
        import block_sparse_attention_47_b200 as bsa
        from block_sparse_attention_47_b200 import build
        build.build()
        keep = bsa.keep_count(derived_sizes(cfg)["nbv"], cfg["keep_ratio"])
        if args.sweep:
            sweep(args, world, rank, local)
            return
        res = measure(cfg, keep, args.steps, args.warmup, world, rank, local,
                      not args.no_e2e, not args.no_dense and world == 1)
        if rank != 0:
            return
        pk, pk_kind = peaks()
        value = whole_job_tflops(world, res["flops"], res["ms_step"])
        attn_tflops = res["flops"] / (res["attn_ms"] / 1e3) / 1e12
        peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded smooth field + noise, no weights)",
            "config": workload_config(cfg, keep, args),
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak,
                         "unit": "TFLOP/s", "frac": attn_tflops / peak,
                         "traffic": attn_traffic(cfg, cfg["keep_ratio"]),
                         "kernel": "attn_fwd_kernel<128,false,%s> (sparse attention, %s)" % (
                             "true" if PATH["path"] == "raster" else "false",
                             "raster tensors" if PATH["path"] == "raster" else "permuted tensors"),
                         "peak_kind": "%s bf16 sustained" % pk_kind,
                         "frac_of_burst": attn_tflops / pk["bf16_tflops"],
                         "frac_of_mma_rate_at_clock": mma_rate_frac(attn_tflops, res["clocks"])},
            "stage_ms": res["stage_ms"],
            "stage_gbs": stage_bandwidth(cfg, res["stage_ms"]),
            "gpu_launches": launches_per_step(cfg) * args.steps,
        }
        if "dense_ms" in res:
            line["dense"] = {"ms": res["dense_ms"],
                             "tflops": res["dense_flops"] / (res["dense_ms"] / 1e3) / 1e12,
                             "speedup_sparse_attention_vs_dense": res["dense_ms"] / res["attn_ms"],
                             "speedup_full_call_vs_dense": res["dense_ms"] / res["ms_step"]}
        if "backward" in res:
            bw = res["backward"]
            # standard count: the backward's five products (S recomputed,
            # dP, dV, dQ, dK) are 2.5x the forward's two per kept tile
            line["backward"] = {
                "fwd_lse_ms": bw["fwd_lse_ms"], "bwd_ms": bw["bwd_ms"],
                "bwd_tflops": 2.5 * res["flops"] / (bw["bwd_ms"] / 1e3) / 1e12,
                "flop_count": "2.5 x the forward's kept-tile FLOPs (the kernels compute S and "
                              "dP in both passes, 3.5 x)"}
        if "e2e" in res:
            e = res["e2e"]
            line["e2e"] = {"value": whole_job_tflops(world, res["flops"], e["ms"]), "unit": "TFLOP/s",
                           "ms_per_step": e["ms"], "h2d_bytes_per_step": e["h2d"],
                           "d2h_bytes_per_step": e["d2h"],
                           "api": "bsa_forward_host, %d heads per group" % e["heads_per_group"]}
        if res["clocks"]:
            line["clocks"] = res["clocks"]
        if world == 1 and not args.no_cpu:
            line["cpu_baseline"] = cpu_baseline(cfg, keep)
        print(json.dumps(line))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


def sweep(args, world, rank, local):
    """ms per call and the layout/permute/pool/select overhead as the keep
    ratio falls, on the 1152x640 grid (plus the 40-layer schedule)."""
    from gen import layer_keep_schedule
    base = config("sweep")
    nbv = derived_sizes(base)["nbv"]
    rows = []
    import block_sparse_attention_47_b200 as bsa
    for r in SWEEP_KEEP_RATIOS:
        keep = bsa.keep_count(nbv, r)
        cfg = dict(base, keep_ratio=r)
        res = measure(cfg, keep, args.steps, args.warmup, world, rank, local, False, False)
        st = res["stage_ms"]
        overhead = sum(st[s] for s in ("layout", "permute", "pool", "select", "unpermute"))
        rows.append({"keep_ratio": r, "keep": keep, "ms_per_call": res["ms_step"],
                     "attention_ms": st["attention"], "overhead_ms": overhead,
                     "overhead_share": overhead / res["ms_step"],
                     "tflops_kept": res["flops"] / (res["ms_step"] / 1e3) / 1e12,
                     "stage_ms": st})
    sched = layer_keep_schedule()
    by_ratio = {row["keep_ratio"]: row["ms_per_call"] for row in rows}
    measured = schedule_ms(base, sched, args, world, rank, local)
    if rank == 0:
        print(json.dumps({"sweep": "1152x640 grid, 92,160 tokens, 24 heads, d=128",
                          "rows": rows,
                          "layer_schedule_40": {"keep_ratios": sched,
                                                "ms_total_measured": measured,
                                                "ms_total_sum_of_rows":
                                                    sum(by_ratio[r] for r in sched)}}))


def schedule_ms(base, sched, args, world, rank, local):
    """The 40-layer schedule timed as 40 consecutive calls on one stream (one
    set of buffers per keep ratio, one set of seeded inputs), the median of
    `args.steps` passes after `args.warmup` untimed ones, max over ranks."""
    import block_sparse_attention_47_b200 as bsa
    dev = torch.device("cuda", local)
    nbv = derived_sizes(base)["nbv"]
    attns = {r: bsa.BlockSparseAttention(
        bsa.Problem.make(**dict(base, keep_blocks=bsa.keep_count(nbv, r))), device=dev)
        for r in sorted(set(sched))}
    q, k, v = make_qkv(base, rank_seed(rank), pad_fill=0.0, device=dev)
    out = torch.empty_like(q)

    def one_pass():
        for r in sched:
            run_step(bsa, attns[r], q, k, v, out, None)

    for _ in range(args.warmup):
        one_pass()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record()
        one_pass()
        b_.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b_))
    for attn in attns.values():
        attn.check_status()
    return max_over_ranks(statistics.median(times), world)


if __name__ == "__main__":
    main()
