"""Benchmark of the B200 masked attention forward.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference] [--workload NAME]
python bench.py --split [--workload split_rightdown_32k] ...   (under torchrun for N > 1)

Prints ONE JSON line (rank 0). A step is one fa_fwd over the whole workload
(every KV tile of every (sequence, head, query block)). The metric counts
only visible (i, j) pairs: TFLOP/s = 4 * D * pairs / time.

Default workload: prefix_8k, B=4, N=16, Sq=Skv=8192, D=128, BNSD, sparseMode 5
(rightDownCausal plus the per-batch prefix [512, 1024, 2048, 4096]), bf16
N(0,1) inputs from seed 5: the largest of the causal, band and prefix
scenarios (1.19 TFLOP of visible work per call). With --gpus N > 1 (under
torchrun) every rank runs its own independent copy of the workload (the
work shards by (batch, head, query block) with no exchange), so the value
is the total over ranks divided by the slowest rank's time (weak scaling).

--split runs the sparseMode page's multi-card scheme instead (sparseMode=7/8
sections): the query tokens of one varlen rightDownCausal or leftUpCausal
job are cut into N parts that balance the visible pairs (fa_split_queries),
K/V stay whole, and rank r runs part r alone on its GPU: no collective in
the forward. The value is the whole job's visible-pair FLOPs over the
slowest rank's time (strong scaling: the job is fixed as N grows).

Timing: W untimed warm-up steps, then K steps each bracketed by CUDA events
on the launching stream; a 256 MiB buffer (larger than the 126 MB L2) is
written between steps, outside the events, so every step starts with a cold
L2. Barrier + synchronize on both sides of the timed region, max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "prefix_8k"
SPLIT_WORKLOAD = "split_rightdown_32k"
METRIC = "masked-attention fwd TFLOP/s (visible pairs) and % of B200 BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="budget of the oracle's bounded CPU sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", action="store_true",
                    help="run this rank's part of the query split of one varlen job")
    args = ap.parse_args()
    if args.split and args.workload == DEFAULT_WORKLOAD:
        args.workload = SPLIT_WORKLOAD
    return args


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload):
    """Per-launch DRAM bytes (read + write) of the workload's main kernel from
    the committed ncu summary; None when that kernel's source changed since
    the capture (the attention kernel's source unless the record names
    another)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        entry = rec.get(workload)
        if entry is None:
            return None
        name = entry.get("source", "fa_kernel_sm100.cu")
        want = entry.get("source_sha256", rec.get("kernel_source_sha256"))
        with open(os.path.join(ROOT, "masked_attention_fa_b200", "csrc", name), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    if sha != want:
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples (200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def workload_args(w):
    import numpy as np
    arrays = {}
    if w.prefix is not None:
        arrays["prefix"] = np.asarray(w.prefix, dtype=np.int64)
    if w.layout == "TND":
        arrays["actual_seq_qlen"] = np.asarray(w.actual_seq_qlen, dtype=np.int64)
        arrays["actual_seq_kvlen"] = np.asarray(w.actual_seq_kvlen, dtype=np.int64)
    return arrays


def kernel_label(w, dense, dev):
    """The attention kernel instance a call of the workload runs: dense-mask
    extras, and claimed work for closed-form lists of at least
    fa.CLAIM_MIN_ITEMS_PER_CTA items per SM."""
    import torch
    import masked_attention_fa_b200 as fa
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                     w.next_tokens, w.scale, w.mask_kind, w.alibi)
    items = fa.fa_plan_stats(d, has_mask=dense, **workload_args(w))[0]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    claim = (not dense) and items >= fa.CLAIM_MIN_ITEMS_PER_CTA * sms
    tf = lambda x: "true" if x else "false"
    return (f"fa_fwd_sm100<{w.D}, true, {tf(dense)}, {tf(claim)}, {tf(w.alibi is not None)}>")


def visible_pairs(w, has_mask, mask_host=None):
    """Visible pairs of the workload from the library's geometry (closed-form
    row intervals); dense-mask workloads count the mask on the host."""
    import masked_attention_fa_b200 as fa
    if has_mask:
        import numpy as np
        import torch
        vis = ~mask_host.to(torch.bool).numpy()
        if w.sparse_mode == 0:  # mode 0: the mask inside the preTokens/nextTokens band
            ii = np.arange(w.Sq)[:, None]
            jj = np.arange(w.Skv)[None, :]
            vis = vis & ((ii - jj <= w.pre_tokens) & (jj - ii <= w.next_tokens))
        # planes: SS one for every (b, h), B1SS one per b, BNSS one per (b, h)
        mult = {"SS": w.B * w.N, "B1SS": w.N, "BNSS": 1}[w.mask_kind]
        return int(vis.sum()) * mult
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                     w.next_tokens, w.scale, w.mask_kind)
    return fa.fa_visible_pairs(d, **workload_args(w))


def prepass_bytes(w):
    """Algorithmic bytes of the dense-mask pre-pass: every mask byte of the
    128 x 128 tiles inside the band (the geometry's non-EMPTY tiles, cut at
    Sq and Skv) is read once, per mask plane; plus one class byte per tile
    written and read again, and 16 bytes of range per 128-row query block."""
    import masked_attention_fa_b200 as fa
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                     w.next_tokens, w.scale, w.mask_kind)
    planes = {"SS": 1, "B1SS": w.B, "BNSS": w.B * w.N}[w.mask_kind]
    n_qt, n_kt = (w.Sq + 127) // 128, (w.Skv + 127) // 128
    per_plane = 0
    for qt in range(n_qt):
        rows = min(128, w.Sq - 128 * qt)
        for kt in range(n_kt):
            if fa.fa_tile_class(d, 0, qt, kt, has_mask=True) != fa.FA_TILE_EMPTY:
                per_plane += rows * min(128, w.Skv - 128 * kt)
    return planes * (per_plane + 2 * n_qt * n_kt + 16 * n_qt)


def paged_bytes(w):
    """Algorithmic bytes of a paged forward: every visible cached key and
    value row once per head (bf16), q and O (bf16) and lse (fp32). Each
    sequence's visible keys run from its first row's lowest to its last
    row's highest key; the paged workloads are rightDownCausal, whose last
    row sees every key."""
    assert w.sparse_mode == 3
    keys = sum(skv for _, skv in w.seq_lens())
    return 2 * keys * w.N * w.D * 2 + 2 * w.Sq * w.N * w.D * 2 + w.N * w.Sq * 4


def cpu_baseline_sample_paged(w, inputs, seconds):
    """The paged oracle on (sequence, head 0) problems, sequences in turn,
    each with its blocks of head 0 gathered to the host once."""
    import numpy as np
    import oracle
    from oracle import Problem
    lens = w.seq_lens()
    table = inputs["block_table"].cpu()
    cases = []
    for bi, (sq, skv) in enumerate(lens):
        nblk = -(-skv // w.block_size)
        blocks = table[bi, :nblk].long().to(inputs["k_cache"].device)
        q0 = int(w.actual_seq_qlen[bi - 1]) if bi else 0
        cases.append((sq, skv, nblk, inputs["q"][q0:q0 + sq, :1].cpu(),
                      inputs["k_cache"][blocks][:, :, :1].cpu(),
                      inputs["v_cache"][blocks][:, :, :1].cpu()))
    pairs, elapsed, done = 0, 0.0, 0
    while elapsed < seconds and done < 100000:
        sq, skv, nblk, q, kc, vc = cases[done % len(cases)]
        pb = Problem("TND", 1, 1, sq, skv, w.D, sparse_mode=w.sparse_mode, scale=w.scale,
                     actual_seq_qlen=[sq], actual_seq_kvlen=[skv])
        t0 = time.perf_counter()
        oracle.attention_paged(pb, q, kc, vc, np.arange(nblk, dtype=np.int32)[None], w.block_size)
        elapsed += time.perf_counter() - t0
        pairs += sq * skv
        done += 1
    tflops = 4.0 * w.D * pairs / elapsed / 1e12
    desc = (f"{done} (sequence, head 0) problems of {w.name}, sequences in turn, K/V blocks "
            f"gathered to the host; {pairs} visible pairs in {elapsed:.1f} s")
    return tflops, oracle.num_threads(), desc


def cpu_baseline_sample(w, inputs, seconds):
    if w.block_size is not None:
        return cpu_baseline_sample_paged(w, inputs, seconds)
    """Time the oracle (as it stands) on a bounded sample of query rows of the
    same workload; returns (TFLOP/s, cores, description)."""
    import numpy as np
    import oracle
    from oracle import Problem
    from masked_attention_fa_b200.workloads import alibi_slopes
    pb_kw = dict(layout=w.layout, B=w.B, N=w.N, Sq=w.Sq, Skv=w.Skv, D=w.D,
                 sparse_mode=w.sparse_mode, pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
                 scale=w.scale)
    # One (batch, head) slice, converted once; rows sampled evenly.
    b, h = 0, 0
    q, k, v = inputs["q"], inputs["k"], inputs["v"]
    if w.layout == "BNSD":
        qs, ks, vs = q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1]
        sub = dict(pb_kw, B=1, N=1)
    elif w.layout == "BSND":
        qs, ks, vs = q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1]
        sub = dict(pb_kw, B=1, N=1)
    else:
        qs, ks, vs = q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1]
        sub = dict(pb_kw, N=1, actual_seq_qlen=w.actual_seq_qlen,
                   actual_seq_kvlen=w.actual_seq_kvlen)
    if w.prefix is not None:
        sub["prefix"] = [w.prefix[b]] if w.layout != "TND" else w.prefix
    mask = inputs.get("mask")
    if mask is not None:
        sub["mask"] = mask.numpy()
        sub["mask_kind"] = w.mask_kind
    pb = Problem(**sub)
    qd, kd, vd = (oracle._f64(x.contiguous()) for x in (qs, ks, vs))
    nrows_total = w.Sq if w.layout != "TND" else w.actual_seq_qlen[0]
    row_pairs = oracle.mask_matrix(pb, 0).sum(axis=1, dtype=np.int64)
    done_rows, pairs, elapsed, chunk = 0, 0, 0.0, 64
    rng = np.random.default_rng(0)
    while elapsed < seconds and done_rows < 1_000_000:
        rows_i = rng.integers(0, nrows_total, size=chunk)
        rows = np.stack([np.zeros(chunk, np.int64), np.zeros(chunk, np.int64), rows_i], 1)
        t0 = time.perf_counter()
        if w.alibi is not None:
            oracle.attention_rows(pb, qd, kd, vd, rows, alibi=w.alibi,
                                  slopes=alibi_slopes(w.N)[h:h + 1])
        else:
            oracle.attention_rows(pb, qd, kd, vd, rows)
        elapsed += time.perf_counter() - t0
        pairs += int(row_pairs[rows_i].sum())
        done_rows += chunk
        chunk = min(chunk * 2, 4096)
    tflops = 4.0 * w.D * pairs / elapsed / 1e12
    desc = (f"{done_rows} query rows drawn uniformly from batch 0, head 0 of {w.name}; "
            f"{pairs} visible pairs in {elapsed:.1f} s")
    return tflops, oracle.num_threads(), desc


def bench_config(w, pairs, world):
    """The `config` object of the JSON line, the same for both arms."""
    paged = w.block_size is not None
    return {"workload": w.name, "layout": w.layout, "B": w.B, "N": w.N, "Sq": w.Sq,
            "Skv": w.Skv, "D": w.D, "sparse_mode": w.sparse_mode, "visible_pairs": int(pairs),
            "per_rank": "independent copy",
            "l2": "cold: a 256 MiB buffer is written between timed GPU steps",
            **({"block_size": w.block_size, "kv_cache": "paged, resident"} if paged else {}),
            **({"alibi": w.alibi, "slopes": "2^(-8 (h + 1) / N), resident"} if w.alibi else {}),
            "parallelism": f"replicas x{world}"}


def oracle_visible_pairs(w, mask_host=None):
    """Visible pairs of the workload counted from the oracle's explicit
    visibility matrices (one per sequence; per head only for a BNSS mask)."""
    import numpy as np
    import oracle
    from oracle import Problem
    kw = dict(layout=w.layout, B=w.B, N=w.N, Sq=w.Sq, Skv=w.Skv, D=w.D,
              sparse_mode=w.sparse_mode, pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
              scale=w.scale, prefix=w.prefix, actual_seq_qlen=w.actual_seq_qlen,
              actual_seq_kvlen=w.actual_seq_kvlen)
    if mask_host is not None:
        kw.update(mask=mask_host.numpy(), mask_kind=w.mask_kind)
    pb = Problem(**kw)
    total = 0
    for b in range(w.B):
        heads = range(w.N) if w.mask_kind == "BNSS" else [0]
        per = sum(int(oracle.mask_matrix(pb, b, h).sum(dtype=np.int64)) for h in heads)
        total += per if w.mask_kind == "BNSS" else per * w.N
    return total


# ------------------------------------------------------------ query split

def split_rank_part(w, world, rank):
    """Part `rank` of `world` of the query split of TND job w (the sparseMode
    page's multi-card scheme, fa_split_queries with cuts that balance the
    visible pairs): its descriptor, cumulative arrays and token ranges."""
    import masked_attention_fa_b200 as fa
    if w.layout != "TND" or w.sparse_mode not in (2, 3):
        raise ValueError("the query split takes a TND job in sparseMode 2 or 3")
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                     w.next_tokens, w.scale)
    return fa.fa_split_queries(d, w.actual_seq_qlen, w.actual_seq_kvlen, world, rank)


def split_part_inputs(inputs, part):
    """The part's own q rows and the key/value rows it reads (views)."""
    return {"q": inputs["q"][part["q_begin"]:part["q_end"]],
            "k": inputs["k"][part["kv_begin"]:part["kv_end"]],
            "v": inputs["v"][part["kv_begin"]:part["kv_end"]]}


def split_step(part, inp, forward):
    """One rank's forward of its part: forward(desc, q, k, v, cu_q, cu_kv)
    -> (o, lse); None for a part without query tokens (nothing to run)."""
    if part["q_end"] <= part["q_begin"]:
        return None
    return forward(part["desc"], inp["q"], inp["k"], inp["v"], part["actual_seq_qlen"],
                   part["actual_seq_kvlen"])


def run_split(args):
    import torch
    import torch.distributed as dist
    import masked_attention_fa_b200 as fa
    from masked_attention_fa_b200.workloads import named_workloads, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = named_workloads()[args.workload]
    part = split_rank_part(w, world, rank)
    inp = {x: t.to(dev) for x, t in split_part_inputs(make_inputs(w), part).items()}
    pd = part["desc"]
    attn = fa.MaskedAttention("TND", pd.B, pd.N, pd.Sq, pd.Skv, pd.D, pd.sparse_mode,
                              pd.pre_tokens, pd.next_tokens, pd.scale)
    oshape, lshape = attn.out_shapes()
    o = torch.empty(oshape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(lshape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def cuda_forward(desc, q, k, v, cu_q, cu_kv):
        return attn(q, k, v, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv, out=o, lse=lse,
                    stream=stream)

    for _ in range(max(args.warmup, 3)):
        split_step(part, inp, cuda_forward)
    torch.cuda.synchronize(dev)
    attn.sync_status()
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        split_step(part, inp, cuda_forward)
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    attn.sync_status()
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                     w.next_tokens, w.scale)
    pairs = fa.fa_visible_pairs(d, **workload_args(w))
    my_pairs = 0
    if part["q_end"] > part["q_begin"]:
        my_pairs = fa.fa_visible_pairs(pd, actual_seq_qlen=part["actual_seq_qlen"],
                                       actual_seq_kvlen=part["actual_seq_kvlen"])
    flops = 4.0 * w.D * pairs
    value = flops / (ms_max * 1e-3) / 1e12
    if rank == 0:
        peaks, peak_src = load_peaks()
        peak = float(peaks["bf16_tflops"])
        achieved = 4.0 * w.D * my_pairs / (ms * 1e-3) / 1e12
        cfg = bench_config(w, pairs, world)
        cfg["parallelism"] = f"query split x{world} (sparseMode=7/8 multi-card scheme)"
        cfg["per_rank"] = (f"part {rank}: query tokens [{part['q_begin']}, {part['q_end']}), "
                           f"keys [{part['kv_begin']}, {part['kv_end']}), sparse_mode "
                           f"{pd.sparse_mode}")
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic", "config": cfg,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                             "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                             "peak_source": f"{peak_src} bf16_tflops (burst)",
                             "kernel": "fa_fwd_sm100 (rank 0's part)", "kernel_ms": ms},
                "cpu_baseline": None, "e2e": None, "gpu_launches": args.steps,
                "clocks": clocks}
        print(json.dumps(line))
    attn.close()
    if world > 1:
        dist.destroy_process_group()


def run_reference(args):
    """The oracle on the host cores, as the reference arm."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from masked_attention_fa_b200.workloads import named_workloads, make_inputs
    import oracle
    w = named_workloads()[args.workload]
    if w.block_size is not None:
        # gigabytes of cache values: drawn by the GPU when there is one
        import torch
        inputs = make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    else:
        inputs = make_inputs(w)
    per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    vals = []
    desc = None
    cores = oracle.num_threads()
    for s in range(args.warmup + args.steps):
        tf, cores, desc = cpu_baseline_sample(w, inputs, per_step)
        if s >= args.warmup:
            vals.append(tf)
    value = statistics.median(vals)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if w.block_size is not None:
        pairs = sum(sq * skv for sq, skv in w.seq_lens()) * w.N  # decode rows see every key
    else:
        pairs = oracle_visible_pairs(w, inputs.get("mask"))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(w, pairs, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.split:
        run_split(args)
        return

    import torch
    import torch.distributed as dist
    import masked_attention_fa_b200 as fa
    from masked_attention_fa_b200.workloads import named_workloads, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    w = named_workloads()[args.workload]
    paged = w.block_size is not None
    if paged:  # caches drawn on the device (gigabytes; see workloads.paged_inputs)
        inputs = make_inputs(w, device=dev)
        q, kc, vc, table = (inputs[x] for x in ("q", "k_cache", "v_cache", "block_table"))
    else:
        inputs = make_inputs(w)
        q, k, v = (inputs[x].to(dev) for x in ("q", "k", "v"))
    mask = inputs["mask"].to(dev) if inputs["mask"] is not None else None
    arrays = workload_args(w)
    attn = fa.MaskedAttention(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                              w.next_tokens, w.scale, w.mask_kind, w.alibi)
    slopes = None
    if w.alibi is not None:  # per-head coefficients: parameters, resident on the device
        from masked_attention_fa_b200.workloads import alibi_slopes
        slopes = torch.tensor(alibi_slopes(w.N), dtype=torch.float32, device=dev)
    oshape, lshape = attn.out_shapes()
    o = torch.empty(oshape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(lshape, dtype=torch.float32, device=dev)
    pairs = visible_pairs(w, mask is not None, inputs["mask"])
    flops = 4.0 * w.D * pairs
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    # Dense-mask workloads: the step is the library's occupancy pre-pass
    # followed by the attention on its ranges (the same two stages fa_fwd
    # runs internally), with an event between them so each kernel is timed.
    dense = mask is not None
    if dense:
        cls_shape, rng_shape = fa.occupancy_shapes(attn.desc)
        tile_cls = torch.empty(cls_shape, dtype=torch.uint8, device=dev)
        ranges = torch.empty(rng_shape, dtype=torch.int32, device=dev)

    def prepass():
        fa.fa_mask_occupancy(attn.desc, mask, tile_class=tile_cls, ranges=ranges, stream=stream)

    def attention():
        if paged:
            attn.paged(q, kc, vc, table, w.actual_seq_qlen, w.actual_seq_kvlen, out=o, lse=lse,
                       stream=stream)
        elif dense:
            attn(q, k, v, atten_mask=mask, out=o, lse=lse, stream=stream, ranges=ranges)
        else:
            attn(q, k, v, atten_mask=mask, out=o, lse=lse, stream=stream, slopes=slopes,
                 **arrays)

    def step():
        if dense:
            prepass()
        attention()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    attn.sync_status()

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        if dense:
            prepass()
        mids[i].record(stream)
        attention()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    attn.sync_status()
    times_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = sum(times_ms) / len(times_ms)
    # the attention kernel alone (the whole step when there is no pre-pass)
    kern_ms = sum(m.elapsed_time(e) for m, e in zip(mids, ends)) / len(mids)
    pre_ms = sum(s.elapsed_time(m) for s, m in zip(starts, mids)) / len(mids)
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    value = world * flops / (ms_max * 1e-3) / 1e12

    # End to end through the public API with host buffers: every step copies
    # its inputs (q, k, v and, for a dense-mask workload, the mask) from
    # pinned host memory to the device, runs fa_fwd and copies O and lse back
    # to pinned host memory. Steps are pipelined the way a serving loop runs
    # them: device buffers are double-buffered, uploads run on one stream,
    # the forward on another and downloads on a third, so step i's upload
    # overlaps step i-1's forward and download (PCIe carries the two
    # directions at once). Events order the reuse of each buffer pair.
    e2e = None
    if not args.no_e2e:
        if paged:  # the caches are the state: resident; q and the block table go up
            host_in = [inputs["q"].cpu().pin_memory(), inputs["block_table"].cpu().pin_memory()]
        else:
            host_in = [inputs[x].pin_memory() for x in ("q", "k", "v")]
        if dense:
            host_in.append(inputs["mask"].pin_memory())
        dev_in = [[torch.empty_like(x, device=dev) for x in host_in] for _ in range(2)]
        dev_o = [torch.empty(oshape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        dev_l = [torch.empty(lshape, dtype=torch.float32, device=dev) for _ in range(2)]
        ho = [torch.empty(oshape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        hl = [torch.empty(lshape, dtype=torch.float32).pin_memory() for _ in range(2)]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_fwd = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            b = i % 2
            with torch.cuda.stream(up):
                if used[b]:
                    up.wait_event(ev_fwd[b])  # the forward of step i-2 has read these inputs
                for d, h in zip(dev_in[b], host_in):
                    d.copy_(h, non_blocking=True)
                ev_up[b].record(up)
            stream.wait_event(ev_up[b])
            if used[b]:
                stream.wait_event(ev_down[b])  # step i-2's outputs have left the device
            if paged:
                attn.paged(dev_in[b][0], kc, vc, dev_in[b][1], w.actual_seq_qlen,
                           w.actual_seq_kvlen, out=dev_o[b], lse=dev_l[b], stream=stream)
            else:
                qb, kb, vb = dev_in[b][:3]
                mb = dev_in[b][3] if dense else None
                attn(qb, kb, vb, atten_mask=mb, out=dev_o[b], lse=dev_l[b], stream=stream,
                     slopes=slopes, **arrays)
            ev_fwd[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_fwd[b])
                ho[b].copy_(dev_o[b], non_blocking=True)
                hl[b].copy_(dev_l[b], non_blocking=True)
                ev_down[b].record(down)
            used[b] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(4, min(args.steps, 10))
        torch.cuda.synchronize(dev)
        e0.record(up)
        for i in range(n_e2e):
            e2e_step(i)
        down.wait_event(ev_down[(n_e2e - 1) % 2])
        e1.record(down)
        torch.cuda.synchronize(dev)
        attn.sync_status()
        ems = e0.elapsed_time(e1) / n_e2e
        te = torch.tensor([ems], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e = {"value": world * flops / (float(te.item()) * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in host_in)),
               "d2h_bytes_per_step": int(ho[0].numel() * ho[0].element_size() +
                                         hl[0].numel() * hl[0].element_size()),
               "ms_per_step": float(te.item()), "steps": n_e2e,
               "pipeline": "2 buffer sets; upload, forward and download on 3 streams"}

    if rank == 0:
        peaks, peak_src = load_peaks()
        peak = float(peaks["bf16_tflops"])
        achieved = flops / (kern_ms * 1e-3) / 1e12
        traffic = load_traffic(w.name)
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                    "kernel": kernel_label(w, dense, dev),
                    "kernel_ms": kern_ms}
        if paged:
            # A few query rows per sequence: every cached K/V byte is used for a
            # handful of FMAs, so HBM bounds the path, not the tensor cores.
            nbytes = paged_bytes(w)
            gbs = nbytes / (kern_ms * 1e-3) / 1e9
            hbm = float(peaks["hbm_gbs"])
            roofline = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                        "frac": gbs / hbm, "traffic": traffic, "bytes_per_launch": nbytes,
                        "peak_source": f"{peak_src} hbm_gbs",
                        "kernel": f"paged_partial<{w.D}> + paged_merge<{w.D}>",
                        "kernel_ms": kern_ms, "tflops": achieved}
        if dense:
            roofline["kernel_ms_includes"] = ("the one-block work-list rebuild "
                                              "(occupancy_schedule) launched just before it")
        prepass_line = None
        if dense:
            mbytes = prepass_bytes(w)
            gbs = mbytes / (pre_ms * 1e-3) / 1e9
            hbm = float(peaks["hbm_gbs"])
            prepass_line = {"kernels": "occupancy_strips", "ms": pre_ms,
                            "bound": "hbm", "bytes": mbytes, "achieved": gbs, "peak": hbm,
                            "unit": "GB/s", "frac": gbs / hbm,
                            "peak_source": f"{peak_src} hbm_gbs"}
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            tf, cores, desc = cpu_baseline_sample(w, inputs, args.cpu_seconds)
            cpu = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                   "sample": desc}
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": bench_config(w, pairs, world),
                "frac_of_peak": value / world / peak,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                # per step: the pre-pass, the work-list rebuild and the attention
                # (dense mask); the partial and merge kernels (paged); else one
                "gpu_launches": args.steps * (3 if dense else (2 if paged else 1)),
                "clocks": clocks,
                "ms_min": min(times_ms), "ms_median": statistics.median(times_ms)}
        if prepass_line is not None:
            line["prepass"] = prepass_line
        print(json.dumps(line))
    attn.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
