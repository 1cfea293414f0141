"""Per-cycle trace of one CTA of the attention kernel (a measurement tool).

    python -m masked_attention_fa_b200.trace --workload prefix_8k [--cta 0] [--out FILE.npz]
    python -m masked_attention_fa_b200.trace --exp-probe

Builds a second copy of the library with -DFA_TRACE=<cta> (in
masked_attention_fa_b200/_trace/, separate from the library itself, whose
kernel has no trace code; one copy per traced CTA), runs the named workload three times, then once
more with the traced CTA's clock64 stamps recorded, and prints:

  - per softmax warpgroup and key tile, the median cycles of each phase:
    waiting for S, loading S (with the mask on boundary tiles), the row
    maximum, waiting for the exponential-unit turn, the exponentials, waiting
    for the previous PV, storing P; and the period between turns;
  - per softmax warp, the exponential phase and the turn hand-over (from the
    last exponential of one warpgroup to the first of the other);
  - the MMA issuers' waits for K/V, for S to be read and for P, and the TMA
    thread's waits for a free ring slot;
  - per softmax warpgroup, the item boundary: reading the next item's
    records and ranges, and handing the finished item's 1/l and lse over;
  - the traced CTA's item starts and its span.

Stamps are clock64 of the SM running the CTA; with --out the raw arrays are
saved. Only this tool and the trace build read them.

--exp-probe builds and runs probe/exp_loop.cu: cycles per 128-key row of the
softmax's exponential loop and of variants of it, one or two warps per SM
sub-partition.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import subprocess
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
TRACE_DIR = os.path.join(HERE, "_trace")
N_TRACE = 1024


def build_trace(cta: int) -> str:
    """Compile the library's sources with -DFA_TRACE=<cta>; returns the path."""
    from masked_attention_fa_b200 import build as b
    os.makedirs(TRACE_DIR, exist_ok=True)
    lib = os.path.join(TRACE_DIR, f"libfa_b200_trace{int(cta)}.so")
    newest = max(os.path.getmtime(f) for f in b._inputs())
    if os.path.exists(lib) and os.path.getmtime(lib) > newest:
        return lib
    cmd = [b.nvcc()] + b.NVCC_FLAGS + [f"-DFA_TRACE={int(cta)}",
                                        "-I" + os.path.join(ROOT, "include"), "-o", lib] + b.sources()
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building the trace library")
    return lib


def record(workload: str, cta: int):
    """Run `workload` on the trace library; returns (tiles, warps) stamp
    arrays [8, 8, N] and [8, 4, N] (0 = not stamped)."""
    import torch
    import masked_attention_fa_b200 as fa
    fa.LIB_PATH = build_trace(cta)
    lib = fa.load_library()
    lib.fa_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    sys.path.insert(0, ROOT)
    import bench
    from masked_attention_fa_b200.workloads import alibi_slopes, make_inputs, named_workloads
    w = named_workloads()[workload]
    inp = make_inputs(w)
    q, k, v = (inp[x].cuda() for x in ("q", "k", "v"))
    arrays = bench.workload_args(w)
    if inp["mask"] is not None:
        arrays["atten_mask"] = inp["mask"].cuda()
    attn = fa.MaskedAttention(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                              w.next_tokens, w.scale, w.mask_kind, w.alibi)
    slopes = torch.tensor(alibi_slopes(w.N), device="cuda") if w.alibi else None
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    o, l = attn(q, k, v, slopes=slopes, **arrays)
    for _ in range(3):
        attn(q, k, v, out=o, lse=l, slopes=slopes, **arrays)
    torch.cuda.synchronize()
    if lib.fa_trace_cta() != int(cta) or lib.fa_trace_clear() != 0:
        raise RuntimeError("trace set-up failed")
    flush.fill_(1.0)  # cold L2, as in the bench
    torch.cuda.synchronize()
    attn(q, k, v, out=o, lse=l, slopes=slopes, **arrays)
    torch.cuda.synchronize()
    attn.sync_status()
    tiles = np.zeros((8, 8, N_TRACE), dtype=np.uint64)
    warps = np.zeros((8, 4, N_TRACE), dtype=np.uint64)
    if lib.fa_trace_read(tiles.ctypes.data, warps.ctypes.data) != 0:
        raise RuntimeError("trace read failed")
    attn.close()
    return tiles.astype(np.int64), warps.astype(np.int64)


def _med(a):
    return int(np.median(a)) if len(a) else -1


def summarize(tiles, warps) -> str:
    """The tables described in the module docstring, as text."""
    out = []
    t0 = tiles[tiles > 0].min()
    names = {1: "S wait", 2: "S load+mask", 3: "row max", 4: "turn wait", 5: "exponentials",
             6: "PV wait", 7: "P store"}
    # Events in the order they occur: 0 S wait, 1 S ready, 2 S loaded, 3 row
    # maximum, then either 4 turn, 5 exponentials done, 6 previous PV done,
    # 7 P handed over, or (P stored inside the exponential loop) 6 before 4.
    e0 = tiles[0]
    both = np.nonzero((e0[4] > 0) & (e0[6] > 0))[0]
    pv_first = len(both) > 0 and np.median(e0[6, both] - e0[4, both]) < 0
    order = [0, 1, 2, 3, 6, 4, 5, 7] if pv_first else list(range(8))
    if pv_first:
        names.update({6: "PV wait", 4: "turn wait", 5: "exponentials + P store", 7: "P hand-over"})
    out.append("| warpgroup | tiles | " + " | ".join(names[k] for k in order[1:]) +
               " | turn period |")
    out.append("|---" * (len(order) + 2) + "|")
    for s in (0, 1):
        e = tiles[s]
        idx = np.nonzero((e[0] > 0) & (e[7] > 0))[0]
        d = np.diff(e[order][:, idx], axis=0)
        per = np.diff(e[4, idx])
        out.append(f"| {s} | {len(idx)} | " + " | ".join(str(_med(d[i])) for i in range(7))
                   + f" | {_med(per)} |")
    ok = np.nonzero((warps[:, 0] > 0).all(0) & (warps[:, 1] > 0).all(0))[0]
    if len(ok):
        ex = warps[:, 1, ok] - warps[:, 0, ok]
        out.append("")
        out.append("exponential phase per softmax warp (median cycles): "
                   + ", ".join(f"w{i} {_med(ex[i])}" for i in range(8)))
        e0, e1 = warps[0:4, 1, ok], warps[4:8, 1, ok]
        s0, s1 = warps[0:4, 0, ok], warps[4:8, 0, ok]
        idx = {t: i for i, t in enumerate(ok)}
        h01 = s1.min(0) - e0.max(0)
        h10 = [s0[:, idx[t + 1]].min() - e1[:, idx[t]].max() for t in ok if t + 1 in idx]
        out.append(f"hand-over, last exponential of one warpgroup to the first of the other "
                   f"(median): 0->1 {_med(h01)}, 1->0 {_med(h10)}; end skew inside a "
                   f"warpgroup {_med(e0.max(0) - e0.min(0))} / {_med(e1.max(0) - e1.min(0))}")
    g = tiles[2]
    first = np.where(g[2] > 0, g[2], g[3])
    m = (g[0] > 0) & (first > 0)
    out.append("")
    out.append(f"QK issuer: K wait median {_med((first - g[0])[m])}; S-read wait before QK0 "
               f"{_med((g[4] - g[2])[(g[2] > 0) & (g[4] > 0)])}, before QK1 "
               f"{_med((g[5] - g[3])[(g[3] > 0) & (g[5] > 0)])}")
    pv = tiles[3]
    first = np.where(pv[2] > 0, pv[2], pv[3])
    m = (pv[0] > 0) & (first > 0)
    out.append(f"PV issuer: V wait median {_med((first - pv[0])[m])}; P wait before PV0 "
               f"{_med((pv[4] - pv[2])[(pv[2] > 0) & (pv[4] > 0)])}, before PV1 "
               f"{_med((pv[5] - pv[3])[(pv[3] > 0) & (pv[5] > 0)])}")
    tma = tiles[6]
    m = (tma[0] > 0) & (tma[1] > 0)
    out.append(f"TMA thread: free-slot wait median {_med((tma[1] - tma[0])[m])} over {m.sum()} "
               f"loads")
    out.append("")
    out.append("item boundary per softmax warpgroup (median cycles over the items after the "
               "first): index -> item record -> sequence record -> tile ranges -> row set-up; "
               "last turn -> 1/l slot free -> lse stored -> next index")
    for s, r in ((0, 5), (1, 7)):
        e = tiles[r]
        ks = [k for k in np.nonzero(e[0] > 0)[0] if k > 0]
        seg = [_med([e[j + 1, k] - e[j, k] for k in ks if e[j + 1, k] > 0]) for j in range(4)]
        end = [_med([e[j + 1, k] - e[j, k] for k in ks if e[j, k] > 0 and e[j + 1, k] > 0])
               for j in (5, 6)]
        nxt = _med([e[0, k] - e[7, k - 1] for k in ks if e[7, k - 1] > 0])
        out.append(f"  warpgroup {s}: {seg[0]} / {seg[1]} / {seg[2]} / {seg[3]}; "
                   f"{end[0]} / {end[1]} / {nxt}")
    starts = tiles[5, 0][tiles[5, 0] > 0] - t0
    out.append(f"items {len(starts)}, starts (cycles from the CTA's first stamp) "
               f"{[int(x) for x in starts[:8]]}{' ...' if len(starts) > 8 else ''}; span "
               f"{int(tiles.max() - t0)} cycles")
    return "\n".join(out)


def exp_probe() -> str:
    """Build and run the exponential-loop probe; returns its table."""
    from masked_attention_fa_b200 import build as b
    os.makedirs(TRACE_DIR, exist_ok=True)
    exe = os.path.join(TRACE_DIR, "exp_loop")
    src = os.path.join(HERE, "probe", "exp_loop.cu")
    res = subprocess.run([b.nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                          "-std=c++17", "-o", exe, src], capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stderr)
        raise RuntimeError("nvcc failed building the probe")
    return subprocess.run([exe], capture_output=True, text=True, check=True).stdout


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="prefix_8k")
    ap.add_argument("--cta", type=int, default=0)
    ap.add_argument("--out", default=None, help="save the raw stamps (.npz)")
    ap.add_argument("--exp-probe", action="store_true")
    args = ap.parse_args()
    if args.exp_probe:
        print(exp_probe())
        return
    tiles, warps = record(args.workload, args.cta)
    if args.out:
        np.savez(args.out, tiles=tiles, warps=warps)
    print(f"## {args.workload}, CTA {args.cta}\n")
    print(summarize(tiles, warps))


if __name__ == "__main__":
    main()
