"""Per-workload measurement report for the five synthetic workloads.

Usage (one GPU):  python -m long_context_misa_b200.report [--workloads NAME ...]
                  [--n-q N] [--no-dense] [--router-sweep]

--n-q N keeps the first N queries of each workload (smaller captures of the
same kernels for profilers); --no-dense skips the dense DSA calls.
--router-sweep instead reports, per workload, router aggregation
(misa_route_heads_agg) and routed head count h, the recall and IoU of MISA's
top-k against dense DSA's and the share of planted needles MISA selects.

For every workload of ``inputs.WORKLOADS`` at full size: the MISA call
(route + routed score + top-k; MISA-dagger through ``dagger_topk`` where the
workload has a k') and the dense DSA indexer, timed with CUDA events around
the calls (median of 5, L2 flushed before each), the token-scoring kernels' own
durations (routed with k' or k, and dense), the throughput in queries/s and
scored head*tokens/s, the fraction of the roofline the workload is bound by
(key bytes against the measured copy bandwidth for decode, useful tensor
flops against the measured bf16 peak for prefill) for the whole call and for
each scorer, and the recall and IoU of
MISA's final selection against the dense DSA selection (for MISA-dagger also
those of the routed pass alone cut to k).  Prints a markdown table.  The CPU
oracle's rate on the same workloads comes from the throughput script's
reference arm (``bench.py --impl reference --workload NAME``).
"""
from __future__ import annotations

import argparse
import json
import os

import numpy as np
import torch

from . import inputs as G
from . import misa as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


def _timed(fn, flush):
    ts = []
    for it in range(7):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        out = fn()
        b.record()
        torch.cuda.synchronize()
        if it >= 2:
            ts.append(a.elapsed_time(b))
    return float(np.median(ts)), out


def _scorer_ms(fn, flush):
    """Median duration of the token-scoring kernel inside fn(), read from the
    library's scoring event hook."""
    ts = []
    for it in range(7):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()  # creates the events; the library records them again around the kernel
        b.record()
        M.debug_time_scoring(a, b)
        flush()
        fn()
        torch.cuda.synchronize()
        M.debug_time_scoring(None, None)
        if it >= 2:
            ts.append(a.elapsed_time(b))
    return float(np.median(ts))


def overlap(sel, ref):
    """Mean recall |S & D| / |D| and mean IoU |S & D| / |S | D| over rows of two
    selections ([n][k] int arrays, -1 padded); rows with an empty D are skipped."""
    rec, iou = [], []
    for a, b in zip(sel, ref):
        sb = set(int(x) for x in b if x >= 0)
        sa = set(int(x) for x in a if x >= 0)
        if sb:
            rec.append(len(sa & sb) / len(sb))
            iou.append(len(sa & sb) / len(sa | sb))
    if not rec:
        return float("nan"), float("nan")
    return float(np.mean(rec)), float(np.mean(iou))


AGG_NAMES = {M.AGG_ABS_SUM: "|w| sum", M.AGG_SIGNED_SUM: "w sum", M.AGG_SUM: "sum", M.AGG_ABS_MAX: "|w| max"}


def router_sweep(names, dev):
    print("| workload | aggregation | h | recall / IoU vs dense | needles selected |")
    print("|---|---|---|---|---|")
    for name in names:
        wl = G.WORKLOADS[name]
        inp = G.make_inputs(wl, 0)
        cache, qs = M.device_inputs(inp, dev)
        M.pool_keys(cache)
        ws = M.Workspace(dev)
        dense = M.dense_score_topk(cache, qs, wl.k, ws=ws).cpu().numpy()
        for agg in AGG_NAMES:
            for h in (4, 8, 16):
                heads = M.route_heads(cache, qs, h, ws=ws, agg=agg)
                top = M.score_topk(cache, qs, heads, wl.k, ws=ws).cpu().numpy()
                hit = [p in set(top[qi].tolist()) for (_, p, qi) in inp.needles]
                rec, iou = overlap(top, dense)
                print(f"| {name} | {AGG_NAMES[agg]} | {h} | {rec:.3f} / {iou:.3f} | {sum(hit)} / {len(hit)} |",
                      flush=True)
        assert cache.device_status() == 0
        del cache, qs, ws
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", nargs="*", default=list(G.WORKLOADS))
    ap.add_argument("--n-q", type=int, default=0)
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--router-sweep", action="store_true")
    args = ap.parse_args()
    if args.router_sweep:
        router_sweep(args.workloads, torch.device("cuda"))
        return
    hbm, tflops, src = _peaks()
    dev = torch.device("cuda")
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush():
        flush_w.zero_()
        flush_r.sum()

    rows = []
    for name in args.workloads:
        wl = G.WORKLOADS[name]
        if args.n_q and wl.mode == "prefill":
            wl = wl.scaled(n_q=min(args.n_q, wl.n_q))
        inp = G.make_inputs(wl, 0)
        cache, qs = M.device_inputs(inp, dev)
        M.pool_keys(cache)
        ws = M.Workspace(dev)
        li = inp.q_pos.astype(np.int64) + 1
        M_i = -(-li // wl.B)

        def misa():
            heads = M.route_heads(cache, qs, wl.h, ws=ws)
            if wl.k_prime:
                return M.dagger_topk(cache, qs, heads, wl.k_prime, wl.k, ws=ws)
            return M.score_topk(cache, qs, heads, wl.k, ws=ws)

        def dense():
            if args.no_dense:
                return torch.full((wl.n_q, wl.k), -1, dtype=torch.int32, device=dev)
            return M.dense_score_topk(cache, qs, wl.k, ws=ws)

        for _ in range(2):
            misa()
            dense()
        torch.cuda.synchronize()
        t_misa, sel = _timed(misa, flush)
        t_dense, ref = _timed(dense, flush)
        heads = M.route_heads(cache, qs, wl.h, ws=ws)
        k_route = wl.k_prime or wl.k
        s_misa = _scorer_ms(lambda: M.score_topk(cache, qs, heads, k_route, ws=ws), flush)
        s_dense = float("nan") if args.no_dense else _scorer_ms(dense, flush)
        assert cache.device_status() == 0
        work = float((wl.h * li + wl.H * M_i + (wl.H * np.minimum(wl.k_prime, li) if wl.k_prime else 0)).sum())
        row_bytes = wl.d * (1 if wl.key_dtype == "fp8" else 2) + (4 if wl.key_dtype == "fp8" else 0)
        if wl.mode == "decode":
            key_bytes = float(li.sum()) * row_bytes
            q_bytes = wl.n_q * wl.d * 2.0
            call = key_bytes / (t_misa * 1e-3) / 1e9 / hbm
            sm = (key_bytes + q_bytes * wl.h) / (s_misa * 1e-3) / 1e9 / hbm
            sd = (key_bytes + q_bytes * wl.H) / (s_dense * 1e-3) / 1e9 / hbm
            bound = f"HBM: call {call:.2f}, routed scorer {sm:.2f}, dense scorer {sd:.2f}"
        else:
            flops = 2.0 * wl.d * (wl.h * float(li.sum()) + wl.H * float(M_i.sum()))
            call = flops / (t_misa * 1e-3) / 1e12 / tflops
            sm = 2.0 * wl.d * wl.h * float(li.sum()) / (s_misa * 1e-3) / 1e12 / tflops
            sd = 2.0 * wl.d * wl.H * float(li.sum()) / (s_dense * 1e-3) / 1e12 / tflops
            bound = f"tensor: call {call:.2f}, routed scorer {sm:.2f}, dense scorer {sd:.2f}"
        ref_np = ref.cpu().numpy()
        rec = "%.3f / %.3f" % overlap(sel.cpu().numpy(), ref_np)
        if wl.k_prime:  # the routed pass alone, cut to k
            plain = M.score_topk(cache, qs, M.route_heads(cache, qs, wl.h, ws=ws), wl.k, ws=ws)
            rec += " (routed only: %.3f / %.3f)" % overlap(plain.cpu().numpy(), ref_np)
        rows.append((name, wl.n_q, t_misa, t_dense, s_misa, s_dense, wl.n_q / (t_misa * 1e-3),
                     work / (t_misa * 1e-3), bound, rec))
        del cache, qs, ws
        torch.cuda.empty_cache()
        print(f"done {name}", flush=True)

    print(f"\npeaks: {hbm} GB/s, {tflops} TFLOP/s ({src})\n")
    print("| workload | queries | MISA call ms | dense DSA ms | routed / dense scorer ms | MISA queries/s | "
          "MISA head*tokens/s | of roofline | recall / IoU vs dense |")
    print("|---|---|---|---|---|---|---|---|---|")
    for name, nq, tm, td, sm, sd, qps, hts, bound, rec in rows:
        print(f"| {name} | {nq} | {tm:.3f} | {td:.3f} | {sm:.3f} / {sd:.3f} | {qps:.3e} | {hts:.3e} | {bound} | {rec} |")


if __name__ == "__main__":
    main()
