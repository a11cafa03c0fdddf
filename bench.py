#!/usr/bin/env python
"""Benchmark of the DashAttention forward path on B200.

One step = the whole prefill hot path over one batch: stage 0 (chunk
summaries), stage 1 (entmax routing + mask), stage 2 (block-sparse
attention), through the C ABI.  Default workload: prefill, bf16, batch 1,
GQA 32/2, head_dim 128, seq 32768, chunk 64.  The same line also carries the
128k prefill and the 128k-cache decode measurements (``also``).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own copy of the workload (the
path shards over independent sequences/KV groups with no exchange), the
step time is the max over ranks and ``value`` counts the tokens of all
ranks (weak scaling).  ``--impl reference`` times the fp64 CPU oracle on a
bounded sample of the same workload (rank 0 only).

Timing: CUDA events on the launching stream; L2 is flushed (a 256 MiB
write) before every timed step and the flush is outside the timed span.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_hierarchical_attention_chunk_b200 import configs, shard, synth  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------
def popcount32(x):
    """Per-element popcount of an int32 tensor (as int64)."""
    x = x.to(torch.int64) & 0xFFFFFFFF
    x = x - ((x >> 1) & 0x55555555)
    x = (x & 0x33333333) + ((x >> 2) & 0x33333333)
    x = (x + (x >> 4)) & 0x0F0F0F0F
    return (x * 0x01010101 & 0xFFFFFFFF) >> 24


def prefill_work(wl, mask):
    """Algorithmic stage-2 FLOPs (active keys per row), tile-executed FLOPs, sparsity."""
    n, B, d, G = wl.seq, wl.chunk, wl.head_dim, wl.group
    act = popcount32(mask).sum(-1)                                  # [b, h_kv, N] routed blocks
    i = torch.arange(n, device=mask.device)
    keys = act * B + (i % B + 1)
    flops = 4.0 * d * G * keys.sum().item()
    P = 128 // G
    tiles = mask.view(wl.batch, wl.n_kv_heads, n // P, P, -1)
    union = tiles[..., 0, :].clone()
    for p in range(1, P):
        union |= tiles[..., p, :]
    nb = popcount32(union).sum(-1) + 1                              # + diagonal block
    exec_flops = 4.0 * d * 128 * B * nb.sum().item()
    elig = (i // B).clamp(min=1)
    frac = (act.double() / elig.double())[..., B:]
    per_head = frac.mean(dim=(0, 2)).tolist()
    return flops, exec_flops, frac.mean().item(), per_head


def stage_bytes(wl, mask, packed=False):
    """Algorithmic HBM bytes of stage 0 (K read, summaries written) and stage 1
    (Q and summaries read, weights and mask written: the dense row of w, or
    with the compact form only the routed entries)."""
    b, hq, hkv, n, d, B = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.seq, wl.head_dim, wl.chunk
    es = 2 if wl.dtype == "bf16" else 4
    n_c = wl.n_chunks
    kbar = b * hkv * (n // B) * d * es
    s0 = b * hkv * n * d * es + kbar
    nw = (n_c + 31) // 32
    routed = popcount32(mask).sum().item()
    w_bytes = routed * 4 if packed else b * hkv * n * n_c * 4
    s1 = b * hq * n * d * es + kbar + w_bytes + b * hkv * n * nw * 4
    return {"summarize": int(s0), "route": int(s1)}


def decode_bytes(wl, mask, lens=None):
    """Algorithmic HBM bytes of one decode step (lens: per-sequence cache
    lengths, else wl.seq for all)."""
    b, hq, hkv, d, B = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.chunk
    Ls = [wl.seq] * b if lens is None else [int(x) for x in lens.tolist()]
    c_qs = [(L - 1) // B for L in Ls]
    n_c = wl.n_chunks
    act = popcount32(mask).sum(-1).double().cpu()                   # [b, h_kv]
    kv_blocks = act.sum().item()
    diag_keys = sum(L - c * B for L, c in zip(Ls, c_qs)) * hkv
    kv = (kv_blocks * B + diag_keys) * d * 2 * 2
    kbar = sum(c_qs) * hkv * d * 2
    qo = 2 * b * hq * d * 2
    wm = b * hkv * (n_c * 4 + ((n_c + 31) // 32) * 4)
    elig = torch.tensor([max(c, 1) for c in c_qs], dtype=torch.float64)[:, None]
    frac = (act / elig).mean().item()
    return int(kv + kbar + qo + wm), frac


def profile_traffic(tag, workload, src):
    """DRAM bytes (read + write) per launch from the committed ncu summary.

    The summary records a hash of the kernel source it was taken on; when
    the source has changed since, the counters no longer describe the
    kernel and None is returned.  Several kernels in one summary are summed.
    """
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{tag}_{workload}.txt")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    cur = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
    if f"sha256[:16] {cur}" not in text:
        return None
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    total = 0.0
    for line in text.splitlines():
        parts = line.split()
        if len(parts) == 4 and parts[0] == "DRAM" and parts[1] in ("read", "write"):
            total += float(parts[2]) * scale[parts[3]]
    return int(total)


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, device):
    from sparse_hierarchical_attention_chunk_b200 import dash

    peaks, peaks_src = load_peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    barrier = shard.barrier

    def max_over_ranks(x):
        return shard.max_over_ranks(x, device)

    def time_prefill(wl, steps, warmup, sigma=None, want_clocks=False, packed=False,
                     keep_routing=False):
        inp = synth.make_prefill(wl, seed=rank, device=device)
        p = dash.problem_for(wl, sigma=sigma)
        Q, K, V, qbar = inp["Q"], inp["K"], inp["V"], inp["qbar"]
        out = dash.alloc_prefill(p, device)
        for _ in range(warmup):
            dash.prefill(p, Q, K, V, qbar, out=out, with_lse=False, packed=packed)
        torch.cuda.synchronize()
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(torch.cuda.current_device()) if want_clocks else None
        if sampler:
            sampler.__enter__()
        for e0, es, ea, e1 in evs:
            flush.fill_(1)
            e0.record(stream)
            dash.dash_summarize(p, K, qbar, out["Kbar"])
            es.record(stream)
            if packed:
                dash.dash_route_packed(p, Q, out["Kbar"], out["mask"], out["w"])
            else:
                dash.dash_route(p, Q, out["Kbar"], out["w"], out["mask"])
            ea.record(stream)
            if packed:
                dash.dash_attn_fwd_packed(p, Q, K, V, out["w"], out["mask"], out["O"])
            else:
                dash.dash_attn_fwd(p, Q, K, V, out["w"], out["mask"], out["O"])
            e1.record(stream)
        torch.cuda.synchronize()
        if sampler:
            sampler.__exit__()
        barrier()
        step_ms = [e0.elapsed_time(e1) for e0, es, ea, e1 in evs]
        sum_ms = [e0.elapsed_time(es) for e0, es, ea, e1 in evs]
        route_ms = [es.elapsed_time(ea) for e0, es, ea, e1 in evs]
        attn_ms = [ea.elapsed_time(e1) for e0, es, ea, e1 in evs]
        clocks = sampler.summary() if sampler else None
        flops, exec_flops, frac, per_head = prefill_work(wl, out["mask"])
        assert dash.dash_get_error() == dash.DASH_OK
        res = {"step_ms": max_over_ranks(statistics.mean(step_ms)),
               "attn_ms": max_over_ranks(statistics.mean(attn_ms)),
               "sum_ms": max_over_ranks(statistics.mean(sum_ms)),
               "route_ms": max_over_ranks(statistics.mean(route_ms)),
               "flops": flops, "exec_flops": exec_flops, "support": frac, "per_head": per_head,
               "clocks": clocks, "inputs": (Q, K, V, qbar), "p": p,
               "stage_bytes": stage_bytes(wl, out["mask"], packed)}
        if keep_routing:
            res["routing"] = {k: out[k].cpu() for k in ("Kbar", "w", "mask")}
            res["routing"]["Q"] = Q.cpu()          # the very inputs the kernels read
        del out
        return res

    def stage_rooflines(res):
        """Achieved GB/s of stages 0 and 1 against the HBM peak."""
        out = {}
        for name, key in (("summarize", "sum_ms"), ("route", "route_ms")):
            nb = res["stage_bytes"][name]
            gbs = nb / (res[key] / 1e3) / 1e9
            out[name] = {"ms": round(res[key], 4), "algorithmic_bytes": nb,
                         "achieved_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        return out

    def time_topk_ablation(wl, steps, warmup):
        """Stage 2 on a fixed-budget top-k mask (the NSA / InfLLMv2-style
        baseline, dash_route_topk) against the alpha-entmax mask of the same
        inputs, with the same kernel and sigma = 0 for both; k = the entmax
        mask's mean number of routed chunks per row, so both spend the same
        total budget."""
        inp = synth.make_prefill(wl, seed=rank, device=device)
        Q, K, V, qbar = inp["Q"], inp["K"], inp["V"], inp["qbar"]
        p0 = dash.problem_for(wl, sigma=0.0)
        out = dash.alloc_prefill(p0, device)
        dash.dash_summarize(p0, K, qbar, out["Kbar"])
        dash.dash_route(p0, Q, out["Kbar"], out["w"], out["mask"])
        cnt = popcount32(out["mask"]).sum(-1)                      # [b, h_kv, N]
        has = torch.arange(wl.seq, device=device) >= wl.chunk
        k = max(1, int(round(cnt[..., has].double().mean().item())))
        tw, tm = torch.empty_like(out["w"]), torch.empty_like(out["mask"])

        def timed(fn):
            for _ in range(max(warmup, 3)):
                fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(steps):
                flush.fill_(1)
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b_.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b_))
            return max_over_ranks(statistics.mean(ts))

        route_ms = timed(lambda: dash.dash_route_topk(p0, Q, out["Kbar"], k, tw, tm))
        attn_entmax = timed(lambda: dash.dash_attn_fwd(p0, Q, K, V, out["w"], out["mask"], out["O"]))
        attn_topk = timed(lambda: dash.dash_attn_fwd(p0, Q, K, V, tw, tm, out["O"]))
        assert dash.dash_get_error() == dash.DASH_OK
        fe, xe, sup_e, _ = prefill_work(wl, out["mask"])
        ft, xt, sup_t, _ = prefill_work(wl, tm)
        entry = {"workload": wl.name, "ablation": "fixed-budget top-k routing vs alpha-entmax routing, "
                                                   "same summaries and stage-2 kernel, sigma = 0",
                 "k": k, "route_topk_ms": round(route_ms, 4),
                 "attn_ms": {"entmax": round(attn_entmax, 4), "topk": round(attn_topk, 4)},
                 "algorithmic_flops": {"entmax": fe, "topk": ft},
                 "tile_executed_flops": {"entmax": xe, "topk": xt},
                 "support_mean": {"entmax": round(sup_e, 4), "topk": round(sup_t, 4)},
                 "note": "dash_route_topk is a CUDA-core reference kernel, not a tuned router"}
        del out, tw, tm, inp
        torch.cuda.empty_cache()
        return entry

    def time_attn_bwd(wl, steps, warmup):
        """Stage-2 backward (dash_attn_bwd: the tcgen05 dQ / dw and dK / dV
        kernels) beside the forward stage 2 on the same routing."""
        inp = synth.make_prefill(wl, seed=rank, device=device)
        Q, K, V, qbar = inp["Q"], inp["K"], inp["V"], inp["qbar"]
        p = dash.problem_for(wl)
        out = dash.prefill(p, Q, K, V, qbar)
        dO = torch.randn_like(Q)
        f32 = dict(dtype=torch.float32, device=device)
        dQ, dK, dV = torch.empty(Q.shape, **f32), torch.empty(K.shape, **f32), torch.empty(V.shape, **f32)
        dw = torch.empty(out["w"].shape, **f32)

        def timed(fn):
            for _ in range(max(warmup, 3)):
                fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(steps):
                flush.fill_(1)
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b_.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b_))
            return max_over_ranks(statistics.mean(ts))

        fwd = timed(lambda: dash.dash_attn_fwd(p, Q, K, V, out["w"], out["mask"], out["O"], out["lse"]))
        bwd = timed(lambda: dash.dash_attn_bwd(p, Q, K, V, out["w"], out["mask"], out["O"], out["lse"],
                                               dO, dQ, dK, dV, dw))
        dKbar = torch.zeros(out["Kbar"].shape, **f32)
        dqbar = torch.zeros(qbar.shape, **f32)
        rbwd = timed(lambda: dash.dash_route_bwd(p, Q, out["Kbar"], dw, dQ, dKbar))
        sbwd = timed(lambda: dash.dash_summarize_bwd(p, K, qbar, dKbar, dK, dqbar))
        assert dash.dash_get_error() == dash.DASH_OK
        flops, _, _, _ = prefill_work(wl, out["mask"])
        entry = {"workload": wl.name, "backward": "stage 2 (dash_attn_bwd: dQ, dK, dV, dw); stage 1 "
                                                  "(dash_route_bwd) and stage 0 (dash_summarize_bwd)",
                 "bwd_ms": round(bwd, 3), "fwd_attn_ms": round(fwd, 3),
                 "route_bwd_ms": round(rbwd, 3), "summarize_bwd_ms": round(sbwd, 3),
                 "algorithmic_flops_bwd": 2.5 * flops,
                 "achieved_tflops": round(2.5 * flops / (bwd / 1e3) / 1e12, 2),
                 "bwd_over_fwd": round(bwd / fwd, 2),
                 "note": "tcgen05 kernels, each output element written once (no atomics); "
                         "backward FLOPs counted as 2.5x the forward's (S recomputed, dP, dQ, dK, dV)"}
        del out, inp, dQ, dK, dV, dw, dO, dKbar, dqbar
        torch.cuda.empty_cache()
        return entry

    def time_decode(wl, steps, warmup, want_clocks=False):
        """One decode step (one new token for every sequence) through dash_decode."""
        inp = synth.make_decode(wl, seed=rank, device=device)
        lens = inp.get("lens")                      # per-sequence lengths, or None
        p5 = dash.problem_for(wl)
        kb = torch.empty(wl.batch, wl.n_kv_heads, wl.seq // wl.chunk, wl.head_dim,
                         dtype=torch.bfloat16, device=device)
        dash.dash_summarize(p5, inp["K"], inp["qbar"], kb)
        table = None
        if wl.paged:
            # the caches as a shuffled pool of one-chunk pages (plus 64 unused ones)
            Kpool, Vpool, table = synth.to_pages(inp["K"], inp["V"], lens.tolist(), wl.chunk,
                                                 seed=rank, extra_pages=64)
            inp["K"], inp["V"] = Kpool, Vpool
            del Kpool, Vpool
            torch.cuda.empty_cache()
        dout = dash.alloc_decode(p5, device)
        for _ in range(max(warmup, 3)):
            dash.decode(p5, inp["q"], inp["K"], inp["V"], kb, out=dout, cache_lens=lens,
                            page_table=table)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        barrier()
        sampler = ClockSampler(torch.cuda.current_device()) if want_clocks else None
        if sampler:
            sampler.__enter__()
        for a, b_ in evs:
            flush.fill_(1)
            a.record(stream)
            dash.decode(p5, inp["q"], inp["K"], inp["V"], kb, out=dout, cache_lens=lens,
                            page_table=table)
            b_.record(stream)
        torch.cuda.synchronize()
        us_eager = statistics.median([a.elapsed_time(b_) * 1e3 for a, b_ in evs])
        # the same step replayed from a CUDA graph, as a serving loop issues it
        graph_err = None
        try:
            cs = torch.cuda.Stream()
            cs.wait_stream(stream)
            with torch.cuda.stream(cs):
                dash.decode(p5, inp["q"], inp["K"], inp["V"], kb, out=dout, cache_lens=lens,
                            page_table=table)
            stream.wait_stream(cs)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                dash.decode(p5, inp["q"], inp["K"], inp["V"], kb, out=dout, cache_lens=lens,
                            page_table=table)
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            for a, b_ in evs:
                flush.fill_(1)
                a.record(stream)
                g.replay()
                b_.record(stream)
            torch.cuda.synchronize()
            us_graph = statistics.median([a.elapsed_time(b_) * 1e3 for a, b_ in evs])
            del g
        except Exception as exc:                     # reported, never hidden
            graph_err = f"{type(exc).__name__}: {exc}"[:200]
            us_graph = None
        if sampler:
            sampler.__exit__()
        assert dash.dash_get_error() == dash.DASH_OK
        us = max_over_ranks(us_graph if us_graph is not None else us_eager)
        us_eager = max_over_ranks(us_eager)
        nbytes, dfrac = decode_bytes(wl, dout["mask"], lens)
        gbs = nbytes / (us * 1e-6) / 1e9
        # end to end: the step's new queries go up, its outputs come back;
        # the KV and summary caches stay resident as in serving
        hq = inp["q"].cpu().pin_memory()
        ho = torch.empty(dout["o"].shape, dtype=dout["o"].dtype).pin_memory()
        dq = torch.empty_like(inp["q"])
        # a varlen step also uploads the sequences' current lengths
        hl = lens.cpu().pin_memory() if lens is not None else None
        dl = torch.empty_like(lens) if lens is not None else None
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            dq.copy_(hq, non_blocking=True)
            if lens is not None:
                dl.copy_(hl, non_blocking=True)
            dash.decode(p5, dq, inp["K"], inp["V"], kb, out=dout, cache_lens=dl, page_table=table)
            ho.copy_(dout["o"], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_us = max_over_ranks(e0.elapsed_time(e1) * 1e3 / steps)
        assert dash.dash_get_error() == dash.DASH_OK
        entry = {"workload": wl.name, "metric": "decode us/step (1 token per sequence)",
                 "us_per_step": round(us, 2), "us_per_token_aggregate": round(us / wl.batch, 3),
                 "roofline": {"bound": "hbm", "scope": "whole dash_decode call (3 kernels: routing, split-KV, merge of partials)",
                              "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": round(gbs / peaks["hbm_gbs"], 4),
                              "peak_source": f"{peaks_src} copy bandwidth",
                              "algorithmic_bytes": nbytes,
                              "traffic": profile_traffic(
                                  "decode", wl.name,
                                  "sparse_hierarchical_attention_chunk_b200/csrc/decode.cuh")},
                 "support_mean": round(dfrac, 4),
                 "launch": "cuda graph replay" if graph_err is None else "eager",
                 "eager_us_per_step": round(us_eager, 2)}
        if graph_err:
            entry["graph_error"] = graph_err
        if lens is not None:
            entry["cache_lens"] = [int(x) for x in lens.tolist()]
            # the summary-cache append of a step in which every sequence completes a chunk
            al = ((lens // wl.chunk).clamp(min=1) * wl.chunk).to(torch.int32)
            for _ in range(3):
                dash.dash_summarize_append(p5, al, inp["K"], inp["qbar"], kb, page_table=table)
            torch.cuda.synchronize()
            for a, b_ in evs:
                flush.fill_(1)
                a.record(stream)
                dash.dash_summarize_append(p5, al, inp["K"], inp["qbar"], kb, page_table=table)
                b_.record(stream)
            torch.cuda.synchronize()
            assert dash.dash_get_error() == dash.DASH_OK
            entry["summary_append_us"] = round(max_over_ranks(
                statistics.median([a.elapsed_time(b_) * 1e3 for a, b_ in evs])), 2)
        e2e = {"value": round(e2e_us, 2), "unit": "us/step",
               "h2d_bytes_per_step": hq.numel() * hq.element_size() +
                                     (hl.numel() * hl.element_size() if hl is not None else 0),
               "d2h_bytes_per_step": ho.numel() * ho.element_size()}
        res = {"us": us, "entry": entry, "e2e": e2e,
               "clocks": sampler.summary() if sampler else None}
        del inp, dout, kb
        torch.cuda.empty_cache()
        return res

    # ------------------------------------------------------------- main line
    wl = configs.BY_NAME[args.workload]
    if wl.kind == "decode":
        d = time_decode(wl, max(args.steps, 20), args.warmup, want_clocks=True)
        line = {
            "metric": "decode us/step (one new token for each of the batch's sequences)",
            "value": d["entry"]["us_per_step"], "unit": "us/step", "n_gpus": world,
            "steps": max(args.steps, 20), "warmup": args.warmup,
            "ms_per_step": round(d["us"] / 1e3, 5), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(wl, world),
                       "support_mean": d["entry"]["support_mean"],
                       "l2": "flushed (256 MiB write) before every timed step"},
            "roofline": d["entry"]["roofline"], "e2e": d["e2e"],
            "launch": d["entry"]["launch"], "eager_us_per_step": d["entry"]["eager_us_per_step"],
            **({"summary_append_us": d["entry"]["summary_append_us"]}
               if "summary_append_us" in d["entry"] else {}),
            **({"graph_error": d["entry"]["graph_error"]} if "graph_error" in d["entry"] else {}),
            "gpu_launches": 3 * max(args.steps, 20), "clocks": d["clocks"], "also": [],
        }
        if rank == 0:
            line["cpu_baseline"] = decode_cpu_baseline(wl, args.cpu_seconds)
        return line
    if args.backward:
        entry = time_attn_bwd(wl, args.steps, args.warmup)
        return {"metric": "stage-2 backward ms (dQ, dK, dV, dw)", "value": entry["bwd_ms"],
                "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
                "config": workload_config(wl, world), "backward": entry}
    main = time_prefill(wl, args.steps, args.warmup, want_clocks=True, keep_routing=rank == 0,
                        packed=args.packed)
    tokens_rank = wl.batch * wl.seq
    value = tokens_rank * world / (main["step_ms"] / 1e3)
    peak = peaks["bf16_tflops"]
    achieved = main["flops"] / (main["attn_ms"] / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "attn_fwd_tc_kernel", "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peaks_src} bf16 burst",
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "traffic": profile_traffic(
                    "attn_fwd_tc_packed" if args.packed else "attn_fwd_tc", wl.name,
                    "sparse_hierarchical_attention_chunk_b200/csrc/attn_tc.cuh"),
                "algorithmic_flops_per_launch": main["flops"],
                "tile_executed_flops_per_launch": main["exec_flops"],
                "tile_executed_frac": round(main["exec_flops"] / (main["attn_ms"] / 1e3) / 1e12 / peak, 4),
                "attn_ms": round(main["attn_ms"], 4)}
    stages = stage_rooflines(main)

    # ------------------------------------------------------------- e2e: host buffers
    # Every step copies its inputs (Q, K, V, qbar) up from pinned host
    # memory, runs the whole prefill through dash.prefill and copies O back
    # down.  Steps are independent requests, so, as a serving loop does, they
    # are pipelined over three streams with two device buffer sets: step i+1's
    # inputs go up while step i computes and step i-1's output comes down.
    # The timed span runs from the first upload to the last download.
    Q, K, V, qbar = main["inputs"]
    p = main["p"]
    hQ, hK, hV, hqb = (t.cpu().pin_memory() for t in (Q, K, V, qbar))
    hO = torch.empty(Q.shape, dtype=Q.dtype).pin_memory()
    bufs = [{"in": tuple(torch.empty_like(t) for t in (Q, K, V, qbar)),
             "out": dash.alloc_prefill(p, device)} for _ in range(2)]
    s_up, s_cmp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        for i in range(n):
            k = i % 2
            din, dout_ = bufs[k]["in"], bufs[k]["out"]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_cmp[k])        # step i-2 is done reading these inputs
                for d_, h_ in zip(din, (hQ, hK, hV, hqb)):
                    d_.copy_(h_, non_blocking=True)
                ev_in[k].record(s_up)
            s_cmp.wait_event(ev_in[k])
            if i >= 2:
                s_cmp.wait_event(ev_out[k])           # step i-2's output has been copied down
            dash.prefill(p, *din, out=dout_, with_lse=False, stream=s_cmp)
            ev_cmp[k].record(s_cmp)
            s_down.wait_event(ev_cmp[k])
            with torch.cuda.stream(s_down):
                hO.copy_(dout_["O"], non_blocking=True)
                ev_out[k].record(s_down)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e2e_steps = max(4, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    e2e_run(e2e_steps)
    s_down.wait_stream(s_cmp)
    e1.record(s_down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    assert dash.dash_get_error() == dash.DASH_OK
    h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV, hqb))
    d2h = hO.numel() * hO.element_size()
    e2e = {"value": round(tokens_rank * world / (e2e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
           "steps": e2e_steps,
           "schedule": "pinned host buffers; upload, prefill and download on three streams, "
                       "consecutive steps overlapped (two device buffer sets)"}
    del hQ, hK, hV, hO, bufs, main["inputs"]
    torch.cuda.empty_cache()

    also = []
    if not args.no_extra:
        # the fixed-budget baseline on the main workload
        also.append(time_topk_ablation(wl, args.steps, args.warmup))
        # the stage-2 backward (reference kernel) on the 8k workload
        also.append(time_attn_bwd(configs.PREFILL_8K, min(args.steps, 5), args.warmup))
        def prefill_entry(wlx, r, sigma=None, packed=False):
            ax = r["flops"] / (r["attn_ms"] / 1e3) / 1e12
            return {"workload": wlx.name, "metric": "prefill tokens/s",
                    "sigma": wlx.sigma if sigma is None else sigma,
                    "routing_form": "compact (dash_route_packed)" if packed else "dense w",
                    "value": round(wlx.batch * wlx.seq * world / (r["step_ms"] / 1e3), 1),
                    "ms_per_step": round(r["step_ms"], 3), "attn_ms": round(r["attn_ms"], 3),
                    "roofline": {"bound": "tensor", "achieved": round(ax, 2), "peak": peak,
                                 "unit": "TFLOP/s", "frac": round(ax / peak, 4),
                                 "algorithmic_flops_per_launch": r["flops"],
                                 "tile_executed_flops_per_launch": r["exec_flops"],
                                 "tile_executed_frac": round(
                                     r["exec_flops"] / (r["attn_ms"] / 1e3) / 1e12 / peak, 4),
                                 "traffic": profile_traffic(
                                     "attn_fwd_tc_packed" if packed else "attn_fwd_tc", wlx.name,
                                     "sparse_hierarchical_attention_chunk_b200/csrc/attn_tc.cuh")
                                 if sigma in (None, wlx.sigma) else None},
                    "stages": stage_rooflines(r),
                    "support_mean": round(r["support"], 4),
                    "support_per_kv_head": [round(x, 4) for x in r["per_head"]]}

        # 8k prefill
        wl2 = configs.PREFILL_8K
        r2 = time_prefill(wl2, args.steps, args.warmup)
        also.append(prefill_entry(wl2, r2))
        del r2
        # the main workload with the compact routing form
        rp = time_prefill(wl, args.steps, args.warmup, packed=True)
        also.append(prefill_entry(wl, rp, packed=True))
        del rp
        torch.cuda.empty_cache()
        # 128k prefill, sigma sweep on the same inputs (the support does not
        # depend on sigma, only the prior's strength does)
        wl4 = configs.PREFILL_128K
        for sg in (wl4.sigmas or (wl4.sigma,)):
            r4 = time_prefill(wl4, max(2, min(args.steps, 3)), args.warmup, sigma=sg)
            also.append(prefill_entry(wl4, r4, sigma=sg))
            del r4
            torch.cuda.empty_cache()
        r4 = time_prefill(wl4, max(2, min(args.steps, 3)), args.warmup, packed=True)
        also.append(prefill_entry(wl4, r4, packed=True))
        del r4
        torch.cuda.empty_cache()
        # decode, 8 sequences x 131072-token cache
        d5 = time_decode(configs.DECODE_128K, max(args.steps, 20), args.warmup)
        also.append(d5["entry"])
        torch.cuda.empty_cache()
        # the same caches with a length per sequence, contiguous and paged
        for wl6 in (configs.DECODE_VARLEN_128K, configs.DECODE_PAGED_128K):
            d6 = time_decode(wl6, max(args.steps, 20), args.warmup)
            also.append(d6["entry"])
            torch.cuda.empty_cache()

    line = {
        "metric": f"prefill tokens/s (stage 0+1+2) at seq {wl.seq}",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(main["step_ms"], 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(wl, world),
                   "routing_form": "compact (dash_route_packed)" if args.packed else "dense w",
                   "support_mean": round(main["support"], 4),
                   "support_per_kv_head": [round(x, 4) for x in main["per_head"]],
                   "l2": "flushed (256 MiB write) before every timed step"},
        "roofline": roofline,
        "stages": stages,
        "e2e": e2e,
        "gpu_launches": 3 * args.steps,
        "clocks": main["clocks"],
        "also": also,
    }
    if rank == 0:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, main.get("routing"))
    return line


# ---------------------------------------------------------------------------
# CPU oracle (the reported baseline; never tuned)
# ---------------------------------------------------------------------------
def oracle_inputs(wl, seed=0):
    """Inputs on the host plus the oracle's stage 0 over every chunk (timed)."""
    import oracle

    inp = synth.make_prefill(wl, seed=seed)
    t0 = time.perf_counter()
    kb = torch.from_numpy(oracle.chunk_summary(inp["K"], inp["qbar"], wl.chunk)).to(torch.bfloat16)
    return inp, kb, time.perf_counter() - t0


def oracle_sample_rate(wl, seconds, state, seed=0):
    """Time the oracle's stages 1-2 on random query positions for ~``seconds``.

    Stage 0 (all chunks; routing needs every summary) was timed once in
    ``state``.  Returns tokens/s for the whole workload, extrapolating the
    per-position time linearly to all positions, plus what was sampled.
    """
    import numpy as np
    import oracle

    inp, kb, t_stage0 = state
    rng = np.random.default_rng(seed)
    done, t_rows = 0, 0.0
    while t_rows < seconds:
        pos = np.sort(rng.choice(np.arange(wl.seq), size=8, replace=False))
        t1 = time.perf_counter()
        w, m, _ = oracle.route(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk, positions=pos)
        oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], w, m, wl.sigma, wl.chunk, positions=pos)
        t_rows += time.perf_counter() - t1
        done += pos.size
    total = t_stage0 + t_rows * wl.seq / done
    return wl.batch * wl.seq / total, done, t_stage0 + t_rows


def routing_flips(wl, routing, n_pos=64, seed=7):
    """Mask bits of the timed run's routing that differ from the oracle's,
    on a seeded sample of positions: stage 1 of the oracle on the GPU's own
    summaries, compared bit by bit; flips are allowed only where some head's
    score lies within 1e-4 of its threshold."""
    import numpy as np
    import oracle

    rng = np.random.default_rng(seed)
    pos = np.sort(rng.choice(np.arange(wl.chunk, wl.seq), size=n_pos, replace=False))
    w, m, near = oracle.route(routing["Q"], routing["Kbar"], wl.alpha, wl.gamma, wl.chunk,
                              positions=pos, near_tol=1e-4)
    gm = routing["mask"].numpy().view(np.uint32)[:, :, pos]
    a, b_ = oracle.unpack_mask(gm, wl.n_chunks), oracle.unpack_mask(m, wl.n_chunks)
    diff = a != b_
    wmax = float(np.abs(routing["w"].numpy()[:, :, pos].astype(np.float64) - w).max())
    return {"positions": int(pos.size), "rows": int(pos.size * wl.batch * wl.n_kv_heads),
            "mask_flips": int(diff.sum()), "flips_within_1e-4_of_tau": int((diff & near).sum()),
            "flips_elsewhere": int((diff & ~near).sum()), "w_max_abs_err": wmax,
            "how": "oracle stage 1 on the GPU's summaries at seeded positions (not timed)"}


def cpu_baseline(wl, seconds, routing=None):
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    state = oracle_inputs(wl)
    rate, done, spent = oracle_sample_rate(wl, seconds, state)
    res = {"value": round(rate, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "host_cpus": os.cpu_count(), "extrapolated": True,
           "sample": f"stage 0 on all chunks + stages 1-2 for {done} sampled query positions "
                     f"(all heads), {spent:.1f} s of CPU time, extrapolated linearly to "
                     f"{wl.seq} positions"}
    if routing is not None:
        res["routing_parity"] = routing_flips(wl, routing)
    return res


def decode_cpu_baseline(wl, seconds):
    """The oracle's decode (summaries + one query) on whole sequences, repeated for ~seconds.

    Returns us/step for the whole batch: the per-sequence time x batch.
    """
    import oracle

    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    inp = synth.make_decode(wl, seed=0)
    lens = inp.get("lens")
    done, spent = 0, 0.0
    while spent < seconds and done < wl.batch:
        sl = slice(done, done + 1)
        L = wl.seq if lens is None else int(lens[done])
        n_c = (L - 1) // wl.chunk
        t0 = time.perf_counter()
        kb = oracle.chunk_summary(inp["K"][sl, :, :L], inp["qbar"], wl.chunk, 0, n_c)
        oracle.decode(inp["q"][sl], inp["K"][sl, :, :L], inp["V"][sl, :, :L], kb, L, wl.alpha,
                      wl.gamma, wl.sigma, wl.chunk)
        spent += time.perf_counter() - t0
        done += 1
    us = spent / done * wl.batch * 1e6
    return {"value": round(us, 1), "unit": "us/step", "cores": threads, "kind": "oracle",
            "host_cpus": os.cpu_count(),
            "sample": f"{done} of {wl.batch} sequences (chunk summaries of the sequence's cache + "
                      f"routing + attention, all heads), {spent:.1f} s of CPU time, scaled "
                      f"to the batch"}


def workload_config(wl, world):
    """The workload-identifying part of a bench line's config (both arms)."""
    cfg = {"workload": wl.name, "batch": wl.batch}
    if wl.kind == "decode":
        cfg["cache_len"] = wl.seq
        lens = synth.cache_lengths(wl, 0)
        if lens is not None:
            cfg["cache_lens"] = [int(x) for x in lens.tolist()]
        if wl.paged:
            cfg["kv_layout"] = "paged (one chunk per page, shuffled pool + 64 unused pages)"
    else:
        cfg["seq_len"] = wl.seq
    cfg.update({"heads": f"{wl.n_q_heads}/{wl.n_kv_heads}", "head_dim": wl.head_dim,
                "chunk": wl.chunk, "alpha": wl.alpha, "gamma": wl.gamma, "sigma": wl.sigma,
                "parallelism": f"replicas x{world} (independent sequences, no exchange)"})
    return cfg


def run_reference(args, rank, world):
    wl = configs.BY_NAME[args.workload]
    if wl.kind == "decode":
        vals = []
        for s in range(args.warmup + args.steps):
            cb = decode_cpu_baseline(wl, args.ref_seconds)
            if s >= args.warmup:
                vals.append(cb["value"])
        v = statistics.mean(vals)
        cb["value"] = round(v, 1)
        return {"impl": "reference",
                "metric": "decode us/step (one new token for each of the batch's sequences)",
                "value": round(v, 1), "unit": "us/step", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(v / 1e3, 3),
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": workload_config(wl, world),
                "cpu_baseline": cb,
                "e2e": {"value": round(v, 1), "unit": "us/step", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    steps = []
    state = oracle_inputs(wl)
    for s in range(args.warmup + args.steps):
        rate, done, spent = oracle_sample_rate(wl, args.ref_seconds, state, seed=s)
        if s >= args.warmup:
            steps.append(rate)
    value = statistics.mean(steps)
    ms = wl.batch * wl.seq / value * 1e3
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    return {"impl": "reference", "metric": f"prefill tokens/s (stage 0+1+2) at seq {wl.seq}",
            "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 1), "extrapolated": True,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, world),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"per step: stage 0 on all chunks (timed once) + stages 1-2 on "
                                       f"~{args.ref_seconds:.0f} s of sampled positions, "
                                       f"extrapolated to {wl.seq} positions"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=configs.PREFILL_32K.name, choices=sorted(configs.BY_NAME))
    ap.add_argument("--no-extra", action="store_true", help="skip the 128k prefill / decode lines")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=8.0)
    ap.add_argument("--packed", action="store_true",
                    help="main line on the compact routing form (dash_route_packed)")
    ap.add_argument("--backward", action="store_true",
                    help="only the stage-2 backward of --workload, beside its forward stage 2")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank, world, local = shard.rank_world()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    line = run_ours(args, rank, world, device)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
