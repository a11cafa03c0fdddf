"""Host-side pieces of bench.py (no GPU): the algorithmic byte count of a
decode step, the workload config that both arms of the bench print, and the
DRAM traffic it takes from the committed ncu summaries."""

import importlib.util
import os
import re
import shutil

import torch

from sparse_hierarchical_attention_chunk_b200 import configs, synth

_spec = importlib.util.spec_from_file_location(
    "bench_mod", os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def _mask(wl, active_per_row, seed=0):
    g = torch.Generator().manual_seed(seed)
    nw = (wl.n_chunks + 31) // 32
    m = torch.zeros(wl.batch, wl.n_kv_heads, nw, dtype=torch.int32)
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            for c in torch.randperm(wl.n_chunks - 1, generator=g)[:active_per_row].tolist():
                m[b, h, c // 32] |= (1 << (c % 32)) if c % 32 < 31 else -(1 << 31)
    return m


def test_decode_bytes_varlen_reduces_to_fixed_length():
    wl = configs.DECODE_128K
    m = _mask(wl, 100)
    fixed, f1 = bench.decode_bytes(wl, m)
    same, f2 = bench.decode_bytes(wl, m, torch.full((wl.batch,), wl.seq, dtype=torch.int32))
    assert fixed == same and abs(f1 - f2) < 1e-12
    # by hand: active K/V blocks + the diagonal keys, the eligible summaries, q/o, w/mask
    B, d, hkv, b = wl.chunk, wl.head_dim, wl.n_kv_heads, wl.batch
    c_q = (wl.seq - 1) // B
    want = ((100 * b * hkv) * B + (wl.seq - c_q * B) * b * hkv) * d * 4 + b * hkv * c_q * d * 2 \
        + 2 * b * wl.n_q_heads * d * 2 + b * hkv * (wl.n_chunks * 4 + ((wl.n_chunks + 31) // 32) * 4)
    assert fixed == want


def test_decode_bytes_shorter_caches_count_fewer_summaries():
    wl = configs.DECODE_VARLEN_128K
    m = _mask(wl, 50)
    full, _ = bench.decode_bytes(wl, m, torch.full((wl.batch,), wl.seq, dtype=torch.int32))
    lens = synth.cache_lengths(wl, 0)
    short, _ = bench.decode_bytes(wl, m, lens)
    assert short < full


def test_workload_config_is_shared_by_both_arms():
    for wl in configs.ALL:
        cfg = bench.workload_config(wl, 1)
        assert cfg["workload"] == wl.name and cfg["batch"] == wl.batch
        assert ("cache_len" in cfg) == (wl.kind == "decode")
        assert ("cache_lens" in cfg) == (wl.min_len_frac > 0)
        assert ("kv_layout" in cfg) == wl.paged


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = "sparse_hierarchical_attention_chunk_b200/csrc/"
PROFILED = [("attn_fwd_tc", "prefill_bf16_s32768", "attn_tc.cuh"),
            ("attn_fwd_tc", "prefill_bf16_s131072", "attn_tc.cuh"),
            ("attn_fwd_tc_packed", "prefill_bf16_s131072", "attn_tc.cuh"),
            ("decode", "decode_bf16_b8_L131072", "decode.cuh"),
            ("decode", "decode_varlen_bf16_b8_L131072", "decode.cuh"),
            ("decode", "decode_paged_bf16_b8_L131072", "decode.cuh")]


def _dram_bytes(text):
    unit = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    return sum(float(v) * unit[u] for v, u in re.findall(r"DRAM (?:read|write)\s+([0-9.]+) (\w+)", text))


def test_profile_traffic_of_the_committed_summaries():
    # every summary the bench line draws on was taken on the current source,
    # and the traffic it reports is the summary's DRAM read + write
    for tag, wl, src in PROFILED:
        got = bench.profile_traffic(tag, wl, CSRC + src)
        assert got is not None, (tag, wl)
        text = open(os.path.join(ROOT, "profiles", f"{tag}_{wl}.txt")).read()
        assert got == int(_dram_bytes(text)), (tag, wl)
        assert got > 0


def test_profile_traffic_is_none_once_the_source_changed(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    shutil.copy(os.path.join(ROOT, "profiles", "attn_fwd_tc_prefill_bf16_s32768.txt"), tmp_path / "profiles")
    src = tmp_path / "attn_tc.cuh"
    src.write_bytes(open(os.path.join(ROOT, CSRC, "attn_tc.cuh"), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("attn_fwd_tc", "prefill_bf16_s32768", "attn_tc.cuh") is not None
    src.write_bytes(src.read_bytes() + b"\n// changed\n")
    assert bench.profile_traffic("attn_fwd_tc", "prefill_bf16_s32768", "attn_tc.cuh") is None
    assert bench.profile_traffic("attn_fwd_tc", "no_such_workload", "attn_tc.cuh") is None
