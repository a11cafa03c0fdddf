"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every case draws its inputs from the seeded generator on the CPU, copies them
to the GPU, and compares element by element with the oracle on the same
values.  Stage-isolated cases hand each CUDA stage the oracle's upstream
result (rounded to the dtype the kernel reads), so a rounding difference in
one stage cannot flip a mask bit in the next.  Tolerances: mask bit-exact
except where some head has |x - tau| < 1e-4 (counted); w max-abs 1e-3; bf16
O max-abs 2e-2; fp32 O max-abs 1e-4.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from sparse_hierarchical_attention_chunk_b200 import configs, dash, synth
from _util import (NEAR_TAU, TOL_LSE, TOL_O_BF16, TOL_O_F32, TOL_W, compare_masks, mask_from_dev,
                   mask_to_dev, np64, oracle_kbar, to_dev)

pytestmark = pytest.mark.gpu

W = configs.Workload
# medium cases: several tiles and chunks, ragged mask words, other GQA shapes
MED = {
    "g16_d128_b64_nc37": W("med_g16", "prefill", 1, 32, 2, 37 * 64, 128, 64, rho=(0.9, 0.9), needles=(3, 2)),
    "g16_d128_b128_s05": W("med_b128", "prefill", 1, 32, 2, 20 * 128, 128, 128, sigma=0.5,
                           rho=(0.9, 0.0), needles=(2, 0)),
    "g8_d64_b64_batch2": W("med_g8", "prefill", 2, 16, 2, 1024, 64, 64, sigma=1.0, rho=(0.8, 0.8),
                           needles=(2, 2)),
    "g4_d128_sigma0": W("med_g4", "prefill", 1, 8, 2, 1024, 128, 64, sigma=0.0, rho=(0.5, 0.9),
                        needles=(1, 1)),
    "alpha2_sparsemax": W("med_a2", "prefill", 1, 32, 2, 1024, 128, 64, alpha=2.0, rho=(0.9, 0.9),
                          needles=(2, 2)),
    "alpha13_generic": W("med_a13", "prefill", 1, 32, 2, 1024, 128, 64, alpha=1.3, rho=(0.9, 0.9),
                         needles=(2, 2)),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_hierarchical_attention_chunk_b200 import build
    build.build()
    dash.lib()


def _dt(wl):
    return synth.torch_dtype(wl.dtype)


def _tol_o(wl):
    return TOL_O_F32 if wl.dtype == "f32" else TOL_O_BF16


# ----------------------------------------------------------------------------
# stage 0
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("zero_qbar", [False, True])
def test_summarize_tiny_f32(zero_qbar):
    wl = configs.TINY_F32
    inp = synth.make_prefill(wl, seed=1, zero_qbar=zero_qbar)
    p = dash.problem_for(wl)
    K, qbar = inp["K"].cuda(), inp["qbar"].cuda()
    Kbar = torch.empty(1, 1, wl.seq // wl.chunk, wl.head_dim, device="cuda")
    dash.dash_summarize(p, K, qbar, Kbar)
    ref = oracle.chunk_summary(inp["K"], inp["qbar"], wl.chunk)
    assert np.abs(np64(Kbar) - ref).max() < 1e-5


@pytest.mark.parametrize("name", ["g16_d128_b64_nc37", "g16_d128_b128_s05", "g8_d64_b64_batch2"])
def test_summarize_bf16(name):
    wl = MED[name]
    inp = synth.make_prefill(wl, seed=2)
    p = dash.problem_for(wl)
    Kbar = torch.empty(wl.batch, wl.n_kv_heads, wl.seq // wl.chunk, wl.head_dim, dtype=torch.bfloat16,
                       device="cuda")
    dash.dash_summarize(p, inp["K"].cuda(), inp["qbar"].cuda(), Kbar)
    ref = oracle.chunk_summary(inp["K"], inp["qbar"], wl.chunk)
    # one bf16 rounding of an fp32 accumulation: relative 2^-8
    err = np.abs(np64(Kbar) - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6)


def test_summarize_partial_range_appends():
    wl = MED["g16_d128_b64_nc37"]
    inp = synth.make_prefill(wl, seed=3)
    p = dash.problem_for(wl)
    Kbar = torch.zeros(1, 2, 37, 128, dtype=torch.bfloat16, device="cuda")
    K, qb = inp["K"].cuda(), inp["qbar"].cuda()
    dash.dash_summarize(p, K, qb, Kbar, 0, 20)
    dash.dash_summarize(p, K, qb, Kbar, 20, 37)
    full = torch.empty_like(Kbar)
    dash.dash_summarize(p, K, qb, full)
    assert torch.equal(Kbar, full)
    empty = torch.zeros_like(Kbar)
    dash.dash_summarize(p, K, qb, empty, 5, 5)          # empty range: no work
    assert int(empty.abs().sum()) == 0


# ----------------------------------------------------------------------------
# stage 1
# ----------------------------------------------------------------------------

def _route_case(wl, seed, positions=None, diag=False):
    inp = synth.make_prefill(wl, seed=seed)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, _dt(wl))
    p = dash.problem_for(wl, estimate_diagonal=diag)
    n_c = wl.n_chunks
    w = torch.empty(wl.batch, wl.n_kv_heads, wl.seq, n_c, device="cuda")
    mask = torch.empty(wl.batch, wl.n_kv_heads, wl.seq, (n_c + 31) // 32, dtype=torch.int32, device="cuda")
    dash.dash_route(p, inp["Q"].cuda(), kb.cuda(), w, mask, K=inp["K"].cuda(), qbar=inp["qbar"].cuda())
    torch.cuda.synchronize()
    wr, mr, near = oracle.route(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk, positions=positions,
                                diag=(inp["K"], inp["qbar"]) if diag else None)
    pos = slice(None) if positions is None else positions
    wg = np64(w)[:, :, pos]
    mg = mask_from_dev(mask)[:, :, pos]
    return wg, mg, wr, mr, near


@pytest.mark.parametrize("name", list(MED))
def test_route_matches_oracle(name):
    wl = MED[name]
    wg, mg, wr, mr, near = _route_case(wl, seed=4)
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    assert n_bad == 0, f"{n_bad} mask bits differ away from tau ({n_diff} total)"
    assert np.abs(wg - wr).max() <= TOL_W
    # rows of the first chunk route nowhere
    assert np.all(wg[:, :, :wl.chunk] == 0) and np.all(mg[:, :, :wl.chunk] == 0)


def test_route_more_than_512_chunks_sampled():
    # 600 chunks: the tensor-core routing kernel keeps 4 positions per CTA and
    # stores chunks >= 512 in the upper 16-lane halves of TMEM
    wl = W("med_split", "prefill", 1, 32, 2, 600 * 64, 128, 64, rho=(0.9, 0.2), needles=(3, 1))
    pos = np.array([0, 63, 64, 100, 511 * 64 + 5, 512 * 64, 513 * 64 + 17, 530 * 64 + 63,
                    599 * 64, 600 * 64 - 1])
    wg, mg, wr, mr, near = _route_case(wl, seed=14, positions=pos)
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    assert n_bad == 0, f"{n_bad} mask bits differ away from tau ({n_diff} total)"
    assert np.abs(wg - wr).max() <= TOL_W


@pytest.mark.parametrize("name", list(MED))
def test_route_estimate_diagonal_matches_oracle(name):
    # the query's own chunk as one more entmax candidate (tensor-core routing
    # for the G = 16, d = 128 cases, the generic kernel for the others)
    wl = MED[name]
    wg, mg, wr, mr, near = _route_case(wl, seed=31, diag=True)
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    print(f"near-threshold mask flips: {n_diff}")
    assert n_bad == 0, f"{n_bad} mask bits differ away from tau ({n_diff} total)"
    assert np.abs(wg - wr).max() <= TOL_W
    # the diagonal's weight is reported in column c_i; rows of the first chunk give it 1
    c_i = np.arange(wl.seq) // wl.chunk
    wd = np.take_along_axis(wg, c_i[None, None, :, None], axis=-1)[..., 0]
    assert np.allclose(wd[:, :, :wl.chunk], 1.0)
    assert np.any((wd > 0) & (wd < 1))                  # the candidate really competes


def test_route_estimate_diagonal_more_than_512_chunks_sampled():
    wl = W("med_split", "prefill", 1, 32, 2, 600 * 64, 128, 64, rho=(0.9, 0.2), needles=(3, 1))
    pos = np.array([0, 63, 64, 100, 511 * 64 + 5, 511 * 64 + 63, 512 * 64, 513 * 64 + 17,
                    530 * 64 + 63, 599 * 64, 600 * 64 - 1])
    wg, mg, wr, mr, near = _route_case(wl, seed=32, positions=pos, diag=True)
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    assert n_bad == 0, f"{n_bad} mask bits differ away from tau ({n_diff} total)"
    assert np.abs(wg - wr).max() <= TOL_W


def test_route_estimate_diagonal_tiny_f32():
    wl = configs.TINY_F32
    wg, mg, wr, mr, near = _route_case(wl, seed=33, diag=True)
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    assert n_bad == 0
    assert np.abs(wg - wr).max() <= 1e-5


def test_route_tiny_f32():
    wl = configs.TINY_F32
    wg, mg, wr, mr, near = _route_case(wl, seed=5)
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    assert n_bad == 0
    assert np.abs(wg - wr).max() <= 1e-5


# ----------------------------------------------------------------------------
# compact routing form: the routed chunks of each row and their weights
# ----------------------------------------------------------------------------

def _route_packed_case(wl, seed, diag=False):
    inp = synth.make_prefill(wl, seed=seed)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, _dt(wl)).cuda()
    p = dash.problem_for(wl, estimate_diagonal=diag)
    n_c, rows = wl.n_chunks, (wl.batch, wl.n_kv_heads, wl.seq)
    Q, K, qb = inp["Q"].cuda(), inp["K"].cuda(), inp["qbar"].cuda()
    w = torch.empty(rows + (n_c,), device="cuda")
    mask = torch.empty(rows + ((n_c + 31) // 32,), dtype=torch.int32, device="cuda")
    dash.dash_route(p, Q, kb, w, mask, K=K, qbar=qb)
    pm = torch.empty_like(mask)
    weight = torch.full(rows + (n_c,), 7.0, device="cuda")     # untouched past each count
    index = torch.full(rows + (n_c,), -7, dtype=torch.int32, device="cuda")
    count = torch.empty(rows, dtype=torch.int32, device="cuda")
    dash.dash_route_packed(p, Q, kb, pm, weight, count, index, K=K, qbar=qb)
    assert dash.dash_get_error() == dash.DASH_OK
    return inp, kb, w, mask, pm, weight, index, count


@pytest.mark.parametrize("name,diag", [("g16_d128_b64_nc37", False), ("g16_d128_b128_s05", False),
                                       ("g8_d64_b64_batch2", False), ("alpha13_generic", False),
                                       ("g16_d128_b64_nc37", True), ("g8_d64_b64_batch2", True)])
def test_route_packed_is_the_dense_routing_compacted(name, diag):
    wl = MED[name]
    inp, kb, w, mask, pm, weight, index, count = _route_packed_case(wl, 38, diag)
    # the same routing, written compactly: the same bits, and every listed
    # weight is the dense kernel's weight at that chunk, in chunk order
    assert torch.equal(pm, mask)
    c_ref, i_ref, w_ref = oracle.pack_weights(np64(w), mask_from_dev(mask))
    cnt = count.cpu().numpy()
    assert (cnt == c_ref).all()
    k = np.arange(wl.n_chunks)[None, None, None, :]
    live = k < cnt[..., None]
    assert (np.where(live, index.cpu().numpy(), -1) == i_ref).all()
    assert (np.where(live, np64(weight), 0.0) == w_ref).all()
    assert (np.where(live, 0, index.cpu().numpy() + 7) == 0).all()       # untouched past count
    assert (np.where(live, 7.0, np64(weight)) == 7.0).all()
    # and against the oracle's routing, packed
    wr, mr, near = oracle.route(inp["Q"], kb.cpu(), wl.alpha, wl.gamma, wl.chunk,
                                diag=(inp["K"], inp["qbar"]) if diag else None)
    n_diff, n_bad = compare_masks(mask_from_dev(pm), mr, near, wl.n_chunks)
    assert n_bad == 0
    dense, _ = oracle.unpack_weights(cnt, index.cpu().numpy(), np64(weight), wl.n_chunks)
    wr_routed = np.where(oracle.unpack_mask(mr, wl.n_chunks), wr, 0.0)
    assert np.abs(dense - wr_routed).max() <= TOL_W


def test_route_packed_more_than_512_chunks():
    wl = W("med_split", "prefill", 1, 32, 2, 600 * 64, 128, 64, rho=(0.9, 0.2), needles=(3, 1))
    inp, kb, w, mask, pm, weight, index, count = _route_packed_case(wl, 39)
    assert torch.equal(pm, mask)
    pos = np.array([0, 64, 511 * 64 + 5, 512 * 64, 530 * 64 + 63, 600 * 64 - 1])
    c_ref, i_ref, w_ref = oracle.pack_weights(np64(w[:, :, pos]), mask_from_dev(mask[:, :, pos]))
    cnt = count[:, :, pos].cpu().numpy()
    assert (cnt == c_ref).all()
    live = np.arange(wl.n_chunks)[None, None, None, :] < cnt[..., None]
    assert (np.where(live, index[:, :, pos].cpu().numpy(), -1) == i_ref).all()
    assert (np.where(live, np64(weight[:, :, pos]), 0.0) == w_ref).all()


@pytest.mark.parametrize("name", ["g16_d128_b64_nc37", "g16_d128_b128_s05", "g4_d128_sigma0"])
def test_attn_packed_gives_the_dense_bits(name):
    wl = MED[name]
    inp, kb, w, mask, pm, weight, index, count = _route_packed_case(wl, 40)
    p = dash.problem_for(wl)
    Q, K, V = inp["Q"].cuda(), inp["K"].cuda(), inp["V"].cuda()
    O1, O2 = torch.empty_like(Q), torch.empty_like(Q)
    l1 = torch.empty(Q.shape[:3], device="cuda")
    l2 = torch.empty_like(l1)
    dash.dash_attn_fwd(p, Q, K, V, w, mask, O1, l1)
    dash.dash_attn_fwd_packed(p, Q, K, V, weight, pm, O2, l2)
    assert dash.dash_get_error() == dash.DASH_OK
    assert torch.equal(O1, O2) and torch.equal(l1, l2)
    Or, lr = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], np64(w), mask_from_dev(mask), wl.sigma,
                             wl.chunk)
    assert np.abs(np64(O2) - Or).max() <= TOL_O_BF16


@pytest.mark.parametrize("zero_qbar", [False, True])
def test_prefill_packed_tiny_f32(zero_qbar):
    wl = configs.TINY_F32
    inp = synth.make_prefill(wl, seed=41, zero_qbar=zero_qbar)
    p = dash.problem_for(wl)
    dev = [inp[n].cuda() for n in ("Q", "K", "V", "qbar")]
    a = dash.prefill(p, *dev)
    b = dash.prefill(p, *dev, packed=True)
    torch.cuda.synchronize()
    assert torch.equal(a["mask"], b["mask"]) and torch.equal(a["O"], b["O"])
    kb = oracle.chunk_summary(inp["K"], inp["qbar"], wl.chunk)
    wr, mr, near = oracle.route(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk)
    Or, _ = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], wr, mr, wl.sigma, wl.chunk)
    assert np.abs(np64(b["O"]) - Or).max() <= TOL_O_F32


# ----------------------------------------------------------------------------
# stage 2
# ----------------------------------------------------------------------------

def _attn_case(wl, seed, sigma=None, dense=False, zero_qbar=False):
    sigma = wl.sigma if sigma is None else sigma
    inp = synth.make_prefill(wl, seed=seed, zero_qbar=zero_qbar)
    n_c = wl.n_chunks
    if dense:
        wr = np.full((wl.batch, wl.n_kv_heads, wl.seq, n_c), 1.0)
        mr = oracle.pack_mask(np.ones_like(wr, dtype=bool))
    else:
        kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, _dt(wl))
        wr, mr, _ = oracle.route(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk)
    p = dash.problem_for(wl, sigma=sigma)
    dt = _dt(wl)
    O = torch.empty(wl.batch, wl.n_q_heads, wl.seq, wl.head_dim, dtype=dt, device="cuda")
    lse = torch.empty(wl.batch, wl.n_q_heads, wl.seq, device="cuda")
    dash.dash_attn_fwd(p, inp["Q"].cuda(), inp["K"].cuda(), inp["V"].cuda(), to_dev(wr, torch.float32),
                       mask_to_dev(mr), O, lse)
    assert dash.dash_get_error() == dash.DASH_OK
    Or, lr = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], wr, mr, sigma, wl.chunk)
    return np64(O), np64(lse), Or, lr, inp


@pytest.mark.parametrize("name", list(MED))
def test_attn_matches_oracle(name):
    wl = MED[name]
    O, lse, Or, lr, _ = _attn_case(wl, seed=6)
    assert np.abs(O - Or).max() <= TOL_O_BF16
    assert np.abs(lse - lr).max() <= TOL_LSE


@pytest.mark.parametrize("sigma", [0.0, 0.5, 1.0])
def test_attn_sigma_sweep(sigma):
    wl = MED["g16_d128_b128_s05"]
    O, lse, Or, lr, _ = _attn_case(wl, seed=7, sigma=sigma)
    assert np.abs(O - Or).max() <= TOL_O_BF16


def test_attn_dense_special_case_is_causal_sdpa():
    # all chunks active, sigma = 0: dense causal attention (torch SDPA in fp32)
    wl = MED["g16_d128_b64_nc37"]
    O, lse, Or, lr, inp = _attn_case(wl, seed=8, sigma=0.0, dense=True)
    assert np.abs(O - Or).max() <= TOL_O_BF16
    q, k, v = (inp[n].cuda().float() for n in ("Q", "K", "V"))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
    assert np.abs(O - np64(ref)).max() <= TOL_O_BF16


@pytest.mark.parametrize("zero_qbar", [False, True])
def test_attn_tiny_f32(zero_qbar):
    wl = configs.TINY_F32
    O, lse, Or, lr, _ = _attn_case(wl, seed=9, zero_qbar=zero_qbar)
    assert np.abs(O - Or).max() <= TOL_O_F32
    assert np.abs(lse - lr).max() <= 1e-4


# ----------------------------------------------------------------------------
# end to end: stage 0 -> 1 -> 2 on the GPU against the oracle's chain
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("zero_qbar", [False, True])
def test_end_to_end_tiny_f32(zero_qbar):
    wl = configs.TINY_F32
    inp = synth.make_prefill(wl, seed=10, zero_qbar=zero_qbar)
    p = dash.problem_for(wl)
    out = dash.prefill(p, inp["Q"].cuda(), inp["K"].cuda(), inp["V"].cuda(), inp["qbar"].cuda())
    torch.cuda.synchronize()
    kb = oracle.chunk_summary(inp["K"], inp["qbar"], wl.chunk)
    wr, mr, near = oracle.route(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk)
    Or, lr = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], wr, mr, wl.sigma, wl.chunk)
    n_diff, n_bad = compare_masks(mask_from_dev(out["mask"]), mr, near, wl.n_chunks)
    assert n_bad == 0
    assert np.abs(np64(out["w"]) - wr).max() <= 1e-5
    assert np.abs(np64(out["O"]) - Or).max() <= TOL_O_F32


def test_end_to_end_bf16():
    # the GPU chain (summaries -> routing -> attention, one dash.prefill call);
    # every output is compared, each stage against the oracle run on the
    # GPU's own upstream result (a bf16 summary one ulp away from the
    # oracle's moves a logit by ~1e-3, which would otherwise decide mask
    # bits near the threshold differently)
    wl = MED["g16_d128_b64_nc37"]
    inp = synth.make_prefill(wl, seed=11)
    p = dash.problem_for(wl)
    out = dash.prefill(p, inp["Q"].cuda(), inp["K"].cuda(), inp["V"].cuda(), inp["qbar"].cuda())
    assert dash.dash_get_error() == dash.DASH_OK
    ref_kb = oracle.chunk_summary(inp["K"], inp["qbar"], wl.chunk)
    kb = np64(out["Kbar"])
    assert np.all(np.abs(kb - ref_kb) <= 2.0 ** -8 * np.abs(ref_kb) + 1e-6)
    wr, mr, near = oracle.route(inp["Q"], out["Kbar"].cpu(), wl.alpha, wl.gamma, wl.chunk)
    mg = mask_from_dev(out["mask"])
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    print(f"near-threshold mask flips: {n_diff}")
    assert n_bad == 0
    wg = np64(out["w"])
    assert np.abs(wg - wr).max() <= TOL_W
    Or, lr = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], wg, mg, wl.sigma, wl.chunk)
    assert np.abs(np64(out["O"]) - Or).max() <= TOL_O_BF16
    assert np.abs(np64(out["lse"]) - lr).max() <= TOL_LSE


def test_end_to_end_estimate_diagonal_bf16():
    # the chain with the diagonal candidate in the routing: every output,
    # each stage on the GPU's own upstream result
    wl = MED["g16_d128_b64_nc37"]
    inp = synth.make_prefill(wl, seed=37)
    p = dash.problem_for(wl, estimate_diagonal=True)
    out = dash.prefill(p, inp["Q"].cuda(), inp["K"].cuda(), inp["V"].cuda(), inp["qbar"].cuda())
    torch.cuda.synchronize()
    wr, mr, near = oracle.route(inp["Q"], out["Kbar"].cpu(), wl.alpha, wl.gamma, wl.chunk,
                                diag=(inp["K"], inp["qbar"]))
    mg = mask_from_dev(out["mask"])
    n_diff, n_bad = compare_masks(mg, mr, near, wl.n_chunks)
    assert n_bad == 0
    wg = np64(out["w"])
    assert np.abs(wg - wr).max() <= TOL_W
    Or, lr = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], wg, mg, wl.sigma, wl.chunk)
    assert np.abs(np64(out["O"]) - Or).max() <= TOL_O_BF16
    assert np.abs(np64(out["lse"]) - lr).max() <= TOL_LSE


# ----------------------------------------------------------------------------
# full-size workloads: sampled rows (rows are independent given K, V, Kbar)
# ----------------------------------------------------------------------------

def _sample_positions(wl, n, seed):
    rng = np.random.default_rng(seed)
    tail = [wl.seq - 1, wl.seq - 8, wl.chunk, wl.chunk - 1, 0]
    pick = rng.choice(np.arange(wl.seq), size=n, replace=False)
    return np.unique(np.concatenate([pick, tail]))


@pytest.mark.parametrize("wl", [configs.PREFILL_8K, configs.PREFILL_32K, configs.PREFILL_128K],
                         ids=lambda w: w.name)
def test_full_size_sampled_rows(wl):
    inp = synth.make_prefill(wl, seed=0)
    p = dash.problem_for(wl)
    dev = {k: inp[k].cuda() for k in ("Q", "K", "V", "qbar")}
    out = dash.prefill(p, dev["Q"], dev["K"], dev["V"], dev["qbar"])
    torch.cuda.synchronize()
    kb_gpu = out["Kbar"]
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16)
    # stage 0 on every chunk
    ref_kb = oracle.chunk_summary(inp["K"], inp["qbar"], wl.chunk)
    assert np.all(np.abs(np64(kb_gpu) - ref_kb) <= 2.0 ** -8 * np.abs(ref_kb) + 1e-6)
    pos = _sample_positions(wl, 24, seed=1)
    # stage 1, isolated: route again on the GPU from the oracle's summaries
    n_c = wl.n_chunks
    w = torch.empty(1, wl.n_kv_heads, wl.seq, n_c, device="cuda")
    mask = torch.empty(1, wl.n_kv_heads, wl.seq, (n_c + 31) // 32, dtype=torch.int32, device="cuda")
    dash.dash_route(p, dev["Q"], kb.cuda(), w, mask)
    wr, mr, near = oracle.route(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk, positions=pos)
    mg = mask_from_dev(mask)[:, :, pos]
    n_diff, n_bad = compare_masks(mg, mr, near, n_c)
    assert n_bad == 0
    assert np.abs(np64(w)[:, :, pos] - wr).max() <= TOL_W
    # stage 2, isolated: GPU attention with this routing, rows at the sampled positions
    sigmas = wl.sigmas or (wl.sigma,)
    for sg in sigmas:
        ps = dash.problem_for(wl, sigma=sg)
        O = torch.empty_like(dev["Q"])
        dash.dash_attn_fwd(ps, dev["Q"], dev["K"], dev["V"], w, mask, O)
        assert dash.dash_get_error() == dash.DASH_OK
        Or, _ = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], np64(w)[:, :, pos],
                                mask_from_dev(mask)[:, :, pos], sg, wl.chunk, positions=pos)
        assert np.abs(np64(O[:, :, pos]) - Or).max() <= TOL_O_BF16
        del O
    del out, dev
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------

DEC = {
    "b2_L1000_ragged": W("dec_small", "decode", 2, 32, 2, 1000, 128, 64, gamma=0.3, rho=(0.9, 0.9),
                         needles=(2, 2)),
    "b3_L64_first_chunk": W("dec_first", "decode", 3, 32, 2, 64, 128, 64, rho=(0.9, 0.9),
                            needles=(0, 0)),
    "b1_L4097_b128_g8": W("dec_b128", "decode", 1, 16, 2, 4097, 128, 128, gamma=0.5, sigma=0.5,
                          rho=(0.9, 0.5), needles=(2, 1)),
    "b4_L3000_d64_g4": W("dec_d64", "decode", 4, 8, 2, 3000, 64, 64, rho=(0.9, 0.5),
                         needles=(2, 1)),
    "b2_L5000_b128_sparsemax_sigma0": W("dec_a2", "decode", 2, 32, 2, 5000, 128, 128, alpha=2.0,
                                        sigma=0.0, rho=(0.9, 0.9), needles=(2, 2)),
    "b2_L2000_alpha13": W("dec_a13", "decode", 2, 32, 2, 2000, 128, 64, alpha=1.3,
                          rho=(0.9, 0.9), needles=(2, 2)),
    # 64 (b, h_kv) segments over 148 CTAs: most CTAs hold pieces of several
    # segments and most segments are merged from several CTAs
    "b32_L1500_g4_many_segments": W("dec_seg", "decode", 32, 8, 2, 1500, 128, 64,
                                    rho=(0.9, 0.9), needles=(1, 1)),
    # every chunk active (near-flat routing scores): the largest number of
    # K/V blocks per split CTA the launch is sized for
    "b32_L65536_d64_dense": W("dec_dense", "decode", 32, 8, 2, 65536, 64, 64, gamma=0.001,
                              rho=(0.9, 0.9), needles=(0, 0)),
}


def _decode_case(wl, seed, diag=False):
    inp = synth.make_decode(wl, seed=seed)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16) if wl.seq >= wl.chunk else \
        torch.zeros(wl.batch, wl.n_kv_heads, 0, wl.head_dim, dtype=torch.bfloat16)
    p = dash.problem_for(wl, estimate_diagonal=diag)
    out = dash.decode(p, inp["q"].cuda(), inp["K"].cuda(), inp["V"].cuda(), kb.cuda(),
                      qbar=inp["qbar"].cuda())
    assert dash.dash_get_error() == dash.DASH_OK
    ref = oracle.decode(inp["q"], inp["K"], inp["V"], kb, wl.seq, wl.alpha, wl.gamma, wl.sigma,
                        wl.chunk, qbar=inp["qbar"] if diag else None)
    return out, ref, inp, kb


@pytest.mark.parametrize("name", list(DEC))
def test_decode_matches_oracle(name):
    wl = DEC[name]
    out, ref, inp, kb = _decode_case(wl, seed=12)
    if name.endswith("_dense"):                    # the case must really be dense
        assert (np64(out["w"])[..., : (wl.seq - 1) // wl.chunk] > 0).all()
    _check_decode(wl, out, ref, inp["q"], inp["K"], inp["V"], None)


@pytest.mark.parametrize("name", ["b2_L1000_ragged", "b3_L64_first_chunk", "b1_L4097_b128_g8",
                                  "b4_L3000_d64_g4", "b2_L2000_alpha13",
                                  "b2_L5000_b128_sparsemax_sigma0"])
def test_decode_estimate_diagonal_matches_oracle(name):
    wl = DEC[name]
    out, ref, inp, kb = _decode_case(wl, seed=34, diag=True)
    _check_decode(wl, out, ref, inp["q"], inp["K"], inp["V"], None)


def test_decode_full_size():
    wl = configs.DECODE_128K
    out, ref, inp, kb = _decode_case(wl, seed=0)
    _check_decode(wl, out, ref, inp["q"], inp["K"], inp["V"], None)


def test_decode_equals_prefill_last_row_on_gpu():
    # the same data through the prefill kernels and through the decode kernels
    wl = MED["g16_d128_b64_nc37"]
    inp = synth.make_prefill(wl, seed=13)
    p = dash.problem_for(wl)
    dev = {k: inp[k].cuda() for k in ("Q", "K", "V", "qbar")}
    out = dash.prefill(p, dev["Q"], dev["K"], dev["V"], dev["qbar"])
    pd = dash.problem_for(wl.with_(kind="decode"))
    dec = dash.decode(pd, dev["Q"][:, :, -1].contiguous(), dev["K"], dev["V"], out["Kbar"])
    torch.cuda.synchronize()
    assert torch.equal(dec["mask"], out["mask"][:, :, -1])
    assert (dec["w"] - out["w"][:, :, -1]).abs().max().item() <= 1e-5
    assert (dec["o"].float() - out["O"][:, :, -1].float()).abs().max().item() <= TOL_O_BF16


# ----------------------------------------------------------------------------
# decode with a cache length per sequence
# ----------------------------------------------------------------------------

DECV = {
    # one token (no complete chunk, a one-key diagonal), exactly one chunk (the
    # query's own chunk is chunk 0), one token past it, ragged, full, full - 1
    "b6_Lmax1000_edges": (W("decv_edges", "decode", 6, 32, 2, 1000, 128, 64, gamma=0.3,
                            rho=(0.9, 0.9), needles=(2, 2)), [1000, 1, 64, 65, 513, 999]),
    "b4_Lmax4097_b128_g8": (W("decv_b128", "decode", 4, 16, 2, 4097, 128, 128, gamma=0.5, sigma=0.5,
                              rho=(0.9, 0.5), needles=(2, 1)), [4097, 128, 129, 2000]),
    # seeded lengths (uniform in [30, 3000])
    "b8_Lmax3000_d64_g4_seeded": (W("decv_d64", "decode", 8, 8, 2, 3000, 64, 64, rho=(0.9, 0.5),
                                    needles=(2, 1), min_len_frac=0.01), None),
}


def _decode_varlen_case(wl, lens, seed, diag=False):
    inp = synth.make_decode(wl, seed=seed)
    lens = inp["lens"] if lens is None else torch.tensor(lens, dtype=torch.int32)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16)
    p = dash.problem_for(wl, estimate_diagonal=diag)
    out = dash.decode(p, inp["q"].cuda(), inp["K"].cuda(), inp["V"].cuda(), kb.cuda(),
                      cache_lens=lens.cuda(), qbar=inp["qbar"].cuda())
    assert dash.dash_get_error() == dash.DASH_OK
    ref = oracle.decode_varlen(inp["q"], inp["K"], inp["V"], kb, lens.tolist(), wl.alpha, wl.gamma,
                               wl.sigma, wl.chunk, qbar=inp["qbar"] if diag else None)
    return out, ref, lens, inp


def _check_decode(wl, out, ref, q, Kc, Vc, lens):
    """Every output of a decode call against the oracle.

    Routing (D0): the mask bit-exact except at chunks where some head's score
    lies within 1e-4 of its threshold (counted and printed), w within 1e-3.
    Attention (D1 + D2): o and lse of every (sequence, KV head), against the
    oracle's stage 2 run on the kernel's own w and mask, so that a legitimate
    flip at the threshold cannot hide or excuse an attention error.  Where the
    whole mask of a (sequence, KV head) equals the oracle's, o is also checked
    against the oracle's own end-to-end result.
    """
    o, lse, w, mask, near = ref
    gm = mask_from_dev(out["mask"])
    n_diff, n_bad = compare_masks(gm, mask, near, wl.n_chunks)
    print(f"near-threshold mask flips: {n_diff}")
    assert n_bad == 0, f"{n_bad} mask bits differ away from tau ({n_diff} total)"
    wg = np64(out["w"])
    assert np.abs(wg - w).max() <= TOL_W
    o_iso, lse_iso = oracle.decode_attend(q, Kc, Vc, wg, gm, lens, wl.sigma, wl.chunk)
    assert np.abs(np64(out["o"]) - o_iso).max() <= TOL_O_BF16
    assert np.abs(np64(out["lse"]) - lse_iso).max() <= TOL_LSE
    same = np.repeat(np.all(gm == mask, axis=-1), wl.group, axis=1)        # [b, h_q]
    assert np.where(same[..., None], np.abs(np64(out["o"]) - o), 0).max() <= TOL_O_BF16


@pytest.mark.parametrize("name", list(DECV))
def test_decode_varlen_matches_oracle(name):
    wl, lens = DECV[name]
    out, ref, lens, inp = _decode_varlen_case(wl, lens, seed=14)
    _check_decode(wl, out, ref, inp["q"], inp["K"], inp["V"], lens.tolist())


@pytest.mark.parametrize("name", list(DECV))
def test_decode_varlen_estimate_diagonal_matches_oracle(name):
    wl, lens = DECV[name]
    out, ref, lens, inp = _decode_varlen_case(wl, lens, seed=35, diag=True)
    _check_decode(wl, out, ref, inp["q"], inp["K"], inp["V"], lens.tolist())


def test_decode_varlen_full_size():
    wl = configs.DECODE_VARLEN_128K
    out, ref, lens, inp = _decode_varlen_case(wl, None, seed=0)
    assert lens.min().item() >= wl.seq // 8 and lens.max().item() <= wl.seq
    _check_decode(wl, out, ref, inp["q"], inp["K"], inp["V"], lens.tolist())


def test_decode_varlen_reads_nothing_past_each_length():
    wl, lens = DECV["b6_Lmax1000_edges"]
    inp = synth.make_decode(wl, seed=15)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16).cuda()
    q, K, V = inp["q"].cuda(), inp["K"].cuda(), inp["V"].cuda()
    dl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = dash.problem_for(wl)
    a = dash.decode(p, q, K, V, kb, cache_lens=dl)
    K2, V2, kb2 = K.clone(), V.clone(), kb.clone()
    for bi, L in enumerate(lens):
        K2[bi, :, L:] = 30.0
        V2[bi, :, L:] = -30.0
        kb2[bi, :, (L - 1) // wl.chunk:] = 30.0
    b = dash.decode(p, q, K2, V2, kb2, cache_lens=dl)
    torch.cuda.synchronize()
    assert dash.dash_get_error() == dash.DASH_OK
    for k in ("o", "lse", "w", "mask"):
        assert torch.equal(a[k], b[k]), k


def test_decode_varlen_equal_lengths_is_decode():
    wl = DEC["b2_L1000_ragged"]
    inp = synth.make_decode(wl, seed=16)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16).cuda()
    q, K, V = inp["q"].cuda(), inp["K"].cuda(), inp["V"].cuda()
    p = dash.problem_for(wl)
    a = dash.decode(p, q, K, V, kb)
    b = dash.decode(p, q, K, V, kb,
                    cache_lens=torch.full((wl.batch,), wl.seq, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    for k in ("o", "lse", "w", "mask"):
        assert torch.equal(a[k], b[k]), k


def test_decode_varlen_length_out_of_range_is_reported():
    # lengths are read on the device: out-of-range ones are clamped (every
    # access stays inside the caches) and reported by dash_get_error
    wl = DEC["b2_L1000_ragged"]
    inp = synth.make_decode(wl, seed=17)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16).cuda()
    q, K, V = inp["q"].cuda(), inp["K"].cuda(), inp["V"].cuda()
    p = dash.problem_for(wl)
    for bad in ([0, 5], [5, wl.seq + 7]):
        dash.decode(p, q, K, V, kb, cache_lens=torch.tensor(bad, dtype=torch.int32, device="cuda"))
        assert dash.dash_get_error() == dash.DASH_ERR_INVALID_ARG
    dash.decode(p, q, K, V, kb, cache_lens=torch.tensor([5, 900], dtype=torch.int32, device="cuda"))
    assert dash.dash_get_error() == dash.DASH_OK


# ----------------------------------------------------------------------------
# decode over paged caches
# ----------------------------------------------------------------------------

def _decode_paged_case(wl, lens, seed, extra_pages=7, diag=False):
    inp = synth.make_decode(wl, seed=seed)
    lens = inp["lens"] if lens is None else torch.tensor(lens, dtype=torch.int32)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16)
    Kp, Vp, table = synth.to_pages(inp["K"], inp["V"], lens.tolist(), wl.chunk, seed=seed,
                                   extra_pages=extra_pages)
    p = dash.problem_for(wl, estimate_diagonal=diag)
    out = dash.decode(p, inp["q"].cuda(), Kp.cuda(), Vp.cuda(), kb.cuda(), cache_lens=lens.cuda(),
                      page_table=table.cuda(), qbar=inp["qbar"].cuda())
    assert dash.dash_get_error() == dash.DASH_OK
    ref = oracle.decode_paged(inp["q"], Kp, Vp, kb, lens.tolist(), table.numpy(), wl.alpha,
                              wl.gamma, wl.sigma, wl.chunk, qbar=inp["qbar"] if diag else None)
    Kc, Vc = oracle.gather_pages(Kp, Vp, lens.tolist(), table.numpy(), wl.chunk)
    return out, ref, (inp["q"], Kc, Vc, lens.tolist())


@pytest.mark.parametrize("name", list(DECV))
def test_decode_paged_matches_oracle(name):
    wl, lens = DECV[name]
    out, ref, (q, Kc, Vc, lens) = _decode_paged_case(wl, lens, seed=18)
    _check_decode(wl, out, ref, q, Kc, Vc, lens)


@pytest.mark.parametrize("name", list(DECV))
def test_decode_paged_estimate_diagonal_matches_oracle(name):
    wl, lens = DECV[name]
    out, ref, (q, Kc, Vc, lens) = _decode_paged_case(wl, lens, seed=36, diag=True)
    _check_decode(wl, out, ref, q, Kc, Vc, lens)


def test_decode_paged_full_size_equals_varlen():
    # the full-size varlen decode is checked against the oracle above; the
    # same data through shuffled pages must give the same bits
    wl = configs.DECODE_PAGED_128K
    inp = synth.make_decode(wl, seed=0, device="cuda")
    lens = inp["lens"]
    p = dash.problem_for(wl)
    kb = torch.empty(wl.batch, wl.n_kv_heads, wl.seq // wl.chunk, wl.head_dim, dtype=torch.bfloat16,
                     device="cuda")
    dash.dash_summarize(p, inp["K"], inp["qbar"], kb)
    a = dash.decode(p, inp["q"], inp["K"], inp["V"], kb, cache_lens=lens)
    Kp, Vp, table = synth.to_pages(inp["K"], inp["V"], lens.tolist(), wl.chunk, seed=0,
                                   extra_pages=64)
    del inp["K"], inp["V"]
    b = dash.decode(p, inp["q"], Kp, Vp, kb, cache_lens=lens, page_table=table)
    torch.cuda.synchronize()
    assert dash.dash_get_error() == dash.DASH_OK
    for k in ("o", "lse", "w", "mask"):
        assert torch.equal(a[k], b[k]), k
    del Kp, Vp
    torch.cuda.empty_cache()


def test_decode_paged_page_id_out_of_range_is_reported():
    wl, lens = DECV["b6_Lmax1000_edges"]
    inp = synth.make_decode(wl, seed=19)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16).cuda()
    Kp, Vp, table = synth.to_pages(inp["K"], inp["V"], lens, wl.chunk, seed=19)
    p = dash.problem_for(wl)
    dl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for bad in (-1, Kp.shape[0]):
        t = table.clone()
        t[0, 0] = bad                                  # chunk 0 of a 1000-token sequence: read
        dash.decode(p, inp["q"].cuda(), Kp.cuda(), Vp.cuda(), kb, cache_lens=dl, page_table=t.cuda())
        assert dash.dash_get_error() == dash.DASH_ERR_INVALID_ARG
    dash.decode(p, inp["q"].cuda(), Kp.cuda(), Vp.cuda(), kb, cache_lens=dl, page_table=table.cuda())
    assert dash.dash_get_error() == dash.DASH_OK


# ----------------------------------------------------------------------------
# summary-cache append and an incremental decode loop
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_summarize_append_gives_the_bits_of_summarize(dtype, d):
    wl = W("app", "decode", 5, 8, 2, 640, d, 64, dtype=dtype)
    dt = synth.torch_dtype(dtype)
    g = torch.Generator().manual_seed(21)
    K = torch.randn(5, 2, 640, d, generator=g).to(dt).cuda()
    qbar = (torch.randn(2, d, generator=g) * 0.3).cuda()
    p = dash.problem_for(wl)
    full = torch.empty(5, 2, 10, d, dtype=dt, device="cuda")
    dash.dash_summarize(p, K, qbar, full)
    kb = torch.full_like(full, 7.0)
    lens = [64, 65, 640, 1, 320]                       # boundaries at 64, 640, 320
    dash.dash_summarize_append(p, torch.tensor(lens, dtype=torch.int32, device="cuda"), K, qbar, kb)
    assert dash.dash_get_error() == dash.DASH_OK
    want = torch.full_like(full, 7.0)
    for bi, L in enumerate(lens):
        if L % 64 == 0:
            want[bi, :, L // 64 - 1] = full[bi, :, L // 64 - 1]
    assert torch.equal(kb, want)
    # the same from a shuffled page pool
    Kp, _, table = synth.to_pages(K, K, lens, 64, seed=21, extra_pages=3)
    kb2 = torch.full_like(full, 7.0)
    dash.dash_summarize_append(p, torch.tensor(lens, dtype=torch.int32, device="cuda"), Kp, qbar, kb2,
                               page_table=table)
    assert dash.dash_get_error() == dash.DASH_OK
    assert torch.equal(kb2, want)


def test_summarize_append_length_out_of_range_is_reported():
    wl = W("app", "decode", 2, 8, 2, 640, 128, 64)
    K = torch.zeros(2, 2, 640, 128, dtype=torch.bfloat16, device="cuda")
    qbar = torch.zeros(2, 128, device="cuda")
    kb = torch.zeros(2, 2, 10, 128, dtype=torch.bfloat16, device="cuda")
    p = dash.problem_for(wl)
    dash.dash_summarize_append(p, torch.tensor([64, 704], dtype=torch.int32, device="cuda"), K, qbar, kb)
    assert dash.dash_get_error() == dash.DASH_ERR_INVALID_ARG


def test_incremental_decode_loop():
    # three sequences grow token by token across chunk boundaries: each step
    # decodes (checked against the oracle) and then appends the summary of any
    # chunk just completed; rows of chunks not yet complete start as garbage,
    # so a missing or late append changes the next step's routing
    wl = W("dec_loop", "decode", 3, 32, 2, 256, 128, 64, gamma=0.3, rho=(0.9, 0.9), needles=(1, 1))
    inp = synth.make_decode(wl, seed=22)
    p = dash.problem_for(wl)
    K, V, qbar = inp["K"].cuda(), inp["V"].cuda(), inp["qbar"].cuda()
    kb_ref = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, torch.bfloat16)
    lens = [62, 63, 127]
    kb = torch.empty(3, 2, 4, 128, dtype=torch.bfloat16, device="cuda")
    dash.dash_summarize(p, K, qbar, kb)
    for bi, L in enumerate(lens):
        kb[bi, :, L // 64:] = 7.0                      # chunks not complete yet
    g = torch.Generator().manual_seed(23)
    for step in range(4):
        lens = [L + 1 for L in lens]
        q = torch.randn(3, 32, 128, generator=g).to(torch.bfloat16)
        dl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        out = dash.decode(p, q.cuda(), K, V, kb, cache_lens=dl)
        assert dash.dash_get_error() == dash.DASH_OK
        ref = oracle.decode_varlen(q, inp["K"], inp["V"], kb_ref, lens, wl.alpha, wl.gamma, wl.sigma,
                                   wl.chunk)
        _check_decode(wl, out, ref, q, inp["K"], inp["V"], lens)
        dash.dash_summarize_append(p, dl, K, qbar, kb)
    full = torch.empty_like(kb)
    dash.dash_summarize(p, K, qbar, full)
    torch.cuda.synchronize()
    for bi, L in enumerate(lens):                      # every complete chunk is summarised now
        assert torch.equal(kb[bi, :, :L // 64], full[bi, :, :L // 64])


# ----------------------------------------------------------------------------
# top-k routing (the fixed-budget baseline) on the same summaries
# ----------------------------------------------------------------------------

TOPK = {
    "g16_d128_b64_nc37_k5": (MED["g16_d128_b64_nc37"], 5),
    "g8_d64_b64_batch2_k3": (MED["g8_d64_b64_batch2"], 3),
    "g16_d128_b128_k40_more_than_eligible": (MED["g16_d128_b128_s05"], 40),
}


@pytest.mark.parametrize("name", list(TOPK))
def test_route_topk_matches_oracle(name):
    wl, k = TOPK[name]
    inp = synth.make_prefill(wl, seed=24)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, synth.torch_dtype(wl.dtype))
    p = dash.problem_for(wl)
    dev = dash.alloc_prefill(p, "cuda")
    dash.dash_route_topk(p, inp["Q"].cuda(), kb.cuda(), k, dev["w"], dev["mask"])
    assert dash.dash_get_error() == dash.DASH_OK
    pos = np.unique(np.concatenate([np.arange(0, wl.seq, 7), [wl.seq - 1]]))
    w_ref, _, score = oracle.route_topk(inp["Q"], kb, k, wl.gamma, wl.chunk, positions=pos)
    wg = np64(dev["w"])[:, :, pos]
    gm = mask_from_dev(dev["mask"])[:, :, pos]
    n_c = wl.n_chunks
    for bi in range(wl.batch):
        for g in range(wl.n_kv_heads):
            for j, i in enumerate(pos):
                ne = min(i // wl.chunk, n_c)
                sel = np.nonzero(wg[bi, g, j])[0]
                assert (oracle.unpack_mask(gm[bi, g, j], n_c) == (wg[bi, g, j] > 0)).all()
                if ne == 0:
                    assert sel.size == 0
                    continue
                kk = min(k, ne)
                assert sel.size == kk and sel.max() < ne
                np.testing.assert_allclose(wg[bi, g, j, sel], 1.0 / kk, rtol=1e-6)
                # a valid top-k of the oracle's scores (fp32 scores may order
                # near-ties differently): nothing left out beats the k-th best
                # by more than the tolerance, nothing taken falls below it
                sc = score[bi, g, j, :ne]
                kth = np.sort(sc)[::-1][kk - 1]
                out_ = np.setdiff1d(np.arange(ne), sel)
                # fp32 logits (|z| up to ~50 with the needles) carry ~1e-4
                # relative error into the scores
                tol = 5e-4 * kth + 1e-12
                assert sc[sel].min() >= kth - tol
                if out_.size:
                    assert sc[out_].max() <= kth + tol
                # where the oracle's k-th and (k+1)-th scores are apart, the
                # choice is unique and both sides make it
                srt = np.sort(sc)[::-1]
                if kk == ne or srt[kk - 1] - srt[kk] > tol:
                    assert (np.nonzero(w_ref[bi, g, j])[0] == sel).all()


def test_attention_on_topk_mask_matches_oracle():
    # the fixed-budget hierarchy: top-k mask, sigma = 0, the same stage-2 kernel
    wl, k = TOPK["g16_d128_b64_nc37_k5"]
    inp = synth.make_prefill(wl, seed=25)
    p = dash.problem_for(wl, sigma=0.0)
    dev = {n: inp[n].cuda() for n in ("Q", "K", "V", "qbar")}
    out = dash.alloc_prefill(p, "cuda")
    dash.dash_summarize(p, dev["K"], dev["qbar"], out["Kbar"])
    dash.dash_route_topk(p, dev["Q"], out["Kbar"], k, out["w"], out["mask"])
    dash.dash_attn_fwd(p, dev["Q"], dev["K"], dev["V"], out["w"], out["mask"], out["O"], out["lse"])
    assert dash.dash_get_error() == dash.DASH_OK
    pos = np.arange(0, wl.seq, 11)
    w = np64(out["w"])
    m = mask_from_dev(out["mask"])
    O, lse = oracle.attn_fwd(inp["Q"], inp["K"], inp["V"], w[:, :, pos], m[:, :, pos], 0.0, wl.chunk,
                             positions=pos)
    assert np.abs(np64(out["O"])[:, :, pos] - O).max() <= TOL_O_BF16
    assert np.abs(np64(out["lse"])[:, :, pos] - lse).max() <= TOL_LSE
    # exactly k routed chunks per row once k are eligible (the fixed budget)
    cnt = oracle.unpack_mask(m, wl.n_chunks).sum(-1)                   # [b, h_kv, N]
    elig = np.minimum(np.arange(wl.seq) // wl.chunk, wl.n_chunks)
    assert (cnt == np.minimum(elig, k)).all()


# ----------------------------------------------------------------------------
# stage 2 backward
# ----------------------------------------------------------------------------

BWD = {
    # CUDA-core reference kernel
    "tiny_f32": (configs.TINY_F32, 1e-4),
    "g8_d64_b64_batch2": (MED["g8_d64_b64_batch2"], 2e-2),
    # tcgen05 kernels: an odd chunk count (a half key block at the end), 128-key
    # chunks with sigma = 0.5, G = 4 with sigma = 0 (no dw), G = 8 over two
    # sequences
    "g16_d128_b64_nc37": (MED["g16_d128_b64_nc37"], 2e-2),
    "g16_d128_b128_s05": (MED["g16_d128_b128_s05"], 2e-2),
    "g4_d128_sigma0": (MED["g4_d128_sigma0"], 2e-2),
    "g8_d128_b128_batch2": (W("med_g8_d128", "prefill", 2, 16, 2, 12 * 128, 128, 128, sigma=1.0,
                              rho=(0.9, 0.5), needles=(2, 1)), 2e-2),
}


@pytest.mark.parametrize("name", list(BWD))
def test_attn_bwd_matches_oracle(name):
    from oracle import dash_oracle_bwd as obwd
    wl, tol = BWD[name]
    inp = synth.make_prefill(wl, seed=26)
    p = dash.problem_for(wl)
    dt = synth.torch_dtype(wl.dtype)
    dev = {n: inp[n].cuda() for n in ("Q", "K", "V", "qbar")}
    out = dash.prefill(p, dev["Q"], dev["K"], dev["V"], dev["qbar"])
    dO = torch.randn(dev["Q"].shape, generator=torch.Generator().manual_seed(27)).to(dt)
    f32 = dict(dtype=torch.float32, device="cuda")
    dQ = torch.empty(dev["Q"].shape, **f32)
    dK = torch.full(dev["K"].shape, 5.0, **f32)      # zeroed by the call
    dV = torch.full(dev["V"].shape, 5.0, **f32)
    dw = torch.full(out["w"].shape, 5.0, **f32)
    dash.dash_attn_bwd(p, dev["Q"], dev["K"], dev["V"], out["w"], out["mask"], out["O"], out["lse"],
                       dO.cuda(), dQ, dK, dV, dw)
    assert dash.dash_get_error() == dash.DASH_OK
    ref = obwd.attn_bwd(inp["Q"], inp["K"], inp["V"], np64(out["w"]), mask_from_dev(out["mask"]),
                        wl.sigma, wl.chunk, dO)
    for got, want, nm in zip((dQ, dK, dV, dw), ref, ("dQ", "dK", "dV", "dw")):
        g = np64(got)
        err = np.abs(g - want).max() / max(np.abs(want).max(), 1e-30)
        assert err <= tol, (nm, err)
    # dw lives only on the active routed blocks
    act = oracle.unpack_mask(mask_from_dev(out["mask"]), wl.n_chunks)
    assert not np64(dw)[~act].any()


@pytest.mark.parametrize("split", [1, 3])
def test_attn_bwd_tc_split_counts(split):
    # the key-major kernel with each key block's tiles in one CTA (dK, dV
    # written directly, as for long sequences) and split over three (partial
    # rows summed by the reduction), on the same inputs as the oracle
    from oracle import dash_oracle_bwd as obwd
    wl = BWD["g16_d128_b64_nc37"][0]
    inp = synth.make_prefill(wl, seed=26)
    p = dash.problem_for(wl)
    dev = {n: inp[n].cuda() for n in ("Q", "K", "V", "qbar")}
    out = dash.prefill(p, dev["Q"], dev["K"], dev["V"], dev["qbar"])
    dO = torch.randn(dev["Q"].shape, generator=torch.Generator().manual_seed(27)).to(torch.bfloat16)
    f32 = dict(dtype=torch.float32, device="cuda")
    g = [torch.full(dev["Q"].shape, 5.0, **f32), torch.full(dev["K"].shape, 5.0, **f32),
         torch.full(dev["V"].shape, 5.0, **f32), torch.full(out["w"].shape, 5.0, **f32)]
    prev = dash.dash_selftest_bwd_split(split)
    try:
        dash.dash_attn_bwd(p, dev["Q"], dev["K"], dev["V"], out["w"], out["mask"], out["O"],
                           out["lse"], dO.cuda(), *g)
        assert dash.dash_get_error() == dash.DASH_OK
    finally:
        dash.dash_selftest_bwd_split(prev)
    ref = obwd.attn_bwd(inp["Q"], inp["K"], inp["V"], np64(out["w"]), mask_from_dev(out["mask"]),
                        wl.sigma, wl.chunk, dO)
    for got, want, nm in zip(g, ref, ("dQ", "dK", "dV", "dw")):
        err = np.abs(np64(got) - want).max() / max(np.abs(want).max(), 1e-30)
        assert err <= 2e-2, (nm, split, err)


def test_attn_bwd_tc_is_deterministic():
    # every output element is written once, in a fixed order: two calls agree bit for bit
    wl = BWD["g16_d128_b64_nc37"][0]
    inp = synth.make_prefill(wl, seed=32)
    p = dash.problem_for(wl)
    assert dash.dash_workspace_bytes(p, 2) > 0
    dev = {n: inp[n].cuda() for n in ("Q", "K", "V", "qbar")}
    out = dash.prefill(p, dev["Q"], dev["K"], dev["V"], dev["qbar"])
    dO = torch.randn(dev["Q"].shape, generator=torch.Generator().manual_seed(33)).to(torch.bfloat16).cuda()
    f32 = dict(dtype=torch.float32, device="cuda")
    res = []
    for _ in range(2):
        g = [torch.empty(dev["Q"].shape, **f32), torch.empty(dev["K"].shape, **f32),
             torch.empty(dev["V"].shape, **f32), torch.empty(out["w"].shape, **f32)]
        dash.dash_attn_bwd(p, dev["Q"], dev["K"], dev["V"], out["w"], out["mask"], out["O"], out["lse"],
                           dO, *g)
        res.append(g)
    assert dash.dash_get_error() == dash.DASH_OK
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_attn_bwd_workspace_checked():
    wl = BWD["g16_d128_b64_nc37"][0]
    p = dash.problem_for(wl)
    need = dash.dash_workspace_bytes(p, 2)
    Q = torch.zeros(wl.batch, wl.n_q_heads, wl.seq, wl.head_dim, dtype=torch.bfloat16, device="cuda")
    K = torch.zeros(wl.batch, wl.n_kv_heads, wl.seq, wl.head_dim, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(wl.batch, wl.n_kv_heads, wl.seq, wl.n_chunks, device="cuda")
    m = torch.zeros(wl.batch, wl.n_kv_heads, wl.seq, (wl.n_chunks + 31) // 32, dtype=torch.int32, device="cuda")
    lse = torch.zeros(wl.batch, wl.n_q_heads, wl.seq, device="cuda")
    dQ, dK = Q.float(), K.float()
    short = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="DASH_ERR_WORKSPACE"):
        dash.dash_attn_bwd(p, Q, K, K, w, m, Q, lse, Q, dQ, dK, dK.clone(), workspace=short)


def test_attn_bwd_full_size_8k():
    # the bench's backward workload (8k, G = 16, 64-key chunks) in the same
    # launch: dQ and dw of sampled positions against the oracle row by row;
    # dK and dV through identities that hold at any size -- summed over the
    # keys, dV equals the group's dO summed over its rows (each row's p sums
    # to 1) and dK vanishes (each row's ds sums to 0)
    from oracle import dash_oracle_bwd as obwd
    wl = configs.PREFILL_8K
    inp = synth.make_prefill(wl, seed=34, device="cuda")
    p = dash.problem_for(wl)
    out = dash.prefill(p, inp["Q"], inp["K"], inp["V"], inp["qbar"])
    dO = torch.randn(inp["Q"].shape, generator=torch.Generator(device="cuda").manual_seed(35),
                     device="cuda").to(torch.bfloat16)
    f32 = dict(dtype=torch.float32, device="cuda")
    dQ, dK, dV = (torch.empty(inp[n].shape, **f32) for n in ("Q", "K", "V"))
    dw = torch.empty(out["w"].shape, **f32)
    dash.dash_attn_bwd(p, inp["Q"], inp["K"], inp["V"], out["w"], out["mask"], out["O"], out["lse"],
                       dO, dQ, dK, dV, dw)
    assert dash.dash_get_error() == dash.DASH_OK
    pos = np.sort(np.random.default_rng(36).choice(wl.seq, 48, replace=False))
    pos = np.unique(np.concatenate([pos, [0, 63, 64, wl.seq - 1]]))
    m = mask_from_dev(out["mask"])[:, :, pos]
    w = np64(out["w"])[:, :, pos]
    dO64 = np64(dO)
    rq, _, _, rdw = obwd.attn_bwd(np64(inp["Q"]), np64(inp["K"]), np64(inp["V"]), w, m, wl.sigma,
                                  wl.chunk, dO64[:, :, pos], positions=pos)
    gq = np64(dQ)[:, :, pos]
    assert np.abs(gq - rq[:, :, pos]).max() / np.abs(rq[:, :, pos]).max() <= 2e-2
    gdw = np64(dw)[:, :, pos]
    assert np.abs(gdw - rdw).max() / max(np.abs(rdw).max(), 1e-30) <= 2e-2
    G = wl.n_q_heads // wl.n_kv_heads
    want_v = dO64.reshape(wl.batch, wl.n_kv_heads, G * wl.seq, wl.head_dim).sum(axis=2)
    got_v = np64(dV).sum(axis=2)
    assert np.abs(got_v - want_v).max() <= 2e-2 * np.abs(want_v).max()
    # dK: the row sums of ds vanish up to O's bf16 rounding in D = dO . O
    got_k = np.abs(np64(dK).sum(axis=2)).max()
    assert got_k <= 2e-2 * np.abs(np64(dK)).sum(axis=2).max()
    assert np.isfinite(np64(dK)).all() and np.isfinite(np64(dV)).all()


RBWD = {
    "tiny_f32": (configs.TINY_F32, 1e-3),
    "g8_d64_b64_batch2": (MED["g8_d64_b64_batch2"], 1e-3),
    "g16_d128_b64_nc37": (MED["g16_d128_b64_nc37"], 1e-3),
}


@pytest.mark.parametrize("name", list(RBWD))
def test_route_and_summarize_bwd_match_oracle(name):
    from oracle import dash_oracle_bwd as obwd
    wl, tol = RBWD[name]
    inp = synth.make_prefill(wl, seed=28)
    dt = synth.torch_dtype(wl.dtype)
    p = dash.problem_for(wl)
    kb = oracle_kbar(inp["K"], inp["qbar"], wl.chunk, dt)
    g = torch.Generator().manual_seed(29)
    dw = torch.randn(wl.batch, wl.n_kv_heads, wl.seq, wl.n_chunks, generator=g)
    dKbar = torch.randn(kb.shape, generator=g)
    f32 = dict(dtype=torch.float32, device="cuda")
    dQ = torch.zeros(inp["Q"].shape, **f32)
    dKb = torch.zeros(kb.shape, **f32)
    dash.dash_route_bwd(p, inp["Q"].cuda(), kb.cuda(), dw.cuda(), dQ, dKb)
    dK = torch.zeros(inp["K"].shape, **f32)
    dqb = torch.zeros(inp["qbar"].shape, **f32)
    dash.dash_summarize_bwd(p, inp["K"].cuda(), inp["qbar"].cuda(), dKbar.cuda(), dK, dqb)
    assert dash.dash_get_error() == dash.DASH_OK
    rq, rkb = obwd.route_bwd(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk, dw)
    rk, rqb = obwd.summary_bwd(inp["K"], inp["qbar"], wl.chunk, dKbar)
    for got, want, nm in ((dQ, rq, "dQ"), (dKb, rkb, "dKbar"), (dK, rk, "dK"), (dqb, rqb, "dqbar")):
        err = np.abs(np64(got) - want).max() / max(np.abs(want).max(), 1e-30)
        assert err <= tol, (nm, err)


@pytest.mark.parametrize("name,tol", [("tiny_f32", 1e-3), ("g8_d64_b64_batch2", 3e-2)])
def test_full_backward_matches_oracle(name, tol):
    # dO -> stage 2 -> dw -> stage 1 -> dKbar -> stage 0, all on the GPU,
    # against the oracle's stages composed on the same routing
    from oracle import dash_oracle_bwd as obwd
    wl = RBWD[name][0]
    inp = synth.make_prefill(wl, seed=30)
    dt = synth.torch_dtype(wl.dtype)
    p = dash.problem_for(wl)
    dev = {n: inp[n].cuda() for n in ("Q", "K", "V", "qbar")}
    out = dash.prefill(p, dev["Q"], dev["K"], dev["V"], dev["qbar"])
    dO = torch.randn(dev["Q"].shape, generator=torch.Generator().manual_seed(31)).to(dt)
    gr = dash.backward(p, dev["Q"], dev["K"], dev["V"], dev["qbar"], out, dO.cuda())
    assert dash.dash_get_error() == dash.DASH_OK
    w, m = np64(out["w"]), mask_from_dev(out["mask"])
    kb = np64(out["Kbar"])
    q2, k2, v2, dwr = obwd.attn_bwd(inp["Q"], inp["K"], inp["V"], w, m, wl.sigma, wl.chunk, dO)
    q1, dkb = obwd.route_bwd(inp["Q"], kb, wl.alpha, wl.gamma, wl.chunk, dwr)
    k0, dqb = obwd.summary_bwd(inp["K"], inp["qbar"], wl.chunk, dkb)
    for nm, want in (("dQ", q2 + q1), ("dK", k2 + k0), ("dV", v2), ("dqbar", dqb)):
        err = np.abs(np64(gr[nm]) - want).max() / max(np.abs(want).max(), 1e-30)
        assert err <= tol, (nm, err)


def test_no_device_error_after_suite():
    assert dash.dash_get_error() == dash.DASH_OK
