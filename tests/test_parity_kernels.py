"""GPU parity of the three kernel-level C-ABI calls against the CPU oracle, on the
seeded workloads (tiny fp32; Llama-3-8B shapes at 1 and 32 requests; Qwen-32B
shapes at 128 requests, sampled), plus the invariants the method fixes: paged
in-place reads equal any page placement, the split count does not matter, requests
are independent, and bad page ids / context lengths are reported, not read.

H-Spec (arXiv 2609.24197) Abstract: attention reuses target KVs in place; Mamba
modules start from projected last-token hidden states; the parallel scan keeps the
block parallel.
"""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_attention_b200 import inputs as I
from tests.parity_util import (BF16_TOL, assert_close, assert_close_stored_bf16, assert_close_stored_bf16_edge,
                               half_ulp_bf16, host, rel_max, rel_rms,
                               sample_requests, sub_cache, to_np)

pytestmark = pytest.mark.gpu

KERNEL_WORKLOADS = ["tiny", "llama_c1", "llama_c32", "qwen_c128"]


@pytest.fixture(scope="module")
def H(cuda):
    from hybrid_mamba_attention_b200 import hspec
    return hspec


def cfg_for(H, sh, **kw):
    return H.make_cfg(sh, **kw)


# ------------------------------------------------------------------ inject

@pytest.mark.parametrize("name", KERNEL_WORKLOADS)
def test_inject_state_matches_oracle(H, cuda, name):
    wl = I.WORKLOADS[name]
    sh = wl.shapes
    inp = I.make_inject_inputs(sh, wl.C, wl.seed, cuda)
    h0 = torch.empty(wl.C, sh.H * sh.P * sh.N, device=cuda)
    H.hspec_inject_state(cfg_for(H, sh), inp["W_inj"], inp["h_last"], h0)
    assert H.hspec_sync_status() == 0
    rows = sample_requests(wl.C, 2, seed=wl.seed)
    ref = oracle.inject(host(inp["W_inj"]), host(inp["h_last"])[rows])
    assert_close(to_np(h0[rows]), ref, "f32", f"inject {name}")


@pytest.mark.parametrize("C,d,HPN", [(3, 200, 3 * 1000), (130, 64, 520), (1, 8, 8)])
def test_inject_ragged_tiles(H, cuda, C, d, HPN):
    # M, N and K all off the 128 / 256 / 64 tile grid (TMA zero-fills the edges)
    sh = I.Shapes("ragged", d=d, Hq=1, Hkv=1, D=2, H=1, P=HPN, N=1, dtype="bf16", rope_theta=1e4)
    g = torch.Generator(device=cuda).manual_seed(9)
    W = torch.randn(HPN, d, device=cuda, generator=g).to(torch.bfloat16)
    h = torch.randn(C, d, device=cuda, generator=g).to(torch.bfloat16)
    h0 = torch.full((C, HPN), float("nan"), device=cuda)
    H.hspec_inject_state(cfg_for(H, sh), W, h, h0)
    assert H.hspec_sync_status() == 0
    assert_close(to_np(h0), oracle.inject(host(W), host(h)), "f32", "inject ragged")


# --------------------------------------------------------------------- SSD

def run_ssd(H, sh, inp, K, chunk=0, want_state=False, h0=True):
    C = inp["x"].shape[0]
    y = torch.empty(C, K, sh.H, sh.P, device=inp["x"].device)
    hK = torch.empty(C, sh.H, sh.P, sh.N, device=y.device) if want_state else None
    H.hspec_ssd_block_scan(cfg_for(H, sh, ssd_chunk=chunk), inp["x"], inp["dt"], inp["A"], inp["B"], inp["Cm"],
                           inp["D"], inp["h0"] if h0 else None, y, hK)
    assert H.hspec_sync_status() == 0
    return y, hK


@pytest.mark.parametrize("name", KERNEL_WORKLOADS)
def test_ssd_scan_matches_sequential_recurrence(H, cuda, name):
    wl = I.WORKLOADS[name]
    sh = wl.shapes
    C = min(wl.C, 8)
    inp = I.make_ssd_inputs(sh, C, wl.K, wl.seed, cuda)
    y, hK = run_ssd(H, sh, inp, wl.K, want_state=True)
    ref_y, ref_h = oracle.ssd_scan(host(inp["x"]), host(inp["dt"]), host(inp["A"]), host(inp["B"]),
                                   host(inp["Cm"]), host(inp["D"]), host(inp["h0"]), want_state=True)
    assert_close(to_np(y), ref_y, "f32", f"ssd y {name}")
    assert_close(to_np(hK), ref_h, "f32", f"ssd hK {name}")


@pytest.mark.parametrize("name,C,K", [("llama_c32", 8, 16), ("qwen_c128", 3, 16), ("llama_c32", 160, 16),
                                     ("llama_c32", 5, 7), ("qwen_c128", 2, 1), ("llama_c32", 8, 32),
                                     ("qwen_c128", 3, 24), ("llama_c32", 150, 17)])
def test_ssd_scan_readout_without_final_state(H, cuda, name, C, K):
    # One bf16 chunk of K <= 32 positions is evaluated with the state readout on the
    # tensor cores (tf32 hi + lo split of the fp32 state, N = 16 or 32 positions per
    # MMA): it must still meet the fp32 bound against the sequential recurrence.
    sh = I.WORKLOADS[name].shapes
    inp = I.make_ssd_inputs(sh, C, K, 31 + C, cuda)
    y, _ = run_ssd(H, sh, inp, K, want_state=False)
    rows = sample_requests(C, min(C, 6), seed=C)
    ref_y = oracle.ssd_scan(host(inp["x"])[rows], host(inp["dt"])[rows], host(inp["A"]), host(inp["B"])[rows],
                               host(inp["Cm"])[rows], host(inp["D"]), host(inp["h0"])[rows], want_state=False)
    assert_close(to_np(y[rows]), ref_y, "f32", f"ssd readout {name} C={C} K={K}")


@pytest.mark.parametrize("name,C,K", [("llama_c32", 6, 16), ("llama_c32", 4, 32), ("qwen_c128", 3, 21),
                                     ("llama_c32", 2, 1), ("llama_c32", 150, 16)])
def test_ssd_tensor_core_scan_with_final_state(H, cuda, name, C, K):
    # The final state hK = exp(cum_{K-1}) h0 + sum_s exp(cum_{K-1} - cum_s) dt_s x_s B_s^T,
    # written by the tensor-core kernel's transform threads from the state rows they
    # already hold, next to y: both at the fp32 bound against the recurrence.
    sh = I.WORKLOADS[name].shapes
    inp = I.make_ssd_inputs(sh, C, K, 51 + C, cuda)
    y, hK = run_ssd(H, sh, inp, K, want_state=True)
    rows = sample_requests(C, min(C, 4), seed=K)
    ref_y, ref_h = oracle.ssd_scan(host(inp["x"])[rows], host(inp["dt"])[rows], host(inp["A"]),
                                   host(inp["B"])[rows], host(inp["Cm"])[rows], host(inp["D"]),
                                   host(inp["h0"])[rows], want_state=True)
    assert_close(to_np(y[rows]), ref_y, "f32", f"ssd y {name} C={C} K={K}")
    assert_close(to_np(hK[rows]), ref_h, "f32", f"ssd hK {name} C={C} K={K}")


@pytest.mark.parametrize("K", [1, 16, 32])
def test_ssd_state_with_every_low_mantissa_bit_set(H, cuda, K):
    # The tensor-core readout takes the tf32 part of the fp32 state as the tensor core
    # reads it from shared memory and adds lo = S - (S with its 13 low mantissa bits
    # cleared) from TMEM.  That is exact only if the tensor core drops those bits (a
    # rounding tensor core would add up to 2^-10 |S| per product).  States whose 13 low
    # bits are all set make every product sensitive to it.
    sh = I.LLAMA
    inp = I.make_ssd_inputs(sh, 2, K, 61, cuda)
    bits = inp["h0"].view(torch.int32)
    inp["h0"] = (bits | 0x1FFF).view(torch.float32)
    y, _ = run_ssd(H, sh, inp, K)
    ref = oracle.ssd_scan(host(inp["x"]), host(inp["dt"]), host(inp["A"]), host(inp["B"]), host(inp["Cm"]),
                          host(inp["D"]), host(inp["h0"]), want_state=False)
    assert_close(to_np(y), ref, "f32", f"ssd low mantissa bits K={K}")


@pytest.mark.parametrize("K,chunks", [(16, (1, 4, 5, 8, 16)), (32, (8, 16, 32)), (7, (3, 7)), (1, (1,))])
def test_ssd_chunk_length_is_only_an_evaluation_order(H, cuda, K, chunks):
    sh = I.LLAMA
    inp = I.make_ssd_inputs(sh, 2, K, 11, cuda)
    ref = oracle.ssd_scan(host(inp["x"]), host(inp["dt"]), host(inp["A"]), host(inp["B"]), host(inp["Cm"]),
                          host(inp["D"]), host(inp["h0"]))
    for q in chunks:
        y, _ = run_ssd(H, sh, inp, K, chunk=q)
        assert_close(to_np(y), ref, "f32", f"ssd K={K} chunk={q}")


@pytest.mark.parametrize("name,C,K", [("llama_c32", 6, 16), ("qwen_c128", 3, 16), ("llama_c32", 4, 7)])
def test_ssd_stateless_scan_matches_zero_state_recurrence(H, cuda, name, C, K):
    # No h0, no final state, one chunk: the stateless form (no state in shared memory,
    # no readout) that the bf16 draft step runs before the injection GEMM adds the h0 term
    sh = I.WORKLOADS[name].shapes
    inp = I.make_ssd_inputs(sh, C, K, 41 + C, cuda)
    y, _ = run_ssd(H, sh, inp, K, h0=False)
    zero = torch.zeros_like(host(inp["h0"]))
    ref = oracle.ssd_scan(host(inp["x"]), host(inp["dt"]), host(inp["A"]), host(inp["B"]), host(inp["Cm"]),
                          host(inp["D"]), zero, want_state=False)
    assert_close(to_np(y), ref, "f32", f"stateless ssd {name} C={C} K={K}")


def test_ssd_zero_injection_equals_zero_state(H, cuda):
    sh = I.TINY
    inp = I.make_ssd_inputs(sh, 2, 8, 5, cuda)
    inp["h0"].zero_()
    a, _ = run_ssd(H, sh, inp, 8)
    b, _ = run_ssd(H, sh, inp, 8, h0=False)
    assert torch.equal(a, b)


# --------------------------------------------------------------- attention

def run_attn(H, sh, inp, K, split=0, causal=False):
    from dataclasses import replace
    sh2 = replace(sh, causal_block=causal)
    cfg = cfg_for(H, sh2, attn_split_tokens=split)
    C = inp["q"].shape[0]
    kv = H.kv_view(inp)
    ws = H.alloc_workspace(H.hspec_attn_workspace_size(cfg, C, K, kv.max_pages))
    out = torch.full_like(inp["q"], float("nan"))
    H.hspec_attn_paged_block(cfg, inp["q"], kv, inp["ctx_lens"], inp["k_blk"], inp["v_blk"], out, ws)
    return out


def oracle_attn(inp, rows, causal=False):
    sc = sub_cache(inp, rows)
    return oracle.attn_paged(host(inp["q"])[rows], sc["k_pool"], sc["v_pool"], sc["page_table"],
                             host(inp["ctx_lens"])[rows], host(inp["k_blk"])[rows], host(inp["v_blk"])[rows],
                             causal_block=causal)


def compare_attn(gpu, ref, sh, what, edge=False):
    # The attention output is stored in bf16.  It is compared with the oracle's exact
    # value, so the store's own rounding is part of the measured error (comparing with
    # a bf16-rounded oracle would count one-ulp rounding flips instead).  The seeded
    # workloads are held to the bf16 bound; edge-shape batches, whose storage alone
    # can miss it, to a kernel error twenty times below it (parity_util).
    if sh.dtype == "bf16":
        if edge:
            return assert_close_stored_bf16_edge(gpu, ref, what)
        return assert_close_stored_bf16(gpu, ref, what)
    return assert_close(gpu, ref, sh.dtype, what)


@pytest.mark.parametrize("name", KERNEL_WORKLOADS)
def test_paged_attention_matches_oracle(H, cuda, name):
    wl = I.WORKLOADS[name]
    sh = wl.shapes
    inp = I.make_attn_inputs(sh, wl, wl.K, wl.seed, cuda, shuffle=wl.shuffle, slack=wl.slack)
    out = run_attn(H, sh, inp, wl.K)
    assert H.hspec_sync_status() == 0
    rows = sample_requests(wl.C, 3, seed=wl.seed)
    compare_attn(to_np(out[rows]), oracle_attn(inp, rows), sh, f"attn {name}")


def test_paged_attention_causal_block(H, cuda):
    wl = I.WORKLOADS["llama_c32"]
    sh = wl.shapes
    lens = torch.tensor([0, 5, 16, 17, 700, 1024], dtype=torch.int32)
    inp = I.make_attn_inputs(sh, lens, 16, 3, cuda)
    out = run_attn(H, sh, inp, 16, causal=True)
    assert H.hspec_sync_status() == 0
    rows = list(range(len(lens)))
    compare_attn(to_np(out), oracle_attn(inp, rows, causal=True), sh, "attn causal", edge=True)


def test_page_placement_is_invisible(H, cuda):
    # the same pages stored at other pool slots (table rewritten) give bit-identical output
    wl = I.WORKLOADS["llama_c32"]
    sh = wl.shapes
    inp = I.make_attn_inputs(sh, wl, wl.K, 7, cuda)
    n = inp["k_pool"].shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(1)).to(cuda)
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(n, device=cuda)
    tbl = inp["page_table"].clone()
    m = tbl >= 0
    tbl[m] = inv[tbl[m].long()].to(torch.int32)
    moved = dict(inp, k_pool=inp["k_pool"][perm].contiguous(), v_pool=inp["v_pool"][perm].contiguous(),
                 page_table=tbl)
    a = run_attn(H, sh, inp, wl.K)
    b = run_attn(H, sh, moved, wl.K)
    assert H.hspec_sync_status() == 0
    assert torch.equal(a, b)


def test_split_count_does_not_change_the_result(H, cuda):
    wl = I.WORKLOADS["llama_c32"]
    sh = wl.shapes
    inp = I.make_attn_inputs(sh, wl, wl.K, 8, cuda)
    rows = sample_requests(wl.C, 3, seed=1)
    ref = oracle_attn(inp, rows)
    for split in (16, 64, 1024, 16384):
        out = run_attn(H, sh, inp, wl.K, split=split)
        assert H.hspec_sync_status() == 0
        compare_attn(to_np(out[rows]), ref, sh, f"attn split {split}", edge=True)


@pytest.mark.parametrize("name,split", [("qwen_c128", 0), ("llama_c32", 64), ("llama_c32", 0)])
def test_attention_repeated_calls_complete_and_agree(H, cuda, name, split):
    # Back-to-back calls (no host sync in between) run the persistent kernel's
    # pipeline under different timings each time: every call must complete (no
    # barrier wait gives up) and give bit-identical output, since the partials do
    # not depend on which SM took which work item.
    wl = I.WORKLOADS[name]
    sh = wl.shapes
    inp = I.make_attn_inputs(sh, wl, wl.K, 11, cuda, shuffle=wl.shuffle, slack=wl.slack)
    outs = [run_attn(H, sh, inp, wl.K, split=split) for _ in range(8)]
    assert H.hspec_sync_status() == 0, H.hspec_last_error()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert torch.isfinite(outs[0]).all()


@pytest.mark.parametrize("C", [1, 8])
def test_attention_few_requests_long_contexts(H, cuda, C):
    # few requests over long contexts: the schedule kernel lengthens the splits (about
    # one work item per SM) and several warps share each output row in the merge
    wl = I.full_workload(C, 16)
    sh = wl.shapes
    inp = I.make_attn_inputs(sh, wl, wl.K, wl.seed, cuda, shuffle=wl.shuffle, slack=wl.slack)
    out = run_attn(H, sh, inp, wl.K)
    again = run_attn(H, sh, inp, wl.K)
    assert H.hspec_sync_status() == 0, H.hspec_last_error()
    assert torch.equal(out, again)
    rows = sample_requests(C, 2, seed=5)
    compare_attn(to_np(out[rows]), oracle_attn(inp, rows), sh, f"attn C={C}", edge=True)


def test_request_order_permutes_output(H, cuda):
    wl = I.WORKLOADS["llama_c32"]
    sh = wl.shapes
    inp = I.make_attn_inputs(sh, wl, wl.K, 9, cuda)
    perm = torch.randperm(wl.C, generator=torch.Generator().manual_seed(2)).to(cuda)
    p = {k: (v[perm] if k in ("q", "k_blk", "v_blk", "page_table", "ctx_lens") else v) for k, v in inp.items()}
    a = run_attn(H, sh, inp, wl.K)
    b = run_attn(H, sh, p, wl.K)
    assert H.hspec_sync_status() == 0
    # The tile line follows the batch order, so a request's pieces move with the
    # permutation, and with them the running max against which P is rounded to bf16
    # and the fp32 summation order: the outputs agree to that rounding.
    # Both are stored in bf16, so one rounding flip may add an ulp of the larger value
    # (up to a few percent of rms(o) at the largest outputs); beyond that ulp they agree
    # to the bf16 bound.
    x, y = to_np(a[perm]), to_np(b)
    rms = np.sqrt((x ** 2).mean())
    beyond = np.maximum(np.abs(x - y) - 2 * half_ulp_bf16(np.maximum(np.abs(x), np.abs(y))), 0.0).max() / rms
    print(f"permuted batch: max-abs/rms {rel_rms(y, x):.3e}, beyond one bf16 ulp {beyond:.3e}")
    assert beyond <= BF16_TOL


def test_empty_context_single_token_returns_block_value(H, cuda):
    sh = I.TINY
    lens = torch.zeros(3, dtype=torch.int32)
    inp = I.make_attn_inputs(sh, lens, 1, 4, cuda, slack=0.0)
    out = run_attn(H, sh, inp, 1)
    assert H.hspec_sync_status() == 0
    G = sh.Hq // sh.Hkv
    want = inp["v_blk"].repeat_interleave(G, dim=2)
    assert rel_max(to_np(out), to_np(want)) <= 1e-6


def test_nan_slack_pages_are_never_read(H, cuda):
    wl = I.WORKLOADS["llama_c32"]
    inp = I.make_attn_inputs(wl.shapes, wl, wl.K, 10, cuda, slack=0.5)
    out = run_attn(H, wl.shapes, inp, wl.K)
    assert H.hspec_sync_status() == 0
    assert torch.isfinite(out.float()).all()


def test_bad_page_id_is_reported_not_read(H, cuda):
    wl = I.WORKLOADS["tiny"]
    inp = I.make_attn_inputs(wl.shapes, wl, wl.K, 11, cuda, shuffle=False, slack=0.0)
    inp["page_table"][0, 1] = inp["k_pool"].shape[0] + 5  # beyond the pool
    run_attn(H, wl.shapes, inp, wl.K)
    assert H.hspec_sync_status() == H.HSPEC_ERR_DEVICE_CHECK
    assert H.hspec_sync_status() == 0  # the flag is cleared once reported


def test_context_longer_than_page_table_is_reported(H, cuda):
    wl = I.WORKLOADS["tiny"]
    inp = I.make_attn_inputs(wl.shapes, wl, wl.K, 12, cuda, shuffle=False, slack=0.0)
    inp["ctx_lens"][0] = inp["page_table"].shape[1] * wl.shapes.page + 1
    run_attn(H, wl.shapes, inp, wl.K)
    assert H.hspec_sync_status() == H.HSPEC_ERR_DEVICE_CHECK


# ------------------------------------------- tensor-core attention edge shapes

@pytest.mark.parametrize("K,lens", [(1, [0, 1, 15, 16, 31, 32, 33, 63, 64, 65, 4097]), (3, [0, 7, 97, 130, 2000]),
                                    (16, [64, 96, 128, 4096, 4100, 8191])])
def test_bf16_attention_ragged_tiles(H, cuda, K, lens):
    # contexts that end inside a page, on a page, on a key tile and past a split
    sh = I.LLAMA
    lens_t = torch.tensor(lens, dtype=torch.int32)
    inp = I.make_attn_inputs(sh, lens_t, K, 21, cuda)
    out = run_attn(H, sh, inp, K)
    assert H.hspec_sync_status() == 0
    compare_attn(to_np(out), oracle_attn(inp, list(range(len(lens)))), sh, f"attn K={K}", edge=True)


def test_bf16_attention_more_than_128_query_rows(H, cuda):
    # Qwen shapes with K=32: K*G = 256 query rows per kv head -> two row blocks
    sh = I.QWEN
    lens = torch.tensor([100, 3000], dtype=torch.int32)
    inp = I.make_attn_inputs(sh, lens, 32, 22, cuda)
    out = run_attn(H, sh, inp, 32)
    assert H.hspec_sync_status() == 0
    compare_attn(to_np(out), oracle_attn(inp, [0, 1]), sh, "attn 256 rows", edge=True)


@pytest.mark.parametrize("K", [33, 40, 64])
def test_bf16_attention_block_keys_span_two_tiles(H, cuda, K):
    # K > 32: the block's own keys take two key tiles; causal masking crosses them
    sh = I.LLAMA
    lens = torch.tensor([0, 17, 1000], dtype=torch.int32)
    inp = I.make_attn_inputs(sh, lens, K, 24, cuda)
    for causal in (False, True):
        out = run_attn(H, sh, inp, K, causal=causal)
        assert H.hspec_sync_status() == 0
        compare_attn(to_np(out), oracle_attn(inp, [0, 1, 2], causal=causal), sh, f"attn K={K} causal={causal}", edge=True)


def test_bf16_attention_head_dim_64(H, cuda):
    sh = I.Shapes("d64", d=256, Hq=4, Hkv=2, D=64, H=4, P=64, N=16, dtype="bf16", rope_theta=1e4)
    lens = torch.tensor([0, 33, 700], dtype=torch.int32)
    inp = I.make_attn_inputs(sh, lens, 8, 23, cuda)
    for causal in (False, True):
        out = run_attn(H, sh, inp, 8, causal=causal)
        assert H.hspec_sync_status() == 0
        compare_attn(to_np(out), oracle_attn(inp, [0, 1, 2], causal=causal), sh, f"attn D=64 causal={causal}", edge=True)


def test_bf16_bad_page_id_is_reported(H, cuda):
    wl = I.WORKLOADS["llama_c1"]
    inp = I.make_attn_inputs(wl.shapes, wl, wl.K, 24, cuda)
    inp["page_table"][0, 3] = -7
    run_attn(H, wl.shapes, inp, wl.K)
    assert H.hspec_sync_status() == H.HSPEC_ERR_DEVICE_CHECK
    inp["page_table"][0, 3] = 0
    inp["ctx_lens"][0] = inp["page_table"].shape[1] * wl.shapes.page + 16
    run_attn(H, wl.shapes, inp, wl.K)
    assert H.hspec_sync_status() == H.HSPEC_ERR_DEVICE_CHECK
    assert H.hspec_sync_status() == 0


@pytest.mark.parametrize("dtype,P,N,K,chunk", [("f32", 20, 12, 7, 3), ("bf16", 36, 20, 16, 0),
                                               ("bf16", 64, 128, 32, 5), ("f32", 8, 4, 1, 0)])
def test_ssd_odd_shapes(H, cuda, dtype, P, N, K, chunk):
    # head dims and state sizes off the 4x4 register-block grid, ragged last chunks
    sh = I.Shapes("odd", d=64, Hq=1, Hkv=1, D=2, H=3, P=P, N=N, dtype=dtype, rope_theta=1e4)
    inp = I.make_ssd_inputs(sh, 3, K, 13, cuda)
    y, hK = run_ssd(H, sh, inp, K, chunk=chunk, want_state=True)
    ref_y, ref_h = oracle.ssd_scan(host(inp["x"]), host(inp["dt"]), host(inp["A"]), host(inp["B"]),
                                   host(inp["Cm"]), host(inp["D"]), host(inp["h0"]), want_state=True)
    assert_close(to_np(y), ref_y, "f32", f"ssd odd y P={P} N={N}")
    assert_close(to_np(hK), ref_h, "f32", f"ssd odd hK P={P} N={N}")
