"""The bounded waits of the tensor-core kernels (GPU).

Every pipeline wait of the tcgen05 kernels (an mbarrier phase or a tile counter)
gives up after hspec_cfg.wait_limit_ns, sets bit 8 of the device error word and lets
the kernel finish; before a CTA exits it still waits, with the full 2 s limit, for
its own TMA copies and MMAs in flight, then frees its TMEM.  These tests make the
waits run out -- a 1 ns limit, which no wait for a copy from HBM meets -- and check
that the call reports HSPEC_ERR_DEVICE_CHECK with the timeout bit, that the context
stays usable, and that the next call with the default limit gives the same output as
before, bit for bit.  No kernel is broken and nothing faults: the limit is an ordinary
argument of every call.
"""
from dataclasses import replace

import pytest
import torch

from hybrid_mamba_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu

TINY_LIMIT_NS = 1


@pytest.fixture(scope="module")
def H(cuda):
    from hybrid_mamba_attention_b200 import hspec
    return hspec


def expect_timeout(H):
    st = H.hspec_sync_status()
    msg = H.hspec_last_error()
    assert st == H.HSPEC_ERR_DEVICE_CHECK, (st, msg)
    bits = int(msg.split("bits 0x")[1].split()[0], 16)
    assert bits & 8, msg
    assert H.hspec_sync_status() == H.HSPEC_OK  # the flag is cleared once reported


def test_injection_gemm_wait_runs_out(H, cuda):
    # the tcgen05 GEMM (TMA ring, MMA issuer, epilogue warps): 256 output tiles of 64
    # K blocks each, a W_inj of 512 MB
    sh = replace(I.LLAMA, H=8)
    inp = I.make_inject_inputs(sh, 4, 41, cuda)
    h0 = torch.empty(4, sh.H * sh.P * sh.N, device=cuda)
    H.hspec_inject_state(H.make_cfg(sh), inp["W_inj"], inp["h_last"], h0)
    assert H.hspec_sync_status() == 0
    want = h0.clone()
    h0.fill_(float("nan"))
    H.hspec_inject_state(H.make_cfg(sh, wait_limit_ns=TINY_LIMIT_NS), inp["W_inj"], inp["h_last"], h0)
    expect_timeout(H)
    H.hspec_inject_state(H.make_cfg(sh), inp["W_inj"], inp["h_last"], h0)
    assert H.hspec_sync_status() == 0
    assert torch.equal(h0, want)


def test_ssd_scan_wait_runs_out(H, cuda):
    # the tcgen05 state readout (TMA producer, MMA issuer, two transform warpgroups)
    sh = I.LLAMA
    C, K = 16, 16
    inp = I.make_ssd_inputs(sh, C, K, 42, cuda)
    y = torch.empty(C, K, sh.H, sh.P, device=cuda)

    def scan(cfg):
        H.hspec_ssd_block_scan(cfg, inp["x"], inp["dt"], inp["A"], inp["B"], inp["Cm"], inp["D"], inp["h0"], y)

    scan(H.make_cfg(sh))
    assert H.hspec_sync_status() == 0
    want = y.clone()
    y.fill_(float("nan"))
    scan(H.make_cfg(sh, wait_limit_ns=TINY_LIMIT_NS))
    expect_timeout(H)
    scan(H.make_cfg(sh))
    assert H.hspec_sync_status() == 0
    assert torch.equal(y, want)


def test_paged_attention_wait_runs_out(H, cuda):
    # the persistent tcgen05 attention (4 TMA producer warps, Q.K^T and P.V issuers, two
    # softmax warpgroups)
    sh = I.LLAMA
    lens = torch.tensor([700, 4096, 1, 3000, 0, 2500, 8191, 64], dtype=torch.int32)
    inp = I.make_attn_inputs(sh, lens, 16, 43, cuda)
    kv = H.kv_view(inp)

    def attn(cfg):
        ws = H.alloc_workspace(H.hspec_attn_workspace_size(cfg, len(lens), 16, kv.max_pages))
        out = torch.full_like(inp["q"], float("nan"))
        H.hspec_attn_paged_block(cfg, inp["q"], kv, inp["ctx_lens"], inp["k_blk"], inp["v_blk"], out, ws)
        return out

    want = attn(H.make_cfg(sh))
    assert H.hspec_sync_status() == 0
    attn(H.make_cfg(sh, wait_limit_ns=TINY_LIMIT_NS))
    expect_timeout(H)
    got = attn(H.make_cfg(sh))
    assert H.hspec_sync_status() == 0
    assert torch.equal(got, want)


def test_draft_step_wait_runs_out(H, cuda):
    # the whole step, whose projection and MLP GEMMs cut their K loops (stream-K at
    # C=8: counters that other CTAs wait on)
    wl = I.full_workload(8, 16)
    st = I.make_step_inputs(wl, cuda)
    sh = wl.shapes
    max_pages = max(c["page_table"].shape[1] for c in st["kv"])

    def step(limit):
        dr = H.Drafter(sh, st["weights"], wait_limit_ns=limit)
        ws = H.alloc_workspace(dr.workspace_size(wl.C, wl.K, max_pages), cuda)
        hidden = torch.full((wl.C, wl.K, sh.d), float("nan"), device=cuda)
        toks = torch.full((wl.C, wl.K), -1, dtype=torch.int32, device=cuda)
        si = dr.step_in(wl.C, wl.K, st["h_last"], st["ctx_lens"], st["kv"], tokens=st["tokens"])
        dr.step(si, H.hspec_step_out(hidden=hidden.data_ptr(), draft_tokens=toks.data_ptr()), ws)
        return dr, hidden, toks

    dr0, want_h, want_t = step(0)
    assert H.hspec_sync_status() == 0
    dr1, _, _ = step(TINY_LIMIT_NS)
    expect_timeout(H)
    dr2, got_h, got_t = step(0)
    assert H.hspec_sync_status() == 0
    assert torch.equal(got_h, want_h) and torch.equal(got_t, want_t)
    for d in (dr0, dr1, dr2):
        d.close()
