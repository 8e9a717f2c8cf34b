"""The allocation-free attention entry point (GPU).

Some callers cannot allocate device memory when they call in -- a serving engine
that gave nearly all HBM to its KV-cache pool at start-up, or a C host program with
no device allocator of its own -- so hspec_attn_paged_block_noalloc keeps its
split-KV partials in a static device array inside the library instead of a
caller-provided workspace.  These tests call it through the C-ABI twice in a row
(different inputs, so a stale scratch would show) and compare it with
hspec_attn_paged_block on the same inputs.  Both run the same kernels on the same
batch, and repeated calls on one batch are bit-identical, so the two outputs must be
equal bit for bit (a stale partial that moved a few ulps would fail).
This file is collected last so that a failure here cannot hide any other test's
result; it passes alone in a fresh process as well as after the other tests.
"""
import ctypes as ct

import pytest
import torch

from hybrid_mamba_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H(cuda):
    from hybrid_mamba_attention_b200 import hspec
    return hspec


def with_workspace(H, cfg, inp, K):
    kv = H.kv_view(inp)
    ws = H.alloc_workspace(H.hspec_attn_workspace_size(cfg, inp["q"].shape[0], K, kv.max_pages))
    out = torch.full_like(inp["q"], float("nan"))
    H.hspec_attn_paged_block(cfg, inp["q"], kv, inp["ctx_lens"], inp["k_blk"], inp["v_blk"], out, ws)
    return out


def without_workspace(H, cfg, inp, K):
    out = torch.full_like(inp["q"], float("nan"))
    H.hspec_attn_paged_block_noalloc(cfg, inp["q"], H.kv_view(inp), inp["ctx_lens"], inp["k_blk"], inp["v_blk"], out)
    return out


# Llama-3-8B shapes with 16 requests of up to 8k context fit the 64 MiB scratch
LLAMA_C16 = I.Workload("llama_c16", I.LLAMA, C=16, K=16, ctx_lo=512, ctx_hi=8192, seed=5)


@pytest.mark.parametrize("name", ["llama_c16", "tiny"])
def test_noalloc_attention_matches_workspace_attention_twice(H, cuda, name):
    wl = LLAMA_C16 if name == "llama_c16" else I.WORKLOADS[name]
    sh = wl.shapes
    cfg = H.make_cfg(sh)
    for call, seed in enumerate((31, 32)):  # two calls in a row through the shared scratch
        lens = I.make_ctx_lens(wl) if call == 0 else torch.flip(I.make_ctx_lens(wl), [0]) // 2
        inp = I.make_attn_inputs(sh, lens, wl.K, seed, cuda, shuffle=wl.shuffle, slack=wl.slack)
        assert H.hspec_attn_workspace_size(cfg, wl.C, wl.K, inp["page_table"].shape[1]) <= \
            H.HSPEC_NOALLOC_SCRATCH_BYTES
        got = without_workspace(H, cfg, inp, wl.K)
        assert H.hspec_sync_status() == 0, H.hspec_last_error()
        want = with_workspace(H, cfg, inp, wl.K)
        assert H.hspec_sync_status() == 0
        assert torch.equal(got, want), f"noalloc vs workspace differ on call {call}"
        assert torch.isfinite(got.float()).all()


def test_noalloc_attention_rejects_oversized_calls(H, cuda):
    sh = I.QWEN
    cfg = H.make_cfg(sh)
    C, K, max_pages = 128, 16, 2048
    assert H.hspec_attn_workspace_size(cfg, C, K, max_pages) > H.HSPEC_NOALLOC_SCRATCH_BYTES
    kv = H.hspec_kv_view(k_pool=256, v_pool=256, num_pages=max_pages, page_table=256, max_pages=max_pages)
    n0 = H.hspec_launch_count()
    st = H._lib.hspec_attn_paged_block_noalloc(ct.byref(cfg), 256, ct.byref(kv), 256, 256, 256, C, K, 256, None)
    assert st == H.HSPEC_ERR_WORKSPACE
    assert "scratch" in H.hspec_last_error()
    assert H.hspec_launch_count() == n0
