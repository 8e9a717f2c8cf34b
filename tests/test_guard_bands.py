"""Writes stay inside their outputs (GPU).

Every output of every entry point is placed in the middle of a larger buffer whose
guard regions on both sides hold a sentinel bit pattern (NaN for floating outputs,
0x7EADBEEF for integer ones).  Each call runs at ragged sizes -- rows, positions and
columns that end inside a tile -- and afterwards both guards must still hold the
sentinel bit for bit, and the output itself must have been written (no sentinel
left in it).  The KV pools carry NaN-filled slack pages, so a stray read through a
wrong page shows up in the outputs as well.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from hybrid_mamba_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu

GUARD_BYTES = 64 << 10   # a multiple of 256 bytes: the output keeps the buffer's alignment
INT_SENTINEL = 0x7EADBEEF


@pytest.fixture(scope="module")
def H(cuda):
    from hybrid_mamba_attention_b200 import hspec
    return hspec


class Guarded:
    """An output tensor inside a sentinel-filled buffer."""

    def __init__(self, shape, dtype, device):
        n = int(np.prod(shape))
        esize = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // esize
        self.buf = torch.empty(self.g + n + self.g, dtype=dtype, device=device)
        if dtype.is_floating_point:
            self.buf.fill_(float("nan"))
        else:
            self.buf.fill_(INT_SENTINEL)
        self.sentinel = self.buf[:1].clone()
        self.out = self.buf[self.g:self.g + n].view(shape)

    def _bits(self, t):
        return t.view(torch.int16 if t.element_size() == 2 else torch.int32)

    def check(self, what, all_written=True):
        s = self._bits(self.sentinel)
        for name, part in (("before", self.buf[:self.g]), ("after", self.buf[-self.g:])):
            ok = torch.all(self._bits(part) == s).item()
            assert ok, f"{what}: a write landed in the guard {name} the output"
        if all_written:
            left = torch.sum(self._bits(self.out) == s).item()
            assert left == 0, f"{what}: {left} elements of the output were not written"


def test_injection_and_ssd_outputs_stay_inside(H, cuda):
    sh = replace(I.LLAMA, H=4)            # H*P*N = 32768 state rows per request
    C, K = 3, 7                           # 3 of 128 GEMM rows; 7 of 16 positions
    cfg = H.make_cfg(sh)
    inp = I.make_inject_inputs(sh, C, 71, cuda)
    h0 = Guarded((C, sh.H * sh.P * sh.N), torch.float32, cuda)
    H.hspec_inject_state(cfg, inp["W_inj"], inp["h_last"], h0.out)
    assert H.hspec_sync_status() == 0
    h0.check("hspec_inject_state h0")
    for Kx, chunk in ((K, 0), (K, 3), (21, 0)):  # tensor-core chunk, CUDA-core chunks, N = 32 positions
        s_in = I.make_ssd_inputs(sh, C, Kx, 72, cuda)
        y = Guarded((C, Kx, sh.H, sh.P), torch.float32, cuda)
        hK = Guarded((C, sh.H, sh.P, sh.N), torch.float32, cuda)
        H.hspec_ssd_block_scan(H.make_cfg(sh, ssd_chunk=chunk), s_in["x"], s_in["dt"], s_in["A"], s_in["B"],
                               s_in["Cm"], s_in["D"], s_in["h0"], y.out, hK.out)
        assert H.hspec_sync_status() == 0
        y.check(f"ssd y K={Kx} chunk={chunk}")
        hK.check(f"ssd hK K={Kx} chunk={chunk}")


@pytest.mark.parametrize("noalloc", [False, True])
def test_attention_output_stays_inside(H, cuda, noalloc):
    sh = I.LLAMA
    lens = torch.tensor([0, 1, 15, 17, 63, 65, 700, 4099], dtype=torch.int32)
    K = 5
    inp = I.make_attn_inputs(sh, lens, K, 73, cuda, slack=0.5)
    cfg = H.make_cfg(sh)
    kv = H.kv_view(inp)
    out = Guarded(tuple(inp["q"].shape), inp["q"].dtype, cuda)
    if noalloc:
        H.hspec_attn_paged_block_noalloc(cfg, inp["q"], kv, inp["ctx_lens"], inp["k_blk"], inp["v_blk"], out.out)
    else:
        ws = H.alloc_workspace(H.hspec_attn_workspace_size(cfg, len(lens), K, kv.max_pages))
        H.hspec_attn_paged_block(cfg, inp["q"], kv, inp["ctx_lens"], inp["k_blk"], inp["v_blk"], out.out, ws)
    assert H.hspec_sync_status() == 0
    out.check("attention out")
    assert torch.isfinite(out.out.float()).all()


@pytest.mark.parametrize("C,K", [(3, 7), (1, 33)])
def test_draft_step_outputs_stay_inside(H, cuda, C, K):
    wl = I.full_workload(C, K)
    st = I.make_step_inputs(wl, cuda)
    sh = wl.shapes
    dr = H.Drafter(sh, st["weights"])
    max_pages = max(c["page_table"].shape[1] for c in st["kv"])
    ws = H.alloc_workspace(dr.workspace_size(C, K, max_pages), cuda)
    hidden = Guarded((C, K, sh.d), torch.float32, cuda)
    toks = Guarded((C, K), torch.int32, cuda)
    normed = Guarded((C, K, sh.d), sh.torch_dtype, cuda)
    top = Guarded((C, K), torch.float32, cuda)
    layers = Guarded((len(sh.layers), C, K, sh.d), torch.float32, cuda)
    si = dr.step_in(C, K, st["h_last"], st["ctx_lens"], st["kv"], tokens=st["tokens"])
    so = H.hspec_step_out(draft_tokens=toks.out.data_ptr(), hidden=hidden.out.data_ptr(),
                          final_normed=normed.out.data_ptr(), top_logit=top.out.data_ptr(),
                          layer_hidden=layers.out.data_ptr())
    dr.step(si, so, ws)
    assert H.hspec_sync_status() == 0
    for g, what in ((hidden, "hidden"), (toks, "draft_tokens"), (normed, "final_normed"), (top, "top_logit"),
                    (layers, "layer_hidden")):
        g.check(f"draft step C={C} K={K} {what}")
    assert ((toks.out >= 0) & (toks.out < sh.vocab)).all()
    dr.close()


def test_verify_outputs_stay_inside(H, cuda):
    C, K, V = 5, 7, 50001  # a vocabulary that ends inside a chunk
    g = torch.Generator(device=cuda).manual_seed(74)
    logits = torch.randn(C, K + 1, V, generator=g, device=cuda).to(torch.bfloat16)
    drafts = torch.randint(0, V, (C, K), generator=g, device=cuda, dtype=torch.int32)
    drafts[:, :3] = logits[:, :3].float().argmax(-1).to(torch.int32)  # some accepted prefixes
    cfg = H.make_cfg(replace(I.LLAMA, vocab=V))
    ws = H.alloc_workspace(H.hspec_verify_workspace_size(cfg, C, K), cuda)
    acc = Guarded((C,), torch.int32, cuda)
    nxt = Guarded((C,), torch.int32, cuda)
    ctx = Guarded((C,), torch.int32, cuda)
    ctx.out.copy_(torch.arange(100, 100 + C, dtype=torch.int32, device=cuda))
    H.hspec_verify_greedy(cfg, logits, drafts, acc.out, nxt.out, ws, ctx_lens=ctx.out)
    assert H.hspec_sync_status() == 0
    acc.check("verify accepted")
    nxt.check("verify next_token")
    ctx.check("verify ctx_lens")
    assert (acc.out >= 3).all()
