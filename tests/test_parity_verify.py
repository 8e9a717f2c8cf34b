"""GPU parity of hspec_verify_greedy (greedy speculative verification) against the CPU
oracle: accepted lengths, next tokens and the advanced context lengths, bit for bit.

Standard speculative-decoding verification, which H-Spec keeps (evolve.pub review of
H-Spec, Frequently asked questions).  Inputs: seeded random logits with drafts built
so that every acceptance length 0..K occurs, plus ties, NaN rows and ragged vocabularies.
"""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H(cuda):
    from hybrid_mamba_attention_b200 import hspec
    return hspec


def make_case(C, K, V, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    lg = torch.randn(C, K + 1, V, generator=g).to(dtype)
    t = lg.float().argmax(-1)
    drafts = torch.randint(0, V, (C, K), generator=g, dtype=torch.int32)
    for c in range(C):  # request c accepts c mod (K + 1) drafts
        L = c % (K + 1)
        drafts[c, :L] = t[c, :L].to(torch.int32)
        if L < K:
            drafts[c, L] = ((t[c, L] + 1) % V).to(torch.int32)
    return lg, drafts


def run_gpu(H, lg, drafts, ctx, dtype):
    C, K1, V = lg.shape
    sh = I.Shapes("verify", d=64, Hq=1, Hkv=1, D=64, H=1, P=64, N=16, dtype=dtype, rope_theta=1e4, vocab=V)
    cfg = H.make_cfg(sh)
    dev = torch.device("cuda")
    ws = H.alloc_workspace(H.hspec_verify_workspace_size(cfg, C, K1 - 1), dev)
    acc = torch.full((C,), -7, dtype=torch.int32, device=dev)
    nxt = torch.full((C,), -7, dtype=torch.int32, device=dev)
    ctx_d = ctx.to(dev).clone()
    H.hspec_verify_greedy(cfg, lg.to(dev), drafts.to(dev), acc, nxt, ws, ctx_lens=ctx_d)
    assert H.hspec_sync_status() == 0, H.hspec_last_error()
    return acc.cpu().numpy(), nxt.cpu().numpy(), ctx_d.cpu().numpy()


@pytest.mark.parametrize("C,K,V,dtype", [(128, 16, 128256, "bf16"), (1, 16, 128256, "bf16"), (8, 32, 32768, "bf16"),
                                         (5, 7, 1000, "f32"), (3, 1, 8191, "bf16"), (2, 64, 8193, "f32"), (4, 3, 16384, "bf16"), (2, 2, 49152, "f32"), (3, 40, 65536, "bf16"), (2, 64, 70000, "bf16"),
                                         (17, 4, 50001, "bf16")])
def test_verify_greedy_matches_oracle(H, cuda, C, K, V, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    lg, drafts = make_case(C, K, V, tdt, seed=C * 7 + K)
    ctx = torch.randint(0, 5000, (C,), generator=torch.Generator().manual_seed(C), dtype=torch.int32)
    acc, nxt, ctx2 = run_gpu(H, lg, drafts, ctx, dtype)
    e_acc, e_nxt, e_ctx = oracle.verify_greedy(lg, drafts, ctx)
    assert np.array_equal(acc, e_acc)
    assert np.array_equal(nxt, e_nxt)
    assert np.array_equal(ctx2, e_ctx)
    assert sorted(set(acc.tolist())) == sorted(set(c % (K + 1) for c in range(C)))


def test_verify_ties_nan_and_empty_rows(H, cuda):
    K, V = 3, 20000
    lg = torch.zeros(2, K + 1, V)
    lg[0, 0, 15000] = lg[0, 0, 9000] = 4.0            # tie across chunks: id 9000
    lg[0, 1, 100] = float("nan")
    lg[0, 1, 19999] = 2.0                             # NaN skipped
    lg[0, 2] = float("nan")                           # no number: -1
    lg[1] = -float("inf")                             # all -inf: id 0 wins (a number)
    drafts = torch.tensor([[9000, 19999, 5], [0, 0, 1]], dtype=torch.int32)
    ctx = torch.tensor([10, 20], dtype=torch.int32)
    for dtype, tdt in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        acc, nxt, ctx2 = run_gpu(H, lg.to(tdt), drafts, ctx, dtype)
        e_acc, e_nxt, e_ctx = oracle.verify_greedy(lg.to(tdt), drafts, ctx)
        assert acc.tolist() == e_acc.tolist() == [2, 2]
        assert nxt.tolist() == e_nxt.tolist() == [-1, 0]
        assert ctx2.tolist() == e_ctx.tolist() == [13, 23]
