"""CPU checks of the seeded input generators that feed both the CUDA path and the oracle.

The parity tests lean on properties of these inputs: a request's pages are its own,
pages no request owns are NaN (so a read through a wrong page id shows up in the
output), and every draw is reproducible from its seed.  These tests pin those
properties on small shapes.
"""
from dataclasses import replace
import math

import pytest
import torch

from hybrid_mamba_attention_b200 import inputs as I

SMALL_BF16 = replace(I.TINY, name="small_bf16", dtype="bf16")


def _bits(t):
    # bitwise view, so that NaN compares equal to the same NaN
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("shuffle", [True, False])
def test_paged_kv_pages_are_private_and_slack_is_nan(shuffle):
    lens = torch.tensor([0, 1, 15, 16, 17, 100, 333], dtype=torch.int32)
    kv = I.make_paged_kv(SMALL_BF16, lens, seed=5, shuffle=shuffle)
    page = SMALL_BF16.page
    n_pages = [(int(l) + page - 1) // page for l in lens]
    used = sum(n_pages)
    assert kv["num_pages"] == used + math.ceil(0.10 * used)
    table = kv["page_table"]
    owned = []
    for c, n in enumerate(n_pages):
        row = table[c]
        assert (row[n:] == -1).all()                       # entries past the context are unused
        owned += row[:n].tolist()
    assert len(set(owned)) == used                          # no page is shared by two requests
    assert all(0 <= p < kv["num_pages"] for p in owned)
    if not shuffle:
        assert owned == list(range(used))
    slack = sorted(set(range(kv["num_pages"])) - set(owned))
    assert len(slack) == kv["num_pages"] - used
    for pool in (kv["k_pool"], kv["v_pool"]):
        assert torch.isnan(pool[slack].float()).all()       # every slack page is NaN
        assert torch.isfinite(pool[owned].float()).all()    # no owned page is


def test_generators_are_reproducible_from_their_seeds():
    lens = torch.tensor([40, 90], dtype=torch.int32)
    a = I.make_paged_kv(SMALL_BF16, lens, seed=3)
    b = I.make_paged_kv(SMALL_BF16, lens, seed=3)
    c = I.make_paged_kv(SMALL_BF16, lens, seed=4)
    for k in ("k_pool", "v_pool", "page_table"):
        assert torch.equal(_bits(a[k]) if a[k].is_floating_point() else a[k],
                           _bits(b[k]) if b[k].is_floating_point() else b[k])
    assert not torch.equal(a["page_table"], c["page_table"]) or not torch.equal(_bits(a["k_pool"]),
                                                                                _bits(c["k_pool"]))
    wa, wb = I.make_weights(SMALL_BF16, seed=9), I.make_weights(SMALL_BF16, seed=9)
    for la, lb in zip(wa["layers"], wb["layers"]):
        for k, t in la.items():
            if torch.is_tensor(t):
                assert torch.equal(_bits(t), _bits(lb[k])), k


def test_weight_draws_follow_the_stated_laws():
    sh = replace(I.LLAMA, name="wide", d=512, Hq=8, Hkv=2, H=16, P=32, N=16)
    w = I.make_weights(sh, seed=1)
    for layer in w["layers"]:
        n = layer["norm"].double()
        assert abs(n.mean().item() - 1.0) < 0.02 and abs(n.std().item() - 0.1) < 0.02   # 1 + 0.1 N(0,1)
        if layer["kind"] == "M":
            A = layer["A"].double()
            assert (A <= -1.0).all() and (A >= -16.0).all()                               # -exp(U[0, ln 16])
            assert (layer["dt_bias"] == -4.0).all()
            W = layer["W_in"].double()
            assert abs(W.std().item() - 1 / math.sqrt(sh.d)) < 0.05 / math.sqrt(sh.d)     # N(0, 1/fan_in)


def test_context_lengths_stay_in_the_workload_range():
    wl = I.full_workload(64, 16)
    lens = I.make_ctx_lens(wl)
    assert lens.dtype == torch.int32 and lens.numel() == 64
    assert (lens >= wl.ctx_lo).all() and (lens <= wl.ctx_hi).all()
    assert torch.equal(lens, I.make_ctx_lens(wl))
