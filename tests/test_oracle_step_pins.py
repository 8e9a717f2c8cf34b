"""Pins of the oracle's full draft step (CPU only).

The reference here is built from library routines (torch float64 matmul, rms_norm,
softplus, silu, scaled_dot_product_attention), RoPE as a complex rotation and the
SSD quadratic dual form -- none of which is the oracle's code -- plus invariants
the method fixes: requests are independent, the paged cache is read in place so
the page placement cannot matter, and a residual block whose output projection is
zero is the identity.  Sources: H-Spec (arXiv 2609.24197) Abstract; evolve.pub
review of H-Spec, Summary (Mamba-2 + attention hybrid, pre-norm blocks);
Dao & Gu (2024) for the SSD dual form.
"""
from dataclasses import replace

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from hybrid_mamba_attention_b200 import inputs as I

SMALL_FULL = I.Shapes("small_full", d=64, Hq=4, Hkv=2, D=16, H=2, P=32, N=8, dtype="f32",
                      rope_theta=1e4, layers="MAMA", d_ff=128, vocab=300)


def wl(sh, C=3, K=5, lo=5, hi=40, seed=7, shuffle=True, slack=0.1):
    return I.Workload("t", sh, C=C, K=K, ctx_lo=lo, ctx_hi=hi, seed=seed, shuffle=shuffle, slack=slack)


def run_oracle(w, st, **kw):
    return oracle.draft_step(w.shapes, st["weights"], st["kv"], st["h_last"], st["ctx_lens"],
                             tokens=st["tokens"], x_in=st["x_in"], **kw)


def d64(t):
    return t.detach().to(torch.float64)


def rope_c(v, theta, pos):
    """RoPE as a complex rotation, v [..., D]."""
    D = v.shape[-1]
    i = torch.arange(D // 2, dtype=torch.float64)
    z = torch.complex(v[..., :D // 2], v[..., D // 2:]) * torch.exp(1j * pos * theta ** (-2.0 * i / D))
    return torch.cat([z.real, z.imag], -1)


def ssd_dual(xs, dt, A, B, Cm, D, h0):
    """Quadratic dual form of the SSD for one request: xs [K,H,P], dt [K,H], B/Cm [K,N], h0 [H,P,N]."""
    cum = torch.cumsum(dt * A[None, :], 0)  # [K,H]
    CB = Cm @ B.T  # [K,K]
    K = xs.shape[0]
    y = torch.zeros_like(xs)
    for t in range(K):
        y[t] = torch.exp(cum[t])[:, None] * torch.einsum("hpn,n->hp", h0, Cm[t]) + D[:, None] * xs[t]
        for s in range(t + 1):
            y[t] += (CB[t, s] * torch.exp(cum[t] - cum[s]) * dt[s])[:, None] * xs[s]
    return y


def reference_step(sh, st):
    """Independent float64 draft step for an fp32 drafter (no bf16 rounding)."""
    W = st["weights"]
    C = st["ctx_lens"].numel()
    outs, toks = [], []
    HP = sh.H * sh.P
    for c in range(C):
        L = int(st["ctx_lens"][c])
        x = d64(W["W_lm"][st["tokens"][c].long()]) if sh.vocab else d64(st["x_in"][c])
        ai = 0
        for w in W["layers"]:
            xn = F.rms_norm(x, (sh.d,), d64(w["norm"]), eps=sh.eps)
            if w["kind"] == "M":
                zx = xn @ d64(w["W_in"]).T
                z, xs = zx[:, :HP], zx[:, HP:2 * HP]
                B, Cm = zx[:, 2 * HP:2 * HP + sh.N], zx[:, 2 * HP + sh.N:2 * HP + 2 * sh.N]
                dt = F.softplus(zx[:, 2 * HP + 2 * sh.N:] + d64(w["dt_bias"]))
                h0 = (d64(w["W_inj"]) @ d64(st["h_last"][c])).reshape(sh.H, sh.P, sh.N)
                y = ssd_dual(xs.reshape(-1, sh.H, sh.P), dt, d64(w["A"]), B, Cm, d64(w["D"]), h0)
                g = F.rms_norm(y.reshape(-1, HP) * F.silu(z), (HP,), d64(w["gnorm"]), eps=sh.eps)
                x = x + g @ d64(w["W_out"]).T
            else:
                qkv = xn @ d64(w["W_qkv"]).T
                K = qkv.shape[0]
                q = qkv[:, :sh.Hq * sh.D].reshape(K, sh.Hq, sh.D)
                kb = qkv[:, sh.Hq * sh.D:(sh.Hq + sh.Hkv) * sh.D].reshape(K, sh.Hkv, sh.D)
                vb = qkv[:, (sh.Hq + sh.Hkv) * sh.D:].reshape(K, sh.Hkv, sh.D)
                pos = torch.arange(K, dtype=torch.float64)[:, None, None] + L
                q, kb = rope_c(q, sh.rope_theta, pos), rope_c(kb, sh.rope_theta, pos)
                cache = st["kv"][ai]
                ai += 1
                pages = cache["page_table"][c, :(L + sh.page - 1) // sh.page].long()
                kc = d64(cache["k_pool"][pages]).reshape(-1, sh.Hkv, sh.D)[:L]
                vc = d64(cache["v_pool"][pages]).reshape(-1, sh.Hkv, sh.D)[:L]
                kk, vv = torch.cat([kc, kb]), torch.cat([vc, vb])
                o = F.scaled_dot_product_attention(q.transpose(0, 1), kk.transpose(0, 1),
                                                   vv.transpose(0, 1), enable_gqa=True)
                x = x + o.transpose(0, 1).reshape(K, -1) @ d64(w["W_o"]).T
            if sh.d_ff:
                xn = F.rms_norm(x, (sh.d,), d64(w["mlp_norm"]), eps=sh.eps)
                a = F.silu(xn @ d64(w["W_gate"]).T) * (xn @ d64(w["W_up"]).T)
                x = x + a @ d64(w["W_down"]).T
        outs.append(x)
        if sh.vocab:
            hn = F.rms_norm(x, (sh.d,), d64(W["final_norm"]), eps=sh.eps)
            toks.append((hn @ d64(W["W_lm"]).T).argmax(-1))
    return torch.stack(outs).numpy(), (torch.stack(toks).numpy() if sh.vocab else None)


def test_tiny_step_matches_library_reference():
    w = replace(I.WORKLOADS["tiny"])
    st = I.make_step_inputs(w)
    got = run_oracle(w, st)
    ref, _ = reference_step(w.shapes, st)
    np.testing.assert_allclose(got["hidden"], ref, rtol=1e-9, atol=1e-9)


def test_full_layer_stack_with_mlp_and_head_matches_library_reference():
    w = wl(SMALL_FULL)
    st = I.make_step_inputs(w)
    got = run_oracle(w, st)
    ref, toks = reference_step(w.shapes, st)
    np.testing.assert_allclose(got["hidden"], ref, rtol=1e-9, atol=1e-9)
    assert np.array_equal(got["draft_tokens"], toks)


def test_request_permutation_permutes_outputs():
    w = wl(SMALL_FULL, C=4)
    st = I.make_step_inputs(w)
    base = run_oracle(w, st)
    perm = torch.tensor([2, 0, 3, 1])
    st2 = dict(st, h_last=st["h_last"][perm], ctx_lens=st["ctx_lens"][perm], tokens=st["tokens"][perm],
               kv=[dict(kv, page_table=kv["page_table"][perm]) for kv in st["kv"]])
    got = run_oracle(w, st2)
    assert np.array_equal(got["hidden"], base["hidden"][perm.numpy()])
    assert np.array_equal(got["draft_tokens"], base["draft_tokens"][perm.numpy()])


def test_page_placement_does_not_change_the_result():
    # Moving every page to another slot of the pool (and rewriting the table) is invisible.
    w = wl(SMALL_FULL, C=3)
    st = I.make_step_inputs(w)
    base = run_oracle(w, st)
    kv2 = []
    for kv in st["kv"]:
        n = kv["k_pool"].shape[0]
        perm = torch.randperm(n, generator=torch.Generator().manual_seed(5))
        inv = torch.empty_like(perm)
        inv[perm] = torch.arange(n)
        tbl = kv["page_table"].clone()
        m = tbl >= 0
        tbl[m] = inv[tbl[m].long()].to(torch.int32)
        kv2.append(dict(kv, k_pool=kv["k_pool"][perm], v_pool=kv["v_pool"][perm], page_table=tbl))
    got = run_oracle(w, dict(st, kv=kv2))
    assert np.array_equal(got["hidden"], base["hidden"])


def test_zero_output_projections_make_layers_identity():
    w = replace(I.WORKLOADS["tiny"])
    st = I.make_step_inputs(w)
    for lw in st["weights"]["layers"]:
        for k in ("W_out", "W_o"):
            if k in lw:
                lw[k].zero_()
    got = run_oracle(w, st)
    assert np.array_equal(got["hidden"], st["x_in"].double().numpy())


def test_zero_injection_equals_zero_initial_state():
    # h_last = 0 projects to h0 = 0; the same step with W_inj = 0 must agree exactly.
    w = replace(I.WORKLOADS["tiny"])
    st = I.make_step_inputs(w)
    st["h_last"].zero_()
    a = run_oracle(w, st)["hidden"]
    st = I.make_step_inputs(w)
    for lw in st["weights"]["layers"]:
        if "W_inj" in lw:
            lw["W_inj"].zero_()
    b = run_oracle(w, st)["hidden"]
    assert np.array_equal(a, b)


def test_bf16_step_rounds_where_bf16_is_stored_and_head_is_consistent():
    sh = replace(SMALL_FULL, dtype="bf16")
    w = wl(sh, C=2)
    st = I.make_step_inputs(w)
    got = run_oracle(w, st)
    fn = got["final_normed"]
    assert np.array_equal(oracle.bf16_round(fn), fn)
    am, t1, t2 = oracle.lm_head_argmax(torch.from_numpy(fn.reshape(-1, sh.d)).float(), st["weights"]["W_lm"])
    assert np.array_equal(am.reshape(got["draft_tokens"].shape), got["draft_tokens"])
    logits = fn.reshape(-1, sh.d) @ st["weights"]["W_lm"].double().numpy().T
    assert np.array_equal(logits.argmax(1).reshape(got["draft_tokens"].shape), got["draft_tokens"])


def test_bf16_step_stays_close_to_fp32_step():
    # Same random draws stored in bf16 vs fp32: the bf16 step must track the fp32 one
    # to within bf16 rounding drift (a missing rounding point would not break this,
    # a wrong one -- e.g. rounding the residual stream -- shows up as larger drift).
    w32 = wl(SMALL_FULL, C=2)
    w16 = wl(replace(SMALL_FULL, dtype="bf16"), C=2)
    st32, st16 = I.make_step_inputs(w32), I.make_step_inputs(w16)
    h32 = run_oracle(w32, st32)["hidden"]
    h16 = run_oracle(w16, st16)["hidden"]
    rel = np.abs(h16 - h32).max() / np.sqrt((h32 ** 2).mean())
    assert rel < 0.1


def test_reduced_draft_head_is_the_full_head_restricted_and_remapped():
    # Reduced-vocabulary draft head (evolve.pub review of H-Spec, Frequently asked
    # questions: the drafter's vocabulary cut to frequent tokens): with the draft rows
    # taken from the full head (W_lm_draft = W_lm[ids]), the draft token is the target id
    # whose logit is highest among ids, read from the full head's own final hidden state.
    sh = replace(SMALL_FULL, draft_vocab=97)
    w = wl(sh)
    st = I.make_step_inputs(w)
    ids = st["weights"]["draft_to_target"]
    assert ids.shape == (97,) and bool((ids[1:] > ids[:-1]).all()) and int(ids.max()) < sh.vocab
    st["weights"]["W_lm_draft"] = st["weights"]["W_lm"][ids.long()].clone()
    full = run_oracle(wl(SMALL_FULL), st)
    got = run_oracle(w, st)
    np.testing.assert_array_equal(got["hidden"], full["hidden"])
    logits = torch.from_numpy(full["final_normed"]) @ d64(st["weights"]["W_lm"]).T  # [C,K,V]
    sub = logits[..., ids.long()]
    want = ids.long()[sub.argmax(-1)].numpy()
    assert np.array_equal(got["draft_tokens"], want)
    np.testing.assert_allclose(got["top1"], sub.max(-1).values.numpy(), rtol=1e-12, atol=1e-12)


def test_reduced_draft_head_with_every_id_in_order_is_the_full_head():
    sh = replace(SMALL_FULL, draft_vocab=SMALL_FULL.vocab)
    w = wl(sh)
    st = I.make_step_inputs(w)
    assert torch.equal(st["weights"]["draft_to_target"].long(), torch.arange(sh.vocab))
    st["weights"]["W_lm_draft"] = st["weights"]["W_lm"].clone()
    full = run_oracle(wl(SMALL_FULL), st)
    got = run_oracle(w, st)
    for k in ("draft_tokens", "top1", "top2"):
        assert np.array_equal(got[k], full[k])
