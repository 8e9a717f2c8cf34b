"""Pins of the CPU oracle against facts other than itself (CPU only).

Each test ties one oracle function to a closed form, a library routine, an
invariant or a special case that the method fixes, chosen so that a plausible
mistake (a dropped term, a wrong sign or index, a transposed operand) fails.

Sources: H-Spec (arXiv 2609.24197) Abstract -- attention reuses the target KVs in
place, Mamba modules start from the projected last-token hidden state, the parallel
scan keeps drafting block-parallel; the Mamba-2 SSD recurrence and its quadratic
("attention-like") dual form from Dao & Gu, "Transformers are SSMs" (2024).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from hybrid_mamba_attention_b200 import inputs as I


def rng(seed):
    return np.random.default_rng(seed)


def f32(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32))


# ------------------------------------------------------------------ bf16 rounding

def test_bf16_round_matches_torch_rne():
    # torch's float32 -> bfloat16 conversion rounds to nearest, ties to even.
    a = rng(0).standard_normal(20000).astype(np.float32) * np.float32(1e3)
    a = np.concatenate([a, np.float32([1e-39, -3e-40, 3.3e38, 65504.0])])
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_round(a.astype(np.float64)), ref)


def test_bf16_round_ties_to_even():
    # bf16 spacing at 1.0 is 2^-7: 1 + 2^-8 ties down to 1.0 (even), 1 + 3*2^-8 ties up.
    assert oracle.bf16_round([1 + 2 ** -8])[0] == 1.0
    assert oracle.bf16_round([1 + 3 * 2 ** -8])[0] == 1 + 2 ** -6
    assert oracle.bf16_round([-(1 + 2 ** -8)])[0] == -1.0


# ------------------------------------------------------------------------ inject

def test_inject_matches_numpy_matmul():
    r = rng(1)
    W = r.standard_normal((96, 40)).astype(np.float32)
    h = r.standard_normal((3, 40)).astype(np.float32)
    got = oracle.inject(f32(W), f32(h))
    ref = h.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


def test_inject_reshape_order_is_head_p_n():
    # W_inj row r = (h*P + p)*N + n selects h_last[(7 r) mod d]; the [H,P,N] view of
    # h0 must then hold h_last[(7((h P + p) N + n)) mod d].
    H, P, N, d = 3, 4, 5, 64
    W = np.zeros((H * P * N, d), np.float32)
    for r in range(H * P * N):
        W[r, (7 * r) % d] = 1.0
    h = rng(2).standard_normal((2, d)).astype(np.float32)
    h0 = oracle.inject(f32(W), f32(h)).reshape(2, H, P, N)
    for c in range(2):
        for hh in range(H):
            for p in range(P):
                for n in range(N):
                    assert h0[c, hh, p, n] == h[c, (7 * ((hh * P + p) * N + n)) % d]


def test_inject_zero_hidden_gives_zero_state():
    W = rng(3).standard_normal((32, 16)).astype(np.float32)
    assert not oracle.inject(f32(W), torch.zeros(2, 16)).any()


def test_inject_bf16_inputs_decoded_exactly():
    r = rng(4)
    W = torch.from_numpy(r.standard_normal((64, 32)).astype(np.float32)).to(torch.bfloat16)
    h = torch.from_numpy(r.standard_normal((2, 32)).astype(np.float32)).to(torch.bfloat16)
    ref = h.double().numpy() @ W.double().numpy().T
    np.testing.assert_allclose(oracle.inject(W, h), ref, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------- SSD

def ssd_case(seed, C=2, K=8, H=3, P=4, N=5):
    r = rng(seed)
    return dict(
        x=r.standard_normal((C, K, H, P)).astype(np.float32),
        dt=np.log1p(np.exp(r.standard_normal((C, K, H)) - 1.0)).astype(np.float32),
        A=(-np.exp(r.uniform(0, math.log(16), H))).astype(np.float32),
        B=r.standard_normal((C, K, N)).astype(np.float32),
        Cm=r.standard_normal((C, K, N)).astype(np.float32),
        D=r.standard_normal(H).astype(np.float32),
        h0=r.standard_normal((C, H, P, N)).astype(np.float32))


def run_ssd(cs, want_state=False, h0=True):
    return oracle.ssd_scan(f32(cs["x"]), f32(cs["dt"]), f32(cs["A"]), f32(cs["B"]), f32(cs["Cm"]),
                           f32(cs["D"]), f32(cs["h0"]) if h0 else None, want_state=want_state)


def ssd_quadratic(cs):
    """SSD dual (quadratic) form, written independently of the recurrence:
    y_t = sum_{s<=t} (C_t . B_s) exp(sum_{r=s+1..t} dt_r A) dt_s x_s
          + exp(sum_{r=0..t} dt_r A) (h0 C_t) + D x_t."""
    x, dt, A, B, Cm, D, h0 = (cs[k].astype(np.float64) for k in ("x", "dt", "A", "B", "Cm", "D", "h0"))
    C, K, H, P = x.shape
    y = np.zeros_like(x)
    for c in range(C):
        cum = np.cumsum(dt[c] * A[None, :], axis=0)  # [K,H]: sum_{r<=t} dt_r A
        CB = Cm[c] @ B[c].T  # [K(t), K(s)]
        for h in range(H):
            for t in range(K):
                acc = np.exp(cum[t, h]) * (h0[c, h] @ Cm[c, t])
                for s in range(t + 1):
                    acc = acc + CB[t, s] * np.exp(cum[t, h] - cum[s, h]) * dt[c, s, h] * x[c, s, h]
                y[c, t, h] = acc + D[h] * x[c, t, h]
    return y


def test_ssd_recurrence_equals_quadratic_dual_form():
    cs = ssd_case(10)
    np.testing.assert_allclose(run_ssd(cs), ssd_quadratic(cs), rtol=1e-10, atol=1e-10)


def test_ssd_final_state_closed_form():
    cs = ssd_case(11)
    _, hK = run_ssd(cs, want_state=True)
    x, dt, A, B, h0 = (cs[k].astype(np.float64) for k in ("x", "dt", "A", "B", "h0"))
    C, K, H, P = x.shape
    for c in range(C):
        cum = np.cumsum(dt[c] * A[None, :], axis=0)
        for h in range(H):
            ref = np.exp(cum[-1, h]) * h0[c, h]
            for s in range(K):
                ref = ref + np.exp(cum[-1, h] - cum[s, h]) * dt[c, s, h] * np.outer(x[c, s, h], B[c, s])
            np.testing.assert_allclose(hK[c, h], ref, rtol=1e-10, atol=1e-10)


def test_ssd_single_step_closed_form():
    cs = ssd_case(12, K=1)
    x, dt, A, B, Cm, D, h0 = (cs[k].astype(np.float64) for k in ("x", "dt", "A", "B", "Cm", "D", "h0"))
    y = run_ssd(cs)
    for c in range(x.shape[0]):
        for h in range(x.shape[2]):
            hs = np.exp(dt[c, 0, h] * A[h]) * h0[c, h] + dt[c, 0, h] * np.outer(x[c, 0, h], B[c, 0])
            np.testing.assert_allclose(y[c, 0, h], hs @ Cm[c, 0] + D[h] * x[c, 0, h], rtol=1e-12)


def test_ssd_zero_dt_keeps_initial_state():
    cs = ssd_case(13)
    cs["dt"][:] = 0.0
    y = run_ssd(cs)
    x, Cm, D, h0 = (cs[k].astype(np.float64) for k in ("x", "Cm", "D", "h0"))
    ref = np.einsum("chpn,ctn->cthp", h0, Cm) + D[None, None, :, None] * x
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_ssd_full_decay_forgets_history():
    # exp(dt A) underflows to 0: h_t = dt_t x_t B_t^T, y_t = dt_t (C_t . B_t) x_t + D x_t.
    cs = ssd_case(14)
    cs["A"][:] = -1e6
    cs["dt"][:] = 1.0
    y = run_ssd(cs)
    x, B, Cm, D = (cs[k].astype(np.float64) for k in ("x", "B", "Cm", "D"))
    cb = np.einsum("ctn,ctn->ct", Cm, B)
    ref = cb[:, :, None, None] * x + D[None, None, :, None] * x
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_ssd_zero_injection_equals_zero_state():
    cs = ssd_case(15)
    cs["h0"][:] = 0.0
    assert np.array_equal(run_ssd(cs), run_ssd(cs, h0=False))


def test_ssd_initial_state_enters_linearly_with_decay():
    # y(h0) - y(0) = exp(sum_{r<=t} dt_r A) h0 C_t
    cs = ssd_case(16)
    diff = run_ssd(cs) - run_ssd(cs, h0=False)
    dt, A, Cm, h0 = (cs[k].astype(np.float64) for k in ("dt", "A", "Cm", "h0"))
    cum = np.cumsum(dt * A[None, None, :], axis=1)  # [C,K,H]
    ref = np.exp(cum)[..., None] * np.einsum("chpn,ctn->cthp", h0, Cm)
    np.testing.assert_allclose(diff, ref, rtol=1e-9, atol=1e-9)


def test_ssd_scalar_worked_example():
    # H=P=N=1, exp(dt A) = 1/2 (A = -ln 2, dt = 1), B = C = 1, D = 0, h0 = 4, x = (1, 2):
    # h_1 = 4/2 + 1 = 3, h_2 = 3/2 + 2 = 3.5, so y = (3, 3.5).
    cs = dict(x=np.float32([[[[1.0]], [[2.0]]]]), dt=np.float32([[[1.0], [1.0]]]),
              A=np.float32([-math.log(2.0)]), B=np.float32([[[1.0], [1.0]]]),
              Cm=np.float32([[[1.0], [1.0]]]), D=np.float32([0.0]), h0=np.float32([[[[4.0]]]]))
    y = run_ssd(cs).reshape(-1)
    np.testing.assert_allclose(y, [3.0, 3.5], rtol=1e-7)


# --------------------------------------------------------------------- attention

def attn_case(seed, C=3, K=4, Hq=4, Hkv=2, D=16, page=4, lens=(9, 0, 13), slack=3):
    r = rng(seed)
    n_pages = [(l + page - 1) // page for l in lens]
    total = sum(n_pages) + slack
    perm = r.permutation(total)
    maxp = max(max(n_pages), 1)
    tbl = -np.ones((C, maxp), np.int32)
    o = 0
    for c in range(C):
        tbl[c, :n_pages[c]] = perm[o:o + n_pages[c]]
        o += n_pages[c]
    kp = r.standard_normal((total, page, Hkv, D)).astype(np.float32)
    vp = r.standard_normal((total, page, Hkv, D)).astype(np.float32)
    for s in perm[o:]:
        kp[s] = np.nan
        vp[s] = np.nan
    return dict(q=r.standard_normal((C, K, Hq, D)).astype(np.float32), k_pool=kp, v_pool=vp,
                page_table=tbl, ctx_lens=np.int32(lens),
                k_blk=r.standard_normal((C, K, Hkv, D)).astype(np.float32),
                v_blk=r.standard_normal((C, K, Hkv, D)).astype(np.float32))


def run_attn(a, causal=False):
    return oracle.attn_paged(f32(a["q"]), f32(a["k_pool"]), f32(a["v_pool"]), a["page_table"],
                             a["ctx_lens"], f32(a["k_blk"]), f32(a["v_blk"]), causal_block=causal)


def gathered(a, c, which):
    page = a["k_pool"].shape[1]
    L = int(a["ctx_lens"][c])
    pool = a[which]
    rows = [pool[a["page_table"][c, t // page], t % page] for t in range(L)]
    blk = a["k_blk" if which == "k_pool" else "v_blk"][c]
    return np.concatenate([np.asarray(rows).reshape(L, *pool.shape[2:]), blk], 0).astype(np.float64)


def test_attention_in_place_equals_contiguous_copy():
    a = attn_case(20)
    C = len(a["ctx_lens"])
    maxc = int(a["ctx_lens"].max())
    kc = np.zeros((C, maxc, *a["k_pool"].shape[2:]), np.float32)
    vc = np.zeros_like(kc)
    for c in range(C):
        L = int(a["ctx_lens"][c])
        kc[c, :L] = gathered(a, c, "k_pool")[:L]
        vc[c, :L] = gathered(a, c, "v_pool")[:L]
    cont = oracle.attn_contiguous(f32(a["q"]), f32(kc), f32(vc), a["ctx_lens"], f32(a["k_blk"]),
                                  f32(a["v_blk"]))
    assert np.array_equal(run_attn(a), cont)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_torch_sdpa(causal):
    a = attn_case(21)
    got = run_attn(a, causal)
    C, K, Hq, D = a["q"].shape
    for c in range(C):
        kk, vv = gathered(a, c, "k_pool"), gathered(a, c, "v_pool")  # [T,Hkv,D]
        L = int(a["ctx_lens"][c])
        T = kk.shape[0]
        mask = None
        if causal:
            mask = torch.ones(K, T, dtype=torch.bool)
            for j in range(K):
                mask[j, L + j + 1:] = False
        q = torch.from_numpy(a["q"][c].astype(np.float64)).transpose(0, 1)  # [Hq,K,D]
        ref = F.scaled_dot_product_attention(q, torch.from_numpy(kk).transpose(0, 1),
                                             torch.from_numpy(vv).transpose(0, 1), attn_mask=mask,
                                             enable_gqa=True)
        np.testing.assert_allclose(got[c], ref.transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_equal_keys_average_values():
    a = attn_case(22)
    a["k_pool"][:] = 0.5
    a["k_blk"][:] = 0.5
    got = run_attn(a)
    G = a["q"].shape[2] // a["k_pool"].shape[2]
    for c in range(len(a["ctx_lens"])):
        mean_v = gathered(a, c, "v_pool").mean(0)  # [Hkv,D]
        for h in range(a["q"].shape[2]):
            np.testing.assert_allclose(got[c, :, h], np.broadcast_to(mean_v[h // G], got[c, :, h].shape),
                                       rtol=1e-12, atol=1e-12)


def test_attention_empty_context_single_key_returns_block_value():
    a = attn_case(23, K=1, lens=(0, 0, 0))
    got = run_attn(a)
    G = a["q"].shape[2] // a["k_pool"].shape[2]
    for h in range(a["q"].shape[2]):
        np.testing.assert_allclose(got[:, 0, h], a["v_blk"][:, 0, h // G], rtol=1e-12)


def test_attention_gqa_head_mapping():
    # every kv head g carries a constant value g + 1: query head h must return h // G + 1.
    a = attn_case(24, Hq=6, Hkv=3)
    for g in range(3):
        a["v_pool"][:, :, g, :] = g + 1.0
        a["v_blk"][:, :, g, :] = g + 1.0
    got = run_attn(a)
    for h in range(6):
        np.testing.assert_allclose(got[:, :, h], h // 2 + 1.0, rtol=1e-12)


def test_attention_rejects_bad_page_id():
    a = attn_case(25)
    a["page_table"][0, 0] = a["k_pool"].shape[0]
    with pytest.raises(ValueError):
        run_attn(a)


# ----------------------------------------------------------- norm / rope / head

def test_rmsnorm_matches_torch():
    r = rng(30)
    x = r.standard_normal((5, 48))
    w = r.standard_normal(48).astype(np.float32)
    ref = F.rms_norm(torch.from_numpy(x), (48,), torch.from_numpy(w.astype(np.float64)), eps=1e-6)
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 1e-6), ref.numpy(), rtol=1e-13)


def test_rope_is_complex_rotation():
    # rotate-half RoPE = multiply z_i = v_i + i v_{i+D/2} by exp(i pos theta^(-2i/D)).
    D, theta, pos = 16, 500000.0, 1234
    v = rng(31).standard_normal(D)
    z = (v[:D // 2] + 1j * v[D // 2:]) * np.exp(1j * pos * theta ** (-2.0 * np.arange(D // 2) / D))
    np.testing.assert_allclose(oracle.rope(v, theta, pos), np.concatenate([z.real, z.imag]), rtol=1e-9,
                               atol=1e-12)


def test_rope_relative_position_and_identity():
    D, theta = 32, 10000.0
    r = rng(32)
    q, k = r.standard_normal(D), r.standard_normal(D)
    assert np.array_equal(oracle.rope(q, theta, 0), q)
    d1 = oracle.rope(q, theta, 40) @ oracle.rope(k, theta, 33)
    d2 = oracle.rope(q, theta, 107) @ oracle.rope(k, theta, 100)
    assert abs(d1 - d2) < 1e-9


def test_lm_head_argmax_matches_numpy_and_breaks_ties_low():
    r = rng(33)
    W = r.standard_normal((500, 24)).astype(np.float32)
    W[400] = W[17]  # duplicate row: ties with id 17 whenever 17 is the maximum
    h = r.standard_normal((6, 24)).astype(np.float32)
    h[0] = W[17]  # makes 17 (and 400) the maximum for row 0
    am, t1, t2 = oracle.lm_head_argmax(f32(h), f32(W))
    logits = h.astype(np.float64) @ W.astype(np.float64).T
    assert np.array_equal(am, logits.argmax(1))  # numpy returns the first maximum
    assert am[0] == 17
    srt = np.sort(logits, 1)
    np.testing.assert_allclose(t1, srt[:, -1], rtol=1e-13)
    np.testing.assert_allclose(t2, srt[:, -2], rtol=1e-13)
