"""ctypes front-end of the CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg import
this module.  It converts torch CPU tensors / numpy arrays into the raw pointers the
C++ oracle takes and returns float64 numpy arrays.  It never imports the product
package, and the product never imports it.
"""
from __future__ import annotations

import ctypes as ct
import os

import numpy as np
import torch

from . import build as _build

F32, BF16 = 0, 1
_lib = None


def lib():
    global _lib
    if _lib is None:
        # HSPEC_ORACLE_LIB loads another build of this same source instead (the mutation
        # test builds copies with one planted mistake each and checks that a pin fails)
        _lib = ct.CDLL(os.environ.get("HSPEC_ORACLE_LIB") or _build.build())
        _lib.oracle_bf16_round.restype = ct.c_double
        _lib.oracle_bf16_round.argtypes = [ct.c_double]
        for name in ("oracle_attn_paged", "oracle_draft_step"):
            getattr(_lib, name).restype = ct.c_int
    return _lib


def threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS or all cores)."""
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


# --------------------------------------------------------------- marshalling

def _cpu(t):
    """-> (contiguous CPU tensor kept alive, element type tag)."""
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(np.ascontiguousarray(t))
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t, BF16
    if t.dtype == torch.float64:
        raise TypeError("oracle inputs are stored as float32 or bfloat16; got float64")
    return t.to(torch.float32), F32


def _ptr(t):
    return ct.c_void_p(t.data_ptr()) if t is not None else None


def _f32(t):
    t = torch.as_tensor(t).detach().to("cpu", torch.float32).contiguous()
    return t


def _i32(t):
    return torch.as_tensor(t).detach().to("cpu", torch.int32).contiguous()


def _f64_out(*shape):
    return np.zeros(shape, dtype=np.float64)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ct.c_void_p)


# --------------------------------------------------------------------- calls

def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty_like(a)
    lib().oracle_bf16_round_array(ct.c_long(a.size), _dptr(a), _dptr(out))
    return out


def inject(W_inj, h_last) -> np.ndarray:
    """h0 = W_inj h_last per request -> [C, H*P*N] (reshape row-major to [H,P,N])."""
    W, wt = _cpu(W_inj)
    h, ht = _cpu(h_last)
    HPN, d = W.shape
    C = h.shape[0]
    out = _f64_out(C, HPN)
    lib().oracle_inject(HPN, d, _ptr(W), wt, _ptr(h), ht, C, _dptr(out))
    return out


def ssd_scan(x, dt, A, B, Cm, D, h0=None, want_state=False):
    """Sequential recurrence. x [C,K,H,P]; dt [C,K,H]; A, D [H]; B, Cm [C,K,N]; h0 [C,H,P,N]."""
    xx, xt = _cpu(x)
    Bb, bt = _cpu(B)
    Cc, ct_ = _cpu(Cm)
    assert bt == ct_
    C, K, H, P = xx.shape
    N = Bb.shape[-1]
    dtt, AA, DD = _f32(dt), _f32(A), _f32(D)
    hh = _f32(h0) if h0 is not None else None
    y = _f64_out(C, K, H, P)
    hK = _f64_out(C, H, P, N) if want_state else None
    lib().oracle_ssd_scan(C, K, H, P, N, _ptr(xx), xt, _ptr(dtt), _ptr(AA), _ptr(Bb), _ptr(Cc), bt,
                          _ptr(DD), _ptr(hh), _dptr(y), _dptr(hK) if hK is not None else None)
    return (y, hK) if want_state else y


def attn_paged(q, k_pool, v_pool, page_table, ctx_lens, k_blk, v_blk, causal_block=False):
    qq, dt = _cpu(q)
    kp, _ = _cpu(k_pool)
    vp, _ = _cpu(v_pool)
    kb, _ = _cpu(k_blk)
    vb, _ = _cpu(v_blk)
    tbl, lens = _i32(page_table), _i32(ctx_lens)
    C, K, Hq, D = qq.shape
    num_pages, page, Hkv, _ = kp.shape
    out = _f64_out(C, K, Hq, D)
    rc = lib().oracle_attn_paged(C, K, Hq, Hkv, D, page, _ptr(qq), _ptr(kp), _ptr(vp), dt, num_pages,
                                 _ptr(tbl), tbl.shape[1], _ptr(lens), _ptr(kb), _ptr(vb),
                                 int(causal_block), _dptr(out))
    if rc != 0:
        raise ValueError("oracle_attn_paged: page table or context length out of range")
    return out


def attn_contiguous(q, k_ctx, v_ctx, ctx_lens, k_blk, v_blk, causal_block=False):
    qq, dt = _cpu(q)
    kc, _ = _cpu(k_ctx)
    vc, _ = _cpu(v_ctx)
    kb, _ = _cpu(k_blk)
    vb, _ = _cpu(v_blk)
    lens = _i32(ctx_lens)
    C, K, Hq, D = qq.shape
    max_ctx, Hkv = kc.shape[1], kc.shape[2]
    out = _f64_out(C, K, Hq, D)
    lib().oracle_attn_contiguous(C, K, Hq, Hkv, D, _ptr(qq), _ptr(kc), _ptr(vc), dt, max_ctx,
                                 _ptr(lens), _ptr(kb), _ptr(vb), int(causal_block), _dptr(out))
    return out


def rmsnorm(x, w, eps=1e-6) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    rows, n = a.reshape(-1, a.shape[-1]).shape
    ww = _f32(w)
    out = np.empty_like(a)
    lib().oracle_rmsnorm(rows, n, _dptr(a), _ptr(ww), ct.c_double(eps), _dptr(out))
    return out


def rope(v, theta, pos) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.empty_like(a)
    lib().oracle_rope(a.shape[-1], ct.c_double(theta), ct.c_long(int(pos)), _dptr(a), _dptr(out))
    return out


def lm_head_argmax(hn, W_lm):
    """hn [rows, d], W_lm [V, d] -> (argmax int32 [rows], top1 [rows], top2 [rows])."""
    h, ht = _cpu(hn)
    W, wt = _cpu(W_lm)
    h2 = h.reshape(-1, h.shape[-1])
    rows, d = h2.shape
    V = W.shape[0]
    am = np.zeros(rows, dtype=np.int32)
    t1, t2 = _f64_out(rows), _f64_out(rows)
    lib().oracle_lm_head_argmax(rows, d, V, _ptr(h2), ht, _ptr(W), wt, _dptr(am), _dptr(t1), _dptr(t2))
    return am, t1, t2


def verify_greedy(logits, drafts, ctx_lens=None):
    """logits [C, K+1, V] (fp32 or bf16), drafts [C, K] int32 -> (accepted [C], next_token
    [C], new ctx_lens [C] or None).  See oracle_verify_greedy."""
    lg, lt = _cpu(logits)
    dr = _i32(drafts)
    C, K1, V = lg.shape
    K = K1 - 1
    assert tuple(dr.shape) == (C, K)
    acc = np.zeros(C, dtype=np.int32)
    nxt = np.zeros(C, dtype=np.int32)
    ctx = None if ctx_lens is None else _i32(ctx_lens).numpy().copy()
    lib().oracle_verify_greedy(C, K, V, _ptr(lg), lt, _ptr(dr), _dptr(acc), _dptr(nxt),
                               _dptr(ctx) if ctx is not None else None)
    return acc, nxt, ctx


# ------------------------------------------------------------ host copies

def host_weights(w: dict) -> dict:
    """Host copy of a weights dict (inputs.make_weights layout)."""
    cpu = lambda v: v.detach().to("cpu") if torch.is_tensor(v) else v
    return {"layers": [{k: cpu(v) for k, v in L.items()} for L in w["layers"]],
            **{k: cpu(v) for k, v in w.items() if k != "layers"}}


def host_sub_cache(cache: dict, rows) -> dict:
    """Host copy of the pages that `rows` of the page table use, with the table
    rewritten to the copied order (the oracle still gathers through the table)."""
    tbl = cache["page_table"].detach().to("cpu")[rows]
    used = tbl[tbl >= 0].unique()
    remap = torch.full((int(cache["k_pool"].shape[0]),), -1, dtype=torch.int32)
    remap[used.long()] = torch.arange(used.numel(), dtype=torch.int32)
    new_tbl = torch.where(tbl >= 0, remap[tbl.clamp(min=0).long()], tbl)
    idx = used.long().to(cache["k_pool"].device)
    return {"k_pool": cache["k_pool"].index_select(0, idx).to("cpu"),
            "v_pool": cache["v_pool"].index_select(0, idx).to("cpu"),
            "page_table": new_tbl.contiguous()}


# ----------------------------------------------------------------- draft step

class _Cfg(ct.Structure):
    _fields_ = [(n, ct.c_int) for n in ("d", "Hq", "Hkv", "D", "H", "P", "N", "page", "d_ff",
                                         "vocab", "n_layers")] + [
        ("kinds", ct.c_char * 16), ("rope_theta", ct.c_double), ("eps", ct.c_double),
        ("dtype", ct.c_int), ("use_rope", ct.c_int), ("use_gate", ct.c_int),
        ("causal_block", ct.c_int), ("mask_token", ct.c_int)]


class _Layer(ct.Structure):
    _fields_ = [("norm", ct.c_void_p), ("W_in", ct.c_void_p), ("dt_bias", ct.c_void_p),
                ("A", ct.c_void_p), ("D", ct.c_void_p), ("gnorm", ct.c_void_p),
                ("W_out", ct.c_void_p), ("W_inj", ct.c_void_p), ("W_qkv", ct.c_void_p),
                ("W_o", ct.c_void_p), ("k_pool", ct.c_void_p), ("v_pool", ct.c_void_p),
                ("num_pages", ct.c_int), ("page_table", ct.c_void_p), ("max_pages", ct.c_int),
                ("mlp_norm", ct.c_void_p), ("W_gate", ct.c_void_p), ("W_up", ct.c_void_p),
                ("W_down", ct.c_void_p)]


class _Step(ct.Structure):
    _fields_ = [("C", ct.c_int), ("K", ct.c_int), ("tokens", ct.c_void_p), ("x_in", ct.c_void_p),
                ("x_in_type", ct.c_int), ("h_last", ct.c_void_p), ("ctx_lens", ct.c_void_p), ("final_norm", ct.c_void_p),
                ("W_lm", ct.c_void_p), ("draft_vocab", ct.c_int), ("W_lm_draft", ct.c_void_p),
                ("draft_to_target", ct.c_void_p), ("hidden", ct.c_void_p), ("layer_out", ct.c_void_p),
                ("final_normed", ct.c_void_p), ("draft_tokens", ct.c_void_p), ("top1", ct.c_void_p),
                ("top2", ct.c_void_p)]


def draft_step(shapes, weights, kv, h_last, ctx_lens, tokens=None, x_in=None, layer_outputs=False):
    """One draft step of the drafter `shapes` (see inputs.Shapes) over the requests
    given (any subset of a batch: requests are independent).

    weights: inputs.make_weights() layout; kv: one dict per attention layer with
    k_pool, v_pool, page_table (rows for exactly these requests); h_last [C,d];
    ctx_lens [C]; tokens [C,K] (with an LM head) or x_in [C,K,d] (without).
    Returns a dict of float64 / int32 numpy arrays.
    """
    sh = shapes
    keep = []

    def hold(t, f32=False):
        if t is None:
            return None
        t2 = _f32(t) if f32 else _cpu(t)[0]
        keep.append(t2)
        return t2.data_ptr()

    cfg = _Cfg(d=sh.d, Hq=sh.Hq, Hkv=sh.Hkv, D=sh.D, H=sh.H, P=sh.P, N=sh.N, page=sh.page,
               d_ff=sh.d_ff, vocab=sh.vocab, n_layers=len(sh.layers), kinds=sh.layers.encode(),
               rope_theta=sh.rope_theta, eps=sh.eps, dtype=F32 if sh.dtype == "f32" else BF16,
               use_rope=int(sh.use_rope), use_gate=int(sh.use_gate),
               causal_block=int(sh.causal_block), mask_token=sh.mask_token)
    layers = (_Layer * len(sh.layers))()
    ai = 0
    for li, w in enumerate(weights["layers"]):
        L = layers[li]
        L.norm = hold(w["norm"], True)
        if w["kind"] == "M":
            L.W_in, L.W_out, L.W_inj = hold(w["W_in"]), hold(w["W_out"]), hold(w["W_inj"])
            L.dt_bias, L.A, L.D = hold(w["dt_bias"], True), hold(w["A"], True), hold(w["D"], True)
            L.gnorm = hold(w["gnorm"], True)
        else:
            L.W_qkv, L.W_o = hold(w["W_qkv"]), hold(w["W_o"])
            cache = kv[ai]
            ai += 1
            L.k_pool, L.v_pool = hold(cache["k_pool"]), hold(cache["v_pool"])
            L.num_pages = int(cache["k_pool"].shape[0])
            tbl = _i32(cache["page_table"])
            keep.append(tbl)
            L.page_table, L.max_pages = tbl.data_ptr(), int(tbl.shape[1])
        if sh.d_ff:
            L.mlp_norm = hold(w["mlp_norm"], True)
            L.W_gate, L.W_up, L.W_down = hold(w["W_gate"]), hold(w["W_up"]), hold(w["W_down"])
    lens = _i32(ctx_lens)
    C = lens.numel()
    K = (tokens if tokens is not None else x_in).shape[1]
    res = {"hidden": _f64_out(C, K, sh.d)}
    if layer_outputs:
        res["layer_out"] = _f64_out(len(sh.layers), C, K, sh.d)
    io = _Step(C=C, K=K, ctx_lens=lens.data_ptr(), h_last=hold(h_last),
               hidden=_dptr(res["hidden"]).value,
               layer_out=_dptr(res["layer_out"]).value if layer_outputs else None)
    if sh.vocab:
        tok = _i32(tokens)
        keep.append(tok)
        io.tokens = tok.data_ptr()
        io.final_norm = hold(weights["final_norm"], True)
        io.W_lm = hold(weights["W_lm"])
        if getattr(sh, "draft_vocab", 0):
            io.draft_vocab = sh.draft_vocab
            io.W_lm_draft = hold(weights["W_lm_draft"])
            d2t = _i32(weights["draft_to_target"])
            keep.append(d2t)
            io.draft_to_target = d2t.data_ptr()
        res["final_normed"] = _f64_out(C, K, sh.d)
        res["draft_tokens"] = np.zeros((C, K), dtype=np.int32)
        res["top1"], res["top2"] = _f64_out(C, K), _f64_out(C, K)
        io.final_normed = _dptr(res["final_normed"]).value
        io.draft_tokens = _dptr(res["draft_tokens"]).value
        io.top1, io.top2 = _dptr(res["top1"]).value, _dptr(res["top2"]).value
    else:
        xt, io.x_in_type = _cpu(x_in)
        keep.append(xt)
        io.x_in = xt.data_ptr()
    rc = lib().oracle_draft_step(ct.byref(cfg), layers, ct.byref(io))
    if rc != 0:
        raise ValueError("oracle_draft_step: page table or context length out of range")
    return res
