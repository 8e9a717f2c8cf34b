"""ctypes binding of libhspec.so -- the C-ABI declared in include/hspec.h.

Argument marshalling only: every step of the draft step runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors passed by data_ptr(); streams default to
torch's current stream.  Importing this module loads the library and fails loudly
(ImportError) if it cannot be built or loaded -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes as ct
import os

import torch

from . import build as _build

HSPEC_OK = 0
HSPEC_ERR_INVALID_ARG = 1
HSPEC_ERR_SHAPE_MISMATCH = 2
HSPEC_ERR_PAGE_OOB = 3
HSPEC_ERR_UNSUPPORTED = 4
HSPEC_ERR_CUDA = 5
HSPEC_ERR_DEVICE_CHECK = 6
HSPEC_ERR_WORKSPACE = 7

HSPEC_DTYPE_F32 = 0
HSPEC_DTYPE_BF16 = 1
HSPEC_FLAG_ROPE = 1
HSPEC_FLAG_GATE = 2
HSPEC_FLAG_CAUSAL_BLOCK = 4
HSPEC_FLAG_FUSE_INJECT = 8
HSPEC_MAX_LAYERS = 16

# Every function include/hspec.h declares (checked by the CPU export test).
EXPORTS = ("hspec_inject_state", "hspec_ssd_block_scan", "hspec_attn_workspace_size",
           "hspec_attn_paged_block", "hspec_drafter_create", "hspec_drafter_destroy",
           "hspec_step_workspace_size", "hspec_draft_step", "hspec_sync_status",
           "hspec_status_string", "hspec_last_error", "hspec_launch_count", "hspec_version",
           "hspec_profile_enable", "hspec_profile_read", "hspec_attn_paged_block_noalloc",
           "hspec_verify_workspace_size", "hspec_verify_greedy")
HSPEC_NOALLOC_SCRATCH_BYTES = 64 << 20


class HspecError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.hspec_status_string(status).decode()} "
                         f"({_lib.hspec_last_error().decode()})")


# ------------------------------------------------------------------ structs

class hspec_cfg(ct.Structure):
    _fields_ = [("d_model", ct.c_int), ("n_q_heads", ct.c_int), ("n_kv_heads", ct.c_int),
                ("head_dim", ct.c_int), ("n_ssm_heads", ct.c_int), ("ssm_head_dim", ct.c_int),
                ("d_state", ct.c_int), ("page_size", ct.c_int), ("d_ff", ct.c_int), ("vocab", ct.c_int),
                ("n_layers", ct.c_int), ("layer_kinds", ct.c_char * HSPEC_MAX_LAYERS),
                ("dtype", ct.c_int), ("flags", ct.c_int), ("rope_theta", ct.c_float),
                ("norm_eps", ct.c_float), ("ssd_chunk", ct.c_int), ("attn_split_tokens", ct.c_int),
                ("draft_vocab", ct.c_int), ("wait_limit_ns", ct.c_longlong)]


class hspec_layer_weights(ct.Structure):
    _fields_ = [(n, ct.c_void_p) for n in ("norm", "W_in", "dt_bias", "A", "D", "gnorm", "W_out", "W_inj",
                                           "W_qkv", "W_o", "mlp_norm", "W_gate", "W_up", "W_down")]


class hspec_model_weights(ct.Structure):
    _fields_ = [("layers", hspec_layer_weights * HSPEC_MAX_LAYERS), ("final_norm", ct.c_void_p),
                ("W_lm", ct.c_void_p), ("W_lm_draft", ct.c_void_p), ("draft_to_target", ct.c_void_p)]


class hspec_kv_view(ct.Structure):
    _fields_ = [("k_pool", ct.c_void_p), ("v_pool", ct.c_void_p), ("num_pages", ct.c_int),
                ("page_table", ct.c_void_p), ("max_pages", ct.c_int)]


class hspec_step_in(ct.Structure):
    _fields_ = [("C", ct.c_int), ("K", ct.c_int), ("tokens", ct.c_void_p), ("x_in", ct.c_void_p),
                ("h_last", ct.c_void_p), ("ctx_lens", ct.c_void_p),
                ("kv", hspec_kv_view * HSPEC_MAX_LAYERS)]


class hspec_step_out(ct.Structure):
    _fields_ = [("draft_tokens", ct.c_void_p), ("hidden", ct.c_void_p), ("final_normed", ct.c_void_p),
                ("top_logit", ct.c_void_p), ("layer_hidden", ct.c_void_p)]


# ------------------------------------------------------------------ library

def _load():
    path = _build.build()
    lib = ct.CDLL(path)
    P, I, Z, V = ct.c_void_p, ct.c_int, ct.c_size_t, ct.c_void_p
    cfgp = ct.POINTER(hspec_cfg)
    sig = {
        "hspec_inject_state": (I, [cfgp, P, P, I, P, V]),
        "hspec_ssd_block_scan": (I, [cfgp, P, P, P, P, P, P, P, I, I, P, P, V]),
        "hspec_attn_workspace_size": (Z, [cfgp, I, I, I]),
        "hspec_attn_paged_block": (I, [cfgp, P, ct.POINTER(hspec_kv_view), P, P, P, I, I, P, P, Z, V]),
        "hspec_drafter_create": (I, [cfgp, ct.POINTER(hspec_model_weights), ct.POINTER(ct.c_void_p)]),
        "hspec_drafter_destroy": (None, [P]),
        "hspec_step_workspace_size": (Z, [cfgp, I, I, I]),
        "hspec_draft_step": (I, [P, ct.POINTER(hspec_step_in), ct.POINTER(hspec_step_out), P, Z, V]),
        "hspec_sync_status": (I, [V]),
        "hspec_status_string": (ct.c_char_p, [I]),
        "hspec_last_error": (ct.c_char_p, []),
        "hspec_launch_count": (ct.c_ulonglong, []),
        "hspec_version": (ct.c_char_p, []),
        "hspec_profile_enable": (I, [I]),
        "hspec_profile_read": (I, [P, P, P, I]),
        "hspec_attn_paged_block_noalloc": (I, [cfgp, P, ct.POINTER(hspec_kv_view), P, P, P, I, I, P, V]),
        "hspec_verify_workspace_size": (Z, [cfgp, I, I]),
        "hspec_verify_greedy": (I, [cfgp, P, P, I, I, P, P, P, P, Z, V]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib, path


try:
    _lib, LIBRARY_PATH = _load()
except Exception as e:  # no silent fallback: the CUDA library is the product
    raise ImportError(f"libhspec.so could not be built or loaded: {e}") from e


def _check(status: int, where: str):
    if status != HSPEC_OK:
        raise HspecError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --------------------------------------------------------------- config helpers

def make_cfg(shapes, ssd_chunk: int = 0, attn_split_tokens: int = 0, fuse_inject: bool = False,
             wait_limit_ns: int = 0) -> hspec_cfg:
    """hspec_cfg from an inputs.Shapes (or any object with the same fields)."""
    sh = shapes
    flags = (HSPEC_FLAG_ROPE if sh.use_rope else 0) | (HSPEC_FLAG_GATE if sh.use_gate else 0) | (
        HSPEC_FLAG_CAUSAL_BLOCK if sh.causal_block else 0) | (HSPEC_FLAG_FUSE_INJECT if fuse_inject else 0)
    return hspec_cfg(d_model=sh.d, n_q_heads=sh.Hq, n_kv_heads=sh.Hkv, head_dim=sh.D, n_ssm_heads=sh.H,
                     ssm_head_dim=sh.P, d_state=sh.N, page_size=sh.page, d_ff=sh.d_ff, vocab=sh.vocab,
                     n_layers=len(sh.layers), layer_kinds=sh.layers.encode(),
                     dtype=HSPEC_DTYPE_F32 if sh.dtype == "f32" else HSPEC_DTYPE_BF16, flags=flags,
                     rope_theta=sh.rope_theta, norm_eps=sh.eps, ssd_chunk=ssd_chunk,
                     attn_split_tokens=attn_split_tokens, draft_vocab=getattr(sh, "draft_vocab", 0),
                     wait_limit_ns=wait_limit_ns)


def kv_view(cache: dict) -> hspec_kv_view:
    """hspec_kv_view of a target cache dict (k_pool, v_pool, page_table)."""
    return hspec_kv_view(k_pool=_ptr(cache["k_pool"]), v_pool=_ptr(cache["v_pool"]),
                         num_pages=int(cache["k_pool"].shape[0]), page_table=_ptr(cache["page_table"]),
                         max_pages=int(cache["page_table"].shape[1]))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A 256-byte aligned device buffer (torch's caching allocator aligns to 512)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


# ------------------------------------------------------------------- entry points

def hspec_inject_state(cfg: hspec_cfg, W_inj, h_last, h0, stream=None):
    _check(_lib.hspec_inject_state(ct.byref(cfg), _ptr(W_inj), _ptr(h_last), int(h_last.shape[0]), _ptr(h0),
                                   _stream(stream)), "hspec_inject_state")


def hspec_ssd_block_scan(cfg: hspec_cfg, x, dt, A, B, Cm, D, h0, y, hK=None, stream=None):
    C, K = int(x.shape[0]), int(x.shape[1])
    _check(_lib.hspec_ssd_block_scan(ct.byref(cfg), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(Cm), _ptr(D),
                                     _ptr(h0), C, K, _ptr(y), _ptr(hK), _stream(stream)),
           "hspec_ssd_block_scan")


def hspec_attn_workspace_size(cfg: hspec_cfg, C: int, K: int, max_pages: int) -> int:
    return int(_lib.hspec_attn_workspace_size(ct.byref(cfg), C, K, max_pages))


def hspec_attn_paged_block(cfg: hspec_cfg, q, kv: hspec_kv_view, ctx_lens, k_blk, v_blk, out, workspace,
                           stream=None):
    C, K = int(q.shape[0]), int(q.shape[1])
    _check(_lib.hspec_attn_paged_block(ct.byref(cfg), _ptr(q), ct.byref(kv), _ptr(ctx_lens), _ptr(k_blk),
                                       _ptr(v_blk), C, K, _ptr(out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)),
           "hspec_attn_paged_block")


def hspec_verify_workspace_size(cfg: hspec_cfg, C: int, K: int) -> int:
    return int(_lib.hspec_verify_workspace_size(ct.byref(cfg), C, K))


def hspec_verify_greedy(cfg: hspec_cfg, logits, drafts, accepted, next_token, workspace, ctx_lens=None,
                        stream=None):
    """Greedy verification: logits [C, K+1, cfg.vocab] (cfg dtype), drafts [C, K] int32;
    writes accepted [C] and next_token [C] (int32) and advances ctx_lens [C] in place when
    given."""
    C, K = int(drafts.shape[0]), int(drafts.shape[1])
    _check(_lib.hspec_verify_greedy(ct.byref(cfg), _ptr(logits), _ptr(drafts), C, K, _ptr(accepted),
                                    _ptr(next_token), _ptr(ctx_lens) if ctx_lens is not None else None,
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)),
           "hspec_verify_greedy")


def hspec_attn_paged_block_noalloc(cfg: hspec_cfg, q, kv: hspec_kv_view, ctx_lens, k_blk, v_blk, out,
                                   stream=None):
    """hspec_attn_paged_block without a workspace argument: the split partials live in
    the library's static scratch (HSPEC_NOALLOC_SCRATCH_BYTES); for callers that
    cannot allocate device memory.  Calls that overlap on the GPU race on it."""
    C, K = int(q.shape[0]), int(q.shape[1])
    _check(_lib.hspec_attn_paged_block_noalloc(ct.byref(cfg), _ptr(q), ct.byref(kv), _ptr(ctx_lens), _ptr(k_blk),
                                               _ptr(v_blk), C, K, _ptr(out), _stream(stream)),
           "hspec_attn_paged_block_noalloc")


def hspec_drafter_create(cfg: hspec_cfg, weights: hspec_model_weights) -> ct.c_void_p:
    h = ct.c_void_p()
    _check(_lib.hspec_drafter_create(ct.byref(cfg), ct.byref(weights), ct.byref(h)), "hspec_drafter_create")
    return h


def hspec_drafter_destroy(handle):
    _lib.hspec_drafter_destroy(handle)


def hspec_step_workspace_size(cfg: hspec_cfg, C: int, K: int, max_pages: int) -> int:
    return int(_lib.hspec_step_workspace_size(ct.byref(cfg), C, K, max_pages))


def hspec_draft_step(handle, step_in: hspec_step_in, step_out: hspec_step_out, workspace, stream=None):
    _check(_lib.hspec_draft_step(handle, ct.byref(step_in), ct.byref(step_out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "hspec_draft_step")


def hspec_sync_status(stream=None) -> int:
    return int(_lib.hspec_sync_status(_stream(stream)))


def hspec_status_string(status: int) -> str:
    return _lib.hspec_status_string(status).decode()


def hspec_last_error() -> str:
    return _lib.hspec_last_error().decode()


def hspec_launch_count() -> int:
    return int(_lib.hspec_launch_count())


def hspec_version() -> str:
    return _lib.hspec_version().decode()


def hspec_profile_enable(on: bool):
    _check(_lib.hspec_profile_enable(int(bool(on))), "hspec_profile_enable")


def hspec_profile_read(max_entries: int = 64) -> dict:
    """{kernel group: (total_ms, occurrences)} recorded since hspec_profile_enable(True)."""
    names = ct.create_string_buffer(32 * max_entries)
    ms = (ct.c_double * max_entries)()
    cnt = (ct.c_int * max_entries)()
    n = _lib.hspec_profile_read(names, ms, cnt, max_entries)
    if n < 0:
        raise HspecError(HSPEC_ERR_CUDA, "hspec_profile_read")
    raw = names.raw
    return {raw[32 * i:32 * i + 32].split(b"\0", 1)[0].decode(): (ms[i], cnt[i]) for i in range(n)}


# ------------------------------------------------------------- drafter wrapper

class Drafter:
    """Holds a drafter handle plus the weights it points at (kept alive here)."""

    def __init__(self, shapes, weights: dict, ssd_chunk: int = 0, attn_split_tokens: int = 0,
                 fuse_inject: bool = False, wait_limit_ns: int = 0):
        self.shapes = shapes
        self.cfg = make_cfg(shapes, ssd_chunk, attn_split_tokens, fuse_inject, wait_limit_ns)
        self.weights = weights
        mw = hspec_model_weights()
        for i, w in enumerate(weights["layers"]):
            L = mw.layers[i]
            for name, _ in hspec_layer_weights._fields_:
                if name in w:
                    setattr(L, name, _ptr(w[name]))
        if "final_norm" in weights:
            mw.final_norm = _ptr(weights["final_norm"])
            mw.W_lm = _ptr(weights["W_lm"])
        if "W_lm_draft" in weights:
            mw.W_lm_draft = _ptr(weights["W_lm_draft"])
            mw.draft_to_target = _ptr(weights["draft_to_target"])
        self._mw = mw
        self.handle = hspec_drafter_create(self.cfg, mw)

    def workspace_size(self, C: int, K: int, max_pages: int) -> int:
        return hspec_step_workspace_size(self.cfg, C, K, max_pages)

    def step_in(self, C, K, h_last, ctx_lens, kv_caches, tokens=None, x_in=None) -> hspec_step_in:
        si = hspec_step_in(C=C, K=K, tokens=_ptr(tokens), x_in=_ptr(x_in), h_last=_ptr(h_last),
                           ctx_lens=_ptr(ctx_lens))
        for i, cache in enumerate(kv_caches):
            si.kv[i] = kv_view(cache)
        return si

    def step(self, step_in: hspec_step_in, step_out: hspec_step_out, workspace, stream=None):
        hspec_draft_step(self.handle, step_in, step_out, workspace, stream)

    def close(self):
        if self.handle:
            hspec_drafter_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
