"""Seeded synthetic workloads for the H-Spec block-parallel draft step.

This module only draws random numbers with the shapes, sizes and value
distributions of the workloads; it holds none of the method's arithmetic.  It is
the one module that both the CPU oracle's tests and the CUDA path's tests and
benchmark use, so that both sides see identical inputs.

Workloads (the drafter sees a target model whose KV it reads in place and whose
last-token hidden state it projects into the Mamba-2 initial state, as the H-Spec
abstract describes):

  tiny       fp32, 1 request, target ctx 64, 4 q / 2 kv heads, head_dim 64, page 16;
             drafter d_model 256, one Mamba-2 layer (4 heads x 64, d_state 16) and one
             attention layer, block K=8; identity page table.
  llama_c1   Llama-3-8B-shaped target KV (32 q / 8 kv heads, head_dim 128,
             d_model 4096), bf16, 1 request, ctx 2048, shuffled page table; drafter
             M,A with Mamba-2 64 heads x 64, d_state 128, K=16.
  llama_c32  same shapes, 32 requests, ctx uniform 512..8192, pages randomly
             permuted across one shared pool.
  qwen_c128  Qwen-32B-shaped target KV (64 q / 8 kv heads, head_dim 128,
             d_model 5120), 128 requests, ctx uniform 1024..32768; Mamba-2 80 heads.
  full       4-layer M,A,M,A drafter on Llama shapes with RMSNorm, SwiGLU (4x) and a
             shared 128256-token LM head; K in {8,16,32} x C in {1,8,32,128},
             ctx uniform 512..16384; each attention layer reads its own KV pool.

Distributions: activations, KV, h_last, B, C, D ~ N(0,1); weight matrices
N(0, 1/fan_in); A = -exp(U[0, ln 16]); dt = softplus(N(-4, 1)) (the draft step
draws dt_bias = -4 so that softplus(dt_raw + dt_bias) has that law when dt_raw ~
N(0,1)); RMSNorm weights 1 + 0.1 N(0,1).  Shared pools carry 10% slack pages
filled with NaN so that a stray page read shows up in the output.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field, replace

import torch

PAGE = 16


@dataclass(frozen=True)
class Shapes:
    name: str
    d: int                  # d_model (drafter = target, the KV dims must match the target's)
    Hq: int                 # attention query heads
    Hkv: int                # attention kv heads (GQA group G = Hq // Hkv)
    D: int                  # attention head dim
    H: int                  # Mamba-2 heads
    P: int                  # Mamba-2 head dim
    N: int                  # Mamba-2 state size
    dtype: str              # "f32" or "bf16" (weights, activations, KV)
    rope_theta: float
    layers: str = "MA"      # layer kinds in order, M = Mamba-2, A = attention
    d_ff: int = 0           # SwiGLU intermediate size, 0 = no MLP sub-layer
    vocab: int = 0          # LM head rows, 0 = no head (output is the hidden state)
    draft_vocab: int = 0    # reduced draft head rows (0 = the full vocab head)
    page: int = PAGE
    eps: float = 1e-6
    use_rope: bool = True
    use_gate: bool = True
    causal_block: bool = False

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def in_proj_rows(self) -> int:
        # Mamba-2 in_proj output order: z (H*P), x (H*P), B (N), C (N), dt (H)
        return 2 * self.H * self.P + 2 * self.N + self.H

    @property
    def qkv_rows(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.D

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def mask_token(self) -> int:
        return max(self.vocab - 1, 0)


TINY = Shapes("tiny", d=256, Hq=4, Hkv=2, D=64, H=4, P=64, N=16, dtype="f32", rope_theta=1e4)
LLAMA = Shapes("llama8b", d=4096, Hq=32, Hkv=8, D=128, H=64, P=64, N=128, dtype="bf16",
               rope_theta=5e5)
QWEN = Shapes("qwen32b", d=5120, Hq=64, Hkv=8, D=128, H=80, P=64, N=128, dtype="bf16",
              rope_theta=1e6)
LLAMA_FULL = replace(LLAMA, name="llama8b_full", layers="MAMA", d_ff=16384, vocab=128256)


@dataclass(frozen=True)
class Workload:
    name: str
    shapes: Shapes
    C: int
    K: int
    ctx_lo: int
    ctx_hi: int
    seed: int
    shuffle: bool = True    # shuffled (True) or identity (False) page table
    slack: float = 0.10     # fraction of NaN-filled unused pages in the pool
    description: str = ""


WORKLOADS = {
    "tiny": Workload("tiny", TINY, C=1, K=8, ctx_lo=64, ctx_hi=64, seed=0, shuffle=False,
                     slack=0.0, description="tiny fp32, 1 request, ctx 64, K=8"),
    "llama_c1": Workload("llama_c1", LLAMA, C=1, K=16, ctx_lo=2048, ctx_hi=2048, seed=1,
                         description="Llama-3-8B shapes, bf16, 1 request, ctx 2048, K=16"),
    "llama_c32": Workload("llama_c32", LLAMA, C=32, K=16, ctx_lo=512, ctx_hi=8192, seed=2,
                          description="Llama-3-8B shapes, bf16, 32 requests, ctx U[512,8192], K=16"),
    "qwen_c128": Workload("qwen_c128", QWEN, C=128, K=16, ctx_lo=1024, ctx_hi=32768, seed=3,
                          description="Qwen-32B shapes, bf16, 128 requests, ctx U[1024,32768], K=16"),
    "full": Workload("full", LLAMA_FULL, C=128, K=16, ctx_lo=512, ctx_hi=16384, seed=4,
                     description="4-layer M,A,M,A drafter, Llama-3-8B shapes, SwiGLU 16384, "
                                 "vocab 128256, ctx U[512,16384]"),
}

FULL_SWEEP_K = (8, 16, 32)
FULL_SWEEP_C = (1, 8, 32, 128)


def full_workload(C: int, K: int, draft_vocab: int = 0) -> Workload:
    """One point of the full-step sweep (K in {8,16,32} x C in {1,8,32,128}); with
    draft_vocab, the same drafter with a reduced draft head of that many rows."""
    wl = replace(WORKLOADS["full"], C=C, K=K, name=f"full_C{C}_K{K}")
    if draft_vocab:
        wl = replace(wl, shapes=replace(wl.shapes, draft_vocab=draft_vocab), name=f"full_C{C}_K{K}_V{draft_vocab}")
    return wl


# ----------------------------------------------------------------------------- rng

def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + zlib.crc32(name.encode())) & 0x7FFF_FFFF_FFFF)
    return g


_CHUNK = 1 << 26


def _randn(shape, std, dtype, device, seed, name, mean=0.0) -> torch.Tensor:
    """N(mean, std^2) drawn in fp32 and stored in `dtype`; filled in chunks so a
    multi-GB bf16 weight never needs a full fp32 copy."""
    g = _gen(seed, name, device)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        tmp = torch.randn(e - s, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        if mean != 0.0:
            tmp.add_(mean)
        flat[s:e].copy_(tmp)
    return out


def _rand(shape, lo, hi, device, seed, name) -> torch.Tensor:
    g = _gen(seed, name, device)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


# ------------------------------------------------------------------------- weights

def make_weights(sh: Shapes, seed: int, device="cpu") -> dict:
    """Random-init drafter weights: {'layers': [dict per layer], 'final_norm', 'W_lm'}.

    Matrices are row-major [out, in] in the workload dtype; A, D, dt_bias and all
    RMSNorm weights are fp32.  The LM head is shared with the target and tied to the
    embedding table (one [vocab, d] matrix).
    """
    dt = sh.torch_dtype
    HP, HPN = sh.H * sh.P, sh.H * sh.P * sh.N
    layers = []
    for li, kind in enumerate(sh.layers):
        p = f"L{li}."
        w = {"kind": kind}
        w["norm"] = _randn((sh.d,), 0.1, torch.float32, device, seed, p + "norm", mean=1.0)
        if kind == "M":
            w["W_in"] = _randn((sh.in_proj_rows, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, p + "W_in")
            w["dt_bias"] = torch.full((sh.H,), -4.0, dtype=torch.float32, device=device)
            w["A"] = -torch.exp(_rand((sh.H,), 0.0, math.log(16.0), device, seed, p + "A"))
            w["D"] = _randn((sh.H,), 1.0, torch.float32, device, seed, p + "D")
            w["gnorm"] = _randn((HP,), 0.1, torch.float32, device, seed, p + "gnorm", mean=1.0)
            w["W_out"] = _randn((sh.d, HP), 1 / math.sqrt(HP), dt, device, seed, p + "W_out")
            w["W_inj"] = _randn((HPN, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, p + "W_inj")
        elif kind == "A":
            w["W_qkv"] = _randn((sh.qkv_rows, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, p + "W_qkv")
            w["W_o"] = _randn((sh.d, sh.Hq * sh.D), 1 / math.sqrt(sh.Hq * sh.D), dt, device, seed, p + "W_o")
        else:
            raise ValueError(f"unknown layer kind {kind!r}")
        if sh.d_ff:
            w["mlp_norm"] = _randn((sh.d,), 0.1, torch.float32, device, seed, p + "mlp_norm", mean=1.0)
            w["W_gate"] = _randn((sh.d_ff, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, p + "W_gate")
            w["W_up"] = _randn((sh.d_ff, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, p + "W_up")
            w["W_down"] = _randn((sh.d, sh.d_ff), 1 / math.sqrt(sh.d_ff), dt, device, seed, p + "W_down")
        layers.append(w)
    out = {"layers": layers}
    if sh.vocab:
        out["final_norm"] = _randn((sh.d,), 0.1, torch.float32, device, seed, "final_norm", mean=1.0)
        out["W_lm"] = _randn((sh.vocab, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, "W_lm")
        if sh.draft_vocab:
            # reduced draft head: its own rows, each standing for one target token (a seeded
            # subset of the vocabulary, in increasing id order)
            out["W_lm_draft"] = _randn((sh.draft_vocab, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, "W_lm_draft")
            g = _gen(seed, "draft_to_target", "cpu")
            ids = torch.randperm(sh.vocab, generator=g)[: sh.draft_vocab].sort().values
            out["draft_to_target"] = ids.to(torch.int32).to(device)
    return out


# ---------------------------------------------------------------------- paged KV

def make_ctx_lens(wl: Workload, device="cpu") -> torch.Tensor:
    g = _gen(wl.seed, "ctx_lens", "cpu")
    lens = torch.randint(wl.ctx_lo, wl.ctx_hi + 1, (wl.C,), generator=g, dtype=torch.int32)
    return lens.to(device)


def make_paged_kv(sh: Shapes, ctx_lens: torch.Tensor, seed: int, device="cpu", shuffle=True,
                  slack=0.10, tag="kv", max_pages=None) -> dict:
    """A target-owned paged KV cache: K and V pools [num_pages, page, Hkv, D], a page
    table [C, max_pages] int32 (unused entries -1) and ctx_lens [C] int32.

    Pages of all requests are drawn as one random permutation of a shared pool
    (shuffle=True) or laid out in order (shuffle=False).  Slack pages that no
    request owns are filled with NaN.
    """
    lens = ctx_lens.to("cpu", torch.int64)
    C = lens.numel()
    n_pages = [(int(l) + sh.page - 1) // sh.page for l in lens]
    used = sum(n_pages)
    n_slack = int(math.ceil(used * slack)) if slack > 0 else 0
    total = max(used + n_slack, 1)
    if max_pages is None:
        max_pages = max(max(n_pages) if n_pages else 0, 1)
    g = _gen(seed, tag + ".perm", "cpu")
    order = torch.randperm(total, generator=g) if shuffle else torch.arange(total)
    table = torch.full((C, max_pages), -1, dtype=torch.int32)
    off = 0
    for c in range(C):
        table[c, :n_pages[c]] = order[off:off + n_pages[c]].to(torch.int32)
        off += n_pages[c]
    slack_ids = order[off:]
    dt = sh.torch_dtype
    k_pool = _randn((total, sh.page, sh.Hkv, sh.D), 1.0, dt, device, seed, tag + ".k")
    v_pool = _randn((total, sh.page, sh.Hkv, sh.D), 1.0, dt, device, seed, tag + ".v")
    if slack_ids.numel():
        idx = slack_ids.to(device)
        k_pool[idx] = float("nan")
        v_pool[idx] = float("nan")
    return {"k_pool": k_pool, "v_pool": v_pool, "page_table": table.to(device),
            "ctx_lens": ctx_lens.to(device=device, dtype=torch.int32), "num_pages": total,
            "max_pages": max_pages}


# ------------------------------------------------------------- per-call inputs

def make_inject_inputs(sh: Shapes, C: int, seed: int, device="cpu") -> dict:
    dt = sh.torch_dtype
    return {"W_inj": _randn((sh.H * sh.P * sh.N, sh.d), 1 / math.sqrt(sh.d), dt, device, seed, "inj.W"),
            "h_last": _randn((C, sh.d), 1.0, dt, device, seed, "inj.h_last")}


def make_ssd_inputs(sh: Shapes, C: int, K: int, seed: int, device="cpu") -> dict:
    dt = sh.torch_dtype
    g = _gen(seed, "ssd.dt", device)
    dt_raw = torch.randn((C, K, sh.H), generator=g, device=device) - 4.0
    return {
        "x": _randn((C, K, sh.H, sh.P), 1.0, dt, device, seed, "ssd.x"),
        "dt": torch.nn.functional.softplus(dt_raw),
        "A": -torch.exp(_rand((sh.H,), 0.0, math.log(16.0), device, seed, "ssd.A")),
        "B": _randn((C, K, sh.N), 1.0, dt, device, seed, "ssd.B"),
        "Cm": _randn((C, K, sh.N), 1.0, dt, device, seed, "ssd.C"),
        "D": _randn((sh.H,), 1.0, torch.float32, device, seed, "ssd.D"),
        "h0": _randn((C, sh.H, sh.P, sh.N), 1.0, torch.float32, device, seed, "ssd.h0"),
    }


def make_attn_inputs(sh: Shapes, wl_or_lens, K: int, seed: int, device="cpu", shuffle=True,
                     slack=0.10) -> dict:
    lens = wl_or_lens if isinstance(wl_or_lens, torch.Tensor) else make_ctx_lens(wl_or_lens)
    C = lens.numel()
    dt = sh.torch_dtype
    out = make_paged_kv(sh, lens, seed, device, shuffle=shuffle, slack=slack, tag="attn.kv")
    out["q"] = _randn((C, K, sh.Hq, sh.D), 1.0, dt, device, seed, "attn.q")
    out["k_blk"] = _randn((C, K, sh.Hkv, sh.D), 1.0, dt, device, seed, "attn.kb")
    out["v_blk"] = _randn((C, K, sh.Hkv, sh.D), 1.0, dt, device, seed, "attn.vb")
    return out


def make_step_inputs(wl: Workload, device="cpu", weights=True) -> dict:
    """Everything one draft step consumes: weights, one KV cache per attention
    layer, h_last [C,d], and either block tokens [C,K] (when the drafter has an LM
    head: the last accepted token followed by K-1 mask tokens) or a direct block
    input x [C,K,d] (kernel-level workloads without embedding / head)."""
    sh, C, K, seed = wl.shapes, wl.C, wl.K, wl.seed
    lens = make_ctx_lens(wl)
    out = {"workload": wl, "ctx_lens": lens.to(device=device)}
    if weights:
        out["weights"] = make_weights(sh, seed, device)
    out["kv"] = [make_paged_kv(sh, lens, seed, device, shuffle=wl.shuffle, slack=wl.slack, tag=f"kv{i}")
                 for i, k in enumerate(sh.layers) if k == "A"]
    out["h_last"] = _randn((C, sh.d), 1.0, sh.torch_dtype, device, seed, "h_last")
    if sh.vocab:
        g = _gen(seed, "tokens", "cpu")
        toks = torch.full((C, K), sh.mask_token, dtype=torch.int32)
        toks[:, 0] = torch.randint(0, sh.vocab - 1, (C,), generator=g, dtype=torch.int32)
        out["tokens"] = toks.to(device)
        out["x_in"] = None
    else:
        out["tokens"] = None
        out["x_in"] = _randn((C, K, sh.d), 1.0, sh.torch_dtype, device, seed, "x_in")
    return out
