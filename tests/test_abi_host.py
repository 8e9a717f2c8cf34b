"""CPU checks of the C-ABI library: it loads, exports every function include/hspec.h
declares, its ctypes structs match the C layout, and host-side validation rejects
bad arguments before anything is launched (no GPU is touched here)."""
import ctypes as ct
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hspec.h")


@pytest.fixture(scope="module")
def H():
    from hybrid_mamba_attention_b200 import hspec
    return hspec


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^HSPEC_API[^;(]*?\b(hspec_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_function(H):
    names = declared_functions()
    assert len(names) >= 13
    lib = ct.CDLL(H.LIBRARY_PATH)
    for n in names:
        assert hasattr(lib, n), f"libhspec.so does not export {n}"
    assert set(names) == set(H.EXPORTS)


def test_struct_layouts_match_header(H, tmp_path):
    prog = tmp_path / "sz.c"
    fields = {"hspec_cfg": ["d_model", "layer_kinds", "dtype", "rope_theta", "attn_split_tokens", "draft_vocab", "wait_limit_ns"],
              "hspec_step_in": ["C", "h_last", "ctx_lens", "kv"],
              "hspec_kv_view": ["v_pool", "num_pages", "page_table", "max_pages"],
              "hspec_model_weights": ["layers", "final_norm", "W_lm", "W_lm_draft", "draft_to_target"],
              "hspec_layer_weights": ["W_inj", "W_down"],
              "hspec_step_out": ["draft_tokens", "top_logit"]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void){"]
    for s, fs in fields.items():
        lines.append(f'printf("%zu\\n", sizeof({s}));')
        for f in fs:
            lines.append(f'printf("%zu\\n", offsetof({s}, {f}));')
    lines.append("return 0;}")
    prog.write_text("\n".join(lines))
    exe = tmp_path / "sz"
    subprocess.run(["gcc", str(prog), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = []
    for s, fs in fields.items():
        cls = getattr(H, s)
        want.append(ct.sizeof(cls))
        for f in fs:
            want.append(getattr(cls, f).offset)
    assert got == want


def small_cfg(H, **kw):
    from hybrid_mamba_attention_b200 import inputs as I
    cfg = H.make_cfg(I.TINY)
    for k, v in kw.items():
        setattr(cfg, k, v)
    return cfg


def test_status_strings_and_version(H):
    assert "sm_100a" in H.hspec_version()
    for s in range(8):
        assert H.hspec_status_string(s)
    assert H.hspec_launch_count() >= 0


def test_null_pointers_rejected_before_launch(H):
    cfg = small_cfg(H)
    n0 = H.hspec_launch_count()
    assert H._lib.hspec_inject_state(ct.byref(cfg), None, None, 1, None, None) == H.HSPEC_ERR_INVALID_ARG
    assert H._lib.hspec_ssd_block_scan(ct.byref(cfg), None, None, None, None, None, None, None, 1, 8, None,
                                       None, None) == H.HSPEC_ERR_INVALID_ARG
    assert H.hspec_launch_count() == n0


def test_bad_config_rejected(H):
    cfg = small_cfg(H, dtype=7)
    assert H._lib.hspec_inject_state(ct.byref(cfg), 16, 16, 1, 16, None) == H.HSPEC_ERR_INVALID_ARG
    assert "dtype" in H.hspec_last_error()
    cfg = small_cfg(H, n_kv_heads=3)
    kv = H.hspec_kv_view(k_pool=16, v_pool=16, num_pages=4, page_table=16, max_pages=4)
    st = H._lib.hspec_attn_paged_block(ct.byref(cfg), 16, ct.byref(kv), 16, 16, 16, 1, 8, 16, 256, 1 << 20, None)
    assert st == H.HSPEC_ERR_SHAPE_MISMATCH
    cfg = small_cfg(H, flags=64)
    assert H._lib.hspec_inject_state(ct.byref(cfg), 16, 16, 1, 16, None) == H.HSPEC_ERR_INVALID_ARG
    cfg = small_cfg(H, wait_limit_ns=-1)
    assert H._lib.hspec_inject_state(ct.byref(cfg), 16, 16, 1, 16, None) == H.HSPEC_ERR_INVALID_ARG
    assert "wait_limit_ns" in H.hspec_last_error()


def test_unsupported_block_size_rejected(H):
    cfg = small_cfg(H)
    st = H._lib.hspec_ssd_block_scan(ct.byref(cfg), 16, 16, 16, 16, 16, 16, None, 1, 65, 16, None, None)
    assert st == H.HSPEC_ERR_UNSUPPORTED
    st = H._lib.hspec_ssd_block_scan(ct.byref(cfg), 16, 16, 16, 16, 16, 16, None, 1, 0, 16, None, None)
    assert st == H.HSPEC_ERR_UNSUPPORTED


def test_attention_workspace_checked(H):
    cfg = small_cfg(H)
    kv = H.hspec_kv_view(k_pool=16, v_pool=16, num_pages=4, page_table=16, max_pages=4)
    need = H.hspec_attn_workspace_size(cfg, 1, 8, 4)
    assert need > 0 and need % 256 == 0
    st = H._lib.hspec_attn_paged_block(ct.byref(cfg), 16, ct.byref(kv), 16, 16, 16, 1, 8, 16, 256, need - 1, None)
    assert st == H.HSPEC_ERR_WORKSPACE
    st = H._lib.hspec_attn_paged_block(ct.byref(cfg), 16, ct.byref(kv), 16, 16, 16, 1, 8, 16, 1024 + 16, need, None)
    assert st == H.HSPEC_ERR_WORKSPACE  # misaligned
    bad = H.hspec_kv_view(k_pool=16, v_pool=16, num_pages=0, page_table=16, max_pages=4)
    st = H._lib.hspec_attn_paged_block(ct.byref(cfg), 16, ct.byref(bad), 16, 16, 16, 1, 8, 16, 256, need, None)
    assert st == H.HSPEC_ERR_PAGE_OOB


def test_workspace_sizes_grow_with_batch_and_context(H):
    from hybrid_mamba_attention_b200 import inputs as I
    cfg = H.make_cfg(I.LLAMA_FULL)
    a = H.hspec_step_workspace_size(cfg, 1, 16, 128)
    b = H.hspec_step_workspace_size(cfg, 8, 16, 128)
    c = H.hspec_step_workspace_size(cfg, 8, 16, 1024)
    assert 0 < a < b <= c
    assert a % 256 == 0


def test_drafter_create_validates(H):
    from hybrid_mamba_attention_b200 import inputs as I
    cfg = H.make_cfg(I.TINY)
    mw = H.hspec_model_weights()
    h = ct.c_void_p()
    assert H._lib.hspec_drafter_create(ct.byref(cfg), ct.byref(mw), ct.byref(h)) == H.HSPEC_ERR_INVALID_ARG
    cfg.layer_kinds = b"MX"
    assert H._lib.hspec_drafter_create(ct.byref(cfg), ct.byref(mw), ct.byref(h)) == H.HSPEC_ERR_INVALID_ARG
    cfg = H.make_cfg(I.TINY)
    cfg.n_layers = 0
    assert H._lib.hspec_drafter_create(ct.byref(cfg), ct.byref(mw), ct.byref(h)) == H.HSPEC_ERR_INVALID_ARG
    # bf16 drafters need TMA-friendly dims
    cfg = H.make_cfg(I.LLAMA)
    cfg.d_model = 4100
    for i in range(2):
        for f, _ in H.hspec_layer_weights._fields_:
            setattr(mw.layers[i], f, 256)
    assert H._lib.hspec_drafter_create(ct.byref(cfg), ct.byref(mw), ct.byref(h)) == H.HSPEC_ERR_UNSUPPORTED
    cfg.d_model = 4096
    assert H._lib.hspec_drafter_create(ct.byref(cfg), ct.byref(mw), ct.byref(h)) == H.HSPEC_OK
    H.hspec_drafter_destroy(h)


def test_step_rejects_missing_inputs(H):
    from hybrid_mamba_attention_b200 import inputs as I
    cfg = H.make_cfg(I.TINY)
    mw = H.hspec_model_weights()
    for i in range(2):
        for f, _ in H.hspec_layer_weights._fields_:
            setattr(mw.layers[i], f, 256)
    h = H.hspec_drafter_create(cfg, mw)
    si = H.hspec_step_in(C=1, K=8)
    so = H.hspec_step_out()
    st = H._lib.hspec_draft_step(h, ct.byref(si), ct.byref(so), 256, 1 << 30, None)
    assert st == H.HSPEC_ERR_INVALID_ARG
    si = H.hspec_step_in(C=1, K=8, h_last=256, x_in=256, ctx_lens=256)
    si.kv[0] = H.hspec_kv_view(k_pool=256, v_pool=256, num_pages=4, page_table=256, max_pages=4)
    st = H._lib.hspec_draft_step(h, ct.byref(si), ct.byref(so), 256, 16, None)
    assert st == H.HSPEC_ERR_WORKSPACE
    H.hspec_drafter_destroy(h)


def test_empty_batches_and_block_sizes_rejected_before_launch(H):
    # C = 0 requests and K outside 1..64 are refused by every entry point before anything is
    # launched (the header states C >= 1 and 1 <= K <= 64); the workspace queries answer 0
    from hybrid_mamba_attention_b200 import inputs as I
    cfg = small_cfg(H)
    kv = H.hspec_kv_view(k_pool=256, v_pool=256, num_pages=4, page_table=256, max_pages=4)
    n0 = H.hspec_launch_count()
    assert H._lib.hspec_inject_state(ct.byref(cfg), 256, 256, 0, 256, None) == H.HSPEC_ERR_INVALID_ARG
    st = H._lib.hspec_ssd_block_scan(ct.byref(cfg), 256, 256, 256, 256, 256, 256, 256, 0, 8, 256, None, None)
    assert st == H.HSPEC_ERR_INVALID_ARG
    for C, K in ((0, 8), (1, 0), (1, 65)):
        st = H._lib.hspec_attn_paged_block(ct.byref(cfg), 256, ct.byref(kv), 256, 256, 256, C, K, 256, 256,
                                           1 << 30, None)
        assert st == H.HSPEC_ERR_UNSUPPORTED, (C, K)
        st = H._lib.hspec_attn_paged_block_noalloc(ct.byref(cfg), 256, ct.byref(kv), 256, 256, 256, C, K, 256,
                                                   None)
        assert st == H.HSPEC_ERR_UNSUPPORTED, (C, K)
    assert H.hspec_attn_workspace_size(cfg, 0, 8, 4) == 0 and H.hspec_attn_workspace_size(cfg, 1, 0, 4) == 0
    # verification over a vocabulary
    vcfg = H.make_cfg(I.LLAMA_FULL)
    for C, K in ((0, 8), (1, 0), (1, 65)):
        st = H._lib.hspec_verify_greedy(ct.byref(vcfg), 256, 256, C, K, 256, 256, None, 256, 1 << 30, None)
        assert st == H.HSPEC_ERR_UNSUPPORTED, (C, K)
    assert H.hspec_verify_workspace_size(vcfg, 0, 8) == 0
    # the whole draft step
    mw = H.hspec_model_weights()
    for i in range(2):
        for f, _ in H.hspec_layer_weights._fields_:
            setattr(mw.layers[i], f, 256)
    h = H.hspec_drafter_create(H.make_cfg(I.TINY), mw)
    so = H.hspec_step_out()
    for C, K in ((0, 8), (1, 0), (1, 65)):
        si = H.hspec_step_in(C=C, K=K, h_last=256, x_in=256, ctx_lens=256)
        si.kv[0] = kv
        assert H._lib.hspec_draft_step(h, ct.byref(si), ct.byref(so), 256, 1 << 30, None) == H.HSPEC_ERR_UNSUPPORTED
    assert H.hspec_step_workspace_size(H.make_cfg(I.TINY), 0, 8, 4) == 0
    H.hspec_drafter_destroy(h)
    assert H.hspec_launch_count() == n0


def test_plain_c_program_links_and_calls_the_library(H, tmp_path):
    # a C caller needs only the header and the shared library: build one against them and
    # call the host-side entry points (no device work)
    prog = tmp_path / "use.c"
    prog.write_text(r'''
#include <stdio.h>
#include "hspec.h"
int main(void) {
  hspec_cfg cfg = {0};
  cfg.d_model = 256; cfg.n_q_heads = 4; cfg.n_kv_heads = 2; cfg.head_dim = 64;
  cfg.n_ssm_heads = 4; cfg.ssm_head_dim = 64; cfg.d_state = 16; cfg.page_size = 16;
  cfg.n_layers = 2; cfg.layer_kinds[0] = 'M'; cfg.layer_kinds[1] = 'A';
  cfg.dtype = HSPEC_DTYPE_F32; cfg.rope_theta = 1e4f; cfg.norm_eps = 1e-6f;
  printf("%s\n", hspec_version());
  printf("%zu\n", hspec_attn_workspace_size(&cfg, 1, 8, 4));
  printf("%d\n", hspec_inject_state(&cfg, NULL, NULL, 1, NULL, NULL));
  printf("%s\n", hspec_status_string(HSPEC_ERR_INVALID_ARG));
  return 0;
}
''')
    libdir = os.path.dirname(H.LIBRARY_PATH)
    exe = tmp_path / "use"
    subprocess.run(["gcc", str(prog), "-I", os.path.join(ROOT, "include"), "-L", libdir, "-l:" +
                    os.path.basename(H.LIBRARY_PATH), f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    assert "sm_100a" in out[0]
    ws = int(out[1])
    assert ws > 0 and ws % 256 == 0
    assert int(out[2]) == H.HSPEC_ERR_INVALID_ARG and out[3]
