"""The C-ABI library loads, exports every entry point its header declares, and rejects
bad arguments before touching the GPU (host-only checks; runs without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

import latent_mixture_experts_moe_b200 as moe
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from latent_mixture_experts_moe_b200 import build
    build.build()
    yield


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(muse_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 8
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(moe.EXPORTS) == names


def test_structs_match_the_c_compilers_layout(tmp_path):
    # compile a probe against the header with gcc and compare every field offset
    fields = [f for f, _ in moe.Config._fields_]
    lay_fields = [f for f, _ in moe.WorkspaceLayout._fields_]
    src = ["#include <stdio.h>", "#include <stddef.h>", '#include "muse_moe.h"', "int main(void) {",
           'printf("%zu\\n", sizeof(muse_moe_config));',
           'printf("%zu\\n", sizeof(muse_moe_workspace_layout));']
    src += [f'printf("%zu\\n", offsetof(muse_moe_config, {f}));' for f in fields]
    src += [f'printf("%zu\\n", offsetof(muse_moe_workspace_layout, {f}));' for f in lay_fields]
    src += ["return 0; }"]
    c = tmp_path / "probe.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(moe.Config)
    assert vals[1] == ctypes.sizeof(moe.WorkspaceLayout)
    assert vals[2:2 + len(fields)] == [getattr(moe.Config, f).offset for f in fields]
    assert vals[2 + len(fields):] == [getattr(moe.WorkspaceLayout, f).offset for f in lay_fields]


def test_status_strings():
    for code in range(7):
        assert moe.status_string(code)
    assert moe.status_string(5) == "device-side wait timed out"


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_workspace_size_and_layout(name):
    w = W.WORKLOADS[name]
    cfg = moe.make_config(w.T, w.D, w.L, w.I, w.E, w.k, w.dtype, w.eps)
    n = moe.workspace_size(cfg)
    lay = moe.workspace_layout(cfg)
    assert lay["total"] == n
    act = 2 if w.dtype == "bf16" else 4
    offs = sorted((v, k) for k, v in lay.items() if k not in ("total", "rows"))
    assert all(v % 256 == 0 for v, _ in offs)
    assert lay["rows"] >= w.T * w.k and lay["rows"] % 16 == 0
    assert lay["rows"] <= w.T * w.k + 16 * min(w.E, w.T * w.k)
    assert n >= lay["c"] + w.T * w.L * act
    assert moe.launch_count(cfg) == 11


@pytest.mark.parametrize("field,value,code", [
    ("T", 0, 1), ("top_k", 0, 1), ("top_k", 9, 1), ("dtype", 7, 1), ("D", 200, 2), ("L", 100, 2),
    ("I", 64, 2), ("E", 2048, 2), ("top_k", 33, 2), ("router_mode", 5, 1), ("norm_mode", 3, 1)])
def test_invalid_configs_are_rejected(field, value, code):
    cfg = moe.make_config(16, 256, 128, 128, 8, 2, "f32")
    if field == "top_k" and value == 33:
        cfg.E = 64
    setattr(cfg, field, value)
    with pytest.raises(moe.MuseError) as e:
        moe.workspace_size(cfg)
    assert e.value.code == code


def test_forward_rejects_null_and_misaligned_pointers_before_any_launch():
    cfg = moe.make_config(16, 256, 128, 128, 8, 2, "f32")
    lib = moe.lib()
    args = [ctypes.c_void_p(4096 * (i + 1)) for i in range(9)]
    for bad in range(9):
        a = list(args)
        a[bad] = ctypes.c_void_p(0)
        assert lib.muse_latent_moe_forward(ctypes.byref(cfg), *a, None) == 1
        a[bad] = ctypes.c_void_p(4096 * (bad + 1) + 8)
        assert lib.muse_latent_moe_forward(ctypes.byref(cfg), *a, None) == 1
    # valid-looking pointers but no workspace
    assert lib.muse_latent_moe_forward(ctypes.byref(cfg), *args, None) == 3
    cfg.workspace = 1 << 20
    cfg.workspace_bytes = 16
    assert lib.muse_latent_moe_forward(ctypes.byref(cfg), *args, None) == 3
    assert lib.muse_latent_moe_forward(None, *args, None) == 1


@pytest.mark.parametrize("name", ["mid", "prefill", "nvfp4_w4a4"])
@pytest.mark.parametrize("G", [1, 2, 8])
def test_expert_parallel_workspaces_hold_only_their_roles_buffers(name, G):
    w = W.WORKLOADS[name]
    cfg = moe.make_config(w.T, w.D, w.L, w.I, w.E, w.k, w.dtype, w.eps,
                          act_format=moe.ACT_NVFP4 if w.act == "nvfp4" else moe.ACT_BF16)
    if w.experts == "nvfp4":
        cfg.expert_weights = moe.EXPERTS_NVFP4
    full = moe.workspace_layout(cfg)
    home = moe.ep_workspace_layout(cfg, G, moe.EP_HOME)
    rows = G * w.T * min(w.k, w.E // G)
    shard = moe.ep_workspace_layout(cfg, G, moe.EP_EXPERTS, rows)
    for n in ("zp", "h", "y", "ss", "zq_codes", "hq_codes"):
        assert home[n] == 0, n
    for n in ("logits", "topk_idx", "topk_w", "z", "c"):
        assert shard[n] == 0, n
        assert home[n] > 0 or n == "logits", n
    assert home["rows"] == w.T * w.k  # the send plan has no padding
    assert shard["rows"] >= rows and shard["rows"] <= rows + 16 * min(w.E // G, rows)
    assert home["total"] < full["total"]
    if G == 1:
        assert shard["total"] < full["total"]
    assert all(v % 256 == 0 for k, v in shard.items() if k not in ("total", "rows"))


def test_expert_parallel_arguments_are_rejected_before_any_launch():
    lib = moe.lib()
    cfg = moe.make_config(16, 256, 128, 128, 8, 2, "f32")
    lay = moe.WorkspaceLayout()
    assert lib.muse_ep_workspace_layout(ctypes.byref(cfg), 3, moe.EP_HOME, 0, ctypes.byref(lay)) == 1  # 8 % 3
    assert lib.muse_ep_workspace_layout(ctypes.byref(cfg), 0, moe.EP_HOME, 0, ctypes.byref(lay)) == 1
    assert lib.muse_ep_workspace_layout(ctypes.byref(cfg), 2, 7, 0, ctypes.byref(lay)) == 1  # unknown role
    assert lib.muse_ep_workspace_layout(ctypes.byref(cfg), 2, moe.EP_EXPERTS, -1, ctypes.byref(lay)) == 1
    p = [ctypes.c_void_p(4096 * (i + 1)) for i in range(9)]
    # dispatch: x, W_router, W_pool, send_z, send_expert, rank_counts
    for bad in range(6):
        a = list(p[:6])
        a[bad] = ctypes.c_void_p(0)
        assert lib.muse_ep_dispatch(ctypes.byref(cfg), 2, *a, None) == 1
    assert lib.muse_ep_dispatch(ctypes.byref(cfg), 2, *p[:6], None) == 3  # no workspace
    # experts: nothing received launches nothing, whatever the pointers
    assert lib.muse_ep_experts(ctypes.byref(cfg), 2, 0, *([None] * 8), None) == 0
    for bad in range(8):
        a = list(p[:8])
        a[bad] = ctypes.c_void_p(0)
        assert lib.muse_ep_experts(ctypes.byref(cfg), 2, 5, *a, None) == 1
    assert lib.muse_ep_experts(ctypes.byref(cfg), 2, 5, *p[:8], None) == 3
    # combine: x, back_y, back_ss, gamma, W_unpool, out
    for bad in range(6):
        a = list(p[:6])
        a[bad] = ctypes.c_void_p(4096 * (bad + 1) + 4)
        assert lib.muse_ep_combine(ctypes.byref(cfg), 2, *a, None) == 1
    assert lib.muse_ep_combine(ctypes.byref(cfg), 2, *p[:6], None) == 3
    assert lib.muse_ep_combine(ctypes.byref(cfg), 3, *p[:6], None) == 1


@pytest.mark.parametrize("w4a4", [False, True])
@pytest.mark.parametrize("pre_expert,ffn_pre,ffn_post", [(0, 0, 0), (1, 0, 0), (0, 1, 1), (1, 1, 0), (0, 0, 1)])
def test_stage_names_match_the_library_launch_count(w4a4, pre_expert, ffn_pre, ffn_post):
    cfg = moe.make_config(64, 1024, 512, 512, 16, 2, "bf16", act_format=moe.ACT_NVFP4 if w4a4 else moe.ACT_BF16)
    if w4a4:
        cfg.expert_weights = moe.EXPERTS_NVFP4
    # any non-null pointer switches a step on; launch_count reads no memory
    cfg.pre_norm_gain = 4096 if pre_expert else None
    cfg.ffn_pre_gain = 4096 if ffn_pre else None
    cfg.ffn_post_gain = 4096 if ffn_post else None
    names = moe.stages(cfg)
    assert len(names) == moe.launch_count(cfg)
    assert len(set(names)) == len(names)
    assert ("quant_z" in names) == w4a4 and ("gather_codes" in names) == w4a4
    assert names.index("pooler") < names.index("gather_codes" if w4a4 else "gather") < names.index("gate_up_swiglu")
