"""The C-ABI library loads, exports every entry point its header declares, and rejects
bad arguments before touching the GPU (host-only checks; runs without a GPU)."""
import ctypes
import os
import re
import subprocess
import sys

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
    assert moe.launch_count(cfg) == 11 == len(moe.stages(cfg))


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


# ------------------------------------------------------------ the shape-checked entry point
def _desc(addr, elem, shape):
    d = moe.Tensor()
    d.data, d.elem, d.ndim = addr, elem, len(shape)
    st = 1
    for i in reversed(range(len(shape))):
        d.shape[i], d.stride[i] = shape[i], st
        st *= shape[i]
    return d


def _checked_args(cfg, nvfp4=False):
    """Descriptors of every argument for cfg at non-overlapping (never dereferenced) addresses."""
    T, D, L, I, E = cfg.T, cfg.D, cfg.L, cfg.I, cfg.E
    a = cfg.dtype
    base = iter(range(1 << 40, 1 << 50, 1 << 36))
    args = {"x": _desc(next(base), a, (T, D)), "W_router": _desc(next(base), a, (E, D)),
            "W_pool": _desc(next(base), a, (L, D)), "gamma": _desc(next(base), a, (E, L)),
            "W_unpool": _desc(next(base), a, (D, L)), "out": _desc(next(base), a, (T, D))}
    for n, (r, c) in (("W_gate", (I, L)), ("W_up", (I, L)), ("W_down", (L, I))):
        if nvfp4:
            args[n] = (moe.Tensor * 3)(_desc(next(base), moe.ELEM_U8, (E, r, c // 2)),
                                       _desc(next(base), moe.ELEM_U8, (E, r, c // 16)),
                                       _desc(next(base), moe.ELEM_F32, (E,)))
        else:
            args[n] = (moe.Tensor * 1)(_desc(next(base), a, (E, r, c)))
    return args


def _call_checked(cfg, args):
    order = ("x", "W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool", "out")
    ptrs = [ctypes.cast(args[n], ctypes.POINTER(moe.Tensor)) if isinstance(args[n], ctypes.Array)
            else ctypes.pointer(args[n]) for n in order]
    return moe.lib().muse_latent_moe_forward_checked(ctypes.byref(cfg), *ptrs, None)


def test_tensor_descriptor_layout_matches_the_c_compiler(tmp_path):
    fields = [f for f, _ in moe.Tensor._fields_]
    src = ["#include <stdio.h>", "#include <stddef.h>", '#include "muse_moe.h"', "int main(void) {",
           'printf("%zu\\n", sizeof(muse_tensor));']
    src += [f'printf("%zu\\n", offsetof(muse_tensor, {f}));' for f in fields]
    src += ["return 0; }"]
    c = tmp_path / "probe_t.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "probe_t"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert vals == [ctypes.sizeof(moe.Tensor)] + [getattr(moe.Tensor, f).offset for f in fields]


@pytest.mark.parametrize("nvfp4", [False, True])
def test_checked_forward_rejects_every_shape_mismatch_before_any_launch(nvfp4):
    """Correct descriptors get past every shape check (and stop at the missing workspace);
    a wrong extent, rank, element type, stride or alignment on any argument, or an output
    overlapping an input, is MUSE_ERR_INVALID_ARG -- all without a GPU."""
    cfg = moe.make_config(64, 1024, 512, 256, 16, 2, "bf16")
    if nvfp4:
        cfg.expert_weights = moe.EXPERTS_NVFP4
    assert _call_checked(cfg, _checked_args(cfg, nvfp4)) == 3        # shapes fine: no workspace
    names = ("x", "W_router", "W_pool", "W_gate", "W_up", "W_down", "gamma", "W_unpool", "out")
    for n in names:
        parts = 3 if (nvfp4 and n.startswith("W_") and n in ("W_gate", "W_up", "W_down")) else 1
        for p in range(parts):
            for corrupt in ("extent", "rank", "elem", "stride", "align", "null"):
                args = _checked_args(cfg, nvfp4)
                d = args[n][p] if isinstance(args[n], ctypes.Array) else args[n]
                if corrupt == "extent":
                    d.shape[0] += 1
                elif corrupt == "rank":
                    d.ndim = d.ndim + 1 if d.ndim < 3 else 1
                elif corrupt == "elem":
                    d.elem = moe.ELEM_F32 if d.elem != moe.ELEM_F32 else moe.ELEM_BF16
                elif corrupt == "stride":
                    d.stride[0] += 1
                elif corrupt == "align":
                    d.data += 8 if not (nvfp4 and p == 2) else 2
                else:
                    d.data = 0
                assert _call_checked(cfg, args) == 1, (n, p, corrupt)
    # the gain shared by all experts is [L]; a per-expert gain given as shared is rejected
    cfg.gamma_shared = 1
    assert _call_checked(cfg, _checked_args(cfg, nvfp4)) == 1
    args = _checked_args(cfg, nvfp4)
    args["gamma"] = _desc(args["gamma"].data, cfg.dtype, (cfg.L,))
    assert _call_checked(cfg, args) == 3
    # out may not overlap an input
    cfg.gamma_shared = 0
    args = _checked_args(cfg, nvfp4)
    args["out"].data = args["x"].data
    assert _call_checked(cfg, args) == 1
    args = _checked_args(cfg, nvfp4)
    w = args["W_down"][0]
    args["out"].data = w.data + 4096
    assert _call_checked(cfg, args) == 1


def test_last_cuda_error_names_no_error_before_any_failure():
    """muse_last_cuda_error() is a host-side query: in a fresh process, before any CUDA call
    has failed, it returns the runtime's "no error" text."""
    code = "import latent_mixture_experts_moe_b200 as moe; print(moe.last_cuda_error())"
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip().splitlines()[-1] == "no error"
