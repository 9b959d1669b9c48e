"""Python binding of libmuse_moe.so, the B200 (sm_100a) latent-MoE block forward pass.

Argument marshalling only: every step of the block runs in the library's CUDA kernels.
PyTorch tensors are accepted as containers of device memory (their data pointers are
passed through the C ABI declared in include/muse_moe.h); nothing here computes.
If the compiled library is missing, importing works but every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmuse_moe.so")

MUSE_F32, MUSE_BF16 = 0, 1
ROUTER_SOFTMAX, ROUTER_SIGMOID = 0, 1
EXPERTS_DENSE, EXPERTS_NVFP4 = 0, 1
ACT_BF16, ACT_NVFP4 = 0, 1
NORM_CENTRED, NORM_INPUT_SCALED = 0, 1

STATUS = {0: "MUSE_OK", 1: "MUSE_ERR_INVALID_ARG", 2: "MUSE_ERR_UNSUPPORTED", 3: "MUSE_ERR_WORKSPACE",
          4: "MUSE_ERR_CUDA", 5: "MUSE_ERR_TIMEOUT", 6: "MUSE_ERR_DEVICE"}

# every extern "C" entry point of include/muse_moe.h
EXPORTS = ("muse_moe_config_init", "muse_latent_moe_workspace_size", "muse_latent_moe_workspace_layout",
           "muse_latent_moe_forward", "muse_latent_moe_forward_host_io", "muse_latent_moe_last_device_status",
           "muse_status_string", "muse_latent_moe_launch_count", "muse_latent_moe_forward_static_scratch",
           "muse_selftest_bounded_wait", "muse_quantize_nvfp4_rows", "muse_latent_moe_forward_host_batches",
           "muse_ep_workspace_layout", "muse_ep_dispatch", "muse_ep_experts", "muse_ep_combine",
           "muse_latent_moe_forward_checked", "muse_latent_moe_stage_name", "muse_last_cuda_error")

# roles of an expert-parallel workspace (muse_ep_role)
EP_HOME, EP_EXPERTS = 1, 2

# size of the library's built-in scratch array (MUSE_STATIC_SCRATCH_BYTES)
STATIC_SCRATCH_BYTES = 16 << 20


class MuseError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {STATUS.get(code, code)} ({status_string(code)})"
        if code == 4:  # MUSE_ERR_CUDA
            msg += f": {last_cuda_error()}"
        super().__init__(msg)


class Config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("D", ctypes.c_int64), ("L", ctypes.c_int64), ("I", ctypes.c_int64),
                ("E", ctypes.c_int64), ("top_k", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("eps", ctypes.c_float), ("router_mode", ctypes.c_int32), ("router_logit_scale", ctypes.c_float),
                ("routed_scaling", ctypes.c_float), ("router_bias", ctypes.c_void_p),
                ("norm_mode", ctypes.c_int32), ("gamma_shared", ctypes.c_int32),
                ("pre_norm_gain", ctypes.c_void_p), ("pre_norm_eps", ctypes.c_float),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("topk_idx_out", ctypes.c_void_p), ("topk_w_out", ctypes.c_void_p),
                ("stage_events", ctypes.c_void_p), ("expert_weights", ctypes.c_int32),
                ("ffn_pre_gain", ctypes.c_void_p), ("ffn_pre_eps", ctypes.c_float),
                ("ffn_post_gain", ctypes.c_void_p), ("ffn_post_eps", ctypes.c_float),
                ("residual_gate", ctypes.c_void_p), ("residual_gate_temperature", ctypes.c_float),
                ("residual_gate_eps", ctypes.c_float), ("act_format", ctypes.c_int32)]


class Tensor(ctypes.Structure):
    """muse_tensor: device pointer, element type, rank, extents and strides (elements)."""
    _fields_ = [("data", ctypes.c_void_p), ("elem", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 3), ("stride", ctypes.c_int64 * 3)]


ELEM_F32, ELEM_BF16, ELEM_U8 = 0, 1, 2


def tensor_desc(t) -> Tensor:
    """The muse_tensor of a torch tensor (its own shape and strides: a non-contiguous view
    is described as it is, and the library rejects it)."""
    import torch
    elem = {torch.float32: ELEM_F32, torch.bfloat16: ELEM_BF16, torch.uint8: ELEM_U8}.get(t.dtype, -1)
    d = Tensor()
    d.data, d.elem, d.ndim = int(t.data_ptr()), elem, t.dim()
    for i in range(min(t.dim(), 3)):
        d.shape[i], d.stride[i] = int(t.shape[i]), int(t.stride(i))
    return d


class Nvfp4Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("block_scales", ctypes.c_void_p), ("matrix_scale", ctypes.c_void_p)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("status", "expert_count", "expert_offset", "logits", "topk_idx",
                                              "topk_w", "inv", "row_token", "z", "zp", "h", "y", "ss", "c",
                                              "xn", "ss_out", "zq_codes", "zq_scales", "hq_codes", "hq_scales",
                                              "total")] + [("rows", ctypes.c_int64)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m latent_mixture_experts_moe_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, cp = ctypes.c_void_p, ctypes.POINTER(Config)
        L.muse_moe_config_init.argtypes = [cp]
        L.muse_moe_config_init.restype = None
        L.muse_latent_moe_workspace_size.argtypes = [cp, ctypes.POINTER(ctypes.c_size_t)]
        L.muse_latent_moe_workspace_size.restype = ctypes.c_int
        L.muse_latent_moe_workspace_layout.argtypes = [cp, ctypes.POINTER(WorkspaceLayout)]
        L.muse_latent_moe_workspace_layout.restype = ctypes.c_int
        L.muse_latent_moe_forward.argtypes = [cp] + [vp] * 10
        L.muse_latent_moe_forward.restype = ctypes.c_int
        L.muse_latent_moe_forward_host_io.argtypes = [cp] + [vp] * 12
        L.muse_latent_moe_forward_host_io.restype = ctypes.c_int
        L.muse_latent_moe_last_device_status.argtypes = [cp, vp, ctypes.POINTER(ctypes.c_uint32)]
        L.muse_latent_moe_last_device_status.restype = ctypes.c_int
        L.muse_status_string.argtypes = [ctypes.c_int]
        L.muse_status_string.restype = ctypes.c_char_p
        L.muse_last_cuda_error.argtypes = []
        L.muse_last_cuda_error.restype = ctypes.c_char_p
        L.muse_latent_moe_forward_static_scratch.argtypes = [cp] + [vp] * 10
        L.muse_latent_moe_forward_static_scratch.restype = ctypes.c_int
        L.muse_selftest_bounded_wait.argtypes = [ctypes.c_uint64, vp, vp]
        L.muse_selftest_bounded_wait.restype = ctypes.c_int
        L.muse_quantize_nvfp4_rows.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp, vp, vp]
        L.muse_quantize_nvfp4_rows.restype = ctypes.c_int
        L.muse_latent_moe_forward_host_batches.argtypes = [cp, ctypes.c_int64, vp, vp, vp, vp] + [vp] * 7 + [vp] * 3
        L.muse_latent_moe_forward_host_batches.restype = ctypes.c_int
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        L.muse_ep_workspace_layout.argtypes = [cp, i32, i32, i64, ctypes.POINTER(WorkspaceLayout)]
        L.muse_ep_workspace_layout.restype = ctypes.c_int
        L.muse_ep_dispatch.argtypes = [cp, i32] + [vp] * 7
        L.muse_ep_dispatch.restype = ctypes.c_int
        L.muse_ep_experts.argtypes = [cp, i32, i64] + [vp] * 9
        L.muse_ep_experts.restype = ctypes.c_int
        L.muse_ep_combine.argtypes = [cp, i32] + [vp] * 7
        L.muse_ep_combine.restype = ctypes.c_int
        L.muse_latent_moe_forward_checked.argtypes = [cp] + [ctypes.POINTER(Tensor)] * 9 + [vp]
        L.muse_latent_moe_forward_checked.restype = ctypes.c_int
        L.muse_latent_moe_stage_name.argtypes = [cp, ctypes.c_int32]
        L.muse_latent_moe_stage_name.restype = ctypes.c_char_p
        L.muse_latent_moe_launch_count.argtypes = [cp]
        L.muse_latent_moe_launch_count.restype = ctypes.c_int32
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().muse_status_string(code).decode()


def last_cuda_error() -> str:
    """The CUDA runtime's description of the last CUDA error behind a MUSE_ERR_CUDA on this
    thread ("no error" when none)."""
    return lib().muse_last_cuda_error().decode()


def _check(code: int, where: str) -> None:
    if code != 0:
        raise MuseError(code, where)


def make_config(T: int, D: int, L: int, I: int, E: int, k: int, dtype: str = "bf16", eps: float = 1e-6,
                router_mode: int = ROUTER_SOFTMAX, router_logit_scale: float = 1.0, routed_scaling: float = 1.0,
                norm_mode: int = NORM_CENTRED, gamma_shared: bool = False, pre_norm_eps: float = 1e-5,
                ffn_pre_eps: float = 1e-5, ffn_post_eps: float = 1e-8, residual_gate_temperature: float = 0.3,
                residual_gate_eps: float = 1e-3, act_format: int = ACT_BF16) -> Config:
    c = Config()
    lib().muse_moe_config_init(ctypes.byref(c))
    c.T, c.D, c.L, c.I, c.E, c.top_k = T, D, L, I, E, k
    c.dtype = {"f32": MUSE_F32, "bf16": MUSE_BF16}[dtype]
    c.eps = eps
    c.router_mode, c.router_logit_scale, c.routed_scaling = router_mode, router_logit_scale, routed_scaling
    c.norm_mode, c.gamma_shared = norm_mode, int(gamma_shared)
    c.pre_norm_eps = pre_norm_eps
    c.ffn_pre_eps, c.ffn_post_eps = ffn_pre_eps, ffn_post_eps
    c.residual_gate_temperature, c.residual_gate_eps = residual_gate_temperature, residual_gate_eps
    c.act_format = act_format
    return c


def workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().muse_latent_moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "workspace_size")
    return int(n.value)


def workspace_layout(cfg: Config) -> Dict[str, int]:
    lay = WorkspaceLayout()
    _check(lib().muse_latent_moe_workspace_layout(ctypes.byref(cfg), ctypes.byref(lay)), "workspace_layout")
    return {name: int(getattr(lay, name)) for name, _ in WorkspaceLayout._fields_}


def launch_count(cfg: Config) -> int:
    return int(lib().muse_latent_moe_launch_count(ctypes.byref(cfg)))


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, ctypes.Structure):
        return ctypes.addressof(t)
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return int(t.data_ptr())


def _stream_handle(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(getattr(stream, "cuda_stream", stream))


def forward(cfg: Config, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out, stream=None) -> None:
    """Enqueue one forward pass; cfg.workspace must point to workspace_size(cfg) bytes."""
    code = lib().muse_latent_moe_forward(ctypes.byref(cfg), _ptr(x), _ptr(W_router), _ptr(W_pool), _ptr(W_gate),
                                         _ptr(W_up), _ptr(W_down), _ptr(gamma), _ptr(W_unpool), _ptr(out),
                                         _stream_handle(stream))
    _check(code, "muse_latent_moe_forward")


def forward_checked(cfg: Config, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out,
                    stream=None) -> None:
    """Enqueue one forward through the shape-checked entry point: every argument is a torch
    tensor (NVFP4 experts: a (codes, block scales, matrix scales) triple each) described by
    its dtype, shape and strides; the library rejects a mismatch before launching anything."""
    def one(t):
        return ctypes.byref(tensor_desc(t))

    def expert(t):
        if isinstance(t, (tuple, list)):
            arr = (Tensor * 3)(*[tensor_desc(p) for p in t])
            return ctypes.cast(arr, ctypes.POINTER(Tensor)), arr
        d = tensor_desc(t)
        return ctypes.pointer(d), d
    eg, eu, ed = expert(W_gate), expert(W_up), expert(W_down)
    code = lib().muse_latent_moe_forward_checked(ctypes.byref(cfg), one(x), one(W_router), one(W_pool), eg[0], eu[0],
                                                 ed[0], one(gamma), one(W_unpool), one(out), _stream_handle(stream))
    _check(code, "muse_latent_moe_forward_checked")


def forward_static_scratch(cfg: Config, x, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool, out,
                           stream=None) -> None:
    """Forward through the allocation-free entry point (workspace = the library's built-in
    scratch array; cfg.workspace is ignored). For callers that cannot allocate device memory."""
    code = lib().muse_latent_moe_forward_static_scratch(ctypes.byref(cfg), _ptr(x), _ptr(W_router), _ptr(W_pool),
                                                        _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(gamma),
                                                        _ptr(W_unpool), _ptr(out), _stream_handle(stream))
    _check(code, "muse_latent_moe_forward_static_scratch")


def forward_host_io(cfg: Config, x_host, x_dev, W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool,
                    out_dev, out_host, stream=None) -> None:
    code = lib().muse_latent_moe_forward_host_io(ctypes.byref(cfg), _ptr(x_host), _ptr(x_dev), _ptr(W_router),
                                                 _ptr(W_pool), _ptr(W_gate), _ptr(W_up), _ptr(W_down),
                                                 _ptr(gamma), _ptr(W_unpool), _ptr(out_dev), _ptr(out_host),
                                                 _stream_handle(stream))
    _check(code, "muse_latent_moe_forward_host_io")


def forward_host_batches(cfg: Config, x_hosts, out_hosts, x_devs, out_devs, W_router, W_pool, W_gate, W_up, W_down,
                         gamma, W_unpool, stream, h2d_stream, d2h_stream) -> None:
    """Batches through the forward with host buffers, copies overlapped with compute (two
    device buffers each for x and out; three distinct torch.cuda.Stream objects)."""
    n = len(x_hosts)
    xh = (ctypes.c_void_p * n)(*[_ptr(t) for t in x_hosts])
    oh = (ctypes.c_void_p * n)(*[_ptr(t) for t in out_hosts])
    xd = (ctypes.c_void_p * 2)(*[_ptr(t) for t in x_devs])
    od = (ctypes.c_void_p * 2)(*[_ptr(t) for t in out_devs])
    code = lib().muse_latent_moe_forward_host_batches(
        ctypes.byref(cfg), n, ctypes.cast(xh, ctypes.c_void_p), ctypes.cast(oh, ctypes.c_void_p),
        ctypes.cast(xd, ctypes.c_void_p), ctypes.cast(od, ctypes.c_void_p), _ptr(W_router), _ptr(W_pool),
        _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(gamma), _ptr(W_unpool), _stream_handle(stream),
        _stream_handle(h2d_stream), _stream_handle(d2h_stream))
    _check(code, "muse_latent_moe_forward_host_batches")


def ep_workspace_layout(cfg: Config, ep_size: int, role: int, rows: int = 0) -> Dict[str, int]:
    """Buffer offsets (and "total" bytes) of an expert-parallel workspace: role EP_HOME for
    cfg.T tokens, EP_EXPERTS for up to `rows` received rows."""
    lay = WorkspaceLayout()
    _check(lib().muse_ep_workspace_layout(ctypes.byref(cfg), int(ep_size), int(role), int(rows), ctypes.byref(lay)),
           "muse_ep_workspace_layout")
    return {name: int(getattr(lay, name)) for name, _ in WorkspaceLayout._fields_}


def ep_dispatch(cfg: Config, ep_size: int, x, W_router, W_pool, send_z, send_expert, rank_counts, stream=None) -> None:
    """Expert-parallel step 1 (cfg.workspace: an EP_HOME workspace)."""
    _check(lib().muse_ep_dispatch(ctypes.byref(cfg), int(ep_size), _ptr(x), _ptr(W_router), _ptr(W_pool), _ptr(send_z),
                                  _ptr(send_expert), _ptr(rank_counts), _stream_handle(stream)), "muse_ep_dispatch")


def ep_experts(cfg: Config, ep_size: int, rows: int, recv_z, recv_expert, W_gate, W_up, W_down, gamma, ret_y, ret_ss,
               stream=None) -> None:
    """Expert-parallel step 3 (cfg.workspace: an EP_EXPERTS workspace)."""
    _check(lib().muse_ep_experts(ctypes.byref(cfg), int(ep_size), int(rows), _ptr(recv_z), _ptr(recv_expert),
                                 _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(gamma), _ptr(ret_y), _ptr(ret_ss),
                                 _stream_handle(stream)), "muse_ep_experts")


def ep_combine(cfg: Config, ep_size: int, x, back_y, back_ss, gamma, W_unpool, out, stream=None) -> None:
    """Expert-parallel step 5 (cfg.workspace: the EP_HOME workspace of step 1)."""
    _check(lib().muse_ep_combine(ctypes.byref(cfg), int(ep_size), _ptr(x), _ptr(back_y), _ptr(back_ss), _ptr(gamma),
                                 _ptr(W_unpool), _ptr(out), _stream_handle(stream)), "muse_ep_combine")


def stages(cfg: Config):
    """Names of the stages one forward launches for cfg, in launch order (from the library:
    muse_latent_moe_stage_name)."""
    names = []
    while True:
        n = lib().muse_latent_moe_stage_name(ctypes.byref(cfg), len(names))
        if n is None:
            return tuple(names)
        names.append(n.decode())


def event_handles(events) -> "ctypes.Array":
    """ctypes array of the raw cudaEvent_t handles of torch.cuda.Event objects (each
    recorded once beforehand so that it exists)."""
    arr = (ctypes.c_void_p * len(events))()
    for i, ev in enumerate(events):
        arr[i] = int(ev.cuda_event)
    return arr


def quantize_nvfp4_rows(src, codes, scales, stream=None) -> None:
    """NVFP4 activation quantiser: src bf16 [rows, K] -> codes uint8 [rows, K/2], scales
    uint8 [rows, K/16] (CUDA tensors)."""
    rows, K = src.shape
    _check(lib().muse_quantize_nvfp4_rows(_ptr(src), int(rows), int(K), _ptr(codes), _ptr(scales),
                                          _stream_handle(stream)), "muse_quantize_nvfp4_rows")


def selftest_bounded_wait(limit_ns: int, status_dev, stream=None) -> None:
    """Run the device-side bounded-wait self-test (status_dev: zeroed CUDA int32[2])."""
    _check(lib().muse_selftest_bounded_wait(int(limit_ns), _ptr(status_dev), _stream_handle(stream)),
           "muse_selftest_bounded_wait")


def last_device_status(cfg: Config, stream=None):
    detail = ctypes.c_uint32(0)
    code = lib().muse_latent_moe_last_device_status(ctypes.byref(cfg), _stream_handle(stream), ctypes.byref(detail))
    return int(code), int(detail.value)


def expert_weight_dims(weights: Dict):
    """(I, L, nvfp4) from the expert weights: dense W_gate [E, I, L], or NVFP4 codes
    W_gate_codes [E, I, L/2]."""
    if "W_gate_codes" in weights:
        _, I, L2 = weights["W_gate_codes"].shape
        return int(I), int(2 * L2), True
    _, I, L = weights["W_gate"].shape
    return int(I), int(L), False


def expert_operands(weights: Dict, nvfp4: bool):
    """The W_gate, W_up, W_down arguments of the C ABI: the dense tensors, or Nvfp4Weight
    descriptors of <name>_codes [E, out, in/2], <name>_scales [E, out, in/16] and
    <name>_mscale [E]."""
    if not nvfp4:
        return tuple(weights[n] for n in ("W_gate", "W_up", "W_down"))
    return tuple(Nvfp4Weight(_ptr(weights[n + "_codes"]), _ptr(weights[n + "_scales"]), _ptr(weights[n + "_mscale"]))
                 for n in ("W_gate", "W_up", "W_down"))


def block_config(T: int, dims: Dict, dtype: str, modes: Dict, weights: Dict, nvfp4: bool, workspace=None) -> Config:
    """Config of the block for T tokens: sizes, modes, the optional pointers found in
    weights (router_bias, pre_norm_gain, ffn_pre_gain, ffn_post_gain, residual_gate) and
    the workspace (a uint8 CUDA tensor) if given."""
    d = dims
    c = make_config(T, d["D"], d["L"], d["I"], d["E"], d["k"], dtype, d["eps"], **modes)
    if nvfp4:
        c.expert_weights = EXPERTS_NVFP4
    if weights.get("router_bias") is not None:
        c.router_bias = _ptr(weights["router_bias"])
    for name in ("pre_norm_gain", "ffn_pre_gain", "ffn_post_gain", "residual_gate"):
        if weights.get(name) is not None:
            setattr(c, name, _ptr(weights[name]))
    if workspace is not None:
        c.workspace = _ptr(workspace)
        c.workspace_bytes = workspace.numel()
    return c


class LatentMoE:
    """Holds the block's device weights and a workspace; calling it runs the forward through
    the shape-checked entry point (muse_latent_moe_forward_checked).

    weights: dict with W_router, W_pool, W_gate, W_up, W_down, gamma, W_unpool (torch
    CUDA tensors in the layouts of include/muse_moe.h); router_bias, pre_norm_gain and the
    feed-forward sublayer's ffn_pre_gain, ffn_post_gain and residual_gate (float32) are
    optional. modes: make_config keywords (router_mode, norm_mode, gamma_shared, ...).
    """

    def __init__(self, weights: Dict, T_max: int, k: int, eps: float = 1e-6, **modes):
        import torch
        self.w = dict(weights)
        E, D = weights["W_router"].shape
        I, L, self.nvfp4 = expert_weight_dims(weights)
        # the expert tensors as the shape-checked entry point takes them
        self.experts = tuple((weights[n + "_codes"], weights[n + "_scales"], weights[n + "_mscale"]) if self.nvfp4
                             else weights[n] for n in ("W_gate", "W_up", "W_down"))
        self.w["W_gate"], self.w["W_up"], self.w["W_down"] = expert_operands(weights, self.nvfp4)
        self.dtype = {torch.float32: "f32", torch.bfloat16: "bf16"}[weights["W_router"].dtype]
        self.dims = dict(D=int(D), L=L, I=I, E=int(E), k=k, eps=eps)
        self.modes = modes
        cfg = self.config(T_max)
        self.workspace = torch.empty(workspace_size(cfg), dtype=torch.uint8, device=weights["W_router"].device)
        self.T_max = T_max

    def config(self, T: int, workspace=None) -> Config:
        return block_config(T, self.dims, self.dtype, self.modes, self.w, self.nvfp4, workspace)

    def __call__(self, x, out=None, stream=None, topk_idx=None, topk_w=None, stage_events=None):
        """stage_events: optional ctypes array of launch_count + 1 cudaEvent_t handles."""
        import torch
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} exceeds T_max={self.T_max}")
        cfg = self.config(T, self.workspace)
        cfg.topk_idx_out, cfg.topk_w_out = _ptr(topk_idx), _ptr(topk_w)
        if stage_events is not None:
            cfg.stage_events = ctypes.cast(stage_events, ctypes.c_void_p)
        if out is None:
            out = torch.empty((T, self.dims["D"]), dtype=x.dtype, device=x.device)
        w = self.w
        forward_checked(cfg, x, w["W_router"], w["W_pool"], *self.experts, w["gamma"], w["W_unpool"], out, stream)
        return out
