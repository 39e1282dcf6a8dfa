"""Python binding of the single-GPU MoE-layer forward library (libmoe_b200.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. torch supplies device memory (inputs, weights, outputs and the
workspace) and the stream. If the library has not been built the import of
the binding fails loudly; there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_NO_WORKSPACE", 5: "MOE_ERR_CUDA",
    6: "MOE_ERR_DEVICE_TIMEOUT", 7: "MOE_ERR_DEVICE_BOUNDS", 8: "MOE_ERR_UNSUPPORTED_DEVICE",
    9: "MOE_ERR_STATIC_SCRATCH_LIMIT",
}
KERNEL_NAMES = ("router", "dispatch_scan", "dispatch_scatter", "expert_gemm", "finalize")

_c_int, _c_size, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p


class MoERouting(ctypes.Structure):
    _fields_ = [("topk_idx", _vp), ("topk_w", _vp), ("expert_count", _vp), ("expert_offset", _vp),
                ("slot_token", _vp), ("slot_topk", _vp), ("num_padded", _vp),
                ("block_m", ctypes.c_int32), ("pool_capacity", ctypes.c_int32)]


class MoEPlanDesc(ctypes.Structure):
    _fields_ = [("T_max", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("block_m", ctypes.c_int32),
                ("pool_capacity", ctypes.c_int32), ("num_sms", ctypes.c_int32),
                ("pair_clusters", ctypes.c_int32), ("cta_pairs", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("workspace_bytes", ctypes.c_size_t),
                ("task_order", ctypes.c_int32), ("half_tails", ctypes.c_int32), ("wide_l1", ctypes.c_int32)]


# exported symbol -> (restype, argtypes); the same list as include/moe_b200.h
SIGNATURES = {
    "moe_plan_create": (_c_int, [ctypes.POINTER(_vp), _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "moe_plan_create_shared": (_c_int, [ctypes.POINTER(_vp), _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                        _c_int]),
    "moe_plan_workspace_bytes": (_c_size, [_vp]),
    "moe_plan_bind_workspace": (_c_int, [_vp, _vp, _c_size]),
    "moe_plan_describe": (_c_int, [_vp, ctypes.POINTER(MoEPlanDesc)]),
    "moe_plan_get_routing": (_c_int, [_vp, ctypes.POINTER(MoERouting)]),
    "moe_forward": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_forward_host": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_forward_shared": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_forward_host_shared": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_forward_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_forward_host_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_quantize_weights_fp8": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp]),
    "moe_forward_host_pipelined": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_forward_host_pipelined_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "moe_host_pipeline_after": (_c_int, [_vp, _vp]),
    "moe_host_pipeline_join": (_c_int, [_vp, _vp]),
    "moe_quantize_x_fp8": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _vp]),
    "moe_route": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _vp]),
    "moe_check": (_c_int, [_vp, _vp, ctypes.POINTER(ctypes.c_int32)]),
    "moe_plan_set_profiling": (_c_int, [_vp, _c_int]),
    "moe_plan_profile_read": (_c_int, [_vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_c_int)]),
    "moe_plan_set_debug": (_c_int, [_vp, _c_int, ctypes.c_uint64]),
    "moe_route_static": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp,
                                  _vp, _vp, _c_int, _vp, _vp, _vp]),
    "moe_plan_set_cta_pairs": (_c_int, [_vp, _c_int]),
    "moe_plan_set_backward": (_c_int, [_vp, _c_int]),
    "moe_backward": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_plan_set_task_order": (_c_int, [_vp, _c_int]),
    "moe_plan_set_half_tails": (_c_int, [_vp, _c_int]),
    "moe_plan_set_wide_l1": (_c_int, [_vp, _c_int]),
    "moe_plan_set_task_log": (_c_int, [_vp, _c_int]),
    "moe_plan_get_task_log": (_c_int, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_c_int)]),
    "moe_plan_set_fp8": (_c_int, [_vp, _c_int]),
    "moe_forward_kernel_count": (_c_int, []),
    "moe_plan_forward_launches": (_c_int, [_vp, _c_int]),
    "moe_plan_destroy": (None, [_vp]),
    "moe_status_string": (ctypes.c_char_p, [_c_int]),
}

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe_b200.so and declare every exported entry point."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m moe_megakernel_b200.build` "
                          "(the CUDA library is the only implementation)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        msg = load_library().moe_status_string(status).decode()
        super().__init__(f"{what}: {name} ({msg})")


def _ok(rc: int, what: str):
    if rc != MOE_OK:
        raise MoEError(rc, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t: torch.Tensor, name: str, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class MoEPlan:
    """A plan for one MoE layer shape plus its device workspace.

    ``forward`` runs gate -> dispatch -> expert FFN -> combine for x [T,H]
    (T <= T_max) and returns y [T,H] bf16. ``routing(T)`` returns views of the
    routing results of the last call.
    """

    def __init__(self, T_max: int, H: int, I: int, E: int, k: int, block_m: int = 0, device=None,
                 n_shared: int = 0, fp8: bool = False, backward: bool = False, task_log: bool = False):
        self.lib = load_library()
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None
                                   else torch.device(device).index or 0)
        self.T_max, self.H, self.I, self.E, self.k, self.n_shared = T_max, H, I, E, k, n_shared
        self._plan = ctypes.c_void_p()
        _ok(self.lib.moe_plan_create_shared(ctypes.byref(self._plan), T_max, H, I, E, k, n_shared, block_m,
                                            self.device.index), "moe_plan_create_shared")
        self.fp8 = bool(fp8)
        if fp8:   # workspace regions of forward_fp8
            _ok(self.lib.moe_plan_set_fp8(self._plan, 1), "moe_plan_set_fp8")
        self.has_backward = bool(backward)
        if backward:   # workspace regions of backward
            _ok(self.lib.moe_plan_set_backward(self._plan, 1), "moe_plan_set_backward")
        if task_log:   # workspace region of the expert GEMM's task log
            _ok(self.lib.moe_plan_set_task_log(self._plan, 1), "moe_plan_set_task_log")
        d = MoEPlanDesc()
        _ok(self.lib.moe_plan_describe(self._plan, ctypes.byref(d)), "moe_plan_describe")
        self.block_m, self.pool_capacity, self.num_sms = d.block_m, d.pool_capacity, d.num_sms
        self.pair_clusters = d.pair_clusters
        self.workspace_bytes = d.workspace_bytes
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        _ok(self.lib.moe_plan_bind_workspace(self._plan, _ptr(self.workspace), self.workspace_bytes),
            "moe_plan_bind_workspace")

    # ------------------------------------------------------------------ calls
    def _check_inputs(self, x, Wg, bias, W=None, Ws=None):
        T = x.shape[0]
        _check(x, "x", (T, self.H), torch.bfloat16, self.device)
        _check(Wg, "Wg", (self.H, self.E), torch.bfloat16, self.device)
        if bias is not None:
            _check(bias, "bias", (self.E,), torch.float32, self.device)
        if W is not None:
            W1, W3, W2 = W
            _check(W1, "W1", (self.E, self.H, self.I), torch.bfloat16, self.device)
            _check(W3, "W3", (self.E, self.H, self.I), torch.bfloat16, self.device)
            _check(W2, "W2", (self.E, self.I, self.H), torch.bfloat16, self.device)
        if self.n_shared and Ws is not None:
            Ws1, Ws3, Ws2 = Ws
            S = self.n_shared
            _check(Ws1, "Ws1", (S, self.H, self.I), torch.bfloat16, self.device)
            _check(Ws3, "Ws3", (S, self.H, self.I), torch.bfloat16, self.device)
            _check(Ws2, "Ws2", (S, self.I, self.H), torch.bfloat16, self.device)
        return T

    def forward(self, x, Wg, bias, W1, W3, W2, y=None, stream=None, Ws1=None, Ws3=None, Ws2=None) -> torch.Tensor:
        """Ws1/Ws3/Ws2: the shared experts' weights, required when the plan has n_shared > 0."""
        T = self._check_inputs(x, Wg, bias, (W1, W3, W2), (Ws1, Ws3, Ws2))
        if y is None:
            y = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        _check(y, "y", (T, self.H), torch.bfloat16, self.device)
        _ok(self.lib.moe_forward_shared(self._plan, _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2),
                                        _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), T, _ptr(y),
                                        _stream_handle(stream, self.device)), "moe_forward_shared")
        return y

    def forward_host(self, x_host, Wg, bias, W1, W3, W2, y_host, stream=None, Ws1=None, Ws3=None, Ws2=None):
        """x_host and y_host are CPU bf16 tensors (pinned for asynchronous copies)."""
        T = x_host.shape[0]
        _check(x_host, "x_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(y_host, "y_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(Wg, "Wg", (self.H, self.E), torch.bfloat16, self.device)
        _ok(self.lib.moe_forward_host_shared(self._plan, _ptr(x_host), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3),
                                             _ptr(W2), _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), T, _ptr(y_host),
                                             _stream_handle(stream, self.device)),
            "moe_forward_host_shared")
        return y_host

    def _check_fp8(self, W1q, s1, W3q, s3, W2q, s2):
        E, H, I = self.E, self.H, self.I
        _check(W1q, "W1q", (E, I, H), torch.uint8, self.device)
        _check(W3q, "W3q", (E, I, H), torch.uint8, self.device)
        _check(W2q, "W2q", (E, H, I), torch.uint8, self.device)
        _check(s1, "s1", (E, I), torch.float32, self.device)
        _check(s3, "s3", (E, I), torch.float32, self.device)
        _check(s2, "s2", (E, H), torch.float32, self.device)

    def forward_fp8(self, x, Wg, bias, W1q, s1, W3q, s3, W2q, s2, y=None, stream=None) -> torch.Tensor:
        """Forward with FP8 E4M3 expert GEMMs; (W1q, s1), (W3q, s3), (W2q, s2) from quantize_weights_fp8."""
        T = self._check_inputs(x, Wg, bias)
        self._check_fp8(W1q, s1, W3q, s3, W2q, s2)
        if y is None:
            y = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        _check(y, "y", (T, self.H), torch.bfloat16, self.device)
        _ok(self.lib.moe_forward_fp8(self._plan, _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1q), _ptr(s1), _ptr(W3q),
                                     _ptr(s3), _ptr(W2q), _ptr(s2), T, _ptr(y), _stream_handle(stream, self.device)),
            "moe_forward_fp8")
        return y

    def forward_host_fp8(self, x_host, Wg, bias, W1q, s1, W3q, s3, W2q, s2, y_host, stream=None):
        """forward_fp8 with x_host / y_host CPU bf16 tensors (pinned for asynchronous copies)."""
        T = x_host.shape[0]
        _check(x_host, "x_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(y_host, "y_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(Wg, "Wg", (self.H, self.E), torch.bfloat16, self.device)
        self._check_fp8(W1q, s1, W3q, s3, W2q, s2)
        _ok(self.lib.moe_forward_host_fp8(self._plan, _ptr(x_host), _ptr(Wg), _ptr(bias), _ptr(W1q), _ptr(s1),
                                          _ptr(W3q), _ptr(s3), _ptr(W2q), _ptr(s2), T, _ptr(y_host),
                                          _stream_handle(stream, self.device)), "moe_forward_host_fp8")
        return y_host

    def forward_host_pipelined(self, x_host, Wg, bias, W1, W3, W2, y_host, stream=None):
        """Pipelined host-buffer forward (copies on the plan's own streams, see the C header);
        call host_pipeline_join(stream) before synchronising and reading y_host."""
        T = x_host.shape[0]
        _check(x_host, "x_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(y_host, "y_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(Wg, "Wg", (self.H, self.E), torch.bfloat16, self.device)
        _ok(self.lib.moe_forward_host_pipelined(self._plan, _ptr(x_host), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3),
                                                _ptr(W2), T, _ptr(y_host), _stream_handle(stream, self.device)),
            "moe_forward_host_pipelined")
        return y_host

    def forward_host_pipelined_fp8(self, x_host, Wg, bias, W1q, s1, W3q, s3, W2q, s2, y_host, stream=None):
        """forward_host_pipelined with FP8 expert GEMMs."""
        T = x_host.shape[0]
        _check(x_host, "x_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(y_host, "y_host", (T, self.H), torch.bfloat16, torch.device("cpu"))
        _check(Wg, "Wg", (self.H, self.E), torch.bfloat16, self.device)
        self._check_fp8(W1q, s1, W3q, s3, W2q, s2)
        _ok(self.lib.moe_forward_host_pipelined_fp8(self._plan, _ptr(x_host), _ptr(Wg), _ptr(bias), _ptr(W1q),
                                                    _ptr(s1), _ptr(W3q), _ptr(s3), _ptr(W2q), _ptr(s2), T,
                                                    _ptr(y_host), _stream_handle(stream, self.device)),
            "moe_forward_host_pipelined_fp8")
        return y_host

    def host_pipeline_after(self, stream=None):
        _ok(self.lib.moe_host_pipeline_after(self._plan, _stream_handle(stream, self.device)), "moe_host_pipeline_after")

    def host_pipeline_join(self, stream=None):
        _ok(self.lib.moe_host_pipeline_join(self._plan, _stream_handle(stream, self.device)), "moe_host_pipeline_join")

    def backward(self, x, Wg, bias, W1, W3, W2, dy, stream=None, out=None) -> dict:
        """Gradients of the layer for the upstream dy [T,H] bf16 (plan made with backward=True):
        dict of dx [T,H] bf16, dWg [H,E] fp32, dbias [E] fp32 (None when bias is None),
        dW1/dW3 [E,H,I] bf16, dW2 [E,I,H] bf16. ``out`` may supply these tensors."""
        T = self._check_inputs(x, Wg, bias, (W1, W3, W2))
        _check(dy, "dy", (T, self.H), torch.bfloat16, self.device)
        o = dict(out) if out is not None else {}
        dev = self.device
        E, H, I = self.E, self.H, self.I
        o.setdefault("dx", torch.empty((T, H), dtype=torch.bfloat16, device=dev))
        o.setdefault("dWg", torch.empty((H, E), dtype=torch.float32, device=dev))
        o.setdefault("dbias", None if bias is None else torch.empty((E,), dtype=torch.float32, device=dev))
        o.setdefault("dW1", torch.empty((E, H, I), dtype=torch.bfloat16, device=dev))
        o.setdefault("dW3", torch.empty((E, H, I), dtype=torch.bfloat16, device=dev))
        o.setdefault("dW2", torch.empty((E, I, H), dtype=torch.bfloat16, device=dev))
        _check(o["dx"], "dx", (T, H), torch.bfloat16, dev)
        _check(o["dWg"], "dWg", (H, E), torch.float32, dev)
        if o["dbias"] is not None:
            _check(o["dbias"], "dbias", (E,), torch.float32, dev)
        _check(o["dW1"], "dW1", (E, H, I), torch.bfloat16, dev)
        _check(o["dW3"], "dW3", (E, H, I), torch.bfloat16, dev)
        _check(o["dW2"], "dW2", (E, I, H), torch.bfloat16, dev)
        _ok(self.lib.moe_backward(self._plan, _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dy),
                                  T, _ptr(o["dx"]), _ptr(o["dWg"]), _ptr(o["dbias"]), _ptr(o["dW1"]), _ptr(o["dW3"]),
                                  _ptr(o["dW2"]), _stream_handle(stream, dev)), "moe_backward")
        return o

    def route(self, x, Wg, bias, stream=None):
        T = self._check_inputs(x, Wg, bias)
        _ok(self.lib.moe_route(self._plan, _ptr(x), _ptr(Wg), _ptr(bias), T,
                               _stream_handle(stream, self.device)), "moe_route")

    def check(self, stream=None) -> int:
        """Synchronise; raise MoEError on a sticky device error (and clear it)."""
        detail = ctypes.c_int32(0)
        rc = self.lib.moe_check(self._plan, _stream_handle(stream, self.device), ctypes.byref(detail))
        self.last_error_detail = detail.value
        _ok(rc, "device")
        return rc

    def routing(self, T: int) -> dict:
        """Views (into the workspace) of the routing results for the last T-token call."""
        r = MoERouting()
        _ok(self.lib.moe_plan_get_routing(self._plan, ctypes.byref(r)), "moe_plan_get_routing")
        base = self.workspace.data_ptr()

        def view(ptr, n, dtype):
            off = ptr - base
            nbytes = n * 4
            return self.workspace[off:off + nbytes].view(dtype)

        E, k = self.E, self.k
        return dict(
            topk_idx=view(r.topk_idx, T * k, torch.int32).view(T, k),
            topk_w=view(r.topk_w, T * k, torch.float32).view(T, k),
            expert_count=view(r.expert_count, E, torch.int32),
            expert_offset=view(r.expert_offset, E + 1, torch.int32),
            slot_token=view(r.slot_token, r.pool_capacity, torch.int32),
            slot_topk=view(r.slot_topk, r.pool_capacity, torch.int32),
            num_padded=view(r.num_padded, 1, torch.int32),
            block_m=r.block_m,
        )

    def task_log(self) -> dict:
        """The expert GEMM's task records of the last launch (plan made with task_log=True), as
        int64 tensors on the host: task, unit, expert, phase, n, smid, cta, t_first_mma,
        t_last_mma, t_done (ns); only the records of tasks that ran."""
        ptr, cap = ctypes.c_void_p(), ctypes.c_int(0)
        _ok(self.lib.moe_plan_get_task_log(self._plan, ctypes.byref(ptr), ctypes.byref(cap)), "moe_plan_get_task_log")
        off = ptr.value - self.workspace.data_ptr()
        raw = self.workspace[off:off + cap.value * 48].cpu()
        u32 = raw.view(torch.int32).view(cap.value, 12).to(torch.int64) & 0xFFFFFFFF
        u64 = raw.view(torch.int64).view(cap.value, 6)
        keep = u32[:, 0] != 0xFFFFFFFF
        return dict(task=u32[keep, 0], unit=u32[keep, 1], expert=u32[keep, 2], phase=u32[keep, 3] >> 16,
                    n=u32[keep, 3] & 0xFFFF, smid=u32[keep, 4], cta=u32[keep, 5], t_first_mma=u64[keep, 3],
                    t_last_mma=u64[keep, 4], t_done=u64[keep, 5])

    def set_profiling(self, enable: bool):
        _ok(self.lib.moe_plan_set_profiling(self._plan, 1 if enable else 0), "moe_plan_set_profiling")

    def profile_read(self):
        """(summed ms per kernel since the last read as a dict, number of forwards)."""
        ms = (ctypes.c_float * 5)()
        n = ctypes.c_int(0)
        _ok(self.lib.moe_plan_profile_read(self._plan, ms, ctypes.byref(n)), "moe_plan_profile_read")
        return dict(zip(KERNEL_NAMES, list(ms))), n.value

    def set_cta_pairs(self, enable: bool):
        _ok(self.lib.moe_plan_set_cta_pairs(self._plan, 1 if enable else 0), "moe_plan_set_cta_pairs")

    def set_task_order(self, mode: int):
        """-1 automatic, 0 staggered, 1 interleaved (see moe_plan_set_task_order)."""
        _ok(self.lib.moe_plan_set_task_order(self._plan, int(mode)), "moe_plan_set_task_order")

    def set_half_tails(self, enable: bool):
        """Run an expert's lone last block as M = 128 pair MMAs (see moe_plan_set_half_tails)."""
        _ok(self.lib.moe_plan_set_half_tails(self._plan, 1 if enable else 0), "moe_plan_set_half_tails")

    def set_wide_l1(self, mode):
        """256-column first-GEMM tasks on CTA pairs: True / 1, False / 0, or -1 automatic
        (see moe_plan_set_wide_l1)."""
        m = int(mode) if not isinstance(mode, bool) else (1 if mode else 0)
        _ok(self.lib.moe_plan_set_wide_l1(self._plan, m), "moe_plan_set_wide_l1")

    def forward_launches(self, fp8: bool = False) -> int:
        """Kernels one forward of this plan launches (see moe_plan_forward_launches)."""
        n = self.lib.moe_plan_forward_launches(self._plan, 1 if fp8 else 0)
        if n < 0:
            raise RuntimeError("moe_plan_forward_launches: no FP8 regions in this plan")
        return n

    @property
    def wide_l1(self) -> bool:
        d = MoEPlanDesc()
        _ok(self.lib.moe_plan_describe(self._plan, ctypes.byref(d)), "moe_plan_describe")
        return bool(d.wide_l1)

    @property
    def half_tails(self) -> bool:
        d = MoEPlanDesc()
        _ok(self.lib.moe_plan_describe(self._plan, ctypes.byref(d)), "moe_plan_describe")
        return bool(d.half_tails)

    @property
    def task_order(self) -> int:
        """The expert-GEMM task order in use: 0 staggered, 1 interleaved."""
        d = MoEPlanDesc()
        _ok(self.lib.moe_plan_describe(self._plan, ctypes.byref(d)), "moe_plan_describe")
        return int(d.task_order)

    @property
    def cta_pairs(self) -> bool:
        """Whether the expert GEMM currently runs on CTA pairs."""
        d = MoEPlanDesc()
        _ok(self.lib.moe_plan_describe(self._plan, ctypes.byref(d)), "moe_plan_describe")
        return bool(d.cta_pairs)

    def set_debug(self, withhold_block: int = -1, timeout_ns: int = 0):
        _ok(self.lib.moe_plan_set_debug(self._plan, withhold_block, timeout_ns), "moe_plan_set_debug")

    def close(self):
        if getattr(self, "_plan", None) and self._plan.value:
            self.lib.moe_plan_destroy(self._plan)
            self._plan = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def quantize_weights_fp8(W: torch.Tensor, stream=None):
    """W bf16 [E, K, N] (W1 / W3: K = H, N = I; W2: K = I, N = H) ->
    (K-major E4M3 codes u8 [E, N, K], per-column scales over K fp32 [E, N])."""
    if not isinstance(W, torch.Tensor) or W.dim() != 3:
        raise TypeError("W must be a 3-D torch.Tensor [E, K, N]")
    E, H, I = W.shape
    _check(W, "W", (E, H, I), torch.bfloat16, None)
    Wq = torch.empty((E, I, H), dtype=torch.uint8, device=W.device)
    sc = torch.empty((E, I), dtype=torch.float32, device=W.device)
    _ok(load_library().moe_quantize_weights_fp8(_ptr(W), _ptr(Wq), _ptr(sc), E, H, I,
                                                _stream_handle(stream, W.device)), "moe_quantize_weights_fp8")
    return Wq, sc


def quantize_x_fp8(x: torch.Tensor, stream=None):
    """x bf16 [T, H] -> (E4M3 codes u8 [T, H], per-token scales fp32 [T]), as the FP8 forward forms them."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise TypeError("x must be a 2-D torch.Tensor [T, H]")
    T, H = x.shape
    _check(x, "x", (T, H), torch.bfloat16, None)
    xq = torch.empty((T, H), dtype=torch.uint8, device=x.device)
    sx = torch.empty((T,), dtype=torch.float32, device=x.device)
    _ok(load_library().moe_quantize_x_fp8(_ptr(x), _ptr(xq), _ptr(sx), T, H, _stream_handle(stream, x.device)),
        "moe_quantize_x_fp8")
    return xq, sx


def kernels_per_forward() -> int:
    return load_library().moe_forward_kernel_count()
