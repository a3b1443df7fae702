"""Thin ctypes binding over libbsattn.so (include/bsattn.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels. Functions keep the C names; tensors are torch CUDA
tensors whose data pointers are passed through, and the stream is torch's
current stream unless one is given. If the shared library is missing the
import fails loudly: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsattn.so")

RULE_TOPK, RULE_TOPP, RULE_WINDOW = 0, 1, 2
_RULES = {"topk": RULE_TOPK, "topp": RULE_TOPP, "window": RULE_WINDOW}

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
          4: "device wait timed out", 5: "device reported a bad kept-list entry",
          6: "workspace missing or too small"}


class BsattnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, 'unknown')} (status {code})")
        self.code = code


class Desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("tile_t", ctypes.c_int), ("tile_h", ctypes.c_int), ("tile_w", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("qk_fp8", ctypes.c_int)]


class Rule(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("k", ctypes.c_int), ("p", ctypes.c_double),
                ("win_t", ctypes.c_int), ("win_h", ctypes.c_int), ("win_w", ctypes.c_int)]


class ScheduleEntry(ctypes.Structure):
    _fields_ = [("first_step", ctypes.c_int), ("desc", Desc), ("rule", Rule)]


class Info(ctypes.Structure):
    _fields_ = [("Tp", ctypes.c_int), ("Hp", ctypes.c_int), ("Wp", ctypes.c_int),
                ("nT", ctypes.c_int), ("nH", ctypes.c_int), ("nW", ctypes.c_int),
                ("n_blocks", ctypes.c_int), ("tile_volume", ctypes.c_int), ("kmax", ctypes.c_int),
                ("softmax_scale", ctypes.c_float),
                ("select_workspace_bytes", ctypes.c_size_t),
                ("forward_workspace_bytes", ctypes.c_size_t),
                ("layer_workspace_bytes", ctypes.c_size_t),
                ("backward_workspace_bytes", ctypes.c_size_t)]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libbsattn.so not built ({path}); run "
                          "python -m block_sparse_attention_reorder_b200.build")
    lib = ctypes.CDLL(path)
    P, I, Z, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_double
    sig = {
        "attn_plan_create": [ctypes.POINTER(Desc), ctypes.POINTER(Rule), ctypes.POINTER(P)],
        "attn_plan_destroy": [P],
        "attn_plan_info": [P, ctypes.POINTER(Info)],
        "attn_status_string": [I],
        "attn_reorder": [P, P, P, P, P],
        "attn_pool": [P, P, P, P],
        "attn_unreorder": [P, P, P, P],
        "attn_block_scores": [P, P, P, P, P],
        "attn_select_from_scores": [P, P, P, P, P],
        "attn_select": [P, P, P, P, P, P, Z, P],
        "attn_select_static": [P, P, P, P, P, P],
        "attn_select_fused": [P, P, P, P, P, P, P, Z, P],
        "attn_quantize_e4m3": [P, P, P, P, P],
        "attn_forward": [P, P, P, P, P, P, P, P, P, P, P, Z, P],
        "attn_forward_natural": [P, P, P, P, P, P, P, P, P, P, P, Z, P],
        "attn_layer": [P, P, P, P, P, P, P, P, P, Z, P],
        "attn_check_device_status": [P, P],
        "attn_backward": [P, P, P, P, P, P, P, P, P, P, P, P, P, Z, P],
        "attn_schedule_create": [ctypes.POINTER(ScheduleEntry), I, ctypes.POINTER(P)],
        "attn_schedule_destroy": [P],
        "attn_schedule_plan": [P, I, ctypes.POINTER(P)],
        "attn_schedule_workspace_bytes": [P, ctypes.POINTER(Z)],
        "attn_schedule_layer": [P, I, P, P, P, P, P, P, P, P, Z, P],
        "attn_testing_force_timeout": [I],
        "attn_testing_set_error_word": [P, I],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "attn_status_string" else (
            None if name in ("attn_plan_destroy", "attn_schedule_destroy") else ctypes.c_int)
    return lib


_lib = load_library()
EXPORTED = ("attn_plan_create", "attn_plan_destroy", "attn_plan_info", "attn_status_string",
            "attn_reorder", "attn_pool", "attn_unreorder", "attn_block_scores",
            "attn_select_from_scores", "attn_select", "attn_select_static", "attn_select_fused",
            "attn_quantize_e4m3",
            "attn_forward", "attn_forward_natural",
            "attn_layer", "attn_check_device_status", "attn_schedule_create", "attn_schedule_destroy",
            "attn_schedule_plan", "attn_schedule_workspace_bytes", "attn_schedule_layer",
            "attn_backward", "attn_testing_force_timeout", "attn_testing_set_error_word")


def _check(code: int, where: str):
    if code != 0:
        raise BsattnError(code, where)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _want(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


class Plan:
    """An immutable problem + rule description (attn_plan_create)."""

    def __init__(self, B, heads, head_dim, T, H, W, rule="topk", k=0, p=0.0, win=(0, 0, 0),
                 tile=(4, 4, 4), softmax_scale=0.0, qk_fp8=False, _handle=None):
        self.desc = Desc(B, heads, head_dim, T, H, W, tile[0], tile[1], tile[2],
                         float(softmax_scale), int(bool(qk_fp8)))
        self.rule = Rule(_RULES[rule] if isinstance(rule, str) else int(rule), int(k), float(p),
                         int(win[0]), int(win[1]), int(win[2]))
        self._owned = _handle is None
        if _handle is None:
            h = ctypes.c_void_p()
            _check(_lib.attn_plan_create(ctypes.byref(self.desc), ctypes.byref(self.rule),
                                         ctypes.byref(h)), "attn_plan_create")
        else:
            h = _handle  # a plan owned by a Schedule
        self.handle = h
        info = Info()
        _check(_lib.attn_plan_info(h, ctypes.byref(info)), "attn_plan_info")
        self.info = info
        self.B, self.heads, self.D = B, heads, head_dim
        self.T, self.H, self.W = T, H, W
        self.L = T * H * W
        self.N = info.n_blocks
        self.V = info.tile_volume
        self.tile = tuple(tile)
        self.kmax = info.kmax
        self.qk_fp8 = bool(qk_fp8)

    @classmethod
    def for_workload(cls, wl):
        return cls(wl.B, wl.heads, wl.head_dim, wl.T, wl.H, wl.W, rule=wl.rule, k=wl.k, p=wl.p,
                   win=wl.win, tile=wl.tile, qk_fp8=wl.qk_fp8)

    def close(self):
        if getattr(self, "handle", None) and getattr(self, "_owned", True):
            _lib.attn_plan_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # shapes
    def natural_shape(self):
        return (self.B, self.L, self.heads, self.D)

    def tiled_shape(self):
        return (self.B, self.heads, self.N, self.V, self.D)

    def list_shapes(self):
        return (self.B, self.heads, self.N, self.kmax), (self.B, self.heads, self.N)

    def workspace(self, which="layer", device="cuda"):
        nbytes = {"select": self.info.select_workspace_bytes,
                  "forward": self.info.forward_workspace_bytes,
                  "layer": self.info.layer_workspace_bytes,
                  "backward": self.info.backward_workspace_bytes}[which]
        return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


class Schedule:
    """Denoising-step-aware list of plans over the same tensors
    (attn_schedule_create). `entries`: (first_step, dict of Plan keyword
    arguments: rule, k, p, win, tile, qk_fp8, softmax_scale)."""

    def __init__(self, B, heads, head_dim, T, H, W, entries):
        arr = (ScheduleEntry * len(entries))()
        for i, (first, kw) in enumerate(entries):
            tile = kw.get("tile", (4, 4, 4))
            rule = kw.get("rule", "topk")
            win = kw.get("win", (0, 0, 0))
            arr[i].first_step = int(first)
            arr[i].desc = Desc(B, heads, head_dim, T, H, W, tile[0], tile[1], tile[2],
                               float(kw.get("softmax_scale", 0.0)), int(bool(kw.get("qk_fp8", False))))
            arr[i].rule = Rule(_RULES[rule] if isinstance(rule, str) else int(rule), int(kw.get("k", 0)),
                               float(kw.get("p", 0.0)), int(win[0]), int(win[1]), int(win[2]))
        h = ctypes.c_void_p()
        _check(_lib.attn_schedule_create(arr, len(entries), ctypes.byref(h)), "attn_schedule_create")
        self.handle = h
        self.first_steps = [int(f) for f, _ in entries]
        self.plans = []
        for i, (first, kw) in enumerate(entries):
            ph = ctypes.c_void_p()
            _check(_lib.attn_schedule_plan(h, int(first), ctypes.byref(ph)), "attn_schedule_plan")
            args = {k: v for k, v in kw.items() if k in ("rule", "k", "p", "win", "tile", "qk_fp8",
                                                         "softmax_scale")}
            self.plans.append(Plan(B, heads, head_dim, T, H, W, _handle=ph, **args))
        nbytes = ctypes.c_size_t()
        _check(_lib.attn_schedule_workspace_bytes(h, ctypes.byref(nbytes)), "attn_schedule_workspace_bytes")
        self.workspace_bytes = int(nbytes.value)

    def plan_for(self, step: int) -> Plan:
        """The plan serving `step` (the same one the library picks)."""
        ph = ctypes.c_void_p()
        _check(_lib.attn_schedule_plan(self.handle, int(step), ctypes.byref(ph)), "attn_schedule_plan")
        for p in self.plans:
            if p.handle.value == ph.value:
                return p
        raise RuntimeError("schedule returned an unknown plan")

    def workspace(self, device="cuda"):
        return torch.empty(max(self.workspace_bytes, 16), dtype=torch.uint8, device=device)

    def close(self):
        if getattr(self, "handle", None):
            for p in self.plans:
                p.handle = None
            _lib.attn_schedule_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def attn_schedule_layer(schedule: Schedule, step: int, q_nat, k_nat, v_nat, o_nat, ws, lse_nat=None,
                        idx=None, cnt=None, stream=None):
    plan = schedule.plan_for(step)
    for name, t in (("q_nat", q_nat), ("k_nat", k_nat), ("v_nat", v_nat), ("o_nat", o_nat)):
        _want(t, torch.bfloat16, plan.natural_shape(), name)
    if lse_nat is not None:
        _want(lse_nat, torch.float32, (plan.B, plan.heads, plan.L), "lse_nat")
    if idx is not None:
        si, sc = plan.list_shapes()
        _want(idx, torch.int32, si, "idx")
        _want(cnt, torch.int32, sc, "cnt")
    _check(_lib.attn_schedule_layer(schedule.handle, int(step), _ptr(q_nat), _ptr(k_nat), _ptr(v_nat),
                                    _ptr(o_nat), _ptr(lse_nat), _ptr(idx), _ptr(cnt), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)),
           "attn_schedule_layer")


def attn_reorder(plan: Plan, x_nat, x_tiled, pooled=None, stream=None):
    _want(x_nat, torch.bfloat16, plan.natural_shape(), "x_nat")
    _want(x_tiled, torch.bfloat16, plan.tiled_shape(), "x_tiled")
    if pooled is not None:
        _want(pooled, torch.float32, (plan.B, plan.heads, plan.N, plan.D), "pooled")
    _check(_lib.attn_reorder(plan.handle, _ptr(x_nat), _ptr(x_tiled), _ptr(pooled),
                             _stream(stream)), "attn_reorder")


def attn_pool(plan: Plan, x_nat, pooled, stream=None):
    _want(x_nat, torch.bfloat16, plan.natural_shape(), "x_nat")
    _want(pooled, torch.float32, (plan.B, plan.heads, plan.N, plan.D), "pooled")
    _check(_lib.attn_pool(plan.handle, _ptr(x_nat), _ptr(pooled), _stream(stream)), "attn_pool")


def attn_unreorder(plan: Plan, x_tiled, x_nat, stream=None):
    _want(x_tiled, torch.bfloat16, plan.tiled_shape(), "x_tiled")
    _want(x_nat, torch.bfloat16, plan.natural_shape(), "x_nat")
    _check(_lib.attn_unreorder(plan.handle, _ptr(x_tiled), _ptr(x_nat), _stream(stream)),
           "attn_unreorder")


def attn_block_scores(plan: Plan, pooled_q, pooled_k, scores, stream=None):
    ps = (plan.B, plan.heads, plan.N, plan.D)
    _want(pooled_q, torch.float32, ps, "pooled_q")
    _want(pooled_k, torch.float32, ps, "pooled_k")
    _want(scores, torch.float32, (plan.B, plan.heads, plan.N, plan.N), "scores")
    _check(_lib.attn_block_scores(plan.handle, _ptr(pooled_q), _ptr(pooled_k), _ptr(scores),
                                  _stream(stream)), "attn_block_scores")


def attn_select_from_scores(plan: Plan, scores, idx, cnt, stream=None):
    si, sc = plan.list_shapes()
    if scores is not None:
        _want(scores, torch.float32, (plan.B, plan.heads, plan.N, plan.N), "scores")
    _want(idx, torch.int32, si, "idx")
    _want(cnt, torch.int32, sc, "cnt")
    _check(_lib.attn_select_from_scores(plan.handle, _ptr(scores), _ptr(idx), _ptr(cnt),
                                        _stream(stream)), "attn_select_from_scores")


def attn_select(plan: Plan, q_nat, k_nat, idx, cnt, ws, stream=None):
    _want(q_nat, torch.bfloat16, plan.natural_shape(), "q_nat")
    _want(k_nat, torch.bfloat16, plan.natural_shape(), "k_nat")
    si, sc = plan.list_shapes()
    _want(idx, torch.int32, si, "idx")
    _want(cnt, torch.int32, sc, "cnt")
    _check(_lib.attn_select(plan.handle, _ptr(q_nat), _ptr(k_nat), _ptr(idx), _ptr(cnt), _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "attn_select")


def attn_select_fused(plan: Plan, q_nat, k_nat, idx, cnt, ws, scores_debug=None, stream=None):
    _want(q_nat, torch.bfloat16, plan.natural_shape(), "q_nat")
    _want(k_nat, torch.bfloat16, plan.natural_shape(), "k_nat")
    si, sc = plan.list_shapes()
    _want(idx, torch.int32, si, "idx")
    _want(cnt, torch.int32, sc, "cnt")
    if scores_debug is not None:
        _want(scores_debug, torch.float32, (plan.B, plan.heads, plan.N, plan.N), "scores_debug")
    _check(_lib.attn_select_fused(plan.handle, _ptr(q_nat), _ptr(k_nat), _ptr(idx), _ptr(cnt),
                                  _ptr(scores_debug), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "attn_select_fused")


STATIC_SELECT_SCRATCH_BYTES = 16 << 20


def attn_select_static(plan: Plan, q_nat, k_nat, idx, cnt, stream=None):
    """attn_select for callers that cannot allocate: scratch is the library's
    static device array (see include/bsattn.h for its limits)."""
    _want(q_nat, torch.bfloat16, plan.natural_shape(), "q_nat")
    _want(k_nat, torch.bfloat16, plan.natural_shape(), "k_nat")
    si, sc = plan.list_shapes()
    _want(idx, torch.int32, si, "idx")
    _want(cnt, torch.int32, sc, "cnt")
    _check(_lib.attn_select_static(plan.handle, _ptr(q_nat), _ptr(k_nat), _ptr(idx), _ptr(cnt),
                                   _stream(stream)), "attn_select_static")


def attn_quantize_e4m3(plan: Plan, x_tiled, codes, scales, stream=None):
    _want(x_tiled, torch.bfloat16, plan.tiled_shape(), "x_tiled")
    _want(codes, torch.uint8, plan.tiled_shape(), "codes")
    _want(scales, torch.float32, (plan.B, plan.heads, plan.N), "scales")
    _check(_lib.attn_quantize_e4m3(plan.handle, _ptr(x_tiled), _ptr(codes), _ptr(scales),
                                   _stream(stream)), "attn_quantize_e4m3")


def attn_forward(plan: Plan, q, k, v, idx, cnt, o_tiled, lse=None, q_scale=None, k_scale=None,
                 ws=None, stream=None):
    qk_dtype = torch.uint8 if plan.qk_fp8 else torch.bfloat16
    _want(q, qk_dtype, plan.tiled_shape(), "q")
    _want(k, qk_dtype, plan.tiled_shape(), "k")
    _want(v, torch.bfloat16, plan.tiled_shape(), "v")
    _want(o_tiled, torch.bfloat16, plan.tiled_shape(), "o_tiled")
    si, sc = plan.list_shapes()
    _want(idx, torch.int32, si, "idx")
    _want(cnt, torch.int32, sc, "cnt")
    if lse is not None:
        _want(lse, torch.float32, (plan.B, plan.heads, plan.N, plan.V), "lse")
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.attn_forward(plan.handle, _ptr(q), _ptr(k), _ptr(q_scale), _ptr(k_scale), _ptr(v),
                             _ptr(idx), _ptr(cnt), _ptr(o_tiled), _ptr(lse), _ptr(ws), wsb,
                             _stream(stream)), "attn_forward")


def attn_forward_natural(plan: Plan, q, k, v_nat, idx, cnt, o_nat, lse_nat=None, q_scale=None,
                         k_scale=None, ws=None, stream=None):
    if plan.qk_fp8:
        _want(q, torch.uint8, plan.tiled_shape(), "q")
        _want(k, torch.uint8, plan.tiled_shape(), "k")
    else:
        _want(q, torch.bfloat16, plan.natural_shape(), "q")
        _want(k, torch.bfloat16, plan.natural_shape(), "k")
    _want(v_nat, torch.bfloat16, plan.natural_shape(), "v_nat")
    _want(o_nat, torch.bfloat16, plan.natural_shape(), "o_nat")
    si, sc = plan.list_shapes()
    _want(idx, torch.int32, si, "idx")
    _want(cnt, torch.int32, sc, "cnt")
    if lse_nat is not None:
        _want(lse_nat, torch.float32, (plan.B, plan.heads, plan.L), "lse_nat")
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.attn_forward_natural(plan.handle, _ptr(q), _ptr(k), _ptr(q_scale), _ptr(k_scale),
                                     _ptr(v_nat), _ptr(idx), _ptr(cnt), _ptr(o_nat), _ptr(lse_nat),
                                     _ptr(ws), wsb, _stream(stream)), "attn_forward_natural")


def attn_layer(plan: Plan, q_nat, k_nat, v_nat, o_nat, ws, lse_nat=None, idx=None, cnt=None,
               stream=None):
    for name, t in (("q_nat", q_nat), ("k_nat", k_nat), ("v_nat", v_nat), ("o_nat", o_nat)):
        _want(t, torch.bfloat16, plan.natural_shape(), name)
    if lse_nat is not None:
        _want(lse_nat, torch.float32, (plan.B, plan.heads, plan.L), "lse_nat")
    if idx is not None:
        si, sc = plan.list_shapes()
        _want(idx, torch.int32, si, "idx")
        _want(cnt, torch.int32, sc, "cnt")
    _check(_lib.attn_layer(plan.handle, _ptr(q_nat), _ptr(k_nat), _ptr(v_nat), _ptr(o_nat),
                           _ptr(lse_nat), _ptr(idx), _ptr(cnt), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream)), "attn_layer")


def attn_backward(plan: Plan, q_t, k_t, v_t, o_t, do_t, lse_t, idx, cnt, dq_t, dk_t, dv_t, ws, stream=None):
    ts = plan.tiled_shape()
    for name, t in (("q", q_t), ("k", k_t), ("v", v_t), ("o", o_t), ("do", do_t), ("dq", dq_t), ("dk", dk_t),
                    ("dv", dv_t)):
        _want(t, torch.bfloat16, ts, name)
    _want(lse_t, torch.float32, (plan.B, plan.heads, plan.N, plan.V), "lse")
    si, sc = plan.list_shapes()
    _want(idx, torch.int32, si, "idx")
    _want(cnt, torch.int32, sc, "cnt")
    _check(_lib.attn_backward(plan.handle, _ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(o_t), _ptr(do_t), _ptr(lse_t),
                              _ptr(idx), _ptr(cnt), _ptr(dq_t), _ptr(dk_t), _ptr(dv_t), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream)), "attn_backward")


def attn_check_device_status(plan: Plan, stream=None) -> int:
    """Synchronise, read and clear the device error word; returns the status code."""
    return int(_lib.attn_check_device_status(plan.handle, _stream(stream)))


def attn_testing_force_timeout(on: bool):
    """Testing hook: attention forward launches take their bounded-wait
    timeout path while on (see include/bsattn.h)."""
    _check(_lib.attn_testing_force_timeout(int(bool(on))), "attn_testing_force_timeout")


def attn_testing_set_error_word(plan: Plan, bits: int):
    """Testing hook: write the plan's device error word."""
    _check(_lib.attn_testing_set_error_word(plan.handle, int(bits)), "attn_testing_set_error_word")


def attn_status_string(code: int) -> str:
    return _lib.attn_status_string(int(code)).decode()


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
