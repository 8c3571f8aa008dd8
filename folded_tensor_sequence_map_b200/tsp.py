"""Thin Python binding of the C ABI in ``include/tsp.h`` (and the test hooks
of ``include/tsp_testing.h``).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity and passed as raw pointers; every step of the layer runs in the
CUDA kernels of ``libtsp.so``.  There is no fallback: if the library is
missing or fails to load, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtsp.so")

TSP_OK = 0
STATUS_NAMES = {
    0: "TSP_OK",
    1: "TSP_ERR_INVALID_ARG",
    2: "TSP_ERR_INDIVISIBLE",
    3: "TSP_ERR_UNSUPPORTED",
    4: "TSP_ERR_ALIGNMENT",
    5: "TSP_ERR_CUDA",
    6: "TSP_ERR_TIMEOUT",
    7: "TSP_ERR_RANGE",
}

EXPORTED = (
    "tsp_plan",
    "tsp_plan_destroy",
    "tsp_zigzag_map",
    "tsp_shard_schedule",
    "tsp_workspace_size",
    "tsp_layer_forward",
    "tsp_layer_prefill",
    "tsp_ring_mlp_workspace_size",
    "tsp_ring_mlp_forward",
    "tsp_layer_backward",
    "tsp_stack_workspace_size",
    "tsp_stack_forward",
    "tsp_stack_backward",
    "tsp_rank_workspace_size",
    "tsp_rank_forward_qkv",
    "tsp_rank_forward_out",
    "tsp_rank_backward_workspace_size",
    "tsp_rank_backward_attn",
    "tsp_rank_backward_qkv",
    "tsp_sync_status",
    "tsp_status_string",
    "tsp_layer_flops",
    "tsp_profile_enable",
    "tsp_profile_read",
    "tsp_kernel_launches",
    "tsp_rmsnorm_backward_noalloc",
    "tsp_test_gemm",
    "tsp_test_buffer_offset",
    "tsp_test_next_visible",
    "tsp_test_step_walk",
    "tsp_test_step_walk_desc",
    "tsp_test_step_walk_rank",
    "tsp_test_rank_kv_order",
    "tsp_test_tables",
    "tsp_test_work_order",
    "tsp_test_wait_timeout",
    "tsp_test_exp2",
)
TSP_NUM_STAGES = 25


class TSPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtsp.so is not built ({LIB_PATH}); run python -m folded_tensor_sequence_map_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ, V = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
    lib.tsp_plan.argtypes = [I, I, I, I64, I, ctypes.POINTER(P)]
    lib.tsp_plan.restype = I
    lib.tsp_plan_destroy.argtypes = [P]
    lib.tsp_plan_destroy.restype = None
    lib.tsp_zigzag_map.argtypes = [P, P]
    lib.tsp_zigzag_map.restype = I
    lib.tsp_shard_schedule.argtypes = [P, I, P]
    lib.tsp_shard_schedule.restype = I
    lib.tsp_workspace_size.argtypes = [P, I, ctypes.POINTER(SZ), ctypes.POINTER(SZ)]
    lib.tsp_workspace_size.restype = I
    lib.tsp_layer_forward.argtypes = [P] + [V] * 11
    lib.tsp_layer_forward.restype = I
    lib.tsp_layer_prefill.argtypes = [P] + [V] * 12
    lib.tsp_layer_prefill.restype = I
    lib.tsp_ring_mlp_workspace_size.argtypes = [P, ctypes.POINTER(SZ)]
    lib.tsp_ring_mlp_workspace_size.restype = I
    lib.tsp_ring_mlp_forward.argtypes = [P] + [V] * 7
    lib.tsp_ring_mlp_forward.restype = I
    lib.tsp_layer_backward.argtypes = [P] + [V] * 18
    lib.tsp_layer_backward.restype = I
    lib.tsp_stack_workspace_size.argtypes = [P, I, ctypes.POINTER(SZ), ctypes.POINTER(SZ), ctypes.POINTER(SZ)]
    lib.tsp_stack_workspace_size.restype = I
    lib.tsp_stack_forward.argtypes = [P, I] + [V] * 12
    lib.tsp_stack_forward.restype = I
    lib.tsp_stack_backward.argtypes = [P, I] + [V] * 19
    lib.tsp_stack_backward.restype = I
    lib.tsp_rank_workspace_size.argtypes = [P, ctypes.POINTER(SZ)]
    lib.tsp_rank_workspace_size.restype = I
    lib.tsp_rank_forward_qkv.argtypes = [P, I] + [V] * 7
    lib.tsp_rank_forward_qkv.restype = I
    lib.tsp_rank_forward_out.argtypes = [P, I] + [V] * 10
    lib.tsp_rank_forward_out.restype = I
    lib.tsp_rank_backward_workspace_size.argtypes = [P, ctypes.POINTER(SZ)]
    lib.tsp_rank_backward_workspace_size.restype = I
    lib.tsp_rank_backward_attn.argtypes = [P, I] + [V] * 13
    lib.tsp_rank_backward_attn.restype = I
    lib.tsp_rank_backward_qkv.argtypes = [P, I] + [V] * 10
    lib.tsp_rank_backward_qkv.restype = I
    lib.tsp_sync_status.argtypes = [P, V]
    lib.tsp_sync_status.restype = I
    lib.tsp_status_string.argtypes = [I]
    lib.tsp_status_string.restype = ctypes.c_char_p
    lib.tsp_layer_flops.argtypes = [P, I]
    lib.tsp_layer_flops.restype = ctypes.c_double
    lib.tsp_test_gemm.argtypes = [I, I, I, I, I, V, I64, V, I64, V, I64, I, I, V]
    lib.tsp_test_gemm.restype = I
    lib.tsp_test_buffer_offset.argtypes = [P, ctypes.c_char_p, ctypes.POINTER(SZ)]
    lib.tsp_test_buffer_offset.restype = I
    lib.tsp_test_next_visible.argtypes = [P, I, I, ctypes.POINTER(I)]
    lib.tsp_test_next_visible.restype = I
    lib.tsp_test_step_walk.argtypes = [P, I, ctypes.POINTER(ctypes.c_int32), I, ctypes.POINTER(I)]
    lib.tsp_test_step_walk.restype = I
    lib.tsp_test_step_walk_desc.argtypes = [P, I, ctypes.POINTER(ctypes.c_int32), I, ctypes.POINTER(I)]
    lib.tsp_test_step_walk_desc.restype = I
    lib.tsp_test_step_walk_rank.argtypes = [P, I, I, ctypes.POINTER(ctypes.c_int32), I, ctypes.POINTER(I)]
    lib.tsp_test_step_walk_rank.restype = I
    lib.tsp_test_rank_kv_order.argtypes = [P, I, I, ctypes.POINTER(ctypes.c_int32), I64, ctypes.POINTER(I64)]
    lib.tsp_test_rank_kv_order.restype = I
    lib.tsp_test_tables.argtypes = [P, I, ctypes.POINTER(ctypes.c_int32), I64, ctypes.POINTER(I64)]
    lib.tsp_test_tables.restype = I
    lib.tsp_test_work_order.argtypes = [P, I, I, ctypes.POINTER(ctypes.c_int32), I64, ctypes.POINTER(I64)]
    lib.tsp_test_work_order.restype = I
    lib.tsp_profile_enable.argtypes = [P, I]
    lib.tsp_profile_enable.restype = I
    lib.tsp_profile_read.argtypes = [P, I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(I64), ctypes.POINTER(I64)]
    lib.tsp_profile_read.restype = I
    lib.tsp_kernel_launches.argtypes = [P]
    lib.tsp_kernel_launches.restype = I64
    lib.tsp_rmsnorm_backward_noalloc.argtypes = [V, V, V, V, V, V, V, I, I, V]
    lib.tsp_rmsnorm_backward_noalloc.restype = I
    lib.tsp_test_wait_timeout.argtypes = [P, ctypes.c_longlong, V, V]
    lib.tsp_test_wait_timeout.restype = I
    lib.tsp_test_exp2.argtypes = [V, V, I, I, V]
    lib.tsp_test_exp2.restype = I
    return lib


_lib = _load()


def _check(status: int, where: str) -> None:
    if status != TSP_OK:
        raise TSPError(status, where)


class Plan:
    """Owner of a ``tsp_plan_t``; freed with the object."""

    def __init__(self, handle: int, h: int, heads: int, ffn: int, S: int, D: int):
        self.handle = ctypes.c_void_p(handle)
        self.h, self.heads, self.ffn, self.S, self.D = h, heads, ffn, S, D

    def __del__(self):
        lib = globals().get("_lib")
        if lib is not None and getattr(self, "handle", None) is not None and self.handle.value:
            lib.tsp_plan_destroy(self.handle)
            self.handle = None


def _ptr(t, name, dtype=None, shape=None):
    """Device pointer of a contiguous CUDA tensor (or a raw int address)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor or an address")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def tsp_plan(h: int, heads: int, ffn: int, S: int, D: int) -> Plan:
    out = ctypes.c_void_p()
    _check(_lib.tsp_plan(h, heads, ffn, S, D, ctypes.byref(out)), "tsp_plan")
    return Plan(out.value, h, heads, ffn, S, D)


def tsp_zigzag_map(plan: Plan) -> np.ndarray:
    m = np.empty(plan.S, dtype=np.int32)
    _check(_lib.tsp_zigzag_map(plan.handle, m.ctypes.data), "tsp_zigzag_map")
    return m


def tsp_shard_schedule(plan: Plan, phase: int) -> np.ndarray:
    s = np.empty((plan.D, plan.D), dtype=np.int32)
    _check(_lib.tsp_shard_schedule(plan.handle, phase, s.ctypes.data), "tsp_shard_schedule")
    return s


def tsp_workspace_size(plan: Plan, training: bool):
    ws, saved = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.tsp_workspace_size(plan.handle, int(bool(training)), ctypes.byref(ws), ctypes.byref(saved)),
           "tsp_workspace_size")
    return ws.value, saved.value


def tsp_layer_flops(plan: Plan, backward: bool) -> float:
    return _lib.tsp_layer_flops(plan.handle, int(bool(backward)))


def tsp_status_string(status: int) -> str:
    return _lib.tsp_status_string(status).decode()


def tsp_layer_forward(plan: Plan, x, g1, wqkv, wo, g2, w1, w2, y, saved, ws, stream=None) -> None:
    import torch

    h, F, S = plan.h, plan.ffn, plan.S
    bf, f32, u8 = torch.bfloat16, torch.float32, None
    args = [
        _ptr(x, "x", bf, (S, h)),
        _ptr(g1, "g1", f32, (h,)),
        _ptr(wqkv, "wqkv", bf, (3 * h, h)),
        _ptr(wo, "wo", bf, (h, h)),
        _ptr(g2, "g2", f32, (h,)),
        _ptr(w1, "w1", bf, (F, h)),
        _ptr(w2, "w2", bf, (h, F)),
        _ptr(y, "y", bf, (S, h)),
        _ptr(saved, "saved", u8),
        _ptr(ws, "ws", u8),
        _stream(stream),
    ]
    _check(_lib.tsp_layer_forward(plan.handle, *args), "tsp_layer_forward")


def tsp_layer_prefill(plan: Plan, x, g1, wqkv, wo, g2, w1, w2, y, k_cache, v_cache, ws, stream=None) -> None:
    import torch

    h, F, S = plan.h, plan.ffn, plan.S
    bf, f32 = torch.bfloat16, torch.float32
    args = [
        _ptr(x, "x", bf, (S, h)),
        _ptr(g1, "g1", f32, (h,)),
        _ptr(wqkv, "wqkv", bf, (3 * h, h)),
        _ptr(wo, "wo", bf, (h, h)),
        _ptr(g2, "g2", f32, (h,)),
        _ptr(w1, "w1", bf, (F, h)),
        _ptr(w2, "w2", bf, (h, F)),
        _ptr(y, "y", bf, (S, h)),
        _ptr(k_cache, "k_cache", torch.float16, (S, h)),
        _ptr(v_cache, "v_cache", torch.float16, (S, h)),
        _ptr(ws, "ws"),
        _stream(stream),
    ]
    _check(_lib.tsp_layer_prefill(plan.handle, *args), "tsp_layer_prefill")


def tsp_ring_mlp_workspace_size(plan: Plan) -> int:
    n = ctypes.c_size_t()
    _check(_lib.tsp_ring_mlp_workspace_size(plan.handle, ctypes.byref(n)), "tsp_ring_mlp_workspace_size")
    return n.value


def tsp_ring_mlp_forward(plan: Plan, b, w1, w2, resid, out, ws, stream=None) -> None:
    import torch

    h, F, S = plan.h, plan.ffn, plan.S
    bf, f32 = torch.bfloat16, torch.float32
    args = [
        _ptr(b, "b", bf, (S, h)),
        _ptr(w1, "w1", bf, (F, h)),
        _ptr(w2, "w2", bf, (h, F)),
        _ptr(resid, "resid", f32, (S, h)),
        _ptr(out, "out", bf, (S, h)),
        _ptr(ws, "ws"),
        _stream(stream),
    ]
    _check(_lib.tsp_ring_mlp_forward(plan.handle, *args), "tsp_ring_mlp_forward")


def tsp_layer_backward(plan: Plan, dy, x, g1, wqkv, wo, g2, w1, w2, saved, ws, dx, dg1, dwqkv, dwo, dg2, dw1, dw2,
                       stream=None) -> None:
    import torch

    h, F, S = plan.h, plan.ffn, plan.S
    bf, f32 = torch.bfloat16, torch.float32
    args = [
        _ptr(dy, "dy", bf, (S, h)),
        _ptr(x, "x", bf, (S, h)),
        _ptr(g1, "g1", f32, (h,)),
        _ptr(wqkv, "wqkv", bf, (3 * h, h)),
        _ptr(wo, "wo", bf, (h, h)),
        _ptr(g2, "g2", f32, (h,)),
        _ptr(w1, "w1", bf, (F, h)),
        _ptr(w2, "w2", bf, (h, F)),
        _ptr(saved, "saved"),
        _ptr(ws, "ws"),
        _ptr(dx, "dx", bf, (S, h)),
        _ptr(dg1, "dg1", f32, (h,)),
        _ptr(dwqkv, "dwqkv", f32, (3 * h, h)),
        _ptr(dwo, "dwo", f32, (h, h)),
        _ptr(dg2, "dg2", f32, (h,)),
        _ptr(dw1, "dw1", f32, (F, h)),
        _ptr(dw2, "dw2", f32, (h, F)),
        _stream(stream),
    ]
    _check(_lib.tsp_layer_backward(plan.handle, *args), "tsp_layer_backward")


def tsp_stack_workspace_size(plan: Plan, layers: int):
    ws, saved, inputs = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.tsp_stack_workspace_size(plan.handle, layers, ctypes.byref(ws), ctypes.byref(saved),
                                         ctypes.byref(inputs)), "tsp_stack_workspace_size")
    return ws.value, saved.value, inputs.value


def _ptr_array(ts, name, dtype, shape):
    """Host array of device pointers, one per layer (kept alive by the caller
    of the C function through the returned object)."""
    arr = (ctypes.c_void_p * len(ts))(*[_ptr(t, f"{name}[{i}]", dtype, shape) for i, t in enumerate(ts)])
    return arr


def tsp_stack_forward(plan: Plan, x, g1, wqkv, wo, g2, w1, w2, z, inputs, saved, ws, stream=None) -> None:
    """g1, wqkv, wo, g2, w1, w2: sequences with one tensor per layer."""
    import torch

    h, F, S, n = plan.h, plan.ffn, plan.S, len(wqkv)
    bf, f32 = torch.bfloat16, torch.float32
    arrs = [_ptr_array(g1, "g1", f32, (h,)), _ptr_array(wqkv, "wqkv", bf, (3 * h, h)),
            _ptr_array(wo, "wo", bf, (h, h)), _ptr_array(g2, "g2", f32, (h,)),
            _ptr_array(w1, "w1", bf, (F, h)), _ptr_array(w2, "w2", bf, (h, F))]
    if any(len(a) != n for a in arrs):
        raise ValueError("one tensor per layer in every weight list")
    _check(_lib.tsp_stack_forward(plan.handle, n, _ptr(x, "x", bf, (S, h)), *[ctypes.cast(a, ctypes.c_void_p) for a in arrs],
                                  _ptr(z, "z", bf, (S, h)), _ptr(inputs, "inputs"), _ptr(saved, "saved"),
                                  _ptr(ws, "ws"), _stream(stream)), "tsp_stack_forward")


def tsp_stack_backward(plan: Plan, dz, x, g1, wqkv, wo, g2, w1, w2, inputs, saved, ws, dx, dg1, dwqkv, dwo, dg2,
                       dw1, dw2, stream=None) -> None:
    """Weight and gradient arguments: sequences with one tensor per layer."""
    import torch

    h, F, S, n = plan.h, plan.ffn, plan.S, len(wqkv)
    bf, f32 = torch.bfloat16, torch.float32
    arrs = [_ptr_array(g1, "g1", f32, (h,)), _ptr_array(wqkv, "wqkv", bf, (3 * h, h)),
            _ptr_array(wo, "wo", bf, (h, h)), _ptr_array(g2, "g2", f32, (h,)),
            _ptr_array(w1, "w1", bf, (F, h)), _ptr_array(w2, "w2", bf, (h, F))]
    grads = [_ptr_array(dg1, "dg1", f32, (h,)), _ptr_array(dwqkv, "dwqkv", f32, (3 * h, h)),
             _ptr_array(dwo, "dwo", f32, (h, h)), _ptr_array(dg2, "dg2", f32, (h,)),
             _ptr_array(dw1, "dw1", f32, (F, h)), _ptr_array(dw2, "dw2", f32, (h, F))]
    if any(len(a) != n for a in arrs + grads):
        raise ValueError("one tensor per layer in every weight and gradient list")
    _check(_lib.tsp_stack_backward(plan.handle, n, _ptr(dz, "dz", bf, (S, h)), _ptr(x, "x", bf, (S, h)),
                                   *[ctypes.cast(a, ctypes.c_void_p) for a in arrs], _ptr(inputs, "inputs"), _ptr(saved, "saved"),
                                   _ptr(ws, "ws"), _ptr(dx, "dx", bf, (S, h)), *[ctypes.cast(a, ctypes.c_void_p) for a in grads],
                                   _stream(stream)), "tsp_stack_backward")


def tsp_rank_workspace_size(plan: Plan) -> int:
    ws = ctypes.c_size_t()
    _check(_lib.tsp_rank_workspace_size(plan.handle, ctypes.byref(ws)), "tsp_rank_workspace_size")
    return ws.value


def tsp_rank_forward_qkv(plan: Plan, rank: int, x, g1, wqkv, k, v, ws, stream=None) -> None:
    import torch

    h, S, L = plan.h, plan.S, plan.S // plan.D
    bf, f32, f16 = torch.bfloat16, torch.float32, torch.float16
    _check(_lib.tsp_rank_forward_qkv(plan.handle, rank, _ptr(x, "x", bf, (L, h)), _ptr(g1, "g1", f32, (h,)),
                                     _ptr(wqkv, "wqkv", bf, (3 * h, h)), _ptr(k, "k", f16, (S, h)),
                                     _ptr(v, "v", f16, (S, h)), _ptr(ws, "ws"), _stream(stream)),
           "tsp_rank_forward_qkv")


def tsp_rank_forward_out(plan: Plan, rank: int, x, k, v, wo, g2, w1, w2, z, ws, stream=None) -> None:
    import torch

    h, F, S, L = plan.h, plan.ffn, plan.S, plan.S // plan.D
    bf, f32, f16 = torch.bfloat16, torch.float32, torch.float16
    _check(_lib.tsp_rank_forward_out(plan.handle, rank, _ptr(x, "x", bf, (L, h)), _ptr(k, "k", f16, (S, h)),
                                     _ptr(v, "v", f16, (S, h)), _ptr(wo, "wo", bf, (h, h)), _ptr(g2, "g2", f32, (h,)),
                                     _ptr(w1, "w1", bf, (F, h)), _ptr(w2, "w2", bf, (h, F)),
                                     _ptr(z, "z", bf, (L, h)), _ptr(ws, "ws"), _stream(stream)),
           "tsp_rank_forward_out")


def tsp_rank_backward_workspace_size(plan: Plan) -> int:
    bws = ctypes.c_size_t()
    _check(_lib.tsp_rank_backward_workspace_size(plan.handle, ctypes.byref(bws)), "tsp_rank_backward_workspace_size")
    return bws.value


def tsp_rank_backward_attn(plan: Plan, rank: int, dz, k, v, g2, ws, bws, dk_part, dv_part, dwo, dg2, dw1, dw2,
                           stream=None) -> None:
    import torch

    h, F, S, L = plan.h, plan.ffn, plan.S, plan.S // plan.D
    bf, f32, f16 = torch.bfloat16, torch.float32, torch.float16
    _check(_lib.tsp_rank_backward_attn(plan.handle, rank, _ptr(dz, "dz", bf, (L, h)), _ptr(k, "k", f16, (S, h)),
                                       _ptr(v, "v", f16, (S, h)), _ptr(g2, "g2", f32, (h,)), _ptr(ws, "ws"),
                                       _ptr(bws, "bws"), _ptr(dk_part, "dk_part", f32, (S, h)),
                                       _ptr(dv_part, "dv_part", f32, (S, h)), _ptr(dwo, "dwo", f32, (h, h)),
                                       _ptr(dg2, "dg2", f32, (h,)), _ptr(dw1, "dw1", f32, (F, h)),
                                       _ptr(dw2, "dw2", f32, (h, F)), _stream(stream)),
           "tsp_rank_backward_attn")


def tsp_rank_backward_qkv(plan: Plan, rank: int, x, g1, dk, dv, ws, bws, dx, dg1, dwqkv, stream=None) -> None:
    import torch

    h, L = plan.h, plan.S // plan.D
    bf, f32 = torch.bfloat16, torch.float32
    _check(_lib.tsp_rank_backward_qkv(plan.handle, rank, _ptr(x, "x", bf, (L, h)), _ptr(g1, "g1", f32, (h,)),
                                      _ptr(dk, "dk", f32, (L, h)), _ptr(dv, "dv", f32, (L, h)), _ptr(ws, "ws"),
                                      _ptr(bws, "bws"), _ptr(dx, "dx", bf, (L, h)), _ptr(dg1, "dg1", f32, (h,)),
                                      _ptr(dwqkv, "dwqkv", f32, (3 * h, h)), _stream(stream)),
           "tsp_rank_backward_qkv")


def tsp_sync_status(plan: Plan, stream=None) -> None:
    _check(_lib.tsp_sync_status(plan.handle, _stream(stream)), "tsp_sync_status")


def tsp_profile_enable(plan: Plan, enable: bool) -> None:
    _check(_lib.tsp_profile_enable(plan.handle, int(bool(enable))), "tsp_profile_enable")


def tsp_profile_read(plan: Plan, stage: int):
    """(name, total_ms, calls, kernel_launches) of one stage."""
    name = ctypes.c_char_p()
    ms = ctypes.c_double()
    calls, launches = ctypes.c_int64(), ctypes.c_int64()
    _check(_lib.tsp_profile_read(plan.handle, stage, ctypes.byref(name), ctypes.byref(ms), ctypes.byref(calls),
                                 ctypes.byref(launches)), "tsp_profile_read")
    return name.value.decode(), ms.value, calls.value, launches.value


def tsp_kernel_launches(plan: Plan) -> int:
    return _lib.tsp_kernel_launches(plan.handle)


def tsp_rmsnorm_backward_noalloc(dout, x, rstd, g, resid, dx, dg, rows: int, h: int, stream=None) -> None:
    """RMSNorm backward + residual with library-owned scratch (no allocation);
    see include/tsp.h for the contract."""
    import torch

    f32, bf = torch.float32, torch.bfloat16
    _check(_lib.tsp_rmsnorm_backward_noalloc(
        _ptr(dout, "dout", f32, (rows, h)), _ptr(x, "x", bf, (rows, h)), _ptr(rstd, "rstd", f32, (rows,)),
        _ptr(g, "g", f32, (h,)), _ptr(resid, "resid", f32, (rows, h)), _ptr(dx, "dx", bf, (rows, h)),
        _ptr(dg, "dg", f32, (h,)), rows, h, _stream(stream)), "tsp_rmsnorm_backward_noalloc")


# ---- test hooks --------------------------------------------------------------

def tsp_test_gemm(a_mn: bool, b_mn: bool, M: int, N: int, K: int, A, lda: int, B, ldb: int, C, ldc: int,
                  force_bn128: bool = False, stream=None, f16: bool = False) -> None:
    _check(_lib.tsp_test_gemm(int(a_mn), int(b_mn), M, N, K, _ptr(A, "A"), lda, _ptr(B, "B"), ldb, _ptr(C, "C"),
                              ldc, int(force_bn128), int(bool(f16)), _stream(stream)), "tsp_test_gemm")


def tsp_test_buffer_offset(plan: Plan, name: str) -> int:
    off = ctypes.c_size_t()
    _check(_lib.tsp_test_buffer_offset(plan.handle, name.encode(), ctypes.byref(off)), "tsp_test_buffer_offset")
    return off.value


def tsp_test_next_visible(plan: Plan, start: int, kv0: int) -> int:
    out = ctypes.c_int()
    _check(_lib.tsp_test_next_visible(plan.handle, start, kv0, ctypes.byref(out)), "tsp_test_next_visible")
    return out.value


def tsp_test_step_walk(plan: Plan, kv0: int, descending: bool = False) -> np.ndarray:
    cap = plan.S // 64
    out = np.zeros(cap, dtype=np.int32)
    n = ctypes.c_int()
    fn = _lib.tsp_test_step_walk_desc if descending else _lib.tsp_test_step_walk
    name = "tsp_test_step_walk_desc" if descending else "tsp_test_step_walk"
    _check(fn(plan.handle, kv0, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cap, ctypes.byref(n)), name)
    return out[:n.value].copy()


def tsp_test_step_walk_rank(plan: Plan, rank: int, kv0: int) -> np.ndarray:
    cap = plan.S // 64
    out = np.zeros(cap, dtype=np.int32)
    n = ctypes.c_int()
    _check(_lib.tsp_test_step_walk_rank(plan.handle, rank, kv0, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                        cap, ctypes.byref(n)), "tsp_test_step_walk_rank")
    return out[:n.value].copy()


def tsp_test_rank_kv_order(plan: Plan, rank: int, num_ctas: int) -> np.ndarray:
    n = ctypes.c_int64()
    _lib.tsp_test_rank_kv_order(plan.handle, rank, num_ctas, None, 0, ctypes.byref(n))  # length query
    out = np.zeros(n.value, dtype=np.int32)
    _check(_lib.tsp_test_rank_kv_order(plan.handle, rank, num_ctas, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                       n.value, ctypes.byref(n)), "tsp_test_rank_kv_order")
    return out


TABLES = {"inv": 0, "qtile_maxpos": 1, "fwd_order": 2, "kv_order": 3, "q_order": 4}


def tsp_test_tables(plan: Plan, name: str) -> np.ndarray:
    n = ctypes.c_int64()
    which = TABLES[name]
    _lib.tsp_test_tables(plan.handle, which, None, 0, ctypes.byref(n))
    out = np.zeros(n.value, dtype=np.int32)
    _check(_lib.tsp_test_tables(plan.handle, which, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n.value,
                                ctypes.byref(n)), "tsp_test_tables")
    return out


def tsp_test_work_order(plan: Plan, name: str, num_ctas: int) -> np.ndarray:
    n = ctypes.c_int64()
    which = TABLES[name]
    _lib.tsp_test_work_order(plan.handle, which, num_ctas, None, 0, ctypes.byref(n))
    out = np.zeros(n.value, dtype=np.int32)
    _check(_lib.tsp_test_work_order(plan.handle, which, num_ctas, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                    n.value, ctypes.byref(n)), "tsp_test_work_order")
    return out


def tsp_test_wait_timeout(plan: Plan, limit_cycles: int, result, stream=None) -> None:
    _check(_lib.tsp_test_wait_timeout(plan.handle, limit_cycles, _ptr(result, "result"), _stream(stream)),
           "tsp_test_wait_timeout")



def tsp_test_exp2(x, y, which: int, stream=None) -> None:
    """y = 2^x (fp32 device tensors of the same length): which 0 the
    attention forward's polynomial, 1 the hardware approximation."""
    import torch

    n = x.numel()
    _check(_lib.tsp_test_exp2(_ptr(x, "x", torch.float32, (n,)), _ptr(y, "y", torch.float32, (n,)), n, which,
                              _stream(stream)), "tsp_test_exp2")
