"""ctypes binding of libkvsculpt.so (argument marshalling only).

Every function named ``kvs_*`` calls the C entry point of the same name in
``include/kvsculpt.h``.  Tensors are torch CUDA tensors (row-major, contiguous,
float32 / int32 / int64 as documented there); ``stream`` defaults to torch's
current stream.  A negative return code raises :class:`KvsError`.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import numpy as np
import torch

__all__ = [
    "KvsError", "KvsBatch", "Schedule", "QuerySpec", "LIB_PATH", "lib",
    "ST_NONFINITE", "ST_NOT_PD", "ST_LS_FAIL",
    "kvs_version", "kvs_launch_count", "kvs_set_wait_limit", "kvs_workspace_bytes", "kvs_lbfgs_state_bytes", "kvs_lbfgs_state_layout", "kvs_build_queries",
    "kvs_targets", "kvs_init_topk", "kvs_loss_grad", "kvs_loss_grad_static", "kvs_fit_values", "kvs_lbfgs_reset",
    "kvs_lbfgs_step", "kvs_compress_batch", "kvs_pilot_allocate", "kvs_adam_step",
    "alloc_workspace", "alloc_state",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvsculpt.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python kv_cache_compression_kvsculpt_b200/build.py`")
lib = ctypes.CDLL(LIB_PATH)

ST_NONFINITE, ST_NOT_PD, ST_LS_FAIL = 1, 2, 4
_ERRORS = {-1: "KVS_EINVAL", -2: "KVS_ECUDA", -3: "KVS_ENOTSUP", -4: "KVS_EWORKSPACE"}

_i32, _i64, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class _Batch(ctypes.Structure):
    _fields_ = [("B", _i32), ("d", _i32), ("q_off", _vp), ("z_off", _vp), ("c_off", _vp),
                ("q_off_h", _vp), ("z_off_h", _vp), ("c_off_h", _vp)]


class _Sched(ctypes.Structure):
    _fields_ = [("outer", _i32), ("steps", _i32), ("history", _i32), ("max_bt", _i32),
                ("persist_history", _i32), ("lam", _f32), ("w_out", _f32), ("w_lse", _f32),
                ("c1", _f32), ("backtrack", _f32)]


class _QSpec(ctypes.Structure):
    _fields_ = [("B", _i32), ("d", _i32), ("g", _i32), ("m_q", _i32), ("n_syn", _i32),
                ("N", _i32), ("rope_base", _f32)]


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in ("scalars", "scalar_bytes", "off_f", "off_count",
                                                "off_head", "x", "g", "dir", "ring_s", "ring_y",
                                                "ring_stride")] + [("slots", _i32)]


_BP, _SP, _QP = ctypes.POINTER(_Batch), ctypes.POINTER(_Sched), ctypes.POINTER(_QSpec)
_SIGS = {
    "kvs_version": (ctypes.c_char_p, []),
    "kvs_last_cuda_error": (ctypes.c_char_p, []),
    "kvs_launch_count": (ctypes.c_uint64, []),
    "kvs_set_wait_limit": (ctypes.c_int, [_i64]),
    "kvs_workspace_bytes": (_sz, [_BP, _SP]),
    "kvs_lbfgs_state_bytes": (_sz, [_BP, _i32]),
    "kvs_lbfgs_state_layout": (ctypes.c_int, [_BP, _i32, ctypes.POINTER(_Layout)]),
    "kvs_build_queries": (ctypes.c_int, [_QP, _vp, _vp, _vp, _vp, _vp]),
    "kvs_targets": (ctypes.c_int, [_BP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "kvs_init_topk": (ctypes.c_int, [_BP, _vp, _vp, _vp, _vp, _vp]),
    "kvs_loss_grad": (ctypes.c_int, [_BP, _vp, _vp, _vp, _vp, _vp, _f32, _f32, _vp, _vp, _vp,
                                     _vp, _sz, _vp]),
    "kvs_loss_grad_static": (ctypes.c_int, [_BP, _vp, _vp, _vp, _vp, _vp, _f32, _f32, _vp, _vp,
                                            _vp, _vp]),
    "kvs_fit_values": (ctypes.c_int, [_BP, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _sz, _vp]),
    "kvs_lbfgs_reset": (ctypes.c_int, [_BP, _SP, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i32, _vp,
                                       _sz, _vp]),
    "kvs_lbfgs_step": (ctypes.c_int, [_BP, _SP, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp,
                                      _vp, _sz, _vp]),
    "kvs_compress_batch": (ctypes.c_int, [_BP, _SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _sz, _vp, _sz, _vp]),
    "kvs_pilot_allocate": (ctypes.c_int, [_i32, _vp, _i64, _i32, _vp, _f32, _vp]),
    "kvs_adam_step": (ctypes.c_int, [_BP, _vp, _vp, _vp, _vp, _i32, _f32, _f32, _f32, _f32, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class KvsError(RuntimeError):
    def __init__(self, name, rc):
        msg = f"{name} failed: {_ERRORS.get(rc, rc)}"
        if rc == -2:
            msg += f" ({lib.kvs_last_cuda_error().decode()})"
        super().__init__(msg)
        self.rc = rc


def _check(name, rc):
    if rc != 0:
        raise KvsError(name, rc)


def _ptr(t, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _off(x):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int64))
    return a


class KvsBatch:
    """Offsets of a batch of head-problems (host and device copies)."""

    def __init__(self, d: int, q_off, z_off, c_off=None, device="cuda"):
        self.d = int(d)
        self.q_off_h = _off(q_off)
        self.z_off_h = _off(z_off)
        self.c_off_h = None if c_off is None else _off(c_off)
        self.device = device
        self.q_off = torch.from_numpy(self.q_off_h).to(device)
        self.z_off = torch.from_numpy(self.z_off_h).to(device)
        self.c_off = None if c_off is None else torch.from_numpy(self.c_off_h).to(device)
        self._s = _Batch(len(self.q_off_h) - 1, self.d,
                         self.q_off.data_ptr(), self.z_off.data_ptr(),
                         None if self.c_off is None else self.c_off.data_ptr(),
                         self.q_off_h.ctypes.data, self.z_off_h.ctypes.data,
                         None if self.c_off_h is None else self.c_off_h.ctypes.data)

    @classmethod
    def uniform(cls, B, d, n_q, z, k=None, device="cuda"):
        c = None if k is None else np.arange(B + 1) * k
        return cls(d, np.arange(B + 1) * n_q, np.arange(B + 1) * z, c, device)

    def with_k(self, k):
        """Same queries and zones with compressed sizes k (int or per-problem list)."""
        kk = np.broadcast_to(np.asarray(k, np.int64), (self.B,))
        return KvsBatch(self.d, self.q_off_h, self.z_off_h, np.concatenate([[0], np.cumsum(kk)]),
                        self.device)

    @property
    def B(self):
        return len(self.q_off_h) - 1

    @property
    def sum_q(self):
        return int(self.q_off_h[-1])

    @property
    def sum_z(self):
        return int(self.z_off_h[-1])

    @property
    def sum_c(self):
        return 0 if self.c_off_h is None else int(self.c_off_h[-1])

    @property
    def ref(self):
        return ctypes.byref(self._s)


@dataclasses.dataclass
class Schedule:
    outer: int = 40
    steps: int = 5
    history: int = 10
    max_bt: int = 20
    persist_history: int = 1
    lam: float = 1e-3
    w_out: float = 1.0
    w_lse: float = 1.0
    c1: float = 1e-4
    backtrack: float = 0.5

    def struct(self):
        return _Sched(self.outer, self.steps, self.history, self.max_bt, int(self.persist_history),
                      self.lam, self.w_out, self.w_lse, self.c1, self.backtrack)


@dataclasses.dataclass
class QuerySpec:
    B: int
    d: int
    g: int
    m_q: int
    n_syn: int
    N: int
    rope_base: float = 1e6

    def struct(self):
        return _QSpec(self.B, self.d, self.g, self.m_q, self.n_syn, self.N, self.rope_base)


def kvs_version() -> str:
    return lib.kvs_version().decode()


def kvs_launch_count() -> int:
    return int(lib.kvs_launch_count())


def kvs_set_wait_limit(cycles: int) -> None:
    """Bound on the tensor-core kernels' pipeline waits, in SM cycles (0: the default);
    for tests of the timeout path."""
    _check("kvs_set_wait_limit", lib.kvs_set_wait_limit(int(cycles)))


def kvs_workspace_bytes(batch: KvsBatch, sched: Optional[Schedule] = None) -> int:
    s = None if sched is None else ctypes.byref(sched.struct())
    return int(lib.kvs_workspace_bytes(batch.ref, s))


def kvs_lbfgs_state_bytes(batch: KvsBatch, history: int) -> int:
    return int(lib.kvs_lbfgs_state_bytes(batch.ref, history))


def kvs_lbfgs_state_layout(batch: KvsBatch, history: int) -> dict:
    """Byte offsets of the L-BFGS state fields inside a state buffer (see the header)."""
    out = _Layout()
    _check("kvs_lbfgs_state_layout", lib.kvs_lbfgs_state_layout(batch.ref, int(history),
                                                                ctypes.byref(out)))
    return {n: int(getattr(out, n)) for n, _ in _Layout._fields_}


def alloc_workspace(batch: KvsBatch, sched: Optional[Schedule] = None, device="cuda"):
    n = kvs_workspace_bytes(batch, sched)
    if n == 0:
        raise KvsError("kvs_workspace_bytes", -1)
    return torch.empty(n, dtype=torch.uint8, device=device)


def alloc_state(batch: KvsBatch, history: int, device="cuda"):
    n = kvs_lbfgs_state_bytes(batch, history)
    if n == 0:
        raise KvsError("kvs_lbfgs_state_bytes", -1)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def kvs_build_queries(spec: QuerySpec, q_retain, q_ctx, pos, Q, stream=None):
    s = spec.struct()
    _check("kvs_build_queries", lib.kvs_build_queries(
        ctypes.byref(s), _ptr(q_retain, torch.float32), _ptr(q_ctx, torch.float32),
        _ptr(pos, torch.int32), _ptr(Q, torch.float32), _stream(stream)))


def kvs_targets(batch: KvsBatch, Q, Kz, Vz, Y, lse, importance, ws, stream=None):
    _check("kvs_targets", lib.kvs_targets(
        batch.ref, _ptr(Q, torch.float32), _ptr(Kz, torch.float32), _ptr(Vz, torch.float32),
        _ptr(Y, torch.float32), _ptr(lse, torch.float32), _ptr(importance, torch.float32),
        _ptr(ws), ws.numel(), _stream(stream)))


def kvs_init_topk(batch: KvsBatch, importance, Kz, idx, Kc, stream=None):
    _check("kvs_init_topk", lib.kvs_init_topk(
        batch.ref, _ptr(importance, torch.float32), _ptr(Kz, torch.float32),
        _ptr(idx, torch.int32), _ptr(Kc, torch.float32), _stream(stream)))


def kvs_loss_grad(batch: KvsBatch, Q, Kc, Vc, Y, lse, w_out, w_lse, loss, parts, dKc, ws,
                  stream=None):
    _check("kvs_loss_grad", lib.kvs_loss_grad(
        batch.ref, _ptr(Q, torch.float32), _ptr(Kc, torch.float32), _ptr(Vc, torch.float32),
        _ptr(Y, torch.float32), _ptr(lse, torch.float32), float(w_out), float(w_lse),
        _ptr(loss, torch.float32), _ptr(parts, torch.float32), _ptr(dKc, torch.float32),
        _ptr(ws), ws.numel(), _stream(stream)))


def kvs_loss_grad_static(batch: KvsBatch, Q, Kc, Vc, Y, lse, w_out, w_lse, loss, parts, dKc,
                         stream=None):
    """kvs_loss_grad without a caller workspace, for callers that cannot allocate device
    memory: scratch comes from a 32 MiB array inside the library (see the header)."""
    _check("kvs_loss_grad_static", lib.kvs_loss_grad_static(
        batch.ref, _ptr(Q, torch.float32), _ptr(Kc, torch.float32), _ptr(Vc, torch.float32),
        _ptr(Y, torch.float32), _ptr(lse, torch.float32), float(w_out), float(w_lse),
        _ptr(loss, torch.float32), _ptr(parts, torch.float32), _ptr(dKc, torch.float32),
        _stream(stream)))


def kvs_fit_values(batch: KvsBatch, Q, Kc, Y, lam, Vc, status, ws, stream=None):
    _check("kvs_fit_values", lib.kvs_fit_values(
        batch.ref, _ptr(Q, torch.float32), _ptr(Kc, torch.float32), _ptr(Y, torch.float32),
        float(lam), _ptr(Vc, torch.float32), _ptr(status, torch.int32), _ptr(ws), ws.numel(),
        _stream(stream)))


def kvs_lbfgs_reset(batch: KvsBatch, sched: Schedule, Q, Y, lse, Vc, Kc, state, clear_history,
                    ws, stream=None):
    s = sched.struct()
    _check("kvs_lbfgs_reset", lib.kvs_lbfgs_reset(
        batch.ref, ctypes.byref(s), _ptr(Q, torch.float32), _ptr(Y, torch.float32),
        _ptr(lse, torch.float32), _ptr(Vc, torch.float32), _ptr(Kc, torch.float32), _ptr(state),
        state.numel(), int(clear_history), _ptr(ws), ws.numel(), _stream(stream)))


def kvs_lbfgs_step(batch: KvsBatch, sched: Schedule, Q, Y, lse, Vc, Kc, state, status, f_out, ws,
                   stream=None):
    s = sched.struct()
    _check("kvs_lbfgs_step", lib.kvs_lbfgs_step(
        batch.ref, ctypes.byref(s), _ptr(Q, torch.float32), _ptr(Y, torch.float32),
        _ptr(lse, torch.float32), _ptr(Vc, torch.float32), _ptr(Kc, torch.float32), _ptr(state),
        state.numel(), _ptr(status, torch.int32), _ptr(f_out, torch.float32), _ptr(ws),
        ws.numel(), _stream(stream)))


def kvs_compress_batch(batch: KvsBatch, sched: Schedule, Q, Kz, Vz, Kc, Vc, idx, loss_trace,
                       parts, status, state, ws, stream=None):
    s = sched.struct()
    _check("kvs_compress_batch", lib.kvs_compress_batch(
        batch.ref, ctypes.byref(s), _ptr(Q, torch.float32), _ptr(Kz, torch.float32),
        _ptr(Vz, torch.float32), _ptr(Kc, torch.float32), _ptr(Vc, torch.float32),
        _ptr(idx, torch.int32), _ptr(loss_trace, torch.float32), _ptr(parts, torch.float32),
        _ptr(status, torch.int32), _ptr(state), state.numel(), _ptr(ws), ws.numel(),
        _stream(stream)))


def kvs_adam_step(batch: KvsBatch, Kc, dKc, m, v, t: int, lr: float, beta1: float = 0.9,
                  beta2: float = 0.999, eps: float = 1e-8, stream=None):
    _check("kvs_adam_step", lib.kvs_adam_step(
        batch.ref, _ptr(Kc, torch.float32), _ptr(dKc, torch.float32), _ptr(m, torch.float32),
        _ptr(v, torch.float32), int(t), float(lr), float(beta1), float(beta2), float(eps),
        _stream(stream)))


def kvs_pilot_allocate(pilot_mse, total: int, k_min: int, k_max, alpha: float = 0.5):
    """Host-only allocation; returns an int32 numpy array of per-problem budgets."""
    mse = np.ascontiguousarray(np.asarray(pilot_mse, np.float32))
    B = len(mse)
    kmax = np.ascontiguousarray(np.broadcast_to(np.asarray(k_max, np.int32), (B,)))
    out = np.zeros(B, np.int32)
    _check("kvs_pilot_allocate", lib.kvs_pilot_allocate(
        B, mse.ctypes.data, int(total), int(k_min), kmax.ctypes.data, float(alpha),
        out.ctypes.data))
    return out
