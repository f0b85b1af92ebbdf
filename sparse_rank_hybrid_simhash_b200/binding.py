"""ctypes binding of libelsaa (include/elsaa.h).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  Torch supplies device memory and the current stream.  There is
no fallback: if ``libelsaa.so`` is missing or was built without the kernels,
every entry point raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libelsaa.so")

ELSAA_BF16, ELSAA_F32 = 0, 1
# elsaa_sort_order: the Sort-LSH chunk order
SORT_ORDERS = {"binary": 0, "gray": 1, "local": 2}
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported problem", 3: "workspace too small",
          4: "CUDA error", 5: "device wait timed out", 6: "device index check failed"}


class ElsaaError(RuntimeError):
    def __init__(self, where: str, code: int):
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")
        self.code = code


class Params(ctypes.Structure):
    """Mirror of ``elsaa_params``."""
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32), ("sort_bits", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("race_tables", ctypes.c_int32),
                ("race_bits", ctypes.c_int32), ("scale", ctypes.c_float),
                ("gate_fixed", ctypes.c_int32), ("gate_s", ctypes.c_float),
                ("gate_r", ctypes.c_float), ("sort_order", ctypes.c_int32),
                ("lookback", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("hash_rounds", ctypes.c_int32)]

    @classmethod
    def make(cls, B, H, N, d, dtype, sort_bits, chunk, race_tables, race_bits, scale=0.0,
             gate_fixed=False, gate_s=0.5, gate_r=0.5, sort_order="binary",
             lookback=1, causal=False, hash_rounds=1) -> "Params":
        dt = ELSAA_BF16 if dtype in ("bf16", torch.bfloat16) else ELSAA_F32
        return cls(B, H, N, d, dt, sort_bits, chunk, race_tables, race_bits, float(scale),
                   int(bool(gate_fixed)), float(gate_s), float(gate_r), SORT_ORDERS[sort_order],
                   int(lookback), int(bool(causal)), int(hash_rounds))

    @classmethod
    def from_workload(cls, w) -> "Params":
        return cls.make(w.B, w.H, w.N, w.d, w.dtype, w.sort_bits, w.chunk, w.race_tables,
                        w.race_bits, 0.0, w.gate_fixed, w.gate_s, w.gate_r, w.sort_order,
                        w.lookback, w.causal, w.hash_rounds)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == ELSAA_BF16 else torch.float32


class Views(ctypes.Structure):
    """Mirror of ``elsaa_views``."""
    _fields_ = [("code_q", ctypes.c_void_p), ("code_k", ctypes.c_void_p),
                ("perm_q", ctypes.c_void_p), ("perm_k", ctypes.c_void_p),
                ("rcode_q", ctypes.c_void_p), ("rcode_k", ctypes.c_void_p),
                ("rcode_bytes", ctypes.c_int32), ("race_count", ctypes.c_void_p),
                ("race_sum", ctypes.c_void_p), ("lse_sp", ctypes.c_void_p),
                ("o_sp", ctypes.c_void_p), ("o_race", ctypes.c_void_p),
                ("ctot", ctypes.c_void_p), ("round_code", ctypes.c_void_p),
                ("round_perm", ctypes.c_void_p), ("hash_rounds", ctypes.c_int32)]


EXPORTS = ("elsaa_validate", "elsaa_workspace_bytes", "elsaa_saved_bytes", "elsaa_forward",
           "elsaa_backward", "elsaa_forward_staged", "elsaa_backward_staged",
           "elsaa_kernel_launches", "elsaa_saved_views", "elsaa_check", "elsaa_status_str",
           "elsaa_uses_tensor_cores", "elsaa_sort_codes_noalloc", "elsaa_path_flags",
           "elsaa_sort_codes_of", "elsaa_sort_codes", "elsaa_race_tables", "elsaa_forward_tables",
           "elsaa_backward_tables", "elsaa_race_value_grad")
# elsaa_path_flags bits
PATH_FLAGS = {"tc_hash": 1, "tc_attn": 2, "slab_fwd": 4, "slab_bwd": 8, "tc_win": 16}
FWD_STAGES = ("hash", "sort", "race_build", "sparse_fwd", "race_fuse")
BWD_STAGES = ("fuse_bwd", "race_bwd", "sparse_bwd", "finish")

_lib = None


def lib() -> ctypes.CDLL:
    """Load libelsaa.so (built in-tree by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libelsaa.so not built ({LIB_PATH}); run "
                           "`python -m sparse_rank_hybrid_simhash_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    L.elsaa_validate.argtypes, L.elsaa_validate.restype = [P], st
    L.elsaa_workspace_bytes.argtypes, L.elsaa_workspace_bytes.restype = [P], sz
    L.elsaa_saved_bytes.argtypes, L.elsaa_saved_bytes.restype = [P], sz
    L.elsaa_uses_tensor_cores.argtypes, L.elsaa_uses_tensor_cores.restype = [P], ctypes.c_int32
    L.elsaa_path_flags.argtypes, L.elsaa_path_flags.restype = [P], ctypes.c_int32
    L.elsaa_sort_codes_of.argtypes = [P] + [vp] * 6 + [sz, vp]
    L.elsaa_sort_codes_of.restype = st
    L.elsaa_sort_codes.argtypes = [P] + [vp] * 3 + [sz, vp]
    L.elsaa_sort_codes.restype = st
    L.elsaa_race_tables.argtypes = [P] + [vp] * 6 + [sz, vp]
    L.elsaa_race_tables.restype = st
    L.elsaa_forward_tables.argtypes = [P] + [vp] * 13 + [sz, vp]
    L.elsaa_forward_tables.restype = st
    L.elsaa_backward_tables.argtypes = [P] + [vp] * 18 + [sz, vp]
    L.elsaa_backward_tables.restype = st
    L.elsaa_race_value_grad.argtypes = [P] + [vp] * 5 + [sz, vp]
    L.elsaa_race_value_grad.restype = st
    L.elsaa_forward.argtypes = [P] + [vp] * 10 + [vp, sz, vp]
    L.elsaa_forward.restype = st
    L.elsaa_backward.argtypes = [P] + [vp] * 17 + [sz, vp]
    L.elsaa_backward.restype = st
    L.elsaa_forward_staged.argtypes = [P] + [vp] * 10 + [vp, sz, vp, vp]
    L.elsaa_forward_staged.restype = st
    L.elsaa_backward_staged.argtypes = [P] + [vp] * 17 + [sz, vp, vp]
    L.elsaa_backward_staged.restype = st
    L.elsaa_kernel_launches.argtypes = [P, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int32)]
    L.elsaa_kernel_launches.restype = st
    L.elsaa_sort_codes_noalloc.argtypes = [P, vp, vp, vp]
    L.elsaa_sort_codes_noalloc.restype = st
    L.elsaa_saved_views.argtypes = [P, vp, ctypes.POINTER(Views)]
    L.elsaa_saved_views.restype = st
    L.elsaa_check.argtypes, L.elsaa_check.restype = [vp, vp], st
    L.elsaa_status_str.argtypes, L.elsaa_status_str.restype = [st], ctypes.c_char_p
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ok(where: str, code: int):
    if code != 0:
        raise ElsaaError(where, code)


def validate(p: Params) -> int:
    return lib().elsaa_validate(ctypes.byref(p))


def workspace_bytes(p: Params) -> int:
    return lib().elsaa_workspace_bytes(ctypes.byref(p))


def saved_bytes(p: Params) -> int:
    return lib().elsaa_saved_bytes(ctypes.byref(p))


def uses_tensor_cores(p: Params) -> bool:
    return bool(lib().elsaa_uses_tensor_cores(ctypes.byref(p)))


def path_flags(p: Params) -> Dict[str, bool]:
    """Which kernel families the operator takes for ``p`` (elsaa_path_flags)."""
    f = lib().elsaa_path_flags(ctypes.byref(p))
    return {name: bool(f & bit) for name, bit in PATH_FLAGS.items()}


def kernel_launches(p: Params):
    """(kernels per forward, kernels per backward) for ``p``."""
    f, b = ctypes.c_int32(), ctypes.c_int32()
    _ok("elsaa_kernel_launches", lib().elsaa_kernel_launches(ctypes.byref(p), ctypes.byref(f),
                                                            ctypes.byref(b)))
    return f.value, b.value


def _events(events):
    """ctypes array of cudaEvent_t handles from torch.cuda.Event objects (or None)."""
    if events is None:
        return None
    handles = []
    for e in events:
        if e is None:
            handles.append(None)
            continue
        if e.cuda_event == 0:      # torch creates the event on first record
            e.record()
        handles.append(e.cuda_event)
    return (ctypes.c_void_p * len(handles))(*handles)


def alloc_workspace(p: Params, device) -> torch.Tensor:
    return torch.empty(max(workspace_bytes(p), 256), dtype=torch.uint8, device=device)


def alloc_saved(p: Params, device) -> torch.Tensor:
    return torch.empty(saved_bytes(p), dtype=torch.uint8, device=device)


def forward(p: Params, q, k, v, r_sort, r_race, gate_w, gate_b, lam, y=None, saved=None,
            ws=None, stream=None, events=None) -> torch.Tensor:
    """y = ELSAA(q, k, v); writes the saved state into ``saved`` when given.
    ``events``: optional list of len(FWD_STAGES) + 1 torch.cuda.Event recorded
    around each stage."""
    if y is None:
        y = torch.empty_like(q)
    if ws is None:
        ws = alloc_workspace(p, q.device)
    code = lib().elsaa_forward_staged(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(r_sort),
                                      _ptr(r_race), _ptr(gate_w), _ptr(gate_b), _ptr(lam),
                                      _ptr(y), _ptr(saved), _ptr(ws), ws.numel(),
                                      _stream(stream), _events(events))
    _ok("elsaa_forward", code)
    return y


def backward(p: Params, q, k, v, r_sort, r_race, gate_w, gate_b, lam, saved, dy, dq=None,
             dk=None, dv=None, dgate_w=None, dgate_b=None, dlam=None, ws=None, stream=None,
             events=None):
    """Gradients of sum(y * dy): (dq, dk, dv, dgate_w, dgate_b, dlambda)."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    dev = q.device
    dgate_w = torch.empty(2, p.d, dtype=torch.float32, device=dev) if dgate_w is None else dgate_w
    dgate_b = torch.empty(2, dtype=torch.float32, device=dev) if dgate_b is None else dgate_b
    dlam = torch.empty(1, dtype=torch.float32, device=dev) if dlam is None else dlam
    if ws is None:
        ws = alloc_workspace(p, dev)
    code = lib().elsaa_backward_staged(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(r_sort),
                                       _ptr(r_race), _ptr(gate_w), _ptr(gate_b), _ptr(lam),
                                       _ptr(saved), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv),
                                       _ptr(dgate_w), _ptr(dgate_b), _ptr(dlam), _ptr(ws),
                                       ws.numel(), _stream(stream), _events(events))
    _ok("elsaa_backward", code)
    return dq, dk, dv, dgate_w, dgate_b, dlam


def sort_codes_noalloc(p: Params, code: torch.Tensor, perm: torch.Tensor, stream=None) -> None:
    """Sort-LSH permutations of ``code`` ([2, B, H, N] int16 view of the uint16
    sort codes, queries then keys) into ``perm`` ([2, B, H, N] int32) with no
    scratch from the caller: for callers that cannot allocate device memory
    while they run (see elsaa_sort_codes_noalloc in include/elsaa.h).  Both
    tensors must be contiguous and on the current CUDA device, whose scratch
    array the call uses."""
    n = 2 * p.B * p.H * p.N
    if code.dtype not in (torch.int16, torch.uint16) or perm.dtype != torch.int32:
        raise TypeError("code must be int16/uint16 and perm int32")
    if code.numel() != n or perm.numel() != n:
        raise ValueError(f"code and perm must hold 2*B*H*N = {n} elements")
    if not (code.is_contiguous() and perm.is_contiguous()):
        raise ValueError("code and perm must be contiguous")
    cur = torch.cuda.current_device()
    for t in (code, perm):
        if t.device.type != "cuda" or t.device.index != cur:
            raise ValueError(f"tensors must be on the current device cuda:{cur}")
    _ok("elsaa_sort_codes_noalloc", lib().elsaa_sort_codes_noalloc(
        ctypes.byref(p), _ptr(code), _ptr(perm), _stream(stream)))


# ---- pieces for a sequence split across devices (shard.py) -------------------

def _tables_shape(p: Params):
    return (p.B, p.H, p.race_tables, 1 << p.race_bits)


def sort_codes_of(p: Params, q, k, r_sort, r_race, ws=None, stream=None) -> torch.Tensor:
    """Sort codes [2, B, H, N] (int16 view of uint16) of q and k."""
    ws = alloc_workspace(p, q.device) if ws is None else ws
    code = torch.empty((2, p.B, p.H, p.N), dtype=torch.int16, device=q.device)
    _ok("elsaa_sort_codes_of", lib().elsaa_sort_codes_of(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(r_sort), _ptr(r_race), _ptr(code), _ptr(ws),
        ws.numel(), _stream(stream)))
    return code


def sort_codes(p: Params, code: torch.Tensor, ws=None, stream=None) -> torch.Tensor:
    """Stable Sort-LSH order [2, B, H, N] int32 of codes [2, B, H, N]."""
    ws = alloc_workspace(p, code.device) if ws is None else ws
    perm = torch.empty((2, p.B, p.H, p.N), dtype=torch.int32, device=code.device)
    _ok("elsaa_sort_codes", lib().elsaa_sort_codes(ctypes.byref(p), _ptr(code), _ptr(perm),
                                                   _ptr(ws), ws.numel(), _stream(stream)))
    return perm


def race_tables(p: Params, k, v, r_race, ws=None, stream=None):
    """RACE tables of k, v: (sums [B, H, L, NB, d] fp32, counts [B, H, L, NB] int32)."""
    ws = alloc_workspace(p, k.device) if ws is None else ws
    sums = torch.empty(_tables_shape(p) + (p.d,), dtype=torch.float32, device=k.device)
    counts = torch.empty(_tables_shape(p), dtype=torch.int32, device=k.device)
    _ok("elsaa_race_tables", lib().elsaa_race_tables(
        ctypes.byref(p), _ptr(k), _ptr(v), _ptr(r_race), _ptr(sums), _ptr(counts), _ptr(ws),
        ws.numel(), _stream(stream)))
    return sums, counts


def forward_tables(p: Params, q, k, v, r_sort, r_race, gate_w, gate_b, lam, sums, counts,
                   y=None, saved=None, ws=None, stream=None) -> torch.Tensor:
    """elsaa_forward with the RACE tables given."""
    y = torch.empty_like(q) if y is None else y
    ws = alloc_workspace(p, q.device) if ws is None else ws
    _ok("elsaa_forward_tables", lib().elsaa_forward_tables(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(r_sort), _ptr(r_race), _ptr(gate_w),
        _ptr(gate_b), _ptr(lam), _ptr(sums), _ptr(counts), _ptr(y), _ptr(saved), _ptr(ws),
        ws.numel(), _stream(stream)))
    return y


def backward_tables(p: Params, q, k, v, r_sort, r_race, gate_w, gate_b, lam, saved, dy, ws,
                    stream=None):
    """(dq, dk, dv without the RACE value gradient, dgate_w, dgate_b, dlambda,
    d_race_sum) of a forward_tables call."""
    dev = q.device
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dgw = torch.empty(2, p.d, dtype=torch.float32, device=dev)
    dgb = torch.empty(2, dtype=torch.float32, device=dev)
    dlam = torch.empty(1, dtype=torch.float32, device=dev)
    dsums = torch.empty(_tables_shape(p) + (p.d,), dtype=torch.float32, device=dev)
    _ok("elsaa_backward_tables", lib().elsaa_backward_tables(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(r_sort), _ptr(r_race), _ptr(gate_w),
        _ptr(gate_b), _ptr(lam), _ptr(saved), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgw),
        _ptr(dgb), _ptr(dlam), _ptr(dsums), _ptr(ws), ws.numel(), _stream(stream)))
    return dq, dk, dv, dgw, dgb, dlam, dsums


def race_value_grad(p: Params, k, r_race, d_sums, dv, ws=None, stream=None) -> None:
    """dv += the RACE branch's value gradient of keys k (in place)."""
    ws = alloc_workspace(p, k.device) if ws is None else ws
    _ok("elsaa_race_value_grad", lib().elsaa_race_value_grad(
        ctypes.byref(p), _ptr(k), _ptr(r_race), _ptr(d_sums), _ptr(dv), _ptr(ws), ws.numel(),
        _stream(stream)))


def check(ws: torch.Tensor, stream=None) -> None:
    _ok("elsaa_check", lib().elsaa_check(_ptr(ws), _stream(stream)))


def saved_views(p: Params, saved: torch.Tensor) -> Dict[str, torch.Tensor]:
    """Torch views (on the saved buffer's device) of a forward's saved state."""
    v = Views()
    _ok("elsaa_saved_views", lib().elsaa_saved_views(ctypes.byref(p), _ptr(saved),
                                                      ctypes.byref(v)))
    B, H, N, d, L, NB = p.B, p.H, p.N, p.d, p.race_tables, 1 << p.race_bits
    base = saved.data_ptr()
    flat = saved.view(torch.uint8)

    def view(addr, count, dtype, shape):
        off = addr - base
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        return flat[off:off + nbytes].view(dtype).view(*shape)

    rdt = torch.uint8 if v.rcode_bytes == 1 else torch.int16
    dt = p.torch_dtype
    n = B * H * N
    return {
        "code_q": view(v.code_q, n, torch.int16, (B, H, N)),
        "code_k": view(v.code_k, n, torch.int16, (B, H, N)),
        "perm_q": view(v.perm_q, n, torch.int32, (B, H, N)),
        "perm_k": view(v.perm_k, n, torch.int32, (B, H, N)),
        "rcode_q": view(v.rcode_q, n * L, rdt, (B, H, N, L)),
        "rcode_k": view(v.rcode_k, n * L, rdt, (B, H, N, L)),
        "race_count": view(v.race_count, B * H * L * NB, torch.int32, (B, H, L, NB)),
        "race_sum": view(v.race_sum, B * H * L * NB * d, torch.float32, (B, H, L, NB, d)),
        "lse_sp": view(v.lse_sp, n, torch.float32, (B, H, N)),
        "o_sp": view(v.o_sp, n * d, dt, (B, H, N, d)),
        "o_race": view(v.o_race, n * d, dt, (B, H, N, d)),
        "ctot": view(v.ctot, n, torch.int32, (B, H, N)),
        # every hash round: [R, 2 (queries, keys), B, H, N]
        "round_code": view(v.round_code, v.hash_rounds * 2 * n, torch.int16,
                           (v.hash_rounds, 2, B, H, N)),
        "round_perm": view(v.round_perm, v.hash_rounds * 2 * n, torch.int32,
                           (v.hash_rounds, 2, B, H, N)),
    }


def unsigned16(t: torch.Tensor) -> torch.Tensor:
    """int16 view of uint16 codes -> int64 values in [0, 65535]."""
    return t.to(torch.int64) & 0xFFFF


class ElsaaFunction(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in libelsaa."""

    @staticmethod
    def forward(ctx, q, k, v, gate_w, gate_b, lam, r_sort, r_race, params: Params):
        saved = alloc_saved(params, q.device)
        ws = alloc_workspace(params, q.device)
        y = forward(params, q.contiguous(), k.contiguous(), v.contiguous(), r_sort, r_race,
                    gate_w, gate_b, lam, saved=saved, ws=ws)
        ctx.params = params
        ctx.save_for_backward(q, k, v, gate_w, gate_b, lam, r_sort, r_race, saved, ws)
        return y

    @staticmethod
    def backward(ctx, dy):
        q, k, v, gate_w, gate_b, lam, r_sort, r_race, saved, ws = ctx.saved_tensors
        dq, dk, dv, dgw, dgb, dlam = backward(ctx.params, q, k, v, r_sort, r_race, gate_w,
                                              gate_b, lam, saved, dy.contiguous(), ws=ws)
        return dq, dk, dv, dgw, dgb, dlam.view_as(lam), None, None, None


def elsaa(q, k, v, gate_w, gate_b, lam, r_sort, r_race, params: Params):
    """Differentiable ELSAA attention on [B, H, N, d] CUDA tensors."""
    return ElsaaFunction.apply(q, k, v, gate_w, gate_b, lam, r_sort, r_race, params)
