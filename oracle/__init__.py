"""CPU oracle for MoE routing, dispatch layout, dispatch and combine.

TEST INFRASTRUCTURE: only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The library itself
never does.  The arithmetic lives in ``ep_oracle.c`` (plain C, fp32 where the
method fixes fp32, fp64 for the sigmoid); this file only compiles it and
marshals numpy arrays.

Every function here is pinned by ``tests/test_oracle_pins.py`` (and the
expert activation by ``tests/test_oracle_activation.py``) against
brute force, closed forms, invariants or a library routine.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libep_oracle.so")

BAD_EXPERT = 1
BAD_REPLICA = 2

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
          "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libep_oracle.so``."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lquadmath", "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, I, F, U8, U16 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                           ctypes.c_uint8, ctypes.c_uint16)
        _lib.orc_route.argtypes = [P, P, I, I, I, I, I, F, I, P, P, P]
        _lib.orc_route.restype = I
        _lib.orc_layout.argtypes = [P, I, I, I, I, I, P, P, I, P, P, P, P, P, P, P, P]
        _lib.orc_layout.restype = I
        _lib.orc_layout_aligned.argtypes = [P, I, I, I, I, I, P, P, I, I, P, P, P, P, P, P, P, P]
        _lib.orc_layout_aligned.restype = I
        _lib.orc_dispatch.argtypes = [P, I, I, I, P, I, I, P, P]
        _lib.orc_dispatch.restype = None
        _lib.orc_quantize_row.argtypes = [P, I, P, P]
        _lib.orc_quantize_row.restype = None
        _lib.orc_combine.argtypes = [P, I, P, P, I, I, I, P]
        _lib.orc_combine.restype = None
        _lib.orc_sigmoid.argtypes = [F, ctypes.POINTER(I)]
        _lib.orc_sigmoid.restype = F
        _lib.orc_e4m3_encode.argtypes = [F]
        _lib.orc_e4m3_encode.restype = U8
        _lib.orc_e4m3_decode.argtypes = [U8]
        _lib.orc_e4m3_decode.restype = F
        _lib.orc_bf16_encode.argtypes = [F]
        _lib.orc_bf16_encode.restype = U16
        _lib.orc_bf16_decode.argtypes = [U16]
        _lib.orc_bf16_decode.restype = F
        _lib.orc_dispatch_backward.argtypes = [P, I, P, I, I, I, P]
        _lib.orc_dispatch_backward.restype = None
        _lib.orc_combine_backward.argtypes = [P, P, I, P, P, I, I, I, P, P]
        _lib.orc_combine_backward.restype = None
        S = ctypes.c_size_t
        U32 = ctypes.c_uint32
        _lib.orc_sigmoid_hard_scan.argtypes = [U32, U32, P, U32]
        _lib.orc_sigmoid_hard_scan.restype = U32
        _lib.orc_e4m3_encode_array.argtypes = [P, S, P]
        _lib.orc_e4m3_encode_array.restype = None
        _lib.orc_bf16_encode_array.argtypes = [P, S, P]
        _lib.orc_bf16_encode_array.restype = None
        _lib.orc_sigmoid_array.argtypes = [P, S, P, P]
        _lib.orc_sigmoid_array.restype = None
        _lib.orc_silu_bf16.argtypes = [U16, ctypes.POINTER(I)]
        _lib.orc_silu_bf16.restype = U16
        _lib.orc_silu_bf16_array.argtypes = [P, S, P, P]
        _lib.orc_silu_mul_row.argtypes = [P, I, P]
        _lib.orc_silu_mul_row.restype = None
        _lib.orc_silu_mul_quant.argtypes = [P, I, I, P, P, I, I, P, P]
        _lib.orc_silu_mul_quant.restype = None
        _lib.orc_silu_bf16_array.restype = None
    return _lib


def _np(a, dtype):
    """A C-contiguous numpy view/copy of ``a`` (numpy array or CPU tensor)."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu()
        if str(a.dtype) == "torch.bfloat16":
            a = a.view(__import__("torch").int16)
        a = a.numpy()
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        a = a.view(dtype) if a.dtype.itemsize == np.dtype(dtype).itemsize else a.astype(dtype)
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data


def _token_ranges(T: int, threads: int):
    """[t0, t1) ranges splitting T tokens over ``threads`` workers."""
    n = max(1, min(int(threads), T)) if T > 0 else 1
    per = -(-T // n) if T > 0 else 0
    return [(t0, min(T, t0 + per)) for t0 in range(0, T, per)] if T > 0 else []


def _run_ranges(fn, T: int, threads: int):
    """Runs fn(t0, t1) over token ranges, on ``threads`` host threads when
    more than one (ctypes releases the GIL for the C call, and tokens are
    independent in routing, dispatch and combine, so each range writes its
    own outputs).  The arithmetic per token is unchanged."""
    ranges = _token_ranges(T, threads)
    if threads <= 1 or len(ranges) <= 1:
        for r in ranges:
            fn(*r)
        return
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=len(ranges)) as ex:
        for f in [ex.submit(fn, *r) for r in ranges]:
            f.result()


def sigmoid_hard_scan(first: int, count: int, cap: int = 1 << 16) -> np.ndarray:
    """fp32 bit patterns in [first, first + count) whose sigmoid lies within
    2^-47 of an fp32 rounding midpoint in fp64 (decided in quad precision)."""
    out = np.zeros(cap, np.uint32)
    n = int(lib().orc_sigmoid_hard_scan(first, count, out.ctypes.data, cap))
    if n > cap:
        raise RuntimeError("more hard inputs than the buffer holds")
    return out[:n].copy()


def sigmoid(x: float):
    """(fp32 sigmoid, hard flag) for one fp32 input."""
    h = ctypes.c_int(0)
    v = lib().orc_sigmoid(ctypes.c_float(x), ctypes.byref(h))
    return np.float32(v), bool(h.value)


def route(logits, bias, n_group: int, topk_group: int, topk: int,
          routed_scale: float, renorm: bool, threads: int = 1):
    """Returns (topk_idx int32 [T,k], topk_w fp32 [T,k], hard uint8 [T]).
    threads > 1 routes token ranges on that many host threads."""
    lg = _np(logits, np.float32)
    T, E = lg.shape
    b = _np(bias, np.float32)
    idx = np.zeros((T, topk), dtype=np.int32)
    w = np.zeros((T, topk), dtype=np.float32)
    hard = np.zeros(T, dtype=np.uint8)
    L = lib()
    if L.orc_route(None, None, 0, E, n_group, topk_group, topk, 1.0, 0, None, None, None):
        raise ValueError(f"routing undefined for E={E}, n_group={n_group}, "
                         f"topk_group={topk_group}, k={topk}")

    def part(t0, t1):
        L.orc_route(_ptr(lg[t0:t1]), _ptr(b), t1 - t0, E, n_group, topk_group, topk,
                    float(routed_scale), int(bool(renorm)), _ptr(idx[t0:t1]), _ptr(w[t0:t1]),
                    _ptr(hard[t0:t1]))
    _run_ranges(part, T, threads)
    return idx, w, hard


def layout(topk_idx, E: int, P: int, R: int, phys_of=None, n_rep=None, row_align: int = 1):
    """Dispatch layout (expert starts padded to row_align rows when > 1).
    Returns a dict of arrays plus ``status`` bits; ``src`` has one entry per
    receive row (padding rows -1)."""
    ti = _np(topk_idx, np.int32)
    T, k = ti.shape
    po = _np(phys_of, np.int32)
    nr = _np(n_rep, np.int32)
    max_rep = 0 if po is None else po.shape[1]
    n_src = T * k + P * (row_align - 1)
    out = dict(
        cnt_expert=np.zeros(P, np.int32), expert_off=np.zeros(P + 1, np.int32),
        rows_rank=np.zeros(R, np.int32), rank_off=np.zeros(R + 1, np.int32),
        tok_rank=np.zeros(R, np.int32), in_rank=np.zeros((T, R), np.uint8),
        slot=np.zeros((T, k), np.int32), src=np.full(n_src, -1, np.int32))
    st = lib().orc_layout_aligned(_ptr(ti), T, k, E, P, R, _ptr(po), _ptr(nr), max_rep,
                                  row_align,
                                  *(_ptr(out[n]) for n in ("cnt_expert", "expert_off",
                                                           "rows_rank", "rank_off", "tok_rank",
                                                           "in_rank", "slot", "src")))
    out["src"] = out["src"][:int(out["expert_off"][P])]
    out["status"] = int(st)
    return out


def quantize_row(x_row):
    """One bf16 row (uint16 bits or bf16 tensor) -> (e4m3 codes, fp32 scales)."""
    xr = _np(x_row, np.uint16)
    H = xr.shape[-1]
    q = np.zeros(H, np.uint8)
    sc = np.zeros(H // 128, np.float32)
    lib().orc_quantize_row(_ptr(xr), H, _ptr(q), _ptr(sc))
    return q, sc


def dispatch(x, slot, fp8: bool, n_rows=None, threads: int = 1):
    """Returns (recv_x, recv_scale); recv_x uint8 [n_rows,H] (fp8) or uint16.
    threads > 1 dispatches token ranges on that many host threads (the
    ranges write disjoint receive rows: slots are distinct)."""
    xs = _np(x, np.uint16)
    T, H = xs.shape
    sl = _np(slot, np.int32)
    k = sl.shape[1]
    n = T * k if n_rows is None else n_rows
    if fp8:
        rx = np.zeros((n, H), np.uint8)
        rs = np.zeros((n, H // 128), np.float32)
    else:
        rx = np.zeros((n, H), np.uint16)
        rs = None
    L = lib()

    def part(t0, t1):
        L.orc_dispatch(_ptr(xs[t0:t1]), t1 - t0, H, k, _ptr(sl[t0:t1]), n, int(bool(fp8)),
                       _ptr(rx), _ptr(rs))
    _run_ranges(part, T, threads)
    return rx, rs


def combine(y, slot, topk_w, threads: int = 1):
    """out bf16 bits (uint16 [T,H]) = sum_j w * y[slot], fp32 in j order.
    threads > 1 combines token ranges on that many host threads."""
    ys = _np(y, np.uint16)
    n, H = ys.shape
    sl = _np(slot, np.int32)
    T, k = sl.shape
    w = _np(topk_w, np.float32)
    out = np.zeros((T, H), np.uint16)
    L = lib()

    def part(t0, t1):
        L.orc_combine(_ptr(ys), n, _ptr(sl[t0:t1]), _ptr(w[t0:t1]), t1 - t0, H, k,
                      _ptr(out[t0:t1]))
    _run_ranges(part, T, threads)
    return out


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(ctypes.c_float(v)))


def e4m3_decode(c: int) -> float:
    return float(lib().orc_e4m3_decode(ctypes.c_uint8(c)))


def bf16_encode(v: float) -> int:
    return int(lib().orc_bf16_encode(ctypes.c_float(v)))


def e4m3_encode_array(v) -> np.ndarray:
    a = _np(v, np.float32)
    out = np.zeros(a.shape, np.uint8)
    lib().orc_e4m3_encode_array(_ptr(a), a.size, _ptr(out))
    return out


def bf16_encode_array(v) -> np.ndarray:
    a = _np(v, np.float32)
    out = np.zeros(a.shape, np.uint16)
    lib().orc_bf16_encode_array(_ptr(a), a.size, _ptr(out))
    return out


def sigmoid_array(x):
    """(fp32 sigmoids, hard flags) of an fp32 array."""
    a = _np(x, np.float32)
    out = np.zeros(a.shape, np.float32)
    hard = np.zeros(a.shape, np.uint8)
    lib().orc_sigmoid_array(_ptr(a), a.size, _ptr(out), _ptr(hard))
    return out, hard


def dispatch_backward(grad_recv, slot):
    """grad_x bf16 bits (uint16 [T,H]) = sum_j grad_recv[slot[t,j]] (fp32, j order)."""
    g = _np(grad_recv, np.uint16)
    n, H = g.shape
    sl = _np(slot, np.int32)
    T, k = sl.shape
    out = np.zeros((T, H), np.uint16)
    lib().orc_dispatch_backward(_ptr(g), n, _ptr(sl), T, H, k, _ptr(out))
    return out


def combine_backward(grad_out, y, slot, topk_w):
    """(grad_y bf16 bits uint16 [T*k,H] (untouched rows 0), grad_w fp32 [T,k])."""
    g = _np(grad_out, np.uint16)
    T, H = g.shape
    ys = _np(y, np.uint16)
    n = ys.shape[0]
    sl = _np(slot, np.int32)
    k = sl.shape[1]
    w = _np(topk_w, np.float32)
    gy = np.zeros((n, H), np.uint16)
    gw = np.zeros((T, k), np.float32)
    lib().orc_combine_backward(_ptr(g), _ptr(ys), n, _ptr(sl), _ptr(w), T, H, k, _ptr(gy),
                               _ptr(gw))
    return gy, gw


def silu_bf16_array(g):
    """(bf16 bits of silu(g) correctly rounded, hard flags) for bf16 bits g."""
    a = _np(g, np.uint16)
    out = np.zeros(a.shape, np.uint16)
    hard = np.zeros(a.shape, np.uint8)
    lib().orc_silu_bf16_array(_ptr(a), a.size, _ptr(out), _ptr(hard))
    return out, hard


def silu_mul_quant(gate_up, fp8: bool, expert_off=None, cnt_expert=None, act=None,
                   act_scale=None):
    """Expert activation of bf16 rows [n_rows, 2I] (uint16 bits).  Returns
    (act, act_scale): e4m3 codes uint8 [n_rows, I] and fp32 [n_rows, I/128]
    when fp8, else bf16 bits uint16 [n_rows, I] and None.  Only the rows the
    counts select are written; pass act / act_scale to see the others kept."""
    gu = _np(gate_up, np.uint16)
    n, I2 = gu.shape
    I = I2 // 2
    if act is None:
        act = np.zeros((n, I), np.uint8 if fp8 else np.uint16)
    if fp8 and act_scale is None:
        act_scale = np.zeros((n, max(I // 128, 1)), np.float32)
    eo = _np(expert_off, np.int32)
    ce = _np(cnt_expert, np.int32)
    P = 0 if ce is None else ce.size
    lib().orc_silu_mul_quant(_ptr(gu), n, I, _ptr(eo), _ptr(ce), P, int(bool(fp8)), _ptr(act),
                             _ptr(act_scale) if fp8 else None)
    return act, (act_scale if fp8 else None)
