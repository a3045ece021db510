"""Thin ctypes binding of libmoeq.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does
nothing but check tensor dtypes/devices, pass raw pointers and sizes, and
turn a non-zero status into an exception.  All arithmetic runs in the CUDA
kernels of the library; there is no CPU fallback: ``load()`` raises when
the library is missing or no CUDA device is present.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoeq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "moeq.h")

LAYOUT_INT4 = 0
LAYOUT_PLANES = 1
DEV_BAD_INDEX = 1
DEV_RANGE = 2
DEV_TIMEOUT = 4

_c_p = ctypes.c_void_p
_c_i = ctypes.c_int
_c_sz = ctypes.c_size_t

_SIGS = {
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_blob_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i]),
    "moe_quant_pack": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p]),
    "moe_route_topk": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p, _c_sz,
                              _c_p]),
    "moe_route_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i]),
    "moe_route_topk_noalloc": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p]),
    "moe_permute": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p, _c_p, _c_p,
                           _c_p, _c_p, _c_sz, _c_p]),
    "moe_permute_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i]),
    "moe_route_permute": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p,
                                 _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "moe_route_permute_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i]),
    "moe_static_bits": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p]),
    "moe_bit_gate": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, _c_p]),
    "moe_ffn_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i]),
    "moe_grouped_ffn_wq": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i,
                                  _c_p, _c_sz, _c_p, _c_p, _c_p]),
    "moe_unpermute_combine": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_p, _c_p]),
    "moe_grouped_ffn_combine": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p,
                                       _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p, _c_p]),
    "moe_ffn_combine_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i, _c_i]),
    "moe_slot_cache_create": (_c_i, [_c_i, _c_i, _c_sz, _c_p, _c_p, ctypes.POINTER(_c_p)]),
    "moe_slot_cache_create_planes": (_c_i, [_c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_p, ctypes.POINTER(_c_p)]),
    "moe_slot_stage": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_p, _c_p, _c_p, _c_p]),
    "moe_slot_ffn": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i, _c_p, _c_sz, _c_p,
                            _c_p, _c_p, _c_p]),
    "moe_slot_cache_destroy": (None, [_c_p]),
    "moe_slot_prefetch": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_p, _c_p]),
    "moe_slot_timing": (_c_i, [_c_p, _c_i]),
    "moe_slot_timing_read": (_c_i, [_c_p, _c_p, _c_p]),
    "moe_predictor_create": (_c_i, [_c_i, _c_i, ctypes.POINTER(_c_p)]),
    "moe_predictor_destroy": (None, [_c_p]),
    "moe_predictor_observe": (_c_i, [_c_p, _c_i, _c_p, _c_p, _c_p, _c_i, _c_i]),
    "moe_predictor_predict": (_c_i, [_c_p, _c_i, _c_p, _c_p, _c_i, _c_i, _c_i, ctypes.c_double, _c_p, _c_p]),
    "moe_debug_inject_fault": (None, [_c_i, _c_i]),
    "moe_debug_force_regime": (None, [_c_i]),
    "moe_debug_set_trace": (None, [_c_p]),
    "moe_debug_ffn_timeout": (None, [_c_i]),
    "moe_debug_route_fused": (None, [_c_i]),
}

_lib = None


class MoeError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def header_symbols() -> list:
    """Names of the functions declared in include/moeq.h."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def open_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """dlopen the library and attach signatures (needs no GPU)."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run quantized_moe_expert_histogram_b200.build.build()")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load():
    """The library, for compute calls; raises without a CUDA device."""
    global _lib
    if not torch.cuda.is_available():
        raise RuntimeError("moeq needs a CUDA device (B200, sm_100a); no CPU fallback exists")
    if _lib is None:
        _lib = open_library()
    return _lib


def _check(fn, code):
    if code != 0:
        raise MoeError(fn, code, _lib.moe_last_error().decode())


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def moe_blob_bytes(d, F, group, layout):
    return int(load().moe_blob_bytes(d, F, group, layout))


def moe_ffn_workspace_bytes(total_rows, E, d, F, layout):
    return int(load().moe_ffn_workspace_bytes(total_rows, E, d, F, layout))


def moe_quant_pack(w_gate, w_up, w_down, group, layout, blobs=None, stream=None):
    lib = load()
    E, F, d = w_gate.shape
    nb = lib.moe_blob_bytes(d, F, group, layout)
    if blobs is None:
        blobs = torch.empty(E, nb, dtype=torch.uint8, device=w_gate.device)
    _check("moe_quant_pack", lib.moe_quant_pack(
        _ptr(w_gate, torch.float32, "w_gate"), _ptr(w_up, torch.float32, "w_up"),
        _ptr(w_down, torch.float32, "w_down"), E, d, F, group, layout,
        _ptr(blobs, torch.uint8, "blobs"), _stream(stream)))
    return blobs


def moe_route_workspace_bytes(T, d, E):
    return int(load().moe_route_workspace_bytes(T, d, E))


def moe_route_topk(x, w_router, bias, k, forced_idx=None, topk_idx=None, topk_w=None, workspace=None,
                   stream=None):
    lib = load()
    T, d = x.shape
    E = w_router.shape[0]
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(lib.moe_route_workspace_bytes(T, d, E), dtype=torch.uint8, device=x.device)
    _check("moe_route_topk", lib.moe_route_topk(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_router, torch.float32, "w_router"),
        _ptr(bias, torch.float32, "bias"), _ptr(forced_idx, torch.int32, "forced_idx"), T, d, E, k,
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return topk_idx, topk_w


def moe_permute_workspace_bytes(T, E, k, nested):
    return int(load().moe_permute_workspace_bytes(T, E, k, int(bool(nested))))


def moe_permute(topk_idx, E, bits=None, x=None, out=None, status=None, workspace=None, stream=None):
    """Returns dict(counts, offsets, perm, inv_perm, x_perm)."""
    lib = load()
    T, k = topk_idx.shape
    nb = 3 * E if bits is not None else E
    dev = topk_idx.device
    d = x.shape[1] if x is not None else 0
    if out is None:
        out = dict(counts=torch.empty(nb, dtype=torch.int32, device=dev),
                   offsets=torch.empty(nb + 1, dtype=torch.int32, device=dev),
                   perm=torch.empty(T * k, dtype=torch.int32, device=dev),
                   inv_perm=torch.empty(T * k, dtype=torch.int32, device=dev),
                   x_perm=torch.empty(T * k, d, dtype=torch.float16, device=dev) if x is not None else None)
    if workspace is None:
        workspace = out.get("perm_ws")
    if workspace is None:
        workspace = torch.empty(lib.moe_permute_workspace_bytes(T, E, k, int(bits is not None)),
                                dtype=torch.uint8, device=dev)
    _check("moe_permute", lib.moe_permute(
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(bits, torch.uint8, "bits"),
        _ptr(x, torch.bfloat16, "x"), T, d, E, k, _ptr(out["counts"], torch.int32),
        _ptr(out["offsets"], torch.int32), _ptr(out["perm"], torch.int32),
        _ptr(out["inv_perm"], torch.int32), _ptr(out["x_perm"], torch.float16),
        _ptr(status, torch.int32, "status"), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return out


def moe_route_permute_workspace_bytes(T, d, E, k, nested):
    return int(load().moe_route_permute_workspace_bytes(T, d, E, k, int(bool(nested))))


def moe_route_permute(x, w_router, bias, k, forced_idx=None, bits=None, w_bit=None, bias_bit=None, out=None,
                      status=None, workspace=None, gather=True, stream=None):
    """Router, optional bit gate (w_bit) or given widths (bits), and the
    permutation in one call.  Returns dict(topk_idx, topk_w, bits, counts,
    offsets, perm, inv_perm, x_perm); 'bits' holds the gate's widths (or the
    given ones, or None)."""
    lib = load()
    T, d = x.shape
    E = w_router.shape[0]
    dev = x.device
    nested = bits is not None or w_bit is not None
    nb = 3 * E if nested else E
    if out is None:
        out = {}
    out = dict(out)
    for key, shape, dt in (("topk_idx", (T, k), torch.int32), ("topk_w", (T, k), torch.float32),
                           ("counts", (nb,), torch.int32), ("offsets", (nb + 1,), torch.int32),
                           ("perm", (T * k,), torch.int32), ("inv_perm", (T * k,), torch.int32)):
        if out.get(key) is None:
            out[key] = torch.empty(*shape, dtype=dt, device=dev)
    if gather and out.get("x_perm") is None:
        out["x_perm"] = torch.empty(T * k, d, dtype=torch.float16, device=dev)
    bits_out = None
    if w_bit is not None:
        bits_out = out.get("bits")
        if bits_out is None:
            bits_out = torch.empty(T, k, dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = torch.empty(lib.moe_route_permute_workspace_bytes(T, d, E, k, int(nested)), dtype=torch.uint8,
                                device=dev)
    _check("moe_route_permute", lib.moe_route_permute(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_router, torch.float32, "w_router"), _ptr(bias, torch.float32, "bias"),
        _ptr(forced_idx, torch.int32, "forced_idx"), _ptr(bits, torch.uint8, "bits"),
        _ptr(w_bit, torch.float32, "w_bit"), _ptr(bias_bit, torch.float32, "bias_bit"), T, d, E, k,
        _ptr(out["topk_idx"], torch.int32), _ptr(out["topk_w"], torch.float32), _ptr(bits_out, torch.uint8),
        _ptr(out["counts"], torch.int32), _ptr(out["offsets"], torch.int32), _ptr(out["perm"], torch.int32),
        _ptr(out["inv_perm"], torch.int32), _ptr(out["x_perm"] if gather else None, torch.float16),
        _ptr(status, torch.int32, "status"), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    out["bits"] = bits_out if w_bit is not None else bits
    return out


def moe_static_bits(topk_idx, width_of, E, bits=None, status=None, stream=None):
    """bits[t][j] = width_of[topk_idx[t][j]] (uint8 [T][k])."""
    lib = load()
    T, k = topk_idx.shape
    if bits is None:
        bits = torch.empty(T, k, dtype=torch.uint8, device=topk_idx.device)
    _check("moe_static_bits", lib.moe_static_bits(
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(width_of, torch.uint8, "width_of"), T, k, E,
        _ptr(bits, torch.uint8, "bits"), _ptr(status, torch.int32, "status"), _stream(stream)))
    return bits


def moe_bit_gate(x, w_bit, bias_bit, topk_idx, bits=None, status=None, stream=None):
    """bits[t][j] = 2 + argmax_c (x[t] . w_bit[e][c] + bias_bit[e][c]) for
    e = topk_idx[t][j] (uint8 [T][k])."""
    lib = load()
    T, d = x.shape
    E = w_bit.shape[0]
    k = topk_idx.shape[1]
    if bits is None:
        bits = torch.empty(T, k, dtype=torch.uint8, device=x.device)
    _check("moe_bit_gate", lib.moe_bit_gate(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_bit, torch.float32, "w_bit"),
        _ptr(bias_bit, torch.float32, "bias_bit"), _ptr(topk_idx, torch.int32, "topk_idx"), T, d, E, k,
        _ptr(bits, torch.uint8, "bits"), _ptr(status, torch.int32, "status"), _stream(stream)))
    return bits


def moe_ffn_combine_workspace_bytes(T, k, E, d, F, layout):
    return int(load().moe_ffn_combine_workspace_bytes(T, k, E, d, F, layout))


def moe_grouped_ffn_combine(x_perm, offsets, blobs, T, k, E, d, F, group, layout, perm, inv_perm, topk_w,
                            residual=None, y=None, y_perm=None, workspace=None, status=None, stream=None):
    """The grouped FFN and the weighted combine in one call; returns (y, y_perm)."""
    lib = load()
    dev = x_perm.device
    if y is None:
        y = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    if y_perm is None:
        y_perm = torch.empty(T * k, d, dtype=torch.float16, device=dev)
    if workspace is None:
        workspace = torch.empty(lib.moe_ffn_combine_workspace_bytes(T, k, E, d, F, layout), dtype=torch.uint8,
                                device=dev)
    _check("moe_grouped_ffn_combine", lib.moe_grouped_ffn_combine(
        _ptr(x_perm, torch.float16, "x_perm"), _ptr(offsets, torch.int32, "offsets"), _ptr(blobs), T, k, E, d, F,
        group, layout, _ptr(perm, torch.int32, "perm"), _ptr(inv_perm, torch.int32, "inv_perm"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(residual, torch.bfloat16, "residual"),
        _ptr(y, torch.bfloat16, "y"), _ptr(y_perm, torch.float16, "y_perm"), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status, torch.int32, "status"), _stream(stream)))
    return y, y_perm


def moe_grouped_ffn_wq(x_perm, offsets, blobs, T, E, d, F, group, layout, slot_of=None,
                       workspace=None, y_perm=None, status=None, stream=None):
    lib = load()
    rows = x_perm.shape[0]
    if workspace is None:
        workspace = torch.empty(lib.moe_ffn_workspace_bytes(rows, E, d, F, layout), dtype=torch.uint8,
                                device=x_perm.device)
    if y_perm is None:
        y_perm = torch.empty(rows, d, dtype=torch.float16, device=x_perm.device)
    _check("moe_grouped_ffn_wq", lib.moe_grouped_ffn_wq(
        _ptr(x_perm, torch.float16, "x_perm"), _ptr(offsets, torch.int32, "offsets"), _ptr(blobs),
        _ptr(slot_of, torch.int32, "slot_of"), rows, T, E, d, F, group, layout, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(y_perm, torch.float16, "y_perm"),
        _ptr(status, torch.int32, "status"), _stream(stream)))
    return y_perm


def moe_unpermute_combine(y_perm, inv_perm, topk_w, residual=None, y=None, stream=None):
    lib = load()
    T, k = topk_w.shape
    d = y_perm.shape[1]
    if y is None:
        y = torch.empty(T, d, dtype=torch.bfloat16, device=y_perm.device)
    _check("moe_unpermute_combine", lib.moe_unpermute_combine(
        _ptr(y_perm, torch.float16, "y_perm"), _ptr(inv_perm, torch.int32, "inv_perm"),
        _ptr(topk_w, torch.float32, "topk_w"), _ptr(residual, torch.bfloat16, "residual"), T, k, d,
        _ptr(y, torch.bfloat16, "y"), _stream(stream)))
    return y


class SlotCache:
    """One layer's GPU slot cache (moe_slot_cache_create / _destroy); with
    planes=(d, F, group) a plane-mode cache of nested-plane blobs
    (moe_slot_cache_create_planes)."""

    def __init__(self, E, slots, blob_bytes, host_blobs, device_pool, planes=None):
        lib = load()
        if not host_blobs.is_pinned():
            raise ValueError("host_blobs must be pinned host memory")
        self._host = host_blobs
        self._pool = device_pool
        h = _c_p()
        if planes is None:
            _check("moe_slot_cache_create", lib.moe_slot_cache_create(
                E, slots, blob_bytes, host_blobs.data_ptr(), _ptr(device_pool), ctypes.byref(h)))
        else:
            d, F, group = planes
            moe_slot_cache_create_planes(E, slots, d, F, group, host_blobs, device_pool, h)
        self.handle = h
        self.E = E
        self._ids = None

    def stage(self, ids_host, copy_stream, compute_stream, bits_host=None):
        """moe_slot_stage; returns (n_waves, [hits, experts copied, bytes])."""
        lib = load()
        ids = ids_host.to(torch.int32).contiguous()
        bits = None if bits_host is None else bits_host.to(torch.uint8).contiguous().cpu()
        self._ids, self._bits = ids, bits
        nw = ctypes.c_int32(0)
        stats = (ctypes.c_int64 * 3)()
        _check("moe_slot_stage", lib.moe_slot_stage(
            self.handle, ids.data_ptr(), None if bits is None else bits.data_ptr(), ids.numel(),
            copy_stream.cuda_stream, compute_stream.cuda_stream, ctypes.byref(nw), stats))
        return nw.value, list(stats)

    def ffn(self, x_perm, offsets, T, d, F, group, layout, workspace, y_perm, status, copy_stream,
            compute_stream):
        lib = load()
        _check("moe_slot_ffn", lib.moe_slot_ffn(
            self.handle, _ptr(x_perm, torch.float16), _ptr(offsets, torch.int32), x_perm.shape[0], T,
            d, F, group, layout, _ptr(workspace), workspace.numel() * workspace.element_size(),
            _ptr(y_perm, torch.float16), _ptr(status, torch.int32), copy_stream.cuda_stream,
            compute_stream.cuda_stream))

    def prefetch(self, ids_host, max_copies, copy_stream):
        """moe_slot_prefetch: stage up to max_copies of the listed experts
        ahead of their layer-step; returns the number of copies issued."""
        return moe_slot_prefetch(self.handle, ids_host, max_copies, copy_stream)

    def timing(self, enable):
        """moe_slot_timing: record copy and FFN busy time from now on."""
        moe_slot_timing(self.handle, enable)

    def timing_read(self):
        """moe_slot_timing_read: (copy_ms, ffn_ms) since the last read."""
        return moe_slot_timing_read(self.handle)

    def close(self):
        if self.handle is not None and self.handle.value:
            load().moe_slot_cache_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_slot_prefetch(handle, ids_host, max_copies, copy_stream):
    ids = ids_host.to(torch.int32).contiguous()
    n = ctypes.c_int32(0)
    _check("moe_slot_prefetch", load().moe_slot_prefetch(handle, ids.data_ptr(), ids.numel(), int(max_copies),
                                                          copy_stream.cuda_stream, ctypes.byref(n)))
    return n.value


def moe_slot_cache_create_planes(E, slots, d, F, group, host_blobs, device_pool, handle):
    _check("moe_slot_cache_create_planes", load().moe_slot_cache_create_planes(
        E, slots, d, F, group, host_blobs.data_ptr(), _ptr(device_pool), ctypes.byref(handle)))
    return handle


def moe_slot_timing(handle, enable):
    _check("moe_slot_timing", load().moe_slot_timing(handle, int(bool(enable))))


def moe_slot_timing_read(handle):
    cm, fm = ctypes.c_double(0), ctypes.c_double(0)
    _check("moe_slot_timing_read", load().moe_slot_timing_read(handle, ctypes.addressof(cm), ctypes.addressof(fm)))
    return cm.value, fm.value


def moe_predictor_create(layers, E):
    h = _c_p()
    _check("moe_predictor_create", load().moe_predictor_create(layers, E, ctypes.byref(h)))
    return h


def moe_predictor_destroy(handle):
    load().moe_predictor_destroy(handle)


def _host_ids(ids):
    return None if ids is None else ids.to(torch.int32).contiguous().cpu()


def moe_predictor_observe(handle, layer, prev_ids, cur_ids, prev2_ids=None):
    prev, cur, prev2 = _host_ids(prev_ids), _host_ids(cur_ids), _host_ids(prev2_ids)
    T, k = prev.shape
    _check("moe_predictor_observe", load().moe_predictor_observe(
        handle, layer, None if prev2 is None else prev2.data_ptr(), prev.data_ptr(), cur.data_ptr(), T, k))


def moe_predictor_predict(handle, layer, prev_ids, max_out, min_score=0.0, prev2_ids=None):
    prev, prev2 = _host_ids(prev_ids), _host_ids(prev2_ids)
    T, k = prev.shape
    out = torch.empty(max(1, max_out), dtype=torch.int32)
    n = ctypes.c_int32(0)
    _check("moe_predictor_predict", load().moe_predictor_predict(
        handle, layer, None if prev2 is None else prev2.data_ptr(), prev.data_ptr(), T, k, max_out,
        float(min_score), out.data_ptr(), ctypes.byref(n)))
    return out[:n.value]


class RoutePredictor:
    """Next-layer expert predictor (moe_predictor_*), host-side."""

    def __init__(self, layers, E):
        self.handle = moe_predictor_create(layers, E)

    def observe(self, layer, prev_ids, cur_ids, prev2_ids=None):
        moe_predictor_observe(self.handle, layer, prev_ids, cur_ids, prev2_ids)

    def predict(self, layer, prev_ids, max_out, min_score=0.0, prev2_ids=None):
        return moe_predictor_predict(self.handle, layer, prev_ids, max_out, min_score, prev2_ids)

    def close(self):
        if self.handle is not None and self.handle.value:
            moe_predictor_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_debug_inject_fault(what, count):
    load().moe_debug_inject_fault(what, count)


def moe_last_error():
    return load().moe_last_error().decode()


def moe_debug_force_regime(regime):
    """0 = by T, 1 = one-token GEMV, 2 = tensor cores, 3 = small-batch mma.sync kernel (test hook)."""
    load().moe_debug_force_regime(regime)


def moe_debug_route_fused(mode):
    """Test hook: 1 (default) one cluster launch for the smallest batches of
    the router, the bit gate and moe_route_permute; 0 the two-launch router,
    the one-kernel bit gate and separate launches at every size (see
    moeq.h)."""
    load().moe_debug_route_fused(int(mode))


def moe_debug_ffn_timeout(enable):
    """Test hook: a withheld arrive and a 20 ms wait limit in the tensor-core FFN."""
    load().moe_debug_ffn_timeout(int(bool(enable)))


def moe_debug_set_trace(pinned_int32=None):
    """Progress record of the tensor-core FFN kernels (test hook)."""
    load().moe_debug_set_trace(None if pinned_int32 is None else pinned_int32.data_ptr())



def moe_route_topk_noalloc(x, w_router, bias, k, forced_idx=None, topk_idx=None, topk_w=None, stream=None):
    """The router without a workspace argument: its scratch is a fixed
    device array inside the library (see include/moeq.h)."""
    lib = load()
    T, d = x.shape
    E = w_router.shape[0]
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    _check("moe_route_topk_noalloc", lib.moe_route_topk_noalloc(
        _ptr(x, torch.bfloat16, "x"), _ptr(w_router, torch.float32, "w_router"),
        _ptr(bias, torch.float32, "bias"), _ptr(forced_idx, torch.int32, "forced_idx"), T, d, E, k,
        _ptr(topk_idx, torch.int32, "topk_idx"), _ptr(topk_w, torch.float32, "topk_w"), _stream(stream)))
    return topk_idx, topk_w
