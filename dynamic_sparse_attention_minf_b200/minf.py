"""Thin ctypes binding of libminf.so (the C ABI declared in include/minf.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch provides device memory and the current stream.  There is no
CPU fallback: if the library is missing, loading fails with an error.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libminf.so")

OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error",
                4: "workspace too small", 5: "device timeout", 6: "device bounds"}
OP_ESTIMATE_VS, OP_ESTIMATE_BS, OP_BUILD_INDEX, OP_SPARSE_ATTN_VS, OP_SPARSE_ATTN_BS, \
    OP_ATTN_ASHAPE, OP_DENSE_ATTN, OP_BUILD_INDEX_EXACT, OP_SPARSE_ATTN_VS_EXACT, OP_SPARSE_ATTN_LAYER, \
    OP_ATTN_GRID = range(11)

EXPORTS = ["minf_vs_wmap_words", "minf_workspace_size", "minf_estimate_vs", "minf_estimate_bs",
           "minf_build_index", "minf_sparse_attn_vs", "minf_sparse_attn_bs", "minf_attn_ashape",
           "minf_dense_attn", "minf_get_device_status", "minf_status_string", "minf_vs_bits_words",
           "minf_vs_twmap_words", "minf_build_index_exact", "minf_sparse_attn_vs_exact",
           "minf_sparse_attn_layer", "minf_selftest_exp2", "minf_attn_grid"]


class MinfError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)} ({code})")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("scale", ctypes.c_float)]


class _VsIndexC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("grp", "grp_cnt", "tgrp", "tgrp_cnt", "wmap", "vcnt", "vidx", "tvcnt", "tvidx")]


class _VsExactIndexC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("tgrp", "tgrp_cnt", "sbits", "vbits", "twmap", "vcnt", "vidx")]


_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libminf.so not found at {LIB_PATH}: run "
                               "`python -m dynamic_sparse_attention_minf_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_int
        sp = ctypes.POINTER(Shape)
        L.minf_vs_wmap_words.argtypes = [i]
        L.minf_vs_wmap_words.restype = sz
        L.minf_vs_bits_words.argtypes = [i]
        L.minf_vs_bits_words.restype = sz
        L.minf_vs_twmap_words.argtypes = [i]
        L.minf_vs_twmap_words.restype = sz
        L.minf_build_index_exact.argtypes = [sp, i, vp, i, vp, i, ctypes.POINTER(_VsExactIndexC), vp, sz, vp]
        L.minf_sparse_attn_vs_exact.argtypes = [sp, vp, vp, vp, vp, i, ctypes.POINTER(_VsExactIndexC), i, i,
                                                vp, vp, vp, sz, vp]
        L.minf_workspace_size.argtypes = [i, sp, i, i, i, i]
        L.minf_workspace_size.restype = sz
        L.minf_estimate_vs.argtypes = [sp, vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp, sz, vp]
        L.minf_estimate_bs.argtypes = [sp, vp, vp, vp, i, i, i, vp, vp, vp, vp, sz, vp]
        L.minf_build_index.argtypes = [sp, i, vp, i, vp, i, ctypes.POINTER(_VsIndexC), vp, sz, vp]
        L.minf_sparse_attn_vs.argtypes = [sp, vp, vp, vp, vp, i, ctypes.POINTER(_VsIndexC), i, i,
                                          vp, vp, vp, sz, vp]
        L.minf_sparse_attn_bs.argtypes = [sp, vp, vp, vp, vp, i, vp, vp, i, vp, vp, vp, sz, vp]
        L.minf_attn_ashape.argtypes = [sp, vp, vp, vp, vp, i, i, i, vp, vp, vp, sz, vp]
        L.minf_dense_attn.argtypes = [sp, vp, vp, vp, vp, i, vp, vp, vp, sz, vp]
        L.minf_selftest_exp2.argtypes = [vp, vp, vp, i, vp]
        L.minf_sparse_attn_layer.argtypes = [sp, vp, vp, vp, vp, i, ctypes.POINTER(_VsIndexC), i, i, vp, i, vp,
                                             vp, i, vp, i, i, i, vp, vp, vp, sz, vp]
        L.minf_attn_grid.argtypes = [sp, vp, vp, vp, vp, i, i, i, vp, vp, vp, vp, vp, sz, vp]
        L.minf_get_device_status.argtypes = [vp, vp]
        L.minf_status_string.argtypes = [st]
        L.minf_status_string.restype = ctypes.c_char_p
        for fn in ("minf_estimate_vs", "minf_estimate_bs", "minf_build_index", "minf_sparse_attn_vs",
                   "minf_sparse_attn_bs", "minf_attn_ashape", "minf_dense_attn", "minf_get_device_status",
                   "minf_build_index_exact", "minf_sparse_attn_vs_exact", "minf_sparse_attn_layer",
                   "minf_selftest_exp2"):
            getattr(L, fn).restype = st
        _lib = L
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != OK:
        raise MinfError(fn, code)


def shape_of(q, k, scale=0.0):
    B, Hq, N, d = q.shape
    return Shape(B, Hq, k.shape[1], N, d, float(scale))


def workspace(op, shape, nh, k_v=0, k_s=0, k_b=0, device="cuda"):
    """A zeroed workspace of the size the library asks for."""
    n = lib().minf_workspace_size(op, ctypes.byref(shape), nh, k_v, k_s, k_b)
    if n == 0:
        raise MinfError("minf_workspace_size", 1)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _heads(heads, device):
    if heads is None:
        return None
    if isinstance(heads, torch.Tensor):
        return heads.to(device=device, dtype=torch.int32).contiguous()
    return torch.tensor(list(heads), dtype=torch.int32, device=device)


@dataclass
class VSIndex:
    """Device buffers of the compact Vertical-Slash index (see minf_vs_index)."""
    grp: torch.Tensor
    grp_cnt: torch.Tensor
    tgrp: torch.Tensor
    tgrp_cnt: torch.Tensor
    wmap: torch.Tensor
    vcnt: torch.Tensor
    vidx: torch.Tensor
    tvcnt: torch.Tensor
    tvidx: torch.Tensor
    k_v: int
    k_s: int

    @staticmethod
    def empty(B, nh, N, k_v, k_s, device="cuda"):
        i32 = dict(dtype=torch.int32, device=device)
        W = lib().minf_vs_wmap_words(N)
        return VSIndex(torch.empty(B, nh, k_s, 2, **i32), torch.empty(B, nh, **i32),
                       torch.empty(B, nh, k_s, 2, **i32), torch.empty(B, nh, **i32),
                       torch.empty(B, nh, W, **i32), torch.empty(B, nh, N // 64, **i32),
                       torch.empty(B, nh, N // 64, k_v, **i32), torch.empty(B, nh, N // 128, **i32),
                       torch.empty(B, nh, N // 128, k_v, **i32), k_v, k_s)

    def c(self):
        return _VsIndexC(*(t.data_ptr() for t in (self.grp, self.grp_cnt, self.tgrp, self.tgrp_cnt,
                                                  self.wmap, self.vcnt, self.vidx, self.tvcnt, self.tvidx)))


# ----------------------------------------------------------------- entry points
def minf_estimate_vs(q, k, heads, k_v, k_s, last_q=64, scale=0.0, return_scores=False,
                     ws=None, stream=None):
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    B, N = shp.B, shp.N
    v_idx = torch.empty(B, nh, k_v, dtype=torch.int32, device=q.device)
    s_idx = torch.empty(B, nh, k_s, dtype=torch.int32, device=q.device)
    vs = ss = None
    if return_scores:
        vs = torch.empty(B, nh, N, dtype=torch.float32, device=q.device)
        ss = torch.empty(B, nh, N, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(OP_ESTIMATE_VS, shp, nh, device=q.device)
    _check("minf_estimate_vs", lib().minf_estimate_vs(
        ctypes.byref(shp), _p(q), _p(k), _p(hd), nh, last_q, k_v, k_s, _p(v_idx), _p(s_idx),
        _p(vs), _p(ss), _p(ws), ws.numel(), _stream(stream)))
    return (v_idx, s_idx, vs, ss) if return_scores else (v_idx, s_idx)


def minf_estimate_bs(q, k, heads, k_b, block=64, scale=0.0, return_scores=False, ws=None, stream=None):
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    nb = shp.N // 64
    blk_idx = torch.empty(shp.B, nh, nb, k_b, dtype=torch.int32, device=q.device)
    blk_cnt = torch.empty(shp.B, nh, nb, dtype=torch.int32, device=q.device)
    sc = torch.empty(shp.B, nh, nb, nb, dtype=torch.float32, device=q.device) if return_scores else None
    if ws is None:
        ws = workspace(OP_ESTIMATE_BS, shp, nh, k_b=k_b, device=q.device)
    _check("minf_estimate_bs", lib().minf_estimate_bs(
        ctypes.byref(shp), _p(q), _p(k), _p(hd), nh, block, k_b, _p(blk_idx), _p(blk_cnt), _p(sc),
        _p(ws), ws.numel(), _stream(stream)))
    return (blk_idx, blk_cnt, sc) if return_scores else (blk_idx, blk_cnt)


def minf_build_index(shape: Shape, v_idx, s_idx, index: VSIndex | None = None, ws=None, stream=None):
    B, nh, k_v = v_idx.shape
    k_s = s_idx.shape[2]
    if index is None:
        index = VSIndex.empty(B, nh, shape.N, k_v, k_s, device=v_idx.device)
    if ws is None:
        ws = workspace(OP_BUILD_INDEX, shape, nh, device=v_idx.device)
    ic = index.c()
    _check("minf_build_index", lib().minf_build_index(
        ctypes.byref(shape), nh, _p(v_idx), k_v, _p(s_idx), k_s, ctypes.byref(ic), _p(ws), ws.numel(),
        _stream(stream)))
    return index


@dataclass
class VSExactIndex:
    """Device buffers of the element-exact Vertical-Slash index (see
    minf_vs_exact_index): per 128-row query tile, offset groups of gap 128,
    offset and key bitmaps, and the verticals outside the groups' ranges."""
    tgrp: torch.Tensor
    tgrp_cnt: torch.Tensor
    sbits: torch.Tensor
    vbits: torch.Tensor
    twmap: torch.Tensor
    vcnt: torch.Tensor
    vidx: torch.Tensor
    k_v: int
    k_s: int

    @staticmethod
    def empty(B, nh, N, k_v, k_s, device="cuda"):
        i32 = dict(dtype=torch.int32, device=device)
        Wb, Wt = lib().minf_vs_bits_words(N), lib().minf_vs_twmap_words(N)
        return VSExactIndex(torch.empty(B, nh, k_s, 2, **i32), torch.empty(B, nh, **i32),
                            torch.empty(B, nh, Wb, **i32), torch.empty(B, nh, Wb, **i32),
                            torch.empty(B, nh, Wt, **i32), torch.empty(B, nh, N // 128, **i32),
                            torch.empty(B, nh, N // 128, k_v, **i32), k_v, k_s)

    def c(self):
        return _VsExactIndexC(*(t.data_ptr() for t in (self.tgrp, self.tgrp_cnt, self.sbits, self.vbits,
                                                       self.twmap, self.vcnt, self.vidx)))


def minf_build_index_exact(shape: Shape, v_idx, s_idx, index: VSExactIndex | None = None, ws=None,
                           stream=None):
    B, nh, k_v = v_idx.shape
    k_s = s_idx.shape[2]
    if index is None:
        index = VSExactIndex.empty(B, nh, shape.N, k_v, k_s, device=v_idx.device)
    if ws is None:
        ws = workspace(OP_BUILD_INDEX_EXACT, shape, nh, device=v_idx.device)
    ic = index.c()
    _check("minf_build_index_exact", lib().minf_build_index_exact(
        ctypes.byref(shape), nh, _p(v_idx), k_v, _p(s_idx), k_s, ctypes.byref(ic), _p(ws), ws.numel(),
        _stream(stream)))
    return index


def _out(q, o, lse, want_lse):
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    return o, lse


def minf_sparse_attn_vs(q, k, v, heads, index: VSIndex, o=None, lse=None, want_lse=True, scale=0.0,
                        ws=None, stream=None):
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    o, lse = _out(q, o, lse, want_lse)
    if ws is None:
        ws = workspace(OP_SPARSE_ATTN_VS, shp, nh, device=q.device)
    ic = index.c()
    _check("minf_sparse_attn_vs", lib().minf_sparse_attn_vs(
        ctypes.byref(shp), _p(q), _p(k), _p(v), _p(hd), nh, ctypes.byref(ic), index.k_v, index.k_s,
        _p(o), _p(lse), _p(ws), ws.numel(), _stream(stream)))
    return o, lse


def minf_sparse_attn_vs_exact(q, k, v, heads, index: VSExactIndex, o=None, lse=None, want_lse=True,
                              scale=0.0, ws=None, stream=None):
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    o, lse = _out(q, o, lse, want_lse)
    if ws is None:
        ws = workspace(OP_SPARSE_ATTN_VS_EXACT, shp, nh, device=q.device)
    ic = index.c()
    _check("minf_sparse_attn_vs_exact", lib().minf_sparse_attn_vs_exact(
        ctypes.byref(shp), _p(q), _p(k), _p(v), _p(hd), nh, ctypes.byref(ic), index.k_v, index.k_s,
        _p(o), _p(lse), _p(ws), ws.numel(), _stream(stream)))
    return o, lse


def minf_sparse_attn_bs(q, k, v, heads, blk_idx, blk_cnt, o=None, lse=None, want_lse=True, scale=0.0,
                        ws=None, stream=None):
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    o, lse = _out(q, o, lse, want_lse)
    if ws is None:
        ws = workspace(OP_SPARSE_ATTN_BS, shp, nh, device=q.device)
    _check("minf_sparse_attn_bs", lib().minf_sparse_attn_bs(
        ctypes.byref(shp), _p(q), _p(k), _p(v), _p(hd), nh, _p(blk_idx), _p(blk_cnt), blk_idx.shape[-1],
        _p(o), _p(lse), _p(ws), ws.numel(), _stream(stream)))
    return o, lse


def minf_attn_ashape(q, k, v, heads, n_sink, n_local, o=None, lse=None, want_lse=True, scale=0.0,
                     ws=None, stream=None):
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    o, lse = _out(q, o, lse, want_lse)
    if ws is None:
        ws = workspace(OP_ATTN_ASHAPE, shp, nh, device=q.device)
    _check("minf_attn_ashape", lib().minf_attn_ashape(
        ctypes.byref(shp), _p(q), _p(k), _p(v), _p(hd), nh, n_sink, n_local, _p(o), _p(lse),
        _p(ws), ws.numel(), _stream(stream)))
    return o, lse


def minf_dense_attn(q, k, v, heads=None, o=None, lse=None, want_lse=True, scale=0.0, ws=None, stream=None):
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel() if hd is not None else shp.Hq
    o, lse = _out(q, o, lse, want_lse)
    if ws is None:
        ws = workspace(OP_DENSE_ATTN, shp, nh, device=q.device)
    _check("minf_dense_attn", lib().minf_dense_attn(
        ctypes.byref(shp), _p(q), _p(k), _p(v), _p(hd), nh, _p(o), _p(lse), _p(ws), ws.numel(),
        _stream(stream)))
    return o, lse


def minf_attn_grid(q, k, v, heads, frame_tokens, k_b, o=None, lse=None, want_lse=True, scale=0.0,
                   return_selection=False, ws=None, stream=None):
    """Grid-pattern attention (see include/minf.h): the Block-Sparse
    treatment of each in-frame position's frame sequence.  With
    ``return_selection`` also returns blk_idx [B, P, nh, F/64, k_b] and
    blk_cnt [B, P, nh, F/64]."""
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    o, lse = _out(q, o, lse, want_lse)
    P = int(frame_tokens)
    bi = bc = None
    if return_selection:
        nbf = shp.N // P // 64
        bi = torch.empty(shp.B, P, nh, nbf, k_b, dtype=torch.int32, device=q.device)
        bc = torch.empty(shp.B, P, nh, nbf, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(OP_ATTN_GRID, shp, nh, k_b=k_b, device=q.device)
    _check("minf_attn_grid", lib().minf_attn_grid(
        ctypes.byref(shp), _p(q), _p(k), _p(v), _p(hd), nh, P, k_b, _p(bi), _p(bc), _p(o), _p(lse),
        _p(ws), ws.numel(), _stream(stream)))
    return (o, lse, bi, bc) if return_selection else (o, lse)


def minf_sparse_attn_layer(q, k, v, vs_heads=None, vs_index: VSIndex | None = None, bs_heads=None,
                           blk_idx=None, blk_cnt=None, a_heads=None, n_sink=0, n_local=1, o=None, lse=None,
                           want_lse=True, scale=0.0, ws=None, stream=None):
    """Every head of a mixed-pattern layer in one launch (see
    minf_sparse_attn_layer in include/minf.h); a group whose heads are None or
    empty is left out."""
    shp = shape_of(q, k, scale)
    vh, bh, ah = (_heads(h, q.device) for h in (vs_heads, bs_heads, a_heads))
    nv, nb, na = (0 if h is None else h.numel() for h in (vh, bh, ah))
    o, lse = _out(q, o, lse, want_lse)
    if ws is None:
        ws = workspace(OP_SPARSE_ATTN_LAYER, shp, max(1, nv + nb + na), device=q.device)
    ic = vs_index.c() if (nv and vs_index is not None) else None
    _check("minf_sparse_attn_layer", lib().minf_sparse_attn_layer(
        ctypes.byref(shp), _p(q), _p(k), _p(v), _p(vh) if nv else None, nv,
        ctypes.byref(ic) if ic is not None else None, vs_index.k_v if nv else 0, vs_index.k_s if nv else 0,
        _p(bh) if nb else None, nb, _p(blk_idx) if nb else None, _p(blk_cnt) if nb else None,
        blk_idx.shape[-1] if nb else 0, _p(ah) if na else None, na, n_sink, n_local, _p(o), _p(lse),
        _p(ws), ws.numel(), _stream(stream)))
    return o, lse


def attn_counters(ws):
    """(executed 128 x 128 key tiles, kept score entries) that the attention
    launches on this workspace counted since it was zeroed."""
    c = ws[:24].cpu().view(torch.int64)
    return int(c[1]), int(c[2])


def minf_get_device_status(ws, stream=None):
    return lib().minf_get_device_status(_p(ws), _stream(stream))


def minf_estimate_vs_noalloc(q, k, heads, k_v, k_s, last_q=64, scale=0.0, return_scores=False, stream=None):
    """minf_estimate_vs without a workspace: the library's built-in scratch
    array is used, so this call allocates nothing on the device beyond the
    outputs it is handed here (see include/minf.h for the limits)."""
    L = lib()
    fn = L.minf_estimate_vs_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    shp = shape_of(q, k, scale)
    hd = _heads(heads, q.device)
    nh = hd.numel()
    v_idx = torch.empty(shp.B, nh, k_v, dtype=torch.int32, device=q.device)
    s_idx = torch.empty(shp.B, nh, k_s, dtype=torch.int32, device=q.device)
    vs = ss = None
    if return_scores:
        vs = torch.empty(shp.B, nh, shp.N, dtype=torch.float32, device=q.device)
        ss = torch.empty(shp.B, nh, shp.N, dtype=torch.float32, device=q.device)
    _check("minf_estimate_vs_noalloc", fn(ctypes.byref(shp), _p(q), _p(k), _p(hd), nh, last_q, k_v, k_s,
                                          _p(v_idx), _p(s_idx), _p(vs), _p(ss), _stream(stream)))
    return (v_idx, s_idx, vs, ss) if return_scores else (v_idx, s_idx)


def minf_noalloc_device_status(stream=None):
    """The status word of minf_estimate_vs_noalloc's built-in scratch
    (synchronizes the stream; reading clears it)."""
    fn = lib().minf_noalloc_device_status
    fn.argtypes = [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return int(fn(_stream(stream)))


def minf_selftest_exp2(x, stream=None):
    """The softmax's two exponentials on device floats x: (polynomial, MUFU)."""
    x = x.contiguous().float()
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _check("minf_selftest_exp2", lib().minf_selftest_exp2(_p(x), _p(yp), _p(ym), x.numel(), _stream(stream)))
    return yp, ym
