"""Thin ctypes binding of libmfa.so (argument marshalling only).

Every computation runs in the library's CUDA kernels; this module only turns
torch tensors and mask descriptions into the C structs of ``include/mfa.h``
and calls the entry points of the same names. It raises if the library is
missing or a call fails: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

from . import workloads as W

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmfa.so")

MFA_OK, MFA_ERR_INVALID_ARG, MFA_ERR_UNSUPPORTED, MFA_ERR_SHAPE_MISMATCH, MFA_ERR_CUDA, MFA_ERR_DEVICE = range(6)
MFA_BF16, MFA_F32 = 0, 1
DEVERR_BOUNDS, DEVERR_SEL, DEVERR_TIMEOUT, DEVERR_MAP = 1, 2, 4, 8

EXPORTS = ("mfa_abi_version", "mfa_status_string", "mfa_tile_map_bytes", "mfa_tile_map_init",
           "mfa_build_tile_map", "mfa_fwd", "mfa_fwd_noalloc", "mfa_get_device_status",
           "mfa_mask_from_sparse_mode", "mfa_bwd_workspace_bytes", "mfa_bwd", "mfa_decode_workspace_bytes",
           "mfa_decode", "mfa_fwd_bias", "mfa_test_arm_fwd_timeout")
BIAS_NONE, BIAS_ALIBI, BIAS_ALIBI_SQRT, BIAS_ALIBI_LEFT = 0, 1, 2, 3
NOALLOC_SCRATCH_BYTES = 16 << 20


class MfaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64), ("D", ctypes.c_int64),
                ("stride", ctypes.c_int64 * 4)]


class MfaTileMap(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hm", ctypes.c_int32), ("Nq", ctypes.c_int32), ("Nk", ctypes.c_int32),
                ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32), ("nqt", ctypes.c_int32),
                ("nkt", ctypes.c_int32), ("kind", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("kminmax", ctypes.c_void_p), ("tile_class", ctypes.c_void_p), ("tile_list", ctypes.c_void_p),
                ("tile_count", ctypes.c_void_p), ("order", ctypes.c_void_p), ("err", ctypes.c_void_p)]


class MfaMaskDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("B", ctypes.c_int32), ("Hm", ctypes.c_int32), ("Nq", ctypes.c_int32),
                ("Nk", ctypes.c_int32), ("sel_k", ctypes.c_int32), ("sel_block", ctypes.c_int32),
                ("reserved", ctypes.c_int32),
                ("lts", ctypes.c_void_p), ("lte", ctypes.c_void_p), ("uts", ctypes.c_void_p), ("ute", ctypes.c_void_p),
                ("pre_tokens", ctypes.c_int64), ("next_tokens", ctypes.c_int64),
                ("sel", ctypes.c_void_p), ("map", ctypes.POINTER(MfaTileMap))]


class MfaSparseMode(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("pre_tokens", ctypes.c_int64), ("next_tokens", ctypes.c_int64),
                ("prefix", ctypes.c_void_p), ("seq_q", ctypes.c_void_p), ("seq_kv", ctypes.c_void_p),
                ("n_seq", ctypes.c_int32), ("reserved2", ctypes.c_int32)]


class MfaBias(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("reserved", ctypes.c_int32), ("slopes", ctypes.c_void_p)]


class MfaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} returned {status} ({msg})")
        self.status = status


_lib: Optional[ctypes.CDLL] = None


def load(path: str = _LIB_PATH) -> ctypes.CDLL:
    """Load libmfa.so (built in-tree by mask_aware_block_mfa_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: run `python -m mask_aware_block_mfa_b200.build`")
    lib = ctypes.CDLL(path)
    lib.mfa_abi_version.restype = ctypes.c_int32
    lib.mfa_status_string.restype = ctypes.c_char_p
    lib.mfa_status_string.argtypes = [ctypes.c_int]
    lib.mfa_tile_map_bytes.restype = ctypes.c_size_t
    lib.mfa_tile_map_bytes.argtypes = [ctypes.c_int32] * 6
    lib.mfa_tile_map_init.restype = ctypes.c_int
    lib.mfa_tile_map_init.argtypes = [ctypes.POINTER(MfaTileMap), ctypes.c_void_p, ctypes.c_size_t] + [ctypes.c_int32] * 6
    lib.mfa_build_tile_map.restype = ctypes.c_int
    lib.mfa_build_tile_map.argtypes = [ctypes.POINTER(MfaMaskDesc), ctypes.POINTER(MfaTileMap), ctypes.c_void_p]
    lib.mfa_fwd.restype = ctypes.c_int
    lib.mfa_fwd.argtypes = [ctypes.POINTER(MfaTensor)] * 3 + [ctypes.POINTER(MfaMaskDesc), ctypes.POINTER(MfaTensor),
                                                              ctypes.c_void_p, ctypes.c_void_p]
    lib.mfa_fwd_noalloc.restype = ctypes.c_int
    lib.mfa_fwd_noalloc.argtypes = [ctypes.POINTER(MfaTensor)] * 3 + [ctypes.POINTER(MfaMaskDesc), ctypes.c_int32,
                                                                      ctypes.c_int32, ctypes.POINTER(MfaTensor),
                                                                      ctypes.c_void_p, ctypes.c_void_p,
                                                                      ctypes.c_void_p]
    lib.mfa_get_device_status.restype = ctypes.c_int
    lib.mfa_get_device_status.argtypes = [ctypes.POINTER(MfaTileMap), ctypes.c_void_p,
                                          ctypes.POINTER(ctypes.c_uint32)]
    lib.mfa_mask_from_sparse_mode.restype = ctypes.c_int
    lib.mfa_mask_from_sparse_mode.argtypes = [ctypes.POINTER(MfaSparseMode)] + [ctypes.c_int32] * 3 + \
        [ctypes.c_void_p] * 4 + [ctypes.POINTER(MfaMaskDesc), ctypes.c_void_p]
    lib.mfa_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.mfa_bwd_workspace_bytes.argtypes = [ctypes.c_int32] * 5
    lib.mfa_bwd.restype = ctypes.c_int
    lib.mfa_bwd.argtypes = [ctypes.POINTER(MfaTensor)] * 5 + [ctypes.c_void_p, ctypes.POINTER(MfaMaskDesc)] + \
        [ctypes.POINTER(MfaTensor)] * 3 + [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    lib.mfa_fwd_bias.restype = ctypes.c_int
    lib.mfa_fwd_bias.argtypes = [ctypes.POINTER(MfaTensor)] * 3 + [ctypes.POINTER(MfaMaskDesc),
                                                                   ctypes.POINTER(MfaBias),
                                                                   ctypes.POINTER(MfaTensor), ctypes.c_void_p,
                                                                   ctypes.c_void_p]
    lib.mfa_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.mfa_decode_workspace_bytes.argtypes = [ctypes.c_int32] * 7
    lib.mfa_decode.restype = ctypes.c_int
    lib.mfa_decode.argtypes = [ctypes.POINTER(MfaTensor)] * 3 + [ctypes.c_void_p, ctypes.c_int32,
                                                                 ctypes.POINTER(MfaTensor), ctypes.c_void_p,
                                                                 ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t,
                                                                 ctypes.c_void_p, ctypes.c_void_p]
    lib.mfa_test_arm_fwd_timeout.restype = ctypes.c_int
    lib.mfa_test_arm_fwd_timeout.argtypes = [ctypes.c_uint32]
    if lib.mfa_abi_version() != 1:
        raise RuntimeError("libmfa.so ABI version mismatch")
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().mfa_status_string(code).decode()


def _check(fn: str, code: int) -> None:
    if code != MFA_OK:
        raise MfaError(fn, code, status_string(code))


def _on_device(name: str, t, device=None, dtype=None, shape=None, contiguous=False) -> None:
    """Host-side checks of a tensor handed to the library as a raw device
    pointer: a CUDA tensor, on `device` when given, with the dtype, shape and
    layout the call reads or writes (the C ABI cannot check these for plain
    pointers, and a host pointer would fault the kernel)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call runs on {device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_lse(lse, q) -> None:
    _on_device("lse", lse, q.device, torch.float32, tuple(q.shape[:3]), contiguous=True)


def _dev(q):
    """The device of the call (q's), after checking that q is a CUDA tensor."""
    _on_device("q", q)
    return q.device


def _same_device(q, *holders) -> None:
    """The device arrays of masks and tile maps must live on q's device."""
    for h in holders:
        ts = [getattr(h, "buf", None), getattr(h, "bounds", None)] + list(getattr(h, "_keep", []))
        for t in ts:
            if isinstance(t, torch.Tensor) and t.device != q.device:
                raise ValueError(f"a mask or tile-map array is on {t.device}, q on {q.device}")


def tensor_desc(t: torch.Tensor, device=None) -> MfaTensor:
    _on_device("tensor", t, device)
    if t.dim() != 4:
        raise ValueError("expected a [B, H, N, D] tensor")
    dt = {torch.bfloat16: MFA_BF16, torch.float32: MFA_F32}.get(t.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {t.dtype}")
    d = MfaTensor()
    d.data = t.data_ptr()
    d.dtype = dt
    d.B, d.H, d.N, d.D = (int(x) for x in t.shape)
    for i in range(4):
        d.stride[i] = int(t.stride(i))
    return d


def _stream_ptr(stream, device=None) -> int:
    """The raw handle of `stream`, by default the current stream of `device`.
    A stream of another device is rejected: the library launches on the
    current device, which every wrapper below sets to the tensors' device."""
    if device is not None:
        device = torch.device(device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and device.type == "cuda" and stream.device != device:
        raise ValueError(f"the stream is on {stream.device}, the call runs on {device}")
    return int(stream.cuda_stream)


def _on(device):
    """Make `device` current for the duration of one library call (the C ABI
    launches on the current device and looks up per-device state there)."""
    return torch.cuda.device(torch.device(device))


class DeviceMask:
    """A mask description whose arrays live on the device, plus its C struct."""

    def __init__(self, mask: W.MaskDesc, device="cuda"):
        self.mask = mask
        self.kind, self.B, self.Hm, self.Nq, self.Nk = mask.kind, mask.B, mask.Hm, mask.Nq, mask.Nk
        self._keep = []
        d = MfaMaskDesc()
        d.kind, d.B, d.Hm, d.Nq, d.Nk = mask.kind, mask.B, mask.Hm, mask.Nq, mask.Nk
        d.sel_k, d.sel_block = mask.sel_k, mask.sel_block
        for f in ("lts", "lte", "uts", "ute", "sel"):
            a = getattr(mask, f)
            if a is None:
                setattr(d, f, None)
                continue
            t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
            self._keep.append(t)
            setattr(d, f, t.data_ptr())
        d.pre_tokens, d.next_tokens = int(mask.pre_tokens), int(mask.next_tokens)
        d.map = None
        self.desc = d


class SparseModeMask:
    """An Ascend sparse mode turned into a device mask description by
    mfa_mask_from_sparse_mode (band modes on the host, prefix and varlen modes
    by a kernel into column-wise bounds owned here). Usable wherever a
    DeviceMask is (build_tile_map, fwd, Attention)."""

    def __init__(self, mode: int, B: int, Nq: int, Nk: int, pre_tokens: int = 0, next_tokens: int = 0,
                 prefix=None, seq_q=None, seq_kv=None, device="cuda", stream=None):
        self.B, self.Hm, self.Nq, self.Nk = B, 1, Nq, Nk
        self._keep = []
        sm = MfaSparseMode()
        sm.mode, sm.pre_tokens, sm.next_tokens = mode, int(pre_tokens), int(next_tokens)

        def dev64(a):
            if a is None:
                return None
            t = torch.as_tensor(np.asarray(a, dtype=np.int64)).to(device)
            self._keep.append(t)
            return t.data_ptr()

        sm.prefix, sm.seq_q, sm.seq_kv = dev64(prefix), dev64(seq_q), dev64(seq_kv)
        sm.n_seq = 0 if seq_q is None else len(seq_q)
        self.sm = sm
        self.bounds = torch.empty(4, max(B, 1), 1, max(Nk, 1), dtype=torch.int32, device=device)
        self.desc = MfaMaskDesc()
        self.convert(stream)
        self.kind = self.desc.kind

    def convert(self, stream=None) -> None:
        """(Re)write the description, and for modes 5-8 the bounds, from the
        mode's inputs already on the device (no allocation, graph-capturable)."""
        ptrs = [self.bounds[i].data_ptr() for i in range(4)]  # lts, lte, uts, ute
        dev = self.bounds.device
        with _on(dev):
            _check("mfa_mask_from_sparse_mode",
                   load().mfa_mask_from_sparse_mode(ctypes.byref(self.sm), self.B, self.Nq, self.Nk, *ptrs,
                                                    ctypes.byref(self.desc), _stream_ptr(stream, dev)))


class TileMap:
    """A tile map in one caller-owned device buffer (see mfa_tile_map in mfa.h)."""

    def __init__(self, B, Hm, Nq, Nk, block_q, block_k, device="cuda"):
        lib = load()
        nbytes = lib.mfa_tile_map_bytes(B, Hm, Nq, Nk, block_q, block_k)
        if nbytes == 0:
            raise MfaError("mfa_tile_map_bytes", MFA_ERR_INVALID_ARG, "bad shape or block sizes")
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        aligned = (base + 255) & ~255
        self.m = MfaTileMap()
        _check("mfa_tile_map_init", lib.mfa_tile_map_init(ctypes.byref(self.m), aligned, nbytes,
                                                          B, Hm, Nq, Nk, block_q, block_k))
        self.offset = aligned - base
        self.nbytes = nbytes

    def arrays(self):
        """Views of the map arrays as torch tensors on the device."""
        m = self.m
        BH, nqt, nkt = m.B * m.Hm, m.nqt, m.nkt

        def view(ptr, dtype, count):
            off = ptr - self.buf.data_ptr()
            el = torch.tensor([], dtype=dtype).element_size()
            return self.buf[off:off + count * el].view(dtype)

        return {
            "kminmax": view(m.kminmax, torch.int32, BH * nkt * 8).view(m.B, m.Hm, nkt, 8),
            "tile_class": view(m.tile_class, torch.uint8, BH * nqt * nkt).view(m.B, m.Hm, nqt, nkt),
            "tile_list": view(m.tile_list, torch.int32, BH * nqt * nkt).view(m.B, m.Hm, nqt, nkt),
            "tile_count": view(m.tile_count, torch.int32, BH * nqt).view(m.B, m.Hm, nqt),
            "order": view(m.order, torch.int32, BH * nqt),
            "err": view(m.err, torch.int32, 1),
        }


def build_tile_map(dmask: DeviceMask, tmap: TileMap, stream=None) -> None:
    dev = tmap.buf.device
    _same_device(tmap.buf, dmask)
    with _on(dev):
        _check("mfa_build_tile_map", load().mfa_build_tile_map(ctypes.byref(dmask.desc), ctypes.byref(tmap.m),
                                                               _stream_ptr(stream, dev)))


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dmask: DeviceMask, tmap: TileMap,
        out: torch.Tensor, lse: torch.Tensor, stream=None) -> None:
    """out, lse <- attention(q, k, v) under dmask, through the tile map (both on the device)."""
    qd, kd, vd, od = (tensor_desc(t, _dev(q)) for t in (q, k, v, out))
    _check_lse(lse, q)
    _same_device(q, tmap, dmask)
    dmask.desc.map = ctypes.pointer(tmap.m)
    with _on(q.device):
        _check("mfa_fwd", load().mfa_fwd(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd),
                                         ctypes.byref(dmask.desc), ctypes.byref(od), lse.data_ptr(),
                                         _stream_ptr(stream, q.device)))


def fwd_bias(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dmask, tmap: TileMap, kind: int,
             slopes: torch.Tensor, out: torch.Tensor, lse: torch.Tensor, stream=None) -> None:
    """Forward pass with an additive ALiBi bias (kind BIAS_*, slopes: float32 device tensor [Hq])."""
    qd, kd, vd, od = (tensor_desc(t, _dev(q)) for t in (q, k, v, out))
    _check_lse(lse, q)
    _on_device("slopes", slopes, q.device, torch.float32, (int(q.shape[1]),), contiguous=True)
    _same_device(q, tmap, dmask)
    dmask.desc.map = ctypes.pointer(tmap.m)
    bias = MfaBias(kind, 0, slopes.data_ptr())
    with _on(q.device):
        _check("mfa_fwd_bias", load().mfa_fwd_bias(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd),
                                                   ctypes.byref(dmask.desc), ctypes.byref(bias), ctypes.byref(od),
                                                   lse.data_ptr(), _stream_ptr(stream, q.device)))


def fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dmask: DeviceMask, block_q: int, block_k: int,
                out: torch.Tensor, lse: torch.Tensor, dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    """Forward pass with the tile map in the library's own device array (no allocation by anyone)."""
    qd, kd, vd, od = (tensor_desc(t, _dev(q)) for t in (q, k, v, out))
    _check_lse(lse, q)
    if dev_err is not None:
        _on_device("dev_err", dev_err, q.device)
        if dev_err.numel() * dev_err.element_size() < 4:
            raise ValueError("dev_err must hold at least 4 bytes")
    _same_device(q, dmask)
    err_ptr = None if dev_err is None else dev_err.data_ptr()
    # The library picks its scratch array and launches on the current device.
    with _on(q.device):
        _check("mfa_fwd_noalloc", load().mfa_fwd_noalloc(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd),
                                                         ctypes.byref(dmask.desc), block_q, block_k,
                                                         ctypes.byref(od), lse.data_ptr(), err_ptr,
                                                         _stream_ptr(stream, q.device)))


def bwd_workspace_bytes(B: int, Hq: int, Nq: int, Nk: int, D: int) -> int:
    return int(load().mfa_bwd_workspace_bytes(B, Hq, Nq, Nk, D))


def bwd(q, k, v, out, dout, lse, dmask, tmap: TileMap, dq, dk, dv, workspace: torch.Tensor, stream=None) -> None:
    """dq, dk, dv <- gradients of attention(q, k, v) under dmask for the output
    gradient dout (out, lse from the forward pass; the map built with 128-key
    tiles); workspace is a uint8 device tensor of bwd_workspace_bytes()."""
    ds = [tensor_desc(t, _dev(q)) for t in (q, k, v, out, dout, dq, dk, dv)]
    _check_lse(lse, q)
    _on_device("workspace", workspace, q.device, torch.uint8, contiguous=True)
    _same_device(q, tmap, dmask)
    dmask.desc.map = ctypes.pointer(tmap.m)
    with _on(q.device):
        _check("mfa_bwd", load().mfa_bwd(*(ctypes.byref(d) for d in ds[:5]), lse.data_ptr(),
                                         ctypes.byref(dmask.desc), *(ctypes.byref(d) for d in ds[5:]),
                                         workspace.data_ptr(), workspace.numel(), _stream_ptr(stream, q.device)))


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, Nq: int, D: int, sel_k: int, n_split: int = 0) -> int:
    return int(load().mfa_decode_workspace_bytes(B, Hq, Hkv, Nq, D, sel_k, n_split))


class Decode:
    """Selected-key attention for a few query rows (mfa_decode): keeps the
    split-K workspace and the device error word between calls."""

    def __init__(self, n_split: int = 0):
        self.n_split = n_split
        self.ws = None
        self.err = None

    def __call__(self, q, k, v, sel, out=None, lse=None, stream=None):
        """sel: int32 device tensor [B, Hkv, Nq, sel_k] of 64-key block indices (-1 = none)."""
        qd, kd, vd = (tensor_desc(t, _dev(q)) for t in (q, k, v))
        B_, Hq, Nq, D = q.shape
        Hkv = int(k.shape[1])
        if sel.dim() != 4:
            raise ValueError("sel must be a [B, Hkv, Nq, sel_k] tensor")
        sel_k = int(sel.shape[-1])
        _on_device("sel", sel, q.device, torch.int32, (B_, Hkv, Nq, sel_k), contiguous=True)
        need = decode_workspace_bytes(B_, Hq, Hkv, Nq, D, sel_k, self.n_split)
        if need == 0:
            raise ValueError("invalid decode sizes")
        if self.ws is None or self.ws.numel() < need or self.ws.device != q.device:
            self.ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        if self.err is None or self.err.device != q.device:
            self.err = torch.zeros(1, dtype=torch.int32, device=q.device)
        out = torch.empty_like(q) if out is None else out
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if lse is None else lse
        od = tensor_desc(out, q.device)
        _check_lse(lse, q)
        with _on(q.device):
            _check("mfa_decode", load().mfa_decode(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd),
                                                   sel.data_ptr(), sel_k, ctypes.byref(od), lse.data_ptr(),
                                                   self.n_split, self.ws.data_ptr(), self.ws.numel(),
                                                   self.err.data_ptr(), _stream_ptr(stream, q.device)))
        return out, lse

    def status(self) -> int:
        """Synchronise and return the device error bits (0 = none)."""
        torch.cuda.synchronize()
        return 0 if self.err is None else int(self.err.item())


def arm_fwd_timeout_test(wait_us: int) -> None:
    """Test hook: the next bf16 forward launch withholds one K tile and uses a
    wait limit of wait_us microseconds, so one bounded wait runs out (see
    mfa_test_arm_fwd_timeout in mfa.h)."""
    _check("mfa_test_arm_fwd_timeout", load().mfa_test_arm_fwd_timeout(int(wait_us)))


def device_status(tmap: TileMap, stream=None) -> int:
    """Synchronise and return the map's device error bits (0 = none)."""
    bits = ctypes.c_uint32(0)
    dev = tmap.buf.device
    with _on(dev):
        code = load().mfa_get_device_status(ctypes.byref(tmap.m), _stream_ptr(stream, dev), ctypes.byref(bits))
    if code not in (MFA_OK, MFA_ERR_DEVICE):
        _check("mfa_get_device_status", code)
    return int(bits.value)


class Attention:
    """Convenience wrapper: upload a mask, build its map once, run forward passes."""

    def __init__(self, mask, block_q: int = 64, block_k: int = 128, device="cuda"):
        # a workloads.MaskDesc (uploaded here) or a mask already on the device
        self.dmask = DeviceMask(mask, device) if isinstance(mask, W.MaskDesc) else mask
        self.tmap = TileMap(mask.B, mask.Hm, mask.Nq, mask.Nk, block_q, block_k, device)
        self.device = device

    def build(self, stream=None):
        build_tile_map(self.dmask, self.tmap, stream)

    def __call__(self, q, k, v, out=None, lse=None, stream=None, bias=None):
        """bias: None or (kind, slopes) with kind one of BIAS_* and slopes a float32 device tensor [Hq]."""
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        if bias is None:
            fwd(q, k, v, self.dmask, self.tmap, out, lse, stream)
        else:
            fwd_bias(q, k, v, self.dmask, self.tmap, bias[0], bias[1], out, lse, stream)
        return out, lse

    def backward(self, q, k, v, out, lse, dout, dq=None, dk=None, dv=None, stream=None):
        """Gradients for the output gradient dout (the map must use 128-key tiles)."""
        B_, Hq, Nq, D = q.shape
        need = bwd_workspace_bytes(B_, Hq, Nq, int(k.shape[2]), D)
        if need == 0:
            raise ValueError("invalid shapes for the backward pass")
        ws = getattr(self, "_bwd_ws", None)
        if ws is None or ws.numel() < need or ws.device != q.device:
            ws = self._bwd_ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        bwd(q, k, v, out, dout, lse, self.dmask, self.tmap, dq, dk, dv, ws, stream)
        return dq, dk, dv
