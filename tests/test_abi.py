"""The C ABI on the host: exports, struct layouts and argument validation.

Nothing here touches a GPU: every call below is rejected by host-side checks
before the library makes a CUDA call, or only carves pointers.
"""
import ctypes
import os
import re
import subprocess

import pytest

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mfa.h")


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mfa_[a-z_]+)\s*\(", text)))


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(B.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", BUILD.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (mfa_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)


def test_struct_layouts_match_header(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(r'''
#include <stdio.h>
#include <stddef.h>
#include "mfa.h"
#define F(T, f) printf(#T "." #f " %zu\n", offsetof(T, f))
int main(void) {
  printf("mfa_tensor %zu\nmfa_tile_map %zu\nmfa_mask_desc %zu\nmfa_sparse_mode %zu\nmfa_bias %zu\n",
         sizeof(mfa_tensor), sizeof(mfa_tile_map), sizeof(mfa_mask_desc), sizeof(mfa_sparse_mode),
         sizeof(mfa_bias));
  F(mfa_bias, kind); F(mfa_bias, slopes);
  F(mfa_sparse_mode, pre_tokens); F(mfa_sparse_mode, prefix); F(mfa_sparse_mode, seq_kv); F(mfa_sparse_mode, n_seq);
  F(mfa_tensor, data); F(mfa_tensor, B); F(mfa_tensor, stride);
  F(mfa_tile_map, kind); F(mfa_tile_map, kminmax); F(mfa_tile_map, err);
  F(mfa_mask_desc, lts); F(mfa_mask_desc, pre_tokens); F(mfa_mask_desc, sel); F(mfa_mask_desc, map);
  return 0;
}''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines())
    assert int(got["mfa_tensor"]) == ctypes.sizeof(B.MfaTensor)
    assert int(got["mfa_tile_map"]) == ctypes.sizeof(B.MfaTileMap)
    assert int(got["mfa_mask_desc"]) == ctypes.sizeof(B.MfaMaskDesc)
    assert int(got["mfa_sparse_mode"]) == ctypes.sizeof(B.MfaSparseMode)
    assert int(got["mfa_bias"]) == ctypes.sizeof(B.MfaBias)
    for key, val in got.items():
        if "." in key:
            struct, field = key.split(".")
            cls = {"mfa_tensor": B.MfaTensor, "mfa_tile_map": B.MfaTileMap, "mfa_mask_desc": B.MfaMaskDesc,
                   "mfa_sparse_mode": B.MfaSparseMode, "mfa_bias": B.MfaBias}[struct]
            assert getattr(cls, field).offset == int(val), key


def test_status_strings(lib):
    assert lib.mfa_abi_version() == 1
    for code in range(6):
        assert lib.mfa_status_string(code)
    assert lib.mfa_status_string(99) == b"unknown status"


def test_tile_map_bytes_and_init(lib):
    assert lib.mfa_tile_map_bytes(1, 1, 8192, 8192, 64, 128) > 0
    assert lib.mfa_tile_map_bytes(1, 1, 8192, 8192, 32, 128) == 0
    assert lib.mfa_tile_map_bytes(0, 1, 8192, 8192, 64, 128) == 0
    nb = lib.mfa_tile_map_bytes(2, 1, 1000, 900, 64, 64)
    nqt, nkt = 16, 15
    expect = 0
    for sz in (2 * nkt * 8 * 4, 2 * nqt * nkt, 2 * nqt * nkt * 4, 2 * nqt * 4, 2 * nqt * 4, 4):
        expect += (sz + 255) // 256 * 256
    assert nb == expect
    m = B.MfaTileMap()
    fake = 0x7000_0000_0000
    assert lib.mfa_tile_map_init(ctypes.byref(m), fake, nb, 2, 1, 1000, 900, 64, 64) == B.MFA_OK
    assert (m.nqt, m.nkt, m.kind) == (nqt, nkt, -1)
    assert m.kminmax == fake and m.err > m.order > m.tile_count > m.tile_list > m.tile_class > m.kminmax
    assert all(p % 256 == 0 for p in (m.kminmax, m.tile_class, m.tile_list, m.tile_count, m.order, m.err))
    assert lib.mfa_tile_map_init(ctypes.byref(m), fake, nb - 1, 2, 1, 1000, 900, 64, 64) == B.MFA_ERR_INVALID_ARG
    assert lib.mfa_tile_map_init(ctypes.byref(m), fake + 16, nb, 2, 1, 1000, 900, 64, 64) == B.MFA_ERR_INVALID_ARG
    assert lib.mfa_tile_map_init(ctypes.byref(m), None, nb, 2, 1, 1000, 900, 64, 64) == B.MFA_ERR_INVALID_ARG
    assert lib.mfa_tile_map_init(ctypes.byref(m), fake, nb, 2, 1, 1000, 900, 96, 64) == B.MFA_ERR_UNSUPPORTED


def _fake_map(lib, Bsz=1, Hm=1, Nq=512, Nk=512, bq=64, bk=128, kind=0):
    m = B.MfaTileMap()
    nb = lib.mfa_tile_map_bytes(Bsz, Hm, Nq, Nk, bq, bk)
    assert lib.mfa_tile_map_init(ctypes.byref(m), 0x7000_0000_0000, nb, Bsz, Hm, Nq, Nk, bq, bk) == 0
    m.kind = kind
    return m


def _fake_tensor(Bsz, H, N, D, dtype=B.MFA_BF16, addr=0x7100_0000_0000):
    t = B.MfaTensor()
    t.data, t.dtype = addr, dtype
    t.B, t.H, t.N, t.D = Bsz, H, N, D
    t.stride[0], t.stride[1], t.stride[2], t.stride[3] = H * N * D, N * D, D, 1
    return t


def _fake_mask(m, kind=0, Bsz=1, Hm=1, Nq=512, Nk=512):
    d = B.MfaMaskDesc()
    d.kind, d.B, d.Hm, d.Nq, d.Nk = kind, Bsz, Hm, Nq, Nk
    d.sel_block = 64
    d.map = ctypes.pointer(m)
    return d


def _fwd(lib, q, k, v, d, o, lse=0x7200_0000_0000):
    return lib.mfa_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(d), ctypes.byref(o),
                       lse, None)


def test_fwd_rejects_bad_arguments_on_host(lib):
    m = _fake_map(lib)
    q, k, v, o = _fake_tensor(1, 8, 512, 128), _fake_tensor(1, 2, 512, 128), _fake_tensor(1, 2, 512, 128), \
        _fake_tensor(1, 8, 512, 128)
    d = _fake_mask(m)
    assert _fwd(lib, q, k, v, d, o, lse=0) == B.MFA_ERR_INVALID_ARG
    qn = _fake_tensor(1, 8, 512, 128, addr=0)
    assert _fwd(lib, qn, k, v, d, o) == B.MFA_ERR_INVALID_ARG
    q32 = _fake_tensor(1, 8, 512, 128, dtype=B.MFA_F32)
    o32 = _fake_tensor(1, 8, 512, 128, dtype=B.MFA_F32)
    k32, v32 = _fake_tensor(1, 2, 512, 128, dtype=B.MFA_F32), _fake_tensor(1, 2, 512, 128, dtype=B.MFA_F32)
    assert _fwd(lib, q32, k, v, d, o) == B.MFA_ERR_INVALID_ARG                # mixed dtypes
    assert _fwd(lib, _fake_tensor(1, 8, 512, 96), _fake_tensor(1, 2, 512, 96), _fake_tensor(1, 2, 512, 96), d,
                _fake_tensor(1, 8, 512, 96)) == B.MFA_ERR_UNSUPPORTED         # head dim 96
    assert _fwd(lib, q, _fake_tensor(1, 3, 512, 128), _fake_tensor(1, 3, 512, 128), d, o) == \
        B.MFA_ERR_SHAPE_MISMATCH                                              # Hq % Hkv != 0
    assert _fwd(lib, q, k, _fake_tensor(1, 2, 256, 128), d, o) == B.MFA_ERR_SHAPE_MISMATCH
    assert _fwd(lib, q, k, v, d, _fake_tensor(1, 8, 256, 128)) == B.MFA_ERR_SHAPE_MISMATCH
    bad_stride = _fake_tensor(1, 8, 512, 128)
    bad_stride.stride[3] = 2
    assert _fwd(lib, bad_stride, k, v, d, o) == B.MFA_ERR_UNSUPPORTED
    unaligned = _fake_tensor(1, 8, 512, 128, addr=0x7100_0000_0002)
    assert _fwd(lib, unaligned, k, v, d, o) == B.MFA_ERR_UNSUPPORTED
    # mask / map disagreements
    d2 = _fake_mask(m, Nq=256)
    assert _fwd(lib, q, k, v, d2, o) == B.MFA_ERR_SHAPE_MISMATCH
    d3 = _fake_mask(m, kind=1)                                                # map built from another kind
    assert _fwd(lib, q, k, v, d3, o) == B.MFA_ERR_SHAPE_MISMATCH
    d4 = _fake_mask(m)
    d4.map = None
    assert _fwd(lib, q, k, v, d4, o) == B.MFA_ERR_INVALID_ARG
    # two heads per tile (block_q = 64) need an even group size and one mask head
    q6 = _fake_tensor(1, 6, 512, 128)
    k6, v6 = _fake_tensor(1, 2, 512, 128), _fake_tensor(1, 2, 512, 128)
    assert _fwd(lib, q6, k6, v6, d, _fake_tensor(1, 6, 512, 128)) == B.MFA_ERR_UNSUPPORTED
    m8 = _fake_map(lib, Hm=8)
    d8 = _fake_mask(m8, Hm=8)
    assert _fwd(lib, q, k, v, d8, o) == B.MFA_ERR_UNSUPPORTED
    m3 = _fake_map(lib, Hm=3, bq=128)
    assert _fwd(lib, q, k, v, _fake_mask(m3, Hm=3), o) == B.MFA_ERR_SHAPE_MISMATCH  # Hm not in {1, Hq}


def test_build_rejects_bad_arguments_on_host(lib):
    m = _fake_map(lib)
    d = _fake_mask(m)
    assert lib.mfa_build_tile_map(None, ctypes.byref(m), None) == B.MFA_ERR_INVALID_ARG
    assert lib.mfa_build_tile_map(ctypes.byref(d), None, None) == B.MFA_ERR_INVALID_ARG
    bad = _fake_mask(m, kind=7)
    assert lib.mfa_build_tile_map(ctypes.byref(bad), ctypes.byref(m), None) == B.MFA_ERR_INVALID_ARG
    other = _fake_mask(m, Nk=256)
    assert lib.mfa_build_tile_map(ctypes.byref(other), ctypes.byref(m), None) == B.MFA_ERR_SHAPE_MISMATCH
    sel = _fake_mask(m, kind=2)
    assert lib.mfa_build_tile_map(ctypes.byref(sel), ctypes.byref(m), None) == B.MFA_ERR_INVALID_ARG  # no list
    sel.sel, sel.sel_k, sel.sel_block = 0x7300_0000_0000, 16, 32
    assert lib.mfa_build_tile_map(ctypes.byref(sel), ctypes.byref(m), None) == B.MFA_ERR_UNSUPPORTED
    m.tile_list = None
    assert lib.mfa_build_tile_map(ctypes.byref(d), ctypes.byref(m), None) == B.MFA_ERR_INVALID_ARG


def test_bwd_workspace_bytes(lib):
    n = lib.mfa_bwd_workspace_bytes(1, 8, 1000, 900, 128)
    # fp32 dq accumulator + lse2/Delta padded to 64-row tiles + transposed lists
    assert n >= 1 * 8 * 1000 * 128 * 4 + 2 * 8 * 1024 * 4 + 8 * 16 * 4
    assert n % 256 == 0
    assert lib.mfa_bwd_workspace_bytes(0, 8, 1000, 900, 128) == 0
    assert lib.mfa_bwd_workspace_bytes(1, 8, -1, 900, 128) == 0


def test_bwd_rejects_bad_arguments_on_host(lib):
    """Every call here fails validation on the host (the pointers are fake, so
    nothing may be launched)."""
    m = _fake_map(lib)
    q, k, v = _fake_tensor(1, 8, 512, 128), _fake_tensor(1, 2, 512, 128), _fake_tensor(1, 2, 512, 128)
    o, do, dq = _fake_tensor(1, 8, 512, 128), _fake_tensor(1, 8, 512, 128), _fake_tensor(1, 8, 512, 128)
    dk, dv = _fake_tensor(1, 2, 512, 128), _fake_tensor(1, 2, 512, 128)
    d = _fake_mask(m)
    ws_bytes = lib.mfa_bwd_workspace_bytes(1, 8, 512, 512, 128)
    ws = 0x7300_0000_0000

    def call(q=q, k=k, v=v, o=o, do=do, lse=0x7200_0000_0000, d=d, dq=dq, dk=dk, dv=dv, ws=ws, nbytes=ws_bytes):
        return lib.mfa_bwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(o), ctypes.byref(do),
                           lse, ctypes.byref(d), ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), ws, nbytes,
                           None)

    assert call(lse=0) == B.MFA_ERR_INVALID_ARG
    assert call(ws=0) == B.MFA_ERR_INVALID_ARG
    assert call(nbytes=ws_bytes - 256) == B.MFA_ERR_INVALID_ARG               # workspace too small
    assert call(ws=ws + 16) == B.MFA_ERR_INVALID_ARG                          # not 256-byte aligned
    assert call(q=_fake_tensor(1, 8, 512, 128, dtype=B.MFA_F32)) == B.MFA_ERR_UNSUPPORTED
    assert call(dk=_fake_tensor(1, 2, 256, 128)) == B.MFA_ERR_SHAPE_MISMATCH
    assert call(do=_fake_tensor(1, 8, 256, 128)) == B.MFA_ERR_SHAPE_MISMATCH
    assert call(k=_fake_tensor(1, 3, 512, 128), v=_fake_tensor(1, 3, 512, 128), dk=_fake_tensor(1, 3, 512, 128),
                dv=_fake_tensor(1, 3, 512, 128)) == B.MFA_ERR_SHAPE_MISMATCH     # Hq % Hkv != 0
    d64 = [_fake_tensor(1, h, 512, 64) for h in (8, 2, 2, 8, 8, 8, 2, 2)]
    assert call(*d64[:5], d=d, dq=d64[5], dk=d64[6], dv=d64[7]) == B.MFA_ERR_UNSUPPORTED   # head dim 64
    m64 = _fake_map(lib, bq=64, bk=64)
    assert call(d=_fake_mask(m64)) == B.MFA_ERR_UNSUPPORTED                    # 64-key map tiles
    m8 = _fake_map(lib, Hm=8)
    assert call(d=_fake_mask(m8, Hm=8)) == B.MFA_ERR_UNSUPPORTED               # one mask per head
    dn = _fake_mask(m)
    dn.map = None
    assert call(d=dn) == B.MFA_ERR_INVALID_ARG
    assert call(d=_fake_mask(m, kind=1)) == B.MFA_ERR_SHAPE_MISMATCH          # map built from another kind
    bad = _fake_tensor(1, 8, 512, 128)
    bad.stride[3] = 2
    assert call(dq=bad) == B.MFA_ERR_UNSUPPORTED


def test_decode_rejects_bad_arguments_on_host(lib):
    """Every call here fails validation on the host (fake pointers: nothing may be launched)."""
    q, k, v, o = _fake_tensor(1, 8, 1, 256), _fake_tensor(1, 2, 4096, 256), _fake_tensor(1, 2, 4096, 256), \
        _fake_tensor(1, 8, 1, 256)
    sel, lse, ws, err = 0x7400_0000_0000, 0x7200_0000_0000, 0x7300_0000_0000, 0x7500_0000_0000
    need = lib.mfa_decode_workspace_bytes(1, 8, 2, 1, 256, 16, 4)
    assert need > 256 and need % 256 == 0
    assert lib.mfa_decode_workspace_bytes(1, 8, 3, 1, 256, 16, 4) == 0          # Hq % Hkv != 0

    def call(q=q, k=k, v=v, sel=sel, sel_k=16, o=o, lse=lse, n_split=4, ws=ws, nbytes=need, err=err):
        return lib.mfa_decode(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), sel, sel_k, ctypes.byref(o), lse,
                              n_split, ws, nbytes, err, None)

    assert call(err=0) == B.MFA_ERR_INVALID_ARG
    assert call(sel=0) == B.MFA_ERR_INVALID_ARG
    assert call(lse=0) == B.MFA_ERR_INVALID_ARG
    assert call(sel_k=0) == B.MFA_ERR_INVALID_ARG
    assert call(n_split=-1) == B.MFA_ERR_INVALID_ARG
    assert call(nbytes=need - 256) == B.MFA_ERR_INVALID_ARG                   # workspace too small
    assert call(ws=0) == B.MFA_ERR_INVALID_ARG
    assert call(sel_k=257) == B.MFA_ERR_UNSUPPORTED
    d64 = [_fake_tensor(1, h, n, 64) for h, n in ((8, 1), (2, 4096), (2, 4096), (8, 1))]
    assert call(q=d64[0], k=d64[1], v=d64[2], o=d64[3]) == B.MFA_ERR_UNSUPPORTED   # head dim 64
    g3 = [_fake_tensor(1, h, n, 256) for h, n in ((6, 1), (2, 4096), (2, 4096), (6, 1))]
    assert call(q=g3[0], k=g3[1], v=g3[2], o=g3[3]) == B.MFA_ERR_UNSUPPORTED      # G = 3
    g16 = [_fake_tensor(1, h, n, 256) for h, n in ((32, 1), (2, 4096), (2, 4096), (32, 1))]
    assert call(q=g16[0], k=g16[1], v=g16[2], o=g16[3]) == B.MFA_ERR_UNSUPPORTED  # G * D > 2048
    assert call(v=_fake_tensor(1, 2, 2048, 256)) == B.MFA_ERR_SHAPE_MISMATCH
    assert call(o=_fake_tensor(1, 8, 2, 256)) == B.MFA_ERR_SHAPE_MISMATCH
    k0, v0 = _fake_tensor(1, 2, 0, 256, addr=0), _fake_tensor(1, 2, 0, 256, addr=0)
    assert call(k=k0, v=v0) == B.MFA_ERR_UNSUPPORTED                             # no keys
    f32 = _fake_tensor(1, 8, 1, 256, dtype=B.MFA_F32)
    assert call(q=f32) == B.MFA_ERR_UNSUPPORTED


def _ws(rows, seg, G, D):
    up = lambda x: -(-x // 256) * 256
    return up(rows * seg * G * D * 4) + up(rows * seg * G * 2 * 4)


def test_decode_workspace_follows_the_slot_partition(lib):
    """The automatic split gives each CTA ceil(rows * sel_k / SMs) of the rows'
    list slots laid end to end (148 SMs: a B200, and the count used without a
    device), widened to a divisor of sel_k while three quarters of the SMs
    stay busy. decode_sel64k: 64 lists of 32 slots, 14 -> 16 slots per CTA,
    128 CTAs, 2 partials per row. 20 lists of 40 slots: 6 slots per CTA (the
    divisor 8 would leave 100 CTAs), so a row meets up to ceil(39 / 6) + 1 = 8
    CTAs. 2000 lists of 256 slots: a CTA takes whole lists (8 at most) and no
    row is split: no workspace. An explicit n_split keeps n_split partials
    per row, none for 1."""
    assert lib.mfa_decode_workspace_bytes(8, 32, 8, 1, 256, 32, 0) == _ws(64, 2, 4, 256)
    assert lib.mfa_decode_workspace_bytes(2, 8, 2, 5, 256, 40, 0) == _ws(20, 8, 4, 256)
    assert lib.mfa_decode_workspace_bytes(1, 4, 2, 1000, 128, 256, 0) == 256
    assert lib.mfa_decode_workspace_bytes(8, 32, 8, 1, 256, 32, 1) == 256
    assert lib.mfa_decode_workspace_bytes(8, 32, 8, 1, 256, 32, 3) == _ws(64, 3, 4, 256)
    assert lib.mfa_decode_workspace_bytes(1, 8, 2, 0, 256, 16, 0) == 256     # no rows


def test_fwd_bias_rejects_bad_arguments_on_host(lib):
    m = _fake_map(lib)
    q, k, v, o = _fake_tensor(1, 8, 512, 128), _fake_tensor(1, 2, 512, 128), _fake_tensor(1, 2, 512, 128), \
        _fake_tensor(1, 8, 512, 128)
    d = _fake_mask(m)

    def call(bias, q=q, k=k, v=v, o=o):
        return lib.mfa_fwd_bias(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(d),
                                None if bias is None else ctypes.byref(bias), ctypes.byref(o), 0x7200_0000_0000, None)

    assert call(None) == B.MFA_ERR_INVALID_ARG
    assert call(B.MfaBias(7, 0, 0x7600_0000_0000)) == B.MFA_ERR_INVALID_ARG       # unknown kind
    assert call(B.MfaBias(B.BIAS_ALIBI, 0, None)) == B.MFA_ERR_INVALID_ARG        # no slopes
    f32 = [_fake_tensor(1, h, 512, 128, dtype=B.MFA_F32) for h in (8, 2, 2, 8)]
    mf = _fake_map(lib, bq=128)
    d = _fake_mask(mf)
    assert call(B.MfaBias(B.BIAS_ALIBI, 0, 0x7600_0000_0000), *f32) == B.MFA_ERR_UNSUPPORTED  # fp32 + bias


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without libmfa.so every entry of the binding raises: there is no fallback path."""
    missing = str(tmp_path / "libmfa.so")
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        B.load(missing)
    monkeypatch.setattr(B.load, "__defaults__", (missing,))
    with pytest.raises(RuntimeError, match="missing"):
        B.status_string(0)
    with pytest.raises(RuntimeError, match="missing"):
        B.decode_workspace_bytes(1, 8, 2, 1, 256, 16)


def test_binding_rejects_host_tensors():
    """A host tensor never reaches a kernel as a pointer: every wrapper raises first."""
    import torch
    q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 8)
    ws = torch.zeros(16, dtype=torch.uint8)
    calls = [
        lambda: B.fwd(q, q, q, None, None, q, lse),
        lambda: B.fwd_bias(q, q, q, None, None, B.BIAS_ALIBI, torch.zeros(2), q, lse),
        lambda: B.fwd_noalloc(q, q, q, None, 64, 128, q, lse),
        lambda: B.bwd(q, q, q, q, q, lse, None, None, q, q, q, ws),
        lambda: B.Decode()(q, q, q, torch.zeros(1, 2, 8, 4, dtype=torch.int32)),
        lambda: B.tensor_desc(q),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_mask_and_map_arrays_must_share_the_call_device():
    """_same_device compares every device array a mask or map holds with q's device."""
    import torch

    class Holder:
        pass

    q = torch.zeros(1, 1, 4, 8)
    same, other = Holder(), Holder()
    same.buf, same._keep = torch.zeros(4), [torch.zeros(2)]
    other.bounds = torch.empty(4, device="meta")
    B._same_device(q, same)
    with pytest.raises(ValueError, match="mask or tile-map array"):
        B._same_device(q, same, other)


def _noalloc(lib, q, k, v, d, o, bq=64, bk=128, lse=0x7200_0000_0000):
    return lib.mfa_fwd_noalloc(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(d), bq, bk,
                               ctypes.byref(o), lse, None, None)


def test_noalloc_rejects_what_fwd_rejects_before_any_launch(lib):
    """mfa_fwd_noalloc runs mfa_fwd's host checks before its map build: every
    call below returns without a CUDA call (this machine has no GPU, so a call
    that reached the device would fail with MFA_ERR_CUDA instead)."""
    m = _fake_map(lib)
    d = _fake_mask(m)
    q, k, v, o = _fake_tensor(1, 8, 512, 128), _fake_tensor(1, 2, 512, 128), _fake_tensor(1, 2, 512, 128), \
        _fake_tensor(1, 8, 512, 128)
    assert _noalloc(lib, q, k, v, d, o, lse=0) == B.MFA_ERR_INVALID_ARG
    assert _noalloc(lib, _fake_tensor(1, 8, 512, 128, addr=0), k, v, d, o) == B.MFA_ERR_INVALID_ARG
    assert _noalloc(lib, _fake_tensor(1, 8, 512, 128, dtype=B.MFA_F32), k, v, d, o) == B.MFA_ERR_INVALID_ARG
    assert _noalloc(lib, _fake_tensor(1, 8, 512, 96), _fake_tensor(1, 2, 512, 96), _fake_tensor(1, 2, 512, 96), d,
                    _fake_tensor(1, 8, 512, 96)) == B.MFA_ERR_UNSUPPORTED
    assert _noalloc(lib, q, _fake_tensor(1, 3, 512, 128), _fake_tensor(1, 3, 512, 128), d, o) == \
        B.MFA_ERR_SHAPE_MISMATCH
    assert _noalloc(lib, q, k, v, d, _fake_tensor(1, 8, 256, 128)) == B.MFA_ERR_SHAPE_MISMATCH
    unaligned = _fake_tensor(1, 8, 512, 128, addr=0x7100_0000_0002)
    assert _noalloc(lib, unaligned, k, v, d, o) == B.MFA_ERR_UNSUPPORTED
    # two heads per 64-row tile need an even group size
    q6, o6 = _fake_tensor(1, 6, 512, 128), _fake_tensor(1, 6, 512, 128)
    assert _noalloc(lib, q6, k, v, d, o6) == B.MFA_ERR_UNSUPPORTED
    assert _noalloc(lib, q, k, v, d, o, bq=96) == B.MFA_ERR_UNSUPPORTED
    assert _noalloc(lib, q, k, v, _fake_mask(m, Nq=256), o) == B.MFA_ERR_SHAPE_MISMATCH


def test_binding_rejects_a_stream_of_another_device():
    """The binding launches on the tensors' device; a stream of another device is refused."""
    import torch

    class FakeStream:
        device = torch.device("cuda", 1)
        cuda_stream = 0

    with pytest.raises(ValueError, match="stream is on"):
        B._stream_ptr(FakeStream(), torch.device("cuda", 0))
    assert B._stream_ptr(FakeStream(), torch.device("cuda", 1)) == 0


def test_timeout_hook_rejects_limits_out_of_range(lib):
    assert lib.mfa_test_arm_fwd_timeout(0) == B.MFA_ERR_INVALID_ARG
    assert lib.mfa_test_arm_fwd_timeout(1_000_001) == B.MFA_ERR_INVALID_ARG
