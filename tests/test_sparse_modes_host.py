"""mfa_mask_from_sparse_mode on the host: the band-type modes (0, 2, 3, 4)
launch nothing, so their conversion is checked here, without a GPU, against
the oracle's own reading of each mode; argument errors are rejected before
any launch."""
import ctypes

import numpy as np
import pytest

from mask_aware_block_mfa_b200 import binding as B
from mask_aware_block_mfa_b200 import workloads as W
from oracle import masks as OM
from oracle import sparse_modes as SM


@pytest.fixture(scope="module")
def lib():
    return B.load()


def convert(lib, mode, Bn, nq, nk, pre=0, nxt=0, arrays=None, n_seq=0, seq=None):
    sm = B.MfaSparseMode()
    sm.mode, sm.pre_tokens, sm.next_tokens, sm.n_seq = mode, pre, nxt, n_seq
    if seq is not None:
        sm.seq_q = sm.seq_kv = seq
    out = B.MfaMaskDesc()
    a = arrays or [None] * 4
    return lib.mfa_mask_from_sparse_mode(ctypes.byref(sm), Bn, nq, nk, *a, ctypes.byref(out), None), out


@pytest.mark.parametrize("nq,nk", [(40, 40), (30, 70), (70, 30), (1, 9)])
@pytest.mark.parametrize("mode,pre,nxt", [(0, 5, 2), (0, 0, 0), (2, 0, 0), (3, 0, 0), (4, 6, -1), (4, 100, 3)])
def test_band_modes_match_the_oracle(lib, mode, pre, nxt, nq, nk):
    st, d = convert(lib, mode, 2, nq, nk, pre, nxt)
    assert st == B.MFA_OK
    assert (d.kind, d.B, d.Hm, d.Nq, d.Nk) == (W.MASK_BAND, 2, 1, nq, nk)
    band = W.MaskDesc(W.MASK_BAND, 2, 1, nq, nk, pre_tokens=d.pre_tokens, next_tokens=d.next_tokens)
    ref = SM.visible_dense(SM.SparseMode(mode, 2, nq, nk, pre, nxt))
    assert np.array_equal(OM.visible_dense(band), ref)


def test_rejections_before_any_launch(lib):
    assert convert(lib, 1, 1, 8, 8)[0] == B.MFA_ERR_UNSUPPORTED
    assert convert(lib, 9, 1, 8, 8)[0] == B.MFA_ERR_UNSUPPORTED
    assert convert(lib, -1, 1, 8, 8)[0] == B.MFA_ERR_UNSUPPORTED
    assert convert(lib, 0, -1, 8, 8)[0] == B.MFA_ERR_INVALID_ARG
    assert convert(lib, 0, 70000, 8, 8)[0] == B.MFA_ERR_INVALID_ARG
    fake = [0x7300_0000_0000] * 4  # never dereferenced: each call below fails on the host
    assert convert(lib, 5, 1, 8, 8)[0] == B.MFA_ERR_INVALID_ARG             # no bound arrays
    assert convert(lib, 5, 1, 8, 8, arrays=fake)[0] == B.MFA_ERR_INVALID_ARG  # no prefix array
    assert convert(lib, 7, 2, 8, 8, arrays=fake, n_seq=1, seq=0x7300_0000_0000)[0] == B.MFA_ERR_INVALID_ARG  # B != 1
    assert convert(lib, 8, 1, 8, 8, arrays=fake, n_seq=0, seq=0x7300_0000_0000)[0] == B.MFA_ERR_INVALID_ARG  # no sequence
    assert convert(lib, 7, 1, 8, 8, arrays=fake, n_seq=2)[0] == B.MFA_ERR_INVALID_ARG                      # no ends
    sm = B.MfaSparseMode()
    assert lib.mfa_mask_from_sparse_mode(ctypes.byref(sm), 1, 8, 8, None, None, None, None, None, None) == \
        B.MFA_ERR_INVALID_ARG
