"""CPU checks of the C ABI: the library loads, exports every symbol that
include/sas.h declares, and its host-side validation rejects bad arguments
before anything touches a GPU (these calls return before any CUDA call)."""
import ctypes
import os
import re

import pytest

from trainable_gated_block_b200 import build, sas

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return sas.lib()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(sas_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    declared = _declared()
    assert {"sas_select", "sas_attn_fwd", "sas_attn_bwd", "sas_decode_paged"} <= declared
    for name in declared:
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_binding_covers_header(L):
    assert _declared() == set(sas.SIGNATURES)


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first


def _fwd(L, **kw):
    a = dict(dtype=sas.SAS_BF16, B=1, S=128, Hq=4, Hkv=2, D=128, bs=64, K=2, scale=0.1)
    a.update(kw)
    return L.sas_attn_fwd(a["dtype"], FAKE, FAKE, FAKE, a["B"], a["S"], a["Hq"], a["Hkv"], a["D"], a["bs"],
                          a["K"], FAKE, FAKE, FAKE, a["scale"], FAKE, FAKE, None)


@pytest.mark.parametrize("kw,code", [
    (dict(S=0), sas.SAS_ERR_INVALID_ARG),
    (dict(Hq=3), sas.SAS_ERR_INVALID_ARG),
    (dict(K=-1), sas.SAS_ERR_INVALID_ARG),
    (dict(B=0), sas.SAS_ERR_INVALID_ARG),
    (dict(bs=32), sas.SAS_ERR_UNSUPPORTED),
    (dict(D=96), sas.SAS_ERR_UNSUPPORTED),
    (dict(dtype=7), sas.SAS_ERR_INVALID_ARG),
    (dict(scale=float("nan")), sas.SAS_ERR_INVALID_ARG),
])
def test_fwd_rejects_bad_arguments(L, kw, code):
    assert _fwd(L, **kw) == code
    assert L.sas_last_error()


def test_select_rejects_bad_arguments(L):
    f = L.sas_select
    assert f(None, 1, 1, 8, 8, None, 64, 2, FAKE, FAKE, FAKE, FAKE, None) == sas.SAS_ERR_INVALID_ARG
    assert f(FAKE, 1, 1, 8, 4, None, 64, 2, FAKE, FAKE, FAKE, FAKE, None) == sas.SAS_ERR_INVALID_ARG
    assert f(FAKE, 1, 1, 8, 8, None, 128, 2, FAKE, FAKE, FAKE, FAKE, None) == sas.SAS_ERR_UNSUPPORTED
    assert f(FAKE, 1, 1, 16386, 16386, None, 64, 2, FAKE, FAKE, FAKE, FAKE, None) == sas.SAS_ERR_UNSUPPORTED
    assert f(FAKE, 1, 1, 8, 8, None, 64, 2, None, FAKE, None, FAKE, None) == sas.SAS_ERR_INVALID_ARG


def test_bwd_and_decode_workspace_queries(L):
    assert L.sas_attn_bwd_workspace_size(sas.SAS_BF16, 1, 0, 4, 2, 128, 2) == 0
    assert L.sas_attn_bwd_workspace_size(sas.SAS_BF16, 1, 100, 4, 2, 128, 2) > 0      # partial last block
    assert L.sas_attn_bwd_workspace_size(sas.SAS_BF16, 1, 128, 4, 2, 128, 2) > 0
    # the tensor-core backward packs block and slot into 16 bits each: 32767 blocks at most
    assert L.sas_attn_bwd_workspace_size(sas.SAS_BF16, 1, 32767 * 64, 4, 2, 128, 2) > 0
    assert L.sas_attn_bwd_workspace_size(sas.SAS_BF16, 1, 32767 * 64 + 1, 4, 2, 128, 2) == 0
    assert L.sas_attn_bwd_varlen_workspace_size(sas.SAS_BF16, 3, 100, 250, 4, 2, 128, 2) > 0
    assert L.sas_attn_bwd_varlen_workspace_size(sas.SAS_BF16, 3, 100, 0, 4, 2, 128, 2) == 0
    assert L.sas_decode_workspace_size(4, 32, 8, 128, 32) > 0
    assert L.sas_decode_workspace_size(4, 32, 8, 64, 32) == 0
    # too-small workspace is rejected on the host
    r = L.sas_attn_bwd(sas.SAS_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE,
                       1, 128, 4, 2, 128, 64, 2, 0.1, FAKE, FAKE, FAKE, FAKE, ctypes.c_void_p(0x10000), 16, None)
    assert r == sas.SAS_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(L):
    f = L.sas_decode_paged
    args = [FAKE, FAKE, FAKE, 10, FAKE, 4, FAKE, 2, 32, 8, 128, 64, 4, FAKE, FAKE, FAKE, 0.1, FAKE, None,
            ctypes.c_void_p(0x10000), 1 << 30, None]
    bad = list(args); bad[10] = 64                       # D = 64
    assert f(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[8] = 24                        # G = 3
    assert f(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[11] = 16                       # page size
    assert f(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[19] = ctypes.c_void_p(0x10010)  # workspace alignment
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG


def test_varlen_rejects_bad_arguments(L):
    f = L.sas_attn_fwd_varlen
    args = [sas.SAS_BF16, FAKE, FAKE, FAKE, FAKE, 3, 100, 250, 4, 2, 128, 64, 2, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE,
            None]
    bad = list(args); bad[4] = None                       # no cu_seqlens
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[7] = 0                          # no token rows
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[6] = 0                          # max_seqlen 0
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[8] = 3                          # Hq % Hkv
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG
    sel = L.sas_select_varlen
    assert sel(FAKE, 3, 2, 2, 2, None, 64, 2, FAKE, FAKE, FAKE, FAKE, None) == sas.SAS_ERR_INVALID_ARG
    b = L.sas_attn_bwd_varlen
    r = b(sas.SAS_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, FAKE, FAKE, FAKE, FAKE, None,
          3, 100, 250, 4, 2, 128, 64, 2, 0.1, FAKE, FAKE, FAKE, FAKE, ctypes.c_void_p(0x10000), 1 << 30, None)
    assert r == sas.SAS_ERR_INVALID_ARG


def test_score_select_rejects_bad_arguments(L):
    f = L.sas_score_select
    ws = ctypes.c_void_p(0x10000)
    #       q     k     noise ld  B  S    Hq Hkv D   bs  K  s     ld_s idx   cnt   lg    lse_s ws  bytes    stream
    args = [FAKE, FAKE, None, 0, 1, 512, 8, 2, 128, 64, 2, FAKE, 8, FAKE, FAKE, FAKE, FAKE, ws, 1 << 30, None]
    bad = list(args); bad[0] = None                         # no q
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[5] = 500                          # S not a multiple of 64
    assert f(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[8] = 96                           # D
    assert f(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[12] = 7                           # ld_s below the 8 blocks
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[5] = 64 * 16386; bad[12] = 16386  # 16385 history blocks
    assert f(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[4] = 32768; bad[5] = 64; bad[12] = 1   # B * Hkv above a grid dimension
    assert f(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[17] = ctypes.c_void_p(0x10010)    # workspace alignment
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[18] = 16                          # workspace too small
    assert f(*bad) == sas.SAS_ERR_INVALID_ARG


def test_pool_pages_and_decode_scorer_reject_bad_arguments(L):
    pool = L.sas_pool_pages
    #          k_cache pages Hkv D   psz pages n   kpool stream
    args = [FAKE, 4, 2, 128, 64, None, 0, FAKE, None]
    bad = list(args); bad[0] = None
    assert pool(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[4] = 32                            # page size
    assert pool(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[3] = 96                            # D
    assert pool(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[7] = ctypes.c_void_p(0x10004)     # kpool alignment
    assert pool(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[5] = FAKE; bad[6] = 0             # an empty page list is a no-op
    assert pool(*bad) == sas.SAS_OK

    dec = L.sas_score_select_decode
    #       q     kpool pages ptab max  kv_len N  Hq Hkv D    psz noise ld_n K  s     ld_s idx   cnt   lg    lse   stream
    args = [FAKE, FAKE, 8, FAKE, 4, FAKE, 2, 8, 2, 128, 64, None, 0, 2, FAKE, 4, FAKE, FAKE, FAKE, FAKE, None]
    bad = list(args); bad[3] = None                          # no page table
    assert dec(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[7] = 6; bad[8] = 4                 # Hq % Hkv
    assert dec(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[11] = FAKE; bad[12] = 3            # noise rows shorter than ld_s
    assert dec(*bad) == sas.SAS_ERR_INVALID_ARG
    bad = list(args); bad[15] = 16385                        # rows longer than the selection handles
    assert dec(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[6] = 40000                         # N * Hkv above a grid dimension
    assert dec(*bad) == sas.SAS_ERR_UNSUPPORTED
    bad = list(args); bad[1] = ctypes.c_void_p(0x10004)     # kpool alignment
    assert dec(*bad) == sas.SAS_ERR_INVALID_ARG
