"""sas_decode_paged_noalloc: paged decode for callers that cannot allocate.

Some callers have no device memory to give a workspace at decode time (a
serving engine whose KV-cache pool owns nearly all of the GPU, or a C host
with only its input/output buffers). They call sas_decode_paged_noalloc,
which keeps its split-KV partials in a static array inside the library.
This test calls it through the C ABI twice in a row, on different inputs,
and checks each result against the workspace entry point sas_decode_paged
within the bf16 output tolerance the other tests use. It also checks that a
size needing more scratch than the static array holds is refused on the host.

Kept in its own file, named to be collected last.
"""
import ctypes

import pytest
import torch

from tests.parity_util import BF16_OUT_TOL
from trainable_gated_block_b200 import build, inputs, sas

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _noalloc(L, xd, sel, o, lse):
    N, Hq, D = xd["q"].shape
    return L.sas_decode_paged_noalloc(
        ctypes.c_void_p(xd["q"].data_ptr()), ctypes.c_void_p(xd["k_cache"].data_ptr()),
        ctypes.c_void_p(xd["v_cache"].data_ptr()), xd["k_cache"].shape[0],
        ctypes.c_void_p(xd["page_table"].data_ptr()), xd["page_table"].shape[1],
        ctypes.c_void_p(xd["kv_len"].data_ptr()), N, Hq, xd["k_cache"].shape[1], D, 64, sel[0].shape[-1],
        ctypes.c_void_p(sel[0].data_ptr()), ctypes.c_void_p(sel[1].data_ptr()), ctypes.c_void_p(sel[2].data_ptr()),
        1.0 / D ** 0.5, ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_workspace_decode_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    L = sas.lib()
    for call, seed in enumerate((41, 42)):
        cfg = inputs.DecodeConfig("noalloc", N=24, Hq=32, Hkv=8, D=128, K=16, min_hist=0, max_hist=96,
                                  partial=True, seed=seed)
        assert sas.decode_workspace_bytes(cfg.N, cfg.Hq, cfg.Hkv, cfg.D, cfg.K) <= SCRATCH_BYTES
        x = inputs.make_decode(cfg)
        xd = {k: v.cuda() for k, v in x.items()}
        sel = sas.select(xd["s"], cfg.K, kv_len=xd["kv_len"])
        ref_o, ref_lse = sas.decode_paged(xd["q"], xd["k_cache"], xd["v_cache"], xd["page_table"], xd["kv_len"],
                                          sel[0], sel[1], sel[2])
        o = torch.full_like(xd["q"], float("nan"))
        lse = torch.full((cfg.N, cfg.Hq), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(L, xd, sel, o, lse) == sas.SAS_OK, L.sas_last_error()
        torch.cuda.synchronize()
        sas.get_error_flag()
        err_o = (o.float() - ref_o.float()).abs().max().item()
        err_l = (lse - ref_lse).abs().max().item()
        assert err_o <= BF16_OUT_TOL and err_l <= BF16_OUT_TOL, (call, err_o, err_l)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    L = sas.lib()
    N, Hq, Hkv, D, K = 4096, 64, 8, 128, 64          # partials far above 16 MiB
    assert sas.decode_workspace_bytes(N, Hq, Hkv, D, K) > SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)                    # never dereferenced: refused first
    code = L.sas_decode_paged_noalloc(fake, fake, fake, 10, fake, 4, fake, N, Hq, Hkv, D, 64, K,
                                      fake, fake, fake, 0.1, fake, None, None)
    assert code == sas.SAS_ERR_INVALID_ARG
    assert b"static scratch" in L.sas_last_error()
