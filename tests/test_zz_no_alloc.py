"""The allocation-free attention entry point.

csa2_sparse_attn_decode_noalloc serves callers that cannot allocate device
memory themselves: code handed only its input and output buffers (a plugin
hook without a workspace), or a decode loop that must not call cudaMalloc
because it can synchronise the device. Its split partials live in a
library-owned device array instead of a caller workspace. This test calls it
through the C ABI twice in a row and checks both results against the regular
entry point (which takes a caller workspace), with the same tolerance as the
other attention tests (max-abs 2e-3, relative L2 1e-3)."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(576)


def test_noalloc_attention_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import inputs, lib, workload
    from oracle_check import assert_attn_close

    wl = inputs.small_workload("noalloc", 3, 2, [3000, 1500, 700], 256, modes=("F",), seed=11)
    dw = workload.DeviceWorkload(wl)
    dw.step()
    B, Sq, k = wl.batch, wl.q_tokens, wl.top_k
    # this shape splits each query's key list, so the partials need scratch
    assert lib.sparse_attn_workspace_bytes(B, Sq, k) > 0
    assert lib.sparse_attn_workspace_bytes(B, Sq, k) <= lib.NOALLOC_SCRATCH_BYTES
    g = dw.group
    idx = g.index(0)
    ref_o, ref_lse = lib.sparse_attn_decode(dw.q[0], g.cache(0), dw.page_table, dw.seq_lens, idx, dw.swa[0],
                                            SCALE)
    ref_o, ref_lse = ref_o.cpu().numpy(), ref_lse.cpu().numpy()
    for call in range(2):
        out = torch.full((B, Sq, 16, 576), float("nan"), device="cuda")
        lse = torch.full((B, Sq, 16), float("nan"), device="cuda")
        lib.sparse_attn_decode_noalloc(dw.q[0], g.cache(0), dw.page_table, dw.seq_lens, idx, dw.swa[0],
                                       SCALE, out, lse)
        assert lib.last_device_error() == 0
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(l).all()
        for b in range(B):
            for j in range(Sq):
                assert_attn_close(o[b, j], l[b, j], ref_o[b, j].astype(np.float64),
                                  ref_lse[b, j].astype(np.float64), f"call {call} b {b} j {j}")


def test_noalloc_scratch_bound_and_argument_checks():
    """The partials of any shape fit the library-owned array on this GPU
    (rows are split into runs only while the runs fit one wave, one partial
    each), and argument errors are reported as themselves, before the scratch
    size is considered; nothing is launched."""
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import ctypes
    from compressed_sparse_attention_quant_b200 import lib
    sizes = [lib.sparse_attn_workspace_bytes(B, Sq, k) for B in (1, 2, 7, 64, 148, 300, 65535)
             for Sq in (1, 4) for k in (1, 64, 2048, 65536) if B * Sq <= 65535]
    assert 0 < max(sizes) <= lib.NOALLOC_SCRATCH_BYTES
    assert lib.sparse_attn_workspace_bytes(65536, 1, 1) == 0            # B * Sq > 65535: unsupported shape
    assert lib.sparse_attn_workspace_bytes(1, 1, 65537) == 0            # k > 65536
    L = lib._L
    cache = lib._Cache(16, 16, 16, 16, 4)                              # host-side checks only: never launched
    before = lib.launch_count()

    def call(B, Sq, H, k):
        return L.csa2_sparse_attn_decode_noalloc(16, B, Sq, H, 576, ctypes.byref(cache), 16, 1, 16, 16, k, 16,
                                                 128, 0.1, 16, 16, None)
    assert call(1, 1, 8, 4) == 2                                         # CSA2_ERR_UNSUPPORTED: 8 heads
    assert call(70000, 1, 16, 4) == 2                                    # B * Sq > 65535
    assert call(1, 1, 16, -1) == 1                                       # CSA2_ERR_INVALID_ARG
    assert call(1, 1, 16, 70000) == 1                                    # k > 65536
    assert lib.launch_count() == before
