"""The five benchmark workloads at full size, in the launch configuration the
benchmark times (DeviceWorkload.step): sampled sequences are checked against
the oracle one query at a time (indices bit-exact, attention within max-abs
2e-3 / relative L2 1e-3), plus sampled cache bytes."""
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_attention_quant_b200 import inputs
from oracle_check import OracleRun, assert_attn_close

pytestmark = pytest.mark.gpu

# workload name -> sequences the oracle checks
SAMPLES = {
    "full_b1_t4k": [0],
    "fru_b8_t16k": [0, 3, 7],
    "decode_b64_t128k": [0, 37],
    "verify_b32_sq4_t32k": [5, 31],
    "long_b4_t1m": [2],
}


@pytest.mark.parametrize("name", list(SAMPLES))
def test_workload_matches_oracle_on_samples(name):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib, workload
    wl = inputs.WORKLOADS[name]
    dw = workload.DeviceWorkload(wl)
    dw.step()
    dw.step()                                   # a second step must give the same result
    assert lib.last_device_error() == 0
    seqs = SAMPLES[name]
    ref = OracleRun(dw, seqs)
    for li in range(len(wl.modes)):
        idx = dw.group.index(li).cpu().numpy()
        o = dw.group.out[li].cpu().numpy()
        lse = dw.group.lse[li].cpu().numpy()
        for b in seqs:
            for j in range(wl.q_tokens):
                r = ref.out[li][(b, j)]
                np.testing.assert_array_equal(idx[b, j], r["idx"], err_msg=f"{name} layer {li} b {b} j {j}")
                assert_attn_close(o[b, j], lse[b, j], r["o"], r["lse"], f"{name} layer {li} b {b} j {j}")
    # sampled cache bytes of every owner
    g = torch.Generator().manual_seed(9)
    for owner, cache in dw.group.caches.items():
        for b in seqs:
            T = wl.lens()[b]
            pos = torch.cat([torch.randint(0, T, (256,), generator=g), torch.arange(T - wl.q_tokens, T)])
            slots = lib.slot_mapping(dw.page_table, b, pos.cuda()).long()
            rows = inputs.kv_rows(wl, owner, b, pos, "cuda")
            rc, rs = oracle.quant_fp4(oracle.bf16_bits(rows))
            np.testing.assert_array_equal(cache.kv_fp4.view(-1, 288)[slots].cpu().numpy(), rc)
            np.testing.assert_array_equal(cache.kv_scale.view(-1, 36)[slots].cpu().numpy(), rs)
