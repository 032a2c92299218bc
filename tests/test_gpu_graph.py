"""The decode step captured as a CUDA graph (StepGraph) launches the same
library kernels as the eager step and gives bit-identical results, and a
replay reads the captured tensors as they are at replay time (inputs
refreshed in place are seen; outputs are rewritten)."""
import zlib

import pytest
import torch

from compressed_sparse_attention_quant_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from compressed_sparse_attention_quant_b200 import lib, workload
    return lib, workload


CASES = [
    # name, B, Sq, lens, k, modes
    ("graph_ragged", 3, 1, [5000, 900, 70], 300, ("F", "R", "U")),
    ("graph_sq4", 2, 4, [2500, 1000], 256, ("F", "U", "R", "U")),
]


def _outputs(dw):
    g = dw.group
    idx = [g.index(li).clone() for li in range(len(g.modes))]
    return idx + [t.clone() for t in g.out] + [t.clone() for t in g.lse]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_graph_replay_equals_eager_step(mods, case):
    lib, workload = mods
    name, B, Sq, lens, k, modes = case
    wl = inputs.small_workload(name, B, Sq, lens, k, modes=modes, random_pages=True,
                               seed=zlib.crc32(name.encode()) % 1000)
    dw = workload.DeviceWorkload(wl)
    n0 = lib.launch_count()
    dw.step()
    torch.cuda.synchronize()
    eager_launches = lib.launch_count() - n0
    want = _outputs(dw)
    assert lib.last_device_error() == 0

    sg = dw.capture()
    assert sg.launches == eager_launches
    for li in range(len(modes)):                     # poison every output the graph must rewrite
        dw.group.out[li].fill_(float("nan"))
        dw.group.lse[li].fill_(float("nan"))
        if modes[li] in ("F", "R"):
            dw.group.index(li).fill_(-7)
    n1 = lib.launch_count()
    sg.replay()
    torch.cuda.synchronize()
    assert lib.launch_count() == n1                  # no host-side launch on replay
    assert lib.last_device_error() == 0
    got = _outputs(dw)
    for a, b in zip(want, got):
        assert torch.equal(a, b)


def test_graph_sees_inputs_refreshed_in_place(mods):
    lib, workload = mods
    wl = inputs.small_workload("graph_refresh", 2, 1, [3000, 1500], 200, modes=("F", "U"), random_pages=True,
                               seed=11)
    dw = workload.DeviceWorkload(wl)
    sg = dw.capture()
    gen = torch.Generator(device="cuda").manual_seed(5)
    # new attention queries and window rows for every layer, new indexer weights
    for t in dw.q + dw.swa:
        t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(t.dtype))
    for t in dw.w.values():
        t.copy_(torch.rand(t.shape, generator=gen, device="cuda"))
    sg.replay()
    torch.cuda.synchronize()
    got = _outputs(dw)
    dw.step()                                        # eager step over the same (refreshed) tensors
    torch.cuda.synchronize()
    want = _outputs(dw)
    assert lib.last_device_error() == 0
    for a, b in zip(want, got):
        assert torch.equal(a, b)
