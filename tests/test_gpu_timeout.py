"""The failure path of the bounded device-side waits, exercised without a
fault: with TB_FLAG_TEST_STALL the batch-1 kernel issues none of its
copies, so every wait runs into its (test-short, about 10 ms) limit and gives
up.  The kernel must still return, write NaN to every output, and the next
tb_sync_status must report TB_ERR_TIMEOUT; a normal call afterwards must
work (the context stays usable) and report TB_OK."""
import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth
from decode_gemv_tb_b200 import tb
from tests.helpers import assert_within, u16, w_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TB_OK, TB_ERR_TIMEOUT = 0, 6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tb.load()


def test_stalled_waits_give_up_and_report(oracle):
    torch.cuda.synchronize()
    assert tb.sync_status() == TB_OK  # nothing pending from earlier tests
    items, refs = [], []
    for i, (grid, N, K) in enumerate(((tb.INT2, 1000, 2048), (tb.INT3, 300, 1024), (tb.TERNARY, 520, 4096))):
        W = synth.gaussian_weights(N, K, seed=9100 + i)
        s_ref = oracle.scales_absmax(w_np(W), grid)
        p_ref, _ = oracle.pack(w_np(W), grid, s_ref)
        x = synth.activations(K, seed=9200 + i)
        refs.append(oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K))
        p = torch.from_numpy(p_ref.reshape(-1).view(np.uint8).copy()).to(DEV)
        s = torch.from_numpy(s_ref.view(np.int16).copy()).to(DEV).view(torch.bfloat16)
        items.append((p, grid, s, x.to(DEV), torch.zeros(N, dtype=torch.float32, device=DEV), N, K))
    tb.tb_layer_gemv(items, flags=tb.FLAG_TEST_STALL)
    assert tb.sync_status() == TB_ERR_TIMEOUT
    for it in items:
        assert torch.all(torch.isnan(it[4])), "a stalled launch must leave NaN, not a result"
    # the status was cleared and the context is usable: the same launch without the hook is correct
    tb.tb_layer_gemv(items)
    assert tb.sync_status() == TB_OK
    for it, (y64, yabs) in zip(items, refs):
        assert_within(it[4], y64, yabs, "f32", oracle, "after the stalled launch")
