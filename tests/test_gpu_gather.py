"""duolm_gather, the hot path's virtual-id gather on its own, against the
table and embedding it reads (bit-exact rows) and the quantities it writes
for the first layer's norm."""
import numpy as np
import pytest

import parity as P
from synth import workloads as W
from synth.rng import Stream, bf16_to_f32
from test_gpu_parity import Q2, Q2_ITEMS

pytestmark = pytest.mark.gpu


def _run_gather(rk, ids: np.ndarray):
    import torch
    n, d = len(ids), Q2.d
    ids_d = torch.from_numpy(ids.astype(np.int32)).cuda()
    x = torch.full((n, d), float("nan"), dtype=torch.float32, device="cuda")
    xg = torch.zeros((n, d), dtype=torch.int16, device="cuda")
    ssp = torch.full((n, d // 64), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    rk.gather(ids_d.data_ptr(), n, x.data_ptr(), xg.data_ptr(), ssp.data_ptr())
    return x, xg, ssp


def _expected_rows(rk, ids: np.ndarray) -> np.ndarray:
    emb = bf16_to_f32(W.model_weights(Q2)[0])                      # [V][d], exact in fp32
    table = rk.debug_table(Q2_ITEMS).view(np.float16).astype(np.float32)  # the library's own fp16 rows
    return np.where((ids < Q2.vocab)[:, None], emb[np.minimum(ids, Q2.vocab - 1)],
                    table[np.clip(ids - Q2.vocab, 0, Q2_ITEMS - 1)])


@pytest.mark.parametrize("n", [1, 37, 1000, 4099])
def test_gather_rows_gain_and_sums(n):
    rk = P.ranker(Q2, Q2_ITEMS)
    s = Stream(4242, n)
    ids = s.integers(n, 0, Q2.vocab + Q2_ITEMS)  # vocabulary and item rows, repeats included
    x, xg, ssp = _run_gather(rk, ids)
    rk.sync()
    x, xg, ssp = x.cpu().numpy(), xg.cpu().numpy().view(np.float16), ssp.cpu().numpy()
    want = _expected_rows(rk, ids)
    assert np.array_equal(x, want)  # a copy: bit-exact
    g = bf16_to_f32(W.model_weights(Q2)[1])  # layer 0 attention-norm gain
    assert np.array_equal(xg, (want * g[None, :]).astype(np.float16))  # fp32 product, round to nearest
    ss = (want.astype(np.float64) ** 2).sum(axis=1)
    assert np.allclose(ssp[:, 0], ss, rtol=1e-5, atol=0)
    assert np.all(ssp[:, 1:] == 0)


def test_gather_out_of_range_id_raises_device_error_and_zeroes_row():
    import shared_prefix_item_b200 as S
    rk = P.ranker(Q2, Q2_ITEMS)
    ids = np.array([5, Q2.vocab + Q2_ITEMS, Q2.vocab + 3], np.int64)  # the middle one is one past the table
    x, _, _ = _run_gather(rk, ids)
    with pytest.raises(S.DuolmError) as e:
        rk.sync()
    assert e.value.code == -7
    x = x.cpu().numpy()
    assert np.all(x[1] == 0)
    assert np.array_equal(x[[0, 2]], _expected_rows(rk, ids[[0, 2]]))
    rk.sync()  # the flag was cleared when it was reported


def test_gather_rejects_bad_arguments():
    import shared_prefix_item_b200 as S
    rk = P.ranker(Q2, Q2_ITEMS)
    with pytest.raises(S.DuolmError) as e:
        rk.gather(0, 10, 0, 0, 0)
    assert e.value.code == -1
    rk.gather(0, 0, 0, 0, 0)  # nothing to do
