"""duolm_embedding_rho_static, the allocation-free rho estimate, against the
context's own duolm_embedding_rho.

Callers that cannot allocate device memory (a server that has already split
the whole GPU into its own pools, a latency-critical loop that cannot wait
for an allocation) pass the embedding and a one-double output they already
own; the per-row scratch is an array built into the library.  This file is
collected last so that a failure here leaves every other test already run;
it creates everything it needs, so it also passes on its own.
"""
import dataclasses

import numpy as np
import pytest

from synth import workloads as W

pytestmark = pytest.mark.gpu


def _static_rho(embed_host: np.ndarray, dtype: int) -> float:
    import torch
    from shared_prefix_item_b200 import _lib
    if embed_host.dtype == np.uint16:
        dev = torch.from_numpy(embed_host.view(np.int16)).cuda()
    else:
        dev = torch.from_numpy(np.ascontiguousarray(embed_host)).cuda()
    out = torch.full((1,), float("nan"), dtype=torch.float64, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    _lib.embedding_rho_static(dev.data_ptr(), dtype, embed_host.shape[0], embed_host.shape[1], out.data_ptr(),
                              stream)
    torch.cuda.synchronize()
    return float(out.item())


def test_rho_static_matches_context_rho_on_consecutive_calls():
    import shared_prefix_item_b200 as S
    big = dataclasses.replace(W.QWEN3_06B, n_layers=1, name="qwen3-shape-1layer")  # 151,936 rows
    small = dataclasses.replace(W.TINY, n_layers=1, name="tiny-1layer")           # 512 rows, fp32
    expect = {}
    for shape in (big, small):
        rk = S.Ranker(shape, W.model_weights(shape))
        try:
            expect[shape.name] = rk.embedding_rho()
        finally:
            rk.close()
    # big, then small (which leaves stale rows from the big call in the
    # scratch), then big again: each result matches the context's estimate
    for shape, dtype in ((big, S.DTYPE_BF16), (small, S.DTYPE_FP32), (big, S.DTYPE_BF16)):
        got = _static_rho(W.model_weights(shape)[0], dtype)
        assert got == pytest.approx(expect[shape.name], rel=1e-12), shape.name


def test_rho_static_rejects_oversized_vocab():
    import torch

    import shared_prefix_item_b200 as S
    from shared_prefix_item_b200 import _lib
    buf = torch.zeros(64, dtype=torch.float64, device="cuda")
    with pytest.raises(S.DuolmError) as e:
        _lib.embedding_rho_static(buf.data_ptr(), S.DTYPE_BF16, _lib.RHO_STATIC_MAX_ROWS + 1, 1024,
                                  buf.data_ptr())
    assert e.value.code == -5
