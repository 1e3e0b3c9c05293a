"""Alg 1 draft-length pruning on the device (dspark_prune_lengths) against the oracle: exact."""
import numpy as np
import pytest
import torch

from oracle import dspark as O
from parity_util import ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


@pytest.mark.parametrize("A,gamma", [(37, 16), (300, 8), (5, 1)])
def test_prune_lengths_match_oracle(A, gamma):
    import block_draft_model_dspark_b200 as dsp
    g = np.random.default_rng(A * 31 + gamma)
    conf = g.random((A, gamma)).astype(np.float32)
    thr = (0.2 + 0.3 * g.random(gamma)).astype(np.float32)
    # edge values: a confidence equal to its threshold, a NaN, a zero at position 0
    conf[0, min(1, gamma - 1)] = thr[min(1, gamma - 1)]
    conf[1 % A, gamma - 1] = np.nan
    conf[2 % A, 0] = 0.0
    got = dsp.prune_lengths(torch.from_numpy(conf).cuda(), torch.from_numpy(thr).cuda())
    torch.cuda.synchronize()
    want = O.prune_lengths(conf, thr)
    np.testing.assert_array_equal(got.cpu().numpy(), want)


def test_prune_lengths_on_round_confidences():
    """The confidences a draft round wrote, pruned with a uniform minConf and with per-position
    thresholds, against the oracle on the same confidence values."""
    import block_draft_model_dspark_b200 as dsp
    from synthetic import small_model
    from parity_util import build
    m = small_model(dtype="bf16")
    cpu, W, model = build(m, 91)
    A, L = 4, 40
    hid = torch.randn(A, L, m.hidden_size, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    cache = dsp.KvCache(model, A, L)
    cache.set_lengths([0] * A)
    pos0 = torch.zeros(A, dtype=torch.int32, device="cuda")
    model.dspark_append_context_kv(cache, hid.cuda(), [L] * A, pos0)
    out = model.draft(cache, torch.arange(A, dtype=torch.int32, device="cuda"),
                      torch.full((A,), L, dtype=torch.int32, device="cuda"), L)
    conf = out["conf"]
    for thr in (torch.full((m.block_size,), float(conf.float().median()), device="cuda"),
                torch.linspace(0.2, 0.8, m.block_size, device="cuda")):
        got = dsp.prune_lengths(conf, thr.float().contiguous())
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.cpu().numpy(), O.prune_lengths(conf.cpu().numpy(), thr.cpu().numpy()))


def test_prune_lengths_refusals():
    import ctypes
    import block_draft_model_dspark_b200 as dsp
    lib = dsp.get_lib()
    conf = torch.zeros(2, 4, device="cuda")
    thr = torch.zeros(4, device="cuda")
    lens = torch.zeros(2, dtype=torch.int32, device="cuda")
    assert lib.dspark_prune_lengths(conf.data_ptr(), 2, 0, thr.data_ptr(), lens.data_ptr(), None) == \
        dsp.DSPARK_ERR_INVALID_ARGUMENT
    assert lib.dspark_prune_lengths(None, 2, 4, thr.data_ptr(), lens.data_ptr(), None) == \
        dsp.DSPARK_ERR_INVALID_ARGUMENT
    assert lib.dspark_prune_lengths(None, 0, 4, None, None, None) == dsp.DSPARK_OK
