"""dspark_attend_no_alloc -- the attention seam for callers that cannot give the
library device scratch memory (its scratch is a static device array inside
libdspark). Checked through the C ABI against dspark_attend, which takes a
caller workspace, on two calls in a row; collected last on purpose."""
import pytest
import torch

from oracle import dspark as O
from parity_util import assert_close, build, ensure_built
from synthetic import small_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_no_alloc_attend_matches_workspace_attend(dtype):
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype=dtype, block_size=8)
    cpu, W, model = build(m, 5)
    tdt = model.kv_torch_dtype              # the seam's tensors are in the KV dtype (fp16 for a bf16 model)
    A, G, nH, nKv, hd = 3, m.block_size, m.num_attention_heads, m.num_global_key_value_heads, m.global_head_dim
    lens = [0, 517, 1000]
    g = torch.Generator().manual_seed(11)
    cache = dsp.KvCache(model, A, 1000)
    cache.k.copy_((torch.randn(cache.k.shape, generator=g) * 0.6).to(tdt))
    cache.v.copy_(torch.randn(cache.v.shape, generator=g).to(tdt))
    cache.set_lengths(lens)
    for call in range(2):                      # two calls in a row share the static scratch
        q = (torch.randn(A, G, nH, hd, generator=g) * 0.6).to(tdt).cuda()
        kb = (torch.randn(A, G, nKv, hd, generator=g) * 0.6).to(tdt).cuda()
        vb = torch.randn(A, G, nKv, hd, generator=g).to(tdt).cuda()
        layer = call % m.num_hidden_layers
        ref = torch.empty(A, G, nH, hd, dtype=tdt, device="cuda")
        got = torch.full_like(ref, float("nan"))
        model.dspark_attend(layer, cache, q, kb, vb, ref, max(lens))
        model.dspark_attend_no_alloc(layer, cache, q, kb, vb, got, max(lens))
        torch.cuda.synchronize()
        assert_close(got.float().cpu().numpy(), ref.float().cpu().numpy(), dtype, f"no-alloc attend, call {call}")
        # and against the oracle's concat-then-attend directly
        kc, vc = cache.k[layer].double().cpu().numpy(), cache.v[layer].double().cpu().numpy()
        for b in range(A):
            want = O.attend_concat(q[b].double().cpu().numpy(), kc[b, :lens[b]], vc[b, :lens[b]],
                                   kb[b].double().cpu().numpy(), vb[b].double().cpu().numpy())
            assert_close(got[b].float().cpu().numpy(), want, dtype, f"no-alloc attend vs oracle, call {call} row {b}")
    assert model.dspark_read_device_status() == 0


def test_no_alloc_attend_refuses_oversized_state():
    import block_draft_model_dspark_b200 as dsp
    m = small_model(dtype="bf16", block_size=8)
    cpu, W, model = build(m, 5)
    A = 300                                    # 300 * 8 heads * 2 parts * 8 * (128 + 2) * 4 B > 16 MiB
    cache = dsp.KvCache(model, A, 64)
    cache.set_lengths([64] * A)
    q = torch.zeros(A, m.block_size, m.num_attention_heads, m.global_head_dim, dtype=model.kv_torch_dtype, device="cuda")
    kv = torch.zeros(A, m.block_size, m.num_global_key_value_heads, m.global_head_dim, dtype=model.kv_torch_dtype,
                     device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(dsp.DsparkError) as ei:
        model.dspark_attend_no_alloc(0, cache, q, kv, kv, out, 64)
    assert ei.value.code == dsp.DSPARK_ERR_WORKSPACE and "16 MiB" in str(ei.value)
