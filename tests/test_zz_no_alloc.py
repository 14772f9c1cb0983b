"""The allocation-free attention entry point (GPU).

Some callers cannot allocate device memory: a plug-in inside an engine that owns
all device memory and passes it only the tensors of the call, or a decode loop
that must not call cudaMalloc because it can synchronise the device.  For them
``asp_sparse_attend_noalloc`` keeps the split-K partials in a fixed array inside
the library.  This file checks, through the C ABI, that it gives the same output
as ``asp_sparse_attend`` with a workspace, on two calls in a row (the second call
reuses the array the first one left behind).
"""
import pytest
import torch

import query_predicted_token_b200 as asp
from query_predicted_token_b200 import _lib as L
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
OUT_ATOL = 2e-2   # bf16 output tolerance of the parity tests


def _cache(B, Hkv, T, d, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    return k, v


def _noalloc(q, kv, idx, cnt, C, out, lse):
    return L.lib().asp_sparse_attend_noalloc(q.data_ptr(), L.ASP_BF16, q.shape[1], kv.ref, idx.data_ptr(),
                                             cnt.data_ptr(), C, None, 0, out.data_ptr(), lse.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("B,Hq,Hkv,d,T,C", [(8, 32, 8, 128, 4096, 2048), (64, 32, 8, 128, 1100, 1024)],
                         ids=["per_item_kernel", "gather_kernel"])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(B, Hq, Hkv, d, T, C):
    from query_predicted_token_b200 import build
    build.build()
    need = asp.attend_workspace_bytes(B, Hq, Hkv, d, C)
    assert 0 < need <= (2 << 20)          # the partials do use scratch, and fit the fixed array
    k, v = _cache(B, Hkv, T, d, seed=5)
    kv = asp.KV(k, v)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    for call, seed in enumerate((11, 12)):
        g = torch.Generator().manual_seed(seed)
        q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16).to(DEV)
        idx, cnt = synth.random_selection(B, Hkv, C, [T] * B, seed=seed)
        idx, cnt = idx.to(DEV), cnt.to(DEV)
        ref = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=DEV)
        ref_lse = torch.empty(B, Hq, device=DEV)
        asp.sparse_attend(q, kv, idx, cnt, C, ref, ref_lse, workspace=ws)
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
        lse = torch.full((B, Hq), float("nan"), device=DEV)
        assert _noalloc(q, kv, idx, cnt, C, out, lse) == L.ASP_OK, f"call {call}"
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= OUT_ATOL, f"call {call}: max abs difference {err}"
        assert torch.allclose(lse, ref_lse, rtol=1e-5, atol=1e-4), f"call {call}: lse"
    # and one unit of the last call against the oracle's attention over the same rows
    import oracle
    G = Hq // Hkv
    b, h = B - 1, Hkv - 1
    K, V = k[b, h].double().cpu().numpy(), v[b, h].double().cpu().numpy()
    S = idx[b, h, :int(cnt[b, h])].cpu().numpy()
    ref_o, _ = oracle.attend_set(q[b, h * G:(h + 1) * G].double().cpu().numpy(), K, V, S)
    err = (out[b, h * G:(h + 1) * G].double().cpu().numpy() - ref_o).__abs__().max()
    assert err <= OUT_ATOL, f"against the oracle: {err}"
    assert asp.device_status() == 0
