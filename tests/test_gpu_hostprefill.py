"""Overlapped prefill from pinned host memory (HostPrefill): the chunked,
three-stream path gives exactly the device-resident result, on two runs in a row
and for a chunk count that does not divide the KV heads."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import dynamic_sparse_attention_build_b200 as m
    return m


@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_host_prefill_equals_device_path(dsa, chunks):
    N, d, B = 3000, 128, 64
    Q, K, V = synth.random_qkv(8, 4, N, d, seed=31)
    pats = [dict(kind="vs", last_q=64, n_vert=60, n_slash=50), dict(kind="ashape", sink=64, window=256),
            dict(kind="block_topk", topk=6), dict(kind="block_threshold", alpha=0.5),
            dict(kind="moba", topk=3), dict(kind="vs", last_q=32, n_vert=20, n_slash=200),
            dict(kind="ashape", sink=0, window=128), dict(kind="block_topk", topk=2)]
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    idx = dsa.build_indices(Qd, Kd, pats, B)
    O_ref, _ = dsa.sparse_prefill(Qd, Kd, Vd, idx)
    torch.cuda.synchronize()
    hp = dsa.HostPrefill(8, 4, N, d, pats, B, chunks=chunks)
    Qh, Kh, Vh = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    for _ in range(2):
        Oh = torch.empty_like(Q).pin_memory()
        hp.run(Qh, Kh, Vh, Oh)
        torch.cuda.current_stream().synchronize()
        st, det = hp.status()
        assert st == 0, (st, det)
        assert torch.equal(Oh, O_ref.cpu())
