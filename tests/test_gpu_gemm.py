"""The tensor-core GEMM the backward is built from, through its test hook, against a
plain PyTorch fp32 product of the same bf16 operands (every operand layout, split-K,
ragged M/N/K)."""
import pytest
import torch

from prototype_sketch_attention_b200 import binding

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,splits", [
    (296, 256, 192, 0, 0, 1), (296, 256, 192, 0, 1, 1), (296, 256, 192, 1, 0, 1),
    (296, 256, 192, 1, 1, 1), (256, 128, 640, 1, 1, 3), (128, 64, 64, 0, 1, 1),
    (1000, 136, 328, 0, 0, 2), (64, 128, 1000, 1, 0, 7)])
def test_gemm_matches_torch(M, N, K, a_mn, b_mn, splits):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N + K)
    A = torch.randn(M, K, device="cuda", generator=g).bfloat16()
    B = torch.randn(N, K, device="cuda", generator=g).bfloat16()
    Am = A.t().contiguous() if a_mn else A
    Bm = B.t().contiguous() if b_mn else B
    out = torch.full((splits, M, N), float("nan"), device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    st = binding.sa_sketch_debug_gemm(Am.data_ptr(), a_mn, Bm.data_ptr(), b_mn, M, N, K, splits,
                                      out.data_ptr(), ws.data_ptr(), 0)
    assert st == 0, binding.sa_status_string(st)
    assert binding.device_status(ws) == 0
    ref = A.float() @ B.float().t()
    got = out.sum(0)
    assert torch.isfinite(got).all()
    assert ((got - ref).norm() / ref.norm()).item() <= 1e-5


def test_gemm_rejects_bad_arguments():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    A = torch.zeros(128, 64, device="cuda").bfloat16()
    out = torch.zeros(128, 128, device="cuda")
    bad = [dict(M=0), dict(splits=0), dict(splits=5), dict(N=130), dict(K=60, a_mn=0)]
    for kw in bad:
        a = dict(M=128, N=128, K=64, a_mn=0, b_mn=0, splits=1)
        a.update(kw)
        st = binding.sa_sketch_debug_gemm(A.data_ptr(), a["a_mn"], A.data_ptr(), a["b_mn"], a["M"],
                                          a["N"], a["K"], a["splits"], out.data_ptr(), ws.data_ptr(), 0)
        assert st == binding.SA_ERR_INVALID_ARG, kw
