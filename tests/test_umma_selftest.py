"""The tcgen05 operand layouts and descriptors (K-major and N-contiguous
128-byte-swizzled bf16 tiles) against a plain fp32 matmul of the same bf16
values, through the lola_selftest_umma hook."""
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from hybrid_linear_attention_lola_b200 import lola as L


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_linear_attention_lola_b200 import build
    build.build()


@pytest.mark.parametrize("layout,N,K", [(0, 80, 128), (0, 144, 256), (0, 128, 64), (0, 16, 16),
                                        (1, 128, 128), (1, 64, 64), (1, 256, 32), (1, 128, 256),
                                        (2, 128, 64), (2, 64, 16), (3, 16, 64), (3, 16, 48)])
def test_umma_matches_matmul(layout, N, K):
    g = torch.Generator().manual_seed(1000 + N + K + layout)
    a_mn = layout >= 2
    b_kmajor = layout in (0, 3)
    A = torch.randn(K, 128, generator=g).to(torch.bfloat16) if a_mn else \
        torch.randn(128, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16) if b_kmajor else \
        torch.randn(K, N, generator=g).to(torch.bfloat16)
    want = (A.float().T if a_mn else A.float()) @ (B.float().T if b_kmajor else B.float())
    Ad, Bd = A.cuda(), B.cuda()
    C = torch.full((128, N), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.load_library().lola_selftest_umma(layout, Ad.data_ptr(), Bd.data_ptr(), C.data_ptr(),
                                             N, K, err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rel = (C.cpu() - want).norm() / want.norm()
    assert rel < 1e-5, float(rel)
