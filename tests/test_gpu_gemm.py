"""The grouped tcgen05 GEMM core against a plain fp32 PyTorch product of the
same operands (bf16 and fp32-faithful three-plane kinds, all four operand-major combinations,
shapes spanning several tiles with ragged tails)."""

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api as A
    return A


def _operands(batch, M, N, K, a_mn, b_mn, dtype, gen):
    A = torch.randn((batch, M, K), generator=gen, device="cuda").to(dtype)
    B = torch.randn((batch, N, K), generator=gen, device="cuda").to(dtype)
    Ain = A.transpose(1, 2).contiguous() if a_mn else A
    Bin = B.transpose(1, 2).contiguous() if b_mn else B
    return A, B, Ain, Bin


SHAPES = [(1, 128, 256, 64), (3, 200, 328, 136), (2, 384, 520, 1000), (1, 8, 8, 8)]


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("shape", SHAPES)
def test_bf16_gemm_matches_fp32_product(api, shape, a_mn, b_mn):
    batch, M, N, K = shape
    gen = torch.Generator(device="cuda").manual_seed(1234)
    A, B, Ain, Bin = _operands(batch, M, N, K, a_mn, b_mn, torch.bfloat16, gen)
    D = api.gemm(Ain, Bin, kind="bf16", a_mn_major=bool(a_mn), b_mn_major=bool(b_mn))
    ref = torch.bmm(A.double(), B.double().transpose(1, 2))
    # exact bf16 products, fp32 accumulation: error ~ sqrt(K) * 2^-24 * |a||b|
    err = (D.double() - ref).abs().max().item()
    assert err <= 1e-5 * K ** 0.5 * 4, err


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("shape", SHAPES)
def test_split3_gemm_is_fp32_faithful(api, shape, a_mn, b_mn):
    batch, M, N, K = shape
    gen = torch.Generator(device="cuda").manual_seed(99)
    A, B, Ain, Bin = _operands(batch, M, N, K, a_mn, b_mn, torch.float32, gen)
    D = api.gemm(Ain, Bin, kind="split3", a_mn_major=bool(a_mn), b_mn_major=bool(b_mn))
    ref = torch.bmm(A.double(), B.double().transpose(1, 2))
    scale = torch.bmm(A.double().abs(), B.double().abs().transpose(1, 2))
    rel = ((D.double() - ref).abs() / scale).max().item()
    # a single bf16 product would sit near 4e-3 here; the three-plane split reaches the
    # fp32 accumulation level, about sqrt(K) units of 2^-24 relative to sum |a||b|
    assert rel < 4 * 2.0 ** -24 * K ** 0.5, rel


def test_gemm_repeatable_bitwise(api):
    gen = torch.Generator(device="cuda").manual_seed(5)
    A = torch.randn((4, 256, 512), generator=gen, device="cuda").to(torch.bfloat16)
    B = torch.randn((4, 512, 512), generator=gen, device="cuda").to(torch.bfloat16)
    d1 = api.gemm(A, B)
    d2 = api.gemm(A, B)
    assert torch.equal(d1, d2)


MIXED = [("bf16_fold", torch.bfloat16, torch.bfloat16), ("split3_bf16", torch.float32, torch.bfloat16),
         ("bf16_split3", torch.bfloat16, torch.float32)]


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 1), (0, 1)])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("kind,adt,bdt", MIXED)
def test_plane_pairs_are_fp32_faithful(api, kind, adt, bdt, shape, a_mn, b_mn):
    """A bf16 operand is exact in one plane: a bf16 x bf16 product folded in fp32,
    and fp32 x bf16 in three products, reach the fp32 accumulation level."""
    batch, M, N, K = shape
    gen = torch.Generator(device="cuda").manual_seed(7)
    A = torch.randn((batch, M, K), generator=gen, device="cuda").to(adt)
    B = torch.randn((batch, N, K), generator=gen, device="cuda").to(bdt)
    Ain = A.transpose(1, 2).contiguous() if a_mn else A
    Bin = B.transpose(1, 2).contiguous() if b_mn else B
    D = api.gemm(Ain, Bin, kind=kind, a_mn_major=bool(a_mn), b_mn_major=bool(b_mn))
    ref = torch.bmm(A.double(), B.double().transpose(1, 2))
    scale = torch.bmm(A.double().abs(), B.double().abs().transpose(1, 2))
    rel = ((D.double() - ref).abs() / scale).max().item()
    assert rel < 4 * 2.0 ** -24 * K ** 0.5, rel


@pytest.mark.parametrize("kernel", ["auto", "one_cta", "cta_pair"])
@pytest.mark.parametrize("shape", SHAPES)
def test_split2_has_sixteen_bit_products(api, shape, kernel):
    """Two planes per operand and three products: about 16 significant bits per
    product, far better than one bf16 product, far from fp32."""
    batch, M, N, K = shape
    gen = torch.Generator(device="cuda").manual_seed(8)
    A = torch.randn((batch, M, K), generator=gen, device="cuda")
    B = torch.randn((batch, N, K), generator=gen, device="cuda")
    D = api.gemm(A, B, kind="split2", kernel=kernel)
    ref = torch.bmm(A.double(), B.double().transpose(1, 2))
    scale = torch.bmm(A.double().abs(), B.double().abs().transpose(1, 2))
    rel = ((D.double() - ref).abs() / scale).max().item()
    assert rel < 2.0 ** -15, rel


PAIR_SHAPES = [(1, 256, 128, 64), (3, 200, 328, 136), (2, 384, 520, 1000), (1, 8, 8, 8), (5, 640, 256, 512)]


@pytest.mark.parametrize("kernel", ["one_cta", "cta_pair"])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("shape", PAIR_SHAPES)
@pytest.mark.parametrize("kind,adt,bdt", [("split3", torch.float32, torch.float32)] + MIXED)
def test_table_kernels_agree(api, kind, adt, bdt, shape, a_mn, b_mn, kernel):
    """Both table-mode kernels (128 x 128 tiles on one CTA; 256 x 128 tiles on a CTA
    pair sharing tcgen05 cta_group::2) reach the fp32 accumulation level, and give
    the same bits, for every plane pair."""
    batch, M, N, K = shape
    gen = torch.Generator(device="cuda").manual_seed(11)
    A = torch.randn((batch, M, K), generator=gen, device="cuda").to(adt)
    B = torch.randn((batch, N, K), generator=gen, device="cuda").to(bdt)
    Ain = A.transpose(1, 2).contiguous() if a_mn else A
    Bin = B.transpose(1, 2).contiguous() if b_mn else B
    D = api.gemm(Ain, Bin, kind=kind, a_mn_major=bool(a_mn), b_mn_major=bool(b_mn), kernel=kernel)
    ref = torch.bmm(A.double(), B.double().transpose(1, 2))
    scale = torch.bmm(A.double().abs(), B.double().abs().transpose(1, 2))
    rel = ((D.double() - ref).abs() / scale).max().item()
    assert rel < 4 * 2.0 ** -24 * K ** 0.5, rel
    other = api.gemm(Ain, Bin, kind=kind, a_mn_major=bool(a_mn), b_mn_major=bool(b_mn),
                     kernel="cta_pair" if kernel == "one_cta" else "one_cta")
    assert torch.equal(D, other)


BF16_PAIR_SHAPES = [(1, 256, 256, 64), (3, 200, 328, 136), (2, 384, 520, 1000), (1, 8, 8, 8), (4, 640, 768, 512)]


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("shape", BF16_PAIR_SHAPES)
def test_bf16_kernels_agree(api, shape, a_mn, b_mn):
    """The bf16 Newton-Schulz products on one CTA (128 x 256 tiles) and on CTA pairs
    (256 x 256 tiles, tcgen05 cta_group::2): both at the fp32 accumulation level of
    exact bf16 products, and the same bits."""
    batch, M, N, K = shape
    gen = torch.Generator(device="cuda").manual_seed(5)
    A, B, Ain, Bin = _operands(batch, M, N, K, a_mn, b_mn, torch.bfloat16, gen)
    ref = torch.bmm(A.double(), B.double().transpose(1, 2))
    outs = []
    for kernel in ("one_cta", "cta_pair"):
        D = api.gemm(Ain, Bin, kind="bf16", a_mn_major=bool(a_mn), b_mn_major=bool(b_mn), kernel=kernel)
        err = (D.double() - ref).abs().max().item()
        assert err <= 1e-5 * K ** 0.5 * 4, (kernel, err)
        outs.append(D)
    assert torch.equal(outs[0], outs[1])
