"""Products from the stored form on the GPU against the oracle's dequant_matmul.

The stored form (packed codes, scales, zeros, g_idx) is drawn at random with the
layout gptq_quantize_layer writes; the repack to sweep order must equal the oracle's
packing of the permuted codes bit for bit, and Y = X Q^T must lie within the
rounding bound of its fp32 sums (each sum of C terms formed as s (sum c x - z sum x),
so within C 2^-24 of sum |x| s (c + z), with a factor 4 of slack)."""
import numpy as np
import pytest
import torch

from oracle import gptq_ref as o
from post_weight_quantization_20_b200 import gptq as G
from post_weight_quantization_20_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _stored(R, C, bits, g, act, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 2 ** bits, size=(R, C))
    Gn = (C + g - 1) // g if g > 0 else 1
    scales = rng.uniform(1e-3, 1e-2, size=(R, Gn)).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, size=(R, Gn)).astype(np.float32)
    perm = rng.permutation(C).astype(np.int32) if act else np.arange(C, dtype=np.int32)
    inv = np.empty(C, np.int64)
    inv[perm] = np.arange(C)
    g_idx = inv // g if g > 0 else np.zeros(C, np.int64)
    return codes, scales, zeros, perm, g_idx


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("cols", [32, 96, 4160])
def test_repack_is_the_sweep_order_bitstream(bits, cols):
    codes, _, _, perm, _ = _stored(7, cols, bits, 0, True, bits + cols)
    packed = torch.from_numpy(o.pack(codes, bits).view(np.int32)).to(DEV)
    out = torch.full((7, G.sweep_words(cols, bits)), -1, dtype=torch.int32, device=DEV)
    G.gptq_repack_sweep_order(packed, bits, torch.from_numpy(perm).to(DEV), out)
    torch.cuda.synchronize()
    want = o.pack(codes[:, perm], bits)
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), want)


@pytest.mark.parametrize("R,C", [(300, 2144), (64, 4160), (17, 96)])
@pytest.mark.parametrize("bits,g", [(4, 128), (3, 0), (2, 32), (8, 64)])
@pytest.mark.parametrize("M", [1, 3, 8, 20])
@pytest.mark.parametrize("act", [False, True])
@pytest.mark.parametrize("xdt", [S.F16, S.BF16, S.F32])
def test_dequant_matmul_matches_oracle(R, C, bits, g, M, act, xdt):
    codes, scales, zeros, perm, g_idx = _stored(R, C, bits, g, act, R + C + bits + M)
    X = S.gen_activations(M, C, xdt, S.ActSpec(), seed=M + bits)
    packed = o.pack(codes, bits)
    ref = o.dequant_matmul(S.to_f64(X, xdt), packed, scales, zeros, g_idx, bits)
    dp = torch.from_numpy(packed.view(np.int32)).to(DEV)
    dperm = torch.from_numpy(perm).to(DEV)
    qp = torch.empty(R, G.sweep_words(C, bits), dtype=torch.int32, device=DEV)
    G.gptq_repack_sweep_order(dp, bits, dperm, qp)
    Xd = torch.from_numpy(X.view(np.int16) if xdt == S.BF16 else X).to(DEV)
    if xdt == S.BF16:
        Xd = Xd.view(torch.bfloat16)
    Y = torch.full((M, R), float("nan"), device=DEV)
    G.gptq_dequant_matmul(Xd, qp, torch.from_numpy(scales).to(DEV), torch.from_numpy(zeros).to(DEV),
                          bits, g, dperm if act else None, Y)
    torch.cuda.synchronize()
    got = Y.cpu().numpy().astype(np.float64)
    # fp32 sums of length C formed as s (sum c x - z sum x): each partial sum is
    # bounded by sum |x| s (c + z), so the error is within C * 2^-24 of that (x4 slack)
    mag = np.abs(S.to_f64(X, xdt)) @ (scales[:, g_idx] * (codes + zeros[:, g_idx])).T
    bound = 4 * C * 2.0 ** -24 * mag + 1e-30
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / bound)


@pytest.mark.parametrize("R,C", [(200, 2112), (70, 640), (129, 4160)])
@pytest.mark.parametrize("g", [0, 64, 128])
@pytest.mark.parametrize("M", [1, 2, 5, 8, 11])
@pytest.mark.parametrize("act", [False, True])
@pytest.mark.parametrize("xdt", [S.F16, S.BF16])
def test_dequant_matmul_4bit_shapes(R, C, g, M, act, xdt):
    """4-bit codes with 16-bit X over group sizes 64 / 128 / per row: the same bound as
    above, on row counts that are not a multiple of a CTA's rows, column counts that end
    inside a staged 2048-column chunk with a short last group, and token counts that
    split into blocks of 8."""
    codes, scales, zeros, perm, g_idx = _stored(R, C, 4, g, act, R + C + g + M)
    X = S.gen_activations(M, C, xdt, S.ActSpec(), seed=M + g)
    packed = o.pack(codes, 4)
    ref = o.dequant_matmul(S.to_f64(X, xdt), packed, scales, zeros, g_idx, 4)
    dp = torch.from_numpy(packed.view(np.int32)).to(DEV)
    dperm = torch.from_numpy(perm).to(DEV)
    qp = torch.empty(R, G.sweep_words(C, 4), dtype=torch.int32, device=DEV)
    G.gptq_repack_sweep_order(dp, 4, dperm, qp)
    Xd = torch.from_numpy(X.view(np.int16) if xdt == S.BF16 else X).to(DEV)
    if xdt == S.BF16:
        Xd = Xd.view(torch.bfloat16)
    Y = torch.full((M, R), float("nan"), device=DEV)
    G.gptq_dequant_matmul(Xd, qp, torch.from_numpy(scales).to(DEV), torch.from_numpy(zeros).to(DEV),
                          4, g, dperm if act else None, Y)
    torch.cuda.synchronize()
    got = Y.cpu().numpy().astype(np.float64)
    mag = np.abs(S.to_f64(X, xdt)) @ (scales[:, g_idx] * (codes + zeros[:, g_idx])).T
    bound = 4 * C * 2.0 ** -24 * mag + 1e-30
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / bound)


@pytest.mark.parametrize("R,C", [(300, 2144), (17, 96)])
@pytest.mark.parametrize("g", [0, 128])
@pytest.mark.parametrize("M", [1, 2, 3])
@pytest.mark.parametrize("act", [False, True])
def test_dequant_matmul_half_sums(R, C, g, M, act):
    # 4-bit codes, fp16 X: word sums in half precision, bound 2^-9 sum |x| s c (+ fp32 part);
    # three tokens are more than the half-precision kernel takes, and run in fp32
    codes, scales, zeros, perm, g_idx = _stored(R, C, 4, g, act, R + C + M)
    X = S.gen_activations(M, C, S.F16, S.ActSpec(), seed=M)
    packed = o.pack(codes, 4)
    ref = o.dequant_matmul(S.to_f64(X, S.F16), packed, scales, zeros, g_idx, 4)
    dperm = torch.from_numpy(perm).to(DEV)
    qp = torch.empty(R, G.sweep_words(C, 4), dtype=torch.int32, device=DEV)
    G.gptq_repack_sweep_order(torch.from_numpy(packed.view(np.int32)).to(DEV), 4, dperm, qp)
    Y = torch.full((M, R), float("nan"), device=DEV)
    G.gptq_dequant_matmul(torch.from_numpy(X).to(DEV), qp, torch.from_numpy(scales).to(DEV),
                          torch.from_numpy(zeros).to(DEV), 4, g, dperm if act else None, Y,
                          half_sums=True)
    torch.cuda.synchronize()
    got = Y.cpu().numpy().astype(np.float64)
    x = np.abs(S.to_f64(X, S.F16))
    bound = (2.0 ** -9 * (x @ (scales[:, g_idx] * codes).T)
             + 4 * C * 2.0 ** -24 * (x @ (scales[:, g_idx] * (codes + zeros[:, g_idx])).T) + 1e-30)
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / bound)
