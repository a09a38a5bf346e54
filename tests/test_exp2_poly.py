"""The softmax's FMA-pipe exponential: 2^x = 2^round(x) * p(x - round(x)) with
a degree-3 polynomial p fitted for relative error on [-1/2, 1/2].

CPU: the algorithm evaluated in float32 with numpy stays within 1e-4 relative
of exact 2^x. GPU (marked gpu): the device function the forward kernel uses
agrees with exact 2^x and with the MUFU ex2.approx path.
"""
import numpy as np
import pytest

C = np.array([0.99992812, 0.69326097, 0.24261054, 0.05517132], dtype=np.float32)


def poly_exp2_f32(x):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-120))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(C[3])
    for c in C[2::-1]:
        p = (p * f + c).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_poly_exp2_relative_error_bound_cpu():
    x = np.linspace(-119.9, 8.0, 2_000_001, dtype=np.float32)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(poly_exp2_f32(x).astype(np.float64) / ref - 1)
    assert rel.max() < 1e-4
    # integers are exact up to the polynomial's value at 0 (error < 1e-4)
    xi = np.arange(-100, 9, dtype=np.float32)
    np.testing.assert_allclose(poly_exp2_f32(xi), np.exp2(xi), rtol=1e-4)


def test_poly_exp2_clamps_below():
    y = poly_exp2_f32(np.array([-200.0, -1000.0, -121.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y <= 2.0 ** -119)


@pytest.mark.gpu
def test_device_exp2_paths_match_exact():
    torch = pytest.importorskip("torch")
    import block_sparse_attention_13_b200 as bsa
    x = torch.linspace(-119.9, 8.0, 1 << 20, dtype=torch.float32, device="cuda")
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    bsa.bsa_selftest_exp2(x, yp, ym)
    torch.cuda.synchronize()
    xd = x.double().cpu().numpy()
    ref = np.exp2(xd)
    yp_np = yp.double().cpu().numpy()
    assert np.max(np.abs(yp_np / ref - 1)) < 1e-4
    assert np.max(np.abs(ym.double().cpu().numpy() / ref - 1)) < 1e-5
    # the device polynomial equals its float32 emulation up to FMA contraction
    np.testing.assert_allclose(yp_np, poly_exp2_f32(x.cpu().numpy()), rtol=2e-6)
