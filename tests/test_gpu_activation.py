"""The fast GELU forms of the tensor-core kernels against CUDA's erff-based
GELU and the oracle's exact GELU, on a dense grid and edge values, through
deltakv_test_activation (include/deltakv_testing.h).

gelu_fast is relu(x) - g(|x|) with the builder's own degree-11 least-squares
fit of g(a) = a Phi(-a) on [0, 5]; its stated bound is |error| <= 1.1e-5 for
every finite x.  gelu_fast2 evaluates the same polynomial with packed fp32x2
instructions, which round every lane like fmaf, so it must equal gelu_fast
bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_strided_b200 import build
    build.build()
    oracle.build()


def _inputs():
    grid = np.linspace(-12.0, 12.0, 1 << 20, dtype=np.float64)
    f32 = np.float32
    edges = [0.0, -0.0, 5.0, -5.0, np.nextafter(f32(5), f32(6)), np.nextafter(f32(5), f32(4)),
             np.nextafter(f32(-5), f32(-6)), np.nextafter(f32(-5), f32(-4)), 1e-40, -1e-40, 1e-30, -1e-30,
             3e38, -3e38, 1e6, -1e6, 40.0, -40.0]
    return torch.tensor(np.concatenate([grid, np.array(edges, dtype=np.float64)]), dtype=torch.float32)


def _run(form, x):
    xd = x.cuda()
    y = torch.empty_like(xd)
    dkv.test_activation(form, xd, y)
    torch.cuda.synchronize()
    return y.cpu()


def test_gelu_fast_within_its_bound_of_exact_gelu():
    x = _inputs()
    fast = _run(dkv.TEST_ACT_GELU_FAST, x).double().numpy()
    erff = _run(dkv.TEST_ACT_GELU_ERFF, x).double().numpy()
    xs = x.double().numpy()
    # exact GELU from the oracle (fp64) on a subsample, erff-based on all
    sub = np.arange(0, xs.size, 97)
    exact = np.array([oracle.act(oracle.ACT_GELU_ERF, float(v)) for v in xs[sub]])
    # 1.1e-5 for the fit plus the float32 rounding of the result
    tol = 1.1e-5 + 2.0 ** -23 * np.abs(exact)
    assert np.all(np.abs(fast[sub] - exact) <= tol), float(np.max(np.abs(fast[sub] - exact) - tol))
    tol_all = 1.1e-5 + 2.0 ** -22 * np.abs(erff)
    assert np.all(np.abs(fast - erff) <= tol_all), float(np.max(np.abs(fast - erff) - tol_all))


def test_gelu_fast2_equals_gelu_fast_bitwise():
    x = _inputs()
    a = _run(dkv.TEST_ACT_GELU_FAST, x)
    b = _run(dkv.TEST_ACT_GELU_FAST2, x)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_tanh_form_matches_the_oracle():
    x = _inputs()[::31]
    got = _run(dkv.TEST_ACT_GELU_TANH, x).double().numpy()
    want = np.array([oracle.act(oracle.ACT_GELU_TANH, float(v)) for v in x.double().numpy()])
    assert np.all(np.abs(got - want) <= 2e-6 + 4e-7 * np.abs(want))


# relative error bound of the special-function unit's tanh.approx.f32, as
# measured on B200 over a dense grid of [-20, 20] (the decode form's tanh)
TANH_APPROX_REL = 2.0 ** -10.5
# the fitted argument's distance from exact GELU with an exact tanh
TANHFIT_FORM_ERR = 2.6e-5


def test_decode_form_within_its_bound_of_exact_gelu():
    """gelu_tanhfit2 (the decode token loop's GELU) against the oracle's exact
    GELU: within the fit's own error plus what the hardware tanh's relative
    error can move x/2 (1 + tanh(y)), i.e. |x|/2 |tanh y| TANH_APPROX_REL."""
    x = _inputs()
    x = x[torch.isfinite(x) & (x.abs() <= 1e4)]
    got = _run(dkv.TEST_ACT_GELU_TANHFIT2, x).double().numpy()
    xs = x.double().numpy()
    sub = np.arange(0, xs.size, 53)
    exact = np.array([oracle.act(oracle.ACT_GELU_ERF, float(v)) for v in xs[sub]])
    tol = TANHFIT_FORM_ERR + 0.5 * np.abs(xs[sub]) * TANH_APPROX_REL + 2.0 ** -22 * np.abs(exact)
    err = np.abs(got[sub] - exact)
    assert np.all(err <= tol), (float(np.max(err - tol)), float(xs[sub][np.argmax(err - tol)]))
    # saturation: beyond |x| = 8 the form returns x or 0
    big = np.abs(xs) > 8
    assert np.allclose(got[big], np.where(xs[big] > 0, xs[big], 0.0), rtol=1e-6, atol=1e-5)
    print(f"decode GELU: max |err| {err.max():.2e}, rms {np.sqrt(np.mean(err ** 2)):.2e}")
