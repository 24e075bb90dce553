"""The FMA-pipe exponential of the attention kernels' softmax (the library's test hook
vmla_debug_exp2_poly runs the same device function on a buffer), against float64 2^x and CUDA's own
exp2f: relative error <= 7.5e-5 for -125 <= x <= 121, and 2^-125 within that error below the clamp,
for -inf and for NaN."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

BOUND = 7.5e-5


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from rank_latent_kv_vmla_b200 import vmla
    return vmla


def _inputs():
    sweep = np.linspace(-130.0, 121.0, 1_000_000, dtype=np.float32)
    ints = np.arange(-130, 122, dtype=np.float32)
    halves = ints + np.float32(0.5)                       # the ends of the fitted interval
    near = np.concatenate([np.nextafter(halves, np.float32(-np.inf)), np.nextafter(halves, np.float32(np.inf))])
    special = np.array([-np.inf, -0.0, 0.0, np.nan, -125.0, -124.5, 120.0, 121.0], dtype=np.float32)
    x = np.concatenate([sweep, ints, halves, near]).astype(np.float32)
    return np.concatenate([x[x <= 121.0], special])


def test_exp2_poly_error_bound(V):
    x = _inputs()
    y = V.debug_exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    xd = x.astype(np.float64)
    floor = np.isnan(xd) | (xd < -125.0)                  # below the clamp, -inf and NaN
    live = ~floor
    ref = np.exp2(xd[live])
    rel = np.abs(y[live] - ref) / ref
    assert rel.max() <= BOUND, (float(rel.max()), float(xd[live][rel.argmax()]))
    assert floor.sum() > 0
    rel_floor = np.abs(y[floor] - 2.0 ** -125) / 2.0 ** -125
    assert rel_floor.max() <= BOUND, float(rel_floor.max())
    # the bound is tight: the fitted cubic's equi-oscillating error reaches close to it
    assert rel.max() >= 0.9 * BOUND


def test_exp2_poly_against_cuda_exp2f(V):
    x = torch.from_numpy(_inputs()).cuda()
    ok = torch.isfinite(x) & (x >= -125.0) & (x <= 121.0)
    y = V.debug_exp2_poly(x)
    ref = torch.exp2(x)                                    # CUDA's exp2f, single precision
    rel = ((y[ok].double() - ref[ok].double()).abs() / ref[ok].double()).max().item()
    assert rel <= BOUND + 2.0 ** -21, rel                  # exp2f itself is within 2 ulp


def test_exp2_poly_empty_and_bad_arguments(V):
    assert V.debug_exp2_poly(torch.empty(0, device="cuda")).numel() == 0
    st = V.LIB.vmla_debug_exp2_poly(None, None, 4, None)
    assert st == V.VMLA_ERR_INVALID_ARG
