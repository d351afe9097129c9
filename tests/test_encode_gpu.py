"""GPU anisotropic code assignment (ah_encode) against the oracle's
restatement (oracle.encode): codes and passes used bit-identical.  Both take
every decision in fp64 with the same operation order."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def enc():
    from mips_ivf_centroid_b200 import build
    build.build()
    from mips_ivf_centroid_b200 import encode
    return encode


def _case(n, d, dpb, seed, unit=True, scale=0.3):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d)).astype(np.float32)
    if unit:
        X /= np.linalg.norm(X, axis=1, keepdims=True)
    cb = (rng.standard_normal((d // dpb, 16, dpb)) * scale).astype(np.float32)
    return X, cb


@pytest.mark.parametrize("n,d,dpb,T,passes,unit", [
    (5000, 100, 2, 0.2, 10, True),      # GloVe-shaped blocks
    (3000, 128, 4, 0.05, 10, True),     # dims_per_block 4
    (2000, 34, 1, 0.3, 10, False),      # odd blocks count per pair, varied norms
    (2000, 64, 2, 0.0, 10, True),       # T = 0: L2 codes
    (1000, 32, 2, 0.5, 0, True),        # no descent
    (1000, 48, 2, 0.2, 100, True),      # to convergence
    (400, 1536, 4, 0.05, 10, True),     # OpenAI-shaped: codebook and unit vectors outside shared memory
])
def test_codes_match_oracle(enc, n, d, dpb, T, passes, unit):
    X, cb = _case(n, d, dpb, seed=n + d + dpb, unit=unit)
    if not unit:
        X[:50] *= np.float32(0.1)       # norms at or below T: eta = 1
        X[50] = 0.0                      # zero vector
    want, want_used = oracle.encode(X, cb, T, passes)
    codes, used = enc(torch.from_numpy(X).cuda(), torch.from_numpy(cb).cuda(), T, passes)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), want)
    np.testing.assert_array_equal(used.cpu().numpy(), want_used)


def test_encode_errors_and_empty(enc):
    from mips_ivf_centroid_b200 import AhError
    X, cb = _case(10, 16, 2, 1)
    Xg, cbg = torch.from_numpy(X).cuda(), torch.from_numpy(cb).cuda()
    c, u = enc(Xg[:0], cbg, 0.2, 10)
    assert c.shape == (0, 4)
    with pytest.raises(AhError) as e:
        enc(Xg, cbg, 0.2, 5000)
    assert e.value.status == 1
    with pytest.raises(AhError) as e:
        enc(Xg[:, :14].contiguous(), cbg[:7].contiguous(), 0.2, 5)   # d = 14 is not a multiple of 2 * 2
    assert e.value.status == 1
