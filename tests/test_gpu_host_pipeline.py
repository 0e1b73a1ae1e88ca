"""The host-input pass (copies of token chunks overlapped with the factor
accumulation on a second stream) gives the same results as the pass over
device-resident inputs with the same chunking: the same launches in the same
order, so every output must be identical.  Two calls in a row check that a
call's copies do not overwrite inputs the previous call still reads."""
import pytest
import torch

from post_quantization_kronq_b200.layer import LayerPass
from synth import llama_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("m,n,T,chunk,bits", [(256, 384, 5000, 1024, 4), (192, 256, 3000, 3000, 2)])
def test_run_from_host_equals_device_run(m, n, T, chunk, bits):
    W, X, G = llama_layer(m, n, T, seed=3, device=DEV)
    ref = LayerPass(m, n, bits=bits, group=128, seed=3)
    ref.run(X, G, W, chunk=chunk)
    torch.cuda.synchronize()
    hX, hG, hW = (t.cpu().pin_memory() for t in (X, G, W))
    X2, G2, W2 = torch.empty_like(X), torch.empty_like(G), torch.empty_like(W)
    lp = LayerPass(m, n, bits=bits, group=128, seed=3)
    for _ in range(2):
        lp.run_from_host(hX, hG, hW, X2, G2, W2, chunk=chunk)
    torch.cuda.synchronize()
    assert int(lp.info.item()) == 0
    assert lp.sens == ref.sens
    for name in ("HX", "HG", "Wt", "d_in", "d_out", "codes", "scales", "zeros"):
        assert torch.equal(getattr(lp, name), getattr(ref, name)), name
    if ref.packed is not None:
        assert torch.equal(lp.packed, ref.packed)
    assert torch.equal(X2, X) and torch.equal(G2, G) and torch.equal(W2, W)
