"""convrot_linear_noalloc: the whole layer for callers that cannot give the
library device memory (a plugin whose host runtime owns every allocation, or
code that must not call cudaMalloc on its path).  It keeps the packed
activations in the library's fixed 16 MiB scratch array instead of a caller
workspace.  Checked through the C ABI against convrot_linear, the entry point
with a caller workspace.  Both run the same kernels on the same inputs, so the outputs
must be bit-identical; the check runs on calls in a row of different shapes
(each later call starts with an earlier call's leftovers in the shared
array), including a 1-4 token call, which takes the one-kernel form and
touches no scratch.

The file name sorts last so that a run stopping at the first failure has
already run every other test."""
import pytest
import torch

import rotated_w4a4_quantized_b200 as cr
from rotated_w4a4_quantized_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from rotated_w4a4_quantized_b200 import build
    build.build()


def _case(M, K, N, group, seed):
    lt = wl.make_random_layer(M, K, N, group, seed=seed)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, group)
    return x, qw, sw, b


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    # first call fills more of the shared array than the second one reads
    for (M, K, N, group, seed) in [(1500, 4096, 640, 64, 21), (37, 1024, 264, 256, 22),
                                   (3, 4096, 520, 64, 24), (300, 2048, 200, 256, 25)]:
        x, qw, sw, b = _case(M, K, N, group, seed)
        y_ws = cr.convrot_linear(x, qw, sw, b, group)
        y_na = cr.convrot_linear_noalloc(x, qw, sw, b, group)
        torch.cuda.synchronize()
        assert cr.convrot_check_device_error() == 0
        assert torch.equal(y_na.view(torch.int16), y_ws.view(torch.int16)), (M, K, N)


def test_noalloc_rejects_requests_beyond_the_scratch_limit():
    x, qw, sw, b = _case(8192, 4096, 16, 64, 23)     # needs 16 MiB + 32 KiB
    assert cr.convrot_linear_workspace_size(8192, 4096) > 16 << 20
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_linear_noalloc(x, qw, sw, b, 64)
    assert e.value.status == 9                        # CONVROT_ERR_SCRATCH_LIMIT
