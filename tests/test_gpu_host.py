"""The pinned-host entry point (mxfp4_block_scaled_fos_b200/host.py): a batch
copied in, quantized and copied back in chunks of entries on three streams
gives the same bytes as one fos.quantize call over the whole batch on the
device, for every chunk size (including one entry, and chunks that do not
divide the batch), for 4/6, 6-only and MXFP4, and for stochastic rounding,
whose counters must follow the global element index across chunks."""
import pytest
import torch

import mxfp4_block_scaled_fos_b200 as F
from mxfp4_block_scaled_fos_b200.host import HostQuantizer

from helpers import assert_bytes_equal, require_gpu

pytestmark = pytest.mark.gpu


def _batch(batch, rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    s = torch.exp2(torch.randint(-8, 8, (batch, 1, 1), generator=g).float())
    return (torch.randn(batch, rows, cols, generator=g) * s).to(torch.bfloat16)


@pytest.mark.parametrize("fmt,rounding", [("nvfp4_46", "rne"), ("nvfp4_46", "sr"), ("nvfp4_6", "rne"),
                                          ("mxfp4", "rne")])
@pytest.mark.parametrize("chunk", [1, 3, 4, 7])
def test_host_pipeline_equals_one_device_call(fmt, rounding, chunk):
    dev = require_gpu()
    batch, rows, cols = 7, 48, 320
    x = _batch(batch, rows, cols, 11 + chunk)
    hq = HostQuantizer(batch, rows, cols, fmt=fmt, rounding=rounding, seed=5, chunk=chunk, device=dev)
    h_x = x.pin_memory()
    h_codes, h_scales, h_ts = hq.host_outputs()
    for _ in range(2):   # a second pass reuses every buffer, stream and event
        hq(h_x, h_codes, h_scales, h_ts)
        torch.cuda.current_stream().synchronize()
    assert int(hq.status.item()) == 0
    ref, _ = F.quantize(x.to(dev), fmt=fmt, rounding=rounding, seed=5, choice=False)
    torch.cuda.synchronize()
    assert_bytes_equal(h_codes.numpy(), ref.codes.cpu().numpy(), "codes")
    assert_bytes_equal(h_scales.numpy(), ref.scales.cpu().numpy(), "scales")
    if fmt != "mxfp4":
        assert torch.equal(h_ts.view(torch.int32), ref.tensor_scale.cpu().view(torch.int32))


def test_host_pipeline_argument_checks():
    dev = require_gpu()
    hq = HostQuantizer(2, 16, 64, device=dev)
    h_codes, h_scales, h_ts = hq.host_outputs()
    with pytest.raises(ValueError):
        hq(torch.zeros(2, 16, 64, dtype=torch.bfloat16), h_codes, h_scales, h_ts)   # not pinned
    with pytest.raises(ValueError):
        hq(torch.zeros(2, 16, 64, dtype=torch.bfloat16).pin_memory(), h_codes, h_scales, None)
