"""The binding's stream lookup on a GPU: with no stream argument a call runs on torch's current
stream of the tensors' device, the same handle torch.cuda.current_stream gives, also inside a
torch.cuda.stream context and after torch.cuda.set_stream."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_default_stream_is_torchs_current_stream(fp8q):
    dev = torch.device("cuda", torch.cuda.current_device())
    assert fp8q._stream(None, dev) == torch.cuda.current_stream(dev).cuda_stream
    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):
        assert fp8q._stream(None, dev) == side.cuda_stream == torch.cuda.current_stream(dev).cuda_stream
    assert fp8q._stream(None, dev) == torch.cuda.current_stream(dev).cuda_stream
    assert fp8q._stream(side, dev) == side.cuda_stream
    assert fp8q._stream(side.cuda_stream, dev) == side.cuda_stream


def test_a_call_on_a_side_stream_is_ordered_on_it(fp8q, orc):
    """Per-token quant enqueued inside a torch.cuda.stream context, the input written just before on
    the same side stream: the codes match the oracle's, so the call ran on that stream."""
    import numpy as np
    from gpu_util import host
    dev = torch.device("cuda", torch.cuda.current_device())
    side = torch.cuda.Stream(dev)
    x = torch.zeros((64, 1024), dtype=torch.bfloat16, device=dev)
    q = torch.empty((64, 1024), dtype=torch.uint8, device=dev)
    s = torch.empty((64, 8), dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev).manual_seed(5)
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        torch.cuda._sleep(2_000_000)                        # keep the side stream busy a while
        x.copy_(torch.randn((64, 1024), generator=g, device=dev).to(torch.bfloat16))
        fp8q.fp8q_per_token_group_quant(x, q, s, 128, fp8q.E4M3FN)
    side.synchronize()
    qo, so = orc.per_token_group_quant(host(x.view(torch.int16)), orc.BF16, 128, fp8q.E4M3FN)
    np.testing.assert_array_equal(host(q), qo)
    np.testing.assert_array_equal(host(s).view(np.uint32), so.view(np.uint32))
