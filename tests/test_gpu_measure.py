"""The measurement entry points on the GPU: they run to completion without a device error and report the
bytes they move (the benchmark divides those by CUDA-event time)."""
import pytest

torch = pytest.importorskip("torch")
import prefill_sigmoid_top_b200 as moe

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("boxes,stages,contiguous,warps", [(1, 10, False, 1), (2, 5, False, 1), (3, 4, True, 1),
                                                           (2, 2, True, 2), (2, 6, False, 2), (1, 12, False, 4),
                                                           (3, 4, False, 4)])
def test_tma_stream_moves_what_it_reports(boxes, stages, contiguous, warps):
    buf = torch.ones(64 << 20, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    steps = 300  # more than one 112-step panel per CTA, and not a multiple of the stage count
    moved = moe.measure_tma_stream(buf, boxes, stages, contiguous, steps, err, warps=warps)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert moved == sms * steps * boxes * 16384
    assert moe.get_device_error(err) == 0


def test_hbm_read_runs():
    buf = torch.ones(256 << 20, dtype=torch.uint8, device="cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.measure_hbm_read(buf, sink)
    torch.cuda.synchronize()
    assert int(sink.item()) == 0  # ones xor-fold to zero words: the sink is never written


@pytest.mark.parametrize("mix,stages", [(0, 4), (1, 2), (2, 4), (3, 3), (4, 4), (4, 2)])
def test_tma_mix_moves_what_it_reports(mix, stages):
    buf = torch.ones(256 << 20, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    steps = 101  # several 28-step panels per CTA; not a multiple of the stage count or of the 4-step scale groups
    moved = moe.measure_tma_mix(buf, mix, stages, steps, err)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    per_step = {0: 32768, 1: 40960, 2: 47104, 3: 47104, 4: 40960 + 3 * 8192 / 4}[mix]
    assert moved == int(per_step * sms * steps)
    assert moe.get_device_error(err) == 0
