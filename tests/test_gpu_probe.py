"""The tensor-core peak probe runs, completes within its bounds and reports a
plausible rate: the dense INT8 / FP8 multiply-adds per clock per SM of a B200
lie between a quarter of and just above the 8,192 its spec rate implies (4.5
POPS dense at 148 SMs and 1.965 GHz, 2 operations per multiply-add)."""
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [0, 1])
def test_tc_probe_rate_is_plausible(kind):
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    cycles = torch.zeros(1, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    iters = 4096
    qa.qattn_tc_probe(kind, iters, n_sm, cycles, err)
    qa.qattn_check(err)
    macs_per_clk = iters * 128 * 256 * 32 / int(cycles.item())
    assert 2048 <= macs_per_clk <= 8192 * 1.05, macs_per_clk
