"""The L2 read-bandwidth measurement kernel that bench.py uses for the fine
kernel's L2 roofline: it completes without a timeout and reports a rate that
is above HBM speed (the buffer is L2-resident) and below an impossible one."""
import pytest
import torch

from trainable_block_sparse_cube_b200 import build as vsa_build
from trainable_block_sparse_cube_b200 import vsa

pytestmark = pytest.mark.gpu


def test_l2_read_measurement():
    vsa_build.build()
    assert torch.cuda.is_available()
    buf = torch.zeros(48 << 20, dtype=torch.uint8, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    vsa.measure_l2_read(buf, 2, status)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    vsa.measure_l2_read(buf, 10, status)
    b.record()
    b.synchronize()
    assert int(status[0]) == 0
    gbs = 10 * buf.numel() / (a.elapsed_time(b) * 1e-3) / 1e9
    print(f"L2 -> SM bulk-copy read: {gbs:.0f} GB/s")
    assert 3000 < gbs < 60000
    with pytest.raises(vsa.VSAError):
        vsa.measure_l2_read(buf[:100], 1, status)       # fewer than 16384 bytes
