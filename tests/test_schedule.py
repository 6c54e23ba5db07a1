"""GPU tile schedule vs the pure-Python schedule, bit for bit."""
import numpy as np
import pytest
import torch

from oracle.schedule import tile_schedule
from workloads import make_workload, offsets_from_lengths

pytestmark = pytest.mark.gpu


def gpu_schedule(gdpa, qo, ko, BM, BN, window=(-1, -1), H=1, D=64):
    B = len(qo) - 1
    dev = torch.device("cuda")
    p = gdpa.make_params(B, H, D, int(qo[-1]), int(ko[-1]), window=window)
    tq = torch.tensor(qo, dtype=torch.int32, device=dev)
    tk = torch.tensor(ko, dtype=torch.int32, device=dev)
    ts = torch.full((B + 1,), -7, dtype=torch.int32, device=dev)
    order = torch.full((max(B, 1),), -7, dtype=torch.int32, device=dev)
    rc = gdpa.gdpa_tile_schedule(p, BM, BN, tq.data_ptr(), tk.data_ptr(), ts.data_ptr(),
                                 order.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return ts.cpu().tolist(), order.cpu().tolist()[:B]


@pytest.mark.parametrize("lens", [
    [0], [1], [127], [128], [129], [0, 0, 0],
    [0, 1, 127, 128, 129, 1000, 5000, 1, 0],
])
@pytest.mark.parametrize("window", [(-1, -1), (127, 0), (3, 9)])
def test_edge_lengths(cuda_lib, lens, window):
    qo = offsets_from_lengths(np.array(lens))
    ko = offsets_from_lengths(np.array(lens[::-1]))
    for BM, BN in ((128, 128), (128, 64), (64, 16)):
        ts, order = gpu_schedule(cuda_lib, qo, ko, BM, BN, window)
        ets, eorder, _ = tile_schedule(qo, ko, BM, BN, *window)
        assert ts == ets and order == eorder


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_workload_schedules(cuda_lib, cfg):
    w = make_workload(cfg)  # full batch sizes; lengths only matter here
    rc, BM, BN = cuda_lib.gdpa_forward_tile_shape(
        cuda_lib.make_params(w.B, w.H, w.D, w.total_q, w.total_kv, phi=w.phi,
                             max_seqlen_kv=w.max_kv))
    assert rc == 0
    ts, order = gpu_schedule(cuda_lib, w.q_offsets, w.kv_offsets, BM, BN,
                             (w.window_left, w.window_right))
    ets, eorder, _ = tile_schedule(w.q_offsets, w.kv_offsets, BM, BN, w.window_left,
                                   w.window_right)
    assert ts == ets and order == eorder


def test_largest_batch(cuda_lib):
    rng = np.random.default_rng(9)
    lens = rng.integers(0, 3000, 16384)
    qo = offsets_from_lengths(lens)
    ko = offsets_from_lengths(rng.integers(0, 300, 16384))
    ts, order = gpu_schedule(cuda_lib, qo, ko, 128, 128, (200, 0))
    ets, eorder, _ = tile_schedule(qo, ko, 128, 128, 200, 0)
    assert ts == ets and order == eorder
