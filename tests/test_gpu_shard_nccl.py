"""ShardedPrefill through a real NCCL process group of one rank on this GPU: the
orchestration's streams, events and in-place collectives (all-gather, broadcast) run
on the device with the library's stages, in both forms, and the result equals the
one-GPU prefill's selection bit for bit and the oracle's attention within the bf16
tolerances.  (Several ranks need several GPUs; their exchange logic is covered by the
gloo tests in test_shard.py and the emulated stages in test_gpu_shard.py.)"""

import math
import socket

import numpy as np
import pytest
import torch

from oracle import spava_oracle as orc
from workloads import CONFIGS

from .helpers import compare_attention, inputs, make_plan

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    import datetime

    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group already exists in this process")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


@pytest.mark.parametrize("overlap", [True, False])
def test_sharded_prefill_one_nccl_rank(nccl_group, overlap):
    from sequence_approximate_attention_b200.sharded import ShardedPrefill
    cfg = CONFIGS["tiny"].with_(n_visual=1024, n_hosts=4, head_dim=128, hq=8, hkv=2, anchor=64, passing=64,
                                probe_r=32, n_text=40)
    g, f64, dev = inputs(cfg)
    sizes = [int(x) for x in g["host_sizes"]]
    plan = make_plan(sab, cfg, sizes)
    sp = ShardedPrefill(plan, 0, 1, plan.shard_owners(1, "zigzag"), group=nccl_group, overlap=overlap)
    k, v = dev["k"].clone(), dev["v"].clone()
    o, lse = sp.forward(dev["q"], k, v)
    torch.cuda.synchronize()
    sab.check_device_error(plan, sp.ws)
    L = sp.layout
    H, rows, P = cfg.n_hosts, plan.score_rows, cfg.passing
    sel = sp.ws[int(L.idx_offset): int(L.idx_offset) + (H - 1) * rows * P * 4].view(torch.int32)
    sel = sel.view(H - 1, rows, P).cpu().numpy().astype(np.int64)
    ref_plan = make_plan(sab, cfg, sizes)
    _, idx1 = sab.score_select(ref_plan, dev["q"], dev["k"])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(sel, idx1.cpu().numpy())
    off = orc.host_offsets(sizes)
    O_ref, L_ref = orc.approx_attention(f64["q"], f64["k"], f64["v"], off, cfg.anchor, sel,
                                        1.0 / math.sqrt(cfg.head_dim))
    compare_attention(o, lse, O_ref, L_ref, f"nccl overlap={overlap}")
    assert torch.equal(k.view(torch.int16), dev["k"].view(torch.int16))   # the anchor broadcast is a no-op here
    ref_plan.close()
    plan.close()
