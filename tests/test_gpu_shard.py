"""The head-sharded call (dist.attention_shard) on one GPU: running every
rank's share in turn must reproduce the unsharded output bit for bit, since
the selection, the quantisation scales and the output are all per head.
Ranks run one after another in one process: nothing waits on another rank."""
import pytest
import torch

import mixed_precision_bit_quant_b200 as mq
from mixed_precision_bit_quant_b200 import dist as mdist, workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hq,Hkv,N,world", [(1, 32, 8, 2048, 2), (2, 8, 4, 700, 3), (3, 4, 2, 300, 4)])
def test_shards_reassemble_the_unsharded_output(B, Hq, Hkv, N, world):
    w = workloads.custom("shard", B, Hq, Hkv, N, 128, True, "llm", 500, 0, seed=B * N)
    q, k, v = (t.cuda() for t in workloads.generate(w))
    full, _ = mq.attention(q, k, v, True, 500)
    o = torch.full_like(q, float("nan"))
    for rank in range(world):
        mdist.attention_shard(q, k, v, True, rank, world, budget_bp=500, o=o)
    st, word = mq.device_status()
    assert st == 0, f"device watchdog raised {word:#x}"
    assert torch.equal(o, full)
