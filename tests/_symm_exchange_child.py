"""Child process of test_peer_exchange_symmetric_memory_group_of_one: one NCCL rank on one
GPU builds its exchange buffer in torch symmetric memory and runs two head-sharded steps
through the fused exchange; prints OK when both equal focus_evict bit for bit."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import attention_delta_token_b200 as F  # noqa: E402
import synth  # noqa: E402
from attention_delta_token_b200 import parallel  # noqa: E402
from focus_testutil import run_evict  # noqa: E402


def main():
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        ex = None
        for seed in (840, 841):
            p = synth.make_problem(1, seed=seed, overrides=dict(R=6))
            g = p.to("cuda")
            dims = F.make_dims(p.R, p.B, p.Hq, p.Hkv, p.d, p.H, p.scale, p.pool_window)
            if ex is None:
                ex = parallel.PeerExchange.symmetric(dims)
            fused = run_evict(g)
            cap = F.plan_capacity(p.decoded, p.budget)
            kept = torch.empty(cap, dtype=torch.int32, device="cuda")
            cu = torch.empty(p.R + 1, dtype=torch.int32, device="cuda")
            packed = torch.empty(cap, p.H, dtype=torch.bfloat16, device="cuda")
            ws = parallel.evict_head_sharded(dims, 0, 1, g.q0, g.k0_prefix, g.k0_block, g.q1,
                                             g.k1_prefix, g.k1_block, g.cu_prefix, g.hidden,
                                             g.decoded, g.budget, kept, cu, packed, exchange=ex)
            assert F.focus_read_device_status(ws) == 0
            assert F.focus_read_device_status(ex.push_ws) == 0
            np.testing.assert_array_equal(cu.cpu().numpy(), fused["cu_seqlens"])
            np.testing.assert_array_equal(kept.cpu().numpy(), fused["kept"])
            np.testing.assert_array_equal(
                packed.view(torch.int16).cpu().numpy().view(np.uint16), fused["packed"])
        del ex
        torch.cuda.synchronize()
        print("OK", flush=True)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
