"""One rank over NCCL on cuda:0: the sequence-sharded forward's exchange path
and the data-parallel gradient all-reduce, run for real through NCCL with a
world of one (no peer to wait for).  Run as a child process by
test_gpu_nccl_one_rank.py; exits 0 when every check passes."""
import datetime
import os
import sys

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from selective_state_space_50_b200 import dp, seqpar, ssm_scan  # noqa: E402
from selective_state_space_50_b200.workloads import Workload, generate, to_torch  # noqa: E402


def main():
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        w = Workload("nccl1", 2, 256, 1200, 16, "bf16", seed=5, A_dist="neg_lognormal",
                     D_dist="u0.5_1.5")
        dv = to_torch(generate(w), w, "cuda:0")
        args = (dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"], dv["delta_bias"], True)
        out, last = seqpar.cuda_forward_rank(*args)
        ref, rlast, _ = ssm_scan.selective_scan_fwd(*args, return_last_state=True)
        torch.cuda.synchronize()
        # a world of one: rank 0's pass 1 is the whole sequence (the variant
        # of the kernel that also sums Δ, so compare within rounding)
        assert torch.allclose(out.float(), ref.float(), rtol=2e-2, atol=2e-2), "sharded forward differs"
        assert torch.allclose(last, rlast, rtol=1e-4, atol=1e-4), "sharded final state differs"
        stacked = seqpar.all_gather_stacked(rlast)
        torch.cuda.synchronize()
        assert stacked.shape == (1,) + tuple(rlast.shape) and torch.equal(stacked[0], rlast)
        g = {"dA": torch.randn(1200, 16, device="cuda:0"), "dD": torch.randn(1200, device="cuda:0"),
             "ddelta_bias": torch.randn(1200, device="cuda:0")}
        before = {k: v.clone() for k, v in g.items()}
        dp.allreduce_param_grads(g)
        torch.cuda.synchronize()
        for k in g:
            assert torch.equal(g[k], before[k]), k
    finally:
        dist.destroy_process_group()
    print("nccl one-rank checks ok")


if __name__ == "__main__":
    main()
