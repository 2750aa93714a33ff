"""Second process of tests/test_gpu_ep.py::test_scatter_into_a_buffer_mapped_from_another_process:
maps the parent's receive buffer from its IPC handle and runs moe_ep_scatter
into it (one rank, one expert: row j of x to row j), then exits 0."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_mixture_experts_04_b200 import api  # noqa: E402


def main() -> int:
    handle, n, d, seed = bytes.fromhex(sys.argv[1]), int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4])
    torch.cuda.set_device(0)
    buf = api.IpcBuffer((n, d), torch.bfloat16, handle=handle)
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((n, d), generator=g).to(torch.bfloat16).cuda()
    prob = api.make_problem(n, d, 1, 1, 64, 0, 0.0, "bf16")
    i32 = dict(dtype=torch.int32, device="cuda")
    seg_off = torch.tensor([0, n], **i32)
    perm = torch.arange(n, **i32)
    delta = torch.zeros(1, dtype=torch.int64, device="cuda")
    recv = torch.tensor([buf.ptr], dtype=torch.int64, device="cuda")
    api.moe_ep_scatter(prob, 1, x, perm, seg_off, recv, delta)
    torch.cuda.synchronize()
    buf.release()
    return 0


if __name__ == "__main__":
    sys.exit(main())
