"""Failure detection without a GPU fault: a bounded wait that runs out.

The test build of the library (libmla_testhook.so, define MLA_TEST_DROP_ARRIVE) leaves out one
K-slab load of the attention kernel's first work range. The MMA warp's wait for that slab can
never complete; it must give up after its 1 s limit, set MLA_DEV_WAIT_TIMEOUT in the device
error word, drain what was issued, free its tensor memory and return, leaving the CUDA context
usable. The run happens in a child process so that the test library does not replace the
normal one in this process.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys, time
sys.path.insert(0, ROOT)
import torch
import mla_latent_kv_44_b200 as mla
mla.LIB_PATH = mla.TEST_LIB_PATH
H, r, dr, bs, L = 128, 512, 64, 64, 2048
dev = "cuda"
g = torch.Generator(device=dev); g.manual_seed(0)
nblk = L // bs
pool = torch.randn((nblk, bs, r + dr), generator=g, device=dev).to(torch.bfloat16)
table = torch.arange(nblk, dtype=torch.int32, device=dev).reshape(1, nblk)
q = (0.25 * torch.randn((1, H, r + dr), generator=g, device=dev)).to(torch.bfloat16)
lens = torch.tensor([L], dtype=torch.int32, device=dev)
cfg = mla.Config(num_heads=H, head_dim=128, kv_rank=r, rope_dim=dr, block_size=bs,
                 dtype="bf16", decode_kernel=mla.DECODE_TENSOR)
ws = torch.empty(mla.decode_workspace_size(cfg, 1, 1), dtype=torch.uint8, device=dev)
out = torch.empty((1, H, r), device=dev); lse = torch.empty((1, H), device=dev)
res = []
for attempt in range(2):
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    t0 = time.time()
    mla.decode(cfg, q, pool, table, lens, 1, ws, out, lse, err)
    torch.cuda.synchronize()
    res.append({"err": int(err.item()), "seconds": time.time() - t0})
x = float(torch.ones(1000, device=dev).sum().item())
print(json.dumps({"runs": res, "after": x}))
""".replace("ROOT", repr(ROOT))


@pytest.mark.gpu
def test_dropped_slab_times_out_and_the_context_stays_usable():
    import mla_latent_kv_44_b200 as mla

    assert os.path.exists(mla.TEST_LIB_PATH), "build the libraries first"
    p = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, timeout=180)
    assert p.returncode == 0, p.stderr[-2000:]
    out = json.loads(p.stdout.strip().splitlines()[-1])
    for run in out["runs"]:
        assert run["err"] & mla.DEV_WAIT_TIMEOUT, run
        assert run["err"] & ~(mla.DEV_WAIT_TIMEOUT) == 0, run
        assert run["seconds"] < 30, run      # a few 1 s limits, not a hang
    assert out["after"] == 1000.0
