"""Programmatic dependent launch: the forward path's kernels are launched so that each may set up
(barriers, TMEM, tensor-map prefetch) while the previous kernel on the stream drains, and wait
for that kernel's completion before touching memory.  A rollout run that way (eager calls and
CUDA-graph replays) must give exactly the results of plain launches (MLA_NO_PDL=1), which this
test runs in a child process since the library reads the switch once per process."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
import numpy as np
import torch
from mla_latent_kv_attn_b200 import api, inputs, rollout

cfg = inputs.small_bf16_config()
c = api.make_config(cfg)
w = rollout.upload_weights(c, inputs.layer_weights(cfg, 0))
ring, buf = rollout.Ring(c), rollout.ChunkBuffers(c)
outs, lses = [], []
for ch in range(cfg.n_chunks):
    buf.x.copy_(torch.from_numpy(inputs.chunk_x(cfg, ch)).to(torch.bfloat16))
    if ch < 2:
        o = rollout.run_chunk(c, w, ring, buf, ch, fused_q=True)
    else:
        o = rollout.ChunkGraph(c, w, ring, buf, ch, fused_q=True).replay()
    outs.append(o.float().cpu().numpy())
    lses.append(buf.lse.cpu().numpy())
torch.cuda.synchronize()
rollout.check_device_status(buf)
np.savez(sys.argv[1], o=np.stack(outs), lse=np.stack(lses), cache=ring.cache.float().cpu().numpy(),
         slot_frame=ring.slot_frame.cpu().numpy())
"""


def _run(path, extra_env):
    env = {k: v for k, v in os.environ.items() if k != "MLA_NO_PDL"}
    env.update(extra_env)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", CHILD, str(path)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    return np.load(path)


def test_programmatic_and_plain_launches_agree(tmp_path):
    a = _run(tmp_path / "pdl.npz", {})
    b = _run(tmp_path / "plain.npz", {"MLA_NO_PDL": "1"})
    for k in ("o", "lse", "cache", "slot_frame"):
        assert np.array_equal(a[k], b[k]), k
