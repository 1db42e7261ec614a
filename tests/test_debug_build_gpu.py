"""The MLA_DEBUG build of the library (libmla_b200_debug.so, built beside the release library by
__graft_entry__.build()): its device-side contract checks report through dev_status and never
trap.  The attention call walks ring slots 0 .. n_valid_frames*tpf - 1 and takes each slot's frame
from slot_frame; a slot whose frame is empty or outside the chunk's window breaks the window rule
the caller promised (the pages' fixed window of the most recent frames).  The debug build writes
MLA_ERR_DEVICE_CHECK for it; the release build does not check.  On valid inputs both builds give
bit-identical results."""
import ctypes

import numpy as np
import pytest
import torch

from mla_latent_kv_attn_b200 import _lib, api, inputs
from parity_util import GpuRun

pytestmark = pytest.mark.gpu


def debug_lib():
    lib = ctypes.CDLL(_lib.DEBUG_LIB_PATH)
    for name, (res, args) in _lib.SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def attend(lib, g: GpuRun, chunk: int, slot_frame, out, status):
    cfg = g.cfg
    first = cfg.first_frame(chunk)
    n_valid = min(first, cfg.window_frames)
    b = g.buf
    status.zero_()
    st = lib.mla_attention_fwd(ctypes.byref(g.c), b.q.data_ptr(), b.chunk_lat.data_ptr(),
                               g.ring.cache.data_ptr(), slot_frame.data_ptr(), n_valid, first,
                               None, out.data_ptr(), None, b.workspace.data_ptr(),
                               b.workspace.numel(), status.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    return int(status.item())


@pytest.mark.parametrize("cfg_id", ["toy", "small"])
def test_debug_build_reports_a_slot_outside_the_window(cfg_id):
    cfg = inputs.CONFIGS[0] if cfg_id == "toy" else inputs.small_bf16_config()
    g = GpuRun(cfg)
    chunk = cfg.window_frames // cfg.chunk_frames + 1          # the window is full
    for ch in range(chunk):
        g.prefill(ch, inputs.chunk_x(cfg, ch))
    g.load_x(inputs.chunk_x(cfg, chunk))
    first = cfg.first_frame(chunk)
    api.mla_project_chunk(g.c, g.buf.x, g.w.w_x, g.w.w_qcat, g.buf.c_q, g.buf.q, g.buf.chunk_lat,
                          first)
    dbg, rel = debug_lib(), _lib.lib()
    status = torch.zeros(1, device="cuda", dtype=torch.int32)
    out_rel = torch.empty_like(g.buf.o_lat)
    out_dbg = torch.full_like(g.buf.o_lat, float("nan"))
    # valid inputs: no report, and the debug build computes exactly what the release build does
    assert attend(rel, g, chunk, g.ring.slot_frame, out_rel, status) == 0
    assert attend(dbg, g, chunk, g.ring.slot_frame, out_dbg, status) == 0
    assert torch.equal(out_dbg, out_rel)
    # a slot holding a frame newer than the chunk, and one holding no frame at all
    for bad in (first + 5, -1):
        sf = g.ring.slot_frame.clone()
        sf[0, 0] = bad
        assert attend(dbg, g, chunk, sf, out_dbg, status) == _lib.MLA_ERR_DEVICE_CHECK
        assert attend(rel, g, chunk, sf, out_rel, status) == 0        # release: no checks
    # the context is still usable after the reports
    assert attend(dbg, g, chunk, g.ring.slot_frame, out_dbg, status) == 0
    assert np.isfinite(out_dbg.float().cpu().numpy()).all()
