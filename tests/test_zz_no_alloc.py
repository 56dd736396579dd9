"""lazy_decode_attn_noalloc: the decode step for callers that cannot allocate.

Some callers of this library have no device allocator to take a workspace
from (a plugin given only its input and output buffers), or must keep
cudaMalloc off their hot path because it synchronises the device.  For them
the library keeps the split-K partials in a fixed array of its own.  These
tests call that entry point through the C ABI and check it against the
workspace-taking lazy_decode_attn, on two calls in a row, so that a call
cannot depend on what an earlier call left in the shared array.  The file is
named to run last, after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from position_agnostic_paged_b200 import lazy_attn as la
from position_agnostic_paged_b200 import workloads as W
from position_agnostic_paged_b200.runner import DevicePool, DeviceStep

MAX_ABS = 1e-2
REL_L2 = 5e-3


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    err = np.abs(a - b)
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert err.max() <= MAX_ABS and rel <= REL_L2, f"max_abs={err.max():.3e} rel_l2={rel:.3e}"


def test_capacity_is_reported_and_oversized_batches_are_refused():
    cap = la.decode_noalloc_capacity()
    assert cap == 16 << 20
    cfg = la.Cfg(64, 8)
    c = cfg.c()
    # a batch whose split partials need more than the array holds is refused
    # on the host, before any launch (the pointers below are never used)
    num_req, max_words = 4096, 1033
    assert la.decode_workspace_bytes(cfg, num_req, max_words) > cap
    rc = la._lib.lazy_decode_attn_noalloc(ctypes.byref(c), 1, 1, num_req, 1, 1, max_words, 1, 1, 1, 1000, 1,
                                          None, None)
    assert rc == la.LAZY_ERANGE


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    results = []
    for name in ("decode_8b", "tiny"):
        wl = W.make(name)
        pool = DevicePool(wl).setup()
        step = [s for s in wl.steps if s.kind == "decode"][0]
        ds = DeviceStep(pool, step)
        ds.write_new_tokens()
        assert la.decode_workspace_bytes(ds.cfg, step.num_req, ds.max_words) <= la.decode_noalloc_capacity()
        ds.attend()
        ref = ds.out.clone()
        out = torch.full_like(ds.out, float("nan"))
        la.decode_attn_noalloc(ds.cfg, ds.q_raw, ds.q_pos, ds.table, ds.table_indptr, ds.max_words,
                               pool.blk_meta, pool.k_pool, pool.v_pool, out, pool.d_status)
        torch.cuda.synchronize()
        assert pool.status() == 0
        _close(out, ref)
        results.append(name)
    assert results == ["decode_8b", "tiny"]
