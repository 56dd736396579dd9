"""lazy_decode_attn_noalloc: the decode step for callers that cannot allocate.

Some callers of this library have no device allocator to take a workspace
from (a plugin given only its input and output buffers), or must keep
cudaMalloc off their hot path because it synchronises the device.  For them
the library keeps the split-K partials in a fixed array of its own.  These
tests call that entry point through the C ABI and check it against the
workspace-taking lazy_decode_attn, which runs the same kernels with the same
split plan, so the outputs must be equal bit for bit: on two calls in a row,
and on a ragged batch right after a large one, so that a call cannot depend
on what an earlier call left in the shared array.  The file is named to run
last, after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from position_agnostic_paged_b200 import lazy_attn as la
from position_agnostic_paged_b200 import workloads as W
from position_agnostic_paged_b200.runner import DevicePool, DeviceStep


def _words(doc_tokens, question_tokens):
    return sum((n + 15) // 16 for n in doc_tokens) + (question_tokens + 15) // 16


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


def test_the_benchmark_decode_shapes_fit_the_array():
    """The decode steps of the benchmark workloads fit the array: decode 8B (64 requests, 8 documents
    of 512 tokens and a 64-token question plus the new token), decode 70B and its uniform variant
    (128 requests, 32 x 512 + 128 + 1), and the mixed 8B step's decodes (192 requests, 8 documents
    of at most 2048 tokens + 64 + 1).  The MQA variant of the mixed step does not fit: its 192
    requests with one KV head run on the tensor-memory decode kernel as 4 CTAs of two softmax
    streams each, 8 partials of 32 query heads per request (about 26 MB), and the entry point
    refuses it before launching anything."""
    cap = la.decode_noalloc_capacity()
    shapes = [(la.Cfg(32, 8), 64, _words([512] * 8, 65)),
              (la.Cfg(64, 8), 128, _words([512] * 32, 129)),
              (la.Cfg(32, 8), 192, _words([2048] * 8, 65))]
    for cfg, num_req, max_words in shapes:
        need = la.decode_workspace_bytes(cfg, num_req, max_words)
        assert 0 < need <= cap, (cfg, num_req, max_words, need)
    mqa = la.Cfg(32, 1)
    num_req, max_words = 192, _words([2048] * 8, 65)
    assert la.decode_workspace_bytes(mqa, num_req, max_words) > cap
    c = mqa.c()
    assert la._lib.lazy_decode_attn_noalloc(ctypes.byref(c), 1, 1, num_req, 1, 1, max_words, 1, 1, 1, 1000, 1,
                                            None, None) == la.LAZY_ERANGE


def _decode_step(name):
    wl = W.make(name)
    pool = DevicePool(wl).setup()
    step = [s for s in wl.steps if s.kind == "decode"][0]
    ds = DeviceStep(pool, step)
    ds.write_new_tokens()
    return pool, ds


def _both(pool, ds):
    """The workspace entry point's output and the no-alloc entry point's output, same inputs."""
    assert la.decode_workspace_bytes(ds.cfg, ds.step.num_req, ds.max_words) <= la.decode_noalloc_capacity()
    ds.attend()
    ref = ds.out.clone()
    out = torch.full_like(ds.out, float("nan"))
    la.decode_attn_noalloc(ds.cfg, ds.q_raw, ds.q_pos, ds.table, ds.table_indptr, ds.max_words,
                           pool.blk_meta, pool.k_pool, pool.v_pool, out, pool.d_status)
    torch.cuda.synchronize()
    assert pool.status() == 0
    return ref, out


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    results = []
    for name in ("decode_8b", "tiny"):
        pool, ds = _decode_step(name)
        ref, out = _both(pool, ds)
        assert torch.equal(out, ref), name
        results.append(name)
    assert results == ["decode_8b", "tiny"]


@pytest.mark.gpu
def test_ragged_batch_after_a_large_call_reads_no_stale_partials():
    """A batch whose requests are far shorter than max_words (most of their splits are empty, and
    empty splits must still write their own partials) right after a large call that filled the
    array: equal bit for bit to the workspace entry point."""
    from tests._cases import make_case
    from tests._gpu_cases import DeviceCase

    pool, ds = _decode_step("decode_8b")
    ref, out = _both(pool, ds)
    assert torch.equal(out, ref)
    reqs = [([(0, 0, 1000)], [999]), ([(1000, 0, 20)], [19]), ([(1020, 7, 3)], [9]),
            ([(1023, 100, 130), (1200, 230, 40)], [269])]
    case = make_case(17, hq=32, hkv=8, d=128, requests=reqs)
    dc = DeviceCase(case)
    assert la.decode_workspace_bytes(dc.cfg, 4, dc.max_words) <= la.decode_noalloc_capacity()
    want = torch.from_numpy(dc.decode()).float()
    q = torch.from_numpy(case.q_raw.view(np.int16)).cuda().view(torch.bfloat16)
    qp = torch.from_numpy(case.q_pos.astype(np.int32)).cuda()
    got = torch.full((4, 32, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    la.decode_attn_noalloc(dc.cfg, q, qp, dc.table, dc.table_indptr, dc.max_words, dc.blk_meta, dc.k_pool,
                           dc.v_pool, got, dc.d_status)
    torch.cuda.synchronize()
    assert dc.status() == 0
    assert torch.equal(got.float().cpu().reshape(-1, 128), want)
