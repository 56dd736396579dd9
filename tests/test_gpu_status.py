"""Device-side status reporting: every LAZY_DSTATUS_* bit is raised by the case it names, the
affected unit of work is skipped, and everything else is unaffected.  Nothing here faults or
hangs a GPU: bad slots and tables are checked by the kernels before any access, and the timeout
case waits on a barrier that nothing completes, with a small poll limit."""
import numpy as np
import pytest
import torch

import oracle
from position_agnostic_paged_b200 import lazy_attn as la
from tests._cases import make_case
from tests._gpu_cases import DeviceCase

pytestmark = pytest.mark.gpu


def _bf16(rng, shape):
    return (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _dev_bf16(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


def _write(tokens_slot, tokens_j, nb=6, hkv=2, seed=5):
    """kv_write of len(tokens_slot) random tokens into sentinel-filled pools; returns the pools,
    metadata and status (host) and the inputs."""
    rng = np.random.default_rng(seed)
    n = len(tokens_slot)
    k, v = _bf16(rng, (n, hkv, 128)), _bf16(rng, (n, hkv, 128))
    cfg = la.Cfg(hkv * 4, hkv)
    kp = torch.full((nb, hkv, 16, 128), 0x1234, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    vp = torch.full_like(kp, 0)
    vp.view(torch.int16).fill_(0x4321)
    meta = torch.zeros(nb, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    la.kv_write(cfg, _dev_bf16(k), _dev_bf16(v), torch.tensor(tokens_slot, dtype=torch.int32, device="cuda"),
                torch.tensor(tokens_j, dtype=torch.int32, device="cuda"), kp, vp, meta, st)
    torch.cuda.synchronize()
    u16 = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    return u16(kp), u16(vp), meta.cpu().numpy().view(np.uint32), int(st.item()), k, v


def test_kv_write_slot_outside_the_pool_is_reported_and_skipped():
    nb = 6
    slots = [3, nb * 16, 17, -1, nb * 16 + 5]          # two good tokens, three outside the pool
    js = [3, 0, 1, 0, 5]
    kp, vp, meta, st, k, v = _write(slots, js, nb=nb)
    assert st & la.DSTATUS_BAD_SLOT and not st & la.DSTATUS_BAD_ALIGN
    written = np.zeros((nb, 16), bool)
    written[0, 3] = written[1, 1] = True
    # the good tokens landed: values verbatim, keys j = 3 / 1 rotated (checked against the oracle)
    okp = np.zeros_like(kp)
    ovp = np.zeros_like(vp)
    ometa = np.zeros(nb, np.uint32)
    oracle.kv_write(k[[0, 2]], v[[0, 2]], np.array([3, 17], np.int32), np.array([3, 1], np.int32), okp, ovp, ometa,
                    500000.0)
    assert np.array_equal(vp[0, :, 3], v[0]) and np.array_equal(vp[1, :, 1], v[2])
    assert np.abs(kp[0, :, 3].astype(np.int32) - okp[0, :, 3].astype(np.int32)).max() <= 1
    assert np.array_equal(meta, ometa)
    # every other slot keeps its sentinel
    ks, vs = kp.transpose(0, 2, 1, 3), vp.transpose(0, 2, 1, 3)
    assert (ks[~written] == 0x1234).all() and (vs[~written] == 0x4321).all()


def test_kv_write_misaligned_local_index_is_reported_and_skipped():
    nb = 4
    slots = [16 + 2, 32 + 7, 5]
    js = [2, 8, 21]                                    # 7 != 8 (mod 16) and 5 == 21 (mod 16)
    kp, vp, meta, st, k, v = _write(slots, js, nb=nb)
    assert st & la.DSTATUS_BAD_ALIGN and not st & la.DSTATUS_BAD_SLOT
    assert np.array_equal(vp[1, :, 2], v[0]) and np.array_equal(vp[0, :, 5], v[2])
    # the misaligned token wrote nothing: its slot and its block's metadata are untouched
    assert (kp[2, :, 7] == 0x1234).all() and (vp[2, :, 7] == 0x4321).all()
    assert meta[2] == 0
    assert meta[1] == ((2 // 16) << 8 | 3) and meta[0] == ((21 // 16) << 8 | 6)


def _two_requests():
    reqs = [([(0, 0, 90), (100, 90, 70)], [159]), ([(200, 0, 40)], [39])]
    return make_case(33, hq=16, hkv=4, d=128, requests=reqs)


def test_decode_request_with_more_words_than_max_words():
    case = _two_requests()
    dc = DeviceCase(case)
    good = dc.decode()
    assert dc.status() == 0
    n0 = int(dc.table_indptr[1] - dc.table_indptr[0])
    assert n0 > dc.max_words - 1 >= 3
    dc.max_words -= 1                                  # request 0 now has more words than announced
    out = dc.decode()
    assert dc.status() & la.DSTATUS_BAD_TABLE
    np.testing.assert_array_equal(out[16:], good[16:])   # request 1 (within the bound) unaffected


@pytest.mark.parametrize("split", [True, False])
def test_prefill_request_with_more_words_than_max_words(split):
    reqs = [([(0, 0, 90), (100, 90, 70)], list(range(150, 170))), ([(200, 0, 40)], list(range(30, 40)))]
    case = make_case(34, hq=16, hkv=4, d=128, requests=reqs)
    dc = DeviceCase(case)
    good = dc.prefill(split=split)
    assert dc.status() == 0
    dc.max_words -= 1
    out = dc.prefill(split=split)
    assert dc.status() & la.DSTATUS_BAD_TABLE
    # the prefill walks each request's own words, so the output itself is still complete
    np.testing.assert_array_equal(out, good)


@pytest.mark.parametrize("polls", [300, 4000])
def test_bounded_wait_runs_out_and_reports_timeout(polls):
    result = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    la.debug_bounded_wait(polls, False, result, st)
    torch.cuda.synchronize()
    assert result.tolist() == [1, 1]                   # the wait gave up; the other role left on the flag
    assert int(st.item()) == la.DSTATUS_TIMEOUT
    # the context is still usable: a completed barrier is waited on normally afterwards
    st.zero_()
    la.debug_bounded_wait(polls, True, result, st)
    torch.cuda.synchronize()
    assert result.tolist() == [0, 0] and int(st.item()) == 0
